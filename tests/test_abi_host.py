"""Host-side checks of the C ABI that need no GPU: the library builds and
loads, exports every function include/csa.h declares, and rejects bad
arguments before any CUDA call."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared_functions():
    names = []
    for fn in os.listdir(os.path.join(ROOT, "include")):
        if not fn.endswith(".h"):
            continue
        src = open(os.path.join(ROOT, "include", fn)).read()
        src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
        names += re.findall(r"^\s*[A-Za-z_][\w \*]*?\b(\w+)\s*\(", src, flags=re.M)
    return sorted(set(n for n in names if n not in ("defined",)))


@pytest.fixture(scope="module")
def L():
    from long_context_attention_csa_b200 import build, lib

    build.build()
    return lib()


def test_every_declared_symbol_is_exported(L):
    names = _declared_functions()
    assert {"csa_compress", "hca_compress", "indexer_scores_topk", "sparse_mqa_attn",
            "dense_hca_attn"} <= set(names)
    for n in names:
        assert hasattr(L, n), f"libcsa.so does not export {n}"


def test_binding_names_match_the_abi():
    import long_context_attention_csa_b200 as pkg

    for n in ("csa_compress", "hca_compress", "indexer_scores_topk", "sparse_mqa_attn",
              "dense_hca_attn", "csa_workspace_bytes", "csa_check_status"):
        assert callable(getattr(pkg, n))


def test_status_strings(L):
    for s in range(6):
        assert len(L.csa_status_string(s)) > 0


def test_workspace_sizes(L):
    from long_context_attention_csa_b200 import CSA_OP_INDEXER, CSA_OP_SPARSE_ATTN

    # at least the status word; scales with the problem
    a = L.csa_workspace_bytes(CSA_OP_INDEXER, 1, 1, 16, 0, 0, 64, 8, 0)
    b = L.csa_workspace_bytes(CSA_OP_INDEXER, 1, 1, 1024, 0, 0, 4096, 8, 0)
    assert 256 <= a < b
    assert L.csa_workspace_bytes(CSA_OP_SPARSE_ATTN, 1, 1, 8, 64, 512, 2048, 512, 128) >= 256
    assert L.csa_workspace_bytes(99, 1, 1, 1, 1, 1, 1, 1, 1) == 0


def test_indexer_workspace_follows_the_selection_scheme(L):
    """bf16 indexer scratch: none for one chunk; for single-token rows of 2 to
    16 chunks of 4096 the raw score rows (the merge selects among them);
    beyond, and for multi-token rows (chunks of 2048), the chunks' top-k
    candidates (score and index)."""
    from long_context_attention_csa_b200 import CSA_OP_INDEXER, CSA_OP_INDEXER_MX

    def ws(B, Tq, N, k, op=CSA_OP_INDEXER):
        return L.csa_workspace_bytes(op, 1, B, Tq, 0, 0, N, k, 0) - 256

    assert ws(3, 1, 4096, 1024) == 0
    assert ws(3, 1, 4097, 1024) == 3 * 2 * 4096 * 4
    assert ws(2, 1, 16 * 4096, 1024) == 2 * 16 * 4096 * 4
    assert ws(2, 1, 16 * 4096 + 1, 1024) == 2 * 17 * 1024 * 8
    assert ws(1, 3, 30000, 512) == 3 * 8 * 4096 * 4
    assert ws(1, 4, 30000, 512) == 4 * 15 * 512 * 8      # 2048-entry chunks, candidates
    assert ws(1, 8, 2048, 512) == 0
    # the MX-FP8 / MX-FP4 calls take single-token units at any Tq
    assert ws(3, 1, 4097, 1024, CSA_OP_INDEXER_MX) == 3 * 2 * 4096 * 4
    assert ws(2, 1, 16 * 4096 + 1, 1024, CSA_OP_INDEXER_MX) == 2 * 17 * 1024 * 8
    assert ws(1, 5, 30000, 64, CSA_OP_INDEXER_MX) == 5 * 8 * 4096 * 4


def _fmt(c=512, r=64, flags=0):
    from long_context_attention_csa_b200 import Fmt

    return Fmt(c=c, rope_dims=r, flags=flags)._c()


def test_compress_rejects_bad_arguments(L):
    f = _fmt()
    dummy = ctypes.c_void_p(4096)   # never dereferenced: validation fails first
    mis = ctypes.c_void_p(4100)     # not 16-byte aligned
    # bad dtype, null fmt, bad m, null pointers, misalignment, bad z_cols
    assert L.csa_compress(7, 1, 64, 4, ctypes.byref(f), dummy, dummy, dummy, dummy, 512, 0, dummy,
                          None, None, 0, None) == 1
    assert L.csa_compress(1, 1, 64, 4, None, dummy, dummy, dummy, dummy, 512, 0, dummy, None,
                          None, 0, None) == 1
    assert L.csa_compress(1, 1, 64, 0, ctypes.byref(f), dummy, dummy, dummy, dummy, 512, 0, dummy,
                          None, None, 0, None) == 1
    assert L.csa_compress(1, 1, 64, 4, ctypes.byref(f), None, dummy, dummy, dummy, 512, 0, dummy,
                          None, None, 0, None) == 1
    assert L.csa_compress(1, 1, 64, 4, ctypes.byref(f), mis, dummy, dummy, dummy, 512, 0, dummy,
                          None, None, 0, None) == 1
    assert L.csa_compress(1, 1, 64, 4, ctypes.byref(f), dummy, dummy, dummy, dummy, 7, 0, dummy,
                          None, None, 0, None) == 1
    # odd RoPE dims, RoPE wider than c
    bad = _fmt(r=63)
    assert L.csa_compress(1, 1, 64, 4, ctypes.byref(bad), dummy, dummy, dummy, dummy, 512, 0,
                          dummy, None, None, 0, None) == 1
    bad = _fmt(c=64, r=128)
    assert L.csa_compress(1, 1, 64, 4, ctypes.byref(bad), dummy, dummy, dummy, dummy, 64, 0,
                          dummy, None, None, 0, None) == 1
    # unsupported: c not a power-of-two number of vectors, overlap too wide
    odd = _fmt(c=520, r=64)
    assert L.csa_compress(1, 1, 64, 4, ctypes.byref(odd), dummy, dummy, dummy, dummy, 520, 0,
                          dummy, None, None, 0, None) == 2
    assert L.csa_compress(1, 1, 1024, 200, ctypes.byref(f), dummy, dummy, dummy, dummy, 512, 0,
                          dummy, None, None, 0, None) == 2
    # empty problems are a no-op
    assert L.csa_compress(1, 0, 64, 4, ctypes.byref(f), None, None, None, None, 512, 0, None, None,
                          None, 0, None) == 0
    assert L.hca_compress(1, 1, 0, 128, ctypes.byref(f), None, None, 512, 0, None, None,
                          None, 0, None) == 0
    # a launchable problem without (or with too small) a workspace
    assert L.csa_compress(1, 1, 64, 4, ctypes.byref(f), dummy, dummy, dummy, dummy, 512, 0, dummy,
                          None, None, 0, None) == 5
    assert L.hca_compress(1, 1, 256, 128, ctypes.byref(f), dummy, dummy, 512, 0, dummy, None,
                          dummy, 255, None) == 5
    assert L.csa_workspace_bytes(4, 1, 1, 64, 0, 0, 0, 0, 0) == 256


def test_indexer_and_attention_reject_bad_arguments(L):
    d = ctypes.c_void_p(4096)
    f = _fmt()
    # indexer: H_I too large, k < 1, missing workspace, workspace too small
    assert L.indexer_scores_topk(1, 1, 4, 65, 128, d, d, d, 16, None, 4, 2, d, None, d, 1 << 20,
                                 None) == 2
    assert L.indexer_scores_topk(1, 1, 4, 64, 128, d, d, d, 16, None, 4, 0, d, None, d, 1 << 20,
                                 None) == 1
    assert L.indexer_scores_topk(1, 1, 4, 64, 128, d, d, d, 16, None, 4, 2, d, None, None, 0,
                                 None) == 5
    assert L.indexer_scores_topk(1, 1, 4, 64, 128, d, d, d, 16, None, 4, 2, d, None, d, 8,
                                 None) == 5
    # attention: idx null with k > 0, negative sizes, c > 512, no workspace
    assert L.sparse_mqa_attn(1, 1, 1, 64, ctypes.byref(f), d, None, d, 16, None, 4, d, 8, None,
                             8, None, 0.0, d, d, 1 << 20, None) == 1
    assert L.sparse_mqa_attn(1, 1, 1, 0, ctypes.byref(f), d, None, d, 16, d, 4, d, 8, None, 8,
                             None, 0.0, d, d, 1 << 20, None) == 1
    big = _fmt(c=1024)
    assert L.dense_hca_attn(1, 1, 1, 64, ctypes.byref(big), d, None, d, 16, 128, d, 8, None, 8,
                            None, 0.0, d, d, 1 << 20, None) == 2
    assert L.dense_hca_attn(1, 1, 1, 64, ctypes.byref(f), d, None, d, 16, 128, d, 8, None, 8,
                            None, 0.0, d, None, 0, None) == 5
    assert L.dense_hca_attn(1, 1, 1, 64, ctypes.byref(f), d, None, d, 16, 0, d, 8, None, 8, None,
                            0.0, d, d, 1 << 20, None) == 1


def test_selftest_wait_rejects_bad_arguments(L):
    """The failure-path self test checks its arguments before any CUDA call."""
    import ctypes
    buf = (ctypes.c_uint8 * 256)()
    assert L.csa_selftest_wait(10 ** 6, None, 256, None) == 1             # null workspace
    assert L.csa_selftest_wait(10 ** 6, ctypes.addressof(buf), 128, None) == 1   # too small
    assert L.csa_selftest_wait(10, ctypes.addressof(buf), 256, None) == 1        # limit too short
    assert L.csa_selftest_wait(10 ** 11, ctypes.addressof(buf), 256, None) == 1  # too long


def test_bf16_shapes_outside_the_tensor_core_kernels_are_unsupported(L):
    """bf16 indexer and attention calls run on the tensor cores only; a shape
    that kernel does not implement is rejected (no silent CUDA-core path).
    float32, and attention with CSA_F_PORTABLE, pass validation (they then
    stop here at the missing workspace)."""
    d = ctypes.c_void_p(4096)
    mis = ctypes.c_void_p(4100)
    # indexer: H_I = 32 or d_I = 64 in bf16 -> unsupported; the same in float32 -> workspace
    assert L.indexer_scores_topk(1, 1, 8, 32, 128, d, d, d, 64, None, 4, 8, d, None, None, 0,
                                 None) == 2
    assert L.indexer_scores_topk(1, 1, 8, 64, 64, d, d, d, 64, None, 4, 8, d, None, None, 0,
                                 None) == 2
    assert L.indexer_scores_topk(0, 1, 8, 32, 128, d, d, d, 64, None, 4, 8, d, None, None, 0,
                                 None) == 5
    # the supported bf16 shape passes validation; misaligned inputs are argument errors
    assert L.indexer_scores_topk(1, 1, 8, 64, 128, d, d, d, 64, None, 4, 8, d, None, None, 0,
                                 None) == 5
    assert L.indexer_scores_topk(1, 1, 8, 64, 128, mis, d, d, 64, None, 4, 8, d, None, None, 0,
                                 None) == 1
    # the no-workspace variant applies the same rule
    assert L.indexer_scores_topk_noalloc(1, 1, 8, 32, 128, d, d, d, 64, None, 4, 8, d, None,
                                         None) == 2
    # attention: 32 heads or 48 RoPE dims are fine, 32 heads is not a multiple of 64
    f = _fmt()
    assert L.sparse_mqa_attn(1, 1, 4, 32, ctypes.byref(f), d, None, d, 16, d, 4, d, 8, None, 8,
                             None, 0.0, d, None, 0, None) == 2
    assert L.dense_hca_attn(1, 1, 4, 32, ctypes.byref(f), d, None, d, 16, 4, d, 8, None, 8,
                            None, 0.0, d, None, 0, None) == 2
    # c = 256 in bf16 -> unsupported; CSA_F_PORTABLE selects the CUDA-core kernel instead
    f256 = _fmt(c=256)
    assert L.dense_hca_attn(1, 1, 4, 64, ctypes.byref(f256), d, None, d, 16, 4, d, 8, None, 8,
                            None, 0.0, d, None, 0, None) == 2
    fp = _fmt(c=256, flags=4)
    assert L.dense_hca_attn(1, 1, 4, 64, ctypes.byref(fp), d, None, d, 16, 4, d, 8, None, 8,
                            None, 0.0, d, None, 0, None) == 5
    # top-k beyond the tensor-core kernel's index list
    assert L.sparse_mqa_attn(1, 1, 4, 64, ctypes.byref(f), d, None, d, 4096, d, 2048, d, 8, None,
                             8, None, 0.0, d, None, 0, None) == 2
    # float32 attention always takes the CUDA-core kernel
    f64c = _fmt(c=64, r=32)
    assert L.dense_hca_attn(0, 1, 4, 4, ctypes.byref(f64c), d, None, d, 16, 4, d, 8, None, 8,
                            None, 0.0, d, None, 0, None) == 5



def test_stream_append_rejects_bad_arguments(L):
    """The streaming compression calls check their arguments before any CUDA
    call; the state size follows the documented layout."""
    f = _fmt()
    d = ctypes.c_void_p(4096)
    mis = ctypes.c_void_p(4100)
    need = L.csa_stream_state_bytes(1, 4, 1, 512, 512)
    assert need == ((16 + 3 * 4 * (512 + 512) * 2 + 255) // 256) * 256
    assert L.csa_stream_state_bytes(1, 128, 0, 512, 1) == ((16 + 128 * 513 * 2 + 255) // 256) * 256
    assert L.csa_stream_state_bytes(1, 4, 1, 512, 7) == 0
    # stride too small / not a multiple of 16, misaligned state, bad z_cols, m too large
    assert L.csa_compress_append(1, 2, 4, ctypes.byref(f), d, d, d, d, 512, 0, d, need - 16, d, 8,
                                 None, d, 256, None) == 1
    assert L.csa_compress_append(1, 2, 4, ctypes.byref(f), d, d, d, d, 512, 0, d, need + 8, d, 8,
                                 None, d, 256, None) == 1
    assert L.csa_compress_append(1, 2, 4, ctypes.byref(f), d, d, d, d, 512, 0, mis, need, d, 8,
                                 None, d, 256, None) == 1
    assert L.csa_compress_append(1, 2, 4, ctypes.byref(f), d, d, d, d, 3, 0, d, need, d, 8,
                                 None, d, 256, None) == 1
    assert L.csa_compress_append(1, 2, 200, ctypes.byref(f), d, d, d, d, 512, 0, d, 1 << 30, d,
                                 8, None, d, 256, None) == 2
    # group b missing for CSA; missing workspace; empty batch is a no-op
    assert L.csa_compress_append(1, 2, 4, ctypes.byref(f), d, None, d, d, 512, 0, d, need, d, 8,
                                 None, d, 256, None) == 1
    assert L.csa_compress_append(1, 2, 4, ctypes.byref(f), d, d, d, d, 512, 0, d, need, d, 8,
                                 None, None, 0, None) == 5
    assert L.hca_compress_append(1, 0, 128, ctypes.byref(f), None, None, 512, 0, None, 0, None, 0,
                                 None, None, 0, None) == 0


def test_projection_rejects_bad_arguments(L):
    d = ctypes.c_void_p(4096)
    # float32, heads not divisible by groups, group width not a multiple of 64 -> unsupported
    assert L.grouped_output_projection(0, 8, 16, 512, 4, 256, 512, d, d, d, d, d, 1 << 30,
                                       None) == 2
    assert L.grouped_output_projection(1, 8, 16, 512, 3, 256, 512, d, d, d, d, d, 1 << 30,
                                       None) == 2
    assert L.grouped_output_projection(1, 8, 1, 96, 1, 256, 512, d, d, d, d, d, 1 << 30,
                                       None) == 2
    # null pointer, short workspace; empty is a no-op
    assert L.grouped_output_projection(1, 8, 16, 512, 4, 256, 512, None, d, d, d, d, 1 << 30,
                                       None) == 1
    need = L.csa_workspace_bytes(5, 1, 1, 8, 0, 0, 4 * 256, 0, 0)
    assert need == 256 + 8 * 1024 * 2
    assert L.grouped_output_projection(1, 8, 16, 512, 4, 256, 512, d, d, d, d, d, need - 1,
                                       None) == 5
    assert L.grouped_output_projection(1, 0, 16, 512, 4, 256, 512, None, None, None, None, None,
                                       0, None) == 0


def test_mxfp8_calls_reject_bad_arguments(L):
    d = ctypes.c_void_p(4096)
    mis = ctypes.c_void_p(4100)
    # quantize: rows of 64 are not the format, misaligned output, empty is a no-op
    assert L.indexer_mxfp8_quantize(1, 1, 8, 64, d, d, d, None) == 2
    assert L.indexer_mxfp8_quantize(1, 1, 8, 128, d, mis, d, None) == 1
    assert L.indexer_mxfp8_quantize(1, 0, 8, 128, None, None, None, None) == 0
    # scores: the tensor-core shape only, workspace required
    assert L.indexer_scores_topk_mxfp8(1, 1, 32, 128, d, d, d, d, d, 64, None, 4, 8, d, None, d,
                                       1 << 20, None) == 2
    assert L.indexer_scores_topk_mxfp8(1, 1, 64, 128, d, d, d, d, d, 64, None, 4, 8, d, None,
                                       None, 0, None) == 5
    assert L.indexer_scores_topk_mxfp8(1, 1, 64, 128, d, None, d, d, d, 64, None, 4, 8, d, None,
                                       d, 1 << 20, None) == 1
    # eight 4096-entry chunks a row: the raw score rows (one merge cluster holds a row)
    assert L.csa_workspace_bytes(6, 1, 32, 1, 0, 0, 32768, 1024, 0) == 256 + 32 * 8 * 4096 * 4


def test_mixed_storage_rejects_bad_arguments(L):
    d = ctypes.c_void_p(4096)
    assert L.csa_mixed_record_bytes(512, 64) == 592
    assert L.csa_mixed_record_bytes(64, 32) == 112
    assert L.csa_mixed_record_bytes(512, 60) == 0
    f = _fmt()
    bad = _fmt(r=60)
    assert L.csa_store_mixed(1, 1, 8, ctypes.byref(bad), d, d, None) == 2
    assert L.csa_store_mixed(1, 1, 8, ctypes.byref(f), None, d, None) == 1
    assert L.csa_store_mixed(1, 0, 8, ctypes.byref(f), None, None, None) == 0
    # attention under CSA_F_MIXED: (c - r) must be a multiple of 32
    fm = _fmt(r=60, flags=8)
    assert L.dense_hca_attn(1, 1, 4, 64, ctypes.byref(fm), d, None, d, 16, 4, d, 8, None, 8,
                            None, 0.0, d, None, 0, None) == 2


def test_mxfp4_calls_reject_bad_arguments(L):
    d = ctypes.c_void_p(4096)
    assert L.indexer_mxfp4_quantize(1, 1, 8, 64, d, d, d, None) == 2
    assert L.indexer_mxfp4_quantize(1, 0, 8, 128, None, None, None, None) == 0
    assert L.indexer_scores_topk_mxfp4(1, 1, 32, 128, d, d, d, d, d, 64, None, 4, 8, d, None, d,
                                       1 << 20, None) == 2
    assert L.indexer_scores_topk_mxfp4(1, 1, 64, 128, d, d, d, d, d, 64, None, 4, 8, d, None,
                                       None, 0, None) == 5

