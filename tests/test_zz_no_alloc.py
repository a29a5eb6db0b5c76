"""The allocation-free indexer entry point, called through the C ABI.

indexer_scores_topk_noalloc serves callers that cannot allocate device memory
at the call site (an engine plug-in whose host owns all device memory, or a
decode loop that must not pay for cudaMalloc).  It keeps its scratch in a
fixed device array inside the library.  Here it must return exactly what the
workspace-taking indexer_scores_topk returns, on two calls in a row (the
second call sees the array as the first call left it).  The file sorts last
so a run that stops at the first failure has run every other test first.
"""
import ctypes

import pytest
import torch

import long_context_attention_csa_b200 as csa
from long_context_attention_csa_b200 import workloads as wl

pytestmark = pytest.mark.gpu


def _noalloc(L, q_I, w, k_I, m, k, q_pos, idx, sc):
    B, Tq, HI, dI = q_I.shape
    N = k_I.shape[1]
    fn = L.indexer_scores_topk_noalloc
    P, i32, i64 = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64
    fn.argtypes = [i32, i64, i64, i32, i32, P, P, P, i64, P, i32, i32, P, P, P]
    fn.restype = i32
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    return fn(csa.CSA_BF16, B, Tq, HI, dI, P(q_I.data_ptr()), P(w.data_ptr()),
              P(k_I.data_ptr()), N, P(q_pos.data_ptr()), m, k, P(idx.data_ptr()),
              P(sc.data_ptr()), stream)


@pytest.mark.parametrize("seed", [0, 1])
def test_noalloc_matches_workspace_indexer_twice(seed):
    L = csa.lib()
    # decode rows over a 128K-token cache: the chunked tensor-core path, whose
    # per-chunk candidates live in the scratch array
    w = wl.scaled(wl.WORKLOADS["csa_decode_b32_128k"], B=8, seed=seed)
    outs = []
    for call in range(2):
        inp = wl.csa_decode_inputs(wl.scaled(w, seed=seed * 10 + call), "cuda")
        ref_idx, ref_sc = csa.indexer_scores_topk(inp["q_I"], inp["w"], inp["k_I"], w.m, w.k,
                                                  q_pos=inp["q_pos"], want_scores=True)
        idx = torch.full_like(ref_idx, -7)
        sc = torch.full_like(ref_sc, 7.0)
        n0 = csa.csa_launch_count()
        st = _noalloc(L, inp["q_I"], inp["w"], inp["k_I"], w.m, w.k, inp["q_pos"], idx, sc)
        assert st == csa.CSA_OK
        assert csa.csa_launch_count() - n0 == 2     # chunk scoring + candidate merge
        torch.cuda.synchronize()
        # index work is compared bit for bit; scores come from the same kernels
        assert torch.equal(idx, ref_idx)
        assert torch.equal(sc, ref_sc)
        outs.append(idx)
    assert not torch.equal(outs[0], outs[1])


def test_noalloc_rejects_problems_beyond_its_array():
    L = csa.lib()
    # float32 takes the CUDA-core path whose scores need B*Tq*N*4 bytes: 64 MiB here
    B, Tq, HI, dI, N = 1, 4096, 2, 32, 4096
    q_I = torch.zeros((B, Tq, HI, dI), device="cuda")
    w = torch.zeros((B, Tq, HI), device="cuda")
    k_I = torch.zeros((B, N, dI), device="cuda")
    idx = torch.empty((B, Tq, 8), dtype=torch.int32, device="cuda")
    fn = L.indexer_scores_topk_noalloc
    P, i32, i64 = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64
    fn.argtypes = [i32, i64, i64, i32, i32, P, P, P, i64, P, i32, i32, P, P, P]
    fn.restype = i32
    st = fn(csa.CSA_F32, B, Tq, HI, dI, P(q_I.data_ptr()), P(w.data_ptr()), P(k_I.data_ptr()),
            N, None, 4, 8, P(idx.data_ptr()), None, None)
    assert st == csa.CSA_E_WORKSPACE


def _call_f32(L, B, Tq, HI, dI, N, k, q_pos, tensors):
    q_I, w, k_I, idx, sc = tensors
    P = ctypes.c_void_p
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    return L.indexer_scores_topk_noalloc(
        csa.CSA_F32, B, Tq, HI, dI, P(q_I.data_ptr()), P(w.data_ptr()), P(k_I.data_ptr()), N,
        P(q_pos.data_ptr()), 4, k, P(idx.data_ptr()), P(sc.data_ptr()), stream)


def test_noalloc_float32_at_the_limit_matches_twice():
    """float32 takes the CUDA-core kernels, whose B*Tq*N*4-byte score matrix
    lives in the array: 64 rows x 32767 entries need exactly 8 MiB - 256
    bytes, the most the array holds next to its status word.  Accepted, and
    equal bit for bit to the workspace path, on two calls in a row."""
    L = csa.lib()
    B, Tq, HI, dI, N, k = 1, 64, 2, 32, 32767, 8
    assert 256 + B * Tq * N * 4 == 8 << 20
    q_pos = torch.full((B, Tq), 4 * N - 1, dtype=torch.int64, device="cuda")
    for call in range(2):
        q_I = wl.randn((B, Tq, HI, dI), 200 + call, "cuda")
        w = wl.randn((B, Tq, HI), 210 + call, "cuda")
        k_I = wl.randn((B, N, dI), 220 + call, "cuda")
        ref_idx, ref_sc = csa.indexer_scores_topk(q_I, w, k_I, 4, k, q_pos=q_pos,
                                                  want_scores=True)
        idx = torch.full_like(ref_idx, -7)
        sc = torch.full_like(ref_sc, 7.0)
        n0 = csa.csa_launch_count()
        assert _call_f32(L, B, Tq, HI, dI, N, k, q_pos, (q_I, w, k_I, idx, sc)) == csa.CSA_OK
        assert csa.csa_launch_count() - n0 == 2     # scores + top-k
        torch.cuda.synchronize()
        assert torch.equal(idx, ref_idx)
        assert torch.equal(sc, ref_sc)


def test_noalloc_float32_four_bytes_over_the_limit_is_rejected():
    """One row over 2097089 entries needs 4 bytes more than the array holds:
    rejected before any launch.  The tensors are allocated at full size, so
    even a wrong size check would only read memory the call was given."""
    L = csa.lib()
    B, Tq, HI, dI, k = 1, 1, 2, 32, 8
    N = ((8 << 20) - 256) // 4 + 1
    q_pos = torch.full((B, Tq), 4 * N - 1, dtype=torch.int64, device="cuda")
    q_I = torch.zeros((B, Tq, HI, dI), device="cuda")
    w = torch.zeros((B, Tq, HI), device="cuda")
    k_I = torch.zeros((B, N, dI), device="cuda")
    idx = torch.empty((B, Tq, k), dtype=torch.int32, device="cuda")
    sc = torch.empty((B, Tq, k), dtype=torch.float32, device="cuda")
    n0 = csa.csa_launch_count()
    assert _call_f32(L, B, Tq, HI, dI, N, k, q_pos, (q_I, w, k_I, idx, sc)) == csa.CSA_E_WORKSPACE
    assert csa.csa_launch_count() == n0

