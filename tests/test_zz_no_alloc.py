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
        st = _noalloc(L, inp["q_I"], inp["w"], inp["k_I"], w.m, w.k, inp["q_pos"], idx, sc)
        assert st == csa.CSA_OK
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
