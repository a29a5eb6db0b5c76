"""GPU parity of mixed BF16 / MX-FP8 storage of compressed entries: the
records csa_store_mixed writes (bit for bit against the oracle's mixed store)
and the attention calls reading them under CSA_F_MIXED (against the oracle's
attention over the oracle's mixed-load of the same entries), on the
tensor-core and the CUDA-core kernels."""
import numpy as np
import pytest
import torch

import oracle
from parity import assert_close, f64
import long_context_attention_csa_b200 as csa
from long_context_attention_csa_b200 import workloads as wl

pytestmark = pytest.mark.gpu

DEV = "cuda"


def parse_records(rec, c, r):
    """Records [..., bytes] -> (codes [..., c-r], exponents [..., (c-r)/32],
    RoPE dims [..., r] as float64, padding bytes)."""
    cq = c - r
    rec = rec.cpu()
    codes = rec[..., :cq].numpy()
    rope = f64(rec[..., cq:cq + 2 * r].contiguous().view(torch.bfloat16))
    exps = rec[..., cq + 2 * r:cq + 2 * r + cq // 32].numpy().astype(np.int64) - 127
    pad = rec[..., cq + 2 * r + cq // 32:].numpy()
    return codes, exps, rope, pad


@pytest.mark.parametrize("dtype,c,r", [(torch.bfloat16, 512, 64), (torch.float32, 64, 32)])
def test_store_mixed_matches_the_oracle(dtype, c, r):
    B, N = 2, 333
    ent = (wl.randn((B, N, c), 601, DEV) * 2).to(dtype)
    ent[0, 3, :32] = 0                       # an all-zero block
    ent[1, 4, :] = -ent[1, 4, :] * 1e-3      # small values, negative zeros after rounding
    rec = csa.csa_store_mixed(ent, csa.Fmt(c=c, rope_dims=r))
    torch.cuda.synchronize()
    assert rec.shape[-1] == csa.csa_mixed_record_bytes(c, r) and rec.shape[-1] % 16 == 0
    codes, exps, rope, pad = parse_records(rec, c, r)
    assert np.all(pad == 0)
    for b in range(B):
        rc, re, rr = oracle.mixed_store(f64(ent[b]), r)
        assert np.array_equal(codes[b], rc), f"codes b={b}"
        assert np.array_equal(exps[b], re), f"exponents b={b}"
        assert np.array_equal(rope[b], rr), f"RoPE dims b={b}"


def _mixed_reference(ent_b, r):
    """The oracle's view of a stored entry: mixed-load of its mixed-store."""
    return oracle.mixed_load(*oracle.mixed_store(f64(ent_b), r))


@pytest.mark.parametrize("flags", [0, csa.CSA_F_PORTABLE])
def test_decode_attention_over_mixed_entries(flags):
    """Eight rows of the csa_decode_b32_128k workload (sparse, top-k 1024)
    with the entry cache stored mixed."""
    w = wl.scaled(wl.WORKLOADS["csa_decode_b32_128k"], B=8)
    inp = wl.csa_decode_inputs(w, DEV)
    counts = torch.tensor([oracle.visible(w.T - 1, w.m, w.n_csa)])
    idx = torch.stack([wl.random_index_sets(counts, w.k, 700 + b) for b in range(w.B)]).to(DEV)
    fmt = csa.Fmt(c=w.c, rope_dims=w.r)
    rec = csa.csa_store_mixed(inp["entries"], fmt)
    out = csa.sparse_mqa_attn(inp["q"], rec, idx, inp["win"],
                              csa.Fmt(c=w.c, rope_dims=w.r, flags=flags | csa.CSA_F_MIXED),
                              w.n_win, sink=inp["sink"], q_pos=inp["q_pos"],
                              win_pos0=inp["win_pos0"])
    torch.cuda.synchronize()
    of = oracle.Fmt(c=w.c, rope_dims=w.r)
    for b in range(w.B):
        ent = _mixed_reference(inp["entries"][b], w.r)
        ref = oracle.attention(f64(inp["q"][b]), ent, f64(inp["win"][b]), of, w.n_win,
                               idx=idx[b].cpu().numpy(), sink=f64(inp["sink"]),
                               q_pos=inp["q_pos"][b].cpu().numpy(),
                               win_pos0=int(inp["win_pos0"][b]))
        assert_close(out[b], ref, torch.bfloat16, f"mixed decode b={b}")


@pytest.mark.parametrize("flags", [0, csa.CSA_F_PORTABLE])
def test_attention_over_mixed_entries_prefill_and_dense(flags):
    """Prefill rows (300 tokens, several 64-key blocks, the window branch in
    the same blocks) sparse, and dense HCA rows over mixed entries."""
    w = wl.scaled(wl.WORKLOADS["csa_prefill_8k"], T=300, k=32)
    g = wl
    q = g.randn((1, w.T, w.H, w.c), 611, DEV, dtype=torch.bfloat16)
    ent = g.randn((1, w.n_csa, w.c), 612, DEV, dtype=torch.bfloat16)
    win = g.randn((1, w.T, w.c), 613, DEV, dtype=torch.bfloat16)
    sink = g.randn((w.H,), 614, DEV)
    counts = torch.tensor([oracle.visible(t, w.m, w.n_csa) for t in range(w.T)])
    idx = g.random_index_sets(counts, w.k, 615).unsqueeze(0).to(DEV)
    fm = csa.Fmt(c=w.c, rope_dims=w.r, flags=flags | csa.CSA_F_MIXED)
    rec = csa.csa_store_mixed(ent, csa.Fmt(c=w.c, rope_dims=w.r))
    outs = csa.sparse_mqa_attn(q, rec, idx, win, fm, w.n_win, sink=sink)
    outd = csa.dense_hca_attn(q, rec, 16, win, fm, w.n_win, sink=sink)
    torch.cuda.synchronize()
    of = oracle.Fmt(c=w.c, rope_dims=w.r)
    e = _mixed_reference(ent[0], w.r)
    rows = np.arange(w.T)
    refs = oracle.attention(f64(q[0]), e, f64(win[0]), of, w.n_win, idx=idx[0].cpu().numpy(),
                            sink=f64(sink), q_pos=rows)
    assert_close(outs[0], refs, torch.bfloat16, "mixed sparse prefill")
    refd = oracle.attention(f64(q[0]), e, f64(win[0]), of, w.n_win, m_dense=16, sink=f64(sink),
                            q_pos=rows)
    assert_close(outd[0], refd, torch.bfloat16, "mixed dense prefill")
