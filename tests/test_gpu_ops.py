"""GPU parity: every C-ABI call against the float64 oracle on the same seeded
inputs, at small sizes that span several tiles and a ragged tail (compared
element by element) and at the full workload sizes (compared on sampled rows).
"""
import numpy as np
import pytest
import torch

import oracle
from parity import assert_close, check_topk_rows, f64
import long_context_attention_csa_b200 as csa
from long_context_attention_csa_b200 import workloads as wl

pytestmark = pytest.mark.gpu

DEV = "cuda"


def ofmt(w, flags=0):
    return oracle.Fmt(c=w.c, rope_dims=w.r, rope_base=w.rope_base, flags=flags)


def gfmt(w, flags=0):
    return csa.Fmt(c=w.c, rope_dims=w.r, rope_base=w.rope_base, flags=flags)


def sample_rows(T, n=40, seed=0):
    g = np.random.default_rng(seed)
    fixed = [0, 1, 2, 3, 4, 5, 126, 127, 128, 129, T // 2, T - 2, T - 1]
    rnd = g.choice(T, size=min(n, T), replace=False).tolist()
    return np.array(sorted(set(r for r in fixed + rnd if 0 <= r < T)))


# ----------------------------------------------------------------- compression

@pytest.mark.parametrize("wname,T,B,pos0,zc", [
    ("tiny_csa_fp32", 256, 1, 0, None),
    ("csa_prefill_8k", 1003, 2, 7, None),
    ("csa_prefill_8k", 1003, 2, 0, 1),
    ("csa_prefill_8k", 8192, 1, 0, None),
])
def test_csa_compress(wname, T, B, pos0, zc):
    w = wl.scaled(wl.WORKLOADS[wname], T=T, B=B)
    inp = wl.csa_prefill_inputs(w, DEV)
    za, zb = inp["z_a"], inp["z_b"]
    if zc == 1:
        za, zb = za[..., :1].contiguous(), zb[..., :1].contiguous()
    ent, win = csa.csa_compress(inp["kv_a"], inp["kv_b"], za, zb, w.m, gfmt(w), pos0=pos0,
                                want_win=True)
    torch.cuda.synchronize()
    assert ent.shape == (B, T // w.m, w.c)
    for b in range(B):
        ref = oracle.csa_compress(f64(inp["kv_a"][b]), f64(inp["kv_b"][b]), f64(za[b]), f64(zb[b]),
                                  w.m, ofmt(w), pos0=pos0)
        assert_close(ent[b], ref, w.dtype, f"entries b={b}")
        refw = oracle.window_rows(f64(inp["kv_a"][b]), ofmt(w), pos0=pos0)
        assert_close(win[b], refw, w.dtype, f"window b={b}")


@pytest.mark.parametrize("T,B,mp", [(1000, 2, 128), (65536, 1, 128), (300, 1, 7)])
def test_hca_compress(T, B, mp):
    w = wl.scaled(wl.WORKLOADS["hca_prefill_64k"], T=T, B=B, m_prime=mp)
    inp = wl.hca_prefill_inputs(w, DEV)
    del inp["q"]
    ent, win = csa.hca_compress(inp["kv"], inp["z"], mp, gfmt(w), want_win=True)
    torch.cuda.synchronize()
    assert ent.shape == (B, T // mp, w.c)
    for b in range(B):
        ref = oracle.hca_compress(f64(inp["kv"][b]), f64(inp["z"][b]), mp, ofmt(w))
        assert_close(ent[b], ref, w.dtype, f"entries b={b}")
        rows = sample_rows(T, 200)
        # window rows at their own positions: the sampled rows one by one
        refw = np.stack([oracle.window_rows(f64(inp["kv"][b][r:r + 1]), ofmt(w), pos0=int(r))[0]
                         for r in rows])
        assert_close(win[b][rows], refw, w.dtype, f"window b={b}")


def test_compress_streaming_path_leaves_the_status_word_clear():
    """The bulk-copy ring of the streaming compression kernels: short and
    ragged sequences (chunks that run past T, the first chunk's previous block
    before token 0) land every copy; the status word stays clear."""
    ws = csa.workspace(csa.csa_workspace_bytes(csa.CSA_OP_COMPRESS, 1, 3, 77))
    w = wl.scaled(wl.WORKLOADS["csa_prefill_8k"], T=77, B=3)
    inp = wl.csa_prefill_inputs(w, DEV)
    ent, win = csa.csa_compress(inp["kv_a"], inp["kv_b"], inp["z_a"], inp["z_b"], w.m, gfmt(w),
                                want_win=True, ws=ws)
    wh = wl.scaled(wl.WORKLOADS["hca_prefill_64k"], T=77, B=3, m_prime=32)
    hin = wl.hca_prefill_inputs(wh, DEV)
    hent, hwin = csa.hca_compress(hin["kv"], hin["z"], 32, gfmt(wh), want_win=True, ws=ws)
    assert csa.csa_check_status(ws) == (csa.CSA_OK, 0)
    for b in range(3):
        ref = oracle.csa_compress(f64(inp["kv_a"][b]), f64(inp["kv_b"][b]), f64(inp["z_a"][b]),
                                  f64(inp["z_b"][b]), w.m, ofmt(w))
        assert_close(ent[b], ref, w.dtype, f"csa entries b={b}")
        assert_close(win[b], oracle.window_rows(f64(inp["kv_a"][b]), ofmt(w)), w.dtype, "window")
        href = oracle.hca_compress(f64(hin["kv"][b]), f64(hin["z"][b]), 32, ofmt(wh))
        assert_close(hent[b], href, wh.dtype, f"hca entries b={b}")


# ----------------------------------------------------------------- indexer

def _indexer_case(w, rows=None, q_pos=None, exact=False):
    inp = wl.csa_prefill_inputs(w, DEV) if w.kind == "csa_prefill" else wl.csa_decode_inputs(w, DEV)
    qp = inp.get("q_pos")
    idx, sc = csa.indexer_scores_topk(inp["q_I"], inp["w"], inp["k_I"], w.m, w.k, q_pos=qp,
                                      want_scores=True)
    torch.cuda.synchronize()
    B, Tq = inp["q_I"].shape[:2]
    rows = np.arange(Tq) if rows is None else rows
    differing = 0
    for b in range(B):
        pos = rows if qp is None else qp[b].cpu().numpy()[rows]
        ref_sc = oracle.indexer_scores(f64(inp["q_I"][b][rows]), f64(inp["w"][b][rows]),
                                       f64(inp["k_I"][b]), w.m, q_pos=pos)
        ref_idx = oracle.topk(ref_sc, w.k, w.m, q_pos=pos)
        gi = idx[b][rows].cpu().numpy()
        differing += check_topk_rows(gi, ref_idx, ref_sc, exact=exact, what=f"b={b}")
        # scores of the GPU's own selection against the oracle's score of the same entries
        gs = sc[b][rows].cpu().numpy().astype(np.float64)
        valid = gi >= 0
        want = np.take_along_axis(ref_sc, np.where(valid, gi, 0), axis=1)
        if exact:
            assert np.array_equal(gs[valid], want[valid])
        else:
            err = np.abs(gs[valid] - want[valid]) / np.maximum(1.0, np.abs(want[valid]))
            assert err.max() <= 1e-4, f"score error {err.max()}"
        assert np.all(np.isneginf(gs[~valid]))
    return differing


def test_indexer_tiny_fp32():
    _indexer_case(wl.WORKLOADS["tiny_csa_fp32"])


@pytest.mark.parametrize("HI,dI,T,k,dt", [(64, 128, 700, 64, torch.bfloat16),
                                           (2, 32, 300, 16, torch.float32),
                                           (64, 128, 1000, 256, torch.bfloat16)])
def test_indexer_integer_inputs_bit_exact(HI, dI, T, k, dt):
    """Small-integer inputs make every product and sum exact in bf16 x bf16 ->
    fp32 (tensor cores) and in float32 (CUDA cores): the selected sets (tie
    rule included) and scores must be identical."""
    B, m = 1, 4
    N = T // m
    qI = wl.randint_like_float((B, T, HI, dI), 11, -2, 3, DEV, dt)
    kI = wl.randint_like_float((B, N, dI), 12, -2, 3, DEV, dt)
    w = wl.randint_like_float((B, T, HI), 13, -2, 3, DEV, torch.float32)
    idx, sc = csa.indexer_scores_topk(qI, w, kI, m, k, want_scores=True)
    torch.cuda.synchronize()
    ref_sc = oracle.indexer_scores(f64(qI[0]), f64(w[0]), f64(kI[0]), m)
    ref_idx = oracle.topk(ref_sc, k, m)
    assert np.array_equal(idx[0].cpu().numpy(), ref_idx)
    gi = idx[0].cpu().numpy()
    v = gi >= 0
    assert np.array_equal(sc[0].cpu().numpy().astype(np.float64)[v],
                          np.take_along_axis(ref_sc, np.where(v, gi, 0), 1)[v])


def test_indexer_csa_prefill_8k_sampled():
    w = wl.WORKLOADS["csa_prefill_8k"]
    d = _indexer_case(w, rows=sample_rows(w.T, 48))
    assert d <= 2


def test_indexer_prefill_multichunk_sampled():
    """More than 2048 entries: the prefill kernel emits per-chunk candidates
    (three chunks here) that the merge kernel reduces; two sequences."""
    w = wl.scaled(wl.WORKLOADS["csa_prefill_8k"], B=2, T=20000)
    d = _indexer_case(w, rows=np.unique(np.concatenate([sample_rows(w.T, 24),
                                                        np.arange(w.T - 8, w.T)])))
    assert d <= 2


def test_indexer_multichunk_integer_bit_exact():
    """Integer inputs (exact sums, many ties) across three 2048-entry chunks:
    candidates and the merge must reproduce the oracle's sets and scores."""
    B, T, HI, dI, m, k = 1, 9000, 64, 128, 4, 256
    N = T // m
    qI = wl.randint_like_float((B, T, HI, dI), 31, -2, 3, DEV, torch.bfloat16)
    kI = wl.randint_like_float((B, N, dI), 32, -2, 3, DEV, torch.bfloat16)
    w = wl.randint_like_float((B, T, HI), 33, -2, 3, DEV, torch.float32)
    idx, sc = csa.indexer_scores_topk(qI, w, kI, m, k, want_scores=True)
    torch.cuda.synchronize()
    rows = sample_rows(T, 12)
    ref_sc = oracle.indexer_scores(f64(qI[0][rows]), f64(w[0][rows]), f64(kI[0]), m, q_pos=rows)
    ref_idx = oracle.topk(ref_sc, k, m, q_pos=rows)
    assert np.array_equal(idx[0][rows].cpu().numpy(), ref_idx)


def test_indexer_prefill_positions():
    """Prefill with explicit positions (a chunk continuing a longer context):
    visibility follows q_pos, not the row index."""
    B, T, HI, dI, m, k = 1, 600, 64, 128, 4, 128
    pos = torch.arange(T, dtype=torch.int64).unsqueeze(0) + 3000
    N = (3000 + T) // m
    qI = wl.randn((B, T, HI, dI), 21, DEV, dtype=torch.bfloat16)
    kI = wl.randn((B, N, dI), 22, DEV, dtype=torch.bfloat16)
    w = wl.randn((B, T, HI), 23, DEV) / 8
    idx, sc = csa.indexer_scores_topk(qI, w, kI, m, k, q_pos=pos.to(DEV), want_scores=True)
    torch.cuda.synchronize()
    rows = sample_rows(T, 16)
    p = pos[0].numpy()[rows]
    ref_sc = oracle.indexer_scores(f64(qI[0][rows]), f64(w[0][rows]), f64(kI[0]), m, q_pos=p)
    ref_idx = oracle.topk(ref_sc, k, m, q_pos=p)
    assert check_topk_rows(idx[0][rows].cpu().numpy(), ref_idx, ref_sc, what="q_pos") <= 1


@pytest.mark.parametrize("wname", ["csa_decode_b32_128k", "decode_pair_b4_1m"])
def test_indexer_decode(wname):
    w = wl.WORKLOADS[wname]
    d = _indexer_case(w)
    assert d <= 1


@pytest.mark.parametrize("N", [40000, 30000])
@pytest.mark.parametrize("k,zero", [(1023, False), (1024, False), (1024, True)])
def test_indexer_decode_select_integer_bit_exact(N, k, zero):
    """Single-token queries over N entries in 4096-entry chunks: 40000 (ten
    chunks: per-chunk candidates, merged by a cluster of two CTAs) and 30000
    (eight chunks: the row's CTAs select as one cluster).  Integer inputs give
    exact sums and many ties across CTA boundaries; an odd k takes the
    unaligned loads; the third context is short (most chunks empty, fewer
    visible than k); zero q_I makes every score equal (the lowest k indices
    win)."""
    B, HI, dI, m = 3, 64, 128, 4
    pos = torch.tensor([[m * N - 1], [m * (N // 2) + 5], [m * 300]], dtype=torch.int64)
    qI = wl.randint_like_float((B, 1, HI, dI), 41, -2, 3, DEV, torch.bfloat16)
    if zero:
        qI.zero_()
    kI = wl.randint_like_float((B, N, dI), 42, -2, 3, DEV, torch.bfloat16)
    w = wl.randint_like_float((B, 1, HI), 43, -2, 3, DEV, torch.float32)
    idx, sc = csa.indexer_scores_topk(qI, w, kI, m, k, q_pos=pos.to(DEV), want_scores=True)
    torch.cuda.synchronize()
    for b in range(B):
        p = pos[b].numpy()
        ref_sc = oracle.indexer_scores(f64(qI[b]), f64(w[b]), f64(kI[b]), m, q_pos=p)
        ref_idx = oracle.topk(ref_sc, k, m, q_pos=p)
        gi = idx[b].cpu().numpy()
        assert np.array_equal(gi, ref_idx), f"row {b}"
        v = gi >= 0
        assert np.array_equal(sc[b].cpu().numpy().astype(np.float64)[v],
                              np.take_along_axis(ref_sc, np.where(v, gi, 0), 1)[v])


@pytest.mark.parametrize("k", [1024, 37])
def test_indexer_decode_select_heavy_boundary_bin(k):
    """One entry per 4096-entry chunk with a score thousands of times the
    others' stretches the chunk's value range, so nearly every score shares
    the boundary bin: the chunk select narrows that bin by a radix pass on the
    scores' keys and ranks the equal integer scores there by index.  Integer
    inputs keep every score exact; sets and scores equal the oracle's."""
    B, N, HI, dI, m = 2, 30000, 64, 128, 4
    pos = torch.tensor([[m * N - 1], [m * (N // 2) + 5]], dtype=torch.int64)
    qI = wl.randint_like_float((B, 1, HI, dI), 44, -2, 3, DEV, torch.bfloat16)
    kI = wl.randint_like_float((B, N, dI), 45, -2, 3, DEV, torch.bfloat16)
    kI[:, 1234::4096, :] = 100.0
    w = wl.randint_like_float((B, 1, HI), 46, -2, 3, DEV, torch.float32)
    idx, sc = csa.indexer_scores_topk(qI, w, kI, m, k, q_pos=pos.to(DEV), want_scores=True)
    torch.cuda.synchronize()
    for b in range(B):
        p = pos[b].numpy()
        ref_sc = oracle.indexer_scores(f64(qI[b]), f64(w[b]), f64(kI[b]), m, q_pos=p)
        assert np.abs(ref_sc[np.isfinite(ref_sc)]).max() < 2 ** 24   # exact in float32
        ref_idx = oracle.topk(ref_sc, k, m, q_pos=p)
        gi = idx[b].cpu().numpy()
        assert np.array_equal(gi, ref_idx), f"row {b}"
        v = gi >= 0
        assert np.array_equal(sc[b].cpu().numpy().astype(np.float64)[v],
                              np.take_along_axis(ref_sc, np.where(v, gi, 0), 1)[v])


def test_indexer_padding_when_few_visible():
    w = wl.scaled(wl.WORKLOADS["csa_prefill_8k"], T=40, k=16)
    _indexer_case(w)


# ----------------------------------------------------------------- attention

PATHS = [0, csa.CSA_F_PORTABLE]


def _attn_inputs_prefill(w, dense=False):
    g = wl
    B, T, H, c = w.B, w.T, w.H, w.c
    N = w.n_hca if dense else w.n_csa
    inp = dict(
        q=g._draw(w, "q", (B, T, H, c), DEV, w.q_scale),
        entries=g._draw(w, "entries", (B, N, c), DEV),
        win=g._draw(w, "win", (B, T, c), DEV),
        sink=g.randn((H,), g._seed(w, "sink"), DEV) if w.sink else None,
    )
    if not dense:
        counts = torch.tensor([oracle.visible(t, w.m, N) for t in range(T)])
        idx = torch.stack([g.random_index_sets(counts, w.k, w.seed * 7 + b) for b in range(B)])
        inp["idx"] = idx.to(DEV)
    return inp


def _check_attn(w, inp, out, rows, dense, flags=0, q_pos=None, win_pos0=None, roundings=1):
    B = out.shape[0]
    for b in range(B):
        pos = rows if q_pos is None else q_pos[b].cpu().numpy()[rows]
        wp0 = 0 if win_pos0 is None else int(win_pos0[b])
        ref = oracle.attention(
            f64(inp["q"][b][rows]), f64(inp["entries"][b]), f64(inp["win"][b]), ofmt(w, flags),
            w.n_win, idx=None if dense else inp["idx"][b][rows].cpu().numpy(),
            m_dense=w.m_prime if dense else 0,
            sink=None if inp["sink"] is None else f64(inp["sink"]), q_pos=pos, win_pos0=wp0)
        assert_close(out[b][rows], ref, w.dtype, f"attention b={b}", roundings=roundings)


@pytest.mark.parametrize("flags", PATHS)
@pytest.mark.parametrize("wname,T,k,sink", [
    ("tiny_csa_fp32", 256, 16, True),
    ("csa_prefill_8k", 300, 32, True),
    ("csa_prefill_8k", 300, 32, False),
    ("csa_prefill_8k", 261, 0, True),
])
def test_sparse_attention_small(wname, T, k, sink, flags):
    w = wl.scaled(wl.WORKLOADS[wname], T=T, k=k, sink=sink)
    if w.dtype == torch.float32 and flags == 0:
        pytest.skip("float32 always runs the portable kernel")
    inp = _attn_inputs_prefill(w)
    out = csa.sparse_mqa_attn(inp["q"], inp["entries"], inp["idx"], inp["win"], gfmt(w, flags),
                              w.n_win, sink=inp["sink"])
    torch.cuda.synchronize()
    _check_attn(w, inp, out, np.arange(T), dense=False, flags=flags)


@pytest.mark.parametrize("flags", PATHS)
@pytest.mark.parametrize("T,mp", [(600, 128), (333, 16)])
def test_dense_attention_small(T, mp, flags):
    w = wl.scaled(wl.WORKLOADS["hca_prefill_64k"], T=T, m_prime=mp)
    inp = _attn_inputs_prefill(w, dense=True)
    out = csa.dense_hca_attn(inp["q"], inp["entries"], mp, inp["win"], gfmt(w, flags), w.n_win,
                             sink=inp["sink"])
    torch.cuda.synchronize()
    _check_attn(w, inp, out, np.arange(T), dense=True, flags=flags)


def test_sparse_attention_csa_prefill_8k_sampled():
    w = wl.WORKLOADS["csa_prefill_8k"]
    inp = _attn_inputs_prefill(w)
    out = csa.sparse_mqa_attn(inp["q"], inp["entries"], inp["idx"], inp["win"], gfmt(w), w.n_win,
                              sink=inp["sink"])
    torch.cuda.synchronize()
    _check_attn(w, inp, out, sample_rows(w.T, 40), dense=False)


def test_dense_attention_hca_prefill_64k_sampled():
    w = wl.WORKLOADS["hca_prefill_64k"]
    inp = _attn_inputs_prefill(w, dense=True)
    out = csa.dense_hca_attn(inp["q"], inp["entries"], w.m_prime, inp["win"], gfmt(w), w.n_win,
                             sink=inp["sink"])
    torch.cuda.synchronize()
    _check_attn(w, inp, out, sample_rows(w.T, 24), dense=True)
    del out, inp
    torch.cuda.empty_cache()


def _decode_idx(w, inp, seed):
    B = inp["q"].shape[0]
    counts = torch.tensor([oracle.visible(w.T - 1, w.m, w.n_csa)])
    return torch.stack([wl.random_index_sets(counts, w.k, seed + b) for b in range(B)]).to(DEV)


@pytest.mark.parametrize("flags", PATHS)
@pytest.mark.parametrize("wname", ["csa_decode_b32_128k", "decode_pair_b4_1m"])
def test_decode_attention(wname, flags):
    w = wl.WORKLOADS[wname]
    inp = wl.csa_decode_inputs(w, DEV)
    inp["idx"] = _decode_idx(w, inp, 5)
    out = csa.sparse_mqa_attn(inp["q"], inp["entries"], inp["idx"], inp["win"], gfmt(w, flags),
                              w.n_win, sink=inp["sink"], q_pos=inp["q_pos"],
                              win_pos0=inp["win_pos0"])
    torch.cuda.synchronize()
    _check_attn(w, inp, out, np.arange(1), dense=False, flags=flags, q_pos=inp["q_pos"],
                win_pos0=inp["win_pos0"].cpu().numpy())
    if wname == "decode_pair_b4_1m":
        h = wl.hca_decode_inputs(w, DEV)
        out = csa.dense_hca_attn(h["q"], h["entries"], w.m_prime, h["win"], gfmt(w, flags),
                                 w.n_win, sink=h["sink"], q_pos=h["q_pos"], win_pos0=h["win_pos0"])
        torch.cuda.synchronize()
        _check_attn(w, h, out, np.arange(1), dense=True, flags=flags, q_pos=h["q_pos"],
                    win_pos0=h["win_pos0"].cpu().numpy())


def test_decode_batch_invariance():
    """A decode row gives bitwise the same output alone as inside a batch of 32."""
    w = wl.WORKLOADS["csa_decode_b32_128k"]
    inp = wl.csa_decode_inputs(w, DEV)
    inp["idx"] = _decode_idx(w, inp, 5)
    args = dict(sink=inp["sink"])
    full = csa.sparse_mqa_attn(inp["q"], inp["entries"], inp["idx"], inp["win"], gfmt(w), w.n_win,
                               q_pos=inp["q_pos"], win_pos0=inp["win_pos0"], **args)
    for b in (0, 13, 31):
        one = csa.sparse_mqa_attn(inp["q"][b:b + 1].contiguous(), inp["entries"][b:b + 1].contiguous(),
                                  inp["idx"][b:b + 1].contiguous(), inp["win"][b:b + 1].contiguous(),
                                  gfmt(w), w.n_win, q_pos=inp["q_pos"][b:b + 1].contiguous(),
                                  win_pos0=inp["win_pos0"][b:b + 1].contiguous(), **args)
        torch.cuda.synchronize()
        assert torch.equal(one[0], full[b])
    # repeat runs are bitwise identical
    again = csa.sparse_mqa_attn(inp["q"], inp["entries"], inp["idx"], inp["win"], gfmt(w),
                                w.n_win, q_pos=inp["q_pos"], win_pos0=inp["win_pos0"], **args)
    assert torch.equal(again, full)


def test_decode_rows_equal_when_ctas_take_several_items():
    """A batch with more split items than SMs (160 here) has persistent CTAs
    that take two items each; the split boundaries and the combine's order
    depend on a row's own key count only, so its rows are bitwise equal to
    the same rows in a batch of 4 (one item per CTA) and match the oracle."""
    w = wl.scaled(wl.WORKLOADS["csa_decode_b32_128k"], B=40)   # 160 split items > 148
    inp = wl.csa_decode_inputs(w, DEV)
    inp["idx"] = _decode_idx(w, inp, 6)
    args = dict(sink=inp["sink"])
    full = csa.sparse_mqa_attn(inp["q"], inp["entries"], inp["idx"], inp["win"], gfmt(w), w.n_win,
                               q_pos=inp["q_pos"], win_pos0=inp["win_pos0"], **args)
    part = slice(8, 12)   # 16 split items: one cluster of 4 per row
    sub = {k: (v if k == "sink" else v[part].contiguous()) for k, v in inp.items()}
    few = csa.sparse_mqa_attn(sub["q"], sub["entries"], sub["idx"], sub["win"], gfmt(w), w.n_win,
                              q_pos=sub["q_pos"], win_pos0=sub["win_pos0"], **args)
    torch.cuda.synchronize()
    assert torch.equal(few, full[part])
    _check_attn(w, sub, few, np.arange(1), dense=False, q_pos=sub["q_pos"],
                win_pos0=sub["win_pos0"].cpu().numpy())


def test_decode_mixed_contexts_and_invariance():
    """Decode rows of very different context lengths in one batch (the split
    size follows each row's own key count, so short rows leave splits empty
    and the index lists padded): parity with the oracle for the CSA layer
    (sparse) and the HCA layer (dense), and each row bitwise equal alone."""
    w = wl.WORKLOADS["decode_pair_b4_1m"]
    H, c, n_win = w.H, w.c, w.n_win
    L = [131072, 9000, 1300, 50]
    B = len(L)
    N, NH = 32768, 8192
    q = wl.randn((B, 1, H, c), 61, DEV, dtype=torch.bfloat16)
    ent = wl.randn((B, N, c), 62, DEV, dtype=torch.bfloat16)
    hent = wl.randn((B, NH, c), 63, DEV, dtype=torch.bfloat16)
    win = wl.randn((B, n_win, c), 64, DEV, dtype=torch.bfloat16)
    sink = wl.randn((H,), 65, DEV)
    q_pos = torch.tensor([[x - 1] for x in L], dtype=torch.int64, device=DEV)
    wp0 = torch.tensor([max(x - n_win, 0) for x in L], dtype=torch.int64, device=DEV)
    idx = torch.stack([wl.random_index_sets(torch.tensor([oracle.visible(x - 1, w.m, N)]), w.k,
                                            70 + b) for b, x in enumerate(L)]).to(DEV)
    fmt = gfmt(w)
    outs = csa.sparse_mqa_attn(q, ent, idx, win, fmt, n_win, sink=sink, q_pos=q_pos, win_pos0=wp0)
    outd = csa.dense_hca_attn(q, hent, w.m_prime, win, fmt, n_win, sink=sink, q_pos=q_pos,
                              win_pos0=wp0)
    torch.cuda.synchronize()
    for b in range(B):
        pos = q_pos[b].cpu().numpy()
        refs = oracle.attention(f64(q[b]), f64(ent[b]), f64(win[b]), ofmt(w), n_win,
                                idx=idx[b].cpu().numpy(), sink=f64(sink), q_pos=pos,
                                win_pos0=int(wp0[b]))
        assert_close(outs[b], refs, w.dtype, f"sparse decode L={L[b]}")
        refd = oracle.attention(f64(q[b]), f64(hent[b]), f64(win[b]), ofmt(w), n_win,
                                m_dense=w.m_prime, sink=f64(sink), q_pos=pos, win_pos0=int(wp0[b]))
        assert_close(outd[b], refd, w.dtype, f"dense decode L={L[b]}")
        sl = slice(b, b + 1)
        one_s = csa.sparse_mqa_attn(q[sl].contiguous(), ent[sl].contiguous(), idx[sl].contiguous(),
                                    win[sl].contiguous(), fmt, n_win, sink=sink,
                                    q_pos=q_pos[sl].contiguous(), win_pos0=wp0[sl].contiguous())
        one_d = csa.dense_hca_attn(q[sl].contiguous(), hent[sl].contiguous(), w.m_prime,
                                   win[sl].contiguous(), fmt, n_win, sink=sink,
                                   q_pos=q_pos[sl].contiguous(), win_pos0=wp0[sl].contiguous())
        torch.cuda.synchronize()
        assert torch.equal(one_s[0], outs[b]), f"sparse row {b} differs alone"
        assert torch.equal(one_d[0], outd[b]), f"dense row {b} differs alone"


def test_sparse_with_every_visible_entry_equals_dense():
    """k >= vis(t) with the index list of every visible entry: sparse MQA over
    the selection equals dense MQA with m' = m over the same entries (the
    method's own reduction, here through the two GPU entry points)."""
    w = wl.scaled(wl.WORKLOADS["csa_prefill_8k"], T=600)
    B, T, H, c, m = 1, w.T, w.H, w.c, w.m
    N = T // m
    q = wl.randn((B, T, H, c), 81, DEV, dtype=torch.bfloat16)
    ent = wl.randn((B, N, c), 82, DEV, dtype=torch.bfloat16)
    win = wl.randn((B, T, c), 83, DEV, dtype=torch.bfloat16)
    sink = wl.randn((H,), 84, DEV)
    idx = torch.full((B, T, N), -1, dtype=torch.int32)
    for t in range(T):
        v = oracle.visible(t, m, N)
        idx[0, t, :v] = torch.arange(v, dtype=torch.int32)
    idx = idx.to(DEV)
    outs = csa.sparse_mqa_attn(q, ent, idx, win, gfmt(w), w.n_win, sink=sink)
    outd = csa.dense_hca_attn(q, ent, m, win, gfmt(w), w.n_win, sink=sink)
    torch.cuda.synchronize()
    assert_close(outs[0], f64(outd[0]), w.dtype, "sparse(all visible) vs dense", roundings=2)


def test_device_wait_timeout_is_reported_and_the_context_survives():
    """A bounded device wait that nothing satisfies runs out (50 ms), the
    kernel records CSA_DEV_TIMEOUT and returns; the host reads and clears the
    status, and the next calls run and are correct."""
    ws = csa.workspace(256)
    csa.csa_selftest_wait(50_000_000, ws)
    st, d = csa.csa_check_status(ws)
    assert st == csa.CSA_E_DEVICE and d == csa.CSA_DEV_TIMEOUT
    st, d = csa.csa_check_status(ws)
    assert st == csa.CSA_OK and d == 0
    w = wl.scaled(wl.WORKLOADS["csa_prefill_8k"], T=64)
    inp = wl.csa_prefill_inputs(w, DEV)
    ent = csa.csa_compress(inp["kv_a"], inp["kv_b"], inp["z_a"], inp["z_b"], w.m, gfmt(w))
    torch.cuda.synchronize()
    ref = oracle.csa_compress(f64(inp["kv_a"][0]), f64(inp["kv_b"][0]), f64(inp["z_a"][0]),
                              f64(inp["z_b"][0]), w.m, ofmt(w))
    assert_close(ent[0], ref, w.dtype, "entries after the timeout")


# ----------------------------------------------------------------- whole layer

def _layer_check(w, inp, ent, win, idx, out, rows):
    """The GPU chain's entries, window rows, index sets and outputs against the
    oracle's own chain on the same raw inputs.  A row whose GPU index set
    differs from the oracle's (legitimately: only within the tie band, which
    check_topk_rows enforces) has its output checked against the oracle's
    attention over the GPU's own set, so every sampled row is checked."""
    x = {kk: (None if v is None else f64(v[0] if v.dim() > 1 else v)) for kk, v in inp.items()}
    ref = oracle.csa_layer(x, ofmt(w), w.m, w.k, w.n_win, rows=rows)
    assert_close(ent[0], ref["entries"], w.dtype, "layer entries")
    assert_close(win[0][rows], ref["win"][rows], w.dtype, "layer window rows")
    gi = idx[0][rows].cpu().numpy()
    check_topk_rows(gi, ref["idx"], ref["scores"], what="layer")
    diff = np.where(~np.all(gi == ref["idx"], axis=1))[0]
    want = ref["out"].copy()
    if len(diff):
        want[diff] = oracle.attention(x["q"][rows[diff]], ref["entries"], ref["win"], ofmt(w),
                                      w.n_win, idx=gi[diff], sink=x["sink"], q_pos=rows[diff])
    # the GPU chain stores the entries and window rows in bf16 before attention
    # and rounds the output again: two bf16 roundings against the float64 chain
    assert_close(out[0][rows], want, w.dtype, f"layer output ({len(diff)} rows on the GPU set)",
                 roundings=2)
    return len(diff)


def _layer_run(w):
    inp = wl.csa_prefill_inputs(w, DEV)
    ent, win = csa.csa_compress(inp["kv_a"], inp["kv_b"], inp["z_a"], inp["z_b"], w.m, gfmt(w),
                                want_win=True)
    idx = csa.indexer_scores_topk(inp["q_I"], inp["w"], inp["k_I"], w.m, w.k)
    out = csa.sparse_mqa_attn(inp["q"], ent, idx, win, gfmt(w), w.n_win, sink=inp["sink"])
    torch.cuda.synchronize()
    return inp, ent, win, idx, out


@pytest.mark.parametrize("wname,T,k", [("tiny_csa_fp32", 256, 16), ("csa_prefill_8k", 512, 64)])
def test_csa_layer_end_to_end(wname, T, k):
    """compress -> indexer -> attention on the GPU against the oracle's own
    chain from the same raw inputs, every row."""
    w = wl.scaled(wl.WORKLOADS[wname], T=T, k=k)
    inp, ent, win, idx, out = _layer_run(w)
    _layer_check(w, inp, ent, win, idx, out, np.arange(T))


def test_csa_layer_csa_prefill_8k_sampled():
    """The whole chain at the full csa_prefill_8k workload (8192 tokens, 2048
    entries, top-k 512) as the benchmark runs it, checked on sampled rows."""
    w = wl.WORKLOADS["csa_prefill_8k"]
    inp, ent, win, idx, out = _layer_run(w)
    _layer_check(w, inp, ent, win, idx, out, sample_rows(w.T, 40))


# ----------------------------------------------------------------- device status

def test_attention_logit_beyond_the_bound_is_flagged():
    """Stored keys 30x larger than unit RMS (not what the compression calls
    produce) push logits more than 60 past the tensor-core kernel's static
    softmax bound: the kernel records CSA_DEV_RANGE in the status word.  The
    CUDA-core kernel keeps an exact running maximum and stays correct."""
    w = wl.scaled(wl.WORKLOADS["csa_prefill_8k"], T=300, k=32)
    inp = _attn_inputs_prefill(w)
    inp["entries"] = (inp["entries"].float() * 30).to(torch.bfloat16)
    ws = csa.workspace(csa.csa_workspace_bytes(csa.CSA_OP_SPARSE_ATTN, 1, 1, w.T, w.H, w.c,
                                               w.n_csa, w.k, w.n_win))
    csa.sparse_mqa_attn(inp["q"], inp["entries"], inp["idx"], inp["win"], gfmt(w), w.n_win,
                        sink=inp["sink"], ws=ws)
    assert csa.csa_check_status(ws) == (csa.CSA_E_DEVICE, csa.CSA_DEV_RANGE)
    assert csa.csa_check_status(ws) == (csa.CSA_OK, 0)    # read and cleared
    out = csa.sparse_mqa_attn(inp["q"], inp["entries"], inp["idx"], inp["win"],
                              gfmt(w, csa.CSA_F_PORTABLE), w.n_win, sink=inp["sink"], ws=ws)
    assert csa.csa_check_status(ws) == (csa.CSA_OK, 0)
    # logits near 100 carry float32 dot-product errors of ~1e-4 absolute, which
    # move the weights by as much relatively: half an ulp more than the output
    # rounding alone (measured 0.66 ulp at |out| ~ 36)
    _check_attn(w, inp, out, np.arange(0, w.T, 3), dense=False, flags=csa.CSA_F_PORTABLE,
                roundings=2)


@pytest.mark.parametrize("flags", PATHS)
def test_attention_index_out_of_range_is_skipped_and_flagged(flags):
    """An index in [N, allocation): the entries tensor has spare rows beyond
    the N the call is given, so a missing guard would read allocated memory,
    not fault.  The kernel skips the index, records CSA_DEV_BAD_INDEX, and the
    output equals the oracle's, which skips it too."""
    w = wl.scaled(wl.WORKLOADS["csa_prefill_8k"], T=300, k=32)
    inp = _attn_inputs_prefill(w)
    N = w.n_csa
    spare = wl.randn((1, N + 16, w.c), 91, DEV, dtype=torch.bfloat16)
    spare[:, :N] = inp["entries"]
    inp["entries"] = spare[:, :N]          # contiguous view of the first N rows
    assert inp["entries"].is_contiguous()
    idx = inp["idx"].clone()
    planted = [10, 50, 100, 101]
    for t in planted:                       # rows with fewer than k visible entries
        v = oracle.visible(t, w.m, N)
        assert v < w.k
        idx[0, t, v] = N + 3
    inp["idx"] = idx
    ws = csa.workspace(csa.csa_workspace_bytes(csa.CSA_OP_SPARSE_ATTN, 1, 1, w.T, w.H, w.c, N,
                                               w.k, w.n_win))
    out = csa.sparse_mqa_attn(inp["q"], inp["entries"], idx, inp["win"], gfmt(w, flags), w.n_win,
                              sink=inp["sink"], ws=ws)
    assert csa.csa_check_status(ws) == (csa.CSA_E_DEVICE, csa.CSA_DEV_BAD_INDEX)
    rows = np.array(sorted(set(planted) | set(range(0, w.T, 5))))
    _check_attn(w, inp, out, rows, dense=False, flags=flags)


def test_prefill_row_agrees_with_the_decode_query_at_its_position():
    """A prefill row t and the same query run as a decode step (one query at
    position t, its key list split into pieces whose float32 partials are
    added in a fixed order) differ only by the float32 summation order: at
    most one bf16 ulp of the larger value, element by element, over rows
    spanning the first blocks, the window's reach and the sequence's end."""
    w = wl.scaled(wl.WORKLOADS["csa_prefill_8k"], T=700, k=128)
    inp = _attn_inputs_prefill(w)
    pre = csa.sparse_mqa_attn(inp["q"], inp["entries"], inp["idx"], inp["win"], gfmt(w), w.n_win,
                              sink=inp["sink"])
    torch.cuda.synchronize()
    for t in (0, 3, 127, 128, 400, 699):
        pos = torch.tensor([[t]], dtype=torch.int64, device=DEV)
        dec = csa.sparse_mqa_attn(inp["q"][:, t:t + 1].contiguous(), inp["entries"],
                                  inp["idx"][:, t:t + 1].contiguous(), inp["win"], gfmt(w),
                                  w.n_win, sink=inp["sink"], q_pos=pos)
        torch.cuda.synchronize()
        a, b = f64(pre[0, t]), f64(dec[0, 0])
        ulp = np.exp2(np.floor(np.log2(np.maximum(np.maximum(np.abs(a), np.abs(b)),
                                                   np.finfo(np.float32).tiny))) - 7)
        assert np.all(np.abs(a - b) <= ulp), f"row {t}: {np.abs(a - b).max()}"
