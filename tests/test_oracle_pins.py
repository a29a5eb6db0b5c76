"""Pins for the float64 oracle: closed forms, invariants, special cases that
reduce to textbook routines, and brute force on tiny inputs.

Each pin is chosen so that a plausible slip in the oracle (a dropped term, a
wrong sign or index, a transposed operand, an off-by-one block) fails at least
one of them.  Sources: page "DeepSeek-V4：迈向高效百万 Token 上下文智能", §3.3
(compression, indexer, top-k, MQA, HCA, RMSNorm, partial RoPE, window); page
"DeepSeek V4 完整技术报告", section "混合注意力：CSA + HCA" (window 128, sink,
RoPE on the last 64 dims).
"""
import json
import math
import os

import numpy as np
import pytest
import torch

import brute
import oracle
from oracle import Fmt, NO_NORM, NO_ROPE

RNG = np.random.default_rng(1234)
GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def rand(*shape, scale=1.0):
    return RNG.standard_normal(shape) * scale


# ---------------------------------------------------------------- transforms

def test_rmsnorm_closed_form():
    x = rand(3, 64)
    for row in x:
        y = oracle.rmsnorm(row, eps=1e-6)
        ms = np.mean(row ** 2)
        # mean square of the output is ms / (ms + eps)
        assert abs(np.mean(y ** 2) - ms / (ms + 1e-6)) < 1e-14
        # direction unchanged
        assert abs(np.dot(y, row) / (np.linalg.norm(y) * np.linalg.norm(row)) - 1) < 1e-14
    # constant vector a: every output is a / sqrt(a^2 + eps)
    y = oracle.rmsnorm(np.full(8, 3.0), eps=0.25)
    assert np.allclose(y, 3.0 / math.sqrt(9.25), rtol=0, atol=1e-15)


def test_rope_worked_values():
    # r = 2: the single pair turns by exactly p radians (theta_0 = base^0 = 1)
    for p in (1, 2, 5, -3, 100):
        y = oracle.rope(np.array([1.0, 0.0]), p, rope_dims=2)
        assert np.allclose(y, [math.cos(p), math.sin(p)], atol=1e-15)
    # r = 4, base 10000: the second pair turns by p * 10000^(-1/2) = p / 100
    y = oracle.rope(np.array([7.0, 7.0, 1.0, 0.0]), 100, rope_dims=4)
    assert np.allclose(y[2:], [math.cos(1.0), math.sin(1.0)], atol=1e-15)
    # and the first pair of the same vector by 100 rad
    assert np.allclose(y[:2], [7 * math.cos(100) - 7 * math.sin(100),
                               7 * math.sin(100) + 7 * math.cos(100)], atol=1e-12)


def test_rope_invariants():
    c, r = 64, 32
    x, y = rand(c), rand(c)
    assert np.allclose(oracle.rope(x, 0, r), x, atol=0)
    for p in (1, 17, 4096, 1 << 20):
        xp = oracle.rope(x, p, r)
        # only the last r dims move, norms are kept
        assert np.array_equal(xp[: c - r], x[: c - r])
        assert abs(np.linalg.norm(xp) - np.linalg.norm(x)) < 1e-12
        # inverse at -p
        assert np.allclose(oracle.rope(xp, -p, r), x, atol=1e-12)
    # relative position: <R_p x, R_q y> == <R_{p-q} x, y>
    for p, q in ((5, 3), (1000, 10), (7, 7), (3, 90)):
        a = np.dot(oracle.rope(x, p, r), oracle.rope(y, q, r))
        b = np.dot(oracle.rope(x, p - q, r), y)
        assert abs(a - b) < 1e-11
    # matches the complex-exponential form
    assert np.allclose(oracle.rope(x, 123, r), brute.rope(x, 123, r), atol=1e-12)


def test_visible_counts():
    # entry s is visible once its last token m(s+1)-1 <= pos
    m = 4
    assert [oracle.visible(p, m, 100) for p in range(10)] == [0, 0, 0, 1, 1, 1, 1, 2, 2, 2]
    assert oracle.visible(10 ** 6, m, 64) == 64
    assert oracle.visible(-1, m, 64) == 0
    assert oracle.visible(127, 128, 10) == 1 and oracle.visible(126, 128, 10) == 0


# ---------------------------------------------------------------- compression

def _fmt(c, r, flags=0):
    return Fmt(c=c, rope_dims=r, flags=flags)


def test_csa_entry_count_and_weights():
    T, c, m = 256, 64, 4
    ca, cb, za, zb = rand(T, c), rand(T, c), rand(T, c), rand(T, c)
    ent, w = oracle.csa_compress(ca, cb, za, zb, m, _fmt(c, 32), want_weights=True)
    assert ent.shape == (64, c)                     # rate exactly 1/m: 256/4
    assert np.allclose(w.sum(axis=1), 1.0, atol=1e-14)
    assert (w >= 0).all()
    assert np.array_equal(w[0, m:], np.zeros((m, c)))   # entry 0 has no b group
    # tail tokens make no entry
    ent2 = oracle.csa_compress(ca[:255], cb[:255], za[:255], zb[:255], m, _fmt(c, 32))
    assert ent2.shape == (63, c)


def test_csa_uniform_logits_is_mean():
    T, c, m = 64, 16, 4
    ca, cb = rand(T, c), rand(T, c)
    z = np.zeros((T, c))
    ent = oracle.csa_compress(ca, cb, z, z, m, _fmt(c, 8, NO_NORM | NO_ROPE))
    for s in range(T // m):
        rows = [ca[m * s:m * s + m]]
        if s >= 1:
            rows.append(cb[m * (s - 1):m * s])
        assert np.allclose(ent[s], np.concatenate(rows).mean(axis=0), atol=1e-14)


@pytest.mark.parametrize("slot", range(8))
def test_csa_one_hot_slot_geometry(slot):
    """A dominant logit on one slot picks exactly that token row: pins which
    token each of the 2m slots of entry s reads (a: m s + j, b: m(s-1) + j)."""
    T, c, m = 64, 8, 4
    ca, cb = rand(T, c), rand(T, c)
    za = np.full((T, c), -1e4)
    zb = np.full((T, c), -1e4)
    n = T // m
    for s in range(1, n):
        if slot < m:
            za[m * s + slot] = 0.0
        else:
            zb[m * (s - 1) + slot - m] = 0.0
    ent = oracle.csa_compress(ca, cb, za, zb, m, _fmt(c, 4, NO_NORM | NO_ROPE))
    for s in range(1, n):
        want = ca[m * s + slot] if slot < m else cb[m * (s - 1) + slot - m]
        assert np.array_equal(ent[s], want)


def test_csa_m1_identity():
    """m = 1, uniform logits and C^b[j] := C^a[j+1]: every entry is C^a[s]."""
    T, c = 32, 16
    ca = rand(T, c)
    cb = np.concatenate([ca[1:], rand(1, c)])
    z = np.zeros((T, c))
    ent = oracle.csa_compress(ca, cb, z, z, 1, _fmt(c, 8, NO_NORM | NO_ROPE))
    assert np.allclose(ent, ca, atol=1e-14)


def test_hca_m1_identity_and_mean():
    T, c = 256, 16
    kv, z = rand(T, c), rand(T, c)
    assert np.array_equal(oracle.hca_compress(kv, z, 1, _fmt(c, 8, NO_NORM | NO_ROPE)), kv)
    ent = oracle.hca_compress(kv, np.zeros((T, c)), 128, _fmt(c, 8, NO_NORM | NO_ROPE))
    assert np.allclose(ent, kv.reshape(2, 128, c).mean(axis=1), atol=1e-14)
    _, w = oracle.hca_compress(kv, z, 128, _fmt(c, 8), want_weights=True)
    assert np.allclose(w.sum(axis=1), 1.0, atol=1e-14)


def test_scalar_logits_broadcast():
    T, c, m = 64, 16, 4
    ca, cb, za, zb = rand(T, c), rand(T, c), rand(T, 1), rand(T, 1)
    f = _fmt(c, 8)
    a = oracle.csa_compress(ca, cb, za, zb, m, f)
    b = oracle.csa_compress(ca, cb, np.repeat(za, c, 1), np.repeat(zb, c, 1), m, f)
    assert np.array_equal(a, b)


def test_channel_permutation_equivariance():
    T, c, m = 64, 16, 4
    ca, cb, za, zb = rand(T, c), rand(T, c), rand(T, c), rand(T, c)
    perm = RNG.permutation(c)
    f = _fmt(c, 8, NO_NORM | NO_ROPE)
    a = oracle.csa_compress(ca, cb, za, zb, m, f)
    b = oracle.csa_compress(ca[:, perm], cb[:, perm], za[:, perm], zb[:, perm], m, f)
    assert np.allclose(a[:, perm], b, atol=1e-15)


def test_compress_position_shift_is_a_rotation():
    T, c, m = 64, 32, 4
    ca, cb, za, zb = rand(T, c), rand(T, c), rand(T, c), rand(T, c)
    a = oracle.csa_compress(ca, cb, za, zb, m, _fmt(c, 16), pos0=0)
    b = oracle.csa_compress(ca, cb, za, zb, m, _fmt(c, 16), pos0=40)
    for s in range(T // m):
        assert np.allclose(oracle.rope(a[s], 40, 16), b[s], atol=1e-12)


def test_compress_matches_brute_force():
    T, c, m, r = 96, 32, 4, 16
    ca, cb, za, zb = rand(T, c), rand(T, c), rand(T, c), rand(T, c)
    ent, w = oracle.csa_compress(ca, cb, za, zb, m, _fmt(c, r), pos0=8, want_weights=True)
    bent, bw = brute.csa_entries(ca, cb, za, zb, m, r, pos0=8)
    assert np.allclose(ent, bent, atol=1e-12)
    assert np.allclose(w, bw, atol=1e-14)
    kv, z = rand(512, c), rand(512, c)
    assert np.allclose(oracle.hca_compress(kv, z, 128, _fmt(c, r)),
                       brute.hca_entries(kv, z, 128, r)[0], atol=1e-12)
    win = oracle.window_rows(ca, _fmt(c, r), pos0=3)
    assert np.allclose(win, brute.transform(ca, 3 + np.arange(T), c, r, 1e4, 1e-6), atol=1e-12)


# ---------------------------------------------------------------- indexer, top-k

def test_indexer_integer_exact():
    T, HI, dI, m = 64, 3, 8, 4
    N = T // m
    qI = RNG.integers(-3, 4, (T, HI, dI)).astype(np.float64)
    kI = RNG.integers(-3, 4, (N, dI)).astype(np.float64)
    w = RNG.integers(-2, 3, (T, HI)).astype(np.float64)
    sc = oracle.indexer_scores(qI, w, kI, m)
    # exact integer arithmetic
    dots = np.einsum("thd,sd->ths", qI.astype(np.int64), kI.astype(np.int64))
    want = np.einsum("th,ths->ts", w.astype(np.int64), np.maximum(dots, 0))
    for t in range(T):
        v = (t + 1) // m
        assert np.array_equal(sc[t, :v], want[t, :v].astype(np.float64))
        assert np.all(np.isneginf(sc[t, v:]))


def test_indexer_golden_worked_example():
    with open(os.path.join(GOLDEN, "indexer_worked_example.json")) as fh:
        g = json.load(fh)
    sc = oracle.indexer_scores(np.array(g["q_I"], float), np.array(g["w"], float),
                               np.array(g["k_I"], float), g["m"], q_pos=g["q_pos"])
    want = np.array([[np.nan if v is None else v for v in row] for row in g["scores"]])
    fin = ~np.isnan(want)
    assert np.array_equal(sc[fin], want[fin])
    assert np.all(np.isneginf(sc[~fin]))
    idx = oracle.topk(sc, g["k"], g["m"], q_pos=g["q_pos"])
    assert idx.tolist() == g["idx"]


def test_indexer_relu_and_sign():
    T, HI, dI, m = 32, 4, 16, 4
    N = T // m
    kI = np.abs(rand(N, dI))
    qI = -np.abs(rand(T, HI, dI))     # every dot <= 0
    w = np.abs(rand(T, HI))
    sc = oracle.indexer_scores(qI, w, kI, m)
    fin = np.isfinite(sc)
    assert np.all(sc[fin] == 0.0)
    # flipping q_I's sign makes every dot positive: score = sum_h w . dot
    sc2 = oracle.indexer_scores(-qI, w, kI, m)
    want = np.einsum("th,ths->ts", w, np.einsum("thd,sd->ths", -qI, kI))
    assert np.allclose(sc2[fin], want[fin], rtol=1e-13)
    # linear in w
    sc3 = oracle.indexer_scores(-qI, 2.5 * w, kI, m)
    assert np.allclose(sc3[fin], 2.5 * sc2[fin], rtol=1e-13)


def test_indexer_matches_brute_force():
    T, HI, dI, m = 128, 4, 16, 4
    qI, kI, w = rand(T, HI, dI), rand(T // m, dI), rand(T, HI)
    assert np.allclose(oracle.indexer_scores(qI, w, kI, m), brute.indexer_scores(qI, w, kI, m),
                       rtol=1e-12, atol=1e-12)


def test_topk_brute_force_and_edges():
    T, N, m = 200, 50, 4
    sc = rand(T, N)
    vis = np.minimum((np.arange(T) + 1) // m, N)
    sc = np.where(np.arange(N)[None, :] < vis[:, None], sc, -np.inf)
    for k in (1, 7, 16, 50, 64):
        idx = oracle.topk(sc, k, m)
        assert np.array_equal(idx, brute.topk(sc, k))
    # k >= visible: everything visible, ascending, -1 padded
    idx = oracle.topk(sc, 64, m)
    for t in range(T):
        assert idx[t, : vis[t]].tolist() == list(range(vis[t]))
        assert np.all(idx[t, vis[t]:] == -1)
    # all-equal scores: ties go to the lower index
    eq = np.where(np.isfinite(sc), 0.0, -np.inf)
    idx = oracle.topk(eq, 5, m)
    assert idx[-1].tolist() == [0, 1, 2, 3, 4]
    # integer ties: equal scores straddling the cut keep the lower indices
    row = np.array([[3.0, 5.0, 3.0, 3.0, 5.0, 1.0, 3.0, 0.0]])
    assert oracle.topk(row, 4, 1, q_pos=[100]).tolist() == [[0, 1, 2, 4]]


# ---------------------------------------------------------------- attention

def _prefill_inputs(T=64, H=3, c=32, r=16, m=4, dI=8, HI=2, sink=True):
    return dict(
        kv_a=rand(T, c), kv_b=rand(T, c), z_a=rand(T, c), z_b=rand(T, c),
        q=rand(T, H, c), q_I=rand(T, HI, dI), k_I=rand(T // m, dI), w=rand(T, HI),
        sink=rand(H) if sink else None)


def test_attention_textbook_causal_softmax():
    """No entries, no sink, window >= T, no norm, no RoPE: plain causal
    softmax attention, as computed by torch's scaled_dot_product_attention."""
    T, H, c = 48, 3, 32
    q, win = rand(T, H, c), rand(T, c)
    out = oracle.attention(q, np.zeros((0, c)), win, _fmt(c, 16, NO_NORM | NO_ROPE), n_win=T,
                           idx=np.full((T, 1), -1), sink=None)
    qt = torch.from_numpy(q).permute(1, 0, 2)[None]           # [1, H, T, c]
    kv = torch.from_numpy(win)[None, None].expand(1, H, T, c)
    ref = torch.nn.functional.scaled_dot_product_attention(qt, kv, kv, is_causal=True)
    assert np.allclose(out, ref[0].permute(1, 0, 2).numpy(), atol=1e-12)
    # with the query RMSNorm (pinned above) still the textbook form
    out2 = oracle.attention(q, np.zeros((0, c)), win, _fmt(c, 16, NO_ROPE), n_win=T,
                            idx=np.full((T, 1), -1), sink=None)
    qn = torch.from_numpy(np.stack([[oracle.rmsnorm(q[t, h]) for h in range(H)]
                                    for t in range(T)])).permute(1, 0, 2)[None]
    ref2 = torch.nn.functional.scaled_dot_product_attention(qn, kv, kv, is_causal=True)
    assert np.allclose(out2, ref2[0].permute(1, 0, 2).numpy(), atol=1e-12)


def test_attention_sink_closed_form():
    T, H, c, m, k = 64, 4, 32, 4, 5
    inp = _prefill_inputs(T, H, c, 16, m)
    f = _fmt(c, 16)
    ent = oracle.csa_compress(inp["kv_a"], inp["kv_b"], inp["z_a"], inp["z_b"], m, f)
    win = oracle.window_rows(inp["kv_a"], f)
    idx = oracle.topk(oracle.indexer_scores(inp["q_I"], inp["w"], inp["k_I"], m), k, m)
    plain, lse = oracle.attention(inp["q"], ent, win, f, 16, idx=idx, sink=None, want_lse=True)
    sink = np.array([0.3, -2.0, 4.0, 1.5])
    o, lse2 = oracle.attention(inp["q"], ent, win, f, 16, idx=idx, sink=sink, want_lse=True)
    S = np.exp(lse)
    ratio = S / (S + np.exp(sink)[None, :])
    assert np.allclose(o, plain * ratio[:, :, None], atol=1e-13)
    assert np.allclose(np.exp(lse2), S + np.exp(sink)[None, :], rtol=1e-13)
    # a huge sink takes (almost) all the weight; -inf equals no sink
    o_big = oracle.attention(inp["q"], ent, win, f, 16, idx=idx, sink=np.full(H, 80.0))
    assert np.abs(o_big).max() < 1e-20
    o_neg = oracle.attention(inp["q"], ent, win, f, 16, idx=idx, sink=np.full(H, -np.inf))
    assert np.array_equal(o_neg, plain)


def test_attention_k_ge_visible_equals_dense():
    """With k >= the number of entries, CSA attends to every visible entry:
    the same as the dense (HCA-style) path over the same entries."""
    T, H, c, m = 64, 3, 32, 4
    inp = _prefill_inputs(T, H, c, 16, m)
    f = _fmt(c, 16)
    ent = oracle.csa_compress(inp["kv_a"], inp["kv_b"], inp["z_a"], inp["z_b"], m, f)
    win = oracle.window_rows(inp["kv_a"], f)
    idx = oracle.topk(oracle.indexer_scores(inp["q_I"], inp["w"], inp["k_I"], m), T // m, m)
    a = oracle.attention(inp["q"], ent, win, f, 8, idx=idx, sink=inp["sink"])
    b = oracle.attention(inp["q"], ent, win, f, 8, m_dense=m, sink=inp["sink"])
    assert np.allclose(a, b, atol=1e-13)


def test_attention_first_query_returns_its_own_row():
    """Query 0 sees no entry and only its own window row; with no sink the
    output is that row rotated back: RMSNorm(C^a[0])."""
    T, H, c, m = 16, 2, 32, 4
    inp = _prefill_inputs(T, H, c, 16, m, sink=False)
    f = _fmt(c, 16)
    ent = oracle.csa_compress(inp["kv_a"], inp["kv_b"], inp["z_a"], inp["z_b"], m, f)
    win = oracle.window_rows(inp["kv_a"], f)
    idx = oracle.topk(oracle.indexer_scores(inp["q_I"], inp["w"], inp["k_I"], m), 4, m)
    out = oracle.attention(inp["q"], ent, win, f, 4, idx=idx, sink=None)
    for h in range(H):
        assert np.allclose(out[0, h], oracle.rmsnorm(inp["kv_a"][0]), atol=1e-13)


def test_attention_translation_invariance():
    """Shifting every position (entries, window rows, queries) by D leaves the
    output unchanged: RoPE plus the inverse rotation make it relative."""
    T, H, c, m = 64, 2, 32, 4
    inp = _prefill_inputs(T, H, c, 16, m)
    f = _fmt(c, 16)
    idx = oracle.topk(oracle.indexer_scores(inp["q_I"], inp["w"], inp["k_I"], m), 6, m)
    outs = []
    for D in (0, 12, 100000):
        ent = oracle.csa_compress(inp["kv_a"], inp["kv_b"], inp["z_a"], inp["z_b"], m, f, pos0=D)
        win = oracle.window_rows(inp["kv_a"], f, pos0=D)
        outs.append(oracle.attention(inp["q"], ent, win, f, 8, idx=idx, sink=inp["sink"],
                                     q_pos=np.arange(T) + D, win_pos0=D))
    assert np.allclose(outs[0], outs[1], atol=1e-12)
    assert np.allclose(outs[0], outs[2], atol=1e-10)


def test_attention_matches_brute_force_dense_mask():
    T, H, c, r, m, n_win, k = 64, 3, 32, 16, 4, 8, 5
    inp = _prefill_inputs(T, H, c, r, m)
    f = _fmt(c, r)
    ent = oracle.csa_compress(inp["kv_a"], inp["kv_b"], inp["z_a"], inp["z_b"], m, f)
    win = oracle.window_rows(inp["kv_a"], f)
    idx = oracle.topk(oracle.indexer_scores(inp["q_I"], inp["w"], inp["k_I"], m), k, m)
    out = oracle.attention(inp["q"], ent, win, f, n_win, idx=idx, sink=inp["sink"])
    ref = brute.attention_dense(inp["q"], ent, win, idx, n_win, inp["sink"], c, r)
    assert np.allclose(out, ref, atol=1e-12)
    # dense HCA over m' = 8 entries
    kv, z = inp["kv_a"], inp["z_a"]
    hent = oracle.hca_compress(kv, z, 8, f)
    out = oracle.attention(inp["q"], hent, win, f, n_win, m_dense=8, sink=inp["sink"])
    ref = brute.attention_dense(inp["q"], hent, win, None, n_win, inp["sink"], c, r, m_dense=8)
    assert np.allclose(out, ref, atol=1e-12)


def test_csa_layer_end_to_end_brute_force():
    """The whole CSA layer (compress, indexer, top-k, attention) against the
    brute-force forms built from raw inputs."""
    T, H, c, r, m, n_win, k = 64, 2, 32, 16, 4, 8, 4
    inp = _prefill_inputs(T, H, c, r, m)
    f = _fmt(c, r)
    res = oracle.csa_layer(inp, f, m, k, n_win)
    ent, _ = brute.csa_entries(inp["kv_a"], inp["kv_b"], inp["z_a"], inp["z_b"], m, r)
    win = brute.transform(inp["kv_a"], np.arange(T), c, r, 1e4, 1e-6)
    idx = brute.topk(brute.indexer_scores(inp["q_I"], inp["w"], inp["k_I"], m), k)
    assert np.array_equal(res["idx"], idx)
    ref = brute.attention_dense(inp["q"], ent, win, idx, n_win, inp["sink"], c, r)
    assert np.allclose(res["out"], ref, atol=1e-12)
