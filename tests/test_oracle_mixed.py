"""Pins for the oracle's mixed-precision entry storage (the next step of the
KV cache: RoPE dims in BF16, the rest in FP8, page "DeepSeek-V4：迈向高效百万
Token 上下文智能", §3.3, last paragraph).  BF16 rounding against closed forms
and against torch's float32 -> bfloat16 conversion; the storage split
against its two parts."""
import numpy as np
import pytest
import torch

import oracle


def test_bf16_closed_forms():
    r = oracle.bf16_round
    assert r(1.0 + 2.0 ** -8) == 1.0                      # tie between 1 and 1 + 2^-7: even
    assert r(1.0 + 3 * 2.0 ** -8) == 1.0 + 2.0 ** -6      # tie: to the even neighbour above
    assert r(1.0 + 2.0 ** -8 + 2.0 ** -30) == 1.0 + 2.0 ** -7   # just above the tie
    assert r(-2.5) == -2.5 and r(0.0) == 0.0
    big = (2.0 - 2.0 ** -7) * 2.0 ** 127                   # largest finite
    assert r(big) == big and r(2.0 ** 128) == np.inf and r(-2.0 ** 128) == -np.inf
    assert r(2.0 ** -133) == 2.0 ** -133                   # smallest subnormal
    assert r(1.5 * 2.0 ** -133) == 2.0 ** -132             # subnormal tie: even


def test_bf16_matches_torch_on_float32_values():
    rng = np.random.default_rng(11)
    x = np.concatenate([rng.standard_normal(4000), rng.standard_normal(1000) * 1e30,
                        rng.standard_normal(1000) * 1e-38]).astype(np.float32)
    want = torch.from_numpy(x).to(torch.bfloat16).to(torch.float64).numpy()
    got = np.array([oracle.bf16_round(float(v)) for v in x])
    assert np.array_equal(got, want)


def test_mixed_store_splits_the_entry():
    rng = np.random.default_rng(2)
    n, c, r = 5, 512, 64
    x = rng.standard_normal((n, c)) * np.exp(rng.uniform(-3, 3, (n, 1)))
    codes, exps, rope = oracle.mixed_store(x, r)
    assert codes.shape == (n, c - r) and exps.shape == (n, (c - r) // 32) and rope.shape == (n, r)
    assert np.array_equal(rope, np.vectorize(oracle.bf16_round)(x[:, c - r:]))
    y = oracle.mixed_load(codes, exps, rope)
    assert np.array_equal(y[:, :c - r], oracle.mxfp8_dequantize(*oracle.mxfp8_quantize(x[:, :c - r])))
    assert np.array_equal(y[:, c - r:], rope)


def test_attention_over_mixed_entries_stays_close():
    """Not a pin: the accuracy cost the storage format carries (unit-RMS
    entries, 3 mantissa bits on 448 of 512 dims)."""
    rng = np.random.default_rng(0)
    c, r, N, T, H = 512, 64, 64, 64, 8
    f = oracle.Fmt(c=c, rope_dims=r)
    ent, win = rng.standard_normal((N, c)), rng.standard_normal((T, c))
    q = rng.standard_normal((T, H, c))
    ml = oracle.mixed_load(*oracle.mixed_store(ent, r))
    a = oracle.attention(q, ent, win, f, 16, m_dense=1, q_pos=np.arange(T))
    b = oracle.attention(q, ml, win, f, 16, m_dense=1, q_pos=np.arange(T))
    assert np.linalg.norm(a - b) / np.linalg.norm(a) < 0.05
