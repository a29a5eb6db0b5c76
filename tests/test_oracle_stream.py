"""Pins for the oracle's streaming compression (decode appends one token at a
time; the KV of an unfinished block waits until the block completes, page
"DeepSeek-V4：迈向高效百万 Token 上下文智能", §3.5).  Streaming must reproduce
the batch compression exactly, emit entry s on token m(s+1)-1, and carry the
previous block's group-b rows across the block boundary."""
import numpy as np
import pytest

import oracle


def _stream(m, fmt, arrays, overlap, pos0):
    ca, za, cb, zb = arrays
    st = oracle.Stream(m, fmt, za.shape[1], overlap=overlap, pos0=pos0)
    wins, ents = [], []
    for t in range(ca.shape[0]):
        w, e = st.append(ca[t], za[t], cb[t] if overlap else None, zb[t] if overlap else None)
        wins.append(w)
        if e is not None:
            ents.append((t, e))
    return np.stack(wins), ents


@pytest.mark.parametrize("T,m,zc,pos0", [(37, 4, 64, 5), (16, 4, 1, 0), (3, 4, 64, 0), (41, 2, 64, 100)])
def test_csa_stream_equals_batch(T, m, zc, pos0):
    rng = np.random.default_rng(T * 31 + m)
    c = 64
    fmt = oracle.Fmt(c=c, rope_dims=32)
    ca, cb = rng.standard_normal((T, c)), rng.standard_normal((T, c))
    za, zb = rng.standard_normal((T, zc)), rng.standard_normal((T, zc))
    wins, ents = _stream(m, fmt, (ca, za, cb, zb), True, pos0)
    ref = oracle.csa_compress(ca, cb, za, zb, m, fmt, pos0=pos0)
    assert [t for t, _ in ents] == [m * (s + 1) - 1 for s in range(T // m)]
    if T // m:
        assert np.array_equal(np.stack([e for _, e in ents]), ref)
    assert np.array_equal(wins, oracle.window_rows(ca, fmt, pos0=pos0))


@pytest.mark.parametrize("T,mp", [(70, 8), (16, 16), (5, 8)])
def test_hca_stream_equals_batch(T, mp):
    rng = np.random.default_rng(T + mp)
    c = 64
    fmt = oracle.Fmt(c=c, rope_dims=16)
    kv, z = rng.standard_normal((T, c)), rng.standard_normal((T, c))
    wins, ents = _stream(mp, fmt, (kv, z, None, None), False, 0)
    ref = oracle.hca_compress(kv, z, mp, fmt)
    assert [t for t, _ in ents] == [mp * (s + 1) - 1 for s in range(T // mp)]
    if T // mp:
        assert np.array_equal(np.stack([e for _, e in ents]), ref)
    assert np.array_equal(wins, oracle.window_rows(kv, fmt))


def test_stream_carries_the_previous_block_b_rows():
    """Block 0's group-b rows do not touch entry 0 and are what entry 1 pools."""
    rng = np.random.default_rng(5)
    T, c, m = 8, 32, 4
    fmt = oracle.Fmt(c=c, rope_dims=0, flags=oracle.NO_NORM | oracle.NO_ROPE)
    ca, cb = rng.standard_normal((T, c)), rng.standard_normal((T, c))
    za, zb = np.zeros((T, c)), np.zeros((T, c))
    cb2 = cb.copy()
    cb2[:m] += 100.0
    _, e1 = _stream(m, fmt, (ca, za, cb, zb), True, 0)
    _, e2 = _stream(m, fmt, (ca, za, cb2, zb), True, 0)
    assert np.array_equal(e1[0][1], e2[0][1])
    # uniform logits: entry 1 is the mean of block 1's a rows and block 0's b rows
    assert np.allclose(e1[1][1], (ca[m:2 * m].sum(0) + cb[:m].sum(0)) / (2 * m))
    assert np.allclose(e2[1][1] - e1[1][1], 100.0 * m / (2 * m))
