"""Pins for the oracle's grouped output projection (the next step after the
attention: page "DeepSeek-V4：迈向高效百万 Token 上下文智能", §3.3, CSA
paragraph)."""
import numpy as np

import oracle


def test_grouped_projection_is_one_block_diagonal_matrix():
    rng = np.random.default_rng(4)
    T, H, c, g, dg, d = 3, 8, 16, 4, 12, 20
    o = rng.standard_normal((T, H, c))
    wg = rng.standard_normal((g, dg, (H // g) * c))
    wo = rng.standard_normal((d, g * dg))
    # the same map as one matrix: block-diagonal group weights, then w_out
    bd = np.zeros((g * dg, H * c))
    for j in range(g):
        bd[j * dg:(j + 1) * dg, j * (H // g) * c:(j + 1) * (H // g) * c] = wg[j]
    want = o.reshape(T, H * c) @ bd.T @ wo.T
    assert np.allclose(oracle.grouped_output_projection(o, wg, wo), want, rtol=1e-12, atol=1e-12)


def test_grouped_projection_with_selector_weights_reads_the_right_heads():
    """Group j's weights pick one dim of one head: the output then lists the
    picked values, so a wrong grouping or transposed operand shows."""
    T, H, c, g = 2, 6, 4, 3
    o = np.arange(T * H * c, dtype=np.float64).reshape(T, H, c)
    hpg = H // g
    wg = np.zeros((g, 1, hpg * c))
    for j in range(g):
        wg[j, 0, (j % hpg) * c + (j % c)] = 1.0   # head j*hpg + j%hpg, dim j%c
    wo = np.eye(g)
    y = oracle.grouped_output_projection(o, wg, wo)
    for t in range(T):
        for j in range(g):
            assert y[t, j] == o[t, j * hpg + j % hpg, j % c]
