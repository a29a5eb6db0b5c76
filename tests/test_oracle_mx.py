"""Pins for the oracle's block-scaled FP8 path (the next step of the
indexer: low-precision QK, page "DeepSeek-V4：迈向高效百万 Token 上下文智能",
§3.3, last paragraph).  Format facts of FP8 E4M3 (FN variant) and of the OCP
Microscaling (MX) block scale; the encoder is pinned by its round trip, its
ties, its error bound, its monotonicity and its saturation."""
import math

import numpy as np
import pytest

import oracle


def test_e4m3_format_values():
    v = oracle.e4m3_value
    assert v(0x38) == 1.0 and v(0xC0) == -2.0
    assert v(0x7E) == 448.0 and v(0xFE) == -448.0      # largest finite
    assert v(0x08) == 2.0 ** -6                        # smallest normal
    assert v(0x01) == 2.0 ** -9                        # smallest subnormal
    assert v(0x07) == 7 * 2.0 ** -9                    # largest subnormal
    assert v(0x00) == 0.0 and math.copysign(1.0, v(0x80)) == -1.0
    assert math.isnan(v(0x7F)) and math.isnan(v(0xFF))
    finite = [v(c) for c in range(0x7F)]
    assert all(a < b for a, b in zip(finite, finite[1:]))   # codes are ordered


def test_e4m3_round_trip_every_finite_code():
    for c in list(range(0x00, 0x7F)) + list(range(0x80, 0xFF)):
        assert oracle.e4m3_encode(oracle.e4m3_value(c)) == c, hex(c)
    assert oracle.e4m3_encode(-0.0) == 0x80          # the sign of zero is kept
    assert oracle.e4m3_encode(float("nan")) == 0x7F


def test_e4m3_ties_go_to_the_even_code():
    for c in range(0x7E):
        lo, hi = oracle.e4m3_value(c), oracle.e4m3_value(c + 1)
        mid = (lo + hi) / 2
        want = c if c % 2 == 0 else c + 1
        assert oracle.e4m3_encode(mid) == want, hex(c)
        assert oracle.e4m3_encode(-mid) == (want | 0x80)   # sign kept, -0 included


def test_e4m3_error_bound_and_monotonicity():
    rng = np.random.default_rng(7)
    xs = np.concatenate([rng.uniform(-448, 448, 3000),
                         np.exp(rng.uniform(np.log(2.0 ** -12), np.log(448), 3000))])
    for x in xs:
        y = oracle.e4m3_value(oracle.e4m3_encode(x))
        if abs(x) >= 2.0 ** -6:
            assert abs(y - x) <= 2.0 ** -4 * abs(x)    # half an ulp of 3 mantissa bits
        else:
            assert abs(y - x) <= 2.0 ** -10            # half the subnormal spacing
    sweep = np.linspace(-460, 460, 20001)
    codes = [oracle.e4m3_value(oracle.e4m3_encode(x)) for x in sweep]
    assert all(a <= b for a, b in zip(codes, codes[1:]))


def test_e4m3_encode_equals_torch_float8_conversion():
    """Against an independent implementation, torch's float32 -> float8_e4m3fn
    conversion (IEEE rounding to nearest even, sign of zero kept), over the
    subnormals, the normals and ties, below the first value that overflows
    (464, halfway to the unrepresentable 480)."""
    import torch

    rng = np.random.default_rng(11)
    xs = np.concatenate([np.linspace(-2.0 ** -5, 2.0 ** -5, 4001), rng.standard_normal(4000) * 50,
                         [(oracle.e4m3_value(c) + oracle.e4m3_value(c + 1)) / 2 * sg
                          for c in range(0x7E) for sg in (1, -1)], [-0.0, 0.0, 460.0, -460.0]])
    xs = xs[np.abs(xs) < 464].astype(np.float32)
    want = torch.from_numpy(xs).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    got = np.array([oracle.e4m3_encode(float(x)) for x in xs])
    assert np.array_equal(got, want)


def test_e4m3_saturates():
    assert oracle.e4m3_encode(449.0) == 0x7E
    assert oracle.e4m3_encode(480.0) == 0x7E
    assert oracle.e4m3_encode(1e30) == 0x7E
    assert oracle.e4m3_encode(-1e30) == 0xFE


@pytest.mark.parametrize("amax,exp", [(1.0, -8), (3.0, -7), (0.75, -9), (448.0, 0), (2.0 ** -20, -28)])
def test_mx_block_scale(amax, exp):
    x = np.zeros(32)
    x[5] = -amax
    codes, exps = oracle.mxfp8_quantize(x)
    assert exps.tolist() == [exp]
    y = oracle.mxfp8_dequantize(codes, exps)
    assert y[5] == -amax and np.all(np.delete(y, 5) == 0)   # powers of two and 3 are exact


def test_mx_zero_block_and_clipping_of_the_top_of_a_block():
    codes, exps = oracle.mxfp8_quantize(np.zeros(64))
    assert exps.tolist() == [-127, -127] and not codes.any()
    # amax 31: scale 2^(4-8), 31 * 16 = 496 lies above 448 and clips to 448
    x = np.arange(32, dtype=np.float64)[::-1].copy()
    y = oracle.mxfp8_dequantize(*oracle.mxfp8_quantize(x))
    assert y[0] == 28.0
    # at this scale the codes step by 1 up to 16 and by 2 from 16 to 28 (ties even)
    small = x <= 16
    assert np.array_equal(y[small], x[small])
    mid = (x > 16) & (x <= 28)
    assert np.all(np.abs(y[mid] - x[mid]) <= 1.0) and np.all(y[mid] % 2 == 0)
    assert np.all(y[x > 28] == 28.0)   # 29 * 16 = 464 and up clip to 448


def test_mx_blocks_are_independent_and_bounded():
    rng = np.random.default_rng(3)
    x = rng.standard_normal((4, 128))
    x[1, 32:64] *= 1000.0                                    # one loud block
    codes, exps = oracle.mxfp8_quantize(x)
    y = oracle.mxfp8_dequantize(codes, exps)
    for r in range(4):
        for b in range(4):
            blk, got = x[r, 32 * b:32 * b + 32], y[r, 32 * b:32 * b + 32]
            X = 2.0 ** exps[r, b]
            assert X == 2.0 ** (math.floor(math.log2(np.abs(blk).max())) - 8)
            inner = (np.abs(blk) >= X * 2.0 ** -6) & (np.abs(blk) <= 448 * X)
            assert np.all(np.abs(got - blk)[inner] <= 2.0 ** -4 * np.abs(blk)[inner])
            assert np.all(np.abs(got - blk)[~inner & (np.abs(blk) < X * 2.0 ** -6)] <= X * 2.0 ** -10)


def test_mx_indexer_top_k_recall_on_the_workload_distribution():
    """Not a pin but the property the low-precision path is judged by: top-k
    recall against the float64 selection, on the workloads' distributions
    (q_I and K_I N(0,1)/sqrt(d_I), w N(0,1)/8)."""
    rng = np.random.default_rng(0)
    T, HI, dI, N, m, k = 256, 64, 128, 64, 4, 16
    q = rng.standard_normal((T, HI, dI)) / np.sqrt(dI)
    kk = rng.standard_normal((N, dI)) / np.sqrt(dI)
    w = rng.standard_normal((T, HI)) / 8
    a = oracle.topk(oracle.indexer_scores(q, w, kk, m), k, m)
    b = oracle.topk(oracle.mxfp8_indexer_scores(q, w, kk, m), k, m)
    rec = [len(set(a[t][a[t] >= 0]) & set(b[t][b[t] >= 0])) / max(1, (a[t] >= 0).sum())
           for t in range(T) if (a[t] >= 0).any()]
    assert np.mean(rec) >= 0.95


# ---------------------------------------------------------------- FP4 (E2M1)

def test_e2m1_format_values():
    mags = [oracle.e2m1_value(c) for c in range(8)]
    assert mags == [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]
    assert [oracle.e2m1_value(8 + c) for c in range(1, 8)] == [-x for x in mags[1:]]


def test_e2m1_round_trip_ties_and_saturation():
    for c in list(range(8)) + list(range(9, 16)):
        assert oracle.e2m1_encode(oracle.e2m1_value(c)) == c
    # midpoints go to the code with an even mantissa bit
    ties = {0.25: 0.0, 0.75: 1.0, 1.25: 1.0, 1.75: 2.0, 2.5: 2.0, 3.5: 4.0, 5.0: 4.0}
    for x, want in ties.items():
        assert oracle.e2m1_value(oracle.e2m1_encode(x)) == want, x
        assert oracle.e2m1_value(oracle.e2m1_encode(-x)) == -want, x
    for x in (6.5, 7.0, 100.0):
        assert oracle.e2m1_value(oracle.e2m1_encode(x)) == 6.0
        assert oracle.e2m1_value(oracle.e2m1_encode(-x)) == -6.0
    sweep = np.linspace(-8, 8, 4001)
    vals = [oracle.e2m1_value(oracle.e2m1_encode(x)) for x in sweep]
    assert all(a <= b for a, b in zip(vals, vals[1:]))
    for x in sweep:   # nearest: no magnitude is closer than the chosen one
        y = oracle.e2m1_value(oracle.e2m1_encode(x))
        best = min(abs(abs(x) - v) for v in [0, 0.5, 1, 1.5, 2, 3, 4, 6])
        assert abs(abs(y) - min(abs(x), 6.0)) <= best + 1e-12 or abs(x) > 6


@pytest.mark.parametrize("amax,exp", [(1.0, -2), (6.0, 0), (0.3, -4), (2.0 ** 10, 8), (5.0, 0)])
def test_mxfp4_block_scale(amax, exp):
    x = np.zeros(32)
    x[9] = amax
    codes, exps = oracle.mxfp4_quantize(x)
    assert exps.tolist() == [exp]
    y = oracle.mxfp4_dequantize(codes, exps)
    # amax / X lies in [4, 8): it is exact when it is a code (4 or 6), else it
    # rounds to the nearest code (5 is a tie: to 4, the even code) or clips to 6
    r = amax / 2.0 ** exp
    want = min((4.0, 6.0), key=lambda v: abs(v - r)) if r < 7 else 6.0
    assert y[9] == want * 2.0 ** exp


def test_mx_fp4_indexer_top_k_recall_on_the_workload_distribution():
    rng = np.random.default_rng(0)
    T, HI, dI, N, m, k = 256, 64, 128, 64, 4, 16
    q = rng.standard_normal((T, HI, dI)) / np.sqrt(dI)
    kk = rng.standard_normal((N, dI)) / np.sqrt(dI)
    w = rng.standard_normal((T, HI)) / 8
    a = oracle.topk(oracle.indexer_scores(q, w, kk, m), k, m)
    b = oracle.topk(oracle.mxfp4_indexer_scores(q, w, kk, m), k, m)
    rec = [len(set(a[t][a[t] >= 0]) & set(b[t][b[t] >= 0])) / max(1, (a[t] >= 0).sum())
           for t in range(T) if (a[t] >= 0).any()]
    assert np.mean(rec) >= 0.90


# ------------------------------------------- FP4 with 16-element E4M3 scales

def test_nvfp4_tensor_and_block_scales():
    rng = np.random.default_rng(9)
    x = rng.standard_normal(64)
    x[37] = 5.0 * np.abs(x).max()                 # the tensor's amax
    codes, scales, g = oracle.nvfp4_quantize(x)
    assert g == np.abs(x).max() / (448.0 * 6.0)
    assert scales.shape == (4,) and oracle.e4m3_value(scales[37 // 16]) == 448.0
    y = oracle.nvfp4_dequantize(codes, scales, g)
    assert y[37] == x[37]                         # amax -> code 6 under scale 448


def test_nvfp4_block_of_representable_values_is_exact():
    # E2M1 magnitudes times 0.25 in one block, 336 in the next: the tensor
    # scale is 336 / 2688 = 1/8, the first block's scale 1.5 / (6 / 8) = 2
    # (an E4M3 value), so every element is exact
    blk = np.array([0, 0.5, 1, 1.5, 2, 3, 4, 6, -6, -4, -3, -2, -1.5, -1, -0.5, 0]) * 0.25
    x2 = np.concatenate([blk, np.r_[336.0, np.zeros(15)]])
    c2, s2, g2 = oracle.nvfp4_quantize(x2)
    assert g2 == 0.125 and oracle.e4m3_value(s2[0]) == 2.0
    assert np.array_equal(oracle.nvfp4_dequantize(c2, s2, g2), x2)


def test_nvfp4_zero_tensor():
    z, zs, zg = oracle.nvfp4_quantize(np.zeros(32))
    assert not z.any() and not zs.any() and zg == 1.0


def test_nvfp4_indexer_top_k_recall_on_the_workload_distribution():
    rng = np.random.default_rng(0)
    T, HI, dI, N, m, k = 256, 64, 128, 64, 4, 16
    q = rng.standard_normal((T, HI, dI)) / np.sqrt(dI)
    kk = rng.standard_normal((N, dI)) / np.sqrt(dI)
    w = rng.standard_normal((T, HI)) / 8
    a = oracle.topk(oracle.indexer_scores(q, w, kk, m), k, m)
    b = oracle.topk(oracle.nvfp4_indexer_scores(q, w, kk, m), k, m)
    rec = [len(set(a[t][a[t] >= 0]) & set(b[t][b[t] >= 0])) / max(1, (a[t] >= 0).sum())
           for t in range(T) if (a[t] >= 0).any()]
    assert np.mean(rec) >= 0.90
