"""Comparison helpers for GPU-vs-oracle parity.

Tolerances (floating point): bf16 outputs max-abs <= 2e-2 and rel-L2 <= 5e-3;
float32 outputs max-abs <= 1e-4 and rel-L2 <= 1e-4.  Top-k sets: bit-exact on
integer-valued inputs; otherwise they may differ only in entries whose oracle
score lies within 1e-3 (relative) of the oracle's k-th score.

A bf16-stored value cannot be nearer its exact value than its own rounding:
half a bf16 ulp, which exceeds 2e-2 once |value| >= 8.  So the per-element
bf16 bound is max(2e-2, n * ulp/2 + 2^-16 |ref|) for a result rounded to bf16
n times on its way out (n = 1 for one kernel's output, 2 for a chain that
stores an intermediate in bf16); 2^-16 |ref| covers the float32 arithmetic
before the rounding.  Every comparison records its worst error in bf16 ulps
of the reference (over elements with |ref| >= 1), reported at the end of the
run.
"""
import os

import numpy as np
import torch

TOL = {torch.bfloat16: (2e-2, 5e-3), torch.float32: (1e-4, 1e-4)}
TOPK_REL = 1e-3


def f64(t) -> np.ndarray:
    if isinstance(t, np.ndarray):
        return t.astype(np.float64)
    return t.detach().to("cpu", torch.float64).numpy()


def errors(gpu, ref):
    g, r = f64(gpu), f64(ref)
    d = g - r
    max_abs = float(np.abs(d).max()) if d.size else 0.0
    rel = float(np.linalg.norm(d.ravel()) / max(np.linalg.norm(r.ravel()), 1e-30))
    return max_abs, rel


def bf16_ulp(x: np.ndarray) -> np.ndarray:
    """One bf16 unit in the last place at |x| (8 significant bits)."""
    ax = np.maximum(np.abs(x), np.finfo(np.float32).tiny)
    return np.exp2(np.floor(np.log2(ax)) - 7)


# (what, worst error in bf16 ulps over |ref| >= 1, max-abs, rel-L2) of every comparison
ULP_LOG = []


def assert_close(gpu, ref, dtype, what="", roundings=1):
    """Element-wise |gpu - ref| <= max(tol_abs, roundings x half a bf16 ulp of
    ref + 2^-16 |ref|) for bf16 outputs, <= tol_abs for float32; and
    rel-L2 <= tol_rel over the whole tensor."""
    tol_abs, tol_rel = TOL[dtype]
    g, r = f64(gpu), f64(ref)
    assert np.isfinite(g).all(), f"{what}: non-finite GPU output"
    max_abs, rel = errors(g, r)
    ulp = bf16_ulp(r)
    big = np.abs(r) >= 1.0
    worst_ulps = float((np.abs(g - r)[big] / ulp[big]).max()) if big.any() else 0.0
    test = os.environ.get("PYTEST_CURRENT_TEST", "").split(" ")[0].split("::")[-1]
    ULP_LOG.append((f"{test}: {what}", worst_ulps, max_abs, rel))
    bound = (np.maximum(tol_abs, roundings * 0.5 * ulp + np.ldexp(np.abs(r), -16))
             if dtype == torch.bfloat16 else tol_abs)
    excess = np.abs(g - r) - bound
    worst = float(excess.max()) if excess.size else -1.0
    assert worst <= 0 and rel <= tol_rel, (
        f"{what}: max_abs {max_abs:.3e} (bound max({tol_abs}, {roundings} x ulp/2), worst "
        f"excess {worst:.3e}, worst {worst_ulps:.3f} ulp), rel_l2 {rel:.3e} (tol {tol_rel})")
    return max_abs, rel


def check_topk_rows(gpu_idx, ref_idx, ref_scores, exact=False, what=""):
    """gpu_idx, ref_idx: [R, k] int; ref_scores: [R, N] oracle scores (-inf
    beyond visibility).  Returns the number of rows whose sets differ."""
    gpu_idx = np.asarray(gpu_idx)
    ref_idx = np.asarray(ref_idx)
    differing = 0
    for r in range(ref_idx.shape[0]):
        g, o = gpu_idx[r], ref_idx[r]
        # structure: ascending valid indices then -1 padding, same count
        gv, ov = g[g >= 0], o[o >= 0]
        assert len(gv) == len(ov), f"{what} row {r}: {len(gv)} vs {len(ov)} selected"
        assert np.all(g[len(gv):] == -1), f"{what} row {r}: padding not -1"
        assert np.all(np.diff(gv) > 0), f"{what} row {r}: not strictly ascending"
        if np.array_equal(g, o):
            continue
        assert not exact, f"{what} row {r}: sets differ on exact inputs"
        differing += 1
        sc = ref_scores[r]
        tau = np.sort(sc[ov])[0]           # oracle k-th score
        band = TOPK_REL * max(abs(tau), 1e-30)
        for s in np.setxor1d(gv, ov):
            assert abs(sc[s] - tau) <= band, (
                f"{what} row {r}: entry {s} score {sc[s]} outside the tie band of {tau}")
    return differing
