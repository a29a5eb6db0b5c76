"""GPU parity of grouped_output_projection (two tcgen05 GEMMs: the grouped
projection to d_g per head group, then the projection of the concatenation
back to d) against the oracle's float64 restatement."""
import numpy as np
import pytest
import torch

import oracle
from parity import assert_close, f64
import long_context_attention_csa_b200 as csa
from long_context_attention_csa_b200 import workloads as wl

pytestmark = pytest.mark.gpu

DEV = "cuda"


def _case(T, H, g, dg, d, seed=0):
    w = wl.scaled(wl.WORKLOADS["csa_prefill_8k"], T=T, H=H, seed=seed)
    return w, wl.projection_inputs(w, g, dg, d, DEV)


@pytest.mark.parametrize("T,H,g,dg,d", [
    (300, 16, 4, 256, 512),      # several tiles in every direction, a ragged row tail
    (129, 8, 2, 96, 160),        # output widths that end inside a 256-column tile
    (1, 64, 8, 1024, 4096),      # one row (decode) at the workload's sizes
])
def test_projection_small(T, H, g, dg, d):
    w, x = _case(T, H, g, dg, d, seed=T)
    y = csa.grouped_output_projection(x["o"], x["w_group"], x["w_out"])
    torch.cuda.synchronize()
    ref = oracle.grouped_output_projection(f64(x["o"]), f64(x["w_group"]), f64(x["w_out"]))
    # v is rounded to bf16 between the GEMMs, y once more on the way out
    assert_close(y, ref, torch.bfloat16, "grouped projection", roundings=2)


def test_projection_csa_prefill_8k_sampled():
    """The workload's projection (8192 rows, 64 heads x 512, g = 8, d_g = 1024,
    d = 4096) as the benchmark runs it, checked on sampled rows."""
    p = wl.PROJ
    w, x = _case(8192, 64, p["g"], p["d_g"], p["d"])
    y = csa.grouped_output_projection(x["o"], x["w_group"], x["w_out"])
    torch.cuda.synchronize()
    rows = np.array(sorted(set([0, 1, 127, 128, 4095, 8190, 8191] +
                               np.random.default_rng(0).choice(8192, 33, replace=False).tolist())))
    ref = oracle.grouped_output_projection(f64(x["o"][rows]), f64(x["w_group"]), f64(x["w_out"]))
    assert_close(y[rows], ref, torch.bfloat16, "grouped projection 8k rows", roundings=2)


def test_projection_rows_do_not_depend_on_the_batch():
    """A row's result is the same bits alone and inside 300 rows (each output
    tile sums its full K in one fixed order)."""
    w, x = _case(300, 16, 4, 256, 512, seed=3)
    y = csa.grouped_output_projection(x["o"], x["w_group"], x["w_out"])
    for r in (0, 137, 299):
        one = csa.grouped_output_projection(x["o"][r:r + 1].contiguous(), x["w_group"],
                                            x["w_out"])
        torch.cuda.synchronize()
        assert torch.equal(one[0], y[r])
