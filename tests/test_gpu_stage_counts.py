"""GPU parity of the weight-only GEMM at the stage counts a tile can have.

The edge cases of the MMA pipeline: tiles of one stage (the accumulators are
written only by that stage's first MMAs), one partial stage (K below 128),
odd stage counts (the TMEM operand ring of three slots wraps mid-tile), and
persistent CTAs running several whole tiles (the ring positions carry over
from tile to tile while each tile restarts its accumulators).  Each case is
checked against the fp64 oracle, and the plan is checked to run the stage
count the case is meant to exercise."""

import numpy as np
import pytest

import weight_only_quantized_prologue_b200 as dq
from oracle import linear as L
from weight_only_quantized_prologue_b200 import synthetic

from gpu_util import bf16_values, check_close, make_layer, run

pytestmark = pytest.mark.gpu

WO_FORMATS = ["int4", "nvfp4", "mxfp4", "fp8", "int4_asym"]


def _case(fmt, M, K, N, seed):
    x, w, b = synthetic.linear_inputs(M, K, N, seed=seed)
    W = w.numpy().astype(np.float64)
    h, st, wdq = make_layer(fmt, W, b.cuda())
    try:
        plan = dq.dqgemm_get_plan(h, M)
        y = bf16_values(run(h, x.cuda(), N))
        xv = bf16_values(x)
        check_close(y, L.linear_ref(xv, wdq, bf16_values(b)), xv, wdq)
    finally:
        dq.dqgemm_destroy(h)
    return plan


@pytest.mark.parametrize("fmt", WO_FORMATS)
@pytest.mark.parametrize("M,N", [(1, 256), (32, 384), (17, 1024), (100, 512)])
def test_one_stage_tiles(fmt, M, N):
    """K = 128: every tile is one stage."""
    plan = _case(fmt, M, 128, N, seed=M)
    assert plan["k_stages"] == 1 and plan["bn"] <= 128


@pytest.mark.parametrize("fmt", ["nvfp4", "mxfp4", "fp8"])
@pytest.mark.parametrize("M,K", [(32, 64), (100, 96)])
def test_one_partial_stage_tiles(fmt, M, K):
    """K < 128 (formats whose blocks allow it): one partial stage per tile."""
    plan = _case(fmt, M, K, 384, seed=K)
    assert plan["k_stages"] == 1 and plan["bn"] <= 128


@pytest.mark.parametrize("fmt", WO_FORMATS)
@pytest.mark.parametrize("M,K", [(5, 384), (40, 640), (64, 1152)])
def test_odd_stage_counts(fmt, M, K):
    """3, 5 or 9 stages per tile (160 output tiles, too many to split K)."""
    plan = _case(fmt, M, K, 20480, seed=K)
    assert plan["max_segments"] == 1 and plan["k_stages"] % 2 == 1 and plan["bn"] <= 128


@pytest.mark.parametrize("fmt", ["int4", "fp8"])
@pytest.mark.parametrize("K", [128, 384])
def test_persistent_tiles(fmt, K):
    """128-row x tiles, more output tiles (160) than SMs, so CTAs run whole
    tiles in a persistent loop: one stage per tile, and three (the operand
    ring wraps across tiles)."""
    plan = _case(fmt, 100, K, 20480, seed=K)
    assert plan["max_segments"] == 1 and plan["bn"] == 128
    assert plan["m_tiles"] * plan["n_tiles"] > plan["grid"]
