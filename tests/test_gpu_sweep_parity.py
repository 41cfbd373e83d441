"""GPU parity at the sweep's sizes, against the fp64 oracle.

The throughput sweep runs M in {1, 16, 32, 128, 1024, 4096} over (K, N) in
{(4096, 4096), (4096, 14336), (14336, 4096)}; these cases run the same paths
under an oracle check: long K on the split-K path (up to 14 stages per CTA),
wide N on the whole-tile path (more output tiles than SMs at M=32), the
128-row tile on the split path, and M=1024 (256 output tiles over the SMs,
64 stages per CTA), compared on a seeded sample of 256 rows.  Every case
asserts through the launch plan that a CTA streams more weight stages than
its weight ring holds, so the ring's wrap (its slot-free waits and phase
flips) runs under the check, and the x ring wraps where the plan says it
must.  Weights ~U(+-1/sqrt(K)), x ~N(0, 1), bf16 bias, as the sweep draws
them ("Define a linear model ..." on each weight-only page)."""

import functools

import numpy as np
import pytest
import torch

import weight_only_quantized_prologue_b200 as dq
from oracle import linear as L
from weight_only_quantized_prologue_b200 import synthetic

from gpu_util import bf16_values, check_close, dev, scales_tensor, static_effective_x

pytestmark = pytest.mark.gpu

FORMATS = ["int4", "nvfp4", "mxfp4", "fp8", "int4_asym", "fp8_static"]
# (M, K, N, rows compared)
CASES = [(1, 14336, 4096, None), (16, 14336, 4096, None), (32, 4096, 14336, None), (128, 4096, 4096, None),
         (1024, 4096, 4096, 256)]


@functools.lru_cache(maxsize=3)
def _weights(K, N):
    _, w, b = synthetic.linear_inputs(1, K, N, seed=K + N)
    return w.numpy().astype(np.float64), b


@functools.lru_cache(maxsize=3)
def _storage(fmt, K, N):
    W, _ = _weights(K, N)
    base = "fp8" if fmt == "fp8_static" else fmt
    st = L.quantize_pack(base, W)
    return st, L.dequant_exact(base, st["packed"], st["scales"], st["global_scale"])


@pytest.mark.parametrize("M,K,N,rows", CASES)
@pytest.mark.parametrize("fmt", FORMATS)
def test_sweep_shapes_match_oracle(fmt, M, K, N, rows):
    st, wdq = _storage(fmt, K, N)
    _, b = _weights(K, N)
    x = synthetic.activations(M, K, seed=M + 7)
    xv = bf16_values(x)
    s_x = L.act_scale(xv.min(), xv.max())
    g = s_x if fmt == "fp8_static" else st["global_scale"]
    bias = None if fmt == "fp8_static" else b.cuda()
    h = dq.dqgemm_create(fmt, K, N, dev(st["packed"]), scales_tensor(fmt, st["scales"]), g, bias)
    try:
        plan = dq.dqgemm_get_plan(h, M)
        assert plan["max_cta_stages"] > plan["stages"], f"weight ring does not wrap: {plan}"
        if M <= 32 or M == 1024:
            assert plan["max_cta_stages"] > plan["x_stages"], f"x ring does not wrap: {plan}"
        if fmt == "fp8_static" and M >= 128:
            q = torch.empty((M, K), dtype=torch.uint8, device="cuda")
            y = torch.full((M, N), float("nan"), dtype=torch.bfloat16, device="cuda")
            dq.dqgemm_quantize_act_fp8(x.cuda(), M, K, s_x, q)
            dq.dqgemm_run_fp8_static_quantized(h, q, M, y)
        else:
            y = torch.full((M, N), float("nan"), dtype=torch.bfloat16, device="cuda")
            dq.dqgemm_run(h, x.cuda(), M, y)
        torch.cuda.synchronize()
        assert dq.dqgemm_last_error(h) == 0
        yv = bf16_values(y)
        sel = np.arange(M) if rows is None else np.sort(np.random.default_rng(M).choice(M, rows, replace=False))
        x_eff = static_effective_x(xv[sel], s_x) if fmt == "fp8_static" else xv[sel]
        ref = L.linear_ref(x_eff, wdq, None if fmt == "fp8_static" else bf16_values(b))
        check_close(yv[sel], ref, x_eff, wdq)
    finally:
        dq.dqgemm_destroy(h)


@pytest.mark.parametrize("fmt", ["int4", "nvfp4", "fp8", "fp8_static", "w4a4_mxfp4"])
@pytest.mark.parametrize("M", [1, 32])
def test_skinny_tiles_more_than_sms(fmt, M):
    # 160 output tiles (N = 20480) at 1 and 32 rows: more tiles than SMs, so
    # the skinny tile is kept and CTAs loop over whole tiles (persistent);
    # with 74..148 tiles the plan takes the 128-row tile instead
    from gpu_util import base_fmt, make_layer, w4a4_effective_x

    K, N = 512, 20480
    x, w, b = synthetic.linear_inputs(M, K, N, seed=M + 5)
    xv = bf16_values(x)
    s_x = L.act_scale(xv.min(), xv.max())
    h, st, wdq = make_layer(fmt, w.numpy().astype(np.float64), None if fmt == "fp8_static" else b.cuda(),
                            act_scale=s_x)
    try:
        plan = dq.dqgemm_get_plan(h, M)
        assert plan["bn"] == (32 if fmt.startswith("w4a4") or M == 32 else 16), plan
        assert plan["max_segments"] == 1 and plan["n_tiles"] > plan["grid"], plan
        y = torch.full((M, N), float("nan"), dtype=torch.bfloat16, device="cuda")
        dq.dqgemm_run(h, x.cuda(), M, y)
        torch.cuda.synchronize()
        assert dq.dqgemm_last_error(h) == 0
        bias = None if fmt == "fp8_static" else bf16_values(b)
        if fmt.startswith("w4a4"):
            x_eff = w4a4_effective_x(fmt, xv)
            ref = L.w4a4_linear_ref(base_fmt(fmt), xv, st["packed"], st["scales"], st["global_scale"], bias)
        else:
            x_eff = static_effective_x(xv, s_x) if fmt == "fp8_static" else xv
            ref = L.linear_ref(x_eff, wdq, bias)
        check_close(bf16_values(y), ref, x_eff, wdq)
    finally:
        dq.dqgemm_destroy(h)


@pytest.mark.parametrize("fmt", ["int4", "fp8"])
def test_skinny_rows_take_the_128_row_tile_when_tiles_fill_the_gpu(fmt):
    # 112 output tiles (N = 14336): the K range cannot be split, so one CTA
    # per SM streams a whole tile, on the 128-row tile
    from gpu_util import make_layer

    K, N, M = 512, 14336, 24
    x, w, b = synthetic.linear_inputs(M, K, N, seed=9)
    h, st, wdq = make_layer(fmt, w.numpy().astype(np.float64), b.cuda())
    try:
        plan = dq.dqgemm_get_plan(h, M)
        assert plan["bn"] == 128 and plan["max_segments"] == 1 and plan["grid"] == 112, plan
        y = torch.full((M, N), float("nan"), dtype=torch.bfloat16, device="cuda")
        dq.dqgemm_run(h, x.cuda(), M, y)
        torch.cuda.synchronize()
        assert dq.dqgemm_last_error(h) == 0
        xv = bf16_values(x)
        check_close(bf16_values(y), L.linear_ref(xv, wdq, bf16_values(b)), xv, wdq)
    finally:
        dq.dqgemm_destroy(h)
