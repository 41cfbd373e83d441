"""Chained static FP8 and the whole-tile (persistent) GEMM path.

dqgemm_run_quantized_out must give exactly the codes dqgemm_quantize_act_fp8
gives for dqgemm_run's bf16 output; a two-layer static MLP chained through
those codes must equal the unchained one bit for bit.  The persistent path
(more 128-channel tiles than SMs, no split-K) is checked against the oracle."""

import numpy as np
import pytest
import torch

import weight_only_quantized_prologue_b200 as dq
from oracle import linear as L
from weight_only_quantized_prologue_b200 import synthetic

from gpu_util import bf16_values, check_close, make_layer, run, static_effective_x

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("fmt", ["int4", "fp8", "fp8_static", "int4_asym"])
@pytest.mark.parametrize("M,N", [(32, 512), (160, 384), (256, 19200)])
def test_quantized_out_equals_run_then_quantize(fmt, M, N):
    K = 256
    x, W, b = synthetic.linear_inputs(M, K, N, seed=M + N)
    s_in = L.act_scale(bf16_values(x).min(), bf16_values(x).max())
    lin = dq.QuantizedLinear.from_float(fmt, W.cuda(), None if fmt == "fp8_static" else b.cuda(), act_scale=s_in)
    try:
        xc = x.cuda()
        y = lin(xc)
        s_out = float(np.float32(max(abs(y.float().min().item()), abs(y.float().max().item())) / 448.0))
        q_ref = torch.empty((M, N), dtype=torch.uint8, device="cuda")
        dq.dqgemm_quantize_act_fp8(y, M, N, s_out, q_ref)
        q = lin.quantized_out(xc, s_out)
        torch.cuda.synchronize()
        assert lin.last_error() == 0
        assert torch.equal(q, q_ref)
        # against the oracle: y within tolerance of the fp64 reference (the GPU
        # packer's storage equals the oracle's byte for byte), and the codes
        # exactly the oracle's Q node applied to that bf16 y
        st = L.quantize_pack("fp8" if fmt == "fp8_static" else fmt, W.numpy().astype(np.float64))
        wdq = L.dequant_exact("fp8" if fmt == "fp8_static" else fmt, st["packed"], st["scales"], st["global_scale"])
        xv = bf16_values(x)
        x_eff = static_effective_x(xv, s_in) if fmt == "fp8_static" else xv
        yv = bf16_values(y)
        check_close(yv, L.linear_ref(x_eff, wdq, None if fmt == "fp8_static" else bf16_values(b)), x_eff, wdq)
        assert np.array_equal(q.cpu().numpy(), L.quantize_act_fp8(yv, s_out))
    finally:
        lin.close()


@pytest.mark.parametrize("M", [32, 160])
def test_two_layer_static_mlp_chained_through_codes(M):
    w1, w2 = synthetic.mlp_weights(seed=4)
    cal = [synthetic.activations(32, 256, seed=s).cuda() for s in range(1, 11)]
    s1 = max(c.abs().max().item() for c in cal) / 448.0
    s2 = max((c @ w1.cuda().t()).abs().max().item() for c in cal) / 448.0
    s1, s2 = float(np.float32(s1)), float(np.float32(s2))
    l1 = dq.QuantizedLinear.from_float("fp8_static", w1.float().cuda(), None, act_scale=s1)
    l2 = dq.QuantizedLinear.from_float("fp8_static", w2.float().cuda(), None, act_scale=s2)
    try:
        x = synthetic.activations(M, 256, seed=9).cuda()
        h = l1(x)
        y_plain = l2(h)
        q = l1.quantized_out(x, s2)
        y_chain = l2.from_codes(q)
        torch.cuda.synchronize()
        assert torch.equal(y_chain.view(torch.int16), y_plain.view(torch.int16))
        # against the oracle: layer 1 within tolerance, the chained codes
        # exactly the oracle's Q node on the GPU's h, and layer 2 on those
        # codes within tolerance
        st1 = L.quantize_pack("fp8", w1.float().numpy().astype(np.float64))
        st2 = L.quantize_pack("fp8", w2.float().numpy().astype(np.float64))
        wdq1 = L.dequant_exact("fp8", st1["packed"], st1["scales"])
        wdq2 = L.dequant_exact("fp8", st2["packed"], st2["scales"])
        xv, hv = bf16_values(x), bf16_values(h)
        x1 = static_effective_x(xv, s1)
        check_close(hv, L.linear_ref(x1, wdq1), x1, wdq1)
        q_ref = L.quantize_act_fp8(hv, s2)
        assert np.array_equal(q.cpu().numpy(), q_ref)
        x2 = static_effective_x(hv, s2)
        check_close(bf16_values(y_chain), L.static_linear(q_ref, s2, st2["packed"], st2["scales"]), x2, wdq2)
    finally:
        l1.close()
        l2.close()


@pytest.mark.parametrize("fmt", ["int4", "nvfp4", "fp8_static", "int4_asym"])
def test_persistent_whole_tile_path_matches_oracle(fmt):
    # more output tiles than SMs with either x tile (2 x 160 tiles of 128
    # rows, or 160 tiles of 256 rows): no split-K, each CTA loops over
    # whole tiles
    M, K, N = 256, 256, 20480
    x, W, b = synthetic.linear_inputs(M, K, N, seed=21)
    W = W.numpy().astype(np.float64)
    xv = bf16_values(x)
    s_x = L.act_scale(xv.min(), xv.max())
    h, st, wdq = make_layer(fmt, W, b.cuda(), act_scale=s_x)
    try:
        plan = dq.dqgemm_get_plan(h, M)
        assert plan["max_segments"] == 1 and plan["m_tiles"] * plan["n_tiles"] > plan["grid"]
        y = bf16_values(run(h, x.cuda(), N))
        x_eff = static_effective_x(xv, s_x) if fmt == "fp8_static" else xv
        check_close(y, L.linear_ref(x_eff, wdq, bf16_values(b)), x_eff, wdq)
    finally:
        dq.dqgemm_destroy(h)
