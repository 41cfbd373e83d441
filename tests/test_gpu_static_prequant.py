"""Static FP8 on activations quantized beforehand: the static page's "Graph
after export" with the Q node as its own step (dqgemm_quantize_act_fp8) and
the FP8 GEMM (dqgemm_run_fp8_static_quantized) after it.  The e4m3 codes are
the same whichever path makes them, so the result must be bit-identical to
the fused dqgemm_run, and within the parity tolerance of the oracle."""

import numpy as np
import pytest
import torch

import weight_only_quantized_prologue_b200 as dq
from oracle import linear as L
from weight_only_quantized_prologue_b200 import synthetic

from gpu_util import bf16_values, check_close, make_layer, run, static_effective_x

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("M,K,N", [(5, 256, 128), (64, 272, 200), (130, 512, 384), (256, 640, 256),
                                   (300, 1024, 4096)])
def test_prequantized_equals_fused_and_oracle(M, K, N):
    x, W, _ = synthetic.linear_inputs(M, K, N, seed=M + N)
    W = W.numpy().astype(np.float64)
    xv = bf16_values(x)
    s_x = L.act_scale(xv.min(), xv.max())
    h, st, wdq = make_layer("fp8_static", W, None, act_scale=s_x)
    try:
        xc = x.cuda()
        y_fused = run(h, xc, N)
        q = torch.empty((M, K), dtype=torch.uint8, device="cuda")
        dq.dqgemm_quantize_act_fp8(xc, M, K, s_x, q)
        y_pre = torch.full((M, N), float("nan"), dtype=torch.bfloat16, device="cuda")
        dq.dqgemm_run_fp8_static_quantized(h, q, M, y_pre)
        torch.cuda.synchronize()
        assert dq.dqgemm_last_error(h) == 0
        assert torch.equal(y_pre.view(torch.int16), y_fused.view(torch.int16))
        x_eff = static_effective_x(xv, s_x)
        check_close(bf16_values(y_pre), L.linear_ref(x_eff, wdq), x_eff, wdq)
    finally:
        dq.dqgemm_destroy(h)


def test_quantized_linear_switches_to_prequantized_path_without_changing_results():
    M, K, N = 192, 512, 256
    x, W, _ = synthetic.linear_inputs(M, K, N, seed=3)
    xc = x.cuda()
    s_x = L.act_scale(bf16_values(x).min(), bf16_values(x).max())
    lin = dq.QuantizedLinear.from_float("fp8_static", W.cuda(), None, act_scale=s_x)
    try:
        assert M >= lin.STATIC_PREQUANT_M
        y = lin(xc)                       # quantize once, then the FP8 GEMM
        y_fused = run(lin.handle, xc, N)  # the fused kernel on the same layer
        assert torch.equal(y.view(torch.int16), y_fused.view(torch.int16))
    finally:
        lin.close()


def test_prequantized_entry_rejects_other_formats():
    M, K, N = 8, 256, 128
    x, W, _ = synthetic.linear_inputs(M, K, N, seed=1)
    h, _, _ = make_layer("int4", W.numpy().astype(np.float64))
    try:
        q = torch.zeros((M, K), dtype=torch.uint8, device="cuda")
        y = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
        with pytest.raises(dq.DQError) as e:
            dq.dqgemm_run_fp8_static_quantized(h, q, M, y)
        assert e.value.status == dq._native.DQ_ERR_UNSUPPORTED
    finally:
        dq.dqgemm_destroy(h)


def _midpoint_activations(M, K, s_x, seed):
    """x = s_x * (values on and next to the e4m3 rounding midpoints), so that
    x / s_x falls on a tie or a few fp32 units from one: the cases in which
    a quantizer that does not divide exactly would pick the other code."""
    rng = np.random.default_rng(seed)
    mags = []
    for e in range(-9, 9):                       # normal and subnormal e4m3 steps
        step = 2.0 ** max(e - 3, -9)
        for k in range(8):
            mags.append((2.0 ** e if e >= -6 else 0.0) + (k + 0.5) * step)
    mags = np.array([m for m in mags if m < 448.0])
    vals = rng.choice(mags, size=(M, K)) * rng.choice([-1.0, 1.0], size=(M, K))
    x = torch.from_numpy((vals * s_x).astype(np.float32)).to(torch.bfloat16)
    # one bf16 unit up or down on a third of the entries
    bits = x.view(torch.int16)
    nudge = torch.from_numpy(rng.integers(-1, 2, size=(M, K)).astype(np.int16))
    return (bits + nudge).view(torch.bfloat16)


@pytest.mark.parametrize("s_x", [3.0, 5.0, 0.0123, 1.0e-3])
def test_quantizer_codes_exact_next_to_e4m3_midpoints(s_x):
    # every quantizer path: the standalone kernels (vector and element-wise)
    # and the fused per-tile quantization of the GEMM, read back through an
    # identity weight (y[m, n] = s_x * dec(q[m, n]) * 448 * f32(1/448),
    # so a different code moves y by a whole e4m3 step)
    s_x = float(np.float32(s_x))
    K = N = 256
    W = np.eye(N, K)
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    bits = np.where((bits & 0x7F80) != 0x7F80, bits, 0).astype(np.uint16)
    every = torch.from_numpy(bits.view(np.int16).reshape(256, 256).copy()).view(torch.bfloat16)
    for M in (16, 32, 64, 100, 256):            # 16-, 32-, 64- and 128-row fused tiles
        # (M = 256: every finite bf16 value once, through 128-row tiles)
        x = every if M == 256 else _midpoint_activations(M, K, s_x, seed=M)
        xv = bf16_values(x)
        ref_codes = L.quantize_act_fp8(xv, s_x)
        q = torch.empty((M, K), dtype=torch.uint8, device="cuda")
        dq.dqgemm_quantize_act_fp8(x.cuda(), M, K, s_x, q)
        qe = torch.full((M * K + 1,), 0, dtype=torch.uint8, device="cuda")
        xe = torch.zeros(M * K + 1, dtype=torch.bfloat16, device="cuda")
        xe[1:] = x.view(-1).cuda()
        lib = dq._native.lib()
        assert lib.dqgemm_quantize_act_fp8(xe.data_ptr() + 2, M, K, s_x, qe.data_ptr() + 1, None) == 0
        torch.cuda.synchronize()
        assert np.array_equal(q.cpu().numpy(), ref_codes)
        assert np.array_equal(qe.cpu().numpy()[1:].reshape(M, K), ref_codes)
        h, st, wdq = make_layer("fp8_static", W, None, act_scale=s_x)
        try:
            y = bf16_values(run(h, x.cuda(), N))
            ref = L.static_linear(ref_codes, s_x, st["packed"], st["scales"])
            tol = np.abs(ref) * 2.0 ** -8 + 1e-30
            ref = np.where(np.isinf(y) & np.isinf(ref) & (np.sign(y) == np.sign(ref)), y, ref)
            bad = np.abs(y - ref) > tol
            assert not bad.any(), f"M={M}: {bad.sum()} outputs off by more than bf16 rounding"
        finally:
            dq.dqgemm_destroy(h)


def test_quantized_linear_prequantizes_earlier_when_tiles_fill_the_gpu():
    # N = 14336 (112 output tiles): from 16 rows the layer quantizes x once
    # and runs the FP8 GEMM on codes, planned on the 128-row tile; same
    # result as the fused kernel, and the oracle's
    M, K, N = 24, 512, 14336
    x, W, _ = synthetic.linear_inputs(M, K, N, seed=8)
    xc = x.cuda()
    xv = bf16_values(x)
    s_x = L.act_scale(xv.min(), xv.max())
    lin = dq.QuantizedLinear.from_float("fp8_static", W.cuda(), None, act_scale=s_x)
    try:
        assert lin._static_prequant_m == lin.STATIC_PREQUANT_M_WIDE <= M < lin.STATIC_PREQUANT_M
        y = lin(xc)
        y_fused = run(lin.handle, xc, N)
        assert torch.equal(y.view(torch.int16), y_fused.view(torch.int16))
        st = L.quantize_pack("fp8", W.numpy().astype(np.float64))
        wdq = L.dequant_exact("fp8", st["packed"], st["scales"])
        x_eff = static_effective_x(xv, s_x)
        check_close(bf16_values(y), L.linear_ref(x_eff, wdq), x_eff, wdq)
    finally:
        lin.close()
