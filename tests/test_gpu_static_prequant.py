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
