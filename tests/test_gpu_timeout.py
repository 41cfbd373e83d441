"""The GEMM's own bounded-wait path, run on the GPU without a fault.

A handle's pipeline waits get a limit so short that the first wait which
does not complete at once gives up (dqgemm_set_wait_limit, a test and
diagnostic knob; the shared default is not touched).  Every CTA then takes
its abort path: it drains its own copies and tensor-core operations, still
sends its (invalid) split-K partials so that every receive of the cluster
completes, and writes no output.  The call must report DQ_ERR_TIMEOUT,
leave y untouched, and leave the context usable: the same handle with the
default limit restored, and the next call, give the oracle's result."""

import numpy as np
import pytest
import torch

import weight_only_quantized_prologue_b200 as dq
from oracle import linear as L
from weight_only_quantized_prologue_b200 import synthetic

from gpu_util import base_fmt, bf16_values, check_close, make_layer, static_effective_x, w4a4_effective_x

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("fmt", ["int4", "nvfp4", "fp8", "fp8_static", "w4a4_mxfp4", "w4a4_nvfp4"])
@pytest.mark.parametrize("M,K,N", [(32, 3072, 4096), (1, 1024, 512), (256, 256, 19200)])
def test_gemm_wait_limit_expires_then_context_recovers(fmt, M, K, N):
    x, w, b = synthetic.linear_inputs(M, K, N, seed=31)
    W = w.numpy().astype(np.float64)
    xv = bf16_values(x)
    s_x = L.act_scale(xv.min(), xv.max())
    h, st, wdq = make_layer(fmt, W, b.cuda(), act_scale=s_x)
    try:
        plan = dq.dqgemm_get_plan(h, M)
        xc = x.cuda()
        y = torch.full((M, N), float("nan"), dtype=torch.bfloat16, device="cuda")
        dq.dqgemm_set_wait_limit(h, 1)
        dq.dqgemm_run(h, xc, M, y)
        torch.cuda.synchronize()
        assert dq.dqgemm_last_error(h) == dq._native.DQ_ERR_TIMEOUT, plan
        assert torch.isnan(y.float()).all(), "an aborted call wrote output"
        dq.dqgemm_set_wait_limit(h, 0)          # back to the default
        dq.dqgemm_run(h, xc, M, y)
        torch.cuda.synchronize()
        assert dq.dqgemm_last_error(h) == 0
        if fmt.startswith("w4a4"):
            ref = L.w4a4_linear_ref(base_fmt(fmt), xv, st["packed"], st["scales"], st["global_scale"],
                                    bf16_values(b))
            check_close(bf16_values(y), ref, w4a4_effective_x(fmt, xv), wdq)
        else:
            x_eff = static_effective_x(xv, s_x) if fmt == "fp8_static" else xv
            check_close(bf16_values(y), L.linear_ref(x_eff, wdq, bf16_values(b)), x_eff, wdq)
    finally:
        dq.dqgemm_destroy(h)


def test_wait_limit_rejects_bad_arguments():
    x, w, b = synthetic.linear_inputs(1, 256, 128, seed=3)
    h, _, _ = make_layer("int4", w.numpy().astype(np.float64))
    try:
        lib = dq._native.lib()
        assert lib.dqgemm_set_wait_limit(h, -1) == dq._native.DQ_ERR_INVALID_ARG
        assert lib.dqgemm_set_wait_limit(None, 5) == dq._native.DQ_ERR_INVALID_ARG
        assert lib.dqgemm_set_wait_limit(h, 0) == dq._native.DQ_OK
    finally:
        dq.dqgemm_destroy(h)


def test_one_launch_mlp_wait_limit_expires_then_context_recovers():
    # the two-layer static MLP in one launch takes its wait limit from layer 1
    w1, w2 = synthetic.mlp_weights(seed=8)
    l1 = dq.QuantizedLinear.from_float("fp8_static", w1.float().cuda(), None, act_scale=0.009)
    l2 = dq.QuantizedLinear.from_float("fp8_static", w2.float().cuda(), None, act_scale=0.004)
    try:
        x = synthetic.activations(32, 256, seed=9).cuda()
        y = torch.full((32, 128), float("nan"), dtype=torch.bfloat16, device="cuda")
        dq.dqgemm_set_wait_limit(l1.handle, 1)
        dq.static_mlp(l1, l2, x, out=y)
        torch.cuda.synchronize()
        assert l1.last_error() == dq._native.DQ_ERR_TIMEOUT
        assert torch.isnan(y.float()).all(), "an aborted call wrote output"
        dq.dqgemm_set_wait_limit(l1.handle, 0)
        y2 = dq.static_mlp(l1, l2, x)
        y3 = l2(l1(x))
        torch.cuda.synchronize()
        assert l1.last_error() == 0 and l2.last_error() == 0
        err = (y2.float() - y3.float()).norm() / y3.float().norm()
        assert err < 2e-2, err          # the same model computed by two launches
    finally:
        l1.close()
        l2.close()
