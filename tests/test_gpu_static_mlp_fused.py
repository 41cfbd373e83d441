"""The static-FP8 two-layer model in one launch (dqgemm_run_static_mlp)
against the fp64 oracle.

"TorchAO Static FP8 Quantization (Linear)", "Define a small two-layer Linear
model" and "Graph after export": x -> Q -> DQ -> Linear1 -> Q -> DQ ->
Linear2.  Layer 1's bf16 output (read back through h_out) is checked against
the oracle's fp64 layer within the parity tolerance; layer 2 is checked
against the oracle's static layer applied to the oracle's own Q node on that
h (the kernel quantizes the same bf16 values with the same scale), and the
whole model against the oracle's end-to-end two-layer reference by SQNR."""

import numpy as np
import pytest
import torch

import weight_only_quantized_prologue_b200 as dq
from oracle import linear as L
from weight_only_quantized_prologue_b200 import synthetic

from gpu_util import bf16_values, check_close, dev, scales_tensor, static_effective_x

pytestmark = pytest.mark.gpu


def _layer(W, s_x, bias=None):
    st = L.quantize_pack("fp8", W)
    N, K = W.shape
    h = dq.dqgemm_create("fp8_static", K, N, dev(st["packed"]), scales_tensor("fp8_static", st["scales"]), s_x,
                         None if bias is None else bias.cuda())
    return h, st, L.dequant_exact("fp8", st["packed"], st["scales"])


def _check(M, K1, N1, N2, seed, bias):
    g = torch.Generator("cpu").manual_seed(seed)
    w1 = ((torch.rand((N1, K1), generator=g) * 2 - 1) / np.sqrt(K1)).to(torch.bfloat16)
    w2 = ((torch.rand((N2, N1), generator=g) * 2 - 1) / np.sqrt(N1)).to(torch.bfloat16)
    b1 = ((torch.rand(N1, generator=g) * 2 - 1) / np.sqrt(K1)).to(torch.bfloat16) if bias else None
    b2 = ((torch.rand(N2, generator=g) * 2 - 1) / np.sqrt(N1)).to(torch.bfloat16) if bias else None
    w1v, w2v = bf16_values(w1), bf16_values(w2)
    cal = [bf16_values(synthetic.activations(32, K1, seed=s)) for s in range(1, 11)]
    s1, s2 = L.calibrate_static_mlp(cal, w1v, w2v)
    x = synthetic.activations(M, K1, seed=seed + 1)
    h1, st1, wdq1 = _layer(w1v, s1, b1)
    h2, st2, wdq2 = _layer(w2v, s2, b2)
    try:
        hid = torch.full((M, N1), float("nan"), dtype=torch.bfloat16, device="cuda")
        y = torch.full((M, N2), float("nan"), dtype=torch.bfloat16, device="cuda")
        dq.dqgemm_run_static_mlp(h1, h2, x.cuda(), M, hid, y)
        torch.cuda.synchronize()
        assert dq.dqgemm_last_error(h1) == 0
        xv = bf16_values(x)
        x1 = static_effective_x(xv, s1)
        hv = bf16_values(hid)
        check_close(hv, L.linear_ref(x1, wdq1, None if b1 is None else bf16_values(b1)), x1, wdq1)
        x2 = static_effective_x(hv, s2)
        ref2 = L.static_linear(L.quantize_act_fp8(hv, s2), s2, st2["packed"], st2["scales"])
        if b2 is not None:
            ref2 = ref2 + bf16_values(b2)[None, :]
        check_close(bf16_values(y), ref2, x2, wdq2)
        if not bias:
            _, y_ref = L.static_mlp(xv, s1, st1["packed"], st1["scales"], s2, st2["packed"], st2["scales"])
            assert L.sqnr(y_ref, bf16_values(y)) > 30.0
        # the same launch without h_out gives the same y, bit for bit
        y2 = torch.empty_like(y)
        dq.dqgemm_run_static_mlp(h1, h2, x.cuda(), M, None, y2)
        torch.cuda.synchronize()
        assert torch.equal(y2.view(torch.int16), y.view(torch.int16))
    finally:
        dq.dqgemm_destroy(h1)
        dq.dqgemm_destroy(h2)


def test_pages_two_layer_model_in_one_launch():
    """256 -> 512 -> 128, no bias, x of 32 rows: the page's model."""
    _check(32, 256, 512, 128, seed=0, bias=False)


@pytest.mark.parametrize("M,K1,N1,N2,bias", [(1, 256, 256, 128, True), (5, 384, 1024, 64, True),
                                               (17, 512, 512, 128, False), (50, 256, 1024, 96, True),
                                               (100, 1024, 512, 128, True), (130, 128, 256, 32, False)])
def test_mlp_shapes(M, K1, N1, N2, bias):
    # 16-, 32- and 64-row x tiles, several m-tiles, clusters of 2, 4 and 8
    # CTAs, ragged layer-2 width, biases on both layers
    _check(M, K1, N1, N2, seed=M + N1, bias=bias)


def test_mlp_rejects_what_it_cannot_run():
    rng = np.random.default_rng(1)
    u = lambda n, k: rng.uniform(-0.05, 0.05, (n, k))
    l1, _, _ = _layer(u(256, 256), 0.01)           # 256 hidden units
    l2, _, _ = _layer(u(128, 256), 0.01)           # a valid layer 2
    l1_odd, _, _ = _layer(u(384, 256), 0.01)       # 384 hidden units: 3 CTAs per cluster
    l2_odd, _, _ = _layer(u(128, 384), 0.01)
    l2_wide, _, _ = _layer(u(200, 256), 0.01)      # 200 outputs > 128
    st = L.quantize_pack("int4", u(128, 256))
    l2_int4 = dq.dqgemm_create("int4", 256, 128, dev(st["packed"]), scales_tensor("int4", st["scales"]), 1.0, None)
    handles = (l1, l2, l1_odd, l2_odd, l2_wide, l2_int4)
    try:
        lib = dq._native.lib()
        x = torch.zeros((4, 256), dtype=torch.bfloat16, device="cuda")
        y = torch.zeros((4, 256), dtype=torch.bfloat16, device="cuda")
        call = lambda a, b, m=4: lib.dqgemm_run_static_mlp(a, b, x.data_ptr(), m, None, y.data_ptr(), None)
        assert call(l1, l2_int4) == dq._native.DQ_ERR_UNSUPPORTED      # layer 2 not static FP8
        assert call(l1_odd, l2) == dq._native.DQ_ERR_INVALID_ARG       # 384 hidden vs K = 256 of layer 2
        assert call(l1_odd, l2_odd) == dq._native.DQ_ERR_UNSUPPORTED   # 3 CTAs per cluster
        assert call(l1, l2_wide) == dq._native.DQ_ERR_UNSUPPORTED      # 200 outputs
        assert call(l1, l2, 0) == dq._native.DQ_ERR_INVALID_ARG
        assert lib.dqgemm_run_static_mlp(l1, l2, x.data_ptr() + 2, 4, None, y.data_ptr(), None) == \
            dq._native.DQ_ERR_ALIGNMENT
        assert call(l1, l2) == dq._native.DQ_OK
        torch.cuda.synchronize()
        assert dq.dqgemm_last_error(l1) == 0
    finally:
        for h in handles:
            dq.dqgemm_destroy(h)


def test_static_mlp_layer_wrapper_matches_the_entry_point():
    w1, w2 = synthetic.mlp_weights(seed=5)
    l1 = dq.QuantizedLinear.from_float("fp8_static", w1.float().cuda(), None, act_scale=0.009)
    l2 = dq.QuantizedLinear.from_float("fp8_static", w2.float().cuda(), None, act_scale=0.004)
    try:
        x = synthetic.activations(32, 256, seed=6).cuda()
        y = dq.static_mlp(l1, l2, x)
        y_ref = torch.empty_like(y)
        dq.dqgemm_run_static_mlp(l1.handle, l2.handle, x, 32, None, y_ref)
        torch.cuda.synchronize()
        assert torch.equal(y.view(torch.int16), y_ref.view(torch.int16))
        with pytest.raises(ValueError):
            dq.static_mlp(l2, l1, x)
    finally:
        l1.close()
        l2.close()
