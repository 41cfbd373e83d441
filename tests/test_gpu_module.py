"""nn.Linear drop-in: quantize_ on a bf16 model gives exactly what the
library's layers give on the same inputs (bit-identical), any leading dims."""

import pytest
import torch

import weight_only_quantized_prologue_b200 as dq
from weight_only_quantized_prologue_b200 import module as M
from weight_only_quantized_prologue_b200 import synthetic

pytestmark = pytest.mark.gpu


def _model(seed):
    torch.manual_seed(seed)
    m = torch.nn.Sequential(torch.nn.Linear(256, 512), torch.nn.ReLU(), torch.nn.Linear(512, 128))
    return m.to(device="cuda", dtype=torch.bfloat16)


@pytest.mark.parametrize("fmt", ["int4", "nvfp4", "mxfp4", "fp8"])
def test_quantize_matches_library_layers(fmt):
    model = _model(1)
    w1, b1 = model[0].weight.float(), model[0].bias
    w2, b2 = model[2].weight.float(), model[2].bias
    l1 = dq.QuantizedLinear.from_float(fmt, w1, b1)
    l2 = dq.QuantizedLinear.from_float(fmt, w2, b2)
    M.quantize_(model, fmt)
    assert isinstance(model[0], M.DQLinear) and isinstance(model[2], M.DQLinear)
    x = synthetic.activations(2 * 24, 256, seed=5).cuda().view(2, 24, 256)   # leading dims
    with torch.no_grad():
        y = model(x)
    ref = l2(torch.relu(l1(x.view(-1, 256)))).view(2, 24, 128)
    torch.cuda.synchronize()
    assert y.shape == (2, 24, 128)
    assert torch.equal(y.view(torch.int16), ref.view(torch.int16))
    l1.close()
    l2.close()


def test_static_fp8_calibrate_then_quantize():
    model = _model(2)
    batches = [synthetic.activations(32, 256, seed=s).cuda() for s in range(1, 11)]
    scales = M.calibrate_static_fp8(model, batches)
    w1, w2 = model[0].weight.float(), model[2].weight.float()
    l1 = dq.QuantizedLinear.from_float("fp8_static", w1, model[0].bias, act_scale=scales["0"])
    l2 = dq.QuantizedLinear.from_float("fp8_static", w2, model[2].bias, act_scale=scales["2"])
    M.quantize_(model, "fp8_static", act_scales=scales)
    x = synthetic.activations(160, 256, seed=11).cuda()      # >= 128 rows: quantize-once path
    with torch.no_grad():
        y = model(x)
    ref = l2(torch.relu(l1(x)))
    torch.cuda.synchronize()
    assert torch.equal(y.view(torch.int16), ref.view(torch.int16))
    l1.close()
    l2.close()


def test_static_fp8_without_scales_is_refused():
    with pytest.raises(ValueError):
        M.quantize_(_model(3), "fp8_static")


@pytest.mark.gpu
def test_layer_rejects_bad_tensors_before_launch():
    # wrong dtype / shape / layout never reach the kernel; an empty batch
    # launches nothing and returns an empty result
    torch.manual_seed(3)
    w = torch.randn(128, 256, device="cuda") * 0.05
    lin = dq.QuantizedLinear.from_float("int4", w.to(torch.bfloat16))    # bf16 weight: converted
    x = synthetic.activations(8, 256, seed=1).cuda()
    with pytest.raises(TypeError):
        lin(x.float())
    with pytest.raises(ValueError):
        lin(x[:, :128])
    with pytest.raises(ValueError):
        lin(torch.empty(256, 8, dtype=torch.bfloat16, device="cuda").t())
    with pytest.raises(ValueError):
        lin(x, out=torch.empty(8, 64, dtype=torch.bfloat16, device="cuda"))
    with pytest.raises(ValueError):
        dq.QuantizedLinear("int4", 256, 128, torch.zeros(128, 100, dtype=torch.uint8, device="cuda"),
                           torch.zeros(128, 2, dtype=torch.int16, device="cuda"))
    y0 = lin(x[:0])
    assert y0.shape == (0, 128)
    y = lin(x)
    torch.cuda.synchronize()
    assert lin.last_error() == 0 and y.shape == (8, 128)
    lin.close()


@pytest.mark.parametrize("fmt", ["int4", "nvfp4", "mxfp4", "fp8", "int4_asym", "fp8_static", "w4a4_mxfp4",
                                 "w4a4_nvfp4"])
def test_quantized_module_matches_oracle(fmt):
    """The pages' flow end to end against the fp64 oracle: a bf16
    nn.Linear(3072, 512) quantized in place by quantize_, called on x with
    leading dims; the reference quantizes the same weight with the oracle's
    own recipe and multiplies in fp64 ("Define a linear model and quantize
    weights to ..." on each weight-only page; static FP8 with its calibrated
    scale, "Define a small two-layer Linear model")."""
    import numpy as np

    from oracle import linear as L

    from gpu_util import base_fmt, bf16_values, check_close, static_effective_x

    torch.manual_seed(7)
    model = torch.nn.Sequential(torch.nn.Linear(3072, 512)).to(device="cuda", dtype=torch.bfloat16)
    W = model[0].weight.detach().float().cpu().numpy().astype(np.float64)
    b = bf16_values(model[0].bias.detach())
    x = synthetic.activations(2 * 20, 3072, seed=12).cuda().view(2, 20, 3072)
    scales = None
    if fmt == "fp8_static":
        scales = M.calibrate_static_fp8(model, [synthetic.activations(32, 3072, seed=s).cuda() for s in range(1, 4)])
    M.quantize_(model, fmt, act_scales=scales)
    with torch.no_grad():
        y = model(x)
    torch.cuda.synchronize()
    assert model[0].layer.last_error() == 0
    base = base_fmt(fmt)
    st = L.quantize_pack(base, W)
    wdq = L.dequant_exact(base, st["packed"], st["scales"], st["global_scale"])
    xv = bf16_values(x.view(-1, 3072))
    if fmt.startswith("w4a4"):
        # W4A4: the activations are quantized per call with the weight's recipe
        from gpu_util import w4a4_effective_x

        x_eff = w4a4_effective_x(fmt, xv)
        ref = L.w4a4_linear_ref(base, xv, st["packed"], st["scales"], st["global_scale"], b)
    else:
        x_eff = static_effective_x(xv, scales["0"]) if fmt == "fp8_static" else xv
        ref = L.linear_ref(x_eff, wdq, b)
    check_close(bf16_values(y.view(-1, 512)), ref, x_eff, wdq)
