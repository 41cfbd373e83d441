"""FP4 x FP4 (W4A4) through the C ABI against the fp64 oracle.

"TorchAO MXFP4 Dynamic Activation + MX Weight (Linear)", intro: the config
quantizes the activations dynamically to MX as well as the weights, and the
native MXFP4 x MXFP4 kernel needs B200.  The library runs it as the tensor
core's block-scaled FP4 MMA (kind::mxf4 / kind::mxf4nvf4) with both
operands' block scales in tensor memory; the NVFP4 variant takes the NVFP4
page's storage for the weight and quantizes x with the same recipe under a
per-call global scale.

Checked here:
  - the activation quantizer, bit for bit against quantize_act_mxfp4 /
    quantize_act_nvfp4 (codes, block scales, g_x);
  - the GEMM against w4a4_linear_ref on shapes that take every x-tile height
    (32, 64, 128, 256 rows), split-K depths 1 to 8, a partial last k-stage,
    ragged M and N tails, with and without bias;
  - one handle serving several M in a row (its activation workspace grows);
  - what the format refuses."""

import numpy as np
import pytest
import torch

import weight_only_quantized_prologue_b200 as dq
from oracle import linear as L
from oracle.quant import pack_nibbles
from weight_only_quantized_prologue_b200 import synthetic

from gpu_util import base_fmt, bf16_values, check_close, dev, make_layer, scales_tensor, w4a4_effective_x

pytestmark = pytest.mark.gpu

W4 = ["w4a4_mxfp4", "w4a4_nvfp4"]


def _x(M, K, seed, scale=1.0):
    g = torch.Generator("cpu").manual_seed(seed)
    return (torch.randn((M, K), generator=g) * scale).to(torch.bfloat16)


# -- the dynamic activation quantizer -----------------------------------------


def _quantize(fmt, x):
    M, K = x.shape
    vs = 32 if fmt == "w4a4_mxfp4" else 16
    codes = torch.full((M, K // 2), 0xAB, dtype=torch.uint8, device="cuda")
    scales = torch.full((M, K // vs), 0xCD, dtype=torch.uint8, device="cuda")
    gx = torch.full((1,), -1.0, dtype=torch.float32, device="cuda")
    dq.dqgemm_quantize_act_fp4(fmt, x.cuda(), M, K, codes, scales, gx if vs == 16 else None)
    torch.cuda.synchronize()
    return codes.cpu().numpy(), scales.cpu().numpy(), float(gx.item())


@pytest.mark.parametrize("fmt", W4)
@pytest.mark.parametrize("M,K", [(1, 64), (5, 256), (33, 3072), (300, 576), (7, 96)])
def test_activation_quantizer_bit_exact(fmt, M, K):
    x = _x(M, K, seed=M * 7 + K, scale=3.0)
    x[0, : min(K, 64)] = 0.0                       # an all-zero block (scale code 0)
    if M > 2:
        x[2, 5] = 30000.0                          # a block whose amax dwarfs the rest
        x[2, 6] = -1e-39                           # (a bf16 subnormal in it)
    xv = bf16_values(x)
    c, s, g = _quantize(fmt, x)
    if fmt == "w4a4_mxfp4":
        rc, rs = L.quantize_act_mxfp4(xv)
    else:
        rc, rs, rg = L.quantize_act_nvfp4(xv)
        assert np.float32(g) == np.float32(rg)
    assert np.array_equal(s, rs), f"{(s != rs).sum()} scale codes differ"
    assert np.array_equal(c, pack_nibbles(rc)), f"{(c != pack_nibbles(rc)).sum()} code bytes differ"


@pytest.mark.parametrize("fmt", W4)
@pytest.mark.parametrize("shift", [0, 120, 135])
def test_activation_quantizer_every_bf16_value(fmt, shift):
    # every finite bf16 bit pattern once, each block of 16 / 32 consecutive
    # patterns a block of x (rolled by `shift` so that the blocks mix
    # magnitudes differently); the NVFP4 codes come from a quotient formed
    # without dividing and must match the exact one
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    bits = np.where((bits & 0x7F80) != 0x7F80, bits, 0).astype(np.uint16)
    bits = np.roll(bits, shift * 97)
    x = torch.from_numpy(bits.view(np.int16).reshape(256, 256).copy()).view(torch.bfloat16)
    if fmt == "w4a4_nvfp4":
        x = x.float().clamp(-1e30, 1e30).to(torch.bfloat16)   # keep amax / 2688 an ordinary fp32 scale
    xv = bf16_values(x)
    c, s, g = _quantize(fmt, x)
    if fmt == "w4a4_mxfp4":
        rc, rs = L.quantize_act_mxfp4(xv)
    else:
        rc, rs, rg = L.quantize_act_nvfp4(xv)
        assert np.float32(g) == np.float32(rg)
    assert np.array_equal(s, rs), f"{(s != rs).sum()} scale codes differ"
    assert np.array_equal(c, pack_nibbles(rc)), f"{(c != pack_nibbles(rc)).sum()} code bytes differ"


def test_nvfp4_activation_quantizer_zero_tensor_and_repeat_calls():
    # an all-zero x takes g_x = 1; the amax reduction's ticket is left at zero
    # by every call, so a second, different call is exact too
    z = torch.zeros((4, 128), dtype=torch.bfloat16)
    c, s, g = _quantize("w4a4_nvfp4", z)
    assert g == 1.0 and not c.any() and not s.any()
    for seed in (1, 2):
        x = _x(300, 1024, seed=seed, scale=seed)   # 300 x 1024 spreads the amax over many blocks
        c, s, g = _quantize("w4a4_nvfp4", x)
        rc, rs, rg = L.quantize_act_nvfp4(bf16_values(x))
        assert np.float32(g) == np.float32(rg)
        assert np.array_equal(s, rs) and np.array_equal(c, pack_nibbles(rc))


# -- the GEMM ----------------------------------------------------------------


def _check_gemm(fmt, M, K, N, seed, bias, layer=None):
    """layer: (handle, storage, exact DQ, bias tensor or None) of an existing
    handle, else one is made from the seed's weights."""
    x, w, b = synthetic.linear_inputs(M, K, N, seed=seed)
    own = layer is None
    if own:
        h, st, wdq = make_layer(fmt, w.numpy().astype(np.float64), b.cuda() if bias else None)
    else:
        h, st, wdq, b = layer
        bias = b is not None
    try:
        y = torch.full((M, N), float("nan"), dtype=torch.bfloat16, device="cuda")
        dq.dqgemm_run(h, x.cuda(), M, y)
        torch.cuda.synchronize()
        assert dq.dqgemm_last_error(h) == 0
        xv = bf16_values(x)
        ref = L.w4a4_linear_ref(base_fmt(fmt), xv, st["packed"], st["scales"], st["global_scale"],
                                bf16_values(b) if bias else None)
        check_close(bf16_values(y), ref, w4a4_effective_x(fmt, xv), wdq)
        return dq.dqgemm_get_plan(h, M)
    finally:
        if own:
            dq.dqgemm_destroy(h)


@pytest.mark.parametrize("fmt", W4)
@pytest.mark.parametrize("M,K,N,bias,bn,split", [
    (32, 3072, 4096, True, 32, 4),       # the pages' Linear: 32 tiles, split-K over 4
    (1, 512, 256, True, 32, 2),          # one row
    (17, 768, 384, False, 32, 2),        # ragged M
    (3, 2048, 128, True, 32, 8),         # one tile, split-K over 8 (8 stages)
    (64, 1024, 512, True, 64, 4),
    (100, 512, 640, False, 128, 2),      # ragged M on a 128-row tile
    (300, 1024, 1024, True, 128, 4),     # three m-tiles
    (1024, 512, 2560, True, 256, 1),     # 256-row tiles, whole tiles over the SMs
    (768, 256, 6400, False, 128, 1),     # 300 128-row tiles: two or three per CTA
    (2048, 1024, 4736, True, 256, 1),    # 296 256-row tiles of 4 stages (more than the x slots), two per
                                         # CTA: a CTA prepares its next tile's first stages while its
                                         # rings still hold this tile's
])
def test_gemm_matches_oracle(fmt, M, K, N, bias, bn, split):
    plan = _check_gemm(fmt, M, K, N, seed=M + K + N, bias=bias)
    assert (plan["bn"], plan["max_segments"]) == (bn, split), plan
    assert plan["workspace_bytes"] > 0


@pytest.mark.parametrize("fmt,K", [("w4a4_mxfp4", 320), ("w4a4_nvfp4", 336), ("w4a4_nvfp4", 16)])
def test_gemm_partial_last_stage(fmt, K):
    # K not a multiple of the 256-k stage: the weight's and x's padding are
    # zero codes (the NVFP4 case K = 16 is a single block)
    _check_gemm(fmt, 33, K, 256, seed=K, bias=True)


@pytest.mark.parametrize("fmt", W4)
def test_one_handle_many_m(fmt):
    # the handle's activation workspace grows with M and is reused after
    K, N = 1024, 512
    _, w, b = synthetic.linear_inputs(1, K, N, seed=77)
    h, st, wdq = make_layer(fmt, w.numpy().astype(np.float64), b.cuda())
    try:
        for M in (1, 300, 32, 1024, 5):
            _check_gemm(fmt, M, K, N, seed=77 + M, bias=True, layer=(h, st, wdq, b))
    finally:
        dq.dqgemm_destroy(h)


@pytest.mark.parametrize("fmt", W4)
def test_layer_wrapper(fmt):
    _, w, b = synthetic.linear_inputs(1, 768, 256, seed=9)
    lin = dq.QuantizedLinear.from_float(fmt, w.cuda(), b.cuda())
    try:
        x = synthetic.activations(20, 768, seed=10)
        y = lin(x.cuda())
        torch.cuda.synchronize()
        st = L.quantize_pack(base_fmt(fmt), w.numpy().astype(np.float64))
        ref = L.w4a4_linear_ref(base_fmt(fmt), bf16_values(x), st["packed"], st["scales"], st["global_scale"],
                                bf16_values(b))
        wdq = L.dequant_exact(base_fmt(fmt), st["packed"], st["scales"], st["global_scale"])
        check_close(bf16_values(y), ref, w4a4_effective_x(fmt, bf16_values(x)), wdq)
    finally:
        lin.close()


def test_w4a4_refusals():
    lib = dq._native.lib()
    N, K = 64, 128
    packed = pack_nibbles(np.zeros((N, K), np.uint8))
    se = np.full((N, K // 32), 127, np.uint8)
    se[3, 1] = 255                                  # NaN exponent
    h = dq._native.ctypes.c_void_p()
    assert lib.dqgemm_create(dq._native.ctypes.byref(h), dq.FORMATS["w4a4_mxfp4"], K, N, dev(packed).data_ptr(),
                             scales_tensor("w4a4_mxfp4", se).data_ptr(), 1.0, None) == dq._native.DQ_ERR_INVALID_ARG
    sb = np.full((N, K // 16), 0x38, np.uint8)
    assert lib.dqgemm_create(dq._native.ctypes.byref(h), dq.FORMATS["w4a4_nvfp4"], K, N, dev(packed).data_ptr(),
                             dev(sb).data_ptr(), 0.0, None) == dq._native.DQ_ERR_INVALID_ARG   # g_w must be > 0
    assert lib.dqgemm_create(dq._native.ctypes.byref(h), dq.FORMATS["w4a4_mxfp4"], 48, N, dev(packed).data_ptr(),
                             dev(se).data_ptr(), 1.0, None) == dq._native.DQ_ERR_INVALID_ARG   # K % 32
    se[3, 1] = 254                                  # the largest exponent is fine (no span limit)
    se[4, 0] = 0
    h = dq.dqgemm_create("w4a4_mxfp4", K, N, dev(packed), scales_tensor("w4a4_mxfp4", se), 1.0, None)
    try:
        x = torch.zeros((4, K), dtype=torch.bfloat16, device="cuda")
        y = torch.zeros((4, N), dtype=torch.bfloat16, device="cuda")
        q = torch.zeros((4, N), dtype=torch.uint8, device="cuda")
        w = torch.zeros((N, K), dtype=torch.bfloat16, device="cuda")
        assert lib.dqgemm_dequantize(h, w.data_ptr(), None) == dq._native.DQ_ERR_UNSUPPORTED
        assert lib.dqgemm_run_quantized_out(h, x.data_ptr(), 4, q.data_ptr(), 1.0, None) == \
            dq._native.DQ_ERR_UNSUPPORTED
        assert lib.dqgemm_run_fp8_static_quantized(h, x.data_ptr(), 4, y.data_ptr(), None) == \
            dq._native.DQ_ERR_UNSUPPORTED
        assert lib.dqgemm_run(h, x.data_ptr() + 2, 4, y.data_ptr(), None) == dq._native.DQ_ERR_ALIGNMENT
        assert lib.dqgemm_run(h, x.data_ptr(), 4, y.data_ptr(), None) == dq._native.DQ_OK
        torch.cuda.synchronize()
        assert dq.dqgemm_last_error(h) == 0
        assert not y.float().any()
    finally:
        dq.dqgemm_destroy(h)
    c = torch.zeros((4, 64), dtype=torch.uint8, device="cuda")
    s = torch.zeros((4, 8), dtype=torch.uint8, device="cuda")
    x = torch.zeros((4, 128), dtype=torch.bfloat16, device="cuda")
    assert lib.dqgemm_quantize_act_fp4(dq.FORMATS["int4"], x.data_ptr(), 4, 128, c.data_ptr(), s.data_ptr(),
                                       None, None) == dq._native.DQ_ERR_UNSUPPORTED
    assert lib.dqgemm_quantize_act_fp4(dq.FORMATS["w4a4_nvfp4"], x.data_ptr(), 4, 128, c.data_ptr(),
                                       s.data_ptr(), None, None) == dq._native.DQ_ERR_INVALID_ARG   # g_x missing
