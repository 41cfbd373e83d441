"""Pins of the FP4 x FP4 (W4A4) oracle: dynamic MX / NVFP4 activation
quantization and the W4A4 reference.  None of them restates its formula:
on-grid activations must reduce it to the (already pinned) weight-only
reference, a tiny case is summed by brute force from the printed E2M1 value
table, and exact symmetries (power-of-two scaling, sign, a zeroed block)
catch a dropped scale, a wrong exponent or a mis-indexed block."""

import json
import os

import numpy as np
import pytest

from oracle import formats as F
from oracle import linear as L
from oracle import quant as Q

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "format_values.json")
FP4 = ("mxfp4", "nvfp4")


def _store(fmt, rng, N, K):
    return L.quantize_pack(fmt, rng.uniform(-1 / np.sqrt(K), 1 / np.sqrt(K), (N, K)))


def _x(rng, M, K):
    return F.bf16(rng.standard_normal((M, K)))


@pytest.mark.parametrize("fmt", FP4)
def test_on_grid_activations_reduce_to_weight_only(fmt):
    rng = np.random.default_rng(1)
    M, K, N = 8, 256, 64
    # activations already on the format's grid: their own dequantization
    xs = L.quantize_pack(fmt, rng.standard_normal((M, K)))
    x = L.dequant_exact(fmt, xs["packed"], xs["scales"], xs["global_scale"])
    st = _store(fmt, rng, N, K)
    b = F.bf16(rng.uniform(-0.05, 0.05, N))
    y = L.w4a4_linear_ref(fmt, x, st["packed"], st["scales"], st["global_scale"], b)
    y_wo = L.linear_ref(x, L.dequant_exact(fmt, st["packed"], st["scales"], st["global_scale"]), b)
    assert np.array_equal(y, y_wo)


def test_brute_force_tiny_mxfp4():
    # every term decoded from the printed E2M1 magnitudes and E8M0 = 2^(c-127)
    mag = json.load(open(GOLDEN))["e2m1"]["magnitude_by_code"]

    def val(code, scode):
        v = mag[int(code) & 7] * 2.0 ** (int(scode) - 127)
        return -v if int(code) & 8 else v

    rng = np.random.default_rng(2)
    M, K, N = 2, 64, 3
    x = _x(rng, M, K)
    st = _store("mxfp4", rng, N, K)
    b = F.bf16(rng.uniform(-0.05, 0.05, N))
    cx, sx = L.quantize_act_mxfp4(x)
    cw = Q.unpack_nibbles(st["packed"])
    y = L.w4a4_linear_ref("mxfp4", x, st["packed"], st["scales"], 1.0, b)
    for m in range(M):
        for n in range(N):
            acc = b[n]
            for k in range(K):
                acc += val(cx[m, k], sx[m, k // 32]) * val(cw[n, k], st["scales"][n, k // 32])
            assert y[m, n] == pytest.approx(acc, rel=1e-14, abs=1e-14)


@pytest.mark.parametrize("fmt", FP4)
@pytest.mark.parametrize("j", [-3, 5])
def test_power_of_two_scaling_is_exact(fmt, j):
    # scaling x by 2^j moves every block exponent (MX) or the global scale
    # (NVFP4) by j and leaves every code alone: y - b scales exactly
    rng = np.random.default_rng(3)
    x = _x(rng, 6, 128)
    st = _store(fmt, rng, 32, 128)
    y0 = L.w4a4_linear_ref(fmt, x, st["packed"], st["scales"], st["global_scale"])
    y1 = L.w4a4_linear_ref(fmt, x * 2.0 ** j, st["packed"], st["scales"], st["global_scale"])
    assert np.array_equal(y1, y0 * 2.0 ** j)


@pytest.mark.parametrize("fmt", FP4)
def test_sign_symmetry(fmt):
    rng = np.random.default_rng(4)
    x = _x(rng, 5, 128)
    st = _store(fmt, rng, 16, 128)
    y0 = L.w4a4_linear_ref(fmt, x, st["packed"], st["scales"], st["global_scale"])
    y1 = L.w4a4_linear_ref(fmt, -x, st["packed"], st["scales"], st["global_scale"])
    assert np.array_equal(y1, -y0)


def test_zero_block_drops_out_mxfp4():
    # a zeroed activation block contributes nothing, and the other blocks'
    # scales do not move: y equals the problem with those 32 columns removed
    rng = np.random.default_rng(5)
    M, K, N = 4, 128, 16
    x = _x(rng, M, K)
    x[:, 32:64] = 0.0
    w = rng.uniform(-0.1, 0.1, (N, K))
    st = L.quantize_pack("mxfp4", w)
    keep = np.r_[0:32, 64:128]
    st2 = L.quantize_pack("mxfp4", w[:, keep])
    y = L.w4a4_linear_ref("mxfp4", x, st["packed"], st["scales"])
    y2 = L.w4a4_linear_ref("mxfp4", x[:, keep], st2["packed"], st2["scales"])
    assert np.array_equal(y, y2)
    cx, sx = L.quantize_act_mxfp4(x)
    assert (sx[:, 1] == 0).all() and (cx[:, 32:64] == 0).all()


def test_mx_activation_error_bound():
    # with 2^e <= amax/4 (amax / 2^e in [4, 8)): elements up to 6 * 2^e round
    # to within half a grid step, at most 2^e; larger ones saturate to 6 * 2^e
    rng = np.random.default_rng(6)
    x = _x(rng, 16, 512)
    cx, sx = L.quantize_act_mxfp4(x)
    xd = F.e2m1_decode(cx) * np.repeat(F.e8m0_decode(sx), 32, axis=1)
    scale = np.repeat(2.0 ** (sx.astype(np.float64) - 127), 32, axis=1)
    amax = np.repeat(np.abs(x).reshape(16, -1, 32).max(axis=2), 32, axis=1)
    assert (amax / scale >= 4).all() and (amax / scale < 8).all()
    err = np.abs(xd - x)
    small = np.abs(x) <= 6 * scale
    assert (err[small] <= scale[small]).all()
    assert (xd[~small] == np.sign(x[~small]) * 6 * scale[~small]).all()


def test_nv_activation_tensor_max_block():
    # the NVFP4 activation recipe puts the tensor's largest element at +-6
    # with block scale 448 (g_x = amax / 2688)
    rng = np.random.default_rng(7)
    x = _x(rng, 8, 256)
    cx, sbx, gx = L.quantize_act_nvfp4(x)
    m, k = np.unravel_index(np.argmax(np.abs(x)), x.shape)
    assert F.e4m3_decode(sbx[m, k // 16]) == 448.0
    assert F.e2m1_decode(cx[m, k]) == np.sign(x[m, k]) * 6.0
    assert gx == float(F.f32(np.abs(x).max() / 2688.0))


@pytest.mark.parametrize("fmt", FP4)
def test_w4a4_close_to_weight_only(fmt):
    # diagnostic bound: quantizing the activations too costs accuracy, but the
    # result stays within a few per cent of the weight-only one on N(0, 1) x
    rng = np.random.default_rng(8)
    x = _x(rng, 32, 512)
    st = _store(fmt, rng, 128, 512)
    y = L.w4a4_linear_ref(fmt, x, st["packed"], st["scales"], st["global_scale"])
    y_wo = L.linear_ref(x, L.dequant_exact(fmt, st["packed"], st["scales"], st["global_scale"]))
    assert 10.0 < L.sqnr(y_wo, y) < 30.0


def test_unknown_format():
    with pytest.raises(ValueError):
        L.w4a4_linear_ref("int4", np.zeros((1, 128)), np.zeros((1, 64), np.uint8), np.zeros((1, 1), np.uint16))
