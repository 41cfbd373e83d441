"""Pins of the oracle's quantizers, packer and dequantizers.

Hand-worked examples below were derived on paper from the recipe
definitions (not by running the oracle); the invariants and the brute-force
checks use torch casts or exhaustive enumeration as the independent side."""

import numpy as np
import pytest
import torch

from oracle import formats as F
from oracle import linear as L
from oracle import quant as Q


def _rng(seed=0):
    return np.random.default_rng(seed)


def _uniform_w(n, k, seed=0):
    b = 1.0 / np.sqrt(k)
    return _rng(seed).uniform(-b, b, (n, k)).astype(np.float32).astype(np.float64)


# -- hand-worked examples ----------------------------------------------------


def test_int4_hand_example_unit_scale():
    # group max 7 -> s = bf16(f32(7/7)) = 1.0 (0x3F80); codes are RNE(W):
    # 3.5 -> 4, 2.5 -> 2, -0.5 -> 0, 1.5 -> 2, 0.25 -> 0, -2.5 -> -2
    w = np.zeros((1, 128))
    w[0, :8] = [7.0, 3.5, 2.5, -0.5, 1.5, -7.0, 0.25, -2.5]
    codes, s = Q.quantize_int4(w)
    assert s.tolist() == [[0x3F80]]
    assert codes[0, :8].tolist() == [7, 4, 2, 0, 2, -7, 0, -2]
    assert not codes[0, 8:].any()


def test_int4_hand_example_divisor_seven():
    # amax 1.0: f32(1/7) = 0x3E124925, its bf16 rounding is 0x3E12 = 0.142578125
    # 1/0.142578125 = 7.01 -> 7; 0.5/.. = 3.51 -> 4; f32(-0.3)/.. = -2.10 -> -2
    w = np.zeros((1, 128))
    w[0, :3] = np.float32([1.0, 0.5, -0.3])
    codes, s = Q.quantize_int4(w)
    assert s.tolist() == [[0x3E12]]
    assert codes[0, :3].tolist() == [7, 4, -2]


def test_int4_zero_group():
    codes, s = Q.quantize_int4(np.zeros((2, 256)))
    assert not codes.any() and not s.any()


def test_nvfp4_hand_example():
    # amax 2688 -> g = 1; block amax 2688 -> sb = e4m3(448) = 0x7E; d = 448.
    # W/d = 6, 3, 1.5, .5, .25(tie->0), -2, 4, 0, ~0, -.22(->-0), 2.5(tie->2),
    #       3.5(tie->4), 5(tie->4), 5.5(->6), .75(tie->1), -6
    w = np.array([[2688, 1344, 672, 224, 112, -896, 1792, 0, 3.0, -100, 1120,
                   1568, 2240, 2464, 336, -2688]], dtype=np.float64)
    codes, sb, g = Q.quantize_nvfp4(w)
    assert g == 1.0
    assert sb.tolist() == [[0x7E]]
    assert codes[0].tolist() == [7, 5, 3, 1, 0, 12, 6, 0, 0, 8, 4, 6, 6, 7, 2, 15]
    assert Q.pack_nibbles(codes)[0].tolist() == [0x57, 0x13, 0xC0, 0x06, 0x80, 0x64, 0x76, 0xF2]


def test_mxfp4_hand_example():
    # block 0: amax 7 = 0.875 * 2**3 -> floor(log2) = 2 -> e = 0 -> code 127
    #   6 -> 7, 5(tie 4|6 -> 4) -> 6, .75(tie .5|1 -> 1) -> 2, .25(tie -> 0) -> 0,
    #   -3.5(tie 3|4 -> 4) -> 14, 2.5(tie -> 2) -> 4, 7(saturates to 6) -> 7, -0.1 -> -0 = 8
    # block 1: amax f32(0.3) = 0.6 * 2**-1 -> floor(log2) = -2 -> e = -4 -> code 123
    #   16*f32(.3) = 4.8 -> 4 (code 6), 16*f32(.1) = 1.6 -> 1.5 (code 3), -3.2 -> -3 (13)
    w = np.zeros((1, 64))
    w[0, :8] = [6.0, 5.0, 0.75, 0.25, -3.5, 2.5, 7.0, -0.1]
    w[0, 32:35] = np.float32([0.3, 0.1, -0.2])
    w = w.astype(np.float32).astype(np.float64)
    codes, se = Q.quantize_mxfp4(w)
    assert se.tolist() == [[127, 123]]
    assert codes[0, :8].tolist() == [7, 6, 2, 0, 14, 4, 7, 8]
    assert codes[0, 32:35].tolist() == [6, 3, 13]
    assert not codes[0, 8:32].any() and not codes[0, 35:].any()


def test_fp8_hand_example():
    # row amax 448 -> s = 1; e4m3 of: 448 -> 0x7E, 17(tie 16|18 -> 16) -> 0x58,
    # -17 -> 0xD8, 1 -> 0x38, 2**-9 -> 0x01, 2**-10(tie 0|2**-9 -> 0) -> 0x00,
    # -1.5*2**-9(tie -> 2*2**-9) -> 0x82, 240 -> 0x77, 232(tie 224|240 -> 224) -> 0x76,
    # .5 -> 0x30
    w = np.zeros((1, 16))
    w[0, :10] = [448, 17, -17, 1.0, 2.0**-9, 2.0**-10, -1.5 * 2.0**-9, 240, 232, 0.5]
    codes, s = Q.quantize_fp8_rows(w)
    assert s.tolist() == [1.0]
    assert codes[0, :10].tolist() == [0x7E, 0x58, 0xD8, 0x38, 0x01, 0x00, 0x82, 0x77, 0x76, 0x30]


def test_act_quant_hand_example():
    # s_x = 2: 896/2 = 448 -> 0x7E, 1000/2 saturates -> 0x7E, 34/2 = 17 -> 16 = 0x58,
    # -17 -> 0xD8, 3/2 = 1.5 -> 0x3C, 2**-11 -> 0x00
    x = np.array([[896.0, 1000.0, 34.0, -34.0, 3.0, 2.0**-10]])
    assert L.quantize_act_fp8(x, 2.0)[0].tolist() == [0x7E, 0x7E, 0x58, 0xD8, 0x3C, 0x00]


def test_pack_nibbles_hand_example():
    assert Q.pack_nibbles(np.array([[1, 2, -1, -8]])).tolist() == [[0x21, 0x8F]]
    assert Q.unpack_nibbles(np.array([[0x21, 0x8F]]), signed=True).tolist() == [[1, 2, -1, -8]]


# -- invariants on realistic weights ------------------------------------------


def test_int4_invariants():
    w = _uniform_w(64, 512)
    codes, s = Q.quantize_int4(w)
    assert codes.min() >= -7 and codes.max() <= 7       # -8 never produced with amax/7
    g = np.abs(codes.reshape(64, 4, 128)).max(axis=2)
    assert (g == 7).all()                                 # every group max maps to +-7
    sv = np.repeat(F.bf16_from_bits(s), 128, axis=1)
    assert (np.abs(w - codes * sv) <= sv / 2 + 1e-12).all()  # round-to-nearest error bound


def test_nvfp4_invariants():
    w = _uniform_w(32, 256, seed=3)
    codes, sb, g = Q.quantize_nvfp4(w)
    amax = np.abs(w).max()
    assert g == F.f32(amax / 2688.0)
    n, j = np.unravel_index(np.argmax(np.abs(w)), w.shape)
    assert sb[n, j // 16] == 0x7E                         # tensor-max block scale is 448
    assert codes[n, j] & 7 == 7                           # and its max element maps to 6
    assert F.e4m3_decode(sb).max() <= 448.0


def test_mxfp4_invariants():
    w = _uniform_w(32, 256, seed=4)
    codes, se = Q.quantize_mxfp4(w)
    ab = np.abs(w.reshape(32, 8, 32)).max(axis=2)
    ratio = ab / F.e8m0_decode(se)
    assert (ratio >= 4).all() and (ratio < 8).all()


def test_fp8_invariants():
    w = _uniform_w(16, 256, seed=5)
    codes, s = Q.quantize_fp8_rows(w)
    rowmax = np.abs(F.e4m3_decode(codes)).max(axis=1)
    assert (rowmax == 448.0).all()


@pytest.mark.parametrize("fmt", ["int4", "nvfp4", "mxfp4", "fp8"])
def test_requantize_dequantized_weights_is_idempotent(fmt):
    """Quantizing DQ(W) again returns the same codes and the same scales."""
    w = _uniform_w(32, 256, seed=7)
    st = L.quantize_pack(fmt, w)
    wd = L.dequant_exact(fmt, st["packed"], st["scales"], st["global_scale"])
    st2 = L.quantize_pack(fmt, wd)
    assert np.array_equal(st["packed"], st2["packed"])
    assert np.array_equal(st["scales"], st2["scales"])
    assert st["global_scale"] == st2["global_scale"]


# -- dequantization: brute force over code x scale code ----------------------


def _torch_e4m3(codes):
    return torch.from_numpy(np.asarray(codes, dtype=np.uint8)).view(torch.float8_e4m3fn).double().numpy()


E2M1_TABLE = [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]


def _e2m1_by_table(codes):
    c = np.asarray(codes)
    return np.where(c & 8, -1.0, 1.0) * np.array(E2M1_TABLE)[c & 7]


def test_nvfp4_dequant_every_code_and_scale():
    # N = 32 rows; each 16-block holds all 16 element codes under one of the
    # 254 finite E4M3 scale codes; g is an arbitrary fp32 value
    sc = np.array([c for c in range(256) if (c & 0x7F) != 0x7F], dtype=np.uint8)
    nblk = len(sc)
    codes = np.tile(np.arange(16), (1, nblk))
    packed = Q.pack_nibbles(codes)
    scales = sc[None, :]
    g = float(np.float32(0.0123))
    exact = L.dequant_exact("nvfp4", packed, scales, g)
    want = _e2m1_by_table(codes) * np.repeat(_torch_e4m3(scales), 16, axis=1) * g
    assert np.array_equal(exact, want)
    bits = L.dequant_bf16_bits("nvfp4", packed, scales, g)
    t = (torch.from_numpy((_e2m1_by_table(codes) * np.repeat(_torch_e4m3(scales), 16, axis=1))
                          .astype(np.float32)) * torch.tensor(g, dtype=torch.float32)).to(torch.bfloat16)
    assert np.array_equal(bits, t.view(torch.int16).numpy().astype(np.uint16))


def test_mxfp4_dequant_every_code_and_scale():
    sc = np.arange(0, 255, dtype=np.uint8)
    codes = np.tile(np.repeat(np.arange(16), 2), (1, len(sc)))
    packed = Q.pack_nibbles(codes)
    exact = L.dequant_exact("mxfp4", packed, sc[None, :])
    e8 = torch.from_numpy(sc).view(torch.float8_e8m0fnu).double().numpy()
    want = _e2m1_by_table(codes) * np.repeat(e8, 32)[None, :]
    assert np.array_equal(exact, want)
    bits = L.dequant_bf16_bits("mxfp4", packed, sc[None, :])
    t = torch.from_numpy(want).to(torch.bfloat16)      # exact products -> one RNE
    assert np.array_equal(bits, t.view(torch.int16).numpy().astype(np.uint16))


def test_int4_dequant_every_code_and_scale():
    rng = _rng(11)
    sbits = np.concatenate([rng.integers(0x0080, 0x7E00, 62), [0x0001, 0x3F80]]).astype(np.uint16)
    codes = np.tile(np.repeat(np.arange(-8, 8), 8), (1, len(sbits)))
    packed = Q.pack_nibbles(codes)
    scales = sbits[None, :]
    sv = torch.from_numpy(sbits.astype(np.int16)).view(torch.bfloat16).double().numpy()
    want = codes * np.repeat(sv, 128)[None, :]
    assert np.array_equal(L.dequant_exact("int4", packed, scales), want)
    t = torch.from_numpy(want.astype(np.float32)).to(torch.bfloat16)   # c*s exact in fp32
    assert np.array_equal(L.dequant_bf16_bits("int4", packed, scales),
                          t.view(torch.int16).numpy().astype(np.uint16))


def test_fp8_dequant_every_code():
    codes = np.array([c for c in range(256) if (c & 0x7F) != 0x7F], dtype=np.uint8)[None, :]
    s = np.array([np.float32(0.0371)], dtype=np.float32)
    want = _torch_e4m3(codes) * float(s[0])
    assert np.array_equal(L.dequant_exact("fp8", codes, s), want)
    t = (torch.from_numpy(_torch_e4m3(codes).astype(np.float32)) * torch.from_numpy(s)).to(torch.bfloat16)
    assert np.array_equal(L.dequant_bf16_bits("fp8", codes, s), t.view(torch.int16).numpy().astype(np.uint16))
