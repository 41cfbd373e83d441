"""Every scale code of every format through the GEMM prologue's unpack.

Handles are built from constructed storage rather than from quantized
weights, so that each block-scale code the formats define meets each element
code: every non-negative finite E4M3 block scale x the 16 E2M1 codes
(NVFP4, the scale decode's subnormal branch included), every E8M0 exponent
x the 16 E2M1 codes (MXFP4, with exponents above 128 so that the handle's
power-of-two shift J is in play), INT4 and asymmetric-INT4 scales at the
bf16 extremes (subnormal, smallest normal, largest finite, zero, negative),
and every non-NaN E4M3 weight code x channel scales at the fp32 extremes.
The debug dequantization (the prologue's own unpack code) must equal the
oracle's bf16 bit patterns exactly ("TorchAO NVFP4 Weight-Only Quantization
(Linear)" and "TorchAO MXFP4 ... (Linear)", intros: block scales; the INT4
and FP8 weight-only pages, intros: group / channel scales).  Stored codes
the formats leave undefined are refused at create."""

import numpy as np
import pytest
import torch

import weight_only_quantized_prologue_b200 as dq
from oracle import linear as L
from oracle.quant import pack_nibbles

from gpu_util import dev, scales_tensor

pytestmark = pytest.mark.gpu


def _debug_bits(fmt, K, N, packed, scales, g=1.0):
    h = dq.dqgemm_create(fmt, K, N, dev(packed), scales_tensor(fmt, scales), g, None)
    try:
        out = torch.empty((N, K), dtype=torch.bfloat16, device="cuda")
        dq.dqgemm_dequantize(h, out)
        torch.cuda.synchronize()
        return out.view(torch.int16).cpu().numpy().view(np.uint16)
    finally:
        dq.dqgemm_destroy(h)


def _cycled_nibbles(N, K):
    """Element codes: row n, column k holds (k + n) mod 16, so every block
    of 16 consecutive k holds all 16 codes."""
    k = np.arange(K)[None, :]
    n = np.arange(N)[:, None]
    return ((k + n) % 16).astype(np.uint8)


def _assert_bits(got, ref):
    mism = np.argwhere(got != ref)
    assert mism.size == 0, (f"{len(mism)} mismatches, first {mism[:3].tolist()}: "
                            f"got {[hex(got[tuple(i)]) for i in mism[:3]]}, want {[hex(ref[tuple(i)]) for i in mism[:3]]}")


@pytest.mark.parametrize("g", [1.0, 3.0e-39, 1.0e30, 0.0173])
def test_nvfp4_every_block_scale_code(g):
    N, K = 128, 128                      # 1024 blocks of 16
    codes = _cycled_nibbles(N, K)
    blk = np.arange(N * (K // 16)).reshape(N, K // 16)
    sb = (blk % 127).astype(np.uint8)    # E4M3 codes 0x00..0x7E: zero, subnormals, normals to 448
    packed = pack_nibbles(codes)
    g = float(np.float32(g))
    ref = L.dequant_bf16_bits("nvfp4", packed, sb, g)
    _assert_bits(_debug_bits("nvfp4", K, N, packed, sb, g), ref)


@pytest.mark.parametrize("lo,hi", [(0, 128), (128, 254), (121, 254)])
def test_mxfp4_every_exponent_code(lo, hi):
    N, K = 160, 128                      # 640 blocks of 32
    codes = _cycled_nibbles(N, K)
    blk = np.arange(N * (K // 32)).reshape(N, K // 32)
    se = (lo + blk % (hi - lo + 1)).astype(np.uint8)
    packed = pack_nibbles(codes)
    ref = L.dequant_bf16_bits("mxfp4", packed, se)
    _assert_bits(_debug_bits("mxfp4", K, N, packed, se), ref)


_BF16_SCALES = np.array([0x0001, 0x0080, 0x007F, 0x3F80, 0x7F7F, 0x0000, 0xBF80, 0x8001, 0x5F00, 0x2000,
                         0x3C01, 0x0040, 0x7F00, 0xFF7F], dtype=np.uint16)


def test_int4_scales_at_bf16_extremes():
    N, K = 256, 512                      # 1024 groups of 128
    codes = _cycled_nibbles(N, K)        # two's-complement nibbles: every code -8..7
    grp = np.arange(N * (K // 128)).reshape(N, K // 128)
    s = _BF16_SCALES[grp % len(_BF16_SCALES)]
    packed = pack_nibbles(codes)
    ref = L.dequant_bf16_bits("int4", packed, s)
    _assert_bits(_debug_bits("int4", K, N, packed, s), ref)


def test_int4_asym_scales_and_zero_points_at_extremes():
    N, K = 256, 512
    codes = _cycled_nibbles(N, K)        # unsigned codes 0..15
    grp = np.arange(N * (K // 128)).reshape(N, K // 128)
    s = _BF16_SCALES[grp % len(_BF16_SCALES)]
    z = ((grp * 7) % 16).astype(np.uint8)
    packed = pack_nibbles(codes)
    sc = L.asym_scales_pack(s, z)
    ref = L.dequant_bf16_bits("int4_asym", packed, sc)
    _assert_bits(_debug_bits("int4_asym", K, N, packed, sc), ref)


_F32_SCALES = np.array([1.0, 2.0**-149, 1.0e-30, 3.4e38 / 448.0, 1.17549435e-38, 0.0, 2.0**-140, 0.0321,
                        1.0e20, 7.0], dtype=np.float32)


@pytest.mark.parametrize("fmt", ["fp8", "fp8_static"])
def test_fp8_every_weight_code_and_channel_scale_extremes(fmt):
    N, K = 40, 256
    codes = np.tile(np.arange(256, dtype=np.uint8), (N, 1))
    codes[codes == 0x7F] = 0x7E          # the two NaN codes are refused at create
    codes[codes == 0xFF] = 0xFE
    codes = np.ascontiguousarray(np.roll(codes, np.arange(N) % 7, axis=1))
    s = _F32_SCALES[np.arange(N) % len(_F32_SCALES)]
    ref = L.dequant_bf16_bits("fp8", codes, s)
    _assert_bits(_debug_bits(fmt, K, N, codes, s, 0.5), ref)


# -- stored codes the formats leave undefined are refused at create ----------


def _create_status(fmt, K, N, packed, scales, g=1.0):
    lib = dq._native.lib()
    p, s = dev(packed), scales_tensor(fmt, scales)
    h = dq._native.ctypes.c_void_p()
    st = lib.dqgemm_create(dq._native.ctypes.byref(h), dq.FORMATS[fmt], K, N, p.data_ptr(), s.data_ptr(),
                           float(g), None)
    if st == 0:
        dq.dqgemm_destroy(h)
    else:
        assert not h.value
    return st


def test_create_refuses_undefined_codes():
    N, K = 32, 128
    fp8 = np.zeros((N, K), dtype=np.uint8)
    fp8[3, 5] = 0xFF
    assert _create_status("fp8", K, N, fp8, np.ones(N, np.float32)) == dq._native.DQ_ERR_INVALID_ARG
    fp8[3, 5] = 0x7F
    assert _create_status("fp8_static", K, N, fp8, np.ones(N, np.float32), 0.1) == dq._native.DQ_ERR_INVALID_ARG
    packed = pack_nibbles(_cycled_nibbles(N, K))
    sb = np.full((N, K // 16), 0x38, np.uint8)
    sb[1, 2] = 0xB8                      # a negative block scale
    assert _create_status("nvfp4", K, N, packed, sb) == dq._native.DQ_ERR_INVALID_ARG
    sb[1, 2] = 0x7F                      # NaN
    assert _create_status("nvfp4", K, N, packed, sb) == dq._native.DQ_ERR_INVALID_ARG
    se = np.full((N, K // 32), 127, np.uint8)
    se[0, 0] = 255
    assert _create_status("mxfp4", K, N, packed, se) == dq._native.DQ_ERR_INVALID_ARG


def test_create_mxfp4_exponent_span():
    N, K = 32, 128
    codes = _cycled_nibbles(N, K)
    se = np.full((N, K // 32), 200, np.uint8)
    se[4, 1] = 66                        # 200 - 134: one binade too far below the largest exponent
    assert _create_status("mxfp4", K, N, pack_nibbles(codes), se) == dq._native.DQ_ERR_UNSUPPORTED
    codes[4, 32:64] = 0                  # ... unless that block is all zeros
    assert _create_status("mxfp4", K, N, pack_nibbles(codes), se) == dq._native.DQ_OK
    codes[4, 32:64] = 8                  # -0 elements are zero too
    assert _create_status("mxfp4", K, N, pack_nibbles(codes), se) == dq._native.DQ_OK
    codes = _cycled_nibbles(N, K)
    se[4, 1] = 67                        # 200 - 133: the edge of the exact range
    assert _create_status("mxfp4", K, N, pack_nibbles(codes), se) == dq._native.DQ_OK
    bits = _debug_bits("mxfp4", K, N, pack_nibbles(codes), se)
    _assert_bits(bits, L.dequant_bf16_bits("mxfp4", pack_nibbles(codes), se))
