"""Weight quantizers and the nibble packer of the five recipes, in fp64.

TEST INFRASTRUCTURE ONLY (see ``oracle/__init__.py``).

W is an ``[N, K]`` array (nn.Linear layout: out_features x in_features) of
fp32-representable values; groups and blocks run along K.  Every fp32
operation of a recipe is written as the exact fp64 operation followed by
``f32()``; for a single division or product this equals the IEEE fp32
operation (fp64 carries more than 2*24+2 bits, so the double rounding is
innocuous).  Where the pages leave a choice open, the reading taken is stated
in the docstring.

Returned codes are unpacked (one code per element); ``pack_nibbles`` makes
the two-codes-per-byte storage.
"""

import numpy as np

from .formats import (
    bf16,
    bf16_bits,
    e2m1_encode,
    e2m1_round,
    e4m3_decode,
    e4m3_encode,
    e4m3_round,
    f32,
)

INT4_GROUP = 128
NVFP4_BLOCK = 16
MXFP4_BLOCK = 32
NVFP4_GLOBAL_DIV = 6.0 * 448.0     # 2688: E2M1 max times E4M3 max


def _blocks(W, size):
    N, K = W.shape
    if K % size:
        raise ValueError(f"K={K} is not a multiple of the block size {size}")
    return W.reshape(N, K // size, size)


def _amax_blocks(W, size):
    return np.abs(_blocks(W, size)).max(axis=2)


def quantize_int4(W, group=INT4_GROUP):
    """Symmetric group-wise INT4 ("TorchAO INT4 Weight-Only Quantization
    (Linear)", intro and "Define a linear model and quantize weights to
    symmetric INT4": symmetric quantizer, zero-point 0, group_size=128).

    Per row n and group j of ``group`` consecutive k:
      a = max |W|;  s = bf16(f32(a / 7));
      code = clamp(RNE(f32(W / s)), -8, 7);  a group with s == 0 has codes 0.
    Readings (the page gives neither): divisor 7 (= amax / qmax of a
    symmetric [-8, 7] code), scale stored in the model dtype bf16.

    Returns (codes int8 [N, K], scale bits uint16 [N, K/group]).
    Parity: pinned by invariants (|code| <= 7, group max maps to +-7),
    idempotence and the scale-one special case in the tests.
    """
    W = np.asarray(W, dtype=np.float64)
    a = _amax_blocks(W, group)
    s = bf16(f32(a / 7.0))
    s_full = np.repeat(s, group, axis=1)
    safe = np.where(s_full > 0, s_full, 1.0)
    q = np.rint(f32(W / safe))
    q = np.clip(q, -8, 7)
    q = np.where(s_full > 0, q, 0.0)
    return q.astype(np.int8), bf16_bits(s)


def quantize_int4_asym(W, group=INT4_GROUP):
    """Asymmetric group-wise INT4 with a per-group zero point: the
    zero-point counterpart of "TorchAO INT4 Weight-Only Quantization
    (Linear)" (that page's quantizer is the symmetric one, zero-point 0).

    Per row n and group j of ``group`` consecutive k:
      lo = min(0, min W),  hi = max(0, max W);  s = bf16(f32(f32(hi - lo) / 15));
      z = clamp(RNE(f32(-lo / s)), 0, 15);
      code = clamp(RNE(f32(W / s)) + z, 0, 15)  (unsigned);
      dequantized weight (code - z) * s;  a group with s == 0 has codes 0, z 0.
    Readings (no page gives them): the range includes 0 so that zero is
    exactly representable, the scale is bf16 like the symmetric format's,
    the zero point an integer in [0, 15], and the range is formed in fp32
    before the division (the order of the fp32 operations is fixed here).

    Returns (codes uint8 [N, K], scale bits uint16 [N, K/group], zero points
    uint8 [N, K/group]).
    Parity: pinned by the on-grid round trip (weights built as
    (c - z) * s with every c in 0..15 quantize back to exactly c, z, s), by
    the all-zero and non-negative special cases, and by idempotence.
    """
    W = np.asarray(W, dtype=np.float64)
    B = _blocks(W, group)
    lo = np.minimum(B.min(axis=2), 0.0)
    hi = np.maximum(B.max(axis=2), 0.0)
    s = bf16(f32(f32(hi - lo) / 15.0))
    safe = np.where(s > 0, s, 1.0)
    z = np.clip(np.rint(f32(-lo / safe)), 0, 15)
    z = np.where(s > 0, z, 0.0)
    s_full = np.repeat(safe, group, axis=1)
    z_full = np.repeat(z, group, axis=1)
    q = np.clip(np.rint(f32(W / s_full)) + z_full, 0, 15)
    q = np.where(np.repeat(s, group, axis=1) > 0, q, 0.0)
    return q.astype(np.uint8), bf16_bits(s), z.astype(np.uint8)


def quantize_nvfp4(W):
    """NVFP4 ("TorchAO NVFP4 Weight-Only Quantization (Linear)", intro:
    packed FP4 E2M1 weights, FP8 E4M3 block scales, FP32 global scale; the
    last two weight dims divisible by 16).

      g  = f32(amax(W) / 2688)            (g = 1 for an all-zero tensor)
      per block of 16 along K:  sb = e4m3(f32(f32(amax_blk / 6) / g))
      d  = f32(dec(sb) * g);  code = e2m1(f32(W / d))   (codes 0 when d == 0)
    Readings: block size 16 (the page states only the divisibility), the
    order of the fp32 operations above, g = 1 for a zero tensor.

    Returns (codes uint8 [N, K] in 0..15, block-scale codes uint8 [N, K/16],
    g as a Python float holding an fp32 value).
    Parity: pinned by the tensor-max block mapping to sb = 448 and to +-6,
    idempotence, and the E2M1/E4M3 codec pins.
    """
    W = np.asarray(W, dtype=np.float64)
    amax = float(np.abs(W).max()) if W.size else 0.0
    g = float(f32(amax / NVFP4_GLOBAL_DIV)) if amax > 0 else 1.0
    ab = _amax_blocks(W, NVFP4_BLOCK)
    sb_val = e4m3_round(f32(f32(ab / 6.0) / g))
    sb = e4m3_encode(sb_val)
    d = np.repeat(f32(sb_val * g), NVFP4_BLOCK, axis=1)
    safe = np.where(d > 0, d, 1.0)
    v = e2m1_round(f32(W / safe))
    v = np.where(d > 0, v, 0.0)
    return e2m1_encode(v), sb, g


def mxfp4_block_exponent(ab):
    """Shared exponent of an MX block: floor(log2(amax)) - 2, clamped to
    [-127, 127]; taken from frexp, so it is exact (no log2 call)."""
    _, ex = np.frexp(np.asarray(ab, dtype=np.float64))
    e = ex.astype(np.int64) - 3          # floor(log2 a) = ex - 1
    return np.clip(e, -127, 127)


def quantize_mxfp4(W):
    """MXFP4 ("TorchAO MXFP4 Dynamic Activation + MX Weight (Linear)", intro:
    packed FP4 E2M1 weights, E8M0 block scales, block size 32; dims divisible
    by 32).

    Per block of 32 along K with a = max |W|:
      e = floor(log2 a) - 2 clamped to [-127, 127];  scale code = e + 127;
      code = e2m1(W * 2**-e)        (the product is exact in fp32);
      a block with a == 0 gets scale code 0 and element codes 0.
    Reading: the exponent comes from the true floor(log2 a) (frexp); for an
    fp32-normal amax this is the exponent field minus 127.

    Returns (codes uint8 [N, K], scale codes uint8 [N, K/32]).
    Parity: pinned by the invariant a / 2**e in [4, 8), idempotence with
    recomputed scales, and the codec pins.
    """
    W = np.asarray(W, dtype=np.float64)
    ab = _amax_blocks(W, MXFP4_BLOCK)
    e = mxfp4_block_exponent(np.where(ab > 0, ab, 1.0))
    code_e = np.where(ab > 0, e + 127, 0)
    e_full = np.repeat(np.where(ab > 0, e, 0), MXFP4_BLOCK, axis=1)
    v = e2m1_round(f32(W * np.ldexp(1.0, -e_full)))
    zero = np.repeat(ab == 0, MXFP4_BLOCK, axis=1)
    v = np.where(zero, 0.0, v)
    return e2m1_encode(v), code_e.astype(np.uint8)


def quantize_fp8_rows(W):
    """FP8 E4M3 with one fp32 scale per output channel ("TorchAO FP8
    Weight-Only Quantization (Linear)", intro; "TorchAO Static FP8
    Quantization (Linear)", "Calibrate, then insert static FP8 Q/DQ": per-
    channel weight min/max observers).

      s[n] = f32(max(|min_n|, |max_n|) / 448);  code = e4m3(f32(W / s[n]))
      a row with s == 0 has codes 0.
    Reading: the weight-only page does not state the scale granularity; one
    scale per output channel is taken, the granularity the static page's
    weight observers use.

    Returns (codes uint8 [N, K], scales float64 [N] holding fp32 values).
    Parity: pinned by the row max mapping to +-448, idempotence and the
    E4M3 codec pins.
    """
    W = np.asarray(W, dtype=np.float64)
    lo = W.min(axis=1)
    hi = W.max(axis=1)
    s = f32(np.maximum(np.abs(lo), np.abs(hi)) / 448.0)
    safe = np.where(s > 0, s, 1.0)[:, None]
    v = e4m3_round(f32(W / safe))
    v = np.where(s[:, None] > 0, v, 0.0)
    return e4m3_encode(v), s


def pack_nibbles(codes):
    """Two 4-bit codes per byte along K: byte[n, j] holds code[n, 2j] in the
    low nibble and code[n, 2j+1] in the high nibble (two's complement for
    INT4).  Reading: the nibble order is not stated on the INT4 page's
    build-time repack; low nibble = even k is taken."""
    c = np.asarray(codes).astype(np.int64) & 0xF
    if c.shape[-1] % 2:
        raise ValueError("K must be even to pack nibbles")
    return (c[..., 0::2] | (c[..., 1::2] << 4)).astype(np.uint8)


def unpack_nibbles(packed, signed=False):
    """Inverse of pack_nibbles; ``signed`` sign-extends (INT4)."""
    p = np.asarray(packed, dtype=np.int64)
    out = np.empty(p.shape[:-1] + (p.shape[-1] * 2,), dtype=np.int64)
    out[..., 0::2] = p & 0xF
    out[..., 1::2] = p >> 4
    if signed:
        out = np.where(out >= 8, out - 16, out)
    return out


def e4m3_values(codes):
    """Alias kept beside the quantizers for readability of callers."""
    return e4m3_decode(codes)
