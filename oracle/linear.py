"""Dequantization, the fp64 reference of the quantized Linear, static-FP8
activation quantization and calibration, and SQNR.

TEST INFRASTRUCTURE ONLY (see ``oracle/__init__.py``).

Format names used here and by the tests:
  "int4"       symmetric group-128 INT4     (INT4 weight-only page)
  "nvfp4"      E2M1 + E4M3/16 + fp32 global (NVFP4 weight-only page)
  "mxfp4"      E2M1 + E8M0/32               (MXFP4 page)
  "fp8"        E4M3 + fp32 per channel      (FP8 weight-only page)
  "fp8_static" E4M3 weights and activations (static FP8 page)

The FP4 x FP4 section at the end (dynamic activation quantization and the
W4A4 reference) is the native-MMA variant the MXFP4 page names.
"""

import numpy as np

from .formats import (
    bf16,
    bf16_bits,
    bf16_from_bits,
    e2m1_decode,
    e4m3_decode,
    e4m3_encode,
    e4m3_round,
    e8m0_decode,
    f32,
)
from .quant import (
    INT4_GROUP,
    MXFP4_BLOCK,
    NVFP4_BLOCK,
    pack_nibbles,
    quantize_fp8_rows,
    quantize_int4,
    quantize_int4_asym,
    quantize_mxfp4,
    quantize_nvfp4,
    unpack_nibbles,
)

FORMATS = ("int4", "nvfp4", "mxfp4", "fp8", "fp8_static", "int4_asym")


def asym_scales_pack(scale_bits, zeros):
    """The canonical scale storage of asymmetric INT4: the bf16 scales
    [N, G] (little-endian bytes, row-major) followed by the zero points
    [N, G], as one uint8 array of 3 * N * G bytes."""
    s = np.ascontiguousarray(scale_bits, dtype="<u2").view(np.uint8).reshape(-1)
    return np.concatenate([s, np.ascontiguousarray(zeros, dtype=np.uint8).reshape(-1)])


def asym_scales_split(buf, N, G):
    """Inverse of asym_scales_pack: (scale bits uint16 [N, G], zeros uint8 [N, G])."""
    buf = np.ascontiguousarray(buf, dtype=np.uint8).reshape(-1)
    s = buf[: 2 * N * G].view("<u2").reshape(N, G)
    return s, buf[2 * N * G: 3 * N * G].reshape(N, G)


def quantize_pack(fmt, W):
    """Quantize W [N, K] and return the storage arrays of the library's
    canonical layout as a dict: ``packed`` (uint8 [N, K/2] for 4-bit formats,
    [N, K] for FP8), ``scales`` (INT4: uint16 bf16 bits [N, K/128]; NVFP4:
    uint8 E4M3 [N, K/16]; MXFP4: uint8 E8M0 [N, K/32]; FP8: float32 [N];
    asymmetric INT4: asym_scales_pack of the bf16 scales and the zero points)
    and ``global_scale`` (NVFP4's g, else 1.0)."""
    if fmt == "int4":
        codes, s = quantize_int4(W)
        return dict(packed=pack_nibbles(codes), scales=s, global_scale=1.0)
    if fmt == "int4_asym":
        codes, s, z = quantize_int4_asym(W)
        return dict(packed=pack_nibbles(codes), scales=asym_scales_pack(s, z), global_scale=1.0)
    if fmt == "nvfp4":
        codes, sb, g = quantize_nvfp4(W)
        return dict(packed=pack_nibbles(codes), scales=sb, global_scale=g)
    if fmt == "mxfp4":
        codes, se = quantize_mxfp4(W)
        return dict(packed=pack_nibbles(codes), scales=se, global_scale=1.0)
    if fmt in ("fp8", "fp8_static"):
        codes, s = quantize_fp8_rows(W)
        return dict(packed=codes, scales=s.astype(np.float32), global_scale=1.0)
    raise ValueError(fmt)


def dequant_exact(fmt, packed, scales, global_scale=1.0):
    """Exact real value of every stored weight, code x scale(s), in fp64
    (no rounding: every such product is exact in fp64).  This is the weight
    the GEMM reference multiplies by.  Parity: pinned by brute force over
    every code x scale code pair and the scale-one special case."""
    if fmt == "int4":
        c = unpack_nibbles(packed, signed=True).astype(np.float64)
        s = np.repeat(bf16_from_bits(scales), INT4_GROUP, axis=1)
        return c * s
    if fmt == "int4_asym":
        u = unpack_nibbles(packed).astype(np.float64)
        N = u.shape[0]
        sb, z = asym_scales_split(scales, N, u.shape[1] // INT4_GROUP)
        s = np.repeat(bf16_from_bits(sb), INT4_GROUP, axis=1)
        return (u - np.repeat(z.astype(np.float64), INT4_GROUP, axis=1)) * s
    if fmt == "nvfp4":
        v = e2m1_decode(unpack_nibbles(packed))
        sb = np.repeat(e4m3_decode(scales), NVFP4_BLOCK, axis=1)
        return v * sb * float(global_scale)
    if fmt == "mxfp4":
        v = e2m1_decode(unpack_nibbles(packed))
        return v * np.repeat(e8m0_decode(scales), MXFP4_BLOCK, axis=1)
    if fmt in ("fp8", "fp8_static"):
        s = np.asarray(scales, dtype=np.float64)[:, None]
        return e4m3_decode(packed) * s
    raise ValueError(fmt)


def dequant_bf16_bits(fmt, packed, scales, global_scale=1.0):
    """The debug dequantization to bf16, as uint16 bit patterns [N, K]:
      INT4   bf16(c * s)                    (c * s is exact in fp32)
      INT4 asymmetric  bf16((c - z) * s)    (exact in fp32 as well)
      NVFP4  bf16(f32(e2m1 * dec(sb) * g))  (e2m1 * dec(sb) is exact)
      MXFP4  bf16(e2m1 * 2**(e-127))
      FP8    bf16(f32(e4m3 * s[n]))
    -0.0 is kept (a negative code times a positive scale, or code -0).
    Parity: pinned by brute force over code x scale pairs in the tests."""
    if fmt in ("int4", "int4_asym"):
        return bf16_bits(bf16(dequant_exact(fmt, packed, scales)))
    if fmt == "nvfp4":
        v = e2m1_decode(unpack_nibbles(packed))
        sb = np.repeat(e4m3_decode(scales), NVFP4_BLOCK, axis=1)
        return bf16_bits(bf16(f32(v * sb * float(global_scale))))
    if fmt == "mxfp4":
        return bf16_bits(bf16(dequant_exact(fmt, packed, scales)))
    if fmt in ("fp8", "fp8_static"):
        return bf16_bits(bf16(f32(dequant_exact(fmt, packed, scales))))
    raise ValueError(fmt)


def linear_ref(x, w_exact, bias=None):
    """y = x . w^T + b in fp64 (nn.Linear; "Define a linear model..." section
    of the weight-only pages).  x [M, K] and bias [N] are taken at their
    stored (bf16) values; the result is not rounded."""
    y = np.asarray(x, dtype=np.float64) @ np.asarray(w_exact, dtype=np.float64).T
    if bias is not None:
        y = y + np.asarray(bias, dtype=np.float64)[None, :]
    return y


# ---------------------------------------------------------------------------
# static FP8 ("TorchAO Static FP8 Quantization (Linear)")
# ---------------------------------------------------------------------------


def quantize_act_fp8(x, s_x):
    """Activation Q of the static recipe (the Q node of the page's "Graph
    after export"): code = e4m3(f32(x / s_x)), x at its bf16 value, s_x an
    fp32 per-tensor scale, saturating at +-448.  Returns uint8 codes.
    Parity: pinned by the E4M3 codec pins and torch's float8 cast."""
    q = e4m3_round(f32(np.asarray(x, dtype=np.float64) / float(s_x)))
    return e4m3_encode(q)


def act_scale(lo, hi):
    """Per-tensor scale from observed min/max: f32(max(|lo|, |hi|) / 448).
    Reading: symmetric E4M3 scaling of the observer range."""
    return float(f32(max(abs(float(lo)), abs(float(hi))) / 448.0))


def static_linear(q_x, s_x, q_w, s_w):
    """One static-FP8 Linear without bias (the page's model has
    bias=False): y = s_x * s_w[n] * sum_k dec(q_x) dec(q_w), in fp64 (the
    FP8 x FP8 products and their sum are exact in fp64 for the page's
    sizes).  The result is not rounded."""
    acc = e4m3_decode(q_x) @ e4m3_decode(q_w).T
    return acc * float(s_x) * np.asarray(s_w, dtype=np.float64)[None, :]


def calibrate_static_mlp(batches, w1, w2):
    """Per-tensor activation scales of the two-layer model from min/max
    observers over calibration batches ("Calibrate, then insert static FP8
    Q/DQ").  Observers watch the float (bf16) model: layer 1's input is the
    batch itself, layer 2's input is h = bf16(x . w1^T).
    Reading: the float model's Linear is taken as the exact product rounded
    once to bf16.  Returns (s_x1, s_x2).  The pages print no scale values;
    parity is pinned by invariants (batch order, monotonicity under an extra
    batch, exact 2^j equivariance) and by constructed cases that fix the
    symmetric range and the bf16 rounding of layer 1's output.  Both the
    oracle and the GPU path receive these scales as inputs, so GEMM parity
    does not depend on them."""
    lo1 = hi1 = lo2 = hi2 = None
    for x in batches:
        x = np.asarray(x, dtype=np.float64)
        h = bf16(x @ np.asarray(w1, dtype=np.float64).T)
        lo1 = x.min() if lo1 is None else min(lo1, x.min())
        hi1 = x.max() if hi1 is None else max(hi1, x.max())
        lo2 = h.min() if lo2 is None else min(lo2, h.min())
        hi2 = h.max() if hi2 is None else max(hi2, h.max())
    return act_scale(lo1, hi1), act_scale(lo2, hi2)


def static_mlp(x, s_x1, q_w1, s_w1, s_x2, q_w2, s_w2):
    """The page's two-layer model after static FP8 Q/DQ: h = bf16(layer1),
    y = bf16(layer2(Q(h))).  Returns (h, y) as fp64 values of bf16.
    Parity: pinned by a two-layer case worked by hand in which the bf16
    rounding of h, layer 2's own activation scale, its Q node and the
    orientation of W1 each change the result."""
    h = bf16(static_linear(quantize_act_fp8(x, s_x1), s_x1, q_w1, s_w1))
    y = bf16(static_linear(quantize_act_fp8(h, s_x2), s_x2, q_w2, s_w2))
    return h, y


def sqnr(a, b):
    """Signal-to-quantization-noise ratio in dB, 20 log10(|a| / |a - b|) with
    the noise norm clamped at 1e-12 (the helper on the static FP8 page,
    "Imports" section).  Diagnostic only: the pages print no SQNR values to
    compare against; the function itself is pinned by closed forms (b = a
    gives the clamp, b = 0 gives 0 dB, b = a (1 + eps) gives -20 log10 eps)."""
    a = np.asarray(a, dtype=np.float64).ravel()
    b = np.asarray(b, dtype=np.float64).ravel()
    noise = max(np.linalg.norm(a - b), 1e-12)
    return 20.0 * np.log10(np.linalg.norm(a) / noise)


# ---------------------------------------------------------------------------
# FP4 x FP4 ("TorchAO MXFP4 Dynamic Activation + MX Weight (Linear)", intro:
# the config is MX dynamic activation + MX weight, and native MXFP4 x MXFP4
# needs B200): the reference of that path.
# ---------------------------------------------------------------------------


def quantize_act_mxfp4(x):
    """Dynamic MX activation quantization: every row of x [M, K] (at its
    bf16 value) is cut into blocks of 32 along K and quantized at call time
    with the same recipe as the MX weight (shared exponent
    floor(log2 amax) - 2, E2M1 elements).
    Reading: "dynamic activation" means the scales come from the call's own
    x, block by block along the reduction dimension, as for the weight.
    Returns (codes uint8 [M, K], E8M0 scale codes uint8 [M, K/32]).
    Parity: pinned by the MX weight pins (same quantizer) and by the
    power-of-two and sign symmetries of the W4A4 tests."""
    return quantize_mxfp4(np.asarray(x, dtype=np.float64))


def quantize_act_nvfp4(x):
    """Dynamic NVFP4 activation quantization: x [M, K] as one tensor through
    the NVFP4 recipe (per-tensor fp32 global scale from amax(x), E4M3 scale
    per block of 16 along K, E2M1 elements).
    Reading: the pages pair NVFP4 only with BF16 activations; this is the
    weight recipe applied to x unchanged, the global scale taken per call.
    Returns (codes uint8 [M, K], E4M3 scale codes uint8 [M, K/16], g_x).
    Parity: pinned as quantize_act_mxfp4."""
    return quantize_nvfp4(np.asarray(x, dtype=np.float64))


def w4a4_linear_ref(fmt, x, packed_w, scales_w, global_scale_w=1.0, bias=None):
    """FP4 x FP4 Linear: y = sum_k deq(Q(x))[m, k] * deq(W)[n, k] + b[n], with
    Q the dynamic activation quantizer of `fmt` ("mxfp4" or "nvfp4") and W in
    the same format's storage.  Every dequantized operand is exact in fp64,
    so this is the exact product of the two dequantized matrices plus the
    bias; not rounded (the kernel rounds to bf16 once).
    Parity: pinned by on-grid activations reducing to the weight-only
    reference, brute force on a tiny case, and exact power-of-two and sign
    symmetries."""
    if fmt == "mxfp4":
        cx, sx = quantize_act_mxfp4(x)
        xd = e2m1_decode(cx) * np.repeat(e8m0_decode(sx), MXFP4_BLOCK, axis=1)
    elif fmt == "nvfp4":
        cx, sx, gx = quantize_act_nvfp4(x)
        xd = e2m1_decode(cx) * np.repeat(e4m3_decode(sx), NVFP4_BLOCK, axis=1) * float(gx)
    else:
        raise ValueError(fmt)
    return linear_ref(xd, dequant_exact(fmt, packed_w, scales_w, global_scale_w), bias)
