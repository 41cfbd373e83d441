"""Number formats used by the five quantized-Linear recipes, written out in fp64.

TEST INFRASTRUCTURE ONLY (see ``oracle/__init__.py``).

Sources.  The pages name the formats without defining them:
  * "TorchAO NVFP4 Weight-Only Quantization (Linear)", intro: packed FP4 E2M1
    weights, FP8 E4M3 block scales, an FP32 global scale.
  * "TorchAO MXFP4 Dynamic Activation + MX Weight (Linear)", intro: packed FP4
    E2M1 weights with E8M0 block scales, block size 32.
  * "TorchAO FP8 Weight-Only Quantization (Linear)" and "TorchAO Static FP8
    Quantization (Linear)", intro: FP8 e4m3.
  * every page's "Define a linear model..." section: the model runs in bf16.
The bit-level definitions below are the public OCP 8-bit / MX format
definitions (E4M3 "fn": bias 7, no infinities, S.1111.111 is NaN, max 448;
E2M1: bias 1, values {0, .5, 1, 1.5, 2, 3, 4, 6}; E8M0: 2^(e-127), 0xFF NaN)
and IEEE-754 binary32 / bfloat16 with round-to-nearest-even.

Everything is computed in fp64, where every value of these formats and every
product used here is exact; rounding happens only where a function says so.
"""

import numpy as np

# ---------------------------------------------------------------------------
# generic round-to-nearest-even onto a binary floating-point grid
# ---------------------------------------------------------------------------


def round_to_grid(v, man_bits, min_exp, max_val=None):
    """Round real values to the nearest point of a binary float grid, ties to
    the even significand (IEEE round-to-nearest-even).

    The grid has ``man_bits`` explicit significand bits, smallest normal
    exponent ``min_exp`` (so subnormals are spaced 2**(min_exp - man_bits)),
    and, when ``max_val`` is given, magnitudes are first clamped to
    ``max_val`` (saturating conversion; ``max_val`` must be a grid point).
    The sign is kept, so a negative value that rounds to zero gives -0.0.

    Parity: pinned by brute-force nearest-point search over every grid
    midpoint (tests/test_oracle_formats.py) and, for bf16 / e4m3, by torch's
    own dtype casts.
    """
    v = np.asarray(v, dtype=np.float64)
    a = np.abs(v)
    if max_val is not None:
        a = np.minimum(a, max_val)
    _, e = np.frexp(a)                      # a = f * 2**e with f in [0.5, 1)
    lead = np.maximum(e - 1, min_exp)       # exponent of the leading bit
    quantum = np.ldexp(1.0, lead - man_bits)
    r = np.rint(a / quantum) * quantum      # np.rint rounds half to even
    return np.copysign(r, v)


# ---------------------------------------------------------------------------
# FP32 and BF16
# ---------------------------------------------------------------------------


def f32(v):
    """IEEE binary32 round-to-nearest-even of real (fp64) values, returned as
    fp64.  This is the rounding every fp32 operation of the recipes applies
    to its exact result.  Parity: numpy's float32 cast is the IEEE
    conversion; pinned by re-deriving a few values by hand in the tests."""
    return np.asarray(v, dtype=np.float64).astype(np.float32).astype(np.float64)


BF16_MAX = float.fromhex("0x1.fep127")


def bf16(v):
    """Round real values to bfloat16 (8 significand bits, exponent range of
    fp32, subnormals kept), ties to even; magnitudes past the largest finite
    bf16 after rounding become +-inf.  Returned as fp64 values.
    Parity: pinned against torch's fp32->bf16 cast (which is RNE)."""
    r = round_to_grid(v, 7, -126)
    return np.where(np.abs(r) > BF16_MAX, np.copysign(np.inf, r), r)


def bf16_bits(v):
    """The 16-bit pattern (uint16) of bf16 values given as fp64 (exactly
    representable in bf16, including -0.0)."""
    v32 = np.asarray(v, dtype=np.float64).astype(np.float32)
    return (v32.view(np.uint32) >> 16).astype(np.uint16)


def bf16_from_bits(bits):
    """fp64 values of bf16 bit patterns."""
    b = np.asarray(bits, dtype=np.uint16).astype(np.uint32) << 16
    return b.view(np.float32).astype(np.float64)


# ---------------------------------------------------------------------------
# E2M1 (FP4)
# ---------------------------------------------------------------------------

E2M1_MAGNITUDES = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0])
E2M1_MAX = 6.0


def e2m1_decode(code):
    """Value of 4-bit E2M1 codes s|e1 e0|m: bias 1, one mantissa bit, the
    subnormal code 0b001 is 0.5; bit 3 is the sign."""
    code = np.asarray(code, dtype=np.int64)
    mag = code & 7
    e = mag >> 1
    m = mag & 1
    val = np.where(e == 0, m * 0.5, np.ldexp(1.0 + m / 2.0, e - 1))
    return np.where(code & 8, -val, val)


def e2m1_round(v):
    """Round to the E2M1 grid, saturating at +-6, ties to even."""
    return round_to_grid(v, 1, 0, E2M1_MAX)


def e2m1_encode(v):
    """Code of values that lie on the E2M1 grid (sign bit kept for -0.0)."""
    v = np.asarray(v, dtype=np.float64)
    a = np.abs(v)
    idx = np.searchsorted(E2M1_MAGNITUDES, a)
    if np.any(idx >= 8) or np.any(E2M1_MAGNITUDES[np.minimum(idx, 7)] != a):
        raise ValueError("value not on the E2M1 grid")
    return (idx | np.where(np.signbit(v), 8, 0)).astype(np.uint8)


# ---------------------------------------------------------------------------
# E4M3 ("fn": no infinities, 0x7F / 0xFF are NaN, max 448)
# ---------------------------------------------------------------------------

E4M3_MAX = 448.0


def e4m3_decode(code):
    """Value of 8-bit E4M3 codes: bias 7, three mantissa bits, subnormals
    m * 2**-9, S.1111.111 is NaN, no infinities."""
    code = np.asarray(code, dtype=np.int64)
    e = (code >> 3) & 15
    m = code & 7
    val = np.where(e == 0, m * 2.0**-9, np.ldexp(1.0 + m / 8.0, e - 7))
    val = np.where((code & 0x7F) == 0x7F, np.nan, val)
    return np.where(code & 0x80, -val, val)


def e4m3_round(v):
    """Saturating E4M3 rounding: clamp to +-448, then round to nearest even.
    NaN stays NaN."""
    return round_to_grid(v, 3, -6, E4M3_MAX)


def e4m3_encode(v):
    """Code of values that lie on the E4M3 grid (sign kept for -0.0; NaN
    encodes as 0x7F)."""
    v = np.asarray(v, dtype=np.float64)
    a = np.abs(v)
    nan = np.isnan(a)
    a = np.where(nan, 0.0, a)
    _, e = np.frexp(a)
    lead = e - 1
    normal = (lead >= -6) & (a > 0)
    field_e = np.where(normal, lead + 7, 0)
    mant = np.where(normal, a / np.ldexp(1.0, lead) - 1.0, a / 2.0**-9) * np.where(normal, 8, 1)
    if np.any(mant != np.rint(mant)) or np.any(field_e > 15):
        raise ValueError("value not on the E4M3 grid")
    code = (field_e.astype(np.int64) << 3) | mant.astype(np.int64)
    code = np.where(np.signbit(v), code | 0x80, code)
    code = np.where(nan, 0x7F, code)
    return code.astype(np.uint8)


# ---------------------------------------------------------------------------
# E8M0 (power-of-two scale)
# ---------------------------------------------------------------------------


def e8m0_decode(code):
    """2**(code - 127); 0xFF is NaN."""
    code = np.asarray(code, dtype=np.int64)
    return np.where(code == 255, np.nan, np.ldexp(1.0, code - 127))
