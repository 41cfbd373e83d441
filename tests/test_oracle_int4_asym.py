"""Pins of the asymmetric INT4 oracle (per-group zero point): checks that
do not restate its formula."""

import numpy as np
import pytest

from oracle import formats as F
from oracle import linear as L
from oracle import quant as Q


def _on_grid(rng, N, groups):
    """Weights built as (c - z) * s, each group holding every code 0..15 at
    least once: quantization must give back exactly c, z and s."""
    c = np.empty((N, groups * 128), dtype=np.int64)
    for n in range(N):
        for g in range(groups):
            blk = np.concatenate([np.arange(16), rng.integers(0, 16, 112)])
            c[n, g * 128:(g + 1) * 128] = rng.permutation(blk)
    z = rng.integers(0, 16, (N, groups))
    s = F.bf16(rng.uniform(1e-3, 0.2, (N, groups)))   # exactly representable in bf16
    W = (c - np.repeat(z, 128, axis=1)) * np.repeat(s, 128, axis=1)
    return W, c, z, s


def test_on_grid_weights_round_trip_exactly():
    rng = np.random.default_rng(0)
    W, c, z, s = _on_grid(rng, 24, 3)
    # the construction itself is exact in fp64 (small integer times bf16)
    codes, sb, zz = Q.quantize_int4_asym(W)
    # hi - lo = 15 s exactly, so the scale, the zero point and every code
    # come back exactly
    assert (F.bf16_from_bits(sb) == s).all()
    assert (zz == z).all()
    assert (codes == c).all()


def test_all_zero_group_and_non_negative_group():
    W = np.zeros((2, 256))
    W[1, 128:] = np.linspace(0.0, 3.0, 128)      # non-negative: zero point 0
    codes, sb, z = Q.quantize_int4_asym(W)
    assert (codes[0] == 0).all() and (codes[1, :128] == 0).all()
    assert sb[0, 0] == 0 and z[0, 0] == 0 and z[1, 1] == 0
    assert F.bf16_from_bits(sb[1, 1]) == F.bf16(F.f32(3.0 / 15.0))
    assert codes[1, 255] == 15 and codes[1, 128] == 0
    # the exact zero of the data dequantizes to exactly zero
    st = L.quantize_pack("int4_asym", W)
    assert L.dequant_exact("int4_asym", st["packed"], st["scales"])[1, 128] == 0.0


def test_range_always_includes_zero():
    W = np.linspace(1.0, 3.0, 128)[None, :]       # strictly positive group
    codes, sb, z = Q.quantize_int4_asym(W)
    assert z[0, 0] == 0
    assert F.bf16_from_bits(sb[0, 0]) == F.bf16(F.f32(3.0 / 15.0))
    W = -np.linspace(1.0, 3.0, 128)[None, :]      # strictly negative group
    codes, sb, z = Q.quantize_int4_asym(W)
    assert z[0, 0] == 15 and codes[0, 0] == 15 - 5 and codes[0, 127] == 0


def test_codes_in_range_and_group_extremes_hit_the_ends():
    rng = np.random.default_rng(1)
    W = rng.normal(0, 1, (16, 512)) * rng.uniform(0.1, 3, (16, 1))
    codes, sb, z = Q.quantize_int4_asym(W)
    assert codes.min() >= 0 and codes.max() <= 15
    B = W.reshape(16, 4, 128)
    C = codes.reshape(16, 4, 128)
    lo_idx, hi_idx = B.argmin(axis=2), B.argmax(axis=2)
    lo_code = np.take_along_axis(C, lo_idx[..., None], 2)[..., 0]
    hi_code = np.take_along_axis(C, hi_idx[..., None], 2)[..., 0]
    assert (lo_code <= 1).all() and (hi_code >= 14).all()


def test_requantizing_the_dequantized_weight_is_idempotent():
    rng = np.random.default_rng(2)
    W = rng.uniform(-0.3, 1.1, (8, 384))
    st = L.quantize_pack("int4_asym", W)
    wd = L.dequant_exact("int4_asym", st["packed"], st["scales"])
    st2 = L.quantize_pack("int4_asym", wd)
    assert (st2["packed"] == st["packed"]).all()
    assert (st2["scales"] == st["scales"]).all()


def test_dequant_error_is_within_half_a_step():
    rng = np.random.default_rng(3)
    W = F.f32(rng.normal(0, 1, (8, 256)))
    st = L.quantize_pack("int4_asym", W)
    wd = L.dequant_exact("int4_asym", st["packed"], st["scales"])
    sb, _ = L.asym_scales_split(st["scales"], 8, 2)
    step = np.repeat(F.bf16_from_bits(sb), 128, axis=1)
    # inside the representable range the error is at most half a step (plus
    # the f32 rounding of W / s)
    assert (np.abs(W - wd) <= 0.5 * step * (1 + 1e-6) + 1e-12).all()


def test_storage_layout_and_bf16_debug_values():
    rng = np.random.default_rng(4)
    W = rng.uniform(-1, 1, (3, 256))
    st = L.quantize_pack("int4_asym", W)
    assert st["packed"].shape == (3, 128) and st["scales"].shape == (3 * 2 * 3,)
    sb, z = L.asym_scales_split(st["scales"], 3, 2)
    codes, sb2, z2 = Q.quantize_int4_asym(W)
    assert (sb == sb2).all() and (z == z2).all()
    bits = L.dequant_bf16_bits("int4_asym", st["packed"], st["scales"])
    assert (bits == F.bf16_bits(F.bf16(L.dequant_exact("int4_asym", st["packed"], st["scales"])))).all()


@pytest.mark.parametrize("K", [100, 130])
def test_k_must_be_a_multiple_of_the_group(K):
    with pytest.raises(ValueError):
        Q.quantize_int4_asym(np.zeros((2, K)))
