"""Pins of the oracle's number formats against things other than the oracle:
hand-written closed-form values, brute-force nearest-point search and torch's
own dtype casts (a library routine independent of the oracle)."""

import json
import os

import numpy as np
import pytest
import torch

from oracle import formats as F


@pytest.fixture(scope="module")
def golden(golden_dir):
    with open(os.path.join(golden_dir, "format_values.json")) as f:
        return json.load(f)


# -- decoders against closed forms / torch ----------------------------------


def test_e2m1_decode_matches_golden_table(golden):
    mags = golden["e2m1"]["magnitude_by_code"]
    for code in range(16):
        want = mags[code & 7] * (-1.0 if code & golden["e2m1"]["sign_bit"] else 1.0)
        got = float(F.e2m1_decode(code))
        assert got == want and np.signbit(got) == bool(code & 8), code


def test_e4m3_decode_all_codes_match_torch(golden):
    codes = np.arange(256)
    ours = F.e4m3_decode(codes)
    ref = torch.arange(256, dtype=torch.uint8).view(torch.float8_e4m3fn).double().numpy()
    nan = np.isnan(ref)
    assert list(np.nonzero(nan)[0]) == golden["e4m3"]["nan_codes"]
    assert np.array_equal(np.isnan(ours), nan)
    assert np.array_equal(ours[~nan], ref[~nan])
    assert np.array_equal(np.signbit(ours[~nan]), np.signbit(ref[~nan]))
    g = golden["e4m3"]
    assert F.e4m3_decode(g["max_code"]) == g["max"] == np.nanmax(ours)
    assert F.e4m3_decode(g["one_code"]) == 1.0
    assert F.e4m3_decode(g["min_normal_code"]) == g["min_normal"]
    assert F.e4m3_decode(g["min_subnormal_code"]) == g["min_subnormal"]


def test_e8m0_decode_matches_torch_and_golden(golden):
    ours = F.e8m0_decode(np.arange(256))
    ref = torch.arange(256, dtype=torch.uint8).view(torch.float8_e8m0fnu).double().numpy()
    assert np.isnan(ours[255]) and np.isnan(ref[255])
    assert np.array_equal(ours[:255], ref[:255])
    for code, val in golden["e8m0"]["code_value_pairs"]:
        assert F.e8m0_decode(code) == val


# -- encoders: round trip ----------------------------------------------------


def test_e2m1_encode_decode_roundtrip():
    codes = np.arange(16)
    assert np.array_equal(F.e2m1_encode(F.e2m1_decode(codes)), codes)


def test_e4m3_encode_decode_roundtrip_every_non_nan_code():
    codes = np.array([c for c in range(256) if (c & 0x7F) != 0x7F])
    assert np.array_equal(F.e4m3_encode(F.e4m3_decode(codes)), codes)


# -- rounding: brute force over every midpoint --------------------------------


def _grid_from_decoder(values):
    v = np.unique(np.abs(values[~np.isnan(values)]))
    return v


def _brute_round(v, grid_mags, even_of):
    """Nearest point of the signed grid, ties to the point whose significand
    is even; computed by exhaustive search."""
    out = []
    for x in v:
        a = min(abs(x), grid_mags[-1])
        d = np.abs(grid_mags - a)
        best = np.flatnonzero(d == d.min())
        if len(best) == 2:
            best = [b for b in best if even_of(grid_mags[b])]
        out.append(np.copysign(grid_mags[best[0]], x))
    return np.array(out)


def _probe_points(grid):
    mids = (grid[:-1] + grid[1:]) / 2
    pts = np.concatenate([grid, mids, np.nextafter(mids, 0), np.nextafter(mids, np.inf),
                          [grid[-1] * 1.01, grid[-1] * 4]])
    return np.concatenate([pts, -pts])


def test_e2m1_round_equals_brute_force(golden):
    grid = np.array(golden["e2m1"]["magnitude_by_code"])
    # even significand <=> even code (codes enumerate the grid in order)
    even = {float(g): (i % 2 == 0) for i, g in enumerate(grid)}
    pts = _probe_points(grid)
    assert np.array_equal(F.e2m1_round(pts), _brute_round(pts, grid, lambda g: even[float(g)]))


def test_e4m3_round_equals_brute_force():
    ref = torch.arange(128, dtype=torch.uint8).view(torch.float8_e4m3fn).double().numpy()
    grid = ref[:127]                      # codes 0..126 in increasing order
    even = {float(g): (i % 2 == 0) for i, g in enumerate(grid)}
    pts = _probe_points(grid)
    assert np.array_equal(F.e4m3_round(pts), _brute_round(pts, grid, lambda g: even[float(g)]))


def test_e4m3_round_matches_torch_cast_in_range():
    rng = np.random.default_rng(1)
    v = np.concatenate([rng.normal(0, 50, 20000), rng.normal(0, 0.01, 20000)])
    ref = torch.arange(127, dtype=torch.uint8).view(torch.float8_e4m3fn).double().numpy()
    mids = (ref[:-1] + ref[1:]) / 2
    v = np.concatenate([v, mids, -mids]).astype(np.float32).astype(np.float64)
    v = v[np.abs(v) <= 464.0]              # torch's cast is not saturating past this
    ours = F.e4m3_encode(F.e4m3_round(v))
    theirs = torch.from_numpy(v.astype(np.float32)).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(ours, theirs)


def test_e4m3_round_saturates():
    assert F.e4m3_round(1e9) == 448.0 and F.e4m3_round(-470.0) == -448.0
    assert F.e4m3_encode(F.e4m3_round(-1e-30)) == 0x80      # -0 keeps its sign


def test_bf16_matches_torch_cast():
    rng = np.random.default_rng(2)
    bits = rng.integers(0, 2**32, 200000, dtype=np.uint64).astype(np.uint32)
    v = bits.view(np.float32)
    v = v[np.isfinite(v)]
    ties = ((rng.integers(0, 2**16, 5000).astype(np.uint32) << 16) | 0x8000).view(np.float32)
    subn = (rng.integers(0, 2**23, 5000).astype(np.uint32)).view(np.float32)
    v = np.concatenate([v, ties[np.isfinite(ties)], subn, [3.3895e38, -3.3895e38, 0.0, -0.0]])
    v = v.astype(np.float32)
    ours = F.bf16(v.astype(np.float64))
    theirs = torch.from_numpy(v).to(torch.bfloat16).double().numpy()
    assert np.array_equal(np.isinf(ours), np.isinf(theirs))
    fin = np.isfinite(theirs)
    assert np.array_equal(ours[fin], theirs[fin])
    assert np.array_equal(np.signbit(ours), np.signbit(theirs))
    assert np.array_equal(F.bf16_bits(ours[fin]),
                          torch.from_numpy(v[fin]).to(torch.bfloat16).view(torch.int16).numpy().astype(np.uint16))


def test_f32_is_ieee_single_rounding():
    # 1/3 in binary32 is 0x3EAAAAAB (round up), 2/3 is 0x3F2AAAAB
    assert np.float32(F.f32(1.0 / 3.0)).view(np.uint32) == 0x3EAAAAAB
    assert np.float32(F.f32(2.0 / 3.0)).view(np.uint32) == 0x3F2AAAAB
    # a tie at the 24-bit boundary goes to even: 1 + 2**-24 -> 1.0
    assert F.f32(1.0 + 2.0**-24) == 1.0 and F.f32(1.0 + 3 * 2.0**-24) == 1.0 + 2.0**-22
