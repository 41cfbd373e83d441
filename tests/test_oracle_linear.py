"""Pins of the oracle's GEMM reference and static-FP8 path: special cases that
reduce to a plain matmul, checked against an exact triple loop, and the
per-channel/per-tensor scale algebra on hand-sized inputs."""

import numpy as np

from oracle import formats as F
from oracle import linear as L
from oracle import quant as Q


def _triple_loop(x, w, b):
    M, K = x.shape
    N = w.shape[0]
    y = np.zeros((M, N))
    for m in range(M):
        for n in range(N):
            acc = 0.0
            for k in range(K):
                acc += float(x[m, k]) * float(w[n, k])
            y[m, n] = acc + (0.0 if b is None else float(b[n]))
    return y


def test_int4_unit_scales_reduce_to_plain_matmul():
    # integer weights in [-7, 7] with every group holding a +-7: s = 1 exactly,
    # so DQ(W) = W and y = x W^T + b
    rng = np.random.default_rng(0)
    w = rng.integers(-7, 8, (5, 256)).astype(np.float64)
    w[:, ::128] = 7.0
    x = rng.integers(-3, 4, (3, 256)).astype(np.float64) * 0.5
    b = np.array([0.5, -1.0, 2.0, 0.0, 0.25])
    st = L.quantize_pack("int4", w)
    assert (F.bf16_from_bits(st["scales"]) == 1.0).all()
    wd = L.dequant_exact("int4", st["packed"], st["scales"])
    assert np.array_equal(wd, w)
    assert np.array_equal(L.linear_ref(x, wd, b), _triple_loop(x, w, b))


def test_mxfp4_zero_exponent_reduces_to_e2m1_matmul():
    # every block max 6 -> e = 0: DQ(W) = W when W lies on the E2M1 grid
    rng = np.random.default_rng(1)
    grid = np.array([0, .5, 1, 1.5, 2, 3, 4, 6, -.5, -1, -1.5, -2, -3, -4, -6])
    w = rng.choice(grid, (4, 64))
    w[:, ::32] = 6.0
    x = rng.normal(size=(2, 64)).astype(np.float32).astype(np.float64)
    st = L.quantize_pack("mxfp4", w)
    assert (st["scales"] == 127).all()
    wd = L.dequant_exact("mxfp4", st["packed"], st["scales"])
    assert np.array_equal(wd, w)
    np.testing.assert_allclose(L.linear_ref(x, wd), _triple_loop(x, w, None), rtol=0, atol=1e-12)


def test_linear_ref_generic_matches_triple_loop():
    rng = np.random.default_rng(2)
    x = rng.normal(size=(3, 32))
    w = rng.normal(size=(4, 32))
    b = rng.normal(size=4)
    np.testing.assert_allclose(L.linear_ref(x, w, b), _triple_loop(x, w, b), rtol=1e-13, atol=1e-13)


def test_static_linear_unit_scales_is_integer_matmul():
    # with s_x = s_w = 1 and x, W on small E4M3 integers the layer is x W^T
    rng = np.random.default_rng(3)
    x = rng.integers(-8, 9, (2, 32)).astype(np.float64)
    w = rng.integers(-8, 9, (3, 32)).astype(np.float64)
    qx = L.quantize_act_fp8(x, 1.0)
    qw = F.e4m3_encode(w)
    y = L.static_linear(qx, 1.0, qw, np.ones(3))
    assert np.array_equal(y, _triple_loop(x, w, None))


def test_static_linear_scale_algebra():
    # y scales linearly with s_x and with each channel's s_w
    rng = np.random.default_rng(4)
    qx = F.e4m3_encode(F.e4m3_round(rng.normal(0, 30, (2, 16))))
    qw = F.e4m3_encode(F.e4m3_round(rng.normal(0, 30, (3, 16))))
    base = L.static_linear(qx, 1.0, qw, np.ones(3))
    y = L.static_linear(qx, 0.25, qw, np.array([1.0, 2.0, 0.5]))
    assert np.array_equal(y, base * 0.25 * np.array([1.0, 2.0, 0.5])[None, :])


def test_static_weight_scale_uses_symmetric_range():
    w = np.array([[-3.0, 1.0, 2.0, 0.0] * 4, [0.5, -0.25, 0.125, 0.0] * 4])
    codes, s = Q.quantize_fp8_rows(w)
    assert s.tolist() == [float(F.f32(3.0 / 448)), float(F.f32(0.5 / 448))]


def test_calibration_uses_min_max_over_all_batches():
    w1 = np.eye(4)
    batches = [np.array([[1.0, -2.0, 0.5, 0.0]]), np.array([[0.0, 3.5, -1.0, 0.0]])]
    s1, s2 = L.calibrate_static_mlp(batches, w1, np.eye(4))
    assert s1 == float(F.f32(3.5 / 448)) and s2 == float(F.f32(3.5 / 448))


def test_sqnr_limits():
    a = np.array([3.0, 4.0])
    assert np.isclose(L.sqnr(a, a), 20 * np.log10(5.0 / 1e-12))
    assert np.isclose(L.sqnr(a, np.zeros(2)), 0.0)


def test_calibration_invariants():
    # order of the batches does not matter, an extra batch never lowers a
    # scale, and scaling every batch by 2^j scales both scales by exactly 2^j
    rng = np.random.default_rng(5)
    w1 = rng.uniform(-0.1, 0.1, (16, 8))
    w2 = rng.uniform(-0.1, 0.1, (4, 16))
    batches = [F.bf16(rng.standard_normal((3, 8)) * (1 + i)) for i in range(5)]
    s = L.calibrate_static_mlp(batches, w1, w2)
    assert L.calibrate_static_mlp(batches[::-1], w1, w2) == s
    s4 = L.calibrate_static_mlp(batches[:4], w1, w2)
    assert s4[0] <= s[0] and s4[1] <= s[1]
    for j in (-4, 3):
        sj = L.calibrate_static_mlp([b * 2.0 ** j for b in batches], w1, w2)
        assert sj == (s[0] * 2.0 ** j, s[1] * 2.0 ** j)


def test_calibration_layer2_sees_bf16_output_and_negative_side():
    # layer 1's output is observed after rounding to bf16: 1 + 2^-10 is not a
    # bf16 value and rounds to 1; the negative side dominates the range here
    x = np.array([[1.0, 0.0], [0.0, -5.0]])
    w1 = np.array([[1.0 + 2.0 ** -10, 0.0]])
    s1, s2 = L.calibrate_static_mlp([x], w1, np.eye(1))
    assert s1 == float(F.f32(5.0 / 448))
    assert s2 == float(F.f32(1.0 / 448))


def test_sqnr_closed_form():
    # b = a (1 + eps) gives |a| / |a - b| = 1 / eps exactly: 20 log10(1 / eps) dB
    a = np.random.default_rng(9).standard_normal(1000)
    for k in (3, 10, 20):
        assert np.isclose(L.sqnr(a, a * (1 + 2.0 ** -k)), 20 * k * np.log10(2.0), rtol=1e-9)


def test_static_mlp_hand_worked_two_layers():
    """The static page's two-layer model after Q/DQ, worked by hand on a
    1 x 2 -> 2 -> 1 case whose numbers force every step to matter.
      layer 1: s_x1 = 1/16, x = [1/8, -3/8]  -> codes [2, -6]
               W1 codes [[1, 1/2], [-2, 1]]  -> sums [2 - 3, -4 - 6] = [-1, -10]
               s_w1 = [f32(545.6), 128]      -> h = bf16([-34.0999985, -80]) = [-34, -80]
      layer 2: s_x2 = 1/4  -> h / s_x2 = [-136, -320]; -136 lies halfway
               between the e4m3 points 128 and 144 and rounds to the even
               mantissa, 128, so the codes are [-128, -320]
               W2 codes [[3, -3/2]], s_w2 = [2] -> sum 96 -> y = 96 * 1/4 * 2 = 48
    Each plausible slip gives another y: without the bf16 rounding of h,
    -34.0999985 / (1/4) rounds to -144 and y = 24; with layer 1's scale in
    layer 2, h / (1/16) saturates at -448 twice and y = -84; without the
    layer-2 Q node y = 36; with W1 transposed the layer-1 sums are [14, -5]."""
    e4m3 = {1.0: 0x38, 0.5: 0x30, -2.0: 0xC0, 3.0: 0x44, -1.5: 0xBC}   # OCP E4M3 bit patterns
    q_w1 = np.array([[e4m3[1.0], e4m3[0.5]], [e4m3[-2.0], e4m3[1.0]]], dtype=np.uint8)
    q_w2 = np.array([[e4m3[3.0], e4m3[-1.5]]], dtype=np.uint8)
    s_w1 = np.array([545.6, 128.0], dtype=np.float32)
    s_w2 = np.array([2.0], dtype=np.float32)
    x = np.array([[0.125, -0.375]])
    h, y = L.static_mlp(x, 0.0625, q_w1, s_w1, 0.25, q_w2, s_w2)
    assert h.tolist() == [[-34.0, -80.0]]
    assert y.tolist() == [[48.0]]
