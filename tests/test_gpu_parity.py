"""GPU parity of the C-ABI library against the fp64 oracle.

Bit-exact: the GPU packer's bytes, the debug dequantization's bf16 bit
patterns (through the GEMM prologue's own unpack code) and the static-FP8
activation codes.  Within the stated float tolerance: the GEMM outputs, at
small shapes spanning several tiles with ragged tails and at the pages' full
sizes (M=32, K=3072, N=4096 and the 256->512->128 static-FP8 MLP)."""

import numpy as np
import pytest
import torch

import weight_only_quantized_prologue_b200 as dq
from oracle import formats as F
from oracle import linear as L
from weight_only_quantized_prologue_b200 import synthetic

from gpu_util import (bf16_values, check_close, dev, make_layer, run, scales_tensor, static_effective_x)

pytestmark = pytest.mark.gpu

WO_FORMATS = ["int4", "nvfp4", "mxfp4", "fp8", "int4_asym"]
ALL_FORMATS = WO_FORMATS + ["fp8_static"]


def _inputs(M, K, N, seed=0, bias=True):
    x, w, b = synthetic.linear_inputs(M, K, N, seed=seed, bias=bias)
    return x, w.numpy().astype(np.float64), b


def _wide_weights(N, K, seed, span):
    rng = np.random.default_rng(seed)
    W = rng.normal(size=(N, K)) * np.exp2(rng.integers(-span, span // 4 + 1, (N, K)))
    W[rng.random((N, K)) < 0.05] = 0.0
    W[0] = 0.0
    return W.astype(np.float32).astype(np.float64)


# -- packer ----------------------------------------------------------------


@pytest.mark.parametrize("fmt", WO_FORMATS)
@pytest.mark.parametrize("N,K", [(256, 512), (96, 3072)])
def test_pack_device_bit_identical_to_oracle(fmt, N, K):
    W = _wide_weights(N, K, seed=1, span=24)
    ref = L.quantize_pack(fmt, W)
    packed = torch.zeros(ref["packed"].shape, dtype=torch.uint8, device="cuda")
    st = scales_tensor(fmt, np.zeros_like(ref["scales"]))
    g = dq.dqgemm_pack_device(fmt, dev(W.astype(np.float32)), packed, st)
    torch.cuda.synchronize()
    assert np.array_equal(packed.cpu().numpy(), ref["packed"])
    assert np.array_equal(st.cpu().numpy().view(np.uint8),
                          np.ascontiguousarray(ref["scales"]).astype(st.cpu().numpy().dtype).view(np.uint8))
    assert np.float32(g) == np.float32(ref["global_scale"])


# -- debug dequantization (the prologue's unpack, bit-exact) -----------------


@pytest.mark.parametrize("fmt", ALL_FORMATS)
@pytest.mark.parametrize("N,K,kind", [(256, 512, "uniform"), (200, 272, "uniform"), (384, 1024, "wide")])
def test_dequantize_bit_exact(fmt, N, K, kind):
    if fmt in ("nvfp4", "mxfp4") and N % 32:
        N = 224
    if fmt in ("int4", "int4_asym") and K % 128:
        K = 384
    if fmt == "mxfp4" and K % 32:
        K = 288
    W = _wide_weights(N, K, seed=2, span=20) if kind == "wide" else _inputs(1, K, N)[1]
    h, st, _ = make_layer(fmt, W, act_scale=0.5)
    try:
        out = torch.empty((N, K), dtype=torch.bfloat16, device="cuda")
        dq.dqgemm_dequantize(h, out)
        torch.cuda.synchronize()
        got = out.view(torch.int16).cpu().numpy().view(np.uint16)
        ref = L.dequant_bf16_bits("fp8" if fmt == "fp8_static" else fmt, st["packed"], st["scales"],
                                  st["global_scale"])
        mism = np.argwhere(got != ref)
        assert mism.size == 0, f"{len(mism)} mismatches, first {mism[:3].tolist()}"
    finally:
        dq.dqgemm_destroy(h)


# -- static FP8 activation quantization (bit-exact) --------------------------


def test_quantize_act_fp8_bit_exact():
    rng = np.random.default_rng(5)
    x = torch.from_numpy(rng.normal(0, 3, (37, 272)).astype(np.float32)).to(torch.bfloat16)
    x[0, :8] = torch.tensor([1e4, -1e4, 0.0, -0.0, 1e-6, -1e-6, 3.0, -448.0])
    s_x = float(np.float32(0.0123))
    q = torch.empty(x.shape, dtype=torch.uint8, device="cuda")
    dq.dqgemm_quantize_act_fp8(x.cuda(), x.shape[0], x.shape[1], s_x, q)
    torch.cuda.synchronize()
    ref = L.quantize_act_fp8(bf16_values(x), s_x)
    assert np.array_equal(q.cpu().numpy(), ref)


def _all_finite_bf16():
    """Every finite bf16 bit pattern (65,024 of the 65,536; NaN and inf
    patterns become zeros), as a [256, 256] tensor."""
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    finite = (bits & 0x7F80) != 0x7F80
    bits = np.where(finite, bits, 0).astype(np.uint16)
    return torch.from_numpy(bits.view(np.int16).reshape(256, 256).copy()).view(torch.bfloat16)


@pytest.mark.parametrize("s_x", [0.0123, 3.0, 1.0 / 3.0, 7.77e-6, 2.5e4, 1.0e-30, 0.1])
def test_quantize_act_fp8_every_bf16_value(s_x):
    # the quantizer forms f32(x / s_x) without dividing (a multiply by the
    # reciprocal and one correction step); its codes must equal those of the
    # exact quotient for every bf16 input, both kernels (vector, and
    # element-wise through an unaligned buffer)
    s_x = float(np.float32(s_x))
    x = _all_finite_bf16()
    ref = L.quantize_act_fp8(bf16_values(x), s_x)
    q = torch.empty((256, 256), dtype=torch.uint8, device="cuda")
    dq.dqgemm_quantize_act_fp8(x.cuda(), 256, 256, s_x, q)
    xe = torch.zeros(65537, dtype=torch.bfloat16, device="cuda")
    xe[1:] = x.view(-1).cuda()
    qe = torch.zeros(65537, dtype=torch.uint8, device="cuda")
    assert dq._native.lib().dqgemm_quantize_act_fp8(xe.data_ptr() + 2, 256, 256, s_x, qe.data_ptr() + 1, None) == 0
    torch.cuda.synchronize()
    got = q.cpu().numpy()
    bad = np.argwhere(got != ref)
    assert bad.size == 0, (f"{len(bad)} codes differ, e.g. x bits {x.view(torch.int16)[tuple(bad[0])].item() & 0xFFFF:#06x}: "
                           f"{got[tuple(bad[0])]:#04x} vs {ref[tuple(bad[0])]:#04x}")
    assert np.array_equal(qe.cpu().numpy()[1:].reshape(256, 256), ref)


@pytest.mark.parametrize("M,K,offset", [(5, 19, 0), (129, 4096, 0), (3, 272, 1), (64, 1000, 3)])
def test_quantize_act_fp8_vector_tail_and_unaligned(M, K, offset):
    # 16 elements per thread where x and q are 16-byte aligned, element-wise
    # for the tail (M*K not a multiple of 16) and for unaligned buffers
    rng = np.random.default_rng(M + K)
    x = torch.from_numpy(rng.normal(0, 5, (M, K)).astype(np.float32)).to(torch.bfloat16)
    x.view(-1)[::97] = 0.0
    x.view(-1)[1::89] = -0.0
    s_x = float(np.float32(0.0371))
    xb = torch.zeros(M * K + 8, dtype=torch.bfloat16, device="cuda")
    xb[offset:offset + M * K] = x.view(-1).cuda()
    qb = torch.full((M * K + 16,), 0xEE, dtype=torch.uint8, device="cuda")
    lib = dq._native.lib()
    st = lib.dqgemm_quantize_act_fp8(xb.data_ptr() + 2 * offset, M, K, s_x, qb.data_ptr() + offset, None)
    assert st == 0
    torch.cuda.synchronize()
    got = qb.cpu().numpy()
    assert np.array_equal(got[offset:offset + M * K], L.quantize_act_fp8(bf16_values(x), s_x).reshape(-1))
    assert (got[:offset] == 0xEE).all() and (got[offset + M * K:] == 0xEE).all()


# -- GEMM parity -----------------------------------------------------------

SHAPES = [(1, 256, 128), (3, 384, 256), (17, 512, 384), (33, 1024, 640), (64, 256, 1152),
          (100, 768, 256), (129, 512, 256), (256, 640, 384)]


@pytest.mark.parametrize("fmt", ALL_FORMATS)
@pytest.mark.parametrize("M,K,N", SHAPES)
def test_gemm_matches_oracle(fmt, M, K, N):
    x, W, b = _inputs(M, K, N, seed=M + K + N)
    s_x = L.act_scale(bf16_values(x).min(), bf16_values(x).max())
    h, st, wdq = make_layer(fmt, W, b.cuda(), act_scale=s_x)
    try:
        y = bf16_values(run(h, x.cuda(), N))
        xv = bf16_values(x)
        x_eff = static_effective_x(xv, s_x) if fmt == "fp8_static" else xv
        check_close(y, L.linear_ref(x_eff, wdq, bf16_values(b)), x_eff, wdq)
    finally:
        dq.dqgemm_destroy(h)


@pytest.mark.parametrize("fmt,K,N", [("int4", 384, 200), ("int4_asym", 640, 136), ("fp8", 400, 136), ("nvfp4", 272, 176),
                                     ("mxfp4", 288, 160), ("fp8_static", 208, 72)])
@pytest.mark.parametrize("M", [5, 40])
def test_gemm_ragged_k_and_n(fmt, K, N, M):
    x, W, b = _inputs(M, K, N, seed=11)
    s_x = L.act_scale(bf16_values(x).min(), bf16_values(x).max())
    h, st, wdq = make_layer(fmt, W, b.cuda(), act_scale=s_x)
    try:
        y = bf16_values(run(h, x.cuda(), N))
        xv = bf16_values(x)
        x_eff = static_effective_x(xv, s_x) if fmt == "fp8_static" else xv
        check_close(y, L.linear_ref(x_eff, wdq, bf16_values(b)), x_eff, wdq)
    finally:
        dq.dqgemm_destroy(h)


@pytest.mark.parametrize("fmt", WO_FORMATS)
def test_gemm_full_size_pages_linear(fmt):
    """The pages' nn.Linear(3072, 4096) with x = randn(32, 3072), every output."""
    x, W, b = _inputs(32, 3072, 4096, seed=0)
    h, st, wdq = make_layer(fmt, W, b.cuda())
    try:
        y1 = run(h, x.cuda(), 4096)
        y2 = run(h, x.cuda(), 4096)
        assert torch.equal(y1.view(torch.int16), y2.view(torch.int16))      # deterministic
        xv = bf16_values(x)
        check_close(bf16_values(y1), L.linear_ref(xv, wdq, bf16_values(b)), xv, wdq)
    finally:
        dq.dqgemm_destroy(h)


def test_static_fp8_two_layer_mlp():
    """The static-FP8 page's 256 -> 512 -> 128 model, scales calibrated on ten
    seeded batches, both layers through the library."""
    w1, w2 = synthetic.mlp_weights(seed=0)
    w1v, w2v = bf16_values(w1), bf16_values(w2)
    cal = [bf16_values(synthetic.activations(32, 256, seed=s)) for s in range(1, 11)]
    s1, s2 = L.calibrate_static_mlp(cal, w1v, w2v)
    x = synthetic.activations(32, 256, seed=0)
    h1, st1, wdq1 = make_layer("fp8_static", w1v, act_scale=s1)
    h2, st2, wdq2 = make_layer("fp8_static", w2v, act_scale=s2)
    try:
        hid = run(h1, x.cuda(), 512)
        y = run(h2, hid, 128)
        xv = bf16_values(x)
        x1 = static_effective_x(xv, s1)
        check_close(bf16_values(hid), L.linear_ref(x1, wdq1), x1, wdq1)
        # layer 2 is compared on the GPU's own hidden activations (ulp-level
        # differences in h move e4m3 codes, so both sides quantize the same h)
        hv = bf16_values(hid)
        x2 = static_effective_x(hv, s2)
        check_close(bf16_values(y), L.linear_ref(x2, wdq2), x2, wdq2)
        q = torch.empty((32, 512), dtype=torch.uint8, device="cuda")
        dq.dqgemm_quantize_act_fp8(hid, 32, 512, s2, q)
        torch.cuda.synchronize()
        assert np.array_equal(q.cpu().numpy(), L.quantize_act_fp8(hv, s2))
        # and the whole model stays close to the oracle's own end-to-end run
        _, y_ref = L.static_mlp(xv, s1, st1["packed"], st1["scales"], s2, st2["packed"], st2["scales"])
        assert L.sqnr(y_ref, bf16_values(y)) > 30.0
    finally:
        dq.dqgemm_destroy(h1)
        dq.dqgemm_destroy(h2)


# -- bounded waits -----------------------------------------------------------


def test_bounded_wait_times_out_and_context_survives():
    assert dq.dqgemm_selftest_timeout(20000) == dq._native.DQ_ERR_TIMEOUT
    x, W, b = _inputs(8, 256, 128, seed=3)
    h, st, wdq = make_layer("int4", W, b.cuda())
    try:
        y = bf16_values(run(h, x.cuda(), 128))
        xv = bf16_values(x)
        check_close(y, L.linear_ref(xv, wdq, bf16_values(b)), xv, wdq)
    finally:
        dq.dqgemm_destroy(h)


def test_run_rejects_bad_arguments_on_gpu():
    x, W, b = _inputs(4, 256, 128)
    h, _, _ = make_layer("int4", W)
    try:
        xt = x.cuda()
        y = torch.empty((4, 128), dtype=torch.bfloat16, device="cuda")
        lib = dq._native.lib()
        assert lib.dqgemm_run(h, xt.data_ptr(), 0, y.data_ptr(), None) == dq._native.DQ_ERR_INVALID_ARG
        assert lib.dqgemm_run(h, xt.data_ptr() + 2, 4, y.data_ptr(), None) == dq._native.DQ_ERR_ALIGNMENT
    finally:
        dq.dqgemm_destroy(h)
