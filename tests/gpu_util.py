"""Helpers shared by the GPU parity tests: upload oracle-made storage, run the
library through its C ABI, and compare against the fp64 oracle with the
tolerances of the quantized-Linear parity contract."""

import numpy as np
import torch

import weight_only_quantized_prologue_b200 as dq
from oracle import formats as F
from oracle import linear as L

# element-wise |y - y_ref| <= ATOL_SCALE * ||x_m|| * ||w_n||, and the relative
# Frobenius error <= REL_FRO (bf16 output rounding alone gives ~1e-3)
ATOL_SCALE = 2e-2
REL_FRO = 5e-3


def dev(a, dtype=None):
    t = torch.from_numpy(np.ascontiguousarray(a))
    if dtype is not None:
        t = t.view(dtype)
    return t.cuda()


def scales_tensor(fmt, scales):
    s = np.ascontiguousarray(scales)
    if fmt == "int4":
        return dev(s.astype(np.uint16).view(np.int16))
    if fmt in ("fp8", "fp8_static"):
        return dev(s.astype(np.float32))
    return dev(s.astype(np.uint8))


def bf16_values(t):
    """fp64 numpy values of a bf16 torch tensor."""
    return t.float().cpu().numpy().astype(np.float64)


def base_fmt(fmt):
    """The oracle's storage format of a library format."""
    return {"fp8_static": "fp8", "w4a4_mxfp4": "mxfp4", "w4a4_nvfp4": "nvfp4"}.get(fmt, fmt)


def make_layer(fmt, W, bias_t=None, act_scale=None):
    """Quantize W (fp64 numpy of fp32 values) with the oracle and build a
    handle from that storage.  Returns (handle, storage dict, exact DQ)."""
    st = L.quantize_pack(base_fmt(fmt), W)
    g = act_scale if fmt == "fp8_static" else st["global_scale"]
    N, K = W.shape
    h = dq.dqgemm_create(fmt, K, N, dev(st["packed"]), scales_tensor(fmt, st["scales"]), g, bias_t)
    wdq = L.dequant_exact(base_fmt(fmt), st["packed"], st["scales"], st["global_scale"])
    return h, st, wdq


def w4a4_effective_x(fmt, x):
    """The activation values an FP4 x FP4 layer multiplies: the oracle's
    dynamic quantization of x (its bf16 values), dequantized exactly."""
    if fmt == "w4a4_mxfp4":
        c, s = L.quantize_act_mxfp4(x)
        return F.e2m1_decode(c) * np.repeat(F.e8m0_decode(s), 32, axis=1)
    c, s, g = L.quantize_act_nvfp4(x)
    return F.e2m1_decode(c) * np.repeat(F.e4m3_decode(s), 16, axis=1) * float(g)


def run(h, x_t, N):
    M = x_t.shape[0]
    y = torch.full((M, N), float("nan"), dtype=torch.bfloat16, device="cuda")
    dq.dqgemm_run(h, x_t, M, y)
    torch.cuda.synchronize()
    assert dq.dqgemm_last_error(h) == 0
    return y


def check_close(y, y_ref, x_eff, wdq, rows=None):
    """y (fp64 numpy), y_ref (fp64), x_eff the activation values the layer
    multiplies (rows of y), wdq the exact weight."""
    err = np.abs(y - y_ref)
    bound = ATOL_SCALE * np.linalg.norm(x_eff, axis=1)[:, None] * np.linalg.norm(wdq, axis=1)[None, :]
    bad = ~(err <= bound + 1e-30)
    assert not bad.any(), f"{bad.sum()} elements over the bound, max err {err.max():.3g}"
    rel = np.linalg.norm(y - y_ref) / max(np.linalg.norm(y_ref), 1e-30)
    assert rel <= REL_FRO, f"relative Frobenius error {rel:.3g}"
    return rel


def static_effective_x(x, s_x):
    return F.e4m3_decode(L.quantize_act_fp8(x, s_x)) * s_x
