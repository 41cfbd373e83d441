"""B200-native quantized nn.Linear with the dequantization in the GEMM prologue.

The compute lives in ``libdqgemm.so`` (hand-written sm_100a CUDA, C ABI in
``include/dqgemm.h``); this package only marshals torch tensors to it.

    from weight_only_quantized_prologue_b200 import QuantizedLinear
    ql = QuantizedLinear.from_float("int4", W_fp32_cuda, bias_bf16_cuda)
    y = ql(x_bf16_cuda)            # y = x . deq(W)^T + b, bf16
"""

import numpy as _np

from . import _native
from ._native import (  # noqa: F401
    FORMATS,
    DQError,
    dqgemm_create,
    dqgemm_dequantize,
    dqgemm_destroy,
    dqgemm_get_plan,
    dqgemm_last_error,
    dqgemm_pack_device,
    dqgemm_pack_device_noalloc,
    dqgemm_pack_host,
    dqgemm_quantize_act_fp8,
    dqgemm_run,
    dqgemm_run_fp8_static_quantized,
    dqgemm_run_fp8_static_quantized_out,
    dqgemm_run_quantized_out,
    dqgemm_selftest_timeout,
    dqgemm_status_string,
    storage_shapes,
)


class QuantizedLinear:
    """One quantized Linear layer on the current CUDA device.

    ``packed`` / ``scales`` are CUDA tensors in the canonical layout of
    ``fmt`` (see ``storage_shapes``); they are copied and re-laid-out by the
    library, so the caller may drop them afterwards."""

    # static FP8 from this many rows on: quantize x once, then the FP8 GEMM
    # (the fused kernel re-quantizes x for every 128-channel tile)
    STATIC_PREQUANT_M = 128

    def __init__(self, fmt, K, N, packed, scales, global_scale=1.0, bias=None):
        self.fmt, self.K, self.N = fmt, K, N
        self.act_scale = float(global_scale) if fmt == "fp8_static" else None
        self._h = dqgemm_create(fmt, K, N, packed, scales, global_scale, bias)

    @classmethod
    def from_float(cls, fmt, W, bias=None, act_scale=None):
        """Quantize a CUDA fp32 weight [N, K] with the GPU packer and build the
        layer.  ``act_scale`` is the static-FP8 per-tensor activation scale."""
        import torch

        N, K = W.shape
        ps, pd, ss, sd = storage_shapes(fmt, K, N)
        tdt = {_np.uint8: torch.uint8, _np.uint16: torch.int16, _np.float32: torch.float32}
        packed = torch.empty(ps, dtype=tdt[pd], device=W.device)
        scales = torch.empty(ss, dtype=tdt[sd], device=W.device)
        g = dqgemm_pack_device("fp8" if fmt == "fp8_static" else fmt, W.contiguous(), packed, scales)
        if fmt == "fp8_static":
            g = act_scale
        return cls(fmt, K, N, packed, scales, g, bias)

    def __call__(self, x, out=None, stream=None):
        import torch

        M = x.shape[0]
        if out is None:
            out = torch.empty((M, self.N), dtype=torch.bfloat16, device=x.device)
        if self.fmt == "fp8_static" and M >= self.STATIC_PREQUANT_M:
            q = torch.empty((M, self.K), dtype=torch.uint8, device=x.device)
            dqgemm_quantize_act_fp8(x, M, self.K, self.act_scale, q, stream)
            dqgemm_run_fp8_static_quantized(self._h, q, M, out, stream)
        else:
            dqgemm_run(self._h, x, M, out, stream)
        return out

    def quantized_out(self, x, s_out, out=None, stream=None):
        """The layer with its result leaving as the next static-FP8 layer's
        e4m3 codes, e4m3(f32(y) / s_out) (uint8 [M, N]); x as for __call__."""
        import torch

        M = x.shape[0]
        if out is None:
            out = torch.empty((M, self.N), dtype=torch.uint8, device=x.device)
        if self.fmt == "fp8_static" and M >= self.STATIC_PREQUANT_M:
            q = torch.empty((M, self.K), dtype=torch.uint8, device=x.device)
            dqgemm_quantize_act_fp8(x, M, self.K, self.act_scale, q, stream)
            dqgemm_run_fp8_static_quantized_out(self._h, q, M, out, s_out, stream)
        else:
            dqgemm_run_quantized_out(self._h, x, M, out, s_out, stream)
        return out

    def from_codes(self, q, out=None, stream=None):
        """Static FP8 only: the layer on activations already quantized with
        its own scale (uint8 e4m3 codes [M, K], e.g. from quantized_out)."""
        import torch

        M = q.shape[0]
        if out is None:
            out = torch.empty((M, self.N), dtype=torch.bfloat16, device=q.device)
        dqgemm_run_fp8_static_quantized(self._h, q, M, out, stream)
        return out

    def dequantize(self, stream=None):
        import torch

        w = torch.empty((self.N, self.K), dtype=torch.bfloat16, device="cuda")
        dqgemm_dequantize(self._h, w, stream)
        return w

    def plan(self, M):
        return dqgemm_get_plan(self._h, M)

    def last_error(self):
        return dqgemm_last_error(self._h)

    @property
    def handle(self):
        return self._h

    def close(self):
        if self._h is not None:
            dqgemm_destroy(self._h)
            self._h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass
