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
    dqgemm_quantize_act_fp4,
    dqgemm_quantize_act_fp8,
    dqgemm_run,
    dqgemm_run_fp8_static_quantized,
    dqgemm_run_fp8_static_quantized_out,
    dqgemm_run_quantized_out,
    dqgemm_run_static_mlp,
    dqgemm_selftest_timeout,
    dqgemm_set_wait_limit,
    dqgemm_status_string,
    storage_shapes,
)


def _require(t, name, shape=None, dtype=None, nbytes=None, device=None):
    """Checks the library cannot make itself: its entry points take bare
    device pointers, so a tensor of the wrong dtype, shape or layout would be
    read or written out of bounds on the GPU."""
    if not getattr(t, "is_cuda", False):
        raise ValueError(f"{name} must be a CUDA tensor")
    if device is not None and t.device != device:
        raise ValueError(f"{name} is on {t.device}, expected {device}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")
    if nbytes is not None and t.numel() * t.element_size() != nbytes:
        raise ValueError(f"{name} must hold {nbytes} bytes, got {t.numel() * t.element_size()}")


def _fits(t, cols, dtype, rows=None, dev=None):
    """Fast form of the _require checks for a 2-D operand [rows, cols]: True
    exactly when _require(t, shape=(rows, cols), dtype, device) would pass,
    `dev` being that device's index (an integer compare: building the
    operand's torch.device on every call costs more than the rest)."""
    try:
        return (t.dtype is dtype and t.is_cuda and t.dim() == 2 and t.shape[1] == cols
                and (rows is None or t.shape[0] == rows) and t.is_contiguous()
                and (dev is None or t.get_device() == dev))
    except AttributeError:
        return False


_torch_mod = None


def _torch():
    """torch, imported on first use (the package itself does not need it)."""
    global _torch_mod
    if _torch_mod is None:
        import torch

        _torch_mod = torch
    return _torch_mod


def _storage_bytes(fmt, K, N):
    ps, pd, ss, sd = storage_shapes(fmt, K, N)
    return (int(_np.prod(ps)) * _np.dtype(pd).itemsize, int(_np.prod(ss)) * _np.dtype(sd).itemsize)


def static_mlp(l1, l2, x, out=None, h_out=None, stream=None):
    """The static-FP8 two-layer model y = l2(l1(x)) in one launch
    (dqgemm_run_static_mlp): l1, l2 are "fp8_static" QuantizedLinear layers
    with l2.K == l1.N, l1.N in {256, 512, 1024}, l2.N <= 128; x bf16
    [M, l1.K] on their device.  Returns y (``out``, allocated if None);
    ``h_out`` (bf16 [M, l1.N]) receives layer 1's output if given."""
    torch = _torch()
    if l1.fmt != "fp8_static" or l2.fmt != "fp8_static":
        raise ValueError("static_mlp needs two fp8_static layers")
    if l2.K != l1.N:
        raise ValueError(f"layer 2 takes {l2.K} inputs, layer 1 gives {l1.N}")
    if l2._dev != l1._dev:
        raise ValueError("both layers must live on the same device")
    M = l1._check_x(x, torch.bfloat16)
    out = l2._out(out, M, torch.bfloat16)
    if h_out is not None:
        _require(h_out, "h_out", shape=(M, l1.N), dtype=torch.bfloat16, device=l1.device)
    if M == 0:
        return out
    dqgemm_run_static_mlp(l1.handle, l2.handle, x, M, h_out, out, stream)
    return out


class QuantizedLinear:
    """One quantized Linear layer on the current CUDA device.

    ``packed`` / ``scales`` are CUDA tensors in the canonical layout of
    ``fmt`` (see ``storage_shapes``); they are copied and re-laid-out by the
    library, so the caller may drop them afterwards."""

    # static FP8 from this many rows on: quantize x once, then the FP8 GEMM
    # (the fused kernel re-quantizes x for every 128-channel tile) ...
    STATIC_PREQUANT_M = 128
    # ... and from this many when the output tiles fill more than half the
    # SMs in one wave: the GEMM on codes then takes the 128-row tile, one CTA
    # per SM over the whole K range, which the fused kernel does not (at
    # 4096 x 14336: 19.6 against 33.6 us at 32 rows; up to 16 rows the fused
    # 16-row tile is faster, 23.2 against 25.5)
    STATIC_PREQUANT_M_WIDE = 17

    def __init__(self, fmt, K, N, packed, scales, global_scale=1.0, bias=None):
        import torch

        self._h = None
        if fmt not in FORMATS:
            raise ValueError(f"unknown format {fmt!r}; one of {tuple(FORMATS)}")
        pb, sb = _storage_bytes(fmt, K, N)
        _require(packed, "packed", nbytes=pb)
        _require(scales, "scales", nbytes=sb, device=packed.device)
        if bias is not None:
            _require(bias, "bias", shape=(N,), dtype=torch.bfloat16, device=packed.device)
        self.fmt, self.K, self.N = fmt, K, N
        sms = torch.cuda.get_device_properties(packed.device).multi_processor_count
        n_tiles = (N + 127) // 128
        self._static_prequant_m = (self.STATIC_PREQUANT_M_WIDE if 2 * n_tiles > sms and n_tiles <= sms
                                   else self.STATIC_PREQUANT_M)
        self.device = packed.device               # the handle belongs to this device
        self._dev = self.device.index
        # with one visible GPU the current device can only be this one
        self._check_current = torch.cuda.device_count() > 1
        self.act_scale = float(global_scale) if fmt == "fp8_static" else None
        self._h = dqgemm_create(fmt, K, N, packed, scales, global_scale, bias)

    @classmethod
    def from_float(cls, fmt, W, bias=None, act_scale=None):
        """Quantize a CUDA fp32 weight [N, K] with the GPU packer and build the
        layer.  ``act_scale`` is the static-FP8 per-tensor activation scale."""
        import torch

        if not getattr(W, "is_cuda", False) or W.dim() != 2:
            raise ValueError("W must be a 2-D CUDA tensor [N, K]")
        W = W.detach().to(torch.float32).contiguous()
        N, K = W.shape
        ps, pd, ss, sd = storage_shapes(fmt, K, N)
        tdt = {_np.uint8: torch.uint8, _np.uint16: torch.int16, _np.float32: torch.float32}
        packed = torch.empty(ps, dtype=tdt[pd], device=W.device)
        scales = torch.empty(ss, dtype=tdt[sd], device=W.device)
        g = dqgemm_pack_device("fp8" if fmt == "fp8_static" else fmt, W, packed, scales)
        if fmt == "fp8_static":
            g = act_scale
        return cls(fmt, K, N, packed, scales, g, bias)

    def _check_x(self, x, dtype, name="x"):
        if not _fits(x, self.K, dtype, dev=self._dev):
            if getattr(x, "dim", lambda: 0)() != 2:
                raise ValueError(f"{name} must be 2-D [M, {self.K}]")
            _require(x, name, shape=(x.shape[0], self.K), dtype=dtype, device=self.device)
        if self._check_current:
            if _torch().cuda.current_device() != self._dev:
                raise ValueError(f"the layer lives on {self.device}; make it the current device "
                                 f"(torch.cuda.set_device / torch.cuda.device) before calling it")
        return x.shape[0]

    def _out(self, out, M, dtype):
        if out is None:
            return _torch().empty((M, self.N), dtype=dtype, device=self.device)
        if not _fits(out, self.N, dtype, M, self._dev):
            _require(out, "out", shape=(M, self.N), dtype=dtype, device=self.device)
        return out

    def __call__(self, x, out=None, stream=None):
        """y = x . deq(W)^T + b; x bf16 [M, K] contiguous on CUDA, y (``out``,
        allocated if None) bf16 [M, N]."""
        torch = _torch()
        M = self._check_x(x, torch.bfloat16)
        out = self._out(out, M, torch.bfloat16)
        if M == 0:
            return out
        if self.fmt == "fp8_static" and M >= self._static_prequant_m:
            q = torch.empty((M, self.K), dtype=torch.uint8, device=self.device)
            dqgemm_quantize_act_fp8(x, M, self.K, self.act_scale, q, stream)
            dqgemm_run_fp8_static_quantized(self._h, q, M, out, stream)
        else:
            # (operands checked above: their pointers go straight to the entry)
            _native.run_ptrs(self._h, x.data_ptr(), M, out.data_ptr(), stream)
        return out

    def quantized_out(self, x, s_out, out=None, stream=None):
        """The layer with its result leaving as the next static-FP8 layer's
        e4m3 codes, e4m3(f32(y) / s_out) (uint8 [M, N]); x as for __call__."""
        torch = _torch()
        M = self._check_x(x, torch.bfloat16)
        out = self._out(out, M, torch.uint8)
        if M == 0:
            return out
        if self.fmt == "fp8_static" and M >= self._static_prequant_m:
            q = torch.empty((M, self.K), dtype=torch.uint8, device=self.device)
            dqgemm_quantize_act_fp8(x, M, self.K, self.act_scale, q, stream)
            dqgemm_run_fp8_static_quantized_out(self._h, q, M, out, s_out, stream)
        else:
            dqgemm_run_quantized_out(self._h, x, M, out, s_out, stream)
        return out

    def from_codes(self, q, out=None, stream=None):
        """Static FP8 only: the layer on activations already quantized with
        its own scale (uint8 e4m3 codes [M, K], e.g. from quantized_out)."""
        import torch

        if self.fmt != "fp8_static":
            raise ValueError("from_codes needs a static FP8 layer")
        M = self._check_x(q, torch.uint8, "q")
        out = self._out(out, M, torch.bfloat16)
        if M == 0:
            return out
        dqgemm_run_fp8_static_quantized(self._h, q, M, out, stream)
        return out

    def dequantize(self, stream=None):
        import torch

        w = torch.empty((self.N, self.K), dtype=torch.bfloat16, device=self.device)
        dqgemm_dequantize(self._h, w, stream)
        return w

    def plan(self, M):
        return dqgemm_get_plan(self._h, M)

    def last_error(self):
        return dqgemm_last_error(self._h)

    @property
    def handle(self):
        return self._h

    # the object owns a library handle (device memory freed by close), so a
    # copy would destroy it twice and a pickle would carry a dead pointer
    def __copy__(self):
        raise TypeError("QuantizedLinear owns a device handle and cannot be copied; build another layer")

    def __deepcopy__(self, memo):
        self.__copy__()

    def __reduce__(self):
        raise TypeError("QuantizedLinear owns a device handle and cannot be pickled")

    def close(self):
        if self._h is not None:
            dqgemm_destroy(self._h)
            self._h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass
