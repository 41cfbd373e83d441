"""nn.Linear drop-in over libdqgemm: a torch custom op and an nn.Module.

The quantized-Linear pages all start from a plain bf16 ``nn.Linear`` model and
quantize it in place before use ("Define a linear model and quantize
weights to ..." on each page); ``quantize_`` does the same with this
library's layers.  Static FP8 needs a per-tensor activation scale for every
layer input, taken from min/max observers over calibration runs of the float
model ("TorchAO Static FP8 Quantization (Linear)", "Define a small two-layer
Linear model"): ``calibrate_static_fp8`` records them.

The op ``dqgemm::linear`` takes the layer's handle as an integer and has a
fake (shape-only) implementation, so modules that use it can be traced; the
real implementation is one ``dqgemm_run`` (or the quantize + FP8 GEMM pair of
static FP8 from 128 rows on) on the current stream.  Nothing here computes:
without ``libdqgemm.so`` the calls raise.
"""

import torch

from . import QuantizedLinear

FORMATS = ("int4", "nvfp4", "mxfp4", "fp8", "fp8_static", "int4_asym", "w4a4_mxfp4", "w4a4_nvfp4")

# live layers by handle value, so the op can reach the Python object (the
# static-FP8 path needs its activation scale and K)
_LAYERS = {}


@torch.library.custom_op("dqgemm::linear", mutates_args=())
def dq_linear(x: torch.Tensor, handle: int, n_out: int) -> torch.Tensor:
    """y = x . deq(W)^T + b for the layer whose handle is `handle`; x is
    bf16 [M, K] contiguous on CUDA, y bf16 [M, n_out]."""
    layer = _LAYERS[handle]
    return layer(x)


@dq_linear.register_fake
def _(x, handle, n_out):
    return x.new_empty((x.shape[0], n_out))


class DQLinear(torch.nn.Module):
    """A quantized ``nn.Linear``: same call contract (any leading dims, last
    dim = in_features), bf16 activations and outputs."""

    def __init__(self, layer: QuantizedLinear):
        super().__init__()
        self.layer = layer
        self.in_features, self.out_features, self.fmt = layer.K, layer.N, layer.fmt
        _LAYERS[self._handle()] = layer

    def _handle(self):
        return int(self.layer.handle.value)

    @classmethod
    def from_linear(cls, linear: torch.nn.Linear, fmt: str, act_scale=None):
        if fmt not in FORMATS:
            raise ValueError(f"unknown format {fmt!r}; one of {FORMATS}")
        if fmt == "fp8_static" and act_scale is None:
            raise ValueError("fp8_static needs the calibrated activation scale (calibrate_static_fp8)")
        w = linear.weight.detach().to(device="cuda", dtype=torch.float32)
        b = None if linear.bias is None else linear.bias.detach().to(device="cuda", dtype=torch.bfloat16)
        return cls(QuantizedLinear.from_float(fmt, w, b, act_scale=act_scale))

    def forward(self, x):
        lead = x.shape[:-1]
        x2 = x.reshape(-1, self.in_features)
        if x2.dtype != torch.bfloat16 or not x2.is_contiguous():
            x2 = x2.to(torch.bfloat16).contiguous()
        y = torch.ops.dqgemm.linear(x2, self._handle(), self.out_features)
        return y.reshape(*lead, self.out_features)

    def extra_repr(self):
        return f"in_features={self.in_features}, out_features={self.out_features}, format={self.fmt}"

    def __del__(self):
        try:
            _LAYERS.pop(self._handle(), None)
        except Exception:
            pass


def calibrate_static_fp8(model, batches):
    """Per-tensor activation scales max(|min|, |max|) / 448 (fp32) of every
    nn.Linear input, observed over forward passes of the float model on
    `batches`.  Returns {module name: scale}."""
    lo, hi, hooks = {}, {}, []
    for name, mod in model.named_modules():
        if isinstance(mod, torch.nn.Linear):
            def hook(m, inp, name=name):
                t = inp[0].detach()
                lo[name] = min(lo.get(name, 0.0), t.min().item())
                hi[name] = max(hi.get(name, 0.0), t.max().item())
            hooks.append(mod.register_forward_pre_hook(hook))
    try:
        with torch.no_grad():
            for b in batches:
                model(b)
    finally:
        for h in hooks:
            h.remove()
    return {n: float(torch.tensor(max(abs(lo[n]), abs(hi[n])), dtype=torch.float32) / 448.0) for n in lo}


def quantize_(model, fmt, act_scales=None, filter_fn=None):
    """Replace, in place, every nn.Linear of `model` (for which
    ``filter_fn(name, module)`` holds, if given) by a DQLinear of format
    `fmt`.  Static FP8 takes ``act_scales`` from calibrate_static_fp8.
    Returns the model."""
    targets = [(n, m) for n, m in model.named_modules()
               if isinstance(m, torch.nn.Linear) and (filter_fn is None or filter_fn(n, m))]
    for name, mod in targets:
        scale = None if act_scales is None else act_scales[name]
        new = DQLinear.from_linear(mod, fmt, act_scale=scale)
        parent = model
        *path, leaf = name.split(".")
        for p in path:
            parent = getattr(parent, p)
        setattr(parent, leaf, new)
    return model
