"""QuantizedLinear rejects tensors the library would read or write out of
bounds, before any call into the library (so these run without a GPU)."""

import pytest
import torch

import weight_only_quantized_prologue_b200 as dq


def _layer(fmt="int4", K=256, N=128):
    # a layer object without a library handle: only the argument checks run
    lin = dq.QuantizedLinear.__new__(dq.QuantizedLinear)
    lin._h, lin.fmt, lin.K, lin.N, lin.act_scale = None, fmt, K, N, None
    lin.device, lin._dev, lin._check_current = torch.device("cuda", 0), 0, False
    return lin


def test_create_rejects_host_tensors_and_wrong_sizes():
    with pytest.raises(ValueError, match="CUDA"):
        dq.QuantizedLinear("int4", 256, 128, torch.zeros(128, 128, dtype=torch.uint8),
                           torch.zeros(128, 2, dtype=torch.int16))
    with pytest.raises(ValueError, match="unknown format"):
        dq.QuantizedLinear("int3", 256, 128, None, None)


def test_from_float_rejects_host_weight():
    with pytest.raises(ValueError, match="CUDA"):
        dq.QuantizedLinear.from_float("int4", torch.zeros(128, 256))


@pytest.mark.parametrize("method", ["__call__", "quantized_out"])
def test_call_rejects_host_x(method):
    lin = _layer()
    x = torch.zeros(4, 256, dtype=torch.bfloat16)
    args = (x,) if method == "__call__" else (x, 1.0)
    with pytest.raises(ValueError, match="CUDA"):
        getattr(lin, method)(*args)


def test_call_rejects_wrong_rank():
    with pytest.raises(ValueError, match="2-D"):
        _layer()(torch.zeros(2, 3, 256, dtype=torch.bfloat16))


def test_from_codes_needs_static_layer():
    with pytest.raises(ValueError, match="static"):
        _layer("int4").from_codes(torch.zeros(4, 256, dtype=torch.uint8))


def test_require_checks_in_order():
    from weight_only_quantized_prologue_b200 import _require

    class FakeCuda:
        """Stands in for a CUDA tensor: the checks only read metadata."""

        def __init__(self, t):
            self.t, self.is_cuda, self.device = t, True, torch.device("cuda", 0)
            self.dtype, self.shape = t.dtype, t.shape

        def is_contiguous(self):
            return self.t.is_contiguous()

        def numel(self):
            return self.t.numel()

        def element_size(self):
            return self.t.element_size()

    good = FakeCuda(torch.zeros(4, 256, dtype=torch.bfloat16))
    _require(good, "x", shape=(4, 256), dtype=torch.bfloat16, nbytes=2048, device=torch.device("cuda", 0))
    with pytest.raises(ValueError, match="contiguous"):
        _require(FakeCuda(torch.zeros(256, 4, dtype=torch.bfloat16).t()), "x")
    with pytest.raises(TypeError, match="bfloat16"):
        _require(FakeCuda(torch.zeros(4, 256)), "x", dtype=torch.bfloat16)
    with pytest.raises(ValueError, match="shape"):
        _require(good, "x", shape=(4, 128))
    with pytest.raises(ValueError, match="bytes"):
        _require(good, "x", nbytes=1024)
    with pytest.raises(ValueError, match="expected"):
        _require(good, "x", device=torch.device("cuda", 1))


def test_layer_cannot_be_copied_or_pickled():
    import copy
    import pickle

    lin = _layer()
    for fn in (copy.copy, copy.deepcopy, pickle.dumps):
        with pytest.raises(TypeError, match="handle"):
            fn(lin)


def test_dqlinear_module_cannot_be_deep_copied():
    # nn.Module deepcopy reaches the layer and stops there, instead of
    # producing two owners of one handle
    import copy

    from weight_only_quantized_prologue_b200 import module as M

    mod = M.DQLinear.__new__(M.DQLinear)
    torch.nn.Module.__init__(mod)
    mod.layer = _layer()
    with pytest.raises(TypeError, match="handle"):
        copy.deepcopy(mod)


def test_x_on_another_device_is_rejected():
    # the handle belongs to cuda:0; an operand on cuda:1 would be read through
    # a pointer of the wrong device
    from weight_only_quantized_prologue_b200 import _fits

    class OnDevice1:
        dtype, is_cuda, shape = torch.bfloat16, True, (4, 256)
        device = torch.device("cuda", 1)

        def dim(self):
            return 2

        def is_contiguous(self):
            return True

        def get_device(self):
            return 1

    lin = _layer()
    assert not _fits(OnDevice1(), 256, torch.bfloat16, dev=lin._dev)
    with pytest.raises(ValueError, match="expected cuda:0"):
        lin(OnDevice1())


def test_buffers_may_be_given_as_integer_addresses():
    # the C entry points take plain pointers: the binding passes an integer
    # address through unchanged, takes a tensor's data_ptr and an array's data
    import numpy as np

    from weight_only_quantized_prologue_b200 import _native

    assert _native._ptr(None) is None
    assert _native._ptr(0x7F0000001000) == 0x7F0000001000
    a = np.zeros(4, dtype=np.float32)
    assert _native._ptr(a) == a.ctypes.data
    t = torch.zeros(4)
    assert _native._ptr(t) == t.data_ptr()
