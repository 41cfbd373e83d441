"""ctypes binding of libdqgemm (include/dqgemm.h): argument marshalling only.

Every computation happens in the CUDA library; this module converts torch
tensors / numpy arrays to pointers and status codes to exceptions.  It raises
at import of the library if ``libdqgemm.so`` has not been built: there is no
fallback implementation.
"""

import ctypes
import os

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libdqgemm.so")

FORMATS = {"int4": 0, "nvfp4": 1, "mxfp4": 2, "fp8": 3, "fp8_static": 4, "int4_asym": 5,
           "w4a4_mxfp4": 6, "w4a4_nvfp4": 7}
STATUS_NAMES = {0: "DQ_OK", 1: "DQ_ERR_INVALID_ARG", 2: "DQ_ERR_UNSUPPORTED", 3: "DQ_ERR_ALIGNMENT",
                4: "DQ_ERR_ALLOC", 5: "DQ_ERR_CUDA", 6: "DQ_ERR_TIMEOUT"}
DQ_OK, DQ_ERR_INVALID_ARG, DQ_ERR_UNSUPPORTED, DQ_ERR_ALIGNMENT = 0, 1, 2, 3
DQ_ERR_ALLOC, DQ_ERR_CUDA, DQ_ERR_TIMEOUT = 4, 5, 6


class DQError(RuntimeError):
    def __init__(self, status, what):
        super().__init__(f"{what}: {STATUS_NAMES.get(status, status)}")
        self.status = status


class Plan(ctypes.Structure):
    _fields_ = [("bn", ctypes.c_int), ("m_tiles", ctypes.c_int), ("n_tiles", ctypes.c_int),
                ("k_stages", ctypes.c_int), ("grid", ctypes.c_int), ("max_segments", ctypes.c_int),
                ("stages", ctypes.c_int), ("smem_bytes", ctypes.c_int),
                ("workspace_bytes", ctypes.c_longlong), ("weight_bytes", ctypes.c_longlong),
                ("x_stages", ctypes.c_int), ("max_cta_stages", ctypes.c_int)]

    def as_dict(self):
        return {f: getattr(self, f) for f, _ in self._fields_}


_VP, _I, _F = ctypes.c_void_p, ctypes.c_int, ctypes.c_float
_SIGNATURES = {
    "dqgemm_create": [ctypes.POINTER(_VP), _I, _I, _I, _VP, _VP, _F, _VP],
    "dqgemm_run": [_VP, _VP, _I, _VP, _VP],
    "dqgemm_run_fp8_static_quantized": [_VP, _VP, _I, _VP, _VP],
    "dqgemm_run_quantized_out": [_VP, _VP, _I, _VP, _F, _VP],
    "dqgemm_run_fp8_static_quantized_out": [_VP, _VP, _I, _VP, _F, _VP],
    "dqgemm_destroy": [_VP],
    "dqgemm_dequantize": [_VP, _VP, _VP],
    "dqgemm_quantize_act_fp8": [_VP, _I, _I, _F, _VP, _VP],
    "dqgemm_quantize_act_fp4": [_I, _VP, _I, _I, _VP, _VP, _VP, _VP],
    "dqgemm_pack_host": [_I, _VP, _I, _I, _VP, _VP, ctypes.POINTER(_F)],
    "dqgemm_pack_device": [_I, _VP, _I, _I, _VP, _VP, ctypes.POINTER(_F), _VP],
    "dqgemm_pack_device_noalloc": [_I, _VP, _I, _I, _VP, _VP, ctypes.POINTER(_F), _VP],
    "dqgemm_last_error": [_VP],
    "dqgemm_selftest_timeout": [_I, _VP],
    "dqgemm_get_plan": [_VP, _I, ctypes.POINTER(Plan)],
    "dqgemm_set_wait_limit": [_VP, ctypes.c_longlong],
    "dqgemm_run_static_mlp": [_VP, _VP, _VP, _I, _VP, _VP, _VP],
}

_lib = None


def lib():
    """The loaded library (loads it on first use; raises if it is not built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"{LIB_PATH} is missing; build it with "
                              "`python -m weight_only_quantized_prologue_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        for name, args in _SIGNATURES.items():
            fn = getattr(L, name)
            fn.argtypes = args
            fn.restype = ctypes.c_int
        L.dqgemm_status_string.argtypes = [ctypes.c_int]
        L.dqgemm_status_string.restype = ctypes.c_char_p
        _lib = L
    return _lib


def _check(status, what):
    if status != DQ_OK:
        raise DQError(status, what)


def _ptr(t):
    """A buffer's address: a tensor's data_ptr, a NumPy array's data, or an
    address given as an integer (the C entry points take plain pointers)."""
    if t is None or type(t) is int:
        return t
    if isinstance(t, np.ndarray):
        return t.ctypes.data_as(ctypes.c_void_p).value
    return t.data_ptr()


def _stream(stream):
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    return int(stream) if not hasattr(stream, "cuda_stream") else stream.cuda_stream


def storage_shapes(fmt, K, N):
    """Canonical (packed shape, packed dtype, scales shape, scales dtype) of a format."""
    if fmt == "int4":
        return (N, K // 2), np.uint8, (N, K // 128), np.uint16
    if fmt == "int4_asym":   # bf16 scales [N, K/128] then u8 zero points [N, K/128], one buffer
        return (N, K // 2), np.uint8, (3 * N * (K // 128),), np.uint8
    if fmt in ("nvfp4", "w4a4_nvfp4"):
        return (N, K // 2), np.uint8, (N, K // 16), np.uint8
    if fmt in ("mxfp4", "w4a4_mxfp4"):
        return (N, K // 2), np.uint8, (N, K // 32), np.uint8
    return (N, K), np.uint8, (N,), np.float32


# ---------------------------------------------------------------------------
# entry points, same names as the C ABI
# ---------------------------------------------------------------------------


def dqgemm_create(fmt, K, N, packed_w, scales, global_scale=1.0, bias=None):
    h = ctypes.c_void_p()
    _check(lib().dqgemm_create(ctypes.byref(h), FORMATS[fmt], K, N, _ptr(packed_w), _ptr(scales),
                               float(global_scale), _ptr(bias)), "dqgemm_create")
    return h


def dqgemm_run(h, x, M, y, stream=None):
    _check(lib().dqgemm_run(h, _ptr(x), int(M), _ptr(y), _stream(stream)), "dqgemm_run")


def run_ptrs(h, x_ptr, M, y_ptr, stream=None):
    """dqgemm_run on raw device addresses, for callers that have checked the
    operands already (QuantizedLinear's per-call path)."""
    _check(lib().dqgemm_run(h, x_ptr, M, y_ptr, _stream(stream)), "dqgemm_run")


def dqgemm_run_fp8_static_quantized(h, q, M, y, stream=None):
    _check(lib().dqgemm_run_fp8_static_quantized(h, _ptr(q), int(M), _ptr(y), _stream(stream)),
           "dqgemm_run_fp8_static_quantized")


def dqgemm_run_quantized_out(h, x, M, q_out, s_out, stream=None):
    _check(lib().dqgemm_run_quantized_out(h, _ptr(x), int(M), _ptr(q_out), float(s_out), _stream(stream)),
           "dqgemm_run_quantized_out")


def dqgemm_run_fp8_static_quantized_out(h, q, M, q_out, s_out, stream=None):
    _check(lib().dqgemm_run_fp8_static_quantized_out(h, _ptr(q), int(M), _ptr(q_out), float(s_out),
                                                      _stream(stream)), "dqgemm_run_fp8_static_quantized_out")


def dqgemm_run_static_mlp(l1, l2, x, M, h_out, y, stream=None):
    _check(lib().dqgemm_run_static_mlp(l1, l2, _ptr(x), int(M), _ptr(h_out), _ptr(y), _stream(stream)),
           "dqgemm_run_static_mlp")


def dqgemm_destroy(h):
    _check(lib().dqgemm_destroy(h), "dqgemm_destroy")


def dqgemm_dequantize(h, w_bf16, stream=None):
    _check(lib().dqgemm_dequantize(h, _ptr(w_bf16), _stream(stream)), "dqgemm_dequantize")


def dqgemm_quantize_act_fp8(x, M, K, s_x, q, stream=None):
    _check(lib().dqgemm_quantize_act_fp8(_ptr(x), M, K, float(s_x), _ptr(q), _stream(stream)),
           "dqgemm_quantize_act_fp8")


def dqgemm_quantize_act_fp4(fmt, x, M, K, codes, scales, g_x=None, stream=None):
    """FP4 activation quantization into canonical storage; g_x is a device
    float32 tensor of one element (NVFP4 formats)."""
    _check(lib().dqgemm_quantize_act_fp4(FORMATS[fmt], _ptr(x), int(M), int(K), _ptr(codes), _ptr(scales),
                                         _ptr(g_x), _stream(stream)), "dqgemm_quantize_act_fp4")


def dqgemm_pack_host(fmt, W):
    """W: float32 numpy [N, K] -> (packed, scales, global_scale) numpy arrays."""
    W = np.ascontiguousarray(W, dtype=np.float32)
    N, K = W.shape
    ps, pd, ss, sd = storage_shapes(fmt, K, N)
    packed = np.zeros(ps, dtype=pd)
    scales = np.zeros(ss, dtype=sd)
    g = ctypes.c_float(0.0)
    _check(lib().dqgemm_pack_host(FORMATS[fmt], _ptr(W), K, N, _ptr(packed), _ptr(scales), ctypes.byref(g)),
           "dqgemm_pack_host")
    return packed, scales, float(g.value)


def dqgemm_pack_device(fmt, W, packed, scales, stream=None):
    """W, packed, scales: CUDA tensors; returns the global scale."""
    N, K = W.shape
    g = ctypes.c_float(0.0)
    _check(lib().dqgemm_pack_device(FORMATS[fmt], _ptr(W), K, N, _ptr(packed), _ptr(scales), ctypes.byref(g),
                                    _stream(stream)), "dqgemm_pack_device")
    return float(g.value)


def dqgemm_pack_device_noalloc(fmt, W, packed, scales, stream=None):
    """As dqgemm_pack_device, with no device allocation (static scratch)."""
    N, K = W.shape
    g = ctypes.c_float(0.0)
    _check(lib().dqgemm_pack_device_noalloc(FORMATS[fmt], _ptr(W), K, N, _ptr(packed), _ptr(scales),
                                            ctypes.byref(g), _stream(stream)), "dqgemm_pack_device_noalloc")
    return float(g.value)


def dqgemm_last_error(h):
    return lib().dqgemm_last_error(h)


def dqgemm_selftest_timeout(timeout_us, stream=None):
    return lib().dqgemm_selftest_timeout(int(timeout_us), _stream(stream))


def dqgemm_set_wait_limit(h, timeout_ns):
    _check(lib().dqgemm_set_wait_limit(h, int(timeout_ns)), "dqgemm_set_wait_limit")


def dqgemm_get_plan(h, M):
    p = Plan()
    _check(lib().dqgemm_get_plan(h, int(M), ctypes.byref(p)), "dqgemm_get_plan")
    return p.as_dict()


def dqgemm_status_string(status):
    return lib().dqgemm_status_string(int(status)).decode()
