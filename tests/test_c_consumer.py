"""The C ABI used from plain C: tests/c_consumer/dq_consumer.c, built with
gcc against include/dqgemm.h and libdqgemm.so only.  On CPU its host packer
output must equal the oracle byte for byte and its argument errors must come
back as the statuses the header states; on a GPU the whole path driven from
C (pack on the device, create, run) must equal the Python binding's result
bit for bit, and the oracle within the GEMM tolerance."""

import os
import shutil
import struct
import subprocess

import numpy as np
import pytest

import weight_only_quantized_prologue_b200 as dq
from oracle import linear as L

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "tests", "c_consumer", "dq_consumer.c")
LIBDIR = os.path.dirname(dq._native.LIB_PATH)
CUDA_HOME = os.environ.get("CUDA_HOME", "/usr/local/cuda")
CODES = {"int4": 0, "nvfp4": 1, "mxfp4": 2, "fp8": 3, "fp8_static": 4, "int4_asym": 5}

pytestmark = pytest.mark.skipif(shutil.which("gcc") is None, reason="needs gcc")


def _build(tmp_path, gpu=False):
    exe = str(tmp_path / ("dq_consumer_gpu" if gpu else "dq_consumer"))
    cmd = ["gcc", "-std=c99", "-O1", "-Wall", "-Wextra", "-Werror", "-pedantic",
           "-I", os.path.join(ROOT, "include"), SRC, "-o", exe,
           "-L", LIBDIR, "-ldqgemm", f"-Wl,-rpath,{LIBDIR}", "-lm"]
    if gpu:
        # the CUDA runtime headers need C11 (anonymous unions); dqgemm.h
        # itself is held to pedantic C99 by the CPU build
        lib64 = os.path.join(CUDA_HOME, "lib64")
        cmd = [c for c in cmd if c != "-pedantic"]
        cmd[1] = "-std=c11"
        cmd[1:1] = ["-DDQ_CONSUMER_GPU", "-I", os.path.join(CUDA_HOME, "include")]
        cmd += ["-L", lib64, "-lcudart", f"-Wl,-rpath,{lib64}"]
    subprocess.run(cmd, check=True, capture_output=True, text=True)
    return exe


@pytest.fixture(scope="module")
def consumer(tmp_path_factory):
    return _build(tmp_path_factory.mktemp("c_consumer"))


def _weights(N, K, seed):
    rng = np.random.default_rng(seed)
    W = rng.uniform(-1, 1, (N, K)) / np.sqrt(K)
    W[3, 128:256] = 0.0                       # a zero group / block
    return W.astype(np.float32)


@pytest.mark.parametrize("fmt", ["int4", "nvfp4", "mxfp4", "fp8", "int4_asym"])
def test_c_pack_host_equals_oracle(consumer, tmp_path, fmt):
    N, K = 64, 384
    W = _weights(N, K, seed=11)
    win, out = tmp_path / "w.f32", tmp_path / "out.bin"
    W.tofile(win)
    r = subprocess.run([consumer, "pack", str(CODES[fmt]), str(K), str(N), str(win), str(out)],
                       capture_output=True, text=True, timeout=60)
    assert r.returncode == 0, r.stderr
    blob = out.read_bytes()
    st, g = struct.unpack("<if", blob[:8])
    ref = L.quantize_pack(fmt, W.astype(np.float64))
    packed = np.frombuffer(blob[8:8 + ref["packed"].size], dtype=np.uint8)
    scales = blob[8 + ref["packed"].size:]
    ref_scales = np.ascontiguousarray(ref["scales"])
    if fmt == "int4":
        ref_scales = ref_scales.astype(np.uint16)
    elif fmt == "fp8":
        ref_scales = ref_scales.astype(np.float32)
    else:
        ref_scales = ref_scales.astype(np.uint8)
    assert st == 0
    assert np.array_equal(packed, ref["packed"].ravel())
    assert scales == ref_scales.tobytes()
    assert np.float32(g) == np.float32(ref["global_scale"])


def test_c_argument_errors(consumer):
    r = subprocess.run([consumer, "errors"], capture_output=True, text=True, timeout=60)
    assert r.returncode == 0, r.stderr
    got = dict(line.split(" ", 1) for line in r.stdout.strip().splitlines())
    invalid = str(dq._native.DQ_ERR_INVALID_ARG)
    for case in ("pack_null_weight", "pack_k_not_group", "pack_unknown_format", "pack_non_finite",
                 "create_null_out", "run_null_handle", "plan_null_handle", "destroy_null",
                 "last_error_null"):
        assert got[case] == invalid, (case, got[case])
    assert got["create_null_weight"] == f"{invalid} 1"       # and *out was set to NULL
    align = str(dq._native.DQ_ERR_ALIGNMENT)
    assert got["create_misaligned"] == align and got["pack_device_misaligned"] == align
    for case in ("pack_device_null", "act_quant_m0", "act_quant_zero_scale", "act_quant_nan_scale"):
        assert got[case] == invalid, (case, got[case])
    assert got["status_string"] == dq.dqgemm_status_string(dq._native.DQ_ERR_INVALID_ARG)


def test_c_usage_error(consumer):
    assert subprocess.run([consumer], capture_output=True, timeout=60).returncode == 2


@pytest.mark.gpu
@pytest.mark.parametrize("fmt", ["int4", "nvfp4", "mxfp4", "fp8", "fp8_static", "int4_asym"])
def test_c_gemm_equals_binding_and_oracle(tmp_path, fmt):
    import torch

    from weight_only_quantized_prologue_b200 import synthetic

    exe = _build(tmp_path, gpu=True)
    M, K, N = 40, 256, 256
    x, w, b = synthetic.linear_inputs(M, K, N, seed=21)
    s_x = L.act_scale(float(x.float().min()), float(x.float().max()))
    w.numpy().astype(np.float32).tofile(tmp_path / "w.f32")
    x.view(torch.int16).numpy().tofile(tmp_path / "x.bf16")
    b.view(torch.int16).numpy().tofile(tmp_path / "b.bf16")
    out = tmp_path / "y.bf16"
    r = subprocess.run([exe, "gemm", str(CODES[fmt]), str(M), str(K), str(N), repr(s_x),
                        str(tmp_path / "w.f32"), str(tmp_path / "x.bf16"), str(tmp_path / "b.bf16"), str(out)],
                       capture_output=True, text=True, timeout=120)
    assert r.returncode == 0, r.stderr
    y_c = np.fromfile(out, dtype=np.int16).reshape(M, N)

    bias = None if fmt == "fp8_static" else b.cuda()
    lin = dq.QuantizedLinear.from_float(fmt, w.cuda(), bias, act_scale=s_x)
    y_py = lin(x.cuda())
    torch.cuda.synchronize()
    assert np.array_equal(y_c, y_py.view(torch.int16).cpu().numpy())
    lin.close()

    base = "fp8" if fmt == "fp8_static" else fmt
    st = L.quantize_pack(base, w.numpy().astype(np.float64))
    wd = L.dequant_exact(base, st["packed"], st["scales"], st["global_scale"])
    xv = x.float().numpy().astype(np.float64)
    if fmt == "fp8_static":
        from oracle import formats as F
        xv = F.e4m3_decode(L.quantize_act_fp8(xv, s_x)) * s_x
    ref = L.linear_ref(xv, wd, None if fmt == "fp8_static" else b.float().numpy().astype(np.float64))
    y = torch.from_numpy(y_c).view(torch.bfloat16).double().numpy()
    assert np.linalg.norm(y - ref) / np.linalg.norm(ref) <= 5e-3
