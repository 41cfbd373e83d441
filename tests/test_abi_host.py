"""Host-side checks of the C ABI (no GPU needed): the library loads and
exports every entry point include/dqgemm.h declares, the host packer is
bit-identical to the oracle, argument errors come back as status codes, and
the split-K arithmetic of the GEMM (K-stage ranges per rank, the owner's
reads of the partial tiles) covers everything exactly once, in rank order."""

import ctypes
import os
import re

import numpy as np
import pytest

import weight_only_quantized_prologue_b200 as dq
from oracle import linear as L

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared_symbols():
    with open(os.path.join(ROOT, "include", "dqgemm.h")) as f:
        text = f.read()
    return sorted(set(re.findall(r"^\s*(?:const\s+char\s*\*|dqgemm_status)\s+(dqgemm_\w+)\s*\(", text, re.M)))


def test_library_exports_every_declared_symbol():
    names = _declared_symbols()
    assert "dqgemm_create" in names and "dqgemm_run" in names and len(names) >= 11
    lib = ctypes.CDLL(dq._native.LIB_PATH)
    missing = [n for n in names if not hasattr(lib, n)]
    assert not missing, missing


def _weights(N, K, seed, kind="uniform"):
    rng = np.random.default_rng(seed)
    if kind == "uniform":
        W = rng.uniform(-1, 1, (N, K)) / np.sqrt(K)
    elif kind == "wide":      # many binades, exact zeros, ties, subnormals
        W = rng.normal(size=(N, K)) * np.exp2(rng.integers(-30, 10, (N, K)))
        W[rng.random((N, K)) < 0.05] = 0.0
        W[0, :] = 0.0                                   # an all-zero row / group / block
        W[1, :64] = np.float32(2.0 ** -140)             # fp32 subnormals
    else:
        raise ValueError(kind)
    return W.astype(np.float32)


@pytest.mark.parametrize("fmt", ["int4", "nvfp4", "mxfp4", "fp8", "int4_asym"])
@pytest.mark.parametrize("kind", ["uniform", "wide"])
def test_pack_host_is_bit_identical_to_oracle(fmt, kind):
    N, K = 96, 512
    W = _weights(N, K, seed=3, kind=kind)
    packed, scales, g = dq.dqgemm_pack_host(fmt, W)
    ref = L.quantize_pack(fmt, W.astype(np.float64))
    assert np.array_equal(packed, ref["packed"])
    assert np.array_equal(scales.view(np.uint8), np.ascontiguousarray(ref["scales"]).astype(scales.dtype).view(np.uint8))
    assert np.float32(g) == np.float32(ref["global_scale"])


def test_pack_host_hand_example_int4():
    # group max 7 -> scale 1.0, codes = RNE(W): 3.5 -> 4, 2.5 -> 2, -2.5 -> -2
    W = np.zeros((1, 128), np.float32)
    W[0, :4] = [7.0, 3.5, 2.5, -2.5]
    packed, scales, _ = dq.dqgemm_pack_host("int4", W)
    assert scales.tolist() == [[0x3F80]]
    assert packed[0, :2].tolist() == [0x47, 0xE2]


@pytest.mark.parametrize("fmt,K,N", [("int4", 100, 8), ("nvfp4", 24, 16), ("nvfp4", 32, 8),
                                     ("mxfp4", 48, 32), ("mxfp4", 64, 16), ("fp8", 8, 4), ("int4", 0, 8),
                                     ("int4_asym", 200, 8)])
def test_pack_host_rejects_bad_shapes(fmt, K, N):
    W = np.zeros((max(N, 1), max(K, 1)), np.float32)
    st = dq._native.lib().dqgemm_pack_host(dq.FORMATS[fmt], W.ctypes.data, K, N, W.ctypes.data, W.ctypes.data, None)
    assert st == dq._native.DQ_ERR_INVALID_ARG


def test_pack_host_rejects_non_finite():
    W = np.ones((16, 128), np.float32)
    W[3, 7] = np.inf
    with pytest.raises(dq.DQError) as e:
        dq.dqgemm_pack_host("int4", W)
    assert e.value.status == dq._native.DQ_ERR_INVALID_ARG


def test_entry_points_reject_null_arguments_without_touching_the_gpu():
    lib = dq._native.lib()
    h = ctypes.c_void_p()
    assert lib.dqgemm_create(ctypes.byref(h), 0, 128, 128, None, None, 1.0, None) == dq._native.DQ_ERR_INVALID_ARG
    assert lib.dqgemm_create(None, 0, 128, 128, None, None, 1.0, None) == dq._native.DQ_ERR_INVALID_ARG
    assert lib.dqgemm_create(ctypes.byref(h), 9, 128, 128, 16, 16, 1.0, None) == dq._native.DQ_ERR_INVALID_ARG
    assert lib.dqgemm_create(ctypes.byref(h), 0, 100, 128, 16, 16, 1.0, None) == dq._native.DQ_ERR_INVALID_ARG
    assert lib.dqgemm_run(None, 16, 4, 16, None) == dq._native.DQ_ERR_INVALID_ARG
    assert lib.dqgemm_destroy(None) == dq._native.DQ_ERR_INVALID_ARG
    assert lib.dqgemm_last_error(None) == dq._native.DQ_ERR_INVALID_ARG
    assert lib.dqgemm_quantize_act_fp8(None, 1, 1, 1.0, None, None) == dq._native.DQ_ERR_INVALID_ARG
    assert lib.dqgemm_quantize_act_fp8(16, 1, 16, -1.0, 16, None) == dq._native.DQ_ERR_INVALID_ARG
    assert lib.dqgemm_selftest_timeout(0, None) == dq._native.DQ_ERR_INVALID_ARG
    assert dq.dqgemm_status_string(6) == "DQ_ERR_TIMEOUT"


# -- split-K: the arithmetic of dq_gemm_kernel's cluster split -------------


def _stage_range(q, KS, S):
    """K stages of rank q (cta_work): [q*KS/S, (q+1)*KS/S)."""
    return q * KS // S, (q + 1) * KS // S


@pytest.mark.parametrize("S", [2, 4, 8])
@pytest.mark.parametrize("KS", [2, 3, 8, 24, 25, 112])
def test_split_k_stage_ranges_cover_k_once(S, KS):
    if S > KS:                 # the planner never splits deeper than k_stages
        return
    seen = np.zeros(KS, dtype=int)
    for q in range(S):
        a, b = _stage_range(q, KS, S)
        assert b > a
        seen[a:b] += 1
    assert (seen == 1).all()


def _owner_reads(q, h, BN, S):
    """(rank, column) pairs that thread half h of rank q reads, in the order
    it adds them: value i is rank i % S of column c0 + h + 2 * (i // S)."""
    cmax, c0 = BN // S, q * (BN // S)
    return [(i % S, c0 + h + 2 * (i // S)) for i in range(BN // 2)]


@pytest.mark.parametrize("BN", [16, 32, 64, 128])
@pytest.mark.parametrize("S", [2, 4, 8])
def test_split_k_owners_read_every_partial_once_in_rank_order(BN, S):
    got = {}
    for q in range(S):
        owned = set(range(q * BN // S, (q + 1) * BN // S))
        for h in range(2):
            reads = _owner_reads(q, h, BN, S)
            for k, (pr, c) in enumerate(reads):
                assert c in owned                      # only its own columns
                assert (pr, c) not in got              # each partial value once
                got[(pr, c)] = (q, h, k)
            # each column's S values are consecutive and in rank order 0..S-1
            for j in range(0, len(reads), S):
                assert [pr for pr, _ in reads[j:j + S]] == list(range(S))
                assert len({c for _, c in reads[j:j + S]}) == 1
    assert len(got) == S * BN                          # every rank x column
