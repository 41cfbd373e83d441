"""dqgemm_pack_device_noalloc: the GPU weight packer without any device
allocation, for callers that cannot call cudaMalloc (a serving process that
reserved its whole memory budget up front, or code that must not trigger the
device-wide synchronization an allocation may cause).  Its only scratch, the
NVFP4 tensor-amax reduction, lives in a static device array shared by every
call, so each call here runs twice in a row: the second call must not be
disturbed by what the first left in that array.

This file is collected last so that a failure here does not hide the rest of
the suite; it passes alone and after the other tests alike."""

import ctypes

import numpy as np
import pytest
import torch

import weight_only_quantized_prologue_b200 as dq

pytestmark = pytest.mark.gpu

_TORCH = {np.uint8: torch.uint8, np.uint16: torch.int16, np.float32: torch.float32}


def _weights(N, K, seed, scale):
    g = torch.Generator("cpu").manual_seed(seed)
    w = torch.randn((N, K), generator=g) * scale
    w[0] = 0.0
    return w.cuda()


def _pack(entry, fmt, W):
    N, K = W.shape
    ps, pd, ss, sd = dq.storage_shapes(fmt, K, N)
    packed = torch.full(ps, 0xAB, dtype=_TORCH[pd], device="cuda")
    scales = torch.full(ss, 77, dtype=_TORCH[sd], device="cuda")
    g = entry(fmt, W, packed, scales)
    torch.cuda.synchronize()
    return packed.cpu().numpy(), scales.cpu().numpy().view(np.uint8), g


@pytest.mark.parametrize("fmt", ["nvfp4", "int4", "mxfp4", "fp8", "int4_asym"])
def test_noalloc_packer_matches_the_allocating_packer_on_two_calls(fmt):
    # the second call has a 1000x smaller tensor amax: a stale maximum left in
    # the shared scratch by the first call would change its global scale
    for call, (N, K, scale) in enumerate([(384, 4096, 3.0), (256, 1024, 0.003)]):
        W = _weights(N, K, seed=10 + call, scale=scale)
        ref = _pack(dq.dqgemm_pack_device, fmt, W)
        got = _pack(dq.dqgemm_pack_device_noalloc, fmt, W)
        assert np.array_equal(got[0], ref[0]), f"call {call}: packed codes differ"
        assert np.array_equal(got[1], ref[1]), f"call {call}: scales differ"
        assert np.float32(got[2]) == np.float32(ref[2]), f"call {call}: global scale differs"


def test_noalloc_packer_rejects_tensors_beyond_its_scratch():
    # NVFP4 keeps one partial maximum per 65536 weights, at most 4096 of them
    W = torch.zeros(16, dtype=torch.float32, device="cuda")
    out = torch.zeros(16, dtype=torch.uint8, device="cuda")
    st = dq._native.lib().dqgemm_pack_device_noalloc(dq.FORMATS["nvfp4"], W.data_ptr(), 16400, 16384,
                                                     out.data_ptr(), out.data_ptr(), None, None)
    assert st == dq._native.DQ_ERR_UNSUPPORTED


def test_noalloc_nvfp4_many_partials_with_the_maximum_in_the_last_partial_chunk():
    # 1040 x 16400 weights: 261 partial maxima (more than one per thread of the
    # final reduction's 256) and a last chunk holding only 16640 weights; the
    # tensor maximum sits in that last, partial chunk.  The second call is
    # smaller and its maximum is in its first chunk, so a stale partial left
    # by the first call would raise its global scale.
    for call, (N, K, where) in enumerate([(1040, 16400, -1), (512, 2048, 0)]):
        W = _weights(N, K, seed=20 + call, scale=0.5)
        flat = W.view(-1)
        flat[where] = 40.0 if call == 0 else 7.0
        ref = _pack(dq.dqgemm_pack_device, "nvfp4", W)
        got = _pack(dq.dqgemm_pack_device_noalloc, "nvfp4", W)
        assert np.array_equal(got[0], ref[0]), f"call {call}: packed codes differ"
        assert np.array_equal(got[1], ref[1]), f"call {call}: scales differ"
        assert np.float32(got[2]) == np.float32(ref[2]), f"call {call}: global scale differs"
        assert np.float32(got[2]) == np.float32(np.float32(40.0 if call == 0 else 7.0) / np.float32(2688.0))
