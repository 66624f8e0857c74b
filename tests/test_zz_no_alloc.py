"""waits_score_static: the scorer for callers that cannot allocate device
memory (an engine plugin whose host owns the device pool, code where an
allocation is forbidden or would synchronise the device).  It must give the
scores of waits_score, whose scratch the caller passes in, on consecutive
calls that reuse the one static scratch array.

This file is collected last on purpose: if it fails, a run that stops at
the first failure has already run every other test.
"""

import ctypes

import numpy as np
import pytest
import torch

from gpu_parity import SCORE_RTOL, assert_scores_close
from prefill_eviction_scoring_b200 import _lib, api
from prefill_eviction_scoring_b200 import workloads as wl


def _score_static_raw(lib, lay, a, b, out):
    T, Hq, d = lay.Q.shape
    shape = api.make_shape(lay.cu_seqlens, T, lay.max_seqlen, Hq, lay.K.shape[1], d)
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    return lib.waits_score_static(ctypes.byref(shape), lay.Q.data_ptr(), lay.K.data_ptr(),
                                  float(a), int(b), out.data_ptr(), stream)


def test_oversized_shape_is_rejected_before_any_launch():
    """A shape whose workspace exceeds the static array returns
    WAITS_ERR_WORKSPACE on the host; no pointer is touched."""
    lib = _lib.load()
    shape = _lib.Shape(1, 131072, 131072, 32, 8, 128, 0x100000)
    n = ctypes.c_size_t(0)
    assert lib.waits_workspace_size(ctypes.byref(shape), ctypes.byref(n)) == 0
    assert n.value > _lib.STATIC_WORKSPACE_BYTES
    st = lib.waits_score_static(ctypes.byref(shape), 0x100000, 0x100000, 1.0, 16, 0x100000,
                                None)
    assert st == 4


@pytest.mark.gpu
def test_static_scratch_matches_workspace_entry_point_twice():
    """Two different layers scored back to back through waits_score_static
    agree with waits_score (caller workspace) within the score tolerance."""
    lib = _lib.load()
    cases = [
        (wl.make_layer("llama8b", lens=(2100, 700), heads=(8, 2), heavy_hitters=16,
                       device="cuda"), 1.0, 16),
        (wl.make_layer("ragged", lens=(900, 129, 1, 450), heads=(14, 2), device="cuda"),
         0.05, 40),
    ]
    for lay, a, b in cases:
        ref = api.score(lay.Q, lay.K, lay.cu_seqlens, sigmoid_a=a, window=b)
        torch.cuda.synchronize()
        ref = ref.double().cpu().numpy()
        for _ in range(2):
            out = torch.full((lay.K.shape[1], lay.total_tokens), -1.0, device="cuda")
            _lib.check("waits_score_static", _score_static_raw(lib, lay, a, b, out))
            torch.cuda.synchronize()
            got = out.double().cpu().numpy()
            assert np.all(got >= 0.0)
            assert_scores_close(got, ref, rtol=SCORE_RTOL)


@pytest.mark.gpu
def test_full_size_layer_fits_the_static_scratch():
    """The 32768-token Llama-3.1-8B-shaped layer fits in the static array."""
    lay = wl.make_layer("llama8b", device="cuda")
    ref = api.score(lay.Q, lay.K, lay.cu_seqlens, sigmoid_a=1.0, window=16)
    out = api.score_static(lay.Q, lay.K, lay.cu_seqlens, sigmoid_a=1.0, window=16)
    torch.cuda.synchronize()
    assert_scores_close(out.double().cpu().numpy(), ref.double().cpu().numpy())


@pytest.mark.gpu
def test_static_status_word_reports_bad_seqlens_then_clears():
    """A malformed cu_seqlens handed to waits_score_static sets the bad-offsets
    bit of the status word in the library's static scratch, which
    waits_read_static_status reads; the next well-formed call clears it."""
    lib = _lib.load()
    lay = wl.make_layer("tiny", lens=(300,), device="cuda")
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    out = torch.empty((lay.K.shape[1], lay.total_tokens), device="cuda")
    st = ctypes.c_uint32(0)
    bad_cu = torch.tensor([0, lay.total_tokens - 7], dtype=torch.int32, device="cuda")
    T, Hq, d = lay.Q.shape
    bad = api.make_shape(bad_cu, T, lay.max_seqlen, Hq, lay.K.shape[1], d)
    _lib.check("waits_score_static", lib.waits_score_static(
        ctypes.byref(bad), lay.Q.data_ptr(), lay.K.data_ptr(), 1.0, 16, out.data_ptr(), stream))
    _lib.check("waits_read_static_status", lib.waits_read_static_status(stream, ctypes.byref(st)))
    assert st.value & _lib.DEV_BAD_SEQLENS
    _lib.check("waits_score_static", _score_static_raw(lib, lay, 1.0, 16, out))
    _lib.check("waits_read_static_status", lib.waits_read_static_status(stream, ctypes.byref(st)))
    assert st.value == 0


def test_static_status_reader_rejects_null():
    lib = _lib.load()
    assert lib.waits_read_static_status(None, None) == 1
