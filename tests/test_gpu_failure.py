"""Failure paths and the scorer's FMA-pipe exponential, on the GPU.

* The scorer's bounded waits: with the MMA warp withholding its work (a
  testing aid read from the environment) every wait for an accumulator runs
  out after a short limit; the call must end with WAITS_DEV_TIMEOUT in the
  status word, without a fault or a hang, and the next normal call on the
  same context must be clean and correct.
* exp2_poly_acc, the 2^x that part of the epilogue computes on the FMA pipe:
  relative error at most 1.02e-4 against exact powers of two over
  [-125, 127], exact at integers, zero at and below -127 (its clamp), and
  within the bound down to -126.5 where the result becomes subnormal.
"""

import ctypes
import time

import numpy as np
import pytest
import torch

import oracle
from gpu_parity import assert_scores_close
from prefill_eviction_scoring_b200 import Compressor, _lib
from prefill_eviction_scoring_b200 import workloads as wl

TIMEOUT_BIT = _lib.DEV_TIMEOUT


def _compressor(lay, B=128):
    T, Hq, d = lay.Q.shape
    return Compressor(lay.cu_seqlens, T, lay.max_seqlen, Hq, lay.K.shape[1], d, B)


@pytest.mark.gpu
@pytest.mark.parametrize("lens,heads,d,a,b", [((512,), (4, 1), 64, 1.0, 16),
                                              ((3000,), (8, 2), 128, 0.0, 16),
                                              ((700, 129, 1500), (8, 2), 128, 0.05, 40)])
def test_withheld_mma_times_out_then_recovers(monkeypatch, lens, heads, d, a, b):
    lay = wl.random_layer(lens, heads[0], heads[1], d, seed=41, device="cuda")
    c = _compressor(lay)
    monkeypatch.setenv("WAITS_WAIT_LIMIT_NS", "1000000")      # 1 ms
    monkeypatch.setenv("WAITS_TEST_WITHHOLD_MMA", "1")
    t0 = time.perf_counter()
    c.score(lay.Q, lay.K, a, b)
    status = c.device_status()                                 # synchronises
    assert status & TIMEOUT_BIT, f"status {status:#x}"
    assert time.perf_counter() - t0 < 10.0
    monkeypatch.delenv("WAITS_TEST_WITHHOLD_MMA")
    monkeypatch.delenv("WAITS_WAIT_LIMIT_NS")
    s = c.score(lay.Q, lay.K, a, b)
    torch.cuda.synchronize()
    assert c.device_status() == 0
    ref = oracle.score(wl.to_numpy64(lay.Q), wl.to_numpy64(lay.K),
                       lay.cu_seqlens.cpu().numpy(), a, b)
    assert_scores_close(s.double().cpu().numpy(), ref)


def _exp2_poly(x: torch.Tensor) -> torch.Tensor:
    lib = _lib.load()
    y = torch.empty_like(x)
    st = lib.waits_test_exp2_poly(x.data_ptr(), y.data_ptr(), x.numel(),
                                  ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    _lib.check("waits_test_exp2_poly", st)
    torch.cuda.synchronize()
    return y


@pytest.mark.gpu
def test_exp2_poly_relative_error_bound():
    grid = np.linspace(-125.0, 127.0, 4_000_001, dtype=np.float64).astype(np.float32)
    # both sides of every rounding boundary n + 1/2, and the integers
    half = np.arange(-125, 127, dtype=np.float64) + 0.5
    edges = np.concatenate([np.nextafter(half.astype(np.float32), np.float32(-200)),
                            half.astype(np.float32),
                            np.nextafter(half.astype(np.float32), np.float32(200))])
    x = np.concatenate([grid, edges]).astype(np.float32)
    y = _exp2_poly(torch.from_numpy(x).cuda()).cpu().numpy().astype(np.float64)
    ref = np.exp2(x.astype(np.float64))
    rel = np.abs(y - ref) / ref
    # the cubic alone is off by at most 1.013e-4 on [-1/2, 1/2] (fp64 scan of
    # 1 + f (c1 + f (c2 + f c3)) against 2^f); fp32 evaluation adds < 1e-6
    assert rel.max() <= 1.02e-4, f"max relative error {rel.max():.3e}"
    assert np.all(np.isfinite(y)) and np.all(y > 0)


@pytest.mark.gpu
def test_exp2_poly_exact_at_integers_and_clamped():
    n = np.arange(-126, 128, dtype=np.float32)
    y = _exp2_poly(torch.from_numpy(n).cuda()).cpu().numpy()
    np.testing.assert_array_equal(y, np.exp2(n.astype(np.float64)).astype(np.float32))
    # raised to -127, whose 2^n pattern is +0: nothing below, like a flush to zero
    far = np.array([-np.inf, -1e30, -1000.0, -127.0, -126.75, -126.5], dtype=np.float32)
    y = _exp2_poly(torch.from_numpy(far).cuda()).cpu().numpy()
    np.testing.assert_array_equal(y, np.zeros(len(far), dtype=np.float32))
    assert not np.signbit(y).any()
    # n = -126 with f in (-1/2, 1/2]: 2^-126 times the cubic, subnormal below 2^-126
    x = np.linspace(-126.49, -125.51, 99).astype(np.float32)
    y = _exp2_poly(torch.from_numpy(x).cuda()).cpu().numpy().astype(np.float64)
    ref = np.exp2(x.astype(np.float64))
    assert (np.abs(y - ref) / ref).max() <= 1.02e-4
