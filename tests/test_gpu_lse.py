"""waits_score_with_lse: the scorer fed the row normalisers by the caller
(as a FlashAttention forward returns them) runs the column-sum pass only and
must give the oracle's scores.  The LSE comes from oracle.row_lse."""

import numpy as np
import pytest
import torch

import oracle
from gpu_parity import assert_scores_close
from prefill_eviction_scoring_b200 import Compressor
from prefill_eviction_scoring_b200 import workloads as wl


def _compressor(lay):
    T, Hq, d = lay.Q.shape
    return Compressor(lay.cu_seqlens, T, lay.max_seqlen, Hq, lay.K.shape[1], d, 128)


def _check(lay, a, b, last=None, monkeypatch=None, env=None):
    if env:
        for k, v in env.items():
            monkeypatch.setenv(k, v)
    cu = lay.cu_seqlens.cpu().numpy()
    Qn, Kn = wl.to_numpy64(lay.Q), wl.to_numpy64(lay.K)
    lse = torch.from_numpy(oracle.row_lse(Qn, Kn, cu, last=last)).float().cuda()
    c = _compressor(lay)
    got = c.score_with_lse(lay.Q, lay.K, lse, a, b).double().cpu().numpy()
    torch.cuda.synchronize()
    assert c.device_status() == 0
    two_pass = c.score(lay.Q, lay.K, a, b).double().cpu().numpy()
    ref = oracle.score(Qn, Kn, cu, a, b)
    assert_scores_close(got, ref)
    # against the two-pass scorer: the same sums with another fp32 normaliser
    big = ref > 1e-30
    assert np.max(np.abs(got[big] - two_pass[big]) / ref[big]) < 2e-4
    return got, ref


@pytest.mark.gpu
@pytest.mark.parametrize("a,b", [(1.0, 16), (0.0, 16), (1e4, 1)])
def test_tiny(a, b):
    _check(wl.make_layer("tiny", device="cuda"), a, b)


@pytest.mark.gpu
@pytest.mark.parametrize("a,b", [(1.0, 16), (10.0, 1), (0.01, 128)])
def test_llama1b_shape(a, b):
    _check(wl.make_layer("llama1b", lens=(1500,), device="cuda"), a, b)


@pytest.mark.gpu
def test_ragged_batch_with_short_sequences():
    lay = wl.make_layer("ragged", lens=(900, 129, 1, 450, 2000), heads=(14, 2), device="cuda")
    _check(lay, 0.05, 40)


@pytest.mark.gpu
def test_planner_kernel_and_general_scorer(monkeypatch):
    lay = wl.make_layer("llama1b", lens=(700, 1300), heads=(8, 2), device="cuda")
    _check(lay, 1.0, 16, monkeypatch=monkeypatch,
           env={"WAITS_PLANNER_KERNEL": "1", "WAITS_SCORER": "tc"})


@pytest.mark.gpu
def test_dense_stationary_keys_mode():
    # a = 0: every row active, many Q tiles: pass 2 holds K tiles (planner kernel)
    lay = wl.random_layer((2500,), 8, 2, 128, seed=5, device="cuda")
    _check(lay, 0.0, 16)


@pytest.mark.gpu
def test_full_size_8b_layer_last_rows():
    # N = 32768, a = 1, b = 16: only the last 105 rows have non-zero fp32
    # weight, so the LSE of the last 128 rows is all the scorer reads
    lay = wl.make_layer("llama8b", device="cuda")
    cu = lay.cu_seqlens.cpu().numpy()
    g = 3
    Qn = wl.to_numpy64(lay.Q[:, 4 * g:4 * g + 4])
    Kn = wl.to_numpy64(lay.K[:, g:g + 1])
    lse_g = oracle.row_lse(Qn, Kn, cu, last=128)
    lse = torch.full((32, lay.total_tokens), float("nan"))
    lse[4 * g:4 * g + 4] = torch.from_numpy(lse_g).float()
    c = _compressor(lay)
    got = c.score_with_lse(lay.Q, lay.K, lse.cuda(), 1.0, 16)[g].double().cpu().numpy()
    ref = oracle.score(Qn, Kn, cu, 1.0, 16)[0]
    assert_scores_close(got[None], ref[None])
