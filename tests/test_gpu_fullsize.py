"""Parity at the workloads' full sizes, in the launch configuration the bench
times: exact oracle values where the oracle finishes in seconds (the 8B
layer per KV head, the ragged batch, the 1B layer), identities that hold at
any size elsewhere (the 131072-token layer)."""

import numpy as np
import pytest
import torch

import oracle
from gpu_parity import (assert_compaction, assert_scores_close, assert_selection,
                        run_gpu)
from prefill_eviction_scoring_b200 import workloads as wl

pytestmark = pytest.mark.gpu


def _group_ref(lay, g, a, b):
    """Oracle scores of KV head g alone (its G query heads, its keys)."""
    Hq, Hkv = lay.Q.shape[1], lay.K.shape[1]
    G = Hq // Hkv
    Q = wl.to_numpy64(lay.Q[:, g * G:(g + 1) * G])
    K = wl.to_numpy64(lay.K[:, g:g + 1])
    return oracle.score(Q, K, lay.cu_seqlens.cpu().numpy(), a, b)[0]


def _group_tail_ref(lay, g, a, b, W):
    """Oracle scores of KV head g from the last W rows of each sequence:
    exact for the last W keys (a key is seen only by rows at or after it)."""
    Hq, Hkv = lay.Q.shape[1], lay.K.shape[1]
    G = Hq // Hkv
    Q = wl.to_numpy64(lay.Q[:, g * G:(g + 1) * G])
    K = wl.to_numpy64(lay.K[:, g:g + 1])
    return oracle.score(Q, K, lay.cu_seqlens.cpu().numpy(), a, b, last=W)[0]


@pytest.mark.parametrize("layer,B,heads", [(0, 2048, tuple(range(8))), (0, 512, (0, 5)),
                                           (31, 128, (2, 7))])
def test_llama8b_full(layer, B, heads):
    spec = wl.CONFIGS["llama8b"]
    lay = wl.make_layer("llama8b", layer=layer, device="cuda")
    a, b = spec.actions[0]
    gpu = run_gpu(lay, a, b, spec.recent, B)
    cu = lay.cu_seqlens.cpu().numpy()
    ref = np.zeros_like(gpu["scores"])
    for g in heads:
        ref[g] = _group_ref(lay, g, a, b)
        assert_scores_close(gpu["scores"][g:g + 1], ref[g:g + 1])
    # selection / compaction for the checked heads
    for g in heads:
        sub_idx = gpu["idx"][:, g:g + 1]
        assert_selection(sub_idx, gpu["kept"], ref[g:g + 1], gpu["scores"][g:g + 1], cu,
                         spec.recent, B)
    assert_compaction(lay, gpu, B)


def test_ragged_full():
    spec = wl.CONFIGS["ragged"]
    lay = wl.make_layer("ragged", device="cuda")
    a, b = spec.actions[0]
    B = spec.budgets[0]
    gpu = run_gpu(lay, a, b, spec.recent, B)
    cu = lay.cu_seqlens.cpu().numpy()
    ref = oracle.score(wl.to_numpy64(lay.Q), wl.to_numpy64(lay.K), cu, a, b)
    assert_scores_close(gpu["scores"], ref)
    assert_selection(gpu["idx"], gpu["kept"], ref, gpu["scores"], cu, spec.recent, B)
    assert_compaction(lay, gpu, B)


@pytest.mark.parametrize("a,b", wl.WAITS_ACTIONS)
def test_llama1b_full(a, b):
    spec = wl.CONFIGS["llama1b"]
    lay = wl.make_layer("llama1b", device="cuda")
    gpu = run_gpu(lay, a, b, spec.recent, spec.budgets[0])
    for g in (0, 7):
        assert_scores_close(gpu["scores"][g:g + 1], _group_ref(lay, g, a, b)[None])
    assert_compaction(lay, gpu, spec.budgets[0])


def test_long_full_properties():
    spec = wl.CONFIGS["long"]
    lay = wl.make_layer("long", device="cuda")
    a, b = spec.actions[0]
    B = spec.budgets[0]
    gpu = run_gpu(lay, a, b, spec.recent, B)
    s = gpu["scores"]
    N = lay.total_tokens
    assert np.all(s >= 0.0) and np.all(np.isfinite(s))
    w = oracle.forgetting_curve(np.arange(N), N, a, b)
    G = lay.Q.shape[1] // lay.K.shape[1]
    for g in range(s.shape[0]):
        assert abs(s[g].sum() - G * w.sum()) <= 1e-4 * G * w.sum()
    cu = lay.cu_seqlens.cpu().numpy()
    self_idx, self_kept = oracle.select(s, cu, spec.recent, B)
    np.testing.assert_array_equal(gpu["idx"], self_idx)
    assert_compaction(lay, gpu, B)


def test_llama8b_dense_properties():
    """The 8B layer with a = 0 (every row active, w = 1/2: the stress shape
    whose plan needs the planner kernel and pass 2's stationary K tiles):
    identities that hold at any size, and the selection of the GPU's own
    scores."""
    spec = wl.CONFIGS["llama8b"]
    lay = wl.make_layer("llama8b", device="cuda")
    B = 2048
    gpu = run_gpu(lay, 0.0, 16, spec.recent, B)
    s = gpu["scores"]
    N = lay.total_tokens
    G = lay.Q.shape[1] // lay.K.shape[1]
    assert np.all(s >= 0.0) and np.all(np.isfinite(s))
    for g in range(s.shape[0]):
        # every row of P sums to 1 and w = 1/2: the scores of a head sum to G N / 2
        assert abs(s[g].astype(np.float64).sum() - G * N / 2) <= 1e-4 * G * N / 2
        # the last key is seen by the last row only
        assert s[g, N - 1] <= G * 0.5 * (1 + 1e-5)
    cu = lay.cu_seqlens.cpu().numpy()
    self_idx, self_kept = oracle.select(s, cu, spec.recent, B)
    np.testing.assert_array_equal(gpu["idx"], self_idx)
    np.testing.assert_array_equal(gpu["kept"], self_kept)
    assert_compaction(lay, gpu, B)


def test_long_full_tail_exact():
    """The 131072-token layer (a = 0.01, b = 128: some 9000 active rows):
    the last 1024 keys of two KV heads against the oracle, element by
    element; they depend only on the last 1024 rows."""
    spec = wl.CONFIGS["long"]
    lay = wl.make_layer("long", device="cuda")
    a, b = spec.actions[0]
    gpu = run_gpu(lay, a, b, spec.recent, spec.budgets[0])
    N, W = lay.total_tokens, 1024
    for g in (1, 6):
        ref = _group_tail_ref(lay, g, a, b, W)
        assert_scores_close(gpu["scores"][g:g + 1, N - W:], ref[None, N - W:])


def test_llama8b_dense_tail_exact():
    """The 8B layer with a = 0 (every row active): the last 2048 keys of two
    KV heads against the oracle, element by element."""
    lay = wl.make_layer("llama8b", layer=7, device="cuda")
    gpu = run_gpu(lay, 0.0, 16, 16, 2048)
    N, W = lay.total_tokens, 2048
    for g in (0, 4):
        ref = _group_tail_ref(lay, g, 0.0, 16, W)
        assert_scores_close(gpu["scores"][g:g + 1, N - W:], ref[None, N - W:])
