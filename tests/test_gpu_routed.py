"""waits_score_routed / waits_compress_routed: one packed batch whose
sequences each take their own forgetting curve (the README's routed WAITS
picks one of its five (a, b) actions per sample).  Every sequence must get
the scores the oracle gives it alone with its own (a, b)."""

import numpy as np
import pytest
import torch

import oracle
from gpu_parity import assert_compaction, assert_scores_close, assert_selection
from prefill_eviction_scoring_b200 import Compressor, _lib
from prefill_eviction_scoring_b200 import workloads as wl

pytestmark = pytest.mark.gpu


def _per_sequence_ref(lay, actions):
    cu = lay.cu_seqlens.cpu().numpy()
    Qn, Kn = wl.to_numpy64(lay.Q), wl.to_numpy64(lay.K)
    ref = np.zeros((lay.K.shape[1], lay.total_tokens))
    for i, (a, b) in enumerate(actions):
        lo, hi = int(cu[i]), int(cu[i + 1])
        ref[:, lo:hi] = oracle.score(Qn[lo:hi], Kn[lo:hi], np.array([0, hi - lo]), a, b)
    return ref


def _run(lay, actions, R, B):
    T, Hq, d = lay.Q.shape
    c = Compressor(lay.cu_seqlens, T, lay.max_seqlen, Hq, lay.K.shape[1], d, B)
    a = torch.tensor([x for x, _ in actions], dtype=torch.float32, device="cuda")
    b = torch.tensor([y for _, y in actions], dtype=torch.int32, device="cuda")
    Ko, Vo, idx, kept, s = c.compress_routed(lay.Q, lay.K, lay.V, a, b, R)
    torch.cuda.synchronize()
    status = c.device_status()
    return c, dict(scores=s.double().cpu().numpy(), idx=idx.cpu().numpy(), kept=kept.cpu().numpy(),
                   Ko=Ko.cpu().view(torch.int16).numpy(), Vo=Vo.cpu().view(torch.int16).numpy()), status


def test_five_actions_round_robin_ragged():
    lens = (700, 1300, 129, 1, 450, 2000, 333, 900)
    lay = wl.make_layer("ragged", lens=lens, device="cuda")
    actions = [wl.WAITS_ACTIONS[i % 5] for i in range(len(lens))]
    R, B = 16, 256
    c, gpu, status = _run(lay, actions, R, B)
    assert status == 0
    ref = _per_sequence_ref(lay, actions)
    assert_scores_close(gpu["scores"], ref)
    cu = lay.cu_seqlens.cpu().numpy()
    assert_selection(gpu["idx"], gpu["kept"], ref, gpu["scores"], cu, R, B)
    assert_compaction(lay, gpu, B)


def test_uniform_actions_equal_the_scalar_call():
    lay = wl.make_layer("ragged", lens=(900, 129, 1, 450), heads=(14, 2), device="cuda")
    T, Hq, d = lay.Q.shape
    c = Compressor(lay.cu_seqlens, T, lay.max_seqlen, Hq, 2, d, 64)
    a = torch.full((4,), 0.05, dtype=torch.float32, device="cuda")
    b = torch.full((4,), 40, dtype=torch.int32, device="cuda")
    routed = c.score_routed(lay.Q, lay.K, a, b).clone()
    scalar = c.score(lay.Q, lay.K, 0.05, 40).clone()
    torch.cuda.synchronize()
    ref = oracle.score(wl.to_numpy64(lay.Q), wl.to_numpy64(lay.K), lay.cu_seqlens.cpu().numpy(),
                       0.05, 40)
    assert_scores_close(routed.double().cpu().numpy(), ref)
    assert_scores_close(scalar.double().cpu().numpy(), ref)


def test_invalid_curve_is_flagged_and_zeroed():
    lens = (300, 200, 400)
    lay = wl.make_layer("ragged", lens=lens, heads=(14, 2), device="cuda")
    actions = [(1.0, 16), (-1.0, 16), (10.0, 1)]
    c, gpu, status = _run(lay, actions, 16, 128)
    assert status & _lib.DEV_BAD_CURVE
    assert np.all(gpu["scores"][:, 300:500] == 0.0)
    ref = _per_sequence_ref(lay, [actions[0], (0.0, 0), actions[2]])
    keep = np.r_[0:300, 500:900]
    assert_scores_close(gpu["scores"][:, keep], ref[:, keep])
