"""waits_compress_heads: a tensor-parallel rank scores, selects and compacts
its own KV heads of a layer in place.  The shards of a layer, put together,
must equal the whole-layer call and the oracle."""

import numpy as np
import pytest
import torch

import oracle
from gpu_parity import assert_scores_close, assert_selection
from prefill_eviction_scoring_b200 import api
from prefill_eviction_scoring_b200 import workloads as wl

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("lens,heads,d,a,b", [((2100, 700), (16, 4), 128, 1.0, 16),
                                              ((1500,), (8, 4), 64, 0.0, 16),
                                              ((900, 129, 1, 450), (28, 4), 128, 10.0, 16)])
def test_head_shards_equal_the_whole_layer(lens, heads, d, a, b):
    lay = wl.make_layer("llama8b", lens=lens, heads=heads, head_dim=d, heavy_hitters=8,
                        device="cuda")
    R, B = 16, 256
    kw = dict(sigmoid_a=a, window=b, recent_budget=R, budget=B)
    full = api.compress(lay.Q, lay.K, lay.V, lay.cu_seqlens, **kw)
    torch.cuda.synchronize()
    full_s = full[4].double().cpu().numpy()
    cu = lay.cu_seqlens.cpu().numpy()
    ref = oracle.score(wl.to_numpy64(lay.Q), wl.to_numpy64(lay.K), cu, a, b)
    Kb, Vb = wl.to_bits(lay.K), wl.to_bits(lay.V)
    Hkv = heads[1]
    for g0, g1 in ((0, 2), (2, 4), (1, 3), (3, 4)):
        Ko, Vo, idx, kept, s = api.compress_heads(lay.Q, lay.K, lay.V, lay.cu_seqlens, (g0, g1),
                                                  **kw)
        torch.cuda.synchronize()
        s = s.double().cpu().numpy()
        assert s.shape == (g1 - g0, lay.total_tokens)
        assert_scores_close(s, ref[g0:g1])
        big = ref[g0:g1] > 1e-30
        assert np.max(np.abs(s[big] - full_s[g0:g1][big]) / ref[g0:g1][big]) < 1e-5
        idx, kept = idx.cpu().numpy(), kept.cpu().numpy()
        assert_selection(idx, kept, ref[g0:g1], s, cu, R, B)
        Kr, Vr = oracle.compact(Kb[:, g0:g1], Vb[:, g0:g1], cu, idx, kept, B)
        np.testing.assert_array_equal(Ko.cpu().view(torch.int16).numpy(), Kr)
        np.testing.assert_array_equal(Vo.cpu().view(torch.int16).numpy(), Vr)


def test_bad_head_ranges_rejected():
    lay = wl.make_layer("tiny", lens=(64,), device="cuda")
    for rng in ((0, 0), (1, 1), (0, 2), (-1, 1)):
        with pytest.raises(Exception):
            api.compress_heads(lay.Q, lay.K, lay.V, lay.cu_seqlens, rng, sigmoid_a=1.0,
                               window=16, recent_budget=16, budget=32)
