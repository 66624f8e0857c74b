"""The seeded input generator: determinism and the structures it plants."""

import torch

from prefill_eviction_scoring_b200 import workloads as wl


def test_deterministic_and_layer_distinct():
    a = wl.make_layer("llama1b", layer=0, lens=(300,))
    b = wl.make_layer("llama1b", layer=0, lens=(300,))
    c = wl.make_layer("llama1b", layer=1, lens=(300,))
    assert torch.equal(a.Q.view(torch.int16), b.Q.view(torch.int16))
    assert torch.equal(a.K.view(torch.int16), b.K.view(torch.int16))
    assert not torch.equal(a.K.view(torch.int16), c.K.view(torch.int16))


def test_shapes_and_layout():
    lay = wl.make_layer("ragged", lens=(100, 7, 33))
    assert lay.Q.shape == (140, 28, 128) and lay.Q.dtype == torch.bfloat16
    assert lay.K.shape == (140, 4, 128) and lay.V.shape == (140, 4, 128)
    assert lay.cu_seqlens.tolist() == [0, 100, 107, 140]
    assert lay.cu_seqlens.dtype == torch.int32


def test_sink_has_eight_times_norm():
    lay = wl.make_layer("llama1b", lens=(2000, 1000), sink=True)
    n = lay.K.float().norm(dim=-1)       # [T, Hkv]
    for lo in (0, 2000):
        ratio = n[lo] / n[lo + 1:lo + 500].mean(0)
        assert torch.all(ratio > 6.0) and torch.all(ratio < 10.0)


def test_heavy_hitters_cosine_half_with_visible_query():
    N, R = 3000, wl.CONFIGS["llama8b"].recent
    lay = wl.make_layer("llama8b", lens=(N,), heads=(8, 2), head_dim=64,
                        heavy_hitters=20)
    assert len(lay.heavy) == 2
    for (_i, g, p, h, qr) in lay.heavy:
        assert torch.all(p >= 1) and torch.all(p < N - R)
        assert torch.all(qr >= p) and torch.all(qr < N)
        assert torch.all(h // 4 == g)
        assert len(set(p.tolist())) == len(p)
        k = lay.K[p, g].float()
        q = lay.Q[qr, h].float()
        cos = (k * q).sum(-1) / (k.norm(dim=-1) * q.norm(dim=-1))
        assert torch.all((cos - 0.5).abs() < 0.02), cos


def test_ragged_lengths_in_range():
    lens = wl.CONFIGS["ragged"].lens
    assert len(lens) == 8 and all(4096 <= n <= 16384 for n in lens)
    assert wl.ragged_lengths(8, 4096, 16384, 4_000_000) == lens


def test_actions_are_the_readme_set():
    assert wl.WAITS_ACTIONS == ((0.0, 1), (0.01, 128), (1.0, 16), (10.0, 1),
                                (10.0, 16))
