"""waits_decode_attention: one decode step over the compacted cache, against
oracle.decode_attention on the same bits.  Tolerance: fp32 arithmetic on bf16
inputs, so every output is held to 1e-4 of sum_j p_j |V_j| (the oracle's
attention applied to |V|, the scale of the sum's terms) and the LSE to 1e-4."""

import numpy as np
import pytest
import torch

import oracle
from prefill_eviction_scoring_b200 import api
from prefill_eviction_scoring_b200 import workloads as wl

pytestmark = pytest.mark.gpu


def _check(q, Kc, Vc, lens):
    out, lse = api.decode_attention(q, Kc, Vc, lens, with_lse=True)
    torch.cuda.synchronize()
    qn, Kn, Vn = (wl.to_numpy64(t) for t in (q, Kc, Vc))
    ln = lens.cpu().numpy()
    ref_o, ref_l = oracle.decode_attention(qn, Kn, Vn, ln)
    scale, _ = oracle.decode_attention(qn, Kn, np.abs(Vn), ln)
    o = out.double().cpu().numpy()
    l = lse.double().cpu().numpy()
    assert np.all(np.abs(o - ref_o) <= 1e-4 * scale + 1e-30)
    fin = np.isfinite(ref_l)
    assert np.all(np.abs(l[fin] - ref_l[fin]) <= 1e-4)
    assert np.all(np.isneginf(l[~fin])) and np.all(o[~fin] == 0.0)


@pytest.mark.parametrize("a,b,B", [(1.0, 16, 512), (0.0, 16, 300)])
def test_decode_after_compress(a, b, B):
    lay = wl.make_layer("llama8b", lens=(2100, 700), heads=(16, 4), heavy_hitters=8,
                        device="cuda")
    Ko, Vo, idx, kept, s = api.compress(lay.Q, lay.K, lay.V, lay.cu_seqlens, sigmoid_a=a,
                                        window=b, recent_budget=16, budget=B)
    g = torch.Generator(device="cuda")
    g.manual_seed(5)
    q = torch.randn((2, 16, 128), generator=g, device="cuda").to(torch.bfloat16)
    _check(q, Ko, Vo, kept)


@pytest.mark.parametrize("d,heads", [(128, (32, 8)), (64, (28, 4)), (128, (16, 16))])
def test_ragged_cache_lengths(d, heads):
    Hq, Hkv = heads
    C = 700
    lens = torch.tensor([0, 1, 255, 256, 257, C, 513], dtype=torch.int32, device="cuda")
    nseq = lens.numel()
    g = torch.Generator(device="cuda")
    g.manual_seed(9)
    q = torch.randn((nseq, Hq, d), generator=g, device="cuda").to(torch.bfloat16)
    Kc = torch.randn((nseq, Hkv, C, d), generator=g, device="cuda").to(torch.bfloat16)
    Vc = torch.randn((nseq, Hkv, C, d), generator=g, device="cuda").to(torch.bfloat16)
    Kc[:, :, 0] *= 8.0   # a sink in the first slot
    _check(q, Kc, Vc, lens)


def test_slots_past_length_are_not_read():
    g = torch.Generator(device="cuda")
    g.manual_seed(13)
    q = torch.randn((1, 8, 128), generator=g, device="cuda").to(torch.bfloat16)
    Kc = torch.randn((1, 2, 600, 128), generator=g, device="cuda").to(torch.bfloat16)
    Vc = torch.randn((1, 2, 600, 128), generator=g, device="cuda").to(torch.bfloat16)
    lens = torch.tensor([300], dtype=torch.int32, device="cuda")
    a = api.decode_attention(q, Kc, Vc, lens).clone()
    Kc[:, :, 300:] = float("nan")
    Vc[:, :, 300:] = float("inf")
    b = api.decode_attention(q, Kc, Vc, lens)
    torch.cuda.synchronize()
    assert torch.equal(a, b)
