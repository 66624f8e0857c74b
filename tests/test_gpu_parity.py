"""CUDA path vs the fp64 oracle, element by element, on seeded inputs that
span several tiles and ragged tails (small enough for the oracle)."""

import numpy as np
import pytest
import torch

import oracle
from gpu_parity import assert_scores_close, full_check, run_gpu
from prefill_eviction_scoring_b200 import workloads as wl

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("a,b", [(1.0, 16), (0.0, 16), (1e4, 1)])
def test_tiny_config(a, b):
    """N=512, 4 query heads on 1 KV head, d=64; a=1,b=16 plus the H2O and
    TOVA limit actions."""
    lay = wl.make_layer("tiny", device="cuda")
    full_check(lay, a, b, 16, 128)


@pytest.mark.parametrize("a,b", wl.WAITS_ACTIONS)
def test_llama1b_shape_actions(a, b):
    """1B-shaped heads (d=64, GQA 4, sink) at a length the oracle finishes
    quickly, every README action."""
    lay = wl.make_layer("llama1b", lens=(1100,), heads=(8, 2), device="cuda")
    full_check(lay, a, b, 16, 128)


@pytest.mark.parametrize("B", [128, 512])
def test_llama8b_shape(B):
    """8B-shaped heads (d=128, GQA 4) with sink and heavy hitters."""
    lay = wl.make_layer("llama8b", lens=(2000,), heads=(8, 2), heavy_hitters=16,
                        device="cuda")
    full_check(lay, 1.0, 16, 16, B)


def test_ragged_qwen_shape():
    """Packed varlen batch with Qwen's G=7 grouping, lengths 1 and 129."""
    lay = wl.make_layer("ragged", lens=(300, 129, 1, 700, 64), heads=(14, 2),
                        device="cuda")
    full_check(lay, 10.0, 16, 16, 128)


def test_long_shape_dense_mode():
    """a=0.01, b=128 activates ~9000 rows at full size; here about 1000 of
    2500, enough for the stationary-K scheduling."""
    lay = wl.make_layer("long", lens=(2500,), heads=(8, 2), heavy_hitters=32,
                        device="cuda")
    full_check(lay, 0.01, 128, 64, 256)


@pytest.mark.parametrize("case", [
    dict(lens=(50,), a=1.0, b=16, R=16, B=128),         # N < tile, N <= B
    dict(lens=(129,), a=1.0, b=16, R=16, B=128),        # one past B
    dict(lens=(700,), a=1.0, b=16, R=0, B=64),          # R = 0
    dict(lens=(700,), a=1.0, b=16, R=64, B=64),         # R = B
    dict(lens=(512,), a=1.0, b=600, R=16, B=128),       # b >= N
    dict(lens=(400,), a=1e4, b=0, R=16, B=128),         # no active row at all
    dict(lens=(1, 1, 300), a=0.0, b=1, R=2, B=4),       # one-token sequences
    dict(lens=(1000,), a=0.3, b=40, R=8, B=300),
])
@pytest.mark.parametrize("d", [64, 128])
def test_edge_cases(case, d):
    lay = wl.random_layer(case["lens"], 8, 2, d, seed=77 + d, device="cuda")
    full_check(lay, case["a"], case["b"], case["R"], case["B"])


def test_exact_ties_bit_exact():
    """a=1e4, b=1 and a zero last query: every score is exactly G/N and the
    kept pool is the lowest indices."""
    N, G = 256, 4
    lay = wl.random_layer((N,), 8, 2, 128, seed=5, device="cuda")
    lay.Q[N - 1] = 0
    gpu = run_gpu(lay, 1e4, 1, 16, 64)
    assert np.all(gpu["scores"] == G / N)
    want = list(range(48)) + list(range(N - 16, N))
    for g in range(2):
        assert gpu["idx"][0, g].tolist() == want


def test_zero_keys_closed_form():
    """K = 0: P[q,k] = 1/(q+1), so at a=0 the scores are (G/2)(H_N - H_k)."""
    N, G = 600, 4
    lay = wl.random_layer((N,), 8, 2, 128, seed=6, device="cuda")
    lay.K.zero_()
    gpu = run_gpu(lay, 0.0, 1, 16, 128)
    H = np.concatenate([[0.0], np.cumsum(1.0 / np.arange(1, N + 1))])
    want = 0.5 * G * (H[N] - H[:N])
    for g in range(2):
        assert_scores_close(gpu["scores"][g:g + 1], want[None, :])


def test_sum_identity():
    """Each query row's P sums to 1: sum_k s[g,k] = G * sum_q w[q]."""
    lay = wl.make_layer("llama8b", lens=(3000, 1000), heads=(8, 2), device="cuda")
    gpu = run_gpu(lay, 0.05, 30, 16, 128)
    cu = lay.cu_seqlens.cpu().numpy()
    for i in range(2):
        N = cu[i + 1] - cu[i]
        w = oracle.forgetting_curve(np.arange(N), N, 0.05, 30)
        for g in range(2):
            tot = gpu["scores"][g, cu[i]:cu[i + 1]].sum()
            assert abs(tot - 4 * w.sum()) <= 1e-5 * 4 * w.sum()


def test_deterministic_bits():
    lay = wl.make_layer("llama8b", lens=(1500, 900), heads=(8, 2), device="cuda")
    a = run_gpu(lay, 0.02, 64, 16, 128)
    b = run_gpu(lay, 0.02, 64, 16, 128)
    assert torch.equal(a["raw_scores"].view(torch.int32), b["raw_scores"].view(torch.int32))
    assert np.array_equal(a["idx"], b["idx"])


@pytest.mark.parametrize("make,a,b", [
    (lambda: wl.make_layer("llama8b", device="cuda"), 1.0, 16),
    (lambda: wl.make_layer("llama1b", device="cuda"), 10.0, 1),
    (lambda: wl.make_layer("ragged", lens=(5000,), heads=(14, 2), device="cuda"), 10.0, 16),
    (lambda: wl.make_layer("ragged", lens=(40,), heads=(4, 4), device="cuda"), 1.0, 16),
    (lambda: wl.make_layer("ragged", lens=(1500, 900, 77), heads=(8, 2), device="cuda"), 1.0, 16),
    (lambda: wl.make_layer("ragged", lens=(300,), heads=(4, 1), device="cuda"), 10.0, 1),
])
def test_in_cta_plan_equals_planner_kernel(make, a, b, monkeypatch):
    """The plan every scorer CTA rebuilds for itself and the planner kernel's
    plan give the same scores bit for bit (same units, same order)."""
    import ctypes
    from prefill_eviction_scoring_b200 import _lib, api
    lay = make()
    T, Hq, d = lay.Q.shape
    shape = api.make_shape(lay.cu_seqlens, T, lay.max_seqlen, Hq, lay.K.shape[1], d)
    lib = _lib.load()

    def kernels():
        n = ctypes.c_int32(0)
        _lib.check("waits_score_kernels", lib.waits_score_kernels(ctypes.byref(shape), a, b,
                                                                  ctypes.byref(n)))
        return n.value

    monkeypatch.delenv("WAITS_PLANNER_KERNEL", raising=False)
    monkeypatch.delenv("WAITS_DEVICE_PLAN", raising=False)
    assert kernels() == 2
    # one-sequence batches: the plan the host builds, then the CTAs' own
    s_local = api.score(lay.Q, lay.K, lay.cu_seqlens, sigmoid_a=a, window=b).clone()
    monkeypatch.setenv("WAITS_DEVICE_PLAN", "1")
    s_device = api.score(lay.Q, lay.K, lay.cu_seqlens, sigmoid_a=a, window=b).clone()
    monkeypatch.setenv("WAITS_PLANNER_KERNEL", "1")
    assert kernels() == 4
    s_kernel = api.score(lay.Q, lay.K, lay.cu_seqlens, sigmoid_a=a, window=b)
    torch.cuda.synchronize()
    assert torch.equal(s_local.view(torch.int32), s_device.view(torch.int32))
    assert torch.equal(s_local.view(torch.int32), s_kernel.view(torch.int32))


def test_separate_calls_equal_fused():
    """waits_score, waits_select and waits_compact called one by one give
    the same bits as waits_compress."""
    from prefill_eviction_scoring_b200 import api
    lay = wl.make_layer("ragged", lens=(400, 250), heads=(7, 1), device="cuda")
    s = api.score(lay.Q, lay.K, lay.cu_seqlens, sigmoid_a=1.0, window=16)
    idx, kept = api.select(s, lay.cu_seqlens, recent_budget=16, budget=128)
    Ko, Vo = api.compact(lay.K, lay.V, lay.cu_seqlens, idx, kept)
    Ko2, Vo2, idx2, kept2, s2 = api.compress(lay.Q, lay.K, lay.V, lay.cu_seqlens, sigmoid_a=1.0,
                                             window=16, recent_budget=16, budget=128)
    torch.cuda.synchronize()
    assert torch.equal(s.view(torch.int32), s2.view(torch.int32))
    assert torch.equal(idx, idx2) and torch.equal(kept, kept2)
    assert torch.equal(Ko.view(torch.int16), Ko2.view(torch.int16))
    assert torch.equal(Vo.view(torch.int16), Vo2.view(torch.int16))


def test_bad_seqlens_flagged_not_faulting():
    """Malformed cu_seqlens are caught on the device: status bit set, no work."""
    from prefill_eviction_scoring_b200 import Compressor, _lib
    lay = wl.random_layer((300, 200), 8, 2, 64, seed=9, device="cuda")
    bad = torch.tensor([0, 350, 500], dtype=torch.int32, device="cuda")   # 350 > max 300
    c = Compressor(bad, 500, 300, 8, 2, 64, 128)
    c(lay.Q, lay.K, lay.V, 1.0, 16, 16)
    torch.cuda.synchronize()
    assert c.device_status() & _lib.DEV_BAD_SEQLENS


@pytest.mark.parametrize("end", [499, 501])
def test_bad_seqlens_one_sequence(end):
    """A one-sequence batch whose offsets are not {0, T} (the host-built plan
    is checked on the device): status bit set, no work, scores untouched."""
    from prefill_eviction_scoring_b200 import Compressor, _lib
    lay = wl.random_layer((500,), 8, 2, 128, seed=11, device="cuda")
    bad = torch.tensor([0, end], dtype=torch.int32, device="cuda")
    c = Compressor(bad, 500, 500, 8, 2, 128, 64)
    c.scores.fill_(-7.0)
    c(lay.Q, lay.K, lay.V, 1.0, 16, 16)
    torch.cuda.synchronize()
    assert c.device_status() & _lib.DEV_BAD_SEQLENS
    assert torch.all(c.scores == -7.0)


def test_compact_bad_index_flagged():
    from prefill_eviction_scoring_b200 import api, _lib
    lay = wl.random_layer((100,), 8, 2, 128, seed=10, device="cuda")
    idx = torch.arange(16, dtype=torch.int32, device="cuda").view(1, 1, 16).repeat(1, 2, 1)
    idx[0, 1, 3] = 100        # == N: out of range
    kept = torch.tensor([16], dtype=torch.int32, device="cuda")
    ws = torch.zeros(4096, dtype=torch.uint8, device="cuda")
    Ko, Vo = api.compact(lay.K, lay.V, lay.cu_seqlens, idx, kept, workspace=ws)
    torch.cuda.synchronize()
    assert int(ws[:4].view(torch.int32).item()) & _lib.DEV_BAD_INDEX
    assert torch.all(Ko[0, 1, 3] == 0)
    assert torch.equal(Ko[0, 0], lay.K[:16, 0])


@pytest.mark.parametrize("pinned_v", [True, False])
def test_host_buffer_entry_point(pinned_v):
    """waits_compress_host gives the same result as the device entry point,
    whether V is read in place (page-locked) or copied first (pageable)."""
    from prefill_eviction_scoring_b200 import HostCompressor
    lay = wl.make_layer("ragged", lens=(900, 333), heads=(14, 2), device="cuda")
    gpu = run_gpu(lay, 1.0, 16, 16, 128, canary=False)
    hc = HostCompressor(lay.cu_seqlens.cpu(), 14, 2, 128, 128)
    Qh, Kh = (t.cpu().pin_memory() for t in (lay.Q, lay.K))
    Vh = lay.V.cpu().pin_memory() if pinned_v else lay.V.cpu()
    Ko, Vo, idx, kept = hc(Qh, Kh, Vh, 1.0, 16, 16)
    torch.cuda.synchronize()
    assert np.array_equal(idx.numpy(), gpu["idx"])
    assert np.array_equal(Ko.view(torch.int16).numpy(), gpu["Ko"])
    assert np.array_equal(Vo.view(torch.int16).numpy(), gpu["Vo"])
    row = 2 * 128 * 2                           # one position of K or V, both KV heads
    k_bytes = 1233 * row
    v_bytes = (128 + 128) * row if pinned_v else 1233 * row   # kept rows only, or all of V
    q_active = 2 * 120 * 14 * 128 * 2          # ~b + 90/a rows per sequence
    lo = k_bytes + v_bytes
    assert lo < hc.h2d_bytes < lo + q_active + 4096   # only the active Q rows


@pytest.mark.parametrize("lens,R,B,levels,signed", [
    ((20000,), 64, 2048, 50, False),          # few levels: many ties at the threshold
    ((40000, 3000), 16, 1024, 7, False),      # ragged batch
    ((50000,), 16, 4096, 1, False),           # every score equal
    ((9000,), 0, 300, 100000, False),         # nearly distinct scores, R = 0
    ((150000, 700), 16, 2048, 3000, False),   # pool past the cluster's staging (8 x 8192 keys)
    ((5000, 2600), 8, 512, 40, True),         # negative values, -0 and +0
    ((3000,), 16, 2999, 5, False),            # one pool position dropped
    ((21, 40, 17, 300), 16, 20, 6, False),    # pools of a few keys: CTAs without a group
    (tuple(range(1, 4000, 97)), 16, 64, 30, False),   # 42 sequences, N <= B among them
])
def test_select_exact_on_synthetic_scores(lens, R, B, levels, signed):
    """waits_select alone, on scores with controlled ties, equals the
    oracle's selection of the same fp32 values."""
    from prefill_eviction_scoring_b200 import api
    g = torch.Generator(device="cuda")
    g.manual_seed(123)
    Hkv, T = 3, sum(lens)
    s = torch.randint(0, levels, (Hkv, T), generator=g, device="cuda").float() / 64.0
    if signed:
        s = s - (levels // 2) / 64.0
        s[s == 0] = torch.where(torch.rand(int((s == 0).sum()), generator=g, device="cuda") < 0.5,
                                -0.0, 0.0)
    cu = torch.tensor([0] + list(np.cumsum(lens)), dtype=torch.int32, device="cuda")
    idx, kept = api.select(s, cu, recent_budget=R, budget=B)
    torch.cuda.synchronize()
    ref_idx, ref_kept = oracle.select(s.double().cpu().numpy(), cu.cpu().numpy(), R, B)
    np.testing.assert_array_equal(idx.cpu().numpy(), ref_idx)
    np.testing.assert_array_equal(kept.cpu().numpy(), ref_kept)


_SELECT_COMPACT_CASES = [
    ((20000,), 64, 2048, 50, 128),            # many ties at the threshold
    ((40000, 3000), 16, 1024, 7, 64),         # ragged batch
    ((50000,), 16, 4096, 1, 128),             # every score equal: one run of slots
    ((9000,), 0, 300, 100000, 128),           # R = 0
    ((150000, 700), 16, 2048, 3000, 128),     # pool past the cluster's staging
    ((3000,), 16, 2999, 5, 64),               # one pool position dropped
    ((3000,), 3000, 3000, 5, 128),            # want = 0: the recent window only
    ((21, 40, 17, 300), 16, 20, 6, 128),      # pools of a few keys, N <= B among them
    (tuple(range(1, 4000, 97)), 16, 64, 30, 64),   # 42 sequences
    ((70000,), 16, 9000, 2, 128),             # rounds of 4096 slots, the last one partial
]


@pytest.mark.parametrize("lens,R,B,levels,d", _SELECT_COMPACT_CASES)
def test_select_compact_exact(lens, R, B, levels, d):
    """waits_select_compact (selection and the K/V copy in one kernel) equals
    the oracle's selection and compaction, bit for bit, and the two separate
    calls."""
    from prefill_eviction_scoring_b200 import api
    g = torch.Generator(device="cuda")
    g.manual_seed(321)
    Hkv, T = 2, sum(lens)
    s = torch.randint(0, levels, (Hkv, T), generator=g, device="cuda").float() / 64.0
    K = torch.randint(-32768, 32767, (T, Hkv, d), generator=g, device="cuda",
                      dtype=torch.int32).to(torch.int16).view(torch.bfloat16)
    V = torch.randint(-32768, 32767, (T, Hkv, d), generator=g, device="cuda",
                      dtype=torch.int32).to(torch.int16).view(torch.bfloat16)
    cu = torch.tensor([0] + list(np.cumsum(lens)), dtype=torch.int32, device="cuda")
    idx, kept, Ko, Vo = api.select_compact(s, K, V, cu, recent_budget=R, budget=B)
    idx2, kept2 = api.select(s, cu, recent_budget=R, budget=B)
    Ko2, Vo2 = api.compact(K, V, cu, idx2, kept2)
    torch.cuda.synchronize()
    ref_idx, ref_kept = oracle.select(s.double().cpu().numpy(), cu.cpu().numpy(), R, B)
    Kb, Vb = (t.view(torch.int16).cpu().numpy() for t in (K, V))
    ref_K, ref_V = oracle.compact(Kb, Vb, cu.cpu().numpy(), ref_idx, ref_kept, B)
    np.testing.assert_array_equal(idx.cpu().numpy(), ref_idx)
    np.testing.assert_array_equal(kept.cpu().numpy(), ref_kept)
    np.testing.assert_array_equal(Ko.view(torch.int16).cpu().numpy(), ref_K)
    np.testing.assert_array_equal(Vo.view(torch.int16).cpu().numpy(), ref_V)
    assert torch.equal(idx, idx2) and torch.equal(kept, kept2)
    assert torch.equal(Ko.view(torch.int16), Ko2.view(torch.int16))
    assert torch.equal(Vo.view(torch.int16), Vo2.view(torch.int16))


def test_select_compact_bad_seqlens_zero_rows():
    """Malformed offsets: status bit set, every output row zero, no K/V read."""
    from prefill_eviction_scoring_b200 import api, _lib
    K = torch.ones((500, 2, 128), dtype=torch.bfloat16, device="cuda")
    s = torch.ones((2, 500), dtype=torch.float32, device="cuda")
    bad = torch.tensor([0, 350, 499], dtype=torch.int32, device="cuda")   # last != T
    lib = _lib.load()
    shape = api.make_shape(bad, 500, 350, 2, 2, 128)
    idx = torch.empty((2, 2, 64), dtype=torch.int32, device="cuda")
    kept = torch.empty((2,), dtype=torch.int32, device="cuda")
    Ko = torch.full((2, 2, 64, 128), 7.0, dtype=torch.bfloat16, device="cuda")
    Vo = torch.full_like(Ko, 7.0)
    ws = torch.zeros(4096, dtype=torch.uint8, device="cuda")
    import ctypes
    st = lib.waits_select_compact(ctypes.byref(shape), s.data_ptr(), K.data_ptr(), K.data_ptr(),
                                  16, 64, idx.data_ptr(), kept.data_ptr(), Ko.data_ptr(),
                                  Vo.data_ptr(), ws.data_ptr(), ws.numel(),
                                  torch.cuda.current_stream().cuda_stream)
    _lib.check("waits_select_compact", st)
    torch.cuda.synchronize()
    assert int(ws[:4].view(torch.int32).item()) & _lib.DEV_BAD_SEQLENS
    assert torch.all(Ko[1] == 0) and torch.all(Vo[1] == 0)
    assert int(kept[1].item()) == 0
