"""Shared checks for the GPU parity tests: run the CUDA path through the C ABI
and compare it with the fp64 oracle on the same bits."""

import numpy as np
import torch

import oracle
from prefill_eviction_scoring_b200 import Compressor
from prefill_eviction_scoring_b200 import workloads as wl

SCORE_RTOL = 1e-3      # relative tolerance on every score (bf16 in, fp32 math)
TINY = 1e-30           # below this an oracle score is compared absolutely


def run_gpu(lay, a, b, R, B, canary=True):
    """waits_compress through the C ABI; outputs copied to the host.
    With ``canary`` the output buffers are checked for writes outside them."""
    T, Hq, d = lay.Q.shape
    Hkv = lay.K.shape[1]
    c = Compressor(lay.cu_seqlens, T, lay.max_seqlen, Hq, Hkv, d, B)
    if canary:
        pad = 64
        big = torch.full((Hkv * T + 2 * pad,), -7.0, device="cuda")
        c.scores = big[pad:pad + Hkv * T].view(Hkv, T)
        nid = c.idx.numel()
        bigi = torch.full((nid + 2 * pad,), -777, dtype=torch.int32, device="cuda")
        c.idx = bigi[pad:pad + nid].view_as(c.idx)
        nk = c.kept_len.numel()
        bigk = torch.full((nk + 2 * pad,), -555, dtype=torch.int32, device="cuda")
        c.kept_len = bigk[pad:pad + nk]
        # K_out / V_out: guard rows of 16-byte vectors (the kernels write whole rows)
        no = c.K_out.numel()
        gpad = 8 * d
        bigo = [torch.full((no + 2 * gpad,), 7.5, dtype=torch.bfloat16, device="cuda")
                for _ in range(2)]
        c.K_out = bigo[0][gpad:gpad + no].view_as(c.K_out)
        c.V_out = bigo[1][gpad:gpad + no].view_as(c.V_out)
    Ko, Vo, idx, kept, s = c(lay.Q, lay.K, lay.V, a, b, R)
    torch.cuda.synchronize()
    status = c.device_status()
    assert status == 0, f"device status {status:#x}"
    if canary:
        assert torch.all(big[:pad] == -7.0) and torch.all(big[pad + Hkv * T:] == -7.0)
        assert torch.all(bigi[:pad] == -777) and torch.all(bigi[pad + nid:] == -777)
        assert torch.all(bigk[:pad] == -555) and torch.all(bigk[pad + nk:] == -555)
        for t in bigo:
            assert torch.all(t[:gpad] == 7.5) and torch.all(t[gpad + no:] == 7.5)
    return dict(scores=s.double().cpu().numpy(), idx=idx.cpu().numpy(),
                kept=kept.cpu().numpy(), Ko=Ko.cpu().view(torch.int16).numpy(),
                Vo=Vo.cpu().view(torch.int16).numpy(), raw_scores=s.clone())


def assert_scores_close(got, ref, rtol=SCORE_RTOL):
    assert got.shape == ref.shape
    big = ref >= TINY
    rel = np.abs(got[big] - ref[big]) / ref[big]
    worst = float(rel.max()) if rel.size else 0.0
    assert worst <= rtol, f"max relative score error {worst:.3e} > {rtol}"
    assert np.all(np.abs(got[~big] - ref[~big]) <= TINY)
    return worst


def assert_selection(gpu_idx, gpu_kept, ref_scores, gpu_scores, cu, R, B):
    """GPU select equals the oracle's select of the GPU's own fp32 scores, and
    differs from the oracle's select of the fp64 scores only at boundary
    ties within the score tolerance."""
    self_idx, self_kept = oracle.select(gpu_scores, cu, R, B)
    np.testing.assert_array_equal(gpu_idx, self_idx)
    np.testing.assert_array_equal(gpu_kept, self_kept)
    ref_idx, ref_kept = oracle.select(ref_scores, cu, R, B)
    np.testing.assert_array_equal(gpu_kept, ref_kept)
    for i in range(len(cu) - 1):
        lo = cu[i]
        n = int(ref_kept[i])
        for g in range(ref_idx.shape[1]):
            a = set(ref_idx[i, g, :n].tolist())
            b = set(gpu_idx[i, g, :n].tolist())
            for x in a - b:
                for y in b - a:
                    sx, sy = ref_scores[g, lo + x], ref_scores[g, lo + y]
                    assert abs(sx - sy) <= SCORE_RTOL * max(sx, sy), (i, g, x, y, sx, sy)


def assert_compaction(lay, gpu, B):
    cu = lay.cu_seqlens.cpu().numpy()
    Kr, Vr = oracle.compact(wl.to_bits(lay.K), wl.to_bits(lay.V), cu, gpu["idx"],
                            gpu["kept"], B)
    np.testing.assert_array_equal(gpu["Ko"], Kr)
    np.testing.assert_array_equal(gpu["Vo"], Vr)


def full_check(lay, a, b, R, B):
    gpu = run_gpu(lay, a, b, R, B)
    cu = lay.cu_seqlens.cpu().numpy()
    ref = oracle.score(wl.to_numpy64(lay.Q), wl.to_numpy64(lay.K), cu, a, b)
    worst = assert_scores_close(gpu["scores"], ref)
    assert_selection(gpu["idx"], gpu["kept"], ref, gpu["scores"], cu, R, B)
    assert_compaction(lay, gpu, B)
    return gpu, ref, worst
