#!/usr/bin/env python
"""WAITS prefill score + select + compact throughput on B200.

Default workload (the headline): the Llama-3.1-8B-shaped stack -- 32 layers
with independently seeded bf16 Q/K/V (sink + 64 heavy hitters per KV head),
batch 1, N=32768, 32 query / 8 KV heads, d=128, a=1, b=16, R=16, B=2048
(``--budget``).  A step runs score -> select -> compact once for every layer,
through the C ABI (waits_score, then waits_select_compact, on one stream).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--config llama8b|tiny|llama1b|ragged|long|stress|all]

``--config`` other than the default prints one JSON line per (action,
budget) of that workload; ``all`` runs every workload.  Multi-GPU (torchrun,
one rank per GPU): every rank owns its own layers (weak scaling); there is
no data-path collective.  Rank 0 prints the JSON lines.
"""

from __future__ import annotations

import argparse
import ctypes
import dataclasses
import datetime
import json
import math
import os
import statistics
import subprocess
import sys
import time
from typing import List, Optional, Sequence, Tuple

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from prefill_eviction_scoring_b200 import _lib, api  # noqa: E402
from prefill_eviction_scoring_b200 import workloads as wl  # noqa: E402

METRIC = "prompt tokens/s scored+compacted per layer (8B shape, N=32K); % of roofline"
UNIT = "tokens/s"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
                  "sm_max_mhz": 1965.0}
KERNELS_OUTSIDE_SCORE = 1   # select+compact (waits_score_kernels gives the scorer's)
EVENT_EVERY = 8         # stack workloads: CUDA events around every 8th layer's scorer
MUFU_EX2_PER_CLK_PER_SM = 16   # sm_100: 4 SFU lanes per SM sub-partition x 4
L2_BYTES = 126 << 20
# DRAM bytes (read + write) of one waits_score call on one 8B-shaped layer
# (N = 32768, a = 1, b = 16) from the committed ncu capture of the sparse
# scorer (both passes).  Valid only for the scorer code it was taken on
# (scorer_source_hash: score_sparse.cu and scorer_common.cuh, comments left
# out).
PROFILED_SCORER = {"sha256_prefix": "bdc00e2d01d32005",
                   "dram_bytes": 68_235_264 + 1_709_312 + 68_376_576 + 1_453_056}
PROFILED_SOURCES = ("score_sparse.cu", "scorer_common.cuh")


@dataclasses.dataclass(frozen=True)
class Case:
    """One bench line: a workload, its (a, b) action, R and B."""
    config: str          # workloads.CONFIGS key the tensors are drawn from
    name: str            # workload name in the JSON line
    a: float
    b: int
    R: int
    B: int
    layers: int


def cases_for(config: str, budget: Optional[int], layers: Optional[int]) -> List[Case]:
    """The bench lines of a workload (the BASELINE configurations)."""
    if config == "stress":
        spec = wl.CONFIGS["llama8b"]
        return [Case("llama8b", "stress", 0.0, 16, spec.recent, budget or 2048, layers or 1)]
    spec = wl.CONFIGS[config]
    budgets = (budget,) if budget else ((2048,) if config == "llama8b" else spec.budgets)
    if config == "llama8b" and budget is None:
        budgets = (2048,)
    out = []
    for a, b in spec.actions:
        for B in budgets:
            out.append(Case(config, config, a, b, spec.recent, B, layers or spec.layers))
    return out


ALL_CONFIGS = ("tiny", "llama1b", "llama8b", "ragged", "long", "stress")


def parse(argv=None):
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=50)
    p.add_argument("--warmup", type=int, default=3)
    p.add_argument("--impl", choices=["ours", "reference"], default="ours")
    p.add_argument("--config", choices=("llama8b",) + ALL_CONFIGS[:1] + ALL_CONFIGS[1:] + ("all",),
                   default="llama8b")
    p.add_argument("--budget", type=int, default=None,
                   help="B (default: 2048 for llama8b, the workload's budget otherwise); "
                        "for llama8b, --budget all sweeps 128, 512 and 2048")
    p.add_argument("--layers", type=int, default=None)
    p.add_argument("--parallel", choices=["layers", "heads"], default="layers",
                   help="multi-GPU split: every rank its own layers (weak scaling, default) "
                        "or every rank its share of the KV heads of the same layers "
                        "(tensor-parallel style, strong scaling)")
    p.add_argument("--e2e-layers", type=int, default=4)
    p.add_argument("--e2e-steps", type=int, default=3)
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--kernel-events", choices=["score", "none"], default="score",
                   help="stack workloads: record CUDA events around every 8th scorer call "
                        "inside the timed region (default), or none (scorer timed after it)")
    args, rest = p.parse_known_args(argv)
    if rest:
        p.error(f"unknown arguments {rest}")
    return args


def head_shard(rank: int, world: int, Hkv: int) -> Tuple[int, int]:
    """KV heads [g0, g1) of ``rank`` when ``world`` ranks split a layer's
    ``Hkv`` heads contiguously (ranks past Hkv own none)."""
    g0 = rank * Hkv // world if world <= Hkv else min(rank, Hkv)
    g1 = (rank + 1) * Hkv // world if world <= Hkv else min(rank + 1, Hkv)
    return g0, g1


# ------------------------------------------------------------ arithmetic ---
def first_active_row(N, a, b):
    """First row with non-zero fp32 forgetting-curve weight (the predicate
    the library's planner uses), by numpy float32."""
    if a == 0.0:
        return 0
    q = np.arange(N)
    c = np.float32(N) - np.float32(b) - np.float32(0.5)
    with np.errstate(over="ignore"):
        w = np.float32(1.0) / (np.float32(1.0) + np.exp(np.float32(-a) * (q.astype(np.float32) - c)))
    nz = np.nonzero(w != 0)[0]
    return int(nz[0]) if len(nz) else N


def scorer_flops(lens, Hq, d, a, b):
    """Algorithmic tensor FLOPs of one scorer call: two passes of causal
    QK^T over the active rows, 2*d FLOPs per logit."""
    logits = 0
    for N in lens:
        q0 = first_active_row(N, a, b)
        logits += (N * (N + 1) - q0 * (q0 + 1)) // 2     # sum_{q=q0}^{N-1} (q+1)
    return 2 * 2 * d * Hq * logits, logits * Hq


def scorer_bytes(lens, Hq, Hkv, d, a, b):
    """Algorithmic HBM bytes of one scorer call: all of K once, the query
    rows with non-zero fp32 weight once, the scores written once."""
    T = sum(lens)
    q_rows = sum(N - min(first_active_row(N, a, b), N) for N in lens)
    return T * Hkv * d * 2 + q_rows * Hq * d * 2 + Hkv * T * 4


def select_compact_bytes(lens, Hkv, d, B):
    """Algorithmic HBM bytes: scores read by select, idx written; compaction
    reads and writes min(B, N) rows of K and of V per KV head."""
    T = sum(lens)
    sel = Hkv * T * 4 + len(lens) * Hkv * B * 4
    rows = sum(min(B, N) for N in lens) * Hkv
    comp = 2 * 2 * rows * d * 2 + len(lens) * Hkv * B * 4
    return sel, comp


def mufu_peak_gexp(pk, sm_count):
    """MUFU ex2 peak in G exp/s: 16 per clock per SM x SMs x max SM clock."""
    return MUFU_EX2_PER_CLK_PER_SM * sm_count * float(pk.get("sm_max_mhz", 1965.0)) / 1e3


def rooflines(lens, Hq, Hkv, d, a, b, B, t_score_ms, t_sc_ms, layer_ms, pk, sm_count,
              traffic=None, peak_kind="measured"):
    """The headline roofline entry and the other views, from the work counts
    and the measured times (milliseconds).

    Scorer roofline (the larger of): both passes' QK^T FLOPs at the bf16
    tensor peak, one pass of exponentials at the MUFU peak, its algorithmic
    bytes at the HBM peak.  frac = roofline time / measured time, which is
    achieved / peak of the binding unit.  The whole layer adds select and
    compact's bytes at the HBM peak."""
    flops, logits = scorer_flops(lens, Hq, d, a, b)
    sbytes = scorer_bytes(lens, Hq, Hkv, d, a, b)
    sel_b, comp_b = select_compact_bytes(lens, Hkv, d, B)
    tflops = float(pk["bf16_tflops"])
    tflops_sus = float(pk.get("bf16_tflops_sustained", tflops))
    hbm = float(pk["hbm_gbs"])
    mufu = mufu_peak_gexp(pk, sm_count)                     # G exp/s
    terms = {"tensor": flops / (tflops * 1e12), "mufu": logits / (mufu * 1e9),
             "hbm": sbytes / (hbm * 1e9)}                   # seconds
    bound = max(terms, key=terms.get)
    t_roof = terms[bound]
    ts = t_score_ms / 1e3
    if bound == "tensor":
        ach, peak, unit, b_name = flops / ts / 1e12, tflops, "TFLOP/s", "tensor"
    elif bound == "mufu":
        ach, peak, unit, b_name = logits / ts / 1e9, mufu, "Gexp/s", "alu"
    else:
        ach, peak, unit, b_name = sbytes / ts / 1e9, hbm, "GB/s", "hbm"
    head = {"kernel": "scorer (waits_score: both passes)", "bound": b_name,
            "achieved": round(ach, 2), "peak": round(peak, 2), "unit": unit,
            "frac": round(ach / peak, 4), "traffic": traffic,
            "traffic_ratio": round(traffic / sbytes, 3) if traffic else None,
            "algorithmic_bytes": sbytes, "flops_per_launch": flops, "active_logits": logits,
            "roofline_us": round(t_roof * 1e6, 2), "launch_us": round(t_score_ms * 1e3, 2),
            "terms_us": {k: round(v * 1e6, 2) for k, v in terms.items()},
            "peak_kind": f"{peak_kind}: bf16_tflops (burst) / MUFU 16 ex2/clk/SM x {sm_count} "
                         f"SMs x max clock / hbm_gbs"}
    sc_b = sel_b + comp_b
    t_layer_roof = t_roof + sc_b / (hbm * 1e9)
    other = [
        {"kernel": "whole layer (scorer + select + compact), algorithmic",
         "bound": b_name, "roofline_us": round(t_layer_roof * 1e6, 2),
         "measured_us": round(layer_ms * 1e3, 2), "frac": round(t_layer_roof / (layer_ms / 1e3), 4)},
        {"kernel": "scorer, tensor view at the sustained bf16 peak", "bound": "tensor",
         "achieved": round(flops / ts / 1e12, 2), "peak": tflops_sus, "unit": "TFLOP/s",
         "frac": round(flops / ts / 1e12 / tflops_sus, 4)},
        {"kernel": "scorer, MUFU view of both passes' exponentials", "bound": "alu",
         "achieved": round(2 * logits / ts / 1e9, 1), "peak": round(mufu, 1), "unit": "Gexp/s",
         "frac": round(2 * logits / ts / 1e9 / mufu, 4)},
    ]
    if t_sc_ms:
        other.append({"kernel": "select+compact (waits_select_compact, one kernel)",
                      "bound": "hbm", "achieved": round(sc_b / (t_sc_ms / 1e3) / 1e9, 1),
                      "peak": hbm, "unit": "GB/s",
                      "frac": round(sc_b / (t_sc_ms / 1e3) / 1e9 / hbm, 4),
                      "bytes_per_launch": sc_b, "launch_us": round(t_sc_ms * 1e3, 2)})
    # Dense-equivalent view (every query row active): both passes' MMAs and
    # one pass of exponentials, plus select and compact's bytes.
    dense_logits = sum(n * (n + 1) // 2 for n in lens) * Hq
    t_dense = max(2 * 2 * d * dense_logits / (tflops * 1e12),
                  dense_logits / (mufu * 1e9)) + sc_b / (hbm * 1e9)
    other.append({"kernel": "whole layer, dense-equivalent work (every query row active)",
                  "bound": "tensor", "roofline_us": round(t_dense * 1e6, 2),
                  "measured_us": round(layer_ms * 1e3, 2),
                  "frac": round(t_dense / (layer_ms / 1e3), 4),
                  "note": "roofline time / measured time; overstates sparse-weight work"})
    return head, other


def code_only(text: str) -> str:
    """A C++/CUDA source without its comments and with whitespace runs
    collapsed: what the compiler sees of it (no string literal in the hashed
    files holds a comment marker)."""
    import re
    text = re.sub(r"/\*.*?\*/", " ", text, flags=re.S)
    text = re.sub(r"//[^\n]*", " ", text)
    return " ".join(text.split())


def scorer_source_hash() -> str:
    """sha256 of the sparse scorer's code (comments and layout left out), in
    PROFILED_SOURCES order: a comment-only edit keeps the profiled counters."""
    import hashlib
    h = hashlib.sha256()
    for name in PROFILED_SOURCES:
        with open(os.path.join(ROOT, "prefill_eviction_scoring_b200", "csrc", name)) as f:
            h.update(code_only(f.read()).encode())
            h.update(b"\0")
    return h.hexdigest()


def profiled_traffic(case: Case):
    """ncu DRAM bytes of the scorer for the headline layer, or None when the
    case differs or the scorer's sources have changed since the capture."""
    if (case.config, case.a, case.b) != ("llama8b", 1.0, 16) or case.name != "llama8b":
        return None
    ok = scorer_source_hash().startswith(PROFILED_SCORER["sha256_prefix"])
    return PROFILED_SCORER["dram_bytes"] if ok else None


def oracle_active_logits(N, a, b):
    """Logits the fp64 oracle visits for one sequence and query head: it
    skips the rows whose fp64 weight is exactly 0."""
    q = np.arange(N, dtype=np.float64)
    with np.errstate(over="ignore"):
        w = 1.0 / (1.0 + np.exp(-a * (q - (N - b - 0.5))))
    act = q[w != 0.0]
    return int(np.sum(act + 1))


def score_kernels(lib, shape, a, b):
    """Kernels one waits_score call enqueues (2, or 3 with the planner)."""
    n = ctypes.c_int32(0)
    _lib.check("waits_score_kernels", lib.waits_score_kernels(ctypes.byref(shape), a, b,
                                                              ctypes.byref(n)))
    return n.value


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            m = json.load(f)
        return m, "measured"
    except (OSError, ValueError):
        return FALLBACK_PEAKS, "fallback"


# ------------------------------------------------------------- plumbing ---
class Dist:
    """One process per GPU (torchrun environment).  ``backend="gloo"`` runs
    the same logic on CPU tensors (used by the multi-rank CPU tests)."""

    def __init__(self, backend: str = "nccl"):
        self.world = int(os.environ.get("WORLD_SIZE", "1"))
        self.rank = int(os.environ.get("RANK", "0"))
        self.local = int(os.environ.get("LOCAL_RANK", "0"))
        self.backend = backend
        self.pg = None

    @property
    def cuda(self) -> bool:
        return self.backend == "nccl"

    def device(self):
        return torch.device("cuda", self.local) if self.cuda else torch.device("cpu")

    def init(self):
        if self.cuda:
            torch.cuda.set_device(self.local)
        if self.world > 1:
            import torch.distributed as dist
            kw = {"device_id": self.device()} if self.cuda else {}
            dist.init_process_group(self.backend, timeout=datetime.timedelta(seconds=180), **kw)
            self.pg = dist

    def barrier(self):
        if self.cuda:
            torch.cuda.synchronize()
        if self.pg:
            self.pg.barrier()
        if self.cuda:
            torch.cuda.synchronize()

    def max(self, x: float) -> float:
        """Largest value over the ranks (every rank must call it)."""
        if not self.pg:
            return x
        t = torch.tensor([x], dtype=torch.float64, device=self.device())
        self.pg.all_reduce(t, op=self.pg.ReduceOp.MAX)
        return float(t.item())

    def close(self):
        if self.pg:
            self.pg.destroy_process_group()


class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
    NAMES = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")
    PERIOD_MS = 10

    def __init__(self, local_rank):
        vis = os.environ.get("CUDA_VISIBLE_DEVICES", "")
        ids = [v.strip() for v in vis.split(",") if v.strip()]
        self.gpu = ids[local_rank] if local_rank < len(ids) else str(local_rank)
        self.proc = None
        self.path = None

    def start(self):
        import tempfile
        fd, self.path = tempfile.mkstemp(prefix="waits_clocks_", suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", self.gpu, f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", str(self.PERIOD_MS)],
                stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None
        time.sleep(0.3)   # the first sample lands before the timed region starts

    def stop(self):
        if not self.proc:
            if self.path:
                try:
                    os.remove(self.path)
                except OSError:
                    pass
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        return self.parse(self.path, remove=True)

    @classmethod
    def parse(cls, path, remove=False):
        sm, mx, reasons, power = [], [], set(), []
        for line in open(path):
            parts = [x.strip() for x in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                mx.append(float(parts[2]))
                power.append(float(parts[3]))
            except ValueError:
                continue
            for name, v in zip(cls.NAMES, parts[5:9]):
                if v.lower() == "active":
                    reasons.add(name)
        if remove:
            try:
                os.remove(path)
            except OSError:
                pass
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(mx) if mx else None,
                "power_w_median": statistics.median(power) if power else None,
                "samples": len(sm), "period_ms": cls.PERIOD_MS, "reasons": sorted(reasons)}


class LayerCall:
    """Preallocated buffers for one layer and its C-ABI calls."""

    def __init__(self, lay, B, shape, workspace, ws_bytes):
        self.lay = lay
        T, Hq, d = lay.Q.shape
        Hkv = lay.K.shape[1]
        nseq = len(lay.lens)
        dev = lay.Q.device
        self.shape = shape
        self.ws, self.ws_bytes = workspace, ws_bytes
        self.scores = torch.empty((Hkv, T), dtype=torch.float32, device=dev)
        self.idx = torch.empty((nseq, Hkv, B), dtype=torch.int32, device=dev)
        self.kept = torch.empty((nseq,), dtype=torch.int32, device=dev)
        self.Ko = torch.empty((nseq, Hkv, B, d), dtype=torch.bfloat16, device=dev)
        self.Vo = torch.empty_like(self.Ko)
        self.B = B

    def score(self, lib, a, b, stream):
        return lib.waits_score(ctypes.byref(self.shape), self.lay.Q.data_ptr(),
                               self.lay.K.data_ptr(), a, b, self.scores.data_ptr(),
                               self.ws.data_ptr(), self.ws_bytes, stream)

    def select_compact(self, lib, R, stream):
        return lib.waits_select_compact(
            ctypes.byref(self.shape), self.scores.data_ptr(), self.lay.K.data_ptr(),
            self.lay.V.data_ptr(), R, self.B, self.idx.data_ptr(), self.kept.data_ptr(),
            self.Ko.data_ptr(), self.Vo.data_ptr(), self.ws.data_ptr(), self.ws_bytes, stream)


# --------------------------------------------------------- CPU baseline ---
def cpu_oracle_sample(lay, a, b, R, B, g=0, prefix=None):
    """Time the fp64 oracle on KV head g of one layer (its G query heads):
    score, select and compact, on the first ``prefix`` tokens of each
    sequence if given.  Returns (seconds, threads, logits visited)."""
    import oracle
    from threadpoolctl import threadpool_info
    Hq, Hkv = lay.Q.shape[1], lay.K.shape[1]
    G = Hq // Hkv
    lens = list(lay.lens)
    cu_full = lay.cu_seqlens.cpu().numpy()
    if prefix is not None:
        rows = np.concatenate([np.arange(cu_full[i], cu_full[i] + min(prefix, n))
                               for i, n in enumerate(lens)]) if lens else np.zeros(0, int)
        lens = [min(prefix, n) for n in lens]
    else:
        rows = np.arange(int(cu_full[-1]))
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    rt = torch.as_tensor(rows, device=lay.Q.device)
    Qn = wl.to_numpy64(lay.Q[rt][:, g * G:(g + 1) * G])
    Kn = wl.to_numpy64(lay.K[rt][:, g:g + 1])
    Kb, Vb = wl.to_bits(lay.K[rt][:, g:g + 1]), wl.to_bits(lay.V[rt][:, g:g + 1])
    t0 = time.perf_counter()
    s = oracle.score(Qn, Kn, cu, a, b)
    idx, kept = oracle.select(s, cu, R, B)
    oracle.compact(Kb, Vb, cu, idx, kept, B)
    dt = time.perf_counter() - t0
    threads = max([i.get("num_threads", 1) for i in threadpool_info()] or [1])
    return dt, threads, sum(oracle_active_logits(n, a, b) for n in lens) * G


def oracle_prefix(lens, a, b, G, budget_logits=2.5e9):
    """Longest common prefix length whose fp64-visited logits (one KV head)
    stay under ``budget_logits`` (about 10-20 s of the oracle on the box's
    cores); None when the whole sequences fit."""
    full = sum(oracle_active_logits(n, a, b) for n in lens) * G
    if full <= budget_logits:
        return None
    lo, hi = 1, max(lens)
    while lo < hi:
        mid = (lo + hi + 1) // 2
        if sum(oracle_active_logits(min(mid, n), a, b) for n in lens) * G <= budget_logits:
            lo = mid
        else:
            hi = mid - 1
    return lo


def cpu_baseline(lay, case: Case, time_budget_s=10.0):
    """The oracle, as it stands, on KV heads of layer 0 until ~time_budget_s
    of work; sequences longer than the oracle can finish in that time are
    cut to a prefix and the time scaled by the fp64-visited logits."""
    Hq, Hkv = lay.Q.shape[1], lay.K.shape[1]
    G = Hq // Hkv
    full_logits = sum(oracle_active_logits(n, case.a, case.b) for n in lay.lens) * G
    prefix = oracle_prefix(lay.lens, case.a, case.b, G)
    dt, heads, threads, logits = 0.0, 0, 1, 0
    while heads < Hkv and dt < time_budget_s:
        t, threads, lg = cpu_oracle_sample(lay, case.a, case.b, case.R, case.B, g=heads,
                                           prefix=prefix)
        dt += t
        logits += lg
        heads += 1
    # seconds for the whole layer: the sample's seconds per visited logit
    # times the layer's visited logits
    per_layer = dt / logits * full_logits * Hkv if logits else dt * Hkv / max(heads, 1)
    what = (f"first {prefix} tokens of each sequence, " if prefix else "")
    return {"value": sum(lay.lens) / per_layer, "unit": UNIT, "cores": threads, "kind": "oracle",
            "sample": f"fp64 numpy oracle (score+select+compact) on {heads} of the {Hkv} KV heads "
                      f"of layer 0 ({what}each with its {G} query heads), {dt:.2f} s; scaled to a "
                      f"whole layer by the logits the oracle visits (rows with fp64 weight != 0)",
            "seconds_measured": round(dt, 3)}


def config_dict(case: Case, lens, spec, L, flushed):
    l2 = ("inputs larger than L2: each layer has its own tensors, a step walks all layers, "
          "so every layer starts L2-cold" if not flushed else
          "L2 flushed between timed steps (a 256 MiB buffer written outside the events)")
    nseq = len(lens)
    seq = f"N={lens[0]}" if nseq == 1 else f"{nseq} sequences, N in [{min(lens)}, {max(lens)}]"
    hh = spec.heavy_hitters if case.config != "ragged" else 0
    return {"workload": f"{case.name}: {L} layer{'s' if L > 1 else ''} x {seq}, "
                        f"Hq={spec.num_q_heads}/Hkv={spec.num_kv_heads}, d={spec.head_dim}, "
                        f"a={case.a}, b={case.b}, R={case.R}, B={case.B}"
                        + (f"; sink + {hh} heavy hitters per KV head" if hh else
                           ("; sink" if spec.sink else "")),
            "layers_per_gpu": L, "seq_len": max(lens), "batch": nseq, "total_tokens": sum(lens),
            "num_q_heads": spec.num_q_heads, "num_kv_heads": spec.num_kv_heads,
            "head_dim": spec.head_dim, "sigmoid_a": case.a, "window": case.b,
            "recent_budget": case.R, "budget": case.B, "l2": l2,
            "parallelism": f"weak: {L}-layer stack per GPU, no collective"}


# ------------------------------------------------------------------ ours ---
def run_heads_case(args, D, lib, case: Case):
    """Every rank compresses its contiguous share of the KV heads of the same
    layers (waits_compress_heads, in place); value = the layers' tokens per
    second of the slowest rank (strong scaling)."""
    dev = torch.device("cuda", D.local)
    spec = wl.CONFIGS[case.config]
    L, a, b, R, B = case.layers, case.a, case.b, case.R, case.B
    layers = [wl.make_layer(case.config, layer=i, device=dev) for i in range(L)]
    lay0 = layers[0]
    T, Hq, d = lay0.Q.shape
    Hkv = lay0.K.shape[1]
    g0, g1 = head_shard(D.rank, D.world, Hkv)
    Hs, nseq = g1 - g0, len(lay0.lens)
    shape = api.make_shape(lay0.cu_seqlens, T, lay0.max_seqlen, Hq, Hkv, d)
    ws_bytes = api.workspace_bytes(shape)
    ws = torch.empty(ws_bytes, dtype=torch.uint8, device=dev)
    scores = torch.empty((max(Hs, 1), T), dtype=torch.float32, device=dev)
    idx = torch.empty((nseq, max(Hs, 1), B), dtype=torch.int32, device=dev)
    kept = torch.empty((nseq,), dtype=torch.int32, device=dev)
    Ko = torch.empty((nseq, max(Hs, 1), B, d), dtype=torch.bfloat16, device=dev)
    Vo = torch.empty_like(Ko)
    sp = ctypes.c_void_p(torch.cuda.current_stream(dev).cuda_stream)

    def step():
        if Hs == 0:
            return
        for l in layers:
            _lib.check("waits_compress_heads", lib.waits_compress_heads(
                ctypes.byref(shape), g0, g1, l.Q.data_ptr(), l.K.data_ptr(), l.V.data_ptr(), a,
                b, R, B, scores.data_ptr(), idx.data_ptr(), kept.data_ptr(), Ko.data_ptr(),
                Vo.data_ptr(), ws.data_ptr(), ws_bytes, sp))

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    clocks = ClockSampler(D.local)
    D.barrier()
    clocks.start()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(args.steps):
        step()
    e1.record()
    torch.cuda.synchronize()
    clk = clocks.stop()
    D.barrier()
    ms = D.max(e0.elapsed_time(e1) / args.steps)
    if D.rank == 0:
        pk, pk_kind = peaks()
        sm_count = torch.cuda.get_device_properties(dev).multi_processor_count
        # the slowest rank against its own share of the work (the whole
        # layer's work split over the ranks that own heads)
        owners = min(D.world, Hkv)
        _, other = rooflines(lay0.lens, Hq, Hkv, d, a, b, B, ms / L, 0.0, ms / L, pk, sm_count,
                             peak_kind=pk_kind)
        layer_roof = dict(other[0])
        layer_roof["roofline_us"] = round(layer_roof["roofline_us"] / owners, 2)
        layer_roof["frac"] = round(layer_roof["roofline_us"] / (ms / L * 1e3), 4)
        cfg = config_dict(case, lay0.lens, spec, L, False)
        cfg["parallelism"] = f"heads: {D.world} ranks split the {Hkv} KV heads of every layer"
        out = {"metric": METRIC, "value": L * sum(lay0.lens) / (ms / 1e3), "unit": UNIT,
               "n_gpus": D.world, "steps": args.steps, "warmup": args.warmup,
               "ms_per_step": ms, "higher_is_better": True, "scaling": "strong",
               "vs_baseline": None, "dtype": "bf16", "data": "synthetic", "config": cfg,
               "roofline": layer_roof, "clocks": clk,
               "gpu_launches": (score_kernels(lib, shape, a, b) + KERNELS_OUTSIDE_SCORE) * L *
               args.steps, "per_layer_us": {"layer": round(ms / L * 1e3, 2)}}
        print(json.dumps(out), flush=True)


def run_case(args, D, lib, case: Case, headline: bool):
    dev = torch.device("cuda", D.local)
    spec = wl.CONFIGS[case.config]
    L = case.layers
    a, b, R, B = case.a, case.b, case.R, case.B
    layers = [wl.make_layer(case.config, layer=i, device=dev)
              for i in wl.split_layers(L, D.world, D.rank)]
    lay0 = layers[0]
    T, Hq, d = lay0.Q.shape
    Hkv = lay0.K.shape[1]
    shape = api.make_shape(lay0.cu_seqlens, T, lay0.max_seqlen, Hq, Hkv, d)
    ws_bytes = api.workspace_bytes(shape)
    ws = torch.empty(ws_bytes, dtype=torch.uint8, device=dev)
    calls = [LayerCall(l, B, api.make_shape(l.cu_seqlens, T, l.max_seqlen, Hq, Hkv, d), ws,
                       ws_bytes) for l in layers]
    stream = torch.cuda.current_stream(dev)
    sp = ctypes.c_void_p(stream.cuda_stream)
    in_bytes = sum(l.Q.numel() * 2 + 2 * l.K.numel() * 2 for l in layers)
    flush = in_bytes < 3 * L2_BYTES
    scratch = torch.empty(256 << 20, dtype=torch.uint8, device=dev) if flush else None
    every = EVENT_EVERY if L >= EVENT_EVERY else 1

    def step(evs=None, which="all"):
        """One pass of the path over every layer.  Events (if given) are
        recorded around the scorer call of every `every`-th layer, and with
        which="all" around every call; an event between two calls stops the
        next kernel from starting early, so with which="score" only a sample
        of the scorer calls is bracketed."""
        for i, c in enumerate(calls):
            timed = evs is not None and (which == "all" or i % every == 0)
            if timed:
                evs[i][0].record(stream)
            _lib.check("waits_score", c.score(lib, a, b, sp))
            if timed:
                evs[i][1].record(stream)
            _lib.check("waits_select_compact", c.select_compact(lib, R, sp))
            if evs is not None and which == "all":
                evs[i][2].record(stream)

    def new_events(k):
        return [[[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in calls]
                for _ in range(k)]

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    st = ctypes.c_uint32(0)
    _lib.check("status", lib.waits_read_device_status(ws.data_ptr(), ws_bytes, sp, ctypes.byref(st)))
    if st.value:
        raise RuntimeError(f"device status {st.value:#x} after warm-up")

    K = args.steps
    in_region = args.kernel_events == "score" and not flush
    evs = new_events(K) if in_region else None
    clocks = ClockSampler(D.local)
    D.barrier()
    clocks.start()
    if not flush:
        # inputs far larger than L2: one bracket around all K steps
        t0e, t1e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        t0e.record(stream)
        for k in range(K):
            step(evs[k] if in_region else None, "score")
        t1e.record(stream)
        torch.cuda.synchronize()
        ms = t0e.elapsed_time(t1e) / K
        timing = "mean over K steps of one CUDA-event bracket around all of them"
    else:
        # small inputs: L2 flushed before every step, outside its events
        pairs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
                 for _ in range(K)]
        for k in range(K):
            scratch.fill_(k & 0xFF)
            pairs[k][0].record(stream)
            step()
            pairs[k][1].record(stream)
        torch.cuda.synchronize()
        ms = statistics.mean(e0.elapsed_time(e1) for e0, e1 in pairs)
        timing = "mean over K steps of CUDA events around each step (L2 flushed between)"
    clk = clocks.stop()
    D.barrier()
    ms = D.max(ms)
    if in_region:
        t_score = D.max(statistics.mean(e[0].elapsed_time(e[1]) for s_ in evs
                                        for i, e in enumerate(s_) if i % every == 0))

    # per-kernel durations: a few more steps with events around every call
    # (outside the timed region; they cut the overlap of calls)
    KS = min(K, 5)
    evs2 = new_events(KS)
    D.barrier()
    for k in range(KS):
        if flush:
            scratch.fill_(k & 0xFF)
        step(evs2[k], "all")
    torch.cuda.synchronize()
    D.barrier()
    if not in_region:
        t_score = D.max(statistics.mean(e[0].elapsed_time(e[1]) for s_ in evs2 for e in s_))
    t_sc = D.max(statistics.mean(e[1].elapsed_time(e[2]) for s_ in evs2 for e in s_))

    tokens_per_step = D.world * L * sum(lay0.lens)
    value = tokens_per_step / (ms / 1e3)
    pk, pk_kind = peaks()
    sm_count = torch.cuda.get_device_properties(dev).multi_processor_count
    roof, other = rooflines(lay0.lens, Hq, Hkv, d, a, b, B, t_score, t_sc, ms / L, pk,
                            sm_count, traffic=profiled_traffic(case), peak_kind=pk_kind)
    roof["timing"] = (f"CUDA events around the waits_score call of every {every}th layer in the "
                      "timed region" if in_region else
                      "CUDA events around waits_score in 5 steps after the timed region")

    # ---- end to end through the host-buffer entry point.  Layers are
    # independent calls: they alternate between two streams, each with its
    # own staging buffers, so one layer's copies to the device overlap the
    # other's kernels and copies back.
    E = min(args.e2e_layers, L)
    NS = 2 if E > 1 else 1
    e2e_streams = [torch.cuda.Stream(dev) for _ in range(NS)]
    hcs = [api.HostCompressor(lay0.cu_seqlens.cpu(), Hq, Hkv, d, B, device=dev)
           for _ in range(NS)]
    host = [tuple(t.cpu().pin_memory() for t in (l.Q, l.K, l.V)) for l in layers[:E]]
    for k in range(NS):
        with torch.cuda.stream(e2e_streams[k]):
            hcs[k](*host[0], a, b, R)
    torch.cuda.synchronize()
    D.barrier()
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    t0.record(stream)
    for es in e2e_streams:
        es.wait_event(t0)
    for _ in range(args.e2e_steps):
        for i, hq in enumerate(host):
            with torch.cuda.stream(e2e_streams[i % NS]):
                hcs[i % NS](*hq, a, b, R)
    for es in e2e_streams:
        stream.wait_stream(es)
    t1.record(stream)
    torch.cuda.synchronize()
    e2e_ms = D.max(t0.elapsed_time(t1)) / args.e2e_steps
    e2e = {"value": D.world * E * sum(lay0.lens) / (e2e_ms / 1e3), "unit": UNIT,
           "h2d_bytes_per_step": hcs[0].h2d_bytes * E, "d2h_bytes_per_step": hcs[0].d2h_bytes * E,
           "step": f"{E} layer{'s' if E > 1 else ''} through waits_compress_host (pinned host "
                   f"buffers; the kept V rows are read in place over the bus)"
                   + (f", alternating over {NS} streams" if NS > 1 else ""),
           "ms_per_step": round(e2e_ms, 3)}
    # the host link carries every input and output byte of the step: its rate
    # says how much of the step the transfers alone account for
    e2e["host_link_gbs"] = round((e2e["h2d_bytes_per_step"] + e2e["d2h_bytes_per_step"])
                                 / (e2e_ms / 1e3) / 1e9, 1)
    e2e["note"] = ("bound by the host link, not the kernels: each step moves "
                   f"{(e2e['h2d_bytes_per_step'] + e2e['d2h_bytes_per_step']) / 1e6:.0f} MB "
                   f"at {e2e['host_link_gbs']} GB/s; the device-resident line is `value`")

    cpu = None
    if D.rank == 0 and D.world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(lay0, case)

    out = None
    if D.rank == 0:
        out = {"metric": METRIC, "value": value, "unit": UNIT, "n_gpus": D.world, "steps": K,
               "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True,
               "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
               "config": config_dict(case, lay0.lens, spec, L, flush),
               "roofline": roof, "roofline_other": other, "cpu_baseline": cpu, "e2e": e2e,
               "gpu_launches": (score_kernels(lib, shape, a, b) + KERNELS_OUTSIDE_SCORE) * L * K,
               "clocks": clk, "timing": timing,
               "per_layer_us": {"score": round(t_score * 1e3, 2),
                                "select+compact": round(t_sc * 1e3, 2),
                                "layer": round(ms / L * 1e3, 2)}}
        if not headline:
            out["metric"] = METRIC.replace("(8B shape, N=32K)", f"({case.name})")
        print(json.dumps(out), flush=True)
    del layers, calls, hcs, host, scratch
    torch.cuda.empty_cache()
    return out


def selected_cases(args):
    if args.config == "all":
        out = []
        for c in ALL_CONFIGS:
            out += cases_for(c, None, None if c != "llama8b" else args.layers) if c != "llama8b" \
                else [x for B in (128, 512, 2048) for x in cases_for(c, B, args.layers)]
        return out
    if args.config == "llama8b" and args.budget is None:
        return cases_for("llama8b", 2048, args.layers)
    return cases_for(args.config, args.budget, args.layers)


def run_ours(args):
    D = Dist()
    D.init()
    lib = _lib.load()
    for case in selected_cases(args):
        if args.parallel == "heads":
            run_heads_case(args, D, lib, case)
            continue
        headline = (case.name == "llama8b" and case.B == 2048 and args.config == "llama8b")
        run_case(args, D, lib, case, headline)
    D.close()


# ------------------------------------------------------------- reference ---
def run_reference(args):
    """The oracle (the pages ship no implementation to install) timed as it
    stands on the host cores, one KV head of layer 0 per step; rank 0 only."""
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    if rank != 0:
        return
    for case in selected_cases(args):
        spec = wl.CONFIGS[case.config]
        dev = "cuda" if torch.cuda.is_available() else "cpu"
        lay = wl.make_layer(case.config, layer=0, device=dev)
        Hq, Hkv = lay.Q.shape[1], lay.K.shape[1]
        G = Hq // Hkv
        prefix = oracle_prefix(lay.lens, case.a, case.b, G)
        full_logits = sum(oracle_active_logits(n, case.a, case.b) for n in lay.lens) * G
        times, threads, logits = [], 1, 0
        for k in range(args.warmup + args.steps):
            dt, threads, lg = cpu_oracle_sample(lay, case.a, case.b, case.R, case.B, g=k % Hkv,
                                                prefix=prefix)
            if k >= args.warmup:
                times.append(dt)
                logits = lg
        step_s = statistics.mean(times)
        per_layer = step_s / logits * full_logits * Hkv
        value = sum(lay.lens) / per_layer
        sample = (f"each step: the fp64 numpy oracle (score+select+compact) on one KV head of "
                  f"layer 0 ({'first %d tokens of each sequence, ' % prefix if prefix else ''}"
                  f"its {G} query heads); value = tokens of a whole layer / (step time x {Hkv} "
                  f"KV heads" + (" x the visited-logit ratio of the full sequences" if prefix
                                 else "") + ")")
        out = {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT,
               "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
               "ms_per_step": step_s * 1e3, "higher_is_better": True, "scaling": "weak",
               "vs_baseline": None, "dtype": "f64", "data": "synthetic",
               "config": config_dict(case, lay.lens, spec, case.layers, False),
               "layer_scaling": {"kv_heads_per_layer": Hkv,
                                 "seconds_per_layer": round(per_layer, 3)},
               "cpu_baseline": {"value": value, "unit": UNIT, "cores": threads, "kind": "oracle",
                                "sample": sample},
               "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0,
                       "d2h_bytes_per_step": 0}}
        if case.name != "llama8b":
            out["metric"] = METRIC.replace("(8B shape, N=32K)", f"({case.name})")
        print(json.dumps(out), flush=True)


def main():
    args = parse()
    if args.warmup < 3 and args.impl == "ours":
        print("warning: fewer than 3 warm-up steps", file=sys.stderr)
    if args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
