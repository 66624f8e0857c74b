"""Seeded synthetic inputs for the WAITS prefill path.

This module only draws and shapes inputs; it holds none of the scoring,
selection or compaction arithmetic, and it is the one piece of code that both
the CUDA path (tests, bench) and the fp64 oracle consume.

The WAITS README (stig.sh/Dirac-Notation/A2SF, Evaluation and Repository
layout) evaluates on LongBench, needle-in-a-haystack and RULER prompts with
Llama-3.2-1B, Llama-3.1-8B, Qwen-2.5-7B and Mistral-7B.  No dataset or model
weight is used here: model-shaped Q/K/V are drawn i.i.d. N(0, 1) and rounded
to bf16, with two structures that real prompts have --

* an attention sink: the key at position 0 of every sequence has 8x norm;
* heavy hitters: chosen keys are rotated to cosine 0.5 with a random query
  that can see them, so a few positions attract far more attention mass.

Seeds: ``1_000_000 * config_number + 1000 * layer + {Q: 0, K: 1, V: 2,
heavy hitters: 3}``; ragged lengths use ``1_000_000 * config_number``.
On CUDA the generator is torch's Philox, on CPU torch's MT19937, so a given
seed gives different (but reproducible) tensors per device; every test and
bench copies the device tensors to the host for the oracle, so both sides
always read the same bits.
"""

from __future__ import annotations

import dataclasses
import math
from typing import List, Optional, Sequence, Tuple

import torch

# (a, b) actions named by the WAITS README ("Training the routing policy":
# --actions "0:1,0.01:128,1:16,10:1,10:16").
WAITS_ACTIONS: Tuple[Tuple[float, int], ...] = (
    (0.0, 1), (0.01, 128), (1.0, 16), (10.0, 1), (10.0, 16))


@dataclasses.dataclass(frozen=True)
class ConfigSpec:
    name: str
    number: int                 # 1-based, used in the seed formula
    lens: Tuple[int, ...]       # per-sequence prompt lengths (ragged: drawn)
    num_q_heads: int
    num_kv_heads: int
    head_dim: int
    sink: bool
    heavy_hitters: int          # per KV head, per sequence
    recent: int                 # R
    budgets: Tuple[int, ...]    # B values
    actions: Tuple[Tuple[float, int], ...]   # (a, b)
    layers: int = 1
    description: str = ""


def ragged_lengths(n: int, lo: int, hi: int, seed: int) -> Tuple[int, ...]:
    g = torch.Generator(device="cpu")
    g.manual_seed(seed)
    return tuple(int(x) for x in torch.randint(lo, hi + 1, (n,), generator=g))


CONFIGS = {
    "tiny": ConfigSpec(
        "tiny", 1, (512,), 4, 1, 64, False, 0, 16, (128,),
        ((1.0, 16), (0.0, 16), (1e4, 1)), 1,
        "1 layer, N=512, 4 query heads on 1 KV head, d=64, i.i.d. N(0,1)"),
    "llama1b": ConfigSpec(
        "llama1b", 2, (4096,), 32, 8, 64, True, 0, 16, (128,),
        WAITS_ACTIONS, 1,
        "Llama-3.2-1B-shaped layer, N=4096, 32/8 heads, d=64, sink"),
    "llama8b": ConfigSpec(
        "llama8b", 3, (32768,), 32, 8, 128, True, 64, 16, (128, 512, 2048),
        ((1.0, 16),), 32,
        "Llama-3.1-8B-shaped stack, 32 layers, N=32768, 32/8 heads, d=128, "
        "sink + 64 heavy hitters per KV head"),
    "ragged": ConfigSpec(
        "ragged", 4, ragged_lengths(8, 4096, 16384, 4_000_000), 28, 4, 128,
        True, 0, 16, (1024,), ((10.0, 16),), 1,
        "Qwen-2.5-7B-shaped layer, 8 sequences N~U[4096,16384], 28/4 heads, "
        "d=128, sink, packed varlen"),
    "long": ConfigSpec(
        "long", 5, (131072,), 32, 8, 128, True, 256, 64, (2048,),
        ((0.01, 128),), 1,
        "Mistral-7B-shaped layer, N=131072, 32/8 heads, d=128, "
        "sink + 256 heavy hitters per KV head"),
}


@dataclasses.dataclass
class Layer:
    """One layer's packed inputs (bf16 Q/K/V, int32 cu_seqlens)."""
    Q: torch.Tensor            # [T, Hq, d] bf16
    K: torch.Tensor            # [T, Hkv, d] bf16
    V: torch.Tensor            # [T, Hkv, d] bf16
    cu_seqlens: torch.Tensor   # [nseq + 1] int32, same device
    lens: Tuple[int, ...]
    heavy: list = dataclasses.field(default_factory=list)

    @property
    def total_tokens(self) -> int:
        return int(sum(self.lens))

    @property
    def max_seqlen(self) -> int:
        return int(max(self.lens)) if self.lens else 0


def _gen(device, seed):
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    return g


def _plant_heavy_hitters(Qf, Kf, lo, N, G, n_heavy, recent, gen):
    """Rotate n_heavy keys per KV head to cosine 0.5 with a visible query."""
    T, Hkv, d = Kf.shape
    hi_pos = N - recent
    planted = []
    if n_heavy <= 0 or hi_pos <= 1:
        return planted
    n_heavy = min(n_heavy, hi_pos - 1)
    dev = Kf.device
    for g in range(Hkv):
        p = torch.randperm(hi_pos - 1, generator=gen, device=dev)[:n_heavy] + 1
        h = g * G + torch.randint(0, G, (n_heavy,), generator=gen, device=dev)
        u01 = torch.rand((n_heavy,), generator=gen, device=dev,
                         dtype=torch.float64)
        qr = p + torch.floor(u01 * (N - p).to(torch.float64)).to(torch.int64)
        qr = torch.minimum(qr, torch.full_like(qr, N - 1))
        u = Qf[lo + qr, h, :]
        u = u / u.norm(dim=-1, keepdim=True)
        v = torch.randn((n_heavy, d), generator=gen, device=dev)
        v = v - (v * u).sum(-1, keepdim=True) * u
        v = v / v.norm(dim=-1, keepdim=True)
        norm = Kf[lo + p, g, :].norm(dim=-1, keepdim=True)
        Kf[lo + p, g, :] = norm * (0.5 * u + (math.sqrt(3.0) / 2.0) * v)
        planted.append((g, p, h, qr))
    return planted


def make_layer(config: str, layer: int = 0, device="cpu",
               lens: Optional[Sequence[int]] = None,
               heads: Optional[Tuple[int, int]] = None,
               head_dim: Optional[int] = None,
               heavy_hitters: Optional[int] = None,
               sink: Optional[bool] = None) -> Layer:
    """Draw one layer of ``config``; keyword overrides give smaller variants
    of the same recipe (e.g. shorter ``lens``) for parity tests."""
    spec = CONFIGS[config]
    lens = tuple(int(n) for n in (spec.lens if lens is None else lens))
    Hq, Hkv = (spec.num_q_heads, spec.num_kv_heads) if heads is None else heads
    d = spec.head_dim if head_dim is None else head_dim
    n_heavy = spec.heavy_hitters if heavy_hitters is None else heavy_hitters
    use_sink = spec.sink if sink is None else sink
    G = Hq // Hkv
    T = sum(lens)
    base = 1_000_000 * spec.number + 1000 * layer
    Qf = torch.randn((T, Hq, d), generator=_gen(device, base + 0),
                     device=device)
    Q = Qf.to(torch.bfloat16)
    Kf = torch.randn((T, Hkv, d), generator=_gen(device, base + 1),
                     device=device)
    V = torch.randn((T, Hkv, d), generator=_gen(device, base + 2),
                    device=device).to(torch.bfloat16)
    cu = [0]
    for n in lens:
        cu.append(cu[-1] + n)
    gh = _gen(device, base + 3)
    Qr = Q.float()
    heavy = []
    for i, n in enumerate(lens):
        lo = cu[i]
        if n == 0:
            continue
        if use_sink:
            Kf[lo] *= 8.0
        for g, p, h, qr in _plant_heavy_hitters(Qr, Kf, lo, n, G, n_heavy,
                                                spec.recent, gh):
            heavy.append((i, g, p, h, qr))
    K = Kf.to(torch.bfloat16)
    cu_t = torch.tensor(cu, dtype=torch.int32, device=device)
    return Layer(Q, K, V, cu_t, lens, heavy)


def random_layer(lens: Sequence[int], Hq: int, Hkv: int, d: int, seed: int,
                 device="cpu", scale: float = 1.0) -> Layer:
    """Plain i.i.d. N(0, scale^2) bf16 layer for edge-case tests."""
    T = int(sum(lens))
    g = _gen(device, seed)
    Q = (scale * torch.randn((T, Hq, d), generator=g, device=device)).to(
        torch.bfloat16)
    K = (scale * torch.randn((T, Hkv, d), generator=g, device=device)).to(
        torch.bfloat16)
    V = torch.randn((T, Hkv, d), generator=g, device=device).to(
        torch.bfloat16)
    cu = [0]
    for n in lens:
        cu.append(cu[-1] + int(n))
    return Layer(Q, K, V, torch.tensor(cu, dtype=torch.int32, device=device),
                 tuple(int(n) for n in lens))


def to_numpy64(t: torch.Tensor):
    """Exact fp64 copy of a bf16 tensor (for the oracle)."""
    return t.detach().to("cpu").to(torch.float64).numpy()


def to_bits(t: torch.Tensor):
    """Raw 16-bit patterns of a bf16 tensor (for bit-exact comparisons)."""
    return t.detach().to("cpu").view(torch.int16).numpy()


def split_layers(n_layers: int, world_size: int, rank: int) -> List[int]:
    """Contiguous block of layer indices owned by ``rank`` (weak scaling:
    every rank owns ``n_layers`` layers of its own, seeded by global index)."""
    return [rank * n_layers + i for i in range(n_layers)]
