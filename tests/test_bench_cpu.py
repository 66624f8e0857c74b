"""The bench's algorithmic work counts (the roofline numerators), against
brute force over the causal mask and the fp32 active-row predicate."""

import os
import sys

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402


def _brute_logits(N, a, b):
    q = np.arange(N, dtype=np.float32)
    c = np.float32(N) - np.float32(b) - np.float32(0.5)
    with np.errstate(over="ignore"):
        w = np.float32(1.0) / (np.float32(1.0) + np.exp(np.float32(-a) * (q - c)))
    active = w != 0
    causal = np.tril(np.ones((N, N), dtype=bool))          # key k <= query q
    return int(causal[active].sum())


@pytest.mark.parametrize("N,a,b", [(300, 1.0, 16), (257, 0.0, 16), (400, 10.0, 1),
                                   (128, 1e4, 1), (1000, 0.01, 128), (90, 1.0, 200)])
def test_scorer_logits_brute_force(N, a, b):
    Hq, d = 4, 64
    flops, logits = bench.scorer_flops([N], Hq, d, a, b)
    want = _brute_logits(N, a, b)
    assert logits == Hq * want
    assert flops == 2 * 2 * d * Hq * want


def test_headline_active_logits():
    # 105 active rows per head at N = 32768, a = 1, b = 16: keys 32664..32768 per row
    _, logits = bench.scorer_flops([32768], 32, 128, 1.0, 16)
    assert bench.first_active_row(32768, 1.0, 16) == 32768 - 105
    assert logits == 32 * 105 * (32664 + 32768) // 2


def test_select_compact_bytes():
    sel, comp = bench.select_compact_bytes([100, 5000], 2, 128, 1024)
    assert sel == 2 * 5100 * 4 + 2 * 2 * 1024 * 4
    assert comp == 2 * 2 * (100 + 1024) * 2 * 128 * 2 + 2 * 2 * 1024 * 4
