"""Plant plausible mistakes in copies of the oracle (on the CPU) and check
that the pin suite catches every one of them."""

import numpy as np
import pytest

import oracle
import pins


def _no_scale(Q, K, cu, a, b):
    return oracle.score(np.asarray(Q) * np.sqrt(np.asarray(Q).shape[2]), K, cu, a, b)


def _neg_slope(Q, K, cu, a, b):
    return oracle.score(Q, K, cu, -a, b)


def _centre_plus_one(Q, K, cu, a, b):
    return oracle.score(Q, K, cu, a, b + 1)


def _centre_no_half(Q, K, cu, a, b):
    return oracle.score(Q, K, cu, a, b - 0.5)


def _gqa_modulo(Q, K, cu, a, b):
    """Query head h wrongly paired with KV head h % Hkv."""
    Q = np.asarray(Q)
    Hq, Hkv = Q.shape[1], np.asarray(K).shape[1]
    G = Hq // Hkv
    perm = [j * Hkv + g for g in range(Hkv) for j in range(G)]
    return oracle.score(Q[:, perm], K, cu, a, b)


def _mean_over_heads(Q, K, cu, a, b):
    G = np.asarray(Q).shape[1] // np.asarray(K).shape[1]
    return oracle.score(Q, K, cu, a, b) / G


def _weight_on_columns(Q, K, cu, a, b):
    """w applied to the key index instead of the query row."""
    s1 = oracle.score(Q, K, cu, 0.0, b) * 2.0
    out = np.zeros_like(s1)
    for i in range(len(cu) - 1):
        lo, hi = int(cu[i]), int(cu[i + 1])
        out[:, lo:hi] = s1[:, lo:hi] * oracle.forgetting_curve(
            np.arange(hi - lo), hi - lo, a, b)[None, :]
    return out


def _plain_python(Q, K, cu, a, b, causal=True, row_norm=True):
    Q = np.asarray(Q, np.float64)
    K = np.asarray(K, np.float64)
    T, Hq, d = Q.shape
    Hkv = K.shape[1]
    G = Hq // Hkv
    s = np.zeros((Hkv, T))
    for i in range(len(cu) - 1):
        lo, hi = int(cu[i]), int(cu[i + 1])
        N = hi - lo
        if N == 0:
            continue
        w = oracle.forgetting_curve(np.arange(N), N, a, b)
        for h in range(Hq):
            L = Q[lo:hi, h] @ K[lo:hi, h // G].T / np.sqrt(d)
            if causal:
                L = np.where(np.tril(np.ones((N, N), bool)), L, -np.inf)
            ax = 1 if row_norm else 0
            E = np.exp(L - L.max(axis=ax, keepdims=True))
            P = E / E.sum(axis=ax, keepdims=True)
            s[h // G, lo:hi] += (w[:, None] * P).sum(axis=0)
    return s


def _non_causal(Q, K, cu, a, b):
    return _plain_python(Q, K, cu, a, b, causal=False)


def _column_softmax(Q, K, cu, a, b):
    """Softmax normalised over queries (a transposed operand)."""
    return _plain_python(Q, K, cu, a, b, row_norm=False)


MUTANTS = [_no_scale, _neg_slope, _centre_plus_one, _centre_no_half,
           _gqa_modulo, _mean_over_heads, _weight_on_columns, _non_causal,
           _column_softmax]


def test_reference_restatement_passes():
    """The plain-loop restatement used to build two mutants is itself right,
    so those mutants differ from the oracle only by the planted mistake."""
    for pin in pins.ALL_PINS:
        pin(_plain_python)


@pytest.mark.parametrize("mutant", MUTANTS, ids=lambda f: f.__name__)
def test_mutant_is_caught(mutant):
    caught = []
    for pin in pins.ALL_PINS:
        try:
            pin(mutant)
        except AssertionError:
            caught.append(pin.__name__)
    assert caught, f"no pin catches {mutant.__name__}"
