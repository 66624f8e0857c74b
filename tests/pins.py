"""Checks that pin a WAITS score function to facts outside itself.

Each ``pin_*`` takes a score function with the oracle's signature
``fn(Q, K, cu_seqlens, a, b) -> s[Hkv, T]`` and raises AssertionError when the
function disagrees with: 40-digit decimal brute force; a closed form; an
exact tie pattern; the H2O/TOVA/SnapKV limits named in the WAITS README
opening summary (computed here with scipy's softmax); or an identity of the
definition.  ``tests/test_oracle_pins.py`` runs them on the oracle and
``tests/test_oracle_mutants.py`` shows each planted mistake trips one.
"""

from fractions import Fraction

import numpy as np
from scipy.special import softmax

from brute_decimal import brute_scores


def _rand(shape, seed, scale=1.0):
    rng = np.random.default_rng(seed)
    x = rng.standard_normal(shape) * scale
    # round to values exactly representable in bf16 (8 significant bits)
    m, e = np.frexp(x)
    return np.ldexp(np.round(m * 256.0) / 256.0, e)


def _cu(lens):
    return np.concatenate([[0], np.cumsum(lens)]).astype(np.int64)


BRUTE_CASES = [
    # (lens, Hq, Hkv, d, a, b)
    ((6,), 4, 2, 8, 1.0, 2),
    ((16,), 4, 2, 8, 0.0, 1),
    ((16,), 4, 2, 8, 0.37, 3),
    ((16,), 2, 2, 4, 10.0, 1),
    ((11,), 4, 2, 8, 1e4, 1),
    ((12,), 4, 2, 8, 1e4, 5),
    ((9,), 4, 2, 8, 2.5, 20),
    ((1, 7, 3), 4, 2, 8, 1.0, 2),
    ((5, 1, 8), 4, 1, 8, 0.5, 0),
    ((13,), 3, 1, 8, 1e4, 0),
]


def pin_brute(fn, cases=BRUTE_CASES, rtol=1e-12):
    for n, (lens, Hq, Hkv, d, a, b) in enumerate(cases):
        T = sum(lens)
        Q = _rand((T, Hq, d), 100 + n, 1.5)
        K = _rand((T, Hkv, d), 200 + n, 1.5)
        cu = _cu(lens)
        ref = brute_scores(Q.tolist(), K.tolist(), cu.tolist(), a, b)
        ref = np.array([[float(x) for x in row] for row in ref])
        got = np.asarray(fn(Q, K, cu, a, b), dtype=np.float64)
        assert got.shape == ref.shape, (got.shape, ref.shape)
        err = np.abs(got - ref)
        bound = rtol * np.abs(ref) + 1e-300
        assert np.all(err <= bound), (
            f"case {n} {lens} a={a} b={b}: max rel err "
            f"{np.max(err / (np.abs(ref) + 1e-300)):.3e}")


def _harmonic(n):
    return sum((Fraction(1, j) for j in range(1, n + 1)), Fraction(0))


def pin_zero_keys(fn, N=300, Hq=4, Hkv=2, d=16):
    """K = 0 makes every causal row uniform: P[q, k] = 1/(q+1).
    a = 0 (w = 1/2): s[g, k] = (G/2)(H_N - H_k).
    a = 1e4, b = W (w = 1 on the last W rows, else 0):
    s[g, k] = G * sum_{q >= max(k, N-W)} 1/(q+1)."""
    G = Hq // Hkv
    Q = _rand((N, Hq, d), 7)
    K = np.zeros((N, Hkv, d))
    cu = _cu((N,))
    HN = _harmonic(N)
    Hk = Fraction(0)
    want0 = []
    for k in range(N):
        want0.append(float(Fraction(G, 2) * (HN - Hk)))
        Hk += Fraction(1, k + 1)
    got0 = np.asarray(fn(Q, K, cu, 0.0, 1))
    for g in range(Hkv):
        np.testing.assert_allclose(got0[g], want0, rtol=1e-13, atol=0)
    W = 37
    wantW = [float(G * sum(Fraction(1, q + 1) for q in range(max(k, N - W), N)))
             for k in range(N)]
    gotW = np.asarray(fn(Q, K, cu, 1e4, W))
    for g in range(Hkv):
        np.testing.assert_allclose(gotW[g], wantW, rtol=1e-13, atol=0)
    return got0


def pin_ties(fn, N=64, Hq=4, Hkv=2, d=8):
    """a = 1e4, b = 1 keeps only the last row; a zero last query makes it
    uniform, so every score is exactly G/N (N a power of two)."""
    G = Hq // Hkv
    Q = _rand((N, Hq, d), 11)
    Q[N - 1] = 0.0
    K = _rand((N, Hkv, d), 12)
    got = np.asarray(fn(Q, K, _cu((N,)), 1e4, 1))
    assert np.all(got == G / N), np.unique(got)
    return got


def _dense_P(Q, K, lo, hi, h, G):
    """Row-softmax of the causal logits of head h, via scipy."""
    d = Q.shape[2]
    L = np.einsum("qd,kd->qk", Q[lo:hi, h], K[lo:hi, h // G]) / np.sqrt(d)
    N = hi - lo
    L = np.where(np.tril(np.ones((N, N), dtype=bool)), L, -np.inf)
    return softmax(L, axis=1)


def pin_limits(fn, lens=(40, 25), Hq=4, Hkv=2, d=16):
    """WAITS README opening summary: a = 0 is H2O (every row, weight 1/2),
    a -> inf with b = 1 is TOVA (last row), with b = W a window of W rows."""
    G = Hq // Hkv
    T = sum(lens)
    Q = _rand((T, Hq, d), 21, 1.3)
    K = _rand((T, Hkv, d), 22, 1.3)
    cu = _cu(lens)
    W = 9
    want = {k: np.zeros((Hkv, T)) for k in ("h2o", "tova", "win")}
    for i in range(len(lens)):
        lo, hi = cu[i], cu[i + 1]
        for h in range(Hq):
            P = _dense_P(Q, K, lo, hi, h, G)
            want["h2o"][h // G, lo:hi] += P.sum(axis=0)
            want["tova"][h // G, lo:hi] += P[-1]
            want["win"][h // G, lo:hi] += P[-W:].sum(axis=0)
    np.testing.assert_allclose(2.0 * np.asarray(fn(Q, K, cu, 0.0, 3)),
                               want["h2o"], rtol=1e-12, atol=0)
    np.testing.assert_allclose(np.asarray(fn(Q, K, cu, 1e4, 1)),
                               want["tova"], rtol=1e-12, atol=0)
    np.testing.assert_allclose(np.asarray(fn(Q, K, cu, 1e4, W)),
                               want["win"], rtol=1e-12, atol=0)


def _curve_scipy(N, a, b):
    from scipy.special import expit
    return expit(a * (np.arange(N) - (N - b - 0.5)))


def pin_invariants(fn, lens=(70, 33, 1), Hq=4, Hkv=2, d=16,
                   params=((1.0, 4), (0.05, 20), (0.0, 1), (3.0, 0))):
    """Rows of P sum to 1, so sum_k s[g, k] = G * sum_q w[q]; s >= 0; the
    last position only sees the last row: s[g, N-1] = w[N-1] *
    sum_h P_h[N-1, N-1]; a one-token sequence scores G * w[0]."""
    G = Hq // Hkv
    T = sum(lens)
    Q = _rand((T, Hq, d), 31, 1.2)
    K = _rand((T, Hkv, d), 32, 1.2)
    cu = _cu(lens)
    for a, b in params:
        s = np.asarray(fn(Q, K, cu, a, b))
        assert np.all(s >= 0.0)
        for i in range(len(lens)):
            lo, hi = cu[i], cu[i + 1]
            N = hi - lo
            w = _curve_scipy(N, a, b)
            for g in range(Hkv):
                np.testing.assert_allclose(s[g, lo:hi].sum(), G * w.sum(),
                                           rtol=1e-12)
                last = sum(_dense_P(Q, K, lo, hi, h, G)[-1, -1]
                           for h in range(g * G, g * G + G))
                np.testing.assert_allclose(s[g, hi - 1], w[-1] * last,
                                           rtol=1e-12)
                if N == 1:
                    np.testing.assert_allclose(s[g, lo], G * w[0], rtol=1e-15)


ALL_PINS = (pin_brute, pin_zero_keys, pin_ties, pin_limits, pin_invariants)
