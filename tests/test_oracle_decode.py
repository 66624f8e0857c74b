"""oracle.decode_attention (one decode step over the compacted cache)
against facts that do not come from itself."""

from decimal import Decimal, localcontext

import numpy as np
import pytest

import oracle
import pins


def _brute(q, K, V, n):
    """Decimal softmax attention of one query over n cache rows."""
    d = len(q)
    with localcontext() as ctx:
        ctx.prec = 40
        root = Decimal(d).sqrt()
        L = [sum(Decimal(float(q[i])) * Decimal(float(K[j][i])) for i in range(d)) / root
             for j in range(n)]
        m = max(L)
        e = [(x - m).exp() for x in L]
        z = sum(e)
        o = [sum(e[j] * Decimal(float(V[j][i])) for j in range(n)) / z for i in range(d)]
        return [float(x) for x in o], float(m + z.ln())


def test_matches_decimal_brute_force():
    q = pins._rand((2, 4, 8), 61)
    K = pins._rand((2, 2, 9, 8), 62)
    V = pins._rand((2, 2, 9, 8), 63)
    lens = np.array([9, 5])
    o, lse = oracle.decode_attention(q, K, V, lens)
    for s in range(2):
        for h in range(4):
            bo, bl = _brute(q[s, h], K[s, h // 2], V[s, h // 2], lens[s])
            np.testing.assert_allclose(o[s, h], bo, rtol=1e-12, atol=1e-13)
            assert lse[s, h] == pytest.approx(bl, rel=1e-12)


def test_zero_keys_average_the_values():
    q = pins._rand((1, 2, 8), 71)
    K = np.zeros((1, 1, 6, 8))
    V = pins._rand((1, 1, 6, 8), 72)
    o, lse = oracle.decode_attention(q, K, V, np.array([4]))
    np.testing.assert_allclose(o[0, 0], V[0, 0, :4].mean(axis=0), rtol=1e-14)
    assert lse[0, 1] == pytest.approx(np.log(4.0), rel=1e-14)


def test_one_entry_returns_its_value_and_empty_cache_is_zero():
    q = pins._rand((2, 2, 4), 81)
    K = pins._rand((2, 2, 3, 4), 82)
    V = pins._rand((2, 2, 3, 4), 83)
    o, lse = oracle.decode_attention(q, K, V, np.array([1, 0]))
    np.testing.assert_allclose(o[0], V[0, :, 0], rtol=1e-15)
    assert lse[0, 0] == pytest.approx(q[0, 0] @ K[0, 0, 0] / 2.0, rel=1e-14)
    assert np.all(o[1] == 0.0) and np.all(np.isneginf(lse[1]))


def test_slots_past_the_length_are_ignored():
    q = pins._rand((1, 2, 8), 91)
    K = pins._rand((1, 1, 10, 8), 92)
    V = pins._rand((1, 1, 10, 8), 93)
    o1, l1 = oracle.decode_attention(q, K, V, np.array([6]))
    K2, V2 = K.copy(), V.copy()
    K2[:, :, 6:] = 1e3
    V2[:, :, 6:] = -1e3
    o2, l2 = oracle.decode_attention(q, K2, V2, np.array([6]))
    np.testing.assert_array_equal(o1, o2)
    np.testing.assert_array_equal(l1, l2)
