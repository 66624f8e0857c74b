"""Oracle selection against Python's sorted(); compaction against a loop."""

import numpy as np
import pytest

import oracle


def _sorted_select(sc, N, R, B):
    """Textbook restatement: sort the pool by (-score, index), keep B-R,
    add the recent window, report ascending."""
    if N <= B:
        return list(range(N))
    pool = sorted(range(N - R), key=lambda k: (-sc[k], k))[:B - R]
    return sorted(pool + list(range(N - R, N)))


@pytest.mark.parametrize("lens,R,B", [((1000,), 16, 128), ((300, 5, 129), 4, 128),
                                      ((128,), 16, 128), ((129,), 0, 128),
                                      ((200,), 128, 128), ((50, 0, 70), 10, 60),
                                      ((1,), 0, 1)])
def test_select_matches_sorted(lens, R, B):
    rng = np.random.default_rng(3)
    T = sum(lens)
    Hkv = 3
    # few distinct values -> many exact ties
    s = rng.integers(0, 40, size=(Hkv, T)).astype(np.float64) / 8.0
    cu = np.concatenate([[0], np.cumsum(lens)])
    idx, kept = oracle.select(s, cu, R, B)
    assert idx.dtype == np.int32 and kept.dtype == np.int32
    for i, N in enumerate(lens):
        lo = cu[i]
        assert kept[i] == min(N, B)
        for g in range(Hkv):
            want = _sorted_select(s[g, lo:lo + N], N, R, B)
            assert idx[i, g, :kept[i]].tolist() == want
            assert np.all(idx[i, g, kept[i]:] == -1)


def test_select_rejects_bad_budgets():
    s = np.zeros((1, 10))
    for R, B in ((5, 4), (-1, 4), (0, 0)):
        with pytest.raises(ValueError):
            oracle.select(s, np.array([0, 10]), R, B)


def test_compact_matches_loop():
    rng = np.random.default_rng(5)
    lens = (40, 3, 17)
    T, Hkv, d, B = sum(lens), 2, 8, 16
    K = rng.integers(-2**15, 2**15, size=(T, Hkv, d)).astype(np.int16)
    V = rng.integers(-2**15, 2**15, size=(T, Hkv, d)).astype(np.int16)
    cu = np.concatenate([[0], np.cumsum(lens)])
    s = rng.random((Hkv, T))
    idx, kept = oracle.select(s, cu, 4, B)
    Ko, Vo = oracle.compact(K, V, cu, idx, kept, B)
    assert Ko.dtype == np.int16 and Ko.shape == (3, Hkv, B, d)
    for i in range(3):
        for g in range(Hkv):
            for j in range(B):
                if j < kept[i]:
                    t = cu[i] + idx[i, g, j]
                    assert np.array_equal(Ko[i, g, j], K[t, g])
                    assert np.array_equal(Vo[i, g, j], V[t, g])
                else:
                    assert not Ko[i, g, j].any() and not Vo[i, g, j].any()


def test_compress_composes():
    rng = np.random.default_rng(9)
    T, Hq, Hkv, d = 90, 4, 2, 8
    Q = rng.standard_normal((T, Hq, d))
    K = rng.standard_normal((T, Hkv, d))
    V = rng.standard_normal((T, Hkv, d))
    cu = np.array([0, 60, 90])
    s, idx, kept, Ko, Vo = oracle.compress(Q, K, V, cu, 1.0, 4, 4, 20)
    np.testing.assert_array_equal(s, oracle.score(Q, K, cu, 1.0, 4))
    i2, k2 = oracle.select(s, cu, 4, 20)
    np.testing.assert_array_equal(idx, i2)
    np.testing.assert_array_equal(Ko, oracle.compact(K, V, cu, i2, k2, 20)[0])
