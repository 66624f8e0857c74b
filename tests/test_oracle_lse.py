"""oracle.row_lse (the row normalisers a caller can hand to the scorer)
against facts that do not come from itself."""

import numpy as np
import pytest

import oracle
import pins
from brute_decimal import brute_lse


@pytest.mark.parametrize("lens,Hq,Hkv,d,seed", [((5,), 2, 1, 4, 1), ((3, 7), 4, 2, 8, 2),
                                                ((1, 9, 2), 2, 2, 3, 3)])
def test_row_lse_matches_decimal_brute_force(lens, Hq, Hkv, d, seed):
    T = sum(lens)
    Q = pins._rand((T, Hq, d), seed)
    K = pins._rand((T, Hkv, d), seed + 100)
    cu = np.concatenate([[0], np.cumsum(lens)])
    got = oracle.row_lse(Q, K, cu)
    ref = brute_lse(Q, K, cu)
    for h in range(Hq):
        for t in range(T):
            assert abs(got[h, t] - float(ref[h][t])) <= 1e-12 * max(1.0, abs(float(ref[h][t])))


def test_zero_keys_give_log_of_row_length():
    # K = 0: every causal logit is 0, so row q sums q + 1 ones
    lens = (37, 5)
    Q = pins._rand((42, 4, 16), 7)
    K = np.zeros((42, 2, 16))
    cu = np.array([0, 37, 42])
    lse = oracle.row_lse(Q, K, cu)
    q = np.concatenate([np.arange(37), np.arange(5)])
    np.testing.assert_allclose(lse, np.broadcast_to(np.log(q + 1.0), lse.shape), rtol=0,
                               atol=1e-14)


def test_first_row_is_its_own_logit():
    # row 0 of a sequence sees key 0 only: lse = Q[0] . K[0] / sqrt(d)
    Q = pins._rand((6, 2, 8), 11)
    K = pins._rand((6, 1, 8), 12)
    cu = np.array([0, 4, 6])
    lse = oracle.row_lse(Q, K, cu)
    for lo in (0, 4):
        for h in range(2):
            assert lse[h, lo] == pytest.approx(Q[lo, h] @ K[lo, 0] / np.sqrt(8.0), rel=1e-14)


def test_lse_normalises_the_score():
    # the score is w-weighted softmax mass: summed over keys it is G * sum_q w[q]
    # exactly when exp(L - lse) sums to 1 over every row
    Q = pins._rand((50, 4, 8), 21)
    K = pins._rand((50, 2, 8), 22)
    cu = np.array([0, 50])
    lse = oracle.row_lse(Q, K, cu)
    for h in range(4):
        L = Q[:, h] @ K[:, h // 2].T / np.sqrt(8.0)
        P = np.where(np.tril(np.ones((50, 50), bool)), np.exp(L - lse[h][:, None]), 0.0)
        np.testing.assert_allclose(P.sum(axis=1), 1.0, rtol=1e-13)


def test_last_rows_only_equal_the_full_computation():
    Q = pins._rand((90, 4, 8), 31)
    K = pins._rand((90, 2, 8), 32)
    cu = np.array([0, 60, 90])
    full = oracle.row_lse(Q, K, cu)
    part = oracle.row_lse(Q, K, cu, last=7)
    rows = np.r_[53:60, 83:90]
    np.testing.assert_array_equal(part[:, rows], full[:, rows])
    others = np.setdiff1d(np.arange(90), rows)
    assert np.all(np.isnan(part[:, others]))
