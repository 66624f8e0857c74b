"""The fp64 oracle against facts that do not come from itself."""

import numpy as np
import pytest
from scipy.special import expit

import oracle
import pins


@pytest.mark.parametrize("pin", pins.ALL_PINS, ids=lambda p: p.__name__)
def test_oracle_pin(pin):
    pin(oracle.score)


def test_row_blocking_is_invisible():
    """Blocks of rows are independent softmaxes: any block size gives the
    same scores (bit for bit up to summation order of the blocks)."""
    Q = pins._rand((300, 4, 16), 41)
    K = pins._rand((300, 2, 16), 42)
    cu = np.array([0, 170, 300])
    ref = oracle.score(Q, K, cu, 0.2, 30)
    for rb in (1, 7, 64, 1000):
        np.testing.assert_allclose(oracle.score(Q, K, cu, 0.2, 30,
                                                row_block=rb),
                                   ref, rtol=1e-13)


def test_zero_key_selection_is_front_and_back():
    """With K = 0 and a = 0 scores fall strictly with k, so the kept set is
    the first B-R positions plus the recent window."""
    s = pins.pin_zero_keys(oracle.score, N=300)
    R, B = 16, 64
    idx, kept = oracle.select(s, np.array([0, 300]), R, B)
    want = np.concatenate([np.arange(B - R), np.arange(300 - R, 300)])
    assert kept.tolist() == [B]
    for g in range(idx.shape[1]):
        assert idx[0, g].tolist() == want.tolist()


def test_exact_ties_go_to_lower_index():
    s = pins.pin_ties(oracle.score, N=64)
    idx, kept = oracle.select(s, np.array([0, 64]), 4, 20)
    want = list(range(16)) + list(range(60, 64))
    for g in range(idx.shape[1]):
        assert idx[0, g].tolist() == want


class TestCurve:
    """Forgetting curve of the WAITS opening summary."""

    @pytest.mark.parametrize("N,a,b", [(512, 1.0, 16), (4096, 0.01, 128),
                                       (100, 10.0, 1), (7, 3.3, 0)])
    def test_midpoint_and_symmetry(self, N, a, b):
        c = N - b - 0.5
        assert oracle.forgetting_curve(c, N, a, b) == 0.5
        x = np.linspace(0.0, 50.0, 101)
        w_hi = oracle.forgetting_curve(c + x, N, a, b)
        w_lo = oracle.forgetting_curve(c - x, N, a, b)
        np.testing.assert_allclose(w_hi + w_lo, 1.0, rtol=0, atol=1e-15)
        q = np.arange(N)
        assert np.all(np.diff(oracle.forgetting_curve(q, N, a, b)) >= 0)

    def test_h2o_limit_is_constant_half(self):
        w = oracle.forgetting_curve(np.arange(1000), 1000, 0.0, 7)
        assert np.all(w == 0.5)

    @pytest.mark.parametrize("b", [1, 16, 128])
    def test_step_limit_keeps_last_b_rows(self, b):
        """a -> inf (a = 1e4): w is exactly 1 on the last b rows, else 0."""
        N = 300
        w = oracle.forgetting_curve(np.arange(N), N, 1e4, b)
        assert np.all(w[N - b:] == 1.0) and np.all(w[:N - b] == 0.0)


def test_one_token_sequence():
    """N = 1: the single key receives G * w[0]."""
    Q = pins._rand((1, 6, 8), 51)
    K = pins._rand((1, 2, 8), 52)
    for a, b in ((0.0, 1), (1.0, 0), (2.0, 5)):
        s = oracle.score(Q, K, np.array([0, 1]), a, b)
        w0 = expit(a * (0 - (1 - b - 0.5)))
        np.testing.assert_allclose(s[:, 0], 3 * w0, rtol=1e-15)


@pytest.mark.parametrize("N,a,b", [(32768, 1.0, 16), (131072, 0.01, 128),
                                   (4096, 10.0, 1), (512, 1e4, 1),
                                   (4096, 0.01, 128)])
def test_fp32_zero_weight_rows_are_negligible(N, a, b):
    """The CUDA path skips rows whose fp32 weight is exactly 0; the fp64
    weight of all such rows together is below 1e-30, far under any score
    tolerance (scores of these inputs are >= 1e-12)."""
    q = np.arange(N)
    c32 = np.float32(N) - np.float32(b) - np.float32(0.5)
    t32 = np.float32(-a) * (q.astype(np.float32) - c32)
    with np.errstate(over="ignore"):
        w32 = np.float32(1.0) / (np.float32(1.0) + np.exp(t32))
    w64 = oracle.forgetting_curve(q, N, a, b)
    assert w64[w32 == 0].sum() < 1e-30
    # and the kept rows form a suffix of the sequence
    act = np.nonzero(w32 != 0)[0]
    assert len(act) == 0 or np.all(act == np.arange(act[0], N))


def test_last_rows_give_the_exact_tail():
    """Key k is seen only by rows q >= k: summing the last W rows gives the
    exact scores of the last W keys of every sequence, and never more than
    the full scores elsewhere."""
    Q = pins._rand((210, 4, 8), 51)
    K = pins._rand((210, 2, 8), 52)
    cu = np.array([0, 130, 210])
    for a, b in ((0.0, 4), (0.05, 20), (1.0, 3)):
        full = oracle.score(Q, K, cu, a, b)
        part = oracle.score(Q, K, cu, a, b, last=25)
        tail = np.r_[105:130, 185:210]
        np.testing.assert_array_equal(part[:, tail], full[:, tail])
        assert np.all(part <= full * (1 + 1e-12))
        assert np.all(part[:, :100] < full[:, :100]) or a > 0.5
