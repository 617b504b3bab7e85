"""Pins of the second-order block score (oracle/sla_oracle_route2.py): zero-variance blocks
give SLA's first-order scores and labels; for a block whose covariance is exactly diagonal
the score agrees with the log of the exact block mean of exp(q . k / sqrt(D)) to fourth
order in the spread (the error falls 16x when the spread halves; a wrong quadratic
coefficient leaves a second-order error); the block variance in closed form.
"""

import math

import numpy as np

from oracle import sla_oracle as so
from oracle import sla_oracle_route2 as r2


def test_zero_variance_blocks_reduce_to_the_first_order_router():
    rng = np.random.default_rng(0)
    B, H, N, D, bq, bk = 1, 2, 70, 16, 16, 8
    Nk = -(-N // bk)
    k = np.repeat(rng.normal(0, 1, (B, H, Nk, D)), bk, axis=2)[:, :, :N]
    q = rng.normal(0, 1, (B, H, N, D))
    S2 = r2.second_order_scores(q, k, bq, bk)
    np.testing.assert_allclose(S2, so.compressed_scores(q, k, bq, bk), rtol=0, atol=1e-15)
    m2, _ = r2.route_second_order(q, k, bq, bk, 0.25, 0.25)
    m1, _ = so.route(q, k, bq, bk, 0.25, 0.25)
    np.testing.assert_array_equal(m2, m1)


def _axis_block_error(eps, seed=1):
    # one query row (bq = 1) and one block of 2D keys kbar +- eps c_d e_d, one pair per
    # channel: the block covariance is exactly diagonal (var_d = eps^2 c_d^2 / D), and the
    # exact block mean of the exponentials is exp(q.kbar/sqrt(D)) mean_d cosh(eps c_d q_d /
    # sqrt(D)); the score keeps its expansion to second order, so the log error is O(eps^4)
    rng = np.random.default_rng(seed)
    D = 16
    q = rng.normal(0, 1, (1, D))
    kbar, c = rng.normal(0, 1, D), rng.uniform(0.5, 2.0, D)
    dev = np.diag(eps * c)
    k = np.concatenate([kbar + dev, kbar - dev])
    exact = math.log(np.mean(np.exp(k @ q[0] / math.sqrt(D))))
    return abs(r2.second_order_scores(q, k, 1, 2 * D)[0, 0] - exact)


def test_score_matches_the_exact_block_mean_to_fourth_order():
    errs = [_axis_block_error(e) for e in (0.8, 0.4, 0.2)]
    r1, r2_ = errs[0] / errs[1], errs[1] / errs[2]
    assert 13.0 < r1 < 19.0 and 13.0 < r2_ < 19.0, errs


def test_block_variance_closed_form():
    rng = np.random.default_rng(2)
    k = rng.normal(0, 1, (21, 3))
    var = r2.block_variance(k, 8)
    np.testing.assert_allclose(var[2], np.var(k[16:], axis=0), rtol=1e-14)
    np.testing.assert_allclose(var[0], ((k[:8] - k[:8].mean(0)) ** 2).sum(0) / 8, rtol=1e-14)
