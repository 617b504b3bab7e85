"""Pins of the PISA oracle (oracle/sla_oracle_pisa.py) against things other than itself:
every block critical is dense softmax attention (torch SDPA in fp64); blocks whose keys are
all equal make the Taylor expansion exact, so any critical set gives dense attention; and
with a key spread eps and the same first-order matrix in every block, the error against
dense attention falls as eps^2 (zero-order plus first-order terms), where a missing or
mis-signed first-order term would leave an eps^1 error.
"""

import numpy as np
import pytest
import torch

from oracle import sla_oracle as so
from oracle import sla_oracle_pisa as pisa


def _dense(q, k, v):
    t = [torch.tensor(x) for x in (q, k, v)]
    return torch.nn.functional.scaled_dot_product_attention(*t).numpy()


def test_every_block_critical_is_dense_attention():
    rng = np.random.default_rng(0)
    q, k, v = (rng.normal(0, 1, (1, 2, 45, 16)) for _ in range(3))
    mask = np.full((1, 2, 3, 6), so.CRITICAL, dtype=np.int8)
    np.testing.assert_allclose(pisa.forward_pisa(q, k, v, 16, 8, mask), _dense(q, k, v), rtol=0, atol=1e-13)


@pytest.mark.parametrize("seed", [1, 2])
def test_blocks_of_equal_keys_make_the_expansion_exact(seed):
    rng = np.random.default_rng(seed)
    B, H, N, D, bq, bk = 1, 2, 45, 16, 16, 8
    Nk = -(-N // bk)
    centres = rng.normal(0, 1, (B, H, Nk, D))
    k = np.repeat(centres, bk, axis=2)[:, :, :N]   # every key of block j is its centroid
    q = rng.normal(0, 1, (B, H, N, D))
    v = rng.normal(0, 1, (B, H, N, D))
    mask = rng.integers(0, 3, (B, H, 3, Nk)).astype(np.int8)
    mask[0, 0, 0] = 0                              # one row with no critical block at all
    np.testing.assert_allclose(pisa.forward_pisa(q, k, v, bq, bk, mask), _dense(q, k, v), rtol=0, atol=1e-13)


def _spread_problem(eps, seed=3):
    # N a multiple of the block, keys k = c_j + eps * d_r and values v = w_j + u_r with the
    # in-block patterns d, u shared by all blocks and sum_r d_r = 0: every block then has
    # the same first-order matrix H_j = eps * sum_r d_r u_r^T, so Hbar = H_j.
    rng = np.random.default_rng(seed)
    B, H, D, bk, Nk = 1, 1, 16, 8, 6
    c = rng.normal(0, 1, (Nk, D))
    d = rng.normal(0, 1, (bk, D))
    d -= d.mean(axis=0)
    w = rng.normal(0, 1, (Nk, D))
    u = rng.normal(0, 1, (bk, D))
    k = (c[:, None, :] + eps * d[None]).reshape(1, 1, Nk * bk, D)
    v = (w[:, None, :] + u[None]).reshape(1, 1, Nk * bk, D)
    q = rng.normal(0, 1, (B, H, Nk * bk, D))
    mask = np.zeros((1, 1, 3, Nk), dtype=np.int8)
    mask[0, 0, :, 0] = so.CRITICAL                 # one exact block per row, five expanded
    mask[0, 0, 1, 3] = so.CRITICAL
    return q, k, v, mask


def test_error_falls_as_the_square_of_the_key_spread():
    errs = []
    for eps in (0.08, 0.04, 0.02):
        q, k, v, mask = _spread_problem(eps)
        errs.append(np.abs(pisa.forward_pisa(q, k, v, 16, 8, mask) - _dense(q, k, v)).max())
    r1, r2 = errs[0] / errs[1], errs[1] / errs[2]
    assert 3.2 < r1 < 4.8 and 3.2 < r2 < 4.8, errs


def test_block_statistics_closed_forms():
    rng = np.random.default_rng(4)
    k, v = rng.normal(0, 1, (21, 4)), rng.normal(0, 1, (21, 4))
    kbar, n, vsum, H = pisa.block_statistics(k, v, 8)
    np.testing.assert_array_equal(n, [8, 8, 5])
    np.testing.assert_allclose(kbar[2], k[16:].sum(axis=0) / 5, rtol=1e-15)
    # H_j = sum_n (k_n - kbar_j) v_n^T, written here as outer products one token at a time
    H2 = sum(np.outer(k[t] - kbar[2], v[t]) for t in range(16, 21))
    np.testing.assert_allclose(H[2], H2, rtol=0, atol=1e-14)
    # the first-order sum of the denominator vanishes: sum_n (k_n - kbar_j) = 0
    np.testing.assert_allclose((k[16:] - kbar[2]).sum(axis=0), 0, atol=1e-14)
