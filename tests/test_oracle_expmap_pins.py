"""Pins of the exponential-feature-map variant (oracle/sla_oracle_expmap.py): every block
marginal is exp-feature linear attention over all keys as torch computes it, alpha = 1 is
the elu+1 forward exactly (the sparse branch does not see phi), and a row with no marginal
block has no linear term.
"""

import numpy as np
import torch

from oracle import sla_oracle as so
from oracle import sla_oracle_expmap as ex


def _inputs(seed, N=45, D=8):
    rng = np.random.default_rng(seed)
    q, k, v = (rng.normal(0, 1, (1, 2, N, D)) for _ in range(3))
    return q, k, v, rng.uniform(0, 1, (2, D))


def test_every_block_marginal_is_exp_feature_linear_attention():
    q, k, v, _ = _inputs(0)
    mask = np.full((1, 2, 3, 6), so.MARGINAL, dtype=np.int8)
    o = ex.forward_expmap(q, k, v, np.zeros((2, 8)), 16, 8, mask=mask)
    tq, tk, tv = (torch.tensor(x) for x in (q, k, v))
    fq, fk = torch.exp(tq), torch.exp(tk)
    ref = (fq @ (fk.transpose(-1, -2) @ tv)) / (fq @ fk.sum(dim=-2, keepdim=True).transpose(-1, -2))
    np.testing.assert_allclose(o, ref.numpy(), rtol=1e-13, atol=1e-13)


def test_alpha_one_is_the_elu_forward():
    q, k, v, _ = _inputs(1)
    rng = np.random.default_rng(2)
    mask = rng.integers(0, 3, (1, 2, 3, 6)).astype(np.int8)
    ones = np.ones((2, 8))
    np.testing.assert_allclose(ex.forward_expmap(q, k, v, ones, 16, 8, mask=mask),
                               so.forward(q, k, v, ones, 16, 8, mask=mask), rtol=0, atol=1e-14)


def test_rows_without_marginal_blocks_have_no_linear_term():
    q, k, v, a = _inputs(3)
    mask = np.full((1, 2, 3, 6), so.CRITICAL, dtype=np.int8)
    mask[..., 4:] = 0
    o = ex.forward_expmap(q, k, v, a, 16, 8, mask=mask)
    np.testing.assert_allclose(o, so.forward(q, k, v, a, 16, 8, mask=mask), rtol=0, atol=1e-14)
