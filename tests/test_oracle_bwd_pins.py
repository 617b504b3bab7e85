"""Pins of the backward oracle (oracle/sla_oracle_bwd.py) against things other than itself.

The backward is the exact derivative of the forward oracle with the labels fixed, so it is
checked against central finite differences through ``sla_oracle.forward`` (every input,
mixed labels, ragged tails, empty branches), against torch autograd of dense softmax
attention (every block critical) and of linear attention (every block marginal), and by
exact zeros for the keys of blocks that are negligible in every row.
"""

import numpy as np
import pytest
import torch

from oracle import sla_oracle as so
from oracle import sla_oracle_bwd as bw


def _problem(seed, B=1, H=2, N=37, D=8, bq=8, bk=8):
    rng = np.random.default_rng(seed)
    q, k, v = (rng.normal(0, 1, (B, H, N, D)) for _ in range(3))
    alpha = rng.uniform(0, 1, (H, D))
    dO = rng.normal(0, 1, (B, H, N, D))
    Nq, Nk = -(-N // bq), -(-N // bk)
    mask = rng.integers(0, 3, (B, H, Nq, Nk)).astype(np.int8)
    mask[0, 0, 0] = np.where(mask[0, 0, 0] == so.CRITICAL, so.MARGINAL, mask[0, 0, 0])  # no critical block
    mask[0, 0, 1] = np.where(mask[0, 0, 1] == so.MARGINAL, 0, mask[0, 0, 1])           # no marginal block
    mask[0, 0, 1, 0] = so.CRITICAL
    return q, k, v, alpha, dO, mask, bq, bk


def _loss(q, k, v, alpha, bq, bk, mask, dO):
    return float((so.forward(q, k, v, alpha, bq, bk, mask=mask) * dO).sum())


@pytest.mark.parametrize("seed, bq", [(0, 8), (1, 16)])
def test_matches_central_differences(seed, bq):
    q, k, v, alpha, dO, mask, _, bk = _problem(seed, bq=bq)
    if bq == 16:
        Nq = -(-q.shape[2] // 16)
        mask = mask[:, :, :Nq]
    grads = bw.backward(q, k, v, alpha, bq, bk, mask, dO)
    rng = np.random.default_rng(seed + 10)
    eps = 1e-6
    inputs = [q, k, v, alpha]
    for which, (x, g) in enumerate(zip(inputs, grads)):
        flat = [np.unravel_index(i, x.shape) for i in range(x.size)]
        pick = flat if x.size <= 64 else [flat[i] for i in rng.choice(x.size, 48, replace=False)]
        for ix in pick:
            args = [t.copy() for t in inputs]
            args[which][ix] += eps
            lp = _loss(*args[:4], bq, bk, mask, dO)
            args[which][ix] -= 2 * eps
            lm = _loss(*args[:4], bq, bk, mask, dO)
            fd = (lp - lm) / (2 * eps)
            assert abs(fd - g[ix]) <= 2e-6 * max(1.0, abs(fd)), (which, ix, fd, g[ix])


def test_every_block_critical_is_dense_softmax_attention():
    rng = np.random.default_rng(2)
    B, H, N, D, bq, bk = 1, 2, 21, 8, 8, 8
    q, k, v, dO = (rng.normal(0, 1, (B, H, N, D)) for _ in range(4))
    alpha = np.ones((H, D))
    mask = np.full((B, H, 3, 3), so.CRITICAL, dtype=np.int8)
    dQ, dK, dV, dA = bw.backward(q, k, v, alpha, bq, bk, mask, dO)
    tq, tk, tv = (torch.tensor(x, requires_grad=True) for x in (q, k, v))
    out = torch.nn.functional.scaled_dot_product_attention(tq, tk, tv)
    out.backward(torch.tensor(dO))
    np.testing.assert_allclose(dQ, tq.grad.numpy(), rtol=0, atol=1e-12)
    np.testing.assert_allclose(dK, tk.grad.numpy(), rtol=0, atol=1e-12)
    np.testing.assert_allclose(dV, tv.grad.numpy(), rtol=0, atol=1e-12)
    # alpha = 1 and no marginal block: dalpha = sum over tokens of dO * O_s
    np.testing.assert_allclose(dA, (dO * out.detach().numpy()).sum(axis=(0, 2)), rtol=0, atol=1e-12)


def test_every_block_marginal_is_linear_attention():
    rng = np.random.default_rng(3)
    B, H, N, D, bq, bk = 1, 2, 21, 8, 8, 8
    q, k, v, dO = (rng.normal(0, 1, (B, H, N, D)) for _ in range(4))
    alpha = np.zeros((H, D))
    mask = np.full((B, H, 3, 3), so.MARGINAL, dtype=np.int8)
    dQ, dK, dV, _ = bw.backward(q, k, v, alpha, bq, bk, mask, dO)
    tq, tk, tv = (torch.tensor(x, requires_grad=True) for x in (q, k, v))
    fq = torch.nn.functional.elu(tq) + 1.0
    fk = torch.nn.functional.elu(tk) + 1.0
    out = (fq @ (fk.transpose(-1, -2) @ tv)) / (fq @ fk.sum(dim=-2, keepdim=True).transpose(-1, -2))
    out.backward(torch.tensor(dO))
    np.testing.assert_allclose(dQ, tq.grad.numpy(), rtol=0, atol=1e-12)
    np.testing.assert_allclose(dK, tk.grad.numpy(), rtol=0, atol=1e-12)
    np.testing.assert_allclose(dV, tv.grad.numpy(), rtol=0, atol=1e-12)


def test_keys_negligible_everywhere_get_no_gradient():
    q, k, v, alpha, dO, mask, bq, bk = _problem(4)
    mask[:, :, :, 2] = 0  # KV block 2 is negligible for every query block
    _, dK, dV, _ = bw.backward(q, k, v, alpha, bq, bk, mask, dO)
    assert not dK[:, :, 16:24].any() and not dV[:, :, 16:24].any()
    assert np.abs(dK[:, :, :16]).sum() > 0


def test_linear_in_the_output_gradient():
    q, k, v, alpha, dO, mask, bq, bk = _problem(5)
    dO2 = np.random.default_rng(6).normal(0, 1, dO.shape)
    g1 = bw.backward(q, k, v, alpha, bq, bk, mask, dO)
    g2 = bw.backward(q, k, v, alpha, bq, bk, mask, dO2)
    g12 = bw.backward(q, k, v, alpha, bq, bk, mask, dO + 2.0 * dO2)
    for a, b, c in zip(g1, g2, g12):
        np.testing.assert_allclose(c, a + 2.0 * b, rtol=1e-12, atol=1e-12)


def test_dphi_matches_elu_derivative():
    x = np.linspace(-5, 5, 1001)
    t = torch.tensor(x, requires_grad=True)
    (torch.nn.functional.elu(t) + 1.0).sum().backward()
    np.testing.assert_allclose(bw.dphi(x), t.grad.numpy(), rtol=1e-15, atol=0)
