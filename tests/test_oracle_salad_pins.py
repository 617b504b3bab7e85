"""Pins of the dropped-linear-branch forward (oracle/sla_oracle_salad.py, SALAD §2 post-tuning
branch dropping): alpha = 1 is the SLA forward for any labels, every block critical is alpha
times dense softmax attention as torch computes it, an empty critical set gives zero, and the
branch is dropped exactly when s < tau_t.
"""

import numpy as np
import torch

from oracle import sla_oracle as so
from oracle import sla_oracle_salad as sd


def _inputs(seed, N=45, D=8):
    rng = np.random.default_rng(seed)
    q, k, v = (rng.normal(0, 1, (1, 2, N, D)) for _ in range(3))
    return q, k, v, rng.uniform(0, 1, (2, D))


def test_alpha_one_is_the_sla_forward():
    q, k, v, _ = _inputs(0)
    mask = np.random.default_rng(1).integers(0, 3, (1, 2, 3, 6)).astype(np.int8)
    ones = np.ones((2, 8))
    np.testing.assert_allclose(sd.forward_dropped(q, k, v, ones, 16, 8, mask=mask),
                               so.forward(q, k, v, ones, 16, 8, mask=mask), rtol=0, atol=1e-14)


def test_every_block_critical_is_alpha_times_dense_attention():
    q, k, v, a = _inputs(2)
    o = sd.forward_dropped(q, k, v, a, 16, 8, kh=1.0, kl=0.0)
    tq, tk, tv = (torch.tensor(x) for x in (q, k, v))
    dense = torch.nn.functional.scaled_dot_product_attention(tq, tk, tv).numpy()
    np.testing.assert_allclose(o, a[None, :, None, :] * dense, rtol=1e-12, atol=1e-13)


def test_no_critical_block_gives_zero():
    q, k, v, a = _inputs(3)
    o = sd.forward_dropped(q, k, v, a, 16, 8, kh=0.0, kl=0.3)
    assert np.all(o == 0.0)


def test_dropped_exactly_below_the_threshold():
    assert sd.linear_dropped(0.1, 0.2)
    assert not sd.linear_dropped(0.2, 0.2)
    assert not sd.linear_dropped(0.0, 0.0)
    assert not sd.linear_dropped(0.5, 0.2)
