"""fp64 reference of the forward with the linear branch dropped (test infrastructure only).

Source: "SALAD: Achieve High-Sparsity Attention via Efficient Linear Attention Tuning for
Video Diffusion Transformer", §2 (post-tuning branch dropping): a model-side dynamic scale
s in (0, 1) says how much the linear branch matters at a denoising step, and the branch is
not run at the steps where s is below a threshold tau_t. Readings:

* the library does not compute s (a trained module); the caller passes s and tau_t, and the
  branch is dropped exactly when s < tau_t;
* with SLA2's blend O = alpha O_s + (1 - alpha) O_l, dropping the linear branch leaves
  O = alpha O_s: the (1 - alpha) O_l term is not computed, and the sparse branch is not
  renormalised (SALAD adds the linear branch to the sparse output, so removing it leaves the
  sparse part as it was);
* when the branch is kept, the forward is SLA's (s only decides whether the branch runs;
  SALAD's learned scaling modules are out of scope).

Parity status: pinned by alpha = 1 giving the SLA forward for any labels, by every block
critical giving alpha times dense softmax attention (torch), and by an empty critical set
giving zero.
"""

from __future__ import annotations

import numpy as np

from .sla_oracle import CRITICAL, as_f64, block_counts, compressed_scores, route_from_scores, sparse_branch


def linear_dropped(linear_scale: float, drop_threshold: float) -> bool:
    """The branch is dropped exactly when s < tau_t."""
    return float(linear_scale) < float(drop_threshold)


def forward_dropped(q, k, v, alpha, block_q: int, block_kv: int, kh: float = 0.0, kl: float = 0.0, mask=None):
    """O = alpha * O_s with SLA's labels (the router, or `mask`), [B,H,N,D] float64."""
    q, k, v, alpha = as_f64(q), as_f64(k), as_f64(v), as_f64(alpha)
    B, H, N, D = q.shape
    Nq, Nk, kc, kn = block_counts(N, block_q, block_kv, kh, kl)
    if mask is None:
        mask = np.zeros((B, H, Nq, Nk), dtype=np.int8)
        for b in range(B):
            for h in range(H):
                mask[b, h] = route_from_scores(compressed_scores(q[b, h], k[b, h], block_q, block_kv), kc, kn)
    mask = np.asarray(mask, dtype=np.int8)
    O = np.empty((B, H, N, D))
    for b in range(B):
        for h in range(H):
            for i in range(Nq):
                s, e = i * block_q, min(N, (i + 1) * block_q)
                crit = np.nonzero(mask[b, h, i] == CRITICAL)[0]
                os_, _ = sparse_branch(q[b, h, s:e], k[b, h], v[b, h], crit, block_kv)
                O[b, h, s:e] = alpha[h] * os_
    return O
