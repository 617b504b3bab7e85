"""fp64 reference of the linear branch with the exponential feature map (test infrastructure only).

Source: "SPLA - Atención de Bloque Dispersa más Lineal para el Modelado de Contexto Largo",
§2.3: the linear attention uses a parameter-free exponential feature map, phi(x) ~ exp(x),
so no projection weights are added. Reading: phi(x) = e^x elementwise on the raw q and k
(no 1/sqrt(D), no per-token max subtraction: a per-token shift of k would change the
result). Everything else is SLA's forward of ``sla_oracle.forward`` (router, sparse
branch, empty-branch conventions, alpha blend); only phi in the states h_j = phi(K_j)^T V_j,
z_j = colsum phi(K_j) and in phi(q) of the linear branch changes.

Parity status: pinned by every block marginal giving exp-feature linear attention as torch
computes it over all keys, and by alpha = 1 giving exactly the elu+1 forward (the sparse
branch does not see phi).
"""

from __future__ import annotations

import numpy as np

from .sla_oracle import CRITICAL, MARGINAL, as_f64, block_counts, route_from_scores, compressed_scores, sparse_branch


def phi_exp(x) -> np.ndarray:
    return np.exp(np.asarray(x, dtype=np.float64))


def forward_expmap(q, k, v, alpha, block_q: int, block_kv: int, kh: float = 0.0, kl: float = 0.0, mask=None):
    """SLA forward with phi(x) = e^x in the linear branch, [B,H,N,D] float64."""
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
            fk = phi_exp(k[b, h])
            hst = np.stack([fk[j * block_kv:(j + 1) * block_kv].T @ v[b, h, j * block_kv:(j + 1) * block_kv]
                            for j in range(Nk)])
            zst = np.stack([fk[j * block_kv:(j + 1) * block_kv].sum(axis=0) for j in range(Nk)])
            for i in range(Nq):
                s, e = i * block_q, min(N, (i + 1) * block_q)
                row = mask[b, h, i]
                os_, _ = sparse_branch(q[b, h, s:e], k[b, h], v[b, h], np.nonzero(row == CRITICAL)[0], block_kv)
                marg = row == MARGINAL
                if marg.any():
                    fq = phi_exp(q[b, h, s:e])
                    ol_ = (fq @ hst[marg].sum(axis=0)) / (fq @ zst[marg].sum(axis=0))[:, None]
                else:
                    ol_ = np.zeros_like(os_)
                O[b, h, s:e] = alpha[h] * os_ + (1.0 - alpha[h]) * ol_
    return O
