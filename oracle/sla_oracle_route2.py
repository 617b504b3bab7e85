"""fp64 reference of the second-order block score for routing (test infrastructure only).

Source: "SPLA - Atención de Bloque Dispersa más Lineal para el Modelado de Contexto Largo",
§2.1: a block's relevance is the expected exponential attention of its tokens, expanded to
second order around the block mean, exp(q . kbar) (1 + 1/2 q^T Cov(k) q), with the
covariance kept diagonal so the score needs only per-block channel statistics.

Readings for SLA's query-block routing (the page scores one decode query):
* the query is the pooled query qbar_i of the query block (as in SLA's router);
* every exponent carries 1/sqrt(D), so the quadratic term is sum_d qbar_d^2 var_d / (2 D);
* var_d is the population variance (divide by the block's valid token count) of channel d
  over the block's valid keys;
* blocks are ranked by log of the score, s_ij = qbar_i . kbar_j / sqrt(D) +
  log1p(sum_d qbar_i,d^2 var_j,d / (2 D)) (log is monotone, so the order is the score's),
  with SLA's total order and counts (``route_from_scores``).

Parity status: pinned by zero-variance blocks reducing to SLA's first-order router, and by
the score matching log of the exact block mean of exp(q . k / sqrt(D)) to fourth order in
the key spread for a block whose covariance is exactly diagonal (pairs of keys along each
channel axis).
"""

from __future__ import annotations

import math

import numpy as np

from .sla_oracle import as_f64, block_counts, pool_mean, route_from_scores


def block_variance(k: np.ndarray, block_kv: int) -> np.ndarray:
    """Population variance per channel over each block's valid keys, [..., Nk, D]."""
    k = as_f64(k)
    N = k.shape[-2]
    out = []
    for s in range(0, N, block_kv):
        kb = k[..., s:min(N, s + block_kv), :]
        out.append(((kb - kb.mean(axis=-2, keepdims=True)) ** 2).mean(axis=-2))
    return np.stack(out, axis=-2)


def second_order_scores(q, k, block_q: int, block_kv: int) -> np.ndarray:
    """log of SPLA's second-order block score, [..., Nq, Nk] (module docstring)."""
    q, k = as_f64(q), as_f64(k)
    D = q.shape[-1]
    qbar = pool_mean(q, block_q)
    kbar = pool_mean(k, block_kv)
    var = block_variance(k, block_kv)
    first = np.matmul(qbar, np.swapaxes(kbar, -1, -2)) / math.sqrt(D)
    quad = np.matmul(qbar ** 2, np.swapaxes(var, -1, -2)) / (2.0 * D)
    return first + np.log1p(quad)


def route_second_order(q, k, block_q: int, block_kv: int, kh: float, kl: float):
    """Labels [B,H,Nq,Nk] from the second-order score, and the scores."""
    N = np.shape(q)[-2]
    _, _, kc, kn = block_counts(N, block_q, block_kv, kh, kl)
    S2 = second_order_scores(q, k, block_q, block_kv)
    return route_from_scores(S2, kc, kn), S2
