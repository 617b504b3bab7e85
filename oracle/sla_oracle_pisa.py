"""fp64 reference of the PISA block attention variant (test infrastructure only).

Source: "PISA - Atención Dispersa por Tramos para Transformers de Difusión Eficientes", §2
(central algorithm, the N_t equation, covariance-aware routing, hardware pipeline). PISA
keeps the same block pipeline as SLA (pooled router, per-block statistics, one fused pass)
but puts its approximation inside the softmax: every KV block that is not critical
contributes a Taylor expansion of its exponentials around the block centroid, in both the
numerator and the denominator, instead of being skipped or sent to a separate branch.

Per query token t of query block i, critical set S_i, the other blocks U_i:

  o_t = N_t / D_t
  N_t = sum_{j in S_i} sum_n e^{s_tn} v_n + sum_{j in U_i} a_tj Vsum_j + (q_t / sqrt(D)) Hbar sum_{j in U_i} a_tj
  D_t = sum_{j in S_i} sum_n e^{s_tn}     + sum_{j in U_i} a_tj n_j

with s_tn = q_t . k_n / sqrt(D), a_tj = exp(q_t . kbar_j / sqrt(D)), kbar_j the mean of block
j's valid keys, n_j their count, Vsum_j = sum_n v_n, H_j = sum_n (k_n - kbar_j) v_n^T (D x D,
the block's first-order matrix) and Hbar the mean of H_j over all KV blocks.

Readings where the page is silent or loose:

* scale: the page's equation omits 1/sqrt(D); every exponent here carries it, so the
  first-order term (the derivative of e^{q k / sqrt(D)} in k) carries q / sqrt(D);
* stabiliser: both N_t and D_t are taken relative to the row maximum over the exact scores
  and the centroid scores (it cancels in the ratio);
* denominator: the page prints only N_t. The zero-order term of block j's exponential sum is
  n_j a_tj; its first-order term, a_tj q_t . sum_n (k_n - kbar_j) / sqrt(D), is zero exactly;
* Hbar: the mean over all KV blocks (the page: over all blocks);
* routing: the critical sets come from the caller's labels (SLA's router: label 2); every
  other block, marginal or negligible, is in U_i. PISA's covariance-aware top-k, which
  mixes the score with ||H_j - Hbar||_2 in a way the page does not state, is not built.

Parity status: pinned by every block critical reducing to dense softmax attention, by blocks
of identical keys (where the expansion is exact and Hbar = 0) reducing to dense attention for
any critical set, and by the error against dense attention falling as the square of the key
spread when every block has the same first-order matrix (a missing or mis-signed first-order
term leaves a first-order error).
"""

from __future__ import annotations

import math

import numpy as np

from .sla_oracle import CRITICAL, as_f64, block_counts


def block_statistics(k: np.ndarray, v: np.ndarray, block_kv: int):
    """(kbar [Nk, D], n [Nk], Vsum [Nk, D], H [Nk, D, D]) over each block's valid tokens."""
    N, D = k.shape
    Nk = -(-N // block_kv)
    kbar = np.zeros((Nk, D))
    n = np.zeros(Nk)
    vsum = np.zeros((Nk, D))
    H = np.zeros((Nk, D, D))
    for j in range(Nk):
        a, e = j * block_kv, min(N, (j + 1) * block_kv)
        kb, vb = k[a:e], v[a:e]
        kbar[j] = kb.mean(axis=0)
        n[j] = e - a
        vsum[j] = vb.sum(axis=0)
        H[j] = (kb - kbar[j]).T @ vb
    return kbar, n, vsum, H


def forward_pisa(q, k, v, block_q: int, block_kv: int, mask) -> np.ndarray:
    """PISA output o [B,H,N,D] (module docstring) with the critical blocks of `mask`."""
    q, k, v = as_f64(q), as_f64(k), as_f64(v)
    B, H_, N, D = q.shape
    Nq, Nk, _, _ = block_counts(N, block_q, block_kv, 0.0, 0.0)
    mask = np.asarray(mask, dtype=np.int8)
    if mask.shape != (B, H_, Nq, Nk):
        raise ValueError("mask shape must be [B, H, Nq, Nk]")
    scale = 1.0 / math.sqrt(D)
    O = np.empty((B, H_, N, D))
    for b in range(B):
        for h in range(H_):
            kbar, n, vsum, Hj = block_statistics(k[b, h], v[b, h], block_kv)
            Hbar = Hj.mean(axis=0)
            for i in range(Nq):
                s, e = i * block_q, min(N, (i + 1) * block_q)
                qb = q[b, h, s:e]
                crit = mask[b, h, i] == CRITICAL
                keys = np.concatenate([np.arange(j * block_kv, min(N, (j + 1) * block_kv))
                                       for j in np.nonzero(crit)[0]] or [np.zeros(0, dtype=int)])
                S = qb @ k[b, h, keys].T * scale                  # exact scores [rows, keys]
                C = qb @ kbar[~crit].T * scale                    # centroid scores [rows, |U|]
                m = np.max(np.concatenate([S, C], axis=1), axis=1, keepdims=True)
                Pe = np.exp(S - m)
                A = np.exp(C - m)
                num = Pe @ v[b, h, keys] + A @ vsum[~crit] + (qb * scale) @ Hbar * A.sum(axis=1, keepdims=True)
                den = Pe.sum(axis=1) + A @ n[~crit]
                O[b, h, s:e] = num / den[:, None]
    return O
