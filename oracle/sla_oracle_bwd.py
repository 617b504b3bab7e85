"""fp64 reference of the SLA backward pass (test infrastructure only).

Source: "SLA: Beyond Sparsity in Diffusion Transformers via Fine-Tunable Sparse-Linear
Attention", Abstract: one kernel covers the forward and the backward pass. The pages give no
backward formulas, so the backward here is the exact derivative of the forward of
``sla_oracle.forward`` with respect to Q, K, V and alpha, with the block labels held fixed:
the hard top-k labels are piecewise constant in Q and K and pass no gradient (the
differentiable SoftTop-k of SLA2 §2.B is a training-time router with learned weights, out of
scope here).

With dO = dL/dO [B,H,N,D], per (b, h) and query block i (rows t, block labels M_i):

  G_s = alpha_h * dO,  G_l = (1 - alpha_h) * dO           (alpha per channel)
  dalpha_h += sum_t dO_t * (O_s,t - O_l,t)

  sparse branch, keys n of the critical blocks (valid tokens), s = q k / sqrt(D), P = softmax:
    dV_n += sum_t P_tn G_s,t
    dS_tn = P_tn (G_s,t . v_n - G_s,t . O_s,t)
    dQ_t += sum_n dS_tn k_n / sqrt(D),  dK_n += sum_t dS_tn q_t / sqrt(D)

  linear branch, u = phi(q_t), num = u H_i, den = u . Z_i, O_l = num / den:
    dnum = G_l,t / den,  dden = -(G_l,t . O_l,t) / den
    dQ_t += (H_i dnum + Z_i dden) * phi'(q_t)
    dH_i += sum_t u dnum^T,  dZ_i += sum_t u dden   -> every marginal block j of row i
  states, h_j = sum_n phi(k_n) v_n^T, z_j = sum_n phi(k_n) over the block's valid tokens:
    dV_n += phi(k_n) dh_j,  dK_n += (dh_j v_n + dz_j) * phi'(k_n)

  phi(x) = x + 1 (x > 0), e^x (x <= 0); phi'(x) = 1 (x > 0), e^x (x <= 0), continuous at 0.

An empty critical set (O_s = 0) or an empty marginal set (O_l = 0) contributes nothing.

Parity status: pinned by central finite differences through ``sla_oracle.forward`` (every
input, mixed labels, tails, empty branches), by torch autograd of dense softmax attention
(every block critical) and of linear attention (every block marginal), and by exact zeros
for keys that are negligible in every row.
"""

from __future__ import annotations

import math
from typing import Tuple

import numpy as np

from .sla_oracle import CRITICAL, MARGINAL, as_f64, block_counts, kv_states, marginal_sums, phi


def dphi(x) -> np.ndarray:
    """Derivative of phi: 1 for x > 0, e^x for x <= 0."""
    x = np.asarray(x, dtype=np.float64)
    return np.where(x > 0, 1.0, np.exp(np.minimum(x, 0.0)))


def _block_tokens(j: int, block_kv: int, N: int) -> np.ndarray:
    return np.arange(j * block_kv, min(N, (j + 1) * block_kv))


def backward(q, k, v, alpha, block_q: int, block_kv: int, mask, dO) -> Tuple[np.ndarray, ...]:
    """(dQ, dK, dV [B,H,N,D], dalpha [H,D]) of L = sum(dO * O) with the labels `mask` fixed."""
    q, k, v, alpha, dO = as_f64(q), as_f64(k), as_f64(v), as_f64(alpha), as_f64(dO)
    B, H, N, D = q.shape
    Nq, Nk, _, _ = block_counts(N, block_q, block_kv, 0.0, 0.0)
    mask = np.asarray(mask, dtype=np.int8)
    if mask.shape != (B, H, Nq, Nk):
        raise ValueError("mask shape must be [B, H, Nq, Nk]")
    scale = 1.0 / math.sqrt(D)
    dQ, dK, dV = np.zeros_like(q), np.zeros_like(k), np.zeros_like(v)
    dalpha = np.zeros((H, D))
    for b in range(B):
        for h in range(H):
            hst, zst = kv_states(k[b, h], v[b, h], block_kv)
            Hs, Zs = marginal_sums(mask[b, h], hst, zst)
            dh = np.zeros((Nk, D, D))
            dz = np.zeros((Nk, D))
            a = alpha[h]
            for i in range(Nq):
                s, e = i * block_q, min(N, (i + 1) * block_q)
                row = mask[b, h, i]
                qb, g = q[b, h, s:e], dO[b, h, s:e]
                crit = np.nonzero(row == CRITICAL)[0]
                marg = np.nonzero(row == MARGINAL)[0]
                O_s = np.zeros_like(qb)
                if len(crit):
                    keys = np.concatenate([_block_tokens(j, block_kv, N) for j in crit])
                    Kc, Vc = k[b, h, keys], v[b, h, keys]
                    S = qb @ Kc.T * scale
                    P = np.exp(S - S.max(axis=1, keepdims=True))
                    P /= P.sum(axis=1, keepdims=True)
                    O_s = P @ Vc
                    Gs = a * g
                    dV[b, h, keys] += P.T @ Gs
                    dS = P * (Gs @ Vc.T - (Gs * O_s).sum(axis=1, keepdims=True))
                    dQ[b, h, s:e] += dS @ Kc * scale
                    dK[b, h, keys] += dS.T @ qb * scale
                O_l = np.zeros_like(qb)
                if len(marg):
                    u = phi(qb)
                    den = u @ Zs[i]
                    O_l = (u @ Hs[i]) / den[:, None]
                    Gl = (1.0 - a) * g
                    dnum = Gl / den[:, None]
                    dden = -(Gl * O_l).sum(axis=1) / den
                    du = dnum @ Hs[i].T + dden[:, None] * Zs[i][None, :]
                    dQ[b, h, s:e] += du * dphi(qb)
                    dHi = u.T @ dnum
                    dZi = u.T @ dden
                    for j in marg:
                        dh[j] += dHi
                        dz[j] += dZi
                dalpha[h] += (g * (O_s - O_l)).sum(axis=0)
            for j in range(Nk):
                toks = _block_tokens(j, block_kv, N)
                kj, vj = k[b, h, toks], v[b, h, toks]
                dV[b, h, toks] += phi(kj) @ dh[j]
                dK[b, h, toks] += (vj @ dh[j].T + dz[j][None, :]) * dphi(kj)
    return dQ, dK, dV, dalpha
