"""fp64 reference implementation of the SLA forward pass (test infrastructure only).

Layout conventions: q, k, v are [B, H, N, D]; alpha is [H, D]; block labels are
int8 [B, H, Nq, Nk] with 2 = critical, 1 = marginal, 0 = negligible. Query block
i covers tokens [i*bq, min(N, (i+1)*bq)), KV block j covers
[j*bk, min(N, (j+1)*bk)).
"""

from __future__ import annotations

import math
from typing import Iterable, Optional, Sequence, Tuple

import numpy as np

CRITICAL = 2
MARGINAL = 1
NEGLIGIBLE = 0


def as_f64(x) -> np.ndarray:
    """Decode a tensor (torch bf16/fp32 or numpy) exactly into a float64 numpy array."""
    if hasattr(x, "detach"):  # torch tensor; bf16 -> f64 is exact
        import torch

        return x.detach().to("cpu", torch.float64).numpy()
    return np.asarray(x, dtype=np.float64)


def block_counts(N: int, block_q: int, block_kv: int, kh: float, kl: float) -> Tuple[int, int, int, int]:
    """Number of query blocks, KV blocks, critical and negligible blocks per row.

    The SLA abstract splits the blocks of a row into critical, marginal and
    negligible; the SLA2 router (§2.B) keeps a hard top-k. The pages give the
    fractions only, so the counts are read as: critical rounded up, negligible
    rounded down, both in integer parts-per-million to keep float artefacts out.
    """
    if N < 1 or block_q < 1 or block_kv < 1:
        raise ValueError("N and block sizes must be positive")
    kh_ppm = int(round(kh * 1e6))
    kl_ppm = int(round(kl * 1e6))
    if not (0 <= kh_ppm <= 1_000_000 and 0 <= kl_ppm <= 1_000_000 and kh_ppm + kl_ppm <= 1_000_000):
        raise ValueError("need 0 <= kh, kl and kh + kl <= 1")
    Nq = -(-N // block_q)
    Nk = -(-N // block_kv)
    kc = -(-(kh_ppm * Nk) // 1_000_000)
    kn = (kl_ppm * Nk) // 1_000_000
    return Nq, Nk, kc, kn


def phi(x: np.ndarray) -> np.ndarray:
    """Linear-attention feature map elu(x) + 1: x + 1 for x > 0, exp(x) for x <= 0."""
    x = np.asarray(x, dtype=np.float64)
    return np.where(x > 0, x + 1.0, np.exp(np.minimum(x, 0.0)))


def _block_ranges(N: int, block: int):
    return [(s, min(N, s + block)) for s in range(0, N, block)]


def pool_mean(x: np.ndarray, block: int) -> np.ndarray:
    """Mean of the valid tokens of every block along axis -2 (SLA2 §2.B pooling of adjacent tokens)."""
    N = x.shape[-2]
    return np.stack([x[..., s:e, :].mean(axis=-2) for s, e in _block_ranges(N, block)], axis=-2)


def compressed_scores(q: np.ndarray, k: np.ndarray, block_q: int, block_kv: int) -> np.ndarray:
    """S = pool(Q) pool(K)^T / sqrt(D), [..., Nq, Nk] (SLA2 §2.B; identity router projections)."""
    D = q.shape[-1]
    qbar = pool_mean(q, block_q)
    kbar = pool_mean(k, block_kv)
    return np.matmul(qbar, np.swapaxes(kbar, -1, -2)) / math.sqrt(D)


def compressed_probs(S: np.ndarray) -> np.ndarray:
    """P_c = row softmax of the compressed scores."""
    e = np.exp(S - S.max(axis=-1, keepdims=True))
    return e / e.sum(axis=-1, keepdims=True)


def route_from_scores(S: np.ndarray, kc: int, kn: int) -> np.ndarray:
    """Label every block of every row from its scores.

    Per row the blocks are put in the total order (score descending, index
    ascending); the first kc are critical, the last kn negligible, the others
    marginal (SLA abstract; hard top-k of SLA2 §2.B).
    """
    Nk = S.shape[-1]
    if kc + kn > Nk:
        raise ValueError("kc + kn exceeds the number of KV blocks")
    idx = np.broadcast_to(np.arange(Nk), S.shape)
    # lexsort: the last key is the primary one -> (-S ascending, then j ascending).
    order = np.lexsort((idx, -S), axis=-1)
    rank = np.empty_like(order)
    np.put_along_axis(rank, order, np.broadcast_to(np.arange(Nk), S.shape), axis=-1)
    mask = np.full(S.shape, MARGINAL, dtype=np.int8)
    mask[rank < kc] = CRITICAL
    mask[rank >= Nk - kn] = NEGLIGIBLE
    return mask


def route(q, k, block_q: int, block_kv: int, kh: float, kl: float):
    """Block router: returns (mask [B,H,Nq,Nk] int8, S [B,H,Nq,Nk] float64)."""
    q = as_f64(q)
    k = as_f64(k)
    N = q.shape[-2]
    _, _, kc, kn = block_counts(N, block_q, block_kv, kh, kl)
    S = compressed_scores(q, k, block_q, block_kv)
    return route_from_scores(S, kc, kn), S


def kv_states(k, v, block_kv: int):
    """Per-KV-block linear-attention states h_j = phi(K_j)^T V_j and z_j = colsum phi(K_j).

    Returns h [B,H,Nk,D,D] and z [B,H,Nk,D] (valid tokens only).
    """
    k = as_f64(k)
    v = as_f64(v)
    N = k.shape[-2]
    fk = phi(k)
    hs, zs = [], []
    for s, e in _block_ranges(N, block_kv):
        hs.append(np.matmul(np.swapaxes(fk[..., s:e, :], -1, -2), v[..., s:e, :]))
        zs.append(fk[..., s:e, :].sum(axis=-2))
    return np.stack(hs, axis=-3), np.stack(zs, axis=-2)


def sparse_branch(q_blk: np.ndarray, k: np.ndarray, v: np.ndarray, crit_blocks: Sequence[int],
                  block_kv: int) -> Tuple[np.ndarray, np.ndarray]:
    """Exact softmax attention of one query block over the tokens of its critical KV blocks.

    The softmax is normalised over the critical keys only (SLA2 §1 item 1: the
    sparse branch re-normalises). Returns (O_s [bq, D], row sums l [bq]); with no
    critical block O_s = 0 and l = 0.
    """
    N, D = k.shape
    if len(crit_blocks) == 0:
        return np.zeros((q_blk.shape[0], D)), np.zeros(q_blk.shape[0])
    keys = np.concatenate([np.arange(j * block_kv, min(N, (j + 1) * block_kv)) for j in crit_blocks])
    s = np.matmul(q_blk, k[keys].T) / math.sqrt(D)
    m = s.max(axis=1, keepdims=True)
    p = np.exp(s - m)
    l = p.sum(axis=1)
    return np.matmul(p, v[keys]) / l[:, None], l


def marginal_sums(labels_rows: np.ndarray, h: np.ndarray, z: np.ndarray) -> Tuple[np.ndarray, np.ndarray]:
    """H_i = sum of h_j and Z_i = sum of z_j over the marginal blocks j of each row i.

    ``labels_rows`` is [R, Nk]; returns H [R, D, D] and Z [R, D]. The sums are
    written as one product with the 0/1 marginal indicator (a plain summation;
    the matmul only serves as the adder).
    """
    w = (labels_rows == MARGINAL).astype(np.float64)  # [R, Nk]
    Nk, D = z.shape
    Hs = (w @ h.reshape(Nk, D * D)).reshape(-1, D, D)
    Zs = w @ z
    return Hs, Zs


def linear_branch(q_blk: np.ndarray, H_i: np.ndarray, Z_i: np.ndarray,
                  n_marginal: int) -> Tuple[np.ndarray, np.ndarray]:
    """Linear attention of one query block over its marginal KV blocks.

    O_l = phi(Q_i) H_i / (phi(Q_i) Z_i) where H_i, Z_i are the sums of the
    marginal blocks' states (SLA abstract: O(N) attention for marginal weights).
    Returns (O_l [bq, D], denominators [bq]); with no marginal block both are 0.
    """
    D = H_i.shape[-1]
    if n_marginal == 0:
        return np.zeros((q_blk.shape[0], D)), np.zeros(q_blk.shape[0])
    fq = phi(q_blk)
    den = fq @ Z_i
    return (fq @ H_i) / den[:, None], den


def forward(q, k, v, alpha, block_q: int, block_kv: int, kh: float = 0.0, kl: float = 0.0,
            mask: Optional[np.ndarray] = None, heads: Optional[Iterable[Tuple[int, int]]] = None,
            query_blocks: Optional[Iterable[int]] = None, return_parts: bool = False):
    """SLA forward with the SLA2 blend, O = alpha * O_s + (1 - alpha) * O_l (SLA2 §2.A).

    ``mask`` (int8 labels) replaces the router when given. ``heads`` (list of
    (b, h)) and ``query_blocks`` (list of i) restrict the work to a sample; rows
    outside the sample are left as NaN in the returned float64 [B,H,N,D] array.
    With ``return_parts`` the result is (O, parts) where parts holds the mask,
    scores, O_s, O_l and the softmax / linear denominators.
    """
    q = as_f64(q)
    k = as_f64(k)
    v = as_f64(v)
    alpha = as_f64(alpha)
    B, H, N, D = q.shape
    Nq, Nk, kc, kn = block_counts(N, block_q, block_kv, kh, kl)
    if heads is None:
        heads = [(b, h) for b in range(B) for h in range(H)]
    heads = list(heads)
    qbs = list(range(Nq)) if query_blocks is None else list(query_blocks)

    S = None
    if mask is None:
        S = np.full((B, H, Nq, Nk), np.nan)
        mask = np.zeros((B, H, Nq, Nk), dtype=np.int8)
        for b, h in heads:
            S[b, h] = compressed_scores(q[b, h], k[b, h], block_q, block_kv)
            mask[b, h] = route_from_scores(S[b, h], kc, kn)
    mask = np.asarray(mask, dtype=np.int8)
    if mask.shape != (B, H, Nq, Nk):
        raise ValueError("mask shape must be [B, H, Nq, Nk]")

    O = np.full((B, H, N, D), np.nan)
    Os = np.full((B, H, N, D), np.nan)
    Ol = np.full((B, H, N, D), np.nan)
    lsum = np.full((B, H, N), np.nan)
    lden = np.full((B, H, N), np.nan)
    for b, h in heads:
        hst, zst = kv_states(k[b, h], v[b, h], block_kv)
        Hs, Zs = marginal_sums(mask[b, h, qbs], hst, zst)
        for r, i in enumerate(qbs):
            s, e = i * block_q, min(N, (i + 1) * block_q)
            row = mask[b, h, i]
            crit = np.nonzero(row == CRITICAL)[0]
            n_marg = int(np.count_nonzero(row == MARGINAL))
            os_, l_ = sparse_branch(q[b, h, s:e], k[b, h], v[b, h], crit, block_kv)
            ol_, d_ = linear_branch(q[b, h, s:e], Hs[r], Zs[r], n_marg)
            a = alpha[h]
            O[b, h, s:e] = a * os_ + (1.0 - a) * ol_
            Os[b, h, s:e], Ol[b, h, s:e] = os_, ol_
            lsum[b, h, s:e], lden[b, h, s:e] = l_, d_
    if return_parts:
        return O, dict(mask=mask, S=S, O_s=Os, O_l=Ol, softmax_sum=lsum, linear_den=lden,
                       counts=(Nq, Nk, kc, kn))
    return O
