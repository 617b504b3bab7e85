"""fp64 reference of the low-bit (FP8 e4m3) sparse branch (test infrastructure only).

Source: "SLA2: Sparse-Linear Attention with Learnable Routing and QAT", §2.C: the sparse
attention branch runs with low-bit (INT8/FP8) operands in the forward pass, the backward
pass stays in 16-bit. The page names no format details, so this module takes the plainest
reading that keeps every quantised value exactly reproducible:

* format: e4m3 (1 sign, 4 exponent bits with bias 7, 3 mantissa bits; largest finite 448,
  smallest normal 2^-6, subnormals in steps of 2^-9; no infinities), rounding to nearest
  with ties to even, saturating at +-448;
* both matmuls of the sparse branch take e4m3 operands: Q K^T and P V;
* Q is scaled per query block, K and V per KV block, by a power of two
  s = 2^(ceil(log2(amax)) - 8), so amax / s lies in (128, 256] and the scaling is exact;
* P is quantised as a single-pass (online-softmax) kernel produces it. Per query row the
  critical KV blocks are visited in ascending index order, in log2 units x = s * log2(e).
  A reference r starts at the first block's row maximum. It moves to a later block's row
  maximum only when that exceeds r by more than P8_SLACK = 8, so every P = 2^(x - r)
  stays at or below 2^8;
* the P of a key in block j is quantised in the units of the largest V scale among the
  row's critical blocks, s_max, at its own value (2^P8_REF_EXP = 2^0): e4m3(P * sv_j /
  s_max) (sv_j / s_max is a power of two <= 1, applied before rounding; the largest
  argument, 2^8 = 256 < 448, never saturates, and e4m3's range below it reaches P = 2^-10).
  It multiplies V_j's codes, is carried to the final reference R by 2^(r - R), and the sum
  is scaled by s_max;
* the softmax normaliser l = sum over the row's critical keys of 2^(x - R) uses the
  unquantised P (the low-bit operands feed the matmuls, the normalisation stays in full
  precision); everything else (router, linear branch, blend) is the full-precision path of
  ``sla_oracle``.

Parity status: the e4m3 rounding and decoding are pinned by the format (every finite code is
a fixed point, halfway cases go to the even code, saturation, subnormal steps, torch's own
float8_e4m3fn); the branch is pinned by the exact case (operands already on the scaled e4m3
grid and P exactly representable, with V blocks at different scales) reducing to the
full-precision branch, by the underflow case (a V block 2^18 below the row's largest drops
out of the numerator but not out of l), and by hand-worked two-block rows on either side of
the reference's slack. Other values are the definition above.
"""

from __future__ import annotations

import math
from typing import Iterable, Optional, Sequence, Tuple

import numpy as np

from .sla_oracle import (CRITICAL, MARGINAL, as_f64, block_counts, compressed_scores, kv_states, linear_branch,
                         marginal_sums, route_from_scores)

E4M3_MAX = 448.0
P8_REF_EXP = 0    # P is quantised at 2^0 times its value
P8_SLACK = 8.0    # log2 units a block maximum may exceed the reference before it moves
# Decisions a float32 kernel may take the other way (see ``sparse_branch_fp8``): a rounding
# of P within this relative distance of the midpoint between two codes, and a reference
# move within this many log2 units of the slack.
NEAR_MIDPOINT_REL = 3e-5
NEAR_SLACK_ABS = 1e-4


def e4m3_round(x) -> np.ndarray:
    """Round to the nearest e4m3 value (ties to the even code), saturating at +-448."""
    x = np.asarray(x, dtype=np.float64)
    ax = np.abs(x)
    _, ex = np.frexp(ax)  # ax = f * 2^ex with f in [0.5, 1): the binade is [2^(ex-1), 2^ex)
    e = ex.astype(np.float64) - 1.0
    # quantum: 2^(e-3) for normal values (exponent e >= -6), 2^-9 in the subnormal range
    quantum = np.exp2(np.maximum(e, -6.0) - 3.0)
    r = np.round(ax / quantum) * quantum  # np.round rounds halfway cases to even
    r = np.minimum(r, E4M3_MAX)
    return np.where(x < 0, -r, r)


def e4m3_decode(codes) -> np.ndarray:
    """Value of each e4m3 byte (uint8 array): sign bit 7, exponent bits 3..6 (bias 7),
    mantissa bits 0..2; exponent 0 is the subnormal range M * 2^-9. The code with all
    exponent and mantissa bits set is NaN."""
    c = np.asarray(codes, dtype=np.uint8).astype(np.int64)
    sign = np.where(c & 0x80, -1.0, 1.0)
    E = (c >> 3) & 0xF
    M = c & 0x7
    mag = np.where(E == 0, M * 2.0 ** -9, (1.0 + M / 8.0) * np.exp2(E - 7.0))
    mag = np.where((E == 15) & (M == 7), np.nan, mag)
    return sign * mag


def pow2_scale(amax: float) -> float:
    """2^(ceil(log2(amax)) - 8): amax / scale lies in (128, 256]; 1 for amax = 0."""
    if amax <= 0:
        return 1.0
    return math.ldexp(1.0, math.ceil(math.log2(amax)) - 8)


def quantize_blocks(x: np.ndarray, block: int) -> Tuple[np.ndarray, np.ndarray]:
    """Per-block power-of-two scales and the e4m3 codes (as float64 values) of x [N, D]."""
    N = x.shape[0]
    q = np.empty_like(x)
    scales = []
    for s in range(0, N, block):
        e = min(N, s + block)
        sc = pow2_scale(float(np.abs(x[s:e]).max()))
        scales.append(sc)
        q[s:e] = e4m3_round(x[s:e] / sc)
    return q, np.asarray(scales)


def online_references(x_blocks: Sequence[np.ndarray]) -> Tuple[list, np.ndarray]:
    """Per-row reference (log2 units) in effect while each block is processed, and the rows
    where some block's maximum lies within NEAR_SLACK_ABS of the slack (a move a float32
    kernel may decide the other way).

    x_blocks[b] is [rows, keys of block b] in the order the blocks are visited."""
    r = x_blocks[0].max(axis=1)
    refs = [r]
    near = np.zeros(r.shape, dtype=bool)
    for xb in x_blocks[1:]:
        mb = xb.max(axis=1)
        near |= np.abs(mb - (r + P8_SLACK)) <= NEAR_SLACK_ABS
        r = np.where(mb > r + P8_SLACK, mb, r)
        refs.append(r)
    return refs, near


def e4m3_quantum(y) -> np.ndarray:
    """Spacing of the e4m3 codes around |y| (the binade's step, 2^-9 below 2^-6)."""
    _, ex = np.frexp(np.abs(np.asarray(y, dtype=np.float64)))
    return np.exp2(np.maximum(ex.astype(np.float64) - 1.0, -6.0) - 3.0)


def sparse_branch_fp8(q_blk: np.ndarray, k: np.ndarray, v: np.ndarray, crit_blocks: Sequence[int],
                      block_kv: int, with_slack: bool = False, x_rel_perturb: float = 0.0):
    """The sparse branch with e4m3 operands for Q K^T and P V (module docstring).

    Returns (O_s [bq, D], l [bq]) with l relative to the final reference; with no critical
    block both are 0.

    with_slack=True also returns (slack [bq, D], near_rows [bq]). A kernel computes P in
    float32, so where P (times the V-scale ratio) lies within NEAR_MIDPOINT_REL of the
    midpoint between two e4m3 codes it may round to the other code; slack bounds, per
    element, how far O_s moves if every such key takes its other code. near_rows marks the
    rows whose reference moves are themselves that close (NEAR_SLACK_ABS).
    x_rel_perturb: the rounding (and only the rounding) sees 2^((x - r)(1 + x_rel_perturb))
    in place of P, a test hook standing for float32 error in P.
    """
    N, D = k.shape
    if len(crit_blocks) == 0:
        z = np.zeros((q_blk.shape[0], D)), np.zeros(q_blk.shape[0])
        return z + (np.zeros((q_blk.shape[0], D)), np.zeros(q_blk.shape[0], dtype=bool)) if with_slack else z
    blocks = sorted(int(j) for j in crit_blocks)
    sq = pow2_scale(float(np.abs(q_blk).max()))
    qh = e4m3_round(q_blk / sq)
    x_blocks, vh_blocks, sv = [], [], []
    for j in blocks:
        a, e = j * block_kv, min(N, (j + 1) * block_kv)
        sk = pow2_scale(float(np.abs(k[a:e]).max()))
        s_j = (qh @ e4m3_round(k[a:e] / sk).T) * (sq * sk) / math.sqrt(D)
        x_blocks.append(s_j * math.log2(math.e))
        sv_j = pow2_scale(float(np.abs(v[a:e]).max()))
        vh_blocks.append(e4m3_round(v[a:e] / sv_j))
        sv.append(sv_j)
    s_max = max(sv)
    refs, near_rows = online_references(x_blocks)
    R = refs[-1]
    ref = 2.0 ** P8_REF_EXP
    num = np.zeros((q_blk.shape[0], D))
    slack = np.zeros((q_blk.shape[0], D))
    l = np.zeros(q_blk.shape[0])
    for xb, vh, sv_j, r in zip(x_blocks, vh_blocks, sv, refs):
        p = np.exp2(xb - r[:, None])
        y = ref * p * (sv_j / s_max)
        y_seen = y * np.exp2((xb - r[:, None]) * x_rel_perturb) if x_rel_perturb else y
        pq = e4m3_round(y_seen) / ref
        carry = np.exp2(r - R)[:, None]
        num += (pq @ vh) * carry
        l += (p * carry).sum(axis=1)
        if with_slack:
            qn = e4m3_quantum(y)
            t = y / qn
            near = np.abs(t - np.floor(t) - 0.5) * qn <= NEAR_MIDPOINT_REL * y
            slack += ((near * qn / ref * carry) @ np.abs(vh))
    out = num * s_max / l[:, None], l
    if with_slack:
        return out + (slack * s_max / l[:, None], near_rows)
    return out


def forward_fp8(q, k, v, alpha, block_q: int, block_kv: int, kh: float = 0.0, kl: float = 0.0, mask=None,
                heads: Optional[Iterable[Tuple[int, int]]] = None, query_blocks: Optional[Iterable[int]] = None,
                with_slack: bool = False):
    """SLA forward with the low-bit sparse branch; router and linear branch as in ``forward``.

    ``heads`` (list of (b, h)) and ``query_blocks`` (list of i) restrict the work to a
    sample; rows outside it are NaN in the returned float64 [B,H,N,D] array. With
    ``with_slack`` the result is (O, slack, near_rows): alpha times the sparse branch's
    slack [B,H,N,D] and its near rows [B,H,N] (``sparse_branch_fp8``)."""
    q, k, v, alpha = as_f64(q), as_f64(k), as_f64(v), as_f64(alpha)
    B, H, N, D = q.shape
    Nq, Nk, kc, kn = block_counts(N, block_q, block_kv, kh, kl)
    heads = [(b, h) for b in range(B) for h in range(H)] if heads is None else list(heads)
    qbs = list(range(Nq)) if query_blocks is None else list(query_blocks)
    if mask is None:
        mask = np.zeros((B, H, Nq, Nk), dtype=np.int8)
        for b, h in heads:
            mask[b, h] = route_from_scores(compressed_scores(q[b, h], k[b, h], block_q, block_kv), kc, kn)
    mask = np.asarray(mask, dtype=np.int8)
    O = np.full((B, H, N, D), np.nan)
    slack = np.zeros((B, H, N, D))
    near_rows = np.zeros((B, H, N), dtype=bool)
    for b, h in heads:
        hst, zst = kv_states(k[b, h], v[b, h], block_kv)
        Hs, Zs = marginal_sums(mask[b, h, qbs], hst, zst)
        for r, i in enumerate(qbs):
            s, e = i * block_q, min(N, (i + 1) * block_q)
            row = mask[b, h, i]
            res = sparse_branch_fp8(q[b, h, s:e], k[b, h], v[b, h], np.nonzero(row == CRITICAL)[0], block_kv,
                                    with_slack=with_slack)
            ol_, _ = linear_branch(q[b, h, s:e], Hs[r], Zs[r], int(np.count_nonzero(row == MARGINAL)))
            O[b, h, s:e] = alpha[h] * res[0] + (1.0 - alpha[h]) * ol_
            if with_slack:
                slack[b, h, s:e] = alpha[h] * res[2]
                near_rows[b, h, s:e] = res[3]
    if with_slack:
        return O, slack, near_rows
    return O
