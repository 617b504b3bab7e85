"""fp64 reference of the low-bit (FP8 e4m3) sparse branch (test infrastructure only).

Source: "SLA2: Sparse-Linear Attention with Learnable Routing and QAT", §2.C: the sparse
attention branch runs with low-bit (INT8/FP8) operands in the forward pass, the backward
pass stays in 16-bit. The page names no format, no scales and no point at which the
softmax weights are rounded. This module takes the plainest reading that keeps the
quantised operands exactly reproducible and leaves the rounding of P to the kernel:

* format: e4m3 (1 sign, 4 exponent bits with bias 7, 3 mantissa bits; largest finite 448,
  smallest normal 2^-6, subnormals in steps of 2^-9; no infinities), rounding to nearest
  with ties to even, saturating at +-448;
* both matmuls of the sparse branch take e4m3 operands: Q K^T and P V;
* Q is scaled per query block, K and V per KV block, by a power of two
  s = 2^(ceil(log2(amax)) - 8), so amax / s lies in (128, 256] and the scaling is exact;
* P enters P V as e4m3 codes. In log2 units x_n = (q . k_n / sqrt(D)) log2(e) over the
  row's critical keys, with m = max_n x_n, the code of key n (in KV block j) is
  e4m3(2^(x_n - r_n) * sv_j / u) for some reference r_n <= m and some power-of-two unit
  u with sv_j <= u <= s_max (the largest V scale among the row's critical blocks), such
  that no code saturates. The reading fixes neither r_n nor u: a single-pass kernel cannot
  know m before it has seen every block, so every such choice is a valid result;
* the softmax normaliser l = sum_n 2^(x_n - m) uses the unrounded P (the low-bit operands
  feed the matmuls, the normalisation stays in full precision); router, linear branch and
  blend are the full-precision path of ``sla_oracle``.

``sparse_branch_fp8`` returns the centre of that set, O* = sum_n P_n vhat_n / l with P
unrounded (P_n = 2^(x_n - m), vhat_n the dequantised e4m3 V row), and a per-element bound
on how far any admissible rounding of P can move it. Half an e4m3 step is at most 2^-4 of
the value in the normal range and 2^-10 in the subnormal range, so a code of value y is off
by at most max(2^-4 y, 2^-10). Carried back to the row maximum's units (times
2^(r_n - m) u / sv_j <= u / sv_j) the error of key n in P_n vhat_n is at most
max(2^-4 P_n |vhat_n|, 2^-10 |vhat_n| s_max / sv_j), whatever r_n <= m and u <= s_max are.
The bound is the sum of those terms over the row's critical keys, divided by l.

Parity status: the e4m3 rounding and decoding are pinned by the format (every finite code is
a fixed point, halfway cases go to the even code, saturation, subnormal steps, torch's own
float8_e4m3fn); the centre reduces to the full-precision branch when the operands lie on
the scaled e4m3 grid; the bound is derived by hand on a two-block row, is attained by a
single key sitting half a step from a code, and holds for several single-pass rounding
schedules (the reference at the row maximum, at the running maximum, moved lazily, a
per-block unit) written independently in the tests.
"""

from __future__ import annotations

import math
from typing import Iterable, Optional, Sequence, Tuple

import numpy as np

from .sla_oracle import (CRITICAL, MARGINAL, as_f64, block_counts, compressed_scores, kv_states, linear_branch,
                         marginal_sums, route_from_scores)

E4M3_MAX = 448.0
# Half an e4m3 step, relative to the value in the normal range and absolute below 2^-6.
HALF_STEP_REL = 2.0 ** -4
HALF_STEP_ABS = 2.0 ** -10


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


def sparse_branch_fp8(q_blk: np.ndarray, k: np.ndarray, v: np.ndarray, crit_blocks: Sequence[int],
                      block_kv: int):
    """The sparse branch with e4m3 operands for Q K^T and P V (module docstring).

    Returns (O* [bq, D], l [bq], bound [bq, D]): the centre (P unrounded), the normaliser
    relative to the row maximum, and the largest move of O* any admissible rounding of P
    can cause. With no critical block all three are 0."""
    N, D = k.shape
    bq = q_blk.shape[0]
    if len(crit_blocks) == 0:
        return np.zeros((bq, D)), np.zeros(bq), np.zeros((bq, D))
    blocks = sorted(int(j) for j in crit_blocks)
    sq = pow2_scale(float(np.abs(q_blk).max()))
    qh = e4m3_round(q_blk / sq) * sq  # dequantised Q
    xs, vs, svs = [], [], []
    for j in blocks:
        a, e = j * block_kv, min(N, (j + 1) * block_kv)
        sk = pow2_scale(float(np.abs(k[a:e]).max()))
        kh = e4m3_round(k[a:e] / sk) * sk
        xs.append((qh @ kh.T) / math.sqrt(D) * math.log2(math.e))
        sv = pow2_scale(float(np.abs(v[a:e]).max()))
        vs.append(e4m3_round(v[a:e] / sv) * sv)
        svs.append(np.full(e - a, sv))
    x = np.concatenate(xs, axis=1)          # [bq, keys] log2 units
    vh = np.concatenate(vs, axis=0)         # [keys, D] dequantised V
    sv = np.concatenate(svs)                # [keys] the V scale of each key's block
    s_max = sv.max()
    m = x.max(axis=1)
    p = np.exp2(x - m[:, None])             # P_n, unrounded, <= 1
    l = p.sum(axis=1)
    o = (p @ vh) / l[:, None]
    # per key: max(2^-4 P_n, 2^-10 s_max / sv_n) |vhat_n|, summed over keys
    w = np.maximum(HALF_STEP_REL * p, HALF_STEP_ABS * (s_max / sv)[None, :])
    bound = (w @ np.abs(vh)) / l[:, None]
    return o, l, bound


def forward_fp8(q, k, v, alpha, block_q: int, block_kv: int, kh: float = 0.0, kl: float = 0.0, mask=None,
                heads: Optional[Iterable[Tuple[int, int]]] = None, query_blocks: Optional[Iterable[int]] = None,
                with_bound: bool = False):
    """SLA forward with the low-bit sparse branch; router and linear branch as in ``forward``.

    ``heads`` (list of (b, h)) and ``query_blocks`` (list of i) restrict the work to a
    sample; rows outside it are NaN in the returned float64 [B,H,N,D] array. The sparse
    branch is the centre O* (P unrounded). With ``with_bound`` the result is (O, bound):
    bound [B,H,N,D] is alpha times the sparse branch's bound, the largest move any
    admissible rounding of P can cause (``sparse_branch_fp8``)."""
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
    bound = np.zeros((B, H, N, D))
    for b, h in heads:
        hst, zst = kv_states(k[b, h], v[b, h], block_kv)
        Hs, Zs = marginal_sums(mask[b, h, qbs], hst, zst)
        for r, i in enumerate(qbs):
            s, e = i * block_q, min(N, (i + 1) * block_q)
            row = mask[b, h, i]
            os_, _, bd = sparse_branch_fp8(q[b, h, s:e], k[b, h], v[b, h], np.nonzero(row == CRITICAL)[0], block_kv)
            ol_, _ = linear_branch(q[b, h, s:e], Hs[r], Zs[r], int(np.count_nonzero(row == MARGINAL)))
            O[b, h, s:e] = alpha[h] * os_ + (1.0 - alpha[h]) * ol_
            bound[b, h, s:e] = alpha[h] * bd
    if with_bound:
        return O, bound
    return O
