// Per-row softmax arithmetic over one 64-key S block, shared by the attention kernels.
// A thread owns one query row; the block's 64 fp32 scores sit in two 32-register halves
// (columns 0..31 and 32..63), as one 32x32b.x32 TMEM load each delivers them.
//
// Source: "SLA: Beyond Sparsity in Diffusion Transformers via Fine-Tunable Sparse-Linear
// Attention", Abstract (exact softmax attention over the critical blocks); the online,
// block-by-block form of the softmax with a running reference maximum is the standard one.
#pragma once

#include "sm100.cuh"

namespace sla {

// The reference maximum m of a row is the row maximum of its tile's first block. A later
// block is exponentiated against it directly; only when the block's sum of 2^(s * scale - m)
// passes kRefMoveSum (some key beats m by more than ~14 in log2 units) does m move to the
// block's maximum, the accumulated row being rescaled by 2^(m_old - m_new). P and the sums
// stay far inside the fp32 and bf16 ranges, and no per-block maximum is needed.
constexpr float kRefMoveSum = 0x1p20f;

// Row maximum of one 64-column S block held as two 32-column halves (raw scores): four
// chains of 3-input maxima.
__device__ __forceinline__ float row_max64(const uint32_t (&sa)[32], const uint32_t (&sb)[32]) {
  float m0 = fmax3(__uint_as_float(sa[0]), __uint_as_float(sa[1]), __uint_as_float(sa[2]));
  float m1 = fmax3(__uint_as_float(sa[3]), __uint_as_float(sa[4]), __uint_as_float(sa[5]));
  float m2 = fmax3(__uint_as_float(sb[0]), __uint_as_float(sb[1]), __uint_as_float(sb[2]));
  float m3 = fmax3(__uint_as_float(sb[3]), __uint_as_float(sb[4]), __uint_as_float(sb[5]));
#pragma unroll
  for (int c = 6; c < 30; c += 4) {
    m0 = fmax3(m0, __uint_as_float(sa[c]), __uint_as_float(sa[c + 1]));
    m1 = fmax3(m1, __uint_as_float(sa[c + 2]), __uint_as_float(sa[c + 3]));
    m2 = fmax3(m2, __uint_as_float(sb[c]), __uint_as_float(sb[c + 1]));
    m3 = fmax3(m3, __uint_as_float(sb[c + 2]), __uint_as_float(sb[c + 3]));
  }
  m0 = fmax3(m0, __uint_as_float(sa[30]), __uint_as_float(sa[31]));
  m2 = fmax3(m2, __uint_as_float(sb[30]), __uint_as_float(sb[31]));
  return fmaxf(fmaxf(m0, m1), fmaxf(m2, m3));
}

// Columns OFF .. OFF + 31 of a block: a column at or past `valid`, or whose bit in `keep`
// is clear, takes -inf.
template <int OFF>
__device__ __forceinline__ void mask_scores(uint32_t (&x)[32], int valid, uint64_t keep) {
#pragma unroll
  for (int c = 0; c < 32; ++c)
    if (c + OFF >= valid || !((keep >> (c + OFF)) & 1ull)) x[c] = __float_as_uint(-INFINITY);
}

// p = 2^(s * scale - m) over a 64-column block held as two halves: one paired FMA per two
// elements (sc2 = scale, nm2 = -m in both lanes), one exponential per element; P as bf16
// pairs into pk (columns 0..31 then 32..63). Returns the block's sum as two fp32 partial sums.
__device__ __forceinline__ uint64_t exp2_block(const uint32_t (&sa)[32], const uint32_t (&sb)[32],
                                               uint32_t (&pk)[32], uint64_t sc2, uint64_t nm2) {
  uint64_t s0 = 0ull, s1 = 0ull;
#pragma unroll
  for (int c = 0; c < 32; c += 2) {
    const uint64_t x0 = f2_fma(static_cast<uint64_t>(sa[c]) | (static_cast<uint64_t>(sa[c + 1]) << 32), sc2, nm2);
    const uint64_t x1 = f2_fma(static_cast<uint64_t>(sb[c]) | (static_cast<uint64_t>(sb[c + 1]) << 32), sc2, nm2);
    const float e0 = fast_exp2(f2_lo(x0)), e1 = fast_exp2(f2_hi(x0));
    const float e2 = fast_exp2(f2_lo(x1)), e3 = fast_exp2(f2_hi(x1));
    s0 = f2_add(s0, f2_make(e0, e1));
    s1 = f2_add(s1, f2_make(e2, e3));
    pk[c >> 1] = pack_bf16x2(e0, e1);
    pk[16 + (c >> 1)] = pack_bf16x2(e2, e3);
  }
  return f2_add(s0, s1);
}

}  // namespace sla
