// Block router for the SLA forward.
//
//   score_kernel      : S_ij = qbar_i . kbar_j / sqrt(D) in fp64 (compressed scores;
//                       the scores output, and the input of select_kernel)
//   score32_kernel    : the same scores in fp32 plus the norms that bound their error
//   select_cert_kernel: per query-block row of up to 2048 blocks, label every KV block
//                       critical (2), marginal (1) or negligible (0): the first kc blocks
//                       in the total order (S descending, j ascending) are critical, the
//                       last kn negligible. Decided on the fp32 scores wherever the error
//                       bound allows, on fp64 scores recomputed for the rest.
//   select_kernel     : the same labels from fp64 scores, for longer rows.
//   mask_lists_kernel : the same outputs from a caller-supplied label mask.
//
// Sources: "SLA2: Sparse-Linear Attention with Learnable Routing and QAT" §2.B
// (pooled Q/K, compressed scores, hard top-k at inference); "SLA: Beyond
// Sparsity in Diffusion Transformers via Fine-Tunable Sparse-Linear Attention",
// Abstract (critical / marginal / negligible). The softmax of the compressed
// scores is monotone, so ranking the raw scores gives the same labels.
//
// The decision is taken in fp64 (pooled sums of bf16 inputs are exact in fp64
// for ordinary inputs), so labels differ from an fp64 reference only where two
// scores agree to the last bits.
#pragma once

#include "sm100.cuh"

namespace sla {

// ---------------------------------------------------------------- scores
// D(8x8) += A(8x4) * B(4x8) in fp64 on the tensor cores (one warp). Fragments:
// a = A[lane/4][lane%4], b = B[lane%4][lane/4], d = D[lane/4][2*(lane%4) + {0,1}].
__device__ __forceinline__ void dmma_8x8x4(double (&d)[2], double a, double b) {
  asm volatile("mma.sync.aligned.m8n8k4.row.col.f64.f64.f64.f64 {%0, %1}, {%2}, {%3}, {%0, %1};"
               : "+d"(d[0]), "+d"(d[1])
               : "d"(a), "d"(b));
}

// grid: (ceil(Nk/64), ceil(Nq/64), BH); block 128 = 2 x 2 warps, each warp a 32 x 32 patch
// of S as 4 x 4 tiles of 8 x 8. D is walked in chunks of 32 staged in shared memory.
template <int D>
__global__ void __launch_bounds__(128) score_kernel(const double* __restrict__ qbar, const double* __restrict__ kbar,
                                                    double* __restrict__ S, int Nq, int Nk) {
  constexpr int T = 64, DC = 32, LDS = DC + 1;
  __shared__ double sq[T * LDS];
  __shared__ double sk[T * LDS];
  const int bh = blockIdx.z, i0 = blockIdx.y * T, j0 = blockIdx.x * T;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int wy = warp >> 1, wx = warp & 1;
  grid_dep_launch();
  grid_dep_wait();  // pooled means come from the previous kernel
  const int fr = lane >> 2, fc = lane & 3;
  const double* qb = qbar + static_cast<size_t>(bh) * Nq * D;
  const double* kb = kbar + static_cast<size_t>(bh) * Nk * D;
  double acc[4][4][2];
#pragma unroll
  for (int a = 0; a < 4; ++a)
#pragma unroll
    for (int b = 0; b < 4; ++b) acc[a][b][0] = acc[a][b][1] = 0.0;
  for (int d0 = 0; d0 < D; d0 += DC) {
    for (int e = tid; e < T * DC; e += 128) {
      const int r = e / DC, d = e % DC;
      sq[r * LDS + d] = (i0 + r < Nq) ? qb[static_cast<size_t>(i0 + r) * D + d0 + d] : 0.0;
      sk[r * LDS + d] = (j0 + r < Nk) ? kb[static_cast<size_t>(j0 + r) * D + d0 + d] : 0.0;
    }
    __syncthreads();
#pragma unroll
    for (int kk = 0; kk < DC; kk += 4) {
      double af[4], bf[4];
#pragma unroll
      for (int a = 0; a < 4; ++a) af[a] = sq[(wy * 32 + a * 8 + fr) * LDS + kk + fc];
#pragma unroll
      for (int b = 0; b < 4; ++b) bf[b] = sk[(wx * 32 + b * 8 + fr) * LDS + kk + fc];
#pragma unroll
      for (int a = 0; a < 4; ++a)
#pragma unroll
        for (int b = 0; b < 4; ++b) dmma_8x8x4(acc[a][b], af[a], bf[b]);
    }
    __syncthreads();
  }
  const double rs = sqrt(static_cast<double>(D));
#pragma unroll
  for (int a = 0; a < 4; ++a) {
    const int i = i0 + wy * 32 + a * 8 + fr;
    if (i >= Nq) continue;
#pragma unroll
    for (int b = 0; b < 4; ++b)
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const int j = j0 + wx * 32 + b * 8 + 2 * fc + h;
        if (j < Nk) S[(static_cast<size_t>(bh) * Nq + i) * Nk + j] = acc[a][b][h] / rs;
      }
  }
}

// fp32 scores for the router's filter: S32_ij = fp32(qbar_i) . fp32(kbar_j) * fp32(1/sqrt(D)),
// accumulated in fp32 (even and odd d separately, then added), plus the norms
// |fp32(qbar_i)| and |fp32(kbar_j)| from which the selection bounds |S32 - S|
// (see select_cert_kernel).
// grid: (ceil(Nk/64), ceil(Nq/64), BH); block 256. The 64 x 64 tile's pooled rows are
// staged whole in shared memory as fp32 [row][d] (pitch D + 4: conflict-free float4
// reads across rows); thread (ty, tx) computes rows ty + 16 a and columns tx + 16 b.
// acc += a * b on two fp32 lanes packed in 64 bits (low word = first lane), each lane
// rounded to nearest as a scalar fmaf would be.
__device__ __forceinline__ void fma_f32x2(uint64_t& acc, uint64_t a, uint64_t b) {
  asm("fma.rn.f32x2 %0, %1, %2, %0;" : "+l"(acc) : "l"(a), "l"(b));
}

template <int D>
struct Score32Smem {
  static constexpr int kPitch = D + 4;
  static constexpr int kBytes = 2 * 64 * kPitch * 4;
};

template <int D>
__global__ void __launch_bounds__(256) score32_kernel(const double* __restrict__ qbar, const double* __restrict__ kbar,
                                                      float* __restrict__ S32, float* __restrict__ nq,
                                                      float* __restrict__ nk, int Nq, int Nk) {
  constexpr int T = 64, P = Score32Smem<D>::kPitch;
  extern __shared__ __align__(16) float smem_f[];
  float* sq = smem_f;           // [64][P]
  float* sk = smem_f + T * P;   // [64][P]
  grid_dep_launch();
  grid_dep_wait();  // pooled means come from the previous kernel
  const int bh = blockIdx.z, i0 = blockIdx.y * T, j0 = blockIdx.x * T;
  const int tid = threadIdx.x;
  const double* qb = qbar + (static_cast<size_t>(bh) * Nq + i0) * D;
  const double* kb = kbar + (static_cast<size_t>(bh) * Nk + j0) * D;
  const int nqr = Nq - i0 < T ? Nq - i0 : T, nkr = Nk - j0 < T ? Nk - j0 : T;
  // coalesced fp64 -> fp32 staging, two values per thread and step; rows past the end are zero
#pragma unroll 8
  for (int e = tid; e < T * D / 2; e += 256) {
    const int r = e / (D / 2), c = 2 * (e % (D / 2));
    double2 q2 = make_double2(0.0, 0.0), k2 = make_double2(0.0, 0.0);
    if (r < nqr) q2 = *reinterpret_cast<const double2*>(qb + static_cast<size_t>(r) * D + c);
    if (r < nkr) k2 = *reinterpret_cast<const double2*>(kb + static_cast<size_t>(r) * D + c);
    *reinterpret_cast<float2*>(sq + r * P + c) = make_float2(static_cast<float>(q2.x), static_cast<float>(q2.y));
    *reinterpret_cast<float2*>(sk + r * P + c) = make_float2(static_cast<float>(k2.x), static_cast<float>(k2.y));
  }
  __syncthreads();
  // norms, once per row: query rows by the first column of tiles, key rows by the first row
  if (tid < T ? (blockIdx.x == 0 && tid < nqr) : (tid < 2 * T && blockIdx.y == 0 && tid - T < nkr)) {
    const float* row = tid < T ? sq + tid * P : sk + (tid - T) * P;
    float acc = 0.f;
#pragma unroll 8
    for (int d = 0; d < D; ++d) acc = fmaf(row[d], row[d], acc);
    if (tid < T)
      nq[static_cast<size_t>(bh) * Nq + i0 + tid] = sqrtf(acc);
    else
      nk[static_cast<size_t>(bh) * Nk + j0 + tid - T] = sqrtf(acc);
  }
  // Each output keeps two fp32 partial sums (even and odd d) in one 64-bit register pair,
  // updated with the paired fp32 FMA; they are added at the end. A warp covers 4 values of
  // ty and 8 of tx, so each of its float4 reads touches 4 or 8 rows in distinct banks.
  const int wid = tid >> 5, ln = tid & 31;
  const int ty = 4 * (wid >> 1) + (ln >> 3), tx = 8 * (wid & 1) + (ln & 7);
  uint64_t acc2[4][4];
#pragma unroll
  for (int x = 0; x < 4; ++x)
#pragma unroll
    for (int y = 0; y < 4; ++y) acc2[x][y] = 0ull;
#pragma unroll 2
  for (int d = 0; d < D; d += 4) {
    ulonglong2 qa[4], ka[4];
#pragma unroll
    for (int x = 0; x < 4; ++x) qa[x] = *reinterpret_cast<const ulonglong2*>(sq + (ty + 16 * x) * P + d);
#pragma unroll
    for (int y = 0; y < 4; ++y) ka[y] = *reinterpret_cast<const ulonglong2*>(sk + (tx + 16 * y) * P + d);
#pragma unroll
    for (int x = 0; x < 4; ++x)
#pragma unroll
      for (int y = 0; y < 4; ++y) {
        fma_f32x2(acc2[x][y], qa[x].x, ka[y].x);
        fma_f32x2(acc2[x][y], qa[x].y, ka[y].y);
      }
  }
  float acc[4][4];
#pragma unroll
  for (int x = 0; x < 4; ++x)
#pragma unroll
    for (int y = 0; y < 4; ++y)
      acc[x][y] = __uint_as_float(static_cast<uint32_t>(acc2[x][y])) +
                  __uint_as_float(static_cast<uint32_t>(acc2[x][y] >> 32));
  const float rs = static_cast<float>(1.0 / sqrt(static_cast<double>(D)));
#pragma unroll
  for (int x = 0; x < 4; ++x) {
    const int i = ty + 16 * x;
    if (i >= nqr) continue;
    float* dst = S32 + (static_cast<size_t>(bh) * Nq + i0 + i) * Nk + j0;
#pragma unroll
    for (int y = 0; y < 4; ++y)
      if (tx + 16 * y < nkr) dst[tx + 16 * y] = acc[x][y] * rs;
  }
}

// ---------------------------------------------------------------- selection

// Order-preserving map from a double to an unsigned key (larger key = larger value).
// -0.0 is folded onto +0.0 so that the two compare equal, as they do as numbers.
__device__ __forceinline__ uint64_t order_key(double s) {
  s = s + 0.0;
  const uint64_t u = static_cast<uint64_t>(__double_as_longlong(s));
  return (u >> 63) ? ~u : (u | (1ull << 63));
}

__device__ __forceinline__ int warp_sum(int v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// Largest t with #{keys >= t} >= k (the k-th largest key), k >= 1, by bisection on the bits.
// If flip, keys are complemented first (gives the complement of the k-th smallest key).
__device__ __forceinline__ uint64_t kth_largest(const uint64_t* keys, int n, int k, bool flip) {
  const int lane = threadIdx.x & 31;
  uint64_t T = 0;
  for (int bit = 63; bit >= 0; --bit) {
    const uint64_t cand = T | (1ull << bit);
    int c = 0;
    for (int j = lane; j < n; j += 32) {
      const uint64_t key = flip ? ~keys[j] : keys[j];
      c += key >= cand;
    }
    if (warp_sum(c) >= k) T = cand;
  }
  return T;
}

struct SelectArgs {
  const double* S;      // [rows, Nk]
  int rows, Nk, kc, kn;
  int8_t* mask;         // [rows, Nk] labels (nullable)
  int32_t* crit;        // [rows, crit_ld] critical block indices, ascending (nullable)
  int crit_ld;
  int32_t* crit_cnt;    // [rows] (nullable)
  __nv_bfloat16* W;     // [rows, w_ld] marginal indicator (1 marginal, else 0), zero padded (nullable)
  int w_ld;
};

// One warp per row; dynamic smem = warps_per_cta * Nk * 8 bytes of keys.
__global__ void __launch_bounds__(256) select_kernel(SelectArgs a) {
  grid_dep_launch();
  grid_dep_wait();  // scores come from the previous kernel
  extern __shared__ uint64_t keys_all[];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int wpc = blockDim.x >> 5;
  const int row = blockIdx.x * wpc + warp;
  if (row >= a.rows) return;  // whole warp leaves; nothing below synchronises the CTA
  uint64_t* keys = keys_all + static_cast<size_t>(warp) * a.Nk;
  const double* srow = a.S + static_cast<size_t>(row) * a.Nk;
  for (int j = lane; j < a.Nk; j += 32) keys[j] = order_key(srow[j]);
  __syncwarp();

  // Critical: the kc largest in (key desc, index asc). Tc = kc-th largest key;
  // every key > Tc is critical and the first (kc - #{> Tc}) keys == Tc by index.
  uint64_t Tc = 0, Tn = 0;
  int need_c = 0, need_n = 0, tot_eq_n = 0;
  if (a.kc > 0) {
    Tc = kth_largest(keys, a.Nk, a.kc, false);
    int gt = 0;
    for (int j = lane; j < a.Nk; j += 32) gt += keys[j] > Tc;
    need_c = a.kc - warp_sum(gt);
  }
  // Negligible: the kn last in the same order = the kn smallest keys, ties
  // resolved towards the higher index. Tn = kn-th smallest key.
  if (a.kn > 0) {
    Tn = ~kth_largest(keys, a.Nk, a.kn, true);
    int lt = 0, eq = 0;
    for (int j = lane; j < a.Nk; j += 32) {
      lt += keys[j] < Tn;
      eq += keys[j] == Tn;
    }
    need_n = a.kn - warp_sum(lt);
    tot_eq_n = warp_sum(eq);
  }

  int eqc_before = 0, eqn_before = 0, crit_before = 0;
  const uint32_t lt_mask = (1u << lane) - 1u;
  for (int j0 = 0; j0 < a.Nk; j0 += 32) {
    const int j = j0 + lane;
    const bool in = j < a.Nk;
    const uint64_t key = in ? keys[j] : 0;
    const bool eqc = in && a.kc > 0 && key == Tc;
    const bool eqn = in && a.kn > 0 && key == Tn;
    const uint32_t bc = __ballot_sync(0xffffffffu, eqc);
    const uint32_t bn = __ballot_sync(0xffffffffu, eqn);
    const int rank_c = eqc_before + __popc(bc & lt_mask);
    const int rank_n = eqn_before + __popc(bn & lt_mask);
    const bool is_c = in && a.kc > 0 && (key > Tc || (eqc && rank_c < need_c));
    // ties at Tn with the highest indices are the negligible ones
    const bool is_n = in && a.kn > 0 && (key < Tn || (eqn && (tot_eq_n - rank_n - 1) < need_n));
    const uint32_t bcrit = __ballot_sync(0xffffffffu, is_c);
    if (in) {
      const int8_t lab = is_c ? 2 : (is_n ? 0 : 1);
      if (a.mask) a.mask[static_cast<size_t>(row) * a.Nk + j] = lab;
      if (a.W) a.W[static_cast<size_t>(row) * a.w_ld + j] = __float2bfloat16_rn(lab == 1 ? 1.f : 0.f);
      if (is_c && a.crit) a.crit[static_cast<size_t>(row) * a.crit_ld + crit_before + __popc(bcrit & lt_mask)] = j;
    }
    eqc_before += __popc(bc);
    eqn_before += __popc(bn);
    crit_before += __popc(bcrit);
  }
  if (a.W)
    for (int j = a.Nk + lane; j < a.w_ld; j += 32) a.W[static_cast<size_t>(row) * a.w_ld + j] = __float2bfloat16_rn(0.f);
  if (lane == 0 && a.crit_cnt) a.crit_cnt[row] = crit_before;
}

// Certified selection from fp32 scores, for rows of up to 32 * KPL blocks.
//
// Bound. With u = 2^-24, rounding qbar and kbar to fp32, the fp32 products and their
// fp32 accumulation (two chains of D/2 terms, then one addition), and the scaling by
// fp32(1/sqrt(D)) give
//   |S32_ij - S_ij| <= (D + 4) u (1 + O(D u)) sum_d |qbar_id kbar_jd| / sqrt(D)
//                   <= (D + 4) u (1 + O(D u)) |qbar_i| |kbar_j| / sqrt(D)   (Cauchy-Schwarz),
// S being the exact score. beta_i = 2 (D + 8) u |qbar_i| max_j |kbar_j| / sqrt(D), from
// the fp32 norms, is above that with a factor near 2 to spare, which covers the
// rounding of the norms and of beta itself.
//
// Decision. With T a threshold on the fp32 scores of the row such that the k-th largest
// is >= T and either fewer than k scores exceed T or exactly k reach it (kth_largest32):
//   S32_j > T + 2 beta  ->  S_j > T + beta, and every block ranked above j has S32 > T,
//                           so fewer than kc blocks precede j: critical for certain;
//   S32_j < T - 2 beta  ->  S_j < T - beta, below every block with S32 >= T, of which
//                           there are at least kc: not critical for certain.
// The blocks in between (the band) are ranked by their fp64 score, recomputed here,
// and then by index; the negligible side is the mirror image. The labels are those of
// the total order (S descending, j ascending) on the fp64 scores.
__device__ __forceinline__ uint32_t order_key32f(float f) {
  f = f + 0.0f;  // -0.0 folds onto +0.0
  const uint32_t u = __float_as_uint(f);
  return (u >> 31) ? ~u : (u | 0x80000000u);
}

// A threshold T on the (optionally complemented) 32-bit keys of the valid slots with
// #{key >= T} >= k whose top-k set is fixed: either T is the k-th largest key, or
// exactly k keys are >= T (T then lies above every other key). k >= 1. Bisection on
// the bits, stopping as soon as the count is exactly k. For finite inputs T is the key
// of a finite float: it is a prefix of the k-th largest key, whose top bit is >= 2^23.
template <int KPL>
__device__ __forceinline__ uint32_t kth_largest32(const uint32_t (&key)[KPL], int nvalid_lane, int k, bool flip) {
  uint32_t T = 0;
#pragma unroll 1
  for (int bit = 31; bit >= 0; --bit) {
    const uint32_t cand = T | (1u << bit);
    uint32_t c = 0;
#pragma unroll
    for (int t = 0; t < KPL; ++t) {
      const uint32_t kk = flip ? ~key[t] : key[t];
      c += (t < nvalid_lane && kk >= cand) ? 1u : 0u;
    }
    const int cnt = static_cast<int>(__reduce_add_sync(0xffffffffu, c));
    if (cnt >= k) T = cand;
    if (cnt == k) break;  // the k keys >= cand are exactly the top k
  }
  return T;
}

// fp64 score of block j for the row whose pooled query (fp64, D values) is spread over
// the lanes as qv[d / 32] for d = lane + 32 m; a fixed reduction order.
template <int D>
__device__ __forceinline__ double exact_score(const double (&qv)[D / 32], const double* kbar_j) {
  const int lane = threadIdx.x & 31;
  double acc = 0.0;
#pragma unroll
  for (int m = 0; m < D / 32; ++m) acc = fma(qv[m], kbar_j[lane + 32 * m], acc);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
  return acc / sqrt(static_cast<double>(D));
}

// Among the slots flagged in `band` (bit t of each lane = block lane + 32 t), pick `need`
// in the order (fp64 score descending, index ascending) when best_high, or (fp64 score
// ascending, index descending) otherwise; returns this lane's picks as a bit mask. Each
// pick walks the remaining band and recomputes its fp64 scores with the whole warp, so no
// per-slot score array is held (the band is a handful of blocks except on degenerate rows).
template <int KPL, int D>
__device__ __forceinline__ uint64_t pick_band(uint64_t band, int need, bool best_high, const double (&qv)[D / 32],
                                              const double* kbar_row0) {
  const int lane = threadIdx.x & 31;
  uint64_t picked = 0;
#pragma unroll 1
  for (int it = 0; it < need; ++it) {
    double best = 0.0;  // warp-uniform: every lane sees the same reduced scores
    int bj = -1;
#pragma unroll 1
    for (int t = 0; t < KPL; ++t) {
      uint32_t who = __ballot_sync(0xffffffffu, ((band & ~picked) >> t) & 1ull);
      while (who) {
        const int l = __ffs(who) - 1;
        who &= who - 1;
        const int j = l + 32 * t;
        const double v = exact_score<D>(qv, kbar_row0 + static_cast<size_t>(j) * D);
        const double w = best_high ? v : -v;
        if (bj < 0 || w > best || (w == best && (best_high ? j < bj : j > bj))) {
          best = w;
          bj = j;
        }
      }
    }
    if (bj < 0) break;
    if ((bj & 31) == lane) picked |= 1ull << (bj >> 5);
  }
  return picked;
}

struct CertArgs {
  const float* S32;     // [rows, Nk]
  const float* nq;      // [rows] |fp32(qbar_i)|
  const float* nk;      // [BH, Nk] |fp32(kbar_j)|
  const double* qbar;   // [rows, D]
  const double* kbar;   // [BH, Nk, D]
  int rows, Nq, Nk, kc, kn;
  int8_t* mask;         // [rows, Nk] labels (nullable)
  int32_t* crit;        // [rows, crit_ld] critical block indices, ascending (nullable)
  int crit_ld;
  int32_t* crit_cnt;    // [rows] (nullable)
  __nv_bfloat16* W;     // [rows, w_ld] marginal indicator (1 marginal, else 0), zero padded (nullable)
  int w_ld;
};

// Per side s of a warp's row, the k_s-th largest of the valid values y_s (side 0: y = x,
// k_0 = kc; side 1: y = -x, k_1 = kn), as a float T_s with #{y_s > T_s} < k_s <= #{y_s >= T_s}.
// Both sides bisect their value interval [L, H] (which holds T) together, keeping #{y >= L}
// and #{y > H}, until at most 32 values lie in it; those are gathered in `cand` (64 floats
// of shared memory per warp) and ranked. ok_s is false for a side whose interval could not
// be narrowed to 32 values (many equal or adjacent values): the caller then bisects on
// the 32-bit keys. A side with k_s = 0 is skipped.
template <int KPL>
__device__ __forceinline__ void kth_values(const float (&x)[KPL], int nvalid_lane, const int (&k)[2], float* cand,
                                           float (&T)[2], bool (&ok)[2]) {
  // Slots past the row end hold NaN: every comparison below is false for them and
  // fminf/fmaxf ignore them, so no per-slot validity test is needed.
  const int lane = threadIdx.x & 31;
  float mn = INFINITY, mx = -INFINITY;
  const int nv = nvalid_lane < 0 ? 0 : (nvalid_lane > KPL ? KPL : nvalid_lane);
#pragma unroll
  for (int t = 0; t < KPL; ++t) {
    mn = fminf(mn, x[t]);
    mx = fmaxf(mx, x[t]);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    mn = fminf(mn, __shfl_xor_sync(0xffffffffu, mn, o));
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
  }
  const int n = static_cast<int>(__reduce_add_sync(0xffffffffu, static_cast<uint32_t>(nv)));
  float L[2] = {mn, -mx}, H[2] = {mx, -mn};
  int ge_L[2] = {n, n}, gt_H[2] = {0, 0};
#pragma unroll 1
  for (int it = 0; it < 48; ++it) {
    float mid[2];
    bool run[2];
#pragma unroll
    for (int s = 0; s < 2; ++s) {
      mid[s] = 0.5f * L[s] + 0.5f * H[s];
      run[s] = k[s] > 0 && ge_L[s] - gt_H[s] > 32 && mid[s] >= L[s] && mid[s] < H[s];
    }
    if (!run[0] && !run[1]) break;
    uint32_t c0 = 0, c1 = 0;
#pragma unroll
    for (int t = 0; t < KPL; ++t) {
      c0 += x[t] > mid[0] ? 1u : 0u;
      c1 += -x[t] > mid[1] ? 1u : 0u;
    }
    const int cnt[2] = {static_cast<int>(__reduce_add_sync(0xffffffffu, c0)),
                        static_cast<int>(__reduce_add_sync(0xffffffffu, c1))};
#pragma unroll
    for (int s = 0; s < 2; ++s) {
      if (!run[s]) continue;
      if (cnt[s] >= k[s]) {  // T > mid
        L[s] = nextafterf(mid[s], INFINITY);
        ge_L[s] = cnt[s];
      } else {  // T <= mid
        H[s] = mid[s];
        gt_H[s] = cnt[s];
      }
    }
  }
  const int m[2] = {ge_L[0] - gt_H[0], ge_L[1] - gt_H[1]};
  const uint32_t lt_mask = (1u << lane) - 1u;
  int base[2] = {0, 0};
#pragma unroll
  for (int t = 0; t < KPL; ++t) {
#pragma unroll
    for (int s = 0; s < 2; ++s) {
      const float y = s ? -x[t] : x[t];
      const bool in = m[s] <= 32 && y >= L[s] && y <= H[s];
      const uint32_t b = __ballot_sync(0xffffffffu, in);
      if (in) cand[32 * s + base[s] + __popc(b & lt_mask)] = y;
      base[s] += __popc(b);
    }
  }
  __syncwarp();
#pragma unroll
  for (int s = 0; s < 2; ++s) {
    ok[s] = false;
    T[s] = 0.f;
    if (k[s] <= 0 || m[s] > 32) continue;
    const float mine = lane < m[s] ? cand[32 * s + lane] : 0.f;
    int g = 0, e = 0;
#pragma unroll
    for (int f = 0; f < 32; ++f) {
      const float o = cand[32 * s + f];
      g += (f < m[s] && o > mine) ? 1 : 0;
      e += (f < m[s] && o >= mine) ? 1 : 0;
    }
    const int kk = k[s] - gt_H[s];  // T is the kk-th largest value in [L, H]
    const uint32_t hit = __ballot_sync(0xffffffffu, lane < m[s] && g < kk && kk <= e);
    T[s] = __shfl_sync(0xffffffffu, mine, hit ? __ffs(hit) - 1 : 0);
    ok[s] = hit != 0u;
  }
  __syncwarp();  // cand may be reused
}

// One side of the certified selection from its threshold T: the first k blocks in the order
// (S descending, j ascending) when !NEG (critical), or (S ascending, j descending) when NEG
// (negligible). Sets this lane's certain members in `sure` and the band members picked by
// their fp64 scores in `pick`; when the band is taken whole or not at all, no fp64 score is
// needed.
template <int KPL, int D, bool NEG>
__device__ __forceinline__ void certify_side(const float (&x)[KPL], int nvalid_lane, int k, float T, float two_beta,
                                             const double (&qv)[D / 32], const double* kbar_row0, uint64_t& sure,
                                             uint64_t& pick) {
  const float hi = __fadd_ru(T, two_beta), lo = __fsub_rd(T, two_beta);  // rounded outwards
  uint64_t band = 0;
  uint32_t nsure = 0, nband = 0;
  sure = 0;
#pragma unroll
  for (int t = 0; t < KPL; ++t) {
    const float y = NEG ? -x[t] : x[t];  // NaN past the row end: neither certain nor in the band
    if (y > hi) {
      sure |= 1ull << t;
      ++nsure;
    } else if (y >= lo) {
      band |= 1ull << t;
      ++nband;
    }
  }
  const int need = k - static_cast<int>(__reduce_add_sync(0xffffffffu, nsure));
  const int nb = static_cast<int>(__reduce_add_sync(0xffffffffu, nband));
  if (need <= 0)
    pick = 0;
  else if (need >= nb)
    pick = band;
  else
    pick = pick_band<KPL, D>(band, need, !NEG, qv, kbar_row0);
}

template <int KPL>
__device__ __forceinline__ float threshold_from_keys(const float (&x)[KPL], int nvalid_lane, int k, bool neg) {
  uint32_t key[KPL];
#pragma unroll
  for (int t = 0; t < KPL; ++t) key[t] = t < nvalid_lane ? order_key32f(x[t]) : 0u;
  uint32_t Tk = kth_largest32<KPL>(key, nvalid_lane, k, neg);
  if (neg) Tk = ~Tk;
  const float Tx = __uint_as_float((Tk >> 31) ? (Tk & 0x7FFFFFFFu) : ~Tk);
  return neg ? -Tx : Tx;
}

template <int KPL, int D>
__global__ void __launch_bounds__(256, KPL <= 16 ? 3 : (KPL <= 40 ? 2 : 1)) select_cert_kernel(CertArgs a) {
  __shared__ float cand_all[8][64];
  grid_dep_launch();
  grid_dep_wait();  // scores come from the previous kernel
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int row = blockIdx.x * (blockDim.x >> 5) + warp;
  if (row >= a.rows) return;  // whole warp leaves; nothing below synchronises the CTA
  const int bh = row / a.Nq;
  const float* srow = a.S32 + static_cast<size_t>(row) * a.Nk;
  const float* nkrow = a.nk + static_cast<size_t>(bh) * a.Nk;
  const int nvalid_lane = (a.Nk - lane + 31) / 32;  // slots t < nvalid_lane hold j = lane + 32 t < Nk
  float x[KPL];
  float nkmax = 0.f;
#pragma unroll
  for (int t = 0; t < KPL; ++t) {
    const bool v = t < nvalid_lane;
    x[t] = v ? srow[lane + 32 * t] : __uint_as_float(0x7FC00000u);  // NaN marks a slot past the row end
    if (v) nkmax = fmaxf(nkmax, nkrow[lane + 32 * t]);
  }
  double qv[D / 32];
  const double* qrow = a.qbar + static_cast<size_t>(row) * D;
#pragma unroll
  for (int m = 0; m < D / 32; ++m) qv[m] = qrow[lane + 32 * m];
  const float nq = a.nq[row];
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) nkmax = fmaxf(nkmax, __shfl_xor_sync(0xffffffffu, nkmax, o));
  const float two_beta = 4.f * static_cast<float>(D + 8) * 0x1p-24f / sqrtf(static_cast<float>(D)) * nq * nkmax;
  const double* kbar_row0 = a.kbar + static_cast<size_t>(bh) * a.Nk * D;

  const int k[2] = {a.kc, a.kn};
  float T[2];
  bool ok[2];
  kth_values<KPL>(x, nvalid_lane, k, cand_all[warp], T, ok);
  uint64_t sure_c = 0, pick_c = 0, sure_n = 0, pick_n = 0;
  if (a.kc > 0) {
    if (!ok[0]) T[0] = threshold_from_keys<KPL>(x, nvalid_lane, a.kc, false);
    certify_side<KPL, D, false>(x, nvalid_lane, a.kc, T[0], two_beta, qv, kbar_row0, sure_c, pick_c);
  }
  if (a.kn > 0) {
    if (!ok[1]) T[1] = threshold_from_keys<KPL>(x, nvalid_lane, a.kn, true);
    certify_side<KPL, D, true>(x, nvalid_lane, a.kn, T[1], two_beta, qv, kbar_row0, sure_n, pick_n);
  }

  const uint32_t lt_mask = (1u << lane) - 1u;
  int crit_before = 0;
#pragma unroll
  for (int t = 0; t < KPL; ++t) {
    if (32 * t >= a.Nk) break;
    const int j = lane + 32 * t;
    const bool in = t < nvalid_lane;
    const bool is_c = in && (((sure_c | pick_c) >> t) & 1ull);
    const bool is_n = in && !is_c && (((sure_n | pick_n) >> t) & 1ull);
    const uint32_t bcrit = __ballot_sync(0xffffffffu, is_c);
    if (in) {
      const int8_t lab = is_c ? 2 : (is_n ? 0 : 1);
      if (a.mask) a.mask[static_cast<size_t>(row) * a.Nk + j] = lab;
      if (a.W) a.W[static_cast<size_t>(row) * a.w_ld + j] = __float2bfloat16_rn(lab == 1 ? 1.f : 0.f);
      const int slot = crit_before + __popc(bcrit & lt_mask);  // < kc whenever the bound holds
      if (is_c && a.crit && slot < a.crit_ld) a.crit[static_cast<size_t>(row) * a.crit_ld + slot] = j;
    }
    crit_before += __popc(bcrit);
  }
  if (a.W)
    for (int j = a.Nk + lane; j < a.w_ld; j += 32) a.W[static_cast<size_t>(row) * a.w_ld + j] = __float2bfloat16_rn(0.f);
  if (lane == 0 && a.crit_cnt) a.crit_cnt[row] = crit_before;
}

// ---------------------------------------------------------------- caller mask
struct MaskListArgs {
  const int8_t* mask;   // [rows, Nk]
  int rows, Nk;
  int32_t* crit;
  int crit_ld;
  int32_t* crit_cnt;
  __nv_bfloat16* W;     // marginal indicator [rows, w_ld] (nullable)
  int w_ld;
  uint32_t* err;
};

// One warp per row: critical list (ascending), counts and marginal indicator
// from the caller's labels. A label outside {0, 1, 2} is reported through the
// device error word and that block is treated as negligible.
__global__ void __launch_bounds__(256) mask_lists_kernel(MaskListArgs a) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int row = blockIdx.x * (blockDim.x >> 5) + warp;
  if (row >= a.rows) return;
  const uint32_t lt_mask = (1u << lane) - 1u;
  int crit_before = 0;
  bool bad = false;
  for (int j0 = 0; j0 < a.Nk; j0 += 32) {
    const int j = j0 + lane;
    const bool in = j < a.Nk;
    int lab = in ? a.mask[static_cast<size_t>(row) * a.Nk + j] : 0;
    if (lab < 0 || lab > 2) {
      bad = true;
      lab = 0;
    }
    const bool is_c = in && lab == 2;
    const uint32_t bcrit = __ballot_sync(0xffffffffu, is_c);
    if (in) {
      if (a.W) a.W[static_cast<size_t>(row) * a.w_ld + j] = __float2bfloat16_rn(lab == 1 ? 1.f : 0.f);
      if (is_c) a.crit[static_cast<size_t>(row) * a.crit_ld + crit_before + __popc(bcrit & lt_mask)] = j;
    }
    crit_before += __popc(bcrit);
  }
  if (a.W)
    for (int j = a.Nk + lane; j < a.w_ld; j += 32) a.W[static_cast<size_t>(row) * a.w_ld + j] = __float2bfloat16_rn(0.f);
  if (lane == 0) a.crit_cnt[row] = crit_before;
  if (__any_sync(0xffffffffu, bad) && lane == 0) record_error(a.err, SLA_DEVERR_BAD_MASK);
}

}  // namespace sla
