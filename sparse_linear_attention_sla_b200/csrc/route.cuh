// Block router for the SLA forward.
//
//   score_kernel : S_ij = qbar_i . kbar_j / sqrt(D) in fp64 (compressed scores)
//   select_kernel: per query-block row, label every KV block critical (2),
//                  marginal (1) or negligible (0): the first kc blocks in the
//                  total order (S descending, j ascending) are critical, the
//                  last kn are negligible.
//   mask_lists_kernel: the same outputs from a caller-supplied label mask.
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

// Register-resident selection for rows of up to 32 * KPL blocks.
//
// Exactness argument: rounding a double to float is monotone, so with
// key32 = order key of (float)S, every block whose key32 is above the
// kc-th largest key32 (T) is above every block whose key32 is <= T in the
// fp64 order too. The blocks with key32 == T are the only ones whose fp64
// order matters; they are resolved by their fp64 key and then their index.
// The result is the same set as the fp64 total order (S desc, j asc).
__device__ __forceinline__ uint32_t order_key32(double s) {
  const float f = static_cast<float>(s) + 0.0f;  // -0.0 folds onto +0.0
  const uint32_t u = __float_as_uint(f);
  return (u >> 31) ? ~u : (u | 0x80000000u);
}

// A threshold T on the (optionally complemented) 32-bit keys of the valid slots with
// #{key >= T} >= k whose top-k set is fixed: either T is the k-th largest key, or
// exactly k keys are >= T (then they are the top k and no key equals a smaller
// candidate). k >= 1. Bisection on the bits, stopping as soon as the count is exactly k.
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

// Among the slots flagged in `group` (bit t of each lane), pick `need` of them in the
// order (fp64 key descending, index ascending) when best_high, or (fp64 key ascending,
// index descending) otherwise; returns this lane's picks as a bit mask.
template <int KPL>
__device__ __forceinline__ uint64_t pick_from_group(const double* srow, uint64_t group, int need, bool best_high) {
  const int lane = threadIdx.x & 31;
  uint64_t picked = 0;
  for (int it = 0; it < need; ++it) {
    // this lane's best candidate
    uint64_t bk = 0;
    int bj = -1;
#pragma unroll
    for (int t = 0; t < KPL; ++t) {
      if (!((group & ~picked) >> t & 1ull)) continue;
      const int j = lane + 32 * t;
      const uint64_t k64 = best_high ? order_key(srow[j]) : ~order_key(srow[j]);
      // higher k64 wins; on equal keys the lower index wins (best_high) or the higher one (otherwise)
      if (bj < 0 || k64 > bk || (k64 == bk && (best_high ? j < bj : j > bj))) {
        bk = k64;
        bj = j;
      }
    }
    // warp arg-best
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      const uint64_t ok = __shfl_xor_sync(0xffffffffu, bk, o);
      const int oj = __shfl_xor_sync(0xffffffffu, bj, o);
      const bool take = oj >= 0 && (bj < 0 || ok > bk || (ok == bk && (best_high ? oj < bj : oj > bj)));
      if (take) {
        bk = ok;
        bj = oj;
      }
    }
    if (bj >= 0 && (bj & 31) == lane) picked |= 1ull << (bj >> 5);
  }
  return picked;
}

template <int KPL>
__global__ void __launch_bounds__(256) select_reg_kernel(SelectArgs a) {
  grid_dep_launch();
  grid_dep_wait();  // scores come from the previous kernel
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int row = blockIdx.x * (blockDim.x >> 5) + warp;
  if (row >= a.rows) return;  // whole warp leaves; nothing below synchronises the CTA
  const double* srow = a.S + static_cast<size_t>(row) * a.Nk;
  const int nvalid_lane = (a.Nk - lane + 31) / 32;  // slots t < nvalid_lane hold j = lane + 32 t < Nk
  uint32_t key[KPL];
#pragma unroll
  for (int t = 0; t < KPL; ++t) key[t] = t < nvalid_lane ? order_key32(srow[lane + 32 * t]) : 0u;

  uint32_t Tc = 0, Tn = 0;
  uint64_t eqc = 0, eqn = 0, pick_c = 0, pick_n = 0;
  if (a.kc > 0) {
    Tc = kth_largest32<KPL>(key, nvalid_lane, a.kc, false);
    uint32_t gt = 0;
#pragma unroll
    for (int t = 0; t < KPL; ++t) {
      const bool v = t < nvalid_lane;
      gt += (v && key[t] > Tc) ? 1u : 0u;
      if (v && key[t] == Tc) eqc |= 1ull << t;
    }
    const int need = a.kc - static_cast<int>(__reduce_add_sync(0xffffffffu, gt));
    const int neq = static_cast<int>(__reduce_add_sync(0xffffffffu, static_cast<uint32_t>(__popcll(eqc))));
    pick_c = need >= neq ? eqc : pick_from_group<KPL>(srow, eqc, need, true);
  }
  if (a.kn > 0) {
    Tn = ~kth_largest32<KPL>(key, nvalid_lane, a.kn, true);
    uint32_t lt = 0;
#pragma unroll
    for (int t = 0; t < KPL; ++t) {
      const bool v = t < nvalid_lane;
      lt += (v && key[t] < Tn) ? 1u : 0u;
      if (v && key[t] == Tn) eqn |= 1ull << t;
    }
    const int need = a.kn - static_cast<int>(__reduce_add_sync(0xffffffffu, lt));
    const int neq = static_cast<int>(__reduce_add_sync(0xffffffffu, static_cast<uint32_t>(__popcll(eqn))));
    pick_n = need >= neq ? eqn : pick_from_group<KPL>(srow, eqn, need, false);
  }

  const uint32_t lt_mask = (1u << lane) - 1u;
  int crit_before = 0;
#pragma unroll
  for (int t = 0; t < KPL; ++t) {
    if (32 * t >= a.Nk) break;
    const int j = lane + 32 * t;
    const bool in = t < nvalid_lane;
    const bool is_c = in && a.kc > 0 && (key[t] > Tc || (pick_c >> t & 1ull));
    const bool is_n = in && a.kn > 0 && !is_c && (key[t] < Tn || (pick_n >> t & 1ull));
    const uint32_t bcrit = __ballot_sync(0xffffffffu, is_c);
    if (in) {
      const int8_t lab = is_c ? 2 : (is_n ? 0 : 1);
      if (a.mask) a.mask[static_cast<size_t>(row) * a.Nk + j] = lab;
      if (a.W) a.W[static_cast<size_t>(row) * a.w_ld + j] = __float2bfloat16_rn(lab == 1 ? 1.f : 0.f);
      if (is_c && a.crit) a.crit[static_cast<size_t>(row) * a.crit_ld + crit_before + __popc(bcrit & lt_mask)] = j;
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
  __nv_bfloat16* W;
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
      a.W[static_cast<size_t>(row) * a.w_ld + j] = __float2bfloat16_rn(lab == 1 ? 1.f : 0.f);
      if (is_c) a.crit[static_cast<size_t>(row) * a.crit_ld + crit_before + __popc(bcrit & lt_mask)] = j;
    }
    crit_before += __popc(bcrit);
  }
  for (int j = a.Nk + lane; j < a.w_ld; j += 32) a.W[static_cast<size_t>(row) * a.w_ld + j] = __float2bfloat16_rn(0.f);
  if (lane == 0) a.crit_cnt[row] = crit_before;
  if (__any_sync(0xffffffffu, bad) && lane == 0) record_error(a.err, SLA_DEVERR_BAD_MASK);
}

}  // namespace sla
