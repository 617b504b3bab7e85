// Per-block statistics of the PISA variant and the mean first-order matrix of each head.
//
// Source: "PISA - Atención Dispersa por Tramos para Transformers de Difusión Eficientes" §2
// (the N_t equation: a non-critical block enters through its centroid key, its value sum and
// a first-order term built from the mean of the blocks' first-order matrices; the hardware
// pipeline computes these once per KV block ahead of the attention pass).
//
//   pisa_stats_kernel: per KV block j of a head, from K_j and V_j,
//       kbar_j = mean of the valid keys (fp64 for the router; bf16 as the centroid key),
//       Vsum_j = sum of the valid value rows (bf16, the centroid value),
//     and per part of a head (a contiguous run of its KV blocks, taken by one CTA)
//       sum over the part of H_j = (K_j - kbar_j)^T V_j (fp32, tcgen05 MMA accumulating in
//       TMEM across the part's blocks).
//   hbar_kernel: Hbar = (1 / Nk) * (sum of the head's parts, in part order).
//
// Both are deterministic: every sum runs in a fixed order.
#pragma once

#include "sm100.cuh"

namespace sla {

// The parts of all heads together number at most max(BH, kPisaParts); a fixed constant, so
// the workspace size and the summation order do not depend on the device.
constexpr int kPisaParts = 148;

__host__ __device__ inline int pisa_parts(int BH, int Nk) {
  int P = kPisaParts / BH;
  if (P > Nk) P = Nk;
  return P < 1 ? 1 : P;
}

struct PisaStatsArgs {
  int BH, N, Nk, P;
  double* kbar;         // [BH, Nk, D] fp64 block means (nullable: no router input)
  __nv_bfloat16* kcen;  // [BH, Nk, D] bf16 block means
  __nv_bfloat16* vsum;  // [BH, Nk, D] bf16 block sums of V
  float* hpart;         // [BH * P, D, D] fp32: per part, the sum of its blocks' H_j
  uint32_t* err;
};

template <int D>
struct PisaSmem {
  static constexpr int NSLOT = 4;
  static constexpr uint32_t SLOT = 32768;               // K (16 KB) then V (16 KB)
  static constexpr uint32_t ZERO = D == 64 ? 8192 : 0;  // rows 64..127 of (K - kbar)^T when D = 64
  static constexpr uint32_t total() { return NSLOT * SLOT + ZERO + 1024; }
};

// Persistent, warp-specialised; one CTA per SM, 576 threads. A CTA takes the parts
// c = blockIdx.x, blockIdx.x + gridDim.x, ... (part c: head c / P, blocks
// [(c % P) Nk / P, (c % P + 1) Nk / P)); its blocks are numbered k = 0, 1, ... in that order.
//   warp 0        TMA producer: K_j and V_j into a 4-slot ring
//   warps 2..13   three column warpgroups taking the blocks in turn (k % 3): per 16-byte
//                 chunk of the K and V tiles, the fp64 sum of the valid keys and the fp32
//                 sum of the value rows (rows past N arrive as zeros); after the reduction
//                 over the warpgroup, kbar_j, Vsum_j out, and the K tile rewritten in place
//                 as bf16(k - kbar_j) (zero past the sequence end)
//   warp 1        tcgen05 issuer: acc += (K_j - kbar_j)^T V_j (M=128, N=D, K=64 tokens, both
//                 operands MN-major), the accumulator cleared at each part's first block;
//                 two TMEM accumulators alternate between parts
//   warps 14..17  epilogue: the part's accumulator, TMEM -> fp32 -> hpart
template <int D>
__global__ void __launch_bounds__(576, 1)
    pisa_stats_kernel(const __grid_constant__ CUtensorMap map_k, const __grid_constant__ CUtensorMap map_v,
                      PisaStatsArgs a) {
  using L = PisaSmem<D>;
  constexpr int NS = L::NSLOT;
  constexpr int KBOX = D / 64;       // 64-column boxes per row
  constexpr int CPR = D / 8;         // 16-byte chunks per row
  constexpr int RG = 128 / CPR;      // row groups of a column warpgroup
  constexpr int RPT = 64 / RG;       // rows per thread
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* zero = smem + NS * L::SLOT;
  __shared__ uint64_t full[NS], col_done[NS], empty[NS], acc_full[2], acc_empty[2], drain;
  __shared__ uint32_t tmem_base_sh;
  __shared__ int abort_flag;
  __shared__ double part_d[3][4][D];  // [column warpgroup][warp][column]
  __shared__ float part_f[3][4][D];
  __shared__ __align__(16) float mean_f[3][D];  // [column warpgroup][column]: fp32(kbar_j)

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int n_parts = a.BH * a.P;
  if (tid == 0) {
    for (int s = 0; s < NS; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&col_done[s], 128);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&acc_full[b], 1);
      mbar_init(&acc_empty[b], 128);
    }
    mbar_init(&drain, 1);
    abort_flag = 0;
    fence_mbar_init();
  }
  if constexpr (D == 64) {
    for (uint32_t o = tid * 16; o < L::ZERO; o += 576 * 16) *reinterpret_cast<uint4*>(zero + o) = make_uint4(0, 0, 0, 0);
    fence_proxy_async_smem();
  }
  if (warp == 1) {
    tmem_alloc(&tmem_base_sh, 256);
    tmem_relinquish();
  }
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_base_sh;
  auto part_range = [&](int c, int& bh, int& j0, int& j1) {
    bh = c / a.P;
    const int p = c % a.P;
    j0 = static_cast<int>(static_cast<long long>(p) * a.Nk / a.P);
    j1 = static_cast<int>(static_cast<long long>(p + 1) * a.Nk / a.P);
  };

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      prefetch_tmap(&map_k);
      prefetch_tmap(&map_v);
      int last_round[NS];
      for (int s = 0; s < NS; ++s) last_round[s] = -1;
      int k = 0;
      bool ok = true;
      for (int c = blockIdx.x; ok && c < n_parts; c += gridDim.x) {
        int bh, j0, j1;
        part_range(c, bh, j0, j1);
        for (int j = j0; j < j1; ++j, ++k) {
          const int s = k % NS, r = k / NS;
          if (r > 0 && !(ok = mbar_wait(&empty[s], (r - 1) & 1, a.err, &abort_flag))) break;
          uint8_t* slot = smem + s * L::SLOT;
          mbar_arrive_expect_tx(&full[s], 64 * D * 2 * 2);
          for (int b = 0; b < KBOX; ++b) {
            tma_load_3d(slot + b * 8192, &map_k, &full[s], b * 64, j * 64, bh);
            tma_load_3d(slot + 16384 + b * 8192, &map_v, &full[s], b * 64, j * 64, bh);
          }
          last_round[s] = r;
        }
      }
      if (abort_flag)
        for (int s = 0; s < NS; ++s)
          if (last_round[s] >= 0) mbar_wait(&full[s], last_round[s] & 1, nullptr, nullptr);
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      const uint32_t idesc = idesc_bf16_f32(128, D, 1, 1);
      int k = 0, m = 0;
      bool ok = true;
      for (int c = blockIdx.x; ok && c < n_parts; c += gridDim.x, ++m) {
        int bh, j0, j1;
        part_range(c, bh, j0, j1);
        const int acc = m & 1;
        if (m >= 2 && !(ok = mbar_wait(&acc_empty[acc], ((m >> 1) - 1) & 1, a.err, &abort_flag))) break;
        for (int j = j0; j < j1; ++j, ++k) {
          const int s = k % NS, r = k / NS;
          if (!(ok = mbar_wait(&col_done[s], r & 1, a.err, &abort_flag))) break;
          tc_fence_after();
          const uint32_t sa = smem_u32(smem + s * L::SLOT);
          const uint32_t lbo_a = D == 64 ? smem_u32(zero) - sa : 8192u;
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) {
            const uint64_t ad = smem_desc_sw128(sa + kk * 2048, lbo_a, 1024);
            const uint64_t bd = smem_desc_sw128(sa + 16384 + kk * 2048, 8192, 1024);
            umma_bf16_ss(tmem + acc * 128, ad, bd, idesc, (j > j0 || kk > 0) ? 1u : 0u);
          }
          umma_commit(&empty[s]);
        }
        if (!ok) break;
        umma_commit(&acc_full[acc]);
      }
      umma_commit(&drain);
      mbar_wait(&drain, 0, nullptr, nullptr);
    }
    __syncwarp();
  } else if (warp < 14) {
    // ------------------------------------------------------------ column passes (3 x 128 threads)
    const int cw = (warp - 2) >> 2;      // this warpgroup takes the blocks with k % 3 == cw
    const int wt = tid - 64 - 128 * cw;  // 0..127
    const int bar_id = 1 + cw;
    const int wq = wt >> 5;
    const int cc = wt % CPR, rg = wt / CPR;
    const uint32_t cb = (cc % 8) * 16;
    bool ok = true;
    int k = 0;
    for (int c = blockIdx.x; ok && c < n_parts; c += gridDim.x) {
      int bh, j0, j1;
      part_range(c, bh, j0, j1);
      for (int j = j0; j < j1; ++j, ++k) {
        if (k % 3 != cw) continue;
        const int s = k % NS, r = k / NS;
        ok = mbar_wait(&full[s], r & 1, a.err, &abort_flag);
        if (!(ok = named_barrier_and(bar_id, 128, ok))) break;
        const int valid = min(64, a.N - j * 64);
        uint8_t* kt = smem + s * L::SLOT + (cc / 8) * 8192;
        const uint8_t* vt = smem + s * L::SLOT + 16384 + (cc / 8) * 8192;
        double ks[8];
        float vs[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          ks[e] = 0.0;
          vs[e] = 0.f;
        }
#pragma unroll
        for (int q = 0; q < RPT; ++q) {
          const int rr = rg + RG * q;
          const uint4 ku = *reinterpret_cast<const uint4*>(kt + sw128_offset(rr, cb));
          const uint4 vu = *reinterpret_cast<const uint4*>(vt + sw128_offset(rr, cb));
          const uint32_t w[4] = {ku.x, ku.y, ku.z, ku.w};
          const uint32_t u[4] = {vu.x, vu.y, vu.z, vu.w};
          if (rr < valid) {
#pragma unroll
            for (int e = 0; e < 4; ++e) {  // a bf16 is exact in fp64, and so is the sum of 64
              const float2 x = unpack_bf16x2(w[e]);
              ks[2 * e] += static_cast<double>(x.x);
              ks[2 * e + 1] += static_cast<double>(x.y);
            }
          }
#pragma unroll
          for (int e = 0; e < 4; ++e) {  // value rows past N are zeros
            const float2 y = unpack_bf16x2(u[e]);
            vs[2 * e] += y.x;
            vs[2 * e + 1] += y.y;
          }
        }
        // lanes that differ only in their row group hold the same columns
#pragma unroll
        for (int o = CPR; o < 32; o <<= 1)
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            ks[e] += __shfl_xor_sync(0xffffffffu, ks[e], o);
            vs[e] += __shfl_xor_sync(0xffffffffu, vs[e], o);
          }
        if (lane < CPR) {
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            part_d[cw][wq][cc * 8 + e] = ks[e];
            part_f[cw][wq][cc * 8 + e] = vs[e];
          }
        }
        named_barrier(bar_id, 128);
        if (wt < D) {
          double sum = 0.0;
          float vsum = 0.f;
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            sum += part_d[cw][q][wt];
            vsum += part_f[cw][q][wt];
          }
          const size_t row = static_cast<size_t>(bh) * a.Nk + j;
          const double mean = sum / static_cast<double>(valid);
          if (a.kbar) a.kbar[row * D + wt] = mean;
          a.kcen[row * D + wt] = __double2bfloat16(mean);
          a.vsum[row * D + wt] = __float2bfloat16_rn(vsum);
          mean_f[cw][wt] = static_cast<float>(mean);
        }
        named_barrier(bar_id, 128);  // the block's means are in mean_f
        // the K tile as bf16(k - kbar_j), in place; this thread's 8 columns of the means in two
        // 16-byte reads
        float mean[8];
        {
          const float4 m0 = *reinterpret_cast<const float4*>(&mean_f[cw][cc * 8]);
          const float4 m1 = *reinterpret_cast<const float4*>(&mean_f[cw][cc * 8 + 4]);
          mean[0] = m0.x; mean[1] = m0.y; mean[2] = m0.z; mean[3] = m0.w;
          mean[4] = m1.x; mean[5] = m1.y; mean[6] = m1.z; mean[7] = m1.w;
        }
#pragma unroll
        for (int q = 0; q < RPT; ++q) {
          const int rr = rg + RG * q;
          uint4* kp = reinterpret_cast<uint4*>(kt + sw128_offset(rr, cb));
          const uint4 ku = *kp;
          const uint32_t w[4] = {ku.x, ku.y, ku.z, ku.w};
          uint32_t o[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const float2 x = unpack_bf16x2(w[e]);
            o[e] = rr < valid ? pack_bf16x2(x.x - mean[2 * e], x.y - mean[2 * e + 1]) : 0u;
          }
          *kp = make_uint4(o[0], o[1], o[2], o[3]);
        }
        fence_proxy_async_smem();
        named_barrier(bar_id, 128);  // partial sums consumed; the next block may overwrite them
        mbar_arrive(&col_done[s]);
      }
    }
  } else {
    // ------------------------------------------------------------ epilogue (warps 14..17, 128 threads)
    const int quarter = warp & 3;
    const int d = quarter * 32 + lane;  // row of the accumulator held in this thread's TMEM lane
    int m = 0;
    for (int c = blockIdx.x; c < n_parts; c += gridDim.x, ++m) {
      const int acc = m & 1;
      bool ok = mbar_wait(&acc_full[acc], (m >> 1) & 1, a.err, &abort_flag);
      if (!named_barrier_and(4, 128, ok)) break;
      tc_fence_after();
      if (quarter * 32 < D) {
        float* dst_row = a.hpart + (static_cast<size_t>(c) * D + d) * D;
#pragma unroll
        for (int c0 = 0; c0 < D; c0 += 32) {
          uint32_t rv[32];
          tmem_ld32(tmem + (static_cast<uint32_t>(quarter * 32) << 16) + acc * 128 + c0, rv);
          tmem_wait_ld();
          float4* dst = reinterpret_cast<float4*>(dst_row + c0);
#pragma unroll
          for (int q = 0; q < 8; ++q)
            dst[q] = make_float4(__uint_as_float(rv[4 * q]), __uint_as_float(rv[4 * q + 1]),
                                 __uint_as_float(rv[4 * q + 2]), __uint_as_float(rv[4 * q + 3]));
        }
      }
      tc_fence_before();
      mbar_arrive(&acc_empty[acc]);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 256);
  }
}

// grid (D, BH), block D: Hbar[bh, d, :] = (1 / Nk) sum_p hpart[bh * P + p, d, :], summed in
// part order; written as bf16 (the attention's operand, nullable) and fp32 (nullable).
template <int D>
__global__ void __launch_bounds__(128) hbar_kernel(const float* __restrict__ hpart, __nv_bfloat16* hbar16,
                                                   float* hbar32, int P, int Nk) {
  const int d = blockIdx.x, bh = blockIdx.y, e = threadIdx.x;
  float s = 0.f;
  for (int p = 0; p < P; ++p) s += hpart[((static_cast<size_t>(bh) * P + p) * D + d) * D + e];
  s /= static_cast<float>(Nk);
  const size_t o = (static_cast<size_t>(bh) * D + d) * D + e;
  if (hbar16) hbar16[o] = __float2bfloat16_rn(s);
  if (hbar32) hbar32[o] = s;
}

}  // namespace sla
