// Per-block precompute for the SLA forward:
//   * pool_mean_kernel: mean of the valid tokens of every query (or KV) block, fp64
//     (the router entry point sla_route);
//   * prep_kernel:      one persistent pass over the forward's items [KV blocks | query
//     blocks]; per KV block j, from K_j and V_j:
//       kbar_j = mean of the valid keys (fp64, router input),
//       z_j    = colsum phi(K_j)            (linear-attention normaliser state),
//       h_j    = phi(K_j)^T V_j (D x D)     (linear-attention state, tcgen05 MMA),
//     with phi(x) = elu(x) + 1 (or e^x, the exponential feature map variant); per query
//     block i, qbar_i = mean of the valid queries.
//
// Sources: "SLA2: Sparse-Linear Attention with Learnable Routing and QAT" §2.B
// (pooling adjacent Q/K tokens for the router); "SLA: Beyond Sparsity in
// Diffusion Transformers via Fine-Tunable Sparse-Linear Attention", Abstract
// (O(N) linear attention for marginal weights). The per-block state form
// h_j, z_j is the standard associative rewrite of linear attention.
#pragma once

#include "sm100.cuh"

namespace sla {

// Feature map of the linear branch: FM = 0 is elu(x) + 1 (x + 1 for x > 0, e^x otherwise);
// FM = 1 is the exponential map e^x ("SPLA - Atención de Bloque Dispersa más Lineal para el
// Modelado de Contexto Largo", §2.3).
template <int FM>
__device__ __forceinline__ float phi_f(float x) {
  if constexpr (FM == 1) return __expf(x);
  return x > 0.f ? x + 1.f : __expf(x);
}

// ---------------------------------------------------------------- pooling
// grid: (nblocks, BH); block: 128 threads. x: [BH, N, D] bf16; out: [BH, nblocks, D] fp64.
template <int D>
__global__ void __launch_bounds__(128) pool_mean_kernel(const __nv_bfloat16* __restrict__ x, double* __restrict__ out,
                                                        int N, int block, int nblocks) {
  constexpr int VEC = 8;                 // bf16 per 16-byte load
  constexpr int VPR = D / VEC;           // vectors per row
  constexpr int RSTEP = 128 / VPR;       // rows per pass
  __shared__ double part[RSTEP][D];
  const int i = blockIdx.x, bh = blockIdx.y, t = threadIdx.x;
  const int r0 = i * block, r1 = min(N, r0 + block);
  const int vec = t % VPR, rr = t / VPR;
  double acc[VEC];
#pragma unroll
  for (int e = 0; e < VEC; ++e) acc[e] = 0.0;
  const __nv_bfloat16* base = x + (static_cast<size_t>(bh) * N) * D + vec * VEC;
  for (int r = r0 + rr; r < r1; r += RSTEP) {
    uint4 u = *reinterpret_cast<const uint4*>(base + static_cast<size_t>(r) * D);
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float2 f = unpack_bf16x2(w[e]);
      acc[2 * e] += static_cast<double>(f.x);
      acc[2 * e + 1] += static_cast<double>(f.y);
    }
  }
#pragma unroll
  for (int e = 0; e < VEC; ++e) part[rr][vec * VEC + e] = acc[e];
  __syncthreads();
  if (t < D) {
    double s = 0.0;
#pragma unroll
    for (int g = 0; g < RSTEP; ++g) s += part[g][t];
    out[(static_cast<size_t>(bh) * nblocks + i) * D + t] = s / static_cast<double>(r1 - r0);
  }
}

// ---------------------------------------------------------------- fused precompute
struct PrepArgs {
  int BH, N, Nq, Nk, block_q;
  double* qbar;            // [BH, Nq, D] query-block means (nullable: no query pooling)
  double* kbar;            // [BH, Nk, D] KV-block means (nullable)
  __nv_bfloat16* hst;      // [BH, Nk, LD] bf16: h_j row-major (D*D) then z_j (D) then zero pad (forward)
  float* h32;              // [BH, Nk, D, D] fp32 (state export), used when hst == nullptr
  float* z32;              // [BH, Nk, D] fp32 (state export)
  int LD;                  // row length of hst in elements (D*D + 128)
  uint32_t* err;
};

template <int D>
struct PrepSmem {
  // Five ring slots and one staging tile: more loads in flight paid more than overlapping two
  // TMA stores (measured: 0.125 -> 0.119 ms at B=1 H=12 N=32760 D=128).
  static constexpr int NSLOT = 5;
  static constexpr uint32_t SLOT = 32768;                // K (16 KB) then V (16 KB), or one query block
  static constexpr uint32_t STAGE = D * 128 * (D / 64);  // bf16 h_j tile for the TMA store
  static constexpr uint32_t ZERO = D == 64 ? 8192 : 0;   // zero rows 64..127 of phi(K)^T when D = 64
  static constexpr uint32_t total() { return NSLOT * SLOT + STAGE + ZERO + 1024; }
};

// Column pass of one warpgroup over a ROWS x D tile (16-byte chunks, 128-byte swizzle):
// thread (cc, rg) owns columns 8cc..8cc+7 of rows rg, rg + RG, ...; it sums the valid
// rows in fp64 and, for a K tile (PHI), sums phi(k) in fp32 and rewrites the tile in
// place as phi(k) (zero past the sequence end). The row groups of a warp are summed with
// shuffles; the warp's partial sums go to part_d / part_f[wq] (wq = warp within the group),
// column 8 cc + e at entry e (D / 8) + cc, so that the lanes' stores fall in distinct banks.
template <int D, int ROWS, bool PHI, int FM = 0>
__device__ __forceinline__ void column_pass(uint8_t* tile0, int cc, int rg, int wq, int valid, double (*part_d)[D],
                                            float (*part_f)[D]) {
  constexpr int RG = 128 / (D / 8);
  uint8_t* tile = tile0 + (cc / 8) * (ROWS * 128);
  const uint32_t cb = (cc % 8) * 16;
  double ks[8];
  float zs[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) {
    ks[e] = 0.0;
    zs[e] = 0.f;
  }
#pragma unroll
  for (int k = 0; k < ROWS / RG; ++k) {
    const int rr = rg + RG * k;
    uint4* p = reinterpret_cast<uint4*>(tile + sw128_offset(rr, cb));
    const uint4 u = *p;
    uint32_t w[4] = {u.x, u.y, u.z, u.w};
    const bool in = rr < valid;
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float2 x = unpack_bf16x2(w[e]);
      float f0 = 0.f, f1 = 0.f;
      if (in) {
        ks[2 * e] += static_cast<double>(x.x);
        ks[2 * e + 1] += static_cast<double>(x.y);
        if (PHI) {
          f0 = phi_f<FM>(x.x);
          f1 = phi_f<FM>(x.y);
          zs[2 * e] += f0;
          zs[2 * e + 1] += f1;
        }
      }
      w[e] = pack_bf16x2(f0, f1);
    }
    if (PHI) *p = make_uint4(w[0], w[1], w[2], w[3]);
  }
  // lanes that differ only in their row group hold the same columns
#pragma unroll
  for (int o = D / 8; o < 32; o <<= 1)
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      ks[e] += __shfl_xor_sync(0xffffffffu, ks[e], o);
      zs[e] += __shfl_xor_sync(0xffffffffu, zs[e], o);
    }
  if ((threadIdx.x & 31) < D / 8) {
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      part_d[wq][e * (D / 8) + cc] = ks[e];
      part_f[wq][e * (D / 8) + cc] = zs[e];
    }
  }
}

// Persistent, warp-specialised precompute; one CTA per SM, 576 threads.
// A CTA walks the items g = blockIdx.x, blockIdx.x + gridDim.x, ... of the list
// [KV blocks of every head | query blocks of every head (when qbar is set)].
//   warp 0      TMA producer: K_j and V_j (or a query block) into a 5-slot ring
//   warps 2..5, 10..13 and 14..17
//               three column-pass warpgroups taking items in turn: over 16-byte
//               chunks, the sum of the valid rows in fp64 (block means), and for KV
//               blocks the sum of phi(k) (z_j) while the K tile is rewritten in
//               place as phi(k) (zero past the sequence end)
//   warp 1      tcgen05 issuer: h_j = phi(K_j)^T V_j (M=128, N=D, K=64 tokens; both
//               operands MN-major) into one of two TMEM accumulators
//   warps 6..9  epilogue: TMEM -> bf16 -> the staging tile -> TMA store (forward),
//               or TMEM -> fp32 straight to global memory (state export)
// For D = 64 the second half of phi(K)^T (rows 64..127 of the M=128 MMA) points
// at a zero tile, so the result rows 64..127 are zero and ignored.
template <int D, int FM = 0>
__global__ void __launch_bounds__(576, 1)
    prep_kernel(const __grid_constant__ CUtensorMap map_q, const __grid_constant__ CUtensorMap map_k,
                const __grid_constant__ CUtensorMap map_v, const __grid_constant__ CUtensorMap map_hout, PrepArgs a) {
  using L = PrepSmem<D>;
  constexpr int NS = L::NSLOT;
  constexpr int KBOX = D / 64;  // 64-column boxes per row
  constexpr int CPR = D / 8;    // 16-byte chunks per row
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* stage0 = smem + NS * L::SLOT;
  uint8_t* zero = stage0 + L::STAGE;
  __shared__ uint64_t full[NS], phi_done[NS], empty[NS], acc_full[2], acc_empty[2], drain;
  __shared__ uint32_t tmem_base_sh;
  __shared__ int abort_flag;
  __shared__ double part_d[3][4][D];  // [column warpgroup][warp][column]
  __shared__ float part_f[3][4][D];

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int n_kv = a.BH * a.Nk;
  const int n_items = n_kv + (a.qbar ? a.BH * a.Nq : 0);
  const bool bf16_out = a.hst != nullptr;
  grid_dep_launch();
  if (tid == 0) {
    for (int s = 0; s < NS; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&phi_done[s], 128);
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

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      prefetch_tmap(&map_k);
      prefetch_tmap(&map_v);
      if (a.qbar) prefetch_tmap(&map_q);
      if (bf16_out) prefetch_tmap(&map_hout);
      int last_round[NS];
      for (int s = 0; s < NS; ++s) last_round[s] = -1;
      int k = 0;
      for (int g = blockIdx.x; g < n_items; g += gridDim.x, ++k) {
        const int s = k % NS, r = k / NS;
        if (r > 0 && !mbar_wait(&empty[s], (r - 1) & 1, a.err, &abort_flag)) break;
        uint8_t* slot = smem + s * L::SLOT;
        if (g < n_kv) {
          const int bh = g / a.Nk, j = g % a.Nk;
          mbar_arrive_expect_tx(&full[s], 64 * D * 2 * 2);
          for (int b = 0; b < KBOX; ++b) {
            tma_load_3d(slot + b * 8192, &map_k, &full[s], b * 64, j * 64, bh);
            tma_load_3d(slot + 16384 + b * 8192, &map_v, &full[s], b * 64, j * 64, bh);
          }
        } else {
          const int q = g - n_kv, bh = q / a.Nq, i = q % a.Nq;
          mbar_arrive_expect_tx(&full[s], a.block_q * D * 2);
          for (int b = 0; b < KBOX; ++b)
            tma_load_3d(slot + b * (a.block_q * 128), &map_q, &full[s], b * 64, i * a.block_q, bh);
        }
        last_round[s] = r;
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
      for (int g = blockIdx.x; g < n_items; g += gridDim.x, ++k) {
        const int s = k % NS, r = k / NS;
        if (!mbar_wait(&phi_done[s], r & 1, a.err, &abort_flag)) break;
        if (g >= n_kv) {  // a query block: nothing to multiply, the slot is free again
          mbar_arrive(&empty[s]);
          continue;
        }
        const int acc = m & 1;
        if (m >= 2 && !mbar_wait(&acc_empty[acc], ((m >> 1) - 1) & 1, a.err, &abort_flag)) break;
        tc_fence_after();
        const uint32_t sa = smem_u32(smem + s * L::SLOT);
        const uint32_t lbo_a = D == 64 ? smem_u32(zero) - sa : 8192u;
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {
          const uint64_t ad = smem_desc_sw128(sa + kk * 2048, lbo_a, 1024);
          const uint64_t bd = smem_desc_sw128(sa + 16384 + kk * 2048, 8192, 1024);
          umma_bf16_ss(tmem + acc * 128, ad, bd, idesc, kk > 0 ? 1u : 0u);
        }
        umma_commit(&empty[s]);
        umma_commit(&acc_full[acc]);
        ++m;
      }
      umma_commit(&drain);
      mbar_wait(&drain, 0, nullptr, nullptr);
    }
    __syncwarp();
  } else if (warp < 6 || warp >= 10) {
    // ------------------------------------------------------------ column passes (2 x 128 threads)
    const int cw = warp < 6 ? 0 : (warp < 14 ? 1 : 2);  // this warpgroup takes the items with k % 3 == cw
    const int wt = tid - (cw == 0 ? 64 : (cw == 1 ? 320 : 448));
    const int bar_id = cw == 0 ? 1 : (cw == 1 ? 3 : 4);
    const int wq = wt >> 5;
    const int cc = wt % CPR, rg = wt / CPR;
    int k = cw;
    for (int g = blockIdx.x + cw * gridDim.x; g < n_items; g += 3 * gridDim.x, k += 3) {
      const int s = k % NS, r = k / NS;
      bool ok = mbar_wait(&full[s], r & 1, a.err, &abort_flag);
      if (!named_barrier_and(bar_id, 128, ok)) break;
      const bool isq = g >= n_kv;
      int bh, idx, rows;
      if (isq) {
        const int q = g - n_kv;
        bh = q / a.Nq;
        idx = q % a.Nq;
        rows = a.block_q;
      } else {
        bh = g / a.Nk;
        idx = g % a.Nk;
        rows = 64;
      }
      const int valid = min(rows, a.N - idx * rows);
      uint8_t* slotp = smem + s * L::SLOT;
      if (isq) {
        if (a.block_q == 128)
          column_pass<D, 128, false>(slotp, cc, rg, wq, valid, part_d[cw], part_f[cw]);
        else
          column_pass<D, 64, false>(slotp, cc, rg, wq, valid, part_d[cw], part_f[cw]);
      } else {
        column_pass<D, 64, true, FM>(slotp, cc, rg, wq, valid, part_d[cw], part_f[cw]);
      }
      if (!isq) fence_proxy_async_smem();
      named_barrier(bar_id, 128);
      if (wt < D) {
        // entry wt of the partial sums is column (wt % (D / 8)) * 8 + wt / (D / 8)
        const int col = (wt % (D / 8)) * 8 + wt / (D / 8);
        double sum = 0.0;
        float zsum = 0.f;
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          sum += part_d[cw][q][wt];
          zsum += part_f[cw][q][wt];
        }
        if (isq) {
          a.qbar[(static_cast<size_t>(bh) * a.Nq + idx) * D + col] = sum / static_cast<double>(valid);
        } else {
          const size_t row = static_cast<size_t>(bh) * a.Nk + idx;
          if (a.kbar) a.kbar[row * D + col] = sum / static_cast<double>(valid);
          if (bf16_out) {
            __nv_bfloat16* zr = a.hst + row * a.LD + D * D;
            zr[col] = __float2bfloat16_rn(zsum);
            if (D == 64) zr[64 + wt] = __float2bfloat16_rn(0.f);
          } else if (a.z32) {
            a.z32[row * D + col] = zsum;
          }
        }
      }
      named_barrier(bar_id, 128);  // partial sums consumed; the next item may overwrite them
      mbar_arrive(&phi_done[s]);
    }
  } else {
    // ------------------------------------------------------------ epilogue (warps 6..9, 128 threads)
    const int et = tid - 192;
    const int quarter = warp & 3;
    const int d = quarter * 32 + lane;  // row of h_j held in this thread's TMEM lane
    int m = 0;
    for (int g = blockIdx.x; g < n_kv; g += gridDim.x, ++m) {
      const int bh = g / a.Nk, j = g % a.Nk;
      const int acc = m & 1;
      bool ok = mbar_wait(&acc_full[acc], (m >> 1) & 1, a.err, &abort_flag);
      if (!named_barrier_and(2, 128, ok)) break;
      tc_fence_after();
      uint8_t* stg = stage0;
      if (bf16_out) {
        if (et == 0) tma_store_wait_read();  // the previous block's store is done reading the staging tile
        named_barrier(2, 128);
      }
      if (quarter * 32 < D) {
        const size_t row = static_cast<size_t>(bh) * a.Nk + j;
#pragma unroll
        for (int c0 = 0; c0 < D; c0 += 32) {
          uint32_t rv[32];
          tmem_ld32(tmem + (static_cast<uint32_t>(quarter * 32) << 16) + acc * 128 + c0, rv);
          tmem_wait_ld();
          if (bf16_out) {
            uint8_t* box = stg + (c0 >> 6) * (D * 128);
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              uint4 u;
              u.x = pack_bf16x2(__uint_as_float(rv[8 * q + 0]), __uint_as_float(rv[8 * q + 1]));
              u.y = pack_bf16x2(__uint_as_float(rv[8 * q + 2]), __uint_as_float(rv[8 * q + 3]));
              u.z = pack_bf16x2(__uint_as_float(rv[8 * q + 4]), __uint_as_float(rv[8 * q + 5]));
              u.w = pack_bf16x2(__uint_as_float(rv[8 * q + 6]), __uint_as_float(rv[8 * q + 7]));
              *reinterpret_cast<uint4*>(box + sw128_offset(d, ((c0 & 63) >> 3) * 16 + q * 16)) = u;
            }
          } else {
            float4* dst = reinterpret_cast<float4*>(a.h32 + (row * D + d) * D + c0);
#pragma unroll
            for (int q = 0; q < 8; ++q)
              dst[q] = make_float4(__uint_as_float(rv[4 * q]), __uint_as_float(rv[4 * q + 1]),
                                   __uint_as_float(rv[4 * q + 2]), __uint_as_float(rv[4 * q + 3]));
          }
        }
      }
      tc_fence_before();
      mbar_arrive(&acc_empty[acc]);
      if (bf16_out) {
        fence_proxy_async_smem();
        named_barrier(2, 128);
        if (et == 0) {
          for (int b = 0; b < KBOX; ++b) tma_store_3d(&map_hout, stg + b * (D * 128), b * 64, 0, bh * a.Nk + j);
          tma_store_commit();
        }
      }
    }
    if (et == 0 && bf16_out) tma_store_wait_all();
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 256);
  }
}

}  // namespace sla
