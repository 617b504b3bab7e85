// Per-block precompute for the SLA forward:
//   * pool_mean_kernel: mean of the valid query tokens of every query block (fp64)
//   * kv_prep_kernel:   per KV block j, in one pass over K_j and V_j:
//       kbar_j = mean of the valid keys (fp64, router input),
//       z_j    = colsum phi(K_j)            (linear-attention normaliser state),
//       h_j    = phi(K_j)^T V_j (D x D)     (linear-attention state, tcgen05 MMA),
//     with phi(x) = elu(x) + 1.
//
// Sources: "SLA2: Sparse-Linear Attention with Learnable Routing and QAT" §2.B
// (pooling adjacent Q/K tokens for the router); "SLA: Beyond Sparsity in
// Diffusion Transformers via Fine-Tunable Sparse-Linear Attention", Abstract
// (O(N) linear attention for marginal weights). The per-block state form
// h_j, z_j is the standard associative rewrite of linear attention.
#pragma once

#include "sm100.cuh"

namespace sla {

__device__ __forceinline__ float phi_f(float x) { return x > 0.f ? x + 1.f : __expf(x); }

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
      float2 f = unpack_bf16x2(w[e]);
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

// ---------------------------------------------------------------- KV states
struct KvPrepArgs {
  int BH, N, Nk;
  double* kbar;            // [BH, Nk, D] (nullable)
  __nv_bfloat16* hst;      // [BH, Nk, LD] bf16: h_j row-major (D*D) then z_j (D) then zero pad (forward)
  float* h32;              // [BH, Nk, D, D] fp32 (state export), used when hst == nullptr
  float* z32;              // [BH, Nk, D] fp32 (state export)
  int LD;                  // row length of hst in elements (D*D + 128)
  uint32_t* err;
};

// One CTA walks over KV blocks g = blockIdx.x, blockIdx.x + gridDim.x, ...
// with a two-stage TMA ring. 128 threads. Dynamic smem: 2 stages x (K 16 KB + V 16 KB).
// For D = 64 the K stage keeps a zeroed second half so the M = 128 MMA reads
// zeros for rows 64..127 of phi(K)^T.
template <int D>
__global__ void __launch_bounds__(128) kv_prep_kernel(const __grid_constant__ CUtensorMap map_k,
                                                      const __grid_constant__ CUtensorMap map_v, KvPrepArgs a) {
  constexpr int BK = 64;
  constexpr int KBOX = D / 64;              // 64-column boxes per row
  constexpr uint32_t TILE = 16384;           // bytes reserved per K (or V) stage
  constexpr uint32_t TX = BK * D * 2 * 2;    // K + V bytes per block
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sK[2] = {smem, smem + 2 * TILE};
  uint8_t* sV[2] = {smem + TILE, smem + 3 * TILE};
  __shared__ uint64_t bar_full[2], bar_mma;
  __shared__ uint32_t tmem_base_sh;
  __shared__ int abort_flag;
  __shared__ double ksum_part[2][D];
  __shared__ float zsum_part[2][D];

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int total = a.BH * a.Nk;
  if (tid == 0) {
    mbar_init(&bar_full[0], 1);
    mbar_init(&bar_full[1], 1);
    mbar_init(&bar_mma, 1);
    abort_flag = 0;
    fence_mbar_init();
    prefetch_tmap(&map_k);
    prefetch_tmap(&map_v);
  }
  if (D == 64) {  // zero the upper halves of both K stages once
    for (int s = 0; s < 2; ++s)
      for (int o = tid * 16; o < 8192; o += 128 * 16) *reinterpret_cast<uint4*>(sK[s] + 8192 + o) = make_uint4(0, 0, 0, 0);
    fence_proxy_async_smem();
  }
  if (warp == 0) {
    tmem_alloc(&tmem_base_sh, 128);
    tmem_relinquish();
  }
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_base_sh;

  // Thread 0 tracks which stages have a load in flight (parity of its phase, or -1)
  // so that an aborted CTA can let them land before it retires.
  int inflight[2] = {-1, -1};
  int mma_parity = -1;
  auto issue_load = [&](int g, int s, int round) {
    const int bh = g / a.Nk, j = g % a.Nk;
    mbar_arrive_expect_tx(&bar_full[s], TX);
#pragma unroll
    for (int b = 0; b < KBOX; ++b) {
      tma_load_3d(sK[s] + b * 8192, &map_k, &bar_full[s], b * 64, j * BK, bh);
      tma_load_3d(sV[s] + b * 8192, &map_v, &bar_full[s], b * 64, j * BK, bh);
    }
    inflight[s] = round & 1;
  };
  if (tid == 0) {
    if (blockIdx.x < total) issue_load(blockIdx.x, 0, 0);
    if (blockIdx.x + gridDim.x < total) issue_load(blockIdx.x + gridDim.x, 1, 0);
  }
  const uint32_t idesc = idesc_bf16_f32(128, D, 1, 1);

  int n = 0;
  for (int g = blockIdx.x; g < total; g += gridDim.x, ++n) {
    const int s = n & 1;
    const int bh = g / a.Nk, j = g % a.Nk;
    const int valid = min(BK, a.N - j * BK);
    bool ok = mbar_wait(&bar_full[s], (n >> 1) & 1, a.err, &abort_flag);
    if (__syncthreads_or(!ok)) break;
    if (tid == 0) inflight[s] = -1;

    // Column pass: a thread owns column c over all rows (D = 128) or half of them (D = 64);
    // it sums k in fp64 and phi(k) in fp32, and rewrites the tile in place as phi(k)
    // (zero on rows past the end of the sequence, which TMA filled with zeros).
    {
      constexpr int HALVES = 128 / D;
      const int c = tid % D, half = tid / D;
      const int rbeg = half * (BK / HALVES), rend = rbeg + BK / HALVES;
      uint8_t* tile = sK[s] + (c / 64) * 8192;
      const uint32_t cb = (c % 64) * 2;
      double ks = 0.0;
      float zs = 0.f;
      for (int r = rbeg; r < rend; ++r) {
        __nv_bfloat16* p = reinterpret_cast<__nv_bfloat16*>(tile + sw128_offset(r, cb));
        float kv = __bfloat162float(*p);
        float f = 0.f;
        if (r < valid) {
          ks += static_cast<double>(kv);
          f = phi_f(kv);
          zs += f;
        }
        *p = __float2bfloat16_rn(f);
      }
      ksum_part[half][c] = ks;
      zsum_part[half][c] = zs;
    }
    fence_proxy_async_smem();
    __syncthreads();
    if (tid == 0) {
      tc_fence_after();
#pragma unroll
      for (int kk = 0; kk < BK / 16; ++kk) {
        uint64_t ad = smem_desc_sw128(smem_u32(sK[s]) + kk * 2048, 8192, 1024);
        uint64_t bd = smem_desc_sw128(smem_u32(sV[s]) + kk * 2048, 8192, 1024);
        umma_bf16_ss(tmem, ad, bd, idesc, kk > 0);
      }
      umma_commit(&bar_mma);
      mma_parity = n & 1;
    }
    // kbar and z while the MMA runs
    if (tid < D) {
      double ks = ksum_part[0][tid];
      float zs = zsum_part[0][tid];
      if (D == 64) {
        ks += ksum_part[1][tid];
        zs += zsum_part[1][tid];
      }
      const size_t row = static_cast<size_t>(bh) * a.Nk + j;
      if (a.kbar) a.kbar[row * D + tid] = ks / static_cast<double>(valid);
      if (a.hst) {
        __nv_bfloat16* zr = a.hst + row * a.LD + D * D;
        zr[tid] = __float2bfloat16_rn(zs);
        if (D == 64) zr[64 + tid] = __float2bfloat16_rn(0.f);
      } else if (a.z32) {
        a.z32[row * D + tid] = zs;
      }
    }
    ok = mbar_wait(&bar_mma, n & 1, a.err, &abort_flag);
    if (__syncthreads_or(!ok)) break;
    tc_fence_after();
    if (tid == 0) mma_parity = -1;
    // The MMA has consumed stage s: refill it with the block two steps ahead.
    if (tid == 0 && g + 2 * gridDim.x < total) issue_load(g + 2 * gridDim.x, s, (n >> 1) + 1);
    // Epilogue: warp w holds rows d = 32 w .. 32 w + 31 of h_j.
    if (warp * 32 < D) {
      const int d = warp * 32 + lane;
      const size_t row = static_cast<size_t>(bh) * a.Nk + j;
#pragma unroll
      for (int c0 = 0; c0 < D; c0 += 32) {
        uint32_t r[32];
        tmem_ld32(tmem + (static_cast<uint32_t>(warp * 32) << 16) + c0, r);
        tmem_wait_ld();
        if (a.hst) {
          uint4* dst = reinterpret_cast<uint4*>(a.hst + row * a.LD + static_cast<size_t>(d) * D + c0);
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            uint4 u;
            u.x = pack_bf16x2(__uint_as_float(r[8 * q + 0]), __uint_as_float(r[8 * q + 1]));
            u.y = pack_bf16x2(__uint_as_float(r[8 * q + 2]), __uint_as_float(r[8 * q + 3]));
            u.z = pack_bf16x2(__uint_as_float(r[8 * q + 4]), __uint_as_float(r[8 * q + 5]));
            u.w = pack_bf16x2(__uint_as_float(r[8 * q + 6]), __uint_as_float(r[8 * q + 7]));
            dst[q] = u;
          }
        } else {
          float4* dst = reinterpret_cast<float4*>(a.h32 + (row * D + d) * D + c0);
#pragma unroll
          for (int q = 0; q < 8; ++q)
            dst[q] = make_float4(__uint_as_float(r[4 * q]), __uint_as_float(r[4 * q + 1]),
                                 __uint_as_float(r[4 * q + 2]), __uint_as_float(r[4 * q + 3]));
        }
      }
    }
    tc_fence_before();
    __syncthreads();
  }
  // After an abort: let loads and the MMA still in flight finish before the CTA retires.
  if (tid == 0) {
    for (int s = 0; s < 2; ++s)
      if (inflight[s] >= 0) mbar_wait(&bar_full[s], inflight[s], nullptr, nullptr);
    if (mma_parity >= 0) mbar_wait(&bar_mma, mma_parity, nullptr, nullptr);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, 128);
  }
}

}  // namespace sla
