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

template <int D>
struct KvPrepSmem {
  static constexpr uint32_t SLOT = 32768;               // K (16 KB, zero upper half when D = 64) + V (16 KB)
  static constexpr uint32_t STAGE = D * 128 * (D / 64); // bf16 h_j staging for the TMA store
  static constexpr uint32_t total() { return 2 * SLOT + STAGE + 1024; }
};

// One CTA walks over KV blocks g = blockIdx.x, blockIdx.x + gridDim.x, ... with a
// two-slot TMA ring; two CTAs share an SM. 128 threads.
//   column pass  16-byte vectors: sum k (fp64) and phi(k) (fp32) per column, and
//                rewrite the K tile in place as phi(k) (zero past the sequence end)
//   MMA          h_j = phi(K_j)^T V_j on tcgen05 (M=128, N=D, K=64 tokens; both
//                operands MN-major); for D = 64 rows 64..127 of phi(K)^T read zeros
//   epilogue     bf16 h_j staged in shared memory and written by one TMA store
//                (forward), or fp32 straight from registers (state export).
template <int D>
__global__ void __launch_bounds__(128, 2) kv_prep_kernel(const __grid_constant__ CUtensorMap map_k,
                                                         const __grid_constant__ CUtensorMap map_v,
                                                         const __grid_constant__ CUtensorMap map_hout, KvPrepArgs a) {
  using L = KvPrepSmem<D>;
  constexpr int BK = 64;
  constexpr int KBOX = D / 64;              // 64-column boxes per row
  constexpr uint32_t TX = BK * D * 2 * 2;   // K + V bytes per block
  constexpr int CPR = D / 8;                // 16-byte chunks per row
  constexpr int RG = 128 / CPR;             // row groups
  constexpr int RPT = BK / RG;              // rows per thread
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* slot[2] = {smem, smem + L::SLOT};
  uint8_t* stage = smem + 2 * L::SLOT;
  __shared__ uint64_t bar_full[2], bar_mma;
  __shared__ uint32_t tmem_base_sh;
  __shared__ int abort_flag;
  __shared__ double ksum_part[RG][D];
  __shared__ float zsum_part[RG][D];

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int total = a.BH * a.Nk;
  const bool bf16_out = a.hst != nullptr;
  if (tid == 0) {
    mbar_init(&bar_full[0], 1);
    mbar_init(&bar_full[1], 1);
    mbar_init(&bar_mma, 1);
    abort_flag = 0;
    fence_mbar_init();
    prefetch_tmap(&map_k);
    prefetch_tmap(&map_v);
    if (bf16_out) prefetch_tmap(&map_hout);
  }
  if (D == 64) {  // zero the upper halves of both K areas once (TMA never writes them)
    for (int s = 0; s < 2; ++s)
      for (int o = tid * 16; o < 8192; o += 128 * 16) *reinterpret_cast<uint4*>(slot[s] + 8192 + o) = make_uint4(0, 0, 0, 0);
    fence_proxy_async_smem();
  }
  if (warp == 0) {
    tmem_alloc(&tmem_base_sh, 128);
    tmem_relinquish();
  }
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_base_sh;

  // Thread 0 tracks which slots have a load in flight (parity of its phase, or -1)
  // so that an aborted CTA can let them land before it retires.
  int inflight[2] = {-1, -1};
  int mma_parity = -1;
  auto issue_load = [&](int g, int s, int round) {
    const int bh = g / a.Nk, j = g % a.Nk;
    mbar_arrive_expect_tx(&bar_full[s], TX);
#pragma unroll
    for (int b = 0; b < KBOX; ++b) {
      tma_load_3d(slot[s] + b * 8192, &map_k, &bar_full[s], b * 64, j * BK, bh);
      tma_load_3d(slot[s] + 16384 + b * 8192, &map_v, &bar_full[s], b * 64, j * BK, bh);
    }
    inflight[s] = round & 1;
  };
  if (tid == 0) {
    if (blockIdx.x < total) issue_load(blockIdx.x, 0, 0);
    if (blockIdx.x + gridDim.x < total) issue_load(blockIdx.x + gridDim.x, 1, 0);
  }
  const uint32_t idesc = idesc_bf16_f32(128, D, 1, 1);
  const int cc = tid % CPR, rg = tid / CPR;

  int n = 0;
  for (int g = blockIdx.x; g < total; g += gridDim.x, ++n) {
    const int s = n & 1;
    const int bh = g / a.Nk, j = g % a.Nk;
    const int valid = min(BK, a.N - j * BK);
    bool ok = mbar_wait(&bar_full[s], (n >> 1) & 1, a.err, &abort_flag);
    if (__syncthreads_or(!ok)) break;
    if (tid == 0) inflight[s] = -1;

    // Column pass over 16-byte chunks: thread (cc, rg) owns columns 8cc..8cc+7 of rows rg + RG*k.
    {
      uint8_t* tile = slot[s] + (cc / 8) * 8192;
      const uint32_t cb = (cc % 8) * 16;
      double ks[8];
      float zs[8];
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        ks[e] = 0.0;
        zs[e] = 0.f;
      }
#pragma unroll
      for (int k = 0; k < RPT; ++k) {
        const int r = rg + RG * k;
        uint4* p = reinterpret_cast<uint4*>(tile + sw128_offset(r, cb));
        const uint4 u = *p;
        uint32_t w[4] = {u.x, u.y, u.z, u.w};
        const bool in = r < valid;
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float2 kv = unpack_bf16x2(w[e]);
          float f0 = 0.f, f1 = 0.f;
          if (in) {
            ks[2 * e] += static_cast<double>(kv.x);
            ks[2 * e + 1] += static_cast<double>(kv.y);
            f0 = phi_f(kv.x);
            f1 = phi_f(kv.y);
            zs[2 * e] += f0;
            zs[2 * e + 1] += f1;
          }
          w[e] = pack_bf16x2(f0, f1);
        }
        *p = make_uint4(w[0], w[1], w[2], w[3]);
      }
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        ksum_part[rg][cc * 8 + e] = ks[e];
        zsum_part[rg][cc * 8 + e] = zs[e];
      }
    }
    fence_proxy_async_smem();
    __syncthreads();
    if (tid == 0) {
      tc_fence_after();
#pragma unroll
      for (int kk = 0; kk < BK / 16; ++kk) {
        uint64_t ad = smem_desc_sw128(smem_u32(slot[s]) + kk * 2048, 8192, 1024);
        uint64_t bd = smem_desc_sw128(smem_u32(slot[s]) + 16384 + kk * 2048, 8192, 1024);
        umma_bf16_ss(tmem, ad, bd, idesc, kk > 0);
      }
      umma_commit(&bar_mma);
      mma_parity = n & 1;
    }
    // kbar and z while the MMA runs
    if (tid < D) {
      double ks = 0.0;
      float zs = 0.f;
#pragma unroll
      for (int q = 0; q < RG; ++q) {
        ks += ksum_part[q][tid];
        zs += zsum_part[q][tid];
      }
      const size_t row = static_cast<size_t>(bh) * a.Nk + j;
      if (a.kbar) a.kbar[row * D + tid] = ks / static_cast<double>(valid);
      if (bf16_out) {
        __nv_bfloat16* zr = a.hst + row * a.LD + D * D;
        zr[tid] = __float2bfloat16_rn(zs);
        if (D == 64) zr[64 + tid] = __float2bfloat16_rn(0.f);
      } else if (a.z32) {
        a.z32[row * D + tid] = zs;
      }
    }
    ok = mbar_wait(&bar_mma, n & 1, a.err, &abort_flag);
    if (tid == 0 && bf16_out) tma_store_wait_read();  // the previous block's store has left the staging tile
    if (__syncthreads_or(!ok)) break;
    tc_fence_after();
    if (tid == 0) mma_parity = -1;
    // The MMA has consumed slot s: refill it with the block two steps ahead.
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
        if (bf16_out) {
          uint8_t* box = stage + (c0 >> 6) * (D * 128);
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            uint4 u;
            u.x = pack_bf16x2(__uint_as_float(r[8 * q + 0]), __uint_as_float(r[8 * q + 1]));
            u.y = pack_bf16x2(__uint_as_float(r[8 * q + 2]), __uint_as_float(r[8 * q + 3]));
            u.z = pack_bf16x2(__uint_as_float(r[8 * q + 4]), __uint_as_float(r[8 * q + 5]));
            u.w = pack_bf16x2(__uint_as_float(r[8 * q + 6]), __uint_as_float(r[8 * q + 7]));
            *reinterpret_cast<uint4*>(box + sw128_offset(d, ((c0 & 63) >> 3) * 16 + q * 16)) = u;
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
    if (bf16_out) fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    if (tid == 0 && bf16_out) {
      for (int b = 0; b < KBOX; ++b) tma_store_3d(&map_hout, stage + b * (D * 128), b * 64, 0, bh * a.Nk + j);
      tma_store_commit();
    }
  }
  // After an abort: let loads and the MMA still in flight finish before the CTA retires.
  if (tid == 0) {
    for (int s = 0; s < 2; ++s)
      if (inflight[s] >= 0) mbar_wait(&bar_full[s], inflight[s], nullptr, nullptr);
    if (mma_parity >= 0) mbar_wait(&bar_mma, mma_parity, nullptr, nullptr);
    if (bf16_out) tma_store_wait_all();
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, 128);
  }
}

}  // namespace sla
