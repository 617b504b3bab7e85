// Marginal-state aggregation for the SLA linear branch:
//
//   [H_i | Z_i] = sum over marginal KV blocks j of [h_j | z_j]
//
// written as one tensor-core GEMM per (batch, head): C = W * Hst, where
// W [Nq x Nk] is the 0/1 marginal indicator from the router and Hst [Nk x LD]
// stacks every block's state h_j (D*D, row-major) followed by z_j (D) and zero
// padding. C row i holds H_i (bf16 output) and Z_i (fp32 output).
//
// Source: "SLA: Beyond Sparsity in Diffusion Transformers via Fine-Tunable
// Sparse-Linear Attention", Abstract (O(N) linear attention over the marginal
// weights). Summing the per-block states of the marginal set is the linear
// branch's definition; the GEMM form only batches those sums over the query
// blocks of a head so that they run on the tensor cores.
#pragma once

#include "sm100.cuh"

namespace sla {

struct AggArgs {
  int Nq, Nk, LD;
  __nv_bfloat16* Hagg;   // [BH, Nq, D*D]
  float* Zagg;           // [BH, Nq, D]
  uint32_t* err;
};

constexpr uint32_t kAggStageBytes = 3 * 16384;  // A for two M-tiles + one B tile (64 x 128)

// grid: (LD/128, ceil(Nq/256), BH); block 128 (warp 0: TMA, warp 1: MMA, all: epilogue).
// One CTA owns 128 state columns for up to two 128-row M-tiles of query blocks, so each
// stacked-state tile is read once per head. Two CTAs share an SM: 2 stages x 48 KB of
// shared memory, 256 TMEM columns (M-tile t accumulates in columns [128 t, 128 t + 128)).
template <int D>
__global__ void __launch_bounds__(128, 2) agg_kernel(const __grid_constant__ CUtensorMap map_w,
                                                     const __grid_constant__ CUtensorMap map_h,
                                                     const __grid_constant__ CUtensorMap map_out, AggArgs a) {
  constexpr int NSTAGE = 2;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  __shared__ uint64_t full[NSTAGE], empty[NSTAGE], acc_full, drain;
  __shared__ uint32_t tmem_base_sh;
  __shared__ int abort_flag;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int n0 = blockIdx.x * 128, m0 = blockIdx.y * 256, bh = blockIdx.z;
  const int nm = (m0 + 128 < a.Nq) ? 2 : 1;  // M-tiles this CTA owns
  const int nk = (a.Nk + 63) / 64;
  if (tid == 0) {
    for (int s = 0; s < NSTAGE; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    mbar_init(&acc_full, 1);
    mbar_init(&drain, 1);
    abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(&tmem_base_sh, 256);
    tmem_relinquish();
  }
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_base_sh;

  if (warp == 0) {
    if (lane == 0) {
      prefetch_tmap(&map_w);
      prefetch_tmap(&map_h);
      prefetch_tmap(&map_out);
      int last_round[NSTAGE] = {-1, -1};
      for (int k = 0; k < nk; ++k) {
        const int s = k % NSTAGE, r = k / NSTAGE;
        if (r > 0 && !mbar_wait(&empty[s], (r - 1) & 1, a.err, &abort_flag)) break;
        uint8_t* st = smem + s * kAggStageBytes;
        mbar_arrive_expect_tx(&full[s], (nm + 1) * 16384);
        for (int t = 0; t < nm; ++t) tma_load_3d(st + t * 16384, &map_w, &full[s], k * 64, m0 + 128 * t, bh);
        for (int b = 0; b < 2; ++b) tma_load_3d(st + 32768 + b * 8192, &map_h, &full[s], n0 + 64 * b, k * 64, bh);
        last_round[s] = r;
      }
      if (abort_flag)
        for (int s = 0; s < NSTAGE; ++s)
          if (last_round[s] >= 0) mbar_wait(&full[s], last_round[s] & 1, nullptr, nullptr);
    }
    __syncwarp();
  } else if (warp == 1) {
    if (lane == 0) {
      const uint32_t idesc = idesc_bf16_f32(128, 128, 0, 1);
      for (int k = 0; k < nk; ++k) {
        const int s = k % NSTAGE;
        if (!mbar_wait(&full[s], (k / NSTAGE) & 1, a.err, &abort_flag)) break;
        tc_fence_after();
        const uint32_t st = smem_u32(smem + s * kAggStageBytes);
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {
          const uint64_t bd = smem_desc_sw128(st + 32768 + kk * 2048, 8192, 1024);
          for (int t = 0; t < nm; ++t) {
            const uint64_t ad = smem_desc_sw128(st + t * 16384 + kk * 32, 16, 1024);
            umma_bf16_ss(tmem + 128 * t, ad, bd, idesc, (k > 0 || kk > 0) ? 1u : 0u);
          }
        }
        umma_commit(&empty[s]);
      }
      umma_commit(&acc_full);
      umma_commit(&drain);
      mbar_wait(&drain, 0, nullptr, nullptr);
    }
    __syncwarp();
  }

  // Epilogue: warp w holds rows m0 + 128 t + 32 w + lane of M-tile t.
  const bool ok = mbar_wait(&acc_full, 0, a.err, &abort_flag);
  const bool go = __syncthreads_and(ok) && !abort_flag;
  const bool z_tile = n0 >= D * D;
  if (go) {
    tc_fence_after();
    for (int t = 0; t < nm; ++t) {
      const int rloc = warp * 32 + lane;
      const int m = m0 + 128 * t + rloc;
      uint8_t* stg = smem + t * 32768;  // two 16 KB boxes per M-tile; the stages are free now
      for (int c0 = 0; c0 < 128; c0 += 32) {
        __syncwarp();
        uint32_t r[32];
        tmem_ld32(tmem + (static_cast<uint32_t>(warp * 32) << 16) + 128 * t + c0, r);
        tmem_wait_ld();
        if (!z_tile) {
          uint8_t* box = stg + (c0 >> 6) * 16384;
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            uint4 u;
            u.x = pack_bf16x2(__uint_as_float(r[8 * q + 0]), __uint_as_float(r[8 * q + 1]));
            u.y = pack_bf16x2(__uint_as_float(r[8 * q + 2]), __uint_as_float(r[8 * q + 3]));
            u.z = pack_bf16x2(__uint_as_float(r[8 * q + 4]), __uint_as_float(r[8 * q + 5]));
            u.w = pack_bf16x2(__uint_as_float(r[8 * q + 6]), __uint_as_float(r[8 * q + 7]));
            *reinterpret_cast<uint4*>(box + sw128_offset(rloc, ((c0 & 63) >> 3) * 16 + q * 16)) = u;
          }
        } else if (m < a.Nq && c0 < D) {
          float4* dst = reinterpret_cast<float4*>(a.Zagg + (static_cast<size_t>(bh) * a.Nq + m) * D + c0);
#pragma unroll
          for (int q = 0; q < 8; ++q)
            dst[q] = make_float4(__uint_as_float(r[4 * q]), __uint_as_float(r[4 * q + 1]),
                                 __uint_as_float(r[4 * q + 2]), __uint_as_float(r[4 * q + 3]));
        }
      }
    }
    if (!z_tile) fence_proxy_async_smem();
  }
  tc_fence_before();
  __syncthreads();
  if (go && !z_tile && tid == 0) {
    for (int t = 0; t < nm; ++t)
      for (int b = 0; b < 2; ++b) tma_store_3d(&map_out, smem + t * 32768 + b * 16384, n0 + 64 * b, m0 + 128 * t, bh);
    tma_store_commit();
    tma_store_wait_all();
  }
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 256);
  }
}

}  // namespace sla
