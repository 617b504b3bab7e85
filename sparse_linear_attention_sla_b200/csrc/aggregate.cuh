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

// grid: (ceil(LD/256), ceil(Nq/128), BH); block 128 (warp 0: TMA, warp 1: MMA, all: epilogue).
// Dynamic smem: 2 stages x (A 16 KB + B 32 KB) + 1 KB alignment. TMEM: 256 columns.
template <int D>
__global__ void __launch_bounds__(128) agg_kernel(const __grid_constant__ CUtensorMap map_w,
                                                  const __grid_constant__ CUtensorMap map_h, AggArgs a) {
  constexpr int NSTAGE = 2;
  constexpr uint32_t ABYTES = 16384, BBYTES = 32768;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  __shared__ uint64_t full[NSTAGE], empty[NSTAGE], acc_full, drain;
  __shared__ uint32_t tmem_base_sh;
  __shared__ int abort_flag;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int n0 = blockIdx.x * 256, m0 = blockIdx.y * 128, bh = blockIdx.z;
  const int ncols = min(256, a.LD - n0);
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
      int last_round[NSTAGE] = {-1, -1};
      for (int k = 0; k < nk; ++k) {
        const int s = k % NSTAGE, r = k / NSTAGE;
        if (r > 0 && !mbar_wait(&empty[s], (r - 1) & 1, a.err, &abort_flag)) break;
        mbar_arrive_expect_tx(&full[s], ABYTES + (ncols / 64) * 8192);
        uint8_t* sa = smem + s * (ABYTES + BBYTES);
        tma_load_3d(sa, &map_w, &full[s], k * 64, m0, bh);
        for (int b = 0; b < ncols / 64; ++b)
          tma_load_3d(sa + ABYTES + b * 8192, &map_h, &full[s], n0 + 64 * b, k * 64, bh);
        last_round[s] = r;
      }
      if (abort_flag)
        for (int s = 0; s < NSTAGE; ++s)
          if (last_round[s] >= 0) mbar_wait(&full[s], last_round[s] & 1, nullptr, nullptr);
    }
    __syncwarp();
  } else if (warp == 1) {
    if (lane == 0) {
      const uint32_t idesc = idesc_bf16_f32(128, ncols, 0, 1);
      for (int k = 0; k < nk; ++k) {
        const int s = k % NSTAGE;
        if (!mbar_wait(&full[s], (k / NSTAGE) & 1, a.err, &abort_flag)) break;
        tc_fence_after();
        const uint32_t sa = smem_u32(smem + s * (ABYTES + BBYTES));
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {
          const uint64_t ad = smem_desc_sw128(sa + kk * 32, 16, 1024);
          const uint64_t bd = smem_desc_sw128(sa + ABYTES + kk * 2048, 8192, 1024);
          umma_bf16_ss(tmem, ad, bd, idesc, (k > 0 || kk > 0) ? 1u : 0u);
        }
        umma_commit(&empty[s]);
      }
      umma_commit(&acc_full);
      umma_commit(&drain);
      mbar_wait(&drain, 0, nullptr, nullptr);
    }
    __syncwarp();
  }

  // Epilogue: all four warps; warp w holds rows m0 + 32 w + lane.
  const bool ok = mbar_wait(&acc_full, 0, a.err, &abort_flag);
  if (__all_sync(0xffffffffu, ok) && !abort_flag) {
    tc_fence_after();
    const int m = m0 + warp * 32 + lane;
    for (int c0 = 0; c0 < ncols; c0 += 32) {
      __syncwarp();
      uint32_t r[32];
      tmem_ld32(tmem + (static_cast<uint32_t>(warp * 32) << 16) + c0, r);
      tmem_wait_ld();
      const int col = n0 + c0;
      if (m >= a.Nq) {
        // row past the last query block: nothing to store
      } else if (col < D * D) {
        uint4* dst = reinterpret_cast<uint4*>(a.Hagg + (static_cast<size_t>(bh) * a.Nq + m) * (D * D) + col);
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          uint4 u;
          u.x = pack_bf16x2(__uint_as_float(r[8 * q + 0]), __uint_as_float(r[8 * q + 1]));
          u.y = pack_bf16x2(__uint_as_float(r[8 * q + 2]), __uint_as_float(r[8 * q + 3]));
          u.z = pack_bf16x2(__uint_as_float(r[8 * q + 4]), __uint_as_float(r[8 * q + 5]));
          u.w = pack_bf16x2(__uint_as_float(r[8 * q + 6]), __uint_as_float(r[8 * q + 7]));
          dst[q] = u;
        }
      } else if (col - D * D < D) {
        float4* dst = reinterpret_cast<float4*>(a.Zagg + (static_cast<size_t>(bh) * a.Nq + m) * D + (col - D * D));
#pragma unroll
        for (int q = 0; q < 8; ++q)
          dst[q] = make_float4(__uint_as_float(r[4 * q]), __uint_as_float(r[4 * q + 1]),
                               __uint_as_float(r[4 * q + 2]), __uint_as_float(r[4 * q + 3]));
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 256);
  }
}

}  // namespace sla
