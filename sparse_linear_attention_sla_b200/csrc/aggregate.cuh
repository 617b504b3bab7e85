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
  int Nq, Nk, LD, BH;
  __nv_bfloat16* Hagg;   // [BH, Nq, D*D]
  float* Zagg;           // [BH, Nq, D]
  uint32_t* err;
  // Nullable. When set, column e of H_i (head h) is written times
  // gamma = (1 - alpha[h, e]) / max(alpha[h, e], kAlphaFloor): the fused attention then adds
  // the linear branch into the sparse branch's accumulator (see attn_kernel). Z_i is unscaled.
  const float* alpha;    // [H, D]
  int H;
};


constexpr int kAggStages = 4;
constexpr uint32_t kAggStageBytes = 3 * 16384;  // A for two M-tiles + one B tile (64 x 128)
constexpr uint32_t kAggStagingBytes = 32768;    // bf16 output of one M-tile: 128 rows x 128 columns

// Persistent, one CTA per SM, 224 threads: warp 0 TMA producer (4-stage ring), warps 1
// and 6 tcgen05 issuers (one per M-tile), warps 2..5 epilogue (TMEM -> bf16 -> one
// shared-memory staging tile per M-tile in turn -> TMA store). A tile is 128 state columns x up to two 128-row M-tiles of query
// blocks of one head (so each stacked-state tile is read once per head); tiles are walked
// columns-fastest. Accumulators are double-buffered in TMEM (2 x 256 columns, M-tile t of
// buffer b at column 256 b + 128 t) so the epilogue of a tile overlaps the next mainloop.
template <int D>
__global__ void __launch_bounds__(224, 1) agg_kernel(const __grid_constant__ CUtensorMap map_w,
                                                     const __grid_constant__ CUtensorMap map_h,
                                                     const __grid_constant__ CUtensorMap map_out, AggArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  __shared__ uint64_t full[kAggStages], empty[kAggStages], acc_full[2], acc_empty[2], drain;
  __shared__ uint32_t tmem_base_sh;
  __shared__ int abort_flag;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int n_nt = a.LD / 128, n_mp = (a.Nq + 255) / 256;
  const int n_tiles = n_nt * n_mp * a.BH;
  const int nk = (a.Nk + 63) / 64;
  if (tid == 0) {
    for (int s = 0; s < kAggStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 2);  // one commit from each issuer
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&acc_full[b], 2);
      mbar_init(&acc_empty[b], 128);
    }
    mbar_init(&drain, 2);
    abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(&tmem_base_sh, 512);
    tmem_relinquish();
  }
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_base_sh;
  grid_dep_launch();
  grid_dep_wait();  // the indicator and the stacked states come from earlier kernels

  auto decode = [&](int t, int& n0, int& m0, int& bh, int& nm) {
    const int nt = t % n_nt, rest = t / n_nt;
    n0 = nt * 128;
    m0 = (rest % n_mp) * 256;
    bh = rest / n_mp;
    nm = (m0 + 128 < a.Nq) ? 2 : 1;
  };

  if (warp == 0) {
    if (lane == 0) {
      prefetch_tmap(&map_w);
      prefetch_tmap(&map_h);
      prefetch_tmap(&map_out);
      int last_round[kAggStages];
      for (int s = 0; s < kAggStages; ++s) last_round[s] = -1;
      uint32_t sc = 0;  // stages filled so far
      bool ok = true;
      for (int t = blockIdx.x; ok && t < n_tiles; t += gridDim.x) {
        int n0, m0, bh, nm;
        decode(t, n0, m0, bh, nm);
        for (int k = 0; k < nk; ++k, ++sc) {
          const int s = sc % kAggStages, r = sc / kAggStages;
          if (r > 0 && !(ok = mbar_wait(&empty[s], (r - 1) & 1, a.err, &abort_flag))) break;
          uint8_t* st = smem + s * kAggStageBytes;
          mbar_arrive_expect_tx(&full[s], (nm + 1) * 16384);
          for (int tt = 0; tt < nm; ++tt) tma_load_3d(st + tt * 16384, &map_w, &full[s], k * 64, m0 + 128 * tt, bh);
          for (int b = 0; b < 2; ++b) tma_load_3d(st + 32768 + b * 8192, &map_h, &full[s], n0 + 64 * b, k * 64, bh);
          last_round[s] = r;
        }
      }
      if (abort_flag)
        for (int s = 0; s < kAggStages; ++s)
          if (last_round[s] >= 0) mbar_wait(&full[s], last_round[s] & 1, nullptr, nullptr);
    }
    __syncwarp();
  } else if (warp == 1 || warp == 6) {
    // Two tcgen05 issuers, one per M-tile: a warp's MMAs run one at a time, so two warps
    // keep two accumulation chains in flight. The whole warp runs the loop; one lane issues.
    const int tt = warp == 1 ? 0 : 1;
    const uint32_t idesc = idesc_bf16_f32(128, 128, 0, 1);
    uint32_t sc = 0;
    int tc = 0;  // tiles issued
    bool ok = true;
    for (int t = blockIdx.x; ok && t < n_tiles; t += gridDim.x, ++tc) {
      int n0, m0, bh, nm;
      decode(t, n0, m0, bh, nm);
      const int ab = tc & 1;
      if (tc >= 2) ok = __all_sync(0xffffffffu, mbar_wait(&acc_empty[ab], ((tc >> 1) - 1) & 1, a.err, &abort_flag));
      for (int k = 0; ok && k < nk; ++k, ++sc) {
        const int s = sc % kAggStages;
        ok = __all_sync(0xffffffffu, mbar_wait(&full[s], (sc / kAggStages) & 1, a.err, &abort_flag));
        if (!ok) break;
        tc_fence_after();
        const uint32_t st = smem_u32(smem + s * kAggStageBytes);
        if (tt < nm) {
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) {
            const uint64_t bd = smem_desc_sw128(st + 32768 + kk * 2048, 8192, 1024);
            const uint64_t ad = smem_desc_sw128(st + tt * 16384 + kk * 32, 16, 1024);
            if (elect_one()) umma_bf16_ss(tmem + ab * 256 + 128 * tt, ad, bd, idesc, (k > 0 || kk > 0) ? 1u : 0u);
          }
        }
        if (elect_one()) umma_commit(&empty[s]);  // both issuers release the stage
        __syncwarp();
      }
      if (!ok) break;
      if (elect_one()) umma_commit(&acc_full[ab]);
      __syncwarp();
    }
    if (elect_one()) umma_commit(&drain);
    mbar_wait(&drain, 0, nullptr, nullptr);
    __syncwarp();
  } else {
    // Epilogue: warp w (quarter w & 3) holds rows m0 + 128 t + 32 (w & 3) + lane of M-tile t.
    const int et = tid - 64;
    const int quarter = warp & 3;
    const int rloc = quarter * 32 + lane;
    const uint32_t lane_addr = tmem + (static_cast<uint32_t>(quarter * 32) << 16);
    uint8_t* stg = smem + kAggStages * kAggStageBytes;
    __shared__ float sGamma[128];  // per-column factor of the current tile (1 when alpha is not given)
    int tc = 0;
    for (int t = blockIdx.x; t < n_tiles; t += gridDim.x, ++tc) {
      int n0, m0, bh, nm;
      decode(t, n0, m0, bh, nm);
      const int ab = tc & 1;
      const bool ok = mbar_wait(&acc_full[ab], (tc >> 1) & 1, a.err, &abort_flag);
      if (!named_barrier_and(1, 128, ok)) break;
      tc_fence_after();
      const bool z_tile = n0 >= D * D;
      if (a.alpha && !z_tile) {  // column c of the tile is channel (n0 + c) % D of h_j's rows
        const float al = a.alpha[(bh % a.H) * D + (n0 + et) % D];
        sGamma[et] = (1.f - al) / fmaxf(al, kAlphaFloor);
      } else {
        sGamma[et] = 1.f;
      }
      named_barrier(1, 128);
      for (int tt = 0; tt < nm; ++tt) {
        if (!z_tile) {  // the staging tile is free once the previous store has read it
          if (et == 0) tma_store_wait_read();
          named_barrier(1, 128);
        }
        const int m = m0 + 128 * tt + rloc;
        uint32_t r[4][32];
#pragma unroll
        for (int q = 0; q < 4; ++q) tmem_ld32(lane_addr + ab * 256 + 128 * tt + 32 * q, r[q]);
        tmem_wait_ld();
        if (!z_tile) {
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            uint8_t* box = stg + (q >> 1) * 16384;
#pragma unroll
            for (int v = 0; v < 4; ++v) {
              const float* g = &sGamma[32 * q + 8 * v];
              *reinterpret_cast<uint4*>(box + sw128_offset(rloc, ((q & 1) * 4 + v) * 16)) = make_uint4(
                  pack_bf16x2(__uint_as_float(r[q][8 * v + 0]) * g[0], __uint_as_float(r[q][8 * v + 1]) * g[1]),
                  pack_bf16x2(__uint_as_float(r[q][8 * v + 2]) * g[2], __uint_as_float(r[q][8 * v + 3]) * g[3]),
                  pack_bf16x2(__uint_as_float(r[q][8 * v + 4]) * g[4], __uint_as_float(r[q][8 * v + 5]) * g[5]),
                  pack_bf16x2(__uint_as_float(r[q][8 * v + 6]) * g[6], __uint_as_float(r[q][8 * v + 7]) * g[7]));
            }
          }
        } else if (m < a.Nq) {
          float4* dst = reinterpret_cast<float4*>(a.Zagg + (static_cast<size_t>(bh) * a.Nq + m) * D);
#pragma unroll
          for (int q = 0; q < D / 32; ++q)
#pragma unroll
            for (int v = 0; v < 8; ++v)
              dst[8 * q + v] = make_float4(__uint_as_float(r[q][4 * v]), __uint_as_float(r[q][4 * v + 1]),
                                           __uint_as_float(r[q][4 * v + 2]), __uint_as_float(r[q][4 * v + 3]));
        }
        if (!z_tile) {
          fence_proxy_async_smem();
          named_barrier(1, 128);
          if (et == 0) {
            for (int b = 0; b < 2; ++b) tma_store_3d(&map_out, stg + b * 16384, n0 + 64 * b, m0 + 128 * tt, bh);
            tma_store_commit();
          }
        }
      }
      tc_fence_before();
      mbar_arrive(&acc_empty[ab]);  // the accumulator has left TMEM
    }
    if (et == 0) tma_store_wait_all();
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

}  // namespace sla
