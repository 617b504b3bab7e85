// Backward pass of the SLA forward: the elementwise and per-KV-block pieces.
//
//   gs_kernel          G_s = alpha * dO (bf16), the sparse branch's output gradient, an
//                      operand of the dP and dV^T contractions
//   w_transpose_kernel W^T: the 0/1 marginal indicator with KV blocks as rows, the A
//                      operand of dh_j = sum over rows i with j marginal of dH_i (the
//                      aggregation GEMM run backwards)
//   bwd_states_kernel  per KV block j, from its states' gradients dh_j (D x D), dz_j (D):
//                      dV_n += phi(k_n) dh_j and dK_n += (dh_j v_n + dz_j) * phi'(k_n)
//                      over the block's valid tokens n (two tcgen05 MMAs, the results
//                      added into dK and dV)
//
// Source: "SLA: Beyond Sparsity in Diffusion Transformers via Fine-Tunable Sparse-Linear
// Attention", Abstract (one kernel covers the forward and the backward pass); the
// formulas are the exact derivative of the forward with the block labels held fixed:
// h_j = phi(K_j)^T V_j and z_j = colsum phi(K_j), so dV_j = phi(K_j) dh_j and
// dK_j = (V_j dh_j^T + 1 dz_j^T) * phi'(K_j), with phi'(x) = 1 for x > 0, e^x otherwise.
#pragma once

#include "sm100.cuh"

namespace sla {

// grid-stride over [BH, N, D] in 8-element chunks; alpha [H, D].
__global__ void __launch_bounds__(256) gs_kernel(const __nv_bfloat16* __restrict__ dO, const float* __restrict__ alpha,
                                                  __nv_bfloat16* __restrict__ gs, int H, int N, int D, size_t chunks) {
  for (size_t c = blockIdx.x * static_cast<size_t>(blockDim.x) + threadIdx.x; c < chunks;
       c += static_cast<size_t>(gridDim.x) * blockDim.x) {
    const size_t e0 = c * 8;
    const int d0 = static_cast<int>(e0 % D);
    const int h = static_cast<int>((e0 / (static_cast<size_t>(N) * D)) % H);
    const uint4 u = *reinterpret_cast<const uint4*>(dO + e0);
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
    uint32_t o[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float2 f = unpack_bf16x2(w[e]);
      o[e] = pack_bf16x2(f.x * alpha[h * D + d0 + 2 * e], f.y * alpha[h * D + d0 + 2 * e + 1]);
    }
    *reinterpret_cast<uint4*>(gs + e0) = make_uint4(o[0], o[1], o[2], o[3]);
  }
}

// W [BH, Nq, w_ld] -> WT [BH, Nk, wt_ld] (bf16 0/1; columns past Nq zero). grid: (ceil(Nk/32),
// ceil(wt_ld/32), BH), block 32 x 8.
__global__ void __launch_bounds__(256) w_transpose_kernel(const __nv_bfloat16* __restrict__ W, int Nq, int Nk,
                                                          int w_ld, __nv_bfloat16* __restrict__ WT, int wt_ld) {
  __shared__ __nv_bfloat16 tile[32][33];
  const int bh = blockIdx.z, j0 = blockIdx.x * 32, i0 = blockIdx.y * 32;
  const int tx = threadIdx.x, ty = threadIdx.y;
  for (int r = ty; r < 32; r += 8) {
    const int i = i0 + r, j = j0 + tx;
    tile[r][tx] = (i < Nq && j < Nk) ? W[(static_cast<size_t>(bh) * Nq + i) * w_ld + j] : __float2bfloat16_rn(0.f);
  }
  __syncthreads();
  for (int r = ty; r < 32; r += 8) {
    const int j = j0 + r, i = i0 + tx;
    if (j < Nk && i < wt_ld) WT[(static_cast<size_t>(bh) * Nk + j) * wt_ld + i] = tile[tx][r];
  }
}

struct BwdStatesArgs {
  int BH, N, Nk;
  const float* dz;        // [BH, Nk, D] fp32
  float* dK;              // [BH, N, D] fp32 (added into)
  float* dV;              // [BH, N, D] fp32 (added into)
  uint32_t* err;
};

// One CTA per KV block (grid BH * Nk), 192 threads, D = 128:
//   warp 0      TMA: K_j and V_j (64 tokens x 128, two 64-column boxes each) and dh_j
//               (128 x 128 bf16, two boxes of 128 rows x 64 columns)
//   warp 1      TMEM owner, tcgen05 issuer:
//                 acc0 [e][n] = sum_d dh_j[d][e] phi(K_j)[n][d]   (dV_j^T; A MN-major, B K-major)
//                 acc1 [d][n] = sum_e dh_j[d][e] V_j[n][e]         (B K-major, A K-major)
//   warps 2..5  phi(K_j) in place (bf16), then, thread = TMEM lane = channel c:
//                 dV[n][c] += acc0[c][n],  dK[n][c] += (acc1[c][n] + dz_j[c]) phi'(k[n][c])
//               over the valid tokens n, with phi'(k) = min(phi(k), 1) read from the
//               rewritten tile (phi(k) > 1 exactly when k > 0, where phi' = 1).
__global__ void __launch_bounds__(192, 1)
    bwd_states_kernel(const __grid_constant__ CUtensorMap map_k, const __grid_constant__ CUtensorMap map_v,
                      const __grid_constant__ CUtensorMap map_dh, BwdStatesArgs a) {
  constexpr int D = 128;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sK = base;            // 2 boxes of 64 rows x 128 B
  uint8_t* sV = base + 16384;    // 2 boxes of 64 rows x 128 B
  uint8_t* sH = base + 32768;    // dh_j: 2 boxes (e 0..63, e 64..127) of 128 rows (d) x 128 B
  __shared__ uint64_t full, phi_done, acc_full;
  __shared__ uint32_t tmem_base_sh;
  __shared__ int abort_flag;
  __shared__ float sdz[D];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int g = blockIdx.x, bh = g / a.Nk, j = g % a.Nk;
  const int valid = min(64, a.N - j * 64);
  if (tid == 0) {
    mbar_init(&full, 1);
    mbar_init(&phi_done, 128);
    mbar_init(&acc_full, 1);
    abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(&tmem_base_sh, 128);
    tmem_relinquish();
  }
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_base_sh;
  grid_dep_wait();  // dh_j and dz_j come from the previous kernel

  if (warp == 0) {
    if (lane == 0) {
      mbar_arrive_expect_tx(&full, 16384 + 16384 + 32768);
      for (int b = 0; b < 2; ++b) {
        tma_load_3d(sK + b * 8192, &map_k, &full, b * 64, j * 64, bh);
        tma_load_3d(sV + b * 8192, &map_v, &full, b * 64, j * 64, bh);
        tma_load_3d(sH + b * 16384, &map_dh, &full, b * 64, 0, g);
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    bool ok = __all_sync(0xffffffffu, mbar_wait(&phi_done, 0, a.err, &abort_flag));
    if (ok) {
      tc_fence_after();
      const uint32_t id_v = idesc_bf16_f32(128, 64, 1, 0), id_k = idesc_bf16_f32(128, 64, 0, 0);
      const uint32_t k0 = smem_u32(sK), v0 = smem_u32(sV), h0 = smem_u32(sH);
#pragma unroll
      for (int kk = 0; kk < D / 16; ++kk) {
        // acc0: A = dh^T (M = e, K = d: 16 rows of dh per step), B = phi(K) (N = n, K = d)
        const uint64_t ad = smem_desc_sw128(h0 + kk * 2048, 16384, 1024);
        const uint64_t bd = smem_desc_sw128(k0 + (kk >> 2) * 8192 + (kk & 3) * 32, 16, 1024);
        if (elect_one()) umma_bf16_ss(tmem, ad, bd, id_v, kk > 0 ? 1u : 0u);
        __syncwarp();
      }
#pragma unroll
      for (int kk = 0; kk < D / 16; ++kk) {
        // acc1: A = dh (M = d, K = e), B = V (N = n, K = e)
        const uint64_t ad = smem_desc_sw128(h0 + (kk >> 2) * 16384 + (kk & 3) * 32, 16, 1024);
        const uint64_t bd = smem_desc_sw128(v0 + (kk >> 2) * 8192 + (kk & 3) * 32, 16, 1024);
        if (elect_one()) umma_bf16_ss(tmem + 64, ad, bd, id_k, kk > 0 ? 1u : 0u);
        __syncwarp();
      }
    }
    if (elect_one()) umma_commit(&acc_full);
    __syncwarp();
  } else {
    const int wt = tid - 64;  // 0..127
    const int quarter = warp & 3, c = quarter * 32 + lane;
    const uint32_t lane_addr = tmem + (static_cast<uint32_t>(quarter * 32) << 16);
    sdz[wt] = a.dz[static_cast<size_t>(g) * D + wt];
    bool ok = mbar_wait(&full, 0, a.err, &abort_flag);
    // phi(K) in place, 16-byte chunks: thread wt takes chunks wt, wt + 128, ... of the
    // 64 x 128 tile (rows past the sequence end become 0, as in the forward's states)
    if (ok) {
      for (int ch = wt; ch < 64 * 16; ch += 128) {
        const int row = ch >> 4, cc = ch & 15;
        uint4* p = reinterpret_cast<uint4*>(sK + (cc >> 3) * 8192 + sw128_offset(row, (cc & 7) * 16));
        const uint4 u = *p;
        uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float2 x = unpack_bf16x2(w[e]);
          const float f0 = row < valid ? (x.x > 0.f ? x.x + 1.f : __expf(x.x)) : 0.f;
          const float f1 = row < valid ? (x.y > 0.f ? x.y + 1.f : __expf(x.y)) : 0.f;
          w[e] = pack_bf16x2(f0, f1);
        }
        *p = make_uint4(w[0], w[1], w[2], w[3]);
      }
      fence_proxy_async_smem();
    }
    named_barrier(1, 128);  // sdz visible, every phi written
    mbar_arrive(&phi_done);
    ok = ok && mbar_wait(&acc_full, 0, a.err, &abort_flag);
    if (ok) {
      tc_fence_after();
      uint32_t r0[32], r1[32];
      const size_t row0 = static_cast<size_t>(bh) * a.N + static_cast<size_t>(j) * 64;
#pragma unroll 1
      for (int h = 0; h < 2; ++h) {  // token halves 0..31, 32..63
        tmem_ld32(lane_addr + 32 * h, r0);
        tmem_ld32(lane_addr + 64 + 32 * h, r1);
        tmem_wait_ld();
        const float dzc = sdz[c];
#pragma unroll 4
        for (int n2 = 0; n2 < 32; ++n2) {
          const int n = 32 * h + n2;
          if (n < valid) {
            const size_t o = (row0 + n) * D + c;
            a.dV[o] += __uint_as_float(r0[n2]);
            // phi(k) of (n, c) as the MMA saw it; phi' = min(phi, 1)
            const uint16_t fb = *reinterpret_cast<const uint16_t*>(sK + (c >> 6) * 8192 +
                                                                  sw128_offset(n, ((c & 63) >> 3) * 16) + (c & 7) * 2);
            const float fk = __uint_as_float(static_cast<uint32_t>(fb) << 16);
            a.dK[o] += (__uint_as_float(r1[n2]) + dzc) * fminf(fk, 1.f);
          }
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 128);
  }
}

}  // namespace sla
