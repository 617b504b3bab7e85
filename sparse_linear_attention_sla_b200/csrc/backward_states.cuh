// Backward pass of the SLA forward: the elementwise and per-KV-block pieces.
//
//   gs_kernel          G_s = alpha * dO (bf16), the sparse branch's output gradient, an
//                      operand of the dP and dV^T contractions
//   w_transpose_kernel W^T: the 0/1 marginal indicator with KV blocks as rows, the A
//                      operand of dh_j = sum over rows i with j marginal of dH_i (the
//                      aggregation GEMM run backwards)
//   crit_transpose_kernel  per KV block, the query tiles holding it as critical (the
//                      KV-block pass walks them)
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

// The query tiles that hold each KV block as critical, in ascending order: tlist[g, :tcnt[g]]
// for g = bh * Nk + j, from the labels [BH, Nq, Nk] (2 = critical). One thread per (bh, j);
// grid (ceil(Nk / 128), BH), block 128 (the threads of a warp read 32 neighbouring labels).
__global__ void __launch_bounds__(128) crit_transpose_kernel(const int8_t* __restrict__ labels, int Nq, int Nk,
                                                             int32_t* __restrict__ tlist, int32_t* __restrict__ tcnt) {
  const int bh = blockIdx.y, j = blockIdx.x * 128 + threadIdx.x;
  if (j >= Nk) return;
  const int8_t* col = labels + static_cast<size_t>(bh) * Nq * Nk + j;
  int32_t* out = tlist + (static_cast<size_t>(bh) * Nk + j) * Nq;
  int cnt = 0;
  for (int i = 0; i < Nq; ++i)
    if (col[static_cast<size_t>(i) * Nk] == 2) out[cnt++] = i;
  tcnt[static_cast<size_t>(bh) * Nk + j] = cnt;
}

}  // namespace sla
