// Router variant: the second-order block score of "SPLA - Atención de Bloque Dispersa más
// Lineal para el Modelado de Contexto Largo", §2.1. A KV block's relevance to a query is the
// expected exponential attention of its tokens expanded to second order around the block
// mean, exp(q . kbar) (1 + 1/2 q^T Cov(k) q), with the covariance kept diagonal. For SLA's
// query blocks (pooled query qbar_i, 1/sqrt(D) in both terms) the log of that score is
//
//   S2_ij = qbar_i . kbar_j / sqrt(D) + log1p(sum_d qbar_i,d^2 var_j,d / (2 D)),
//
// var_j,d the population variance of channel d over the block's valid keys. Blocks are
// ranked by S2 with the same total order and counts as the first-order router (the fp64
// selection, select_kernel).
//   block_var_kernel : kbar_j and var_j per KV block, fp64 (exact sums of bf16 values and
//                      of their squares, then the mean and E[k^2] - mean^2)
//   score2_kernel    : S2 in fp64
#pragma once

#include "prep.cuh"

namespace sla {

// grid: (Nk, BH); block: 128 threads. k: [BH, N, D] bf16; kbar, var: [BH, Nk, D] fp64.
template <int D>
__global__ void __launch_bounds__(128) block_var_kernel(const __nv_bfloat16* __restrict__ k, double* __restrict__ kbar,
                                                        double* __restrict__ var, int N) {
  constexpr int VEC = 8, VPR = D / VEC, RSTEP = 128 / VPR;
  __shared__ double part[2][RSTEP][D];
  const int j = blockIdx.x, bh = blockIdx.y, t = threadIdx.x, Nk = gridDim.x;
  const int r0 = j * 64, r1 = min(N, r0 + 64);
  const int vec = t % VPR, rr = t / VPR;
  double s1[VEC], s2[VEC];
#pragma unroll
  for (int e = 0; e < VEC; ++e) s1[e] = s2[e] = 0.0;
  const __nv_bfloat16* base = k + static_cast<size_t>(bh) * N * D + vec * VEC;
  for (int r = r0 + rr; r < r1; r += RSTEP) {
    const uint4 u = *reinterpret_cast<const uint4*>(base + static_cast<size_t>(r) * D);
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float2 f = unpack_bf16x2(w[e]);
      const double x0 = f.x, x1 = f.y;  // exact; their squares are exact in fp64 too
      s1[2 * e] += x0;
      s1[2 * e + 1] += x1;
      s2[2 * e] += x0 * x0;
      s2[2 * e + 1] += x1 * x1;
    }
  }
#pragma unroll
  for (int e = 0; e < VEC; ++e) {
    part[0][rr][vec * VEC + e] = s1[e];
    part[1][rr][vec * VEC + e] = s2[e];
  }
  __syncthreads();
  if (t < D) {
    double a = 0.0, b = 0.0;
#pragma unroll
    for (int g = 0; g < RSTEP; ++g) {
      a += part[0][g][t];
      b += part[1][g][t];
    }
    const double n = static_cast<double>(r1 - r0);
    const double mean = a / n;
    const size_t o = (static_cast<size_t>(bh) * Nk + j) * D + t;
    kbar[o] = mean;
    var[o] = fmax(b / n - mean * mean, 0.0);
  }
}

// grid: (ceil(Nk/32), ceil(Nq/32), BH); block: 256 threads, each 4 scores of a 32 x 32 tile.
// qbar [BH, Nq, D], kbar / var [BH, Nk, D] fp64; S2 [BH, Nq, Nk] fp64.
template <int D>
__global__ void __launch_bounds__(256) score2_kernel(const double* __restrict__ qbar, const double* __restrict__ kbar,
                                                     const double* __restrict__ var, double* __restrict__ S2, int Nq,
                                                     int Nk) {
  constexpr int T = 32, DC = 32;
  __shared__ double sq[T][DC + 1], sk[T][DC + 1], sv[T][DC + 1];
  const int bh = blockIdx.z, i0 = blockIdx.y * T, j0 = blockIdx.x * T, tid = threadIdx.x;
  const int ti = tid >> 3, tj = (tid & 7) * 4;  // row ti, columns tj .. tj + 3 of the tile
  const double* qb = qbar + static_cast<size_t>(bh) * Nq * D;
  const double* kb = kbar + static_cast<size_t>(bh) * Nk * D;
  const double* vb = var + static_cast<size_t>(bh) * Nk * D;
  double first[4] = {0, 0, 0, 0}, quad[4] = {0, 0, 0, 0};
  for (int d0 = 0; d0 < D; d0 += DC) {
    for (int e = tid; e < T * DC; e += 256) {
      const int r = e / DC, c = e % DC;
      sq[r][c] = i0 + r < Nq ? qb[static_cast<size_t>(i0 + r) * D + d0 + c] : 0.0;
      sk[r][c] = j0 + r < Nk ? kb[static_cast<size_t>(j0 + r) * D + d0 + c] : 0.0;
      sv[r][c] = j0 + r < Nk ? vb[static_cast<size_t>(j0 + r) * D + d0 + c] : 0.0;
    }
    __syncthreads();
#pragma unroll 8
    for (int c = 0; c < DC; ++c) {
      const double qv = sq[ti][c];
      const double q2 = qv * qv;
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        first[u] = fma(qv, sk[tj + u][c], first[u]);
        quad[u] = fma(q2, sv[tj + u][c], quad[u]);
      }
    }
    __syncthreads();
  }
  const int i = i0 + ti;
  if (i >= Nq) return;
  const double inv_sqrt_d = 1.0 / sqrt(static_cast<double>(D)), inv_2d = 0.5 / static_cast<double>(D);
#pragma unroll
  for (int u = 0; u < 4; ++u) {
    const int j = j0 + tj + u;
    if (j < Nk) S2[(static_cast<size_t>(bh) * Nq + i) * Nk + j] = first[u] * inv_sqrt_d + log1p(quad[u] * inv_2d);
  }
}

}  // namespace sla
