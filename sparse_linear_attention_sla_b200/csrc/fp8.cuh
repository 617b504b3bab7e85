// Low-bit (FP8 e4m3) pieces of the sparse branch: e4m3 packing, power-of-two block
// scales, the tcgen05 kind::f8f6f4 MMAs, and the K/V block quantiser.
//
// Source: "SLA2: Sparse-Linear Attention with Learnable Routing and QAT", §2.C (the
// sparse branch runs with low-bit operands in the forward pass). The page fixes no format;
// the reading taken here: e4m3 with round-to-nearest-even and saturation at +-448, one
// power-of-two scale 2^e per block with amax / 2^e in (128, 256] (Q per query block, K
// and V per KV block), so scaling is exact and every code is reproducible bit for bit.
#pragma once

#include "sm100.cuh"

namespace sla {

// Two fp32 values to two e4m3 codes, `lo` in bits 0..7 and `hi` in bits 8..15
// (cvt puts its first source operand in the upper byte).
__device__ __forceinline__ uint32_t pack_e4m3x2(float lo, float hi) {
  uint16_t r;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(hi), "f"(lo));
  return r;
}

// Four values to four codes, the first in the lowest byte.
__device__ __forceinline__ uint32_t pack_e4m3x4(float a, float b, float c, float d) {
  return pack_e4m3x2(a, b) | (pack_e4m3x2(c, d) << 16);
}

// Exponent e of the block scale 2^e with amax / 2^e in (128, 256]; 0 when amax is 0.
// With amax = f * 2^x, f in [0.5, 1): ceil(log2 amax) is x - 1 when f = 0.5, else x.
__device__ __forceinline__ int pow2_scale_exp(float amax) {
  if (!(amax > 0.f)) return 0;
  int x;
  const float f = frexpf(amax, &x);
  return (f == 0.5f ? x - 1 : x) - 8;
}

// x * 2^k, exact whenever the result is a normal float; |k| <= 252.
__device__ __forceinline__ float mul_pow2(float x, int k) {
  if (k >= -126 && k <= 127) return x * __int_as_float((127 + k) << 23);
  const int h = k / 2;
  return (x * __int_as_float((127 + h) << 23)) * __int_as_float((127 + k - h) << 23);
}

// |x| of a bf16 as the bit pattern of its magnitude: for non-NaN values the integer order of
// these patterns is the order of the magnitudes.
__device__ __forceinline__ uint32_t bf16x2_absmax_bits(uint32_t w) {
  return max(w & 0x7FFFu, (w >> 16) & 0x7FFFu);
}

// Instruction descriptor for kind::f8f6f4 with e4m3 A and B and fp32 D (A/B format 0).
//   a_mn / b_mn: 1 if that operand is MN-major, 0 if K-major.
__host__ __device__ constexpr uint32_t idesc_e4m3_f32(int M, int N, int a_mn, int b_mn) {
  return (1u << 4)                                  // D format: f32
         | (static_cast<uint32_t>(a_mn) << 15)      // A major
         | (static_cast<uint32_t>(b_mn) << 16)      // B major
         | (static_cast<uint32_t>(N >> 3) << 17)    // N / 8
         | (static_cast<uint32_t>(M >> 4) << 24);   // M / 16
}

// D[tmem] (+)= A[smem] * B[smem]^T, kind::f8f6f4 (K = 32 per instruction), one CTA.
__device__ __forceinline__ void umma_e4m3_ss(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                             uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// D[tmem] (+)= A[tmem] * B[smem]^T, kind::f8f6f4. A (M=128 rows) sits in TMEM lanes
// 0..127 with four codes per 32-bit column (the first in the lowest byte); one K=32
// step reads 8 columns starting at a_tmem.
__device__ __forceinline__ void umma_e4m3_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc, uint32_t idesc,
                                             uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// ---------------------------------------------------------------------- K/V quantiser
//
// One CTA per (KV block j, head bh): the block's valid rows of K and of V (bf16
// [BH, N, D]) are read once, the two block amaxes reduced, and the e4m3 codes written to
// k8 / v8 (uint8 [BH, N, D], same indexing), the scale exponents to kexp / vexp
// ([BH, Nk] int32, scale = 2^exp). HBM-bound: 4 bytes read and 2 written per element.
template <int D>
__global__ void __launch_bounds__(256) quant_kv_kernel(const __nv_bfloat16* __restrict__ k,
                                                       const __nv_bfloat16* __restrict__ v, uint8_t* __restrict__ k8,
                                                       uint8_t* __restrict__ v8, int32_t* __restrict__ kexp,
                                                       int32_t* __restrict__ vexp, int N, int Nk) {
  constexpr int CH = D / 8;          // 16-byte chunks (8 values) per row
  constexpr int PER = 64 * CH / 256; // chunks per thread per tensor
  grid_dep_launch();
  const int j = blockIdx.x, bh = blockIdx.y, tid = threadIdx.x;
  const int rows = min(64, N - j * 64);
  const size_t base = (static_cast<size_t>(bh) * N + static_cast<size_t>(j) * 64) * D;
  const uint4* K4 = reinterpret_cast<const uint4*>(k + base);
  const uint4* V4 = reinterpret_cast<const uint4*>(v + base);
  uint4 kr[PER], vr[PER];
  uint32_t km = 0, vm = 0;
#pragma unroll
  for (int u = 0; u < PER; ++u) {
    const int c = tid + 256 * u;
    if (c / CH < rows) {
      kr[u] = K4[c];
      vr[u] = V4[c];
    } else {
      kr[u] = make_uint4(0, 0, 0, 0);
      vr[u] = make_uint4(0, 0, 0, 0);
    }
    km = max(km, max(max(bf16x2_absmax_bits(kr[u].x), bf16x2_absmax_bits(kr[u].y)),
                     max(bf16x2_absmax_bits(kr[u].z), bf16x2_absmax_bits(kr[u].w))));
    vm = max(vm, max(max(bf16x2_absmax_bits(vr[u].x), bf16x2_absmax_bits(vr[u].y)),
                     max(bf16x2_absmax_bits(vr[u].z), bf16x2_absmax_bits(vr[u].w))));
  }
  km = __reduce_max_sync(0xffffffffu, km);
  vm = __reduce_max_sync(0xffffffffu, vm);
  __shared__ uint32_t red[2][8];
  if ((tid & 31) == 0) {
    red[0][tid >> 5] = km;
    red[1][tid >> 5] = vm;
  }
  __syncthreads();
#pragma unroll
  for (int w = 0; w < 8; ++w) {
    km = max(km, red[0][w]);
    vm = max(vm, red[1][w]);
  }
  const int ek = pow2_scale_exp(__uint_as_float(km << 16));
  const int ev = pow2_scale_exp(__uint_as_float(vm << 16));
  if (tid == 0) {
    kexp[static_cast<size_t>(bh) * Nk + j] = ek;
    vexp[static_cast<size_t>(bh) * Nk + j] = ev;
  }
  uint2* K8 = reinterpret_cast<uint2*>(k8 + base);
  uint2* V8 = reinterpret_cast<uint2*>(v8 + base);
#pragma unroll
  for (int u = 0; u < PER; ++u) {
    const int c = tid + 256 * u;
    if (c / CH >= rows) continue;
    const uint32_t kw[4] = {kr[u].x, kr[u].y, kr[u].z, kr[u].w};
    const uint32_t vw[4] = {vr[u].x, vr[u].y, vr[u].z, vr[u].w};
    uint32_t ko[2], vo[2];
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      ko[h] = pack_e4m3x4(mul_pow2(__uint_as_float(kw[2 * h] << 16), -ek),
                          mul_pow2(__uint_as_float(kw[2 * h] & 0xFFFF0000u), -ek),
                          mul_pow2(__uint_as_float(kw[2 * h + 1] << 16), -ek),
                          mul_pow2(__uint_as_float(kw[2 * h + 1] & 0xFFFF0000u), -ek));
      vo[h] = pack_e4m3x4(mul_pow2(__uint_as_float(vw[2 * h] << 16), -ev),
                          mul_pow2(__uint_as_float(vw[2 * h] & 0xFFFF0000u), -ev),
                          mul_pow2(__uint_as_float(vw[2 * h + 1] << 16), -ev),
                          mul_pow2(__uint_as_float(vw[2 * h + 1] & 0xFFFF0000u), -ev));
    }
    K8[c] = make_uint2(ko[0], ko[1]);
    V8[c] = make_uint2(vo[0], vo[1]);
  }
  // Nothing above reads the previous kernel's results; waiting for it here makes this
  // kernel's completion imply the previous one's, so a dependent launched after this
  // kernel may read both.
  grid_dep_wait();
}

}  // namespace sla
