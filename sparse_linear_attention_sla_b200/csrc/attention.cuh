// Fused SLA attention: each output tile is one query block (128 query rows) of
// one (batch, head):
//
//   sparse branch  O_s = softmax over the keys of the critical KV blocks only
//                        (online softmax, renormalised over that set)
//   linear branch  O_l = phi(Q_i) H_i / (phi(Q_i) Z_i), H_i, Z_i = sums of the
//                        marginal blocks' states (precomputed per row)
//   blend          O   = alpha_h * O_s + (1 - alpha_h) * O_l        (per channel)
//
// Sources: "SLA: Beyond Sparsity in Diffusion Transformers via Fine-Tunable
// Sparse-Linear Attention", Abstract (exact attention for critical weights,
// linear attention for marginal ones, negligible ones skipped, one fused
// kernel); "SLA2: Sparse-Linear Attention with Learnable Routing and QAT" §1
// item 1 (the sparse branch renormalises over its keys) and §2.A
// (O = alpha * O_s + (1 - alpha) * O_l).
//
// Persistent: two CTAs per SM (<= 98 KB shared memory, 256 TMEM columns, <= 168
// registers per thread each) walk the tiles t = blockIdx.x, blockIdx.x + gridDim.x, ...
// in head-major order, so a head's K/V stay in L2 and the next tile's loads overlap the
// current tile's epilogue. Warp roles (192 threads):
//   warp 0      TMA producer: per tile Q, then K_j / V_j of every critical block
//               through a 2-slot ring, then H_i into the next slot (a pseudo-block
//               of the ring: its two halves complete the slot's K and V barriers).
//   warp 1      TMEM owner and tcgen05 issuer (the warp runs the loop, one elected lane
//               issues):
//               S = Q K_j^T (M=128, N=64), O_s += P V_j (M=128, N=D, P read from
//               TMEM), O_l = phi(Q) H_i (M=128, N=D).
//   warps 2..5  softmax / epilogue warpgroup: a thread owns one query row (= TMEM lane)
//               and all 64 columns of each S block; P_n is published before S_{n+1} is
//               waited for.
//
// TMEM columns: S ping-pong [0,64) [64,128) (P, bf16, is written back over the
// first 32 columns of its S), O_s [128,128+D); after a tile's sparse loop O_l
// reuses [0,D) until the epilogue has read it. tcgen05 MMAs issued by one thread
// run in order, so S_{n+2} never overwrites P_n before PV_n has read it.
// An empty critical set gives O_s = 0; an empty marginal set gives Z_i = 0 and O_l = 0.
#pragma once

#include "sm100.cuh"

namespace sla {

struct AttnArgs {
  int H, N, Nq, block_q, n_tiles;
  const int32_t* crit;      // [BH*Nq, crit_ld] critical KV block indices, ascending
  int crit_ld;
  const int32_t* crit_cnt;  // [BH*Nq]
  const float* Zagg;        // [BH*Nq, D]
  const float* alpha;       // [H, D]
  __nv_bfloat16* out;       // [BH, N, D]
  float scale_log2;         // log2(e) / sqrt(D)
  uint32_t* err;
};

__device__ __forceinline__ float fast_exp2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

template <int D>
struct AttnSmem {
  static constexpr uint32_t Q = 128 * D * 2;       // Q tile (rewritten as phi(Q) at the end of a tile)
  static constexpr uint32_t KV = 64 * D * 2;       // one K or one V tile
  static constexpr uint32_t SLOT = 2 * KV;         // one ring slot: K then V (or the H_i tile)
  static constexpr uint32_t HT = D * D * 2;        // H_i tile
  static_assert(HT <= SLOT, "H_i tile must fit in a ring slot");
  static constexpr uint32_t total() { return Q + 2 * SLOT + 1024; }
};

template <int D>
__global__ void __launch_bounds__(192, 2)
    attn_kernel(const __grid_constant__ CUtensorMap map_q, const __grid_constant__ CUtensorMap map_k,
                const __grid_constant__ CUtensorMap map_v, const __grid_constant__ CUtensorMap map_h, AttnArgs a) {
  using L = AttnSmem<D>;
  constexpr int DB = D / 64;  // 64-column boxes per row
  constexpr uint32_t TMEM_COLS = 256;
  constexpr uint32_t OS = 128, OL = 0;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sQ = base;
  uint8_t* sRing = sQ + L::Q;  // slot s at sRing + s * SLOT: K at +0, V at +KV

  __shared__ uint64_t q_full, q_free, phiq_full, ol_done, tmem_free, drain;
  __shared__ uint64_t k_full[2], k_empty[2], v_full[2], v_empty[2];
  __shared__ uint64_t s_full[2], p_full[2], pv_done[2];
  __shared__ uint32_t tmem_base_sh;
  __shared__ int abort_flag;
  __shared__ __align__(16) float sZ[D];
  __shared__ __align__(16) float sAlpha[D];

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

  if (tid == 0) {
    mbar_init(&q_full, 1);
    mbar_init(&q_free, 1);
    mbar_init(&phiq_full, 128);
    mbar_init(&ol_done, 1);
    mbar_init(&tmem_free, 128);
    mbar_init(&drain, 1);
    for (int s = 0; s < 2; ++s) {
      mbar_init(&k_full[s], 1);
      mbar_init(&k_empty[s], 1);
      mbar_init(&v_full[s], 1);
      mbar_init(&v_empty[s], 1);
      mbar_init(&s_full[s], 1);
      mbar_init(&p_full[s], 128);
      mbar_init(&pv_done[s], 1);
    }
    abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(&tmem_base_sh, TMEM_COLS);
    tmem_relinquish();
  }
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_base_sh;
  grid_dep_wait();  // critical lists, H_i and Z_i come from earlier kernels

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      prefetch_tmap(&map_q);
      prefetch_tmap(&map_k);
      prefetch_tmap(&map_v);
      prefetch_tmap(&map_h);
      int k_round[2] = {-1, -1}, v_round[2] = {-1, -1};
      int q_loads = 0;
      uint32_t nb = 0;  // ring uses so far (K/V blocks and H_i pseudo-blocks)
      bool ok = true;
      int k = 0;
      for (int t = blockIdx.x; ok && t < a.n_tiles; t += gridDim.x, ++k) {
        const int bh = t / a.Nq, i = t % a.Nq;
        const int kc = a.crit_cnt[t];
        const int32_t* clist = a.crit + static_cast<size_t>(t) * a.crit_ld;
        if (k > 0 && !(ok = mbar_wait(&q_free, (k - 1) & 1, a.err, &abort_flag))) break;
        mbar_arrive_expect_tx(&q_full, L::Q);
        for (int b = 0; b < DB; ++b) tma_load_3d(sQ + b * 16384, &map_q, &q_full, b * 64, i * a.block_q, bh);
        ++q_loads;
        for (int n = 0; n <= kc; ++n, ++nb) {  // n == kc is the H_i pseudo-block
          const int s = nb & 1, r = nb >> 1;
          uint8_t* slot = sRing + s * L::SLOT;
          // The K half is refilled as soon as S of its previous block is done, the V half
          // once P*V of its previous block is done.
          if (r > 0 && !(ok = mbar_wait(&k_empty[s], (r - 1) & 1, a.err, &abort_flag))) break;
          const int j = n < kc ? clist[n] : 0;
          if (n < kc) {
            mbar_arrive_expect_tx(&k_full[s], L::KV);
            for (int b = 0; b < DB; ++b) tma_load_3d(slot + b * 8192, &map_k, &k_full[s], b * 64, j * 64, bh);
          } else if (D == 128) {  // H_i rows 0..63 land in the K half, rows 64..127 in the V half
            mbar_arrive_expect_tx(&k_full[s], L::KV);
            for (int eh = 0; eh < 2; ++eh) tma_load_2d(slot + eh * 8192, &map_h, &k_full[s], eh * 64, t * D);
          } else {
            mbar_arrive_expect_tx(&k_full[s], L::HT);
            tma_load_2d(slot, &map_h, &k_full[s], 0, t * D);
          }
          k_round[s] = r;
          if (r > 0 && !(ok = mbar_wait(&v_empty[s], (r - 1) & 1, a.err, &abort_flag))) break;
          if (n < kc) {
            mbar_arrive_expect_tx(&v_full[s], L::KV);
            for (int b = 0; b < DB; ++b) tma_load_3d(slot + L::KV + b * 8192, &map_v, &v_full[s], b * 64, j * 64, bh);
          } else if (D == 128) {
            mbar_arrive_expect_tx(&v_full[s], L::KV);
            for (int eh = 0; eh < 2; ++eh)
              tma_load_2d(slot + L::KV + eh * 8192, &map_h, &v_full[s], eh * 64, t * D + 64);
          } else {
            mbar_arrive(&v_full[s]);
          }
          v_round[s] = r;
        }
      }
      if (abort_flag) {  // let every load still in flight land before the CTA retires
        if (q_loads > 0) mbar_wait(&q_full, (q_loads - 1) & 1, nullptr, nullptr);
        for (int s = 0; s < 2; ++s) {
          if (k_round[s] >= 0) mbar_wait(&k_full[s], k_round[s] & 1, nullptr, nullptr);
          if (v_round[s] >= 0) mbar_wait(&v_full[s], v_round[s] & 1, nullptr, nullptr);
        }
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    // The whole warp runs the loop (waits and descriptors are warp-uniform); one elected
    // lane issues each tcgen05 operation.
    const uint32_t id_s = idesc_bf16_f32(128, 64, 0, 0);
    const uint32_t id_o = idesc_bf16_f32(128, D, 0, 1);
    const uint32_t q0 = smem_u32(sQ), ring0 = smem_u32(sRing);
    uint32_t nb = 0, ns = 0;  // ring uses, S/P blocks
    bool ok = true;
    auto wait_all = [&](uint64_t* bar, uint32_t parity) -> bool {
      return __all_sync(0xffffffffu, mbar_wait(bar, parity, a.err, &abort_flag));
    };
    auto commit = [&](uint64_t* bar) {
      if (elect_one()) umma_commit(bar);
      __syncwarp();
    };
    // P*V of the block at ring use nbm, S/P index nsm; `first` overwrites O_s.
    auto issue_pv = [&](uint32_t nbm, uint32_t nsm, bool first) -> bool {
      const int s = nbm & 1, b = nsm & 1;
      if (!wait_all(&p_full[b], (nsm >> 1) & 1)) return false;
      if (!wait_all(&v_full[s], (nbm >> 1) & 1)) return false;
      tc_fence_after();
      const uint32_t vb = ring0 + s * L::SLOT + L::KV;
#pragma unroll
      for (int kk = 0; kk < 4; ++kk) {
        const uint64_t bd = smem_desc_sw128(vb + kk * 2048, 8192, 1024);
        if (elect_one()) umma_bf16_ts(tmem + OS, tmem + b * 64 + kk * 8, bd, id_o, (first && kk == 0) ? 0u : 1u);
        __syncwarp();
      }
      commit(&pv_done[b]);
      commit(&v_empty[s]);
      return true;
    };
    int k = 0;
    for (int t = blockIdx.x; ok && t < a.n_tiles; t += gridDim.x, ++k) {
      const int kc = a.crit_cnt[t];
      if (!(ok = wait_all(&q_full, k & 1))) break;
      // the epilogue of the previous tile has read O_s and O_l out of TMEM
      if (k > 0 && !(ok = wait_all(&tmem_free, (k - 1) & 1))) break;
      for (int n = 0; n < kc; ++n, ++nb, ++ns) {
        const int s = nb & 1, b = ns & 1;
        if (!(ok = wait_all(&k_full[s], (nb >> 1) & 1))) break;
        tc_fence_after();
        const uint32_t kb = ring0 + s * L::SLOT;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint64_t ad = smem_desc_sw128(q0 + (kk >> 2) * 16384 + (kk & 3) * 32, 16, 1024);
          const uint64_t bd = smem_desc_sw128(kb + (kk >> 2) * 8192 + (kk & 3) * 32, 16, 1024);
          if (elect_one()) umma_bf16_ss(tmem + b * 64, ad, bd, id_s, kk > 0 ? 1u : 0u);
          __syncwarp();
        }
        commit(&s_full[b]);
        commit(&k_empty[s]);
        if (n >= 1 && !(ok = issue_pv(nb - 1, ns - 1, n == 1))) break;
      }
      if (!ok) break;
      if (kc > 0 && !(ok = issue_pv(nb - 1, ns - 1, kc == 1))) break;
      // linear branch: O_l = phi(Q) H_i once H_i has landed and the warpgroup rewrote Q as phi(Q)
      const int s = nb & 1;
      if (!(ok = wait_all(&k_full[s], (nb >> 1) & 1))) break;
      if (!(ok = wait_all(&v_full[s], (nb >> 1) & 1))) break;
      if (!(ok = wait_all(&phiq_full, k & 1))) break;
      tc_fence_after();
      const uint32_t hb = ring0 + s * L::SLOT;
#pragma unroll
      for (int kk = 0; kk < D / 16; ++kk) {
        const uint64_t ad = smem_desc_sw128(q0 + (kk >> 2) * 16384 + (kk & 3) * 32, 16, 1024);
        const uint64_t bd = smem_desc_sw128(hb + (kk >> 2) * DB * 8192 + (kk & 3) * 2048, 8192, 1024);
        if (elect_one()) umma_bf16_ss(tmem + OL, ad, bd, id_o, kk > 0 ? 1u : 0u);
        __syncwarp();
      }
      commit(&ol_done);
      commit(&q_free);
      commit(&k_empty[s]);
      commit(&v_empty[s]);
      ++nb;
    }
    commit(&drain);  // every MMA issued above has finished once this arrives
    mbar_wait(&drain, 0, nullptr, nullptr);
  } else {
    // ------------------------------------------------------------ softmax / epilogue warpgroup
    // Thread = query row r = TMEM lane; it owns all 64 columns of every S block. P_n is
    // published as soon as it is stored, so the MMA warp can issue P_n V_n and S_{n+2}
    // while this warpgroup waits for S_{n+1}.
    const int quarter = warp & 3;               // TMEM lane quarter this warp may access
    const int r = quarter * 32 + lane;          // query row within the tile
    const int wt = tid - 64;                    // 0..127
    const uint32_t lane_addr = tmem + (static_cast<uint32_t>(quarter * 32) << 16);
    const float sc = a.scale_log2;
    uint32_t ns = 0;  // S/P blocks so far
    bool ok = true;
    int k = 0;
    // Every barrier of the warpgroup ANDs the threads' status, so a failed wait makes all
    // 128 threads leave together.
    for (int t = blockIdx.x; t < a.n_tiles; t += gridDim.x, ++k) {
      const int bh = t / a.Nq, i = t % a.Nq, h = bh % a.H;
      const int kc = a.crit_cnt[t];
      const int32_t* clist = a.crit + static_cast<size_t>(t) * a.crit_ld;
      if (!named_barrier_and(1, 128, ok)) break;  // the previous tile's epilogue is done with sZ / sAlpha
      for (int c = wt; c < D; c += 128) {
        sZ[c] = a.Zagg[static_cast<size_t>(t) * D + c];
        sAlpha[c] = a.alpha[h * D + c];
      }
      if (!named_barrier_and(1, 128, ok)) break;  // sZ / sAlpha of this tile are visible
      float m_run = -INFINITY, l_run = 0.f;  // running max (scaled, log2 units) and row sum
      uint32_t sa[32], sb[32];               // S columns [0, 32) and [32, 64) of the current block
      int j_cur = kc > 0 ? clist[0] : 0;
      if (kc > 0) {
        ok = ok && __all_sync(0xffffffffu, mbar_wait(&s_full[ns & 1], (ns >> 1) & 1, a.err, &abort_flag));
        if (ok) {
          tc_fence_after();
          tmem_ld32(lane_addr + (ns & 1) * 64, sa);
          tmem_ld32(lane_addr + (ns & 1) * 64 + 32, sb);
          tmem_wait_ld();
        }
      }
      for (int n = 0; ok && n < kc; ++n, ++ns) {
        const int b = ns & 1;
        const int j_next = n + 1 < kc ? clist[n + 1] : 0;
        const int valid = min(64, a.N - j_cur * 64);  // valid key columns of this block
        if (valid < 64) {
#pragma unroll
          for (int c = 0; c < 32; ++c) {
            if (c >= valid) sa[c] = __float_as_uint(-INFINITY);
            if (c + 32 >= valid) sb[c] = __float_as_uint(-INFINITY);
          }
        }
        // row maximum: four independent chains of 3-input maxima
        float m0 = fmax3(__uint_as_float(sa[0]), __uint_as_float(sa[1]), __uint_as_float(sa[2]));
        float m1 = fmax3(__uint_as_float(sa[3]), __uint_as_float(sa[4]), __uint_as_float(sa[5]));
        float m2 = fmax3(__uint_as_float(sb[0]), __uint_as_float(sb[1]), __uint_as_float(sb[2]));
        float m3 = fmax3(__uint_as_float(sb[3]), __uint_as_float(sb[4]), __uint_as_float(sb[5]));
#pragma unroll
        for (int c = 6; c < 30; c += 4) {
          m0 = fmax3(m0, __uint_as_float(sa[c]), __uint_as_float(sa[c + 1]));
          m1 = fmax3(m1, __uint_as_float(sa[c + 2]), __uint_as_float(sa[c + 3]));
          m2 = fmax3(m2, __uint_as_float(sb[c]), __uint_as_float(sb[c + 1]));
          m3 = fmax3(m3, __uint_as_float(sb[c + 2]), __uint_as_float(sb[c + 3]));
        }
        m0 = fmax3(m0, __uint_as_float(sa[30]), __uint_as_float(sa[31]));
        m2 = fmax3(m2, __uint_as_float(sb[30]), __uint_as_float(sb[31]));
        const float mx = fmaxf(fmaxf(m0, m1), fmaxf(m2, m3)) * sc;
        if (n == 0) {
          m_run = mx;
        } else if (__any_sync(0xffffffffu, mx > m_run + 8.f)) {
          // The running maximum grew by more than 2^8: rescale the row of O_s (needs P*V of
          // the previous block finished).
          ok = __all_sync(0xffffffffu, mbar_wait(&pv_done[(ns - 1) & 1], ((ns - 1) >> 1) & 1, a.err, &abort_flag));
          if (!ok) break;
          tc_fence_after();
          const float m_new = fmaxf(m_run, mx);
          const float f = fast_exp2(m_run - m_new);
          const uint64_t f2 = f2_make(f, f);
#pragma unroll 1
          for (int c0 = 0; c0 < D; c0 += 16) {
            uint32_t o[16];
            tmem_ld16(lane_addr + OS + c0, o);
            tmem_wait_ld();
#pragma unroll
            for (int c = 0; c < 16; c += 2) {
              const uint64_t y = f2_mul(static_cast<uint64_t>(o[c]) | (static_cast<uint64_t>(o[c + 1]) << 32), f2);
              o[c] = static_cast<uint32_t>(y);
              o[c + 1] = static_cast<uint32_t>(y >> 32);
            }
            tmem_st16(lane_addr + OS + c0, o);
          }
          tmem_wait_st();
          l_run *= f;
          m_run = m_new;
        }
        // p = 2^(s * scale - m): one paired FMA per two elements and one exponential per
        // element; the even and odd columns are summed in the two lanes of a paired add.
        const uint64_t sc2 = f2_make(sc, sc), nm2 = f2_make(-m_run, -m_run);
        uint64_t ps2 = 0ull, ps2b = 0ull;
        uint32_t pk[32];
#pragma unroll
        for (int c = 0; c < 32; c += 2) {
          const uint64_t x2 = f2_fma(static_cast<uint64_t>(sa[c]) | (static_cast<uint64_t>(sa[c + 1]) << 32), sc2, nm2);
          const uint64_t y2 = f2_fma(static_cast<uint64_t>(sb[c]) | (static_cast<uint64_t>(sb[c + 1]) << 32), sc2, nm2);
          const float e0 = fast_exp2(f2_lo(x2)), e1 = fast_exp2(f2_hi(x2));
          const float e2 = fast_exp2(f2_lo(y2)), e3 = fast_exp2(f2_hi(y2));
          ps2 = f2_add(ps2, f2_make(e0, e1));
          ps2b = f2_add(ps2b, f2_make(e2, e3));
          pk[c >> 1] = pack_bf16x2(e0, e1);
          pk[16 + (c >> 1)] = pack_bf16x2(e2, e3);
        }
        const uint64_t pst = f2_add(ps2, ps2b);
        l_run += f2_lo(pst) + f2_hi(pst);
        tmem_st32(lane_addr + b * 64, pk);  // P over the first 32 columns of its S
        // Publish P_n before waiting for S_{n+1}: P*V of this block, and the S two blocks on
        // (which reuses these columns), can then be issued while S_{n+1} is still in flight.
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(&p_full[b]);
        if (n + 1 < kc) {
          ok = __all_sync(0xffffffffu, mbar_wait(&s_full[b ^ 1], ((ns + 1) >> 1) & 1, a.err, &abort_flag));
          if (ok) {
            tc_fence_after();
            tmem_ld32(lane_addr + (b ^ 1) * 64, sa);
            tmem_ld32(lane_addr + (b ^ 1) * 64 + 32, sb);
            tmem_wait_ld();
          }
        }
        j_cur = j_next;
      }
      // Every MMA that reads Q (or the S/P columns) has finished once the last PV has.
      if (ok && kc > 0)
        ok = __all_sync(0xffffffffu, mbar_wait(&pv_done[(ns - 1) & 1], ((ns - 1) >> 1) & 1, a.err, &abort_flag));
      if (ok) ok = __all_sync(0xffffffffu, mbar_wait(&q_full, k & 1, a.err, &abort_flag));

      // phi(Q) in place (bf16) over the row, and the linear-branch denominator phi(q) . Z_i
      // with the same rounded phi(q) the MMA sees. Column pairs in paired arithmetic:
      // phi(x) = x + 1 for x > 0, else e^x = 2^(x log2 e); even and odd columns' products
      // with Z_i are summed in the two lanes.
      uint64_t den2 = 0ull;
      if (ok) {
        const uint64_t one2 = f2_make(1.f, 1.f), log2e2 = f2_make(1.4426950408889634f, 1.4426950408889634f);
#pragma unroll 2
        for (int c8 = 0; c8 < D / 8; ++c8) {
          uint4* p = reinterpret_cast<uint4*>(sQ + (c8 >> 3) * 16384 + sw128_offset(r, (c8 & 7) * 16));
          uint4 u = *p;
          uint32_t w[4] = {u.x, u.y, u.z, u.w};
          const uint4 z01 = *reinterpret_cast<const uint4*>(&sZ[c8 * 8]);
          const uint4 z23 = *reinterpret_cast<const uint4*>(&sZ[c8 * 8 + 4]);
          const uint64_t z2[4] = {static_cast<uint64_t>(z01.x) | (static_cast<uint64_t>(z01.y) << 32),
                                  static_cast<uint64_t>(z01.z) | (static_cast<uint64_t>(z01.w) << 32),
                                  static_cast<uint64_t>(z23.x) | (static_cast<uint64_t>(z23.y) << 32),
                                  static_cast<uint64_t>(z23.z) | (static_cast<uint64_t>(z23.w) << 32)};
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            // bf16 -> fp32 is a shift into the high half-word
            const uint64_t x2 = static_cast<uint64_t>(w[e] << 16) | (static_cast<uint64_t>(w[e] & 0xFFFF0000u) << 32);
            const uint64_t pos2 = f2_add(x2, one2);
            const uint64_t t2 = f2_mul(x2, log2e2);
            const float g0 = f2_lo(x2) > 0.f ? f2_lo(pos2) : fast_exp2(f2_lo(t2));
            const float g1 = f2_hi(x2) > 0.f ? f2_hi(pos2) : fast_exp2(f2_hi(t2));
            w[e] = pack_bf16x2(g0, g1);
            const uint64_t gr2 = static_cast<uint64_t>(w[e] << 16) | (static_cast<uint64_t>(w[e] & 0xFFFF0000u) << 32);
            den2 = f2_fma(gr2, z2[e], den2);
          }
          *p = make_uint4(w[0], w[1], w[2], w[3]);
        }
        fence_proxy_async_smem();
      }
      const float den_tot = f2_lo(den2) + f2_hi(den2);
      tc_fence_before();
      mbar_arrive(&phiq_full);
      if (ok) ok = __all_sync(0xffffffffu, mbar_wait(&ol_done, k & 1, a.err, &abort_flag));
      if (!(ok = named_barrier_and(1, 128, ok))) break;

      // Epilogue: O = alpha * O_s / l + (1 - alpha) * O_l / den, bf16, straight to global memory.
      tc_fence_after();
      const float inv_l = l_run > 0.f ? 1.f / l_run : 0.f;
      const float inv_d = den_tot > 0.f ? 1.f / den_tot : 0.f;
      const int tok = i * a.block_q + r;
      const bool store = r < a.block_q && tok < a.N;
      __nv_bfloat16* orow = a.out + (static_cast<size_t>(bh) * a.N + tok) * D;
      // per column pair: y = (alpha inv_l) O_s + ((1 - alpha) inv_d) O_l in paired arithmetic;
      // O_s is not read when the critical set is empty (its TMEM columns were never written)
      const uint64_t il2 = f2_make(inv_l, inv_l), id2 = f2_make(inv_d, inv_d);
#pragma unroll 1
      for (int c0 = 0; c0 < D; c0 += 16) {
        uint32_t os[16], ol[16];
        if (kc > 0) tmem_ld16(lane_addr + OS + c0, os);
        tmem_ld16(lane_addr + OL + c0, ol);
        tmem_wait_ld();
        uint32_t pk[8];
#pragma unroll
        for (int c = 0; c < 16; c += 2) {
          const uint64_t al2 = *reinterpret_cast<const uint64_t*>(&sAlpha[c0 + c]);
          const uint64_t wl = f2_fma(al2 ^ 0x8000000080000000ull, id2, id2);  // (1 - alpha) inv_d
          uint64_t y = f2_mul(wl, static_cast<uint64_t>(ol[c]) | (static_cast<uint64_t>(ol[c + 1]) << 32));
          if (kc > 0)
            y = f2_fma(f2_mul(al2, il2), static_cast<uint64_t>(os[c]) | (static_cast<uint64_t>(os[c + 1]) << 32), y);
          pk[c >> 1] = pack_bf16x2(f2_lo(y), f2_hi(y));
        }
        if (store) {
          uint4* dst = reinterpret_cast<uint4*>(orow + c0);
          dst[0] = make_uint4(pk[0], pk[1], pk[2], pk[3]);
          dst[1] = make_uint4(pk[4], pk[5], pk[6], pk[7]);
        }
      }
      tc_fence_before();
      mbar_arrive(&tmem_free);  // O_s and O_l have left TMEM: the next tile may overwrite them
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, TMEM_COLS);
  }
}

}  // namespace sla
