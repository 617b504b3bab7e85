// Fused SLA attention: each output tile is one query block (128 query rows) of
// one (batch, head):
//
//   sparse branch  O_s = softmax over the keys of the critical KV blocks only
//                        (online softmax, renormalised over that set)
//   linear branch  O_l = phi(Q_i) H_i / (phi(Q_i) Z_i), H_i, Z_i = sums of the
//                        marginal blocks' states (aggregated per query block)
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
//               through a 2-slot ring, then H~_i into the next slot (a pseudo-block
//               of the ring: its two halves complete the slot's K and V barriers). The
//               next tile's Q is loaded once the tile's last S MMA is done and every row
//               of the warpgroup has read its Q for phi(q).
//   warp 1      TMEM owner and tcgen05 issuer (the warp runs the loop, one elected lane
//               issues):
//               S = Q K_j^T (M=128, N=64), acc += P V_j (M=128, N=D, P read from
//               TMEM), and after the last block acc += P_lin H~_i (P_lin from TMEM).
//   warps 2..5  softmax / epilogue warpgroup: a thread owns one query row (= TMEM lane)
//               and all 64 columns of each S block; P_n is published before S_{n+1} is
//               waited for.
//
// The linear branch shares the sparse branch's accumulator. With l the softmax
// normaliser, den = phi(q) . Z_i and H~_i = H_i diag((1 - alpha) / alpha) (the aggregation
// writes H_i scaled so), the blend is
//     O = alpha acc / l + (1 - alpha) phi(q) H_i / den = alpha (acc + (l / den) phi(q) H~_i) / l,
// so the warpgroup writes P_lin = (l / den) phi(q) into TMEM and the epilogue reads one
// accumulator (alpha is floored at 2^-24 on both sides).
//
// TMEM columns: S ping-pong [0,64) [64,128) (P, bf16, is written back over the
// first 32 columns of its S), acc [128,128+D); after a tile's sparse loop P_lin takes the
// S columns the next block would have used. tcgen05 MMAs issued by one thread run in
// order, so S_{n+2} never overwrites P_n before PV_n has read it, and the next tile's S
// never overwrites P_lin before the linear MMA has read it. The next tile's first write
// of acc waits for this tile's epilogue.
// An empty critical set gives O_s = 0 (l taken as 1); an empty marginal set gives Z_i = 0
// and no linear term.
//
// PISA (template flag; "PISA - Atención Dispersa por Tramos para Transformers de Difusión
// Eficientes" §2): no alpha and no linear branch. Every block that is not critical enters
// the softmax through its centroid: after the critical blocks the tile runs ceil(Nk / 64)
// pseudo-blocks whose keys are the block means kbar_j and whose values are the block sums
// Vsum_j, the centroid of a critical block (and of a block past Nk) masked out. With
// p_j = 2^(q . kbar_j log2(e) / sqrt(D) - m) the pseudo-block adds p_j Vsum_j to the
// accumulator (the MMA), n_j p_j to the normaliser and p_j to A = sum_j p_j; the tail writes
// P_lin = (A / sqrt(D)) q and H~ = Hbar, the mean first-order matrix of the head, so that
// O = (acc + (q / sqrt(D)) Hbar A) / l.
#pragma once

#include "softmax_block.cuh"

namespace sla {

struct AttnArgs {
  int H, N, Nq, block_q, n_tiles;
  int Nk, nc, n_last;       // PISA: KV blocks, centroid pseudo-blocks (ceil(Nk / 64)), keys of the last block
  int h_mode;               // the H~ tile of tile t: 0 row t * D (per query block), 1 row bh * D (per head), 2 row 0 (one tile)
  float inv_sqrt_d;         // PISA: 1 / sqrt(D)
  const int32_t* crit;      // [BH*Nq, crit_ld] critical KV block indices, ascending
  int crit_ld;
  const int32_t* crit_cnt;  // [BH*Nq]
  const float* Zagg;        // [BH*Nq, D] (nullable: Z_i = 0, no linear term)
  const float* alpha;       // [H, D]
  __nv_bfloat16* out;       // [BH, N, D]
  float scale_log2;         // log2(e) / sqrt(D)
  uint32_t* err;
};

template <int D>
struct AttnSmem {
  static constexpr uint32_t Q = 128 * D * 2;       // Q tile (rewritten as phi(Q) at the end of a tile)
  static constexpr uint32_t KV = 64 * D * 2;       // one K or one V tile
  static constexpr uint32_t SLOT = 2 * KV;         // one ring slot: K then V (or the H_i tile)
  static constexpr uint32_t HT = D * D * 2;        // H_i tile
  static_assert(HT <= SLOT, "H_i tile must fit in a ring slot");
  static constexpr uint32_t total() { return Q + 2 * SLOT + 1024; }
};

// FM: feature map of the linear branch, 0 elu + 1, 1 e^x. PISA: the piecewise variant (see
// the end of the header comment); map_kc / map_vc are read only then.
template <int D, int FM = 0, bool PISA = false>
__global__ void __launch_bounds__(192, 2)
    attn_kernel(const __grid_constant__ CUtensorMap map_q, const __grid_constant__ CUtensorMap map_k,
                const __grid_constant__ CUtensorMap map_v, const __grid_constant__ CUtensorMap map_h,
                const __grid_constant__ CUtensorMap map_o, const __grid_constant__ CUtensorMap map_kc,
                const __grid_constant__ CUtensorMap map_vc, AttnArgs a) {
  using L = AttnSmem<D>;
  constexpr int DB = D / 64;  // 64-column boxes per row
  constexpr uint32_t TMEM_COLS = 256;
  constexpr uint32_t OS = 128;  // the accumulator's first TMEM column
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sQ = base;
  uint8_t* sRing = sQ + L::Q;  // slot s at sRing + s * SLOT: K at +0, V at +KV

  __shared__ uint64_t q_full, q_free, plin_full, lin_done, tmem_free, drain;
  __shared__ uint64_t k_full[2], k_empty[2], v_full[2], v_empty[2];
  __shared__ uint64_t s_full[2], p_full[2], pv_done[2];
  __shared__ uint32_t tmem_base_sh;
  __shared__ int abort_flag;
  __shared__ __align__(16) float sZ[D];      // Z_i of the current tile
  __shared__ __align__(16) float sAlpha[D];  // max(alpha, 2^-24) of the current tile's head

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

  if (tid == 0) {
    mbar_init(&q_full, 1);
    mbar_init(&q_free, 1 + 128);  // the tile's last S MMA, and every row read for phi(q)
    mbar_init(&plin_full, 128);
    mbar_init(&lin_done, 1);
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
      if constexpr (PISA) {
        prefetch_tmap(&map_kc);
        prefetch_tmap(&map_vc);
      }
      int k_round[2] = {-1, -1}, v_round[2] = {-1, -1};
      int q_loads = 0;
      uint32_t nb = 0;  // ring uses so far (K/V blocks and H_i pseudo-blocks)
      bool ok = true;
      int k = 0;
      for (int t = blockIdx.x; ok && t < a.n_tiles; t += gridDim.x, ++k) {
        const int bh = t / a.Nq, i = t % a.Nq;
        const int kc = a.crit_cnt[t];
        const int nblk = kc + (PISA ? a.nc : 0);  // blocks of the softmax: critical, then centroid
        const int32_t* clist = a.crit + static_cast<size_t>(t) * a.crit_ld;
        const int h_row = (a.h_mode == 0 ? t : (a.h_mode == 1 ? bh : 0)) * D;  // first row of this tile's H~
        if (k > 0 && !(ok = mbar_wait(&q_free, (k - 1) & 1, a.err, &abort_flag))) break;
        mbar_arrive_expect_tx(&q_full, L::Q);
        for (int b = 0; b < DB; ++b) tma_load_3d(sQ + b * 16384, &map_q, &q_full, b * 64, i * a.block_q, bh);
        ++q_loads;
        for (int n = 0; n <= nblk; ++n, ++nb) {  // n == nblk is the H~ pseudo-block
          const int s = nb & 1, r = nb >> 1;
          uint8_t* slot = sRing + s * L::SLOT;
          // The K half is refilled as soon as S of its previous block is done, the V half
          // once P*V of its previous block is done.
          if (r > 0 && !(ok = mbar_wait(&k_empty[s], (r - 1) & 1, a.err, &abort_flag))) break;
          const int j = n < kc ? clist[n] : n - kc;  // KV block, or centroid pseudo-block
          const CUtensorMap* mk = n < kc ? &map_k : &map_kc;
          const CUtensorMap* mv = n < kc ? &map_v : &map_vc;
          if (n < nblk) {
            mbar_arrive_expect_tx(&k_full[s], L::KV);
            for (int b = 0; b < DB; ++b) tma_load_3d(slot + b * 8192, mk, &k_full[s], b * 64, j * 64, bh);
          } else if (D == 128) {  // H~ rows 0..63 land in the K half, rows 64..127 in the V half
            mbar_arrive_expect_tx(&k_full[s], L::KV);
            for (int eh = 0; eh < 2; ++eh) tma_load_2d(slot + eh * 8192, &map_h, &k_full[s], eh * 64, h_row);
          } else {
            mbar_arrive_expect_tx(&k_full[s], L::HT);
            tma_load_2d(slot, &map_h, &k_full[s], 0, h_row);
          }
          k_round[s] = r;
          if (r > 0 && !(ok = mbar_wait(&v_empty[s], (r - 1) & 1, a.err, &abort_flag))) break;
          if (n < nblk) {
            mbar_arrive_expect_tx(&v_full[s], L::KV);
            for (int b = 0; b < DB; ++b) tma_load_3d(slot + L::KV + b * 8192, mv, &v_full[s], b * 64, j * 64, bh);
          } else if (D == 128) {
            mbar_arrive_expect_tx(&v_full[s], L::KV);
            for (int eh = 0; eh < 2; ++eh)
              tma_load_2d(slot + L::KV + eh * 8192, &map_h, &v_full[s], eh * 64, h_row + 64);
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
    // P*V of the block at ring use nbm, S/P index nsm; `first` overwrites O_s, which the
    // previous tile's epilogue must have read (tile k > 0).
    int k = 0;
    auto issue_pv = [&](uint32_t nbm, uint32_t nsm, bool first) -> bool {
      const int s = nbm & 1, b = nsm & 1;
      if (first && k > 0 && !wait_all(&tmem_free, (k - 1) & 1)) return false;
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
    for (int t = blockIdx.x; ok && t < a.n_tiles; t += gridDim.x, ++k) {
      const int kc = a.crit_cnt[t] + (PISA ? a.nc : 0);  // blocks of the softmax
      if (!(ok = wait_all(&q_full, k & 1))) break;
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
        if (n + 1 == kc) commit(&q_free);  // no MMA of this tile reads Q after its last S
        if (n >= 1 && !(ok = issue_pv(nb - 1, ns - 1, n == 1))) break;
      }
      if (!ok) break;
      if (kc == 0) commit(&q_free);
      if (kc > 0 && !(ok = issue_pv(nb - 1, ns - 1, kc == 1))) break;
      // Linear branch, added into the sparse accumulator: O_s += P_lin H~_i with
      // P_lin = (l / den) phi(Q) written by the warpgroup into the S columns after the last
      // block (ns & 1) and H~_i (H_i with its columns scaled by (1 - alpha) / alpha) in the
      // next ring slot. With no critical block this is the first write of O_s.
      const int s = nb & 1;
      if (kc == 0 && k > 0 && !(ok = wait_all(&tmem_free, (k - 1) & 1))) break;
      if (!(ok = wait_all(&k_full[s], (nb >> 1) & 1))) break;
      if (!(ok = wait_all(&v_full[s], (nb >> 1) & 1))) break;
      if (!(ok = wait_all(&plin_full, k & 1))) break;
      tc_fence_after();
      const uint32_t hb = ring0 + s * L::SLOT;
      const uint32_t pl = tmem + (ns & 1) * 64;
#pragma unroll
      for (int kk = 0; kk < D / 16; ++kk) {
        const uint64_t bd = smem_desc_sw128(hb + (kk >> 2) * DB * 8192 + (kk & 3) * 2048, 8192, 1024);
        if (elect_one()) umma_bf16_ts(tmem + OS, pl + kk * 8, bd, id_o, (kc > 0 || kk > 0) ? 1u : 0u);
        __syncwarp();
      }
      commit(&lin_done);  // the H~_i slot is released by the warpgroup once the output staged there is stored
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
    uint32_t ns = 0;   // S/P blocks so far
    uint32_t nbw = 0;  // ring uses so far (K/V blocks and H~_i pseudo-blocks)
    int release_slot = -1;  // (thread 0 of the warpgroup) ring slot still held by an output store
    bool ok = true;
    int k = 0;
    // This thread's entries of Z_i and alpha for the tile after the current one, loaded
    // during the current tile so that their latency stays off the tile boundary.
    float z_next = 0.f, a_next = 1.f;
    if (!PISA && wt < D && static_cast<int>(blockIdx.x) < a.n_tiles) {
      if (a.Zagg) z_next = a.Zagg[static_cast<size_t>(blockIdx.x) * D + wt];
      a_next = a.alpha[(blockIdx.x / a.Nq % a.H) * D + wt];
    }
    // Every barrier of the warpgroup ANDs the threads' status, so a failed wait makes all
    // 128 threads leave together.
    for (int t = blockIdx.x; t < a.n_tiles; t += gridDim.x, ++k) {
      const int bh = t / a.Nq, i = t % a.Nq;
      const int kc = a.crit_cnt[t];
      const int nblk = kc + (PISA ? a.nc : 0);  // blocks of the softmax: critical, then centroid
      const int32_t* clist = a.crit + static_cast<size_t>(t) * a.crit_ld;
      const uint32_t hs = (nbw + nblk) & 1;  // ring slot of this tile's H~, reused to stage O
      nbw += nblk + 1;
      if (!named_barrier_and(1, 128, ok)) break;  // the previous tile's epilogue is done with sZ / sAlpha
      if (wt < D) {
        sZ[wt] = z_next;
        sAlpha[wt] = fmaxf(a_next, kAlphaFloor);
      }
      if (!named_barrier_and(1, 128, ok)) break;  // sZ / sAlpha of this tile are visible
      // The previous tile's output, staged in its H~_i slot, has been read out by the TMA
      // store once this thread's bulk group is done reading: the slot may take a K/V block
      // again (the next one needed there is this tile's second block, or a later one).
      if (release_slot >= 0) {
        tma_store_wait_read();
        mbar_arrive(&k_empty[release_slot]);
        mbar_arrive(&v_empty[release_slot]);
        release_slot = -1;
      }
      if (!PISA && wt < D && t + static_cast<int>(gridDim.x) < a.n_tiles) {
        const int tn = t + gridDim.x;
        if (a.Zagg) z_next = a.Zagg[static_cast<size_t>(tn) * D + wt];
        a_next = a.alpha[(tn / a.Nq % a.H) * D + wt];
      }
      float m_run = -INFINITY, l_run = 0.f;  // running max (scaled, log2 units) and row sum
      float a_run = 0.f;                     // PISA: sum of the centroid weights p_j
      int cp = 0;                            // PISA: first critical entry not yet met by a pseudo-block
      uint32_t sa[32], sb[32];               // S columns [0, 32) and [32, 64) of the current block
      int j_cur = kc > 0 ? clist[0] : 0;
      if (nblk > 0) {
        ok = ok && __all_sync(0xffffffffu, mbar_wait(&s_full[ns & 1], (ns >> 1) & 1, a.err, &abort_flag));
        if (ok) {
          tc_fence_after();
          tmem_ld32(lane_addr + (ns & 1) * 64, sa);
          tmem_ld32(lane_addr + (ns & 1) * 64 + 32, sb);
          tmem_wait_ld();
        }
      }
      const uint64_t sc2 = f2_make(sc, sc);
      uint32_t pk[32];  // P of the current block, bf16 pairs
      for (int n = 0; ok && n < nblk; ++n, ++ns) {
        const int b = ns & 1;
        const int j_next = n + 1 < kc ? clist[n + 1] : 0;
        const bool centroid = PISA && n >= kc;
        uint64_t keep = ~0ull;  // PISA: the centroids of this pseudo-block that take part
        int valid = 64;         // valid key columns of this block
        if (!centroid) {
          valid = min(64, a.N - j_cur * 64);
        } else {
          // centroids 64 pb .. 64 pb + 63: drop those of critical blocks (the ascending list
          // is walked once over the tile's pseudo-blocks) and those past Nk
          const int pb = n - kc;
          while (cp < kc && clist[cp] < 64 * (pb + 1)) {
            keep &= ~(1ull << (clist[cp] - 64 * pb));
            ++cp;
          }
          const int nv = min(64, a.Nk - 64 * pb);
          if (nv < 64) keep &= (1ull << nv) - 1ull;
        }
        if (!centroid) {
          if (valid < 64) {
            mask_scores<0>(sa, valid, ~0ull);
            mask_scores<32>(sb, valid, ~0ull);
          }
        } else if (keep != ~0ull) {
          mask_scores<0>(sa, 64, keep);
          mask_scores<32>(sb, 64, keep);
        }
        // Reference maximum: the tile's first block sets it; it moves only past kRefMoveSum.
        if (n == 0) m_run = row_max64(sa, sb) * sc;
        uint64_t nm2 = f2_make(-m_run, -m_run);
        uint64_t pst = exp2_block(sa, sb, pk, sc2, nm2);
        float psum = f2_lo(pst) + f2_hi(pst);
        if (__any_sync(0xffffffffu, psum > kRefMoveSum)) {
          // Move the reference to the block's maximum: rescale the row of O_s (needs P*V of
          // the previous block finished) and l, then recompute P.
          const float m_new = fmaxf(m_run, row_max64(sa, sb) * sc);
          const float f = fast_exp2(m_run - m_new);
          if (n > 0) {  // the first block of a tile never gets here: its sum is at most 64
            ok = __all_sync(0xffffffffu, mbar_wait(&pv_done[(ns - 1) & 1], ((ns - 1) >> 1) & 1, a.err, &abort_flag));
            if (!ok) break;
            tc_fence_after();
            const uint64_t f2 = f2_make(f, f);
#pragma unroll 1
            for (int c0 = 0; c0 < D; c0 += 16) {
              uint32_t o[16];
              tmem_ld16(lane_addr + OS + c0, o);
              tmem_wait_ld();
#pragma unroll
              for (int c = 0; c < 16; c += 2) {
                const uint64_t y =
                    f2_mul(static_cast<uint64_t>(o[c]) | (static_cast<uint64_t>(o[c + 1]) << 32), f2);
                o[c] = static_cast<uint32_t>(y);
                o[c + 1] = static_cast<uint32_t>(y >> 32);
              }
              tmem_st16(lane_addr + OS + c0, o);
            }
            tmem_wait_st();
          }
          l_run *= f;
          a_run *= f;
          m_run = m_new;
          nm2 = f2_make(-m_run, -m_run);
          pst = exp2_block(sa, sb, pk, sc2, nm2);
          psum = f2_lo(pst) + f2_hi(pst);
        }
        if (!centroid) {
          l_run += psum;
        } else {
          // centroid j weighs n_j in the normaliser: 64, except a short last block
          float wsum = 64.f * psum;
          const int cl = a.Nk - 1 - 64 * (a.nc - 1);  // column of block Nk - 1 in the last pseudo-block
          if (a.n_last < 64 && n + 1 == nblk && ((keep >> cl) & 1ull)) {
            float s_l = 0.f;
#pragma unroll
            for (int c = 0; c < 32; ++c) {
              if (c == cl) s_l = __uint_as_float(sa[c]);
              if (c + 32 == cl) s_l = __uint_as_float(sb[c]);
            }
            wsum -= static_cast<float>(64 - a.n_last) * fast_exp2(fmaf(s_l, sc, -m_run));
          }
          l_run += wsum;
          a_run += psum;
        }
        tmem_st32(lane_addr + b * 64, pk);  // P over the first 32 columns of its S
        // Publish P_n before waiting for S_{n+1}: P*V of this block, and the S two blocks on
        // (which reuses these columns), can then be issued while S_{n+1} is still in flight.
        // (Loading S_{n+1} from TMEM before this store, or during the exponentials, measured
        // slower.)
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(&p_full[b]);
        if (n + 1 < nblk) {
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
      // Linear branch. P_lin goes into the S columns the next block would have used
      // (ns & 1); their last reader is the P*V two blocks back (with one block or none, an
      // MMA of an earlier tile, finished before this tile's lin_done was seen).
      if (ok && nblk >= 2)
        ok = __all_sync(0xffffffffu, mbar_wait(&pv_done[(ns - 2) & 1], ((ns - 2) >> 1) & 1, a.err, &abort_flag));
      if (ok) ok = __all_sync(0xffffffffu, mbar_wait(&q_full, k & 1, a.err, &abort_flag));
      // Pass 1: phi(q) (bf16, as the tensor core takes it) into the P_lin columns, 32
      // elements at a time, and den = phi(q) . Z_i from those rounded values; then the Q tile
      // is released (the next tile's Q may land). Column pairs in paired arithmetic:
      // phi(x) = x + 1 for x > 0, else e^x = 2^(x log2 e) (with FM = 1, e^x throughout).
      const uint32_t pl = lane_addr + (ns & 1) * 64;
      float l_eff;
      if constexpr (PISA) {
        // First-order term: P_lin = (A / sqrt(D)) q in bf16 against H~ = Hbar; l > 0 always
        // (the row maximum is a key or a centroid that takes part).
        l_eff = l_run;
        if (ok) {
          const float cq = a_run * a.inv_sqrt_d;
          const uint64_t c2 = f2_make(cq, cq);
#pragma unroll 1
          for (int g = 0; g < D / 32; ++g) {
            uint32_t w[16];
#pragma unroll
            for (int c = 0; c < 4; ++c) {
              const int c8 = 4 * g + c;
              const uint4 u = *reinterpret_cast<const uint4*>(sQ + (c8 >> 3) * 16384 + sw128_offset(r, (c8 & 7) * 16));
              w[4 * c] = u.x;
              w[4 * c + 1] = u.y;
              w[4 * c + 2] = u.z;
              w[4 * c + 3] = u.w;
            }
#pragma unroll
            for (int e = 0; e < 16; ++e) {
              const uint64_t y2 = f2_mul(c2, static_cast<uint64_t>(w[e] << 16) | (static_cast<uint64_t>(w[e] & 0xFFFF0000u) << 32));
              w[e] = pack_bf16x2(f2_lo(y2), f2_hi(y2));
            }
            tmem_st16(pl + 16 * g, w);
          }
          tmem_wait_st();
        }
        mbar_arrive(&q_free);
      } else {
        uint64_t den2 = 0ull;
        if (ok) {
          const uint64_t one2 = f2_make(1.f, 1.f), log2e2 = f2_make(1.4426950408889634f, 1.4426950408889634f);
#pragma unroll 1
          for (int g = 0; g < D / 32; ++g) {
            uint32_t w[16];
#pragma unroll
            for (int c = 0; c < 4; ++c) {
              const int c8 = 4 * g + c;
              const uint4 u = *reinterpret_cast<const uint4*>(sQ + (c8 >> 3) * 16384 + sw128_offset(r, (c8 & 7) * 16));
              w[4 * c] = u.x;
              w[4 * c + 1] = u.y;
              w[4 * c + 2] = u.z;
              w[4 * c + 3] = u.w;
            }
#pragma unroll
            for (int e = 0; e < 16; ++e) {
              // bf16 -> fp32 is a shift into the high half-word
              const uint64_t x2 = static_cast<uint64_t>(w[e] << 16) | (static_cast<uint64_t>(w[e] & 0xFFFF0000u) << 32);
              const uint64_t pos2 = f2_add(x2, one2);
              const uint64_t t2 = f2_mul(x2, log2e2);
              const float g0 = FM == 0 && f2_lo(x2) > 0.f ? f2_lo(pos2) : fast_exp2(f2_lo(t2));
              const float g1 = FM == 0 && f2_hi(x2) > 0.f ? f2_hi(pos2) : fast_exp2(f2_hi(t2));
              w[e] = pack_bf16x2(g0, g1);
              const uint64_t gr2 = static_cast<uint64_t>(w[e] << 16) | (static_cast<uint64_t>(w[e] & 0xFFFF0000u) << 32);
              den2 = f2_fma(gr2, *reinterpret_cast<const uint64_t*>(&sZ[32 * g + 2 * e]), den2);
            }
            tmem_st16(pl + 16 * g, w);
          }
        }
        mbar_arrive(&q_free);
        // The blend O = alpha O_s / l + (1 - alpha) O_l / den, with the accumulator holding
        // l O_s and H~_i = H_i (1 - alpha) / alpha, is alpha (acc + (l / den) phi(q) H~_i) / l.
        // With no critical block l is taken as 1 (acc starts at 0); with no marginal block
        // (den = 0) the linear term is 0.
        const float den_tot = f2_lo(den2) + f2_hi(den2);
        l_eff = kc > 0 ? l_run : 1.f;
        const float c_lin = den_tot > 0.f ? l_eff / den_tot : 0.f;
        // Pass 2: P_lin = (l / den) phi(q), rounded to bf16 in place.
        if (ok) {
          tmem_wait_st();
          const uint64_t c2 = f2_make(c_lin, c_lin);
#pragma unroll 1
          for (int g = 0; g < D / 64; ++g) {
            uint32_t w[32];
            tmem_ld32(pl + 32 * g, w);
            tmem_wait_ld();
#pragma unroll
            for (int e = 0; e < 32; ++e) {
              const uint64_t g2 = f2_mul(c2, static_cast<uint64_t>(w[e] << 16) | (static_cast<uint64_t>(w[e] & 0xFFFF0000u) << 32));
              w[e] = pack_bf16x2(f2_lo(g2), f2_hi(g2));
            }
            tmem_st32(pl + 32 * g, w);
          }
          tmem_wait_st();
        }
      }
      tc_fence_before();
      mbar_arrive(&plin_full);
      if (ok) ok = __all_sync(0xffffffffu, mbar_wait(&lin_done, k & 1, a.err, &abort_flag));
      if (!(ok = named_barrier_and(1, 128, ok))) break;

      // Epilogue: O = alpha acc / l in bf16, staged row by row in the H~_i slot (the linear MMA
      // has read it) in the 128-byte swizzle and written by TMA stores of block_q rows (rows
      // past N are clipped by the tensor map; with block_q = 64 the tile's upper 64 rows belong
      // to the next query block and are not stored); the loads of the next 32 columns overlap
      // the arithmetic and shared-memory writes of the current ones.
      tc_fence_after();
      const float inv_l = 1.f / l_eff;
      uint8_t* stage = sRing + hs * L::SLOT;  // DB boxes of 128 rows x 64 columns
      const uint64_t il2 = f2_make(inv_l, inv_l);
      uint32_t ob[2][32];
      tmem_ld32(lane_addr + OS, ob[0]);
      tmem_wait_ld();
#pragma unroll
      for (int q = 0; q < D / 32; ++q) {
        if (q + 1 < D / 32) tmem_ld32(lane_addr + OS + 32 * (q + 1), ob[(q + 1) & 1]);
        uint32_t pk[16];
#pragma unroll
        for (int c = 0; c < 32; c += 2) {
          const uint64_t al2 = *reinterpret_cast<const uint64_t*>(&sAlpha[32 * q + c]);
          const uint64_t y = f2_mul(f2_mul(al2, il2), static_cast<uint64_t>(ob[q & 1][c]) |
                                                          (static_cast<uint64_t>(ob[q & 1][c + 1]) << 32));
          pk[c >> 1] = pack_bf16x2(f2_lo(y), f2_hi(y));
        }
        uint8_t* box = stage + (q >> 1) * 16384;
#pragma unroll
        for (int v = 0; v < 4; ++v)
          *reinterpret_cast<uint4*>(box + sw128_offset(r, ((q & 1) * 4 + v) * 16)) =
              make_uint4(pk[4 * v], pk[4 * v + 1], pk[4 * v + 2], pk[4 * v + 3]);
        if (q + 1 < D / 32) tmem_wait_ld();
      }
      fence_proxy_async_smem();
      named_barrier(1, 128);
      if (wt == 0) {
        for (int b = 0; b < DB; ++b) tma_store_3d(&map_o, stage + b * 16384, b * 64, i * a.block_q, bh);
        tma_store_commit();
        release_slot = static_cast<int>(hs);  // released at the next tile's start (see there)
      }
      tc_fence_before();
      mbar_arrive(&tmem_free);  // the accumulator has left TMEM: the next tile may overwrite it
    }
  }
  if (tid == 64) tma_store_wait_all();
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, TMEM_COLS);
  }
}

}  // namespace sla
