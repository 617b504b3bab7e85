// Backward pass of the SLA forward, per query tile (128 query rows of one (batch, head)),
// D = 128. With dO the output gradient, G_s = alpha dO and G_l = (1 - alpha) dO:
//
//   pass 1 (the tile's critical blocks, as the forward): online softmax of S = Q K_j^T / sqrt(D)
//            gives the row maximum m and sum l, hence LSE = m + log2 l (log2 units) and
//            O_s = P V / l; Delta = rowsum(G_s * O_s)
//   linear   u = phi(Q), O_l = u H_i / den, den = u . Z_i; dalpha += sum_t dO (O_s - O_l);
//            dnum = G_l / den, dden = -(G_l . O_l) / den;
//            dQ  = (dnum H_i^T + dden Z_i^T) * phi'(q)      (dnum H_i^T: tcgen05, two N=64 MMAs)
//            dH_i = u^T dnum  (tcgen05),  dZ_i = u^T dden   (written stacked, [dH_i | dZ_i],
//            for the aggregation run backwards)
//   pass 2 (the critical blocks again): P = 2^(S log2e - LSE), dP = G_s V_j^T,
//            dS = P (dP - Delta) / sqrt(D); dQ += dS K_j (accumulated in TMEM over the
//            blocks). LSE and Delta of every row are written out: the KV-block pass
//            (bwd_kv_kernel) recomputes P and dS from them for dK_j and dV_j.
//
// Source: "SLA: Beyond Sparsity in Diffusion Transformers via Fine-Tunable Sparse-Linear
// Attention", Abstract (one kernel covers forward and backward). The formulas are the exact
// derivative of the forward with the block labels held fixed (the hard top-k passes no
// gradient); the sparse branch's are those of softmax attention renormalised over the
// critical keys.
//
// Persistent, one CTA per SM, 192 threads:
//   warp 0      TMA: per tile Q, G_s and dO (128 rows each), then through a 2-slot ring K_j / V_j
//               of every critical block (pass 1), H_i (one slot), K_j / V_j again (pass 2)
//   warp 1      TMEM owner and tcgen05 issuer (one elected lane)
//   warps 2..5  thread = query row = TMEM lane for the row-wise work; for dH_i the TMEM lane
//               is a channel
// TMEM (512 columns): pass 1 S [0,64) [64,128), acc [128,256); linear O_l [256,384),
// dnum H^T [384,512), dH [0,128); pass 2 S / dP pairs [0,128) [128,256) (S at +0, dP at
// +64), dQ [256,384).
// Shared memory: Q, G_s, U (phi(Q); in pass 2 dS), dO / dnum: 32 KB each; ring 2 x 32 KB.
#pragma once

#include "softmax_block.cuh"

namespace sla {

struct BwdArgs {
  int H, N, Nq, n_tiles, LD;
  const int32_t* crit;      // [BH*Nq, crit_ld] ascending
  int crit_ld;
  const int32_t* crit_cnt;  // [BH*Nq]
  const float* Zagg;        // [BH*Nq, D]
  const float* alpha;       // [H, D]
  float* dQ;                // [BH, N, D]   written
  float* lse;               // [BH, N]      written: log2-sum-exp of the row's critical scores
  float* delta;             // [BH, N]      written: rowsum(G_s * O_s)
  float* dalpha_part;       // [n_tiles, D] written: the tile's sum over rows of dO (O_s - O_l)
  __nv_bfloat16* dHst;      // [BH*Nq, LD]  written: dH_i row-major (D*D), then dZ_i (D), then 0
  float scale_log2;         // log2(e) / sqrt(D)
  uint32_t* err;
};

__global__ void __launch_bounds__(192, 1)
    bwd_kernel(const __grid_constant__ CUtensorMap map_q, const __grid_constant__ CUtensorMap map_g,
               const __grid_constant__ CUtensorMap map_k, const __grid_constant__ CUtensorMap map_v,
               const __grid_constant__ CUtensorMap map_h, const __grid_constant__ CUtensorMap map_do, BwdArgs a) {
  constexpr int D = 128;
  constexpr uint32_t TILE = 32768, SLOT = 32768, KV = 16384;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sQ = base;
  uint8_t* sG = base + TILE;
  uint8_t* sU = base + 2 * TILE;   // phi(Q); in pass 2: dS [128 x 64] at +16384
  uint8_t* sDn = base + 3 * TILE;  // dO of the tile (TMA), rewritten row by row as dnum
  uint8_t* sRing = base + 4 * TILE;
  uint8_t* sdS = sU + 16384;

  __shared__ uint64_t q_full, q_free, u_full, ol_done, dn_full, lin_done, t1_free, tile_done;
  __shared__ uint64_t k_full[2], k_empty[2], v_full[2], v_empty[2];
  __shared__ uint64_t s_full[2], p_full[2], pv_done[2];
  __shared__ uint64_t s2_full[2], ds_full, g2_done, drain;
  __shared__ uint32_t tmem_base_sh;
  __shared__ int abort_flag;
  __shared__ __align__(16) float sZ[D];
  __shared__ __align__(16) float sAl[D];
  __shared__ float sDden[128];
  __shared__ float sRed[4][D];  // per-warp partial sums of the tile's dalpha

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  if (tid == 0) {
    mbar_init(&q_full, 1);
    mbar_init(&q_free, 1 + 128);  // the tile's last MMA reading Q / G_s, and every row's last read of Q
    mbar_init(&u_full, 128);
    mbar_init(&ol_done, 1);
    mbar_init(&dn_full, 128);
    mbar_init(&lin_done, 1);
    mbar_init(&t1_free, 128);
    mbar_init(&tile_done, 128);
    for (int s = 0; s < 2; ++s) {
      mbar_init(&k_full[s], 1);
      mbar_init(&k_empty[s], 1);
      mbar_init(&v_full[s], 1);
      mbar_init(&v_empty[s], 1);
      mbar_init(&s_full[s], 1);
      mbar_init(&p_full[s], 128);
      mbar_init(&pv_done[s], 1);
    }
    mbar_init(&s2_full[0], 1);
    mbar_init(&s2_full[1], 1);
    mbar_init(&ds_full, 128);
    mbar_init(&g2_done, 1);
    mbar_init(&drain, 1);
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
  grid_dep_wait();

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      int k_round[2] = {-1, -1}, v_round[2] = {-1, -1};
      int q_loads = 0;
      uint32_t nb = 0;
      bool ok = true;
      int k = 0;
      auto load_kv = [&](int j, int bh) -> bool {
        const int s = nb & 1, r = nb >> 1;
        uint8_t* slot = sRing + s * SLOT;
        if (r > 0 && !mbar_wait(&k_empty[s], (r - 1) & 1, a.err, &abort_flag)) return false;
        mbar_arrive_expect_tx(&k_full[s], KV);
        for (int b = 0; b < 2; ++b) tma_load_3d(slot + b * 8192, &map_k, &k_full[s], b * 64, j * 64, bh);
        k_round[s] = r;
        if (r > 0 && !mbar_wait(&v_empty[s], (r - 1) & 1, a.err, &abort_flag)) return false;
        mbar_arrive_expect_tx(&v_full[s], KV);
        for (int b = 0; b < 2; ++b) tma_load_3d(slot + KV + b * 8192, &map_v, &v_full[s], b * 64, j * 64, bh);
        v_round[s] = r;
        ++nb;
        return true;
      };
      for (int t = blockIdx.x; ok && t < a.n_tiles; t += gridDim.x, ++k) {
        const int bh = t / a.Nq, i = t % a.Nq;
        const int kc = a.crit_cnt[t];
        const int32_t* clist = a.crit + static_cast<size_t>(t) * a.crit_ld;
        if (k > 0 && !(ok = mbar_wait(&q_free, (k - 1) & 1, a.err, &abort_flag))) break;
        mbar_arrive_expect_tx(&q_full, 3 * TILE);
        for (int b = 0; b < 2; ++b) {
          tma_load_3d(sQ + b * 16384, &map_q, &q_full, b * 64, i * 128, bh);
          tma_load_3d(sG + b * 16384, &map_g, &q_full, b * 64, i * 128, bh);
          tma_load_3d(sDn + b * 16384, &map_do, &q_full, b * 64, i * 128, bh);
        }
        ++q_loads;
        for (int n = 0; ok && n < kc; ++n) ok = load_kv(clist[n], bh);
        if (!ok) break;
        {  // H_i: rows 0..63 in the K half of the slot, rows 64..127 in the V half
          const int s = nb & 1, r = nb >> 1;
          uint8_t* slot = sRing + s * SLOT;
          if (r > 0 && !(ok = mbar_wait(&k_empty[s], (r - 1) & 1, a.err, &abort_flag))) break;
          mbar_arrive_expect_tx(&k_full[s], KV);
          for (int eh = 0; eh < 2; ++eh) tma_load_2d(slot + eh * 8192, &map_h, &k_full[s], eh * 64, t * D);
          k_round[s] = r;
          if (r > 0 && !(ok = mbar_wait(&v_empty[s], (r - 1) & 1, a.err, &abort_flag))) break;
          mbar_arrive_expect_tx(&v_full[s], KV);
          for (int eh = 0; eh < 2; ++eh) tma_load_2d(slot + KV + eh * 8192, &map_h, &v_full[s], eh * 64, t * D + 64);
          v_round[s] = r;
          ++nb;
        }
        for (int n = 0; ok && n < kc; ++n) ok = load_kv(clist[n], bh);
      }
      if (abort_flag) {
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
    const uint32_t id_s = idesc_bf16_f32(128, 64, 0, 0);   // A, B K-major, N = 64
    const uint32_t id_o = idesc_bf16_f32(128, D, 0, 1);    // A K-major, B MN-major, N = D
    const uint32_t id_t = idesc_bf16_f32(128, D, 1, 1);    // A, B MN-major, N = D
    const uint32_t q0 = smem_u32(sQ), g0 = smem_u32(sG), u0 = smem_u32(sU), dn0 = smem_u32(sDn);
    const uint32_t ring0 = smem_u32(sRing), ds0 = smem_u32(sdS);
    uint32_t nb = 0, ns = 0;
    bool ok = true;
    auto wait_all = [&](uint64_t* bar, uint32_t parity) -> bool {
      return __all_sync(0xffffffffu, mbar_wait(bar, parity, a.err, &abort_flag));
    };
    auto commit = [&](uint64_t* bar) {
      if (elect_one()) umma_commit(bar);
      __syncwarp();
    };
    auto mma_ss = [&](uint32_t d, uint64_t ad, uint64_t bd, uint32_t id, uint32_t acc) {
      if (elect_one()) umma_bf16_ss(d, ad, bd, id, acc);
      __syncwarp();
    };
    // A K-major (128 rows x 128, two 64-column boxes of 128 rows) step kk of 16 columns
    auto kmaj128 = [](uint32_t t0, int kk) { return smem_desc_sw128(t0 + (kk >> 2) * 16384 + (kk & 3) * 32, 16, 1024); };
    // B K-major (64 rows x 128, two boxes of 64 rows) step kk
    auto kmaj64 = [](uint32_t t0, int kk) { return smem_desc_sw128(t0 + (kk >> 2) * 8192 + (kk & 3) * 32, 16, 1024); };
    int k = 0;
    int n2 = 0;  // pass-2 blocks so far (over all tiles)
    for (int t = blockIdx.x; ok && t < a.n_tiles; t += gridDim.x, ++k) {
      const int kc = a.crit_cnt[t];
      if (!(ok = wait_all(&q_full, k & 1))) break;
      if (k > 0 && !(ok = wait_all(&tile_done, (k - 1) & 1))) break;  // the last tile's dQ was read
      // ---- pass 1: S, P V (as the forward)
      auto issue_pv = [&](uint32_t nbm, uint32_t nsm, bool first) -> bool {
        const int s = nbm & 1, b = nsm & 1;
        if (!wait_all(&p_full[b], (nsm >> 1) & 1)) return false;
        if (!wait_all(&v_full[s], (nbm >> 1) & 1)) return false;
        tc_fence_after();
        const uint32_t vb = ring0 + s * SLOT + KV;
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {
          const uint64_t bd = smem_desc_sw128(vb + kk * 2048, 8192, 1024);
          if (elect_one()) umma_bf16_ts(tmem + 128, tmem + b * 64 + kk * 8, bd, id_o, (first && kk == 0) ? 0u : 1u);
          __syncwarp();
        }
        commit(&pv_done[b]);
        commit(&v_empty[s]);
        return true;
      };
      for (int n = 0; n < kc; ++n, ++nb, ++ns) {
        const int s = nb & 1, b = ns & 1;
        if (!(ok = wait_all(&k_full[s], (nb >> 1) & 1))) break;
        tc_fence_after();
        const uint32_t kb = ring0 + s * SLOT;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) mma_ss(tmem + b * 64, kmaj128(q0, kk), kmaj64(kb, kk), id_s, kk > 0);
        commit(&s_full[b]);
        commit(&k_empty[s]);
        if (n >= 1 && !(ok = issue_pv(nb - 1, ns - 1, n == 1))) break;
      }
      if (!ok) break;
      if (kc > 0 && !(ok = issue_pv(nb - 1, ns - 1, kc == 1))) break;
      // ---- linear branch: O_l = U H_i, then dnum H_i^T and dH = U^T dnum
      const int sh = nb & 1;
      const uint32_t hb = ring0 + sh * SLOT;
      if (!(ok = wait_all(&k_full[sh], (nb >> 1) & 1))) break;
      if (!(ok = wait_all(&v_full[sh], (nb >> 1) & 1))) break;
      if (!(ok = wait_all(&u_full, k & 1))) break;
      tc_fence_after();
#pragma unroll
      for (int kk = 0; kk < D / 16; ++kk)
        mma_ss(tmem + 256, kmaj128(u0, kk), smem_desc_sw128(hb + (kk >> 2) * 2 * 8192 + (kk & 3) * 2048, 8192, 1024),
               id_o, kk > 0);
      commit(&ol_done);
      if (!(ok = wait_all(&dn_full, k & 1))) break;
      tc_fence_after();
      // dnum H^T: output columns d in two halves (H rows 0..63 in the K half, 64..127 in V)
      for (int hh = 0; hh < 2; ++hh)
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk)
          mma_ss(tmem + 384 + 64 * hh, kmaj128(dn0, kk), kmaj64(hb + hh * KV, kk), id_s, kk > 0);
      // dH = U^T dnum: M = channel d, N = channel e, K = the tile's 128 rows
#pragma unroll
      for (int kk = 0; kk < 8; ++kk)
        mma_ss(tmem, smem_desc_sw128(u0 + kk * 2048, 16384, 1024), smem_desc_sw128(dn0 + kk * 2048, 16384, 1024),
               id_t, kk > 0);
      commit(&lin_done);
      commit(&k_empty[sh]);
      commit(&v_empty[sh]);
      ++nb;
      // ---- pass 2: S, dP of block n into the pair (n2 & 1), then dQ += dS K of block n - 1
      if (!(ok = wait_all(&t1_free, k & 1))) break;  // dH, O_l, dnum H^T and acc have left TMEM
      // dQ += dS K_j of the pass-2 block at ring use nbm, pass-2 index m (onto the linear part
      // the warpgroup wrote into the accumulator); frees the block's ring slot and the dS tile
      auto issue_dq = [&](uint32_t nbm, int m) -> bool {
        if (!wait_all(&ds_full, m & 1)) return false;
        tc_fence_after();
        const uint32_t kb = ring0 + (nbm & 1) * SLOT;
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)  // K = 64 keys
          mma_ss(tmem + 256, smem_desc_sw128(ds0 + kk * 32, 16, 1024), smem_desc_sw128(kb + kk * 2048, 8192, 1024),
                 id_o, 1u);
        commit(&g2_done);
        commit(&k_empty[nbm & 1]);
        commit(&v_empty[nbm & 1]);
        return true;
      };
      for (int n = 0; n < kc; ++n, ++nb, ++n2) {
        const int s = nb & 1, b = n2 & 1;
        if (!(ok = wait_all(&k_full[s], (nb >> 1) & 1))) break;
        if (!(ok = wait_all(&v_full[s], (nb >> 1) & 1))) break;
        tc_fence_after();
        const uint32_t kb = ring0 + s * SLOT, vb = kb + KV;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) mma_ss(tmem + b * 128, kmaj128(q0, kk), kmaj64(kb, kk), id_s, kk > 0);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) mma_ss(tmem + b * 128 + 64, kmaj128(g0, kk), kmaj64(vb, kk), id_s, kk > 0);
        commit(&s2_full[b]);
        if (n >= 1 && !(ok = issue_dq(nb - 1, n2 - 1))) break;
      }
      if (!ok) break;
      if (kc > 0 && !(ok = issue_dq(nb - 1, n2 - 1))) break;
      if (!ok) break;
      commit(&q_free);
    }
    commit(&drain);
    mbar_wait(&drain, 0, nullptr, nullptr);
  } else {
    // ------------------------------------------------------------ row / channel work (warps 2..5)
    const int quarter = warp & 3, r = quarter * 32 + lane, wt = tid - 64, wq = warp - 2;
    const uint32_t lane_addr = tmem + (static_cast<uint32_t>(quarter * 32) << 16);
    const float sc = a.scale_log2;
    constexpr float kLn2 = 0.6931471805599453f;
    uint32_t ns = 0;
    bool ok = true;
    int k = 0, n2 = 0;
    for (int t = blockIdx.x; t < a.n_tiles; t += gridDim.x, ++k) {
      const int bh = t / a.Nq, i = t % a.Nq, h = bh % a.H;
      const int kc = a.crit_cnt[t];
      const int32_t* clist = a.crit + static_cast<size_t>(t) * a.crit_ld;
      const int tok = i * 128 + r;
      const bool row_ok = tok < a.N;
      if (!named_barrier_and(1, 128, ok)) break;
      sZ[wt] = a.Zagg[static_cast<size_t>(t) * D + wt];
      sAl[wt] = a.alpha[h * D + wt];
      if (!named_barrier_and(1, 128, ok)) break;
      // ---- pass 1: online softmax as in the forward (reference maximum from the tile's first
      // block, moved, with the accumulator rescaled, only when a block's sum passes kRefMoveSum)
      float m_run = -INFINITY, l_run = 0.f;
      const uint64_t sc2 = f2_make(sc, sc);
      for (int n = 0; ok && n < kc; ++n, ++ns) {
        const int b = ns & 1;
        const int valid = min(64, a.N - clist[n] * 64);
        ok = __all_sync(0xffffffffu, mbar_wait(&s_full[b], (ns >> 1) & 1, a.err, &abort_flag));
        if (!ok) break;
        tc_fence_after();
        uint32_t sa[32], sb[32];
        tmem_ld32(lane_addr + b * 64, sa);
        tmem_ld32(lane_addr + b * 64 + 32, sb);
        tmem_wait_ld();
        if (valid < 64) {
          mask_scores<0>(sa, valid, ~0ull);
          mask_scores<32>(sb, valid, ~0ull);
        }
        if (n == 0) m_run = row_max64(sa, sb) * sc;
        uint32_t pk[32];
        uint64_t pst = exp2_block(sa, sb, pk, sc2, f2_make(-m_run, -m_run));
        float psum = f2_lo(pst) + f2_hi(pst);
        if (n > 0 && __any_sync(0xffffffffu, psum > kRefMoveSum)) {  // (the first block sums to <= 64)
          ok = __all_sync(0xffffffffu, mbar_wait(&pv_done[(ns - 1) & 1], ((ns - 1) >> 1) & 1, a.err, &abort_flag));
          if (!ok) break;
          tc_fence_after();
          const float m_new = fmaxf(m_run, row_max64(sa, sb) * sc);
          const float f = fast_exp2(m_run - m_new);
          const uint64_t f2 = f2_make(f, f);
#pragma unroll 1
          for (int c0 = 0; c0 < D; c0 += 32) {
            uint32_t o[32];
            tmem_ld32(lane_addr + 128 + c0, o);
            tmem_wait_ld();
#pragma unroll
            for (int c = 0; c < 32; c += 2) {
              const uint64_t y = f2_mul(static_cast<uint64_t>(o[c]) | (static_cast<uint64_t>(o[c + 1]) << 32), f2);
              o[c] = static_cast<uint32_t>(y);
              o[c + 1] = static_cast<uint32_t>(y >> 32);
            }
            tmem_st32(lane_addr + 128 + c0, o);
          }
          tmem_wait_st();
          l_run *= f;
          m_run = m_new;
          pst = exp2_block(sa, sb, pk, sc2, f2_make(-m_run, -m_run));
          psum = f2_lo(pst) + f2_hi(pst);
        }
        l_run += psum;
        tmem_st32(lane_addr + b * 64, pk);
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(&p_full[b]);
      }
      if (ok && kc > 0)
        ok = __all_sync(0xffffffffu, mbar_wait(&pv_done[(ns - 1) & 1], ((ns - 1) >> 1) & 1, a.err, &abort_flag));
      if (ok) ok = __all_sync(0xffffffffu, mbar_wait(&q_full, k & 1, a.err, &abort_flag));
      const float lse = kc > 0 ? m_run + log2f(l_run) : -INFINITY;  // log2 units
      const float inv_l = kc > 0 ? 1.f / l_run : 0.f;
      // ---- phi(Q) into U (bf16, the layout of Q) and den = phi(q) . Z_i from those values
      float den = 0.f;
      if (ok) {
#pragma unroll 1
        for (int c8 = 0; c8 < D / 8; ++c8) {
          const uint32_t off = (c8 >> 3) * 16384 + sw128_offset(r, (c8 & 7) * 16);
          const uint4 u = *reinterpret_cast<const uint4*>(sQ + off);
          uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const float2 x = unpack_bf16x2(w[e]);
            const float f0 = x.x > 0.f ? x.x + 1.f : __expf(x.x), f1 = x.y > 0.f ? x.y + 1.f : __expf(x.y);
            w[e] = pack_bf16x2(f0, f1);
            const float2 fr = unpack_bf16x2(w[e]);
            den += fr.x * sZ[c8 * 8 + 2 * e] + fr.y * sZ[c8 * 8 + 2 * e + 1];
          }
          *reinterpret_cast<uint4*>(sU + off) = make_uint4(w[0], w[1], w[2], w[3]);
        }
        fence_proxy_async_smem();
      }
      tc_fence_before();
      mbar_arrive(&u_full);
      if (ok) ok = __all_sync(0xffffffffu, mbar_wait(&ol_done, k & 1, a.err, &abort_flag));
      // ---- per row: O_s, O_l, Delta, dalpha, dnum, dden (32 channels at a time)
      const float inv_den = den > 0.f ? 1.f / den : 0.f;
      float delta = 0.f, dden_acc = 0.f;
      if (ok) {
        tc_fence_after();
#pragma unroll 1
        for (int c0 = 0; c0 < D; c0 += 32) {
          uint32_t os[32], ol[32];
          tmem_ld32(lane_addr + 128 + c0, os);
          tmem_ld32(lane_addr + 256 + c0, ol);
          tmem_wait_ld();
          uint32_t dn[16];
#pragma unroll
          for (int c = 0; c < 32; c += 8) {
            // this row's dO (rows past N arrive as zeros); its dnum is written over it below
            const int c8d = (c0 + c) >> 3;
            const uint4 du4 = *reinterpret_cast<const uint4*>(sDn + (c8d >> 3) * 16384 + sw128_offset(r, (c8d & 7) * 16));
            const uint32_t dw[4] = {du4.x, du4.y, du4.z, du4.w};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const float2 g = unpack_bf16x2(dw[e]);
              const int cc = c + 2 * e;
              const float al0 = sAl[c0 + cc], al1 = sAl[c0 + cc + 1];
              const float os0 = __uint_as_float(os[cc]) * inv_l, os1 = __uint_as_float(os[cc + 1]) * inv_l;
              const float ol0 = __uint_as_float(ol[cc]) * inv_den, ol1 = __uint_as_float(ol[cc + 1]) * inv_den;
              // G_s and G_l from dO; Delta from the same bf16 G_s the MMAs see
              const float2 gs = unpack_bf16x2(pack_bf16x2(al0 * g.x, al1 * g.y));
              delta += gs.x * os0 + gs.y * os1;
              const float gl0 = (1.f - al0) * g.x, gl1 = (1.f - al1) * g.y;
              dden_acc += gl0 * ol0 + gl1 * ol1;
              dn[(cc >> 1)] = pack_bf16x2(gl0 * inv_den, gl1 * inv_den);
              // dalpha: sum over rows of dO (O_s - O_l), per channel
              os[cc] = __float_as_uint(row_ok ? g.x * (os0 - ol0) : 0.f);
              os[cc + 1] = __float_as_uint(row_ok ? g.y * (os1 - ol1) : 0.f);
            }
          }
          // dnum row into its tile (the layout of Q)
#pragma unroll
          for (int v = 0; v < 4; ++v) {
            const int c8 = (c0 >> 3) + v;
            *reinterpret_cast<uint4*>(sDn + (c8 >> 3) * 16384 + sw128_offset(r, (c8 & 7) * 16)) =
                make_uint4(dn[4 * v], dn[4 * v + 1], dn[4 * v + 2], dn[4 * v + 3]);
          }
          // dalpha partial over this warp's 32 rows (butterfly), then one row per warp
#pragma unroll
          for (int c = 0; c < 32; ++c) {
            float v = __uint_as_float(os[c]);
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
            if (lane == c) sRed[wq][c0 + c] = v;
          }
        }
        fence_proxy_async_smem();
      }
      const float dden = -dden_acc * inv_den;
      if (row_ok) {  // for the KV-block pass
        a.lse[static_cast<size_t>(bh) * a.N + tok] = lse;
        a.delta[static_cast<size_t>(bh) * a.N + tok] = delta;
      }
      sDden[r] = dden;
      tc_fence_before();
      mbar_arrive(&dn_full);
      if (!(ok = named_barrier_and(1, 128, ok))) break;  // sRed, sDden complete
      a.dalpha_part[static_cast<size_t>(t) * D + wt] = sRed[0][wt] + sRed[1][wt] + sRed[2][wt] + sRed[3][wt];
      ok = __all_sync(0xffffffffu, mbar_wait(&lin_done, k & 1, a.err, &abort_flag));
      if (ok) {
        tc_fence_after();
        // dQ (linear part) = (dnum H^T + dden Z) * phi'(q), row r, into the dQ accumulator's TMEM
        // columns (O_l has been read out of them): pass 2 adds the sparse part on top and dQ
        // leaves TMEM once, at the end of the tile
#pragma unroll 1
        for (int c0 = 0; c0 < D; c0 += 32) {
          uint32_t du[32];
          tmem_ld32(lane_addr + 384 + c0, du);
          tmem_wait_ld();
#pragma unroll
          for (int c = 0; c < 32; c += 8) {
            const uint4 q4 = *reinterpret_cast<const uint4*>(sQ + ((c0 + c) >> 6) * 16384 +
                                                              sw128_offset(r, (((c0 + c) & 63) >> 3) * 16));
            const uint32_t qw[4] = {q4.x, q4.y, q4.z, q4.w};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const float2 x = unpack_bf16x2(qw[e]);
              const int cc = c + 2 * e;
              const float o0 = (__uint_as_float(du[cc]) + dden * sZ[c0 + cc]) * (x.x > 0.f ? 1.f : __expf(x.x));
              const float o1 = (__uint_as_float(du[cc + 1]) + dden * sZ[c0 + cc + 1]) * (x.y > 0.f ? 1.f : __expf(x.y));
              du[cc] = __float_as_uint(row_ok ? o0 : 0.f);
              du[cc + 1] = __float_as_uint(row_ok ? o1 : 0.f);
            }
          }
          tmem_st32(lane_addr + 256 + c0, du);
        }
        tmem_wait_st();
      }
      mbar_arrive(&q_free);  // this row's last read of Q (phi'(q)); pass 2 reads Q through MMAs only
      if (ok) {
        // dH_i (TMEM lane = channel d = r, columns e) and dZ_i = sum_t u[t][d] dden[t], stacked
        __nv_bfloat16* drow = a.dHst + static_cast<size_t>(t) * a.LD;
#pragma unroll 1
        for (int c0 = 0; c0 < D; c0 += 32) {
          uint32_t hv[32];
          tmem_ld32(lane_addr + c0, hv);
          tmem_wait_ld();
          uint32_t pk[16];
#pragma unroll
          for (int c = 0; c < 32; c += 2) pk[c >> 1] = pack_bf16x2(__uint_as_float(hv[c]), __uint_as_float(hv[c + 1]));
          uint4* dst = reinterpret_cast<uint4*>(drow + static_cast<size_t>(r) * D + c0);
#pragma unroll
          for (int v = 0; v < 4; ++v) dst[v] = make_uint4(pk[4 * v], pk[4 * v + 1], pk[4 * v + 2], pk[4 * v + 3]);
        }
        float dz = 0.f;
#pragma unroll 4
        for (int tt = 0; tt < 128; ++tt) {
          const uint16_t ub = *reinterpret_cast<const uint16_t*>(sU + (r >> 6) * 16384 +
                                                                 sw128_offset(tt, ((r & 63) >> 3) * 16) + (r & 7) * 2);
          dz += __uint_as_float(static_cast<uint32_t>(ub) << 16) * sDden[tt];
        }
        drow[D * D + r] = __float2bfloat16_rn(dz);
      }
      // O_s / O_l / dnum H^T / dH have left TMEM, and U may take P and dS
      tc_fence_before();
      if (!(ok = named_barrier_and(1, 128, ok))) break;
      mbar_arrive(&t1_free);
      // ---- pass 2
      const float lse_r = lse;
      const float shift = log2f(sc * kLn2) - lse_r;  // log2(1 / sqrt(D)) - LSE
      const uint64_t sh2 = f2_make(shift, shift), nd2 = f2_make(-delta, -delta);
      for (int n = 0; ok && n < kc; ++n, ++n2) {
        const int j = clist[n];
        const int valid = min(64, a.N - j * 64);
        const int b = n2 & 1;
        ok = __all_sync(0xffffffffu, mbar_wait(&s2_full[b], (n2 >> 1) & 1, a.err, &abort_flag));
        if (!ok) break;
        tc_fence_after();
        uint32_t dk[32];
#pragma unroll 1
        for (int hh = 0; hh < 2; ++hh) {
          uint32_t sx[32], dp[32];
          tmem_ld32(lane_addr + b * 128 + 32 * hh, sx);
          tmem_ld32(lane_addr + b * 128 + 64 + 32 * hh, dp);
          tmem_wait_ld();
          // P / sqrt(D) = 2^(S log2(e) / sqrt(D) - LSE + log2(1 / sqrt(D))); dS = (P / sqrt(D)) (dP - Delta)
#pragma unroll
          for (int c = 0; c < 32; c += 2) {
            const int n0 = 32 * hh + c;
            const uint64_t x2 = f2_fma(static_cast<uint64_t>(sx[c]) | (static_cast<uint64_t>(sx[c + 1]) << 32), sc2, sh2);
            const float p0 = (row_ok && n0 < valid) ? fast_exp2(f2_lo(x2)) : 0.f;
            const float p1 = (row_ok && n0 + 1 < valid) ? fast_exp2(f2_hi(x2)) : 0.f;
            const uint64_t d2 = f2_add(static_cast<uint64_t>(dp[c]) | (static_cast<uint64_t>(dp[c + 1]) << 32), nd2);
            const uint64_t g2 = f2_mul(f2_make(p0, p1), d2);
            dk[16 * hh + (c >> 1)] = pack_bf16x2(f2_lo(g2), f2_hi(g2));
          }
        }
        // dS may overwrite its tile once the previous block's dQ MMAs have read it
        if (n2 > 0) ok = __all_sync(0xffffffffu, mbar_wait(&g2_done, (n2 - 1) & 1, a.err, &abort_flag));
        if (!ok) break;
#pragma unroll
        for (int v = 0; v < 8; ++v)
          *reinterpret_cast<uint4*>(sdS + sw128_offset(r, v * 16)) =
              make_uint4(dk[4 * v], dk[4 * v + 1], dk[4 * v + 2], dk[4 * v + 3]);
        fence_proxy_async_smem();
        tc_fence_before();
        mbar_arrive(&ds_full);
      }
      // the tile's last dQ MMAs are done
      if (ok && kc > 0) ok = __all_sync(0xffffffffu, mbar_wait(&g2_done, (n2 - 1) & 1, a.err, &abort_flag));
      // ---- dQ (linear part plus the sparse part, the last pass-2 MMAs done) leaves TMEM
      if (ok) {
        tc_fence_after();
        float* dqrow = a.dQ + (static_cast<size_t>(bh) * a.N + tok) * D;
#pragma unroll 1
        for (int c0 = 0; c0 < D; c0 += 32) {
          uint32_t qv[32];
          tmem_ld32(lane_addr + 256 + c0, qv);
          tmem_wait_ld();
          if (row_ok) {
#pragma unroll
            for (int c = 0; c < 32; c += 4)
              *reinterpret_cast<float4*>(dqrow + c0 + c) = make_float4(__uint_as_float(qv[c]), __uint_as_float(qv[c + 1]),
                                                                       __uint_as_float(qv[c + 2]), __uint_as_float(qv[c + 3]));
          }
        }
      }
      tc_fence_before();
      mbar_arrive(&tile_done);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// dalpha[h, :] = sum over the (batch entry, query tile) pairs of head h of the tiles' partial
// sums: eight interleaved partial sums per channel, then added in a fixed order.
// grid (H, D / 32), block (32, 8).
__global__ void __launch_bounds__(256) dalpha_kernel(const float* __restrict__ part, float* __restrict__ dalpha, int B,
                                                     int H, int Nq, int D) {
  __shared__ float red[8][32];
  const int h = blockIdx.x, d = blockIdx.y * 32 + threadIdx.x, g = threadIdx.y;
  float s = 0.f;
  for (int u = g; u < B * Nq; u += 8) {
    const int b = u / Nq, i = u % Nq;
    s += part[(static_cast<size_t>(b * H + h) * Nq + i) * D + d];
  }
  red[g][threadIdx.x] = s;
  __syncthreads();
  if (g == 0) {
    float t = 0.f;
#pragma unroll
    for (int q = 0; q < 8; ++q) t += red[q][threadIdx.x];
    dalpha[h * D + d] = t;
  }
}

}  // namespace sla
