// Backward pass of the SLA forward, per KV block: the sparse branch's dK_j and dV_j summed
// over the query tiles that hold block j as critical, plus the linear branch's per-block
// states, written once (no atomics, a fixed summation order).
//
// Per KV block j of head bh (D = 128), over the query tiles i whose critical set holds j, in
// ascending i, with LSE and Delta of every row from the query-tile pass:
//   S = Q_i K_j^T, dP = G_s,i V_j^T                    (tcgen05, M = 128 rows, N = 64 keys)
//   P = 2^(S log2(e) / sqrt(D) - LSE), dS = P (dP - Delta) / sqrt(D)
//   dV_j^T += G_s,i^T P, dK_j^T += Q_i^T dS            (M = 128 channels, N = 64 keys, K = 128 rows)
// then the states' part (h_j = phi(K_j)^T V_j, z_j = colsum phi(K_j)):
//   dV_j^T += dh_j^T phi(K_j)^T, A1 = dh_j V_j^T, dK_j = (dK_j^T)^T + (A1^T + dz_j) * phi'(K_j)
// with phi'(k) = 1 for k > 0 and e^k otherwise, which is min(phi(k), 1).
//
// Source: "SLA: Beyond Sparsity in Diffusion Transformers via Fine-Tunable Sparse-Linear
// Attention", Abstract (one kernel covers the forward and the backward pass). The formulas
// are the exact derivative of the forward with the block labels held fixed.
//
// Persistent, one CTA per SM (512 TMEM columns), 192 threads; a CTA takes the KV blocks
// g = blockIdx.x, blockIdx.x + gridDim.x, ... (g = bh * Nk + j):
//   warp 0      TMA: K_j and V_j (one 32 KB buffer), then Q_i and G_s,i of each tile and
//               finally dh_j through a ring of five 32 KB slots (a tile takes two
//               consecutive slots, dh_j one), so the next tile's Q_i can land before the
//               previous tile's slots are free
//   warp 1      TMEM owner and tcgen05 issuer (one elected lane): S, dP of tile n, then
//               dV^T, dK^T of tile n - 1; after the block's last tile the states' MMAs
//   warps 2..5  thread = query row (TMEM lane) for P and dS (bf16 tiles in shared memory);
//               phi(K_j) in place once the block's S MMAs are done; in the epilogue thread
//               = channel (TMEM lane) for the rows of dK_j and dV_j
// TMEM columns: S / dP pairs [0,128) [128,256) (S at +0, dP at +64), dV^T [256,320),
// dK^T [320,384), A1 [384,448).
#pragma once

#include "sm100.cuh"

namespace sla {

struct BwdKVArgs {
  int BH, N, Nq, Nk;
  const int32_t* tlist;  // [BH*Nk, Nq] query tiles holding block j as critical, ascending
  const int32_t* tcnt;   // [BH*Nk]
  const float* lse;      // [BH, N] log-sum-exp of each row's critical scores (log2 units)
  const float* delta;    // [BH, N] rowsum(G_s * O_s)
  const float* dz;       // [BH*Nk, D] gradients of the z_j
  float* dK;             // [BH, N, D] written
  float* dV;             // [BH, N, D] written
  float scale_log2;      // log2(e) / sqrt(D)
  uint32_t* err;
};

struct BwdKVSmem {
  static constexpr uint32_t KV = 16384;    // K_j or V_j: 64 rows x 128 (two 64-column boxes)
  static constexpr int NSLOT = 5;          // ring slots
  static constexpr uint32_t SLOT = 32768;  // Q_i, G_s,i or dh_j: 128 rows x 128 (two 64-column boxes)
  static constexpr uint32_t PT = 16384;    // P or dS: 128 rows x 64 keys
  static constexpr uint32_t total() { return 2 * KV + NSLOT * SLOT + 2 * PT + 1024; }
};

__global__ void __launch_bounds__(192, 1)
    bwd_kv_kernel(const __grid_constant__ CUtensorMap map_q, const __grid_constant__ CUtensorMap map_g,
                  const __grid_constant__ CUtensorMap map_k, const __grid_constant__ CUtensorMap map_v,
                  const __grid_constant__ CUtensorMap map_dh, BwdKVArgs a) {
  using L = BwdKVSmem;
  constexpr int D = 128;
  constexpr uint32_t DV = 256, DK = 320, A1 = 384;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sK = base;
  uint8_t* sV = base + L::KV;
  uint8_t* sRing = base + 2 * L::KV;  // slot s at sRing + s * SLOT
  uint8_t* sP = sRing + L::NSLOT * L::SLOT;
  uint8_t* sdS = sP + L::PT;

  constexpr int NS = L::NSLOT;
  __shared__ uint64_t kv_full, kv_free, sl_full[NS], sl_empty[NS], s_full[2], ds_full, pds_free, phi_full, acc_full,
      tmem_free, drain;
  __shared__ uint32_t tmem_base_sh;
  __shared__ int abort_flag;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int n_blocks = a.BH * a.Nk;
  if (tid == 0) {
    mbar_init(&kv_full, 1);
    mbar_init(&kv_free, 1 + 128);  // the block's last MMA, and every thread's last read of phi(K_j)
    for (int s = 0; s < NS; ++s) {
      mbar_init(&sl_full[s], 1);
      mbar_init(&sl_empty[s], 1);
    }
    for (int s = 0; s < 2; ++s) mbar_init(&s_full[s], 1);
    mbar_init(&ds_full, 128);
    mbar_init(&pds_free, 1);
    mbar_init(&phi_full, 128);
    mbar_init(&acc_full, 1);
    mbar_init(&tmem_free, 128);
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
  grid_dep_wait();  // LSE, Delta, the tile lists and dh_j, dz_j come from earlier kernels

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      int kv_loads = 0, st_round[NS];
      for (int s = 0; s < NS; ++s) st_round[s] = -1;
      uint32_t ru = 0;  // ring uses: two per tile (Q_i, G_s,i), one per dh_j
      // wait for slot ru % NS to be free, then load `boxes` 128-row boxes of map into it
      auto load_slot = [&](const CUtensorMap* m, int boxes, int c_row, int c_z) -> bool {
        const int s = ru % NS, r = ru / NS;
        if (r > 0 && !mbar_wait(&sl_empty[s], (r - 1) & 1, a.err, &abort_flag)) return false;
        uint8_t* st = sRing + s * L::SLOT;
        mbar_arrive_expect_tx(&sl_full[s], boxes * 16384);
        for (int b = 0; b < boxes; ++b) tma_load_3d(st + b * 16384, m, &sl_full[s], b * 64, c_row, c_z);
        st_round[s] = r;
        ++ru;
        return true;
      };
      bool ok = true;
      int nkv = 0;
      for (int g = blockIdx.x; ok && g < n_blocks; g += gridDim.x, ++nkv) {
        const int bh = g / a.Nk, j = g % a.Nk;
        const int tc = a.tcnt[g];
        const int32_t* list = a.tlist + static_cast<size_t>(g) * a.Nq;
        if (nkv > 0 && !(ok = mbar_wait(&kv_free, (nkv - 1) & 1, a.err, &abort_flag))) break;
        mbar_arrive_expect_tx(&kv_full, 2 * L::KV);
        for (int b = 0; b < 2; ++b) {
          tma_load_3d(sK + b * 8192, &map_k, &kv_full, b * 64, j * 64, bh);
          tma_load_3d(sV + b * 8192, &map_v, &kv_full, b * 64, j * 64, bh);
        }
        ++kv_loads;
        for (int n = 0; ok && n < tc; ++n) {
          const int i = list[n];
          ok = load_slot(&map_q, 2, i * 128, bh) && load_slot(&map_g, 2, i * 128, bh);
        }
        if (ok) ok = load_slot(&map_dh, 2, 0, g);
      }
      if (abort_flag) {  // let every load still in flight land before the CTA retires
        if (kv_loads > 0) mbar_wait(&kv_full, (kv_loads - 1) & 1, nullptr, nullptr);
        for (int s = 0; s < NS; ++s)
          if (st_round[s] >= 0) mbar_wait(&sl_full[s], st_round[s] & 1, nullptr, nullptr);
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    const uint32_t id_s = idesc_bf16_f32(128, 64, 0, 0);    // A, B K-major, N = 64
    const uint32_t id_t = idesc_bf16_f32(128, 64, 1, 1);    // A, B MN-major, N = 64
    const uint32_t id_v = idesc_bf16_f32(128, 64, 1, 0);    // A MN-major, B K-major
    const uint32_t k0 = smem_u32(sK), v0 = smem_u32(sV), ring0 = smem_u32(sRing);
    const uint32_t p0 = smem_u32(sP), ds0 = smem_u32(sdS);
    uint32_t ru = 0, ns = 0;
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
    auto kmaj128 = [](uint32_t t0, int kk) { return smem_desc_sw128(t0 + (kk >> 2) * 16384 + (kk & 3) * 32, 16, 1024); };
    auto kmaj64 = [](uint32_t t0, int kk) { return smem_desc_sw128(t0 + (kk >> 2) * 8192 + (kk & 3) * 32, 16, 1024); };
    int nkv = 0;
    // dV^T += G^T P, dK^T += Q^T dS of the tile at ring use rum, S/P index nsm; `first` overwrites
    // the accumulators, which the previous block's epilogue must have read.
    auto issue_dvdk = [&](uint32_t rum, uint32_t nsm, bool first) -> bool {
      if (first && nkv > 0 && !wait_all(&tmem_free, (nkv - 1) & 1)) return false;
      if (!wait_all(&ds_full, nsm & 1)) return false;
      tc_fence_after();
      const uint32_t q0 = ring0 + (rum % NS) * L::SLOT, g0 = ring0 + ((rum + 1) % NS) * L::SLOT;
#pragma unroll
      for (int kk = 0; kk < 8; ++kk) {
        const uint32_t acc = (first && kk == 0) ? 0u : 1u;
        mma_ss(tmem + DV, smem_desc_sw128(g0 + kk * 2048, 16384, 1024), smem_desc_sw128(p0 + kk * 2048, 8192, 1024),
               id_t, acc);
        mma_ss(tmem + DK, smem_desc_sw128(q0 + kk * 2048, 16384, 1024), smem_desc_sw128(ds0 + kk * 2048, 8192, 1024),
               id_t, acc);
      }
      commit(&pds_free);
      commit(&sl_empty[rum % NS]);
      commit(&sl_empty[(rum + 1) % NS]);
      return true;
    };
    for (int g = blockIdx.x; ok && g < n_blocks; g += gridDim.x, ++nkv) {
      const int tc = a.tcnt[g];
      if (!(ok = wait_all(&kv_full, nkv & 1))) break;
      for (int n = 0; n < tc; ++n, ru += 2, ++ns) {
        const int sq = ru % NS, sg = (ru + 1) % NS, b = ns & 1;
        const uint32_t q0 = ring0 + sq * L::SLOT, g0 = ring0 + sg * L::SLOT;
        const uint32_t sd = tmem + b * 128;
        if (!(ok = wait_all(&sl_full[sq], (ru / NS) & 1))) break;
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) mma_ss(sd, kmaj128(q0, kk), kmaj64(k0, kk), id_s, kk > 0);
        if (!(ok = wait_all(&sl_full[sg], ((ru + 1) / NS) & 1))) break;
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) mma_ss(sd + 64, kmaj128(g0, kk), kmaj64(v0, kk), id_s, kk > 0);
        commit(&s_full[b]);
        if (n >= 1 && !(ok = issue_dvdk(ru - 2, ns - 1, n == 1))) break;
      }
      if (!ok) break;
      if (tc > 0 && !(ok = issue_dvdk(ru - 2, ns - 1, tc == 1))) break;
      // the states' part: dh_j in the next stage, phi(K_j) in place of K_j
      if (tc == 0 && nkv > 0 && !(ok = wait_all(&tmem_free, (nkv - 1) & 1))) break;
      const int s = ru % NS;
      if (!(ok = wait_all(&sl_full[s], (ru / NS) & 1))) break;
      if (!(ok = wait_all(&phi_full, nkv & 1))) break;
      tc_fence_after();
      const uint32_t h0 = ring0 + s * L::SLOT;
#pragma unroll
      for (int kk = 0; kk < D / 16; ++kk)  // dV^T += dh^T phi(K)^T: M = e, K = d, N = keys
        mma_ss(tmem + DV, smem_desc_sw128(h0 + kk * 2048, 16384, 1024), kmaj64(k0, kk), id_v,
               (tc > 0 || kk > 0) ? 1u : 0u);
#pragma unroll
      for (int kk = 0; kk < D / 16; ++kk)  // A1 = dh V^T: M = d, K = e, N = keys
        mma_ss(tmem + A1, kmaj128(h0, kk), kmaj64(v0, kk), id_s, kk > 0 ? 1u : 0u);
      commit(&acc_full);
      commit(&sl_empty[s]);
      commit(&kv_free);
      ++ru;
    }
    commit(&drain);  // every MMA issued above has finished once this arrives
    mbar_wait(&drain, 0, nullptr, nullptr);
  } else {
    // ------------------------------------------------------------ rows / channels (warps 2..5)
    const int quarter = warp & 3, r = quarter * 32 + lane, wt = tid - 64;
    const uint32_t lane_addr = tmem + (static_cast<uint32_t>(quarter * 32) << 16);
    const float sc = a.scale_log2;
    const float dsc = sc * 0.6931471805599453f;  // 1 / sqrt(D)
    const uint64_t sc2 = f2_make(sc, sc), dsc2 = f2_make(dsc, dsc);
    uint32_t ns = 0;
    bool ok = true;
    int nkv = 0;
    for (int g = blockIdx.x; g < n_blocks; g += gridDim.x, ++nkv) {
      const int bh = g / a.Nk, j = g % a.Nk;
      const int tc = a.tcnt[g];
      const int32_t* list = a.tlist + static_cast<size_t>(g) * a.Nq;
      const int valid = min(64, a.N - j * 64);  // valid keys of the block
      const float* lse_h = a.lse + static_cast<size_t>(bh) * a.N;
      const float* dl_h = a.delta + static_cast<size_t>(bh) * a.N;
      // this row's LSE and Delta loaded one tile ahead and the tile indices two ahead, so that no
      // load waits on another inside an iteration
      int tok = tc > 0 ? list[0] * 128 + r : a.N;
      int i_nn = tc > 1 ? list[1] : 0;
      float lse_n = tok < a.N ? lse_h[tok] : 0.f, dl_n = tok < a.N ? dl_h[tok] : 0.f;
      for (int n = 0; ok && n < tc; ++n, ++ns) {
        const int b = ns & 1;
        const bool row_ok = tok < a.N;
        const float lse = lse_n, dl = dl_n;
        const int i_nnn = n + 2 < tc ? list[n + 2] : 0;
        if (n + 1 < tc) {
          tok = i_nn * 128 + r;
          lse_n = tok < a.N ? lse_h[tok] : 0.f;
          dl_n = tok < a.N ? dl_h[tok] : 0.f;
        }
        i_nn = i_nnn;
        ok = __all_sync(0xffffffffu, mbar_wait(&s_full[b], (ns >> 1) & 1, a.err, &abort_flag));
        if (!ok) break;
        tc_fence_after();
        const uint64_t nl2 = f2_make(-lse, -lse), nd2 = f2_make(-dl, -dl);
        uint32_t pk[32], dk[32];
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
          uint32_t sx[32], dp[32];
          tmem_ld32(lane_addr + b * 128 + 32 * hh, sx);
          tmem_ld32(lane_addr + b * 128 + 64 + 32 * hh, dp);
          tmem_wait_ld();
#pragma unroll
          for (int c = 0; c < 32; c += 2) {
            const int n0 = 32 * hh + c;
            const uint64_t x2 = f2_fma(static_cast<uint64_t>(sx[c]) | (static_cast<uint64_t>(sx[c + 1]) << 32), sc2, nl2);
            const float p0 = (row_ok && n0 < valid) ? fast_exp2(f2_lo(x2)) : 0.f;
            const float p1 = (row_ok && n0 + 1 < valid) ? fast_exp2(f2_hi(x2)) : 0.f;
            pk[16 * hh + (c >> 1)] = pack_bf16x2(p0, p1);
            const uint64_t d2 = f2_add(static_cast<uint64_t>(dp[c]) | (static_cast<uint64_t>(dp[c + 1]) << 32), nd2);
            const uint64_t g2 = f2_mul(f2_mul(f2_make(p0, p1), dsc2), d2);
            dk[16 * hh + (c >> 1)] = pack_bf16x2(f2_lo(g2), f2_hi(g2));
          }
        }
        // P and dS may overwrite their tiles once the previous tile's dV^T, dK^T MMAs are done
        if (ns > 0) ok = __all_sync(0xffffffffu, mbar_wait(&pds_free, (ns - 1) & 1, a.err, &abort_flag));
        if (!ok) break;
#pragma unroll
        for (int v = 0; v < 8; ++v) {
          const uint32_t off = sw128_offset(r, v * 16);
          *reinterpret_cast<uint4*>(sP + off) = make_uint4(pk[4 * v], pk[4 * v + 1], pk[4 * v + 2], pk[4 * v + 3]);
          *reinterpret_cast<uint4*>(sdS + off) = make_uint4(dk[4 * v], dk[4 * v + 1], dk[4 * v + 2], dk[4 * v + 3]);
        }
        fence_proxy_async_smem();
        tc_fence_before();
        mbar_arrive(&ds_full);
      }
      // phi(K_j) in place: every S MMA of the block has finished (the last s_full above; with no
      // tile, K_j must have landed). Rows past the sequence end become 0.
      if (ok) ok = __all_sync(0xffffffffu, mbar_wait(&kv_full, nkv & 1, a.err, &abort_flag));
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
      if (!(ok = named_barrier_and(1, 128, ok))) break;  // every phi(k) written
      mbar_arrive(&phi_full);
      // epilogue: thread = channel c = TMEM lane; rows n of the block. phi'(k) of this channel
      // is taken out of shared memory first (phi' = min(phi, 1), exact in bf16), so K_j's buffer
      // is released before the stores and the next block's K_j, V_j load under them.
      const int c = r;
      const float dzc = a.dz[static_cast<size_t>(g) * D + c];
      ok = __all_sync(0xffffffffu, mbar_wait(&acc_full, nkv & 1, a.err, &abort_flag));
      // phi'(k) of keys 2m (low half) and 2m + 1 (high half), bf16: keys 0..31 in pd0, 32..63 in pd1
      uint32_t pd0[16], pd1[16];
      if (ok) {
        const uint8_t* col = sK + (c >> 6) * 8192 + (c & 7) * 2;
        auto dphi2 = [&](int m) {
          const uint16_t f0 = *reinterpret_cast<const uint16_t*>(col + sw128_offset(2 * m, ((c & 63) >> 3) * 16));
          const uint16_t f1 = *reinterpret_cast<const uint16_t*>(col + sw128_offset(2 * m + 1, ((c & 63) >> 3) * 16));
          return pack_bf16x2(fminf(__uint_as_float(static_cast<uint32_t>(f0) << 16), 1.f),
                             fminf(__uint_as_float(static_cast<uint32_t>(f1) << 16), 1.f));
        };
#pragma unroll
        for (int m = 0; m < 16; ++m) {
          pd0[m] = dphi2(m);
          pd1[m] = dphi2(16 + m);
        }
      }
      mbar_arrive(&kv_free);  // phi(K_j) read for the last time
      if (ok) {
        tc_fence_after();
        const size_t row0 = static_cast<size_t>(bh) * a.N + static_cast<size_t>(j) * 64;
#pragma unroll 1
        for (int hh = 0; hh < 2; ++hh) {
          uint32_t dv[32], dkt[32], a1[32];
          tmem_ld32(lane_addr + DV + 32 * hh, dv);
          tmem_ld32(lane_addr + DK + 32 * hh, dkt);
          tmem_ld32(lane_addr + A1 + 32 * hh, a1);
          tmem_wait_ld();
#pragma unroll
          for (int n2 = 0; n2 < 32; ++n2) {
            const int n = 32 * hh + n2;
            if (n < valid) {
              const size_t o = (row0 + n) * D + c;
              const uint32_t pw = hh ? pd1[n2 >> 1] : pd0[n2 >> 1];
              const float dphi = __uint_as_float((n & 1) ? (pw & 0xFFFF0000u) : (pw << 16));
              const float dks = tc > 0 ? __uint_as_float(dkt[n2]) : 0.f;
              a.dV[o] = __uint_as_float(dv[n2]);
              a.dK[o] = dks + (__uint_as_float(a1[n2]) + dzc) * dphi;
            }
          }
        }
      }
      tc_fence_before();
      mbar_arrive(&tmem_free);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

}  // namespace sla
