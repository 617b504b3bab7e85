// Fused SLA attention with a low-bit (e4m3) sparse branch, D = 128. Same tile, blend and
// linear branch as attn_kernel; the two matmuls of the sparse branch take e4m3 operands:
//
//   S   = Q8 K8_j^T  (tcgen05 kind::f8f6f4, K = 32 per instruction: 4 MMAs per block)
//   O_s += P8 V8_j   (P8 from TMEM, V8 MN-major: 2 MMAs per block)
//
// Sources: "SLA2: Sparse-Linear Attention with Learnable Routing and QAT", §2.C (low-bit
// sparse branch in the forward pass), §1 item 1 and §2.A (renormalised sparse branch,
// alpha blend); "SLA: Beyond Sparsity in Diffusion Transformers via Fine-Tunable
// Sparse-Linear Attention", Abstract (critical / marginal / negligible split, one kernel).
//
// Quantisation (the pages fix no format):
//   Q   per query block: the softmax warpgroup reduces the bf16 tile's amax, picks
//       2^eq with amax / 2^eq in (128, 256] and writes the e4m3 tile next to the bf16 one
//       (which stays for phi(Q) in the linear branch);
//   K,V per KV block: codes and exponents come from quant_kv_kernel;
//   P   coded as e4m3 against a per-row reference r (log2 units). Any r at or below the
//       row maximum that saturates no code gives a valid result; this kernel starts r at
//       the first block's row maximum and moves it to a later block's maximum only when
//       that exceeds r by more than kP8Slack = 8 (so O is rescaled rarely, as in
//       attn_kernel). r is always some block's maximum, so r <= the row maximum, and a key
//       of block j contributes e4m3(2^(x - r) * 2^(ev_j - ev_max)) <= 256 < 448 with ev_max
//       the largest V exponent of the tile's critical blocks; the normaliser l sums the
//       unquantised 2^(x - r).
//   O_s = 2^c acc / l with c = ev_max - kP8RefExp.
//
// The linear branch shares the sparse branch's accumulator as in attn_kernel: with H~_i =
// H_i diag((1 - alpha) / alpha) from the aggregation,
//     O = alpha (2^c acc / l + phi(q) H~_i / den) = alpha 2^c (acc + (l 2^-c / den) phi(q) H~_i) / l,
// so the warpgroup writes P_lin = (l 2^-c / den) phi(q) (bf16) into TMEM and one bf16 MMA
// adds P_lin H~_i into acc; with no critical block l = 1 and c = 0.
//
// Persistent, two CTAs per SM (<= 100 KB shared memory, 256 TMEM columns each). Warp roles
// (192 threads):
//   warp 0      TMA producer: per tile the bf16 Q tile, then K8_j / V8_j of every critical
//               block through a 3-slot ring, then H~_i as two pseudo-blocks (rows 0..63 and
//               64..127, each filling a whole slot). The next tile's Q is loaded once the
//               warpgroup has read this one for phi(q).
//   warp 1      TMEM owner and single-thread tcgen05 issuer.
//   warps 2..5  softmax / epilogue warpgroup: a thread owns one query row (= TMEM lane).
//               The output is staged in the two H~_i slots and written by TMA stores; the
//               slots return to the ring when the stores have read them (next tile).
//
// TMEM columns: S ping-pong [0,64) [64,128) (P8, 16 columns, is written over the first
// columns of its S), acc [128,256); after the sparse loop P_lin (64 columns) takes the S
// columns the next block would have used.
#pragma once

#include "attention.cuh"
#include "fp8.cuh"

namespace sla {

constexpr int kP8RefExp = 0;       // P is quantised at 2^0 times its value
constexpr float kP8Slack = 8.f;    // log2 units a block maximum may pass the reference

struct AttnFp8Args {
  int H, N, Nq, Nk, block_q, n_tiles;
  const int32_t* crit;      // [BH*Nq, crit_ld] critical KV block indices, ascending
  int crit_ld;
  const int32_t* crit_cnt;  // [BH*Nq]
  const int32_t* kexp;      // [BH, Nk] K block scale exponents
  const int32_t* vexp;      // [BH, Nk] V block scale exponents
  const float* Zagg;        // [BH*Nq, 128]
  const float* alpha;       // [H, 128]
  __nv_bfloat16* out;       // [BH, N, 128]
  float scale_log2;         // log2(e) / sqrt(D)
  uint32_t* err;
};

struct AttnFp8Smem {
  static constexpr uint32_t QB = 128 * 128 * 2;   // bf16 Q tile (phi(Q) at the end of a tile)
  static constexpr uint32_t Q8 = 128 * 128;       // e4m3 Q tile
  static constexpr uint32_t KV = 64 * 128;        // one K8 or V8 block
  static constexpr uint32_t SLOT = 2 * KV;        // K8 then V8, or one half of H_i (64 x 128 bf16)
  static constexpr int NSLOT = 3;
  static constexpr uint32_t total() { return QB + Q8 + NSLOT * SLOT + 1024; }
};

__global__ void __launch_bounds__(192, 2)
    attn_fp8_kernel(const __grid_constant__ CUtensorMap map_q, const __grid_constant__ CUtensorMap map_k8,
                    const __grid_constant__ CUtensorMap map_v8, const __grid_constant__ CUtensorMap map_h,
                    const __grid_constant__ CUtensorMap map_o, AttnFp8Args a) {
  using L = AttnFp8Smem;
  constexpr int D = 128;
  constexpr int NS = L::NSLOT;
  constexpr uint32_t TMEM_COLS = 256;
  constexpr uint32_t OS = 128;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sQb = base;
  uint8_t* sQ8 = sQb + L::QB;
  uint8_t* sRing = sQ8 + L::Q8;  // slot s at sRing + s * SLOT: K8 at +0, V8 at +KV

  __shared__ uint64_t q_full, q8_full, q_free, plin_full, lin_done, tmem_free, drain;
  __shared__ uint64_t k_full[NS], k_empty[NS], v_full[NS], v_empty[NS];
  __shared__ uint64_t s_full[2], p_full[2], pv_done[2];
  __shared__ uint32_t tmem_base_sh;
  __shared__ int abort_flag;
  __shared__ uint32_t sQmax[2];  // bf16 magnitude bits of the Q tile's amax (by tile parity)
  __shared__ int sVmax[2];       // largest V exponent over the tile's critical blocks (by tile parity)
  __shared__ __align__(16) float sZ[D];
  __shared__ __align__(16) float sAlpha[D];

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

  if (tid == 0) {
    mbar_init(&q_full, 1);
    mbar_init(&q8_full, 128);
    mbar_init(&q_free, 128);     // every row read for phi(q)
    mbar_init(&plin_full, 128);
    mbar_init(&lin_done, 1);
    mbar_init(&tmem_free, 128);
    mbar_init(&drain, 1);
    for (int s = 0; s < NS; ++s) {
      mbar_init(&k_full[s], 1);
      mbar_init(&k_empty[s], 1);
      mbar_init(&v_full[s], 1);
      mbar_init(&v_empty[s], 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(&s_full[s], 1);
      mbar_init(&p_full[s], 128);
      mbar_init(&pv_done[s], 1);
    }
    abort_flag = 0;
    sQmax[0] = sQmax[1] = 0u;
    sVmax[0] = sVmax[1] = -1000000;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(&tmem_base_sh, TMEM_COLS);
    tmem_relinquish();
  }
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_base_sh;
  grid_dep_wait();  // critical lists, H~_i, Z_i and the K/V codes come from earlier kernels

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      prefetch_tmap(&map_q);
      prefetch_tmap(&map_k8);
      prefetch_tmap(&map_v8);
      prefetch_tmap(&map_h);
      prefetch_tmap(&map_o);
      int k_round[NS], v_round[NS];
      for (int s = 0; s < NS; ++s) k_round[s] = v_round[s] = -1;
      int q_loads = 0;
      uint32_t nb = 0;  // ring uses so far (K/V blocks and H_i halves)
      bool ok = true;
      int k = 0;
      for (int t = blockIdx.x; ok && t < a.n_tiles; t += gridDim.x, ++k) {
        const int bh = t / a.Nq, i = t % a.Nq;
        const int kc = a.crit_cnt[t];
        const int32_t* clist = a.crit + static_cast<size_t>(t) * a.crit_ld;
        if (k > 0 && !(ok = mbar_wait(&q_free, (k - 1) & 1, a.err, &abort_flag))) break;
        mbar_arrive_expect_tx(&q_full, L::QB);
        for (int b = 0; b < 2; ++b) tma_load_3d(sQb + b * 16384, &map_q, &q_full, b * 64, i * a.block_q, bh);
        ++q_loads;
        for (int n = 0; n < kc + 2; ++n, ++nb) {  // n >= kc: the two halves of H_i
          const int s = static_cast<int>(nb % NS), r = static_cast<int>(nb / NS);
          uint8_t* slot = sRing + s * L::SLOT;
          if (r > 0 && !(ok = mbar_wait(&k_empty[s], (r - 1) & 1, a.err, &abort_flag))) break;
          if (n < kc) {
            // K8 refills as soon as S of the slot's previous block is done, V8 once P*V is
            const int j = clist[n];
            mbar_arrive_expect_tx(&k_full[s], L::KV);
            tma_load_3d(slot, &map_k8, &k_full[s], 0, j * 64, bh);
            k_round[s] = r;
            if (r > 0 && !(ok = mbar_wait(&v_empty[s], (r - 1) & 1, a.err, &abort_flag))) break;
            mbar_arrive_expect_tx(&v_full[s], L::KV);
            tma_load_3d(slot + L::KV, &map_v8, &v_full[s], 0, j * 64, bh);
            v_round[s] = r;
          } else {
            // an H_i half spans the whole slot: both halves of the slot must be free
            if (r > 0 && !(ok = mbar_wait(&v_empty[s], (r - 1) & 1, a.err, &abort_flag))) break;
            const int e = n - kc;
            mbar_arrive_expect_tx(&k_full[s], L::SLOT);
            for (int c = 0; c < 2; ++c) tma_load_2d(slot + c * 8192, &map_h, &k_full[s], c * 64, t * D + e * 64);
            k_round[s] = r;
            mbar_arrive(&v_full[s]);
            v_round[s] = r;
          }
        }
      }
      if (abort_flag) {  // let every load still in flight land before the CTA retires
        if (q_loads > 0) mbar_wait(&q_full, (q_loads - 1) & 1, nullptr, nullptr);
        for (int s = 0; s < NS; ++s) {
          if (k_round[s] >= 0) mbar_wait(&k_full[s], k_round[s] & 1, nullptr, nullptr);
          if (v_round[s] >= 0) mbar_wait(&v_full[s], v_round[s] & 1, nullptr, nullptr);
        }
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      const uint32_t id_s = idesc_e4m3_f32(128, 64, 0, 0);
      const uint32_t id_pv = idesc_e4m3_f32(128, D, 0, 1);
      const uint32_t id_ol = idesc_bf16_f32(128, D, 0, 1);
      const uint32_t q80 = smem_u32(sQ8), ring0 = smem_u32(sRing);
      uint32_t nb = 0, ns = 0;  // ring uses, S/P blocks
      bool ok = true;
      int k = 0;
      // P*V of the block at ring use nbm, S/P index nsm; `first` overwrites acc, which the
      // previous tile's epilogue must have read (tile k > 0). V8 is MN-major: rows of 128
      // codes (one swizzle atom wide), K = 32 rows = 4096 bytes a step.
      auto issue_pv = [&](uint32_t nbm, uint32_t nsm, bool first) -> bool {
        const int s = static_cast<int>(nbm % NS), b = nsm & 1;
        if (first && k > 0 && !mbar_wait(&tmem_free, (k - 1) & 1, a.err, &abort_flag)) return false;
        if (!mbar_wait(&p_full[b], (nsm >> 1) & 1, a.err, &abort_flag)) return false;
        if (!mbar_wait(&v_full[s], (nbm / NS) & 1, a.err, &abort_flag)) return false;
        tc_fence_after();
        const uint32_t vb = ring0 + s * L::SLOT + L::KV;
#pragma unroll
        for (int kk = 0; kk < 2; ++kk) {
          const uint64_t bd = smem_desc_sw128(vb + kk * 4096, 8192, 1024);
          umma_e4m3_ts(tmem + OS, tmem + b * 64 + kk * 8, bd, id_pv, (first && kk == 0) ? 0u : 1u);
        }
        umma_commit(&pv_done[b]);
        umma_commit(&v_empty[s]);
        return true;
      };
      for (int t = blockIdx.x; ok && t < a.n_tiles; t += gridDim.x, ++k) {
        const int kc = a.crit_cnt[t];
        // the warpgroup has written this tile's e4m3 Q
        if (!(ok = mbar_wait(&q8_full, k & 1, a.err, &abort_flag))) break;
        for (int n = 0; n < kc; ++n, ++nb, ++ns) {
          const int s = static_cast<int>(nb % NS), b = ns & 1;
          if (!(ok = mbar_wait(&k_full[s], (nb / NS) & 1, a.err, &abort_flag))) break;
          tc_fence_after();
          const uint32_t kb = ring0 + s * L::SLOT;
#pragma unroll
          for (int kk = 0; kk < D / 32; ++kk) {
            const uint64_t ad = smem_desc_sw128(q80 + kk * 32, 16, 1024);
            const uint64_t bd = smem_desc_sw128(kb + kk * 32, 16, 1024);
            umma_e4m3_ss(tmem + b * 64, ad, bd, id_s, kk > 0 ? 1u : 0u);
          }
          umma_commit(&s_full[b]);
          umma_commit(&k_empty[s]);
          if (n >= 1 && !(ok = issue_pv(nb - 1, ns - 1, n == 1))) break;
        }
        if (!ok) break;
        if (kc > 0 && !(ok = issue_pv(nb - 1, ns - 1, kc == 1))) break;
        // Linear branch, added into the sparse accumulator: acc += P_lin H~_i, P_lin written
        // by the warpgroup into the S columns after the last block (ns & 1), H~_i in two ring
        // slots (rows 0..63, 64..127). With no critical block this is the first write of acc.
        // The slots are released by the warpgroup once the output staged there is stored.
        const int s0 = static_cast<int>(nb % NS), s1 = static_cast<int>((nb + 1) % NS);
        if (kc == 0 && k > 0 && !(ok = mbar_wait(&tmem_free, (k - 1) & 1, a.err, &abort_flag))) break;
        if (!(ok = mbar_wait(&k_full[s0], (nb / NS) & 1, a.err, &abort_flag))) break;
        if (!(ok = mbar_wait(&v_full[s0], (nb / NS) & 1, a.err, &abort_flag))) break;
        if (!(ok = mbar_wait(&k_full[s1], ((nb + 1) / NS) & 1, a.err, &abort_flag))) break;
        if (!(ok = mbar_wait(&v_full[s1], ((nb + 1) / NS) & 1, a.err, &abort_flag))) break;
        if (!(ok = mbar_wait(&plin_full, k & 1, a.err, &abort_flag))) break;
        tc_fence_after();
        const uint32_t pl = tmem + (ns & 1) * 64;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t hb = ring0 + (kk < 4 ? s0 : s1) * L::SLOT;
          const uint64_t bd = smem_desc_sw128(hb + (kk & 3) * 2048, 8192, 1024);
          umma_bf16_ts(tmem + OS, pl + kk * 8, bd, id_ol, (kc > 0 || kk > 0) ? 1u : 0u);
        }
        umma_commit(&lin_done);
        nb += 2;
      }
      umma_commit(&drain);  // every MMA issued above has finished once this arrives
      mbar_wait(&drain, 0, nullptr, nullptr);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ softmax / epilogue warpgroup
    const int quarter = warp & 3;               // TMEM lane quarter this warp may access
    const int r = quarter * 32 + lane;          // query row within the tile
    const int wt = tid - 64;                    // 0..127
    const uint32_t lane_addr = tmem + (static_cast<uint32_t>(quarter * 32) << 16);
    uint32_t ns = 0;   // S/P blocks so far
    uint32_t nbw = 0;  // ring uses so far (K/V blocks and H~_i halves)
    int rel0 = -1, rel1 = -1;  // (thread 0 of the warpgroup) ring slots still held by an output store
    bool ok = true;
    int k = 0;
    // Every barrier of the warpgroup ANDs the threads' status, so a failed wait makes all
    // 128 threads leave together.
    for (int t = blockIdx.x; t < a.n_tiles; t += gridDim.x, ++k) {
      const int bh = t / a.Nq, i = t % a.Nq, h = bh % a.H;
      const int kc = a.crit_cnt[t];
      // the ring slots of this tile's H~_i halves, reused to stage O
      const int hs0 = static_cast<int>((nbw + kc) % NS), hs1 = static_cast<int>((nbw + kc + 1) % NS);
      nbw += kc + 2;
      const int32_t* clist = a.crit + static_cast<size_t>(t) * a.crit_ld;
      const int32_t* kexp = a.kexp + static_cast<size_t>(bh) * a.Nk;
      const int32_t* vexp = a.vexp + static_cast<size_t>(bh) * a.Nk;
      const int tok = i * a.block_q + r;
      const bool row_valid = r < a.block_q && tok < a.N;
      // The previous tile is done with sZ, sAlpha and the parity-(k+1) reduction slots.
      if (!named_barrier_and(1, 128, ok)) break;
      // The previous tile's output has been read out of its two slots once this thread's bulk
      // group is done reading: the slots may take K8/V8 blocks again.
      if (rel0 >= 0) {
        tma_store_wait_read();
        mbar_arrive(&k_empty[rel0]);
        mbar_arrive(&v_empty[rel0]);
        mbar_arrive(&k_empty[rel1]);
        mbar_arrive(&v_empty[rel1]);
        rel0 = rel1 = -1;
      }
      const int par = k & 1;
      if (wt == 0) {
        sQmax[par ^ 1] = 0u;
        sVmax[par ^ 1] = -1000000;
      }
      // global loads first, so their latency overlaps the wait for Q and the amax pass
      const float z_in = a.Zagg[static_cast<size_t>(t) * D + wt];
      const float al_in = a.alpha[h * D + wt];
      int vmax_l = -1000000;
      for (int n = wt; n < kc; n += 128) vmax_l = max(vmax_l, vexp[clist[n]]);
      // the Q tile's amax over the valid rows
      ok = ok && __all_sync(0xffffffffu, mbar_wait(&q_full, k & 1, a.err, &abort_flag));
      uint32_t qm = 0;
      if (ok && row_valid) {
#pragma unroll
        for (int c = 0; c < 16; ++c) {
          const uint4 u = *reinterpret_cast<const uint4*>(sQb + (c >> 3) * 16384 + sw128_offset(r, (c & 7) * 16));
          qm = max(qm, max(max(bf16x2_absmax_bits(u.x), bf16x2_absmax_bits(u.y)),
                           max(bf16x2_absmax_bits(u.z), bf16x2_absmax_bits(u.w))));
        }
      }
      qm = __reduce_max_sync(0xffffffffu, qm);
      vmax_l = __reduce_max_sync(0xffffffffu, vmax_l);
      if (lane == 0) {
        atomicMax(&sQmax[par], qm);
        if (kc > 0) atomicMax(&sVmax[par], vmax_l);
      }
      sZ[wt] = z_in;
      sAlpha[wt] = fmaxf(al_in, kAlphaFloor);  // H~_i was scaled with the same floor
      if (!named_barrier_and(1, 128, ok)) break;
      const int eq = pow2_scale_exp(__uint_as_float(sQmax[par] << 16));
      const int vmax = sVmax[par];
      // this row's e4m3 codes: chunk c (16 codes, d = 16c .. 16c+15) at its swizzled place
#pragma unroll 2
      for (int c = 0; c < 8; ++c) {
        uint4 o = make_uint4(0, 0, 0, 0);
        if (row_valid) {
          const uint8_t* src = sQb + (c >> 2) * 16384;
          const uint4 u0 = *reinterpret_cast<const uint4*>(src + sw128_offset(r, (c & 3) * 32));
          const uint4 u1 = *reinterpret_cast<const uint4*>(src + sw128_offset(r, (c & 3) * 32 + 16));
          const uint32_t w[8] = {u0.x, u0.y, u0.z, u0.w, u1.x, u1.y, u1.z, u1.w};
          uint32_t pk[4];
#pragma unroll
          for (int e = 0; e < 4; ++e)
            pk[e] = pack_e4m3x4(mul_pow2(__uint_as_float(w[2 * e] << 16), -eq),
                                mul_pow2(__uint_as_float(w[2 * e] & 0xFFFF0000u), -eq),
                                mul_pow2(__uint_as_float(w[2 * e + 1] << 16), -eq),
                                mul_pow2(__uint_as_float(w[2 * e + 1] & 0xFFFF0000u), -eq));
          o = make_uint4(pk[0], pk[1], pk[2], pk[3]);
        }
        *reinterpret_cast<uint4*>(sQ8 + r * 128 + ((c ^ (r & 7)) << 4)) = o;
      }
      fence_proxy_async_smem();
      mbar_arrive(&q8_full);

      float m_run = -INFINITY, l_run = 0.f;  // reference (log2 units) and row sum
      uint32_t sa[32], sb[32];               // S columns [0, 32) and [32, 64) of the current block
      // block indices run two blocks ahead of their exponents, so no load waits on another
      // inside an iteration
      int j_cur = kc > 0 ? clist[0] : 0;
      int j_nxt = kc > 1 ? clist[1] : 0;
      int ek_cur = kc > 0 ? kexp[j_cur] : 0, ev_cur = kc > 0 ? vexp[j_cur] : 0;
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
        const int j_nn = n + 2 < kc ? clist[n + 2] : 0;
        const int ek_next = n + 1 < kc ? kexp[j_nxt] : 0, ev_next = n + 1 < kc ? vexp[j_nxt] : 0;
        const float sc = mul_pow2(a.scale_log2, eq + ek_cur);  // raw S -> log2 units
        const int pe = kP8RefExp + ev_cur - vmax;             // P is quantised at 2^pe
        const int valid = min(64, a.N - j_cur * 64);           // valid key columns of this block
        if (valid < 64) {
#pragma unroll
          for (int c = 0; c < 32; ++c) {
            if (c >= valid) sa[c] = __float_as_uint(-INFINITY);
            if (c + 32 >= valid) sb[c] = __float_as_uint(-INFINITY);
          }
        }
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
        } else {
          // Per row: the reference moves to this block's maximum only past the slack; the
          // warp rescales the rows that moved (factor 1 for the others).
          const bool move = mx > m_run + kP8Slack;
          if (__any_sync(0xffffffffu, move)) {
            ok = __all_sync(0xffffffffu,
                            mbar_wait(&pv_done[(ns - 1) & 1], ((ns - 1) >> 1) & 1, a.err, &abort_flag));
            if (!ok) break;
            tc_fence_after();
            const float f = move ? fast_exp2(m_run - mx) : 1.f;
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
            if (move) m_run = mx;
          }
        }
        // e = 2^(s * sc - m + pe) = 2^pe * P: one paired FMA per two elements, one
        // exponential per element; the block's sum is brought back to P units by 2^-pe.
        const float shift = static_cast<float>(pe) - m_run;
        const uint64_t sc2 = f2_make(sc, sc), sh2 = f2_make(shift, shift);
        uint64_t ps2 = 0ull, ps2b = 0ull;
        uint32_t pk[16];
#pragma unroll
        for (int c = 0; c < 32; c += 4) {
          const uint64_t x01 = f2_fma(static_cast<uint64_t>(sa[c]) | (static_cast<uint64_t>(sa[c + 1]) << 32), sc2, sh2);
          const uint64_t x23 = f2_fma(static_cast<uint64_t>(sa[c + 2]) | (static_cast<uint64_t>(sa[c + 3]) << 32), sc2, sh2);
          const uint64_t y01 = f2_fma(static_cast<uint64_t>(sb[c]) | (static_cast<uint64_t>(sb[c + 1]) << 32), sc2, sh2);
          const uint64_t y23 = f2_fma(static_cast<uint64_t>(sb[c + 2]) | (static_cast<uint64_t>(sb[c + 3]) << 32), sc2, sh2);
          const float e0 = fast_exp2(f2_lo(x01)), e1 = fast_exp2(f2_hi(x01));
          const float e2 = fast_exp2(f2_lo(x23)), e3 = fast_exp2(f2_hi(x23));
          const float g0 = fast_exp2(f2_lo(y01)), g1 = fast_exp2(f2_hi(y01));
          const float g2 = fast_exp2(f2_lo(y23)), g3 = fast_exp2(f2_hi(y23));
          ps2 = f2_add(ps2, f2_add(f2_make(e0, e1), f2_make(e2, e3)));
          ps2b = f2_add(ps2b, f2_add(f2_make(g0, g1), f2_make(g2, g3)));
          pk[c >> 2] = pack_e4m3x4(e0, e1, e2, e3);
          pk[8 + (c >> 2)] = pack_e4m3x4(g0, g1, g2, g3);
        }
        const uint64_t pst = f2_add(ps2, ps2b);
        l_run += mul_pow2(f2_lo(pst) + f2_hi(pst), -pe);
        tmem_st16(lane_addr + b * 64, pk);  // P8 over the first 16 columns of its S
        // P_n is published before S_{n+1} is waited for (see attn_kernel)
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
        j_cur = j_nxt;
        j_nxt = j_nn;
        ek_cur = ek_next;
        ev_cur = ev_next;
      }
      // Linear branch. P_lin goes into the S columns the next block would have used
      // (ns & 1); their last reader is the P*V two blocks back (with one block or none, an
      // MMA of an earlier tile, finished before that tile's lin_done was seen).
      if (ok && kc >= 2)
        ok = __all_sync(0xffffffffu, mbar_wait(&pv_done[(ns - 2) & 1], ((ns - 2) >> 1) & 1, a.err, &abort_flag));
      // Pass 1: phi(q) (bf16, as the tensor core takes it) into the P_lin columns, 32 elements
      // at a time, and den = phi(q) . Z_i from those rounded values; then the bf16 Q tile is
      // released (the next tile's Q may land).
      const uint32_t pl = lane_addr + (ns & 1) * 64;
      uint64_t den2 = 0ull;
      if (ok) {
        const uint64_t one2 = f2_make(1.f, 1.f), log2e2 = f2_make(1.4426950408889634f, 1.4426950408889634f);
#pragma unroll 1
        for (int g = 0; g < D / 32; ++g) {
          uint32_t w[16];
#pragma unroll
          for (int c = 0; c < 4; ++c) {
            const int c8 = 4 * g + c;
            const uint4 u = *reinterpret_cast<const uint4*>(sQb + (c8 >> 3) * 16384 + sw128_offset(r, (c8 & 7) * 16));
            w[4 * c] = u.x;
            w[4 * c + 1] = u.y;
            w[4 * c + 2] = u.z;
            w[4 * c + 3] = u.w;
          }
#pragma unroll
          for (int e = 0; e < 16; ++e) {
            const uint64_t x2 = static_cast<uint64_t>(w[e] << 16) | (static_cast<uint64_t>(w[e] & 0xFFFF0000u) << 32);
            const uint64_t pos2 = f2_add(x2, one2);
            const uint64_t t2 = f2_mul(x2, log2e2);
            const float g0 = f2_lo(x2) > 0.f ? f2_lo(pos2) : fast_exp2(f2_lo(t2));
            const float g1 = f2_hi(x2) > 0.f ? f2_hi(pos2) : fast_exp2(f2_hi(t2));
            w[e] = pack_bf16x2(g0, g1);
            const uint64_t gr2 = static_cast<uint64_t>(w[e] << 16) | (static_cast<uint64_t>(w[e] & 0xFFFF0000u) << 32);
            den2 = f2_fma(gr2, *reinterpret_cast<const uint64_t*>(&sZ[32 * g + 2 * e]), den2);
          }
          tmem_st16(pl + 16 * g, w);
        }
      }
      mbar_arrive(&q_free);
      // With no critical block l is taken as 1 and c as 0 (acc starts at 0); with no marginal
      // block (den = 0) the linear term is 0.
      const float den_tot = f2_lo(den2) + f2_hi(den2);
      const int cexp = kc > 0 ? vmax - kP8RefExp : 0;
      const float l_eff = kc > 0 ? l_run : 1.f;
      const float c_lin = den_tot > 0.f ? mul_pow2(l_eff, -cexp) / den_tot : 0.f;
      // Pass 2: P_lin = (l 2^-c / den) phi(q), rounded to bf16 in place.
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
      tc_fence_before();
      mbar_arrive(&plin_full);
      if (ok) ok = __all_sync(0xffffffffu, mbar_wait(&lin_done, k & 1, a.err, &abort_flag));
      if (!(ok = named_barrier_and(1, 128, ok))) break;

      // Epilogue: O = alpha 2^c acc / l in bf16, staged row by row in the two H~_i slots (the
      // linear MMA has read them; columns 0..63 in the first, 64..127 in the second) in the
      // 128-byte swizzle and written by TMA stores of block_q rows (rows past N are clipped by
      // the tensor map; with block_q = 64 the upper 64 rows belong to the next query block).
      tc_fence_after();
      const float inv_l = mul_pow2(1.f / l_eff, cexp);
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
        uint8_t* box = sRing + ((q >> 1) == 0 ? hs0 : hs1) * L::SLOT;
#pragma unroll
        for (int v = 0; v < 4; ++v)
          *reinterpret_cast<uint4*>(box + sw128_offset(r, ((q & 1) * 4 + v) * 16)) =
              make_uint4(pk[4 * v], pk[4 * v + 1], pk[4 * v + 2], pk[4 * v + 3]);
        if (q + 1 < D / 32) tmem_wait_ld();
      }
      fence_proxy_async_smem();
      named_barrier(1, 128);
      if (wt == 0) {
        tma_store_3d(&map_o, sRing + hs0 * L::SLOT, 0, i * a.block_q, bh);
        tma_store_3d(&map_o, sRing + hs1 * L::SLOT, 64, i * a.block_q, bh);
        tma_store_commit();
        rel0 = hs0;  // released at the next tile's start (see there)
        rel1 = hs1;
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
