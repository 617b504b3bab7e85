/*
 * sla.h - C ABI of the B200 (sm_100a) sparse-plus-linear block attention forward.
 *
 * The method: "SLA: Beyond Sparsity in Diffusion Transformers via Fine-Tunable
 * Sparse-Linear Attention" (Abstract) splits attention weights into critical
 * (exact softmax attention), marginal (linear attention) and negligible
 * (skipped) parts at block granularity; "SLA2: Sparse-Linear Attention with
 * Learnable Routing and QAT" (§2.A) blends the two branch outputs as
 *     O = alpha * O_s + (1 - alpha) * O_l,
 * with a router (§2.B) that pools adjacent Q and K tokens and keeps a hard
 * top-k at inference.
 *
 * What this library computes, per batch b, head h and query block i
 * (block_q query tokens) against KV blocks j (block_kv = 64 tokens):
 *   qbar_i, kbar_j  mean of the valid tokens of the block (fp64)
 *   S_ij            qbar_i . kbar_j / sqrt(D)
 *   labels          per row i, total order (S desc, j asc): first kc blocks
 *                   critical (2), last kn negligible (0), the rest marginal (1);
 *                   kc = ceil(kh_ppm * Nk / 1e6), kn = floor(kl_ppm * Nk / 1e6),
 *                   kh_ppm = round(kh * 1e6), kl_ppm = round(kl * 1e6)
 *   O_s             softmax(q k^T / sqrt(D)) v over the tokens of the critical
 *                   blocks only (0 when there is none)
 *   O_l             phi(q) H_i / (phi(q) . Z_i), H_i = sum h_j, Z_i = sum z_j over
 *                   the marginal blocks, h_j = phi(K_j)^T V_j, z_j = colsum phi(K_j),
 *                   phi(x) = elu(x) + 1 (0 when there is no marginal block)
 *   O               alpha[h, :] * O_s + (1 - alpha[h, :]) * O_l
 *
 * Conventions (all entry points):
 *   - Tensors are device pointers owned by the caller; no entry point allocates
 *     device memory (the only library-owned device memory is the fixed scratch
 *     array of sla_route_noalloc, part of the loaded module). Q, K, V and O are
 *     [B, H, N, D] bf16, contiguous, D fastest, 16-byte aligned. alpha is [H, D] fp32.
 *   - Supported: D in {64, 128}; block_q in {64, 128}; block_kv = 64;
 *     1 <= N; Nk = ceil(N / 64) <= 16384; 0 <= kh, kl and kh + kl <= 1.
 *   - Work is enqueued on the caller's stream; calls return before it runs.
 *   - Argument errors are found on the host before anything is enqueued; then
 *     nothing is written. Errors found on the device (a bounded wait that ran
 *     out, a caller label outside {0,1,2}) are recorded in the workspace's
 *     error word and reported by sla_check.
 *   - No entry point throws or exits; each returns an sla_status, and
 *     sla_last_error() gives a message for the calling thread's last failure.
 *   - The workspace (ws, ws_bytes >= sla_workspace_size) is caller memory,
 *     256-byte aligned; its first 256 bytes hold the device error word and
 *     must be zero before the first call that uses it (sla_check clears it).
 *     Concurrent calls must not share a workspace.
 */
#ifndef SLA_H_
#define SLA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  SLA_OK = 0,
  SLA_ERR_INVALID_ARG = 1, /* bad pointer, size, alignment or fraction */
  SLA_ERR_UNSUPPORTED = 2, /* valid but not implemented (e.g. D = 96) */
  SLA_ERR_WORKSPACE = 3,   /* workspace missing, misaligned or too small */
  SLA_ERR_CUDA = 4,        /* a CUDA runtime/driver call failed */
  SLA_ERR_TIMEOUT = 5,     /* a device-side bounded wait ran out (reported by sla_check) */
  SLA_ERR_BAD_MASK = 6     /* caller label outside {0,1,2} (reported by sla_check) */
} sla_status;

/* Problem shape. kh / kl: critical / negligible fractions of the KV blocks per row. */
typedef struct {
  int B, H, N, D;
  int block_q, block_kv;
  float kh, kl;
} sla_problem;

/* Block counts: Nq = ceil(N / block_q), Nk = ceil(N / block_kv), kc and kn as above.
 * Host only. Any output pointer may be NULL. */
sla_status sla_counts(const sla_problem* p, int* Nq, int* Nk, int* kc, int* kn);

/* Bytes of workspace sla_route / sla_forward need for this shape (0 on invalid shape).
 * Host only. */
size_t sla_workspace_size(const sla_problem* p);

/* Block router (SLA2 §2.B; SLA Abstract).
 *   q, k          [B,H,N,D] bf16 device
 *   mask_out      [B,H,Nq,Nk] int8 device: 2 critical, 1 marginal, 0 negligible
 *   crit_idx_out  [B,H,Nq,kc] int32 device, critical block indices ascending (nullable)
 *   scores_out    [B,H,Nq,Nk] fp64 device, raw compressed scores S (nullable)
 *   ws, ws_bytes  workspace
 *   stream        cudaStream_t (0 = legacy default stream) */
sla_status sla_route(const sla_problem* p, const void* q, const void* k, int8_t* mask_out,
                     int32_t* crit_idx_out, double* scores_out, void* ws, size_t ws_bytes,
                     void* stream);

/* Per-KV-block linear-attention states (SLA Abstract: O(N) branch).
 *   k, v   [B,H,N,D] bf16 device
 *   h_out  [B,H,Nk,D,D] fp32 device, h_j = phi(K_j)^T V_j over the block's valid tokens
 *   z_out  [B,H,Nk,D] fp32 device, z_j = colsum phi(K_j)
 *   ws     workspace for the error word (nullable: device errors then go unreported) */
sla_status sla_kv_states(const sla_problem* p, const void* k, const void* v, float* h_out,
                         float* z_out, void* ws, size_t ws_bytes, void* stream);

/* Fused forward (SLA Abstract; SLA2 §2.A blend).
 *   q, k, v   [B,H,N,D] bf16 device
 *   alpha     [H,D] fp32 device, blend ratio per head and channel
 *   mask      [B,H,Nq,Nk] int8 device labels replacing the router (nullable);
 *             with a mask, kh and kl are ignored and each row may hold any counts
 *   out       [B,H,N,D] bf16 device; must not alias q, k or v
 *   ws        workspace */
sla_status sla_forward(const sla_problem* p, const void* q, const void* k, const void* v,
                       const float* alpha, const int8_t* mask, void* out, void* ws, size_t ws_bytes,
                       void* stream);

/* sla_forward plus per-stage device times. Records CUDA events on the stream
 * between the stages, waits for the last one, and writes stage_ms[4] (host):
 * [0] per-block precompute (pooling, KV states), [1] routing (scores and
 * selection, or the caller-mask lists), [2] marginal-state aggregation,
 * [3] fused attention. The launches are those of sla_forward, with the same
 * results. Synchronises the stream; meant for measurement. */
sla_status sla_forward_timed(const sla_problem* p, const void* q, const void* k, const void* v,
                             const float* alpha, const int8_t* mask, void* out, void* ws,
                             size_t ws_bytes, void* stream, float* stage_ms);

/* ---------------------------------------------------------------- low-bit sparse branch
 *
 * SLA2 §2.C ("SLA2: Sparse-Linear Attention with Learnable Routing and QAT"): the
 * sparse branch runs with low-bit operands in the forward pass. The page fixes no
 * format; the library's reading:
 *   - e4m3 codes (round to nearest even, saturating at +-448) with one power-of-two
 *     scale 2^e per block, amax / 2^e in (128, 256] (e = 0 for an all-zero block):
 *     Q per query block, K and V per KV block; both matmuls of the sparse branch,
 *     Q K^T and P V, take e4m3 operands with fp32 accumulation;
 *   - P enters P V as e4m3 codes: with x the row's logits in log2 units and m their
 *     maximum, the P of a key of block j is coded as e4m3(2^(x - r) * 2^(ev_j - u)) for a
 *     reference r <= m and a unit exponent ev_j <= u <= ev_max (the largest V exponent
 *     among the row's critical blocks) that saturate no code. The reading leaves r and u
 *     to the kernel, and every such choice is a valid result: this kernel keeps r at a
 *     block's row maximum, moved to a later block's only when that exceeds r by more than
 *     8, and u = ev_max. The softmax normaliser sums the unrounded P;
 *   - the router, the linear branch and the blend are those of sla_forward.
 * Supported: D = 128 (else SLA_ERR_UNSUPPORTED), the block sizes of sla_forward. */

/* Workspace bytes for sla_forward_fp8: sla_workspace_size plus the e4m3 codes of K
 * and V (2 * B*H*N*D bytes) and their block exponents. 0 for an invalid problem. */
size_t sla_workspace_size_fp8(const sla_problem* p);

/* Fused forward with the low-bit sparse branch. Arguments as for sla_forward; ws
 * must hold sla_workspace_size_fp8(p) bytes. */
sla_status sla_forward_fp8(const sla_problem* p, const void* q, const void* k, const void* v,
                           const float* alpha, const int8_t* mask, void* out, void* ws,
                           size_t ws_bytes, void* stream);

/* sla_forward_fp8 plus per-stage device times, stage_ms[5] (host): [0] precompute,
 * [1] routing, [2] aggregation, [3] K/V quantiser, [4] fused attention. Synchronises
 * the stream; meant for measurement. */
sla_status sla_forward_fp8_timed(const sla_problem* p, const void* q, const void* k, const void* v,
                                 const float* alpha, const int8_t* mask, void* out, void* ws,
                                 size_t ws_bytes, void* stream, float* stage_ms);

/* Device addresses inside ws (sla_workspace_size_fp8(p) bytes) of the e4m3 codes of K and V
 * ([B,H,N,D] uint8) and of their block exponents ([B,H,Nk] int32) that the last
 * sla_forward_fp8 on this workspace wrote. Host only, nothing is enqueued. For tests and
 * inspection. */
sla_status sla_lowbit_codes(const sla_problem* p, void* ws, size_t ws_bytes, void** k8, void** v8, void** kexp,
                            void** vexp);

/* The K/V block quantiser of the low-bit branch on its own (the kernel sla_forward_fp8 runs).
 *   k, v                [B,H,N,D] bf16 device, 16-byte aligned
 *   k8_out, v8_out      [B,H,N,D] uint8 device e4m3 codes (8-byte aligned): sign bit 7,
 *                       exponent bits 3..6 (bias 7), mantissa bits 0..2; code * 2^exp
 *                       approximates the input
 *   kexp_out, vexp_out  [B,H,Nk] int32 device: the exponent of each KV block's scale
 * D = 64 or 128. Asynchronous on the stream; writes nothing on an argument error. */
sla_status sla_quantize_kv(const sla_problem* p, const void* k, const void* v, uint8_t* k8_out,
                           uint8_t* v8_out, int32_t* kexp_out, int32_t* vexp_out, void* stream);

/* Marginal-state aggregation on its own (SLA Abstract: the O(N) linear branch over the
 * marginal blocks): for each (b, h) and query block i,
 *   H_i = sum of h_j, Z_i = sum of z_j over the KV blocks j labelled marginal (1) in row i,
 * with h_j = phi(K_j)^T V_j and z_j = colsum phi(K_j) over the block's valid tokens.
 * The forward computes the same sums (there H_i is written scaled per channel for its blend).
 * Precision: phi(k) enters the tensor core in bf16, h_j and z_j are rounded to bf16, the sums
 * accumulate in fp32, H_i is rounded to bf16.
 *   k, v    [B,H,N,D] bf16 device, 16-byte aligned
 *   mask    [B,H,Nq,Nk] int8 device labels (e.g. from sla_route); values outside {0,1,2}
 *           are reported by sla_check
 *   H_out   [B,H,Nq,D,D] bf16 device (row-major D x D per query block), 16-byte aligned
 *   Z_out   [B,H,Nq,D] fp32 device, 16-byte aligned
 *   ws      workspace of at least sla_workspace_size(p) bytes
 * Asynchronous on the stream; writes nothing on an argument error. */
sla_status sla_aggregate_states(const sla_problem* p, const void* k, const void* v, const int8_t* mask,
                                void* H_out, float* Z_out, void* ws, size_t ws_bytes, void* stream);

/* Number of kernel launches sla_forward (low_bit = 0) or sla_forward_fp8 (low_bit = 1)
 * enqueues for this problem, with (with_mask = 1) or without a caller mask: one per stage
 * (precompute; labels: the caller mask's lists, or the router's scores and selection;
 * aggregation; the K/V quantiser for low_bit; attention). Host only; -1 for an invalid
 * problem. For measurement. */
int sla_forward_launches(const sla_problem* p, int with_mask, int low_bit);

/* ---------------------------------------------------------------- backward
 *
 * "SLA: Beyond Sparsity in Diffusion Transformers via Fine-Tunable Sparse-Linear Attention",
 * Abstract: one kernel covers the forward and the backward pass. The pages give no backward
 * formulas; this is the exact derivative of sla_forward's output with respect to q, k, v
 * and alpha with the block labels held fixed (the hard top-k passes no gradient):
 *   sparse branch  softmax attention renormalised over the critical keys, with
 *                  G_s = alpha dO: dV += P^T G_s, dS = P (G_s V^T - rowsum(G_s O_s)),
 *                  dQ += dS K / sqrt(D), dK += dS^T Q / sqrt(D)
 *   linear branch  with u = phi(q), den = u . Z_i, G_l = (1 - alpha) dO:
 *                  dQ += (G_l H_i^T / den - (G_l . O_l) Z_i / den) phi'(q), and through
 *                  dH_i = u^T G_l / den, dZ_i = -u^T (G_l . O_l) / den summed into every
 *                  marginal block's h_j, z_j: dV += phi(K_j) dh_j, dK += (V_j dh_j^T + dz_j) phi'(K_j)
 *   blend          dalpha[h, :] = sum over rows of dO (O_s - O_l)
 * phi'(x) = 1 for x > 0, e^x otherwise. Operands enter the tensor cores in bf16 (G_s, the
 * softmax P and dS, phi(q), dnum = G_l / den, the per-block states and their gradients);
 * accumulation is fp32. Every sum runs in a fixed order (the sparse branch's dK and dV per KV
 * block over the query tiles that hold it as critical, in ascending order; dalpha over the
 * tiles), so two calls give identical results.
 *   q, k, v, dO   [B,H,N,D] bf16 device, 16-byte aligned
 *   alpha         [H,D] fp32 device
 *   mask          [B,H,Nq,Nk] int8 device labels of the forward (nullable: the router runs)
 *   dQ, dK, dV    [B,H,N,D] fp32 device outputs, 16-byte aligned
 *   dalpha        [H,D] fp32 device output
 *   ws            workspace of sla_workspace_size_backward(p) bytes
 * Supported: D = 128 and block_q = 128 (else SLA_ERR_UNSUPPORTED). Asynchronous on the
 * stream; writes nothing on an argument error. */

/* Workspace bytes for sla_backward (0 for an invalid problem). */
size_t sla_workspace_size_backward(const sla_problem* p);

sla_status sla_backward(const sla_problem* p, const void* q, const void* k, const void* v, const float* alpha,
                        const int8_t* mask, const void* dO, float* dQ, float* dK, float* dV, float* dalpha,
                        void* ws, size_t ws_bytes, void* stream);

/* ---------------------------------------------------------------- variants
 *
 * Variants of the router and of the linear branch's feature map from "SPLA - Atención de
 * Bloque Dispersa más Lineal para el Modelado de Contexto Largo":
 *   feature_map  0: phi(x) = elu(x) + 1 (SLA, as sla_forward);
 *                1: phi(x) = e^x on the raw q and k (§2.3, the parameter-free exponential
 *                   map), in h_j, z_j and phi(q) of the linear branch;
 *   block_score  0: S_ij = qbar_i . kbar_j / sqrt(D) (SLA2 §2.B, as sla_route);
 *                1: the second-order block score (§2.1, diagonal covariance), ranked as its
 *                   log: S2_ij = qbar_i . kbar_j / sqrt(D) + log1p(sum_d qbar_i,d^2 var_j,d / (2 D)),
 *                   var_j,d the population variance of channel d over the block's valid
 *                   keys; labels from S2 with the same total order and counts.
 * and the post-tuning branch dropping of "SALAD: Achieve High-Sparsity Attention via Efficient
 * Linear Attention Tuning for Video Diffusion Transformer" §2:
 *   linear_scale, drop_threshold  the model's dynamic scale s of the linear branch at this
 *                   step and the threshold tau_t (both from the caller; the library computes
 *                   neither). When s < tau_t the linear branch is not run (no states, no
 *                   aggregation) and O = alpha * O_s; otherwise the forward is SLA's (s does
 *                   not scale the branch). Zero for both (a zero-initialised struct) keeps
 *                   the branch. Must be finite.
 * The sparse branch and the blend are those of sla_forward. */
typedef struct {
  int feature_map;
  int block_score;
  float linear_scale;
  float drop_threshold;
} sla_variant;

/* sla_route with a variant's block score. scores_out (nullable) receives the variant's
 * scores (S2 for block_score = 1). Other arguments as for sla_route; SLA_ERR_INVALID_ARG
 * for a variant field outside {0, 1}. */
sla_status sla_route_variant(const sla_problem* p, const sla_variant* variant, const void* q, const void* k,
                             int8_t* mask_out, int32_t* crit_idx_out, double* scores_out, void* ws,
                             size_t ws_bytes, void* stream);

/* sla_forward with a variant's block score (when mask is NULL), feature map and branch
 * dropping. Arguments as for sla_forward; the workspace of sla_workspace_size serves. */
sla_status sla_forward_variant(const sla_problem* p, const sla_variant* variant, const void* q, const void* k,
                               const void* v, const float* alpha, const int8_t* mask, void* out, void* ws,
                               size_t ws_bytes, void* stream);

/* ---------------------------------------------------------------- PISA
 *
 * "PISA - Atención Dispersa por Tramos para Transformers de Difusión Eficientes" §2: the
 * blocks that are not critical stay inside the softmax through a Taylor expansion of their
 * exponentials around the block's centroid, in the numerator and the denominator. Per query
 * token t of query block i with critical set S_i and the other blocks U_i:
 *   o_t = N_t / D_t
 *   N_t = sum_{j in S_i} sum_n e^{s_tn} v_n + sum_{j in U_i} a_tj Vsum_j
 *         + (q_t / sqrt(D)) Hbar sum_{j in U_i} a_tj
 *   D_t = sum_{j in S_i} sum_n e^{s_tn} + sum_{j in U_i} a_tj n_j
 * s_tn = q_t . k_n / sqrt(D), a_tj = e^{q_t . kbar_j / sqrt(D)}, kbar_j the mean of block
 * j's valid keys, n_j their count, Vsum_j the sum of its value rows, Hbar the mean over all
 * KV blocks of H_j = sum_n (k_n - kbar_j) v_n^T. Readings: every exponent carries 1 / sqrt(D)
 * (the first-order term's q_t / sqrt(D) follows); the denominator keeps the zero-order term
 * (the first-order one sums to zero); the critical sets are SLA's (label 2), every other
 * block is in U_i; the covariance-aware top-k the page mentions is not built. No alpha.
 * Precision: the critical blocks as sla_forward; kbar_j and Vsum_j enter the tensor cores
 * in bf16, Hbar in bf16 (summed in fp32 in a fixed order), the first-order operand
 * (sum_j a_tj / sqrt(D)) q_t in bf16. */

/* Workspace bytes for sla_forward_pisa and sla_pisa_hbar (0 for an invalid problem). */
size_t sla_workspace_size_pisa(const sla_problem* p);

/* The PISA output.
 *   q, k, v   [B,H,N,D] bf16 device, 16-byte aligned
 *   labels    [B,H,Nq,Nk] int8 device (nullable): the critical blocks are those labelled 2,
 *             labels outside {0, 1, 2} are reported by sla_check; NULL runs the router
 *             with p->kh, p->kl
 *   out       [B,H,N,D] bf16 device, 16-byte aligned, not aliasing q, k or v
 *   ws        workspace of sla_workspace_size_pisa(p) bytes
 * Asynchronous on the stream; writes nothing on an argument error. */
sla_status sla_forward_pisa(const sla_problem* p, const void* q, const void* k, const void* v, const int8_t* labels,
                            void* out, void* ws, size_t ws_bytes, void* stream);

/* Hbar of every head, [B,H,D,D] fp32 device (row d: key channel, column e: value channel),
 * as the PISA forward computes it before rounding it to bf16. k, v as for sla_forward_pisa;
 * ws of sla_workspace_size_pisa(p) bytes. For tests and inspection. */
sla_status sla_pisa_hbar(const sla_problem* p, const void* k, const void* v, float* hbar_out, void* ws,
                         size_t ws_bytes, void* stream);

/* Synchronise the stream, read and clear the workspace's device error word.
 * Returns SLA_OK, SLA_ERR_TIMEOUT or SLA_ERR_BAD_MASK (or SLA_ERR_CUDA). */
sla_status sla_check(void* ws, void* stream);

/* The block router for callers that cannot allocate device memory.
 *
 * There is no counterpart on the pages: this is a deployment variant of
 * sla_route. Some callers may not call cudaMalloc or hand the library an extra
 * buffer: a plugin running inside an inference server or graph runtime that owns
 * every byte of device memory, or a real-time loop with a fixed memory budget.
 * This entry point takes the same inputs and outputs as sla_route but no
 * workspace; its scratch is a 32 MiB array compiled into the library, which every
 * GPU that loads the library holds until the process exits.
 *   q, k, mask_out, crit_idx_out, scores_out   as for sla_route
 *   stream                                     cudaStream_t
 * Limits and behaviour:
 *   - The scratch holds the pooled means, plus the scores when scores_out is NULL
 *     and the critical lists when crit_idx_out is NULL. A problem that needs more
 *     than 32 MiB is rejected with SLA_ERR_WORKSPACE before anything is enqueued
 *     (the Wan2.1-1.3B shape B=1, H=12, N=32760, D=128 fits with both outputs NULL).
 *   - The library allocates nothing (no cudaMalloc, cudaFree or allocating library
 *     routine). Every call looks up the array's device address in the calling
 *     thread's current context (cudaGetSymbolAddress), so the call follows the
 *     context: after a cudaDeviceReset the next call uses the array of the new
 *     context. The first call on a device loads the module there; make it before
 *     any stream capture.
 *   - Every call shares the one array, which keeps the last call's contents. Calls
 *     whose work overlaps on the GPU (other streams, other host threads) race on it
 *     and must be ordered by the caller.
 *   - There is no error word: the router's kernels have no bounded waits and read no
 *     caller labels, so they raise no device-side error for sla_check to report.
 *     Launch failures are returned as SLA_ERR_CUDA. */
sla_status sla_route_noalloc(const sla_problem* p, const void* q, const void* k, int8_t* mask_out,
                             int32_t* crit_idx_out, double* scores_out, void* stream);

/* Self-test of the device-side failure path (no counterpart on the pages).
 *
 * Enqueues on `stream` one thread that waits on an mbarrier nothing ever arrives on,
 * through the same bounded wait every kernel of the library uses, with a limit of
 * limit_us microseconds instead of the kernels' 2 s. When the limit runs out the thread
 * records the timeout in the workspace's error word and returns; no fault, trap or hang
 * is involved and the context stays usable. A following sla_check on the same workspace
 * returns SLA_ERR_TIMEOUT and clears the word.
 *   ws, ws_bytes : a workspace (any problem's; only its 256-byte error word is used),
 *                  256-byte aligned, at least 256 bytes.
 *   limit_us     : 1 .. 1000000.
 * Returns SLA_ERR_WORKSPACE or SLA_ERR_INVALID_ARG on bad arguments (nothing enqueued),
 * SLA_ERR_CUDA if the launch fails, else SLA_OK. */
sla_status sla_selftest_wait_timeout(void* ws, size_t ws_bytes, unsigned limit_us, void* stream);

/* Message for the calling thread's most recent failed call ("" if none). */
const char* sla_last_error(void);

/* Library version string. */
const char* sla_version(void);

#ifdef __cplusplus
}
#endif

#endif /* SLA_H_ */
