// Host side of the C ABI declared in include/sla.h: argument checks, block
// counts, workspace layout, TMA descriptors and kernel launches.
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <mutex>
#include <string>
#include <utility>

#include <cudaTypedefs.h>

#include "../../include/sla.h"
#include "aggregate.cuh"
#include "attention.cuh"
#include "attention_fp8.cuh"
#include "backward.cuh"
#include "backward_kv.cuh"
#include "backward_states.cuh"
#include "fp8.cuh"
#include "pisa.cuh"
#include "prep.cuh"
#include "route.cuh"
#include "variants.cuh"

namespace {

using sla::AggArgs;
using sla::AttnArgs;
using sla::AttnFp8Args;
using sla::MaskListArgs;
using sla::CertArgs;
using sla::SelectArgs;

constexpr int kMaxNk = 16384;
thread_local std::string g_last_error;

sla_status fail(sla_status st, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof(buf), fmt, ap);
  va_end(ap);
  g_last_error = buf;
  return st;
}

#define SLA_CUDA(call)                                                                     \
  do {                                                                                     \
    cudaError_t e_ = (call);                                                               \
    if (e_ != cudaSuccess) return fail(SLA_ERR_CUDA, "%s: %s", #call, cudaGetErrorString(e_)); \
  } while (0)

// ------------------------------------------------------------------ shape

struct Shape {
  int B, H, N, D, bq, bk, BH;
  int Nq, Nk, kc, kn;
  int LD;     // row length of the stacked per-block states (D*D + 128)
  int w_ld;   // row stride of the marginal indicator (Nk rounded up to 64)
};

sla_status make_shape(const sla_problem* p, Shape* s) {
  if (!p) return fail(SLA_ERR_INVALID_ARG, "problem is NULL");
  if (p->B < 1 || p->H < 1 || p->N < 1) return fail(SLA_ERR_INVALID_ARG, "B, H, N must be >= 1");
  if (p->D != 64 && p->D != 128) return fail(SLA_ERR_UNSUPPORTED, "D=%d not supported (64 or 128)", p->D);
  if (p->block_kv != 64) return fail(SLA_ERR_UNSUPPORTED, "block_kv=%d not supported (64)", p->block_kv);
  if (p->block_q != 64 && p->block_q != 128)
    return fail(SLA_ERR_UNSUPPORTED, "block_q=%d not supported (64 or 128)", p->block_q);
  if (!std::isfinite(p->kh) || !std::isfinite(p->kl)) return fail(SLA_ERR_INVALID_ARG, "kh, kl must be finite");
  const long long kh_ppm = llround(static_cast<double>(p->kh) * 1e6);
  const long long kl_ppm = llround(static_cast<double>(p->kl) * 1e6);
  if (kh_ppm < 0 || kl_ppm < 0 || kh_ppm + kl_ppm > 1000000)
    return fail(SLA_ERR_INVALID_ARG, "need 0 <= kh, kl and kh + kl <= 1 (got %g, %g)", p->kh, p->kl);
  const long long BH = static_cast<long long>(p->B) * p->H;
  if (BH > 65535) return fail(SLA_ERR_UNSUPPORTED, "B*H=%lld exceeds 65535", BH);
  s->B = p->B;
  s->H = p->H;
  s->N = p->N;
  s->D = p->D;
  s->bq = p->block_q;
  s->bk = p->block_kv;
  s->BH = static_cast<int>(BH);
  s->Nq = (p->N + p->block_q - 1) / p->block_q;
  s->Nk = (p->N + p->block_kv - 1) / p->block_kv;
  if (s->Nk > kMaxNk) return fail(SLA_ERR_UNSUPPORTED, "N=%d gives %d KV blocks (max %d)", p->N, s->Nk, kMaxNk);
  if (static_cast<long long>(s->BH) * s->Nq * s->D >= (1ll << 31))
    return fail(SLA_ERR_UNSUPPORTED, "B*H*Nq*D too large");
  s->kc = static_cast<int>((kh_ppm * s->Nk + 999999) / 1000000);
  s->kn = static_cast<int>((kl_ppm * s->Nk) / 1000000);
  s->LD = s->D * s->D + 128;
  s->w_ld = (s->Nk + 63) / 64 * 64;
  return SLA_OK;
}

// ------------------------------------------------------------------ workspace

struct Workspace {
  uint32_t* err;
  double* qbar;
  double* kbar;
  double* var;  // per-block channel variances of K (the second-order block score)
  double* S;    // fp64 scores (the long-row selection)
  float* S32;   // fp32 scores (the certified selection), aliases S
  float* nq;    // fp32 norms of the pooled queries
  float* nk;    // fp32 norms of the pooled keys
  int8_t* mask;
  int32_t* crit;
  int32_t* crit_cnt;
  __nv_bfloat16* W;
  __nv_bfloat16* hst;
  __nv_bfloat16* Hagg;
  float* Zagg;
  __nv_bfloat16* zero_h;  // one D x D bf16 tile of zeros (the linear term when the branch is dropped)
  // backward only
  __nv_bfloat16* gs;    // alpha * dO [BH, N, D]
  __nv_bfloat16* dHst;  // [BH, Nq, LD]: dH_i row-major, then dZ_i, then zero pad
  __nv_bfloat16* WT;    // marginal indicator transposed [BH, Nk, wt_ld]
  __nv_bfloat16* dh;    // [BH, Nk, D*D] gradients of the per-block states
  float* dz;            // [BH, Nk, D]
  float* lse;           // [BH, N] log2-sum-exp of each row's critical scores
  float* delta;         // [BH, N] rowsum(G_s * O_s)
  float* dalpha_part;   // [BH * Nq, D] per-tile partial sums of dalpha
  int32_t* tlist;       // [BH * Nk, Nq] query tiles holding each KV block as critical
  int32_t* tcnt;        // [BH * Nk]
  int wt_ld;
  // low-bit sparse branch only
  uint8_t* k8;     // e4m3 codes of K [BH, N, D]
  uint8_t* v8;     // e4m3 codes of V [BH, N, D]
  int32_t* kexp;   // K block scale exponents [BH, Nk]
  int32_t* vexp;   // V block scale exponents [BH, Nk]
  // PISA only
  __nv_bfloat16* kcen;  // centroid keys: block means of K [BH, Nk, D]
  __nv_bfloat16* vsum;  // centroid values: block sums of V [BH, Nk, D]
  float* hpart;         // per-part sums of the centred first-order matrices [BH * P, D, D]
  __nv_bfloat16* hbar;  // mean first-order matrix per head [BH, D, D]
  size_t bytes;
};

size_t align256(size_t x) { return (x + 255) / 256 * 256; }

Workspace layout(const Shape& s, uint8_t* base, bool fp8 = false, bool bwd = false, bool pisa = false) {
  Workspace w{};
  size_t off = 0;
  auto take = [&](size_t bytes) {
    uint8_t* p = base ? base + off : nullptr;
    off += align256(bytes);
    return p;
  };
  const size_t BH = s.BH;
  w.err = reinterpret_cast<uint32_t*>(take(256));
  w.qbar = reinterpret_cast<double*>(take(BH * s.Nq * s.D * sizeof(double)));
  w.kbar = reinterpret_cast<double*>(take(BH * s.Nk * s.D * sizeof(double)));
  w.var = reinterpret_cast<double*>(take(BH * s.Nk * s.D * sizeof(double)));
  w.S = reinterpret_cast<double*>(take(BH * s.Nq * s.Nk * sizeof(double)));
  w.S32 = reinterpret_cast<float*>(w.S);
  w.nq = reinterpret_cast<float*>(take(BH * s.Nq * sizeof(float)));
  w.nk = reinterpret_cast<float*>(take(BH * s.Nk * sizeof(float)));
  w.mask = reinterpret_cast<int8_t*>(take(BH * s.Nq * s.Nk));
  w.crit = reinterpret_cast<int32_t*>(take(BH * s.Nq * s.Nk * sizeof(int32_t)));
  w.crit_cnt = reinterpret_cast<int32_t*>(take(BH * s.Nq * sizeof(int32_t)));
  w.W = reinterpret_cast<__nv_bfloat16*>(take(BH * s.Nq * s.w_ld * 2));
  w.hst = reinterpret_cast<__nv_bfloat16*>(take(BH * s.Nk * static_cast<size_t>(s.LD) * 2));
  w.Hagg = reinterpret_cast<__nv_bfloat16*>(take(BH * s.Nq * static_cast<size_t>(s.D) * s.D * 2));
  w.Zagg = reinterpret_cast<float*>(take(BH * s.Nq * s.D * sizeof(float)));
  w.zero_h = reinterpret_cast<__nv_bfloat16*>(take(static_cast<size_t>(s.D) * s.D * 2));
  if (bwd) {
    w.wt_ld = (s.Nq + 63) / 64 * 64;
    w.gs = reinterpret_cast<__nv_bfloat16*>(take(BH * s.N * static_cast<size_t>(s.D) * 2));
    w.dHst = reinterpret_cast<__nv_bfloat16*>(take(BH * s.Nq * static_cast<size_t>(s.LD) * 2));
    w.WT = reinterpret_cast<__nv_bfloat16*>(take(BH * s.Nk * static_cast<size_t>(w.wt_ld) * 2));
    w.dh = reinterpret_cast<__nv_bfloat16*>(take(BH * s.Nk * static_cast<size_t>(s.D) * s.D * 2));
    w.dz = reinterpret_cast<float*>(take(BH * s.Nk * s.D * sizeof(float)));
    w.lse = reinterpret_cast<float*>(take(BH * s.N * sizeof(float)));
    w.delta = reinterpret_cast<float*>(take(BH * s.N * sizeof(float)));
    w.dalpha_part = reinterpret_cast<float*>(take(BH * s.Nq * s.D * sizeof(float)));
    w.tlist = reinterpret_cast<int32_t*>(take(BH * s.Nk * s.Nq * sizeof(int32_t)));
    w.tcnt = reinterpret_cast<int32_t*>(take(BH * s.Nk * sizeof(int32_t)));
  }
  if (fp8) {
    w.k8 = take(BH * s.N * static_cast<size_t>(s.D));
    w.v8 = take(BH * s.N * static_cast<size_t>(s.D));
    w.kexp = reinterpret_cast<int32_t*>(take(BH * s.Nk * sizeof(int32_t)));
    w.vexp = reinterpret_cast<int32_t*>(take(BH * s.Nk * sizeof(int32_t)));
  }
  if (pisa) {
    const size_t DD = static_cast<size_t>(s.D) * s.D;
    w.kcen = reinterpret_cast<__nv_bfloat16*>(take(BH * s.Nk * s.D * 2));
    w.vsum = reinterpret_cast<__nv_bfloat16*>(take(BH * s.Nk * s.D * 2));
    w.hpart = reinterpret_cast<float*>(take(BH * sla::pisa_parts(s.BH, s.Nk) * DD * sizeof(float)));
    w.hbar = reinterpret_cast<__nv_bfloat16*>(take(BH * DD * 2));
  }
  w.bytes = off;
  return w;
}

sla_status check_ws(const Shape& s, void* ws, size_t ws_bytes, Workspace* w, bool fp8 = false, bool bwd = false,
                    bool pisa = false) {
  if (!ws) return fail(SLA_ERR_WORKSPACE, "workspace is NULL");
  if (reinterpret_cast<uintptr_t>(ws) % 256) return fail(SLA_ERR_WORKSPACE, "workspace must be 256-byte aligned");
  *w = layout(s, static_cast<uint8_t*>(ws), fp8, bwd, pisa);
  if (ws_bytes < w->bytes)
    return fail(SLA_ERR_WORKSPACE, "workspace too small: %zu bytes given, %zu needed", ws_bytes, w->bytes);
  return SLA_OK;
}

bool aligned16(const void* p) { return p && (reinterpret_cast<uintptr_t>(p) % 16) == 0; }

// ------------------------------------------------------------------ TMA descriptors

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(f);
  });
  return fn;
}

// Tensor map with 128-byte swizzle (bf16, or uint8 for e4m3 codes). dims/strides in
// elements (innermost first).
sla_status make_map(CUtensorMap* m, const void* ptr, int rank, const uint64_t* dims, const uint64_t* strides_el,
                    const uint32_t* box, bool u8 = false) {
  auto fn = encode_fn();
  if (!fn) return fail(SLA_ERR_CUDA, "cuTensorMapEncodeTiled is not available from the driver");
  cuuint64_t d[5], st[4];
  cuuint32_t b[5], es[5];
  for (int r = 0; r < rank; ++r) {
    d[r] = dims[r];
    b[r] = box[r];
    es[r] = 1;
  }
  for (int r = 0; r + 1 < rank; ++r) st[r] = strides_el[r] * (u8 ? 1 : 2);
  CUresult res = fn(m, u8 ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, rank, const_cast<void*>(ptr), d, st, b, es,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (res != CUDA_SUCCESS) return fail(SLA_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", static_cast<int>(res));
  return SLA_OK;
}

// [BH, N, D] activation map with a box of `rows` tokens x 64 channels.
sla_status act_map(CUtensorMap* m, const void* ptr, const Shape& s, uint32_t rows) {
  const uint64_t dims[3] = {static_cast<uint64_t>(s.D), static_cast<uint64_t>(s.N), static_cast<uint64_t>(s.BH)};
  const uint64_t strides[2] = {static_cast<uint64_t>(s.D), static_cast<uint64_t>(s.N) * s.D};
  const uint32_t box[3] = {64, rows, 1};
  return make_map(m, ptr, 3, dims, strides, box);
}

// [BH, N, 128] e4m3-code map with a box of `rows` tokens x 128 channels (128 bytes).
sla_status code_map(CUtensorMap* m, const void* ptr, const Shape& s, uint32_t rows) {
  const uint64_t dims[3] = {static_cast<uint64_t>(s.D), static_cast<uint64_t>(s.N), static_cast<uint64_t>(s.BH)};
  const uint64_t strides[2] = {static_cast<uint64_t>(s.D), static_cast<uint64_t>(s.N) * s.D};
  const uint32_t box[3] = {128, rows, 1};
  return make_map(m, ptr, 3, dims, strides, box, true);
}

// ------------------------------------------------------------------ launch helpers

int sm_count() {
  int dev = 0, n = 148;
  if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
  return n;
}

template <typename K>
sla_status allow_smem(K kernel, int bytes) {
  cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  if (e != cudaSuccess) return fail(SLA_ERR_CUDA, "cudaFuncSetAttribute: %s", cudaGetErrorString(e));
  return SLA_OK;
}

// Launch `kernel` as a programmatic dependent of the previous kernel in the stream: it may
// be scheduled while the predecessor drains and waits (griddepcontrol.wait) before
// reading the predecessor's results.
template <typename... KArgs, typename... Args>
sla_status launch_dependent(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                            const char* what, Args&&... args) {
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  cudaError_t e = cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
  if (e != cudaSuccess) return fail(SLA_ERR_CUDA, "launch of %s failed: %s", what, cudaGetErrorString(e));
  return SLA_OK;
}

sla_status launched(const char* what) {
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return fail(SLA_ERR_CUDA, "launch of %s failed: %s", what, cudaGetErrorString(e));
  return SLA_OK;
}

#define SLA_TRY(x)                 \
  do {                             \
    sla_status st_ = (x);          \
    if (st_ != SLA_OK) return st_; \
  } while (0)

template <int D>
sla_status launch_pool(const void* x, double* out, const Shape& s, int block, int nblocks, cudaStream_t st) {
  sla::pool_mean_kernel<D><<<dim3(nblocks, s.BH), 128, 0, st>>>(static_cast<const __nv_bfloat16*>(x), out, s.N,
                                                                  block, nblocks);
  return launched("pool_mean_kernel");
}

// Fused precompute: query-block means (when qbar is set), KV-block means, z_j and h_j.
template <int D, int FM = 0>
sla_status launch_prep(const void* q, const void* k, const void* v, const Shape& s, const sla::PrepArgs& args,
                       cudaStream_t st) {
  CUtensorMap mq, mk, mv, mh;
  std::memset(&mq, 0, sizeof(mq));
  std::memset(&mh, 0, sizeof(mh));
  if (args.qbar) SLA_TRY(act_map(&mq, q, s, static_cast<uint32_t>(s.bq)));
  SLA_TRY(act_map(&mk, k, s, 64));
  SLA_TRY(act_map(&mv, v, s, 64));
  if (args.hst) {
    // h_j tiles inside the stacked-state rows: (e, d, block) -> row * LD + d * D + e
    const uint64_t dims[3] = {static_cast<uint64_t>(s.D), static_cast<uint64_t>(s.D),
                              static_cast<uint64_t>(s.BH) * s.Nk};
    const uint64_t strides[2] = {static_cast<uint64_t>(s.D), static_cast<uint64_t>(s.LD)};
    const uint32_t box[3] = {64, static_cast<uint32_t>(s.D), 1};
    SLA_TRY(make_map(&mh, args.hst, 3, dims, strides, box));
  }
  constexpr int smem = sla::PrepSmem<D>::total();
  SLA_TRY(allow_smem(sla::prep_kernel<D, FM>, smem));
  const long long items = static_cast<long long>(s.BH) * s.Nk + (args.qbar ? static_cast<long long>(s.BH) * s.Nq : 0);
  const int grid = static_cast<int>(items < sm_count() ? items : sm_count());
  sla::prep_kernel<D, FM><<<grid, 576, smem, st>>>(mq, mk, mv, mh, args);
  return launched("prep_kernel");
}

template <int D>
sla_status launch_scores(const double* qbar, const double* kbar, double* S, const Shape& s, cudaStream_t st) {
  dim3 grid((s.Nk + 63) / 64, (s.Nq + 63) / 64, s.BH);
  return launch_dependent(sla::score_kernel<D>, grid, dim3(128), 0, st, "score_kernel", qbar, kbar, S, s.Nq, s.Nk);
}

template <int D>
sla_status launch_scores32(const Shape& s, const Workspace& w, cudaStream_t st) {
  dim3 grid((s.Nk + 63) / 64, (s.Nq + 63) / 64, s.BH);
  constexpr int smem = sla::Score32Smem<D>::kBytes;
  SLA_TRY(allow_smem(sla::score32_kernel<D>, smem));
  return launch_dependent(sla::score32_kernel<D>, grid, dim3(256), smem, st, "score32_kernel", w.qbar, w.kbar, w.S32,
                          w.nq, w.nk, s.Nq, s.Nk);
}

template <int KPL, int D>
sla_status launch_cert(const CertArgs& a, cudaStream_t st) {
  const int wpc = 8;
  return launch_dependent(sla::select_cert_kernel<KPL, D>, dim3((a.rows + wpc - 1) / wpc), dim3(wpc * 32), 0, st,
                          "select_cert_kernel", a);
}

// Rows of up to kCertMaxNk blocks are selected from fp32 scores with fp64 resolution of
// the uncertain band (keys in registers); longer rows from fp64 scores in shared memory.
constexpr int kCertMaxNk = 32 * 64;

sla_status launch_select64(const Shape& s, const Workspace& w, const double* S, int8_t* mask, int32_t* crit,
                           int crit_ld, __nv_bfloat16* W, cudaStream_t st);

// Labels, critical lists and the marginal indicator from the pooled means in w.qbar and
// w.kbar. scores64 (nullable) receives the fp64 scores whenever it is given.
template <int D>
sla_status launch_router(const Shape& s, const Workspace& w, double* scores64, int8_t* mask, int32_t* crit,
                         int crit_ld, __nv_bfloat16* W, cudaStream_t st) {
  if (s.Nk <= kCertMaxNk) {
    if (scores64) SLA_TRY(launch_scores<D>(w.qbar, w.kbar, scores64, s, st));
    SLA_TRY(launch_scores32<D>(s, w, st));
    CertArgs a{};
    a.S32 = w.S32;
    a.nq = w.nq;
    a.nk = w.nk;
    a.qbar = w.qbar;
    a.kbar = w.kbar;
    a.rows = s.BH * s.Nq;
    a.Nq = s.Nq;
    a.Nk = s.Nk;
    a.kc = s.kc;
    a.kn = s.kn;
    a.mask = mask;
    a.crit = crit;
    a.crit_ld = crit_ld;
    a.crit_cnt = w.crit_cnt;
    a.W = W;
    a.w_ld = s.w_ld;
    if (s.Nk <= 32 * 8) return launch_cert<8, D>(a, st);
    if (s.Nk <= 32 * 16) return launch_cert<16, D>(a, st);
    if (s.Nk <= 32 * 32) return launch_cert<32, D>(a, st);
    if (s.Nk <= 32 * 40) return launch_cert<40, D>(a, st);
    return launch_cert<64, D>(a, st);
  }
  double* S = scores64 ? scores64 : w.S;
  SLA_TRY(launch_scores<D>(w.qbar, w.kbar, S, s, st));
  return launch_select64(s, w, S, mask, crit, crit_ld, W, st);
}

// Labels, critical lists and the marginal indicator from fp64 scores S [BH, Nq, Nk].
sla_status launch_select64(const Shape& s, const Workspace& w, const double* S, int8_t* mask, int32_t* crit,
                           int crit_ld, __nv_bfloat16* W, cudaStream_t st) {
  SelectArgs a{};
  a.S = S;
  a.rows = s.BH * s.Nq;
  a.Nk = s.Nk;
  a.kc = s.kc;
  a.kn = s.kn;
  a.mask = mask;
  a.crit = crit;
  a.crit_ld = crit_ld;
  a.crit_cnt = w.crit_cnt;
  a.W = W;
  a.w_ld = s.w_ld;
  const size_t per_warp = static_cast<size_t>(a.Nk) * 8;
  int wpc = static_cast<int>((200 * 1024) / per_warp);
  wpc = wpc < 1 ? 1 : (wpc > 8 ? 8 : wpc);
  const int smem = static_cast<int>(wpc * per_warp);
  SLA_TRY(allow_smem(sla::select_kernel, smem));
  const int grid = (a.rows + wpc - 1) / wpc;
  return launch_dependent(sla::select_kernel, dim3(grid), dim3(wpc * 32), smem, st, "select_kernel", a);
}

// C[m, :] = sum_k A[m, k] Bst[k, :] per head (the aggregation GEMM): A [BH, M, a_ld] bf16 0/1,
// Bst [BH, K, LD] bf16 stacked states, C split into its first D*D columns (bf16, Cd) and the
// next D (fp32, Cz). Run forwards (A = W, M = Nq, K = Nk) and, for the backward, with the
// indicator transposed (A = W^T, M = Nk, K = Nq).
template <int D>
sla_status launch_agg_gemm(int M, int K, int BH, int LD, const __nv_bfloat16* A, int a_ld, const __nv_bfloat16* Bst,
                           __nv_bfloat16* Cd, float* Cz, uint32_t* err, const float* alpha, int H,
                           cudaStream_t st) {
  CUtensorMap mw, mh;
  {
    const uint64_t dims[3] = {static_cast<uint64_t>(K), static_cast<uint64_t>(M), static_cast<uint64_t>(BH)};
    const uint64_t strides[2] = {static_cast<uint64_t>(a_ld), static_cast<uint64_t>(M) * a_ld};
    const uint32_t box[3] = {64, 128, 1};
    SLA_TRY(make_map(&mw, A, 3, dims, strides, box));
  }
  {
    const uint64_t dims[3] = {static_cast<uint64_t>(LD), static_cast<uint64_t>(K), static_cast<uint64_t>(BH)};
    const uint64_t strides[2] = {static_cast<uint64_t>(LD), static_cast<uint64_t>(K) * LD};
    const uint32_t box[3] = {64, 64, 1};
    SLA_TRY(make_map(&mh, Bst, 3, dims, strides, box));
  }
  CUtensorMap mo;
  {
    const uint64_t DD = static_cast<uint64_t>(D) * D;
    const uint64_t dims[3] = {DD, static_cast<uint64_t>(M), static_cast<uint64_t>(BH)};
    const uint64_t strides[2] = {DD, static_cast<uint64_t>(M) * DD};
    const uint32_t box[3] = {64, 128, 1};
    SLA_TRY(make_map(&mo, Cd, 3, dims, strides, box));
  }
  const int smem = sla::kAggStages * sla::kAggStageBytes + sla::kAggStagingBytes + 1024;
  SLA_TRY(allow_smem(sla::agg_kernel<D>, smem));
  AggArgs a{M, K, LD, BH, Cd, Cz, err, alpha, H};
  const long long tiles = static_cast<long long>(LD / 128) * ((M + 255) / 256) * BH;
  const int grid = static_cast<int>(tiles < sm_count() ? tiles : sm_count());
  return launch_dependent(sla::agg_kernel<D>, dim3(grid), dim3(224), smem, st, "agg_kernel", mw, mh, mo, a);
}

template <int D>
sla_status launch_agg(const Shape& s, const Workspace& w, const float* alpha, cudaStream_t st) {
  return launch_agg_gemm<D>(s.Nq, s.Nk, s.BH, s.LD, w.W, s.w_ld, w.hst, w.Hagg, w.Zagg, w.err, alpha, s.H, st);
}

// PISA: the centroid pseudo-blocks from w.kcen / w.vsum and H~ = w.hbar (one per head).
// no_linear: the linear term is read from the workspace's zero tile (one for every tile) with
// no Z_i, so it adds nothing (the branch is dropped).
template <int D, int FM = 0, bool PISA = false>
sla_status launch_attn(const Shape& s, const void* q, const void* k, const void* v, const float* alpha, void* out,
                       const Workspace& w, int crit_ld, cudaStream_t st, bool no_linear = false) {
  CUtensorMap mq, mk, mv, mh, mo, mkc, mvc;
  SLA_TRY(act_map(&mq, q, s, 128));
  // output boxes of block_q rows: the staged 128-row tile holds the next query block's rows
  // past block_q when block_q = 64, and those must not be written
  SLA_TRY(act_map(&mo, out, s, static_cast<uint32_t>(s.bq)));
  SLA_TRY(act_map(&mk, k, s, 64));
  SLA_TRY(act_map(&mv, v, s, 64));
  {
    const uint64_t rows = no_linear ? static_cast<uint64_t>(s.D) : static_cast<uint64_t>(s.BH) * (PISA ? 1 : s.Nq) * s.D;
    const uint64_t dims[2] = {static_cast<uint64_t>(s.D), rows};
    const uint64_t strides[1] = {static_cast<uint64_t>(s.D)};
    const uint32_t box[2] = {64, 64};
    SLA_TRY(make_map(&mh, no_linear ? w.zero_h : (PISA ? w.hbar : w.Hagg), 2, dims, strides, box));
  }
  if (PISA) {
    // [BH, Nk, D]: the last pseudo-block's rows past Nk read as zeros
    const uint64_t dims[3] = {static_cast<uint64_t>(s.D), static_cast<uint64_t>(s.Nk), static_cast<uint64_t>(s.BH)};
    const uint64_t strides[2] = {static_cast<uint64_t>(s.D), static_cast<uint64_t>(s.Nk) * s.D};
    const uint32_t box[3] = {64, 64, 1};
    SLA_TRY(make_map(&mkc, w.kcen, 3, dims, strides, box));
    SLA_TRY(make_map(&mvc, w.vsum, 3, dims, strides, box));
  } else {
    mkc = mk;
    mvc = mv;
  }
  constexpr int smem = sla::AttnSmem<D>::total();
  SLA_TRY(allow_smem(sla::attn_kernel<D, FM, PISA>, smem));
  AttnArgs a;
  a.H = s.H;
  a.N = s.N;
  a.Nq = s.Nq;
  a.block_q = s.bq;
  a.n_tiles = s.BH * s.Nq;
  a.crit = w.crit;
  a.crit_ld = crit_ld;
  a.crit_cnt = w.crit_cnt;
  a.Zagg = (PISA || no_linear) ? nullptr : w.Zagg;
  a.h_mode = no_linear ? 2 : (PISA ? 1 : 0);
  a.alpha = PISA ? nullptr : alpha;
  a.out = static_cast<__nv_bfloat16*>(out);
  a.scale_log2 = static_cast<float>(1.4426950408889634 / std::sqrt(static_cast<double>(D)));
  a.Nk = s.Nk;
  a.nc = (s.Nk + 63) / 64;
  a.n_last = s.N - (s.Nk - 1) * 64;
  a.inv_sqrt_d = static_cast<float>(1.0 / std::sqrt(static_cast<double>(D)));
  a.err = w.err;
  // persistent: two CTAs per SM walk the tiles
  const int grid = a.n_tiles < 2 * sm_count() ? a.n_tiles : 2 * sm_count();
  return launch_dependent(sla::attn_kernel<D, FM, PISA>, dim3(grid), dim3(192), smem, st, "attn_kernel", mq, mk, mv,
                          mh, mo, mkc, mvc, a);
}

template <int D>
sla_status launch_quant(const Shape& s, const void* k, const void* v, uint8_t* k8, uint8_t* v8, int32_t* kexp,
                        int32_t* vexp, cudaStream_t st) {
  const dim3 grid(s.Nk, s.BH);
  auto kb = static_cast<const __nv_bfloat16*>(k);
  auto vb = static_cast<const __nv_bfloat16*>(v);
  sla::quant_kv_kernel<D><<<grid, 256, 0, st>>>(kb, vb, k8, v8, kexp, vexp, s.N, s.Nk);
  return launched("quant_kv_kernel");
}

sla_status launch_attn_fp8(const Shape& s, const void* q, const float* alpha, void* out, const Workspace& w,
                           int crit_ld, cudaStream_t st) {
  CUtensorMap mq, mk, mv, mh, mo;
  SLA_TRY(act_map(&mq, q, s, 128));
  SLA_TRY(act_map(&mo, out, s, static_cast<uint32_t>(s.bq)));  // boxes of block_q rows, as in launch_attn
  SLA_TRY(code_map(&mk, w.k8, s, 64));
  SLA_TRY(code_map(&mv, w.v8, s, 64));
  {
    const uint64_t dims[2] = {static_cast<uint64_t>(s.D), static_cast<uint64_t>(s.BH) * s.Nq * s.D};
    const uint64_t strides[1] = {static_cast<uint64_t>(s.D)};
    const uint32_t box[2] = {64, 64};
    SLA_TRY(make_map(&mh, w.Hagg, 2, dims, strides, box));
  }
  constexpr int smem = sla::AttnFp8Smem::total();
  SLA_TRY(allow_smem(sla::attn_fp8_kernel, smem));
  AttnFp8Args a;
  a.H = s.H;
  a.N = s.N;
  a.Nq = s.Nq;
  a.Nk = s.Nk;
  a.block_q = s.bq;
  a.n_tiles = s.BH * s.Nq;
  a.crit = w.crit;
  a.crit_ld = crit_ld;
  a.crit_cnt = w.crit_cnt;
  a.kexp = w.kexp;
  a.vexp = w.vexp;
  a.Zagg = w.Zagg;
  a.alpha = alpha;
  a.out = static_cast<__nv_bfloat16*>(out);
  a.scale_log2 = static_cast<float>(1.4426950408889634 / std::sqrt(static_cast<double>(s.D)));
  a.err = w.err;
  const int grid = a.n_tiles < 2 * sm_count() ? a.n_tiles : 2 * sm_count();
  return launch_dependent(sla::attn_fp8_kernel, dim3(grid), dim3(192), smem, st, "attn_fp8_kernel", mq, mk, mv, mh,
                          mo, a);
}

// ------------------------------------------------------------------ entry points (templated on D)

template <int D>
sla_status route_impl(const Shape& s, const void* q, const void* k, int8_t* mask_out, int32_t* crit_out,
                      double* scores_out, const Workspace& w, cudaStream_t st) {
  SLA_TRY(launch_pool<D>(q, w.qbar, s, s.bq, s.Nq, st));
  SLA_TRY(launch_pool<D>(k, w.kbar, s, s.bk, s.Nk, st));
  return launch_router<D>(s, w, scores_out, mask_out, crit_out ? crit_out : w.crit, crit_out ? s.kc : s.Nk, nullptr,
                          st);
}

// ------------------------------------------------------------------ backward

sla_status backward_impl(const Shape& s, const void* q, const void* k, const void* v, const float* alpha,
                         const int8_t* mask, const void* dO, float* dQ, float* dK, float* dV, float* dalpha,
                         const Workspace& w, cudaStream_t st) {
  constexpr int D = 128;
  // states, labels and H_i, Z_i as in the forward (H_i unscaled)
  sla::PrepArgs pa{};
  pa.BH = s.BH;
  pa.N = s.N;
  pa.Nq = s.Nq;
  pa.Nk = s.Nk;
  pa.block_q = s.bq;
  pa.qbar = mask ? nullptr : w.qbar;
  pa.kbar = mask ? nullptr : w.kbar;
  pa.hst = w.hst;
  pa.LD = s.LD;
  pa.err = w.err;
  SLA_TRY(launch_prep<D>(q, k, v, s, pa, st));
  if (mask) {
    MaskListArgs m{mask, s.BH * s.Nq, s.Nk, w.crit, s.Nk, w.crit_cnt, w.W, s.w_ld, w.err};
    sla::mask_lists_kernel<<<(m.rows + 7) / 8, 256, 0, st>>>(m);
    SLA_TRY(launched("mask_lists_kernel"));
  } else {
    SLA_TRY(launch_router<D>(s, w, nullptr, w.mask, w.crit, s.Nk, w.W, st));
  }
  SLA_TRY(launch_agg<D>(s, w, nullptr, st));
  // G_s = alpha dO
  const size_t chunks = static_cast<size_t>(s.BH) * s.N * D / 8;
  sla::gs_kernel<<<4 * sm_count(), 256, 0, st>>>(static_cast<const __nv_bfloat16*>(dO), alpha, w.gs, s.H, s.N, D,
                                                  chunks);
  SLA_TRY(launched("gs_kernel"));
  // per query tile: dQ, the tile's dalpha sums, dH_i / dZ_i, and each row's LSE and Delta
  {
    CUtensorMap mq, mg, mk, mv, mh, mdo;
    SLA_TRY(act_map(&mq, q, s, 128));
    SLA_TRY(act_map(&mg, w.gs, s, 128));
    SLA_TRY(act_map(&mdo, dO, s, 128));
    SLA_TRY(act_map(&mk, k, s, 64));
    SLA_TRY(act_map(&mv, v, s, 64));
    const uint64_t dims[2] = {static_cast<uint64_t>(D), static_cast<uint64_t>(s.BH) * s.Nq * D};
    const uint64_t strides[1] = {static_cast<uint64_t>(D)};
    const uint32_t box[2] = {64, 64};
    SLA_TRY(make_map(&mh, w.Hagg, 2, dims, strides, box));
    sla::BwdArgs a{};
    a.H = s.H;
    a.N = s.N;
    a.Nq = s.Nq;
    a.n_tiles = s.BH * s.Nq;
    a.LD = s.LD;
    a.crit = w.crit;
    a.crit_ld = s.Nk;
    a.crit_cnt = w.crit_cnt;
    a.Zagg = w.Zagg;
    a.alpha = alpha;
    a.dQ = dQ;
    a.lse = w.lse;
    a.delta = w.delta;
    a.dalpha_part = w.dalpha_part;
    a.dHst = w.dHst;
    a.scale_log2 = static_cast<float>(1.4426950408889634 / std::sqrt(static_cast<double>(D)));
    a.err = w.err;
    const int smem = 6 * 32768 + 1024;
    SLA_TRY(allow_smem(sla::bwd_kernel, smem));
    const int grid = a.n_tiles < sm_count() ? a.n_tiles : sm_count();
    SLA_TRY(launch_dependent(sla::bwd_kernel, dim3(grid), dim3(192), smem, st, "bwd_kernel", mq, mg, mk, mv, mh, mdo,
                             a));
  }
  // dh_j, dz_j = sums of dH_i, dZ_i over the rows i where j is marginal
  sla::w_transpose_kernel<<<dim3((s.Nk + 31) / 32, w.wt_ld / 32, s.BH), dim3(32, 8), 0, st>>>(w.W, s.Nq, s.Nk, s.w_ld,
                                                                                           w.WT, w.wt_ld);
  SLA_TRY(launched("w_transpose_kernel"));
  SLA_TRY(launch_agg_gemm<D>(s.Nk, s.Nq, s.BH, s.LD, w.WT, w.wt_ld, w.dHst, w.dh, w.dz, w.err, nullptr, s.H, st));
  sla::dalpha_kernel<<<dim3(s.H, D / 32), dim3(32, 8), 0, st>>>(w.dalpha_part, dalpha, s.B, s.H, s.Nq, D);
  SLA_TRY(launched("dalpha_kernel"));
  // per KV block: the sparse branch's dK_j, dV_j over the tiles holding it as critical, plus
  // the states' part
  sla::crit_transpose_kernel<<<dim3((s.Nk + 127) / 128, s.BH), 128, 0, st>>>(mask ? mask : w.mask, s.Nq, s.Nk,
                                                                             w.tlist, w.tcnt);
  SLA_TRY(launched("crit_transpose_kernel"));
  {
    CUtensorMap mq, mg, mk, mv, mdh;
    SLA_TRY(act_map(&mq, q, s, 128));
    SLA_TRY(act_map(&mg, w.gs, s, 128));
    SLA_TRY(act_map(&mk, k, s, 64));
    SLA_TRY(act_map(&mv, v, s, 64));
    const uint64_t dims[3] = {static_cast<uint64_t>(D), static_cast<uint64_t>(D), static_cast<uint64_t>(s.BH) * s.Nk};
    const uint64_t strides[2] = {static_cast<uint64_t>(D), static_cast<uint64_t>(D) * D};
    const uint32_t box[3] = {64, 128, 1};
    SLA_TRY(make_map(&mdh, w.dh, 3, dims, strides, box));
    sla::BwdKVArgs a{};
    a.BH = s.BH;
    a.N = s.N;
    a.Nq = s.Nq;
    a.Nk = s.Nk;
    a.tlist = w.tlist;
    a.tcnt = w.tcnt;
    a.lse = w.lse;
    a.delta = w.delta;
    a.dz = w.dz;
    a.dK = dK;
    a.dV = dV;
    a.scale_log2 = static_cast<float>(1.4426950408889634 / std::sqrt(static_cast<double>(D)));
    a.err = w.err;
    constexpr int smem = sla::BwdKVSmem::total();
    SLA_TRY(allow_smem(sla::bwd_kv_kernel, smem));
    const int blocks = s.BH * s.Nk;
    const int grid = blocks < sm_count() ? blocks : sm_count();
    SLA_TRY(launch_dependent(sla::bwd_kv_kernel, dim3(grid), dim3(192), smem, st, "bwd_kv_kernel", mq, mg, mk, mv,
                             mdh, a));
  }
  return SLA_OK;
}

// ------------------------------------------------------------------ variants (SPLA §2.1, §2.3)

struct Variant {
  int fm;      // feature map: 0 elu + 1, 1 e^x
  int score2;  // block score: 0 first order, 1 second order
  bool drop;   // the linear branch is not run (the caller's scale is below its threshold)
};

sla_status read_variant(const sla_variant* v, Variant* out) {
  if (!v) return fail(SLA_ERR_INVALID_ARG, "variant is NULL");
  if (v->feature_map != 0 && v->feature_map != 1)
    return fail(SLA_ERR_INVALID_ARG, "feature_map must be 0 (elu + 1) or 1 (exp), got %d", v->feature_map);
  if (v->block_score != 0 && v->block_score != 1)
    return fail(SLA_ERR_INVALID_ARG, "block_score must be 0 (first order) or 1 (second order), got %d", v->block_score);
  if (!std::isfinite(v->linear_scale) || !std::isfinite(v->drop_threshold))
    return fail(SLA_ERR_INVALID_ARG, "linear_scale and drop_threshold must be finite");
  out->fm = v->feature_map;
  out->score2 = v->block_score;
  out->drop = v->linear_scale < v->drop_threshold;
  return SLA_OK;
}

template <int D>
sla_status launch_block_var(const void* k, const Shape& s, const Workspace& w, cudaStream_t st) {
  sla::block_var_kernel<D><<<dim3(s.Nk, s.BH), 128, 0, st>>>(static_cast<const __nv_bfloat16*>(k), w.kbar, w.var, s.N);
  return launched("block_var_kernel");
}

template <int D>
sla_status launch_score2(const Shape& s, const Workspace& w, double* S2, cudaStream_t st) {
  sla::score2_kernel<D><<<dim3((s.Nk + 31) / 32, (s.Nq + 31) / 32, s.BH), 256, 0, st>>>(w.qbar, w.kbar, w.var, S2,
                                                                                           s.Nq, s.Nk);
  return launched("score2_kernel");
}

// Second-order labels from w.qbar (already pooled) and K: block means and variances, S2,
// the fp64 selection. S2 goes to scores64 when given, else to the workspace.
template <int D>
sla_status route_second_order(const Shape& s, const void* k, const Workspace& w, double* scores64, int8_t* mask,
                              int32_t* crit, int crit_ld, __nv_bfloat16* W, cudaStream_t st) {
  SLA_TRY(launch_block_var<D>(k, s, w, st));
  double* S2 = scores64 ? scores64 : w.S;
  SLA_TRY(launch_score2<D>(s, w, S2, st));
  return launch_select64(s, w, S2, mask, crit, crit_ld, W, st);
}

template <int D>
sla_status route_variant_impl(const Shape& s, const Variant& var, const void* q, const void* k, int8_t* mask_out,
                              int32_t* crit_out, double* scores_out, const Workspace& w, cudaStream_t st) {
  if (!var.score2) return route_impl<D>(s, q, k, mask_out, crit_out, scores_out, w, st);
  SLA_TRY(launch_pool<D>(q, w.qbar, s, s.bq, s.Nq, st));
  return route_second_order<D>(s, k, w, scores_out, mask_out, crit_out ? crit_out : w.crit, crit_out ? s.kc : s.Nk,
                               nullptr, st);
}

// The forward with a variant: one launch per stage over every head.
template <int D, int FM>
sla_status forward_variant_impl(const Shape& s, const Variant& var, const void* q, const void* k, const void* v,
                                const float* alpha, const int8_t* mask, void* out, const Workspace& w,
                                cudaStream_t st) {
  if (var.drop) {
    // SALAD's branch dropping: no states and no aggregation; the labels, then the sparse
    // branch against a zero linear term (O = alpha O_s)
    SLA_CUDA(cudaMemsetAsync(w.zero_h, 0, static_cast<size_t>(D) * D * 2, st));
    if (mask) {
      MaskListArgs m{mask, s.BH * s.Nq, s.Nk, w.crit, s.Nk, w.crit_cnt, nullptr, s.w_ld, w.err};
      sla::mask_lists_kernel<<<(m.rows + 7) / 8, 256, 0, st>>>(m);
      SLA_TRY(launched("mask_lists_kernel"));
    } else {
      SLA_TRY(launch_pool<D>(q, w.qbar, s, s.bq, s.Nq, st));
      if (var.score2) {
        SLA_TRY(route_second_order<D>(s, k, w, nullptr, nullptr, w.crit, s.Nk, nullptr, st));
      } else {
        SLA_TRY(launch_pool<D>(k, w.kbar, s, s.bk, s.Nk, st));
        SLA_TRY(launch_router<D>(s, w, nullptr, nullptr, w.crit, s.Nk, nullptr, st));
      }
    }
    return launch_attn<D, FM>(s, q, k, v, alpha, out, w, s.Nk, st, true);
  }
  sla::PrepArgs pa{};
  pa.BH = s.BH;
  pa.N = s.N;
  pa.Nq = s.Nq;
  pa.Nk = s.Nk;
  pa.block_q = s.bq;
  pa.qbar = mask ? nullptr : w.qbar;
  pa.kbar = mask ? nullptr : w.kbar;
  pa.hst = w.hst;
  pa.LD = s.LD;
  pa.err = w.err;
  SLA_TRY((launch_prep<D, FM>(q, k, v, s, pa, st)));
  if (mask) {
    MaskListArgs m{mask, s.BH * s.Nq, s.Nk, w.crit, s.Nk, w.crit_cnt, w.W, s.w_ld, w.err};
    sla::mask_lists_kernel<<<(m.rows + 7) / 8, 256, 0, st>>>(m);
    SLA_TRY(launched("mask_lists_kernel"));
  } else if (var.score2) {
    SLA_TRY(route_second_order<D>(s, k, w, nullptr, nullptr, w.crit, s.Nk, w.W, st));
  } else {
    SLA_TRY(launch_router<D>(s, w, nullptr, nullptr, w.crit, s.Nk, w.W, st));
  }
  SLA_TRY(launch_agg<D>(s, w, alpha, st));
  return launch_attn<D, FM>(s, q, k, v, alpha, out, w, s.Nk, st);
}

// ------------------------------------------------------------------ PISA

// Centroid keys and values, the per-part first-order sums and (with_kbar) the fp64 block
// means for the router.
template <int D>
sla_status launch_pisa_stats(const void* k, const void* v, const Shape& s, const Workspace& w, bool with_kbar,
                             cudaStream_t st) {
  CUtensorMap mk, mv;
  SLA_TRY(act_map(&mk, k, s, 64));
  SLA_TRY(act_map(&mv, v, s, 64));
  sla::PisaStatsArgs a{s.BH, s.N, s.Nk, sla::pisa_parts(s.BH, s.Nk), with_kbar ? w.kbar : nullptr, w.kcen, w.vsum,
                       w.hpart, w.err};
  constexpr int smem = sla::PisaSmem<D>::total();
  SLA_TRY(allow_smem(sla::pisa_stats_kernel<D>, smem));
  const int parts = s.BH * a.P;
  const int grid = parts < sm_count() ? parts : sm_count();
  sla::pisa_stats_kernel<D><<<grid, 576, smem, st>>>(mk, mv, a);
  return launched("pisa_stats_kernel");
}

template <int D>
sla_status launch_hbar(const Shape& s, const Workspace& w, __nv_bfloat16* h16, float* h32, cudaStream_t st) {
  sla::hbar_kernel<D><<<dim3(D, s.BH), D, 0, st>>>(w.hpart, h16, h32, sla::pisa_parts(s.BH, s.Nk), s.Nk);
  return launched("hbar_kernel");
}

// The PISA forward: statistics, critical sets (the router's label 2, or the caller's labels),
// Hbar, the fused pass.
template <int D>
sla_status forward_pisa_impl(const Shape& s, const void* q, const void* k, const void* v, const int8_t* labels,
                             void* out, const Workspace& w, cudaStream_t st) {
  SLA_TRY(launch_pisa_stats<D>(k, v, s, w, labels == nullptr, st));
  if (labels) {
    MaskListArgs m{labels, s.BH * s.Nq, s.Nk, w.crit, s.Nk, w.crit_cnt, nullptr, s.w_ld, w.err};
    sla::mask_lists_kernel<<<(m.rows + 7) / 8, 256, 0, st>>>(m);
    SLA_TRY(launched("mask_lists_kernel"));
  } else {
    SLA_TRY(launch_pool<D>(q, w.qbar, s, s.bq, s.Nq, st));
    SLA_TRY(launch_router<D>(s, w, nullptr, nullptr, w.crit, s.Nk, nullptr, st));
  }
  SLA_TRY(launch_hbar<D>(s, w, w.hbar, nullptr, st));
  return launch_attn<D, 0, true>(s, q, k, v, nullptr, out, w, s.Nk, st);
}

// Stage boundaries for sla_forward_timed: ev[0] before the per-block precompute,
// ev[1] after it, ev[2] after routing, ev[3] after aggregation, ev[4] after attention.
// sla_forward_fp8_timed: ev[4] after the K/V quantiser, ev[5] after attention.
struct StageEvents {
  cudaEvent_t ev[6];
  bool on;
  sla_status mark(int i, cudaStream_t st) {
    if (!on) return SLA_OK;
    cudaError_t e = cudaEventRecord(ev[i], st);
    if (e != cudaSuccess) return fail(SLA_ERR_CUDA, "cudaEventRecord: %s", cudaGetErrorString(e));
    return SLA_OK;
  }
};

template <int D>
sla_status forward_impl(const Shape& s, const void* q, const void* k, const void* v, const float* alpha,
                        const int8_t* mask, void* out, const Workspace& w, cudaStream_t st, StageEvents& ev,
                        bool fp8 = false) {
  sla::PrepArgs pa{};
  pa.BH = s.BH;
  pa.N = s.N;
  pa.Nq = s.Nq;
  pa.Nk = s.Nk;
  pa.block_q = s.bq;
  pa.qbar = mask ? nullptr : w.qbar;
  pa.kbar = mask ? nullptr : w.kbar;
  pa.hst = w.hst;
  pa.LD = s.LD;
  pa.err = w.err;
  SLA_TRY(ev.mark(0, st));
  SLA_TRY(launch_prep<D>(q, k, v, s, pa, st));
  SLA_TRY(ev.mark(1, st));
  if (mask) {
    MaskListArgs m{mask, s.BH * s.Nq, s.Nk, w.crit, s.Nk, w.crit_cnt, w.W, s.w_ld, w.err};
    sla::mask_lists_kernel<<<(m.rows + 7) / 8, 256, 0, st>>>(m);
    SLA_TRY(launched("mask_lists_kernel"));
  } else {
    SLA_TRY(launch_router<D>(s, w, nullptr, nullptr, w.crit, s.Nk, w.W, st));
  }
  SLA_TRY(ev.mark(2, st));
  // both attention kernels add the linear branch into their accumulator and take H_i scaled
  // per channel by (1 - alpha) / alpha
  SLA_TRY(launch_agg<D>(s, w, alpha, st));
  SLA_TRY(ev.mark(3, st));
  if (fp8) {
    if constexpr (D != 128) return fail(SLA_ERR_UNSUPPORTED, "the low-bit sparse branch needs D=128");
    SLA_TRY(launch_quant<D>(s, k, v, w.k8, w.v8, w.kexp, w.vexp, st));
    SLA_TRY(ev.mark(4, st));
    SLA_TRY(launch_attn_fp8(s, q, alpha, out, w, s.Nk, st));
    return ev.mark(5, st);
  }
  SLA_TRY(launch_attn<D>(s, q, k, v, alpha, out, w, s.Nk, st));
  return ev.mark(4, st);
}

sla_status forward_checked(const sla_problem* p, const void* q, const void* k, const void* v, const float* alpha,
                           const int8_t* mask, void* out, void* ws, size_t ws_bytes, cudaStream_t st,
                           StageEvents& ev, bool fp8 = false);

bool overlaps(const void* a, const void* b, size_t bytes) {
  const uintptr_t x = reinterpret_cast<uintptr_t>(a), y = reinterpret_cast<uintptr_t>(b);
  return x < y + bytes && y < x + bytes;
}

sla_status forward_checked(const sla_problem* p, const void* q, const void* k, const void* v, const float* alpha,
                           const int8_t* mask, void* out, void* ws, size_t ws_bytes, cudaStream_t st,
                           StageEvents& ev, bool fp8) {
  Shape s;
  SLA_TRY(make_shape(p, &s));
  if (fp8 && s.D != 128) return fail(SLA_ERR_UNSUPPORTED, "the low-bit sparse branch needs D=128 (got %d)", s.D);
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out))
    return fail(SLA_ERR_INVALID_ARG, "q, k, v and out must be non-NULL and 16-byte aligned");
  if (!alpha || reinterpret_cast<uintptr_t>(alpha) % 4) return fail(SLA_ERR_INVALID_ARG, "alpha must be 4-byte aligned");
  const size_t act = static_cast<size_t>(s.BH) * s.N * s.D * 2;
  if (overlaps(out, q, act) || overlaps(out, k, act) || overlaps(out, v, act))
    return fail(SLA_ERR_INVALID_ARG, "out must not alias q, k or v");
  Workspace w;
  SLA_TRY(check_ws(s, ws, ws_bytes, &w, fp8));
  if (s.D == 64) return forward_impl<64>(s, q, k, v, alpha, mask, out, w, st, ev, fp8);
  return forward_impl<128>(s, q, k, v, alpha, mask, out, w, st, ev, fp8);
}

// Shared body of the two timed entry points: `n` stages between n + 1 events.
sla_status forward_timed_common(const sla_problem* p, const void* q, const void* k, const void* v,
                                const float* alpha, const int8_t* mask, void* out, void* ws, size_t ws_bytes,
                                cudaStream_t st, float* stage_ms, bool fp8) {
  if (!stage_ms) return fail(SLA_ERR_INVALID_ARG, "stage_ms is NULL");
  const int n = fp8 ? 5 : 4;
  StageEvents ev{};
  ev.on = true;
  for (int i = 0; i <= n; ++i) {
    cudaError_t e = cudaEventCreate(&ev.ev[i]);
    if (e != cudaSuccess) {
      for (int j = 0; j < i; ++j) cudaEventDestroy(ev.ev[j]);
      return fail(SLA_ERR_CUDA, "cudaEventCreate: %s", cudaGetErrorString(e));
    }
  }
  sla_status rc = forward_checked(p, q, k, v, alpha, mask, out, ws, ws_bytes, st, ev, fp8);
  if (rc == SLA_OK) {
    cudaError_t e = cudaEventSynchronize(ev.ev[n]);
    for (int i = 0; i < n && e == cudaSuccess; ++i) e = cudaEventElapsedTime(&stage_ms[i], ev.ev[i], ev.ev[i + 1]);
    if (e != cudaSuccess) rc = fail(SLA_ERR_CUDA, "timing events: %s", cudaGetErrorString(e));
  }
  for (int i = 0; i <= n; ++i) cudaEventDestroy(ev.ev[i]);
  return rc;
}

}  // namespace

// ====================================================================== C ABI

namespace {
// One thread waits on an mbarrier that nothing arrives on, through the same bounded wait the
// kernels use, with a caller-chosen limit: the timeout path records SLA_DEVERR_TIMEOUT in the
// error word and the kernel returns normally, leaving the context usable.
__global__ void wait_selftest_kernel(uint32_t* err, uint64_t limit_ns) {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  sla::mbar_init(&bar, 1);
  abort_flag = 0;
  sla::fence_mbar_init();
  sla::mbar_wait_for(&bar, 0, err, &abort_flag, limit_ns);
}
}  // namespace

extern "C" {

sla_status sla_counts(const sla_problem* p, int* Nq, int* Nk, int* kc, int* kn) {
  Shape s;
  SLA_TRY(make_shape(p, &s));
  if (Nq) *Nq = s.Nq;
  if (Nk) *Nk = s.Nk;
  if (kc) *kc = s.kc;
  if (kn) *kn = s.kn;
  return SLA_OK;
}

size_t sla_workspace_size(const sla_problem* p) {
  Shape s;
  if (make_shape(p, &s) != SLA_OK) return 0;
  return layout(s, nullptr).bytes;
}

sla_status sla_route(const sla_problem* p, const void* q, const void* k, int8_t* mask_out, int32_t* crit_idx_out,
                     double* scores_out, void* ws, size_t ws_bytes, void* stream) {
  Shape s;
  SLA_TRY(make_shape(p, &s));
  if (!aligned16(q) || !aligned16(k)) return fail(SLA_ERR_INVALID_ARG, "q and k must be non-NULL and 16-byte aligned");
  if (!mask_out) return fail(SLA_ERR_INVALID_ARG, "mask_out is NULL");
  if (crit_idx_out && (reinterpret_cast<uintptr_t>(crit_idx_out) % 4))
    return fail(SLA_ERR_INVALID_ARG, "crit_idx_out must be 4-byte aligned");
  if (scores_out && (reinterpret_cast<uintptr_t>(scores_out) % 8))
    return fail(SLA_ERR_INVALID_ARG, "scores_out must be 8-byte aligned");
  Workspace w;
  SLA_TRY(check_ws(s, ws, ws_bytes, &w));
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (s.D == 64) return route_impl<64>(s, q, k, mask_out, crit_idx_out, scores_out, w, st);
  return route_impl<128>(s, q, k, mask_out, crit_idx_out, scores_out, w, st);
}

sla_status sla_kv_states(const sla_problem* p, const void* k, const void* v, float* h_out, float* z_out, void* ws,
                         size_t ws_bytes, void* stream) {
  Shape s;
  SLA_TRY(make_shape(p, &s));
  if (!aligned16(k) || !aligned16(v)) return fail(SLA_ERR_INVALID_ARG, "k and v must be non-NULL and 16-byte aligned");
  if (!aligned16(h_out) || !aligned16(z_out))
    return fail(SLA_ERR_INVALID_ARG, "h_out and z_out must be non-NULL and 16-byte aligned");
  uint32_t* err = nullptr;
  if (ws) {
    if (reinterpret_cast<uintptr_t>(ws) % 256 || ws_bytes < 256)
      return fail(SLA_ERR_WORKSPACE, "workspace must be 256-byte aligned and hold at least 256 bytes");
    err = static_cast<uint32_t*>(ws);
  }
  sla::PrepArgs pa{};
  pa.BH = s.BH;
  pa.N = s.N;
  pa.Nq = s.Nq;
  pa.Nk = s.Nk;
  pa.block_q = s.bq;
  pa.h32 = h_out;
  pa.z32 = z_out;
  pa.LD = s.LD;
  pa.err = err;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (s.D == 64) return launch_prep<64>(nullptr, k, v, s, pa, st);
  return launch_prep<128>(nullptr, k, v, s, pa, st);
}

sla_status sla_forward(const sla_problem* p, const void* q, const void* k, const void* v, const float* alpha,
                       const int8_t* mask, void* out, void* ws, size_t ws_bytes, void* stream) {
  StageEvents ev{};
  ev.on = false;
  return forward_checked(p, q, k, v, alpha, mask, out, ws, ws_bytes, static_cast<cudaStream_t>(stream), ev);
}

sla_status sla_forward_timed(const sla_problem* p, const void* q, const void* k, const void* v, const float* alpha,
                             const int8_t* mask, void* out, void* ws, size_t ws_bytes, void* stream,
                             float* stage_ms) {
  return forward_timed_common(p, q, k, v, alpha, mask, out, ws, ws_bytes, static_cast<cudaStream_t>(stream),
                              stage_ms, false);
}

size_t sla_workspace_size_fp8(const sla_problem* p) {
  Shape s;
  if (make_shape(p, &s) != SLA_OK) return 0;
  return layout(s, nullptr, true).bytes;
}

sla_status sla_forward_fp8(const sla_problem* p, const void* q, const void* k, const void* v, const float* alpha,
                           const int8_t* mask, void* out, void* ws, size_t ws_bytes, void* stream) {
  StageEvents ev{};
  ev.on = false;
  return forward_checked(p, q, k, v, alpha, mask, out, ws, ws_bytes, static_cast<cudaStream_t>(stream), ev, true);
}

sla_status sla_forward_fp8_timed(const sla_problem* p, const void* q, const void* k, const void* v,
                                 const float* alpha, const int8_t* mask, void* out, void* ws, size_t ws_bytes,
                                 void* stream, float* stage_ms) {
  return forward_timed_common(p, q, k, v, alpha, mask, out, ws, ws_bytes, static_cast<cudaStream_t>(stream),
                              stage_ms, true);
}

sla_status sla_quantize_kv(const sla_problem* p, const void* k, const void* v, uint8_t* k8_out, uint8_t* v8_out,
                           int32_t* kexp_out, int32_t* vexp_out, void* stream) {
  Shape s;
  SLA_TRY(make_shape(p, &s));
  if (!aligned16(k) || !aligned16(v)) return fail(SLA_ERR_INVALID_ARG, "k and v must be non-NULL and 16-byte aligned");
  if (!k8_out || !v8_out || reinterpret_cast<uintptr_t>(k8_out) % 8 || reinterpret_cast<uintptr_t>(v8_out) % 8)
    return fail(SLA_ERR_INVALID_ARG, "k8_out and v8_out must be non-NULL and 8-byte aligned");
  if (!kexp_out || !vexp_out || reinterpret_cast<uintptr_t>(kexp_out) % 4 ||
      reinterpret_cast<uintptr_t>(vexp_out) % 4)
    return fail(SLA_ERR_INVALID_ARG, "kexp_out and vexp_out must be non-NULL and 4-byte aligned");
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (s.D == 64) return launch_quant<64>(s, k, v, k8_out, v8_out, kexp_out, vexp_out, st);
  return launch_quant<128>(s, k, v, k8_out, v8_out, kexp_out, vexp_out, st);
}

sla_status sla_aggregate_states(const sla_problem* p, const void* k, const void* v, const int8_t* mask,
                                void* H_out, float* Z_out, void* ws, size_t ws_bytes, void* stream) {
  Shape s;
  SLA_TRY(make_shape(p, &s));
  if (!aligned16(k) || !aligned16(v)) return fail(SLA_ERR_INVALID_ARG, "k and v must be non-NULL and 16-byte aligned");
  if (!mask) return fail(SLA_ERR_INVALID_ARG, "mask is NULL");
  if (!aligned16(H_out) || !aligned16(Z_out))
    return fail(SLA_ERR_INVALID_ARG, "H_out and Z_out must be non-NULL and 16-byte aligned");
  Workspace w;
  SLA_TRY(check_ws(s, ws, ws_bytes, &w));
  w.Hagg = static_cast<__nv_bfloat16*>(H_out);
  w.Zagg = Z_out;
  sla::PrepArgs pa{};
  pa.BH = s.BH;
  pa.N = s.N;
  pa.Nq = s.Nq;
  pa.Nk = s.Nk;
  pa.block_q = s.bq;
  pa.hst = w.hst;
  pa.LD = s.LD;
  pa.err = w.err;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  MaskListArgs m{mask, s.BH * s.Nq, s.Nk, w.crit, s.Nk, w.crit_cnt, w.W, s.w_ld, w.err};
  if (s.D == 64) {
    SLA_TRY(launch_prep<64>(nullptr, k, v, s, pa, st));
  } else {
    SLA_TRY(launch_prep<128>(nullptr, k, v, s, pa, st));
  }
  sla::mask_lists_kernel<<<(m.rows + 7) / 8, 256, 0, st>>>(m);
  SLA_TRY(launched("mask_lists_kernel"));
  if (s.D == 64) return launch_agg<64>(s, w, nullptr, st);
  return launch_agg<128>(s, w, nullptr, st);
}

int sla_forward_launches(const sla_problem* p, int with_mask, int low_bit) {
  Shape s;
  if (make_shape(p, &s) != SLA_OK) return -1;
  // precompute, labels (router: scores + selection), aggregation, attention (+ the K/V quantiser)
  return 1 + (with_mask ? 1 : 2) + 1 + 1 + (low_bit ? 1 : 0);
}

sla_status sla_route_variant(const sla_problem* p, const sla_variant* variant, const void* q, const void* k,
                             int8_t* mask_out, int32_t* crit_idx_out, double* scores_out, void* ws, size_t ws_bytes,
                             void* stream) {
  Shape s;
  SLA_TRY(make_shape(p, &s));
  Variant var;
  SLA_TRY(read_variant(variant, &var));
  if (!aligned16(q) || !aligned16(k)) return fail(SLA_ERR_INVALID_ARG, "q and k must be non-NULL and 16-byte aligned");
  if (!mask_out) return fail(SLA_ERR_INVALID_ARG, "mask_out is NULL");
  if (crit_idx_out && (reinterpret_cast<uintptr_t>(crit_idx_out) % 4))
    return fail(SLA_ERR_INVALID_ARG, "crit_idx_out must be 4-byte aligned");
  if (scores_out && (reinterpret_cast<uintptr_t>(scores_out) % 8))
    return fail(SLA_ERR_INVALID_ARG, "scores_out must be 8-byte aligned");
  Workspace w;
  SLA_TRY(check_ws(s, ws, ws_bytes, &w));
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (s.D == 64) return route_variant_impl<64>(s, var, q, k, mask_out, crit_idx_out, scores_out, w, st);
  return route_variant_impl<128>(s, var, q, k, mask_out, crit_idx_out, scores_out, w, st);
}

sla_status sla_forward_variant(const sla_problem* p, const sla_variant* variant, const void* q, const void* k,
                               const void* v, const float* alpha, const int8_t* mask, void* out, void* ws,
                               size_t ws_bytes, void* stream) {
  Shape s;
  SLA_TRY(make_shape(p, &s));
  Variant var;
  SLA_TRY(read_variant(variant, &var));
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out))
    return fail(SLA_ERR_INVALID_ARG, "q, k, v and out must be non-NULL and 16-byte aligned");
  if (!alpha || reinterpret_cast<uintptr_t>(alpha) % 4) return fail(SLA_ERR_INVALID_ARG, "alpha must be 4-byte aligned");
  const size_t act = static_cast<size_t>(s.BH) * s.N * s.D * 2;
  if (overlaps(out, q, act) || overlaps(out, k, act) || overlaps(out, v, act))
    return fail(SLA_ERR_INVALID_ARG, "out must not alias q, k or v");
  Workspace w;
  SLA_TRY(check_ws(s, ws, ws_bytes, &w));
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (s.D == 64) {
    if (var.fm) return forward_variant_impl<64, 1>(s, var, q, k, v, alpha, mask, out, w, st);
    return forward_variant_impl<64, 0>(s, var, q, k, v, alpha, mask, out, w, st);
  }
  if (var.fm) return forward_variant_impl<128, 1>(s, var, q, k, v, alpha, mask, out, w, st);
  return forward_variant_impl<128, 0>(s, var, q, k, v, alpha, mask, out, w, st);
}

sla_status sla_lowbit_codes(const sla_problem* p, void* ws, size_t ws_bytes, void** k8, void** v8, void** kexp,
                            void** vexp) {
  Shape s;
  SLA_TRY(make_shape(p, &s));
  if (!k8 || !v8 || !kexp || !vexp) return fail(SLA_ERR_INVALID_ARG, "output pointers must be non-NULL");
  Workspace w;
  SLA_TRY(check_ws(s, ws, ws_bytes, &w, true));
  *k8 = w.k8;
  *v8 = w.v8;
  *kexp = w.kexp;
  *vexp = w.vexp;
  return SLA_OK;
}

size_t sla_workspace_size_pisa(const sla_problem* p) {
  Shape s;
  if (make_shape(p, &s) != SLA_OK) return 0;
  return layout(s, nullptr, false, false, true).bytes;
}

sla_status sla_forward_pisa(const sla_problem* p, const void* q, const void* k, const void* v, const int8_t* labels,
                            void* out, void* ws, size_t ws_bytes, void* stream) {
  Shape s;
  SLA_TRY(make_shape(p, &s));
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out))
    return fail(SLA_ERR_INVALID_ARG, "q, k, v and out must be non-NULL and 16-byte aligned");
  const size_t act = static_cast<size_t>(s.BH) * s.N * s.D * 2;
  if (overlaps(out, q, act) || overlaps(out, k, act) || overlaps(out, v, act))
    return fail(SLA_ERR_INVALID_ARG, "out must not alias q, k or v");
  Workspace w;
  SLA_TRY(check_ws(s, ws, ws_bytes, &w, false, false, true));
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (s.D == 64) return forward_pisa_impl<64>(s, q, k, v, labels, out, w, st);
  return forward_pisa_impl<128>(s, q, k, v, labels, out, w, st);
}

sla_status sla_pisa_hbar(const sla_problem* p, const void* k, const void* v, float* hbar_out, void* ws,
                         size_t ws_bytes, void* stream) {
  Shape s;
  SLA_TRY(make_shape(p, &s));
  if (!aligned16(k) || !aligned16(v)) return fail(SLA_ERR_INVALID_ARG, "k and v must be non-NULL and 16-byte aligned");
  if (!hbar_out || reinterpret_cast<uintptr_t>(hbar_out) % 4)
    return fail(SLA_ERR_INVALID_ARG, "hbar_out must be non-NULL and 4-byte aligned");
  Workspace w;
  SLA_TRY(check_ws(s, ws, ws_bytes, &w, false, false, true));
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (s.D == 64) {
    SLA_TRY(launch_pisa_stats<64>(k, v, s, w, false, st));
    return launch_hbar<64>(s, w, nullptr, hbar_out, st);
  }
  SLA_TRY(launch_pisa_stats<128>(k, v, s, w, false, st));
  return launch_hbar<128>(s, w, nullptr, hbar_out, st);
}

size_t sla_workspace_size_backward(const sla_problem* p) {
  Shape s;
  if (make_shape(p, &s) != SLA_OK) return 0;
  return layout(s, nullptr, false, true).bytes;
}

sla_status sla_backward(const sla_problem* p, const void* q, const void* k, const void* v, const float* alpha,
                        const int8_t* mask, const void* dO, float* dQ, float* dK, float* dV, float* dalpha, void* ws,
                        size_t ws_bytes, void* stream) {
  Shape s;
  SLA_TRY(make_shape(p, &s));
  if (s.D != 128) return fail(SLA_ERR_UNSUPPORTED, "the backward needs D=128 (got %d)", s.D);
  if (s.bq != 128) return fail(SLA_ERR_UNSUPPORTED, "the backward needs block_q=128 (got %d)", s.bq);
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(dO))
    return fail(SLA_ERR_INVALID_ARG, "q, k, v and dO must be non-NULL and 16-byte aligned");
  if (!aligned16(dQ) || !aligned16(dK) || !aligned16(dV))
    return fail(SLA_ERR_INVALID_ARG, "dQ, dK and dV must be non-NULL and 16-byte aligned");
  if (!alpha || reinterpret_cast<uintptr_t>(alpha) % 4) return fail(SLA_ERR_INVALID_ARG, "alpha must be 4-byte aligned");
  if (!dalpha || reinterpret_cast<uintptr_t>(dalpha) % 4)
    return fail(SLA_ERR_INVALID_ARG, "dalpha must be non-NULL and 4-byte aligned");
  Workspace w;
  SLA_TRY(check_ws(s, ws, ws_bytes, &w, false, true));
  return backward_impl(s, q, k, v, alpha, mask, dO, dQ, dK, dV, dalpha, w, static_cast<cudaStream_t>(stream));
}

sla_status sla_check(void* ws, void* stream) {
  if (!ws) return fail(SLA_ERR_WORKSPACE, "workspace is NULL");
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  SLA_CUDA(cudaStreamSynchronize(st));
  uint32_t word = 0;
  SLA_CUDA(cudaMemcpy(&word, ws, sizeof(word), cudaMemcpyDeviceToHost));
  if (word == 0) return SLA_OK;
  const uint32_t zero = 0;
  SLA_CUDA(cudaMemcpy(ws, &zero, sizeof(zero), cudaMemcpyHostToDevice));
  if (word & sla::SLA_DEVERR_TIMEOUT) return fail(SLA_ERR_TIMEOUT, "a device-side wait timed out (error word %u)", word);
  return fail(SLA_ERR_BAD_MASK, "caller mask held a label outside {0,1,2} (error word %u)", word);
}

sla_status sla_selftest_wait_timeout(void* ws, size_t ws_bytes, unsigned limit_us, void* stream) {
  if (!ws || reinterpret_cast<uintptr_t>(ws) % 256)
    return fail(SLA_ERR_WORKSPACE, "workspace must be non-NULL and 256-byte aligned");
  if (ws_bytes < 256) return fail(SLA_ERR_WORKSPACE, "workspace too small: %zu bytes given, 256 needed", ws_bytes);
  if (limit_us < 1 || limit_us > 1000000) return fail(SLA_ERR_INVALID_ARG, "limit_us must be in [1, 1000000]");
  wait_selftest_kernel<<<1, 1, 0, static_cast<cudaStream_t>(stream)>>>(static_cast<uint32_t*>(ws),
                                                                       static_cast<uint64_t>(limit_us) * 1000u);
  return launched("wait_selftest_kernel");
}

const char* sla_last_error(void) { return g_last_error.c_str(); }

const char* sla_version(void) { return "sla-b200 0.1.0 (sm_100a)"; }

}  // extern "C"

// ====================================================================== router without caller scratch
//
// sla_route_noalloc: the router for callers that cannot allocate device memory
// themselves. Its scratch (pooled means, and the scores and critical lists when
// the caller does not ask for them) lives in the file-scope array below instead
// of a caller workspace. Every GPU that loads this library holds the array
// until the process exits.

namespace {

constexpr size_t kRouteScratchBytes = size_t(32) << 20;  // 32 MiB
__device__ __align__(256) unsigned char g_route_scratch[kRouteScratchBytes];

// Device address of g_route_scratch in the calling thread's current CUDA context.
// Looked up on every call: the lookup is a host-side table read, and an address
// cached per device number would go stale when the context it came from is
// destroyed (cudaDeviceReset) or when the caller runs under another context of the
// same device. Host code must never pass the array's name itself to a kernel (it
// is a host-side stand-in there), only this address.
sla_status route_scratch_address(void** out) {
  void* p = nullptr;
  cudaError_t e = cudaGetSymbolAddress(&p, g_route_scratch);
  if (e != cudaSuccess || !p) return fail(SLA_ERR_CUDA, "cudaGetSymbolAddress(route scratch): %s", cudaGetErrorString(e));
  *out = p;
  return SLA_OK;
}

}  // namespace

extern "C" sla_status sla_route_noalloc(const sla_problem* p, const void* q, const void* k, int8_t* mask_out,
                                         int32_t* crit_idx_out, double* scores_out, void* stream) {
  Shape s;
  SLA_TRY(make_shape(p, &s));
  if (!aligned16(q) || !aligned16(k)) return fail(SLA_ERR_INVALID_ARG, "q and k must be non-NULL and 16-byte aligned");
  if (!mask_out) return fail(SLA_ERR_INVALID_ARG, "mask_out is NULL");
  if (crit_idx_out && (reinterpret_cast<uintptr_t>(crit_idx_out) % 4))
    return fail(SLA_ERR_INVALID_ARG, "crit_idx_out must be 4-byte aligned");
  if (scores_out && (reinterpret_cast<uintptr_t>(scores_out) % 8))
    return fail(SLA_ERR_INVALID_ARG, "scores_out must be 8-byte aligned");
  // Scratch layout inside the static array (256-byte aligned pieces).
  const size_t BH = s.BH;
  const size_t qbar_b = align256(BH * s.Nq * s.D * sizeof(double));
  const size_t kbar_b = align256(BH * s.Nk * s.D * sizeof(double));
  // Scores: fp32 for the certified selection (rows of up to kCertMaxNk blocks), else
  // fp64 unless the caller's scores_out holds them.
  const size_t S_b = s.Nk <= kCertMaxNk ? align256(BH * s.Nq * s.Nk * sizeof(float))
                                        : (scores_out ? 0 : align256(BH * s.Nq * s.Nk * sizeof(double)));
  const size_t nq_b = align256(BH * s.Nq * sizeof(float));
  const size_t nk_b = align256(BH * s.Nk * sizeof(float));
  const size_t crit_b = crit_idx_out ? 0 : align256(BH * s.Nq * s.Nk * sizeof(int32_t));
  const size_t cnt_b = align256(BH * s.Nq * sizeof(int32_t));
  const size_t need = qbar_b + kbar_b + S_b + nq_b + nk_b + crit_b + cnt_b;
  if (need > kRouteScratchBytes)
    return fail(SLA_ERR_WORKSPACE,
                "sla_route_noalloc: this problem needs %zu bytes of scratch, above the built-in maximum of %zu "
                "bytes; pass scores_out/crit_idx_out or use sla_route with a workspace",
                need, kRouteScratchBytes);
  void* base = nullptr;
  SLA_TRY(route_scratch_address(&base));
  uint8_t* b = static_cast<uint8_t*>(base);
  Workspace w{};
  size_t off = 0;
  auto piece = [&](size_t bytes) {
    uint8_t* p = bytes ? b + off : nullptr;
    off += bytes;
    return p;
  };
  w.qbar = reinterpret_cast<double*>(piece(qbar_b));
  w.kbar = reinterpret_cast<double*>(piece(kbar_b));
  w.S = reinterpret_cast<double*>(piece(S_b));
  w.S32 = reinterpret_cast<float*>(w.S);
  w.nq = reinterpret_cast<float*>(piece(nq_b));
  w.nk = reinterpret_cast<float*>(piece(nk_b));
  w.crit = reinterpret_cast<int32_t*>(piece(crit_b));
  w.crit_cnt = reinterpret_cast<int32_t*>(piece(cnt_b));
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (s.D == 64) return route_impl<64>(s, q, k, mask_out, crit_idx_out, scores_out, w, st);
  return route_impl<128>(s, q, k, mask_out, crit_idx_out, scores_out, w, st);
}
