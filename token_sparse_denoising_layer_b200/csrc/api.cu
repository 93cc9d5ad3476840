// api.cu - the extern "C" boundary of libhsa: argument validation, context
// and scratch management, and composition of the kernels into the calls of
// the Heterogeneous Step Allocation (HSA) denoising step ("Technical Summary:
// Heterogeneous Step Allocation (HSA) for Efficient Video Generation",
// sections 2.1-2.4).  See include/hsa.h for the contract of each call.

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>
#include <stdio.h>

#include <new>
#include <string>

#include "../../include/hsa.h"
#include "internal.h"

using hsa::Ctx;

struct hsa_ctx {
  Ctx c;
};

namespace {

thread_local std::string g_create_err;

hsa_status fail(hsa_ctx* ctx, hsa_status st, const std::string& msg) {
  if (ctx) ctx->c.err = msg;
  else g_create_err = msg;
  return st;
}

hsa_status cuda_fail(hsa_ctx* ctx, cudaError_t e, const char* what) {
  std::string msg = std::string(what) + ": " + cudaGetErrorString(e);
  return fail(ctx, HSA_ERR_CUDA, msg);
}

bool aligned16(const void* p) { return p != nullptr && (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

#define HSA_CHECK_PTR(ctx, p)                                                       \
  do {                                                                              \
    if (!aligned16(p))                                                              \
      return fail(ctx, HSA_ERR_INVALID_ARG, std::string(#p) + " is NULL or not 16-byte aligned"); \
  } while (0)

#define HSA_CHECK_CTX(ctx) \
  do {                     \
    if ((ctx) == nullptr) return fail(nullptr, HSA_ERR_INVALID_ARG, "ctx is NULL"); \
  } while (0)

hsa_status check_n(hsa_ctx* ctx, int n) {
  if (n < 0 || n > ctx->c.cfg.N)
    return fail(ctx, HSA_ERR_INVALID_ARG, "n must be in [0, N], got " + std::to_string(n));
  return HSA_OK;
}

hsa_status launched(hsa_ctx* ctx, cudaError_t e, const char* what, const std::string& why = "") {
  if (e == cudaSuccess) return HSA_OK;
  if (!why.empty()) return fail(ctx, HSA_ERR_INVALID_ARG, std::string(what) + ": " + why);
  return cuda_fail(ctx, e, what);
}

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  if (fn == nullptr) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  }
  return fn;
}

}  // namespace

namespace hsa {

bool make_tmap_bf16(CUtensorMap* map, const void* base, uint64_t rows, uint64_t cols,
                    uint64_t row_stride_elems, uint32_t box_rows, std::string* why) {
  EncodeTiledFn fn = encode_fn();
  if (fn == nullptr) {
    if (why) *why = "cuTensorMapEncodeTiled is not available from the driver";
    return false;
  }
  const cuuint64_t dims[2] = {cols, rows};
  const cuuint64_t strides[1] = {row_stride_elems * 2};
  const cuuint32_t box[2] = {64, box_rows};
  const cuuint32_t estr[2] = {1, 1};
  const CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims,
                        strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                        CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) {
    if (why) *why = "cuTensorMapEncodeTiled failed (code " + std::to_string(static_cast<int>(r)) + ")";
    return false;
  }
  return true;
}

}  // namespace hsa

extern "C" {

const char* hsa_last_error(const hsa_ctx* ctx) {
  return ctx ? ctx->c.err.c_str() : g_create_err.c_str();
}

hsa_status hsa_create(const hsa_model_cfg* cfg, int T, const int* budgets, const int* counts, int K,
                      int m, void* stream, hsa_ctx** out) {
  if (out == nullptr) return fail(nullptr, HSA_ERR_INVALID_ARG, "out is NULL");
  *out = nullptr;
  if (cfg == nullptr || budgets == nullptr || counts == nullptr)
    return fail(nullptr, HSA_ERR_INVALID_ARG, "cfg, budgets and counts must not be NULL");
  const hsa_model_cfg c = *cfg;
  if (c.N < 1 || c.C != 16 || c.H < 1 || c.D < 128 || c.D % 128 != 0 || c.D % c.H != 0 ||
      c.F < 64 || c.F % 64 != 0 || c.L < 0)
    return fail(nullptr, HSA_ERR_SHAPE,
                "unsupported shape: need N >= 1, C == 16, D % 128 == 0, F % 64 == 0");
  const int d = c.D / c.H;
  if (d != 64 && d != 128) return fail(nullptr, HSA_ERR_SHAPE, "head_dim D/H must be 64 or 128");
  if (K < 1 || K > hsa::kMaxGroups) return fail(nullptr, HSA_ERR_INVALID_ARG, "K must be in [1, 8]");
  if (T < 1) return fail(nullptr, HSA_ERR_BUDGET, "T must be positive");
  if (budgets[0] != T) return fail(nullptr, HSA_ERR_BUDGET, "the baseline group needs s_1 == T");
  long long total = 0;
  for (int k = 0; k < K; ++k) {
    if (budgets[k] < 1 || T % budgets[k] != 0)
      return fail(nullptr, HSA_ERR_BUDGET, "budget " + std::to_string(budgets[k]) + " does not divide T");
    if (k > 0 && budgets[k] >= budgets[k - 1])
      return fail(nullptr, HSA_ERR_BUDGET, "budgets must be strictly decreasing");
    if (counts[k] < 0) return fail(nullptr, HSA_ERR_BUDGET, "group counts must be >= 0");
    total += counts[k];
  }
  if (total != c.N) return fail(nullptr, HSA_ERR_BUDGET, "group counts must sum to N");
  if (m < 0 || 2 * m > T) return fail(nullptr, HSA_ERR_INVALID_ARG, "phase window needs 0 <= 2m <= T");

  hsa_ctx* ctx = new (std::nothrow) hsa_ctx();
  if (ctx == nullptr) return fail(nullptr, HSA_ERR_OOM, "host allocation failed");
  Ctx& x = ctx->c;
  x.cfg = c;
  x.T = T;
  x.K = K;
  x.m = m;
  for (int k = 0; k < K; ++k) {
    x.budgets[k] = budgets[k];
    x.counts[k] = counts[k];
    x.strides[k] = T / budgets[k];
  }
  x.stream = static_cast<cudaStream_t>(stream);
  cudaGetDevice(&x.device);
  cudaDeviceGetAttribute(&x.num_sms, cudaDevAttrMultiProcessorCount, x.device);
  const size_t nd = static_cast<size_t>(c.N) * c.D * 2;
  const size_t nf = static_cast<size_t>(c.N) * c.F * 2;
  cudaError_t e = cudaSuccess;
  if (e == cudaSuccess) e = cudaMalloc(&x.u, nd);
  if (e == cudaSuccess) e = cudaMalloc(&x.q, nd);
  if (e == cudaSuccess) e = cudaMalloc(&x.o, nd);
  if (e == cudaSuccess) e = cudaMalloc(&x.hmid, nf);
  if (e == cudaSuccess)
    e = cudaMalloc(reinterpret_cast<void**>(&x.attn_part_o),
                   static_cast<size_t>(hsa::kMaxAttnParts) * 256 * 128 * sizeof(float));
  if (e == cudaSuccess)
    e = cudaMalloc(reinterpret_cast<void**>(&x.attn_part_ml),
                   static_cast<size_t>(hsa::kMaxAttnParts) * 256 * 2 * sizeof(float));
  if (e == cudaSuccess) e = cudaMalloc(reinterpret_cast<void**>(&x.cuts), 2 * hsa::kMaxGroups * sizeof(uint32_t));
  if (e == cudaSuccess) e = cudaMalloc(reinterpret_cast<void**>(&x.flag), sizeof(int));
  if (e == cudaSuccess) e = cudaMemsetAsync(x.flag, 0, sizeof(int), x.stream);
  if (e == cudaSuccess) e = cudaStreamSynchronize(x.stream);
  if (e != cudaSuccess) {
    std::string msg = std::string("scratch allocation failed: ") + cudaGetErrorString(e);
    cudaGetLastError();
    hsa_destroy(ctx);
    return fail(nullptr, HSA_ERR_OOM, msg);
  }
  *out = ctx;
  return HSA_OK;
}

void hsa_destroy(hsa_ctx* ctx) {
  if (ctx == nullptr) return;
  Ctx& x = ctx->c;
  cudaStreamSynchronize(x.stream);
  for (auto& r : x.times)
    for (cudaEvent_t ev : r.pairs) cudaEventDestroy(ev);
  for (cudaEvent_t ev : x.event_pool) cudaEventDestroy(ev);
  cudaFree(x.u);
  cudaFree(x.q);
  cudaFree(x.o);
  cudaFree(x.hmid);
  cudaFree(x.attn_part_o);
  cudaFree(x.attn_part_ml);
  cudaFree(x.cuts);
  cudaFree(x.flag);
  delete ctx;
}

hsa_status hsa_set_stream(hsa_ctx* ctx, void* stream) {
  HSA_CHECK_CTX(ctx);
  ctx->c.stream = static_cast<cudaStream_t>(stream);
  return HSA_OK;
}

hsa_status hsa_sync_check(hsa_ctx* ctx) {
  HSA_CHECK_CTX(ctx);
  cudaError_t e = cudaStreamSynchronize(ctx->c.stream);
  if (e != cudaSuccess) return cuda_fail(ctx, e, "stream synchronize");
  int flag = 0;
  e = cudaMemcpy(&flag, ctx->c.flag, sizeof(int), cudaMemcpyDeviceToHost);
  if (e != cudaSuccess) return cuda_fail(ctx, e, "read device flag");
  if (flag == 0) return HSA_OK;
  // cleared on the context's stream, so the next launch there sees it cleared
  e = cudaMemsetAsync(ctx->c.flag, 0, sizeof(int), ctx->c.stream);
  if (e != cudaSuccess) return cuda_fail(ctx, e, "clear device flag");
  std::string msg = "device check flag " + std::to_string(flag) + ":";
  if (flag & hsa::DEV_TIMEOUT) msg += " a bounded wait timed out;";
  if (flag & hsa::DEV_BAD_INDEX) msg += " an index was out of range;";
  if (flag & hsa::DEV_BAD_SCORE) msg += " a score was NaN, negative or infinite;";
  if (flag & hsa::DEV_BAD_GROUP) msg += " a group id was >= K;";
  return fail(ctx, (flag & hsa::DEV_TIMEOUT) ? HSA_ERR_TIMEOUT : HSA_ERR_DEVICE_CHECK, msg);
}

hsa_status hsa_selftest_timeout(hsa_ctx* ctx, int timeout_us) {
  HSA_CHECK_CTX(ctx);
  if (timeout_us < 1 || timeout_us > 2000000)
    return fail(ctx, HSA_ERR_INVALID_ARG, "timeout_us must be in [1, 2000000]");
  return launched(ctx, hsa::launch_selftest_timeout(ctx->c, 1000ull * timeout_us),
                  "selftest_timeout");
}

uint64_t hsa_kernel_launches(const hsa_ctx* ctx) { return ctx ? ctx->c.launches : 0; }

hsa_status hsa_time_kernels(hsa_ctx* ctx, int on) {
  HSA_CHECK_CTX(ctx);
  ctx->c.timing = on != 0;
  return HSA_OK;
}

hsa_status hsa_kernel_times(hsa_ctx* ctx, hsa_kernel_class_time* out, int n_classes) {
  HSA_CHECK_CTX(ctx);
  if (out == nullptr || n_classes < 0) return fail(ctx, HSA_ERR_INVALID_ARG, "out is NULL");
  Ctx& c = ctx->c;
  cudaError_t e = cudaStreamSynchronize(c.stream);
  if (e != cudaSuccess) return cuda_fail(ctx, e, "stream synchronize");
  hsa_status st = HSA_OK;
  for (int k = 0; k < hsa::TC_COUNT; ++k) {
    hsa::TimeRec& r = c.times[k];
    double ms = 0.0;
    for (size_t j = 0; j + 1 < r.pairs.size(); j += 2) {
      float t = 0.f;
      e = cudaEventElapsedTime(&t, r.pairs[j], r.pairs[j + 1]);
      if (e != cudaSuccess) st = cuda_fail(ctx, e, "event elapsed time");
      ms += t;
    }
    if (k < n_classes) {
      out[k].calls = r.calls;
      out[k].ms = ms;
      out[k].work = r.work;
    }
    for (cudaEvent_t ev : r.pairs) c.event_pool.push_back(ev);
    r = hsa::TimeRec{};
  }
  return st;
}

int hsa_n_active(const hsa_ctx* ctx, int i) {
  if (ctx == nullptr || i < 0 || i >= ctx->c.T) return -1;
  const Ctx& x = ctx->c;
  const bool window = x.m > 0 && (i < x.m || i >= x.T - x.m);
  int n = 0;
  for (int k = 0; k < x.K; ++k)
    if (window || i % x.strides[k] == 0) n += x.counts[k];
  return n;
}

hsa_status hsa_schedule(hsa_ctx* ctx, int i, const uint8_t* g, uint8_t* mask, int32_t* active_idx,
                        int32_t* n_active_dev, int* n_active) {
  HSA_CHECK_CTX(ctx);
  HSA_CHECK_PTR(ctx, g);
  HSA_CHECK_PTR(ctx, mask);
  HSA_CHECK_PTR(ctx, active_idx);
  if (i < 0 || i >= ctx->c.T) return fail(ctx, HSA_ERR_INVALID_ARG, "iteration i outside [0, T)");
  if (n_active) *n_active = hsa_n_active(ctx, i);
  return launched(ctx, hsa::launch_schedule(ctx->c, i, g, mask, active_idx, n_active_dev), "schedule");
}

hsa_status hsa_score(hsa_ctx* ctx, const float* v_prev, const float* v_cur, float* score) {
  HSA_CHECK_CTX(ctx);
  HSA_CHECK_PTR(ctx, v_prev);
  HSA_CHECK_PTR(ctx, v_cur);
  HSA_CHECK_PTR(ctx, score);
  return launched(ctx, hsa::launch_score(ctx->c, v_prev, v_cur, score), "score");
}

hsa_status hsa_select_from_score(hsa_ctx* ctx, const float* score, uint8_t* g) {
  HSA_CHECK_CTX(ctx);
  HSA_CHECK_PTR(ctx, score);
  HSA_CHECK_PTR(ctx, g);
  return launched(ctx, hsa::launch_select(ctx->c, score, g), "select");
}

hsa_status hsa_select_groups(hsa_ctx* ctx, const float* v_prev, const float* v_cur, float* score,
                             uint8_t* g) {
  hsa_status st = hsa_score(ctx, v_prev, v_cur, score);
  if (st != HSA_OK) return st;
  return hsa_select_from_score(ctx, score, g);
}

hsa_status hsa_ln_gather(hsa_ctx* ctx, const float* x, const int32_t* idx, int n, void* u) {
  HSA_CHECK_CTX(ctx);
  if (hsa_status st = check_n(ctx, n)) return st;
  if (n == 0) return HSA_OK;
  HSA_CHECK_PTR(ctx, x);
  HSA_CHECK_PTR(ctx, idx);
  HSA_CHECK_PTR(ctx, u);
  return launched(ctx, hsa::launch_ln_gather(ctx->c, x, idx, n, u), "ln_gather");
}

hsa_status hsa_linear(hsa_ctx* ctx, const void* a, int M, int Kd, const void* w, int Ncols, void* out) {
  HSA_CHECK_CTX(ctx);
  if (M < 0 || Kd <= 0 || Ncols <= 0 || Kd % 64 != 0 || Ncols % 32 != 0)
    return fail(ctx, HSA_ERR_SHAPE, "linear needs M >= 0, K % 64 == 0, Ncols % 32 == 0");
  if (M == 0) return HSA_OK;
  HSA_CHECK_PTR(ctx, a);
  HSA_CHECK_PTR(ctx, w);
  HSA_CHECK_PTR(ctx, out);
  hsa::GemmArgs g{};
  g.A = a;
  g.B = w;
  g.M = M;
  g.Ncols = Ncols;
  g.Kd = Kd;
  g.epi = hsa::EPI_STORE;
  g.out = out;
  g.ld_out = Ncols;
  std::string why;
  cudaError_t e = hsa::launch_gemm(ctx->c, g, &why);
  return launched(ctx, e, "linear", why);
}

hsa_status hsa_qkv_project(hsa_ctx* ctx, const void* w_qkv, const void* u, const int32_t* idx,
                           int n, void* q, void* k_cache, void* v_cache) {
  HSA_CHECK_CTX(ctx);
  if (hsa_status st = check_n(ctx, n)) return st;
  if (n == 0) return HSA_OK;
  HSA_CHECK_PTR(ctx, w_qkv);
  HSA_CHECK_PTR(ctx, u);
  HSA_CHECK_PTR(ctx, idx);
  HSA_CHECK_PTR(ctx, q);
  HSA_CHECK_PTR(ctx, k_cache);
  HSA_CHECK_PTR(ctx, v_cache);
  const int D = ctx->c.cfg.D;
  hsa::GemmArgs g{};
  g.A = u;
  g.B = w_qkv;
  g.M = n;
  g.Ncols = 3 * D;
  g.Kd = D;
  g.epi = hsa::EPI_QKV;
  g.out = q;
  g.ld_out = D;
  g.k_cache = k_cache;
  g.v_cache = v_cache;
  g.idx = idx;
  g.N = ctx->c.cfg.N;
  std::string why;
  return launched(ctx, hsa::launch_gemm(ctx->c, g, &why), "qkv_project", why);
}

hsa_status hsa_qkv_project_peers(hsa_ctx* ctx, const void* w_qkv, const void* u,
                                 const int32_t* idx, int n, void* q, void* const* k_caches,
                                 void* const* v_caches, int n_caches) {
  HSA_CHECK_CTX(ctx);
  if (hsa_status st = check_n(ctx, n)) return st;
  if (n_caches < 1 || n_caches > hsa::kMaxCaches)
    return fail(ctx, HSA_ERR_INVALID_ARG, "n_caches outside [1, 8]");
  if (k_caches == nullptr || v_caches == nullptr)
    return fail(ctx, HSA_ERR_INVALID_ARG, "k_caches or v_caches is NULL");
  for (int g = 0; g < n_caches; ++g) {
    if (!aligned16(k_caches[g]) || !aligned16(v_caches[g]))
      return fail(ctx, HSA_ERR_INVALID_ARG,
                  "cache " + std::to_string(g) + " is NULL or not 16-byte aligned");
  }
  if (n == 0) return HSA_OK;
  HSA_CHECK_PTR(ctx, w_qkv);
  HSA_CHECK_PTR(ctx, u);
  HSA_CHECK_PTR(ctx, idx);
  HSA_CHECK_PTR(ctx, q);
  const int D = ctx->c.cfg.D;
  hsa::GemmArgs g{};
  g.A = u;
  g.B = w_qkv;
  g.M = n;
  g.Ncols = 3 * D;
  g.Kd = D;
  g.epi = hsa::EPI_QKV;
  g.out = q;
  g.ld_out = D;
  g.n_caches = n_caches;
  for (int c = 0; c < n_caches; ++c) {
    g.k_caches[c] = k_caches[c];
    g.v_caches[c] = v_caches[c];
  }
  g.idx = idx;
  g.N = ctx->c.cfg.N;
  std::string why;
  return launched(ctx, hsa::launch_gemm(ctx->c, g, &why), "qkv_project_peers", why);
}

hsa_status hsa_kv_scatter(hsa_ctx* ctx, const void* k_rows, const void* v_rows,
                          const int32_t* idx, int n, void* k_cache, void* v_cache) {
  HSA_CHECK_CTX(ctx);
  if (hsa_status st = check_n(ctx, n)) return st;
  if (n == 0) return HSA_OK;
  HSA_CHECK_PTR(ctx, k_rows);
  HSA_CHECK_PTR(ctx, v_rows);
  HSA_CHECK_PTR(ctx, idx);
  HSA_CHECK_PTR(ctx, k_cache);
  HSA_CHECK_PTR(ctx, v_cache);
  return launched(ctx,
                  hsa::launch_kv_scatter(ctx->c, k_rows, v_rows, ctx->c.cfg.D, idx, n, k_cache,
                                         v_cache),
                  "kv_scatter");
}

hsa_status hsa_kv_scatter_packed(hsa_ctx* ctx, const void* kv_rows, const int32_t* idx, int n,
                                 void* k_cache, void* v_cache) {
  HSA_CHECK_CTX(ctx);
  if (hsa_status st = check_n(ctx, n)) return st;
  if (n == 0) return HSA_OK;
  HSA_CHECK_PTR(ctx, kv_rows);
  HSA_CHECK_PTR(ctx, idx);
  HSA_CHECK_PTR(ctx, k_cache);
  HSA_CHECK_PTR(ctx, v_cache);
  const int D = ctx->c.cfg.D;
  const void* v_rows = static_cast<const uint16_t*>(kv_rows) + D;
  return launched(ctx,
                  hsa::launch_kv_scatter(ctx->c, kv_rows, v_rows, 2 * D, idx, n, k_cache, v_cache),
                  "kv_scatter_packed");
}

hsa_status hsa_attention(hsa_ctx* ctx, const void* q, int n, const void* k_cache,
                         const void* v_cache, void* o) {
  HSA_CHECK_CTX(ctx);
  if (hsa_status st = check_n(ctx, n)) return st;
  if (n == 0) return HSA_OK;
  HSA_CHECK_PTR(ctx, q);
  HSA_CHECK_PTR(ctx, k_cache);
  HSA_CHECK_PTR(ctx, v_cache);
  HSA_CHECK_PTR(ctx, o);
  std::string why;
  return launched(ctx,
                  hsa::launch_attention(ctx->c, q, n, k_cache, v_cache, ctx->c.cfg.N, o, &why),
                  "attention", why);
}

hsa_status hsa_attention_kv(hsa_ctx* ctx, const void* q, int n, const void* k, const void* v,
                            int n_kv, void* o) {
  HSA_CHECK_CTX(ctx);
  if (hsa_status st = check_n(ctx, n)) return st;
  if (n_kv <= 0) return fail(ctx, HSA_ERR_SHAPE, "attention_kv needs n_kv >= 1");
  if (n == 0) return HSA_OK;
  HSA_CHECK_PTR(ctx, q);
  HSA_CHECK_PTR(ctx, k);
  HSA_CHECK_PTR(ctx, v);
  HSA_CHECK_PTR(ctx, o);
  std::string why;
  return launched(ctx, hsa::launch_attention(ctx->c, q, n, k, v, n_kv, o, &why), "attention_kv",
                  why);
}

namespace {

// x[idx[m]] += gate * (o[m] W^T) for a [D, D] projection; gate NULL means 1.
hsa_status proj_residual(hsa_ctx* ctx, const void* w, const void* o, const int32_t* idx, int n,
                         float* x, const float* gate, const char* what) {
  const int D = ctx->c.cfg.D;
  hsa::GemmArgs g{};
  g.A = o;
  g.B = w;
  g.M = n;
  g.Ncols = D;
  g.Kd = D;
  g.epi = hsa::EPI_RESID;
  g.x = x;
  g.ld_x = D;
  g.gate = gate;
  g.idx = idx;
  g.N = ctx->c.cfg.N;
  std::string why;
  return launched(ctx, hsa::launch_gemm(ctx->c, g, &why), what, why);
}

// x[idx[m]] += gate * GELU(u W_1^T) W_2^T with u = LN(x[idx[m]]) * (1 + scale) + shift.
hsa_status mlp_residual(hsa_ctx* ctx, const void* w_1, const void* w_2, float* x,
                        const int32_t* idx, int n, const float* shift, const float* scale,
                        const float* gate) {
  Ctx& c = ctx->c;
  const int D = c.cfg.D, F = c.cfg.F;
  cudaError_t e = hsa::launch_ln_gather(c, x, idx, n, c.u, shift, scale);
  if (e != cudaSuccess) return cuda_fail(ctx, e, "ln_gather");
  std::string why;
  hsa::GemmArgs up{};
  up.A = c.u;
  up.B = w_1;
  up.M = n;
  up.Ncols = F;
  up.Kd = D;
  up.epi = hsa::EPI_GELU;
  up.out = c.hmid;
  up.ld_out = F;
  e = hsa::launch_gemm(c, up, &why);
  if (e != cudaSuccess) return launched(ctx, e, "mlp_up", why);
  hsa::GemmArgs dn{};
  dn.A = c.hmid;
  dn.B = w_2;
  dn.M = n;
  dn.Ncols = D;
  dn.Kd = F;
  dn.epi = hsa::EPI_RESID;
  dn.x = x;
  dn.ld_x = D;
  dn.gate = gate;
  dn.idx = idx;
  dn.N = c.cfg.N;
  return launched(ctx, hsa::launch_gemm(c, dn, &why), "mlp_down", why);
}

}  // namespace

hsa_status hsa_out_proj_residual(hsa_ctx* ctx, const void* w_o, const void* o,
                                 const int32_t* idx, int n, float* x) {
  HSA_CHECK_CTX(ctx);
  if (hsa_status st = check_n(ctx, n)) return st;
  if (n == 0) return HSA_OK;
  HSA_CHECK_PTR(ctx, w_o);
  HSA_CHECK_PTR(ctx, o);
  HSA_CHECK_PTR(ctx, idx);
  HSA_CHECK_PTR(ctx, x);
  return proj_residual(ctx, w_o, o, idx, n, x, nullptr, "out_proj");
}


hsa_status hsa_out_proj_residual_gated(hsa_ctx* ctx, const void* w_o, const void* o,
                                       const int32_t* idx, int n, float* x, const float* gate) {
  HSA_CHECK_CTX(ctx);
  if (hsa_status st = check_n(ctx, n)) return st;
  if (gate != nullptr && (reinterpret_cast<uintptr_t>(gate) & 15) != 0)
    return fail(ctx, HSA_ERR_INVALID_ARG, "gate must be 16-byte aligned");
  if (n == 0) return HSA_OK;
  HSA_CHECK_PTR(ctx, w_o);
  HSA_CHECK_PTR(ctx, o);
  HSA_CHECK_PTR(ctx, idx);
  HSA_CHECK_PTR(ctx, x);
  return proj_residual(ctx, w_o, o, idx, n, x, gate, "out_proj");
}

hsa_status hsa_ln_gather_mod(hsa_ctx* ctx, const float* x, const int32_t* idx, int n, void* u,
                             const float* shift, const float* scale) {
  HSA_CHECK_CTX(ctx);
  if (hsa_status st = check_n(ctx, n)) return st;
  if ((shift == nullptr) != (scale == nullptr))
    return fail(ctx, HSA_ERR_INVALID_ARG, "shift and scale are given together or not at all");
  if (shift != nullptr) {
    HSA_CHECK_PTR(ctx, shift);
    HSA_CHECK_PTR(ctx, scale);
  }
  if (n == 0) return HSA_OK;
  HSA_CHECK_PTR(ctx, x);
  HSA_CHECK_PTR(ctx, idx);
  HSA_CHECK_PTR(ctx, u);
  return launched(ctx, hsa::launch_ln_gather(ctx->c, x, idx, n, u, shift, scale), "ln_gather");
}

hsa_status hsa_mlp_residual_mod(hsa_ctx* ctx, const void* w_1, const void* w_2, float* x,
                                const int32_t* idx, int n, const float* shift,
                                const float* scale, const float* gate) {
  HSA_CHECK_CTX(ctx);
  if (hsa_status st = check_n(ctx, n)) return st;
  if ((shift == nullptr) != (scale == nullptr))
    return fail(ctx, HSA_ERR_INVALID_ARG, "shift and scale are given together or not at all");
  for (const float* v : {shift, scale, gate})
    if (v != nullptr && (reinterpret_cast<uintptr_t>(v) & 15) != 0)
      return fail(ctx, HSA_ERR_INVALID_ARG, "modulation rows must be 16-byte aligned");
  if (n == 0) return HSA_OK;
  HSA_CHECK_PTR(ctx, w_1);
  HSA_CHECK_PTR(ctx, w_2);
  HSA_CHECK_PTR(ctx, x);
  HSA_CHECK_PTR(ctx, idx);
  return mlp_residual(ctx, w_1, w_2, x, idx, n, shift, scale, gate);
}

hsa_status hsa_mlp_residual(hsa_ctx* ctx, const void* w_1, const void* w_2, float* x,
                            const int32_t* idx, int n) {
  HSA_CHECK_CTX(ctx);
  if (hsa_status st = check_n(ctx, n)) return st;
  if (n == 0) return HSA_OK;
  HSA_CHECK_PTR(ctx, w_1);
  HSA_CHECK_PTR(ctx, w_2);
  HSA_CHECK_PTR(ctx, x);
  HSA_CHECK_PTR(ctx, idx);
  return mlp_residual(ctx, w_1, w_2, x, idx, n, nullptr, nullptr, nullptr);
}

hsa_status hsa_layer_forward(hsa_ctx* ctx, const hsa_layer_weights* w, float* x,
                             const int32_t* idx, int n, void* k_cache, void* v_cache) {
  return hsa_layer_forward_cond(ctx, w, nullptr, nullptr, x, idx, n, k_cache, v_cache);
}

hsa_status hsa_layer_forward_cond(hsa_ctx* ctx, const hsa_layer_weights* w, const float* mod,
                                  const hsa_cross_attn* xa, float* x, const int32_t* idx, int n,
                                  void* k_cache, void* v_cache) {
  HSA_CHECK_CTX(ctx);
  if (w == nullptr) return fail(ctx, HSA_ERR_INVALID_ARG, "w is NULL");
  if (hsa_status st = check_n(ctx, n)) return st;
  if (mod != nullptr && (reinterpret_cast<uintptr_t>(mod) & 15) != 0)
    return fail(ctx, HSA_ERR_INVALID_ARG, "mod must be 16-byte aligned");
  if (xa != nullptr) {
    if (xa->n_txt <= 0) return fail(ctx, HSA_ERR_SHAPE, "cross-attention needs n_txt >= 1");
    HSA_CHECK_PTR(ctx, xa->w_q);
    HSA_CHECK_PTR(ctx, xa->w_o);
    HSA_CHECK_PTR(ctx, xa->k_txt);
    HSA_CHECK_PTR(ctx, xa->v_txt);
  }
  if (n == 0) return HSA_OK;
  Ctx& c = ctx->c;
  const int D = c.cfg.D;
  // mod rows: shift_a, scale_a, gate_a, shift_m, scale_m, gate_m.
  const float* m = mod;
  auto row = [&](int r) { return m == nullptr ? nullptr : m + static_cast<size_t>(r) * D; };
  HSA_CHECK_PTR(ctx, x);
  HSA_CHECK_PTR(ctx, idx);
  cudaError_t e = hsa::launch_ln_gather(c, x, idx, n, c.u, row(0), row(1));
  if (e != cudaSuccess) return cuda_fail(ctx, e, "ln_gather");
  hsa_status st = hsa_qkv_project(ctx, w->w_qkv, c.u, idx, n, c.q, k_cache, v_cache);
  if (st == HSA_OK) st = hsa_attention(ctx, c.q, n, k_cache, v_cache, c.o);
  if (st == HSA_OK) {
    HSA_CHECK_PTR(ctx, w->w_o);
    st = proj_residual(ctx, w->w_o, c.o, idx, n, x, row(2), "out_proj");
  }
  if (st == HSA_OK && xa != nullptr) {
    e = hsa::launch_ln_gather(c, x, idx, n, c.u);
    if (e != cudaSuccess) return cuda_fail(ctx, e, "ln_gather");
    st = hsa_linear(ctx, c.u, n, D, xa->w_q, D, c.q);
    if (st == HSA_OK) st = hsa_attention_kv(ctx, c.q, n, xa->k_txt, xa->v_txt, xa->n_txt, c.o);
    if (st == HSA_OK) st = proj_residual(ctx, xa->w_o, c.o, idx, n, x, nullptr, "cross_out_proj");
  }
  if (st == HSA_OK) {
    HSA_CHECK_PTR(ctx, w->w_1);
    HSA_CHECK_PTR(ctx, w->w_2);
    st = mlp_residual(ctx, w->w_1, w->w_2, x, idx, n, row(3), row(4), row(5));
  }
  return st;
}

hsa_status hsa_embed(hsa_ctx* ctx, const float* w_in, const float* x_lat, const int32_t* idx,
                     int n, float* h) {
  HSA_CHECK_CTX(ctx);
  if (hsa_status st = check_n(ctx, n)) return st;
  if (n == 0) return HSA_OK;
  HSA_CHECK_PTR(ctx, w_in);
  HSA_CHECK_PTR(ctx, x_lat);
  HSA_CHECK_PTR(ctx, idx);
  HSA_CHECK_PTR(ctx, h);
  return launched(ctx, hsa::launch_embed(ctx->c, w_in, x_lat, idx, n, h), "embed");
}

hsa_status hsa_head(hsa_ctx* ctx, const float* w_head, const float* h, const int32_t* idx, int n,
                    float* v_fresh) {
  HSA_CHECK_CTX(ctx);
  if (hsa_status st = check_n(ctx, n)) return st;
  if (n == 0) return HSA_OK;
  HSA_CHECK_PTR(ctx, w_head);
  HSA_CHECK_PTR(ctx, h);
  HSA_CHECK_PTR(ctx, idx);
  HSA_CHECK_PTR(ctx, v_fresh);
  return launched(ctx, hsa::launch_head(ctx->c, w_head, h, idx, n, v_fresh), "head");
}

hsa_status hsa_euler_step(hsa_ctx* ctx, float* x, float* v_hat, float* v_hat_prev,
                          const float* v_fresh, const uint8_t* mask, float sigma_i,
                          float sigma_next) {
  HSA_CHECK_CTX(ctx);
  HSA_CHECK_PTR(ctx, x);
  HSA_CHECK_PTR(ctx, v_hat);
  HSA_CHECK_PTR(ctx, v_hat_prev);
  HSA_CHECK_PTR(ctx, v_fresh);
  HSA_CHECK_PTR(ctx, mask);
  return launched(ctx, hsa::launch_euler(ctx->c, x, v_hat, v_hat_prev, v_fresh, mask, sigma_i,
                                         sigma_next),
                  "euler");
}

hsa_status hsa_euler_step_score(hsa_ctx* ctx, float* x, float* v_hat, float* v_hat_prev,
                                const float* v_fresh, const uint8_t* mask, float sigma_i,
                                float sigma_next, float* score) {
  HSA_CHECK_CTX(ctx);
  HSA_CHECK_PTR(ctx, x);
  HSA_CHECK_PTR(ctx, v_hat);
  HSA_CHECK_PTR(ctx, v_hat_prev);
  HSA_CHECK_PTR(ctx, v_fresh);
  HSA_CHECK_PTR(ctx, mask);
  HSA_CHECK_PTR(ctx, score);
  return launched(ctx, hsa::launch_euler(ctx->c, x, v_hat, v_hat_prev, v_fresh, mask, sigma_i,
                                         sigma_next, score),
                  "euler_score");
}

hsa_status hsa_step(hsa_ctx* ctx, const hsa_model_weights* w, const hsa_state* s, int i,
                    float sigma_i, float sigma_next, int regroup) {
  return hsa_step_cond(ctx, w, s, nullptr, i, sigma_i, sigma_next, regroup);
}

hsa_status hsa_step_cond(hsa_ctx* ctx, const hsa_model_weights* w, const hsa_state* s,
                         const hsa_cond* cond, int i, float sigma_i, float sigma_next,
                         int regroup) {
  HSA_CHECK_CTX(ctx);
  if (w == nullptr || s == nullptr || (w->layers == nullptr && ctx->c.cfg.L > 0))
    return fail(ctx, HSA_ERR_INVALID_ARG, "weights and state must not be NULL");
  if (ctx->c.cfg.L > 0 && (s->k_cache == nullptr || s->v_cache == nullptr))
    return fail(ctx, HSA_ERR_INVALID_ARG, "state needs L cache pointers");
  int n = 0;
  hsa_status st = hsa_schedule(ctx, i, s->g, s->mask, s->active_idx, nullptr, &n);
  if (st == HSA_OK) st = hsa_embed(ctx, w->w_in, s->x, s->active_idx, n, s->h);
  for (int l = 0; st == HSA_OK && l < ctx->c.cfg.L; ++l) {
    const float* mod = (cond != nullptr && cond->mod != nullptr) ? cond->mod[l] : nullptr;
    const hsa_cross_attn* xa = (cond != nullptr && cond->xa != nullptr) ? &cond->xa[l] : nullptr;
    st = hsa_layer_forward_cond(ctx, &w->layers[l], mod, xa, s->h, s->active_idx, n,
                                s->k_cache[l], s->v_cache[l]);
  }
  if (st == HSA_OK) st = hsa_head(ctx, w->w_head, s->h, s->active_idx, n, s->v_fresh);
  // re-grouping from iteration T / s_K on (every token then has two cached
  // velocities), not after the last; its score is written by the Euler pass
  const int from = ctx->c.T / ctx->c.budgets[ctx->c.K - 1];
  const bool regroup_now = regroup && i >= from && i < ctx->c.T - 1;
  if (st == HSA_OK && !regroup_now)
    st = hsa_euler_step(ctx, s->x, s->v_hat, s->v_hat_prev, s->v_fresh, s->mask, sigma_i,
                        sigma_next);
  if (st == HSA_OK && regroup_now)
    st = hsa_euler_step_score(ctx, s->x, s->v_hat, s->v_hat_prev, s->v_fresh, s->mask, sigma_i,
                              sigma_next, s->score);
  if (st == HSA_OK && regroup_now) st = hsa_select_from_score(ctx, s->score, s->g);
  return st;
}

}  // extern "C"
