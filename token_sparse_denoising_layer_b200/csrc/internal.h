// internal.h - context layout and kernel launchers shared by the .cu files of libhsa.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <atomic>
#include <string>
#include <vector>

#include "../../include/hsa.h"

namespace hsa {

constexpr int kMaxGroups = 8;
constexpr int kMaxCaches = 8;  // copies of a KV cache one QKV launch can write (ranks of a step)

// Bits a kernel can set in the context's device flag (read by hsa_sync_check).
enum : int { DEV_OK = 0, DEV_TIMEOUT = 1, DEV_BAD_INDEX = 2, DEV_BAD_SCORE = 4, DEV_BAD_GROUP = 8 };
constexpr int kRadixBins = 256;
// Attention work split: the units of the last, partial wave are split into
// at most kMaxSplitParts key ranges each, and into at most kMaxAttnParts
// parts in total (their partial results live in the context's scratch:
// kMaxAttnParts x 256 rows x 128 fp32 = 64 MiB).
constexpr int kMaxSplitParts = 32;
constexpr int kMaxAttnParts = 512;

// Kernel classes timed by hsa_time_kernels (CUDA events around each launch).
enum TimeClass : int { TC_ATTN = 0, TC_GEMM = 1, TC_ROWS = 2, TC_TOKENS = 3, TC_COUNT = 4 };

struct TimeRec {
  std::vector<cudaEvent_t> pairs;  // start, stop, start, stop, ...
  uint64_t calls = 0;
  double work = 0.0;  // algorithmic FLOP (attention, GEMM) or bytes (rows, tokens)
};

struct Ctx {
  hsa_model_cfg cfg{};
  int T = 0, K = 0, m = 0;
  int budgets[kMaxGroups]{};
  int counts[kMaxGroups]{};
  int strides[kMaxGroups]{};
  cudaStream_t stream = nullptr;
  int device = 0;
  int num_sms = 148;
  std::string err;
  mutable uint64_t launches = 0;  // kernels launched through this context
  // scratch (device)
  void* u = nullptr;      // bf16 [N, D] LN output of the active rows
  void* q = nullptr;      // bf16 [N, D] compact queries
  void* o = nullptr;      // bf16 [N, D] compact attention output
  void* hmid = nullptr;   // bf16 [N, F] compact MLP hidden
  float* attn_part_o = nullptr;   // [kMaxAttnParts][256][128] attention partial O
  float* attn_part_ml = nullptr;  // [kMaxAttnParts][256][2] partial (max, sum)
  uint32_t* cuts = nullptr;  // selector cut keys, 2 words per cut
  int* flag = nullptr;       // device error flag
  // per-launch timing (off unless hsa_time_kernels turned it on)
  mutable bool timing = false;
  mutable TimeRec times[TC_COUNT];
  mutable std::vector<cudaEvent_t> event_pool;
  cudaEvent_t take_event() const {
    cudaEvent_t e = nullptr;
    if (!event_pool.empty()) {
      e = event_pool.back();
      event_pool.pop_back();
    } else if (cudaEventCreate(&e) != cudaSuccess) {
      e = nullptr;
    }
    return e;
  }
};

// While timing is on, brackets the launches made in its scope with two CUDA
// events on the context's stream and adds `work` to the class's total.
class Timed {
 public:
  Timed(const Ctx& c, int cls, double work) : c_(c), cls_(cls) {
    if (!c_.timing) return;
    start_ = c_.take_event();
    if (start_ != nullptr) cudaEventRecord(start_, c_.stream);
    c_.times[cls_].work += work;
    c_.times[cls_].calls += 1;
  }
  ~Timed() {
    if (!c_.timing || start_ == nullptr) return;
    cudaEvent_t stop = c_.take_event();
    if (stop == nullptr) return;
    cudaEventRecord(stop, c_.stream);
    c_.times[cls_].pairs.push_back(start_);
    c_.times[cls_].pairs.push_back(stop);
  }
  Timed(const Timed&) = delete;
  Timed& operator=(const Timed&) = delete;

 private:
  const Ctx& c_;
  int cls_;
  cudaEvent_t start_ = nullptr;
};

// Row-index guard used by kernels that follow idx: out-of-range rows are
// skipped and reported through the device flag.
__device__ __forceinline__ bool row_ok(int32_t r, int N, int* flag) {
  if (static_cast<uint32_t>(r) < static_cast<uint32_t>(N)) return true;
  atomicOr(flag, DEV_BAD_INDEX);
  return false;
}

// Raise a kernel's dynamic shared-memory limit, once per device (bit d of `done`).
template <typename Kernel>
cudaError_t ensure_smem_limit(Kernel* kernel, int bytes, int device, std::atomic<uint64_t>& done) {
  const uint64_t bit = 1ull << (device & 63);
  if (done.load(std::memory_order_acquire) & bit) return cudaSuccess;
  const cudaError_t e =
      cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  if (e == cudaSuccess) done.fetch_or(bit, std::memory_order_acq_rel);
  return e;
}

// ---- launchers (return cudaGetLastError() of the launch)
cudaError_t launch_schedule(const Ctx& c, int i, const uint8_t* g, uint8_t* mask, int32_t* idx,
                            int32_t* n_dev);
cudaError_t launch_score(const Ctx& c, const float* v_prev, const float* v_cur, float* score);
cudaError_t launch_select(const Ctx& c, const float* score, uint8_t* g);
cudaError_t launch_select_groups_raw(cudaStream_t stream, const float* v_prev, const float* v_cur,
                                     int N, const int* counts, int K, float* score,
                                     uint32_t* cuts, uint8_t* g, int* flag);
cudaError_t launch_selftest_timeout(const Ctx& c, uint64_t limit_ns);
// With `score` set, the same pass also writes the re-grouping score of every
// token from the updated (v_hat_prev, v_hat), bit for bit as launch_score does.
cudaError_t launch_euler(const Ctx& c, float* x, float* v_hat, float* v_hat_prev,
                         const float* v_fresh, const uint8_t* mask, float s0, float s1,
                         float* score = nullptr);
cudaError_t launch_ln_gather(const Ctx& c, const float* x, const int32_t* idx, int n, void* u,
                             const float* shift = nullptr, const float* scale = nullptr);
cudaError_t launch_kv_scatter(const Ctx& c, const void* k_rows, const void* v_rows, int src_ld,
                              const int32_t* idx, int n, void* kc, void* vc);
cudaError_t launch_embed(const Ctx& c, const float* w_in, const float* x_lat, const int32_t* idx,
                         int n, float* h);
cudaError_t launch_head(const Ctx& c, const float* w_head, const float* h, const int32_t* idx,
                        int n, float* v_fresh);

// GEMM epilogues: C[m, j] = sum_k A[m, k] * B[j, k]  (A [M, K], B [Ncols, K], both bf16).
enum GemmEpi : int {
  EPI_STORE = 0,  // out bf16 [M, Ncols]
  EPI_QKV = 1,    // Q -> out [M, D]; K, V -> caches rows idx[m]
  EPI_RESID = 2,  // x[idx[m], j] += C  (fp32)
  EPI_GELU = 3,   // out bf16 [M, Ncols] = GELU(C)
};

struct GemmArgs {
  const void* A;   // bf16 [M, Kd]
  const void* B;   // bf16 [Ncols, Kd]
  int M, Ncols, Kd;
  int epi;
  void* out;          // EPI_STORE / EPI_GELU / EPI_QKV (Q)
  int ld_out;         // elements
  void* k_cache;      // EPI_QKV
  void* v_cache;      // EPI_QKV
  // EPI_QKV into several copies of the caches (this GPU's and peers' over
  // NVLink): when n_caches > 0, every fresh K/V row goes to rows idx[m] of
  // k_caches[0 .. n_caches) and v_caches[..] instead of k_cache / v_cache
  int n_caches = 0;
  void* k_caches[kMaxCaches]{};
  void* v_caches[kMaxCaches]{};
  float* x;           // EPI_RESID
  int ld_x;
  const float* gate = nullptr;  // EPI_RESID: x[.., j] += gate[j] * C (fp32 [Ncols]) if set
  const int32_t* idx; // EPI_QKV / EPI_RESID
  int N;              // rows of caches / x (bounds for idx)
};

cudaError_t launch_gemm(const Ctx& c, const GemmArgs& a, std::string* why);

// Attention of n queries against n_kv key/value rows (row stride D).
cudaError_t launch_attention(const Ctx& c, const void* q, int n, const void* kc, const void* vc,
                             int n_kv, void* o, std::string* why);

// TMA descriptor for a row-major bf16 matrix [rows, cols] with a
// box of [box_rows, 64] and 128-byte swizzle.  Returns false on failure.
bool make_tmap_bf16(CUtensorMap* map, const void* base, uint64_t rows, uint64_t cols,
                    uint64_t row_stride_elems, uint32_t box_rows, std::string* why);

}  // namespace hsa
