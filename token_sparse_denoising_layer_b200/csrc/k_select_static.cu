// k_select_static.cu - group selection that allocates no device memory.
//
// hsa_select_groups needs a context, and hsa_create allocates the context's
// scratch with cudaMalloc.  Some callers cannot do that: a host framework
// that owns every byte of device memory through its own pool and forbids a
// library from allocating behind its back, or a latency-critical serving loop
// where cudaMalloc's implicit device-wide synchronisation would stall other
// streams.  hsa_select_groups_static gives them the same selection (scores,
// exact radix cut search, group assignment) with its scratch -- the per-token
// scores and the cut keys -- in one file-scope device array of fixed size.
//
// That array exists once per GPU that loads this library and stays allocated
// until the process exits.  Every call shares it and it keeps the previous
// call's contents; calls that overlap on the GPU (on two streams, or from two
// threads) race on it.

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <mutex>

#include "../../include/hsa.h"
#include "internal.h"

namespace {

constexpr int kStaticMaxN = HSA_SELECT_STATIC_MAX_N;
constexpr size_t kScoreBytes = static_cast<size_t>(kStaticMaxN) * sizeof(float);
constexpr size_t kCutBytes = 2 * hsa::kMaxGroups * sizeof(uint32_t);
constexpr size_t kScratchBytes = kScoreBytes + kCutBytes + 256;

// scores [kStaticMaxN] fp32 | cut keys [16] u32 | error flag (int) at an aligned offset
static __device__ __align__(256) unsigned char g_select_scratch[kScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_setup_mutex;
void* g_scratch_addr[kMaxDevices] = {};
unsigned long long g_scratch_ctx[kMaxDevices] = {};  // id of the context the address is for

// Unique id of the current CUDA context (cuCtxGetId, through the runtime's
// driver entry point), or 0 when the driver cannot say.
unsigned long long current_context_id() {
  typedef CUresult (*GetCurrentFn)(CUcontext*);
  typedef CUresult (*GetIdFn)(CUcontext, unsigned long long*);
  static GetCurrentFn get_current = nullptr;
  static GetIdFn get_id = nullptr;
  static bool looked = false;
  if (!looked) {
    void* a = nullptr;
    void* b = nullptr;
    cudaDriverEntryPointQueryResult qa, qb;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &a, cudaEnableDefault, &qa) == cudaSuccess &&
        qa == cudaDriverEntryPointSuccess &&
        cudaGetDriverEntryPoint("cuCtxGetId", &b, cudaEnableDefault, &qb) == cudaSuccess &&
        qb == cudaDriverEntryPointSuccess) {
      get_current = reinterpret_cast<GetCurrentFn>(a);
      get_id = reinterpret_cast<GetIdFn>(b);
    }
    looked = true;
  }
  CUcontext ctx = nullptr;
  unsigned long long id = 0;
  if (get_current == nullptr || get_id == nullptr || get_current(&ctx) != CUDA_SUCCESS ||
      ctx == nullptr || get_id(ctx, &id) != CUDA_SUCCESS)
    return 0;
  return id;
}

// Device address of the scratch array on the current device.  In host code
// the array's name is only a host-side stand-in.  The address is looked up
// once per device and context: the first call on a device does it, and so
// does the first call after a device reset replaced the context (or every
// call, if the context cannot be identified).  Errors are reported by status
// code only: this entry point has no context to hold a message.
hsa_status scratch_address(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return HSA_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return HSA_ERR_INVALID_ARG;
  std::lock_guard<std::mutex> lock(g_setup_mutex);
  const unsigned long long ctx_id = current_context_id();
  if (g_scratch_addr[dev] == nullptr || ctx_id == 0 || ctx_id != g_scratch_ctx[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_select_scratch) != cudaSuccess || p == nullptr)
      return HSA_ERR_CUDA;
    g_scratch_addr[dev] = p;
    g_scratch_ctx[dev] = ctx_id;
  }
  *out = g_scratch_addr[dev];
  return HSA_OK;
}

bool aligned16(const void* p) { return p != nullptr && (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace

extern "C" {

hsa_status hsa_select_groups_static(const float* v_prev, const float* v_cur, int N,
                                    const int* counts, int K, uint8_t* g, void* stream) {
  if (N > kStaticMaxN) return HSA_ERR_SCRATCH_LIMIT;  // beyond the static scratch
  if (N < 1 || K < 1 || K > hsa::kMaxGroups || counts == nullptr) return HSA_ERR_INVALID_ARG;
  long long total = 0;
  for (int k = 0; k < K; ++k) {
    if (counts[k] < 0) return HSA_ERR_BUDGET;
    total += counts[k];
  }
  if (total != N) return HSA_ERR_BUDGET;  // group counts must sum to N
  if (!aligned16(v_prev) || !aligned16(v_cur) || !aligned16(g)) return HSA_ERR_INVALID_ARG;
  void* base = nullptr;
  if (hsa_status st = scratch_address(&base)) return st;
  auto* bytes = static_cast<unsigned char*>(base);
  float* score = reinterpret_cast<float*>(bytes);
  uint32_t* cuts = reinterpret_cast<uint32_t*>(bytes + kScoreBytes);
  int* flag = reinterpret_cast<int*>(bytes + kScoreBytes + kCutBytes);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  // the device check flag must start at zero; scores and cuts are fully rewritten
  cudaError_t e = cudaMemsetAsync(flag, 0, sizeof(int), s);
  if (e == cudaSuccess)
    e = hsa::launch_select_groups_raw(s, v_prev, v_cur, N, counts, K, score, cuts, g, flag);
  return e == cudaSuccess ? HSA_OK : HSA_ERR_CUDA;
}

}  // extern "C"
