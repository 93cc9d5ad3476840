// k_attn.cu - full-context attention of the active queries against the
// per-layer KV cache, on the 5th-generation tensor cores.
//
// "Technical Summary: Heterogeneous Step Allocation (HSA) for Efficient Video
// Generation", section 2.2, steps 3-4: the |A_i| active tokens compute
// queries against the full cached K, V (fresh rows for active tokens, stale
// rows for skipped ones), which costs O(|A_i| * N) instead of O(N^2).
//
// One CTA = 128 queries x one head.  Per 128-key tile j:
//   S_j = Q K_j^T            tcgen05.mma, fp32 in TMEM (double-buffered)
//   P_j = exp2(S_j*c - m)    softmax warps, bf16 into 128B-swizzled smem
//   O  += P_j V_j            tcgen05.mma, fp32 in TMEM
// The running max m is only raised when a row's max grows by more than 2^8
// (then O and l are rescaled in TMEM/registers); otherwise the stale max is
// kept, which is exact because the same m scales both O and l.
// Warp 0: TMA producer.  Warp 1: TMEM owner and MMA issuer.  Warps 2..5:
// softmax, rescale and the output epilogue (warp w owns TMEM lanes 32*(w%4)).

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>

#include <string>

#include "internal.h"
#include "ptx.cuh"

namespace hsa {

namespace {

constexpr int kQ = 128;        // queries per CTA
constexpr int kKV = 128;       // keys per tile
constexpr int kKStages = 2;
constexpr int kVStages = 2;
constexpr int kAttnThreads = 192;
constexpr uint32_t kTmemCols = 512;
constexpr float kRescaleThreshold = 8.0f;  // log2 units

template <int HD>
struct AttnCfg {
  static constexpr int kRegions = HD / 64;          // 64-element (128 B) column regions
  static constexpr int kRegionBytes = 128 * 128;    // 128 rows x 128 B
  static constexpr int kTileBytes = kRegions * kRegionBytes;  // Q, K or V tile
  static constexpr int kPBytes = 2 * kRegionBytes;  // P: 128 x 128 bf16
  static constexpr int kSmemData = kTileBytes * (1 + kKStages + kVStages) + kPBytes;
  // The HD=64 kernel pads its request so that only one CTA is resident per
  // SM: every CTA allocates all 512 TMEM columns.
  static constexpr int kSmem = (HD == 64 ? 160 * 1024 : kSmemData + 1024 + 256);
};

struct AttnParams {
  int n;        // active queries
  int N;        // cached rows
  int H;
  float scale_log2;  // log2(e) / sqrt(d)
  __nv_bfloat16* o;
  int ld;       // D
  int* flag;
};

template <int HD>
__global__ void __launch_bounds__(kAttnThreads, 1)
    k_attn(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
           const __grid_constant__ CUtensorMap tmV, AttnParams p) {
  using Cfg = AttnCfg<HD>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint8_t* sQ = smem;
  uint8_t* sK = sQ + Cfg::kTileBytes;
  uint8_t* sV = sK + kKStages * Cfg::kTileBytes;
  uint8_t* sP = sV + kVStages * Cfg::kTileBytes;
  uint64_t* bars = reinterpret_cast<uint64_t*>(sP + Cfg::kPBytes);
  uint64_t* q_full = bars;
  uint64_t* k_full = bars + 1;
  uint64_t* k_empty = k_full + kKStages;
  uint64_t* v_full = k_empty + kKStages;
  uint64_t* v_empty = v_full + kVStages;
  uint64_t* s_full = v_empty + kVStages;  // [2]
  uint64_t* p_full = s_full + 2;
  uint64_t* pv_done = p_full + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(pv_done + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int q0 = blockIdx.x * kQ;
  const int h = blockIdx.y;
  const int col0 = h * HD;
  const int nkv = (p.N + kKV - 1) / kKV;

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    for (int s = 0; s < kKStages; ++s) {
      mbar_init(&k_full[s], 1);
      mbar_init(&k_empty[s], 1);
    }
    for (int s = 0; s < kVStages; ++s) {
      mbar_init(&v_full[s], 1);
      mbar_init(&v_empty[s], 1);
    }
    mbar_init(&s_full[0], 1);
    mbar_init(&s_full[1], 1);
    mbar_init(p_full, 128);
    mbar_init(pv_done, 1);
    fence_barrier_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tmQ);
    tma_prefetch_desc(&tmK);
    tma_prefetch_desc(&tmV);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t tS = tmem;              // S buffers at columns 0 and 128
  const uint32_t tO = tmem + 2 * kKV;    // O at column 256
  bool ok = true;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      const uint64_t keep = l2_policy_evict_last();  // K/V of a head is shared by its q-tiles
      mbar_arrive_expect_tx(q_full, Cfg::kTileBytes);
      for (int r = 0; r < Cfg::kRegions; ++r)
        tma_load_2d(sQ + r * Cfg::kRegionBytes, &tmQ, q_full, col0 + 64 * r, q0);
      for (int j = 0; j < nkv && ok; ++j) {
        const int ks = j % kKStages;
        if (!mbar_wait(&k_empty[ks], ((j / kKStages) & 1) ^ 1)) {
          ok = false;
          break;
        }
        mbar_arrive_expect_tx(&k_full[ks], Cfg::kTileBytes);
        for (int r = 0; r < Cfg::kRegions; ++r)
          tma_load_2d_hint(sK + ks * Cfg::kTileBytes + r * Cfg::kRegionBytes, &tmK, &k_full[ks],
                           col0 + 64 * r, j * kKV, keep);
        const int vs = j % kVStages;
        if (!mbar_wait(&v_empty[vs], ((j / kVStages) & 1) ^ 1)) {
          ok = false;
          break;
        }
        mbar_arrive_expect_tx(&v_full[vs], Cfg::kTileBytes);
        for (int r = 0; r < Cfg::kRegions; ++r)
          tma_load_2d_hint(sV + vs * Cfg::kTileBytes + r * Cfg::kRegionBytes, &tmV, &v_full[vs],
                           col0 + 64 * r, j * kKV, keep);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idS = idesc_bf16(kQ, kKV, false, false);
      constexpr uint32_t idPV = idesc_bf16(kQ, HD, false, true);
      const uint32_t q_addr = smem_u32(sQ);
      const uint32_t p_addr = smem_u32(sP);
      auto issue_s = [&](int j) -> bool {
        const int ks = j % kKStages;
        if (!mbar_wait(&k_full[ks], (j / kKStages) & 1)) return false;
        tc_fence_after();
        const uint32_t k_addr = smem_u32(sK + ks * Cfg::kTileBytes);
#pragma unroll
        for (int kk = 0; kk < HD / 16; ++kk) {
          const uint32_t off = (kk >> 2) * Cfg::kRegionBytes + (kk & 3) * 32;
          umma_bf16(tS + (j & 1) * kKV, sdesc_sw128(q_addr + off, 16, 1024),
                    sdesc_sw128(k_addr + off, 16, 1024), idS, kk > 0 ? 1u : 0u);
        }
        umma_commit(&s_full[j & 1]);
        umma_commit(&k_empty[ks]);
        return true;
      };
      if (!mbar_wait(q_full, 0)) ok = false;
      if (ok && !issue_s(0)) ok = false;
      for (int j = 0; j < nkv && ok; ++j) {
        if (j + 1 < nkv && !issue_s(j + 1)) {
          ok = false;
          break;
        }
        if (!mbar_wait(p_full, j & 1)) {
          ok = false;
          break;
        }
        const int vs = j % kVStages;
        if (!mbar_wait(&v_full[vs], (j / kVStages) & 1)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t v_addr = smem_u32(sV + vs * Cfg::kTileBytes);
#pragma unroll
        for (int kk = 0; kk < kKV / 16; ++kk) {
          const uint32_t a_off = (kk >> 2) * Cfg::kRegionBytes + (kk & 3) * 32;
          // V tile is MN-major for this product: rows = keys (K), 128 B of head dim
          // per row; 16 keys per step = 2048 B; regions of 64 dims are LBO apart.
          umma_bf16(tO, sdesc_sw128(p_addr + a_off, 16, 1024),
                    sdesc_sw128(v_addr + kk * 2048, Cfg::kRegionBytes, 1024), idPV,
                    (j > 0 || kk > 0) ? 1u : 0u);
        }
        umma_commit(pv_done);
        umma_commit(&v_empty[vs]);
      }
    }
  } else {
    // ------------------------------------------------------------ softmax warps
    const int qd = warp & 3;
    const int row = 32 * qd + lane;
    const uint32_t lane_base = static_cast<uint32_t>(32 * qd) << 16;
    float m_run = -INFINITY, l_run = 0.f;
    uint8_t* prow = sP + row * 128;
    const int sw = row & 7;
    for (int j = 0; j < nkv; ++j) {
      if (!__all_sync(0xffffffffu, mbar_wait(&s_full[j & 1], (j >> 1) & 1))) {
        ok = false;
        break;
      }
      tc_fence_after();
      float s[kKV];
#pragma unroll
      for (int c = 0; c < kKV / 32; ++c) {
        uint32_t r[32];
        tmem_ld32(tS + lane_base + (j & 1) * kKV + 32 * c, r);
#pragma unroll
        for (int e = 0; e < 32; ++e) s[32 * c + e] = __uint_as_float(r[e]);
      }
      const int valid = p.N - j * kKV;  // keys past N are zero-filled: mask them
      float tmax = -INFINITY;
#pragma unroll
      for (int e = 0; e < kKV; ++e) {
        s[e] = (e < valid) ? s[e] * p.scale_log2 : -INFINITY;
        tmax = fmaxf(tmax, s[e]);
      }
      const bool raise = tmax > m_run + kRescaleThreshold;
      const float m_use = raise ? tmax : m_run;
      const float alpha = raise ? ex2_approx(m_run - m_use) : 1.0f;
      // PV_{j-1} must be done before P is overwritten and before O is rescaled.
      if (j > 0 && !__all_sync(0xffffffffu, mbar_wait(pv_done, (j - 1) & 1))) {
        ok = false;
        break;
      }
      float rs = 0.f;
#pragma unroll
      for (int c = 0; c < kKV / 8; ++c) {  // 16-byte chunks of 8 keys
        float pv[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          pv[e] = ex2_approx(s[8 * c + e] - m_use);
          rs += pv[e];
        }
        const uint4 w = make_uint4(pack_bf16(pv[0], pv[1]), pack_bf16(pv[2], pv[3]),
                                   pack_bf16(pv[4], pv[5]), pack_bf16(pv[6], pv[7]));
        const int region = c >> 3, cc = c & 7;
        *reinterpret_cast<uint4*>(prow + region * Cfg::kRegionBytes + ((cc ^ sw) << 4)) = w;
      }
      l_run = l_run * alpha + rs;
      m_run = m_use;
      if (j > 0 && __any_sync(0xffffffffu, raise)) {
#pragma unroll 1
        for (int c = 0; c < HD / 32; ++c) {
          uint32_t r[32];
          tmem_ld32(tO + lane_base + 32 * c, r);
#pragma unroll
          for (int e = 0; e < 32; ++e) r[e] = __float_as_uint(__uint_as_float(r[e]) * alpha);
          tmem_st32(tO + lane_base + 32 * c, r);
        }
      }
      fence_proxy_async_smem();
      tc_fence_before();
      mbar_arrive(p_full);
    }
    // epilogue: O / l -> bf16 rows of the compact output
    if (ok && __all_sync(0xffffffffu, mbar_wait(pv_done, (nkv - 1) & 1))) {
      tc_fence_after();
      const float inv = 1.0f / l_run;
      const int qrow = q0 + row;
      __nv_bfloat16* orow = p.o + static_cast<size_t>(qrow) * p.ld + col0;
#pragma unroll 1
      for (int c = 0; c < HD / 32; ++c) {
        uint32_t r[32];
        __syncwarp();
        tmem_ld32(tO + lane_base + 32 * c, r);
        if (qrow < p.n) {
          uint4* d4 = reinterpret_cast<uint4*>(orow + 32 * c);
#pragma unroll
          for (int v = 0; v < 4; ++v)
            d4[v] = make_uint4(
                pack_bf16(__uint_as_float(r[8 * v]) * inv, __uint_as_float(r[8 * v + 1]) * inv),
                pack_bf16(__uint_as_float(r[8 * v + 2]) * inv, __uint_as_float(r[8 * v + 3]) * inv),
                pack_bf16(__uint_as_float(r[8 * v + 4]) * inv, __uint_as_float(r[8 * v + 5]) * inv),
                pack_bf16(__uint_as_float(r[8 * v + 6]) * inv, __uint_as_float(r[8 * v + 7]) * inv));
        }
      }
    } else {
      ok = false;
    }
  }
  if (!ok) atomicOr(p.flag, DEV_TIMEOUT);
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

template <int HD>
cudaError_t launch_hd(const Ctx& c, const void* q, int n, const void* kc, const void* vc, void* o,
                      std::string* why) {
  const int D = c.cfg.D, N = c.cfg.N;
  CUtensorMap tq, tk, tv;
  if (!make_tmap_bf16(&tq, q, n, D, D, kQ, why)) return cudaErrorInvalidValue;
  if (!make_tmap_bf16(&tk, kc, N, D, D, kKV, why)) return cudaErrorInvalidValue;
  if (!make_tmap_bf16(&tv, vc, N, D, D, kKV, why)) return cudaErrorInvalidValue;
  AttnParams p{};
  p.n = n;
  p.N = N;
  p.H = c.cfg.H;
  p.scale_log2 = static_cast<float>(1.4426950408889634 / sqrt(static_cast<double>(HD)));
  p.o = static_cast<__nv_bfloat16*>(o);
  p.ld = D;
  p.flag = c.flag;
  constexpr int smem = AttnCfg<HD>::kSmem;
  static bool attr_set = false;
  if (!attr_set) {
    cudaError_t e =
        cudaFuncSetAttribute(k_attn<HD>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    attr_set = true;
  }
  const dim3 grid((n + kQ - 1) / kQ, c.cfg.H);
  k_attn<HD><<<grid, kAttnThreads, smem, c.stream>>>(tq, tk, tv, p);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_attention(const Ctx& c, const void* q, int n, const void* kc, const void* vc,
                             void* o, std::string* why) {
  if (n <= 0) return cudaSuccess;
  const int d = c.cfg.D / c.cfg.H;
  if (d == 128) return launch_hd<128>(c, q, n, kc, vc, o, why);
  if (d == 64) return launch_hd<64>(c, q, n, kc, vc, o, why);
  if (why) *why = "attention supports head_dim 64 or 128";
  return cudaErrorInvalidValue;
}

}  // namespace hsa
