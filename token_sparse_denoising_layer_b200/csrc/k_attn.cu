// k_attn.cu - full-context attention of the active queries against the
// per-layer KV cache, on the 5th-generation tensor cores.
//
// "Technical Summary: Heterogeneous Step Allocation (HSA) for Efficient Video
// Generation", section 2.2, steps 3-4: the |A_i| active tokens compute
// queries against the full cached K, V (fresh rows for active tokens, stale
// rows for skipped ones), which costs O(|A_i| * N) instead of O(N^2).
//
// One CTA = two 128-query tiles (t = 0, 1) of one head; both share every
// 128-key K/V tile the producer streams in.  Per key tile j and query tile t:
//   S_t = Q_t K_j^T          tcgen05.mma, fp32 in TMEM
//   P_t = exp2(S_t*c - m_t)  softmax warpgroup t, written back into TMEM as
//                            bf16 over the columns of S_t
//   O_t += P_t V_j           tcgen05.mma with A = P_t read from TMEM
// The two query tiles ping-pong: while warpgroup 0 turns S_0 into P_0, the
// tensor core runs P_1 V and the next Q_1 K^T, and the other way round.
// The running max m is set by the first key tile and raised only when a
// tile's P would pass 2^64 (seen from its row sum, so no row-max pass precedes
// the exponentials); otherwise the stale max is kept, which is exact because
// the same m scales both O and the row sum l.  A commit that signals S_t(j+1) also covers the
// earlier P_t(j) V_j, so softmax sees a stable O_t and a free P_t region.
//
// Warp 0: TMA producer.  Warp 1: TMEM owner and MMA issuer.  Warps 2..5 and
// 6..9: the softmax warpgroups of tiles 0 and 1 (warp w reads TMEM lanes
// 32*(w%4)..+31), which also rescale O and write the output.

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

constexpr int kQ = 128;        // queries per tile
constexpr int kKV = 128;       // keys per tile
constexpr int kStages = 2;     // K and V ring depth
constexpr int kAttnThreads = 320;
constexpr uint32_t kTmemCols = 512;

template <int HD>
struct AttnCfg {
  static constexpr int kRegions = HD / 64;          // 64-element (128 B) column regions
  static constexpr int kRegionBytes = 128 * 128;    // 128 rows x 128 B
  static constexpr int kTileBytes = kRegions * kRegionBytes;  // one Q, K or V tile
  static constexpr int kSmemData = kTileBytes * (2 + 2 * kStages);
  // Every CTA allocates all 512 TMEM columns, so only one may be resident
  // per SM: the HD=64 kernel pads its shared-memory request to ensure that.
  static constexpr int kSmem = (HD == 64 ? 160 * 1024 : kSmemData + 1024 + 256);
  static constexpr uint32_t kColS0 = 0, kColS1 = 128, kColO0 = 256, kColO1 = 256 + HD;
};

struct AttnParams {
  int n;             // active queries
  int N;             // cached rows
  float scale_log2;  // log2(e) / sqrt(d)
  __nv_bfloat16* o;
  int ld;            // D
  int* flag;
  // Work decomposition.  A unit is one (pair of query tiles, head), ordered
  // head-major.  CTAs [0, n_full) each do a whole unit; the remaining
  // units (the last, partial wave) are each split into `split` key ranges,
  // one CTA per range, which write unnormalised partial results that
  // k_attn_combine merges.
  int n_qpairs;      // units per head
  int n_full;        // units done whole
  int split;         // key-range parts per remaining unit
  float* part_o;     // [part][256 rows][HD] fp32, unnormalised
  float2* part_ml;   // [part][256 rows] (running max, row sum)
};

// Largest P (and so row sum) a tile may reach before the running max must be
// raised: far inside the range of bf16 and of the fp32 row sums and O.
constexpr float kSumLimit = 18446744073709551616.0f;  // 2^64

__device__ __forceinline__ float row_max(const uint32_t (&sr)[kKV]) {
  float mx[8];
#pragma unroll
  for (int u = 0; u < 8; ++u) mx[u] = __uint_as_float(sr[u]);
#pragma unroll
  for (int e = 8; e < kKV; ++e) mx[e & 7] = fmaxf(mx[e & 7], __uint_as_float(sr[e]));
  return fmaxf(fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3])),
               fmaxf(fmaxf(mx[4], mx[5]), fmaxf(mx[6], mx[7])));
}

// P = exp2(S*c - m) as bf16 pairs in w (packed f32x2 arithmetic: two lanes
// per FMA/add instruction); returns the row sum of P.
__device__ __forceinline__ float exp_row(const uint32_t (&sr)[kKV], float c, float m,
                                         uint32_t (&w)[kKV / 2]) {
  float rs0[4] = {0.f, 0.f, 0.f, 0.f}, rs1[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
  for (int e = 0; e < kKV; e += 2) {
    float xa, xb;
    fma2(xa, xb, __uint_as_float(sr[e]), __uint_as_float(sr[e + 1]), c, -m);
    const float a = ex2_approx(xa);
    const float b = ex2_approx(xb);
    add2(rs0[(e >> 1) & 3], rs1[(e >> 1) & 3], a, b);
    w[e / 2] = pack_bf16(a, b);
  }
  return ((rs0[0] + rs1[0]) + (rs0[1] + rs1[1])) + ((rs0[2] + rs1[2]) + (rs0[3] + rs1[3]));
}

template <int HD>
__global__ void __launch_bounds__(kAttnThreads, 1)
    k_attn(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
           const __grid_constant__ CUtensorMap tmV, AttnParams p) {
  using Cfg = AttnCfg<HD>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint8_t* sQ = smem;                              // [2] tiles
  uint8_t* sK = sQ + 2 * Cfg::kTileBytes;          // [kStages]
  uint8_t* sV = sK + kStages * Cfg::kTileBytes;    // [kStages]
  uint64_t* bars = reinterpret_cast<uint64_t*>(sV + kStages * Cfg::kTileBytes);
  uint64_t* q_full = bars;
  uint64_t* k_full = q_full + 1;
  uint64_t* k_empty = k_full + kStages;
  uint64_t* v_full = k_empty + kStages;
  uint64_t* v_empty = v_full + kStages;
  uint64_t* s_full = v_empty + kStages;  // [2] per query tile
  uint64_t* p_full = s_full + 2;         // [2]
  uint64_t* o_done = p_full + 2;         // [2]
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(o_done + 2);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nkv_all = (p.N + kKV - 1) / kKV;
  int unit, part = -1, j0 = 0, nkv = nkv_all;
  if (static_cast<int>(blockIdx.x) < p.n_full) {
    unit = blockIdx.x;
  } else {
    part = blockIdx.x - p.n_full;
    unit = p.n_full + part / p.split;
    const int piece = part % p.split;
    j0 = piece * nkv_all / p.split;
    nkv = (piece + 1) * nkv_all / p.split - j0;  // key tiles j0 .. j0+nkv-1
  }
  const int q0 = (unit % p.n_qpairs) * (2 * kQ);
  const int h = unit / p.n_qpairs;
  const int col0 = h * HD;
  const int ntile = (q0 + kQ < p.n) ? 2 : 1;  // second query tile empty on the last CTA

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&k_full[s], 1);
      mbar_init(&k_empty[s], 1);
      mbar_init(&v_full[s], 1);
      mbar_init(&v_empty[s], 1);
    }
    for (int t = 0; t < 2; ++t) {
      mbar_init(&s_full[t], 1);
      mbar_init(&p_full[t], 4);  // one arrival per softmax warp
      mbar_init(&o_done[t], 1);
    }
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
  bool ok = true;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      const uint64_t keep = l2_policy_evict_last();  // a head's K/V is shared by its q-tiles
      mbar_arrive_expect_tx(q_full, ntile * Cfg::kTileBytes);
      for (int t = 0; t < ntile; ++t)
        for (int r = 0; r < Cfg::kRegions; ++r)
          tma_load_2d(sQ + t * Cfg::kTileBytes + r * Cfg::kRegionBytes, &tmQ, q_full,
                      col0 + 64 * r, q0 + t * kQ);
      for (int j = 0; j < nkv; ++j) {
        const int s = j % kStages;
        const uint32_t ph = ((j / kStages) & 1) ^ 1;
        if (!mbar_wait(&k_empty[s], ph)) {
          ok = false;
          break;
        }
        mbar_arrive_expect_tx(&k_full[s], Cfg::kTileBytes);
        for (int r = 0; r < Cfg::kRegions; ++r)
          tma_load_2d_hint(sK + s * Cfg::kTileBytes + r * Cfg::kRegionBytes, &tmK, &k_full[s],
                           col0 + 64 * r, (j0 + j) * kKV, keep);
        if (!mbar_wait(&v_empty[s], ph)) {
          ok = false;
          break;
        }
        mbar_arrive_expect_tx(&v_full[s], Cfg::kTileBytes);
        for (int r = 0; r < Cfg::kRegions; ++r)
          tma_load_2d_hint(sV + s * Cfg::kTileBytes + r * Cfg::kRegionBytes, &tmV, &v_full[s],
                           col0 + 64 * r, (j0 + j) * kKV, keep);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idS = idesc_bf16(kQ, kKV, false, false);
      constexpr uint32_t idPV = idesc_bf16(kQ, HD, false, true);
      // S_t = Q_t K^T for the K tile in stage s
      auto issue_s = [&](int t, int s) {
        const uint32_t q_addr = smem_u32(sQ + t * Cfg::kTileBytes);
        const uint32_t k_addr = smem_u32(sK + s * Cfg::kTileBytes);
#pragma unroll
        for (int kk = 0; kk < HD / 16; ++kk) {
          const uint32_t off = (kk >> 2) * Cfg::kRegionBytes + (kk & 3) * 32;
          umma_bf16(tmem + (t == 0 ? Cfg::kColS0 : Cfg::kColS1), sdesc_sw128(q_addr + off, 16, 1024),
                    sdesc_sw128(k_addr + off, 16, 1024), idS, kk > 0 ? 1u : 0u);
        }
      };
      // O_t (+)= P_t V for the V tile in stage s; P_t sits in the S_t columns
      auto issue_pv = [&](int t, int s, bool acc) {
        const uint32_t v_addr = smem_u32(sV + s * Cfg::kTileBytes);
#pragma unroll
        for (int kk = 0; kk < kKV / 16; ++kk) {
          // V is MN-major here: rows = keys (K), 128 B of head dim per row,
          // 16 keys per step = 2048 B, 64-dim regions are LBO apart.
          umma_bf16_ta(tmem + (t == 0 ? Cfg::kColO0 : Cfg::kColO1),
                       tmem + (t == 0 ? Cfg::kColS0 : Cfg::kColS1) + kk * 8,
                       sdesc_sw128(v_addr + kk * 2048, Cfg::kRegionBytes, 1024), idPV,
                       (acc || kk > 0) ? 1u : 0u);
        }
      };
      ok = mbar_wait(q_full, 0) && mbar_wait(&k_full[0], 0);
      if (ok) {
        tc_fence_after();
        for (int t = 0; t < ntile; ++t) {
          issue_s(t, 0);
          umma_commit(&s_full[t]);
        }
        umma_commit(&k_empty[0]);
      }
      for (int j = 0; j < nkv && ok; ++j) {
        const int s = j % kStages;
        const int s1 = (j + 1) % kStages;
        for (int t = 0; t < ntile && ok; ++t) {
          if (!mbar_wait(&p_full[t], j & 1)) {
            ok = false;
            break;
          }
          if (t == 0 && !mbar_wait(&v_full[s], (j / kStages) & 1)) {
            ok = false;
            break;
          }
          tc_fence_after();
          issue_pv(t, s, j > 0);
          if (t == ntile - 1) umma_commit(&v_empty[s]);
          if (j + 1 < nkv) {
            if (t == 0 && !mbar_wait(&k_full[s1], ((j + 1) / kStages) & 1)) {
              ok = false;
              break;
            }
            tc_fence_after();
            issue_s(t, s1);
            umma_commit(&s_full[t]);
            if (t == ntile - 1) umma_commit(&k_empty[s1]);
          } else {
            umma_commit(&o_done[t]);
          }
        }
      }
    }
  } else {
    // ------------------------------------------------------------ softmax warpgroups
    const int t = (warp - 2) >> 2;  // query tile of this warpgroup
    const int qd = warp & 3;        // TMEM lane quarter
    const int row = 32 * qd + lane;
    const uint32_t lane_base = static_cast<uint32_t>(32 * qd) << 16;
    const uint32_t tS = tmem + lane_base + (t == 0 ? Cfg::kColS0 : Cfg::kColS1);
    const uint32_t tO = tmem + lane_base + (t == 0 ? Cfg::kColO0 : Cfg::kColO1);
    const bool active = t < ntile;
    float m_run = -INFINITY, l_run = 0.f;
    for (int j = 0; j < nkv && active; ++j) {
      if (!__all_sync(0xffffffffu, mbar_wait(&s_full[t], j & 1))) {
        ok = false;
        break;
      }
      tc_fence_after();
      const int valid = p.N - (j0 + j) * kKV;  // keys past N are zero-filled: mask them
      // the whole S row of this tile in one TMEM load
      uint32_t sr[kKV];
      tmem_ld128(tS, sr);
      if (valid < kKV) {
#pragma unroll
        for (int e = 0; e < kKV; ++e)
          if (e >= valid) sr[e] = __float_as_uint(-INFINITY);
      }
      // After the first tile the exponentials are taken against the running
      // max as it stands, without a row-max pass first: any P below 2^64 is
      // safe (bf16 and the fp32 sums hold it), and the row sum tells whether a
      // value went past that.  Only then (rare) is S read again, its max taken,
      // O and l rescaled and P recomputed.  The first tile takes the max first.
      float m_use = m_run, alpha = 1.0f, rs;
      if (j == 0) m_use = row_max(sr) * p.scale_log2;
      uint32_t w[kKV / 2];
#pragma unroll 1
      for (int pass = 0;; ++pass) {
        rs = exp_row(sr, p.scale_log2, m_use, w);
        const bool over = !(rs <= kSumLimit);
        if (j == 0 || pass == 1 || !__any_sync(0xffffffffu, over)) break;
        // P is not stored yet, so S is still in TMEM: read it for its max,
        // rescale O, then read it again for P (few live registers at a time)
        tmem_ld128(tS, sr);
        if (valid < kKV) {
#pragma unroll
          for (int e = 0; e < kKV; ++e)
            if (e >= valid) sr[e] = __float_as_uint(-INFINITY);
        }
        const float tmax = row_max(sr) * p.scale_log2;
        if (over) {
          m_use = fmaxf(tmax, m_run);
          alpha = ex2_approx(m_run - m_use);
        }
        // O_t is stable here: the commit behind s_full covers P_t(j-1) V_{j-1}.
#pragma unroll 1
        for (int c = 0; c < HD / 32; ++c) {
          uint32_t r[32];
          tmem_ld32(tO + 32 * c, r);
#pragma unroll
          for (int e = 0; e < 32; ++e) r[e] = __float_as_uint(__uint_as_float(r[e]) * alpha);
          tmem_st32(tO + 32 * c, r);
        }
        tmem_ld128(tS, sr);
        if (valid < kKV) {
#pragma unroll
          for (int e = 0; e < kKV; ++e)
            if (e >= valid) sr[e] = __float_as_uint(-INFINITY);
        }
      }
      tmem_st64(tS, w);
      l_run = l_run * alpha + rs;
      m_run = m_use;
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&p_full[t]);
    }
    // epilogue: O / l -> bf16 rows of the compact output, or, for a key-range
    // part, the unnormalised O with its (m, l) for k_attn_combine
    if (active && ok) {
      if (__all_sync(0xffffffffu, mbar_wait(&o_done[t], 0))) {
        tc_fence_after();
        const float inv = 1.0f / l_run;
        const int qrow = q0 + t * kQ + row;
        __nv_bfloat16* orow = p.o + static_cast<size_t>(qrow) * p.ld + col0;
        const size_t prow = static_cast<size_t>(part) * (2 * kQ) + t * kQ + row;
        if (part >= 0) p.part_ml[prow] = make_float2(m_run, l_run);
#pragma unroll 1
        for (int c = 0; c < HD / 32; ++c) {
          uint32_t r[32];
          __syncwarp();
          tmem_ld32(tO + 32 * c, r);
          if (part >= 0) {
            float4* d4 = reinterpret_cast<float4*>(p.part_o + prow * HD + 32 * c);
#pragma unroll
            for (int v = 0; v < 8; ++v)
              d4[v] = make_float4(__uint_as_float(r[4 * v]), __uint_as_float(r[4 * v + 1]),
                                  __uint_as_float(r[4 * v + 2]), __uint_as_float(r[4 * v + 3]));
          } else if (qrow < p.n) {
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
  }
  if (!ok) atomicOr(p.flag, DEV_TIMEOUT);
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

// Merge the key-range parts of the split units: one warp per query row,
// O = sum_i O_i 2^(m_i - M) / sum_i l_i 2^(m_i - M) with M = max_i m_i.
template <int HD>
__global__ void __launch_bounds__(256) k_attn_combine(AttnParams p) {
  const int lane = threadIdx.x & 31;
  const int rr = blockIdx.x * 8 + (threadIdx.x >> 5);  // row over the split units
  const int u = blockIdx.y;                             // split unit 0..r-1
  if (rr >= 2 * kQ) return;
  const int unit = p.n_full + u;
  const int q0 = (unit % p.n_qpairs) * (2 * kQ);
  const int h = unit / p.n_qpairs;
  const int qrow = q0 + rr;
  if (qrow >= p.n) return;
  float M = -INFINITY;
  for (int i = 0; i < p.split; ++i) {
    const size_t prow = static_cast<size_t>(u * p.split + i) * (2 * kQ) + rr;
    M = fmaxf(M, p.part_ml[prow].x);
  }
  constexpr int kPer = HD / 32;  // columns per lane
  float acc[kPer];
#pragma unroll
  for (int c = 0; c < kPer; ++c) acc[c] = 0.f;
  float L = 0.f;
  for (int i = 0; i < p.split; ++i) {
    const size_t prow = static_cast<size_t>(u * p.split + i) * (2 * kQ) + rr;
    const float2 ml = p.part_ml[prow];
    const float wgt = ex2_approx(ml.x - M);
    L += ml.y * wgt;
    const float* po = p.part_o + prow * HD;
#pragma unroll
    for (int c = 0; c < kPer; ++c) acc[c] += po[lane + 32 * c] * wgt;
  }
  const float inv = 1.0f / L;
  __nv_bfloat16* orow = p.o + static_cast<size_t>(qrow) * p.ld + h * HD;
#pragma unroll
  for (int c = 0; c < kPer; ++c) orow[lane + 32 * c] = __float2bfloat16_rn(acc[c] * inv);
}

template <int HD>
cudaError_t launch_hd(const Ctx& c, const void* q, int n, const void* kc, const void* vc, int N,
                      void* o, std::string* why) {
  const int D = c.cfg.D;
  CUtensorMap tq, tk, tv;
  if (!make_tmap_bf16(&tq, q, n, D, D, kQ, why)) return cudaErrorInvalidValue;
  if (!make_tmap_bf16(&tk, kc, N, D, D, kKV, why)) return cudaErrorInvalidValue;
  if (!make_tmap_bf16(&tv, vc, N, D, D, kKV, why)) return cudaErrorInvalidValue;
  AttnParams p{};
  p.n = n;
  p.N = N;
  p.scale_log2 = static_cast<float>(1.4426950408889634 / sqrt(static_cast<double>(HD)));
  p.o = static_cast<__nv_bfloat16*>(o);
  p.ld = D;
  p.flag = c.flag;
  constexpr int smem = AttnCfg<HD>::kSmem;
  static std::atomic<uint64_t> smem_set{0};  // per device
  {
    const cudaError_t e = ensure_smem_limit(k_attn<HD>, smem, c.device, smem_set);
    if (e != cudaSuccess) return e;
  }
  // Work plan: whole units fill complete waves of the SMs; the units of the
  // last, partial wave are split along the keys so that wave is short too.
  p.n_qpairs = (n + 2 * kQ - 1) / (2 * kQ);
  const int units = p.n_qpairs * c.cfg.H;
  const int nkv_all = (N + kKV - 1) / kKV;
  const int rem = units % c.num_sms;
  // Split each remaining unit into s key ranges, choosing s to minimise the
  // tail's length in units of a whole wave, ceil(rem*s / SMs) / s, with a
  // 1% charge per extra part for its prologue, partial store and combine.
  int split = 1;
  if (rem > 0) {
    double best = 1.0;
    for (int sp = 2; sp <= nkv_all && sp <= kMaxSplitParts && rem * sp <= kMaxAttnParts; ++sp) {
      const double rounds = static_cast<double>((rem * sp + c.num_sms - 1) / c.num_sms) / sp;
      const double cost = rounds * (1.0 + 0.01 * sp);
      if (cost < best) best = cost, split = sp;
    }
  }
  p.n_full = split > 1 ? units - rem : units;
  p.split = split;
  p.part_o = c.attn_part_o;
  p.part_ml = reinterpret_cast<float2*>(c.attn_part_ml);
  const int n_parts = (units - p.n_full) * split;
  k_attn<HD><<<p.n_full + n_parts, kAttnThreads, smem, c.stream>>>(tq, tk, tv, p);
  c.launches += 1;
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess || n_parts == 0) return e;
  k_attn_combine<HD><<<dim3(2 * kQ / 8, units - p.n_full), 256, 0, c.stream>>>(p);
  c.launches += 1;
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_attention(const Ctx& c, const void* q, int n, const void* kc, const void* vc,
                             int n_kv, void* o, std::string* why) {
  if (n <= 0) return cudaSuccess;
  Timed timed(c, TC_ATTN, 4.0 * n * n_kv * c.cfg.D);
  const int d = c.cfg.D / c.cfg.H;
  if (d == 128) return launch_hd<128>(c, q, n, kc, vc, n_kv, o, why);
  if (d == 64) return launch_hd<64>(c, q, n, kc, vc, n_kv, o, why);
  if (why) *why = "attention supports head_dim 64 or 128";
  return cudaErrorInvalidValue;
}

}  // namespace hsa
