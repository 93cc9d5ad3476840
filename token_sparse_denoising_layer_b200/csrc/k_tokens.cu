// k_tokens.cu - per-token kernels of the HSA step: group schedule, L1
// relative-change score, exact radix selection of the groups, and the
// cached Euler update.
//
// Method: "Technical Summary: Heterogeneous Step Allocation (HSA) for
// Efficient Video Generation", section 2.1 (Token Partitioning and
// Scheduling, Dynamic Selection) and section 2.3 (Cached Euler Update).

#include <cuda_runtime.h>
#include <stdint.h>

#include "internal.h"
#include "ptx.cuh"

namespace hsa {

// ============================================================ schedule (2.1)
//
// Token n of group k is active at iteration i iff i mod (T/s_k) == 0; in the
// phase window (first/last m iterations, section 2.4) every token is active.
// Each CTA owns a 1024-token chunk (four tokens per thread, one 32-bit load
// of group ids and one 32-bit mask store), so N = 32760 spreads over 32 CTAs
// and N = 75600 over 74.  A CTA counts the active tokens of all earlier chunks
// itself (at most N bytes, read from L2 with 16-byte loads), so the
// compaction needs one launch and no inter-CTA waiting.  Output order is
// ascending.

constexpr int kSchedThreads = 256;
constexpr int kSchedChunk = kSchedThreads * 4;

struct SchedParams {
  int strides[kMaxGroups];
  int K, i, T, m, N;
};

__device__ __forceinline__ uint32_t active_group_bits(const SchedParams& p) {
  const bool window = p.m > 0 && (p.i < p.m || p.i >= p.T - p.m);
  uint32_t bits = 0;
  for (int k = 0; k < p.K; ++k)
    if (window || (p.i % p.strides[k]) == 0) bits |= 1u << k;
  return bits;
}

__device__ __forceinline__ int on_of(uint32_t gbyte, uint32_t bits) {
  return gbyte < 32u ? static_cast<int>((bits >> gbyte) & 1u) : 0;
}

__device__ __forceinline__ int count_on_word(uint32_t w, uint32_t bits) {
  return on_of(w & 0xFF, bits) + on_of((w >> 8) & 0xFF, bits) + on_of((w >> 16) & 0xFF, bits) +
         on_of(w >> 24, bits);
}

// Block-wide exclusive scan of one int per thread; returns the exclusive
// prefix and writes the block total to *total.
__device__ __forceinline__ int block_exclusive_scan(int v, int* warp_sums, int* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    int y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) warp_sums[warp] = x;
  __syncthreads();
  if (warp == 0) {
    const int nw = blockDim.x >> 5;
    int s = lane < nw ? warp_sums[lane] : 0;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      int y = __shfl_up_sync(0xffffffffu, s, o);
      if (lane >= o) s += y;
    }
    if (lane < nw) warp_sums[lane] = s;  // inclusive
  }
  __syncthreads();
  const int before = (warp > 0 ? warp_sums[warp - 1] : 0) + x - v;
  *total = warp_sums[(blockDim.x >> 5) - 1];
  __syncthreads();
  return before;
}

__device__ __forceinline__ int block_sum(int v, int* warp_sums) {
  int total;
  block_exclusive_scan(v, warp_sums, &total);
  return total;
}

__global__ void __launch_bounds__(kSchedThreads) k_schedule(const uint8_t* __restrict__ g,
                                                            uint8_t* __restrict__ mask,
                                                            int32_t* __restrict__ idx,
                                                            int32_t* __restrict__ n_dev,
                                                            SchedParams p, int* flag) {
  __shared__ int warp_sums[32];
  const uint32_t bits = active_group_bits(p);
  const int base = blockIdx.x * kSchedChunk;

  // 1. this thread's four tokens (g and mask are 16-byte aligned, base and n0
  //    are multiples of 4: a whole word is in bounds unless it holds the tail)
  const int n0 = base + 4 * threadIdx.x;
  uint32_t gw = 0xFFFFFFFFu;
  if (n0 + 4 <= p.N) {
    gw = __ldg(reinterpret_cast<const uint32_t*>(g + n0));
  } else {
    for (int j = 0; j < 4 && n0 + j < p.N; ++j)
      gw = (gw & ~(0xFFu << (8 * j))) | (static_cast<uint32_t>(g[n0 + j]) << (8 * j));
  }
  int on[4];
  int bad = 0;
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const uint32_t gb = (gw >> (8 * j)) & 0xFFu;
    const bool in = n0 + j < p.N;
    if (in && gb >= static_cast<uint32_t>(p.K)) bad = 1;
    on[j] = (in && gb < static_cast<uint32_t>(p.K)) ? on_of(gb, bits) : 0;
  }
  if (bad) atomicOr(flag, DEV_BAD_GROUP);

  // 2. active tokens before this chunk (base is a multiple of 16)
  int before = 0;
  const uint4* gv = reinterpret_cast<const uint4*>(g);
#pragma unroll 4
  for (int v = threadIdx.x; v < base / 16; v += blockDim.x) {
    const uint4 w = __ldg(gv + v);
    before += count_on_word(w.x, bits) + count_on_word(w.y, bits) + count_on_word(w.z, bits) +
              count_on_word(w.w, bits);
  }
  const int mine = on[0] + on[1] + on[2] + on[3];
  before = block_sum(before, warp_sums);
  int total;
  int pos = before + block_exclusive_scan(mine, warp_sums, &total);
  if (n0 + 4 <= p.N) {
    *reinterpret_cast<uint32_t*>(mask + n0) = static_cast<uint32_t>(on[0]) |
                                              (static_cast<uint32_t>(on[1]) << 8) |
                                              (static_cast<uint32_t>(on[2]) << 16) |
                                              (static_cast<uint32_t>(on[3]) << 24);
  } else {
    for (int j = 0; j < 4 && n0 + j < p.N; ++j) mask[n0 + j] = static_cast<uint8_t>(on[j]);
  }
#pragma unroll
  for (int j = 0; j < 4; ++j)
    if (on[j]) idx[pos++] = n0 + j;
  if (n_dev != nullptr && threadIdx.x == 0 && base + kSchedChunk >= p.N) *n_dev = before + total;
}

cudaError_t launch_schedule(const Ctx& c, int i, const uint8_t* g, uint8_t* mask, int32_t* idx,
                            int32_t* n_dev) {
  Timed timed(c, TC_TOKENS, 0.0);
  SchedParams p{};
  for (int k = 0; k < c.K; ++k) p.strides[k] = c.strides[k];
  p.K = c.K;
  p.i = i;
  p.T = c.T;
  p.m = c.m;
  p.N = c.cfg.N;
  const int blocks = (c.cfg.N + kSchedChunk - 1) / kSchedChunk;
  k_schedule<<<blocks, kSchedThreads, 0, c.stream>>>(g, mask, idx, n_dev, p, c.flag);
  c.launches += 1;
  return cudaGetLastError();
}

// ============================================================ selector (2.1)
//
// Score: r_n = sum_c |v_cur - v_prev| / (sum_c |v_prev| + 1e-6) in float32,
// channel order, explicit round-to-nearest operations (no contraction), so
// the value is reproducible bit for bit.

constexpr float kScoreEps = 1e-6f;

__global__ void __launch_bounds__(256) k_score(const float4* __restrict__ v_prev,
                                               const float4* __restrict__ v_cur,
                                               float* __restrict__ score, int N, int* flag) {
  const int n = blockIdx.x * blockDim.x + threadIdx.x;
  if (n >= N) return;
  float num = 0.f, den = 0.f;
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    const float4 a = __ldg(v_prev + 4 * n + q);
    const float4 b = __ldg(v_cur + 4 * n + q);
    num = __fadd_rn(num, fabsf(__fsub_rn(b.x, a.x)));
    den = __fadd_rn(den, fabsf(a.x));
    num = __fadd_rn(num, fabsf(__fsub_rn(b.y, a.y)));
    den = __fadd_rn(den, fabsf(a.y));
    num = __fadd_rn(num, fabsf(__fsub_rn(b.z, a.z)));
    den = __fadd_rn(den, fabsf(a.z));
    num = __fadd_rn(num, fabsf(__fsub_rn(b.w, a.w)));
    den = __fadd_rn(den, fabsf(a.w));
  }
  den = __fadd_rn(den, kScoreEps);
  const float r = __fadd_rn(__fdiv_rn(num, den), 0.0f);
  if (!(r >= 0.f) || isinf(r)) atomicOr(flag, DEV_BAD_SCORE);
  score[n] = r;
}

cudaError_t launch_score(const Ctx& c, const float* v_prev, const float* v_cur, float* score) {
  Timed timed(c, TC_TOKENS, 0.0);
  const int N = c.cfg.N;
  k_score<<<(N + 255) / 256, 256, 0, c.stream>>>(reinterpret_cast<const float4*>(v_prev),
                                                 reinterpret_cast<const float4*>(v_cur), score, N,
                                                 c.flag);
  c.launches += 1;
  return cudaGetLastError();
}

// Ranking key: tokens sorted by (score descending, index ascending) are the
// tokens sorted by the 64-bit key (~bits(score), n) ascending.  For finite
// non-negative floats the bit pattern is monotone in the value.
__device__ __forceinline__ uint32_t key_hi(float r) { return ~__float_as_uint(__fadd_rn(r, 0.0f)); }

// One CTA per cut j: find the key of rank R_j (0-based), where
// R_j = n_1 + ... + n_j.  Four 8-bit radix passes fix the high word exactly;
// the index tie-break is then the (R_j - count(hi < hv))-th token, in index
// order, among those whose high word equals hv.  Only integer shared-memory
// atomics are used, so the result is deterministic.
constexpr int kSelThreads = 1024;

struct CutParams {
  int rank[kMaxGroups];
};

__global__ void __launch_bounds__(kSelThreads) k_radix_cut(const float* __restrict__ score, int N,
                                                           CutParams cp, uint32_t* cuts,
                                                           int* flag) {
  __shared__ int hist[kRadixBins];
  __shared__ int warp_sums[32];
  __shared__ uint32_t s_sel[2];
  const int j = blockIdx.x;
  const int R = cp.rank[j];
  if (R >= N) {  // empty tail groups: a cut no key reaches
    if (threadIdx.x == 0) {
      cuts[2 * j] = 0xFFFFFFFFu;
      cuts[2 * j + 1] = 0xFFFFFFFFu;
    }
    return;
  }
  uint32_t prefix = 0, pmask = 0;
  int remaining = R;
  for (int pass = 0; pass < 4; ++pass) {
    const int shift = 24 - 8 * pass;
    for (int b = threadIdx.x; b < kRadixBins; b += blockDim.x) hist[b] = 0;
    __syncthreads();
    for (int n = threadIdx.x; n < N; n += blockDim.x) {
      const float r = __ldg(score + n);
      if (pass == 0 && !(r >= 0.f)) atomicOr(flag, DEV_BAD_SCORE);
      const uint32_t h = key_hi(r);
      if ((h & pmask) == prefix) atomicAdd(&hist[(h >> shift) & 0xFF], 1);
    }
    __syncthreads();
    if (threadIdx.x < 32) {
      // lane l owns bins 8l..8l+7
      const int lane = threadIdx.x;
      int loc[8];
      int s = 0;
#pragma unroll
      for (int t = 0; t < 8; ++t) {
        loc[t] = hist[8 * lane + t];
        s += loc[t];
      }
      int incl = s;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        int y = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += y;
      }
      int cum = incl - s;
#pragma unroll
      for (int t = 0; t < 8; ++t) {
        if (cum <= remaining && remaining < cum + loc[t]) {
          s_sel[0] = static_cast<uint32_t>(8 * lane + t);
          s_sel[1] = static_cast<uint32_t>(cum);
        }
        cum += loc[t];
      }
    }
    __syncthreads();
    const uint32_t bin = s_sel[0];
    remaining -= static_cast<int>(s_sel[1]);
    prefix |= bin << shift;
    pmask |= 0xFFu << shift;
    __syncthreads();
  }
  // tie-break by index: the remaining-th token (0-based) with key_hi == prefix
  int running = 0;
  for (int base = 0; base < N; base += blockDim.x) {
    const int n = base + threadIdx.x;
    const int eq = (n < N && key_hi(__ldg(score + n)) == prefix) ? 1 : 0;
    int total;
    const int pos = running + block_exclusive_scan(eq, warp_sums, &total);
    if (eq && pos == remaining) {
      cuts[2 * j] = prefix;
      cuts[2 * j + 1] = static_cast<uint32_t>(n);
    }
    running += total;
    if (running > remaining) break;  // uniform across the block
  }
}

// The same cut search with a cluster of kCutCluster CTAs per cut.  CTA c
// holds the high words of the contiguous index range [c span, (c+1) span) in
// shared memory; each radix pass sums the CTAs' 256-bin histograms through
// distributed shared memory, so every CTA takes the same bin (one cluster
// barrier per pass: the histograms alternate between two buffers); the index
// tie-break adds the CTAs' counts of keys equal to the final high word in
// rank order.  Every CTA runs the same cluster barriers, and a last one keeps
// each CTA's shared memory alive while the others read it.
constexpr int kCutCluster = 8;
constexpr int kCutThreads = 512;
constexpr int kCutSpanMax = 16384;  // keys per CTA: 64 KB of shared memory
constexpr int kCutClusterMaxN = kCutCluster * kCutSpanMax;

__device__ __forceinline__ uint32_t mapa_rank(uint32_t saddr, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(saddr), "r"(rank));
  return r;
}

__device__ __forceinline__ int ld_cluster_s32(uint32_t caddr) {
  int v;
  asm volatile("ld.shared::cluster.s32 %0, [%1];" : "=r"(v) : "r"(caddr) : "memory");
  return v;
}

__global__ void __cluster_dims__(kCutCluster, 1, 1) __launch_bounds__(kCutThreads)
    k_radix_cut_cluster(const float* __restrict__ score, int N, int span, CutParams cp,
                        uint32_t* cuts, int* flag) {
  extern __shared__ uint32_t skey[];  // [span]
  // this CTA's histogram, read by the cluster; two buffers, alternating by
  // pass, so a CTA may clear the next pass's buffer while others still read
  // this pass's (they have all passed the barrier behind the one it clears)
  __shared__ int hist2[2][kRadixBins];
  __shared__ int ghist[kRadixBins];   // the cluster's
  __shared__ int warp_sums[32];
  __shared__ uint32_t s_sel[2];
  __shared__ int s_cnt;  // keys of this CTA equal to the final high word, read by the cluster
  const int j = blockIdx.x / kCutCluster;
  const uint32_t crank = cluster_ctarank();
  const int R = cp.rank[j];
  if (R >= N) {  // empty tail groups (uniform over the cluster: no barrier is reached)
    if (crank == 0 && threadIdx.x == 0) {
      cuts[2 * j] = 0xFFFFFFFFu;
      cuts[2 * j + 1] = 0xFFFFFFFFu;
    }
    return;
  }
  const int lo = min(N, static_cast<int>(crank) * span);
  const int cnt = min(N, lo + span) - lo;
  for (int i = threadIdx.x; i < cnt; i += blockDim.x) {
    const float r = __ldg(score + lo + i);
    if (!(r >= 0.f)) atomicOr(flag, DEV_BAD_SCORE);
    skey[i] = key_hi(r);
  }
  uint32_t prefix = 0, pmask = 0;
  int remaining = R;
  for (int pass = 0; pass < 4; ++pass) {
    const int shift = 24 - 8 * pass;
    int* hist = hist2[pass & 1];
    for (int b = threadIdx.x; b < kRadixBins; b += blockDim.x) hist[b] = 0;
    __syncthreads();
    for (int i = threadIdx.x; i < cnt; i += blockDim.x) {
      const uint32_t h = skey[i];
      if ((h & pmask) == prefix) atomicAdd(&hist[(h >> shift) & 0xFF], 1);
    }
    cluster_sync();  // every CTA's histogram is complete and visible, and every
                     // CTA has finished reading the other buffer (two passes ago)
    for (int b = threadIdx.x; b < kRadixBins; b += blockDim.x) {
      const uint32_t a = smem_u32(&hist[b]);
      int sum = 0;
      for (int r = 0; r < kCutCluster; ++r) sum += ld_cluster_s32(mapa_rank(a, r));
      ghist[b] = sum;
    }
    __syncthreads();
    if (threadIdx.x < 32) {
      // lane l owns bins 8l..8l+7
      const int lane = threadIdx.x;
      int loc[8];
      int sl = 0;
#pragma unroll
      for (int t = 0; t < 8; ++t) {
        loc[t] = ghist[8 * lane + t];
        sl += loc[t];
      }
      int incl = sl;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        int y = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += y;
      }
      int cum = incl - sl;
#pragma unroll
      for (int t = 0; t < 8; ++t) {
        if (cum <= remaining && remaining < cum + loc[t]) {
          s_sel[0] = static_cast<uint32_t>(8 * lane + t);
          s_sel[1] = static_cast<uint32_t>(cum);
        }
        cum += loc[t];
      }
    }
    __syncthreads();
    const uint32_t bin = s_sel[0];
    remaining -= static_cast<int>(s_sel[1]);
    prefix |= bin << shift;
    pmask |= 0xFFu << shift;
  }
  // tie-break by index: the remaining-th key (0-based) whose high word is prefix
  int eq_local = 0;
  for (int i = threadIdx.x; i < cnt; i += blockDim.x) eq_local += (skey[i] == prefix) ? 1 : 0;
  const int eq_cta = block_sum(eq_local, warp_sums);
  if (threadIdx.x == 0) s_cnt = eq_cta;
  cluster_sync();
  int before = 0;
  {
    const uint32_t a = smem_u32(&s_cnt);
    for (uint32_t r = 0; r < crank; ++r) before += ld_cluster_s32(mapa_rank(a, r));
  }
  cluster_sync();  // all counts have been read: CTAs may now leave
  if (remaining >= before && remaining < before + eq_cta) {
    const int want = remaining - before;
    int running = 0;
    for (int base = 0; base < cnt; base += blockDim.x) {
      const int i = base + threadIdx.x;
      const int eq = (i < cnt && skey[i] == prefix) ? 1 : 0;
      int total;
      const int pos = running + block_exclusive_scan(eq, warp_sums, &total);
      if (eq && pos == want) {
        cuts[2 * j] = prefix;
        cuts[2 * j + 1] = static_cast<uint32_t>(lo + i);
      }
      running += total;
      if (running > want) break;  // uniform across the block
    }
  }
}

__global__ void __launch_bounds__(256) k_assign(const float* __restrict__ score,
                                                const uint32_t* __restrict__ cuts, int ncut,
                                                uint8_t* __restrict__ g, int N) {
  __shared__ uint32_t s_cut[2 * kMaxGroups];
  if (threadIdx.x < 2 * ncut) s_cut[threadIdx.x] = cuts[threadIdx.x];
  __syncthreads();
  const int n = blockIdx.x * blockDim.x + threadIdx.x;
  if (n >= N) return;
  const uint32_t h = key_hi(__ldg(score + n));
  uint32_t k = 0;
  for (int j = 0; j < ncut; ++j) {
    const uint32_t ch = s_cut[2 * j], ci = s_cut[2 * j + 1];
    k += (h > ch || (h == ch && static_cast<uint32_t>(n) >= ci)) ? 1u : 0u;
  }
  g[n] = static_cast<uint8_t>(k);
}

cudaError_t launch_select(const Ctx& c, const float* score, uint8_t* g) {
  Timed timed(c, TC_TOKENS, 0.0);
  const int N = c.cfg.N;
  const int ncut = c.K - 1;
  if (ncut == 0) {
    cudaError_t e = cudaMemsetAsync(g, 0, static_cast<size_t>(N), c.stream);
    return e;
  }
  CutParams cp{};
  int acc = 0;
  for (int j = 0; j < ncut; ++j) {
    acc += c.counts[j];
    cp.rank[j] = acc;
  }
  cudaError_t e;
  if (N <= kCutClusterMaxN) {
    static std::atomic<uint64_t> smem_set{0};  // per device
    e = ensure_smem_limit(k_radix_cut_cluster, kCutSpanMax * 4, c.device, smem_set);
    if (e != cudaSuccess) return e;
    const int span = (N + kCutCluster - 1) / kCutCluster;
    k_radix_cut_cluster<<<ncut * kCutCluster, kCutThreads, span * 4, c.stream>>>(
        score, N, span, cp, c.cuts, c.flag);
  } else {
    k_radix_cut<<<ncut, kSelThreads, 0, c.stream>>>(score, N, cp, c.cuts, c.flag);
  }
  c.launches += 2;  // with k_assign below
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  k_assign<<<(N + 255) / 256, 256, 0, c.stream>>>(score, c.cuts, ncut, g, N);
  return cudaGetLastError();
}

// Score, cut search and assignment on caller-given buffers: score [N], cuts
// [2 * (K - 1)] words, flag [1].  Used by the allocation-free entry point.
cudaError_t launch_select_groups_raw(cudaStream_t stream, const float* v_prev, const float* v_cur,
                                     int N, const int* counts, int K, float* score,
                                     uint32_t* cuts, uint8_t* g, int* flag) {
  k_score<<<(N + 255) / 256, 256, 0, stream>>>(reinterpret_cast<const float4*>(v_prev),
                                               reinterpret_cast<const float4*>(v_cur), score, N,
                                               flag);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess || K == 1) {
    if (e == cudaSuccess) e = cudaMemsetAsync(g, 0, static_cast<size_t>(N), stream);
    return e;
  }
  CutParams cp{};
  int acc = 0;
  for (int j = 0; j < K - 1; ++j) {
    acc += counts[j];
    cp.rank[j] = acc;
  }
  k_radix_cut<<<K - 1, kSelThreads, 0, stream>>>(score, N, cp, cuts, flag);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  k_assign<<<(N + 255) / 256, 256, 0, stream>>>(score, cuts, K - 1, g, N);
  return cudaGetLastError();
}

// ============================================================ failure-detection self-test
//
// One thread waits on an mbarrier that nothing ever arrives at, through the
// same bounded wait the pipelined kernels use.  The wait gives up after
// limit_ns, the kernel records DEV_TIMEOUT and returns: no trap, no hang.

__global__ void k_selftest_timeout(uint64_t limit_ns, int* flag) {
  __shared__ uint64_t bar;
  mbar_init(&bar, 1);
  fence_barrier_init();
  if (!mbar_wait(&bar, 0, limit_ns)) atomicOr(flag, DEV_TIMEOUT);
}

cudaError_t launch_selftest_timeout(const Ctx& c, uint64_t limit_ns) {
  k_selftest_timeout<<<1, 1, 0, c.stream>>>(limit_ns, c.flag);
  c.launches += 1;
  return cudaGetLastError();
}

// ============================================================ cached Euler (2.3)
//
// One pass over all N tokens, four channels per thread (128-bit accesses):
// active tokens rotate their velocity cache (v_hat_prev <- v_hat <- v_fresh),
// then every token advances by (sigma_next - sigma_i) * v_hat.  Inactive
// tokens read neither v_fresh nor write the caches (predicated, not branched
// per warp).  Float32 with one rounding per operation.
//
// With kScore the same pass also writes the re-grouping score of every token
// from the two caches as they leave it (section 2.1, Dynamic Selection), so a
// re-grouping step reads the velocities once: the four threads of a token
// hold channels 0-3, 4-7, 8-11, 12-15, and the two sums run through them in
// channel order (each thread continues its left neighbour's partial sums), in
// the same order and rounding as k_score.

template <bool kScore>
__global__ void __launch_bounds__(256) k_euler(float4* __restrict__ x, float4* __restrict__ v_hat,
                                               float4* __restrict__ v_hat_prev,
                                               const float4* __restrict__ v_fresh,
                                               const uint8_t* __restrict__ mask, float s0,
                                               float s1, int n4, float* __restrict__ score,
                                               int* flag) {
  const int t = blockIdx.x * blockDim.x + threadIdx.x;
  if (!kScore && t >= n4) return;
  const bool live = t < n4;  // n4 = 4N: a token's four threads are all live or all not
  const float d = __fsub_rn(s1, s0);
  const bool on = live && __ldg(mask + (t >> 2)) != 0;
  float4 h = make_float4(0.f, 0.f, 0.f, 0.f), xx = h, prev = h;
  if (live) {
    h = kScore ? v_hat[t] : __ldcs(v_hat + t);
    xx = __ldcs(x + t);
  }
  if (on) {
    const float4 f = __ldcs(v_fresh + t);
    if (kScore) {
      v_hat_prev[t] = h;
      v_hat[t] = f;
    } else {
      __stcs(v_hat_prev + t, h);
      __stcs(v_hat + t, f);
    }
    prev = h;
    h = f;
  } else if (kScore && live) {
    prev = v_hat_prev[t];
  }
  if (live) {
    xx.x = __fadd_rn(xx.x, __fmul_rn(d, h.x));
    xx.y = __fadd_rn(xx.y, __fmul_rn(d, h.y));
    xx.z = __fadd_rn(xx.z, __fmul_rn(d, h.z));
    xx.w = __fadd_rn(xx.w, __fmul_rn(d, h.w));
    __stcs(x + t, xx);
  }
  if (kScore) {
    const int q = threadIdx.x & 3;  // blockDim is a multiple of 4: quads stay in one warp
    float num = 0.f, den = 0.f;
#pragma unroll
    for (int r = 0; r < 4; ++r) {
      const float pn = __shfl_up_sync(0xffffffffu, num, 1);
      const float pd = __shfl_up_sync(0xffffffffu, den, 1);
      if (q == r) {
        float a = r == 0 ? 0.f : pn, b = r == 0 ? 0.f : pd;
        a = __fadd_rn(a, fabsf(__fsub_rn(h.x, prev.x)));
        b = __fadd_rn(b, fabsf(prev.x));
        a = __fadd_rn(a, fabsf(__fsub_rn(h.y, prev.y)));
        b = __fadd_rn(b, fabsf(prev.y));
        a = __fadd_rn(a, fabsf(__fsub_rn(h.z, prev.z)));
        b = __fadd_rn(b, fabsf(prev.z));
        a = __fadd_rn(a, fabsf(__fsub_rn(h.w, prev.w)));
        b = __fadd_rn(b, fabsf(prev.w));
        num = a;
        den = b;
      }
    }
    if (q == 3 && live) {
      den = __fadd_rn(den, kScoreEps);
      const float r = __fadd_rn(__fdiv_rn(num, den), 0.0f);
      if (!(r >= 0.f) || isinf(r)) atomicOr(flag, DEV_BAD_SCORE);
      score[t >> 2] = r;
    }
  }
}

cudaError_t launch_euler(const Ctx& c, float* x, float* v_hat, float* v_hat_prev,
                         const float* v_fresh, const uint8_t* mask, float s0, float s1,
                         float* score) {
  Timed timed(c, TC_TOKENS, 0.0);
  const int n4 = c.cfg.N * (c.cfg.C / 4);
  const dim3 grid((n4 + 255) / 256);
  if (score != nullptr)
    k_euler<true><<<grid, 256, 0, c.stream>>>(
        reinterpret_cast<float4*>(x), reinterpret_cast<float4*>(v_hat),
        reinterpret_cast<float4*>(v_hat_prev), reinterpret_cast<const float4*>(v_fresh), mask,
        s0, s1, n4, score, c.flag);
  else
    k_euler<false><<<grid, 256, 0, c.stream>>>(
        reinterpret_cast<float4*>(x), reinterpret_cast<float4*>(v_hat),
        reinterpret_cast<float4*>(v_hat_prev), reinterpret_cast<const float4*>(v_fresh), mask,
        s0, s1, n4, nullptr, c.flag);
  c.launches += 1;
  return cudaGetLastError();
}

}  // namespace hsa
