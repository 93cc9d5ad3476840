// k_gemm.cu - active-row GEMMs of the HSA layer on the 5th-generation tensor
// cores (tcgen05.mma, fp32 accumulators in TMEM, operands staged by TMA).
//
// C[m, j] = sum_k A[m, k] * B[j, k], A = compact bf16 activations of the
// active rows [M = |A_i|, K], B = a Linear weight [Ncols, K].  The epilogue
// is where the sparse structure of the method lives ("Technical Summary:
// Heterogeneous Step Allocation (HSA) for Efficient Video Generation",
// section 2.2): fresh K/V rows are scattered into the KV cache rows idx[m],
// and out-projection / MLP results are added into residual rows idx[m].
//
// Persistent: one CTA per SM walks its share of the 128 x BN output tiles
// (BN = 256, 192 or 128), K-block 64, through a multi-stage TMA ring that runs
// on across tiles.  Warp 0 issues TMA, warp 1 owns TMEM and issues the MMAs
// (one thread) into one of two TMEM accumulators, and eight epilogue warps
// drain the other accumulator (two per TMEM lane quarter, one per column
// half), so a tile's epilogue overlaps the next tile's main loop.

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <string>

#include "internal.h"
#include "ptx.cuh"

namespace hsa {

namespace {

constexpr int kBM = 128;
constexpr int kBK = 64;
constexpr int kGemmThreads = 320;  // TMA warp, MMA warp, 8 epilogue warps
constexpr int kEpiWarps = 8;
// relative cost per output element of a CTA-pair tile vs a 1-CTA 256-wide tile
constexpr double kPairCost = 0.8;

// Shared-memory staging for the residual epilogue: one 32 x 32 fp32 chunk
// per epilogue warp.  The 16-byte group g of row r is stored at group
// g ^ (r & 7), which keeps both the row-wise writes and the column-wise reads
// below free of bank conflicts without padding.
constexpr int kStageWarpFloats = 32 * 32;
constexpr int kEpiStageBytes = kEpiWarps * kStageWarpFloats * 4;

template <int BN>
struct GemmCfg {
  static constexpr int kStages = BN == 128 ? 6 : 4;
  // two accumulators of BN fp32 columns, allocated as a power of two
  static constexpr uint32_t kTmemCols = 2 * BN <= 256 ? 256 : 512;
  static constexpr int kABytes = kBM * kBK * 2;
  static constexpr int kBBytes = BN * kBK * 2;
  static constexpr int kStageBytes = kABytes + kBBytes;
  static constexpr int kBarBytes = 256;
  static constexpr int kSmem = kStages * kStageBytes + kBarBytes + kEpiStageBytes + 1024;
};

struct EpiParams {
  int M, Ncols, Kd, epi;
  __nv_bfloat16* out;
  int ld_out;
  __nv_bfloat16* kc[kMaxCaches];  // EPI_QKV: n_caches copies of the K and V caches
  __nv_bfloat16* vc[kMaxCaches];
  int n_caches;
  float* x;
  int ld_x;
  const float* gate;
  const int32_t* idx;
  int N;
  int* flag;
};

struct F2 {
  float x, y;
};

// d = a * b + c, two lanes per instruction (packed f32x2).
__device__ __forceinline__ F2 fma_x2(F2 a, F2 b, F2 c) {
  F2 d;
  asm("{\n\t.reg .b64 ra, rb, rc, rd;\n\t"
      "mov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\tmov.b64 rc, {%6, %7};\n\t"
      "fma.rn.f32x2 rd, ra, rb, rc;\n\tmov.b64 {%0, %1}, rd;\n\t}"
      : "=f"(d.x), "=f"(d.y)
      : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y), "f"(c.x), "f"(c.y));
  return d;
}

__device__ __forceinline__ F2 mul_x2(F2 a, F2 b) {
  F2 d;
  asm("{\n\t.reg .b64 ra, rb, rd;\n\t"
      "mov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\t"
      "mul.rn.f32x2 rd, ra, rb;\n\tmov.b64 {%0, %1}, rd;\n\t}"
      : "=f"(d.x), "=f"(d.y)
      : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
  return d;
}

__device__ __forceinline__ F2 splat(float v) { return F2{v, v}; }

__device__ __forceinline__ float rcp_approx(float x) {
  float y;
  asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// GELU, erf form, of two values: v Phi(v), with Phi(v) = 1 - erfc(v / sqrt 2) / 2
// for v >= 0 and erfc(|v| / sqrt 2) / 2 for v < 0.  erfc(z), z >= 0, is the
// Chebyshev fit of Press, Teukolsky, Vetterling & Flannery, Numerical Recipes,
// section 6.2: t = 1 / (1 + z/2), erfc(z) = t exp(-z^2 + P(t)) with a degree-9
// P, a fractional error below 1.2e-7 for every z.  A relative bound matters
// here: for v < 0 the result is a small tail value that is then rounded to
// bf16.  Evaluated on packed f32x2 lanes with P's coefficients negated (Horner
// commutes with negation), and the 1/2 folded into the exponent; two MUFU
// operations per value, no branches.
__device__ __forceinline__ F2 gelu_x2(F2 v) {
  const F2 zn = F2{fabsf(v.x) * -0.70710678118654752440f, fabsf(v.y) * -0.70710678118654752440f};
  const F2 d = fma_x2(zn, splat(-0.5f), splat(1.0f));  // 1 + z/2
  const F2 t = F2{rcp_approx(d.x), rcp_approx(d.y)};
  F2 q = fma_x2(splat(-0.17087277f), t, splat(0.82215223f));  // -P(t) by Horner
  q = fma_x2(q, t, splat(-1.48851587f));
  q = fma_x2(q, t, splat(1.13520398f));
  q = fma_x2(q, t, splat(-0.27886807f));
  q = fma_x2(q, t, splat(0.18628806f));
  q = fma_x2(q, t, splat(-0.09678418f));
  q = fma_x2(q, t, splat(-0.37409196f));
  q = fma_x2(q, t, splat(-1.00002368f));
  q = fma_x2(q, t, splat(1.26551223f));
  q = fma_x2(zn, zn, q);  // z^2 - P(t)
  // log2 of erfc(z) / 2 / t: (P(t) - z^2) log2(e) - 1
  const F2 s = fma_x2(q, splat(-1.4426950408889634f), splat(-1.0f));
  const F2 he = mul_x2(t, F2{ex2_approx(s.x), ex2_approx(s.y)});  // erfc(z) / 2
  const F2 phi = F2{v.x >= 0.f ? 1.0f - he.x : he.x, v.y >= 0.f ? 1.0f - he.y : he.y};
  return mul_x2(v, phi);
}

// 32 fp32 accumulators -> 32 bf16 (rounded to nearest even) in four 16-byte words.
__device__ __forceinline__ void pack_bf16x32(const uint32_t (&r)[32], uint4 (&w)[4]) {
#pragma unroll
  for (int v = 0; v < 4; ++v)
    w[v] = make_uint4(pack_bf16(__uint_as_float(r[8 * v]), __uint_as_float(r[8 * v + 1])),
                      pack_bf16(__uint_as_float(r[8 * v + 2]), __uint_as_float(r[8 * v + 3])),
                      pack_bf16(__uint_as_float(r[8 * v + 4]), __uint_as_float(r[8 * v + 5])),
                      pack_bf16(__uint_as_float(r[8 * v + 6]), __uint_as_float(r[8 * v + 7])));
}

// 32 fp32 accumulators -> 32 bf16 at dst (64 contiguous bytes, 16-byte aligned).
template <bool kGelu>
__device__ __forceinline__ void store_bf16x32(__nv_bfloat16* dst, const uint32_t (&r)[32]) {
  uint4* d4 = reinterpret_cast<uint4*>(dst);
#pragma unroll
  for (int v = 0; v < 4; ++v) {
    uint32_t w[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      float a = __uint_as_float(r[8 * v + 2 * e]);
      float b = __uint_as_float(r[8 * v + 2 * e + 1]);
      if (kGelu) {
        const F2 g = gelu_x2(F2{a, b});
        a = g.x;
        b = g.y;
      }
      w[e] = pack_bf16(a, b);
    }
    d4[v] = make_uint4(w[0], w[1], w[2], w[3]);
  }
}


// x[dst_row(r), col .. col+31] += chunk row r for the warp's 32 rows, as
// vector reductions that L2 performs, so the epilogue never waits for the
// residual rows it updates.  The chunk (row r in lane r's registers) goes
// through shared memory so that one reduction instruction covers four rows
// and 128 contiguous bytes of each: lanes 8k'..8k'+7 own row 4k + k'.  Each
// element gets exactly one addition per launch: x + v rounded once (with a
// gate, gate * v is rounded first).
__device__ __forceinline__ void resid_chunk(const EpiParams& p, const uint32_t (&r)[32],
                                            int32_t dst_row, int col, float* stage) {
  const int lane = threadIdx.x & 31;
  float* srow = stage + lane * 32;
#pragma unroll
  for (int v = 0; v < 8; ++v)
    *reinterpret_cast<float4*>(srow + 4 * (v ^ (lane & 7))) =
        make_float4(__uint_as_float(r[4 * v]), __uint_as_float(r[4 * v + 1]),
                    __uint_as_float(r[4 * v + 2]), __uint_as_float(r[4 * v + 3]));
  __syncwarp();
  const int g4 = lane & 7;  // this lane's 16-byte group of the row
  float4 g = make_float4(1.f, 1.f, 1.f, 1.f);
  if (p.gate != nullptr) g = __ldg(reinterpret_cast<const float4*>(p.gate + col + 4 * g4));
#pragma unroll
  for (int k = 0; k < 8; ++k) {
    const int rr = 4 * k + (lane >> 3);
    const int32_t d = __shfl_sync(0xffffffffu, dst_row, rr);
    float4 v = *reinterpret_cast<const float4*>(stage + rr * 32 + 4 * (g4 ^ (rr & 7)));
    if (d >= 0) {
      if (p.gate != nullptr) {
        v.x *= g.x;
        v.y *= g.y;
        v.z *= g.z;
        v.w *= g.w;
      }
      float* dst = p.x + static_cast<size_t>(d) * p.ld_x + col + 4 * g4;
      asm volatile("red.global.add.v4.f32 [%0], {%1, %2, %3, %4};" ::"l"(dst), "f"(v.x),
                   "f"(v.y), "f"(v.z), "f"(v.w)
                   : "memory");
    }
  }
  __syncwarp();  // the stage is reused by the next chunk
}

// Drain one accumulator tile: this warp's 32 rows (TMEM lanes at tbase),
// output row m (this lane's), columns n0 .. n0 + kCols - 1.  TMEM loads run
// one 32-column chunk ahead of the chunk being stored.
template <int kCols, int kEpi>
__device__ __forceinline__ void drain_tile(const EpiParams& p, uint32_t tbase, int m, int n0,
                                           float* stage) {
  constexpr int NC = kCols / 32;
  const bool mrow = m < p.M;
  int32_t dst_row = -1;
  if ((kEpi == EPI_QKV || kEpi == EPI_RESID) && mrow) {
    dst_row = __ldg(p.idx + m);
    if (!row_ok(dst_row, p.N, p.flag)) dst_row = -1;
  }
  uint32_t ra[32], rb[32];
  __syncwarp();
  tmem_ld32_nowait(tbase, ra);
#pragma unroll
  for (int c = 0; c < NC; ++c) {
    uint32_t(&cur)[32] = (c & 1) ? rb : ra;
    uint32_t(&nxt)[32] = (c & 1) ? ra : rb;
    tmem_wait_ld();
    if (c + 1 < NC) {
      __syncwarp();
      tmem_ld32_nowait(tbase + 32 * (c + 1), nxt);
    }
    const int col = n0 + 32 * c;
    if (col >= p.Ncols) continue;  // uniform over the warp
    if (kEpi == EPI_RESID) {
      resid_chunk(p, cur, dst_row, col, stage);
    } else if (mrow) {
      if (kEpi == EPI_STORE || kEpi == EPI_GELU) {
        store_bf16x32<kEpi == EPI_GELU>(p.out + static_cast<size_t>(m) * p.ld_out + col, cur);
      } else {  // EPI_QKV
        const int D = p.ld_out;
        const int which = col / D;
        const int cc = col - which * D;
        if (which == 0) {
          store_bf16x32<false>(p.out + static_cast<size_t>(m) * D + cc, cur);
        } else if (dst_row >= 0 && p.n_caches == 1) {
          __nv_bfloat16* cache = which == 1 ? p.kc[0] : p.vc[0];
          store_bf16x32<false>(cache + static_cast<size_t>(dst_row) * D + cc, cur);
        } else if (dst_row >= 0) {
          // the fresh row into every copy of this layer's cache (this GPU's,
          // and peers' when a sharded step writes them directly)
          uint4 w4[4];
          pack_bf16x32(cur, w4);
#pragma unroll
          for (int g = 0; g < kMaxCaches; ++g) {
            if (g >= p.n_caches) break;
            __nv_bfloat16* cache = which == 1 ? p.kc[g] : p.vc[g];
            uint4* d4 = reinterpret_cast<uint4*>(cache + static_cast<size_t>(dst_row) * D + cc);
            d4[0] = w4[0];
            d4[1] = w4[1];
            d4[2] = w4[2];
            d4[3] = w4[3];
          }
        }
      }
    }
  }
}

template <int kCols>
__device__ __forceinline__ void drain(const EpiParams& p, uint32_t tbase, int m, int n0,
                                      float* stage) {
  switch (p.epi) {
    case EPI_STORE: drain_tile<kCols, EPI_STORE>(p, tbase, m, n0, stage); break;
    case EPI_GELU: drain_tile<kCols, EPI_GELU>(p, tbase, m, n0, stage); break;
    case EPI_QKV: drain_tile<kCols, EPI_QKV>(p, tbase, m, n0, stage); break;
    case EPI_RESID: drain_tile<kCols, EPI_RESID>(p, tbase, m, n0, stage); break;
    default: break;
  }
}

template <int BN>
__global__ void __launch_bounds__(kGemmThreads, 1)
    k_gemm(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
           EpiParams p, int n_tiles, int total_tiles) {
  using Cfg = GemmCfg<BN>;
  constexpr int S = Cfg::kStages;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint8_t* sA = smem;
  uint8_t* sB = smem + S * Cfg::kABytes;
  uint64_t* full = reinterpret_cast<uint64_t*>(sB + S * Cfg::kBBytes);
  uint64_t* empty = full + S;
  uint64_t* acc_full = empty + S;     // [2] accumulator buffer ready for the epilogue
  uint64_t* acc_empty = acc_full + 2; // [2] accumulator buffer drained
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(acc_empty + 2);
  float* stage = reinterpret_cast<float*>(reinterpret_cast<uint8_t*>(full) + Cfg::kBarBytes);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nk = p.Kd / kBK;

  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&acc_full[b], 1);
      mbar_init(&acc_empty[b], kEpiWarps);  // one arrival per epilogue warp
    }
    fence_barrier_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmB);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, Cfg::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  bool ok = true;

  // Tiles are visited t = blockIdx.x, +gridDim.x, ...; tile t covers rows
  // (t / n_tiles) * 128 and columns (t % n_tiles) * BN, so tiles running at the
  // same time share A row blocks and sweep the (L2-resident) weight.
  if (warp == 0) {
    if (lane == 0) {
      int it = 0;
      for (int t = blockIdx.x; t < total_tiles && ok; t += gridDim.x) {
        const int m0 = (t / n_tiles) * kBM, n0 = (t % n_tiles) * BN;
        for (int kb = 0; kb < nk; ++kb, ++it) {
          const int s = it % S;
          if (!mbar_wait(&empty[s], ((it / S) & 1) ^ 1)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&full[s], Cfg::kStageBytes);
          tma_load_2d(sA + s * Cfg::kABytes, &tmA, &full[s], kb * kBK, m0);
          tma_load_2d(sB + s * Cfg::kBBytes, &tmB, &full[s], kb * kBK, n0);
        }
      }
      if (!ok) {  // let copies already in flight land before the CTA exits
        for (int k = it > S ? it - S : 0; k < it; ++k) (void)mbar_wait(&full[k % S], (k / S) & 1);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_bf16(kBM, BN, false, false);
      int it = 0, lt = 0;
      for (int t = blockIdx.x; t < total_tiles && ok; t += gridDim.x, ++lt) {
        const int b = lt & 1;
        if (!mbar_wait(&acc_empty[b], ((lt >> 1) & 1) ^ 1)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t acc = tmem + b * BN;
        for (int kb = 0; kb < nk; ++kb, ++it) {
          const int s = it % S;
          if (!mbar_wait(&full[s], (it / S) & 1)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a0 = smem_u32(sA + s * Cfg::kABytes);
          const uint32_t b0 = smem_u32(sB + s * Cfg::kBBytes);
#pragma unroll
          for (int kk = 0; kk < kBK / 16; ++kk) {
            const uint64_t ad = sdesc_sw128(a0 + kk * 32, 16, 1024);
            const uint64_t bd = sdesc_sw128(b0 + kk * 32, 16, 1024);
            umma_bf16(acc, ad, bd, idesc, (kb > 0 || kk > 0) ? 1u : 0u);
          }
          umma_commit(&empty[s]);
        }
        umma_commit(&acc_full[b]);
      }
    }
  } else {
    // epilogue: warp w reads TMEM lanes [32*(w%4), +32) = tile rows, and
    // column half (w - 2) / 4 of the tile
    const int q = warp & 3;
    const int half = (warp - 2) >> 2;
    const int row = 32 * q + lane;
    int lt = 0;
    for (int t = blockIdx.x; t < total_tiles; t += gridDim.x, ++lt) {
      const int b = lt & 1;
      if (!__all_sync(0xffffffffu, mbar_wait(&acc_full[b], (lt >> 1) & 1))) {
        ok = false;
        break;
      }
      tc_fence_after();
      const int m = (t / n_tiles) * kBM + row, n0 = (t % n_tiles) * BN + half * (BN / 2);
      const uint32_t tbase =
          tmem + b * BN + half * (BN / 2) + (static_cast<uint32_t>(32 * q) << 16);
      drain<BN / 2>(p, tbase, m, n0, stage + (warp - 2) * kStageWarpFloats);
      // the buffer may be refilled once every lane's TMEM reads are done
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&acc_empty[b]);
    }
  }
  if (!ok) atomicOr(p.flag, DEV_TIMEOUT);
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, Cfg::kTmemCols);
  }
}

// ------------------------------------------------------------ CTA-pair GEMM
// 256 x 256 output tiles computed by a cluster of two CTAs with one
// tcgen05.mma.cta_group::2 per K-step: each CTA stages its own 128 rows of A
// and one 128-row half of B, so a CTA moves half the B bytes of a 1-CTA
// 128 x 256 tile through shared memory for the same MMA work.  Rank 0 issues
// the MMAs; both CTAs load, and both run the epilogue on the 128 rows of the
// accumulator held in their own TMEM.

constexpr int kPairStages = 6;
constexpr int kPairABytes = 128 * kBK * 2;
constexpr int kPairBBytes = 128 * kBK * 2;
constexpr int kPairStageBytes = kPairABytes + kPairBBytes;
constexpr int kPairSmem = kPairStages * kPairStageBytes + 256 + kEpiStageBytes + 1024;

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kGemmThreads, 1)
    k_gemm_pair(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                EpiParams p, int n_tiles, int total_tiles) {
  constexpr int S = kPairStages;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint8_t* sA = smem;
  uint8_t* sB = smem + S * kPairABytes;
  uint64_t* full = reinterpret_cast<uint64_t*>(sB + S * kPairBBytes);  // used in rank 0
  uint64_t* empty = full + S;
  uint64_t* acc_full = empty + S;      // [2]
  uint64_t* acc_empty = acc_full + 2;  // [2], used in rank 0
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(acc_empty + 2);
  float* stage = reinterpret_cast<float*>(reinterpret_cast<uint8_t*>(full) + 256);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const int pair = blockIdx.x >> 1, npairs = gridDim.x >> 1;
  const int nk = p.Kd / kBK;

  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&acc_full[b], 1);
      mbar_init(&acc_empty[b], 2 * kEpiWarps);  // every epilogue warp of both CTAs
    }
    fence_barrier_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmB);
  }
  if (warp == 1) {
    tmem_alloc_pair(tmem_slot, 512);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  cluster_sync();  // both CTAs' barriers initialised and TMEM allocated
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  bool ok = true;

  if (warp == 0) {
    if (lane == 0) {
      int it = 0;
      for (int t = pair; t < total_tiles && ok; t += npairs) {
        const int m0 = (t / n_tiles) * 256 + rank * 128, n0 = (t % n_tiles) * 256 + rank * 128;
        for (int kb = 0; kb < nk; ++kb, ++it) {
          const int s = it % S;
          if (!mbar_wait(&empty[s], ((it / S) & 1) ^ 1)) {
            ok = false;
            break;
          }
          if (rank == 0) mbar_arrive_expect_tx(&full[s], 2 * kPairStageBytes);
          const uint32_t lead = to_leader(smem_u32(&full[s]));
          tma_load_2d_pair(sA + s * kPairABytes, &tmA, lead, kb * kBK, m0);
          tma_load_2d_pair(sB + s * kPairBBytes, &tmB, lead, kb * kBK, n0);
        }
      }
    }
  } else if (warp == 1) {
    if (lane == 0 && rank == 0) {
      constexpr uint32_t idesc = idesc_bf16(256, 256, false, false);
      int it = 0, lt = 0;
      for (int t = pair; t < total_tiles && ok; t += npairs, ++lt) {
        const int b = lt & 1;
        if (!mbar_wait(&acc_empty[b], ((lt >> 1) & 1) ^ 1)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t acc = tmem + b * 256;
        for (int kb = 0; kb < nk; ++kb, ++it) {
          const int s = it % S;
          if (!mbar_wait(&full[s], (it / S) & 1)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a0 = smem_u32(sA + s * kPairABytes);
          const uint32_t b0 = smem_u32(sB + s * kPairBBytes);
#pragma unroll
          for (int kk = 0; kk < kBK / 16; ++kk)
            umma_bf16_pair(acc, sdesc_sw128(a0 + kk * 32, 16, 1024),
                           sdesc_sw128(b0 + kk * 32, 16, 1024), idesc, (kb > 0 || kk > 0) ? 1u : 0u);
          umma_commit_pair(&empty[s], 0x3);
        }
        umma_commit_pair(&acc_full[b], 0x3);
      }
    }
  } else {
    const int q = warp & 3;
    const int half = (warp - 2) >> 2;  // column half of the tile
    const int row = 32 * q + lane;
    const uint32_t lead_empty0 = to_leader(smem_u32(&acc_empty[0]));
    const uint32_t lead_empty1 = to_leader(smem_u32(&acc_empty[1]));
    int lt = 0;
    for (int t = pair; t < total_tiles; t += npairs, ++lt) {
      const int b = lt & 1;
      if (!__all_sync(0xffffffffu, mbar_wait(&acc_full[b], (lt >> 1) & 1))) {
        ok = false;
        break;
      }
      tc_fence_after();
      const int m = (t / n_tiles) * 256 + rank * 128 + row, n0 = (t % n_tiles) * 256 + half * 128;
      const uint32_t tbase = tmem + b * 256 + half * 128 + (static_cast<uint32_t>(32 * q) << 16);
      drain<128>(p, tbase, m, n0, stage + (warp - 2) * kStageWarpFloats);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(b == 0 ? lead_empty0 : lead_empty1);
    }
  }
  if (!ok) atomicOr(p.flag, DEV_TIMEOUT);
  tc_fence_before();
  cluster_sync();  // no CTA leaves while its peer may still signal its barriers
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tmem, 512);
  }
}

// The caches an EPI_QKV launch writes: the list when one is given, else the pair.
void set_caches(EpiParams& p, const GemmArgs& a) {
  if (a.n_caches > 0) {
    p.n_caches = a.n_caches;
    for (int g = 0; g < a.n_caches; ++g) {
      p.kc[g] = static_cast<__nv_bfloat16*>(a.k_caches[g]);
      p.vc[g] = static_cast<__nv_bfloat16*>(a.v_caches[g]);
    }
  } else {
    p.n_caches = 1;
    p.kc[0] = static_cast<__nv_bfloat16*>(a.k_cache);
    p.vc[0] = static_cast<__nv_bfloat16*>(a.v_cache);
  }
}

static_assert(kPairSmem <= 227 * 1024, "CTA-pair GEMM exceeds the shared memory of a CTA");
static_assert(GemmCfg<256>::kSmem <= 227 * 1024 && GemmCfg<192>::kSmem <= 227 * 1024 &&
                  GemmCfg<128>::kSmem <= 227 * 1024,
              "GEMM tile exceeds the shared memory of a CTA");

cudaError_t launch_pair(const Ctx& c, const GemmArgs& a, std::string* why) {
  CUtensorMap ta, tb;
  if (!make_tmap_bf16(&ta, a.A, a.M, a.Kd, a.Kd, 128, why)) return cudaErrorInvalidValue;
  if (!make_tmap_bf16(&tb, a.B, a.Ncols, a.Kd, a.Kd, 128, why)) return cudaErrorInvalidValue;
  EpiParams p{};
  p.M = a.M;
  p.Ncols = a.Ncols;
  p.Kd = a.Kd;
  p.epi = a.epi;
  p.out = static_cast<__nv_bfloat16*>(a.out);
  p.ld_out = a.ld_out;
  set_caches(p, a);
  p.x = a.x;
  p.ld_x = a.ld_x;
  p.gate = a.gate;
  p.idx = a.idx;
  p.N = a.N;
  p.flag = c.flag;
  static std::atomic<uint64_t> smem_set{0};  // per device
  {
    const cudaError_t e = ensure_smem_limit(k_gemm_pair, kPairSmem, c.device, smem_set);
    if (e != cudaSuccess) return e;
  }
  const int n_tiles = (a.Ncols + 255) / 256;
  const int total = n_tiles * ((a.M + 255) / 256);
  const int pairs = total < c.num_sms / 2 ? total : c.num_sms / 2;
  k_gemm_pair<<<2 * pairs, kGemmThreads, kPairSmem, c.stream>>>(ta, tb, p, n_tiles, total);
  c.launches += 1;
  return cudaGetLastError();
}

template <int BN>
cudaError_t launch_bn(const Ctx& c, const GemmArgs& a, std::string* why) {
  CUtensorMap ta, tb;
  if (!make_tmap_bf16(&ta, a.A, a.M, a.Kd, a.Kd, kBM, why)) return cudaErrorInvalidValue;
  if (!make_tmap_bf16(&tb, a.B, a.Ncols, a.Kd, a.Kd, BN, why)) return cudaErrorInvalidValue;
  EpiParams p{};
  p.M = a.M;
  p.Ncols = a.Ncols;
  p.Kd = a.Kd;
  p.epi = a.epi;
  p.out = static_cast<__nv_bfloat16*>(a.out);
  p.ld_out = a.ld_out;
  set_caches(p, a);
  p.x = a.x;
  p.ld_x = a.ld_x;
  p.gate = a.gate;
  p.idx = a.idx;
  p.N = a.N;
  p.flag = c.flag;
  constexpr int smem = GemmCfg<BN>::kSmem;
  static std::atomic<uint64_t> smem_set{0};  // per device
  {
    const cudaError_t e = ensure_smem_limit(k_gemm<BN>, smem, c.device, smem_set);
    if (e != cudaSuccess) return e;
  }
  const int n_tiles = (a.Ncols + BN - 1) / BN;
  const int total = n_tiles * ((a.M + kBM - 1) / kBM);
  const int grid = total < c.num_sms ? total : c.num_sms;
  k_gemm<BN><<<grid, kGemmThreads, smem, c.stream>>>(ta, tb, p, n_tiles, total);
  c.launches += 1;
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_gemm(const Ctx& c, const GemmArgs& a, std::string* why) {
  if (a.M <= 0) return cudaSuccess;
  Timed timed(c, TC_GEMM, 2.0 * a.M * a.Ncols * a.Kd);
  if (a.Kd % kBK != 0 || a.Ncols % 32 != 0) {
    if (why) *why = "GEMM needs K % 64 == 0 and Ncols % 32 == 0";
    return cudaErrorInvalidValue;
  }
  // Pick the tile width with the fewest tile-waves x tile width, where a
  // narrower tile costs a little more per column (more smem traffic per FLOP).
  const int mt = (a.M + kBM - 1) / kBM;
  auto cost = [&](int bn, double per_col) {
    const long tiles = static_cast<long>(mt) * ((a.Ncols + bn - 1) / bn);
    const long waves = (tiles + c.num_sms - 1) / c.num_sms;
    return static_cast<double>(waves) * bn * per_col;
  };
  double best = 1e300;
  int bn = 128;
  // CTA pairs: 256 x 256 tiles over SMs/2 pairs, about 0.8x the cost per output
  // element of a 1-CTA 256-wide tile (half the B traffic through shared memory)
  if (a.Ncols % 256 == 0 && a.M >= 256) {
    const int mt2 = (a.M + 255) / 256;
    const long tiles2 = static_cast<long>(mt2) * (a.Ncols / 256);
    const int pairs = c.num_sms / 2;
    // a pair tile is the same work per SM as a 1-CTA 128 x 256 tile
    const double pc = static_cast<double>((tiles2 + pairs - 1) / pairs) * 256 * kPairCost;
    if (pc < best) best = pc, bn = -1;
  }
  if (a.Ncols % 256 == 0 && cost(256, 1.0) < best) best = cost(256, 1.0), bn = 256;
  if (a.Ncols % 192 == 0 && cost(192, 1.03) < best) best = cost(192, 1.03), bn = 192;
  if (cost(128, 1.12) < best) best = cost(128, 1.12), bn = 128;
  if (bn == -1) return launch_pair(c, a, why);
  if (bn == 256) return launch_bn<256>(c, a, why);
  if (bn == 192) return launch_bn<192>(c, a, why);
  return launch_bn<128>(c, a, why);
}

}  // namespace hsa
