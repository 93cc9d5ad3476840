// k_rows.cu - row kernels around the active-only forward of the HSA step:
// LayerNorm gather of the active rows, the standalone KV-cache scatter, the
// latent embed of the active rows and the velocity head.
//
// Method: "Technical Summary: Heterogeneous Step Allocation (HSA) for
// Efficient Video Generation", section 2.2 (KV-Cache Synchronization): only
// the active tokens A_i are processed, and their fresh K/V rows overwrite the
// stale rows of the per-layer cache.

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "internal.h"
#include "ptx.cuh"

namespace hsa {

constexpr float kLnEps = 1e-5f;

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// Mean and reciprocal standard deviation of a row held as NCH float4 per lane
// (the row is 128*NCH wide); two passes over registers.
template <int NCH>
__device__ __forceinline__ void row_stats(const float4 (&v)[NCH], int D, float& mean, float& rstd) {
  float s = 0.f;
#pragma unroll
  for (int c = 0; c < NCH; ++c) s += (v[c].x + v[c].y) + (v[c].z + v[c].w);
  mean = warp_sum(s) / static_cast<float>(D);
  float q = 0.f;
#pragma unroll
  for (int c = 0; c < NCH; ++c) {
    const float a = v[c].x - mean, b = v[c].y - mean, e = v[c].z - mean, f = v[c].w - mean;
    q += (a * a + b * b) + (e * e + f * f);
  }
  const float var = warp_sum(q) / static_cast<float>(D);
  rstd = 1.0f / sqrtf(var + kLnEps);
}

// ------------------------------------------------------------ LN gather
// One warp per active row: u[m] = bf16(LN(x[idx[m]])).  D = 128 * NCH.
// With `shift`/`scale` (fp32 [D], both or neither) the normalised row is
// modulated: u = LN(x) * (1 + scale) + shift.
template <int NCH>
__global__ void __launch_bounds__(256) k_ln_gather(const float* __restrict__ x,
                                                   const int32_t* __restrict__ idx, int n, int N,
                                                   __nv_bfloat16* __restrict__ u, int* flag,
                                                   const float* __restrict__ shift,
                                                   const float* __restrict__ scale) {
  const int m = blockIdx.x * 8 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (m >= n) return;
  constexpr int D = 128 * NCH;
  const int r = __ldg(idx + m);
  uint2* out = reinterpret_cast<uint2*>(u + static_cast<size_t>(m) * D);
  if (!row_ok(r, N, flag)) {
#pragma unroll
    for (int c = 0; c < NCH; ++c) out[c * 32 + lane] = make_uint2(0u, 0u);
    return;
  }
  const float4* xr = reinterpret_cast<const float4*>(x + static_cast<size_t>(r) * D);
  float4 v[NCH];
#pragma unroll
  for (int c = 0; c < NCH; ++c) v[c] = __ldg(xr + c * 32 + lane);
  float mean, rstd;
  row_stats<NCH>(v, D, mean, rstd);
#pragma unroll
  for (int c = 0; c < NCH; ++c) {
    float4 y = make_float4((v[c].x - mean) * rstd, (v[c].y - mean) * rstd,
                           (v[c].z - mean) * rstd, (v[c].w - mean) * rstd);
    if (scale != nullptr) {
      const float4 sc = __ldg(reinterpret_cast<const float4*>(scale) + c * 32 + lane);
      const float4 sh = __ldg(reinterpret_cast<const float4*>(shift) + c * 32 + lane);
      y = make_float4(fmaf(y.x, 1.f + sc.x, sh.x), fmaf(y.y, 1.f + sc.y, sh.y),
                      fmaf(y.z, 1.f + sc.z, sh.z), fmaf(y.w, 1.f + sc.w, sh.w));
    }
    out[c * 32 + lane] = make_uint2(pack_bf16(y.x, y.y), pack_bf16(y.z, y.w));
  }
}

// Any D multiple of 128: three passes over the row (L1/L2 serve the re-reads).
__global__ void __launch_bounds__(256) k_ln_gather_any(const float* __restrict__ x,
                                                       const int32_t* __restrict__ idx, int n,
                                                       int N, int D,
                                                       __nv_bfloat16* __restrict__ u, int* flag,
                                                       const float* __restrict__ shift,
                                                       const float* __restrict__ scale) {
  const int m = blockIdx.x * 8 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (m >= n) return;
  const int r = __ldg(idx + m);
  uint2* out = reinterpret_cast<uint2*>(u + static_cast<size_t>(m) * D);
  const int nv = D / 4;
  if (!row_ok(r, N, flag)) {
    for (int c = lane; c < nv; c += 32) out[c] = make_uint2(0u, 0u);
    return;
  }
  const float4* xr = reinterpret_cast<const float4*>(x + static_cast<size_t>(r) * D);
  float s = 0.f;
  for (int c = lane; c < nv; c += 32) {
    const float4 a = __ldg(xr + c);
    s += (a.x + a.y) + (a.z + a.w);
  }
  const float mean = warp_sum(s) / static_cast<float>(D);
  float q = 0.f;
  for (int c = lane; c < nv; c += 32) {
    const float4 a = __ldg(xr + c);
    const float p0 = a.x - mean, p1 = a.y - mean, p2 = a.z - mean, p3 = a.w - mean;
    q += (p0 * p0 + p1 * p1) + (p2 * p2 + p3 * p3);
  }
  const float rstd = 1.0f / sqrtf(warp_sum(q) / static_cast<float>(D) + kLnEps);
  for (int c = lane; c < nv; c += 32) {
    const float4 a = __ldg(xr + c);
    float4 y = make_float4((a.x - mean) * rstd, (a.y - mean) * rstd, (a.z - mean) * rstd,
                           (a.w - mean) * rstd);
    if (scale != nullptr) {
      const float4 sc = __ldg(reinterpret_cast<const float4*>(scale) + c);
      const float4 sh = __ldg(reinterpret_cast<const float4*>(shift) + c);
      y = make_float4(fmaf(y.x, 1.f + sc.x, sh.x), fmaf(y.y, 1.f + sc.y, sh.y),
                      fmaf(y.z, 1.f + sc.z, sh.z), fmaf(y.w, 1.f + sc.w, sh.w));
    }
    out[c] = make_uint2(pack_bf16(y.x, y.y), pack_bf16(y.z, y.w));
  }
}

cudaError_t launch_ln_gather(const Ctx& c, const float* x, const int32_t* idx, int n, void* u,
                             const float* shift, const float* scale) {
  if (n <= 0) return cudaSuccess;
  const int D = c.cfg.D, N = c.cfg.N;
  Timed timed(c, TC_ROWS, static_cast<double>(n) * D * (4 + 2));
  const dim3 grid((n + 7) / 8), block(256);
  auto* uo = static_cast<__nv_bfloat16*>(u);
  switch (D / 128) {
    case 1: k_ln_gather<1><<<grid, block, 0, c.stream>>>(x, idx, n, N, uo, c.flag, shift, scale); break;
    case 2: k_ln_gather<2><<<grid, block, 0, c.stream>>>(x, idx, n, N, uo, c.flag, shift, scale); break;
    case 4: k_ln_gather<4><<<grid, block, 0, c.stream>>>(x, idx, n, N, uo, c.flag, shift, scale); break;
    case 8: k_ln_gather<8><<<grid, block, 0, c.stream>>>(x, idx, n, N, uo, c.flag, shift, scale); break;
    case 12: k_ln_gather<12><<<grid, block, 0, c.stream>>>(x, idx, n, N, uo, c.flag, shift, scale); break;
    case 16: k_ln_gather<16><<<grid, block, 0, c.stream>>>(x, idx, n, N, uo, c.flag, shift, scale); break;
    default: k_ln_gather_any<<<grid, block, 0, c.stream>>>(x, idx, n, N, D, uo, c.flag, shift, scale); break;
  }
  c.launches += 1;
  return cudaGetLastError();
}

// ------------------------------------------------------------ KV scatter
// k_cache[idx[m]] = k_rows[m], v_cache[idx[m]] = v_rows[m]; 16-byte vectors.
// Source row m of K (V) starts at k_rows (v_rows) + m * src_ld, in 16-byte units.
__global__ void __launch_bounds__(256) k_kv_scatter(const uint4* __restrict__ k_rows,
                                                    const uint4* __restrict__ v_rows, int src_ld,
                                                    const int32_t* __restrict__ idx, int n, int N,
                                                    int vec_per_row, uint4* __restrict__ kc,
                                                    uint4* __restrict__ vc, int* flag) {
  const size_t total = static_cast<size_t>(n) * vec_per_row;
  for (size_t t = blockIdx.x * static_cast<size_t>(blockDim.x) + threadIdx.x; t < total;
       t += static_cast<size_t>(gridDim.x) * blockDim.x) {
    const int m = static_cast<int>(t / vec_per_row);
    const int c = static_cast<int>(t - static_cast<size_t>(m) * vec_per_row);
    const int r = __ldg(idx + m);
    if (!row_ok(r, N, flag)) continue;
    const size_t dst = static_cast<size_t>(r) * vec_per_row + c;
    const size_t src = static_cast<size_t>(m) * src_ld + c;
    __stcs(kc + dst, __ldcs(k_rows + src));
    __stcs(vc + dst, __ldcs(v_rows + src));
  }
}

cudaError_t launch_kv_scatter(const Ctx& c, const void* k_rows, const void* v_rows, int src_ld,
                              const int32_t* idx, int n, void* kc, void* vc) {
  if (n <= 0) return cudaSuccess;
  Timed timed(c, TC_ROWS, static_cast<double>(n) * c.cfg.D * 2 * 2 * 2);
  const int vpr = c.cfg.D / 8;
  const size_t total = static_cast<size_t>(n) * vpr;
  size_t blocks = (total + 255) / 256;
  const size_t cap = static_cast<size_t>(c.num_sms) * 16;
  if (blocks > cap) blocks = cap;
  k_kv_scatter<<<static_cast<unsigned>(blocks), 256, 0, c.stream>>>(
      static_cast<const uint4*>(k_rows), static_cast<const uint4*>(v_rows), src_ld / 8, idx, n,
      c.cfg.N, vpr,
      static_cast<uint4*>(kc), static_cast<uint4*>(vc), c.flag);
  c.launches += 1;
  return cudaGetLastError();
}

// ------------------------------------------------------------ embed
// h[idx[m], j] = sum_c W_in[j, c] * x_lat[idx[m], c]; C = 16.  A thread owns
// four hidden columns j0..j0+3: it loads their 64 weights once and reuses them
// for kEmbedRows active rows, each row's 16 latent values being one broadcast
// load for the whole warp; every row's four outputs are one 16-byte store
// (a warp stores 512 contiguous bytes).
constexpr int kEmbedRows = 16;
constexpr int kEmbedThreads = 128;

__global__ void __launch_bounds__(kEmbedThreads) k_embed(const float* __restrict__ w_in,
                                                         const float* __restrict__ x_lat,
                                                         const int32_t* __restrict__ idx, int n,
                                                         int N, int D, float* __restrict__ h,
                                                         int* flag) {
  const int j0 = (blockIdx.x * kEmbedThreads + threadIdx.x) * 4;
  if (j0 >= D) return;
  float w[4][16];
#pragma unroll
  for (int jj = 0; jj < 4; ++jj) {
    const float4* wr = reinterpret_cast<const float4*>(w_in + static_cast<size_t>(j0 + jj) * 16);
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const float4 v = __ldg(wr + q);
      w[jj][4 * q] = v.x;
      w[jj][4 * q + 1] = v.y;
      w[jj][4 * q + 2] = v.z;
      w[jj][4 * q + 3] = v.w;
    }
  }
  const int m0 = blockIdx.y * kEmbedRows;
  const int m1 = min(n, m0 + kEmbedRows);
  for (int m = m0; m < m1; ++m) {
    const int r = __ldg(idx + m);
    if (!row_ok(r, N, flag)) continue;
    const float4* xl = reinterpret_cast<const float4*>(x_lat + static_cast<size_t>(r) * 16);
    float xv[16];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const float4 a = __ldg(xl + q);
      xv[4 * q] = a.x;
      xv[4 * q + 1] = a.y;
      xv[4 * q + 2] = a.z;
      xv[4 * q + 3] = a.w;
    }
    float acc[4];
#pragma unroll
    for (int jj = 0; jj < 4; ++jj) {
      float s = 0.f;
#pragma unroll
      for (int c = 0; c < 16; ++c) s = fmaf(w[jj][c], xv[c], s);
      acc[jj] = s;
    }
    *reinterpret_cast<float4*>(h + static_cast<size_t>(r) * D + j0) =
        make_float4(acc[0], acc[1], acc[2], acc[3]);
  }
}

cudaError_t launch_embed(const Ctx& c, const float* w_in, const float* x_lat, const int32_t* idx,
                         int n, float* h) {
  if (n <= 0) return cudaSuccess;
  Timed timed(c, TC_ROWS, static_cast<double>(n) * (64 + 4.0 * c.cfg.D));
  const int D = c.cfg.D;
  const dim3 grid((D / 4 + kEmbedThreads - 1) / kEmbedThreads, (n + kEmbedRows - 1) / kEmbedRows);
  k_embed<<<grid, kEmbedThreads, 0, c.stream>>>(w_in, x_lat, idx, n, c.cfg.N, D, h, c.flag);
  c.launches += 1;
  return cudaGetLastError();
}

// ------------------------------------------------------------ velocity head
// v_fresh[idx[m], o] = sum_j LN(h[idx[m]])_j W_head[o, j], fp32 throughout.
// One warp takes kHeadRows active rows: the statistics of each row come from
// two passes over it (mean, then the centred sum of squares), and the dot
// products with the 16 rows of W_head read each W_head vector once for all of
// the warp's rows, so W_head's L1 traffic is shared kHeadRows ways.  The 16
// sums of each row are reduced with butterflies.
constexpr int kHeadRows = 4;

__global__ void __launch_bounds__(128) k_head(const float* __restrict__ w_head,
                                              const float* __restrict__ h,
                                              const int32_t* __restrict__ idx, int n, int N,
                                              int D, float* __restrict__ v_fresh, int* flag) {
  const int m0 = (blockIdx.x * 4 + (threadIdx.x >> 5)) * kHeadRows;
  const int lane = threadIdx.x & 31;
  if (m0 >= n) return;
  const int nv = D / 4;
  const float4* hr[kHeadRows];
  int r[kHeadRows];
  bool use[kHeadRows];
#pragma unroll
  for (int k = 0; k < kHeadRows; ++k) {
    r[k] = m0 + k < n ? __ldg(idx + m0 + k) : 0;
    use[k] = m0 + k < n && row_ok(r[k], N, flag);
    hr[k] = reinterpret_cast<const float4*>(h + static_cast<size_t>(use[k] ? r[k] : 0) * D);
  }
  float mean[kHeadRows], rstd[kHeadRows];
#pragma unroll
  for (int k = 0; k < kHeadRows; ++k) {
    float s = 0.f;
    for (int c = lane; c < nv; c += 32) {
      const float4 a = __ldg(hr[k] + c);
      s += (a.x + a.y) + (a.z + a.w);
    }
    mean[k] = warp_sum(s) / static_cast<float>(D);
    float q = 0.f;
    for (int c = lane; c < nv; c += 32) {
      const float4 a = __ldg(hr[k] + c);
      const float p0 = a.x - mean[k], p1 = a.y - mean[k], p2 = a.z - mean[k], p3 = a.w - mean[k];
      q += (p0 * p0 + p1 * p1) + (p2 * p2 + p3 * p3);
    }
    rstd[k] = 1.0f / sqrtf(warp_sum(q) / static_cast<float>(D) + kLnEps);
  }
  float acc[kHeadRows][16];
#pragma unroll
  for (int k = 0; k < kHeadRows; ++k)
#pragma unroll
    for (int o = 0; o < 16; ++o) acc[k][o] = 0.f;
  for (int c = lane; c < nv; c += 32) {
    float4 a[kHeadRows];
#pragma unroll
    for (int k = 0; k < kHeadRows; ++k) {
      a[k] = __ldg(hr[k] + c);
      a[k].x = (a[k].x - mean[k]) * rstd[k];
      a[k].y = (a[k].y - mean[k]) * rstd[k];
      a[k].z = (a[k].z - mean[k]) * rstd[k];
      a[k].w = (a[k].w - mean[k]) * rstd[k];
    }
#pragma unroll
    for (int o = 0; o < 16; ++o) {
      const float4 w = __ldg(reinterpret_cast<const float4*>(w_head + static_cast<size_t>(o) * D) + c);
#pragma unroll
      for (int k = 0; k < kHeadRows; ++k)
        acc[k][o] = fmaf(a[k].x, w.x, fmaf(a[k].y, w.y, fmaf(a[k].z, w.z, fmaf(a[k].w, w.w, acc[k][o]))));
    }
  }
#pragma unroll
  for (int k = 0; k < kHeadRows; ++k) {
#pragma unroll
    for (int o = 0; o < 16; ++o) acc[k][o] = warp_sum(acc[k][o]);
    if (use[k] && lane < 4) {
      // lane l writes channels 4l..4l+3 (constant register indices)
      float4 outv = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
      for (int l = 0; l < 4; ++l)
        if (lane == l)
          outv = make_float4(acc[k][4 * l], acc[k][4 * l + 1], acc[k][4 * l + 2], acc[k][4 * l + 3]);
      reinterpret_cast<float4*>(v_fresh + static_cast<size_t>(r[k]) * 16)[lane] = outv;
    }
  }
}

cudaError_t launch_head(const Ctx& c, const float* w_head, const float* h, const int32_t* idx,
                        int n, float* v_fresh) {
  if (n <= 0) return cudaSuccess;
  Timed timed(c, TC_ROWS, static_cast<double>(n) * (4.0 * c.cfg.D + 64));
  const int warps = (n + kHeadRows - 1) / kHeadRows;
  k_head<<<(warps + 3) / 4, 128, 0, c.stream>>>(w_head, h, idx, n, c.cfg.N, c.cfg.D, v_fresh,
                                                 c.flag);
  c.launches += 1;
  return cudaGetLastError();
}

}  // namespace hsa
