// Memory-bound kernels of the image half: index setup, RoPE angle table,
// patch gather (im2col with the processor normalisation), RMSNorm, merge
// gather, masked scatter and weight packing. Every one is a coalesced,
// vectorised streaming kernel; none uses the tensor cores.
#include <algorithm>
#include <type_traits>

#include "gemm_rows.cuh"
#include "kernels.cuh"
#include "nvfp4.cuh"

#define VLM_DEBUG_FILE_ID 1

namespace vlm {

VLM_DEBUG_UNIT(debug_word_small_kernels)

// ---------------------------------------------------------------------------
// Index setup: per-image tables and per-token (row, col) positions.
// ---------------------------------------------------------------------------
__global__ void setup_kernel(ImageChunk chunk, ImgInfo* info, int32_t* cu, int32_t* qt, int32_t* i2c,
                             int32_t* pos, int n_images) {
  griddep_wait();
  griddep_launch_dependents();
  const int tid = blockIdx.x * blockDim.x + threadIdx.x;
  if (tid < chunk.count) {
    const int b = chunk.first + tid;
    ImgInfo in;
    in.h = chunk.h[tid];
    in.w = chunk.w[tid];
    in.H = chunk.H[tid];
    in.W = chunk.W[tid];
    in.tok_off = chunk.tok_off[tid];
    in.m_off = chunk.m_off[tid];
    in.qt_off = chunk.qt_off[tid];
    in.pad = 0;
    in.pix_off = chunk.pix_off[tid];
    info[b] = in;
    cu[b] = chunk.tok_off[tid];
    qt[b] = chunk.qt_off[tid];
    if (i2c != nullptr) i2c[b] = chunk.i2c_off[tid];
    if (b == n_images - 1) {
      cu[n_images] = chunk.tok_off[tid + 1];
      qt[n_images] = chunk.qt_off[tid + 1];
      if (i2c != nullptr) i2c[n_images] = chunk.i2c_off[tid + 1];
    }
  }
  if (pos == nullptr) return;
  const int t0 = chunk.tok_off[0], t1 = chunk.tok_off[chunk.count];
  for (int t = t0 + tid; t < t1; t += gridDim.x * blockDim.x) {
    int lo = 0, hi = chunk.count - 1;  // last image whose offset <= t
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (chunk.tok_off[mid] <= t) lo = mid; else hi = mid - 1;
    }
    const int local = t - chunk.tok_off[lo];
    const int w = chunk.w[lo];
    if (VLM_DCHECK(local >= 0 && local < chunk.h[lo] * w)) pos[t] = ((local / w) << 16) | (local % w);
  }
}

// 2D RoPE angle table: tab[p][i] = (cos, sin)(p * w_k), w_k = theta^(-2k/dh),
// k = 2i for the row half (i < dh/4) and k = 2(i - dh/4) + 1 for the column half.
__global__ void rope_table_kernel(float theta, int head_dim, int max_pos, float2* tab) {
  griddep_wait();
  griddep_launch_dependents();
  const int half = head_dim / 2, quarter = head_dim / 4;
  const int idx = blockIdx.x * blockDim.x + threadIdx.x;
  if (idx >= max_pos * half) return;
  const int p = idx / half, i = idx % half;
  const int k = i < quarter ? 2 * i : 2 * (i - quarter) + 1;
  const double omega = pow(static_cast<double>(theta), -2.0 * k / head_dim);
  double s, c;
  sincos(static_cast<double>(p) * omega, &s, &c);
  tab[idx] = make_float2(static_cast<float>(c), static_cast<float>(s));
}

__device__ __forceinline__ int find_block(const int32_t* cu, int n, int t) {
  int lo = 0, hi = n - 1;  // last b with cu[b] <= t
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (__ldg(cu + mid) <= t) lo = mid; else hi = mid - 1;
  }
  return lo;
}

// ---------------------------------------------------------------------------
// Patch gather: one warp per patch; column k = ch*p*p + ky*p + kx of the
// conv weight; columns >= 3p^2 are zero padding.
// ---------------------------------------------------------------------------
__constant__ float c_mean[3] = {0.48145466f, 0.4578275f, 0.40821073f};
__constant__ float c_std[3] = {0.26862954f, 0.26130258f, 0.27577711f};
// (x - mean) / std as one fused multiply-add: x * (1 / std) + (-mean / std), both rounded once from double
__constant__ float c_inv_std[3] = {static_cast<float>(1.0 / 0.26862954), static_cast<float>(1.0 / 0.26130258),
                                   static_cast<float>(1.0 / 0.27577711)};
__constant__ float c_shift[3] = {static_cast<float>(-0.48145466 / 0.26862954), static_cast<float>(-0.4578275 / 0.26130258),
                                 static_cast<float>(-0.40821073 / 0.27577711)};

__global__ void im2col_kernel(const float* __restrict__ pix, const ImgInfo* __restrict__ info,
                              const int32_t* __restrict__ cu, int n_images, int64_t T, int p, int kp,
                              int normalize, __nv_bfloat16* __restrict__ out) {
  griddep_wait();
  griddep_launch_dependents();
  const int lane = threadIdx.x & 31;
  const int64_t warps = static_cast<int64_t>(gridDim.x) * (blockDim.x >> 5);
  const int pp = p * p, kreal = 3 * pp;
  for (int64_t t = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5; t < T; t += warps) {
    const int b = find_block(cu, n_images, static_cast<int>(t));
    const ImgInfo in = info[b];
    const int local = static_cast<int>(t) - in.tok_off;
    if (!VLM_DCHECK(local >= 0 && local < in.h * in.w && in.h * p <= in.H && in.w * p <= in.W)) continue;
    const int r = local / in.w, c = local % in.w;
    const float* base = pix + in.pix_off;
    uint32_t* orow = reinterpret_cast<uint32_t*>(out + t * kp);
    for (int k2 = lane; k2 < kp / 2; k2 += 32) {
      float v[2];
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const int k = 2 * k2 + e;
        float val = 0.f;
        if (k < kreal) {
          const int ch = k / pp, rem = k - ch * pp, ky = rem / p, kx = rem - ky * p;
          val = __ldg(base + (static_cast<int64_t>(ch) * in.H + r * p + ky) * in.W + c * p + kx);
          if (normalize) val = (val - c_mean[ch]) / c_std[ch];
        }
        v[e] = val;
      }
      orow[k2] = pack_bf16x2(v[0], v[1]);
    }
  }
}

// Tiled patch gather for patch size P (14 or 16): a work item is a segment of
// up to kI2cPatches patches of one patch row. The item's 3 x P pixel-row
// segments are read with coalesced loads into shared memory (normalised on the
// way), then the item's patch rows are written as consecutive bf16 pairs.
constexpr int kI2cThreads = 128;  // 4 warps: small CTAs, so several items per SM are in flight at once

template <int P>
__global__ void __launch_bounds__(kI2cThreads) im2col_tiled_kernel(const float* __restrict__ pix,
                                                           const ImgInfo* __restrict__ info,
                                                           const int32_t* __restrict__ i2c, int n_images,
                                                           int items, int kp, int normalize,
                                                           __nv_bfloat16* __restrict__ out) {
  constexpr int PP = P * P, SEGMAX = kI2cPatches * P;
  __shared__ __align__(16) float tile[3 * P * SEGMAX];
  griddep_wait();
  griddep_launch_dependents();
  for (int g = blockIdx.x; g < items; g += gridDim.x) {
    const int b = find_block(i2c, n_images, g);
    const ImgInfo in = info[b];
    const int nch = (in.w + kI2cPatches - 1) / kI2cPatches;
    const int local = g - __ldg(i2c + b);
    const int r = local / nch, c0 = (local - r * nch) * kI2cPatches;
    // the item lies inside its image (the same decision in every thread of the CTA)
    if (!VLM_DCHECK(local >= 0 && r < in.h && c0 < in.w && in.h * P <= in.H && in.w * P <= in.W)) continue;
    const int npat = min(kI2cPatches, in.w - c0), seg = npat * P;
    const float* base = pix + in.pix_off;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    // pixel-row segments warp, warp + 8, ...: every load of the lane is issued
    // before the first one is used, so their latencies overlap
    constexpr int NWARPS = kI2cThreads / 32, ROWS = 3 * P, RPW = (ROWS + NWARPS - 1) / NWARPS, XPL = (SEGMAX + 31) / 32;
    float buf[RPW][XPL];
#pragma unroll
    for (int i = 0; i < RPW; ++i) {
      const int row = warp + NWARPS * i;
      if (row < ROWS) {
        const int ch = row / P, ky = row - ch * P;
        const float* src = base + (static_cast<int64_t>(ch) * in.H + r * P + ky) * in.W + c0 * P;
#pragma unroll
        for (int q = 0; q < XPL; ++q) {
          const int x = lane + 32 * q;
          buf[i][q] = x < seg ? __ldg(src + x) : 0.f;
        }
      }
    }
    __syncthreads();  // the previous item's readers are done with the tile
#pragma unroll
    for (int i = 0; i < RPW; ++i) {
      const int row = warp + NWARPS * i;
      if (row < ROWS) {
        const int ch = row / P;
        const float scale = normalize ? c_inv_std[ch] : 1.0f, shift = normalize ? c_shift[ch] : 0.0f;
#pragma unroll
        for (int q = 0; q < XPL; ++q) {
          const int x = lane + 32 * q;
          if (x < seg) tile[row * SEGMAX + x] = fmaf(buf[i][q], scale, shift);
        }
      }
    }
    __syncthreads();
    // each output bf16 pair (kx, kx + 1) of pixel row (ch, ky) is two adjacent tile floats
    constexpr int HALF_P = P / 2, REAL_PAIRS = 3 * PP / 2;
    const int half = kp / 2;
    const int64_t t0 = in.tok_off + static_cast<int64_t>(r) * in.w + c0;
    // pair k2 of a patch row is (pixel row k2 / (P/2), pair k2 % (P/2)); a lane steps
    // k2 by 32, i.e. the row by 32 / (P/2) and the pair by 32 % (P/2), with a carry
    constexpr int STEP_ROW = 32 / HALF_P, STEP_PAIR = 32 % HALF_P;
    const int row0 = lane / HALF_P, pair0 = lane % HALF_P;
    for (int pi = warp; pi < npat; pi += NWARPS) {  // one patch row per warp
      uint32_t* orow = reinterpret_cast<uint32_t*>(out + (t0 + pi) * kp);
      const float* trow = tile + pi * P;
      int row = row0, pair = pair0;
      for (int k2 = lane; k2 < half; k2 += 32) {
        uint32_t w = 0u;  // the zero padding past 3 P^2
        if (k2 < REAL_PAIRS) {
          const float2 v = *reinterpret_cast<const float2*>(&trow[row * SEGMAX + 2 * pair]);
          w = pack_bf16x2(v.x, v.y);
        }
        orow[k2] = w;
        row += STEP_ROW;
        pair += STEP_PAIR;
        if (pair >= HALF_P) { pair -= HALF_P; ++row; }
      }
    }
  }
}

// ---------------------------------------------------------------------------
// RMSNorm, one warp per row of `width` fp32 values (width % 128 == 0, <= 2048).
// With g0: y = norm(x) * g0 is written back to x, and out = bf16(norm(y) * g1).
// Without g0: out = bf16(norm(x) * g1).
// OUT 1: out is E4M3 instead, of norm(.) * g1 * f8_scale (round to nearest
// even, saturating). OUT 2: out is NVFP4 -- E2M1 codes [rows, width / 2] and
// block scales in out_sf -- of the fp32 values norm(.) * g1 with global scale
// f8_scale (a block of 16 spans four lanes).
// ---------------------------------------------------------------------------
template <int NV, int OUT = 0>
__global__ void rmsnorm_kernel(float* __restrict__ x, const float* __restrict__ g0,
                               const float* __restrict__ g1, void* __restrict__ out_v,
                               int64_t rows, float eps, float f8_scale, uint8_t* __restrict__ out_sf) {
  constexpr bool kF8 = OUT == 1;
  griddep_wait();
  griddep_launch_dependents();
  constexpr int width = NV * 128;
  const int lane = threadIdx.x & 31;
  const int64_t warps = static_cast<int64_t>(gridDim.x) * (blockDim.x >> 5);
  for (int64_t row = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5; row < rows;
       row += warps) {
    float4* xr = reinterpret_cast<float4*>(x + row * width);
    float4 v[NV];
    float ss = 0.f;
#pragma unroll
    for (int j = 0; j < NV; ++j) {
      v[j] = xr[lane + 32 * j];
      ss += v[j].x * v[j].x + v[j].y * v[j].y + v[j].z * v[j].z + v[j].w * v[j].w;
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
    float rs = rsqrtf(ss / width + eps);
    if (g0 != nullptr) {
      const float4* gr = reinterpret_cast<const float4*>(g0);
      ss = 0.f;
#pragma unroll
      for (int j = 0; j < NV; ++j) {
        const float4 g = __ldg(gr + lane + 32 * j);
        v[j].x *= rs * g.x; v[j].y *= rs * g.y; v[j].z *= rs * g.z; v[j].w *= rs * g.w;
        xr[lane + 32 * j] = v[j];
        ss += v[j].x * v[j].x + v[j].y * v[j].y + v[j].z * v[j].z + v[j].w * v[j].w;
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
      rs = rsqrtf(ss / width + eps);
    }
    const float4* gr = reinterpret_cast<const float4*>(g1);
    if constexpr (OUT == 2) {
      uint16_t* orow = reinterpret_cast<uint16_t*>(static_cast<uint8_t*>(out_v) + row * (width / 2));
      const float six_sg = 6.0f * f8_scale;
#pragma unroll
      for (int j = 0; j < NV; ++j) {
        const float4 g = __ldg(gr + lane + 32 * j);
        const float y0 = v[j].x * rs * g.x, y1 = v[j].y * rs * g.y, y2 = v[j].z * rs * g.z, y3 = v[j].w * rs * g.w;
        float amax = fmaxf(fmaxf(fabsf(y0), fabsf(y1)), fmaxf(fabsf(y2), fabsf(y3)));
        amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 1));
        amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 2));
        float r;
        const uint32_t sb = nvfp4_block_scale(amax, f8_scale, six_sg, r);
        orow[lane + 32 * j] = static_cast<uint16_t>(e2m1x2(y0 * r, y1 * r) | (e2m1x2(y2 * r, y3 * r) << 8));
        if ((lane & 3) == 0) out_sf[nvfp4_sf_offset(row, (lane + 32 * j) >> 2, width)] = static_cast<uint8_t>(sb);
      }
    } else if constexpr (kF8) {
      uint32_t* orow = reinterpret_cast<uint32_t*>(static_cast<uint8_t*>(out_v) + row * width);
#pragma unroll
      for (int j = 0; j < NV; ++j) {
        const float4 g = __ldg(gr + lane + 32 * j);
        orow[lane + 32 * j] = pack_e4m3x4(v[j].x * rs * g.x * f8_scale, v[j].y * rs * g.y * f8_scale,
                                          v[j].z * rs * g.z * f8_scale, v[j].w * rs * g.w * f8_scale);
      }
    } else {
      uint2* orow = reinterpret_cast<uint2*>(static_cast<__nv_bfloat16*>(out_v) + row * width);
#pragma unroll
      for (int j = 0; j < NV; ++j) {
        const float4 g = __ldg(gr + lane + 32 * j);
        uint2 o;
        o.x = pack_bf16x2(v[j].x * rs * g.x, v[j].y * rs * g.y);
        o.y = pack_bf16x2(v[j].z * rs * g.z, v[j].w * rs * g.w);
        orow[lane + 32 * j] = o;
      }
    }
  }
}


// RMSNorm of bf16 rows into bf16 (in place allowed), one warp per row.
template <int NV>
__global__ void rmsnorm_bf16_kernel(const __nv_bfloat16* x, const float* __restrict__ g, __nv_bfloat16* out,
                                    int64_t rows, float eps) {
  griddep_wait();
  griddep_launch_dependents();
  constexpr int width = NV * 128;
  const int lane = threadIdx.x & 31;
  const int64_t warps = static_cast<int64_t>(gridDim.x) * (blockDim.x >> 5);
  for (int64_t t = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5; t < rows; t += warps) {
    const uint2* xr = reinterpret_cast<const uint2*>(x + t * width);
    float v[NV][4];
    float ss = 0.f;
#pragma unroll
    for (int j = 0; j < NV; ++j) {
      const uint2 u = xr[lane + 32 * j];
      const __nv_bfloat162 a = *reinterpret_cast<const __nv_bfloat162*>(&u.x);
      const __nv_bfloat162 bb = *reinterpret_cast<const __nv_bfloat162*>(&u.y);
      v[j][0] = __low2float(a); v[j][1] = __high2float(a);
      v[j][2] = __low2float(bb); v[j][3] = __high2float(bb);
#pragma unroll
      for (int e = 0; e < 4; ++e) ss += v[j][e] * v[j][e];
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
    const float rs = rsqrtf(ss / width + eps);
    uint2* orow = reinterpret_cast<uint2*>(out + t * width);
    const float4* gr = reinterpret_cast<const float4*>(g);
#pragma unroll
    for (int j = 0; j < NV; ++j) {
      const float4 gg = __ldg(gr + lane + 32 * j);
      uint2 o;
      o.x = pack_bf16x2(v[j][0] * rs * gg.x, v[j][1] * rs * gg.y);
      o.y = pack_bf16x2(v[j][2] * rs * gg.z, v[j][3] * rs * gg.w);
      orow[lane + 32 * j] = o;
    }
  }
}

// ---------------------------------------------------------------------------
// Masked scatter: (1) placeholder count per 256-id chunk, (2) one-block scan
// and total check, (3) destination row of every placeholder, (4) row copy.
// Steps 3 and 4 do nothing unless step 2 found count == n_image_tokens.
// ---------------------------------------------------------------------------
__global__ void scatter_count_kernel(const int64_t* __restrict__ ids, int64_t n, int64_t token,
                                     int32_t* __restrict__ chunk_count) {
  griddep_wait();
  griddep_launch_dependents();
  const int64_t i = static_cast<int64_t>(blockIdx.x) * 256 + threadIdx.x;
  const int flag = (i < n && ids[i] == token) ? 1 : 0;
  const int wc = __popc(__ballot_sync(0xffffffffu, flag));
  __shared__ int s[8];
  if ((threadIdx.x & 31) == 0) s[threadIdx.x >> 5] = wc;
  __syncthreads();
  if (threadIdx.x == 0) {
    int tot = 0;
#pragma unroll
    for (int w = 0; w < 8; ++w) tot += s[w];
    chunk_count[blockIdx.x] = tot;
  }
}

__global__ void scatter_scan_kernel(const int32_t* __restrict__ chunk_count, int64_t n_chunks,
                                    int64_t expected, int64_t* __restrict__ chunk_base,
                                    int32_t* __restrict__ ok_flag, int32_t* status) {
  griddep_wait();
  griddep_launch_dependents();
  // 1024 threads; sequential over blocks of 1024 chunks with a running carry.
  __shared__ int64_t warp_sums[32];
  __shared__ int64_t carry;
  if (threadIdx.x == 0) carry = 0;
  __syncthreads();
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  for (int64_t base = 0; base < n_chunks; base += 1024) {
    const int64_t i = base + threadIdx.x;
    const int64_t v = i < n_chunks ? chunk_count[i] : 0;
    int64_t incl = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int64_t y = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += y;
    }
    if (lane == 31) warp_sums[warp] = incl;
    __syncthreads();
    if (warp == 0) {
      int64_t ws = warp_sums[lane];
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int64_t y = __shfl_up_sync(0xffffffffu, ws, o);
        if (lane >= o) ws += y;
      }
      warp_sums[lane] = ws;  // inclusive over warps
    }
    __syncthreads();
    const int64_t before = carry + (warp > 0 ? warp_sums[warp - 1] : 0) + incl - v;
    if (i < n_chunks) chunk_base[i] = before;
    __syncthreads();
    if (threadIdx.x == 0) carry += warp_sums[31];
    __syncthreads();
  }
  if (threadIdx.x == 0) {
    const int good = (carry == expected) ? 1 : 0;
    *ok_flag = good;
    if (!good) set_status(status, VLM_ERR_COUNT_MISMATCH);
  }
}

__global__ void scatter_positions_kernel(const int64_t* __restrict__ ids, int64_t n, int64_t token,
                                         const int64_t* __restrict__ chunk_base,
                                         const int32_t* __restrict__ ok_flag,
                                         int64_t* __restrict__ dst_rows, int64_t n_img) {
  griddep_wait();
  griddep_launch_dependents();
  if (*ok_flag == 0) return;
  const int64_t i = static_cast<int64_t>(blockIdx.x) * 256 + threadIdx.x;
  const int flag = (i < n && ids[i] == token) ? 1 : 0;
  const unsigned ballot = __ballot_sync(0xffffffffu, flag);
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  __shared__ int s[8];
  if (lane == 0) s[warp] = __popc(ballot);
  __syncthreads();
  int before = 0;
  for (int w = 0; w < warp; ++w) before += s[w];
  before += __popc(ballot & ((1u << lane) - 1u));
  if (flag) {
    const int64_t k = chunk_base[blockIdx.x] + before;
    if (VLM_DCHECK(k >= 0 && k < n_img)) dst_rows[k] = i;
  }
}

__global__ void scatter_copy_kernel(const uint4* __restrict__ img, uint4* __restrict__ text,
                                    const int64_t* __restrict__ dst_rows,
                                    const int32_t* __restrict__ ok_flag, int64_t n_rows,
                                    int64_t vec_per_row, int64_t n_text) {
  griddep_wait();
  griddep_launch_dependents();
  if (*ok_flag == 0) return;
  const int lane = threadIdx.x & 31;
  const int64_t warps = static_cast<int64_t>(gridDim.x) * (blockDim.x >> 5);
  for (int64_t k = static_cast<int64_t>(blockIdx.x) * (blockDim.x >> 5) + (threadIdx.x >> 5); k < n_rows;
       k += warps) {
    const int64_t d = dst_rows[k];
    if (!VLM_DCHECK(d >= 0 && d < n_text)) continue;
    const uint4* src = img + k * vec_per_row;
    uint4* dst = text + d * vec_per_row;
    int64_t j = lane;
    for (; j + 96 < vec_per_row; j += 128) {
      const uint4 a = __ldg(src + j), b = __ldg(src + j + 32), c = __ldg(src + j + 64), d = __ldg(src + j + 96);
      dst[j] = a;
      dst[j + 32] = b;
      dst[j + 64] = c;
      dst[j + 96] = d;
    }
    for (; j < vec_per_row; j += 32) dst[j] = __ldg(src + j);
  }
}

// Single-launch masked scatter for up to kScatterFusedMaxIds ids. Each CTA
// owns a slice [k0, k1) of the image rows. Its thread 0 first starts bulk
// copies (cp.async.bulk, no multicast) of the slice's first rows into a ring
// of row buffers in shared memory; meanwhile all threads (1) turn the ids into
// a placeholder bitmask with coalesced loads, (2) count the bits of a
// contiguous range of words per thread and rank them with one block scan and
// (3) record the text row of each row of the slice. Only if the placeholder
// total equals n_img does thread 0 then (4) store each buffered row to its
// text row with a bulk copy and refill the buffer with the next row of the
// slice. All CTAs compute the same total, so either every slice is copied or
// nothing is written; CTA 0 reports a mismatch. Every wait is bounded.
constexpr int kScatterFusedThreads = 512;
constexpr int64_t kScatterFusedMaxIds = 32768;
constexpr int kScatterFusedMaxRows = 2048;      // image rows per CTA slice
constexpr int kScatterRingBytes = 96 * 1024;    // row buffers per CTA
constexpr int kScatterRingMaxRows = 8;

__device__ __forceinline__ void bulk_load_row(uint32_t dst, const void* src, uint32_t bytes, uint32_t bar) {
  asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(dst),
               "l"(src), "r"(bytes), "r"(bar)
               : "memory");
}
__device__ __forceinline__ void bulk_store_row(void* dst, uint32_t src, uint32_t bytes) {
  asm volatile("cp.async.bulk.global.shared::cta.bulk_group [%0], [%1], %2;" ::"l"(dst), "r"(src), "r"(bytes)
               : "memory");
}
__device__ __forceinline__ void bulk_wait_read_le(int n) {  // at most n of this thread's bulk groups still reading
  if (n <= 0) asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
  else if (n == 1) asm volatile("cp.async.bulk.wait_group.read 1;" ::: "memory");
  else if (n == 2) asm volatile("cp.async.bulk.wait_group.read 2;" ::: "memory");
  else if (n == 3) asm volatile("cp.async.bulk.wait_group.read 3;" ::: "memory");
  else if (n == 4) asm volatile("cp.async.bulk.wait_group.read 4;" ::: "memory");
  else if (n == 5) asm volatile("cp.async.bulk.wait_group.read 5;" ::: "memory");
  else if (n == 6) asm volatile("cp.async.bulk.wait_group.read 6;" ::: "memory");
  else asm volatile("cp.async.bulk.wait_group.read 7;" ::: "memory");
}

__global__ void __launch_bounds__(kScatterFusedThreads)
    scatter_fused_kernel(const int64_t* __restrict__ ids, int n, int64_t token, const uint8_t* __restrict__ img,
                         uint8_t* __restrict__ text, int64_t n_img, int64_t row_bytes, int rows_per_cta, int ring,
                         int32_t* status) {
  extern __shared__ __align__(128) uint8_t s_ring[];  // ring x row_bytes
  __shared__ uint32_t s_bits[kScatterFusedMaxIds / 32];
  __shared__ int64_t s_dst[kScatterFusedMaxRows];
  __shared__ int s_warp[kScatterFusedThreads / 32];
  __shared__ __align__(8) uint64_t s_full[kScatterRingMaxRows];
  __shared__ int s_abort;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  constexpr int kWarps = kScatterFusedThreads / 32;
  const int64_t k0 = static_cast<int64_t>(blockIdx.x) * rows_per_cta;
  const int64_t k1 = min(n_img, k0 + rows_per_cta);
  const int n_rows = static_cast<int>(k1 > k0 ? k1 - k0 : 0);
  const uint32_t bytes = static_cast<uint32_t>(row_bytes);
  if (threadIdx.x == 0) {
    for (int i = 0; i < ring; ++i) mbar_init(smem_u32(s_full + i), 1);
    s_abort = 0;
    fence_mbar_init();
  }
  __syncthreads();
  griddep_wait();
  griddep_launch_dependents();
  volatile int* abort_v = &s_abort;
  // the slice's first rows start loading now; the scan below hides their latency
  if (threadIdx.x == 0) {
    for (int i = 0; i < min(ring, n_rows); ++i) {
      mbar_arrive_expect_tx(smem_u32(s_full + i), bytes);
      bulk_load_row(smem_u32(s_ring + static_cast<size_t>(i) * row_bytes), img + (k0 + i) * row_bytes, bytes,
                    smem_u32(s_full + i));
    }
  }
  const int n_words = (n + 31) / 32;
  // (1) bitmask: id c + threadIdx.x -> bit lane of word (c + 32 warp) / 32
#pragma unroll 4
  for (int c = 0; c < n; c += kScatterFusedThreads) {
    const int i = c + threadIdx.x;
    const bool f = i < n && __ldg(ids + i) == token;
    const uint32_t b = __ballot_sync(0xffffffffu, f);
    if (lane == 0 && (c >> 5) + warp < n_words) s_bits[(c >> 5) + warp] = b;
  }
  __syncthreads();
  // (2) thread t owns words [t * wpt, (t + 1) * wpt): contiguous ids, so an
  // exclusive scan of the per-thread counts gives every placeholder's rank
  const int wpt = (n_words + kScatterFusedThreads - 1) / kScatterFusedThreads;
  const int w0 = min(n_words, static_cast<int>(threadIdx.x) * wpt), w1 = min(n_words, w0 + wpt);
  int cnt = 0;
  for (int w = w0; w < w1; ++w) cnt += __popc(s_bits[w]);
  int incl = cnt;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += y;
  }
  if (lane == 31) s_warp[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    int v = lane < kWarps ? s_warp[lane] : 0;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, v, o);
      if (lane >= o) v += y;
    }
    if (lane < kWarps) s_warp[lane] = v;
  }
  __syncthreads();
  const int total = s_warp[kWarps - 1];
  const bool good = total == n_img;
  // (3) text rows of this CTA's image rows
  if (good) {
    int64_t k = (warp > 0 ? s_warp[warp - 1] : 0) + incl - cnt;
    if (k < k1 && k + cnt > k0) {
      for (int w = w0; w < w1; ++w) {
        uint32_t b = s_bits[w];
        while (b) {
          const int bit = __ffs(b) - 1;
          b &= b - 1;
          if (k >= k0 && k < k1) s_dst[k - k0] = static_cast<int64_t>(w) * 32 + bit;
          ++k;
        }
      }
    }
  } else if (blockIdx.x == 0 && threadIdx.x == 0) {
    set_status(status, VLM_ERR_COUNT_MISMATCH);
  }
  __syncthreads();
  if (threadIdx.x != 0) return;
  // (4) thread 0: each buffered row to its text row. The buffer of the row
  // stored `lag` rows earlier takes the row `ring` after it once that store
  // has read it, so `lag` stores and ring - lag loads stay in flight.
  const int lag = ring / 2;
  int issued = min(ring, n_rows), done = 0;
  if (good) {
    for (int r = 0; r < n_rows; ++r) {
      if (!mbar_wait(smem_u32(s_full + r % ring), (r / ring) & 1, abort_v, status)) break;
      if (VLM_DCHECK(s_dst[r] >= 0 && s_dst[r] < n)) {
        bulk_store_row(text + s_dst[r] * row_bytes, smem_u32(s_ring + static_cast<size_t>(r % ring) * row_bytes),
                       bytes);
      }
      bulk_commit();
      done = r + 1;
      const int q = r - lag;  // its store is older than the newest `lag` ones
      if (q >= 0 && q + ring < n_rows) {
        bulk_wait_read_le(lag);
        const int buf = q % ring;
        mbar_arrive_expect_tx(smem_u32(s_full + buf), bytes);
        bulk_load_row(smem_u32(s_ring + static_cast<size_t>(buf) * row_bytes), img + (k0 + q + ring) * row_bytes,
                      bytes, smem_u32(s_full + buf));
        issued = q + ring + 1;
      }
    }
  }
  // loads still in flight must land before the CTA's shared memory goes away
  for (int r = done; r < issued; ++r)
    if (!mbar_wait(smem_u32(s_full + r % ring), (r / ring) & 1, abort_v, status)) break;
  bulk_wait<0>();
}

// ---------------------------------------------------------------------------
// Weight packing (exact copies / reorderings of bf16 values)
// ---------------------------------------------------------------------------
// dst [2F, D]: rows 32j..32j+15 = gate rows 16j.., rows 32j+16..32j+31 = up rows 16j..
__global__ void pack_gate_up_kernel(const uint4* __restrict__ gate, const uint4* __restrict__ up,
                                    uint4* __restrict__ dst, int64_t f, int64_t vec_per_row) {
  const int64_t total = 2 * f * vec_per_row;
  for (int64_t idx = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; idx < total;
       idx += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t row = idx / vec_per_row, j = idx - row * vec_per_row;
    const int64_t grp = row >> 5, within = row & 31;
    const int64_t src_row = grp * 16 + (within & 15);
    dst[idx] = (within < 16 ? gate : up)[src_row * vec_per_row + j];
  }
}

// Per-row E4M3 quantisation, one warp per destination row (see launch_quant_rows).
__global__ void quant_rows_kernel(const __nv_bfloat16* __restrict__ src, const __nv_bfloat16* __restrict__ src2,
                                  int mode, int64_t rows, int64_t cols, uint8_t* __restrict__ dst,
                                  float* __restrict__ colscale, float act_scale) {
  const int lane = threadIdx.x & 31;
  const int64_t warps = static_cast<int64_t>(gridDim.x) * (blockDim.x >> 5);
  for (int64_t r = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5; r < rows; r += warps) {
    const __nv_bfloat16* sr;
    if (mode == 1) {
      const int64_t grp = r >> 5, within = r & 31;
      sr = (within < 16 ? src : src2) + (grp * 16 + (within & 15)) * cols;
    } else {
      sr = src + r * cols;
    }
    float amax = 0.f;
    for (int64_t k = lane; k < cols; k += 32) amax = fmaxf(amax, fabsf(__bfloat162float(sr[k])));
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
    float sc = __fdiv_rn(amax, 448.0f);
    if (!(sc > 0.f)) sc = 1.0f;
    uint8_t* dr = dst + r * cols;
    for (int64_t k = 4 * lane; k < cols; k += 128)
      *reinterpret_cast<uint32_t*>(dr + k) =
          pack_e4m3x4(__fdiv_rn(__bfloat162float(sr[k]), sc), __fdiv_rn(__bfloat162float(sr[k + 1]), sc),
                      __fdiv_rn(__bfloat162float(sr[k + 2]), sc), __fdiv_rn(__bfloat162float(sr[k + 3]), sc));
    if (lane == 0) colscale[r] = __fmul_rn(act_scale, sc);
  }
}

// dst [rows, dst_cols] from src [rows, src_cols], bf16:
//   mode 0 (pad):     dst[r, k] = k < src_cols ? src[r, k] : 0
//   mode 1 (permute): dst[r, slot*D + c] = src[r, c*mm + slot]  (D = src_cols / mm)
__global__ void pack_cols_kernel(const __nv_bfloat16* __restrict__ src, __nv_bfloat16* __restrict__ dst,
                                 int64_t rows, int64_t src_cols, int64_t dst_cols, int mode, int mm) {
  const int64_t total = rows * dst_cols;
  for (int64_t idx = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; idx < total;
       idx += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t r = idx / dst_cols, k = idx - r * dst_cols;
    __nv_bfloat16 v;
    if (mode == 0) {
      v = k < src_cols ? src[r * src_cols + k] : __float2bfloat16(0.f);
    } else {
      const int64_t d = src_cols / mm;
      const int64_t slot = k / d, c = k - slot * d;
      v = src[r * src_cols + c * mm + slot];
    }
    dst[idx] = v;
  }
}

__global__ void f32_to_bf16_kernel(const float* __restrict__ x, __nv_bfloat16* __restrict__ y, int64_t n) {
  griddep_wait();
  griddep_launch_dependents();
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; 2 * i < n;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const float2 v = reinterpret_cast<const float2*>(x)[i];
    reinterpret_cast<uint32_t*>(y)[i] = pack_bf16x2(v.x, v.y);
  }
}

// ---------------------------------------------------------------------------
// Host launchers
// ---------------------------------------------------------------------------
static int grid_for(int64_t work_items, int per_block) {
  const int64_t blocks = (work_items + per_block - 1) / per_block;
  const int64_t cap = static_cast<int64_t>(num_sms()) * 16;
  return static_cast<int>(blocks < 1 ? 1 : (blocks > cap ? cap : blocks));
}

int launch_setup(const ImageChunk& chunk, ImgInfo* info, int32_t* cu, int32_t* qt, int32_t* i2c, int32_t* pos,
                 int n_images, cudaStream_t s) {
  const int64_t tokens = chunk.tok_off[chunk.count] - chunk.tok_off[0];
  const int grid = grid_for(tokens > chunk.count ? tokens : chunk.count, 256);
  launch_begin(KC_SETUP, s);
  const cudaError_t e =
      launch_pdl(setup_kernel, dim3(grid), dim3(256), 0, s, chunk, info, cu, qt, i2c, pos, n_images);
  launch_end(KC_SETUP, s);
  return e == cudaSuccess ? VLM_OK : VLM_ERR_CUDA;
}

int launch_rope_table(float theta, int head_dim, int max_pos, float2* tab, cudaStream_t s) {
  const int n = max_pos * head_dim / 2;
  launch_begin(KC_SETUP, s);
  const cudaError_t e = launch_pdl(rope_table_kernel, dim3((n + 255) / 256), dim3(256), 0, s, theta, head_dim, max_pos, tab);
  launch_end(KC_SETUP, s);
  return e == cudaSuccess ? VLM_OK : VLM_ERR_CUDA;
}

int launch_im2col(const float* pix, const ImgInfo* info, const int32_t* cu, const int32_t* i2c, int i2c_items,
                  int n_images, int64_t T, int p, int kp, int normalize, __nv_bfloat16* out, cudaStream_t s) {
  launch_begin(KC_IM2COL, s);
  cudaError_t e;
  // one item per CTA up to 16 CTAs per SM, then a grid-stride loop
  const int tgrid = i2c_items < num_sms() * 16 ? (i2c_items > 0 ? i2c_items : 1) : num_sms() * 16;
  if (p == 14 && i2c != nullptr)
    e = launch_pdl(im2col_tiled_kernel<14>, dim3(tgrid), dim3(kI2cThreads), 0, s, pix, info, i2c, n_images,
                   i2c_items, kp, normalize, out);
  else if (p == 16 && i2c != nullptr)
    e = launch_pdl(im2col_tiled_kernel<16>, dim3(tgrid), dim3(kI2cThreads), 0, s, pix, info, i2c, n_images,
                   i2c_items, kp, normalize, out);
  else
    e = launch_pdl(im2col_kernel, dim3(grid_for(T * 32, 256)), dim3(256), 0, s, pix, info, cu, n_images, T, p, kp,
                   normalize, out);
  launch_end(KC_IM2COL, s);
  return e == cudaSuccess ? VLM_OK : VLM_ERR_CUDA;
}

int launch_rmsnorm(float* x, const float* g0, const float* g1, void* out, int64_t rows, int width, float eps,
                   cudaStream_t s, float f8_scale) {
  if (width % 128 || width > 2048 || width <= 0) return VLM_ERR_UNSUPPORTED;
  const int grid = grid_for(rows * 32, 256);
  launch_begin(KC_NORM, s);
  cudaError_t e = cudaErrorInvalidValue;
  const bool f8 = f8_scale > 0.f;
  switch (width / 128) {
#define VLM_NORM_CASE(nv)                                                                                       \
  case nv:                                                                                                    \
    e = f8 ? launch_pdl(rmsnorm_kernel<nv, 1>, dim3(grid), dim3(256), 0, s, x, g0, g1, out, rows, eps, f8_scale, \
                        nullptr)                                                                          \
           : launch_pdl(rmsnorm_kernel<nv, 0>, dim3(grid), dim3(256), 0, s, x, g0, g1, out, rows, eps, 0.f,  \
                        nullptr);                                                                         \
    break;
    VLM_NORM_CASE(1) VLM_NORM_CASE(2) VLM_NORM_CASE(3) VLM_NORM_CASE(4) VLM_NORM_CASE(5)
    VLM_NORM_CASE(6) VLM_NORM_CASE(7) VLM_NORM_CASE(8) VLM_NORM_CASE(9) VLM_NORM_CASE(10)
    VLM_NORM_CASE(11) VLM_NORM_CASE(12) VLM_NORM_CASE(13) VLM_NORM_CASE(14) VLM_NORM_CASE(15)
    VLM_NORM_CASE(16)
#undef VLM_NORM_CASE
    default: break;
  }
  launch_end(KC_NORM, s);
  return e == cudaSuccess ? VLM_OK : VLM_ERR_CUDA;
}

// RMSNorm to NVFP4 for widths that are a multiple of 512: lane l holds the 16
// consecutive values of blocks l + 32 b (b < NB), so each block is quantised
// by one lane (no shuffles, no repeated scale arithmetic across lanes) and its
// 8 code bytes are one store. One warp per row; loads are 64 contiguous bytes
// per lane.
template <int NB>
__global__ void rmsnorm_nvfp4_kernel(float* __restrict__ x, const float* __restrict__ g0,
                                     const float* __restrict__ g1, uint8_t* __restrict__ q,
                                     uint8_t* __restrict__ sf, int64_t rows, float eps, float sg) {
  griddep_wait();
  griddep_launch_dependents();
  constexpr int width = NB * 512;
  const int lane = threadIdx.x & 31;
  const float six_sg = 6.0f * sg;
  const int64_t warps = static_cast<int64_t>(gridDim.x) * (blockDim.x >> 5);
  for (int64_t row = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5; row < rows;
       row += warps) {
    float4* xr = reinterpret_cast<float4*>(x + row * width);
    float4 v[NB][4];
    float ss = 0.f;
#pragma unroll
    for (int b = 0; b < NB; ++b)
#pragma unroll
      for (int t = 0; t < 4; ++t) {
        v[b][t] = xr[4 * (lane + 32 * b) + t];
        ss += v[b][t].x * v[b][t].x + v[b][t].y * v[b][t].y + v[b][t].z * v[b][t].z + v[b][t].w * v[b][t].w;
      }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
    float rs = rsqrtf(ss / width + eps);
    if (g0 != nullptr) {
      const float4* gr = reinterpret_cast<const float4*>(g0);
      ss = 0.f;
#pragma unroll
      for (int b = 0; b < NB; ++b)
#pragma unroll
        for (int t = 0; t < 4; ++t) {
          const float4 g = __ldg(gr + 4 * (lane + 32 * b) + t);
          float4& u = v[b][t];
          u.x *= rs * g.x; u.y *= rs * g.y; u.z *= rs * g.z; u.w *= rs * g.w;
          xr[4 * (lane + 32 * b) + t] = u;
          ss += u.x * u.x + u.y * u.y + u.z * u.z + u.w * u.w;
        }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
      rs = rsqrtf(ss / width + eps);
    }
    const float4* gr = reinterpret_cast<const float4*>(g1);
#pragma unroll
    for (int b = 0; b < NB; ++b) {
      float y[16], amax = 0.0f;
#pragma unroll
      for (int t = 0; t < 4; ++t) {
        const float4 g = __ldg(gr + 4 * (lane + 32 * b) + t);
        y[4 * t] = v[b][t].x * rs * g.x;
        y[4 * t + 1] = v[b][t].y * rs * g.y;
        y[4 * t + 2] = v[b][t].z * rs * g.z;
        y[4 * t + 3] = v[b][t].w * rs * g.w;
      }
#pragma unroll
      for (int k = 0; k < 16; ++k) amax = fmaxf(amax, fabsf(y[k]));
      uint2 codes;
      const uint32_t sb = nvfp4_quant16(y, amax, sg, six_sg, codes);
      const int blk = lane + 32 * b;
      *reinterpret_cast<uint2*>(q + row * (width / 2) + 8 * blk) = codes;
      sf[nvfp4_sf_offset(row, blk, width)] = static_cast<uint8_t>(sb);
    }
  }
}

int launch_rmsnorm_nvfp4(float* x, const float* g0, const float* g1, uint8_t* q, uint8_t* sf, int64_t rows,
                         int width, float eps, float s_global, cudaStream_t s) {
  if (width % 512 == 0 && width <= 2048 && width > 0) {
    if (q == nullptr || sf == nullptr || !(s_global > 0.f)) return VLM_ERR_INVALID_ARG;
    if (reinterpret_cast<uintptr_t>(q) & 7) return VLM_ERR_INVALID_ARG;
    const int grid = grid_for(rows * 32, 256);
    launch_begin(KC_NORM, s);
    cudaError_t e = cudaErrorInvalidValue;
    switch (width / 512) {
      case 1: e = launch_pdl(rmsnorm_nvfp4_kernel<1>, dim3(grid), dim3(256), 0, s, x, g0, g1, q, sf, rows, eps, s_global); break;
      case 2: e = launch_pdl(rmsnorm_nvfp4_kernel<2>, dim3(grid), dim3(256), 0, s, x, g0, g1, q, sf, rows, eps, s_global); break;
      case 3: e = launch_pdl(rmsnorm_nvfp4_kernel<3>, dim3(grid), dim3(256), 0, s, x, g0, g1, q, sf, rows, eps, s_global); break;
      case 4: e = launch_pdl(rmsnorm_nvfp4_kernel<4>, dim3(grid), dim3(256), 0, s, x, g0, g1, q, sf, rows, eps, s_global); break;
      default: break;
    }
    launch_end(KC_NORM, s);
    return e == cudaSuccess ? VLM_OK : VLM_ERR_CUDA;
  }
  if (width % 128 || width > 2048 || width <= 0) return VLM_ERR_UNSUPPORTED;
  if (q == nullptr || sf == nullptr || !(s_global > 0.f)) return VLM_ERR_INVALID_ARG;
  const int grid = grid_for(rows * 32, 256);
  launch_begin(KC_NORM, s);
  cudaError_t e = cudaErrorInvalidValue;
  switch (width / 128) {
#define VLM_NORM_CASE(nv)                                                                                      \
  case nv:                                                                                                   \
    e = launch_pdl(rmsnorm_kernel<nv, 2>, dim3(grid), dim3(256), 0, s, x, g0, g1, static_cast<void*>(q), rows, \
                   eps, s_global, sf);                                                                       \
    break;
    VLM_NORM_CASE(1) VLM_NORM_CASE(2) VLM_NORM_CASE(3) VLM_NORM_CASE(4) VLM_NORM_CASE(5)
    VLM_NORM_CASE(6) VLM_NORM_CASE(7) VLM_NORM_CASE(8) VLM_NORM_CASE(9) VLM_NORM_CASE(10)
    VLM_NORM_CASE(11) VLM_NORM_CASE(12) VLM_NORM_CASE(13) VLM_NORM_CASE(14) VLM_NORM_CASE(15)
    VLM_NORM_CASE(16)
#undef VLM_NORM_CASE
    default: break;
  }
  launch_end(KC_NORM, s);
  return e == cudaSuccess ? VLM_OK : VLM_ERR_CUDA;
}

// ---------------------------------------------------------------------------
// Projector RMSNorm + m x m merge gather (bf16 in/out). Patch (r, c) of image
// b goes to merged token m_off_b + (r/m)(w/m) + c/m, slot (r%m)*m + c%m, i.e.
// z[token, slot*D + ch] (patch-major). A CTA takes kMergeRows consecutive
// patches: one bulk copy brings their rows into shared memory; meanwhile each
// warp finds its rows' destinations and holds the gains in registers; then it
// normalises each row in place and one lane bulk-stores the row to its slot.
// The bulk engine keeps many bytes in flight at few registers per thread.
// g == nullptr: gather only (the merge-first reading normalises later).
// ---------------------------------------------------------------------------
constexpr int kMergeThreads = 256;
constexpr int kMergeSmem = 64 * 1024;

template <int NV>
__global__ void __launch_bounds__(kMergeThreads, 3) merge_norm_kernel(const __nv_bfloat16* __restrict__ x,
                                                                   const float* __restrict__ g,
                                                                   const ImgInfo* __restrict__ info,
                                                                   const int32_t* __restrict__ cu, int n_images,
                                                                   int64_t T, int m, float eps, int rows_per_cta,
                                                                   __nv_bfloat16* __restrict__ z, int32_t* status) {
  extern __shared__ __align__(128) uint8_t s_rows[];  // rows_per_cta x width bf16
  __shared__ __align__(8) uint64_t s_full;
  __shared__ int s_abort;
  constexpr int width = NV * 128;
  constexpr uint32_t kRowBytes = width * 2;
  constexpr int kWarps = kMergeThreads / 32;
  constexpr int kMaxRowsPerWarp = kMergeSmem / kRowBytes / kWarps > 0 ? kMergeSmem / kRowBytes / kWarps : 1;
  // 16-byte accesses (8 values per lane) when the row holds a whole number of
  // 256-value warp chunks, 8-byte ones (4 values) otherwise
  constexpr int VE = (NV % 2 == 0) ? 8 : 4, NL = width / (32 * VE);
  using Vec = typename std::conditional<VE == 8, uint4, uint2>::type;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int64_t t0 = static_cast<int64_t>(blockIdx.x) * rows_per_cta;
  const int nrows = static_cast<int>(min(static_cast<int64_t>(rows_per_cta), T - t0));
  if (threadIdx.x == 0) {
    mbar_init(smem_u32(&s_full), 1);
    s_abort = 0;
    fence_mbar_init();
  }
  __syncthreads();
  griddep_wait();
  griddep_launch_dependents();
  if (threadIdx.x == 0) {
    mbar_arrive_expect_tx(smem_u32(&s_full), nrows * kRowBytes);
    asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
                     smem_u32(s_rows)),
                 "l"(x + t0 * width), "r"(nrows * kRowBytes), "r"(smem_u32(&s_full))
                 : "memory");
  }
  // while the rows arrive: their destinations and the gains
  int64_t dst[kMaxRowsPerWarp];
#pragma unroll
  for (int i = 0; i < kMaxRowsPerWarp; ++i) {
    const int lr = warp + kWarps * i;
    dst[i] = -1;
    if (lr < nrows) {
      const int t = static_cast<int>(t0 + lr);
      const int b = find_block(cu, n_images, t);
      const ImgInfo in = info[b];
      const int local = t - in.tok_off;
      const int r = local / in.w, c = local % in.w;
      const int64_t mt = in.m_off + (r / m) * (in.w / m) + c / m;
      if (VLM_DCHECK(local >= 0 && local < in.h * in.w && (mt + 1) * m * m <= T))
        dst[i] = (mt * m * m + (r % m) * m + c % m) * width;
    }
  }
  float gv[NL][VE];
#pragma unroll
  for (int j = 0; j < NL; ++j)
#pragma unroll
    for (int q = 0; q < VE / 4; ++q) {
      const float4 gg = g != nullptr ? __ldg(reinterpret_cast<const float4*>(g) + (lane + 32 * j) * (VE / 4) + q)
                                     : make_float4(1.f, 1.f, 1.f, 1.f);
      gv[j][4 * q] = gg.x;
      gv[j][4 * q + 1] = gg.y;
      gv[j][4 * q + 2] = gg.z;
      gv[j][4 * q + 3] = gg.w;
    }
  const bool ok = mbar_wait(smem_u32(&s_full), 0, &s_abort, status);
  if (ok) {
#pragma unroll
    for (int i = 0; i < kMaxRowsPerWarp; ++i) {
      if (dst[i] < 0) break;
      Vec* row = reinterpret_cast<Vec*>(s_rows + static_cast<size_t>(warp + kWarps * i) * kRowBytes);
      Vec u[NL];
      float ss = 0.f;
#pragma unroll
      for (int j = 0; j < NL; ++j) {
        u[j] = row[lane + 32 * j];
        const __nv_bfloat162* h2 = reinterpret_cast<const __nv_bfloat162*>(&u[j]);
#pragma unroll
        for (int e = 0; e < VE / 2; ++e) {
          const float a0 = __low2float(h2[e]), a1 = __high2float(h2[e]);
          ss += a0 * a0 + a1 * a1;
        }
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
      const float rs = g != nullptr ? rsqrtf(ss / width + eps) : 1.0f;
#pragma unroll
      for (int j = 0; j < NL; ++j) {
        const __nv_bfloat162* h2 = reinterpret_cast<const __nv_bfloat162*>(&u[j]);
        Vec o;
        uint32_t* ow = reinterpret_cast<uint32_t*>(&o);
#pragma unroll
        for (int e = 0; e < VE / 2; ++e)
          ow[e] = pack_bf16x2(__low2float(h2[e]) * rs * gv[j][2 * e], __high2float(h2[e]) * rs * gv[j][2 * e + 1]);
        row[lane + 32 * j] = o;
      }
      fence_proxy_async_smem();  // the row's new values are visible to the bulk copy below
      __syncwarp();
      if (lane == 0) {
        asm volatile("cp.async.bulk.global.shared::cta.bulk_group [%0], [%1], %2;" ::"l"(z + dst[i]),
                     "r"(smem_u32(row)), "r"(kRowBytes)
                     : "memory");
        asm volatile("cp.async.bulk.commit_group;" ::: "memory");
      }
    }
  }
  if (lane == 0) asm volatile("cp.async.bulk.wait_group 0;" ::: "memory");  // stores done before the CTA ends
}

int launch_merge_norm(const __nv_bfloat16* x, const float* g, const ImgInfo* info, const int32_t* cu,
                      int n_images, int64_t T, int width, int m, float eps, __nv_bfloat16* z, int32_t* status,
                      cudaStream_t s) {
  if (width % 128 || width > 2048 || width <= 0) return VLM_ERR_UNSUPPORTED;
  if (T <= 0) return VLM_OK;
  const int row_bytes = width * 2;
  const int warps = kMergeThreads / 32;
  // rows per CTA: as many as fit the shared buffer, a whole number per warp
  const int per_warp = std::max(1, kMergeSmem / row_bytes / warps);
  const int rows = per_warp * warps;
  const int64_t grid = (T + rows - 1) / rows;
  const size_t smem = static_cast<size_t>(rows) * row_bytes;
  static bool attr_done[64][17] = {};
  int dev = 0;
  cudaGetDevice(&dev);
  launch_begin(KC_MERGE, s);
  cudaError_t e = cudaErrorInvalidValue;
  switch (width / 128) {
#define VLM_MERGE_CASE(nv)                                                                                         \
  case nv:                                                                                                         \
    if (dev < 64 && !attr_done[dev][nv]) {                                                                         \
      if (cudaFuncSetAttribute(merge_norm_kernel<nv>, cudaFuncAttributeMaxDynamicSharedMemorySize, kMergeSmem) != \
          cudaSuccess)                                                                                             \
        break;                                                                                                     \
      attr_done[dev][nv] = true;                                                                                   \
    }                                                                                                              \
    e = launch_pdl(merge_norm_kernel<nv>, dim3(static_cast<unsigned>(grid)), dim3(kMergeThreads), smem, s, x, g,  \
                   info, cu, n_images, T, m, eps, rows, z, status);                                                \
    break;
    VLM_MERGE_CASE(1) VLM_MERGE_CASE(2) VLM_MERGE_CASE(3) VLM_MERGE_CASE(4) VLM_MERGE_CASE(5)
    VLM_MERGE_CASE(6) VLM_MERGE_CASE(7) VLM_MERGE_CASE(8) VLM_MERGE_CASE(9) VLM_MERGE_CASE(10)
    VLM_MERGE_CASE(11) VLM_MERGE_CASE(12) VLM_MERGE_CASE(13) VLM_MERGE_CASE(14) VLM_MERGE_CASE(15)
    VLM_MERGE_CASE(16)
#undef VLM_MERGE_CASE
    default: break;
  }
  launch_end(KC_MERGE, s);
  return e == cudaSuccess ? VLM_OK : VLM_ERR_CUDA;
}

int launch_rmsnorm_bf16(const __nv_bfloat16* x, const float* g, __nv_bfloat16* out, int64_t rows, int width,
                        float eps, cudaStream_t s) {
  if (width % 128 || width > 2048 || width <= 0) return VLM_ERR_UNSUPPORTED;
  const int grid = grid_for(rows * 32, 256);
  launch_begin(KC_MERGE, s);
  cudaError_t e = cudaErrorInvalidValue;
  switch (width / 128) {
#define VLM_NORM16_CASE(nv) \
  case nv: e = launch_pdl(rmsnorm_bf16_kernel<nv>, dim3(grid), dim3(256), 0, s, x, g, out, rows, eps); break;
    VLM_NORM16_CASE(1) VLM_NORM16_CASE(2) VLM_NORM16_CASE(3) VLM_NORM16_CASE(4) VLM_NORM16_CASE(5)
    VLM_NORM16_CASE(6) VLM_NORM16_CASE(7) VLM_NORM16_CASE(8) VLM_NORM16_CASE(9) VLM_NORM16_CASE(10)
    VLM_NORM16_CASE(11) VLM_NORM16_CASE(12) VLM_NORM16_CASE(13) VLM_NORM16_CASE(14) VLM_NORM16_CASE(15)
    VLM_NORM16_CASE(16)
#undef VLM_NORM16_CASE
    default: break;
  }
  launch_end(KC_MERGE, s);
  return e == cudaSuccess ? VLM_OK : VLM_ERR_CUDA;
}

int launch_scatter(const int64_t* ids, int64_t n, int64_t token, const void* img, int64_t n_img,
                   void* text, int64_t row_bytes, ScatterWs ws, int32_t* status, cudaStream_t s) {
  const int ring = static_cast<int>(row_bytes > 0 ? std::min<int64_t>(kScatterRingMaxRows, kScatterRingBytes / row_bytes) : 0);
  if (n <= kScatterFusedMaxIds && ring >= 2) {
    // one launch; the workspace is not used
    const int64_t slots = 2LL * num_sms();
    int64_t rows = n_img > n ? 1 : (n_img + slots - 1) / slots;  // more rows than ids can only mismatch
    rows = rows < 1 ? 1 : (rows > kScatterFusedMaxRows ? kScatterFusedMaxRows : rows);
    const int64_t grid = n_img > n ? 1 : (n_img + rows - 1) / rows;
    const size_t smem = static_cast<size_t>(ring) * static_cast<size_t>(row_bytes);
    static bool attr_done[64] = {};
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev < 64 && !attr_done[dev]) {
      if (cudaFuncSetAttribute(scatter_fused_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kScatterRingBytes) !=
          cudaSuccess)
        return VLM_ERR_CUDA;
      attr_done[dev] = true;
    }
    launch_begin(KC_SCATTER, s);
    const cudaError_t e = launch_pdl(scatter_fused_kernel, dim3(static_cast<unsigned>(grid < 1 ? 1 : grid)),
                                     dim3(kScatterFusedThreads), smem, s, ids, static_cast<int>(n), token,
                                     static_cast<const uint8_t*>(img), static_cast<uint8_t*>(text), n_img, row_bytes,
                                     static_cast<int>(rows), ring, status);
    launch_end(KC_SCATTER, s);
    return e == cudaSuccess ? VLM_OK : VLM_ERR_CUDA;
  }
  const int64_t n_chunks = (n + 255) / 256;
  launch_begin(KC_SCATTER, s);
  const dim3 chunks(static_cast<unsigned>(n_chunks));
  cudaError_t e = launch_pdl(scatter_count_kernel, chunks, dim3(256), 0, s, ids, n, token, ws.chunk_count);
  if (e == cudaSuccess)
    e = launch_pdl(scatter_scan_kernel, dim3(1), dim3(1024), 0, s, ws.chunk_count, n_chunks, n_img, ws.chunk_base,
                   ws.ok_flag, status);
  if (e == cudaSuccess)
    e = launch_pdl(scatter_positions_kernel, chunks, dim3(256), 0, s, ids, n, token, ws.chunk_base, ws.ok_flag,
                   ws.dst_rows, n_img);
  const int64_t vec = row_bytes / 16;
  if (e == cudaSuccess)
    e = launch_pdl(scatter_copy_kernel, dim3(grid_for(n_img * 32, 256)), dim3(256), 0, s,
                   static_cast<const uint4*>(img), static_cast<uint4*>(text), ws.dst_rows, ws.ok_flag, n_img, vec, n);
  launch_end(KC_SCATTER, s);
  note_extra_launches(3);
  return e == cudaSuccess ? VLM_OK : VLM_ERR_CUDA;
}

// The placeholder positions of up to kScatterRowsOneCta ids in one CTA: each
// thread counts a contiguous run of ids, one block scan ranks the runs, and
// the runs' placeholders are written in order once the total is known to
// equal n_img (otherwise ok_flag = 0 and nothing is written). A thread's run
// is read one id after another, so longer id sequences go to the count, scan
// and positions kernels, which spread them over many CTAs (16,384 ids: 33 us
// in one CTA).
constexpr int kScatterRowsOneCta = 4096;
__global__ void __launch_bounds__(1024) scatter_rows_one_cta_kernel(const int64_t* __restrict__ ids, int n,
                                                                      int64_t token, int64_t n_img,
                                                                      int64_t* __restrict__ dst_rows,
                                                                      int32_t* __restrict__ ok_flag, int32_t* status) {
  griddep_wait();
  griddep_launch_dependents();
  __shared__ int warp_sums[32];
  const int per = (n + 1023) / 1024;
  const int beg = min(n, static_cast<int>(threadIdx.x) * per), end = min(n, beg + per);
  int cnt = 0;
  for (int i = beg; i < end; ++i) cnt += __ldg(ids + i) == token ? 1 : 0;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int incl = cnt;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += y;
  }
  if (lane == 31) warp_sums[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    int w = warp_sums[lane];
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, w, o);
      if (lane >= o) w += y;
    }
    warp_sums[lane] = w;  // inclusive over warps
  }
  __syncthreads();
  const int total = warp_sums[31];
  if (total != n_img) {
    if (threadIdx.x == 0) {
      *ok_flag = 0;
      set_status(status, VLM_ERR_COUNT_MISMATCH);
    }
    return;
  }
  int64_t k = (warp > 0 ? warp_sums[warp - 1] : 0) + incl - cnt;
  for (int i = beg; i < end; ++i)
    if (__ldg(ids + i) == token && VLM_DCHECK(k >= 0 && k < n_img)) dst_rows[k++] = i;
  if (threadIdx.x == 0) *ok_flag = 1;
}

int launch_scatter_rows(const int64_t* ids, int64_t n, int64_t token, int64_t n_img, const ScatterWs& ws,
                        int32_t* status, cudaStream_t s) {
  if (n <= 0) return VLM_ERR_BAD_SHAPE;
  if (n <= kScatterRowsOneCta) {
    launch_begin(KC_SCATTER, s);
    const cudaError_t e = launch_pdl(scatter_rows_one_cta_kernel, dim3(1), dim3(1024), 0, s, ids, static_cast<int>(n),
                                     token, n_img, ws.dst_rows, ws.ok_flag, status);
    launch_end(KC_SCATTER, s);
    return e == cudaSuccess ? VLM_OK : VLM_ERR_CUDA;
  }
  const int64_t n_chunks = (n + 255) / 256;
  const dim3 chunks(static_cast<unsigned>(n_chunks));
  launch_begin(KC_SCATTER, s);
  cudaError_t e = launch_pdl(scatter_count_kernel, chunks, dim3(256), 0, s, ids, n, token, ws.chunk_count);
  if (e == cudaSuccess)
    e = launch_pdl(scatter_scan_kernel, dim3(1), dim3(1024), 0, s, ws.chunk_count, n_chunks, n_img, ws.chunk_base,
                   ws.ok_flag, status);
  if (e == cudaSuccess)
    e = launch_pdl(scatter_positions_kernel, chunks, dim3(256), 0, s, ids, n, token, ws.chunk_base, ws.ok_flag,
                   ws.dst_rows, n_img);
  launch_end(KC_SCATTER, s);
  note_extra_launches(2);
  return e == cudaSuccess ? VLM_OK : VLM_ERR_CUDA;
}

// The scatter's first two kernels, reused by the placeholder expansion (the
// caller brackets them with its own launch_begin / launch_end).
int launch_marker_count(const int64_t* ids, int64_t n, int64_t token, int32_t* chunk_count, cudaStream_t s) {
  const dim3 chunks(static_cast<unsigned>((n + 255) / 256));
  return launch_pdl(scatter_count_kernel, chunks, dim3(256), 0, s, ids, n, token, chunk_count) == cudaSuccess
             ? VLM_OK : VLM_ERR_CUDA;
}

int launch_marker_scan(const int32_t* chunk_count, int64_t n_chunks, int64_t expected, int64_t* chunk_base,
                       int32_t* ok_flag, int32_t* status, cudaStream_t s) {
  return launch_pdl(scatter_scan_kernel, dim3(1), dim3(1024), 0, s, chunk_count, n_chunks, expected, chunk_base,
                    ok_flag, status) == cudaSuccess ? VLM_OK : VLM_ERR_CUDA;
}

int launch_quant_rows(const void* src, const void* src2, int mode, int64_t rows, int64_t cols, void* dst,
                      float* colscale, float act_scale, cudaStream_t s) {
  if (cols % 128 != 0 || rows <= 0) return VLM_ERR_UNSUPPORTED;
  launch_begin(KC_PACK, s);
  quant_rows_kernel<<<grid_for(rows * 32, 256), 256, 0, s>>>(
      static_cast<const __nv_bfloat16*>(src), static_cast<const __nv_bfloat16*>(src2), mode, rows, cols,
      static_cast<uint8_t*>(dst), colscale, act_scale);
  launch_end(KC_PACK, s);
  return cudaGetLastError() == cudaSuccess ? VLM_OK : VLM_ERR_CUDA;
}

int launch_pack_gate_up(const void* gate, const void* up, void* dst, int64_t f, int64_t d, cudaStream_t s) {
  const int64_t vec = d * 2 / 16;
  launch_begin(KC_PACK, s);
  pack_gate_up_kernel<<<grid_for(2 * f * vec, 256), 256, 0, s>>>(
      static_cast<const uint4*>(gate), static_cast<const uint4*>(up), static_cast<uint4*>(dst), f, vec);
  launch_end(KC_PACK, s);
  return cudaGetLastError() == cudaSuccess ? VLM_OK : VLM_ERR_CUDA;
}

int launch_pack_cols(const void* src, void* dst, int64_t rows, int64_t src_cols, int64_t dst_cols, int mode,
                     int mm, cudaStream_t s) {
  launch_begin(KC_PACK, s);
  pack_cols_kernel<<<grid_for(rows * dst_cols, 256), 256, 0, s>>>(
      static_cast<const __nv_bfloat16*>(src), static_cast<__nv_bfloat16*>(dst), rows, src_cols, dst_cols,
      mode, mm);
  launch_end(KC_PACK, s);
  return cudaGetLastError() == cudaSuccess ? VLM_OK : VLM_ERR_CUDA;
}

int launch_f32_to_bf16(const float* x, __nv_bfloat16* y, int64_t n, cudaStream_t s) {
  launch_begin(KC_NORM, s);
  const cudaError_t e = launch_pdl(f32_to_bf16_kernel, dim3(grid_for(n / 2, 256)), dim3(256), 0, s, x, y, n);
  launch_end(KC_NORM, s);
  return e == cudaSuccess ? VLM_OK : VLM_ERR_CUDA;
}

}  // namespace vlm

namespace vlm {

// ---------------------------------------------------------------------------
// Self-test of the bounded barrier wait: one thread waits on an mbarrier that
// nothing arrives on, with a budget of `budget_cycles`, exactly as the GEMM and
// attention roles wait on theirs; the wait must give up, record
// VLM_ERR_TIMEOUT in *status and let the kernel return normally.
// ---------------------------------------------------------------------------
// Debug builds only: threads i < 2n would write buf[i] behind the check i < n,
// so the check fails for every i >= n, records its code and skips the write.
// (Release builds never launch it: the entry point refuses first.)
__global__ void debug_selftest_kernel(int32_t* buf, int n) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i < 2 * n && VLM_DCHECK(i < n)) buf[i] = i + 1;
}

int launch_debug_selftest(int32_t* buf, int n, cudaStream_t s) {
#ifdef VLM_DEBUG
  if (buf == nullptr || n <= 0 || n > (1 << 20)) return VLM_ERR_INVALID_ARG;
  debug_selftest_kernel<<<(2 * n + 255) / 256, 256, 0, s>>>(buf, n);
  return cudaGetLastError() == cudaSuccess ? VLM_OK : VLM_ERR_CUDA;
#else
  (void)buf;
  (void)n;
  (void)s;
  return VLM_ERR_UNSUPPORTED;
#endif
}

__global__ void wait_timeout_selftest_kernel(long long budget_cycles, int32_t* status) {
  __shared__ __align__(8) uint64_t bar;
  if (threadIdx.x != 0) return;
  mbar_init(smem_u32(&bar), 1);
  fence_mbar_init();
  const uint32_t b = smem_u32(&bar);
  // the phase of parity 0 never completes: nobody arrives
  if (mbar_try_wait(b, 0)) return;
  const long long t0 = clock64();
  for (uint32_t i = 1;; ++i) {
    if (mbar_try_wait(b, 0)) return;
    if ((i & 255u) == 0 && clock64() - t0 > budget_cycles) {
      set_status(status, VLM_ERR_TIMEOUT);
      return;
    }
  }
}

int launch_wait_timeout_selftest(long long budget_cycles, int32_t* status, cudaStream_t s) {
  launch_begin(KC_SETUP, s);
  wait_timeout_selftest_kernel<<<1, 32, 0, s>>>(budget_cycles, status);
  launch_end(KC_SETUP, s);
  return cudaGetLastError() == cudaSuccess ? VLM_OK : VLM_ERR_CUDA;
}

}  // namespace vlm
