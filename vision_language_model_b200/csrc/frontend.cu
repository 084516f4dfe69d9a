// The steps just before and just after the path: the processor's resize onto
// the patch grid (with Pixtral's 1024-pixel tiling folded into the same pass)
// and the expansion of one image marker per image into its run of
// image_token_id placeholders.
#include "kernels.cuh"

#define VLM_DEBUG_FILE_ID 2

namespace vlm {

VLM_DEBUG_UNIT(debug_word_frontend)

// ---------------------------------------------------------------------------
// Bilinear resize, u8 RGB HWC -> fp32 CHW in [0, 1], optionally tiled.
//
// Output pixel (y, x) of an out_h x out_w image samples the source at
// ((2y+1) H - out_h) / (2 out_h) (and likewise for x): half-pixel centres,
// clamped to the image, interpolating the four neighbours. The integer part
// q and the remainder r of that coordinate are exact integers (one division
// per 4 output pixels, then exact stepping by the precomputed quotient and
// remainder of 2W / 2out_w), so the neighbour choice never depends on float
// rounding; the fraction is r * (1 / 2out_w).
//
// Work unit: one column segment (<= 512 pixels, a multiple of 4) of one
// output row. A unit stages the byte span of its two source rows that its
// taps touch into shared memory with 16-byte loads, then each thread blends 4
// consecutive pixels and writes one float4 per channel plane (out_w % 4 == 0
// and tile % 4 == 0, so a float4 never straddles a tile edge).
// Source bytes become floats as (0x4B000000 | byte) - 2^23 (exact for 0..255),
// avoiding integer-to-float conversions.
// ---------------------------------------------------------------------------
__device__ __forceinline__ float byte_as_float(uint32_t v) {
  return __uint_as_float(0x4B000000u | v) - 8388608.f;
}

struct Tap {
  int i0, i1;
  float f;
};

// Floor quotient and remainder of ((2o+1) n_in - n_out) / (2 n_out); q = -1
// when the sample lies before the first pixel centre.
template <typename Idx>
__device__ __forceinline__ void coord_qr(int o, int n_in, int n_out, int& q, int& r) {
  const Idx den = 2 * static_cast<Idx>(n_out);
  const Idx num = (2 * static_cast<Idx>(o) + 1) * n_in - n_out;
  if (num >= 0) {
    const Idx qq = num / den;
    q = static_cast<int>(qq);
    r = static_cast<int>(num - qq * den);
  } else {  // num > -den always
    q = -1;
    r = static_cast<int>(num + den);
  }
}

__device__ __forceinline__ Tap make_tap(int q, int r, int n_in, float inv_den) {
  Tap t;
  if (q < 0) {
    t.i0 = 0;
    t.f = 0.f;
  } else if (q >= n_in - 1) {
    t.i0 = n_in - 1;
    t.f = 0.f;
  } else {
    t.i0 = q;
    t.f = byte_as_float(static_cast<uint32_t>(r)) * inv_den;  // r < 2^22: exact conversion
  }
  t.i1 = min(t.i0 + 1, n_in - 1);
  return t;
}

// Copies `n` source bytes starting at byte offset `off` into smem, from the
// 16-byte boundary at or below it; returns the smem index of byte `off`.
// Whole 16-byte chunks inside the source buffer are vector loads; a ragged
// last chunk is read byte by byte.
__device__ __forceinline__ int stage_bytes(const uint8_t* __restrict__ src, int64_t src_bytes, int64_t off, int n,
                                           uint8_t* smem) {
  const int64_t a0 = off & ~15LL;
  const int shift = static_cast<int>(off - a0);
  const int chunks = (shift + n + 15) >> 4;
  for (int k = threadIdx.x; k < chunks; k += blockDim.x) {
    const int64_t at = a0 + 16LL * k;
    if (at + 16 <= src_bytes) {
      *reinterpret_cast<uint4*>(smem + 16 * k) = __ldg(reinterpret_cast<const uint4*>(src + at));
    } else {
      for (int j = 0; j < 16; ++j) smem[16 * k + j] = at + j < src_bytes ? __ldg(src + at + j) : 0;
    }
  }
  return shift;
}

// kStaged: taps read the staged row spans (each at most ch.stage_bytes);
// otherwise every tap is a read-only global byte load. Idx: integer type of
// the coordinate numerators ((2o+1) n_in must fit).
template <bool kStaged, typename Idx>
__global__ void __launch_bounds__(128) resize_tile_kernel(const uint8_t* __restrict__ src, int64_t src_bytes,
                                                          ResizeChunk ch, float* __restrict__ dst) {
  extern __shared__ __align__(16) uint8_t sbuf[];
  griddep_wait();
  griddep_launch_dependents();
  const int units = ch.unit_off[ch.count];
  for (int u = blockIdx.x; u < units; u += gridDim.x) {
    int b = 0;
    while (b + 1 < ch.count && ch.unit_off[b + 1] <= u) ++b;
    const int local = u - ch.unit_off[b];
    const int nseg = ch.nseg[b];
    const int y = local / nseg, seg = local - y * nseg;
    const int sh = ch.sh[b], sw = ch.sw[b], oh = ch.oh[b], ow = ch.ow[b];
    const int xs = seg * ch.segw[b], xe = min(ow, xs + ch.segw[b]);
    if (xs >= xe) continue;  // uniform over the CTA
    int q, r;
    coord_qr<Idx>(y, sh, oh, q, r);
    const Tap ty = make_tap(q, r, sh, ch.inv_den_y[b]);
    const int64_t img = ch.src_off[b];
    const int64_t row_bytes = 3LL * sw;
    // both source rows of the unit lie inside its image (uniform over the CTA)
    if (!VLM_DCHECK(ty.i0 >= 0 && ty.i1 < sh && img >= 0 && img + sh * row_bytes <= src_bytes)) continue;
    const uint8_t* r0;
    const uint8_t* r1;
    if constexpr (kStaged) {
      int ql, rl, qh, rh;
      coord_qr<Idx>(xs, sw, ow, ql, rl);
      coord_qr<Idx>(xe - 1, sw, ow, qh, rh);
      const int c_lo = make_tap(ql, rl, sw, 0.f).i0;
      const int c_hi = make_tap(qh, rh, sw, 0.f).i1;
      const int n = 3 * (c_hi - c_lo + 1);
      __syncthreads();  // the previous unit's readers are done with the buffer
      const int s0 = stage_bytes(src, src_bytes, img + ty.i0 * row_bytes + 3LL * c_lo, n, sbuf);
      const int s1 = stage_bytes(src, src_bytes, img + ty.i1 * row_bytes + 3LL * c_lo, n, sbuf + ch.stage_bytes);
      __syncthreads();
      r0 = sbuf + s0 - 3 * c_lo;  // indexed only at 3 * column >= 3 * c_lo
      r1 = sbuf + ch.stage_bytes + s1 - 3 * c_lo;
    } else {
      r0 = src + img + ty.i0 * row_bytes;
      r1 = src + img + ty.i1 * row_bytes;
    }
    const int x4 = xs + 4 * threadIdx.x;
    if (x4 >= xe) continue;
    const int tile = ch.tile;
    int64_t plane, o;
    if (tile > 0) {
      plane = static_cast<int64_t>(tile) * tile;
      o = ch.dst_off[b] + (static_cast<int64_t>(y / tile) * (ow / tile) + x4 / tile) * 3 * plane +
          static_cast<int64_t>(y % tile) * tile + (x4 % tile);
    } else {
      plane = static_cast<int64_t>(oh) * ow;
      o = ch.dst_off[b] + static_cast<int64_t>(y) * ow + x4;
    }
    coord_qr<Idx>(x4, sw, ow, q, r);
    const int den = 2 * ow, sq = ch.sq[b], sr = ch.sr[b];
    const float inv_x = ch.inv_den_x[b];
    float out[3][4];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const Tap tx = make_tap(q, r, sw, inv_x);
      q += sq;
      r += sr;
      if (r >= den) {
        r -= den;
        ++q;
      }
      const int a0 = 3 * tx.i0, a1 = 3 * tx.i1;
#pragma unroll
      for (int c = 0; c < 3; ++c) {
        uint32_t b00, b01, b10, b11;
        if constexpr (kStaged) {
          b00 = r0[a0 + c]; b01 = r0[a1 + c]; b10 = r1[a0 + c]; b11 = r1[a1 + c];
        } else {
          b00 = __ldg(r0 + a0 + c); b01 = __ldg(r0 + a1 + c); b10 = __ldg(r1 + a0 + c); b11 = __ldg(r1 + a1 + c);
        }
        const float p00 = byte_as_float(b00), p10 = byte_as_float(b10);
        const float top = fmaf(byte_as_float(b01) - p00, tx.f, p00);
        const float bot = fmaf(byte_as_float(b11) - p10, tx.f, p10);
        out[c][e] = fmaf(bot - top, ty.f, top) * (1.f / 255.f);
      }
    }
#pragma unroll
    for (int c = 0; c < 3; ++c)
      *reinterpret_cast<float4*>(dst + o + c * plane) = make_float4(out[c][0], out[c][1], out[c][2], out[c][3]);
  }
}

int launch_resize_tile(const uint8_t* src, int64_t src_bytes, const ResizeChunk& ch, float* dst, cudaStream_t s) {
  const int units = ch.unit_off[ch.count];
  const bool staged = ch.stage_bytes > 0;
  const size_t smem = staged ? 2 * static_cast<size_t>(ch.stage_bytes) : 0;
  static bool attr_set[64] = {};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 64 && !attr_set[dev]) {
    for (auto k : {resize_tile_kernel<true, int32_t>, resize_tile_kernel<true, int64_t>})
      if (cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, 2 * kResizeStageMax) != cudaSuccess)
        return VLM_ERR_CUDA;
    attr_set[dev] = true;
  }
  int grid = num_sms() * 16;
  if (units < grid) grid = units < 1 ? 1 : units;
  launch_begin(KC_FRONT, s);
  cudaError_t e;
  if (staged)
    e = ch.wide ? launch_pdl(resize_tile_kernel<true, int64_t>, dim3(grid), dim3(128), smem, s, src, src_bytes, ch, dst)
                : launch_pdl(resize_tile_kernel<true, int32_t>, dim3(grid), dim3(128), smem, s, src, src_bytes, ch, dst);
  else
    e = ch.wide ? launch_pdl(resize_tile_kernel<false, int64_t>, dim3(grid), dim3(128), 0, s, src, src_bytes, ch, dst)
                : launch_pdl(resize_tile_kernel<false, int32_t>, dim3(grid), dim3(128), 0, s, src, src_bytes, ch, dst);
  launch_end(KC_FRONT, s);
  return e == cudaSuccess ? VLM_OK : VLM_ERR_CUDA;
}

// ---------------------------------------------------------------------------
// Placeholder expansion. With r(i) the number of markers before position i
// and P the exclusive prefix of the per-image counts, id i lands at
// (i - r(i)) + P[r(i)]; a marker there opens its run of P[r+1] - P[r]
// image_token_id entries. The marker count per 256-id chunk and its scan are
// the masked scatter's first two kernels (the scan also checks the total
// against the number of images and raises VLM_ERR_COUNT_MISMATCH).
// ---------------------------------------------------------------------------
__global__ void prefix_fill_kernel(I64Chunk ch, int64_t* __restrict__ dst) {
  griddep_wait();
  griddep_launch_dependents();
  for (int i = threadIdx.x; i < ch.count; i += blockDim.x) dst[ch.first + i] = ch.v[i];
}

__global__ void __launch_bounds__(256) expand_kernel(const int64_t* __restrict__ ids, int64_t n, int64_t marker,
                                                     const int64_t* __restrict__ chunk_base,
                                                     const int64_t* __restrict__ prefix,
                                                     const int32_t* __restrict__ ok_flag, int64_t image_token,
                                                     int64_t* __restrict__ out, int64_t n_out, int n_images) {
  griddep_wait();
  griddep_launch_dependents();
  if (*ok_flag == 0) return;
  const int64_t i = static_cast<int64_t>(blockIdx.x) * 256 + threadIdx.x;
  const int64_t id = i < n ? ids[i] : 0;
  const int flag = (i < n && id == marker) ? 1 : 0;
  const unsigned ballot = __ballot_sync(0xffffffffu, flag);
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  __shared__ int warp_count[8];
  __shared__ int64_t run_start[256], run_len[256];
  __shared__ int n_runs;
  if (lane == 0) warp_count[warp] = __popc(ballot);
  __syncthreads();
  int before = 0, total = 0;
  for (int w = 0; w < 8; ++w) {
    if (w < warp) before += warp_count[w];
    total += warp_count[w];
  }
  before += __popc(ballot & ((1u << lane) - 1u));
  const int64_t r = chunk_base[blockIdx.x] + before;  // markers before i
  if (i < n) {
    // a marker's run is [at, at + len); another id lands at `at` (checked in debug builds)
    const bool ok_r = VLM_DCHECK(r >= 0 && r + flag <= n_images);
    const int64_t at = ok_r ? (i - r) + prefix[r] : 0;
    const int64_t len = (ok_r && flag) ? prefix[r + 1] - prefix[r] : 0;
    const bool ok = ok_r && VLM_DCHECK(at >= 0 && (flag ? at + len <= n_out : at < n_out));
    if (flag) {
      run_start[before] = at;
      run_len[before] = ok ? len : 0;
    } else if (ok) {
      out[at] = id;
    }
  }
  if (threadIdx.x == 0) n_runs = total;
  __syncthreads();
  for (int k = 0; k < n_runs; ++k) {
    const int64_t start = run_start[k], len = run_len[k];
    for (int64_t j = threadIdx.x; j < len; j += 256) out[start + j] = image_token;
  }
}

int launch_expand(const int64_t* ids, int64_t n, int64_t marker, const int64_t* counts, int n_images,
                  int64_t image_token, int64_t* out, ExpandWs ws, int32_t* status, cudaStream_t s) {
  launch_begin(KC_EXPAND, s);
  int rc = VLM_OK;
  // prefix[0..n_images] from the host's counts, in by-value chunks.
  int64_t acc = 0;
  int launches = 0;
  for (int first = 0; first <= n_images && rc == VLM_OK; first += kI64Chunk) {
    I64Chunk ch;
    ch.first = first;
    ch.count = 0;
    for (int k = first; k <= n_images && ch.count < kI64Chunk; ++k) {
      ch.v[ch.count++] = acc;
      if (k < n_images) acc += counts[k];
    }
    if (launch_pdl(prefix_fill_kernel, dim3(1), dim3(256), 0, s, ch, ws.prefix) != cudaSuccess) rc = VLM_ERR_CUDA;
    ++launches;
  }
  const int64_t n_chunks = (n + 255) / 256;
  if (rc == VLM_OK) rc = launch_marker_count(ids, n, marker, ws.chunk_count, s);
  if (rc == VLM_OK) rc = launch_marker_scan(ws.chunk_count, n_chunks, n_images, ws.chunk_base, ws.ok_flag, status, s);
  if (rc == VLM_OK &&
      launch_pdl(expand_kernel, dim3(static_cast<unsigned>(n_chunks)), dim3(256), 0, s, ids, n, marker,
                 ws.chunk_base, ws.prefix, ws.ok_flag, image_token, out, n - n_images + acc, n_images) != cudaSuccess)
    rc = VLM_ERR_CUDA;
  launch_end(KC_EXPAND, s);
  note_extra_launches(launches + 2);
  return rc;
}

}  // namespace vlm
