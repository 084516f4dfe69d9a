// Block-diagonal (per-image) bidirectional attention, head_dim 64, over a
// packed variable-resolution sequence: for query t of block b,
// o_t = sum_u softmax_u(q_t . k_u / 8) v_u over the keys u of block b only.
//
// One CTA = one 128-query tile of one block and one head (8 warps x 16 query
// rows). Key/value tiles of 64 rows stream through a double-buffered cp.async
// ring in XOR-swizzled shared memory; S = Q K^T and O += P V run on
// mma.sync.m16n8k16 (bf16 in, fp32 accumulate) with an online (running max)
// softmax in registers. Query tiles never straddle two blocks, and keys past
// the block end are masked to -inf and read as zeros, so a block's output does
// not depend on any other block (bit-identical isolation).
#include "kernels.cuh"

namespace vlm {

namespace {

constexpr int BQ = kAttnBQ;  // 128 queries per CTA
constexpr int BKV = 64;      // keys per tile
constexpr int DH = 64;
constexpr int kThreads = 256;

__device__ __forceinline__ uint32_t swz(int row, int chunk) {
  // byte offset of 16-byte chunk `chunk` (0..7) of 128-byte row `row`
  return static_cast<uint32_t>(row * 128 + ((chunk ^ (row & 7)) << 4));
}

__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src, bool valid) {
  const int n = valid ? 16 : 0;  // src-size 0 -> zero fill
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(n) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}

__device__ __forceinline__ void mma16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
      "{%0, %1, %2, %3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// Loads rows [row0, row0 + nrows) of one 64-wide head slice (element column
// `col`) of a [*, ld] bf16 matrix into a swizzled tile; rows >= row_end read as 0.
__device__ __forceinline__ void load_tile(uint32_t sbase, const __nv_bfloat16* g, int64_t ld, int col, int row0,
                                          int nrows, int row_end) {
  for (int i = threadIdx.x; i < nrows * 8; i += kThreads) {
    const int r = i >> 3, ch = i & 7;
    const int gr = row0 + r;
    const bool valid = gr < row_end;
    const __nv_bfloat16* src = g + static_cast<int64_t>(valid ? gr : 0) * ld + col + ch * 8;
    cp_async16(sbase + swz(r, ch), src, valid);
  }
}

__global__ void __launch_bounds__(kThreads)
    attn_mma_kernel(const __nv_bfloat16* __restrict__ qkv, int heads, const int32_t* __restrict__ cu,
                    const int32_t* __restrict__ qt, int n_blocks, __nv_bfloat16* __restrict__ out) {
  extern __shared__ __align__(128) uint8_t smem[];
  const uint32_t sQ = smem_u32(smem);
  const uint32_t sK0 = sQ + BQ * 128;
  const uint32_t sV0 = sK0 + 2 * BKV * 128;

  const int tile = blockIdx.x, h = blockIdx.y;
  int lo = 0, hi = n_blocks - 1;  // last block b with qt[b] <= tile
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (__ldg(qt + mid) <= tile) lo = mid; else hi = mid - 1;
  }
  const int b = lo;
  const int kbeg = __ldg(cu + b), kend = __ldg(cu + b + 1);
  const int q0 = kbeg + (tile - __ldg(qt + b)) * BQ;
  const int64_t ld = static_cast<int64_t>(3) * heads * DH;
  const int qcol = h * DH, kcol = heads * DH + h * DH, vcol = 2 * heads * DH + h * DH;

  const int n_kv = (kend - kbeg + BKV - 1) / BKV;
  load_tile(sQ, qkv, ld, qcol, q0, BQ, kend);
  load_tile(sK0, qkv, ld, kcol, kbeg, BKV, kend);
  load_tile(sV0, qkv, ld, vcol, kbeg, BKV, kend);
  cp_async_commit();

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, t4 = lane & 3;
  const float sl2 = 1.4426950408889634f * 0.125f;  // log2(e) / sqrt(64)

  uint32_t qa[4][4];
  float o[8][4];
#pragma unroll
  for (int j = 0; j < 8; ++j) o[j][0] = o[j][1] = o[j][2] = o[j][3] = 0.f;
  float m0 = -INFINITY, m1 = -INFINITY, l0 = 0.f, l1 = 0.f;

  for (int it = 0; it < n_kv; ++it) {
    const int buf = it & 1;
    if (it + 1 < n_kv) {
      const int nb = buf ^ 1;
      load_tile(sK0 + nb * BKV * 128, qkv, ld, kcol, kbeg + (it + 1) * BKV, BKV, kend);
      load_tile(sV0 + nb * BKV * 128, qkv, ld, vcol, kbeg + (it + 1) * BKV, BKV, kend);
      cp_async_commit();
      cp_async_wait<1>();
    } else {
      cp_async_wait<0>();
    }
    __syncthreads();
    if (it == 0) {
#pragma unroll
      for (int ks = 0; ks < 4; ++ks) {
        const int row = warp * 16 + (lane & 15);
        ldsm_x4(sQ + swz(row, ks * 2 + (lane >> 4)), qa[ks][0], qa[ks][1], qa[ks][2], qa[ks][3]);
      }
    }
    const uint32_t sK = sK0 + buf * BKV * 128, sV = sV0 + buf * BKV * 128;

    // S = Q K^T for this warp's 16 rows x 64 keys
    float s[8][4];
#pragma unroll
    for (int j = 0; j < 8; ++j) s[j][0] = s[j][1] = s[j][2] = s[j][3] = 0.f;
#pragma unroll
    for (int ks = 0; ks < 4; ++ks) {
#pragma unroll
      for (int np = 0; np < 4; ++np) {  // pairs of 8-key n-tiles
        const int mi = lane >> 3;
        const int key = np * 16 + (mi >> 1) * 8 + (lane & 7);
        uint32_t b0, b1, b2, b3;
        ldsm_x4(sK + swz(key, ks * 2 + (mi & 1)), b0, b1, b2, b3);
        mma16816(s[2 * np], qa[ks], b0, b1);
        mma16816(s[2 * np + 1], qa[ks], b2, b3);
      }
    }
    // mask keys beyond the block and take the running max
    const int kbase = kbeg + it * BKV;
    float mx0 = m0, mx1 = m1;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const int key = kbase + j * 8 + 2 * t4;
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const bool valid = key + e < kend;
        s[j][e] = valid ? s[j][e] * sl2 : -INFINITY;
        s[j][2 + e] = valid ? s[j][2 + e] * sl2 : -INFINITY;
        mx0 = fmaxf(mx0, s[j][e]);
        mx1 = fmaxf(mx1, s[j][2 + e]);
      }
    }
#pragma unroll
    for (int off = 1; off < 4; off <<= 1) {
      mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, off));
      mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, off));
    }
    const float c0 = ex2(m0 - mx0), c1 = ex2(m1 - mx1);
    m0 = mx0;
    m1 = mx1;
    l0 *= c0;
    l1 *= c1;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      o[j][0] *= c0; o[j][1] *= c0;
      o[j][2] *= c1; o[j][3] *= c1;
    }
    uint32_t pa[4][4];
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const float p0 = ex2(s[j][0] - m0), p1 = ex2(s[j][1] - m0);
      const float p2 = ex2(s[j][2] - m1), p3 = ex2(s[j][3] - m1);
      l0 += p0 + p1;
      l1 += p2 + p3;
      const int kk = j >> 1, hi8 = j & 1;
      pa[kk][hi8 * 2 + 0] = pack_bf16x2(p0, p1);
      pa[kk][hi8 * 2 + 1] = pack_bf16x2(p2, p3);
    }
    // O += P V
#pragma unroll
    for (int kk = 0; kk < 4; ++kk) {
#pragma unroll
      for (int dp = 0; dp < 4; ++dp) {  // pairs of 8-wide head-dim n-tiles
        const int mi = lane >> 3;
        const int key = kk * 16 + (mi & 1) * 8 + (lane & 7);
        uint32_t b0, b1, b2, b3;
        ldsm_x4_t(sV + swz(key, dp * 2 + (mi >> 1)), b0, b1, b2, b3);
        mma16816(o[2 * dp], pa[kk], b0, b1);
        mma16816(o[2 * dp + 1], pa[kk], b2, b3);
      }
    }
    __syncthreads();
  }

#pragma unroll
  for (int off = 1; off < 4; off <<= 1) {
    l0 += __shfl_xor_sync(0xffffffffu, l0, off);
    l1 += __shfl_xor_sync(0xffffffffu, l1, off);
  }
  const float inv0 = 1.f / l0, inv1 = 1.f / l1;
  const int r0 = q0 + warp * 16 + g, r1 = r0 + 8;
  const int64_t ldo = static_cast<int64_t>(heads) * DH;
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    const int col = h * DH + j * 8 + 2 * t4;
    if (r0 < kend)
      *reinterpret_cast<uint32_t*>(out + r0 * ldo + col) = pack_bf16x2(o[j][0] * inv0, o[j][1] * inv0);
    if (r1 < kend)
      *reinterpret_cast<uint32_t*>(out + r1 * ldo + col) = pack_bf16x2(o[j][2] * inv1, o[j][3] * inv1);
  }
}

}  // namespace

int launch_attention(const __nv_bfloat16* qkv, int64_t T, int heads, const int32_t* cu, const int32_t* qt,
                     int n_blocks, int total_qtiles, __nv_bfloat16* out, int32_t* status, cudaStream_t s) {
  (void)T;
  (void)status;
  if (total_qtiles <= 0) return VLM_OK;
  constexpr int smem = BQ * 128 + 4 * BKV * 128;  // Q + double-buffered K and V = 48 KiB
  static bool attr_done[64] = {};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 64 && !attr_done[dev]) {
    if (cudaFuncSetAttribute(attn_mma_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess)
      return VLM_ERR_CUDA;
    attr_done[dev] = true;
  }
  dim3 grid(total_qtiles, heads);
  launch_begin(KC_ATTN, s);
  attn_mma_kernel<<<grid, kThreads, smem, s>>>(qkv, heads, cu, qt, n_blocks, out);
  launch_end(KC_ATTN, s);
  return cudaGetLastError() == cudaSuccess ? VLM_OK : VLM_ERR_CUDA;
}

}  // namespace vlm
