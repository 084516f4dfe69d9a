// NVFP4 quantisation: the per-tensor global scale and the E2M1 codes with
// their E4M3 block scales (layout in nvfp4.cuh). Every scaling step is one
// IEEE fp32 operation in a fixed order:
//   s_b = e4m3(amax_b / fp32(6 s_g)), r = 1 / fp32(s_b s_g) (0 if s_b is 0),
//   q = e2m1(x r),
// both roundings to nearest even with saturation (cvt.rn.satfinite).
#include "nvfp4.cuh"

namespace vlm {

namespace {

__device__ __forceinline__ void load16(const void* x, int dtype, int64_t off, float (&v)[16]) {
  if (dtype == 0) {
    const uint4* p = reinterpret_cast<const uint4*>(static_cast<const __nv_bfloat16*>(x) + off);
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const uint4 u = __ldg(p + h);
      const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        v[8 * h + 2 * j] = __uint_as_float(w[j] << 16);
        v[8 * h + 2 * j + 1] = __uint_as_float(w[j] & 0xFFFF0000u);
      }
    }
  } else {
    const float4* p = reinterpret_cast<const float4*>(static_cast<const float*>(x) + off);
#pragma unroll
    for (int h = 0; h < 4; ++h) {
      const float4 f = __ldg(p + h);
      v[4 * h] = f.x; v[4 * h + 1] = f.y; v[4 * h + 2] = f.z; v[4 * h + 3] = f.w;
    }
  }
}

// fp32 -> E4M3 byte and back (exact), round to nearest even, saturating.
__device__ __forceinline__ uint32_t e4m3_byte(float v) {
  uint16_t r;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(0.0f), "f"(v));
  return r & 0xFFu;
}
__device__ __forceinline__ float e4m3_value(uint32_t byte) {
  uint32_t h2;
  const uint16_t b = static_cast<uint16_t>(byte);
  asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h2) : "h"(b));
  return __half2float(__ushort_as_half(static_cast<unsigned short>(h2 & 0xFFFFu)));
}
// Two fp32 values -> one byte of E2M1 codes, lo in the low nibble.
__device__ __forceinline__ uint32_t e2m1x2(float lo, float hi) {
  uint16_t r;
  asm("{\n\t.reg .b8 t;\n\tcvt.rn.satfinite.e2m1x2.f32 t, %1, %2;\n\tcvt.u16.u8 %0, t;\n\t}"
      : "=h"(r)
      : "f"(hi), "f"(lo));
  return r;
}

__global__ void amax_kernel(const void* __restrict__ x, int dtype, int64_t n, unsigned int* __restrict__ out_bits) {
  griddep_wait();
  griddep_launch_dependents();
  float m = 0.0f;
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  if (dtype == 0) {
    const __nv_bfloat16* p = static_cast<const __nv_bfloat16*>(x);
    for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < n; i += stride)
      m = fmaxf(m, fabsf(__bfloat162float(p[i])));
  } else {
    const float* p = static_cast<const float*>(x);
    for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < n; i += stride)
      m = fmaxf(m, fabsf(p[i]));
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  // non-negative floats order like their bit patterns
  if ((threadIdx.x & 31) == 0 && m > 0.0f) atomicMax(out_bits, __float_as_uint(m));
}

__global__ void scale_finish_kernel(unsigned int* bits, float divisor) {
  griddep_wait();
  griddep_launch_dependents();
  if (threadIdx.x == 0) {
    const float amax = __uint_as_float(*bits);
    *reinterpret_cast<float*>(bits) = __fdiv_rn(amax, divisor);
  }
}

// One thread per block of 16 values; threads of a warp take consecutive blocks
// of a row (coalesced 32- or 64-byte reads and 8-byte code writes). Rows from
// `rows` up to the end of the last 128-row group only write scale 0.
__global__ void quant_nvfp4_kernel(const void* __restrict__ x, int dtype, int64_t rows, int64_t k,
                                   const float* __restrict__ s_global, uint8_t* __restrict__ q,
                                   uint8_t* __restrict__ sf) {
  griddep_wait();
  griddep_launch_dependents();
  const int64_t kb = k / kFp4Block;
  const int64_t rows_pad = (rows + 127) / 128 * 128;
  const int64_t total = rows_pad * kb;
  const float sg = __ldg(s_global);
  const float six_sg = 6.0f * sg;
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < total; i += stride) {
    const int64_t row = i / kb, blk = i - row * kb;
    if (row >= rows) {
      sf[nvfp4_sf_offset(row, blk, k)] = 0;
      continue;
    }
    float v[16];
    load16(x, dtype, row * k + blk * kFp4Block, v);
    float amax = 0.0f;
#pragma unroll
    for (int j = 0; j < 16; ++j) amax = fmaxf(amax, fabsf(v[j]));
    const uint32_t code = six_sg > 0.0f ? e4m3_byte(__fdiv_rn(amax, six_sg)) : 0u;
    const float denom = e4m3_value(code) * sg;
    const float r = denom > 0.0f ? __fdiv_rn(1.0f, denom) : 0.0f;
    uint32_t w[2] = {0u, 0u};
#pragma unroll
    for (int j = 0; j < 8; ++j) w[j >> 2] |= e2m1x2(v[2 * j] * r, v[2 * j + 1] * r) << (8 * (j & 3));
    *reinterpret_cast<uint2*>(q + row * (k / 2) + blk * 8) = make_uint2(w[0], w[1]);
    sf[nvfp4_sf_offset(row, blk, k)] = static_cast<uint8_t>(code);
  }
}

}  // namespace

int launch_amax_scale(const void* x, int dtype, int64_t n, float divisor, float* out, cudaStream_t s) {
  if (x == nullptr || out == nullptr || (dtype != 0 && dtype != 1)) return VLM_ERR_INVALID_ARG;
  if (n <= 0 || !(divisor > 0.0f)) return VLM_ERR_BAD_SHAPE;
  if (cudaMemsetAsync(out, 0, sizeof(float), s) != cudaSuccess) return VLM_ERR_CUDA;
  const int64_t want = (n + 255) / 256;
  const int grid = static_cast<int>(want < 4 * num_sms() ? want : 4 * num_sms());
  launch_begin(KC_PACK, s);
  cudaError_t e = launch_pdl(amax_kernel, dim3(grid), dim3(256), 0, s, x, dtype, n,
                             reinterpret_cast<unsigned int*>(out));
  if (e == cudaSuccess)
    e = launch_pdl(scale_finish_kernel, dim3(1), dim3(32), 0, s, reinterpret_cast<unsigned int*>(out), divisor);
  launch_end(KC_PACK, s);
  return e == cudaSuccess ? VLM_OK : VLM_ERR_CUDA;
}

int launch_quant_nvfp4(const void* x, int dtype, int64_t rows, int64_t k, const float* s_global, uint8_t* q,
                       uint8_t* sf, cudaStream_t s) {
  if (x == nullptr || s_global == nullptr || q == nullptr || sf == nullptr || (dtype != 0 && dtype != 1))
    return VLM_ERR_INVALID_ARG;
  if (rows <= 0 || k <= 0 || rows > (1LL << 31) - 1) return VLM_ERR_BAD_SHAPE;
  if (k % 64 != 0) return VLM_ERR_UNSUPPORTED;
  if ((reinterpret_cast<uintptr_t>(x) & 15) || (reinterpret_cast<uintptr_t>(q) & 7)) return VLM_ERR_INVALID_ARG;
  const int64_t total = (rows + 127) / 128 * 128 * (k / kFp4Block);
  const int64_t want = (total + 255) / 256;
  const int grid = static_cast<int>(want < 8 * num_sms() ? want : 8 * num_sms());
  launch_begin(KC_PACK, s);
  const cudaError_t e = launch_pdl(quant_nvfp4_kernel, dim3(grid), dim3(256), 0, s, x, dtype, rows, k, s_global, q, sf);
  launch_end(KC_PACK, s);
  return e == cudaSuccess ? VLM_OK : VLM_ERR_CUDA;
}

}  // namespace vlm
