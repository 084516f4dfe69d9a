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
// x2 != nullptr: output rows 32j..32j+15 are rows 16j.. of x, rows
// 32j+16..32j+31 rows 16j.. of x2 (the gate / up interleave).
__global__ void quant_nvfp4_kernel(const void* __restrict__ x, const void* __restrict__ x2, int dtype, int64_t rows,
                                   int64_t k, const float* __restrict__ s_global, uint8_t* __restrict__ q,
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
    if (x2 == nullptr) {
      load16(x, dtype, row * k + blk * kFp4Block, v);
    } else {
      const int64_t src = (row >> 5) * 16 + (row & 15);
      load16((row & 16) ? x2 : x, dtype, src * k + blk * kFp4Block, v);
    }
    float amax = 0.0f;
#pragma unroll
    for (int j = 0; j < 16; ++j) amax = fmaxf(amax, fabsf(v[j]));
    uint2 codes;
    const uint32_t sb = nvfp4_quant16(v, amax, sg, six_sg, codes);
    *reinterpret_cast<uint2*>(q + row * (k / 2) + blk * 8) = codes;
    sf[nvfp4_sf_offset(row, blk, k)] = static_cast<uint8_t>(sb);
  }
}

}  // namespace

int launch_amax_scale(const void* x, int dtype, int64_t n, float divisor, float* out, cudaStream_t s) {
  return launch_amax_scale_multi(&x, &n, 1, dtype, divisor, out, s);
}

int launch_amax_scale_multi(const void* const* xs, const int64_t* ns, int count, int dtype, float divisor, float* out,
                            cudaStream_t s) {
  if (xs == nullptr || ns == nullptr || count <= 0 || out == nullptr || (dtype != 0 && dtype != 1))
    return VLM_ERR_INVALID_ARG;
  if (!(divisor > 0.0f)) return VLM_ERR_BAD_SHAPE;
  for (int i = 0; i < count; ++i) {
    if (xs[i] == nullptr) return VLM_ERR_INVALID_ARG;
    if (ns[i] <= 0) return VLM_ERR_BAD_SHAPE;
  }
  if (cudaMemsetAsync(out, 0, sizeof(float), s) != cudaSuccess) return VLM_ERR_CUDA;
  launch_begin(KC_PACK, s);
  cudaError_t e = cudaSuccess;
  for (int i = 0; i < count && e == cudaSuccess; ++i) {
    const int64_t want = (ns[i] + 255) / 256;
    const int grid = static_cast<int>(want < 4 * num_sms() ? want : 4 * num_sms());
    e = launch_pdl(amax_kernel, dim3(grid), dim3(256), 0, s, xs[i], dtype, ns[i], reinterpret_cast<unsigned int*>(out));
  }
  if (e == cudaSuccess)
    e = launch_pdl(scale_finish_kernel, dim3(1), dim3(32), 0, s, reinterpret_cast<unsigned int*>(out), divisor);
  launch_end(KC_PACK, s);
  return e == cudaSuccess ? VLM_OK : VLM_ERR_CUDA;
}

int launch_quant_nvfp4(const void* x, int dtype, int64_t rows, int64_t k, const float* s_global, uint8_t* q,
                       uint8_t* sf, cudaStream_t s) {
  return launch_quant_nvfp4_rows(x, nullptr, dtype, rows, k, s_global, q, sf, s);
}

int launch_quant_nvfp4_rows(const void* x, const void* x2, int dtype, int64_t rows, int64_t k,
                            const float* s_global, uint8_t* q, uint8_t* sf, cudaStream_t s) {
  if (x == nullptr || s_global == nullptr || q == nullptr || sf == nullptr || (dtype != 0 && dtype != 1))
    return VLM_ERR_INVALID_ARG;
  if (rows <= 0 || k <= 0 || rows > (1LL << 31) - 1) return VLM_ERR_BAD_SHAPE;
  if (k % 64 != 0 || (x2 != nullptr && rows % 32 != 0)) return VLM_ERR_UNSUPPORTED;
  if ((reinterpret_cast<uintptr_t>(x) & 15) || (reinterpret_cast<uintptr_t>(x2) & 15) ||
      (reinterpret_cast<uintptr_t>(q) & 7))
    return VLM_ERR_INVALID_ARG;
  const int64_t total = (rows + 127) / 128 * 128 * (k / kFp4Block);
  const int64_t want = (total + 255) / 256;
  const int grid = static_cast<int>(want < 8 * num_sms() ? want : 8 * num_sms());
  launch_begin(KC_PACK, s);
  const cudaError_t e =
      launch_pdl(quant_nvfp4_kernel, dim3(grid), dim3(256), 0, s, x, x2, dtype, rows, k, s_global, q, sf);
  launch_end(KC_PACK, s);
  return e == cudaSuccess ? VLM_OK : VLM_ERR_CUDA;
}

}  // namespace vlm
