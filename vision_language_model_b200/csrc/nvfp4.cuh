// NVFP4 operands: E2M1 values (two per byte, the lower K index in the low
// nibble) with one E4M3 scale per 16 values of a row along K and one fp32
// global scale per tensor. Declarations shared by the quantiser, the
// block-scaled GEMM and the C-ABI layer.
//
// Scale layout (the order in which the tensor cores take block scales into
// tensor memory): rows are grouped by 128 and K by 64 (four scales). Each
// (row group, K group) pair is one 512-byte atom, atoms ordered K group
// fastest; inside an atom, row r's four scales are bytes
// 16 * (r % 32) + 4 * ((r % 128) / 32) + (k / 16) % 4.
#pragma once

#include "kernels.cuh"

namespace vlm {

constexpr int kFp4Block = 16;      // values per block scale
constexpr int kSfAtomBytes = 512;  // 128 rows x 4 scales

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

// One block of 16 fp32 values with global scale sg (six_sg = fp32(6 sg)):
// returns the E4M3 block scale byte s_b = e4m3(amax / six_sg) and sets the
// 8 bytes of E2M1 codes e2m1(v * fp32(1 / fp32(s_b sg))) (all 0 when s_b is 0).
// amax: max |v| of the block, computed by the caller.
// The block scale alone: returns s_b and sets r = fp32(1 / fp32(s_b sg)).
__device__ __forceinline__ uint32_t nvfp4_block_scale(float amax, float sg, float six_sg, float& r) {
  const uint32_t sb = six_sg > 0.0f ? e4m3_byte(__fdiv_rn(amax, six_sg)) : 0u;
  const float denom = e4m3_value(sb) * sg;
  r = denom > 0.0f ? __frcp_rn(denom) : 0.0f;  // the correctly rounded reciprocal
  return sb;
}
__device__ __forceinline__ uint32_t nvfp4_quant16(const float (&v)[16], float amax, float sg, float six_sg,
                                                  uint2& codes) {
  float r;
  const uint32_t sb = nvfp4_block_scale(amax, sg, six_sg, r);
  uint32_t w[2] = {0u, 0u};
#pragma unroll
  for (int j = 0; j < 8; ++j) w[j >> 2] |= e2m1x2(v[2 * j] * r, v[2 * j + 1] * r) << (8 * (j & 3));
  codes = make_uint2(w[0], w[1]);
  return sb;
}

__host__ __device__ inline int64_t nvfp4_sf_offset(int64_t row, int64_t kblock, int64_t k) {
  const int64_t atom = (row / 128) * (k / 64) + kblock / 4;
  return atom * kSfAtomBytes + 16 * (row % 32) + 4 * ((row % 128) / 32) + (kblock % 4);
}
inline int64_t nvfp4_sf_bytes(int64_t rows, int64_t k) { return (rows + 127) / 128 * (k / 64) * kSfAtomBytes; }

// out[0] = fp32(max |x| / divisor) over n values (dtype 0 bf16, 1 fp32).
int launch_amax_scale(const void* x, int dtype, int64_t n, float divisor, float* out, cudaStream_t s);
// The same over the concatenation of `count` tensors (one global scale for
// several weight matrices that one GEMM multiplies as a whole).
int launch_amax_scale_multi(const void* const* xs, const int64_t* ns, int count, int dtype, float divisor, float* out,
                            cudaStream_t s);
// x [rows, k] (row stride k) -> E2M1 codes q [rows, k / 2] and block scales
// sf (nvfp4_sf_bytes(rows, k) bytes; rows past `rows` in the last 128-row
// group get scale 0) with the global scale *s_global (device memory).
int launch_quant_nvfp4(const void* x, int dtype, int64_t rows, int64_t k, const float* s_global, uint8_t* q,
                       uint8_t* sf, cudaStream_t s);
// launch_quant_nvfp4 with x2 != nullptr: output rows 32j..32j+15 from rows
// 16j.. of x and 32j+16..32j+31 from rows 16j.. of x2 (rows % 32 == 0).
int launch_quant_nvfp4_rows(const void* x, const void* x2, int dtype, int64_t rows, int64_t k,
                            const float* s_global, uint8_t* q, uint8_t* sf, cudaStream_t s);
// c = fp32(g_a g_b) * (A . B^T) on NVFP4 operands (A [M, K], B [N, K]);
// epi VLM_EPI_BF16 (c bf16 [M, N]) or VLM_EPI_RESID (c fp32 [M, N], c += result).
int launch_gemm_nvfp4(int epi, const uint8_t* a, const uint8_t* a_sf, const float* g_a, const uint8_t* b,
                      const uint8_t* b_sf, const float* g_b, int64_t M, int64_t N, int64_t K, void* c,
                      int32_t* status, cudaStream_t s);

// launch_gemm_nvfp4 with two more epilogues, both for N % 256 == 0:
// VLM_EPI_ROPE -- c bf16 [M, N], the 2D rotary embedding applied to columns
// below rope_cols (pos: per-row (row << 16 | col) positions, rope: the angle
// table); VLM_EPI_SWIGLU -- accumulator columns 32g..32g+15 gate and
// 32g+16..32g+31 up of hidden columns 16g..16g+15: c holds the NVFP4 codes of
// silu(gate) * up [M, N / 2] (N / 4 bytes per row), c_sf their block scales
// (rows of [M, N / 2]), out_sg their global scale.
int launch_gemm_nvfp4_ex(int epi, const uint8_t* a, const uint8_t* a_sf, const float* g_a, const uint8_t* b,
                         const uint8_t* b_sf, const float* g_b, int64_t M, int64_t N, int64_t K, void* c,
                         uint8_t* c_sf, float out_sg, const int32_t* pos, const float2* rope, int64_t rope_cols,
                         int32_t* status, cudaStream_t s);

// RMSNorm (as launch_rmsnorm) whose output is NVFP4 with global scale
// s_global: codes q [rows, width / 2], block scales sf (nvfp4_sf_bytes(rows,
// width) bytes; the caller zeroes the scales of the padding rows).
int launch_rmsnorm_nvfp4(float* x, const float* g0, const float* g1, uint8_t* q, uint8_t* sf, int64_t rows,
                         int width, float eps, float s_global, cudaStream_t s);

}  // namespace vlm
