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

__host__ __device__ inline int64_t nvfp4_sf_offset(int64_t row, int64_t kblock, int64_t k) {
  const int64_t atom = (row / 128) * (k / 64) + kblock / 4;
  return atom * kSfAtomBytes + 16 * (row % 32) + 4 * ((row % 128) / 32) + (kblock % 4);
}
inline int64_t nvfp4_sf_bytes(int64_t rows, int64_t k) { return (rows + 127) / 128 * (k / 64) * kSfAtomBytes; }

// out[0] = fp32(max |x| / divisor) over n values (dtype 0 bf16, 1 fp32).
int launch_amax_scale(const void* x, int dtype, int64_t n, float divisor, float* out, cudaStream_t s);
// x [rows, k] (row stride k) -> E2M1 codes q [rows, k / 2] and block scales
// sf (nvfp4_sf_bytes(rows, k) bytes; rows past `rows` in the last 128-row
// group get scale 0) with the global scale *s_global (device memory).
int launch_quant_nvfp4(const void* x, int dtype, int64_t rows, int64_t k, const float* s_global, uint8_t* q,
                       uint8_t* sf, cudaStream_t s);
// c = fp32(g_a g_b) * (A . B^T) on NVFP4 operands (A [M, K], B [N, K]);
// epi VLM_EPI_BF16 (c bf16 [M, N]) or VLM_EPI_RESID (c fp32 [M, N], c += result).
int launch_gemm_nvfp4(int epi, const uint8_t* a, const uint8_t* a_sf, const float* g_a, const uint8_t* b,
                      const uint8_t* b_sf, const float* g_b, int64_t M, int64_t N, int64_t K, void* c,
                      int32_t* status, cudaStream_t s);

}  // namespace vlm
