// The bf16 GEMM whose epilogue writes each output row to a row of another
// table chosen per row: the masked scatter ("Mistral 3", Mistral3Model: image
// features written at the image_token_id positions of the token embeddings)
// fused into the projector's last linear.
#pragma once
#include <cstdint>

#include <cuda_runtime.h>

namespace vlm {

// Epilogue code of the row-scattered store (internal: not a vlm_gemm epilogue).
constexpr int kEpiRows = 6;

// C = A B^T (bf16 operands, fp32 accumulation, bf16 result), row r of C written
// to row dst_rows[r] of the table `c` (c_rows rows of N bf16 values), and only
// when *ok_flag != 0; nothing is written otherwise. A is [M, K], B is [N, K]
// (K-contiguous), as for launch_gemm. dst_rows and ok_flag are device memory
// written by earlier kernels of the same stream (the scatter's count, scan and
// positions kernels).
int launch_gemm_rows(const void* a, const void* b, int64_t M, int64_t N, int64_t K, void* c, int64_t c_rows,
                     const int64_t* dst_rows, const int32_t* ok_flag, int32_t* status, cudaStream_t s);

// The masked scatter's placeholder positions without its copy, over ids[0, n)
// (one kernel up to 4,096 ids, else the count, scan and positions kernels). dst_rows[k] = the position of the k-th
// id equal to `token`; *ok_flag = 1 when there are exactly n_img of them,
// otherwise 0 (dst_rows is then not written) and *status takes
// VLM_ERR_COUNT_MISMATCH. Uses ws.chunk_count, ws.chunk_base, ws.dst_rows and
// ws.ok_flag (see carve_scatter).
struct ScatterWs;
int launch_scatter_rows(const int64_t* ids, int64_t n, int64_t token, int64_t n_img, const ScatterWs& ws,
                        int32_t* status, cudaStream_t s);

// The index-checked build's failure word of the GEMM file (0: no check failed).
int debug_word_gemm(bool clear);

}  // namespace vlm
