/*
 * vlm_kernels.h -- per-kernel entry points of the B200 image-half library.
 *
 * vlm_encode / vlm_merge_project / vlm_scatter (vlm.h) chain these kernels;
 * they are exported on their own so each can be checked against the CPU
 * oracle at full size. Conventions (ownership, status word, streams, error
 * returns) are those of vlm.h. Page citations use the same keys:
 * [K] "Mistral 3" (KerasFormers), [P] "Pixtral-12B-2409".
 */
#ifndef VLM_B200_KERNELS_H
#define VLM_B200_KERNELS_H

#include <stddef.h>
#include <stdint.h>

#include "vlm.h"

#ifdef __cplusplus
extern "C" {
#endif

/* Epilogues of vlm_gemm (what is done with the fp32 accumulator acc[M, N]):
 *   BF16   c = bf16(acc)                                  c: bf16 [M, N]
 *   F32    c = acc                                        c: fp32 [M, N]
 *   RESID  c += acc (fp32 residual update in place);      c: fp32 [M, N]
 *          if c_bf16 != NULL also c_bf16 = bf16(new c)    c_bf16: bf16 [M, N]
 *   SWIGLU with B rows interleaved in groups of 16 (rows 32j..32j+15 gate
 *          rows 16j.., rows 32j+16..32j+31 up rows 16j..):
 *          c[:, 16j+i] = bf16(silu(acc[:, 32j+i]) * acc[:, 32j+16+i]),
 *          silu(z) = z / (1 + e^-z)                       c: bf16 [M, N/2]
 *          (the gated-SiLU MLP's first half; [K]/[P] give its width 4096)
 *   ROPE   c = bf16(acc) after rotating, in columns [0, rope_cols), each
 *          64-column head's pairs (i, i+32) by the angle table entry of the
 *          row's position: pairs i < 16 use the patch row r, pairs i >= 16
 *          the patch column c ([K] Mistral3VisionModel "2D-rotary")
 *                                                          c: bf16 [M, N]
 *          d_pos: int32 [M] = (r << 16) | c; d_rope_table: from vlm_rope_table
 *   GELU   c = bf16(gelu(acc)), gelu(z) = z (1 + erf(z / sqrt 2)) / 2
 *                                                          c: bf16 [M, N]
 */
enum {
  VLM_EPI_BF16 = 0,
  VLM_EPI_F32 = 1,
  VLM_EPI_RESID = 2,
  VLM_EPI_SWIGLU = 3,
  VLM_EPI_ROPE = 4,
  VLM_EPI_GELU = 5
};

/* acc = A . B^T on the sm_100a tensor cores (tcgen05.mma kind::f16, fp32
 * accumulation in TMEM, operands staged by TMA), followed by `epilogue`.
 * A: device bf16 [M, K]; B: device bf16 [N, K]; both row-major, 16-byte
 * aligned. Requires K % 64 == 0, N % 128 == 0 (N % 256 == 0 for SWIGLU and
 * ROPE), M >= 1. Returns VLM_ERR_UNSUPPORTED otherwise. */
VLM_API int vlm_gemm(int epilogue, const void* d_a, const void* d_b, int64_t M, int64_t N, int64_t K,
             void* d_c, void* d_c_bf16, const int32_t* d_pos, const void* d_rope_table,
             int64_t rope_cols, int32_t* d_status, void* stream);

/* The same product with E4M3 operands (tcgen05.mma kind::f8f6f4, fp32
 * accumulation), then the accumulator column n is multiplied by
 * d_colscale[n] (device fp32 [N], 16-byte aligned) before `epilogue`.
 * A: device E4M3 [M, K]; B: device E4M3 [N, K]. Requires K % 128 == 0,
 * N % 256 == 0. Epilogues BF16, RESID, ROPE (as for vlm_gemm) and SWIGLU,
 * whose output is E4M3 [M, N/2] holding the gated values times out_scale
 * (round to nearest even, saturating to +-448); others return
 * VLM_ERR_UNSUPPORTED. */
VLM_API int vlm_gemm_fp8(int epilogue, const void* d_a, const void* d_b, const float* d_colscale, float out_scale,
                         int64_t M, int64_t N, int64_t K, void* d_c, void* d_c_bf16, const int32_t* d_pos,
                         const void* d_rope_table, int64_t rope_cols, int32_t* d_status, void* stream);

/* 2D RoPE angle table ([K] vision_rope_theta): entry [p][i] (float2 cos, sin)
 * of the angle p * w, w = theta^(-2k/head_dim) with k = 2i for i < head_dim/4
 * (row frequencies) and k = 2(i - head_dim/4) + 1 otherwise (column
 * frequencies). d_table: device float2 [max_pos, head_dim/2]. */
VLM_API int vlm_rope_table(float theta, int head_dim, int max_pos, void* d_table, void* stream);

/* Block-diagonal bidirectional attention over a packed sequence:
 * out[t, h*64:(h+1)*64] = softmax_u(q_t . k_u / 8) v_u over the keys u of
 * t's own block [cu[b], cu[b+1]) only ([K] Mistral3VisionModel, packed
 * variable-resolution sequence; one block per image or per [P] tile).
 * d_qkv: device bf16 [T, 3 * heads * 64] with q, k, v column blocks (RoPE
 * already applied). cu_seqlens: HOST int32 [n_blocks + 1], cu[0] = 0,
 * cu[n_blocks] = T, non-decreasing. d_out: device bf16 [T, heads * 64].
 * head_dim must be 64. */
VLM_API size_t vlm_attention_workspace_size(int n_blocks);
VLM_API int vlm_attention(const void* d_qkv, int64_t T, int heads, int head_dim, const int32_t* cu_seqlens,
                  int n_blocks, void* d_out, void* d_workspace, size_t ws_bytes, int32_t* d_status,
                  void* stream);

/* RMSNorm over rows of width `width` (a multiple of 128, <= 2048):
 * y = x / sqrt(mean(x^2) + eps) * g. If d_g0 != NULL the row is first
 * normalised with gain g0 and written back to d_x (fp32, in place), and the
 * bf16 output is the RMSNorm of that result with gain g1; otherwise
 * d_out = bf16(rmsnorm(x) * g1). d_x: fp32 [rows, width]. */
VLM_API int vlm_rmsnorm(float* d_x, const float* d_g0, const float* d_g1, void* d_out, int64_t rows,
                int width, float eps, void* stream);

/* vlm_rmsnorm with an E4M3 output: d_out holds norm(.) * g1 * f8_scale rounded
 * to E4M3 (nearest even, saturating to +-448); f8_scale > 0. */
VLM_API int vlm_rmsnorm_fp8(float* d_x, const float* d_g0, const float* d_g1, void* d_out, int64_t rows, int width,
                            float eps, float f8_scale, void* stream);

/* NVFP4 operands. The vllm.cpp issue ("Mistral3ForConditionalGeneration ...",
 * "Why this one is smaller than it looks", quantisation loaders) loads NVFP4
 * weights: 4-bit E2M1 values with one E4M3 scale per block. Reading: a block
 * is 16 consecutive values of a row along K and the tensor has one fp32
 * global scale s_g, so x ~ q * s_b * s_g; both GEMM operands use this format.
 *
 * Codes: uint8 [rows, K/2], value k of a row in byte k/2, the low nibble for
 * even k (E2M1 code s.ee.m, magnitudes 0, .5, 1, 1.5, 2, 3, 4, 6).
 * Block scales: vlm_nvfp4_sf_bytes(rows, K) bytes of E4M3 codes in 512-byte
 * atoms: rows grouped by 128, K by 64; atom (row/128) * (K/64) + k/64; inside
 * it, row r's scale of block k/16 is byte 16 (r % 32) + 4 ((r % 128) / 32)
 * + (k/16) % 4. This is the order in which the block-scaled tensor-core
 * product takes its scales. Rows past `rows` in the last group have scale 0.
 * Returns 0 for a K that is not a positive multiple of 64 or rows < 1. */
VLM_API size_t vlm_nvfp4_sf_bytes(int64_t rows, int64_t K);

/* Element types of vlm_amax_scale and vlm_quant_nvfp4 inputs. */
enum { VLM_DTYPE_BF16 = 0, VLM_DTYPE_F32 = 1 };

/* d_out[0] = fp32(max |x| / divisor) over n values of d_x (dtype VLM_DTYPE_BF16
 * or VLM_DTYPE_F32, device memory). With divisor 2688 (= 6 * 448) this is an
 * NVFP4 global scale: the largest block of the tensor gets scale 448. */
VLM_API int vlm_amax_scale(const void* d_x, int dtype, int64_t n, float divisor, float* d_out, void* stream);

/* x [rows, K] (bf16 or fp32 by dtype, row-major, 16-byte aligned, K % 64 == 0)
 * to NVFP4 with the global scale *d_sg (device fp32): per block of 16,
 * s_b = e4m3(amax / fp32(6 s_g)); r = 1 / fp32(s_b s_g) (0 when s_b = 0);
 * q = e2m1(x r); each step one IEEE fp32 operation, both roundings to nearest
 * even and saturating (+-448, +-6). d_q: [rows, K/2] (8-byte aligned);
 * d_sf: vlm_nvfp4_sf_bytes(rows, K) bytes. */
VLM_API int vlm_quant_nvfp4(const void* d_x, int dtype, int64_t rows, int64_t K, const float* d_sg, void* d_q,
                            void* d_sf, void* stream);

/* acc = A . B^T on NVFP4 operands (tcgen05.mma kind::mxf4nvf4 with block
 * scales, fp32 accumulation in TMEM), times fp32(*d_ga * *d_gb), then
 * `epilogue`: BF16 (d_c bf16 [M, N]) or RESID (d_c fp32 [M, N], d_c += result).
 * A: codes [M, K/2] and scales for M rows; B: codes [N, K/2] and scales for N
 * rows; all 16-byte aligned. Requires K % 256 == 0, N % 128 == 0, M >= 1;
 * other epilogues or shapes return VLM_ERR_UNSUPPORTED. */
VLM_API int vlm_gemm_nvfp4(int epilogue, const void* d_a, const void* d_a_sf, const float* d_ga, const void* d_b,
                           const void* d_b_sf, const float* d_gb, int64_t M, int64_t N, int64_t K, void* d_c,
                           int32_t* d_status, void* stream);

/* vlm_gemm_nvfp4 with the two tower epilogues of vlm_encode_nvfp4, both for
 * N % 256 == 0:
 * ROPE: d_c bf16 [M, N]; the 2D rotary embedding (as vlm_gemm's ROPE: d_pos
 *   int32 [M] = row << 16 | col, d_rope from vlm_rope_table) rotates columns
 *   below rope_cols (a multiple of 64), pair (i, i + 32) of every 64.
 * SWIGLU: accumulator columns 32g..32g+15 are gate and 32g+16..32g+31 up of
 *   hidden columns 16g..16g+15; h = silu(gate) * up in fp32 is quantised to
 *   NVFP4 with global scale out_sg > 0 as vlm_quant_nvfp4 does: d_c codes
 *   [M, N/4] bytes, d_c_sf block scales of an [M, N/2] operand (4-byte
 *   aligned; scales of rows >= M are not written).
 * BF16 and RESID as vlm_gemm_nvfp4 (d_c_sf, out_sg, d_pos, d_rope unused). */
VLM_API int vlm_gemm_nvfp4_ex(int epilogue, const void* d_a, const void* d_a_sf, const float* d_ga, const void* d_b,
                              const void* d_b_sf, const float* d_gb, int64_t M, int64_t N, int64_t K, void* d_c,
                              void* d_c_sf, float out_sg, const int32_t* d_pos, const void* d_rope, int64_t rope_cols,
                              int32_t* d_status, void* stream);

/* The first steps of vlm_encode alone: index setup, the normalising patch
 * gather and the patch-embed GEMM ([K] Mistral3VisionModel: conv patch
 * embed), d_x = fp32 [T, width] patch features before ln_pre. d_packed_tower:
 * any packed tower (vlm_pack_tower, _fp8 or _nvfp4: each starts with w_pe).
 * d_workspace: 256-byte aligned, at least vlm_encode_workspace_size bytes. */
VLM_API int vlm_patch_embed(const vlm_config* cfg, const float* pixels, const int32_t* image_hw, int n_images,
                            const void* d_packed_tower, float* d_x, void* d_workspace, size_t ws_bytes,
                            int32_t* d_status, void* stream);

/* vlm_rmsnorm whose output is NVFP4: the fp32 values norm(.) * g1 quantised
 * with global scale s_global > 0 as vlm_quant_nvfp4 does; d_q codes
 * [rows, width/2], d_sf vlm_nvfp4_sf_bytes(rows, width) bytes (scales of the
 * padding rows are not written). */
VLM_API int vlm_rmsnorm_nvfp4(float* d_x, const float* d_g0, const float* d_g1, void* d_q, void* d_sf, int64_t rows,
                              int width, float eps, float s_global, void* stream);

/* vlm_attention whose output is NVFP4: the fp32 attention output quantised
 * with global scale s_global > 0 as vlm_quant_nvfp4 does; d_q codes
 * [T, heads * 32] (16-byte aligned), d_sf vlm_nvfp4_sf_bytes(T, heads * 64)
 * bytes (scales of the padding rows are not written). */
VLM_API int vlm_attention_nvfp4(const void* d_qkv, int64_t T, int heads, int head_dim, const int32_t* cu_seqlens,
                                int n_blocks, void* d_q, void* d_sf, float s_global, void* d_workspace,
                                size_t ws_bytes, int32_t* d_status, void* stream);

/* Failure-detection self-test (no counterpart on the pages): launches one
 * thread that waits on a shared-memory mbarrier nothing arrives on, using the
 * same bounded wait as every barrier wait of the GEMM and attention kernels,
 * with a budget of budget_cycles SM clocks (1 .. 2^32). The wait gives up,
 * writes VLM_ERR_TIMEOUT to *d_status and the kernel returns; the CUDA context
 * stays usable. Nothing faults, traps or hangs. */
VLM_API int vlm_selftest_wait_timeout(int64_t budget_cycles, int32_t* d_status, void* stream);

/* Debug build (no counterpart on the pages). The library can be compiled with
 * -DVLM_DEBUG (libvlm_b200_debug.so, built beside the release library): every
 * index that a kernel computes from tables or data before a global access --
 * token positions, patch-gather items and pixel rows, merge destinations,
 * scatter and expansion destinations, resize source rows, attention output
 * rows -- is checked; a failing check records a code (source file id << 16 |
 * line) in a device word and the access is skipped. Nothing traps. TMA
 * transfers need no check: their tensor maps bound them.
 *
 * vlm_debug_build: 1 in a debug build, 0 otherwise (no CUDA call).
 * vlm_debug_checks: synchronises the device, writes the first failing check's
 *   code to *first_failure (0 when none failed) and clears the record.
 *   VLM_OK in a debug build; VLM_ERR_UNSUPPORTED (and 0 written) otherwise;
 *   VLM_ERR_CUDA if the record cannot be read.
 * vlm_debug_selftest_bounds: debug builds only; threads i < 2n would write
 *   d_buf[i] (int32) behind the check i < n, so the check must fail for
 *   i >= n and leave d_buf[n .. 2n) untouched (d_buf holds 2n values,
 *   1 <= n <= 2^20). Release builds return VLM_ERR_UNSUPPORTED and launch
 *   nothing. */
VLM_API int vlm_debug_build(void);
VLM_API int vlm_debug_checks(int32_t* first_failure);
VLM_API int vlm_debug_selftest_bounds(int32_t* d_buf, int n, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* VLM_B200_KERNELS_H */
