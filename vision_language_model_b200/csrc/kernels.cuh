// Internal declarations shared by the kernel files and the C-ABI layer.
#pragma once

#include "common.cuh"

namespace vlm {

// Per-image table kept on the device.
struct ImgInfo {
  int32_t h, w;        // patch grid
  int32_t H, W;        // pixels
  int32_t tok_off;     // first patch of the image in the packed sequence
  int32_t m_off;       // first merged token of the image
  int32_t qt_off;      // first attention query tile of the image
  int32_t pad;
  int64_t pix_off;     // first float of the image in the pixel buffer
};

// Up to kChunk images' host-computed tables, passed by value to the setup kernel.
constexpr int kChunk = 64;
struct ImageChunk {
  int32_t first, count;
  int32_t h[kChunk], w[kChunk], H[kChunk], W[kChunk];
  int32_t tok_off[kChunk + 1], m_off[kChunk + 1], qt_off[kChunk + 1];
  int32_t i2c_off[kChunk + 1];  // first patch-gather work item of each image
  int64_t pix_off[kChunk];
};

// Patches per work item of the tiled patch gather (one patch row segment).
constexpr int kI2cPatches = 8;

struct ScatterWs {
  int32_t* chunk_count;
  int64_t* chunk_base;
  int64_t* dst_rows;
  int32_t* ok_flag;
};

// Up to kResizeChunk images of one resize launch, passed by value.
constexpr int kResizeChunk = 32;
constexpr int kResizeSegMax = 512;        // output pixels per work unit (a row segment)
constexpr int kResizeStageMax = 48 * 1024;  // largest staged source span per row
struct ResizeChunk {
  int32_t count;
  int32_t tile;          // 0: no tiling
  int32_t wide;          // 1: (2 out + 1) * in overflows int32 for some image: 64-bit coordinates
  int32_t stage_bytes;   // shared memory per staged source row span; 0: taps read global memory
  int32_t sh[kResizeChunk], sw[kResizeChunk];  // source size (pixels)
  int32_t oh[kResizeChunk], ow[kResizeChunk];  // output size (pixels)
  int32_t nseg[kResizeChunk], segw[kResizeChunk];  // row segments per output row, and their width
  int32_t sq[kResizeChunk], sr[kResizeChunk];  // 2 sw = sq * (2 ow) + sr
  float inv_den_x[kResizeChunk], inv_den_y[kResizeChunk];  // 1 / (2 ow), 1 / (2 oh)
  int32_t unit_off[kResizeChunk + 1];          // first work unit of each image in this chunk
  int64_t src_off[kResizeChunk];               // first byte of each source image
  int64_t dst_off[kResizeChunk];               // first float of each output image
};

// Up to kI64Chunk int64 values written by one launch (table upload without a copy call).
constexpr int kI64Chunk = 256;
struct I64Chunk {
  int32_t first, count;
  int64_t v[kI64Chunk];
};

struct ExpandWs {
  int32_t* chunk_count;
  int64_t* chunk_base;
  int64_t* prefix;
  int32_t* ok_flag;
};

// Query rows per attention CTA tile.
constexpr int kAttnBQ = 128;

void note_extra_launches(int n);

// Debug words of the files with index checks (see VLM_DCHECK): the first
// failing check's code or 0 (-1 if the read failed); `clear` resets the word.
int debug_word_small_kernels(bool clear);
int debug_word_frontend(bool clear);
int debug_word_attention(bool clear);
int launch_debug_selftest(int32_t* buf, int n, cudaStream_t s);

int launch_setup(const ImageChunk& chunk, ImgInfo* info, int32_t* cu, int32_t* qt, int32_t* i2c, int32_t* pos,
                 int n_images, cudaStream_t s);
int launch_rope_table(float theta, int head_dim, int max_pos, float2* tab, cudaStream_t s);
// i2c / i2c_items: work items of the tiled gather (p 14 or 16); other patch
// sizes use one warp per patch.
int launch_im2col(const float* pix, const ImgInfo* info, const int32_t* cu, const int32_t* i2c, int i2c_items,
                  int n_images, int64_t T, int p, int kp, int normalize, __nv_bfloat16* out, cudaStream_t s);
// f8_scale > 0: `out` is E4M3 holding the normalised values times f8_scale; else bf16.
int launch_rmsnorm(float* x, const float* g0, const float* g1, void* out, int64_t rows, int width, float eps,
                   cudaStream_t s, float f8_scale = 0.f);
// RMSNorm of bf16 rows [rows, width] into bf16 (out may equal x).
int launch_rmsnorm_bf16(const __nv_bfloat16* x, const float* g, __nv_bfloat16* out, int64_t rows, int width,
                        float eps, cudaStream_t s);
// g == nullptr: gather only (no normalisation).
int launch_merge_norm(const __nv_bfloat16* x, const float* g, const ImgInfo* info, const int32_t* cu,
                      int n_images, int64_t T, int width, int m, float eps, __nv_bfloat16* z, int32_t* status,
                      cudaStream_t s);
int launch_scatter(const int64_t* ids, int64_t n, int64_t token, const void* img, int64_t n_img,
                   void* text, int64_t row_bytes, ScatterWs ws, int32_t* status, cudaStream_t s);
int launch_marker_count(const int64_t* ids, int64_t n, int64_t token, int32_t* chunk_count, cudaStream_t s);
int launch_marker_scan(const int32_t* chunk_count, int64_t n_chunks, int64_t expected, int64_t* chunk_base,
                       int32_t* ok_flag, int32_t* status, cudaStream_t s);
int launch_resize_tile(const uint8_t* src, int64_t src_bytes, const ResizeChunk& ch, float* dst, cudaStream_t s);
int launch_expand(const int64_t* ids, int64_t n, int64_t marker, const int64_t* counts, int n_images,
                  int64_t image_token, int64_t* out, ExpandWs ws, int32_t* status, cudaStream_t s);
int launch_pack_gate_up(const void* gate, const void* up, void* dst, int64_t f, int64_t d, cudaStream_t s);
int launch_pack_cols(const void* src, void* dst, int64_t rows, int64_t src_cols, int64_t dst_cols, int mode,
                     int mm, cudaStream_t s);
int launch_f32_to_bf16(const float* x, __nv_bfloat16* y, int64_t n, cudaStream_t s);
int launch_wait_timeout_selftest(long long budget_cycles, int32_t* status, cudaStream_t s);

// 2D tensor map (bf16 or fp32 elements), 128-byte swizzle, box box_outer x box_inner.
bool make_tmap_2d(CUtensorMap* map, const void* ptr, bool fp32, uint64_t inner, uint64_t outer, uint64_t row_bytes,
                  uint32_t box_inner, uint32_t box_outer);
// 2D bf16 tensor map, 128-byte swizzle, box box_outer x box_inner (box_inner * 2 == 128 bytes).
bool make_tmap_2d_bf16(CUtensorMap* map, const void* ptr, uint64_t inner, uint64_t outer, uint64_t row_bytes,
                       uint32_t box_inner, uint32_t box_outer);

int launch_gemm(int epi, const void* a, const void* b, int64_t M, int64_t N, int64_t K, void* c,
                void* c_bf16, const int32_t* pos, const float2* rope, int64_t rope_cols, int32_t* status,
                cudaStream_t s);

// E4M3 x E4M3 -> fp32 GEMM on two-SM pairs (N % 256 == 0, K % 128 == 0): the
// accumulator column n is multiplied by colscale[n]; epilogues BF16, RESID,
// ROPE, and SWIGLU with E4M3 output (values times out_scale).
int launch_gemm_f8(int epi, const void* a, const void* b, const float* colscale, float out_scale, int64_t M,
                   int64_t N, int64_t K, void* c, void* c_bf16, const int32_t* pos, const float2* rope,
                   int64_t rope_cols, int32_t* status, cudaStream_t s);

// f8_scale > 0: `out` is E4M3 holding the attention output times f8_scale; else bf16.
// out_sf != nullptr: `out` is NVFP4 instead -- E2M1 codes [T, heads * 64 / 2] and
// block scales in out_sf -- of the fp32 attention output with global scale f8_scale.
int launch_attention(const __nv_bfloat16* qkv, int64_t T, int heads, const int32_t* cu, const int32_t* qt,
                     int n_blocks, int total_qtiles, void* out, int32_t* status, cudaStream_t s,
                     float f8_scale = 0.f, uint8_t* out_sf = nullptr);
// Per-row E4M3 quantisation of bf16 weight rows for the FP8 tower GEMMs:
// s[r] = amax_r / 448 (1 for a zero row), dst[r, :] = e4m3(src[r, :] / s[r]),
// colscale[r] = act_scale * s[r]. mode 0: row r of src; mode 1: the gate/up
// interleave of pack_gate_up (rows 32j..32j+15 from gate rows 16j.., 32j+16..
// from up rows 16j..; src = gate, src2 = up).
int launch_quant_rows(const void* src, const void* src2, int mode, int64_t rows, int64_t cols, void* dst,
                      float* colscale, float act_scale, cudaStream_t s);

}  // namespace vlm
