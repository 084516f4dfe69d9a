/*
 * vlm.h -- C ABI of the B200 (sm_100a) image half of the Mistral 3 / Pixtral
 * multimodal forward: vision tower, 2x2 patch-merging projector, and the
 * masked scatter of image embeddings into the text-embedding sequence.
 *
 * Sources (web pages, cited by title and section):
 *   [K] "Mistral 3" (KerasFormers): intro; API tables Mistral3Model,
 *       Mistral3VisionModel, Mistral3ImageProcessor; "Several images in one
 *       conversation" (one placeholder run per image).
 *   [P] "Pixtral-12B-2409" (inference-research): vision dimensions, patch 16,
 *       no spatial merge, 1024x1024 tiles (VISION TOKENS).
 *   [I] vllm.cpp issue "Mistral3ForConditionalGeneration ...", section
 *       "What we would contribute", item 2: projector plus masked-scatter merge
 *       into the decoder, gated so text rows stay byte-identical.
 *   [N] NeMo AutoModel mistral3_vlm, Mistral3FP8VLMForConditionalGeneration.forward:
 *       input_ids [B, S], pixel_values, image_sizes.
 *
 * Conventions shared by every call:
 *   - Every pointer named d_* or documented as "device" is CUDA device memory
 *     owned by the caller. The library never allocates, frees or keeps device
 *     memory and never synchronises the stream (except vlm_status_sync).
 *     Host arrays (image_hw) are read during the call only.
 *   - `stream` is a cudaStream_t passed as void* (NULL = legacy default stream).
 *   - A negative return value means the arguments were rejected on the host and
 *     nothing was launched. VLM_OK means the work was enqueued; errors found on
 *     the device (a placeholder-count mismatch, a barrier wait that ran out of
 *     its time budget) are written to the caller's int32 status word d_status
 *     (first error wins; the library never clears it: zero it before a call
 *     sequence) and read back with vlm_status_sync.
 *   - Matrices are row-major. Weights use nn.Linear's [out, in] layout.
 *     bf16 means IEEE bfloat16 with round-to-nearest-even conversions.
 *   - Calls keep no state between them (apart from the optional profiling
 *     counters); concurrent calls on different streams must use different
 *     workspaces.
 */
#ifndef VLM_B200_H
#define VLM_B200_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define VLM_API __attribute__((visibility("default")))
#else
#define VLM_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  VLM_OK = 0,
  VLM_ERR_INVALID_ARG = -1,    /* null pointer, bad config value */
  VLM_ERR_BAD_SHAPE = -2,      /* image off the patch grid / merge grid, empty batch, too many tokens */
  VLM_ERR_WORKSPACE = -3,      /* workspace or packed buffer smaller than the size function returns */
  VLM_ERR_COUNT_MISMATCH = -4, /* device: placeholder count != number of image rows */
  VLM_ERR_TIMEOUT = -5,        /* device: a barrier wait exceeded its time budget */
  VLM_ERR_CUDA = -6,           /* a CUDA runtime call failed */
  VLM_ERR_UNSUPPORTED = -7     /* shape the kernels do not implement (e.g. head_dim != 64) */
} vlm_status;

/* Hyperparameters of the vision side. [K] Mistral3Model: vision_embed_dim
 * (width) 1024, vision_mlp_dim 4096, vision_num_layers 24, vision_num_heads 16,
 * patch_size 14, vision_rope_theta 1e4, spatial_merge_size 2, image_token_id 10,
 * text embed_dim 5120 (proj_out). [P]: patch 16, merge 1.
 * eps: RMSNorm epsilon (reading: 1e-5, the only norm_eps the pages give).
 * normalize: 1 = `pixels` hold raw [0,1] values and the processor's per-channel
 * (x - mean)/std ([K] Mistral3ImageProcessor) is applied while gathering
 * patches; 0 = `pixels` are already normalised.
 * norm_after_merge: 0 = the projector RMSNorm runs per patch before the merge
 * (reading); 1 = the other reading of the pages' order: after the merge
 * linear, on the merged width-vector (same gain). No effect with merge == 1. */
typedef struct {
  int32_t layers, width, heads, head_dim, mlp, patch, merge, proj_out, image_token_id;
  float rope_theta, eps;
  int32_t normalize;
  int32_t norm_after_merge;
  /* SM budget of the calls that take this config (0 = every SM): the
   * persistent GEMMs hold at most this many SMs, and attention is launched in
   * successive grids of at most 2 CTAs per budgeted SM, so that work on other
   * streams keeps the rest of the GPU. Results are bit-identical for every
   * budget; a budget above the SM count means every SM. Negative: rejected. */
  int32_t sm_budget;
} vlm_config;

/* Tower weights, device pointers, stacked over layers (L = cfg.layers,
 * D = width, F = mlp, p = patch):
 *   w_pe   bf16 [D, 3, p, p]  patch-embed conv weight (no bias: reading)
 *   g_pre  fp32 [D]           ln_pre RMSNorm gain
 *   wq, wk, wv, wo bf16 [L, D, D]
 *   w_gate, w_up   bf16 [L, F, D]
 *   w_down         bf16 [L, D, F]
 *   g_attn, g_ffn  fp32 [L, D] pre-attention / pre-MLP RMSNorm gains
 * With layers == 0 the per-layer pointers may be NULL. */
typedef struct {
  const void* w_pe;
  const float* g_pre;
  const void *wq, *wk, *wv, *wo, *w_gate, *w_up, *w_down;
  const float *g_attn, *g_ffn;
} vlm_tower_weights;

/* Projector weights, device pointers (E = proj_out, m = merge):
 *   g_proj  fp32 [D]            RMSNorm gain, applied per patch before the merge (reading)
 *   w_merge bf16 [D, m*m*D]     merge linear; input column c*m*m + dy*m + dx is
 *                               channel c of patch (m*i+dy, m*j+dx) (unfold order).
 *                               Ignored when merge == 1.
 *   w1      bf16 [E, D]; w2 bf16 [E, E]   ([K] Mistral3Model: projector_bias False) */
typedef struct {
  const float* g_proj;
  const void *w_merge, *w1, *w2;
} vlm_projector_weights;

/* Status name for a vlm_status value (static string). */
VLM_API const char* vlm_status_string(int status);

/* Synchronises `stream`, then returns *d_status (an int32 on the device).
 * Returns VLM_ERR_CUDA if the synchronisation itself failed. */
VLM_API int vlm_status_sync(const int32_t* d_status, void* stream);

/* Presets: fills *cfg with [K]'s Mistral 3 vision values (preset 0) or [P]'s
 * Pixtral-12B values (preset 1); normalize = 1. Returns VLM_ERR_INVALID_ARG
 * for an unknown preset. */
VLM_API int vlm_config_preset(int preset, vlm_config* cfg);

/* ---------------------------------------------------------------------------
 * Weight packing (one-time, exact: only copies and reorders values)
 *
 * The packed tower holds per layer: [wq;wk;wv] [3D, D]; wo; gate/up rows
 * interleaved in groups of 16 [2F, D]; w_down; the two gains; plus w_pe
 * zero-padded to [D, Kp] (Kp = 3p^2 rounded up to 64) and g_pre.
 * The packed projector holds g_proj, w_merge with its columns reordered to
 * patch-major (dy*m+dx)*D + c, w1, w2.
 * Returns VLM_ERR_WORKSPACE if packed_bytes is smaller than the size function.
 * ------------------------------------------------------------------------- */
VLM_API size_t vlm_tower_packed_bytes(const vlm_config* cfg);
VLM_API int vlm_pack_tower(const vlm_config* cfg, const vlm_tower_weights* w, void* d_packed,
                   size_t packed_bytes, void* stream);
VLM_API size_t vlm_projector_packed_bytes(const vlm_config* cfg);
VLM_API int vlm_pack_projector(const vlm_config* cfg, const vlm_projector_weights* w, void* d_packed,
                       size_t packed_bytes, void* stream);

/* Number of patches T of a batch, or a negative vlm_status if an image is off
 * the patch grid (H or W not a multiple of p), its patch grid is not a multiple
 * of the merge size, or the batch is empty. image_hw is host int32 [n, 2] of
 * (H, W) in pixels ([N] image_sizes). */
VLM_API int64_t vlm_num_patches(const vlm_config* cfg, const int32_t* image_hw, int n_images);
/* Number of merged tokens T_m = sum_b (h_b/m)(w_b/m), or a negative vlm_status. */
VLM_API int64_t vlm_num_merged(const vlm_config* cfg, const int32_t* image_hw, int n_images);

/* ---------------------------------------------------------------------------
 * vlm_encode -- the vision tower ([K] Mistral3VisionModel: conv patch embed ->
 * RMS pre-norm -> 2D-rotary blocks over a packed variable-resolution patch
 * sequence).
 *
 * pixels: device fp32, the images' [3, H_b, W_b] CHW blocks concatenated in
 *   call order, no padding. A large Pixtral image is passed as its 1024x1024
 *   tiles, each tile one image ([P] VISION TOKENS).
 * image_hw: host int32 [n_images, 2].
 * d_packed_tower: output of vlm_pack_tower.
 * d_out: device bf16 [T, width], patches concatenated image after image,
 *   row-major within an image; the residual stream after the last block (no
 *   final norm: reading).
 * Attention is bidirectional within each image only; RoPE positions restart
 *   at (0,0) in each image (reading).
 * d_workspace: device scratch of at least vlm_encode_workspace_size bytes,
 *   256-byte aligned. Overwritten.
 * ------------------------------------------------------------------------- */
VLM_API size_t vlm_encode_workspace_size(const vlm_config* cfg, const int32_t* image_hw, int n_images);
VLM_API int vlm_encode(const vlm_config* cfg, const float* pixels, const int32_t* image_hw, int n_images,
               const void* d_packed_tower, void* d_out, void* d_workspace, size_t ws_bytes,
               int32_t* d_status, void* stream);

/* ---------------------------------------------------------------------------
 * FP8 tower: the four GEMMs of every block (QKV, O, gate/up, down) on E4M3
 * operands with fp32 accumulation (tcgen05.mma kind::f8f6f4), for the
 * FP8-native deployments the pages describe ([K] intro; [I]). The patch
 * embed, norms, RoPE, attention (bf16 q, k, v) and the residual stream are as
 * in vlm_encode.
 *
 * Quantisation (reading; the pages give no recipe):
 *   - weights per output row: s_w[n] = fp32(amax_n / 448) (1 for a zero row),
 *     q = E4M3(fp32(w / s_w[n])), round to nearest even, saturating;
 *   - activations with one static scale per GEMM input: q = E4M3(fp32(a) *
 *     fp32(1 / s_a)); act_scales is host fp32 [layers][4] = the scales of the
 *     attention-norm output, the attention output, the MLP-norm output and the
 *     gated hidden state, each > 0;
 *   - acc[m, n] * fp32(s_a * s_w[n]) dequantises a GEMM result.
 *
 * vlm_pack_tower_fp8: quantises the bf16 weights of vlm_tower_weights (same
 *   meaning as for vlm_pack_tower) into d_packed (device, at least
 *   vlm_tower_fp8_packed_bytes) with the given act_scales.
 * vlm_encode_fp8: vlm_encode with the packed FP8 tower; act_scales must be the
 *   array the tower was packed with. Workspace: vlm_encode_workspace_size.
 * Requires width % 256 == 0 and mlp % 256 == 0 (else VLM_ERR_UNSUPPORTED).
 * ------------------------------------------------------------------------- */
VLM_API size_t vlm_tower_fp8_packed_bytes(const vlm_config* cfg);
VLM_API int vlm_pack_tower_fp8(const vlm_config* cfg, const vlm_tower_weights* w, const float* act_scales,
                               void* d_packed, size_t packed_bytes, void* stream);
VLM_API int vlm_encode_fp8(const vlm_config* cfg, const float* pixels, const int32_t* image_hw, int n_images,
                           const void* d_packed_tower_fp8, const float* act_scales, void* d_out, void* d_workspace,
                           size_t ws_bytes, int32_t* d_status, void* stream);

/* ---------------------------------------------------------------------------
 * vlm_encode_nvfp4 -- vlm_encode with the four tower GEMMs (QKV, O, gate/up,
 * down) on NVFP4 operands (E2M1 values, one E4M3 scale per 16 values of a
 * row along K, one fp32 global scale per tensor) with fp32 accumulation
 * (tcgen05.mma kind::mxf4nvf4, block16), for the NVFP4 checkpoints the
 * deployments load ([I] "Why this one is smaller than it looks", the
 * quantisation loaders). Patch embed, norms, RoPE, attention (bf16 q, k, v)
 * and the residual stream are as in vlm_encode.
 *
 * Quantisation (reading; the pages name the format, not a recipe):
 *   - a block of 16 fp32 values x with global scale s_g:
 *     s_b = E4M3(fp32(amax_b / fp32(6 s_g))), q = E2M1(fp32(x *
 *     fp32(1 / fp32(s_b s_g)))) (q = 0 when s_b is 0), each rounding to
 *     nearest even with saturation;
 *   - weights: s_g = fp32(amax(W) / 2688) over the weight the GEMM executes
 *     ([Wq; Wk; Wv] and [W_gate; W_up] as one tensor each);
 *   - activations: one static s_g per GEMM input, block scales from the data;
 *     act_scales is host fp32 [layers][4] = the global scales of the
 *     attention-norm output, the attention output, the MLP-norm output and
 *     the gated hidden state, each > 0; every input is quantised from fp32
 *     inside the kernel that produces it;
 *   - a GEMM result is acc * fp32(s_g(A) * s_g(W)).
 *
 * vlm_pack_tower_nvfp4: quantises the bf16 weights of vlm_tower_weights (same
 *   meaning as for vlm_pack_tower) into d_packed (device, 256-byte aligned, at
 *   least vlm_tower_nvfp4_packed_bytes) and stores act_scales beside them.
 * vlm_encode_nvfp4: act_scales must be the array the tower was packed with.
 *   d_workspace: 256-byte aligned, at least vlm_encode_nvfp4_workspace_size.
 * Requires width % 256 == 0 and mlp % 256 == 0 (else VLM_ERR_UNSUPPORTED).
 * ------------------------------------------------------------------------- */
VLM_API size_t vlm_tower_nvfp4_packed_bytes(const vlm_config* cfg);
VLM_API int vlm_pack_tower_nvfp4(const vlm_config* cfg, const vlm_tower_weights* w, const float* act_scales,
                                 void* d_packed, size_t packed_bytes, void* stream);
VLM_API size_t vlm_encode_nvfp4_workspace_size(const vlm_config* cfg, const int32_t* image_hw, int n_images);
VLM_API int vlm_encode_nvfp4(const vlm_config* cfg, const float* pixels, const int32_t* image_hw, int n_images,
                             const void* d_packed_tower_nvfp4, const float* act_scales, void* d_out,
                             void* d_workspace, size_t ws_bytes, int32_t* d_status, void* stream);

/* ---------------------------------------------------------------------------
 * vlm_merge_project -- the patch-merging projector ([K] Mistral3Model: 2x2
 * patch-merging projector, spatial_merge_size, projector_bias False):
 * RMSNorm per patch, m x m unfold + concat, merge linear (m*m*D -> D), then
 * W1 (D -> E), exact GELU, W2 (E -> E). With merge == 1 ([P]) the unfold and
 * merge linear are skipped.
 *
 * d_tower_out: device bf16 [T, width] from vlm_encode with the same image_hw,
 *   16-byte aligned (VLM_ERR_INVALID_ARG otherwise).
 * d_out: device bf16 [T_m, proj_out], merged tokens row-major per image,
 *   images concatenated.
 * ------------------------------------------------------------------------- */
VLM_API size_t vlm_merge_project_workspace_size(const vlm_config* cfg, const int32_t* image_hw, int n_images);
VLM_API int vlm_merge_project(const vlm_config* cfg, const void* d_tower_out, const int32_t* image_hw,
                      int n_images, const void* d_packed_projector, void* d_out, void* d_workspace,
                      size_t ws_bytes, int32_t* d_status, void* stream);

/* ---------------------------------------------------------------------------
 * vlm_scatter -- masked scatter ([I] item 2; [K] image_token_id 10 and
 * "Several images in one conversation"): the k-th position i (in order) with
 * input_ids[i] == image_token_id receives row k of image_embeds; all other
 * rows of text_embeds are left untouched (bit-identical).
 *
 * d_input_ids: device int64 [n_tokens] ([N] input_ids [B, S], flattened).
 * d_image_embeds: device, n_image_tokens rows of row_bytes bytes.
 * d_text_embeds: device, n_tokens rows of row_bytes bytes, updated in place.
 * row_bytes: bytes per row (e.g. 5120 * 2 for bf16), a multiple of 16.
 * If the number of placeholders differs from n_image_tokens the call writes
 *   no row and sets *d_status = VLM_ERR_COUNT_MISMATCH.
 * d_workspace: at least vlm_scatter_workspace_size(n_tokens) bytes.
 * ------------------------------------------------------------------------- */
VLM_API size_t vlm_scatter_workspace_size(int64_t n_tokens);
VLM_API int vlm_scatter(const int64_t* d_input_ids, int64_t n_tokens, int64_t image_token_id,
                const void* d_image_embeds, int64_t n_image_tokens, void* d_text_embeds,
                int64_t row_bytes, void* d_workspace, size_t ws_bytes, int32_t* d_status,
                void* stream);

/* ---------------------------------------------------------------------------
 * vlm_merge_project_scatter -- vlm_merge_project followed by vlm_scatter in
 * one call, without the [T_m, proj_out] embedding buffer between them: the
 * projector's last linear (W2) writes each merged token's row straight to its
 * placeholder row of text_embeds ([K] Mistral3Model: the image features
 * replace the image_token_id positions of the token embeddings; [I] item 2).
 *
 * The rows written are bit-identical to those that vlm_merge_project followed
 * by vlm_scatter(d_input_ids, n_tokens, cfg->image_token_id, ...) would write;
 * all other rows of text_embeds are left untouched.
 *
 * d_tower_out, image_hw, n_images, d_packed_projector: as for
 *   vlm_merge_project.
 * d_input_ids: device int64 [n_tokens]; the placeholder is
 *   cfg->image_token_id; n_tokens >= 1 (VLM_ERR_BAD_SHAPE otherwise).
 * d_text_embeds: device bf16 [n_tokens, proj_out], 16-byte aligned, updated in
 *   place.
 * If the number of placeholders differs from T_m (vlm_num_merged) the call
 *   writes no row and sets *d_status = VLM_ERR_COUNT_MISMATCH.
 * d_workspace: 256-byte aligned, at least
 *   vlm_merge_project_scatter_workspace_size(cfg, image_hw, n_images,
 *   n_tokens) bytes (VLM_ERR_WORKSPACE otherwise). Host-side argument errors
 *   are returned before anything is launched.
 * ------------------------------------------------------------------------- */
VLM_API size_t vlm_merge_project_scatter_workspace_size(const vlm_config* cfg, const int32_t* image_hw,
                                                        int n_images, int64_t n_tokens);
VLM_API int vlm_merge_project_scatter(const vlm_config* cfg, const void* d_tower_out, const int32_t* image_hw,
                                      int n_images, const void* d_packed_projector, const int64_t* d_input_ids,
                                      int64_t n_tokens, void* d_text_embeds, void* d_workspace, size_t ws_bytes,
                                      int32_t* d_status, void* stream);

/* ---------------------------------------------------------------------------
 * vlm_scatter_noalloc -- vlm_scatter for callers that cannot allocate device
 * memory. The pages have no counterpart: this is a library convenience.
 *
 * vlm_scatter takes its scratch (placeholder counts and destination rows) from
 * a caller workspace. A serving engine that gives all free device memory to
 * its own pools at start-up, or a plugin host that passes an operator only its
 * input and output buffers, has no workspace to offer. This entry point keeps
 * that scratch in a fixed array inside the library's device memory (about
 * 2 MiB, held on every GPU that loads the library until the process exits),
 * so the caller passes only inputs and outputs; no call allocates or frees
 * anything.
 *
 * Arguments, layouts, results and device-side errors are those of vlm_scatter.
 * n_tokens above VLM_SCATTER_NOALLOC_MAX_TOKENS returns VLM_ERR_BAD_SHAPE
 * before anything is launched.
 * All calls share the one array: calls that overlap on the GPU (other streams,
 * other host threads on the same device) race and must be serialised by the
 * caller. Each call writes all the scratch it reads, so nothing carries over.
 * The first call on a device looks up the array's device address
 * (cudaGetSymbolAddress, with that device current) and caches it under the
 * device and its current context; make that first call before any stream
 * capture begins. After a device reset the first call in the new context
 * looks the address up again (so it, too, belongs before any capture).
 * ------------------------------------------------------------------------- */
#define VLM_SCATTER_NOALLOC_MAX_TOKENS 262144
VLM_API int vlm_scatter_noalloc(const int64_t* d_input_ids, int64_t n_tokens, int64_t image_token_id,
                                const void* d_image_embeds, int64_t n_image_tokens, void* d_text_embeds,
                                int64_t row_bytes, int32_t* d_status, void* stream);

/* ---------------------------------------------------------------------------
 * Image front end: the steps just before the path ([K] intro and
 * Mistral3ImageProcessor: the processor scales an image down until its longer
 * side is at most longest_edge = 1540, with both sides kept on the patch grid;
 * [P] VISION TOKENS: a large image is cut into 1024x1024 tiles).
 *
 * vlm_resize_target (host only, launches nothing): the processor's resize
 *   size. Reading (the pages give no formula): when max(H, W) > longest_edge
 *   both sides are divided by r = max(H, W) / longest_edge (in double) and
 *   floored; images are never enlarged by this step; then each side is rounded
 *   up to a multiple of `grid` (patch * merge, so the 2x2 merge always finds
 *   whole blocks: 28 for [K]; the tile size 1024 for [P]'s tiling).
 *   Both sides then stay within longest_edge, which must itself be a
 *   multiple of grid: any other longest_edge returns VLM_ERR_BAD_SHAPE (a
 *   side rounded up could pass it).
 *   Returns VLM_ERR_INVALID_ARG for a non-positive argument.
 *
 * vlm_preprocess: bilinear resize of decoded images onto out_hw.
 *   d_src: device uint8, the images' [H_b, W_b, 3] RGB (HWC, interleaved)
 *     blocks concatenated in call order, no padding.
 *   src_hw, out_hw: host int32 [n_images, 2] source and output (H, W);
 *     every output width a multiple of 4.
 *   tile: 0, or the tile edge (a multiple of 4 dividing every output H and W).
 *   d_out: device fp32, 16-byte aligned; per image [3, oh, ow] CHW in call
 *     order, values u8 / 255 in [0, 1] (reading: [K]'s mean/std are in these
 *     units); with tile > 0 each image is instead written as its
 *     (oh/tile)(ow/tile) tiles, row-major over the tile grid, each a
 *     [3, tile, tile] block -- exactly the `pixels` vlm_encode takes with
 *     every tile listed as one (tile, tile) image.
 *   Resampling (reading: the pages name no filter): output pixel (y, x)
 *   samples the source at ((y + 1/2) H / oh - 1/2, (x + 1/2) W / ow - 1/2),
 *   clamped to the image, interpolating the 4 neighbours; no antialiasing.
 *   Host-side errors only (VLM_ERR_BAD_SHAPE for a size rule above).
 * ------------------------------------------------------------------------- */
VLM_API int vlm_resize_target(int32_t height, int32_t width, int32_t longest_edge, int32_t grid, int32_t* out_h,
                              int32_t* out_w);
VLM_API int vlm_preprocess(const uint8_t* d_src, const int32_t* src_hw, int n_images, const int32_t* out_hw,
                           int32_t tile, float* d_out, void* stream);

/* ---------------------------------------------------------------------------
 * vlm_expand_placeholders -- the step between the projector and the scatter
 * ([K] "Several images in one conversation": each image's marker in the
 * prompt becomes as many image_token_id positions as that image has merged
 * tokens).
 *
 * d_input_ids: device int64 [n_ids] holding one marker_id per image, in
 *   image order.
 * counts: host int64 [n_images], the merged-token count of each image
 *   ((H/p/m)(W/p/m) for an image on the grid).
 * d_out_ids: device int64, capacity out_capacity; receives the expanded ids:
 *   the k-th marker replaced by counts[k] copies of image_token_id, every
 *   other id copied in order.
 * *out_len (host) is set to n_ids - n_images + sum(counts) before anything
 *   is launched; VLM_ERR_WORKSPACE if that exceeds out_capacity.
 * If the number of markers on the device differs from n_images, nothing is
 *   written and *d_status = VLM_ERR_COUNT_MISMATCH.
 * n_ids == 0 with n_images == 0 sets *out_len = 0 and launches nothing.
 * d_workspace: 256-byte aligned, at least
 *   vlm_expand_placeholders_workspace_size(n_ids, n_images) bytes.
 * ------------------------------------------------------------------------- */
VLM_API size_t vlm_expand_placeholders_workspace_size(int64_t n_ids, int n_images);
VLM_API int vlm_expand_placeholders(const int64_t* d_input_ids, int64_t n_ids, int64_t marker_id,
                                    const int64_t* counts, int n_images, int64_t image_token_id,
                                    int64_t* d_out_ids, int64_t out_capacity, int64_t* out_len,
                                    void* d_workspace, size_t ws_bytes, int32_t* d_status, void* stream);

/* ---------------------------------------------------------------------------
 * Instrumentation (host-side, not thread-safe)
 * ------------------------------------------------------------------------- */
/* Total kernels this library has launched in the process. */
VLM_API int64_t vlm_launch_count(void);
/* Turns per-kernel CUDA-event timing on (1) or off (0) and clears it. */
VLM_API int vlm_profile_enable(int on);
/* Kernel classes: 0 GEMM, 1 attention, 2 RMSNorm, 3 patch gather, 4 merge
 * gather, 5 scatter, 6 index setup, 7 weight packing, 8 image resize,
 * 9 placeholder expansion. Synchronises on the last
 * recorded event, then returns the launches and summed device milliseconds
 * recorded for `kclass` since profiling was enabled. */
VLM_API int vlm_profile_query(int kclass, int64_t* launches, double* total_ms);

#ifdef __cplusplus
}
#endif

#endif /* VLM_B200_H */
