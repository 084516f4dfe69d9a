// vlm_scatter_noalloc: the masked scatter without a caller-provided workspace.
//
// vlm_scatter needs scratch memory for its placeholder positions (per-chunk
// counts, their prefix sums and the destination row of every placeholder)
// and takes it from the caller as a workspace. Some callers have no way to
// provide one: a serving engine that hands all free device memory to its own
// pools at start-up (KV cache, activation arena) and does not allow any other
// allocation on the request path, or a plugin host that gives the operator
// only its input and output buffers. This entry point keeps the scratch in a
// fixed-size array in the library's own device memory instead, so the caller
// passes only inputs and outputs and nothing is allocated per call.
//
// The array holds enough for VLM_SCATTER_NOALLOC_MAX_TOKENS ids
// (about 2 MiB); every GPU that loads the library holds it until the process
// exits. All calls share it, so calls that overlap on the GPU (different
// streams, or different host threads on one device) race on it and must be
// serialised by the caller. Each call writes every scratch word before reading
// it, so nothing has to be cleared between calls.
//
// In host code `g_scatter_scratch` names a host-side stand-in, not device
// memory; its device address comes from cudaGetSymbolAddress, looked up by the
// first call made on a device (with that device current) and cached under the
// device and the current context's unique ID. A device reset (or any teardown
// and re-creation of the context) reloads the module at a new address; the new
// context has a new ID, so the next call looks the address up again instead of
// using the stale one.
#include <mutex>

#include "kernels.cuh"

namespace vlm {
namespace {

constexpr int64_t kMaxTokens = VLM_SCATTER_NOALLOC_MAX_TOKENS;
constexpr int64_t kMaxChunks = (kMaxTokens + 255) / 256;
constexpr size_t align256(size_t x) { return (x + 255) / 256 * 256; }
// Layout: ok flag | per-chunk counts | per-chunk bases | destination rows.
constexpr size_t kOffFlag = 0;
constexpr size_t kOffCount = 256;
constexpr size_t kOffBase = kOffCount + align256(kMaxChunks * sizeof(int32_t));
constexpr size_t kOffRows = kOffBase + align256(kMaxChunks * sizeof(int64_t));
constexpr size_t kScratchBytes = kOffRows + kMaxTokens * sizeof(int64_t);

static __device__ __align__(256) uint8_t g_scatter_scratch[kScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_mutex;
struct CachedAddress {
  unsigned long long ctx_id;  // unique ID of the context the address belongs to
  void* addr;
};
CachedAddress g_scratch_addr[kMaxDevices] = {};

using CtxGetCurrentFn = CUresult (*)(CUcontext*);
using CtxGetIdFn = CUresult (*)(CUcontext, unsigned long long*);

// Unique ID of the calling thread's current context (0 when there is none).
int current_context_id(unsigned long long* id) {
  static CtxGetCurrentFn get_current = nullptr;
  static CtxGetIdFn get_id = nullptr;
  if (get_current == nullptr || get_id == nullptr) {
    void* p = nullptr;
    void* q = nullptr;
    cudaDriverEntryPointQueryResult r1, r2;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &r1) != cudaSuccess ||
        r1 != cudaDriverEntryPointSuccess ||
        cudaGetDriverEntryPoint("cuCtxGetId", &q, cudaEnableDefault, &r2) != cudaSuccess ||
        r2 != cudaDriverEntryPointSuccess)
      return VLM_ERR_CUDA;
    get_current = reinterpret_cast<CtxGetCurrentFn>(p);
    get_id = reinterpret_cast<CtxGetIdFn>(q);
  }
  CUcontext ctx = nullptr;
  if (get_current(&ctx) != CUDA_SUCCESS) return VLM_ERR_CUDA;
  *id = 0;
  if (ctx != nullptr && get_id(ctx, id) != CUDA_SUCCESS) return VLM_ERR_CUDA;
  return VLM_OK;
}

// Device address of g_scatter_scratch on the current device and context.
int scratch_address(void** out) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) return VLM_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return VLM_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_mutex);
  unsigned long long id = 0;
  int rc = current_context_id(&id);
  if (rc != VLM_OK) return rc;
  if (id == 0 || g_scratch_addr[dev].addr == nullptr || g_scratch_addr[dev].ctx_id != id) {
    void* p = nullptr;  // the lookup also makes the device's primary context current if none was
    if (cudaGetSymbolAddress(&p, g_scatter_scratch) != cudaSuccess || p == nullptr) return VLM_ERR_CUDA;
    rc = current_context_id(&id);
    if (rc != VLM_OK) return rc;
    if (id == 0) return VLM_ERR_CUDA;
    g_scratch_addr[dev] = CachedAddress{id, p};
  }
  *out = g_scratch_addr[dev].addr;
  return VLM_OK;
}

}  // namespace
}  // namespace vlm

extern "C" int vlm_scatter_noalloc(const int64_t* d_input_ids, int64_t n_tokens, int64_t image_token_id,
                                   const void* d_image_embeds, int64_t n_image_tokens, void* d_text_embeds,
                                   int64_t row_bytes, int32_t* d_status, void* stream) {
  using namespace vlm;
  if (n_tokens < 0 || n_image_tokens < 0 || row_bytes <= 0 || row_bytes % 16) return VLM_ERR_INVALID_ARG;
  if (n_tokens > kMaxTokens) return VLM_ERR_BAD_SHAPE;  // more ids than the fixed scratch holds
  if (n_tokens == 0) return n_image_tokens == 0 ? VLM_OK : VLM_ERR_BAD_SHAPE;
  if (d_input_ids == nullptr || d_text_embeds == nullptr || d_status == nullptr ||
      (n_image_tokens > 0 && d_image_embeds == nullptr))
    return VLM_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(d_image_embeds) | reinterpret_cast<uintptr_t>(d_text_embeds)) & 15)
    return VLM_ERR_INVALID_ARG;
  void* base = nullptr;
  const int rc = scratch_address(&base);
  if (rc != VLM_OK) return rc;
  uint8_t* b = static_cast<uint8_t*>(base);
  ScatterWs ws;
  ws.ok_flag = reinterpret_cast<int32_t*>(b + kOffFlag);
  ws.chunk_count = reinterpret_cast<int32_t*>(b + kOffCount);
  ws.chunk_base = reinterpret_cast<int64_t*>(b + kOffBase);
  ws.dst_rows = reinterpret_cast<int64_t*>(b + kOffRows);
  return launch_scatter(d_input_ids, n_tokens, image_token_id, d_image_embeds, n_image_tokens, d_text_embeds,
                        row_bytes, ws, d_status, static_cast<cudaStream_t>(stream));
}
