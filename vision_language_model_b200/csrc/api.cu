// C-ABI layer: argument validation, workspace layout, and the kernel chains of
// vlm_encode / vlm_merge_project / vlm_scatter (declared in include/vlm.h and
// include/vlm_kernels.h).
#include <algorithm>
#include <climits>
#include <cmath>
#include <atomic>
#include <vector>

#include "../../include/vlm_kernels.h"
#include "gemm_rows.cuh"
#include "kernels.cuh"
#include "nvfp4.cuh"

namespace vlm {

// ---------------------------------------------------------------------------
// Launch bookkeeping and optional per-kernel event timing
// ---------------------------------------------------------------------------
namespace {
std::atomic<int64_t> g_launches{0};
bool g_profile = false;
struct EventRec { int kclass; cudaEvent_t start, stop; };
std::vector<EventRec> g_records;
std::vector<cudaEvent_t> g_pool;
cudaEvent_t g_pending_start = nullptr;

cudaEvent_t take_event() {
  if (!g_pool.empty()) {
    cudaEvent_t e = g_pool.back();
    g_pool.pop_back();
    return e;
  }
  cudaEvent_t e = nullptr;
  cudaEventCreate(&e);
  return e;
}
}  // namespace

void launch_begin(int kclass, cudaStream_t s) {
  (void)kclass;
  g_launches.fetch_add(1, std::memory_order_relaxed);
  if (g_profile) {
    g_pending_start = take_event();
    cudaEventRecord(g_pending_start, s);
  }
}

void launch_end(int kclass, cudaStream_t s) {
  if (g_profile && g_pending_start != nullptr) {
    cudaEvent_t stop = take_event();
    cudaEventRecord(stop, s);
    g_records.push_back({kclass, g_pending_start, stop});
    g_pending_start = nullptr;
  }
}

void note_extra_launches(int n) { g_launches.fetch_add(n, std::memory_order_relaxed); }

thread_local int g_sm_budget = 0;  // set by the entry points for the launches they issue

int sm_budget() {
  const int n = num_sms();
  return g_sm_budget > 0 && g_sm_budget < n ? g_sm_budget : n;
}

SmBudgetScope::SmBudgetScope(int budget) : prev_(g_sm_budget) { g_sm_budget = budget; }
SmBudgetScope::~SmBudgetScope() { g_sm_budget = prev_; }

int num_sms() {
  static int cache[64] = {};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev >= 64) dev = 63;
  if (cache[dev] == 0) {
    int n = 0;
    cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    cache[dev] = n > 0 ? n : 148;
  }
  return cache[dev];
}

namespace {

inline size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// Bump allocator over a caller-provided workspace (sizes only when base == nullptr).
struct Carver {
  uint8_t* base;
  size_t used = 0;
  explicit Carver(void* b) : base(static_cast<uint8_t*>(b)) {}
  template <typename T>
  T* take(size_t count) {
    used = align_up(used, 256);
    T* p = base ? reinterpret_cast<T*>(base + used) : nullptr;
    used += count * sizeof(T);
    return p;
  }
};

int check_config(const vlm_config* c) {
  if (c == nullptr) return VLM_ERR_INVALID_ARG;
  if (c->layers < 0 || c->width <= 0 || c->heads <= 0 || c->head_dim <= 0 || c->mlp <= 0 || c->patch <= 0 ||
      c->merge <= 0 || c->proj_out <= 0 || !(c->rope_theta > 0.f) || !(c->eps >= 0.f))
    return VLM_ERR_INVALID_ARG;
  if (c->norm_after_merge != 0 && c->norm_after_merge != 1) return VLM_ERR_INVALID_ARG;
  if (c->sm_budget < 0) return VLM_ERR_INVALID_ARG;
  if (c->head_dim != 64 || c->heads * c->head_dim != c->width) return VLM_ERR_UNSUPPORTED;
  if (c->width % 256 || c->width > 2048 || c->mlp % 128 || c->proj_out % 256) return VLM_ERR_UNSUPPORTED;
  if (c->patch > 64) return VLM_ERR_UNSUPPORTED;
  return VLM_OK;
}

inline int64_t kpad(int p) { return align_up(static_cast<size_t>(3 * p * p), 64); }

// Host-side per-image tables of a batch.
struct Batch {
  int n = 0;
  int64_t T = 0, Tm = 0;
  int total_qtiles = 0;
  int max_pos = 0;
  int i2c_items = 0;
  std::vector<int32_t> h, w, H, W, tok_off, m_off, qt_off, i2c_off;
  std::vector<int64_t> pix_off;
};

int make_batch(const vlm_config* c, const int32_t* hw, int n, Batch* b) {
  if (hw == nullptr || n <= 0) return VLM_ERR_BAD_SHAPE;
  b->n = n;
  b->h.resize(n); b->w.resize(n); b->H.resize(n); b->W.resize(n);
  b->tok_off.resize(n + 1); b->m_off.resize(n + 1); b->qt_off.resize(n + 1); b->pix_off.resize(n);
  b->i2c_off.resize(n + 1);
  int64_t t = 0, tm = 0, qt = 0, pix = 0, i2c = 0;
  int maxp = 1;
  for (int i = 0; i < n; ++i) {
    const int Hh = hw[2 * i], Ww = hw[2 * i + 1];
    if (Hh <= 0 || Ww <= 0 || Hh % c->patch || Ww % c->patch) return VLM_ERR_BAD_SHAPE;
    const int hp = Hh / c->patch, wp = Ww / c->patch;
    if (hp % c->merge || wp % c->merge) return VLM_ERR_BAD_SHAPE;
    if (hp >= 32768 || wp >= 32768) return VLM_ERR_BAD_SHAPE;
    b->H[i] = Hh; b->W[i] = Ww; b->h[i] = hp; b->w[i] = wp;
    b->tok_off[i] = static_cast<int32_t>(t);
    b->m_off[i] = static_cast<int32_t>(tm);
    b->qt_off[i] = static_cast<int32_t>(qt);
    b->i2c_off[i] = static_cast<int32_t>(i2c);
    b->pix_off[i] = pix;
    i2c += static_cast<int64_t>(hp) * ((wp + kI2cPatches - 1) / kI2cPatches);
    const int64_t L = static_cast<int64_t>(hp) * wp;
    t += L;
    tm += L / (c->merge * c->merge);
    qt += (L + kAttnBQ - 1) / kAttnBQ;
    pix += 3LL * Hh * Ww;
    maxp = std::max(maxp, std::max(hp, wp));
    if (t > (1LL << 31) - 1 || qt > (1LL << 31) - 1) return VLM_ERR_BAD_SHAPE;
  }
  b->tok_off[n] = static_cast<int32_t>(t);
  b->m_off[n] = static_cast<int32_t>(tm);
  b->qt_off[n] = static_cast<int32_t>(qt);
  b->i2c_off[n] = static_cast<int32_t>(i2c);
  b->i2c_items = static_cast<int>(i2c);
  b->T = t;
  b->Tm = tm;
  b->total_qtiles = static_cast<int>(qt);
  b->max_pos = maxp;
  return VLM_OK;
}

// Device tables of a batch, carved from a workspace.
struct BatchDev {
  ImgInfo* info;
  int32_t* cu;
  int32_t* qt;
  int32_t* i2c;
  int32_t* pos;
  float2* rope;
};

BatchDev carve_batch(Carver& cv, const Batch& b, bool with_pos, int head_dim) {
  BatchDev d;
  d.info = cv.take<ImgInfo>(b.n);
  d.cu = cv.take<int32_t>(b.n + 1);
  d.qt = cv.take<int32_t>(b.n + 1);
  d.i2c = with_pos ? cv.take<int32_t>(b.n + 1) : nullptr;
  d.pos = with_pos ? cv.take<int32_t>(b.T) : nullptr;
  d.rope = with_pos ? cv.take<float2>(static_cast<size_t>(b.max_pos) * head_dim / 2) : nullptr;
  return d;
}

int upload_batch(const Batch& b, const BatchDev& d, cudaStream_t s) {
  for (int first = 0; first < b.n; first += kChunk) {
    ImageChunk ch;
    ch.first = first;
    ch.count = std::min(kChunk, b.n - first);
    for (int i = 0; i < ch.count; ++i) {
      ch.h[i] = b.h[first + i]; ch.w[i] = b.w[first + i];
      ch.H[i] = b.H[first + i]; ch.W[i] = b.W[first + i];
      ch.tok_off[i] = b.tok_off[first + i];
      ch.m_off[i] = b.m_off[first + i];
      ch.qt_off[i] = b.qt_off[first + i];
      ch.i2c_off[i] = b.i2c_off[first + i];
      ch.pix_off[i] = b.pix_off[first + i];
    }
    ch.tok_off[ch.count] = b.tok_off[first + ch.count];
    ch.m_off[ch.count] = b.m_off[first + ch.count];
    ch.qt_off[ch.count] = b.qt_off[first + ch.count];
    ch.i2c_off[ch.count] = b.i2c_off[first + ch.count];
    const int rc = launch_setup(ch, d.info, d.cu, d.qt, d.i2c, d.pos, b.n, s);
    if (rc != VLM_OK) return rc;
  }
  return VLM_OK;
}

// Packed tower layout (byte offsets).
struct TowerLayout {
  size_t w_pe, g_pre, layer0, layer_stride;
  size_t wqkv, wo, wgu, wdown, g_attn, g_ffn;  // offsets inside a layer
  size_t total;
};

TowerLayout tower_layout(const vlm_config* c) {
  TowerLayout L;
  const size_t D = c->width, F = c->mlp;
  size_t off = 0;
  L.w_pe = off; off = align_up(off + D * kpad(c->patch) * 2, 256);
  L.g_pre = off; off = align_up(off + D * 4, 256);
  L.layer0 = off;
  size_t lo = 0;
  L.wqkv = lo; lo = align_up(lo + 3 * D * D * 2, 256);
  L.wo = lo; lo = align_up(lo + D * D * 2, 256);
  L.wgu = lo; lo = align_up(lo + 2 * F * D * 2, 256);
  L.wdown = lo; lo = align_up(lo + D * F * 2, 256);
  L.g_attn = lo; lo = align_up(lo + D * 4, 256);
  L.g_ffn = lo; lo = align_up(lo + D * 4, 256);
  L.layer_stride = lo;
  L.total = off + lo * static_cast<size_t>(c->layers);
  return L;
}

// Packed FP8 tower layout (byte offsets): w_pe and g_pre as in the bf16 layout;
// per layer the four GEMM weights as E4M3 (same row orders), their fp32 column
// scales (s_a * s_w[n]) and the two gains.
struct TowerF8Layout {
  size_t w_pe, g_pre, layer0, layer_stride;
  size_t wqkv, wo, wgu, wdown, cs_qkv, cs_o, cs_gu, cs_down, g_attn, g_ffn;
  size_t total;
};

TowerF8Layout tower_f8_layout(const vlm_config* c) {
  TowerF8Layout L;
  const size_t D = c->width, F = c->mlp;
  size_t off = 0;
  L.w_pe = off; off = align_up(off + D * kpad(c->patch) * 2, 256);
  L.g_pre = off; off = align_up(off + D * 4, 256);
  L.layer0 = off;
  size_t lo = 0;
  L.wqkv = lo; lo = align_up(lo + 3 * D * D, 256);
  L.wo = lo; lo = align_up(lo + D * D, 256);
  L.wgu = lo; lo = align_up(lo + 2 * F * D, 256);
  L.wdown = lo; lo = align_up(lo + D * F, 256);
  L.cs_qkv = lo; lo = align_up(lo + 3 * D * 4, 256);
  L.cs_o = lo; lo = align_up(lo + D * 4, 256);
  L.cs_gu = lo; lo = align_up(lo + 2 * F * 4, 256);
  L.cs_down = lo; lo = align_up(lo + D * 4, 256);
  L.g_attn = lo; lo = align_up(lo + D * 4, 256);
  L.g_ffn = lo; lo = align_up(lo + D * 4, 256);
  L.layer_stride = lo;
  L.total = off + lo * static_cast<size_t>(c->layers);
  return L;
}

// fp32(1 / s) of a static activation scale, computed in double.
inline float inv_scale(float s) { return static_cast<float>(1.0 / static_cast<double>(s)); }

// Packed NVFP4 tower layout (byte offsets): w_pe and g_pre as in the bf16
// layout; per layer the four GEMM weights as E2M1 codes (the executed row
// orders: [Wq; Wk; Wv], Wo, gate / up interleaved, W_down) with their block
// scales, the four weight global scales, the four activation global scales
// (device copies of act_scales, the GEMMs' A-operand scales) and the gains.
struct TowerF4Layout {
  size_t w_pe, g_pre, layer0, layer_stride;
  size_t qkv, qkv_sf, o, o_sf, gu, gu_sf, down, down_sf, gw, act, g_attn, g_ffn;
  size_t total;
};

TowerF4Layout tower_f4_layout(const vlm_config* c) {
  TowerF4Layout L;
  const int64_t D = c->width, F = c->mlp;
  size_t off = 0;
  L.w_pe = off; off = align_up(off + D * kpad(c->patch) * 2, 256);
  L.g_pre = off; off = align_up(off + D * 4, 256);
  L.layer0 = off;
  size_t lo = 0;
  L.qkv = lo; lo = align_up(lo + 3 * D * D / 2, 256);
  L.qkv_sf = lo; lo = align_up(lo + nvfp4_sf_bytes(3 * D, D), 256);
  L.o = lo; lo = align_up(lo + D * D / 2, 256);
  L.o_sf = lo; lo = align_up(lo + nvfp4_sf_bytes(D, D), 256);
  L.gu = lo; lo = align_up(lo + 2 * F * D / 2, 256);
  L.gu_sf = lo; lo = align_up(lo + nvfp4_sf_bytes(2 * F, D), 256);
  L.down = lo; lo = align_up(lo + D * F / 2, 256);
  L.down_sf = lo; lo = align_up(lo + nvfp4_sf_bytes(D, F), 256);
  L.gw = lo; lo = align_up(lo + 4 * 4, 256);
  L.act = lo; lo = align_up(lo + 4 * 4, 256);
  L.g_attn = lo; lo = align_up(lo + D * 4, 256);
  L.g_ffn = lo; lo = align_up(lo + D * 4, 256);
  L.layer_stride = lo;
  L.total = off + lo * static_cast<size_t>(c->layers);
  return L;
}

int check_act_scales(const vlm_config* c, const float* act) {
  if (act == nullptr) return VLM_ERR_INVALID_ARG;
  for (int i = 0; i < 4 * c->layers; ++i)
    if (!(act[i] > 0.f) || !(act[i] < 3.0e38f)) return VLM_ERR_INVALID_ARG;
  return VLM_OK;
}

struct ProjLayout { size_t g_proj, w_merge, w1, w2, total; };

ProjLayout proj_layout(const vlm_config* c) {
  ProjLayout L;
  const size_t D = c->width, E = c->proj_out, mm = static_cast<size_t>(c->merge) * c->merge;
  size_t off = 0;
  L.g_proj = off; off = align_up(off + D * 4, 256);
  L.w_merge = off; off = align_up(off + (c->merge > 1 ? D * mm * D * 2 : 0), 256);
  L.w1 = off; off = align_up(off + E * D * 2, 256);
  L.w2 = off; off = align_up(off + E * E * 2, 256);
  L.total = off;
  return L;
}

// Encode workspace layout.
struct EncodeWs {
  BatchDev bd;
  float* x;
  __nv_bfloat16 *xn, *qkv, *attn, *hbuf, *cols;
  size_t used;
};

EncodeWs carve_encode(void* ws, const vlm_config* c, const Batch& b) {
  Carver cv(ws);
  EncodeWs e;
  e.bd = carve_batch(cv, b, true, c->head_dim);
  const size_t T = b.T, D = c->width, F = c->mlp;
  e.x = cv.take<float>(T * D);
  e.xn = cv.take<__nv_bfloat16>(T * D);
  e.qkv = cv.take<__nv_bfloat16>(T * 3 * D);
  e.attn = cv.take<__nv_bfloat16>(T * D);
  const size_t hsz = std::max(T * F, T * static_cast<size_t>(kpad(c->patch)));
  e.hbuf = cv.take<__nv_bfloat16>(hsz);
  e.cols = e.hbuf;  // the patch gather is consumed before the first MLP
  e.used = align_up(cv.used, 256);
  return e;
}

// The NVFP4 encode: the bf16 workspace (its bf16 buffers hold the E2M1 codes
// of the GEMM inputs) plus the block scales of the three quantised inputs.
struct EncodeF4Ws {
  EncodeWs e;
  uint8_t *xn_sf, *attn_sf, *h_sf;
  size_t sf_bytes_d, sf_bytes_f;
  size_t used;
};

EncodeF4Ws carve_encode_f4(void* ws, const vlm_config* c, const Batch& b) {
  EncodeF4Ws f;
  f.e = carve_encode(ws, c, b);
  Carver cv(ws);
  cv.used = f.e.used;
  f.sf_bytes_d = nvfp4_sf_bytes(b.T, c->width);
  f.sf_bytes_f = nvfp4_sf_bytes(b.T, c->mlp);
  f.xn_sf = cv.take<uint8_t>(f.sf_bytes_d);
  f.attn_sf = cv.take<uint8_t>(f.sf_bytes_d);
  f.h_sf = cv.take<uint8_t>(f.sf_bytes_f);
  f.used = align_up(cv.used, 256);
  return f;
}

struct ProjWs {
  BatchDev bd;
  __nv_bfloat16 *z, *y, *g;
  size_t used;
};

ProjWs carve_proj(void* ws, const vlm_config* c, const Batch& b) {
  Carver cv(ws);
  ProjWs p;
  p.bd = carve_batch(cv, b, false, c->head_dim);
  const size_t D = c->width, E = c->proj_out;
  p.z = cv.take<__nv_bfloat16>(b.T * D);  // [T_m, m*m*D] == [T, D] elements
  p.y = c->merge > 1 ? cv.take<__nv_bfloat16>(b.Tm * D) : nullptr;
  p.g = cv.take<__nv_bfloat16>(b.Tm * E);
  p.used = align_up(cv.used, 256);
  return p;
}

ScatterWs carve_scatter(void* ws, int64_t n_tokens, size_t* used) {
  Carver cv(ws);
  const int64_t n_chunks = (n_tokens + 255) / 256;
  ScatterWs s;
  s.ok_flag = cv.take<int32_t>(1);
  s.chunk_count = cv.take<int32_t>(n_chunks);
  s.chunk_base = cv.take<int64_t>(n_chunks);
  s.dst_rows = cv.take<int64_t>(n_tokens);
  if (used) *used = align_up(cv.used, 256);
  return s;
}

inline cudaStream_t as_stream(void* s) { return static_cast<cudaStream_t>(s); }

#define VLM_TRY(expr)             \
  do {                            \
    const int _rc = (expr);       \
    if (_rc != VLM_OK) return _rc; \
  } while (0)

}  // namespace
}  // namespace vlm

using namespace vlm;

extern "C" {

const char* vlm_status_string(int status) {
  switch (status) {
    case VLM_OK: return "VLM_OK";
    case VLM_ERR_INVALID_ARG: return "VLM_ERR_INVALID_ARG";
    case VLM_ERR_BAD_SHAPE: return "VLM_ERR_BAD_SHAPE";
    case VLM_ERR_WORKSPACE: return "VLM_ERR_WORKSPACE";
    case VLM_ERR_COUNT_MISMATCH: return "VLM_ERR_COUNT_MISMATCH";
    case VLM_ERR_TIMEOUT: return "VLM_ERR_TIMEOUT";
    case VLM_ERR_CUDA: return "VLM_ERR_CUDA";
    case VLM_ERR_UNSUPPORTED: return "VLM_ERR_UNSUPPORTED";
    default: return "VLM_ERR_UNKNOWN";
  }
}

int vlm_status_sync(const int32_t* d_status, void* stream) {
  if (d_status == nullptr) return VLM_ERR_INVALID_ARG;
  int32_t h = 0;
  if (cudaMemcpyAsync(&h, d_status, sizeof(h), cudaMemcpyDeviceToHost, as_stream(stream)) != cudaSuccess)
    return VLM_ERR_CUDA;
  if (cudaStreamSynchronize(as_stream(stream)) != cudaSuccess) return VLM_ERR_CUDA;
  return h;
}

int vlm_config_preset(int preset, vlm_config* cfg) {
  if (cfg == nullptr || (preset != 0 && preset != 1)) return VLM_ERR_INVALID_ARG;
  cfg->layers = 24;
  cfg->width = 1024;
  cfg->heads = 16;
  cfg->head_dim = 64;
  cfg->mlp = 4096;
  cfg->patch = preset == 0 ? 14 : 16;
  cfg->merge = preset == 0 ? 2 : 1;
  cfg->proj_out = 5120;
  cfg->image_token_id = 10;
  cfg->rope_theta = 10000.0f;
  cfg->eps = 1e-5f;
  cfg->normalize = 1;
  cfg->norm_after_merge = 0;
  cfg->sm_budget = 0;
  return VLM_OK;
}

int64_t vlm_num_patches(const vlm_config* cfg, const int32_t* image_hw, int n_images) {
  const int rc = check_config(cfg);
  if (rc != VLM_OK) return rc;
  Batch b;
  const int rb = make_batch(cfg, image_hw, n_images, &b);
  return rb != VLM_OK ? rb : b.T;
}

int64_t vlm_num_merged(const vlm_config* cfg, const int32_t* image_hw, int n_images) {
  const int rc = check_config(cfg);
  if (rc != VLM_OK) return rc;
  Batch b;
  const int rb = make_batch(cfg, image_hw, n_images, &b);
  return rb != VLM_OK ? rb : b.Tm;
}

size_t vlm_tower_packed_bytes(const vlm_config* cfg) {
  return check_config(cfg) == VLM_OK ? tower_layout(cfg).total : 0;
}

size_t vlm_projector_packed_bytes(const vlm_config* cfg) {
  return check_config(cfg) == VLM_OK ? proj_layout(cfg).total : 0;
}

int vlm_pack_tower(const vlm_config* cfg, const vlm_tower_weights* w, void* d_packed, size_t packed_bytes,
                   void* stream) {
  VLM_TRY(check_config(cfg));
  if (w == nullptr || d_packed == nullptr || !w->w_pe || !w->g_pre) return VLM_ERR_INVALID_ARG;
  if (cfg->layers > 0 && (!w->wq || !w->wk || !w->wv || !w->wo || !w->w_gate || !w->w_up || !w->w_down ||
                          !w->g_attn || !w->g_ffn))
    return VLM_ERR_INVALID_ARG;  // the per-layer stacks may be empty (null) only without layers
  const TowerLayout L = tower_layout(cfg);
  if (packed_bytes < L.total) return VLM_ERR_WORKSPACE;
  cudaStream_t s = as_stream(stream);
  uint8_t* dst = static_cast<uint8_t*>(d_packed);
  const size_t D = cfg->width, F = cfg->mlp;
  const int p = cfg->patch;
  VLM_TRY(launch_pack_cols(w->w_pe, dst + L.w_pe, D, 3 * p * p, kpad(p), 0, 1, s));
  if (cudaMemcpyAsync(dst + L.g_pre, w->g_pre, D * 4, cudaMemcpyDeviceToDevice, s) != cudaSuccess)
    return VLM_ERR_CUDA;
  for (int l = 0; l < cfg->layers; ++l) {
    uint8_t* ly = dst + L.layer0 + L.layer_stride * l;
    const uint8_t* wq = static_cast<const uint8_t*>(w->wq) + l * D * D * 2;
    const uint8_t* wk = static_cast<const uint8_t*>(w->wk) + l * D * D * 2;
    const uint8_t* wv = static_cast<const uint8_t*>(w->wv) + l * D * D * 2;
    const uint8_t* wo = static_cast<const uint8_t*>(w->wo) + l * D * D * 2;
    const uint8_t* wg = static_cast<const uint8_t*>(w->w_gate) + l * F * D * 2;
    const uint8_t* wu = static_cast<const uint8_t*>(w->w_up) + l * F * D * 2;
    const uint8_t* wd = static_cast<const uint8_t*>(w->w_down) + l * D * F * 2;
    bool ok = cudaMemcpyAsync(ly + L.wqkv, wq, D * D * 2, cudaMemcpyDeviceToDevice, s) == cudaSuccess;
    ok = ok && cudaMemcpyAsync(ly + L.wqkv + D * D * 2, wk, D * D * 2, cudaMemcpyDeviceToDevice, s) == cudaSuccess;
    ok = ok && cudaMemcpyAsync(ly + L.wqkv + 2 * D * D * 2, wv, D * D * 2, cudaMemcpyDeviceToDevice, s) == cudaSuccess;
    ok = ok && cudaMemcpyAsync(ly + L.wo, wo, D * D * 2, cudaMemcpyDeviceToDevice, s) == cudaSuccess;
    ok = ok && cudaMemcpyAsync(ly + L.wdown, wd, D * F * 2, cudaMemcpyDeviceToDevice, s) == cudaSuccess;
    ok = ok && cudaMemcpyAsync(ly + L.g_attn, w->g_attn + l * D, D * 4, cudaMemcpyDeviceToDevice, s) == cudaSuccess;
    ok = ok && cudaMemcpyAsync(ly + L.g_ffn, w->g_ffn + l * D, D * 4, cudaMemcpyDeviceToDevice, s) == cudaSuccess;
    if (!ok) return VLM_ERR_CUDA;
    VLM_TRY(launch_pack_gate_up(wg, wu, ly + L.wgu, F, D, s));
  }
  return VLM_OK;
}

int vlm_pack_projector(const vlm_config* cfg, const vlm_projector_weights* w, void* d_packed,
                       size_t packed_bytes, void* stream) {
  VLM_TRY(check_config(cfg));
  if (w == nullptr || d_packed == nullptr || !w->g_proj || !w->w1 || !w->w2 || (cfg->merge > 1 && !w->w_merge))
    return VLM_ERR_INVALID_ARG;
  const ProjLayout L = proj_layout(cfg);
  if (packed_bytes < L.total) return VLM_ERR_WORKSPACE;
  cudaStream_t s = as_stream(stream);
  uint8_t* dst = static_cast<uint8_t*>(d_packed);
  const size_t D = cfg->width, E = cfg->proj_out;
  const int mm = cfg->merge * cfg->merge;
  bool ok = cudaMemcpyAsync(dst + L.g_proj, w->g_proj, D * 4, cudaMemcpyDeviceToDevice, s) == cudaSuccess;
  ok = ok && cudaMemcpyAsync(dst + L.w1, w->w1, E * D * 2, cudaMemcpyDeviceToDevice, s) == cudaSuccess;
  ok = ok && cudaMemcpyAsync(dst + L.w2, w->w2, E * E * 2, cudaMemcpyDeviceToDevice, s) == cudaSuccess;
  if (!ok) return VLM_ERR_CUDA;
  if (cfg->merge > 1) VLM_TRY(launch_pack_cols(w->w_merge, dst + L.w_merge, D, D * mm, D * mm, 1, mm, s));
  return VLM_OK;
}

size_t vlm_encode_workspace_size(const vlm_config* cfg, const int32_t* image_hw, int n_images) {
  if (check_config(cfg) != VLM_OK) return 0;
  Batch b;
  if (make_batch(cfg, image_hw, n_images, &b) != VLM_OK) return 0;
  return carve_encode(nullptr, cfg, b).used;
}

int vlm_encode(const vlm_config* cfg, const float* pixels, const int32_t* image_hw, int n_images,
               const void* d_packed_tower, void* d_out, void* d_workspace, size_t ws_bytes, int32_t* d_status,
               void* stream) {
  VLM_TRY(check_config(cfg));
  const SmBudgetScope budget(cfg->sm_budget);
  if (pixels == nullptr || d_packed_tower == nullptr || d_out == nullptr || d_workspace == nullptr)
    return VLM_ERR_INVALID_ARG;
  if (reinterpret_cast<uintptr_t>(d_workspace) & 255) return VLM_ERR_INVALID_ARG;
  Batch b;
  VLM_TRY(make_batch(cfg, image_hw, n_images, &b));
  const EncodeWs e = carve_encode(d_workspace, cfg, b);
  if (ws_bytes < e.used) return VLM_ERR_WORKSPACE;
  cudaStream_t s = as_stream(stream);
  const TowerLayout L = tower_layout(cfg);
  const uint8_t* pk = static_cast<const uint8_t*>(d_packed_tower);
  const int64_t T = b.T, D = cfg->width, F = cfg->mlp, kp = kpad(cfg->patch);

  VLM_TRY(upload_batch(b, e.bd, s));
  VLM_TRY(launch_rope_table(cfg->rope_theta, cfg->head_dim, b.max_pos, e.bd.rope, s));
  VLM_TRY(launch_im2col(pixels, e.bd.info, e.bd.cu, e.bd.i2c, b.i2c_items, b.n, T, cfg->patch,
                        static_cast<int>(kp), cfg->normalize, e.cols, s));
  VLM_TRY(launch_gemm(VLM_EPI_F32, e.cols, pk + L.w_pe, T, D, kp, e.x, nullptr, nullptr, nullptr, 0, d_status, s));
  for (int l = 0; l < cfg->layers; ++l) {
    const uint8_t* ly = pk + L.layer0 + L.layer_stride * l;
    const float* g_attn = reinterpret_cast<const float*>(ly + L.g_attn);
    const float* g_ffn = reinterpret_cast<const float*>(ly + L.g_ffn);
    // ln_pre is fused into the first block's attention norm
    const float* g0 = l == 0 ? reinterpret_cast<const float*>(pk + L.g_pre) : nullptr;
    VLM_TRY(launch_rmsnorm(e.x, g0, g_attn, e.xn, T, static_cast<int>(D), cfg->eps, s));
    VLM_TRY(launch_gemm(VLM_EPI_ROPE, e.xn, ly + L.wqkv, T, 3 * D, D, e.qkv, nullptr, e.bd.pos, e.bd.rope, 2 * D,
                        d_status, s));
    VLM_TRY(launch_attention(e.qkv, T, cfg->heads, e.bd.cu, e.bd.qt, b.n, b.total_qtiles, e.attn, d_status, s));
    VLM_TRY(launch_gemm(VLM_EPI_RESID, e.attn, ly + L.wo, T, D, D, e.x, nullptr, nullptr, nullptr, 0, d_status, s));
    VLM_TRY(launch_rmsnorm(e.x, nullptr, g_ffn, e.xn, T, static_cast<int>(D), cfg->eps, s));
    VLM_TRY(launch_gemm(VLM_EPI_SWIGLU, e.xn, ly + L.wgu, T, 2 * F, D, e.hbuf, nullptr, nullptr, nullptr, 0,
                        d_status, s));
    const bool last = l == cfg->layers - 1;
    VLM_TRY(launch_gemm(VLM_EPI_RESID, e.hbuf, ly + L.wdown, T, D, F, e.x, last ? d_out : nullptr, nullptr,
                        nullptr, 0, d_status, s));
  }
  if (cfg->layers == 0) {
    // ln_pre alone: normalise in place, then convert
    VLM_TRY(launch_rmsnorm(e.x, reinterpret_cast<const float*>(pk + L.g_pre),
                           reinterpret_cast<const float*>(pk + L.g_pre), e.xn, T, static_cast<int>(D), cfg->eps, s));
    VLM_TRY(launch_f32_to_bf16(e.x, static_cast<__nv_bfloat16*>(d_out), T * D, s));
  }
  return VLM_OK;
}

size_t vlm_tower_fp8_packed_bytes(const vlm_config* cfg) {
  return check_config(cfg) == VLM_OK ? tower_f8_layout(cfg).total : 0;
}

int vlm_pack_tower_fp8(const vlm_config* cfg, const vlm_tower_weights* w, const float* act_scales, void* d_packed,
                       size_t packed_bytes, void* stream) {
  VLM_TRY(check_config(cfg));
  if (w == nullptr || d_packed == nullptr || !w->w_pe || !w->g_pre) return VLM_ERR_INVALID_ARG;
  if (cfg->layers > 0 && (!w->wq || !w->wk || !w->wv || !w->wo || !w->w_gate || !w->w_up || !w->w_down ||
                          !w->g_attn || !w->g_ffn))
    return VLM_ERR_INVALID_ARG;  // the per-layer stacks may be empty (null) only without layers
  VLM_TRY(check_act_scales(cfg, act_scales));
  if (cfg->mlp % 256 || cfg->width % 256) return VLM_ERR_UNSUPPORTED;
  const TowerF8Layout L = tower_f8_layout(cfg);
  if (packed_bytes < L.total) return VLM_ERR_WORKSPACE;
  cudaStream_t s = as_stream(stream);
  uint8_t* dst = static_cast<uint8_t*>(d_packed);
  const size_t D = cfg->width, F = cfg->mlp;
  const int p = cfg->patch;
  VLM_TRY(launch_pack_cols(w->w_pe, dst + L.w_pe, D, 3 * p * p, kpad(p), 0, 1, s));
  if (cudaMemcpyAsync(dst + L.g_pre, w->g_pre, D * 4, cudaMemcpyDeviceToDevice, s) != cudaSuccess)
    return VLM_ERR_CUDA;
  for (int l = 0; l < cfg->layers; ++l) {
    uint8_t* ly = dst + L.layer0 + L.layer_stride * l;
    const float* act = act_scales + 4 * l;
    auto at = [&](const void* base, size_t elems) { return static_cast<const uint8_t*>(base) + l * elems * 2; };
    float* cs_qkv = reinterpret_cast<float*>(ly + L.cs_qkv);
    VLM_TRY(launch_quant_rows(at(w->wq, D * D), nullptr, 0, D, D, ly + L.wqkv, cs_qkv, act[0], s));
    VLM_TRY(launch_quant_rows(at(w->wk, D * D), nullptr, 0, D, D, ly + L.wqkv + D * D, cs_qkv + D, act[0], s));
    VLM_TRY(launch_quant_rows(at(w->wv, D * D), nullptr, 0, D, D, ly + L.wqkv + 2 * D * D, cs_qkv + 2 * D, act[0], s));
    VLM_TRY(launch_quant_rows(at(w->wo, D * D), nullptr, 0, D, D, ly + L.wo, reinterpret_cast<float*>(ly + L.cs_o),
                              act[1], s));
    VLM_TRY(launch_quant_rows(at(w->w_gate, F * D), at(w->w_up, F * D), 1, 2 * F, D, ly + L.wgu,
                              reinterpret_cast<float*>(ly + L.cs_gu), act[2], s));
    VLM_TRY(launch_quant_rows(at(w->w_down, D * F), nullptr, 0, D, F, ly + L.wdown,
                              reinterpret_cast<float*>(ly + L.cs_down), act[3], s));
    bool ok = cudaMemcpyAsync(ly + L.g_attn, w->g_attn + l * D, D * 4, cudaMemcpyDeviceToDevice, s) == cudaSuccess;
    ok = ok && cudaMemcpyAsync(ly + L.g_ffn, w->g_ffn + l * D, D * 4, cudaMemcpyDeviceToDevice, s) == cudaSuccess;
    if (!ok) return VLM_ERR_CUDA;
  }
  return VLM_OK;
}

int vlm_encode_fp8(const vlm_config* cfg, const float* pixels, const int32_t* image_hw, int n_images,
                   const void* d_packed_tower_fp8, const float* act_scales, void* d_out, void* d_workspace,
                   size_t ws_bytes, int32_t* d_status, void* stream) {
  VLM_TRY(check_config(cfg));
  const SmBudgetScope budget(cfg->sm_budget);
  if (pixels == nullptr || d_packed_tower_fp8 == nullptr || d_out == nullptr || d_workspace == nullptr)
    return VLM_ERR_INVALID_ARG;
  VLM_TRY(check_act_scales(cfg, act_scales));
  if (cfg->mlp % 256 || cfg->width % 256) return VLM_ERR_UNSUPPORTED;
  if (reinterpret_cast<uintptr_t>(d_workspace) & 255) return VLM_ERR_INVALID_ARG;
  Batch b;
  VLM_TRY(make_batch(cfg, image_hw, n_images, &b));
  const EncodeWs e = carve_encode(d_workspace, cfg, b);  // the E4M3 operands fit the bf16 buffers
  if (ws_bytes < e.used) return VLM_ERR_WORKSPACE;
  cudaStream_t s = as_stream(stream);
  const TowerF8Layout L = tower_f8_layout(cfg);
  const uint8_t* pk = static_cast<const uint8_t*>(d_packed_tower_fp8);
  const int64_t T = b.T, D = cfg->width, F = cfg->mlp, kp = kpad(cfg->patch);

  VLM_TRY(upload_batch(b, e.bd, s));
  VLM_TRY(launch_rope_table(cfg->rope_theta, cfg->head_dim, b.max_pos, e.bd.rope, s));
  VLM_TRY(launch_im2col(pixels, e.bd.info, e.bd.cu, e.bd.i2c, b.i2c_items, b.n, T, cfg->patch,
                        static_cast<int>(kp), cfg->normalize, e.cols, s));
  VLM_TRY(launch_gemm(VLM_EPI_F32, e.cols, pk + L.w_pe, T, D, kp, e.x, nullptr, nullptr, nullptr, 0, d_status, s));
  for (int l = 0; l < cfg->layers; ++l) {
    const uint8_t* ly = pk + L.layer0 + L.layer_stride * l;
    const float* act = act_scales + 4 * l;
    auto f32 = [&](size_t off) { return reinterpret_cast<const float*>(ly + off); };
    const float* g0 = l == 0 ? reinterpret_cast<const float*>(pk + L.g_pre) : nullptr;
    VLM_TRY(launch_rmsnorm(e.x, g0, f32(L.g_attn), e.xn, T, static_cast<int>(D), cfg->eps, s, inv_scale(act[0])));
    VLM_TRY(launch_gemm_f8(VLM_EPI_ROPE, e.xn, ly + L.wqkv, f32(L.cs_qkv), 1.f, T, 3 * D, D, e.qkv, nullptr,
                           e.bd.pos, e.bd.rope, 2 * D, d_status, s));
    VLM_TRY(launch_attention(e.qkv, T, cfg->heads, e.bd.cu, e.bd.qt, b.n, b.total_qtiles, e.attn, d_status, s,
                             inv_scale(act[1])));
    VLM_TRY(launch_gemm_f8(VLM_EPI_RESID, e.attn, ly + L.wo, f32(L.cs_o), 1.f, T, D, D, e.x, nullptr, nullptr,
                           nullptr, 0, d_status, s));
    VLM_TRY(launch_rmsnorm(e.x, nullptr, f32(L.g_ffn), e.xn, T, static_cast<int>(D), cfg->eps, s,
                           inv_scale(act[2])));
    VLM_TRY(launch_gemm_f8(VLM_EPI_SWIGLU, e.xn, ly + L.wgu, f32(L.cs_gu), inv_scale(act[3]), T, 2 * F, D, e.hbuf,
                           nullptr, nullptr, nullptr, 0, d_status, s));
    const bool last = l == cfg->layers - 1;
    VLM_TRY(launch_gemm_f8(VLM_EPI_RESID, e.hbuf, ly + L.wdown, f32(L.cs_down), 1.f, T, D, F, e.x,
                           last ? d_out : nullptr, nullptr, nullptr, 0, d_status, s));
  }
  if (cfg->layers == 0) {
    VLM_TRY(launch_rmsnorm(e.x, reinterpret_cast<const float*>(pk + L.g_pre),
                           reinterpret_cast<const float*>(pk + L.g_pre), e.xn, T, static_cast<int>(D), cfg->eps, s));
    VLM_TRY(launch_f32_to_bf16(e.x, static_cast<__nv_bfloat16*>(d_out), T * D, s));
  }
  return VLM_OK;
}

int vlm_patch_embed(const vlm_config* cfg, const float* pixels, const int32_t* image_hw, int n_images,
                    const void* d_packed_tower, float* d_x, void* d_workspace, size_t ws_bytes, int32_t* d_status,
                    void* stream) {
  VLM_TRY(check_config(cfg));
  const SmBudgetScope budget(cfg->sm_budget);
  if (pixels == nullptr || d_packed_tower == nullptr || d_x == nullptr || d_workspace == nullptr)
    return VLM_ERR_INVALID_ARG;
  if (reinterpret_cast<uintptr_t>(d_workspace) & 255) return VLM_ERR_INVALID_ARG;
  Batch b;
  VLM_TRY(make_batch(cfg, image_hw, n_images, &b));
  const EncodeWs e = carve_encode(d_workspace, cfg, b);
  if (ws_bytes < e.used) return VLM_ERR_WORKSPACE;
  cudaStream_t s = as_stream(stream);
  const int64_t T = b.T, D = cfg->width, kp = kpad(cfg->patch);
  // every packed tower layout starts with w_pe at offset 0
  const uint8_t* w_pe = static_cast<const uint8_t*>(d_packed_tower) + tower_layout(cfg).w_pe;
  VLM_TRY(upload_batch(b, e.bd, s));
  VLM_TRY(launch_im2col(pixels, e.bd.info, e.bd.cu, e.bd.i2c, b.i2c_items, b.n, T, cfg->patch,
                        static_cast<int>(kp), cfg->normalize, e.cols, s));
  return launch_gemm(VLM_EPI_F32, e.cols, w_pe, T, D, kp, d_x, nullptr, nullptr, nullptr, 0, d_status, s);
}

size_t vlm_tower_nvfp4_packed_bytes(const vlm_config* cfg) {
  return check_config(cfg) == VLM_OK ? tower_f4_layout(cfg).total : 0;
}

int vlm_pack_tower_nvfp4(const vlm_config* cfg, const vlm_tower_weights* w, const float* act_scales,
                         void* d_packed, size_t packed_bytes, void* stream) {
  VLM_TRY(check_config(cfg));
  if (w == nullptr || d_packed == nullptr || !w->w_pe || !w->g_pre) return VLM_ERR_INVALID_ARG;
  if (cfg->layers > 0 && (!w->wq || !w->wk || !w->wv || !w->wo || !w->w_gate || !w->w_up || !w->w_down ||
                          !w->g_attn || !w->g_ffn))
    return VLM_ERR_INVALID_ARG;
  VLM_TRY(check_act_scales(cfg, act_scales));
  if (cfg->mlp % 256 || cfg->width % 256) return VLM_ERR_UNSUPPORTED;
  if (reinterpret_cast<uintptr_t>(d_packed) & 255) return VLM_ERR_INVALID_ARG;
  const TowerF4Layout L = tower_f4_layout(cfg);
  if (packed_bytes < L.total) return VLM_ERR_WORKSPACE;
  cudaStream_t s = as_stream(stream);
  uint8_t* dst = static_cast<uint8_t*>(d_packed);
  const int64_t D = cfg->width, F = cfg->mlp;
  const int p = cfg->patch;
  constexpr float kFp4Range = 6.0f * 448.0f;  // largest E2M1 value times largest E4M3 block scale
  VLM_TRY(launch_pack_cols(w->w_pe, dst + L.w_pe, D, 3 * p * p, kpad(p), 0, 1, s));
  if (cudaMemcpyAsync(dst + L.g_pre, w->g_pre, D * 4, cudaMemcpyDeviceToDevice, s) != cudaSuccess)
    return VLM_ERR_CUDA;
  for (int l = 0; l < cfg->layers; ++l) {
    uint8_t* ly = dst + L.layer0 + L.layer_stride * l;
    float* gw = reinterpret_cast<float*>(ly + L.gw);
    auto at = [&](const void* base, int64_t elems) { return static_cast<const uint8_t*>(base) + l * elems * 2; };
    // [Wq; Wk; Wv] under one global scale; each part fills whole 128-row scale groups
    const void* qkv_parts[3] = {at(w->wq, D * D), at(w->wk, D * D), at(w->wv, D * D)};
    const int64_t dd[3] = {D * D, D * D, D * D};
    VLM_TRY(launch_amax_scale_multi(qkv_parts, dd, 3, 0, kFp4Range, gw + 0, s));
    for (int j = 0; j < 3; ++j)
      VLM_TRY(launch_quant_nvfp4(qkv_parts[j], 0, D, D, gw + 0, ly + L.qkv + j * D * D / 2,
                                 ly + L.qkv_sf + j * nvfp4_sf_bytes(D, D), s));
    VLM_TRY(launch_amax_scale(at(w->wo, D * D), 0, D * D, kFp4Range, gw + 1, s));
    VLM_TRY(launch_quant_nvfp4(at(w->wo, D * D), 0, D, D, gw + 1, ly + L.o, ly + L.o_sf, s));
    const void* gu_parts[2] = {at(w->w_gate, F * D), at(w->w_up, F * D)};
    const int64_t fd[2] = {F * D, F * D};
    VLM_TRY(launch_amax_scale_multi(gu_parts, fd, 2, 0, kFp4Range, gw + 2, s));
    VLM_TRY(launch_quant_nvfp4_rows(gu_parts[0], gu_parts[1], 0, 2 * F, D, gw + 2, ly + L.gu, ly + L.gu_sf, s));
    VLM_TRY(launch_amax_scale(at(w->w_down, D * F), 0, D * F, kFp4Range, gw + 3, s));
    VLM_TRY(launch_quant_nvfp4(at(w->w_down, D * F), 0, D, F, gw + 3, ly + L.down, ly + L.down_sf, s));
    bool ok = cudaMemcpyAsync(ly + L.act, act_scales + 4 * l, 4 * 4, cudaMemcpyHostToDevice, s) == cudaSuccess;
    ok = ok && cudaMemcpyAsync(ly + L.g_attn, w->g_attn + l * D, D * 4, cudaMemcpyDeviceToDevice, s) == cudaSuccess;
    ok = ok && cudaMemcpyAsync(ly + L.g_ffn, w->g_ffn + l * D, D * 4, cudaMemcpyDeviceToDevice, s) == cudaSuccess;
    if (!ok) return VLM_ERR_CUDA;
  }
  return VLM_OK;
}

size_t vlm_encode_nvfp4_workspace_size(const vlm_config* cfg, const int32_t* image_hw, int n_images) {
  if (check_config(cfg) != VLM_OK) return 0;
  Batch b;
  if (make_batch(cfg, image_hw, n_images, &b) != VLM_OK) return 0;
  return carve_encode_f4(nullptr, cfg, b).used;
}

int vlm_encode_nvfp4(const vlm_config* cfg, const float* pixels, const int32_t* image_hw, int n_images,
                     const void* d_packed_tower_nvfp4, const float* act_scales, void* d_out, void* d_workspace,
                     size_t ws_bytes, int32_t* d_status, void* stream) {
  VLM_TRY(check_config(cfg));
  const SmBudgetScope budget(cfg->sm_budget);
  if (pixels == nullptr || d_packed_tower_nvfp4 == nullptr || d_out == nullptr || d_workspace == nullptr)
    return VLM_ERR_INVALID_ARG;
  VLM_TRY(check_act_scales(cfg, act_scales));
  if (cfg->mlp % 256 || cfg->width % 256) return VLM_ERR_UNSUPPORTED;
  if ((reinterpret_cast<uintptr_t>(d_workspace) & 255) || (reinterpret_cast<uintptr_t>(d_packed_tower_nvfp4) & 255))
    return VLM_ERR_INVALID_ARG;
  Batch b;
  VLM_TRY(make_batch(cfg, image_hw, n_images, &b));
  const EncodeF4Ws f = carve_encode_f4(d_workspace, cfg, b);
  if (ws_bytes < f.used) return VLM_ERR_WORKSPACE;
  const EncodeWs& e = f.e;
  cudaStream_t s = as_stream(stream);
  const TowerF4Layout L = tower_f4_layout(cfg);
  const uint8_t* pk = static_cast<const uint8_t*>(d_packed_tower_nvfp4);
  const int64_t T = b.T, D = cfg->width, F = cfg->mlp, kp = kpad(cfg->patch);
  uint8_t* xn_q = reinterpret_cast<uint8_t*>(e.xn);
  uint8_t* attn_q = reinterpret_cast<uint8_t*>(e.attn);
  uint8_t* h_q = reinterpret_cast<uint8_t*>(e.hbuf);

  // the producers write the scales of real rows only: padding rows keep scale 0
  bool ok = cudaMemsetAsync(f.xn_sf, 0, f.sf_bytes_d, s) == cudaSuccess;
  ok = ok && cudaMemsetAsync(f.attn_sf, 0, f.sf_bytes_d, s) == cudaSuccess;
  ok = ok && cudaMemsetAsync(f.h_sf, 0, f.sf_bytes_f, s) == cudaSuccess;
  if (!ok) return VLM_ERR_CUDA;
  VLM_TRY(upload_batch(b, e.bd, s));
  VLM_TRY(launch_rope_table(cfg->rope_theta, cfg->head_dim, b.max_pos, e.bd.rope, s));
  VLM_TRY(launch_im2col(pixels, e.bd.info, e.bd.cu, e.bd.i2c, b.i2c_items, b.n, T, cfg->patch,
                        static_cast<int>(kp), cfg->normalize, e.cols, s));
  VLM_TRY(launch_gemm(VLM_EPI_F32, e.cols, pk + L.w_pe, T, D, kp, e.x, nullptr, nullptr, nullptr, 0, d_status, s));
  for (int l = 0; l < cfg->layers; ++l) {
    const uint8_t* ly = pk + L.layer0 + L.layer_stride * l;
    const float* act = act_scales + 4 * l;                       // host copies: kernel arguments
    const float* act_d = reinterpret_cast<const float*>(ly + L.act);  // device copies: GEMM A scales
    const float* gw = reinterpret_cast<const float*>(ly + L.gw);
    auto f32 = [&](size_t off) { return reinterpret_cast<const float*>(ly + off); };
    const float* g0 = l == 0 ? reinterpret_cast<const float*>(pk + L.g_pre) : nullptr;
    VLM_TRY(launch_rmsnorm_nvfp4(e.x, g0, f32(L.g_attn), xn_q, f.xn_sf, T, static_cast<int>(D), cfg->eps, act[0], s));
    VLM_TRY(launch_gemm_nvfp4_ex(VLM_EPI_ROPE, xn_q, f.xn_sf, act_d + 0, ly + L.qkv, ly + L.qkv_sf, gw + 0, T, 3 * D,
                                 D, e.qkv, nullptr, 1.f, e.bd.pos, e.bd.rope, 2 * D, d_status, s));
    VLM_TRY(launch_attention(e.qkv, T, cfg->heads, e.bd.cu, e.bd.qt, b.n, b.total_qtiles, attn_q, d_status, s,
                             act[1], f.attn_sf));
    VLM_TRY(launch_gemm_nvfp4(VLM_EPI_RESID, attn_q, f.attn_sf, act_d + 1, ly + L.o, ly + L.o_sf, gw + 1, T, D, D,
                              e.x, d_status, s));
    VLM_TRY(launch_rmsnorm_nvfp4(e.x, nullptr, f32(L.g_ffn), xn_q, f.xn_sf, T, static_cast<int>(D), cfg->eps, act[2],
                                 s));
    VLM_TRY(launch_gemm_nvfp4_ex(VLM_EPI_SWIGLU, xn_q, f.xn_sf, act_d + 2, ly + L.gu, ly + L.gu_sf, gw + 2, T, 2 * F,
                                 D, h_q, f.h_sf, act[3], nullptr, nullptr, 0, d_status, s));
    VLM_TRY(launch_gemm_nvfp4(VLM_EPI_RESID, h_q, f.h_sf, act_d + 3, ly + L.down, ly + L.down_sf, gw + 3, T, D, F,
                              e.x, d_status, s));
  }
  if (cfg->layers == 0)
    VLM_TRY(launch_rmsnorm(e.x, reinterpret_cast<const float*>(pk + L.g_pre),
                           reinterpret_cast<const float*>(pk + L.g_pre), e.xn, T, static_cast<int>(D), cfg->eps, s));
  VLM_TRY(launch_f32_to_bf16(e.x, static_cast<__nv_bfloat16*>(d_out), T * D, s));
  return VLM_OK;
}

namespace {
// The projector up to its last linear ("Mistral 3", Mistral3MultiModalProjector:
// RMSNorm, the 2x2 patch merger, linear_1 + GELU): merge gather (normalising
// each patch unless the norm follows the merge linear), merge linear, W1 with
// GELU into p.g.
int projector_head(const vlm_config* cfg, const void* d_tower_out, const Batch& b, const ProjWs& p, const uint8_t* pk,
                   const ProjLayout& L, int32_t* d_status, cudaStream_t s) {
  const int64_t D = cfg->width, E = cfg->proj_out, mm = static_cast<int64_t>(cfg->merge) * cfg->merge;
  const bool after = cfg->norm_after_merge != 0 && cfg->merge > 1;
  const float* g_proj = reinterpret_cast<const float*>(pk + L.g_proj);
  VLM_TRY(upload_batch(b, p.bd, s));
  VLM_TRY(launch_merge_norm(static_cast<const __nv_bfloat16*>(d_tower_out), after ? nullptr : g_proj, p.bd.info,
                            p.bd.cu, b.n, b.T, static_cast<int>(D), cfg->merge, cfg->eps, p.z, d_status, s));
  const __nv_bfloat16* y = p.z;
  if (cfg->merge > 1) {
    VLM_TRY(launch_gemm(VLM_EPI_BF16, p.z, pk + L.w_merge, b.Tm, D, mm * D, p.y, nullptr, nullptr, nullptr, 0,
                        d_status, s));
    y = p.y;
    if (after) VLM_TRY(launch_rmsnorm_bf16(p.y, g_proj, p.y, b.Tm, static_cast<int>(D), cfg->eps, s));
  }
  return launch_gemm(VLM_EPI_GELU, y, pk + L.w1, b.Tm, E, D, p.g, nullptr, nullptr, nullptr, 0, d_status, s);
}
}  // namespace

size_t vlm_merge_project_workspace_size(const vlm_config* cfg, const int32_t* image_hw, int n_images) {
  if (check_config(cfg) != VLM_OK) return 0;
  Batch b;
  if (make_batch(cfg, image_hw, n_images, &b) != VLM_OK) return 0;
  return carve_proj(nullptr, cfg, b).used;
}

int vlm_merge_project(const vlm_config* cfg, const void* d_tower_out, const int32_t* image_hw, int n_images,
                      const void* d_packed_projector, void* d_out, void* d_workspace, size_t ws_bytes,
                      int32_t* d_status, void* stream) {
  VLM_TRY(check_config(cfg));
  const SmBudgetScope budget(cfg->sm_budget);
  if (d_tower_out == nullptr || d_packed_projector == nullptr || d_out == nullptr || d_workspace == nullptr)
    return VLM_ERR_INVALID_ARG;
  if (reinterpret_cast<uintptr_t>(d_workspace) & 255) return VLM_ERR_INVALID_ARG;
  if (reinterpret_cast<uintptr_t>(d_tower_out) & 15) return VLM_ERR_INVALID_ARG;  // read by bulk copies
  Batch b;
  VLM_TRY(make_batch(cfg, image_hw, n_images, &b));
  const ProjWs p = carve_proj(d_workspace, cfg, b);
  if (ws_bytes < p.used) return VLM_ERR_WORKSPACE;
  cudaStream_t s = as_stream(stream);
  const ProjLayout L = proj_layout(cfg);
  const uint8_t* pk = static_cast<const uint8_t*>(d_packed_projector);
  const int64_t E = cfg->proj_out;
  VLM_TRY(projector_head(cfg, d_tower_out, b, p, pk, L, d_status, s));
  VLM_TRY(launch_gemm(VLM_EPI_BF16, p.g, pk + L.w2, b.Tm, E, E, d_out, nullptr, nullptr, nullptr, 0, d_status, s));
  return VLM_OK;
}

size_t vlm_merge_project_scatter_workspace_size(const vlm_config* cfg, const int32_t* image_hw, int n_images,
                                                int64_t n_tokens) {
  if (check_config(cfg) != VLM_OK || n_tokens <= 0 || n_tokens > (1LL << 40)) return 0;
  Batch b;
  if (make_batch(cfg, image_hw, n_images, &b) != VLM_OK) return 0;
  size_t sc = 0;
  carve_scatter(nullptr, n_tokens, &sc);
  return carve_proj(nullptr, cfg, b).used + sc;
}

int vlm_merge_project_scatter(const vlm_config* cfg, const void* d_tower_out, const int32_t* image_hw, int n_images,
                              const void* d_packed_projector, const int64_t* d_input_ids, int64_t n_tokens,
                              void* d_text_embeds, void* d_workspace, size_t ws_bytes, int32_t* d_status,
                              void* stream) {
  VLM_TRY(check_config(cfg));
  const SmBudgetScope budget(cfg->sm_budget);
  if (d_tower_out == nullptr || d_packed_projector == nullptr || d_input_ids == nullptr || d_text_embeds == nullptr ||
      d_workspace == nullptr || d_status == nullptr)
    return VLM_ERR_INVALID_ARG;
  if (n_tokens <= 0 || n_tokens > (1LL << 40)) return VLM_ERR_BAD_SHAPE;
  if ((reinterpret_cast<uintptr_t>(d_workspace) & 255) ||
      ((reinterpret_cast<uintptr_t>(d_tower_out) | reinterpret_cast<uintptr_t>(d_text_embeds)) & 15))
    return VLM_ERR_INVALID_ARG;
  Batch b;
  VLM_TRY(make_batch(cfg, image_hw, n_images, &b));
  const ProjWs p = carve_proj(d_workspace, cfg, b);
  size_t sc = 0;
  const ScatterWs sw = carve_scatter(static_cast<uint8_t*>(d_workspace) + p.used, n_tokens, &sc);
  if (ws_bytes < p.used + sc) return VLM_ERR_WORKSPACE;
  cudaStream_t s = as_stream(stream);
  const ProjLayout L = proj_layout(cfg);
  const uint8_t* pk = static_cast<const uint8_t*>(d_packed_projector);
  const int64_t E = cfg->proj_out;
  // the placeholders' rows first: on a count mismatch ok_flag stays 0 and the
  // last linear writes nothing
  VLM_TRY(launch_scatter_rows(d_input_ids, n_tokens, cfg->image_token_id, b.Tm, sw, d_status, s));
  VLM_TRY(projector_head(cfg, d_tower_out, b, p, pk, L, d_status, s));
  return launch_gemm_rows(p.g, pk + L.w2, b.Tm, E, E, d_text_embeds, n_tokens, sw.dst_rows, sw.ok_flag, d_status,
                          s);
}

size_t vlm_scatter_workspace_size(int64_t n_tokens) {
  if (n_tokens < 0) return 0;
  size_t used = 0;
  carve_scatter(nullptr, n_tokens, &used);
  return used;
}

int vlm_scatter(const int64_t* d_input_ids, int64_t n_tokens, int64_t image_token_id, const void* d_image_embeds,
                int64_t n_image_tokens, void* d_text_embeds, int64_t row_bytes, void* d_workspace, size_t ws_bytes,
                int32_t* d_status, void* stream) {
  if (n_tokens < 0 || n_image_tokens < 0 || row_bytes <= 0 || row_bytes % 16) return VLM_ERR_INVALID_ARG;
  if (n_tokens == 0) return n_image_tokens == 0 ? VLM_OK : VLM_ERR_BAD_SHAPE;
  if (d_input_ids == nullptr || d_text_embeds == nullptr || d_workspace == nullptr || d_status == nullptr ||
      (n_image_tokens > 0 && d_image_embeds == nullptr))
    return VLM_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(d_image_embeds) | reinterpret_cast<uintptr_t>(d_text_embeds)) & 15)
    return VLM_ERR_INVALID_ARG;
  if (reinterpret_cast<uintptr_t>(d_workspace) & 255) return VLM_ERR_INVALID_ARG;
  if (n_tokens > (1LL << 40)) return VLM_ERR_BAD_SHAPE;
  size_t used = 0;
  const ScatterWs ws = carve_scatter(d_workspace, n_tokens, &used);
  if (ws_bytes < used) return VLM_ERR_WORKSPACE;
  return launch_scatter(d_input_ids, n_tokens, image_token_id, d_image_embeds, n_image_tokens, d_text_embeds,
                        row_bytes, ws, d_status, as_stream(stream));
}

int vlm_resize_target(int32_t height, int32_t width, int32_t longest_edge, int32_t grid, int32_t* out_h,
                      int32_t* out_w) {
  if (out_h == nullptr || out_w == nullptr || height <= 0 || width <= 0 || longest_edge <= 0 || grid <= 0)
    return VLM_ERR_INVALID_ARG;
  // rounding up to the grid must not carry a side past longest_edge
  if (longest_edge % grid) return VLM_ERR_BAD_SHAPE;
  double h = height, w = width;
  const double ratio = static_cast<double>(std::max(height, width)) / static_cast<double>(longest_edge);
  if (ratio > 1.0) {
    h = std::floor(h / ratio);
    w = std::floor(w / ratio);
  }
  const int64_t hh = std::max<int64_t>(static_cast<int64_t>(h), 1), ww = std::max<int64_t>(static_cast<int64_t>(w), 1);
  const int64_t rh = (hh + grid - 1) / grid * grid, rw = (ww + grid - 1) / grid * grid;
  if (rh > (1LL << 30) || rw > (1LL << 30)) return VLM_ERR_BAD_SHAPE;
  *out_h = static_cast<int32_t>(rh);
  *out_w = static_cast<int32_t>(rw);
  return VLM_OK;
}

int vlm_preprocess(const uint8_t* d_src, const int32_t* src_hw, int n_images, const int32_t* out_hw, int32_t tile,
                   float* d_out, void* stream) {
  if (d_src == nullptr || src_hw == nullptr || out_hw == nullptr || d_out == nullptr || n_images <= 0 || tile < 0)
    return VLM_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(d_out) | reinterpret_cast<uintptr_t>(d_src)) & 15) return VLM_ERR_INVALID_ARG;
  if (tile % 4) return VLM_ERR_BAD_SHAPE;
  for (int i = 0; i < n_images; ++i) {
    const int32_t sh = src_hw[2 * i], sw = src_hw[2 * i + 1], oh = out_hw[2 * i], ow = out_hw[2 * i + 1];
    if (sh <= 0 || sw <= 0 || oh <= 0 || ow <= 0 || ow % 4) return VLM_ERR_BAD_SHAPE;
    if (sh > 65536 || sw > 65536 || oh > 32768 || ow > 32768) return VLM_ERR_BAD_SHAPE;
    if (tile > 0 && (oh % tile || ow % tile)) return VLM_ERR_BAD_SHAPE;
  }
  cudaStream_t s = as_stream(stream);
  int64_t src_bytes = 0;
  for (int i = 0; i < n_images; ++i) src_bytes += 3LL * src_hw[2 * i] * src_hw[2 * i + 1];
  int64_t src_off = 0, dst_off = 0;
  for (int first = 0; first < n_images; first += kResizeChunk) {
    ResizeChunk ch;
    ch.count = std::min(kResizeChunk, n_images - first);
    ch.tile = tile;
    ch.wide = 0;
    int64_t units = 0, stage = 0;
    for (int k = 0; k < ch.count; ++k) {
      const int i = first + k;
      const int64_t sh = src_hw[2 * i], sw = src_hw[2 * i + 1], oh = out_hw[2 * i], ow = out_hw[2 * i + 1];
      ch.sh[k] = static_cast<int32_t>(sh); ch.sw[k] = static_cast<int32_t>(sw);
      ch.oh[k] = static_cast<int32_t>(oh); ch.ow[k] = static_cast<int32_t>(ow);
      const int64_t nseg = (ow + kResizeSegMax - 1) / kResizeSegMax;
      const int64_t segw = ((ow + nseg - 1) / nseg + 3) / 4 * 4;
      ch.nseg[k] = static_cast<int32_t>(nseg);
      ch.segw[k] = static_cast<int32_t>(segw);
      ch.sq[k] = static_cast<int32_t>((2 * sw) / (2 * ow));
      ch.sr[k] = static_cast<int32_t>((2 * sw) % (2 * ow));
      ch.inv_den_x[k] = static_cast<float>(1.0 / (2.0 * ow));
      ch.inv_den_y[k] = static_cast<float>(1.0 / (2.0 * oh));
      if ((2 * ow + 1) * sw > INT32_MAX || (2 * oh + 1) * sh > INT32_MAX) ch.wide = 1;
      ch.unit_off[k] = static_cast<int32_t>(units);
      ch.src_off[k] = src_off;
      ch.dst_off[k] = dst_off;
      units += oh * nseg;
      // source columns one segment's taps can touch: floor((segw - 1) sw / ow) + 3
      const int64_t cols = std::min<int64_t>((segw - 1) * sw / ow + 3, sw);
      stage = std::max<int64_t>(stage, (3 * cols + 15 + 15) / 16 * 16);
      src_off += 3 * sh * sw;
      dst_off += 3 * oh * ow;
    }
    ch.unit_off[ch.count] = static_cast<int32_t>(units);
    ch.stage_bytes = stage <= kResizeStageMax ? static_cast<int32_t>(stage) : 0;
    VLM_TRY(launch_resize_tile(d_src, src_bytes, ch, d_out, s));
  }
  return VLM_OK;
}

size_t vlm_expand_placeholders_workspace_size(int64_t n_ids, int n_images) {
  if (n_ids < 0 || n_images < 0) return 0;
  Carver cv(nullptr);
  const int64_t chunks = (n_ids + 255) / 256;
  cv.take<int32_t>(chunks > 0 ? chunks : 1);
  cv.take<int64_t>(chunks > 0 ? chunks : 1);
  cv.take<int64_t>(static_cast<size_t>(n_images) + 1);
  cv.take<int32_t>(1);
  return cv.used;
}

int vlm_expand_placeholders(const int64_t* d_input_ids, int64_t n_ids, int64_t marker_id, const int64_t* counts,
                            int n_images, int64_t image_token_id, int64_t* d_out_ids, int64_t out_capacity,
                            int64_t* out_len, void* d_workspace, size_t ws_bytes, int32_t* d_status, void* stream) {
  if (n_ids == 0 && n_images == 0 && out_len != nullptr) {
    *out_len = 0;
    return VLM_OK;
  }
  if (n_ids <= 0 || n_images < 0 || d_input_ids == nullptr || d_out_ids == nullptr || out_len == nullptr ||
      d_workspace == nullptr || d_status == nullptr || (n_images > 0 && counts == nullptr))
    return VLM_ERR_INVALID_ARG;
  if (reinterpret_cast<uintptr_t>(d_workspace) & 255) return VLM_ERR_INVALID_ARG;
  if (n_ids > (1LL << 40)) return VLM_ERR_BAD_SHAPE;
  int64_t total = n_ids - n_images;
  for (int i = 0; i < n_images; ++i) {
    if (counts[i] < 0 || counts[i] > (1LL << 40)) return VLM_ERR_BAD_SHAPE;
    total += counts[i];
  }
  if (total < 0) return VLM_ERR_BAD_SHAPE;  // more images than ids
  if (total > out_capacity) return VLM_ERR_WORKSPACE;
  if (ws_bytes < vlm_expand_placeholders_workspace_size(n_ids, n_images)) return VLM_ERR_WORKSPACE;
  Carver cv(d_workspace);
  const int64_t chunks = (n_ids + 255) / 256;
  ExpandWs ws;
  ws.chunk_count = cv.take<int32_t>(chunks);
  ws.chunk_base = cv.take<int64_t>(chunks);
  ws.prefix = cv.take<int64_t>(static_cast<size_t>(n_images) + 1);
  ws.ok_flag = cv.take<int32_t>(1);
  *out_len = total;
  return launch_expand(d_input_ids, n_ids, marker_id, counts, n_images, image_token_id, d_out_ids, ws, d_status,
                       as_stream(stream));
}

int64_t vlm_launch_count(void) { return g_launches.load(); }

int vlm_profile_enable(int on) {
  for (auto& r : g_records) {
    g_pool.push_back(r.start);
    g_pool.push_back(r.stop);
  }
  g_records.clear();
  g_profile = on != 0;
  return VLM_OK;
}

int vlm_profile_query(int kclass, int64_t* launches, double* total_ms) {
  if (launches == nullptr || total_ms == nullptr || kclass < 0 || kclass >= KC_COUNT) return VLM_ERR_INVALID_ARG;
  *launches = 0;
  *total_ms = 0.0;
  if (!g_records.empty() && cudaEventSynchronize(g_records.back().stop) != cudaSuccess) return VLM_ERR_CUDA;
  for (const auto& r : g_records) {
    if (r.kclass != kclass) continue;
    float ms = 0.f;
    if (cudaEventElapsedTime(&ms, r.start, r.stop) != cudaSuccess) return VLM_ERR_CUDA;
    *launches += 1;
    *total_ms += ms;
  }
  return VLM_OK;
}

// ---------------------------------------------------------------------------
// Per-kernel entry points (include/vlm_kernels.h)
// ---------------------------------------------------------------------------
int vlm_gemm(int epilogue, const void* d_a, const void* d_b, int64_t M, int64_t N, int64_t K, void* d_c,
             void* d_c_bf16, const int32_t* d_pos, const void* d_rope_table, int64_t rope_cols, int32_t* d_status,
             void* stream) {
  return launch_gemm(epilogue, d_a, d_b, M, N, K, d_c, d_c_bf16, d_pos, static_cast<const float2*>(d_rope_table),
                     rope_cols, d_status, as_stream(stream));
}

int vlm_gemm_fp8(int epilogue, const void* d_a, const void* d_b, const float* d_colscale, float out_scale,
                 int64_t M, int64_t N, int64_t K, void* d_c, void* d_c_bf16, const int32_t* d_pos,
                 const void* d_rope_table, int64_t rope_cols, int32_t* d_status, void* stream) {
  return launch_gemm_f8(epilogue, d_a, d_b, d_colscale, out_scale, M, N, K, d_c, d_c_bf16, d_pos,
                        static_cast<const float2*>(d_rope_table), rope_cols, d_status, as_stream(stream));
}

int vlm_rmsnorm_fp8(float* d_x, const float* d_g0, const float* d_g1, void* d_out, int64_t rows, int width,
                    float eps, float f8_scale, void* stream) {
  if (d_x == nullptr || d_g1 == nullptr || d_out == nullptr || rows < 0 || !(f8_scale > 0.f))
    return VLM_ERR_INVALID_ARG;
  if (rows == 0) return VLM_OK;
  return launch_rmsnorm(d_x, d_g0, d_g1, d_out, rows, width, eps, as_stream(stream), f8_scale);
}

size_t vlm_nvfp4_sf_bytes(int64_t rows, int64_t K) {
  if (rows < 1 || K < 64 || K % 64 != 0 || rows > (1LL << 31) - 1 || K > (1LL << 31) - 1) return 0;
  return static_cast<size_t>(nvfp4_sf_bytes(rows, K));
}

int vlm_amax_scale(const void* d_x, int dtype, int64_t n, float divisor, float* d_out, void* stream) {
  return launch_amax_scale(d_x, dtype, n, divisor, d_out, as_stream(stream));
}

int vlm_quant_nvfp4(const void* d_x, int dtype, int64_t rows, int64_t K, const float* d_sg, void* d_q, void* d_sf,
                    void* stream) {
  return launch_quant_nvfp4(d_x, dtype, rows, K, d_sg, static_cast<uint8_t*>(d_q), static_cast<uint8_t*>(d_sf),
                            as_stream(stream));
}

int vlm_gemm_nvfp4(int epilogue, const void* d_a, const void* d_a_sf, const float* d_ga, const void* d_b,
                   const void* d_b_sf, const float* d_gb, int64_t M, int64_t N, int64_t K, void* d_c,
                   int32_t* d_status, void* stream) {
  return launch_gemm_nvfp4(epilogue, static_cast<const uint8_t*>(d_a), static_cast<const uint8_t*>(d_a_sf), d_ga,
                           static_cast<const uint8_t*>(d_b), static_cast<const uint8_t*>(d_b_sf), d_gb, M, N, K,
                           d_c, d_status, as_stream(stream));
}

int vlm_gemm_nvfp4_ex(int epilogue, const void* d_a, const void* d_a_sf, const float* d_ga, const void* d_b,
                      const void* d_b_sf, const float* d_gb, int64_t M, int64_t N, int64_t K, void* d_c, void* d_c_sf,
                      float out_sg, const int32_t* d_pos, const void* d_rope, int64_t rope_cols, int32_t* d_status,
                      void* stream) {
  return launch_gemm_nvfp4_ex(epilogue, static_cast<const uint8_t*>(d_a), static_cast<const uint8_t*>(d_a_sf), d_ga,
                              static_cast<const uint8_t*>(d_b), static_cast<const uint8_t*>(d_b_sf), d_gb, M, N, K,
                              d_c, static_cast<uint8_t*>(d_c_sf), out_sg, d_pos, static_cast<const float2*>(d_rope),
                              rope_cols, d_status, as_stream(stream));
}

int vlm_rmsnorm_nvfp4(float* d_x, const float* d_g0, const float* d_g1, void* d_q, void* d_sf, int64_t rows,
                      int width, float eps, float s_global, void* stream) {
  if (d_x == nullptr || d_g1 == nullptr || d_q == nullptr || d_sf == nullptr || rows < 0 || !(s_global > 0.f) ||
      !(s_global < 3.0e38f))
    return VLM_ERR_INVALID_ARG;
  if (rows == 0) return VLM_OK;
  return launch_rmsnorm_nvfp4(d_x, d_g0, d_g1, static_cast<uint8_t*>(d_q), static_cast<uint8_t*>(d_sf), rows, width,
                              eps, s_global, as_stream(stream));
}

int vlm_rope_table(float theta, int head_dim, int max_pos, void* d_table, void* stream) {
  if (d_table == nullptr || head_dim != 64 || max_pos <= 0 || !(theta > 0.f)) return VLM_ERR_INVALID_ARG;
  return launch_rope_table(theta, head_dim, max_pos, static_cast<float2*>(d_table), as_stream(stream));
}

size_t vlm_attention_workspace_size(int n_blocks) {
  if (n_blocks <= 0) return 0;
  return align_up(static_cast<size_t>(n_blocks) * sizeof(ImgInfo), 256) + 2 * align_up((n_blocks + 1) * 4, 256);
}

namespace {
int attention_host_blocks(const void* d_qkv, int64_t T, int heads, int head_dim, const int32_t* cu_seqlens,
                          int n_blocks, void* d_out, void* d_workspace, size_t ws_bytes, int32_t* d_status,
                          void* stream, float f8_scale, uint8_t* out_sf) {
  if (d_qkv == nullptr || d_out == nullptr || cu_seqlens == nullptr || d_workspace == nullptr || n_blocks <= 0 ||
      heads <= 0)
    return VLM_ERR_INVALID_ARG;
  if (head_dim != 64) return VLM_ERR_UNSUPPORTED;
  if (ws_bytes < vlm_attention_workspace_size(n_blocks)) return VLM_ERR_WORKSPACE;
  if (cu_seqlens[0] != 0 || cu_seqlens[n_blocks] != T || T > (1LL << 31) - 1) return VLM_ERR_BAD_SHAPE;
  Batch b;
  b.n = n_blocks;
  b.T = T;
  b.h.assign(n_blocks, 1); b.w.assign(n_blocks, 1); b.H.assign(n_blocks, 0); b.W.assign(n_blocks, 0);
  b.tok_off.resize(n_blocks + 1); b.m_off.assign(n_blocks + 1, 0); b.qt_off.resize(n_blocks + 1);
  b.i2c_off.assign(n_blocks + 1, 0);
  b.pix_off.assign(n_blocks, 0);
  int64_t qt = 0;
  for (int i = 0; i < n_blocks; ++i) {
    const int64_t L = static_cast<int64_t>(cu_seqlens[i + 1]) - cu_seqlens[i];
    if (L < 0) return VLM_ERR_BAD_SHAPE;
    b.tok_off[i] = cu_seqlens[i];
    b.w[i] = L > 0 ? static_cast<int32_t>(L) : 1;
    b.qt_off[i] = static_cast<int32_t>(qt);
    qt += (L + kAttnBQ - 1) / kAttnBQ;
  }
  b.tok_off[n_blocks] = cu_seqlens[n_blocks];
  b.qt_off[n_blocks] = static_cast<int32_t>(qt);
  Carver cv(d_workspace);
  BatchDev d;
  d.info = cv.take<ImgInfo>(n_blocks);
  d.cu = cv.take<int32_t>(n_blocks + 1);
  d.qt = cv.take<int32_t>(n_blocks + 1);
  d.i2c = nullptr;
  d.pos = nullptr;
  d.rope = nullptr;
  cudaStream_t s = as_stream(stream);
  VLM_TRY(upload_batch(b, d, s));
  return launch_attention(static_cast<const __nv_bfloat16*>(d_qkv), T, heads, d.cu, d.qt, n_blocks,
                          static_cast<int>(qt), d_out, d_status, s, f8_scale, out_sf);
}
}  // namespace

int vlm_attention(const void* d_qkv, int64_t T, int heads, int head_dim, const int32_t* cu_seqlens, int n_blocks,
                  void* d_out, void* d_workspace, size_t ws_bytes, int32_t* d_status, void* stream) {
  return attention_host_blocks(d_qkv, T, heads, head_dim, cu_seqlens, n_blocks, d_out, d_workspace, ws_bytes,
                               d_status, stream, 0.f, nullptr);
}

int vlm_attention_nvfp4(const void* d_qkv, int64_t T, int heads, int head_dim, const int32_t* cu_seqlens,
                        int n_blocks, void* d_q, void* d_sf, float s_global, void* d_workspace, size_t ws_bytes,
                        int32_t* d_status, void* stream) {
  if (d_sf == nullptr || !(s_global > 0.f) || !(s_global < 3.0e38f)) return VLM_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(d_q) & 15) || (reinterpret_cast<uintptr_t>(d_sf) & 1)) return VLM_ERR_INVALID_ARG;
  return attention_host_blocks(d_qkv, T, heads, head_dim, cu_seqlens, n_blocks, d_q, d_workspace, ws_bytes, d_status,
                               stream, s_global, static_cast<uint8_t*>(d_sf));
}

int vlm_selftest_wait_timeout(int64_t budget_cycles, int32_t* d_status, void* stream) {
  if (d_status == nullptr || budget_cycles <= 0 || budget_cycles > (1LL << 32)) return VLM_ERR_INVALID_ARG;
  return launch_wait_timeout_selftest(budget_cycles, d_status, as_stream(stream));
}

int vlm_debug_build(void) {
#ifdef VLM_DEBUG
  return 1;
#else
  return 0;
#endif
}

int vlm_debug_checks(int32_t* first_failure) {
  if (first_failure == nullptr) return VLM_ERR_INVALID_ARG;
  *first_failure = 0;
#ifdef VLM_DEBUG
  if (cudaDeviceSynchronize() != cudaSuccess) return VLM_ERR_CUDA;
  const int words[4] = {debug_word_small_kernels(true), debug_word_frontend(true), debug_word_attention(true),
                        debug_word_gemm(true)};
  for (int w : words) {
    if (w < 0) return VLM_ERR_CUDA;
    if (w != 0 && *first_failure == 0) *first_failure = w;
  }
  return VLM_OK;
#else
  return VLM_ERR_UNSUPPORTED;
#endif
}

int vlm_debug_selftest_bounds(int32_t* d_buf, int n, void* stream) {
  return launch_debug_selftest(d_buf, n, as_stream(stream));
}

int vlm_rmsnorm(float* d_x, const float* d_g0, const float* d_g1, void* d_out, int64_t rows, int width, float eps,
                void* stream) {
  if (d_x == nullptr || d_g1 == nullptr || d_out == nullptr || rows < 0) return VLM_ERR_INVALID_ARG;
  if (rows == 0) return VLM_OK;
  return launch_rmsnorm(d_x, d_g0, d_g1, d_out, rows, width, eps, as_stream(stream));
}

}  // extern "C"
