// Persistent tcgen05 GEMM for sm_100a: acc[M, N] = A[M, K] . B[N, K]^T with
// bf16 operands and fp32 accumulation in tensor memory, followed by a fused
// epilogue (bf16 / fp32 store, fp32 residual update, SiLU-gated product, 2D
// RoPE, GELU).
//
// CTA = 6 warps:
//   warp 0      TMA producer (one thread): A and B k-blocks into a STAGES-deep
//               shared-memory ring of 128-byte-swizzled tiles.
//   warp 1      allocates TMEM; one thread issues tcgen05.mma (M=128, N=BN,
//               K=16 per instruction) and commits to mbarriers.
//   warps 2..5  epilogue: tcgen05.ld of the accumulator (warp w owns TMEM
//               lanes = tile rows 32*(w%4)..+31), math, then each warp stages
//               128-byte row chunks of its 32 rows in swizzled shared memory
//               and writes them with TMA bulk tensor stores (rows past M are
//               clipped by the tensor map). The fp32 residual of the RESID
//               epilogue is read with coalesced loads, one chunk ahead.
// Two TMEM accumulators (2 x BN columns) let the epilogue of tile i overlap the
// MMAs of tile i+1. Tiles are handed out statically (tile += gridDim.x) over a
// grid of one CTA per SM. No TMA multicast is used.
//
// Variants further down: gemm_pair_kernel, the same design on two-SM pairs
// (cta_group::2, 256-row tiles) with bf16 or E4M3 operands, and
// gemm_nvfp4_pair_kernel, the pair design on NVFP4 operands with block scales
// copied into TMEM.
#include <cudaTypedefs.h>

#define VLM_DEBUG_FILE_ID 4

#include "gemm_rows.cuh"
#include "kernels.cuh"
#include "nvfp4.cuh"

namespace vlm {

VLM_DEBUG_UNIT(debug_word_gemm)

namespace {

constexpr int GBM = 128;
constexpr int GBK = 64;
constexpr int kEpiWarps = 4;
constexpr int kStageBufBytes = 32 * 128;  // one epilogue warp's 32 rows x 128 bytes
constexpr int kStageBufs = 2;             // per epilogue warp (store of chunk i overlaps chunk i+1)

struct GemmArgs {
  int M, N, K;
  int m_tiles, n_tiles;
  void* c;
  __nv_bfloat16* c_bf16;
  const int32_t* pos;
  const float2* rope;
  int rope_cols;
  int32_t* status;
  const float* colscale;  // E4M3 operands: per-output-column dequantisation factor (s_a * s_w[n])
  float out_scale;        // E4M3 output (SwiGLU): values are multiplied by this before rounding
  const float* g_a = nullptr;  // NVFP4 operands: the two global scales (device memory); the
  const float* g_b = nullptr;  // epilogue multiplies by fp32(g_a * g_b)
  uint8_t* c_sf = nullptr;     // NVFP4 output (SwiGLU): block scales; out_scale is its global scale
  const int64_t* dst_rows = nullptr;  // row-scattered store: destination row of each output row
  const int32_t* ok_flag = nullptr;   // row-scattered store: nothing is written while *ok_flag == 0
  int64_t c_rows = 0;                 // row-scattered store: rows of the destination table
};

template <int BN>
struct GemmShape {
  static constexpr int STAGES = BN == 256 ? 4 : 6;
  static constexpr int A_BYTES = GBM * GBK * 2;
  static constexpr int B_BYTES = BN * GBK * 2;
  static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
  static constexpr int EPI_BYTES = kEpiWarps * kStageBufs * kStageBufBytes;
  static constexpr int TMEM_COLS = 2 * BN;
  static constexpr int BAR_BYTES = 256;
  static constexpr int SMEM_BYTES = STAGES * STAGE_BYTES + EPI_BYTES + BAR_BYTES + 1024;
};

// One epilogue warp's pair of staging buffers and its TMA-store bookkeeping.
struct Stager {
  uint8_t* base;
  const CUtensorMap* map;
  int cur;
  int lane;

  // Buffer for the next chunk; the bulk store that last read it has finished.
  __device__ __forceinline__ uint8_t* acquire() {
    if (lane == 0) bulk_wait_read<kStageBufs - 1>();
    __syncwarp();
    return base + cur * kStageBufBytes;
  }
  // This lane's 128-byte row (row = lane) into the 128-byte-swizzled buffer.
  __device__ __forceinline__ void write_row(uint8_t* buf, const uint32_t (&w)[32]) const {
    uint4* r = reinterpret_cast<uint4*>(buf + lane * 128);
#pragma unroll
    for (int j = 0; j < 8; ++j) r[j ^ (lane & 7)] = make_uint4(w[4 * j], w[4 * j + 1], w[4 * j + 2], w[4 * j + 3]);
  }
  // Stores the buffer's 32 rows at element (x, y) of the output tensor, or
  // (reduce) adds them to what is there.
  template <bool kReduce = false>
  __device__ __forceinline__ void commit(uint8_t* buf, int x, int y) {
    fence_proxy_async_smem();
    __syncwarp();
    if (lane == 0) {
      if constexpr (kReduce) {
        tma_reduce_add_2d(map, smem_u32(buf), x, y);
      } else {
        tma_store_2d(map, smem_u32(buf), x, y);
      }
      bulk_commit();
    }
    cur ^= 1;
  }
  __device__ __forceinline__ void drain() {
    if (lane == 0) bulk_wait<0>();
    __syncwarp();
  }
};

// silu(z) = z / (1 + e^-z) with MUFU ex2 and rcp (about 1 ulp each); z -> -inf gives -0.
__device__ __forceinline__ float silu_f(float z) {
  float e, r;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(e) : "f"(z * -1.4426950408889634f));
  asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(1.0f + e));
  return z * r;
}
// silu(z) = z * sigmoid(z) with sigmoid(z) = (1 + tanh(z / 2)) / 2: one MUFU
// operation (tanh.approx, absolute error about 2^-11) instead of ex2 and rcp.
// For the NVFP4 SwiGLU epilogue only, whose output is rounded to E2M1 next:
// an error of 2^-11 |z| is far below a block's quantisation step.
__device__ __forceinline__ float silu_tanh_f(float z) {
  float t;
  asm("tanh.approx.f32 %0, %1;" : "=f"(t) : "f"(0.5f * z));
  return z * fmaf(0.5f, t, 0.5f);
}
__device__ __forceinline__ float gelu_f(float z) { return 0.5f * z * (1.0f + erff(z * 0.70710678118654752f)); }

template <int EPI>
__device__ __forceinline__ float act(float v) {
  if constexpr (EPI == VLM_EPI_GELU) return gelu_f(v);
  return v;
}

// 32 consecutive column scales (the same for every lane: broadcast loads).
__device__ __forceinline__ void load_cs32(const float* p, float (&cs)[32]) {
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    const float4 v = __ldg(reinterpret_cast<const float4*>(p) + j);
    cs[4 * j] = v.x; cs[4 * j + 1] = v.y; cs[4 * j + 2] = v.z; cs[4 * j + 3] = v.w;
  }
}

// Epilogue of one 128 x BN tile: this warp's 32 rows (row0 = first of them;
// this lane's row is row0 + lane), accumulator columns at TMEM address tbase.
// kF8: the accumulator holds sums of E4M3 products; every column is first
// multiplied by its colscale (SwiGLU also writes E4M3).
template <int BN, int EPI, bool kF8 = false>
__device__ __forceinline__ void epilogue_tile(const GemmArgs& args, Stager& st, uint32_t tbase, int row0, int n0) {
  const int lane = st.lane;
  const int row = row0 + lane;
  const bool live = row < args.M;
  // dequantise 32 accumulator words in place (E4M3 operands only)
  auto deq = [&](uint32_t (&v)[32], int col) {
    if constexpr (kF8) {
      float cs[32];
      load_cs32(args.colscale + col, cs);
#pragma unroll
      for (int i = 0; i < 32; ++i) v[i] = __float_as_uint(__uint_as_float(v[i]) * cs[i]);
    }
  };
  if constexpr (kF8 && EPI == VLM_EPI_SWIGLU) {
    // 256 accumulator columns -> 128 E4M3 outputs = one 128-byte row chunk;
    // columns 32g..32g+15 are gate and 32g+16..32g+31 up of outputs 16g..16g+15
#pragma unroll 1
    for (int c = 0; c < BN; c += 256) {
      uint32_t w[32];
#pragma unroll
      for (int g = 0; g < 8; ++g) {
        uint32_t r[32];
        tmem_ld32(tbase + c + 32 * g, r);
        deq(r, n0 + c + 32 * g);
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          float h[4];
#pragma unroll
          for (int k = 0; k < 4; ++k)
            h[k] = silu_f(__uint_as_float(r[4 * e + k])) * __uint_as_float(r[16 + 4 * e + k]) * args.out_scale;
          w[4 * g + e] = pack_e4m3x4(h[0], h[1], h[2], h[3]);
        }
      }
      uint8_t* buf = st.acquire();
      st.write_row(buf, w);
      st.commit(buf, (n0 + c) / 2, row0);
    }
  } else if constexpr (EPI == VLM_EPI_BF16 || EPI == VLM_EPI_GELU) {
#pragma unroll 1
    for (int c = 0; c < BN; c += 64) {
      uint32_t a[32], b[32], w[32];
      tmem_ld32(tbase + c, a);
      tmem_ld32(tbase + c + 32, b);
      deq(a, n0 + c);
      deq(b, n0 + c + 32);
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        w[i] = pack_bf16x2(act<EPI>(__uint_as_float(a[2 * i])), act<EPI>(__uint_as_float(a[2 * i + 1])));
        w[16 + i] = pack_bf16x2(act<EPI>(__uint_as_float(b[2 * i])), act<EPI>(__uint_as_float(b[2 * i + 1])));
      }
      uint8_t* buf = st.acquire();
      st.write_row(buf, w);
      st.commit(buf, n0 + c, row0);
    }
  } else if constexpr (EPI == VLM_EPI_F32) {
#pragma unroll 1
    for (int c = 0; c < BN; c += 32) {
      uint32_t a[32];
      tmem_ld32(tbase + c, a);
      deq(a, n0 + c);
      uint8_t* buf = st.acquire();
      st.write_row(buf, a);
      st.commit(buf, n0 + c, row0);
    }
  } else if constexpr (EPI == VLM_EPI_RESID) {
    if (args.c_bf16 == nullptr) {
      // x[row, n0 + c ..] += acc by a bulk tensor reduce-add: no residual reads on the SM
#pragma unroll 1
      for (int c = 0; c < BN; c += 32) {
        uint32_t a[32];
        tmem_ld32(tbase + c, a);
        deq(a, n0 + c);
        uint8_t* buf = st.acquire();
        st.write_row(buf, a);
        st.template commit<true>(buf, n0 + c, row0);
      }
      return;
    }
    // with the bf16 copy the new values are needed here: read the residual.
    // x[row, n0 + c ..] += acc: the warp reads the 32 x 32 fp32 residual chunk
    // with coalesced 16-byte loads (lane -> row 4i + lane/8, 16-byte piece lane%8),
    // one chunk ahead, and parks it in the staging buffer in swizzled order.
    const float* x = static_cast<const float*>(args.c);
    float4 pre[8];
    auto load_res = [&](int c) {
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const int r = row0 + 4 * i + (lane >> 3);
        pre[i] = r < args.M ? __ldg(reinterpret_cast<const float4*>(x + static_cast<int64_t>(r) * args.N + n0 + c) +
                                    (lane & 7))
                            : make_float4(0.f, 0.f, 0.f, 0.f);
      }
    };
    load_res(0);
#pragma unroll 1
    for (int c = 0; c < BN; c += 32) {
      uint8_t* buf = st.acquire();
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const int r = 4 * i + (lane >> 3), ch = lane & 7;
        *reinterpret_cast<float4*>(buf + r * 128 + ((ch ^ (r & 7)) << 4)) = pre[i];
      }
      if (c + 32 < BN) load_res(c + 32);
      uint32_t a[32];
      tmem_ld32(tbase + c, a);
      deq(a, n0 + c);
      __syncwarp();
      float4* rp = reinterpret_cast<float4*>(buf + lane * 128);
      float v[32];
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        float4 o = rp[j ^ (lane & 7)];
        o.x += __uint_as_float(a[4 * j]);
        o.y += __uint_as_float(a[4 * j + 1]);
        o.z += __uint_as_float(a[4 * j + 2]);
        o.w += __uint_as_float(a[4 * j + 3]);
        rp[j ^ (lane & 7)] = o;
        v[4 * j] = o.x; v[4 * j + 1] = o.y; v[4 * j + 2] = o.z; v[4 * j + 3] = o.w;
      }
      if (args.c_bf16 != nullptr && live) {
        uint4* db = reinterpret_cast<uint4*>(args.c_bf16 + static_cast<int64_t>(row) * args.N + n0 + c);
#pragma unroll
        for (int j = 0; j < 4; ++j)
          db[j] = make_uint4(pack_bf16x2(v[8 * j], v[8 * j + 1]), pack_bf16x2(v[8 * j + 2], v[8 * j + 3]),
                             pack_bf16x2(v[8 * j + 4], v[8 * j + 5]), pack_bf16x2(v[8 * j + 6], v[8 * j + 7]));
      }
      st.commit(buf, n0 + c, row0);
    }
  } else if constexpr (EPI == VLM_EPI_SWIGLU) {
    // accumulator columns 32g..32g+15 are gate, 32g+16..32g+31 the matching up
    // values of output columns 16g..16g+15; a 128-column chunk gives 64 outputs
#pragma unroll 1
    for (int c = 0; c < BN; c += 128) {
      uint32_t w[32];
#pragma unroll
      for (int g = 0; g < 4; ++g) {
        uint32_t r[32];
        tmem_ld32(tbase + c + 32 * g, r);
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          const float h0 = silu_f(__uint_as_float(r[2 * e])) * __uint_as_float(r[16 + 2 * e]);
          const float h1 = silu_f(__uint_as_float(r[2 * e + 1])) * __uint_as_float(r[16 + 2 * e + 1]);
          w[8 * g + e] = pack_bf16x2(h0, h1);
        }
      }
      uint8_t* buf = st.acquire();
      st.write_row(buf, w);
      st.commit(buf, (n0 + c) / 2, row0);
    }
  } else if constexpr (EPI == VLM_EPI_ROPE) {
    const int pk = live ? __ldg(args.pos + row) : 0;
    const int pr = pk >> 16, pc = pk & 0xFFFF;
#pragma unroll 1
    for (int c = 0; c < BN; c += 64) {
      uint32_t a[32], b[32], w[32];
      tmem_ld32(tbase + c, a);
      tmem_ld32(tbase + c + 32, b);
      deq(a, n0 + c);
      deq(b, n0 + c + 32);
      float x[32], y[32];
#pragma unroll
      for (int i = 0; i < 32; ++i) { x[i] = __uint_as_float(a[i]); y[i] = __uint_as_float(b[i]); }
      if (n0 + c < args.rope_cols) {
        const float2* tr = args.rope + pr * 32;
        const float2* tc = args.rope + pc * 32;
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          const float2 cs = __ldg(i < 16 ? tr + i : tc + i);
          const float xi = x[i], yi = y[i];
          x[i] = xi * cs.x - yi * cs.y;
          y[i] = yi * cs.x + xi * cs.y;
        }
      }
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        w[i] = pack_bf16x2(x[2 * i], x[2 * i + 1]);
        w[16 + i] = pack_bf16x2(y[2 * i], y[2 * i + 1]);
      }
      uint8_t* buf = st.acquire();
      st.write_row(buf, w);
      st.commit(buf, n0 + c, row0);
    }
  } else if constexpr (EPI == kEpiRows) {
    // the masked scatter fused in: this lane's bf16 row goes to row
    // dst_rows[row] of the table, 128 bytes per 64 columns with 16-byte
    // stores. The 32 lanes write 32 different rows (no TMA box fits scattered
    // rows), but the output is a small share of this GEMM's traffic (each
    // output row costs K values of A read), and the stores are not waited on
    const int64_t dst = live && *args.ok_flag != 0 ? __ldg(args.dst_rows + row) : -1;
    const bool put = dst >= 0 && VLM_DCHECK(dst < args.c_rows);
#pragma unroll 1
    for (int c = 0; c < BN; c += 64) {
      uint32_t a[32], b[32];
      tmem_ld32(tbase + c, a);
      tmem_ld32(tbase + c + 32, b);
      if (put) {
        uint4* d = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(args.c) + dst * args.N + n0 + c);
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          d[j] = make_uint4(pack_bf16x2(__uint_as_float(a[8 * j]), __uint_as_float(a[8 * j + 1])),
                            pack_bf16x2(__uint_as_float(a[8 * j + 2]), __uint_as_float(a[8 * j + 3])),
                            pack_bf16x2(__uint_as_float(a[8 * j + 4]), __uint_as_float(a[8 * j + 5])),
                            pack_bf16x2(__uint_as_float(a[8 * j + 6]), __uint_as_float(a[8 * j + 7])));
          d[4 + j] = make_uint4(pack_bf16x2(__uint_as_float(b[8 * j]), __uint_as_float(b[8 * j + 1])),
                                pack_bf16x2(__uint_as_float(b[8 * j + 2]), __uint_as_float(b[8 * j + 3])),
                                pack_bf16x2(__uint_as_float(b[8 * j + 4]), __uint_as_float(b[8 * j + 5])),
                                pack_bf16x2(__uint_as_float(b[8 * j + 6]), __uint_as_float(b[8 * j + 7])));
        }
      }
    }
  }
}

template <int BN, int EPI>
__global__ void __launch_bounds__(192, 1)
    gemm_tcgen05_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                        const __grid_constant__ CUtensorMap tmC, const GemmArgs args) {
  using S = GemmShape<BN>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sA = smem;
  uint8_t* sB = smem + S::STAGES * S::A_BYTES;
  uint8_t* sEpi = smem + S::STAGES * S::STAGE_BYTES;
  uint64_t* bars = reinterpret_cast<uint64_t*>(sEpi + S::EPI_BYTES);
  uint64_t* full = bars;
  uint64_t* empty = bars + S::STAGES;
  uint64_t* tfull = bars + 2 * S::STAGES;
  uint64_t* tempty = tfull + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(tempty + 2);
  int* abort_flag = reinterpret_cast<int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int total_tiles = args.m_tiles * args.n_tiles;
  const int nk = args.K / GBK;

  if (threadIdx.x == 0) {
    for (int s = 0; s < S::STAGES; ++s) {
      mbar_init(smem_u32(full + s), 1);
      mbar_init(smem_u32(empty + s), 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(smem_u32(tfull + a), 1);
      mbar_init(smem_u32(tempty + a), 128);
    }
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tmap(&tmA);
    prefetch_tmap(&tmB);
    prefetch_tmap(&tmC);
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_slot), S::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  volatile int* abort_v = abort_flag;
  griddep_wait();  // A, C (and the residual) belong to the previous kernels until here
  griddep_launch_dependents();

  if (warp == 0) {
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      for (int tile = blockIdx.x; tile < total_tiles && ok; tile += gridDim.x) {
        const int mt = tile / args.n_tiles, nt = tile - mt * args.n_tiles;
        for (int kb = 0; kb < nk; ++kb) {
          if (!mbar_wait(smem_u32(empty + stage), phase ^ 1u, abort_v, args.status)) { ok = false; break; }
          const uint32_t fb = smem_u32(full + stage);
          mbar_arrive_expect_tx(fb, S::STAGE_BYTES);
          tma_load_2d(smem_u32(sA + stage * S::A_BYTES), &tmA, fb, kb * GBK, mt * GBM);
          tma_load_2d(smem_u32(sB + stage * S::B_BYTES), &tmB, fb, kb * GBK, nt * BN);
          if (++stage == S::STAGES) { stage = 0; phase ^= 1u; }
        }
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_bf16(GBM, BN);
      int stage = 0;
      uint32_t phase = 0;
      int acc = 0;
      uint32_t acc_phase = 0;
      bool ok = true;
      for (int tile = blockIdx.x; tile < total_tiles && ok; tile += gridDim.x) {
        if (!mbar_wait(smem_u32(tempty + acc), acc_phase ^ 1u, abort_v, args.status)) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(acc * BN);
        for (int kb = 0; kb < nk; ++kb) {
          if (!mbar_wait(smem_u32(full + stage), phase, abort_v, args.status)) { ok = false; break; }
          tc_fence_after();
          const uint64_t adesc = smem_desc_sw128(smem_u32(sA + stage * S::A_BYTES));
          const uint64_t bdesc = smem_desc_sw128(smem_u32(sB + stage * S::B_BYTES));
#pragma unroll
          for (int k = 0; k < GBK / 16; ++k) {
            // +32 bytes along K inside the 128-byte swizzled row = +2 in the address field
            umma_bf16_ss(d_tmem, adesc + 2 * k, bdesc + 2 * k, idesc, (kb | k) != 0 ? 1u : 0u);
          }
          umma_commit(smem_u32(empty + stage));
          if (++stage == S::STAGES) { stage = 0; phase ^= 1u; }
        }
        if (!ok) break;
        umma_commit(smem_u32(tfull + acc));
        acc ^= 1;
        if (acc == 0) acc_phase ^= 1u;
      }
    }
  } else {
    const int q = warp & 3;  // TMEM lane quadrant this warp may access
    Stager st{sEpi + (warp - 2) * kStageBufs * kStageBufBytes, &tmC, 0, lane};
    int acc = 0;
    uint32_t acc_phase = 0;
    for (int tile = blockIdx.x; tile < total_tiles; tile += gridDim.x) {
      const int mt = tile / args.n_tiles, nt = tile - mt * args.n_tiles;
      if (!mbar_wait_warp(smem_u32(tfull + acc), acc_phase, abort_v, args.status)) break;
      tc_fence_after();
      const uint32_t tbase = tmem_base + (static_cast<uint32_t>(q * 32) << 16) + static_cast<uint32_t>(acc * BN);
      epilogue_tile<BN, EPI>(args, st, tbase, mt * GBM + q * 32, nt * BN);
      tc_fence_before();
      mbar_arrive(smem_u32(tempty + acc));
      acc ^= 1;
      if (acc == 0) acc_phase ^= 1u;
    }
    st.drain();
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, S::TMEM_COLS);
  }
}

// ---------------------------------------------------------------------------
// Two-SM variant (N % 256 == 0): a cluster of two CTAs computes a 256 x 256
// tile with tcgen05.mma.cta_group::2 (M = 256). Each CTA stages its own 128
// rows of A and its own half (128 rows) of the B tile, so per k-block an SM
// reads 32 KiB instead of 48 KiB; the even CTA issues the MMAs and both CTAs'
// TMEM receive their 128 x 256 accumulator rows. Both CTAs run the same
// producer (TMA completion counted on the even CTA's barrier) and epilogue;
// the odd CTA's epilogue hands the accumulator back with a remote arrive.
// ---------------------------------------------------------------------------
struct PairShape {
  static constexpr int BN = 256;
  static constexpr int STAGES = 6;
  static constexpr int A_BYTES = GBM * GBK * 2;         // this CTA's 128 rows of A
  static constexpr int B_BYTES = (BN / 2) * GBK * 2;    // this CTA's 128 rows of B
  static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
  static constexpr int EPI_BYTES = kEpiWarps * kStageBufs * kStageBufBytes;
  static constexpr int TMEM_COLS = 2 * BN;
  static constexpr int BAR_BYTES = 256;
  static constexpr int SMEM_BYTES = STAGES * STAGE_BYTES + EPI_BYTES + BAR_BYTES + 1024;
};

template <int EPI, bool kF8 = false>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(192, 1)
    gemm_pair_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                     const __grid_constant__ CUtensorMap tmC, const GemmArgs args) {
  using S = PairShape;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sA = smem;
  uint8_t* sB = smem + S::STAGES * S::A_BYTES;
  uint8_t* sEpi = smem + S::STAGES * S::STAGE_BYTES;
  uint64_t* bars = reinterpret_cast<uint64_t*>(sEpi + S::EPI_BYTES);
  uint64_t* full = bars;                     // used on the even CTA
  uint64_t* empty = bars + S::STAGES;        // both CTAs
  uint64_t* tfull = bars + 2 * S::STAGES;    // both CTAs
  uint64_t* tempty = tfull + 2;              // used on the even CTA (8 warp arrivals)
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(tempty + 2);
  int* abort_flag = reinterpret_cast<int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const int pair = blockIdx.x >> 1, n_pairs = gridDim.x >> 1;
  const int total_tiles = args.m_tiles * args.n_tiles;  // m_tiles counts 256-row pair tiles here
  // a stage holds 128 bytes of every operand row: 64 bf16 or 128 E4M3 values of K
  constexpr int kBK = kF8 ? 2 * GBK : GBK;
  const int nk = args.K / kBK;

  if (threadIdx.x == 0) {
    for (int s = 0; s < S::STAGES; ++s) {
      mbar_init(smem_u32(full + s), 1);
      mbar_init(smem_u32(empty + s), 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(smem_u32(tfull + a), 1);
      mbar_init(smem_u32(tempty + a), 2 * kEpiWarps);
    }
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tmap(&tmA);
    prefetch_tmap(&tmB);
    prefetch_tmap(&tmC);
  }
  if (warp == 1) {
    tmem_alloc_pair(smem_u32(tmem_slot), S::TMEM_COLS);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync_all();  // both CTAs' barriers are initialised before any cross-CTA signal
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  volatile int* abort_v = abort_flag;
  griddep_wait();  // A, C (and the residual) belong to the previous kernels until here
  griddep_launch_dependents();

  if (warp == 0) {
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      for (int tile = pair; tile < total_tiles && ok; tile += n_pairs) {
        const int mt = tile / args.n_tiles, nt = tile - mt * args.n_tiles;
        const int arow = mt * 256 + static_cast<int>(rank) * GBM;
        const int brow = nt * S::BN + static_cast<int>(rank) * (S::BN / 2);
        for (int kb = 0; kb < nk; ++kb) {
          if (!mbar_wait(smem_u32(empty + stage), phase ^ 1u, abort_v, args.status)) { ok = false; break; }
          const uint32_t fb = smem_u32(full + stage) & kPeerBitMask;
          if (rank == 0) mbar_arrive_expect_tx(smem_u32(full + stage), 2 * S::STAGE_BYTES);
          tma_load_2d_pair(smem_u32(sA + stage * S::A_BYTES), &tmA, fb, kb * kBK, arow);
          tma_load_2d_pair(smem_u32(sB + stage * S::B_BYTES), &tmB, fb, kb * kBK, brow);
          if (++stage == S::STAGES) { stage = 0; phase ^= 1u; }
        }
      }
    }
  } else if (warp == 1) {
    if (rank == 0 && lane == 0) {
      constexpr uint32_t idesc = kF8 ? idesc_e4m3(2 * GBM, S::BN) : idesc_bf16(2 * GBM, S::BN);
      int stage = 0;
      uint32_t phase = 0;
      int acc = 0;
      uint32_t acc_phase = 0;
      bool ok = true;
      for (int tile = pair; tile < total_tiles && ok; tile += n_pairs) {
        if (!mbar_wait_cluster(smem_u32(tempty + acc), acc_phase ^ 1u, abort_v, args.status)) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(acc * S::BN);
        for (int kb = 0; kb < nk; ++kb) {
          if (!mbar_wait(smem_u32(full + stage), phase, abort_v, args.status)) { ok = false; break; }
          tc_fence_after();
          const uint64_t adesc = smem_desc_sw128(smem_u32(sA + stage * S::A_BYTES));
          const uint64_t bdesc = smem_desc_sw128(smem_u32(sB + stage * S::B_BYTES));
#pragma unroll
          for (int k = 0; k < 4; ++k) {  // 32 bytes of K per instruction
            if constexpr (kF8)
              umma_f8_ss_pair(d_tmem, adesc + 2 * k, bdesc + 2 * k, idesc, (kb | k) != 0 ? 1u : 0u);
            else
              umma_bf16_ss_pair(d_tmem, adesc + 2 * k, bdesc + 2 * k, idesc, (kb | k) != 0 ? 1u : 0u);
          }
          umma_commit_pair_mc(smem_u32(empty + stage), 0x3);
          if (++stage == S::STAGES) { stage = 0; phase ^= 1u; }
        }
        if (!ok) break;
        umma_commit_pair_mc(smem_u32(tfull + acc), 0x3);
        acc ^= 1;
        if (acc == 0) acc_phase ^= 1u;
      }
    }
  } else {
    const int q = warp & 3;  // TMEM lane quadrant this warp may access
    Stager st{sEpi + (warp - 2) * kStageBufs * kStageBufBytes, &tmC, 0, lane};
    const uint32_t leader_tempty = mapa_shared(smem_u32(tempty), 0);
    int acc = 0;
    uint32_t acc_phase = 0;
    for (int tile = pair; tile < total_tiles; tile += n_pairs) {
      const int mt = tile / args.n_tiles, nt = tile - mt * args.n_tiles;
      if (!mbar_wait_warp(smem_u32(tfull + acc), acc_phase, abort_v, args.status)) break;
      tc_fence_after();
      const uint32_t tbase = tmem_base + (static_cast<uint32_t>(q * 32) << 16) + static_cast<uint32_t>(acc * S::BN);
      epilogue_tile<S::BN, EPI, kF8>(args, st, tbase, mt * 256 + static_cast<int>(rank) * GBM + q * 32, nt * S::BN);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster_relaxed(leader_tempty + static_cast<uint32_t>(acc * 8));
      acc ^= 1;
      if (acc == 0) acc_phase ^= 1u;
    }
    st.drain();
  }

  tc_fence_before();
  __syncthreads();
  cluster_sync_all();  // neither CTA leaves while its pair may still signal or read it
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tmem_base, S::TMEM_COLS);
  }
}

template <int EPI, bool kF8 = false>
int run_gemm_pair(const CUtensorMap& ta, const CUtensorMap& tb, const CUtensorMap& tc, const GemmArgs& args,
                  cudaStream_t s) {
  auto kern = gemm_pair_kernel<EPI, kF8>;
  static bool attr_done[64] = {};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 64 && !attr_done[dev]) {
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, PairShape::SMEM_BYTES) !=
        cudaSuccess)
      return VLM_ERR_CUDA;
    attr_done[dev] = true;
  }
  const int tiles = args.m_tiles * args.n_tiles;
  const int max_pairs = sm_budget() / 2 > 0 ? sm_budget() / 2 : 1;
  const int pairs = tiles < max_pairs ? tiles : max_pairs;
  launch_begin(KC_GEMM, s);
  const cudaError_t e = launch_pdl(kern, dim3(2 * pairs), dim3(192), PairShape::SMEM_BYTES, s, ta, tb, tc, args);
  launch_end(KC_GEMM, s);
  return e == cudaSuccess ? VLM_OK : VLM_ERR_CUDA;
}

int dispatch_pair(int epi, const CUtensorMap& ta, const CUtensorMap& tb, const CUtensorMap& tc, const GemmArgs& args,
                  cudaStream_t s) {
  switch (epi) {
    case VLM_EPI_BF16: return run_gemm_pair<VLM_EPI_BF16>(ta, tb, tc, args, s);
    case VLM_EPI_F32: return run_gemm_pair<VLM_EPI_F32>(ta, tb, tc, args, s);
    case VLM_EPI_RESID: return run_gemm_pair<VLM_EPI_RESID>(ta, tb, tc, args, s);
    case VLM_EPI_SWIGLU: return run_gemm_pair<VLM_EPI_SWIGLU>(ta, tb, tc, args, s);
    case VLM_EPI_ROPE: return run_gemm_pair<VLM_EPI_ROPE>(ta, tb, tc, args, s);
    case VLM_EPI_GELU: return run_gemm_pair<VLM_EPI_GELU>(ta, tb, tc, args, s);
    case kEpiRows: return run_gemm_pair<kEpiRows>(ta, tb, tc, args, s);
    default: return VLM_ERR_INVALID_ARG;
  }
}

int dispatch_pair_f8(int epi, const CUtensorMap& ta, const CUtensorMap& tb, const CUtensorMap& tc,
                     const GemmArgs& args, cudaStream_t s) {
  switch (epi) {
    case VLM_EPI_BF16: return run_gemm_pair<VLM_EPI_BF16, true>(ta, tb, tc, args, s);
    case VLM_EPI_RESID: return run_gemm_pair<VLM_EPI_RESID, true>(ta, tb, tc, args, s);
    case VLM_EPI_SWIGLU: return run_gemm_pair<VLM_EPI_SWIGLU, true>(ta, tb, tc, args, s);
    case VLM_EPI_ROPE: return run_gemm_pair<VLM_EPI_ROPE, true>(ta, tb, tc, args, s);
    default: return VLM_ERR_UNSUPPORTED;
  }
}

// ---------------------------------------------------------------------------
// NVFP4 two-SM variant: E2M1 operands with E4M3 block scales
// (tcgen05.mma.kind::mxf4nvf4.block_scale.block16; M = 256, N = BN, K = 64
// per instruction). A stage holds 128 bytes (256 values) of every operand row
// and the stage's scale atoms of each operand: this CTA's 128 rows of A, and
// all BN columns of B (each CTA loads its own copy; no multicast). The even
// CTA copies the atoms into tensor memory with tcgen05.cp (one
// 32x128b.warpx4 copy per atom, into both CTAs' TMEM from each CTA's own
// shared memory). Per K = 64 step the A scales take 4 TMEM columns (row r's
// four scales sit in lane r % 32 of every lane quarter, column (r % 128) / 32)
// and the B scales 4 per 128 columns of the tile.
//
// Each tcgen05 instruction costs its issuing thread close to a hundred cycles,
// not far from what one K = 64 MMA of this shape takes on the tensor pipe
// (128 cycles), so one thread issuing a stage's 4 MMAs and its 12 scale copies
// cannot keep the pipe busy. The copies are therefore issued by copy warps of
// the even CTA (two for A and two per 128 columns of B, two copies each), into
// two scale slots used in turn. A copy followed by an MMA is a pipelined pair
// of tcgen05 instructions: the MMA executes after the copy when it is issued
// after it, and tcgen05.fence::before_thread_sync / after_thread_sync around
// an mbarrier hand-off carry that issue order across threads. So a copy warp
// arrives on sf_full[slot] as soon as its copies are issued, and the MMA
// thread issues the stage's MMAs behind them without waiting for the copies
// to complete. An MMA followed by a copy is not such a pair: a copy warp
// refills a slot only once the MMAs that last read it have completed, which
// their commit to empty[] signals. The MMA thread issues only MMAs and commits.
//
// TMEM (512 columns): BN = 128 keeps two 128-column accumulators side by side
// and the scale slots behind them. BN = 256 would need 512 columns for two
// accumulators alone, so the second one starts at column 160 and shares 96
// columns with the first; the scale slots take columns 416..511. The epilogue
// reads the shared columns of a tile first and then signals `ovl`: the next
// tile's MMAs (into the other accumulator) wait for that signal and for the
// other accumulator's own release, so they start while the epilogue is still
// working through the tile's other columns.
// ---------------------------------------------------------------------------
template <int BN_>
struct Fp4Shape {
  static constexpr int BN = BN_;
  static constexpr bool kOverlap = BN == 256;
  static constexpr int STAGES = BN == 256 ? 5 : 6;
  static constexpr int A_BYTES = GBM * 128;        // this CTA's 128 rows x 256 values
  static constexpr int B_BYTES = (BN / 2) * 128;   // this CTA's half of the B tile
  static constexpr int SFA_BYTES = 4 * 512;        // four 512-byte scale atoms
  static constexpr int SFB_BLOCKS = BN / 128;      // 128-column groups of B scales
  static constexpr int SFB_BYTES = SFB_BLOCKS * 4 * 512;
  static constexpr int STAGE_BYTES = A_BYTES + B_BYTES + SFA_BYTES + SFB_BYTES;
  static constexpr int EPI_BYTES = kEpiWarps * kStageBufs * kStageBufBytes;
  static constexpr int ACC_STRIDE = kOverlap ? 160 : BN;  // TMEM column of the second accumulator
  // Two scale slots used in turn: the copies of stage g + 1 fill one while the
  // MMAs of stage g read the other. A slot holds 4 columns per K = 64 step for
  // A and 4 per step per 128 columns of B.
  static constexpr int SF_SLOT_COLS = 16 + 16 * SFB_BLOCKS;
  static constexpr int SF_BASE = kOverlap ? 416 : 2 * BN;
  static constexpr int TMEM_COLS = 512;
  // copy warps of the even CTA: two for the A scales and two per 128-column
  // group of B, each issuing the copies of two K = 64 steps
  static constexpr int COPY_WARPS = 2 * (1 + SFB_BLOCKS);
  static constexpr int THREADS = 192 + 32 * COPY_WARPS;
  static constexpr int BAR_BYTES = 256;
  static constexpr int SMEM_BYTES = STAGES * STAGE_BYTES + EPI_BYTES + BAR_BYTES + 1024;
  static_assert(SF_BASE + 2 * SF_SLOT_COLS <= TMEM_COLS, "scale columns past the allocation");
  static_assert(!kOverlap || SF_BASE >= ACC_STRIDE + BN, "scale slots overlap the second accumulator");
  static_assert(SMEM_BYTES <= 232448, "shared memory per CTA");
};

// Instruction descriptor of kind::mxf4nvf4: E2M1 A and B (format code 1), E4M3
// scales (scale format 0), scale-factor ids 0, both operands K-major.
__host__ __device__ constexpr uint32_t idesc_nvfp4(int m, int n) {
  return (1u << 7)                                  // A format: E2M1
         | (1u << 10)                               // B format: E2M1
         | (static_cast<uint32_t>(n >> 3) << 17)    // N / 8
         | (0u << 23)                               // scale format: E4M3
         | (static_cast<uint32_t>(m >> 4) << 24);   // M / 16
}

// Descriptor of one 512-byte scale atom as a tcgen05.cp source: 32 rows of 16
// bytes, no swizzle, 8-row groups 128 bytes apart.
__device__ __forceinline__ uint64_t smem_desc_sf_atom(uint32_t saddr) {
  return static_cast<uint64_t>((saddr & 0x3FFFFu) >> 4) | (static_cast<uint64_t>(128 >> 4) << 32) |
         (1ull << 46);  // descriptor version (sm100); layout: no swizzle
}
__device__ __forceinline__ void tmem_cp_atom_pair(uint32_t taddr, uint64_t sdesc) {
  asm volatile("tcgen05.cp.cta_group::2.32x128b.warpx4 [%0], %1;" ::"r"(taddr), "l"(sdesc) : "memory");
}
__device__ __forceinline__ void umma_nvfp4_pair(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                                uint32_t sfa_tmem, uint32_t sfb_tmem, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::mxf4nvf4.block_scale.block16 [%0], %1, %2, %3, [%5], [%6], p;\n\t}" ::"r"(
          d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate), "r"(sfa_tmem), "r"(sfb_tmem)
      : "memory");
}

// 32 accumulator columns (fp32 bits) scaled by alpha, as 16 packed bf16 pairs at w[OFF..OFF+15].
template <int OFF, int N>
__device__ __forceinline__ void pack_scaled16(const uint32_t (&a)[32], uint32_t (&w)[N], float alpha) {
#pragma unroll
  for (int j = 0; j < 16; ++j)
    w[OFF + j] = pack_bf16x2(__uint_as_float(a[2 * j]) * alpha, __uint_as_float(a[2 * j + 1]) * alpha);
}
__device__ __forceinline__ void scale32(uint32_t (&a)[32], float alpha) {
#pragma unroll
  for (int j = 0; j < 32; ++j) a[j] = __float_as_uint(__uint_as_float(a[j]) * alpha);
}

// This warp's 32 rows of a 128 x BN tile held at TMEM address tbase, scaled by
// alpha: bf16 stores (64-column chunks), or an fp32 bulk reduce-add into c
// (32-column chunks). With overlapping accumulators (kOverlap: BN = 256, the
// second accumulator 160 columns after the first) the 96 columns both share --
// tile columns 160..255 of accumulator 0, 0..95 of accumulator 1 -- are read
// from TMEM first and held in registers; on_shared() then releases them to
// the next tile's MMAs before any of them is stored.
//
// ROPE (kOverlap only): bf16 output like BF16, with the 2D rotary embedding
// applied in fp32 to the columns below rope_cols: a 64-column chunk is one
// head, pair (i, i + 32) rotated by the angle of the row's position (row
// frequencies for i < 16, column frequencies above). The shared half-head
// waits in fp32 registers for its partner half.
// SWIGLU (kOverlap only): accumulator columns 32g..32g+15 hold gate and
// 32g+16..32g+31 the matching up values of hidden columns 16g..16g+15, one
// NVFP4 block: h = silu(gate) * up in fp32, quantised with global scale
// args.out_scale; codes and block scales are stored straight from registers.
template <int EPI, int BN, bool kOverlap, typename F>
__device__ __forceinline__ void epilogue_nvfp4(const GemmArgs& args, Stager& st, uint32_t tbase, int row0, int n0,
                                               int acc, float alpha, F&& on_shared) {
  static_assert(!kOverlap || BN == 256, "the overlap layout is for 256-column tiles");
  static_assert(kOverlap || (EPI != VLM_EPI_ROPE && EPI != VLM_EPI_SWIGLU), "rope / swiglu need 256-column tiles");
  if constexpr (EPI == VLM_EPI_ROPE) {
    const int lane = st.lane, row = row0 + lane;
    const int pk = row < args.M ? __ldg(args.pos + row) : 0;
    const float2* tr = args.rope + (pk >> 16) * 32;
    const float2* tcol = args.rope + (pk & 0xFFFF) * 32;
    auto finish = [&](float (&x)[32], float (&y)[32], int c) {
      if (n0 + c < args.rope_cols) {
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          const float2 cs = __ldg(i < 16 ? tr + i : tcol + i);
          const float xi = x[i], yi = y[i];
          x[i] = xi * cs.x - yi * cs.y;
          y[i] = yi * cs.x + xi * cs.y;
        }
      }
      uint32_t w[32];
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        w[i] = pack_bf16x2(x[2 * i], x[2 * i + 1]);
        w[16 + i] = pack_bf16x2(y[2 * i], y[2 * i + 1]);
      }
      uint8_t* buf = st.acquire();
      st.write_row(buf, w);
      st.commit(buf, n0 + c, row0);
    };
    auto load_scaled = [&](uint32_t col, float (&v)[32]) {
      uint32_t a[32];
      tmem_ld32(tbase + col, a);
#pragma unroll
      for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(a[i]) * alpha;
    };
    // the shared columns: head cp whole, and half ho of head ch
    const int cp = acc == 0 ? 192 : 0, ch = acc == 0 ? 128 : 64, ho = acc == 0 ? 32 : 0;
    float x[32], y[32], hv[32];
    load_scaled(cp, x);
    load_scaled(cp + 32, y);
    load_scaled(ch + ho, hv);
    on_shared();
    finish(x, y, cp);
    load_scaled(ch + 32 - ho, x);
    if (ho == 0) {
      finish(hv, x, ch);
    } else {
      finish(x, hv, ch);
    }
    const int c_rest = acc == 0 ? 0 : 128;
#pragma unroll 1
    for (int i = 0; i < 2; ++i) {
      const int c = c_rest + 64 * i;
      load_scaled(c, x);
      load_scaled(c + 32, y);
      finish(x, y, c);
    }
  } else if constexpr (EPI == VLM_EPI_SWIGLU) {
    const int lane = st.lane, row = row0 + lane;
    const bool live = row < args.M;
    const int kh = args.N / 2;  // hidden width: the K of the GEMM that reads these codes
    uint8_t* codes_row = static_cast<uint8_t*>(args.c) + static_cast<int64_t>(row) * (kh / 2) + n0 / 4;
    const float sg = args.out_scale, six_sg = 6.0f * sg;
    uint32_t sf_lo = 0, sf_hi = 0;  // scale bytes of blocks g = 0..3 and 4..7 of the tile
    auto block = [&](int g, const uint32_t (&r)[32]) {
      float h[16], amax = 0.0f;
#pragma unroll
      for (int e = 0; e < 16; ++e) {
        h[e] = silu_tanh_f(__uint_as_float(r[e]) * alpha) * (__uint_as_float(r[16 + e]) * alpha);
        amax = fmaxf(amax, fabsf(h[e]));
      }
      uint2 q;
      const uint32_t sb = nvfp4_quant16(h, amax, sg, six_sg, q);
      if (g < 4) sf_lo |= sb << (8 * g);
      else sf_hi |= sb << (8 * (g - 4));
      if (live) *reinterpret_cast<uint2*>(codes_row + 8 * g) = q;
    };
    // the shared columns: blocks 5..7 of accumulator 0, 0..2 of accumulator 1
    const int gs = acc == 0 ? 5 : 0;
    uint32_t r0[32], r1[32], r2[32];
    tmem_ld32(tbase + 32 * gs, r0);
    tmem_ld32(tbase + 32 * (gs + 1), r1);
    tmem_ld32(tbase + 32 * (gs + 2), r2);
    on_shared();
    block(gs, r0);
    block(gs + 1, r1);
    block(gs + 2, r2);
    const int g_rest = acc == 0 ? 0 : 3;
#pragma unroll 1
    for (int i = 0; i < 5; ++i) {
      tmem_ld32(tbase + 32 * (g_rest + i), r0);
      block(g_rest + i, r0);
    }
    if (live) {
      const int kb0 = n0 / 32;  // first block of the tile (a multiple of 8)
      *reinterpret_cast<uint32_t*>(args.c_sf + nvfp4_sf_offset(row, kb0, kh)) = sf_lo;
      *reinterpret_cast<uint32_t*>(args.c_sf + nvfp4_sf_offset(row, kb0 + 4, kh)) = sf_hi;
    }
  } else if constexpr (EPI == VLM_EPI_BF16) {
    int c_rest = 0;  // first of the chunks outside the shared columns
    if constexpr (kOverlap) {
      // the shared columns: one whole chunk (cp) and one half of another (ch + ho)
      const int cp = acc == 0 ? 192 : 0, ch = acc == 0 ? 128 : 64, ho = acc == 0 ? 32 : 0;
      uint32_t a[32], wp[32], wh[16];
      tmem_ld32(tbase + cp, a);
      pack_scaled16<0>(a, wp, alpha);
      tmem_ld32(tbase + cp + 32, a);
      pack_scaled16<16>(a, wp, alpha);
      tmem_ld32(tbase + ch + ho, a);
      pack_scaled16<0>(a, wh, alpha);
      on_shared();
      uint8_t* buf = st.acquire();
      st.write_row(buf, wp);
      st.commit(buf, n0 + cp, row0);
      // the chunk with one shared half
      tmem_ld32(tbase + ch + (32 - ho), a);
      uint32_t w[32];
      if (ho == 0) {
#pragma unroll
        for (int j = 0; j < 16; ++j) w[j] = wh[j];
        pack_scaled16<16>(a, w, alpha);
      } else {
        pack_scaled16<0>(a, w, alpha);
#pragma unroll
        for (int j = 0; j < 16; ++j) w[16 + j] = wh[j];
      }
      buf = st.acquire();
      st.write_row(buf, w);
      st.commit(buf, n0 + ch, row0);
      c_rest = acc == 0 ? 0 : 128;
    }
    constexpr int kRest = kOverlap ? 2 : BN / 64;
#pragma unroll 1
    for (int i = 0; i < kRest; ++i) {
      const int c = c_rest + 64 * i;
      uint32_t a[32], w[32];
      tmem_ld32(tbase + c, a);
      pack_scaled16<0>(a, w, alpha);
      tmem_ld32(tbase + c + 32, a);
      pack_scaled16<16>(a, w, alpha);
      uint8_t* buf = st.acquire();
      st.write_row(buf, w);
      st.commit(buf, n0 + c, row0);
    }
  } else {
    int c_rest = 0;
    if constexpr (kOverlap) {
      const int cs = acc == 0 ? 160 : 0;  // the three shared 32-column chunks
      uint32_t a0[32], a1[32], a2[32];
      tmem_ld32(tbase + cs, a0);
      tmem_ld32(tbase + cs + 32, a1);
      tmem_ld32(tbase + cs + 64, a2);
      on_shared();
      scale32(a0, alpha);
      uint8_t* buf = st.acquire();
      st.write_row(buf, a0);
      st.template commit<true>(buf, n0 + cs, row0);
      scale32(a1, alpha);
      buf = st.acquire();
      st.write_row(buf, a1);
      st.template commit<true>(buf, n0 + cs + 32, row0);
      scale32(a2, alpha);
      buf = st.acquire();
      st.write_row(buf, a2);
      st.template commit<true>(buf, n0 + cs + 64, row0);
      c_rest = acc == 0 ? 0 : 96;
    }
    constexpr int kRest = kOverlap ? 5 : BN / 32;
#pragma unroll 1
    for (int i = 0; i < kRest; ++i) {
      const int c = c_rest + 32 * i;
      uint32_t a[32];
      tmem_ld32(tbase + c, a);
      scale32(a, alpha);
      uint8_t* buf = st.acquire();
      st.write_row(buf, a);
      st.template commit<true>(buf, n0 + c, row0);
    }
  }
}

template <int EPI, int BN>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(Fp4Shape<BN>::THREADS, 1)
    gemm_nvfp4_pair_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                           const __grid_constant__ CUtensorMap tmSFA, const __grid_constant__ CUtensorMap tmSFB,
                           const __grid_constant__ CUtensorMap tmC, const GemmArgs args) {
  using S = Fp4Shape<BN>;
  static_assert(!S::kOverlap || S::ACC_STRIDE == 160, "the epilogue reads the shared columns 160..255 / 0..95");
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sA = smem;
  uint8_t* sB = sA + S::STAGES * S::A_BYTES;
  uint8_t* sSFA = sB + S::STAGES * S::B_BYTES;
  uint8_t* sSFB = sSFA + S::STAGES * S::SFA_BYTES;
  uint8_t* sEpi = sSFB + S::STAGES * S::SFB_BYTES;
  uint64_t* bars = reinterpret_cast<uint64_t*>(sEpi + S::EPI_BYTES);
  uint64_t* full = bars;                     // used on the even CTA
  uint64_t* empty = bars + S::STAGES;        // both CTAs
  uint64_t* tfull = bars + 2 * S::STAGES;    // both CTAs
  uint64_t* tempty = tfull + 2;              // used on the even CTA (8 warp arrivals)
  uint64_t* ovl = tempty + 2;                // used on the even CTA (8 warp arrivals)
  uint64_t* sf_full = ovl + 1;               // used on the even CTA (copies issued into a scale slot)
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sf_full + 2);
  int* abort_flag = reinterpret_cast<int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const int pair = blockIdx.x >> 1, n_pairs = gridDim.x >> 1;
  const int total_tiles = args.m_tiles * args.n_tiles;  // 256-row x BN-column pair tiles
  const int nk = args.K / 256;                          // a stage holds 256 values of K
  const int katoms = args.K / 64;                       // scale atoms per 128-row group

  if (threadIdx.x == 0) {
    for (int s = 0; s < S::STAGES; ++s) {
      mbar_init(smem_u32(full + s), 1);
      mbar_init(smem_u32(empty + s), 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(smem_u32(tfull + a), 1);
      mbar_init(smem_u32(tempty + a), 2 * kEpiWarps);
    }
    mbar_init(smem_u32(ovl), 2 * kEpiWarps);
    for (int b = 0; b < 2; ++b) mbar_init(smem_u32(sf_full + b), S::COPY_WARPS);  // one arrival per copy warp
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tmap(&tmA);
    prefetch_tmap(&tmB);
    prefetch_tmap(&tmSFA);
    prefetch_tmap(&tmSFB);
    prefetch_tmap(&tmC);
  }
  if (warp == 1) {
    tmem_alloc_pair(smem_u32(tmem_slot), S::TMEM_COLS);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync_all();  // both CTAs' barriers are initialised before any cross-CTA signal
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  volatile int* abort_v = abort_flag;
  griddep_wait();  // operands and c belong to the previous kernels until here
  griddep_launch_dependents();

  if (warp == 0) {
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      for (int tile = pair; tile < total_tiles && ok; tile += n_pairs) {
        const int mt = tile / args.n_tiles, nt = tile - mt * args.n_tiles;
        const int arow = mt * 256 + static_cast<int>(rank) * GBM;
        const int brow = nt * S::BN + static_cast<int>(rank) * (S::BN / 2);
        const int sfa_atom = (2 * mt + static_cast<int>(rank)) * katoms;
        const int sfb_atom = nt * S::SFB_BLOCKS * katoms;
        for (int kb = 0; kb < nk; ++kb) {
          if (!mbar_wait(smem_u32(empty + stage), phase ^ 1u, abort_v, args.status)) { ok = false; break; }
          const uint32_t fb = smem_u32(full + stage) & kPeerBitMask;
          if (rank == 0) mbar_arrive_expect_tx(smem_u32(full + stage), 2 * S::STAGE_BYTES);
          tma_load_2d_pair(smem_u32(sA + stage * S::A_BYTES), &tmA, fb, kb * 128, arow);
          tma_load_2d_pair(smem_u32(sB + stage * S::B_BYTES), &tmB, fb, kb * 128, brow);
          tma_load_2d_pair(smem_u32(sSFA + stage * S::SFA_BYTES), &tmSFA, fb, 0, sfa_atom + 4 * kb);
#pragma unroll
          for (int j = 0; j < S::SFB_BLOCKS; ++j)
            tma_load_2d_pair(smem_u32(sSFB + stage * S::SFB_BYTES + j * 2048), &tmSFB, fb, 0,
                             sfb_atom + j * katoms + 4 * kb);
          if (++stage == S::STAGES) { stage = 0; phase ^= 1u; }
        }
      }
    }
  } else if (warp == 1) {
    if (rank == 0 && lane == 0) {
      constexpr uint32_t idesc = idesc_nvfp4(2 * GBM, S::BN);
      int stage = 0;
      uint32_t g = 0;  // stages consumed so far: scale slot g & 1, its use (g >> 1)
      int acc = 0;
      uint32_t acc_phase = 0, ovl_phase = 0;
      bool ok = true;
      for (int tile = pair; tile < total_tiles && ok; tile += n_pairs) {
        if (!mbar_wait_cluster(smem_u32(tempty + acc), acc_phase ^ 1u, abort_v, args.status)) break;
        if constexpr (S::kOverlap) {
          // the previous tile's epilogue has read the columns both accumulators share
          if (!mbar_wait_cluster(smem_u32(ovl), ovl_phase ^ 1u, abort_v, args.status)) break;
          ovl_phase ^= 1u;
        }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(acc * S::ACC_STRIDE);
        for (int kb = 0; kb < nk; ++kb) {
          // the copy warps arrive on sf_full only after they have seen the stage's operands land (full)
          if (!mbar_wait(smem_u32(sf_full + (g & 1u)), (g >> 1) & 1u, abort_v, args.status)) { ok = false; break; }
          tc_fence_after();
          const uint64_t adesc = smem_desc_sw128(smem_u32(sA + stage * S::A_BYTES));
          const uint64_t bdesc = smem_desc_sw128(smem_u32(sB + stage * S::B_BYTES));
          const uint32_t sfa_t = tmem_base + S::SF_BASE + (g & 1u) * S::SF_SLOT_COLS, sfb_t = sfa_t + 16;
#pragma unroll
          for (int k = 0; k < 4; ++k)  // 32 bytes (64 values) of K per instruction
            umma_nvfp4_pair(d_tmem, adesc + 2 * k, bdesc + 2 * k, idesc, sfa_t + 4 * k,
                            sfb_t + 4 * S::SFB_BLOCKS * k, (kb | k) != 0 ? 1u : 0u);
          // completes when the MMAs have read the stage's operands and its scale slot
          umma_commit_pair_mc(smem_u32(empty + stage), 0x3);
          ++g;
          if (++stage == S::STAGES) stage = 0;
        }
        if (!ok) break;
        umma_commit_pair_mc(smem_u32(tfull + acc), 0x3);
        acc ^= 1;
        if (acc == 0) acc_phase ^= 1u;
      }
    }
  } else if (warp < 2 + kEpiWarps) {
    const int q = warp & 3;  // TMEM lane quadrant this warp may access
    Stager st{sEpi + (warp - 2) * kStageBufs * kStageBufBytes, &tmC, 0, lane};
    const uint32_t leader_tempty = mapa_shared(smem_u32(tempty), 0);
    const uint32_t leader_ovl = mapa_shared(smem_u32(ovl), 0);
    const float alpha = __ldg(args.g_a) * __ldg(args.g_b);
    int acc = 0;
    uint32_t acc_phase = 0;
    for (int tile = pair; tile < total_tiles; tile += n_pairs) {
      const int mt = tile / args.n_tiles, nt = tile - mt * args.n_tiles;
      if (!mbar_wait_warp(smem_u32(tfull + acc), acc_phase, abort_v, args.status)) break;
      tc_fence_after();
      const uint32_t tbase =
          tmem_base + (static_cast<uint32_t>(q * 32) << 16) + static_cast<uint32_t>(acc * S::ACC_STRIDE);
      epilogue_nvfp4<EPI, S::BN, S::kOverlap>(args, st, tbase, mt * 256 + static_cast<int>(rank) * GBM + q * 32,
                                              nt * S::BN, acc, alpha, [&] {
                                   if constexpr (S::kOverlap) {
                                     tc_fence_before();
                                     __syncwarp();
                                     if (lane == 0) mbar_arrive_cluster_relaxed(leader_ovl);
                                   }
                                 });
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster_relaxed(leader_tempty + static_cast<uint32_t>(acc * 8));
      acc ^= 1;
      if (acc == 0) acc_phase ^= 1u;
    }
    st.drain();
  } else if (rank == 0 && lane == 0) {
    // copy warp c: K = 64 steps 2 (c & 1) and 2 (c & 1) + 1 of the A scales
    // (c < 2) or of the B scales of 128-column group c / 2 - 1
    const int c = warp - 2 - kEpiWarps;
    const int grp = c >> 1, k0 = 2 * (c & 1);
    int stage = 0;
    uint32_t phase = 0;
    uint32_t g = 0;  // stages filled so far
    bool ok = true;
    for (int tile = pair; tile < total_tiles && ok; tile += n_pairs) {
      for (int kb = 0; kb < nk; ++kb) {
        if (!mbar_wait(smem_u32(full + stage), phase, abort_v, args.status)) { ok = false; break; }
        if (g >= 2) {  // the slot's previous reader, stage g - 2, has completed its MMAs
          const uint32_t h = g - 2;
          if (!mbar_wait(smem_u32(empty + h % S::STAGES), (h / S::STAGES) & 1u, abort_v, args.status)) {
            ok = false;
            break;
          }
        }
        tc_fence_after();
        const uint32_t slot = tmem_base + S::SF_BASE + (g & 1u) * S::SF_SLOT_COLS;
        if (grp == 0) {
          const uint32_t sfa_s = smem_u32(sSFA + stage * S::SFA_BYTES);
#pragma unroll
          for (int k = k0; k < k0 + 2; ++k) tmem_cp_atom_pair(slot + 4 * k, smem_desc_sf_atom(sfa_s + 512 * k));
        } else {
          const int j = grp - 1;
          const uint32_t sfb_s = smem_u32(sSFB + stage * S::SFB_BYTES + 2048 * j);
#pragma unroll
          for (int k = k0; k < k0 + 2; ++k)
            tmem_cp_atom_pair(slot + 16 + 4 * (S::SFB_BLOCKS * k + j), smem_desc_sf_atom(sfb_s + 512 * k));
        }
        // issued, not completed: the MMAs that read the slot are issued behind these copies
        tc_fence_before();
        mbar_arrive(smem_u32(sf_full + (g & 1u)));
        ++g;
        if (++stage == S::STAGES) { stage = 0; phase ^= 1u; }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  cluster_sync_all();  // neither CTA leaves while its pair may still signal or read it
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tmem_base, S::TMEM_COLS);
  }
}

template <int EPI, int BN>
int run_gemm_nvfp4(const CUtensorMap& ta, const CUtensorMap& tb, const CUtensorMap& tsa, const CUtensorMap& tsb,
                   const CUtensorMap& tc, const GemmArgs& args, cudaStream_t s) {
  using S = Fp4Shape<BN>;
  auto kern = gemm_nvfp4_pair_kernel<EPI, BN>;
  static bool attr_done[64] = {};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 64 && !attr_done[dev]) {
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, S::SMEM_BYTES) != cudaSuccess)
      return VLM_ERR_CUDA;
    attr_done[dev] = true;
  }
  const int tiles = args.m_tiles * args.n_tiles;
  const int max_pairs = sm_budget() / 2 > 0 ? sm_budget() / 2 : 1;
  const int pairs = tiles < max_pairs ? tiles : max_pairs;
  launch_begin(KC_GEMM, s);
  const cudaError_t e =
      launch_pdl(kern, dim3(2 * pairs), dim3(S::THREADS), S::SMEM_BYTES, s, ta, tb, tsa, tsb, tc, args);
  launch_end(KC_GEMM, s);
  return e == cudaSuccess ? VLM_OK : VLM_ERR_CUDA;
}

template <int BN, int EPI>
int run_gemm(const CUtensorMap& ta, const CUtensorMap& tb, const CUtensorMap& tc, const GemmArgs& args,
             cudaStream_t s) {
  using S = GemmShape<BN>;
  auto kern = gemm_tcgen05_kernel<BN, EPI>;
  static bool attr_done[64] = {};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 64 && !attr_done[dev]) {
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, S::SMEM_BYTES) != cudaSuccess)
      return VLM_ERR_CUDA;
    attr_done[dev] = true;
  }
  const int tiles = args.m_tiles * args.n_tiles;
  const int grid = tiles < sm_budget() ? tiles : sm_budget();
  launch_begin(KC_GEMM, s);
  const cudaError_t e = launch_pdl(kern, dim3(grid), dim3(192), S::SMEM_BYTES, s, ta, tb, tc, args);
  launch_end(KC_GEMM, s);
  return e == cudaSuccess ? VLM_OK : VLM_ERR_CUDA;
}

template <int BN>
int dispatch_epi(int epi, const CUtensorMap& ta, const CUtensorMap& tb, const CUtensorMap& tc, const GemmArgs& args,
                 cudaStream_t s) {
  switch (epi) {
    case VLM_EPI_BF16: return run_gemm<BN, VLM_EPI_BF16>(ta, tb, tc, args, s);
    case VLM_EPI_F32: return run_gemm<BN, VLM_EPI_F32>(ta, tb, tc, args, s);
    case VLM_EPI_RESID: return run_gemm<BN, VLM_EPI_RESID>(ta, tb, tc, args, s);
    case VLM_EPI_SWIGLU: return run_gemm<BN, VLM_EPI_SWIGLU>(ta, tb, tc, args, s);
    case VLM_EPI_ROPE: return run_gemm<BN, VLM_EPI_ROPE>(ta, tb, tc, args, s);
    case VLM_EPI_GELU: return run_gemm<BN, VLM_EPI_GELU>(ta, tb, tc, args, s);
    case kEpiRows: return run_gemm<BN, kEpiRows>(ta, tb, tc, args, s);
    default: return VLM_ERR_INVALID_ARG;
  }
}

}  // namespace

namespace {
PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (fn == nullptr) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  }
  return fn;
}
}  // namespace

bool make_tmap_2d(CUtensorMap* map, const void* ptr, bool fp32, uint64_t inner, uint64_t outer, uint64_t row_bytes,
                  uint32_t box_inner, uint32_t box_outer) {
  auto enc = tensor_map_encoder();
  if (enc == nullptr) return false;
  cuuint64_t dims[2] = {inner, outer};
  cuuint64_t strides[1] = {row_bytes};
  cuuint32_t box[2] = {box_inner, box_outer};
  cuuint32_t estr[2] = {1, 1};
  const CUresult r =
      enc(map, fp32 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(ptr),
          dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
          CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

bool make_tmap_2d_bf16(CUtensorMap* map, const void* ptr, uint64_t inner, uint64_t outer, uint64_t row_bytes,
                       uint32_t box_inner, uint32_t box_outer) {
  return make_tmap_2d(map, ptr, false, inner, outer, row_bytes, box_inner, box_outer);
}

bool make_tmap_2d_u8(CUtensorMap* map, const void* ptr, uint64_t inner, uint64_t outer, uint64_t row_bytes,
                     uint32_t box_inner, uint32_t box_outer) {
  auto enc = tensor_map_encoder();
  if (enc == nullptr) return false;
  cuuint64_t dims[2] = {inner, outer};
  cuuint64_t strides[1] = {row_bytes};
  cuuint32_t box[2] = {box_inner, box_outer};
  cuuint32_t estr[2] = {1, 1};
  return enc(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(ptr), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

namespace {
// Tile indices (and, for NVFP4, scale-atom rows) are 32-bit in the kernels and in TMA
// coordinates: reject shapes whose 128 x 128 tile count would not fit.
bool tiles_fit(int64_t M, int64_t N) { return (M + 127) / 128 * ((N + 127) / 128) <= INT32_MAX; }
}  // namespace

int launch_gemm_f8(int epi, const void* a, const void* b, const float* colscale, float out_scale, int64_t M,
                   int64_t N, int64_t K, void* c, void* c_bf16, const int32_t* pos, const float2* rope,
                   int64_t rope_cols, int32_t* status, cudaStream_t s) {
  if (a == nullptr || b == nullptr || c == nullptr || colscale == nullptr) return VLM_ERR_INVALID_ARG;
  if (M <= 0 || N <= 0 || K <= 0 || M > (1LL << 31) - 1 || N > 65535 * 256LL || K > (1 << 20) || !tiles_fit(M, N))
    return VLM_ERR_BAD_SHAPE;
  if (K % 128 != 0 || N % 256 != 0) return VLM_ERR_UNSUPPORTED;
  if (epi != VLM_EPI_BF16 && epi != VLM_EPI_RESID && epi != VLM_EPI_SWIGLU && epi != VLM_EPI_ROPE)
    return VLM_ERR_UNSUPPORTED;
  if (epi == VLM_EPI_ROPE && (pos == nullptr || rope == nullptr || rope_cols % 64 != 0)) return VLM_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(a) | reinterpret_cast<uintptr_t>(b) | reinterpret_cast<uintptr_t>(c) |
       reinterpret_cast<uintptr_t>(colscale)) & 15)
    return VLM_ERR_INVALID_ARG;
  CUtensorMap ta, tb, tc;
  if (!make_tmap_2d_u8(&ta, a, K, M, K, 128, GBM)) return VLM_ERR_CUDA;
  if (!make_tmap_2d_u8(&tb, b, K, N, K, 128, 128)) return VLM_ERR_CUDA;
  // output: 32-row boxes of 128 bytes (64 bf16, 32 fp32 or, for SwiGLU, 128 E4M3 columns)
  bool ok;
  if (epi == VLM_EPI_SWIGLU) ok = make_tmap_2d_u8(&tc, c, N / 2, M, N / 2, 128, 32);
  else if (epi == VLM_EPI_RESID) ok = make_tmap_2d(&tc, c, true, N, M, N * 4, 32, 32);
  else ok = make_tmap_2d(&tc, c, false, N, M, N * 2, 64, 32);
  if (!ok) return VLM_ERR_CUDA;
  GemmArgs args;
  args.M = static_cast<int>(M);
  args.N = static_cast<int>(N);
  args.K = static_cast<int>(K);
  args.m_tiles = static_cast<int>((M + 255) / 256);
  args.n_tiles = static_cast<int>(N / 256);
  args.c = c;
  args.c_bf16 = static_cast<__nv_bfloat16*>(c_bf16);
  args.pos = pos;
  args.rope = rope;
  args.rope_cols = static_cast<int>(rope_cols);
  args.status = status;
  args.colscale = colscale;
  args.out_scale = out_scale;
  return dispatch_pair_f8(epi, ta, tb, tc, args, s);
}

int launch_gemm(int epi, const void* a, const void* b, int64_t M, int64_t N, int64_t K, void* c, void* c_bf16,
                const int32_t* pos, const float2* rope, int64_t rope_cols, int32_t* status, cudaStream_t s) {
  if (a == nullptr || b == nullptr || c == nullptr) return VLM_ERR_INVALID_ARG;
  if (epi < VLM_EPI_BF16 || epi > VLM_EPI_GELU) return VLM_ERR_INVALID_ARG;  // launch_gemm_rows has its own entry
  if (M <= 0 || N <= 0 || K <= 0 || M > (1LL << 31) - 1 || N > 65535 * 256LL || K > (1 << 20) || !tiles_fit(M, N))
    return VLM_ERR_BAD_SHAPE;
  if (K % GBK != 0 || N % 128 != 0) return VLM_ERR_UNSUPPORTED;
  const bool needs256 = epi == VLM_EPI_SWIGLU || epi == VLM_EPI_ROPE;
  if (needs256 && N % 256 != 0) return VLM_ERR_UNSUPPORTED;
  if (epi == VLM_EPI_ROPE && (pos == nullptr || rope == nullptr || rope_cols % 64 != 0)) return VLM_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(a) | reinterpret_cast<uintptr_t>(b) | reinterpret_cast<uintptr_t>(c)) & 15)
    return VLM_ERR_INVALID_ARG;
  const int bn = N % 256 == 0 ? 256 : 128;

  CUtensorMap ta, tb;
  if (!make_tmap_2d_bf16(&ta, a, K, M, K * 2, GBK, GBM)) return VLM_ERR_CUDA;
  if (!make_tmap_2d_bf16(&tb, b, K, N, K * 2, GBK, bn)) return VLM_ERR_CUDA;
  // output: 32-row boxes of 128 bytes (64 bf16 or 32 fp32 columns)
  CUtensorMap tc;
  const bool out_f32 = epi == VLM_EPI_F32 || epi == VLM_EPI_RESID;
  const uint64_t out_cols = epi == VLM_EPI_SWIGLU ? N / 2 : N;
  if (!make_tmap_2d(&tc, c, out_f32, out_cols, M, out_cols * (out_f32 ? 4 : 2), out_f32 ? 32 : 64, 32))
    return VLM_ERR_CUDA;

  GemmArgs args;
  args.M = static_cast<int>(M);
  args.N = static_cast<int>(N);
  args.K = static_cast<int>(K);
  args.m_tiles = static_cast<int>((M + GBM - 1) / GBM);
  args.n_tiles = static_cast<int>(N / bn);
  args.c = c;
  args.c_bf16 = static_cast<__nv_bfloat16*>(c_bf16);
  args.pos = pos;
  args.rope = rope;
  args.rope_cols = static_cast<int>(rope_cols);
  args.status = status;
  args.colscale = nullptr;
  args.out_scale = 1.0f;
  if (bn == 256) {
    // two-SM pairs: 256-row tiles of A (128 per CTA) and 128-row halves of the B tile
    CUtensorMap tb2;
    if (!make_tmap_2d_bf16(&tb2, b, K, N, K * 2, GBK, 128)) return VLM_ERR_CUDA;
    args.m_tiles = static_cast<int>((M + 255) / 256);
    return dispatch_pair(epi, ta, tb2, tc, args, s);
  }
  return dispatch_epi<128>(epi, ta, tb, tc, args, s);
}

int launch_gemm_rows(const void* a, const void* b, int64_t M, int64_t N, int64_t K, void* c, int64_t c_rows,
                     const int64_t* dst_rows, const int32_t* ok_flag, int32_t* status, cudaStream_t s) {
  if (a == nullptr || b == nullptr || c == nullptr || dst_rows == nullptr || ok_flag == nullptr)
    return VLM_ERR_INVALID_ARG;
  if (M <= 0 || N <= 0 || K <= 0 || c_rows <= 0 || M > (1LL << 31) - 1 || N > 65535 * 256LL || K > (1 << 20) ||
      !tiles_fit(M, N))
    return VLM_ERR_BAD_SHAPE;
  if (K % GBK != 0 || N % 128 != 0) return VLM_ERR_UNSUPPORTED;
  if ((reinterpret_cast<uintptr_t>(a) | reinterpret_cast<uintptr_t>(b) | reinterpret_cast<uintptr_t>(c)) & 15)
    return VLM_ERR_INVALID_ARG;
  const int bn = N % 256 == 0 ? 256 : 128;
  CUtensorMap ta, tb, tc;
  if (!make_tmap_2d_bf16(&ta, a, K, M, K * 2, GBK, GBM)) return VLM_ERR_CUDA;
  if (!make_tmap_2d_bf16(&tb, b, K, N, K * 2, GBK, bn == 256 ? 128 : bn)) return VLM_ERR_CUDA;
  // the kernels take an output map; this epilogue stores without it
  if (!make_tmap_2d(&tc, c, false, N, c_rows, N * 2, 64, 1)) return VLM_ERR_CUDA;
  GemmArgs args;
  args.M = static_cast<int>(M);
  args.N = static_cast<int>(N);
  args.K = static_cast<int>(K);
  args.m_tiles = static_cast<int>(bn == 256 ? (M + 255) / 256 : (M + GBM - 1) / GBM);
  args.n_tiles = static_cast<int>(N / bn);
  args.c = c;
  args.c_bf16 = nullptr;
  args.pos = nullptr;
  args.rope = nullptr;
  args.rope_cols = 0;
  args.status = status;
  args.colscale = nullptr;
  args.out_scale = 1.0f;
  args.dst_rows = dst_rows;
  args.ok_flag = ok_flag;
  args.c_rows = c_rows;
  if (bn == 256) return dispatch_pair(kEpiRows, ta, tb, tc, args, s);
  return dispatch_epi<128>(kEpiRows, ta, tb, tc, args, s);
}

namespace {
// Scale atoms as a 2D tensor of 32-bit words: one 512-byte atom per row, four
// atoms (one stage) per box, no swizzle.
bool make_tmap_sf(CUtensorMap* map, const void* ptr, uint64_t atoms) {
  auto enc = tensor_map_encoder();
  if (enc == nullptr) return false;
  cuuint64_t dims[2] = {128, atoms};
  cuuint64_t strides[1] = {512};
  cuuint32_t box[2] = {128, 4};
  cuuint32_t estr[2] = {1, 1};
  return enc(map, CU_TENSOR_MAP_DATA_TYPE_UINT32, 2, const_cast<void*>(ptr), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}
}  // namespace

int launch_gemm_nvfp4_ex(int epi, const uint8_t* a, const uint8_t* a_sf, const float* g_a, const uint8_t* b,
                         const uint8_t* b_sf, const float* g_b, int64_t M, int64_t N, int64_t K, void* c,
                         uint8_t* c_sf, float out_sg, const int32_t* pos, const float2* rope, int64_t rope_cols,
                         int32_t* status, cudaStream_t s) {
  if (a == nullptr || a_sf == nullptr || g_a == nullptr || b == nullptr || b_sf == nullptr || g_b == nullptr ||
      c == nullptr)
    return VLM_ERR_INVALID_ARG;
  if (M <= 0 || N <= 0 || K <= 0 || M > (1LL << 31) - 1 || N > 65535 * 128LL || K > (1 << 20) || !tiles_fit(M, N) ||
      (M + 127) / 128 * (K / 64) > INT32_MAX || N / 128 * (K / 64) > INT32_MAX)
    return VLM_ERR_BAD_SHAPE;
  if (K % 256 != 0 || N % 128 != 0) return VLM_ERR_UNSUPPORTED;
  if (epi != VLM_EPI_BF16 && epi != VLM_EPI_RESID && epi != VLM_EPI_ROPE && epi != VLM_EPI_SWIGLU)
    return VLM_ERR_UNSUPPORTED;
  const bool needs256 = epi == VLM_EPI_ROPE || epi == VLM_EPI_SWIGLU;
  if (needs256 && N % 256 != 0) return VLM_ERR_UNSUPPORTED;
  if (epi == VLM_EPI_ROPE && (pos == nullptr || rope == nullptr || rope_cols < 0 || rope_cols % 64 != 0))
    return VLM_ERR_INVALID_ARG;
  if (epi == VLM_EPI_SWIGLU && (c_sf == nullptr || !(out_sg > 0.f) || (reinterpret_cast<uintptr_t>(c_sf) & 3)))
    return VLM_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(a) | reinterpret_cast<uintptr_t>(b) | reinterpret_cast<uintptr_t>(a_sf) |
       reinterpret_cast<uintptr_t>(b_sf) | reinterpret_cast<uintptr_t>(c)) & 15)
    return VLM_ERR_INVALID_ARG;
  const int bn = N % 256 == 0 ? 256 : 128;
  CUtensorMap ta, tb, tsa, tsb, tc;
  if (!make_tmap_2d_u8(&ta, a, K / 2, M, K / 2, 128, GBM)) return VLM_ERR_CUDA;
  if (!make_tmap_2d_u8(&tb, b, K / 2, N, K / 2, 128, bn / 2)) return VLM_ERR_CUDA;
  if (!make_tmap_sf(&tsa, a_sf, static_cast<uint64_t>((M + 127) / 128 * (K / 64)))) return VLM_ERR_CUDA;
  if (!make_tmap_sf(&tsb, b_sf, static_cast<uint64_t>(N / 128 * (K / 64)))) return VLM_ERR_CUDA;
  // the SwiGLU epilogue stores codes from registers: its output map is never used
  const bool ok = epi == VLM_EPI_RESID    ? make_tmap_2d(&tc, c, true, N, M, N * 4, 32, 32)
                  : epi == VLM_EPI_SWIGLU ? make_tmap_2d_u8(&tc, c, N / 4, M, N / 4, 64, 32)
                                          : make_tmap_2d(&tc, c, false, N, M, N * 2, 64, 32);
  if (!ok) return VLM_ERR_CUDA;
  GemmArgs args;
  args.M = static_cast<int>(M);
  args.N = static_cast<int>(N);
  args.K = static_cast<int>(K);
  args.m_tiles = static_cast<int>((M + 255) / 256);
  args.n_tiles = static_cast<int>(N / bn);
  args.c = c;
  args.c_bf16 = nullptr;
  args.pos = pos;
  args.rope = rope;
  args.rope_cols = static_cast<int>(rope_cols);
  args.status = status;
  args.colscale = nullptr;
  args.out_scale = out_sg;
  args.g_a = g_a;
  args.g_b = g_b;
  args.c_sf = c_sf;
  if (bn == 256) {
    switch (epi) {
      case VLM_EPI_RESID: return run_gemm_nvfp4<VLM_EPI_RESID, 256>(ta, tb, tsa, tsb, tc, args, s);
      case VLM_EPI_ROPE: return run_gemm_nvfp4<VLM_EPI_ROPE, 256>(ta, tb, tsa, tsb, tc, args, s);
      case VLM_EPI_SWIGLU: return run_gemm_nvfp4<VLM_EPI_SWIGLU, 256>(ta, tb, tsa, tsb, tc, args, s);
      default: return run_gemm_nvfp4<VLM_EPI_BF16, 256>(ta, tb, tsa, tsb, tc, args, s);
    }
  }
  return epi == VLM_EPI_RESID ? run_gemm_nvfp4<VLM_EPI_RESID, 128>(ta, tb, tsa, tsb, tc, args, s)
                              : run_gemm_nvfp4<VLM_EPI_BF16, 128>(ta, tb, tsa, tsb, tc, args, s);
}

int launch_gemm_nvfp4(int epi, const uint8_t* a, const uint8_t* a_sf, const float* g_a, const uint8_t* b,
                      const uint8_t* b_sf, const float* g_b, int64_t M, int64_t N, int64_t K, void* c,
                      int32_t* status, cudaStream_t s) {
  if (epi != VLM_EPI_BF16 && epi != VLM_EPI_RESID) return VLM_ERR_UNSUPPORTED;
  return launch_gemm_nvfp4_ex(epi, a, a_sf, g_a, b, b_sf, g_b, M, N, K, c, nullptr, 1.0f, nullptr, nullptr, 0,
                              status, s);
}

}  // namespace vlm
