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
//   warps 2..5  epilogue: tcgen05.ld of the accumulator (warp w reads TMEM
//               lanes 32*(w%4)..+31), math, vectorised global stores.
// Two TMEM accumulators (2 x BN columns) let the epilogue of tile i overlap the
// MMAs of tile i+1. Tiles are handed out statically (tile += gridDim.x) over a
// grid of one CTA per SM. No TMA multicast is used.
#include <cudaTypedefs.h>

#include "kernels.cuh"

namespace vlm {

namespace {

constexpr int GBM = 128;
constexpr int GBK = 64;

struct GemmArgs {
  int M, N, K;
  int m_tiles, n_tiles;
  void* c;
  __nv_bfloat16* c_bf16;
  const int32_t* pos;
  const float2* rope;
  int rope_cols;
  int32_t* status;
};

template <int BN>
struct GemmShape {
  static constexpr int STAGES = BN == 256 ? 4 : 6;
  static constexpr int A_BYTES = GBM * GBK * 2;
  static constexpr int B_BYTES = BN * GBK * 2;
  static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
  static constexpr int TMEM_COLS = 2 * BN;
  static constexpr int BAR_BYTES = 256;
  static constexpr int SMEM_BYTES = STAGES * STAGE_BYTES + BAR_BYTES + 1024;
};

__device__ __forceinline__ float silu_f(float z) { return z / (1.0f + __expf(-z)); }
__device__ __forceinline__ float gelu_f(float z) { return 0.5f * z * (1.0f + erff(z * 0.70710678118654752f)); }

template <int EPI>
__device__ __forceinline__ float act(float v) {
  if constexpr (EPI == VLM_EPI_GELU) return gelu_f(v);
  return v;
}

// Epilogue of one 128 x BN tile for this thread's row.
template <int BN, int EPI>
__device__ __forceinline__ void epilogue_tile(const GemmArgs& args, uint32_t tbase, int row, int n0) {
  const bool live = row < args.M;
  if constexpr (EPI == VLM_EPI_BF16 || EPI == VLM_EPI_GELU) {
    __nv_bfloat16* out = static_cast<__nv_bfloat16*>(args.c) + static_cast<int64_t>(row) * args.N + n0;
#pragma unroll 1
    for (int c = 0; c < BN; c += 32) {
      uint32_t r[32];
      tmem_ld32(tbase + c, r);
      if (live) {
        uint4* dst = reinterpret_cast<uint4*>(out + c);
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          uint4 v;
          v.x = pack_bf16x2(act<EPI>(__uint_as_float(r[8 * j + 0])), act<EPI>(__uint_as_float(r[8 * j + 1])));
          v.y = pack_bf16x2(act<EPI>(__uint_as_float(r[8 * j + 2])), act<EPI>(__uint_as_float(r[8 * j + 3])));
          v.z = pack_bf16x2(act<EPI>(__uint_as_float(r[8 * j + 4])), act<EPI>(__uint_as_float(r[8 * j + 5])));
          v.w = pack_bf16x2(act<EPI>(__uint_as_float(r[8 * j + 6])), act<EPI>(__uint_as_float(r[8 * j + 7])));
          dst[j] = v;
        }
      }
    }
  } else if constexpr (EPI == VLM_EPI_F32 || EPI == VLM_EPI_RESID) {
    float* out = static_cast<float*>(args.c) + static_cast<int64_t>(row) * args.N + n0;
    __nv_bfloat16* outb = args.c_bf16 ? args.c_bf16 + static_cast<int64_t>(row) * args.N + n0 : nullptr;
#pragma unroll 1
    for (int c = 0; c < BN; c += 32) {
      uint32_t r[32];
      tmem_ld32(tbase + c, r);
      if (live) {
        float4* dst = reinterpret_cast<float4*>(out + c);
        float4 v[8];
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          v[j] = make_float4(__uint_as_float(r[4 * j]), __uint_as_float(r[4 * j + 1]),
                             __uint_as_float(r[4 * j + 2]), __uint_as_float(r[4 * j + 3]));
          if constexpr (EPI == VLM_EPI_RESID) {
            const float4 o = dst[j];
            v[j].x += o.x; v[j].y += o.y; v[j].z += o.z; v[j].w += o.w;
          }
          dst[j] = v[j];
        }
        if (outb != nullptr) {
          uint4* db = reinterpret_cast<uint4*>(outb + c);
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            uint4 u;
            u.x = pack_bf16x2(v[2 * j].x, v[2 * j].y);
            u.y = pack_bf16x2(v[2 * j].z, v[2 * j].w);
            u.z = pack_bf16x2(v[2 * j + 1].x, v[2 * j + 1].y);
            u.w = pack_bf16x2(v[2 * j + 1].z, v[2 * j + 1].w);
            db[j] = u;
          }
        }
      }
    }
  } else if constexpr (EPI == VLM_EPI_SWIGLU) {
    // columns 32j..32j+15 are gate, 32j+16..32j+31 the matching up values
    __nv_bfloat16* out = static_cast<__nv_bfloat16*>(args.c) + static_cast<int64_t>(row) * (args.N / 2) + n0 / 2;
#pragma unroll 1
    for (int c = 0; c < BN; c += 32) {
      uint32_t r[32];
      tmem_ld32(tbase + c, r);
      if (live) {
        uint4* dst = reinterpret_cast<uint4*>(out + c / 2);
#pragma unroll
        for (int j = 0; j < 2; ++j) {
          uint32_t w[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const int i = 8 * j + 2 * e;
            const float h0 = silu_f(__uint_as_float(r[i])) * __uint_as_float(r[16 + i]);
            const float h1 = silu_f(__uint_as_float(r[i + 1])) * __uint_as_float(r[16 + i + 1]);
            w[e] = pack_bf16x2(h0, h1);
          }
          dst[j] = make_uint4(w[0], w[1], w[2], w[3]);
        }
      }
    }
  } else if constexpr (EPI == VLM_EPI_ROPE) {
    __nv_bfloat16* out = static_cast<__nv_bfloat16*>(args.c) + static_cast<int64_t>(row) * args.N + n0;
    const int pk = live ? __ldg(args.pos + row) : 0;
    const int pr = pk >> 16, pc = pk & 0xFFFF;
#pragma unroll 1
    for (int c = 0; c < BN; c += 64) {
      uint32_t a[32], b[32];
      tmem_ld32(tbase + c, a);
      tmem_ld32(tbase + c + 32, b);
      if (live) {
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
        uint4* dst = reinterpret_cast<uint4*>(out + c);
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          dst[j] = make_uint4(pack_bf16x2(x[8 * j], x[8 * j + 1]), pack_bf16x2(x[8 * j + 2], x[8 * j + 3]),
                              pack_bf16x2(x[8 * j + 4], x[8 * j + 5]), pack_bf16x2(x[8 * j + 6], x[8 * j + 7]));
          dst[4 + j] = make_uint4(pack_bf16x2(y[8 * j], y[8 * j + 1]), pack_bf16x2(y[8 * j + 2], y[8 * j + 3]),
                                  pack_bf16x2(y[8 * j + 4], y[8 * j + 5]), pack_bf16x2(y[8 * j + 6], y[8 * j + 7]));
        }
      }
    }
  }
}

template <int BN, int EPI>
__global__ void __launch_bounds__(192, 1)
    gemm_tcgen05_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                        const GemmArgs args) {
  using S = GemmShape<BN>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sA = smem;
  uint8_t* sB = smem + S::STAGES * S::A_BYTES;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + S::STAGES * S::STAGE_BYTES);
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
    int acc = 0;
    uint32_t acc_phase = 0;
    for (int tile = blockIdx.x; tile < total_tiles; tile += gridDim.x) {
      const int mt = tile / args.n_tiles, nt = tile - mt * args.n_tiles;
      if (!mbar_wait_warp(smem_u32(tfull + acc), acc_phase, abort_v, args.status)) break;
      tc_fence_after();
      const int row = mt * GBM + q * 32 + lane;
      const uint32_t tbase = tmem_base + (static_cast<uint32_t>(q * 32) << 16) + static_cast<uint32_t>(acc * BN);
      epilogue_tile<BN, EPI>(args, tbase, row, nt * BN);
      tc_fence_before();
      mbar_arrive(smem_u32(tempty + acc));
      acc ^= 1;
      if (acc == 0) acc_phase ^= 1u;
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, S::TMEM_COLS);
  }
}

template <int BN, int EPI>
int run_gemm(const CUtensorMap& ta, const CUtensorMap& tb, const GemmArgs& args, cudaStream_t s) {
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
  const int grid = tiles < num_sms() ? tiles : num_sms();
  launch_begin(KC_GEMM, s);
  kern<<<grid, 192, S::SMEM_BYTES, s>>>(ta, tb, args);
  launch_end(KC_GEMM, s);
  return cudaGetLastError() == cudaSuccess ? VLM_OK : VLM_ERR_CUDA;
}

template <int BN>
int dispatch_epi(int epi, const CUtensorMap& ta, const CUtensorMap& tb, const GemmArgs& args, cudaStream_t s) {
  switch (epi) {
    case VLM_EPI_BF16: return run_gemm<BN, VLM_EPI_BF16>(ta, tb, args, s);
    case VLM_EPI_F32: return run_gemm<BN, VLM_EPI_F32>(ta, tb, args, s);
    case VLM_EPI_RESID: return run_gemm<BN, VLM_EPI_RESID>(ta, tb, args, s);
    case VLM_EPI_SWIGLU: return run_gemm<BN, VLM_EPI_SWIGLU>(ta, tb, args, s);
    case VLM_EPI_ROPE: return run_gemm<BN, VLM_EPI_ROPE>(ta, tb, args, s);
    case VLM_EPI_GELU: return run_gemm<BN, VLM_EPI_GELU>(ta, tb, args, s);
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

bool make_tmap_2d_bf16(CUtensorMap* map, const void* ptr, uint64_t inner, uint64_t outer, uint64_t row_bytes,
                       uint32_t box_inner, uint32_t box_outer) {
  auto enc = tensor_map_encoder();
  if (enc == nullptr) return false;
  cuuint64_t dims[2] = {inner, outer};
  cuuint64_t strides[1] = {row_bytes};
  cuuint32_t box[2] = {box_inner, box_outer};
  cuuint32_t estr[2] = {1, 1};
  const CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(ptr), dims, strides, box,
                         estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                         CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

int launch_gemm(int epi, const void* a, const void* b, int64_t M, int64_t N, int64_t K, void* c, void* c_bf16,
                const int32_t* pos, const float2* rope, int64_t rope_cols, int32_t* status, cudaStream_t s) {
  if (a == nullptr || b == nullptr || c == nullptr) return VLM_ERR_INVALID_ARG;
  if (M <= 0 || N <= 0 || K <= 0 || M > (1LL << 31) - 1 || N > 65535 * 256LL || K > (1 << 20))
    return VLM_ERR_BAD_SHAPE;
  if (K % GBK != 0 || N % 128 != 0) return VLM_ERR_UNSUPPORTED;
  const bool needs256 = epi == VLM_EPI_SWIGLU || epi == VLM_EPI_ROPE;
  if (needs256 && N % 256 != 0) return VLM_ERR_UNSUPPORTED;
  if (epi == VLM_EPI_ROPE && (pos == nullptr || rope == nullptr || rope_cols % 64 != 0)) return VLM_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(a) | reinterpret_cast<uintptr_t>(b) | reinterpret_cast<uintptr_t>(c)) & 15)
    return VLM_ERR_INVALID_ARG;
  const int bn = (needs256 || (N % 256 == 0 && N >= 2048)) ? 256 : 128;

  CUtensorMap ta, tb;
  if (!make_tmap_2d_bf16(&ta, a, K, M, K * 2, GBK, GBM)) return VLM_ERR_CUDA;
  if (!make_tmap_2d_bf16(&tb, b, K, N, K * 2, GBK, bn)) return VLM_ERR_CUDA;

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
  return bn == 256 ? dispatch_epi<256>(epi, ta, tb, args, s) : dispatch_epi<128>(epi, ta, tb, args, s);
}

}  // namespace vlm
