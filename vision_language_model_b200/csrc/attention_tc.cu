// Block-diagonal (per-image) bidirectional attention on the sm_100a tensor
// cores, head_dim 64: for query t of block b,
//   o_t = sum_u softmax_u(q_t . k_u / 8) v_u   over the keys u of block b only.
//
// One CTA = one 128-query tile of one block and one head; two CTAs share an
// SM so one CTA's softmax overlaps the other's MMAs. 10 warps:
//   warp 0      TMA: the Q tile once, then K and V tiles of 128 keys into two
//               2-stage rings (128-byte swizzle). A K stage is released when
//               S = Q K^T has read it and a V stage when O += P V has, so the
//               next K load never waits for a P V product.
//   warp 1      allocates 256 TMEM columns; one thread issues
//                 S  = Q K^T      (tcgen05.mma kind::f16, M=128 N=128, A and B in smem)
//                 O += P V        (M=128 N=64, A = P in TMEM, B = V in smem, MN-major)
//               S_{j+1} is issued as soon as the softmax has copied S_j out.
//   warps 2..9  softmax, two threads per query row (TMEM lane): warp w and
//               warp w + 4 read the same 32 lanes, keys [0,64) and [64,128) of
//               the tile (64 fp32 each). Each finds its half's max with four
//               short 3-input-max chains; the two halves exchange them through
//               shared memory (a 64-thread named barrier per row group), so
//               both keep the same running max m (log2 units), which only
//               moves when the tile max exceeds it by more than 8 (otherwise
//               the stale max is kept; P stays <= 2^8 and the final division
//               by l is exact). Each computes its 64 P = 2^(s*log2e/8 - m) with
//               packed fp32x2 FMAs and MUFU ex2 (one pair in eight from an
//               FMA-pipe polynomial), writes them to TMEM as bf16, sums the
//               fp32 values into its part of l with packed adds, rescales its
//               32 O columns when m moved, and finally writes those columns
//               of O / l (l = the sum of both parts).
// TMEM: S in columns [0,128), P in [128,192) (bf16 pairs), O in [192,256).
// Keys past the block end are masked to -inf; their V rows are finite (rows of
// the next block) or TMA zero fill (past the sequence). Query tiles never
// straddle two blocks, so every block's result is independent of the others.
#include <algorithm>

#include "exp2_poly.cuh"
#include "kernels.cuh"
#include "nvfp4.cuh"

#define VLM_DEBUG_FILE_ID 3

namespace vlm {

VLM_DEBUG_UNIT(debug_word_attention)

namespace {

constexpr int BQ = kAttnBQ;  // 128
constexpr int BKV = 128;
constexpr int DH = 64;
constexpr int HK = BKV / 2;  // keys per softmax thread
constexpr int kThreads = 320;
constexpr int kKStages = 2;  // K ring: a stage is free once S = Q K^T has read it
constexpr int kVStages = 2;  // V ring: a stage is free once O += P V has read it
constexpr int kTileBytes = 128 * DH * 2;  // 16 KiB: 128 rows x 128 bytes
constexpr int kXchOffset = (1 + kKStages + kVStages) * kTileBytes + 256;
constexpr int kSmemBytes = kXchOffset + 3072 + 1024;
constexpr uint32_t kColS = 0, kColP = 128, kColO = 192, kTmemCols = 256;
constexpr float kRescaleThreshold = 8.0f;  // log2 units

__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ float max3f(float a, float b, float c) {
  float r;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}

// Packed pairs of fp32 (first value in the low word) for the f32x2 instructions.
__device__ __forceinline__ uint64_t pack2(uint32_t lo, uint32_t hi) {
  uint64_t r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "r"(lo), "r"(hi));
  return r;
}
__device__ __forceinline__ uint64_t pair_f32(float v) { return pack2(__float_as_uint(v), __float_as_uint(v)); }
__device__ __forceinline__ void unpack2(uint64_t v, float& lo, float& hi) {
  asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
}
__device__ __forceinline__ uint64_t fma2(uint64_t a, uint64_t b, uint64_t c) {
  uint64_t d;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
  return d;
}
__device__ __forceinline__ uint64_t add2(uint64_t a, uint64_t b) {
  uint64_t d;
  asm("add.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}

// Row maximum of N values with four independent chains of 3-input max.
template <int N>
__device__ __forceinline__ float row_max(const uint32_t (&u)[N]) {
  constexpr int NC = 4;
  float m[NC];
#pragma unroll
  for (int i = 0; i < NC; ++i) m[i] = -INFINITY;
#pragma unroll
  for (int c = 0; c < N; c += 2 * NC) {
#pragma unroll
    for (int i = 0; i < NC; ++i) m[i] = max3f(m[i], __uint_as_float(u[c + 2 * i]), __uint_as_float(u[c + 2 * i + 1]));
  }
#pragma unroll
  for (int w = NC / 2; w > 0; w /= 2)
#pragma unroll
    for (int i = 0; i < w; ++i) m[i] = fmaxf(m[i], m[i + w]);
  return m[0];
}

// 32 lanes x 64 columns of 32-bit TMEM words into registers (one lane per
// thread), waiting for completion inside the same asm block.
__device__ __forceinline__ void tmem_ld64(uint32_t taddr, uint32_t (&r)[64]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x64.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, "
      "%16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31, "
      "%32, %33, %34, %35, %36, %37, %38, %39, %40, %41, %42, %43, %44, %45, %46, %47, "
      "%48, %49, %50, %51, %52, %53, %54, %55, %56, %57, %58, %59, %60, %61, %62, %63}, [%64];\n\t"
      "tcgen05.wait::ld.sync.aligned;"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
        "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
        "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31]),
        "=r"(r[32]), "=r"(r[33]), "=r"(r[34]), "=r"(r[35]), "=r"(r[36]), "=r"(r[37]), "=r"(r[38]), "=r"(r[39]),
        "=r"(r[40]), "=r"(r[41]), "=r"(r[42]), "=r"(r[43]), "=r"(r[44]), "=r"(r[45]), "=r"(r[46]), "=r"(r[47]),
        "=r"(r[48]), "=r"(r[49]), "=r"(r[50]), "=r"(r[51]), "=r"(r[52]), "=r"(r[53]), "=r"(r[54]), "=r"(r[55]),
        "=r"(r[56]), "=r"(r[57]), "=r"(r[58]), "=r"(r[59]), "=r"(r[60]), "=r"(r[61]), "=r"(r[62]), "=r"(r[63])
      : "r"(taddr)
      : "memory");
}

// The two softmax warps of one row group (warps w and w + 4) meet here: a
// named barrier of 64 threads, id 1 + the TMEM lane group.
__device__ __forceinline__ void pair_sync(int q) {
  asm volatile("bar.sync %0, 64;" ::"r"(1 + q) : "memory");
}

// One pair of scores in kPolyPairEvery takes its two exponentials from
// exp2_poly (FMA and ALU pipes) instead of ex2.approx (MUFU), so the two kinds
// of pipe share the softmax's exponentials. MUFU is the softmax's bottleneck;
// one pair in eight measured fastest: one in four fits the 96 registers a
// thread has at 2 CTAs of 320 threads per SM but is no faster, one in three
// spills.
#ifndef VLM_ATTN_POLY_PAIR_EVERY
#define VLM_ATTN_POLY_PAIR_EVERY 8
#endif
constexpr int kPolyPairEvery = VLM_ATTN_POLY_PAIR_EVERY;

// 2^x without MUFU: k = round(x) by adding 1.5 * 2^23, f = x - k in
// [-1/2, 1/2], 2^f from the degree-3 minimax polynomial of exp2_poly.cuh
// (relative error < 7.5e-5, fitted by fit_exp2_poly.py with the Remez
// algorithm), then k added to the exponent field. Scalar arithmetic with
// immediate constants (no register pairs). x is clamped to -126 so the
// exponent cannot wrap; the result is then ~1e-38 instead of 0, so keys that
// must weigh exactly 0 never take this path.
__device__ __forceinline__ float exp2_poly(float x) {
  x = fmaxf(x, -126.0f);
  const float j = x + 12582912.0f;
  const float f = x - (j - 12582912.0f);
  const float p = fmaf(fmaf(fmaf(kExp2C3, f, kExp2C2), f, kExp2C1), f, kExp2C0);
  return __int_as_float(__float_as_int(p) + (__float_as_int(j) << 23));
}

// p_c = 2^(s_c * sl2 - m) for the thread's N scores of the row, packed as bf16 pairs into
// pk; returns sum_c p_c (fp32, before rounding). The elements are independent.
// kPoly: let exp2_poly take one pair in kPolyPairEvery (never on a tile with
// masked keys, whose weights must be exactly 0).
template <bool kPoly, int N>
__device__ __forceinline__ float row_exp(const uint32_t (&u)[N], uint64_t sl2x2, float m, uint32_t (&pk)[N / 2]) {
  const uint64_t negm2 = pair_f32(-m);
  uint64_t acc[4] = {0, 0, 0, 0};
#pragma unroll
  for (int c = 0; c < N; c += 2) {
    float x0, x1, p0, p1;
    unpack2(fma2(pack2(u[c], u[c + 1]), sl2x2, negm2), x0, x1);
    if (kPoly && kPolyPairEvery > 0 && (c >> 1) % (kPolyPairEvery > 0 ? kPolyPairEvery : 1) == kPolyPairEvery - 1) {
      p0 = exp2_poly(x0);
      p1 = exp2_poly(x1);
    } else {
      p0 = ex2(x0);
      p1 = ex2(x1);
    }
    const int i = (c >> 1) & 3;
    acc[i] = add2(acc[i], pack2(__float_as_uint(p0), __float_as_uint(p1)));
    pk[c >> 1] = pack_bf16x2(p0, p1);
  }
  float s0, s1, s2, s3, s4, s5, s6, s7;
  unpack2(acc[0], s0, s1);
  unpack2(acc[1], s2, s3);
  unpack2(acc[2], s4, s5);
  unpack2(acc[3], s6, s7);
  return ((s0 + s1) + (s2 + s3)) + ((s4 + s5) + (s6 + s7));
}

struct AttnArgs {
  const int32_t* cu;
  const int32_t* qt;
  int n_blocks;
  int heads;
  void* out;        // bf16; E4M3 (OUT 1); NVFP4 codes (OUT 2)
  int32_t* status;
  float f8_scale;   // E4M3 output: O / l times this before rounding; NVFP4: the global scale
  uint8_t* out_sf;  // NVFP4 block scales
  int tile_base;    // query tile of blockIdx.x == 0 (launches split along the query tiles)
};

// OUT: 0 bf16, 1 E4M3, 2 NVFP4 output.
template <int OUT>
__global__ void __launch_bounds__(kThreads, 2)
    attn_tc_kernel(const __grid_constant__ CUtensorMap tm_qkv, const AttnArgs args) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sQ = smem;
  uint8_t* sK = smem + kTileBytes;                     // [kKStages] tiles
  uint8_t* sV = smem + (1 + kKStages) * kTileBytes;    // [kVStages] tiles
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + (1 + kKStages + kVStages) * kTileBytes);
  uint64_t* q_full = bars;
  uint64_t* k_full = bars + 1;                          // [kKStages]
  uint64_t* k_empty = k_full + kKStages;                // [kKStages]
  uint64_t* v_full = k_empty + kKStages;                // [kVStages]
  uint64_t* v_empty = v_full + kVStages;                // [kVStages]
  uint64_t* s_full = v_empty + kVStages;
  uint64_t* s_free = s_full + 1;
  uint64_t* p_full = s_full + 2;
  uint64_t* o_done = s_full + 3;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(o_done + 1);
  int* abort_flag = reinterpret_cast<int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;


  if (threadIdx.x == 0) {
    mbar_init(smem_u32(q_full), 1);
    for (int s = 0; s < kKStages; ++s) {
      mbar_init(smem_u32(k_full + s), 1);
      mbar_init(smem_u32(k_empty + s), 1);
    }
    for (int s = 0; s < kVStages; ++s) {
      mbar_init(smem_u32(v_full + s), 1);
      mbar_init(smem_u32(v_empty + s), 1);
    }
    mbar_init(smem_u32(s_full), 1);
    mbar_init(smem_u32(s_free), 256);
    mbar_init(smem_u32(p_full), 256);
    mbar_init(smem_u32(o_done), 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) prefetch_tmap(&tm_qkv);
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_slot), kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  volatile int* abort_v = abort_flag;
  griddep_wait();  // the block tables, q, k, v and the output belong to the previous kernels until here
  griddep_launch_dependents();

  // this CTA's block, query tile and head
  const int tile = blockIdx.x + args.tile_base, h = blockIdx.y;
  int lo = 0, hi = args.n_blocks - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (__ldg(args.qt + mid) <= tile) lo = mid; else hi = mid - 1;
  }
  const int kbeg = __ldg(args.cu + lo), kend = __ldg(args.cu + lo + 1);
  const int q0 = kbeg + (tile - __ldg(args.qt + lo)) * BQ;
  const int n_kv = (kend - kbeg + BKV - 1) / BKV;
  const int D = args.heads * DH;

  if (warp == 0) {
    if (lane == 0) {
      const uint32_t qb = smem_u32(q_full);
      mbar_arrive_expect_tx(qb, kTileBytes);
      tma_load_2d(smem_u32(sQ), &tm_qkv, qb, h * DH, q0);
      // K tile j, then V tile j - 1: V is needed only after the softmax of its tile,
      // so a V stage still being read never holds back the next K load
      for (int j = 0; j <= n_kv; ++j) {
        if (j < n_kv) {
          const int st = j % kKStages;
          if (!mbar_wait(smem_u32(k_empty + st), ((j / kKStages) & 1) ^ 1, abort_v, args.status)) break;
          const uint32_t fb = smem_u32(k_full + st);
          mbar_arrive_expect_tx(fb, kTileBytes);
          tma_load_2d(smem_u32(sK + st * kTileBytes), &tm_qkv, fb, D + h * DH, kbeg + j * BKV);
        }
        if (j > 0) {
          const int jv = j - 1, st = jv % kVStages;
          if (!mbar_wait(smem_u32(v_empty + st), ((jv / kVStages) & 1) ^ 1, abort_v, args.status)) break;
          const uint32_t fb = smem_u32(v_full + st);
          mbar_arrive_expect_tx(fb, kTileBytes);
          tma_load_2d(smem_u32(sV + st * kTileBytes), &tm_qkv, fb, 2 * D + h * DH, kbeg + jv * BKV);
        }
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      constexpr uint32_t idesc_s = idesc_bf16(BQ, BKV);
      constexpr uint32_t idesc_o = idesc_bf16(BQ, DH, /*b_mn_major=*/true);
      bool ok = mbar_wait(smem_u32(q_full), 0, abort_v, args.status);
      const uint64_t qdesc = smem_desc_sw128(smem_u32(sQ));
      for (int j = 0; ok && j <= n_kv; ++j) {
        if (j < n_kv) {
          const int st = j % kKStages;
          if (!mbar_wait(smem_u32(k_full + st), (j / kKStages) & 1, abort_v, args.status)) break;
          if (j > 0 && !mbar_wait(smem_u32(s_free), (j - 1) & 1, abort_v, args.status)) break;
          tc_fence_after();
          const uint64_t kdesc = smem_desc_sw128(smem_u32(sK + st * kTileBytes));
#pragma unroll
          for (int k = 0; k < DH / 16; ++k)
            umma_bf16_ss(tmem + kColS, qdesc + 2 * k, kdesc + 2 * k, idesc_s, k > 0 ? 1u : 0u);
          umma_commit(smem_u32(s_full));
          umma_commit(smem_u32(k_empty + st));
        }
        if (j > 0) {
          const int jp = j - 1, st = jp % kVStages;
          if (!mbar_wait(smem_u32(p_full), jp & 1, abort_v, args.status)) break;
          if (!mbar_wait(smem_u32(v_full + st), (jp / kVStages) & 1, abort_v, args.status)) break;
          tc_fence_after();
          const uint64_t vdesc = smem_desc_sw128(smem_u32(sV + st * kTileBytes));
#pragma unroll
          for (int kk = 0; kk < BKV / 16; ++kk)  // 16 keys = 8 TMEM columns of bf16 pairs = 2048 smem bytes
            umma_bf16_ts(tmem + kColO, tmem + kColP + 8 * kk, vdesc + 128 * kk, idesc_o,
                         (jp > 0 || kk > 0) ? 1u : 0u);
          umma_commit(smem_u32(v_empty + st));
          umma_commit(smem_u32(o_done));
        }
      }
    }
  } else {
    // softmax, warps 2..9: warp w and warp w + 4 own the same 32 query rows
    // (TMEM lanes 32 (w % 4) ..), keys [0, 64) and [64, 128) of every tile. The
    // pair agrees on the row maximum through shared memory; each keeps its own
    // part of the row sum and owns 32 of the 64 O columns.
    const int q = warp & 3;
    const int hf = (warp - 2) >> 2;
    const int r = q * 32 + lane;
    const uint32_t trow = tmem + (static_cast<uint32_t>(q * 32) << 16);
    float* xmax = reinterpret_cast<float*>(smem + kXchOffset);  // [tile parity][half][row]
    float* xsum = xmax + 512;                                   // [half][row]
    const float sl2 = 1.4426950408889634f * 0.125f;  // log2(e) / sqrt(64)
    const uint64_t sl2x2 = pair_f32(sl2);
    float m = -INFINITY, l = 0.f;
    bool ok = true;
    // A warp whose wait failed stays in the loop and keeps meeting its partner
    // at pair_sync, doing nothing else, so the partner never waits for it.
    for (int j = 0; j < n_kv; ++j) {
      if (ok) ok = mbar_wait_warp(smem_u32(s_full), j & 1, abort_v, args.status);
      if (!ok) {
        pair_sync(q);
        continue;
      }
      tc_fence_after();
      uint32_t u[HK];
      tmem_ld64(trow + kColS + HK * hf, u);
      tc_fence_before();
      mbar_arrive(smem_u32(s_free));
      const int nvalid = kend - (kbeg + j * BKV) - HK * hf;
      if (nvalid < HK) {  // keys past the block end get probability 0
#pragma unroll
        for (int c = 0; c < HK; ++c)
          if (c >= nvalid) u[c] = __float_as_uint(-INFINITY);
      }
      const float m_own = row_max(u) * sl2;
      xmax[((j & 1) * 2 + hf) * BQ + r] = m_own;
      pair_sync(q);
      const float m_cand = fmaxf(m_own, xmax[((j & 1) * 2 + (hf ^ 1)) * BQ + r]);
      const bool grow = m_cand > m + kRescaleThreshold;
      const float m_new = grow ? m_cand : m;
      const float corr = grow ? ex2(m - m_new) : 1.0f;
      const bool any_grow = __any_sync(0xffffffffu, grow);
      m = m_new;
      uint32_t pk[HK / 2];
      const float sum = nvalid < HK ? row_exp<false>(u, sl2x2, m, pk) : row_exp<true>(u, sl2x2, m, pk);
      l = l * corr + sum;

      if (j > 0) {
        // PV of the previous tile must be done before O is rescaled and P overwritten
        ok = mbar_wait_warp(smem_u32(o_done), (j - 1) & 1, abort_v, args.status);
        if (!ok) continue;
        tc_fence_after();
      }
      tmem_st32(trow + kColP + 32 * hf, pk);
      if (j > 0 && any_grow) {
        uint32_t o[32];
        tmem_ld32(trow + kColO + 32 * hf, o);
#pragma unroll
        for (int i = 0; i < 32; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * corr);
        tmem_st32(trow + kColO + 32 * hf, o);
      }
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(smem_u32(p_full));
    }
    xsum[hf * BQ + r] = l;
    pair_sync(q);
    l += xsum[(hf ^ 1) * BQ + r];
    if (ok && mbar_wait_warp(smem_u32(o_done), (n_kv - 1) & 1, abort_v, args.status)) {
      tc_fence_after();
      const float inv = 1.0f / l;
      const int row = q0 + r;
      const int c = 32 * hf;  // this thread's O columns
      if constexpr (OUT == 2) {
        // blocks of 16 values along the row: four per head, two per 32-column load
        uint8_t* dst = static_cast<uint8_t*>(args.out) + static_cast<int64_t>(row) * (D / 2) + h * (DH / 2);
        const float sg = args.f8_scale, six_sg = 6.0f * sg;
        uint32_t o[32];
        tmem_ld32(trow + kColO + c, o);
        if (row < kend && VLM_DCHECK(kend <= __ldg(args.cu + args.n_blocks))) {
          uint32_t sbs = 0;
          uint2 codes[2];
#pragma unroll
          for (int b = 0; b < 2; ++b) {
            float v[16], amax = 0.0f;
#pragma unroll
            for (int k = 0; k < 16; ++k) {
              v[k] = __uint_as_float(o[16 * b + k]) * inv;
              amax = fmaxf(amax, fabsf(v[k]));
            }
            sbs |= nvfp4_quant16(v, amax, sg, six_sg, codes[b]) << (8 * b);
          }
          *reinterpret_cast<uint4*>(dst + c / 2) = make_uint4(codes[0].x, codes[0].y, codes[1].x, codes[1].y);
          // blocks (h DH + c) / 16 and the next: two adjacent scale bytes
          *reinterpret_cast<uint16_t*>(args.out_sf + nvfp4_sf_offset(row, (h * DH + c) / 16, D)) =
              static_cast<uint16_t>(sbs);
        }
      } else if constexpr (OUT == 1) {
        const float f = inv * args.f8_scale;
        uint8_t* dst = static_cast<uint8_t*>(args.out) + static_cast<int64_t>(row) * D + h * DH;
        uint32_t o[32];
        tmem_ld32(trow + kColO + c, o);
        if (row < kend && VLM_DCHECK(kend <= __ldg(args.cu + args.n_blocks))) {
          uint4* d4 = reinterpret_cast<uint4*>(dst + c);
#pragma unroll
          for (int jj = 0; jj < 2; ++jj) {
            uint32_t w[4];
#pragma unroll
            for (int k = 0; k < 4; ++k)
              w[k] = pack_e4m3x4(__uint_as_float(o[16 * jj + 4 * k]) * f, __uint_as_float(o[16 * jj + 4 * k + 1]) * f,
                                 __uint_as_float(o[16 * jj + 4 * k + 2]) * f, __uint_as_float(o[16 * jj + 4 * k + 3]) * f);
            d4[jj] = make_uint4(w[0], w[1], w[2], w[3]);
          }
        }
      } else {
        __nv_bfloat16* dst = static_cast<__nv_bfloat16*>(args.out) + static_cast<int64_t>(row) * D + h * DH;
        uint32_t o[32];
        tmem_ld32(trow + kColO + c, o);
        if (row < kend && VLM_DCHECK(kend <= __ldg(args.cu + args.n_blocks))) {
          uint4* d4 = reinterpret_cast<uint4*>(dst + c);
#pragma unroll
          for (int jj = 0; jj < 4; ++jj)
            d4[jj] = make_uint4(pack_bf16x2(__uint_as_float(o[8 * jj]) * inv, __uint_as_float(o[8 * jj + 1]) * inv),
                                pack_bf16x2(__uint_as_float(o[8 * jj + 2]) * inv, __uint_as_float(o[8 * jj + 3]) * inv),
                                pack_bf16x2(__uint_as_float(o[8 * jj + 4]) * inv, __uint_as_float(o[8 * jj + 5]) * inv),
                                pack_bf16x2(__uint_as_float(o[8 * jj + 6]) * inv, __uint_as_float(o[8 * jj + 7]) * inv));
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

}  // namespace

int launch_attention(const __nv_bfloat16* qkv, int64_t T, int heads, const int32_t* cu, const int32_t* qt,
                     int n_blocks, int total_qtiles, void* out, int32_t* status, cudaStream_t s, float f8_scale,
                     uint8_t* out_sf) {
  if (total_qtiles <= 0) return VLM_OK;
  if (heads <= 0 || heads > 65535) return VLM_ERR_UNSUPPORTED;
  CUtensorMap tm;
  const uint64_t row = 3ull * heads * DH;
  if (!make_tmap_2d_bf16(&tm, qkv, row, static_cast<uint64_t>(T), row * 2, DH, BQ)) return VLM_ERR_CUDA;
  static bool attr_done[64] = {};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 64 && !attr_done[dev]) {
    if (cudaFuncSetAttribute(attn_tc_kernel<0>, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes) !=
            cudaSuccess ||
        cudaFuncSetAttribute(attn_tc_kernel<1>, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes) !=
            cudaSuccess ||
        cudaFuncSetAttribute(attn_tc_kernel<2>, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes) !=
            cudaSuccess)
      return VLM_ERR_CUDA;
    attr_done[dev] = true;
  }
  if (out_sf != nullptr && !(f8_scale > 0.f)) return VLM_ERR_INVALID_ARG;
  AttnArgs args{cu, qt, n_blocks, heads, out, status, f8_scale, out_sf, 0};
  auto kern = out_sf != nullptr ? attn_tc_kernel<2> : f8_scale > 0.f ? attn_tc_kernel<1> : attn_tc_kernel<0>;
  launch_begin(KC_ATTN, s);
  cudaError_t e = cudaSuccess;
  if (sm_budget() >= num_sms()) {
    e = launch_pdl(kern, dim3(total_qtiles, heads), dim3(kThreads), kSmemBytes, s, tm, args);
  } else {
    // at most two CTAs per budgeted SM at a time: successive grids over the query
    // tiles, plain launches (a programmatic launch would let the next grid's CTAs
    // take SMs while they wait for this one)
    const int chunk = std::max(1, 2 * sm_budget() / heads);
    int launches = 0;
    for (int t0 = 0; t0 < total_qtiles && e == cudaSuccess; t0 += chunk) {
      args.tile_base = t0;
      kern<<<dim3(std::min(chunk, total_qtiles - t0), heads), dim3(kThreads), kSmemBytes, s>>>(tm, args);
      e = cudaGetLastError();
      ++launches;
    }
    note_extra_launches(launches - 1);
  }
  launch_end(KC_ATTN, s);
  return e == cudaSuccess ? VLM_OK : VLM_ERR_CUDA;
}

}  // namespace vlm
