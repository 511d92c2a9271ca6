// K2: the packed 4-bit x 4-bit GEMM of the rotated W4A4 linear layer, with the
// DiRotQ low-rank residual (K3) fused into its epilogue.
//
//   y[m, n] = s_a[m] * sum_g s_w[g, n] * sum_{k in g} A[m, k] B[n, k]  (+ c[m] . L[n])
//
// (OrbitQuant abstract: the rotation folded into the weights cancels inside
// the layer, leaving a plain low-bit GEMM on rotated codes; DiRotQ abstract:
// 4-bit GEMM plus a thin high-precision GEMM on the r PCA coefficients, and
// NVFP4 on Blackwell.)
//
// Two mainloops, one epilogue:
//  * FP8 path (INT4 or Lloyd-Max codes, 4-bit activations, 4- or 2-bit
//    weights): TMA brings the packed codes into shared memory; four expansion
//    warps turn every code into its exactly representable E4M3 byte through a
//    16-entry byte LUT (prmt) and write the 128-byte-swizzled K-major operand
//    tiles that tcgen05.mma.kind::f8f6f4 reads; one thread issues the MMAs into
//    a TMEM accumulator.  INT4 weights carry one scale per 128 rotated
//    coordinates, so every 128-wide K group is accumulated into its own TMEM
//    partial (double-buffered) and the epilogue folds s_w[g, n] * partial into
//    a TMEM running sum while the tensor core works on the next group.
//  * NVFP4 path: TMA brings packed E2M1 tiles (128B swizzle) and 1-D bulk copies
//    bring the UE4M3 block scales, already in the 128x4 tile layout K1 writes;
//    tcgen05.cp moves the scales into TMEM and
//    tcgen05.mma.kind::mxf4nvf4.block_scale.block16 applies them in hardware.
//  * K3: a rank-r BF16 UMMA (kind::f16) c . L^T into its own TMEM columns,
//    added after the per-token scale.
// Every mbarrier wait is bounded (see rq_ptx.cuh); a timeout is reported through
// the caller's status word and all warps leave together.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cstdint>
#include <cstring>

#include "rq_internal.h"
#include "rq_ptx.cuh"

namespace rq {

namespace {

constexpr int BM = 128;

struct __align__(64) TMaps {
  CUtensorMap a;   // packed activation codes
  CUtensorMap b;   // packed weight codes
  CUtensorMap c;   // low-rank coefficients (M x r BF16)
  CUtensorMap l;   // low-rank weights (N x r BF16)
};

struct __align__(16) GemmParams {
  int M, N, K;
  int a_fmt, w_fmt;
  const float* a_scale;
  const float* w_scale;     // INT4: [K/128][N]; else [N]
  const uint8_t* a_bscale;  // NVFP4 swizzled block scales
  const uint8_t* w_bscale;
  uint32_t a_lut[4];        // 16 e4m3 bytes, little-endian by code
  uint32_t w_lut[4];
  int has_lr;
  void* Y;
  int out_fp32;
  int32_t* status;
};

// ------------------------------------------------------------------ helpers
__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel) {
  uint32_t d;
  asm("prmt.b32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(sel));
  return d;
}

// Four 4-bit codes (bits 0-15 of x) -> four LUT bytes.
__device__ __forceinline__ uint32_t lut16x4(uint32_t x, const uint32_t (&L)[4]) {
  const uint32_t sel = x & 0x7777u;
  const uint32_t lo = prmt(L[0], L[1], sel);
  const uint32_t hi = prmt(L[2], L[3], sel);
  const uint32_t pick = ((x & 0x8888u) >> 1) | 0x3210u;
  return prmt(lo, hi, pick);
}

// Eight 2-bit codes (bits 0-15 of x) -> eight LUT bytes (lo word: codes 0-3).
__device__ __forceinline__ void lut4x8(uint32_t x, uint32_t L0, uint32_t& o0, uint32_t& o1) {
  uint32_t t = (x | (x << 8)) & 0x00FF00FFu;
  t = (t | (t << 4)) & 0x0F0F0F0Fu;
  t = (t | (t << 2)) & 0x33333333u;
  o0 = prmt(L0, 0u, t & 0xFFFFu);
  o1 = prmt(L0, 0u, t >> 16);
}

__device__ __forceinline__ void st_shared_v4(uint32_t addr, uint32_t a, uint32_t b, uint32_t c, uint32_t d) {
  asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(a), "r"(b), "r"(c), "r"(d)
               : "memory");
}
__device__ __forceinline__ uint4 ld_shared_v4(uint32_t addr) {
  uint4 v;
  asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "r"(addr)
               : "memory");
  return v;
}

__device__ __forceinline__ void tmem_st32(uint32_t taddr, const float (&v)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], "
      "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
      "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};" ::"r"(taddr),
      "f"(v[0]), "f"(v[1]), "f"(v[2]), "f"(v[3]), "f"(v[4]), "f"(v[5]), "f"(v[6]), "f"(v[7]), "f"(v[8]),
      "f"(v[9]), "f"(v[10]), "f"(v[11]), "f"(v[12]), "f"(v[13]), "f"(v[14]), "f"(v[15]), "f"(v[16]),
      "f"(v[17]), "f"(v[18]), "f"(v[19]), "f"(v[20]), "f"(v[21]), "f"(v[22]), "f"(v[23]), "f"(v[24]),
      "f"(v[25]), "f"(v[26]), "f"(v[27]), "f"(v[28]), "f"(v[29]), "f"(v[30]), "f"(v[31])
      : "memory");
}
__device__ __forceinline__ void tmem_st_wait() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

// Store 32 consecutive outputs of one row (FP32 or BF16), masked to n < N.
__device__ __forceinline__ void store_row32(void* Y, int out_fp32, int N, int m, int n0, const float (&v)[32]) {
  if (out_fp32) {
    float* dst = reinterpret_cast<float*>(Y) + (size_t)m * N + n0;
    if (n0 + 32 <= N) {
#pragma unroll
      for (int i = 0; i < 32; i += 4) *reinterpret_cast<float4*>(dst + i) = make_float4(v[i], v[i + 1], v[i + 2], v[i + 3]);
    } else {
      for (int i = 0; i < 32 && n0 + i < N; ++i) dst[i] = v[i];
    }
  } else {
    __nv_bfloat16* dst = reinterpret_cast<__nv_bfloat16*>(Y) + (size_t)m * N + n0;
    uint32_t w[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      __nv_bfloat162 h = __floats2bfloat162_rn(v[2 * i], v[2 * i + 1]);
      w[i] = *reinterpret_cast<uint32_t*>(&h);
    }
    if (n0 + 32 <= N) {
#pragma unroll
      for (int i = 0; i < 16; i += 4)
        *reinterpret_cast<uint4*>(dst + 2 * i) = make_uint4(w[i], w[i + 1], w[i + 2], w[i + 3]);
    } else {
      for (int i = 0; i < 32 && n0 + i < N; ++i) dst[i] = __float2bfloat16_rn(v[i]);
    }
  }
}

// Instruction descriptors (tcgen05): D format F32 at bits 4-5, A/B formats at
// bits 7-9 / 10-12, K-major A and B, N >> 3 at bits 17-22, M >> 4 at bits 24-28.
__host__ __device__ constexpr uint32_t idesc_f8(int n) {
  return (1u << 4) | (0u << 7) | (0u << 10) | ((uint32_t)(n >> 3) << 17) | ((uint32_t)(BM >> 4) << 24);
}
__host__ __device__ constexpr uint32_t idesc_bf16(int n) {
  return (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(n >> 3) << 17) | ((uint32_t)(BM >> 4) << 24);
}
// Block-scaled NVFP4: E2M1 (1) for A and B, UE4M3 scales (bit 23 = 0),
// scale-factor ids 0, K = 64 per instruction (bit 31 = 0).
__host__ __device__ constexpr uint32_t idesc_nvf4(int n) {
  return (1u << 7) | (1u << 10) | ((uint32_t)(n >> 3) << 17) | ((uint32_t)(BM >> 4) << 24);
}

// ====================================================================== FP8
// Shared-memory plan (per CTA), all operand buffers 1024-byte aligned:
//   packed A  [SP][128 x 64 B]   (TMA, 64B swizzle)
//   packed B  [SP][BN x WROW]    (TMA, 64B swizzle; 32B swizzle for 2-bit codes)
//   e4m3 A    [SE][128 x 128 B]  (128B swizzle, K-major UMMA operand)
//   e4m3 B    [SE][BN x 128 B]
//   c tile    [128 x 64 B], L tile [BN x 64 B] (64B swizzle)
//   barriers, TMEM base address, abort flag
template <int BN, int WBITS>
struct Fp8Plan {
  static constexpr int SP = 4, SE = 3;
  static constexpr int WROW = WBITS == 4 ? 64 : 32;  // packed weight bytes per row per 128-K tile
  static constexpr int PA = BM * 64, PB = BN * WROW, EA = BM * 128, EB = BN * 128;
  static constexpr int OFF_PA = 0;
  static constexpr int OFF_PB = OFF_PA + SP * PA;
  static constexpr int OFF_EA = OFF_PB + SP * PB;
  static constexpr int OFF_EB = OFF_EA + SE * EA;
  static constexpr int OFF_C = OFF_EB + SE * EB;
  static constexpr int OFF_L = OFF_C + BM * 64;
  static constexpr int OFF_BAR = OFF_L + BN * 64;
  static constexpr int NBAR = 2 * SP + 2 * SE + 4 + 2;
  static constexpr int BYTES = OFF_BAR + NBAR * 8 + 16 + 1024;  // + alignment slack
};

// TMEM columns: acc[0] at 0, acc[1] at BN, running sum at 2BN, low-rank at 3BN.
template <int BN, int WBITS>
__global__ void __launch_bounds__(384, 1) gemm_fp8_kernel(const __grid_constant__ TMaps tm, const __grid_constant__ GemmParams p) {
  using P = Fp8Plan<BN, WBITS>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
  const uint32_t sbase = smem_u32(smem);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + P::OFF_BAR);
  uint64_t* pfull = bars;                  // [SP] TMA -> expansion
  uint64_t* pempty = pfull + P::SP;        // [SP] expansion -> TMA
  uint64_t* efull = pempty + P::SP;        // [SE] expansion -> MMA
  uint64_t* eempty = efull + P::SE;        // [SE] MMA -> expansion
  uint64_t* accfull = eempty + P::SE;      // [2]  MMA -> epilogue
  uint64_t* accempty = accfull + 2;        // [2]  epilogue -> MMA
  uint64_t* lrfull = accempty + 2;         // low-rank tiles landed
  uint64_t* lrdone = lrfull + 1;           // low-rank MMA done
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + P::NBAR);
  volatile int32_t* abort_flag = reinterpret_cast<volatile int32_t*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n0 = blockIdx.x * BN, m0 = blockIdx.y * BM;
  const int nk = p.K / 128;                // 128-wide K tiles == INT4 groups
  const bool grouped = p.w_fmt == RQ_FMT_INT4;

  if (threadIdx.x == 0) {
    for (int i = 0; i < P::SP; ++i) { mbar_init(&pfull[i], 1); mbar_init(&pempty[i], 4); }
    for (int i = 0; i < P::SE; ++i) { mbar_init(&efull[i], 4); mbar_init(&eempty[i], 1); }
    for (int i = 0; i < 2; ++i) { mbar_init(&accfull[i], 1); mbar_init(&accempty[i], 4); }
    mbar_init(lrfull, 1);
    mbar_init(lrdone, 1);
    *abort_flag = 0;
    fence_mbar_init();
    prefetch_tmap(&tm.a);
    prefetch_tmap(&tm.b);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      if (p.has_lr) {
        mbar_expect_tx(lrfull, BM * 64 + BN * 64);
        tma_load_2d(smem + P::OFF_C, &tm.c, 0, m0, lrfull);
        tma_load_2d(smem + P::OFF_L, &tm.l, 0, n0, lrfull);
      }
      for (int kt = 0; kt < nk; ++kt) {
        const int s = kt % P::SP;
        if (kt >= P::SP && !mbar_wait(&pempty[s], ((kt / P::SP) - 1) & 1, p.status, ST_TIMEOUT_EMPTY, abort_flag)) break;
        mbar_expect_tx(&pfull[s], P::PA + P::PB);
        tma_load_2d(smem + P::OFF_PA + s * P::PA, &tm.a, kt * 64, m0, &pfull[s]);
        tma_load_2d(smem + P::OFF_PB + s * P::PB, &tm.b, kt * P::WROW, n0, &pfull[s]);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      if (p.has_lr) {
        if (mbar_wait(lrfull, 0, p.status, ST_TIMEOUT_FULL, abort_flag)) {
          tc_fence_after();
          const uint32_t ca = sbase + P::OFF_C, la = sbase + P::OFF_L;
#pragma unroll
          for (int kk = 0; kk < 2; ++kk)
            umma_bf16(tmem + 3 * BN, smem_desc(ca + kk * 32, 16, 512, 4), smem_desc(la + kk * 32, 16, 512, 4),
                      idesc_bf16(BN), kk > 0);
          tc_commit(lrdone);
        }
      }
      const uint32_t idesc = idesc_f8(BN);
      int g = 0;  // accumulator group index
      for (int kt = 0; kt < nk && !*abort_flag; ++kt) {
        const int s = kt % P::SE;
        const bool first_of_group = grouped || kt == 0;
        const int buf = grouped ? (g & 1) : 0;
        if (first_of_group && grouped && g >= 2) {
          if (!mbar_wait(&accempty[buf], ((g >> 1) - 1) & 1, p.status, ST_TIMEOUT_EPI, abort_flag)) break;
        }
        if (!mbar_wait(&efull[s], (kt / P::SE) & 1, p.status, ST_TIMEOUT_FULL, abort_flag)) break;
        tc_fence_after();
        const uint32_t a = sbase + P::OFF_EA + s * P::EA, b = sbase + P::OFF_EB + s * P::EB;
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
          umma_f8(tmem + buf * BN, smem_desc(a + kk * 32, 16, 1024, 2), smem_desc(b + kk * 32, 16, 1024, 2), idesc,
                  (first_of_group && kk == 0) ? 0u : 1u);
        tc_commit(&eempty[s]);
        if (grouped) {
          tc_commit(&accfull[buf]);
          ++g;
        }
      }
      if (!grouped) tc_commit(&accfull[0]);
    }
  } else if (warp >= 4 && warp < 8) {
    // ------------------------------------------------------------ epilogue
    const int q = warp - 4;                  // TMEM lane quadrant
    const int row = m0 + q * 32 + lane;
    const uint32_t lane_off = (uint32_t)(q * 32) << 16;
    const float sa = row < p.M ? __ldg(p.a_scale + row) : 0.f;
    const int G = grouped ? nk : 1;
    bool ok = true;
    for (int g = 0; g < G && ok; ++g) {
      const int buf = g & 1;
      ok = mbar_wait(&accfull[buf], (g >> 1) & 1, p.status, ST_TIMEOUT_MMA, abort_flag);
      if (!ok) break;
      tc_fence_after();
      const bool last = g == G - 1;
      if (last && p.has_lr) {
        ok = mbar_wait(lrdone, 0, p.status, ST_TIMEOUT_MMA, abort_flag);
        if (!ok) break;
        tc_fence_after();
      }
#pragma unroll 1
      for (int ch = 0; ch < BN / 32; ++ch) {
        const int nc = n0 + ch * 32;
        uint32_t acc[32];
        tmem_ld32(tmem + lane_off + buf * BN + ch * 32, acc);
        float run[32];
        if (grouped && g > 0) {
          uint32_t r[32];
          tmem_ld32(tmem + lane_off + 2 * BN + ch * 32, r);
          tmem_ld_wait();
#pragma unroll
          for (int i = 0; i < 32; ++i) run[i] = __uint_as_float(r[i]);
        } else {
          tmem_ld_wait();
#pragma unroll
          for (int i = 0; i < 32; ++i) run[i] = 0.f;
        }
        // weight scales for these 32 columns (broadcast loads)
        const float* sw = grouped ? p.w_scale + (size_t)g * p.N + nc : p.w_scale + nc;
        float swv[32];
        if (nc + 32 <= p.N) {
#pragma unroll
          for (int i = 0; i < 32; i += 4) {
            const float4 t = __ldg(reinterpret_cast<const float4*>(sw + i));
            swv[i] = t.x; swv[i + 1] = t.y; swv[i + 2] = t.z; swv[i + 3] = t.w;
          }
        } else {
#pragma unroll
          for (int i = 0; i < 32; ++i) swv[i] = nc + i < p.N ? __ldg(sw + i) : 0.f;
        }
#pragma unroll
        for (int i = 0; i < 32; ++i) run[i] = fmaf(swv[i], __uint_as_float(acc[i]), run[i]);
        if (!last) {
          tmem_st32(tmem + lane_off + 2 * BN + ch * 32, run);
        } else {
          if (p.has_lr) {
            uint32_t lr[32];
            tmem_ld32(tmem + lane_off + 3 * BN + ch * 32, lr);
            tmem_ld_wait();
#pragma unroll
            for (int i = 0; i < 32; ++i) run[i] = fmaf(run[i], sa, __uint_as_float(lr[i]));
          } else {
#pragma unroll
            for (int i = 0; i < 32; ++i) run[i] *= sa;
          }
          if (row < p.M) store_row32(p.Y, p.out_fp32, p.N, row, nc, run);
        }
      }
      if (!last) tmem_st_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&accempty[buf]);
    }
  } else if (warp >= 8) {
    // ------------------------------------------------------------ code -> e4m3 expansion
    const int t = threadIdx.x - 256;        // 0..127
    uint32_t LA[4], LW[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) { LA[i] = p.a_lut[i]; LW[i] = p.w_lut[i]; }
    for (int kt = 0; kt < nk; ++kt) {
      const int sp = kt % P::SP, se = kt % P::SE;
      if (!mbar_wait(&pfull[sp], (kt / P::SP) & 1, p.status, ST_TIMEOUT_FULL, abort_flag)) break;
      if (kt >= P::SE && !mbar_wait(&eempty[se], ((kt / P::SE) - 1) & 1, p.status, ST_TIMEOUT_EMPTY, abort_flag)) break;
      const uint32_t pa = sbase + P::OFF_PA + sp * P::PA, pb = sbase + P::OFF_PB + sp * P::PB;
      const uint32_t ea = sbase + P::OFF_EA + se * P::EA, eb = sbase + P::OFF_EB + se * P::EB;
      // A: 128 rows x 4 segments of 16 packed bytes (32 codes each)
#pragma unroll
      for (int it = 0; it < 4; ++it) {
        const int idx = it * 128 + t;
        const int r = (idx >> 5) * 8 + (idx & 7), seg = (idx >> 3) & 3;
        const uint4 v = ld_shared_v4(pa + r * 64 + ((seg ^ ((r >> 1) & 3)) << 4));
        const uint32_t w[4] = {v.x, v.y, v.z, v.w};
        uint32_t o[8];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          o[2 * j] = lut16x4(w[j] & 0xFFFFu, LA);
          o[2 * j + 1] = lut16x4(w[j] >> 16, LA);
        }
        const uint32_t rowb = ea + r * 128;
        st_shared_v4(rowb + (((2 * seg) ^ (r & 7)) << 4), o[0], o[1], o[2], o[3]);
        st_shared_v4(rowb + (((2 * seg + 1) ^ (r & 7)) << 4), o[4], o[5], o[6], o[7]);
      }
      if constexpr (WBITS == 4) {
#pragma unroll
        for (int it = 0; it < BN / 32; ++it) {
          const int idx = it * 128 + t;
          const int r = (idx >> 5) * 8 + (idx & 7), seg = (idx >> 3) & 3;
          const uint4 v = ld_shared_v4(pb + r * 64 + ((seg ^ ((r >> 1) & 3)) << 4));
          const uint32_t w[4] = {v.x, v.y, v.z, v.w};
          uint32_t o[8];
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            o[2 * j] = lut16x4(w[j] & 0xFFFFu, LW);
            o[2 * j + 1] = lut16x4(w[j] >> 16, LW);
          }
          const uint32_t rowb = eb + r * 128;
          st_shared_v4(rowb + (((2 * seg) ^ (r & 7)) << 4), o[0], o[1], o[2], o[3]);
          st_shared_v4(rowb + (((2 * seg + 1) ^ (r & 7)) << 4), o[4], o[5], o[6], o[7]);
        }
      } else {
        // 2-bit weights: 32 packed bytes per row = 2 segments of 64 codes
#pragma unroll
        for (int it = 0; it < BN / 64; ++it) {
          const int idx = it * 128 + t;
          const int r = (idx >> 4) * 8 + (idx & 7), seg = (idx >> 3) & 1;
          const uint4 v = ld_shared_v4(pb + r * 32 + ((seg ^ ((r >> 2) & 1)) << 4));
          const uint32_t w[4] = {v.x, v.y, v.z, v.w};
          uint32_t o[16];
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            lut4x8(w[j] & 0xFFFFu, LW[0], o[4 * j], o[4 * j + 1]);
            lut4x8(w[j] >> 16, LW[0], o[4 * j + 2], o[4 * j + 3]);
          }
          const uint32_t rowb = eb + r * 128;
#pragma unroll
          for (int c = 0; c < 4; ++c)
            st_shared_v4(rowb + (((4 * seg + c) ^ (r & 7)) << 4), o[4 * c], o[4 * c + 1], o[4 * c + 2], o[4 * c + 3]);
        }
      }
      fence_proxy_async_smem();  // make the generic-proxy writes visible to the tensor core
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(&efull[se]);
        mbar_arrive(&pempty[sp]);
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// ===================================================================== NVFP4
// Per stage: packed A 128 x 128 B, packed B BN x 128 B (256 E2M1 per row, 128B
// swizzle), scale tiles 128 x 16 B and BN x 16 B (4 chunks of 32 x 16 B per
// 128 rows, the layout tcgen05.cp 32x128b.warpx4 reads).
template <int BN>
struct Nvf4Plan {
  static constexpr int S = BN == 256 ? 4 : 5;
  static constexpr int PA = BM * 128, PB = BN * 128, SA = BM * 16, SB = BN * 16;
  static constexpr int STAGE = PA + PB + SA + SB;
  static constexpr bool LR = BN == 128;   // the low-rank branch runs with BN = 128 only
  static constexpr int OFF_C = S * STAGE;
  static constexpr int OFF_L = OFF_C + (LR ? BM * 64 : 0);
  static constexpr int OFF_BAR = OFF_L + (LR ? BN * 64 : 0);
  static constexpr int NBAR = 2 * S + 2 + 2;
  static constexpr int BYTES = OFF_BAR + NBAR * 8 + 16 + 1024;
};

// TMEM columns: acc at 0 (BN), low-rank at 128 (only when BN == 128), SFA at
// 256..271 (4 MMAs x 4 columns), SFB at 272.. (4 MMAs x BN/32 columns).
template <int BN>
__global__ void __launch_bounds__(256, 1) gemm_nvf4_kernel(const __grid_constant__ TMaps tm, const __grid_constant__ GemmParams p) {
  using P = Nvf4Plan<BN>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
  const uint32_t sbase = smem_u32(smem);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + P::OFF_BAR);
  uint64_t* full = bars;
  uint64_t* empty = full + P::S;
  uint64_t* accfull = empty + P::S;
  uint64_t* lrfull = accfull + 1;
  uint64_t* lrdone = lrfull + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + P::NBAR);
  volatile int32_t* abort_flag = reinterpret_cast<volatile int32_t*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n0 = blockIdx.x * BN, m0 = blockIdx.y * BM;
  const int nk = p.K / 256;
  const int ktiles64 = p.K / 64;          // scale tiles per 128 rows

  if (threadIdx.x == 0) {
    for (int i = 0; i < P::S; ++i) { mbar_init(&full[i], 1); mbar_init(&empty[i], 1); }
    mbar_init(accfull, 1);
    mbar_init(lrfull, 1);
    mbar_init(lrdone, 1);
    *abort_flag = 0;
    fence_mbar_init();
    prefetch_tmap(&tm.a);
    prefetch_tmap(&tm.b);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t t_sfa = tmem + 256, t_sfb = tmem + 272;

  if (warp == 0) {
    if (lane == 0) {
      if (P::LR && p.has_lr) {
        mbar_expect_tx(lrfull, BM * 64 + BN * 64);
        tma_load_2d(smem + P::OFF_C, &tm.c, 0, m0, lrfull);
        tma_load_2d(smem + P::OFF_L, &tm.l, 0, n0, lrfull);
      }
      const uint8_t* sfa_src = p.a_bscale + (size_t)(m0 / 128) * ktiles64 * 512;
      // weight scale tiles that exist (the last tile column may cover only 128 rows)
      const int nb_valid = min(BN / 128, (p.N + 127) / 128 - n0 / 128);
      for (int kt = 0; kt < nk; ++kt) {
        const int s = kt % P::S;
        if (kt >= P::S && !mbar_wait(&empty[s], ((kt / P::S) - 1) & 1, p.status, ST_TIMEOUT_EMPTY, abort_flag)) break;
        uint8_t* st = smem + s * P::STAGE;
        mbar_expect_tx(&full[s], P::PA + P::PB + P::SA + nb_valid * 2048);
        tma_load_2d(st, &tm.a, kt * 128, m0, &full[s]);
        tma_load_2d(st + P::PA, &tm.b, kt * 128, n0, &full[s]);
        // 4 scale chunks (k tiles of 64) x 512 B, contiguous in the K1 layout
        bulk_g2s(st + P::PA + P::PB, sfa_src + (size_t)kt * 4 * 512, 2048, &full[s]);
        for (int nb = 0; nb < nb_valid; ++nb)
          bulk_g2s(st + P::PA + P::PB + P::SA + nb * 2048,
                   p.w_bscale + ((size_t)(n0 / 128 + nb) * ktiles64 + (size_t)kt * 4) * 512, 2048, &full[s]);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      if (p.has_lr) {
        if (mbar_wait(lrfull, 0, p.status, ST_TIMEOUT_FULL, abort_flag)) {
          tc_fence_after();
          const uint32_t ca = sbase + P::OFF_C, la = sbase + P::OFF_L;
#pragma unroll
          for (int kk = 0; kk < 2; ++kk)
            umma_bf16(tmem + BN, smem_desc(ca + kk * 32, 16, 512, 4), smem_desc(la + kk * 32, 16, 512, 4),
                      idesc_bf16(BN), kk > 0);
          tc_commit(lrdone);
        }
      }
      const uint32_t idesc = idesc_nvf4(BN);
      for (int kt = 0; kt < nk; ++kt) {
        const int s = kt % P::S;
        if (!mbar_wait(&full[s], (kt / P::S) & 1, p.status, ST_TIMEOUT_FULL, abort_flag)) break;
        tc_fence_after();
        const uint32_t st = sbase + s * P::STAGE;
        const uint32_t sfa = st + P::PA + P::PB, sfb = sfa + P::SA;
        // scale factors -> TMEM: per MMA (K = 64) one 512 B chunk per 128 rows
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {
          tc_cp_32x128b_warpx4(t_sfa + kk * 4, smem_desc(sfa + kk * 512, 16, 128, 0));
#pragma unroll
          for (int nb = 0; nb < BN / 128; ++nb)
            tc_cp_32x128b_warpx4(t_sfb + kk * (BN / 32) + nb * 4, smem_desc(sfb + nb * 2048 + kk * 512, 16, 128, 0));
        }
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
          umma_nvf4(tmem, smem_desc(st + kk * 32, 16, 1024, 2), smem_desc(st + P::PA + kk * 32, 16, 1024, 2), idesc,
                    t_sfa + kk * 4, t_sfb + kk * (BN / 32), (kt > 0 || kk > 0) ? 1u : 0u);
        tc_commit(&empty[s]);
      }
      tc_commit(accfull);
    }
  } else if (warp >= 4) {
    const int q = warp - 4;
    const int row = m0 + q * 32 + lane;
    const uint32_t lane_off = (uint32_t)(q * 32) << 16;
    const float sa = row < p.M ? __ldg(p.a_scale + row) : 0.f;
    bool ok = mbar_wait(accfull, 0, p.status, ST_TIMEOUT_MMA, abort_flag);
    if (ok && p.has_lr) ok = mbar_wait(lrdone, 0, p.status, ST_TIMEOUT_MMA, abort_flag);
    if (ok) {
      tc_fence_after();
#pragma unroll 1
      for (int ch = 0; ch < BN / 32; ++ch) {
        const int nc = n0 + ch * 32;
        uint32_t acc[32];
        tmem_ld32(tmem + lane_off + ch * 32, acc);
        uint32_t lr[32];
        if (p.has_lr) tmem_ld32(tmem + lane_off + BN + ch * 32, lr);
        tmem_ld_wait();
        float v[32];
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          const float swv = nc + i < p.N ? __ldg(p.w_scale + nc + i) : 0.f;
          v[i] = __uint_as_float(acc[i]) * (sa * swv);
          if (p.has_lr) v[i] += __uint_as_float(lr[i]);
        }
        if (row < p.M) store_row32(p.Y, p.out_fp32, p.N, row, nc, v);
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// ================================================================== host side
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn get_encode() {
  static EncodeTiledFn fn = nullptr;
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  }
  return fn;
}

bool make_map_2d(CUtensorMap* m, CUtensorMapDataType dt, const void* base, uint64_t inner, uint64_t outer,
                 uint64_t row_bytes, uint32_t box_inner, uint32_t box_outer, CUtensorMapSwizzle swz) {
  EncodeTiledFn enc = get_encode();
  if (!enc) return false;
  cuuint64_t dims[2] = {inner, outer};
  cuuint64_t strides[1] = {row_bytes};
  cuuint32_t box[2] = {box_inner, box_outer};
  cuuint32_t es[2] = {1, 1};
  return enc(m, dt, 2, const_cast<void*>(base), dims, strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE, swz,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <class Kern>
cudaError_t launch(Kern k, int smem, dim3 grid, int threads, const TMaps& tm, const GemmParams& gp, cudaStream_t st) {
  cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  k<<<grid, threads, smem, st>>>(tm, gp);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_gemm(const GemmLaunch& a, cudaStream_t st, const char** why) {
  TMaps tm;
  memset(&tm, 0, sizeof(tm));
  GemmParams gp{};
  gp.M = a.M; gp.N = a.N; gp.K = a.K;
  gp.a_fmt = a.a_fmt; gp.w_fmt = a.w_fmt;
  gp.a_scale = a.a_scale; gp.w_scale = a.w_scale;
  gp.a_bscale = a.a_bscale; gp.w_bscale = a.w_bscale;
  memcpy(gp.a_lut, a.a_lut, 16);
  memcpy(gp.w_lut, a.w_lut, 16);
  gp.has_lr = a.c != nullptr;
  gp.Y = a.Y; gp.out_fp32 = a.out_fp32; gp.status = a.status;

  const bool nvf4 = a.a_fmt == RQ_FMT_NVFP4;
  const int BN = (nvf4 && !gp.has_lr) ? 256 : 128;
  bool ok = true;
  if (gp.has_lr) {
    ok &= make_map_2d(&tm.c, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, a.c, a.r, a.M, (uint64_t)a.r * 2, 32, BM,
                      CU_TENSOR_MAP_SWIZZLE_64B);
    ok &= make_map_2d(&tm.l, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, a.L, a.r, a.N, (uint64_t)a.r * 2, 32, BN,
                      CU_TENSOR_MAP_SWIZZLE_64B);
  }
  dim3 grid((a.N + BN - 1) / BN, (a.M + BM - 1) / BM);
  if (nvf4) {
    ok &= make_map_2d(&tm.a, CU_TENSOR_MAP_DATA_TYPE_UINT8, a.a_codes, a.K / 2, a.M, a.K / 2, 128, BM,
                      CU_TENSOR_MAP_SWIZZLE_128B);
    ok &= make_map_2d(&tm.b, CU_TENSOR_MAP_DATA_TYPE_UINT8, a.w_codes, a.K / 2, a.N, a.K / 2, 128, BN,
                      CU_TENSOR_MAP_SWIZZLE_128B);
    if (!ok) { *why = "cuTensorMapEncodeTiled failed"; return cudaErrorInvalidValue; }
    if (BN == 256) return launch(gemm_nvf4_kernel<256>, Nvf4Plan<256>::BYTES, grid, 256, tm, gp, st);
    return launch(gemm_nvf4_kernel<128>, Nvf4Plan<128>::BYTES, grid, 256, tm, gp, st);
  }
  const bool w2 = a.w_fmt == RQ_FMT_LM4;
  ok &= make_map_2d(&tm.a, CU_TENSOR_MAP_DATA_TYPE_UINT8, a.a_codes, a.K / 2, a.M, a.K / 2, 64, BM,
                    CU_TENSOR_MAP_SWIZZLE_64B);
  if (w2)
    ok &= make_map_2d(&tm.b, CU_TENSOR_MAP_DATA_TYPE_UINT8, a.w_codes, a.K / 4, a.N, a.K / 4, 32, BN,
                      CU_TENSOR_MAP_SWIZZLE_32B);
  else
    ok &= make_map_2d(&tm.b, CU_TENSOR_MAP_DATA_TYPE_UINT8, a.w_codes, a.K / 2, a.N, a.K / 2, 64, BN,
                      CU_TENSOR_MAP_SWIZZLE_64B);
  if (!ok) { *why = "cuTensorMapEncodeTiled failed"; return cudaErrorInvalidValue; }
  if (w2) return launch(gemm_fp8_kernel<128, 2>, Fp8Plan<128, 2>::BYTES, grid, 384, tm, gp, st);
  return launch(gemm_fp8_kernel<128, 4>, Fp8Plan<128, 4>::BYTES, grid, 384, tm, gp, st);
}

}  // namespace rq
