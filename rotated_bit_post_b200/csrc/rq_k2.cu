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
//  * Codebook path (Lloyd-Max codes, 4-bit activations, 4- or 2-bit weights):
//    TMA brings the packed codes into shared memory; expansion warps turn every
//    code into its exactly representable E4M3 byte through a 16-entry byte LUT
//    (prmt) and write the 128-byte-swizzled K-major operand tiles that
//    tcgen05.mma.kind::f8f6f4 reads; one thread issues the MMAs into TMEM.
//    The 256-wide tiles run on CTA pairs (cta_group::2, M = 256): each CTA of a
//    cluster of two loads and expands its own 128 token rows and half of the
//    tile's weight rows, and the even CTA issues the pair's MMAs.
//  * INT4 path: a two's-complement nibble v placed in the high half of a byte
//    is the int8 value 16 v, so expansion is two masks and a shift per eight
//    codes (even and odd codes land in separate words; A and B use the same
//    order, which a dot product over k does not see) and
//    tcgen05.mma.kind::i8 accumulates 256 * sum(qa qw) exactly in S32.  INT4
//    weights carry one scale per 128 rotated coordinates, so every 128-wide K
//    group is accumulated into its own TMEM partial (three buffers) and the
//    epilogue folds (s_w[g, n] / 256) * partial into running sums held in
//    registers while the tensor core works on the next groups.
//  * NVFP4 path: TMA brings packed E2M1 tiles (128B swizzle) and 1-D bulk copies
//    bring the UE4M3 block scales, already in the 128x4 tile layout K1 writes;
//    tcgen05.cp moves the scales into TMEM and
//    tcgen05.mma.kind::mxf4nvf4.block_scale.block16 applies them in hardware.
//  * K3: a rank-r BF16 UMMA (kind::f16) c . L^T into its own TMEM columns,
//    added after the per-token scale.
// Every mbarrier wait is bounded (see rq_ptx.cuh); a timeout is reported through
// the caller's status word and all warps leave together.
#include <mutex>
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cstdint>
#include <cstring>
#include <type_traits>

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
  CUtensorMap y;   // BF16 output, 32 x 32 boxes, 64-byte swizzle (TMA-store epilogue)
};

struct __align__(16) GemmParams {
  int M, N, K;
  int nk128;                // 128-wide K tiles, ceil(K / 128)
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
  int tma_store;           // BF16 output written through shared memory + TMA stores
  int32_t* status;
  uint64_t wait_ns;        // limit of every bounded wait
  uint32_t inject_tx;      // test hook: extra expect-tx bytes on the first operand stage
  const float* a_zp;       // asymmetric INT4 activations: per-token zero point, or null
  const float* w_zsum;     // per weight row: sum_g s_w[g, n] * (sum of the group's codes)
};

// ------------------------------------------------------------------ helpers
__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel) {
  uint32_t d;
  asm("prmt.b32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(sel));
  return d;
}


// Eight 16-level codes in their stored sign-magnitude form (bits 0-2: distance
// from the centre, bit 3: lower half) -> eight e4m3 bytes in code order.  The
// magnitude comes from the 8-entry table of the upper half's centroids (T0, T1);
// the sign from bit 3, which a sign-replicating permute of the code word (and
// of the word shifted by 4 for the even nibbles) moves to each byte's sign bit.
__device__ __forceinline__ void lut_sm8(uint32_t w, uint32_t T0, uint32_t T1, uint32_t& o0, uint32_t& o1) {
  const uint32_t sel = w & 0x77777777u, w4 = w << 4;
  o0 = prmt(T0, T1, sel) | (prmt(w4, w, 0xD9C8u) & 0x80808080u);
  o1 = prmt(T0, T1, sel >> 16) | (prmt(w4, w, 0xFBEAu) & 0x80808080u);
}

// Sixteen 2-bit codes (one 32-bit word, nibble i holding codes i and i+8 in
// bits 0-1 and 2-3) -> sixteen LUT bytes in code order: the two crumbs of every
// nibble are already prmt selectors.
__device__ __forceinline__ void lut4x16(uint32_t w, uint32_t L0, uint32_t (&o)[4]) {
  const uint32_t lo = w & 0x33333333u, hi = (w >> 2) & 0x33333333u;
  o[0] = prmt(L0, 0u, lo);
  o[1] = prmt(L0, 0u, lo >> 16);
  o[2] = prmt(L0, 0u, hi);
  o[3] = prmt(L0, 0u, hi >> 16);
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

// 32 lanes x 32 bit, 16 consecutive columns -> 16 registers per thread.
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
}
// run += w * (as_float(x + 0x4B400000) - 1.5 * 2^23) on two lanes of packed
// FP32 arithmetic.  For |x| < 2^22 the integer add lands x in the mantissa of
// a float whose unit in the last place is 1, so the subtraction recovers x
// exactly: an exact S32 -> F32 conversion on the full-rate pipes.
__device__ __forceinline__ void fma_s32x2(float& r0, float& r1, float w0, float w1, uint32_t x0, uint32_t x1) {
  asm("{\n\t.reg .b64 f, m, w, r;\n\t"
      "mov.b64 f, {%2, %3};\n\t"
      "mov.b64 m, {%6, %6};\n\t"
      "mov.b64 w, {%4, %5};\n\t"
      "mov.b64 r, {%0, %1};\n\t"
      "sub.rn.f32x2 f, f, m;\n\t"
      "fma.rn.f32x2 r, w, f, r;\n\t"
      "mov.b64 {%0, %1}, r;\n\t}"
      : "+f"(r0), "+f"(r1)
      : "r"(x0 + 0x4B400000u), "r"(x1 + 0x4B400000u), "f"(w0), "f"(w1), "f"(12582912.0f));
}

// Store 32 consecutive outputs of one row (FP32 or BF16), masked to n < N;
// 16-byte stores where the row and the chunk are whole and aligned (N a
// multiple of 4 FP32 or 8 BF16 values), element stores otherwise.
__device__ __forceinline__ void store_row32(void* Y, int out_fp32, int N, int m, int n0, const float (&v)[32]) {
  if (out_fp32) {
    float* dst = reinterpret_cast<float*>(Y) + (size_t)m * N + n0;
    if (n0 + 32 <= N && (N & 3) == 0) {
#pragma unroll
      for (int i = 0; i < 32; i += 4) *reinterpret_cast<float4*>(dst + i) = make_float4(v[i], v[i + 1], v[i + 2], v[i + 3]);
    } else {
#pragma unroll
      for (int i = 0; i < 32; ++i)   // unrolled with predicates: v stays in registers
        if (n0 + i < N) dst[i] = v[i];
    }
  } else {
    __nv_bfloat16* dst = reinterpret_cast<__nv_bfloat16*>(Y) + (size_t)m * N + n0;
    uint32_t w[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      __nv_bfloat162 h = __floats2bfloat162_rn(v[2 * i], v[2 * i + 1]);
      w[i] = *reinterpret_cast<uint32_t*>(&h);
    }
    if (n0 + 32 <= N && (N & 7) == 0) {
#pragma unroll
      for (int i = 0; i < 16; i += 4)
        *reinterpret_cast<uint4*>(dst + 2 * i) = make_uint4(w[i], w[i + 1], w[i + 2], w[i + 3]);
    } else {
#pragma unroll
      for (int i = 0; i < 32; ++i)
        if (n0 + i < N) dst[i] = __float2bfloat16_rn(v[i]);
    }
  }
}

// Instruction descriptors (tcgen05): D format F32 at bits 4-5, A/B formats at
// bits 7-9 / 10-12, K-major A and B, N >> 3 at bits 17-22, M >> 4 at bits 24-28.
__host__ __device__ constexpr uint32_t idesc_f8(int n) {
  return (1u << 4) | (0u << 7) | (0u << 10) | ((uint32_t)(n >> 3) << 17) | ((uint32_t)(BM >> 4) << 24);
}
// Signed 8-bit A and B (format 1), S32 accumulator (format 2).
__host__ __device__ constexpr uint32_t idesc_i8(int n) {
  return (2u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(n >> 3) << 17) | ((uint32_t)(BM >> 4) << 24);
}
__host__ __device__ constexpr uint32_t idesc_bf16(int n) {
  return (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(n >> 3) << 17) | ((uint32_t)(BM >> 4) << 24);
}
// Block-scaled NVFP4: E2M1 (1) for A and B, UE4M3 scales (bit 23 = 0),
// scale-factor ids 0, K = 64 per instruction (bit 31 = 0).
__host__ __device__ constexpr uint32_t idesc_nvf4(int n) {
  return (1u << 7) | (1u << 10) | ((uint32_t)(n >> 3) << 17) | ((uint32_t)(BM >> 4) << 24);
}

// ===================================================================== shared
// Named barrier among the epilogue warps.
template <int NT>
__device__ __forceinline__ void epi_bar_n() { asm volatile("bar.sync 1, %0;" ::"n"(NT) : "memory"); }

__device__ __forceinline__ void load_scales_smem(float* slot, const float* src, int n0, int N, int BNv, int tid,
                                                 int nthreads = 128) {
  for (int i = tid; i < BNv; i += nthreads) slot[i] = n0 + i < N ? __ldg(src + n0 + i) : 0.f;
}

// Epilogue of one 32-column chunk for a finished (non-grouped) accumulator:
// y = acc * (s_a[m] * s_w[n]) (+ low-rank), stored to Y.
// With a staging area (two 2 KB buffers per warp, smem address stg) and BF16
// output, the warp's 32 x 32 block goes to shared memory in the 64-byte
// swizzled layout of the output tensor map and out with one TMA store; the
// buffer is rewritten only after the store two chunks back has read it.
__device__ __forceinline__ void epi_chunk_final(const GemmParams& p, uint32_t tacc, uint32_t tlr, bool lr,
                                                const float* sw, float sa, int row, int nc,
                                                const CUtensorMap* ymap = nullptr, uint32_t stg = 0,
                                                uint32_t* sc = nullptr, int row0 = 0) {
  uint32_t acc[32];
  tmem_ld32(tacc, acc);
  uint32_t l[32];
  if (lr) tmem_ld32(tlr, l);
  // s_a * s_w for the 32 columns, formed before the wait (which orders every
  // memory access around it) so that the scale reads overlap it
  float s[32];
#pragma unroll
  for (int i = 0; i < 32; i += 4) {
    const float4 w4 = *reinterpret_cast<const float4*>(sw + i);
    s[i] = sa * w4.x;
    s[i + 1] = sa * w4.y;
    s[i + 2] = sa * w4.z;
    s[i + 3] = sa * w4.w;
  }
  tmem_ld_wait();
  float v[32];
#pragma unroll
  for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(acc[i]) * s[i];
  if (lr) {
#pragma unroll
    for (int i = 0; i < 32; ++i) v[i] += __uint_as_float(l[i]);
  }
  if (stg == 0 || !p.tma_store) {
    if (row < p.M) store_row32(p.Y, p.out_fp32, p.N, row, nc, v);
    return;
  }
  const int lane = threadIdx.x & 31;
  const uint32_t buf = stg + (*sc & 1u) * 2048u;
  if (*sc >= 2) {
    if (lane == 0) bulk_wait_group_read<1>();
    __syncwarp();
  }
  uint32_t w[16];
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    __nv_bfloat162 h = __floats2bfloat162_rn(v[2 * i], v[2 * i + 1]);
    w[i] = *reinterpret_cast<uint32_t*>(&h);
  }
#pragma unroll
  for (int c = 0; c < 4; ++c)
    st_shared_v4(buf + lane * 64 + ((c ^ ((lane >> 1) & 3)) << 4), w[4 * c], w[4 * c + 1], w[4 * c + 2], w[4 * c + 3]);
  fence_proxy_async_smem();
  __syncwarp();
  if (lane == 0) {
    tma_store_2d(ymap, buf, nc, row0);   // rows >= M and columns >= N are clipped by the map
    bulk_commit_group();
  }
  ++*sc;
}

// (x0, x1) * (y0, y1) on one packed FP32 pair
__device__ __forceinline__ void mul2_f32(float& x0, float& x1, float y0, float y1) {
  asm("{\n\t.reg .b64 a, b;\n\tmov.b64 a, {%0, %1};\n\tmov.b64 b, {%2, %3};\n\t"
      "mul.rn.f32x2 a, a, b;\n\tmov.b64 {%0, %1}, a;\n\t}"
      : "+f"(x0), "+f"(x1)
      : "f"(y0), "f"(y1));
}

// tcgen05.wait::ld that also names the destination registers of the loads it
// waits for, so that no use of them can be scheduled before it.
__device__ __forceinline__ void tmem_ld_wait_regs16(uint32_t (&r)[16]) {
  asm volatile("tcgen05.wait::ld.sync.aligned;"
               : "+r"(r[0]), "+r"(r[1]), "+r"(r[2]), "+r"(r[3]), "+r"(r[4]), "+r"(r[5]), "+r"(r[6]), "+r"(r[7]),
                 "+r"(r[8]), "+r"(r[9]), "+r"(r[10]), "+r"(r[11]), "+r"(r[12]), "+r"(r[13]), "+r"(r[14]),
                 "+r"(r[15])
               :
               : "memory");
}

// y for four consecutive columns: acc * (s_a * s_w), on packed FP32 pairs
__device__ __forceinline__ void scale4w(const uint32_t* a, float4 w4, float sa, float (&y)[4]) {
  float s0 = sa, s1 = sa, s2 = sa, s3 = sa;
  mul2_f32(s0, s1, w4.x, w4.y);
  mul2_f32(s2, s3, w4.z, w4.w);
  y[0] = __uint_as_float(a[0]);
  y[1] = __uint_as_float(a[1]);
  y[2] = __uint_as_float(a[2]);
  y[3] = __uint_as_float(a[3]);
  mul2_f32(y[0], y[1], s0, s1);
  mul2_f32(y[2], y[3], s2, s3);
}
__device__ __forceinline__ void scale4(const uint32_t* a, const float* sw, float sa, float (&y)[4]) {
  scale4w(a, *reinterpret_cast<const float4*>(sw), sa, y);
}

// Epilogue of the 256 x 512 pair tiles: this warp drains 16 * NCH accumulator
// columns of its 32 token rows.  BF16 output: 16 columns at a time, the TMEM
// load of the next 16 in flight while these are scaled and written to one of
// this warp's two 2 KB staging buffers; every 32 columns go out as one TMA
// store.  FP32 output (used for verification): 32 columns at a time, stored
// straight to global memory, the same FP32 values.
template <int NCH>
__device__ __forceinline__ void epi_cols_wide(const GemmParams& p, const CUtensorMap* ymap, uint32_t tacc,
                                              const float* sw, float sa, int row, int n0, int row0, uint32_t stg,
                                              uint32_t& stc) {
  const int lane = threadIdx.x & 31;
  if (!p.tma_store) {
#pragma unroll 1
    for (int ch = 0; ch < NCH / 2; ++ch) {
      uint32_t a[32];
      tmem_ld32(tacc + ch * 32, a);
      tmem_ld_wait();
      float v[32];
#pragma unroll
      for (int i = 0; i < 32; i += 4) {
        float y[4];
        scale4(a + i, sw + ch * 32 + i, sa, y);
        v[i] = y[0]; v[i + 1] = y[1]; v[i + 2] = y[2]; v[i + 3] = y[3];
      }
      if (row < p.M) store_row32(p.Y, p.out_fp32, p.N, row, n0 + ch * 32, v);
    }
    return;
  }
  uint32_t acc[2][16];
  tmem_ld16(tacc, acc[0]);
#pragma unroll
  for (int hc = 0; hc < NCH; ++hc) {
    // this chunk's weight scales, read before the wait so that their latency
    // overlaps it (the wait orders every memory access around it)
    float4 w4[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) w4[i] = *reinterpret_cast<const float4*>(sw + hc * 16 + 4 * i);
    tmem_ld_wait_regs16(acc[hc & 1]);
    if (hc + 1 < NCH) tmem_ld16(tacc + (hc + 1) * 16, acc[(hc + 1) & 1]);
    const uint32_t buf = stg + (stc & 1u) * 2048u;
    if ((hc & 1) == 0 && stc >= 2) {   // the store two boxes back must have read this buffer
      if (lane == 0) bulk_wait_group_read<1>();
      __syncwarp();
    }
#pragma unroll
    for (int c = 0; c < 2; ++c) {   // 8 columns -> one 16-byte shared store of BF16
      float y0[4], y1[4];
      scale4w(acc[hc & 1] + 8 * c, w4[2 * c], sa, y0);
      scale4w(acc[hc & 1] + 8 * c + 4, w4[2 * c + 1], sa, y1);
      __nv_bfloat162 h0 = __floats2bfloat162_rn(y0[0], y0[1]), h1 = __floats2bfloat162_rn(y0[2], y0[3]);
      __nv_bfloat162 h2 = __floats2bfloat162_rn(y1[0], y1[1]), h3 = __floats2bfloat162_rn(y1[2], y1[3]);
      const int cc = 2 * (hc & 1) + c;   // 16-byte column of the 32 x 32 box
      st_shared_v4(buf + lane * 64 + ((cc ^ ((lane >> 1) & 3)) << 4), *reinterpret_cast<uint32_t*>(&h0),
                   *reinterpret_cast<uint32_t*>(&h1), *reinterpret_cast<uint32_t*>(&h2),
                   *reinterpret_cast<uint32_t*>(&h3));
    }
    if (hc & 1) {
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) {
        tma_store_2d(ymap, buf, n0 + (hc >> 1) * 32, row0);   // rows >= M, columns >= N clipped by the map
        bulk_commit_group();
      }
      ++stc;
    }
  }
}

// ====================================================================== FP8
// Persistent, warp-specialised.  Shared-memory plan (operand buffers 1024-B aligned):
//   packed A  [SP][128 x 64 B]   (TMA, 64B swizzle)
//   packed B  [SP][BN x WROW]    (TMA, 64B swizzle; 32B swizzle for 2-bit codes)
//   e4m3 A    [SE][128 x 128 B]  (128B swizzle, K-major UMMA operand)
//   e4m3 B    [SE][BN x 128 B]
//   c / L     [128 x 64 B] / [BN x 64 B] (64B swizzle, BN == 128 only)
//   weight-scale slots [2][BN] FP32, barriers, TMEM address, abort flag
template <int BN, int WBITS, bool PAIR = false, bool A8 = false>
struct Fp8Plan {
  // BN = 256: two expanded stages (the expansion, not the MMA, sets the pace),
  // a deeper packed ring and 16 KB of output staging for the TMA-store
  // epilogue (4 warps x 2 x 2 KB); BN = 128: three expanded stages and 32 KB
  // of staging (16 grouped epilogue warps x 2 KB, or 4 warps x 2 x 2 KB).
  // PAIR (a CTA pair sharing 256 x 256 tiles): each CTA holds half of the
  // tile's weight rows, so four expanded stages fit.  BN = 512 (CTA pairs
  // only, 256 x 512 tiles): each CTA holds 256 weight rows per stage, two
  // 128-row halves of the two 256-wide output halves; three expanded stages
  // with two packed ones, which lets the expansion run a stage further ahead
  // of the MMAs (W2A4 GEMM 769 -> 722 us).  To fit them with 4-bit weights the
  // tile's weight scales take one slot (refilled after the drain) and the plan
  // carries no alignment slack: the kernel checks that its dynamic shared
  // memory starts 1024-byte aligned.
  static constexpr bool WIDE = BN == 512;
  static constexpr int BR = PAIR ? BN / 2 : BN;       // weight rows held by this CTA
  static constexpr int SP = WIDE ? 2 : PAIR ? 4 : BN == 256 ? (WBITS == 4 ? 4 : 5) : 4;
  static constexpr int SE = WIDE ? 3 : PAIR ? 4 : BN == 256 ? 2 : 3;
  static constexpr int STG = WIDE ? 32768 : BN >= 256 ? 16384 : 32768;
  static constexpr int WROW = WBITS == 4 ? 64 : 32;  // packed weight bytes per row per 128-wide K tile
  // A8 (8-bit activations, W4A8): the activation tile arrives as int8 in the
  // 128-byte-swizzled layout the MMA reads, straight into the packed stage
  static constexpr int PA = BM * (A8 ? 128 : 64), PB = BR * WROW, EA = A8 ? 0 : BM * 128, EB = BR * 128;
  static constexpr bool LR = BN == 128;
  static constexpr int OFF_PA = 0;
  static constexpr int OFF_PB = OFF_PA + SP * PA;
  static constexpr int OFF_EA = ((OFF_PB + SP * PB) + 1023) & ~1023;
  static constexpr int OFF_EB = OFF_EA + SE * EA;
  static constexpr int OFF_C = OFF_EB + SE * EB;
  static constexpr int OFF_L = OFF_C + (LR ? BM * 64 : 0);
  static constexpr int OFF_SC = OFF_L + (LR ? BN * 64 : 0);
  static constexpr int SCS = BN == 128 ? 12 : 2;               // grouped scale ring depth (BN 128 only)
  static constexpr int SC_BYTES = WIDE ? BN * 4 : (SCS * BN * 4 > 2 * BN * 4 ? SCS * BN * 4 : 2 * BN * 4);
  static constexpr int OFF_STG = (OFF_SC + SC_BYTES + 1023) & ~1023;
  static constexpr int OFF_BAR = OFF_STG + STG;
  static constexpr int NBAR = 2 * SP + 2 * SE + 6 + 4 + 2 * SCS + 1;   // + MMA drain after an abort
  static constexpr int SLACK = WIDE ? 0 : 1024;                 // alignment slack
  static constexpr int BYTES = OFF_BAR + NBAR * 8 + 16 + SLACK;
  static_assert(BYTES <= 232448, "shared memory plan exceeds 227 KB");
};

// Threads: warp 0 TMA producer, warp 1 TMEM owner + MMA issuer, then the
// epilogue warps from warp 4 (4 warps; 16 when GROUPED: four per TMEM lane
// quadrant, each owning 32 of the 128 columns and their running sums) and the
// code expansion warps: sixteen after the epilogue for BN = 256 (eight for
// BN = 128; the codebook lookups are issue-bound and four warps per scheduler
// hide their latencies), or, when
// GROUPED, warps 2-3 plus two after the epilogue (704 threads, so that the 16
// epilogue warps keep their running sums in registers without spilling).
// TMEM columns: GROUPED (INT4 weights, BN = 128): three per-group partials at
// 0, 128, 256 (the running sum lives in the epilogue's registers), low-rank at
// 384.  Otherwise: accumulators at 0 and BN (double-buffered across tiles),
// low-rank at 384 when BN == 128.
template <int BN, bool GROUPED>
constexpr int fp8_threads() { return GROUPED ? 704 : BN == 512 ? 640 : BN == 256 ? 768 : 512; }

template <int BN, int WBITS, bool GROUPED, bool PAIR = false, bool A8 = false>
__global__ void __launch_bounds__(fp8_threads<BN, GROUPED>(), 1) gemm_fp8_kernel(const __grid_constant__ TMaps tm, const __grid_constant__ GemmParams p) {
  static_assert(!PAIR || ((BN == 256 || BN == 512) && !GROUPED), "CTA pairs run the codebook tiles only");
  static_assert(BN != 512 || PAIR, "512-wide tiles run on CTA pairs");
  static_assert(!A8 || GROUPED, "8-bit activations run on the grouped INT4-weight kernel");
  using P = Fp8Plan<BN, WBITS, PAIR, A8>;
  // WIDE (256 x 512 pair tiles): two N = 256 pair MMAs per K step share the
  // expanded activation tile, accumulating into TMEM columns 0-255 and 256-511
  constexpr bool WIDE = P::WIDE;
  constexpr int MMA_N = WIDE ? 256 : BN;
  constexpr int NW = fp8_threads<BN, GROUPED>() / 32;
  // WIDE: epilogue warps 2-9 (two per TMEM lane quadrant, one per 256-column
  // half), expansion warps 10-19; otherwise epilogue from warp 4
  constexpr int EPI0 = (BN == 512) ? 2 : 4;      // first epilogue warp
  constexpr int NEPI = GROUPED ? 16 : (BN == 512) ? 8 : 4;   // epilogue warps
  constexpr int EXP0 = EPI0 + NEPI;              // first expansion warp
  constexpr int NXW = GROUPED ? 4 : NW - EXP0;   // expansion warps
  constexpr int NXT = NXW * 32;                  // expansion threads
  constexpr int NPART = 3;                       // GROUPED partial buffers
  extern __shared__ uint8_t smem_raw[];
  if constexpr (P::SLACK == 0) {
    // a plan without slack needs the dynamic shared memory 1024-byte aligned
    // (every CTA sees the same base, so all leave here together)
    if (smem_u32(smem_raw) & 1023u) {
      if (threadIdx.x == 0) atomicCAS(p.status, 0, ST_SMEM_ALIGN);
      return;
    }
  }
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
  const uint32_t sbase = smem_u32(smem);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + P::OFF_BAR);
  uint64_t* pfull = bars;                  // [SP] TMA -> expansion
  uint64_t* pempty = pfull + P::SP;        // [SP] expansion -> TMA
  uint64_t* efull = pempty + P::SP;        // [SE] expansion -> MMA
  uint64_t* eempty = efull + P::SE;        // [SE] MMA -> expansion
  uint64_t* accfull = eempty + P::SE;      // [3]  MMA -> epilogue
  uint64_t* accempty = accfull + 3;        // [3]  epilogue -> MMA
  uint64_t* lrfull = accempty + 3;         // c / L tiles landed (TMA -> MMA)
  uint64_t* lrsmem_empty = lrfull + 1;     // low-rank MMA read them (MMA -> TMA)
  uint64_t* lrdone = lrsmem_empty + 1;     // low-rank accumulator ready (MMA -> epilogue)
  uint64_t* lracc_empty = lrdone + 1;      // epilogue read it (epilogue -> MMA)
  uint64_t* scfull = lracc_empty + 1;      // [SCS] group scales landed (TMA -> epilogue)
  uint64_t* scempty = scfull + P::SCS;     // [SCS] epilogue used them (epilogue -> TMA)
  uint64_t* mdrain = scempty + P::SCS;     // MMA thread's own commits, drained after an abort
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + P::NBAR);
  volatile int32_t* abort_flag = reinterpret_cast<volatile int32_t*>(tmem_slot + 1);
  float* sc_slots = reinterpret_cast<float*>(smem + P::OFF_SC);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // 128-wide K tiles (== INT4 groups); codebook codes may end in a half tile
  // (K % 128 == 64): its zero-filled upper half is expanded but never multiplied.
  // (The count comes from the host: derived from K in the kernel, the codebook
  // loop measured ~0.8% slower.)
  const int nk = p.nk128;
  const int kk_last = (p.K - (nk - 1) * 128) / 32;   // 32-code MMAs in the last K tile (2 or 4)
  constexpr bool grouped = GROUPED;
  const bool lr = P::LR && p.has_lr;
  // PAIR: the two CTAs of a cluster share 256 x BN tiles; CTA `crank` takes
  // rows crank*128 .. +127 of the tile and weight rows crank*BN/2 .. +BN/2-1,
  // and the even CTA issues the pair's MMAs.
  const uint32_t crank = PAIR ? cluster_ctarank() : 0u;
  constexpr int TM = PAIR ? 2 * BM : BM;
  const int nN = (p.N + BN - 1) / BN, nM = (p.M + TM - 1) / TM;
  const int ntiles = nM * nN;
  const int tile0 = PAIR ? (int)(blockIdx.x >> 1) : (int)blockIdx.x;
  const int tstep = PAIR ? (int)(gridDim.x >> 1) : (int)gridDim.x;
  // Work items, the same sequence for every role: tiles tile0, tile0 + tstep,
  // ...  WIDE: when the last round of tiles would leave at least half of the
  // pairs idle, its tiles are split into their two 256-column halves, one
  // half per pair (half = 0 or 1; -1 is the whole tile), so that round takes
  // about half as long.  Only with few rounds, where the tail is a sizeable
  // share of the work (FLUX QKV: 4 full rounds and 28 of 74 pairs busy in the
  // fifth, 128.5 -> 125.7 us); with many rounds it measured no gain.
  const int nfull = ntiles / tstep, nrem = ntiles - nfull * tstep;
  const bool split_tail = WIDE && nfull < 8 && nrem > 0 && 2 * nrem <= tstep;
  auto item_at = [&](int i, int& tile, int& half) -> bool {
    half = -1;
    tile = tile0 + i * tstep;
    if (!split_tail || i < nfull) return tile < ntiles;
    if (i > nfull || tile0 >= 2 * nrem) return false;
    tile = nfull * tstep + (tile0 >> 1);
    half = tile0 & 1;
    return true;
  };

  if (threadIdx.x == 0) {
    // (A8: the MMA thread also releases each stage, after reading its activation tile)
    for (int i = 0; i < P::SP; ++i) { mbar_init(&pfull[i], 1); mbar_init(&pempty[i], NXW + (A8 ? 1 : 0)); }
    // PAIR: efull / accempty of the even CTA count both CTAs' warps; eempty and
    // accfull take one multicast commit arrival in each CTA
    for (int i = 0; i < P::SE; ++i) { mbar_init(&efull[i], PAIR ? 2 * NXW : NXW); mbar_init(&eempty[i], 1); }
    // PAIR: every epilogue warp of both CTAs (WIDE: per 256-column half)
    constexpr int ACC_ARRIVALS = PAIR ? 2 * NEPI : NEPI;
    for (int i = 0; i < 3; ++i) { mbar_init(&accfull[i], 1); mbar_init(&accempty[i], ACC_ARRIVALS); }
    mbar_init(lrfull, 1);
    mbar_init(lrsmem_empty, 1);
    mbar_init(lrdone, 1);
    mbar_init(lracc_empty, NEPI);
    for (int i = 0; i < P::SCS; ++i) { mbar_init(&scfull[i], 1); mbar_init(&scempty[i], NEPI); }
    mbar_init(mdrain, 1);
    *abort_flag = 0;
    fence_mbar_init();
    prefetch_tmap(&tm.a);
    prefetch_tmap(&tm.b);
  }
  if (warp == 1) {
    if constexpr (PAIR) {
      tmem_alloc2(tmem_slot, 512);
      tmem_relinquish2();
    } else {
      tmem_alloc(tmem_slot, 512);
      tmem_relinquish();
    }
  }
  tc_fence_before();
  if constexpr (PAIR)
    cluster_sync();   // both CTAs' barriers exist before either arrives on the other's
  else
    __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  // launched as a programmatic dependent of the activation kernel: the
  // prologue above overlaps its tail; nothing it writes is read before this
  griddep_wait();

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      uint32_t kc = 0;
      int tc = 0;
      uint32_t sgc = 0;                    // group-scale ring counter (GROUPED)
      int lr_issued = 0;
      int tile, half;
      for (int i = 0; item_at(i, tile, half) && !*abort_flag; ++i, ++tc) {
        const int m0 = (tile / nN) * TM + (int)crank * BM, n0 = (tile % nN) * BN;
        for (int kt = 0; kt < nk; ++kt, ++kc) {
          if constexpr (GROUPED) {
            // this group's weight scales s_w[kt, n0 .. n0+127] (one contiguous row slice)
            const int ss = sgc % P::SCS;
            if (sgc >= P::SCS && !mbar_wait(&scempty[ss], ((sgc / P::SCS) - 1) & 1, p.status, ST_TIMEOUT_EMPTY, abort_flag, p.wait_ns)) break;
            const uint32_t nbytes = (uint32_t)min(128, p.N - n0) * 4;
            mbar_expect_tx(&scfull[ss], nbytes);
            bulk_g2s(sc_slots + ss * 128, p.w_scale + (size_t)kt * p.N + n0, nbytes, &scfull[ss]);
            ++sgc;
          }
          const int s = kc % P::SP;
          if (kc >= P::SP && !mbar_wait(&pempty[s], ((kc / P::SP) - 1) & 1, p.status, ST_TIMEOUT_EMPTY, abort_flag, p.wait_ns)) break;
          // (the test hook overstates the first stage's byte count: the copies
          // land, the consumers' bounded waits for the stage run out)
          mbar_expect_tx(&pfull[s], P::PA + (half < 0 ? P::PB : P::PB / 2) + (kc == 0 ? p.inject_tx : 0u));
          tma_load_2d(smem + P::OFF_PA + s * P::PA, &tm.a, kt * (A8 ? 128 : 64), m0, &pfull[s]);
          if constexpr (WIDE) {
            // this CTA's 128 rows of each 256-wide half of the tile's weight
            // rows (of the one half a split item computes)
#pragma unroll
            for (int h = 0; h < 2; ++h)
              if (half < 0 || h == half)
                tma_load_2d(smem + P::OFF_PB + s * P::PB + h * 128 * P::WROW, &tm.b, kt * P::WROW,
                            n0 + h * 256 + (int)crank * 128, &pfull[s]);
          } else {
            tma_load_2d(smem + P::OFF_PB + s * P::PB, &tm.b, kt * P::WROW, n0 + (int)crank * P::BR, &pfull[s]);
          }
        }
        // the tile's low-rank operands go after its K tiles, so waiting for the
        // previous tile's low-rank MMA never stalls the K-tile prefetch
        if (lr) {
          if (tc > 0 && !mbar_wait(lrsmem_empty, (tc - 1) & 1, p.status, ST_TIMEOUT_EMPTY, abort_flag, p.wait_ns)) break;
          mbar_expect_tx(lrfull, BM * 64 + BN * 64);
          tma_load_2d(smem + P::OFF_C, &tm.c, 0, m0, lrfull);
          tma_load_2d(smem + P::OFF_L, &tm.l, 0, n0, lrfull);
          ++lr_issued;
        }
      }
      if (*abort_flag) {
        // after an abort: let the copies already issued land (bounded) before
        // this CTA's shared memory is released
        for (uint32_t c = kc > (uint32_t)P::SP ? kc - P::SP : 0; c < kc; ++c)
          mbar_drain(&pfull[c % P::SP], (c / P::SP) & 1, p.wait_ns);
        for (uint32_t c = sgc > (uint32_t)P::SCS ? sgc - P::SCS : 0; c < sgc; ++c)
          mbar_drain(&scfull[c % P::SCS], (c / P::SCS) & 1, p.wait_ns);
        if (lr_issued > 0) mbar_drain(lrfull, (lr_issued - 1) & 1, p.wait_ns);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0 && crank == 0) {
      // (PAIR: M = 256, the instruction descriptor's M field is M / 16)
      const uint32_t idesc =
          GROUPED ? idesc_i8(BN) : PAIR ? (idesc_f8(MMA_N) & ~(0x1Fu << 24)) | (16u << 24) : idesc_f8(BN);
      uint32_t kc = 0, gc = 0;
      int tc = 0;
      bool ok = true;
      // The low-rank MMA of a tile is issued after its K loop, when the epilogue
      // has long finished reading the previous tile's low-rank accumulator.
      auto lowrank = [&](int tcx) -> bool {
        if (!(mbar_wait(lrfull, tcx & 1, p.status, ST_TIMEOUT_FULL, abort_flag, p.wait_ns) &&
              (tcx == 0 || mbar_wait(lracc_empty, (tcx - 1) & 1, p.status, ST_TIMEOUT_EPI, abort_flag, p.wait_ns))))
          return false;
        tc_fence_after();
        const uint32_t ca = sbase + P::OFF_C, la = sbase + P::OFF_L;
#pragma unroll
        for (int kk = 0; kk < 2; ++kk)
          umma_bf16(tmem + 384, smem_desc(ca + kk * 32, 16, 512, 4), smem_desc(la + kk * 32, 16, 512, 4),
                    idesc_bf16(BN), kk > 0);
        tc_commit(lrdone);
        tc_commit(lrsmem_empty);
        return true;
      };
      if constexpr (WIDE) {
        // single accumulators (all 512 columns): the first MMA of a tile into
        // either half waits until the epilogue has drained that half of the
        // previous tile.  Two copies of the loop: whole last K tiles (the
        // common case, no per-step test) or half ones (K % 128 == 64)
        static_assert(P::SE >= 2, "the first two K tiles of a tile are held at once");
        auto wide_loop = [&](auto half_tail) {
        constexpr bool HALF = decltype(half_tail)::value;
        int tile, half;
        // one K tile's MMAs into half h (TMEM columns h*256 ..) from stage s
        // (none for the half a split item leaves out)
        auto issue = [&](int h, int s, int kt) {
          if (half >= 0 && h != half) return;
          const uint32_t a = sbase + P::OFF_EA + s * P::EA, b = sbase + P::OFF_EB + s * P::EB;
          const int kkn = (HALF && kt == nk - 1) ? 2 : 4;
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            if (!HALF || kk < kkn)
              umma_f8_2(tmem + h * 256, smem_desc(a + kk * 32, 16, 1024, 2),
                        smem_desc(b + h * 128 * 128 + kk * 32, 16, 1024, 2), idesc, (kt == 0 && kk == 0) ? 0u : 1u);
        };
        for (int i = 0; item_at(i, tile, half) && ok; ++i, ++tc) {
          int kt = 0;
          if (tc > 0 && nk >= 2) {
            // the epilogue frees the first half first: its MMAs of the first
            // K tiles (as many as there are expanded stages) run while the
            // second half is still being drained
            const int npre = nk < P::SE ? nk : P::SE;
            ok = mbar_wait(&accempty[0], (tc - 1) & 1, p.status, ST_TIMEOUT_EPI, abort_flag, p.wait_ns);
            for (int j = 0; j < npre && ok; ++j) {
              ok = mbar_wait(&efull[(kc + j) % P::SE], ((kc + j) / P::SE) & 1, p.status, ST_TIMEOUT_FULL, abort_flag,
                             p.wait_ns);
              if (!ok) break;
              tc_fence_after();
              issue(0, (kc + j) % P::SE, j);
            }
            if (!ok) break;
            ok = mbar_wait(&accempty[1], (tc - 1) & 1, p.status, ST_TIMEOUT_EPI, abort_flag, p.wait_ns);
            if (!ok) break;
            tc_fence_after();
            for (int j = 0; j < npre; ++j) {
              issue(1, (kc + j) % P::SE, j);
              tc_commit2_mc(&eempty[(kc + j) % P::SE], 0x3);   // the stage is free in both CTAs
            }
            kt = npre;
            kc += npre;
          }
          for (; kt < nk; ++kt, ++kc) {
            const int s = kc % P::SE;
            ok = mbar_wait(&efull[s], (kc / P::SE) & 1, p.status, ST_TIMEOUT_FULL, abort_flag, p.wait_ns);
            if (!ok) break;
            tc_fence_after();
#pragma unroll
            for (int h = 0; h < 2; ++h) {
              if (kt == 0 && tc > 0) {   // (a single K tile per output tile)
                ok = mbar_wait(&accempty[h], (tc - 1) & 1, p.status, ST_TIMEOUT_EPI, abort_flag, p.wait_ns);
                if (!ok) break;
                tc_fence_after();
              }
              issue(h, s, kt);
            }
            if (!ok) break;
            tc_commit2_mc(&eempty[s], 0x3);   // the stage is free in both CTAs
          }
          if (!ok) break;
          tc_commit2_mc(&accfull[0], 0x3);
        }
        };
        if (kk_last == 4)
          wide_loop(std::false_type{});
        else
          wide_loop(std::true_type{});
      }
      for (int tile = tile0; tile < ntiles && ok && !WIDE; tile += tstep, ++tc) {
        const uint32_t ab = tc & 1;
        if (!grouped && tc >= 2) {
          ok = mbar_wait(&accempty[ab], ((tc >> 1) - 1) & 1, p.status, ST_TIMEOUT_EPI, abort_flag, p.wait_ns);
          if (!ok) break;
          tc_fence_after();
        }
        for (int kt = 0; kt < nk; ++kt, ++kc) {
          uint32_t buf = ab;
          if (grouped) {
            buf = gc % NPART;
            if (gc >= NPART) {
              ok = mbar_wait(&accempty[buf], ((gc / NPART) - 1) & 1, p.status, ST_TIMEOUT_EPI, abort_flag, p.wait_ns);
              if (!ok) break;
              tc_fence_after();
            }
          }
          const int s = kc % P::SE;
          ok = mbar_wait(&efull[s], (kc / P::SE) & 1, p.status, ST_TIMEOUT_FULL, abort_flag, p.wait_ns);
          if (A8 && ok)   // the activation tile of this stage (landed before the expansion began)
            ok = mbar_wait(&pfull[kc % P::SP], (kc / P::SP) & 1, p.status, ST_TIMEOUT_FULL, abort_flag, p.wait_ns);
          if (!ok) break;
          tc_fence_after();
          const uint32_t a = A8 ? sbase + P::OFF_PA + (kc % P::SP) * P::PA : sbase + P::OFF_EA + s * P::EA;
          const uint32_t b = sbase + P::OFF_EB + s * P::EB;
          const bool fresh = grouped || kt == 0;
          const int kkn = kt == nk - 1 ? kk_last : 4;
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) {
            if (kk >= kkn) break;
            if constexpr (GROUPED)
              umma_i8(tmem + buf * 128, smem_desc(a + kk * 32, 16, 1024, 2), smem_desc(b + kk * 32, 16, 1024, 2),
                      idesc, (fresh && kk == 0) ? 0u : 1u);
            else if constexpr (PAIR)
              umma_f8_2(tmem + buf * BN, smem_desc(a + kk * 32, 16, 1024, 2), smem_desc(b + kk * 32, 16, 1024, 2),
                        idesc, (fresh && kk == 0) ? 0u : 1u);
            else
              umma_f8(tmem + buf * BN, smem_desc(a + kk * 32, 16, 1024, 2), smem_desc(b + kk * 32, 16, 1024, 2),
                      idesc, (fresh && kk == 0) ? 0u : 1u);
          }
          if constexpr (PAIR)
            tc_commit2_mc(&eempty[s], 0x3);   // the stage is free in both CTAs
          else
            tc_commit(&eempty[s]);
          if constexpr (A8) tc_commit(&pempty[kc % P::SP]);
          if (grouped) {
            tc_commit(&accfull[buf]);
            ++gc;
          }
        }
        if (!ok) break;
        if constexpr (PAIR)
          tc_commit2_mc(&accfull[ab], 0x3);
        else if (!grouped)
          tc_commit(&accfull[ab]);
        if (lr && !(ok = lowrank(tc))) break;
      }
      if (!ok) {
        // after an abort: wait (bounded) for the MMAs already issued before
        // TMEM and the operand stages are released
        if constexpr (PAIR)
          tc_commit2_mc(mdrain, 0x1);
        else
          tc_commit(mdrain);
        mbar_drain(mdrain, 0, p.wait_ns);
      }
    }
  } else if (warp >= EPI0 && warp < EXP0) {
    // ------------------------------------------------------------ epilogue
    const int e = warp - EPI0;
    const int q = warp & 3;                  // TMEM lane quadrant (warp id % 4)
    const int tid = threadIdx.x - 32 * EPI0; // 0 .. 32*NEPI-1
    const uint32_t lane_off = (uint32_t)(q * 32) << 16;
    uint32_t gc = 0;
    uint32_t stc = 0;   // TMA-store chunks issued by this warp
    const uint32_t stg = sbase + P::OFF_STG + (uint32_t)e * (GROUPED ? 2048u : 4096u);
    int tc = 0;
    bool ok = true;
    // Without GROUPED the epilogue warps meet at named barriers every tile, so
    // after an abort they keep walking the tile loop (skipping the work) rather
    // than leaving it one by one: every warp reaches every barrier.
    int tile, half;
    for (int i = 0; item_at(i, tile, half) && (ok || !GROUPED); ++i, ++tc) {
      const int m0 = (tile / nN) * TM + (int)crank * BM, n0 = (tile % nN) * BN;
      const int row = m0 + q * 32 + lane;
      const float sa = row < p.M ? __ldg(p.a_scale + row) : 0.f;
      if constexpr (GROUPED) {
        // per 128-wide K group: running[n] += s_w[g, n] * partial_g[m, n], in
        // registers; this warp owns columns h*32 .. h*32+31 of the tile.  The
        // 1/256 of the 16 x 16 code scaling is applied once at the end (exact).
        const int h = e >> 2;
        float run[32];
#pragma unroll
        for (int i = 0; i < 32; ++i) run[i] = 0.f;
        for (int g = 0; g < nk; ++g, ++gc) {
          const uint32_t buf = gc % NPART;
          const int ss = gc % P::SCS;
          ok = mbar_wait(&scfull[ss], (gc / P::SCS) & 1, p.status, ST_TIMEOUT_FULL, abort_flag, p.wait_ns) &&
               mbar_wait(&accfull[buf], (gc / NPART) & 1, p.status, ST_TIMEOUT_MMA, abort_flag, p.wait_ns);
          if (!ok) break;
          tc_fence_after();
          const float* sw = sc_slots + ss * 128 + h * 32;
#pragma unroll
          for (int c = 0; c < 2; ++c) {
            uint32_t acc[16];
            tmem_ld16(tmem + lane_off + buf * 128 + h * 32 + c * 16, acc);
            // the group scales, read before the wait (which orders every
            // memory access around it) so that their latency overlaps it
            float4 w4[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) w4[i] = *reinterpret_cast<const float4*>(sw + c * 16 + 4 * i);
            tmem_ld_wait_regs16(acc);
#pragma unroll
            for (int i = 0; i < 4; ++i) {
              // S32 partials (|x| <= 256 * 49 * 128 < 2^21) convert to FP32 exactly
              fma_s32x2(run[c * 16 + 4 * i], run[c * 16 + 4 * i + 1], w4[i].x, w4[i].y, acc[4 * i], acc[4 * i + 1]);
              fma_s32x2(run[c * 16 + 4 * i + 2], run[c * 16 + 4 * i + 3], w4[i].z, w4[i].w, acc[4 * i + 2],
                        acc[4 * i + 3]);
            }
          }
          tc_fence_before();
          __syncwarp();
          if (lane == 0) {
            mbar_arrive(&accempty[buf]);   // the tensor core may reuse this partial
            mbar_arrive(&scempty[ss]);     // the producer may refill this scale slot
          }
        }
        if (!ok) break;
        // codes enter the MMA as 16 v (4-bit) or as themselves (8-bit activations)
        const float sa256 = sa * (A8 ? 0.0625f : 0.00390625f);
        if (lr) {
          ok = mbar_wait(lrdone, tc & 1, p.status, ST_TIMEOUT_MMA, abort_flag, p.wait_ns);
          if (!ok) break;
          tc_fence_after();
#pragma unroll
          for (int c = 0; c < 2; ++c) {
            uint32_t l[16];
            tmem_ld16(tmem + lane_off + 384 + h * 32 + c * 16, l);
            tmem_ld_wait();
#pragma unroll
            for (int i = 0; i < 16; ++i) run[c * 16 + i] = fmaf(run[c * 16 + i], sa256, __uint_as_float(l[i]));
          }
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(lracc_empty);
        } else {
#pragma unroll
          for (int i = 0; i < 32; ++i) run[i] *= sa256;
        }
        if (p.a_zp) {
          // asymmetric activations: x = s_a (nibble + z), so the layer adds
          // s_a z sum_g s_w[g, n] sum_k q_w[n, k] (TR-DQ section 3.1, Eq. 1-3)
          const float szp = row < p.M ? sa * __ldg(p.a_zp + row) : 0.f;
          const int nb = n0 + h * 32;
#pragma unroll
          for (int i = 0; i < 32; ++i)
            if (nb + i < p.N) run[i] = fmaf(szp, __ldg(p.w_zsum + nb + i), run[i]);
        }
        if (!p.tma_store) {
          if (row < p.M) store_row32(p.Y, p.out_fp32, p.N, row, n0 + h * 32, run);
        } else {
          // the warp's 32 x 32 block through shared memory and one TMA store
          // (single buffer: the previous tile's store has read it long ago)
          if (stc > 0) {
            if (lane == 0) bulk_wait_group_read<0>();
            __syncwarp();
          }
          uint32_t w[16];
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            __nv_bfloat162 hb = __floats2bfloat162_rn(run[2 * i], run[2 * i + 1]);
            w[i] = *reinterpret_cast<uint32_t*>(&hb);
          }
#pragma unroll
          for (int c = 0; c < 4; ++c)
            st_shared_v4(stg + lane * 64 + ((c ^ ((lane >> 1) & 3)) << 4), w[4 * c], w[4 * c + 1], w[4 * c + 2],
                         w[4 * c + 3]);
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) {
            tma_store_2d(&tm.y, stg, n0 + h * 32, m0 + q * 32);
            bulk_commit_group();
          }
          ++stc;
        }
      } else if constexpr (WIDE) {
        // all eight warps drain the first 256-column half, then the second:
        // the next tile's MMAs into the first half start while the second
        // drains.  This warp takes 128 columns of each half.
        const int part = e >> 2;
        // one scale slot: filled once every epilogue warp has finished the
        // previous tile (the barrier after the drain below)
        float* sw = sc_slots;
        load_scales_smem(sw, p.w_scale, n0, p.N, BN, tid, 32 * NEPI);
        epi_bar_n<32 * NEPI>();
        ok = ok && mbar_wait(&accfull[0], tc & 1, p.status, ST_TIMEOUT_MMA, abort_flag, p.wait_ns);
        if (ok) {
          tc_fence_after();
#pragma unroll 1
          for (int hh = 0; hh < 2; ++hh) {
            const int c0 = hh * 256 + part * 128;
            if (half < 0 || hh == half)
              epi_cols_wide<8>(p, &tm.y, tmem + lane_off + c0, sw + c0, sa, row, n0 + c0, m0 + q * 32, stg, stc);
            // this half may take the next tile's first MMAs
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive_cluster(&accempty[hh], 0);
          }
        }
        epi_bar_n<32 * NEPI>();   // the scale slot is free
      } else {
        const uint32_t ab = tc & 1;
        float* sw = sc_slots + ab * BN;
        load_scales_smem(sw, p.w_scale, n0, p.N, BN, tid);
        epi_bar_n<32 * NEPI>();
        ok = ok && mbar_wait(&accfull[ab], (tc >> 1) & 1, p.status, ST_TIMEOUT_MMA, abort_flag, p.wait_ns) &&
             (!lr || mbar_wait(lrdone, tc & 1, p.status, ST_TIMEOUT_MMA, abort_flag, p.wait_ns));
        if (ok) {
          tc_fence_after();
#pragma unroll 1
          for (int ch = 0; ch < BN / 32; ++ch)
            epi_chunk_final(p, tmem + lane_off + ab * BN + ch * 32, tmem + lane_off + 384 + ch * 32, lr,
                            sw + ch * 32, sa, row, n0 + ch * 32, &tm.y, stg, &stc, m0 + q * 32);
          tc_fence_before();
          __syncwarp();
          if (lane == 0) {
            if constexpr (PAIR)
              mbar_arrive_cluster(&accempty[ab], 0);
            else
              mbar_arrive(&accempty[ab]);
            if (lr) mbar_arrive(lracc_empty);
          }
        }
      }
    }
    // the staging buffers must outlive the TMA stores that read them
    if (lane == 0) bulk_wait_group<0>();
  } else if (warp >= EXP0 || (GROUPED && warp >= 2)) {
    // ------------------------------------------------------------ code expansion
    const int t = (GROUPED && warp < 4 ? warp - 2 + (NW - EXP0) : warp - EXP0) * 32 + lane;  // 0 .. NXT-1
    uint32_t LA[4], LW[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      LA[i] = p.a_lut[i];
      LW[i] = GROUPED ? LA[i] : p.w_lut[i];   // INT4 x INT4 shares one table
    }
    uint32_t kc = 0;
    bool ok = true;
    int tile, half;
    for (int i = 0; item_at(i, tile, half) && ok; ++i) {
      // the weight rows this CTA expands: both 128-row halves, or the one a
      // split item computes (items [bo, bo + bl) of the loops below)
      const int bitems = P::BR * (WBITS == 4 ? 4 : 2);
      const int bl = half < 0 ? bitems : bitems / 2, bo = half < 0 ? 0 : half * (bitems / 2);
      for (int kt = 0; kt < nk; ++kt, ++kc) {
        const int sp = kc % P::SP, se = kc % P::SE;
        ok = mbar_wait(&pfull[sp], (kc / P::SP) & 1, p.status, ST_TIMEOUT_FULL, abort_flag, p.wait_ns) &&
             (kc < P::SE || mbar_wait(&eempty[se], ((kc / P::SE) - 1) & 1, p.status, ST_TIMEOUT_EMPTY, abort_flag, p.wait_ns));
        if (!ok) break;
        const uint32_t pa = sbase + P::OFF_PA + sp * P::PA, pb = sbase + P::OFF_PB + sp * P::PB;
        const uint32_t ea = sbase + P::OFF_EA + se * P::EA, eb = sbase + P::OFF_EB + se * P::EB;
        if constexpr (GROUPED) {
          // INT4 codes -> int8 16 v: word j of a 16-byte segment becomes
          // {even codes << 4, odd codes} (same k order for A and B; with
          // 8-bit activations, which arrive in natural k order, the two
          // halves are interleaved back into natural order)
          // loads in batches of four: the shared-memory accesses are ordered,
          // so batching keeps four in flight at once
          // (A8: only the weight codes; the activation tile is already the operand)
          constexpr int NIT = (A8 ? 512 : 1024) / NXT, NB = 4;
#pragma unroll
          for (int b0 = 0; b0 < NIT; b0 += NB) {
            uint4 vin[NB];
#pragma unroll
            for (int j = 0; j < NB; ++j) {
              const int idx0 = (b0 + j) * NXT + t + (A8 ? 512 : 0);
              const bool isb = idx0 >= 512;
              const int idx = isb ? idx0 - 512 : idx0;
              const int r = (idx >> 5) * 8 + (idx & 7), seg = (idx >> 3) & 3;
              vin[j] = ld_shared_v4((isb ? pb : pa) + r * 64 + ((seg ^ ((r >> 1) & 3)) << 4));
            }
#pragma unroll
            for (int j = 0; j < NB; ++j) {
              const int idx0 = (b0 + j) * NXT + t + (A8 ? 512 : 0);
              const bool isb = idx0 >= 512;
              const int idx = isb ? idx0 - 512 : idx0;
              const int r = (idx >> 5) * 8 + (idx & 7), seg = (idx >> 3) & 3;
              const uint32_t dst = isb ? eb : ea;
              const uint32_t w[4] = {vin[j].x, vin[j].y, vin[j].z, vin[j].w};
              uint32_t o[8];
#pragma unroll
              for (int q = 0; q < 4; ++q) {
                const uint32_t lo = (w[q] << 4) & 0xF0F0F0F0u, hi = w[q] & 0xF0F0F0F0u;
                if constexpr (A8) {
                  o[2 * q] = __byte_perm(lo, hi, 0x5140);
                  o[2 * q + 1] = __byte_perm(lo, hi, 0x7362);
                } else {
                  o[2 * q] = lo;
                  o[2 * q + 1] = hi;
                }
              }
              const uint32_t rowb = dst + r * 128;
              st_shared_v4(rowb + (((2 * seg) ^ (r & 7)) << 4), o[0], o[1], o[2], o[3]);
              st_shared_v4(rowb + (((2 * seg + 1) ^ (r & 7)) << 4), o[4], o[5], o[6], o[7]);
            }
          }
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) {
            mbar_arrive(&efull[se]);
            mbar_arrive(&pempty[sp]);
          }
          continue;
        }
        // A: 128 rows x 4 segments of 16 packed bytes (32 codes); 8 consecutive
        // threads take 8 consecutive rows of one segment (conflict-free both ways)
        constexpr int NA = (512 + NXT - 1) / NXT;
        uint4 va[NA];
#pragma unroll
        for (int it = 0; it < NA; ++it) {
          const int idx = it * NXT + t;
          const int r = (idx >> 5) * 8 + (idx & 7), seg = (idx >> 3) & 3;
          if (idx < 512) va[it] = ld_shared_v4(pa + r * 64 + ((seg ^ ((r >> 1) & 3)) << 4));
        }
#pragma unroll
        for (int it = 0; it < NA; ++it) {
          const int idx = it * NXT + t;
          if (idx >= 512) break;
          const int r = (idx >> 5) * 8 + (idx & 7), seg = (idx >> 3) & 3;
          const uint4 v = va[it];
          const uint32_t w[4] = {v.x, v.y, v.z, v.w};
          uint32_t o[8];
#pragma unroll
          for (int j = 0; j < 4; ++j) lut_sm8(w[j], LA[2], LA[3], o[2 * j], o[2 * j + 1]);
          const uint32_t rowb = ea + r * 128;
          st_shared_v4(rowb + (((2 * seg) ^ (r & 7)) << 4), o[0], o[1], o[2], o[3]);
          st_shared_v4(rowb + (((2 * seg + 1) ^ (r & 7)) << 4), o[4], o[5], o[6], o[7]);
        }
        if constexpr (WBITS == 4) {
          constexpr int NBI = (P::BR * 4 + NXT - 1) / NXT;
          uint4 vb[NBI];
#pragma unroll
          for (int it = 0; it < NBI; ++it) {
            const int idx = it * NXT + t + bo;
            const int r = (idx >> 5) * 8 + (idx & 7), seg = (idx >> 3) & 3;
            if (idx < bo + bl) vb[it] = ld_shared_v4(pb + r * 64 + ((seg ^ ((r >> 1) & 3)) << 4));
          }
#pragma unroll
          for (int it = 0; it < NBI; ++it) {
            const int idx = it * NXT + t + bo;
            if (idx >= bo + bl) break;
            const int r = (idx >> 5) * 8 + (idx & 7), seg = (idx >> 3) & 3;
            const uint4 v = vb[it];
            const uint32_t w[4] = {v.x, v.y, v.z, v.w};
            uint32_t o[8];
#pragma unroll
            for (int j = 0; j < 4; ++j) lut_sm8(w[j], LW[2], LW[3], o[2 * j], o[2 * j + 1]);
            const uint32_t rowb = eb + r * 128;
            st_shared_v4(rowb + (((2 * seg) ^ (r & 7)) << 4), o[0], o[1], o[2], o[3]);
            st_shared_v4(rowb + (((2 * seg + 1) ^ (r & 7)) << 4), o[4], o[5], o[6], o[7]);
          }
        } else {
          // 2-bit weights: 32 packed bytes per row = 2 segments of 64 codes
          constexpr int NBI = (P::BR * 2 + NXT - 1) / NXT;
          uint4 vb[NBI];
#pragma unroll
          for (int it = 0; it < NBI; ++it) {
            const int idx = it * NXT + t + bo;
            const int r = (idx >> 4) * 8 + (idx & 7), seg = (idx >> 3) & 1;
            if (idx < bo + bl) vb[it] = ld_shared_v4(pb + r * 32 + ((seg ^ ((r >> 2) & 1)) << 4));
          }
#pragma unroll
          for (int it = 0; it < NBI; ++it) {
            const int idx = it * NXT + t + bo;
            if (idx >= bo + bl) break;
            const int r = (idx >> 4) * 8 + (idx & 7), seg = (idx >> 3) & 1;
            const uint4 v = vb[it];
            const uint32_t w[4] = {v.x, v.y, v.z, v.w};
            uint32_t o[16];
#pragma unroll
            for (int j = 0; j < 4; ++j) {
              uint32_t q[4];
              lut4x16(w[j], LW[0], q);
              o[4 * j] = q[0];
              o[4 * j + 1] = q[1];
              o[4 * j + 2] = q[2];
              o[4 * j + 3] = q[3];
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
          if constexpr (PAIR)
            mbar_arrive_cluster(&efull[se], 0);   // the even CTA's MMA waits for both halves
          else
            mbar_arrive(&efull[se]);
          mbar_arrive(&pempty[sp]);
        }
      }
    }
    if constexpr (PAIR) {
      // the even CTA's last commits land in this CTA's barriers: wait for them
      // before this CTA may leave
      for (uint32_t c = kc > (uint32_t)P::SE ? kc - P::SE : 0; ok && c < kc; ++c)
        ok = mbar_wait(&eempty[c % P::SE], (c / P::SE) & 1, p.status, ST_TIMEOUT_EMPTY, abort_flag, p.wait_ns);
    }
  }

  tc_fence_before();
  if constexpr (PAIR) {
    cluster_sync();   // neither CTA leaves while the other may still touch its barriers
    if (warp == 1) {
      tc_fence_after();
      tmem_dealloc2(tmem, 512);
    }
  } else {
    __syncthreads();
    if (warp == 1) {
      tc_fence_after();
      tmem_dealloc(tmem, 512);
    }
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
  static constexpr int NACC = BN == 256 ? 1 : 2;
  static constexpr int OFF_C = S * STAGE;
  static constexpr int OFF_L = OFF_C + (LR ? BM * 64 : 0);
  static constexpr int OFF_SC = OFF_L + (LR ? BN * 64 : 0);
  static constexpr int OFF_BAR = OFF_SC + 2 * BN * 4;
  static constexpr int NBAR = 2 * S + 4 + 4 + 8 + 2;   // + MMA and scale-copy drains after an abort
  static constexpr int BYTES = OFF_BAR + NBAR * 8 + 16 + 1024;
  static_assert(BYTES <= 232448, "shared memory plan exceeds 227 KB");
};

// Persistent.  TMEM columns: accumulator(s) at 0 (BN = 256: one; BN = 128: two,
// at 0 and 128), low-rank at 384 (BN = 128), scale factors in a ring of slots
// from column 256 (BN = 256: 4 slots of 48 columns; BN = 128: 4 slots of 32),
// one slot per k-tile in flight, so a k-tile's tcgen05.cp never waits for the
// previous k-tile's MMAs to finish reading their scales.
// Threads: warp 0 TMA producer, warp 1 TMEM owner + MMA issuer, warp 2 scale
// factors -> TMEM, warp 3 idle, warps 4-11 epilogue (two per TMEM lane quadrant,
// each half of the tile's columns: the BN = 256 accumulator is single-buffered,
// so the epilogue's length is a pipeline bubble).
constexpr int NVF4_THREADS = 384;

template <int BN>
__global__ void __launch_bounds__(NVF4_THREADS, 1) gemm_nvf4_kernel(const __grid_constant__ TMaps tm, const __grid_constant__ GemmParams p) {
  using P = Nvf4Plan<BN>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
  const uint32_t sbase = smem_u32(smem);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + P::OFF_BAR);
  uint64_t* full = bars;
  uint64_t* empty = full + P::S;
  uint64_t* accfull = empty + P::S;        // [2]
  uint64_t* accempty = accfull + 2;        // [2]
  uint64_t* lrfull = accempty + 2;
  uint64_t* lrsmem_empty = lrfull + 1;
  uint64_t* lrdone = lrsmem_empty + 1;
  uint64_t* lracc_empty = lrdone + 1;
  uint64_t* sffull = lracc_empty + 1;      // [4] scale factors in TMEM (copy warp -> MMA)
  uint64_t* sfempty = sffull + 4;          // [4] MMAs done with a slot (MMA -> copy warp)
  uint64_t* mdrain = sfempty + 4;          // MMA thread's own commits, drained after an abort
  uint64_t* cdrain = mdrain + 1;           // scale-copy thread's own commits, likewise
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + P::NBAR);
  volatile int32_t* abort_flag = reinterpret_cast<volatile int32_t*>(tmem_slot + 1);
  float* sc_slots = reinterpret_cast<float*>(smem + P::OFF_SC);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // 256-wide K steps; the last may hold 1-3 of its four 64-wide scale tiles
  // (K % 64 == 0): only those are copied and multiplied
  const int nk = (p.K + 255) / 256;
  const int ktiles64 = p.K / 64;          // scale tiles per 128 rows
  const bool lr = P::LR && p.has_lr;
  const int nN = (p.N + BN - 1) / BN, nM = (p.M + BM - 1) / BM;
  const int ntiles = nM * nN;

  if (threadIdx.x == 0) {
    for (int i = 0; i < P::S; ++i) { mbar_init(&full[i], 1); mbar_init(&empty[i], 1); }
    for (int i = 0; i < 2; ++i) { mbar_init(&accfull[i], 1); mbar_init(&accempty[i], 8); }
    mbar_init(lrfull, 1);
    mbar_init(lrsmem_empty, 1);
    mbar_init(lrdone, 1);
    mbar_init(lracc_empty, 8);
    for (int i = 0; i < 4; ++i) { mbar_init(&sffull[i], 1); mbar_init(&sfempty[i], 1); }
    mbar_init(mdrain, 1);
    mbar_init(cdrain, 1);
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
  // launched as a programmatic dependent of the activation kernel: the
  // prologue above overlaps its tail; nothing it writes is read before this
  griddep_wait();
  constexpr uint32_t SF_COLS = 16 + 4 * (BN / 32);   // SFA 4 x 4 columns + SFB 4 x BN/32
  constexpr int SF_SLOTS = 4;

  if (warp == 0) {
    if (lane == 0) {
      uint32_t kc = 0;
      int tc = 0;
      int lr_issued = 0;
      for (int tile = blockIdx.x; tile < ntiles && !*abort_flag; tile += gridDim.x, ++tc) {
        const int m0 = (tile / nN) * BM, n0 = (tile % nN) * BN;
        const uint8_t* sfa_src = p.a_bscale + (size_t)(m0 / 128) * ktiles64 * 512;
        // weight scale tiles that exist (the last tile column may cover only 128 rows)
        const int nb_valid = min(BN / 128, (p.N + 127) / 128 - n0 / 128);
        for (int kt = 0; kt < nk; ++kt, ++kc) {
          const int s = kc % P::S;
          if (kc >= P::S && !mbar_wait(&empty[s], ((kc / P::S) - 1) & 1, p.status, ST_TIMEOUT_EMPTY, abort_flag, p.wait_ns)) break;
          uint8_t* st = smem + s * P::STAGE;
          const uint32_t sfb = (uint32_t)min(4, ktiles64 - kt * 4) * 512;   // scale bytes per 128 rows
          mbar_expect_tx(&full[s], P::PA + P::PB + sfb + nb_valid * sfb + (kc == 0 ? p.inject_tx : 0u));
          tma_load_2d(st, &tm.a, kt * 128, m0, &full[s]);
          tma_load_2d(st + P::PA, &tm.b, kt * 128, n0, &full[s]);
          // up to 4 scale chunks (k tiles of 64) x 512 B, contiguous in the K1 layout
          bulk_g2s(st + P::PA + P::PB, sfa_src + (size_t)kt * 4 * 512, sfb, &full[s]);
          for (int nb = 0; nb < nb_valid; ++nb)
            bulk_g2s(st + P::PA + P::PB + P::SA + nb * 2048,
                     p.w_bscale + ((size_t)(n0 / 128 + nb) * ktiles64 + (size_t)kt * 4) * 512, sfb, &full[s]);
        }
        if (lr) {   // after the K tiles (see the codebook kernel)
          if (tc > 0 && !mbar_wait(lrsmem_empty, (tc - 1) & 1, p.status, ST_TIMEOUT_EMPTY, abort_flag, p.wait_ns)) break;
          mbar_expect_tx(lrfull, BM * 64 + BN * 64);
          tma_load_2d(smem + P::OFF_C, &tm.c, 0, m0, lrfull);
          tma_load_2d(smem + P::OFF_L, &tm.l, 0, n0, lrfull);
          ++lr_issued;
        }
      }
      if (*abort_flag) {   // let the copies already issued land (bounded)
        for (uint32_t c = kc > (uint32_t)P::S ? kc - P::S : 0; c < kc; ++c)
          mbar_drain(&full[c % P::S], (c / P::S) & 1, p.wait_ns);
        if (lr_issued > 0) mbar_drain(lrfull, (lr_issued - 1) & 1, p.wait_ns);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      const uint32_t idesc = idesc_nvf4(BN);
      uint32_t kc = 0;
      int tc = 0;
      bool ok = true;
      for (int tile = blockIdx.x; tile < ntiles && ok; tile += gridDim.x, ++tc) {
        const uint32_t ab = tc % P::NACC;
        if (tc >= P::NACC) {
          ok = mbar_wait(&accempty[ab], ((tc / P::NACC) - 1) & 1, p.status, ST_TIMEOUT_EPI, abort_flag, p.wait_ns);
          if (!ok) break;
          tc_fence_after();
        }
        for (int kt = 0; kt < nk; ++kt, ++kc) {
          const int s = kc % P::S;
          const int sl = kc % SF_SLOTS;
          ok = mbar_wait(&full[s], (kc / P::S) & 1, p.status, ST_TIMEOUT_FULL, abort_flag, p.wait_ns) &&
               mbar_wait(&sffull[sl], (kc / SF_SLOTS) & 1, p.status, ST_TIMEOUT_FULL, abort_flag, p.wait_ns);
          if (!ok) break;
          tc_fence_after();
          const uint32_t st = sbase + s * P::STAGE;
          const uint32_t t_sfa = tmem + 256 + sl * SF_COLS, t_sfb = t_sfa + 16;
          const int kkn = min(4, ktiles64 - kt * 4);
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            if (kk < kkn)
              umma_nvf4(tmem + ab * BN, smem_desc(st + kk * 32, 16, 1024, 2), smem_desc(st + P::PA + kk * 32, 16, 1024, 2),
                      idesc, t_sfa + kk * 4, t_sfb + kk * (BN / 32), (kt > 0 || kk > 0) ? 1u : 0u);
          tc_commit(&empty[s]);
          tc_commit(&sfempty[sl]);
        }
        if (!ok) break;
        tc_commit(&accfull[ab]);
        if (lr) {
          // low-rank MMA after the K loop (see the codebook kernel)
          ok = mbar_wait(lrfull, tc & 1, p.status, ST_TIMEOUT_FULL, abort_flag, p.wait_ns) &&
               (tc == 0 || mbar_wait(lracc_empty, (tc - 1) & 1, p.status, ST_TIMEOUT_EPI, abort_flag, p.wait_ns));
          if (!ok) break;
          tc_fence_after();
          const uint32_t ca = sbase + P::OFF_C, la = sbase + P::OFF_L;
#pragma unroll
          for (int kk = 0; kk < 2; ++kk)
            umma_bf16(tmem + 384, smem_desc(ca + kk * 32, 16, 512, 4), smem_desc(la + kk * 32, 16, 512, 4),
                      idesc_bf16(BN), kk > 0);
          tc_commit(lrdone);
          tc_commit(lrsmem_empty);
        }
      }
      if (!ok) {   // wait (bounded) for the MMAs already issued
        tc_commit(mdrain);
        mbar_drain(mdrain, 0, p.wait_ns);
      }
    }
  } else if (warp == 2) {
    // ------------------------------------------------------------ scale factors -> TMEM
    // (UE4M3, per MMA one 512 B chunk per 128 rows) into a ring of SF_SLOTS
    // column groups, on their own issue stream so the copies overlap the MMAs
    if (lane == 0) {
      uint32_t kc = 0;
      bool ok = true;
      for (int tile = blockIdx.x; tile < ntiles && ok; tile += gridDim.x) {
        for (int kt = 0; kt < nk; ++kt, ++kc) {
          const int s = kc % P::S;
          const int sl = kc % SF_SLOTS;
          ok = (kc < (uint32_t)SF_SLOTS ||
                mbar_wait(&sfempty[sl], ((kc / SF_SLOTS) - 1) & 1, p.status, ST_TIMEOUT_EMPTY, abort_flag, p.wait_ns)) &&
               mbar_wait(&full[s], (kc / P::S) & 1, p.status, ST_TIMEOUT_FULL, abort_flag, p.wait_ns);
          if (!ok) break;
          tc_fence_after();
          const uint32_t sfa = sbase + s * P::STAGE + P::PA + P::PB, sfb = sfa + P::SA;
          const uint32_t t_a = tmem + 256 + sl * SF_COLS, t_b = t_a + 16;
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) {
            tc_cp_32x128b_warpx4(t_a + kk * 4, smem_desc(sfa + kk * 512, 16, 128, 0));
#pragma unroll
            for (int nb = 0; nb < BN / 128; ++nb)
              tc_cp_32x128b_warpx4(t_b + kk * (BN / 32) + nb * 4, smem_desc(sfb + nb * 2048 + kk * 512, 16, 128, 0));
          }
          tc_commit(&sffull[sl]);
        }
      }
      if (!ok) {   // wait (bounded) for the scale copies already issued
        tc_commit(cdrain);
        mbar_drain(cdrain, 0, p.wait_ns);
      }
    }
  } else if (warp >= 4) {
    const int q = warp & 3;                  // TMEM lane quadrant (warp id % 4)
    const int half = (warp - 4) >> 2;        // this warp's half of the columns
    const int tid = threadIdx.x - 128;       // 0 .. 255
    const uint32_t lane_off = (uint32_t)(q * 32) << 16;
    int tc = 0;
    bool ok = true;
    // the warps meet at a named barrier every tile: after an abort they keep
    // walking the tile loop (skipping the work), so every warp reaches it
    for (int tile = blockIdx.x; tile < ntiles; tile += gridDim.x, ++tc) {
      const int m0 = (tile / nN) * BM, n0 = (tile % nN) * BN;
      const int row = m0 + q * 32 + lane;
      const float sa = row < p.M ? __ldg(p.a_scale + row) : 0.f;
      const uint32_t ab = tc % P::NACC;
      float* sw = sc_slots + (tc & 1) * BN;
      load_scales_smem(sw, p.w_scale, n0, p.N, BN, tid, 256);
      epi_bar_n<256>();
      ok = ok && mbar_wait(&accfull[ab], (tc / P::NACC) & 1, p.status, ST_TIMEOUT_MMA, abort_flag, p.wait_ns) &&
           (!lr || mbar_wait(lrdone, tc & 1, p.status, ST_TIMEOUT_MMA, abort_flag, p.wait_ns));
      if (!ok) continue;
      tc_fence_after();
#pragma unroll 1
      for (int ch = half * (BN / 64); ch < (half + 1) * (BN / 64); ++ch)
        epi_chunk_final(p, tmem + lane_off + ab * BN + ch * 32, tmem + lane_off + 384 + ch * 32, lr, sw + ch * 32,
                        sa, row, n0 + ch * 32);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(&accempty[ab]);
        if (lr) mbar_arrive(lracc_empty);
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

// Every GEMM launch is a programmatic dependent launch (the kernels call
// griddep_wait() before touching their inputs), so its prologue overlaps the
// tail of the previous kernel on the stream, normally the activation kernel.
template <class Kern>
cudaError_t launch(Kern k, int smem, dim3 grid, int threads, const TMaps& tm, const GemmParams& gp, cudaStream_t st) {
  cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = dim3(threads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, k, tm, gp);
}

// CTA-pair kernels: clusters of two, as many pairs as can be resident at once
// (at most `pairs`).
template <class Kern>
cudaError_t launch_pair(Kern k, int smem, int pairs, int threads, const TMaps& tm, const GemmParams& gp,
                        cudaStream_t st) {
  cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(2 * pairs);
  cfg.blockDim = dim3(threads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cfg.attrs = attr;
  cfg.numAttrs = 1;   // the occupancy query below sees the cluster shape only
  // resident-pair counts per kernel, computed once (guarded: host threads may
  // launch concurrently)
  static std::mutex mu;
  static const void* cached_k[8] = {};
  static int cached_n[8] = {};
  int resident = 0;
  {
    std::lock_guard<std::mutex> lock(mu);
    for (int i = 0; i < 8; ++i)
      if (cached_k[i] == (const void*)k) resident = cached_n[i];
  }
  if (resident == 0) {
    e = cudaOccupancyMaxActiveClusters(&resident, k, &cfg);
    if (e != cudaSuccess) return e;
    if (resident < 1) return cudaErrorInvalidConfiguration;
    std::lock_guard<std::mutex> lock(mu);
    for (int i = 0; i < 8; ++i)
      if (!cached_k[i] || cached_k[i] == (const void*)k) {
        cached_k[i] = (const void*)k;
        cached_n[i] = resident;
        break;
      }
  }
  cfg.gridDim = dim3(2 * (pairs < resident ? pairs : resident));
  cfg.numAttrs = 2;
  return cudaLaunchKernelEx(&cfg, k, tm, gp);
}

}  // namespace

cudaError_t launch_gemm(const GemmLaunch& a, cudaStream_t st, const char** why) {
  TMaps tm;
  memset(&tm, 0, sizeof(tm));
  GemmParams gp{};
  gp.M = a.M; gp.N = a.N; gp.K = a.K;
  gp.nk128 = (a.K + 127) / 128;
  gp.a_fmt = a.a_fmt; gp.w_fmt = a.w_fmt;
  gp.a_scale = a.a_scale; gp.w_scale = a.w_scale;
  gp.a_bscale = a.a_bscale; gp.w_bscale = a.w_bscale;
  memcpy(gp.a_lut, a.a_lut, 16);
  memcpy(gp.w_lut, a.w_lut, 16);
  gp.has_lr = a.c != nullptr;
  gp.Y = a.Y; gp.out_fp32 = a.out_fp32; gp.status = a.status;
  gp.wait_ns = a.wait_ns; gp.inject_tx = a.inject_tx;
  gp.a_zp = a.a_zp; gp.w_zsum = a.w_zsum;
  gp.tma_store = 0;

  const bool nvf4 = a.a_fmt == RQ_FMT_NVFP4;
  const bool grouped = a.w_fmt == RQ_FMT_INT4;
  // 128 x 256 tiles unless the INT4 group epilogue or the low-rank branch needs the TMEM
  const int BN = (grouped || gp.has_lr) ? 128 : 256;
  bool ok = true;
  if (gp.has_lr) {
    ok &= make_map_2d(&tm.c, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, a.c, a.r, a.M, (uint64_t)a.r * 2, 32, BM,
                      CU_TENSOR_MAP_SWIZZLE_64B);
    ok &= make_map_2d(&tm.l, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, a.L, a.r, a.N, (uint64_t)a.r * 2, 32, BN,
                      CU_TENSOR_MAP_SWIZZLE_64B);
  }
  const int ntiles = ((a.M + BM - 1) / BM) * ((a.N + BN - 1) / BN);
  const int sms = a.num_sms > 0 ? a.num_sms : 148;
  dim3 grid(ntiles < sms ? ntiles : sms);
  if (nvf4) {
    ok &= make_map_2d(&tm.a, CU_TENSOR_MAP_DATA_TYPE_UINT8, a.a_codes, a.K / 2, a.M, a.K / 2, 128, BM,
                      CU_TENSOR_MAP_SWIZZLE_128B);
    ok &= make_map_2d(&tm.b, CU_TENSOR_MAP_DATA_TYPE_UINT8, a.w_codes, a.K / 2, a.N, a.K / 2, 128, BN,
                      CU_TENSOR_MAP_SWIZZLE_128B);
    if (!ok) { *why = "cuTensorMapEncodeTiled failed"; return cudaErrorInvalidValue; }
    if (BN == 256) return launch(gemm_nvf4_kernel<256>, Nvf4Plan<256>::BYTES, grid, NVF4_THREADS, tm, gp, st);
    return launch(gemm_nvf4_kernel<128>, Nvf4Plan<128>::BYTES, grid, NVF4_THREADS, tm, gp, st);
  }
  const bool w2 = a.w_fmt == RQ_FMT_LM4;
  if (!a.out_fp32 && a.N % 8 == 0) {   // (the map's row pitch must be a multiple of 16 bytes)
    // BF16 output through 32 x 32 boxes (the epilogue's TMA stores)
    ok &= make_map_2d(&tm.y, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, a.Y, a.N, a.M, (uint64_t)a.N * 2, 32, 32,
                      CU_TENSOR_MAP_SWIZZLE_64B);
    gp.tma_store = 1;
  }
  const bool a8 = a.a_fmt == RQ_FMT_INT8;
  if (a8)   // int8 activation codes: 128-byte rows of the K tile, the MMA's own swizzle
    ok &= make_map_2d(&tm.a, CU_TENSOR_MAP_DATA_TYPE_UINT8, a.a_codes, a.K, a.M, a.K, 128, BM,
                      CU_TENSOR_MAP_SWIZZLE_128B);
  else
    ok &= make_map_2d(&tm.a, CU_TENSOR_MAP_DATA_TYPE_UINT8, a.a_codes, a.K / 2, a.M, a.K / 2, 64, BM,
                      CU_TENSOR_MAP_SWIZZLE_64B);
  // codebook tiles run on CTA pairs, 256 x 512 per pair: each CTA loads and
  // expands its 128 token rows once per K step for 512 output columns, and
  // 128 rows of each 256-wide half of the tile's weight rows
  const bool pair = !grouped && BN == 256;
  const uint32_t brows = pair ? 128 : BN;
  if (w2)
    ok &= make_map_2d(&tm.b, CU_TENSOR_MAP_DATA_TYPE_UINT8, a.w_codes, a.K / 4, a.N, a.K / 4, 32, brows,
                      CU_TENSOR_MAP_SWIZZLE_32B);
  else
    ok &= make_map_2d(&tm.b, CU_TENSOR_MAP_DATA_TYPE_UINT8, a.w_codes, a.K / 2, a.N, a.K / 2, 64, brows,
                      CU_TENSOR_MAP_SWIZZLE_64B);
  if (!ok) { *why = "cuTensorMapEncodeTiled failed"; return cudaErrorInvalidValue; }
  if (grouped && a8)
    return launch(gemm_fp8_kernel<128, 4, true, false, true>, Fp8Plan<128, 4, false, true>::BYTES, grid,
                  fp8_threads<128, true>(), tm, gp, st);
  if (grouped) return launch(gemm_fp8_kernel<128, 4, true>, Fp8Plan<128, 4>::BYTES, grid, fp8_threads<128, true>(), tm, gp, st);
  if (pair) {
    const int ptiles = ((a.M + 2 * BM - 1) / (2 * BM)) * ((a.N + 511) / 512);
    const int pairs = ptiles < sms / 2 ? ptiles : sms / 2;
    if (w2)
      return launch_pair(gemm_fp8_kernel<512, 2, false, true>, Fp8Plan<512, 2, true>::BYTES, pairs,
                         fp8_threads<512, false>(), tm, gp, st);
    return launch_pair(gemm_fp8_kernel<512, 4, false, true>, Fp8Plan<512, 4, true>::BYTES, pairs,
                       fp8_threads<512, false>(), tm, gp, st);
  }
  if (w2) return launch(gemm_fp8_kernel<128, 2, false>, Fp8Plan<128, 2>::BYTES, grid, fp8_threads<128, false>(), tm, gp, st);
  return launch(gemm_fp8_kernel<128, 4, false>, Fp8Plan<128, 4>::BYTES, grid, fp8_threads<128, false>(), tm, gp, st);
}

}  // namespace rq
