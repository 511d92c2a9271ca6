// K1: fused rotate -> normalise -> quantize -> pack, one pass over each row,
// for rows with the DiRotQ low-rank projection (the other calls run in
// rq_k1r.cu unless its shared-memory plan does not fit).
//
// Implements the online activation transform of the rotated W4A4 linear layer
// (OrbitQuant abstract: randomized permuted block-Hadamard (RPBH) rotation,
// per-token normalisation, Lloyd-Max codes; TR-DQ section 3.1, Eq. 1-3: uniform
// grid with online min/max; DiRotQ abstract: NVFP4, PCA coefficients kept in
// BF16) and, on weight rows, the offline folding W' = W R^T followed by the same
// quantizers (OrbitQuant abstract; TR-DQ Eq. 9).
//
// Data flow per CTA (persistent over groups of R rows):
//   HBM --cp.async.bulk--> smem row buffer (mbarrier)
//   [projection: c = bf16(x U) from the BF16 rows, each of the R x 32 sums one
//    sequential FP32 chain per 128-channel chunk, the chunk sums added in
//    order; the rows are widened to FP32 in place and x_res = x - c U^T
//    (sequential over j) overwrites them]
//   a group of L = b/32 lanes owns one b-wide Hadamard block of one row: lane j
//   of the group holds the 32 consecutive rotated coordinates 32j .. 32j+31,
//   gathered from smem through the signed-permutation table; butterfly stages
//   h = 1..16 run in registers, h = 32..b/2 through __shfl_xor_sync (log2 L
//   stages); block partials (max|y|, pairwise sum of squares) -> smem
//   row scales computed once per row (sum of squares added block by block, in order)
//   quantize, pack 32 codes per lane, one 128-bit (64-bit for 2-bit codes) store.
//
// FP32 contract (bit-exact against the CPU oracle): every add/multiply/divide is
// an explicit round-to-nearest-even intrinsic (no contraction); the only fused
// multiply-adds are the projection's, whose products of two BF16 values are
// exact in FP32 so the fused and unfused results agree.
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>
#include <cstring>

#include "rq_internal.h"
#include "rq_ptx.cuh"

namespace rq {

namespace {

constexpr int K1_THREADS = 512;
constexpr int K1_LUT_MAX = 512;
constexpr int K1_ROW_PAD = 8;   // BF16 elements (16 bytes) after each staged row
constexpr int K1_WARPS = K1_THREADS / 32;

struct __align__(16) K1Params {
  const uint16_t* x;       // rows x K, BF16 bits
  const int32_t* rot;      // signed permutation: bits 0-30 source channel, bit 31 sign
  const uint16_t* U;       // K x r BF16 (projection) or null
  uint16_t* coef;          // rows x r BF16 output (c or L) or null
  uint8_t* codes;          // packed codes
  float* scale;            // act: [rows]; weight INT4: [K/128][rows]; else [rows]
  uint8_t* bscale;         // NVFP4 block scales, 128x4 swizzled tiles
  int32_t* status;
  int32_t rows, K, r;
  int32_t R;               // rows per group
  int32_t ngroups;
  float inv_sqrt_b;        // fp32(1/sqrt(block))
  float sqrtK;             // fp32(sqrt(K))
  int32_t nbnd;            // number of codebook boundaries (levels - 1)
  float bnd[15];
  // codebook search table: u * 2^lut_shift, clamped to [lut_gmin, lut_gmin +
  // lut_n - 1] and floored, indexes cells of width 2^-lut_shift holding at most
  // one boundary each: code = lut[g].x + (u >= lut[g].y as float)
  int32_t lut_shift, lut_gmin, lut_n;
  uint2 lut[K1_LUT_MAX];
  float rcp_e4m3[128];     // fp32(1 / e4m3 value) for the positive e4m3 codes, 0 for code 0
  uint64_t wait_ns;        // limit of every bounded wait
  uint32_t inject_tx;      // test hook: extra expect-tx bytes on the CTA's first row group
};


// Swizzled NVFP4 block-scale offset: 128-row x 4-scale tiles of 512 bytes,
// tiles ordered [row tile][k tile]; inside: (m%32)*16 + ((m%128)/32)*4 + kb%4.
__device__ __forceinline__ size_t sf_offset(int m, int kb, int K) {
  const int tiles_k = K / 64;
  return ((size_t)(m >> 7) * tiles_k + (kb >> 2)) * 512 + (m & 31) * 16 + ((m >> 5) & 3) * 4 + (kb & 3);
}

// acc + a * b for BF16 a, b (half AH of word a, half BH of word b; 0 = low
// 16 bits), FP32 acc, one rounding: the product of two BF16 values is exact.
template <int AH, int BH>
__device__ __forceinline__ float fma_bf16(uint32_t a, uint32_t b, float acc) {
  float d;
  asm("{\n\t.reg .b16 a0, a1, b0, b1;\n\t"
      "mov.b32 {a0, a1}, %1;\n\t"
      "mov.b32 {b0, b1}, %2;\n\t"
      "fma.rn.f32.bf16 %0, a%4, b%5, %3;\n\t}"
      : "=f"(d)
      : "r"(a), "r"(b), "f"(acc), "n"(AH), "n"(BH));
  return d;
}

// Packed FP32 pairs (sm_100 f32x2 arithmetic): each lane rounds exactly like
// the scalar instruction, two elements per issue slot.
__device__ __forceinline__ uint64_t pack2(float a, float b) {
  uint64_t r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(a), "f"(b));
  return r;
}
// (a, b) -> (a + b, a - b) for the element pairs (a0, b0) and (a1, b1)
__device__ __forceinline__ void bfly2(float& a0, float& a1, float& b0, float& b1) {
  asm("{\n\t.reg .b64 a, b, s, d;\n\t"
      "mov.b64 a, {%0, %1};\n\tmov.b64 b, {%2, %3};\n\t"
      "add.rn.f32x2 s, a, b;\n\tsub.rn.f32x2 d, a, b;\n\t"
      "mov.b64 {%0, %1}, s;\n\tmov.b64 {%2, %3}, d;\n\t}"
      : "+f"(a0), "+f"(a1), "+f"(b0), "+f"(b1));
}
// v = s * v + o on two elements, s a packed pair
__device__ __forceinline__ void fma2(float& v0, float& v1, uint64_t s2, float o0, float o1) {
  asm("{\n\t.reg .b64 v, o;\n\t"
      "mov.b64 v, {%0, %1};\n\tmov.b64 o, {%3, %4};\n\t"
      "fma.rn.f32x2 v, %2, v, o;\n\tmov.b64 {%0, %1}, v;\n\t}"
      : "+f"(v0), "+f"(v1) : "l"(s2), "f"(o0), "f"(o1));
}
// acc (two FP32 in one 64-bit register) = (c, c) * u2 + acc: one IEEE FMA per
// element, c broadcast, u2 two packed FP32 values
__device__ __forceinline__ void fma2_bcast(uint64_t& acc, float c, uint64_t u2) {
  asm("{\n\t.reg .b64 cc;\n\tmov.b64 cc, {%1, %1};\n\tfma.rn.f32x2 %0, cc, %2, %0;\n\t}"
      : "+l"(acc)
      : "f"(c), "l"(u2));
}
// the two BF16 halves of a word, widened to FP32 and packed (low half first)
__device__ __forceinline__ uint64_t widen2(uint32_t w) {
  uint64_t r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "r"(w << 16), "r"(w & 0xFFFF0000u));
  return r;
}
// v = v * s on two elements, s a packed pair
__device__ __forceinline__ void mul2(float& v0, float& v1, uint64_t s2) {
  asm("{\n\t.reg .b64 v;\n\tmov.b64 v, {%0, %1};\n\tmul.rn.f32x2 v, v, %2;\n\tmov.b64 {%0, %1}, v;\n\t}"
      : "+f"(v0), "+f"(v1) : "l"(s2));
}
// round to the nearest integer, ties to even, for |x| < 2^22 (full-rate FP32
// add in place of a conversion)
__device__ __forceinline__ int rint_small(float x) {
  return __float_as_int(__fadd_rn(x, 12582912.0f)) - 0x4B400000;
}

// Projection layout in shared memory: U^T as BF16 rows of KP = K + 8 entries
// (the 16-byte pad spreads the 32 rows over all banks).
__host__ __device__ constexpr int ut_pitch(int K) { return K + 8; }


template <int L, int FMT, bool PROJ, bool WEIGHT, int IPW>
__global__ void __launch_bounds__(K1_THREADS, IPW == 1 ? 2 : 1) k1_rotate_quantize(const __grid_constant__ K1Params p) {
  constexpr int B = L * 32;                // Hadamard block
  constexpr int GPW = 32 / L;              // lane groups (block slots) per warp
  constexpr int SLOTS = K1_WARPS * GPW;    // block slots per CTA pass
  constexpr bool RESID = PROJ && !WEIGHT;  // activations: rotate the residual
  extern __shared__ __align__(128) uint8_t smem[];
  const int K = p.K;
  const int R = p.R;
  const int nblk = K / B;
  const int KS = PROJ ? K : K + K1_ROW_PAD;   // row stride of the BF16 row buffers
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int lq = lane % L;                 // lane inside its group
  const int slot0 = warp * GPW + lane / L; // first block slot of this lane group
  // shuffles stay inside the lane group (groups of one warp may take different branches)
  const unsigned gmask = L == 32 ? 0xffffffffu : (((1u << L) - 1u) << (lane & ~(L - 1)));

  // smem layout
  //   without projection: [2][R][K] bf16 row buffers (the next group streams in
  //   while this one is transformed)
  //   with projection: [R][K] fp32 rows (the bf16 rows land in its upper half
  //   and are widened in place) | [32][K+8] bf16 U^T | [R][32] fp32 -c
  //   then [K] int32 signed permutation | [2][R][nblk] fp32 block sum-of-squares |
  //   [2][R][ngrp] u32 amax bits | mbarriers | abort flag | boundaries |
  //   [128] fp32 e4m3 reciprocals | [lut_n] codebook search cells
  uint16_t* xs = reinterpret_cast<uint16_t*>(smem);
  float* xf = reinterpret_cast<float*>(smem);
  uint16_t* land = reinterpret_cast<uint16_t*>(smem + (PROJ ? (size_t)R * K * 2 : 0));
  size_t off;
  uint16_t* ut = nullptr;
  float* negc = nullptr;
  int32_t* rot_s = nullptr;
  if constexpr (PROJ) {
    off = (size_t)R * K * 4;
    ut = reinterpret_cast<uint16_t*>(smem + off);
    off += (size_t)32 * ut_pitch(K) * 2;
    negc = reinterpret_cast<float*>(smem + off);
    off += (size_t)R * 32 * 4;
  } else {
    off = (size_t)2 * R * (K + K1_ROW_PAD) * 2;
  }
  rot_s = reinterpret_cast<int32_t*>(smem + off);
  off += (size_t)K * 4;
  // block partials, double-buffered by group parity so that no barrier is
  // needed between a group's quantization and the next group's reductions
  float* part_ss2 = reinterpret_cast<float*>(smem + off);
  off += (size_t)2 * R * nblk * 4;
  const int ngrp = (WEIGHT && FMT == RQ_FMT_INT4) ? K / 128 : 1;
  uint32_t* amax_bits2 = reinterpret_cast<uint32_t*>(smem + off);
  off += (size_t)2 * R * ngrp * 4;
  off = (off + 15) & ~(size_t)15;
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + off);
  volatile int32_t* abort_flag = reinterpret_cast<volatile int32_t*>(smem + off + 16);
  float* rcp_s = reinterpret_cast<float*>(smem + off + 96);
  uint2* lut_s = reinterpret_cast<uint2*>(smem + off + 96 + 512);
  if constexpr (FMT == RQ_FMT_NVFP4)
    for (int i = threadIdx.x; i < 128; i += K1_THREADS) rcp_s[i] = p.rcp_e4m3[i];
  if constexpr (FMT == RQ_FMT_LM16 || FMT == RQ_FMT_LM4)
    for (int i = threadIdx.x; i < p.lut_n; i += K1_THREADS) lut_s[i] = p.lut[i];

  const uint32_t row_bytes = (uint32_t)K * 2;

  if (threadIdx.x == 0) {
    mbar_init(&full[0], 1);
    mbar_init(&full[1], 1);
    *abort_flag = 0;
    fence_mbar_init();
    // the GEMM that consumes these codes may be scheduled now: its CTAs only
    // take SMs this persistent grid leaves free, and it waits for this grid's
    // completion before reading anything it writes
    griddep_launch_dependents();
  }
  __syncthreads();

  auto issue_group = [&](int g, int buf) {
    const int r0 = g * R;
    const int nr = min(R, p.rows - r0);
    uint16_t* dst = PROJ ? land : xs + (size_t)buf * R * KS;
    // (the test hook overstates the first group's byte count: every row still
    // lands, the wait for it runs out)
    mbar_expect_tx(&full[buf], (uint32_t)nr * row_bytes + (g == (int)blockIdx.x ? p.inject_tx : 0u));
    for (int i = 0; i < nr; ++i) bulk_g2s(dst + (size_t)i * KS, p.x + (size_t)(r0 + i) * K, row_bytes, &full[buf]);
  };

  if (threadIdx.x == 0 && blockIdx.x < p.ngroups) issue_group(blockIdx.x, 0);

  if constexpr (PROJ) {
    // stage U^T (row j holds U[0..K-1][j]) and the signed permutation once per
    // CTA, while the first rows stream in.  A rank below 32 is padded with zero
    // columns: their coefficients are 0 and their products in the residual are
    // zeros, so every chain's result is that of the first r terms.
    const int KP = ut_pitch(K);
    const int rq8 = p.r / 8;   // 16-byte words per row of U
    for (int t = threadIdx.x; t < K * 4; t += K1_THREADS) {
      const int k = t >> 2, q = t & 3;
      const uint4 w4 = q < rq8 ? __ldg(reinterpret_cast<const uint4*>(p.U + (size_t)k * p.r) + q) : make_uint4(0, 0, 0, 0);
      const uint32_t ww[4] = {w4.x, w4.y, w4.z, w4.w};
#pragma unroll
      for (int h = 0; h < 4; ++h) {
        ut[(size_t)(8 * q + 2 * h) * KP + k] = (uint16_t)(ww[h] & 0xFFFFu);
        ut[(size_t)(8 * q + 2 * h + 1) * KP + k] = (uint16_t)(ww[h] >> 16);
      }
    }
  }
  // the signed permutation, interleaved per block so that the lanes of a group
  // read consecutive 16-byte words: entry e of lane lq in block bk (rotated
  // coordinate bk*B + 32*lq + e) sits at bk*B + (e/4)*4L + 4*lq + e%4
  for (int t = threadIdx.x; t < K / 4; t += K1_THREADS) {
    const int i = 4 * t, bk = i / B, w = i % B, l = w >> 5, e = w & 31;
    reinterpret_cast<int4*>(rot_s)[(bk * B + (e >> 2) * 4 * L + 4 * l) >> 2] =
        __ldg(reinterpret_cast<const int4*>(p.rot) + t);
  }

  for (int i = threadIdx.x; i < 2 * R * ngrp; i += K1_THREADS) amax_bits2[i] = 0u;
  int it = 0;
  for (int g = blockIdx.x; g < p.ngroups; g += gridDim.x, ++it) {
    const int buf = PROJ ? 0 : (it & 1);
    const int r0 = g * R;
    const int nr = min(R, p.rows - r0);
    const bool has_next = g + (int)gridDim.x < p.ngroups;
    float* part_ss = part_ss2 + (size_t)(it & 1) * R * nblk;
    uint32_t* amax_bits = amax_bits2 + (size_t)(it & 1) * R * ngrp;
    const uint32_t par = PROJ ? (it & 1) : ((it >> 1) & 1);
    mbar_wait(&full[buf], par, p.status, ST_TIMEOUT_LOAD, abort_flag, p.wait_ns);
    // everyone has finished the previous group past this barrier
    __syncthreads();
    if (*abort_flag) {
      // the rows of this group were the only copies in flight: let them land
      // (bounded) before the CTA's shared memory goes away
      if (threadIdx.x == 0) mbar_drain(&full[buf], par, p.wait_ns);
      break;
    }
    if constexpr (!PROJ) {
      // prefetch the next group into the other buffer (last read by the
      // previous group's gather)
      if (threadIdx.x == 0 && has_next) {
        fence_proxy_async_smem();
        issue_group(g + gridDim.x, buf ^ 1);
      }
    }
    const uint16_t* xg = xs + (size_t)buf * R * KS;

    if constexpr (PROJ) {
      // ---------------------------------------------------------- coefficients
      // c[row][j] = bf16(sum_k x[row][k] U[k][j]) with the sum cut into
      // 128-wide chunks of k: inside a chunk one sequential FP32 chain in k
      // order, read straight from the BF16 rows as they landed; the chunk sums
      // are then added in chunk order.  fma.rn.f32.bf16 rounds the exact product
      // plus the running sum once, like an add of the (exact) product.  Lane j
      // takes column j; a warp takes units of four rows of one chunk (four
      // independent chains sharing each U^T load).  The chunk sums go to the
      // lower half of the FP32 row buffer, unused until the rows are widened.
      {
        const int nch = K / 128;
        const int RG = (nr + 3) >> 2;
        float* cpart = xf;   // [nr][nch][32]
        for (int gi = warp; gi < RG * nch; gi += K1_WARPS) {
          const int t = gi / RG, rb = (gi - t * RG) * 4;
          const uint4* uj = reinterpret_cast<const uint4*>(ut + (size_t)lane * ut_pitch(K) + t * 128);
          const uint4* xr[4];
#pragma unroll
          for (int i = 0; i < 4; ++i)
            xr[i] = reinterpret_cast<const uint4*>(land + (size_t)min(rb + i, nr - 1) * K + t * 128);
          float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll 4
          for (int k8 = 0; k8 < 16; ++k8) {
            const uint4 u = uj[k8];
#pragma unroll
            for (int i = 0; i < 4; ++i) {
              const uint4 a = xr[i][k8];
              acc[i] = fma_bf16<0, 0>(a.x, u.x, acc[i]);
              acc[i] = fma_bf16<1, 1>(a.x, u.x, acc[i]);
              acc[i] = fma_bf16<0, 0>(a.y, u.y, acc[i]);
              acc[i] = fma_bf16<1, 1>(a.y, u.y, acc[i]);
              acc[i] = fma_bf16<0, 0>(a.z, u.z, acc[i]);
              acc[i] = fma_bf16<1, 1>(a.z, u.z, acc[i]);
              acc[i] = fma_bf16<0, 0>(a.w, u.w, acc[i]);
              acc[i] = fma_bf16<1, 1>(a.w, u.w, acc[i]);
            }
          }
#pragma unroll
          for (int i = 0; i < 4; ++i)
            if (rb + i < nr) cpart[((size_t)(rb + i) * nch + t) * 32 + lane] = acc[i];
        }
        __syncthreads();
        for (int idx = threadIdx.x; idx < nr * 32; idx += K1_THREADS) {
          const int row = idx >> 5, j = idx & 31;
          const float* cp = cpart + (size_t)row * nch * 32 + j;
          float s = cp[0];
          for (int t = 1; t < nch; ++t) s = __fadd_rn(s, cp[t * 32]);
          const uint16_t h = __bfloat16_as_ushort(__float2bfloat16_rn(s));
          if (j < p.r) p.coef[(size_t)(r0 + row) * p.r + j] = h;
          negc[row * 32 + j] = -bf16_bits_to_f32(h);
        }
      }
      __syncthreads();

      // ---------------------------------------------------------- widen
      // BF16 -> FP32 in place (exact).  A stage converts the rows [u, v) whose
      // FP32 targets end before landing row u; the last row overlaps its own
      // landing row and goes through registers.
      {
        const uint32_t* land32 = reinterpret_cast<const uint32_t*>(land);
        int u = 0;
        while (u < nr) {
          const int v = min(nr, (R + u) >> 1);
          if (v > u) {
            for (int t = threadIdx.x; t < (v - u) * K / 2; t += K1_THREADS) {
              const uint32_t w2 = land32[(size_t)u * K / 2 + t];
              reinterpret_cast<float2*>(xf)[(size_t)u * K / 2 + t] =
                  make_float2(__uint_as_float(w2 << 16), __uint_as_float(w2 & 0xFFFF0000u));
            }
            u = v;
          } else {
            uint32_t w[4];   // K <= 3072: at most three words per thread
#pragma unroll
            for (int i = 0; i < 4; ++i) {
              const int t = threadIdx.x + i * K1_THREADS;
              if (t < K / 2) w[i] = land32[(size_t)u * K / 2 + t];
            }
            __syncthreads();
#pragma unroll
            for (int i = 0; i < 4; ++i) {
              const int t = threadIdx.x + i * K1_THREADS;
              if (t < K / 2)
                reinterpret_cast<float2*>(xf)[(size_t)u * K / 2 + t] =
                    make_float2(__uint_as_float(w[i] << 16), __uint_as_float(w[i] & 0xFFFF0000u));
            }
            u = u + 1;
          }
          __syncthreads();
        }
      }

      // ---------------------------------------------------------- residual
      if constexpr (RESID) {
        // x - sum_j c_j U[k, j] in place, subtracted in order j = 0..31.  Work
        // unit = (k pair, one of eight row sets): U[k..k+1][0..31] is widened
        // once per unit and each broadcast -c load serves both k; the units of
        // a warp share the row set (K % 64 == 0).  4K units: the same count for
        // every thread.
        const int KP = ut_pitch(K);
        const int RU = (nr + 7) >> 3;
        const int KH = K / 2;
        for (int uu = threadIdx.x; uu < 8 * KH; uu += K1_THREADS) {
          const int set = uu / KH, k = 2 * (uu - set * KH);
          const int ra = set * RU, rb = min(nr, ra + RU);
          if (ra >= rb) continue;
          // j outermost in blocks of four, the unit's rows (at most four) inner:
          // every (row, k) chain still runs j = 0..31 in order.  The next
          // block's U^T words and -c vectors are loaded one block ahead.
          const int n = rb - ra;
          const float4* c4[4];
          uint64_t vab[4];   // (x[k], x[k+1]) of each row, packed: both chains in one FMA
#pragma unroll
          for (int r = 0; r < 4; ++r) {
            const int rr = ra + (r < n ? r : 0);
            c4[r] = reinterpret_cast<const float4*>(negc + rr * 32);
            vab[r] = *reinterpret_cast<const uint64_t*>(xf + (size_t)rr * K + k);
          }
          const uint16_t* uk = ut + k;
          uint32_t wn[4];
          float4 cn[4];
#pragma unroll
          for (int i = 0; i < 4; ++i) wn[i] = *reinterpret_cast<const uint32_t*>(uk + (size_t)i * KP);
#pragma unroll
          for (int r = 0; r < 4; ++r) cn[r] = c4[r][0];
#pragma unroll
          for (int q = 0; q < 8; ++q) {
            uint64_t u2[4];   // (U[k][j], U[k+1][j]) for the four j of this block
            float4 cc[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) u2[i] = widen2(wn[i]);
#pragma unroll
            for (int r = 0; r < 4; ++r) cc[r] = cn[r];
            if (q < 7) {
#pragma unroll
              for (int i = 0; i < 4; ++i) wn[i] = *reinterpret_cast<const uint32_t*>(uk + (size_t)(4 * q + 4 + i) * KP);
#pragma unroll
              for (int r = 0; r < 4; ++r) cn[r] = c4[r][q + 1];
            }
#pragma unroll
            for (int r = 0; r < 4; ++r) {   // exact products; j in order per chain
              fma2_bcast(vab[r], cc[r].x, u2[0]);
              fma2_bcast(vab[r], cc[r].y, u2[1]);
              fma2_bcast(vab[r], cc[r].z, u2[2]);
              fma2_bcast(vab[r], cc[r].w, u2[3]);
            }
          }
          // rows past the set's end computed a copy of its first row: not stored
#pragma unroll
          for (int r = 0; r < 4; ++r)
            if (r < n) *reinterpret_cast<uint64_t*>(xf + (size_t)(ra + r) * K + k) = vab[r];
        }
        __syncthreads();
      }
    }

    // Items (row, block): without the projection rows vary fastest, so the lane
    // groups of a warp gather the same columns of consecutive rows, whose
    // padded buffers (row stride K + 8) put them on different banks.
    auto item_row = [&](int item) { return PROJ ? item / nblk : item % nr; };
    auto item_blk = [&](int item) { return PROJ ? item % nblk : item / nr; };
    // ------------------------------------------------------------ phase A
    // gather, transform, block partials; y stays in registers until phase B
    const int nitems = nr * nblk;
    float y[IPW][32];
    float red[IPW];   // the lane's block partial per item
    // with two items the partials go out after both items' loads were issued
    // (a shared store before them would order the second item's gathers behind it)
    auto publish = [&](int ri, int bk, float val) {
      if constexpr (FMT == RQ_FMT_LM16 || FMT == RQ_FMT_LM4) {
        if (lq == 0) part_ss[ri * nblk + bk] = val;
      } else if constexpr (WEIGHT && FMT == RQ_FMT_INT4) {
        if ((lq & 3) == 0) atomicMax(&amax_bits[ri * ngrp + (bk * B + lq * 32) / 128], __float_as_uint(val));
      } else {
        if (lq == 0) atomicMax(&amax_bits[ri], __float_as_uint(val));
      }
    };
#pragma unroll
    for (int s = 0; s < IPW; ++s) {
      const int item = slot0 + s * SLOTS;
      if (item < nitems) {
        const int ri = item_row(item), bk = item_blk(item);
        float* v = y[s];
        const int4* rp = reinterpret_cast<const int4*>(rot_s + bk * B + 4 * lq);
#pragma unroll
        for (int e4 = 0; e4 < 8; ++e4) {
          const int4 rv = rp[e4 * L];
          const int rr[4] = {rv.x, rv.y, rv.z, rv.w};
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            const int src = rr[q] & 0x7fffffff;
            float xv;
            if constexpr (PROJ) xv = xf[(size_t)ri * K + src];
            else xv = bf16_bits_to_f32(xg[(size_t)ri * KS + src]);
            v[4 * e4 + q] = __uint_as_float(__float_as_uint(xv) ^ ((uint32_t)rr[q] & 0x80000000u));
          }
        }
        // butterflies inside the lane: stride h pairs (e, e+h) with bit h of e
        // clear; from h = 2 on, the butterflies of e and e+1 share a packed op
#pragma unroll
        for (int e = 0; e < 32; e += 2) {
          const float a = v[e], b = v[e + 1];
          v[e] = __fadd_rn(a, b);
          v[e + 1] = __fsub_rn(a, b);
        }
#pragma unroll
        for (int h = 2; h < 32; h <<= 1) {
#pragma unroll
          for (int e = 0; e < 32; e += 2)
            if ((e & h) == 0) bfly2(v[e], v[e + 1], v[e + h], v[e + h + 1]);
        }
        // butterflies across the L lanes of the group: stride 32m pairs lane j
        // (bit m clear) with lane j^m; one exact FFMA per element: lower lane
        // v + o, upper lane o - v (+-1 * v is exact)
#pragma unroll
        for (int m = 1; m < L; m <<= 1) {
          const float sgn = (lq & m) ? -1.0f : 1.0f;
          const uint64_t sgn2 = pack2(sgn, sgn);
#pragma unroll
          for (int e = 0; e < 32; e += 2) {
            const float o0 = __shfl_xor_sync(gmask, v[e], m), o1 = __shfl_xor_sync(gmask, v[e + 1], m);
            fma2(v[e], v[e + 1], sgn2, o0, o1);
          }
        }
        float amax = 0.f;
        const uint64_t isb2 = pack2(p.inv_sqrt_b, p.inv_sqrt_b);
#pragma unroll
        for (int e = 0; e < 32; e += 2) {
          mul2(v[e], v[e + 1], isb2);
          amax = fmaxf(amax, fmaxf(fabsf(v[e]), fabsf(v[e + 1])));
        }
        if constexpr (FMT == RQ_FMT_LM16 || FMT == RQ_FMT_LM4) {
          // perfect pairwise tree: five in-lane levels, then lanes by xor 1, 2, ..
          float sq[32];
#pragma unroll
          for (int e = 0; e < 32; ++e) sq[e] = __fmul_rn(v[e], v[e]);
#pragma unroll
          for (int w = 1; w < 32; w <<= 1) {
#pragma unroll
            for (int e = 0; e < 32; e += 2 * w) sq[e] = __fadd_rn(sq[e], sq[e + w]);
          }
          float ss = sq[0];
#pragma unroll
          for (int m = 1; m < L; m <<= 1) ss = __fadd_rn(ss, __shfl_xor_sync(gmask, ss, m));
          red[s] = ss;
          if constexpr (IPW == 1) publish(ri, bk, ss);
        } else if constexpr (WEIGHT && FMT == RQ_FMT_INT4) {
          // one scale per 128 rotated coordinates = 4 lanes
#pragma unroll
          for (int m = 1; m < (L < 4 ? L : 4); m <<= 1) amax = fmaxf(amax, __shfl_xor_sync(gmask, amax, m));
          red[s] = amax;
          if constexpr (IPW == 1) publish(ri, bk, amax);
        } else {
#pragma unroll
          for (int m = 1; m < L; m <<= 1) amax = fmaxf(amax, __shfl_xor_sync(gmask, amax, m));
          red[s] = amax;
          if constexpr (IPW == 1) publish(ri, bk, amax);
        }
      }
    }
    if constexpr (IPW > 1) {
#pragma unroll
      for (int s = 0; s < IPW; ++s) {
        const int item = slot0 + s * SLOTS;
        if (item < nitems) publish(item_row(item), item_blk(item), red[s]);
      }
    }
    __syncthreads();
    if constexpr (PROJ) {
      // the row buffer is free: stream the next group in behind the quantization
      if (threadIdx.x == 0 && has_next) {
        fence_proxy_async_smem();
        issue_group(g + gridDim.x, 0);
      }
    }
    // the other parity's amax words are free again (the previous group's
    // quantization finished before the barrier above)
    for (int i = threadIdx.x; i < R * ngrp; i += K1_THREADS) amax_bits2[(size_t)((it & 1) ^ 1) * R * ngrp + i] = 0u;

    // ------------------------------------------------------------ phase B
#pragma unroll
    for (int s = 0; s < IPW; ++s) {
      const int item = slot0 + s * SLOTS;
      if (item < nitems) {
        const int ri = item_row(item), bk = item_blk(item);
        const int row = r0 + ri;
        const int i0 = bk * B + lq * 32;
        float* v = y[s];
        uint32_t pk[4] = {0u, 0u, 0u, 0u};   // 32 codes, nibble e at bits 4(e%8) of word e/8
        // row (or group) scale, derived by every lane from the block partials;
        // the first lane of the row's (group's) first block writes it out
        float mlt;
        if constexpr (FMT == RQ_FMT_INT4) {
          const float amax = __uint_as_float(amax_bits[ri * ngrp + (WEIGHT ? i0 / 128 : 0)]);
          mlt = amax > 0.f ? __fdiv_rn(7.0f, amax) : 0.f;
          if (WEIGHT ? (i0 % 128 == 0) : (bk == 0 && lq == 0)) {
            const float sc = amax > 0.f ? __fdiv_rn(amax, 7.0f) : 0.f;
            if constexpr (WEIGHT) p.scale[(size_t)(i0 / 128) * p.rows + row] = sc;
            else p.scale[row] = sc;
          }
        } else if constexpr (FMT == RQ_FMT_LM16 || FMT == RQ_FMT_LM4) {
          // the row's sum of squares, block by block in order: the group's
          // first lane adds, the others take its result
          float ss = 0.f;
          if (lq == 0) {
            ss = part_ss[ri * nblk];
            for (int j = 1; j < nblk; ++j) ss = __fadd_rn(ss, part_ss[ri * nblk + j]);
          }
          ss = __shfl_sync(gmask, ss, lane & ~(L - 1));
          const float nrm = __fsqrt_rn(ss);
          mlt = nrm > 0.f ? __fdiv_rn(p.sqrtK, nrm) : 0.f;
          if (bk == 0 && lq == 0) p.scale[row] = nrm > 0.f ? __fdiv_rn(nrm, p.sqrtK) : 0.f;
        } else {
          const float amax = __uint_as_float(amax_bits[ri]);
          mlt = amax > 0.f ? __fdiv_rn(2688.0f, amax) : 0.f;
          if (bk == 0 && lq == 0) p.scale[row] = amax > 0.f ? __fdiv_rn(amax, 2688.0f) : 0.f;
        }
        if constexpr (FMT == RQ_FMT_INT4) {
          const float inv = mlt;
#pragma unroll
          for (int e = 0; e < 32; ++e) {
            int q = rint_small(__fmul_rn(v[e], inv));   // |v * inv| <= 7 (+ rounding)
            q = max(-7, min(7, q));
            pk[e >> 3] |= ((uint32_t)q & 0xFu) << (4 * (e & 7));
          }
        } else if constexpr (FMT == RQ_FMT_LM16 || FMT == RQ_FMT_LM4) {
          // code = number of boundaries <= u, read from the cell of u: its
          // base count plus one compare against the cell's boundary (if any);
          // 16-level codes are stored sign-magnitude (c - 8 above the centre,
          // (7 - c) | 8 below), both candidates held in the cell
          const float inv = mlt;
          const float cscale = __int_as_float((127 + p.lut_shift) << 23);   // 2^lut_shift
          const float tlo = (float)p.lut_gmin, thi = (float)(p.lut_gmin + p.lut_n - 1) + 0.5f;
          const int gbias = 0x4B400000 + p.lut_gmin;
#pragma unroll
          for (int e = 0; e < 32; ++e) {
            const float u = __fmul_rn(v[e], inv);
            const float t = fminf(fmaxf(__fmul_rn(u, cscale), tlo), thi);   // exact scaling
            const int g = __float_as_int(__fadd_rd(t, 12582912.0f)) - gbias;  // floor(t) - gmin
            const uint2 cell = lut_s[g];
            const bool up = u >= __uint_as_float(cell.y);
            if constexpr (FMT == RQ_FMT_LM16) {
              const uint32_t d = (cell.x >> (up ? 8 : 0)) & 0xFu;
              pk[e >> 3] |= d << (4 * (e & 7));
            } else {
              const uint32_t c = cell.x + (up ? 1u : 0u);
              pk[e >> 4] |= c << (4 * (e & 7) + 2 * ((e >> 3) & 1));   // nibble e%8: elements e%8, e%8+8
            }
          }
        } else {  // NVFP4: two 16-element groups per lane
          const float inv_t = mlt;
          uint16_t sbs = 0;
#pragma unroll
          for (int gq = 0; gq < 2; ++gq) {
            float* u = v + 16 * gq;   // scaled in place
            float m16 = 0.f;
            const uint64_t it2 = pack2(inv_t, inv_t);
#pragma unroll
            for (int e = 0; e < 16; e += 2) {
              mul2(u[e], u[e + 1], it2);
              m16 = fmaxf(m16, fmaxf(fabsf(u[e]), fabsf(u[e + 1])));
            }
            const float sbf = __fdiv_rn(m16, 6.0f);
            const uint8_t sb = (uint8_t)(cvt_e4m3x2(0.f, sbf) & 0xFF);
            const float rcp = rcp_s[sb & 0x7F];   // 1 / e4m3 value, 0 for code 0
#pragma unroll
            for (int e = 0; e < 16; e += 2) {
              const uint32_t byte = sb ? (uint32_t)cvt_e2m1x2(__fmul_rn(u[e + 1], rcp), __fmul_rn(u[e], rcp)) : 0u;
              const int ee = 16 * gq + e;
              pk[ee >> 3] |= byte << (4 * (ee & 7));
            }
            sbs |= (uint16_t)sb << (8 * gq);
          }
          // block scales kb, kb+1 (kb even) are adjacent bytes of the tile layout
          *reinterpret_cast<uint16_t*>(p.bscale + sf_offset(row, i0 / 16, K)) = sbs;
        }
        if constexpr (FMT == RQ_FMT_LM4) {
          *reinterpret_cast<uint2*>(p.codes + (size_t)row * (K / 4) + i0 / 4) = make_uint2(pk[0], pk[1]);
        } else {
          *reinterpret_cast<uint4*>(p.codes + (size_t)row * (K / 2) + i0 / 2) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
        }
      }
    }
  }
}


size_t k1_smem_bytes(int R, int K, int nblk, bool proj, int ngrp, int lut_n) {
  size_t off = proj ? (size_t)R * K * 4 + (size_t)32 * ut_pitch(K) * 2 + (size_t)R * 32 * 4
                    : (size_t)2 * R * (K + K1_ROW_PAD) * 2;
  off += (size_t)K * 4;
  off += (size_t)2 * R * nblk * 4;
  off += (size_t)2 * R * ngrp * 4;
  off = (off + 15) & ~(size_t)15;
  return off + 96 + 512 + (size_t)lut_n * 8;
}

// Host: e4m3 code (positive) -> value.
float e4m3_value(int c) {
  const int e = (c >> 3) & 15, m = c & 7;
  return e == 0 ? std::ldexp((float)m, -9) : std::ldexp(1.0f + m / 8.0f, e - 7);
}

// Host: the codebook search table over cells of width 2^-shift, the coarsest
// grid whose cells hold at most one boundary each.  Entry: the code of the
// cell's lower part and the cell's boundary (+inf if none); with
// `sign_magnitude` (16-level codes) the entry holds the stored forms of both
// codes, lower part in bits 0-7 and upper part in bits 8-15.
bool build_code_lut(K1Params& p, const float* bnd, int nbnd, bool sign_magnitude) {
  for (int shift = 3; shift <= 14; ++shift) {
    long cell[15];
    bool ok = true;
    for (int i = 0; i < nbnd; ++i) {
      cell[i] = (long)std::floor(std::ldexp((double)bnd[i], shift));   // exact
      if (i > 0 && cell[i] <= cell[i - 1]) ok = false;
    }
    if (!ok) continue;
    const long gmin = cell[0] - 1, gmax = cell[nbnd - 1] + 1;
    if (gmax - gmin + 1 > K1_LUT_MAX) return false;
    p.lut_shift = shift;
    p.lut_gmin = (int32_t)gmin;
    p.lut_n = (int32_t)(gmax - gmin + 1);
    for (long g = gmin; g <= gmax; ++g) {
      uint32_t base = 0, b = 0x7f800000u;   // no boundary in the cell: +inf
      for (int i = 0; i < nbnd; ++i) {
        if (cell[i] < g) ++base;
        if (cell[i] == g) std::memcpy(&b, &bnd[i], 4);
      }
      if (sign_magnitude) {
        // stored form of code c: c - 8 for c >= 8, (7 - c) | 8 below
        auto sm = [](uint32_t c) { return c >= 8 ? c - 8 : (7 - c) | 8u; };
        const uint32_t hi = base + 1 <= 15 ? base + 1 : 15;
        p.lut[g - gmin] = make_uint2(sm(base) | (sm(hi) << 8), b);
      } else {
        p.lut[g - gmin] = make_uint2(base, b);
      }
    }
    return true;
  }
  return false;
}

template <int L, int FMT, bool PROJ, bool WEIGHT, int IPW>
cudaError_t launch_k1_t(const K1Launch& a, cudaStream_t st) {
  constexpr int SLOTS = K1_WARPS * (32 / L);
  K1Params p{};
  p.x = a.x;
  p.rot = a.rot;
  p.U = a.U;
  p.coef = a.coef;
  p.codes = a.codes;
  p.scale = a.scale;
  p.bscale = a.bscale;
  p.status = a.status;
  p.wait_ns = a.wait_ns;
  p.inject_tx = a.inject_tx;
  p.rows = a.rows;
  p.K = a.K;
  p.r = a.r;
  p.inv_sqrt_b = a.inv_sqrt_b;
  p.sqrtK = a.sqrtK;
  p.nbnd = a.nbnd;
  for (int i = 0; i < 15; ++i) p.bnd[i] = i < a.nbnd ? a.bnd[i] : 0.f;
  p.lut_n = 0;
  if constexpr (FMT == RQ_FMT_LM16 || FMT == RQ_FMT_LM4) {
    if (a.nbnd < 1 || !build_code_lut(p, a.bnd, a.nbnd, FMT == RQ_FMT_LM16)) return cudaErrorInvalidValue;
  }
  for (int c = 0; c < 128; ++c) p.rcp_e4m3[c] = (c == 0 || c == 0x7F) ? 0.f : 1.0f / e4m3_value(c);
  const int nblk = a.K / (L * 32);
  const int ngrp = (WEIGHT && FMT == RQ_FMT_INT4) ? a.K / 128 : 1;
  const int sms = a.num_sms > 0 ? a.num_sms : 148;
  // rows per group: as many as fill IPW passes of the block slots; with the
  // projection no more than one wave needs (every SM busy with the chains)
  int R = (SLOTS * IPW) / nblk;
  if (R < 1) return cudaErrorInvalidValue;
  if (R > 24 && !PROJ) R = 24;
  // (the coefficient and residual mappings cover at most 32 rows)
  if (PROJ) R = min(min(R, 32), max(1, (a.rows + sms - 1) / sms));
  // few rows: smaller groups, so that every resident CTA gets some
  else R = min(R, max(1, (a.rows + (IPW == 1 ? 2 : 1) * sms - 1) / ((IPW == 1 ? 2 : 1) * sms)));
  size_t smem = k1_smem_bytes(R, a.K, nblk, PROJ, ngrp, p.lut_n);
  // two CTAs per SM for the single-pass variant
  const size_t cap = PROJ ? 232448 : IPW == 1 ? 110 * 1024 : 200 * 1024;
  while (smem > cap && R > 1) {
    --R;
    smem = k1_smem_bytes(R, a.K, nblk, PROJ, ngrp, p.lut_n);
  }
  if (smem > cap) return cudaErrorInvalidValue;
  p.R = R;
  p.ngroups = (a.rows + R - 1) / R;
  auto kern = k1_rotate_quantize<L, FMT, PROJ, WEIGHT, IPW>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  int grid = sms * (IPW == 1 ? 2 : 1);
  if (grid > p.ngroups) grid = p.ngroups;
  kern<<<grid, K1_THREADS, smem, st>>>(p);
  return cudaGetLastError();
}

template <int L, int FMT, bool PROJ, bool WEIGHT>
cudaError_t launch_k1_ipw(const K1Launch& a, cudaStream_t st) {
  // single pass (two CTAs per SM) whenever one row fits in the block slots and
  // one row's buffers fit half of shared memory; the projection keeps one CTA
  // per SM (its staged U fills shared memory)
  constexpr int SLOTS = K1_WARPS * (32 / L);
  if constexpr (!PROJ) {
    const int nblk = a.K / (L * 32);
    const int ngrp = (WEIGHT && FMT == RQ_FMT_INT4) ? a.K / 128 : 1;
    if (SLOTS / nblk >= 1 && k1_smem_bytes(1, a.K, nblk, false, ngrp, K1_LUT_MAX) <= 110 * 1024)
      return launch_k1_t<L, FMT, PROJ, WEIGHT, 1>(a, st);
  }
  return launch_k1_t<L, FMT, PROJ, WEIGHT, 2>(a, st);
}

// this kernel serves the calls with the low-rank projection and, for blocks of
// 128-512, any call whose shared-memory plan the rows-as-lanes kernel
// (rq_k1r.cu) cannot fit
template <int L, int FMT>
cudaError_t launch_k1_mode(const K1Launch& a, cudaStream_t st) {
  const bool proj = a.U != nullptr;
  if (a.weight) {
    if (proj) return launch_k1_ipw<L, FMT, true, true>(a, st);
    return launch_k1_ipw<L, FMT, false, true>(a, st);
  }
  if (proj) return launch_k1_ipw<L, FMT, true, false>(a, st);
  return launch_k1_ipw<L, FMT, false, false>(a, st);
}

template <int L>
cudaError_t launch_k1_fmt(const K1Launch& a, cudaStream_t st) {
  switch (a.fmt) {
    case RQ_FMT_INT4: return launch_k1_mode<L, RQ_FMT_INT4>(a, st);
    case RQ_FMT_LM16: return launch_k1_mode<L, RQ_FMT_LM16>(a, st);
    case RQ_FMT_LM4: return launch_k1_mode<L, RQ_FMT_LM4>(a, st);
    case RQ_FMT_NVFP4: return launch_k1_mode<L, RQ_FMT_NVFP4>(a, st);
  }
  return cudaErrorInvalidValue;
}

}  // namespace

cudaError_t launch_k1(const K1Launch& a, cudaStream_t st) {
  // the rows-as-lanes kernel: for what only it does (double rotation, INT4A,
  // INT8, the weight code sums, blocks outside 128-512, K an odd multiple of
  // 64) and where its layout pays: whole rows of 32
  // tokens per warp (K <= 1536) and enough row groups to fill the GPU twice;
  // measured on B200: Wan-like K = 1536 169 us against 186 us, while the
  // PixArt-width, FLUX QKV and FLUX down-projection layers ran faster here
  const bool only_r = a.rot2 || a.fmt == RQ_FMT_INT4A || a.fmt == RQ_FMT_INT8 || a.wz || a.K % 128 ||
                      (a.block != 128 && a.block != 256 && a.block != 512);
  const int sms = a.num_sms > 0 ? a.num_sms : 148;
  const bool r_pays = a.K <= 1536 && a.block <= 128 && a.rows >= 32 * 2 * sms;
  if (k1r_supports(a) && (only_r || (r_pays && !a.U))) {
    const cudaError_t e = launch_k1r(a, st);
    if (e != cudaErrorInvalidValue) return e;
  }
  if (only_r) return cudaErrorInvalidValue;
  switch (a.block) {
    case 128: return launch_k1_fmt<4>(a, st);
    case 256: return launch_k1_fmt<8>(a, st);
    case 512: return launch_k1_fmt<16>(a, st);
  }
  return cudaErrorInvalidValue;
}

}  // namespace rq
