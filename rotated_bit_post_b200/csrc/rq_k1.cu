// K1: fused rotate -> normalise -> quantize -> pack, one pass over each row.
//
// Implements the online activation transform of the rotated W4A4 linear layer
// (OrbitQuant abstract: randomized permuted block-Hadamard (RPBH) rotation,
// per-token normalisation, Lloyd-Max codes; TR-DQ section 3.1, Eq. 1-3: uniform
// grid with online min/max; DiRotQ abstract: NVFP4, PCA coefficients kept in
// BF16) and, on weight rows, the offline folding W' = W R^T followed by the same
// quantizers (OrbitQuant abstract; TR-DQ Eq. 9).
//
// Data flow per CTA (persistent over groups of R rows):
//   HBM --cp.async.bulk--> smem row buffer (double-buffered, mbarrier)
//   [projection: c = bf16(x U) sequentially over k, x_res = x - c U^T]
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

#include <cstdint>

#include "rq_internal.h"
#include "rq_ptx.cuh"

namespace rq {

namespace {

constexpr int K1_THREADS = 512;
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
};


// Swizzled NVFP4 block-scale offset: 128-row x 4-scale tiles of 512 bytes,
// tiles ordered [row tile][k tile]; inside: (m%32)*16 + ((m%128)/32)*4 + kb%4.
__device__ __forceinline__ size_t sf_offset(int m, int kb, int K) {
  const int tiles_k = K / 64;
  return ((size_t)(m >> 7) * tiles_k + (kb >> 2)) * 512 + (m & 31) * 16 + ((m >> 5) & 3) * 4 + (kb & 3);
}

template <int L, int FMT, bool PROJ, bool WEIGHT, int IPW>
__global__ void __launch_bounds__(K1_THREADS, IPW == 1 ? 2 : 1) k1_rotate_quantize(const __grid_constant__ K1Params p) {
  constexpr int B = L * 32;                // Hadamard block
  constexpr int GPW = 32 / L;              // lane groups (block slots) per warp
  constexpr int SLOTS = K1_WARPS * GPW;    // block slots per CTA pass
  extern __shared__ __align__(128) uint8_t smem[];
  const int K = p.K;
  const int R = p.R;
  const int nblk = K / B;
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int lq = lane % L;                 // lane inside its group
  const int slot0 = warp * GPW + lane / L; // first block slot of this lane group
  // shuffles stay inside the lane group (groups of one warp may take different branches)
  const unsigned gmask = L == 32 ? 0xffffffffu : (((1u << L) - 1u) << (lane & ~(L - 1)));

  // smem layout: [2][R][K] bf16 row buffers | (PROJ) [R][K] fp32 x / residual |
  // (PROJ) [R][32] fp32 coefficients | (PROJ) [K/2][32] U as BF16 pairs over k |
  // [R][nblk] fp32 block sum-of-squares | [R][ngrp] u32 amax bits |
  // [R][ngrp] fp32 row/group multipliers | mbarriers | abort flag | boundaries
  uint16_t* xs = reinterpret_cast<uint16_t*>(smem);
  size_t off = (size_t)2 * R * K * 2;
  float* xr = nullptr;
  float* cf = nullptr;
  uint32_t* up = nullptr;
  if constexpr (PROJ) {
    xr = reinterpret_cast<float*>(smem + off);
    off += (size_t)R * K * 4;
    cf = reinterpret_cast<float*>(smem + off);
    off += (size_t)R * 32 * 4;
    up = reinterpret_cast<uint32_t*>(smem + off);
    off += (size_t)(K / 2) * 32 * 4;
  }
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
  float* bnd_s = reinterpret_cast<float*>(smem + off + 32);  // 16 codebook boundaries
  if (threadIdx.x < 16) bnd_s[threadIdx.x] = threadIdx.x < p.nbnd ? p.bnd[threadIdx.x] : __int_as_float(0x7f800000);

  const uint32_t row_bytes = (uint32_t)K * 2;

  if (threadIdx.x == 0) {
    mbar_init(&full[0], 1);
    mbar_init(&full[1], 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if constexpr (PROJ) {
    // stage U (K x 32 BF16) once per CTA as words {U[2i][j], U[2i+1][j]}
    for (int t = threadIdx.x; t < (K / 2) * 32; t += K1_THREADS) {
      const int k2 = t >> 5, j = t & 31;
      up[t] = (uint32_t)__ldg(p.U + (size_t)(2 * k2) * 32 + j) |
              ((uint32_t)__ldg(p.U + (size_t)(2 * k2 + 1) * 32 + j) << 16);
    }
  }
  __syncthreads();

  auto issue_group = [&](int g, int buf) {
    const int r0 = g * R;
    const int nr = min(R, p.rows - r0);
    mbar_expect_tx(&full[buf], (uint32_t)nr * row_bytes);
    for (int i = 0; i < nr; ++i)
      bulk_g2s(xs + ((size_t)buf * R + i) * K, p.x + (size_t)(r0 + i) * K, row_bytes, &full[buf]);
  };

  if (threadIdx.x == 0 && blockIdx.x < p.ngroups) issue_group(blockIdx.x, 0);

  for (int i = threadIdx.x; i < 2 * R * ngrp; i += K1_THREADS) amax_bits2[i] = 0u;
  int it = 0;
  for (int g = blockIdx.x; g < p.ngroups; g += gridDim.x, ++it) {
    const int buf = it & 1;
    const int r0 = g * R;
    const int nr = min(R, p.rows - r0);
    float* part_ss = part_ss2 + (size_t)buf * R * nblk;
    uint32_t* amax_bits = amax_bits2 + (size_t)buf * R * ngrp;
    mbar_wait(&full[buf], (it >> 1) & 1, p.status, ST_TIMEOUT_LOAD, abort_flag);
    // everyone has finished the previous group past this barrier
    __syncthreads();
    if (*abort_flag) break;
    // prefetch the next group into the other buffer (last read by the previous
    // group's gather) and clear the other reductions (last read by the previous
    // group's quantization)
    if (threadIdx.x == 0 && g + (int)gridDim.x < p.ngroups) {
      fence_proxy_async_smem();
      issue_group(g + gridDim.x, buf ^ 1);
    }
    for (int i = threadIdx.x; i < R * ngrp; i += K1_THREADS) amax_bits2[(size_t)(buf ^ 1) * R * ngrp + i] = 0u;
    const uint16_t* xg = xs + (size_t)buf * R * K;

    // ------------------------------------------------------------ projection
    if constexpr (PROJ) {
      // rows -> FP32 (exact), the buffer that becomes the residual in place
      for (int t = threadIdx.x; t < nr * K / 2; t += K1_THREADS) {
        const uint32_t w2 = reinterpret_cast<const uint32_t*>(xg)[t];
        reinterpret_cast<float2*>(xr)[t] = make_float2(__uint_as_float(w2 << 16), __uint_as_float(w2 & 0xFFFF0000u));
      }
      __syncthreads();
      // c[row][j] = bf16(sum_k x[row][k] U[k][j]), each sum sequential in k.
      // Thread -> (pair of rows, j): two independent chains share every U load.
      const int npair = (nr + 1) >> 1;
      if (threadIdx.x < npair * 32) {
        const int j = lane;
        const int ra = 2 * (threadIdx.x >> 5);
        const int rb = min(ra + 1, nr - 1);
        const float4* xa = reinterpret_cast<const float4*>(xr + (size_t)ra * K);
        const float4* xb = reinterpret_cast<const float4*>(xr + (size_t)rb * K);
        float acc_a = 0.f, acc_b = 0.f;
#pragma unroll 4
        for (int k4 = 0; k4 < K / 4; ++k4) {
          const float4 va = xa[k4], vb = xb[k4];
          const uint32_t u01 = up[(2 * k4) * 32 + j], u23 = up[(2 * k4 + 1) * 32 + j];
          const float u0 = __uint_as_float(u01 << 16), u1 = __uint_as_float(u01 & 0xFFFF0000u);
          const float u2 = __uint_as_float(u23 << 16), u3 = __uint_as_float(u23 & 0xFFFF0000u);
          // every product of two BF16 values is exact in FP32: fma == add of the product
          acc_a = __fmaf_rn(va.x, u0, acc_a); acc_b = __fmaf_rn(vb.x, u0, acc_b);
          acc_a = __fmaf_rn(va.y, u1, acc_a); acc_b = __fmaf_rn(vb.y, u1, acc_b);
          acc_a = __fmaf_rn(va.z, u2, acc_a); acc_b = __fmaf_rn(vb.z, u2, acc_b);
          acc_a = __fmaf_rn(va.w, u3, acc_a); acc_b = __fmaf_rn(vb.w, u3, acc_b);
        }
        const uint16_t ca = __bfloat16_as_ushort(__float2bfloat16_rn(acc_a));
        const uint16_t cb = __bfloat16_as_ushort(__float2bfloat16_rn(acc_b));
        p.coef[(size_t)(r0 + ra) * 32 + j] = ca;
        cf[ra * 32 + j] = bf16_bits_to_f32(ca);
        if (rb != ra) {
          p.coef[(size_t)(r0 + rb) * 32 + j] = cb;
          cf[rb * 32 + j] = bf16_bits_to_f32(cb);
        }
      }
      __syncthreads();
      if constexpr (!WEIGHT) {
        // residual x - sum_j c_j U[k, j], subtracted in order j = 0..31.
        // Thread -> one k: U[k][0..31] loaded once, applied to every row.
        for (int k = threadIdx.x; k < K; k += K1_THREADS) {
          float u[32];
          const uint4* urow = reinterpret_cast<const uint4*>(p.U + (size_t)k * 32);
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            const uint4 w4 = __ldg(urow + q);
            const uint32_t ww[4] = {w4.x, w4.y, w4.z, w4.w};
#pragma unroll
            for (int h = 0; h < 4; ++h) {
              u[8 * q + 2 * h] = __uint_as_float(ww[h] << 16);
              u[8 * q + 2 * h + 1] = __uint_as_float(ww[h] & 0xFFFF0000u);
            }
          }
          for (int ri = 0; ri < nr; ++ri) {
            float v = xr[(size_t)ri * K + k];
            const float4* c4 = reinterpret_cast<const float4*>(cf + ri * 32);
#pragma unroll
            for (int q = 0; q < 8; ++q) {
              const float4 cc = c4[q];
              v = __fmaf_rn(-cc.x, u[4 * q], v);      // exact product
              v = __fmaf_rn(-cc.y, u[4 * q + 1], v);
              v = __fmaf_rn(-cc.z, u[4 * q + 2], v);
              v = __fmaf_rn(-cc.w, u[4 * q + 3], v);
            }
            xr[(size_t)ri * K + k] = v;
          }
        }
        __syncthreads();
      }
    }

    // ------------------------------------------------------------ phase A
    // gather, transform, block partials; y stays in registers until phase B
    const int nitems = nr * nblk;
    float y[IPW][32];
#pragma unroll
    for (int s = 0; s < IPW; ++s) {
      const int item = slot0 + s * SLOTS;
      if (item < nitems) {
        const int ri = item / nblk, bk = item - ri * nblk;
        const int i0 = bk * B + lq * 32;
        float* v = y[s];
        const int4* rp = reinterpret_cast<const int4*>(p.rot + i0);
#pragma unroll
        for (int e4 = 0; e4 < 8; ++e4) {
          const int4 rv = __ldg(rp + e4);
          const int rr[4] = {rv.x, rv.y, rv.z, rv.w};
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            const int src = rr[q] & 0x7fffffff;
            float xv;
            if constexpr (PROJ) xv = xr[(size_t)ri * K + src];
            else xv = bf16_bits_to_f32(xg[(size_t)ri * K + src]);
            v[4 * e4 + q] = __uint_as_float(__float_as_uint(xv) ^ ((uint32_t)rr[q] & 0x80000000u));
          }
        }
        // butterflies inside the lane: stride h pairs (e, e+h) with bit h of e clear
#pragma unroll
        for (int h = 1; h < 32; h <<= 1) {
#pragma unroll
          for (int e = 0; e < 32; ++e) {
            if ((e & h) == 0) {
              const float a = v[e], b = v[e + h];
              v[e] = __fadd_rn(a, b);
              v[e + h] = __fsub_rn(a, b);
            }
          }
        }
        // butterflies across the L lanes of the group: stride 32m pairs lane j
        // (bit m clear) with lane j^m; one exact FFMA per element: lower lane
        // v + o, upper lane o - v (+-1 * v is exact)
#pragma unroll
        for (int m = 1; m < L; m <<= 1) {
          const float sgn = (lq & m) ? -1.0f : 1.0f;
#pragma unroll
          for (int e = 0; e < 32; ++e) v[e] = __fmaf_rn(sgn, v[e], __shfl_xor_sync(gmask, v[e], m));
        }
        float amax = 0.f;
#pragma unroll
        for (int e = 0; e < 32; ++e) {
          v[e] = __fmul_rn(v[e], p.inv_sqrt_b);
          amax = fmaxf(amax, fabsf(v[e]));
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
          if (lq == 0) part_ss[ri * nblk + bk] = ss;
        } else if constexpr (WEIGHT && FMT == RQ_FMT_INT4) {
          // one scale per 128 rotated coordinates = 4 lanes
#pragma unroll
          for (int m = 1; m < (L < 4 ? L : 4); m <<= 1) amax = fmaxf(amax, __shfl_xor_sync(gmask, amax, m));
          if ((lq & 3) == 0) atomicMax(&amax_bits[ri * ngrp + i0 / 128], __float_as_uint(amax));
        } else {
#pragma unroll
          for (int m = 1; m < L; m <<= 1) amax = fmaxf(amax, __shfl_xor_sync(gmask, amax, m));
          if (lq == 0) atomicMax(&amax_bits[ri], __float_as_uint(amax));
        }
      }
    }
    __syncthreads();

    // ------------------------------------------------------------ phase B
#pragma unroll
    for (int s = 0; s < IPW; ++s) {
      const int item = slot0 + s * SLOTS;
      if (item < nitems) {
        const int ri = item / nblk, bk = item - ri * nblk;
        const int row = r0 + ri;
        const int i0 = bk * B + lq * 32;
        const float* v = y[s];
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
          float ss = part_ss[ri * nblk];
          for (int j = 1; j < nblk; ++j) ss = __fadd_rn(ss, part_ss[ri * nblk + j]);
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
            int q = __float2int_rn(__fmul_rn(v[e], inv));
            q = max(-7, min(7, q));
            pk[e >> 3] |= ((uint32_t)q & 0xFu) << (4 * (e & 7));
          }
        } else if constexpr (FMT == RQ_FMT_LM16 || FMT == RQ_FMT_LM4) {
          const float inv = mlt;
#pragma unroll
          for (int e = 0; e < 32; ++e) {
            const float u = __fmul_rn(v[e], inv);
            // number of boundaries <= u (ascending, padded with +inf to 16)
            uint32_t c = 0;
            if constexpr (FMT == RQ_FMT_LM16) {
#pragma unroll
              for (int step = 8; step >= 1; step >>= 1)
                if (u >= bnd_s[c + step - 1]) c += step;
              pk[e >> 3] |= c << (4 * (e & 7));
            } else {
              c = (u >= bnd_s[0]) + (u >= bnd_s[1]) + (u >= bnd_s[2]);
              pk[e >> 4] |= c << (2 * (e & 15));
            }
          }
        } else {  // NVFP4: two 16-element groups per lane
          const float inv_t = mlt;
          uint16_t sbs = 0;
#pragma unroll
          for (int gq = 0; gq < 2; ++gq) {
            float u[16];
            float m16 = 0.f;
#pragma unroll
            for (int e = 0; e < 16; ++e) {
              u[e] = __fmul_rn(v[16 * gq + e], inv_t);
              m16 = fmaxf(m16, fabsf(u[e]));
            }
            const float sbf = __fdiv_rn(m16, 6.0f);
            const uint8_t sb = (uint8_t)(cvt_e4m3x2(0.f, sbf) & 0xFF);
            const float rcp = sb ? __fdiv_rn(1.0f, e4m3_to_f32(sb)) : 0.f;
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

size_t k1_smem_bytes(int R, int K, int nblk, bool proj, int ngrp) {
  size_t off = (size_t)2 * R * K * 2;
  if (proj) off += (size_t)R * K * 4 + (size_t)R * 32 * 4 + (size_t)(K / 2) * 32 * 4;
  off += (size_t)2 * R * nblk * 4;
  off += (size_t)2 * R * ngrp * 4;
  off = (off + 15) & ~(size_t)15;
  return off + 32 + 64;
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
  p.rows = a.rows;
  p.K = a.K;
  p.r = a.r;
  p.inv_sqrt_b = a.inv_sqrt_b;
  p.sqrtK = a.sqrtK;
  p.nbnd = a.nbnd;
  for (int i = 0; i < 15; ++i) p.bnd[i] = i < a.nbnd ? a.bnd[i] : 0.f;
  const int nblk = a.K / (L * 32);
  // rows per group: as many as fill IPW passes of the block slots
  int R = (SLOTS * IPW) / nblk;
  if (R < 1) return cudaErrorInvalidValue;
  if (R > 24) R = 24;
  if (PROJ && R > 12) R = 12;
  const int ngrp = (WEIGHT && FMT == RQ_FMT_INT4) ? a.K / 128 : 1;
  size_t smem = k1_smem_bytes(R, a.K, nblk, PROJ, ngrp);
  // two CTAs per SM for the single-pass variant
  const size_t cap = IPW == 1 ? 110 * 1024 : 200 * 1024;
  while (smem > cap && R > 1) {
    --R;
    smem = k1_smem_bytes(R, a.K, nblk, PROJ, ngrp);
  }
  if (smem > cap) return cudaErrorInvalidValue;
  p.R = R;
  p.ngroups = (a.rows + R - 1) / R;
  auto kern = k1_rotate_quantize<L, FMT, PROJ, WEIGHT, IPW>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  int grid = (a.num_sms > 0 ? a.num_sms : 148) * (IPW == 1 ? 2 : 1);
  if (grid > p.ngroups) grid = p.ngroups;
  kern<<<grid, K1_THREADS, smem, st>>>(p);
  return cudaGetLastError();
}

template <int L, int FMT, bool PROJ, bool WEIGHT>
cudaError_t launch_k1_ipw(const K1Launch& a, cudaStream_t st) {
  // single pass (two CTAs per SM) whenever one row fits in the block slots;
  // the projection keeps one CTA per SM (its staged U fills shared memory)
  constexpr int SLOTS = K1_WARPS * (32 / L);
  if constexpr (!PROJ) {
    if (SLOTS / (a.K / (L * 32)) >= 1) return launch_k1_t<L, FMT, PROJ, WEIGHT, 1>(a, st);
  }
  return launch_k1_t<L, FMT, PROJ, WEIGHT, 2>(a, st);
}

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
  switch (a.block) {
    case 128: return launch_k1_fmt<4>(a, st);
    case 256: return launch_k1_fmt<8>(a, st);
    case 512: return launch_k1_fmt<16>(a, st);
  }
  return cudaErrorInvalidValue;
}

}  // namespace rq
