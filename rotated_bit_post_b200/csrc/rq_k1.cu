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
//   each warp owns one b-wide Hadamard block of one row at a time: lane l holds
//   elements l*E .. l*E+E-1 (E = b/32) after the signed-permutation gather from
//   smem; butterfly stages h < E in registers, h >= E through __shfl_xor_sync;
//   block partials (max|y|, pairwise sum of squares) -> smem
//   row scale from the partials (sum of squares added block by block, in order)
//   quantize, pack nibbles / crumbs, 8..64-bit stores.
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

__device__ __forceinline__ float warp_max(float v, unsigned lanes_mask_bits) {
  // max over groups of 2^lanes_mask_bits consecutive lanes (order-free)
  for (int m = 1; m < (1 << lanes_mask_bits); m <<= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, m));
  return v;
}

// Swizzled NVFP4 block-scale offset: 128-row x 4-scale tiles of 512 bytes,
// tiles ordered [row tile][k tile]; inside: (m%32)*16 + ((m%128)/32)*4 + kb%4.
__device__ __forceinline__ size_t sf_offset(int m, int kb, int K) {
  const int tiles_k = K / 64;
  return ((size_t)(m >> 7) * tiles_k + (kb >> 2)) * 512 + (m & 31) * 16 + ((m >> 5) & 3) * 4 + (kb & 3);
}

template <int E, int FMT, bool PROJ, bool WEIGHT, int IPW>
__global__ void __launch_bounds__(K1_THREADS, 1) k1_rotate_quantize(const __grid_constant__ K1Params p) {
  constexpr int B = E * 32;  // Hadamard block
  extern __shared__ __align__(128) uint8_t smem[];
  const int K = p.K;
  const int R = p.R;
  const int nblk = K / B;
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  // smem layout: [2][R][K] bf16 row buffers | (PROJ) [R][K] fp32 residual |
  // (PROJ) [R][32] fp32 coefficients | [R][nblk] fp32 block sum-of-squares |
  // [R][ngrp] u32 amax bits | mbarriers | abort flag
  uint16_t* xs = reinterpret_cast<uint16_t*>(smem);
  size_t off = (size_t)2 * R * K * 2;
  float* xr = nullptr;
  float* cf = nullptr;
  if constexpr (PROJ) {
    xr = reinterpret_cast<float*>(smem + off);
    off += (size_t)R * K * 4;
    cf = reinterpret_cast<float*>(smem + off);
    off += (size_t)R * 32 * 4;
  }
  float* part_ss = reinterpret_cast<float*>(smem + off);
  off += (size_t)R * nblk * 4;
  const int ngrp = (WEIGHT && FMT == RQ_FMT_INT4) ? K / 128 : 1;
  uint32_t* amax_bits = reinterpret_cast<uint32_t*>(smem + off);
  off += (size_t)R * ngrp * 4;
  off = (off + 15) & ~(size_t)15;
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + off);
  volatile int32_t* abort_flag = reinterpret_cast<volatile int32_t*>(smem + off + 16);

  const uint32_t row_bytes = (uint32_t)K * 2;

  if (threadIdx.x == 0) {
    mbar_init(&full[0], 1);
    mbar_init(&full[1], 1);
    *abort_flag = 0;
    fence_mbar_init();
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

  int it = 0;
  for (int g = blockIdx.x; g < p.ngroups; g += gridDim.x, ++it) {
    const int buf = it & 1;
    const int r0 = g * R;
    const int nr = min(R, p.rows - r0);
    // clear per-group reductions (visible after the wait + barrier below)
    for (int i = threadIdx.x; i < R * ngrp; i += K1_THREADS) amax_bits[i] = 0u;
    if (!mbar_wait(&full[buf], (it >> 1) & 1, p.status, ST_TIMEOUT_LOAD, abort_flag)) {
      // fall through to the barrier; every thread leaves together below
    }
    // prefetch the next group into the other buffer (its readers finished
    // before the trailing __syncthreads of the previous iteration)
    if (threadIdx.x == 0 && g + (int)gridDim.x < p.ngroups) {
      fence_proxy_async_smem();
      issue_group(g + gridDim.x, buf ^ 1);
    }
    __syncthreads();
    if (*abort_flag) break;
    const uint16_t* xg = xs + (size_t)buf * R * K;

    // ------------------------------------------------------------ projection
    if constexpr (PROJ) {
      // coefficients: thread t -> (row t / 32, j = t % 32), sequential over k.
      for (int t = threadIdx.x; t < nr * 32; t += K1_THREADS) {
        const int ri = t >> 5, j = t & 31;
        float acc = 0.f;
        if (j < p.r) {
          const uint16_t* xrow = xg + (size_t)ri * K;
          const uint16_t* Uj = p.U + j;
#pragma unroll 8
          for (int k = 0; k < K; ++k) {
            const float xv = bf16_bits_to_f32(xrow[k]);
            const float uv = bf16_bits_to_f32(__ldg(Uj + (size_t)k * p.r));
            acc = __fmaf_rn(xv, uv, acc);  // exact product: equals RN(acc + x*u)
          }
          // round to BF16 (RNE) and keep the rounded value
          const uint16_t cb = __bfloat16_as_ushort(__float2bfloat16_rn(acc));
          p.coef[(size_t)(r0 + ri) * p.r + j] = cb;
          acc = bf16_bits_to_f32(cb);
        }
        cf[ri * 32 + j] = acc;
      }
      __syncthreads();
      // residual x - sum_j c_j U[k, j] in order j = 0..r-1 (weight rows keep x)
      for (int t = threadIdx.x; t < nr * K; t += K1_THREADS) {
        const int ri = t / K, k = t - ri * K;
        float v = bf16_bits_to_f32(xg[(size_t)ri * K + k]);
        if constexpr (!WEIGHT) {
          const uint16_t* Uk = p.U + (size_t)k * p.r;
          for (int j = 0; j < p.r; ++j)
            v = __fmaf_rn(-cf[ri * 32 + j], bf16_bits_to_f32(__ldg(Uk + j)), v);  // exact product
        }
        xr[(size_t)ri * K + k] = v;
      }
      __syncthreads();
    }

    // ------------------------------------------------------------ phase A
    const int nitems = nr * nblk;
    float y[IPW][E];
#pragma unroll
    for (int s = 0; s < IPW; ++s) {
      const int item = warp + s * K1_WARPS;
      if (item < nitems) {
        const int ri = item / nblk, bk = item - ri * nblk;
        const int i0 = bk * B + lane * E;
        float v[E];
#pragma unroll
        for (int e = 0; e < E; e += 4) {
          const int4 rv = __ldg(reinterpret_cast<const int4*>(p.rot + i0 + e));
          const int rr[4] = {rv.x, rv.y, rv.z, rv.w};
#pragma unroll
          for (int q = 0; q < 4 && e + q < E; ++q) {
            const int src = rr[q] & 0x7fffffff;
            float xv;
            if constexpr (PROJ) xv = xr[(size_t)ri * K + src];
            else xv = bf16_bits_to_f32(xg[(size_t)ri * K + src]);
            v[e + q] = __uint_as_float(__float_as_uint(xv) ^ ((uint32_t)rr[q] & 0x80000000u));
          }
        }
        // butterflies inside the lane: stride h pairs (e, e+h) with bit h of e clear
#pragma unroll
        for (int h = 1; h < E; h <<= 1) {
#pragma unroll
          for (int e = 0; e < E; ++e) {
            if ((e & h) == 0) {
              const float a = v[e], b = v[e + h];
              v[e] = __fadd_rn(a, b);
              v[e + h] = __fsub_rn(a, b);
            }
          }
        }
        // butterflies across lanes: stride h = E*m pairs lane l (bit m clear) with l^m
#pragma unroll
        for (int m = 1; m < 32; m <<= 1) {
          const bool upper = (lane & m) != 0;
#pragma unroll
          for (int e = 0; e < E; ++e) {
            const float o = __shfl_xor_sync(0xffffffffu, v[e], m);
            v[e] = upper ? __fsub_rn(o, v[e]) : __fadd_rn(v[e], o);
          }
        }
        float amax = 0.f;
#pragma unroll
        for (int e = 0; e < E; ++e) {
          y[s][e] = __fmul_rn(v[e], p.inv_sqrt_b);
          amax = fmaxf(amax, fabsf(y[s][e]));
        }
        if constexpr (FMT == RQ_FMT_LM16 || FMT == RQ_FMT_LM4) {
          // perfect pairwise tree: in-lane levels, then lanes by xor 1,2,4,8,16
          float sq[E];
#pragma unroll
          for (int e = 0; e < E; ++e) sq[e] = __fmul_rn(y[s][e], y[s][e]);
#pragma unroll
          for (int w = 1; w < E; w <<= 1) {
#pragma unroll
            for (int e = 0; e < E; e += 2 * w) sq[e] = __fadd_rn(sq[e], sq[e + w]);
          }
          float ss = sq[0];
#pragma unroll
          for (int m = 1; m < 32; m <<= 1) ss = __fadd_rn(ss, __shfl_xor_sync(0xffffffffu, ss, m));
          if (lane == 0) part_ss[ri * nblk + bk] = ss;
        } else if constexpr (WEIGHT && FMT == RQ_FMT_INT4) {
          // per 128-element group of the rotated row
          constexpr int LPG = (128 / E) < 32 ? (128 / E) : 32;  // lanes per group inside this block
          constexpr int BITS = LPG == 32 ? 5 : LPG == 16 ? 4 : LPG == 8 ? 3 : LPG == 4 ? 2 : LPG == 2 ? 1 : 0;
          const float gm = warp_max(amax, BITS);
          if ((lane & (LPG - 1)) == 0) {
            const int grp = (i0) / 128;
            atomicMax(&amax_bits[ri * ngrp + grp], __float_as_uint(gm));
          }
        } else {
          const float gm = warp_max(amax, 5);
          if (lane == 0) atomicMax(&amax_bits[ri], __float_as_uint(gm));
        }
      }
    }
    __syncthreads();

    // ------------------------------------------------------------ phase B
#pragma unroll
    for (int s = 0; s < IPW; ++s) {
      const int item = warp + s * K1_WARPS;
      if (item < nitems) {
        const int ri = item / nblk, bk = item - ri * nblk;
        const int row = r0 + ri;
        const int i0 = bk * B + lane * E;
        uint32_t packed_lo = 0, packed_hi = 0;  // up to 64 bits of packed codes
        if constexpr (FMT == RQ_FMT_INT4) {
          float amax;
          if constexpr (WEIGHT) amax = __uint_as_float(amax_bits[ri * ngrp + i0 / 128]);
          else amax = __uint_as_float(amax_bits[ri]);
          const float inv = amax > 0.f ? __fdiv_rn(7.0f, amax) : 0.f;
#pragma unroll
          for (int e = 0; e < E; ++e) {
            int q = __float2int_rn(__fmul_rn(y[s][e], inv));
            q = max(-7, min(7, q));
            const uint32_t nib = (uint32_t)q & 0xFu;
            if (e < 8) packed_lo |= nib << (4 * e);
            else packed_hi |= nib << (4 * (e - 8));
          }
          if constexpr (WEIGHT) {
            if ((i0 & 127) == 0) {  // first lane of each group writes its scale
              p.scale[(size_t)(i0 / 128) * p.rows + row] = amax > 0.f ? __fdiv_rn(amax, 7.0f) : 0.f;
            }
          } else if (bk == 0 && lane == 0) {
            p.scale[row] = amax > 0.f ? __fdiv_rn(amax, 7.0f) : 0.f;
          }
        } else if constexpr (FMT == RQ_FMT_LM16 || FMT == RQ_FMT_LM4) {
          float ss = part_ss[ri * nblk];
          for (int j = 1; j < nblk; ++j) ss = __fadd_rn(ss, part_ss[ri * nblk + j]);
          const float nrm = __fsqrt_rn(ss);
          const float inv = nrm > 0.f ? __fdiv_rn(p.sqrtK, nrm) : 0.f;
#pragma unroll
          for (int e = 0; e < E; ++e) {
            const float u = __fmul_rn(y[s][e], inv);
            uint32_t c = 0;
#pragma unroll
            for (int i = 0; i < 15; ++i)
              if (i < p.nbnd) c += (u >= p.bnd[i]) ? 1u : 0u;
            if constexpr (FMT == RQ_FMT_LM4) {
              if (e < 16) packed_lo |= (c & 3u) << (2 * e);
            } else {
              if (e < 8) packed_lo |= c << (4 * e);
              else packed_hi |= c << (4 * (e - 8));
            }
          }
          if (bk == 0 && lane == 0) p.scale[row] = nrm > 0.f ? __fdiv_rn(nrm, p.sqrtK) : 0.f;
        } else {  // NVFP4
          const float amax = __uint_as_float(amax_bits[ri]);
          const float inv_t = amax > 0.f ? __fdiv_rn(2688.0f, amax) : 0.f;
          float u[E];
          float lm = 0.f;
#pragma unroll
          for (int e = 0; e < E; ++e) {
            u[e] = __fmul_rn(y[s][e], inv_t);
            lm = fmaxf(lm, fabsf(u[e]));
          }
          // 16-element groups: E=4 -> 4 lanes, E=8 -> 2 lanes, E=16 -> 1 lane
          constexpr int LPG16 = 16 / E;
          constexpr int B16 = LPG16 == 4 ? 2 : LPG16 == 2 ? 1 : 0;
          const float m16 = warp_max(lm, B16);
          const float sbf = __fdiv_rn(m16, 6.0f);
          const uint8_t sb = (uint8_t)(cvt_e4m3x2(0.f, sbf) & 0xFF);
          const float sbv = e4m3_to_f32(sb);
          const float rcp = sb ? __fdiv_rn(1.0f, sbv) : 0.f;
#pragma unroll
          for (int e = 0; e < E; e += 2) {
            uint32_t byte = sb ? (uint32_t)cvt_e2m1x2(__fmul_rn(u[e + 1], rcp), __fmul_rn(u[e], rcp)) : 0u;
            const int sh = 4 * e;
            if (e < 8) packed_lo |= byte << sh;
            else packed_hi |= byte << (sh - 32);
          }
          if ((lane & (LPG16 - 1)) == 0) {
            const int kb = i0 / 16;
            p.bscale[sf_offset(row, kb, K)] = sb;
          }
          if (bk == 0 && lane == 0) p.scale[row] = amax > 0.f ? __fdiv_rn(amax, 2688.0f) : 0.f;
        }
        // store this lane's packed codes
        if constexpr (FMT == RQ_FMT_LM4) {
          uint8_t* dst = p.codes + (size_t)row * (K / 4) + i0 / 4;
          if constexpr (E == 4) *dst = (uint8_t)packed_lo;
          else if constexpr (E == 8) *reinterpret_cast<uint16_t*>(dst) = (uint16_t)packed_lo;
          else *reinterpret_cast<uint32_t*>(dst) = packed_lo;
        } else {
          uint8_t* dst = p.codes + (size_t)row * (K / 2) + i0 / 2;
          if constexpr (E == 4) *reinterpret_cast<uint16_t*>(dst) = (uint16_t)packed_lo;
          else if constexpr (E == 8) *reinterpret_cast<uint32_t*>(dst) = packed_lo;
          else *reinterpret_cast<uint2*>(dst) = make_uint2(packed_lo, packed_hi);
        }
      }
    }
    __syncthreads();
  }
}

template <int E, int FMT, bool PROJ, bool WEIGHT>
constexpr int ipw_for() {
  return E == 4 ? 8 : E == 8 ? 6 : 3;
}

size_t k1_smem_bytes(int R, int K, int nblk, bool proj, int ngrp) {
  size_t off = (size_t)2 * R * K * 2;
  if (proj) off += (size_t)R * K * 4 + (size_t)R * 32 * 4;
  off += (size_t)R * nblk * 4;
  off += (size_t)R * ngrp * 4;
  off = (off + 15) & ~(size_t)15;
  return off + 32;
}

template <int E, int FMT, bool PROJ, bool WEIGHT>
cudaError_t launch_k1_t(const K1Launch& a, cudaStream_t st) {
  constexpr int IPW = ipw_for<E, FMT, PROJ, WEIGHT>();
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
  const int nblk = a.K / (E * 32);
  int R = (K1_WARPS * IPW) / nblk;
  if (R < 1) return cudaErrorInvalidValue;
  if (R > 16) R = 16;
  if (PROJ && R > 8) R = 8;
  const int ngrp = (WEIGHT && FMT == RQ_FMT_INT4) ? a.K / 128 : 1;
  size_t smem = k1_smem_bytes(R, a.K, nblk, PROJ, ngrp);
  while (smem > 200 * 1024 && R > 1) {
    --R;
    smem = k1_smem_bytes(R, a.K, nblk, PROJ, ngrp);
  }
  if (smem > 200 * 1024) return cudaErrorInvalidValue;
  p.R = R;
  p.ngroups = (a.rows + R - 1) / R;
  auto kern = k1_rotate_quantize<E, FMT, PROJ, WEIGHT, IPW>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  int grid = a.num_sms > 0 ? a.num_sms : 148;
  if (grid > p.ngroups) grid = p.ngroups;
  kern<<<grid, K1_THREADS, smem, st>>>(p);
  return cudaGetLastError();
}

template <int E, int FMT>
cudaError_t launch_k1_mode(const K1Launch& a, cudaStream_t st) {
  const bool proj = a.U != nullptr;
  if (a.weight) {
    if (proj) return launch_k1_t<E, FMT, true, true>(a, st);
    return launch_k1_t<E, FMT, false, true>(a, st);
  }
  if (proj) return launch_k1_t<E, FMT, true, false>(a, st);
  return launch_k1_t<E, FMT, false, false>(a, st);
}

template <int E>
cudaError_t launch_k1_fmt(const K1Launch& a, cudaStream_t st) {
  switch (a.fmt) {
    case RQ_FMT_INT4: return launch_k1_mode<E, RQ_FMT_INT4>(a, st);
    case RQ_FMT_LM16: return launch_k1_mode<E, RQ_FMT_LM16>(a, st);
    case RQ_FMT_LM4: return launch_k1_mode<E, RQ_FMT_LM4>(a, st);
    case RQ_FMT_NVFP4: return launch_k1_mode<E, RQ_FMT_NVFP4>(a, st);
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
