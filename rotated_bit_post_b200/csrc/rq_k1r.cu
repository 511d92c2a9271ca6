// K1, rows-as-lanes form: rotate -> normalise -> quantize -> pack for
// activation and weight rows without the low-rank projection.
//
// Implements the online activation transform of the rotated W4A4 linear layer
// (OrbitQuant abstract: randomized permuted block-Hadamard (RPBH) rotation,
// per-token normalisation, Lloyd-Max codes; TR-DQ section 3.1, Eq. 1-3: uniform
// grid with online min/max, symmetric or with a zero point, 4 or 8 bits (the
// W4A8 setting of Tables 1-5); DiRotQ abstract:
// NVFP4 on Blackwell) and, on weight rows, the offline folding W' = W R^T
// followed by the same quantizers (OrbitQuant abstract; TR-DQ Eq. 9).  With a
// second table it applies TR-DQ's double block rotation R2 P R1 (section 3.2,
// Eq. 9: block rotation, zigzag permutation, block rotation).
//
// Data flow per CTA (persistent over groups of R rows):
//   HBM --cp.async.bulk--> landing buffer (R rows)
//   restage: every row copied to a second buffer with the random signs applied
//     (BF16 sign bit) at a row pitch of an odd number of 32-bit words, so that
//     lanes reading the same rotated coordinate of different rows hit
//     different banks; the landing buffer is then free for the next group
//   [double rotation: the first block rotation on the natural channel order,
//    its FP32 output stored at an odd-word row pitch, gathered again through
//    the zigzag permutation]
//   phase A: a warp's lanes are R rows x F segments; a thread owns one segment
//     of 128 consecutive rotated coordinates of one row (64 when K is an odd
//     multiple of 64), gathered through the
//     permutation table (byte offsets) into registers; butterflies of blocks up
//     to 128 run in registers (blocks of 256-1024: T = b/128 threads, the last
//     log2 T stages through __shfl_xor_sync); y = v * fp32(1/sqrt b); per-block
//     pairwise sums of squares or per-segment maxima go to shared memory
//   phase B: every thread derives its row's scale from the partials in the
//     same order, quantizes its segment, packs it and stores its codes.
//
// FP32 contract (bit-exact against the CPU oracle): explicit round-to-nearest-
// even operations, no contraction; packed f32x2 operations round each lane
// like the scalar instruction.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>
#include <cstring>

#include "rq_internal.h"
#include "rq_ptx.cuh"

namespace rq {

namespace {

constexpr int R_THREADS = 384;     // 12 warps
constexpr int R_LUT_MAX = 1536;    // codebook cells
// rotated coordinates per thread (SEG): 128, or 64 for rows with K % 128 != 0
// (blocks up to 64; codebook and NVFP4 codes); the gather table's stride per
// segment is SEG + 4 entries, which breaks bank aliasing

struct __align__(16) K1RParams {
  const uint16_t* x;       // rows x K, BF16 bits
  const int32_t* rot;      // signed permutation of the (first) rotation
  const int32_t* rot2;     // double rotation: signed permutation of the second (zigzag) or null
  uint8_t* codes;
  float* scale;            // act: [rows]; weight INT4: [K/128][rows]; else [rows]
  float* zp;               // asymmetric INT4: per-row zero point (code offset)
  float* wz;               // INT4 weights: per-row sum over groups of scale x code sum (or null)
  uint8_t* bscale;         // NVFP4 block scales (128 x 4 tiles)
  int32_t* status;
  uint64_t wait_ns;
  uint32_t inject_tx;
  int32_t rows, K, R, ngroups;
  int32_t B;               // Hadamard block (16 .. 1024)
  int32_t F;               // segments per warp (1, 2, 4, 8, 16); rows per group R = 32 / F
  int32_t dbl;             // 1: TR-DQ double rotation (rot2 given)
  float inv_sqrt_b, sqrtK;
  // codebook cells: t = u * 2^lut_shift; cell = floor(t) - lut_gmin, clamped to
  // [0, lut_n - 1]; code = t >= cell.y ? cell.x >> 8 : cell.x & 0xFF
  int32_t lut_shift, lut_gmin, lut_n;
  uint2 lut[R_LUT_MAX];
  float rcp_e4m3[128];     // fp32(1 / e4m3 value) of the positive e4m3 codes, 0 for code 0
};

__device__ __forceinline__ size_t sf_off(int m, int kb, int K) {
  const int tiles_k = K / 64;
  return ((size_t)(m >> 7) * tiles_k + (kb >> 2)) * 512 + (m & 31) * 16 + ((m >> 5) & 3) * 4 + (kb & 3);
}

// (a, b) -> (a + b, a - b) on the pairs (a0, a1), (b0, b1)
__device__ __forceinline__ void bfly2(float& a0, float& a1, float& b0, float& b1) {
  asm("{\n\t.reg .b64 a, b, s, d;\n\t"
      "mov.b64 a, {%0, %1};\n\tmov.b64 b, {%2, %3};\n\t"
      "add.rn.f32x2 s, a, b;\n\tsub.rn.f32x2 d, a, b;\n\t"
      "mov.b64 {%0, %1}, s;\n\tmov.b64 {%2, %3}, d;\n\t}"
      : "+f"(a0), "+f"(a1), "+f"(b0), "+f"(b1));
}
// (v0, v1) = s * (v0, v1) + (o0, o1), s = +-1 on both lanes: one exact FMA each
__device__ __forceinline__ void fma2s(float& v0, float& v1, float s, float o0, float o1) {
  asm("{\n\t.reg .b64 v, o, ss;\n\t"
      "mov.b64 v, {%0, %1};\n\tmov.b64 o, {%3, %4};\n\tmov.b64 ss, {%2, %2};\n\t"
      "fma.rn.f32x2 v, ss, v, o;\n\tmov.b64 {%0, %1}, v;\n\t}"
      : "+f"(v0), "+f"(v1)
      : "f"(s), "f"(o0), "f"(o1));
}
// (v0, v1) *= (s, s)
__device__ __forceinline__ void mul2s(float& v0, float& v1, float s) {
  asm("{\n\t.reg .b64 v, ss;\n\tmov.b64 v, {%0, %1};\n\tmov.b64 ss, {%2, %2};\n\t"
      "mul.rn.f32x2 v, v, ss;\n\tmov.b64 {%0, %1}, v;\n\t}"
      : "+f"(v0), "+f"(v1)
      : "f"(s));
}
// Butterflies of the thread's SEG registers: blocks of min(b, SEG), stages in
// ascending stride; stride 1 pairs share a register pair (scalar), strides 2+
// run as packed pairs; then the cross-thread strides SEG .. b/2 with the lanes
// l ^ m of the same block (lower lane v + o, upper lane o - v, both exact
// single roundings).
template <int B, int SEG>
__device__ __forceinline__ void fwht_seg(float (&v)[SEG], int part) {
  constexpr int IN = B < SEG ? B : SEG;
  constexpr int T = B > SEG ? B / SEG : 1;
#pragma unroll
  for (int e = 0; e < SEG; e += 2) {
    const float a = v[e], c = v[e + 1];
    v[e] = __fadd_rn(a, c);
    v[e + 1] = __fsub_rn(a, c);
  }
#pragma unroll
  for (int h = 2; h < IN; h <<= 1) {
#pragma unroll
    for (int e = 0; e < SEG; e += 2)
      if ((e & h) == 0) bfly2(v[e], v[e + 1], v[e + h], v[e + h + 1]);
  }
#pragma unroll
  for (int m = 1; m < T; m <<= 1) {
    {
      const float sgn = (part & m) ? -1.0f : 1.0f;
#pragma unroll
      for (int e = 0; e < SEG; e += 2) {
        const float o0 = __shfl_xor_sync(0xffffffffu, v[e], m), o1 = __shfl_xor_sync(0xffffffffu, v[e + 1], m);
        fma2s(v[e], v[e + 1], sgn, o0, o1);
      }
    }
  }
}

// Pairwise sum of squares of v[I .. I+N-1] (natural order, a perfect binary
// tree), evaluated depth first so that only the partial sums of the open
// subtrees are live; every subtree of size `in` (the block, at most 128) is
// written to out[its first index / in].
template <int SEG, int I, int N>
struct SqTree {
  static __device__ __forceinline__ float run(const float (&v)[SEG], int in, float* out) {
    float r;
    if constexpr (N == 1) {
      r = __fmul_rn(v[I], v[I]);
    } else {
      r = __fadd_rn(SqTree<SEG, I, N / 2>::run(v, in, out), SqTree<SEG, I + N / 2, N / 2>::run(v, in, out));
    }
    if constexpr (N >= 16) {   // blocks are at least 16 wide
      if (N == in) out[I / N] = r;
    }
    return r;
  }
};

template <int FMT, bool WEIGHT, int B, int SEG>
__global__ void __launch_bounds__(R_THREADS, 1) k1r_kernel(const __grid_constant__ K1RParams p) {
  static_assert(SEG == 128 || (B <= 64 && (FMT == RQ_FMT_LM16 || FMT == RQ_FMT_LM4 || FMT == RQ_FMT_NVFP4)),
                "64-wide segments carry codebook and NVFP4 rows with blocks up to 64");
  constexpr int TS = SEG + 4;
  constexpr int T = B > SEG ? B / SEG : 1;        // threads per Hadamard block (<= F)
  const int F = p.F;
  const bool DBL = p.dbl != 0;
  constexpr int NBT = B < SEG ? SEG / B : 1;      // blocks per thread
  const int RW = 32 / F;                          // rows of a group (= rows per warp)
  extern __shared__ __align__(128) uint8_t smem[];
  const int K = p.K;
  const int S = K / SEG;                          // segments per row
  const int nblk = K / B;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int rl = lane / F;                        // row inside the group
  const int seg = warp * F + lane % F;            // this thread's segment
  const int part = seg % T;                       // part of a block > 128
  const bool active = seg < S;
  const int nwarps = (S + F - 1) / F;
  const uint32_t P = 2u * K + 4u;                 // staged BF16 row pitch (odd words)
  const uint32_t P2 = 4u * K + 4u;                // staged FP32 row pitch (double rotation)

  // shared memory: landing [R][K] bf16 | staged [R][P] | (DBL) [R][P2] fp32 |
  // gather tables [S][TS] u32 (x2 for DBL) | sign words [K/8] | partials |
  // mbarrier + abort flag | e4m3 reciprocals | codebook cells
  uint8_t* land = smem;
  uint8_t* stg = land + (size_t)RW * K * 2;
  uint8_t* y1 = stg + (size_t)RW * P;
  size_t off = (size_t)RW * K * 2 + (size_t)RW * P + (DBL ? (size_t)RW * P2 : 0);
  off = (off + 15) & ~(size_t)15;
  uint32_t* gtab = reinterpret_cast<uint32_t*>(smem + off);          // second (or only) gather
  off += (size_t)S * TS * 4;
  uint32_t* sgnw = reinterpret_cast<uint32_t*>(smem + off);          // sign words of the staged rows
  off += (size_t)(K / 8) * 4;
  constexpr int NPART = (FMT == RQ_FMT_LM16 || FMT == RQ_FMT_LM4) ? 1 : 2;   // ss | max, min
  float* partials = reinterpret_cast<float*>(smem + off);            // [2][RW][max(nblk, nwarps)][NPART]
  const int pstride = (nblk > S ? nblk : S) * NPART;
  off += (size_t)2 * RW * pstride * 4;
  off = (off + 15) & ~(size_t)15;
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + off);
  volatile int32_t* abort_flag = reinterpret_cast<volatile int32_t*>(smem + off + 8);
  float* rcp_s = reinterpret_cast<float*>(smem + off + 16);
  uint2* lut_s = reinterpret_cast<uint2*>(smem + off + 16 + 512);

  if (threadIdx.x == 0) {
    mbar_init(full, 1);
    *abort_flag = 0;
    fence_mbar_init();
    griddep_launch_dependents();
  }
  // tables: the gather offsets of the (second) rotation and the signs of the
  // staged rows, as XOR words: for the 8 channels 8j..8j+7, pair k's two sign
  // bits at bits 15 - k and 31 - k of word j
  const int32_t* grot = DBL ? p.rot2 : p.rot;
  for (int i = threadIdx.x; i < K; i += blockDim.x) {
    const uint32_t g = (uint32_t)__ldg(grot + i) & 0x7fffffffu;
    gtab[(i / SEG) * TS + i % SEG] = DBL ? 4u * g : 2u * g;
  }
  for (int j = threadIdx.x; j < K / 8; j += blockDim.x) sgnw[j] = 0u;
  if constexpr (FMT == RQ_FMT_NVFP4)
    for (int i = threadIdx.x; i < 128; i += blockDim.x) rcp_s[i] = p.rcp_e4m3[i];
  if constexpr (FMT == RQ_FMT_LM16 || FMT == RQ_FMT_LM4)
    for (int i = threadIdx.x; i < p.lut_n; i += blockDim.x) lut_s[i] = p.lut[i];
  __syncthreads();
  for (int i = threadIdx.x; i < K; i += blockDim.x) {
    // the sign of channel c (first rotation: rot[i] names channel c = perm[i]
    // with its sign in bit 31; the double rotation's first stage is the
    // identity permutation, so rot[c] holds channel c's own sign)
    const int32_t rv = __ldg(p.rot + i);
    const uint32_t c = (uint32_t)rv & 0x7fffffffu;
    if (rv < 0) {
      const uint32_t k = (c & 7u) >> 1;
      atomicOr(&sgnw[c >> 3], 1u << ((c & 1u) ? 31u - k : 15u - k));
    }
  }

  const uint32_t row_bytes = (uint32_t)K * 2;
  auto issue_group = [&](int g) {
    const int r0 = g * RW;
    const int nr = min(RW, p.rows - r0);
    mbar_expect_tx(full, (uint32_t)nr * row_bytes + (g == (int)blockIdx.x ? p.inject_tx : 0u));
    for (int i = 0; i < nr; ++i) bulk_g2s(land + (size_t)i * K * 2, p.x + (size_t)(r0 + i) * K, row_bytes, full);
  };
  __syncthreads();
  if (threadIdx.x == 0 && blockIdx.x < p.ngroups) issue_group(blockIdx.x);

  int it = 0;
  for (int g = blockIdx.x; g < p.ngroups; g += gridDim.x, ++it) {
    const int r0 = g * RW;
    const int nr = min(RW, p.rows - r0);
    float* pt = partials + (size_t)(it & 1) * RW * pstride;
    // a thread whose wait runs out skips the restage; the decision to leave is
    // taken by the whole CTA after the barrier below (the abort flag is set
    // before it), so no thread heads for a barrier that another has left
    const bool ok = mbar_wait(full, it & 1, p.status, ST_TIMEOUT_LOAD, abort_flag, p.wait_ns);
    // ------------------------------------------------------------ restage
    // (row, 16-byte unit) advanced by the block's stride without a division per step
    const int K8 = K / 8, dr = (int)blockDim.x / K8, dj = (int)blockDim.x - dr * K8;
    for (int r = (int)threadIdx.x / K8, j = (int)threadIdx.x - r * K8; ok && r < nr;) {
      const uint4 d = *reinterpret_cast<const uint4*>(land + (size_t)r * K * 2 + (size_t)j * 16);
      const uint32_t sw = sgnw[j];
      uint32_t* dst = reinterpret_cast<uint32_t*>(stg + (size_t)r * P + (size_t)j * 16);
      dst[0] = d.x ^ (sw & 0x80008000u);
      dst[1] = d.y ^ ((sw << 1) & 0x80008000u);
      dst[2] = d.z ^ ((sw << 2) & 0x80008000u);
      dst[3] = d.w ^ ((sw << 3) & 0x80008000u);
      j += dj;
      r += dr;
      if (j >= K8) {
        j -= K8;
        ++r;
      }
    }
    __syncthreads();
    if (*abort_flag) {
      // the rows of this group were the only copies in flight: let them land
      // (bounded) before the CTA's shared memory goes away
      if (threadIdx.x == 0) mbar_drain(full, it & 1, p.wait_ns);
      break;
    }
    // the landing buffer is free: the next group streams in behind this one
    if (threadIdx.x == 0 && g + (int)gridDim.x < p.ngroups) {
      fence_proxy_async_smem();
      issue_group(g + gridDim.x);
    }
    const int row = r0 + rl;
    const bool live = active && rl < nr && warp < nwarps;

    float v[SEG];
    if (DBL) {
      // ---------------------------------------------------------- first rotation
      // natural channel order: segment seg of the staged row, compile-time offsets
      if (live) {
        const uint16_t* src = reinterpret_cast<const uint16_t*>(stg + (size_t)rl * P) + seg * SEG;
#pragma unroll
        for (int e = 0; e < SEG; ++e) v[e] = bf16_bits_to_f32(src[e]);
      }
      fwht_seg<B, SEG>(v, part);
#pragma unroll
      for (int e = 0; e < SEG; e += 2) mul2s(v[e], v[e + 1], p.inv_sqrt_b);
      if (live) {
        float* dst = reinterpret_cast<float*>(y1 + (size_t)rl * P2) + seg * SEG;
#pragma unroll
        for (int e = 0; e < SEG; ++e) dst[e] = v[e];
      }
      __syncthreads();
    }
    // ------------------------------------------------------------ phase A
    if (live) {
      const uint32_t* tb = gtab + seg * TS;
      if (DBL) {
        const uint8_t* src = y1 + (size_t)rl * P2;
#pragma unroll
        for (int e4 = 0; e4 < SEG / 4; ++e4) {
          const uint4 t4 = *reinterpret_cast<const uint4*>(tb + 4 * e4);
          v[4 * e4] = *reinterpret_cast<const float*>(src + t4.x);
          v[4 * e4 + 1] = *reinterpret_cast<const float*>(src + t4.y);
          v[4 * e4 + 2] = *reinterpret_cast<const float*>(src + t4.z);
          v[4 * e4 + 3] = *reinterpret_cast<const float*>(src + t4.w);
        }
      } else {
        const uint8_t* src = stg + (size_t)rl * P;
#pragma unroll
        for (int e4 = 0; e4 < SEG / 4; ++e4) {
          const uint4 t4 = *reinterpret_cast<const uint4*>(tb + 4 * e4);
          v[4 * e4] = bf16_bits_to_f32(*reinterpret_cast<const uint16_t*>(src + t4.x));
          v[4 * e4 + 1] = bf16_bits_to_f32(*reinterpret_cast<const uint16_t*>(src + t4.y));
          v[4 * e4 + 2] = bf16_bits_to_f32(*reinterpret_cast<const uint16_t*>(src + t4.z));
          v[4 * e4 + 3] = bf16_bits_to_f32(*reinterpret_cast<const uint16_t*>(src + t4.w));
        }
      }
    }
    fwht_seg<B, SEG>(v, part);
#pragma unroll
    for (int e = 0; e < SEG; e += 2) mul2s(v[e], v[e + 1], p.inv_sqrt_b);

    // per-row partials: sums of squares per block, or this warp's maximum (and
    // minimum) over the row's segments
    if constexpr (FMT == RQ_FMT_LM16 || FMT == RQ_FMT_LM4) {
      // blocks up to 128: their trees straight to the partials; larger blocks:
      // the 128-wide subtrees added across the block's threads (xor 1, 2, 4)
      // (a thread that is not live passes block width 0: nothing is written)
      float ss = SqTree<SEG, 0, SEG>::run(v, (live && B <= SEG) ? B : 0, pt + rl * pstride + seg * NBT);
#pragma unroll
      for (int m = 1; m < T; m <<= 1) ss = __fadd_rn(ss, __shfl_xor_sync(0xffffffffu, ss, m));
      if (B > SEG && live && part == 0) pt[rl * pstride + seg / T] = ss;
    } else if constexpr (WEIGHT && FMT == RQ_FMT_INT4) {
      // one scale per 128 rotated coordinates (this thread's own segment); the
      // group's scale x code sum goes to the partials for the row's sum over
      // groups (the zero-point term of asymmetric activations)
      if (live) {
        float amax = 0.f;
#pragma unroll
        for (int e = 0; e < SEG; ++e) amax = fmaxf(amax, fabsf(v[e]));
        const float inv = amax > 0.f ? __fdiv_rn(7.0f, amax) : 0.f;
        int csum = 0;
#pragma unroll
        for (int e = 0; e < SEG; ++e)
          csum += (int)(__float_as_uint(__fadd_rn(__fmul_rn(v[e], inv), 12582912.0f)) - 0x4B400000u);
        const float sc = amax > 0.f ? __fdiv_rn(amax, 7.0f) : 0.f;
        pt[rl * pstride + seg * NPART] = __fmul_rn(sc, (float)csum);
      }
    } else {
      float mx = 0.f, mn = 0.f;
      if constexpr (FMT == RQ_FMT_INT4A) {
        mx = v[0];
        mn = v[0];
#pragma unroll
        for (int e = 1; e < SEG; ++e) {
          mx = fmaxf(mx, v[e]);
          mn = fminf(mn, v[e]);
        }
      } else {
#pragma unroll
        for (int e = 0; e < SEG; ++e) mx = fmaxf(mx, fabsf(v[e]));
      }
      if (!live) { mx = -INFINITY; mn = INFINITY; }
#pragma unroll
      for (int m = 1; m < 32; m <<= 1) {
        if (m < F) {
          mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, m));
          if constexpr (FMT == RQ_FMT_INT4A) mn = fminf(mn, __shfl_xor_sync(0xffffffffu, mn, m));
        }
      }
      if (lane % F == 0 && rl < nr && warp < nwarps) {
        pt[rl * pstride + warp * NPART] = mx;
        if constexpr (FMT == RQ_FMT_INT4A) pt[rl * pstride + warp * NPART + 1] = mn;
      }
    }
    __syncthreads();

    // ------------------------------------------------------------ phase B
    if (!live) continue;
    float mlt;
    float zpt = 0.f;
    if constexpr (FMT == RQ_FMT_LM16 || FMT == RQ_FMT_LM4) {
      // the row's sum of squares: block partials added in block order
      const float* pr = pt + rl * pstride;
      float ss = pr[0];
      for (int j = 1; j < nblk; ++j) ss = __fadd_rn(ss, pr[j]);
      const float nrm = __fsqrt_rn(ss);
      mlt = nrm > 0.f ? __fdiv_rn(p.sqrtK, nrm) : 0.f;
      if (seg == 0) p.scale[row] = nrm > 0.f ? __fdiv_rn(nrm, p.sqrtK) : 0.f;
    } else if constexpr (WEIGHT && FMT == RQ_FMT_INT4) {
      // one scale per 128 rotated coordinates: this thread's own segment
      float amax = 0.f;
#pragma unroll
      for (int e = 0; e < SEG; ++e) amax = fmaxf(amax, fabsf(v[e]));
      mlt = amax > 0.f ? __fdiv_rn(7.0f, amax) : 0.f;
      p.scale[(size_t)seg * p.rows + row] = amax > 0.f ? __fdiv_rn(amax, 7.0f) : 0.f;
      if (p.wz && seg == 0) {   // sum over the row's groups, in group order
        const float* pr = pt + rl * pstride;
        float z = pr[0];
        for (int s2 = 1; s2 < S; ++s2) z = __fadd_rn(z, pr[s2 * NPART]);
        p.wz[row] = z;
      }
    } else {
      const float* pr = pt + rl * pstride;
      float amax = pr[0], amin = 0.f;
      if constexpr (FMT == RQ_FMT_INT4A) amin = pr[1];
      for (int w = 1; w < nwarps; ++w) {
        amax = fmaxf(amax, pr[w * NPART]);
        if constexpr (FMT == RQ_FMT_INT4A) amin = fminf(amin, pr[w * NPART + 1]);
      }
      if constexpr (FMT == RQ_FMT_INT4) {
        mlt = amax > 0.f ? __fdiv_rn(7.0f, amax) : 0.f;
        if (seg == 0) p.scale[row] = amax > 0.f ? __fdiv_rn(amax, 7.0f) : 0.f;
      } else if constexpr (FMT == RQ_FMT_INT8) {
        mlt = amax > 0.f ? __fdiv_rn(127.0f, amax) : 0.f;
        if (seg == 0) p.scale[row] = amax > 0.f ? __fdiv_rn(amax, 127.0f) : 0.f;
      } else if constexpr (FMT == RQ_FMT_NVFP4) {
        mlt = amax > 0.f ? __fdiv_rn(2688.0f, amax) : 0.f;
        if (seg == 0) p.scale[row] = amax > 0.f ? __fdiv_rn(amax, 2688.0f) : 0.f;
      } else {   // INT4A: range [min, max] onto 0..15
        const float rng = __fsub_rn(amax, amin);
        mlt = rng > 0.f ? __fdiv_rn(15.0f, rng) : 0.f;
        zpt = rng > 0.f ? rintf(__fmul_rn(amin, mlt)) : 0.f;
        if (seg == 0) {
          p.scale[row] = rng > 0.f ? __fdiv_rn(rng, 15.0f) : 0.f;
          p.zp[row] = __fadd_rn(zpt, 8.0f);
        }
      }
    }

    // ------------------------------------------------------------ quantize + pack
    if constexpr (FMT == RQ_FMT_INT8) {
      // one byte per code (two's complement), 32 codes per pair of 16-byte stores
      uint4* dst = reinterpret_cast<uint4*>(p.codes + (size_t)row * K + (size_t)seg * SEG);
#pragma unroll
      for (int c = 0; c < SEG / 32; ++c) {
        uint32_t w[8];
#pragma unroll
        for (int j = 0; j < 8; ++j) w[j] = 0u;
#pragma unroll
        for (int e = 0; e < 32; ++e) {
          // |v * inv| <= 127 (+ rounding): the 1.5 * 2^23 add rounds to nearest even
          const uint32_t b = __float_as_uint(__fadd_rn(__fmul_rn(v[32 * c + e], mlt), 12582912.0f));
          w[e >> 2] |= (b & 0xFFu) << (8 * (e & 3));
        }
        dst[2 * c] = make_uint4(w[0], w[1], w[2], w[3]);
        dst[2 * c + 1] = make_uint4(w[4], w[5], w[6], w[7]);
      }
    } else if constexpr (FMT == RQ_FMT_INT4 || FMT == RQ_FMT_INT4A) {
      uint32_t pk[SEG / 8];
#pragma unroll
      for (int w = 0; w < SEG / 8; ++w) pk[w] = 0u;
      if constexpr (FMT == RQ_FMT_INT4) {
#pragma unroll
        for (int e = 0; e < SEG; ++e) {
          // round to nearest even by the 1.5 * 2^23 add; |v * inv| <= 7 (+ rounding)
          const uint32_t b = __float_as_uint(__fadd_rn(__fmul_rn(v[e], mlt), 12582912.0f));
          pk[e >> 3] |= (b & 0xFu) << (4 * (e & 7));
        }
      } else {
#pragma unroll
        for (int e = 0; e < SEG; ++e) {
          float q = __fsub_rn(rintf(__fmul_rn(v[e], mlt)), zpt);
          q = fminf(fmaxf(q, 0.f), 15.f);
          const uint32_t b = (uint32_t)((int)q - 8);
          pk[e >> 3] |= (b & 0xFu) << (4 * (e & 7));
        }
      }
      uint4* dst = reinterpret_cast<uint4*>(p.codes + (size_t)row * (K / 2) + (size_t)seg * (SEG / 2));
#pragma unroll
      for (int c = 0; c < SEG / 32; ++c) dst[c] = make_uint4(pk[4 * c], pk[4 * c + 1], pk[4 * c + 2], pk[4 * c + 3]);
    } else if constexpr (FMT == RQ_FMT_LM16 || FMT == RQ_FMT_LM4) {
      // t = u * 2^s, exactly 2^s * fp32(v * inv) (the scaling is exact): the
      // cell of t and one compare against the cell's scaled boundary
      const float mlt_s = __fmul_rn(mlt, __int_as_float((127 + p.lut_shift) << 23));
      const uint32_t gbias = 0x4B400000u + (uint32_t)p.lut_gmin;
      const uint32_t nmax = (uint32_t)p.lut_n - 1u;
      constexpr int NW32 = FMT == RQ_FMT_LM16 ? SEG / 8 : SEG / 16;
      uint32_t pk[NW32];
#pragma unroll
      for (int w = 0; w < NW32; ++w) pk[w] = 0u;
#pragma unroll
      for (int e = 0; e < SEG; ++e) {
        const float t = __fmul_rn(v[e], mlt_s);
        const uint32_t cell = min((uint32_t)__float_as_int(__fadd_rd(t, 12582912.0f)) - gbias, nmax);
        const uint2 cv = lut_s[cell];
        const uint32_t d = (t >= __uint_as_float(cv.y)) ? (cv.x >> 8) : (cv.x & 0xFFu);
        if constexpr (FMT == RQ_FMT_LM16) {
          pk[e >> 3] |= d << (4 * (e & 7));
        } else {   // nibble e%8 of word e/16 holds elements e%8 (bits 0-1) and e%8+8 (bits 2-3)
          pk[e >> 4] |= d << (4 * (e & 7) + 2 * ((e >> 3) & 1));
        }
      }
      if constexpr (FMT == RQ_FMT_LM16) {
        uint4* dst = reinterpret_cast<uint4*>(p.codes + (size_t)row * (K / 2) + (size_t)seg * (SEG / 2));
#pragma unroll
        for (int c = 0; c < SEG / 32; ++c) dst[c] = make_uint4(pk[4 * c], pk[4 * c + 1], pk[4 * c + 2], pk[4 * c + 3]);
      } else {
        uint4* dst = reinterpret_cast<uint4*>(p.codes + (size_t)row * (K / 4) + (size_t)seg * (SEG / 4));
#pragma unroll
        for (int c = 0; c < SEG / 64; ++c) dst[c] = make_uint4(pk[4 * c], pk[4 * c + 1], pk[4 * c + 2], pk[4 * c + 3]);
      }
    } else {   // NVFP4: SEG / 16 groups of 16 elements
      uint32_t pk[SEG / 8];
      uint32_t sbw[2] = {0u, 0u};
#pragma unroll
      for (int gq = 0; gq < SEG / 16; ++gq) {
        float* u = v + 16 * gq;
        float m16 = 0.f;
#pragma unroll
        for (int e = 0; e < 16; e += 2) {
          mul2s(u[e], u[e + 1], mlt);
          m16 = fmaxf(m16, fmaxf(fabsf(u[e]), fabsf(u[e + 1])));
        }
        const float sbf = __fdiv_rn(m16, 6.0f);
        const uint32_t sb = cvt_e4m3x2(0.f, sbf) & 0xFFu;
        const float rcp = rcp_s[sb & 0x7Fu];
#pragma unroll
        for (int e = 0; e < 16; e += 8) {
          uint32_t w = 0u;
#pragma unroll
          for (int k = 0; k < 8; k += 2) {
            float a = u[e + k], b = u[e + k + 1];
            mul2s(a, b, rcp);
            const uint32_t byte = sb ? (uint32_t)cvt_e2m1x2(b, a) : 0u;
            w |= byte << (4 * k);
          }
          pk[2 * gq + (e >> 3)] = w;
        }
        sbw[gq >> 2] |= sb << (8 * (gq & 3));
      }
      uint4* dst = reinterpret_cast<uint4*>(p.codes + (size_t)row * (K / 2) + (size_t)seg * (SEG / 2));
#pragma unroll
      for (int c = 0; c < SEG / 32; ++c) dst[c] = make_uint4(pk[4 * c], pk[4 * c + 1], pk[4 * c + 2], pk[4 * c + 3]);
      // block scales kb .. kb+3 (kb % 4 == 0) are four adjacent bytes of the tile layout
      const int kb = seg * (SEG / 16);
      *reinterpret_cast<uint32_t*>(p.bscale + sf_off(row, kb, K)) = sbw[0];
      if constexpr (SEG == 128) *reinterpret_cast<uint32_t*>(p.bscale + sf_off(row, kb + 4, K)) = sbw[1];
    }
  }
}

// ------------------------------------------------------------------ host side
size_t k1r_smem(int RW, int K, int S, int ts, bool dbl, int nblk, int nwarps, int npart, int lut_n) {
  size_t off = (size_t)RW * K * 2 + (size_t)RW * (2 * K + 4) + (dbl ? (size_t)RW * (4 * K + 4) : 0);
  off = (off + 15) & ~(size_t)15;
  off += (size_t)S * ts * 4;
  off += (size_t)(K / 8) * 4;
  off += (size_t)2 * RW * (nblk > S ? nblk : S) * npart * 4;
  off = (off + 15) & ~(size_t)15;
  return off + 16 + 512 + (size_t)lut_n * 8;
}

float e4m3_val(int c) {
  const int e = (c >> 3) & 15, m = c & 7;
  return e == 0 ? std::ldexp((float)m, -9) : std::ldexp(1.0f + m / 8.0f, e - 7);
}

// The codebook cells: the coarsest width 2^-s whose cells hold at most one
// boundary, covering |u| <= sqrt(K) (u = y sqrt(K) / ||y|| cannot leave it, up
// to rounding, hence the margin) so that one clamp suffices.  Entry: the code
// of the cell's lower part (bits 0-7), of its upper part (bits 8-15) and the
// cell's boundary scaled by 2^s (+inf if none).  16-level codes are stored
// sign-magnitude: c - 8 for c >= 8, (7 - c) | 8 below.
bool build_cells(K1RParams& p, const float* bnd, int nbnd, int K, bool sign_magnitude) {
  const double lim = std::sqrt((double)K) * 1.001 + 1.0;
  for (int shift = 0; shift <= 14; ++shift) {
    long cell[15];
    bool ok = true;
    for (int i = 0; i < nbnd; ++i) {
      cell[i] = (long)std::floor(std::ldexp((double)bnd[i], shift));   // exact
      if (i > 0 && cell[i] <= cell[i - 1]) ok = false;
    }
    if (!ok) continue;
    const long gmin = std::min((long)std::floor(-std::ldexp(lim, shift)), cell[0]) - 1;
    const long gmax = std::max((long)std::floor(std::ldexp(lim, shift)), cell[nbnd - 1]) + 1;
    if (gmax - gmin + 1 > R_LUT_MAX) return false;
    p.lut_shift = shift;
    p.lut_gmin = (int32_t)gmin;
    p.lut_n = (int32_t)(gmax - gmin + 1);
    auto sm = [](uint32_t c) { return c >= 8 ? c - 8 : (7 - c) | 8u; };
    for (long g = gmin; g <= gmax; ++g) {
      uint32_t base = 0, b = 0x7f800000u;   // no boundary in the cell: +inf
      for (int i = 0; i < nbnd; ++i) {
        if (cell[i] < g) ++base;
        if (cell[i] == g) {
          const float bs = std::ldexp(bnd[i], shift);   // exact
          std::memcpy(&b, &bs, 4);
        }
      }
      const uint32_t hi = base + 1 <= (uint32_t)nbnd ? base + 1 : (uint32_t)nbnd;
      const uint32_t lo_c = sign_magnitude ? sm(base) : base, hi_c = sign_magnitude ? sm(hi) : hi;
      p.lut[g - gmin] = make_uint2(lo_c | (hi_c << 8), b);
    }
    return true;
  }
  return false;
}

template <int FMT, bool WEIGHT, int B, int SEG>
cudaError_t launch_r(const K1Launch& a, cudaStream_t st) {
  constexpr int T = B > SEG ? B / SEG : 1;
  K1RParams p{};
  p.x = a.x;
  p.rot = a.rot;
  p.rot2 = a.rot2;
  p.codes = a.codes;
  p.scale = a.scale;
  p.zp = a.zp;
  p.wz = a.wz;
  p.bscale = a.bscale;
  p.status = a.status;
  p.wait_ns = a.wait_ns;
  p.inject_tx = a.inject_tx;
  p.rows = a.rows;
  p.K = a.K;
  p.B = a.block;
  p.dbl = a.rot2 != nullptr;
  p.inv_sqrt_b = a.inv_sqrt_b;
  p.sqrtK = a.sqrtK;
  p.lut_n = 0;
  if constexpr (FMT == RQ_FMT_LM16 || FMT == RQ_FMT_LM4) {
    if (a.nbnd < 1 || !build_cells(p, a.bnd, a.nbnd, a.K, FMT == RQ_FMT_LM16)) return cudaErrorInvalidValue;
  }
  for (int c = 0; c < 128; ++c) p.rcp_e4m3[c] = (c == 0 || c == 0x7F) ? 0.f : 1.0f / e4m3_val(c);
  // F (segments per warp): the fewest that keep the warps at most 12 and the
  // shared-memory plan within 227 KB, and at least the threads of one block
  // (K = 12288 with blocks of 256: two rows of 16 segments per warp)
  const int S = a.K / SEG;
  const int npart = (FMT == RQ_FMT_LM16 || FMT == RQ_FMT_LM4) ? 1 : 2;
  int F = 0;
  size_t smem = 0;
  for (int f = 1; f <= 16; f *= 2) {
    const int nw = (S + f - 1) / f;
    const size_t sm = k1r_smem(32 / f, a.K, S, SEG + 4, p.dbl != 0, a.K / a.block, nw, npart, p.lut_n);
    if (f >= T && nw <= R_THREADS / 32 && sm <= 232448) {
      F = f;
      smem = sm;
      break;
    }
  }
  if (F == 0) return cudaErrorInvalidValue;
  p.F = F;
  p.R = 32 / F;
  p.ngroups = (a.rows + p.R - 1) / p.R;
  const int nwarps = (S + F - 1) / F;
  auto kern = k1r_kernel<FMT, WEIGHT, B, SEG>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  const int sms = a.num_sms > 0 ? a.num_sms : 148;
  const int grid = p.ngroups < sms ? p.ngroups : sms;
  kern<<<grid, nwarps * 32, smem, st>>>(p);
  return cudaGetLastError();
}

}  // namespace

bool k1r_supports(const K1Launch& a) {
  if (a.U) return false;
  if (a.K % 64) return false;
  // 64-wide segments: codebook and NVFP4 codes with blocks up to 64, one rotation
  if (a.K % 128 && (a.block > 64 || a.rot2 || a.wz ||
                    (a.fmt != RQ_FMT_LM16 && a.fmt != RQ_FMT_LM4 && a.fmt != RQ_FMT_NVFP4)))
    return false;
  if (a.rot2 && a.K > 8192) return false;   // the FP32 row copy of the double rotation
  switch (a.block) {
    case 16: case 32: case 64: case 128: case 256: case 512: case 1024: return true;
  }
  return false;
}

namespace {
// rows whose K is an odd multiple of 64 (blocks up to 64): 64-wide segments
template <int BS>
cudaError_t launch_r_t64(const K1Launch& a, cudaStream_t st) {
  if constexpr (BS <= 64) {
    switch (a.fmt) {
      case RQ_FMT_LM16: return a.weight ? launch_r<RQ_FMT_LM16, true, BS, 64>(a, st) : launch_r<RQ_FMT_LM16, false, BS, 64>(a, st);
      case RQ_FMT_LM4: return a.weight ? launch_r<RQ_FMT_LM4, true, BS, 64>(a, st) : cudaErrorInvalidValue;
      case RQ_FMT_NVFP4: return a.weight ? launch_r<RQ_FMT_NVFP4, true, BS, 64>(a, st) : launch_r<RQ_FMT_NVFP4, false, BS, 64>(a, st);
    }
  }
  return cudaErrorInvalidValue;
}

template <int BS>
cudaError_t launch_r_t(const K1Launch& a, cudaStream_t st) {
  if (a.K % 128) return launch_r_t64<BS>(a, st);
  if (a.weight) {
    switch (a.fmt) {
      case RQ_FMT_INT4: return launch_r<RQ_FMT_INT4, true, BS, 128>(a, st);
      case RQ_FMT_LM16: return launch_r<RQ_FMT_LM16, true, BS, 128>(a, st);
      case RQ_FMT_LM4: return launch_r<RQ_FMT_LM4, true, BS, 128>(a, st);
      case RQ_FMT_NVFP4: return launch_r<RQ_FMT_NVFP4, true, BS, 128>(a, st);
    }
    return cudaErrorInvalidValue;
  }
  switch (a.fmt) {
    case RQ_FMT_INT4: return launch_r<RQ_FMT_INT4, false, BS, 128>(a, st);
    case RQ_FMT_INT4A: return launch_r<RQ_FMT_INT4A, false, BS, 128>(a, st);
    case RQ_FMT_INT8: return launch_r<RQ_FMT_INT8, false, BS, 128>(a, st);
    case RQ_FMT_LM16: return launch_r<RQ_FMT_LM16, false, BS, 128>(a, st);
    case RQ_FMT_NVFP4: return launch_r<RQ_FMT_NVFP4, false, BS, 128>(a, st);
  }
  return cudaErrorInvalidValue;
}
}  // namespace

cudaError_t launch_k1r(const K1Launch& a, cudaStream_t st) {
  switch (a.block) {
    case 16: return launch_r_t<16>(a, st);
    case 32: return launch_r_t<32>(a, st);
    case 64: return launch_r_t<64>(a, st);
    case 128: return launch_r_t<128>(a, st);
    case 256: return launch_r_t<256>(a, st);
    case 512: return launch_r_t<512>(a, st);
    case 1024: return launch_r_t<1024>(a, st);
  }
  return cudaErrorInvalidValue;
}

}  // namespace rq
