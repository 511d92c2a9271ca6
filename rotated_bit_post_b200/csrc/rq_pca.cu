// DiRotQ's full PCA rotation (DiRotQ abstract: the activations rotated into a
// calibrated PCA basis, the coordinates of the dominant directions kept in
// BF16 and the remaining ones quantized to 4 bits, the inverse rotation folded
// into the weights offline).
//
// Two kernels:
//  * dense_gemm_kernel<false>: Y = X V, a dense K x K contraction on the
//    tensor cores (tcgen05.mma kind::f16, BF16 operands, FP32 accumulation in
//    TMEM), TMA-fed, 128 x 256 tiles, persistent, double-buffered
//    accumulators; FP32 output to the caller's workspace.  The order of the
//    FP32 additions inside the tensor core is not specified, so this product
//    is held to an error bound, not to bit equality.
//    dense_gemm_kernel<true> is the same pipeline on 8-bit operands
//    (kind::i8, exact S32 accumulation) with a scaled epilogue: the W8A8 GEMM
//    (TR-DQ, Tables 1-5: 8-bit per-token activations against 8-bit
//    per-channel weights), Y = s_a[m] s_w[n] sum_k q_a q_w.
//  * pca_quant_kernel: per row, the first r coordinates rounded to BF16 (the
//    coefficients c, or L for weight rows), the others quantized to INT4
//    (symmetric, absmax per token; one scale per 128 coordinates for weight
//    rows), the first r positions carrying code 0 so that the 4-bit GEMM runs
//    over all K positions and c L^T adds them back.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cstdint>
#include <cstring>

#include "rq_internal.h"
#include "rq_ptx.cuh"

namespace rq {

namespace {

constexpr int PBM = 128, PROW = 128;   // tile rows; 128 bytes of K per row per stage
constexpr int P_THREADS = 256;         // warp 0 TMA, warp 1 MMA, warps 4-7 epilogue

// Shared-memory plan for BN output columns per tile (128 or 256): PSTAGES
// operand stages, then (FP32 output through TMA stores) four epilogue warps'
// two 4 KB staging boxes, then the barriers.
template <int BN>
struct DensePlan {
  static constexpr int PSTAGES = BN == 128 ? 5 : 4;
  static constexpr int PA_BYTES = PBM * PROW, PB_BYTES = BN * PROW;
  static constexpr int PSTAGE = PA_BYTES + PB_BYTES;
  static constexpr int OFF_STG = PSTAGES * PSTAGE;
  static constexpr int STG = 4 * 2 * 4096;
  static constexpr int OFF_BAR = OFF_STG + STG;
  static constexpr int NBAR = 2 * PSTAGES + 5;   // + the MMA drain barrier
  static constexpr int SMEM = OFF_BAR + NBAR * 8 + 16 + 1024;
  static_assert(SMEM <= 232448, "shared memory plan exceeds 227 KB");
};

struct __align__(64) DenseMaps {
  CUtensorMap a;   // [M][K] K-major: X (BF16) or the activation codes (int8)
  CUtensorMap b;   // [N][K] K-major: V^T (BF16, row n = column n of V) or the weight codes (int8)
  CUtensorMap y;   // FP32 output [M][N], 32 x 32 boxes, 128-byte swizzle (BF16 operands)
};

struct DenseParams {
  int M, N, K;         // K in elements
  void* Y;             // [M][N]: FP32 (BF16 operands), FP32 or BF16 (8-bit operands)
  int out_fp32;
  const float* sa;     // 8-bit operands: per-row scales of A [M] and of B [N]
  const float* sw;
  int32_t* status;
  uint64_t wait_ns;
};

// K-major A and B, N = BN, M = 128; BF16 operands with an F32 accumulator,
// or signed 8-bit operands with an S32 accumulator
template <bool S8, int BN>
__host__ __device__ constexpr uint32_t idesc_dense() {
  return (S8 ? (2u << 4) : (1u << 4)) | (1u << 7) | (1u << 10) | ((uint32_t)(BN >> 3) << 17) |
         ((uint32_t)(PBM >> 4) << 24);
}

template <bool S8, int PBN>
__global__ void __launch_bounds__(P_THREADS, 1) dense_gemm_kernel(const __grid_constant__ DenseMaps tm,
                                                                  const __grid_constant__ DenseParams p) {
  using L = DensePlan<PBN>;
  constexpr int PSTAGES = L::PSTAGES, PA_BYTES = L::PA_BYTES, PSTAGE = L::PSTAGE, P_NBAR = L::NBAR;
  constexpr int PBK = S8 ? 128 : 64;   // elements of K per stage
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
  const uint32_t sbase = smem_u32(smem);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::OFF_BAR);
  uint64_t* full = bars;
  uint64_t* empty = full + PSTAGES;
  uint64_t* accfull = empty + PSTAGES;   // [2]
  uint64_t* accempty = accfull + 2;      // [2]
  uint64_t* mdrain = accempty + 2;       // MMAs issued before an abort
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + P_NBAR);
  volatile int32_t* abort_flag = reinterpret_cast<volatile int32_t*>(tmem_slot + 1);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nk = p.K / PBK;
  const int nN = (p.N + PBN - 1) / PBN, nM = (p.M + PBM - 1) / PBM;
  const int ntiles = nM * nN;

  if (threadIdx.x == 0) {
    for (int i = 0; i < PSTAGES; ++i) { mbar_init(&full[i], 1); mbar_init(&empty[i], 1); }
    for (int i = 0; i < 2; ++i) { mbar_init(&accfull[i], 1); mbar_init(&accempty[i], 4); }
    mbar_init(mdrain, 1);
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
    if (lane == 0) {
      uint32_t kc = 0;
      for (int tile = blockIdx.x; tile < ntiles && !*abort_flag; tile += gridDim.x) {
        const int m0 = (tile / nN) * PBM, n0 = (tile % nN) * PBN;
        for (int kt = 0; kt < nk; ++kt, ++kc) {
          const int s = kc % PSTAGES;
          if (kc >= PSTAGES &&
              !mbar_wait(&empty[s], ((kc / PSTAGES) - 1) & 1, p.status, ST_TIMEOUT_EMPTY, abort_flag, p.wait_ns))
            break;
          mbar_expect_tx(&full[s], PSTAGE);
          tma_load_2d(smem + s * PSTAGE, &tm.a, kt * PBK, m0, &full[s]);
#pragma unroll
          for (int h = 0; h < PBN / 128; ++h)   // B in boxes of 128 rows
            tma_load_2d(smem + s * PSTAGE + PA_BYTES + h * 128 * PROW, &tm.b, kt * PBK, n0 + h * 128, &full[s]);
        }
      }
      if (*abort_flag)   // let the copies already issued land (bounded)
        for (uint32_t c = kc > (uint32_t)PSTAGES ? kc - PSTAGES : 0; c < kc; ++c)
          mbar_drain(&full[c % PSTAGES], (c / PSTAGES) & 1, p.wait_ns);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      uint32_t kc = 0;
      int tc = 0;
      bool ok = true;
      for (int tile = blockIdx.x; tile < ntiles && ok; tile += gridDim.x, ++tc) {
        const uint32_t ab = tc & 1;
        if (tc >= 2) {
          ok = mbar_wait(&accempty[ab], ((tc >> 1) - 1) & 1, p.status, ST_TIMEOUT_EPI, abort_flag, p.wait_ns);
          if (!ok) break;
          tc_fence_after();
        }
        for (int kt = 0; kt < nk; ++kt, ++kc) {
          const int s = kc % PSTAGES;
          ok = mbar_wait(&full[s], (kc / PSTAGES) & 1, p.status, ST_TIMEOUT_FULL, abort_flag, p.wait_ns);
          if (!ok) break;
          tc_fence_after();
          const uint32_t a = sbase + s * PSTAGE, b = a + PA_BYTES;
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) {   // 32 bytes of K per instruction along the swizzled row
            if constexpr (S8)
              umma_i8(tmem + ab * PBN, smem_desc(a + kk * 32, 16, 1024, 2), smem_desc(b + kk * 32, 16, 1024, 2),
                      idesc_dense<true, PBN>(), (kt > 0 || kk > 0) ? 1u : 0u);
            else
              umma_bf16(tmem + ab * PBN, smem_desc(a + kk * 32, 16, 1024, 2), smem_desc(b + kk * 32, 16, 1024, 2),
                        idesc_dense<false, PBN>(), (kt > 0 || kk > 0) ? 1u : 0u);
          }
          tc_commit(&empty[s]);
        }
        if (!ok) break;
        tc_commit(&accfull[ab]);
      }
      if (!ok) {
        tc_commit(mdrain);
        mbar_drain(mdrain, 0, p.wait_ns);
      }
    }
  } else if (warp >= 4) {
    const int q = warp & 3;
    const uint32_t lane_off = (uint32_t)(q * 32) << 16;
    const uint32_t stg = sbase + L::OFF_STG + (uint32_t)(warp - 4) * 8192u;   // two 4 KB boxes
    uint32_t stc = 0;   // boxes stored by this warp
    int tc = 0;
    bool ok = true;
    for (int tile = blockIdx.x; tile < ntiles && ok; tile += gridDim.x, ++tc) {
      const int m0 = (tile / nN) * PBM, n0 = (tile % nN) * PBN;
      const int row = m0 + q * 32 + lane;
      const uint32_t ab = tc & 1;
      ok = mbar_wait(&accfull[ab], (tc >> 1) & 1, p.status, ST_TIMEOUT_MMA, abort_flag, p.wait_ns);
      if (!ok) break;
      tc_fence_after();
      const float sa = S8 && row < p.M ? p.sa[row] : 0.f;
#pragma unroll 1
      for (int ch = 0; ch < PBN / 32; ++ch) {
        uint32_t v[32];
        tmem_ld32(tmem + lane_off + ab * PBN + ch * 32, v);
        tmem_ld_wait();
        const int n = n0 + ch * 32;
        if constexpr (S8) {
          if (row < p.M && n < p.N) {
            float y[32];
#pragma unroll
            for (int i = 0; i < 32; ++i)
              y[i] = __fmul_rn(__fmul_rn((float)(int32_t)v[i], sa), n + i < p.N ? __ldg(p.sw + n + i) : 0.f);
            // 16-byte stores where the chunk is whole and the rows aligned, element stores otherwise
            if (p.out_fp32) {
              float* dst = reinterpret_cast<float*>(p.Y) + (size_t)row * p.N + n;
              if (n + 32 <= p.N && (p.N & 3) == 0) {
#pragma unroll
                for (int i = 0; i < 32; i += 4)
                  *reinterpret_cast<float4*>(dst + i) = make_float4(y[i], y[i + 1], y[i + 2], y[i + 3]);
              } else {
#pragma unroll
                for (int i = 0; i < 32; ++i)
                  if (n + i < p.N) dst[i] = y[i];
              }
            } else {
              __nv_bfloat16* dst = reinterpret_cast<__nv_bfloat16*>(p.Y) + (size_t)row * p.N + n;
              if (n + 32 <= p.N && (p.N & 7) == 0) {
#pragma unroll
                for (int i = 0; i < 32; i += 8) {
                  __nv_bfloat162 h0 = __floats2bfloat162_rn(y[i], y[i + 1]), h1 = __floats2bfloat162_rn(y[i + 2], y[i + 3]);
                  __nv_bfloat162 h2 = __floats2bfloat162_rn(y[i + 4], y[i + 5]), h3 = __floats2bfloat162_rn(y[i + 6], y[i + 7]);
                  *reinterpret_cast<uint4*>(dst + i) =
                      make_uint4(*reinterpret_cast<uint32_t*>(&h0), *reinterpret_cast<uint32_t*>(&h1),
                                 *reinterpret_cast<uint32_t*>(&h2), *reinterpret_cast<uint32_t*>(&h3));
                }
              } else {
#pragma unroll
                for (int i = 0; i < 32; ++i)
                  if (n + i < p.N) dst[i] = __float2bfloat16_rn(y[i]);
              }
            }
          }
        } else {
          // FP32 through a 32 x 32 staging box (128-byte swizzle) and one TMA
          // store; rows >= M and columns >= N are clipped by the tensor map.
          // A box is rewritten only after the store two boxes back has read it.
          const uint32_t buf = stg + (stc & 1u) * 4096u;
          if (stc >= 2) {
            if (lane == 0) bulk_wait_group_read<1>();
            __syncwarp();
          }
#pragma unroll
          for (int i = 0; i < 8; ++i)
            asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(buf + lane * 128 + ((i ^ (lane & 7)) << 4)),
                         "r"(v[4 * i]), "r"(v[4 * i + 1]), "r"(v[4 * i + 2]), "r"(v[4 * i + 3])
                         : "memory");
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) {
            tma_store_2d(&tm.y, buf, n, m0 + q * 32);
            bulk_commit_group();
          }
          ++stc;
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&accempty[ab]);
    }
    if (lane == 0) bulk_wait_group<0>();   // the staging boxes outlive the stores that read them
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// One CTA per row: the first r coordinates to BF16, the rest to INT4 with
// per-token absmax (activations) or one scale per 128 coordinates (weights).
// The arithmetic of the quantizer is the FP32 contract of the activation
// kernel: inv = 7 / amax, q = rne(y inv), scale = amax / 7.
// One warp per row, eight rows per CTA: the first r coordinates to BF16, the
// rest to INT4 with per-token absmax (activations) or one scale per 128
// coordinates (weights).  The arithmetic of the quantizer is the FP32
// contract of the activation kernel: inv = 7 / amax, q = rne(y inv),
// scale = amax / 7.  A lane takes 8 consecutive coordinates (two 16-byte
// loads, one 32-bit word of codes), a warp 256 per step: two 128-wide groups,
// each held by 16 lanes.
constexpr int PQ_ROWS = 8;

template <bool WEIGHT>
__global__ void __launch_bounds__(32 * PQ_ROWS) pca_quant_kernel(const float* __restrict__ Y, int rows, int K, int r,
                                                                 uint16_t* __restrict__ coef,
                                                                 uint8_t* __restrict__ codes,
                                                                 float* __restrict__ scale) {
  const int lane = threadIdx.x & 31;
  const int row = blockIdx.x * PQ_ROWS + (threadIdx.x >> 5);
  if (row >= rows) return;
  const float* y = Y + (size_t)row * K;
  for (int j = lane; j < r; j += 32) coef[(size_t)row * r + j] = __bfloat16_as_ushort(__float2bfloat16_rn(y[j]));
  // 8 coordinates k0 .. k0+7 of this row, those below r read as 0
  auto load8 = [&](int k0, float (&v)[8]) {
    const float4 a = __ldg(reinterpret_cast<const float4*>(y + k0));
    const float4 b = __ldg(reinterpret_cast<const float4*>(y + k0 + 4));
    v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w; v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
    if (k0 < r) {
#pragma unroll
      for (int e = 0; e < 8; ++e)
        if (k0 + e < r) v[e] = 0.f;
    }
  };
  float inv_row = 0.f;
  if constexpr (!WEIGHT) {
    float m = 0.f;
    for (int k0 = lane * 8; k0 < K; k0 += 256) {
      float v[8];
      load8(k0, v);
#pragma unroll
      for (int e = 0; e < 8; ++e) m = fmaxf(m, fabsf(v[e]));
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    inv_row = m > 0.f ? __fdiv_rn(7.0f, m) : 0.f;
    if (lane == 0) scale[row] = m > 0.f ? __fdiv_rn(m, 7.0f) : 0.f;
  }
  // K % 128 == 0: every step covers whole groups, the lanes past K idle
  for (int base = 0; base < K; base += 256) {
    const int k0 = base + lane * 8;
    const bool live = k0 < K;
    float v[8];
    if (live) load8(k0, v);
    else {
#pragma unroll
      for (int e = 0; e < 8; ++e) v[e] = 0.f;
    }
    float inv = inv_row;
    if constexpr (WEIGHT) {
      // absmax of this lane's 128-wide group over its 16 lanes
      float m = 0.f;
#pragma unroll
      for (int e = 0; e < 8; ++e) m = fmaxf(m, fabsf(v[e]));
#pragma unroll
      for (int o = 8; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
      inv = m > 0.f ? __fdiv_rn(7.0f, m) : 0.f;
      if (live && (lane & 15) == 0) scale[(size_t)(k0 / 128) * rows + row] = m > 0.f ? __fdiv_rn(m, 7.0f) : 0.f;
    }
    if (live) {
      uint32_t w = 0u;
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        const uint32_t b = __float_as_uint(__fadd_rn(__fmul_rn(v[e], inv), 12582912.0f));
        w |= (b & 0xFu) << (4 * e);
      }
      *reinterpret_cast<uint32_t*>(codes + (size_t)row * (K / 2) + k0 / 2) = w;
    }
  }
}

typedef CUresult (*EncodeFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                             const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                             CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

// A K-major operand [outer][inner] of 2-byte (BF16) or 1-byte elements, 128-byte
// swizzle, boxes of 128 bytes of K by box_outer rows.
bool map_kmajor(CUtensorMap* m, const void* base, uint64_t inner, uint64_t outer, uint32_t box_outer, bool s8) {
  static EncodeFn fn = nullptr;
  if (!fn) {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      return false;
    fn = reinterpret_cast<EncodeFn>(f);
  }
  const uint64_t esz = s8 ? 1 : 2;
  cuuint64_t dims[2] = {inner, outer};
  cuuint64_t strides[1] = {inner * esz};
  cuuint32_t box[2] = {(cuuint32_t)(PROW / esz), box_outer};
  cuuint32_t es[2] = {1, 1};
  return fn(m, s8 ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims,
            strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <bool S8, int BN>
cudaError_t launch_dense_bn(const DenseMaps& tm, const DenseParams& p, int sms, cudaStream_t st) {
  constexpr int SMEM = DensePlan<BN>::SMEM;
  cudaError_t e = cudaFuncSetAttribute(dense_gemm_kernel<S8, BN>, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM);
  if (e != cudaSuccess) return e;
  const int ntiles = ((p.M + PBM - 1) / PBM) * ((p.N + BN - 1) / BN);
  dense_gemm_kernel<S8, BN><<<ntiles < sms ? ntiles : sms, P_THREADS, SMEM, st>>>(tm, p);
  return cudaGetLastError();
}

// 128 x 256 tiles, or 128 x 128 where the 256-wide tiles would leave the last
// round of the persistent loop mostly empty (e.g. 160 tiles on 148 SMs)
template <bool S8>
cudaError_t launch_dense(const DenseMaps& tm, const DenseParams& p, int num_sms, cudaStream_t st) {
  const int sms = num_sms > 0 ? num_sms : 148;
  const int mt = (p.M + PBM - 1) / PBM;
  const int t256 = mt * ((p.N + 255) / 256), t128 = mt * ((p.N + 127) / 128);
  const int r256 = (t256 + sms - 1) / sms, r128 = (t128 + sms - 1) / sms;   // rounds of the tile loop
  if (2 * r256 > r128 + 1) return launch_dense_bn<S8, 128>(tm, p, sms, st);
  return launch_dense_bn<S8, 256>(tm, p, sms, st);
}

bool map_y_f32(CUtensorMap* m, void* base, uint64_t cols, uint64_t rows) {
  static EncodeFn fn = nullptr;
  if (!fn) {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      return false;
    fn = reinterpret_cast<EncodeFn>(f);
  }
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {cols * 4};
  cuuint32_t box[2] = {32, 32};
  cuuint32_t es[2] = {1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, base, dims, strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE,
            CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) ==
         CUDA_SUCCESS;
}

}  // namespace

cudaError_t launch_gemm_w8a8(const GemmLaunch& a, cudaStream_t st) {
  DenseMaps tm;
  memset(&tm, 0, sizeof(tm));
  if (!map_kmajor(&tm.a, a.a_codes, a.K, a.M, PBM, true) || !map_kmajor(&tm.b, a.w_codes, a.K, a.N, 128, true))
    return cudaErrorInvalidValue;
  DenseParams p{a.M, a.N, a.K, a.Y, a.out_fp32, a.a_scale, a.w_scale, a.status, a.wait_ns};
  return launch_dense<true>(tm, p, a.num_sms, st);
}

cudaError_t launch_pca(const PcaLaunch& a, cudaStream_t st) {
  DenseMaps tm;
  memset(&tm, 0, sizeof(tm));
  // (the B box is 128 rows: the 256-wide tiles load it in two boxes)
  if (!map_kmajor(&tm.a, a.x, a.K, a.rows, PBM, false) || !map_kmajor(&tm.b, a.vt, a.K, a.K, 128, false) ||
      !map_y_f32(&tm.y, a.y, a.K, a.rows))
    return cudaErrorInvalidValue;
  DenseParams p{a.rows, a.K, a.K, a.y, 1, nullptr, nullptr, a.status, a.wait_ns};
  cudaError_t e = launch_dense<false>(tm, p, a.num_sms, st);
  if (e != cudaSuccess) return e;
  const int qgrid = (a.rows + PQ_ROWS - 1) / PQ_ROWS;
  if (a.weight)
    pca_quant_kernel<true><<<qgrid, 32 * PQ_ROWS, 0, st>>>(a.y, a.rows, a.K, a.r, a.coef, a.codes, a.scale);
  else
    pca_quant_kernel<false><<<qgrid, 32 * PQ_ROWS, 0, st>>>(a.y, a.rows, a.K, a.r, a.coef, a.codes, a.scale);
  return cudaGetLastError();
}

}  // namespace rq
