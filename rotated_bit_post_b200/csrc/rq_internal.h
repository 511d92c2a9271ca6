// Internal launch descriptors shared by the C-ABI layer and the kernels.
#pragma once
#include <cuda_runtime.h>

#include <cstdint>

#define RQ_FMT_INT4 1
#define RQ_FMT_LM16 2
#define RQ_FMT_NVFP4 3
#define RQ_FMT_LM4 4
#define RQ_FMT_INT4A 5
#define RQ_FMT_INT8 6

namespace rq {

struct K1Launch {
  int fmt;
  int weight;              // 1: weight rows (INT4 per-128-group scales, L = W U)
  const uint16_t* x;
  int rows, K, block;
  const int32_t* rot;
  const int32_t* rot2;     // double rotation: the second rotation's table, or null
  float inv_sqrt_b, sqrtK;
  int nbnd;
  const float* bnd;        // host, nbnd entries
  const uint16_t* U;
  int r;
  uint16_t* coef;
  uint8_t* codes;
  float* scale;
  float* zp;               // asymmetric INT4: per-row zero point
  float* wz;               // INT4 weights: per-row sum over groups of scale x code sum (or null)
  uint8_t* bscale;
  int32_t* status;
  int num_sms;
  uint64_t wait_ns;        // bounded-wait limit of every mbarrier wait
  uint32_t inject_tx;      // test hook: extra expect-tx bytes on the first load (0: off)
};

cudaError_t launch_k1(const K1Launch& a, cudaStream_t st);
// the rows-as-lanes activation kernel (every case without the projection)
bool k1r_supports(const K1Launch& a);
cudaError_t launch_k1r(const K1Launch& a, cudaStream_t st);

struct GemmLaunch {
  int a_fmt, w_fmt;
  int M, N, K;
  const uint8_t* a_codes;
  const float* a_scale;
  const uint8_t* a_bscale;
  const uint8_t* w_codes;
  const float* w_scale;
  const uint8_t* w_bscale;
  uint8_t a_lut[16];       // e4m3 bytes per code (FP8 path)
  uint8_t w_lut[16];
  const float* a_zp;       // asymmetric INT4 activations: per-token zero point (or null)
  const float* w_zsum;     // with a_zp: per weight row, sum_g s_w[g, n] * sum_{k in g} q_w[n, k]
  const uint16_t* c;       // M x r BF16 (low-rank branch) or null
  const uint16_t* L;       // N x r BF16
  int r;
  void* Y;
  int out_fp32;
  int32_t* status;
  int num_sms;
  uint64_t wait_ns;
  uint32_t inject_tx;
};

cudaError_t launch_gemm(const GemmLaunch& a, cudaStream_t st, const char** why);
// W8A8: 8-bit per-token activations x 8-bit per-channel weights (no expansion)
cudaError_t launch_gemm_w8a8(const GemmLaunch& a, cudaStream_t st);

// DiRotQ full PCA rotation: y = x V (FP32, into the caller's workspace), then
// the first r coordinates to BF16 and the rest to INT4.
struct PcaLaunch {
  int weight;              // 1: weight rows (one INT4 scale per 128 coordinates)
  const uint16_t* x;       // rows x K BF16
  const uint16_t* vt;      // K x K BF16, row n = column n of V
  int rows, K, r;
  float* y;                // rows x K FP32 workspace
  uint16_t* coef;          // rows x r BF16
  uint8_t* codes;          // rows x K/2
  float* scale;            // rows (activations) or K/128 x rows (weights)
  int32_t* status;
  int num_sms;
  uint64_t wait_ns;
};

cudaError_t launch_pca(const PcaLaunch& a, cudaStream_t st);

}  // namespace rq
