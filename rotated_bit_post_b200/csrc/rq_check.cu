// Verification entry points (include/rq_check.h): the device conversions of
// the activation kernel, launched on their own.
#include <cuda_runtime.h>

#include <cstdint>

#include "../../include/rq_check.h"
#include "rq_ptx.cuh"

namespace rq {
namespace {

// One pair (in[2i], in[2i+1]) per thread: the same cvt_e4m3x2 / cvt_e2m1x2
// helpers K1 calls, with the even element in the low half of each result.
__global__ void convert_check_kernel(const float* __restrict__ in, int npairs, uint8_t* __restrict__ e4m3,
                                     uint8_t* __restrict__ e2m1) {
  for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < npairs; i += gridDim.x * blockDim.x) {
    const float lo = in[2 * i], hi = in[2 * i + 1];
    const uint16_t e8 = cvt_e4m3x2(hi, lo);
    const uint8_t e4 = cvt_e2m1x2(hi, lo);
    e4m3[2 * i] = (uint8_t)(e8 & 0xFF);
    e4m3[2 * i + 1] = (uint8_t)(e8 >> 8);
    e2m1[2 * i] = e4 & 0xF;
    e2m1[2 * i + 1] = e4 >> 4;
  }
}

}  // namespace
}  // namespace rq

extern "C" rq_status rq_convert_check(const float* in, int32_t n, uint8_t* e4m3, uint8_t* e2m1, void* stream) {
  if (n < 0 || (n & 1)) return RQ_ERR_INVALID_ARG;
  if (n == 0) return RQ_OK;
  if (!in || !e4m3 || !e2m1) return RQ_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(in) | reinterpret_cast<uintptr_t>(e4m3) | reinterpret_cast<uintptr_t>(e2m1)) & 15)
    return RQ_ERR_ALIGNMENT;
  const int npairs = n / 2;
  int grid = (npairs + 255) / 256;
  if (grid > 4096) grid = 4096;
  rq::convert_check_kernel<<<grid, 256, 0, static_cast<cudaStream_t>(stream)>>>(in, npairs, e4m3, e2m1);
  return cudaGetLastError() == cudaSuccess ? RQ_OK : RQ_ERR_CUDA;
}
