// C ABI of the rotated W4A4 linear layer (declared in include/rq.h): argument
// checking, host-side table preparation and kernel dispatch.
#include <cuda_runtime.h>

#include <atomic>
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <mutex>
#include <vector>

#include "../../include/rq.h"
#include "../../include/rq_check.h"
#include "rq_host.h"
#include "rq_internal.h"

// The workspace of rq_pca_rotate_quantize_act_noalloc: a static device array
// (one per GPU that loads the library, held until the process exits).  In
// host code `g_noalloc_scratch` names the host-side stand-in of the symbol,
// not a device address: the address is looked up once per device, on first
// use, with that device current (noalloc_scratch below).
static __device__ __align__(256) float g_noalloc_scratch[RQ_NOALLOC_MAX_ELEMS];

namespace {

thread_local char g_err[512] = "";

// Bounded-wait limit of the kernels and the fault-injection test hook
// (include/rq_check.h); read at every launch.
constexpr uint64_t kDefaultWaitNs = 2000000000ull;   // 2 s: far above any legitimate wait
std::atomic<uint64_t> g_wait_ns{kDefaultWaitNs};
std::atomic<uint32_t> g_inject_tx{0};

rq_status fail(rq_status s, const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_err, sizeof(g_err), fmt, ap);
  va_end(ap);
  return s;
}

rq_status ok() {
  g_err[0] = 0;
  return RQ_OK;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int num_sms() {
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 148;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) return 148;
  return n;
}

rq_status check_rows_call(int32_t fmt, bool weight, const void* X, int32_t rows, int32_t K, int32_t block,
                          const int32_t* rot, const float* boundaries, const uint16_t* U, int32_t r,
                          const void* coef, const void* codes, const void* scale, const void* bscale,
                          const int32_t* rot2 = nullptr, const void* zp = nullptr) {
  const bool fmt_ok = fmt == RQ_INT4 || fmt == RQ_LM16 || fmt == RQ_NVFP4 || fmt == RQ_INT8 ||
                      (weight && fmt == RQ_LM4) || (!weight && fmt == RQ_INT4A);
  if (!fmt_ok) return fail(RQ_ERR_INVALID_ARG, "unknown or unsupported format %d", fmt);
  if (rows < 0 || K <= 0) return fail(RQ_ERR_INVALID_ARG, "bad shape rows=%d K=%d", rows, K);
  if (block < 16 || block > 1024 || (block & (block - 1)))
    return fail(RQ_ERR_UNSUPPORTED, "block %d: a power of two from 16 to 1024", block);
  if (U && block != 128 && block != 256 && block != 512)
    return fail(RQ_ERR_UNSUPPORTED, "block %d with the low-rank branch: 128, 256 or 512", block);
  if (K % block) return fail(RQ_ERR_INVALID_ARG, "K=%d is not a multiple of block=%d", K, block);
  if (K > 16384) return fail(RQ_ERR_UNSUPPORTED, "K=%d exceeds 16384", K);
  // codebook and NVFP4 rows need K % 64 (their packed rows stay whole 16-byte
  // units for the GEMM's tensor maps); INT4 groups, 8-bit codes, the low-rank
  // branch and the double rotation need K % 128
  const bool k64 = (fmt == RQ_LM16 || fmt == RQ_LM4 || fmt == RQ_NVFP4) && !U && !rot2;
  if (K % (k64 ? 64 : 128)) return fail(RQ_ERR_INVALID_ARG, "K=%d must be a multiple of %d", K, k64 ? 64 : 128);
  if (fmt == RQ_NVFP4 && U && K % 256) return fail(RQ_ERR_INVALID_ARG, "NVFP4 with the low-rank branch needs K %% 256 == 0 (K=%d)", K);
  if (rot2 && U) return fail(RQ_ERR_UNSUPPORTED, "the double rotation runs without the low-rank branch");
  if (rot2 && K > 8192) return fail(RQ_ERR_UNSUPPORTED, "the double rotation supports K <= 8192 (got %d)", K);
  if (fmt == RQ_INT4A && !zp) return fail(RQ_ERR_INVALID_ARG, "asymmetric INT4 needs a zero-point output");
  if ((fmt == RQ_INT4A || fmt == RQ_INT8) && U) return fail(RQ_ERR_UNSUPPORTED, "format %d runs without the low-rank branch", fmt);
  if ((rot2 && !aligned16(rot2)) || (zp && !aligned16(zp))) return fail(RQ_ERR_ALIGNMENT, "rot2 / zero point not 16-byte aligned");
  if (!X || !rot || !codes || !scale) return fail(RQ_ERR_INVALID_ARG, "null input/output pointer");
  if ((fmt == RQ_LM16 || fmt == RQ_LM4) && !boundaries)
    return fail(RQ_ERR_INVALID_ARG, "codebook format needs boundaries");
  if (fmt == RQ_NVFP4 && !bscale) return fail(RQ_ERR_INVALID_ARG, "NVFP4 needs block_scale");
  if (U) {
    if (r < 8 || r > 32 || r % 8)
      return fail(RQ_ERR_UNSUPPORTED, "low-rank branch supports r in {8, 16, 24, 32} (got %d)", r);
    if (K > 3072) return fail(RQ_ERR_UNSUPPORTED, "low-rank branch supports K <= 3072 (got %d)", K);
    if (!coef) return fail(RQ_ERR_INVALID_ARG, "U given without a coefficient output");
    if (!aligned16(U) || !aligned16(coef)) return fail(RQ_ERR_ALIGNMENT, "U / coefficient output not 16-byte aligned");
  }
  if (!aligned16(X) || !aligned16(rot) || !aligned16(codes) || !aligned16(scale) || (bscale && !aligned16(bscale)))
    return fail(RQ_ERR_ALIGNMENT, "device pointers must be 16-byte aligned");
  return RQ_OK;
}

rq_status run_k1(int32_t fmt, bool weight, const uint16_t* X, int32_t rows, int32_t K, int32_t block,
                 const int32_t* rot, const float* boundaries, const uint16_t* U, int32_t r, uint16_t* coef,
                 uint8_t* codes, float* scale, uint8_t* bscale, int32_t* status, void* stream,
                 const int32_t* rot2 = nullptr, float* zp = nullptr, float* wz = nullptr) {
  rq_status s =
      check_rows_call(fmt, weight, X, rows, K, block, rot, boundaries, U, r, coef, codes, scale, bscale, rot2, zp);
  if (s != RQ_OK) return s;
  if (rows == 0) return ok();
  rq::K1Launch a{};
  a.fmt = fmt;
  // INT8 weight rows (per output channel) take the per-token quantizer as is
  a.weight = weight && fmt != RQ_INT8 ? 1 : 0;
  a.x = X;
  a.rows = rows;
  a.K = K;
  a.block = block;
  a.rot = rot;
  a.rot2 = rot2;
  a.zp = zp;
  a.wz = wz;
  a.inv_sqrt_b = (float)(1.0 / std::sqrt((double)block));
  a.sqrtK = std::sqrt((float)K);
  a.nbnd = fmt == RQ_LM16 ? 15 : fmt == RQ_LM4 ? 3 : 0;
  if (a.nbnd) {   // the boundaries must ascend
    for (int i = 1; i < a.nbnd; ++i)
      if (!(boundaries[i] > boundaries[i - 1])) return fail(RQ_ERR_INVALID_ARG, "codebook boundaries must ascend");
  }
  a.bnd = boundaries;
  a.U = U;
  a.r = U ? r : 0;
  a.coef = coef;
  a.codes = codes;
  a.scale = scale;
  a.bscale = bscale;
  a.status = status;
  a.num_sms = num_sms();
  a.wait_ns = g_wait_ns.load();
  a.inject_tx = g_inject_tx.load();
  cudaError_t e = rq::launch_k1(a, static_cast<cudaStream_t>(stream));
  if (e == cudaErrorInvalidValue)   // no kernel configuration fits this format, K and block
    return fail(RQ_ERR_UNSUPPORTED, "format %d with K=%d, block=%d: no kernel configuration fits", fmt, K, block);
  if (e != cudaSuccess) return fail(RQ_ERR_CUDA, "rotate/quantize launch failed: %s", cudaGetErrorString(e));
  return ok();
}

constexpr int kMaxDevices = 64;
std::once_flag g_noalloc_once[kMaxDevices];
float* g_noalloc_ptr[kMaxDevices];
cudaError_t g_noalloc_err[kMaxDevices];

rq_status noalloc_scratch(float** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return fail(RQ_ERR_CUDA, "cudaGetDevice failed: %s", cudaGetErrorString(e));
  if (dev < 0 || dev >= kMaxDevices) return fail(RQ_ERR_UNSUPPORTED, "device %d beyond %d", dev, kMaxDevices);
  std::call_once(g_noalloc_once[dev], [dev] {
    void* p = nullptr;
    g_noalloc_err[dev] = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    g_noalloc_ptr[dev] = g_noalloc_err[dev] == cudaSuccess ? static_cast<float*>(p) : nullptr;
  });
  if (g_noalloc_err[dev] != cudaSuccess || !g_noalloc_ptr[dev])
    return fail(RQ_ERR_CUDA, "workspace address lookup failed on device %d: %s", dev,
                cudaGetErrorString(g_noalloc_err[dev]));
  *out = g_noalloc_ptr[dev];
  return RQ_OK;
}

}  // namespace

extern "C" {

const char* rq_last_error(void) { return g_err; }

rq_status rq_make_rotation(int32_t K, int32_t block, uint64_t seed, int8_t* sign, int32_t* perm, int32_t* rot) {
  if (K <= 0 || block < 2 || (block & (block - 1)) || K % block)
    return fail(RQ_ERR_INVALID_ARG, "K=%d must be a positive multiple of a power-of-two block (block=%d)", K, block);
  rq::make_rotation(K, seed, sign, perm, rot);
  return ok();
}

rq_status rq_make_zigzag(const float* channel_mag, int32_t K, int32_t block, int32_t* perm, int32_t* rot2) {
  if (!channel_mag || (!perm && !rot2)) return fail(RQ_ERR_INVALID_ARG, "null pointer");
  if (K <= 0 || block < 1 || K % block) return fail(RQ_ERR_INVALID_ARG, "K=%d must be a multiple of block=%d", K, block);
  for (int i = 0; i < K; ++i)
    if (!(channel_mag[i] >= 0.f)) return fail(RQ_ERR_INVALID_ARG, "channel magnitudes must be finite and >= 0");
  rq::make_zigzag(channel_mag, K, block, perm, rot2);
  return ok();
}

rq_status rq_make_codebook(int32_t K, int32_t levels, double* centroids, double* boundaries, float* boundaries_f32,
                           uint8_t* centroids_e4m3) {
  if (K < 4) return fail(RQ_ERR_INVALID_ARG, "K=%d too small", K);
  if (levels != 4 && levels != 16) return fail(RQ_ERR_UNSUPPORTED, "levels=%d (4 or 16)", levels);
  std::vector<double> c, b;
  if (!rq::lloyd_max(K, levels, c, b)) return fail(RQ_ERR_INVALID_ARG, "Lloyd iteration did not converge");
  for (int i = 0; i < levels; ++i) {
    if (centroids) centroids[i] = c[i];
    if (centroids_e4m3) centroids_e4m3[i] = rq::e4m3_encode((double)(float)c[i]);
  }
  for (int i = 0; i < levels - 1; ++i) {
    if (boundaries) boundaries[i] = b[i];
    if (boundaries_f32) boundaries_f32[i] = (float)b[i];
  }
  return ok();
}

rq_status rq_pca_basis(const uint16_t* calib, int32_t n, int32_t K, int32_t r, uint16_t* U, double* eigenvalues) {
  if (!calib || !U) return fail(RQ_ERR_INVALID_ARG, "null pointer");
  if (r < 1 || r > 64 || n < r || K < r) return fail(RQ_ERR_INVALID_ARG, "bad PCA shape n=%d K=%d r=%d", n, K, r);
  if (!rq::pca_basis(calib, n, K, r, U, eigenvalues))
    return fail(RQ_ERR_INVALID_ARG, "calibration tokens have rank below r");
  return ok();
}

rq_status rq_rotate_quantize_act(int32_t fmt, const uint16_t* X, int32_t M, int32_t K, int32_t block,
                                 const int32_t* rot, const float* boundaries, const uint16_t* U, int32_t r,
                                 uint16_t* c_out, uint8_t* codes, float* scale, uint8_t* block_scale,
                                 int32_t* status, void* stream) {
  return run_k1(fmt, false, X, M, K, block, rot, boundaries, U, r, c_out, codes, scale, block_scale, status, stream);
}

rq_status rq_quantize_weights(int32_t fmt, const uint16_t* W, int32_t N, int32_t K, int32_t block,
                              const int32_t* rot, const float* boundaries, const uint16_t* U, int32_t r,
                              uint16_t* L_out, uint8_t* codes, float* scale, uint8_t* block_scale,
                              int32_t* status, void* stream) {
  return run_k1(fmt, true, W, N, K, block, rot, boundaries, U, r, L_out, codes, scale, block_scale, status, stream);
}

rq_status rq_rotate_quantize_act2(int32_t fmt, const uint16_t* X, int32_t M, int32_t K, int32_t block,
                                  const int32_t* rot, const int32_t* rot2, const float* boundaries, uint8_t* codes,
                                  float* scale, float* zero_point, uint8_t* block_scale, int32_t* status,
                                  void* stream) {
  return run_k1(fmt, false, X, M, K, block, rot, boundaries, nullptr, 0, nullptr, codes, scale, block_scale, status,
                stream, rot2, zero_point, nullptr);
}

rq_status rq_quantize_weights2(int32_t fmt, const uint16_t* W, int32_t N, int32_t K, int32_t block,
                               const int32_t* rot, const int32_t* rot2, const float* boundaries, uint8_t* codes,
                               float* scale, uint8_t* block_scale, float* zsum, int32_t* status, void* stream) {
  if (zsum && fmt != RQ_INT4) return fail(RQ_ERR_INVALID_ARG, "code sums are an output of INT4 weights");
  if (zsum && !aligned16(zsum)) return fail(RQ_ERR_ALIGNMENT, "zsum not 16-byte aligned");
  return run_k1(fmt, true, W, N, K, block, rot, boundaries, nullptr, 0, nullptr, codes, scale, block_scale, status,
                stream, rot2, nullptr, zsum);
}

static rq_status pca_impl(bool weight, const uint16_t* X, int32_t rows, int32_t K, const uint16_t* Vt, int32_t r,
                          float* workspace, uint16_t* coef, uint8_t* codes, float* scale, int32_t* status,
                          void* stream) {
  if (rows < 0 || K <= 0 || K % 128 || K > 16384)
    return fail(RQ_ERR_INVALID_ARG, "bad PCA shape rows=%d K=%d (K %% 128 == 0, K <= 16384)", rows, K);
  if (r < 0 || r > K) return fail(RQ_ERR_INVALID_ARG, "r=%d outside 0..K", r);
  if (!X || !Vt || !workspace || !codes || !scale || (r > 0 && !coef))
    return fail(RQ_ERR_INVALID_ARG, "null input/output pointer");
  if (!aligned16(X) || !aligned16(Vt) || !aligned16(workspace) || !aligned16(codes) || !aligned16(scale))
    return fail(RQ_ERR_ALIGNMENT, "device pointers must be 16-byte aligned");
  if (rows == 0) return ok();
  rq::PcaLaunch a{};
  a.weight = weight ? 1 : 0;
  a.x = X;
  a.vt = Vt;
  a.rows = rows;
  a.K = K;
  a.r = r;
  a.y = workspace;
  a.coef = coef;
  a.codes = codes;
  a.scale = scale;
  a.status = status;
  a.num_sms = num_sms();
  a.wait_ns = g_wait_ns.load();
  cudaError_t e = rq::launch_pca(a, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return fail(RQ_ERR_CUDA, "PCA rotation launch failed: %s", cudaGetErrorString(e));
  return ok();
}

rq_status rq_pca_rotate_quantize_act(const uint16_t* X, int32_t M, int32_t K, const uint16_t* Vt, int32_t r,
                                     float* workspace, uint16_t* c_out, uint8_t* codes, float* scale,
                                     int32_t* status, void* stream) {
  return pca_impl(false, X, M, K, Vt, r, workspace, c_out, codes, scale, status, stream);
}

rq_status rq_pca_quantize_weights(const uint16_t* W, int32_t N, int32_t K, const uint16_t* Vt, int32_t r,
                                  float* workspace, uint16_t* L_out, uint8_t* codes, float* scale,
                                  int32_t* status, void* stream) {
  return pca_impl(true, W, N, K, Vt, r, workspace, L_out, codes, scale, status, stream);
}

rq_status rq_pca_rotate_quantize_act_noalloc(const uint16_t* X, int32_t M, int32_t K, const uint16_t* Vt, int32_t r,
                                             uint16_t* c_out, uint8_t* codes, float* scale, int32_t* status,
                                             void* stream) {
  if (M < 0 || K <= 0 || (int64_t)M * K > RQ_NOALLOC_MAX_ELEMS)
    return fail(RQ_ERR_INVALID_ARG, "M x K = %lld exceeds the built-in workspace of %d FP32 values",
                (long long)M * K, RQ_NOALLOC_MAX_ELEMS);
  float* ws = nullptr;
  const rq_status s = noalloc_scratch(&ws);
  if (s != RQ_OK) return s;
  return pca_impl(false, X, M, K, Vt, r, ws, c_out, codes, scale, status, stream);
}

static rq_status linear_impl(int32_t a_fmt, int32_t w_fmt, int32_t M, int32_t N, int32_t K, const uint8_t* a_codes,
                             const float* a_scale, const uint8_t* a_bscale, const float* a_zp, const uint8_t* w_codes,
                             const float* w_scale, const uint8_t* w_bscale, const float* w_zsum,
                             const uint8_t* a_lut, const uint8_t* w_lut, const uint16_t* c, const uint16_t* L,
                             int32_t r, void* Y, int32_t out_fp32, int32_t* status, void* stream);

rq_status rq_w4a4_linear(int32_t a_fmt, int32_t w_fmt, int32_t M, int32_t N, int32_t K, const uint8_t* a_codes,
                         const float* a_scale, const uint8_t* a_bscale, const uint8_t* w_codes,
                         const float* w_scale, const uint8_t* w_bscale, const uint8_t* a_lut,
                         const uint8_t* w_lut, const uint16_t* c, const uint16_t* L, int32_t r, void* Y,
                         int32_t out_fp32, int32_t* status, void* stream) {
  if (a_fmt == RQ_INT4A) return fail(RQ_ERR_UNSUPPORTED, "asymmetric activations go through rq_w4a4_linear2");
  return linear_impl(a_fmt, w_fmt, M, N, K, a_codes, a_scale, a_bscale, nullptr, w_codes, w_scale, w_bscale, nullptr,
                     a_lut, w_lut, c, L, r, Y, out_fp32, status, stream);
}

rq_status rq_w4a4_linear2(int32_t M, int32_t N, int32_t K, const uint8_t* a_codes, const float* a_scale,
                          const float* a_zero_point, const uint8_t* w_codes, const float* w_scale,
                          const float* w_zsum, void* Y, int32_t out_fp32, int32_t* status, void* stream) {
  if (!a_zero_point || !w_zsum) return fail(RQ_ERR_INVALID_ARG, "zero points and weight code sums are required");
  if (!aligned16(a_zero_point) || !aligned16(w_zsum)) return fail(RQ_ERR_ALIGNMENT, "zero point / code sums not 16-byte aligned");
  return linear_impl(RQ_INT4A, RQ_INT4, M, N, K, a_codes, a_scale, nullptr, a_zero_point, w_codes, w_scale, nullptr,
                     w_zsum, nullptr, nullptr, nullptr, nullptr, 0, Y, out_fp32, status, stream);
}

static rq_status linear_impl(int32_t a_fmt, int32_t w_fmt, int32_t M, int32_t N, int32_t K, const uint8_t* a_codes,
                             const float* a_scale, const uint8_t* a_bscale, const float* a_zp, const uint8_t* w_codes,
                             const float* w_scale, const uint8_t* w_bscale, const float* w_zsum,
                             const uint8_t* a_lut, const uint8_t* w_lut, const uint16_t* c, const uint16_t* L,
                             int32_t r, void* Y, int32_t out_fp32, int32_t* status, void* stream) {
  const bool pair_ok = (a_fmt == RQ_INT4 && w_fmt == RQ_INT4) || (a_fmt == RQ_INT4A && w_fmt == RQ_INT4) ||
                       (a_fmt == RQ_INT8 && w_fmt == RQ_INT4) || (a_fmt == RQ_INT8 && w_fmt == RQ_INT8) ||
                       (a_fmt == RQ_LM16 && w_fmt == RQ_LM16) ||
                       (a_fmt == RQ_LM16 && w_fmt == RQ_LM4) || (a_fmt == RQ_NVFP4 && w_fmt == RQ_NVFP4);
  if (!pair_ok) return fail(RQ_ERR_UNSUPPORTED, "format pair (%d, %d) not supported", a_fmt, w_fmt);
  if (M < 0 || N <= 0 || K <= 0) return fail(RQ_ERR_INVALID_ARG, "bad shape M=%d N=%d K=%d", M, N, K);
  if (w_fmt == RQ_INT4 && N % 4)   // the group scales of a tile are copied 16 bytes at a time
    return fail(RQ_ERR_INVALID_ARG, "INT4 weights need N %% 4 == 0 (N=%d)", N);
  // codebook and NVFP4 codes: K % 64 (a ragged last K step issues only its
  // MMAs inside K); INT4 and 8-bit weights: whole 128-wide groups
  const bool k64 = a_fmt == RQ_LM16 || a_fmt == RQ_NVFP4;
  if (K % (k64 ? 64 : 128)) return fail(RQ_ERR_INVALID_ARG, "K=%d must be a multiple of %d", K, k64 ? 64 : 128);
  if (!a_codes || !a_scale || !w_codes || !w_scale || !Y) return fail(RQ_ERR_INVALID_ARG, "null pointer");
  if (a_fmt == RQ_NVFP4 && (!a_bscale || !w_bscale)) return fail(RQ_ERR_INVALID_ARG, "NVFP4 needs block scales");
  if (a_fmt == RQ_LM16 && (!a_lut || !w_lut)) return fail(RQ_ERR_INVALID_ARG, "codebook formats need LUTs");
  if ((c != nullptr) != (L != nullptr)) return fail(RQ_ERR_INVALID_ARG, "c and L must both be given or both NULL");
  // 16-level codes are stored sign-magnitude: the GEMM reads the upper half of
  // the table and takes the lower half as its mirror image
  auto symmetric16 = [](const uint8_t* lut) {
    for (int m = 0; m < 8; ++m)
      if (lut[7 - m] != (uint8_t)(lut[8 + m] | 0x80u)) return false;
    return true;
  };
  if (a_fmt == RQ_LM16 && !symmetric16(a_lut))
    return fail(RQ_ERR_UNSUPPORTED, "16-level activation table is not symmetric (entry 7-m must be -(entry 8+m))");
  if (w_fmt == RQ_LM16 && !symmetric16(w_lut))
    return fail(RQ_ERR_UNSUPPORTED, "16-level weight table is not symmetric (entry 7-m must be -(entry 8+m))");
  if (c && (r < 8 || r > 32 || r % 8))
    return fail(RQ_ERR_UNSUPPORTED, "low-rank branch supports r in {8, 16, 24, 32} (got %d)", r);
  if (c && (a_fmt == RQ_INT8 || a_fmt == RQ_INT4A))
    return fail(RQ_ERR_UNSUPPORTED, "the low-rank branch runs with 4-bit activations");
  const void* ptrs[] = {a_codes, a_scale, w_codes, w_scale, Y, a_bscale, w_bscale, c, L};
  for (const void* q : ptrs)
    if (q && !aligned16(q)) return fail(RQ_ERR_ALIGNMENT, "device pointers must be 16-byte aligned");
  if (M == 0) return ok();
  rq::GemmLaunch g{};
  g.a_fmt = a_fmt == RQ_INT4A ? RQ_INT4 : a_fmt;   // the same signed-nibble GEMM, plus the zero-point term
  g.w_fmt = w_fmt;
  g.M = M;
  g.N = N;
  g.K = K;
  g.a_codes = a_codes;
  g.a_scale = a_scale;
  g.a_bscale = a_bscale;
  g.w_codes = w_codes;
  g.w_scale = w_scale;
  g.w_bscale = w_bscale;
  g.a_zp = a_zp;
  g.w_zsum = w_zsum;
  if (a_fmt == RQ_INT4 || a_fmt == RQ_INT4A || a_fmt == RQ_INT8) {
    for (int i = 0; i < 16; ++i) {
      const int v = i < 8 ? i : i - 16;  // two's-complement nibble
      g.a_lut[i] = g.w_lut[i] = rq::e4m3_encode((double)v);
    }
  } else if (a_fmt == RQ_LM16) {
    std::memcpy(g.a_lut, a_lut, 16);
    std::memcpy(g.w_lut, w_lut, w_fmt == RQ_LM4 ? 4 : 16);
  }
  g.c = c;
  g.L = L;
  g.r = c ? r : 0;
  g.Y = Y;
  g.out_fp32 = out_fp32 ? 1 : 0;
  g.status = status;
  g.num_sms = num_sms();
  g.wait_ns = g_wait_ns.load();
  g.inject_tx = g_inject_tx.load();
  const char* why = nullptr;
  cudaError_t e = a_fmt == RQ_INT8 && w_fmt == RQ_INT8 ? rq::launch_gemm_w8a8(g, static_cast<cudaStream_t>(stream))
                                                       : rq::launch_gemm(g, static_cast<cudaStream_t>(stream), &why);
  if (e != cudaSuccess)
    return fail(RQ_ERR_CUDA, "GEMM launch failed: %s%s%s", cudaGetErrorString(e), why ? " / " : "", why ? why : "");
  return ok();
}

rq_status rq_set_wait_limit(uint64_t limit_ns, uint64_t* previous) {
  if (limit_ns == 0) limit_ns = kDefaultWaitNs;
  if (limit_ns > 20000000000ull) return fail(RQ_ERR_INVALID_ARG, "wait limit above 20 s");
  const uint64_t old = g_wait_ns.exchange(limit_ns);
  if (previous) *previous = old;
  return ok();
}

rq_status rq_set_fault_injection(uint32_t extra_tx_bytes) {
  if (extra_tx_bytes % 16 || extra_tx_bytes > 4096)
    return fail(RQ_ERR_INVALID_ARG, "extra bytes must be a multiple of 16 and at most 4096");
  g_inject_tx.store(extra_tx_bytes);
  return ok();
}

rq_status rq_read_status(const int32_t* status, void* stream, int32_t* code_out) {
  if (!status) return fail(RQ_ERR_INVALID_ARG, "null status");
  cudaError_t e = cudaStreamSynchronize(static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return fail(RQ_ERR_CUDA, "stream sync failed: %s", cudaGetErrorString(e));
  int32_t v = 0;
  e = cudaMemcpy(&v, status, 4, cudaMemcpyDeviceToHost);
  if (e != cudaSuccess) return fail(RQ_ERR_CUDA, "status read failed: %s", cudaGetErrorString(e));
  if (code_out) *code_out = v;
  if (v == 0x201) return fail(RQ_ERR_CUDA, "a kernel found its shared memory misaligned (code 0x%x)", v);
  if (v != 0) return fail(RQ_ERR_TIMEOUT, "a kernel gave up a bounded wait (code 0x%x)", v);
  return ok();
}

}  // extern "C"
