/*
 * rq.h -- C ABI of the rotated W4A4 linear layer for NVIDIA B200 (sm_100a).
 *
 * The layer is y = Q_a(R x) . Q_w(W R^T)^T (+ c . L^T):
 *   - R is a randomized permuted block-Hadamard (RPBH) rotation: random signs,
 *     one fixed permutation of the K input channels, then an orthonormal
 *     Walsh-Hadamard transform per block of `block` channels (OrbitQuant
 *     abstract, "randomized permuted block-Hadamard"; TR-DQ: Time-Rotation
 *     Diffusion Quantization, section 3.2, Eq. 8, block-diagonal rotation).
 *   - The weight side W R^T is folded and quantized offline, so the rotation
 *     cancels inside the layer and only R x runs online (OrbitQuant abstract;
 *     TR-DQ Eq. 9).
 *   - Q is one of: symmetric uniform INT4 (TR-DQ section 3.1, Eq. 1-3, absmax
 *     form), a Lloyd-Max codebook for the marginal of a rotated coordinate after
 *     per-token normalisation (OrbitQuant abstract), or NVFP4 (E2M1 elements with
 *     a UE4M3 scale per 16 elements; DiRotQ abstract, NVFP4 on Blackwell).
 *   - c . L^T is the optional DiRotQ low-rank branch: r PCA coefficients of the
 *     activation kept in BF16 (DiRotQ abstract).
 *
 * Conventions for every call
 *   - All buffers are owned by the caller.  No call allocates device memory or
 *     keeps a pointer after it returns.
 *   - "device" pointers must be device-accessible global memory of the current
 *     CUDA device, 16-byte aligned; "host" pointers are ordinary host memory
 *     read or written before the call returns.
 *   - Device work is enqueued on `stream` (a cudaStream_t, NULL = legacy default
 *     stream) and is asynchronous to the host.
 *   - BF16 tensors are passed as their 16-bit patterns (uint16_t).
 *   - Matrices are row-major.  Packed 4-bit codes store element 2j in bits 0-3
 *     and element 2j+1 in bits 4-7 of byte j of the row; packed 2-bit codes go 16
 *     to a little-endian 32-bit word, nibble i of word w holding element 16w+i in
 *     bits 0-1 and element 16w+8+i in bits 2-3.  A 16-level codebook code c
 *     (the count of boundaries at or below the value) is stored in its nibble
 *     sign-magnitude: c - 8 for c >= 8, (7 - c) | 8 below the centre.
 *   - Argument errors are detected on the host before anything is enqueued and
 *     return RQ_ERR_INVALID_ARG / RQ_ERR_UNSUPPORTED / RQ_ERR_ALIGNMENT with a
 *     message for rq_last_error().  A failed launch returns RQ_ERR_CUDA.
 *   - An empty batch (zero token rows, zero weight rows, M = 0) passes the same
 *     argument checks and returns RQ_OK without enqueuing anything.
 *   - `status` (device int32, caller-initialised to 0) receives a non-zero code
 *     if a kernel gave up a bounded wait (or could not start, see
 *     rq_read_status); read it back with rq_read_status().
 *     Kernels never wait without bound.
 */
#ifndef RQ_H_
#define RQ_H_

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef int32_t rq_status;
#define RQ_OK 0
#define RQ_ERR_INVALID_ARG 1
#define RQ_ERR_UNSUPPORTED 2
#define RQ_ERR_ALIGNMENT 3
#define RQ_ERR_CUDA 4
#define RQ_ERR_TIMEOUT 5

/* Quantization formats. */
#define RQ_INT4 1  /* symmetric INT4 in -7..7, two's-complement nibbles          */
#define RQ_LM16 2  /* 16-level Lloyd-Max codebook index, sign-magnitude nibbles   */
#define RQ_NVFP4 3 /* E2M1 nibbles + UE4M3 block scale per 16 + FP32 row scale    */
#define RQ_LM4 4   /* 4-level Lloyd-Max codebook index, 2-bit (weights only)       */
#define RQ_INT4A 5 /* asymmetric INT4 (activations only): nibble q - 8, per-token
                      scale s and zero point z + 8, x = s (nibble + zero point)  */
#define RQ_INT8 6  /* symmetric INT8 (W4A8 / W8A8 settings): one byte per code in
                      -127..127, scale amax/127 per token (activations) or per
                      output channel (weight rows)                              */

/*
 * rq_make_rotation -- host.  Draw the RPBH rotation for K channels.
 *   Source: OrbitQuant abstract ("randomized permuted block-Hadamard (RPBH)
 *   rotation"); TR-DQ section 3.2 (a permutation is an orthogonal matrix;
 *   Eq. 8 block-diagonal structure with K / block blocks).
 *   K      number of input channels, K % block == 0.
 *   block  Hadamard block size, a power of two, 16 <= block <= 1024 for the
 *          device calls (any power of two >= 2 here).
 *   seed   64-bit seed of the SplitMix64 stream: K sign draws first (negative
 *          when bit 63 is set), then a Fisher-Yates shuffle of 0..K-1 from the
 *          top index down with unbiased rejection draws.
 *   sign   [out, host, K] int8 +1/-1 per input channel (may be NULL).
 *   perm   [out, host, K] int32: output position i reads channel perm[i] (may be NULL).
 *   rot    [out, host, K] int32 signed permutation: bits 0-30 = perm[i], bit 31
 *          set when sign[perm[i]] < 0.  This is the table the device calls
 *          take (copy it to device memory).  May be NULL.
 *   R x is then y_i = (1/sqrt(block)) sum_j H[i mod block][j mod block]
 *   sign[perm[j]] x[perm[j]] over j in the block of i.
 */
rq_status rq_make_rotation(int32_t K, int32_t block, uint64_t seed, int8_t* sign, int32_t* perm, int32_t* rot);

/*
 * rq_make_zigzag -- host.  TR-DQ's zigzag permutation (TR-DQ section 3.2, the
 * paragraph before Eq. 9): channels ranked by magnitude (largest first; equal
 * magnitudes by channel index) are dealt to the K / block blocks back and
 * forth -- blocks 0, 1, ..., then ..., 1, 0, and so on -- and keep inside a
 * block the order in which they arrive.  For the double rotation R2 P R1 the
 * magnitudes are those of the channels after the first block rotation (for
 * example the maximum of |(x R1)_j| over calibration tokens).
 *   channel_mag  [in, host, K] finite, >= 0.   K % block == 0.
 *   perm   [out, host, K] int32: output position i reads channel perm[i] (may be NULL).
 *   rot2   [out, host, K] int32: the same as a signed permutation without
 *          signs, the table rq_rotate_quantize_act2 takes as `rot2` (may be NULL).
 */
rq_status rq_make_zigzag(const float* channel_mag, int32_t K, int32_t block, int32_t* perm, int32_t* rot2);

/*
 * rq_make_codebook -- host.  Lloyd-Max quantizer for the marginal of one
 * coordinate of a rotated row normalised to norm sqrt(K):
 * f(u) ~ (1 - u^2/K)^((K-3)/2) on |u| < sqrt(K) (OrbitQuant abstract: after RPBH
 * every coordinate follows one known marginal, so one Lloyd-Max codebook serves
 * all inputs of a given dimension).  FP64 Lloyd iteration (centroid = conditional
 * mean, boundary = midpoint) on the symmetric density until no value moves by
 * 1e-13.
 *   K       input dimension (>= 4).    levels  4 or 16.
 *   centroids       [out, host, levels] FP64, ascending (may be NULL)
 *   boundaries      [out, host, levels-1] FP64 (may be NULL)
 *   boundaries_f32  [out, host, levels-1] FP32 rounding of the boundaries: the
 *                   table the quantizer compares against (may be NULL)
 *   centroids_e4m3  [out, host, levels] E4M3 bytes of the FP32-rounded
 *                   centroids: the values the FP8 GEMM multiplies (may be NULL)
 */
rq_status rq_make_codebook(int32_t K, int32_t levels, double* centroids, double* boundaries,
                           float* boundaries_f32, uint8_t* centroids_e4m3);

/*
 * rq_pca_basis -- host.  Top-r eigenvectors of the uncentered second moment
 * X^T X / n of n calibration tokens (DiRotQ abstract: a low-rank subspace of
 * dominant activation variance via PCA), FP64 Jacobi eigen-solver on the n x n
 * Gram matrix, each vector's largest-magnitude entry made positive.
 *   calib  [in, host, n x K] BF16 bits.   n >= r, 1 <= r <= 64.
 *   U      [out, host, K x r] BF16 bits (column j = eigenvector j).
 *   eigenvalues [out, host, r] FP64, descending (may be NULL).
 */
rq_status rq_pca_basis(const uint16_t* calib, int32_t n, int32_t K, int32_t r, uint16_t* U, double* eigenvalues);

/*
 * rq_rotate_quantize_act -- device, async.  The online activation transform:
 * rotate each row of X with R, normalise per token, quantize, pack.
 * (OrbitQuant abstract: only a forward rotation on the activations remains at
 * run time; TR-DQ section 3.2: dynamic per-token ranges computed online.)
 *   fmt    RQ_INT4 | RQ_LM16 | RQ_NVFP4.
 *   X      [device, M x K] BF16.     M >= 1.  K % block == 0, K <= 16384;
 *          K % 64 == 0 for RQ_LM16 and RQ_NVFP4 (their packed rows stay whole
 *          16-byte units for the GEMM's tensor maps), K % 128 == 0 for RQ_INT4
 *          (weight groups of 128) and with U; with U: block 128, 256 or 512
 *          and, for NVFP4, K % 256 == 0.
 *   rot    [device, K] signed permutation from rq_make_rotation.
 *   boundaries [host, levels-1] FP32 codebook boundaries (RQ_LM16), else NULL.
 *   U, r   [device, K x r] BF16 PCA basis and its rank (r in {8, 16, 24, 32}, K <= 3072:
 *          U^T is staged whole in shared memory), or NULL / 0.
 *          With U: c = bf16(x U) (FP32: a sequential chain over each 128-channel
 *          chunk in k order, the chunk sums added in order) is written to c_out
 *          and the residual x - c U^T is what gets rotated and quantized.
 *   c_out  [device, M x r] BF16 or NULL.
 *   codes  [device, M x K/2] packed nibbles.
 *   scale  [device, M] FP32 per-token scale: amax/7 (INT4), ||y||/sqrt(K)
 *          (codebook), amax/2688 (NVFP4).
 *   block_scale [device] NVFP4 only: UE4M3 scale per 16 elements in 128-row x
 *          64-column tiles of 512 bytes, tile (mt, kt) at (mt*(K/64)+kt)*512, entry
 *          (m, kb) inside at (m%32)*16 + ((m%128)/32)*4 + kb%4; size
 *          ceil(M/128)*128*(K/16) bytes.  Padding rows are never read as data.
 *   status [device] int32 error word (see above).
 */
rq_status rq_rotate_quantize_act(int32_t fmt, const uint16_t* X, int32_t M, int32_t K, int32_t block,
                                 const int32_t* rot, const float* boundaries, const uint16_t* U, int32_t r,
                                 uint16_t* c_out, uint8_t* codes, float* scale, uint8_t* block_scale,
                                 int32_t* status, void* stream);

/*
 * rq_quantize_weights -- device, async.  Offline weight preparation: every row
 * w_n of W becomes R w_n (the row of W R^T) and is quantized with the same
 * procedure (OrbitQuant abstract: the same quantizer extended to weight rows,
 * the rotation absorbed into the weights).
 *   fmt    RQ_INT4 (one scale per 128 rotated coordinates) | RQ_LM16 | RQ_LM4 |
 *          RQ_NVFP4.
 *   W      [device, N x K] BF16.  K as for rq_rotate_quantize_act (RQ_LM4:
 *          K % 64 == 0).
 *   U, r, L_out  optional (r in {8, 16, 24, 32}, K <= 3072): L = bf16(W U) [device, N x r]
 *          (FP32, the same chunked order) for the low-rank branch
 *          (the full row is still what gets quantized).
 *   codes  [device, N x K/2] (RQ_LM4: N x K/4).
 *   scale  [device] RQ_INT4: [K/128][N] group-major; otherwise [N].
 *   block_scale  NVFP4 only, same layout as for activations with N rows.
 */
rq_status rq_quantize_weights(int32_t fmt, const uint16_t* W, int32_t N, int32_t K, int32_t block,
                              const int32_t* rot, const float* boundaries, const uint16_t* U, int32_t r,
                              uint16_t* L_out, uint8_t* codes, float* scale, uint8_t* block_scale,
                              int32_t* status, void* stream);

/*
 * rq_rotate_quantize_act2 -- device, async.  The activation transform without
 * the low-rank branch, with two additions (TR-DQ: Time-Rotation Diffusion
 * Quantization):
 *   - rot2 (optional, [device, K] signed permutation, from rq_make_zigzag):
 *     the double block rotation of section 3.2, Eq. 9, y = R2 P R1 x: R1 =
 *     the random signs of `rot` (its permutation must be the identity) and an
 *     orthonormal Walsh-Hadamard transform per natural block, P = rot2's
 *     permutation (its sign bits must be clear), R2 a second per-block
 *     transform; K <= 8192 (the kernel keeps the once-rotated row in shared
 *     memory as FP32).  Without rot2 the rotation is the one of `rot`, as in
 *     rq_rotate_quantize_act.
 *   - fmt RQ_INT8: 8-bit activations for the W4A8 setting (Tables 1-5): inv =
 *     127 / amax, q = clamp(rne(y inv), -127, 127), one byte per code (codes
 *     [device, M x K]), scale[m] = amax / 127.
 *   - fmt RQ_INT4A: asymmetric INT4 (section 3.1, Eq. 1-3, per token): inv =
 *     15 / (max - min), z = rne(min inv), q = clamp(rne(y inv) - z, 0, 15),
 *     nibble q - 8; scale[m] = (max - min) / 15 and zero_point[m] = z + 8
 *     ([device, M] FP32), so that x = scale (nibble + zero point).  A row with
 *     max == min gets scale 0, nibbles -8 and zero point 8.
 * Other arguments as rq_rotate_quantize_act; block: any power of two from 16
 * to 1024 dividing K.  zero_point is required for RQ_INT4A, else ignored.
 */
rq_status rq_rotate_quantize_act2(int32_t fmt, const uint16_t* X, int32_t M, int32_t K, int32_t block,
                                  const int32_t* rot, const int32_t* rot2, const float* boundaries, uint8_t* codes,
                                  float* scale, float* zero_point, uint8_t* block_scale, int32_t* status,
                                  void* stream);

/*
 * rq_quantize_weights2 -- device, async.  Weight preparation without the
 * low-rank branch, with the optional double rotation `rot2` (as above; the
 * rows of W are folded with the same R2 P R1) and, for INT4 weights, the
 * optional output zsum ([device, N] FP32): for each row n, the sum over its
 * 128-wide groups g, in group order, of scale[g, n] times the sum of the
 * group's codes.  rq_w4a4_linear2 takes it for the zero-point term of
 * asymmetric activations.  fmt RQ_INT8: 8-bit weights for the W8A8 setting
 * (TR-DQ: per-channel weight quantization), the per-token INT8 quantizer
 * applied to each rotated weight row (codes [device, N x K], scale [device,
 * N] = amax / 127).  Other arguments as rq_quantize_weights.
 */
rq_status rq_quantize_weights2(int32_t fmt, const uint16_t* W, int32_t N, int32_t K, int32_t block,
                               const int32_t* rot, const int32_t* rot2, const float* boundaries, uint8_t* codes,
                               float* scale, uint8_t* block_scale, float* zsum, int32_t* status, void* stream);

/*
 * rq_pca_rotate_quantize_act -- device, async.  DiRotQ's full PCA rotation
 * (DiRotQ abstract: activations rotated into a calibrated PCA basis, the
 * coordinates along the dominant directions kept in BF16, the rest quantized
 * to 4 bits; the inverse rotation folded into the weights offline):
 * y = x V on the tensor cores (BF16 operands, FP32 accumulation, order of the
 * additions not specified), then per row c = bf16(y[0:r]) and the INT4 codes
 * of y with its first r coordinates set to zero (codes 0 there): inv =
 * 7 / amax, q = rne(y inv), scale = amax / 7 over coordinates r..K-1.
 * rq_w4a4_linear(RQ_INT4, RQ_INT4, ..., c, L, r) then gives the layer output.
 *   X      [device, M x K] BF16.  M >= 0, K % 128 == 0, K <= 16384.
 *   Vt     [device, K x K] BF16, row n = column n of V (V orthogonal: the
 *          PCA basis of the calibration tokens, all K eigenvectors, dominant
 *          first).
 *   r      0 <= r <= K (the GEMM's low-rank term takes r in {8, 16, 24, 32}).
 *   workspace [device, M x K] FP32, caller-allocated scratch: y is written
 *          there (and may be read back; it is the rotated activation).
 *   c_out  [device, M x r] BF16 (may be NULL when r == 0).
 *   codes  [device, M x K/2] packed nibbles.  scale [device, M] FP32.
 *   All device pointers 16-byte aligned; status as above.
 */
rq_status rq_pca_rotate_quantize_act(const uint16_t* X, int32_t M, int32_t K, const uint16_t* Vt, int32_t r,
                                     float* workspace, uint16_t* c_out, uint8_t* codes, float* scale,
                                     int32_t* status, void* stream);

/*
 * rq_pca_quantize_weights -- device, async.  The weight side of the PCA
 * rotation: every row w_n becomes w_n V (x W^T = (x V)(W V)^T for orthogonal
 * V); L = bf16((W V)[:, 0:r]) and the INT4 codes of W V with its first r
 * coordinates zeroed, one scale per 128 coordinates ([K/128][N] group-major,
 * the layout rq_w4a4_linear reads).  Arguments as for the activations with
 * N rows; workspace [device, N x K] FP32.
 */
rq_status rq_pca_quantize_weights(const uint16_t* W, int32_t N, int32_t K, const uint16_t* Vt, int32_t r,
                                  float* workspace, uint16_t* L_out, uint8_t* codes, float* scale,
                                  int32_t* status, void* stream);

/*
 * rq_pca_rotate_quantize_act_noalloc -- device, async.  The paper has no
 * counterpart: this is rq_pca_rotate_quantize_act for callers that cannot
 * allocate device memory.  Such callers are, for example, extensions loaded
 * into a host framework that has reserved the GPU's memory through its own
 * caching allocator and passes them no allocator (a cudaMalloc there fails
 * once the pool holds the memory, or forces the framework to give back its
 * cache), and services that fix their memory budget at start-up and may not
 * allocate while serving.  They still pass every input and output buffer;
 * only the FP32 workspace is replaced.
 *
 * The workspace is a static device array of RQ_NOALLOC_MAX_ELEMS FP32 values
 * (16 MiB) inside the library: every GPU that loads the library holds it
 * until the process exits.  The first call on each device looks up the
 * array's device address on that device (cudaGetSymbolAddress) and keeps it;
 * make that first call before any stream capture.  The call allocates
 * nothing: no cudaMalloc, cudaFree or allocating library routine.
 *
 *   M * K must not exceed RQ_NOALLOC_MAX_ELEMS; a larger call returns
 *   RQ_ERR_INVALID_ARG and launches nothing.
 *   All calls share the one array, which keeps the last call's contents.
 *   Nothing in it needs to start at zero: the rotation writes every element
 *   that the split then reads.  Calls that overlap on the GPU (two streams,
 *   or two host threads, with no ordering between the calls) race on the
 *   array and give wrong results; order them on one stream.
 * Other arguments, results and errors as rq_pca_rotate_quantize_act, which
 * runs the same kernels.
 */
#define RQ_NOALLOC_MAX_ELEMS 4194304
rq_status rq_pca_rotate_quantize_act_noalloc(const uint16_t* X, int32_t M, int32_t K, const uint16_t* Vt, int32_t r,
                                             uint16_t* c_out, uint8_t* codes, float* scale, int32_t* status,
                                             void* stream);

/*
 * rq_w4a4_linear -- device, async.  The 4-bit x 4-bit GEMM on rotated codes with
 * per-token x per-group (INT4) or per-token x per-row scales, plus the optional
 * low-rank term (OrbitQuant abstract: the rotation cancels inside each linear
 * layer; DiRotQ abstract: a 4-bit GEMM plus a thin rank-r GEMM):
 *   Y[m, n] = a_scale[m] * sum_g w_scale[g, n] * sum_{k in g} a(m, k) w(n, k)
 *             + sum_j c[m, j] L[n, j]
 * with a(m,k), w(n,k) the dequantized code values (INT4 integers, E4M3 codebook
 * centroids, or E2M1 x UE4M3 block scale) and one group spanning all of K for
 * non-INT4 weights.
 *   a_fmt/w_fmt  (RQ_INT4, RQ_INT4) | (RQ_LM16, RQ_LM16) | (RQ_LM16, RQ_LM4) |
 *          (RQ_NVFP4, RQ_NVFP4) | (RQ_INT8, RQ_INT4): W4A8, 8-bit activation
 *          codes (from rq_rotate_quantize_act2) against INT4 weights |
 *          (RQ_INT8, RQ_INT8): W8A8, Y[m, n] = a_scale[m] w_scale[n] sum_k
 *          q_a q_w (exact integer sums), against weights from
 *          rq_quantize_weights2.  The 8-bit pairs run without the low-rank
 *          branch.
 *   a_codes/w_codes, a_scale/w_scale, a_bscale/w_bscale: as produced above.
 *   a_lut/w_lut  [host, 16 / 4 bytes] E4M3 value of each codebook index
 *          (rq_make_codebook's centroids_e4m3) for LM formats; NULL otherwise.
 *          Read during the argument checks.  A 16-entry table must be
 *          symmetric (entry 7-m = entry 8+m with the sign bit set), which the
 *          symmetric Lloyd-Max codebook is; otherwise RQ_ERR_UNSUPPORTED.
 *   c, L, r  [device] low-rank branch (r in {8, 16, 24, 32}; M x r and N x r BF16) or NULL / 0.
 *   Y      [device, M x N] FP32 (out_fp32 = 1) or BF16 (out_fp32 = 0).
 *   Shapes: M >= 0, N >= 1 (INT4 weights: N % 4 == 0, their group scales are
 *          copied 16 bytes at a time).  K % 64 == 0 for the codebook and NVFP4
 *          pairs (a last K step that is only partly inside K is zero-filled by
 *          the loads and only its MMAs inside K are issued); K % 128 == 0 when
 *          the weights are INT4 or INT8 (whole 128-wide groups).
 *          BF16 rows of Y go out through TMA stores when N % 8 == 0 (16-byte
 *          aligned rows) and through masked element stores otherwise.
 */
rq_status rq_w4a4_linear(int32_t a_fmt, int32_t w_fmt, int32_t M, int32_t N, int32_t K, const uint8_t* a_codes,
                         const float* a_scale, const uint8_t* a_bscale, const uint8_t* w_codes,
                         const float* w_scale, const uint8_t* w_bscale, const uint8_t* a_lut,
                         const uint8_t* w_lut, const uint16_t* c, const uint16_t* L, int32_t r, void* Y,
                         int32_t out_fp32, int32_t* status, void* stream);

/*
 * rq_w4a4_linear2 -- device, async.  The GEMM for asymmetric INT4 activations
 * (RQ_INT4A, from rq_rotate_quantize_act2) and INT4 weights (TR-DQ section
 * 3.1, Eq. 1-3: x = s (nibble + z)):
 *   Y[m, n] = a_scale[m] * ( sum_g w_scale[g, n] sum_{k in g} a(m, k) w(n, k)
 *                            + a_zero_point[m] * w_zsum[n] )
 * with a(m, k) the signed nibbles and w_zsum from rq_quantize_weights2.
 * Shapes and other arguments as rq_w4a4_linear (no low-rank branch).
 */
rq_status rq_w4a4_linear2(int32_t M, int32_t N, int32_t K, const uint8_t* a_codes, const float* a_scale,
                          const float* a_zero_point, const uint8_t* w_codes, const float* w_scale,
                          const float* w_zsum, void* Y, int32_t out_fp32, int32_t* status, void* stream);

/*
 * rq_read_status -- synchronises `stream`, reads the device status word and
 * returns RQ_OK, RQ_ERR_TIMEOUT (a kernel gave up a bounded wait: word
 * 0x101-0x105; the word is left set), or RQ_ERR_CUDA (a failed copy or sync,
 * or word 0x201: a GEMM found its dynamic shared memory not 1024-byte aligned
 * and left before doing any work).  `code_out` (host, may be NULL) receives
 * the word.
 */
rq_status rq_read_status(const int32_t* status, void* stream, int32_t* code_out);

/* Message for the last error returned on the calling thread ("" if none). */
const char* rq_last_error(void);

#ifdef __cplusplus
}
#endif

#endif /* RQ_H_ */
