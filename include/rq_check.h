/*
 * rq_check.h -- verification entry points of the rotated W4A4 library.
 *
 * These calls are not steps of the layer.  They expose, on their own, pieces
 * of device arithmetic that the layer's kernels use, so that tests can compare
 * them with a CPU reference outside of a full layer.  Conventions (ownership,
 * streams, errors) are those of rq.h.
 */
#ifndef RQ_CHECK_H_
#define RQ_CHECK_H_

#include <stdint.h>

#include "rq.h"

#ifdef __cplusplus
extern "C" {
#endif

/*
 * rq_convert_check -- device, async.  Encodes FP32 values with the two
 * hardware conversions the activation kernel uses for NVFP4 (DiRotQ abstract:
 * NVFP4 on Blackwell; element formats E4M3 and E2M1 of the OCP Microscaling
 * specification): cvt.rn.satfinite.e4m3x2.f32 (the UE4M3 block scale) and
 * cvt.rn.satfinite.e2m1x2.f32 (the elements), both round to nearest even and
 * saturating to the largest finite value.
 *   in    [device, n] FP32, finite.   n >= 0, even.
 *   e4m3  [device, n] out: E4M3 byte of in[i] (sign in bit 7).
 *   e2m1  [device, n] out: E2M1 nibble of in[i] in bits 0-3 (sign in bit 3).
 * All pointers 16-byte aligned.  Errors: RQ_ERR_INVALID_ARG (odd n or null
 * pointer), RQ_ERR_ALIGNMENT, RQ_ERR_CUDA (launch failure).
 */
rq_status rq_convert_check(const float* in, int32_t n, uint8_t* e4m3, uint8_t* e2m1, void* stream);

/*
 * rq_set_wait_limit -- host.  Every mbarrier wait in the library's kernels is
 * bounded; this sets the bound, in nanoseconds, for launches made after the
 * call (from any thread).  0 restores the default of 2 s; values above 20 s
 * return RQ_ERR_INVALID_ARG.  `previous` (may be NULL) receives the old bound.
 * A kernel whose wait runs out records a code in the caller's status word
 * (rq_read_status then returns RQ_ERR_TIMEOUT), stops issuing copies and
 * MMAs, waits (bounded) for the ones already issued, frees its tensor memory
 * and exits; the outputs of that call are undefined.
 */
rq_status rq_set_wait_limit(uint64_t limit_ns, uint64_t* previous);

/*
 * rq_set_fault_injection -- host, test hook.  While `extra_tx_bytes` is non-zero,
 * the first operand load of every CTA of later launches (the first row group of
 * the activation and weight kernels, the first K stage of the GEMM kernels)
 * announces that many more bytes than its copies bring.  Every copy still
 * lands; only the barrier never completes, so the bounded waits on it run out
 * and the call reports RQ_ERR_TIMEOUT.  0 switches it off.  A multiple of 16,
 * at most 4096, else RQ_ERR_INVALID_ARG.
 */
rq_status rq_set_fault_injection(uint32_t extra_tx_bytes);

#ifdef __cplusplus
}
#endif

#endif /* RQ_CHECK_H_ */
