/*
 * mx_debug.h -- testing hooks of libmx.  Not part of the computation: these
 * exist so that the failure paths of the kernels can be exercised without
 * faulting a GPU.  (The pages define no such facility.)
 */
#ifndef MX_DEBUG_H
#define MX_DEBUG_H

#include "mx.h"

#ifdef __cplusplus
extern "C" {
#endif

/*
 * mx_debug_gemm_skip_stage -- arm (k_tile >= 0) or disarm (k_tile < 0) a
 * one-shot injected stall for the next mx_gemm or mx_gemm_quantize call made
 * by the calling host thread (calls from other threads are not affected):
 * the producer of the first CTA does not issue the loads of its first tile's
 * k-tile `k_tile`, so the MMA issuer's bounded wait on that stage runs out
 * (after about 2 s).  The kernel then records MX_ERR_TIMEOUT in the device
 * status word (read with mx_last_device_status), waits for the copies it did
 * issue, frees its tensor memory and returns; the CUDA context stays usable.
 * C is left partly unwritten.  Returns MX_OK.
 */
MX_API int mx_debug_gemm_skip_stage(int k_tile);

#ifdef __cplusplus
}
#endif

#endif /* MX_DEBUG_H */
