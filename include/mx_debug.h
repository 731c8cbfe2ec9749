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

/*
 * mx_debug_gemm_force_kernel -- choose the GEMM kernel of the calling host
 * thread's later mx_gemm / mx_gemm_quantize calls instead of the automatic
 * choice, so that tests reach every kernel on any shape: 0 the one-SM kernel
 * (128 x 192 tiles), 1 the one-SM kernel with a resident B panel (128 x 192
 * tiles, at most six 128-byte K slices: a GEMM with a longer K then returns
 * MX_ERR_UNSUPPORTED), 256 or 192 the CTA-pair kernel with 256 x 256 or
 * 256 x 192 tiles, -1 back to automatic.  Results are the same up to the
 * order of the fp32 sums.  Returns MX_OK, or MX_ERR_ARG for another value.
 */
MX_API int mx_debug_gemm_force_kernel(int tile_n);

/*
 * mx_debug_cast_force_cpasync -- on != 0: the calling host thread's later
 * column and dual casts (mx_quantize with block_axis 0, mx_quantize_dual and
 * their shard forms) stage their input tiles with 16-byte cp.async copies
 * instead of TMA tensor copies, the path taken otherwise only for inputs a
 * tensor map cannot describe (a row or column count beyond int32 range).  The
 * results are identical.  on == 0 restores the automatic choice.  Returns
 * MX_OK.
 */
MX_API int mx_debug_cast_force_cpasync(int on);

/*
 * mx_debug_cast_skip_tile -- arm (on != 0) or disarm a one-shot injected
 * stall for the next column or dual cast of the calling host thread: the
 * first CTA does not issue the TMA copy of its first tile, so its bounded
 * wait on that tile runs out (after about 2 s).  The CTA records
 * MX_ERR_TIMEOUT in the cast status word (read with mx_last_device_status),
 * waits, again bounded, for the copies it did issue, and returns; the CUDA
 * context stays usable and the outputs are left partly unwritten.  A call
 * that stages with cp.async (mx_debug_cast_force_cpasync) consumes the hook
 * without effect.  Returns MX_OK.
 */
MX_API int mx_debug_cast_skip_tile(int on);

/*
 * mx_debug_cast_cut_codes_cap -- one shot, for the next mx_quantize (or
 * shard) call of the calling host thread: the size of the codes buffer the
 * kernels are told is `bytes` smaller than the true one.  Only the debug
 * build (libmx_debug.so, MX_DEBUG) checks stores against that size: there the
 * blocks whose codes would reach past it are not written and
 * mx_last_device_status reports MX_ERR_BOUNDS, which tests the bounds checks
 * without any access outside a real buffer.  The release build ignores it.
 * Returns MX_OK, or MX_ERR_ARG for a negative size.
 */
MX_API int mx_debug_cast_cut_codes_cap(int64_t bytes);

#ifdef __cplusplus
}
#endif

#endif /* MX_DEBUG_H */
