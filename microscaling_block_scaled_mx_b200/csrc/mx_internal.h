// mx_internal.h -- host-side glue between the C ABI (mx_api.cu) and the
// kernel launchers.  Arguments reaching these functions are already
// validated.
#pragma once

#include <atomic>
#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>

#include "mx.h"

struct MxQuantizeArgs {
    const void *x;
    int xdt;
    int64_t rows, cols, ldx;
    int block_axis;
    int fmt;
    int rnd;
    uint64_t seed;
    bool hadamard;
    uint32_t sign_mask;
    void *codes;
    void *scales;
    int sl;
    int num_sms;
    // stochastic-rounding position of output element (o, i): sr_base + o * sr_stride + i
    uint64_t sr_base, sr_stride;
};

struct MxQuantizeDualArgs {
    const void *x;
    int xdt;
    int64_t rows, cols, ldx;
    int fmt;
    int rnd_rows, rnd_cols;
    uint64_t seed_rows, seed_cols;
    bool hadamard;            // column (block_axis 0) output only
    uint32_t sign_mask;
    void *codes_rows, *scales_rows, *codes_cols, *scales_cols;
    int sl;
    int num_sms;
    uint64_t sr_base_rows, sr_stride_rows, sr_base_cols, sr_stride_cols;
};

struct MxNvfp4Args {
    const void *x;
    int xdt;
    int64_t rows, cols, ldx;
    int64_t domain_rows;       // 0: one global domain
    void *codes;
    void *scales;
    int sl;
    float *enc_scales;
    int num_sms;
};

struct MxDequantArgs {
    const void *codes;
    const void *scales;
    int fmt;
    int sl;
    int64_t outer, inner;
    void *y;
    int ydt;
    int64_t ldy;
    int num_sms;
};

struct MxGemmArgs {
    const void *a_codes, *a_scales, *b_codes, *b_scales;
    int fa, fb;
    int64_t M, N, K;
    float alpha;
    void *c;
    int cdt;
    int64_t ldc;
    // quantized output (mx_gemm_quantize): q_codes non-NULL replaces c
    void *q_codes, *q_scales;
    int q_fmt, q_rnd, q_sl;
    uint64_t q_seed;
    // NVFP4 operands (mx_gemm_nvfp4): E2M1 codes with 16-element E4M3 blocks
    // and per-domain fp32 encode scales; a_lines / b_lines rows per domain (0: one)
    bool nv;
    bool x4;                   // operand scales in MX_SCALES_MMA_X4
    const float *enc_a, *enc_b;
    int64_t a_lines, b_lines;
    int num_sms;
    int device;
};

// MurmurHash3 32-bit finaliser on the host (seed key of stochastic rounding).
inline uint32_t fmix32_host(uint32_t h) {
    h ^= h >> 16;
    h *= 0x85ebca6bu;
    h ^= h >> 13;
    h *= 0xc2b2ae35u;
    h ^= h >> 16;
    return h;
}

cudaError_t mx_launch_quantize(const MxQuantizeArgs &a, cudaStream_t st);
cudaError_t mx_launch_quantize_dual(const MxQuantizeDualArgs &a, cudaStream_t st);
cudaError_t mx_launch_dequantize(const MxDequantArgs &a, cudaStream_t st);
cudaError_t mx_launch_quantize_nvfp4(const MxNvfp4Args &a, cudaStream_t st);
// returns an mx_status (MX_OK, MX_ERR_CUDA, MX_ERR_UNSUPPORTED)
int mx_launch_gemm(const MxGemmArgs &a, cudaStream_t st);
// reads and clears the device status word of the current device (after a sync)
int mx_read_device_status(cudaStream_t st);
// reads and clears the cast kernels' status word (the caller has synchronised)
int mx_read_cast_status();
// reads and clears the NVFP4 unit's debug-build bounds word (the caller has synchronised)
int mx_read_nvfp4_bounds_status();

namespace mxg {
// Encodes (or takes from a per-process cache) a 2-D tiled tensor map: d0 x d1
// elements of type dt at base, row stride `stride` bytes, boxes of b0 x b1,
// no interleave, zero fill outside the tensor.  False if the driver refuses.
bool encode_2d(CUtensorMap *map, CUtensorMapDataType dt, const void *base, uint64_t d0, uint64_t d1,
               uint64_t stride, uint32_t b0, uint32_t b1, CUtensorMapSwizzle swz);
}

// Raises a kernel's dynamic shared-memory limit on the current device the
// first time that device launches it.  The attribute belongs to the device's
// context, so `done` keeps one bit per device (devices 64 and up set it on
// every launch).  Setting it twice is harmless, so two threads that race on a
// first launch need no lock.
template <typename Kern>
cudaError_t ensure_smem_limit(Kern kern, int bytes, std::atomic<uint64_t> &done) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    const uint64_t bit = (dev >= 0 && dev < 64) ? (1ull << dev) : 0ull;
    if (bit && (done.load(std::memory_order_acquire) & bit)) return cudaSuccess;
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
    if (e == cudaSuccess && bit) done.fetch_or(bit, std::memory_order_acq_rel);
    return e;
}
