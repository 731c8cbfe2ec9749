// mx_cast.cu -- MX cast (Algorithm 1 of "Microscaling Data Formats for Deep
// Learning", summary page, section 3) and exact decode (section 2) on sm_100a.
//
// Both casts are HBM-bound streaming kernels: every input byte is read once
// with 16-byte coalesced loads, every code and scale byte written once.
//  * cast_rows: blocks run along the contiguous axis.  Four lanes cover one
//    32-block (8 values each, one 16-byte bf16 load); the block amax is two
//    xor-shuffles.  A warp walks a 256-element segment of one row.
//  * cast_cols: blocks run down columns.  A CTA stages a 128-row x 64-column
//    tile in shared memory with coalesced row loads; each thread then owns one
//    column block of 32 values in registers, where the optional fixed-sign
//    32-point Hadamard ("Format-Aware Fusion for Fast FP4 Pretraining",
//    abstract) runs as five fp32 butterfly stages, and writes its codes as
//    one row of the transposed (block-axis-major) output.
#include <cstdint>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "mx.h"
#include "mx_device.cuh"
#include "mx_internal.h"

namespace mxk {

struct CastParams {
    const void *x;
    int64_t rows, cols, ldx;
    uint8_t *codes;
    uint8_t *scales;
    int mma_scales;      // 0 plain, 1 MMA layout
    int64_t k_blocks;    // blocks per output row (inner / 32)
    int64_t k_groups;    // ceil(k_blocks / 4), MMA layout
    uint32_t key;        // stochastic-rounding seed key
    uint32_t sign_mask;  // Hadamard signs
};

__device__ __forceinline__ void store_scale(const CastParams &p, int64_t o, int64_t kb, uint32_t s) {
    // scale buffers are far below 4 GiB: offsets in 32-bit arithmetic
    const uint32_t oo = static_cast<uint32_t>(o), k = static_cast<uint32_t>(kb);
    const uint32_t off = p.mma_scales ? mma_scale_offset32(oo, k, static_cast<uint32_t>(p.k_groups))
                                      : oo * static_cast<uint32_t>(p.k_blocks) + k;
    p.scales[off] = static_cast<uint8_t>(s);
}

// Encode n (even) scaled values u[] to codes; sign is carried by u.
template <int FMT, bool SR>
__device__ __forceinline__ void encode_values(float *u, int n, const uint32_t *rnd_words, uint32_t *pairs) {
#pragma unroll
    for (int j = 0; j < n; j += 2) {
        float a = u[j], b = u[j + 1];
        if (SR) {
            uint32_t ra = (rnd_words[j >> 2] >> (8 * (j & 3))) & 255u;
            uint32_t rb = (rnd_words[(j + 1) >> 2] >> (8 * ((j + 1) & 3))) & 255u;
            a = copysignf(sr_magnitude<FMT>(fabsf(a), ra), a);
            b = copysignf(sr_magnitude<FMT>(fabsf(b), rb), b);
        }
        pairs[j >> 1] = cvt_pair<FMT>(a, b);
    }
}

// ---------------------------------------------------------------------------
// Row cast: block axis contiguous.
// ---------------------------------------------------------------------------
// One oct = 8 consecutive values of a row, owned by one lane; the four lanes
// 4b..4b+3 of a warp hold one 32-block.  A warp walks 32-oct segments of one
// row; U segments are loaded before any of them is processed so that every
// thread keeps U 16-byte loads (bf16; 2U for fp32) in flight.
template <bool BF16_IN>
struct OctLoad {
    uint4 w[BF16_IN ? 1 : 2];
};

template <bool BF16_IN>
__device__ __forceinline__ void load_oct(const CastParams &p, int64_t row, int64_t col8, bool valid,
                                         OctLoad<BF16_IN> &o) {
    if (BF16_IN) {
        o.w[0] = make_uint4(0, 0, 0, 0);
        if (valid)
            o.w[0] = __ldcs(reinterpret_cast<const uint4 *>(static_cast<const uint16_t *>(p.x) + row * p.ldx + col8 * 8));
    } else {
        o.w[0] = o.w[BF16_IN ? 0 : 1] = make_uint4(0, 0, 0, 0);
        if (valid) {
            const uint4 *src = reinterpret_cast<const uint4 *>(static_cast<const float *>(p.x) + row * p.ldx + col8 * 8);
            o.w[0] = __ldcs(src);
            o.w[BF16_IN ? 0 : 1] = __ldcs(src + 1);
        }
    }
}

template <int FMT, bool SR, bool BF16_IN>
__device__ __forceinline__ void cast_oct(const CastParams &p, int64_t row, int64_t col8, bool valid,
                                         const OctLoad<BF16_IN> &o, int lane) {
    constexpr int BITS = Fmt<FMT>::bits;
    float v[8];
    uint32_t amax_bits;
    if (BF16_IN) {
        const uint4 w = o.w[0];
        const uint32_t m = __vmaxu2(__vmaxu2(w.x & 0x7fff7fffu, w.y & 0x7fff7fffu),
                                    __vmaxu2(w.z & 0x7fff7fffu, w.w & 0x7fff7fffu));
        amax_bits = max(m & 0xffffu, m >> 16) << 16;
        const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            v[2 * i] = __uint_as_float(ws[i] << 16);
            v[2 * i + 1] = __uint_as_float(ws[i] & 0xffff0000u);
        }
    } else {
        const uint4 a = o.w[0], b = o.w[BF16_IN ? 0 : 1];
        const uint32_t ws[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
        amax_bits = 0;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            v[i] = __uint_as_float(ws[i]);
            amax_bits = max(amax_bits, ws[i] & 0x7fffffffu);
        }
    }
    amax_bits = max(amax_bits, __shfl_xor_sync(0xffffffffu, amax_bits, 1));
    amax_bits = max(amax_bits, __shfl_xor_sync(0xffffffffu, amax_bits, 2));
    if (!valid) return;

    const bool nan_block = amax_bits >= 0x7f800000u;
    const int e = block_exponent<FMT>(amax_bits);
    float u[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) u[i] = scale_down<FMT>(v[i], e);

    uint32_t rw[2] = {0u, 0u};
    if (SR) {
        const uint64_t idx0 = static_cast<uint64_t>(row * p.cols + col8 * 8);
        const uint32_t g = static_cast<uint32_t>(idx0 >> 2);
        rw[0] = fmix32(g ^ p.key);
        rw[1] = fmix32((g + 1u) ^ p.key);
    }
    uint32_t c[4];
    encode_values<FMT, SR>(u, 8, rw, c);
    if (nan_block) c[0] = c[1] = c[2] = c[3] = 0u;

    if (BITS == 8) {
        uint2 out = make_uint2(c[0] | (c[1] << 16), c[2] | (c[3] << 16));
        *reinterpret_cast<uint2 *>(p.codes + row * p.cols + col8 * 8) = out;
    } else if (BITS == 4) {
        uint32_t out = c[0] | (c[1] << 8) | (c[2] << 16) | (c[3] << 24);
        *reinterpret_cast<uint32_t *>(p.codes + row * (p.cols >> 1) + col8 * 4) = out;
    } else {
        uint64_t w = 0;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            w |= static_cast<uint64_t>(c[i] & 0x3fu) << (12 * i);
            w |= static_cast<uint64_t>((c[i] >> 8) & 0x3fu) << (12 * i + 6);
        }
        uint8_t *dst = p.codes + row * (p.cols / 4 * 3) + col8 * 6;
        if ((col8 & 1) == 0) {
            *reinterpret_cast<uint32_t *>(dst) = static_cast<uint32_t>(w);
            *reinterpret_cast<uint16_t *>(dst + 4) = static_cast<uint16_t>(w >> 32);
        } else {
            *reinterpret_cast<uint16_t *>(dst) = static_cast<uint16_t>(w);
            *reinterpret_cast<uint32_t *>(dst + 2) = static_cast<uint32_t>(w >> 16);
        }
    }
    if ((lane & 3) == 0) store_scale(p, row, col8 >> 2, nan_block ? 0xffu : static_cast<uint32_t>(e + 127));
}

template <int FMT, bool SR, bool BF16_IN>
__global__ void __launch_bounds__(256) cast_rows_kernel(CastParams p) {
    constexpr int U = BF16_IN ? 4 : 2;                  // segments in flight per warp
    const int lane = threadIdx.x & 31;
    const int64_t octs_per_row = p.cols >> 3;
    const int64_t spr = (octs_per_row + 31) >> 5;       // 32-oct segments per row
    const int64_t warp0 = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
    const int64_t n_warps = (static_cast<int64_t>(gridDim.x) * blockDim.x) >> 5;
    // segment s = row * spr + seg; consecutive visits of a warp are n_warps
    // apart, stepped without a division inside the loop
    int64_t row = warp0 / spr, seg = warp0 - row * spr;
    const int64_t step_rows = n_warps / spr, step_seg = n_warps - step_rows * spr;

    while (row < p.rows) {
        int64_t r[U], c8[U];
        bool ok[U];
        OctLoad<BF16_IN> ld[U];
#pragma unroll
        for (int u = 0; u < U; ++u) {
            r[u] = row;
            c8[u] = seg * 32 + lane;
            ok[u] = row < p.rows && c8[u] < octs_per_row;
            load_oct<BF16_IN>(p, row, c8[u], ok[u], ld[u]);
            seg += step_seg;
            row += step_rows;
            if (seg >= spr) { seg -= spr; ++row; }
        }
#pragma unroll
        for (int u = 0; u < U; ++u) cast_oct<FMT, SR, BF16_IN>(p, r[u], c8[u], ok[u], ld[u], lane);
    }
}

// ---------------------------------------------------------------------------
// Column cast: block axis strided, output transposed.
// ---------------------------------------------------------------------------
constexpr int COL_TILE_R = 128;   // 4 blocks down
constexpr int COL_TILE_C = 64;    // columns per tile

template <int FMT, bool SR, bool BF16_IN, bool HAD>
__global__ void __launch_bounds__(256) cast_cols_kernel(CastParams p) {
    using TIn = typename std::conditional<BF16_IN, uint16_t, float>::type;
    __shared__ __align__(16) TIn tile[COL_TILE_R][COL_TILE_C];
    constexpr int BITS = Fmt<FMT>::bits;
    constexpr int ELEMS_PER_CHUNK = 16 / sizeof(TIn);
    constexpr int CHUNKS_PER_ROW = COL_TILE_C / ELEMS_PER_CHUNK;

    const int64_t R = p.rows, C = p.cols;
    const int64_t tiles_r = (R + COL_TILE_R - 1) / COL_TILE_R;
    const int64_t tiles_c = (C + COL_TILE_C - 1) / COL_TILE_C;
    const int64_t n_tiles = tiles_r * tiles_c;
    const TIn *x = static_cast<const TIn *>(p.x);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    for (int64_t t = blockIdx.x; t < n_tiles; t += gridDim.x) {
        const int64_t tr = t / tiles_c, tc = t - tr * tiles_c;
        const int64_t r0 = tr * COL_TILE_R, c0 = tc * COL_TILE_C;

        // stage the tile with 16-byte row loads (ragged edges element-wise)
        for (int ch = threadIdx.x; ch < COL_TILE_R * CHUNKS_PER_ROW; ch += blockDim.x) {
            const int rr = ch / CHUNKS_PER_ROW, cc = (ch % CHUNKS_PER_ROW) * ELEMS_PER_CHUNK;
            const int64_t gr = r0 + rr, gc = c0 + cc;
            uint4 w = make_uint4(0, 0, 0, 0);
            if (gr < R) {
                const TIn *src = x + gr * p.ldx + gc;
                if (gc + ELEMS_PER_CHUNK <= C) {
                    w = __ldcs(reinterpret_cast<const uint4 *>(src));
                } else {
                    TIn tmp[ELEMS_PER_CHUNK];
#pragma unroll
                    for (int i = 0; i < ELEMS_PER_CHUNK; ++i) tmp[i] = (gc + i < C) ? src[i] : TIn(0);
                    w = *reinterpret_cast<uint4 *>(tmp);
                }
            }
            *reinterpret_cast<uint4 *>(&tile[rr][cc]) = w;
        }
        __syncthreads();

        // one column block of 32 values per thread
        const int blk = warp & 3;
        const int col = (warp >> 2) * 32 + lane;
        const int64_t gc = c0 + col, gr0 = r0 + blk * 32;
        if (gc < C && gr0 < R) {
            float v[32];
#pragma unroll
            for (int i = 0; i < 32; ++i) {
                if (BF16_IN) v[i] = __uint_as_float(static_cast<uint32_t>(tile[blk * 32 + i][col]) << 16);
                else v[i] = tile[blk * 32 + i][col];
            }
            if (HAD) {
#pragma unroll
                for (int j = 0; j < 32; ++j)
                    if (!((p.sign_mask >> j) & 1u)) v[j] = -v[j];
#pragma unroll
                for (int h = 1; h < 32; h <<= 1) {
#pragma unroll
                    for (int i = 0; i < 32; ++i) {
                        if (i & h) continue;
                        const float a = v[i], b = v[i + h];
                        v[i] = __fadd_rn(a, b);
                        v[i + h] = __fsub_rn(a, b);
                    }
                }
            }
            uint32_t amax_bits = 0;
#pragma unroll
            for (int i = 0; i < 32; ++i) amax_bits = max(amax_bits, __float_as_uint(v[i]) & 0x7fffffffu);
            const bool nan_block = amax_bits >= 0x7f800000u;
            const int e = block_exponent<FMT>(amax_bits);
#pragma unroll
            for (int i = 0; i < 32; ++i) v[i] = scale_down<FMT>(v[i], e);

            uint32_t rw[8];
            if (SR) {
                const uint64_t idx0 = static_cast<uint64_t>(gc * R + gr0);
                const uint32_t g = static_cast<uint32_t>(idx0 >> 2);
#pragma unroll
                for (int i = 0; i < 8; ++i) rw[i] = fmix32((g + i) ^ p.key);
            }
            uint32_t c[16];
            encode_values<FMT, SR>(v, 32, rw, c);
            if (nan_block) {
#pragma unroll
                for (int i = 0; i < 16; ++i) c[i] = 0u;
            }
            if (BITS == 8) {
                uint4 *dst = reinterpret_cast<uint4 *>(p.codes + gc * R + gr0);
                dst[0] = make_uint4(c[0] | (c[1] << 16), c[2] | (c[3] << 16), c[4] | (c[5] << 16), c[6] | (c[7] << 16));
                dst[1] = make_uint4(c[8] | (c[9] << 16), c[10] | (c[11] << 16), c[12] | (c[13] << 16), c[14] | (c[15] << 16));
            } else if (BITS == 4) {
                uint32_t w[4];
#pragma unroll
                for (int i = 0; i < 4; ++i)
                    w[i] = c[4 * i] | (c[4 * i + 1] << 8) | (c[4 * i + 2] << 16) | (c[4 * i + 3] << 24);
                *reinterpret_cast<uint4 *>(p.codes + gc * (R >> 1) + (gr0 >> 1)) = make_uint4(w[0], w[1], w[2], w[3]);
            } else {
                uint64_t *dst = reinterpret_cast<uint64_t *>(p.codes + gc * (R / 4 * 3) + gr0 / 4 * 3);
#pragma unroll
                for (int q = 0; q < 3; ++q) {     // 3 words of 64 bits = 32 codes of 6 bits
                    uint64_t w = 0;
#pragma unroll
                    for (int j = 0; j < 32; ++j) {
                        const int bit = 6 * j - 64 * q;
                        const uint64_t code = (c[j >> 1] >> (8 * (j & 1))) & 0x3fu;
                        if (bit >= 0 && bit < 64) w |= code << bit;
                        else if (bit < 0 && bit > -6) w |= code >> (-bit);
                    }
                    dst[q] = w;
                }
            }
            store_scale(p, gc, gr0 >> 5, nan_block ? 0xffu : static_cast<uint32_t>(e + 127));
        }
        __syncthreads();
    }
}

// ---------------------------------------------------------------------------
// Dequantize: v = 2^(s-127) * P, rounded once to the output type.
// ---------------------------------------------------------------------------
template <int FMT> __device__ __forceinline__ void decode_pair(uint32_t pair_bits, float &a, float &b);

__device__ __forceinline__ void half2_to_floats(uint32_t h2, float &a, float &b) {
    __half2 h = *reinterpret_cast<__half2 *>(&h2);
    a = __low2float(h);
    b = __high2float(h);
}
template <> __device__ __forceinline__ void decode_pair<MX_E4M3>(uint32_t p2, float &a, float &b) {
    uint32_t h; uint16_t s = static_cast<uint16_t>(p2);
    asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h) : "h"(s));
    half2_to_floats(h, a, b);
}
template <> __device__ __forceinline__ void decode_pair<MX_E5M2>(uint32_t p2, float &a, float &b) {
    uint32_t h; uint16_t s = static_cast<uint16_t>(p2);
    asm("cvt.rn.f16x2.e5m2x2 %0, %1;" : "=r"(h) : "h"(s));
    half2_to_floats(h, a, b);
}
template <> __device__ __forceinline__ void decode_pair<MX_E2M3>(uint32_t p2, float &a, float &b) {
    uint32_t h; uint16_t s = static_cast<uint16_t>(p2);
    asm("cvt.rn.f16x2.e2m3x2 %0, %1;" : "=r"(h) : "h"(s));
    half2_to_floats(h, a, b);
}
template <> __device__ __forceinline__ void decode_pair<MX_E3M2>(uint32_t p2, float &a, float &b) {
    uint32_t h; uint16_t s = static_cast<uint16_t>(p2);
    asm("cvt.rn.f16x2.e3m2x2 %0, %1;" : "=r"(h) : "h"(s));
    half2_to_floats(h, a, b);
}
template <> __device__ __forceinline__ void decode_pair<MX_E2M1>(uint32_t p2, float &a, float &b) {
    uint32_t h;
    asm("{\n\t.reg .b8 t;\n\tcvt.u8.u32 t, %1;\n\tcvt.rn.f16x2.e2m1x2 %0, t;\n\t}" : "=r"(h) : "r"(p2 & 0xffu));
    half2_to_floats(h, a, b);
}
template <> __device__ __forceinline__ void decode_pair<MX_INT8>(uint32_t p2, float &a, float &b) {
    a = static_cast<float>(static_cast<int8_t>(p2 & 0xffu)) * 0.015625f;
    b = static_cast<float>(static_cast<int8_t>((p2 >> 8) & 0xffu)) * 0.015625f;
}

// scale by 2^(s-127) with IEEE rounding (no flush): one multiply when the
// factor is normal, and for s == 0 the factor 2^-127 is itself exact.
__device__ __forceinline__ float apply_scale(float pv, uint32_t s) {
    if (s == 0xffu) return __uint_as_float(0x7fc00000u);
    const float f = s == 0 ? __uint_as_float(0x00400000u) : __uint_as_float(s << 23);
    return __fmul_rn(pv, f);
}

struct DequantParams {
    const uint8_t *codes;
    const uint8_t *scales;
    int mma_scales;
    int64_t outer, inner, k_blocks, k_groups;
    void *y;
    int64_t ldy;
};

template <int FMT, bool BF16_OUT>
__global__ void __launch_bounds__(256) dequant_kernel(DequantParams p) {
    constexpr int BITS = Fmt<FMT>::bits;
    const int64_t octs_per_row = p.inner >> 3;
    const int64_t n = p.outer * octs_per_row;
    for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n;
         i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
        const int64_t o = i / octs_per_row, oc = i - o * octs_per_row;
        const int64_t kb = oc >> 2;
        const uint32_t s = p.scales[p.mma_scales ? mma_scale_offset(o, kb, p.k_groups) : o * p.k_blocks + kb];
        uint32_t pairs[4];
        if (BITS == 8) {
            uint2 w = *reinterpret_cast<const uint2 *>(p.codes + o * p.inner + oc * 8);
            pairs[0] = w.x & 0xffffu; pairs[1] = w.x >> 16; pairs[2] = w.y & 0xffffu; pairs[3] = w.y >> 16;
        } else if (BITS == 4) {
            uint32_t w = *reinterpret_cast<const uint32_t *>(p.codes + o * (p.inner >> 1) + oc * 4);
            pairs[0] = w & 0xffu; pairs[1] = (w >> 8) & 0xffu; pairs[2] = (w >> 16) & 0xffu; pairs[3] = w >> 24;
        } else {
            const uint8_t *src = p.codes + o * (p.inner / 4 * 3) + oc * 6;
            uint64_t w = 0;
#pragma unroll
            for (int b = 0; b < 6; ++b) w |= static_cast<uint64_t>(src[b]) << (8 * b);
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                const uint32_t c0 = (w >> (12 * k)) & 0x3fu, c1 = (w >> (12 * k + 6)) & 0x3fu;
                pairs[k] = c0 | (c1 << 8);
            }
        }
        float val[8];
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            decode_pair<FMT>(pairs[k], val[2 * k], val[2 * k + 1]);
            val[2 * k] = apply_scale(val[2 * k], s);
            val[2 * k + 1] = apply_scale(val[2 * k + 1], s);
        }
        if (BF16_OUT) {
            uint32_t h[4];
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                __nv_bfloat162 b2 = __floats2bfloat162_rn(val[2 * k], val[2 * k + 1]);
                h[k] = *reinterpret_cast<uint32_t *>(&b2);
            }
            *reinterpret_cast<uint4 *>(static_cast<uint16_t *>(p.y) + o * p.ldy + oc * 8) = make_uint4(h[0], h[1], h[2], h[3]);
        } else {
            float4 *dst = reinterpret_cast<float4 *>(static_cast<float *>(p.y) + o * p.ldy + oc * 8);
            dst[0] = make_float4(val[0], val[1], val[2], val[3]);
            dst[1] = make_float4(val[4], val[5], val[6], val[7]);
        }
    }
}

// ---------------------------------------------------------------------------
// Host-side launchers (arguments already validated by the C ABI layer).
// ---------------------------------------------------------------------------
static int grid_for(int64_t work_items, int per_block, int max_blocks) {
    int64_t b = (work_items + per_block - 1) / per_block;
    if (b > max_blocks) b = max_blocks;
    return static_cast<int>(b < 1 ? 1 : b);
}

template <int FMT, bool SR>
static cudaError_t launch_cast_fmt(const CastParams &p, int xdt, int block_axis, bool had, int sms,
                                   cudaStream_t st) {
    const bool bf = xdt == MX_BF16;
    if (block_axis == 1) {
        const int64_t segs = p.rows * (((p.cols >> 3) + 31) >> 5);
        const int grid = grid_for(segs, 8, sms * 8);
        if (bf) cast_rows_kernel<FMT, SR, true><<<grid, 256, 0, st>>>(p);
        else cast_rows_kernel<FMT, SR, false><<<grid, 256, 0, st>>>(p);
    } else {
        const int64_t tiles = ((p.rows + COL_TILE_R - 1) / COL_TILE_R) * ((p.cols + COL_TILE_C - 1) / COL_TILE_C);
        const int grid = grid_for(tiles, 1, sms * 8);
        if (had) {
            if (bf) cast_cols_kernel<FMT, SR, true, true><<<grid, 256, 0, st>>>(p);
            else cast_cols_kernel<FMT, SR, false, true><<<grid, 256, 0, st>>>(p);
        } else {
            if (bf) cast_cols_kernel<FMT, SR, true, false><<<grid, 256, 0, st>>>(p);
            else cast_cols_kernel<FMT, SR, false, false><<<grid, 256, 0, st>>>(p);
        }
    }
    return cudaGetLastError();
}

template <int FMT>
static cudaError_t launch_cast_rnd(const CastParams &p, int xdt, int block_axis, bool sr, bool had, int sms,
                                   cudaStream_t st) {
    return sr ? launch_cast_fmt<FMT, true>(p, xdt, block_axis, had, sms, st)
              : launch_cast_fmt<FMT, false>(p, xdt, block_axis, had, sms, st);
}

}  // namespace mxk

cudaError_t mx_launch_quantize(const MxQuantizeArgs &a, cudaStream_t st) {
    using namespace mxk;
    CastParams p;
    p.x = a.x;
    p.rows = a.rows;
    p.cols = a.cols;
    p.ldx = a.ldx;
    p.codes = static_cast<uint8_t *>(a.codes);
    p.scales = static_cast<uint8_t *>(a.scales);
    p.mma_scales = a.sl == MX_SCALES_MMA;
    const int64_t inner = a.block_axis == 1 ? a.cols : a.rows;
    p.k_blocks = inner / 32;
    p.k_groups = (p.k_blocks + 3) / 4;
    p.key = fmix32_host(static_cast<uint32_t>(a.seed)) ^ static_cast<uint32_t>(a.seed >> 32);
    p.sign_mask = a.sign_mask;
    const bool sr = a.rnd == MX_SR;
    switch (a.fmt) {
        case MX_E4M3: return launch_cast_rnd<MX_E4M3>(p, a.xdt, a.block_axis, sr, a.hadamard, a.num_sms, st);
        case MX_E5M2: return launch_cast_rnd<MX_E5M2>(p, a.xdt, a.block_axis, sr, a.hadamard, a.num_sms, st);
        case MX_E2M3: return launch_cast_rnd<MX_E2M3>(p, a.xdt, a.block_axis, sr, a.hadamard, a.num_sms, st);
        case MX_E3M2: return launch_cast_rnd<MX_E3M2>(p, a.xdt, a.block_axis, sr, a.hadamard, a.num_sms, st);
        case MX_E2M1: return launch_cast_rnd<MX_E2M1>(p, a.xdt, a.block_axis, sr, a.hadamard, a.num_sms, st);
        case MX_INT8: return launch_cast_rnd<MX_INT8>(p, a.xdt, a.block_axis, sr, a.hadamard, a.num_sms, st);
    }
    return cudaErrorInvalidValue;
}

cudaError_t mx_launch_dequantize(const MxDequantArgs &a, cudaStream_t st) {
    using namespace mxk;
    DequantParams p;
    p.codes = static_cast<const uint8_t *>(a.codes);
    p.scales = static_cast<const uint8_t *>(a.scales);
    p.mma_scales = a.sl == MX_SCALES_MMA;
    p.outer = a.outer;
    p.inner = a.inner;
    p.k_blocks = a.inner / 32;
    p.k_groups = (p.k_blocks + 3) / 4;
    p.y = a.y;
    p.ldy = a.ldy;
    const int grid = grid_for(a.outer * (a.inner / 8), 256, a.num_sms * 8);
    const bool bf = a.ydt == MX_BF16;
#define MX_DQ(F)                                                        \
    case F:                                                             \
        if (bf) dequant_kernel<F, true><<<grid, 256, 0, st>>>(p);       \
        else dequant_kernel<F, false><<<grid, 256, 0, st>>>(p);         \
        break;
    switch (a.fmt) {
        MX_DQ(MX_E4M3)
        MX_DQ(MX_E5M2)
        MX_DQ(MX_E2M3)
        MX_DQ(MX_E3M2)
        MX_DQ(MX_E2M1)
        MX_DQ(MX_INT8)
        default: return cudaErrorInvalidValue;
    }
#undef MX_DQ
    return cudaGetLastError();
}
