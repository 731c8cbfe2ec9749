// mx_encode.cuh -- the 32-block encoder shared by the row cast, the dual cast
// and the quantizing GEMM epilogue.
#pragma once

#include <cstdint>

#include "mx_device.cuh"

namespace mxk {

// Where the encoded blocks of a row-major tensor go: `inner` elements per row,
// codes packed with no padding (row pitch inner * bits / 8 bytes), one E8M0
// scale per block in the plain (row-major) or MMA layout.
struct BlockSink {
    uint8_t *codes;
    uint8_t *scales;
    int64_t inner;
    uint32_t k_blocks;   // inner / 32
    uint32_t k_groups;   // ceil(k_blocks / 4), MMA layout
    int mma_scales;      // scale layout: 0 plain, 1 MMA, 2 MMA x4
    uint32_t key;        // stochastic-rounding seed key
    // stochastic-rounding position of element (row, i): sr_base + row * sr_stride + i
    // (a whole tensor: 0 and inner; a shard: its place in the whole tensor's output)
    uint64_t sr_base, sr_stride;
    uint64_t codes_cap, scales_cap;   // buffer sizes in bytes (checked by the debug build)
};

__device__ __forceinline__ void sink_scale(const BlockSink &o, int64_t row, int64_t kb, uint32_t s) {
    // scale buffers are far below 4 GiB: offsets in 32-bit arithmetic
    put_scale(o.scales, o.mma_scales, static_cast<uint32_t>(row), static_cast<uint32_t>(kb), o.k_blocks,
              o.k_groups, s, o.scales_cap);
}

__device__ __forceinline__ uint64_t f2_mul_ftz(uint64_t a, uint64_t b) {
    uint64_t r;
    asm("mul.rn.ftz.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
    return r;
}

// 32 code bytes of one block: one 32-byte store when the buffers are 32-byte
// aligned (V32), else two 16-byte stores
template <bool V32>
__device__ __forceinline__ void store_code32(uint8_t *dst, const uint4 &a, const uint4 &b) {
    if (V32) {
        asm volatile("st.global.v8.u32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};"
                     ::"l"(dst), "r"(a.x), "r"(a.y), "r"(a.z), "r"(a.w), "r"(b.x), "r"(b.y), "r"(b.z), "r"(b.w)
                     : "memory");
    } else {
        reinterpret_cast<uint4 *>(dst)[0] = a;
        reinterpret_cast<uint4 *>(dst)[1] = b;
    }
}

// Encode one 32-block along a row from its values as FP32 bit patterns
// (Algorithm 1 of the MX summary page, section 3): block amax -> E8M0
// exponent, V * 2^-e (flushing FP32 subnormals), RNE or stochastic rounding,
// and the packed codes and scale byte of block (row, kb).  SR's index is the
// element's position sr_base + row * sr_stride + kb * 32 + j in the output of
// the whole tensor.
// amax_bits: the largest |b[i]| as FP32 bits (sign cleared), computed by the
// caller (encode_block32 below, or bf16_max_bits of the packed input); for a
// block holding a NaN it may be any pattern at or above 0x7f800000.
template <int FMT, bool SR, bool V32>
__device__ __forceinline__ void encode_block32_amax(const BlockSink &o, int64_t row, int64_t kb, uint32_t (&b)[32],
                                                    uint32_t amax_bits) {
    constexpr int BITS = Fmt<FMT>::bits;
    const bool nan_block = amax_bits >= 0x7f800000u;
    const int e = block_exponent<FMT>(amax_bits);

    // V * 2^-e with the subnormal flush (mul.ftz), two values per instruction
    float u[32];
    if (FMT == MX_INT8 && !SR && e >= -120 && e <= 120) {
        // INT8 codes are round(V * 2^(6 - e)) clamped to +-127: fold the 2^6 into
        // the (exact) power-of-two scale, clamp, round half to even
        const uint32_t f = __float_as_uint(pow2f(6 - e));
        const uint64_t ff = static_cast<uint64_t>(f) | (static_cast<uint64_t>(f) << 32);
        uint32_t c[8];
#pragma unroll
        for (int i = 0; i < 32; i += 2) {
            const uint64_t r = f2_mul_ftz(static_cast<uint64_t>(b[i]) | (static_cast<uint64_t>(b[i + 1]) << 32), ff);
            const float x0 = fminf(fmaxf(__uint_as_float(static_cast<uint32_t>(r)), -127.0f), 127.0f);
            const float x1 = fminf(fmaxf(__uint_as_float(static_cast<uint32_t>(r >> 32)), -127.0f), 127.0f);
            const uint32_t q0 = static_cast<uint32_t>(__float2int_rn(x0)) & 0xffu;
            const uint32_t q1 = static_cast<uint32_t>(__float2int_rn(x1)) & 0xffu;
            if ((i & 2) == 0) c[i >> 2] = q0 | (q1 << 8);
            else c[i >> 2] |= (q0 << 16) | (q1 << 24);
        }
        if (nan_block) {
#pragma unroll
            for (int i = 0; i < 8; ++i) c[i] = 0u;
        }
        if (in_bounds(static_cast<uint64_t>(row * o.inner + kb * 32), 32, o.codes_cap))
            store_code32<V32>(o.codes + row * o.inner + kb * 32, make_uint4(c[0], c[1], c[2], c[3]),
                              make_uint4(c[4], c[5], c[6], c[7]));
        sink_scale(o, row, kb, nan_block ? 0xffu : static_cast<uint32_t>(e + 127));
        return;
    }
    if (Fmt<FMT>::emax == 0) {
#pragma unroll
        for (int i = 0; i < 32; ++i) u[i] = scale_down<FMT>(__uint_as_float(b[i]), e);
    } else {
        const uint32_t f = __float_as_uint(pow2f(-e));
        const uint64_t ff = static_cast<uint64_t>(f) | (static_cast<uint64_t>(f) << 32);
#pragma unroll
        for (int i = 0; i < 32; i += 2) {
            const uint64_t r = f2_mul_ftz(static_cast<uint64_t>(b[i]) | (static_cast<uint64_t>(b[i + 1]) << 32), ff);
            u[i] = __uint_as_float(static_cast<uint32_t>(r));
            u[i + 1] = __uint_as_float(static_cast<uint32_t>(r >> 32));
        }
    }
    // pw[w]: the codes of values 4w .. 4w + 3, one per byte (per nibble for E2M1)
    constexpr int SLOT = BITS == 4 ? 4 : 8;
    uint32_t pw[8];
    if (SR) {
        uint32_t rw[8];
        sr_block_words(o.sr_base + static_cast<uint64_t>(row) * o.sr_stride + static_cast<uint64_t>(kb * 32), o.key, rw);
#pragma unroll
        for (int w = 0; w < 8; ++w)
            pw[w] = sr_quad<FMT>(u[4 * w], u[4 * w + 1], u[4 * w + 2], u[4 * w + 3], rw[w]);
    } else {
#pragma unroll
        for (int w = 0; w < 8; ++w)
            pw[w] = cvt_pair<FMT>(u[4 * w], u[4 * w + 1]) | (cvt_pair<FMT>(u[4 * w + 2], u[4 * w + 3]) << (2 * SLOT));
    }
    const uint32_t keep = nan_block ? 0u : 0xffffffffu;     // a NaN/Inf block stores zero codes
    const int64_t code_off = row * (o.inner * BITS / 8) + kb * (32 * BITS / 8);
    uint8_t *dst = o.codes + code_off;
    if (!in_bounds(static_cast<uint64_t>(code_off), 32 * BITS / 8, o.codes_cap)) {
        // (debug build) the block's codes fall outside the buffer: skip them
    } else if (BITS == 8) {
        store_code32<V32>(dst, make_uint4(pw[0] & keep, pw[1] & keep, pw[2] & keep, pw[3] & keep),
                          make_uint4(pw[4] & keep, pw[5] & keep, pw[6] & keep, pw[7] & keep));
    } else if (BITS == 4) {
        uint32_t w[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) w[i] = (pw[2 * i] | (pw[2 * i + 1] << 16)) & keep;
        *reinterpret_cast<uint4 *>(dst) = make_uint4(w[0], w[1], w[2], w[3]);
    } else {
        uint64_t *d = reinterpret_cast<uint64_t *>(dst);     // 24 bytes, 8-byte aligned
#pragma unroll
        for (int q = 0; q < 3; ++q) {
            uint64_t w = 0;
#pragma unroll
            for (int j = 0; j < 32; ++j) {
                const int bit = 6 * j - 64 * q;
                const uint64_t code = (pw[j >> 2] >> (8 * (j & 3))) & 0x3fu;
                if (bit >= 0 && bit < 64) w |= code << bit;
                else if (bit < 0 && bit > -6) w |= code >> (-bit);
            }
            d[q] = w & (static_cast<uint64_t>(keep) << 32 | keep);
        }
    }
    sink_scale(o, row, kb, nan_block ? 0xffu : static_cast<uint32_t>(e + 127));
}



template <int FMT, bool SR, bool V32>
__device__ __forceinline__ void encode_block32(const BlockSink &o, int64_t row, int64_t kb, uint32_t (&b)[32]) {
    float m = 0.0f;
#pragma unroll
    for (int i = 0; i < 32; i += 2) m = max_abs3(m, __uint_as_float(b[i]), __uint_as_float(b[i + 1]));
    encode_block32_amax<FMT, SR, V32>(o, row, kb, b, __float_as_uint(m));
}

// Packed 16-bit maximum of |bf16| over NW words of two bf16 values each (one
// 3-input max per two words): the low and high halves hold the maxima of the
// even and odd elements.  Widening bf16 to FP32 appends 16 zero bits, so a
// half shifted left by 16 is the FP32 magnitude bits of that maximum.
template <int NW>
__device__ __forceinline__ uint32_t bf16_pair_max(const uint32_t *w) {
    uint32_t m = 0;
#pragma unroll
    for (int i = 0; i < NW; i += 2) m = __vimax3_u16x2(m, w[i] & 0x7fff7fffu, w[i + 1] & 0x7fff7fffu);
    return m;
}
__device__ __forceinline__ uint32_t bf16_max_bits(uint32_t m) {
    const uint32_t lo = m << 16, hi = m & 0xffff0000u;
    return lo > hi ? lo : hi;
}

}  // namespace mxk
