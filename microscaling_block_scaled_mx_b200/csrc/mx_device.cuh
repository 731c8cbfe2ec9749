// mx_device.cuh -- device-side MX element formats for sm_100a.
//
// The cast of "Microscaling Data Formats for Deep Learning" (summary page,
// section 3, Algorithm 1): per 32-block, X = 2^(floor(log2 amax) - emax),
// P_i = round(V_i / X) with overflow clamped to the largest normal and FP32
// subnormal inputs set to zero.  Rounding to the element grid uses the
// hardware conversions (cvt.rn.satfinite.{e4m3,e5m2,e2m3,e3m2,e2m1}x2.f32),
// whose round-to-nearest-even with saturation to the largest finite value is
// exactly the clamp that section asks for.  Stochastic rounding (the
// row-gradient rounding of "Format-Aware Fusion for Fast FP4 Pretraining")
// truncates onto the grid and adds one grid step when the 8 bits below it plus
// a random byte carry out.
#pragma once

#include <cstdint>
#include <cuda_bf16.h>

#include "mx.h"

namespace mxk {

// Per-format constants: code width, emax (exponent of the largest binade),
// mantissa bits, smallest normal exponent, largest finite value.
template <int FMT> struct Fmt;
template <> struct Fmt<MX_E4M3> { static constexpr int bits = 8, emax = 8,  mbits = 3, emin = -6;  static constexpr float maxv = 448.0f; };
template <> struct Fmt<MX_E5M2> { static constexpr int bits = 8, emax = 15, mbits = 2, emin = -14; static constexpr float maxv = 57344.0f; };
template <> struct Fmt<MX_E2M3> { static constexpr int bits = 6, emax = 2,  mbits = 3, emin = 0;   static constexpr float maxv = 7.5f; };
template <> struct Fmt<MX_E3M2> { static constexpr int bits = 6, emax = 4,  mbits = 2, emin = -2;  static constexpr float maxv = 28.0f; };
template <> struct Fmt<MX_E2M1> { static constexpr int bits = 4, emax = 2,  mbits = 1, emin = 0;   static constexpr float maxv = 6.0f; };
// INT8: fixed point with 6 fraction bits; treated as one binade with spacing 2^-6.
template <> struct Fmt<MX_INT8> { static constexpr int bits = 8, emax = 0,  mbits = 6, emin = 0;   static constexpr float maxv = 127.0f / 64.0f; };

__device__ __forceinline__ float pow2f(int k) {  // 2^k for k in [-126, 127]
    return __uint_as_float(static_cast<uint32_t>(k + 127) << 23);
}

// E8M0 scale exponent of a block from the largest |bits| (sign cleared) of
// its FP32 values.  Returns e with X = 2^e; 0x7f800000 or above means the
// block held an Inf or NaN (handled by the caller).  Subnormal magnitudes
// count as zero: they are flushed before the cast.
template <int FMT>
__device__ __forceinline__ int block_exponent(uint32_t amax_bits) {
    if (amax_bits < 0x00800000u) return -127;               // all zero after the flush
    int e = static_cast<int>(amax_bits >> 23) - 127 - Fmt<FMT>::emax;
    return e < -127 ? -127 : (e > 127 ? 127 : e);
}

// V * 2^-e with the FP32-subnormal flush folded in: mul.ftz treats subnormal
// inputs as signed zeros (the section-3 flush); a subnormal product is also
// flushed, which is harmless because every element format rounds anything
// below 2^-126 to zero.  e = 127 (only reachable for INT8) takes two steps so
// that no factor is itself subnormal.
template <int FMT>
__device__ __forceinline__ float scale_down(float v, int e) {
    float r;
    if (Fmt<FMT>::emax == 0 && e > 126) {
        asm("mul.rn.ftz.f32 %0, %1, %2;" : "=f"(r) : "f"(v), "f"(pow2f(-64)));
        asm("mul.rn.ftz.f32 %0, %1, %2;" : "=f"(r) : "f"(r), "f"(pow2f(64 - e)));
    } else {
        asm("mul.rn.ftz.f32 %0, %1, %2;" : "=f"(r) : "f"(v), "f"(pow2f(-e)));
    }
    return r;
}

// Round-to-nearest-even with saturation of two FP32 values; returns the codes
// of a (bits 0..7) and b (bits 8..15), sign bits included.  For FP6 each code
// sits in the low 6 bits of its byte, for FP4 in the low nibble of bits 0..7
// (a) and the high nibble (b).
template <int FMT> __device__ __forceinline__ uint32_t cvt_pair(float a, float b);

template <> __device__ __forceinline__ uint32_t cvt_pair<MX_E4M3>(float a, float b) {
    uint16_t d;
    asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(d) : "f"(b), "f"(a));
    return d;
}
template <> __device__ __forceinline__ uint32_t cvt_pair<MX_E5M2>(float a, float b) {
    uint16_t d;
    asm("cvt.rn.satfinite.e5m2x2.f32 %0, %1, %2;" : "=h"(d) : "f"(b), "f"(a));
    return d;
}
template <> __device__ __forceinline__ uint32_t cvt_pair<MX_E2M3>(float a, float b) {
    uint16_t d;
    asm("cvt.rn.satfinite.e2m3x2.f32 %0, %1, %2;" : "=h"(d) : "f"(b), "f"(a));
    return d;
}
template <> __device__ __forceinline__ uint32_t cvt_pair<MX_E3M2>(float a, float b) {
    uint16_t d;
    asm("cvt.rn.satfinite.e3m2x2.f32 %0, %1, %2;" : "=h"(d) : "f"(b), "f"(a));
    return d;
}
template <> __device__ __forceinline__ uint32_t cvt_pair<MX_E2M1>(float a, float b) {
    uint32_t d;
    asm("{\n\t.reg .b8 t;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 t, %1, %2;\n\t"
        "cvt.u32.u8 %0, t;\n\t}" : "=r"(d) : "f"(b), "f"(a));
    return d;
}
// INT8: round |v| * 64 to the nearest even integer, clamp to 127, two's complement.
template <> __device__ __forceinline__ uint32_t cvt_pair<MX_INT8>(float a, float b) {
    auto one = [](float v) -> uint32_t {
        float m = rintf(fabsf(v) * 64.0f);
        int q = static_cast<int>(fminf(m, 127.0f));
        if (__float_as_uint(v) >> 31) q = -q;
        return static_cast<uint32_t>(q) & 0xffu;
    };
    return one(a) | (one(b) << 8);
}

// Stochastic rounding of a non-negative FP32 value a onto the element grid:
// with lo the grid point at or below a and s the grid step there, F = the 8
// bits of (a - lo) / s just below the step; the result is lo + s when F + r >=
// 256, else lo (r the random byte).  In integer arithmetic: for a >= 2^emin the
// grid step of a's binade is one unit of fp32 mantissa bit (23 - mbits), so
// adding r at the eight bits below that unit carries into it exactly when
// F + r >= 256, and truncation then gives lo or lo + step.  For a < 2^emin
// (the element's subnormal range, uniform step 2^(emin - mbits)) a is first
// shifted to a + 2^emin with a round-toward-zero add, which keeps every bit
// that F depends on, rounded the same way, and shifted back exactly.  Returns
// the rounded magnitude (callers convert it with a saturating conversion).
// INT8 uses it directly; the other formats round the same way in hardware
// (sr_quad below).
template <int FMT>
__device__ __forceinline__ float sr_magnitude_int(float a, uint32_t r) {
    using F = Fmt<FMT>;
    const float t = a < pow2f(F::emin) ? pow2f(F::emin) : 0.0f;
    const float w = __fadd_rz(a, t);
    constexpr int UNIT = 23 - F::mbits;
    uint32_t wb = __float_as_uint(w) + (r << (UNIT - 8));
    wb &= ~((1u << UNIT) - 1u);
    // may exceed max by one grid step when |a| >= max: the saturating
    // conversions that follow clamp it to max, which is the rule for |a| >= max
    return __fsub_rn(__uint_as_float(wb), t);
}

// The same stochastic rounding for four scaled values, v_k taking byte k of
// rw, done by the sm_100a conversion cvt.rs.satfinite.<fmt>x4.f32 d, {p0, p1,
// p2, p3}, rbits.  Measured on B200 (every operand, every random bit, every
// element format): d holds p0 in its top code slot down to p3 in slot 0, and
// each operand rounds up iff the 16 bits of its value below the kept mantissa
// plus a 16-bit random number R carry out, with R = rbits[31:16] for p1 and
// rbits[15:0] for p3 (E2M1: bytes 3:1 and 2:0), while p0 and p2 read the same
// bits reversed.  So only p1 and p3 carry values here, each with its byte in
// the top half of R and zeros below: frac16 + r * 2^8 carries out exactly when
// frac8 + r does, the rule of sr_magnitude_int (saturation and signs agree
// too; 2^20 values per format matched it bit for bit).  p0 = p2 = 0 stay 0.
// Returns the codes packed as cvt_pair(v0, v1) | cvt_pair(v2, v3) << (16, or 8
// for E2M1).  INT8 has no such conversion and keeps the integer path.
template <int FMT> __device__ __forceinline__ uint32_t cvt_rs_x4(float p1, float p3, uint32_t rbits);
template <> __device__ __forceinline__ uint32_t cvt_rs_x4<MX_E4M3>(float p1, float p3, uint32_t rbits) {
    uint32_t d;
    asm("cvt.rs.satfinite.e4m3x4.f32 %0, {%1, %2, %3, %4}, %5;" : "=r"(d) : "f"(0.0f), "f"(p1), "f"(0.0f), "f"(p3), "r"(rbits));
    return d;
}
template <> __device__ __forceinline__ uint32_t cvt_rs_x4<MX_E5M2>(float p1, float p3, uint32_t rbits) {
    uint32_t d;
    asm("cvt.rs.satfinite.e5m2x4.f32 %0, {%1, %2, %3, %4}, %5;" : "=r"(d) : "f"(0.0f), "f"(p1), "f"(0.0f), "f"(p3), "r"(rbits));
    return d;
}
template <> __device__ __forceinline__ uint32_t cvt_rs_x4<MX_E2M3>(float p1, float p3, uint32_t rbits) {
    uint32_t d;
    asm("cvt.rs.satfinite.e2m3x4.f32 %0, {%1, %2, %3, %4}, %5;" : "=r"(d) : "f"(0.0f), "f"(p1), "f"(0.0f), "f"(p3), "r"(rbits));
    return d;
}
template <> __device__ __forceinline__ uint32_t cvt_rs_x4<MX_E3M2>(float p1, float p3, uint32_t rbits) {
    uint32_t d;
    asm("cvt.rs.satfinite.e3m2x4.f32 %0, {%1, %2, %3, %4}, %5;" : "=r"(d) : "f"(0.0f), "f"(p1), "f"(0.0f), "f"(p3), "r"(rbits));
    return d;
}
template <> __device__ __forceinline__ uint32_t cvt_rs_x4<MX_E2M1>(float p1, float p3, uint32_t rbits) {
    uint16_t d;
    asm("cvt.rs.satfinite.e2m1x4.f32 %0, {%1, %2, %3, %4}, %5;" : "=h"(d) : "f"(0.0f), "f"(p1), "f"(0.0f), "f"(p3), "r"(rbits));
    return d;
}

template <int FMT>
__device__ __forceinline__ uint32_t sr_quad(float v0, float v1, float v2, float v3, uint32_t rw) {
    if constexpr (FMT == MX_INT8) {
        auto m = [](float v, uint32_t r) { return copysignf(sr_magnitude_int<FMT>(fabsf(v), r), v); };
        return cvt_pair<FMT>(m(v0, rw & 255u), m(v1, (rw >> 8) & 255u)) |
               (cvt_pair<FMT>(m(v2, (rw >> 16) & 255u), m(v3, rw >> 24)) << 16);
    } else {
        constexpr bool FP4 = FMT == MX_E2M1;
        // rbits: byte 2 of rw as v2's top byte, byte 0 as v0's (and 3, 1 for v3, v1)
        const uint32_t ra = __byte_perm(rw, 0u, FP4 ? 0x2044u : 0x2404u);
        const uint32_t rb = __byte_perm(rw, 0u, FP4 ? 0x3144u : 0x3414u);
        const uint32_t a = cvt_rs_x4<FMT>(v2, v0, ra);   // v0 in slot 0, v2 in slot 2
        const uint32_t b = cvt_rs_x4<FMT>(v3, v1, rb);   // v1 in slot 0, v3 in slot 2
        return a | (b << (FP4 ? 4 : 8));
    }
}

// Running block amax: max(m, |a|, |b|) for m >= 0 with one 3-input max.  A
// NaN input gives the canonical NaN 0x7fffffff (like any NaN, at or above
// the Inf pattern 0x7f800000 that marks a NaN/Inf block); subnormal inputs are
// kept (no .ftz), so the result's bits equal the integer maximum of the
// magnitude bits for every non-NaN input.
__device__ __forceinline__ float max_abs3(float m, float a, float b) {
    float r;
    asm("{\n\t.reg .f32 ta, tb;\n\tabs.f32 ta, %2;\n\tabs.f32 tb, %3;\n\tmax.NaN.f32 %0, %1, ta, tb;\n\t}"
        : "=f"(r) : "f"(m), "f"(a), "f"(b));
    return r;
}

// MurmurHash3 32-bit finaliser (public domain, A. Appleby), and its steps
// after the first (h ^= h >> 16).
__device__ __forceinline__ uint32_t fmix32_rest(uint32_t h) {
    h *= 0x85ebca6bu;
    h ^= h >> 13;
    h *= 0xc2b2ae35u;
    h ^= h >> 16;
    return h;
}
__device__ __forceinline__ uint32_t fmix32(uint32_t h) { return fmix32_rest(h ^ (h >> 16)); }

// The eight random words of a 32-value block whose first value has
// stochastic-rounding index i0: word w = fmix32((floor(i0 / 4) + w) ^ key),
// whose bytes round values 4w .. 4w + 3.  When i0 is a multiple of 32 the
// words are g .. g + 7 with g a multiple of 8, so (g + w) ^ key = G ^ w for
// G = g ^ key, and the finaliser's first step maps G ^ w to H ^ w for
// H = G ^ (G >> 16) (w < 8 leaves the high half alone): one XOR per word
// replaces the add, the key XOR and that step.
__device__ __forceinline__ void sr_block_words(uint64_t i0, uint32_t key, uint32_t (&rw)[8]) {
    const uint32_t g = static_cast<uint32_t>(i0 >> 2);
    if ((i0 & 31u) == 0) {
        const uint32_t G = g ^ key, H = G ^ (G >> 16);
#pragma unroll
        for (int w = 0; w < 8; ++w) rw[w] = fmix32_rest(H ^ static_cast<uint32_t>(w));
    } else {
#pragma unroll
        for (int w = 0; w < 8; ++w) rw[w] = fmix32((g + static_cast<uint32_t>(w)) ^ key);
    }
}

// Byte offset of the scale of (outer row o, k-block kb) in the MMA layout:
// 512-byte atoms of 128 rows x 4 k-blocks, k-groups fastest; inside an atom
// (o % 32) * 16 + ((o / 32) % 4) * 4 + kb % 4.
__device__ __forceinline__ int64_t mma_scale_offset(int64_t o, int64_t kb, int64_t k_groups) {
    int64_t atom = (o >> 7) * k_groups + (kb >> 2);
    return (atom << 9) + ((o & 31) << 4) + (((o >> 5) & 3) << 2) + (kb & 3);
}

__device__ __forceinline__ uint32_t mma_scale_offset32(uint32_t o, uint32_t kb, uint32_t k_groups) {
    const uint32_t atom = (o >> 7) * k_groups + (kb >> 2);
    return (atom << 9) + ((o & 31u) << 4) + (((o >> 5) & 3u) << 2) + (kb & 3u);
}

// Scale layout codes of the kernels (the mx_scale_layout values).
constexpr int SL_PLAIN = 0, SL_MMA = 1, SL_MMA_X4 = 2;

// Byte offset of the first copy of (o, kb)'s scale in the x4 layout: atoms of
// 2048 bytes, each holding the MMA atom four times.
__device__ __forceinline__ uint32_t x4_scale_offset32(uint32_t o, uint32_t kb, uint32_t k_groups) {
    const uint32_t atom = (o >> 7) * k_groups + (kb >> 2);
    return (atom << 11) + ((o & 31u) << 4) + (((o >> 5) & 3u) << 2) + (kb & 3u);
}

// Debug build (MX_DEBUG, libmx_debug.so): a store or load of `bytes` bytes at
// offset `off` of a buffer of `cap` bytes goes ahead only inside the buffer;
// otherwise this translation unit's bounds word records MX_ERR_BOUNDS (read by
// mx_last_device_status) and the caller skips the access.  The release build
// compiles the check away.
namespace {
__device__ int g_bounds_status;
}
__device__ __forceinline__ bool in_bounds(uint64_t off, uint64_t bytes, uint64_t cap) {
#ifdef MX_DEBUG
    if (off + bytes <= cap) return true;
    atomicExch(&g_bounds_status, MX_ERR_BOUNDS);
    return false;
#else
    (void)off; (void)bytes; (void)cap;
    return true;
#endif
}

// Writes scale byte s of (o, kb) in layout sl (plain rows of k_blocks bytes,
// MMA atoms, or the four copies of the x4 layout) into a buffer of cap bytes.
__device__ __forceinline__ void put_scale(uint8_t *scales, int sl, uint32_t o, uint32_t kb, uint32_t k_blocks,
                                          uint32_t k_groups, uint32_t s, uint64_t cap) {
    if (sl == SL_MMA_X4) {
        const uint32_t off = x4_scale_offset32(o, kb, k_groups);
        if (!in_bounds(off, 3u * 512u + 1u, cap)) return;
#pragma unroll
        for (uint32_t j = 0; j < 4; ++j) scales[off + 512u * j] = static_cast<uint8_t>(s);
    } else {
        const uint32_t off = sl == SL_MMA ? mma_scale_offset32(o, kb, k_groups) : o * k_blocks + kb;
        if (!in_bounds(off, 1, cap)) return;
        scales[off] = static_cast<uint8_t>(s);
    }
}

}  // namespace mxk
