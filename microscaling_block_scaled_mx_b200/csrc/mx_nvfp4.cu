// mx_nvfp4.cu -- the NVFP4 cast: 16-element E2M1 blocks with an E4M3 block
// scale and one fp32 encode scale per scale domain, the "global NVFP4" and
// "cooperative-thread-array-local NVFP4" domains named by the abstract of
// "Format-Aware Fusion for Fast FP4 Pretraining".  The pages do not define
// them; the reading taken (the public NVFP4 format) is stated in include/mx.h
// at mx_quantize_nvfp4.
//
// Kernels (blocks along rows, the K axis of a GEMM operand), the same three
// for both kinds of domain (the global domain is one domain of all rows):
//   nv_amax_kernel   largest finite |x| of each domain: every CTA reduces a
//                    contiguous piece of one domain and adds it to
//                    enc_scales[d] with one atomic max (as bits; non-negative
//                    floats order as their bit patterns)
//   nv_quant_kernel  every block, E from its domain's maximum (the same
//                    pieces, so E is computed once per CTA; the second read of
//                    a tensor that fits in L2 is served from there)
//   nv_final_kernel  enc_scales[d] <- E of domain d
// A domain's blocks are contiguous in row-major order and are split evenly
// over `parts` CTAs, so there are enough CTAs to fill the GPU whether there is
// one domain or thousands.
// Every step is one IEEE fp32 operation (no fused multiply-add, no flush), in
// the order the reading states, so results equal the CPU reference bit for
// bit.
#include <algorithm>
#include <cfloat>
#include <cstdint>
#include <cuda_runtime.h>

#include "mx.h"
#include "mx_device.cuh"
#include "mx_internal.h"

namespace mxnv {

constexpr int NV_BLOCK = 16;
constexpr uint32_t NV_SCALE_NAN = 0x7Fu;
constexpr int THREADS = 256;

struct NvParams {
    const void *x;
    int64_t rows, cols, ldx;
    uint8_t *codes;
    uint8_t *scales;
    int mma;               // scale layout: 0 plain, 1 MMA, 2 MMA x4
    uint32_t k_blocks;     // cols / 16
    uint32_t k_groups;     // ceil(k_blocks / 4)
    float *enc;            // one fp32 per domain
    int64_t lines;         // rows per domain
    int64_t n_dom;         // domains
    int parts;             // CTAs per domain
    uint32_t row_step, kb_step;   // THREADS blocks = row_step rows + kb_step blocks
    uint64_t codes_cap, scales_cap;   // buffer sizes in bytes (checked by the debug build)
};

__device__ __forceinline__ float encode_scale(float amax) {
    if (!(amax > 0.0f)) return 1.0f;
    float e = __fdiv_rn(2688.0f, amax);
    if (isinf(e)) e = FLT_MAX;
    return e;
}

// value of a positive E4M3 code (sign bit clear, not 0x7F)
__device__ __forceinline__ float e4m3_value(uint32_t s) {
    const uint32_t e = (s >> 3) & 15u, m = s & 7u;
    return e == 0 ? static_cast<float>(m) * 0.001953125f                                   // m * 2^-9
                  : __uint_as_float(((e + 120u) << 23) | (m << 20));                       // (1 + m/8) 2^(e-7)
}

// the 16 values of block kb of row `row`, widened to fp32; LAST: the last read
// of these bytes (streaming), else keep them in L2 for the second pass
template <bool BF16_IN, bool LAST>
__device__ __forceinline__ void load_block(const NvParams &p, int64_t row, int64_t kb, float (&v)[NV_BLOCK]) {
    if (BF16_IN) {
        const uint4 *src = reinterpret_cast<const uint4 *>(static_cast<const uint16_t *>(p.x) + row * p.ldx + kb * 16);
        const uint4 a = LAST ? __ldcs(src) : __ldg(src), b = LAST ? __ldcs(src + 1) : __ldg(src + 1);
        const uint32_t w[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            v[2 * i] = __uint_as_float(w[i] << 16);
            v[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
        }
    } else {
        const float4 *src = reinterpret_cast<const float4 *>(static_cast<const float *>(p.x) + row * p.ldx + kb * 16);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const float4 f = LAST ? __ldcs(src + i) : __ldg(src + i);
            v[4 * i] = f.x;
            v[4 * i + 1] = f.y;
            v[4 * i + 2] = f.z;
            v[4 * i + 3] = f.w;
        }
    }
}

// largest finite magnitude; `finite` false when a NaN or Inf is present
__device__ __forceinline__ float block_max(const float (&v)[NV_BLOCK], bool &finite) {
    float m = 0.0f;
    finite = true;
#pragma unroll
    for (int i = 0; i < NV_BLOCK; ++i) {
        const float a = fabsf(v[i]);
        if (!(a <= FLT_MAX)) finite = false;
        else m = fmaxf(m, a);
    }
    return m;
}

template <bool BF16_IN>
__device__ __forceinline__ void quant_block(const NvParams &p, int64_t row, int64_t kb, float E) {
    float v[NV_BLOCK];
    load_block<BF16_IN, true>(p, row, kb, v);
    bool finite;
    const float amax = block_max(v, finite);
    uint32_t s = NV_SCALE_NAN;
    uint2 c = make_uint2(0u, 0u);
    if (finite) {
        const float t = __fmul_rn(__fdiv_rn(amax, 6.0f), E);
        s = mxk::cvt_pair<MX_E4M3>(t, 0.0f) & 0xffu;          // t >= 0: a positive code
        const float d = e4m3_value(s);
        const float r = d > 0.0f ? __fdiv_rn(E, d) : 0.0f;
        uint32_t w[2] = {0u, 0u};
#pragma unroll
        for (int i = 0; i < NV_BLOCK; i += 2) {
            const uint32_t byte = mxk::cvt_pair<MX_E2M1>(__fmul_rn(v[i], r), __fmul_rn(v[i + 1], r));
            w[i >> 3] |= byte << (4 * (i & 7));
        }
        c = make_uint2(w[0], w[1]);
    }
    if (mxk::in_bounds(static_cast<uint64_t>(row * (p.cols / 2) + kb * 8), 8, p.codes_cap))
        *reinterpret_cast<uint2 *>(p.codes + row * (p.cols / 2) + kb * 8) = c;
    mxk::put_scale(p.scales, p.mma, static_cast<uint32_t>(row), static_cast<uint32_t>(kb), p.k_blocks, p.k_groups,
                   s, p.scales_cap);
}

// bf16 input, a block as the 8 words of its 16 values (element 2i in the low
// half of word i).  |x| of a bf16 is its bits with the sign cleared, and
// magnitudes order as those 16-bit integers (Inf and NaN at 0x7F80 and above),
// so the block maximum is a packed 16-bit integer max.
constexpr uint32_t ABS16 = 0x7fff7fffu;
constexpr uint32_t NONFINITE16 = 0x7f80u;

__device__ __forceinline__ uint32_t max_half(uint32_t m) { return max(m & 0xffffu, m >> 16); }

// largest |x| bits of the block (>= 0x7F80 when it holds a NaN or Inf)
__device__ __forceinline__ uint32_t block_max_bits(const uint4 &a, const uint4 &b) {
    uint32_t m = __vimax3_u16x2(a.x & ABS16, a.y & ABS16, a.z & ABS16);
    m = __vimax3_u16x2(m, a.w & ABS16, b.x & ABS16);
    m = __vimax3_u16x2(m, b.y & ABS16, b.z & ABS16);
    return max_half(__vmaxu2(m, b.w & ABS16));
}

// largest finite |x| bits of the block (non-finite values count as zero)
__device__ __forceinline__ uint32_t block_finite_max_bits(const uint4 &a, const uint4 &b) {
    auto fin = [](uint32_t w) {
        const uint32_t h = w & ABS16;
        return h & ~__vcmpgeu2(h, (NONFINITE16 << 16) | NONFINITE16);
    };
    uint32_t m = __vimax3_u16x2(fin(a.x), fin(a.y), fin(a.z));
    m = __vimax3_u16x2(m, fin(a.w), fin(b.x));
    m = __vimax3_u16x2(m, fin(b.y), fin(b.z));
    return max_half(__vmaxu2(m, fin(b.w)));
}

__device__ __forceinline__ uint64_t f2_mul_rn(uint64_t a, uint64_t b) {   // two IEEE fp32 products
    uint64_t r;
    asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
    return r;
}

__device__ __forceinline__ const uint4 *bf16_block_ptr(const NvParams &p, int64_t row, uint32_t kb) {
    return reinterpret_cast<const uint4 *>(static_cast<const uint16_t *>(p.x) + row * p.ldx + kb * 16);
}

// quant_block for bf16 input whose 32 bytes are already loaded
__device__ __forceinline__ void quant_block_bf16(const NvParams &p, int64_t row, uint32_t kb, float E,
                                                 const uint4 &a, const uint4 &b) {
    const uint32_t mb = block_max_bits(a, b);
    uint32_t s = NV_SCALE_NAN;
    uint2 c = make_uint2(0u, 0u);
    if (mb < NONFINITE16) {
        const float amax = __uint_as_float(mb << 16);
        const float t = __fmul_rn(__fdiv_rn(amax, 6.0f), E);
        s = mxk::cvt_pair<MX_E4M3>(t, 0.0f) & 0xffu;          // t >= 0: a positive code
        const float d = e4m3_value(s);
        const float r = d > 0.0f ? __fdiv_rn(E, d) : 0.0f;
        const uint64_t rr = (static_cast<uint64_t>(__float_as_uint(r)) << 32) | __float_as_uint(r);
        const uint32_t w[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
        uint32_t q[2] = {0u, 0u};
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const uint64_t pr = f2_mul_rn((static_cast<uint64_t>(w[i] & 0xffff0000u) << 32) | (w[i] << 16), rr);
            const uint32_t byte = mxk::cvt_pair<MX_E2M1>(__uint_as_float(static_cast<uint32_t>(pr)),
                                                         __uint_as_float(static_cast<uint32_t>(pr >> 32)));
            q[i >> 2] |= byte << (8 * (i & 3));
        }
        c = make_uint2(q[0], q[1]);
    }
    if (mxk::in_bounds(static_cast<uint64_t>(row * (p.cols / 2) + kb * 8), 8, p.codes_cap))
        *reinterpret_cast<uint2 *>(p.codes + row * (p.cols / 2) + kb * 8) = c;
    mxk::put_scale(p.scales, p.mma, static_cast<uint32_t>(row), kb, p.k_blocks, p.k_groups, s, p.scales_cap);
}

// largest value over the CTA (every thread gets it)
__device__ __forceinline__ float cta_max(float m, float *red) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (lane == 0) red[warp] = m;
    __syncthreads();
    if (warp == 0) {
        m = lane < THREADS / 32 ? red[lane] : 0.0f;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
        if (lane == 0) red[0] = m;
    }
    __syncthreads();
    m = red[0];
    __syncthreads();
    return m;
}

// The piece of domain d that this CTA covers: blocks [b0, b1) of the domain,
// counted row-major from its first row r0.
struct Piece {
    int64_t d, r0, b0, b1;
};
__device__ __forceinline__ Piece piece_of(const NvParams &p) {
    Piece q;
    q.d = blockIdx.x / p.parts;
    const int64_t part = blockIdx.x % p.parts;
    q.r0 = q.d * p.lines;
    const int64_t nb = min(p.lines, p.rows - q.r0) * static_cast<int64_t>(p.k_blocks);
    const int64_t chunk = (nb + p.parts - 1) / p.parts;
    q.b0 = min(nb, part * chunk);
    q.b1 = min(nb, q.b0 + chunk);
    return q;
}

// Calls f(row, kb) for this thread's blocks of the piece: block b0 + tid, then
// every THREADS blocks, stepping (row, kb) without a division per block.
template <typename F>
__device__ __forceinline__ void for_each_block(const NvParams &p, const Piece &q, F f) {
    int64_t i = q.b0 + threadIdx.x;
    if (i >= q.b1) return;
    int64_t row = q.r0 + i / p.k_blocks;
    uint32_t kb = static_cast<uint32_t>(i % p.k_blocks);
    for (; i < q.b1; i += THREADS) {
        f(row, kb);
        row += p.row_step;
        kb += p.kb_step;
        if (kb >= p.k_blocks) { kb -= p.k_blocks; ++row; }
    }
}

// bf16: this thread's blocks of the piece with the next block's two loads
// issued before the current block is processed; f(row, kb, a, b)
template <bool LAST, typename F>
__device__ __forceinline__ void for_each_bf16_block(const NvParams &p, const Piece &q, F f) {
    int64_t i = q.b0 + threadIdx.x;
    if (i >= q.b1) return;
    int64_t row = q.r0 + i / p.k_blocks;
    uint32_t kb = static_cast<uint32_t>(i % p.k_blocks);
    const uint4 *src = bf16_block_ptr(p, row, kb);
    uint4 a = LAST ? __ldcs(src) : __ldg(src), b = LAST ? __ldcs(src + 1) : __ldg(src + 1);
    for (; i < q.b1; i += THREADS) {
        int64_t row_n = row + p.row_step;
        uint32_t kb_n = kb + p.kb_step;
        if (kb_n >= p.k_blocks) { kb_n -= p.k_blocks; ++row_n; }
        uint4 an = a, bn = b;
        if (i + THREADS < q.b1) {
            const uint4 *nx = bf16_block_ptr(p, row_n, kb_n);
            an = LAST ? __ldcs(nx) : __ldg(nx);
            bn = LAST ? __ldcs(nx + 1) : __ldg(nx + 1);
        }
        f(row, kb, a, b);
        row = row_n;
        kb = kb_n;
        a = an;
        b = bn;
    }
}

template <bool BF16_IN>
__global__ void __launch_bounds__(THREADS) nv_amax_kernel(NvParams p) {
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    asm volatile("griddepcontrol.wait;" ::: "memory");
    __shared__ float red[THREADS / 32];
    const Piece q = piece_of(p);
    float m = 0.0f;
    if constexpr (BF16_IN) {
        uint32_t mb = 0;
        for_each_bf16_block<false>(p, q, [&](int64_t, uint32_t, const uint4 &a, const uint4 &b) {
            mb = max(mb, block_finite_max_bits(a, b));
        });
        m = __uint_as_float(mb << 16);
    } else {
        for_each_block(p, q, [&](int64_t row, uint32_t kb) {
            float v[NV_BLOCK];
            load_block<BF16_IN, false>(p, row, kb, v);
            bool finite;
            m = fmaxf(m, block_max(v, finite));
        });
    }
    m = cta_max(m, red);
    if (threadIdx.x == 0) atomicMax(reinterpret_cast<unsigned int *>(p.enc + q.d), __float_as_uint(m));
}

template <bool BF16_IN>
__global__ void __launch_bounds__(THREADS) nv_quant_kernel(NvParams p) {
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    asm volatile("griddepcontrol.wait;" ::: "memory");
    const Piece q = piece_of(p);
    const float E = encode_scale(p.enc[q.d]);             // enc[d] holds the domain's maximum here
    if constexpr (BF16_IN)
        for_each_bf16_block<true>(p, q, [&](int64_t row, uint32_t kb, const uint4 &a, const uint4 &b) {
            quant_block_bf16(p, row, kb, E, a, b);
        });
    else
        for_each_block(p, q, [&](int64_t row, uint32_t kb) { quant_block<BF16_IN>(p, row, kb, E); });
}

__global__ void __launch_bounds__(THREADS) nv_final_kernel(float *enc, int64_t n_dom) {
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    asm volatile("griddepcontrol.wait;" ::: "memory");
    const int64_t d = blockIdx.x * static_cast<int64_t>(THREADS) + threadIdx.x;
    if (d < n_dom) enc[d] = encode_scale(enc[d]);
}

template <auto Kernel, typename... Args>
cudaError_t launch(int grid, cudaStream_t st, Args... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(THREADS);
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, Kernel, args...);
}

template <bool BF16_IN>
cudaError_t run(const NvParams &p, cudaStream_t st) {
    // the maxima accumulate in enc_scales, which start at zero
    cudaError_t e = cudaMemsetAsync(p.enc, 0, static_cast<size_t>(p.n_dom) * sizeof(float), st);
    if (e != cudaSuccess) return e;
    const int grid = static_cast<int>(p.n_dom * p.parts);
    if ((e = launch<nv_amax_kernel<BF16_IN>>(grid, st, p)) != cudaSuccess) return e;
    if ((e = launch<nv_quant_kernel<BF16_IN>>(grid, st, p)) != cudaSuccess) return e;
    return launch<nv_final_kernel>(static_cast<int>((p.n_dom + THREADS - 1) / THREADS), st, p.enc, p.n_dom);
}

}  // namespace mxnv

cudaError_t mx_launch_quantize_nvfp4(const MxNvfp4Args &a, cudaStream_t st) {
    using namespace mxnv;
    NvParams p;
    p.x = a.x;
    p.rows = a.rows;
    p.cols = a.cols;
    p.ldx = a.ldx;
    p.codes = static_cast<uint8_t *>(a.codes);
    p.scales = static_cast<uint8_t *>(a.scales);
    p.mma = a.sl;
    p.k_blocks = static_cast<uint32_t>(a.cols / NV_BLOCK);
    p.k_groups = (p.k_blocks + 3) / 4;
    p.codes_cap = static_cast<uint64_t>(a.rows) * static_cast<uint64_t>(a.cols / 2);
    p.scales_cap = mx_nvfp4_scales_bytes(static_cast<mx_scale_layout>(a.sl), a.rows, a.cols);
    p.enc = a.enc_scales;
    p.lines = (a.domain_rows == 0 || a.domain_rows > a.rows) ? a.rows : a.domain_rows;
    p.n_dom = (a.rows + p.lines - 1) / p.lines;
    // about eight CTAs of THREADS per SM over all domains, at least one per domain
    const int64_t target = static_cast<int64_t>(a.num_sms) * 8;
    const int64_t per_dom = p.lines * static_cast<int64_t>(p.k_blocks);
    int64_t parts = (target + p.n_dom - 1) / p.n_dom;
    parts = std::min<int64_t>(parts, (per_dom + THREADS - 1) / THREADS);   // no CTA without a block
    p.parts = static_cast<int>(std::max<int64_t>(parts, 1));
    if (p.n_dom * p.parts > 0x7fffffffll) return cudaErrorInvalidConfiguration;
    p.row_step = static_cast<uint32_t>(THREADS / p.k_blocks);
    p.kb_step = static_cast<uint32_t>(THREADS % p.k_blocks);
    return a.xdt == MX_BF16 ? run<true>(p, st) : run<false>(p, st);
}

// Reads and clears this unit's debug-build bounds word (after the caller
// synchronised).
int mx_read_nvfp4_bounds_status() {
    int b = 0;
    if (cudaMemcpyFromSymbol(&b, mxk::g_bounds_status, sizeof(int)) != cudaSuccess) return MX_ERR_CUDA;
    const int zero = 0;
    if (cudaMemcpyToSymbol(mxk::g_bounds_status, &zero, sizeof(int)) != cudaSuccess) return MX_ERR_CUDA;
    return b;
}
