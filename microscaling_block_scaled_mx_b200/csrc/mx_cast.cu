// mx_cast.cu -- MX cast (Algorithm 1 of "Microscaling Data Formats for Deep
// Learning", summary page, section 3) and exact decode (section 2) on sm_100a.
//
// The casts are streaming kernels: every input byte is read once, every code
// and scale byte written once (a scale byte four times in the x4 layout, one
// per copy of its atom).
//  * cast_rows: blocks run along the contiguous axis.  One lane owns one
//    32-block (two 32-byte loads for bf16); a warp covers 32 consecutive
//    blocks of a row, with the next two chunks' loads in flight in a ring of
//    register slots.
//  * cast_cols: blocks run down columns.  A CTA stages 128 x 128 tiles in
//    shared memory (double-buffered; one TMA tensor copy per tile, or 16-byte
//    cp.async copies when the input is not 16-byte aligned); each thread owns one column
//    pair of a 32-row block, where the optional fixed-sign 32-point Hadamard
//    ("Format-Aware Fusion for Fast FP4 Pretraining", abstract) runs as five
//    packed fp32 butterfly stages, and writes its codes as rows of the
//    transposed (block-axis-major) output.
//  * cast_dual: both of the above from one staged tile.
#include <cstdint>
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "mx.h"
#include "mx_device.cuh"
#include "mx_encode.cuh"
#include "mx_debug.h"
#include "mx_internal.h"

namespace mxk {

struct CastParams {
    const void *x;
    int64_t rows, cols, ldx;
    uint8_t *codes;
    uint8_t *scales;
    int mma_scales;      // scale layout: 0 plain, 1 MMA, 2 MMA x4
    int64_t k_blocks;    // blocks per output row (inner / 32)
    int64_t k_groups;    // ceil(k_blocks / 4), MMA layout
    uint32_t key;        // stochastic-rounding seed key
    uint32_t sign_mask;  // Hadamard signs
    // stochastic-rounding position of output element (o, i): sr_base + o * sr_stride + i
    uint64_t sr_base, sr_stride;
    int skip_first;      // testing hook: CTA 0 withholds the copy of its first staged tile
    int stage_scales;    // column casts: a full tile's scale atom goes out through shared memory
    uint64_t codes_cap, scales_cap;   // buffer sizes in bytes (checked by the debug build)
};

__device__ __forceinline__ void store_scale(const CastParams &p, int64_t o, int64_t kb, uint32_t s) {
    // scale buffers are far below 4 GiB: offsets in 32-bit arithmetic
    put_scale(p.scales, p.mma_scales, static_cast<uint32_t>(o), static_cast<uint32_t>(kb),
              static_cast<uint32_t>(p.k_blocks), static_cast<uint32_t>(p.k_groups), s, p.scales_cap);
}

// ---------------------------------------------------------------------------
// Row cast: block axis contiguous.
// ---------------------------------------------------------------------------
// One lane owns one 32-block (64 bytes of bf16: two 32-byte loads, or four
// 16-byte loads when rows are not 32-byte aligned), so the block's amax,
// exponent, scale byte and addresses are computed once per 32 values; a warp
// covers 32 consecutive blocks (1024 values) of one row.  The loads of the
// next two chunks are in flight while the current chunk is converted.
template <bool BF16_IN>
struct BlockLoad {
    uint4 w[BF16_IN ? 4 : 8];
};

struct ChunkPos {
    int64_t row, chunk;   // chunk = 32 consecutive blocks of one row
};

// 32-byte global load (two uint4), streaming: no L1 allocation
__device__ __forceinline__ void ld32_stream(const void *src, uint4 &a, uint4 &b) {
    asm volatile("ld.global.nc.L1::no_allocate.v8.u32 {%0, %1, %2, %3, %4, %5, %6, %7}, [%8];"
                 : "=r"(a.x), "=r"(a.y), "=r"(a.z), "=r"(a.w), "=r"(b.x), "=r"(b.y), "=r"(b.z), "=r"(b.w)
                 : "l"(src));
}

// V32: the input rows are 32-byte aligned, so each lane fetches its block with
// 32-byte loads (every sector a load touches is used in full).
template <bool BF16_IN, bool V32>
__device__ __forceinline__ void load_block(const CastParams &p, const ChunkPos &cp, int64_t blocks_per_row, int lane,
                                           BlockLoad<BF16_IN> &o) {
    constexpr int NW = BF16_IN ? 4 : 8;
    const int64_t kb = cp.chunk * 32 + lane;
    if (cp.row < p.rows && kb < blocks_per_row) {
        constexpr int EB = BF16_IN ? 2 : 4;
        const uint4 *src = reinterpret_cast<const uint4 *>(static_cast<const uint8_t *>(p.x) +
                                                           (cp.row * p.ldx + kb * 32) * EB);
        if (V32) {
#pragma unroll
            for (int i = 0; i < NW; i += 2) ld32_stream(src + i, o.w[i], o.w[i + 1]);
        } else {
#pragma unroll
            for (int i = 0; i < NW; ++i) o.w[i] = __ldcs(src + i);
        }
    } else {
#pragma unroll
        for (int i = 0; i < NW; ++i) o.w[i] = make_uint4(0, 0, 0, 0);
    }
}

// The row cast's blocks go to the shared 32-block encoder (mx_encode.cuh).
__device__ __forceinline__ BlockSink row_sink(const CastParams &p) {
    BlockSink o;
    o.codes = p.codes;
    o.scales = p.scales;
    o.inner = p.cols;
    o.k_blocks = static_cast<uint32_t>(p.k_blocks);
    o.k_groups = static_cast<uint32_t>(p.k_groups);
    o.mma_scales = p.mma_scales;
    o.key = p.key;
    o.sr_base = p.sr_base;
    o.sr_stride = p.sr_stride;
    o.codes_cap = p.codes_cap;
    o.scales_cap = p.scales_cap;
    return o;
}

template <int FMT, bool SR, bool V32>
__device__ __forceinline__ void encode_row_block(const CastParams &p, int64_t row, int64_t kb, uint32_t (&b)[32]) {
    encode_block32<FMT, SR, V32>(row_sink(p), row, kb, b);
}
template <int FMT, bool SR, bool V32>
__device__ __forceinline__ void encode_row_block(const CastParams &p, int64_t row, int64_t kb, uint32_t (&b)[32],
                                                 uint32_t amax_bits) {
    encode_block32_amax<FMT, SR, V32>(row_sink(p), row, kb, b, amax_bits);
}

template <int FMT, bool SR, bool BF16_IN, bool V32>
__device__ __forceinline__ void cast_block(const CastParams &p, const ChunkPos &cp, int64_t blocks_per_row,
                                           const BlockLoad<BF16_IN> &o, int lane) {
    const int64_t kb = cp.chunk * 32 + lane;
    if (cp.row >= p.rows || kb >= blocks_per_row) return;
    // the 32 values as fp32 bit patterns
    uint32_t b[32];
    if (BF16_IN) {
        uint32_t words[16];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const uint32_t ws[4] = {o.w[i].x, o.w[i].y, o.w[i].z, o.w[i].w};
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                words[4 * i + k] = ws[k];
                b[8 * i + 2 * k] = ws[k] << 16;
                b[8 * i + 2 * k + 1] = ws[k] & 0xffff0000u;
            }
        }
        encode_row_block<FMT, SR, V32>(p, cp.row, kb, b, bf16_max_bits(bf16_pair_max<16>(words)));
        return;
    } else {
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            b[4 * i] = o.w[i].x; b[4 * i + 1] = o.w[i].y; b[4 * i + 2] = o.w[i].z; b[4 * i + 3] = o.w[i].w;
        }
    }
    encode_row_block<FMT, SR, V32>(p, cp.row, kb, b);
}

template <int FMT, bool SR, bool BF16_IN, bool V32>
__global__ void __launch_bounds__(256, 2) cast_rows_kernel(CastParams p) {
    constexpr int DIST = 2;                               // chunks in flight while one is converted
    const int lane = threadIdx.x & 31;
    const int64_t blocks_per_row = p.cols >> 5;
    const int64_t cpr = (blocks_per_row + 31) >> 5;      // chunks per row
    const int64_t warp0 = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
    const int64_t n_warps = (static_cast<int64_t>(gridDim.x) * blockDim.x) >> 5;
    const int64_t step_rows = n_warps / cpr, step_chunk = n_warps - step_rows * cpr;
    auto advance = [&](ChunkPos &q) {
        q.chunk += step_chunk;
        q.row += step_rows;
        if (q.chunk >= cpr) { q.chunk -= cpr; ++q.row; }
    };
    // Programmatic dependent launch: let the next kernel in the stream start
    // placing its CTAs as this grid's CTAs finish, and touch no global memory
    // before the grid this one depends on has completed and flushed.
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    asm volatile("griddepcontrol.wait;" ::: "memory");
    // a ring of DIST + 1 load slots, indexed statically by unrolling one turn
    // of the ring: slot u is converted while slot (u + DIST) % (DIST + 1) loads
    ChunkPos pos[DIST + 1];
    BlockLoad<BF16_IN> ld[DIST + 1];
    pos[0].row = warp0 / cpr;
    pos[0].chunk = warp0 - pos[0].row * cpr;
#pragma unroll
    for (int i = 1; i <= DIST; ++i) {
        pos[i] = pos[i - 1];
        advance(pos[i]);
    }
#pragma unroll
    for (int i = 0; i < DIST; ++i) load_block<BF16_IN, V32>(p, pos[i], blocks_per_row, lane, ld[i]);
    for (;;) {
#pragma unroll
        for (int u = 0; u <= DIST; ++u) {
            constexpr int NEXT = DIST;                    // slot offset of the chunk to load
            const int nxt = (u + NEXT) % (DIST + 1);
            if (pos[u].row >= p.rows) return;
            load_block<BF16_IN, V32>(p, pos[nxt], blocks_per_row, lane, ld[nxt]);
            cast_block<FMT, SR, BF16_IN, V32>(p, pos[u], blocks_per_row, ld[u], lane);
            pos[u] = pos[nxt];                            // this slot's next chunk: one after pos[nxt]
            advance(pos[u]);
        }
    }
}

// ---------------------------------------------------------------------------
// Column cast: block axis strided, output transposed.
// ---------------------------------------------------------------------------
// A CTA owns a 128-row x 128-column input tile at a time, staged in shared
// memory by 16-byte cp.async copies (zero-filled outside the tensor) into one
// of two buffers, so the next tile streams in while the current one is
// converted.  Each thread owns two adjacent columns of one 32-row block: one
// 4- or 8-byte shared load feeds both, and the Hadamard butterflies run as
// packed f32x2 adds on the pair.
constexpr int COL_TILE_R = 128;   // 4 blocks down
constexpr int COL_TILE_C = 128;   // 64 column pairs
constexpr int COL_THREADS = 256;  // 64 pairs x 4 blocks

__device__ __forceinline__ uint64_t f2_pack(float lo, float hi) {
    return static_cast<uint64_t>(__float_as_uint(lo)) | (static_cast<uint64_t>(__float_as_uint(hi)) << 32);
}
__device__ __forceinline__ uint64_t f2_add(uint64_t a, uint64_t b) {
    uint64_t r;
    asm("add.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
    return r;
}
__device__ __forceinline__ uint64_t f2_sub(uint64_t a, uint64_t b) {
    uint64_t r;
    asm("sub.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
    return r;
}
__device__ __forceinline__ uint64_t f2_mul(uint64_t a, uint64_t b) {   // exact uses only (x +-1)
    uint64_t r;
    asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
    return r;
}

__device__ __forceinline__ void cp_async16(uint32_t dst, const void *src, uint32_t src_bytes) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(src_bytes) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait_prev() { asm volatile("cp.async.wait_group 1;" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_group 0;" ::: "memory"); }

// Tile staging by the tensor-memory-access (TMA) engine: one thread issues a
// tensor copy per tile (per 128-byte-wide box for the swizzled dual-cast
// layout) that completes on the buffer's mbarrier; every thread waits on that
// barrier.  Compared with 16-byte cp.async copies this takes the per-chunk
// address, bounds and zero-fill arithmetic off every thread (the copy engine
// fills the part of a box outside the tensor with zeros).
__device__ int g_cast_status;   // MX_ERR_TIMEOUT once a staging wait gave up

constexpr unsigned long long STAGE_WAIT_NS = 2000000000ull;    // 2 s per tile wait
constexpr unsigned long long STAGE_DRAIN_NS = 200000000ull;    // 0.2 s for copies in flight after that

__device__ __forceinline__ void stage_bar_init(uint32_t bar) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(bar) : "memory");
}
__device__ __forceinline__ void stage_expect(uint32_t bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes) : "memory");
}
__device__ __forceinline__ void tma_tile_load(uint32_t dst, const CUtensorMap *map, int x, int y, uint32_t bar) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];"
        ::"r"(dst), "l"(map), "r"(x), "r"(y), "r"(bar) : "memory");
}
__device__ __forceinline__ bool stage_try_wait(uint32_t bar, uint32_t parity) {
    uint32_t ok;
    asm volatile("{\n\t.reg .pred p;\n\tmbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
                 "selp.u32 %0, 1, 0, p;\n\t}"
                 : "=r"(ok) : "r"(bar), "r"(parity) : "memory");
    return ok != 0;
}
// Bounded wait for phase `parity` of a staging barrier: false after `limit`
// ns, with the timeout recorded in the status word (read by
// mx_last_device_status).
__device__ __noinline__ bool stage_wait_slow(uint32_t bar, uint32_t parity, unsigned long long limit) {
    unsigned long long t0;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t0));
    for (uint32_t it = 0;; ++it) {
        if (stage_try_wait(bar, parity)) return true;
        if ((it & 63u) == 63u) {
            unsigned long long t;
            asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
            if (t - t0 > limit) {
                atomicExch(&g_cast_status, MX_ERR_TIMEOUT);
                return false;
            }
        }
    }
}
__device__ __forceinline__ bool stage_wait(uint32_t bar, uint32_t parity, unsigned long long limit = STAGE_WAIT_NS) {
    return stage_try_wait(bar, parity) || stage_wait_slow(bar, parity, limit);
}

// Shared-memory layout of a staged tile: the buffers start at the first
// ALIGN boundary of the dynamic buffer (1024 bytes for the 128-byte swizzle,
// whose pattern repeats every 1024 bytes), followed by one mbarrier per buffer
// and two 512-byte scale atoms (one per buffer).  The cp.async path uses the
// same layout with ALIGN's slack left unused.
template <int ALIGN>
struct StagedTiles {
    uint8_t *tiles;     // generic pointer to buffer 0
    uint32_t base;      // its shared-memory address
    uint32_t bars;      // barrier of buffer b at bars + 8 b
    uint8_t *atoms;     // scale atom of buffer b at atoms + 512 b
    __device__ StagedTiles(uint8_t *raw, int tile_bytes) {
        const uint32_t r = static_cast<uint32_t>(__cvta_generic_to_shared(raw));
        base = (r + ALIGN - 1) & ~static_cast<uint32_t>(ALIGN - 1);
        tiles = raw + (base - r);
        bars = base + 2 * tile_bytes;
        atoms = tiles + 2 * tile_bytes + 16;
    }
};

// Shared-memory position of 16-byte chunk q of tile row rr.  Unswizzled for
// the column cast.  The dual cast, which also reads 32-element row segments,
// XORs the chunk's index inside its 128-byte span with the span index and the
// row's parity, so both its column reads (a warp reads 128 contiguous bytes of
// one row) and its row reads (eight lanes read the same chunk of 2 rows x 4
// row blocks) touch distinct banks.
template <bool BF16_IN, bool SWZ>
__device__ __forceinline__ int tile_chunk(int rr, int q) {
    if (!SWZ) return q;
    constexpr int SH = BF16_IN ? 1 : 2;                      // spans per row: 2 (bf16), 4 (fp32)
    return q ^ (((rr & 1) << SH) | (q >> 3));
}

template <bool BF16_IN, bool SWZ = false>
__device__ __forceinline__ void stage_tile(const CastParams &p, uint8_t *buf, int64_t r0, int64_t c0) {
    using TIn = typename std::conditional<BF16_IN, uint16_t, float>::type;
    constexpr int EPC = 16 / sizeof(TIn);                   // elements per 16-byte chunk
    constexpr int CPR = COL_TILE_C / EPC;                   // chunks per tile row
    const TIn *x = static_cast<const TIn *>(p.x);
    const uint32_t sbuf = static_cast<uint32_t>(__cvta_generic_to_shared(buf));
    for (int ch = threadIdx.x; ch < COL_TILE_R * CPR; ch += COL_THREADS) {
        const int rr = ch / CPR, q = ch % CPR, cc = q * EPC;
        const int64_t gr = r0 + rr, gc = c0 + cc;
        int64_t valid = (gr < p.rows) ? (p.cols - gc) : 0;
        valid = valid < 0 ? 0 : (valid > EPC ? EPC : valid);
        const TIn *src = valid > 0 ? x + gr * p.ldx + gc : x;
        cp_async16(sbuf + rr * COL_TILE_C * sizeof(TIn) + tile_chunk<BF16_IN, SWZ>(rr, q) * 16, src,
                   static_cast<uint32_t>(valid * sizeof(TIn)));
    }
}

// Encode the two column blocks (columns gc, gc + 1; rows gr0 .. gr0 + 31) held
// as packed f32x2 values x[j] = (column gc, column gc + 1) at row gr0 + j:
// optional fixed-sign Hadamard, amax -> E8M0, exact scaling with the FP32
// subnormal flush, RNE or stochastic rounding, and the codes as rows gc and
// gc + 1 of the transposed output.  SR's index is the element's position
// sr_base + (gc + col) * sr_stride + gr0 + j in the whole tensor's output
// (sr_base 0 and sr_stride = rows for a whole tensor).
// KEYED: the caller passes the packed 16-bit maxima of |bf16| of the two
// columns (bf16_pair_max over the raw words), valid without the Hadamard.
// Sign flip of the fixed-sign Hadamard with the default mask, applied while
// loading: row j of a block is negated (both columns of the pair, an exact
// sign-bit flip, the same as multiplying by -1) unless bit j of the mask is
// set.  With the mask a compile-time constant this is one XOR on half of the
// rows and nothing on the others.
__device__ __forceinline__ constexpr bool default_mask_negates(int j) {
    return ((MX_DEFAULT_SIGN_MASK >> j) & 1u) == 0u;
}

// SIGNED: the caller has already applied the Hadamard's sign flips to x
// (the default mask, folded into the loads).
// satom: when set, the scale bytes go to this 512-byte shared-memory copy of
// the tile's scale atom (the caller writes the atom out), else to global memory.
template <int FMT, bool SR, bool HAD, bool KEYED = false, bool SIGNED = false>
__device__ __forceinline__ void encode_col_pair(const CastParams &p, uint64_t (&x)[32], int64_t gc, int64_t gr0,
                                                uint32_t pair_max16 = 0, uint8_t *satom = nullptr) {
    static_assert(!(KEYED && HAD), "the bf16 maxima describe the values before the Hadamard");
    constexpr int BITS = Fmt<FMT>::bits;
    const int64_t R = p.rows, C = p.cols;
    if (HAD) {
        if (!SIGNED) {
#pragma unroll
            for (int j = 0; j < 32; ++j) {
                const float sg = ((p.sign_mask >> j) & 1u) ? 1.0f : -1.0f;
                x[j] = f2_mul(x[j], f2_pack(sg, sg));
            }
        }
#pragma unroll
        for (int h = 1; h < 32; h <<= 1) {
#pragma unroll
            for (int i = 0; i < 32; ++i) {
                if (i & h) continue;
                const uint64_t a = x[i], b = x[i + h];
                x[i] = f2_add(a, b);
                x[i + h] = f2_sub(a, b);
            }
        }
    }
    const bool has_second = gc + 1 < C;
    // block amax and exponent of both columns
    uint32_t am0 = 0, am1 = 0;
    if (KEYED) {
        am0 = pair_max16 << 16;
        am1 = pair_max16 & 0xffff0000u;
    } else {
        float m0 = 0.0f, m1 = 0.0f;
#pragma unroll
        for (int j = 0; j < 32; j += 2) {
            m0 = max_abs3(m0, __uint_as_float(static_cast<uint32_t>(x[j])), __uint_as_float(static_cast<uint32_t>(x[j + 1])));
            m1 = max_abs3(m1, __uint_as_float(static_cast<uint32_t>(x[j] >> 32)),
                          __uint_as_float(static_cast<uint32_t>(x[j + 1] >> 32)));
        }
        am0 = __float_as_uint(m0);
        am1 = __float_as_uint(m1);
    }
    const int e0 = block_exponent<FMT>(am0), e1 = block_exponent<FMT>(am1);
    // V * 2^-e for both columns with one packed multiply (flushing
    // FP32 subnormals); INT8's e = 127 case takes the two-step path
    const bool packed = Fmt<FMT>::emax != 0 || (e0 <= 126 && e1 <= 126);
    if (packed) {
        const uint64_t ff = f2_pack(pow2f(-e0), pow2f(-e1));
#pragma unroll
        for (int j = 0; j < 32; ++j) x[j] = f2_mul_ftz(x[j], ff);
    }
#pragma unroll
    for (int col = 0; col < 2; ++col) {
        if (col == 1 && !has_second) break;
        const uint32_t amax_bits = col ? am1 : am0;
        const int e = col ? e1 : e0;
        const bool nan_block = amax_bits >= 0x7f800000u;
        float v[32];
#pragma unroll
        for (int j = 0; j < 32; ++j) {
            v[j] = __uint_as_float(static_cast<uint32_t>(x[j] >> (32 * col)));
            if (!packed) v[j] = scale_down<FMT>(v[j], e);
        }
        const int64_t oc = gc + col;                 // output row
        // pw[w]: the codes of values 4w .. 4w + 3, one per byte (per nibble for E2M1)
        constexpr int SLOT = BITS == 4 ? 4 : 8;
        uint32_t pw[8];
        if (SR) {
            uint32_t rw[8];
            sr_block_words(p.sr_base + static_cast<uint64_t>(oc) * p.sr_stride + static_cast<uint64_t>(gr0), p.key, rw);
#pragma unroll
            for (int w = 0; w < 8; ++w)
                pw[w] = sr_quad<FMT>(v[4 * w], v[4 * w + 1], v[4 * w + 2], v[4 * w + 3], rw[w]);
        } else {
#pragma unroll
            for (int w = 0; w < 8; ++w)
                pw[w] = cvt_pair<FMT>(v[4 * w], v[4 * w + 1]) | (cvt_pair<FMT>(v[4 * w + 2], v[4 * w + 3]) << (2 * SLOT));
        }
        const uint32_t keep = nan_block ? 0u : 0xffffffffu;     // a NaN/Inf block stores zero codes
        if (!in_bounds(static_cast<uint64_t>(oc * (R * BITS / 8) + gr0 * BITS / 8), 32 * BITS / 8, p.codes_cap)) {
            // (debug build) the block's codes fall outside the buffer: skip them
        } else if (BITS == 8) {
            uint4 *dst = reinterpret_cast<uint4 *>(p.codes + oc * R + gr0);
            dst[0] = make_uint4(pw[0] & keep, pw[1] & keep, pw[2] & keep, pw[3] & keep);
            dst[1] = make_uint4(pw[4] & keep, pw[5] & keep, pw[6] & keep, pw[7] & keep);
        } else if (BITS == 4) {
            uint32_t w[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) w[i] = (pw[2 * i] | (pw[2 * i + 1] << 16)) & keep;
            *reinterpret_cast<uint4 *>(p.codes + oc * (R >> 1) + (gr0 >> 1)) = make_uint4(w[0], w[1], w[2], w[3]);
        } else {
            uint64_t *dst = reinterpret_cast<uint64_t *>(p.codes + oc * (R / 4 * 3) + gr0 / 4 * 3);
#pragma unroll
            for (int q = 0; q < 3; ++q) {     // 3 words of 64 bits = 32 codes of 6 bits
                uint64_t w = 0;
#pragma unroll
                for (int j = 0; j < 32; ++j) {
                    const int bit = 6 * j - 64 * q;
                    const uint64_t code = (pw[j >> 2] >> (8 * (j & 3))) & 0x3fu;
                    if (bit >= 0 && bit < 64) w |= code << bit;
                    else if (bit < 0 && bit > -6) w |= code >> (-bit);
                }
                dst[q] = w & (static_cast<uint64_t>(keep) << 32 | keep);
            }
        }
        const uint32_t sbyte = nan_block ? 0xffu : static_cast<uint32_t>(e + 127);
        if (satom)
            satom[((oc & 31) << 4) + (((oc >> 5) & 3) << 2) + ((gr0 >> 5) & 3)] = static_cast<uint8_t>(sbyte);
        else
            store_scale(p, oc, gr0 >> 5, sbyte);
    }
}

// A column tile's scales: 128 columns (outer rows of the output) x 4 blocks
// down the tile, exactly one 512-byte atom of the MMA layout (the tile's first
// column and row are multiples of 128).  For a full tile the encoders write
// the atom's bytes into shared memory and, after the tile's barrier, warp j
// writes copy j of it (one copy in the MMA layout, four in the x4 layout) with
// one 16-byte store per lane: 16 or 64 whole 32-byte sectors per tile instead
// of 512 or 2048 scattered single bytes.
__device__ __forceinline__ bool tile_stages_scales(const CastParams &p, int64_t r0, int64_t c0) {
    return p.stage_scales && r0 + COL_TILE_R <= p.rows && c0 + COL_TILE_C <= p.cols;
}
__device__ __forceinline__ void write_scale_atom(const CastParams &p, const uint8_t *satom, int64_t r0, int64_t c0,
                                                 int warp, int lane) {
    const int copies = p.mma_scales == SL_MMA_X4 ? 4 : 1;
    if (warp >= copies) return;
    const int64_t atom = (c0 >> 7) * p.k_groups + (r0 >> 7);
    const int64_t off = (atom << (copies == 4 ? 11 : 9)) + warp * 512;
    if (!in_bounds(static_cast<uint64_t>(off), 512, p.scales_cap)) return;
    reinterpret_cast<uint4 *>(p.scales + off)[lane] = reinterpret_cast<const uint4 *>(satom)[lane];
}

// After a staging wait gave up at tile use `use` (buffer `buf`): wait, again
// bounded, for the copies that may still be landing in shared memory (that
// tile's, and the next one's if it was issued) before the CTA exits.
__device__ __noinline__ void drain_staged(uint32_t bars, int buf, uint32_t use, bool next_issued) {
    (void)stage_wait(bars + 8 * buf, (use >> 1) & 1u, STAGE_DRAIN_NS);
    if (next_issued) (void)stage_wait(bars + 8 * (buf ^ 1), ((use + 1) >> 1) & 1u, STAGE_DRAIN_NS);
}

// DEFM: the Hadamard uses the default sign mask, folded into the loads.
// TMA: tiles staged by tensor copies of `tmap` (the input as a rows x cols
// tensor, boxes of 128 x 128), else by cp.async.
template <int FMT, bool SR, bool BF16_IN, bool HAD, bool DEFM, bool TMA>
__global__ void __launch_bounds__(COL_THREADS, 2) cast_cols_kernel(CastParams p, const __grid_constant__ CUtensorMap tmap) {
    using TIn = typename std::conditional<BF16_IN, uint16_t, float>::type;
    constexpr int TILE_BYTES = COL_TILE_R * COL_TILE_C * sizeof(TIn);
    extern __shared__ __align__(16) uint8_t col_smem[];
    const StagedTiles<128> st(col_smem, TILE_BYTES);
    uint8_t *const tiles = TMA ? st.tiles : col_smem;

    const int64_t R = p.rows, C = p.cols;
    const int64_t tiles_r = (R + COL_TILE_R - 1) / COL_TILE_R;
    const int64_t tiles_c = (C + COL_TILE_C - 1) / COL_TILE_C;
    const int64_t n_tiles = tiles_r * tiles_c;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int blk = warp & 3;                       // 32-row block inside the tile
    const int pair = (warp >> 2) * 32 + lane;       // column pair inside the tile
    // thread 0: the copy of tile `tile` into buffer b (TMA staging)
    auto issue = [&](int64_t tile, int b) {
        stage_expect(st.bars + 8 * b, TILE_BYTES);
        tma_tile_load(st.base + b * TILE_BYTES, &tmap, static_cast<int>((tile % tiles_c) * COL_TILE_C),
                      static_cast<int>((tile / tiles_c) * COL_TILE_R), st.bars + 8 * b);
    };
    if (TMA) {
        if (threadIdx.x == 0) {
            stage_bar_init(st.bars);
            stage_bar_init(st.bars + 8);
            asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        }
        __syncthreads();
    }

    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    asm volatile("griddepcontrol.wait;" ::: "memory");     // inputs of the previous kernel are visible
    int64_t t = blockIdx.x;
    if (TMA) {
        if (t < n_tiles && threadIdx.x == 0 && !(p.skip_first && blockIdx.x == 0)) issue(t, 0);
    } else {
        if (t < n_tiles) stage_tile<BF16_IN>(p, col_smem, (t / tiles_c) * COL_TILE_R, (t % tiles_c) * COL_TILE_C);
        cp_async_commit();
    }
    uint32_t use = 0;                // tiles this CTA has taken: buffer use % 2, phase (use / 2) % 2
    bool ok = true;
    for (int buf = 0; t < n_tiles; t += gridDim.x, buf ^= 1, ++use) {
        const int64_t tn = t + gridDim.x;
        if (TMA) {
            if (tn < n_tiles && threadIdx.x == 0) issue(tn, buf ^ 1);
            ok = stage_wait(st.bars + 8 * buf, (use >> 1) & 1u);
        } else {
            if (tn < n_tiles)
                stage_tile<BF16_IN>(p, col_smem + (buf ^ 1) * TILE_BYTES, (tn / tiles_c) * COL_TILE_R,
                                    (tn % tiles_c) * COL_TILE_C);
            cp_async_commit();
            cp_async_wait_prev();        // this tile's copies (the older group) have landed
            __syncthreads();
        }

        const int64_t r0 = (t / tiles_c) * COL_TILE_R, c0 = (t % tiles_c) * COL_TILE_C;
        const int64_t gc = c0 + 2 * pair, gr0 = r0 + blk * 32;
        const bool stage_sc = tile_stages_scales(p, r0, c0);
        uint8_t *const satom = stage_sc ? st.atoms + buf * 512 : nullptr;
        if (ok && gc < C && gr0 < R) {
            const TIn *tile = reinterpret_cast<const TIn *>(tiles + buf * TILE_BYTES);
            // x[j] = (column gc, column gc + 1) at row gr0 + j, as packed f32x2
            uint64_t x[32];
            uint32_t words[32];
#pragma unroll
            for (int j = 0; j < 32; ++j) {
                const int off = (blk * 32 + j) * COL_TILE_C + 2 * pair;
                if (BF16_IN) {
                    uint32_t w = *reinterpret_cast<const uint32_t *>(tile + off);
                    words[j] = w;
                    if (HAD && DEFM && default_mask_negates(j)) w ^= 0x80008000u;
                    x[j] = f2_pack(__uint_as_float(w << 16), __uint_as_float(w & 0xffff0000u));
                } else {
                    x[j] = *reinterpret_cast<const uint64_t *>(tile + off);
                    if (HAD && DEFM && default_mask_negates(j)) x[j] ^= 0x8000000080000000ull;
                }
            }
            if (BF16_IN && !HAD) encode_col_pair<FMT, SR, false, true>(p, x, gc, gr0, bf16_pair_max<32>(words), satom);
            else encode_col_pair<FMT, SR, HAD, false, DEFM>(p, x, gc, gr0, 0u, satom);
        }
        // everyone is done with `buf` (and has written its scale bytes) before
        // it is refilled; with TMA staging a wait that gave up (in any thread)
        // ends the CTA's loop
        if (TMA) {
            if (!__syncthreads_and(ok)) {
                if (threadIdx.x == 0) drain_staged(st.bars, buf, use, tn < n_tiles);
                break;
            }
        } else {
            __syncthreads();
        }
        if (stage_sc) write_scale_atom(p, satom, r0, c0, warp, lane);
    }
    if (!TMA) cp_async_wait_all();
}

// ---------------------------------------------------------------------------
// Dual cast: one read of the input, codes along both axes.
// ---------------------------------------------------------------------------
// The forward GEMM contracts an activation over its columns (blocks along
// rows) and the weight-gradient GEMM over its rows (blocks down columns,
// transposed output); section 3 of the MX summary notes that the two
// quantizations of one tensor differ, so both are needed.  This kernel stages
// each 128 x 128 tile once (swizzled, see tile_chunk) and writes both: every
// thread encodes one column pair of one 32-row block (as cast_cols) and two
// 32-element row blocks (as cast_rows, RNE or SR with its own seed).  The
// result equals mx_quantize along rows plus mx_quantize along columns.
// TMA: the tile is staged by tensor copies of `tmap` in boxes 128 bytes wide
// (64 bf16 or 32 fp32 columns) with the copy engine's 128-byte swizzle: box h
// of the tile occupies 16 KiB at h * 16 KiB, tile row r at r * 128 bytes, and
// its 16-byte chunk c at position c XOR (r % 8).  The column reads (a warp
// reads one 128-byte box row) and the row reads (eight lanes read the same
// chunk of eight consecutive rows) then touch distinct banks.  Without TMA,
// cp.async copies with the tile_chunk swizzle.
template <int FMT, bool BF16_IN, bool HAD, bool DEFM, bool TMA>
__global__ void __launch_bounds__(COL_THREADS, 2) cast_dual_kernel(CastParams pr, CastParams pc, int sr_rows,
                                                                   int sr_cols,
                                                                   const __grid_constant__ CUtensorMap tmap) {
    using TIn = typename std::conditional<BF16_IN, uint16_t, float>::type;
    constexpr int TILE_BYTES = COL_TILE_R * COL_TILE_C * sizeof(TIn);
    constexpr int ROW_BYTES = COL_TILE_C * sizeof(TIn);
    constexpr int CPB = 32 * sizeof(TIn) / 16;              // 16-byte chunks per 32-element row block
    constexpr int BOX_C = 128 / sizeof(TIn);                // columns per 128-byte box (TMA)
    constexpr int BOXES = COL_TILE_C / BOX_C;
    constexpr int BOX_BYTES = COL_TILE_R * 128;
    extern __shared__ __align__(16) uint8_t col_smem[];
    const StagedTiles<1024> st(col_smem, TILE_BYTES);
    uint8_t *const tiles = TMA ? st.tiles : col_smem;

    const int64_t R = pc.rows, C = pc.cols;
    const int64_t tiles_r = (R + COL_TILE_R - 1) / COL_TILE_R;
    const int64_t tiles_c = (C + COL_TILE_C - 1) / COL_TILE_C;
    const int64_t n_tiles = tiles_r * tiles_c;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int blk = warp & 3;                       // column part: 32-row block inside the tile
    const int pair = (warp >> 2) * 32 + lane;       // column part: column pair inside the tile
    // row part: 32-column block rb of tile rows rrow and rrow + 64 (with TMA,
    // eight consecutive lanes take the same block of eight consecutive rows)
    const int rb = TMA ? (lane >> 3) : (threadIdx.x & 3);
    const int rrow = TMA ? (warp * 8 + (lane & 7)) : (threadIdx.x >> 2);

    // the column pair's byte offset inside even and odd tile rows (cp.async
    // layout), or inside tile row blk * 32 before the row's swizzle (TMA)
    const int cbyte = 2 * pair * static_cast<int>(sizeof(TIn));
    const int col_off[2] = {tile_chunk<BF16_IN, true>(0, cbyte >> 4) * 16 + (cbyte & 15),
                            tile_chunk<BF16_IN, true>(1, cbyte >> 4) * 16 + (cbyte & 15)};
    const int col_box = (cbyte >> 7) * BOX_BYTES + blk * 32 * 128 + (cbyte & 127);

    auto issue = [&](int64_t tile, int b) {     // thread 0, TMA staging
        stage_expect(st.bars + 8 * b, TILE_BYTES);
        const int x0 = static_cast<int>((tile % tiles_c) * COL_TILE_C), y0 = static_cast<int>((tile / tiles_c) * COL_TILE_R);
#pragma unroll
        for (int h = 0; h < BOXES; ++h)
            tma_tile_load(st.base + b * TILE_BYTES + h * BOX_BYTES, &tmap, x0 + h * BOX_C, y0, st.bars + 8 * b);
    };
    if (TMA) {
        if (threadIdx.x == 0) {
            stage_bar_init(st.bars);
            stage_bar_init(st.bars + 8);
            asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        }
        __syncthreads();
    }

    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    asm volatile("griddepcontrol.wait;" ::: "memory");     // inputs of the previous kernel are visible
    int64_t t = blockIdx.x;
    if (TMA) {
        if (t < n_tiles && threadIdx.x == 0 && !(pc.skip_first && blockIdx.x == 0)) issue(t, 0);
    } else {
        if (t < n_tiles) stage_tile<BF16_IN, true>(pc, col_smem, (t / tiles_c) * COL_TILE_R, (t % tiles_c) * COL_TILE_C);
        cp_async_commit();
    }
    uint32_t use = 0;                // tiles this CTA has taken: buffer use % 2, phase (use / 2) % 2
    bool ok = true;
    for (int buf = 0; t < n_tiles; t += gridDim.x, buf ^= 1, ++use) {
        const int64_t tn = t + gridDim.x;
        if (TMA) {
            if (tn < n_tiles && threadIdx.x == 0) issue(tn, buf ^ 1);
            ok = stage_wait(st.bars + 8 * buf, (use >> 1) & 1u);
        } else {
            if (tn < n_tiles)
                stage_tile<BF16_IN, true>(pc, col_smem + (buf ^ 1) * TILE_BYTES, (tn / tiles_c) * COL_TILE_R,
                                          (tn % tiles_c) * COL_TILE_C);
            cp_async_commit();
            cp_async_wait_prev();        // this tile's copies (the older group) have landed
            __syncthreads();
        }

        const uint8_t *tile = tiles + buf * TILE_BYTES;
        const int64_t r0 = (t / tiles_c) * COL_TILE_R, c0 = (t % tiles_c) * COL_TILE_C;
        const bool stage_sc = tile_stages_scales(pc, r0, c0);
        uint8_t *const satom = stage_sc ? st.atoms + buf * 512 : nullptr;
        // ---- column blocks ----
        const int64_t gc = c0 + 2 * pair, gr0 = r0 + blk * 32;
        if (ok && gc < C && gr0 < R) {
            uint64_t x[32];
            uint32_t words[32];
#pragma unroll
            for (int j = 0; j < 32; ++j) {
                // TMA: row blk * 32 + j, whose chunks are permuted by j % 8
                const uint8_t *src = TMA ? tile + ((col_box ^ ((j & 7) << 4)) + j * 128)
                                         : tile + (blk * 32 + j) * ROW_BYTES + col_off[j & 1];
                if (BF16_IN) {
                    uint32_t w = *reinterpret_cast<const uint32_t *>(src);
                    words[j] = w;
                    if (HAD && DEFM && default_mask_negates(j)) w ^= 0x80008000u;
                    x[j] = f2_pack(__uint_as_float(w << 16), __uint_as_float(w & 0xffff0000u));
                } else {
                    x[j] = *reinterpret_cast<const uint64_t *>(src);
                    if (HAD && DEFM && default_mask_negates(j)) x[j] ^= 0x8000000080000000ull;
                }
            }
            if (BF16_IN && !HAD) {
                const uint32_t m16 = bf16_pair_max<32>(words);
                if (sr_cols) encode_col_pair<FMT, true, false, true>(pc, x, gc, gr0, m16, satom);
                else encode_col_pair<FMT, false, false, true>(pc, x, gc, gr0, m16, satom);
            } else {
                if (sr_cols) encode_col_pair<FMT, true, HAD, false, DEFM>(pc, x, gc, gr0, 0u, satom);
                else encode_col_pair<FMT, false, HAD, false, DEFM>(pc, x, gc, gr0, 0u, satom);
            }
        }
        // ---- row blocks ----
#pragma unroll 1
        for (int h = 0; h < 2; ++h) {
            const int rr = rrow + 64 * h;
            const int64_t row = r0 + rr, kb = (c0 >> 5) + rb;
            if (!ok || row >= R || 32 * kb >= C) continue;
            uint32_t b[32];
            uint32_t words[16];
#pragma unroll
            for (int i = 0; i < CPB; ++i) {
                // chunk q of the row: box q / 8, chunk q % 8 permuted by rr % 8 (TMA)
                const int q = rb * CPB + i;
                const int off = TMA ? (q >> 3) * BOX_BYTES + rr * 128 + (((q & 7) ^ (rr & 7)) << 4)
                                    : rr * ROW_BYTES + tile_chunk<BF16_IN, true>(rr, q) * 16;
                const uint4 w = *reinterpret_cast<const uint4 *>(tile + off);
                if (BF16_IN) {
                    const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
                    for (int k = 0; k < 4; ++k) {
                        words[4 * i + k] = ws[k];
                        b[8 * i + 2 * k] = ws[k] << 16;
                        b[8 * i + 2 * k + 1] = ws[k] & 0xffff0000u;
                    }
                } else {
                    b[4 * i] = w.x; b[4 * i + 1] = w.y; b[4 * i + 2] = w.z; b[4 * i + 3] = w.w;
                }
            }
            if (BF16_IN) {
                const uint32_t amax = bf16_max_bits(bf16_pair_max<16>(words));
                if (sr_rows) encode_row_block<FMT, true, false>(pr, row, kb, b, amax);
                else encode_row_block<FMT, false, false>(pr, row, kb, b, amax);
            } else {
                if (sr_rows) encode_row_block<FMT, true, false>(pr, row, kb, b);
                else encode_row_block<FMT, false, false>(pr, row, kb, b);
            }
        }
        // everyone is done with `buf` (and has written its scale bytes) before
        // it is refilled; with TMA staging a wait that gave up (in any thread)
        // ends the CTA's loop
        if (TMA) {
            if (!__syncthreads_and(ok)) {
                if (threadIdx.x == 0) drain_staged(st.bars, buf, use, tn < n_tiles);
                break;
            }
        } else {
            __syncthreads();
        }
        if (stage_sc) write_scale_atom(pc, satom, r0, c0, warp, lane);
    }
    if (!TMA) cp_async_wait_all();
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
    uint64_t codes_cap, scales_cap;   // buffer sizes in bytes (checked by the debug build)
};

template <int FMT, bool BF16_OUT>
__global__ void __launch_bounds__(256) dequant_kernel(DequantParams p) {
    constexpr int BITS = Fmt<FMT>::bits;
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    asm volatile("griddepcontrol.wait;" ::: "memory");     // inputs of the previous kernel are visible

    const int64_t octs_per_row = p.inner >> 3;
    const int64_t n = p.outer * octs_per_row;
    for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n;
         i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
        const int64_t o = i / octs_per_row, oc = i - o * octs_per_row;
        const int64_t kb = oc >> 2;
        const int64_t so = p.mma_scales == SL_MMA_X4 ? static_cast<int64_t>(x4_scale_offset32(
                               static_cast<uint32_t>(o), static_cast<uint32_t>(kb), static_cast<uint32_t>(p.k_groups)))
                           : p.mma_scales == SL_MMA ? mma_scale_offset(o, kb, p.k_groups) : o * p.k_blocks + kb;
        if (!in_bounds(static_cast<uint64_t>(so), 1, p.scales_cap) ||
            !in_bounds(static_cast<uint64_t>(o * (p.inner * BITS / 8) + oc * BITS), BITS, p.codes_cap))
            continue;                                   // (debug build) outside a buffer: skipped
        const uint32_t s = p.scales[so];
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

// Blocks of `Kernel` that fit on one SM at once (queried once per kernel;
// the cache is per template instance, i.e. per kernel): grid-stride kernels
// are launched with exactly the resident number of blocks.
template <auto Kernel>
static int resident_blocks_per_sm(int threads, int smem) {
    static int cached = 0;
    if (cached == 0) {
        int n = 0;
        if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, Kernel, threads, smem) != cudaSuccess || n < 1) n = 1;
        cached = n;
    }
    return cached;
}

// Launch allowed to overlap the previous kernel in the stream (programmatic
// dependent launch); the kernel waits for that kernel's results itself.
template <auto Kernel, typename... Args>
static cudaError_t launch_overlapped(int grid, int block, int smem, cudaStream_t st, Args... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(block);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, Kernel, args...);
}

// Testing hooks (include/mx_debug.h), per host thread.
thread_local bool t_force_cpasync = false;
thread_local bool t_skip_first = false;
thread_local uint64_t t_codes_cap_cut = 0;

// Tensor map of a cast's input for TMA staging: the rows x cols tensor in
// boxes of 128 rows x 128 columns, unswizzled (column cast), or x 128 bytes
// with the 128-byte swizzle (dual cast).  False when the input cannot be
// staged that way (base address or row pitch not a multiple of 16 bytes, a
// coordinate beyond int32, an encoding the driver refuses): the kernels then
// stage with cp.async.
static bool make_input_map(CUtensorMap *map, const CastParams &p, bool bf16, bool swizzled) {
    if (t_force_cpasync) return false;
    const int64_t esz = bf16 ? 2 : 4;
    if ((reinterpret_cast<uintptr_t>(p.x) & 15u) != 0 || ((p.ldx * esz) & 15) != 0) return false;
    if (p.rows > INT32_MAX - COL_TILE_R || p.cols > INT32_MAX - COL_TILE_C) return false;
    return mxg::encode_2d(map, bf16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT32, p.x,
                          static_cast<uint64_t>(p.cols), static_cast<uint64_t>(p.rows),
                          static_cast<uint64_t>(p.ldx * esz), swizzled ? static_cast<uint32_t>(128 / esz) : COL_TILE_C,
                          COL_TILE_R, swizzled ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_NONE);
}

// Dynamic shared memory of the column and dual casts: two tile buffers, their
// two staging barriers, and slack to align the buffers for TMA.
static int staged_smem_bytes(int in_bytes, int align) {
    return 2 * COL_TILE_R * COL_TILE_C * in_bytes + 16 + 2 * 512 + align;
}

// Column cast: two tile buffers of dynamic shared memory, a resident grid.
template <auto Kernel>
static cudaError_t launch_cols(int in_bytes, const CastParams &p, int64_t tiles, int sms, cudaStream_t st,
                               const CUtensorMap &map) {
    const int smem = staged_smem_bytes(in_bytes, 128);
    static std::atomic<uint64_t> configured{0};    // per kernel, one bit per device
    if (cudaError_t e = ensure_smem_limit(Kernel, smem, configured); e != cudaSuccess) return e;
    return launch_overlapped<Kernel>(grid_for(tiles, 1, sms * resident_blocks_per_sm<Kernel>(COL_THREADS, smem)),
                                     COL_THREADS, smem, st, p, map);
}

// The TMA-staged instance when `map` is set, else the cp.async one.
template <int FMT, bool SR, bool BF, bool HAD, bool DEFM>
static cudaError_t launch_cols_staged(const CastParams &p, int64_t tiles, int sms, cudaStream_t st,
                                      const CUtensorMap *map) {
    if (map) return launch_cols<cast_cols_kernel<FMT, SR, BF, HAD, DEFM, true>>(BF ? 2 : 4, p, tiles, sms, st, *map);
    return launch_cols<cast_cols_kernel<FMT, SR, BF, HAD, DEFM, false>>(BF ? 2 : 4, p, tiles, sms, st, CUtensorMap{});
}

template <int FMT, bool SR>
static cudaError_t launch_cast_fmt(const CastParams &p, int xdt, int block_axis, bool had, int sms,
                                   cudaStream_t st) {
    const bool bf = xdt == MX_BF16;
    if (block_axis == 1) {
        const int64_t chunks = p.rows * (((p.cols >> 5) + 31) >> 5);    // 32-block chunks, one per warp
        // 32-byte accesses need 32-byte aligned input rows and code rows (a code
        // row is cols * bits / 8 bytes, a multiple of 32 for 8-bit formats)
        const bool v32 = (reinterpret_cast<uintptr_t>(p.x) & 31u) == 0 && ((p.ldx * (bf ? 2 : 4)) & 31) == 0 &&
                         (reinterpret_cast<uintptr_t>(p.codes) & 31u) == 0;
        if (bf) {
            if (v32) {
                constexpr auto k = cast_rows_kernel<FMT, SR, true, true>;
                return launch_overlapped<k>(grid_for(chunks, 8, sms * resident_blocks_per_sm<k>(256, 0)), 256, 0, st, p);
            } else {
                constexpr auto k = cast_rows_kernel<FMT, SR, true, false>;
                return launch_overlapped<k>(grid_for(chunks, 8, sms * resident_blocks_per_sm<k>(256, 0)), 256, 0, st, p);
            }
        } else {
            if (v32) {
                constexpr auto k = cast_rows_kernel<FMT, SR, false, true>;
                return launch_overlapped<k>(grid_for(chunks, 8, sms * resident_blocks_per_sm<k>(256, 0)), 256, 0, st, p);
            } else {
                constexpr auto k = cast_rows_kernel<FMT, SR, false, false>;
                return launch_overlapped<k>(grid_for(chunks, 8, sms * resident_blocks_per_sm<k>(256, 0)), 256, 0, st, p);
            }
        }
    } else {
        const int64_t tiles = ((p.rows + COL_TILE_R - 1) / COL_TILE_R) * ((p.cols + COL_TILE_C - 1) / COL_TILE_C);
        CUtensorMap m;
        const CUtensorMap *map = make_input_map(&m, p, bf, false) ? &m : nullptr;
        if (had && p.sign_mask == MX_DEFAULT_SIGN_MASK) {
            if (bf) return launch_cols_staged<FMT, SR, true, true, true>(p, tiles, sms, st, map);
            return launch_cols_staged<FMT, SR, false, true, true>(p, tiles, sms, st, map);
        }
        if (had) {
            if (bf) return launch_cols_staged<FMT, SR, true, true, false>(p, tiles, sms, st, map);
            return launch_cols_staged<FMT, SR, false, true, false>(p, tiles, sms, st, map);
        }
        if (bf) return launch_cols_staged<FMT, SR, true, false, false>(p, tiles, sms, st, map);
        return launch_cols_staged<FMT, SR, false, false, false>(p, tiles, sms, st, map);
    }
    return cudaGetLastError();
}

template <int FMT>
static cudaError_t launch_cast_rnd(const CastParams &p, int xdt, int block_axis, bool sr, bool had, int sms,
                                   cudaStream_t st) {
    return sr ? launch_cast_fmt<FMT, true>(p, xdt, block_axis, had, sms, st)
              : launch_cast_fmt<FMT, false>(p, xdt, block_axis, had, sms, st);
}

// Dual cast: the column cast's tile buffers and resident grid.
template <auto Kernel>
static cudaError_t launch_dual(int in_bytes, const CastParams &pr, const CastParams &pc, int sr_rows, int sr_cols,
                               int64_t tiles, int sms, cudaStream_t st, const CUtensorMap &map) {
    const int smem = staged_smem_bytes(in_bytes, 1024);
    static std::atomic<uint64_t> configured{0};    // per kernel, one bit per device
    if (cudaError_t e = ensure_smem_limit(Kernel, smem, configured); e != cudaSuccess) return e;
    return launch_overlapped<Kernel>(grid_for(tiles, 1, sms * resident_blocks_per_sm<Kernel>(COL_THREADS, smem)),
                                     COL_THREADS, smem, st, pr, pc, sr_rows, sr_cols, map);
}

template <int FMT, bool BF, bool HAD, bool DEFM>
static cudaError_t launch_dual_staged(const CastParams &pr, const CastParams &pc, int sr_rows, int sr_cols,
                                      int64_t tiles, int sms, cudaStream_t st, const CUtensorMap *map) {
    if (map)
        return launch_dual<cast_dual_kernel<FMT, BF, HAD, DEFM, true>>(BF ? 2 : 4, pr, pc, sr_rows, sr_cols, tiles,
                                                                       sms, st, *map);
    return launch_dual<cast_dual_kernel<FMT, BF, HAD, DEFM, false>>(BF ? 2 : 4, pr, pc, sr_rows, sr_cols, tiles, sms,
                                                                    st, CUtensorMap{});
}

template <int FMT>
static cudaError_t launch_dual_fmt(const CastParams &pr, const CastParams &pc, int xdt, bool had, int sr_rows,
                                   int sr_cols, int sms, cudaStream_t st) {
    const int64_t tiles = ((pc.rows + COL_TILE_R - 1) / COL_TILE_R) * ((pc.cols + COL_TILE_C - 1) / COL_TILE_C);
    const bool bf = xdt == MX_BF16;
    CUtensorMap m;
    const CUtensorMap *map = make_input_map(&m, pc, bf, true) ? &m : nullptr;
    if (had && pc.sign_mask == MX_DEFAULT_SIGN_MASK) {
        if (bf) return launch_dual_staged<FMT, true, true, true>(pr, pc, sr_rows, sr_cols, tiles, sms, st, map);
        return launch_dual_staged<FMT, false, true, true>(pr, pc, sr_rows, sr_cols, tiles, sms, st, map);
    }
    if (had) {
        if (bf) return launch_dual_staged<FMT, true, true, false>(pr, pc, sr_rows, sr_cols, tiles, sms, st, map);
        return launch_dual_staged<FMT, false, true, false>(pr, pc, sr_rows, sr_cols, tiles, sms, st, map);
    }
    if (bf) return launch_dual_staged<FMT, true, false, false>(pr, pc, sr_rows, sr_cols, tiles, sms, st, map);
    return launch_dual_staged<FMT, false, false, false>(pr, pc, sr_rows, sr_cols, tiles, sms, st, map);
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
    p.mma_scales = a.sl;
    const int64_t inner = a.block_axis == 1 ? a.cols : a.rows;
    p.k_blocks = inner / 32;
    p.k_groups = (p.k_blocks + 3) / 4;
    p.key = fmix32_host(static_cast<uint32_t>(a.seed)) ^ static_cast<uint32_t>(a.seed >> 32);
    p.sign_mask = a.sign_mask;
    p.sr_base = a.sr_base;
    p.sr_stride = a.sr_stride;
    p.skip_first = 0;
    p.stage_scales = (a.sl == SL_MMA || a.sl == SL_MMA_X4) && (reinterpret_cast<uintptr_t>(a.scales) & 15u) == 0;
    p.codes_cap = mx_codes_bytes(static_cast<mx_fmt>(a.fmt), a.block_axis == 1 ? a.rows : a.cols, inner);
    p.scales_cap = mx_scales_bytes(static_cast<mx_scale_layout>(a.sl), a.block_axis == 1 ? a.rows : a.cols, inner);
    p.codes_cap -= t_codes_cap_cut < p.codes_cap ? t_codes_cap_cut : p.codes_cap;   // testing hook, one shot
    t_codes_cap_cut = 0;
    if (a.block_axis == 0) {         // the one-shot hook applies to staged (column) casts
        p.skip_first = t_skip_first ? 1 : 0;
        t_skip_first = false;
    }
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
    p.mma_scales = a.sl;
    p.outer = a.outer;
    p.inner = a.inner;
    p.k_blocks = a.inner / 32;
    p.k_groups = (p.k_blocks + 3) / 4;
    p.y = a.y;
    p.ldy = a.ldy;
    p.codes_cap = mx_codes_bytes(static_cast<mx_fmt>(a.fmt), a.outer, a.inner);
    p.scales_cap = mx_scales_bytes(static_cast<mx_scale_layout>(a.sl), a.outer, a.inner);
    const int grid = grid_for(a.outer * (a.inner / 8), 256, a.num_sms * 8);
    const bool bf = a.ydt == MX_BF16;
#define MX_DQ(F)                                                                                      \
    case F:                                                                                           \
        return bf ? launch_overlapped<dequant_kernel<F, true>>(grid, 256, 0, st, p)                   \
                  : launch_overlapped<dequant_kernel<F, false>>(grid, 256, 0, st, p);
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
}

cudaError_t mx_launch_quantize_dual(const MxQuantizeDualArgs &a, cudaStream_t st) {
    using namespace mxk;
    auto key = [](uint64_t seed) {
        return fmix32_host(static_cast<uint32_t>(seed)) ^ static_cast<uint32_t>(seed >> 32);
    };
    CastParams pr, pc;
    pr.x = pc.x = a.x;
    pr.rows = pc.rows = a.rows;
    pr.cols = pc.cols = a.cols;
    pr.ldx = pc.ldx = a.ldx;
    pr.mma_scales = pc.mma_scales = a.sl;
    pr.codes = static_cast<uint8_t *>(a.codes_rows);
    pr.scales = static_cast<uint8_t *>(a.scales_rows);
    pr.k_blocks = a.cols / 32;
    pr.k_groups = (pr.k_blocks + 3) / 4;
    pr.key = key(a.seed_rows);
    pr.sign_mask = 0;
    pr.sr_base = a.sr_base_rows;
    pr.sr_stride = a.sr_stride_rows;
    pc.codes = static_cast<uint8_t *>(a.codes_cols);
    pc.scales = static_cast<uint8_t *>(a.scales_cols);
    pc.k_blocks = a.rows / 32;
    pc.k_groups = (pc.k_blocks + 3) / 4;
    pc.key = key(a.seed_cols);
    pc.sign_mask = a.sign_mask;
    pc.sr_base = a.sr_base_cols;
    pc.sr_stride = a.sr_stride_cols;
    pr.skip_first = 0;
    pc.skip_first = t_skip_first ? 1 : 0;
    pr.stage_scales = 0;
    pc.stage_scales = (a.sl == SL_MMA || a.sl == SL_MMA_X4) && (reinterpret_cast<uintptr_t>(a.scales_cols) & 15u) == 0;
    pr.codes_cap = mx_codes_bytes(static_cast<mx_fmt>(a.fmt), a.rows, a.cols);
    pr.scales_cap = mx_scales_bytes(static_cast<mx_scale_layout>(a.sl), a.rows, a.cols);
    pc.codes_cap = mx_codes_bytes(static_cast<mx_fmt>(a.fmt), a.cols, a.rows);
    pc.scales_cap = mx_scales_bytes(static_cast<mx_scale_layout>(a.sl), a.cols, a.rows);
    t_skip_first = false;
    const int sr_r = a.rnd_rows == MX_SR, sr_c = a.rnd_cols == MX_SR;
    switch (a.fmt) {
        case MX_E4M3: return launch_dual_fmt<MX_E4M3>(pr, pc, a.xdt, a.hadamard, sr_r, sr_c, a.num_sms, st);
        case MX_E5M2: return launch_dual_fmt<MX_E5M2>(pr, pc, a.xdt, a.hadamard, sr_r, sr_c, a.num_sms, st);
        case MX_E2M3: return launch_dual_fmt<MX_E2M3>(pr, pc, a.xdt, a.hadamard, sr_r, sr_c, a.num_sms, st);
        case MX_E3M2: return launch_dual_fmt<MX_E3M2>(pr, pc, a.xdt, a.hadamard, sr_r, sr_c, a.num_sms, st);
        case MX_E2M1: return launch_dual_fmt<MX_E2M1>(pr, pc, a.xdt, a.hadamard, sr_r, sr_c, a.num_sms, st);
        case MX_INT8: return launch_dual_fmt<MX_INT8>(pr, pc, a.xdt, a.hadamard, sr_r, sr_c, a.num_sms, st);
    }
    return cudaErrorInvalidValue;
}

// Reads and clears the casts' status word and, in this unit, the debug
// build's bounds word (after the caller synchronised); a timeout comes first.
int mx_read_cast_status() {
    int v = 0, b = 0;
    if (cudaMemcpyFromSymbol(&v, mxk::g_cast_status, sizeof(int)) != cudaSuccess) return MX_ERR_CUDA;
    if (cudaMemcpyFromSymbol(&b, mxk::g_bounds_status, sizeof(int)) != cudaSuccess) return MX_ERR_CUDA;
    const int zero = 0;
    if (cudaMemcpyToSymbol(mxk::g_cast_status, &zero, sizeof(int)) != cudaSuccess) return MX_ERR_CUDA;
    if (cudaMemcpyToSymbol(mxk::g_bounds_status, &zero, sizeof(int)) != cudaSuccess) return MX_ERR_CUDA;
    return v != MX_OK ? v : b;
}

extern "C" int mx_debug_cast_force_cpasync(int on) {
    mxk::t_force_cpasync = on != 0;
    return MX_OK;
}

extern "C" int mx_debug_cast_skip_tile(int on) {
    mxk::t_skip_first = on != 0;
    return MX_OK;
}

extern "C" int mx_debug_cast_cut_codes_cap(int64_t bytes) {
    if (bytes < 0) return MX_ERR_ARG;
    mxk::t_codes_cap_cut = static_cast<uint64_t>(bytes);
    return MX_OK;
}
