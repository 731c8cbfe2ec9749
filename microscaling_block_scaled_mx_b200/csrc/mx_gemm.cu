// mx_gemm.cu -- block-scaled GEMM C = alpha * A * B^T on the sm_100a tensor
// cores: the quantized dot products of the compute flow in "Microscaling Data
// Formats for Deep Learning" (summary page, section 4), which take MX inputs
// and return scalar floats.
//
// Design (one persistent CTA per SM, 320 threads, warp-specialized):
//   warp 0      TMA producer: 128 x 128-byte A tile and 192 x 128-byte B tile
//               per stage (128-byte swizzle), plus the 512-byte E8M0 scale
//               atoms of both operands (bulk copies; the MMA layout written by
//               mx_quantize is already the tensor-core layout).
//   warp 1      TMEM owner and MMA issuer (one thread): tcgen05.cp moves each
//               scale atom smem -> TMEM (32x128b, replicated to the four lane
//               quarters), then four tcgen05.mma.block_scale per stage
//               (kind::mxf8f6f4 K=32 for MXFP8, kind::mxf4 K=64 for MXFP4)
//               accumulate into one of two 128 x 192 fp32 TMEM accumulators,
//               so the epilogue of a tile overlaps the mainloop of the next.
//   warps 2-9   epilogue: two warps per TMEM lane quarter, 96 columns each,
//               three tcgen05.ld of 32 columns per wait, times alpha, rounded
//               to fp32 / bf16, written to a per-warp shared-memory piece of
//               32 rows x 64 bytes and stored to C by one TMA store per piece
//               (the copy engine clips the ragged edges of C).
// The scale copies are the largest cost after the MMAs: with the replicating
// 32x128b.warpx4 form (one per 512-byte atom) they take a fifth to a third of
// the MXFP4 pair kernel's time.  With operand scales in the x4 layout (each
// atom stored four times, written so by the cast) the pair kernel uses the
// 128-lane 128x256b / 128x128b forms instead, two atoms per copy: half the
// copy instructions and 9-11 % less time on MXFP4.  Building those replicas
// inside the SM (an expander warp, or the epilogue warps writing the scale
// factors with tcgen05.st) measured slower: both need a per-stage cross-CTA
// handshake that costs more than the copies.
// A 192-column tile starts 64 rows into a 128-row scale atom on odd tiles;
// the B scale-factor TMEM address then starts two columns later.
// Every mbarrier wait is bounded; on expiry the kernel records MX_ERR_TIMEOUT
// in the device status word, drains what it issued (bounded again), frees
// its TMEM and returns.
#include <cstdint>
#include <cstring>
#include <atomic>
#include <mutex>

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include "mx.h"
#include "mx_debug.h"
#include "mx_encode.cuh"
#include "mx_internal.h"

// Device status word: kernels that give up a bounded wait record MX_ERR_TIMEOUT here.
__device__ int g_mx_status;

namespace mxg {

constexpr int BM = 128;            // tile rows (A rows, TMEM lanes)
constexpr int BN = 192;            // tile columns (B rows, accumulator columns)
constexpr int BK_BYTES = 128;      // K bytes per stage: 128 fp8 or 256 fp4 elements
constexpr int STAGES = 4;
constexpr int EPI_WARPS = 8;
constexpr int NUM_THREADS = 64 + 32 * EPI_WARPS;
constexpr int A_STAGE_BYTES = BM * BK_BYTES;   // 16 KiB
constexpr int B_STAGE_BYTES = BN * BK_BYTES;   // 24 KiB
constexpr int ATOM = 512;                      // scale atom: 128 rows x 4 k-blocks
constexpr uint32_t TMEM_COLS = 512;
constexpr uint32_t ACC_COLS = BN;              // accumulator b at columns [b * 192, (b + 1) * 192)
constexpr uint32_t SF_COL = 2 * ACC_COLS;      // scale-factor columns from 384
constexpr int EPI_PIECE = 2048;                // one staged piece of C: 32 rows x 64 bytes
constexpr int EPI_WARP_BYTES = 2 * EPI_PIECE;  // two pieces per epilogue warp (double buffer)
constexpr unsigned long long WAIT_LIMIT_NS = 2000000000ull;   // 2 s per wait
constexpr unsigned long long DRAIN_LIMIT_NS = 200000000ull;   // 0.2 s when draining
constexpr unsigned long long DRAIN_SETTLE_NS = 1000000ull;    // 1 ms for loads in flight after an abort

template <bool FP4> struct Cfg {
    static constexpr int G = FP4 ? 2 : 1;             // scale atoms along K per stage
    static constexpr int SFA_BYTES = ATOM * G;        // per stage
    static constexpr int SFB_BYTES = 2 * ATOM * G;    // the two 128-row scale blocks a tile touches
    static constexpr int SFA_COLS = 4 * G;            // TMEM columns per stage
    static constexpr int SFB_COLS = 8 * G;
    static constexpr int SF_STAGE_COLS = SFA_COLS + SFB_COLS;
};

struct Smem {
    // offsets inside the 1024-aligned dynamic shared buffer
    static constexpr int A = 0;
    static constexpr int B = A + STAGES * A_STAGE_BYTES;
    static constexpr int SFA = B + STAGES * B_STAGE_BYTES;
    static constexpr int SFB = SFA + STAGES * 2 * ATOM;       // sized for the FP4 case
    static constexpr int EPI = (SFB + STAGES * 4 * ATOM + 1023) / 1024 * 1024;
    static constexpr int BAR = EPI + EPI_WARPS * EPI_WARP_BYTES;
    // full[STAGES], empty[STAGES], acc_full[2], acc_empty[2], drain
    static constexpr int NUM_BARS = 2 * STAGES + 5;
    static constexpr int TMEM_SLOT = BAR + NUM_BARS * 8;
    static constexpr int ABORT = TMEM_SLOT + 4;
    static constexpr int TOTAL = ABORT + 4;
};
constexpr int SMEM_BYTES = Smem::TOTAL + 1024;   // slack for 1024-byte alignment
static_assert(SMEM_BYTES <= 232448, "shared memory per block");

// Output of the epilogue: C in fp32 or bf16, or C quantized along its rows
// (blocks of 32 consecutive columns) to MX codes and E8M0 scales.
constexpr int OUT_F32 = 0, OUT_BF16 = 1, OUT_MX = 2;

struct MxOut {
    uint8_t *codes;      // M x (N * bits / 8) bytes
    uint8_t *scales;     // plain or MMA layout for (M, N)
    int fmt;             // element format
    int sr;              // stochastic rounding (else RNE)
    int mma;             // scale layout: 0 plain, 1 MMA, 2 MMA x4
    uint32_t key;        // stochastic-rounding seed key
};

struct Params {
    const uint8_t *a_scales;
    const uint8_t *b_scales;
    void *c;
    int64_t ldc;
    int M, N, K;
    int k_tiles;     // K bytes / BK_BYTES
    int k_groups;    // scale atoms along K per 128-row block (K / 128 elements)
    int tiles_m, tiles_n;
    float alpha;
    uint32_t idesc;  // instruction descriptor without the scale-factor ids
    uint32_t ab_tx;  // bytes the A and B loads of one stage deliver (packed size in global)
    uint32_t a_tx;   // the A load's share of ab_tx
    int skip_k_tile; // testing hook: CTA 0 withholds this k-tile of its first tile (-1: off)
    int raster_group, raster_n_major;   // tile order (tile_coords)
    MxOut q;         // OUT_MX only
};

// Tile order.  Tiles are taken in bands of `group` tiles along the major
// axis (M, or N when n_major), the band's tiles along the minor axis one after
// the other.  The host picks the order per shape (see raster_for): with the
// band as wide as the whole axis, the CTAs in flight share the operand whose
// panels all stay in L2 while the other operand streams through once; narrow
// bands bound the working set when neither operand fits.
__device__ __forceinline__ void tile_coords(int tile, int tiles_m, int tiles_n, int group, int n_major, int &tm,
                                            int &tn) {
    const int major = n_major ? tiles_n : tiles_m, minor_tiles = n_major ? tiles_m : tiles_n;
    const int per_band = group * minor_tiles;
    const int band = tile / per_band, r = tile - band * per_band;
    const int j0 = band * group;
    const int width = major - j0 < group ? major - j0 : group;
    const int j = j0 + r % width, i = r / width;
    tm = n_major ? i : j;
    tn = n_major ? j : i;
}

// ------------------------------------------------------------------------
// PTX wrappers
// ------------------------------------------------------------------------
__device__ __forceinline__ uint32_t smem_u32(const void *p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count));
}
__device__ __forceinline__ void mbar_expect_tx(uint32_t bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes) : "memory");
}
__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok) : "r"(bar), "r"(parity) : "memory");
    return ok != 0;
}
__device__ __forceinline__ unsigned long long globaltimer() {
    unsigned long long t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

// Bounded wait.  Returns false (and flags the CTA and the device) when the
// phase does not complete within `limit` ns or another role already aborted.
__device__ __forceinline__ bool wait_bounded(uint32_t bar, uint32_t parity, volatile int *abort_flag,
                                             unsigned long long limit = WAIT_LIMIT_NS) {
    if (mbar_try_wait(bar, parity)) return true;
    const unsigned long long t0 = globaltimer();
    for (uint32_t it = 0;; ++it) {
        if (mbar_try_wait(bar, parity)) return true;
        if ((it & 63u) == 63u) {
            if (*abort_flag) return false;
            if (globaltimer() - t0 > limit) {
                *abort_flag = 1;
                atomicExch(&g_mx_status, MX_ERR_TIMEOUT);
                return false;
            }
        }
    }
}

__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap *map, int x, int y, uint32_t bar) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];"
        ::"r"(dst), "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(bar) : "memory");
}
__device__ __forceinline__ void bulk_load(uint32_t dst, const void *src, uint32_t bytes, uint32_t bar) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
        ::"r"(dst), "l"(src), "r"(bytes), "r"(bar) : "memory");
}

// TMA store of a shared-memory box to global memory, tracked by bulk groups
__device__ __forceinline__ void tma_store_2d(const CUtensorMap *map, uint32_t src, int x, int y) {
    asm volatile("cp.async.bulk.tensor.2d.global.shared::cta.bulk_group [%0, {%1, %2}], [%3];"
                 ::"l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(src) : "memory");
}
__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
// at most N committed bulk groups may still be reading their shared-memory source
template <int N>
__device__ __forceinline__ void bulk_wait_read() { asm volatile("cp.async.bulk.wait_group.read %0;" ::"n"(N) : "memory"); }
// every committed bulk group has completed
__device__ __forceinline__ void bulk_wait_all() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }
// generic-proxy shared-memory writes become visible to the copy engine
__device__ __forceinline__ void fence_async_smem() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }
__device__ __forceinline__ void st_shared_v4(uint32_t addr, uint32_t a, uint32_t b, uint32_t c, uint32_t d) {
    asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(a), "r"(b), "r"(c), "r"(d) : "memory");
}

__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

__device__ __forceinline__ void tc_commit(uint32_t bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar) : "memory");
}

// Shared-memory matrix descriptor (tcgen05 format): start address, leading
// and stride byte offsets in 16-byte units, version 1, layout type.
__device__ __forceinline__ uint64_t smem_desc(uint32_t addr, uint32_t lbo, uint32_t sbo, uint32_t layout) {
    uint64_t d = 0;
    d |= static_cast<uint64_t>((addr >> 4) & 0x3FFFu);
    d |= static_cast<uint64_t>((lbo >> 4) & 0x3FFFu) << 16;
    d |= static_cast<uint64_t>((sbo >> 4) & 0x3FFFu) << 32;
    d |= 1ull << 46;                                   // descriptor version for sm_100
    d |= static_cast<uint64_t>(layout & 7u) << 61;
    return d;
}
constexpr uint32_t LAYOUT_SW128 = 2;
constexpr uint32_t LAYOUT_NONE = 0;

// K-major operand tile with 128-byte rows and 128-byte swizzle: 8-row groups
// 1024 bytes apart.  k_off moves along K inside the swizzled row.
__device__ __forceinline__ uint64_t operand_desc(uint32_t tile_addr, uint32_t k_off_bytes) {
    return smem_desc(tile_addr + k_off_bytes, 16, 1024, LAYOUT_SW128);
}
// One 512-byte scale atom: 32 rows of 16 bytes, no swizzle, 8-row core
// matrices 128 bytes apart.
__device__ __forceinline__ uint64_t scale_atom_desc(uint32_t addr) {
    return smem_desc(addr, 16, 128, LAYOUT_NONE);
}

__device__ __forceinline__ void tc_cp_scale_atom(uint32_t taddr, uint64_t desc) {
    asm volatile("tcgen05.cp.cta_group::1.32x128b.warpx4 [%0], %1;" ::"r"(taddr), "l"(desc) : "memory");
}

template <bool FP4>
__device__ __forceinline__ void tc_mma(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                       uint32_t sfa_tmem, uint32_t sfb_tmem, uint32_t accumulate) {
    if (FP4) {
        asm volatile(
            "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %6, 0;\n\t"
            "tcgen05.mma.cta_group::1.kind::mxf4.block_scale.scale_vec::2X [%0], %1, %2, %3, [%4], [%5], p;\n\t}"
            ::"r"(d_tmem), "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(sfa_tmem), "r"(sfb_tmem), "r"(accumulate)
            : "memory");
    } else {
        asm volatile(
            "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %6, 0;\n\t"
            "tcgen05.mma.cta_group::1.kind::mxf8f6f4.block_scale.scale_vec::1X [%0], %1, %2, %3, [%4], [%5], p;\n\t}"
            ::"r"(d_tmem), "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(sfa_tmem), "r"(sfb_tmem), "r"(accumulate)
            : "memory");
    }
}

// ------------------------------------------------------------------------
// The kernel
// ------------------------------------------------------------------------
__device__ __forceinline__ void tmem_ld_x32_nowait(uint32_t taddr, uint32_t *r) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
        "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, "
        "%16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
          "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
          "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
        : "r"(taddr));
}
__device__ __forceinline__ void tmem_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }

// alpha * (32 consecutive accumulator values of row m), quantized as one MX
// block of C's row: the block (m, n0 / 32) of mx_quantize along the rows of
// an M x N tensor holding fl32(alpha * acc).  N is a multiple of 32, so a
// chunk that starts inside C lies wholly inside it.
template <int FMT>
__device__ __forceinline__ void quantize_chunk_fmt(const mxk::BlockSink &o, int m, int kb, uint32_t (&b)[32], bool sr) {
    if (sr) mxk::encode_block32<FMT, true, false>(o, m, kb, b);
    else mxk::encode_block32<FMT, false, false>(o, m, kb, b);
}

__device__ __forceinline__ void quantize_chunk(const Params &p, int m, int n0, const uint32_t *r) {
    uint32_t b[32];
#pragma unroll
    for (int i = 0; i < 32; ++i) b[i] = __float_as_uint(__fmul_rn(__uint_as_float(r[i]), p.alpha));
    mxk::BlockSink o;
    o.codes = p.q.codes;
    o.scales = p.q.scales;
    o.inner = p.N;
    o.k_blocks = static_cast<uint32_t>(p.N) >> 5;
    o.k_groups = (o.k_blocks + 3) >> 2;
    o.mma_scales = p.q.mma;
    o.key = p.q.key;
    o.sr_base = 0;
    o.sr_stride = static_cast<uint64_t>(p.N);
    // the epilogue already keeps every block inside M x N (the output's own
    // shape): its stores are not range-checked again by the debug build
    o.codes_cap = ~0ull;
    o.scales_cap = ~0ull;
    const int kb = n0 >> 5;
    const bool sr = p.q.sr != 0;
    switch (p.q.fmt) {
        case MX_E4M3: quantize_chunk_fmt<MX_E4M3>(o, m, kb, b, sr); break;
        case MX_E5M2: quantize_chunk_fmt<MX_E5M2>(o, m, kb, b, sr); break;
        case MX_E2M3: quantize_chunk_fmt<MX_E2M3>(o, m, kb, b, sr); break;
        case MX_E3M2: quantize_chunk_fmt<MX_E3M2>(o, m, kb, b, sr); break;
        case MX_E2M1: quantize_chunk_fmt<MX_E2M1>(o, m, kb, b, sr); break;
        default: quantize_chunk_fmt<MX_INT8>(o, m, kb, b, sr); break;
    }
}

// Epilogue through shared memory: an epilogue warp owns 32 rows of C; a piece
// is those 32 rows x 64 bytes (32 bf16 or 16 fp32 columns), written by each
// lane for its own row into one of the warp's two 2 KB buffers and stored to
// C with one TMA store.  The buffers use the copy engine's 64-byte swizzle
// (16-byte granule g of row r sits at granule g ^ ((r >> 1) & 3)), so the
// lanes' 16-byte writes spread over all banks.  The tensor map clips rows
// >= M exactly, but along a row the copy engine writes whole 16-byte units,
// so the one piece of a row of tiles that reaches past column N is written
// with bounds-checked plain stores instead.
struct EpiWriter {
    const CUtensorMap *map;
    uint32_t buf;      // this warp's two pieces (1024-byte aligned)
    int count;         // pieces issued so far (selects the buffer)
    int lane;
    void *c;           // C and its shape, for the piece at the right edge
    int64_t ldc;
    int M, N;
};
// vals: 32 accumulator words (bf16 output) or 16 (fp32 output) of this lane's row;
// NBUF staging buffers per warp (2: a store may still read one while the
// other is written; 1: each piece waits for the previous store's read)
template <int OUT, int NBUF = 2>
__device__ __forceinline__ void epi_piece(EpiWriter &w, const uint32_t *vals, float alpha, int x, int y) {
    constexpr int PC = OUT == OUT_BF16 ? 32 : 16;   // columns per piece
    if (x + PC > w.N) {
        // right edge of C: plain stores of the columns that exist, rows < M
        const int m = y + w.lane;
        if (m < w.M) {
            if constexpr (OUT == OUT_BF16) {
                __nv_bfloat16 *row = static_cast<__nv_bfloat16 *>(w.c) + static_cast<int64_t>(m) * w.ldc + x;
#pragma unroll
                for (int i = 0; i < PC; ++i)
                    if (x + i < w.N) row[i] = __float2bfloat16_rn(__fmul_rn(__uint_as_float(vals[i]), alpha));
            } else {
                float *row = static_cast<float *>(w.c) + static_cast<int64_t>(m) * w.ldc + x;
#pragma unroll
                for (int i = 0; i < PC; ++i)
                    if (x + i < w.N) row[i] = __fmul_rn(__uint_as_float(vals[i]), alpha);
            }
        }
        return;
    }
    const uint32_t b = w.buf + static_cast<uint32_t>(w.count % NBUF) * EPI_PIECE;
    if (w.lane == 0) bulk_wait_read<NBUF - 1>();   // this buffer's previous store has read it
    __syncwarp();
    uint32_t q[16];
    if constexpr (OUT == OUT_BF16) {
#pragma unroll
        for (int i = 0; i < 16; ++i) {
            __nv_bfloat162 h = __floats2bfloat162_rn(__fmul_rn(__uint_as_float(vals[2 * i]), alpha),
                                                     __fmul_rn(__uint_as_float(vals[2 * i + 1]), alpha));
            q[i] = *reinterpret_cast<uint32_t *>(&h);
        }
    } else {
#pragma unroll
        for (int i = 0; i < 16; ++i) q[i] = __float_as_uint(__fmul_rn(__uint_as_float(vals[i]), alpha));
    }
    const uint32_t row = b + static_cast<uint32_t>(w.lane) * 64u;
    const uint32_t sw = (static_cast<uint32_t>(w.lane) >> 1) & 3u;
#pragma unroll
    for (uint32_t g = 0; g < 4; ++g)
        st_shared_v4(row + ((g ^ sw) << 4), q[4 * g], q[4 * g + 1], q[4 * g + 2], q[4 * g + 3]);
    fence_async_smem();
    __syncwarp();
    if (w.lane == 0) {
        tma_store_2d(w.map, b, x, y);
        bulk_commit();
    }
    ++w.count;
}

// 32 consecutive accumulator values of one row -> one MX block of C's row
// (quantizing epilogue; rows >= M and blocks past N are skipped).
__device__ __forceinline__ void store_chunk_mx(const Params &p, int m, int n0, const uint32_t *r) {
    if (m >= p.M || n0 >= p.N) return;
    quantize_chunk(p, m, n0, r);
}

template <bool FP4, int OUT>
__global__ void __launch_bounds__(NUM_THREADS, 1)
mx_gemm_kernel(const __grid_constant__ CUtensorMap tma_a, const __grid_constant__ CUtensorMap tma_b,
               const __grid_constant__ CUtensorMap tma_c, Params p) {
    using C = Cfg<FP4>;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t sbase = smem_u32(smem);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + Smem::ABORT);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + Smem::TMEM_SLOT);

    auto full_bar = [&](int s) { return sbase + Smem::BAR + 8u * s; };
    auto empty_bar = [&](int s) { return sbase + Smem::BAR + 8u * (STAGES + s); };
    auto acc_full = [&](int b) { return sbase + Smem::BAR + 8u * (2 * STAGES + b); };
    auto acc_empty = [&](int b) { return sbase + Smem::BAR + 8u * (2 * STAGES + 2 + b); };
    const uint32_t drain_bar = sbase + Smem::BAR + 8u * (2 * STAGES + 4);

    if (threadIdx.x == 0) {
        *abort_flag = 0;
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(full_bar(s), 1);
            mbar_init(empty_bar(s), 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(acc_full(b), 1);
            mbar_init(acc_empty(b), EPI_WARPS);
        }
        mbar_init(drain_bar, 1);
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    }
    if (warp == 1) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;"
                     ::"r"(smem_u32(tmem_slot)), "r"(TMEM_COLS) : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const int num_tiles = p.tiles_m * p.tiles_n;
    // programmatic dependent launch: barriers and tensor memory are set up
    // above; no global memory is touched before the previous kernel is done
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    asm volatile("griddepcontrol.wait;" ::: "memory");

    if (warp == 0) {
        // ------------------------------ producer ------------------------------
        if (lane == 0) {
            int s = 0;
            uint32_t ph = 0;
            uint32_t outstanding = 0;   // bit s: stage s has loads in flight not yet observed
            bool ok = true;
            for (int tile = blockIdx.x; tile < num_tiles && ok; tile += gridDim.x) {
                int tm, tn;
                tile_coords(tile, p.tiles_m, p.tiles_n, p.raster_group, p.raster_n_major, tm, tn);
                const int m0 = tm * BM, n0 = tn * BN;
                const int rb_a = m0 / 128, rb_b = n0 / 128;   // 128-row scale blocks
                const bool b_second = (rb_b + 1) * 128 < p.N;
                for (int kt = 0; kt < p.k_tiles; ++kt) {
                    if (!wait_bounded(empty_bar(s), ph ^ 1u, abort_flag)) { ok = false; break; }
                    if (kt == p.skip_k_tile && tile == static_cast<int>(blockIdx.x) && blockIdx.x == 0) {
                        ok = false;          // injected stall: this stage is never filled
                        break;
                    }
                    const uint32_t bytes = p.ab_tx + C::SFA_BYTES + (b_second ? 2 : 1) * (C::SFB_BYTES / 2);
                    const uint32_t fb = full_bar(s);
                    mbar_expect_tx(fb, bytes);
                    tma_load_2d(sbase + Smem::A + s * A_STAGE_BYTES, &tma_a, kt * BK_BYTES, m0, fb);
                    tma_load_2d(sbase + Smem::B + s * B_STAGE_BYTES, &tma_b, kt * BK_BYTES, n0, fb);
                    const int kg = kt * C::G;
                    bulk_load(sbase + Smem::SFA + s * 2 * ATOM,
                              p.a_scales + (static_cast<int64_t>(rb_a) * p.k_groups + kg) * ATOM, C::SFA_BYTES, fb);
                    bulk_load(sbase + Smem::SFB + s * 4 * ATOM,
                              p.b_scales + (static_cast<int64_t>(rb_b) * p.k_groups + kg) * ATOM, C::SFB_BYTES / 2, fb);
                    if (b_second)
                        bulk_load(sbase + Smem::SFB + s * 4 * ATOM + C::SFB_BYTES / 2,
                                  p.b_scales + (static_cast<int64_t>(rb_b + 1) * p.k_groups + kg) * ATOM,
                                  C::SFB_BYTES / 2, fb);
                    outstanding |= 1u << s;
                    if (++s == STAGES) { s = 0; ph ^= 1u; }
                    outstanding &= ~(1u << s);   // its previous use was released by the MMA
                }
            }
            if (!ok) {
                // drain: wait (bounded) for every stage whose loads may still land
                int ds = s;
                uint32_t dph = ph;
                for (int i = 0; i < STAGES; ++i) {
                    ds = ds == 0 ? STAGES - 1 : ds - 1;
                    if (ds == STAGES - 1) dph ^= 1u;
                    if (outstanding & (1u << ds)) {
                        volatile int no_abort = 0;
                        (void)wait_bounded(full_bar(ds), dph, &no_abort, DRAIN_LIMIT_NS);
                    }
                }
            }
        }
    } else if (warp == 1) {
        // ------------------------------ MMA issuer ----------------------------
        if (lane == 0) {
            int s = 0;
            uint32_t ph = 0;
            bool ok = true;
            bool issued = false;
            int local = 0;
            for (int tile = blockIdx.x; tile < num_tiles && ok; tile += gridDim.x, ++local) {
                const int b = local & 1;
                const uint32_t acc_ph = (local >> 1) & 1;
                if (!wait_bounded(acc_empty(b), acc_ph ^ 1u, abort_flag)) { ok = false; break; }
                tc_fence_after();
                int tm, tn;
                tile_coords(tile, p.tiles_m, p.tiles_n, p.raster_group, p.raster_n_major, tm, tn);
                const uint32_t d_tmem = tmem + b * ACC_COLS;
                const uint32_t sfb_shift = (tn & 1) ? 2u : 0u;   // odd 192-column tiles
                for (int kt = 0; kt < p.k_tiles; ++kt) {
                    if (!wait_bounded(full_bar(s), ph, abort_flag)) { ok = false; break; }
                    tc_fence_after();
                    const uint32_t sfa_t = tmem + SF_COL + s * C::SF_STAGE_COLS;
                    const uint32_t sfb_t = sfa_t + C::SFA_COLS;
                    const uint32_t sfa_s = sbase + Smem::SFA + s * 2 * ATOM;
                    const uint32_t sfb_s = sbase + Smem::SFB + s * 4 * ATOM;
#pragma unroll
                    for (int g = 0; g < C::G; ++g) {
                        tc_cp_scale_atom(sfa_t + 4 * g, scale_atom_desc(sfa_s + g * ATOM));
#pragma unroll
                        for (int h = 0; h < 2; ++h)
                            tc_cp_scale_atom(sfb_t + 8 * g + 4 * h,
                                             scale_atom_desc(sfb_s + h * (C::SFB_BYTES / 2) + g * ATOM));
                    }
                    const uint32_t a_s = sbase + Smem::A + s * A_STAGE_BYTES;
                    const uint32_t b_s = sbase + Smem::B + s * B_STAGE_BYTES;
#pragma unroll
                    for (int k = 0; k < 4; ++k) {
                        // FP8: k-block k of the atom; FP4: k-blocks 2k, 2k+1 (atom k/2, bytes 2k%4..)
                        const uint32_t g = FP4 ? (k >> 1) : 0u;
                        const uint32_t sf_id = FP4 ? ((2u * k) & 3u) : static_cast<uint32_t>(k);
                        const uint32_t idesc = p.idesc | (sf_id << 4) | (sf_id << 29);
                        tc_mma<FP4>(d_tmem, operand_desc(a_s, 32u * k), operand_desc(b_s, 32u * k), idesc,
                                    sfa_t + 4 * g, sfb_t + 8 * g + sfb_shift, (kt > 0 || k > 0) ? 1u : 0u);
                    }
                    issued = true;
                    tc_commit(empty_bar(s));
                    if (++s == STAGES) { s = 0; ph ^= 1u; }
                }
                if (!ok) break;
                tc_commit(acc_full(b));
            }
            if (issued) {
                // all issued MMAs must finish before TMEM is released
                tc_commit(drain_bar);
                volatile int no_abort = 0;
                (void)wait_bounded(drain_bar, 0, &no_abort, ok ? WAIT_LIMIT_NS : DRAIN_LIMIT_NS);
            }
        }
    } else {
        // ------------------------------ epilogue ------------------------------
        const int q = warp & 3;                  // TMEM lane quarter this warp may access
        const int half = (warp - 2) >> 2;        // which 96 columns of the tile
        EpiWriter ew{&tma_c, sbase + Smem::EPI + static_cast<uint32_t>(warp - 2) * EPI_WARP_BYTES, 0, lane,
                     p.c, p.ldc, p.M, p.N};
        int local = 0;
        for (int tile = blockIdx.x; tile < num_tiles; tile += gridDim.x, ++local) {
            const int b = local & 1;
            const uint32_t acc_ph = (local >> 1) & 1;
            // one lane waits, the warp follows its verdict: tcgen05.ld below
            // must be executed by all 32 lanes together
            int ok = 1;
            if (lane == 0) ok = wait_bounded(acc_full(b), acc_ph, abort_flag) ? 1 : 0;
            ok = __shfl_sync(0xffffffffu, ok, 0);
            if (!ok) break;
            tc_fence_after();
            int tm, tn;
            tile_coords(tile, p.tiles_m, p.tiles_n, p.raster_group, p.raster_n_major, tm, tn);
            const int m = tm * BM + q * 32 + lane;
            const int c0 = half * (BN / 2);
            const uint32_t taddr = tmem + b * ACC_COLS + (static_cast<uint32_t>(q * 32) << 16) + c0;
            uint32_t r[96];
            tmem_ld_x32_nowait(taddr, r);
            tmem_ld_x32_nowait(taddr + 32, r + 32);
            tmem_ld_x32_nowait(taddr + 64, r + 64);
            tmem_wait_ld();
            // the accumulator buffer can be refilled as soon as it is in registers
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(acc_empty(b));
            const int n_base = tn * BN + c0;
            if constexpr (OUT == OUT_MX) {
#pragma unroll
                for (int j = 0; j < 3; ++j) store_chunk_mx(p, m, n_base + 32 * j, r + 32 * j);
            } else {
                const int m_warp = tm * BM + q * 32;
                constexpr int PC = OUT == OUT_BF16 ? 32 : 16;   // columns per piece
                if (m_warp < p.M) {
#pragma unroll
                    for (int j = 0; j < (BN / 2) / PC; ++j)
                        if (n_base + PC * j < p.N) epi_piece<OUT>(ew, r + PC * j, p.alpha, n_base + PC * j, m_warp);
                }
            }
        }
        if (lane == 0) bulk_wait_all();          // stores done reading shared memory and written
    }

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 1) {
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(TMEM_COLS) : "memory");
    }
}

// ------------------------------------------------------------------------
// Resident-B kernel for short K (one SM per CTA, 128 x 192 tiles): when the
// whole K of a 192-row B panel fits in shared memory (at most six 128-byte K
// slices: K <= 768 for MXFP8, 1536 for MXFP4), each CTA takes a contiguous
// range of tiles in panel-major order (all M tiles of one N panel, then the
// next), loads its B panel and the panel's scale atoms once, and streams only
// A per tile.  The one-SM kernel reloads a 24 KiB B slice with every 16 KiB
// A slice; on such shapes the operand stream from L2 is what bounds it.  The
// panel's B scale factors stay in tensor memory for the whole panel, so a K
// slice needs one scale copy (A's) instead of three.
// ------------------------------------------------------------------------
constexpr int PANEL_MAX_SLICES = 6;
constexpr int PANEL_A_STAGES = 3;

template <bool FP4> struct PanelCfg {
    static constexpr int G = FP4 ? 2 : 1;                        // scale atoms along K per slice
    static constexpr int MAX_ATOMS = PANEL_MAX_SLICES * G;       // per 128-row scale block
    static constexpr int OFF_B = 0;                              // the panel: slice k at k * B_STAGE_BYTES
    static constexpr int OFF_SFB = OFF_B + PANEL_MAX_SLICES * B_STAGE_BYTES;   // two row blocks of atoms
    static constexpr int OFF_A = OFF_SFB + 2 * MAX_ATOMS * ATOM;
    static constexpr int OFF_SFA = OFF_A + PANEL_A_STAGES * A_STAGE_BYTES;
    static constexpr int OFF_EPI = (OFF_SFA + PANEL_A_STAGES * G * ATOM + 1023) / 1024 * 1024;
    static constexpr int OFF_BAR = OFF_EPI + EPI_WARPS * EPI_PIECE;          // one staged piece per warp
    // a_full[S], a_empty[S], acc_full[2], acc_empty[2], panel_full, panel_empty, drain
    static constexpr int NUM_BARS = 2 * PANEL_A_STAGES + 7;
    static constexpr int OFF_TMEM = OFF_BAR + NUM_BARS * 8;
    static constexpr int OFF_ABORT = OFF_TMEM + 4;
    static constexpr int SMEM = OFF_ABORT + 4 + 1024;                        // + alignment slack
    // tensor memory: two 192-column accumulators, the panel's B scale factors
    // (8 columns per k-group: both row blocks), then A's per stage
    static constexpr uint32_t SFB_COL = 2 * ACC_COLS;
    static constexpr uint32_t SFA_COL = SFB_COL + 8 * MAX_ATOMS;
    static_assert(OFF_A % 1024 == 0, "operand tiles 1024-byte aligned");
    static_assert(SFA_COL + PANEL_A_STAGES * 4 * G <= TMEM_COLS, "tensor memory columns");
    static_assert(SMEM <= 232448, "shared memory per block");
};

template <bool FP4, int OUT>
__global__ void __launch_bounds__(NUM_THREADS, 1)
mx_gemm_panel_kernel(const __grid_constant__ CUtensorMap tma_a, const __grid_constant__ CUtensorMap tma_b,
                     const __grid_constant__ CUtensorMap tma_c, Params p) {
    using C = Cfg<FP4>;
    using PC = PanelCfg<FP4>;
    constexpr int S = PANEL_A_STAGES;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t sbase = smem_u32(smem);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + PC::OFF_ABORT);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + PC::OFF_TMEM);

    auto a_full = [&](int s) { return sbase + PC::OFF_BAR + 8u * s; };
    auto a_empty = [&](int s) { return sbase + PC::OFF_BAR + 8u * (S + s); };
    auto acc_full = [&](int b) { return sbase + PC::OFF_BAR + 8u * (2 * S + b); };
    auto acc_empty = [&](int b) { return sbase + PC::OFF_BAR + 8u * (2 * S + 2 + b); };
    const uint32_t panel_full = sbase + PC::OFF_BAR + 8u * (2 * S + 4);
    const uint32_t panel_empty = sbase + PC::OFF_BAR + 8u * (2 * S + 5);
    const uint32_t drain_bar = sbase + PC::OFF_BAR + 8u * (2 * S + 6);

    if (threadIdx.x == 0) {
        *abort_flag = 0;
        for (int s = 0; s < S; ++s) {
            mbar_init(a_full(s), 1);
            mbar_init(a_empty(s), 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(acc_full(b), 1);
            mbar_init(acc_empty(b), EPI_WARPS);
        }
        mbar_init(panel_full, 1);
        mbar_init(panel_empty, 1);
        mbar_init(drain_bar, 1);
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    }
    if (warp == 1) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;"
                     ::"r"(smem_u32(tmem_slot)), "r"(TMEM_COLS) : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    // this CTA's tiles: a contiguous range in panel-major order (tile t: N panel
    // t / tiles_m, M tile t % tiles_m)
    const int64_t num_tiles = static_cast<int64_t>(p.tiles_m) * p.tiles_n;
    const int t_begin = static_cast<int>(num_tiles * blockIdx.x / gridDim.x);
    const int t_end = static_cast<int>(num_tiles * (blockIdx.x + 1) / gridDim.x);
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    asm volatile("griddepcontrol.wait;" ::: "memory");

    if (warp == 0) {
        // ------------------------------ producer ------------------------------
        if (lane == 0) {
            int s = 0;
            uint32_t ph = 0;
            uint32_t outstanding = 0;   // bit s: stage s has loads in flight not yet observed
            int panel = -1, panels = 0;
            bool panel_out = false;     // the latest panel load may still be in flight
            bool ok = true;
            for (int t = t_begin; t < t_end && ok; ++t) {
                const int tn = t / p.tiles_m, tm = t % p.tiles_m;
                if (tn != panel) {
                    // the MMAs are done with the previous panel; load this one
                    if (panels > 0 && !wait_bounded(panel_empty, (panels - 1) & 1, abort_flag)) { ok = false; break; }
                    const int n0 = tn * BN, rb_b = n0 / 128;
                    const bool b_second = (rb_b + 1) * 128 < p.N;
                    const uint32_t at_bytes = static_cast<uint32_t>(p.k_groups) * ATOM;
                    mbar_expect_tx(panel_full, static_cast<uint32_t>(p.k_tiles) * (p.ab_tx - p.a_tx) +
                                                   (b_second ? 2u : 1u) * at_bytes);
                    for (int kt = 0; kt < p.k_tiles; ++kt)
                        tma_load_2d(sbase + PC::OFF_B + kt * B_STAGE_BYTES, &tma_b, kt * BK_BYTES, n0, panel_full);
                    bulk_load(sbase + PC::OFF_SFB, p.b_scales + static_cast<int64_t>(rb_b) * p.k_groups * ATOM,
                              at_bytes, panel_full);
                    if (b_second)
                        bulk_load(sbase + PC::OFF_SFB + PC::MAX_ATOMS * ATOM,
                                  p.b_scales + static_cast<int64_t>(rb_b + 1) * p.k_groups * ATOM, at_bytes,
                                  panel_full);
                    panel = tn;
                    ++panels;
                    panel_out = true;
                }
                const int m0 = tm * BM, rb_a = m0 / 128;
                for (int kt = 0; kt < p.k_tiles; ++kt) {
                    if (!wait_bounded(a_empty(s), ph ^ 1u, abort_flag)) { ok = false; break; }
                    if (kt == p.skip_k_tile && t == t_begin && blockIdx.x == 0) {
                        ok = false;          // injected stall: this stage is never filled
                        break;
                    }
                    const uint32_t fb = a_full(s);
                    mbar_expect_tx(fb, p.a_tx + C::G * ATOM);
                    tma_load_2d(sbase + PC::OFF_A + s * A_STAGE_BYTES, &tma_a, kt * BK_BYTES, m0, fb);
                    bulk_load(sbase + PC::OFF_SFA + s * C::G * ATOM,
                              p.a_scales + (static_cast<int64_t>(rb_a) * p.k_groups + kt * C::G) * ATOM,
                              C::G * ATOM, fb);
                    outstanding |= 1u << s;
                    if (++s == S) { s = 0; ph ^= 1u; }
                    outstanding &= ~(1u << s);   // its previous use was released by the MMA
                }
            }
            if (!ok) {
                // drain: wait (bounded) for every stage and the panel whose loads may still land
                volatile int no_abort = 0;
                int ds = s;
                uint32_t dph = ph;
                for (int i = 0; i < S; ++i) {
                    ds = ds == 0 ? S - 1 : ds - 1;
                    if (ds == S - 1) dph ^= 1u;
                    if (outstanding & (1u << ds)) (void)wait_bounded(a_full(ds), dph, &no_abort, DRAIN_LIMIT_NS);
                }
                if (panel_out) (void)wait_bounded(panel_full, (panels - 1) & 1, &no_abort, DRAIN_LIMIT_NS);
            }
        }
    } else if (warp == 1) {
        // ------------------------------ MMA issuer ----------------------------
        if (lane == 0) {
            int s = 0;
            uint32_t ph = 0;
            bool ok = true;
            bool issued = false;
            int panel = -1, panels = 0;
            int local = 0;
            for (int t = t_begin; t < t_end && ok; ++t, ++local) {
                const int tn = t / p.tiles_m;
                if (tn != panel) {
                    // the previous panel is free once its MMAs complete
                    if (panels > 0) tc_commit(panel_empty);
                    if (!wait_bounded(panel_full, panels & 1, abort_flag)) { ok = false; break; }
                    tc_fence_after();
                    // the panel's B scale atoms -> tensor memory, 8 columns per k-group
                    const uint32_t sfb_s = sbase + PC::OFF_SFB;
                    for (int g = 0; g < p.k_groups; ++g)
                        for (int h = 0; h < 2; ++h)
                            tc_cp_scale_atom(tmem + PC::SFB_COL + 8 * g + 4 * h,
                                             scale_atom_desc(sfb_s + h * PC::MAX_ATOMS * ATOM + g * ATOM));
                    issued = true;
                    panel = tn;
                    ++panels;
                }
                const int b = local & 1;
                const uint32_t acc_ph = (local >> 1) & 1;
                if (!wait_bounded(acc_empty(b), acc_ph ^ 1u, abort_flag)) { ok = false; break; }
                tc_fence_after();
                const uint32_t d_tmem = tmem + b * ACC_COLS;
                const uint32_t sfb_shift = (tn & 1) ? 2u : 0u;   // odd 192-column tiles
                for (int kt = 0; kt < p.k_tiles; ++kt) {
                    if (!wait_bounded(a_full(s), ph, abort_flag)) { ok = false; break; }
                    tc_fence_after();
                    const uint32_t sfa_t = tmem + PC::SFA_COL + s * 4 * C::G;
                    const uint32_t sfa_s = sbase + PC::OFF_SFA + s * C::G * ATOM;
#pragma unroll
                    for (int g = 0; g < C::G; ++g) tc_cp_scale_atom(sfa_t + 4 * g, scale_atom_desc(sfa_s + g * ATOM));
                    const uint32_t a_s = sbase + PC::OFF_A + s * A_STAGE_BYTES;
                    const uint32_t b_s = sbase + PC::OFF_B + kt * B_STAGE_BYTES;
#pragma unroll
                    for (int k = 0; k < 4; ++k) {
                        // FP8: k-block k of the atom; FP4: k-blocks 2k, 2k+1 (atom k/2, bytes 2k%4..)
                        const uint32_t g = FP4 ? (k >> 1) : 0u;
                        const uint32_t sf_id = FP4 ? ((2u * k) & 3u) : static_cast<uint32_t>(k);
                        const uint32_t idesc = p.idesc | (sf_id << 4) | (sf_id << 29);
                        tc_mma<FP4>(d_tmem, operand_desc(a_s, 32u * k), operand_desc(b_s, 32u * k), idesc,
                                    sfa_t + 4 * g,
                                    tmem + PC::SFB_COL + 8 * (kt * C::G + g) + sfb_shift, (kt > 0 || k > 0) ? 1u : 0u);
                    }
                    issued = true;
                    tc_commit(a_empty(s));
                    if (++s == S) { s = 0; ph ^= 1u; }
                }
                if (!ok) break;
                tc_commit(acc_full(b));
            }
            if (issued) {
                // all issued MMAs and copies must finish before TMEM is released
                tc_commit(drain_bar);
                volatile int no_abort = 0;
                (void)wait_bounded(drain_bar, 0, &no_abort, ok ? WAIT_LIMIT_NS : DRAIN_LIMIT_NS);
            }
        }
    } else {
        // ------------------------------ epilogue ------------------------------
        const int q = warp & 3;                  // TMEM lane quarter this warp may access
        const int half = (warp - 2) >> 2;        // which 96 columns of the tile
        EpiWriter ew{&tma_c, sbase + PC::OFF_EPI + static_cast<uint32_t>(warp - 2) * EPI_PIECE, 0, lane,
                     p.c, p.ldc, p.M, p.N};
        int local = 0;
        for (int t = t_begin; t < t_end; ++t, ++local) {
            const int b = local & 1;
            const uint32_t acc_ph = (local >> 1) & 1;
            int ok = 1;
            if (lane == 0) ok = wait_bounded(acc_full(b), acc_ph, abort_flag) ? 1 : 0;
            ok = __shfl_sync(0xffffffffu, ok, 0);
            if (!ok) break;
            tc_fence_after();
            const int tn = t / p.tiles_m, tm = t % p.tiles_m;
            const int m = tm * BM + q * 32 + lane;
            const int c0 = half * (BN / 2);
            const uint32_t taddr = tmem + b * ACC_COLS + (static_cast<uint32_t>(q * 32) << 16) + c0;
            uint32_t r[96];
            tmem_ld_x32_nowait(taddr, r);
            tmem_ld_x32_nowait(taddr + 32, r + 32);
            tmem_ld_x32_nowait(taddr + 64, r + 64);
            tmem_wait_ld();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(acc_empty(b));
            const int n_base = tn * BN + c0;
            if constexpr (OUT == OUT_MX) {
#pragma unroll
                for (int j = 0; j < 3; ++j) store_chunk_mx(p, m, n_base + 32 * j, r + 32 * j);
            } else {
                const int m_warp = tm * BM + q * 32;
                constexpr int PCOL = OUT == OUT_BF16 ? 32 : 16;  // columns per piece
                if (m_warp < p.M) {
#pragma unroll
                    for (int j = 0; j < (BN / 2) / PCOL; ++j)
                        if (n_base + PCOL * j < p.N)
                            epi_piece<OUT, 1>(ew, r + PCOL * j, p.alpha, n_base + PCOL * j, m_warp);
                }
            }
        }
        if (lane == 0) bulk_wait_all();          // stores done reading shared memory and written
    }

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 1) {
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(TMEM_COLS) : "memory");
    }
}

// ------------------------------------------------------------------------
// Two-SM kernel (cta_group::2): a cluster of two CTAs computes a 256 x 256
// tile.  CTA r of the pair holds rows [128 r, 128 r + 128) of A and B rows
// [128 r, 128 r + 128) in its shared memory; one tcgen05.mma.cta_group::2
// issued by CTA 0 consumes both halves and writes each CTA's 128 accumulator
// rows into that CTA's tensor memory.  Every tensor-memory copy and MMA
// therefore covers twice the work of the one-SM kernel, and each SM loads only
// half of the B tile.  Each CTA keeps its own A scales and the full B scales
// (the pair-wide tcgen05.cp copies each CTA's shared memory into its own
// tensor memory).  All loads of both CTAs complete on CTA 0's stage barrier
// (the two-SM form of the TMA load); CTA 0's commit frees the stage in both
// CTAs.  Two tile widths: 256 columns, whose fp32 accumulator leaves no room
// for a second one next to the scale factors (the epilogue first drains the
// accumulator into registers, releases it to the MMA issuer, and only then
// stores to C), and 192 columns with two accumulators, so the next tile's
// MMAs run while the epilogue drains the previous one.  A 192-column tile at
// an odd position starts 64 rows into a 128-row B scale atom: its B scale
// factors are addressed two tensor-memory columns later.
// ------------------------------------------------------------------------
constexpr int PAIR_BM = 256;
constexpr int PAIR_A_BYTES = 128 * BK_BYTES;             // 16 KiB per CTA per stage

// NV: NVFP4 operands (kind::mxf4nvf4, 16-element blocks with E4M3 scales, so
// four scale atoms per 256-element K slice instead of two).
// KS: 128-byte K slices per pipeline stage.  Two slices per stage halve the
// barrier handshakes per K step between the producers and the MMA thread,
// which set the stage rate more than the bytes do (a loads-only probe of this
// operand stream: 18.4 TB/s with one slice per stage for any stage count from
// 3 to 6, 22.3 TB/s with two slices in 3 stages); the 256-column tiles of MX
// operands take them, the tensor memory of the other configurations has no
// room for the doubled scale columns.
// X4: operand scales in the x4 layout (each 512-byte atom stored four times,
// 2048 bytes): TMA lands the copies in the source layout of the 128-lane
// tcgen05.cp shapes, so a stage needs three copies (MXFP4: one 128x256b for
// A's two atoms, one 128x256b per k-group for B's two row blocks) instead of
// six replicating 32x128b.warpx4 copies.  One slice per stage (the scale
// bytes per stage are four times larger).
template <bool FP4, int PBN, bool NV = false, bool X4 = false> struct PairCfg {
    static constexpr int BN = PBN;                       // tile columns (B rows)
    static constexpr int B_ROWS = PBN / 2;               // B rows per CTA
    static constexpr int B_SLICE = B_ROWS * BK_BYTES;    // B bytes per CTA per K slice
    static constexpr int ACC_BUFS = PBN == 256 ? 1 : 2;  // accumulators in tensor memory
    static constexpr uint32_t SF_COL = ACC_BUFS * PBN;   // scale factors after the accumulators
    static constexpr int KS = (PBN == 256 && !NV && !X4) ? 2 : 1;
    static constexpr int G1 = NV ? 4 : (FP4 ? 2 : 1);    // scale atoms along K per slice
    static constexpr int G = KS * G1;                    // scale atoms along K per stage
    static constexpr int STAGES = X4 ? (NV ? 3 : (FP4 ? 4 : 5)) : (KS == 2 ? 3 : ((PBN == 192 && !FP4) ? 6 : 5));
    static constexpr int A_BYTES = KS * PAIR_A_BYTES;    // per CTA per stage
    static constexpr int B_BYTES = KS * B_SLICE;
    static constexpr int ATOM_BYTES = X4 ? 4 * ATOM : ATOM;   // one atom's bytes in memory
    static constexpr int SFA_BYTES = ATOM_BYTES * G;
    static constexpr int SFB_BYTES = 2 * ATOM_BYTES * G; // both 128-row scale blocks the tile touches
    static constexpr int SFA_COLS = 4 * G;
    static constexpr int SFB_COLS = 8 * G;
    static constexpr int SF_STAGE_COLS = SFA_COLS + SFB_COLS;
    static constexpr int EPI_BUFS = KS == 2 ? 1 : 2;     // staged pieces of C per epilogue warp
    // shared-memory layout
    static constexpr int OFF_A = 0;
    static constexpr int OFF_B = OFF_A + STAGES * A_BYTES;
    static constexpr int OFF_SFA = OFF_B + STAGES * B_BYTES;
    static constexpr int OFF_SFB = OFF_SFA + STAGES * SFA_BYTES;
    static constexpr int OFF_EPI = (OFF_SFB + STAGES * SFB_BYTES + 1023) / 1024 * 1024;
    static constexpr int EPI_WARP = EPI_BUFS * EPI_PIECE;
    static constexpr int OFF_BAR = OFF_EPI + EPI_WARPS * EPI_WARP;
    static constexpr int NUM_BARS = 2 * STAGES + 5;      // full, empty, acc_full, acc_empty, drain (+2 spare)
    static constexpr int OFF_TMEM = OFF_BAR + NUM_BARS * 8;
    static constexpr int OFF_ABORT = OFF_TMEM + 4;
    static constexpr int USED = OFF_ABORT + 4;
    // Slack for aligning the dynamic shared memory to 1024 bytes (128-byte
    // swizzled operand tiles).  Where the layout leaves no room for it, the
    // kernel requires the base to be aligned already and reports
    // MX_ERR_ALIGN through the device status word otherwise.
    static constexpr bool SLACK = USED + 1024 <= 232448;
    static constexpr int SMEM = USED + (SLACK ? 1024 : 0);
    static_assert(SF_COL + STAGES * SF_STAGE_COLS <= 512, "tensor memory columns");
    static_assert(SMEM <= 232448, "shared memory per block");
    static_assert(PBN == 256 || PBN == 192, "pair tile widths");
    static_assert(!X4 || PBN == 256, "x4 scales: 256-column tiles");
};

struct PairParams {
    void *c;
    int64_t ldc;
    int M, N, K;
    int k_tiles;
    int k_groups;
    int tiles_m, tiles_n;      // 256-row pair tiles
    float alpha;
    uint32_t idesc;
    uint32_t ab_tx;            // bytes one CTA's A and B loads of a stage deliver
    int skip_k_tile;
    int raster_group, raster_n_major;   // tile order (tile_coords)
    MxOut q;                   // OUT_MX only
    // NVFP4 only: the operands' per-domain encode scales and rows per domain
    // (0: one domain); C = alpha * acc / (E_A[m / a_lines] * E_B[n / b_lines])
    const float *enc_a, *enc_b;
    int a_lines, b_lines;
};

__device__ __forceinline__ uint32_t cluster_rank() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}
// address of the same shared-memory location in cluster CTA `rank`
__device__ __forceinline__ uint32_t map_to_rank(uint32_t addr, uint32_t rank) {
    uint32_t r;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(addr), "r"(rank));
    return r;
}
__device__ __forceinline__ void cluster_sync() {
    asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}
__device__ __forceinline__ void mbar_arrive_cluster(uint32_t cluster_addr) {
    asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(cluster_addr) : "memory");
}
// two-SM TMA load: data to this CTA's shared memory, bytes counted on the
// barrier at `bar_cluster_addr` (CTA 0's)
__device__ __forceinline__ void tma_load_2d_pair(uint32_t dst, const CUtensorMap *map, int x, int y,
                                                 uint32_t bar_cluster_addr) {
    asm volatile(
        "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];"
        ::"r"(dst), "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(bar_cluster_addr) : "memory");
}
__device__ __forceinline__ void tc_commit_pair(uint32_t bar) {
    asm volatile(
        "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], %1;"
        ::"r"(bar), "h"(static_cast<uint16_t>(3)) : "memory");
}
// x4 scales: 128 lanes x 256 bits (two 2048-byte atom copies, `lbo` bytes
// apart, into 8 columns) or 128 lanes x 128 bits (one, into 4 columns)
__device__ __forceinline__ void tc_cp_x4_pair_256b(uint32_t taddr, uint32_t src, uint32_t lbo) {
    asm volatile("tcgen05.cp.cta_group::2.128x256b [%0], %1;"
                 ::"r"(taddr), "l"(smem_desc(src, lbo, 128, LAYOUT_NONE)) : "memory");
}
__device__ __forceinline__ void tc_cp_x4_pair_128b(uint32_t taddr, uint32_t src) {
    asm volatile("tcgen05.cp.cta_group::2.128x128b [%0], %1;"
                 ::"r"(taddr), "l"(smem_desc(src, 16, 128, LAYOUT_NONE)) : "memory");
}
__device__ __forceinline__ void tc_cp_scale_atom_pair(uint32_t taddr, uint64_t desc) {
    asm volatile("tcgen05.cp.cta_group::2.32x128b.warpx4 [%0], %1;" ::"r"(taddr), "l"(desc) : "memory");
}
template <bool FP4, bool NV = false>
__device__ __forceinline__ void tc_mma_pair(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                            uint32_t sfa_tmem, uint32_t sfb_tmem, uint32_t accumulate) {
    if (NV) {
        asm volatile(
            "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %6, 0;\n\t"
            "tcgen05.mma.cta_group::2.kind::mxf4nvf4.block_scale.scale_vec::4X [%0], %1, %2, %3, [%4], [%5], p;\n\t}"
            ::"r"(d_tmem), "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(sfa_tmem), "r"(sfb_tmem), "r"(accumulate)
            : "memory");
    } else if (FP4) {
        asm volatile(
            "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %6, 0;\n\t"
            "tcgen05.mma.cta_group::2.kind::mxf4.block_scale.scale_vec::2X [%0], %1, %2, %3, [%4], [%5], p;\n\t}"
            ::"r"(d_tmem), "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(sfa_tmem), "r"(sfb_tmem), "r"(accumulate)
            : "memory");
    } else {
        asm volatile(
            "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %6, 0;\n\t"
            "tcgen05.mma.cta_group::2.kind::mxf8f6f4.block_scale.scale_vec::1X [%0], %1, %2, %3, [%4], [%5], p;\n\t}"
            ::"r"(d_tmem), "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(sfa_tmem), "r"(sfb_tmem), "r"(accumulate)
            : "memory");
    }
}

template <bool FP4, int OUT, int PBN, bool NV = false, bool X4 = false>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(NUM_THREADS, 1)
mx_gemm_pair_kernel(const __grid_constant__ CUtensorMap tma_a, const __grid_constant__ CUtensorMap tma_b,
                    const __grid_constant__ CUtensorMap tma_sfa, const __grid_constant__ CUtensorMap tma_sfb,
                    const __grid_constant__ CUtensorMap tma_c, PairParams p) {
    using C = PairCfg<FP4, PBN, NV, X4>;
    constexpr int STAGES_P = C::STAGES;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    if (!C::SLACK && (smem_u32(smem_raw) & 1023u) != 0) {
        // no room to realign (both CTAs of the pair see the same base and leave here)
        if (threadIdx.x == 0) atomicExch(&g_mx_status, MX_ERR_ALIGN);
        return;
    }
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t sbase = smem_u32(smem);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t rank = cluster_rank();
    volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + C::OFF_ABORT);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + C::OFF_TMEM);

    auto full_bar = [&](int s) { return sbase + C::OFF_BAR + 8u * s; };
    auto empty_bar = [&](int s) { return sbase + C::OFF_BAR + 8u * (STAGES_P + s); };
    auto acc_full = [&](int b) { return sbase + C::OFF_BAR + 8u * (2 * STAGES_P + b); };
    auto acc_empty = [&](int b) { return sbase + C::OFF_BAR + 8u * (2 * STAGES_P + 2 + b); };
    const uint32_t drain_bar = sbase + C::OFF_BAR + 8u * (2 * STAGES_P + 4);

    if (threadIdx.x == 0) {
        *abort_flag = 0;
        for (int s = 0; s < STAGES_P; ++s) {
            mbar_init(full_bar(s), 1);          // CTA 0's producer; bytes from both CTAs
            mbar_init(empty_bar(s), 1);         // CTA 0's commit, multicast to both CTAs
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(acc_full(b), 1);
            mbar_init(acc_empty(b), 2 * EPI_WARPS);   // epilogue warps of both CTAs (on CTA 0)
        }
        mbar_init(drain_bar, 1);
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    }
    if (warp == 1) {
        asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;"
                     ::"r"(smem_u32(tmem_slot)), "r"(TMEM_COLS) : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
    }
    tc_fence_before();
    cluster_sync();                  // barriers of both CTAs initialised, tensor memory allocated
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const int num_tiles = p.tiles_m * p.tiles_n;
    // programmatic dependent launch: barriers and tensor memory are set up
    // above; no global memory is touched before the previous kernel is done
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    asm volatile("griddepcontrol.wait;" ::: "memory");
    const int cluster_id = blockIdx.x >> 1, n_clusters = gridDim.x >> 1;

    if (warp == 0) {
        // ------------------------------ producer (both CTAs) -------------------
        if (lane == 0) {
            int s = 0;
            uint32_t ph = 0;
            bool ok = true;
            for (int tile = cluster_id; tile < num_tiles && ok; tile += n_clusters) {
                int tm, tn;
                tile_coords(tile, p.tiles_m, p.tiles_n, p.raster_group, p.raster_n_major, tm, tn);
                // this CTA's A rows and B rows; a half that lies wholly past M (or N)
                // only feeds discarded outputs, so its loads are clamped to rows
                // that exist and no TMA box is ever entirely outside its tensor
                const int m0 = min(tm * PAIR_BM + 128 * static_cast<int>(rank), p.M - 1);
                const int nb0 = min(tn * PBN + C::B_ROWS * static_cast<int>(rank), p.N - 1);
                const int rb_a = m0 / 128, rb_b = (tn * PBN) / 128;
                const int rb_b1 = min(rb_b + 1, (p.N - 1) / 128);
                for (int kt = 0; kt < p.k_tiles; kt += C::KS) {
                    if (!wait_bounded(empty_bar(s), ph ^ 1u, abort_flag)) { ok = false; break; }
                    if (rank == 0 && p.skip_k_tile >= kt && p.skip_k_tile < kt + C::KS && tile == cluster_id &&
                        cluster_id == 0) {
                        ok = false;          // injected stall: CTA 0 never arms this stage
                        break;
                    }
                    // K slices in this stage (the last stage may hold fewer); the
                    // scale boxes always cover the stage's G atoms, the atoms past
                    // the slices present being read but unused (zero past the end)
                    const int ns = min(C::KS, p.k_tiles - kt);
                    const uint32_t fb = map_to_rank(full_bar(s), 0);
                    if (rank == 0)
                        mbar_expect_tx(full_bar(s), 2 * (static_cast<uint32_t>(ns) * p.ab_tx + C::SFA_BYTES +
                                                         C::SFB_BYTES));
                    for (int q = 0; q < ns; ++q) {
                        tma_load_2d_pair(sbase + C::OFF_A + s * C::A_BYTES + q * PAIR_A_BYTES, &tma_a,
                                         (kt + q) * BK_BYTES, m0, fb);
                        tma_load_2d_pair(sbase + C::OFF_B + s * C::B_BYTES + q * C::B_SLICE, &tma_b,
                                         (kt + q) * BK_BYTES, nb0, fb);
                    }
                    // scale atoms: a scale buffer is viewed as rows of 256 bytes (two per
                    // atom; eight per x4 atom)
                    const int kg = kt * C::G1;
                    tma_load_2d_pair(sbase + C::OFF_SFA + s * C::SFA_BYTES, &tma_sfa, 0,
                                     C::ATOM_BYTES / 256 * (rb_a * p.k_groups + kg), fb);
                    tma_load_2d_pair(sbase + C::OFF_SFB + s * C::SFB_BYTES, &tma_sfb, 0,
                                     C::ATOM_BYTES / 256 * (rb_b * p.k_groups + kg), fb);
                    tma_load_2d_pair(sbase + C::OFF_SFB + s * C::SFB_BYTES + C::SFB_BYTES / 2, &tma_sfb, 0,
                                     C::ATOM_BYTES / 256 * (rb_b1 * p.k_groups + kg), fb);
                    if (++s == STAGES_P) { s = 0; ph ^= 1u; }
                }
            }
            if (!ok) {
                // this CTA's loads complete on CTA 0's barriers, which it cannot
                // wait on: after an abort, give any load still in flight far more
                // than its latency (microseconds) to land before the CTA may exit
                const unsigned long long t0 = globaltimer();
                while (globaltimer() - t0 < DRAIN_SETTLE_NS) {
                }
            }
        }
    } else if (warp == 1) {
        // ------------------------------ MMA issuer (CTA 0) ---------------------
        if (lane == 0 && rank == 0) {
            int s = 0;
            uint32_t ph = 0;
            bool ok = true;
            bool issued = false;
            int local = 0;
            for (int tile = cluster_id; tile < num_tiles && ok; tile += n_clusters, ++local) {
                const int b = local % C::ACC_BUFS;
                const uint32_t acc_ph = (local / C::ACC_BUFS) & 1;
                if (!wait_bounded(acc_empty(b), acc_ph ^ 1u, abort_flag)) { ok = false; break; }
                tc_fence_after();
                int tm, tn;
                tile_coords(tile, p.tiles_m, p.tiles_n, p.raster_group, p.raster_n_major, tm, tn);
                const uint32_t d_tmem = tmem + static_cast<uint32_t>(b * PBN);
                const uint32_t sfb_shift = ((tn * PBN) & 127) ? 2u : 0u;   // tile starts 64 rows into an atom
                for (int kt = 0; kt < p.k_tiles; kt += C::KS) {
                    if (!wait_bounded(full_bar(s), ph, abort_flag)) { ok = false; break; }
                    tc_fence_after();
                    const int ns = min(C::KS, p.k_tiles - kt);
                    const uint32_t sfa_t = tmem + C::SF_COL + s * C::SF_STAGE_COLS;
                    const uint32_t sfb_t = sfa_t + C::SFA_COLS;
                    const uint32_t sfa_s = sbase + C::OFF_SFA + s * C::SFA_BYTES;
                    const uint32_t sfb_s = sbase + C::OFF_SFB + s * C::SFB_BYTES;
                    if constexpr (X4) {
                        // A: the slice's atoms two per copy (one for MXFP8); B: per
                        // k-group, its two row blocks' atoms side by side
                        if (FP4) {
#pragma unroll
                            for (int i = 0; i < C::G / 2; ++i)
                                tc_cp_x4_pair_256b(sfa_t + 8 * i, sfa_s + 2 * i * C::ATOM_BYTES, C::ATOM_BYTES);
                        } else {
                            tc_cp_x4_pair_128b(sfa_t, sfa_s);
                        }
#pragma unroll
                        for (int g = 0; g < C::G; ++g)
                            tc_cp_x4_pair_256b(sfb_t + 8 * g, sfb_s + g * C::ATOM_BYTES, C::SFB_BYTES / 2);
                    }
#pragma unroll
                    for (int g = 0; g < C::G; ++g) {
                        if (!X4 && g < ns * C::G1) {
                            tc_cp_scale_atom_pair(sfa_t + 4 * g, scale_atom_desc(sfa_s + g * ATOM));
#pragma unroll
                            for (int h = 0; h < 2; ++h)
                                tc_cp_scale_atom_pair(sfb_t + 8 * g + 4 * h,
                                                      scale_atom_desc(sfb_s + h * (C::SFB_BYTES / 2) + g * ATOM));
                        }
                    }
#pragma unroll
                    for (int q = 0; q < C::KS; ++q) {
                        if (q < ns) {
                            const uint32_t a_s = sbase + C::OFF_A + s * C::A_BYTES + q * PAIR_A_BYTES;
                            const uint32_t b_s = sbase + C::OFF_B + s * C::B_BYTES + q * C::B_SLICE;
#pragma unroll
                            for (int k = 0; k < 4; ++k) {
                                // MXFP8: k-block k of the slice's atom; MXFP4: k-blocks 2k, 2k + 1
                                // of atom k / 2; NVFP4: all four 16-element blocks of atom k
                                const uint32_t g = q * C::G1 + (NV ? static_cast<uint32_t>(k) : (FP4 ? (k >> 1) : 0u));
                                const uint32_t sf_id = NV ? 0u : (FP4 ? ((2u * k) & 3u) : static_cast<uint32_t>(k));
                                const uint32_t idesc = p.idesc | (sf_id << 4) | (sf_id << 29);
                                tc_mma_pair<FP4, NV>(d_tmem, operand_desc(a_s, 32u * k), operand_desc(b_s, 32u * k),
                                                     idesc, sfa_t + 4 * g, sfb_t + 8 * g + sfb_shift,
                                                     (kt > 0 || q > 0 || k > 0) ? 1u : 0u);
                            }
                        }
                    }
                    issued = true;
                    tc_commit_pair(empty_bar(s));
                    if (++s == STAGES_P) { s = 0; ph ^= 1u; }
                }
                if (!ok) break;
                tc_commit_pair(acc_full(b));
            }
            if (issued) {
                tc_commit_pair(drain_bar);   // same cta_group as every other tcgen05 op here
                volatile int no_abort = 0;
                (void)wait_bounded(drain_bar, 0, &no_abort, ok ? WAIT_LIMIT_NS : DRAIN_LIMIT_NS);
            }
        }
    } else {
        // ------------------------------ epilogue (both CTAs) -------------------
        const int q = warp & 3;
        const int half = (warp - 2) >> 2;
        EpiWriter ew{&tma_c, sbase + C::OFF_EPI + static_cast<uint32_t>(warp - 2) * C::EPI_WARP, 0, lane,
                     p.c, p.ldc, p.M, p.N};
        int local = 0;
        constexpr int NCH = PBN / 2 / 32;        // 32-column chunks per warp
        for (int tile = cluster_id; tile < num_tiles; tile += n_clusters, ++local) {
            const int b = local % C::ACC_BUFS;
            const uint32_t acc_ph = (local / C::ACC_BUFS) & 1;
            int ok = 1;
            if (lane == 0) ok = wait_bounded(acc_full(b), acc_ph, abort_flag) ? 1 : 0;
            ok = __shfl_sync(0xffffffffu, ok, 0);
            if (!ok) break;
            tc_fence_after();
            int tm, tn;
            tile_coords(tile, p.tiles_m, p.tiles_n, p.raster_group, p.raster_n_major, tm, tn);
            const int m = tm * PAIR_BM + 128 * static_cast<int>(rank) + q * 32 + lane;
            const int c0 = half * (PBN / 2);
            const uint32_t taddr = tmem + static_cast<uint32_t>(b * PBN) + (static_cast<uint32_t>(q * 32) << 16) + c0;
            uint32_t r[32 * NCH];
#pragma unroll
            for (int j = 0; j < NCH; ++j) tmem_ld_x32_nowait(taddr + 32 * j, r + 32 * j);
            tmem_wait_ld();
            // the accumulator is in registers: hand it back to the MMA issuer
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive_cluster(map_to_rank(acc_empty(b), 0));
            const int n_base = tn * PBN + c0;
            if constexpr (OUT == OUT_MX) {
                Params pp;
                pp.c = p.c; pp.ldc = p.ldc; pp.M = p.M; pp.N = p.N; pp.alpha = p.alpha; pp.q = p.q;
#pragma unroll
                for (int j = 0; j < NCH; ++j) store_chunk_mx(pp, m, n_base + 32 * j, r + 32 * j);
            } else {
                const int m_warp = tm * PAIR_BM + 128 * static_cast<int>(rank) + q * 32;
                constexpr int PC = OUT == OUT_BF16 ? 32 : 16;   // columns per piece
                // NVFP4: alpha / E_A of this row, then / E_B of the piece's columns
                float fa = p.alpha;
                if (NV) fa = __fdiv_rn(p.alpha, p.enc_a[p.a_lines ? min(m, p.M - 1) / p.a_lines : 0]);
                if (m_warp < p.M) {
#pragma unroll
                    for (int j = 0; j < (PBN / 2) / PC; ++j) {
                        const int n0 = n_base + PC * j;
                        if (n0 >= p.N) continue;
                        const float f = NV ? __fdiv_rn(fa, p.enc_b[p.b_lines ? n0 / p.b_lines : 0]) : fa;
                        epi_piece<OUT, C::EPI_BUFS>(ew, r + PC * j, f, n0, m_warp);
                    }
                }
            }
        }
        if (lane == 0) bulk_wait_all();          // stores done reading shared memory and written
    }

    tc_fence_before();
    cluster_sync();                  // all MMAs drained and all epilogue reads done in both CTAs
    tc_fence_after();
    if (warp == 1) {
        asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(TMEM_COLS) : "memory");
    }
}

// ------------------------------------------------------------------------
// Host side
// ------------------------------------------------------------------------
PFN_cuTensorMapEncodeTiled_v12000 get_encode() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
    });
    return fn;
}

int elem_bits(int f) { return f == MX_E2M1 ? 4 : (f == MX_E2M3 || f == MX_E3M2) ? 6 : 8; }

// Encoded 2-D tensor maps, reused across calls.  A map is a pure function of
// the arguments of its encoding (address, element type, sizes, row stride,
// box, swizzle), so a cached map stays valid whatever buffer lives at that
// address later.  Direct-mapped, 256 entries, one lock.
struct MapKey {
    const void *base;
    uint64_t d0, d1, stride;
    uint32_t b0, b1;
    int dt, swz;
    bool operator==(const MapKey &o) const {
        return base == o.base && d0 == o.d0 && d1 == o.d1 && stride == o.stride && b0 == o.b0 && b1 == o.b1 &&
               dt == o.dt && swz == o.swz;
    }
};
struct MapSlot {
    bool used = false;
    MapKey key{};
    CUtensorMap map{};
};
constexpr int kMapSlots = 256;
MapSlot g_map_cache[kMapSlots];
std::mutex g_map_lock;

bool encode_2d(CUtensorMap *map, CUtensorMapDataType dt, const void *base, uint64_t d0, uint64_t d1,
               uint64_t stride, uint32_t b0, uint32_t b1, CUtensorMapSwizzle swz) {
    const MapKey key{base, d0, d1, stride, b0, b1, static_cast<int>(dt), static_cast<int>(swz)};
    uint64_t h = reinterpret_cast<uintptr_t>(base) >> 4;
    for (uint64_t v : {d0, d1, stride, static_cast<uint64_t>(b0) << 32 | b1,
                       static_cast<uint64_t>(key.dt) << 8 | static_cast<uint64_t>(key.swz)})
        h = (h ^ v) * 0x100000001b3ull;
    MapSlot &slot = g_map_cache[(h ^ (h >> 29)) % kMapSlots];
    {
        std::lock_guard<std::mutex> g(g_map_lock);
        if (slot.used && slot.key == key) {
            *map = slot.map;
            return true;
        }
    }
    auto encode = get_encode();
    if (!encode) return false;
    cuuint64_t dims[2] = {d0, d1};
    cuuint64_t strides[1] = {stride};
    cuuint32_t box[2] = {b0, b1};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = encode(map, dt, 2, const_cast<void *>(base), dims, strides, box, estr,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, swz, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return false;
    std::lock_guard<std::mutex> g(g_map_lock);
    slot.used = true;
    slot.key = key;
    slot.map = *map;
    return true;
}

// Tensor map over one operand's codes (rows x K, K contiguous), a box of
// box_rows x one stage of K, 128-byte swizzle; rows past the end read as zero.
// kind::mxf4 takes E2M1 codes packed two to a byte, so its stage is 128 bytes
// = 256 codes of a uint8 view.  kind::mxf8f6f4 takes one code per byte in
// shared memory: FP8 codes are bytes already, and the copy engine expands
// FP6 (16 codes in 12 bytes) and FP4 (16 codes in 8 bytes) to 16 bytes each
// on the way in (the 16U6 / 16U4 packed tensor-map types), so a stage is 128
// codes in 128 bytes of shared memory for every element format.
bool make_operand_map(CUtensorMap *map, const void *base, int64_t rows, int64_t K, int fmt, bool mxf4,
                      int box_rows) {
    const int bits = elem_bits(fmt);
    CUtensorMapDataType dt = CU_TENSOR_MAP_DATA_TYPE_UINT8;
    uint64_t inner = static_cast<uint64_t>(K);                 // elements along K
    if (mxf4) inner = static_cast<uint64_t>(K / 2);            // bytes of packed pairs
    else if (bits == 6) dt = CU_TENSOR_MAP_DATA_TYPE_16U6_ALIGN16B;
    else if (bits == 4) dt = CU_TENSOR_MAP_DATA_TYPE_16U4_ALIGN16B;
    return encode_2d(map, dt, base, inner, static_cast<uint64_t>(rows), static_cast<uint64_t>(K * bits / 8),
                     BK_BYTES, static_cast<uint32_t>(box_rows), CU_TENSOR_MAP_SWIZZLE_128B);
}

// Bytes one stage's load of box_rows rows delivers: the packed size in global
// memory (128 bytes per row for FP8 and packed FP4, 96 for FP6, 64 for FP4
// expanded to bytes).
uint32_t stage_tx_bytes(int fmt, bool mxf4, int box_rows) {
    const int per_row = mxf4 ? BK_BYTES : BK_BYTES * elem_bits(fmt) / 8;
    return static_cast<uint32_t>(per_row * box_rows);
}

// 2-D uint8 view of an MMA-layout scale buffer as rows of 256 bytes (two rows
// per 512-byte atom); a box of 2 * atoms rows x 256 bytes, no swizzle.
bool make_scale_map(CUtensorMap *map, const void *base, int64_t bytes, int atoms_per_box) {
    if (bytes % 256 != 0) return false;
    return encode_2d(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, base, 256, static_cast<uint64_t>(bytes / 256), 256, 256,
                     static_cast<uint32_t>(2 * atoms_per_box), CU_TENSOR_MAP_SWIZZLE_NONE);
}

// Tensor map over C (M x N, leading dimension ldc) for the epilogue's TMA
// stores: boxes of 32 rows x 64 bytes (32 bf16 or 16 fp32 columns), 64-byte
// swizzle, matching the staged pieces.  Without a C (quantizing epilogue) the
// map is zeroed and never used.
bool make_c_map(CUtensorMap *map, const MxGemmArgs &a) {
    if (a.q_codes) {
        std::memset(map, 0, sizeof(*map));
        return true;
    }
    const bool bf16 = a.cdt == MX_BF16;
    const uint64_t esz = bf16 ? 2 : 4;
    return encode_2d(map, bf16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT32, a.c,
                     static_cast<uint64_t>(a.N), static_cast<uint64_t>(a.M), static_cast<uint64_t>(a.ldc) * esz,
                     bf16 ? 32u : 16u, 32u, CU_TENSOR_MAP_SWIZZLE_64B);
}

uint32_t make_idesc(int fa, int fb, bool fp4, int m = BM, int n = BN, bool nv = false) {
    auto code = [&](int f) -> uint32_t {
        if (fp4) return 1u;               // kind::mxf4: E2M1
        switch (f) {                      // kind::mxf8f6f4 operand type codes
            case MX_E5M2: return 1u;
            case MX_E2M3: return 3u;
            case MX_E3M2: return 4u;
            case MX_E2M1: return 5u;
            default: return 0u;           // E4M3
        }
    };
    uint32_t d = 0;
    d |= code(fa) << 7;
    d |= code(fb) << 10;
    d |= static_cast<uint32_t>(n >> 3) << 17;
    if (!nv) d |= 1u << 23;                // scale factors are UE8M0 (NVFP4: UE4M3, bit clear)
    d |= static_cast<uint32_t>(m >> 4) << 24;
    return d;
}

// Launch allowed to overlap the previous kernel in the stream (programmatic
// dependent launch); the kernel waits for that kernel's results itself.
template <typename Kern, typename... Args>
cudaError_t launch_overlapped(Kern kern, int grid, int smem, cudaStream_t st, const Args &...args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(NUM_THREADS);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kern, args...);
}

template <bool FP4, int OUT, int PBN, bool NV = false, bool X4 = false>
cudaError_t launch_pair(const CUtensorMap &ta, const CUtensorMap &tb, const CUtensorMap &tsa,
                        const CUtensorMap &tsb, const CUtensorMap &tc, const PairParams &p, int grid,
                        cudaStream_t st) {
    auto kern = mx_gemm_pair_kernel<FP4, OUT, PBN, NV, X4>;
    constexpr int smem = PairCfg<FP4, PBN, NV, X4>::SMEM;
    static std::atomic<uint64_t> configured{0};   // per instantiation, one bit per device
    if (cudaError_t e = ensure_smem_limit(kern, smem, configured); e != cudaSuccess) return e;
    return launch_overlapped(kern, grid, smem, st, ta, tb, tsa, tsb, tc, p);
}

template <bool FP4, int OUT>
cudaError_t launch(const CUtensorMap &ta, const CUtensorMap &tb, const CUtensorMap &tc, const Params &p, int grid,
                   cudaStream_t st) {
    auto kern = mx_gemm_kernel<FP4, OUT>;
    static std::atomic<uint64_t> configured{0};   // per instantiation, one bit per device
    if (cudaError_t e = ensure_smem_limit(kern, SMEM_BYTES, configured); e != cudaSuccess) return e;
    return launch_overlapped(kern, grid, SMEM_BYTES, st, ta, tb, tc, p);
}

template <bool FP4, int PBN>
cudaError_t launch_pair_out(int out, const CUtensorMap &ta, const CUtensorMap &tb, const CUtensorMap &tsa,
                            const CUtensorMap &tsb, const CUtensorMap &tc, const PairParams &p, int grid,
                            cudaStream_t st) {
    if (out == OUT_MX) return launch_pair<FP4, OUT_MX, PBN>(ta, tb, tsa, tsb, tc, p, grid, st);
    if (out == OUT_BF16) return launch_pair<FP4, OUT_BF16, PBN>(ta, tb, tsa, tsb, tc, p, grid, st);
    return launch_pair<FP4, OUT_F32, PBN>(ta, tb, tsa, tsb, tc, p, grid, st);
}

template <bool FP4, int OUT>
cudaError_t launch_panel(const CUtensorMap &ta, const CUtensorMap &tb, const CUtensorMap &tc, const Params &p,
                         int grid, cudaStream_t st) {
    auto kern = mx_gemm_panel_kernel<FP4, OUT>;
    constexpr int smem = PanelCfg<FP4>::SMEM;
    static std::atomic<uint64_t> configured{0};   // per instantiation, one bit per device
    if (cudaError_t e = ensure_smem_limit(kern, smem, configured); e != cudaSuccess) return e;
    return launch_overlapped(kern, grid, smem, st, ta, tb, tc, p);
}

template <bool FP4>
cudaError_t launch_panel_out(int out, const CUtensorMap &ta, const CUtensorMap &tb, const CUtensorMap &tc,
                             const Params &p, int grid, cudaStream_t st) {
    if (out == OUT_MX) return launch_panel<FP4, OUT_MX>(ta, tb, tc, p, grid, st);
    if (out == OUT_BF16) return launch_panel<FP4, OUT_BF16>(ta, tb, tc, p, grid, st);
    return launch_panel<FP4, OUT_F32>(ta, tb, tc, p, grid, st);
}

template <bool FP4>
cudaError_t launch_out(int out, const CUtensorMap &ta, const CUtensorMap &tb, const CUtensorMap &tc,
                       const Params &p, int grid, cudaStream_t st) {
    if (out == OUT_MX) return launch<FP4, OUT_MX>(ta, tb, tc, p, grid, st);
    if (out == OUT_BF16) return launch<FP4, OUT_BF16>(ta, tb, tc, p, grid, st);
    return launch<FP4, OUT_F32>(ta, tb, tc, p, grid, st);
}

int out_mode(const MxGemmArgs &a) {
    return a.q_codes ? OUT_MX : (a.cdt == MX_BF16 ? OUT_BF16 : OUT_F32);
}

MxOut mx_out(const MxGemmArgs &a) {
    MxOut q;
    q.codes = static_cast<uint8_t *>(a.q_codes);
    q.scales = static_cast<uint8_t *>(a.q_scales);
    q.fmt = a.q_fmt;
    q.sr = a.q_rnd == MX_SR;
    q.mma = a.q_sl;
    q.key = fmix32_host(static_cast<uint32_t>(a.q_seed)) ^ static_cast<uint32_t>(a.q_seed >> 32);
    return q;
}

}  // namespace mxg

namespace {
// armed by mx_debug_gemm_skip_stage; consumed by the next GEMM call of the same host thread
thread_local int g_skip_k_tile = -1;
// set by mx_debug_gemm_force_kernel for this host thread's GEMM calls (-1: automatic)
thread_local int g_force_kernel = -1;
}

extern "C" int mx_debug_gemm_force_kernel(int tile_n) {
    if (tile_n != -1 && tile_n != 0 && tile_n != 1 && tile_n != 192 && tile_n != 256) return MX_ERR_ARG;
    g_force_kernel = tile_n;
    return MX_OK;
}

extern "C" int mx_debug_gemm_skip_stage(int k_tile) {
    g_skip_k_tile = k_tile < 0 ? -1 : k_tile;
    return MX_OK;
}

namespace {

// Tile order for a shape: keep the operand whose codes fit in a third of the
// L2 resident (M fastest when A fits, N fastest when B fits) so that each
// operand is read from HBM about once; otherwise bands of 8 row-tiles.
void raster_for(const MxGemmArgs &a, int tiles_m, int tiles_n, int &group, int &n_major) {
    constexpr int64_t kResident = 40ll << 20;
    const int64_t a_bytes = a.M * a.K * mxg::elem_bits(a.fa) / 8, b_bytes = a.N * a.K * mxg::elem_bits(a.fb) / 8;
    if (a_bytes <= kResident) { group = tiles_m; n_major = 0; }
    else if (b_bytes <= kResident) { group = tiles_n; n_major = 1; }
    else { group = 8; n_major = 0; }
}

// E2M1 x E2M1 with K a multiple of 256 runs kind::mxf4 on packed codes (256
// per stage); every other pair, and FP4 x FP4 with K = 128 (mod 256), runs
// kind::mxf8f6f4 with 128 codes per stage.
bool use_mxf4(const MxGemmArgs &a) {
    return a.fa == MX_E2M1 && a.fb == MX_E2M1 && a.K % 256 == 0;
}

// The two-SM kernel: 256 x pbn tiles over CTA pairs (pbn 256 or 192; NVFP4
// operands 256 only).
int launch_gemm_pair(const MxGemmArgs &a, int pbn, cudaStream_t st) {
    using namespace mxg;
    const bool fp4 = a.nv || use_mxf4(a);
    const int64_t k_bytes = fp4 ? a.K / 2 : a.K;     // K bytes of a uint8 stage view
    // scale atoms one stage's boxes cover: per 128-byte K slice, times the
    // slices per stage (PairCfg::KS: two on 256-column tiles of MX operands
    // with MMA-layout scales); a box row is 256 bytes, two per atom, eight
    // per x4 atom
    const int G = (a.nv ? 4 : (fp4 ? 2 : 1)) * ((pbn == 256 && !a.nv && !a.x4) ? 2 : 1);
    const int box_atoms = a.x4 ? 4 * G : G;
    // scale atoms along K: four blocks each, of 32 elements (MX) or 16 (NVFP4)
    const int64_t k_groups = a.nv ? a.K / 64 : a.K / 128;
    CUtensorMap ta, tb, tsa, tsb, tc;
    if (!make_c_map(&tc, a)) return MX_ERR_CUDA;
    if (!make_operand_map(&ta, a.a_codes, a.M, a.K, a.fa, fp4, 128)) return MX_ERR_CUDA;
    if (!make_operand_map(&tb, a.b_codes, a.N, a.K, a.fb, fp4, pbn / 2)) return MX_ERR_CUDA;
    const int64_t sa_bytes = (a.M + 127) / 128 * 128 * k_groups * 4 * (a.x4 ? 4 : 1);
    const int64_t sb_bytes = (a.N + 127) / 128 * 128 * k_groups * 4 * (a.x4 ? 4 : 1);
    if (!make_scale_map(&tsa, a.a_scales, sa_bytes, box_atoms)) return MX_ERR_CUDA;
    if (!make_scale_map(&tsb, a.b_scales, sb_bytes, box_atoms)) return MX_ERR_CUDA;
    PairParams p;
    p.c = a.c;
    p.ldc = a.ldc;
    p.M = static_cast<int>(a.M);
    p.N = static_cast<int>(a.N);
    p.K = static_cast<int>(a.K);
    p.k_tiles = static_cast<int>(k_bytes / BK_BYTES);
    p.k_groups = static_cast<int>(k_groups);
    p.tiles_m = static_cast<int>((a.M + PAIR_BM - 1) / PAIR_BM);
    p.tiles_n = static_cast<int>((a.N + pbn - 1) / pbn);
    p.alpha = a.alpha;
    p.idesc = make_idesc(a.fa, a.fb, fp4, PAIR_BM, pbn, a.nv);
    p.ab_tx = stage_tx_bytes(a.fa, fp4, 128) + stage_tx_bytes(a.fb, fp4, pbn / 2);
    p.enc_a = a.enc_a;
    p.enc_b = a.enc_b;
    p.a_lines = static_cast<int>(a.a_lines);
    p.b_lines = static_cast<int>(a.b_lines);
    raster_for(a, p.tiles_m, p.tiles_n, p.raster_group, p.raster_n_major);
    p.skip_k_tile = g_skip_k_tile;
    g_skip_k_tile = -1;
    const int tiles = p.tiles_m * p.tiles_n;
    const int clusters = tiles < a.num_sms / 2 ? tiles : a.num_sms / 2;
    const int grid = 2 * (clusters < 1 ? 1 : clusters);
    cudaError_t e;
    p.q = mx_out(a);
    const int out = out_mode(a);
    if (a.x4 && a.nv) {
        if (pbn != 256 || out == OUT_MX) return MX_ERR_UNSUPPORTED;
        e = out == OUT_BF16 ? launch_pair<true, OUT_BF16, 256, true, true>(ta, tb, tsa, tsb, tc, p, grid, st)
                            : launch_pair<true, OUT_F32, 256, true, true>(ta, tb, tsa, tsb, tc, p, grid, st);
    } else if (a.x4) {
        if (pbn != 256) return MX_ERR_UNSUPPORTED;
        if (out == OUT_MX) e = fp4 ? launch_pair<true, OUT_MX, 256, false, true>(ta, tb, tsa, tsb, tc, p, grid, st)
                                   : launch_pair<false, OUT_MX, 256, false, true>(ta, tb, tsa, tsb, tc, p, grid, st);
        else if (out == OUT_BF16)
            e = fp4 ? launch_pair<true, OUT_BF16, 256, false, true>(ta, tb, tsa, tsb, tc, p, grid, st)
                    : launch_pair<false, OUT_BF16, 256, false, true>(ta, tb, tsa, tsb, tc, p, grid, st);
        else e = fp4 ? launch_pair<true, OUT_F32, 256, false, true>(ta, tb, tsa, tsb, tc, p, grid, st)
                     : launch_pair<false, OUT_F32, 256, false, true>(ta, tb, tsa, tsb, tc, p, grid, st);
    } else if (a.nv) {
        if (pbn != 256 || out == OUT_MX) return MX_ERR_UNSUPPORTED;
        e = out == OUT_BF16 ? launch_pair<true, OUT_BF16, 256, true>(ta, tb, tsa, tsb, tc, p, grid, st)
                            : launch_pair<true, OUT_F32, 256, true>(ta, tb, tsa, tsb, tc, p, grid, st);
    } else if (pbn == 256) e = fp4 ? launch_pair_out<true, 256>(out, ta, tb, tsa, tsb, tc, p, grid, st)
                            : launch_pair_out<false, 256>(out, ta, tb, tsa, tsb, tc, p, grid, st);
    else e = fp4 ? launch_pair_out<true, 192>(out, ta, tb, tsa, tsb, tc, p, grid, st)
                 : launch_pair_out<false, 192>(out, ta, tb, tsa, tsb, tc, p, grid, st);
    return e == cudaSuccess ? MX_OK : MX_ERR_CUDA;
}

}  // namespace

// Kernel choice.  CTA pairs on 256-row tiles have the higher steady-state
// rate (each MMA and scale copy covers two SMs, each SM loads half of B), but
// a shape with few such tiles or few K steps per tile is dominated by wave
// quantisation and per-tile start-up, where the one-SM kernel's smaller tiles
// and overlapped epilogue win (measured on the GPT-2-shaped GEMMs).
// Returns the pair tile width to use, or 0 for the one-SM kernel.
int pair_tile_n(const MxGemmArgs &a) {
    if (g_force_kernel >= 0) return g_force_kernel == 1 ? 0 : g_force_kernel;   // 1: the panel kernel
    if (a.M <= 128 || a.K < 2048) return 0;
    const int64_t pair_tiles = ((a.M + 255) / 256) * ((a.N + 255) / 256);
    return pair_tiles >= a.num_sms ? 256 : 0;
}

int mx_launch_gemm(const MxGemmArgs &a, cudaStream_t st) {
    using namespace mxg;
    if (a.nv) return launch_gemm_pair(a, 256, st);   // NVFP4 runs on the CTA-pair kernel only
    if (a.x4) {
        // x4 scales: the 256-column pair kernel only (any shape)
        if (g_force_kernel >= 0 && g_force_kernel != 256) return MX_ERR_UNSUPPORTED;
        return launch_gemm_pair(a, 256, st);
    }
    if (const int pbn = pair_tile_n(a); pbn != 0) return launch_gemm_pair(a, pbn, st);
    const bool fp4 = use_mxf4(a);
    const int64_t k_bytes = fp4 ? a.K / 2 : a.K;
    CUtensorMap ta, tb, tc;
    if (!make_c_map(&tc, a)) return MX_ERR_CUDA;
    if (!make_operand_map(&ta, a.a_codes, a.M, a.K, a.fa, fp4, BM)) return MX_ERR_CUDA;
    if (!make_operand_map(&tb, a.b_codes, a.N, a.K, a.fb, fp4, BN)) return MX_ERR_CUDA;
    Params p;
    p.a_scales = static_cast<const uint8_t *>(a.a_scales);
    p.b_scales = static_cast<const uint8_t *>(a.b_scales);
    p.c = a.c;
    p.ldc = a.ldc;
    p.M = static_cast<int>(a.M);
    p.N = static_cast<int>(a.N);
    p.K = static_cast<int>(a.K);
    p.k_tiles = static_cast<int>(k_bytes / BK_BYTES);
    p.k_groups = static_cast<int>(a.K / 128);
    p.tiles_m = static_cast<int>((a.M + BM - 1) / BM);
    p.tiles_n = static_cast<int>((a.N + BN - 1) / BN);
    p.alpha = a.alpha;
    p.idesc = make_idesc(a.fa, a.fb, fp4);
    p.ab_tx = stage_tx_bytes(a.fa, fp4, BM) + stage_tx_bytes(a.fb, fp4, BN);
    p.a_tx = stage_tx_bytes(a.fa, fp4, BM);
    raster_for(a, p.tiles_m, p.tiles_n, p.raster_group, p.raster_n_major);
    p.skip_k_tile = g_skip_k_tile;
    g_skip_k_tile = -1;
    const int tiles = p.tiles_m * p.tiles_n;
    const int grid = tiles < a.num_sms ? tiles : a.num_sms;
    cudaError_t e;
    p.q = mx_out(a);
    const int out = out_mode(a);
    // the resident-B kernel where a B panel's whole K fits in shared memory and
    // each panel serves several M tiles (or when forced)
    const bool panel = g_force_kernel == 1 ||
                       (g_force_kernel < 0 && p.k_tiles <= PANEL_MAX_SLICES && p.tiles_m >= 4);
    if (panel) {
        if (p.k_tiles > PANEL_MAX_SLICES) return MX_ERR_UNSUPPORTED;
        e = fp4 ? launch_panel_out<true>(out, ta, tb, tc, p, grid, st)
                : launch_panel_out<false>(out, ta, tb, tc, p, grid, st);
    } else {
        e = fp4 ? launch_out<true>(out, ta, tb, tc, p, grid, st) : launch_out<false>(out, ta, tb, tc, p, grid, st);
    }
    return e == cudaSuccess ? MX_OK : MX_ERR_CUDA;
}

int mx_read_device_status(cudaStream_t st) {
    if (cudaStreamSynchronize(st) != cudaSuccess) return MX_ERR_CUDA;
    int v = 0, b = 0;
    if (cudaMemcpyFromSymbol(&v, g_mx_status, sizeof(int)) != cudaSuccess) return MX_ERR_CUDA;
    if (cudaMemcpyFromSymbol(&b, mxk::g_bounds_status, sizeof(int)) != cudaSuccess) return MX_ERR_CUDA;
    const int zero = 0;
    if (cudaMemcpyToSymbol(g_mx_status, &zero, sizeof(int)) != cudaSuccess) return MX_ERR_CUDA;
    if (cudaMemcpyToSymbol(mxk::g_bounds_status, &zero, sizeof(int)) != cudaSuccess) return MX_ERR_CUDA;
    return v != MX_OK ? v : b;        // the debug build's bounds word after a timeout
}
