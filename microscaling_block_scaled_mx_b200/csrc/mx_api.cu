// mx_api.cu -- the C ABI of libmx (declared in include/mx.h): argument
// validation, status codes and launches on the caller's stream.  No entry
// point allocates device memory or synchronises, except
// mx_last_device_status, which synchronises the given stream by contract.
#include <cstdint>
#include <cstdlib>
#include <cstring>
#include <cuda_runtime.h>
#include <nvtx3/nvToolsExt.h>

#include "mx.h"
#include "mx_internal.h"

namespace {

// Optional NVTX ranges (environment MX_NVTX=1, read once per process): every
// entry point that launches work marks a range named after itself, so a
// profiler's timeline shows the library's calls.  Off by default; NVTX's
// header-only API costs nothing when no tool is attached.
bool nvtx_on() {
    static const bool on = [] {
        const char *e = std::getenv("MX_NVTX");
        return e != nullptr && e[0] == '1';
    }();
    return on;
}
struct NvtxRange {
    bool on;
    explicit NvtxRange(const char *name) : on(nvtx_on()) {
        if (on) nvtxRangePushA(name);
    }
    ~NvtxRange() {
        if (on) nvtxRangePop();
    }
};

constexpr int kMaxDevices = 64;
int g_sm_count[kMaxDevices];   // 0 = not queried yet

int sm_count(int *device_out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return -1;
    if (device_out) *device_out = dev;
    if (dev < 0 || dev >= kMaxDevices) return -1;
    if (g_sm_count[dev] == 0) {
        int n = 0;
        if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return -1;
        g_sm_count[dev] = n;
    }
    return g_sm_count[dev];
}

bool valid_layout(mx_scale_layout sl) {
    return sl == MX_SCALES_PLAIN || sl == MX_SCALES_MMA || sl == MX_SCALES_MMA_X4;
}

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
bool aligned32(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 31u) == 0; }

int elem_bits(int fmt) {
    switch (fmt) {
        case MX_E4M3: case MX_E5M2: case MX_INT8: return 8;
        case MX_E2M3: case MX_E3M2: return 6;
        case MX_E2M1: return 4;
        default: return 0;
    }
}

int dtype_bytes(int dt) { return dt == MX_F32 ? 4 : (dt == MX_BF16 ? 2 : 0); }

}  // namespace

extern "C" {

int mx_abi_version(void) { return 1; }

const char *mx_status_str(int status) {
    switch (status) {
        case MX_OK: return "MX_OK";
        case MX_ERR_ARG: return "MX_ERR_ARG: invalid argument (null pointer, bad enum or size)";
        case MX_ERR_ALIGN: return "MX_ERR_ALIGN: pointer or leading dimension not 16-byte aligned";
        case MX_ERR_SHAPE: return "MX_ERR_SHAPE: block-axis length is not a multiple of 32";
        case MX_ERR_UNSUPPORTED: return "MX_ERR_UNSUPPORTED: combination not implemented";
        case MX_ERR_SR_RANGE: return "MX_ERR_SR_RANGE: stochastic-rounding index space exceeds 2^34";
        case MX_ERR_CUDA: return "MX_ERR_CUDA: CUDA call or kernel launch failed";
        case MX_ERR_TIMEOUT: return "MX_ERR_TIMEOUT: a bounded device wait expired";
        case MX_ERR_BOUNDS: return "MX_ERR_BOUNDS: a debug-build bounds check skipped an access";
        default: return "unknown mx status";
    }
}

size_t mx_codes_bytes(mx_fmt fmt, int64_t outer, int64_t inner) {
    const int b = elem_bits(fmt);
    if (b == 0 || outer < 0 || inner < 0 || inner % 32 != 0) return 0;
    return static_cast<size_t>(outer) * static_cast<size_t>(inner / 32 * 4 * b);
}

size_t mx_scales_bytes(mx_scale_layout sl, int64_t outer, int64_t inner) {
    if (outer < 0 || inner < 0 || inner % 32 != 0) return 0;
    const int64_t kb = inner / 32;
    if (sl == MX_SCALES_PLAIN) return static_cast<size_t>(outer * kb);
    if (sl != MX_SCALES_MMA && sl != MX_SCALES_MMA_X4) return 0;
    return static_cast<size_t>((outer + 127) / 128 * 128) * static_cast<size_t>((kb + 3) / 4 * 4) *
           (sl == MX_SCALES_MMA_X4 ? 4u : 1u);
}

size_t mx_gemm_workspace_bytes(int64_t, int64_t, int64_t) { return 0; }

}  // extern "C"

namespace {

// Where a tensor sits in the whole tensor its stochastic-rounding positions
// refer to; NULL means the tensor is the whole.  Returns MX_OK or an error.
struct Placement {
    int64_t row0 = 0, col0 = 0, total_rows = 0, total_cols = 0;
};

int place(const mx_shard *shard, int64_t rows, int64_t cols, Placement &pl) {
    if (!shard) {
        pl.total_rows = rows;
        pl.total_cols = cols;
        return MX_OK;
    }
    pl.row0 = shard->row0;
    pl.col0 = shard->col0;
    pl.total_rows = shard->total_rows;
    pl.total_cols = shard->total_cols;
    if (pl.row0 < 0 || pl.col0 < 0 || pl.total_rows < 0 || pl.total_cols < 0) return MX_ERR_ARG;
    if (rows > pl.total_rows - pl.row0 || cols > pl.total_cols - pl.col0) return MX_ERR_ARG;
    return MX_OK;
}

// SR position of output element (o, i) = base + o * stride + i, for the output
// along `block_axis` of a tensor placed by pl.
void sr_position(const Placement &pl, int block_axis, uint64_t &base, uint64_t &stride) {
    if (block_axis == 1) {
        stride = static_cast<uint64_t>(pl.total_cols);
        base = static_cast<uint64_t>(pl.row0) * stride + static_cast<uint64_t>(pl.col0);
    } else {
        stride = static_cast<uint64_t>(pl.total_rows);
        base = static_cast<uint64_t>(pl.col0) * stride + static_cast<uint64_t>(pl.row0);
    }
}

int quantize_impl(const void *x, mx_dtype xdt, int64_t rows, int64_t cols, int64_t ldx, int block_axis,
                  mx_fmt fmt, mx_round rnd, uint64_t seed, const mx_precond *pre, const mx_shard *shard,
                  void *codes, void *scales, mx_scale_layout sl, void *stream) {
    if ((xdt != MX_F32 && xdt != MX_BF16) || elem_bits(fmt) == 0) return MX_ERR_ARG;
    if ((rnd != MX_RNE && rnd != MX_SR) || !valid_layout(sl)) return MX_ERR_ARG;
    if (block_axis != 0 && block_axis != 1) return MX_ERR_ARG;
    if (rows < 0 || cols < 0) return MX_ERR_ARG;
    Placement pl;
    if (int rc = place(shard, rows, cols, pl); rc != MX_OK) return rc;
    const int64_t outer = block_axis == 1 ? rows : cols;
    const int64_t inner = block_axis == 1 ? cols : rows;
    const int64_t inner_off = block_axis == 1 ? pl.col0 : pl.row0;
    const int64_t inner_total = block_axis == 1 ? pl.total_cols : pl.total_rows;
    if (inner % 32 != 0 || inner_off % 32 != 0 || inner_total % 32 != 0) return MX_ERR_SHAPE;
    if (outer == 0 || inner == 0) return MX_OK;          // empty: pointers may be NULL
    if (!x || !codes || !scales) return MX_ERR_ARG;
    if (ldx < cols) return MX_ERR_ARG;
    if (!aligned16(x) || (ldx * dtype_bytes(xdt)) % 16 != 0 || !aligned16(codes)) return MX_ERR_ALIGN;
    const bool had = pre && pre->hadamard;
    if (had && block_axis != 0) return MX_ERR_UNSUPPORTED;
    if (rnd == MX_SR &&
        static_cast<uint64_t>(pl.total_rows) * static_cast<uint64_t>(pl.total_cols) > (1ull << 34))
        return MX_ERR_SR_RANGE;
    if (mx_scales_bytes(sl, outer, inner) >= (1ull << 32)) return MX_ERR_UNSUPPORTED;  // 32-bit scale offsets

    MxQuantizeArgs a;
    a.x = x; a.xdt = xdt; a.rows = rows; a.cols = cols; a.ldx = ldx;
    a.block_axis = block_axis; a.fmt = fmt; a.rnd = rnd; a.seed = seed;
    a.hadamard = had; a.sign_mask = had ? pre->sign_mask : 0u;
    a.codes = codes; a.scales = scales; a.sl = sl;
    sr_position(pl, block_axis, a.sr_base, a.sr_stride);
    a.num_sms = sm_count(nullptr);
    if (a.num_sms <= 0) return MX_ERR_CUDA;
    return mx_launch_quantize(a, static_cast<cudaStream_t>(stream)) == cudaSuccess ? MX_OK : MX_ERR_CUDA;
}

int quantize_dual_impl(const void *x, mx_dtype xdt, int64_t rows, int64_t cols, int64_t ldx, mx_fmt fmt,
                       mx_round rnd_rows, uint64_t seed_rows, mx_round rnd_cols, uint64_t seed_cols,
                       const mx_precond *pre_cols, const mx_shard *shard, void *codes_rows, void *scales_rows,
                       void *codes_cols, void *scales_cols, mx_scale_layout sl, void *stream) {
    if ((xdt != MX_F32 && xdt != MX_BF16) || elem_bits(fmt) == 0) return MX_ERR_ARG;
    if ((rnd_rows != MX_RNE && rnd_rows != MX_SR) || (rnd_cols != MX_RNE && rnd_cols != MX_SR)) return MX_ERR_ARG;
    if (!valid_layout(sl)) return MX_ERR_ARG;
    if (rows < 0 || cols < 0) return MX_ERR_ARG;
    Placement pl;
    if (int rc = place(shard, rows, cols, pl); rc != MX_OK) return rc;
    if (rows % 32 != 0 || cols % 32 != 0) return MX_ERR_SHAPE;
    if (pl.row0 % 32 != 0 || pl.col0 % 32 != 0 || pl.total_rows % 32 != 0 || pl.total_cols % 32 != 0)
        return MX_ERR_SHAPE;
    if (rows == 0 || cols == 0) return MX_OK;            // empty: pointers may be NULL
    if (!x || !codes_rows || !scales_rows || !codes_cols || !scales_cols) return MX_ERR_ARG;
    if (ldx < cols) return MX_ERR_ARG;
    if (!aligned16(x) || (ldx * dtype_bytes(xdt)) % 16 != 0 || !aligned16(codes_rows) || !aligned16(codes_cols))
        return MX_ERR_ALIGN;
    if ((rnd_rows == MX_SR || rnd_cols == MX_SR) &&
        static_cast<uint64_t>(pl.total_rows) * static_cast<uint64_t>(pl.total_cols) > (1ull << 34))
        return MX_ERR_SR_RANGE;
    if (mx_scales_bytes(sl, rows, cols) >= (1ull << 32) || mx_scales_bytes(sl, cols, rows) >= (1ull << 32))
        return MX_ERR_UNSUPPORTED;
    const bool had = pre_cols && pre_cols->hadamard;
    MxQuantizeDualArgs a;
    a.x = x; a.xdt = xdt; a.rows = rows; a.cols = cols; a.ldx = ldx; a.fmt = fmt;
    a.rnd_rows = rnd_rows; a.rnd_cols = rnd_cols; a.seed_rows = seed_rows; a.seed_cols = seed_cols;
    a.hadamard = had; a.sign_mask = had ? pre_cols->sign_mask : 0u;
    a.codes_rows = codes_rows; a.scales_rows = scales_rows; a.codes_cols = codes_cols; a.scales_cols = scales_cols;
    a.sl = sl;
    sr_position(pl, 1, a.sr_base_rows, a.sr_stride_rows);
    sr_position(pl, 0, a.sr_base_cols, a.sr_stride_cols);
    a.num_sms = sm_count(nullptr);
    if (a.num_sms <= 0) return MX_ERR_CUDA;
    return mx_launch_quantize_dual(a, static_cast<cudaStream_t>(stream)) == cudaSuccess ? MX_OK : MX_ERR_CUDA;
}

}  // namespace

extern "C" {

int mx_quantize(const void *x, mx_dtype xdt, int64_t rows, int64_t cols, int64_t ldx,
                int block_axis, mx_fmt fmt, mx_round rnd, uint64_t seed,
                const mx_precond *pre, void *codes, void *scales, mx_scale_layout sl,
                void *stream) {
    const NvtxRange nvtx_range("mx_quantize");
    return quantize_impl(x, xdt, rows, cols, ldx, block_axis, fmt, rnd, seed, pre, nullptr, codes, scales, sl,
                         stream);
}

int mx_quantize_shard(const void *x, mx_dtype xdt, int64_t rows, int64_t cols, int64_t ldx,
                      int block_axis, mx_fmt fmt, mx_round rnd, uint64_t seed,
                      const mx_precond *pre, const mx_shard *shard, void *codes, void *scales,
                      mx_scale_layout sl, void *stream) {
    const NvtxRange nvtx_range("mx_quantize_shard");
    if (!shard) return MX_ERR_ARG;
    return quantize_impl(x, xdt, rows, cols, ldx, block_axis, fmt, rnd, seed, pre, shard, codes, scales, sl,
                         stream);
}

int mx_quantize_dual(const void *x, mx_dtype xdt, int64_t rows, int64_t cols, int64_t ldx, mx_fmt fmt,
                     mx_round rnd_rows, uint64_t seed_rows, mx_round rnd_cols, uint64_t seed_cols,
                     const mx_precond *pre_cols, void *codes_rows, void *scales_rows, void *codes_cols,
                     void *scales_cols, mx_scale_layout sl, void *stream) {
    const NvtxRange nvtx_range("mx_quantize_dual");
    return quantize_dual_impl(x, xdt, rows, cols, ldx, fmt, rnd_rows, seed_rows, rnd_cols, seed_cols, pre_cols,
                              nullptr, codes_rows, scales_rows, codes_cols, scales_cols, sl, stream);
}

int mx_quantize_dual_shard(const void *x, mx_dtype xdt, int64_t rows, int64_t cols, int64_t ldx, mx_fmt fmt,
                           mx_round rnd_rows, uint64_t seed_rows, mx_round rnd_cols, uint64_t seed_cols,
                           const mx_precond *pre_cols, const mx_shard *shard, void *codes_rows,
                           void *scales_rows, void *codes_cols, void *scales_cols, mx_scale_layout sl,
                           void *stream) {
    const NvtxRange nvtx_range("mx_quantize_dual_shard");
    if (!shard) return MX_ERR_ARG;
    return quantize_dual_impl(x, xdt, rows, cols, ldx, fmt, rnd_rows, seed_rows, rnd_cols, seed_cols, pre_cols,
                              shard, codes_rows, scales_rows, codes_cols, scales_cols, sl, stream);
}

size_t mx_nvfp4_scales_bytes(mx_scale_layout sl, int64_t rows, int64_t cols) {
    if (rows < 0 || cols < 0 || cols % 16 != 0) return 0;
    return mx_scales_bytes(sl, rows, 2 * cols);       // one byte per 16-block, the same atoms
}

int64_t mx_nvfp4_domains(int64_t rows, int64_t domain_rows) {
    if (rows < 0 || domain_rows < 0) return 0;
    if (domain_rows == 0) return 1;
    return (rows + domain_rows - 1) / domain_rows;
}

int mx_quantize_nvfp4(const void *x, mx_dtype xdt, int64_t rows, int64_t cols, int64_t ldx, int64_t domain_rows,
                      void *codes, void *scales, mx_scale_layout sl, float *enc_scales, void *stream) {
    const NvtxRange nvtx_range("mx_quantize_nvfp4");
    if (xdt != MX_F32 && xdt != MX_BF16) return MX_ERR_ARG;
    if (!valid_layout(sl)) return MX_ERR_ARG;
    if (rows < 0 || cols < 0 || domain_rows < 0) return MX_ERR_ARG;
    if (cols % 16 != 0) return MX_ERR_SHAPE;
    if (rows == 0 || cols == 0) return MX_OK;             // empty: pointers may be NULL
    if (!x || !codes || !scales || !enc_scales || ldx < cols) return MX_ERR_ARG;
    if (!aligned16(x) || (ldx * dtype_bytes(xdt)) % 16 != 0 || !aligned16(codes) ||
        (reinterpret_cast<uintptr_t>(enc_scales) & 3u) != 0)
        return MX_ERR_ALIGN;
    if (mx_nvfp4_scales_bytes(sl, rows, cols) >= (1ull << 32)) return MX_ERR_UNSUPPORTED;
    MxNvfp4Args a;
    a.x = x; a.xdt = xdt; a.rows = rows; a.cols = cols; a.ldx = ldx; a.domain_rows = domain_rows;
    a.codes = codes; a.scales = scales; a.sl = sl; a.enc_scales = enc_scales;
    a.num_sms = sm_count(nullptr);
    if (a.num_sms <= 0) return MX_ERR_CUDA;
    return mx_launch_quantize_nvfp4(a, static_cast<cudaStream_t>(stream)) == cudaSuccess ? MX_OK : MX_ERR_CUDA;
}

int mx_dequantize(const void *codes, const void *scales, mx_fmt fmt, mx_scale_layout sl,
                  int64_t outer, int64_t inner, void *y, mx_dtype ydt, int64_t ldy, void *stream) {
    const NvtxRange nvtx_range("mx_dequantize");
    if (elem_bits(fmt) == 0 || (ydt != MX_F32 && ydt != MX_BF16)) return MX_ERR_ARG;
    if (!valid_layout(sl)) return MX_ERR_ARG;
    if (outer < 0 || inner < 0) return MX_ERR_ARG;
    if (inner % 32 != 0) return MX_ERR_SHAPE;
    if (outer == 0 || inner == 0) return MX_OK;          // empty: pointers may be NULL
    if (!codes || !scales || !y || ldy < inner) return MX_ERR_ARG;
    if (!aligned16(codes) || !aligned16(y) || (ldy * dtype_bytes(ydt)) % 16 != 0) return MX_ERR_ALIGN;
    MxDequantArgs a;
    a.codes = codes; a.scales = scales; a.fmt = fmt; a.sl = sl;
    a.outer = outer; a.inner = inner; a.y = y; a.ydt = ydt; a.ldy = ldy;
    a.num_sms = sm_count(nullptr);
    if (a.num_sms <= 0) return MX_ERR_CUDA;
    return mx_launch_dequantize(a, static_cast<cudaStream_t>(stream)) == cudaSuccess ? MX_OK : MX_ERR_CUDA;
}

}  // extern "C"

namespace {

// Checks shared by mx_gemm and mx_gemm_quantize on the operands; MX_OK to go on.
int check_gemm_operands(const void *a_codes, const void *a_scales, mx_fmt fa, const void *b_codes,
                        const void *b_scales, mx_fmt fb, int64_t K) {
    if (K > 0 && (!a_codes || !a_scales || !b_codes || !b_scales)) return MX_ERR_ARG;
    if (fa == MX_INT8 || fb == MX_INT8) return MX_ERR_UNSUPPORTED;   // no block-scaled INT8 MMA
    if (K % 128 != 0) return MX_ERR_UNSUPPORTED;
    if (!aligned16(a_codes) || !aligned16(b_codes) || !aligned16(a_scales) || !aligned16(b_scales))
        return MX_ERR_ALIGN;
    // FP6 codes, and FP4 codes outside the E2M1 x E2M1 (K % 256 == 0) case, are
    // read through packed tensor maps, which need 32-byte aligned bases
    const bool mxf4 = fa == MX_E2M1 && fb == MX_E2M1 && K % 256 == 0;
    if (!mxf4 && ((elem_bits(fa) < 8 && !aligned32(a_codes)) || (elem_bits(fb) < 8 && !aligned32(b_codes))))
        return MX_ERR_ALIGN;
    return MX_OK;
}

// The GEMM kernels index rows, columns, K and tiles with 32-bit integers.
bool gemm_dims_fit(int64_t M, int64_t N, int64_t K) {
    constexpr int64_t kMax = 2147483647;
    if (M > kMax || N > kMax || K > kMax) return false;
    return ((M + 127) / 128) * ((N + 127) / 128) <= kMax;
}

MxGemmArgs gemm_args(const void *a_codes, const void *a_scales, mx_fmt fa, const void *b_codes,
                     const void *b_scales, mx_fmt fb, int64_t M, int64_t N, int64_t K, float alpha) {
    MxGemmArgs a;
    a.a_codes = a_codes; a.a_scales = a_scales; a.b_codes = b_codes; a.b_scales = b_scales;
    a.fa = fa; a.fb = fb; a.M = M; a.N = N; a.K = K; a.alpha = alpha;
    a.c = nullptr; a.cdt = MX_F32; a.ldc = 0;
    a.q_codes = nullptr; a.q_scales = nullptr; a.q_fmt = 0; a.q_rnd = MX_RNE; a.q_sl = MX_SCALES_MMA; a.q_seed = 0;
    a.nv = false; a.x4 = false; a.enc_a = nullptr; a.enc_b = nullptr; a.a_lines = 0; a.b_lines = 0;
    a.num_sms = 0; a.device = 0;
    return a;
}

int gemm_impl(const void *a_codes, const void *a_scales, mx_fmt fa, const void *b_codes, const void *b_scales,
              mx_fmt fb, int64_t M, int64_t N, int64_t K, float alpha, void *c, mx_dtype cdt, int64_t ldc,
              bool x4, void *stream) {
    if (elem_bits(fa) == 0 || elem_bits(fb) == 0 || (cdt != MX_F32 && cdt != MX_BF16)) return MX_ERR_ARG;
    if (M < 0 || N < 0 || K < 0) return MX_ERR_ARG;
    if (!gemm_dims_fit(M, N, K)) return MX_ERR_UNSUPPORTED;
    if (K % 32 != 0) return MX_ERR_SHAPE;
    if (M == 0 || N == 0) return MX_OK;                  // empty: pointers may be NULL
    if (!c || ldc < N) return MX_ERR_ARG;
    const int rc = check_gemm_operands(a_codes, a_scales, fa, b_codes, b_scales, fb, K);
    if (rc != MX_OK) return rc;
    if (!aligned16(c) || (ldc * dtype_bytes(cdt)) % 16 != 0) return MX_ERR_ALIGN;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (K == 0) {
        const size_t esz = static_cast<size_t>(dtype_bytes(cdt));
        return cudaMemset2DAsync(c, ldc * esz, 0, N * esz, M, st) == cudaSuccess ? MX_OK : MX_ERR_CUDA;
    }
    MxGemmArgs a = gemm_args(a_codes, a_scales, fa, b_codes, b_scales, fb, M, N, K, alpha);
    a.c = c; a.cdt = cdt; a.ldc = ldc; a.x4 = x4;
    a.num_sms = sm_count(&a.device);
    if (a.num_sms <= 0) return MX_ERR_CUDA;
    return mx_launch_gemm(a, st);
}

int gemm_quantize_impl(const void *a_codes, const void *a_scales, mx_fmt fa, const void *b_codes,
                       const void *b_scales, mx_fmt fb, int64_t M, int64_t N, int64_t K, float alpha,
                       mx_fmt out_fmt, mx_round out_rnd, uint64_t out_seed, void *out_codes, void *out_scales,
                       mx_scale_layout out_sl, bool x4, void *stream) {
    if (elem_bits(fa) == 0 || elem_bits(fb) == 0 || elem_bits(out_fmt) == 0) return MX_ERR_ARG;
    if ((out_rnd != MX_RNE && out_rnd != MX_SR) || !valid_layout(out_sl))
        return MX_ERR_ARG;
    if (M < 0 || N < 0 || K < 0) return MX_ERR_ARG;
    if (!gemm_dims_fit(M, N, K)) return MX_ERR_UNSUPPORTED;
    if (K % 32 != 0 || N % 32 != 0) return MX_ERR_SHAPE;  // C's blocks run along N
    if (M == 0 || N == 0) return MX_OK;                   // empty: pointers may be NULL
    if (!out_codes || !out_scales) return MX_ERR_ARG;
    const int rc = check_gemm_operands(a_codes, a_scales, fa, b_codes, b_scales, fb, K);
    if (rc != MX_OK) return rc;
    if (!aligned16(out_codes)) return MX_ERR_ALIGN;
    if (out_rnd == MX_SR && static_cast<uint64_t>(M) * static_cast<uint64_t>(N) > (1ull << 34))
        return MX_ERR_SR_RANGE;
    const size_t sbytes = mx_scales_bytes(out_sl, M, N);
    if (sbytes >= (1ull << 32)) return MX_ERR_UNSUPPORTED;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (K == 0) {
        // C = 0: every block is all zero (code 0, scale code 0)
        if (cudaMemsetAsync(out_codes, 0, mx_codes_bytes(out_fmt, M, N), st) != cudaSuccess) return MX_ERR_CUDA;
        return cudaMemsetAsync(out_scales, 0, sbytes, st) == cudaSuccess ? MX_OK : MX_ERR_CUDA;
    }
    MxGemmArgs a = gemm_args(a_codes, a_scales, fa, b_codes, b_scales, fb, M, N, K, alpha);
    a.q_codes = out_codes; a.q_scales = out_scales; a.q_fmt = out_fmt; a.q_rnd = out_rnd; a.q_sl = out_sl;
    a.q_seed = out_seed; a.x4 = x4;
    a.num_sms = sm_count(&a.device);
    if (a.num_sms <= 0) return MX_ERR_CUDA;
    return mx_launch_gemm(a, st);
}

}  // namespace

extern "C" {

int mx_gemm(const void *a_codes, const void *a_scales, mx_fmt fa,
            const void *b_codes, const void *b_scales, mx_fmt fb,
            int64_t M, int64_t N, int64_t K, float alpha,
            void *c, mx_dtype cdt, int64_t ldc, void *workspace, size_t ws_bytes, void *stream) {
    const NvtxRange nvtx_range("mx_gemm");
    (void)workspace;
    (void)ws_bytes;
    return gemm_impl(a_codes, a_scales, fa, b_codes, b_scales, fb, M, N, K, alpha, c, cdt, ldc, false, stream);
}

int mx_gemm_x4(const void *a_codes, const void *a_scales, mx_fmt fa,
               const void *b_codes, const void *b_scales, mx_fmt fb,
               int64_t M, int64_t N, int64_t K, float alpha,
               void *c, mx_dtype cdt, int64_t ldc, void *stream) {
    const NvtxRange nvtx_range("mx_gemm_x4");
    return gemm_impl(a_codes, a_scales, fa, b_codes, b_scales, fb, M, N, K, alpha, c, cdt, ldc, true, stream);
}

int mx_gemm_quantize(const void *a_codes, const void *a_scales, mx_fmt fa,
                     const void *b_codes, const void *b_scales, mx_fmt fb,
                     int64_t M, int64_t N, int64_t K, float alpha,
                     mx_fmt out_fmt, mx_round out_rnd, uint64_t out_seed,
                     void *out_codes, void *out_scales, mx_scale_layout out_sl, void *stream) {
    const NvtxRange nvtx_range("mx_gemm_quantize");
    return gemm_quantize_impl(a_codes, a_scales, fa, b_codes, b_scales, fb, M, N, K, alpha, out_fmt, out_rnd,
                              out_seed, out_codes, out_scales, out_sl, false, stream);
}

int mx_gemm_quantize_x4(const void *a_codes, const void *a_scales, mx_fmt fa,
                        const void *b_codes, const void *b_scales, mx_fmt fb,
                        int64_t M, int64_t N, int64_t K, float alpha,
                        mx_fmt out_fmt, mx_round out_rnd, uint64_t out_seed,
                        void *out_codes, void *out_scales, mx_scale_layout out_sl, void *stream) {
    const NvtxRange nvtx_range("mx_gemm_quantize_x4");
    return gemm_quantize_impl(a_codes, a_scales, fa, b_codes, b_scales, fb, M, N, K, alpha, out_fmt, out_rnd,
                              out_seed, out_codes, out_scales, out_sl, true, stream);
}

}  // extern "C"

namespace {

int gemm_nvfp4_impl(const void *a_codes, const void *a_scales, const float *a_enc, int64_t a_domain_rows,
                    const void *b_codes, const void *b_scales, const float *b_enc, int64_t b_domain_rows,
                    int64_t M, int64_t N, int64_t K, float alpha, void *c, mx_dtype cdt, int64_t ldc, bool x4,
                    void *stream) {
    if (cdt != MX_F32 && cdt != MX_BF16) return MX_ERR_ARG;
    if (M < 0 || N < 0 || K < 0 || a_domain_rows < 0 || b_domain_rows < 0) return MX_ERR_ARG;
    if (!gemm_dims_fit(M, N, K)) return MX_ERR_UNSUPPORTED;
    if (K % 16 != 0) return MX_ERR_SHAPE;
    if (K % 256 != 0 || b_domain_rows % 32 != 0) return MX_ERR_UNSUPPORTED;
    if (M == 0 || N == 0) return MX_OK;                  // empty: pointers may be NULL
    if (!c || ldc < N) return MX_ERR_ARG;
    if (!aligned16(c) || (ldc * dtype_bytes(cdt)) % 16 != 0) return MX_ERR_ALIGN;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (K == 0) {
        const size_t esz = static_cast<size_t>(dtype_bytes(cdt));
        return cudaMemset2DAsync(c, ldc * esz, 0, N * esz, M, st) == cudaSuccess ? MX_OK : MX_ERR_CUDA;
    }
    if (!a_codes || !a_scales || !a_enc || !b_codes || !b_scales || !b_enc) return MX_ERR_ARG;
    if (!aligned16(a_codes) || !aligned16(b_codes) || !aligned16(a_scales) || !aligned16(b_scales) ||
        (reinterpret_cast<uintptr_t>(a_enc) & 3u) != 0 || (reinterpret_cast<uintptr_t>(b_enc) & 3u) != 0)
        return MX_ERR_ALIGN;
    MxGemmArgs a = gemm_args(a_codes, a_scales, MX_E2M1, b_codes, b_scales, MX_E2M1, M, N, K, alpha);
    a.c = c; a.cdt = cdt; a.ldc = ldc;
    a.nv = true; a.x4 = x4; a.enc_a = a_enc; a.enc_b = b_enc;
    a.a_lines = a_domain_rows >= M ? 0 : a_domain_rows;   // a domain covering every row: one domain
    a.b_lines = b_domain_rows >= N ? 0 : b_domain_rows;
    a.num_sms = sm_count(&a.device);
    if (a.num_sms <= 0) return MX_ERR_CUDA;
    return mx_launch_gemm(a, st);
}

}  // namespace

extern "C" {

int mx_gemm_nvfp4(const void *a_codes, const void *a_scales, const float *a_enc, int64_t a_domain_rows,
                  const void *b_codes, const void *b_scales, const float *b_enc, int64_t b_domain_rows,
                  int64_t M, int64_t N, int64_t K, float alpha, void *c, mx_dtype cdt, int64_t ldc,
                  void *stream) {
    const NvtxRange nvtx_range("mx_gemm_nvfp4");
    return gemm_nvfp4_impl(a_codes, a_scales, a_enc, a_domain_rows, b_codes, b_scales, b_enc, b_domain_rows, M, N,
                           K, alpha, c, cdt, ldc, false, stream);
}

int mx_gemm_nvfp4_x4(const void *a_codes, const void *a_scales, const float *a_enc, int64_t a_domain_rows,
                     const void *b_codes, const void *b_scales, const float *b_enc, int64_t b_domain_rows,
                     int64_t M, int64_t N, int64_t K, float alpha, void *c, mx_dtype cdt, int64_t ldc,
                     void *stream) {
    const NvtxRange nvtx_range("mx_gemm_nvfp4_x4");
    return gemm_nvfp4_impl(a_codes, a_scales, a_enc, a_domain_rows, b_codes, b_scales, b_enc, b_domain_rows, M, N,
                           K, alpha, c, cdt, ldc, true, stream);
}

int mx_last_device_status(void *stream) {
    // the GEMMs', the casts' and the NVFP4 unit's status words, all read and
    // cleared; a timeout takes precedence over a debug-build bounds report
    const int g = mx_read_device_status(static_cast<cudaStream_t>(stream));
    const int c = mx_read_cast_status();
    const int n = mx_read_nvfp4_bounds_status();
    if (g == MX_ERR_TIMEOUT || c == MX_ERR_TIMEOUT) return MX_ERR_TIMEOUT;
    return g != MX_OK ? g : (c != MX_OK ? c : n);
}

}  // extern "C"
