/*
 * mx_oracle.c -- plain, slow, obviously-correct CPU oracle for the MX cast
 * (scalar float -> MX block) and the block-scaled GEMM.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path may link, load or
 * call this file: only the tests, the smoke check and the CPU-baseline leg of
 * the benchmark use it.  It shares no code, header, table or constant
 * generator with the CUDA library; it includes nothing from include/ or from
 * the package.
 *
 * Sources (page title, section):
 *  - "Microscaling Data Formats for Deep Learning" (AI summary page), section 2
 *    "Microscaling": an MX block is k values sharing one scale X with k scalar
 *    elements P_i; v_i = X * P_i; a NaN scale makes the whole block NaN; the
 *    scale is E8M0; storage layout is up to the implementation.
 *  - same page, section 3 "Scalar Float to MX Format Conversion" (Algorithm 1):
 *    the shared exponent maps the largest input exponent onto the element
 *    format's largest binade; P_i = quantize(V_i / X) with overflowing normals
 *    clamped; FP32 subnormal inputs give P_i = 0; the block axis is a choice
 *    because conversion and transposition do not commute.
 *  - same page, section 4 "Experimental Results", compute flow: dot products
 *    take MX inputs and return scalar floats.
 *  - "Format-Aware Fusion for Fast FP4 Pretraining", abstract: MXFP4 with
 *    row-gradient stochastic rounding and fixed-sign 32-value Hadamard
 *    weight-gradient preconditioning.
 *
 * The pages print no bit layouts.  Element formats are decoded here from their
 * definition (sign bit, exponent field, mantissa field, bias), which is the
 * OCP MX v1.0 definition the summary page refers to.  Readings taken where the
 * pages are silent (all-zero block scale, signed zero, INT8 -128, the
 * stochastic-rounding width and hash, the Hadamard normalisation and sign mask)
 * are marked "reading:" below.  Parity unpinned: nothing outside the oracle
 * fixes which of those readings the pages' authors used, so the functions
 * that apply them are pinned only on their arithmetic (round-up counts,
 * published hash vectors, the Sylvester matrix product), not on the choice.
 *
 * Build: gcc -O2 -std=c11 -fopenmp -ffp-contract=off -fPIC -shared.
 * No fast-math, no FMA contraction: every float operation is a single IEEE
 * operation in the stated precision.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define MXO_OK 0
#define MXO_ERR_ARG (-1)
#define MXO_ERR_SHAPE (-3)
#define MXO_ERR_SR_RANGE (-5)

enum { FMT_E4M3 = 0, FMT_E5M2 = 1, FMT_E2M3 = 2, FMT_E3M2 = 3, FMT_E2M1 = 4,
       FMT_INT8 = 5, FMT_COUNT = 6 };
enum { DT_F32 = 0, DT_BF16 = 1 };
enum { RND_RNE = 0, RND_SR = 1 };
enum { SL_PLAIN = 0, SL_MMA = 1, SL_MMA_X4 = 2 };

#define BLOCK 32

/* ------------------------------------------------------------------------ */
/* Element formats, from their definition.                                  */
/* ------------------------------------------------------------------------ */

typedef struct {
    int bits;   /* code width in bits                                  */
    int ebits;  /* exponent field width (0 for the integer format)     */
    int mbits;  /* mantissa field width                                */
    int bias;   /* exponent bias                                       */
} fmt_def;

static const fmt_def FMTS[FMT_COUNT] = {
    {8, 4, 3, 7},   /* E4M3 */
    {8, 5, 2, 15},  /* E5M2 */
    {6, 2, 3, 1},   /* E2M3 */
    {6, 3, 2, 3},   /* E3M2 */
    {4, 2, 1, 1},   /* E2M1 */
    {8, 0, 0, 0},   /* INT8: two's complement, value = code * 2^-6 */
};

/* Decode one element code to its exact value (double holds every one). */
double mxref_decode_elem(int fmt, unsigned code)
{
    const fmt_def *f = &FMTS[fmt];
    if (fmt == FMT_INT8) {
        int8_t s = (int8_t)(uint8_t)code;
        return ldexp((double)s, -6);
    }
    unsigned sign = (code >> (f->bits - 1)) & 1u;
    unsigned efield = (code >> f->mbits) & ((1u << f->ebits) - 1u);
    unsigned mfield = code & ((1u << f->mbits) - 1u);
    double mag;
    if (fmt == FMT_E5M2 && efield == 31u) {
        /* E5M2 keeps IEEE specials: all-ones exponent is Inf (mantissa 0) or NaN */
        mag = (mfield == 0u) ? INFINITY : NAN;
    } else if (fmt == FMT_E4M3 && efield == 15u && mfield == 7u) {
        mag = NAN;  /* E4M3: only S.1111.111 is NaN, there is no Inf */
    } else if (efield == 0u) {
        /* subnormal: 0.m * 2^(1 - bias) */
        mag = ldexp((double)mfield, 1 - f->bias - f->mbits);
    } else {
        /* normal: 1.m * 2^(e - bias) */
        mag = ldexp((double)((1u << f->mbits) | mfield), (int)efield - f->bias - f->mbits);
    }
    return sign ? -mag : mag;
}

/* Sorted table of the non-negative finite magnitudes and their codes. */
typedef struct {
    int n;
    double mag[128];
    unsigned code[128];
    double maxv;
    int emax;      /* exponent of the largest binade: floor(log2(max)) */
} fmt_table;

static fmt_table TABLES[FMT_COUNT];
static int tables_ready = 0;

static void build_tables(void)
{
    if (tables_ready) return;
    for (int fmt = 0; fmt < FMT_COUNT; ++fmt) {
        fmt_table *t = &TABLES[fmt];
        t->n = 0;
        if (fmt == FMT_INT8) {
            /* reading: symmetric clamp to +-127; code -128 (= -2) is decoded but never produced */
            for (unsigned c = 0; c <= 127u; ++c) {
                t->mag[t->n] = mxref_decode_elem(fmt, c);
                t->code[t->n] = c;
                t->n++;
            }
        } else {
            unsigned ncodes = 1u << (FMTS[fmt].bits - 1);   /* sign bit clear */
            for (unsigned c = 0; c < ncodes; ++c) {
                double v = mxref_decode_elem(fmt, c);
                if (!isfinite(v)) continue;
                t->mag[t->n] = v;
                t->code[t->n] = c;
                t->n++;
            }
        }
        /* the positive codes decode in increasing order; keep it checked */
        for (int i = 1; i < t->n; ++i)
            if (!(t->mag[i] > t->mag[i - 1])) abort();
        t->maxv = t->mag[t->n - 1];
        int ex;
        frexp(t->maxv, &ex);     /* maxv = f * 2^ex, f in [0.5, 1) */
        t->emax = ex - 1;
    }
    tables_ready = 1;
}

int mxref_emax(int fmt) { build_tables(); return TABLES[fmt].emax; }
double mxref_max(int fmt) { build_tables(); return TABLES[fmt].maxv; }

static unsigned sign_code(int fmt, unsigned code, int neg)
{
    if (!neg) return code;
    if (fmt == FMT_INT8) return (unsigned)(uint8_t)(-(int)code);
    return code | (1u << (FMTS[fmt].bits - 1));
}

/* index of the largest table magnitude <= mag (mag finite, >= 0, < max) */
static int floor_index(const fmt_table *t, double mag)
{
    int lo = 0, hi = t->n - 1;     /* invariant: mag[lo] <= mag < mag[hi] */
    while (hi - lo > 1) {
        int mid = (lo + hi) / 2;
        if (t->mag[mid] <= mag) lo = mid; else hi = mid;
    }
    return lo;
}

/* Round-to-nearest-even onto the element grid, clamping overflow to +-max
 * (section 3: overflowing normals are clamped).  u must be finite. */
unsigned mxref_encode_rne(int fmt, double u)
{
    build_tables();
    const fmt_table *t = &TABLES[fmt];
    int neg = signbit(u) != 0;
    double mag = fabs(u);
    int idx;
    if (mag >= t->maxv) {
        idx = t->n - 1;
    } else {
        int i = floor_index(t, mag);
        /* both differences are exact: neighbouring grid points are within a
         * factor of two of each other (Sterbenz), or the lower one is zero */
        double dlo = mag - t->mag[i];
        double dhi = t->mag[i + 1] - mag;
        if (dlo < dhi) idx = i;
        else if (dhi < dlo) idx = i + 1;
        else idx = (t->code[i] & 1u) ? i + 1 : i;   /* tie: even mantissa LSB */
    }
    /* reading: FP formats keep the sign of zero; INT8 has a single zero */
    return sign_code(fmt, t->code[idx], neg);
}

/* Stochastic rounding with an 8-bit random byte r (reading: the pages give no
 * width).  With lo <= |u| < hi adjacent grid points, F = floor(256*(|u|-lo)/(hi-lo))
 * and the magnitude rounds up iff F + r >= 256; |u| >= max gives max. */
unsigned mxref_encode_sr(int fmt, double u, unsigned r)
{
    build_tables();
    const fmt_table *t = &TABLES[fmt];
    int neg = signbit(u) != 0;
    double mag = fabs(u);
    int idx;
    if (mag >= t->maxv) {
        idx = t->n - 1;
    } else {
        int i = floor_index(t, mag);
        double frac = (mag - t->mag[i]) / (t->mag[i + 1] - t->mag[i]);
        unsigned F = (unsigned)floor(frac * 256.0);
        idx = (F + (r & 255u) >= 256u) ? i + 1 : i;
    }
    return sign_code(fmt, t->code[idx], neg);
}

/* ------------------------------------------------------------------------ */
/* Counter-based random bytes for stochastic rounding (reading).            */
/* fmix32 is the public-domain MurmurHash3 32-bit finaliser (A. Appleby).   */
/* ------------------------------------------------------------------------ */

uint32_t mxref_fmix32(uint32_t h)
{
    h ^= h >> 16;
    h *= 0x85ebca6bu;
    h ^= h >> 13;
    h *= 0xc2b2ae35u;
    h ^= h >> 16;
    return h;
}

static uint32_t seed_key(uint64_t seed)
{
    return mxref_fmix32((uint32_t)(seed & 0xffffffffu)) ^ (uint32_t)(seed >> 32);
}

/* random byte for the element with linear index idx in block-axis-major
 * output coordinates: byte (idx mod 4) of fmix32(floor(idx/4) xor key) */
unsigned mxref_sr_byte(uint64_t seed, uint64_t idx)
{
    uint32_t g = (uint32_t)(idx >> 2);
    uint32_t w = mxref_fmix32(g ^ seed_key(seed));
    return (w >> (8u * (unsigned)(idx & 3u))) & 255u;
}

/* ------------------------------------------------------------------------ */
/* Fixed-sign 32-point Hadamard (reading of the FP4 pretraining abstract):   */
/* x_j <- s_j x_j with s_j = +1 where bit j of the mask is set, else -1;    */
/* then the unnormalised Sylvester butterfly, h = 1, 2, 4, 8, 16, in fp32.  */
/* ------------------------------------------------------------------------ */

void mxref_hadamard32(float *x, uint32_t sign_mask)
{
    for (int j = 0; j < BLOCK; ++j)
        if (!((sign_mask >> j) & 1u)) x[j] = -x[j];
    for (int h = 1; h < BLOCK; h <<= 1) {
        for (int i = 0; i < BLOCK; ++i) {
            if (i & h) continue;
            float a = x[i], b = x[i + h];
            x[i] = a + b;
            x[i + h] = a - b;
        }
    }
}

/* ------------------------------------------------------------------------ */
/* Storage layout (section 2: implementation-dependent).                    */
/*  codes: one row per block-axis line ("outer"), inner elements packed:    */
/*         8-bit one per byte; FP6 four codes per 3 bytes (c0 in bits 0-5   */
/*         of a little-endian 24-bit word, c1 bits 6-11, ...); FP4 two per  */
/*         byte, even element in the low nibble.                            */
/*  scales: plain = outer x (inner/32) row-major; MMA = rows padded to 128, */
/*         k-blocks padded to 4, 512-byte atoms of 128 rows x 4 k-blocks,   */
/*         atoms k-fastest, inside an atom (r%32)*16 + ((r/32)%4)*4 + kb%4; */
/*         MMA x4 = the MMA layout with every atom stored four times in a   */
/*         row (2048 bytes per atom; reads use the first copy).             */
/* ------------------------------------------------------------------------ */

int64_t mxref_codes_bytes(int fmt, int64_t outer, int64_t inner)
{
    int64_t bits = FMTS[fmt].bits;
    return outer * ((inner * bits) / 8);
}

int64_t mxref_scales_bytes(int sl, int64_t outer, int64_t inner)
{
    int64_t kb = inner / BLOCK;
    if (sl == SL_PLAIN) return outer * kb;
    int64_t rows = (outer + 127) / 128 * 128;
    int64_t kbp = (kb + 3) / 4 * 4;
    return rows * kbp * (sl == SL_MMA_X4 ? 4 : 1);
}

static int64_t scale_offset(int sl, int64_t outer_idx, int64_t kb, int64_t kb_total);

/* writes the scale byte of (outer_idx, kb): once, or in all four copies of
 * its atom in the x4 layout */
static void put_scale(uint8_t *scales, int sl, int64_t outer_idx, int64_t kb, int64_t kb_total, unsigned s)
{
    int64_t off = scale_offset(sl, outer_idx, kb, kb_total);
    for (int j = 0; j < (sl == SL_MMA_X4 ? 4 : 1); ++j) scales[off + 512 * j] = (uint8_t)s;
}

static int64_t scale_offset(int sl, int64_t outer_idx, int64_t kb, int64_t kb_total)
{
    if (sl == SL_PLAIN) return outer_idx * kb_total + kb;
    int64_t katoms = (kb_total + 3) / 4;
    int64_t atom = (outer_idx / 128) * katoms + kb / 4;
    int64_t r = outer_idx % 128;
    return atom * (sl == SL_MMA_X4 ? 2048 : 512) + (r % 32) * 16 + (r / 32) * 4 + (kb % 4);
}

static void put_code(int fmt, uint8_t *row, int64_t i, unsigned code)
{
    int bits = FMTS[fmt].bits;
    if (bits == 8) {
        row[i] = (uint8_t)code;
    } else if (bits == 4) {
        uint8_t b = row[i / 2];
        if (i % 2 == 0) b = (uint8_t)((b & 0xF0u) | (code & 0xFu));
        else b = (uint8_t)((b & 0x0Fu) | ((code & 0xFu) << 4));
        row[i / 2] = b;
    } else { /* 6-bit */
        int64_t g = i / 4, j = i % 4;
        uint8_t *p = row + 3 * g;
        uint32_t w = (uint32_t)p[0] | ((uint32_t)p[1] << 8) | ((uint32_t)p[2] << 16);
        w &= ~(0x3Fu << (6 * j));
        w |= (code & 0x3Fu) << (6 * j);
        p[0] = (uint8_t)w; p[1] = (uint8_t)(w >> 8); p[2] = (uint8_t)(w >> 16);
    }
}

unsigned mxref_get_code(int fmt, const uint8_t *row, int64_t i)
{
    int bits = FMTS[fmt].bits;
    if (bits == 8) return row[i];
    if (bits == 4) return (i % 2 == 0) ? (row[i / 2] & 0xFu) : (row[i / 2] >> 4);
    int64_t g = i / 4, j = i % 4;
    const uint8_t *p = row + 3 * g;
    uint32_t w = (uint32_t)p[0] | ((uint32_t)p[1] << 8) | ((uint32_t)p[2] << 16);
    return (w >> (6 * j)) & 0x3Fu;
}

/* ------------------------------------------------------------------------ */
/* Algorithm 1 on one block of 32 values.                                   */
/* ------------------------------------------------------------------------ */

static float load_elem(const void *x, int xdt, int64_t off)
{
    if (xdt == DT_F32) return ((const float *)x)[off];
    uint32_t bits = (uint32_t)((const uint16_t *)x)[off] << 16;   /* bf16 widens exactly */
    float f;
    memcpy(&f, &bits, 4);
    return f;
}

/* v: 32 fp32 inputs (already preconditioned if requested); idx0: linear
 * output index of v[0]; returns the E8M0 scale code. */
static unsigned quantize_block(int fmt, int rnd, uint64_t seed, const float *vin,
                               uint64_t idx0, unsigned *codes)
{
    const fmt_table *t = &TABLES[fmt];
    float v[BLOCK];
    /* section 3: FP32 subnormal inputs become zero (reading: sign kept, and
     * flushed before the amax so an all-subnormal block is an all-zero block) */
    for (int j = 0; j < BLOCK; ++j)
        v[j] = (fpclassify(vin[j]) == FP_SUBNORMAL) ? copysignf(0.0f, vin[j]) : vin[j];

    /* reading: a NaN or Inf anywhere makes the block NaN (scale 0xFF, codes 0) */
    for (int j = 0; j < BLOCK; ++j) {
        if (!isfinite(v[j])) {
            for (int k = 0; k < BLOCK; ++k) codes[k] = 0;
            return 0xFFu;
        }
    }

    double amax = 0.0;
    for (int j = 0; j < BLOCK; ++j)
        if (fabs((double)v[j]) > amax) amax = fabs((double)v[j]);

    int e;
    if (amax == 0.0) {
        e = -127;      /* reading: floor(log2 0) = -inf, clamped to the smallest scale */
    } else {
        int ex;
        frexp(amax, &ex);                  /* amax = f * 2^ex, f in [0.5, 1) */
        e = (ex - 1) - t->emax;            /* floor(log2 amax) - emax        */
        if (e < -127) e = -127;
        if (e > 127) e = 127;
    }

    for (int j = 0; j < BLOCK; ++j) {
        double u = ldexp((double)v[j], -e);    /* V_i / X, exact in double */
        if (rnd == RND_RNE)
            codes[j] = mxref_encode_rne(fmt, u);
        else
            codes[j] = mxref_encode_sr(fmt, u, mxref_sr_byte(seed, idx0 + (uint64_t)j));
    }
    return (unsigned)(e + 127);
}

/*
 * Cast a rows x cols tensor (row pitch ldx elements) to MX.
 * block_axis 1: blocks run along a row (contiguous); output is rows x cols.
 * block_axis 0: blocks run down a column (strided); output is cols x rows,
 *               i.e. block-axis-major (transposed on the way out).
 * hadamard != 0 applies the fixed-sign 32-point transform to each block.
 * codes / scales are written in full (packing bytes are overwritten); padding
 * entries of the MMA scale layout are left untouched.
 *
 * Shards (reading: stochastic rounding draws its random byte from the
 * element's position in the block-axis-major output of the WHOLE tensor, so
 * a tensor cut into pieces casts to the same bytes as the whole).  The tensor
 * given is the piece whose element (0, 0) is element (row0, col0) of a
 * total_rows x total_cols tensor; the element at (r, c) of the piece then has
 * stochastic-rounding index (row0 + r) * total_cols + col0 + c along rows
 * (block_axis 1) and (col0 + c) * total_rows + row0 + r along columns
 * (block_axis 0).  Blocks stay those of the whole tensor, so the offset along
 * the block axis is a multiple of 32.  Codes and scales are the piece's own
 * (its block-axis-major output, in local coordinates).
 */
int mxref_quantize_shard(const void *x, int xdt, int64_t rows, int64_t cols, int64_t ldx,
                         int block_axis, int fmt, int rnd, uint64_t seed,
                         int hadamard, uint32_t sign_mask,
                         int64_t row0, int64_t col0, int64_t total_rows, int64_t total_cols,
                         uint8_t *codes, uint8_t *scales, int sl)
{
    build_tables();
    if (!x || !codes || !scales) return MXO_ERR_ARG;
    if (fmt < 0 || fmt >= FMT_COUNT || (xdt != DT_F32 && xdt != DT_BF16)) return MXO_ERR_ARG;
    if (block_axis != 0 && block_axis != 1) return MXO_ERR_ARG;
    if (rows < 0 || cols < 0 || ldx < cols) return MXO_ERR_ARG;
    if (row0 < 0 || col0 < 0 || row0 + rows > total_rows || col0 + cols > total_cols) return MXO_ERR_ARG;
    int64_t outer = block_axis == 1 ? rows : cols;
    int64_t inner = block_axis == 1 ? cols : rows;
    int64_t inner_total = block_axis == 1 ? total_cols : total_rows;
    int64_t inner_off = block_axis == 1 ? col0 : row0;
    int64_t outer_off = block_axis == 1 ? row0 : col0;
    if (inner % BLOCK != 0 || inner_total % BLOCK != 0 || inner_off % BLOCK != 0) return MXO_ERR_SHAPE;
    /* the random-word counter floor(i / 4) must fit 32 bits: at most 2^34 elements */
    if (rnd == RND_SR && (uint64_t)total_rows * (uint64_t)total_cols > (1ull << 34)) return MXO_ERR_SR_RANGE;
    int64_t kb_total = inner / BLOCK;
    int64_t row_bytes = mxref_codes_bytes(fmt, 1, inner);

    #pragma omp parallel for schedule(static)
    for (int64_t o = 0; o < outer; ++o) {
        uint8_t *crow = codes + o * row_bytes;
        for (int64_t kb = 0; kb < kb_total; ++kb) {
            float v[BLOCK];
            unsigned c[BLOCK];
            for (int j = 0; j < BLOCK; ++j) {
                int64_t in = kb * BLOCK + j;
                int64_t r = block_axis == 1 ? o : in;
                int64_t cc = block_axis == 1 ? in : o;
                v[j] = load_elem(x, xdt, r * ldx + cc);
            }
            if (hadamard) mxref_hadamard32(v, sign_mask);
            /* position of the block's first element in the whole tensor's output */
            uint64_t idx0 = (uint64_t)((outer_off + o) * inner_total + inner_off + kb * BLOCK);
            unsigned s = quantize_block(fmt, rnd, seed, v, idx0, c);
            for (int j = 0; j < BLOCK; ++j) put_code(fmt, crow, kb * BLOCK + j, c[j]);
            put_scale(scales, sl, o, kb, kb_total, s);
        }
    }
    return MXO_OK;
}

/* The whole tensor: a piece at (0, 0) of itself. */
int mxref_quantize(const void *x, int xdt, int64_t rows, int64_t cols, int64_t ldx,
                   int block_axis, int fmt, int rnd, uint64_t seed,
                   int hadamard, uint32_t sign_mask,
                   uint8_t *codes, uint8_t *scales, int sl)
{
    return mxref_quantize_shard(x, xdt, rows, cols, ldx, block_axis, fmt, rnd, seed, hadamard, sign_mask,
                                0, 0, rows, cols, codes, scales, sl);
}

/* Exact decode v = 2^(scale - 127) * P (section 2); a 0xFF scale gives NaN. */
int mxref_dequantize(const uint8_t *codes, const uint8_t *scales, int fmt, int sl,
                     int64_t outer, int64_t inner, double *y)
{
    build_tables();
    if (!codes || !scales || !y) return MXO_ERR_ARG;
    if (fmt < 0 || fmt >= FMT_COUNT) return MXO_ERR_ARG;
    if (inner % BLOCK != 0) return MXO_ERR_SHAPE;
    int64_t kb_total = inner / BLOCK;
    int64_t row_bytes = mxref_codes_bytes(fmt, 1, inner);
    #pragma omp parallel for schedule(static)
    for (int64_t o = 0; o < outer; ++o) {
        for (int64_t i = 0; i < inner; ++i) {
            unsigned s = scales[scale_offset(sl, o, i / BLOCK, kb_total)];
            unsigned c = mxref_get_code(fmt, codes + o * row_bytes, i);
            double p = mxref_decode_elem(fmt, c);
            y[o * inner + i] = (s == 0xFFu) ? NAN : ldexp(p, (int)s - 127);
        }
    }
    return MXO_OK;
}

/* ------------------------------------------------------------------------ */
/* Rounding of exact doubles to the output types (round to nearest even).    */
/* ------------------------------------------------------------------------ */

void mxref_round_f32(const double *in, float *out, int64_t n)
{
    for (int64_t i = 0; i < n; ++i) out[i] = (float)in[i];   /* C cast: current mode, RNE */
}

/* direct double -> bf16 (8 significant bits, exponent range of fp32) */
static uint16_t to_bf16(double d)
{
    if (isnan(d)) return 0x7FC0u;
    int neg = signbit(d) != 0;
    double a = fabs(d);
    uint16_t sign = neg ? 0x8000u : 0u;
    if (a == 0.0) return sign;
    /* grid spacing for a: 2^(floor(log2 a) - 7), but never below the
     * subnormal spacing 2^-133 */
    int ex;
    frexp(a, &ex);                       /* a = f * 2^ex, f in [0.5,1) */
    int q = (ex - 1) - 7;
    if (q < -133) q = -133;
    double k = nearbyint(ldexp(a, -q));   /* RNE to an integer multiple of 2^q */
    double r = ldexp(k, q);
    if (r >= ldexp(1.0, 128)) return sign | 0x7F80u;   /* overflow -> Inf */
    float f = (float)r;                  /* exact: r has <= 8 significant bits */
    uint32_t bits;
    memcpy(&bits, &f, 4);
    return (uint16_t)(bits >> 16) | sign;
}

void mxref_round_bf16(const double *in, uint16_t *out, int64_t n)
{
    for (int64_t i = 0; i < n; ++i) out[i] = to_bf16(in[i]);
}

/* ------------------------------------------------------------------------ */
/* Block-scaled GEMM (section 4 compute flow): C = alpha * A * B^T with A   */
/* M x K and B N x K, both quantized along K (MMA scale layout).  Every     */
/* element is decoded exactly and the sum runs in fp64 in k order; also     */
/* returns bound[m,n] = |alpha| * sum_k |a_mk * b_nk|.                      */
/* ------------------------------------------------------------------------ */

static double decoded(int fmt, const uint8_t *codes, const uint8_t *scales,
                      int64_t o, int64_t k, int64_t K, int sl)
{
    int64_t row_bytes = mxref_codes_bytes(fmt, 1, K);
    unsigned s = scales[scale_offset(sl, o, k / BLOCK, K / BLOCK)];
    unsigned c = mxref_get_code(fmt, codes + o * row_bytes, k);
    if (s == 0xFFu) return NAN;
    return ldexp(mxref_decode_elem(fmt, c), (int)s - 127);
}

static void gemm_entry(const uint8_t *ac, const uint8_t *as, int fa,
                       const uint8_t *bc, const uint8_t *bs, int fb,
                       int64_t K, double alpha, int sl, int64_t m, int64_t n,
                       double *c, double *bound)
{
    double acc = 0.0, mag = 0.0;
    for (int64_t k = 0; k < K; ++k) {
        double a = decoded(fa, ac, as, m, k, K, sl);
        double b = decoded(fb, bc, bs, n, k, K, sl);
        acc += a * b;
        mag += fabs(a * b);
    }
    *c = alpha * acc;
    *bound = fabs(alpha) * mag;
}

int mxref_gemm_f64(const uint8_t *a_codes, const uint8_t *a_scales, int fa,
                   const uint8_t *b_codes, const uint8_t *b_scales, int fb,
                   int64_t M, int64_t N, int64_t K, double alpha, int sl,
                   double *c, double *bound)
{
    build_tables();
    if (!a_codes || !a_scales || !b_codes || !b_scales || !c || !bound) return MXO_ERR_ARG;
    if (K % BLOCK != 0) return MXO_ERR_SHAPE;
    #pragma omp parallel for schedule(dynamic, 1)
    for (int64_t m = 0; m < M; ++m)
        for (int64_t n = 0; n < N; ++n)
            gemm_entry(a_codes, a_scales, fa, b_codes, b_scales, fb, K, alpha, sl, m, n,
                       &c[m * N + n], &bound[m * N + n]);
    return MXO_OK;
}

/* the same sum for a list of (m, n) entries only */
int mxref_gemm_entries(const uint8_t *a_codes, const uint8_t *a_scales, int fa,
                       const uint8_t *b_codes, const uint8_t *b_scales, int fb,
                       int64_t K, double alpha, int sl,
                       const int64_t *ms, const int64_t *ns, int64_t count,
                       double *c, double *bound)
{
    build_tables();
    if (!a_codes || !a_scales || !b_codes || !b_scales || !c || !bound) return MXO_ERR_ARG;
    if (K % BLOCK != 0) return MXO_ERR_SHAPE;
    #pragma omp parallel for schedule(dynamic, 16)
    for (int64_t i = 0; i < count; ++i)
        gemm_entry(a_codes, a_scales, fa, b_codes, b_scales, fb, K, alpha, sl, ms[i], ns[i],
                   &c[i], &bound[i]);
    return MXO_OK;
}

/* ------------------------------------------------------------------------ */
/* NVFP4 scale domains (reading of "global NVFP4" and "cooperative-thread-  */
/* array-local NVFP4", FP4 pretraining abstract; the pages name these       */
/* domains but do not define them, so this follows the public NVFP4         */
/* format):                                                                 */
/*  - blocks of 16 consecutive elements along the block axis (rows, here);   */
/*    elements E2M1; one E4M3 block scale (positive; 0x7F, the E4M3 NaN     */
/*    code, marks a block holding a NaN or Inf, whose codes are then 0);     */
/*  - one fp32 encode scale E per domain: the whole tensor ("global"), or    */
/*    each group of domain_lines consecutive rows ("CTA-local": the rows one */
/*    CTA of the cast owns, all of the block axis);                          */
/*  - every step in fp32 IEEE arithmetic (round to nearest even, no fused    */
/*    multiply-add, no flush): a_D = largest finite |x| of the domain,       */
/*    E = 2688 / a_D (6 * 448: the largest E2M1 and E4M3 values; 1 when      */
/*    a_D = 0, the largest finite fp32 when the quotient overflows); per     */
/*    block a_b = largest |x|, block scale s = E4M3(RNE, saturating) of      */
/*    (a_b / 6) * E, d its value, r = E / d (0 when d = 0), and each code    */
/*    E2M1(RNE, saturating) of x * r;                                        */
/*  - the value of a code P in a block with scale value d is P * d / E.      */
/* ------------------------------------------------------------------------ */
#define NV_BLOCK 16
#define NV_SCALE_NAN 0x7Fu

static float nv_encode_scale(float amax)
{
    if (!(amax > 0.0f)) return 1.0f;
    float e = 2688.0f / amax;
    if (isinf(e)) e = 3.40282346638528859812e+38f;      /* largest finite fp32 */
    return e;
}

int64_t mxref_nvfp4_scales_bytes(int sl, int64_t rows, int64_t cols)
{
    /* one byte per 16-block; the MMA layout is the MX atom layout over 16-blocks */
    return mxref_scales_bytes(sl, rows, cols * 2);
}

/* Cast along rows (block axis 1).  domain_lines 0: one global domain, else
 * rows are grouped domain_lines at a time.  codes: rows x cols/2 bytes (E2M1,
 * even element in the low nibble); scales: plain rows x cols/16 or the MMA
 * atom layout; enc_scales: one fp32 per domain. */
int mxref_nvfp4_quantize(const void *x, int xdt, int64_t rows, int64_t cols, int64_t ldx,
                         int64_t domain_lines, uint8_t *codes, uint8_t *scales, int sl, float *enc_scales)
{
    build_tables();
    if (!x || !codes || !scales || !enc_scales) return MXO_ERR_ARG;
    if ((xdt != DT_F32 && xdt != DT_BF16) || rows < 0 || cols < 0 || ldx < cols || domain_lines < 0)
        return MXO_ERR_ARG;
    if (cols % NV_BLOCK != 0) return MXO_ERR_SHAPE;
    const int64_t lines = domain_lines == 0 ? (rows > 0 ? rows : 1) : domain_lines;
    const int64_t n_dom = (rows + lines - 1) / lines;
    const int64_t kb_total = cols / NV_BLOCK;
    const int64_t row_bytes = cols / 2;

    for (int64_t d = 0; d < n_dom; ++d) {
        float amax = 0.0f;
        for (int64_t r = d * lines; r < rows && r < (d + 1) * lines; ++r)
            for (int64_t c = 0; c < cols; ++c) {
                float v = load_elem(x, xdt, r * ldx + c);
                if (isfinite(v) && fabsf(v) > amax) amax = fabsf(v);
            }
        enc_scales[d] = nv_encode_scale(amax);
    }

    #pragma omp parallel for schedule(static)
    for (int64_t o = 0; o < rows; ++o) {
        const float E = enc_scales[o / lines];
        uint8_t *crow = codes + o * row_bytes;
        for (int64_t kb = 0; kb < kb_total; ++kb) {
            float v[NV_BLOCK];
            int finite = 1;
            float amax = 0.0f;
            for (int j = 0; j < NV_BLOCK; ++j) {
                v[j] = load_elem(x, xdt, o * ldx + kb * NV_BLOCK + j);
                if (!isfinite(v[j])) finite = 0;
                else if (fabsf(v[j]) > amax) amax = fabsf(v[j]);
            }
            unsigned s;
            if (!finite) {
                s = NV_SCALE_NAN;
                for (int j = 0; j < NV_BLOCK; ++j) put_code(FMT_E2M1, crow, kb * NV_BLOCK + j, 0);
            } else {
                float t = (amax / 6.0f) * E;
                s = mxref_encode_rne(FMT_E4M3, (double)t);      /* t >= 0: a positive code */
                float dval = (float)mxref_decode_elem(FMT_E4M3, s);
                float r = dval > 0.0f ? E / dval : 0.0f;
                for (int j = 0; j < NV_BLOCK; ++j) {
                    float u = v[j] * r;
                    put_code(FMT_E2M1, crow, kb * NV_BLOCK + j, mxref_encode_rne(FMT_E2M1, (double)u));
                }
            }
            put_scale(scales, sl, o, kb, kb_total, s);
        }
    }
    return MXO_OK;
}

/* Decode: P * d / E in double (P * d is exact; the one division rounds); a
 * 0x7F block scale gives NaN for its block. */
int mxref_nvfp4_dequantize(const uint8_t *codes, const uint8_t *scales, int sl, int64_t rows, int64_t cols,
                           const float *enc_scales, int64_t domain_lines, double *y)
{
    build_tables();
    if (!codes || !scales || !enc_scales || !y || domain_lines < 0) return MXO_ERR_ARG;
    if (cols % NV_BLOCK != 0) return MXO_ERR_SHAPE;
    const int64_t lines = domain_lines == 0 ? (rows > 0 ? rows : 1) : domain_lines;
    const int64_t kb_total = cols / NV_BLOCK;
    for (int64_t o = 0; o < rows; ++o) {
        const double E = (double)enc_scales[o / lines];
        const uint8_t *crow = codes + o * (cols / 2);
        for (int64_t kb = 0; kb < kb_total; ++kb) {
            unsigned s = scales[scale_offset(sl, o, kb, kb_total)];
            double dval = s == NV_SCALE_NAN ? NAN : mxref_decode_elem(FMT_E4M3, s);
            for (int j = 0; j < NV_BLOCK; ++j) {
                double p = mxref_decode_elem(FMT_E2M1, mxref_get_code(FMT_E2M1, crow, kb * NV_BLOCK + j));
                y[o * cols + kb * NV_BLOCK + j] = (p * dval) / E;
            }
        }
    }
    return MXO_OK;
}
