"""GPU parity of the block-scaled GEMM (compute flow of "Microscaling Data
Formats for Deep Learning", summary page, section 4: dot products on MX inputs
return scalar floats) against the oracle.

Tolerance (stated for the GEMM): |C - C_ref| <= 1e-5 * |alpha| * sum_k |a_mk b_nk|
for fp32 output, plus one bf16 ulp of C_ref for bf16 output.  Where every
partial sum is exact in fp32 the result must be bit-exact.
"""
import numpy as np
import pytest
import torch

from gpu_helpers import dev, host, to_device
from microscaling_block_scaled_mx_b200 import inputs as I
from microscaling_block_scaled_mx_b200 import mx

pytestmark = pytest.mark.gpu

REL_TOL = 1e-5


def bf16_ulp(x):
    a = np.abs(np.asarray(x, dtype=np.float64))
    _, ex = np.frexp(a)
    e = np.maximum(ex - 1, -126)
    return np.exp2(e - 7.0)


def check(got, ref, bound, out_dtype, what=""):
    got = np.asarray(got, dtype=np.float64)
    tol = REL_TOL * bound
    if out_dtype == torch.bfloat16:
        tol = tol + bf16_ulp(ref)
    err = np.abs(got - ref)
    bad = err > tol
    assert not np.any(np.isnan(got)), (what, "NaN in output")
    if np.any(bad):
        i = np.argwhere(bad)[:5]
        raise AssertionError((what, int(bad.sum()), [(tuple(j), got[tuple(j)], ref[tuple(j)], tol[tuple(j)])
                                                     for j in i]))


def to_f64(t):
    return host(t.float()).astype(np.float64) if t.dtype == torch.bfloat16 else host(t).astype(np.float64)


def run_gemm(oracle, a, b, fmt, M, N, K, alpha=1.0, out_dtype=torch.float32, ldc=None, rows=None, fb=None):
    """a: M x K, b: N x K host arrays (float32 or bf16 bits); both cast along K
    by the GPU (verified bit-exact elsewhere) and by the oracle.  A is cast to
    fmt, B to fb (default fmt)."""
    fb = fmt if fb is None else fb
    ac, as_ = mx.quantize(to_device(a), 1, fmt)
    bc, bs = mx.quantize(to_device(b), 1, fb)
    if ldc is None:
        out = torch.empty((M, N), dtype=out_dtype, device=dev())
    else:
        out = torch.empty((M, ldc), dtype=out_dtype, device=dev())[:, :N]
    out.fill_(float("nan"))
    mx.gemm(ac, as_, bc, bs, M, N, K, fa=fmt, fb=fb, alpha=alpha, out=out)
    torch.cuda.synchronize()
    f, g = oracle.FORMATS[fmt], oracle.FORMATS[fb]
    oac, oas = oracle.quantize(a, 1, f, scale_layout=oracle.MMA)
    obc, obs = oracle.quantize(b, 1, g, scale_layout=oracle.MMA)
    ref, bound = oracle.gemm_decoded(oac, oas, f, obc, obs, g, M, N, K, alpha=alpha, rows=rows)
    got = to_f64(out)
    if rows is not None:
        got = got[np.asarray(rows)]
    return got, ref, bound


def small_int_operand(rng, rows, K):
    """Small integers times a power of two per 32-block: every product and
    partial sum is exact in fp32, and the block scales vary."""
    v = rng.integers(-3, 4, (rows, K)).astype(np.float64)
    v *= np.exp2(np.repeat(rng.integers(-2, 3, (rows, K // 32)), 32, axis=1))
    return v.astype(np.float32)


@pytest.mark.parametrize("fmt,K", [("e4m3", 128), ("e4m3", 512), ("e2m1", 256), ("e2m1", 1024),
                                   ("e5m2", 256)])
def test_gemm_single_tile_bit_exact(oracle, fmt, K):
    rng = np.random.default_rng(K)
    M, N = 128, 256
    a = small_int_operand(rng, M, K)
    b = small_int_operand(rng, N, K)
    if fmt == "e2m1":   # keep the values on the E2M1 grid: {0, .5, 1, 1.5, 2, 3} x 2^k
        a = np.clip(a, -3, 3)
        b = np.clip(b, -3, 3)
    got, ref, bound = run_gemm(oracle, a, b, fmt, M, N, K)
    exact = oracle.round_f32(ref).astype(np.float64)
    assert np.array_equal(got, exact), np.argwhere(got != exact)[:5]


@pytest.mark.parametrize("fmt,K", [("e4m3", 256), ("e2m1", 512), ("e5m2", 128)])
@pytest.mark.parametrize("M,N", [(256, 192), (256, 384), (512, 576)])
def test_gemm_one_sm_multi_tile_bit_exact(oracle, fmt, K, M, N):
    """Short-K shapes run on the one-SM kernel (128 x 192 tiles); N = 384 and
    576 include odd 192-column tiles, whose B scales start 64 rows into a
    scale block."""
    rng = np.random.default_rng(M + N + K)
    a = small_int_operand(rng, M, K)
    b = small_int_operand(rng, N, K)
    if fmt == "e2m1":
        a = np.clip(a, -3, 3)
        b = np.clip(b, -3, 3)
    got, ref, bound = run_gemm(oracle, a, b, fmt, M, N, K)
    exact = oracle.round_f32(ref).astype(np.float64)
    assert np.array_equal(got, exact), np.argwhere(got != exact)[:5]


@pytest.mark.parametrize("fmt", ["e4m3", "e2m1"])
def test_gemm_two_sm_tiles_bit_exact(oracle, fmt):
    """K >= 2048 with at least one 256 x 256 tile per SM runs on CTA pairs
    (cta_group::2); ragged M and N exercise the clamped loads of a pair half
    that lies wholly past the edge."""
    K = 2048 if fmt == "e4m3" else 4096
    for (M, N) in [(4096, 2560), (4000, 2600)]:
        rng = np.random.default_rng(M + N)
        a = small_int_operand(rng, M, K)
        b = small_int_operand(rng, N, K)
        if fmt == "e2m1":
            a = np.clip(a, -3, 3)
            b = np.clip(b, -3, 3)
        got, ref, bound = run_gemm(oracle, a, b, fmt, M, N, K)
        exact = oracle.round_f32(ref).astype(np.float64)
        assert np.array_equal(got, exact), (M, N, np.argwhere(got != exact)[:5])


# Mixed and FP6 pairs run kind::mxf8f6f4 with FP6 and FP4 codes expanded to
# one per byte by the copy engine; E2M1 x E2M1 with K = 128 (mod 256) takes
# the same route instead of kind::mxf4.
MIXED_PAIRS = [("e2m1", "e3m2"), ("e3m2", "e2m1"), ("e2m3", "e2m3"), ("e3m2", "e3m2"),
               ("e4m3", "e2m1"), ("e2m1", "e5m2"), ("e5m2", "e2m3"), ("e2m3", "e4m3")]


@pytest.mark.parametrize("fa,fb", MIXED_PAIRS + [("e2m1", "e2m1")])
@pytest.mark.parametrize("M,N,K", [(128, 256, 128), (256, 384, 384), (512, 576, 256)])
def test_gemm_mixed_one_sm_bit_exact(oracle, fa, fb, M, N, K):
    rng = np.random.default_rng(M + N + K + len(fa + fb))
    # values clipped to [-3, 3] times the block's power of two sit on every element grid
    a = np.clip(small_int_operand(rng, M, K), -3, 3)
    b = np.clip(small_int_operand(rng, N, K), -3, 3)
    if fa == fb == "e2m1" and K % 256 == 0:
        K = K + 128          # the FP4 x FP4 case of interest here is K = 128 (mod 256)
        a = np.concatenate([a, a[:, :128]], axis=1)
        b = np.concatenate([b, b[:, :128]], axis=1)
    got, ref, bound = run_gemm(oracle, a, b, fa, M, N, K, fb=fb)
    exact = oracle.round_f32(ref).astype(np.float64)
    assert np.array_equal(got, exact), (fa, fb, np.argwhere(got != exact)[:5])


@pytest.mark.parametrize("fa,fb", [("e2m1", "e3m2"), ("e3m2", "e3m2"), ("e4m3", "e2m3")])
def test_gemm_mixed_two_sm_bit_exact(oracle, fa, fb):
    """Pair-kernel shapes (K >= 2048, >= one 256 x 256 tile per SM), ragged
    second shape."""
    K = 2048
    for (M, N) in [(4096, 2560), (4000, 2600)]:
        rng = np.random.default_rng(M + N + 1)
        a, b = small_int_operand(rng, M, K), small_int_operand(rng, N, K)
        a, b = np.clip(a, -3, 3), np.clip(b, -3, 3)
        got, ref, bound = run_gemm(oracle, a, b, fa, M, N, K, fb=fb)
        exact = oracle.round_f32(ref).astype(np.float64)
        assert np.array_equal(got, exact), (fa, fb, M, N, np.argwhere(got != exact)[:5])


@pytest.mark.parametrize("fa,fb", MIXED_PAIRS)
@pytest.mark.parametrize("out_dtype", [torch.float32, torch.bfloat16])
def test_gemm_mixed_tolerance(oracle, fa, fb, out_dtype):
    rng = np.random.default_rng(17)
    for (M, N, K) in [(384, 768, 1024), (200, 300, 384)]:
        a = (rng.standard_normal((M, K)) * np.exp2(rng.uniform(-4, 4, (M, 1)))).astype(np.float32)
        b = rng.standard_t(3, size=(N, K)).astype(np.float32)
        ldc = (N + 7) // 8 * 8 + 8          # padded pitch, a multiple of 16 bytes
        got, ref, bound = run_gemm(oracle, a, b, fa, M, N, K, alpha=0.75, out_dtype=out_dtype, fb=fb, ldc=ldc)
        check(got, ref, bound, out_dtype, (fa, fb, M, N, K))


@pytest.mark.parametrize("fmt", ["e4m3", "e5m2", "e2m1"])
@pytest.mark.parametrize("out_dtype", [torch.float32, torch.bfloat16])
def test_gemm_multi_tile_tolerance(oracle, fmt, out_dtype):
    rng = np.random.default_rng(7)
    M, N, K = 384, 768, 2048
    a = (rng.standard_normal((M, K)) * np.exp2(rng.uniform(-4, 4, (M, 1)))).astype(np.float32)
    b = rng.standard_t(3, size=(N, K)).astype(np.float32)
    got, ref, bound = run_gemm(oracle, a, b, fmt, M, N, K, alpha=0.75, out_dtype=out_dtype)
    check(got, ref, bound, out_dtype, fmt)


@pytest.mark.parametrize("fmt,K", [("e4m3", 384), ("e2m1", 512)])
def test_gemm_ragged_m_n_and_pitched_c(oracle, fmt, K):
    rng = np.random.default_rng(11)
    for (M, N) in [(200, 300), (1, 1), (129, 257), (130, 100), (300, 200), (520, 97)]:
        a = rng.standard_normal((M, K)).astype(np.float32)
        b = rng.standard_normal((N, K)).astype(np.float32)
        for out_dtype in (torch.float32, torch.bfloat16):
            ldc = (N + 7) // 8 * 8 + 8        # padded pitch, a multiple of 16 bytes
            got, ref, bound = run_gemm(oracle, a, b, fmt, M, N, K, out_dtype=out_dtype, ldc=ldc)
            check(got, ref, bound, out_dtype, (fmt, M, N))


def test_gemm_k_zero_and_empty():
    c = torch.full((4, 8), 7.0, device=dev())
    z = torch.empty(0, dtype=torch.uint8, device=dev())
    mx.gemm(z, z, z, z, 4, 8, 0, fa="e4m3", out=c)
    torch.cuda.synchronize()
    assert torch.all(c == 0)
    mx.gemm(z, z, z, z, 0, 8, 128, fa="e4m3", out=torch.empty((0, 8), device=dev()))


def test_gemm_roundtrip_config(oracle):
    """fp32 A 256x512 (blocks along K = rows of A) times B 512x256 (K x N,
    blocks along K = down its columns), E4M3, fp32 out, every entry."""
    d = I.config_roundtrip()
    A, B = d["A"], d["B"]
    M, K = A.shape
    N = B.shape[1]
    ac, as_ = mx.quantize(to_device(A), 1, "e4m3")
    bc, bs = mx.quantize(to_device(B), 0, "e4m3")        # N x K codes
    c = mx.gemm(ac, as_, bc, bs, M, N, K, fa="e4m3", out_dtype=torch.float32)
    torch.cuda.synchronize()
    oac, oas = oracle.quantize(A, 1, 0, scale_layout=1)
    obc, obs = oracle.quantize(B, 0, 0, scale_layout=1)
    ref, bound = oracle.gemm(oac, oas, 0, obc, obs, 0, M, N, K)
    check(to_f64(c), ref, bound, torch.float32)


@pytest.mark.parametrize("idx", [0, 1])
def test_gemm_gpt2_config(oracle, idx):
    """GPT-2-small-shaped MXFP8 GEMMs (M=8192, 768->3072 and 3072->768), bf16
    activations N(0,1) and weights N(0,0.02^2) cast along K, bf16 out: all of C."""
    M, N, K = I.GPT2_GEMMS[idx]
    x, w = I.linear_operands(M, K, N, 2, stream=idx)
    got, ref, bound = run_gemm(oracle, x, w, "e4m3", M, N, K, out_dtype=torch.bfloat16)
    check(got, ref, bound, torch.bfloat16, (M, N, K))


@pytest.mark.parametrize("idx", [0, 1, 2])
def test_gemm_llama3_config(oracle, idx):
    """Llama-3-8B-shaped MXFP4 GEMMs along K, bf16 out: 512 sampled rows of C
    (every column) and four whole 128 x 128 output tiles."""
    M, N, K = I.LLAMA3_GEMMS[idx]
    x, w = I.linear_operands(M, K, N, 3, stream=idx)
    rng = np.random.default_rng(idx)
    rows = np.sort(rng.choice(M, 512, replace=False))
    tiles = [(int(rng.integers(M // 128)) * 128, int(rng.integers(N // 128)) * 128) for _ in range(4)]
    tile_rows = np.unique(np.concatenate([np.arange(m0, m0 + 128) for m0, _ in tiles]))
    all_rows = np.union1d(rows, tile_rows)
    got, ref, bound = run_gemm(oracle, x, w, "e2m1", M, N, K, out_dtype=torch.bfloat16, rows=all_rows)
    pos = {int(r): i for i, r in enumerate(all_rows)}
    sel = np.array([pos[int(r)] for r in rows])
    check(got[sel], ref[sel], bound[sel], torch.bfloat16, (M, N, K, "rows"))
    for m0, n0 in tiles:
        ti = np.array([pos[r] for r in range(m0, m0 + 128)])
        check(got[ti, n0:n0 + 128], ref[ti, n0:n0 + 128], bound[ti, n0:n0 + 128], torch.bfloat16,
              (M, N, K, "tile", m0, n0))


def test_gemm_llama3_along_m(oracle):
    """The same activations cast along M (transposed blocks): the weight-gradient
    shaped product C^T X contracts over the 8192 tokens.  C is the forward
    output of the 4096->6144 GEMM (bf16), cast along M as well."""
    M, N, K = I.LLAMA3_GEMMS[0]
    x, w = I.linear_operands(M, K, N, 3, stream=0)
    xd = to_device(x)
    ac, as_ = mx.quantize(xd, 1, "e2m1")
    bc, bs = mx.quantize(to_device(w), 1, "e2m1")
    c = mx.gemm(ac, as_, bc, bs, M, N, K, fa="e2m1", out_dtype=torch.bfloat16)      # 8192 x 6144
    gc, gs = mx.quantize(c, 0, "e2m1")            # 6144 x 8192 codes (blocks along tokens)
    xc, xs = mx.quantize(xd, 0, "e2m1")           # 4096 x 8192 codes
    dw = mx.gemm(gc, gs, xc, xs, N, K, M, fa="e2m1", out_dtype=torch.float32)       # 6144 x 4096
    torch.cuda.synchronize()
    c_bits = host(c)
    ogc, ogs = oracle.quantize(c_bits, 0, oracle.E2M1, scale_layout=oracle.MMA)
    oxc, oxs = oracle.quantize(x, 0, oracle.E2M1, scale_layout=oracle.MMA)
    assert np.array_equal(host(gc), ogc) and np.array_equal(host(xc), oxc)
    rows = np.sort(np.random.default_rng(5).choice(N, 256, replace=False))
    ref, bound = oracle.gemm_decoded(ogc, ogs, oracle.E2M1, oxc, oxs, oracle.E2M1, N, K, M, rows=rows)
    check(to_f64(dw)[rows], ref, bound, torch.float32, "along M")


def test_gemm_wgrad_config(oracle, wgrad_oracle_operands):
    """dW = alpha * dY^T X with tokens K=16384: dY 16384x4096 and X 16384x14336
    (Student-t), both cast along tokens with the fixed-sign Hadamard and
    stochastic rounding to E2M1, alpha = 1/32, fp32 out; 512 sampled rows and
    four whole 128 x 128 tiles.  The reference is computed from the oracle's
    own casts of dY and X; the GPU's casts must equal them byte for byte."""
    d = wgrad_oracle_operands
    dy, xx = d["dy"], d["xx"]
    T, Do = dy.shape
    Di = xx.shape[1]
    (oac, oas), (obc, obs) = d["dy_q"], d["xx_q"]
    ac, as_ = mx.quantize(to_device(dy), 0, "e2m1", rnd="sr", seed=42, hadamard=True, sign_mask=d["mask"])
    bc, bs = mx.quantize(to_device(xx), 0, "e2m1", rnd="sr", seed=43, hadamard=True, sign_mask=d["mask"])
    dw = mx.gemm(ac, as_, bc, bs, Do, Di, T, fa="e2m1", alpha=1.0 / 32, out_dtype=torch.float32)
    torch.cuda.synchronize()
    assert np.array_equal(host(ac), oac) and np.array_equal(host(as_)[:oas.size], oas)
    assert np.array_equal(host(bc), obc) and np.array_equal(host(bs)[:obs.size], obs)
    rng = np.random.default_rng(9)
    rows = np.sort(rng.choice(Do, 512, replace=False))
    tiles = [(int(rng.integers(Do // 128)) * 128, int(rng.integers(Di // 128)) * 128) for _ in range(4)]
    all_rows = np.union1d(rows, np.concatenate([np.arange(m0, m0 + 128) for m0, _ in tiles]))
    ref, bound = oracle.gemm_decoded(oac, oas, oracle.E2M1, obc, obs, oracle.E2M1, Do, Di, T,
                                     alpha=1.0 / 32, rows=all_rows)
    got = to_f64(dw)[all_rows]
    check(got, ref, bound, torch.float32, "wgrad")
    pos = {int(r): i for i, r in enumerate(all_rows)}
    for m0, n0 in tiles:
        ti = np.array([pos[r] for r in range(m0, m0 + 128)])
        check(got[ti, n0:n0 + 128], ref[ti, n0:n0 + 128], bound[ti, n0:n0 + 128], torch.float32,
              ("wgrad tile", m0, n0))


@pytest.mark.parametrize("M,N,K", [(256, 256, 1024), (1024, 384, 512), (4096, 2560, 2048)])
def test_gemm_bounded_wait_reports_timeout(M, N, K):
    """A stage that is never filled: the MMA issuer's bounded wait runs out, the
    kernel records MX_ERR_TIMEOUT and returns; the context stays usable.  The
    shapes run on the one-SM kernel, the resident-B kernel and CTA pairs."""
    rng = np.random.default_rng(1)
    a = to_device(rng.standard_normal((M, K)).astype(np.float32))
    b = to_device(rng.standard_normal((N, K)).astype(np.float32))
    ac, as_ = mx.quantize(a, 1, "e4m3")
    bc, bs = mx.quantize(b, 1, "e4m3")
    assert mx.last_device_status() == 0
    mx.lib().mx_debug_gemm_skip_stage(3)
    mx.gemm(ac, as_, bc, bs, M, N, K, fa="e4m3", out_dtype=torch.float32)
    assert mx.last_device_status() == -7
    assert mx.last_device_status() == 0          # read-and-clear
    c = mx.gemm(ac, as_, bc, bs, M, N, K, fa="e4m3", out_dtype=torch.float32)
    torch.cuda.synchronize()
    assert mx.last_device_status() == 0
    assert torch.isfinite(c).all()


@pytest.mark.parametrize("M,N,K", [(200, 300, 384), (520, 97, 512), (4000, 2600, 2048)])
@pytest.mark.parametrize("out_dtype", [torch.float32, torch.bfloat16])
def test_gemm_writes_only_inside_c(oracle, M, N, K, out_dtype):
    """The epilogue's stores stay inside the M x N window of a pitched C: the
    columns between N and the leading dimension and the rows after M keep
    their contents (one-SM and CTA-pair kernels, both output types)."""
    rng = np.random.default_rng(M * 7 + N)
    a = rng.standard_normal((M, K)).astype(np.float32)
    b = rng.standard_normal((N, K)).astype(np.float32)
    ac, as_ = mx.quantize(to_device(a), 1, "e4m3")
    bc, bs = mx.quantize(to_device(b), 1, "e4m3")
    ldc = (N + 7) // 8 * 8 + 40
    buf = torch.full((M + 3, ldc), 123.0, dtype=out_dtype, device=dev())
    out = buf[:M, :N]
    mx.gemm(ac, as_, bc, bs, M, N, K, fa="e4m3", out=out)
    torch.cuda.synchronize()
    h = to_f64(buf)
    assert np.all(h[:M, N:] == 123.0) and np.all(h[M:, :] == 123.0)
    oac, oas = oracle.quantize(a, 1, oracle.E4M3, scale_layout=oracle.MMA)
    obc, obs = oracle.quantize(b, 1, oracle.E4M3, scale_layout=oracle.MMA)
    ref, bound = oracle.gemm_decoded(oac, oas, oracle.E4M3, obc, obs, oracle.E4M3, M, N, K)
    check(h[:M, :N], ref, bound, out_dtype, (M, N, K))


# Every kernel on every shape: the automatic choice picks one kernel per
# shape; mx_debug_gemm_force_kernel (include/mx_debug.h) lets these tests run
# the one-SM kernel (0) and both CTA-pair tile widths (256, 192) on the same
# operands.
KERNELS = [0, 1, 256, 192]   # one-SM, one-SM with a resident B panel, CTA pairs


class forced_kernel:
    def __init__(self, tile_n):
        self.tile_n = tile_n

    def __enter__(self):
        assert mx.lib().mx_debug_gemm_force_kernel(self.tile_n) == 0
        return self

    def __exit__(self, *exc):
        mx.lib().mx_debug_gemm_force_kernel(-1)
        return False


@pytest.mark.parametrize("kernel", KERNELS)
@pytest.mark.parametrize("fa,fb,K", [("e4m3", "e4m3", 512), ("e2m1", "e2m1", 1024), ("e3m2", "e2m1", 384),
                                     ("e5m2", "e2m3", 256)])
def test_gemm_each_kernel_bit_exact(oracle, kernel, fa, fb, K):
    """Exact partial sums, so every kernel must return the oracle's C bit for
    bit; shapes with several tiles along both axes, odd 192-column tiles and
    ragged edges on both axes."""
    for (M, N) in [(512, 576), (300, 200), (640, 1000)]:
        rng = np.random.default_rng(M + N + K + kernel)
        a = np.clip(small_int_operand(rng, M, K), -3, 3)
        b = np.clip(small_int_operand(rng, N, K), -3, 3)
        with forced_kernel(kernel):
            got, ref, bound = run_gemm(oracle, a, b, fa, M, N, K, fb=fb)
        exact = oracle.round_f32(ref).astype(np.float64)
        assert np.array_equal(got, exact), (kernel, fa, fb, M, N, np.argwhere(got != exact)[:5])
    assert mx.last_device_status() == 0


@pytest.mark.parametrize("kernel", KERNELS)
@pytest.mark.parametrize("out_dtype", [torch.float32, torch.bfloat16])
def test_gemm_each_kernel_tolerance_and_window(oracle, kernel, out_dtype):
    """General data on every kernel, pitched C with sentinels around the
    M x N window (nothing outside it is written)."""
    rng = np.random.default_rng(23 + kernel)
    # the resident-B kernel holds at most six K slices (MXFP4 K <= 1536)
    for (M, N, K, fmt) in [(700, 900, 1536 if kernel == 1 else 2048, "e2m1"), (264, 392, 768, "e4m3")]:
        a = (rng.standard_normal((M, K)) * np.exp2(rng.uniform(-3, 3, (M, 1)))).astype(np.float32)
        b = rng.standard_t(3, size=(N, K)).astype(np.float32)
        ac, as_ = mx.quantize(to_device(a), 1, fmt)
        bc, bs = mx.quantize(to_device(b), 1, fmt)
        ldc = (N + 7) // 8 * 8 + 24
        buf = torch.full((M + 2, ldc), -5.0, dtype=out_dtype, device=dev())
        with forced_kernel(kernel):
            mx.gemm(ac, as_, bc, bs, M, N, K, fa=fmt, alpha=0.5, out=buf[:M, :N])
        torch.cuda.synchronize()
        h = to_f64(buf)
        assert np.all(h[:M, N:] == -5.0) and np.all(h[M:, :] == -5.0), (kernel, M, N)
        f = oracle.FORMATS[fmt]
        oac, oas = oracle.quantize(a, 1, f, scale_layout=oracle.MMA)
        obc, obs = oracle.quantize(b, 1, f, scale_layout=oracle.MMA)
        ref, bound = oracle.gemm_decoded(oac, oas, f, obc, obs, f, M, N, K, alpha=0.5)
        check(h[:M, :N], ref, bound, out_dtype, (kernel, M, N, K))
    assert mx.last_device_status() == 0


@pytest.mark.parametrize("kernel", [256, 192])
def test_gemm_pair_kernels_on_llama_shape(oracle, kernel):
    """The first Llama-3 MXFP4 shape (8192 x 6144 x 4096) on both pair tile
    widths: 512 sampled rows against the oracle."""
    M, N, K = I.LLAMA3_GEMMS[0]
    x, w = I.linear_operands(M, K, N, 3, stream=0)
    rows = np.sort(np.random.default_rng(kernel).choice(M, 512, replace=False))
    with forced_kernel(kernel):
        got, ref, bound = run_gemm(oracle, x, w, "e2m1", M, N, K, out_dtype=torch.bfloat16, rows=rows)
    check(got, ref, bound, torch.bfloat16, (kernel, M, N, K))


def test_gemm_panel_kernel_refuses_long_k():
    """Forced onto the resident-B kernel, a K of more than six slices is refused."""
    z = torch.zeros(1 << 20, dtype=torch.uint8, device=dev())
    c = torch.empty((256, 256), dtype=torch.float32, device=dev())
    with forced_kernel(1):
        rc = mx.lib().mx_gemm(z.data_ptr(), z.data_ptr(), 0, z.data_ptr(), z.data_ptr(), 0, 256, 256, 1024, 1.0,
                              c.data_ptr(), 0, 256, None, 0, None)
    assert rc == -4


def test_gemm_panel_kernel_gpt2_up_projection(oracle):
    """The GPT-2 MLP up-projection shape (8192 x 3072 x 768, MXFP8), which the
    automatic choice gives to the resident-B kernel: all of C within the
    tolerance, and equal to the one-SM kernel's C bit for bit (same sums in
    the same order)."""
    M, N, K = 8192, 3072, 768
    x, w = I.linear_operands(M, K, N, 2, stream=0)
    ac, as_ = mx.quantize(to_device(x), 1, "e4m3")
    bc, bs = mx.quantize(to_device(w), 1, "e4m3")
    c_auto = mx.gemm(ac, as_, bc, bs, M, N, K, fa="e4m3", out_dtype=torch.float32)
    with forced_kernel(0):
        c_one = mx.gemm(ac, as_, bc, bs, M, N, K, fa="e4m3", out_dtype=torch.float32)
    torch.cuda.synchronize()
    assert mx.last_device_status() == 0
    assert torch.equal(c_auto.view(torch.int32), c_one.view(torch.int32))
    oac, oas = oracle.quantize(x, 1, oracle.E4M3, scale_layout=oracle.MMA)
    obc, obs = oracle.quantize(w, 1, oracle.E4M3, scale_layout=oracle.MMA)
    ref, bound = oracle.gemm_decoded(oac, oas, oracle.E4M3, obc, obs, oracle.E4M3, M, N, K)
    check(to_f64(c_auto), ref, bound, torch.float32, "gpt2 up-projection")
