"""GPU parity of the GEMM with a quantizing epilogue: C = alpha * A * B^T
("Microscaling Data Formats for Deep Learning", summary page, section 4)
written as MX codes and scales along C's rows (Algorithm 1, section 3), the
layout the next GEMM reads (the FP4-pretraining abstract's producer writing
its consumer's layout).

Where every partial sum of the GEMM is exact in fp32 (small integers times
powers of two, alpha a power of two), the fp32 C the epilogue quantizes is
the exact C, so codes and scales must equal, bit for bit, the oracle's cast
of round_f32(alpha * C_exact).  On general inputs the accumulator differs from
the exact sum by up to the GEMM tolerance (1e-5 * |alpha| * sum_k |a b|), so
the checks there are the error bound of the quantization plus that tolerance,
and equal scales away from power-of-two boundaries.
"""
import numpy as np
import pytest
import torch

from gpu_helpers import FMTS, dev, first_mismatch, host, to_device
from microscaling_block_scaled_mx_b200 import mx

pytestmark = pytest.mark.gpu

FILL = 0xAB
REL_TOL = 1e-5
EMAX = {"e4m3": 8, "e5m2": 15, "e2m3": 2, "e3m2": 4, "e2m1": 2, "int8": 0}
MBITS = {"e4m3": 3, "e5m2": 2, "e2m3": 3, "e3m2": 2, "e2m1": 1, "int8": 6}
MAXV = {"e4m3": 448.0, "e5m2": 57344.0, "e2m3": 7.5, "e3m2": 28.0, "e2m1": 6.0, "int8": 127 / 64}


def small_int_operand(rng, rows, K):
    """Integers in [-3, 3] times a power of two per 32-block: on every element
    grid, and every product and partial sum is exact in fp32."""
    v = rng.integers(-3, 4, (rows, K)).astype(np.float64)
    v *= np.exp2(np.repeat(rng.integers(-2, 3, (rows, K // 32)), 32, axis=1))
    return v.astype(np.float32)


def operands(oracle, a, b, fa, fb):
    """GPU casts of the operands along K, and the oracle's casts of the same data."""
    ga = mx.quantize(to_device(a), 1, fa)
    gb = mx.quantize(to_device(b), 1, fb)
    oa = oracle.quantize(a, 1, oracle.FORMATS[fa], scale_layout=oracle.MMA)
    ob = oracle.quantize(b, 1, oracle.FORMATS[fb], scale_layout=oracle.MMA)
    return ga, gb, oa, ob


def gpu_gemm_quant(ga, gb, M, N, K, fa, fb, alpha, out_fmt, rnd, seed, sl):
    codes = torch.full((M, mx.codes_row_bytes(out_fmt, N)), FILL, dtype=torch.uint8, device=dev())
    scales = torch.full((max(mx.scales_bytes(sl, M, N), 1),), FILL, dtype=torch.uint8, device=dev())
    mx.gemm_quantize(ga[0], ga[1], gb[0], gb[1], M, N, K, fa=fa, fb=fb, alpha=alpha, out_fmt=out_fmt,
                     rnd=rnd, seed=seed, scale_layout=sl, out=(codes, scales))
    torch.cuda.synchronize()
    assert mx.last_device_status() == 0
    return host(codes), host(scales)


def oracle_c(oracle, oa, ob, fa, fb, M, N, K, alpha):
    f, g = oracle.FORMATS[fa], oracle.FORMATS[fb]
    return oracle.gemm_decoded(oa[0], oa[1], f, ob[0], ob[1], g, M, N, K, alpha=alpha)


def oracle_quant(oracle, c32, out_fmt, rnd, seed, sl):
    return oracle.quantize(c32, 1, oracle.FORMATS[out_fmt], rnd=1 if rnd == "sr" else 0, seed=seed,
                           scale_layout=1 if sl == "mma" else 0, fill=FILL)


def assert_same(got, want, what):
    (gc, gs), (wc, ws) = got, want
    assert gc.shape == wc.shape, (what, gc.shape, wc.shape)
    assert np.array_equal(gs[:ws.size], ws), (what, "scales", first_mismatch(gs[:ws.size], ws))
    assert np.array_equal(gc, wc), (what, "codes", first_mismatch(gc, wc))


@pytest.mark.parametrize("fa,fb", [("e4m3", "e4m3"), ("e2m1", "e2m1"), ("e2m1", "e3m2")])
@pytest.mark.parametrize("rnd", ["rne", "sr"])
def test_gemm_quantize_bit_exact_one_sm(oracle, fa, fb, rnd):
    """Short K: the one-SM kernel (128 x 192 tiles, odd tiles included); every
    output format and both scale layouts."""
    M, N, K = 256, 384, 256
    rng = np.random.default_rng(500)
    ga, gb, oa, ob = operands(oracle, small_int_operand(rng, M, K), small_int_operand(rng, N, K), fa, fb)
    ref, _ = oracle_c(oracle, oa, ob, fa, fb, M, N, K, 0.5)
    c32 = oracle.round_f32(ref)
    for out_fmt in FMTS:
        for sl in ("mma", "plain"):
            got = gpu_gemm_quant(ga, gb, M, N, K, fa, fb, 0.5, out_fmt, rnd, 7, sl)
            assert_same(got, oracle_quant(oracle, c32, out_fmt, rnd, 7, sl), (fa, fb, out_fmt, rnd, sl))


@pytest.mark.parametrize("fa,fb,out_fmt", [("e2m1", "e2m1", "e2m1"), ("e4m3", "e4m3", "e4m3"),
                                           ("e2m1", "e3m2", "e3m2")])
def test_gemm_quantize_bit_exact_two_sm(oracle, fa, fb, out_fmt):
    """Pair-kernel shapes (K >= 2048, >= 148 tiles of 256 x 256), one ragged in M."""
    K = 2048
    for (M, N) in [(4096, 2560), (4000, 2592)]:
        rng = np.random.default_rng(M + N + 5)
        ga, gb, oa, ob = operands(oracle, small_int_operand(rng, M, K), small_int_operand(rng, N, K), fa, fb)
        ref, _ = oracle_c(oracle, oa, ob, fa, fb, M, N, K, 0.25)
        got = gpu_gemm_quant(ga, gb, M, N, K, fa, fb, 0.25, out_fmt, "rne", 0, "mma")
        assert_same(got, oracle_quant(oracle, oracle.round_f32(ref), out_fmt, "rne", 0, "mma"), (M, N, out_fmt))


def block_error_bound(out_fmt, X, rnd):
    """Largest |decode(code) - c| for a block with scale X: half a grid step of
    the top binade (a full step for SR), or the clamp of values between max
    and 2^(emax + 1)."""
    e, m = EMAX[out_fmt], MBITS[out_fmt]
    step = 2.0 ** (e - m) if out_fmt != "int8" else 2.0 ** -6
    return X * max(step if rnd == "sr" else step / 2, 2.0 ** (e + 1) - MAXV[out_fmt])


@pytest.mark.parametrize("out_fmt", FMTS)
@pytest.mark.parametrize("rnd", ["rne", "sr"])
def test_gemm_quantize_general_inputs(oracle, out_fmt, rnd):
    """Normal / Student-t data with row scales spread over 2^+-4: decoded codes
    within the quantization bound plus the GEMM tolerance of the exact C, and
    the GPU's scales equal to the oracle's except for blocks whose amax lies
    within the GEMM tolerance of a power of two."""
    M, N, K = 384, 768, 1024
    rng = np.random.default_rng(501)
    a = (rng.standard_normal((M, K)) * np.exp2(rng.uniform(-4, 4, (M, 1)))).astype(np.float32)
    b = rng.standard_t(3, size=(N, K)).astype(np.float32)
    ga, gb, oa, ob = operands(oracle, a, b, "e4m3", "e4m3")
    alpha = 0.75
    ref, bound = oracle_c(oracle, oa, ob, "e4m3", "e4m3", M, N, K, alpha)
    gc, gs = gpu_gemm_quant(ga, gb, M, N, K, "e4m3", "e4m3", alpha, out_fmt, rnd, 3, "plain")
    dec = oracle.dequantize(gc, gs, oracle.FORMATS[out_fmt], M, N, oracle.PLAIN)
    tol = REL_TOL * bound
    X = np.exp2(gs.reshape(M, N // 32).astype(np.float64) - 127)
    err_bound = np.repeat(block_error_bound(out_fmt, X, rnd), 32, axis=1) + tol
    err = np.abs(dec - ref)
    assert np.all(err <= err_bound), (out_fmt, rnd, int((err > err_bound).sum()))
    # scales: the oracle's cast of the exact C, up to boundary blocks
    _, ws = oracle_quant(oracle, oracle.round_f32(ref), out_fmt, rnd, 3, "plain")
    ws = ws.reshape(M, N // 32)
    gs = gs.reshape(M, N // 32)
    amax = np.maximum(np.abs(ref).reshape(M, N // 32, 32).max(axis=2), 1e-300)
    tmax = tol.reshape(M, N // 32, 32).max(axis=2)
    near = np.abs(amax - np.exp2(np.round(np.log2(amax)))) <= 2 * tmax
    diff = gs != ws
    assert not np.any(diff & ~near), (out_fmt, rnd, int((diff & ~near).sum()))
    assert np.all(np.abs(gs.astype(int) - ws.astype(int)) <= 1)


def test_gemm_quantize_feeds_next_gemm(oracle):
    """C1 = X W1^T written as E4M3 codes + MMA-layout scales by the epilogue is
    consumed directly as the A operand of C2 = C1 W2^T (K2 = N1)."""
    M, K1, N1, N2 = 512, 256, 384, 256
    rng = np.random.default_rng(502)
    ga, gb, oa, ob = operands(oracle, small_int_operand(rng, M, K1), small_int_operand(rng, N1, K1), "e4m3", "e4m3")
    c1_codes, c1_scales = mx.gemm_quantize(ga[0], ga[1], gb[0], gb[1], M, N1, K1, fa="e4m3", alpha=0.5,
                                           out_fmt="e4m3")
    w2 = rng.standard_normal((N2, N1)).astype(np.float32)
    g2 = mx.quantize(to_device(w2), 1, "e4m3")
    c2 = mx.gemm(c1_codes, c1_scales, g2[0], g2[1], M, N2, N1, fa="e4m3", out_dtype=torch.float32)
    torch.cuda.synchronize()
    # oracle: exact C1 (exact regime), its cast, then the second GEMM
    ref1, _ = oracle_c(oracle, oa, ob, "e4m3", "e4m3", M, N1, K1, 0.5)
    q1 = oracle.quantize(oracle.round_f32(ref1), 1, oracle.FORMATS["e4m3"], scale_layout=oracle.MMA)
    assert np.array_equal(host(c1_codes), q1[0]) and np.array_equal(host(c1_scales), q1[1])
    o2 = oracle.quantize(w2, 1, oracle.FORMATS["e4m3"], scale_layout=oracle.MMA)
    ref2, bound2 = oracle.gemm_decoded(q1[0], q1[1], 0, o2[0], o2[1], 0, M, N2, N1)
    got = host(c2).astype(np.float64)
    assert np.all(np.abs(got - ref2) <= REL_TOL * bound2)


def test_gemm_quantize_k_zero_empty_and_shape():
    z = torch.empty(0, dtype=torch.uint8, device=dev())
    codes = torch.full((4, 64), FILL, dtype=torch.uint8, device=dev())
    scales = torch.full((mx.scales_bytes("mma", 4, 64),), FILL, dtype=torch.uint8, device=dev())
    mx.gemm_quantize(z, z, z, z, 4, 64, 0, out_fmt="e4m3", out=(codes, scales))
    torch.cuda.synchronize()
    assert torch.all(codes == 0) and torch.all(scales == 0)
    mx.gemm_quantize(z, z, z, z, 0, 64, 128, out_fmt="e4m3", out=(z, z))
    with pytest.raises(mx.MxError, match="MX_ERR_SHAPE"):
        mx.gemm_quantize(z, z, z, z, 4, 48, 128, out_fmt="e4m3", out=(codes, scales))


@pytest.mark.parametrize("kernel", [0, 1, 256, 192])
@pytest.mark.parametrize("out_fmt", ["e4m3", "e2m1", "e3m2", "int8"])
def test_gemm_quantize_each_kernel_bit_exact(oracle, kernel, out_fmt):
    """The quantizing epilogue on every kernel (forced with
    mx_debug_gemm_force_kernel), exact partial sums: codes and scales equal
    the oracle's cast of the exact C, ragged M and several N tiles."""
    M, N, K = 520, 640, 512
    rng = np.random.default_rng(kernel + len(out_fmt))
    a = np.clip(small_int_operand(rng, M, K), -3, 3)
    b = np.clip(small_int_operand(rng, N, K), -3, 3)
    ga, gb, oa, ob = operands(oracle, a, b, "e4m3", "e4m3")
    c, _ = oracle_c(oracle, oa, ob, "e4m3", "e4m3", M, N, K, 0.25)
    c32 = oracle.round_f32(c)
    assert mx.lib().mx_debug_gemm_force_kernel(kernel) == 0
    try:
        got = gpu_gemm_quant(ga, gb, M, N, K, "e4m3", "e4m3", 0.25, out_fmt, "sr", 11, "mma")
    finally:
        mx.lib().mx_debug_gemm_force_kernel(-1)
    assert_same(got, oracle_quant(oracle, c32, out_fmt, "sr", 11, "mma"), (kernel, out_fmt))
