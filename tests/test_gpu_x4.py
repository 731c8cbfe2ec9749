"""GPU parity of the x4 scale layout (MX_SCALES_MMA_X4: the MMA atom layout
with every 512-byte atom stored four times): the casts write it byte for byte
as the oracle does (padding bytes included: both sides start from 0xAB), the
decode reads it, and the x4 GEMM entry points (mx_gemm_x4,
mx_gemm_quantize_x4) give the MMA-layout GEMM's results bit for bit and the
oracle's within the GEMM tolerance (|C - C_ref| <= 1e-5 * |alpha| *
sum_k |a b|, + one bf16 ulp of C_ref for bf16 output)."""
import numpy as np
import pytest
import torch

from gpu_helpers import FMTS, dev, first_mismatch, host, to_device
from microscaling_block_scaled_mx_b200 import inputs as I
from microscaling_block_scaled_mx_b200 import mx
from test_gpu_cast import MASK, mixed_input
from test_gpu_gemm import check, to_f64

pytestmark = pytest.mark.gpu
X4 = 2


def gpu_cast_x4(x_np, axis, fmt, rnd="rne", seed=0, hadamard=False):
    x = to_device(x_np)
    outer, inner = (x.shape[0], x.shape[1]) if axis == 1 else (x.shape[1], x.shape[0])
    codes = torch.full((outer, mx.codes_row_bytes(fmt, inner)), 0xAB, dtype=torch.uint8, device=dev())
    scales = torch.full((mx.scales_bytes("mma_x4", outer, inner),), 0xAB, dtype=torch.uint8, device=dev())
    mx.quantize(x, axis, fmt, rnd=rnd, seed=seed, hadamard=hadamard, sign_mask=MASK, scale_layout="mma_x4",
                codes=codes, scales=scales)
    torch.cuda.synchronize()
    return host(codes), host(scales)


def oracle_cast_x4(oracle, x_np, axis, fmt, rnd="rne", seed=0, hadamard=False):
    return oracle.quantize(x_np, axis, oracle.FORMATS[fmt], rnd=1 if rnd == "sr" else 0, seed=seed,
                           hadamard=hadamard, sign_mask=MASK, scale_layout=X4, fill=0xAB)


@pytest.mark.parametrize("fmt", FMTS)
@pytest.mark.parametrize("axis", [1, 0])
def test_cast_x4_parity(oracle, fmt, axis):
    for i, (rows, cols) in enumerate([(224, 288), (64, 128), (320, 96)]):
        x = mixed_input(rows, cols, 900 + i, bf16=i % 2 == 0)
        for rnd, had in (("rne", False), ("sr", axis == 0)):
            gc, gs = gpu_cast_x4(x, axis, fmt, rnd=rnd, seed=11, hadamard=had)
            oc, os_ = oracle_cast_x4(oracle, x, axis, fmt, rnd=rnd, seed=11, hadamard=had)
            assert np.array_equal(gc, oc), (fmt, axis, rnd, first_mismatch(gc, oc))
            assert np.array_equal(gs, os_), (fmt, axis, rnd, first_mismatch(gs, os_))


@pytest.mark.parametrize("fmt", ["e4m3", "e2m1"])
def test_dual_cast_x4_parity(oracle, fmt):
    x = mixed_input(256, 160, 910, bf16=True)
    out = [torch.full((n,), 0xAB, dtype=torch.uint8, device=dev()) for n in (
        256 * mx.codes_row_bytes(fmt, 160), mx.scales_bytes("mma_x4", 256, 160),
        160 * mx.codes_row_bytes(fmt, 256), mx.scales_bytes("mma_x4", 160, 256))]
    out[0] = out[0].view(256, -1)
    out[2] = out[2].view(160, -1)
    mx.quantize_dual(to_device(x), fmt, rnd_rows="rne", rnd_cols="sr", seed_cols=7, hadamard=True,
                     scale_layout="mma_x4", out=tuple(out))
    torch.cuda.synchronize()
    ocr, osr = oracle_cast_x4(oracle, x, 1, fmt)
    occ, osc = oracle_cast_x4(oracle, x, 0, fmt, rnd="sr", seed=7, hadamard=True)
    for got, want in zip(out, (ocr, osr, occ, osc)):
        assert np.array_equal(host(got).reshape(want.shape), want), (fmt, first_mismatch(host(got).reshape(want.shape), want))


@pytest.mark.parametrize("fmt", FMTS)
def test_dequantize_x4(oracle, fmt):
    x = mixed_input(130, 224, 920, bf16=False)
    oc, os_ = oracle_cast_x4(oracle, x, 1, fmt)
    y = mx.dequantize(to_device(oc), to_device(os_), fmt, 130, 224, scale_layout="mma_x4",
                      out_dtype=torch.float32)
    torch.cuda.synchronize()
    want = oracle.round_f32(oracle.dequantize(oc, os_, oracle.FORMATS[fmt], 130, 224, X4))
    assert np.array_equal(host(y).view(np.uint32), want.view(np.uint32))


def x4_gemm_pair(oracle, a_np, b_np, fa, fb, M, N, K, alpha=1.0, out_dtype=torch.float32, ldc=None):
    """The x4 GEMM and the MMA-layout GEMM on the same operands (cast by the
    GPU in both layouts), and the oracle's reference."""
    ac, as1 = mx.quantize(to_device(a_np), 1, fa)
    bc, bs1 = mx.quantize(to_device(b_np), 1, fb)
    _, as4 = mx.quantize(to_device(a_np), 1, fa, scale_layout="mma_x4")
    _, bs4 = mx.quantize(to_device(b_np), 1, fb, scale_layout="mma_x4")

    def run(scales_a, scales_b, sl):
        if ldc is None:
            out = torch.empty((M, N), dtype=out_dtype, device=dev())
        else:
            out = torch.empty((M, ldc), dtype=out_dtype, device=dev())[:, :N]
        out.fill_(float("nan"))
        mx.gemm(ac, scales_a, bc, scales_b, M, N, K, fa=fa, fb=fb, alpha=alpha, out=out, scale_layout=sl)
        torch.cuda.synchronize()
        assert mx.last_device_status() == 0
        return out
    c4, c1 = run(as4, bs4, "mma_x4"), run(as1, bs1, "mma")
    oac, oas = oracle.quantize(a_np, 1, oracle.FORMATS[fa], scale_layout=oracle.MMA)
    obc, obs = oracle.quantize(b_np, 1, oracle.FORMATS[fb], scale_layout=oracle.MMA)
    ref, bound = oracle.gemm_decoded(oac, oas, oracle.FORMATS[fa], obc, obs, oracle.FORMATS[fb], M, N, K,
                                     alpha=alpha)
    return c4, c1, ref, bound


@pytest.mark.parametrize("fa,fb", [("e4m3", "e4m3"), ("e2m1", "e2m1"), ("e5m2", "e4m3"), ("e2m3", "e2m1"),
                                   ("e3m2", "e3m2")])
def test_gemm_x4_equals_mma_gemm(oracle, fa, fb):
    rng = np.random.default_rng(930)
    # ragged tiles; K = 384 takes the mxf8f6f4 path for FP4 x FP4 (K = 128 mod 256)
    for M, N, K in [(300, 200, 512), (100, 520, 384), (512, 256, 1024)]:
        a = (rng.standard_normal((M, K)) * np.exp2(rng.uniform(-6, 6, (M, 1)))).astype(np.float32)
        b = (rng.standard_normal((N, K)) * 0.02).astype(np.float32)
        for out_dtype in (torch.float32, torch.bfloat16):
            c4, c1, ref, bound = x4_gemm_pair(oracle, a, b, fa, fb, M, N, K, alpha=0.75, out_dtype=out_dtype)
            assert torch.equal(c4.view(torch.int16 if out_dtype == torch.bfloat16 else torch.int32),
                               c1.view(torch.int16 if out_dtype == torch.bfloat16 else torch.int32)), (fa, fb, M, N, K)
            check(to_f64(c4), ref, bound, out_dtype, (fa, fb, M, N, K))


def test_gemm_x4_exact_and_strided(oracle):
    """Small-integer operands: every partial sum exact, so C is the oracle's bit for bit."""
    rng = np.random.default_rng(931)
    M, N, K = 260, 136, 768
    a = rng.integers(-4, 5, (M, K)).astype(np.float32)
    b = rng.integers(-4, 5, (N, K)).astype(np.float32)
    c4, c1, ref, bound = x4_gemm_pair(oracle, a, b, "e4m3", "e4m3", M, N, K, ldc=N + 8)
    assert np.array_equal(to_f64(c4), ref)


def test_gemm_quantize_x4_chain(oracle):
    """The quantizing epilogue on x4 operands writes C's codes and x4 scales,
    equal to mx_gemm_quantize's (MMA-layout operands, x4 output)."""
    rng = np.random.default_rng(932)
    M, N, K = 256, 512, 512
    a = rng.integers(-3, 4, (M, K)).astype(np.float32)
    b = rng.integers(-3, 4, (N, K)).astype(np.float32)
    ac, as1 = mx.quantize(to_device(a), 1, "e4m3")
    bc, bs1 = mx.quantize(to_device(b), 1, "e4m3")
    _, as4 = mx.quantize(to_device(a), 1, "e4m3", scale_layout="mma_x4")
    _, bs4 = mx.quantize(to_device(b), 1, "e4m3", scale_layout="mma_x4")
    q4 = mx.gemm_quantize(ac, as4, bc, bs4, M, N, K, fa="e4m3", out_fmt="e2m1", scale_layout="mma_x4",
                          operand_layout="mma_x4")
    q1 = mx.gemm_quantize(ac, as1, bc, bs1, M, N, K, fa="e4m3", out_fmt="e2m1", scale_layout="mma_x4")
    torch.cuda.synchronize()
    assert torch.equal(q4[0], q1[0])
    # compare the written copies (padding is never written)
    c = oracle.round_f32(oracle.gemm(*oracle.quantize(a, 1, oracle.E4M3, scale_layout=oracle.MMA),
                                     oracle.E4M3, *oracle.quantize(b, 1, oracle.E4M3, scale_layout=oracle.MMA),
                                     oracle.E4M3, M, N, K)[0])
    oc, os_ = oracle.quantize(c, 1, oracle.E2M1, scale_layout=X4, fill=0xAB)
    s4 = host(q4[1])
    written = os_ != 0xAB
    assert np.array_equal(host(q4[0]), oc)
    assert np.array_equal(s4[written], os_[written]) and np.array_equal(host(q1[1])[written], os_[written])


def test_gemm_x4_llama_shape_rows(oracle):
    """Llama-3-8B 8192 x 6144 x 4096 MXFP4 on x4 scales, 512 rows from four row tiles."""
    M, N, K = 8192, 6144, 4096
    x, w = I.linear_operands(M, K, N, 3, stream=0)
    ac, _ = mx.quantize(to_device(x), 1, "e2m1")
    bc, _ = mx.quantize(to_device(w), 1, "e2m1")
    _, as4 = mx.quantize(to_device(x), 1, "e2m1", scale_layout="mma_x4")
    _, bs4 = mx.quantize(to_device(w), 1, "e2m1", scale_layout="mma_x4")
    c = mx.gemm(ac, as4, bc, bs4, M, N, K, fa="e2m1", out_dtype=torch.bfloat16, scale_layout="mma_x4")
    torch.cuda.synchronize()
    rows = np.concatenate([np.arange(0, 128), np.arange(2048, 2176), np.arange(5000, 5128), np.arange(M - 128, M)])
    oac, oas = oracle.quantize(x, 1, oracle.E2M1, scale_layout=oracle.MMA)
    obc, obs = oracle.quantize(w, 1, oracle.E2M1, scale_layout=oracle.MMA)
    ref, bound = oracle.gemm_decoded(oac, oas, oracle.E2M1, obc, obs, oracle.E2M1, M, N, K, rows=rows)
    check(to_f64(c)[rows], ref, bound, torch.bfloat16, "llama x4")


def test_gemm_x4_force_hook():
    """Only the pair kernel takes x4 scales: forcing another one is refused."""
    L = mx.lib()
    z = torch.zeros(1 << 16, dtype=torch.uint8, device=dev())
    c = torch.empty((256, 256), dtype=torch.float32, device=dev())
    try:
        for kern, want in ((0, -4), (192, -4)):
            assert L.mx_debug_gemm_force_kernel(kern) == 0
            rc = L.mx_gemm_x4(z.data_ptr(), z.data_ptr(), 0, z.data_ptr(), z.data_ptr(), 0, 256, 256, 256, 1.0,
                              c.data_ptr(), 0, 256, None)
            assert rc == want, (kern, rc)
    finally:
        L.mx_debug_gemm_force_kernel(-1)


@pytest.mark.parametrize("domain_rows", [0, 32])
def test_nvfp4_x4_cast_and_gemm(oracle, domain_rows):
    """NVFP4 with x4 block scales: the cast writes the oracle's bytes and the
    x4 GEMM equals the MMA-layout NVFP4 GEMM bit for bit."""
    rng = np.random.default_rng(940 + domain_rows)
    M, N, K = 300, 264, 768
    a = (rng.standard_normal((M, K)) * np.exp2(rng.uniform(-6, 6, (M, 1)))).astype(np.float32)
    b = (rng.standard_normal((N, K)) * 0.02).astype(np.float32)
    a4 = mx.quantize_nvfp4(to_device(a), domain_rows, scale_layout="mma_x4")
    b4 = mx.quantize_nvfp4(to_device(b), 0, scale_layout="mma_x4")
    a1 = mx.quantize_nvfp4(to_device(a), domain_rows)
    b1 = mx.quantize_nvfp4(to_device(b), 0)
    torch.cuda.synchronize()
    oc, os_, oe = oracle.nvfp4_quantize(a, domain_rows, scale_layout=X4, fill=0xAB)
    written = os_ != 0xAB
    assert np.array_equal(host(a4[0]), oc)
    assert np.array_equal(host(a4[1])[written], os_[written])
    for out_dtype in (torch.float32, torch.bfloat16):
        c4 = mx.gemm_nvfp4(a4, b4, M, N, K, domain_rows, 0, alpha=0.5, out_dtype=out_dtype, scale_layout="mma_x4")
        c1 = mx.gemm_nvfp4(a1, b1, M, N, K, domain_rows, 0, alpha=0.5, out_dtype=out_dtype)
        torch.cuda.synchronize()
        assert mx.last_device_status() == 0
        iv = torch.int16 if out_dtype == torch.bfloat16 else torch.int32
        assert torch.equal(c4.view(iv), c1.view(iv)), (domain_rows, out_dtype)
