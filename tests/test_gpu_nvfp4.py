"""GPU parity of the NVFP4 cast (mx_quantize_nvfp4): the global and the
CTA-local scale domains the abstract of "Format-Aware Fusion for Fast FP4
Pretraining" names, in the reading stated in include/mx.h (16-element E2M1
blocks, E4M3 block scales, one fp32 encode scale per domain).  Every step is
one IEEE fp32 operation, so codes, block scales and domain scales must equal
the oracle's byte for byte."""
import numpy as np
import pytest
import torch

import mx_independent as ind
from gpu_helpers import dev, first_mismatch, host, to_device
from microscaling_block_scaled_mx_b200 import inputs as I
from microscaling_block_scaled_mx_b200 import mx

pytestmark = pytest.mark.gpu


def special_input(rows, cols, seed, bf16):
    rng = np.random.default_rng(seed)
    x = (rng.standard_normal((rows, cols)) * np.exp2(rng.uniform(-6, 6, (rows, 1)))).astype(np.float32)
    flat = x.reshape(-1)
    flat[rng.choice(flat.size, flat.size // 50, replace=False)] = 0.0
    sub = rng.choice(flat.size, flat.size // 200, replace=False)
    flat[sub] = (rng.integers(1, 1 << 23, sub.size).astype(np.uint32)
                 | (rng.integers(0, 2, sub.size).astype(np.uint32) << 31)).view(np.float32)
    x[3, 17 % cols] = np.nan
    x[5, 40 % cols] = np.inf
    x[7, :] = 0.0
    return ind.f32_to_bf16_bits_rne(x) if bf16 else x


def check(x_np, domain_rows, sl, what):
    rows, cols = x_np.shape
    codes, scales, enc = mx.quantize_nvfp4(to_device(x_np), domain_rows, scale_layout=sl)
    torch.cuda.synchronize()
    assert mx.last_device_status() == 0
    import oracle
    oc, os_, oe = oracle.nvfp4_quantize(x_np, domain_rows, scale_layout=oracle.MMA if sl == "mma" else oracle.PLAIN)
    assert np.array_equal(host(enc).view(np.uint32)[:oe.size], oe.view(np.uint32)), (what, host(enc)[:8], oe[:8])
    assert np.array_equal(host(codes), oc), (what, first_mismatch(host(codes), oc))
    if sl == "mma":            # padding bytes of the atom layout are never written
        keep = oc.shape[0]
        perm = ind.mma_scale_permutation(keep, cols // 16).reshape(-1)
        assert np.array_equal(host(scales)[perm], os_[perm]), what
    else:
        assert np.array_equal(host(scales), os_), (what, first_mismatch(host(scales), os_))


@pytest.mark.parametrize("bf16", [True, False])
@pytest.mark.parametrize("domain_rows", [0, 32, 7])
@pytest.mark.parametrize("sl", ["plain", "mma"])
def test_nvfp4_cast_parity(oracle, bf16, domain_rows, sl):
    for i, (rows, cols) in enumerate([(100, 256), (256, 4096), (33, 16)]):
        check(special_input(rows, cols, 50 + i, bf16), domain_rows, sl, (bf16, domain_rows, sl, rows, cols))


@pytest.mark.parametrize("domain_rows", [0, 32])
def test_nvfp4_cast_llama_activation(oracle, domain_rows):
    """A Llama-3-8B activation, 8192 x 4096 bf16 N(0,1)."""
    x, _ = I.linear_operands(8192, 4096, 128, 3, stream=0)
    check(x, domain_rows, "mma", ("llama", domain_rows))


# ---------------------------------------------------------------------------
# GEMM on NVFP4 operands (mx_gemm_nvfp4).  Tolerance as for the MX GEMM:
# |C - C_ref| <= 1e-5 * |alpha| * sum_k |a_mk b_nk| (+ one bf16 ulp of C_ref
# for bf16 output), C_ref the fp64 product of the oracle's exact decodes.

def gemm_check(oracle, a_np, b_np, a_lines, b_lines, out_dtype, alpha=1.0, ldc=None, rows=None):
    from test_gpu_gemm import check, to_f64
    M, K = a_np.shape
    N = b_np.shape[0]
    a = mx.quantize_nvfp4(to_device(a_np), a_lines)
    b = mx.quantize_nvfp4(to_device(b_np), b_lines)
    if ldc is None:
        out = torch.empty((M, N), dtype=out_dtype, device=dev())
    else:
        out = torch.empty((M, ldc), dtype=out_dtype, device=dev())[:, :N]
    out.fill_(float("nan"))
    mx.gemm_nvfp4(a, b, M, N, K, a_lines, b_lines, alpha=alpha, out=out)
    torch.cuda.synchronize()
    assert mx.last_device_status() == 0
    oa = oracle.nvfp4_quantize(a_np, a_lines, scale_layout=oracle.MMA)
    ob = oracle.nvfp4_quantize(b_np, b_lines, scale_layout=oracle.MMA)
    # the operands the GPU multiplied are the oracle's, byte for byte
    assert np.array_equal(host(a[0]), oa[0]) and np.array_equal(host(b[0]), ob[0])
    assert np.array_equal(host(a[2]).view(np.uint32)[:oa[2].size], oa[2].view(np.uint32))
    ref, bound = oracle.nvfp4_gemm_decoded(oa, ob, M, N, K, alpha=alpha, a_lines=a_lines, b_lines=b_lines,
                                           rows=rows)
    got = to_f64(out)
    if rows is not None:
        got = got[np.asarray(rows)]
    check(got, ref, bound, out_dtype, (M, N, K, a_lines, b_lines))


def spread_input(rows, cols, seed):
    """N(0,1) rows with per-row magnitudes over 2^-8..2^8, so that domains and
    blocks get different scales."""
    rng = np.random.default_rng(seed)
    return (rng.standard_normal((rows, cols)) * np.exp2(rng.uniform(-8, 8, (rows, 1)))).astype(np.float32)


@pytest.mark.parametrize("out_dtype", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("a_lines,b_lines", [(0, 0), (32, 32), (7, 64), (128, 0)])
def test_nvfp4_gemm_parity(oracle, out_dtype, a_lines, b_lines):
    # ragged M and N over several 256 x 256 tiles, K over several stages
    for i, (M, N, K) in enumerate([(300, 200, 512), (600, 520, 1024), (64, 32, 256)]):
        a = spread_input(M, K, 70 + i)
        b = spread_input(N, K, 80 + i)
        gemm_check(oracle, a, b, a_lines, b_lines, out_dtype, alpha=0.75)


def test_nvfp4_gemm_strided_c_and_bf16_input(oracle):
    M, N, K = 260, 136, 768
    a = ind.f32_to_bf16_bits_rne(spread_input(M, K, 90))
    b = ind.f32_to_bf16_bits_rne(spread_input(N, K, 91))
    gemm_check(oracle, a, b, 32, 32, torch.float32, ldc=N + 8)
    gemm_check(oracle, a, b, 0, 0, torch.bfloat16, ldc=N + 24)


def test_nvfp4_gemm_zero_domain(oracle):
    """A domain of zeros (E = 1, every block scale 0) next to ordinary ones."""
    M, N, K = 256, 256, 512
    a = spread_input(M, K, 92)
    a[32:64] = 0.0
    b = spread_input(N, K, 93)
    b[64:96] = 0.0
    gemm_check(oracle, a, b, 32, 32, torch.float32)


@pytest.mark.parametrize("a_lines,b_lines", [(0, 0), (128, 128)])
def test_nvfp4_gemm_llama_shape(oracle, a_lines, b_lines):
    """Llama-3-8B attention-output shape 8192 x 4096 x 4096 in the launch
    configuration the benchmark uses, checked on 512 rows from four row
    tiles (first, two middle, last)."""
    M, N, K = 8192, 4096, 4096
    x, w = I.linear_operands(M, K, N, 5, stream=0)
    rows = np.concatenate([np.arange(0, 128), np.arange(2048, 2176), np.arange(5000, 5128),
                           np.arange(M - 128, M)])
    gemm_check(oracle, x, w, a_lines, b_lines, torch.bfloat16, rows=rows)
