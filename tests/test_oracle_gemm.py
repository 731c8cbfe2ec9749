"""Pins for the oracle's block-scaled GEMM.

Compute flow ("Microscaling Data Formats for Deep Learning", summary page,
section 4): dot products take MX-quantized inputs and return scalar floats.
The oracle decodes every element exactly and sums in fp64; here that sum is
checked against numpy's fp64 matmul of matrices decoded by the independent
decoder (the special case that reduces to a library routine), on inputs where
every partial sum is exact so equality must be bitwise.
"""
import numpy as np
import pytest

import mx_independent as ind

NAMES = ind.FMT_NAMES


def fid(name):
    return NAMES.index(name)


def _decode_full(name, codes, scales_mma, outer, inner):
    un = ind.unpack_codes(name, codes, inner)
    perm = ind.mma_scale_permutation(outer, inner // 32)
    s = scales_mma[perm].astype(np.float64)
    return ind.decode(name, un) * np.exp2(np.repeat(s - 127, 32, axis=1))


@pytest.mark.parametrize("fa,fb", [("e4m3", "e4m3"), ("e2m1", "e2m1"), ("e5m2", "e4m3"),
                                   ("e3m2", "e2m1"), ("e2m3", "e2m3")])
@pytest.mark.parametrize("M,N,K", [(128, 128, 32), (128, 256, 64), (256, 128, 128), (40, 24, 96)])
def test_gemm_equals_decoded_matmul(oracle, fa, fb, M, N, K):
    rng = np.random.default_rng(M * 7 + N * 3 + K)
    # small-exponent inputs so that every product and partial sum is exact in fp64
    a = (rng.integers(-8, 9, (M, K)) * np.exp2(rng.integers(-3, 4, (M, 1)))).astype(np.float32)
    b = (rng.integers(-8, 9, (N, K)) * np.exp2(rng.integers(-3, 4, (N, 1)))).astype(np.float32)
    ac, as_ = oracle.quantize(a, 1, fid(fa), scale_layout=1)
    bc, bs = oracle.quantize(b, 1, fid(fb), scale_layout=1)
    A = _decode_full(fa, ac, as_, M, K)
    B = _decode_full(fb, bc, bs, N, K)
    c, bound = oracle.gemm(ac, as_, fid(fa), bc, bs, fid(fb), M, N, K, alpha=1.0)
    np.testing.assert_array_equal(c, A @ B.T)
    np.testing.assert_array_equal(bound, np.abs(A) @ np.abs(B).T)
    c2, bound2 = oracle.gemm(ac, as_, fid(fa), bc, bs, fid(fb), M, N, K, alpha=-0.25)
    np.testing.assert_array_equal(c2, -0.25 * (A @ B.T))
    np.testing.assert_array_equal(bound2, 0.25 * bound)


def test_gemm_entries_match_full(oracle):
    rng = np.random.default_rng(3)
    M, N, K = 64, 48, 256
    a = rng.standard_normal((M, K)).astype(np.float32)
    b = rng.standard_normal((N, K)).astype(np.float32)
    ac, as_ = oracle.quantize(a, 1, fid("e2m1"), scale_layout=1)
    bc, bs = oracle.quantize(b, 1, fid("e2m1"), scale_layout=1)
    c, bound = oracle.gemm(ac, as_, 4, bc, bs, 4, M, N, K, alpha=0.5)
    ms = rng.integers(0, M, 50)
    ns = rng.integers(0, N, 50)
    ce, be = oracle.gemm_entries(ac, as_, 4, bc, bs, 4, K, ms, ns, alpha=0.5)
    np.testing.assert_array_equal(ce, c[ms, ns])
    np.testing.assert_array_equal(be, bound[ms, ns])
    assert np.all(np.abs(c) <= bound)


def test_gemm_plain_and_mma_layouts_agree(oracle):
    rng = np.random.default_rng(5)
    M, N, K = 130, 70, 160
    a = rng.standard_normal((M, K)).astype(np.float32)
    b = rng.standard_normal((N, K)).astype(np.float32)
    res = []
    for sl in (0, 1, 2):                      # plain, MMA, MMA x4
        ac, as_ = oracle.quantize(a, 1, 0, scale_layout=sl)
        bc, bs = oracle.quantize(b, 1, 0, scale_layout=sl)
        res.append(oracle.gemm(ac, as_, 0, bc, bs, 0, M, N, K, scale_layout=sl)[0])
    np.testing.assert_array_equal(res[0], res[1])
    np.testing.assert_array_equal(res[0], res[2])


def test_gemm_random_close_to_fp64_of_inputs(oracle):
    """MX GEMM approximates the unquantized product (sanity on the whole chain)."""
    rng = np.random.default_rng(7)
    M, N, K = 32, 32, 512
    a = rng.standard_normal((M, K)).astype(np.float32)
    b = rng.standard_normal((N, K)).astype(np.float32)
    ac, as_ = oracle.quantize(a, 1, 0, scale_layout=1)
    bc, bs = oracle.quantize(b, 1, 0, scale_layout=1)
    c, bound = oracle.gemm(ac, as_, 0, bc, bs, 0, M, N, K)
    exact = a.astype(np.float64) @ b.astype(np.float64).T
    # E4M3 relative element error <= 2^-4, so |C - exact| <= ~2^-3 * sum|ab|
    assert np.all(np.abs(c - exact) <= 0.13 * bound)


def test_gemm_decoded_matches_scalar_loop(oracle):
    """The matmul route used for large shapes agrees with the scalar oracle."""
    rng = np.random.default_rng(9)
    M, N, K = 96, 80, 512
    a = (rng.standard_normal((M, K)) * np.exp2(rng.integers(-20, 20, (M, 1)))).astype(np.float32)
    b = rng.standard_t(3, size=(N, K)).astype(np.float32)
    for f in (0, 1, 4):
        ac, as_ = oracle.quantize(a, 1, f, scale_layout=1)
        bc, bs = oracle.quantize(b, 1, f, scale_layout=1)
        c1, b1 = oracle.gemm(ac, as_, f, bc, bs, f, M, N, K, alpha=0.03125)
        c2, b2 = oracle.gemm_decoded(ac, as_, f, bc, bs, f, M, N, K, alpha=0.03125)
        np.testing.assert_allclose(c2, c1, rtol=0, atol=1e-12 * b1.max())
        np.testing.assert_allclose(b2, b1, rtol=1e-12)
        rows = [3, 50, 95]
        c3, _ = oracle.gemm_decoded(ac, as_, f, bc, bs, f, M, N, K, alpha=0.03125, rows=rows)
        np.testing.assert_array_equal(c3, c2[rows])
