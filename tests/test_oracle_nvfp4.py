"""Pins of the oracle's NVFP4 cast (the "global" and "cooperative-thread-array-
local" NVFP4 scale domains the FP4 pretraining abstract names; reading in
oracle/mx_oracle.c: 16-element E2M1 blocks, an E4M3 block scale, one fp32
encode scale E = 2688 / amax per domain).

Pins, each independent of the oracle's own arithmetic:
  * exact reconstruction: tensors built as P * d / E from chosen E2M1 codes
    P, E4M3 block scales d and a power-of-two E (one block per domain
    holding the 448 scale and a +-6 code, so that E is recovered exactly)
    cast back to exactly those codes, scales and E;
  * the block scale is torch's float8_e4m3fn rounding of (amax / 6) * E
    (in range), and the domain maximum's block gets the 448 code;
  * the decode is an independent numpy decode of the codes and scales;
  * non-finite blocks and all-zero domains;
  * the GEMM reference equals numpy's fp64 product of the decoded operands.
"""
from __future__ import annotations

import numpy as np
import pytest
import torch

import mx_independent as ind


def build_exact(rng, rows, cols, lines, e_pow):
    """Codes, block scales and per-domain E = 2^e_pow[d]; returns x (fp32) and
    the expected codes (E2M1, unpacked), scale codes (plain) and E."""
    kb = cols // 16
    codes = rng.integers(0, 16, (rows, cols))
    scales = rng.integers(0x10, 0x7E, (rows, kb))          # normal positive E4M3 codes below 448
    # every block holds a +-6 (E2M1 codes 0x7 / 0xF)
    for r in range(rows):
        for b in range(kb):
            codes[r, b * 16 + rng.integers(16)] = 0x7 | (rng.integers(2) << 3)
    n_dom = 1 if lines == 0 else (rows + lines - 1) // lines
    L = rows if lines == 0 else lines
    for d in range(n_dom):                                    # the domain maximum: scale 448, code 6
        r = d * L + rng.integers(min(L, rows - d * L))
        scales[r, rng.integers(kb)] = 0x7E
    E = np.exp2(np.asarray(e_pow, dtype=np.float64))[:n_dom]
    P = ind.decode("e2m1", codes)
    D = ind.decode("e4m3", np.repeat(scales, 16, axis=1))
    dom = np.arange(rows) // L
    x = (P * D / E[dom][:, None]).astype(np.float32)
    assert np.all(x.astype(np.float64) == P * D / E[dom][:, None])   # exactly representable
    return x, codes, scales, E.astype(np.float32)


@pytest.mark.parametrize("lines", [0, 32])
def test_exact_reconstruction(oracle, lines):
    rng = np.random.default_rng(11 + lines)
    rows, cols = 96, 128
    x, codes, scales, E = build_exact(rng, rows, cols, lines, [-3, 2, 5])
    c, s, e = oracle.nvfp4_quantize(x, lines)
    assert np.array_equal(e, E)
    assert np.array_equal(ind.unpack_codes("e2m1", c, cols), codes)
    assert np.array_equal(s.reshape(rows, cols // 16), scales)


def test_block_scale_is_e4m3_rounding(oracle):
    """In-range block scales equal torch's float8_e4m3fn rounding of
    (amax / 6) * E computed in fp32, and the domain maximum's block is 448."""
    rng = np.random.default_rng(2)
    x = (rng.standard_normal((64, 256)) * np.exp2(rng.uniform(-4, 4, (64, 1)))).astype(np.float32)
    c, s, e = oracle.nvfp4_quantize(x, 0)
    amax_b = np.abs(x).reshape(64, 16, 16).max(axis=2).astype(np.float32)
    t = (amax_b / np.float32(6.0)) * e[0]
    assert t.dtype == np.float32
    want = torch.from_numpy(t).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(s.reshape(64, 16), want)
    assert e[0] == np.float32(2688.0) / np.abs(x).max()
    r, b = np.unravel_index(np.argmax(amax_b), amax_b.shape)
    assert s.reshape(64, 16)[r, b] == 0x7E


def test_decode_matches_independent(oracle):
    rng = np.random.default_rng(3)
    x = rng.standard_t(3, (64, 192)).astype(np.float32)
    for lines in (0, 32):
        c, s, e = oracle.nvfp4_quantize(x, lines)
        y = oracle.nvfp4_dequantize(c, s, e, 64, 192, lines)
        P = ind.decode("e2m1", ind.unpack_codes("e2m1", c, 192))
        D = ind.decode("e4m3", np.repeat(s.reshape(64, 12), 16, axis=1))
        dom = np.arange(64) // (64 if lines == 0 else lines)
        assert np.array_equal(y, P * D / e[dom].astype(np.float64)[:, None])
        # every value within the block's quantization error: half the E2M1
        # spacing at the code, or the saturation step at the top
        err = np.abs(x - y)
        step = ind.grid_spacing("e2m1", P) * D / e[dom].astype(np.float64)[:, None]
        assert np.all(err <= 0.5 * step * (1 + 1e-6) + np.maximum(np.abs(x) - 6 * D / e[dom][:, None], 0))


def test_nonfinite_and_zero(oracle):
    x = np.zeros((64, 32), dtype=np.float32)
    x[40:, :] = 1.0
    x[41, 3] = np.nan
    x[42, 20] = -np.inf
    c, s, e = oracle.nvfp4_quantize(x, 32)
    assert e[0] == 1.0                                       # all-zero domain
    assert e[1] == np.float32(2688.0)                        # amax 1 (non-finite ignored)
    sc = s.reshape(64, 2)
    assert sc[41, 0] == oracle.NV_SCALE_NAN and sc[42, 1] == oracle.NV_SCALE_NAN
    assert np.all(c[41, :8] == 0) and np.all(c[42, 8:] == 0)
    assert np.all(sc[:32] == 0) and np.all(c[:32] == 0)


def test_gemm_reference_is_matmul(oracle):
    rng = np.random.default_rng(5)
    M, N, K = 64, 96, 256
    a = oracle.nvfp4_quantize(rng.standard_normal((M, K)).astype(np.float32), 32, scale_layout=oracle.MMA)
    b = oracle.nvfp4_quantize((rng.standard_normal((N, K)) * 0.02).astype(np.float32), 0,
                              scale_layout=oracle.MMA)
    c, bound = oracle.nvfp4_gemm_decoded(a, b, M, N, K, alpha=0.5, a_lines=32, b_lines=0)
    # independent decode (plain layout via the permutation)
    def dec(q, rows, lines):
        codes, scales, enc = q
        perm = ind.mma_scale_permutation(rows, K // 16)
        plain = scales[perm]
        P = ind.decode("e2m1", ind.unpack_codes("e2m1", codes, K))
        D = ind.decode("e4m3", np.repeat(plain, 16, axis=1))
        dom = np.arange(rows) // (rows if lines == 0 else lines)
        return P * D / enc[dom].astype(np.float64)[:, None]
    A, B = dec(a, M, 32), dec(b, N, 0)
    assert np.allclose(c, 0.5 * (A @ B.T), rtol=0, atol=1e-12 * np.abs(c).max())
    assert np.all(bound >= np.abs(c) - 1e-12)


def test_local_domains_are_global_casts_of_their_rows(oracle):
    """A CTA-local cast is, domain by domain, the global cast of that
    domain's rows alone (a ragged last domain included)."""
    rng = np.random.default_rng(6)
    x = (rng.standard_normal((100, 64)) * np.exp2(rng.uniform(-5, 5, (100, 1)))).astype(np.float32)
    c, s, e = oracle.nvfp4_quantize(x, 32)
    s = s.reshape(100, 4)
    for d, r0 in enumerate(range(0, 100, 32)):
        r1 = min(r0 + 32, 100)
        cg, sg, eg = oracle.nvfp4_quantize(np.ascontiguousarray(x[r0:r1]), 0)
        assert e[d] == eg[0]
        assert np.array_equal(c[r0:r1], cg)
        assert np.array_equal(s[r0:r1].reshape(-1), sg)
