"""GPU parity of the sharded casts (mx_quantize_shard, mx_quantize_dual_shard).

A piece of a larger tensor, cast with its placement, gives exactly the bytes
of the matching slice of the whole tensor's cast: stochastic rounding draws
from the element's position in the whole tensor's output (the reading of
"row-gradient stochastic rounding", "Format-Aware Fusion for Fast FP4
Pretraining", abstract, that makes results independent of how the work is
split).  Checked against the oracle's sharded cast and against the GPU's own
whole-tensor cast, including the weight-gradient dY split by tokens.
"""
import numpy as np
import pytest
import torch

import mx_independent as ind
from gpu_helpers import dev, first_mismatch, host, to_device
from microscaling_block_scaled_mx_b200 import inputs as I
from microscaling_block_scaled_mx_b200 import mx

pytestmark = pytest.mark.gpu

MASK = mx.DEFAULT_SIGN_MASK


def pieces(n, cuts):
    edges = [0] + list(cuts) + [n]
    return list(zip(edges[:-1], edges[1:]))


def plain_scales(s, outer, inner):
    return s[:outer * (inner // 32)].reshape(outer, inner // 32)


@pytest.mark.parametrize("fmt", ["e2m1", "e4m3", "e3m2", "int8"])
@pytest.mark.parametrize("axis", [0, 1])
@pytest.mark.parametrize("hadamard", [False, True])
def test_shard_cast_parity(oracle, fmt, axis, hadamard):
    if hadamard and axis == 1:
        pytest.skip("the Hadamard runs along the strided axis only")
    rng = np.random.default_rng(40 + axis)
    R, C = 320, 288
    x = ind.f32_to_bf16_bits_rne(rng.standard_t(3, size=(R, C)).astype(np.float32))
    xd = to_device(x)
    f = oracle.FORMATS[fmt]
    whole_c, whole_s = mx.quantize(xd, axis, fmt, rnd="sr", seed=99, hadamard=hadamard, sign_mask=MASK,
                                   scale_layout="plain")
    outer, inner = (R, C) if axis == 1 else (C, R)
    wc = ind.unpack_codes(fmt, host(whole_c), inner)
    ws = plain_scales(host(whole_s), outer, inner)
    # cuts along the block axis fall on block boundaries; across it, rows are cut
    # anywhere and columns on 8-column (16-byte) boundaries, the row-pitch rule
    row_cuts = [96, 224] if axis == 0 else [45, 200]
    col_cuts = [64, 160] if axis == 1 else [40, 168]
    for r0, r1 in pieces(R, row_cuts):
        for c0, c1 in pieces(C, col_cuts):
            piece = np.ascontiguousarray(x[r0:r1, c0:c1])
            # each piece in its own (aligned) buffer, as a rank would hold it
            gc, gs = mx.quantize(to_device(piece), axis, fmt, rnd="sr", seed=99, hadamard=hadamard,
                                 sign_mask=MASK, scale_layout="plain", shard=(r0, c0, R, C))
            torch.cuda.synchronize()
            oc, os_ = oracle.quantize(piece, axis, f, rnd=oracle.SR, seed=99, hadamard=hadamard, sign_mask=MASK,
                                      shard=(r0, c0, R, C))
            assert np.array_equal(host(gc), oc), (r0, c0, first_mismatch(host(gc), oc))
            assert np.array_equal(host(gs)[:os_.size], os_), (r0, c0)
            o0, o1, i0, i1 = (r0, r1, c0, c1) if axis == 1 else (c0, c1, r0, r1)
            assert np.array_equal(ind.unpack_codes(fmt, host(gc), i1 - i0), wc[o0:o1, i0:i1])
            assert np.array_equal(plain_scales(host(gs), o1 - o0, i1 - i0), ws[o0:o1, i0 // 32:i1 // 32])


@pytest.mark.parametrize("fmt", ["e2m1", "e4m3"])
def test_dual_shard_parity(oracle, fmt):
    rng = np.random.default_rng(3)
    R, C = 256, 320
    x = ind.f32_to_bf16_bits_rne(rng.standard_normal((R, C)).astype(np.float32))
    f = oracle.FORMATS[fmt]
    for r0, r1 in pieces(R, [64, 192]):
        for c0, c1 in pieces(C, [96]):
            piece = np.ascontiguousarray(x[r0:r1, c0:c1])
            # plain scale layout: the tensor-core layout pads these piece shapes, and
            # padding bytes are never written
            cr, sr_, cc, sc = mx.quantize_dual(to_device(piece), fmt, rnd_rows="sr", seed_rows=5, rnd_cols="sr",
                                               seed_cols=6, hadamard=True, sign_mask=MASK, scale_layout="plain",
                                               shard=(r0, c0, R, C))
            torch.cuda.synchronize()
            ocr, osr = oracle.quantize(piece, 1, f, rnd=oracle.SR, seed=5, shard=(r0, c0, R, C))
            occ, osc = oracle.quantize(piece, 0, f, rnd=oracle.SR, seed=6, hadamard=True, sign_mask=MASK,
                                       shard=(r0, c0, R, C))
            assert np.array_equal(host(cr), ocr) and np.array_equal(host(cc), occ), (r0, c0)
            assert np.array_equal(host(sr_), osr) and np.array_equal(host(sc), osc), (r0, c0)


def test_wgrad_token_shards_reproduce_whole_cast():
    """dY 16384 x 4096 split into two token shards of 8192 (the data-parallel
    weight-gradient split), each cast along tokens with the Hadamard and
    stochastic rounding as its place in the whole tensor: the two code blocks
    are the halves of the whole tensor's codes, byte for byte."""
    dy, _ = I.wgrad_operands()
    T, D = dy.shape
    d = to_device(dy)
    whole_c, whole_s = mx.quantize(d, 0, "e2m1", rnd="sr", seed=42, hadamard=True, sign_mask=MASK,
                                   scale_layout="plain")
    wc, ws = host(whole_c), plain_scales(host(whole_s), D, T)
    h = T // 2
    for t0 in (0, h):
        gc, gs = mx.quantize(d[t0:t0 + h], 0, "e2m1", rnd="sr", seed=42, hadamard=True, sign_mask=MASK,
                             scale_layout="plain", shard=(t0, 0, T, D))
        torch.cuda.synchronize()
        assert np.array_equal(host(gc), wc[:, t0 // 2:(t0 + h) // 2]), t0
        assert np.array_equal(plain_scales(host(gs), D, h), ws[:, t0 // 32:(t0 + h) // 32]), t0
