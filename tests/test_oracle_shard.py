"""Sharded casts in the oracle: a tensor cut into pieces casts to the bytes of
the whole.

Stochastic rounding draws each element's random byte from its position in the
block-axis-major output of the whole tensor (the reading of the FP4
pretraining abstract's stochastic rounding taken throughout: results do not
depend on how the work is split).  A piece at (row0, col0) of a larger tensor
therefore reproduces, byte for byte, the matching slice of the whole tensor's
codes and scales, for both block axes, with and without the fixed-sign
Hadamard.  This is what lets data-parallel ranks cast their token shards of
the weight-gradient operands independently.
"""
from __future__ import annotations

import numpy as np
import pytest

import mx_independent as ind

MASK = 0x6A09E667


def pieces(n, cuts):
    edges = [0] + list(cuts) + [n]
    return list(zip(edges[:-1], edges[1:]))


@pytest.mark.parametrize("fmt", ["e2m1", "e4m3", "e3m2", "int8"])
@pytest.mark.parametrize("axis", [0, 1])
@pytest.mark.parametrize("hadamard", [False, True])
def test_pieces_reproduce_whole(oracle, fmt, axis, hadamard):
    f = oracle.FORMATS[fmt]
    rng = np.random.default_rng(31 + axis + 2 * hadamard)
    R, C = 192, 160
    x = ind.f32_to_bf16_bits_rne(rng.standard_t(3, size=(R, C)).astype(np.float32))
    whole_c, whole_s = oracle.quantize(x, axis, f, rnd=oracle.SR, seed=1234, hadamard=hadamard, sign_mask=MASK)
    outer, inner = (R, C) if axis == 1 else (C, R)
    wc = ind.unpack_codes(fmt, whole_c, inner)
    ws = whole_s.reshape(outer, inner // 32)
    # cuts along the block axis fall on block boundaries; the other axis is cut anywhere
    row_cuts = [64, 128] if axis == 0 else [37, 100]
    col_cuts = [32, 96] if axis == 1 else [51, 77]
    for r0, r1 in pieces(R, row_cuts):
        for c0, c1 in pieces(C, col_cuts):
            piece = np.ascontiguousarray(x[r0:r1, c0:c1])
            pc, ps = oracle.quantize(piece, axis, f, rnd=oracle.SR, seed=1234, hadamard=hadamard, sign_mask=MASK,
                                     shard=(r0, c0, R, C))
            o0, o1, i0, i1 = (r0, r1, c0, c1) if axis == 1 else (c0, c1, r0, r1)
            assert np.array_equal(ind.unpack_codes(fmt, pc, i1 - i0), wc[o0:o1, i0:i1]), (r0, c0)
            assert np.array_equal(ps.reshape(o1 - o0, (i1 - i0) // 32), ws[o0:o1, i0 // 32:i1 // 32]), (r0, c0)


def test_local_positions_would_differ(oracle):
    """Casting a piece as if it were a whole tensor (local positions) does not
    reproduce the whole tensor's bytes: the shard placement is what does."""
    rng = np.random.default_rng(2)
    x = rng.standard_normal((128, 64)).astype(np.float32)
    whole_c, _ = oracle.quantize(x, 0, oracle.E2M1, rnd=oracle.SR, seed=5)
    piece = np.ascontiguousarray(x[64:, :])
    local_c, _ = oracle.quantize(piece, 0, oracle.E2M1, rnd=oracle.SR, seed=5)
    placed_c, _ = oracle.quantize(piece, 0, oracle.E2M1, rnd=oracle.SR, seed=5, shard=(64, 0, 128, 64))
    assert np.array_equal(placed_c, whole_c[:, 32:])
    assert not np.array_equal(local_c, whole_c[:, 32:])


def test_shard_validation(oracle):
    x = np.zeros((64, 64), dtype=np.float32)
    with pytest.raises(oracle.OracleError):     # block-axis offset not on a block boundary
        oracle.quantize(x, 0, oracle.E4M3, rnd=oracle.SR, shard=(16, 0, 128, 64))
    with pytest.raises(oracle.OracleError):     # piece outside the whole tensor
        oracle.quantize(x, 1, oracle.E4M3, shard=(100, 0, 128, 64))
    oracle.quantize(x, 1, oracle.E4M3, rnd=oracle.SR, shard=(17, 0, 128, 64))   # rows are not the block axis
