"""Pins for the oracle's block cast (Algorithm 1), layouts, Hadamard and decode.

"Microscaling Data Formats for Deep Learning" (summary page):
  section 2 -- v_i = X * P_i, NaN scale => NaN block, E8M0 scale;
  section 3 -- largest input exponent onto the element format's largest binade,
               overflowing normals clamped, FP32 subnormals -> 0, axis matters.
"Format-Aware Fusion for Fast FP4 Pretraining" (abstract) -- fixed-sign
  32-value Hadamard preconditioning and stochastic rounding.
"""
import numpy as np
import pytest

import mx_independent as ind

NAMES = ind.FMT_NAMES


def fid(name):
    return NAMES.index(name)


def _unpacked(oracle, name, codes, inner):
    return ind.unpack_codes(name, codes, inner)


@pytest.mark.parametrize("name", NAMES)
def test_emax_closed_form(oracle, name):
    """amax = 2^t gives scale code clamp(t - emax, -127, 127) + 127 and the amax
    element lands on 2^emax (when the scale is not clamped)."""
    f = fid(name)
    emax = int(ind.FORMATS[name]["emax"])
    rng = np.random.default_rng(5)
    ts = list(range(-126, 128))
    x = np.zeros((len(ts), 32), dtype=np.float32)
    for i, t in enumerate(ts):
        x[i] = (rng.uniform(-1, 1, 32) * 2.0 ** t).astype(np.float32)
        x[i, i % 32] = np.float32(2.0 ** t)
        small = np.abs(x[i]) < 2.0 ** -126
        x[i][small] = 0.0
    codes, scales = oracle.quantize(x, 1, f)
    for i, t in enumerate(ts):
        e = min(max(t - emax, -127), 127)
        assert scales[i] == e + 127, (name, t, scales[i])
        if t - emax >= -127:
            c = _unpacked(oracle, name, codes, 32)[i, i % 32]
            assert ind.decode(name, np.array([c]))[0] == 2.0 ** emax


@pytest.mark.parametrize("name", NAMES)
def test_exact_reconstruction(oracle, name):
    """Codes with an element in the top binade, times any E8M0 scale, decode to
    values that quantize back to the same codes and scale."""
    f = fid(name)
    rng = np.random.default_rng(17 + f)
    bits = int(ind.FORMATS[name]["bits"])
    emax = int(ind.FORMATS[name]["emax"])
    allv = ind.decode(name, np.arange(1 << bits))
    finite = np.nonzero(np.isfinite(allv))[0]
    if name == "int8":
        finite = finite[finite != 0x80]
    top = [c for c in finite if abs(allv[c]) >= 2.0 ** emax]
    R = 400
    codes = rng.choice(finite, size=(R, 32))
    codes[np.arange(R), rng.integers(0, 32, R)] = rng.choice(top, size=R)
    scale = rng.integers(127 - 100, 127 + 100, size=R)
    vals = ind.decode(name, codes) * np.exp2(scale - 127.0)[:, None]
    x = vals.astype(np.float32)
    assert np.array_equal(x.astype(np.float64), vals)       # fp32-exact inputs
    got_codes, got_scales = oracle.quantize(x, 1, f)
    np.testing.assert_array_equal(got_scales, scale)
    got = _unpacked(oracle, name, got_codes, 32)
    # codes agree as values (+0/-0 are distinct codes and must agree too)
    np.testing.assert_array_equal(ind.decode(name, got), ind.decode(name, codes))
    np.testing.assert_array_equal(np.signbit(ind.decode(name, got)),
                                  np.signbit(ind.decode(name, codes)))


def test_zero_and_subnormal_blocks(oracle):
    f = fid("e4m3")
    sub = np.array([1e-40, -1e-40, 1e-45, -3e-39], dtype=np.float32)   # fp32 subnormals
    x = np.zeros((3, 32), dtype=np.float32)
    x[0] = 0.0
    x[0, 5] = -0.0
    x[1] = np.resize(sub, 32)                       # all subnormal -> all-zero block
    x[2] = np.linspace(-3, 3, 32).astype(np.float32)
    x[2, 7] = np.float32(-1e-40)                    # one subnormal in a normal block
    codes, scales = oracle.quantize(x, 1, f)
    assert scales[0] == 0 and scales[1] == 0        # reading: amax 0 -> smallest scale
    assert codes[0, 5] == 0x80 and np.all(np.delete(codes[0], 5) == 0)
    want1 = np.where(np.signbit(x[1]), 0x80, 0x00)
    np.testing.assert_array_equal(codes[1], want1)
    assert codes[2, 7] == 0x80                      # flushed, sign kept
    # the amax of block 2 is 3 -> floor(log2 3) - 8 = -7
    assert scales[2] == 127 - 7


def test_bf16_subnormals_flush(oracle):
    f = fid("e2m1")
    bits = np.zeros((1, 32), dtype=np.uint16)
    bits[0, :] = 0x0001                  # smallest bf16 subnormal
    bits[0, 3] = 0x8003
    bits[0, 4] = 0x3F80                  # 1.0
    codes, scales = oracle.quantize(bits, 1, f)
    got = ind.unpack_codes("e2m1", codes, 32)[0]
    assert got[4] == 0x6                 # 1.0 / 2^-2 = 4
    assert got[3] == 0x8                 # -0
    assert np.all(got[[0, 1, 2, 5, 6]] == 0)
    assert scales[0] == 127 + 0 - 2      # amax 1.0: floor(log2 1) - emax(E2M1=2)


def test_nonfinite_block_is_nan(oracle):
    f = fid("e4m3")
    x = np.ones((3, 32), dtype=np.float32)
    x[0, 3] = np.nan
    x[1, 9] = np.inf
    codes, scales = oracle.quantize(x, 1, f)
    assert scales[0] == 0xFF and scales[1] == 0xFF and scales[2] == 127 - 8
    assert np.all(codes[:2] == 0)
    y = oracle.dequantize(codes, scales, f, 3, 32)
    assert np.all(np.isnan(y[:2])) and np.all(y[2] == 1.0)


@pytest.mark.parametrize("name", NAMES)
def test_rne_error_bound(oracle, name):
    """Each decoded element is within half a grid step (times the scale) of
    its input, unless it saturated at +-max."""
    f = fid(name)
    rng = np.random.default_rng(23)
    x = (rng.standard_normal((64, 128)) * np.exp2(rng.uniform(-8, 8, (64, 1)))).astype(np.float32)
    codes, scales = oracle.quantize(x, 1, f)
    y = oracle.dequantize(codes, scales, f, 64, 128)
    X = np.exp2(np.repeat(scales.reshape(64, 4).astype(np.float64) - 127, 32, axis=1))
    u = x.astype(np.float64) / X
    sat = np.abs(u) >= ind.FORMATS[name]["max"]
    err = np.abs(y - x) / X
    lo = np.abs(y) / X                       # grid point chosen
    half = 0.5 * np.maximum(ind.grid_spacing(name, np.minimum(np.abs(u), lo)),
                            ind.grid_spacing(name, lo))
    assert np.all(err[~sat] <= half[~sat])
    assert np.all(np.abs(y[sat]) == ind.FORMATS[name]["max"] * X[sat])


def test_axis0_is_axis1_of_transpose(oracle):
    """The strided cast of X equals the contiguous cast of X^T, including the
    stochastic-rounding indices (both are defined in output coordinates)."""
    rng = np.random.default_rng(29)
    x = rng.standard_normal((96, 40)).astype(np.float32)
    for name in ("e4m3", "e2m3", "e2m1", "int8"):
        f = fid(name)
        for rnd in (0, 1):
            a = oracle.quantize(x, 0, f, rnd=rnd, seed=9, scale_layout=1)
            b = oracle.quantize(np.ascontiguousarray(x.T), 1, f, rnd=rnd, seed=9, scale_layout=1)
            np.testing.assert_array_equal(a[0], b[0])
            np.testing.assert_array_equal(a[1], b[1])


def test_axis_choice_does_not_commute(oracle):
    """Section 3: conversion and transposition do not commute."""
    rng = np.random.default_rng(31)
    x = (rng.standard_normal((64, 64)) * np.exp2(rng.uniform(-6, 6, (64, 1)))).astype(np.float32)
    f = fid("e2m1")
    c1, s1 = oracle.quantize(x, 1, f)
    c0, s0 = oracle.quantize(x, 0, f)
    y1 = oracle.dequantize(c1, s1, f, 64, 64)          # rows of x
    y0 = oracle.dequantize(c0, s0, f, 64, 64).T        # back to x's orientation
    assert not np.array_equal(y1, y0)


def test_ldx_pitch(oracle):
    rng = np.random.default_rng(37)
    big = rng.standard_normal((64, 80)).astype(np.float32)
    x = big[:, :64]
    for axis in (0, 1):
        want = oracle.quantize(np.ascontiguousarray(x), axis, fid("e5m2"))
        got = oracle.quantize(big, axis, fid("e5m2"), ldx=80, cols=64)
        np.testing.assert_array_equal(got[0], want[0])
        np.testing.assert_array_equal(got[1], want[1])


@pytest.mark.parametrize("name", ["e2m3", "e3m2", "e2m1"])
def test_packing_matches_independent_packer(oracle, name):
    rng = np.random.default_rng(41)
    x = rng.standard_normal((8, 64)).astype(np.float32)
    f = fid(name)
    codes, scales = oracle.quantize(x, 1, f)
    un = ind.unpack_codes(name, codes, 64)
    np.testing.assert_array_equal(ind.pack_codes(name, un), codes)
    # element values agree with an element-wise decode of the unpacked codes
    y = oracle.dequantize(codes, scales, f, 8, 64)
    X = np.exp2(np.repeat(scales.reshape(8, 2).astype(np.float64) - 127, 32, axis=1))
    np.testing.assert_array_equal(y, ind.decode(name, un) * X)


def test_fp6_bit_positions(oracle):
    """c0 in bits 0-5, c1 in 6-11, c2 in 12-17, c3 in 18-23 of a 24-bit word."""
    f = fid("e2m3")
    x = np.zeros((1, 32), dtype=np.float32)
    x[0, :4] = [7.5, 0.125, 1.0, -7.5]      # amax 7.5 -> scale 2^0
    codes, scales = oracle.quantize(x, 1, f)
    assert scales[0] == 127
    w = int(codes[0, 0]) | (int(codes[0, 1]) << 8) | (int(codes[0, 2]) << 16)
    assert [(w >> (6 * j)) & 63 for j in range(4)] == [0x1F, 0x01, 0x08, 0x3F]


def test_fp4_nibble_order(oracle):
    f = fid("e2m1")
    x = np.zeros((1, 32), dtype=np.float32)
    x[0, 0], x[0, 1] = 6.0, -0.5              # amax 6 -> scale 2^0
    codes, scales = oracle.quantize(x, 1, f)
    assert scales[0] == 127 and codes[0, 0] == 0x97   # low nibble 0x7 (6), high 0x9 (-0.5)


def test_mma_scale_layout(oracle):
    rng = np.random.default_rng(43)
    for outer, inner in [(128, 128), (200, 96), (300, 32 * 9)]:
        x = rng.standard_normal((outer, inner)).astype(np.float32)
        _, plain = oracle.quantize(x, 1, fid("e4m3"), scale_layout=0)
        _, mma = oracle.quantize(x, 1, fid("e4m3"), scale_layout=1, fill=0xAB)
        kb = inner // 32
        assert mma.size == ((outer + 127) // 128 * 128) * ((kb + 3) // 4 * 4)
        perm = ind.mma_scale_permutation(outer, kb)
        np.testing.assert_array_equal(mma[perm], plain.reshape(outer, kb))
        untouched = np.ones(mma.size, bool)
        untouched[perm.reshape(-1)] = False
        assert np.all(mma[untouched] == 0xAB)


def test_sizes(oracle):
    for name, per32 in [("e4m3", 32), ("e5m2", 32), ("int8", 32), ("e2m3", 24), ("e3m2", 24),
                        ("e2m1", 16)]:
        assert oracle.codes_bytes(fid(name), 10, 64) == 10 * 2 * per32
    assert oracle.scales_bytes(0, 10, 64) == 20
    assert oracle.scales_bytes(1, 10, 64) == 128 * 4
    assert oracle.scales_bytes(1, 129, 32 * 5) == 256 * 8


# --------------------------------------------------------------------------
# Hadamard (reading of "fixed-sign 32-value Hadamard preconditioning")
# --------------------------------------------------------------------------

def test_hadamard_is_sylvester_product(oracle):
    H = ind.sylvester_h32()
    np.testing.assert_array_equal(H.T @ H, 32 * np.eye(32))
    rng = np.random.default_rng(47)
    for mask in (0xFFFFFFFF, 0x6A09E667, 0x0, 0x12345678):
        s = np.array([1.0 if (mask >> j) & 1 else -1.0 for j in range(32)])
        for _ in range(20):
            x = rng.integers(-1000, 1000, 32).astype(np.float32)   # sums stay exact
            got = oracle.hadamard32(x, mask)
            np.testing.assert_array_equal(got.astype(np.float64), H @ (s * x.astype(np.float64)))


def test_hadamard_preserves_wgrad_product():
    """alpha * (H D dY)^T (H D X) = dY^T X with alpha = 1/32, in exact arithmetic."""
    H = ind.sylvester_h32()
    mask = 0x6A09E667
    D = np.diag([1.0 if (mask >> j) & 1 else -1.0 for j in range(32)])
    rng = np.random.default_rng(53)
    dy = rng.standard_normal((64, 8))
    x = rng.standard_normal((64, 12))
    Q = np.kron(np.eye(2), H @ D)          # per 32-block along tokens
    lhs = (Q @ dy).T @ (Q @ x) / 32.0
    np.testing.assert_allclose(lhs, dy.T @ x, rtol=1e-12, atol=1e-12)


def test_hadamard_cast_uses_blocks_along_axis(oracle):
    """The fused cast equals: transform each 32-block along the block axis in
    fp32, then the plain cast of the transformed values."""
    rng = np.random.default_rng(59)
    x = rng.standard_t(3, size=(64, 48)).astype(np.float32)
    mask = 0x6A09E667
    f = fid("e2m1")
    codes, scales = oracle.quantize(x, 0, f, rnd=1, seed=42, hadamard=True, sign_mask=mask)
    xt = np.ascontiguousarray(x.T)
    pre = np.empty_like(xt)
    for c in range(48):
        for b in range(2):
            pre[c, 32 * b:32 * b + 32] = oracle.hadamard32(xt[c, 32 * b:32 * b + 32], mask)
    want = oracle.quantize(pre, 1, f, rnd=1, seed=42)
    np.testing.assert_array_equal(codes, want[0])
    np.testing.assert_array_equal(scales, want[1])


# --------------------------------------------------------------------------
# output rounding of decoded values
# --------------------------------------------------------------------------

def test_round_bf16_matches_bit_rounding(oracle):
    rng = np.random.default_rng(61)
    bits = rng.integers(0, 1 << 32, 200_000, dtype=np.uint64).astype(np.uint32)
    x = bits.view(np.float32)
    x = x[np.isfinite(x)]
    x = x[np.abs(x) < 3.0e38]
    got = oracle.round_bf16(x.astype(np.float64))
    want = ind.f32_to_bf16_bits_rne(x)
    np.testing.assert_array_equal(got, want)


def test_round_f32_is_nearest(oracle):
    y = np.array([1.0 + 2.0 ** -24, 1.0 + 3 * 2.0 ** -24, -(1.0 + 2.0 ** -23 + 2.0 ** -40)])
    got = oracle.round_f32(y)
    np.testing.assert_array_equal(got, np.array([1.0, 1.0 + 2.0 ** -22, -(1.0 + 2.0 ** -23)],
                                                dtype=np.float32))


def test_mma_x4_scale_layout(oracle):
    """The x4 layout: the MMA layout's 512-byte atoms, each stored four times
    in a row (built here by repeating the plain scales through the MMA index
    map), for both block axes, every format, SR and the Hadamard; decodes
    agree with the plain layout's."""
    rng = np.random.default_rng(44)
    for outer, inner in [(128, 128), (200, 96), (300, 32 * 9)]:
        for axis in (0, 1):
            rows, cols = (outer, inner) if axis == 1 else (inner, outer)
            x = rng.standard_normal((rows, cols)).astype(np.float32)
            for name in ("e4m3", "e2m1", "e3m2", "int8"):
                kw = dict(rnd=oracle.SR, seed=5, hadamard=axis == 0)
                c_plain, plain = oracle.quantize(x, axis, fid(name), scale_layout=oracle.PLAIN, **kw)
                c_x4, x4 = oracle.quantize(x, axis, fid(name), scale_layout=oracle.MMA_X4, fill=0xAB, **kw)
                kb = inner // 32
                assert x4.size == 4 * ((outer + 127) // 128 * 128) * ((kb + 3) // 4 * 4)
                perm = ind.mma_scale_permutation(outer, kb)            # MMA layout positions
                atom, within = perm // 512, perm % 512
                for j in range(4):
                    np.testing.assert_array_equal(x4[atom * 2048 + 512 * j + within], plain.reshape(outer, kb))
                written = np.zeros(x4.size, bool)
                for j in range(4):
                    written[(atom * 2048 + 512 * j + within).reshape(-1)] = True
                assert np.all(x4[~written] == 0xAB)
                assert np.array_equal(c_x4, c_plain)
                y_plain = oracle.dequantize(c_plain, plain, fid(name), outer, inner, oracle.PLAIN)
                y_x4 = oracle.dequantize(c_x4, x4, fid(name), outer, inner, oracle.MMA_X4)
                np.testing.assert_array_equal(y_x4, y_plain)
    assert oracle.scales_bytes(oracle.MMA_X4, 129, 32 * 5) == 4 * 256 * 8
