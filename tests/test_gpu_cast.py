"""GPU parity of the MX cast and decode against the oracle: bit-exact codes and
scales (Algorithm 1, "Microscaling Data Formats for Deep Learning" summary
page, section 3), bit-exact stochastic rounding and Hadamard preconditioning
("Format-Aware Fusion for Fast FP4 Pretraining", abstract), and exact decode
(section 2) rounded once to fp32 / bf16."""
import numpy as np
import pytest
import torch

import mx_independent as ind
from gpu_helpers import FMTS, dev, first_mismatch, host, to_device
from microscaling_block_scaled_mx_b200 import inputs as I
from microscaling_block_scaled_mx_b200 import mx

pytestmark = pytest.mark.gpu

MASK = mx.DEFAULT_SIGN_MASK


def gpu_cast(x_np, axis, fmt, rnd="rne", seed=0, hadamard=False, sl="mma", ldx=None, cols=None, sign_mask=MASK):
    x = to_device(x_np)
    if cols is not None:
        x = x[:, :cols]
    outer, inner = (x.shape[0], x.shape[1]) if axis == 1 else (x.shape[1], x.shape[0])
    codes = torch.full((outer, mx.codes_row_bytes(fmt, inner)), 0xAB, dtype=torch.uint8, device=dev())
    scales = torch.full((max(mx.scales_bytes(sl, outer, inner), 1),), 0xAB, dtype=torch.uint8, device=dev())
    mx.quantize(x, axis, fmt, rnd=rnd, seed=seed, hadamard=hadamard, sign_mask=sign_mask,
                scale_layout=sl, codes=codes, scales=scales)
    torch.cuda.synchronize()
    return host(codes), host(scales)


def oracle_cast(oracle, x_np, axis, fmt, rnd="rne", seed=0, hadamard=False, sl="mma", cols=None):
    f = oracle.FORMATS[fmt]
    kw = {}
    if cols is not None:
        kw = {"cols": cols, "ldx": x_np.shape[1]}
    c, s = oracle.quantize(x_np, axis, f, rnd=1 if rnd == "sr" else 0, seed=seed, hadamard=hadamard,
                           sign_mask=MASK, scale_layout=1 if sl == "mma" else 0, fill=0xAB, **kw)
    return c, s


def assert_same(got, want, what):
    (gc, gs), (wc, ws) = got, want
    assert gc.shape == wc.shape, (what, gc.shape, wc.shape)
    assert np.array_equal(gs[:ws.size], ws), (what, "scales", first_mismatch(gs[:ws.size], ws))
    assert np.array_equal(gc, wc), (what, "codes", first_mismatch(gc, wc))


def mixed_input(rows, cols, seed, bf16):
    rng = np.random.default_rng(seed)
    x = I.roundtrip_matrix(rows, cols, rng)
    # a few outliers, negative zeros and whole special blocks
    flat = x.reshape(-1)
    flat[rng.choice(flat.size, max(1, flat.size // 500), replace=False)] *= np.float32(1e3)
    flat[rng.choice(flat.size, max(1, flat.size // 300), replace=False)] = np.float32(-0.0)
    return I.to_bf16_bits(x) if bf16 else x


SHAPES_ROWS = [(37, 416), (257, 1024), (3, 32)]
SHAPES_COLS = [(288, 200), (128, 64), (32, 8), (416, 136)]


@pytest.mark.parametrize("fmt", FMTS)
@pytest.mark.parametrize("rnd", ["rne", "sr"])
@pytest.mark.parametrize("bf16", [True, False])
def test_cast_rows_parity(oracle, fmt, rnd, bf16):
    for i, (r, c) in enumerate(SHAPES_ROWS):
        x = mixed_input(r, c, 100 + i, bf16)
        for sl in ("mma", "plain"):
            assert_same(gpu_cast(x, 1, fmt, rnd, seed=77, sl=sl),
                        oracle_cast(oracle, x, 1, fmt, rnd, seed=77, sl=sl), (fmt, rnd, bf16, r, c, sl))


@pytest.mark.parametrize("fmt", FMTS)
@pytest.mark.parametrize("rnd", ["rne", "sr"])
@pytest.mark.parametrize("bf16", [True, False])
def test_cast_cols_parity(oracle, fmt, rnd, bf16):
    for i, (r, c) in enumerate(SHAPES_COLS):
        x = mixed_input(r, c, 200 + i, bf16)
        for sl in ("mma", "plain"):
            assert_same(gpu_cast(x, 0, fmt, rnd, seed=5, sl=sl),
                        oracle_cast(oracle, x, 0, fmt, rnd, seed=5, sl=sl), (fmt, rnd, bf16, r, c, sl))


@pytest.mark.parametrize("fmt", FMTS)
@pytest.mark.parametrize("rnd", ["rne", "sr"])
def test_cast_hadamard_parity(oracle, fmt, rnd):
    rng = np.random.default_rng(300)
    for bf16 in (True, False):
        x = rng.standard_t(3, size=(288, 200)).astype(np.float32)
        x[:32, :5] = 0.0
        x[40, 7] = np.float32(1e-40)
        x = I.to_bf16_bits(x) if bf16 else x
        assert_same(gpu_cast(x, 0, fmt, rnd, seed=42, hadamard=True),
                    oracle_cast(oracle, x, 0, fmt, rnd, seed=42, hadamard=True), (fmt, rnd, bf16))


@pytest.mark.parametrize("axis", [0, 1])
def test_cast_pitched_input(oracle, axis):
    rng = np.random.default_rng(301)
    big = I.to_bf16_bits(rng.standard_normal((96, 200)).astype(np.float32))
    cols = 150 if axis == 0 else 160       # 150: a 16-byte chunk straddles the edge
    got = gpu_cast(big, axis, "e2m1", "sr", seed=3, cols=cols)
    want = oracle_cast(oracle, big, axis, "e2m1", "sr", seed=3, cols=cols)
    assert_same(got, want, axis)


def special_blocks():
    x = np.ones((12, 64), dtype=np.float32)
    x[0, 3] = np.nan
    x[1, 40] = np.inf
    x[2, 0] = -np.inf
    x[3, :32] = 0.0
    x[4, :32] = -0.0
    x[5, :32] = np.resize(np.array([1e-40, -2e-39, 1e-45, -0.0], np.float32), 32)
    x[6, :32] = np.linspace(-1, 1, 32)
    x[6, 3] = -1e-41
    x[7, :32] = 3.0e38                 # largest binades: scale clamps and overflow paths
    x[8, :32] = np.float32(2.0 ** -126)
    x[9, :32] = np.float32(1.7e38) * np.linspace(-1, 1, 32).astype(np.float32)
    x[10, :32] = np.float32(2.0 ** 127) * np.float32(1.9)
    x[11, :] = np.float32(5.877e-39)   # 2^-127: subnormal
    return x


@pytest.mark.parametrize("fmt", FMTS)
@pytest.mark.parametrize("rnd", ["rne", "sr"])
def test_cast_special_blocks(oracle, fmt, rnd):
    x = special_blocks()
    assert_same(gpu_cast(x, 1, fmt, rnd, seed=1), oracle_cast(oracle, x, 1, fmt, rnd, seed=1), fmt)
    xt = np.ascontiguousarray(np.tile(x, (1, 1)).T[:, :])   # 64 x 12, blocks down columns
    assert_same(gpu_cast(xt, 0, fmt, rnd, seed=1), oracle_cast(oracle, xt, 0, fmt, rnd, seed=1), fmt)
    assert_same(gpu_cast(I.to_bf16_bits(x), 1, fmt, rnd, seed=1),
                oracle_cast(oracle, I.to_bf16_bits(x), 1, fmt, rnd, seed=1), fmt)


@pytest.mark.parametrize("fmt", FMTS)
@pytest.mark.parametrize("rnd", ["rne", "sr"])
def test_element_sweep_at_unit_scale(oracle, fmt, rnd):
    """~1M fp32 bit patterns per format, one leading 2^emax per block so the
    block scale is 2^0: every element decision is checked against the oracle."""
    rng = np.random.default_rng(400 + FMTS.index(fmt))
    emax = {"e4m3": 8, "e5m2": 15, "e2m3": 2, "e3m2": 4, "e2m1": 2, "int8": 0}[fmt]
    n_blocks = 1 << 15
    mant = rng.integers(0, 1 << 23, (n_blocks, 32), dtype=np.uint32)
    exps = rng.integers(127 + emax - 30, 127 + emax + 1, (n_blocks, 32), dtype=np.uint32)
    sign = rng.integers(0, 2, (n_blocks, 32), dtype=np.uint32)
    bits = (sign << 31) | (exps << 23) | mant
    bits[:, 0] = ((127 + emax) << 23) | (sign[:, 0] << 31)
    x = bits.view(np.float32).reshape(n_blocks // 8, 256)
    got = gpu_cast(x, 1, fmt, rnd, seed=11)
    want = oracle_cast(oracle, x, 1, fmt, rnd, seed=11)
    assert_same(got, want, fmt)


@pytest.mark.parametrize("fmt", FMTS)
@pytest.mark.parametrize("out_dtype", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("sl", ["mma", "plain"])
def test_dequantize_parity(oracle, fmt, out_dtype, sl):
    x = special_blocks()
    rng = np.random.default_rng(500)
    x = np.concatenate([x, I.roundtrip_matrix(300, 64, rng)], axis=0)
    codes, scales = oracle_cast(oracle, x, 1, fmt, sl=sl)
    # every scale code including the extremes
    scales = scales.copy()
    outer, inner = x.shape
    y = mx.dequantize(torch.from_numpy(codes).to(dev()), torch.from_numpy(scales).to(dev()), fmt,
                      outer, inner, scale_layout=sl, out_dtype=out_dtype)
    want64 = oracle.dequantize(codes, scales, oracle.FORMATS[fmt], outer, inner,
                               1 if sl == "mma" else 0)
    got = host(y)
    if out_dtype == torch.float32:
        want = oracle.round_f32(want64)
        assert np.array_equal(np.isnan(got), np.isnan(want))
        ok = ~np.isnan(want)
        assert np.array_equal(got.view(np.uint32)[ok], want.view(np.uint32)[ok])
    else:
        want = oracle.round_bf16(want64)
        nan = np.isnan(want64)
        assert np.all((got[nan] & 0x7FFF) > 0x7F80)
        assert np.array_equal(got[~nan], want[~nan]), first_mismatch(got[~nan], want[~nan])


@pytest.mark.parametrize("fmt", FMTS)
def test_dequantize_all_scales(oracle, fmt):
    """All 256 scale codes against every element code."""
    nb = 1 << {"e4m3": 8, "e5m2": 8, "e2m3": 6, "e3m2": 6, "e2m1": 4, "int8": 8}[fmt]
    per_block = np.resize(np.arange(nb), 32)
    codes_un = np.tile(per_block, (256, 1))
    import mx_independent as ind
    codes = ind.pack_codes(fmt, codes_un)
    scales = np.arange(256, dtype=np.uint8)
    y = mx.dequantize(torch.from_numpy(codes).to(dev()), torch.from_numpy(scales).to(dev()), fmt,
                      256, 32, scale_layout="plain", out_dtype=torch.float32)
    want = oracle.round_f32(oracle.dequantize(codes, scales, oracle.FORMATS[fmt], 256, 32, 0))
    got = host(y)
    assert np.array_equal(np.isnan(got), np.isnan(want))
    ok = ~np.isnan(want)
    assert np.array_equal(got.view(np.uint32)[ok], want.view(np.uint32)[ok])


def test_empty_is_a_no_op():
    x = torch.empty((0, 64), dtype=torch.bfloat16, device=dev())
    c, s = mx.quantize(x, 1, "e4m3")
    assert c.numel() == 0
    x = torch.empty((64, 0), dtype=torch.bfloat16, device=dev())
    c, s = mx.quantize(x, 0, "e2m1")
    assert c.shape[0] == 0


# --------------------------------------------------------------------------
# full-size workloads
# --------------------------------------------------------------------------

def test_roundtrip_config(oracle):
    """fp32 A 256x512 along K (rows), B 512x256 along K (columns), E4M3, RNE,
    decoded to fp32: bit-exact codes, scales and decoded values."""
    d = I.config_roundtrip()
    for name, x, axis in (("A", d["A"], 1), ("B", d["B"], 0)):
        got = gpu_cast(x, axis, "e4m3")
        want = oracle_cast(oracle, x, axis, "e4m3")
        assert_same(got, want, name)
        outer, inner = (x.shape[0], x.shape[1]) if axis == 1 else (x.shape[1], x.shape[0])
        y = mx.dequantize(torch.from_numpy(got[0]).to(dev()), torch.from_numpy(got[1]).to(dev()),
                          "e4m3", outer, inner, "mma", torch.float32)
        w = oracle.round_f32(oracle.dequantize(want[0], want[1], 0, outer, inner, 1))
        assert np.array_equal(host(y).view(np.uint32), w.view(np.uint32))


@pytest.mark.parametrize("fmt", [f for f in FMTS if f != "int8"])
@pytest.mark.parametrize("rnd", ["rne", "sr"])
def test_rounding_classes_at_unit_scale(oracle, fmt, rnd):
    """Every RNE rounding class of fp32 inputs (all exponents up to the block's
    top binade, both signs, every kept + guard + round bit pattern, the sticky
    cases; see mx_independent.rounding_class_bits), 31 per block after a
    leading 2^emax that fixes the block scale at 2^0: every code against the
    oracle, including the exact ties and the saturation band."""
    emax = {"e4m3": 8, "e5m2": 15, "e2m3": 2, "e3m2": 4, "e2m1": 2}[fmt]
    mbits = {"e4m3": 3, "e5m2": 2, "e2m3": 3, "e3m2": 2, "e2m1": 1}[fmt]
    cls = ind.rounding_class_bits(mbits)
    cls = cls[((cls >> 23) & 0xff) <= 127 + emax]            # inside the scale-2^0 block
    nb = -(-cls.size // 31)
    nb = -(-nb // 8) * 8                                     # whole rows of 8 blocks
    body = np.zeros(nb * 31, dtype=np.uint32)
    body[:cls.size] = cls
    bits = np.empty((nb, 32), dtype=np.uint32)
    bits[:, 0] = (127 + emax) << 23
    bits[:, 1:] = body.reshape(nb, 31)
    x = bits.view(np.float32).reshape(nb // 8, 256)
    got = gpu_cast(x, 1, fmt, rnd, seed=17)
    want = oracle_cast(oracle, x, 1, fmt, rnd, seed=17)
    assert_same(got, want, (fmt, rnd))
    assert np.count_nonzero(got[1] == 127) == nb             # every block at scale 2^0 (the rest is padding)


@pytest.mark.parametrize("fmt", [f for f in FMTS if f != "int8"])
@pytest.mark.parametrize("axis", [1, 0])
def test_sr_carry_boundary(oracle, fmt, axis):
    """Stochastic rounding where only the 8 bits below the grid may decide:
    values whose fraction of a grid step is f8 / 256 plus 255, 128, 1 or 0
    65536ths, on the subnormal grid and in every binade of a scale-2^0 block,
    both signs.  A rounding that looked at more than 8 bits of the fraction,
    or at more random bits than the element's byte, would round up the
    f8 + r = 255 cases (about 1 in 256) that must round down."""
    emax = {"e4m3": 8, "e5m2": 15, "e2m3": 2, "e3m2": 4, "e2m1": 2}[fmt]
    mbits = {"e4m3": 3, "e5m2": 2, "e2m3": 3, "e3m2": 2, "e2m1": 1}[fmt]
    emin = {"e4m3": -6, "e5m2": -14, "e2m3": 0, "e3m2": -2, "e2m1": 0}[fmt]
    rng = np.random.default_rng(31)
    nb = 8 * 512
    n = nb * 31
    binade = rng.integers(emin - 1, emax + 1, n)              # emin - 1: the subnormal grid
    k = rng.integers(0, 1 << mbits, n)
    f = rng.integers(0, 256, n) / 256.0 + rng.choice([255, 128, 1, 0], n) / 65536.0
    base = np.where(binade < emin, 0.0, float(1 << mbits))
    step = np.exp2(np.maximum(binade, emin) - mbits)
    v = (base + k + f) * step * rng.choice([-1.0, 1.0], n)
    assert np.all(v.astype(np.float32).astype(np.float64) == v)   # exact in fp32
    x = np.empty((nb, 32), dtype=np.float32)
    x[:, 0] = 2.0 ** emax
    x[:, 1:] = v.reshape(nb, 31)
    x = x.reshape(nb // 8, 256)
    if axis == 0:
        x = np.ascontiguousarray(x.T)
    got = gpu_cast(x, axis, fmt, "sr", seed=23)
    want = oracle_cast(oracle, x, axis, fmt, "sr", seed=23)
    assert_same(got, want, (fmt, axis))


@pytest.mark.parametrize("fmt", FMTS)
def test_cast_sweep_full_size(oracle, fmt):
    """bf16 8192 x 8192 with outliers, blocks along rows, RNE: every byte."""
    x = _sweep_input()
    assert_same(gpu_cast(x, 1, fmt), oracle_cast(oracle, x, 1, fmt), fmt)


_SWEEP = {}


def _sweep_input():
    if "x" not in _SWEEP:
        _SWEEP["x"] = I.cast_sweep_input()
    return _SWEEP["x"]


def test_wgrad_casts_full_size(oracle, wgrad_oracle_operands):
    """dY 16384 x 4096 and X 16384 x 14336 (bf16, Student-t), cast along tokens
    with the fixed-sign Hadamard and stochastic rounding to E2M1: every byte."""
    d = wgrad_oracle_operands
    for name, t, seed, want in (("dY", d["dy"], 42, d["dy_q"]), ("X", d["xx"], 43, d["xx_q"])):
        got = gpu_cast(t, 0, "e2m1", "sr", seed=seed, hadamard=True)
        assert_same(got, want, name)


@pytest.mark.parametrize("mask", [0x00000000, 0xFFFFFFFF, 0x12345678, MASK ^ 1])
@pytest.mark.parametrize("bf16", [True, False])
def test_hadamard_any_sign_mask(oracle, mask, bf16):
    """The default mask is compiled into the loads; any other mask takes the
    general path.  Both match the oracle byte for byte (column cast and the
    dual cast's column output), SR and RNE."""
    x = mixed_input(256, 96, 77, bf16)
    xd = to_device(x)
    for rnd in ("rne", "sr"):
        got = gpu_cast(x, 0, "e2m1", rnd, seed=3, hadamard=True, sign_mask=mask, sl="plain")
        oc, os_ = oracle.quantize(x, 0, oracle.E2M1, rnd=1 if rnd == "sr" else 0, seed=3, hadamard=True,
                                  sign_mask=mask, scale_layout=oracle.PLAIN)
        assert_same(got, (oc, os_), (hex(mask), rnd))
        _, _, cc, sc = mx.quantize_dual(xd, "e2m1", rnd_cols=rnd, seed_cols=3, hadamard=True, sign_mask=mask,
                                        scale_layout="plain")
        torch.cuda.synchronize()
        assert np.array_equal(host(cc), oc) and np.array_equal(host(sc), os_), (hex(mask), rnd)
