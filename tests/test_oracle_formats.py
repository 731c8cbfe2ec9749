"""Pins for the oracle's element formats and scalar rounding.

Each test checks the oracle against something other than itself: the
element-format fixed points of tests/golden (OCP MX v1.0 definitions, which the
"Microscaling Data Formats for Deep Learning" summary page refers to), a
second encoder written by significand arithmetic (tests/mx_independent.py),
or torch's own float8 conversions.
"""
import numpy as np
import pytest
import torch

import mx_independent as ind

NAMES = ind.FMT_NAMES


def fmt_id(name):
    return NAMES.index(name)


@pytest.mark.parametrize("name", NAMES)
def test_format_extremes_match_definition(oracle, name):
    fm = ind.FORMATS[name]
    f = fmt_id(name)
    assert oracle.emax(f) == int(fm["emax"])
    assert oracle.max_value(f) == fm["max"]
    bits = int(fm["bits"])
    pos = [c for c in range(1 << (bits - 1))] if name != "int8" else list(range(128))
    vals = [oracle.decode_elem(f, c) for c in pos]
    finite = [v for v in vals if np.isfinite(v)]
    assert len(finite) == int(fm["finite_positive"])
    nonzero = sorted(v for v in finite if v > 0)
    assert nonzero[0] == fm["min_subnormal"]
    assert max(finite) == fm["max"]
    # smallest value with a nonzero exponent field is the min normal
    if name != "int8":
        eb, mb, bias = ind.FIELDS[name]
        assert oracle.decode_elem(f, 1 << mb) == fm["min_normal"]


def test_decode_golden_codes(oracle):
    for name, code, val in ind.load_codes():
        got = oracle.decode_elem(fmt_id(name), code)
        if val == "nan":
            assert np.isnan(got), (name, hex(code))
        elif val in ("inf", "-inf"):
            assert got == float(val), (name, hex(code))
        elif val == "-0":
            assert got == 0.0 and np.signbit(got), (name, hex(code))
        else:
            assert got == float(val), (name, hex(code), got, val)


@pytest.mark.parametrize("name", NAMES)
def test_decode_agrees_with_independent_decoder(oracle, name):
    f = fmt_id(name)
    bits = int(ind.FORMATS[name]["bits"])
    codes = np.arange(1 << bits)
    mine = ind.decode(name, codes)
    theirs = np.array([oracle.decode_elem(f, int(c)) for c in codes])
    np.testing.assert_array_equal(np.isnan(mine), np.isnan(theirs))
    ok = ~np.isnan(mine)
    np.testing.assert_array_equal(mine[ok], theirs[ok])
    np.testing.assert_array_equal(np.signbit(mine[ok]), np.signbit(theirs[ok]))


@pytest.mark.parametrize("name", NAMES)
def test_exhaustive_code_round_trip(oracle, name):
    """decode then encode at scale 2^0 returns every finite code."""
    f = fmt_id(name)
    bits = int(ind.FORMATS[name]["bits"])
    n_checked = 0
    for c in range(1 << bits):
        v = oracle.decode_elem(f, c)
        if not np.isfinite(v):
            continue
        got = oracle.encode_rne(f, v)
        if name == "int8" and c == 0x80:
            assert got == 0x81   # -2 is outside the symmetric clamp: -127/64
        else:
            assert got == c, (name, hex(c), v, hex(got))
        n_checked += 1
    expected = {"e2m1": 16, "e2m3": 64, "e3m2": 64, "e4m3": 254, "e5m2": 248, "int8": 256}
    assert n_checked == expected[name]


@pytest.mark.parametrize("name,u,expect", [
    ("e4m3", 460.0, 448.0), ("e4m3", 500.0, 448.0), ("e4m3", 1.9375 * 256, 448.0),
    ("e4m3", 1e30, 448.0), ("e4m3", -1e30, -448.0),
    ("e2m1", 5.0, 4.0), ("e2m1", 2.5, 2.0), ("e2m1", 0.25, 0.0), ("e2m1", 0.75, 1.0),
    ("e2m1", 1.25, 1.0), ("e2m1", 1.75, 2.0), ("e2m1", 3.5, 4.0), ("e2m1", 7.9, 6.0),
    ("e2m1", -5.0, -4.0), ("e2m1", 0.2499, 0.0), ("e2m1", 0.2501, 0.5),
    ("int8", 127.5 / 64, 127 / 64), ("int8", 126.5 / 64, 126 / 64), ("int8", 0.5 / 64, 0.0),
    ("int8", 1.5 / 64, 2 / 64), ("int8", -3.0, -127 / 64),
    ("e5m2", 61440.0, 57344.0), ("e5m2", 1e9, 57344.0),
    ("e2m3", 7.75, 7.5), ("e2m3", 0.0625, 0.0), ("e2m3", 0.1875, 0.25),
    ("e3m2", 30.0, 28.0), ("e3m2", 0.03125, 0.0), ("e3m2", 0.09375, 0.125),
])
def test_rne_fixed_points(oracle, name, u, expect):
    f = fmt_id(name)
    got = oracle.decode_elem(f, oracle.encode_rne(f, u))
    assert got == expect


@pytest.mark.parametrize("name", ["e4m3", "e2m3", "e3m2", "e2m1", "e5m2"])
def test_signed_zero_is_kept(oracle, name):
    f = fmt_id(name)
    tiny = oracle.decode_elem(f, 1) / 4.0    # rounds to zero
    c = oracle.encode_rne(f, -tiny)
    assert oracle.decode_elem(f, c) == 0.0 and np.signbit(oracle.decode_elem(f, c))
    assert oracle.encode_rne(f, -0.0) == c
    assert oracle.encode_rne(f, 0.0) == 0


def _sample_f32(n, rng, lo_exp=-20, hi_exp=20):
    """fp32 values spread over binades, plus exact ties of every format's grid."""
    mant = rng.integers(0, 1 << 23, size=n, dtype=np.uint32)
    exp = rng.integers(127 + lo_exp, 127 + hi_exp, size=n, dtype=np.uint32)
    sign = rng.integers(0, 2, size=n, dtype=np.uint32)
    bits = (sign << 31) | (exp << 23) | mant
    return bits.view(np.float32)


def _ties(name):
    """Every midpoint between neighbouring grid points, both signs."""
    f_vals = np.unique(np.abs(ind.decode(name, np.arange(1 << int(ind.FORMATS[name]["bits"])))))
    f_vals = f_vals[np.isfinite(f_vals)]
    mids = (f_vals[:-1] + f_vals[1:]) / 2
    return np.concatenate([mids, -mids, f_vals, -f_vals, [f_vals[-1] * 1.0001]])


@pytest.mark.parametrize("name", NAMES)
def test_rne_agrees_with_significand_encoder(oracle, name):
    """Oracle table search vs textbook significand rounding on ~200k values."""
    f = fmt_id(name)
    rng = np.random.default_rng(7 + f)
    u = np.concatenate([_sample_f32(200_000, rng, -12, 18).astype(np.float64), _ties(name)])
    want = ind.encode_rne(name, u)
    lib = oracle.lib()
    got = np.fromiter((lib.mxref_encode_rne(f, float(x)) for x in u), dtype=np.int64, count=u.size)
    bad = np.nonzero(got != want)[0]
    assert bad.size == 0, [(u[i], hex(got[i]), hex(want[i])) for i in bad[:10]]


def _rounding_classes(name):
    return ind.rounding_class_bits(ind.FIELDS[name][1]).view(np.float32).astype(np.float64)


@pytest.mark.parametrize("name", [n for n in NAMES if n != "int8"])
def test_rne_rounding_classes_exhaustive(oracle, name):
    """Oracle vs the significand-arithmetic encoder on every rounding class of
    fp32 inputs (all exponents, all kept + guard + round bit patterns, the
    sticky cases).  The classes at the grid's smallest binade cover the
    element-subnormal range; those above the largest cover saturation."""
    f = fmt_id(name)
    u = _rounding_classes(name)
    want = ind.encode_rne(name, u)
    lib = oracle.lib()
    got = np.fromiter((lib.mxref_encode_rne(f, float(x)) for x in u), dtype=np.int64, count=u.size)
    bad = np.nonzero(got != want)[0]
    assert bad.size == 0, [(u[i], hex(got[i]), hex(want[i])) for i in bad[:10]]


def test_rne_int8_rounding_classes_exhaustive(oracle):
    """INT8 (x 2^-6): every integer step 0..128 with fractions 0, just above 0,
    just below, at and just above one half, just below one, both signs, and
    values far beyond the clamp."""
    eps = 2.0 ** -30
    k = np.arange(0, 129, dtype=np.float64)
    fr = np.array([0.0, eps, 0.5 - eps, 0.5, 0.5 + eps, 1.0 - eps])
    mag = ((k[:, None] + fr[None, :]) / 64.0).reshape(-1)
    mag = np.concatenate([mag, [3.0, 1e10, 2.0 ** -40]])
    u = np.concatenate([mag, -mag])
    want = ind.encode_rne("int8", u)
    lib = oracle.lib()
    f = fmt_id("int8")
    got = np.fromiter((lib.mxref_encode_rne(f, float(x)) for x in u), dtype=np.int64, count=u.size)
    bad = np.nonzero(got != want)[0]
    assert bad.size == 0, [(u[i], hex(got[i]), hex(want[i])) for i in bad[:10]]


@pytest.mark.parametrize("name,dtype,lim", [("e4m3", torch.float8_e4m3fn, 448.0),
                                            ("e5m2", torch.float8_e5m2, 57344.0)])
def test_rne_agrees_with_torch_float8(oracle, name, dtype, lim):
    """In range, MX FP8 element rounding is plain IEEE-style RNE to the format:
    the special case that torch's float8 conversion implements."""
    f = fmt_id(name)
    rng = np.random.default_rng(11)
    u = _sample_f32(100_000, rng, -20, 17)
    u = u[np.abs(u) <= lim]
    u = np.concatenate([u, _ties(name).astype(np.float32)])
    u = u[np.abs(u) <= lim]
    want = torch.from_numpy(u.copy()).to(dtype).view(torch.uint8).numpy().astype(np.int64)
    lib = oracle.lib()
    got = np.fromiter((lib.mxref_encode_rne(f, float(x)) for x in u), dtype=np.int64, count=u.size)
    bad = np.nonzero(got != want)[0]
    assert bad.size == 0, [(u[i], hex(got[i]), hex(want[i])) for i in bad[:10]]


# --------------------------------------------------------------------------
# stochastic rounding (reading of "row-gradient stochastic rounding")
# --------------------------------------------------------------------------

def _murmur3(oracle, data: bytes, seed: int) -> int:
    """MurmurHash3_x86_32 built around the oracle's fmix32."""
    c1, c2 = 0xCC9E2D51, 0x1B873593
    rotl = lambda x, r: ((x << r) | (x >> (32 - r))) & 0xFFFFFFFF
    h = seed & 0xFFFFFFFF
    nblk = len(data) // 4
    for i in range(nblk):
        k = int.from_bytes(data[4 * i:4 * i + 4], "little")
        k = rotl((k * c1) & 0xFFFFFFFF, 15)
        h ^= (k * c2) & 0xFFFFFFFF
        h = (rotl(h, 13) * 5 + 0xE6546B64) & 0xFFFFFFFF
    tail = data[4 * nblk:]
    if tail:
        k = int.from_bytes(tail, "little")
        k = rotl((k * c1) & 0xFFFFFFFF, 15)
        h ^= (k * c2) & 0xFFFFFFFF
    h ^= len(data)
    return oracle.fmix32(h)


def test_fmix32_published_vectors(oracle):
    import ast
    import os
    path = os.path.join(ind.GOLDEN, "murmur3_x86_32.txt")
    n = 0
    with open(path) as f:
        for line in f:
            if line.startswith("#") or not line.strip():
                continue
            seed, want, rest = line.split(None, 2)
            data = ast.literal_eval(rest.strip())
            assert _murmur3(oracle, data, int(seed, 16)) == int(want, 16), line
            n += 1
    assert n == 8


def test_sr_byte_definition(oracle):
    """byte (idx mod 4) of fmix32(floor(idx/4) xor (fmix32(seed_lo) xor seed_hi))."""
    seed = 0x0123456789ABCDEF
    key = oracle.fmix32(seed & 0xFFFFFFFF) ^ (seed >> 32)
    for idx in [0, 1, 2, 3, 4, 5, 1023, 1 << 20, (1 << 34) - 1]:
        w = oracle.fmix32(((idx >> 2) ^ key) & 0xFFFFFFFF)
        assert oracle.sr_byte(seed, idx) == (w >> (8 * (idx & 3))) & 255


@pytest.mark.parametrize("name", NAMES)
def test_sr_round_up_count_is_exact(oracle, name):
    """Over all 256 random bytes the number of round-ups is floor(256*frac)."""
    f = fmt_id(name)
    rng = np.random.default_rng(3)
    vmax = ind.FORMATS[name]["max"]
    us = np.concatenate([rng.uniform(-vmax, vmax, 40), [vmax * 0.999, -vmax * 0.999]])
    for u in us:
        a = abs(u)
        lo_code = oracle.encode_sr(f, u, 0)
        lo = abs(oracle.decode_elem(f, lo_code))
        sp = ind.grid_spacing(name, np.array([lo]))[0]
        if lo + sp > vmax and a > lo:
            sp = vmax - lo
        frac = (a - lo) / sp
        ups = sum(abs(oracle.decode_elem(f, oracle.encode_sr(f, u, r))) > lo for r in range(256))
        assert ups == int(np.floor(frac * 256)), (name, u, lo, frac, ups)
        assert lo <= a < lo + sp or a >= vmax


@pytest.mark.parametrize("name", NAMES)
def test_sr_keeps_representable_values(oracle, name):
    f = fmt_id(name)
    bits = int(ind.FORMATS[name]["bits"])
    for c in range(1 << bits):
        v = oracle.decode_elem(f, c)
        if not np.isfinite(v) or (name == "int8" and c == 0x80):
            continue
        for r in (0, 1, 128, 255):
            assert oracle.decode_elem(f, oracle.encode_sr(f, v, r)) == v


def test_sr_is_unbiased(oracle):
    """Mean of SR(u) over many element indices converges to u (4 sigma)."""
    f = fmt_id("e2m1")
    for u in (0.3, 1.1, 2.9, 4.7, -3.3):
        n = 20000
        vals = np.array([oracle.decode_elem(f, oracle.encode_sr(f, u, oracle.sr_byte(42, i)))
                         for i in range(n)])
        # 8-bit resolution: expected value is lo + sp * floor(256 frac)/256
        lo = np.floor(abs(u) / ind.grid_spacing("e2m1", np.array([abs(u)]))[0])
        sd = vals.std() / np.sqrt(n)
        assert abs(vals.mean() - u) < 4 * sd + 1.0 / 256 * 2, (u, vals.mean())
