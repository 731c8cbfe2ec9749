"""A second, independent statement of the MX element formats, for pinning the oracle.

Test-only.  It shares nothing with ``oracle/`` (which searches a decoded table)
or with the CUDA library: here the element formats are handled by integer and
significand arithmetic in numpy, vectorised, the way a textbook states
round-to-nearest-even (scale to an integer significand, ``np.rint``, which
rounds half to even).  Agreement between the two over millions of inputs pins
both the oracle's tables and its tie and saturation handling.

Format parameters are read from tests/golden/element_formats.txt.
"""
from __future__ import annotations

import os

import numpy as np

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")

FMT_NAMES = ["e4m3", "e5m2", "e2m3", "e3m2", "e2m1", "int8"]
# exponent / mantissa field widths and bias of each float element format
FIELDS = {"e4m3": (4, 3, 7), "e5m2": (5, 2, 15), "e2m3": (2, 3, 1), "e3m2": (3, 2, 3),
          "e2m1": (2, 1, 1)}


def load_formats():
    out: dict[str, dict[str, float]] = {}
    with open(os.path.join(GOLDEN, "element_formats.txt")) as f:
        for line in f:
            line = line.split("#", 1)[0].strip()
            if not line:
                continue
            name, key, val = line.split()
            out.setdefault(name, {})[key] = float(val)
    return out


def load_codes():
    rows = []
    with open(os.path.join(GOLDEN, "element_codes.txt")) as f:
        for line in f:
            line = line.split("#", 1)[0].strip()
            if not line:
                continue
            name, code, val = line.split()
            rows.append((name, int(code, 16), val))
    return rows


FORMATS = load_formats()


def decode(name: str, codes: np.ndarray) -> np.ndarray:
    """Vectorised decode of element codes to float64 (specials included)."""
    codes = np.asarray(codes, dtype=np.int64)
    if name == "int8":
        s = np.where(codes >= 128, codes - 256, codes)
        return s.astype(np.float64) / 64.0
    eb, mb, bias = FIELDS[name]
    bits = 1 + eb + mb
    sign = (codes >> (bits - 1)) & 1
    e = (codes >> mb) & ((1 << eb) - 1)
    m = codes & ((1 << mb) - 1)
    sig = np.where(e == 0, m, m + (1 << mb)).astype(np.float64)
    exp = np.where(e == 0, 1 - bias, e - bias) - mb
    mag = sig * np.exp2(exp.astype(np.float64))
    if name == "e5m2":
        mag = np.where(e == 31, np.where(m == 0, np.inf, np.nan), mag)
    if name == "e4m3":
        mag = np.where((e == 15) & (m == 7), np.nan, mag)
    return np.where(sign == 1, -mag, mag)


def encode_rne(name: str, u: np.ndarray) -> np.ndarray:
    """Round-to-nearest-even with saturation, by significand arithmetic.

    u: finite float64 values (already divided by the block scale).
    """
    u = np.asarray(u, dtype=np.float64)
    a = np.abs(u)
    neg = np.signbit(u)
    fm = FORMATS[name]
    vmax = fm["max"]
    if name == "int8":
        n = np.minimum(np.rint(a * 64.0), 127.0).astype(np.int64)
        code = np.where(neg, (256 - n) % 256, n)
        return code.astype(np.int64)
    eb, mb, bias = FIELDS[name]
    emin = 1 - bias
    _, ex = np.frexp(a)                       # a = f * 2^ex, f in [0.5, 1)
    e = np.where(a > 0, ex - 1, emin)
    e = np.maximum(e, emin)
    q = np.exp2((e - mb).astype(np.float64))  # grid spacing in that binade
    n = np.rint(a / q)                        # half to even on the significand
    v = np.minimum(n * q, vmax)
    v = np.where(a >= vmax, vmax, v)
    # value -> code
    _, vx = np.frexp(v)
    ve = np.where(v > 0, vx - 1, emin)
    normal = v >= np.exp2(float(emin))
    efield = np.where(normal, ve + bias, 0)
    ve_c = np.maximum(ve, emin)
    sig = v / np.exp2((ve_c - mb).astype(np.float64))
    mfield = np.where(normal, sig - (1 << mb), sig).astype(np.int64)
    code = (efield.astype(np.int64) << mb) | mfield
    bits = 1 + eb + mb
    return np.where(neg, code | (1 << (bits - 1)), code).astype(np.int64)


def grid_spacing(name: str, a: np.ndarray) -> np.ndarray:
    """Distance between the grid points around |a| (for error bounds)."""
    a = np.abs(np.asarray(a, dtype=np.float64))
    if name == "int8":
        return np.full(a.shape, 1.0 / 64.0)
    eb, mb, bias = FIELDS[name]
    emin = 1 - bias
    _, ex = np.frexp(a)
    e = np.maximum(np.where(a > 0, ex - 1, emin), emin)
    return np.exp2((e - mb).astype(np.float64))


def bf16_bits_to_f32(bits: np.ndarray) -> np.ndarray:
    return (np.asarray(bits, dtype=np.uint32) << 16).view(np.float32)


def f32_to_bf16_bits_rne(x: np.ndarray) -> np.ndarray:
    """Round float32 to bf16 (nearest even) by integer arithmetic on the bits."""
    b = np.asarray(x, dtype=np.float32).view(np.uint32).astype(np.uint64)
    lsb = (b >> 16) & 1
    r = (b + 0x7FFF + lsb) >> 16
    return r.astype(np.uint16)


def sylvester_h32() -> np.ndarray:
    """The unnormalised 32x32 Sylvester Hadamard matrix, H_{2n} = [[H, H], [H, -H]]."""
    h = np.array([[1.0]])
    for _ in range(5):
        h = np.block([[h, h], [h, -h]])
    return h


def mma_scale_permutation(outer: int, kblocks: int) -> np.ndarray:
    """Index map plain -> MMA scale layout built from reshapes.

    Returns perm with mma_buffer[perm[o, kb]] holding plain[o, kb]; rows are
    padded to 128 and k-blocks to 4.  The MMA layout is 512-byte atoms of
    128 rows x 4 k-blocks, atoms ordered k-fastest; inside an atom the byte
    order is (row mod 32, row div 32, kb mod 4) -- written here as an axis
    permutation of a padded array rather than as an offset formula.
    """
    rp = (outer + 127) // 128 * 128
    kp = (kblocks + 3) // 4 * 4
    ids = np.arange(rp * kp).reshape(rp, kp)                       # plain ids, padded
    t = ids.reshape(rp // 128, 4, 32, kp // 4, 4)                  # (rb, r/32, r%32, kg, kb%4)
    t = t.transpose(0, 3, 2, 1, 4)                                 # (rb, kg, r%32, r/32, kb%4)
    flat = t.reshape(-1)                                           # position -> plain id
    pos = np.empty(rp * kp, dtype=np.int64)
    pos[flat] = np.arange(rp * kp)
    return pos.reshape(rp, kp)[:outer, :kblocks]


def pack_codes(name: str, codes: np.ndarray) -> np.ndarray:
    """Pack a (outer, inner) array of element codes into bytes per row."""
    codes = np.asarray(codes, dtype=np.uint32)
    outer, inner = codes.shape
    bits = 8 if name in ("e4m3", "e5m2", "int8") else (6 if name in ("e2m3", "e3m2") else 4)
    if bits == 8:
        return codes.astype(np.uint8)
    if bits == 4:
        lo = codes[:, 0::2] & 0xF
        hi = codes[:, 1::2] & 0xF
        return (lo | (hi << 4)).astype(np.uint8)
    g = codes.reshape(outer, inner // 4, 4) & 0x3F
    w = g[..., 0] | (g[..., 1] << 6) | (g[..., 2] << 12) | (g[..., 3] << 18)
    out = np.stack([w & 0xFF, (w >> 8) & 0xFF, (w >> 16) & 0xFF], axis=-1)
    return out.reshape(outer, inner // 4 * 3).astype(np.uint8)


def unpack_codes(name: str, packed: np.ndarray, inner: int) -> np.ndarray:
    packed = np.asarray(packed, dtype=np.uint32)
    outer = packed.shape[0]
    bits = 8 if name in ("e4m3", "e5m2", "int8") else (6 if name in ("e2m3", "e3m2") else 4)
    if bits == 8:
        return packed.astype(np.int64)
    if bits == 4:
        out = np.empty((outer, inner), dtype=np.int64)
        out[:, 0::2] = packed & 0xF
        out[:, 1::2] = packed >> 4
        return out
    t = packed.reshape(outer, inner // 4, 3)
    w = t[..., 0] | (t[..., 1] << 8) | (t[..., 2] << 16)
    out = np.stack([(w >> (6 * j)) & 0x3F for j in range(4)], axis=-1)
    return out.reshape(outer, inner).astype(np.int64)


def rounding_class_bits(mbits: int) -> np.ndarray:
    """fp32 bit patterns covering every case round-to-nearest-even onto a grid
    with `mbits` mantissa bits distinguishes: every fp32 exponent field 0..254,
    both signs, every pattern of the top mbits + 2 mantissa bits (kept bits of
    a binade plus the next two, which decide the rounding of binades down to
    two below) and the sticky patterns below them (none, only the lowest bit,
    all bits, the top sticky bit alone).  Sorted, unique, uint32."""
    top = mbits + 2
    low_bits = 23 - top
    lows = np.array([0, 1, (1 << low_bits) - 1, 1 << (low_bits - 1)], dtype=np.uint32)
    exp = np.arange(0, 255, dtype=np.uint32)
    hi = np.arange(1 << top, dtype=np.uint32) << low_bits
    sign = np.array([0, 1], dtype=np.uint32) << 31
    bits = (sign[:, None, None, None] | (exp[None, :, None, None] << 23) | hi[None, None, :, None]
            | lows[None, None, None, :]).reshape(-1)
    return np.unique(bits)
