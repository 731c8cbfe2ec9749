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


# --------------------------------------------------------------------------
# Stochastic rounding and the whole block cast, restated independently.
#
# The oracle's stochastic rounding (C, table search, one scalar element at a
# time) is pinned here by a vectorised numpy restatement of the definition:
#   * the random byte of the element at linear position i of the
#     block-axis-major OUTPUT (i = outer_index * inner_length + inner_index)
#     is byte (i mod 4) of fmix32(floor(i / 4) xor key), where
#     key = fmix32(low 32 bits of the seed) xor (high 32 bits of the seed) and
#     fmix32 is the MurmurHash3 32-bit finaliser;
#   * with lo <= |u| < hi the two grid points around |u|, the magnitude rounds
#     up iff floor(256 (|u| - lo) / (hi - lo)) + r >= 256; |u| >= max gives max;
#     the sign is put back afterwards (FP formats keep the sign of zero).
# The hash below is checked on its own against the published MurmurHash3
# vectors (tests/golden/murmur3_x86_32.txt), so nothing here is taken from the
# oracle.
# --------------------------------------------------------------------------

_M32 = np.uint64(0xFFFFFFFF)


def fmix32(h) -> np.ndarray:
    """MurmurHash3's 32-bit finaliser, vectorised (uint32 in, uint32 out)."""
    h = np.asarray(h, dtype=np.uint64) & _M32
    h ^= h >> np.uint64(16)
    h = (h * np.uint64(0x85EBCA6B)) & _M32
    h ^= h >> np.uint64(13)
    h = (h * np.uint64(0xC2B2AE35)) & _M32
    h ^= h >> np.uint64(16)
    return h.astype(np.uint32)


def murmur3_x86_32(data: bytes, seed: int) -> int:
    """The whole MurmurHash3_x86_32 around this module's fmix32."""
    c1, c2 = 0xCC9E2D51, 0x1B873593

    def rotl(x, r):
        return ((x << r) | (x >> (32 - r))) & 0xFFFFFFFF

    h = seed & 0xFFFFFFFF
    n = len(data) // 4
    for i in range(n):
        k = int.from_bytes(data[4 * i:4 * i + 4], "little")
        h ^= (rotl((k * c1) & 0xFFFFFFFF, 15) * c2) & 0xFFFFFFFF
        h = (rotl(h, 13) * 5 + 0xE6546B64) & 0xFFFFFFFF
    if len(data) % 4:
        k = int.from_bytes(data[4 * n:], "little")
        h ^= (rotl((k * c1) & 0xFFFFFFFF, 15) * c2) & 0xFFFFFFFF
    return int(fmix32(h ^ len(data)))


def sr_key(seed: int) -> int:
    seed &= (1 << 64) - 1
    return int(fmix32(seed & 0xFFFFFFFF)) ^ (seed >> 32)


def sr_bytes(seed: int, idx) -> np.ndarray:
    """Random byte of each linear output position idx (any integer array)."""
    idx = np.asarray(idx, dtype=np.uint64)
    words = fmix32(((idx >> np.uint64(2)) & _M32) ^ np.uint64(sr_key(seed)))
    shift = (np.uint64(8) * (idx & np.uint64(3))).astype(np.uint32)
    return ((words >> shift) & np.uint32(0xFF)).astype(np.int64)


def encode_sr(name: str, u: np.ndarray, r: np.ndarray) -> np.ndarray:
    """Stochastic rounding onto the element grid by significand arithmetic.

    u: finite float64 values already divided by the block scale; r: one
    random byte (0..255) per value."""
    u = np.asarray(u, dtype=np.float64)
    r = np.asarray(r, dtype=np.int64)
    a = np.abs(u)
    neg = np.signbit(u)
    vmax = FORMATS[name]["max"]
    q = grid_spacing(name, a)                  # spacing of the grid at |u|
    lo = np.floor(a / q) * q                   # exact: q is a power of two
    f = np.floor((a - lo) / q * 256.0).astype(np.int64)
    mag = np.where(f + r >= 256, lo + q, lo)
    mag = np.where(a >= vmax, vmax, mag)
    # the magnitude is on the grid: its RNE code is its code
    code = encode_rne(name, mag)
    if name == "int8":
        return np.where(neg & (code != 0), (256 - code) % 256, code).astype(np.int64)
    bits = 8 if name == "e5m2" or name == "e4m3" else (6 if name in ("e2m3", "e3m2") else 4)
    return np.where(neg, code | (1 << (bits - 1)), code).astype(np.int64)


def hadamard_blocks(v: np.ndarray, sign_mask: int) -> np.ndarray:
    """Fixed-sign 32-point Hadamard on the last axis (length 32), in float32.

    Position j is negated unless bit j of sign_mask is set; then five butterfly
    stages with distance 1, 2, 4, 8, 16, each replacing the pair (x_i, x_{i+h})
    (i with bit h clear) by (x_i + x_{i+h}, x_i - x_{i+h}), every operation an
    IEEE float32 add or subtract."""
    x = np.array(v, dtype=np.float32, copy=True)
    keep = ((np.uint64(sign_mask) >> np.arange(32, dtype=np.uint64)) & np.uint64(1)).astype(bool)
    x[..., ~keep] = -x[..., ~keep]
    pos = np.arange(32)
    for h in (1, 2, 4, 8, 16):
        i = pos[(pos & h) == 0]
        a, b = x[..., i].copy(), x[..., i + h].copy()
        x[..., i] = a + b
        x[..., i + h] = a - b
    return x


def quantize(x: np.ndarray, block_axis: int, name: str, sr: bool = False, seed: int = 0,
             hadamard: bool = False, sign_mask: int = 0, mma_layout: bool = False):
    """The whole MX cast of a 2-D tensor: float32 values, or bf16 bits as uint16.

    Returns (packed codes, scales) in the library's storage layout: codes one
    row per line along the block axis (transposed for block_axis 0), scales
    plain (outer x inner/32) or in the tensor-core layout (padding bytes 0)."""
    v = bf16_bits_to_f32(x) if x.dtype == np.uint16 else np.asarray(x, dtype=np.float32)
    if block_axis == 0:
        v = v.T
    outer, inner = v.shape
    assert inner % 32 == 0
    blocks = np.ascontiguousarray(v).reshape(outer, inner // 32, 32)
    if hadamard:
        blocks = hadamard_blocks(blocks, sign_mask)
    # FP32 subnormal -> signed zero, before anything else looks at the values
    tiny = np.abs(blocks) < np.float32(2.0 ** -126)
    blocks = np.where(tiny, np.copysign(np.float32(0.0), blocks), blocks).astype(np.float32)
    w = blocks.astype(np.float64)
    bad = ~np.all(np.isfinite(w), axis=-1)
    amax = np.max(np.abs(np.where(np.isfinite(w), w, 0.0)), axis=-1)
    _, ex = np.frexp(amax)
    emax = {"e4m3": 8, "e5m2": 15, "e2m3": 2, "e3m2": 4, "e2m1": 2, "int8": 0}[name]
    e = np.clip(np.where(amax > 0, ex - 1 - emax, -127), -127, 127)
    u = np.where(np.isfinite(w), w, 0.0) * np.exp2(-e.astype(np.float64))[..., None]
    if sr:
        idx = (np.arange(outer, dtype=np.uint64)[:, None] * np.uint64(inner)
               + np.arange(inner, dtype=np.uint64)[None, :]).reshape(outer, inner // 32, 32)
        codes = encode_sr(name, u, sr_bytes(seed, idx))
    else:
        codes = encode_rne(name, u)
    codes = np.where(bad[..., None], 0, codes)
    scale = np.where(bad, 255, e + 127).astype(np.uint8)
    packed = pack_codes(name, codes.reshape(outer, inner))
    if not mma_layout:
        return packed, scale.reshape(-1)
    perm = mma_scale_permutation(outer, inner // 32)
    rp, kp = (outer + 127) // 128 * 128, (inner // 32 + 3) // 4 * 4
    out = np.zeros(rp * kp, dtype=np.uint8)
    out[perm.reshape(-1)] = scale.reshape(-1)
    return packed, out
