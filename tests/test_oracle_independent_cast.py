"""The oracle's whole MX cast against an independent numpy restatement.

Pins the parts of the oracle that no closed form reaches on its own: the
stochastic-rounding random byte of each element (its linear position in the
block-axis-major output, byte i mod 4 of the hashed word floor(i/4)), the
round-up rule, the fixed-sign Hadamard as it feeds the cast, the scale
exponent, packing and both scale layouts.  The restatement
(tests/mx_independent.py) works on whole arrays with significand arithmetic
and shares no code with the oracle's scalar C; its hash is checked on its own
against the published MurmurHash3 vectors.

Sources: "Microscaling Data Formats for Deep Learning" (summary page,
section 3, Algorithm 1) for the cast; "Format-Aware Fusion for Fast FP4
Pretraining" (abstract) for stochastic rounding and the fixed-sign 32-value
Hadamard of the weight-gradient operands.
"""
from __future__ import annotations

import ast
import os

import numpy as np
import pytest

import mx_independent as ind

NAMES = ind.FMT_NAMES
SIGN_MASK = 0x6A09E667


def fmt_id(name):
    return NAMES.index(name)


def test_independent_hash_matches_published_vectors():
    path = os.path.join(ind.GOLDEN, "murmur3_x86_32.txt")
    n = 0
    with open(path) as f:
        for line in f:
            if line.startswith("#") or not line.strip():
                continue
            seed, want, rest = line.split(None, 2)
            assert ind.murmur3_x86_32(ast.literal_eval(rest.strip()), int(seed, 16)) == int(want, 16), line
            n += 1
    assert n == 8


def test_random_bytes_agree_with_oracle(oracle):
    """The oracle's per-element byte equals the restated one at scattered
    positions, including ones past 2^32 (the word counter is floor(i / 4))."""
    rng = np.random.default_rng(5)
    idx = np.concatenate([np.arange(64), rng.integers(0, 1 << 34, 2000), [(1 << 34) - 1, 1 << 32]])
    for seed in (0, 42, 0x0123456789ABCDEF, (1 << 64) - 1):
        mine = ind.sr_bytes(seed, idx)
        theirs = np.array([oracle.sr_byte(seed, int(i)) for i in idx])
        assert np.array_equal(mine, theirs), seed


def _tensor(rng, rows, cols, dtype, special=True):
    x = (rng.standard_normal((rows, cols)) * np.exp2(rng.integers(-6, 7, (rows, 1)))).astype(np.float32)
    if special:
        x.flat[rng.choice(x.size, max(1, x.size // 50), replace=False)] = 0.0
        sub = rng.choice(x.size, max(1, x.size // 200), replace=False)
        x.flat[sub] = (rng.integers(1, 1 << 23, sub.size).astype(np.uint32)
                       | (rng.integers(0, 2, sub.size).astype(np.uint32) << 31)).view(np.float32)
        x[0, :] = -0.0                                      # an all-negative-zero line
        x[1, :] *= np.float32(2.0 ** -120)                  # a line of tiny normals
    if dtype == "bf16":
        return ind.f32_to_bf16_bits_rne(x)
    return x


@pytest.mark.parametrize("name", NAMES)
@pytest.mark.parametrize("axis", [0, 1])
@pytest.mark.parametrize("hadamard", [False, True])
def test_sr_cast_matches_independent(oracle, name, axis, hadamard):
    """Every code byte and scale byte of a stochastic-rounding cast, on a
    ragged multi-line tensor, for both block axes and both scale layouts."""
    rng = np.random.default_rng(100 + fmt_id(name) + 10 * axis + 20 * hadamard)
    rows, cols = (96, 160) if axis == 1 else (160, 96)
    for dtype in ("f32", "bf16"):
        x = _tensor(rng, rows, cols, dtype)
        for seed in (42, 0xDEADBEEF00C0FFEE):
            for mma in (False, True):
                want_c, want_s = ind.quantize(x, axis, name, sr=True, seed=seed, hadamard=hadamard,
                                              sign_mask=SIGN_MASK, mma_layout=mma)
                got_c, got_s = oracle.quantize(x, axis, fmt_id(name), rnd=oracle.SR, seed=seed,
                                               hadamard=hadamard, sign_mask=SIGN_MASK,
                                               scale_layout=oracle.MMA if mma else oracle.PLAIN, fill=0)
                assert np.array_equal(got_c, want_c), (dtype, seed, mma)
                assert np.array_equal(got_s, want_s), (dtype, seed, mma)


@pytest.mark.parametrize("name", NAMES)
@pytest.mark.parametrize("axis", [0, 1])
def test_rne_cast_matches_independent(oracle, name, axis):
    """The same comparison for round-to-nearest-even, with the Hadamard on the
    strided axis."""
    rng = np.random.default_rng(200 + fmt_id(name) + 10 * axis)
    rows, cols = (64, 224) if axis == 1 else (224, 64)
    x = _tensor(rng, rows, cols, "f32")
    for hadamard in (False, True):
        want_c, want_s = ind.quantize(x, axis, name, hadamard=hadamard, sign_mask=SIGN_MASK, mma_layout=True)
        got_c, got_s = oracle.quantize(x, axis, fmt_id(name), hadamard=hadamard, sign_mask=SIGN_MASK,
                                       scale_layout=oracle.MMA, fill=0)
        assert np.array_equal(got_c, want_c)
        assert np.array_equal(got_s, want_s)


def test_sr_nonfinite_block(oracle):
    """A NaN or Inf in a block: scale 0xFF and zero codes under SR as well."""
    x = np.ones((4, 64), dtype=np.float32)
    x[1, 5] = np.inf
    x[2, 40] = np.nan
    want_c, want_s = ind.quantize(x, 1, "e2m1", sr=True, seed=9)
    got_c, got_s = oracle.quantize(x, 1, oracle.E2M1, rnd=oracle.SR, seed=9)
    assert np.array_equal(got_c, want_c) and np.array_equal(got_s, want_s)
    assert want_s.reshape(4, 2)[1, 0] == 255 and want_s.reshape(4, 2)[2, 1] == 255


@pytest.mark.parametrize("mistake", ["block_not_element", "input_coordinates", "word_not_quarter"])
def test_comparison_catches_index_mistakes(oracle, mistake):
    """The comparison above has teeth: a restatement given one of the
    plausible index mistakes (the block number where the element position
    belongs, the input's coordinates instead of the output's, one word per
    element) disagrees with the oracle."""
    rng = np.random.default_rng(7)
    rows, cols, seed = 64, 96, 42
    x = rng.standard_normal((rows, cols)).astype(np.float32)
    got_c, _ = oracle.quantize(x, 0, oracle.E2M1, rnd=oracle.SR, seed=seed)
    outer, inner = cols, rows
    o = np.arange(outer)[:, None]
    i = np.arange(inner)[None, :]
    if mistake == "block_not_element":
        idx = o * inner + i // 32 + i % 32
    elif mistake == "input_coordinates":
        idx = i * cols + o                      # row-major position in x
    else:
        idx = (o * inner + i) * 4
    idx = idx.astype(np.uint64)
    v = np.ascontiguousarray(x.T).reshape(outer, inner // 32, 32).astype(np.float64)
    amax = np.max(np.abs(v), axis=-1)
    _, ex = np.frexp(amax)
    e = np.clip(ex - 1 - 2, -127, 127)
    u = v * np.exp2(-e.astype(np.float64))[..., None]
    codes = ind.encode_sr("e2m1", u, ind.sr_bytes(seed, idx.reshape(outer, inner // 32, 32)))
    wrong = ind.pack_codes("e2m1", codes.reshape(outer, inner))
    assert not np.array_equal(wrong, got_c)
