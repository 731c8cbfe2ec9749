"""Tile staging of the column and dual casts: the TMA tensor-copy path (taken
for every input the ABI accepts) and the cp.async path (kept for inputs a
tensor map cannot describe, reached here through mx_debug_cast_force_cpasync)
give the oracle's bytes ("Microscaling Data Formats for Deep Learning",
summary page, section 3, along columns; with the fixed-sign Hadamard of
"Format-Aware Fusion for Fast FP4 Pretraining", abstract), and a staging wait
that runs out reports MX_ERR_TIMEOUT and leaves the context usable."""
import numpy as np
import pytest
import torch

from gpu_helpers import dev, first_mismatch, host, to_device
from microscaling_block_scaled_mx_b200 import inputs as I
from microscaling_block_scaled_mx_b200 import mx

pytestmark = pytest.mark.gpu

MASK = mx.DEFAULT_SIGN_MASK
FILL = 0xAB


@pytest.fixture
def cpasync():
    L = mx.lib()
    assert L.mx_debug_cast_force_cpasync(1) == 0
    yield
    L.mx_debug_cast_force_cpasync(0)


def col_cast(x, fmt, rnd, seed, had):
    R, C = x.shape
    codes = torch.full((C, mx.codes_row_bytes(fmt, R)), FILL, dtype=torch.uint8, device=dev())
    scales = torch.full((max(mx.scales_bytes("mma", C, R), 1),), FILL, dtype=torch.uint8, device=dev())
    mx.quantize(x, 0, fmt, rnd=rnd, seed=seed, hadamard=had, sign_mask=MASK, scale_layout="mma",
                codes=codes, scales=scales)
    torch.cuda.synchronize()
    return host(codes), host(scales)


def dual_cast(x, fmt, rnd_rows, rnd_cols, had):
    R, C = x.shape
    u8 = dict(dtype=torch.uint8, device=dev())
    out = (torch.full((R, mx.codes_row_bytes(fmt, C)), FILL, **u8),
           torch.full((max(mx.scales_bytes("mma", R, C), 1),), FILL, **u8),
           torch.full((C, mx.codes_row_bytes(fmt, R)), FILL, **u8),
           torch.full((max(mx.scales_bytes("mma", C, R), 1),), FILL, **u8))
    mx.quantize_dual(x, fmt, rnd_rows=rnd_rows, seed_rows=21, rnd_cols=rnd_cols, seed_cols=22, hadamard=had,
                     sign_mask=MASK, scale_layout="mma", out=out)
    torch.cuda.synchronize()
    return [host(t) for t in out]


def oracle_cols(oracle, x_np, fmt, rnd, seed, had):
    return oracle.quantize(x_np, 0, oracle.FORMATS[fmt], rnd=1 if rnd == "sr" else 0, seed=seed, hadamard=had,
                           sign_mask=MASK, scale_layout=1, fill=FILL)


def oracle_dual(oracle, x_np, fmt, rnd_rows, rnd_cols, had):
    f = oracle.FORMATS[fmt]
    cr, sr = oracle.quantize(x_np, 1, f, rnd=1 if rnd_rows == "sr" else 0, seed=21, scale_layout=1, fill=FILL)
    cc, sc = oracle.quantize(x_np, 0, f, rnd=1 if rnd_cols == "sr" else 0, seed=22, hadamard=had,
                             sign_mask=MASK, scale_layout=1, fill=FILL)
    return [cr, sr, cc, sc]


def same(got, want, what):
    for i, (g, w) in enumerate(zip(got, want)):
        g = g.reshape(-1)[:w.size].reshape(w.shape) if g.shape != w.shape else g
        assert np.array_equal(g, w), (what, i, first_mismatch(g, w))


def ragged_input(rows, cols, seed, bf16):
    rng = np.random.default_rng(seed)
    x = I.roundtrip_matrix(rows, cols, rng)
    return I.to_bf16_bits(x) if bf16 else x


# a ragged edge in both directions, several tiles each way
SHAPE = (288, 416)


@pytest.mark.parametrize("staging", ["tma", "cpasync"])
@pytest.mark.parametrize("bf16", [True, False])
@pytest.mark.parametrize("fmt,rnd,had", [("e2m1", "sr", True), ("e4m3", "rne", False), ("e2m3", "sr", False)])
def test_column_cast_staging(oracle, request, staging, bf16, fmt, rnd, had):
    if staging == "cpasync":
        request.getfixturevalue("cpasync")
    x = ragged_input(*SHAPE, 900 + bf16, bf16)
    same(col_cast(to_device(x), fmt, rnd, 7, had), oracle_cols(oracle, x, fmt, rnd, 7, had), (staging, bf16, fmt))


@pytest.mark.parametrize("staging", ["tma", "cpasync"])
@pytest.mark.parametrize("bf16", [True, False])
@pytest.mark.parametrize("fmt,rnd_rows,rnd_cols,had", [("e2m1", "rne", "sr", True), ("e4m3", "rne", "rne", False)])
def test_dual_cast_staging(oracle, request, staging, bf16, fmt, rnd_rows, rnd_cols, had):
    if staging == "cpasync":
        request.getfixturevalue("cpasync")
    x = ragged_input(*SHAPE, 910 + bf16, bf16)
    same(dual_cast(to_device(x), fmt, rnd_rows, rnd_cols, had), oracle_dual(oracle, x, fmt, rnd_rows, rnd_cols, had),
         (staging, bf16, fmt))


# 16 x 20 tiles of 128 x 128: more tiles than the resident grid, so the CTA
# that withholds its first copy has also issued its second one when it gives up
@pytest.mark.parametrize("kind", ["cols", "dual"])
def test_staging_wait_reports_timeout(oracle, kind):
    rng = np.random.default_rng(5)
    x_np = I.to_bf16_bits(rng.standard_normal((2048, 2560)).astype(np.float32))
    x = to_device(x_np)
    run = (lambda: col_cast(x, "e2m1", "sr", 3, True)) if kind == "cols" else \
          (lambda: dual_cast(x, "e2m1", "rne", "sr", True))
    assert mx.last_device_status() == 0
    assert mx.lib().mx_debug_cast_skip_tile(1) == 0
    run()
    assert mx.last_device_status() == -7
    assert mx.last_device_status() == 0          # read-and-clear
    got = run()
    assert mx.last_device_status() == 0
    small = x_np[:256, :384]
    want = oracle_cols(oracle, small, "e2m1", "sr", 3, True) if kind == "cols" else None
    # the context is usable: a full rerun is deterministic and a small cast matches the oracle
    assert all(np.array_equal(a, b) for a, b in zip(got, run()))
    sx = to_device(small)
    if kind == "cols":
        same(col_cast(sx, "e2m1", "sr", 3, True), want, kind)
    else:
        same(dual_cast(sx, "e2m1", "rne", "sr", True), oracle_dual(oracle, small, "e2m1", "rne", "sr", True), kind)


# The scales of a full 128 x 128 column tile leave through shared memory as one
# atom (and its copies); ragged tiles, the plain layout and a scale buffer
# that is not 16-byte aligned keep the per-byte stores.  Every path gives the
# oracle's bytes, and the bytes around an offset scale buffer stay untouched.
@pytest.mark.parametrize("sl", ["mma", "mma_x4", "plain"])
@pytest.mark.parametrize("offset", [0, 1])
def test_column_scales_staged_and_scattered(oracle, sl, offset):
    x = ragged_input(384, 416, 920 + offset, True)
    R, C = x.shape
    layout = {"plain": 0, "mma": 1, "mma_x4": 2}[sl]
    n = mx.scales_bytes(sl, C, R)
    codes = torch.full((C, mx.codes_row_bytes("e2m1", R)), FILL, dtype=torch.uint8, device=dev())
    buf = torch.full((n + 32,), FILL, dtype=torch.uint8, device=dev())
    scales = buf[offset:offset + n]
    mx.quantize(to_device(x), 0, "e2m1", rnd="sr", seed=4, hadamard=True, sign_mask=MASK, scale_layout=sl,
                codes=codes, scales=scales)
    torch.cuda.synchronize()
    wc, ws = oracle.quantize(x, 0, oracle.FORMATS["e2m1"], rnd=1, seed=4, hadamard=True, sign_mask=MASK,
                             scale_layout=layout, fill=FILL)
    got = host(buf)
    same([host(codes), got[offset:offset + n]], [wc, ws.reshape(-1)[:n]], (sl, offset))
    assert (got[:offset] == FILL).all() and (got[offset + n:] == FILL).all()
