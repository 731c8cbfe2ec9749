"""GPU parity of the dual cast (both quantizations of one tensor from a single
read) against the oracle: each of its two outputs must equal, bit for bit, the
oracle's Algorithm 1 ("Microscaling Data Formats for Deep Learning", summary
page, section 3) along that axis, with that axis' rounding, seed and (for the
column output) fixed-sign Hadamard ("Format-Aware Fusion for Fast FP4
Pretraining", abstract)."""
import numpy as np
import pytest
import torch

from gpu_helpers import FMTS, dev, first_mismatch, host, to_device
from microscaling_block_scaled_mx_b200 import inputs as I
from microscaling_block_scaled_mx_b200 import mx

pytestmark = pytest.mark.gpu

MASK = mx.DEFAULT_SIGN_MASK
FILL = 0xAB


def gpu_dual(x_np, fmt, rnd_rows, seed_rows, rnd_cols, seed_cols, hadamard, sl="mma", cols=None):
    x = to_device(x_np)
    if cols is not None:
        x = x[:, :cols]
    R, C = x.shape
    u8 = dict(dtype=torch.uint8, device=dev())
    out = (torch.full((R, mx.codes_row_bytes(fmt, C)), FILL, **u8),
           torch.full((max(mx.scales_bytes(sl, R, C), 1),), FILL, **u8),
           torch.full((C, mx.codes_row_bytes(fmt, R)), FILL, **u8),
           torch.full((max(mx.scales_bytes(sl, C, R), 1),), FILL, **u8))
    mx.quantize_dual(x, fmt, rnd_rows=rnd_rows, seed_rows=seed_rows, rnd_cols=rnd_cols, seed_cols=seed_cols,
                     hadamard=hadamard, sign_mask=MASK, scale_layout=sl, out=out)
    torch.cuda.synchronize()
    return [host(t) for t in out]


def oracle_both(oracle, x_np, fmt, rnd_rows, seed_rows, rnd_cols, seed_cols, hadamard, sl="mma", cols=None):
    f = oracle.FORMATS[fmt]
    kw = {"cols": cols, "ldx": x_np.shape[1]} if cols is not None else {}
    layout = 1 if sl == "mma" else 0
    cr, sr = oracle.quantize(x_np, 1, f, rnd=1 if rnd_rows == "sr" else 0, seed=seed_rows,
                             scale_layout=layout, fill=FILL, **kw)
    cc, sc = oracle.quantize(x_np, 0, f, rnd=1 if rnd_cols == "sr" else 0, seed=seed_cols, hadamard=hadamard,
                             sign_mask=MASK, scale_layout=layout, fill=FILL, **kw)
    return [cr, sr, cc, sc]


def assert_dual(got, want, what):
    names = ("row codes", "row scales", "col codes", "col scales")
    for name, g, w in zip(names, got, want):
        g = g.reshape(-1)[:w.size].reshape(w.shape) if name.endswith("scales") else g
        assert g.shape == w.shape, (what, name, g.shape, w.shape)
        assert np.array_equal(g, w), (what, name, first_mismatch(g, w))


def mixed_input(rows, cols, seed, bf16):
    rng = np.random.default_rng(seed)
    x = I.roundtrip_matrix(rows, cols, rng)
    flat = x.reshape(-1)
    flat[rng.choice(flat.size, max(1, flat.size // 500), replace=False)] *= np.float32(1e3)
    flat[rng.choice(flat.size, max(1, flat.size // 300), replace=False)] = np.float32(-0.0)
    return I.to_bf16_bits(x) if bf16 else x


# 128 x 128 tiles: a single block, one full tile, ragged rows and columns,
# several tiles in both directions
SHAPES = [(32, 32), (128, 128), (160, 224), (288, 416)]
ROUNDINGS = [("rne", "rne"), ("sr", "sr"), ("rne", "sr")]


@pytest.mark.parametrize("fmt", FMTS)
@pytest.mark.parametrize("bf16", [True, False])
@pytest.mark.parametrize("rnd_rows,rnd_cols", ROUNDINGS)
def test_dual_parity(oracle, fmt, bf16, rnd_rows, rnd_cols):
    for i, (r, c) in enumerate(SHAPES):
        x = mixed_input(r, c, 400 + i, bf16)
        for had in (False, True):
            args = (fmt, rnd_rows, 11, rnd_cols, 12, had)
            assert_dual(gpu_dual(x, *args), oracle_both(oracle, x, *args), (args, bf16, r, c))


@pytest.mark.parametrize("sl", ["mma", "plain"])
def test_dual_plain_scales_and_pitch(oracle, sl):
    rng = np.random.default_rng(401)
    big = I.to_bf16_bits(rng.standard_t(3, size=(96, 200)).astype(np.float32))
    args = ("e2m1", "sr", 5, "sr", 6, True)
    assert_dual(gpu_dual(big, *args, sl=sl, cols=160), oracle_both(oracle, big, *args, sl=sl, cols=160), sl)


def test_dual_special_blocks(oracle):
    x = np.ones((64, 64), dtype=np.float32)
    x[0, 3] = np.nan                       # NaN: its row block and column block become NaN blocks
    x[5, 40] = np.inf
    x[32:64, 0:32] = 0.0                   # an all-zero tile quarter
    x[33, 33] = np.float32(1e-40)          # a subnormal in a normal block
    x[40:48, 40:64] = np.float32(-3e-39)   # subnormals only in some row blocks
    for fmt in FMTS:
        args = (fmt, "rne", 0, "sr", 9, False)
        assert_dual(gpu_dual(x, *args), oracle_both(oracle, x, *args), fmt)


def test_dual_wgrad_operand_full_size(oracle):
    """dY of the weight-gradient step, 16384 x 4096 bf16 (Student-t, 3 degrees of
    freedom): rows RNE for the data-gradient GEMM, columns Hadamard + SR for
    the weight-gradient GEMM; every code and scale against the oracle."""
    dy, _ = I.wgrad_operands()
    args = ("e2m1", "rne", 0, "sr", 42, True)
    assert_dual(gpu_dual(dy, *args), oracle_both(oracle, dy, *args), "dY")


def test_dual_matches_two_single_casts():
    """The dual kernel's outputs equal the two single-axis casts on a large
    Llama-3 activation (8192 x 4096), which are themselves oracle-checked."""
    rng = np.random.default_rng(402)
    x = to_device(I.to_bf16_bits(rng.standard_normal((8192, 4096)).astype(np.float32)))
    cr, sr, cc, sc = mx.quantize_dual(x, "e4m3", rnd_rows="sr", seed_rows=1, rnd_cols="sr", seed_cols=2)
    r1 = mx.quantize(x, 1, "e4m3", rnd="sr", seed=1)
    r0 = mx.quantize(x, 0, "e4m3", rnd="sr", seed=2)
    torch.cuda.synchronize()
    assert torch.equal(cr, r1[0]) and torch.equal(cc, r0[0])
    n1, n0 = mx.scales_bytes("mma", 8192, 4096), mx.scales_bytes("mma", 4096, 8192)
    assert torch.equal(sr[:n1], r1[1][:n1]) and torch.equal(sc[:n0], r0[1][:n0])


def test_dual_empty_and_shape_errors():
    z = torch.empty((0, 64), dtype=torch.bfloat16, device=dev())
    mx.quantize_dual(z, "e4m3", out=(z, z, z, z))             # empty: a no-op
    x = torch.zeros((48, 64), dtype=torch.bfloat16, device=dev())
    with pytest.raises(mx.MxError, match="MX_ERR_SHAPE"):
        mx.quantize_dual(x, "e4m3")                          # 48 rows: not a multiple of 32
