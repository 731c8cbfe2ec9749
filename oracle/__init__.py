"""CPU oracle for the MX cast and the block-scaled GEMM.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` may import this package.  The product path
(the CUDA library and its Python binding) never imports, links or runs it, and
this package imports nothing from the product.

The arithmetic lives in ``mx_oracle.c`` (plain scalar C, fp64 where the pages
fix no precision, fp32 where the method itself works in fp32); this module
only compiles it with gcc and marshals numpy arrays through ctypes.

Sources: "Microscaling Data Formats for Deep Learning" (summary page,
sections 2-4) for the MX block, Algorithm 1 and the compute flow; "Format-Aware
Fusion for Fast FP4 Pretraining" (abstract) for stochastic rounding and the
fixed-sign 32-value Hadamard.  See the C file's header for the readings taken
where the pages are silent.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "mx_oracle.c")
_BUILD_DIR = os.path.join(_HERE, "_build")
_LIB_PATH = os.path.join(_BUILD_DIR, "libmxoracle.so")

E4M3, E5M2, E2M3, E3M2, E2M1, INT8 = range(6)
FORMATS = {"e4m3": E4M3, "e5m2": E5M2, "e2m3": E2M3, "e3m2": E3M2, "e2m1": E2M1, "int8": INT8}
BITS = {E4M3: 8, E5M2: 8, E2M3: 6, E3M2: 6, E2M1: 4, INT8: 8}
F32, BF16 = 0, 1
RNE, SR = 0, 1
PLAIN, MMA, MMA_X4 = 0, 1, 2

_lock = threading.Lock()
_lib = None

_i64 = ctypes.c_int64
_vp = ctypes.c_void_p


def build(force: bool = False) -> str:
    """Compile the oracle with gcc (no fast-math, no FMA contraction)."""
    os.makedirs(_BUILD_DIR, exist_ok=True)
    if (not force and os.path.exists(_LIB_PATH)
            and os.path.getmtime(_LIB_PATH) >= os.path.getmtime(_SRC)):
        return _LIB_PATH
    tmp = _LIB_PATH + f".tmp{os.getpid()}"
    cmd = ["gcc", "-O2", "-std=c11", "-fopenmp", "-ffp-contract=off", "-fno-fast-math",
           "-fPIC", "-shared", "-o", tmp, _SRC, "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def lib() -> ctypes.CDLL:
    global _lib
    with _lock:
        if _lib is None:
            path = build()
            L = ctypes.CDLL(path)
            L.mxref_decode_elem.restype = ctypes.c_double
            L.mxref_decode_elem.argtypes = [ctypes.c_int, ctypes.c_uint]
            L.mxref_encode_rne.restype = ctypes.c_uint
            L.mxref_encode_rne.argtypes = [ctypes.c_int, ctypes.c_double]
            L.mxref_encode_sr.restype = ctypes.c_uint
            L.mxref_encode_sr.argtypes = [ctypes.c_int, ctypes.c_double, ctypes.c_uint]
            L.mxref_emax.restype = ctypes.c_int
            L.mxref_emax.argtypes = [ctypes.c_int]
            L.mxref_max.restype = ctypes.c_double
            L.mxref_max.argtypes = [ctypes.c_int]
            L.mxref_fmix32.restype = ctypes.c_uint32
            L.mxref_fmix32.argtypes = [ctypes.c_uint32]
            L.mxref_sr_byte.restype = ctypes.c_uint
            L.mxref_sr_byte.argtypes = [ctypes.c_uint64, ctypes.c_uint64]
            L.mxref_hadamard32.restype = None
            L.mxref_hadamard32.argtypes = [_vp, ctypes.c_uint32]
            L.mxref_codes_bytes.restype = _i64
            L.mxref_codes_bytes.argtypes = [ctypes.c_int, _i64, _i64]
            L.mxref_scales_bytes.restype = _i64
            L.mxref_scales_bytes.argtypes = [ctypes.c_int, _i64, _i64]
            L.mxref_quantize.restype = ctypes.c_int
            L.mxref_quantize.argtypes = [_vp, ctypes.c_int, _i64, _i64, _i64, ctypes.c_int,
                                         ctypes.c_int, ctypes.c_int, ctypes.c_uint64,
                                         ctypes.c_int, ctypes.c_uint32, _vp, _vp, ctypes.c_int]
            L.mxref_quantize_shard.restype = ctypes.c_int
            L.mxref_quantize_shard.argtypes = [_vp, ctypes.c_int, _i64, _i64, _i64, ctypes.c_int,
                                               ctypes.c_int, ctypes.c_int, ctypes.c_uint64,
                                               ctypes.c_int, ctypes.c_uint32, _i64, _i64, _i64, _i64,
                                               _vp, _vp, ctypes.c_int]
            L.mxref_nvfp4_scales_bytes.restype = _i64
            L.mxref_nvfp4_scales_bytes.argtypes = [ctypes.c_int, _i64, _i64]
            L.mxref_nvfp4_quantize.restype = ctypes.c_int
            L.mxref_nvfp4_quantize.argtypes = [_vp, ctypes.c_int, _i64, _i64, _i64, _i64, _vp, _vp,
                                               ctypes.c_int, _vp]
            L.mxref_nvfp4_dequantize.restype = ctypes.c_int
            L.mxref_nvfp4_dequantize.argtypes = [_vp, _vp, ctypes.c_int, _i64, _i64, _vp, _i64, _vp]
            L.mxref_dequantize.restype = ctypes.c_int
            L.mxref_dequantize.argtypes = [_vp, _vp, ctypes.c_int, ctypes.c_int, _i64, _i64, _vp]
            L.mxref_round_f32.restype = None
            L.mxref_round_f32.argtypes = [_vp, _vp, _i64]
            L.mxref_round_bf16.restype = None
            L.mxref_round_bf16.argtypes = [_vp, _vp, _i64]
            L.mxref_gemm_f64.restype = ctypes.c_int
            L.mxref_gemm_f64.argtypes = [_vp, _vp, ctypes.c_int, _vp, _vp, ctypes.c_int,
                                         _i64, _i64, _i64, ctypes.c_double, ctypes.c_int,
                                         _vp, _vp]
            L.mxref_gemm_entries.restype = ctypes.c_int
            L.mxref_gemm_entries.argtypes = [_vp, _vp, ctypes.c_int, _vp, _vp, ctypes.c_int,
                                             _i64, ctypes.c_double, ctypes.c_int,
                                             _vp, _vp, _i64, _vp, _vp]
            _lib = L
    return _lib


def _ptr(a: np.ndarray) -> int:
    assert a.flags["C_CONTIGUOUS"], "oracle arrays must be C-contiguous"
    return a.ctypes.data


class OracleError(RuntimeError):
    pass


def _check(rc: int, what: str) -> None:
    if rc != 0:
        raise OracleError(f"{what} failed with status {rc}")


# --------------------------------------------------------------------------
# scalar helpers
# --------------------------------------------------------------------------

def decode_elem(fmt: int, code: int) -> float:
    return lib().mxref_decode_elem(fmt, code)


def encode_rne(fmt: int, u: float) -> int:
    return lib().mxref_encode_rne(fmt, u)


def encode_sr(fmt: int, u: float, r: int) -> int:
    return lib().mxref_encode_sr(fmt, u, r)


def emax(fmt: int) -> int:
    return lib().mxref_emax(fmt)


def max_value(fmt: int) -> float:
    return lib().mxref_max(fmt)


def fmix32(h: int) -> int:
    return lib().mxref_fmix32(h & 0xFFFFFFFF)


def sr_byte(seed: int, idx: int) -> int:
    return lib().mxref_sr_byte(seed, idx)


def hadamard32(x: np.ndarray, sign_mask: int) -> np.ndarray:
    v = np.ascontiguousarray(x, dtype=np.float32).copy()
    assert v.shape == (32,)
    lib().mxref_hadamard32(_ptr(v), sign_mask)
    return v


def codes_bytes(fmt: int, outer: int, inner: int) -> int:
    return lib().mxref_codes_bytes(fmt, outer, inner)


def scales_bytes(sl: int, outer: int, inner: int) -> int:
    return lib().mxref_scales_bytes(sl, outer, inner)


# --------------------------------------------------------------------------
# tensor-level calls (same parameters as the C-ABI, host arrays)
# --------------------------------------------------------------------------

def quantize(x: np.ndarray, block_axis: int, fmt: int, rnd: int = RNE, seed: int = 0,
             hadamard: bool = False, sign_mask: int = 0, scale_layout: int = PLAIN,
             ldx: int | None = None, cols: int | None = None, fill: int = 0, shard=None):
    """Cast a 2-D float32 array, or bf16 given as a uint16 bit array, to MX.

    With ``cols``/``ldx`` given, x is a pitched buffer: the logical tensor is
    its first ``cols`` columns and rows are ``ldx`` elements apart.
    ``shard`` = (row0, col0, total_rows, total_cols) places x at (row0, col0)
    of a larger tensor: stochastic rounding then uses the whole tensor's
    element positions (mxref_quantize_shard).

    Returns (codes, scales) as uint8 arrays: codes has one row per block-axis
    line (transposed for block_axis=0); scales is flat in the chosen layout.
    """
    if x.dtype == np.float32:
        xdt = F32
    elif x.dtype == np.uint16:
        xdt = BF16
    else:
        raise TypeError("x must be float32 or bf16 bits (uint16)")
    x = np.ascontiguousarray(x)
    rows, full_cols = x.shape
    cols = full_cols if cols is None else cols
    ld = full_cols if ldx is None else ldx
    assert ld <= full_cols and cols <= ld
    outer, inner = (rows, cols) if block_axis == 1 else (cols, rows)
    row_bytes = codes_bytes(fmt, 1, inner) if inner % 32 == 0 else 0
    codes = np.full((outer, row_bytes), fill, dtype=np.uint8)
    scales = np.full(max(scales_bytes(scale_layout, outer, inner), 0), fill, dtype=np.uint8)
    if shard is None:
        rc = lib().mxref_quantize(_ptr(x), xdt, rows, cols, ld, block_axis, fmt, rnd, seed,
                                  1 if hadamard else 0, sign_mask & 0xFFFFFFFF,
                                  _ptr(codes), _ptr(scales), scale_layout)
    else:
        row0, col0, total_rows, total_cols = shard
        rc = lib().mxref_quantize_shard(_ptr(x), xdt, rows, cols, ld, block_axis, fmt, rnd, seed,
                                        1 if hadamard else 0, sign_mask & 0xFFFFFFFF,
                                        row0, col0, total_rows, total_cols,
                                        _ptr(codes), _ptr(scales), scale_layout)
    _check(rc, "mxref_quantize")
    return codes, scales


def dequantize(codes: np.ndarray, scales: np.ndarray, fmt: int, outer: int, inner: int,
               scale_layout: int = PLAIN) -> np.ndarray:
    """Exact decode to float64 (v = 2^(s-127) * P; 0xFF scale -> NaN)."""
    y = np.empty((outer, inner), dtype=np.float64)
    rc = lib().mxref_dequantize(_ptr(np.ascontiguousarray(codes)),
                                _ptr(np.ascontiguousarray(scales)), fmt, scale_layout,
                                outer, inner, _ptr(y))
    _check(rc, "mxref_dequantize")
    return y


def round_f32(y: np.ndarray) -> np.ndarray:
    y = np.ascontiguousarray(y, dtype=np.float64)
    out = np.empty(y.shape, dtype=np.float32)
    lib().mxref_round_f32(_ptr(y), _ptr(out), y.size)
    return out


def round_bf16(y: np.ndarray) -> np.ndarray:
    """Round-to-nearest-even double -> bf16, returned as uint16 bits."""
    y = np.ascontiguousarray(y, dtype=np.float64)
    out = np.empty(y.shape, dtype=np.uint16)
    lib().mxref_round_bf16(_ptr(y), _ptr(out), y.size)
    return out


def gemm(a_codes, a_scales, fa, b_codes, b_scales, fb, M, N, K, alpha=1.0,
         scale_layout: int = MMA):
    """C = alpha * A * B^T, exact decode, fp64 sum; returns (C, bound)."""
    c = np.empty((M, N), dtype=np.float64)
    bound = np.empty((M, N), dtype=np.float64)
    rc = lib().mxref_gemm_f64(_ptr(np.ascontiguousarray(a_codes)),
                              _ptr(np.ascontiguousarray(a_scales)), fa,
                              _ptr(np.ascontiguousarray(b_codes)),
                              _ptr(np.ascontiguousarray(b_scales)), fb,
                              M, N, K, float(alpha), scale_layout, _ptr(c), _ptr(bound))
    _check(rc, "mxref_gemm_f64")
    return c, bound


def gemm_entries(a_codes, a_scales, fa, b_codes, b_scales, fb, K, ms, ns, alpha=1.0,
                 scale_layout: int = MMA):
    """The same sum for selected (m, n) entries only; returns (c, bound)."""
    ms = np.ascontiguousarray(ms, dtype=np.int64)
    ns = np.ascontiguousarray(ns, dtype=np.int64)
    assert ms.shape == ns.shape
    c = np.empty(ms.shape, dtype=np.float64)
    bound = np.empty(ms.shape, dtype=np.float64)
    rc = lib().mxref_gemm_entries(_ptr(np.ascontiguousarray(a_codes)),
                                  _ptr(np.ascontiguousarray(a_scales)), fa,
                                  _ptr(np.ascontiguousarray(b_codes)),
                                  _ptr(np.ascontiguousarray(b_scales)), fb,
                                  K, float(alpha), scale_layout, _ptr(ms), _ptr(ns),
                                  ms.size, _ptr(c), _ptr(bound))
    _check(rc, "mxref_gemm_entries")
    return c, bound


def gemm_decoded(a_codes, a_scales, fa, b_codes, b_scales, fb, M, N, K, alpha=1.0,
                 rows=None, scale_layout: int = MMA):
    """The same C = alpha * A * B^T with numpy's fp64 matmul as the summation step.

    Both operands are decoded exactly by the oracle (mxref_dequantize); the
    dot products are then an fp64 matrix product, whose rounding error
    (about K * 2^-53 relative to sum |a b|) is far below any tolerance used.
    `rows` restricts the result to those rows of A.  Returns (C, bound).
    """
    A = dequantize(a_codes, a_scales, fa, M, K, scale_layout)
    B = dequantize(b_codes, b_scales, fb, N, K, scale_layout)
    if rows is not None:
        A = A[np.asarray(rows)]
    c = alpha * (A @ B.T)
    bound = abs(alpha) * (np.abs(A) @ np.abs(B).T)
    return c, bound


# --------------------------------------------------------------------------
# NVFP4 scale domains (reading; see mx_oracle.c): 16-element E2M1 blocks with
# an E4M3 block scale and one fp32 encode scale per domain.
# --------------------------------------------------------------------------

NV_SCALE_NAN = 0x7F


def nvfp4_scales_bytes(sl: int, rows: int, cols: int) -> int:
    return lib().mxref_nvfp4_scales_bytes(sl, rows, cols)


def nvfp4_quantize(x: np.ndarray, domain_lines: int = 0, scale_layout: int = PLAIN, fill: int = 0):
    """Cast a rows x cols float32 array (or bf16 bits as uint16) along its rows
    to NVFP4.  domain_lines 0: one global domain; else one domain per that many
    rows.  Returns (codes, scales, enc_scales)."""
    if x.dtype == np.float32:
        xdt = F32
    elif x.dtype == np.uint16:
        xdt = BF16
    else:
        raise TypeError("x must be float32 or bf16 bits (uint16)")
    x = np.ascontiguousarray(x)
    rows, cols = x.shape
    n_dom = 1 if domain_lines == 0 else (rows + domain_lines - 1) // domain_lines
    codes = np.full((rows, cols // 2), fill, dtype=np.uint8)
    scales = np.full(max(nvfp4_scales_bytes(scale_layout, rows, cols), 0), fill, dtype=np.uint8)
    enc = np.zeros(max(n_dom, 1), dtype=np.float32)
    rc = lib().mxref_nvfp4_quantize(_ptr(x), xdt, rows, cols, cols, domain_lines, _ptr(codes), _ptr(scales),
                                    scale_layout, _ptr(enc))
    _check(rc, "mxref_nvfp4_quantize")
    return codes, scales, enc


def nvfp4_dequantize(codes, scales, enc_scales, rows: int, cols: int, domain_lines: int = 0,
                     scale_layout: int = PLAIN) -> np.ndarray:
    y = np.empty((rows, cols), dtype=np.float64)
    rc = lib().mxref_nvfp4_dequantize(_ptr(np.ascontiguousarray(codes)), _ptr(np.ascontiguousarray(scales)),
                                      scale_layout, rows, cols,
                                      _ptr(np.ascontiguousarray(enc_scales, dtype=np.float32)),
                                      domain_lines, _ptr(y))
    _check(rc, "mxref_nvfp4_dequantize")
    return y


def nvfp4_gemm_decoded(a, b, M, N, K, alpha=1.0, a_lines=0, b_lines=0, scale_layout: int = MMA, rows=None):
    """C = alpha * A * B^T on NVFP4 operands a = (codes, scales, enc) (M x K)
    and b (N x K), both cast along K: exact decode, numpy fp64 matrix product.
    Returns (C, bound) with bound = |alpha| * sum_k |a b|."""
    A = nvfp4_dequantize(a[0], a[1], a[2], M, K, a_lines, scale_layout)
    B = nvfp4_dequantize(b[0], b[1], b[2], N, K, b_lines, scale_layout)
    if rows is not None:
        A = A[np.asarray(rows)]
    return alpha * (A @ B.T), abs(alpha) * (np.abs(A) @ np.abs(B).T)
