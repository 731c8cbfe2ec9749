"""Thin Python binding of libmx (include/mx.h): argument marshalling only.

Every step of the cast and of the GEMM runs in the CUDA kernels of libmx.so;
PyTorch only provides device memory and streams.  There is no CPU fallback:
if libmx.so is missing or fails to load, every call raises.

Functions take and return torch tensors on the current CUDA device; bf16 and
fp32 inputs are accepted, codes and scales are uint8 tensors laid out as
documented in include/mx.h.
"""
from __future__ import annotations

import ctypes
import os
import threading

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libmx.so")

FMT = {"e4m3": 0, "e5m2": 1, "e2m3": 2, "e3m2": 3, "e2m1": 4, "int8": 5}
FMT_BITS = {0: 8, 1: 8, 2: 6, 3: 6, 4: 4, 5: 8}
ROUND = {"rne": 0, "sr": 1}
LAYOUT = {"plain": 0, "mma": 1, "mma_x4": 2}
DTYPE = {torch.float32: 0, torch.bfloat16: 1}
DEFAULT_SIGN_MASK = 0x6A09E667

MX_OK = 0
STATUS_NAMES = {0: "MX_OK", -1: "MX_ERR_ARG", -2: "MX_ERR_ALIGN", -3: "MX_ERR_SHAPE",
                -4: "MX_ERR_UNSUPPORTED", -5: "MX_ERR_SR_RANGE", -6: "MX_ERR_CUDA",
                -7: "MX_ERR_TIMEOUT", -8: "MX_ERR_BOUNDS"}


class MxError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__(f"{what}: {status_str(status)} ({status})")


class _Precond(ctypes.Structure):
    _fields_ = [("hadamard", ctypes.c_int32), ("sign_mask", ctypes.c_uint32)]


class _Shard(ctypes.Structure):
    _fields_ = [("row0", ctypes.c_int64), ("col0", ctypes.c_int64),
                ("total_rows", ctypes.c_int64), ("total_cols", ctypes.c_int64)]


_lock = threading.Lock()
_lib = None


def lib() -> ctypes.CDLL:
    """Load libmx.so (raises if it has not been built)."""
    global _lib
    with _lock:
        if _lib is None:
            if not os.path.exists(LIB_PATH):
                raise RuntimeError(
                    f"libmx.so not found at {LIB_PATH}; build it with "
                    "`python -m microscaling_block_scaled_mx_b200.build`")
            L = ctypes.CDLL(LIB_PATH)
            vp, i64, i32, u32, u64 = (ctypes.c_void_p, ctypes.c_int64, ctypes.c_int,
                                      ctypes.c_uint32, ctypes.c_uint64)
            L.mx_quantize.restype = i32
            L.mx_quantize.argtypes = [vp, i32, i64, i64, i64, i32, i32, i32, u64,
                                      ctypes.POINTER(_Precond), vp, vp, i32, vp]
            L.mx_quantize_shard.restype = i32
            L.mx_quantize_shard.argtypes = [vp, i32, i64, i64, i64, i32, i32, i32, u64,
                                            ctypes.POINTER(_Precond), ctypes.POINTER(_Shard), vp, vp, i32, vp]
            L.mx_quantize_dual_shard.restype = i32
            L.mx_quantize_dual_shard.argtypes = [vp, i32, i64, i64, i64, i32, i32, u64, i32, u64,
                                                 ctypes.POINTER(_Precond), ctypes.POINTER(_Shard),
                                                 vp, vp, vp, vp, i32, vp]
            L.mx_quantize_dual.restype = i32
            L.mx_quantize_dual.argtypes = [vp, i32, i64, i64, i64, i32, i32, u64, i32, u64,
                                           ctypes.POINTER(_Precond), vp, vp, vp, vp, i32, vp]
            L.mx_quantize_nvfp4.restype = i32
            L.mx_quantize_nvfp4.argtypes = [vp, i32, i64, i64, i64, i64, vp, vp, i32, vp, vp]
            L.mx_nvfp4_scales_bytes.restype = ctypes.c_size_t
            L.mx_nvfp4_scales_bytes.argtypes = [i32, i64, i64]
            L.mx_nvfp4_domains.restype = i64
            L.mx_nvfp4_domains.argtypes = [i64, i64]
            L.mx_dequantize.restype = i32
            L.mx_dequantize.argtypes = [vp, vp, i32, i32, i64, i64, vp, i32, i64, vp]
            L.mx_gemm.restype = i32
            L.mx_gemm.argtypes = [vp, vp, i32, vp, vp, i32, i64, i64, i64, ctypes.c_float,
                                  vp, i32, i64, vp, ctypes.c_size_t, vp]
            L.mx_gemm_nvfp4_x4.restype = i32
            L.mx_gemm_nvfp4_x4.argtypes = [vp, vp, vp, i64, vp, vp, vp, i64, i64, i64, i64, ctypes.c_float,
                                           vp, i32, i64, vp]
            L.mx_gemm_nvfp4.restype = i32
            L.mx_gemm_nvfp4.argtypes = [vp, vp, vp, i64, vp, vp, vp, i64, i64, i64, i64, ctypes.c_float,
                                        vp, i32, i64, vp]
            L.mx_gemm_x4.restype = i32
            L.mx_gemm_x4.argtypes = [vp, vp, i32, vp, vp, i32, i64, i64, i64, ctypes.c_float, vp, i32, i64, vp]
            L.mx_gemm_quantize_x4.restype = i32
            L.mx_gemm_quantize_x4.argtypes = [vp, vp, i32, vp, vp, i32, i64, i64, i64, ctypes.c_float,
                                              i32, i32, u64, vp, vp, i32, vp]
            L.mx_gemm_quantize.restype = i32
            L.mx_gemm_quantize.argtypes = [vp, vp, i32, vp, vp, i32, i64, i64, i64, ctypes.c_float,
                                           i32, i32, u64, vp, vp, i32, vp]
            L.mx_codes_bytes.restype = ctypes.c_size_t
            L.mx_codes_bytes.argtypes = [i32, i64, i64]
            L.mx_scales_bytes.restype = ctypes.c_size_t
            L.mx_scales_bytes.argtypes = [i32, i64, i64]
            L.mx_gemm_workspace_bytes.restype = ctypes.c_size_t
            L.mx_gemm_workspace_bytes.argtypes = [i64, i64, i64]
            L.mx_last_device_status.restype = i32
            L.mx_last_device_status.argtypes = [vp]
            L.mx_status_str.restype = ctypes.c_char_p
            L.mx_status_str.argtypes = [i32]
            L.mx_abi_version.restype = i32
            L.mx_abi_version.argtypes = []
            L.mx_debug_gemm_skip_stage.restype = i32
            L.mx_debug_gemm_skip_stage.argtypes = [i32]
            L.mx_debug_gemm_force_kernel.restype = i32
            L.mx_debug_gemm_force_kernel.argtypes = [i32]
            L.mx_debug_cast_force_cpasync.restype = i32
            L.mx_debug_cast_force_cpasync.argtypes = [i32]
            L.mx_debug_cast_skip_tile.restype = i32
            L.mx_debug_cast_skip_tile.argtypes = [i32]
            L.mx_debug_cast_cut_codes_cap.restype = i32
            L.mx_debug_cast_cut_codes_cap.argtypes = [i64]
            _lib = L
    return _lib


def status_str(status: int) -> str:
    return lib().mx_status_str(status).decode()


def _fmt(f) -> int:
    return FMT[f] if isinstance(f, str) else int(f)


def _layout(sl) -> int:
    return LAYOUT[sl] if isinstance(sl, str) else int(sl)


def _stream(stream) -> int:
    s = stream if stream is not None else torch.cuda.current_stream()
    return s.cuda_stream


def _check(rc: int, what: str) -> None:
    if rc != MX_OK:
        raise MxError(rc, what)


def codes_bytes(fmt, outer: int, inner: int) -> int:
    return lib().mx_codes_bytes(_fmt(fmt), outer, inner)


def scales_bytes(scale_layout, outer: int, inner: int) -> int:
    return lib().mx_scales_bytes(_layout(scale_layout), outer, inner)


def codes_row_bytes(fmt, inner: int) -> int:
    return inner * FMT_BITS[_fmt(fmt)] // 8


def quantize(x: torch.Tensor, block_axis: int = 1, fmt="e4m3", rnd="rne", seed: int = 0,
             hadamard: bool = False, sign_mask: int = DEFAULT_SIGN_MASK, scale_layout="mma",
             codes: torch.Tensor | None = None, scales: torch.Tensor | None = None,
             stream=None, shard=None):
    """MX cast of a 2-D CUDA tensor (rows x cols, row pitch x.stride(0)).

    Returns (codes, scales): codes is (outer, packed_inner_bytes) uint8 with
    outer = rows for block_axis=1 and cols for block_axis=0; scales is flat.
    shard = (row0, col0, total_rows, total_cols) casts x as the piece at
    (row0, col0) of a larger tensor (mx_quantize_shard).
    """
    if x.dim() != 2 or x.stride(1) != 1:
        raise ValueError("x must be 2-D with unit column stride")
    if x.dtype not in DTYPE:
        raise TypeError("x must be float32 or bfloat16")
    f = _fmt(fmt)
    sl = _layout(scale_layout)
    rows, cols = x.shape
    outer, inner = (rows, cols) if block_axis == 1 else (cols, rows)
    if codes is None:
        codes = torch.empty((outer, codes_row_bytes(f, inner)), dtype=torch.uint8, device=x.device)
    if scales is None:
        scales = torch.empty(max(scales_bytes(sl, outer, inner), 1), dtype=torch.uint8, device=x.device)
    pre = _Precond(1 if hadamard else 0, sign_mask & 0xFFFFFFFF)
    r = ROUND[rnd] if isinstance(rnd, str) else int(rnd)
    if shard is None:
        rc = lib().mx_quantize(x.data_ptr(), DTYPE[x.dtype], rows, cols, x.stride(0), block_axis, f,
                               r, seed & (2**64 - 1), ctypes.byref(pre), codes.data_ptr(), scales.data_ptr(),
                               sl, _stream(stream))
        _check(rc, "mx_quantize")
    else:
        sh = _Shard(*shard)
        rc = lib().mx_quantize_shard(x.data_ptr(), DTYPE[x.dtype], rows, cols, x.stride(0), block_axis, f,
                                     r, seed & (2**64 - 1), ctypes.byref(pre), ctypes.byref(sh),
                                     codes.data_ptr(), scales.data_ptr(), sl, _stream(stream))
        _check(rc, "mx_quantize_shard")
    return codes, scales


def quantize_dual(x: torch.Tensor, fmt="e4m3", rnd_rows="rne", seed_rows: int = 0, rnd_cols="rne",
                  seed_cols: int = 0, hadamard: bool = False, sign_mask: int = DEFAULT_SIGN_MASK,
                  scale_layout="mma", out=None, stream=None, shard=None):
    """Both MX casts of a 2-D CUDA tensor from one read of it.

    Returns (codes_rows, scales_rows, codes_cols, scales_cols): the results of
    quantize(x, 1, ...) with (rnd_rows, seed_rows) and of quantize(x, 0, ...)
    with (rnd_cols, seed_cols, hadamard); `out` may supply the four buffers.
    shard = (row0, col0, total_rows, total_cols) casts x as that piece of a
    larger tensor (mx_quantize_dual_shard).
    """
    if x.dim() != 2 or x.stride(1) != 1:
        raise ValueError("x must be 2-D with unit column stride")
    if x.dtype not in DTYPE:
        raise TypeError("x must be float32 or bfloat16")
    f = _fmt(fmt)
    sl = _layout(scale_layout)
    rows, cols = x.shape
    if out is None:
        u8 = dict(dtype=torch.uint8, device=x.device)
        out = (torch.empty((rows, codes_row_bytes(f, cols)), **u8),
               torch.empty(max(scales_bytes(sl, rows, cols), 1), **u8),
               torch.empty((cols, codes_row_bytes(f, rows)), **u8),
               torch.empty(max(scales_bytes(sl, cols, rows), 1), **u8))
    cr, sr_, cc, sc = out
    pre = _Precond(1 if hadamard else 0, sign_mask & 0xFFFFFFFF)
    rnd = lambda r: ROUND[r] if isinstance(r, str) else int(r)
    if shard is None:
        rc = lib().mx_quantize_dual(x.data_ptr(), DTYPE[x.dtype], rows, cols, x.stride(0), f,
                                    rnd(rnd_rows), seed_rows & (2**64 - 1), rnd(rnd_cols), seed_cols & (2**64 - 1),
                                    ctypes.byref(pre), cr.data_ptr(), sr_.data_ptr(), cc.data_ptr(), sc.data_ptr(),
                                    sl, _stream(stream))
        _check(rc, "mx_quantize_dual")
    else:
        sh = _Shard(*shard)
        rc = lib().mx_quantize_dual_shard(x.data_ptr(), DTYPE[x.dtype], rows, cols, x.stride(0), f,
                                          rnd(rnd_rows), seed_rows & (2**64 - 1), rnd(rnd_cols),
                                          seed_cols & (2**64 - 1), ctypes.byref(pre), ctypes.byref(sh),
                                          cr.data_ptr(), sr_.data_ptr(), cc.data_ptr(), sc.data_ptr(),
                                          sl, _stream(stream))
        _check(rc, "mx_quantize_dual_shard")
    return cr, sr_, cc, sc


def quantize_nvfp4(x: torch.Tensor, domain_rows: int = 0, scale_layout="mma", out=None, stream=None):
    """NVFP4 cast of a 2-D CUDA tensor along its rows (mx_quantize_nvfp4):
    domain_rows 0 for one global scale domain, else rows per CTA-local domain.
    Returns (codes, scales, enc_scales)."""
    if x.dim() != 2 or x.stride(1) != 1:
        raise ValueError("x must be 2-D with unit column stride")
    if x.dtype not in DTYPE:
        raise TypeError("x must be float32 or bfloat16")
    rows, cols = x.shape
    sl = _layout(scale_layout)
    if out is None:
        u8 = dict(dtype=torch.uint8, device=x.device)
        out = (torch.empty((rows, cols // 2), **u8),
               torch.empty(max(lib().mx_nvfp4_scales_bytes(sl, rows, cols), 1), **u8),
               torch.empty(max(lib().mx_nvfp4_domains(rows, domain_rows), 1), dtype=torch.float32,
                           device=x.device))
    codes, scales, enc = out
    rc = lib().mx_quantize_nvfp4(x.data_ptr(), DTYPE[x.dtype], rows, cols, x.stride(0), domain_rows,
                                 codes.data_ptr(), scales.data_ptr(), sl, enc.data_ptr(), _stream(stream))
    _check(rc, "mx_quantize_nvfp4")
    return codes, scales, enc


def dequantize(codes: torch.Tensor, scales: torch.Tensor, fmt, outer: int, inner: int,
               scale_layout="mma", out_dtype=torch.float32, out: torch.Tensor | None = None,
               stream=None) -> torch.Tensor:
    """Exact decode X * P, rounded once to out_dtype; returns (outer, inner)."""
    if out is None:
        out = torch.empty((outer, inner), dtype=out_dtype, device=codes.device)
    rc = lib().mx_dequantize(codes.data_ptr(), scales.data_ptr(), _fmt(fmt), _layout(scale_layout),
                             outer, inner, out.data_ptr(), DTYPE[out.dtype], out.stride(0),
                             _stream(stream))
    _check(rc, "mx_dequantize")
    return out


def gemm(a_codes: torch.Tensor, a_scales: torch.Tensor, b_codes: torch.Tensor,
         b_scales: torch.Tensor, M: int, N: int, K: int, fa="e4m3", fb=None, alpha: float = 1.0,
         out_dtype=torch.bfloat16, out: torch.Tensor | None = None, stream=None,
         scale_layout="mma") -> torch.Tensor:
    """C = alpha * A * B^T on MX operands quantized along K; scale_layout is the
    operands' scale layout, "mma" (mx_gemm) or "mma_x4" (mx_gemm_x4)."""
    fb = fa if fb is None else fb
    if out is None:
        out = torch.empty((M, N), dtype=out_dtype, device=a_codes.device)
    args = (a_codes.data_ptr(), a_scales.data_ptr(), _fmt(fa), b_codes.data_ptr(), b_scales.data_ptr(), _fmt(fb),
            M, N, K, float(alpha), out.data_ptr(), DTYPE[out.dtype], out.stride(0))
    if _layout(scale_layout) == LAYOUT["mma_x4"]:
        rc = lib().mx_gemm_x4(*args, _stream(stream))
        _check(rc, "mx_gemm_x4")
    elif _layout(scale_layout) == LAYOUT["mma"]:
        rc = lib().mx_gemm(*args, None, 0, _stream(stream))
        _check(rc, "mx_gemm")
    else:
        raise ValueError("GEMM operand scales are in the mma or mma_x4 layout")
    return out


def gemm_nvfp4(a, b, M: int, N: int, K: int, a_domain_rows: int = 0, b_domain_rows: int = 0,
               alpha: float = 1.0, out_dtype=torch.bfloat16, out: torch.Tensor | None = None,
               stream=None, scale_layout="mma") -> torch.Tensor:
    """C = alpha * A * B^T on NVFP4 operands (mx_gemm_nvfp4, or mx_gemm_nvfp4_x4
    for scale_layout "mma_x4"): a and b are the (codes, scales, enc_scales)
    triples quantize_nvfp4 returns in that layout."""
    (ac, asc, ae), (bc, bsc, be) = a, b
    if out is None:
        out = torch.empty((M, N), dtype=out_dtype, device=ac.device)
    fn = {LAYOUT["mma"]: "mx_gemm_nvfp4", LAYOUT["mma_x4"]: "mx_gemm_nvfp4_x4"}.get(_layout(scale_layout))
    if fn is None:
        raise ValueError("NVFP4 GEMM operand scales are in the mma or mma_x4 layout")
    rc = getattr(lib(), fn)(ac.data_ptr(), asc.data_ptr(), ae.data_ptr(), a_domain_rows,
                            bc.data_ptr(), bsc.data_ptr(), be.data_ptr(), b_domain_rows, M, N, K,
                            float(alpha), out.data_ptr(), DTYPE[out.dtype], out.stride(0), _stream(stream))
    _check(rc, fn)
    return out


def gemm_quantize(a_codes: torch.Tensor, a_scales: torch.Tensor, b_codes: torch.Tensor,
                  b_scales: torch.Tensor, M: int, N: int, K: int, fa="e4m3", fb=None, alpha: float = 1.0,
                  out_fmt="e4m3", rnd="rne", seed: int = 0, scale_layout="mma", out=None, stream=None,
                  operand_layout="mma"):
    """alpha * A * B^T quantized along its rows in the GEMM epilogue.

    Returns (codes, scales): M x (N * bits / 8) codes and the scales of an
    M x N tensor in `scale_layout`; `out` may supply both buffers."""
    fb = fa if fb is None else fb
    of = _fmt(out_fmt)
    sl = _layout(scale_layout)
    if out is None:
        dev = a_codes.device
        out = (torch.empty((M, codes_row_bytes(of, N)), dtype=torch.uint8, device=dev),
               torch.empty(max(scales_bytes(sl, M, N), 1), dtype=torch.uint8, device=dev))
    codes, scales = out
    fn = {LAYOUT["mma"]: "mx_gemm_quantize", LAYOUT["mma_x4"]: "mx_gemm_quantize_x4"}.get(_layout(operand_layout))
    if fn is None:
        raise ValueError("GEMM operand scales are in the mma or mma_x4 layout")
    rc = getattr(lib(), fn)(a_codes.data_ptr(), a_scales.data_ptr(), _fmt(fa), b_codes.data_ptr(),
                            b_scales.data_ptr(), _fmt(fb), M, N, K, float(alpha), of,
                            ROUND[rnd] if isinstance(rnd, str) else int(rnd), seed & (2**64 - 1),
                            codes.data_ptr(), scales.data_ptr(), sl, _stream(stream))
    _check(rc, fn)
    return codes, scales


def last_device_status(stream=None) -> int:
    return lib().mx_last_device_status(_stream(stream))
