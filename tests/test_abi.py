"""The C ABI (include/mx.h) without a GPU: the library loads, exports every
declared entry point, sizes agree with the oracle, and host-side argument
validation returns the documented status codes before touching the device."""
import ctypes
import os
import re

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def mx():
    from microscaling_block_scaled_mx_b200 import build, mx as m
    build.build()
    return m


def declared_functions():
    names = set()
    for h in sorted(os.listdir(os.path.join(ROOT, "include"))):
        if h.endswith(".h"):
            txt = open(os.path.join(ROOT, "include", h)).read()
            names |= set(re.findall(r"MX_API\s+[\w\s\*]+?\b(mx_\w+)\s*\(", txt))
    return sorted(names)


def test_header_declares_the_boundary():
    names = declared_functions()
    for n in ["mx_quantize", "mx_dequantize", "mx_gemm", "mx_codes_bytes", "mx_scales_bytes",
              "mx_gemm_workspace_bytes", "mx_last_device_status", "mx_status_str", "mx_abi_version",
              "mx_debug_gemm_skip_stage"]:
        assert n in names


def test_library_exports_every_declared_symbol(mx):
    L = mx.lib()
    for name in declared_functions():
        assert hasattr(L, name), name
    assert L.mx_abi_version() == 1


def test_debug_library_exports_every_declared_symbol():
    # libmx_debug.so (MX_DEBUG bounds checks) is built beside libmx.so by the
    # package build; it must offer the same boundary
    import ctypes
    from microscaling_block_scaled_mx_b200 import build as B
    if not os.path.exists(B.DEBUG_LIB):
        pytest.skip("libmx_debug.so not built")
    L = ctypes.CDLL(B.DEBUG_LIB)
    for name in declared_functions():
        assert hasattr(L, name), name
    assert L.mx_abi_version() == 1


def test_status_strings(mx):
    for code, name in mx.STATUS_NAMES.items():
        assert mx.status_str(code).startswith(name)


@pytest.mark.parametrize("fmt", list(range(6)))
@pytest.mark.parametrize("outer,inner", [(0, 32), (7, 64), (128, 4096), (300, 96)])
def test_sizes_agree_with_oracle(mx, oracle, fmt, outer, inner):
    assert mx.codes_bytes(fmt, outer, inner) == oracle.codes_bytes(fmt, outer, inner)
    for sl in (0, 1):
        assert mx.scales_bytes(sl, outer, inner) == oracle.scales_bytes(sl, outer, inner)


def test_sizes_reject_bad_shapes(mx):
    assert mx.codes_bytes(0, 4, 33) == 0
    assert mx.codes_bytes(9, 4, 32) == 0
    assert mx.scales_bytes(3, 4, 32) == 0


def _q(mx, x=16, dt=1, rows=64, cols=64, ldx=64, axis=1, fmt=0, rnd=0, codes=16, scales=16,
       sl=1, pre=None):
    L = mx.lib()
    return L.mx_quantize(x, dt, rows, cols, ldx, axis, fmt, rnd, 0, pre, codes, scales, sl, None)


def test_quantize_validation(mx):
    assert _q(mx, x=None) == -1
    assert _q(mx, codes=None) == -1
    assert _q(mx, dt=7) == -1
    assert _q(mx, fmt=6) == -1
    assert _q(mx, rnd=2) == -1
    assert _q(mx, axis=2) == -1
    assert _q(mx, sl=3) == -1
    assert _q(mx, ldx=32) == -1                   # ldx < cols
    assert _q(mx, rows=-1) == -1
    assert _q(mx, cols=48, ldx=48) == -3          # along cols, 48 % 32
    assert _q(mx, rows=48, axis=0) == -3          # along rows, 48 % 32
    assert _q(mx, x=8) == -2                      # misaligned input
    assert _q(mx, ldx=68) == -2                   # 68 * 2 bytes is not a multiple of 16
    assert _q(mx, codes=24) == -2
    pre = mx._Precond(1, 0xFFFFFFFF)
    assert _q(mx, pre=ctypes.byref(pre), axis=1) == -4   # Hadamard only on the strided axis
    assert _q(mx, rnd=1, rows=(1 << 20) + 1, cols=1 << 14, ldx=1 << 14) == -5


def test_dequantize_validation(mx):
    L = mx.lib()
    assert L.mx_dequantize(None, 16, 0, 1, 4, 64, 16, 0, 64, None) == -1
    assert L.mx_dequantize(16, 16, 0, 1, 4, 48, 16, 0, 48, None) == -3
    assert L.mx_dequantize(16, 16, 0, 1, 4, 64, 8, 0, 64, None) == -2
    assert L.mx_dequantize(16, 16, 0, 1, 4, 32, 16, 1, 36, None) == -2


def _d(mx, rows=64, cols=64, x=16, ldx=64, xdt=1, fmt=0, rr=0, rc=0, cr=16, sr=16, cc=16, sc=16, sl=1):
    L = mx.lib()
    return L.mx_quantize_dual(x, xdt, rows, cols, ldx, fmt, rr, 0, rc, 0, None, cr, sr, cc, sc, sl, None)


def test_quantize_dual_validation(mx):
    assert _d(mx, fmt=9) == -1
    assert _d(mx, rr=2) == -1
    assert _d(mx, sl=3) == -1
    assert _d(mx, rows=-32) == -1
    assert _d(mx, rows=48) == -3                  # both axes are block axes
    assert _d(mx, cols=80, ldx=80) == -3
    assert _d(mx, rows=0) == 0                    # empty: no-op, pointers unused
    assert _d(mx, cols=0, x=None, cr=None) == 0
    assert _d(mx, cc=None) == -1
    assert _d(mx, ldx=32) == -1
    assert _d(mx, x=8) == -2
    assert _d(mx, ldx=68) == -2                   # 136-byte bf16 row pitch
    assert _d(mx, cr=24) == -2
    assert _d(mx, rows=2 ** 20, cols=2 ** 15, ldx=2 ** 15, rc=1) == -5   # 2^35 elements with SR


def _g(mx, fa=0, fb=0, M=128, N=128, K=256, c=16, cdt=1, ldc=128, a=16):
    L = mx.lib()
    return L.mx_gemm(a, 16, fa, 16, 16, fb, M, N, K, 1.0, c, cdt, ldc, None, 0, None)


def L_gemm_b_misaligned(mx, fa, fb):
    return mx.lib().mx_gemm(32, 16, fa, 48, 16, fb, 128, 128, 256, 1.0, 16, 1, 128, None, 0, None)


def test_gemm_validation(mx):
    assert _g(mx, a=None) == -1
    assert _g(mx, fa=8) == -1
    assert _g(mx, M=-1) == -1
    assert _g(mx, ldc=64) == -1
    assert _g(mx, K=48) == -3
    assert _g(mx, fa=5, fb=5) == -4               # no block-scaled INT8 MMA
    assert _g(mx, fa=0, fb=5) == -4               # INT8 in either operand
    assert _g(mx, K=160) == -4                    # K % 128
    assert _g(mx, fa=2, fb=3, K=160) == -4
    assert _g(mx, fa=4, fb=4, K=192) == -4
    # FP6 codes, and FP4 codes fed to kind::mxf8f6f4, need 32-byte aligned bases
    assert _g(mx, fa=2, fb=2, a=48) == -2
    assert _g(mx, fa=0, fb=1, a=48) != -2         # FP8 codes at 16 bytes are fine ...
    assert L_gemm_b_misaligned(mx, fa=0, fb=3) == -2   # ... FP6 B at 16 bytes is not
    assert _g(mx, fa=4, fb=4, K=384, a=48) == -2  # FP4 x FP4, K = 128 (mod 256)
    assert _g(mx, c=8) == -2
    assert _g(mx, ldc=129, cdt=1) == -2


def test_gemm_rejects_sizes_past_32_bit_indexing(mx):
    """M, N, K up to 2^31 - 1 and at most 2^31 - 1 tiles of 128 x 128: larger
    sizes are refused on the host (MX_ERR_UNSUPPORTED) instead of wrapping."""
    big = 2 ** 31
    assert _g(mx, M=big, ldc=128) == -4
    assert _g(mx, N=big, ldc=big) == -4
    assert _g(mx, K=big) == -4
    assert _g(mx, M=2 ** 30, N=2 ** 24, ldc=2 ** 24) == -4       # 2^23 x 2^17 tiles
    assert _gq(mx, M=big) == -4
    assert _gq(mx, K=big) == -4
    assert _gq(mx, M=2 ** 30, N=2 ** 24) == -4


def _gq(mx, M=128, N=128, K=256, fa=0, fb=0, of=0, rnd=0, codes=16, scales=16, sl=1, a=16):
    L = mx.lib()
    return L.mx_gemm_quantize(a, 16, fa, 16, 16, fb, M, N, K, 1.0, of, rnd, 0, codes, scales, sl, None)


def test_gemm_quantize_validation(mx):
    assert _gq(mx, of=6) == -1
    assert _gq(mx, rnd=5) == -1
    assert _gq(mx, sl=3) == -1
    assert _gq(mx, M=-1) == -1
    assert _gq(mx, N=48) == -3                    # C's blocks run along N
    assert _gq(mx, K=48) == -3
    assert _gq(mx, M=0) == 0                      # empty
    assert _gq(mx, codes=None) == -1
    assert _gq(mx, a=None) == -1
    assert _gq(mx, fa=5) == -4
    assert _gq(mx, K=160) == -4
    assert _gq(mx, codes=24) == -2
    assert _gq(mx, fa=2, fb=2, a=48) == -2
    assert _gq(mx, M=2 ** 20, N=2 ** 15, rnd=1) == -5


def test_binding_fails_loudly_without_library(monkeypatch, tmp_path):
    from microscaling_block_scaled_mx_b200 import mx as m
    monkeypatch.setattr(m, "LIB_PATH", str(tmp_path / "missing.so"))
    monkeypatch.setattr(m, "_lib", None)
    with pytest.raises(RuntimeError, match="libmx.so not found"):
        m.lib()


def test_shard_validation(mx):
    """Host-side checks of the sharded casts (nothing is launched)."""
    import ctypes as C
    L = mx.lib()
    pre = mx._Precond(0, 0)

    def q(axis, shard, rows=64, cols=64, rnd=1):
        sh = mx._Shard(*shard) if shard is not None else None
        return L.mx_quantize_shard(16, 1, rows, cols, cols, axis, 4, rnd, 0, C.byref(pre),
                                   C.byref(sh) if sh is not None else None, 16, 16, 1, None)

    def d(shard, rows=64, cols=64):
        sh = mx._Shard(*shard)
        return L.mx_quantize_dual_shard(16, 1, rows, cols, cols, 4, 1, 0, 1, 0, C.byref(pre), C.byref(sh),
                                        16, 16, 16, 16, 1, None)

    assert q(0, None) == -1                             # shard is required
    assert q(0, (16, 0, 128, 64)) == -3                 # block-axis offset off a block boundary
    assert q(1, (0, 16, 64, 128)) == -3
    assert q(0, (0, 0, 112, 64), rows=64) == -3         # whole length along the block axis % 32
    assert q(0, (96, 0, 128, 64)) == -1                 # piece past the end of the whole tensor
    assert q(1, (-1, 0, 128, 64)) == -1
    assert q(0, (0, 0, 2 ** 20, 2 ** 15)) == -5         # SR range counts the whole tensor
    assert q(0, (0, 0, 2 ** 20, 2 ** 15), rnd=0) != -5
    assert q(1, (0, 0, 64, 64), rows=0) == 0            # empty piece
    assert d((16, 0, 128, 64)) == -3                    # both axes are block axes in the dual cast
    assert d((0, 16, 64, 128)) == -3
    assert d((96, 0, 128, 64)) == -1


def test_nvfp4_validation(mx):
    """Host-side checks of mx_quantize_nvfp4 (nothing is launched)."""
    L = mx.lib()
    assert L.mx_quantize_nvfp4(16, 1, 64, 40, 64, 0, 16, 16, 1, 16, None) == -3     # cols % 16
    assert L.mx_quantize_nvfp4(16, 1, 64, 64, 64, -1, 16, 16, 1, 16, None) == -1    # domain_rows
    assert L.mx_quantize_nvfp4(16, 3, 64, 64, 64, 0, 16, 16, 1, 16, None) == -1     # dtype
    assert L.mx_quantize_nvfp4(24, 1, 64, 64, 64, 0, 16, 16, 1, 16, None) == -2     # x alignment
    assert L.mx_quantize_nvfp4(16, 1, 64, 64, 64, 0, 16, 16, 1, 18, None) == -2     # enc alignment
    assert L.mx_quantize_nvfp4(16, 1, 0, 64, 64, 0, None, None, 1, None, None) == 0  # empty
    assert L.mx_nvfp4_domains(100, 32) == 4 and L.mx_nvfp4_domains(100, 0) == 1
    assert L.mx_nvfp4_scales_bytes(0, 100, 64) == 400
    assert L.mx_nvfp4_scales_bytes(1, 100, 64) == 128 * 4


def test_nvfp4_gemm_validation(mx):
    """Host-side checks of mx_gemm_nvfp4 (nothing is launched)."""
    L = mx.lib()

    def call(M=256, N=256, K=512, a_dom=0, b_dom=0, cdt=1, ldc=256, c=16, a_codes=16, a_enc=16, b_enc=16):
        return L.mx_gemm_nvfp4(a_codes, 16, a_enc, a_dom, 16, 16, b_enc, b_dom, M, N, K, 1.0, c, cdt, ldc, None)

    assert call(K=520) == -3                    # K % 16
    assert call(K=384) == -4                    # K % 256
    assert call(b_dom=48) == -4                 # E_B per 32 columns
    assert call(a_dom=-1) == -1 and call(M=-1) == -1
    assert call(cdt=2) == -1                    # output dtype
    assert call(ldc=100) == -1                  # ldc < N
    assert call(c=24) == -2 and call(a_codes=8) == -2 and call(a_enc=18) == -2 and call(b_enc=2) == -2
    assert call(M=1 << 31) == -4                # past 32-bit indexing
    assert L.mx_gemm_nvfp4(None, None, None, 0, None, None, None, 0, 0, 256, 512, 1.0, None, 1, 256,
                           None) == 0          # empty


def test_x4_layout_sizes_and_entries(mx):
    """The x4 scale layout's sizes and an unknown layout code's refusal; the
    x4 GEMM entries validate like mx_gemm."""
    L = mx.lib()
    assert L.mx_scales_bytes(2, 129, 32 * 5) == 4 * L.mx_scales_bytes(1, 129, 32 * 5)
    assert L.mx_scales_bytes(3, 128, 128) == 0
    assert L.mx_quantize_nvfp4(16, 1, 64, 64, 64, 0, 16, 16, 3, 16, None) == -1     # layout code
    # empty casts and GEMMs are no-ops for the x4 layout as for the others
    assert L.mx_quantize(None, 1, 0, 64, 64, 1, 0, 0, 0, None, None, None, 2, None) == 0
    assert L.mx_gemm_x4(None, None, 0, None, None, 0, 0, 64, 128, 1.0, None, 0, 64, None) == 0
    # argument checks before any launch
    assert L.mx_gemm_x4(16, 16, 0, 16, 16, 0, 128, 128, 100, 1.0, 16, 0, 128, None) == -3     # K % 32
    assert L.mx_gemm_x4(16, 16, 5, 16, 16, 0, 128, 128, 128, 1.0, 16, 0, 128, None) == -4     # INT8
    assert L.mx_gemm_x4(16, 16, 0, 16, 16, 0, 128, 128, 128, 1.0, 24, 0, 128, None) == -2     # C alignment
    assert L.mx_gemm_quantize_x4(16, 16, 0, 16, 16, 0, 128, 100, 128, 1.0, 0, 0, 0, 16, 16, 2, None) == -3
    assert L.mx_gemm_nvfp4_x4(16, 16, 16, 0, 16, 16, 16, 0, 256, 256, 384, 1.0, 16, 1, 256, None) == -4   # K % 256
    assert L.mx_nvfp4_scales_bytes(2, 100, 64) == 4 * L.mx_nvfp4_scales_bytes(1, 100, 64)
