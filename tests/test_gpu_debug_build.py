"""The debug build (libmx_debug.so, compiled with MX_DEBUG): its kernels check
every code and scale store (and the decode's loads) against the buffer sizes.
On valid calls it gives the release build's bytes and reports MX_OK; when the
size the kernels are told is cut short (mx_debug_cast_cut_codes_cap, so that
no access outside a real buffer happens), the blocks past it are skipped and
mx_last_device_status reports MX_ERR_BOUNDS."""
import os
import subprocess
import sys
import textwrap

import numpy as np
import pytest
import torch

from gpu_helpers import dev, host, to_device
from microscaling_block_scaled_mx_b200 import build as B
from microscaling_block_scaled_mx_b200 import inputs as I
from microscaling_block_scaled_mx_b200 import mx

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

# The same calls in both processes: casts along rows and columns (x4 scales),
# a dual cast, an NVFP4 cast, a decode and a quantizing GEMM.
CALLS = textwrap.dedent("""
    import numpy as np, torch
    from microscaling_block_scaled_mx_b200 import inputs as I
    def run(mx, dev):
        # every output starts as 0xAB, so the padding bytes of the scale
        # layouts compare equal too
        u8 = lambda n: torch.full((max(n, 1),), 0xAB, dtype=torch.uint8, device=dev)
        rng = np.random.default_rng(77)
        x = torch.from_numpy(I.to_bf16_bits(rng.standard_normal((384, 416)).astype(np.float32)).view(np.int16)
                             ).view(torch.bfloat16).to(dev)
        R, C = x.shape
        L = mx.lib()
        out = {}
        out["rows"] = (u8(R * C), u8(mx.scales_bytes("mma", R, C)))
        mx.quantize(x, 1, "e4m3", codes=out["rows"][0].view(R, C), scales=out["rows"][1])
        out["cols_x4"] = (u8(C * R // 2), u8(mx.scales_bytes("mma_x4", C, R)))
        mx.quantize(x, 0, "e2m1", rnd="sr", seed=5, hadamard=True, scale_layout="mma_x4",
                    codes=out["cols_x4"][0].view(C, R // 2), scales=out["cols_x4"][1])
        out["dual"] = (u8(R * C // 2).view(R, C // 2), u8(mx.scales_bytes("mma", R, C)),
                       u8(C * R // 2).view(C, R // 2), u8(mx.scales_bytes("mma", C, R)))
        mx.quantize_dual(x, "e2m1", rnd_cols="sr", seed_cols=6, hadamard=True, out=out["dual"])
        out["nvfp4"] = (u8(R * C // 2).view(R, C // 2), u8(L.mx_nvfp4_scales_bytes(1, R, C)),
                        torch.zeros(L.mx_nvfp4_domains(R, 128), dtype=torch.float32, device=dev))
        mx.quantize_nvfp4(x, 128, out=out["nvfp4"])
        c, s = out["rows"]
        out["decode"] = (mx.dequantize(c.view(R, C), s, "e4m3", R, C),)
        a = mx.quantize(x[:256, :384].contiguous(), 1, "e4m3")
        b = mx.quantize(x[128:384, :384].contiguous(), 1, "e4m3")
        out["gemm_q"] = mx.gemm_quantize(a[0], a[1], b[0], b[1], 256, 256, 384, fa="e4m3", out_fmt="e2m1")
        torch.cuda.synchronize()
        status = mx.last_device_status()
        return {k: [t.cpu().numpy().copy() for t in v] for k, v in out.items()}, status
""")

CHILD = textwrap.dedent("""
    import sys, pickle, torch
    sys.path.insert(0, {root!r})
    from microscaling_block_scaled_mx_b200 import mx
    mx.LIB_PATH = {lib!r}
    ns = {{}}
    exec({calls!r}, ns)
    out, status = ns["run"](mx, torch.device("cuda:0"))
    # the cut hook: the next cast's codes buffer reads as 32 bytes short
    x = torch.randn(64, 256, device="cuda:0").to(torch.bfloat16)
    codes = torch.full((64, 256), 0xAB, dtype=torch.uint8, device="cuda:0")
    scales = torch.full((mx.scales_bytes("mma", 64, 256),), 0xAB, dtype=torch.uint8, device="cuda:0")
    assert mx.lib().mx_debug_cast_cut_codes_cap(32) == 0
    mx.quantize(x, 1, "e4m3", codes=codes, scales=scales)
    torch.cuda.synchronize()
    cut_status = mx.last_device_status()
    full = mx.quantize(x, 1, "e4m3")
    torch.cuda.synchronize()
    after_status = mx.last_device_status()
    pickle.dump((out, status, codes.cpu().numpy(), full[0].cpu().numpy(), cut_status, after_status),
                open({path!r}, "wb"))
""")


@pytest.fixture(scope="module")
def debug_lib():
    return B.build(debug=True)


def test_debug_build_matches_release_and_reports_bounds(debug_lib, tmp_path):
    path = str(tmp_path / "debug_out.pkl")
    child = CHILD.format(root=ROOT, lib=debug_lib, calls=CALLS, path=path)
    r = subprocess.run([sys.executable, "-c", child], capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-3000:]
    import pickle
    dbg, dbg_status, cut_codes, full_codes, cut_status, after_status = pickle.load(open(path, "rb"))
    ns = {}
    exec(CALLS, ns)
    rel, rel_status = ns["run"](mx, dev())
    assert rel_status == 0 and dbg_status == 0
    for k in rel:
        for i, (a, b) in enumerate(zip(rel[k], dbg[k])):
            assert np.array_equal(a, b), (k, i)
    # the last 32 code bytes (the last block of the last row) were not written
    assert cut_status == -8 and after_status == 0
    assert (cut_codes.reshape(-1)[-32:] == 0xAB).all()
    assert np.array_equal(cut_codes.reshape(-1)[:-32], full_codes.reshape(-1)[:-32])
