"""GPU parity of the NVFP4 cast (mx_quantize_nvfp4): the global and the
CTA-local scale domains the abstract of "Format-Aware Fusion for Fast FP4
Pretraining" names, in the reading stated in include/mx.h (16-element E2M1
blocks, E4M3 block scales, one fp32 encode scale per domain).  Every step is
one IEEE fp32 operation, so codes, block scales and domain scales must equal
the oracle's byte for byte."""
import numpy as np
import pytest
import torch

import mx_independent as ind
from gpu_helpers import dev, first_mismatch, host, to_device
from microscaling_block_scaled_mx_b200 import inputs as I
from microscaling_block_scaled_mx_b200 import mx

pytestmark = pytest.mark.gpu


def special_input(rows, cols, seed, bf16):
    rng = np.random.default_rng(seed)
    x = (rng.standard_normal((rows, cols)) * np.exp2(rng.uniform(-6, 6, (rows, 1)))).astype(np.float32)
    flat = x.reshape(-1)
    flat[rng.choice(flat.size, flat.size // 50, replace=False)] = 0.0
    sub = rng.choice(flat.size, flat.size // 200, replace=False)
    flat[sub] = (rng.integers(1, 1 << 23, sub.size).astype(np.uint32)
                 | (rng.integers(0, 2, sub.size).astype(np.uint32) << 31)).view(np.float32)
    x[3, 17 % cols] = np.nan
    x[5, 40 % cols] = np.inf
    x[7, :] = 0.0
    return ind.f32_to_bf16_bits_rne(x) if bf16 else x


def check(x_np, domain_rows, sl, what):
    rows, cols = x_np.shape
    codes, scales, enc = mx.quantize_nvfp4(to_device(x_np), domain_rows, scale_layout=sl)
    torch.cuda.synchronize()
    assert mx.last_device_status() == 0
    import oracle
    oc, os_, oe = oracle.nvfp4_quantize(x_np, domain_rows, scale_layout=oracle.MMA if sl == "mma" else oracle.PLAIN)
    assert np.array_equal(host(enc).view(np.uint32)[:oe.size], oe.view(np.uint32)), (what, host(enc)[:8], oe[:8])
    assert np.array_equal(host(codes), oc), (what, first_mismatch(host(codes), oc))
    if sl == "mma":            # padding bytes of the atom layout are never written
        keep = oc.shape[0]
        perm = ind.mma_scale_permutation(keep, cols // 16).reshape(-1)
        assert np.array_equal(host(scales)[perm], os_[perm]), what
    else:
        assert np.array_equal(host(scales), os_), (what, first_mismatch(host(scales), os_))


@pytest.mark.parametrize("bf16", [True, False])
@pytest.mark.parametrize("domain_rows", [0, 32, 7])
@pytest.mark.parametrize("sl", ["plain", "mma"])
def test_nvfp4_cast_parity(oracle, bf16, domain_rows, sl):
    for i, (rows, cols) in enumerate([(100, 256), (256, 4096), (33, 16)]):
        check(special_input(rows, cols, 50 + i, bf16), domain_rows, sl, (bf16, domain_rows, sl, rows, cols))


@pytest.mark.parametrize("domain_rows", [0, 32])
def test_nvfp4_cast_llama_activation(oracle, domain_rows):
    """A Llama-3-8B activation, 8192 x 4096 bf16 N(0,1)."""
    x, _ = I.linear_operands(8192, 4096, 128, 3, stream=0)
    check(x, domain_rows, "mma", ("llama", domain_rows))
