import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)
HERE = os.path.dirname(os.path.abspath(__file__))
if HERE not in sys.path:
    sys.path.insert(0, HERE)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a B200 (sm_100a) and the built CUDA library")
    config.addinivalue_line("markers", "slow: long CPU-only sweeps (deselected unless asked for)")


@pytest.fixture(scope="session")
def oracle():
    import oracle as O
    O.build()
    return O


@pytest.fixture(scope="session")
def wgrad_oracle_operands(oracle):
    """The weight-gradient operands (dY 16384 x 4096, X 16384 x 14336, bf16,
    Student-t) and the oracle's casts of both along tokens: fixed-sign
    Hadamard with the default mask, stochastic rounding (seeds 42 and 43),
    E2M1, tensor-core scale layout.  Computed once per session and shared by
    the cast and GEMM parity tests."""
    from microscaling_block_scaled_mx_b200 import inputs as I
    mask = 0x6A09E667
    dy, xx = I.wgrad_operands()
    out = {"dy": dy, "xx": xx, "mask": mask}
    for name, t, seed in (("dy", dy, 42), ("xx", xx, 43)):
        out[name + "_q"] = oracle.quantize(t, 0, oracle.E2M1, rnd=oracle.SR, seed=seed, hadamard=True,
                                           sign_mask=mask, scale_layout=oracle.MMA)
    return out
