import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")


@pytest.fixture(scope="session")
def orc():
    import oracle
    oracle.build()
    return oracle


def row_rel_err(got, ref):
    """Max over rows (all leading indices) of ||got - ref||_inf / ||ref||_inf."""
    import numpy as np
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    num = np.abs(got - ref).max(axis=-1)
    den = np.abs(ref).max(axis=-1)
    den = np.where(den == 0, 1.0, den)
    return float((num / den).max()) if num.size else 0.0


def tol_for(dtype):
    """Parity bar: 1e-4 for fp32 inputs, 2e-2 for bf16/fp16 inputs (fp32 state)."""
    import torch
    return 1e-4 if dtype == torch.float32 else 2e-2


@pytest.fixture(scope="session")
def la():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import kernelized_causal_sequence_b200 as la_mod
    la_mod.lib()
    return la_mod
