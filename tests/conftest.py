import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA GPU (B200, sm_100a)")
    config.addinivalue_line("markers", "slow: long-running CPU test")


def bank_dict(bank):
    """synth.Bank -> the plain dict layout the oracle reads."""
    if bank is None:
        return None
    d = bank.arrays()
    d["fmt"] = bank.fmt
    d["group"] = bank.group
    return d


@pytest.fixture(scope="session")
def tiny_layer():
    from expert_routed_ffn_route_b200 import synth
    return synth.make_layer("tiny")


def bf16_half_ulp(v):
    """Half a unit in the last place of bf16 at |v| (8 significant bits)."""
    import numpy as np
    a = np.maximum(np.abs(v), np.finfo(np.float32).tiny)
    return np.ldexp(1.0, np.floor(np.log2(a)).astype(np.int64) - 8)


def output_excess(got, ref):
    """Per-element error of a bf16 output beyond its own rounding: |got - ref| minus half a
    bf16 ulp at max(|got|, |ref|). The layer bound (1e-2 * rms(ref) + 1e-3) applies to this."""
    import numpy as np
    return np.abs(got - ref) - bf16_half_ulp(np.maximum(np.abs(got), np.abs(ref)))


def out_tol(ref):
    import numpy as np
    return 1e-2 * float(np.sqrt(np.mean(ref ** 2))) + 1e-3
