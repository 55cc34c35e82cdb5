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
