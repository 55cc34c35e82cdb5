"""Failure detection on the GPU without a GPU fault: a bounded device wait is made to run
out and its status is read back on the host.

The workspace's hold word is set through moe_test_inject_hold with a budget of a few
thousand clock cycles. The kernels that check it (the single-kernel 1-token layer at its
first grid barrier, the fused routing kernel after its ticket barrier) then wait for a word
that nothing clears during the call; the wait gives up after the budget, the kernel records
MOE_ERR_TIMEOUT, drains its copies and returns. The host reads the code with
moe_device_status; the same workspace, once the word is cleared, and a fresh one then give
results that match the oracle. Nothing traps, faults or waits without a bound.
"""
import numpy as np
import pytest

from oracle import moe_oracle as O
from expert_routed_ffn_route_b200 import synth
from conftest import out_tol, output_excess
from gpu_helpers import bf16_to_np, oracle_run, to_dev_x

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

MOE_ERR_TIMEOUT = -4
BUDGET_CYCLES = 20000  # about 10 microseconds


@pytest.fixture(scope="module")
def B():
    from expert_routed_ffn_route_b200 import binding
    if not torch.cuda.is_available():
        pytest.skip("no GPU")
    binding.load_library()
    return binding


# the wait sites the hold reaches (moe_device_wait_site): the single-kernel layer's first
# grid barrier, the fused routing kernel's test hold
@pytest.mark.parametrize("T,path,launches,site", [(1, "fused", 1, 22), (5, "gemv", None, 2)])
def test_bounded_wait_runs_out_and_is_reported(B, T, path, launches, site):
    cfg = synth.LayerConfig("hold", T=T, d=2048, E=64, k=8, f=1024, fmt="int4", seed=43)
    L = synth.make_layer(cfg)
    dl = B.DeviceLayer(L)
    desc = dl.descriptor(T, path)
    if launches is not None:
        assert B.launches_per_call(desc) == launches
    x = to_dev_x(L.x)
    ref = oracle_run(L)

    def matches_oracle(out):
        got = O.widen_bf16(bf16_to_np(out))
        return float(output_excess(got, ref["out"]).max()) <= out_tol(ref["out"])

    ws = B.alloc_workspace(desc)
    B.test_inject_hold(desc, ws, True, BUDGET_CYCLES)
    B.layer_forward(desc, x, ws)
    torch.cuda.synchronize()
    assert B.device_status(desc, ws) == MOE_ERR_TIMEOUT
    assert B.device_status(desc, ws) == 0  # read and cleared
    assert B.device_wait_site(desc, ws) == site
    assert B.device_wait_site(desc, ws) == 0

    # the same workspace, hold cleared: its barrier words and counters are consistent
    B.test_inject_hold(desc, ws, False)
    for _ in range(2):
        out = B.layer_forward(desc, x, ws)
        torch.cuda.synchronize()
        assert B.device_status(desc, ws) == 0
        assert B.device_wait_site(desc, ws) == 0
        assert matches_oracle(out)

    # a fresh workspace
    ws2 = B.alloc_workspace(desc)
    out = B.layer_forward(desc, x, ws2)
    torch.cuda.synchronize()
    assert B.device_status(desc, ws2) == 0
    assert matches_oracle(out)
