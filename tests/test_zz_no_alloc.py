"""The entry point for callers that cannot allocate device memory (the library's built-in
scratch). Kept in a file of its own that runs after every other test: it must agree with
the workspace entry point, on two calls in a row, alone or after the rest of the suite."""
import numpy as np
import pytest

from oracle import moe_oracle as O
from expert_routed_ffn_route_b200 import synth
from conftest import out_tol, output_excess

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("name,cfg", [
    ("tiny16", synth.LayerConfig("tiny16", T=16, d=256, E=16, k=2, f=128, fmt="bf16")),
    ("int4", synth.LayerConfig("ns-int4", T=8, d=512, E=32, k=4, f=256, fmt="int4", seed=21)),
    # one token: the single-kernel layer, whose grid-barrier word and per-tile arrival
    # counters live in the scratch and must be back at their start values for the second call
    ("fused1", synth.LayerConfig("ns-fused1", T=1, d=2048, E=64, k=8, f=1024, fmt="int4",
                                 seed=22)),
])
def test_static_scratch_matches_workspace_entry_point(name, cfg):
    from expert_routed_ffn_route_b200 import binding as B
    if not torch.cuda.is_available():
        pytest.skip("no GPU")
    L = synth.make_layer(cfg)
    dl = B.DeviceLayer(L)
    desc = dl.descriptor(cfg.T)
    if name == "fused1":
        assert B.launches_per_call(desc) == 1, "single-kernel layer not taken"
    x = torch.from_numpy(L.x.view(np.int16)).cuda().view(torch.bfloat16)
    ws = B.alloc_workspace(desc)
    ref = B.layer_forward(desc, x, ws)
    first = B.layer_forward_static(desc, x)
    second = B.layer_forward_static(desc, x)
    torch.cuda.synchronize()
    assert B.device_status(desc, ws) == 0
    assert B.static_device_status() == 0  # no device-side error in either static call
    r = O.widen_bf16(ref.view(torch.int16).cpu().numpy().view(np.uint16))
    for got in (first, second):
        g = O.widen_bf16(got.view(torch.int16).cpu().numpy().view(np.uint16))
        assert float(output_excess(g, r).max()) <= out_tol(r)
        assert np.array_equal(g, r)  # same kernels, same inputs: bit for bit


def test_static_scratch_rejects_oversized_request():
    from expert_routed_ffn_route_b200 import binding as B
    if not torch.cuda.is_available():
        pytest.skip("no GPU")
    cfg = synth.CONFIGS["prefill"]  # T = 512 needs far more than the built-in scratch
    fake = 1 << 20
    bank = lambda n: B.MoeBank(4, 128, n, 0, fake, fake, fake, fake, fake, fake)
    desc = B.MoeLayer(cfg.T, cfg.d, cfg.f, cfg.E, cfg.k, 0, fake, None, bank(cfg.E), bank(1))
    x = torch.empty((cfg.T, cfg.d), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(B.MoeError) as e:
        B.layer_forward_static(desc, x)
    assert e.value.status == -7
