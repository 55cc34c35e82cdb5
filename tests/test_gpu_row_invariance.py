"""Row invariance of the automatic path (TandemLLM docs, "17 Qwen3.8-Flash-Next", §17.3: a
load-time check compares decode rows with the rows of 2..32-row verify chains bit for bit).

Up to 32 rows, a token's output bits, expert indices and gates do not depend on the other
tokens of the call: a token called alone (the single-kernel 1-token layer) equals its row in
2-, 5-, 16- and 32-row calls (the GEMV kernels), in whatever position. Checked on a small
layer and on the decode/verify layer of the workloads (d 2560, E 512, k 10, f 1024, int4),
which also meets the oracle on the 32-row call."""
import numpy as np
import pytest

from expert_routed_ffn_route_b200 import synth
from conftest import out_tol, output_excess
from gpu_helpers import bf16_to_np, oracle_run, to_dev_x

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def B():
    from expert_routed_ffn_route_b200 import binding
    if not torch.cuda.is_available():
        pytest.skip("no GPU")
    binding.load_library()
    return binding


CONFIGS = {
    "small": synth.LayerConfig("ri-small", T=32, d=512, E=64, k=4, f=256, fmt="int4", seed=29),
    "decode": synth.LayerConfig("ri-decode", T=32, d=2560, E=512, k=10, f=1024, fmt="int4"),
}


@pytest.mark.parametrize("name", ["small", "decode"])
def test_auto_path_row_invariance(B, name):
    cfg = CONFIGS[name]
    L = synth.make_layer(cfg)
    dl = B.DeviceLayer(L)
    x = to_dev_x(L.x)
    k = cfg.k

    def run(xx):
        T = xx.shape[0]
        desc = dl.descriptor(T, "auto")
        ws = B.alloc_workspace(desc)
        idx = torch.empty((T, k), dtype=torch.int32, device="cuda")
        w = torch.empty((T, k), dtype=torch.float32, device="cuda")
        out = B.layer_forward(desc, xx.contiguous(), ws, topk_idx=idx, topk_w=w)
        torch.cuda.synchronize()
        assert B.device_status(desc, ws) == 0
        return out.view(torch.int16), idx, w, B.launches_per_call(desc)

    o32, i32, w32, _ = run(x)
    for t in range(cfg.T):  # every token alone: the single-kernel layer
        o1, i1, w1, n1 = run(x[t:t + 1])
        assert n1 == 1, "the 1-token call is expected on the single-kernel layer"
        assert torch.equal(i1[0], i32[t]) and torch.equal(w1[0], w32[t]), t
        assert torch.equal(o1[0], o32[t]), t
    for T in (2, 5, 16):
        o, i, w, _ = run(x[:T])
        assert torch.equal(o, o32[:T]) and torch.equal(i, i32[:T]) and torch.equal(w, w32[:T]), T
    perm = torch.randperm(cfg.T, generator=torch.Generator().manual_seed(3)).cuda()
    o, _, _, _ = run(x[perm])
    assert torch.equal(o, o32[perm])
    o16, _, _, _ = run(x[16:])  # the second half on its own
    assert torch.equal(o16, o32[16:])

    # and the 32-row call meets the oracle
    ref = oracle_run(L)
    got = synth.bf16_bits_to_f32(bf16_to_np(o32.view(torch.bfloat16))).astype(np.float64)
    assert np.array_equal(i32.cpu().numpy(), ref["idx"])
    assert float(output_excess(got, ref["out"]).max()) <= out_tol(ref["out"])
