"""Parity of the CUDA library (called through the C ABI) against the fp64 oracle.

Bar: expert indices, the plan (offsets, perm, inv) bit-exact; gates within 1e-5;
the bf16 layer output within max|d| <= 1e-2 * rms(oracle) + 1e-3 (the tolerance the
workload states for fp32 accumulation), counted beyond the output's own rounding to
bf16 (half a bf16 ulp of the element, which alone exceeds the bound for |out| >= 2);
bitwise run-to-run determinism.
"""
import numpy as np
import pytest

from oracle import moe_oracle as O
from expert_routed_ffn_route_b200 import synth
from conftest import out_tol, output_excess
from gpu_helpers import bf16_to_np, check_layer, oracle_run, plan_edge_tokens, to_dev_x

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def B():
    from expert_routed_ffn_route_b200 import binding
    if not torch.cuda.is_available():
        pytest.skip("no GPU")
    binding.load_library()
    return binding


# ------------------------------------------------------------------ small shapes

@pytest.fixture(scope="module")
def tiny(B):
    L = synth.make_layer("tiny")
    return L, B.DeviceLayer(L)


@pytest.mark.parametrize("path", ["gemv"])
def test_tiny_full(B, tiny, path):
    L, dl = tiny
    check_layer(B, dl, L, L.x, path)


@pytest.mark.parametrize("T", [1, 3, 33])
def test_tiny_ragged_T(B, tiny, T):
    L, dl = tiny
    x = synth.make_hidden(L.cfg, L.router_w, L.router_bias, T=T, stream=f"ragged{T}")
    check_layer(B, dl, L, x, "gemv")


@pytest.mark.parametrize("fmt", ["int4", "int8", "bf16"])
@pytest.mark.parametrize("shared", [1, 0])
def test_formats_small(B, fmt, shared):
    cfg = synth.LayerConfig(f"small-{fmt}", T=40, d=384, E=12, k=3, f=256, n_shared=shared,
                            fmt=fmt, seed=3)
    L = synth.make_layer(cfg)
    check_layer(B, B.DeviceLayer(L), L, L.x, "gemv")


def test_zipf_bias_and_k1(B):
    cfg = synth.LayerConfig("bias-k1", T=50, d=256, E=20, k=1, f=128, fmt="int8", zipf_s=1.1,
                            seed=5)
    L = synth.make_layer(cfg)
    check_layer(B, B.DeviceLayer(L), L, L.x, "gemv")


def test_all_experts_selected(B):
    cfg = synth.LayerConfig("k=E", T=17, d=256, E=4, k=4, f=128, fmt="int4", seed=7)
    L = synth.make_layer(cfg)
    check_layer(B, B.DeviceLayer(L), L, L.x, "gemv")


def test_many_rows_per_expert(B):
    """One expert gets most rows (more than one 8-token chunk, ragged tail)."""
    cfg = synth.LayerConfig("hot", T=100, d=256, E=8, k=2, f=128, fmt="int4", zipf_s=3.0, seed=9)
    L = synth.make_layer(cfg)
    check_layer(B, B.DeviceLayer(L), L, L.x, "gemv")


# ------------------------------------------------------------------ full-size workloads

@pytest.fixture(scope="module")
def int4_bank(B):
    cfg = synth.CONFIGS["decode"]
    routed = synth.make_bank(cfg, "routed")
    shared = synth.make_bank(cfg, "shared")
    return routed, shared


@pytest.mark.parametrize("name", ["decode", "verify16", "verify32", "prefill"])
def test_full_size_int4(B, int4_bank, name):
    """Full-size int4 workloads in the launch configuration the bench times (path auto).
    Every output row of the decode and verify calls is compared; at prefill, 128 rows:
    the edges of the units of the 8 most loaded experts and a seeded random draw."""
    cfg = synth.CONFIGS[name]
    routed, shared = int4_bank
    L = synth.make_layer(cfg, routed=routed, shared=shared)
    dl = B.DeviceLayer(L)
    sample = None
    if cfg.T > 32:
        sample = plan_edge_tokens(L, n_hot=8, n_total=128, seed=1)
        assert len(sample) == 128
    check_layer(B, dl, L, L.x, "auto", sample=sample, check_stages=(cfg.T <= 32))


@pytest.mark.parametrize("path,shared", [("gemv", True), ("fused", True), ("fused", False)])
def test_full_size_decode_paths(B, int4_bank, path, shared):
    """The decode workload through the multi-kernel GEMV path and the single-kernel path
    (with and without the shared expert), on several tokens."""
    cfg = synth.CONFIGS["decode"]
    routed, sh = int4_bank
    L = synth.make_layer(cfg, routed=routed, shared=sh)
    if not shared:
        L.shared = None
    dl = B.DeviceLayer(L)
    for i in range(3):
        x = L.x if i == 0 else synth.make_hidden(cfg, L.router_w, L.router_bias, stream=f"pool{i}")
        check_layer(B, dl, L, x, path, check_stages=(i == 0))


def test_full_size_long_int8(B):
    """The long Zipf-skewed int8 workload: 256 output rows, including the first row of each
    of the 5 most loaded experts and the first and last rows of their last (ragged)
    tensor-core unit, the rest a seeded random draw (every hot expert's units alternate
    between the two accumulator buffers of the gate/up GEMM)."""
    cfg = synth.CONFIGS["long"]
    L = synth.make_layer(cfg)
    dl = B.DeviceLayer(L)
    sample = plan_edge_tokens(L, n_hot=5, n_total=256, seed=2)
    assert len(sample) == 256
    check_layer(B, dl, L, L.x, "auto", sample=sample, check_stages=False)


# ------------------------------------------------------------------ errors

def test_errors_reported(B, tiny):
    L, dl = tiny
    desc = dl.descriptor(8)
    ws = B.alloc_workspace(desc)
    x = to_dev_x(L.x[:8])
    with pytest.raises(B.MoeError) as e:
        B.layer_forward(desc, x, ws[1:])          # misaligned and too small
    assert e.value.status == -5
    bad = dl.descriptor(8)
    bad.k = 0
    with pytest.raises(B.MoeError) as e:
        B.layer_forward(bad, x, ws)
    assert e.value.status == -1


# ------------------------------------------------------------------ tensor-core path

@pytest.mark.parametrize("fmt", ["int4", "int8", "bf16"])
@pytest.mark.parametrize("shared", [1, 0])
def test_tc_formats_small(B, fmt, shared):
    cfg = synth.LayerConfig(f"tc-{fmt}", T=96, d=384, E=12, k=3, f=256, n_shared=shared,
                            fmt=fmt, seed=11)
    L = synth.make_layer(cfg)
    check_layer(B, B.DeviceLayer(L), L, L.x, "tc")


@pytest.mark.parametrize("fmt", ["int4", "int8", "bf16"])
def test_tc_formats_many_rows_per_expert(B, fmt):
    """32+ rows per routed expert on average: the gate/up GEMM's two-accumulator layout."""
    cfg = synth.LayerConfig(f"tc-wide-{fmt}", T=160, d=384, E=6, k=2, f=256, n_shared=1,
                            fmt=fmt, seed=17)
    assert cfg.T * cfg.k >= 32 * cfg.E
    L = synth.make_layer(cfg)
    check_layer(B, B.DeviceLayer(L), L, L.x, "tc")


@pytest.mark.parametrize("routed,shared", [("int4", "int8"), ("int8", "int4"), ("int4", "bf16")])
@pytest.mark.parametrize("T,path", [(1, "auto"), (5, "gemv"), (96, "tc")])
def test_mixed_bank_formats(B, routed, shared, T, path):
    """The shared expert in another encoding than the routed experts: the grouped products
    run once per bank (the TMA GEMV takes int4/int8 pairs, one launch per bank; a bf16 bank
    takes the register-streaming GEMV; the single-kernel 1-token layer declines such
    layers)."""
    cfg = synth.LayerConfig(f"mixed-{routed}-{shared}", T=T, d=384, E=12, k=3, f=256,
                            n_shared=1, fmt=routed, shared_fmt=shared, seed=19)
    L = synth.make_layer(cfg)
    assert L.shared.fmt == shared and L.routed.fmt == routed
    check_layer(B, B.DeviceLayer(L), L, L.x, path)


@pytest.mark.parametrize("routed,shared", [("int4", "int4"), ("int8", "int8"), ("int4", "int8")])
def test_gemv_path_row_invariance(B, routed, shared):
    """On the GEMV path a token's output bits do not depend on the other tokens of the call
    (up to 32): the first T rows of a 32-token call equal a T-token call bit for bit, and
    permuting the tokens permutes the outputs bit for bit (int8 banks and W8 shared beside
    W4 routed on the TMA GEMV too)."""
    cfg = synth.LayerConfig("ri", T=32, d=512, E=64, k=4, f=256, n_shared=1, fmt=routed,
                            shared_fmt=shared, seed=23)
    L = synth.make_layer(cfg)
    dl = B.DeviceLayer(L)
    x = torch.from_numpy(L.x.view(np.int16)).cuda().view(torch.bfloat16)

    def run(xx):
        desc = dl.descriptor(xx.shape[0], "gemv")
        out = B.layer_forward(desc, xx.contiguous(), B.alloc_workspace(desc))
        torch.cuda.synchronize()
        return out.view(torch.int16)

    o32 = run(x)
    for T in (1, 2, 5, 16):
        assert torch.equal(run(x[:T]), o32[:T]), T
    perm = torch.randperm(32, generator=torch.Generator().manual_seed(1)).cuda()
    assert torch.equal(run(x[perm]), o32[perm])


@pytest.mark.parametrize("routed,shared,T", [("int8", "int8", 1), ("int8", "int8", 16),
                                             ("int4", "int8", 1), ("int4", "int8", 32)])
def test_w8_layers_full_size_gemv(B, routed, shared, T):
    """W8 edge layers (int8 routed and shared) and a W8 shared expert beside W4 routed
    experts, at the decode/verify layer size, on the automatic path (the TMA GEMV kernels up
    to 32 rows): every row against the oracle."""
    cfg = synth.LayerConfig(f"w8-{routed}-{shared}", T=T, d=2560, E=512, k=10, f=1024,
                            fmt=routed, shared_fmt=shared, seed=31)
    L = synth.make_layer(cfg)
    check_layer(B, B.DeviceLayer(L), L, L.x, "auto", check_stages=False)


def test_tc_tiny(B, tiny):
    L, dl = tiny
    check_layer(B, dl, L, L.x, "tc")


@pytest.mark.parametrize("T", [1, 33])
def test_tc_ragged_T(B, tiny, T):
    L, dl = tiny
    x = synth.make_hidden(L.cfg, L.router_w, L.router_bias, T=T, stream=f"tcragged{T}")
    check_layer(B, dl, L, x, "tc")


def test_tc_many_m_tiles(B):
    """One expert gets several 128-row m-tiles (skewed routing), ragged last tile."""
    cfg = synth.LayerConfig("tc-hot", T=700, d=256, E=8, k=2, f=256, fmt="int8", zipf_s=3.0,
                            seed=13)
    L = synth.make_layer(cfg)
    check_layer(B, B.DeviceLayer(L), L, L.x, "tc", sample=[0, 1, 350, 699])


# ------------------------------------------------------------------ single-kernel 1-token layer

def _fused_case(B, cfg):
    L = synth.make_layer(cfg)
    dl = B.DeviceLayer(L)
    assert B.launches_per_call(dl.descriptor(1, "fused")) == 1, "fused path not taken"
    return L, dl


@pytest.mark.parametrize("shared", [1, 0])
@pytest.mark.parametrize("shape", [(384, 256, 12, 3), (512, 256, 32, 4), (2048, 1024, 64, 8)])
def test_fused_t1_small(B, shape, shared):
    d, f, E, k = shape
    cfg = synth.LayerConfig(f"fused-{d}", T=1, d=d, E=E, k=k, f=f, n_shared=shared, fmt="int4",
                            seed=31)
    L, dl = _fused_case(B, cfg)
    check_layer(B, dl, L, L.x, "fused")


def test_fused_t1_many_calls_and_graph(B):
    """Ten calls in a row on different tokens (the barrier word and the tile counters carry
    over between calls), then the same calls replayed from a CUDA graph, bit for bit."""
    cfg = synth.LayerConfig("fused-seq", T=1, d=2048, E=64, k=8, f=1024, fmt="int4", seed=33)
    L, dl = _fused_case(B, cfg)
    desc = dl.descriptor(1, "fused")
    ws = B.alloc_workspace(desc)
    xs = [synth.make_hidden(cfg, L.router_w, L.router_bias, T=1, stream=f"seq{i}")
          for i in range(10)]
    xd = [to_dev_x(x) for x in xs]
    outs = [B.layer_forward(desc, x, ws) for x in xd]
    torch.cuda.synchronize()
    assert B.device_status(desc, ws) == 0
    for x, o in zip(xs, outs):
        ref = oracle_run(L, x=x)
        got = O.widen_bf16(bf16_to_np(o))
        assert float(output_excess(got, ref["out"]).max()) <= out_tol(ref["out"])
    st = torch.cuda.Stream()
    gout = [torch.empty_like(o) for o in outs]
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=st):
        for x, o in zip(xd, gout):
            B.layer_forward(desc, x, ws, out=o, stream=st)
    for _ in range(2):
        g.replay()
    torch.cuda.synchronize()
    assert B.device_status(desc, ws) == 0
    for a, b in zip(outs, gout):
        assert torch.equal(a.view(torch.int16), b.view(torch.int16))


def test_fused_unsupported_reported(B):
    cfg = synth.LayerConfig("fused-int8", T=1, d=256, E=8, k=2, f=128, fmt="int8", seed=35)
    L = synth.make_layer(cfg)
    dl = B.DeviceLayer(L)
    desc = dl.descriptor(1, "fused")
    ws = B.alloc_workspace(desc)
    with pytest.raises(B.MoeError) as e:
        B.layer_forward(desc, to_dev_x(L.x), ws)
    assert e.value.status == -2
