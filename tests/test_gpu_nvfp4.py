"""Parity of the NVFP4 (W4A4) routed experts on the FP4 tensor cores against the NVFP4 oracle
(``oracle/nvfp4.py``), through the C ABI.

Bar:
  - the activation quantiser (``moe_nvfp4_quantize_rows``, the device function every NVFP4
    kernel uses) equals the oracle's ``nvfp4_quantize_rows`` exactly: E2M1 values, E4M3
    block-scale codes and fp32 row scales (integer decisions taken in fp32 on both sides);
  - the scale packing equals its layout definition byte for byte;
  - the layer: expert indices and the plan bit-exact, gates within 1e-5, the bf16 output
    within the layer bound 1e-2 * rms(oracle) + 1e-3 beyond the output's own bf16 rounding,
    and bitwise run-to-run determinism. h = silu(gate) * up is quantised to 4 bits per row; the
    kernel's fp32 sums and the oracle's exact ones can sit on opposite sides of a rounding
    boundary of that quantisation, which moves one h element by one E2M1 step (a few tenths
    of a percent of the output's rms after the down projection and the gate weight), inside
    the bound.
"""
import numpy as np
import pytest

from oracle import nvfp4 as N
from expert_routed_ffn_route_b200 import synth
from conftest import bank_dict, out_tol, output_excess
from gpu_helpers import GATE_TOL, bf16_to_np, plan_edge_tokens, to_dev_x

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def B():
    from expert_routed_ffn_route_b200 import binding
    if not torch.cuda.is_available():
        pytest.skip("no GPU")
    binding.load_library()
    return binding


def pack_reference(s, rows, K):
    """The packed scale layout written out: per matrix, 128-row tile and 64-K step a 512-byte
    block; row 128 t + 32 q + i, block 4 step + j at byte 16 i + 4 q + j."""
    n_mats = s.shape[0]
    out = np.zeros(n_mats * rows * (K // 16), np.uint8)
    KS = K // 64
    for m in range(n_mats):
        for r in range(rows):
            t, q, i = r // 128, (r % 128) // 32, r % 32
            for b in range(K // 16):
                step, j = b // 4, b % 4
                chunk = (m * (rows // 128) + t) * KS + step
                out[chunk * 512 + 16 * i + 4 * q + j] = s[m, r, b]
    return out


def test_pack_scales_layout(B):
    rng = np.random.default_rng(5)
    n_mats, rows, K = 2, 256, 192
    s = rng.integers(0, 256, (n_mats, rows, K // 16), dtype=np.uint8)
    got = B.nvfp4_pack_scales(torch.from_numpy(s).cuda(), n_mats, rows, K)
    torch.cuda.synchronize()
    assert np.array_equal(got.cpu().numpy().reshape(-1), pack_reference(s, rows, K))


def _quantiser_rows():
    rng = np.random.default_rng(11)
    rows = [rng.standard_normal(512) * 10 ** rng.uniform(-6, 3) for _ in range(48)]
    rows.append(np.zeros(512))                                   # zero row
    r = rng.standard_normal(512)
    r[:16] = 0.0                                                 # a zero block
    rows.append(r)
    r = np.zeros(512)
    r[7] = -3.5                                                  # one non-zero element
    rows.append(r)
    # exact E2M1 ties inside blocks: values on half-steps of a scale that is a power of two
    ties = np.array([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0, 6.0] * 2)
    rows.append(np.tile(np.concatenate([ties, -ties]), 16))
    return np.stack(rows).astype(np.float32)


def test_quantiser_matches_oracle(B):
    v = _quantiser_rows()
    codes, scales, g = B.nvfp4_quantize_rows(torch.from_numpy(v).cuda())
    torch.cuda.synchronize()
    c_ref, s_ref, g_ref = N.nvfp4_quantize_rows(v)
    assert np.array_equal(g.cpu().numpy(), g_ref.astype(np.float32))
    assert np.array_equal(scales.cpu().numpy(), s_ref.astype(np.uint8))
    got_vals = N.e2m1_value(N.unpack_fp4(codes.cpu().numpy(), v.shape[1]))
    assert np.array_equal(got_vals, N.e2m1_value(c_ref))  # -0 and +0 compare equal


def _layer(cfg_kw, T=None):
    cfg = synth.LayerConfig(**cfg_kw)
    return synth.make_layer(cfg, T=T)


def check_nvfp4_layer(B, L, dl, x_bits, tokens=None):
    T = x_bits.shape[0]
    desc = dl.descriptor(T)
    ws = B.alloc_workspace(desc)
    x = to_dev_x(x_bits)
    k, E = L.cfg.k, L.cfg.E
    idx = torch.empty((T, k), dtype=torch.int32, device="cuda")
    w = torch.empty((T, k), dtype=torch.float32, device="cuda")
    offs = torch.empty(E + 1, dtype=torch.int32, device="cuda")
    perm = torch.empty(T * k, dtype=torch.int32, device="cuda")
    out = B.layer_forward(desc, x, ws, topk_idx=idx, topk_w=w, offsets=offs, perm=perm)
    out2 = B.layer_forward(desc, x, ws)
    torch.cuda.synchronize()
    assert B.device_status(desc, ws) == 0
    assert torch.equal(out.view(torch.int16), out2.view(torch.int16)), "not deterministic"
    tokens = np.arange(T) if tokens is None else np.asarray(tokens)
    ref = N.layer_forward_nvfp4(x_bits, L.router_w, L.router_bias, bank_dict(L.routed),
                                bank_dict(L.shared), k, tokens=tokens)
    assert np.array_equal(idx.cpu().numpy(), ref["idx"])
    np.testing.assert_allclose(w.cpu().numpy(), ref["gates"], rtol=0, atol=GATE_TOL)
    assert np.array_equal(offs.cpu().numpy(), ref["offsets"])
    assert np.array_equal(perm.cpu().numpy(), ref["perm"])
    got = synth.bf16_bits_to_f32(bf16_to_np(out)).astype(np.float64)[tokens]
    err = output_excess(got, ref["out"])
    raw = float(np.abs(got - ref["out"]).max())
    rms = float(np.sqrt(np.mean(ref["out"] ** 2)))
    print(f"[nvfp4 T={T} d={L.cfg.d} E={E}] rows {len(tokens)}: max|d| {raw:.3e} "
          f"(rms {rms:.3e}), beyond bf16 rounding {float(err.max()):.3e}, "
          f"bound {out_tol(ref['out']):.3e}")
    assert float(err.max()) <= out_tol(ref["out"])
    # the four stage entry points give the layer call's result bit for bit
    i2, w2 = B.route(desc, x, ws)
    o2, p2, inv2 = B.permute(desc, i2, ws)
    ya, ys = B.grouped_ffn(desc, x, o2, p2, ws, has_shared=dl.has_shared)
    out3 = B.combine(desc, ya, ys, inv2, w2)
    torch.cuda.synchronize()
    assert torch.equal(i2, idx) and torch.equal(w2, w)
    assert torch.equal(out3.view(torch.int16), out.view(torch.int16))
    return ref


SMALL = dict(name="nvfp4-small", T=40, d=512, E=16, k=4, f=256, fmt="nvfp4",
             shared_fmt="bf16", seed=7)


@pytest.fixture(scope="module")
def small(B):
    L = _layer(SMALL)
    return L, B.DeviceLayer(L)


@pytest.mark.parametrize("T", [1, 5, 40, 130])
def test_small_layer(B, small, T):
    L, dl = small
    x = L.x if T == L.cfg.T else synth.make_hidden(L.cfg, L.router_w, L.router_bias, T=T,
                                                   stream=f"nv{T}")
    check_nvfp4_layer(B, L, dl, x)


def test_small_layer_no_shared(B):
    L = _layer(dict(SMALL, name="nvfp4-noshared", n_shared=0, T=70, seed=8))
    check_nvfp4_layer(B, L, B.DeviceLayer(L), L.x)


def test_rows_independent_of_the_call(B, small):
    # a row's result depends on that row alone: the first rows of a 130-token call equal a
    # 40-token call of the same rows bit for bit (both above 32 rows, where the same routing
    # kernels run)
    L, dl = small
    x = synth.make_hidden(L.cfg, L.router_w, L.router_bias, T=130, stream="nv130")
    outs = []
    for T in (40, 130):
        desc = dl.descriptor(T)
        ws = B.alloc_workspace(desc)
        outs.append(B.layer_forward(desc, to_dev_x(x[:T]), ws))
    torch.cuda.synchronize()
    assert torch.equal(outs[0].view(torch.int16), outs[1][:40].view(torch.int16))


@pytest.mark.parametrize("T,n_rows", [(512, 32), (4096, 24)])
def test_full_size(B, T, n_rows):
    cfg = dict(name=f"nvfp4-{T}", T=T, d=2560, E=512, k=10, f=1024, fmt="nvfp4",
               shared_fmt="bf16", zipf_s=1.1 if T == 4096 else None)
    L = _layer(cfg)
    dl = B.DeviceLayer(L)
    check_nvfp4_layer(B, L, dl, L.x, tokens=plan_edge_tokens(L, n_hot=3, n_total=n_rows))
