"""Pins of the fp64 oracle against facts that do not come from the oracle itself:
hand-derived closed forms, library routines with the same definition, exact
invariants of the layer, and brute force on tiny inputs. A planted-mistake
section checks that these pins fail when a plausible bug is put in the oracle."""
import json
import math
import os

import numpy as np
import pytest
import torch

from oracle import moe_oracle as O
from expert_routed_ffn_route_b200 import synth
from conftest import bank_dict

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _bits(a):
    return synth.bf16_bits(np.asarray(a, np.float32))


def _worked():
    with open(os.path.join(GOLDEN, "worked_layer.json")) as fh:
        g = json.load(fh)
    bank = lambda b: dict(fmt="bf16", group=128, s_gate=None, s_up=None, s_down=None,
                          w_gate=_bits(b["w_gate"]), w_up=_bits(b["w_up"]),
                          w_down=_bits(b["w_down"]))
    return g, _bits(g["x"]), _bits(g["router_w"]), bank(g["routed"]), bank(g["shared"])


def _closed(expr):
    s1 = 1.0 / (1.0 + math.exp(-1.0))
    s2 = 1.0 / (1.0 + math.exp(-2.0))
    return eval(expr, {"__builtins__": {}}, {"s1": s1, "s2": s2})


def _check_worked(forward=O.layer_forward):
    g, x, wr, routed, shared = _worked()
    r = forward(x, wr, None, routed, shared, g["k"])
    ex = g["expect"]
    assert r["idx"].tolist() == ex["idx"]
    np.testing.assert_allclose(r["gates"], [[_closed(v) for v in row] for row in ex["gates"]],
                               rtol=0, atol=1e-15)
    assert r["counts"].tolist() == ex["counts"]
    assert r["offsets"].tolist() == ex["offsets"]
    assert r["perm"].tolist() == ex["perm"]
    assert r["inv"].tolist() == ex["inv"]
    np.testing.assert_allclose(r["out"], [[_closed(v) for v in row] for row in ex["out"]],
                               rtol=0, atol=1e-14)


def test_worked_example_closed_form():
    _check_worked()


def test_worked_example_loops():
    g, x, wr, routed, shared = _worked()
    out = O.layer_forward_loops(x, wr, None, routed, shared, g["k"])
    np.testing.assert_allclose(out, [[_closed(v) for v in row] for row in g["expect"]["out"]],
                               rtol=0, atol=1e-14)


# ------------------------------------------------------------ encodings

def test_int4_unpack_golden():
    with open(os.path.join(GOLDEN, "int4_layout.json")) as fh:
        g = json.load(fh)
    words = np.array([int(h, 16) for h in g["words_hex"]], np.uint32)[:, None]
    vals = O.unpack_int4(words, 8)
    assert vals.tolist() == g["values"]
    for h, v in g["scale_bits_hex"].items():
        assert O.widen_bf16(np.array([int(h, 16)], np.uint16))[0] == v


def test_dequant_groups_golden():
    with open(os.path.join(GOLDEN, "int4_layout.json")) as fh:
        c = json.load(fh)["dequant_case"]
    K, G = c["K"], c["group"]
    # word pattern for nibbles (kk % 8) - 4 = -4..3 -> nibbles 0xC,0xD,0xE,0xF,0,1,2,3
    word = 0
    for i in range(8):
        word |= ((i - 4) & 0xF) << (4 * i)
    words = np.full((1, K // 8), word, np.uint32)
    s = np.array([[int(h, 16) for h in c["scale_bits_hex"]]], np.uint16)
    W = O.dequantize(words, s, "int4", G, K)
    kk = np.arange(K)
    expect = ((kk % 8) - 4) * np.where(kk < 128, 0.5, 2.0)
    assert np.array_equal(W[0], expect)
    # int8: the same values stored plainly
    W8 = O.dequantize(((kk % 8) - 4).astype(np.int8)[None, :], s, "int8", G, K)
    assert np.array_equal(W8[0], expect)


def test_bf16_widen_matches_torch():
    rng = np.random.default_rng(1)
    v = rng.standard_normal(1000).astype(np.float32) * 10
    bits = synth.bf16_bits(v)
    ref = torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).to(torch.float64).numpy()
    assert np.array_equal(O.widen_bf16(bits), ref)


def test_round_to_bf16_matches_torch_on_float32_values():
    rng = np.random.default_rng(2)
    v = (rng.standard_normal(5000) * 3).astype(np.float32)
    ref = torch.from_numpy(v).to(torch.bfloat16).to(torch.float64).numpy()
    assert np.array_equal(O.round_to_bf16_f64(v.astype(np.float64)), ref)


def test_quantiser_roundtrip_with_oracle_dequant():
    """Re-quantising the oracle's dequantised weights returns the same codes,
    and |w - q s| <= s/2 (rounding to nearest) unless clamped at qmax."""
    rng = np.random.default_rng(3)
    w = (rng.standard_normal((8, 256)) * 0.02).astype(np.float32)
    for fmt, qmax in (("int4", 7), ("int8", 127)):
        q, sb = synth.quantize_groups(w, qmax, 128)
        enc = synth.pack_int4(q) if fmt == "int4" else q
        W = O.dequantize(enc, sb, fmt, 128, 256)
        s = np.repeat(O.widen_bf16(sb), 128, axis=1)
        assert np.array_equal(np.rint(W / s), q.astype(np.float64))
        err = np.abs(w.astype(np.float64) - W)
        clamped = np.abs(q) == qmax
        assert np.all(err[~clamped] <= s[~clamped] / 2 * (1 + 1e-6))
        assert np.abs(q).max() <= qmax


# ------------------------------------------------------------ routing

def test_topk_matches_stable_argsort_with_ties():
    rng = np.random.default_rng(4)
    logits = rng.integers(-3, 4, size=(50, 24)).astype(np.float64)  # many ties
    for k in (1, 3, 8, 24):
        idx, gates = O.select_topk(logits, k)
        ref = np.argsort(-logits, axis=1, kind="stable")[:, :k]
        assert np.array_equal(idx, ref)


def test_gates_are_renormalised_full_softmax():
    rng = np.random.default_rng(5)
    logits = rng.standard_normal((40, 32)) * 3
    idx, gates = O.select_topk(logits, 5)
    np.testing.assert_allclose(gates.sum(1), 1.0, rtol=0, atol=1e-12)
    full = np.exp(logits) / np.exp(logits).sum(1, keepdims=True)
    sel = np.take_along_axis(full, idx, 1)
    np.testing.assert_allclose(gates, sel / sel.sum(1, keepdims=True), rtol=1e-12, atol=0)
    assert np.all(np.diff(gates, axis=1) <= 0)   # rank order = gate order


def test_route_plan_matches_library_routines():
    rng = np.random.default_rng(6)
    T, k, E = 37, 4, 11
    idx = np.stack([rng.choice(E, k, replace=False) for _ in range(T)])
    counts, offsets, perm, inv = O.route_plan(idx, E)
    flat = idx.ravel()
    assert np.array_equal(counts, np.bincount(flat, minlength=E))
    assert np.array_equal(offsets, np.concatenate([[0], np.cumsum(np.bincount(flat, minlength=E))]))
    a = np.arange(T * k)
    ref_perm = np.argsort(flat * (T * k) + a, kind="stable")
    assert np.array_equal(perm, ref_perm)
    assert np.array_equal(inv[perm], a)
    assert np.array_equal(flat[perm], np.sort(flat))


def test_silu_against_tanh_identity():
    z = np.linspace(-6, 30, 1001)
    np.testing.assert_allclose(O.silu(z), z * (1 + np.tanh(z / 2)) / 2, rtol=1e-12, atol=1e-15)
    zn = np.linspace(-40, 0, 1001)       # tail: the same function written as z e^z / (1 + e^z)
    np.testing.assert_allclose(O.silu(zn), zn * np.exp(zn) / (1 + np.exp(zn)), rtol=1e-13, atol=0)
    assert O.silu(np.array([-800.0]))[0] == 0.0
    assert O.silu(np.array([1.0]))[0] == 1.0 / (1.0 + math.exp(-1.0))


# ------------------------------------------------------------ layer invariants

def _tiny_args(L):
    return (L.x, L.router_w, L.router_bias, bank_dict(L.routed), bank_dict(L.shared), L.cfg.k)


def test_tiny_vectorised_equals_loops(tiny_layer):
    toks = [0, 5, 17, 63]
    r = O.layer_forward(*_tiny_args(tiny_layer), tokens=toks)
    loops = O.layer_forward_loops(*_tiny_args(tiny_layer), tokens=toks)
    np.testing.assert_allclose(r["out"], loops, rtol=1e-12, atol=1e-14)


def test_token_permutation_equivariance(tiny_layer):
    L = tiny_layer
    args = _tiny_args(L)
    r = O.layer_forward(*args)
    p = np.random.default_rng(7).permutation(L.cfg.T)
    r2 = O.layer_forward(L.x[p], *args[1:])
    assert np.array_equal(r2["idx"], r["idx"][p])
    np.testing.assert_array_equal(r2["out"], r["out"][p])


def test_single_expert_reduces_to_dense_swiglu():
    """E = 1, k = 1, no shared expert: the layer is a dense SwiGLU MLP (gate 1)."""
    cfg = synth.LayerConfig("e1", T=9, d=256, E=1, k=1, f=128, n_shared=0, fmt="int4")
    wr, bias = synth.make_router(cfg)
    x = synth.make_hidden(cfg, wr, bias)
    bank = synth.make_bank(cfg, "routed")
    r = O.layer_forward(x, wr, None, bank_dict(bank), None, 1)
    assert np.all(r["gates"] == 1.0) and np.all(r["idx"] == 0)
    X = torch.from_numpy(x.view(np.int16)).view(torch.bfloat16).to(torch.float64)
    def W(words, sb, K):
        q = torch.from_numpy(O.unpack_int4(words, K)).to(torch.float64)
        s = torch.from_numpy(sb.view(np.int16)).view(torch.bfloat16).to(torch.float64)
        return q * s.repeat_interleave(128, dim=1)
    Wg, Wu, Wd = W(bank.w_gate[0], bank.s_gate[0], 256), W(bank.w_up[0], bank.s_up[0], 256), \
        W(bank.w_down[0], bank.s_down[0], 128)
    dense = torch.nn.functional.linear(
        torch.nn.functional.silu(torch.nn.functional.linear(X, Wg)) * torch.nn.functional.linear(X, Wu), Wd)
    np.testing.assert_allclose(r["out"], dense.numpy(), rtol=1e-11, atol=1e-13)


def test_shared_and_routed_parts_separate(tiny_layer):
    L = tiny_layer
    x, wr, b, routed, shared, k = _tiny_args(L)
    full = O.layer_forward(x, wr, b, routed, shared, k)["out"]
    only_shared = O.layer_forward(x, wr, b, routed, shared, k, routed_scale=0.0)["out"]
    only_routed = O.layer_forward(x, wr, b, routed, None, k)["out"]
    np.testing.assert_allclose(full, only_shared + only_routed, rtol=1e-12, atol=1e-15)
    double = O.layer_forward(x, wr, b, routed, shared, k, routed_scale=2.0)["out"]
    np.testing.assert_allclose(double, only_shared + 2 * only_routed, rtol=1e-12, atol=1e-15)
    # the shared part alone is the dense SwiGLU of the shared expert on every token
    Wg, Wu, Wd = (O.widen_bf16(shared[n][0]) for n in ("w_gate", "w_up", "w_down"))
    X = O.widen_bf16(x)
    h = (X @ Wg.T) * (1 + np.tanh((X @ Wg.T) / 2)) / 2 * (X @ Wu.T)
    np.testing.assert_allclose(only_shared, h @ Wd.T, rtol=1e-10, atol=1e-14)



def test_mixed_bank_formats_shared_part_is_dense_int8_swiglu():
    """int4 routed experts beside an int8 shared expert: the layer minus its routed part is the
    dense SwiGLU of the shared expert's dequantised int8 weights (q * s, group 128) on every
    token, computed here with torch matmuls in fp64."""
    cfg = synth.LayerConfig("mixed", T=7, d=256, E=6, k=2, f=128, n_shared=1, fmt="int4",
                            shared_fmt="int8", seed=5)
    L = synth.make_layer(cfg)
    assert L.routed.fmt == "int4" and L.shared.fmt == "int8"
    routed, shared = bank_dict(L.routed), bank_dict(L.shared)
    full = O.layer_forward(L.x, L.router_w, L.router_bias, routed, shared, cfg.k)["out"]
    no_shared = O.layer_forward(L.x, L.router_w, L.router_bias, routed, None, cfg.k)["out"]
    X = torch.from_numpy(L.x.view(np.int16)).view(torch.bfloat16).to(torch.float64)
    def W(q8, sb):
        q = torch.from_numpy(q8.astype(np.float64))
        s = torch.from_numpy(sb.view(np.int16)).view(torch.bfloat16).to(torch.float64)
        return q * s.repeat_interleave(128, dim=1)
    Wg, Wu, Wd = (W(getattr(L.shared, "w_" + n)[0], getattr(L.shared, "s_" + n)[0])
                  for n in ("gate", "up", "down"))
    F = torch.nn.functional
    dense = F.linear(F.silu(F.linear(X, Wg)) * F.linear(X, Wu), Wd).numpy()
    np.testing.assert_allclose(full - no_shared, dense, rtol=1e-9, atol=1e-13)

# ------------------------------------------------------------ planted mistakes

@pytest.mark.parametrize("mistake", ["tie_high_index", "silu_sign", "drop_shared",
                                     "gates_unnormalised", "plan_unstable", "down_transposed"])
def test_planted_mistakes_are_caught(monkeypatch, mistake):
    """Each plausible bug, planted in the oracle, fails at least one pin."""
    if mistake == "tie_high_index":
        def bad(logits, k):
            T, E = logits.shape
            idx = np.empty((T, k), np.int64); gates = np.empty((T, k))
            for t in range(T):
                sel = sorted(range(E), key=lambda e: (-logits[t, e], -e))[:k]
                idx[t] = sel; z = np.exp(logits[t, sel] - logits[t, sel].max()); gates[t] = z / z.sum()
            return idx, gates
        monkeypatch.setattr(O, "select_topk", bad)
    elif mistake == "silu_sign":
        monkeypatch.setattr(O, "silu", lambda z: z / (1.0 + np.exp(z)))
    elif mistake == "drop_shared":
        real = O.layer_forward
        monkeypatch.setattr(O, "layer_forward",
                            lambda x, wr, b, r, s, k, **kw: real(x, wr, b, r, None, k, **kw))
    elif mistake == "gates_unnormalised":
        real = O.select_topk
        def bad(logits, k):
            idx, g = real(logits, k)
            return idx, np.take_along_axis(np.exp(logits), idx, 1)
        monkeypatch.setattr(O, "select_topk", bad)
    elif mistake == "plan_unstable":
        real = O.route_plan
        def bad(idx, E):
            c, o, p, i = real(idx, E)
            p = p.copy(); i = i.copy()
            # reverse the token order inside the expert with most rows
            e = int(np.argmax(c)); seg = p[o[e]:o[e + 1]][::-1].copy(); p[o[e]:o[e + 1]] = seg
            i[p] = np.arange(p.size)
            return c, o, p, i
        monkeypatch.setattr(O, "route_plan", bad)
    elif mistake == "down_transposed":
        monkeypatch.setattr(O, "expert_ffn",
                            lambda x, Wg, Wu, Wd: (O.silu(x @ Wg.T) * (x @ Wu.T)) @ Wd[::-1].T)
    with pytest.raises(AssertionError):
        _check_worked(O.layer_forward)


def test_bf16_half_ulp_helper():
    """The rounding allowance used by the parity tests equals the distance to the next
    bf16 value / 2 (checked with torch's own bf16 rounding)."""
    from conftest import bf16_half_ulp
    v = np.array([1.0, 1.5, 1.99, 2.0, 3.9, 0.3, -0.7, 1e-3])
    nxt = torch.from_numpy(v).to(torch.bfloat16).view(torch.int16) + 1
    gap = (nxt.view(torch.bfloat16).to(torch.float64) -
           torch.from_numpy(v).to(torch.bfloat16).to(torch.float64)).abs().numpy()
    assert np.array_equal(bf16_half_ulp(v), gap / 2)
