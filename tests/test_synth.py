"""The seeded input generator: determinism, encodings, routing margin, skew."""
import numpy as np

from expert_routed_ffn_route_b200 import synth
from oracle import moe_oracle as O


def test_deterministic_and_subset_regeneration():
    cfg = synth.LayerConfig("s", T=8, d=256, E=8, k=2, f=128, fmt="int4")
    a = synth.make_bank(cfg, "routed")
    b = synth.make_bank(cfg, "routed", experts=[3])
    assert np.array_equal(a.w_gate[3], b.w_gate[3]) and np.array_equal(a.s_down[3], b.s_down[3])
    c = synth.make_bank(cfg, "routed")
    for n in ("w_gate", "w_up", "w_down", "s_gate", "s_up", "s_down"):
        assert np.array_equal(getattr(a, n), getattr(c, n))
    assert a.w_gate.shape == (8, 128, 32) and a.w_gate.dtype == np.uint32
    assert a.s_gate.shape == (8, 128, 2) and a.w_down.shape == (8, 256, 16)


def test_int4_codes_in_range():
    cfg = synth.LayerConfig("s", T=8, d=256, E=2, k=1, f=128, fmt="int4")
    bank = synth.make_bank(cfg, "routed")
    q = O.unpack_int4(bank.w_gate, 256)
    assert q.min() >= -7 and q.max() <= 7


def test_routing_margin_holds():
    cfg = synth.CONFIGS["decode"]
    wr, bias = synth.make_router(cfg)
    x = synth.make_hidden(cfg, wr, bias, T=64)
    l = O.router_logits(x, wr, bias)
    top = -np.sort(-l, axis=1)[:, :cfg.k + 1]
    assert np.all(top[:, :-1] - top[:, 1:] >= cfg.margin)


def test_zipf_bias_skews_load():
    cfg = synth.CONFIGS["long"]
    wr, bias = synth.make_router(cfg)
    x = synth.make_hidden(cfg, wr, bias, T=512)
    idx = np.argsort(-O.router_logits(x, wr, bias), axis=1, kind="stable")[:, :cfg.k]
    cnt = np.bincount(idx.ravel(), minlength=cfg.E)
    mean = idx.size / cfg.E
    assert cnt.max() > 10 * mean


def test_shared_bank_format_option():
    """shared_fmt draws the shared bank in its own encoding; the routed bank is unchanged."""
    base = synth.LayerConfig("m", T=4, d=256, E=4, k=2, f=128, fmt="int4", seed=3)
    mixed = synth.LayerConfig("m", T=4, d=256, E=4, k=2, f=128, fmt="int4", shared_fmt="int8",
                              seed=3)
    a, b = synth.make_layer(base), synth.make_layer(mixed)
    assert b.shared.fmt == "int8" and b.routed.fmt == "int4"
    assert np.array_equal(a.routed.w_gate, b.routed.w_gate)
    assert b.shared.w_gate.dtype == np.int8 and np.abs(b.shared.w_gate.astype(np.int32)).max() <= 127
