"""Helpers shared by the GPU parity tests: device transfers, the oracle run of a layer and
the element-by-element comparison of one library call against it.

Bar: expert indices, the plan (offsets, perm, inv) bit-exact; gates within 1e-5; the bf16
layer output within max|d| <= 1e-2 * rms(oracle) + 1e-3, counted beyond the output's own
rounding to bf16; bitwise run-to-run determinism.
"""
import numpy as np

from oracle import moe_oracle as O
from expert_routed_ffn_route_b200 import synth
from conftest import bank_dict, out_tol, output_excess

GATE_TOL = 1e-5
TC_ROWS_PER_TILE = 64  # token rows of one tensor-core unit (an m-tile of an expert's rows)


def to_dev_x(x_bits):
    import torch
    return torch.from_numpy(x_bits.view(np.int16)).cuda().view(torch.bfloat16)


def bf16_to_np(t):
    import torch
    return t.view(torch.int16).cpu().numpy().view(np.uint16)


def oracle_run(L: synth.LayerInputs, tokens=None, x=None):
    x = L.x if x is None else x
    return O.layer_forward(x, L.router_w, L.router_bias, bank_dict(L.routed),
                           bank_dict(L.shared), L.cfg.k, tokens=tokens)


def plan_edge_tokens(L: synth.LayerInputs, n_hot=5, n_total=0, seed=0):
    """Tokens whose rows sit at the edges of the tensor-core units of the most loaded
    experts (the oracle's plan): the first grouped row of each hot expert, the first and
    last row of its last (ragged) m-tile and the row before that tile, and the first and
    last token; then tokens drawn with a seeded generator until ``n_total`` are listed.
    Sorted, without repeats."""
    lg = O.router_logits(L.x, L.router_w, L.router_bias)
    idx, _ = O.select_topk(lg, L.cfg.k)
    counts, offsets, perm, _ = O.route_plan(idx, L.cfg.E)
    hot = np.argsort(-counts, kind="stable")[:n_hot]
    toks = set()
    for e in hot:
        lo, hi = int(offsets[e]), int(offsets[e + 1])
        if hi <= lo:
            continue
        last0 = lo + ((hi - lo - 1) // TC_ROWS_PER_TILE) * TC_ROWS_PER_TILE
        for r in {lo, last0, hi - 1, max(lo, last0 - 1)}:
            toks.add(int(perm[r]) // L.cfg.k)
    T = L.x.shape[0]
    toks.update({0, T - 1})
    if n_total > len(toks):
        rng = np.random.default_rng(seed)
        rest = np.setdiff1d(np.arange(T), np.fromiter(toks, int, len(toks)))
        n = min(n_total - len(toks), rest.size)
        toks.update(int(t) for t in rng.choice(rest, size=n, replace=False))
    return sorted(toks)


def check_layer(B, dl, L, x_bits, path, sample=None, check_stages=True):
    import torch
    T = x_bits.shape[0]
    desc = dl.descriptor(T, path)
    ws = B.alloc_workspace(desc)
    x = to_dev_x(x_bits)
    idx = torch.empty((T, L.cfg.k), dtype=torch.int32, device="cuda")
    w = torch.empty((T, L.cfg.k), dtype=torch.float32, device="cuda")
    offs = torch.empty(L.cfg.E + 1, dtype=torch.int32, device="cuda")
    perm = torch.empty(T * L.cfg.k, dtype=torch.int32, device="cuda")
    out = B.layer_forward(desc, x, ws, topk_idx=idx, topk_w=w, offsets=offs, perm=perm)
    out2 = B.layer_forward(desc, x, ws)
    torch.cuda.synchronize()
    assert B.device_status(desc, ws) == 0
    assert torch.equal(out.view(torch.int16), out2.view(torch.int16)), "not deterministic"

    tokens = np.arange(T) if sample is None else np.asarray(sample)
    ref = oracle_run(L, tokens=tokens, x=x_bits)
    assert np.array_equal(idx.cpu().numpy(), ref["idx"]), "expert indices differ"
    np.testing.assert_allclose(w.cpu().numpy(), ref["gates"], rtol=0, atol=GATE_TOL)
    assert np.array_equal(offs.cpu().numpy(), ref["offsets"])
    assert np.array_equal(perm.cpu().numpy(), ref["perm"])
    got = O.widen_bf16(bf16_to_np(out))[tokens]
    err = float(output_excess(got, ref["out"]).max())
    raw = float(np.abs(got - ref["out"]).max())
    print(f"[{L.cfg.name} T={T} {path}] rows {len(tokens)}: max|d| {raw:.3e}, beyond bf16 "
          f"rounding {err:.3e}, bound {out_tol(ref['out']):.3e}")
    assert err <= out_tol(ref["out"]), f"max excess {err} > {out_tol(ref['out'])}"

    if check_stages:
        # the four stage entry points give the multi-kernel call's result bit for bit (the
        # single-kernel 1-token layer sums in another order: there, both meet the oracle)
        i2, w2 = B.route(desc, x, ws)
        o2, p2, inv2 = B.permute(desc, i2, ws)
        ya, ys = B.grouped_ffn(desc, x, o2, p2, ws, has_shared=dl.has_shared)
        out3 = B.combine(desc, ya, ys, inv2, w2)
        torch.cuda.synchronize()
        one_kernel = B.launches_per_call(desc) == 1
        assert torch.equal(i2, idx)
        if one_kernel:  # logits summed in another order: gates agree to the gate tolerance
            np.testing.assert_allclose(w2.cpu().numpy(), w.cpu().numpy(), rtol=0, atol=GATE_TOL)
        else:
            assert torch.equal(w2, w)
        assert torch.equal(o2, offs) and torch.equal(p2, perm)
        assert np.array_equal(inv2.cpu().numpy(), ref["inv"])
        if one_kernel:
            got3 = O.widen_bf16(bf16_to_np(out3))[tokens]
            assert float(output_excess(got3, ref["out"]).max()) <= out_tol(ref["out"])
        else:
            assert torch.equal(out3.view(torch.int16), out.view(torch.int16))
    return err, ref
