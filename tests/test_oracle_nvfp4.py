"""Pins of the NVFP4 (W4A4) oracle: the format's value sets and rounding against torch's
float8_e4m3fn and brute force, exact results on exactly representable rows, the dense
single-expert reduction through torch matmuls, row independence, the quantisation error
against the unquantised layer, and a planted mistake."""
import numpy as np
import pytest
import torch

from oracle import moe_oracle as O
from oracle import nvfp4 as N
from expert_routed_ffn_route_b200 import synth
from conftest import bank_dict


def test_e2m1_decode_enumerates_the_format():
    expect = [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]
    v = N.e2m1_value(np.arange(16))
    assert v[:8].tolist() == expect
    assert (-v[8:]).tolist() == expect
    assert np.signbit(v[8]) and not np.signbit(v[0])


def test_e4m3_decode_matches_torch():
    codes = np.arange(256, dtype=np.uint8)
    ref = torch.from_numpy(codes).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    got = N.e4m3_value(codes)
    assert np.array_equal(np.isnan(ref), np.isnan(got))
    ok = ~np.isnan(ref)
    assert np.array_equal(ref[ok], got[ok])
    assert np.nanmax(got) == 448.0


def test_round_e4m3_matches_torch():
    rng = np.random.default_rng(1)
    v = np.exp(rng.uniform(np.log(1e-4), np.log(448.0), 20000)).astype(np.float32)
    finite = N.e4m3_value(np.arange(0x7F))
    mids = ((finite[1:] + finite[:-1]) / 2).astype(np.float32)  # exact ties
    v = np.concatenate([v, mids, finite.astype(np.float32), np.float32([0.0, 448.0])])
    ref = torch.from_numpy(v).to(torch.float8_e4m3fn).view(torch.uint8).numpy().astype(np.int64)
    assert np.array_equal(N.round_e4m3(v), ref)
    assert N.round_e4m3(np.float32([1000.0, 449.0])).tolist() == [0x7E, 0x7E]  # saturates


def test_round_e2m1_brute_force():
    grid = [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]
    rng = np.random.default_rng(2)
    vals = list(rng.uniform(-8, 8, 3000)) + [0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0, -5.0, 6.5]
    got = N.round_e2m1(np.array(vals))
    for v, c in zip(vals, got):
        a = min(abs(v), 6.0)
        best = None
        for code, g in enumerate(grid):       # nearest, ties to the even code
            dist = abs(a - g)
            if best is None or dist < best[0] or (dist == best[0] and code % 2 == 0):
                best = (dist, code)
        assert c == best[1] | (8 if v < 0 else 0), (v, c, best)


def test_exactly_representable_rows_round_trip():
    # row amax 6c with blocks of amax 6c, 3c and 1.5c, c = 448 * 2^-12: the row scale
    # g = 6c / (6 * 448) = 2^-12 and the block scales 448, 224 and 112 are exact, so every
    # element lands on the grid and every step is exact
    c = 448.0 * 2.0 ** -12
    grid = np.array([0, .5, 1, 1.5, 2, 3, 4, 6, 0, -.5, -1, -1.5, -2, -3, -4, -6])
    row = np.concatenate([grid * c, grid * c / 2, grid * c / 4]).astype(np.float32)[None, :]
    codes, sc, g = N.nvfp4_quantize_rows(row)
    assert g[0] == np.float32(2.0 ** -12)
    assert N.e4m3_value(sc[0]).tolist() == [448.0, 224.0, 112.0]
    assert np.array_equal(N.nvfp4_dequantize(codes, sc, g), row.astype(np.float64))
    z_codes, z_sc, z_g = N.nvfp4_quantize_rows(np.zeros((1, 32), np.float32))
    assert z_g[0] == 0 and not z_codes.any() and not z_sc.any()


def test_row_quantisation_error_bound():
    """Every element is the nearest grid point of v / scale (brute force) times the scale."""
    rng = np.random.default_rng(3)
    rows = (rng.standard_normal((6, 64)) * rng.uniform(0.01, 3, (6, 1))).astype(np.float32)
    rows[2, 16:32] = 0.0                                 # a zero block
    codes, sc, g = N.nvfp4_quantize_rows(rows)
    deq = N.nvfp4_dequantize(codes, sc, g)
    scale32 = N.e4m3_value(sc).astype(np.float32) * g[:, None]         # the decision's scale
    exact = N.e4m3_value(sc) * g.astype(np.float64)[:, None]          # the value's scale
    grid = np.array([0, .5, 1, 1.5, 2, 3, 4, 6])
    for r in range(rows.shape[0]):
        for k in range(64):
            if scale32[r, k // 16] == 0:
                assert deq[r, k] == 0
                continue
            y = min(abs(np.float64(np.float32(rows[r, k] / scale32[r, k // 16]))), 6.0)
            best = min(abs(y - gv) for gv in grid)
            level = abs(deq[r, k]) / exact[r, k // 16]
            assert level in grid and abs(y - level) <= best       # a nearest grid point
            assert deq[r, k] == 0 or np.sign(deq[r, k]) == np.sign(rows[r, k])


def _layer(T=5, E=4, k=2, shared="bf16", seed=7):
    cfg = synth.LayerConfig("nv", T=T, d=256, E=E, k=k, f=128, fmt="nvfp4", shared_fmt=shared,
                            seed=seed, n_shared=1 if shared else 0)
    L = synth.make_layer(cfg)
    routed = dict(fmt="nvfp4", **L.routed.arrays())
    return cfg, L, routed, (bank_dict(L.shared) if L.shared is not None else None)


def test_generator_follows_the_weight_recipe():
    cfg, L, routed, _ = _layer(T=2)
    w = synth._normal((cfg.f, cfg.d), cfg.weight_std, cfg.seed, "routed", "gate", 1)
    g = np.float32(L.routed.g_gate[1])
    assert g == np.float32(np.abs(w).max() / np.float32(2688.0))
    amax_b = np.abs(w.reshape(cfg.f, -1, 16)).max(axis=2)
    assert np.array_equal(L.routed.s_gate[1], N.round_e4m3(amax_b / (np.float32(6) * g)))
    deq = N.nvfp4_dequantize(N.unpack_fp4(L.routed.w_gate[1], cfg.d), L.routed.s_gate[1], g)
    step = np.repeat(N.e4m3_value(L.routed.s_gate[1]), 16, axis=1) * np.float64(g)
    assert np.all(np.abs(deq - w) <= step + 1e-12)     # within one grid step of the scale


def test_single_expert_reduces_to_dense_w4a4_mlp():
    cfg, L, routed, _ = _layer(T=4, E=1, k=1, shared=None)
    r = N.layer_forward_nvfp4(L.x, L.router_w, None, routed, None, 1)
    assert np.all(r["gates"] == 1.0) and np.all(r["idx"] == 0)
    Wg, Wu, Wd = (torch.from_numpy(N.nvfp4_dequantize(
        N.unpack_fp4(routed["w_" + n][0], K), routed["s_" + n][0], np.float64(routed["g_" + n][0])))
        for n, K in (("gate", 256), ("up", 256), ("down", 128)))
    X = O.widen_bf16(L.x).astype(np.float32)
    xq = torch.from_numpy(N.nvfp4_dequantize(*N.nvfp4_quantize_rows(X)))
    F = torch.nn.functional
    h = F.silu(F.linear(xq, Wg)) * F.linear(xq, Wu)
    hq = torch.from_numpy(N.nvfp4_dequantize(*N.nvfp4_quantize_rows(h.numpy().astype(np.float32))))
    np.testing.assert_allclose(r["out"], F.linear(hq, Wd).numpy(), rtol=1e-12, atol=1e-15)


def test_rows_are_independent():
    cfg, L, routed, shared = _layer(T=6)
    full = N.layer_forward_nvfp4(L.x, L.router_w, L.router_bias, routed, shared, cfg.k)["out"]
    for t in (0, 3, 5):
        one = N.layer_forward_nvfp4(L.x[t:t + 1], L.router_w, L.router_bias, routed, shared,
                                    cfg.k)["out"]
        np.testing.assert_allclose(one[0], full[t], rtol=1e-12, atol=1e-16)  # BLAS order aside


def test_token_subset_equals_the_full_call():
    """The ``tokens`` option computes the listed rows only (routing and the plan stay those of
    the whole call): each listed row equals the full call's row, in the order listed (up to the
    fp64 matrix routine's summation order over a different number of rows)."""
    cfg, L, routed, shared = _layer(T=6)
    full = N.layer_forward_nvfp4(L.x, L.router_w, L.router_bias, routed, shared, cfg.k)
    sub = N.layer_forward_nvfp4(L.x, L.router_w, L.router_bias, routed, shared, cfg.k,
                                tokens=[4, 1, 5])
    np.testing.assert_allclose(sub["out"], full["out"][[4, 1, 5]], rtol=1e-12, atol=1e-16)  # BLAS order aside
    assert np.array_equal(sub["idx"], full["idx"]) and np.array_equal(sub["perm"], full["perm"])


def test_generator_e2m1_rounding_matches_the_oracle():
    """The generator's vectorised E2M1 rounding (which fixes the stored weight codes) takes
    the oracle's decisions: nearest, ties to the even code, saturation at 6, the sign bit."""
    rng = np.random.default_rng(13)
    grid = N.e2m1_value(np.arange(8))
    mids = (grid[1:] + grid[:-1]) / 2
    v = np.concatenate([rng.uniform(-8, 8, 20000), mids, -mids, grid, -grid,
                        [6.5, -7.0, 0.0, -0.0, 1e-9, -1e-9]]).astype(np.float32)
    assert np.array_equal(synth.e2m1_codes(v).astype(np.int64), N.round_e2m1(v))


def _unquantised_error(layer_fn):
    cfg, L, routed, shared = _layer(T=8, E=6, k=2, seed=11)
    w4a4 = layer_fn(L.x, L.router_w, L.router_bias, routed, shared, cfg.k)["out"]
    # the same weights unquantised in the activations: decoded NVFP4 weights as a bf16-free
    # float64 bank through the plain expert, same routing
    exact = np.zeros_like(w4a4)
    X = O.widen_bf16(L.x)
    idx, gates = O.select_topk(O.router_logits(L.x, L.router_w, L.router_bias), cfg.k)
    for t in range(cfg.T):
        for j in range(cfg.k):
            e = int(idx[t, j])
            W = [N.nvfp4_dequantize(N.unpack_fp4(routed["w_" + n][e], K), routed["s_" + n][e],
                                    np.float64(routed["g_" + n][e]))
                 for n, K in (("gate", cfg.d), ("up", cfg.d), ("down", cfg.f))]
            exact[t] += gates[t, j] * O.expert_ffn(X[t:t + 1], *W)[0]
    exact += _shared_only(L)
    return np.sqrt(np.mean((w4a4 - exact) ** 2)) / np.sqrt(np.mean(exact ** 2))


def _shared_only(L):
    X = O.widen_bf16(L.x)
    Wg, Wu, Wd = (O.widen_bf16(L.shared.arrays()["w_" + n][0]) for n in ("gate", "up", "down"))
    return O.expert_ffn(X, Wg, Wu, Wd)


def test_activation_quantisation_error_is_bounded():
    """4-bit activations (x and h) cost about a tenth of the output's rms (0.092 at this
    seed), far from the thousands a misplaced scale gives."""
    err = _unquantised_error(N.layer_forward_nvfp4)
    assert 0.0 < err < 0.2, err


def test_planted_mistake_dropped_row_scale_is_caught(monkeypatch):
    real = N.nvfp4_dequantize

    def wrong(codes, scale_codes, g):  # forgets the tensor scale of activation rows
        if np.ndim(g) == 1:
            return real(codes, scale_codes, np.ones_like(np.asarray(g)))
        return real(codes, scale_codes, g)
    monkeypatch.setattr(N, "nvfp4_dequantize", wrong)
    with pytest.raises(AssertionError):
        test_activation_quantisation_error_is_bounded()
