"""Seeded synthetic inputs for the expert-routed MoE FFN layer.

This module only draws and encodes inputs. It holds none of the layer's own
arithmetic (routing, grouping, the SwiGLU experts, the weighted combine): the
CUDA library and the fp64 oracle each implement that on their own, and both
read the arrays produced here.

Workload shapes follow the model the pages describe (TandemLLM docs,
"17 Qwen3.8-Flash-Next", Table 17.1: 512 experts a layer, 10 routed + 1 shared
per token, residual stream 2,560 wide) and its weight format
(Qwen3.8-Flash-Next-Dual-GPU README, "Model artifact and memory placement":
routed experts symmetric W4 or W8 with groups of 128, BF16 group scales,
router kept in BF16/F32). The expert width 1,024 is not on the pages; it is
the width this workload fixes.

Encodings produced here (the library's input layouts):

* bf16 tensors are numpy ``uint16`` arrays holding the bf16 bit pattern.
* ``int4``: two's-complement nibbles, 8 per ``uint32`` along K; element ``kk``
  of a row sits in word ``kk // 8`` at bits ``4 * (kk % 8)``.
* ``int8``: plain ``int8`` along K.
* scales: bf16 bits, shape ``[..., N, K // group]``.

Quantiser (the encoding step, done once here): per group of ``group`` weights
along K, ``s = bf16(max|w| / qmax)`` and ``q = clamp(round_half_even(w / s),
-qmax, qmax)`` with ``qmax`` 7 (int4) or 127 (int8); an all-zero group gets
``s = 0, q = 0``.

Routing margin: every token is redrawn until the gaps between adjacent logits
among its top ``k + 1`` (bias included, evaluated in float64 on the bf16
values) are at least ``margin``, so that the top-k set and its order are
well-defined under any accumulation order. This evaluation only filters draws.
"""
from __future__ import annotations

import hashlib
import os
from concurrent.futures import ThreadPoolExecutor
from dataclasses import dataclass, field

import numpy as np

__all__ = [
    "LayerConfig", "CONFIGS", "Bank", "LayerInputs", "make_layer", "make_bank",
    "make_router", "make_hidden", "bf16_bits", "bf16_bits_to_f32", "pack_int4",
    "quantize_groups", "derive_seed", "FMT_BITS", "plant_ties",
]

FMT_BITS = {"bf16": 16, "int8": 8, "int4": 4, "nvfp4": 4}


@dataclass(frozen=True)
class LayerConfig:
    name: str
    T: int          # tokens
    d: int          # d_model (K of gate/up, N of down)
    E: int          # routed experts
    k: int          # routed experts per token
    f: int          # expert width (N of gate/up, K of down)
    n_shared: int = 1
    fmt: str = "int4"            # routed bank format (and the shared bank's by default)
    group: int = 128
    weight_std: float = 0.02
    zipf_s: float | None = None  # router bias popularity exponent (None: no bias)
    margin: float = 1e-3
    seed: int = 0
    shared_fmt: str | None = None  # shared bank format when it differs from fmt


# The five workloads. "tiny" is small enough for brute force on the CPU.
CONFIGS = {
    "tiny": LayerConfig("tiny", T=64, d=256, E=16, k=2, f=128, fmt="bf16"),
    "decode": LayerConfig("decode", T=1, d=2560, E=512, k=10, f=1024, fmt="int4"),
    "verify16": LayerConfig("verify16", T=16, d=2560, E=512, k=10, f=1024, fmt="int4"),
    "verify32": LayerConfig("verify32", T=32, d=2560, E=512, k=10, f=1024, fmt="int4"),
    "prefill": LayerConfig("prefill", T=512, d=2560, E=512, k=10, f=1024, fmt="int4"),
    "long": LayerConfig("long", T=4096, d=2560, E=512, k=10, f=1024, fmt="int8",
                        zipf_s=1.1),
    # the W4A4 variant (NVFP4 routed experts, BF16 shared expert) on the prefill shapes
    "prefill_nvfp4": LayerConfig("prefill_nvfp4", T=512, d=2560, E=512, k=10, f=1024,
                                 fmt="nvfp4", shared_fmt="bf16"),
    "long_nvfp4": LayerConfig("long_nvfp4", T=4096, d=2560, E=512, k=10, f=1024, fmt="nvfp4",
                              shared_fmt="bf16", zipf_s=1.1),
}


def derive_seed(*parts) -> int:
    """A 63-bit seed from a tuple of labels (stable across machines)."""
    h = hashlib.blake2b(repr(parts).encode(), digest_size=8).digest()
    return int.from_bytes(h, "little") & ((1 << 63) - 1)


def _normal(shape, std, *seed_parts) -> np.ndarray:
    """float32 N(0, std^2) from a PCG64 stream keyed by ``seed_parts``."""
    rng = np.random.default_rng(derive_seed(*seed_parts))
    a = rng.standard_normal(shape, dtype=np.float32)
    if std != 1.0:
        a *= np.float32(std)
    return a


def bf16_bits(a) -> np.ndarray:
    """Round finite float32 values to bf16 (nearest-even); return uint16 bits."""
    u = np.ascontiguousarray(a, dtype=np.float32).view(np.uint32)
    r = (u + np.uint32(0x7FFF) + ((u >> np.uint32(16)) & np.uint32(1))) >> np.uint32(16)
    return r.astype(np.uint16)


def bf16_bits_to_f32(u: np.ndarray) -> np.ndarray:
    return (u.astype(np.uint32) << 16).view(np.float32)


def pack_int4(q: np.ndarray) -> np.ndarray:
    """int8 values in [-8, 7], shape [..., K] -> uint32 [..., K // 8]."""
    K = q.shape[-1]
    assert K % 8 == 0
    nib = (q.astype(np.int32) & 0xF).astype(np.uint32).reshape(*q.shape[:-1], K // 8, 8)
    shifts = (4 * np.arange(8, dtype=np.uint32))
    return np.bitwise_or.reduce(nib << shifts, axis=-1).astype(np.uint32)


def quantize_groups(w: np.ndarray, qmax: int, group: int):
    """Symmetric per-group quantiser along the last axis (float32 arithmetic).

    Returns (q int8 [N, K], scale bits uint16 [N, K // group]).
    """
    N, K = w.shape
    wg = w.reshape(N, K // group, group)
    amax = np.abs(wg).max(axis=-1)
    sb = bf16_bits(amax / np.float32(qmax))
    s = bf16_bits_to_f32(sb)
    safe = np.where(s > 0, s, np.float32(1.0))
    q = np.rint(wg / safe[..., None])          # rint: round half to even
    np.clip(q, -qmax, qmax, out=q)
    q[s == 0] = 0
    return q.astype(np.int8).reshape(N, K), sb


# ---------------------------------------------------------------- NVFP4 encoding
# NVFP4 (NVIDIA's 4-bit floating-point weight format): E2M1 elements (magnitudes 0, 0.5, 1,
# 1.5, 2, 3, 4, 6), one E4M3 scale per 16 consecutive elements along K, one float32 scale per
# tensor; value = e2m1 * e4m3 * scale. Weights are encoded once here, in float32 arithmetic:
# tensor scale g = amax / (6 * 448), block scale = E4M3(amax_block / (6 g)) (round to nearest
# even, at most 448), element = E2M1(w / (block scale * g)) (round to nearest even, saturating
# at 6). Codes: bit 3 sign, bits 2..1 exponent, bit 0 mantissa; two per byte, element k in the
# nibble at bit 4 * (k % 2) of byte k // 2.
NVFP4_BLOCK = 16
_E2M1_GRID = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0], np.float32)


def e2m1_codes(v: np.ndarray) -> np.ndarray:
    """float32 values -> E2M1 codes (uint8), nearest, ties to the even code, saturating."""
    a = np.abs(v).astype(np.float32)
    mids = (_E2M1_GRID[1:] + _E2M1_GRID[:-1]) / np.float32(2)
    i = np.zeros(a.shape, np.uint8)  # number of mids strictly below a
    tie = np.zeros(a.shape, bool)    # a on a mid whose lower neighbour has an odd code
    for m, mid in enumerate(mids):
        i += a > mid
        if m % 2 == 1:
            tie |= a == mid
    i += tie
    return i | (np.signbit(v).astype(np.uint8) << 3)


def e4m3_codes(v: np.ndarray) -> np.ndarray:
    """Non-negative float32 values -> E4M3 (fn) codes, nearest even, at most 448."""
    import torch
    c = np.minimum(np.asarray(v, np.float32), np.float32(448.0))
    return torch.from_numpy(np.ascontiguousarray(c)).to(torch.float8_e4m3fn).view(torch.uint8).numpy()


def e4m3_to_f32(codes: np.ndarray) -> np.ndarray:
    import torch
    t = torch.from_numpy(np.ascontiguousarray(codes, np.uint8)).view(torch.float8_e4m3fn)
    return t.to(torch.float32).numpy()


def quantize_nvfp4(w: np.ndarray):
    """float32 [N, K] -> (packed codes uint8 [N, K/2], block scales uint8 [N, K/16],
    tensor scale float32)."""
    N, K = w.shape
    assert K % NVFP4_BLOCK == 0
    w = np.asarray(w, np.float32)
    g = np.float32(np.abs(w).max() / np.float32(6.0 * 448.0))
    wb = w.reshape(N, K // NVFP4_BLOCK, NVFP4_BLOCK)
    if g == 0:
        return (np.zeros((N, K // 2), np.uint8), np.zeros((N, K // NVFP4_BLOCK), np.uint8), g)
    amax_b = np.abs(wb).max(axis=-1)
    sc = e4m3_codes(amax_b / (np.float32(6.0) * g))
    scale = (e4m3_to_f32(sc) * g).astype(np.float32)
    safe = np.where(scale > 0, scale, np.float32(1.0))
    codes = e2m1_codes((wb / safe[..., None]).astype(np.float32))
    codes[scale == 0] = 0
    codes = codes.reshape(N, K)
    packed = (codes[:, 0::2] | (codes[:, 1::2] << 4)).astype(np.uint8)
    return packed, sc, g


@dataclass
class Bank:
    """One expert bank: n_exp experts of gate [f,d], up [f,d], down [d,f]."""
    fmt: str
    group: int
    n_exp: int
    d: int
    f: int
    w_gate: np.ndarray
    w_up: np.ndarray
    w_down: np.ndarray
    s_gate: np.ndarray | None = None
    s_up: np.ndarray | None = None
    s_down: np.ndarray | None = None
    # nvfp4 only: one float32 scale per (expert, matrix)
    g_gate: np.ndarray | None = None
    g_up: np.ndarray | None = None
    g_down: np.ndarray | None = None

    def arrays(self):
        a = dict(w_gate=self.w_gate, w_up=self.w_up, w_down=self.w_down,
                 s_gate=self.s_gate, s_up=self.s_up, s_down=self.s_down)
        if self.fmt == "nvfp4":
            a.update(g_gate=self.g_gate, g_up=self.g_up, g_down=self.g_down)
        return a


def _encode(w: np.ndarray, fmt: str, group: int):
    if fmt == "bf16":
        return bf16_bits(w), None
    if fmt == "int8":
        q, s = quantize_groups(w, 127, group)
        return q, s
    if fmt == "int4":
        q, s = quantize_groups(w, 7, group)
        return pack_int4(q), s
    raise ValueError(fmt)


def _alloc(fmt: str, n_exp: int, N: int, K: int, group: int):
    if fmt == "bf16":
        return np.empty((n_exp, N, K), np.uint16), None
    if fmt == "int8":
        return np.empty((n_exp, N, K), np.int8), np.empty((n_exp, N, K // group), np.uint16)
    return (np.empty((n_exp, N, K // 8), np.uint32),
            np.empty((n_exp, N, K // group), np.uint16))


def make_bank(cfg: LayerConfig, which: str, n_exp: int | None = None,
              experts=None) -> Bank:
    """Draw and encode an expert bank.

    ``which`` is "routed" (cfg.E experts) or "shared" (cfg.n_shared experts).
    Every (matrix, expert) pair has its own random stream, so any subset of
    experts can be regenerated alone. ``experts`` optionally restricts which
    experts are drawn (others stay uninitialised); used by CPU-side checks.
    """
    if n_exp is None:
        n_exp = cfg.E if which == "routed" else cfg.n_shared
    fmt = cfg.shared_fmt if (which == "shared" and cfg.shared_fmt) else cfg.fmt
    if fmt == "nvfp4":
        return _make_nvfp4_bank(cfg, which, n_exp, experts)
    d, f, g = cfg.d, cfg.f, cfg.group
    wg, sg = _alloc(fmt, n_exp, f, d, g)
    wu, su = _alloc(fmt, n_exp, f, d, g)
    wd, sd = _alloc(fmt, n_exp, d, f, g)
    todo = range(n_exp) if experts is None else experts
    jobs = [(int(e), name, shape, wa, sa) for e in todo
            for name, shape, wa, sa in (("gate", (f, d), wg, sg), ("up", (f, d), wu, su),
                                        ("down", (d, f), wd, sd))]

    def one(job):
        e, name, shape, wa, sa = job
        w = _normal(shape, cfg.weight_std, cfg.seed, which, name, e)
        q, s = _encode(w, fmt, g)
        wa[e] = q
        if sa is not None:
            sa[e] = s

    if len(jobs) <= 3:
        for j in jobs:
            one(j)
    else:
        with ThreadPoolExecutor(max_workers=min(32, os.cpu_count() or 1)) as ex:
            list(ex.map(one, jobs))
    return Bank(fmt, g, n_exp, d, f, wg, wu, wd, sg, su, sd)


def _make_nvfp4_bank(cfg: LayerConfig, which: str, n_exp: int, experts=None) -> Bank:
    """An NVFP4 bank over the same weight draws as the other formats."""
    d, f = cfg.d, cfg.f
    arrs = {}
    for name, (N, K) in (("gate", (f, d)), ("up", (f, d)), ("down", (d, f))):
        arrs[name] = (np.zeros((n_exp, N, K // 2), np.uint8),
                      np.zeros((n_exp, N, K // NVFP4_BLOCK), np.uint8),
                      np.zeros(n_exp, np.float32))
    todo = range(n_exp) if experts is None else experts
    jobs = [(int(e), name, N, K) for e in todo
            for name, (N, K) in (("gate", (f, d)), ("up", (f, d)), ("down", (d, f)))]

    def one(job):
        e, name, N, K = job
        w = _normal((N, K), cfg.weight_std, cfg.seed, which, name, e)
        q, sc, g = quantize_nvfp4(w)
        arrs[name][0][e], arrs[name][1][e], arrs[name][2][e] = q, sc, g

    if len(jobs) <= 3:
        for j in jobs:
            one(j)
    else:
        with ThreadPoolExecutor(max_workers=min(32, os.cpu_count() or 1)) as ex:
            list(ex.map(one, jobs))
    return Bank("nvfp4", NVFP4_BLOCK, n_exp, d, f, arrs["gate"][0], arrs["up"][0], arrs["down"][0],
                arrs["gate"][1], arrs["up"][1], arrs["down"][1],
                arrs["gate"][2], arrs["up"][2], arrs["down"][2])


def make_router(cfg: LayerConfig):
    """Router weights [E, d] (bf16 bits, std 1/sqrt(d)) and the optional
    Zipf popularity bias [E] (float32) or None."""
    wr = bf16_bits(_normal((cfg.E, cfg.d), 1.0 / np.sqrt(cfg.d), cfg.seed, "router"))
    bias = None
    if cfg.zipf_s is not None:
        perm = np.random.default_rng(derive_seed(cfg.seed, "zipf-perm")).permutation(cfg.E)
        r = np.arange(1, cfg.E + 1, dtype=np.float64)
        p = r ** (-cfg.zipf_s)
        p /= p.sum()
        pe = np.empty(cfg.E)
        pe[perm] = p
        bias = (0.5 * np.log(cfg.E * pe)).astype(np.float32)
    return wr, bias


def _margins_ok(logits: np.ndarray, k: int, margin: float, ties=None) -> np.ndarray:
    if ties:
        return np.array([_margins_ok_ties(row, k, margin, ties) for row in logits], bool)
    kk = min(k + 1, logits.shape[1])
    top = -np.sort(-logits, axis=1)[:, :kk]
    if kk < 2:
        return np.ones(logits.shape[0], bool)
    return np.all(top[:, :-1] - top[:, 1:] >= margin, axis=1)


def _margins_ok_ties(row: np.ndarray, k: int, margin: float, ties) -> bool:
    """The margin rule with planted tie groups (experts whose logits are equal by
    construction): each group counts as one entry of its size, and the entries that cover
    the first k + 1 experts must be ``margin`` apart."""
    drop = np.zeros(row.size, bool)
    size = np.ones(row.size, np.int64)
    for g in ties:
        g = sorted(int(e) for e in g)
        drop[g[1:]] = True
        size[g[0]] = len(g)
    keep = np.flatnonzero(~drop)
    order = keep[np.argsort(-row[keep], kind="stable")]
    covered, vals = 0, []
    for e in order:
        vals.append(row[e])
        covered += size[e]
        if covered >= k + 1:
            break
    v = np.asarray(vals)
    return bool(np.all(v[:-1] - v[1:] >= margin))


def make_hidden(cfg: LayerConfig, wr_bits: np.ndarray, bias, T: int | None = None,
                stream: str = "x", max_tries: int = 1000, ties=None) -> np.ndarray:
    """Hidden states [T, d] (bf16 bits), N(0,1), every row redrawn (from its own
    stream) until its routing margin holds. ``ties`` lists groups of experts whose logits
    are planted equal (identical router rows and bias); each group counts once."""
    T = cfg.T if T is None else T
    wrf = bf16_bits_to_f32(wr_bits).astype(np.float64)
    b = np.zeros(cfg.E) if bias is None else bias.astype(np.float64)
    out = np.empty((T, cfg.d), np.uint16)
    pending = np.arange(T)
    tries = 0
    while pending.size:
        rows = np.stack([bf16_bits(_normal((cfg.d,), 1.0, cfg.seed, stream, int(t), tries))
                         for t in pending])
        lg = bf16_bits_to_f32(rows).astype(np.float64) @ wrf.T + b
        ok = _margins_ok(lg, cfg.k, cfg.margin, ties)
        out[pending[ok]] = rows[ok]
        pending = pending[~ok]
        tries += 1
        if tries > max_tries:
            raise RuntimeError("routing margin could not be met")
    return out


@dataclass
class LayerInputs:
    cfg: LayerConfig
    x: np.ndarray             # [T, d] bf16 bits
    router_w: np.ndarray      # [E, d] bf16 bits
    router_bias: np.ndarray | None
    routed: Bank
    shared: Bank | None
    extra: dict = field(default_factory=dict)


def plant_ties(wr_bits: np.ndarray, bias, groups, lifts):
    """Router with planted ties: every expert of ``groups[i]`` gets the router row of the
    group's first expert and the bias ``lifts[i]`` (experts outside the groups keep their
    rows and get bias 0, or keep the given bias). Identical rows and bias give logits that
    are equal in any arithmetic that treats the rows alike. Returns (router bits, bias)."""
    wr = wr_bits.copy()
    b = np.zeros(wr.shape[0], np.float32) if bias is None else bias.astype(np.float32).copy()
    for g, lift in zip(groups, lifts):
        g = [int(e) for e in g]
        wr[g] = wr[g[0]]
        b[g] = np.float32(lift)
    return wr, b


def make_layer(cfg: LayerConfig | str, T: int | None = None, routed: Bank | None = None,
               shared: Bank | None = None) -> LayerInputs:
    """All inputs of one layer call. Banks may be passed in to reuse a draw
    (e.g. several token counts over the same weights)."""
    if isinstance(cfg, str):
        cfg = CONFIGS[cfg]
    wr, bias = make_router(cfg)
    x = make_hidden(cfg, wr, bias, T=T)
    if routed is None:
        routed = make_bank(cfg, "routed")
    if shared is None and cfg.n_shared > 0:
        shared = make_bank(cfg, "shared")
    return LayerInputs(cfg, x, wr, bias, routed, shared)
