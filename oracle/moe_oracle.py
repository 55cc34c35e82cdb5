"""fp64 CPU oracle of the expert-routed MoE FFN layer.

TEST INFRASTRUCTURE ONLY. Only the test suite, the smoke check and the CPU
baseline leg of the benchmark may import this module. The CUDA library never
calls it, and it shares no code, tables or helpers with the CUDA library; the
only input it has in common with the library is the seeded synthetic data.

What is computed, step by step (plain, unfused, in float64):

1. Router logits ``l[t, e] = x_t . Wr_e (+ b_e)`` on the bf16 inputs widened
   exactly to float64. The router stays in BF16/F32 (Qwen3.8-Flash-Next-Dual-GPU
   README, "Model artifact and memory placement", quantisation table: router and
   other critical controls are not quantised).
2. A deterministic stable top-k: experts ordered by logit, largest first, ties
   to the lower expert index; the first k are the token's routes
   (same README, "Independent decode lane": the 512-expert router uses a
   deterministic stable top-k). Reading taken: the selection is made on the raw
   logits, and the gate weights are the softmax over the k selected logits, which
   equals the softmax over all experts renormalised over the selected k.
3. The route plan: an expert-major ordering of the (token, slot) assignments,
   counts per expert, their exclusive scan (group offsets) and the inverse map
   (same README, "Dedicated prefill lane", step 1; TandemLLM docs,
   "17 Qwen3.8-Flash-Next", §17.4: a chunk sorts its (row, expert) pairs by
   expert). Within one expert the assignments keep token order.
4. Each expert is a SwiGLU FFN ``y = Wd (silu(Wg x) * (Wu x))`` with
   ``silu(z) = z / (1 + exp(-z))``; quantised weights are dequantised exactly as
   ``W[n, k] = q[n, k] * s[n, k // group]`` (symmetric W4/W8 with groups of 128
   and BF16 group scales: README, "Model artifact and memory placement").
5. The combine: ``out_t = sum_j g[t, j] * y_{t, j} + sum_s y_shared_{s, t}``,
   summed over j in rank order, then the shared experts (README, "Dedicated
   prefill lane", step 5: each token's ten routes reduced in a fixed order; the
   shared expert runs on every token with weight 1: TandemLLM docs Table 17.1,
   "10 routed and 1 shared run a token"; reading taken: no gate on it).

Input encodings (bf16 as uint16 bit patterns; int4 as two's-complement
nibbles, 8 per uint32 along K, element kk at bits 4*(kk % 8) of word kk // 8;
int8 plain) are decoded here from their definition.

Pins (the tests that hold this file to something other than itself) are in
tests/test_oracle_pins.py.
"""
from __future__ import annotations

import numpy as np

__all__ = [
    "widen_bf16", "unpack_int4", "dequantize", "router_logits", "select_topk",
    "route_plan", "silu", "expert_ffn", "layer_forward", "layer_forward_loops",
    "round_to_bf16_f64",
]


# ---------------------------------------------------------------- decoding

def widen_bf16(bits: np.ndarray) -> np.ndarray:
    """bf16 bit patterns (uint16) -> exact float64 values."""
    b = np.asarray(bits).astype(np.uint32) << np.uint32(16)
    return b.view(np.float32).astype(np.float64)


def unpack_int4(words: np.ndarray, K: int) -> np.ndarray:
    """uint32 words [..., K/8] -> int64 values [..., K] in [-8, 7].

    Element kk lives in word kk // 8 at bit offset 4 * (kk % 8); a nibble of 8
    or more is negative (two's complement).
    """
    w = np.asarray(words).astype(np.int64)
    out = np.empty(w.shape[:-1] + (K,), np.int64)
    for i in range(8):
        nib = (w >> (4 * i)) & 0xF
        out[..., i::8] = np.where(nib >= 8, nib - 16, nib)
    return out


def dequantize(wq: np.ndarray, scales: np.ndarray | None, fmt: str, group: int,
               K: int) -> np.ndarray:
    """One expert matrix [N, K] in float64: W = q * s (per group along K)."""
    if fmt == "bf16":
        return widen_bf16(wq)
    if fmt == "int4":
        q = unpack_int4(wq, K).astype(np.float64)
    elif fmt == "int8":
        q = np.asarray(wq).astype(np.float64)
    else:
        raise ValueError(fmt)
    s = widen_bf16(scales)                       # [N, K // group]
    return q * np.repeat(s, group, axis=1)


# ---------------------------------------------------------------- routing

def router_logits(x_bits, wr_bits, bias=None) -> np.ndarray:
    """l = X Wr^T (+ b), float64 [T, E]."""
    l = widen_bf16(x_bits) @ widen_bf16(wr_bits).T
    if bias is not None:
        l = l + np.asarray(bias).astype(np.float64)[None, :]
    return l


def select_topk(logits: np.ndarray, k: int):
    """Per token: the k experts with the largest logits (ties: lower index
    first), in that rank order, and their gate weights (softmax over the k
    selected logits)."""
    T, E = logits.shape
    idx = np.empty((T, k), np.int64)
    gates = np.empty((T, k), np.float64)
    for t in range(T):
        order = sorted(range(E), key=lambda e: (-logits[t, e], e))
        sel = order[:k]
        idx[t] = sel
        ls = logits[t, sel]
        z = np.exp(ls - ls.max())
        gates[t] = z / z.sum()
    return idx, gates


def route_plan(idx: np.ndarray, E: int):
    """Expert-major plan of the T*k assignments a = t*k + j.

    Returns counts [E], offsets [E+1] (exclusive scan of counts), perm [T*k]
    (perm[r] = assignment at grouped row r; experts ascending, then tokens
    ascending) and inv [T*k] (inv[a] = grouped row of assignment a).
    """
    T, k = idx.shape
    counts = np.zeros(E, np.int64)
    for e in idx.ravel():
        counts[e] += 1
    offsets = np.zeros(E + 1, np.int64)
    for e in range(E):
        offsets[e + 1] = offsets[e] + counts[e]
    fill = offsets[:-1].copy()
    perm = np.empty(T * k, np.int64)
    inv = np.empty(T * k, np.int64)
    for t in range(T):                    # token order => stable within an expert
        for j in range(k):
            e = idx[t, j]
            r = fill[e]
            fill[e] += 1
            perm[r] = t * k + j
            inv[t * k + j] = r
    return counts, offsets, perm, inv


# ---------------------------------------------------------------- experts

def silu(z: np.ndarray) -> np.ndarray:
    with np.errstate(over="ignore"):
        return z / (1.0 + np.exp(-z))


def expert_ffn(x: np.ndarray, Wg: np.ndarray, Wu: np.ndarray, Wd: np.ndarray) -> np.ndarray:
    """SwiGLU expert on rows x [R, d] (float64): Wd (silu(Wg x) * (Wu x))."""
    h = silu(x @ Wg.T) * (x @ Wu.T)
    return h @ Wd.T


def _bank_expert(bank: dict, e: int, d: int, f: int):
    fmt, g = bank["fmt"], bank["group"]
    Wg = dequantize(bank["w_gate"][e], None if bank["s_gate"] is None else bank["s_gate"][e], fmt, g, d)
    Wu = dequantize(bank["w_up"][e], None if bank["s_up"] is None else bank["s_up"][e], fmt, g, d)
    Wd = dequantize(bank["w_down"][e], None if bank["s_down"] is None else bank["s_down"][e], fmt, g, f)
    return Wg, Wu, Wd


# ---------------------------------------------------------------- layer

def layer_forward(x_bits, router_w, router_bias, routed: dict, shared: dict | None,
                  k: int, tokens=None, routed_scale: float = 1.0):
    """The whole layer in float64.

    ``routed`` / ``shared`` are dicts with keys fmt, group, w_gate, w_up,
    w_down, s_gate, s_up, s_down (expert-major arrays as encoded by the input
    generator). ``tokens`` optionally restricts which output rows are computed
    (routing and the plan always cover all tokens). ``routed_scale`` multiplies
    every gate weight (1 in the layer; other values only serve invariance tests).

    Returns a dict with logits, idx, gates, counts, offsets, perm, inv, out
    (float64 [len(tokens), d]) and tokens.
    """
    xf = widen_bf16(x_bits)
    T, d = xf.shape
    E = router_w.shape[0]
    logits = router_logits(x_bits, router_w, router_bias)
    idx, gates = select_topk(logits, k)
    counts, offsets, perm, inv = route_plan(idx, E)
    tokens = np.arange(T) if tokens is None else np.asarray(tokens)
    pos = {int(t): i for i, t in enumerate(tokens)}
    f = routed["w_gate"].shape[1]
    out = np.zeros((len(tokens), d), np.float64)
    # y for every needed (token, slot), expert by expert (each expert dequantised once)
    y_routed = np.zeros((len(tokens), k, d), np.float64)
    needed = {}
    for t in tokens:
        for j in range(k):
            needed.setdefault(int(idx[t, j]), []).append((int(t), j))
    for e in sorted(needed):
        Wg, Wu, Wd = _bank_expert(routed, e, d, f)
        rows = needed[e]
        xs = xf[[t for t, _ in rows]]
        ys = expert_ffn(xs, Wg, Wu, Wd)
        for (t, j), y in zip(rows, ys):
            y_routed[pos[t], j] = y
    for i, t in enumerate(tokens):
        acc = np.zeros(d, np.float64)
        for j in range(k):
            acc = acc + (routed_scale * gates[t, j]) * y_routed[i, j]
        out[i] = acc
    if shared is not None:
        for s in range(shared["w_gate"].shape[0]):
            Wg, Wu, Wd = _bank_expert(shared, s, d, f)
            out += expert_ffn(xf[tokens], Wg, Wu, Wd)
    return dict(logits=logits, idx=idx, gates=gates, counts=counts, offsets=offsets,
                perm=perm, inv=inv, out=out, tokens=tokens)


def layer_forward_loops(x_bits, router_w, router_bias, routed: dict, shared: dict | None,
                        k: int, tokens=None) -> np.ndarray:
    """The same layer with scalar Python loops, token by token, for tiny shapes
    only (no matrix routines, no vectorised softmax or top-k). Returns the
    float64 output rows of ``tokens`` (default: all)."""
    import math
    xf = widen_bf16(x_bits)
    T, d = xf.shape
    E = router_w.shape[0]
    wr = widen_bf16(router_w)
    b = None if router_bias is None else np.asarray(router_bias).astype(np.float64)
    f = routed["w_gate"].shape[1]
    cache = {}

    def W(bank, tag, e):
        key = (id(bank), e)
        if key not in cache:
            cache[key] = _bank_expert(bank, e, d, f)
        return cache[key]

    def ffn(Wg, Wu, Wd, x):
        h = [0.0] * f
        for n in range(f):
            g = 0.0
            u = 0.0
            for c in range(d):
                g += Wg[n, c] * x[c]
                u += Wu[n, c] * x[c]
            h[n] = (g / (1.0 + math.exp(-g)) if g > -700 else 0.0) * u
        y = [0.0] * d
        for n in range(d):
            acc = 0.0
            for c in range(f):
                acc += Wd[n, c] * h[c]
            y[n] = acc
        return y

    tokens = range(T) if tokens is None else tokens
    out = np.zeros((len(tokens), d))
    for i, t in enumerate(tokens):
        x = xf[t]
        l = []
        for e in range(E):
            acc = 0.0
            for c in range(d):
                acc += x[c] * wr[e, c]
            if b is not None:
                acc += b[e]
            l.append(acc)
        chosen = []
        for _ in range(k):                     # k rounds of "largest, lowest index"
            best = None
            for e in range(E):
                if e in chosen:
                    continue
                if best is None or l[e] > l[best]:
                    best = e
            chosen.append(best)
        m = max(l[e] for e in chosen)
        z = [math.exp(l[e] - m) for e in chosen]
        zs = sum(z)
        acc = [0.0] * d
        for j, e in enumerate(chosen):
            y = ffn(*W(routed, "r", e), x)
            for n in range(d):
                acc[n] += (z[j] / zs) * y[n]
        if shared is not None:
            for s in range(shared["w_gate"].shape[0]):
                y = ffn(*W(shared, "s", s), x)
                for n in range(d):
                    acc[n] += y[n]
        out[i] = acc
    return out


def round_to_bf16_f64(a: np.ndarray) -> np.ndarray:
    """float64 -> nearest bf16 value (ties to even), returned as float64.

    Two-step rounding through float32 can double-round; this rounds once, from
    the float64 value, by locating the two neighbouring bf16 values.
    """
    a = np.asarray(a, np.float64)
    m, ex = np.frexp(a)                      # a = m * 2**ex, 0.5 <= |m| < 1
    scaled = np.ldexp(m, 8)                  # 8 significant bits for bf16
    r = np.round(scaled)                     # numpy round: half to even
    return np.ldexp(r, ex - 8)
