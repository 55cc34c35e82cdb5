"""fp64 CPU oracle of the NVFP4 (W4A4) variant of the expert-routed MoE FFN layer.

TEST INFRASTRUCTURE ONLY. Only the test suite may import this module. The CUDA library never
calls it and shares no code, tables or helpers with it; the only input in common is the seeded
synthetic data (the weight codes are written once by the input generator).

The variant (Anvil serving benchmarks, "Qwen3.8 Flash Next", section "Quantization
boundary"): ModelOpt NVFP4 W4A4 on the routed experts, i.e. both their weights and the
activations entering them are 4-bit floating point; the shared expert (and the router) stay
BF16. Routing, the route plan and the combine are those of the BF16/int layer
(``moe_oracle``).

NVFP4, as NVIDIA defines it (the pages name the format but do not spell it out):
  - element E2M1: 4 bits, sign (bit 3), exponent (bits 2..1, bias 1), mantissa (bit 0);
    exponent 0 is subnormal (value = mantissa / 2), otherwise 2^(e-1) * (1 + m / 2);
    magnitudes 0, 0.5, 1, 1.5, 2, 3, 4, 6; no infinity or NaN.
  - a block of 16 consecutive elements along K shares one E4M3 scale: 8 bits, sign,
    exponent (4 bits, bias 7), mantissa (3 bits); exponent 0 is subnormal
    (m / 8 * 2^-6); the code with all exponent and mantissa bits set is NaN; largest 448.
  - one float32 scale per tensor. value = e2m1 * e4m3 * scale.

Readings taken where neither the pages nor the format fix a step:
  N1  weights: encoded once by the generator, block scale = E4M3(amax_block / (6 g)) with
      g = amax(matrix) / (6 * 448), element = E2M1(w / (block scale * g)), both rounded to
      nearest even, elements saturating at 6 (the usual NVFP4 recipe).
  N2  activations: quantised at run time per token row (x for gate/up, h for down) with the
      same recipe and the row's own tensor scale g = amax(row) / (6 * 448), so that a row's
      result depends on that row alone; ModelOpt's calibrated static activation scales need
      data the pages do not give.
  N3  the decisions of N2 are taken in float32, the precision a kernel takes them in: every
      scale and quotient is an IEEE float32 operation (``float32`` numpy arithmetic), the
      comparisons with the rounding boundaries are exact.
  N4  products and sums are exact here (float64 over exactly decoded values); h =
      silu(gate) * up is formed in float64 and rounded to float32 before it is quantised.
"""
from __future__ import annotations

import numpy as np

from oracle import moe_oracle as M

__all__ = ["e2m1_value", "e4m3_value", "round_e2m1", "round_e4m3", "unpack_fp4",
           "nvfp4_quantize_rows", "nvfp4_dequantize", "expert_ffn_w4a4", "layer_forward_nvfp4"]

BLOCK = 16
AMAX_E2M1 = 6.0
AMAX_E4M3 = 448.0


# ---------------------------------------------------------------- decoding (format definition)

def e2m1_value(code: np.ndarray) -> np.ndarray:
    """E2M1 codes (low 4 bits) -> float64 values."""
    c = np.asarray(code).astype(np.int64) & 0xF
    sign = np.where(c & 0x8, -1.0, 1.0)
    e = (c >> 1) & 0x3
    m = c & 0x1
    mag = np.where(e == 0, m * 0.5, np.ldexp(1.0 + m / 2.0, e - 1))
    return sign * mag


def e4m3_value(code: np.ndarray) -> np.ndarray:
    """E4M3 (fn) codes -> float64 values; the NaN codes (0x7F, 0xFF) give NaN."""
    c = np.asarray(code).astype(np.int64) & 0xFF
    sign = np.where(c & 0x80, -1.0, 1.0)
    e = (c >> 3) & 0xF
    m = c & 0x7
    mag = np.where(e == 0, np.ldexp(m / 8.0, -6), np.ldexp(1.0 + m / 8.0, e - 7))
    mag = np.where((c & 0x7F) == 0x7F, np.nan, mag)
    return sign * mag


def unpack_fp4(packed: np.ndarray, K: int) -> np.ndarray:
    """uint8 bytes [..., K/2] -> E2M1 codes [..., K]; element k is the nibble at bit
    4 * (k % 2) of byte k // 2."""
    b = np.asarray(packed).astype(np.int64)
    out = np.empty(b.shape[:-1] + (K,), np.int64)
    out[..., 0::2] = b & 0xF
    out[..., 1::2] = (b >> 4) & 0xF
    return out


# ---------------------------------------------------------------- rounding (nearest, ties even)

def _nearest_code(a: np.ndarray, codes: np.ndarray, values: np.ndarray) -> np.ndarray:
    """Nearest of the ascending non-negative ``values`` (with their ``codes``) to each
    non-negative a; on a tie the code with the even low bit (the even mantissa)."""
    a = np.asarray(a, np.float64)
    i = np.clip(np.searchsorted(values, a, side="left"), 1, len(values) - 1)
    lo, hi = values[i - 1], values[i]
    pick_hi = (a - lo > hi - a) | ((a - lo == hi - a) & (codes[i] % 2 == 0))
    j = np.where(pick_hi, i, i - 1)
    j = np.where(a <= values[0], 0, j)
    j = np.where(a >= values[-1], len(values) - 1, j)
    return codes[j]


_E2M1_CODES = np.arange(8)
_E2M1_VALUES = e2m1_value(_E2M1_CODES)
_E4M3_CODES = np.arange(0x7F)  # non-negative finite codes, ascending values
_E4M3_VALUES = e4m3_value(_E4M3_CODES)


def round_e2m1(v: np.ndarray) -> np.ndarray:
    """Values -> E2M1 codes: nearest, ties to even, magnitudes above 6 saturate to 6."""
    v = np.asarray(v, np.float64)
    c = _nearest_code(np.abs(v), _E2M1_CODES, _E2M1_VALUES)
    return (c | np.where(np.signbit(v), 8, 0)).astype(np.int64)


def round_e4m3(v: np.ndarray) -> np.ndarray:
    """Non-negative values -> E4M3 codes: nearest, ties to even, saturating at 448."""
    return _nearest_code(np.asarray(v, np.float64), _E4M3_CODES, _E4M3_VALUES).astype(np.int64)


# ---------------------------------------------------------------- NVFP4 of activation rows

def nvfp4_quantize_rows(v32: np.ndarray):
    """float32 rows [R, K] -> (E2M1 codes [R, K], E4M3 block-scale codes [R, K/16], float32
    row scales [R]) by readings N2 and N3: g = amax(row) / (6 * 448); block scale =
    E4M3(amax_block / (6 g)); element = E2M1(v / (block scale * g)); every operation in float32;
    a zero scale gives zero elements."""
    v32 = np.asarray(v32, np.float32)
    R, K = v32.shape
    assert K % BLOCK == 0
    g = (np.abs(v32).max(axis=1) / np.float32(AMAX_E2M1 * AMAX_E4M3)).astype(np.float32)
    vb = v32.reshape(R, K // BLOCK, BLOCK)
    amax_b = np.abs(vb).max(axis=2)
    denom = (np.float32(AMAX_E2M1) * g).astype(np.float32)[:, None]
    with np.errstate(divide="ignore", invalid="ignore"):
        ratio = np.where(denom > 0, amax_b / np.where(denom > 0, denom, np.float32(1)), 0)
    ratio = ratio.astype(np.float32)
    sc = round_e4m3(ratio)
    scale = (e4m3_value(sc).astype(np.float32) * g[:, None]).astype(np.float32)
    safe = np.where(scale > 0, scale, np.float32(1))
    q = (vb / safe[..., None]).astype(np.float32)
    codes = round_e2m1(q)
    codes = np.where((scale > 0)[..., None], codes, 0).reshape(R, K)
    return codes, sc, g


# every code's value, from the definitions above (a table lookup decodes whole matrices fast)
_E2M1_TABLE = e2m1_value(np.arange(16))
_E4M3_TABLE = e4m3_value(np.arange(256))


def nvfp4_dequantize(codes: np.ndarray, scale_codes: np.ndarray, g: np.ndarray) -> np.ndarray:
    """E2M1 codes [..., K], E4M3 block-scale codes [..., K/16], float32 tensor scale(s)
    (broadcast over the leading axes) -> float64 values (exact)."""
    v = _E2M1_TABLE[np.asarray(codes).astype(np.int64) & 0xF]
    s = np.repeat(_E4M3_TABLE[np.asarray(scale_codes).astype(np.int64) & 0xFF], BLOCK, axis=-1)
    return v * s * np.asarray(g, np.float64)[..., None]


# ---------------------------------------------------------------- the W4A4 expert and the layer

def _weights(bank: dict, e: int, d: int, f: int):
    out = []
    for name, K in (("gate", d), ("up", d), ("down", f)):
        codes = unpack_fp4(bank["w_" + name][e], K)
        out.append(nvfp4_dequantize(codes, bank["s_" + name][e],
                                    np.float64(np.float32(bank["g_" + name][e]))))
    return out


def expert_ffn_w4a4(x32: np.ndarray, Wg: np.ndarray, Wu: np.ndarray, Wd: np.ndarray):
    """One routed expert on float32 rows [R, d]: the rows quantised to NVFP4, then
    h = silu(Wg x) * (Wu x) exactly, rounded to float32 and quantised to NVFP4 (N4), then
    y = Wd h exactly. Returns float64 [R, d_out]."""
    cx, sx, gx = nvfp4_quantize_rows(x32)
    xq = nvfp4_dequantize(cx, sx, gx)
    h = M.silu(xq @ Wg.T) * (xq @ Wu.T)
    ch, sh, gh = nvfp4_quantize_rows(h.astype(np.float32))
    hq = nvfp4_dequantize(ch, sh, gh)
    return hq @ Wd.T


def layer_forward_nvfp4(x_bits, router_w, router_bias, routed: dict, shared: dict | None,
                        k: int, tokens=None) -> dict:
    """The layer with NVFP4 W4A4 routed experts (``routed``: dict with fmt "nvfp4", packed
    E2M1 codes w_*, E4M3 block scales s_*, float32 tensor scales g_* per expert) and an
    optional BF16/int shared expert (``shared``: a bank dict of ``moe_oracle``). ``tokens``
    optionally restricts which output rows are computed (routing and the plan always cover
    all tokens; a row's result depends on that row alone). Returns the same fields as
    ``moe_oracle.layer_forward`` (``out``: float64 [len(tokens), d])."""
    assert routed["fmt"] == "nvfp4"
    x = M.widen_bf16(x_bits)                      # bf16 values, exact in float32
    T, d = x.shape
    E = routed["w_gate"].shape[0]
    f = routed["w_gate"].shape[1]
    logits = M.router_logits(x_bits, router_w, router_bias)
    idx, gates = M.select_topk(logits, k)
    counts, offsets, perm, inv = M.route_plan(idx, E)
    x32 = x.astype(np.float32)
    tokens = np.arange(T) if tokens is None else np.asarray(tokens)
    pos = {int(t): i for i, t in enumerate(tokens)}
    # y for every needed (token, slot), expert by expert (each expert decoded once); a row is
    # quantised on its own (N2), so grouping rows does not change any row's result
    y = np.zeros((len(tokens), k, d), np.float64)
    needed = {}
    for t in tokens:
        for j in range(k):
            needed.setdefault(int(idx[t, j]), []).append((int(t), j))
    for e in sorted(needed):
        Wg, Wu, Wd = _weights(routed, e, d, f)
        rows = needed[e]
        ys = expert_ffn_w4a4(x32[[t for t, _ in rows]], Wg, Wu, Wd)
        for (t, j), yy in zip(rows, ys):
            y[pos[t], j] = yy
    out = np.zeros((len(tokens), d), np.float64)
    for i in range(len(tokens)):
        acc = np.zeros(d, np.float64)
        for j in range(k):                        # rank order, then the shared expert
            acc = acc + gates[tokens[i], j] * y[i, j]
        out[i] = acc
    if shared is not None:
        for s in range(shared["w_gate"].shape[0]):
            Wg, Wu, Wd = M._bank_expert(shared, s, d, f)
            out += M.expert_ffn(x[tokens], Wg, Wu, Wd)
    return dict(logits=logits, idx=idx, gates=gates, counts=counts, offsets=offsets,
                perm=perm, inv=inv, out=out)
