"""The tie rule of the stable top-k on the GPU: equal logits go to the lower expert index
(Qwen3.8-Flash-Next-Dual-GPU README, "Independent decode lane": a deterministic stable
top-k over the 512 experts).

Ties are planted, not hoped for: every expert of a group gets the same router row and the
same bias, so their fp32 logits are equal in any kernel that treats the rows alike, and
the oracle (fp64) sees them equal too. The bias lifts a group above the other experts for
every token. Three placements:

  inside    a group of 3 at the top: ranks 0..2 in index order, the rest of the picks
            come from ordinary experts;
  straddle  a group of 8 at the top, then a group of 4 across ranks k-1 / k: only its
            two lowest indices are picked;
  many      64 equal logits spread over 8 chunks of 32 experts (8 in each): the picks are
            the 10 lowest indices; in the single-kernel layer more than 32 candidates
            survive its pruning, which takes the table-scan branch of its merge.

Each placement runs through every top-k implementation: the single-kernel 1-token layer,
the fused routing kernel (calls of up to 32 tokens) and the tensor-core router with the
per-token top-k kernel (larger calls). Indices and the plan are compared bit for bit with
the oracle, gates within 1e-5, the output within the layer tolerance.
"""
import numpy as np
import pytest

from oracle import moe_oracle as O
from expert_routed_ffn_route_b200 import synth
from gpu_helpers import check_layer

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

CFG = synth.LayerConfig("ties", T=1, d=512, E=512, k=10, f=256, n_shared=1, fmt="int4",
                        seed=41)

PATTERNS = {
    "inside": ([[3, 17, 40]], [20.0]),
    "straddle": ([[100, 2, 50, 400, 7, 250, 33, 499], [301, 9, 300, 5]], [20.0, 10.0]),
    "many": ([[32 * c + 4 * i for c in range(8) for i in range(8)]], [20.0]),
}


@pytest.fixture(scope="module")
def B():
    from expert_routed_ffn_route_b200 import binding
    if not torch.cuda.is_available():
        pytest.skip("no GPU")
    binding.load_library()
    return binding


@pytest.fixture(scope="module")
def banks():
    return synth.make_bank(CFG, "routed"), synth.make_bank(CFG, "shared")


def tie_layer(banks, pattern, T):
    groups, lifts = PATTERNS[pattern]
    wr0, _ = synth.make_router(CFG)
    wr, bias = synth.plant_ties(wr0, None, groups, lifts)
    x = synth.make_hidden(CFG, wr, bias, T=T, stream=f"ties-{pattern}-{T}", ties=groups)
    cfg = synth.LayerConfig(CFG.name, T=T, d=CFG.d, E=CFG.E, k=CFG.k, f=CFG.f,
                            n_shared=CFG.n_shared, fmt=CFG.fmt, seed=CFG.seed)
    return synth.LayerInputs(cfg, x, wr, bias, banks[0], banks[1]), groups


def expected_picks(groups, idx_row, k):
    """What the tie rule fixes about one token's picks, from the planted groups alone."""
    top = sorted(groups[0])
    if len(groups) == 1 and len(top) >= k:
        return top[:k]
    if len(groups) == 2:
        return top + sorted(groups[1])[:k - len(top)]
    return top + list(idx_row[len(top):])


@pytest.mark.parametrize("pattern", list(PATTERNS))
@pytest.mark.parametrize("T,path", [(1, "fused"), (1, "gemv"), (16, "auto"), (40, "auto")])
def test_tie_rule_on_gpu(B, banks, pattern, T, path):
    L, groups = tie_layer(banks, pattern, T)
    dl = B.DeviceLayer(L)
    desc = dl.descriptor(T, path)
    if path == "fused":
        assert B.launches_per_call(desc) == 1, "single-kernel layer not taken"
    # the oracle's own picks follow the rule (a check of the planted inputs, in fp64)
    ref_idx, _ = O.select_topk(O.router_logits(L.x, L.router_w, L.router_bias), CFG.k)
    for t in range(T):
        assert list(ref_idx[t]) == expected_picks(groups, ref_idx[t], CFG.k)
    check_layer(B, dl, L, L.x, path, check_stages=(T <= 16))
