"""The expert-parallel layer on the library's kernels (``LibraryOps``), two ranks on one GPU.

The two ranks are host threads that share the device; their exchanges go through a host-side
stand-in for ``all_to_all_single`` (no kernel of one rank ever waits on the other, so running
them on one GPU is sound). Each rank owns half of the experts; its output meets the fp64
oracle of the whole layer on its own tokens within the layer bound."""
import threading

import numpy as np
import pytest

from oracle import moe_oracle as O
from expert_routed_ffn_route_b200 import synth
from conftest import out_tol, output_excess
from gpu_helpers import bf16_to_np, to_dev_x

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu


class ThreadExchange:
    """all_to_all_single between threads of one process (equal splits when none given)."""

    def __init__(self, world):
        self.world = world
        self.slots = [[None] * world for _ in range(world)]
        self.barrier = threading.Barrier(world)
        self.rank_of = {}

    def all_to_all_single(self, out, inp, output_split_sizes=None, input_split_sizes=None,
                          group=None):
        me = self.rank_of[threading.get_ident()]
        n = inp.shape[0]
        sizes = input_split_sizes or [n // self.world] * self.world
        parts = torch.split(inp, sizes)
        for dst in range(self.world):
            self.slots[me][dst] = parts[dst].clone()
        torch.cuda.synchronize()
        self.barrier.wait()
        got = [self.slots[src][me] for src in range(self.world)]
        if sum(g.shape[0] for g in got):
            out.copy_(torch.cat(got))
        torch.cuda.synchronize()
        self.barrier.wait()


def test_two_ranks_on_the_library_kernels():
    from expert_routed_ffn_route_b200 import binding as B
    from expert_routed_ffn_route_b200.expert_parallel import ExpertParallelLayer, LibraryOps
    if not torch.cuda.is_available():
        pytest.skip("no GPU")
    B.load_library()
    world = 2
    cfg = synth.LayerConfig("ep-gpu", T=24, d=512, E=16, k=4, f=256, fmt="int4", seed=43)
    L = synth.make_layer(cfg)
    dl = B.DeviceLayer(L)
    full = dl.banks["routed"]
    E_loc = cfg.E // world
    xs = [synth.make_hidden(cfg, L.router_w, L.router_bias, T=T, stream=f"epg{r}")
          for r, T in enumerate((24, 9))]
    ex = ThreadExchange(world)
    outs, errors = [None] * world, []

    def rank_main(r):
        try:
            torch.cuda.set_device(0)
            ex.rank_of[threading.get_ident()] = r
            local = dict(full, n_exp=E_loc)
            for key in ("w_gate", "w_up", "w_down", "s_gate", "s_up", "s_down"):
                local[key] = full[key][r * E_loc:(r + 1) * E_loc]
            ops = LibraryOps(cfg, dl.router_w, dl.router_bias, local, dl.banks["shared"], world)
            layer = ExpertParallelLayer(ops, cfg.k, cfg.E, r, world, ex)
            outs[r] = layer.forward(to_dev_x(xs[r]))
            torch.cuda.synchronize()
        except Exception as e:  # surfaced below
            errors.append(e)
            ex.barrier.abort()

    threads = [threading.Thread(target=rank_main, args=(r,)) for r in range(world)]
    for t in threads:
        t.start()
    for t in threads:
        t.join(timeout=300)
    assert not errors, errors
    for r in range(world):
        ref = O.layer_forward(xs[r], L.router_w, L.router_bias,
                              {**L.routed.arrays(), "fmt": L.routed.fmt, "group": L.routed.group},
                              {**L.shared.arrays(), "fmt": L.shared.fmt, "group": L.shared.group},
                              cfg.k)["out"]
        got = O.widen_bf16(bf16_to_np(outs[r]))
        err = float(output_excess(got, ref).max())
        print(f"[ep rank {r}] max excess {err:.3e}, bound {out_tol(ref):.3e}")
        assert err <= out_tol(ref)
