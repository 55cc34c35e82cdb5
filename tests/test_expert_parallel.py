"""Expert parallelism (the routed experts split across ranks, one exchange each way) on CPU
ranks over gloo: the exchange plumbing, the owner ranges and the fixed-order combine.

Each rank's arithmetic is given by the fp64 oracle here (``OracleOps``); on GPUs the same
layer runs the library's stage entry points (``LibraryOps``; tests/test_gpu_expert_parallel.py
runs two such ranks sharing one device). The expert-parallel result on every rank equals the
single-process oracle layer on that rank's tokens (up to the fp64 matrix routine's order), for
2 and 4 ranks, with uneven token counts per rank, and is the same bits when repeated."""
import os
import socket

import numpy as np
import pytest
import torch

from oracle import moe_oracle as O
from expert_routed_ffn_route_b200 import synth
from expert_routed_ffn_route_b200.expert_parallel import (ExpertParallelLayer, local_expert_ids,
                                                          owner_counts)
from conftest import bank_dict


def test_owner_ranges():
    offsets = np.array([0, 2, 2, 5, 9, 9, 10, 12, 12])  # 8 experts
    assert owner_counts(offsets, 2).tolist() == [9, 3]
    assert owner_counts(offsets, 4).tolist() == [2, 7, 1, 2]
    assert local_expert_ids(offsets, 2).tolist() == [0, 0, 2, 2, 2, 3, 3, 3, 3, 1, 2, 2]
    assert local_expert_ids(offsets, 4).tolist() == [0, 0, 0, 0, 0, 1, 1, 1, 1, 1, 0, 0]


CFG = synth.LayerConfig("ep", T=8, d=128, E=8, k=2, f=128, n_shared=1, fmt="int4", seed=41)


def _slice_bank(bank: dict, e0: int, e1: int) -> dict:
    out = dict(bank)
    for key in ("w_gate", "w_up", "w_down", "s_gate", "s_up", "s_down"):
        if out.get(key) is not None:
            out[key] = out[key][e0:e1]
    return out


class OracleOps:
    """Per-rank arithmetic in fp64 (test stand-in for the library's stage entry points)."""

    def __init__(self, L, local: dict, e0: int):
        self.L, self.local, self.e0 = L, local, e0
        self.wr = O.widen_bf16(L.router_w)

    def route(self, x):
        lg = x.numpy() @ self.wr.T
        if self.L.router_bias is not None:
            lg = lg + self.L.router_bias.astype(np.float64)[None, :]
        idx, gates = O.select_topk(lg, CFG.k)
        return torch.from_numpy(idx.astype(np.int32)), torch.from_numpy(gates)

    def permute(self, idx):
        _, offsets, perm, inv = O.route_plan(idx.numpy().astype(np.int64), CFG.E)
        return (torch.from_numpy(offsets.astype(np.int32)), torch.from_numpy(perm.astype(np.int32)),
                torch.from_numpy(inv.astype(np.int32)))

    def gather(self, x, rows):
        return x.index_select(0, rows)

    def local_ffn(self, x_rows, ids):
        y = np.zeros((x_rows.shape[0], CFG.d))
        ids = ids.numpy()
        for e in np.unique(ids):
            rows = np.nonzero(ids == e)[0]
            W = O._bank_expert(self.local, int(e), CFG.d, CFG.f)
            y[rows] = O.expert_ffn(x_rows.numpy()[rows], *W)
        return torch.from_numpy(y)

    def shared_ffn(self, x):
        W = O._bank_expert(bank_dict(self.L.shared), 0, CFG.d, CFG.f)
        return torch.from_numpy(O.expert_ffn(x.numpy(), *W))

    def combine(self, y_assign, y_shared, inv, gates):
        T = gates.shape[0]
        y, inv, g = y_assign.numpy(), inv.numpy(), gates.numpy()
        out = np.zeros((T, CFG.d))
        for t in range(T):
            acc = np.zeros(CFG.d)
            for j in range(CFG.k):  # rank order, then the shared expert
                acc = acc + g[t, j] * y[inv[t * CFG.k + j]]
            out[t] = acc
        return torch.from_numpy(out + y_shared.numpy())


def _rank_main(rank, world, port, tokens_per_rank):
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        L = synth.make_layer(CFG)  # the same seeded weights on every rank
        full = bank_dict(L.routed)
        E_loc = CFG.E // world
        local = _slice_bank(full, rank * E_loc, (rank + 1) * E_loc)
        x_bits = synth.make_hidden(CFG, L.router_w, L.router_bias, T=tokens_per_rank[rank],
                                   stream=f"ep-rank{rank}")
        x = torch.from_numpy(O.widen_bf16(x_bits))
        layer = ExpertParallelLayer(OracleOps(L, local, rank * E_loc), CFG.k, CFG.E, rank, world,
                                    dist)
        out = layer.forward(x).numpy()
        again = layer.forward(x).numpy()
        assert np.array_equal(out, again), "not deterministic"
        ref = O.layer_forward(x_bits, L.router_w, L.router_bias, full, bank_dict(L.shared),
                              CFG.k)["out"]
        np.testing.assert_allclose(out, ref, rtol=1e-12, atol=1e-14)
    finally:
        dist.destroy_process_group()


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


@pytest.mark.parametrize("world,tokens", [(2, (5, 9)), (4, (1, 7, 3, 6))])
def test_expert_parallel_matches_single_process(world, tokens):
    import torch.multiprocessing as mp
    mp.spawn(_rank_main, args=(world, _free_port(), tokens), nprocs=world, join=True)
