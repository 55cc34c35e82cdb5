"""Expert parallelism: the layer's routed experts split across the ranks of a process group
(one process per GPU), with one exchange each way.

Every rank holds the router and the shared expert (replicated) and a contiguous range of
E / W routed experts (rank r owns global experts [r * E/W, (r + 1) * E/W)). A call on rank r
takes that rank's own tokens and:

  1. routes them with the full router (``moe_route``) and builds the expert-major plan over
     all E experts (``moe_permute``); in that grouped order the rows bound for each owner are
     one contiguous block, in owner order;
  2. sends every grouped row (its token's hidden state and the expert's local index) to the
     expert's owner (``all_to_all_single``: the first exchange);
  3. on each owner: the received rows, grouped by its local experts, go through the grouped
     FFN (``moe_permute`` + ``moe_grouped_ffn`` of a layer over the owner's experts with one
     assignment a row), one fp32 row per assignment;
  4. sends each row back to the rank it came from (the second exchange), where it lands in
     the grouped row of its assignment;
  5. combines on the home rank with ``moe_combine``: the token's k routes in rank order, then
     the shared expert (computed on the home rank), summed in fp32 and rounded once.

The combine of step 5 is the only reduction across ranks' results, and it runs in the fixed
order of the single-GPU layer, so the result is deterministic whatever the number of ranks
(TandemLLM docs v0.8.3, "33 Roadmap", §33.5: a fixed reduction order across devices;
Qwen3.8-Flash-Next-Dual-GPU README, "Dedicated prefill lane", step 5: a fixed-order
reduction of each token's routes without atomics).

The exchanges are collectives of ``torch.distributed`` (NCCL on GPUs); the arithmetic runs in
the library's kernels through ``ops`` (the C-ABI stage entry points by default). Row gathers
that arrange the exchanged rows are tensor indexing.
"""
from __future__ import annotations

import numpy as np


def owner_counts(offsets_host: np.ndarray, world: int) -> np.ndarray:
    """Grouped rows bound for each owner: owner o holds experts [o E/W, (o+1) E/W), whose rows
    are [offsets[o E/W], offsets[(o+1) E/W]) of the expert-major order."""
    E = len(offsets_host) - 1
    assert E % world == 0, "the experts split evenly across the ranks"
    bounds = np.asarray(offsets_host, np.int64)[:: E // world]
    return np.diff(bounds)


def local_expert_ids(offsets_host: np.ndarray, world: int) -> np.ndarray:
    """For every grouped row, its expert's index within the owner's range."""
    E = len(offsets_host) - 1
    counts = np.diff(np.asarray(offsets_host, np.int64))
    experts = np.repeat(np.arange(E, dtype=np.int64), counts)
    return (experts % (E // world)).astype(np.int32)


class ExpertParallelLayer:
    """One MoE layer whose routed experts are spread over ``world`` ranks.

    ``ops`` provides the per-rank arithmetic (see ``LibraryOps``); ``dist`` is
    ``torch.distributed`` (or anything with ``all_to_all_single`` and the same meaning), and
    ``group`` its process group.
    """

    def __init__(self, ops, k: int, E: int, rank: int, world: int, dist, group=None):
        assert E % world == 0
        self.ops, self.k, self.E = ops, k, E
        self.rank, self.world = rank, world
        self.dist, self.group = dist, group

    def _exchange(self, send, send_counts, recv_counts):
        import torch
        out = torch.empty((int(sum(recv_counts)),) + tuple(send.shape[1:]), dtype=send.dtype,
                          device=send.device)
        self.dist.all_to_all_single(out, send.contiguous(),
                                    output_split_sizes=[int(c) for c in recv_counts],
                                    input_split_sizes=[int(c) for c in send_counts],
                                    group=self.group)
        return out

    def forward(self, x):
        import torch
        ops, k = self.ops, self.k
        idx, gates = ops.route(x)
        offsets, perm, inv = ops.permute(idx)
        offsets_host = offsets.cpu().numpy()
        send_counts = owner_counts(offsets_host, self.world)
        counts_t = torch.as_tensor(send_counts, dtype=torch.int64, device=x.device)
        recv_t = torch.empty_like(counts_t)
        self.dist.all_to_all_single(recv_t, counts_t, group=self.group)
        recv_counts = recv_t.cpu().numpy()

        # rows in grouped (expert-major) order: owner blocks are contiguous
        tok = perm.long() // k
        x_send = ops.gather(x, tok)
        ids = torch.as_tensor(local_expert_ids(offsets_host, self.world), device=x.device)
        x_recv = self._exchange(x_send, send_counts, recv_counts)
        id_recv = self._exchange(ids, send_counts, recv_counts)
        y_recv = ops.local_ffn(x_recv, id_recv)
        y_back = self._exchange(y_recv, recv_counts, send_counts)  # grouped order again
        y_shared = ops.shared_ffn(x)
        return ops.combine(y_back, y_shared, inv, gates)


class LibraryOps:
    """The per-rank arithmetic through the library's C-ABI stage entry points.

    ``cfg`` is the global layer (d, f, E, k); ``router_w`` / ``router_bias`` the full router;
    ``local_routed`` the bank dict (as in ``binding.DeviceLayer.banks``) of this rank's
    E / W experts; ``shared`` the shared expert's bank dict or None. Workspaces are allocated
    per shape and kept."""

    def __init__(self, cfg, router_w, router_bias, local_routed: dict, shared: dict | None,
                 world: int):
        from . import binding as B
        self.B = B
        self.cfg, self.world = cfg, world
        self.E_loc = cfg.E // world
        self.router_w, self.router_bias = router_w, router_bias
        self.local, self.shared = local_routed, shared
        self._ws = {}

    def _ws_for(self, key, desc):
        if key not in self._ws or self._ws[key].numel() < self.B.workspace_size(desc):
            self._ws[key] = self.B.alloc_workspace(desc, device=self.router_w.device)
        return self._ws[key]

    def _desc(self, T, E, k, routed, shared):
        B, cfg = self.B, self.cfg
        return B.MoeLayer(T, cfg.d, cfg.f, E, k, B.PATH_CODE["auto"],
                          self.router_w.data_ptr(),
                          None if self.router_bias is None else self.router_bias.data_ptr(),
                          B.bank_struct(routed), B.bank_struct(shared))

    def _full(self, T):
        # route, permute and combine read the router and the plan only, never a bank's weights;
        # the descriptor names this rank's bank with the global expert count for validation
        routed = dict(self.local, n_exp=self.cfg.E)
        return self._desc(T, self.cfg.E, self.cfg.k, routed, self.shared)

    def route(self, x):
        desc = self._full(x.shape[0])
        return self.B.route(desc, x, self._ws_for(("full", x.shape[0]), desc))

    def permute(self, idx):
        desc = self._full(idx.shape[0])
        return self.B.permute(desc, idx, self._ws_for(("full", idx.shape[0]), desc))

    def gather(self, x, rows):
        return x.index_select(0, rows)

    def _one_per_row(self, x, ids, bank, E):
        """The grouped FFN of a layer over ``bank``'s E experts with one assignment a row,
        returned in the rows' order."""
        import torch
        R = x.shape[0]
        if R == 0:
            return torch.empty((0, self.cfg.d), dtype=torch.float32, device=x.device)
        desc = self._desc(R, E, 1, bank, None)
        ws = self._ws_for(("one", E, R), desc)
        offsets, perm, inv = self.B.permute(desc, ids.view(R, 1).contiguous(), ws)
        y_assign, _ = self.B.grouped_ffn(desc, x, offsets, perm, ws, has_shared=False)
        return y_assign.index_select(0, inv.long())

    def local_ffn(self, x_rows, local_ids):
        return self._one_per_row(x_rows, local_ids, self.local, self.E_loc)

    def shared_ffn(self, x):
        import torch
        if self.shared is None:
            return None
        ids = torch.zeros(x.shape[0], dtype=torch.int32, device=x.device)
        return self._one_per_row(x, ids, self.shared, 1)

    def combine(self, y_assign, y_shared, inv, gates):
        desc = self._full(gates.shape[0])
        return self.B.combine(desc, y_assign, y_shared, inv, gates)
