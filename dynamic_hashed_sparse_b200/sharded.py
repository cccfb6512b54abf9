"""Hash-sharded engine: one table per rank, each key owned by one rank.

Sources: the RecIS overview (code-architecture section: the collective
All-to-All of parameter aggregation) and the DLRM explainer (practice cases 1
and 2: embedding rows split across cards, lookups exchanged by all-to-all,
while the dense layers stay data-parallel).

A step on each rank (its own batch of ids and bags):

  forward   ht_shard_route groups the ids by owner rank; the keys go to their
            owners (all-to-all); each owner looks its received keys up, with
            insertion, through embbag_forward (one id per bag, so the "pooled"
            output is the rows themselves); the rows come back (all-to-all);
            ht_shard_pool pools them per bag.
  backward  ht_shard_grads forms each id's gradient row (its bag's row, and
            the id's weight or bag length); they go to the owners; each owner
            runs embbag_backward_update(_ex) on them, one id per bag.

Every kernel of the step is the library's; the exchanges are NCCL all-to-all
calls through torch.distributed (plumbing).  Owners receive ids in (source
rank, position) order, so sums run over the concatenated global batch in its
order: pooled outputs are formed as one table forms them (bit for bit from the
same rows), and each key's update is that of one table fed the ranks' batches
one after another, up to the association of the fp64 partial sums.

The step is written as a generator that yields at each exchange, so that the
same code runs over NCCL (forward / backward_update) or over any other
exchange that drives the generators of all ranks in lockstep.
"""
from __future__ import annotations

from typing import List, Optional

import torch

from . import _binding as B


class NcclExchange:
    """All-to-all over a torch.distributed process group (NCCL for CUDA
    tensors; the same calls work over gloo for CPU tensors)."""

    def __init__(self, group=None):
        import torch.distributed as tdist
        self._d = tdist
        self.group = group
        self.world = tdist.get_world_size(group)
        self.rank = tdist.get_rank(group)

    def counts(self, send_counts: List[int], device) -> List[int]:
        """recv[r] = what rank r sends to this rank."""
        s = torch.tensor(send_counts, dtype=torch.int64, device=device)
        r = torch.empty_like(s)
        self._d.all_to_all_single(r, s, group=self.group)
        return [int(x) for x in r.tolist()]

    def exchange(self, x: torch.Tensor, send_counts: List[int], recv_counts: List[int]) -> torch.Tensor:
        """Rows [send_counts[0] for rank 0, ...] out; rows from each rank in
        rank order in."""
        out = torch.empty((sum(recv_counts),) + tuple(x.shape[1:]), dtype=x.dtype, device=x.device)
        self._d.all_to_all_single(out, x.contiguous(), output_split_sizes=list(recv_counts),
                                  input_split_sizes=list(send_counts), group=self.group)
        return out


class ShardedTable:
    """This rank's shard: a table holding the keys it owns, and the routing of
    its own batches.  world / rank come from the exchange (or are given, for
    a driver that runs several ranks in one process)."""

    def __init__(self, dim: int, optimizer: str = "sgd", exchange=None, world: Optional[int] = None,
                 rank: Optional[int] = None, **table_kwargs):
        self.ex = exchange
        if world is None:
            if exchange is None:
                self.ex = NcclExchange()
            world, rank = self.ex.world, self.ex.rank
        if not 1 <= world <= 256 or not 0 <= rank < world:
            raise ValueError("world must be in [1, 256] and rank in [0, world)")
        self.world, self.rank = world, rank
        self.dim = dim
        self.table = B.ht_create(dim, optimizer, **table_kwargs)
        self._ctx = None

    def close(self):
        self.table.close()

    # ---- the step as generators: each yield is one exchange ----
    # ("counts", send_counts) -> recv_counts
    # ("rows", tensor, send_counts, recv_counts) -> received tensor

    def forward_steps(self, keys: torch.Tensor, bag_offsets: torch.Tensor,
                      per_sample_weights: Optional[torch.Tensor] = None, mode: str = "sum"):
        if mode not in ("sum", "mean"):
            raise ValueError("mode must be 'sum' or 'mean'")
        send_keys, slot_of, counts = B.ht_shard_route(self.table, keys, self.world)
        recv_counts = yield ("counts", counts)
        recv_keys = yield ("rows", send_keys, counts, recv_counts)
        # owner side: insert / look up the received keys, one id per bag
        ident = torch.arange(recv_keys.numel() + 1, dtype=torch.int64, device=keys.device)
        rows = B.embbag_forward(self.table, recv_keys, ident)
        back = yield ("rows", rows, recv_counts, counts)
        pooled = B.ht_shard_pool(self.table, back, slot_of, bag_offsets, per_sample_weights, mode)
        self._ctx = (bag_offsets, per_sample_weights, mode, slot_of, counts, recv_counts, recv_keys, ident)
        return pooled

    def backward_steps(self, grad: torch.Tensor, lr: float):
        if self._ctx is None:
            raise RuntimeError("backward_update needs the forward of the same step first")
        bag_offsets, psw, mode, slot_of, counts, recv_counts, recv_keys, ident = self._ctx
        self._ctx = None
        send, fact = B.ht_shard_grads(self.table, grad, bag_offsets, slot_of, psw, mode)
        recv = yield ("rows", send, counts, recv_counts)
        rfact = None
        if fact is not None:
            rfact = yield ("rows", fact, counts, recv_counts)
        # owner side: one id per bag, the factor carried as a per-id weight
        # (sum pooling) or divisor (mean pooling)
        if rfact is None:
            B.embbag_backward_update(self.table, recv_keys, ident, recv, lr)
        else:
            B.embbag_backward_update_ex(self.table, recv_keys, ident, recv, lr, per_sample_weights=rfact,
                                        mode="sum" if mode == "sum" else "divide")

    # ---- driven by this rank's exchange ----

    def _run(self, gen, device):
        try:
            req = next(gen)
            while True:
                if req[0] == "counts":
                    resp = self.ex.counts(req[1], device)
                else:
                    resp = self.ex.exchange(req[1], req[2], req[3])
                req = gen.send(resp)
        except StopIteration as stop:
            return stop.value

    def forward(self, keys: torch.Tensor, bag_offsets: torch.Tensor,
                per_sample_weights: Optional[torch.Tensor] = None, mode: str = "sum") -> torch.Tensor:
        return self._run(self.forward_steps(keys, bag_offsets, per_sample_weights, mode), keys.device)

    def backward_update(self, grad: torch.Tensor, lr: float):
        self._run(self.backward_steps(grad, lr), grad.device)


def run_lockstep(gens):
    """Drive the step generators of all ranks of one process in lockstep
    (rank r = gens[r]), doing each exchange with device copies.  Returns each
    generator's result."""
    W = len(gens)
    results = [None] * W
    reqs = []
    for g in gens:
        reqs.append(next(g))
    live = [True] * W
    while any(live):
        kinds = {r[0] for r, a in zip(reqs, live) if a}
        if len(kinds) != 1 or not all(live):
            raise RuntimeError("ranks out of step")
        if reqs[0][0] == "counts":
            resp = [[reqs[src][1][dst] for src in range(W)] for dst in range(W)]
        else:
            resp = []
            for dst in range(W):
                parts = []
                for src in range(W):
                    x, send_counts = reqs[src][1], reqs[src][2]
                    off = sum(send_counts[:dst])
                    parts.append(x[off:off + send_counts[dst]])
                resp.append(torch.cat(parts) if parts else reqs[dst][1][:0])
        for r, g in enumerate(gens):
            try:
                reqs[r] = g.send(resp[r])
            except StopIteration as stop:
                results[r] = stop.value
                live[r] = False
    return results
