"""Host-side logic of the hash-sharded engine, no GPU: the exchange over two
gloo ranks on CPU (counts and row blocks in rank order), and the step-driving
protocol -- the same step generators run over gloo (ShardedTable's own
driver) and in one process (run_lockstep) give the same results."""
import os
import socket
import sys
import types

import torch
import torch.multiprocessing as mp

from tests.conftest import ROOT


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _fake_step(rank, world):
    """A step shaped like the engine's: send counts, then rows whose values
    say who sent them to whom, then a second exchange of the received rows
    back; returns what came in."""
    counts = [rank + d + 1 for d in range(world)]
    rows = torch.cat([torch.full((c, 2), 0.0) + torch.tensor([rank, d], dtype=torch.float32)
                      for d, c in enumerate(counts)])
    recv_counts = yield ("counts", counts)
    got = yield ("rows", rows, counts, recv_counts)
    back = yield ("rows", got * 10, recv_counts, counts)
    return recv_counts, got, back


def _expected(rank, world):
    recv_counts = [src + rank + 1 for src in range(world)]
    got = torch.cat([torch.tensor([[src, rank]], dtype=torch.float32).repeat(c, 1)
                     for src, c in enumerate(recv_counts)])
    back = torch.cat([torch.tensor([[rank, d]], dtype=torch.float32).repeat(rank + d + 1, 1) * 10
                      for d in range(world)])
    return recv_counts, got, back


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    sys.path.insert(0, ROOT)
    import datetime

    import torch.distributed as tdist
    tdist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        from dynamic_hashed_sparse_b200.sharded import NcclExchange, ShardedTable
        ex = NcclExchange()
        assert (ex.world, ex.rank) == (world, rank)
        driver = types.SimpleNamespace(ex=ex)
        res = ShardedTable._run(driver, _fake_step(rank, world), torch.device("cpu"))
        exp = _expected(rank, world)
        ok = res[0] == exp[0] and torch.equal(res[1], exp[1]) and torch.equal(res[2], exp[2])
        q.put((rank, ok))
    finally:
        tdist.destroy_process_group()


def test_exchange_and_step_driver_over_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    out = sorted(q.get(timeout=180) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert out == [(0, True), (1, True)]


def test_lockstep_driver_in_one_process():
    from dynamic_hashed_sparse_b200.sharded import run_lockstep
    for world in (1, 2, 3, 5):
        res = run_lockstep([_fake_step(r, world) for r in range(world)])
        for r in range(world):
            exp = _expected(r, world)
            assert res[r][0] == exp[0]
            assert torch.equal(res[r][1], exp[1]) and torch.equal(res[r][2], exp[2])
