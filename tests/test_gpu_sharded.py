"""GPU parity of the hash-sharded engine: W ranks run in one process on one
GPU, their exchanges done by run_lockstep (device copies; no kernel waits on
another), against the CPU oracle fed the ranks' batches concatenated in rank
order.

Checked: the routing (owner of every key by an independent implementation of
the documented owner function; groups in rank order, positions in order
within a group), pooled outputs (bit for bit on fresh rows, within the parity
bar once rows have been updated), every shard's key -> row map exactly (a
shard inserts its keys in the global batch's order), and the updated weights
and state of every key within the parity bar."""
import numpy as np
import pytest
import torch

import dynamic_hashed_sparse_b200 as dhs
from dynamic_hashed_sparse_b200.sharded import ShardedTable, run_lockstep
from oracle import Oracle
from tests.parity import assert_close, dev, host

pytestmark = pytest.mark.gpu

M64 = (1 << 64) - 1


def owner_np(keys: np.ndarray, world: int) -> np.ndarray:
    """The owner function as the header defines it: splitmix64's finaliser
    of key XOR 0x5DEECE66D, upper 32 bits times world, upper 32 bits of that."""
    out = np.empty(keys.size, np.int64)
    for i, k in enumerate(keys.tolist()):
        z = (k ^ 0x5DEECE66D) & M64
        z = ((z ^ (z >> 30)) * 0xBF58476D1CE4E5B9) & M64
        z = ((z ^ (z >> 27)) * 0x94D049BB133111EB) & M64
        z ^= z >> 31
        out[i] = ((z >> 32) * world) >> 32
    return out


def _batch(rng, n_bags, max_len, universe):
    lens = rng.integers(0, max_len + 1, size=n_bags)
    offs = np.concatenate([[0], np.cumsum(lens)]).astype(np.int64)
    n = int(offs[-1])
    keys = (rng.zipf(1.2, size=n) % universe).astype(np.int64) * 1000003 + 17
    return keys, offs


def test_route_groups_by_owner_in_position_order():
    rng = np.random.default_rng(5)
    t = dhs.ht_create(8, "sgd")
    try:
        for world in (1, 2, 3, 8, 256):
            keys = rng.integers(0, 1 << 50, size=20_000).astype(np.int64)
            keys[::7] = keys[3]  # repeats
            send, slot, counts = dhs.ht_shard_route(t, dev(keys), world)
            own = owner_np(keys, world)
            np.testing.assert_array_equal(counts, np.bincount(own, minlength=world))
            order = np.argsort(own, kind="stable")
            np.testing.assert_array_equal(host(send), keys[order])
            inv = np.empty(keys.size, np.int64)
            inv[order] = np.arange(keys.size)
            np.testing.assert_array_equal(host(slot), inv)
        _, _, counts = dhs.ht_shard_route(t, dev(np.zeros(0, np.int64)), 4)
        assert counts == [0, 0, 0, 0]
        with pytest.raises(dhs.DhsError):
            dhs.ht_shard_route(t, dev(keys), 0)
        with pytest.raises(dhs.DhsError):
            dhs.ht_shard_route(t, dev(keys), 257)
    finally:
        t.close()


def _oracle_step(o, batches, grads, lr, psws, mode):
    """The oracle on the ranks' batches concatenated in rank order."""
    keys = np.concatenate([b[0] for b in batches])
    offs, base = [np.zeros(1, np.int64)], 0
    for k, off in batches:
        offs.append(off[1:] + base)
        base += k.size
    offs = np.concatenate(offs)
    psw = np.concatenate(psws) if psws[0] is not None else None
    pooled, rc = o.forward(keys, offs, psw, mode)
    assert rc == 0
    assert o.backward_update(keys, offs, np.concatenate(grads), lr, psw, mode) == 0
    cuts = np.cumsum([0] + [off.size - 1 for _, off in batches])
    return [pooled[cuts[r]:cuts[r + 1]] for r in range(len(batches))]


@pytest.mark.parametrize("form", ["sum", "weights", "mean"])
@pytest.mark.parametrize("world,dim,opt", [(2, 64, "adagrad"), (3, 16, "adam"), (4, 128, "adagrad"),
                                           (2, 32, "adagrad_rowwise"), (5, 8, "sgd")])
def test_sharded_steps_match_one_table(world, dim, opt, form):
    rng = np.random.default_rng(world * 100 + dim)
    mode = "mean" if form == "mean" else "sum"
    shards = [ShardedTable(dim, opt, world=world, rank=r, block_rows=1024) for r in range(world)]
    o = Oracle(dim, opt)
    lr = 0.05
    try:
        for step in range(3):
            batches = [_batch(rng, 400 + 50 * r, 3 if step % 2 else 9, 4000) for r in range(world)]
            psws = [rng.uniform(0.5, 1.5, k.size).astype(np.float32) if form == "weights" else None
                    for k, _ in batches]
            pooled = run_lockstep([
                s.forward_steps(dev(k), dev(off), dev(p) if p is not None else None, mode)
                for s, (k, off), p in zip(shards, batches, psws)])
            grads = [rng.standard_normal((off.size - 1, dim)).astype(np.float32) for _, off in batches]
            run_lockstep([s.backward_steps(dev(g), lr) for s, g in zip(shards, grads)])
            ref = _oracle_step(o, batches, grads, lr, psws, mode)
            for r in range(world):
                # fresh rows: bit for bit; updated rows carry the association
                # of the fp64 partial sums, so later steps are held to the bar
                if step == 0:
                    np.testing.assert_array_equal(host(pooled[r]), ref[r], err_msg=f"rank {r} pooled")
                else:
                    assert_close(host(pooled[r]), ref[r], f"step {step} rank {r} pooled")
        # every key in exactly one shard, its owner; weights and state as one table's
        ok, orows = o.export()
        got = {}
        for r, s in enumerate(shards):
            assert dhs.ht_sync(s.table) == 0
            gk, grows, rc = dhs.ht_export(s.table)
            assert rc == 0
            assert (owner_np(gk, world) == r).all(), f"shard {r} holds keys it does not own"
            for k, row in zip(gk.tolist(), grows):
                got[k] = row
        assert sorted(got) == sorted(ok.tolist())
        ref_rows = np.stack([orows[i] for i in range(ok.size)])
        mine = np.stack([got[k] for k in ok.tolist()])
        assert_close(mine[:, :dim], ref_rows[:, :dim], f"W={world} {opt} {form}: weights")
        if opt != "adagrad_rowwise" and ref_rows.shape[1] > dim:
            assert_close(mine[:, dim:], ref_rows[:, dim:], f"W={world} {opt} {form}: state")
    finally:
        for s in shards:
            s.close()
        o.close()


def test_shard_key_to_row_maps_follow_the_global_order():
    """Shard r inserts its keys in the order they first occur in the global
    stream (rank 0's batch, then rank 1's, ...), over several steps."""
    world, dim = 3, 8
    rng = np.random.default_rng(11)
    shards = [ShardedTable(dim, "sgd", world=world, rank=r, block_rows=512) for r in range(world)]
    oracles = [Oracle(dim, "sgd") for _ in range(world)]
    try:
        for step in range(4):
            batches = [_batch(rng, 300, 5, 20000) for _ in range(world)]
            run_lockstep([s.forward_steps(dev(k), dev(off)) for s, (k, off) in zip(shards, batches)])
            allk = np.concatenate([k for k, _ in batches])
            own = owner_np(allk, world)
            for r in range(world):
                oracles[r].lookup_or_insert(allk[own == r])
        for r in range(world):
            gk, _, rc = dhs.ht_export(shards[r].table, rows=False)
            ok, _ = oracles[r].export()
            assert rc == 0
            np.testing.assert_array_equal(gk, ok)
    finally:
        for s in shards:
            s.close()
        for o in oracles:
            o.close()


def test_sharded_engine_through_nccl_with_one_rank():
    """ShardedTable's own driver over a real NCCL process group (one rank on
    this GPU: every call on this pool gets one GPU), against the oracle."""
    import datetime
    import socket

    import torch.distributed as tdist
    with socket.socket() as so:
        so.bind(("127.0.0.1", 0))
        port = so.getsockname()[1]
    tdist.init_process_group("nccl", init_method=f"tcp://127.0.0.1:{port}", world_size=1, rank=0,
                             timeout=datetime.timedelta(seconds=60))
    rng = np.random.default_rng(3)
    dim, lr = 32, 0.05
    s = o = None
    try:
        s = ShardedTable(dim, "adagrad", block_rows=1024)
        assert (s.world, s.rank) == (1, 0)
        o = Oracle(dim, "adagrad")
        for step in range(3):
            keys, offs = _batch(rng, 600, 6, 5000)
            pooled = host(s.forward(dev(keys), dev(offs), mode="mean"))
            grad = rng.standard_normal((offs.size - 1, dim)).astype(np.float32)
            s.backward_update(dev(grad), lr)
            ref, rc = o.forward(keys, offs, None, "mean")
            assert rc == 0
            assert o.backward_update(keys, offs, grad, lr, None, "mean") == 0
            if step == 0:
                np.testing.assert_array_equal(pooled, ref)
            else:
                assert_close(pooled, ref, f"step {step} pooled")
        assert dhs.ht_sync(s.table) == 0
        gk, grows, rc = dhs.ht_export(s.table)
        ok, orows = o.export()
        assert rc == 0
        np.testing.assert_array_equal(gk, ok)  # one rank owns every key, in stream order
        assert_close(grows[:, :dim], orows[:, :dim], "weights")
        assert_close(grows[:, dim:], orows[:, dim:], "state")
    finally:
        if s is not None:
            s.close()
        if o is not None:
            o.close()
        tdist.destroy_process_group()
