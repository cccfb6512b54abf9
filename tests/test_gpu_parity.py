"""GPU-vs-oracle parity through the C ABI (needs a B200).

Every test feeds the same seeded inputs to libdhs.so and to the CPU oracle
and compares: key packing and key -> row maps exactly, pooled outputs and
updated rows / optimizer state within the 1e-5 relative bar."""
import numpy as np
import pytest
import torch

import dynamic_hashed_sparse_b200 as dhs
from oracle import Oracle, pack_keys
from tests.parity import assert_close, close_report, dev, host
from workloads import gen

pytestmark = pytest.mark.gpu


def make_pair(dim, opt, block_rows=1024, eps=1e-8, beta1=0.9, beta2=0.999, max_rows=0):
    t = dhs.ht_create(dim, opt, block_rows=block_rows, max_rows=max_rows, eps=eps, beta1=beta1, beta2=beta2)
    o = Oracle(dim, opt, eps=eps, beta1=beta1, beta2=beta2)
    return t, o


def compare_tables(t, o, what=""):
    gk, grows, rc = dhs.ht_export(t)
    ok_, orows = o.export()
    assert rc == 0, f"{what}: latched status {rc}"
    np.testing.assert_array_equal(gk, ok_, err_msg=f"{what}: key -> row map")
    d = t.dim
    assert_close(grows[:, :d], orows[:, :d], f"{what}: weights")
    if t.optimizer == "adagrad_rowwise":
        assert_close(grows[:, d], orows[:, d], f"{what}: row accumulator")
    elif orows.shape[1] > d:
        assert_close(grows[:, d:], orows[:, d:], f"{what}: optimizer state")


def pack_both(tids, ids):
    ko, rc = pack_keys(tids, ids)
    kg = dhs.dhs_pack_keys(dev(tids.astype(np.int32)), dev(ids.astype(np.int64)))
    np.testing.assert_array_equal(host(kg), ko)
    return kg, ko


def step_both(t, o, kg, ko, offs, grad, lr, check=True):
    og = dev(offs)
    pg = dhs.embbag_forward(t, kg, og)
    po, rco = o.forward(ko, offs)
    if check:
        assert_close(host(pg), po, "pooled")
    if grad is not None:
        dhs.embbag_backward_update(t, kg, og, dev(grad), lr)
        o.backward_update(ko, offs, grad, lr)
    return host(pg), po


def run_workload(w, steps=None, block_rows=1024, compare_each=True):
    t, o = make_pair(w.dim, w.optimizer, block_rows=block_rows, eps=w.eps, beta1=w.beta1, beta2=w.beta2)
    try:
        for tids, ids in w.preinsert():
            kg, ko = pack_both(tids, ids)
            og = host(dhs.ht_lookup_or_insert(t, kg))
            oo, _ = o.lookup_or_insert(ko)
            np.testing.assert_array_equal(og, oo)
        for s in range(w.steps if steps is None else steps):
            b = w.batch(s)
            kg, ko = pack_both(b.table_ids, b.ids)
            grad = w.grads(s, b.n_bags)
            step_both(t, o, kg, ko, b.bag_offsets, grad, w.lr)
            if compare_each:
                assert dhs.ht_sync(t) == 0
        compare_tables(t, o, w.name)
        return dhs.ht_counters(t)
    finally:
        t.close()
        o.close()


# --------------------------------------------------------------------------------------

def test_pack_keys():
    rng = np.random.default_rng(0)
    n = 10007
    tids = rng.integers(-2, 1 << 15 + 1, size=n).astype(np.int32)
    ids = rng.integers(-5, 1 << 49, size=n).astype(np.int64)
    ids[:50] = (1 << 48) - 1
    pack_both(tids, ids)


def test_lookup_or_insert_maps_first_occurrence_across_calls_and_growth():
    # > 32768 keys forces IDMap rehashes; 512-row blocks force many appends
    t, o = make_pair(8, "sgd", block_rows=512)
    rng = np.random.default_rng(1)
    try:
        seen = np.zeros(0, np.int64)
        for call, n in enumerate([1, 4096, 33333, 70001, 5, 0, 25000]):
            fresh = rng.integers(0, 1 << 62, size=n // 2 + 1, dtype=np.int64)
            old = seen[rng.integers(0, max(1, seen.size), size=max(0, n - n // 2 - 1))] if seen.size else fresh[:0]
            keys = rng.permutation(np.concatenate([fresh, old, fresh[: n // 7]]))[:n]
            g = host(dhs.ht_lookup_or_insert(t, dev(keys)))
            r, _ = o.lookup_or_insert(keys)
            np.testing.assert_array_equal(g, r, err_msg=f"call {call}")
            seen = np.concatenate([seen, keys])
        n_rows, rc = dhs.ht_size(t)
        assert rc == 0 and n_rows == o.size
        c = dhs.ht_counters(t)
        assert c["rehashes"] >= 2 and c["blocks"] >= n_rows // 512
        compare_tables(t, o, "lookup_or_insert")
        # read-only lookup: hits and misses, nothing inserted
        probe = np.concatenate([seen[:1000], rng.integers(1 << 62, (1 << 63) - 1, size=500, dtype=np.int64),
                                np.array([-7], np.int64)])
        g = host(dhs.ht_lookup(t, dev(probe)))
        np.testing.assert_array_equal(g, o.lookup(probe))
        assert dhs.ht_size(t)[0] == n_rows
        # full rows by key, NaN for absent keys
        rows = host(dhs.ht_get_rows(t, dev(probe)))
        ref, missing = o.get_rows(probe)
        assert missing == 501
        assert np.array_equal(np.isnan(rows[:, 0]), np.isnan(ref[:, 0]))
        np.testing.assert_array_equal(rows[:1000], ref[:1000])
    finally:
        t.close()
        o.close()


@pytest.mark.parametrize("name", gen.NAMES)
def test_workload_parity_small(name):
    w = gen.small(name)
    c = run_workload(w)
    assert c["rows"] > 0


def test_forward_is_bit_exact():
    w = gen.small("sequence_bags")
    t, o = make_pair(w.dim, w.optimizer)
    try:
        for s in range(2):
            b = w.batch(s)
            kg, ko = pack_both(b.table_ids, b.ids)
            pg, po = step_both(t, o, kg, ko, b.bag_offsets, w.grads(s, b.n_bags), w.lr)
            assert np.array_equal(pg, po), close_report(pg, po)
    finally:
        t.close()
        o.close()


DIMS = [4, 8, 12, 16, 32, 40, 64, 128, 132, 200, 260, 512]


@pytest.mark.parametrize("bags", ["long", "short"])
@pytest.mark.parametrize("opt", ["sgd", "adagrad", "adam", "adagrad_rowwise"])
@pytest.mark.parametrize("dim", DIMS)
def test_dims_and_optimizers(dim, opt, bags):
    """Every row width the kernels are instantiated for, with every optimizer.
    Long bags (about 5.5 ids each) take the split forward (probe kernel, then
    the gather from row references); short bags (about 1.5 ids each) the fused
    probe + pool kernel.  Together the widths reach each (group, columns)
    instantiation of both forward kernels and of both segment kernels."""
    rng = np.random.default_rng(dim * 7 + len(opt) + (0 if bags == "long" else 1000))
    t, o = make_pair(dim, opt, block_rows=256)
    try:
        dhs.ht_set_phase_timing(t, True)
        for s in range(3):
            nb = int(rng.integers(300, 900))
            lens = rng.integers(0, 12 if bags == "long" else 4, size=nb)
            lens[rng.integers(0, nb, size=5)] = 0
            offs = np.concatenate([[0], np.cumsum(lens)]).astype(np.int64)
            n = int(offs[-1])
            keys = np.where(rng.random(n) < 0.3, rng.integers(0, 8, size=n),
                            rng.integers(0, 3000, size=n)).astype(np.int64) * 1000003
            grad = rng.standard_normal((nb, dim)).astype(np.float32)
            step_both(t, o, dev(keys), keys, offs, grad, 0.05)
        assert dhs.ht_sync(t) == 0
        ph = dhs.ht_phase_times(t)
        # the split forward runs its probe as a phase of its own; the fused one does not
        assert (ph["fwd_probe"][1] == 3) == (bags == "long"), ph
        compare_tables(t, o, f"dim {dim} {opt} {bags} bags")
    finally:
        t.close()
        o.close()


@pytest.mark.parametrize("occ", [255, 256, 257, 600, 1000, 1030, 1060, 5000, 8200, 40000])
def test_hot_key_spanning_many_sort_chunks(occ):
    """One key occurs `occ` times (its run covers one sort chunk of 32 pairs up
    to hundreds of them), mixed with a tail of other keys before and after it
    in row order; both segment kernels (narrow and wide rows), every
    optimizer.  Runs of about 32 chunks (1,000 to 1,060 occurrences) sit at
    the boundary between a long segment that the segment kernel's warp or
    lane group finishes and one that goes to the combine kernels."""
    rng = np.random.default_rng(occ)
    for dim, opt in ((32, "adagrad"), (32, "adam"), (32, "adagrad_rowwise"), (12, "adagrad"), (128, "sgd"),
                     (16, "sgd"), (20, "adam"), (16, "adagrad_rowwise")):
        t, o = make_pair(dim, opt)
        try:
            warm = np.arange(1, 600, dtype=np.int64)  # rows 0.. for the tail keys
            hot = np.int64(424242)
            pre = np.concatenate([warm[:300], [hot], warm[300:]])
            dhs.ht_lookup_or_insert(t, dev(pre))
            o.lookup_or_insert(pre)
            n_other = 3000
            keys = np.concatenate([np.full(occ, hot), rng.choice(warm, size=n_other)])
            keys = rng.permutation(keys).astype(np.int64)
            nb = 700
            cuts = np.sort(rng.integers(0, keys.size, size=nb - 1))
            offs = np.concatenate([[0], cuts, [keys.size]]).astype(np.int64)
            grad = rng.standard_normal((nb, dim)).astype(np.float32)
            step_both(t, o, dev(keys), keys, offs, grad, 0.01)
            step_both(t, o, dev(keys), keys, offs, grad * 0.5, 0.01)
            assert dhs.ht_sync(t) == 0
            compare_tables(t, o, f"hot {occ} {opt}")
            c = dhs.ht_counters(t)
            assert c["unique_updated"] == 2 * np.unique(keys).size
        finally:
            t.close()
            o.close()


@pytest.mark.parametrize("dim", [16, 64])
@pytest.mark.parametrize("n_target", [20_000, 150_000, 700_000])
def test_segment_runs_at_every_chunk_alignment(n_target, dim):
    """Rows with run lengths that put segment starts and ends at every offset
    of the sort chunks (32 or 64 pairs, by batch size),
    including runs of exactly C, 2C, 3C and one longer or shorter."""
    rng = np.random.default_rng(n_target)
    special = []
    for C in (32, 64, 128, 256):
        special += [C - 1, C, C + 1, 2 * C - 1, 2 * C, 2 * C + 1, 3 * C - 1, 3 * C, 3 * C + 1]
    lens = []
    while sum(lens) < n_target:
        lens += list(rng.permutation(special + list(range(1, 40))))
    lens = np.array(lens, np.int64)
    keys_by_row = np.arange(lens.size, dtype=np.int64) * 7 + 11
    for opt in ("adagrad", "adam"):
        t, o = make_pair(dim, opt)
        try:
            dhs.ht_lookup_or_insert(t, dev(keys_by_row))
            o.lookup_or_insert(keys_by_row)
            keys = rng.permutation(np.repeat(keys_by_row, lens))
            nb = keys.size // 3
            cuts = np.sort(rng.integers(0, keys.size, size=nb - 1))
            offs = np.concatenate([[0], cuts, [keys.size]]).astype(np.int64)
            grad = rng.standard_normal((nb, dim)).astype(np.float32)
            step_both(t, o, dev(keys), keys, offs, grad, 0.01)
            assert dhs.ht_sync(t) == 0
            compare_tables(t, o, f"runs {n_target} {opt}")
        finally:
            t.close()
            o.close()


@pytest.mark.parametrize("dim,opt,short", [(64, "adagrad", True), (16, "adam", False), (128, "sgd", True),
                                           (64, "adagrad", False), (128, "sgd", False)])
def test_backward_with_keys_other_than_the_last_forward(dim, opt, short):
    """Backward calls whose keys are not those of the forward just before:
    the keys of an older forward, the same keys at other positions, a third
    of them replaced by other known keys, more positions than the forward
    before, and after a lookup-or-insert and growth, all against the
    oracle."""
    rng = np.random.default_rng(dim + (7 if short else 0))
    t, o = make_pair(dim, opt, block_rows=512)
    try:
        def batch(n_bags, universe):
            # short bags run the fused forward; long ones (at least 4 ids per
            # bag on average) the split forward, whose record of keys and rows
            # the backward reads where its keys are the forward's
            lens = rng.integers(0, 3, size=n_bags) if short else rng.integers(2, 12, size=n_bags)
            offs = np.concatenate([[0], np.cumsum(lens)]).astype(np.int64)
            keys = (rng.integers(0, universe, size=int(offs[-1])) * 7 + 5).astype(np.int64)
            return keys, offs

        def fwd(keys, offs):
            pg = host(dhs.embbag_forward(t, dev(keys), dev(offs)))
            po, rc = o.forward(keys, offs)
            assert rc == 0
            assert_close(pg, po, "pooled")

        def bwd(keys, offs):
            grad = rng.standard_normal((offs.size - 1, dim)).astype(np.float32)
            dhs.embbag_backward_update(t, dev(keys), dev(offs), dev(grad), 0.03)
            assert o.backward_update(keys, offs, grad, 0.03) == 0

        a, b = batch(800, 3000), batch(900, 3000)
        fwd(*a)
        fwd(*b)
        bwd(*a)  # keys of an older forward
        c = batch(700, 5000)
        fwd(*c)
        kc, oc = c
        perm = rng.permutation(kc.size)
        bwd(kc[perm], oc)  # same keys, other positions
        fwd(*c)
        mixed = kc.copy()
        mixed[::3] = a[0][: mixed[::3].size]  # a third replaced by other known keys
        bwd(mixed, oc)
        bwd(*c)  # the keys of the last forward, after another backward
        bwd(*c)
        d = batch(1500, 20000)  # more positions than the last forward, with growth
        fwd(d[0][:-100], np.minimum(d[1], d[0].size - 100))
        fwd(*d)
        bwd(*d)
        e = batch(400, 3000)
        dhs.ht_lookup_or_insert(t, dev(e[0]))
        o.lookup_or_insert(e[0])
        bwd(*e)  # after a lookup-or-insert
        assert dhs.ht_sync(t) == 0
        compare_tables(t, o, f"dim {dim} {opt}")
    finally:
        t.close()
        o.close()


def test_empty_inputs_and_empty_bags():
    t, o = make_pair(16, "adam")
    try:
        # no ids at all, some bags
        offs = np.zeros(6, np.int64)
        step_both(t, o, dev(np.zeros(0, np.int64)), np.zeros(0, np.int64), offs,
                  np.ones((5, 16), np.float32), 0.1)
        # no bags
        out = dhs.embbag_forward(t, dev(np.zeros(0, np.int64)), dev(np.zeros(1, np.int64)))
        assert out.shape == (0, 16)
        # leading / trailing / interior empty bags and one giant bag
        rng = np.random.default_rng(3)
        lens = np.array([0, 0, 3, 0, 10000, 0, 1, 0, 0], np.int64)
        offs = np.concatenate([[0], np.cumsum(lens)]).astype(np.int64)
        keys = rng.integers(0, 5000, size=int(offs[-1])).astype(np.int64)
        grad = rng.standard_normal((lens.size, 16)).astype(np.float32)
        for _ in range(2):
            step_both(t, o, dev(keys), keys, offs, grad, 0.1)
        assert dhs.ht_sync(t) == 0
        compare_tables(t, o, "empty bags")
    finally:
        t.close()
        o.close()


def test_negative_and_missing_keys_are_latched_and_skipped():
    t, o = make_pair(8, "sgd")
    try:
        keys = np.array([5, -3, 7, 5], np.int64)
        offs = np.array([0, 2, 4], np.int64)
        pg, po = step_both(t, o, dev(keys), keys, offs, None, 0.1)
        assert dhs.ht_sync(t) == 1           # invalid argument latched
        assert dhs.ht_sync(t) == 0           # and cleared by the read
        # backward with a key that was never inserted
        bkeys = np.array([5, 99, 7], np.int64)
        boffs = np.array([0, 1, 3], np.int64)
        grad = np.ones((2, 8), np.float32)
        dhs.embbag_backward_update(t, dev(bkeys), dev(boffs), dev(grad), 0.5)
        rc = o.backward_update(bkeys, boffs, grad, 0.5)
        assert rc == 5 and dhs.ht_sync(t) == 5
        compare_tables(t, o, "missing key")
    finally:
        t.close()
        o.close()


def test_malformed_bag_offsets_are_reported():
    t = dhs.ht_create(8, "sgd")
    try:
        keys = dev(np.arange(10, dtype=np.int64))
        for offs in ([0, 5, 3, 10], [0, 4, 8, 9], [1, 4, 8, 10], [0, 4, 12, 10]):
            dhs.embbag_forward(t, keys, dev(np.array(offs, np.int64)))
            assert dhs.ht_sync(t) == 1, offs
            dhs.embbag_backward_update(t, keys, dev(np.array(offs, np.int64)),
                                       torch.zeros((3, 8), device="cuda"), 0.1)
            assert dhs.ht_sync(t) == 1, offs
    finally:
        t.close()


def test_row_limit_and_bad_arguments():
    t = dhs.ht_create(8, "sgd", block_rows=16, max_rows=100)
    try:
        dhs.ht_lookup_or_insert(t, dev(np.arange(90, dtype=np.int64)))
        with pytest.raises(dhs.DhsError) as e:
            dhs.ht_lookup_or_insert(t, dev(np.arange(1000, 1020, dtype=np.int64)))
        assert e.value.status == 4
        assert dhs.ht_size(t) == (90, 0)
        with pytest.raises(dhs.DhsError):
            dhs.embbag_backward_update(t, dev(np.arange(3, dtype=np.int64)), dev(np.array([0, 3], np.int64)),
                                       torch.zeros((1, 8), device="cuda"), float("nan"))
    finally:
        t.close()


def test_deterministic_across_runs():
    w = gen.small("hot_key")
    outs = []
    for _ in range(2):
        t = dhs.ht_create(w.dim, w.optimizer, block_rows=4096)
        try:
            for tids, ids in w.preinsert():
                dhs.ht_lookup_or_insert(t, dhs.dhs_pack_keys(dev(tids), dev(ids)))
            pooled = []
            for s in range(w.steps):
                b = w.batch(s)
                kg = dhs.dhs_pack_keys(dev(b.table_ids), dev(b.ids))
                og = dev(b.bag_offsets)
                pooled.append(host(dhs.embbag_forward(t, kg, og)))
                dhs.embbag_backward_update(t, kg, og, dev(w.grads(s, b.n_bags)), w.lr)
            k, rows, rc = dhs.ht_export(t)
            outs.append((np.concatenate(pooled), k, rows))
        finally:
            t.close()
    assert np.array_equal(outs[0][0], outs[1][0])
    assert np.array_equal(outs[0][1], outs[1][1])
    assert np.array_equal(outs[0][2], outs[1][2])
