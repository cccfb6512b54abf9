"""Parity at the workloads' full sizes, in the launch configuration bench.py
uses (default block size, capacity reserved up front), against the CPU
oracle: in full where the oracle holds the whole table, else by key on the
batch's keys (rows the batch never touched are initial rows, a function of
the key, so a fresh oracle fed only the batch sees the same values)."""
import numpy as np
import pytest
import torch

import dynamic_hashed_sparse_b200 as dhs
from oracle import Oracle, pack_keys
from tests.parity import assert_close, dev, host
from workloads import gen

pytestmark = pytest.mark.gpu


def _pack(b):
    ko, rc = pack_keys(b.table_ids, b.ids)
    assert rc == 0
    kg = dhs.dhs_pack_keys(dev(b.table_ids), dev(b.ids))
    np.testing.assert_array_equal(host(kg), ko)
    return kg, ko


def _compare_full(t, o, what):
    gk, grows, rc = dhs.ht_export(t)
    ok_, orows = o.export()
    assert rc == 0
    np.testing.assert_array_equal(gk, ok_, err_msg=what)
    assert_close(grows[:, : t.dim], orows[:, : t.dim], what + " weights")
    if orows.shape[1] > t.dim and t.optimizer != "adagrad_rowwise":
        assert_close(grows[:, t.dim:], orows[:, t.dim:], what + " state")


def _run(w, steps, reserve):
    t = dhs.ht_create(w.dim, w.optimizer, block_rows=w.block_rows, eps=w.eps, beta1=w.beta1, beta2=w.beta2)
    o = Oracle(w.dim, w.optimizer, eps=w.eps, beta1=w.beta1, beta2=w.beta2)
    try:
        dhs.ht_reserve(t, reserve)
        for s in range(steps):
            b = w.batch(s)
            kg, ko = _pack(b)
            og = dev(b.bag_offsets)
            pg = dhs.embbag_forward(t, kg, og)
            po, _ = o.forward(ko, b.bag_offsets)
            assert_close(host(pg), po, f"{w.name} step {s} pooled")
            g = w.grads(s, b.n_bags)
            dhs.embbag_backward_update(t, kg, og, dev(g), w.lr)
            o.backward_update(ko, b.bag_offsets, g, w.lr)
            assert dhs.ht_sync(t) == 0
        _compare_full(t, o, w.name)
    finally:
        t.close()
        o.close()


def test_dlrm_merged_26_full_size():
    _run(gen.full("dlrm_merged_26"), steps=3, reserve=6_000_000)


def test_sequence_bags_full_size():
    _run(gen.full("sequence_bags"), steps=1, reserve=4_000_000)


def test_growth_stream_full_size():
    _run(gen.full("growth_stream"), steps=8, reserve=0)


def test_growth_stream_all_steps_key_map():
    """All 200 steps of the growth stream (forward + backward per step, the
    table growing on demand from empty to about 3.2e7 rows: many IDMap
    doublings and block appends) against the oracle's key -> row map over the
    same key stream.  The map depends on the keys alone, not on dim or on the
    optimizer, so the oracle runs at dim 4 and only its map is compared."""
    w = gen.full("growth_stream")
    t = dhs.ht_create(w.dim, w.optimizer, block_rows=w.block_rows, eps=w.eps, beta1=w.beta1, beta2=w.beta2)
    o = Oracle(4, "sgd")
    try:
        for s in range(w.steps):
            b = w.batch(s)
            kg, ko = _pack(b)
            og = dev(b.bag_offsets)
            dhs.embbag_forward(t, kg, og)
            dhs.embbag_backward_update(t, kg, og, w.torch_grads(s, b.n_bags, "cuda"), w.lr)
            o.lookup_or_insert(ko)
            if s % 50 == 49:
                assert dhs.ht_sync(t) == 0, f"step {s}"
        gk, _, rc = dhs.ht_export(t, rows=False)
        assert rc == 0
        ok_, _ = o.export()
        assert gk.size == ok_.size == w.inserted_before(w.steps)
        np.testing.assert_array_equal(gk, ok_)
        c = dhs.ht_counters(t)
        # the IDMap grew to hold the keys at load <= 0.5, and blocks cover every row
        assert c["slots"] >= 2 * gk.size and c["rehashes"] >= 5
        assert c["blocks"] >= -(-gk.size // w.block_rows)
    finally:
        t.close()
        o.close()


def test_tiny_uniform_full_size():
    _run(gen.full("tiny_uniform"), steps=10, reserve=0)


def test_hot_key_full_size_by_key():
    w = gen.full("hot_key")
    t = dhs.ht_create(w.dim, w.optimizer, block_rows=w.block_rows, eps=w.eps)
    try:
        rows_total = int(w.params["rows"])
        dhs.ht_reserve(t, rows_total + 1)
        for tids, ids in w.preinsert():
            dhs.ht_lookup_or_insert(t, dhs.dhs_pack_keys(dev(tids), dev(ids)))
        n_rows, rc = dhs.ht_size(t)
        assert rc == 0 and n_rows == rows_total
        # keys were inserted in rank order: rank r has row r - 1
        rng = np.random.default_rng(0)
        ranks = np.concatenate([np.arange(1, 101), rng.integers(1, rows_total + 1, size=5000)])
        keys, _ = pack_keys(np.zeros(ranks.size, np.int32), gen.rank_to_id(ranks - 1))
        np.testing.assert_array_equal(host(dhs.ht_lookup(t, dev(keys))), ranks - 1)

        b = w.batch(0)
        kg, ko = _pack(b)
        og = dev(b.bag_offsets)
        pg = host(dhs.embbag_forward(t, kg, og))
        g = w.grads(0, b.n_bags)
        dhs.embbag_backward_update(t, kg, og, dev(g), w.lr)
        assert dhs.ht_sync(t) == 0
        assert dhs.ht_size(t)[0] == rows_total  # nothing new

        o = Oracle(w.dim, w.optimizer, eps=w.eps)
        try:
            po, _ = o.forward(ko, b.bag_offsets)
            assert_close(pg, po, "hot_key pooled")
            o.backward_update(ko, b.bag_offsets, g, w.lr)
            uk = np.unique(ko)
            ref, missing = o.get_rows(uk)
            assert missing == 0
            got = host(dhs.ht_get_rows(t, dev(uk)))
            assert_close(got[:, : w.dim], ref[:, : w.dim], "hot_key weights")
            assert_close(got[:, w.dim:], ref[:, w.dim:], "hot_key accumulators")
            c = dhs.ht_counters(t)
            assert c["unique_updated"] == uk.size
        finally:
            o.close()
    finally:
        t.close()
