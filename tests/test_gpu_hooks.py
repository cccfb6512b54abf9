"""GPU parity of feature admission and eviction (the HashtableHook readings)
through the C ABI, against the CPU oracle on the same seeded inputs: the key
-> row map (free rows included, key -1), pooled outputs, updated rows of live
keys, lookups of keys not admitted, and the live-row count."""
import numpy as np
import pytest
import torch

import dynamic_hashed_sparse_b200 as dhs
from oracle import Oracle
from tests.parity import assert_close, dev, host

pytestmark = pytest.mark.gpu


def _pair(dim, opt, admit, track, block_rows=1024):
    t = dhs.ht_create(dim, opt, block_rows=block_rows)
    dhs.ht_set_hooks(t, admit_threshold=admit, track_access=track)
    o = Oracle(dim, opt)
    o.set_hooks(admit_threshold=admit, track_access=track)
    return t, o


def _compare(t, o, what):
    gk, grows, rc = dhs.ht_export(t)
    ok_, orows = o.export()
    assert rc == 0, f"{what}: latched status {rc}"
    np.testing.assert_array_equal(gk, ok_, err_msg=f"{what}: key -> row map")
    live = ok_ >= 0
    d = t.dim
    assert_close(grows[live][:, :d], orows[live][:, :d], f"{what}: weights")
    if t.optimizer != "adagrad_rowwise" and orows.shape[1] > d:
        assert_close(grows[live][:, d:], orows[live][:, d:], f"{what}: state")
    n_live, rc = dhs.ht_live_rows(t)
    assert rc == 0 and n_live == o.live, (n_live, o.live)


def _batch(rng, universe, bags, short):
    lens = rng.integers(0, 4 if short else 12, size=bags)
    offs = np.concatenate([[0], np.cumsum(lens)]).astype(np.int64)
    n = int(offs[-1])
    # skewed frequencies: a few keys often, most rarely
    keys = (rng.zipf(1.3, size=n) % universe).astype(np.int64) * 7919 + 3
    return keys, offs


def _step(t, o, keys, offs, dim, rng, lr=0.05):
    kg, og = dev(keys), dev(offs)
    pg = host(dhs.embbag_forward(t, kg, og))
    po, rc = o.forward(keys, offs)
    assert rc == 0
    assert_close(pg, po, "pooled")
    grad = rng.standard_normal((offs.size - 1, dim)).astype(np.float32)
    dhs.embbag_backward_update(t, kg, og, dev(grad), lr)
    assert o.backward_update(keys, offs, grad, lr) == 0


@pytest.mark.parametrize("short", [False, True])
@pytest.mark.parametrize("admit", [2, 3])
@pytest.mark.parametrize("dim,opt", [(16, "adagrad"), (64, "adam")])
def test_admission(dim, opt, admit, short):
    rng = np.random.default_rng(admit * 10 + dim + short)
    t, o = _pair(dim, opt, admit, track=False)
    try:
        for step in range(6):
            keys, offs = _batch(rng, 5000, 700, short)
            _step(t, o, keys, offs, dim, rng)
            assert dhs.ht_sync(t) == 0, f"step {step}"
        _compare(t, o, f"admission {admit}")
        # lookups: keys not admitted give -1, admitted ones their rows
        probe = np.unique(keys)
        np.testing.assert_array_equal(host(dhs.ht_lookup(t, dev(probe))), o.lookup(probe))
        assert (o.lookup(probe) == -1).any() and (o.lookup(probe) >= 0).any()
        # lookup_or_insert counts occurrences too (one more call)
        off_g = host(dhs.ht_lookup_or_insert(t, dev(keys)))
        off_o, _ = o.lookup_or_insert(keys)
        np.testing.assert_array_equal(off_g, off_o)
        _compare(t, o, f"admission {admit} after lookup_or_insert")
    finally:
        t.close()
        o.close()


@pytest.mark.parametrize("admit", [1, 2])
@pytest.mark.parametrize("dim,opt", [(8, "sgd"), (32, "adagrad_rowwise"), (128, "adagrad")])
def test_eviction_and_row_reuse(dim, opt, admit):
    """Calls over a drifting key range, evictions with different windows, new
    keys reusing free rows, and enough keys that the IDMap grows (rehash with
    tombstones, counts and stamps) between evictions."""
    rng = np.random.default_rng(dim + admit)
    t, o = _pair(dim, opt, admit, track=True, block_rows=4096)
    try:
        base = 0
        for step in range(12):
            # a drifting key range, so that old keys go idle; small calls
            # until the first eviction (step 3) leaves tombstones, then calls
            # whose claimed slots outgrow the initial IDMap of 32,768 keys,
            # so that the rehash meets tombstones, counts and stamps
            universe, bags = (3000, 1000) if step <= 3 else (30000, 6000)
            keys, offs = _batch(rng, universe, bags, short=step % 2 == 0)
            keys = keys + base
            base += universe * 7919 // 3
            _step(t, o, keys, offs, dim, rng)
            if step in (3, 6, 9, 10):
                max_idle = {3: 1, 6: 2, 9: 0, 10: 3}[step]
                assert dhs.ht_evict(t, max_idle) == o.evict(max_idle)
                _compare(t, o, f"evict at step {step}")
        assert dhs.ht_sync(t) == 0
        _compare(t, o, "final")
        c = dhs.ht_counters(t)
        assert c["rehashes"] >= 1
    finally:
        t.close()
        o.close()


def test_hooks_argument_rules():
    t = dhs.ht_create(8, "sgd")
    try:
        dhs.ht_lookup_or_insert(t, dev(np.arange(5, dtype=np.int64)))
        with pytest.raises(dhs.DhsError) as e:
            dhs.ht_set_hooks(t, admit_threshold=2)
        assert e.value.status == 1  # only on a new table
        with pytest.raises(dhs.DhsError) as e:
            dhs.ht_evict(t, 1)
        assert e.value.status == 1  # needs access tracking
    finally:
        t.close()
    t = dhs.ht_create(8, "sgd")
    try:
        dhs.ht_set_hooks(t, track_access=True)
        with pytest.raises(dhs.DhsError):
            dhs.ht_set_hooks(t, track_access=True)  # once
        assert dhs.ht_evict(t, 0) == 0  # nothing to evict yet
    finally:
        t.close()
