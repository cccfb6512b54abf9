"""The allocation-free backward entry point, for callers that cannot allocate
device memory while their training steps run (a runtime that forbids
cudaMalloc once its loop starts, or one that hands this library only buffers
it owns).  Its scratch is one fixed device array inside the library.

Each case runs two calls in a row (the shared scratch keeps the previous
call's contents), compares the table against the CPU oracle and against the
regular embbag_backward_update on the same inputs, and checks through a
counting allocator that the call requested no device memory.  Collected
last, so that a run stopping at the first failure has run every other test
first."""
import numpy as np
import pytest
import torch

import dynamic_hashed_sparse_b200 as dhs
from oracle import Oracle
from tests.parity import assert_close, dev, host

pytestmark = pytest.mark.gpu


def _batch(rng, n_target, nb, hot_frac):
    """nb bags holding exactly n_target ids; hot_frac of them from 5 hot keys
    (runs that span many sort chunks), the rest from 40,000 keys."""
    cuts = np.sort(rng.integers(0, n_target + 1, size=nb - 1))
    offs = np.concatenate([[0], cuts, [n_target]]).astype(np.int64)
    keys = np.where(rng.random(n_target) < hot_frac, rng.integers(0, 5, size=n_target),
                    rng.integers(0, 40000, size=n_target)).astype(np.int64) * 97 + 3
    return keys, offs


CASES = [
    # dim, optimizer, ids of the first call, ids of the second call
    (128, "adagrad", dhs.NOALLOC_MAX_KEYS, 70_001),   # the key limit at the widest row
    (128, "adam", 90_000, dhs.NOALLOC_MAX_KEYS),
    (64, "adagrad", 50_000, 110_000),
    (16, "sgd", dhs.NOALLOC_MAX_KEYS, 20_000),        # the narrow-row segment kernel
    (16, "adagrad_rowwise", 60_000, 120_000),
]


@pytest.mark.parametrize("dim,opt,n1,n2", CASES)
def test_noalloc_backward_matches_oracle_and_regular_backward(dim, opt, n1, n2):
    rng = np.random.default_rng(dim * 31 + n1 % 977)
    counting = dhs.TorchAllocator()
    a = dhs.ht_create(dim, opt, block_rows=4096)
    b = dhs.ht_create(dim, opt, block_rows=4096, allocator=counting)
    o = Oracle(dim, opt)
    try:
        for call, n in enumerate((n1, n2)):  # two calls in a row: the shared scratch is reused
            nb = n // 3 + 1
            keys, offs = _batch(rng, n, nb, 0.15)
            grad = rng.standard_normal((nb, dim)).astype(np.float32)
            kg, og, gg = dev(keys), dev(offs), dev(grad)
            pa = host(dhs.embbag_forward(a, kg, og))
            pb = host(dhs.embbag_forward(b, kg, og))
            po, _ = o.forward(keys, offs)
            assert np.array_equal(pa, pb)
            assert_close(pb, po, f"call {call} pooled")
            torch.cuda.synchronize()
            allocs_before = counting.alloc_calls
            dhs.embbag_backward_update_noalloc(b, kg, og, gg, 0.01)
            torch.cuda.synchronize()
            assert counting.alloc_calls == allocs_before, "the allocation-free call allocated"
            dhs.embbag_backward_update(a, kg, og, gg, 0.01)
            o.backward_update(keys, offs, grad, 0.01)
            assert dhs.ht_sync(a) == 0 and dhs.ht_sync(b) == 0
            ka, ra, _ = dhs.ht_export(a)
            kb_, rb, _ = dhs.ht_export(b)
            ko, ro = o.export()
            np.testing.assert_array_equal(kb_, ko)
            np.testing.assert_array_equal(ka, ko)
            assert_close(rb[:, :dim], ro[:, :dim], f"call {call} weights vs oracle")
            if opt == "adagrad_rowwise":
                assert_close(rb[:, dim], ro[:, dim], f"call {call} row accumulator vs oracle")
            elif ro.shape[1] > dim:
                assert_close(rb[:, dim:], ro[:, dim:], f"call {call} state vs oracle")
            assert_close(rb, ra, f"call {call} vs the regular backward")
        assert counting.alloc_calls > 0  # the table did use the allocator for its own storage
    finally:
        a.close()
        b.close()
        o.close()


def test_noalloc_rejects_calls_beyond_its_limits():
    t = dhs.ht_create(16, "sgd")
    wide = dhs.ht_create(256, "sgd")
    try:
        n = dhs.NOALLOC_MAX_KEYS + 1
        keys = torch.arange(n, dtype=torch.int64, device="cuda")
        offs = torch.tensor([0, n], dtype=torch.int64, device="cuda")
        with pytest.raises(dhs.DhsError) as e:
            dhs.embbag_backward_update_noalloc(t, keys, offs, torch.zeros((1, 16), device="cuda"), 0.1)
        assert e.value.status == 1
        small = keys[:10]
        offs10 = torch.tensor([0, 10], dtype=torch.int64, device="cuda")
        with pytest.raises(dhs.DhsError) as e:
            dhs.embbag_backward_update_noalloc(wide, small, offs10, torch.zeros((1, 256), device="cuda"), 0.1)
        assert e.value.status == 1
    finally:
        t.close()
        wide.close()
