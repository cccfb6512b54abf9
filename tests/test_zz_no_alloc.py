"""The allocation-free backward entry point (for callers that cannot allocate
device memory during a step) against the regular one.  Collected last, so
that a run stopping at the first failure has run every other test first."""
import numpy as np
import pytest
import torch

import dynamic_hashed_sparse_b200 as dhs
from tests.parity import assert_close, dev, host

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("opt", ["adagrad", "adam"])
def test_noalloc_backward_matches_regular_backward(opt):
    rng = np.random.default_rng(2024)
    dim = 64
    a = dhs.ht_create(dim, opt, block_rows=4096)
    b = dhs.ht_create(dim, opt, block_rows=4096)
    try:
        for call in range(2):  # two calls in a row: the shared scratch is reused
            nb = 20000
            lens = rng.integers(0, 6, size=nb)
            offs = np.concatenate([[0], np.cumsum(lens)]).astype(np.int64)
            n = int(offs[-1])
            assert n <= dhs.NOALLOC_MAX_KEYS
            keys = np.where(rng.random(n) < 0.2, rng.integers(0, 5, size=n),
                            rng.integers(0, 40000, size=n)).astype(np.int64) * 97 + 3
            kg, og = dev(keys), dev(offs)
            grad = dev(rng.standard_normal((nb, dim)).astype(np.float32))
            pa = host(dhs.embbag_forward(a, kg, og))
            pb = host(dhs.embbag_forward(b, kg, og))
            assert np.array_equal(pa, pb)
            dhs.embbag_backward_update(a, kg, og, grad, 0.01)
            dhs.embbag_backward_update_noalloc(b, kg, og, grad, 0.01)
            assert dhs.ht_sync(a) == 0 and dhs.ht_sync(b) == 0
            ka, ra, _ = dhs.ht_export(a)
            kb_, rb, _ = dhs.ht_export(b)
            np.testing.assert_array_equal(ka, kb_)
            assert_close(rb, ra, f"call {call}")
    finally:
        a.close()
        b.close()


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
