"""GPU parity of EmbeddingBag's other forms (mean pooling, per-sample
weights) through the C ABI, against the CPU oracle on the same seeded
inputs: pooled outputs, the key -> row map, and the updated rows and
optimizer state within the 1e-5 relative bar."""
import numpy as np
import pytest
import torch

import dynamic_hashed_sparse_b200 as dhs
from oracle import Oracle
from tests.parity import assert_close, dev, host

pytestmark = pytest.mark.gpu

DIMS = [4, 8, 12, 16, 32, 40, 64, 128, 132, 200, 260, 512]
OPTS = ["sgd", "adagrad", "adam", "adagrad_rowwise"]


def _compare(t, o, what):
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


def _step(t, o, keys, offs, grad, lr, form, psw):
    kw_g = dict(mode="mean") if form == "mean" else dict(per_sample_weights=dev(psw))
    kw_o = dict(mode="mean") if form == "mean" else dict(per_sample_weights=psw)
    kg, og = dev(keys), dev(offs)
    pg = host(dhs.embbag_forward_ex(t, kg, og, **kw_g))
    po, rc = o.forward(keys, offs, **kw_o)
    assert rc == 0
    assert_close(pg, po, f"{form} pooled")
    dhs.embbag_backward_update_ex(t, kg, og, dev(grad), lr, **kw_g)
    assert o.backward_update(keys, offs, grad, lr, **kw_o) == 0


@pytest.mark.parametrize("bags", ["long", "short"])
@pytest.mark.parametrize("form", ["mean", "weighted"])
@pytest.mark.parametrize("dim", DIMS)
def test_pooling_forms_every_width(dim, form, bags):
    """Every width (each forward and segment-kernel instantiation), both
    forms, short bags (fused probe + pool) and long bags (split forward); the
    optimizers rotate over the widths."""
    opt = OPTS[DIMS.index(dim) % 4]
    rng = np.random.default_rng(dim * 13 + (7 if form == "mean" else 0) + (100 if bags == "long" else 0))
    t = dhs.ht_create(dim, opt, block_rows=256)
    o = Oracle(dim, opt)
    try:
        for _ in range(3):
            nb = int(rng.integers(300, 900))
            lens = rng.integers(0, 12 if bags == "long" else 4, size=nb)
            lens[rng.integers(0, nb, size=5)] = 0
            offs = np.concatenate([[0], np.cumsum(lens)]).astype(np.int64)
            n = int(offs[-1])
            keys = np.where(rng.random(n) < 0.3, rng.integers(0, 8, size=n),
                            rng.integers(0, 3000, size=n)).astype(np.int64) * 1000003
            psw = rng.uniform(-1.5, 1.5, size=n).astype(np.float32)
            grad = rng.standard_normal((nb, dim)).astype(np.float32)
            _step(t, o, keys, offs, grad, 0.05, form, psw)
        assert dhs.ht_sync(t) == 0
        _compare(t, o, f"dim {dim} {opt} {form} {bags}")
    finally:
        t.close()
        o.close()


@pytest.mark.parametrize("form", ["mean", "weighted"])
@pytest.mark.parametrize("dim,opt", [(32, "adagrad"), (12, "adam"), (128, "sgd"), (64, "adagrad_rowwise")])
def test_pooling_forms_with_hot_keys_across_sort_chunks(dim, opt, form):
    """Hot keys whose runs span many sort chunks (finished by the long-run
    combine) with weighted / mean-scaled pieces, over 150k ids."""
    rng = np.random.default_rng(dim + len(opt))
    t = dhs.ht_create(dim, opt, block_rows=4096)
    o = Oracle(dim, opt)
    try:
        for _ in range(2):
            n = 150_000
            keys = np.where(rng.random(n) < 0.25, rng.integers(0, 6, size=n),
                            rng.integers(0, 20000, size=n)).astype(np.int64) * 31 + 7
            nb = n // 6
            cuts = np.sort(rng.integers(0, n + 1, size=nb - 1))
            offs = np.concatenate([[0], cuts, [n]]).astype(np.int64)
            psw = rng.uniform(-2.0, 2.0, size=n).astype(np.float32)
            grad = rng.standard_normal((nb, dim)).astype(np.float32)
            _step(t, o, keys, offs, grad, 0.01, form, psw)
        assert dhs.ht_sync(t) == 0
        _compare(t, o, f"hot {dim} {opt} {form}")
    finally:
        t.close()
        o.close()


def test_unit_weights_equal_the_plain_sum_bit_for_bit():
    rng = np.random.default_rng(9)
    a = dhs.ht_create(64, "adagrad")
    b = dhs.ht_create(64, "adagrad")
    try:
        for _ in range(2):
            nb = 5000
            lens = rng.integers(0, 10, size=nb)
            offs = dev(np.concatenate([[0], np.cumsum(lens)]).astype(np.int64))
            n = int(lens.sum())
            keys = dev(rng.integers(0, 30000, size=n).astype(np.int64))
            grad = dev(rng.standard_normal((nb, 64)).astype(np.float32))
            ones = torch.ones(n, dtype=torch.float32, device="cuda")
            pa = dhs.embbag_forward(a, keys, offs)
            pb = dhs.embbag_forward_ex(b, keys, offs, per_sample_weights=ones)
            assert torch.equal(pa, pb)
            dhs.embbag_backward_update(a, keys, offs, grad, 0.01)
            dhs.embbag_backward_update_ex(b, keys, offs, grad, 0.01, per_sample_weights=ones)
        ka, ra, _ = dhs.ht_export(a)
        kb, rb, _ = dhs.ht_export(b)
        assert np.array_equal(ka, kb) and np.array_equal(ra, rb)
    finally:
        a.close()
        b.close()


def test_mean_with_weights_and_bad_mode_are_rejected():
    t = dhs.ht_create(8, "sgd")
    try:
        keys = torch.arange(4, dtype=torch.int64, device="cuda")
        offs = torch.tensor([0, 2, 4], dtype=torch.int64, device="cuda")
        w = torch.ones(4, dtype=torch.float32, device="cuda")
        with pytest.raises(dhs.DhsError) as e:
            dhs.embbag_forward_ex(t, keys, offs, per_sample_weights=w, mode="mean")
        assert e.value.status == 1
        with pytest.raises(dhs.DhsError) as e:
            dhs.embbag_backward_update_ex(t, keys, offs, torch.zeros((2, 8), device="cuda"), 0.1,
                                          per_sample_weights=w, mode="mean")
        assert e.value.status == 1
        out = torch.empty((2, 8), device="cuda")
        rc = dhs.lib().embbag_forward_ex(t.handle, keys.data_ptr(), 4, offs.data_ptr(), 2, None, 7,
                                         out.data_ptr(), None)
        assert rc == 1
        assert dhs.ht_size(t) == (0, 0)  # nothing ran
    finally:
        t.close()
