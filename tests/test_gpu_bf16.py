"""GPU parity of tables with bf16 weights and fp32 optimizer state, through
the C ABI, against the CPU oracle's bf16 table on the same seeded inputs:
pooled outputs, the key -> row map, updated weights (which must sit on the
bf16 grid) and optimizer state."""
import numpy as np
import pytest
import torch

import dynamic_hashed_sparse_b200 as dhs
from oracle import Oracle
from tests.parity import assert_close, dev, host

pytestmark = pytest.mark.gpu

# dims reaching each bf16 pool shape (16-byte units of 8 weights per lane:
# groups of 4, 8, 16, 32 lanes, 1 or 2 units each) and each lane width of the
# warp segment kernel (1..16 columns per lane)
DIMS = [32, 40, 64, 128, 136, 256, 264, 512]
OPTS = ["sgd", "adagrad", "adam", "adagrad_rowwise"]


def _pair(dim, opt, block_rows=256, **kw):
    t = dhs.ht_create(dim, opt, block_rows=block_rows, weights="bf16", **kw)
    o = Oracle(dim, opt, storage="bf16")
    return t, o


def _compare(t, o, what):
    gk, grows, rc = dhs.ht_export(t)
    ok_, orows = o.export()
    assert rc == 0, f"{what}: latched status {rc}"
    np.testing.assert_array_equal(gk, ok_, err_msg=f"{what}: key -> row map")
    d = t.dim
    w = grows[:, :d]
    # every stored weight is a bf16 value
    assert np.array_equal(w.view(np.uint32) & np.uint32(0xffff), np.zeros_like(w, np.uint32)), f"{what}: off grid"
    assert_close(w, orows[:, :d], f"{what}: weights")
    if t.optimizer == "adagrad_rowwise":
        assert_close(grows[:, d], orows[:, d], f"{what}: row accumulator")
    elif orows.shape[1] > d:
        assert_close(grows[:, d:], orows[:, d:], f"{what}: optimizer state")


def _batch(rng, bags):
    nb = int(rng.integers(300, 900))
    lens = rng.integers(0, 12 if bags == "long" else 4, size=nb)
    lens[rng.integers(0, nb, size=5)] = 0
    offs = np.concatenate([[0], np.cumsum(lens)]).astype(np.int64)
    n = int(offs[-1])
    keys = np.where(rng.random(n) < 0.3, rng.integers(0, 8, size=n),
                    rng.integers(0, 3000, size=n)).astype(np.int64) * 1000003
    return nb, offs, keys


@pytest.mark.parametrize("bags", ["long", "short"])
@pytest.mark.parametrize("opt", OPTS)
@pytest.mark.parametrize("dim", DIMS)
def test_bf16_every_width_and_optimizer(dim, opt, bags):
    rng = np.random.default_rng(dim * 5 + len(opt) + (50 if bags == "short" else 0))
    t, o = _pair(dim, opt)
    try:
        for _ in range(3):
            nb, offs, keys = _batch(rng, bags)
            grad = rng.standard_normal((nb, dim)).astype(np.float32)
            kg, og = dev(keys), dev(offs)
            pg = host(dhs.embbag_forward(t, kg, og))
            po, _ = o.forward(keys, offs)
            assert_close(pg, po, "bf16 pooled")
            dhs.embbag_backward_update(t, kg, og, dev(grad), 0.05)
            o.backward_update(keys, offs, grad, 0.05)
        assert dhs.ht_sync(t) == 0
        _compare(t, o, f"bf16 dim {dim} {opt} {bags}")
    finally:
        t.close()
        o.close()


@pytest.mark.parametrize("form", ["mean", "weighted"])
@pytest.mark.parametrize("dim,opt", [(32, "adam"), (128, "adagrad"), (264, "sgd")])
def test_bf16_pooling_forms(dim, opt, form):
    rng = np.random.default_rng(dim + 3)
    t, o = _pair(dim, opt)
    try:
        for bags in ("long", "short"):
            nb, offs, keys = _batch(rng, bags)
            psw = rng.uniform(-1.5, 1.5, size=keys.size).astype(np.float32)
            grad = rng.standard_normal((nb, dim)).astype(np.float32)
            kw_g = dict(mode="mean") if form == "mean" else dict(per_sample_weights=dev(psw))
            kw_o = dict(mode="mean") if form == "mean" else dict(per_sample_weights=psw)
            kg, og = dev(keys), dev(offs)
            pg = host(dhs.embbag_forward_ex(t, kg, og, **kw_g))
            po, _ = o.forward(keys, offs, **kw_o)
            assert_close(pg, po, f"bf16 {form} pooled")
            dhs.embbag_backward_update_ex(t, kg, og, dev(grad), 0.02, **kw_g)
            o.backward_update(keys, offs, grad, 0.02, **kw_o)
        assert dhs.ht_sync(t) == 0
        _compare(t, o, f"bf16 {form} dim {dim}")
    finally:
        t.close()
        o.close()


@pytest.mark.parametrize("dim,opt", [(64, "adagrad"), (128, "adam")])
def test_bf16_hot_keys_and_the_allocation_free_backward(dim, opt):
    """Hot keys whose runs span many sort chunks (long-run combine on bf16
    rows), once through the regular backward, once through the
    allocation-free one."""
    rng = np.random.default_rng(dim)
    t, o = _pair(dim, opt, block_rows=4096)
    try:
        for call in range(2):
            n = 120_000
            keys = np.where(rng.random(n) < 0.3, rng.integers(0, 5, size=n),
                            rng.integers(0, 20000, size=n)).astype(np.int64) * 17 + 1
            nb = n // 4
            cuts = np.sort(rng.integers(0, n + 1, size=nb - 1))
            offs = np.concatenate([[0], cuts, [n]]).astype(np.int64)
            grad = rng.standard_normal((nb, dim)).astype(np.float32)
            kg, og, gg = dev(keys), dev(offs), dev(grad)
            pg = host(dhs.embbag_forward(t, kg, og))
            po, _ = o.forward(keys, offs)
            assert_close(pg, po, "bf16 hot pooled")
            if call == 0:
                dhs.embbag_backward_update(t, kg, og, gg, 0.01)
            else:
                dhs.embbag_backward_update_noalloc(t, kg, og, gg, 0.01)
            o.backward_update(keys, offs, grad, 0.01)
            assert dhs.ht_sync(t) == 0
            _compare(t, o, f"bf16 hot call {call}")
    finally:
        t.close()
        o.close()


def test_bf16_rows_need_a_multiple_of_8_of_at_least_32():
    for dim in (12, 16, 24, 36):
        with pytest.raises(dhs.DhsError) as e:
            dhs.ht_create(dim, "sgd", weights="bf16")
        assert e.value.status == 6  # unsupported
    t = dhs.ht_create(48, "adam", weights="bf16")
    try:
        assert t.stride == 48 + 96  # exported rows: weights widened, then the state
    finally:
        t.close()
