"""Pins of the CPU oracle to facts outside itself (no GPU needed).

Each test ties one part of the oracle to something the pages or mathematics
fix: a worked example, a library routine that computes the same definition,
a closed form, brute force over a tiny id range, or published test values.
"""
import json
import math
import os
from fractions import Fraction

import numpy as np
import pytest
import torch

from oracle import Oracle, init_row, pack_keys, round_bf16, splitmix64_outputs
from tests.conftest import GOLDEN

SCALE = np.float32(0.05) * np.float32(2.0 ** -23)


def _golden(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f) if name.endswith(".json") else f.read()


def _ulp(x):
    x = np.abs(np.asarray(x, np.float32))
    return np.spacing(x)


# --- splitmix64 / row initialisation -------------------------------------------------

def test_splitmix64_published_values():
    txt = _golden("splitmix64_seed0.txt")
    want = [int(l, 16) for l in txt.splitlines() if l.strip() and not l.startswith("#")]
    assert splitmix64_outputs(0, len(want)) == want


def test_init_row_range_grid_and_moments():
    keys = np.arange(4000, dtype=np.int64) * 7919 + 12345
    rows = np.stack([init_row(int(k), 32) for k in keys])
    assert rows.min() >= -0.05 and rows.max() < 0.05
    # every value is the fp32 product of an integer in [-2^23, 2^23) and the step
    u = np.round(rows.astype(np.float64) / float(SCALE))
    assert np.array_equal(u.astype(np.float32) * SCALE, rows)
    assert u.min() >= -(2 ** 23) and u.max() < 2 ** 23
    # uniform on [-0.05, 0.05): mean 0, variance 0.05^2/3 (128k samples)
    assert abs(rows.mean()) < 3 * 0.05 / math.sqrt(3 * rows.size) * 1.5
    assert abs(rows.var() / (0.05 ** 2 / 3) - 1) < 0.02
    # elements within a row and across keys are not visibly correlated
    c = np.corrcoef(rows[:, 0], rows[:, 1])[0, 1]
    assert abs(c) < 0.05


def test_init_row_uses_successive_outputs_of_the_key_stream():
    # element j is the (j+1)-th output of the generator seeded with the key;
    # a shifted or reused output would break this
    for key in (0, 1, 2 ** 40 + 3, (5 << 48) | 77):
        outs = splitmix64_outputs(key, 8)
        row = init_row(key, 8)
        for j, z in enumerate(outs):
            u = np.int64(z >> 40) - 2 ** 23
            assert row[j] == np.float32(u) * SCALE


def test_init_independent_of_insertion_order():
    keys = np.array([9, 3, 77, 2 ** 47, 5], np.int64)
    a, b = Oracle(8), Oracle(8)
    a.lookup_or_insert(keys)
    b.lookup_or_insert(keys[::-1])
    ra, _ = a.get_rows(keys)
    rb, _ = b.get_rows(keys)
    assert np.array_equal(ra, rb)


# --- key -> row mapping ---------------------------------------------------------------

def test_mapping_is_first_occurrence_order_brute_force():
    rng = np.random.default_rng(5)
    o = Oracle(4)
    seen = []
    for step in range(6):
        keys = rng.integers(0, 50, size=int(rng.integers(0, 40)), dtype=np.int64)
        off, rc = o.lookup_or_insert(keys)
        assert rc == 0
        seen.extend(keys.tolist())
        # independent computation: distinct keys ordered by first index in the
        # concatenated stream (np.unique + argsort of first indices)
        allk = np.array(seen, np.int64)
        uniq, first = np.unique(allk, return_index=True)
        order = uniq[np.argsort(first)]
        rank = {int(k): r for r, k in enumerate(order)}
        assert off.tolist() == [rank[int(k)] for k in keys]
        assert o.size == len(order)


def test_read_only_lookup_brute_force():
    """orc_lookup: a hit gives the offset the first-occurrence enumeration
    assigned (computed here by a plain dict over the stream), an absent or
    negative key gives -1, and nothing is inserted."""
    rng = np.random.default_rng(11)
    o = Oracle(4)
    stream = []
    for _ in range(4):
        keys = rng.integers(0, 300, size=int(rng.integers(1, 120)), dtype=np.int64) * 13 + 5
        o.lookup_or_insert(keys)
        stream.extend(keys.tolist())
    rank = {}
    for k in stream:
        rank.setdefault(k, len(rank))
    size = o.size
    probe = np.concatenate([np.array(stream[::3], np.int64),
                            np.arange(0, 4000, 7, dtype=np.int64),  # mostly absent
                            np.array([-1, -5, -(2 ** 62)], np.int64)])
    got = o.lookup(probe)
    want = [rank.get(int(k), -1) if k >= 0 else -1 for k in probe]
    assert got.tolist() == want
    assert (got == -1).sum() > 100 and (got >= 0).sum() > 100
    assert o.size == size
    # a hit is exactly what lookup_or_insert returns for the same key
    off, _ = o.lookup_or_insert(np.array(stream[:50], np.int64))
    np.testing.assert_array_equal(o.lookup(np.array(stream[:50], np.int64)), off)


def test_get_rows_absent_keys_are_nan_and_counted():
    o = Oracle(8, "adam")
    present = np.array([3, 10, 77], np.int64)
    o.lookup_or_insert(present)
    _, rows = o.export()
    ask = np.array([10, 999, 3, -4, 77, 1000], np.int64)
    got, missing = o.get_rows(ask)
    assert missing == 3
    assert got.shape == (6, o.stride)
    for i in (1, 3, 5):
        assert np.all(np.isnan(got[i]))
    # present rows are the stored rows (weights = init of the key, state 0)
    np.testing.assert_array_equal(got[0], rows[1])
    np.testing.assert_array_equal(got[2], rows[0])
    np.testing.assert_array_equal(got[4], rows[2])
    np.testing.assert_array_equal(got[0, :8], init_row(10, 8))
    assert np.all(got[[0, 2, 4], 8:] == 0)


def test_modulo_collision_ids_get_distinct_rows():
    g = _golden("modulo_collision.json")
    a, b = g["ids"]
    assert a % g["modulus"] == g["residue"] == b % g["modulus"]
    o = Oracle(16)
    off, _ = o.lookup_or_insert(np.array([a, b, a], np.int64))
    assert off[0] != off[1] and off[2] == off[0]
    rows, _ = o.get_rows(np.array([a, b], np.int64))
    assert not np.array_equal(rows[0], rows[1])


def test_pack_keys_layout_and_validation():
    t = np.array([0, 1, 25, 32767, -1, 3], np.int32)
    i = np.array([5, 5, 2 ** 48 - 1, 0, 1, 2 ** 48], np.int64)
    k, rc = pack_keys(t, i)
    assert k[0] == 5 and k[1] == (1 << 48) + 5
    assert k[2] == (25 << 48) + 2 ** 48 - 1 and k[3] == 32767 << 48
    assert k[4] == -1 and k[5] == -1 and rc != 0
    assert np.all(k[:4] >= 0)


# --- forward -----------------------------------------------------------------------

def test_forward_matches_torch_embedding_bag_sum():
    d = 12
    o = Oracle(d)
    o.lookup_or_insert(np.arange(64, dtype=np.int64))  # key k -> row k
    _, rows = o.export()
    weight = torch.from_numpy(rows[:, :d].copy())
    rng = np.random.default_rng(1)
    lens = rng.integers(0, 9, size=37)
    lens[[0, 5, 36]] = 0  # empty bags, including the first and the last
    offs = np.concatenate([[0], np.cumsum(lens)]).astype(np.int64)
    keys = rng.integers(0, 64, size=int(offs[-1]), dtype=np.int64)
    pooled, rc = o.forward(keys, offs)
    assert rc == 0
    ref = torch.nn.functional.embedding_bag(torch.from_numpy(keys), weight,
                                            torch.from_numpy(offs[:-1]), mode="sum").numpy()
    assert np.all(pooled[lens == 0] == 0)
    np.testing.assert_allclose(pooled, ref, rtol=1e-6, atol=1e-7)


def _dense_case(d, seed, max_len=9):
    """An oracle whose keys 0..63 map to rows 0..63, those rows as a torch
    weight, and a batch of bags (empty ones included) over the 64 keys."""
    o = Oracle(d)
    o.lookup_or_insert(np.arange(64, dtype=np.int64))
    _, rows = o.export()
    rng = np.random.default_rng(seed)
    lens = rng.integers(0, max_len, size=41)
    lens[[0, 7, 40]] = 0
    offs = np.concatenate([[0], np.cumsum(lens)]).astype(np.int64)
    keys = rng.integers(0, 64, size=int(offs[-1]), dtype=np.int64)
    psw = rng.uniform(-2.0, 2.0, size=keys.size).astype(np.float32)
    return o, torch.from_numpy(rows[:, :d].copy()), lens, offs, keys, psw


def test_mean_and_weighted_forward_match_torch_embedding_bag():
    d = 12
    o, weight, lens, offs, keys, psw = _dense_case(d, 2)
    tk, to = torch.from_numpy(keys), torch.from_numpy(offs[:-1])
    mean, rc = o.forward(keys, offs, mode="mean")
    assert rc == 0
    ref = torch.nn.functional.embedding_bag(tk, weight, to, mode="mean").numpy()
    np.testing.assert_allclose(mean, ref, rtol=2e-6, atol=1e-7)
    assert np.all(mean[lens == 0] == 0)
    wsum, rc = o.forward(keys, offs, per_sample_weights=psw)
    assert rc == 0
    ref = torch.nn.functional.embedding_bag(tk, weight, to, mode="sum",
                                            per_sample_weights=torch.from_numpy(psw)).numpy()
    np.testing.assert_allclose(wsum, ref, rtol=2e-6, atol=2e-7)


def test_pooling_mode_special_cases_are_exact():
    d = 8
    o, _, lens, offs, keys, psw = _dense_case(d, 3)
    plain, _ = o.forward(keys, offs)
    ones, _ = o.forward(keys, offs, per_sample_weights=np.ones(keys.size, np.float32))
    assert np.array_equal(ones, plain)
    # a power-of-two weight scales every product and every partial sum exactly
    twos, _ = o.forward(keys, offs, per_sample_weights=np.full(keys.size, 2.0, np.float32))
    assert np.array_equal(twos, 2 * plain)
    # mean over bags of one id is the id's row
    single = np.arange(keys.size + 1, dtype=np.int64)
    a, _ = o.forward(keys, single, mode="mean")
    b, _ = o.forward(keys, single)
    assert np.array_equal(a, b)
    # mean pooling takes no per-sample weights (rejected, nothing computed)
    _, rc = o.forward(keys, offs, per_sample_weights=psw, mode="mean")
    assert rc == 1
    assert o.backward_update(keys, offs, np.ones((lens.size, d), np.float32), 0.1,
                             per_sample_weights=psw, mode="mean") == 1


@pytest.mark.parametrize("opt", ["sgd", "adagrad"])
@pytest.mark.parametrize("form", ["mean", "weighted"])
def test_mean_and_weighted_backward_match_torch_autograd(form, opt):
    """A dense table's gradient from torch autograd through embedding_bag,
    then torch's SGD / Adagrad step (rows without gradient do not move).
    Torch sums a row's occurrence gradients in fp32 (the oracle sums them
    exactly in fp64): with up to ~10 occurrences of |w g| <= ~4 per step the
    fp32 sum is off by at most ~10 * 4 * 6e-8 = 2.4e-6, times lr 0.05 over
    3 steps about 4e-7 on a weight, hence the absolute term next to the
    relative bar.  A dropped weight or mean divisor moves weights by ~1e-2."""
    d, lr = 12, 0.05
    o = Oracle(d, opt)
    o.lookup_or_insert(np.arange(64, dtype=np.int64))
    _, rows = o.export()
    _, _, lens, offs, keys, psw = _dense_case(d, 4)
    rng = np.random.default_rng(5)
    weight = torch.nn.Parameter(torch.from_numpy(rows[:, :d].copy()))
    torch_opt = torch.optim.SGD([weight], lr=lr) if opt == "sgd" else \
        torch.optim.Adagrad([weight], lr=lr, eps=1e-8)
    for _ in range(3):
        grad = rng.standard_normal((lens.size, d)).astype(np.float32)
        kw = dict(mode="mean") if form == "mean" else dict(per_sample_weights=psw)
        assert o.backward_update(keys, offs, grad, lr, **kw) == 0
        tkw = dict(mode="mean") if form == "mean" else dict(mode="sum", per_sample_weights=torch.from_numpy(psw))
        out = torch.nn.functional.embedding_bag(torch.from_numpy(keys), weight, torch.from_numpy(offs[:-1]), **tkw)
        torch_opt.zero_grad()
        (out * torch.from_numpy(grad)).sum().backward()
        torch_opt.step()
    _, got = o.export()
    want = weight.detach().numpy()
    assert np.all(np.abs(got[:, :d] - want) <= 1e-5 * np.abs(want) + 4e-7)
    touched = np.unique(keys)
    untouched = np.setdiff1d(np.arange(64), touched)
    assert np.array_equal(got[untouched, :d], rows[untouched, :d])


def test_mean_gradient_closed_form():
    """Each key in exactly one bag of length L: its gradient is fl(g / L)
    (the exact quotient, rounded once), so SGD moves it by fl(lr * fl(g / L))."""
    d, lr = 4, 0.5
    o = Oracle(d, "sgd")
    lens = np.array([1, 3, 7, 2], np.int64)
    keys = np.arange(lens.sum(), dtype=np.int64) + 100
    offs = np.concatenate([[0], np.cumsum(lens)]).astype(np.int64)
    o.lookup_or_insert(keys)
    _, before = o.export()
    g = np.array([[1.0, -3.0, 0.1, 7.0]] * lens.size, np.float32) * np.arange(1, 5, dtype=np.float32)[:, None]
    assert o.backward_update(keys, offs, g, lr, mode="mean") == 0
    _, after = o.export()
    bag = np.repeat(np.arange(lens.size), lens)
    gk = (g[bag].astype(np.float64) / lens[bag][:, None]).astype(np.float32)
    want = before[:, :d] - np.float32(lr) * gk
    assert np.array_equal(after[:, :d], want)


def test_merged_tables_equal_separate_tables():
    g = _golden("dlrm_shape_example.json")
    bsz, d, T = g["batch"], g["dim"], g["tables"]
    rng = np.random.default_rng(3)
    raw = rng.integers(0, 6, size=(bsz, T)).astype(np.int64)  # same raw ids recur across tables
    tids = np.broadcast_to(np.arange(T, dtype=np.int32), (bsz, T)).copy()
    keys, rc = pack_keys(tids.reshape(-1), raw.reshape(-1))
    assert rc == 0
    merged = Oracle(d)
    out, _ = merged.forward(keys, np.arange(bsz * T + 1, dtype=np.int64))
    out = out.reshape(bsz, T, d)
    for t in range(T):
        sep = Oracle(d)
        kt, _ = pack_keys(np.full(bsz, t, np.int32), raw[:, t])
        ot, _ = sep.forward(kt, np.arange(bsz + 1, dtype=np.int64))
        assert list(ot.shape) == g["per_table_shape"]
        assert np.array_equal(out[:, t, :], ot)
    # equal raw ids in different tables are different rows
    assert merged.size == len({(t, int(raw[s, t])) for s in range(bsz) for t in range(T)})


# --- backward ----------------------------------------------------------------------

def test_worked_sgd_example():
    g = _golden("worked_sgd_example.json")
    n, d, lr, ids = g["num_embeddings"], g["dim"], g["lr"], g["ids"]
    o = Oracle(d, "sgd")
    o.lookup_or_insert(np.arange(n, dtype=np.int64))
    _, before = o.export()
    keys = np.array(ids, np.int64)
    offs = np.arange(len(ids) + 1, dtype=np.int64)
    vecs, _ = o.forward(keys, offs)
    grad = 2.0 * vecs                     # dL/de for L = sum e^2
    assert o.backward_update(keys, offs, grad, lr) == 0
    _, after = o.export()
    for r in range(n):
        if r in ids:
            want = np.float32(g["touched_factor"]) * before[r]
            assert np.all(np.abs(after[r] - want) <= 2 * _ulp(want))
        else:
            assert np.array_equal(after[r], before[r])
    # the same step through torch nn.Embedding + optim.SGD
    emb = torch.nn.Embedding(n, d)
    with torch.no_grad():
        emb.weight.copy_(torch.from_numpy(before))
    opt = torch.optim.SGD(emb.parameters(), lr=lr)
    loss = (emb(torch.tensor(ids)) ** 2).sum()
    opt.zero_grad()
    loss.backward()
    opt.step()
    w = emb.weight.detach().numpy()
    assert np.all(np.abs(after - w) <= _ulp(w))


@pytest.mark.parametrize("opt", ["sgd", "adagrad"])
def test_dense_table_equivalence(opt):
    """Sparse touched-rows-only steps equal dense torch steps over keys [0, 64):
    a dense SGD/Adagrad step with zero gradient leaves a row unchanged."""
    d, V, lr, eps = 8, 64, 0.05, 1e-8
    o = Oracle(d, opt, eps=eps)
    o.lookup_or_insert(np.arange(V, dtype=np.int64))
    _, rows = o.export()
    W = torch.nn.Parameter(torch.from_numpy(rows[:, :d].copy()))
    topt = (torch.optim.SGD([W], lr=lr) if opt == "sgd"
            else torch.optim.Adagrad([W], lr=lr, eps=eps, initial_accumulator_value=0.0))
    rng = np.random.default_rng(11)
    for step in range(5):
        lens = rng.integers(0, 6, size=23)
        offs = np.concatenate([[0], np.cumsum(lens)]).astype(np.int64)
        keys = rng.integers(0, 20 if step % 2 else V, size=int(offs[-1]), dtype=np.int64)
        grad = rng.standard_normal((23, d)).astype(np.float32)
        pooled, _ = o.forward(keys, offs)
        assert o.backward_update(keys, offs, grad, lr) == 0
        out = torch.nn.functional.embedding_bag(torch.from_numpy(keys), W,
                                                torch.from_numpy(offs[:-1]), mode="sum")
        np.testing.assert_allclose(pooled, out.detach().numpy(), rtol=1e-6, atol=1e-7)
        topt.zero_grad()
        (out * torch.from_numpy(grad)).sum().backward()
        topt.step()
    _, rows = o.export()
    np.testing.assert_allclose(rows[:, :d], W.detach().numpy(), rtol=1e-5, atol=1e-7)
    if opt == "adagrad":
        G = topt.state[W]["sum"].numpy()
        np.testing.assert_allclose(rows[:, d:], G, rtol=1e-5, atol=1e-7)


def test_lazy_adam_matches_torch_sparse_adam():
    d, V, lr, eps, b1, b2 = 8, 64, 1e-2, 1e-8, 0.9, 0.999
    o = Oracle(d, "adam", eps=eps, beta1=b1, beta2=b2)
    o.lookup_or_insert(np.arange(V, dtype=np.int64))
    _, rows = o.export()
    bag = torch.nn.EmbeddingBag(V, d, mode="sum", sparse=True)
    with torch.no_grad():
        bag.weight.copy_(torch.from_numpy(rows[:, :d]))
    topt = torch.optim.SparseAdam(bag.parameters(), lr=lr, betas=(b1, b2), eps=eps)
    rng = np.random.default_rng(12)
    for step in range(6):
        lens = rng.integers(1, 5, size=17)
        offs = np.concatenate([[0], np.cumsum(lens)]).astype(np.int64)
        keys = rng.integers(0, 30 if step % 2 else V, size=int(offs[-1]), dtype=np.int64)
        grad = rng.standard_normal((17, d)).astype(np.float32)
        o.forward(keys, offs)
        assert o.backward_update(keys, offs, grad, lr) == 0
        out = bag(torch.from_numpy(keys), torch.from_numpy(offs[:-1]))
        topt.zero_grad()
        (out * torch.from_numpy(grad)).sum().backward()
        topt.step()
    _, rows = o.export()
    np.testing.assert_allclose(rows[:, :d], bag.weight.detach().numpy(), rtol=1e-5, atol=1e-6)
    # SparseAdam moves the moments as m + (1-b1)(g-m) and v + (1-b2)(g^2-v):
    # the same values in exact arithmetic, rounded differently (the cancellation
    # in g^2 - v costs a few more ulps), hence the looser bound on the moments
    st = topt.state[bag.weight]
    np.testing.assert_allclose(rows[:, d:2 * d], st["exp_avg"].numpy(), rtol=5e-5, atol=1e-7)
    np.testing.assert_allclose(rows[:, 2 * d:], st["exp_avg_sq"].numpy(), rtol=5e-5, atol=1e-7)


def test_touched_rows_only():
    d = 16
    for opt in ("sgd", "adagrad", "adam", "adagrad_rowwise"):
        o = Oracle(d, opt)
        allk = np.arange(100, dtype=np.int64) * 3
        o.lookup_or_insert(allk)
        _, before = o.export()
        keys = np.array([3, 3, 30, 297], np.int64)
        offs = np.array([0, 2, 4], np.int64)
        o.forward(keys, offs)
        o.backward_update(keys, offs, np.ones((2, d), np.float32), 0.1)
        _, after = o.export()
        touched = {1, 10, 99}
        for r in range(100):
            assert np.array_equal(after[r], before[r]) == (r not in touched), (opt, r)


def test_coalesce_is_the_exact_sum_rounded_once():
    """g_k = fl(exact sum of the occurrence gradients): checked through the
    Adagrad accumulator, G = fl(g*g) after one step from G = 0.  The grads are
    chosen so that a running fp32 sum would round differently."""
    d = 4
    o = Oracle(d, "adagrad")
    key = np.array([42], np.int64)
    o.lookup_or_insert(key)
    occ = 257
    keys = np.full(occ, 42, np.int64)
    offs = np.arange(occ + 1, dtype=np.int64)
    g = np.zeros((occ, d), np.float32)
    g[0] = [1.0, -1.0, 3.0, 0.5]
    g[1:] = np.float32(2.0 ** -25)          # each one alone is lost in fp32 next to 1.0
    g[1:, 2] = np.float32(-1e-3)
    o.backward_update(keys, offs, g, 0.0)
    rows, _ = o.get_rows(key)
    for j in range(d):
        exact = sum((Fraction(float(x)) for x in g[:, j]), Fraction(0))
        gj = np.float32(float(exact))        # round once
        assert rows[0, d + j] == gj * gj, j
    # and a running fp32 sum would have given another value in column 0
    run = np.float32(0)
    for x in g[:, 0]:
        run = np.float32(run + x)
    assert run != np.float32(float(sum(Fraction(float(x)) for x in g[:, 0])))


def test_adagrad_closed_form():
    d, lr, eps, T = 4, 0.01, 1e-8, 50
    o = Oracle(d, "adagrad", eps=eps)
    key = np.array([7], np.int64)
    o.lookup_or_insert(key)
    w0, _ = o.get_rows(key)
    gval = np.array([0.5, -0.25, 2.0, 1.0], np.float32)
    for _ in range(T):
        o.backward_update(key, np.array([0, 1], np.int64), gval[None, :], lr)
    rows, _ = o.get_rows(key)
    # G_t = t g^2 ; w_T = w_0 - sum_t lr g / (sqrt(t) |g| + eps)
    for j in range(d):
        g = float(gval[j])
        want_w = float(w0[0, j]) - sum(lr * g / (math.sqrt(t) * abs(g) + eps) for t in range(1, T + 1))
        assert rows[0, d + j] == np.float32(T * g * g)
        assert abs(rows[0, j] - want_w) <= 1e-5 * abs(want_w) + 1e-7


def test_adam_closed_form_constant_gradient():
    """With a constant gradient, bias-corrected moments equal g and g^2, so each
    step moves the weight by lr * g / (|g| + eps)."""
    d, lr, eps, T = 4, 1e-3, 1e-8, 40
    o = Oracle(d, "adam", eps=eps, beta1=0.9, beta2=0.999)
    key = np.array([11], np.int64)
    o.lookup_or_insert(key)
    w0, _ = o.get_rows(key)
    gval = np.array([0.5, -0.25, 2.0, -1.0], np.float32)
    for _ in range(T):
        o.backward_update(key, np.array([0, 1], np.int64), gval[None, :], lr)
    rows, _ = o.get_rows(key)
    for j in range(d):
        g = float(gval[j])
        want = float(w0[0, j]) - T * lr * g / (abs(g) + eps)
        assert abs(rows[0, j] - want) <= 1e-4 * T * lr
        assert abs(rows[0, d + j] - (1 - 0.9 ** T) * g) <= 1e-5 * abs(g)
        assert abs(rows[0, 2 * d + j] - (1 - 0.999 ** T) * g * g) <= 1e-5 * g * g


def test_rowwise_adagrad_single_accumulator():
    d, lr, eps = 8, 0.1, 1e-8
    o = Oracle(d, "adagrad_rowwise", eps=eps)
    assert o.stride == d + 1
    key = np.array([5], np.int64)
    o.lookup_or_insert(key)
    w0, _ = o.get_rows(key)
    g = np.arange(1, d + 1, dtype=np.float32)[None, :]
    o.backward_update(key, np.array([0, 1], np.int64), g, lr)
    rows, _ = o.get_rows(key)
    G = float(np.mean(g.astype(np.float64) ** 2))     # 25.5
    assert rows[0, d] == np.float32(G)
    want = w0[0, :d].astype(np.float64) - lr * g[0] / (math.sqrt(G) + eps)
    np.testing.assert_allclose(rows[0, :d], want, rtol=1e-6)


# --- error handling and degenerate cases ------------------------------------------

def test_missing_and_negative_keys_are_reported_and_skipped():
    o = Oracle(4, "sgd")
    o.lookup_or_insert(np.array([1, 2], np.int64))
    _, before = o.export()
    rc = o.backward_update(np.array([1, 99], np.int64), np.array([0, 1, 2], np.int64),
                           np.ones((2, 4), np.float32), 0.5)
    assert rc == 5
    _, after = o.export()
    assert not np.array_equal(after[0], before[0]) and np.array_equal(after[1], before[1])
    assert o.size == 2
    off, rc = o.lookup_or_insert(np.array([-3, 2], np.int64))
    assert rc == 1 and off.tolist() == [-1, 1]


def test_empty_batch_and_empty_bags():
    o = Oracle(4, "adam")
    out, rc = o.forward(np.zeros(0, np.int64), np.array([0], np.int64))
    assert out.shape == (0, 4) and rc == 0
    out, rc = o.forward(np.zeros(0, np.int64), np.array([0, 0, 0], np.int64))
    assert np.all(out == 0) and o.size == 0
    assert o.backward_update(np.zeros(0, np.int64), np.array([0, 0], np.int64),
                             np.ones((1, 4), np.float32), 0.1) == 0


def test_bytes_per_row_arithmetic():
    g = _golden("memory_arith.json")
    for c in g["cases"]:
        gb = c["rows"] * c["dim"] * c["bytes_per_float"] / 1e9
        assert abs(gb - c["stated_gb"]) / c["stated_gb"] < 0.03


# --- bf16 row storage -----------------------------------------------------------------

def _torch_bf16(x):
    return torch.from_numpy(np.ascontiguousarray(x, np.float32)).to(torch.bfloat16).to(torch.float32).numpy()


def test_round_bf16_matches_torch_conversion():
    """Round to nearest, ties to even, against torch's float -> bfloat16 cast:
    random values over the whole exponent range, exact ties (both parities),
    subnormals, signed zeros, infinities, the largest finite values, NaN."""
    rng = np.random.default_rng(17)
    rand = rng.integers(0, 2 ** 32, size=20000, dtype=np.uint64).astype(np.uint32).view(np.float32)
    hi = rng.integers(0, 2 ** 16, size=2000, dtype=np.uint64).astype(np.uint32) << np.uint32(16)
    ties = (hi | np.uint32(0x8000)).view(np.float32)            # exactly half way
    near = np.concatenate([(hi | np.uint32(0x7fff)), (hi | np.uint32(0x8001))]).view(np.float32)
    special = np.array([0.0, -0.0, np.inf, -np.inf, 1e-45, -1e-45, 1e-40, 3.4028235e38, -3.4028235e38,
                        3.3961776e38, 1.0, 1.00390625, 1.005859375, 0.05, -0.05], np.float32)
    x = np.concatenate([rand, ties, near, special])
    got, want = round_bf16(x), _torch_bf16(x)
    nan = np.isnan(want)
    assert np.array_equal(np.isnan(got), nan)
    assert np.array_equal(got[~nan].view(np.uint32), want[~nan].view(np.uint32))
    assert np.isnan(round_bf16(np.array([np.nan], np.float32)))[0]


@pytest.mark.parametrize("opt", ["sgd", "adagrad", "adam", "adagrad_rowwise"])
def test_bf16_table_rounds_every_stored_weight(opt):
    """A bf16 table keeps every weight on the bf16 grid (initial rows and each
    step's result), its state in fp32, and equals the fp32 table's arithmetic
    with one rounding (torch's cast) per stored weight: checked step by step
    from the same pre-step rows."""
    d, lr = 8, 0.05
    rng = np.random.default_rng(23)
    o = Oracle(d, opt, storage="bf16")
    keys = np.arange(40, dtype=np.int64) * 3 + 1
    o.lookup_or_insert(keys)
    _, rows = o.export()
    assert np.array_equal(rows[:, :d], _torch_bf16(np.stack([init_row(int(k), d) for k in keys])))
    for step in range(3):
        offs = np.arange(0, 41, 4, dtype=np.int64)
        grad = rng.standard_normal((10, d)).astype(np.float32)
        _, before = o.export()
        assert o.backward_update(keys, offs, grad, lr) == 0
        _, after = o.export()
        # the same step on an fp32 table holding the pre-step rows, then one cast
        ref = Oracle(d, opt)
        ref.lookup_or_insert(keys)
        _set_rows(ref, before)
        for _ in range(step):  # Adam's step count: empty calls advance it
            ref.backward_update(np.zeros(0, np.int64), np.zeros(1, np.int64), np.zeros((0, d), np.float32), lr)
        ref.backward_update(keys, offs, grad, lr)
        _, r32 = ref.export()
        ref.close()
        assert np.array_equal(after[:, :d], _torch_bf16(r32[:, :d]))
        assert np.array_equal(after[:, d:], r32[:, d:])  # fp32 state, unrounded
    assert np.array_equal(after[:, :d], _torch_bf16(after[:, :d]))


def _set_rows(o, rows):
    """Overwrite an oracle table's stored rows with `rows` (row order)."""
    import ctypes as C
    from oracle.oracle import lib
    n, s = rows.shape
    buf = np.ascontiguousarray(rows, np.float32)
    lib().orc_import_rows(o.h, buf.ctypes.data_as(C.c_void_p), n)


def test_bf16_forward_sums_the_stored_values():
    d = 8
    o = Oracle(d, "sgd", storage="bf16")
    o.lookup_or_insert(np.arange(64, dtype=np.int64))
    _, rows = o.export()
    weight = torch.from_numpy(rows[:, :d].copy())  # the stored (bf16-exact) values
    rng = np.random.default_rng(29)
    lens = rng.integers(0, 9, size=30)
    offs = np.concatenate([[0], np.cumsum(lens)]).astype(np.int64)
    keys = rng.integers(0, 64, size=int(offs[-1]), dtype=np.int64)
    pooled, _ = o.forward(keys, offs)
    ref = torch.nn.functional.embedding_bag(torch.from_numpy(keys), weight, torch.from_numpy(offs[:-1]),
                                            mode="sum").numpy()
    np.testing.assert_allclose(pooled, ref, rtol=1e-6, atol=1e-7)


# --- admission / eviction (readings of the hook the pages only name) --------------------

def _same_tables(a, b, d):
    ka, ra = a.export()
    kb, rb = b.export()
    assert np.array_equal(ka, kb) and np.array_equal(ra[:, :d], rb[:, :d]) and np.array_equal(ra, rb)


def test_admission_threshold_one_is_the_plain_table():
    rng = np.random.default_rng(41)
    a, b = Oracle(8, "adagrad"), Oracle(8, "adagrad")
    b.set_hooks(admit_threshold=1, track_access=True)
    for _ in range(4):
        lens = rng.integers(0, 6, size=50)
        offs = np.concatenate([[0], np.cumsum(lens)]).astype(np.int64)
        keys = rng.integers(0, 120, size=int(offs[-1])).astype(np.int64)
        pa, _ = a.forward(keys, offs)
        pb, _ = b.forward(keys, offs)
        assert np.array_equal(pa, pb)
        g = rng.standard_normal((50, 8)).astype(np.float32)
        assert a.backward_update(keys, offs, g, 0.1) == b.backward_update(keys, offs, g, 0.1) == 0
    _same_tables(a, b, 8)


def test_admission_closed_form_and_zero_contribution():
    """A key occurring c times in every call is admitted in call ceil(A / c)
    with its initial row; until then each of its ids pools as if it were
    absent from its bag (the pooled rows equal those of a plain table fed the
    batch without those ids) and its gradients are dropped."""
    A, d = 5, 4
    o = Oracle(d, "sgd")
    o.set_hooks(admit_threshold=A)
    counts = {100: 1, 200: 2, 300: 3, 400: 5, 500: 7}
    keys = np.array([k for k, c in counts.items() for _ in range(c)], np.int64)
    rng = np.random.default_rng(43)
    for call in range(1, 7):
        keys_c = rng.permutation(keys)
        offs = np.array([0, keys_c.size // 2, keys_c.size], np.int64)
        before = {k for k in counts if -(-A // counts[k]) < call}  # admitted in an earlier call
        now = {k for k in counts if -(-A // counts[k]) <= call}
        pooled, _ = o.forward(keys_c, offs)
        # reference: a plain table holding only the admitted keys, same values
        ref = Oracle(d, "sgd")
        keep = np.array([k in now for k in keys_c])
        ref_off = np.concatenate([[0], np.cumsum([keep[:keys_c.size // 2].sum(), keep[keys_c.size // 2:].sum()])])
        ref_keys = keys_c[keep]
        got_rows, missing = o.get_rows(np.array(sorted(now), np.int64)) if now else (None, 0)
        assert missing == 0
        ref.lookup_or_insert(np.array(sorted(now), np.int64))
        if now:
            _set_rows(ref, got_rows)
        rp, _ = ref.forward(ref_keys, ref_off.astype(np.int64))
        np.testing.assert_array_equal(pooled, rp)
        for k in now - before:  # admitted in this call: the initial row
            r, _ = o.get_rows(np.array([k], np.int64))
            assert np.array_equal(r[0, :d], init_row(k, d))
        assert o.live == len(now)
        g = np.ones((2, d), np.float32)
        assert o.backward_update(keys_c, offs, g, 0.5) == 0  # keys not admitted: skipped, no error
        ref.close()


def test_eviction_live_set_and_row_reuse():
    """After evict(max_idle) the live keys are exactly those seen in the last
    max_idle + 1 calls (a set computed from the stream); freed rows are handed
    to the next admitted keys smallest first, with their initial values; rows
    of surviving keys are bit-identical."""
    d = 4
    o = Oracle(d, "adam")
    o.set_hooks(track_access=True)
    rng = np.random.default_rng(47)
    calls = [rng.choice(60, size=25, replace=False).astype(np.int64) * 7 + 1 for _ in range(6)]
    for ks in calls:
        o.forward(ks, np.array([0, ks.size], np.int64))
        o.backward_update(ks, np.array([0, ks.size], np.int64), rng.standard_normal((1, d)).astype(np.float32), 0.1)
    keys_before, rows_before = o.export()
    max_idle = 2
    recent = set(np.concatenate(calls[-(max_idle + 1):]).tolist())
    freed = o.evict(max_idle)
    keys_after, rows_after = o.export()
    live = set(keys_after[keys_after >= 0].tolist())
    assert live == recent and o.live == len(recent)
    free_rows = sorted(np.nonzero(keys_after < 0)[0].tolist())
    assert freed == len(free_rows) and freed == len(set(keys_before.tolist()) - recent)
    surv = keys_after >= 0
    assert np.array_equal(rows_after[surv], rows_before[surv])
    # new keys take the free rows smallest first, then appended rows
    fresh = np.array([10_001, 10_002, 10_003] + [20_000 + i for i in range(len(free_rows))], np.int64)
    off, _ = o.lookup_or_insert(fresh)
    expect = free_rows + list(range(len(keys_after), len(keys_after) + fresh.size - len(free_rows)))
    assert off.tolist() == expect
    r, _ = o.get_rows(fresh[:1])
    assert np.array_equal(r[0, :d], init_row(int(fresh[0]), d)) and np.all(r[0, d:] == 0)
    # an evicted key that returns is a new key: a fresh initial row
    gone = sorted(set(keys_before.tolist()) - recent)[0]
    o.lookup_or_insert(np.array([gone], np.int64))
    r, _ = o.get_rows(np.array([gone], np.int64))
    assert np.array_equal(r[0, :d], init_row(int(gone), d)) and np.all(r[0, d:] == 0)
