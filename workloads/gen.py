"""Seeded synthetic input streams for the hashed embedding engine.

This module is shared by the CUDA path's tests and bench and by the CPU
oracle's tests.  It draws random numbers and lays them out as the engine's
inputs (table ids, raw feature ids, bag offsets, output gradients) and holds
none of the engine's arithmetic: no key packing, no hashing, no row
initialisation, no pooling, no optimizer step.

The five workloads are the ones the recommender pages describe in words:
a tiny single table, a 26-table DLRM-style merged lookup (DLRM explainer,
"Embedding tables" module; the Criteo field count of 26 in the MindSpore
tutorial, section 2.1), long sequence bags (DLRM practice article,
section 2.1: EmbeddingBag for variable-length behaviour sequences), a
table that grows from empty (RecIS overview, "Embedding Engine": blocks are
appended as the table grows) and a hot-key stream (Zipf alpha 1.4).
Where the pages leave a parameter open the value chosen here is the one the
design document lists under "input recipe".
"""
from __future__ import annotations

import dataclasses
import math
from typing import Dict, Optional

import numpy as np

ID_BITS = 48
_MASK48 = np.uint64((1 << ID_BITS) - 1)
# Odd multiplier: r -> r * C mod 2^48 is a bijection on [0, 2^48), so distinct
# ranks/counters give distinct raw ids, spread over the whole id space.
_SCRAMBLE = np.uint64(0x9E3779B97F4B)


def rank_to_id(r: np.ndarray) -> np.ndarray:
    """Map 0-based ranks / counters (uint64 or int64) to raw 48-bit ids (int64)."""
    r = np.asarray(r).astype(np.uint64)
    with np.errstate(over="ignore"):
        out = (r * _SCRAMBLE) & _MASK48
    return out.astype(np.int64)


def _rng(seed: int, *stream: int) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(np.random.SeedSequence([seed, *stream])))


# ---------------------------------------------------------------------------
# Bounded Zipf sampling by rejection-inversion (Hoermann & Derflinger 1996,
# "Rejection-inversion to generate variates from monotone discrete
# distributions", ACM TOMACS 6(3)).  P(k) proportional to k^-s, k in [1, n].
# ---------------------------------------------------------------------------
class ZipfSampler:
    def __init__(self, n: int, s: float):
        if n < 1 or s <= 0.0 or s == 1.0:
            raise ValueError("ZipfSampler needs n >= 1 and s > 0, s != 1")
        self.n = int(n)
        self.s = float(s)
        self.q = 1.0 - self.s
        self.h_x1 = self._H(1.5) - 1.0
        self.h_n = self._H(self.n + 0.5)
        self.s_const = 2.0 - self._Hinv(self._H(2.5) - self._h(2.0))

    def _H(self, x):
        # integral of t^-s: (x^(1-s) - 1) / (1-s)
        return np.expm1(self.q * np.log(x)) / self.q

    def _Hinv(self, y):
        return np.exp(np.log1p(self.q * y) / self.q)

    def _h(self, x):
        return np.exp(-self.s * np.log(x))

    def sample(self, rng: np.random.Generator, size: int) -> np.ndarray:
        out = np.empty(size, dtype=np.int64)
        todo = np.arange(size)
        while todo.size:
            u = self.h_n + rng.random(todo.size) * (self.h_x1 - self.h_n)
            x = self._Hinv(u)
            k = np.clip(np.floor(x + 0.5), 1, self.n)
            ok = (k - x <= self.s_const) | (u >= self._H(k + 0.5) - self._h(k))
            out[todo[ok]] = k[ok].astype(np.int64)
            todo = todo[~ok]
        return out


@dataclasses.dataclass
class Batch:
    """One step's inputs.  Bag b holds flat positions [bag_offsets[b], bag_offsets[b+1])."""
    table_ids: np.ndarray    # int32 [N]
    ids: np.ndarray          # int64 [N], raw ids < 2^48
    bag_offsets: np.ndarray  # int64 [B+1], CSR, [0] = 0, [B] = N

    @property
    def n(self) -> int:
        return int(self.ids.shape[0])

    @property
    def n_bags(self) -> int:
        return int(self.bag_offsets.shape[0] - 1)


@dataclasses.dataclass
class Workload:
    """A seeded stream of batches with fixed embedding dim and optimizer."""
    name: str
    dim: int
    optimizer: str            # "sgd" | "adagrad" | "adam"
    lr: float
    steps: int
    seed: int
    eps: float = 1e-8
    beta1: float = 0.9
    beta2: float = 0.999
    block_rows: int = 1 << 20
    params: Dict[str, float] = dataclasses.field(default_factory=dict)

    # -- per-workload hooks (overridden by subclasses) --
    def batch(self, step: int) -> Batch:  # pragma: no cover - abstract
        raise NotImplementedError

    def preinsert(self):
        """Chunks of (table_ids, ids) to insert, untimed, before step 0."""
        return iter(())

    def grads(self, step: int, n_bags: int) -> np.ndarray:
        """N(0,1) fp32 output gradients [n_bags, dim] for this step."""
        return _rng(self.seed, 2, step).standard_normal((n_bags, self.dim), dtype=np.float32)

    def torch_grads(self, step: int, n_bags: int, device):
        """Same distribution, drawn on the device by torch's seeded generator
        (used where host generation of hundreds of MB per step is too slow)."""
        import torch
        g = torch.Generator(device=device)
        g.manual_seed(self.seed * 1_000_003 + step)
        return torch.randn((n_bags, self.dim), generator=g, device=device, dtype=torch.float32)


class TinyUniform(Workload):
    """65,536 distinct keys uniform in [0, 2^40); per step 1024 bags x 1 id drawn
    uniformly (with replacement) from the pool; one table."""

    def __init__(self, seed=1001, pool=65536, bags=1024, steps=10, dim=16):
        super().__init__("tiny_uniform", dim, "sgd", 0.01, steps, seed)
        self.params = dict(pool=pool, bags=bags)
        rng = _rng(seed, 0)
        keys = np.unique(rng.integers(0, 1 << 40, size=pool, dtype=np.int64))
        while keys.size < pool:
            more = rng.integers(0, 1 << 40, size=pool - keys.size, dtype=np.int64)
            keys = np.unique(np.concatenate([keys, more]))
        self.pool = rng.permutation(keys)

    def batch(self, step: int) -> Batch:
        rng = _rng(self.seed, 1, step)
        b = int(self.params["bags"])
        ids = self.pool[rng.integers(0, self.pool.size, size=b)]
        return Batch(np.zeros(b, np.int32), ids.astype(np.int64), np.arange(b + 1, dtype=np.int64))


class DlrmMerged(Workload):
    """26 categorical tables merged into one map; cardinalities log-uniform in
    [1e3, 1e7]; each sample has one id per table (pooling 1), Zipf(1.05) over
    the table's ranks.  Bag b = sample * 26 + table, so the pooled output
    reshapes to [batch, 26, dim]."""

    def __init__(self, seed=1002, batch=65536, tables=26, steps=50, dim=128,
                 card_lo=1e3, card_hi=1e7, alpha=1.05):
        super().__init__("dlrm_merged_26", dim, "adagrad", 0.01, steps, seed)
        self.params = dict(batch=batch, tables=tables, alpha=alpha)
        rng = _rng(seed, 0)
        lo, hi = math.log(card_lo), math.log(card_hi)
        self.cards = np.floor(np.exp(rng.uniform(lo, hi, size=tables))).astype(np.int64)
        self.samplers = [ZipfSampler(int(c), alpha) for c in self.cards]

    def batch(self, step: int) -> Batch:
        bsz, t = int(self.params["batch"]), int(self.params["tables"])
        ids = np.empty((bsz, t), np.int64)
        for j, zs in enumerate(self.samplers):
            ids[:, j] = rank_to_id(zs.sample(_rng(self.seed, 1, step, j), bsz) - 1)
        tids = np.broadcast_to(np.arange(t, dtype=np.int32), (bsz, t))
        n = bsz * t
        return Batch(np.ascontiguousarray(tids).reshape(n), ids.reshape(n), np.arange(n + 1, dtype=np.int64))


class SequenceBags(Workload):
    """8 tables, one bag per (sample, table); bag length min(Poisson(50), 200);
    each batch has floor(20%) of its ids never seen before (a per-table counter
    above the Zipf range), the rest Zipf(1.2) over 1e6 ranks per table."""

    FRESH_STRIDE = 1 << 23   # counters reserved per step and table

    def __init__(self, seed=1003, batch=16384, tables=8, steps=50, dim=64,
                 mean_len=50.0, max_len=200, universe=1_000_000, alpha=1.2, fresh=0.2):
        super().__init__("sequence_bags", dim, "sgd", 0.05, steps, seed)
        self.params = dict(batch=batch, tables=tables, mean_len=mean_len, max_len=max_len,
                           universe=universe, alpha=alpha, fresh=fresh)
        self.sampler = ZipfSampler(universe, alpha)

    def batch(self, step: int) -> Batch:
        p = self.params
        bsz, t = int(p["batch"]), int(p["tables"])
        rng = _rng(self.seed, 1, step)
        lens = np.minimum(rng.poisson(p["mean_len"], size=bsz * t), int(p["max_len"])).astype(np.int64)
        offs = np.zeros(bsz * t + 1, np.int64)
        np.cumsum(lens, out=offs[1:])
        n = int(offs[-1])
        bag_table = np.tile(np.arange(t, dtype=np.int32), bsz)
        tids = np.repeat(bag_table, lens)
        ids = rank_to_id(self.sampler.sample(rng, n) - 1)
        n_fresh = int(math.floor(p["fresh"] * n))
        pos = np.sort(rng.choice(n, size=n_fresh, replace=False))
        # fresh ids: per table, consecutive counters in flat order
        ft = tids[pos]
        order = np.argsort(ft, kind="stable")
        counts = np.bincount(ft, minlength=t)
        start = np.zeros(t, np.int64)
        np.cumsum(counts[:-1], out=start[1:])
        within = np.empty(n_fresh, np.int64)
        within[order] = np.arange(n_fresh) - np.repeat(start, counts)
        base = int(p["universe"]) + step * self.FRESH_STRIDE
        ids[pos] = rank_to_id(base + within)
        return Batch(tids, ids, offs)


class GrowthStream(Workload):
    """One table, empty at start; 131,072 bags x 4 ids; step 0 all fresh; later
    steps floor(30%) fresh ids, the rest uniform over ids already inserted."""

    def __init__(self, seed=1004, bags=131072, pooling=4, steps=200, dim=32, fresh=0.3):
        super().__init__("growth_stream", dim, "adam", 1e-3, steps, seed)
        self.params = dict(bags=bags, pooling=pooling, fresh=fresh)

    def _fresh_per_step(self) -> int:
        return int(math.floor(self.params["fresh"] * self.params["bags"] * self.params["pooling"]))

    def inserted_before(self, step: int) -> int:
        n = int(self.params["bags"] * self.params["pooling"])
        return 0 if step == 0 else n + (step - 1) * self._fresh_per_step()

    def batch(self, step: int) -> Batch:
        b, k = int(self.params["bags"]), int(self.params["pooling"])
        n = b * k
        rng = _rng(self.seed, 1, step)
        c0 = self.inserted_before(step)
        if step == 0:
            ctr = rng.permutation(n).astype(np.int64)
        else:
            ctr = rng.integers(0, c0, size=n, dtype=np.int64)
            nf = self._fresh_per_step()
            pos = rng.choice(n, size=nf, replace=False)
            ctr[pos] = c0 + rng.permutation(nf)
        return Batch(np.zeros(n, np.int32), rank_to_id(ctr), np.arange(0, n + 1, k, dtype=np.int64))


class HotKey(Workload):
    """Table pre-populated with `rows` keys in rank order; 262,144 bags x 20 ids,
    Zipf(1.4) over the pre-populated ranks."""

    def __init__(self, seed=1005, rows=50_000_000, bags=262144, pooling=20, steps=20, dim=64,
                 alpha=1.4, chunk=1 << 22):
        super().__init__("hot_key", dim, "adagrad", 0.01, steps, seed)
        self.params = dict(rows=rows, bags=bags, pooling=pooling, alpha=alpha, chunk=chunk)
        self.sampler = ZipfSampler(rows, alpha)

    def preinsert(self):
        rows, chunk = int(self.params["rows"]), int(self.params["chunk"])
        for a in range(0, rows, chunk):
            r = np.arange(a, min(rows, a + chunk), dtype=np.int64)
            yield np.zeros(r.size, np.int32), rank_to_id(r)

    def batch(self, step: int) -> Batch:
        b, k = int(self.params["bags"]), int(self.params["pooling"])
        ids = rank_to_id(self.sampler.sample(_rng(self.seed, 1, step), b * k) - 1)
        return Batch(np.zeros(b * k, np.int32), ids, np.arange(0, b * k + 1, k, dtype=np.int64))


def full(name: str) -> Workload:
    """The five workloads at their stated sizes."""
    return {
        "tiny_uniform": TinyUniform,
        "dlrm_merged_26": DlrmMerged,
        "sequence_bags": SequenceBags,
        "growth_stream": GrowthStream,
        "hot_key": HotKey,
    }[name]()


def small(name: str, seed_offset: int = 0) -> Workload:
    """Reduced versions the oracle finishes in seconds; they keep each
    workload's structure (tables, distributions, pooling) and still span many
    CUDA tiles with ragged tails."""
    s = seed_offset
    if name == "tiny_uniform":
        return TinyUniform(seed=1001 + s)
    if name == "dlrm_merged_26":
        return DlrmMerged(seed=1002 + s, batch=1531, steps=3, card_lo=1e2, card_hi=1e5)
    if name == "sequence_bags":
        return SequenceBags(seed=1003 + s, batch=263, steps=3, universe=20000)
    if name == "growth_stream":
        return GrowthStream(seed=1004 + s, bags=2999, steps=5)
    if name == "hot_key":
        return HotKey(seed=1005 + s, rows=200_003, bags=5003, steps=3, chunk=65536)
    raise KeyError(name)


NAMES = ("tiny_uniform", "dlrm_merged_26", "sequence_bags", "growth_stream", "hot_key")
