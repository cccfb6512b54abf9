"""Benchmark of the hashed embedding training step (lookup-or-insert + sum-pool
forward, coalesced sparse-gradient + fused optimizer backward) on B200.

One step = key packing, embbag_forward and embbag_backward_update over one
batch of the 26-table DLRM-style merged workload (65,536 samples x 26 ids,
pooling 1, dim 128 fp32, Adagrad, Zipf 1.05 ids; synthetic, seeded).  The
table starts empty: warm-up steps are the stream's first steps, timed steps
the ones after.  After the headline, the other four workloads (tiny uniform,
sequence bags, growth stream, hot key), the headline's and the sequence
stream on tables with bf16 weights, and the headline with row-wise Adagrad
are each run whole with their own step counts and reported
under "workloads", with capacity reserved before step 0; the growth stream
runs a second time with its table growing on demand inside the timed steps
("growth_stream:on-demand").  "e2e" repeats the headline steps through the public
API from pinned host buffers, with the copies pipelined against the compute.
Prints one JSON line.

Timing: CUDA events on the launching stream at each step's start, at the
forward / backward boundary and at its end, nothing else inside the timed
steps but the IDMap growth phase's own events; "fwd" is key packing +
embbag_forward, "bwd" is embbag_backward_update.  "phases_ms_per_step" (and
the roofline's kernel time) come from a replay of the timed steps on the same
table with an event around every phase; a replay inserts no keys, so its
forward assignment phase is empty.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl dhs|reference]

--impl reference times the CPU oracle (single core) on a bounded sample of
the same workload.  Under torchrun each rank runs an independent replica
(its own table and seed): the path does not shard, so there is no data-path
collective; value is the ids of all ranks over the slowest rank's time.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

from workloads import gen  # noqa: E402

METRIC = "IDs/sec & HBM GB/s (% of peak): hashed lookup+bag-sum fwd, sparse update bwd"
UNIT = "IDs/s"
# kernel selection thresholds of the library (compile-time constants there)
POOL_SPLIT_LEN = 4   # bags of >= 4 ids on average: probe kernel + gather from references
SEGW_MIN_DIM = 32    # rows of >= 32 floats: warp-per-chunk segment kernel ...
NARROW_MAX_DIM = 64  # ... except fp32 rows of 33-64 floats with fewer than
NARROW_RUN = 8       # 8 ids per updated row on average: the lane-group kernel
WORKLOAD = "dlrm_merged_26"


# ---------------------------------------------------------------------------
# algorithmic bytes (compulsory traffic: each datum once)
# ---------------------------------------------------------------------------
def stride_floats(dim: int, opt: str) -> int:
    return dim + {"sgd": 0, "adagrad": dim, "adam": 2 * dim, "adagrad_rowwise": 4}[opt]


def row_bytes(dim: int, opt: str, weights: str = "f32"):
    """(R, S): bytes of a row's weights, and of the whole row with its fp32
    optimizer state."""
    r = (2 if weights == "bf16" else 4) * dim
    return r, r + 4 * (stride_floats(dim, opt) - dim)


def alg_bytes(n: int, b: int, u: int, m: int, dim: int, opt: str, weights: str = "f32") -> dict:
    """Per step.  n ids, b bags, u distinct keys, m of them new."""
    R, S = row_bytes(dim, opt, weights)
    pack = 4 * n + 8 * n + 8 * n
    fwd_pool = 8 * n + 8 * (b + 1) + 16 * u + 16 * m + R * (u - m) + 4 * dim * b
    fwd_assign = S * m + 16 * m
    # the split forward (long bags) gathers every distinct row, new ones included,
    # after the assignment wrote them
    fwd_refs = 8 * (b + 1) + R * u + 4 * dim * b
    bwd = 8 * n + 8 * (b + 1) + 16 * u + 4 * dim * b + 2 * S * u
    # the timed forward is key packing + embbag_forward
    return dict(pack=pack, fwd_pool=fwd_pool, fwd_refs=fwd_refs, fwd_assign=fwd_assign,
                fwd=pack + fwd_pool + fwd_assign, bwd=bwd,
                bwd_seg=4 * dim * b + 2 * S * u + 8 * n)


def load_peaks() -> dict:
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return dict(hbm_gbs=float(d["hbm_gbs"]), source="measured")
    return dict(hbm_gbs=6650.0, source="fallback")


def narrow_seg(dim: int, weights: str, n_ids: int, unique: int) -> bool:
    """Which segment kernel the library runs (the lane-group one for narrow
    rows, and for fp32 rows of 33-64 floats whose rows get few ids)."""
    if dim < SEGW_MIN_DIM:
        return True
    return (weights == "f32" and SEGW_MIN_DIM < dim <= NARROW_MAX_DIM and unique > 0
            and n_ids < NARROW_RUN * unique)


def load_traffic(kernel: str):
    """DRAM bytes per launch of `kernel` from the committed ncu summary, if it
    was taken on the current kernel sources (else None)."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    with open(p) as f:
        d = json.load(f)
    ent = d.get(kernel)
    if not ent:
        return None
    from dynamic_hashed_sparse_b200 import build as B
    if ent.get("source_digest") != B._digest():
        return None
    return ent


# ---------------------------------------------------------------------------
# clocks during the timed region
# ---------------------------------------------------------------------------
class ClockSampler:
    """SM clock and clock-event reasons of this process's GPU, sampled every
    ~2 ms by a thread through NVML while the timed region runs (two cheap
    queries per sample, so the sampling does not hold up the GPU driver or
    the launching thread)."""

    REASONS = (("hw_slowdown", "nvmlClocksEventReasonHwSlowdown"),
               ("hw_thermal_slowdown", "nvmlClocksEventReasonHwThermalSlowdown"),
               ("sw_thermal_slowdown", "nvmlClocksEventReasonSwThermalSlowdown"),
               ("sw_power_cap", "nvmlClocksEventReasonSwPowerCap"),
               ("hw_power_brake", "nvmlClocksEventReasonHwPowerBrakeSlowdown"))

    def __init__(self, cuda_index: int, period_s: float = 0.002):
        self.idx = cuda_index
        self.period = period_s
        self.samples = []
        self.max_mhz = None
        self._stop = None
        self._thread = None
        self.err = None

    def _handle(self, nv):
        try:
            import torch
            p = torch.cuda.get_device_properties(self.idx)
            bus = f"{p.pci_domain_id:08x}:{p.pci_bus_id:02x}:{p.pci_device_id:02x}.0"
            return nv.nvmlDeviceGetHandleByPciBusId(bus)
        except Exception:
            return nv.nvmlDeviceGetHandleByIndex(self.idx)

    def _run(self):
        import pynvml as nv
        try:
            nv.nvmlInit()
            h = self._handle(nv)
            self.max_mhz = nv.nvmlDeviceGetMaxClockInfo(h, nv.NVML_CLOCK_SM)
            bits = [(name, getattr(nv, attr, 0)) for name, attr in self.REASONS]
            while not self._stop.is_set():
                mhz = nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM)
                r = nv.nvmlDeviceGetCurrentClocksEventReasons(h)
                self.samples.append((time.perf_counter(), mhz, [n for n, bit in bits if bit and r & bit]))
                self._stop.wait(self.period)
        except Exception as e:  # no NVML: the line says so
            self.err = repr(e)

    def __enter__(self):
        import threading
        self._stop = threading.Event()
        self._thread = threading.Thread(target=self._run, daemon=True)
        self._thread.start()
        time.sleep(0.05)
        self.t0 = time.perf_counter()
        return self

    def __exit__(self, *a):
        self.t1 = time.perf_counter()
        time.sleep(0.02)
        self._stop.set()
        self._thread.join(timeout=5)

    def summary(self) -> dict:
        inside = [x for x in self.samples if self.t0 <= x[0] <= self.t1]
        if not inside and self.samples:  # region shorter than one period: nearest samples
            inside = sorted(self.samples, key=lambda x: min(abs(x[0] - self.t0), abs(x[0] - self.t1)))[:2]
        if not inside:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": ["unsampled"], "samples": 0,
                    "error": self.err}
        return {"sm_mhz": statistics.median(x[1] for x in inside), "sm_max_mhz": self.max_mhz,
                "reasons": sorted({r for x in inside for r in x[2]}), "samples": len(inside)}


# ---------------------------------------------------------------------------
# distributed plumbing (independent replicas; max over ranks)
# ---------------------------------------------------------------------------
def dist_env():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


def init_dist(world: int, backend: str):
    if world <= 1:
        return None
    import datetime

    import torch.distributed as dist
    dist.init_process_group(backend=backend, timeout=datetime.timedelta(seconds=120))
    return dist


def max_over_ranks(x: float, dist, device=None) -> float:
    if dist is None:
        return x
    import torch
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def sum_over_ranks(x: float, dist, device=None) -> float:
    if dist is None:
        return x
    import torch
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.SUM)
    return float(t.item())


def barrier(dist, device=None):
    if dist is not None:
        import torch
        t = torch.zeros(1, device=device)
        dist.all_reduce(t)


# ---------------------------------------------------------------------------
# CPU oracle timing (reference arm and cpu_baseline)
# ---------------------------------------------------------------------------
def time_oracle(w, steps, frac: float, timed_from: int = 0):
    """Run the oracle on the first `steps` steps of the workload, each batch cut
    to its first `frac` of bags, timing the steps from `timed_from` on;
    returns (timed ids, seconds)."""
    from oracle import Oracle, pack_keys
    o = Oracle(w.dim, w.optimizer, eps=w.eps, beta1=w.beta1, beta2=w.beta2)
    ids = 0
    secs = 0.0
    try:
        for s in range(steps):
            b = w.batch(s)
            nb = max(1, int(b.n_bags * frac))
            offs = b.bag_offsets[: nb + 1]
            n = int(offs[-1])
            grad = w.grads(s, nb)  # the first nb rows of the step's gradients
            t0 = time.perf_counter()
            keys, _ = pack_keys(b.table_ids[:n], b.ids[:n])
            o.forward(keys, offs)
            o.backward_update(keys, offs, grad, w.lr)
            if s >= timed_from:
                secs += time.perf_counter() - t0
                ids += n
    finally:
        o.close()
    return ids, secs


def cpu_cores_used() -> int:
    return 1


def run_reference(args):
    world, rank, _ = dist_env()
    if rank != 0:
        return 0
    w = make_workload(args.workload, 0, args.batch)
    frac = args.ref_frac
    ids, secs = time_oracle(w, args.warmup + args.steps, frac, timed_from=args.warmup)
    value = ids / secs if secs > 0 else 0.0
    sample = (f"steps {args.warmup}..{args.warmup + args.steps - 1} of {w.name} timed after "
              f"{args.warmup} untimed, first {frac:.4f} of each batch's bags ({ids} timed ids), "
              f"oracle single-threaded")
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * secs / max(1, args.steps),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "f32", "data": "synthetic",
        "config": workload_config(w, 0, False),
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": cpu_cores_used(), "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


L2_BYTES = 126 << 20
PHASE_TIMING = True  # per-phase events inside the timed steps (--no-phases: off)

DESCRIPTIONS = {
    "tiny_uniform": "1024 bags x 1 id drawn uniformly from 65,536 distinct keys in [0, 2^40), one table, "
                    "dim 16 fp32, SGD lr 0.01",
    "dlrm_merged_26": "26 tables merged in one IDMap, {batch} samples x 26 ids (pooling 1), Zipf 1.05 per "
                      "table over log-uniform [1e3, 1e7] cardinalities, dim 128 fp32, Adagrad lr 0.01 eps 1e-8",
    "sequence_bags": "16,384 samples x 8 tables, bag length min(Poisson(50), 200), 20% of ids never seen "
                     "before, the rest Zipf 1.2 over 1e6 ranks per table, dim 64 fp32, SGD lr 0.05",
    "growth_stream": "one table from empty, 131,072 bags x 4 ids, 30% never-seen ids per step, the rest "
                     "uniform over inserted ids, dim 32 fp32, Adam lr 1e-3 (b1 0.9, b2 0.999), blocks of 2^20 rows",
    "hot_key": "5e7 keys pre-inserted (untimed), 262,144 bags x 20 ids, Zipf 1.4 over them, dim 64 fp32, "
               "Adagrad lr 0.01 eps 1e-8",
}


def make_workload(name: str, rank: int = 0, batch: int = 0):
    """The named workload; replicas (rank > 0) draw their own streams."""
    if name == "dlrm_merged_26":
        return gen.DlrmMerged(seed=1002 + 7919 * rank, batch=batch or 65536)
    w = gen.full(name)
    w.seed += 7919 * rank
    return w


def default_reserve(w, steps: int) -> int:
    """Keys the stream holds after `steps` steps plus one batch of new keys."""
    if w.name == "tiny_uniform":
        return 65536
    if w.name == "dlrm_merged_26":
        return 6_000_000
    if w.name == "sequence_bags":
        return int(8e6 + (steps + 1) * 1.4e6)
    if w.name == "growth_stream":
        return w.inserted_before(steps) + 2 * 524288
    return int(w.params["rows"]) + 1


def resolve_reserve(w, steps: int, policy) -> int:
    """Keys reserved before step 0: an explicit count, -1 for the workload's
    default, or "on-demand" (0: the table grows inside the timed steps; a
    pre-populated table still gets room for its pre-inserted keys)."""
    if policy == "on-demand":
        return int(w.params["rows"]) + 1 if w.name == "hot_key" else 0
    policy = int(policy)
    return default_reserve(w, steps) if policy < 0 else policy


def workload_config(w, reserve: int, flush: bool) -> dict:
    table = ("starts as the workload defines it; "
             + (f"capacity for {reserve} keys reserved before step 0" if reserve
                else "grows on demand inside the timed steps (no reservation)")
             + "; warm-up = the stream's first steps")
    return {"workload": f"{w.name}: " + DESCRIPTIONS[w.name].format(batch=w.params.get("batch")),
            "dim": w.dim, "optimizer": w.optimizer,
            "l2": ("L2 flushed (512 MB written) before each timed step; each step is timed on its own"
                   if flush else "inputs larger than L2 (per-step gradients and ids exceed 2 x 126 MB)"),
            "table": table}


def setup_table(dhs, w, reserve: int, weights: str = "f32"):
    """A table for the workload, capacity reserved and any pre-insertion done."""
    import torch
    t = dhs.ht_create(w.dim, w.optimizer, block_rows=w.block_rows, eps=w.eps, beta1=w.beta1, beta2=w.beta2,
                      weights=weights)
    if reserve:
        dhs.ht_reserve(t, reserve)
    for tids, ids in w.preinsert():
        keys = dhs.dhs_pack_keys(torch.from_numpy(tids).cuda(), torch.from_numpy(ids).cuda())
        dhs.ht_lookup_or_insert(t, keys)
    torch.cuda.synchronize()
    return t


# ---------------------------------------------------------------------------
# host inputs, generated in a process pool started before the first CUDA call
# ---------------------------------------------------------------------------
_WORKLOAD_CACHE = {}


def _gen_batch(job):
    name, rank, batch, step = job
    key = (name, rank, batch)
    if key not in _WORKLOAD_CACHE:
        _WORKLOAD_CACHE[key] = make_workload(name, rank, batch)
    b = _WORKLOAD_CACHE[key].batch(step)
    return step, b.table_ids, b.ids, b.bag_offsets


class BatchSource:
    """Seeded host batches of a workload's steps.  Generation runs in a
    `spawn` process pool (no CUDA state is inherited), so that the long
    streams' inputs are ready in seconds."""

    def __init__(self, procs: int):
        self.pool = None
        if procs > 1:
            import multiprocessing as mp
            self.pool = mp.get_context("spawn").Pool(procs)

    def batches(self, name: str, rank: int, batch: int, steps: int):
        jobs = [(name, rank, batch, s) for s in range(steps)]
        out = self.pool.map(_gen_batch, jobs, chunksize=1) if self.pool else [_gen_batch(j) for j in jobs]
        out.sort(key=lambda x: x[0])
        return [gen.Batch(t, i, o) for _, t, i, o in out]

    def close(self):
        if self.pool:
            self.pool.close()
            self.pool.join()
            self.pool = None


# ---------------------------------------------------------------------------
# the device run
# ---------------------------------------------------------------------------
def measure(dhs, w, host_batches, device, dist, warmup: int, reserve: int, grad_buffers: int,
            clock_index: int, want_traffic: bool, weights: str = "f32") -> dict:
    """Run the workload's first warmup + K steps (K = len(host_batches) -
    warmup) with every input resident in HBM, timing the last K with CUDA
    events on the launching stream (one event per step boundary; the time is
    the max over ranks).  Returns the measured quantities."""
    import torch
    total = len(host_batches)
    K = total - warmup
    batches = [(torch.from_numpy(b.table_ids).to(device), torch.from_numpy(b.ids).to(device),
                torch.from_numpy(b.bag_offsets).to(device), b.n, b.n_bags) for b in host_batches]
    n_max = max(x[3] for x in batches)
    nb_max = max(x[4] for x in batches)
    n_grad = min(total, grad_buffers)
    grads = [w.torch_grads(s, nb_max, device) for s in range(n_grad)]
    pooled = torch.empty((nb_max, w.dim), dtype=torch.float32, device=device)
    keys = torch.empty(max(1, n_max), dtype=torch.int64, device=device)
    # a step whose inputs fit in twice the L2 gets the L2 flushed before it
    step_bytes = n_max * 12 + (nb_max + 1) * 8 + nb_max * w.dim * 4
    flush = step_bytes < 2 * L2_BYTES
    fbuf = torch.empty(512 << 20, dtype=torch.uint8, device=device) if flush else None

    t = setup_table(dhs, w, reserve, weights)
    stream = torch.cuda.current_stream()

    def fwd(s):
        tids, ids, offs, n, nb = batches[s]
        k = keys[:n]
        dhs.dhs_pack_keys(tids, ids, out=k)
        dhs.embbag_forward(t, k, offs, out=pooled[:nb])

    def bwd(s):
        tids, ids, offs, n, nb = batches[s]
        dhs.embbag_backward_update(t, keys[:n], offs, grads[s % n_grad][:nb], w.lr)

    for s in range(warmup):
        fwd(s)
        bwd(s)
    torch.cuda.synchronize()
    c0 = dhs.ht_counters(t)
    dhs.ht_phase_times(t)  # clear
    dhs.ht_set_phase_timing(t, 2)  # IDMap growth inside the timed steps, reported on its own
    barrier(dist, device)
    torch.cuda.synchronize()
    # timed steps: events at each step's start, forward / backward boundary
    # and end only (per-phase events would perturb the launches they sit
    # between)
    E = lambda: torch.cuda.Event(enable_timing=True)  # noqa: E731
    marks = []
    with ClockSampler(clock_index) as clk:
        prev = None
        for s in range(warmup, total):
            if flush or prev is None:
                if flush:
                    fbuf.zero_()
                prev = E()
                prev.record(stream)
            mid, end = E(), E()
            fwd(s)
            mid.record(stream)
            bwd(s)
            end.record(stream)
            marks.append((prev, mid, end))
            prev = end
        torch.cuda.synchronize()
    spans = [a.elapsed_time(c) for a, _, c in marks]
    fwd_spans = [a.elapsed_time(b) for a, b, _ in marks]
    bwd_spans = [b.elapsed_time(c) for _, b, c in marks]
    ms_local = sum(spans)
    barrier(dist, device)
    dhs.ht_set_phase_timing(t, 0)
    growth = dhs.ht_phase_times(t)
    c1 = dhs.ht_counters(t)
    status = dhs.ht_sync(t)
    if status != 0:
        raise RuntimeError(f"{w.name}: device status {status} ({dhs.dhs_status_str(status)}) after the timed steps")
    # phase breakdown: the timed steps replayed on the same table with an
    # event around every phase (the replay inserts no keys: its forward
    # assignment phase is empty; the other phases do the timed steps' work)
    phases = {}
    if PHASE_TIMING:
        dhs.ht_phase_times(t)  # clear
        dhs.ht_set_phase_timing(t, True)
        for s in range(warmup, total):
            if flush:
                fbuf.zero_()
            fwd(s)
            bwd(s)
        torch.cuda.synchronize()
        dhs.ht_set_phase_timing(t, False)
        phases = dhs.ht_phase_times(t)
        status = dhs.ht_sync(t)
        if status != 0:
            raise RuntimeError(f"{w.name}: device status {status} after the phase replay")

    n_ids = sum(batches[s][3] for s in range(warmup, total))
    n_bags = sum(batches[s][4] for s in range(warmup, total))
    U = c1["unique_updated"] - c0["unique_updated"]
    M = c1["inserted"] - c0["inserted"]
    launches = c1["launches"] - c0["launches"] + K  # + one key-packing kernel per step
    ms = max_over_ranks(ms_local, dist, device)
    ids_all = sum_over_ranks(float(n_ids), dist, device)

    ab = alg_bytes(n_ids, n_bags, U, M, w.dim, w.optimizer, weights)
    peaks = load_peaks()
    ph_ms = {k: v[0] for k, v in phases.items()}
    ph_cnt = {k: v[1] for k, v in phases.items()}
    fwd_ms = max_over_ranks(sum(fwd_spans), dist, device)
    bwd_ms = max_over_ranks(sum(bwd_spans), dist, device)
    dom = max(("fwd_probe_pool", "bwd_seg_update"), key=lambda k: ph_ms.get(k, 0.0))
    dom_kernel = {"fwd_probe_pool": ("fwd_pool_refs_kernel" if n_ids >= POOL_SPLIT_LEN * n_bags
                                     else "fwd_probe_pool_kernel"),
                  "bwd_seg_update": "bwd_seg_kernel" if narrow_seg(w.dim, weights, n_ids, U)
                  else "bwd_segw_kernel"}[dom]
    dom_bytes = ((ab["fwd_refs"] if dom_kernel == "fwd_pool_refs_kernel" else ab["fwd_pool"])
                 if dom == "fwd_probe_pool" else ab["bwd_seg"])
    dom_launch_ms = ph_ms.get(dom, 0.0) / max(1, ph_cnt.get(dom, 0))
    dom_bytes_per_launch = dom_bytes / max(1, ph_cnt.get(dom, 0))
    achieved = dom_bytes_per_launch / (dom_launch_ms / 1e3) / 1e9 if dom_launch_ms else 0.0
    traffic = load_traffic(dom_kernel) if want_traffic else None
    roofline = {
        "bound": "hbm", "kernel": dom_kernel, "achieved": achieved, "peak": peaks["hbm_gbs"],
        "peak_source": peaks["source"], "unit": "GB/s", "frac": achieved / peaks["hbm_gbs"],
        "traffic": (traffic["dram_bytes_per_launch"] * dom_bytes_per_launch / traffic["alg_bytes_per_launch"]
                    if traffic and traffic.get("alg_bytes_per_launch") else None),
        "alg_bytes_per_launch": dom_bytes_per_launch, "launch_ms": dom_launch_ms,
    }

    def gbs(nbytes, t_ms):
        return nbytes / (t_ms / 1e3) / 1e9 if t_ms else None

    def frac(nbytes, t_ms):
        g = gbs(nbytes, t_ms)
        return g / peaks["hbm_gbs"] if g is not None else None

    res = {
        "value": ids_all / (ms / 1e3), "ms_per_step": ms / K, "steps": K, "warmup": warmup,
        "median_step_ms": statistics.median(spans) if spans else None,
        "flush": flush, "reserve": reserve,
        "fwd": {"ids_per_s": n_ids / (fwd_ms / 1e3) if fwd_ms else None, "ms_per_step": fwd_ms / K,
                "gbs": gbs(ab["fwd"], fwd_ms), "frac_of_peak": frac(ab["fwd"], fwd_ms)},
        "bwd": {"ids_per_s": n_ids / (bwd_ms / 1e3) if bwd_ms else None, "ms_per_step": bwd_ms / K,
                "gbs": gbs(ab["bwd"], bwd_ms), "frac_of_peak": frac(ab["bwd"], bwd_ms)},
        "step_gbs": gbs(ab["fwd"] + ab["bwd"], ms_local),
        "phases_ms_per_step": {k: v / K for k, v in ph_ms.items() if ph_cnt[k] and k != "idmap_growth"},
        "per_step": {"ids": n_ids / K, "bags": n_bags / K, "unique": U / K, "new": M / K},
        "roofline": roofline,
        "gpu_launches": launches,
        "table": {"rows": c1["rows"], "slots": c1["slots"], "blocks": c1["blocks"], "rehashes": c1["rehashes"],
                  "reserved_keys": reserve,
                  "timed_growth": {"rehashes": c1["rehashes"] - c0["rehashes"],
                                   "blocks_appended": c1["blocks"] - c0["blocks"],
                                   "device_allocs": c1["allocs"] - c0["allocs"],
                                   "alloc_ms": (c1["alloc_ns"] - c0["alloc_ns"]) / 1e6,
                                   "idmap_growth_ms": growth.get("idmap_growth", (0.0, 0))[0],
                                   "host_waits": c1["host_waits"] - c0["host_waits"],
                                   "host_wait_ms": (c1["host_wait_ns"] - c0["host_wait_ns"]) / 1e6}},
        "clocks": clk.summary(),
        "config": dict(workload_config(w, reserve, flush), weights=weights),
    }
    t.close()
    del grads, batches, fbuf, pooled, keys
    torch.cuda.empty_cache()
    return res


# the other configs, each run whole: (label, workload, weight storage,
# capacity policy, optimizer in place of the workload's or None)
EXTRA_WORKLOADS = (
    ("tiny_uniform", "tiny_uniform", "f32", "-1", None),
    ("sequence_bags", "sequence_bags", "f32", "-1", None),
    ("growth_stream", "growth_stream", "f32", "-1", None),
    ("growth_stream:on-demand", "growth_stream", "f32", "on-demand", None),
    ("hot_key", "hot_key", "f32", "-1", None),
    ("dlrm_merged_26:bf16", "dlrm_merged_26", "bf16", "-1", None),
    # the headline config with Adagrad's row-wise form (one accumulator per row)
    ("dlrm_merged_26:rowwise", "dlrm_merged_26", "f32", "-1", "adagrad_rowwise"),
    ("sequence_bags:bf16", "sequence_bags", "bf16", "-1", None),
)


def run_l2_peak(mib: int = 32, copies: int = 100, replays: int = 5):
    """Copy bandwidth of buffers that stay in L2 (two 32 MiB buffers, half
    the 126 MB L2): read + write bytes per second of `copies` back-to-back
    copies captured in one CUDA graph (no host launch gaps), replayed
    `replays` times after a warm-up and timed with CUDA events.  Prints one
    JSON line."""
    import torch
    n = mib << 20
    a = torch.empty(n, dtype=torch.uint8, device="cuda").fill_(1)
    b = torch.empty_like(a)
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        for _ in range(4):
            b.copy_(a)
    torch.cuda.current_stream().wait_stream(s)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        for i in range(copies):
            (b if i % 2 == 0 else a).copy_(a if i % 2 == 0 else b)
    g.replay()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(replays):
        g.replay()
    e1.record()
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1)
    del g
    print(json.dumps({"l2_copy_gbs": 2.0 * n * copies * replays / (ms / 1e3) / 1e9, "buffer_bytes": n,
                      "copies": copies * replays, "ms": ms, "method": "torch copy kernels in one CUDA graph"}))
    return 0


def run_pcie_peak(mib: int = 896, reps: int = 5):
    """Host <-> device copy rates from pinned memory: each direction alone
    and both at once on two streams (the bound of the end-to-end leg, whose
    steps copy their inputs in while the previous outputs come back).
    Prints one JSON line."""
    import torch
    n = mib << 20
    h_in = torch.empty(n, dtype=torch.uint8).pin_memory()
    h_out = torch.empty(n, dtype=torch.uint8).pin_memory()
    d_in = torch.empty(n, dtype=torch.uint8, device="cuda")
    d_out = torch.empty(n, dtype=torch.uint8, device="cuda")
    s_in, s_out = torch.cuda.Stream(), torch.cuda.Stream()

    def h2d():
        s_in.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(s_in):
            d_in.copy_(h_in, non_blocking=True)

    def d2h():
        s_out.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(s_out):
            h_out.copy_(d_out, non_blocking=True)

    def timed(fns):
        for f in fns:
            f()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for _ in range(reps):
            for f in fns:
                f()
        torch.cuda.current_stream().wait_stream(s_in)
        torch.cuda.current_stream().wait_stream(s_out)
        e1.record()
        torch.cuda.synchronize()
        return e0.elapsed_time(e1) / reps

    out = {"buffer_bytes": n, "method": "pinned host buffers, cudaMemcpyAsync through torch, CUDA events"}
    for name, fns in (("h2d_gbs", [h2d]), ("d2h_gbs", [d2h]), ("both_gbs_per_direction", [h2d, d2h])):
        out[name] = n / (timed(fns) / 1e3) / 1e9
    print(json.dumps(out))
    return 0


def run_dhs(args):
    world, rank, local = dist_env()
    procs = max(1, min(16, (os.cpu_count() or 2) // max(1, world) - 1))
    src = BatchSource(procs)  # before the first CUDA call
    import torch
    torch.cuda.set_device(local)
    device = torch.device("cuda", local)
    dist = init_dist(world, "nccl")
    import dynamic_hashed_sparse_b200 as dhs

    w = make_workload(args.workload, rank, args.batch)
    total = args.warmup + args.steps
    reserve = resolve_reserve(w, total, args.reserve_keys)
    host_batches = src.batches(args.workload, rank, args.batch, total)
    head = measure(dhs, w, host_batches, device, dist, args.warmup, reserve, args.grad_buffers, local,
                   want_traffic=(w.name == "dlrm_merged_26" and not args.batch))
    K = args.steps
    line = {
        "metric": METRIC, "value": head["value"], "unit": UNIT, "n_gpus": world, "steps": K,
        "warmup": args.warmup, "ms_per_step": head["ms_per_step"], "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "timing_valid": args.warmup >= 3,
        "dtype": "f32", "data": "synthetic", "config": head["config"],
    }
    for k in ("fwd", "bwd", "step_gbs", "median_step_ms", "phases_ms_per_step", "per_step", "roofline",
              "gpu_launches", "table", "clocks"):
        line[k] = head[k]

    # the other configs, each run whole with its own step count
    wanted = [] if args.workloads == "none" else (
        [e for e in EXTRA_WORKLOADS if not (e[0] == args.workload)] if args.workloads == "all"
        else [e for e in EXTRA_WORKLOADS if e[0] in args.workloads.split(",")])
    if wanted:
        extra = {}
        for label, name, weights, policy, opt in wanted:
            wx = make_workload(name, rank)
            if opt:
                wx.optimizer = opt
            wsteps = wx.steps
            wwarm = min(3, wsteps - 1)
            hb = src.batches(name, rank, 0, wsteps)
            r = measure(dhs, wx, hb, device, dist, wwarm, resolve_reserve(wx, wsteps, policy),
                        args.grad_buffers, local, want_traffic=False, weights=weights)
            extra[label] = {"ids_per_s": r["value"], "ms_per_step": r["ms_per_step"],
                            "median_step_ms": r["median_step_ms"], "steps": r["steps"], "warmup": r["warmup"],
                            "fwd": r["fwd"], "bwd": r["bwd"], "roofline": r["roofline"],
                            "phases_ms_per_step": r["phases_ms_per_step"], "per_step": r["per_step"],
                            "table": r["table"], "clocks": r["clocks"], "config": r["config"]}
            del hb
        line["workloads"] = extra
    src.close()

    if not args.no_e2e:
        line["e2e"] = run_e2e(dhs, w, host_batches, device, dist, reserve, args.warmup)
    del host_batches
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        ids, secs = time_oracle(make_workload(args.workload, 0, args.batch), args.cpu_steps, args.cpu_frac)
        line["cpu_baseline"] = {"value": ids / secs, "unit": UNIT, "cores": cpu_cores_used(), "kind": "oracle",
                                "sample": f"steps 0..{args.cpu_steps - 1} of {w.name}, first {args.cpu_frac:g} "
                                          f"of each batch's bags ({ids} ids, {secs:.1f} s), oracle "
                                          "single-threaded, no pre-inserted keys"}
    if dist is not None:
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(line), flush=True)
    return 0


def run_e2e(dhs, w, host_batches, device, dist, reserve, warmup):
    """The same steps through the public API with host inputs.  Every step
    copies its ids, table ids, bag offsets and gradients in from pinned host
    memory and copies its pooled output back, all inside the timed region.
    The copies are pipelined: step s+2's inputs go in on one copy stream and
    step s's pooled output comes back on another while step s computes
    (device inputs and outputs double-buffered, ordered by events), so a step
    costs about its larger transfer rather than the sum of both."""
    import torch

    total = len(host_batches)
    K = total - warmup
    hb = [(torch.from_numpy(b.table_ids).pin_memory(), torch.from_numpy(b.ids).pin_memory(),
           torch.from_numpy(b.bag_offsets).pin_memory(), b.n, b.n_bags) for b in host_batches]
    n_max = max(x[3] for x in hb)
    nb_max = max(x[4] for x in hb)
    hgrads = [w.torch_grads(s, nb_max, device).cpu().pin_memory() for s in range(2)]
    hpooled = [torch.empty((nb_max, w.dim), dtype=torch.float32).pin_memory() for _ in range(2)]

    def dbuf():
        return {"tids": torch.empty(max(1, n_max), dtype=torch.int32, device=device),
                "ids": torch.empty(max(1, n_max), dtype=torch.int64, device=device),
                "keys": torch.empty(max(1, n_max), dtype=torch.int64, device=device),
                "offs": torch.empty(nb_max + 1, dtype=torch.int64, device=device),
                "grad": torch.empty((nb_max, w.dim), dtype=torch.float32, device=device),
                "pooled": torch.empty((nb_max, w.dim), dtype=torch.float32, device=device)}

    bufs = [dbuf(), dbuf()]
    t = setup_table(dhs, w, reserve)
    s_in, s_cmp, s_out = torch.cuda.Stream(device), torch.cuda.Stream(device), torch.cuda.Stream(device)
    ev_in = [torch.cuda.Event() for _ in range(2)]
    ev_cmp = [torch.cuda.Event() for _ in range(2)]
    ev_out = [torch.cuda.Event() for _ in range(2)]
    moved = {"h2d": 0, "d2h": 0}

    def h2d(s):
        k = s % 2
        tids, ids, offs, n, nb = hb[s]
        d = bufs[k]
        with torch.cuda.stream(s_in):
            s_in.wait_event(ev_cmp[k])  # step s-2 has finished reading this buffer
            d["tids"][:n].copy_(tids, non_blocking=True)
            d["ids"][:n].copy_(ids, non_blocking=True)
            d["offs"][: nb + 1].copy_(offs, non_blocking=True)
            d["grad"][:nb].copy_(hgrads[s % 2][:nb], non_blocking=True)
            ev_in[k].record(s_in)
        moved["h2d"] += tids.numel() * 4 + ids.numel() * 8 + (nb + 1) * 8 + nb * w.dim * 4

    def compute_and_d2h(s):
        k = s % 2
        _, _, _, n, nb = hb[s]
        d = bufs[k]
        with torch.cuda.stream(s_cmp):
            s_cmp.wait_event(ev_in[k])
            s_cmp.wait_event(ev_out[k])  # step s-2's output has left this buffer
            kk = d["keys"][:n]
            dhs.dhs_pack_keys(d["tids"][:n], d["ids"][:n], out=kk, stream=s_cmp)
            dhs.embbag_forward(t, kk, d["offs"][: nb + 1], out=d["pooled"][:nb], stream=s_cmp)
            dhs.embbag_backward_update(t, kk, d["offs"][: nb + 1], d["grad"][:nb], w.lr, stream=s_cmp)
            ev_cmp[k].record(s_cmp)
        with torch.cuda.stream(s_out):
            s_out.wait_event(ev_cmp[k])
            hpooled[k][:nb].copy_(d["pooled"][:nb], non_blocking=True)
            ev_out[k].record(s_out)
        moved["d2h"] += nb * w.dim * 4

    def run(first, last):
        for s in range(first, min(first + 2, last)):
            h2d(s)
        for s in range(first, last):
            compute_and_d2h(s)
            if s + 2 < last:
                h2d(s + 2)

    run(0, warmup)
    torch.cuda.synchronize()
    moved["h2d"] = moved["d2h"] = 0
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier(dist, device)
    torch.cuda.synchronize()
    e0.record(s_in)
    run(warmup, total)
    s_out.wait_stream(s_cmp)
    s_out.wait_stream(s_in)
    e1.record(s_out)
    torch.cuda.synchronize()
    ms = max_over_ranks(e0.elapsed_time(e1), dist, device)
    ids = sum_over_ranks(float(sum(hb[s][3] for s in range(warmup, total))), dist, device)
    status = dhs.ht_sync(t)
    t.close()
    del bufs, hb, hgrads, hpooled
    torch.cuda.empty_cache()
    if status != 0:
        raise RuntimeError(f"device status {status} in the end-to-end run")
    return {"value": ids / (ms / 1e3), "unit": UNIT, "h2d_bytes_per_step": moved["h2d"] // K,
            "d2h_bytes_per_step": moved["d2h"] // K, "ms_per_step": ms / K,
            "pipeline": "H2D of step s+2 and D2H of step s overlap the compute of step s (3 streams, "
                        "double-buffered device inputs/outputs)"}


def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=40)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", default="dhs", choices=["dhs", "reference"])
    ap.add_argument("--l2-peak", action="store_true",
                    help="only measure the L2-resident copy bandwidth (the yardstick of L2-bound workloads)")
    ap.add_argument("--pcie-peak", action="store_true",
                    help="only measure host <-> device copy rates (the yardstick of the end-to-end leg)")
    ap.add_argument("--workload", default=WORKLOAD, choices=list(gen.NAMES))
    ap.add_argument("--workloads", default="all",
                    help="other configs measured after the headline, each run whole: 'all', 'none' or a "
                         "comma-separated list of labels (" + ", ".join(e[0] for e in EXTRA_WORKLOADS) + ")")
    ap.add_argument("--grad-buffers", type=int, default=32)
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-phases", action="store_true",
                    help="time the steps without the per-phase events (no phase breakdown)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-steps", type=int, default=5)
    ap.add_argument("--ref-frac", type=float, default=1.0 / 16)
    ap.add_argument("--reserve-keys", default="-1",
                    help="headline: capacity reserved (ht_reserve) before step 0; -1 = what the workload "
                         "reaches in the run plus one batch; 0 or 'on-demand' = grow inside the timed steps")
    ap.add_argument("--cpu-frac", type=float, default=1.0,
                    help="fraction of each batch's bags the CPU-baseline oracle processes")
    ap.add_argument("--batch", type=int, default=0,
                    help="samples per step (default: the workload's 65,536); smaller only for profiling")
    args = ap.parse_args(argv)
    global PHASE_TIMING
    PHASE_TIMING = not args.no_phases
    if args.warmup < 0 or args.steps < 1:
        ap.error("--steps must be >= 1 and --warmup >= 0")
    if args.l2_peak:
        return run_l2_peak()
    if args.pcie_peak:
        return run_pcie_peak()
    if args.impl == "reference":
        return run_reference(args)
    return run_dhs(args)


if __name__ == "__main__":
    sys.exit(main())
