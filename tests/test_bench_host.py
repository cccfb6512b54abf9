"""Host-side logic of bench.py that needs no GPU: the replica-mode reductions
over ranks (2 gloo ranks on CPU), the algorithmic-byte formula, and the
reference arm's JSON line."""
import json
import os
import socket
import subprocess
import sys

import pytest
import torch.multiprocessing as mp

from tests.conftest import ROOT


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    sys.path.insert(0, ROOT)
    import bench
    dist = bench.init_dist(world, "gloo")
    try:
        bench.barrier(dist)
        m = bench.max_over_ranks(10.0 * (rank + 1), dist)
        s = bench.sum_over_ranks(1000.0 + rank, dist)
        q.put((rank, m, s))
    finally:
        dist.destroy_process_group()


def test_replica_reductions_over_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    out = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert out == [(0, 20.0, 2001.0), (1, 20.0, 2001.0)]


def test_algorithmic_bytes_formula():
    sys.path.insert(0, ROOT)
    import bench
    ab = bench.alg_bytes(n=10, b=4, u=6, m=2, dim=8, opt="adagrad")
    R, S = 32, 64
    assert ab["fwd_pool"] == 8 * 10 + 8 * 5 + 16 * 6 + 16 * 2 + R * 4 + 4 * 8 * 4
    assert ab["fwd_assign"] == S * 2 + 16 * 2
    # the timed forward includes key packing (table ids 4 B + ids 8 B read, keys 8 B written)
    assert ab["pack"] == 20 * 10
    assert ab["fwd"] == ab["pack"] + ab["fwd_pool"] + ab["fwd_assign"]
    assert ab["fwd_refs"] == 8 * 5 + R * 6 + 4 * 8 * 4
    assert ab["bwd"] == 8 * 10 + 8 * 5 + 16 * 6 + 4 * 8 * 4 + 2 * S * 6
    assert bench.stride_floats(32, "adam") == 96 and bench.stride_floats(16, "adagrad_rowwise") == 20
    # bf16 weights: 2 bytes per weight, fp32 state
    assert bench.row_bytes(8, "adagrad", "bf16") == (16, 16 + 32)
    bf = bench.alg_bytes(n=10, b=4, u=6, m=2, dim=8, opt="adagrad", weights="bf16")
    assert bf["fwd_pool"] == ab["fwd_pool"] - 16 * 4 and bf["bwd"] == ab["bwd"] - 2 * 16 * 6


def test_reference_arm_line_on_cpu():
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--workload", "tiny_uniform", "--steps", "2", "--warmup", "1", "--ref-frac", "1"],
                       capture_output=True, text=True, timeout=300, cwd=ROOT)
    assert r.returncode == 0, r.stderr
    line = json.loads(r.stdout.strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["unit"] == "IDs/s" and line["value"] > 0
    assert line["cpu_baseline"]["kind"] == "oracle" and line["cpu_baseline"]["cores"] == 1
    assert line["e2e"]["h2d_bytes_per_step"] == 0


def test_pooled_generation_equals_serial_generation():
    """The bench's spawn-pool input generation yields the same seeded batches,
    in step order, as generating them one by one."""
    sys.path.insert(0, ROOT)
    import numpy as np

    import bench
    src = bench.BatchSource(2)
    try:
        got = src.batches("growth_stream", 0, 0, 3)
    finally:
        src.close()
    w = bench.make_workload("growth_stream", 0)
    for s, b in enumerate(got):
        ref = w.batch(s)
        assert np.array_equal(b.ids, ref.ids) and np.array_equal(b.table_ids, ref.table_ids)
        assert np.array_equal(b.bag_offsets, ref.bag_offsets)


def test_reserve_policy():
    sys.path.insert(0, ROOT)
    import bench
    w = bench.make_workload("growth_stream", 0)
    assert bench.resolve_reserve(w, 200, "on-demand") == 0
    assert bench.resolve_reserve(w, 200, "0") == 0
    assert bench.resolve_reserve(w, 200, "12345") == 12345
    assert bench.resolve_reserve(w, 10, "-1") == bench.default_reserve(w, 10)
    hot = bench.make_workload("hot_key", 0)
    assert bench.resolve_reserve(hot, 20, "on-demand") == 50_000_001


def test_segment_kernel_label_follows_the_library_rule():
    """The roofline names the segment kernel the library runs: the lane-group
    kernel below 32 floats, and for fp32 rows of 33-64 floats while rows get
    fewer than 8 ids on average; the warp kernel otherwise."""
    sys.path.insert(0, ROOT)
    import bench
    assert bench.narrow_seg(16, "f32", 1000, 10)
    assert not bench.narrow_seg(32, "f32", 1000, 999)          # 32 floats: the warp kernel
    assert bench.narrow_seg(64, "f32", 6_550_000, 1_780_000)   # sequence_bags: 3.7 ids per row
    assert not bench.narrow_seg(64, "f32", 5_240_000, 85_000)  # hot_key: 62 ids per row
    assert not bench.narrow_seg(64, "bf16", 6_550_000, 1_780_000)
    assert not bench.narrow_seg(128, "f32", 1_700_000, 380_000)
    assert not bench.narrow_seg(64, "f32", 100, 0)             # no backward seen yet
