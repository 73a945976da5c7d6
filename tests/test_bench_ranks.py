"""Host logic of the N>1 bench path on CPU: world_size-2 gloo ranks.

bench.py runs N independent replicas (the path shards across (b, kv-head)
with no exchange); the only collectives are the barrier and the
max-over-ranks timing, and the reference arm runs on rank 0 alone."""
import os
import sys

import pytest
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    sys.path.insert(0, ROOT)
    import bench
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        m = bench.max_over_ranks(10.0 + 5.0 * rank, world, device="cpu")
        bench.barrier(world)
        # replicas: each rank's value counts its own units; the job value is
        # units of all ranks over the max time
        w = bench.WORKLOADS["t4k"]
        value = bench.credited_flops(w) * world / (m * 1e-3) / 1e12
        q.put((rank, m, value))
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_and_weak_scaling_value():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = 29500 + os.getpid() % 2000
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
    res = sorted(q.get(timeout=5) for _ in range(2))
    assert all(p.exitcode == 0 for p in procs)
    assert [r[1] for r in res] == [15.0, 15.0]
    assert res[0][2] == res[1][2]


def test_reference_arm_runs_on_rank0_only(monkeypatch):
    sys.path.insert(0, ROOT)
    import bench
    monkeypatch.setenv("RANK", "1")
    monkeypatch.setenv("WORLD_SIZE", "2")

    class A:
        steps, warmup, ref_rows = 1, 3, 4
    assert bench.reference_arm(A, bench.WORKLOADS["tiny_f32"]) == 0


def test_launcher_starts_two_ranks_and_partitions_heads():
    """``python bench.py --gpus 2`` outside torchrun starts the two ranks
    itself (torch.distributed.run, gloo in the dry run); the kv-head shards
    of the ranks are disjoint, cover every head and add up to the whole
    workload's FLOPs (strong scaling)."""
    import json
    import subprocess
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--gpus", "2", "--dry-run",
                        "--partition", "heads", "--workload", "t4k"],
                       capture_output=True, text=True, timeout=240, cwd=ROOT)
    assert r.returncode == 0, r.stderr[-2000:]
    line = json.loads([ln for ln in r.stdout.splitlines() if ln.startswith("{")][-1])
    assert line["n_gpus"] == 2 and line["scaling"] == "strong"
    shares = sorted(line["shares"], key=lambda s: s["rank"])
    assert [s["kv_heads"] for s in shares] == [[0, 2], [2, 4]]
    assert [s["q_heads"] for s in shares] == [[0, 16], [16, 32]]
    assert line["job_flops"] == line["full_flops"]


def test_head_shards_need_no_exchange():
    """The oracle's output for each rank's kv-head shard, computed from that
    shard's inputs alone, equals the full workload's output on those heads:
    the head partition needs no data exchange between ranks."""
    import numpy as np
    sys.path.insert(0, ROOT)
    import bench
    import oracle
    from moda_inputs import Workload, make_inputs
    w = Workload("shard", 2, 40, 8, 4, 16, 3, "f32", 77)
    x = make_inputs(w)
    full, full_lse = oracle.forward(x["q"], x["k"], x["v"], x["kd"], x["vd"], w.scale)
    for world in (2, 4):
        for rank in range(world):
            ws, xs = bench.shard_heads(w, x, rank, world)
            o, l = oracle.forward(xs["q"], xs["k"], xs["v"], xs["kd"], xs["vd"], ws.scale)
            q0 = rank * (w.Hq // world)
            np.testing.assert_array_equal(o, full[:, :, q0:q0 + ws.Hq])
            np.testing.assert_array_equal(l, full_lse[:, q0:q0 + ws.Hq])
