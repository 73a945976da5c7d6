"""Benchmark of the MoDA fused forward (causal sequence + same-token depth
attention) on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload t64k]
    python bench.py --impl reference ...      (the float64 CPU oracle arm)

One step = one MoDA forward over the 64K long-context workload (B=1,
T=65536, Hq=32, Hkv=4, d=128, Ld=28, bf16, seeded N(0,1) inputs) with inputs
resident in HBM. With N > 1 GPUs (launched by torchrun, or by this script
itself when started as ``python bench.py --gpus N``) every rank is one
process on its own GPU: ``--partition replicas`` (default) runs the whole
workload on every rank (weak scaling); ``--partition heads`` gives rank r the
kv-heads [r*Hkv/N, (r+1)*Hkv/N) and their query heads (strong scaling: the
path needs no exchange across (b, kv-head)). NCCL carries only the barrier
and the max-over-ranks time. Rank 0 prints one JSON line.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import re
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import torch  # noqa: E402

from moda_inputs import WORKLOADS, make_depth_sel, make_inputs, pack_depth_sel, sample_rows  # noqa: E402

METRIC = "MoDA fwd TFLOP/s at T=64K (1×B200), % BF16 peak, overhead vs Ld=0 attention"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
TRAFFIC_FILE = os.path.join(ROOT, "profiles", "traffic.json")


def credited_flops(w, Ld=None) -> float:
    """4*B*Hq*d*(T(T+1)/2 + T*Ld): the two contractions (QK^T and PV) over the
    causal keys and the same-token depth keys."""
    Ld = w.Ld if Ld is None else Ld
    return 4.0 * w.B * w.Hq * w.d * (w.T * (w.T + 1) / 2 + w.T * Ld)


def row_flops(w, t) -> float:
    return 4.0 * w.d * (t + 1 + w.Ld)


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            return json.load(f), "measured"
    return FALLBACK_PEAKS, "fallback"


# ------------------------------------------------------------------ clocks
class ClockSampler:
    """nvidia-smi clocks / throttle reasons sampled every 200 ms."""

    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.path = None

    def start(self):
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.index), f"--query-gpu={self.Q}",
                 "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        rows = []
        with open(self.path) as f:
            for line in f:
                p = [x.strip() for x in line.split(",")]
                if len(p) >= 9:
                    rows.append(p)
        os.unlink(self.path)
        if not rows:
            return None
        sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        mx = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({n for r in rows for n, v in zip(names, r[5:9]) if v.lower() == "active"})
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(mx) if mx else None, "reasons": reasons, "samples": len(rows)}


# ------------------------------------------------------------------- timing
def dist_setup(n_gpus: int, cpu_only: bool = False):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if cpu_only:
        if world > 1:
            import datetime

            import torch.distributed as dist
            dist.init_process_group("gloo", timeout=datetime.timedelta(seconds=60))
        return world, rank, local
    if world > 1:
        import datetime

        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    else:
        torch.cuda.set_device(local)
    return world, rank, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(x: float, world: int, device: str = "cuda") -> float:
    if world == 1:
        return x
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def timed(fn, steps, warmup, world, per_launch=True):
    """W warm-up calls, then K calls between barrier+synchronize; returns
    (max-over-ranks ms per step, mean per-launch ms from events on the
    launching stream)."""
    for _ in range(warmup):
        fn()
    torch.cuda.synchronize()
    barrier(world)
    torch.cuda.synchronize()
    stream = torch.cuda.current_stream()
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(steps)]
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    t0.record(stream)
    for a, b in evs:
        a.record(stream)
        fn()
        b.record(stream)
    t1.record(stream)
    torch.cuda.synchronize()
    barrier(world)
    total = t0.elapsed_time(t1) / steps
    launch = statistics.mean(a.elapsed_time(b) for a, b in evs)
    return max_over_ranks(total, world), launch


def timed_interleaved(fns, steps_each, warmup, world, block=5):
    """Interleaved timing of several step functions: rounds of ``block`` calls
    of each function in turn (A x block, B x block, A x block, ...), so that
    slow drifts (clocks, power) hit every arm alike. Returns, per function,
    the max-over-ranks mean ms per call over ``steps_each`` calls."""
    for fn in fns:
        for _ in range(warmup):
            fn()
    torch.cuda.synchronize()
    barrier(world)
    stream = torch.cuda.current_stream()
    rounds = max(1, (steps_each + block - 1) // block)
    evs = [[] for _ in fns]
    for _ in range(rounds):
        for i, fn in enumerate(fns):
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            for _ in range(block):
                fn()
            b.record(stream)
            evs[i].append((a, b))
    torch.cuda.synchronize()
    barrier(world)
    return [max_over_ranks(sum(a.elapsed_time(b) for a, b in e) / (rounds * block), world)
            for e in evs]


# --------------------------------------------------------------- cpu oracle
def oracle_sample(w, seconds: float, x=None, rng_heads=None):
    """Time the float64 oracle on seed-sampled query rows of workload ``w``
    until about ``seconds`` of CPU work; returns (TFLOP/s, rows, secs)."""
    import oracle
    x = make_inputs(w) if x is None else x
    rows = sample_rows(w, 64)
    flops, done, t_start = 0.0, 0, time.perf_counter()
    h = 0
    while True:
        b = h // w.Hq % w.B
        oracle.forward_rows(x["q"], x["k"], x["v"], x["kd"], x["vd"], w.scale, b, h % w.Hq, rows)
        flops += sum(row_flops(w, t) for t in rows)
        done += len(rows)
        h += 1
        el = time.perf_counter() - t_start
        if el >= seconds:
            return flops / el / 1e12, done, el


def blas_threads():
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads") for i in threadpool_info() if i.get("user_api") == "blas"]
        return max(n) if n else os.cpu_count()
    except Exception:
        return os.cpu_count()


def reference_arm(args, w):
    """The float64 CPU oracle, as it stands, on the host cores (rank 0 only)."""
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    import oracle
    x = make_inputs(w)
    rows = sample_rows(w, args.ref_rows)

    def step(i):
        b, h = (i // w.Hq) % w.B, i % w.Hq
        oracle.forward_rows(x["q"], x["k"], x["v"], x["kd"], x["vd"], w.scale, b, h, rows)

    for i in range(args.warmup):
        step(i)
    t0 = time.perf_counter()
    for i in range(args.steps):
        step(args.warmup + i)
    el = time.perf_counter() - t0
    flops = sum(row_flops(w, t) for t in rows) * args.steps
    val = flops / el / 1e12
    sample = (f"{len(rows)} seed-sampled query rows (t=0..15, T-1, uniform) of one (b, head) per "
              f"step, heads in turn; credited FLOPs 4*d*(t+1+Ld) per row")
    line = {
        "metric": METRIC, "value": val, "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": el / args.steps * 1e3, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "impl": "reference",
        "config": workload_config(w),
        "cpu_baseline": {"value": val, "unit": "TFLOP/s", "cores": blas_threads(), "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": val, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def workload_config(w):
    nbytes = (w.B * w.T * w.Hq * w.d * 2 + 2 * w.B * w.T * w.Hkv * w.d
              + 2 * w.B * w.T * w.Ld * w.Hkv * w.d) * (2 if w.dtype == "bf16" else 4)
    return {"workload": f"{w.name}: B={w.B} T={w.T} Hq={w.Hq} Hkv={w.Hkv} (G={w.G}) d={w.d} "
                        f"Ld={w.Ld} {w.dtype}, q,k,v,kd,vd ~ N(0,1) seed {w.seed}",
            "B": w.B, "T": w.T, "Hq": w.Hq, "Hkv": w.Hkv, "d": w.d, "Ld": w.Ld,
            "l2": f"inputs+outputs {nbytes / 1e9:.2f} GB > 126 MB L2 (no flush)",
            "parallelism": "replicas"}


def make_step(moda, w, x, mode, kernel, depth_sel=None):
    """The timed step on device-resident inputs: one forward, or forward and
    backward; with ``depth_sel`` (int64 [B, T] slot masks on the device) the
    selected-depth entry points. Returns (step, launches of this library's
    kernels per step, out, lse)."""
    out = torch.empty_like(x["q"])
    lse = torch.empty((w.B, w.Hq, w.T), device="cuda", dtype=torch.float32)
    if mode == "fwd":
        if depth_sel is not None:
            def step():
                moda.moda_fwd_sel(x["q"], x["k"], x["v"], x["kd"], x["vd"], depth_sel, w.scale,
                                  out=out, lse=lse, impl=kernel)
            return step, 1, out, lse

        def step():
            moda.moda_fwd(x["q"], x["k"], x["v"], x["kd"], x["vd"], w.scale, out=out, lse=lse,
                          impl=kernel)
        return step, 1, out, lse
    grads = (torch.empty_like(x["q"]), torch.empty_like(x["k"]), torch.empty_like(x["v"]),
             torch.empty_like(x["kd"]) if w.Ld else None, torch.empty_like(x["vd"]) if w.Ld else None)
    ws = torch.empty(max(16, moda.moda_bwd_workspace_bytes(w.B, w.T, w.Hq, w.Hkv, w.d, w.Ld,
                                                            x["q"].dtype)),
                     device="cuda", dtype=torch.uint8)

    def step():
        if depth_sel is not None:
            moda.moda_fwd_sel(x["q"], x["k"], x["v"], x["kd"], x["vd"], depth_sel, w.scale,
                              out=out, lse=lse, impl=kernel)
            moda.moda_bwd_sel(x["q"], x["k"], x["v"], x["kd"], x["vd"], depth_sel, out, lse,
                              x["dout"], w.scale, grads=grads, workspace=ws, impl=kernel)
            return
        moda.moda_fwd(x["q"], x["k"], x["v"], x["kd"], x["vd"], w.scale, out=out, lse=lse,
                      impl=kernel)
        moda.moda_bwd(x["q"], x["k"], x["v"], x["kd"], x["vd"], out, lse, x["dout"], w.scale,
                      grads=grads, workspace=ws, impl=kernel)
    # forward 1; tensor-core backward: dq, one dk/dv launch (its grid also
    # holds the depth dk/dv CTAs), 2 conversions; SIMT backward: D~, dq,
    # dk/dv, depth (Ld > 0)
    bwd = 3 + (1 if w.Ld else 0) if kernel == "simt" else 4
    return step, 1 + bwd, out, lse


def measure_secondary(moda, w, world, kernel, steps=20, warmup=3):
    """Forward TFLOP/s and overhead vs Ld = 0 of another workload (the two
    arms interleaved, ``steps`` calls each); for the forward+backward
    workload also the backward time and fwd+bwd TFLOP/s."""
    x = {k: v.cuda() for k, v in make_inputs(w, with_dout=w.backward).items()}
    step, _, out, lse = make_step(moda, w, x, "fwd", kernel)
    x0 = dict(x, kd=None, vd=None)
    w0 = w.with_(Ld=0)
    step0, _, _, _ = make_step(moda, w0, x0, "fwd", kernel)
    ms, ms0 = timed_interleaved([step, step0], steps, warmup, world)
    res = {"config": f"B={w.B} T={w.T} Hq={w.Hq} Hkv={w.Hkv} d={w.d} Ld={w.Ld}",
           "fwd_ms": ms, "fwd_tflops": credited_flops(w) / (ms * 1e-3) / 1e12,
           "ld0_fwd_ms": ms0, "overhead_vs_ld0": ms / ms0 - 1.0,
           "depth_stream_gbs": depth_stream_gbs(w, ms, ms0),
           "timing": f"Ld and Ld=0 arms interleaved in blocks of 5, {steps} calls each"}
    if w.Ld and kernel != "simt":
        res["depth_q8"] = measure_q8(moda, w, x, world, kernel, step, step0, steps, warmup)
    # Selected depth: each token keeps a window of its most recent slots
    # (width uniform in [0, Ld]), the same FLOPs are issued (whole tiles).
    sel = pack_depth_sel(make_depth_sel(w, "window")).cuda() if w.Ld else None
    if sel is not None:
        steps_sel, _, _, _ = make_step(moda, w, x, "fwd", kernel, depth_sel=sel)
        ms_a, mss = timed_interleaved([step, steps_sel], steps, warmup, world)
        res.update({"sel_window_fwd_ms": mss, "sel_vs_all_slots": mss / ms_a - 1.0})
    if w.backward:
        stepb, _, _, _ = make_step(moda, w, x, "fwdbwd", kernel)
        ms_f, msb = timed_interleaved([step, stepb], steps, warmup, world)
        res.update({"fwd_bwd_ms": msb, "bwd_ms": msb - ms_f,
                    "bwd_tflops": 2.5 * credited_flops(w) / ((msb - ms_f) * 1e-3) / 1e12,
                    "fwd_bwd_tflops": 3.5 * credited_flops(w) / (msb * 1e-3) / 1e12})
        if sel is not None:
            stepbs, _, _, _ = make_step(moda, w, x, "fwdbwd", kernel, depth_sel=sel)
            msb2, msbs = timed_interleaved([stepb, stepbs], steps, warmup, world)
            res.update({"sel_window_fwd_bwd_ms": msbs, "sel_fwd_bwd_vs_all_slots": msbs / msb2 - 1.0})
    del x
    torch.cuda.empty_cache()
    return res


def measure_q8(moda, w, x, world, kernel, step_bf16, step_ld0, steps, warmup):
    """The 8-bit depth cache against the bf16 one and Ld = 0: three forwards
    interleaved. The depth stream shrinks from 2d to d + 4 bytes per row."""
    kd8, vd8, ks, vs = moda.moda_depth_quantize_q8(x["kd"], x["vd"])
    out = torch.empty_like(x["q"])
    lse = torch.empty((w.B, w.Hq, w.T), device="cuda", dtype=torch.float32)

    def step_q8():
        moda.moda_fwd_q8(x["q"], x["k"], x["v"], kd8, vd8, ks, vs, w.scale, out=out, lse=lse, impl=kernel)
    msb, msq, ms0 = timed_interleaved([step_bf16, step_q8, step_ld0], steps, warmup, world)
    q8_bytes = 2 * w.B * w.T * w.Ld * w.Hkv * (w.d + 4)
    return {"fwd_q8_ms": msq, "fwd_bf16_depth_ms": msb, "ld0_fwd_ms": ms0,
            "q8_overhead_vs_ld0": msq / ms0 - 1.0, "bf16_overhead_vs_ld0": msb / ms0 - 1.0,
            "q8_vs_bf16_depth": msq / msb - 1.0,
            "depth_bytes_q8": q8_bytes, "depth_bytes_bf16": depth_stream_bytes(w),
            "timing": f"bf16-depth, 8-bit-depth and Ld=0 forwards interleaved in blocks of 5, "
                      f"{steps} calls each"}


def measure_write_step(moda, w, x, world, steps, warmup):
    """The write step of one layer at this workload's shape: its key / value
    projections (x [B*T, Hq*d] @ W [Hq*d, Hkv*d], torch GEMMs standing in
    for the model's) written (a) to contiguous k, v and then copied into
    depth slot 0 by moda_depth_write, or (b) straight into the slot through
    moda_depth_slot_layout's strided views (no copy pass). Interleaved."""
    g = torch.Generator(device="cuda")
    g.manual_seed(7)
    dm = w.Hq * w.d
    xin = torch.randn(w.B * w.T, dm, device="cuda", generator=g).to(torch.bfloat16)
    wk = (torch.randn(dm, w.Hkv * w.d, device="cuda", generator=g) / dm ** 0.5).to(torch.bfloat16)
    wv = (torch.randn(dm, w.Hkv * w.d, device="cuda", generator=g) / dm ** 0.5).to(torch.bfloat16)
    k = torch.empty(w.B, w.T, w.Hkv, w.d, device="cuda", dtype=torch.bfloat16)
    v = torch.empty_like(k)
    kd, vd = x["kd"], x["vd"]
    views = (moda.depth_slot_view(kd, 0).view(w.B * w.T, w.Hkv * w.d),
             moda.depth_slot_view(vd, 0).view(w.B * w.T, w.Hkv * w.d))

    def copy_path():
        torch.mm(xin, wk, out=k.view(w.B * w.T, -1))
        torch.mm(xin, wv, out=v.view(w.B * w.T, -1))
        moda.moda_depth_write(k, v, kd, vd, 0)

    def strided_path():
        torch.mm(xin, wk, out=views[0])
        torch.mm(xin, wv, out=views[1])

    def write_only():
        moda.moda_depth_write(k, v, kd, vd, 0)
    ms_c, ms_s, ms_w = timed_interleaved([copy_path, strided_path, write_only], steps, warmup, world)
    del xin, wk, wv, k, v
    return {"proj_plus_depth_write_ms": ms_c, "proj_into_slot_ms": ms_s, "depth_write_ms": ms_w,
            "depth_write_gbs": 4 * w.B * w.T * w.Hkv * w.d * 2 / (ms_w * 1e-3) / 1e9,
            "saved_vs_copy": 1.0 - ms_s / ms_c,
            "timing": f"projections of one layer (torch GEMMs, x [{w.B * w.T}, {dm}] @ [{dm}, "
                      f"{w.Hkv * w.d}] for k and v) into contiguous k, v + moda_depth_write, or into "
                      f"the slot views; interleaved, {steps} calls each"}


def depth_stream_bytes(w) -> int:
    """Algorithmic bytes of the depth stream: kd and vd read once."""
    return 2 * w.B * w.T * w.Ld * w.Hkv * w.d * (2 if w.dtype == "bf16" else 4)


def depth_stream_gbs(w, ms, ms0):
    """Depth-stream bandwidth as the time the depth keys add: bytes(kd + vd)
    / (t(Ld) - t(Ld=0)); None when the difference is not positive (the depth
    work hidden within run-to-run noise)."""
    dt = (ms - ms0) * 1e-3
    return depth_stream_bytes(w) / dt / 1e9 if dt > 0 else None


def code_hash(paths) -> str:
    """SHA-256 (16 hex digits) of CUDA sources with their comments and all
    whitespace removed: it changes when the code changes, not when a comment
    or the layout does."""
    h = hashlib.sha256()
    for path in ([paths] if isinstance(paths, str) else paths):
        with open(path) as f:
            src = f.read()
        src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
        src = re.sub(r"//[^\n]*", "", src)
        src = re.sub(r"\s+", "", src)
        h.update(src.encode())
    return h.hexdigest()[:16]


# The forward kernel's code: its file and the headers its device code uses.
FWD_SOURCES = [os.path.join(ROOT, "depth_kv_attention_b200", "csrc", f)
               for f in ("moda_fwd_sm100.cu", "fwd_softmax.cuh", "sm100_ptx.cuh", "depth_mask.cuh")]


def traffic_for(kernel_srcs):
    """DRAM bytes per launch from the committed ncu summary, or None when the
    kernel's code changed since the counters were taken."""
    if not os.path.exists(TRAFFIC_FILE):
        return None
    with open(TRAFFIC_FILE) as f:
        t = json.load(f)
    if t.get("code_sha256_16") != code_hash(kernel_srcs):
        return None
    return t.get("dram_bytes_per_launch")


def relaunch_under_torchrun(argv, n_gpus: int) -> int:
    """``python bench.py --gpus N`` outside torchrun: start N ranks (one
    process per GPU) under torch.distributed.run on this node and return its
    exit status."""
    import socket
    with socket.socket() as sk:
        sk.bind(("127.0.0.1", 0))
        port = sk.getsockname()[1]
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", f"--nproc-per-node={n_gpus}",
           "--master-addr", "127.0.0.1", f"--master-port={port}", os.path.abspath(__file__)] + list(argv)
    return subprocess.call(cmd)


def shard_heads(w, x, rank: int, world: int):
    """Rank ``rank``'s share under head partitioning: kv-heads
    [rank*Hkv/world, (rank+1)*Hkv/world) and their G query heads each, as
    contiguous tensors (what a head-parallel layer holds). No exchange is
    needed: each GQA group's output depends only on its own q, k, v, kd, vd."""
    if w.Hkv % world:
        raise SystemExit(f"--partition heads needs the world size ({world}) to divide Hkv={w.Hkv}")
    hk = w.Hkv // world
    g0, g1 = rank * hk, (rank + 1) * hk
    q0, q1 = g0 * w.G, g1 * w.G
    xs = {"q": x["q"][:, :, q0:q1], "k": x["k"][:, :, g0:g1], "v": x["v"][:, :, g0:g1],
          "kd": x["kd"][:, :, :, g0:g1], "vd": x["vd"][:, :, :, g0:g1]}
    if "dout" in x:
        xs["dout"] = x["dout"][:, :, q0:q1]
    return w.with_(name=f"{w.name}-heads{g0}-{g1}", Hq=q1 - q0, Hkv=hk), \
        {k: v.contiguous() for k, v in xs.items()}


def dry_run(args, w) -> int:
    """``--dry-run``: the rank plumbing without a GPU. Ranks join over gloo,
    each takes its partition of the workload (shapes only, nothing timed),
    the shares are gathered and rank 0 prints one JSON line with the plan."""
    import torch.distributed as dist
    world, rank, _ = dist_setup(args.gpus, cpu_only=True)
    if args.partition == "heads" and world > 1:
        if w.Hkv % world:
            raise SystemExit(f"--partition heads needs the world size ({world}) to divide Hkv={w.Hkv}")
        hk = w.Hkv // world
        share = {"rank": rank, "kv_heads": [rank * hk, (rank + 1) * hk],
                 "q_heads": [rank * hk * w.G, (rank + 1) * hk * w.G],
                 "flops": credited_flops(w.with_(Hq=hk * w.G, Hkv=hk))}
    else:
        share = {"rank": rank, "kv_heads": [0, w.Hkv], "q_heads": [0, w.Hq],
                 "flops": credited_flops(w)}
    shares = [None] * world
    if world > 1:
        dist.all_gather_object(shares, share)
        barrier(world)
    else:
        shares = [share]
    if rank == 0:
        print(json.dumps({"dry_run": True, "n_gpus": world, "partition": args.partition,
                          "workload": w.name, "job_flops": sum(x["flops"] for x in shares),
                          "full_flops": credited_flops(w),
                          "scaling": "weak" if args.partition == "replicas" else "strong",
                          "shares": shares}), flush=True)
    if world > 1:
        dist.destroy_process_group()
    return 0


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default="t64k", choices=sorted(WORKLOADS))
    ap.add_argument("--kernel", default="auto", choices=["auto", "simt", "tc"])
    ap.add_argument("--partition", default="replicas", choices=["replicas", "heads"],
                    help="N > 1: every rank runs the whole workload (replicas, weak scaling) "
                         "or its share of the kv-heads (heads, strong scaling)")
    ap.add_argument("--cpu-seconds", type=float, default=12.0)
    ap.add_argument("--ref-rows", type=int, default=128)
    ap.add_argument("--e2e-steps", type=int, default=3)
    ap.add_argument("--extra-steps", type=int, default=20,
                    help="calls per arm of the interleaved overhead / pack / secondary timings")
    ap.add_argument("--no-extra", action="store_true",
                    help="skip the Ld=0, pack, e2e and secondary-workload runs")
    ap.add_argument("--mode", default="fwd", choices=["fwd", "fwdbwd"],
                    help="step = forward, or forward + backward (credited 3.5x the forward FLOPs)")
    ap.add_argument("--shape", default=None,
                    help="B,T,Hq,Hkv,d,Ld override of the workload (profiling runs)")
    ap.add_argument("--dry-run", action="store_true",
                    help="no GPU: start the ranks (gloo), print the partition plan, time nothing")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    if args.gpus > 1 and "WORLD_SIZE" not in os.environ and args.impl == "ours":
        return relaunch_under_torchrun(sys.argv[1:], args.gpus)
    w = WORKLOADS[args.workload]
    if args.shape:
        B, T, Hq, Hkv, d, Ld = (int(v) for v in args.shape.split(","))
        w = w.with_(name=f"{w.name}-shape", B=B, T=T, Hq=Hq, Hkv=Hkv, d=d, Ld=Ld)
    if args.impl == "reference":
        return reference_arm(args, w)
    if args.dry_run:
        return dry_run(args, w)

    import depth_kv_attention_b200 as moda

    world, rank, local = dist_setup(args.gpus)
    peaks, peaks_kind = load_peaks()
    w_full = w
    x_host = make_inputs(w, with_dout=args.mode == "fwdbwd")
    if args.partition == "heads" and world > 1:
        w, x_host = shard_heads(w, x_host, rank, world)
    x = {k: v.cuda() for k, v in x_host.items()}
    step, launches_per_step, out, lse = make_step(moda, w, x, args.mode, args.kernel)

    step()
    torch.cuda.synchronize()
    if moda.moda_device_status() != 0:
        raise RuntimeError("device status word set after the first step")
    clocks = ClockSampler(local)
    clocks.start()
    ms, launch_ms = timed(step, args.steps, args.warmup, world)
    clk = clocks.stop()
    mult = 3.5 if args.mode == "fwdbwd" else 1.0
    flops_rank = credited_flops(w) * mult
    # whole-job work: every replica's, or the one workload split over ranks
    flops_job = credited_flops(w_full) * mult * (world if args.partition == "replicas" else 1)
    value = flops_job / (ms * 1e-3) / 1e12
    extra = {}
    if not args.no_extra and args.mode == "fwd" and not args.shape:
        # the same library's own causal attention with Ld = 0, interleaved
        # with the Ld forward; the difference gives the depth stream's rate
        out0 = torch.empty_like(out)
        lse0 = torch.empty_like(lse)

        def step0():
            moda.moda_fwd(x["q"], x["k"], x["v"], None, None, w.scale, out=out0, lse=lse0,
                          impl=args.kernel)
        ms_a, ms0 = timed_interleaved([step, step0], args.extra_steps, args.warmup, world)
        extra["ld0_ms_per_step"] = ms0
        extra["overhead_vs_ld0"] = ms_a / ms0 - 1.0
        extra["overhead_timing"] = (f"Ld={w.Ld} and Ld=0 forwards interleaved in blocks of 5, "
                                    f"{args.extra_steps} calls each ({ms_a:.3f} vs {ms0:.3f} ms)")
        extra["depth_stream_gbs"] = depth_stream_gbs(w, ms_a, ms0)
        extra["depth_stream_bytes"] = depth_stream_bytes(w)
        if args.kernel != "simt":
            extra["depth_q8"] = measure_q8(moda, w, x, world, args.kernel, step, step0, args.extra_steps,
                                           args.warmup)
        del out0, lse0
        # the optional repack: moda_pack_depth + moda_fwd_packed against the
        # forward on the native depth layout
        packed = moda.moda_pack_depth(x["kd"], x["vd"])
        outp = torch.empty_like(out)

        def step_pack():
            moda.moda_pack_depth(x["kd"], x["vd"], packed=packed)

        def step_fwd_packed():
            moda.moda_fwd_packed(x["q"], x["k"], x["v"], packed, w.Ld, w.scale, out=outp, lse=lse)

        def step_pack_fwd():
            step_pack()
            step_fwd_packed()
        ms_n, ms_p, ms_fp, ms_pf = timed_interleaved([step, step_pack, step_fwd_packed, step_pack_fwd],
                                                     args.extra_steps, args.warmup, world)
        extra["write_step"] = measure_write_step(moda, w, x, world, args.extra_steps, args.warmup)
        extra["pack_depth"] = {
            "t_fwd_native_ms": ms_n, "t_pack_ms": ms_p, "t_fwd_packed_ms": ms_fp,
            "t_pack_plus_fwd_packed_ms": ms_pf, "pack_vs_native": ms_pf / ms_n - 1.0,
            "pack_gbs": 2 * depth_stream_bytes(w) / (ms_p * 1e-3) / 1e9,
            "timing": f"four arms interleaved in blocks of 5, {args.extra_steps} calls each"}
        del packed, outp
        torch.cuda.empty_cache()

    e2e = None
    if not args.no_extra and args.mode == "fwd":
        pinned = {k: v.pin_memory() for k, v in x_host.items()}
        out_h = torch.empty(out.shape, dtype=out.dtype, pin_memory=True)
        lse_h = torch.empty(lse.shape, dtype=lse.dtype, pin_memory=True)
        staging = torch.empty(moda.moda_fwd_host_staging_bytes(w.B, w.T, w.Hq, w.Hkv, w.d, w.Ld,
                                                                x_host["q"].dtype),
                              dtype=torch.uint8, device="cuda")

        def step_e2e():
            moda.moda_fwd_from_host(pinned["q"], pinned["k"], pinned["v"], pinned["kd"], pinned["vd"],
                                    w.scale, out_host=out_h, lse_host=lse_h, staging=staging)
        ms_e2e, _ = timed(step_e2e, args.e2e_steps, 3, world)
        h2d = sum(v.numel() * v.element_size() for v in pinned.values())
        d2h = out_h.numel() * out_h.element_size() + lse_h.numel() * lse_h.element_size()
        e2e = {"value": flops_job / (ms_e2e * 1e-3) / 1e12, "unit": "TFLOP/s",
               "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": ms_e2e,
               "api": "moda_fwd_host (C ABI): pinned host inputs -> device staging -> forward -> "
                      "out, lse to pinned host (copies and forward pipelined over chunks of query "
                      "tokens), then a stream synchronize"}
        del staging
        torch.cuda.empty_cache()

    kernel_src = ([os.path.join(ROOT, "depth_kv_attention_b200", "csrc", "moda_simt.cu")]
                  if args.kernel == "simt" else FWD_SOURCES)
    peak = peaks["bf16_tflops"]
    achieved = flops_rank / (launch_ms * 1e-3) / 1e12
    roofline = {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                "frac": achieved / peak, "traffic": traffic_for(kernel_src),
                "peak_kind": f"{peaks_kind} bf16 burst (cuBLAS 8192^3)",
                "frac_of_sustained": achieved / peaks["bf16_tflops_sustained"],
                "frac_of_nominal_2250": achieved / 2250.0}

    if not args.no_extra and not args.shape and args.partition == "replicas":
        extra["other_workloads"] = {
            name: measure_secondary(moda, WORKLOADS[name], world, args.kernel, steps=args.extra_steps)
            for name in ("t4k", "t16k_b2", "g32_fwdbwd") if name != w.name}

    cpu = None
    if rank == 0 and world == 1 and args.cpu_seconds > 0 and args.mode == "fwd":
        tf, nrows, secs = oracle_sample(w, args.cpu_seconds, x_host)
        cpu = {"value": tf, "unit": "TFLOP/s", "cores": blas_threads(), "kind": "oracle",
               "sample": f"{nrows} seed-sampled query rows (64 per (b, head), heads in turn) "
                         f"of the same workload, {secs:.1f} s, credited FLOPs 4*d*(t+1+Ld) per row"}

    if rank == 0:
        cfg = workload_config(w_full)
        cfg["parallelism"] = (f"replicas x{world}" if args.partition == "replicas"
                              else f"kv-head shards x{world}")
        line = {
            "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
            "higher_is_better": True,
            "scaling": "weak" if args.partition == "replicas" else "strong",
            "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic", "config": cfg,
            "pct_of_bf16_peak": 100.0 * achieved / peak,
            "clocks": clk, "e2e": e2e, "gpu_launches": launches_per_step * args.steps,
            "roofline": roofline, "cpu_baseline": cpu, "kernel_family": args.kernel,
            "mode": args.mode,
        }
        line.update(extra)
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
