"""Benchmark of the MoDA fused forward (causal sequence + same-token depth
attention) on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload t64k]
    python bench.py --impl reference ...      (the float64 CPU oracle arm)

One step = one MoDA forward over the 64K long-context workload (B=1,
T=65536, Hq=32, Hkv=4, d=128, Ld=28, bf16, seeded N(0,1) inputs) with inputs
resident in HBM. N>1 runs N independent replicas (one process per GPU, no
data-path collective; the barrier and the max-over-ranks timing use NCCL).
Rank 0 prints one JSON line.
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
def dist_setup(n_gpus: int):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
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
    # forward 1; backward: D, depth dq, depth dk/dv (Ld > 0), sequence, 3 conversions
    return step, 1 + 6 + (1 if w.Ld else 0), out, lse


def measure_secondary(moda, w, world, kernel, steps=5, warmup=3):
    """Forward TFLOP/s and overhead vs Ld = 0 of another workload; for the
    forward+backward workload also the backward time and fwd+bwd TFLOP/s."""
    x = {k: v.cuda() for k, v in make_inputs(w, with_dout=w.backward).items()}
    step, _, out, lse = make_step(moda, w, x, "fwd", kernel)
    ms, _ = timed(step, steps, warmup, world)
    x0 = dict(x, kd=None, vd=None)
    w0 = w.with_(Ld=0)
    step0, _, _, _ = make_step(moda, w0, x0, "fwd", kernel)
    ms0, _ = timed(step0, steps, warmup, world)
    res = {"config": f"B={w.B} T={w.T} Hq={w.Hq} Hkv={w.Hkv} d={w.d} Ld={w.Ld}",
           "fwd_ms": ms, "fwd_tflops": credited_flops(w) / (ms * 1e-3) / 1e12,
           "ld0_fwd_ms": ms0, "overhead_vs_ld0": ms / ms0 - 1.0}
    # Selected depth: each token keeps a window of its most recent slots
    # (width uniform in [0, Ld]), the same FLOPs are issued (whole tiles).
    sel = pack_depth_sel(make_depth_sel(w, "window")).cuda() if w.Ld else None
    if sel is not None:
        steps_sel, _, _, _ = make_step(moda, w, x, "fwd", kernel, depth_sel=sel)
        mss, _ = timed(steps_sel, steps, warmup, world)
        res.update({"sel_window_fwd_ms": mss, "sel_vs_all_slots": mss / ms - 1.0})
    if w.backward:
        stepb, _, _, _ = make_step(moda, w, x, "fwdbwd", kernel)
        msb, _ = timed(stepb, steps, warmup, world)
        res.update({"fwd_bwd_ms": msb, "bwd_ms": msb - ms,
                    "bwd_tflops": 2.5 * credited_flops(w) / ((msb - ms) * 1e-3) / 1e12,
                    "fwd_bwd_tflops": 3.5 * credited_flops(w) / (msb * 1e-3) / 1e12})
        if sel is not None:
            stepbs, _, _, _ = make_step(moda, w, x, "fwdbwd", kernel, depth_sel=sel)
            msbs, _ = timed(stepbs, steps, warmup, world)
            res.update({"sel_window_fwd_bwd_ms": msbs, "sel_fwd_bwd_vs_all_slots": msbs / msb - 1.0})
    del x
    torch.cuda.empty_cache()
    return res


def code_hash(path: str) -> str:
    """SHA-256 (16 hex digits) of a CUDA source with its comments and all
    whitespace removed: it changes when the code changes, not when a comment
    or the layout does."""
    with open(path) as f:
        src = f.read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    src = re.sub(r"//[^\n]*", "", src)
    src = re.sub(r"\s+", "", src)
    return hashlib.sha256(src.encode()).hexdigest()[:16]


def traffic_for(kernel_src: str):
    """DRAM bytes per launch from the committed ncu summary, or None when the
    kernel's code changed since the counters were taken."""
    if not os.path.exists(TRAFFIC_FILE):
        return None
    with open(TRAFFIC_FILE) as f:
        t = json.load(f)
    if t.get("code_sha256_16") != code_hash(kernel_src):
        return None
    return t.get("dram_bytes_per_launch")


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default="t64k", choices=sorted(WORKLOADS))
    ap.add_argument("--kernel", default="auto", choices=["auto", "simt", "tc"])
    ap.add_argument("--cpu-seconds", type=float, default=12.0)
    ap.add_argument("--ref-rows", type=int, default=128)
    ap.add_argument("--e2e-steps", type=int, default=3)
    ap.add_argument("--no-extra", action="store_true", help="skip the Ld=0 and e2e runs")
    ap.add_argument("--mode", default="fwd", choices=["fwd", "fwdbwd"],
                    help="step = forward, or forward + backward (credited 3.5x the forward FLOPs)")
    ap.add_argument("--shape", default=None,
                    help="B,T,Hq,Hkv,d,Ld override of the workload (profiling runs)")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    w = WORKLOADS[args.workload]
    if args.shape:
        B, T, Hq, Hkv, d, Ld = (int(v) for v in args.shape.split(","))
        w = w.with_(name=f"{w.name}-shape", B=B, T=T, Hq=Hq, Hkv=Hkv, d=d, Ld=Ld)
    if args.impl == "reference":
        return reference_arm(args, w)

    import depth_kv_attention_b200 as moda

    world, rank, local = dist_setup(args.gpus)
    peaks, peaks_kind = load_peaks()
    x_host = make_inputs(w, with_dout=args.mode == "fwdbwd")
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
    flops = credited_flops(w) * (3.5 if args.mode == "fwdbwd" else 1.0)
    value = flops * world / (ms * 1e-3) / 1e12

    extra = {}
    if not args.no_extra and args.mode == "fwd" and not args.shape:
        # the same library's own causal attention with Ld = 0
        out0 = torch.empty_like(out)

        def step0():
            moda.moda_fwd(x["q"], x["k"], x["v"], None, None, w.scale, out=out0, lse=lse,
                          impl=args.kernel)
        ms0, _ = timed(step0, args.steps, args.warmup, world)
        extra["ld0_ms_per_step"] = ms0
        extra["overhead_vs_ld0"] = ms / ms0 - 1.0
        del out0

    e2e = None
    if not args.no_extra and args.mode == "fwd":
        pinned = {k: v.pin_memory() for k, v in x_host.items()}
        out_h = torch.empty(out.shape, dtype=out.dtype, pin_memory=True)
        lse_h = torch.empty(lse.shape, dtype=lse.dtype, pin_memory=True)
        bufs = dict(x, out=out, lse=lse)

        def step_e2e():
            moda.moda_fwd_from_host(pinned["q"], pinned["k"], pinned["v"], pinned["kd"], pinned["vd"],
                                    w.scale, out_host=out_h, lse_host=lse_h, dev_bufs=bufs,
                                    impl=args.kernel)
        ms_e2e, _ = timed(step_e2e, args.e2e_steps, 3, world)
        h2d = sum(v.numel() * v.element_size() for v in pinned.values())
        d2h = out_h.numel() * out_h.element_size() + lse_h.numel() * lse_h.element_size()
        e2e = {"value": flops * world / (ms_e2e * 1e-3) / 1e12, "unit": "TFLOP/s",
               "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": ms_e2e}

    kernel_src = os.path.join(ROOT, "depth_kv_attention_b200", "csrc",
                              "moda_simt.cu" if args.kernel == "simt" else "moda_fwd_sm100.cu")
    peak = peaks["bf16_tflops"]
    achieved = flops / (launch_ms * 1e-3) / 1e12
    roofline = {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                "frac": achieved / peak, "traffic": traffic_for(kernel_src),
                "peak_kind": f"{peaks_kind} bf16 burst (cuBLAS 8192^3)",
                "frac_of_sustained": achieved / peaks["bf16_tflops_sustained"],
                "frac_of_nominal_2250": achieved / 2250.0}

    if not args.no_extra and not args.shape:
        extra["other_workloads"] = {name: measure_secondary(moda, WORKLOADS[name], world, args.kernel)
                                    for name in ("t4k", "t16k_b2", "g32_fwdbwd") if name != w.name}

    cpu = None
    if rank == 0 and world == 1 and args.cpu_seconds > 0 and args.mode == "fwd":
        tf, nrows, secs = oracle_sample(w, args.cpu_seconds, x_host)
        cpu = {"value": tf, "unit": "TFLOP/s", "cores": blas_threads(), "kind": "oracle",
               "sample": f"{nrows} seed-sampled query rows (64 per (b, head), heads in turn) "
                         f"of the same workload, {secs:.1f} s, credited FLOPs 4*d*(t+1+Ld) per row"}

    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic", "config": workload_config(w),
            "pct_of_bf16_peak": 100.0 * value / world / peak,
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
