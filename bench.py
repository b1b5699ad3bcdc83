"""Prop2D forward benchmark (one JSON line on rank 0).

A step is one gspn_prop2d_fwd call over one batch of the workload (default:
the C-GSPN 1K layer, B=32, Cc=64, 74x74, bf16 inputs, fp32 state, four
directions, per-channel weights), inputs resident in HBM; compact-mode
workloads (shared weights) call gspn_prop2d_fwd_ws with a workspace.  The metric is
Prop2D forward GB/s of algorithmic traffic (x once; lambda, u and the three
logits once per direction; y once), whole job over all ranks.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--workload 1k]
  python bench.py --impl reference ...   (the CPU oracle on host cores)

Multi-GPU (torchrun, one rank per GPU): every rank runs its own batch (the
planes are independent, so there is no collective on the data path); time
is the max over ranks.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import torch  # noqa: E402

from spatial_propagation_vision_b200.workloads import WORKLOADS, workload_inputs  # noqa: E402

L2_BYTES = 126 * 1024 * 1024
NOMINAL_HBM_GBS = 8000.0   # B200 HBM3e nominal, reported beside the measured-peak fraction
FALLBACK_HBM_GBS = 6650.0


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            p = json.load(f)
        return float(p["hbm_gbs"]), "measured"
    return FALLBACK_HBM_GBS, "fallback"


# The sources of each kernel's device code: the headers that define it and
# the translation units (and their launch headers) that instantiate it.
KERNEL_UNITS = {
    "prop2d_dir_kernel": ("device_common.cuh", "prop2d_dir.cuh", "dir_"),
    "prop2d_pair_kernel": ("device_common.cuh", "prop2d_pair.cuh", "pair_"),
    "prop2d_split_kernel": ("device_common.cuh", "prop2d_dir.cuh", "prop2d_split.cuh", "split_"),
    "prop2d_generic_kernel": ("device_common.cuh", "prop2d_generic.cuh", "generic_"),
    "prop2d_norm_kernel": ("device_common.cuh", "prop2d_norm.cuh", "norm_"),
    "prop2d_bwd_kernel": ("device_common.cuh", "prop2d_bwd.cuh", "bwd_"),
}


def kernel_sources_sha(kernel: str = "prop2d_dir_kernel") -> str:
    """sha256 over the code (comments and blank lines left out) of one
    kernel's device sources, sorted by name: the files under csrc/ whose
    names start with one of the kernel's KERNEL_UNITS entries. Host-only files (the C ABI, launch.h, other kernels'
    launchers) are left out, so they can change without invalidating a
    profile; the planner's choice is checked separately, since a profile also
    records the launch geometry it was taken with."""
    import glob
    import hashlib
    import re
    h = hashlib.sha256()
    units = KERNEL_UNITS.get(kernel, ())
    files = sorted(f for f in glob.glob(os.path.join(ROOT, "spatial_propagation_vision_b200", "csrc", "*"))
                   if os.path.basename(f).startswith(units))
    # comments and blank lines do not change the code: they are left out
    strip = re.compile(r"//[^\n]*|/\*.*?\*/", re.S)
    for f in files:
        h.update(os.path.basename(f).encode())
        with open(f, encoding="utf-8") as fh:
            code = strip.sub("", fh.read())
        h.update("\n".join(ln.rstrip() for ln in code.splitlines() if ln.strip()).encode())
    return h.hexdigest()


KERNEL_OF_PATH = {"pair": "prop2d_pair_kernel", "dir": "prop2d_dir_kernel",
                  "dir-shared": "prop2d_dir_kernel", "dir-yglobal": "prop2d_dir_kernel",
                  "dir-banded": "prop2d_dir_kernel", "dir-half": "prop2d_dir_kernel",
                  "split": "prop2d_split_kernel", "generic": "prop2d_generic_kernel"}


def profile_path(kernel: str, workload: str) -> str:
    return os.path.join(ROOT, "profiles", f"{kernel.replace('_kernel', '')}_{workload}.md")


def profiled_traffic(kernel: str, workload: str, launch: dict | None = None):
    """DRAM bytes per launch from the committed ncu summary of this kernel on
    this workload, if it was captured on the current device sources and (when
    `launch` is given) with the same grid, block and shared memory; else None."""
    import re
    path = profile_path(kernel, workload)
    if not os.path.exists(path):
        return None
    text = open(path).read()
    sha = re.search(r"kernel_sources_sha256:\s*([0-9a-f]{64})", text)
    tb = re.search(r"traffic_bytes_per_launch:\s*([0-9]+)", text)
    if not sha or not tb or sha.group(1) != kernel_sources_sha(kernel):
        return None
    if launch is not None:
        geo = re.search(r"launch_geometry:\s*grid=(\d+)\s+block=(\d+)\s+smem=(\d+)", text)
        if not geo or tuple(int(g) for g in geo.groups()) != (launch["grid"], launch["block"], launch["smem"]):
            return None
    return int(tb.group(1))


def dist_env():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


def max_over_ranks(value: float, world: int, device) -> float:
    if world == 1:
        return value
    import torch.distributed as dist
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_value(bytes_per_rank: int, world: int, seconds: float) -> float:
    """Whole-job GB/s: bytes processed by all ranks over the slowest rank's time."""
    return bytes_per_rank * world / seconds / 1e9


# ----------------------------------------------------------------------------
# clocks during the timed region
# ----------------------------------------------------------------------------

class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.samples = []
        self.proc = None
        self.t0 = self.t1 = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "20"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
            return
        self.thread = threading.Thread(target=self._read, daemon=True)
        self.thread.start()
        deadline = time.time() + 5
        while not self.samples and time.time() < deadline:
            time.sleep(0.02)

    def _read(self):
        for line in self.proc.stdout:
            self.samples.append((time.time(), line.strip()))

    def mark(self, which):
        setattr(self, which, time.time())

    def stop(self):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def window(self, a, b):
        """Statistics of the samples taken between marks `a` and `b`."""
        rows = []
        for ts, line in self.samples:
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            rows.append((ts, parts))
        t0, t1 = getattr(self, a, None), getattr(self, b, None)
        use = [r for r in rows if t0 is not None and t1 is not None and t0 <= r[0] <= t1]
        if not use:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}

        def num(s):
            try:
                return float(s)
            except ValueError:
                return None
        sm = [num(p[1]) for _, p in use if num(p[1]) is not None]
        smax = [num(p[2]) for _, p in use if num(p[2]) is not None]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({n for _, p in use for n, v in zip(names, p[5:9]) if v.strip() == "Active"})
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(smax) if smax else None,
                "reasons": reasons, "samples": len(use),
                "power_w_max": max((num(p[3]) or 0.0) for _, p in use)}

    def summary(self):
        """Clocks of the timed region; when it was too short for a sample
        (20 ms polling), those of the load window run just before it, which
        is said so in `source`."""
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"],
                    "samples": 0, "source": "none"}
        timed = self.window("t0", "t1")
        load = self.window("l0", "l1")
        if timed["samples"]:
            out = dict(timed, source="timed region")
        else:
            out = dict(load, source="no sample in the timed region (shorter than the 20 ms "
                                    "polling interval); load window of the same call run for "
                                    "about 1 s just before it")
        out["timed_region_samples"] = timed["samples"]
        out["load_window"] = load
        return out


# ----------------------------------------------------------------------------
# CPU oracle (reference arm and cpu_baseline)
# ----------------------------------------------------------------------------

def oracle_planes_seconds(inp64, planes):
    import oracle
    t0 = time.perf_counter()
    for (b, c) in planes:
        oracle.prop2d(inp64["x"][b:b + 1, c:c + 1], inp64["lam"][b:b + 1, :, c:c + 1],
                      inp64["wlogit"][b:b + 1, :, c:c + 1] if inp64["wlogit"].shape[2] > 1
                      else inp64["wlogit"][b:b + 1], inp64["u"][b:b + 1, :, c:c + 1])
    return time.perf_counter() - t0


def cpu_inputs_f64(w, seed=0, planes=None):
    inp = workload_inputs(w, seed=seed)
    return {k: v.double().numpy() for k, v in inp.items()}


def cpu_oracle_baseline(w, budget_s=12.0, max_passes=20):
    """The oracle as it stands, one host core, on whole passes over the
    workload's planes (repeated until about budget_s)."""
    inp = cpu_inputs_f64(w)
    planes = [(b, c) for b in range(w.B) for c in range(w.Cc)]
    per_plane = w.algorithmic_bytes() / len(planes)
    done, secs = 0, 0.0
    chunk = 64
    t_start = time.perf_counter()
    while done < max_passes * len(planes):
        sel = [planes[(done + i) % len(planes)] for i in range(chunk)]
        secs += oracle_planes_seconds(inp, sel)
        done += chunk
        if time.perf_counter() - t_start > budget_s:
            break
    return {"value": per_plane * done / secs / 1e9, "unit": "GB/s", "cores": 1, "kind": "oracle",
            "sample": f"{done} planes ({done / len(planes):.2f} passes) of the {w.name} workload, "
                      f"fp64 single-threaded C, {secs:.1f} s"}


def run_reference(args, w):
    world, rank, _ = dist_env()
    if rank != 0:
        return
    inp = cpu_inputs_f64(w)
    planes = [(b, c) for b in range(w.B) for c in range(w.Cc)]
    per_plane = w.algorithmic_bytes() / len(planes)
    n = args.ref_planes
    k = 0

    def step():
        nonlocal k
        sel = [planes[(k * n + i) % len(planes)] for i in range(n)]
        k += 1
        return oracle_planes_seconds(inp, sel)

    for _ in range(args.warmup):
        step()
    secs = sum(step() for _ in range(args.steps))
    value = per_plane * n * args.steps / secs / 1e9
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "GB/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": secs / args.steps * 1e3, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": config_of(w, world),
        "cpu_baseline": {"value": value, "unit": "GB/s", "cores": 1, "kind": "oracle",
                         "sample": f"{n} planes of the {w.name} workload per step"},
        "e2e": {"value": value, "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
        "gpu_launches": 0,
    }
    print(json.dumps(line), flush=True)


# ----------------------------------------------------------------------------
# GPU arm
# ----------------------------------------------------------------------------

METRIC = "Prop2D fwd GB/s (algorithmic HBM bytes / time); % of B200 HBM peak; ms/call"


def config_of(w, world):
    inbytes = w.algorithmic_bytes()
    return {"workload": f"{w.name}: B={w.B} Cc={w.Cc} H={w.H} W={w.W} {w.dtype} inputs, fp32 state, "
                        f"dirs={w.dirs}, share_w={w.share_w}",
            "B": w.B, "Cc": w.Cc, "H": w.H, "W": w.W, "dirs": w.dirs, "share_w": w.share_w,
            "algorithmic_bytes_per_step_per_gpu": inbytes,
            "l2": ("inputs larger than L2, no flush" if inbytes > L2_BYTES
                   else "L2 flushed (256 MiB write) between timed steps"),
            "parallelism": f"replicas x{world} (independent planes, no collective)"}


def run_ours(args, w):
    world, rank, local = dist_env()
    if world > 1:
        import torch.distributed as dist
        from datetime import timedelta
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=timedelta(seconds=120))
    dev = torch.device("cuda", local if world > 1 else 0)
    torch.cuda.set_device(dev)
    from spatial_propagation_vision_b200 import prop2d

    inp_cpu = workload_inputs(w, seed=rank)
    d = {k: v.to(dev) for k, v in inp_cpu.items()}
    out = torch.empty_like(d["x"])
    stream = torch.cuda.Stream(dev)
    nbytes = w.algorithmic_bytes()
    flush = None
    if nbytes <= L2_BYTES:
        flush = torch.empty(256 * 1024 * 1024 // 4, dtype=torch.float32, device=dev)

    # the compact mode normalises its shared weights once per call into a
    # workspace allocated here, outside the timed region
    kw = {}
    if w.share_w:
        B, Cc, H, W = d["x"].shape
        nws = prop2d.workspace_bytes(B, Cc, H, W, w.dirs, w.share_w, d["x"].dtype)
        kw["workspace"] = torch.empty(nws, dtype=torch.uint8, device=dev)

    def call():
        prop2d.prop2d_fwd(d["x"], d["lam"], d["wlogit"], d["u"], dirs=w.dirs,
                          share_w=w.share_w, out=out, stream=stream, **kw)

    with torch.cuda.stream(stream):
        for _ in range(args.warmup):
            if flush is not None:
                flush.fill_(1.0)
            call()
    torch.cuda.synchronize(dev)
    info = prop2d.launch_info()

    sampler = ClockSampler(dev.index)
    sampler.start()
    # load window: the same call for about 1 s (untimed), sampled for clocks
    # in case the timed region below is shorter than the polling interval
    torch.cuda.synchronize(dev)
    sampler.mark("l0")
    t_load = time.time()
    with torch.cuda.stream(stream):
        while time.time() - t_load < 1.0:
            for _ in range(20):
                if flush is not None:
                    flush.fill_(1.0)
                call()
            torch.cuda.synchronize(dev)
    sampler.mark("l1")
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(args.steps)]
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
    torch.cuda.synchronize(dev)
    sampler.mark("t0")
    start = torch.cuda.Event(enable_timing=True)
    end = torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        start.record(stream)
        for i in range(args.steps):
            if flush is not None:
                flush.fill_(1.0)
            ev[i][0].record(stream)
            call()
            ev[i][1].record(stream)
        end.record(stream)
    torch.cuda.synchronize(dev)
    sampler.mark("t1")
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
    sampler.stop()
    kernel_ms = [a.elapsed_time(b) for a, b in ev]
    region_ms = start.elapsed_time(end)
    if flush is not None:
        # the flush writes are not Prop2D work: time only the calls
        step_ms = sum(kernel_ms) / args.steps
    else:
        step_ms = region_ms / args.steps
    step_ms = max_over_ranks(step_ms, world, dev)
    avg_kernel_ms = max_over_ranks(statistics.mean(kernel_ms), world, dev)

    # end to end: host buffers -> device -> Prop2D -> host, through the C ABI
    e2e_steps = max(1, min(args.steps, args.e2e_steps))
    h = {k: v.pin_memory() for k, v in inp_cpu.items()}
    h["out"] = torch.empty_like(inp_cpu["x"]).pin_memory()
    dd = {k: torch.empty_like(v, device=dev) for k, v in h.items()}
    prop2d.prop2d_fwd_host(h, dd, dirs=w.dirs, share_w=w.share_w, stream=stream)
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
    torch.cuda.synchronize(dev)
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(e2e_steps):
        prop2d.prop2d_fwd_host(h, dd, dirs=w.dirs, share_w=w.share_w, stream=stream)
    e1.record(stream)
    torch.cuda.synchronize(dev)
    e2e_ms = max_over_ranks(e0.elapsed_time(e1) / e2e_steps, world, dev)
    h2d = sum(v.numel() * v.element_size() for k, v in inp_cpu.items())
    d2h = h["out"].numel() * h["out"].element_size()

    if world > 1:
        import torch.distributed as dist
        dist.barrier()
        dist.destroy_process_group()
    if rank != 0:
        return

    peak, peak_kind = peaks()
    achieved = nbytes / (avg_kernel_ms * 1e-3) / 1e9
    kernel = KERNEL_OF_PATH.get(info["path"], info["path"])
    traffic = args.traffic if args.traffic is not None else profiled_traffic(kernel, w.name, info)
    value = job_value(nbytes, world, step_ms * 1e-3)
    line = {
        "metric": METRIC, "value": value, "unit": "GB/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": step_ms,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "bf16" if w.dtype == "bf16" else "f32", "data": "synthetic (seeded)",
        "config": config_of(w, world),
        "hbm_frac_of_measured_peak": value / world / peak,
        "hbm_frac_of_nominal_peak": value / world / NOMINAL_HBM_GBS,
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                     "frac": achieved / peak,
                     "traffic": traffic,
                     "traffic_source": "ncu dram__bytes_read.sum + dram__bytes_write.sum per launch "
                                       f"({os.path.relpath(profile_path(kernel, w.name), ROOT)}, "
                                       "same kernel sources) or null",
                     "peak_source": f"{peak_kind} (MEASURED_PEAKS.json hbm_gbs)"
                     if peak_kind == "measured" else "fallback 6.65 TB/s",
                     "kernel": kernel, "avg_launch_ms": avg_kernel_ms},
        "e2e": {"value": job_value(nbytes, world, e2e_ms * 1e-3), "unit": "GB/s",
                "ms_per_step": e2e_ms, "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                "api": "gspn_prop2d_fwd_host (pinned host buffers)"},
        "gpu_launches": args.steps * info["launches"],
        "launch": info,
        "clocks": sampler.summary(),
    }
    if args.cpu_baseline and world == 1:
        line["cpu_baseline"] = cpu_oracle_baseline(w, budget_s=args.cpu_budget)
    print(json.dumps(line), flush=True)


def backward_bytes(w) -> int:
    """Bytes the backward must move once: x, lambda, u, the logits and gy
    read (input dtype), the fp32 gradients of x, lambda, u and the logits
    written."""
    s = w.in_bytes
    nd = bin(w.dirs).count("1")
    E = w.elems
    logits = 3 * nd * w.B * (1 if w.share_w else w.Cc) * w.H * w.W
    return E * s * (2 + 2 * nd) + logits * s + 4 * (E * (1 + 2 * nd) + logits)


def run_backward(args, w):
    """`--pass bwd`: gspn_prop2d_bwd on the workload, one GPU (a separate
    line; the default line is the forward's)."""
    from spatial_propagation_vision_b200 import prop2d
    dev = torch.device("cuda:0")
    torch.cuda.set_device(dev)
    d = {k: v.to(dev) for k, v in workload_inputs(w, seed=0).items()}
    gy = torch.randn(tuple(d["x"].shape), generator=torch.Generator().manual_seed(1)).to(d["x"].dtype).to(dev)
    call = lambda: prop2d.prop2d_bwd(d["x"], d["lam"], d["wlogit"], d["u"], gy, dirs=w.dirs,
                                     share_w=w.share_w)
    for _ in range(args.warmup):
        call()
    torch.cuda.synchronize()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record()
    for _ in range(args.steps):
        call()
    b.record()
    torch.cuda.synchronize()
    ms = a.elapsed_time(b) / args.steps
    nb = backward_bytes(w)
    print(json.dumps({"metric": "Prop2D bwd GB/s (bytes moved once / time); ms/call", "pass": "bwd",
                      "value": nb / ms / 1e6, "unit": "GB/s", "n_gpus": 1, "steps": args.steps,
                      "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True,
                      "dtype": {2: "bf16", 4: "f32"}[w.in_bytes], "data": "synthetic (seeded)",
                      "config": {"workload": w.name, "bytes_per_step": nb},
                      "launch": prop2d.launch_info()}), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="1k", choices=sorted(WORKLOADS))
    ap.add_argument("--e2e-steps", type=int, default=10)
    ap.add_argument("--ref-planes", type=int, default=64, help="oracle planes per reference step")
    ap.add_argument("--no-cpu-baseline", dest="cpu_baseline", action="store_false")
    ap.add_argument("--cpu-budget", type=float, default=12.0)
    ap.add_argument("--cc", type=int, default=None,
                    help="override the workload's channel count (a smaller case of the same "
                         "kernel, for ncu captures that must stay within a few GB)")
    ap.add_argument("--pass", dest="pass_", choices=["fwd", "bwd"], default="fwd",
                    help="bwd: time gspn_prop2d_bwd on the workload instead (one GPU, own line)")
    ap.add_argument("--traffic", type=float, default=None,
                    help="ncu dram bytes per launch of the dominant kernel, if captured for "
                         "the current build")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    w = WORKLOADS[args.workload]
    if args.cc is not None:
        import dataclasses
        w = dataclasses.replace(w, Cc=args.cc, name=f"{w.name}-cc{args.cc}")
    if args.pass_ == "bwd":
        run_backward(args, w)
    elif args.impl == "reference":
        run_reference(args, w)
    else:
        run_ours(args, w)


if __name__ == "__main__":
    main()
