"""Host logic of bench.py without a GPU: whole-job arithmetic, the max over
ranks on two gloo ranks (the replicas path under torchrun), the reference
arm's JSON line and rank behaviour, and the profile-traffic lookup."""
import json
import os
import socket
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import bench  # noqa: E402
from spatial_propagation_vision_b200.workloads import WORKLOADS  # noqa: E402


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _max_worker(rank, world, port, out_dir):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        w, r, local = bench.dist_env()
        assert (w, r, local) == (world, rank, rank)
        # each rank's time; the job's time is the slowest rank's
        t = bench.max_over_ranks(1.5 + rank, world, torch.device("cpu"))
        with open(os.path.join(out_dir, f"rank{rank}.txt"), "w") as f:
            f.write(repr(t))
    finally:
        dist.destroy_process_group()


def test_max_over_two_gloo_ranks(tmp_path):
    world = 2
    mp.spawn(_max_worker, args=(world, _free_port(), str(tmp_path)), nprocs=world, join=True)
    vals = [float(open(tmp_path / f"rank{r}.txt").read()) for r in range(world)]
    assert vals == [2.5, 2.5]


def test_single_rank_max_is_identity():
    assert bench.max_over_ranks(0.25, 1, None) == 0.25


def test_job_value_is_whole_job():
    # two ranks of 493,453,312 B each in 0.5 ms: 1973.8 GB/s for the job
    v = bench.job_value(493_453_312, 2, 0.5e-3)
    assert abs(v - 2 * 493_453_312 / 0.5e-3 / 1e9) < 1e-9


def test_reference_arm_line(capsys, monkeypatch):
    args = bench.argparse.Namespace(steps=2, warmup=1, ref_planes=2)
    monkeypatch.setenv("WORLD_SIZE", "1")
    monkeypatch.setenv("RANK", "0")
    bench.run_reference(args, WORKLOADS["tiny"])
    line = json.loads(capsys.readouterr().out.strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["unit"] == "GB/s" and line["value"] > 0
    assert line["cpu_baseline"]["kind"] == "oracle" and line["cpu_baseline"]["value"] == line["value"]
    assert line["e2e"] == {"value": line["value"], "unit": "GB/s",
                           "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}
    assert line["steps"] == 2 and line["warmup"] == 1 and line["gpu_launches"] == 0


def test_reference_arm_other_ranks_are_silent(capsys, monkeypatch):
    args = bench.argparse.Namespace(steps=2, warmup=1, ref_planes=2)
    monkeypatch.setenv("WORLD_SIZE", "2")
    monkeypatch.setenv("RANK", "1")
    bench.run_reference(args, WORKLOADS["tiny"])
    assert capsys.readouterr().out == ""


@pytest.mark.parametrize("matches", [True, False])
def test_profile_traffic_needs_current_sources(tmp_path, monkeypatch, matches):
    os.makedirs(tmp_path / "profiles")
    sha = bench.kernel_sources_sha("prop2d_pair_kernel") if matches else "0" * 64
    (tmp_path / "profiles" / "prop2d_pair_1k.md").write_text(
        f"kernel_sources_sha256: {sha}\ntraffic_bytes_per_launch: 12345\n"
        "launch_geometry: grid=444 block=128 smem=53552\n")
    real_sha = {k: bench.kernel_sources_sha(k) for k in bench.KERNEL_UNITS}
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    monkeypatch.setattr(bench, "kernel_sources_sha", lambda kernel="prop2d_dir_kernel": real_sha[kernel])
    assert bench.profiled_traffic("prop2d_pair_kernel", "1k") == (12345 if matches else None)
    assert bench.profiled_traffic("prop2d_dir_kernel", "1k") is None
    same = {"grid": 444, "block": 128, "smem": 53552}
    other = dict(same, grid=592)
    assert bench.profiled_traffic("prop2d_pair_kernel", "1k", same) == (12345 if matches else None)
    assert bench.profiled_traffic("prop2d_pair_kernel", "1k", other) is None


def test_clock_summary_is_honest_about_short_windows():
    """A timed region with no clock sample reports the load window, labelled."""
    cs = bench.ClockSampler(0)
    cs.proc = object()
    row = "0, 1965, 1965, 700.0, 0x0, Not Active, Not Active, Not Active, Not Active"
    cs.samples = [(10.0, row), (10.5, row), (11.2, row)]
    cs.l0, cs.l1, cs.t0, cs.t1 = 9.9, 11.0, 11.05, 11.06
    out = cs.summary()
    assert out["timed_region_samples"] == 0 and out["samples"] == 2
    assert out["source"].startswith("no sample in the timed region")
    cs.t1 = 11.3
    out = cs.summary()
    assert out["source"] == "timed region" and out["samples"] == 1 and out["sm_mhz"] == 1965.0


def test_kernel_hash_ignores_host_only_files():
    """A kernel's source hash covers its own headers and units, not the C ABI
    or another kernel's sources."""
    import glob
    csrc = os.path.join(bench.ROOT, "spatial_propagation_vision_b200", "csrc")
    names = {os.path.basename(f) for f in glob.glob(os.path.join(csrc, "*"))}
    assert "gspn_api.cu" in names and "launch.h" in names and "bwd_launch.cu" in names
    shas = {k: bench.kernel_sources_sha(k) for k in bench.KERNEL_UNITS}
    assert len(set(shas.values())) == len(shas)     # every kernel has its own units
