"""The bench's JSON line keeps its contract: the keys the driver reads, consistent units, and
the same metric / config on both arms.  The reference arm (the fp64 oracle on the host) runs
here on the CPU; the GPU arm is checked on the small n = 1024 workload."""

from __future__ import annotations

import json
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
BASE_KEYS = {"metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
             "higher_is_better", "scaling", "vs_baseline", "dtype", "data", "config", "e2e"}


def _run(*args, timeout=600):
    out = subprocess.run([sys.executable, "bench.py", *args], cwd=ROOT, capture_output=True,
                         text=True, timeout=timeout)
    assert out.returncode == 0, out.stderr[-2000:]
    lines = [l for l in out.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1, out.stdout[-2000:]
    return json.loads(lines[0])


def test_reference_arm_line():
    line = _run("--impl", "reference", "--steps", "1", "--warmup", "0")
    assert BASE_KEYS <= set(line)
    assert line["impl"] == "reference"
    assert line["unit"] == "tokens/s" and line["higher_is_better"] is True
    assert line["value"] > 0 and line["n_gpus"] == 1 and line["steps"] == 1
    cb = line["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] >= 1 and cb["value"] == line["value"]
    assert line["e2e"]["value"] == line["value"]
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["e2e"]["d2h_bytes_per_step"] == 0
    sys.path.insert(0, ROOT)
    import bench
    assert line["metric"] == bench.METRIC
    assert line["config"] == bench.default_config(1)


@pytest.mark.gpu
def test_gpu_arm_line_small_workload():
    line = _run("--workload", "csa_f32_n1024", "--steps", "5", "--warmup", "3", "--no-cpu-baseline")
    assert BASE_KEYS <= set(line)
    assert {"roofline", "gpu_launches", "clocks"} <= set(line)
    r = line["roofline"]
    assert r["bound"] == "hbm" and r["unit"] == "GB/s" and r["peak"] > 0
    assert abs(r["frac"] - r["achieved"] / r["peak"]) < 1e-9
    assert line["gpu_launches"] == 5
    e = line["e2e"]
    assert e["h2d_bytes_per_step"] > 0 and e["d2h_bytes_per_step"] > 0 and e["value"] > 0
    assert e["value"] < line["value"]  # host copies inside its timed region
    assert line["warmup"] >= 3


def test_algorithmic_bytes_match_the_window_definition():
    """The roofline's numerator counts every stream element the windows read exactly once:
    enumerate the windows of a small problem by brute force and compare, then check the
    default step's figures."""
    sys.path.insert(0, ROOT)
    import bench

    for batch, n, c in ((1, 4 * 37, 64), (3, 4 * 37 + 2, 128), (2, 128 * 5 + 9, 512)):
        ne, nh = n // 4, n // 128
        read = set()
        for b in range(batch):
            for i in range(ne):  # CSA: a-block of entry i in Z^a, C^a; b-block in Z^b, C^b
                for k in range(4):
                    read |= {("Za", b, 4 * i + k), ("Ca", b, 4 * i + k)}
                    if i > 0:
                        read |= {("Zb", b, 4 * (i - 1) + k), ("Cb", b, 4 * (i - 1) + k)}
        csa = len(read) * c * 2 + 2 * 4 * c * 4 + batch * ne * c * 2
        hread = {(s, b, r) for b in range(batch) for i in range(nh) for r in range(128 * i, 128 * i + 128)
                 for s in ("Z", "C")}
        hca = len(hread) * c * 2 + 128 * c * 4 + batch * nh * c * 2
        assert bench.algorithmic_bytes(batch, n, c) == (csa, hca)
    assert bench.algorithmic_bytes() == (4_563_410_944, 2_156_134_400)


def test_cpu_baseline_all_cores_small():
    # The all-cores oracle timing on two spawned processes with a tiny sample: it reports
    # the processes it used and a positive rate, or no figure on a one-core host.
    import bench

    if len(os.sched_getaffinity(0)) < 2:
        assert bench.cpu_baseline_all_cores(2e4, seconds=0.1, max_tokens=2048) is None
        return
    r = bench.cpu_baseline_all_cores(2e4, seconds=0.1, max_tokens=2048, max_workers=2)
    assert "error" not in r, r
    assert r["cores"] == 2 and r["kind"] == "oracle" and r["unit"] == "tokens/s"
    assert r["host_cores"] == len(os.sched_getaffinity(0))
    assert r["value"] > 0 and r["wall_s"] >= r["slowest_process_s"] > 0


def test_reference_arm_other_ranks_do_no_work():
    # Under torchrun rank 0 alone times the oracle and prints; the other ranks exit 0 silently.
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1")
    out = subprocess.run([sys.executable, "bench.py", "--impl", "reference", "--gpus", "2",
                          "--steps", "1", "--warmup", "0"], cwd=ROOT, capture_output=True,
                         text=True, timeout=300, env=env)
    assert out.returncode == 0, out.stderr[-2000:]
    assert out.stdout.strip() == ""


def test_workload_cpu_baselines():
    # The oracle beside the other configs: the whole small CSA workload, and sampled entries
    # of the fused HCA one (marked as sampled); workloads without one get none.
    import bench

    full = bench.cpu_baseline_workload("csa_f32_n1024")
    assert full["kind"] == "oracle" and full["cores"] == 1 and full["sampled"] is False
    assert full["value"] > 0 and abs(full["entries_per_s"] * 4 - full["value"]) < 1e-6 * full["value"]
    samp = bench.cpu_baseline_workload("fused_hca")
    assert samp["sampled"] is True and "sampled" in samp["sample"]
    assert abs(samp["entries_per_s"] * 128 - samp["value"]) < 1e-6 * samp["value"]
    assert bench.cpu_baseline_workload("decode_entries") is None


def test_cpu_baseline_survives_a_failed_all_cores_run(monkeypatch):
    # The one-core figure is reported even when the all-cores processes cannot be started.
    import bench

    def no_processes(*a, **k):
        raise OSError("cannot start processes")

    monkeypatch.setattr(bench, "cpu_baseline_all_cores", no_processes)
    monkeypatch.setattr(bench, "oracle_inputs", lambda tokens, seed=0: None)
    monkeypatch.setattr(bench, "oracle_time", lambda d: 0.5)
    r = bench.cpu_baseline(budget_s=0.01)
    assert r["value"] > 0 and r["cores"] == 1
    assert r["all_cores"]["error"].startswith("all-cores timing failed")


def test_profile_commands_name_existing_bench_options():
    # Every summary under profiles/ gives the command that produced it; the bench options it
    # names must still exist (argparse rejects an unknown choice before it reaches --help).
    import glob
    import re

    used = set()
    for f in glob.glob(os.path.join(ROOT, "profiles", "*")):
        used |= set(re.findall(r"--(profile-case|workload) ([a-z0-9_]+)", open(f).read()))
    assert ("profile-case", "hca") in used
    for opt, val in sorted(used):
        out = subprocess.run([sys.executable, "bench.py", f"--{opt}", val, "--help"], cwd=ROOT,
                             capture_output=True, text=True, timeout=120)
        assert out.returncode == 0, (opt, val, out.stderr[-500:])
