"""Throughput of the B200 token-level KV compressor (one JSON line on rank 0).

Default workload: the long-context streams, batch 1, n = 2^20 tokens, c = 512, bf16
C^a, C^b, Z^a, Z^b ~ N(0, 1) with per-row logit offsets U(-4, 4); one step runs the CSA
compressor (m = 4, overlap) and the HCA compressor (m' = 128, C := C^a, Z := Z^a) over
the same streams, i.e. both softmax-pool kernels of the hot path.  Inputs (4.3 GB) are
far larger than L2 (126 MB), so no flush is needed between steps.

Usage: python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
For N > 1 launch under torchrun: every rank runs the same per-GPU workload on its own
seeded inputs (weak scaling, no data-path collective); times are max over ranks.

--impl reference times the fp64 CPU oracle (the only reference implementation this
project has) on a bounded sample of the same workload on the host cores.
"""

from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "input tokens/s and compressed entries/s at c=512; HBM GB/s % of peak"
N_TOK = 1 << 20
C = 512
M_CSA = 4
M_HCA = 128
Z_OFF = 4.0
FALLBACK_HBM_GBS = 6650.0


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    return FALLBACK_HBM_GBS, "fallback"


def algorithmic_bytes(batch=1, n=N_TOK, c=C):
    """Compulsory bytes per launch: every stream element the window definition reads,
    the biases, and the output (bf16 in, bf16 out)."""
    ne = n // M_CSA
    csa = (2 * batch * ne * M_CSA * c * 2            # Z^a, C^a: a-ranges of all entries
           + 2 * batch * max(ne - 1, 0) * M_CSA * c * 2  # Z^b, C^b: b-ranges of entries 1..
           + 2 * M_CSA * c * 4                          # B^a, B^b
           + batch * ne * c * 2)                        # output
    nh = n // M_HCA
    hca = (2 * batch * nh * M_HCA * c * 2 + M_HCA * c * 4 + batch * nh * c * 2)
    return csa, hca


def _traffic(key):
    """DRAM bytes per launch of a kernel from the committed ncu summaries (None if absent)."""
    prof = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(prof):
        return None
    with open(prof) as f:
        return json.load(f).get(key)


class ClockSampler:
    """nvidia-smi sampled every 100 ms while the timed region runs."""

    Q = ("timestamp,index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_id):
        self.proc = None
        self.gpu = gpu_id  # nvidia-smi -i accepts the UUID (it ignores CUDA_VISIBLE_DEVICES)
        self.t0 = self.t1 = None

    def mark(self, start: bool):
        if start:
            self.t0 = time.time()
        else:
            self.t1 = time.time()

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.Q}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
        time.sleep(0.6)

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        time.sleep(0.15)
        self.proc.terminate()
        out, _ = self.proc.communicate(timeout=10)
        import datetime

        rows = []
        for r in out.strip().splitlines():
            f = [x.strip() for x in r.split(",")]
            if len(f) < 10:
                continue
            try:
                ts = datetime.datetime.strptime(f[0], "%Y/%m/%d %H:%M:%S.%f").timestamp()
            except ValueError:
                continue
            if self.t0 is not None and not (self.t0 <= ts <= self.t1 + 0.05):
                continue  # keep only samples taken inside the timed region
            rows.append(f)
        sm = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        mx = [float(r[3]) for r in rows if r[3].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[k] for r in rows for k in range(4) if r[6 + k].strip() == "Active"})
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(mx) if mx else None, "reasons": reasons, "samples": len(rows)}


class NvmlClockSampler:
    """Clocks and clock-event reasons read through NVML by a host thread every ~2 ms, so
    that even a timed region of a few tens of milliseconds holds several samples.  Reads
    only; nothing is set.  `stop()` returns the same fields as :class:`ClockSampler`."""

    REASONS = (("hw_slowdown", "nvmlClocksEventReasonHwSlowdown", 0x8),
               ("hw_thermal_slowdown", "nvmlClocksEventReasonHwThermalSlowdown", 0x40),
               ("sw_thermal_slowdown", "nvmlClocksEventReasonSwThermalSlowdown", 0x20),
               ("sw_power_cap", "nvmlClocksEventReasonSwPowerCap", 0x4))

    def __init__(self, uuid, period_s=0.002):
        import threading

        import pynvml

        self.nv = pynvml
        pynvml.nvmlInit()
        self.h = pynvml.nvmlDeviceGetHandleByUUID(uuid.encode() if isinstance(uuid, str) else uuid)
        self.max_mhz = float(pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM))
        self.period = period_s
        self.samples = []
        self.t0 = self.t1 = None
        self.halt = threading.Event()
        self.thread = threading.Thread(target=self._run, daemon=True)

    def _reasons(self):
        nv = self.nv
        get = getattr(nv, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
            nv.nvmlDeviceGetCurrentClocksThrottleReasons
        return int(get(self.h))

    def _run(self):
        nv = self.nv
        while not self.halt.is_set():
            try:
                mhz = float(nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM))
                self.samples.append((time.time(), mhz, self._reasons()))
            except Exception:
                pass
            time.sleep(self.period)

    def mark(self, start: bool):
        if start:
            self.t0 = time.time()
        else:
            self.t1 = time.time()

    def start(self):
        self.thread.start()
        time.sleep(0.05)

    def stop(self):
        self.halt.set()
        self.thread.join(timeout=5)
        try:
            self.nv.nvmlShutdown()
        except Exception:
            pass
        rows = [s for s in self.samples
                if self.t0 is None or (self.t0 <= s[0] <= (self.t1 or s[0]) + 0.002)]
        bits = {name: getattr(self.nv, attr, val) for name, attr, val in self.REASONS}
        reasons = sorted({name for _, _, r in rows for name, b in bits.items() if r & b})
        sm = [r[1] for r in rows]
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": self.max_mhz,
                "reasons": reasons, "samples": len(rows), "source": "nvml, ~2 ms period"}


def clock_sampler(uuid):
    """The NVML sampler when NVML answers, else nvidia-smi every 100 ms."""
    try:
        return NvmlClockSampler(uuid)
    except Exception:
        return ClockSampler(uuid)


def dist_setup(n_gpus):
    import torch

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world != n_gpus:
        raise SystemExit(f"--gpus {n_gpus} but WORLD_SIZE={world}")
    if world > 1:
        import datetime

        import torch.distributed as dist

        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    else:
        torch.cuda.set_device(0)
    return rank, world, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist

        dist.barrier()


def max_over_ranks(x, world):
    if world == 1:
        return x
    import torch
    import torch.distributed as dist

    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


# ------------------------------------------------------------------------------ oracle

def oracle_inputs(tokens: int, seed=0):
    """Host copy of the first `tokens` tokens of the workload (seeded, bf16 values)."""
    from kv_token_compressor_b200 import synth

    d = synth.stream_inputs("csa", 1, tokens, C, M_CSA, "bf16", seed=seed, z_row_offset=Z_OFF)
    rng = np.random.default_rng(seed + 1)
    d["Bh"] = (rng.standard_normal((M_HCA, C), dtype=np.float32) * np.float32(np.sqrt(0.1)))
    return d


def oracle_time(d):
    """Seconds the fp64 oracle (as it stands) takes for CSA m=4 overlap then HCA m'=128
    on the same streams."""
    from oracle import compressor as O

    t0 = time.perf_counter()
    O.csa_compress(d["Ca"], d["Cb"], d["Za"], d["Zb"], d["Ba"], d["Bb"], M_CSA, True)
    O.hca_compress(d["Ca"], d["Za"], d["Bh"], M_HCA)
    return time.perf_counter() - t0


def cpu_baseline(budget_s=12.0, all_cores=True):
    probe = 4096
    rate = probe / oracle_time(oracle_inputs(probe))
    tokens = int(max(probe, min(1 << 18, rate * budget_s)) // M_HCA * M_HCA)
    dt = oracle_time(oracle_inputs(tokens))
    out = {"value": tokens / dt, "unit": "tokens/s", "cores": 1, "kind": "oracle",
           "sample": f"first {tokens} of the {N_TOK} tokens (CSA m=4 + HCA m'=128, fp64 numpy, "
                     f"single-threaded elementwise), {dt:.1f} s"}
    if all_cores:
        try:
            out["all_cores"] = cpu_baseline_all_cores(tokens / dt)
        except Exception as e:  # the one-core figure stands without it
            out["all_cores"] = {"error": f"all-cores timing failed: {e!r}"}
    return out


def cpu_baseline_workload(name):
    """The oracle, as it stands, on one host core for a named workload: the whole workload
    for the two small streaming ones; for the fused ones, sampled entries (first, last and
    evenly spaced) of a 4096-token H with the workload's d and c, since the work per entry
    does not depend on n (the oracle projects only the rows an entry reads).  BLAS is held
    to one thread.  None for the other workloads."""
    from threadpoolctl import threadpool_limits

    from kv_token_compressor_b200 import synth
    from oracle import compressor as O

    def timed(f):
        with threadpool_limits(limits=1):
            t0 = time.perf_counter()
            f()
            return time.perf_counter() - t0

    if name in ("csa_f32_n1024", "hca_n65536", "hca_n65536_prepared"):
        mode, n, m, dt = (("csa", 1024, M_CSA, "f32") if name == "csa_f32_n1024"
                          else ("hca", 65536, M_HCA, "bf16"))
        d = synth.stream_inputs(mode, 1, n, C, m, dt, seed=0)
        if mode == "csa":
            s = timed(lambda: O.csa_compress(d["Ca"], d["Cb"], d["Za"], d["Zb"], d["Ba"], d["Bb"],
                                             m, True))
        else:
            s = timed(lambda: O.hca_compress(d["C"], d["Z"], d["B"], m))
        return {"value": n / s, "unit": "tokens/s", "entries_per_s": (n // m) / s, "cores": 1,
                "kind": "oracle", "sampled": False,
                "sample": f"the whole workload ({n} tokens; fp64 numpy, one thread), {s:.2f} s"}
    if name in ("fused_csa", "fused_hca"):
        csa = name == "fused_csa"
        m, dm, n, k = (M_CSA, 7168, 4096, 48) if csa else (M_HCA, 4096, 4096, 8)
        f = synth.fused_inputs("csa" if csa else "hca", 1, n, dm, C, m, seed=0)
        ne = n // m
        ents = sorted({(0, int(i)) for i in np.linspace(0, ne - 1, k).round()})
        if csa:
            s = timed(lambda: O.csa_compress_fused(f["H"], f["W_kva"], f["W_kvb"], f["W_za"],
                                                   f["W_zb"], f["Ba"], f["Bb"], 1, n, m, True,
                                                   entries=ents))
        else:
            s = timed(lambda: O.hca_compress_fused(f["H"], f["W_kv"], f["W_z"], f["B"], 1, n, m,
                                                   entries=ents))
        eps = len(ents) / s
        return {"value": eps * m, "unit": "tokens/s", "entries_per_s": eps, "cores": 1,
                "kind": "oracle", "sampled": True,
                "sample": f"sampled: {len(ents)} entries of a {n}-token H, d={dm}, c={C}, m={m} "
                          f"(fp64, one thread), {s:.2f} s; value = entries/s x m"}
    return None


def _oracle_worker(seed, tokens, reps, barrier, results):
    """One process of the all-cores oracle timing: its own seeded piece of the workload,
    generated before the common start; then `reps` passes of the oracle as it stands."""
    try:
        d = oracle_inputs(tokens, seed=seed)
        import oracle.compressor  # noqa: F401  (the import stays out of the timed region)

        barrier.wait()
        t0 = time.perf_counter()
        for _ in range(reps):
            oracle_time(d)
        results.put(time.perf_counter() - t0)
    except Exception as e:  # reported by the parent, which then gives no figure
        barrier.abort()
        results.put(repr(e))


def cpu_baseline_all_cores(rate1, seconds=4.0, max_tokens=1 << 19, max_workers=64):
    """The same oracle on every host core this process may use: one spawned process per
    core, each on its own seeded piece of the workload's shape (inputs are generated in the
    process, outside the timed region), released together by a barrier.  The figure is the
    tokens all processes handled over the parent's wall-clock time from the release to the
    last result.  `rate1` (tokens/s on one core) sizes each process to ~`seconds` of work;
    `max_tokens` bounds the tokens held at once by all processes together (8 KB each);
    at most `max_workers` processes."""
    import multiprocessing

    host_cores = cores = len(os.sched_getaffinity(0))
    if max_workers:
        cores = min(cores, max_workers)
    if cores < 2:
        return None
    tokens = int(max(M_HCA, min(max_tokens // cores, rate1 * seconds)) // M_HCA * M_HCA)
    reps = max(1, round(rate1 * seconds / tokens))
    ctx = multiprocessing.get_context("spawn")  # never fork a process that holds a GPU context
    barrier, results = ctx.Barrier(cores + 1), ctx.Queue()
    pin = {k: "1" for k in ("OMP_NUM_THREADS", "OPENBLAS_NUM_THREADS", "MKL_NUM_THREADS")}
    saved = {k: os.environ.get(k) for k in pin}
    os.environ.update(pin)  # one thread per process: the processes are the parallelism
    procs = []
    try:
        for w in range(cores):
            p = ctx.Process(target=_oracle_worker, args=(1000 + 2 * w, tokens, reps, barrier,
                                                         results), daemon=True)
            p.start()
            procs.append(p)
    except Exception:
        barrier.abort()  # the processes already started leave their wait
        for p in procs:
            p.terminate()
        raise
    finally:
        for k, v in saved.items():
            if v is None:
                os.environ.pop(k, None)
            else:
                os.environ[k] = v
    try:
        barrier.wait(timeout=300)
        t0 = time.perf_counter()
        got = [results.get(timeout=300) for _ in procs]
        wall = time.perf_counter() - t0
    except Exception as e:
        why = []
        try:  # a worker that raised has queued its exception
            while len(why) < len(procs):
                g = results.get(timeout=5)
                if isinstance(g, str):
                    why.append(g)
        except Exception:
            pass
        for p in procs:
            p.terminate()
        return {"error": f"all-cores timing failed: {e!r}" + (f" ({why[0]})" if why else "")}
    finally:
        for p in procs:
            p.join(timeout=60)
    if any(isinstance(g, str) for g in got):
        return {"error": next(g for g in got if isinstance(g, str))}
    return {"value": cores * tokens * reps / wall, "unit": "tokens/s", "cores": cores,
            "host_cores": host_cores, "kind": "oracle", "wall_s": wall, "slowest_process_s": max(got),
            "sample": f"{cores} processes x {reps} passes over {tokens} tokens each (own seeded "
                      f"piece of the workload's shape; CSA m=4 + HCA m'=128, fp64 numpy, one "
                      f"thread per process)"}


def default_config(world: int) -> dict:
    """The default step's workload description, shared by both arms."""
    return {"workload": "long-context streams: batch 1, n=2^20, c=512, bf16 in/out; "
                        "CSA m=4 overlap + HCA m'=128 on the same streams",
            "batch": 1, "n": N_TOK, "c": C, "m": M_CSA, "m_hca": M_HCA,
            "l2": "inputs 4.3 GB > 126 MB L2, no flush",
            "parallelism": f"weak: {world} independent replicas"}


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    steps, warm = args.steps, args.warmup
    probe = 2048
    probe_rate = probe / oracle_time(oracle_inputs(probe))
    per_step = 120.0 / max(steps + warm, 1)  # seconds: the whole run within a few minutes
    tokens = int(max(M_HCA, min(1 << 16, probe_rate * per_step)) // M_HCA * M_HCA)
    d = oracle_inputs(tokens)
    for _ in range(warm):
        oracle_time(d)
    times = [oracle_time(d) for _ in range(steps)]
    t = sum(times)
    value = steps * tokens / t
    ne = tokens // M_CSA + tokens // M_HCA
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s",
        "entries_per_s": steps * ne / t, "n_gpus": args.gpus, "steps": steps, "warmup": warm,
        "ms_per_step": 1e3 * t / steps, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": default_config(args.gpus),
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": 1, "kind": "oracle",
                         "sample": f"first {tokens} of the {N_TOK} tokens per step (CSA m=4 + "
                                   f"HCA m'=128, fp64 numpy, single-threaded elementwise)"},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


# ------------------------------------------------------------------------------ ours

def run_ours(args):
    import torch

    from kv_token_compressor_b200 import kvc, synth

    rank, world, local = dist_setup(args.gpus)
    dev = torch.device("cuda", local if world > 1 else 0)
    t = synth.stream_inputs_torch("csa", 1, N_TOK, C, M_CSA, "bf16", seed=rank,
                                  z_row_offset=Z_OFF, device=dev)
    g = torch.Generator(device=dev)
    g.manual_seed(1000 + rank)
    Bh = torch.randn((M_HCA, C), generator=g, device=dev) * float(np.sqrt(0.1))
    out_c = torch.empty((1, N_TOK // M_CSA, C), device=dev, dtype=torch.bfloat16)
    out_h = torch.empty((1, N_TOK // M_HCA, C), device=dev, dtype=torch.bfloat16)
    stream = torch.cuda.current_stream(dev)

    def step(ev=None):
        if ev is not None:
            ev[0].record(stream)
        kvc.csa_compress(t["Ca"], t["Cb"], t["Za"], t["Zb"], t["Ba"], t["Bb"], m=M_CSA,
                         out=out_c, out_dtype=torch.bfloat16, stream=stream)
        if ev is not None:
            ev[1].record(stream)
        kvc.hca_compress(t["Ca"], t["Za"], Bh, m=M_HCA, out=out_h, out_dtype=torch.bfloat16,
                         stream=stream)
        if ev is not None:
            ev[2].record(stream)

    for _ in range(max(args.warmup, 3)):
        step()
    torch.cuda.synchronize()
    if kvc.device_status(stream) != kvc.KVC_OK:
        raise SystemExit("device error during warm-up")

    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(args.steps)]
    props = torch.cuda.get_device_properties(dev)
    uuid = str(getattr(props, "uuid", ""))
    sampler = clock_sampler(("GPU-" + uuid) if uuid and not uuid.startswith("GPU-") else (uuid or "0"))
    sampler.start()
    barrier(world)
    torch.cuda.synchronize()
    sampler.mark(True)
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    t0.record(stream)
    for k in range(args.steps):
        step(evs[k])
    t1.record(stream)
    torch.cuda.synchronize()
    sampler.mark(False)
    barrier(world)
    clocks = sampler.stop()
    elapsed_ms = max_over_ranks(t0.elapsed_time(t1), world)
    csa_ms = statistics.mean(e[0].elapsed_time(e[1]) for e in evs)
    hca_ms = statistics.mean(e[1].elapsed_time(e[2]) for e in evs)
    csa_ms = max_over_ranks(csa_ms, world)
    hca_ms = max_over_ranks(hca_ms, world)

    # e2e through the public API with host buffers: H2D of the step's inputs from pinned
    # memory, both compressors, D2H of both outputs, all inside the timed region.
    host = {k: t[k].cpu().pin_memory() for k in ("Ca", "Cb", "Za", "Zb", "Ba", "Bb")}
    host["Bh"] = Bh.cpu().pin_memory()
    h_out_c = torch.empty(out_c.shape, dtype=out_c.dtype).pin_memory()
    h_out_h = torch.empty(out_h.shape, dtype=out_h.dtype).pin_memory()
    h2d = sum(v.numel() * v.element_size() for v in host.values())
    d2h = h_out_c.numel() * 2 + h_out_h.numel() * 2

    def e2e_step():
        dv = {k: v.to(dev, non_blocking=True) for k, v in host.items()}
        kvc.csa_compress(dv["Ca"], dv["Cb"], dv["Za"], dv["Zb"], dv["Ba"], dv["Bb"], m=M_CSA,
                         out=out_c, out_dtype=torch.bfloat16, stream=stream)
        kvc.hca_compress(dv["Ca"], dv["Za"], dv["Bh"], m=M_HCA, out=out_h,
                         out_dtype=torch.bfloat16, stream=stream)
        h_out_c.copy_(out_c, non_blocking=True)
        h_out_h.copy_(out_h, non_blocking=True)
        del dv

    del t
    torch.cuda.empty_cache()
    e2e_steps = max(3, min(args.steps, 10))
    e2e_step()
    torch.cuda.synchronize()
    barrier(world)
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(e2e_steps):
        e2e_step()
    e1.record(stream)
    torch.cuda.synchronize()
    barrier(world)
    e2e_ms = max_over_ranks(e0.elapsed_time(e1), world) / e2e_steps

    fused = None
    if world == 1 and not args.no_fused:
        del host, h_out_c, h_out_h
        fused = time_fused(dev, stream)

    peak, peak_kind = peaks()
    csa_bytes, hca_bytes = algorithmic_bytes()
    csa_gbs = csa_bytes / (csa_ms * 1e-3) / 1e9
    hca_gbs = hca_bytes / (hca_ms * 1e-3) / 1e9
    ms_step = elapsed_ms / args.steps
    tokens_per_s = world * N_TOK / (ms_step * 1e-3)
    entries = N_TOK // M_CSA + N_TOK // M_HCA
    traffic = _traffic("csa_compress_bf16_n1048576")
    if rank == 0:
        line = {
            "metric": METRIC, "value": tokens_per_s, "unit": "tokens/s",
            "entries_per_s": world * entries / (ms_step * 1e-3),
            "n_gpus": world, "steps": args.steps, "warmup": max(args.warmup, 3),
            "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f32", "data": "synthetic",
            "config": default_config(world),
            "roofline": {"bound": "hbm", "kernel": "csa_compress (csa_small_m_kernel<bf16,bf16,4>)",
                         "achieved": csa_gbs, "peak": peak, "unit": "GB/s",
                         "frac": csa_gbs / peak, "peak_kind": peak_kind, "traffic": traffic,
                         "algorithmic_bytes": csa_bytes},
            "kernels": {
                "csa_compress": {"ms": csa_ms, "GB/s": csa_gbs, "frac": csa_gbs / peak,
                                 "tokens_per_s": N_TOK / (csa_ms * 1e-3),
                                 "entries_per_s": (N_TOK // M_CSA) / (csa_ms * 1e-3)},
                "hca_compress": {"ms": hca_ms, "GB/s": hca_gbs, "frac": hca_gbs / peak,
                                 "traffic": _traffic("hca_compress_bf16_n1048576"),
                                 "tokens_per_s": N_TOK / (hca_ms * 1e-3),
                                 "entries_per_s": (N_TOK // M_HCA) / (hca_ms * 1e-3)},
            },
            "gpu_launches": 2 * args.steps,
            "clocks": clocks,
            "e2e": {"value": world * N_TOK / (e2e_ms * 1e-3), "unit": "tokens/s",
                    "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms},
        }
        if fused:
            line["kernels"].update(fused)
        if world == 1 and not args.no_cpu_baseline:
            line["cpu_baseline"] = cpu_baseline()
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist

        dist.destroy_process_group()


def time_fused(dev, stream, reps=20):
    """The fused projection + pool kernels on their own workloads (CSA: H [32768, 7168],
    c = 512; HCA: 4 x 131072 tokens, d = 4096, c = 512), timed after the default step's
    timed region and reported beside it: CUDA events around each of `reps` back-to-back
    launches on the launching stream after 3 warm-up launches; clocks sampled meanwhile.
    FLOPs = 2 * tokens * d * (streams * c); fractions of the measured burst and sustained
    bf16 GEMM rates."""
    import torch

    from kv_token_compressor_b200 import kvc

    burst, kind = _peak("tensor")
    sust, _ = _peak("tensor", sustained=True)
    props = torch.cuda.get_device_properties(dev)
    uuid = str(getattr(props, "uuid", ""))
    res = {}
    for name in ("fused_csa", "fused_hca"):
        w = _workload(name, dev)
        for _ in range(3):
            w["launch"](w["inputs"], stream)
        torch.cuda.synchronize()
        kernel = kvc.last_kernel()
        evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
               for _ in range(reps)]
        sampler = clock_sampler(("GPU-" + uuid) if uuid and not uuid.startswith("GPU-")
                                else (uuid or "0"))
        sampler.start()
        sampler.mark(True)
        for a, b in evs:
            a.record(stream)
            w["launch"](w["inputs"], stream)
            b.record(stream)
        torch.cuda.synchronize()
        sampler.mark(False)
        clocks = sampler.stop()
        if kvc.device_status(stream) != kvc.KVC_OK:
            raise SystemExit(f"device error in {name}")
        ms = statistics.mean(a.elapsed_time(b) for a, b in evs)
        tf = w["units"] / (ms * 1e-3) / 1e12
        res[name] = {"kernel": kernel, "workload": w["config"]["workload"], "ms": ms,
                     "flops": w["units"], "TFLOP/s": tf, "frac": tf / burst,
                     "frac_sustained": tf / sust, "peak": burst, "peak_sustained": sust,
                     "peak_kind": kind, "unit": "TFLOP/s",
                     "traffic": _traffic(w["traffic_key"]) if w.get("traffic_key") else None,
                     "tokens_per_s": w["tokens"] / (ms * 1e-3),
                     "entries_per_s": w["entries"] / (ms * 1e-3), "launches": reps,
                     "clocks": clocks}
        del w
        torch.cuda.empty_cache()
    return res


# ------------------------------------------------------------------------------ split sequence
# --split sequence: ONE sequence of world x 2^20 tokens, each rank holding only the token
# rows its entries read (kv_token_compressor_b200.shard.plan: contiguous entry ranges, a
# one-block halo for the CSA b-rows; HCA windows need none).  Rows are drawn per 65536-row
# piece from (seed, piece), so every rank, and the checker, draw the same sequence.

SPLIT_SEED = 11


def split_plan(n_total, world, rank):
    """Rows [lo, hi) this rank holds, and its CSA and HCA shards."""
    from kv_token_compressor_b200 import shard

    pc = shard.plan(n_total, M_CSA, world, True)[rank]
    ph = shard.plan(n_total, M_HCA, world, False)[rank]
    return min(pc.row0, ph.row0), max(pc.row1, ph.row1), pc, ph


def split_inputs(n_total, world, rank, c, dtype, device):
    from kv_token_compressor_b200 import synth

    lo, hi, pc, ph = split_plan(n_total, world, rank)
    t = synth.stream_rows_torch(lo, hi, c, dtype, seed=SPLIT_SEED, z_row_offset=Z_OFF, device=device)
    t["Ba"] = synth.bias_torch(M_CSA, c, SPLIT_SEED + 1, device=device)
    t["Bb"] = synth.bias_torch(M_CSA, c, SPLIT_SEED + 2, device=device)
    t["Bh"] = synth.bias_torch(M_HCA, c, SPLIT_SEED + 3, device=device)
    return t, lo, pc, ph


def split_compress(t, lo, pc, ph, csa_fn, hca_fn, out_c, out_h):
    """The rank's part: CSA over its rows (halo first) into out_c [1, entries + halo, c],
    HCA into out_h [1, entries, c].  Returns the owned entries (the halo entry dropped)."""
    sl = {k: t[k][:, pc.row0 - lo:pc.row1 - lo] for k in ("Ca", "Cb", "Za", "Zb")}
    if pc.entries:
        csa_fn(sl, t["Ba"], t["Bb"], out_c)
    if ph.entries:
        hca_fn(t["Ca"][:, ph.row0 - lo:ph.row1 - lo], t["Za"][:, ph.row0 - lo:ph.row1 - lo],
               t["Bh"], out_h)
    return (out_c[:, 1:] if pc.drop_first else out_c), out_h


def split_check(world, rank, pc, ph, owned_c, owned_h, c, dtype, device, single_csa, single_hca,
                per_rank=16):
    """Sampled cross-rank check: every rank sends its first, second and last owned entries
    (the first one depends on the halo) and a few others of each compressor to rank 0 over
    the process group; rank 0 redraws the rows each entry reads and recomputes it on its
    own as a one-sequence problem (single_csa(rows, Ba, Bb, j) -> entry j of those rows,
    single_hca(C, Z, B) -> their one entry, numpy float64), then compares.  The tolerance
    allows one output rounding on each side.  Returns (entries checked, max error / max
    |ref|, ok) on rank 0, None elsewhere."""
    import torch
    import torch.distributed as dist

    from kv_token_compressor_b200 import synth

    def pick(e0, e1, k):
        n = e1 - e0
        if n <= 0:
            return []
        rng = np.random.default_rng(1000 + rank)
        idx = {e0, e1 - 1, min(e0 + 1, e1 - 1)} | set((e0 + rng.integers(0, n, k)).tolist())
        return sorted(idx)[:k + 3]

    rows = []
    for mode, shard, owned in (("csa", pc, owned_c), ("hca", ph, owned_h)):
        for e in pick(shard.e0, shard.e1, per_rank if mode == "csa" else 4):
            v = owned[0, e - shard.e0].float().cpu()
            rows.append(torch.cat([torch.tensor([0.0 if mode == "csa" else 1.0, float(e)]), v]))
    width, slots = 2 + c, per_rank + 3 + 4 + 3
    mine = torch.full((slots, width), -1.0, dtype=torch.float32)
    for i, r in enumerate(rows):
        mine[i] = r
    if world > 1:
        dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
        got = [torch.empty_like(mine, device=dev) for _ in range(world)]
        dist.all_gather(got, mine.to(dev))
        got = [g.cpu() for g in got]
    else:
        got = [mine]
    if rank != 0:
        return None
    Ba = synth.bias_torch(M_CSA, c, SPLIT_SEED + 1, device=device)
    Bb = synth.bias_torch(M_CSA, c, SPLIT_SEED + 2, device=device)
    Bh = synth.bias_torch(M_HCA, c, SPLIT_SEED + 3, device=device)
    worst, checked, ok = 0.0, 0, True
    for g in got:
        for r in g:
            if r[1] < 0:
                continue
            mode, e = int(r[0]), int(r[1])
            if mode == 0:
                lo = M_CSA * (e - 1) if e > 0 else 0
                x = synth.stream_rows_torch(lo, M_CSA * (e + 1), c, dtype, seed=SPLIT_SEED,
                                            z_row_offset=Z_OFF, device=device)
                ref = single_csa(x, Ba, Bb, 1 if e > 0 else 0)
            else:
                x = synth.stream_rows_torch(M_HCA * e, M_HCA * (e + 1), c, dtype, seed=SPLIT_SEED,
                                            z_row_offset=Z_OFF, device=device)
                ref = single_hca(x["Ca"], x["Za"], Bh)
            err = np.abs(r[2:].double().numpy() - ref)
            scale = max(float(np.abs(ref).max()), 1e-30)
            if dtype == "bf16":
                bound = 2.0 ** -7 * np.abs(ref) + 1e-5 * scale
            else:
                bound = 1e-5 * scale
            ok = ok and bool(np.all(err <= bound))
            worst = max(worst, float(err.max()) / scale)
            checked += 1
    return checked, worst, ok


def run_split(args):
    """--split sequence: one world x 2^20-token sequence, each rank compressing its own rows
    (CSA m = 4 with the halo, HCA m' = 128); timed like the default step (CUDA events, max
    over ranks); then the sampled cross-rank check against single-GPU recomputation."""
    import torch

    from kv_token_compressor_b200 import kvc

    rank, world, local = dist_setup(args.gpus)
    dev = torch.device("cuda", local if world > 1 else 0)
    stream = torch.cuda.current_stream(dev)
    n_total = world * N_TOK
    t, lo, pc, ph = split_inputs(n_total, world, rank, C, "bf16", dev)
    out_c = torch.empty((1, pc.entries + int(pc.drop_first), C), device=dev, dtype=torch.bfloat16)
    out_h = torch.empty((1, ph.entries, C), device=dev, dtype=torch.bfloat16)

    def csa_fn(sl, Ba, Bb, out):
        kvc.csa_compress(sl["Ca"], sl["Cb"], sl["Za"], sl["Zb"], Ba, Bb, m=M_CSA, out=out,
                         stream=stream)

    def hca_fn(Cs, Zs, B, out):
        kvc.hca_compress(Cs, Zs, B, m=M_HCA, out=out, stream=stream)

    for _ in range(max(args.warmup, 3)):
        split_compress(t, lo, pc, ph, csa_fn, hca_fn, out_c, out_h)
    torch.cuda.synchronize()
    if kvc.device_status(stream) != kvc.KVC_OK:
        raise SystemExit("device error during warm-up")
    barrier(world)
    torch.cuda.synchronize()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(args.steps):
        owned_c, owned_h = split_compress(t, lo, pc, ph, csa_fn, hca_fn, out_c, out_h)
    e1.record(stream)
    torch.cuda.synchronize()
    barrier(world)
    ms = max_over_ranks(e0.elapsed_time(e1), world) / args.steps

    def single_csa(x, Ba, Bb, j):
        o = kvc.csa_compress(x["Ca"], x["Cb"], x["Za"], x["Zb"], Ba, Bb, m=M_CSA,
                             out_dtype=torch.float32)
        return o[0, j].double().cpu().numpy()

    def single_hca(Cs, Zs, B):
        return kvc.hca_compress(Cs, Zs, B, m=M_HCA, out_dtype=torch.float32)[0, 0].double().cpu().numpy()

    check = split_check(world, rank, pc, ph, owned_c, owned_h, C, "bf16", dev, single_csa,
                        single_hca)
    if rank == 0:
        entries = n_total // M_CSA + n_total // M_HCA
        line = {
            "metric": METRIC, "value": n_total / (ms * 1e-3), "unit": "tokens/s",
            "entries_per_s": entries / (ms * 1e-3), "n_gpus": world, "steps": args.steps,
            "warmup": max(args.warmup, 3), "ms_per_step": ms, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f32", "data": "synthetic",
            "config": {"workload": f"one sequence of {world} x 2^20 tokens, c=512, bf16 in/out; "
                                   "CSA m=4 overlap + HCA m'=128 on the same streams",
                       "n": n_total, "c": C, "m": M_CSA, "m_hca": M_HCA,
                       "l2": "inputs 4.3 GB per rank > 126 MB L2, no flush",
                       "parallelism": f"sequence split over {world} ranks: contiguous entry "
                                      "ranges, one-block CSA halo, no data-path collective"},
            "gpu_launches": 2 * args.steps,
            "split_check": {"entries": check[0], "max_rel_err": check[1], "ok": check[2],
                            "against": "each sampled entry recomputed on rank 0 as a "
                                       "one-sequence problem of its own rows"},
        }
        print(json.dumps(line), flush=True)
        if not check[2]:
            raise SystemExit("split check failed")
    if world > 1:
        import torch.distributed as dist

        dist.destroy_process_group()


# ------------------------------------------------------------------------------ other paths

def _peak(kind, sustained=False):
    """Measured roofline denominators (MEASURED_PEAKS.json), else the recipe's fallback.
    For the tensor pipe: the burst cuBLAS figure, or the seconds-long sustained one."""
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        if kind == "hbm":
            return float(d["hbm_gbs"]), "measured"
        key = "bf16_tflops_sustained" if sustained and "bf16_tflops_sustained" in d else "bf16_tflops"
        return float(d[key]), "measured"
    return (FALLBACK_HBM_GBS if kind == "hbm" else (1400.0 if sustained else 1590.0)), "fallback"


def _workload(name, dev):
    """Inputs, launch function, outputs and roofline units of one named workload."""
    import torch

    from kv_token_compressor_b200 import kvc, synth

    bf = torch.bfloat16
    if name in ("fused_csa", "fused_indexer_keys"):
        n, d, c = 32768, 7168, (512 if name == "fused_csa" else 128)
        t = synth.fused_inputs_torch("csa", 1, n, d, c, 4, seed=0, device=dev)
        out = torch.empty((1, n // 4, c), device=dev, dtype=bf)

        def launch(x, st):
            kvc.csa_compress_fused_proj(x["H"], x["W_kva"], x["W_kvb"], x["W_za"], x["W_zb"],
                                        x["Ba"], x["Bb"], 1, n, m=4, out=out, stream=st)
        return dict(inputs=t, launch=launch, outputs=[out], tokens=n, entries=n // 4,
                    bound="tensor", units=2.0 * n * d * 4 * c, flush=False,
                    kernel=("fused_pair_kernel<CSA> (CTA pairs, M=256)" if c % 128 == 0
                            else "fused_pool_kernel<CSA>"),
                    traffic_key="fused_csa_n32768_d7168" if (n, d, c) == (32768, 7168, 512) else None,
                    config={"workload": f"CSA fused projection + pool: H [{n}, {d}] bf16, 4 W "
                                        f"[{d}, {c}] bf16, m=4 overlap, bf16 out", "n": n,
                            "d": d, "c": c, "m": 4})
    if name == "fused_csa_cache":
        n, d, c, r = 32768, 7168, 512, 64
        t = synth.fused_inputs_torch("csa", 1, n, d, c, 4, seed=0, device=dev)
        t["inv_freq"] = (10000.0 ** (-torch.arange(r // 2, device=dev, dtype=torch.float64)
                                     * 2 / r)).float()
        nope = torch.empty((n // 4, c - r), device=dev, dtype=torch.uint8)
        rope = torch.empty((n // 4, r), device=dev, dtype=bf)

        def launch(x, st):
            kvc.csa_compress_fused_proj_cache(x["H"], x["W_kva"], x["W_kvb"], x["W_za"],
                                              x["W_zb"], x["Ba"], x["Bb"], 1, n, r,
                                              x["inv_freq"], out_nope=nope, out_rope=rope,
                                              stream=st)
        return dict(inputs=t, launch=launch, outputs=[nope, rope], tokens=n, entries=n // 4,
                    bound="tensor", units=2.0 * n * d * 4 * c, flush=False,
                    kernel="fused_pair_kernel<CSA, cache layout> (CTA pairs, M=256)",
                    config={"workload": f"CSA fused projection + pool, cache layout: H [{n}, {d}] "
                                        f"bf16, 4 W [{d}, {c}] bf16, m=4 overlap, E4M3 [c-{r}] "
                                        f"+ RoPE'd bf16 [{r}]", "n": n, "d": d, "c": c, "m": 4,
                            "r": r})
    if name in ("fused_csa_scalar", "fused_hca_scalar"):
        csa = name == "fused_csa_scalar"
        b, n, d, c, m = (1, 32768, 7168, 512, 4) if csa else (4, 131072, 4096, 512, 128)
        t = synth.fused_scalar_inputs_torch("csa" if csa else "hca", b, n, d, c, m, seed=0,
                                            device=dev)
        out = torch.empty((b, n // m, c), device=dev, dtype=bf)

        def launch(x, st):
            if csa:
                kvc.csa_compress_fused_proj_scalar(x["H"], x["W_kva"], x["W_kvb"], x["w_za"],
                                                   x["w_zb"], x["ba"], x["bb"], b, n, out=out,
                                                   stream=st)
            else:
                kvc.hca_compress_fused_proj_scalar(x["H"], x["W_kv"], x["w_z"], x["b"], b, n,
                                                   out=out, stream=st)
        streams = 2 if csa else 1
        return dict(inputs=t, launch=launch, outputs=[out], tokens=b * n, entries=b * n // m,
                    bound="tensor", units=2.0 * b * n * d * streams * c, flush=False,
                    kernel=f"fused_scalar_kernel<{'CSA' if csa else 'HCA'}> (CTA pairs, M=256; "
                           "scores on the CUDA cores beside the MMAs)",
                    config={"workload": f"{'CSA' if csa else 'HCA'} fused projection + pool, "
                                        f"scalar logits: batch {b}, n={n}, H d={d} bf16, "
                                        f"{streams} value W [{d}, {c}] + {streams} score vectors "
                                        f"[{d}], m={m}, bf16 out; FLOPs count the value "
                                        f"projections (tensor cores), not the 2 x {streams} "
                                        f"x n x d of the scores",
                            "batch": b, "n": n, "d": d, "c": c, "m": m})
    if name == "fused_hca":
        b, n, d, c = 4, 131072, 4096, 512
        t = synth.fused_inputs_torch("hca", b, n, d, c, 128, seed=0, device=dev)
        out = torch.empty((b, n // 128, c), device=dev, dtype=bf)

        def launch(x, st):
            kvc.hca_compress_fused_proj(x["H"], x["W_kv"], x["W_z"], x["B"], b, n, m=128,
                                        out=out, stream=st)
        return dict(inputs=t, launch=launch, outputs=[out], tokens=b * n, entries=b * n // 128,
                    bound="tensor", units=2.0 * b * n * d * 2 * c, flush=False,
                    kernel="fused_pair_kernel<HCA> (CTA pairs, M=256)",
                    traffic_key="fused_hca_4x131072_d4096",
                    config={"workload": f"HCA fused projection + pool: batch {b}, n={n}, H d={d} "
                                        f"bf16, W_kv, W_z [{d}, {c}], m'=128, bf16 out",
                            "batch": b, "n": n, "d": d, "c": c, "m": 128})
    if name == "indexer_decode":
        T, H, S, k = 8, 64, 1 << 18, 1024
        t = synth.indexer_inputs_torch(T, H, T * S, seed=0, device=dev)
        t["key_start"] = torch.arange(T, dtype=torch.int64, device=dev) * S
        t["n_visible"] = torch.full((T,), S, dtype=torch.int64, device=dev)
        scores = torch.empty((T, S), dtype=torch.float32, device=dev)
        idx = torch.empty((T, k), dtype=torch.int32, device=dev)
        val = torch.empty((T, k), dtype=torch.float32, device=dev)

        def score(x, st):
            kvc.lightning_indexer_scores(x["q"], x["w"], x["K"], x["key_start"], x["n_visible"],
                                         S, scores=scores, stream=st)

        def select(x, st):
            kvc.indexer_topk(scores, x["n_visible"], k, S, out_idx=idx, out_score=val, stream=st)

        def launch(x, st):
            score(x, st)
            select(x, st)
        score_bytes = float(T * S * 128 * 2 + T * S * 4 + T * H * 128 * 2 + T * H * 4)
        topk_bytes = float(T * S * 4 + T * k * 8)
        return dict(inputs=t, launch=launch, outputs=[idx, val], tokens=T * S * 4, entries=T * S,
                    bound="hbm", units=score_bytes, flush=False, resident=("K",),
                    kernel="indexer_score_kernel (tcgen05, keys on M, heads on N)",
                    traffic_key="indexer_scores_decode_8x262144",
                    parts=[dict(name="indexer_score_kernel", launch=score, units=score_bytes,
                                bound="hbm"),
                           dict(name="indexer_topk_kernel", launch=select, units=topk_bytes,
                                bound="hbm")],
                    config={"workload": f"lightning-indexer decode step: {T} sequences of 2^20 "
                                        f"tokens ({S} compressed indexer keys each, 128 wide, "
                                        f"bf16), one {H}-head query per sequence, top-{k}",
                            "queries": T, "keys_per_query": S, "heads": H, "k": k})
    if name == "scalar_long":
        n, c, m = 1 << 20, 512, 4
        t = synth.scalar_inputs_torch("csa", 1, n, c, m, "bf16", seed=0, device=dev)
        out = torch.empty((1, n // m, c), device=dev, dtype=bf)

        def launch(x, st):
            kvc.csa_compress_scalar_logits(x["Ca"], x["Cb"], x["za"], x["zb"], x["ba"], x["bb"],
                                           m=m, out=out, stream=st)
        ne = n // m
        rows = ne * m + (ne - 1) * m  # a-rows of every entry + b-rows of entries 1..
        nbytes = rows * c * 2 + rows * 2 + 2 * m * 4 + ne * c * 2  # values, logits, biases, out
        return dict(inputs=t, launch=launch, outputs=[out], tokens=n, entries=ne, bound="hbm",
                    units=float(nbytes), flush=False, kernel="scalar_small_m_kernel",
                    traffic_key="csa_scalar_bf16_n1048576",
                    config={"workload": f"scalar-logit CSA: batch 1, n={n}, c={c}, m=4 overlap, "
                                        "bf16 streams and logits", "n": n, "c": c, "m": m})
    if name == "cache_long":
        n, c, m, r = 1 << 20, 512, 4, 64
        t = synth.stream_inputs_torch("csa", 1, n, c, m, "bf16", seed=0, z_row_offset=Z_OFF,
                                      device=dev)
        t["inv_freq"] = (10000.0 ** (-torch.arange(r // 2, device=dev, dtype=torch.float64)
                                     * 2 / r)).float()
        ne = n // m
        nope = torch.empty((ne, c - r), device=dev, dtype=torch.uint8)
        rope = torch.empty((ne, r), device=dev, dtype=bf)

        def launch(x, st):
            kvc.csa_compress_cache(x["Ca"], x["Cb"], x["Za"], x["Zb"], x["Ba"], x["Bb"], r,
                                   x["inv_freq"], 4.0, 1.5, 1.0, m=m, out_nope=nope,
                                   out_rope=rope, stream=st)
        nbytes = (2 * ne * m + 2 * (ne - 1) * m) * c * 2 + 2 * m * c * 4 + ne * ((c - r) + 2 * r)
        return dict(inputs=t, launch=launch, outputs=[nope, rope], tokens=n, entries=ne,
                    bound="hbm", units=float(nbytes), flush=False,
                    kernel="csa_small_m_kernel (cache layout)", traffic_key="csa_cache_bf16_n1048576",
                    config={"workload": f"CSA n={n}, c={c}, m=4, bf16 streams, entries written "
                                        f"as E4M3 [c-{r}] + RoPE'd bf16 [{r}]", "n": n, "c": c,
                            "m": m, "r": r})
    if name == "decode_entries":
        seqs, c, m = 4096, 512, 4
        g = torch.Generator(device=dev)
        g.manual_seed(0)
        lens = torch.randint(8, 1024, (seqs,), generator=g, device=dev) // m * m
        starts = torch.cumsum(lens, 0) - lens
        rows = int(lens.sum().item())
        t = synth.stream_inputs_torch("csa", 1, rows, c, m, "bf16", seed=0, device=dev)
        t = {k: (v[0] if v.dim() == 3 else v) for k, v in t.items()}
        # K lists, list j naming entry (last - j) of every sequence: consecutive launches
        # read distinct rows (K x 68 MB, far beyond the 126 MB L2), so no flush is needed
        K = 8
        ne_seq = (lens // m).to(torch.int64)
        ents = torch.stack([(ne_seq - 1 - j) % ne_seq for j in range(K)])
        t.update(seq_start=starts.to(torch.int64), seq_len=lens.to(torch.int64), entry=ents)
        out = torch.empty((seqs, c), device=dev, dtype=bf)
        turn = [0]
        lists = [ents[j] for j in range(K)]  # taken apart before timing, not in the launch

        def launch(x, st):
            j = turn[0] % K
            turn[0] += 1
            kvc.csa_compress_entries(x["Ca"], x["Cb"], x["Za"], x["Zb"], x["Ba"], x["Bb"],
                                     x["seq_start"], x["seq_len"],
                                     lists[j] if x is t else x["entry"][j], m=m, out=out,
                                     stream=st)
        nbytes = seqs * (4 * m * c * 2 + c * 2 + 24) + 2 * m * c * 4
        return dict(inputs=t, launch=launch, outputs=[out], tokens=seqs * m, entries=seqs,
                    bound="hbm", units=float(nbytes), flush=False,
                    l2=f"{K} entry lists over distinct rows ({K} x {nbytes / 1e6:.0f} MB) taken "
                       "in turn, no flush",
                    kernel="csa_small_m_kernel (listed)",
                    traffic_key="csa_compress_entries_decode_4096",
                    resident=("Ca", "Cb", "Za", "Zb", "Ba", "Bb"),
                    config={"workload": f"decode step: {seqs} sequences (lengths U[8, 1024)) each "
                                        f"emitting one CSA entry (the newest, or one of the {K - 1} "
                                        f"before it), c={c}, m=4, bf16",
                            "sequences": seqs, "c": c, "m": m})
    if name in ("hca_n65536", "hca_n65536_prepared", "csa_f32_n1024", "indexer_keys"):
        if name in ("hca_n65536", "hca_n65536_prepared"):
            mode, n, c, m, dt = "hca", 65536, 512, 128, "bf16"
        elif name == "csa_f32_n1024":
            mode, n, c, m, dt = "csa", 1024, 512, 4, "f32"
        else:
            mode, n, c, m, dt = "csa", 1 << 20, 128, 4, "bf16"
        tdt = bf if dt == "bf16" else torch.float32
        out = torch.empty((1, n // m, c), device=dev, dtype=tdt)
        es = 2 if dt == "bf16" else 4
        streams = ("C", "Z") if mode == "hca" else ("Ca", "Cb", "Za", "Zb")
        one = len(streams) * n * c * es
        # problems smaller than a few L2s: K seeded input sets taken in turn, together well
        # beyond the 126 MB L2, so each launch reads from DRAM with no flush between launches
        K = max(1, -(-(512 << 20) // one)) if one < 4 * (126 << 20) else 1
        sets = [synth.stream_inputs_torch(mode, 1, n, c, m, dt, seed=j, device=dev) for j in range(K)]
        t = {k: torch.stack([st_[k] for st_ in sets]) for k in streams}
        t.update({k: v for k, v in sets[0].items() if k not in streams})  # the biases of set 0
        del sets
        if name == "hca_n65536_prepared":
            # the bias is a weight: prepared once, outside the timed region
            t["ws"] = kvc.hca_prepare_bias(t["B"], tdt)
        # each set's tensors, taken apart once here: indexing the stacks between the event
        # records would put host time inside the timed launch
        views = [{k: (v[j] if k in streams else v) for k, v in t.items()} for j in range(K)]
        one_set = views[0]
        turn = [0]

        def pick(x):
            if x is not t:  # a single set (e2e)
                return x
            j = turn[0] % K
            turn[0] += 1
            return views[j]
        if name == "hca_n65536_prepared":
            def launch(x, st):
                y = pick(x)
                kvc.hca_compress_prepared(y["C"], y["Z"], y["ws"], m=m, out=out, stream=st)
            nbytes = 2 * n * c * es + m * c * 4 + (n // m) * c * es
        elif mode == "hca":
            def launch(x, st):
                y = pick(x)
                kvc.hca_compress(y["C"], y["Z"], y["B"], m=m, out=out, stream=st)
            nbytes = 2 * n * c * es + m * c * 4 + (n // m) * c * es
        else:
            def launch(x, st):
                y = pick(x)
                kvc.csa_compress(y["Ca"], y["Cb"], y["Za"], y["Zb"], y["Ba"], y["Bb"], m=m,
                                 out=out, stream=st)
            ne = n // m
            nbytes = (2 * ne * m + 2 * (ne - 1) * m) * c * es + 2 * m * c * 4 + ne * c * es
        return dict(inputs=t, e2e_inputs=one_set, launch=launch, outputs=[out], tokens=n,
                    entries=n // m, bound="hbm", units=float(nbytes), flush=False,
                    l2=(f"{K} seeded input sets taken in turn ({K} x {one / 1e6:.1f} MB), no flush"
                        if K > 1 else "inputs larger than L2"),
                    kernel=("csa_tma_kernel (TMA-fed, small problems)" if name == "csa_f32_n1024"
                            else "window_tma_kernel (prepared bias, 8 row groups)"
                            if name == "hca_n65536_prepared"
                            else "csa_small_m_kernel" if mode == "csa" else
                            "window_tma_kernel (TMA-fed, 8 row groups)"),
                    traffic_key={"hca_n65536": "hca_compress_bf16_n65536",
                                 "csa_f32_n1024": "csa_compress_f32_n1024",
                                 "indexer_keys": "csa_compress_bf16_c128_n1048576"}.get(name),
                    config={"workload": f"{mode.upper()} streams: batch 1, n={n}, c={c}, m={m}, "
                                        f"{dt} in/out"
                                        + (", bias prepared once" if name.endswith("prepared")
                                           else ""), "n": n, "c": c, "m": m})
    raise SystemExit(f"unknown workload {name}")


def run_workload(args):
    """One JSON line for a named workload other than the default step (1 GPU, or weak
    replicas under torchrun); the kernel is timed per launch with CUDA events, L2 flushed
    between launches when the inputs are not far larger than L2."""
    import torch

    from kv_token_compressor_b200 import kvc

    rank, world, local = dist_setup(args.gpus)
    dev = torch.device("cuda", local if world > 1 else 0)
    w = _workload(args.workload, dev)
    st = torch.cuda.current_stream(dev)
    flush = torch.empty(512 << 20, dtype=torch.uint8, device=dev) if w["flush"] else None
    for _ in range(max(args.warmup, 3)):
        w["launch"](w["inputs"], st)
    torch.cuda.synchronize()
    if kvc.device_status(st) != kvc.KVC_OK:
        raise SystemExit("device error during warm-up")
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(args.steps)]
    uuid = str(getattr(torch.cuda.get_device_properties(dev), "uuid", ""))
    sampler = clock_sampler(("GPU-" + uuid) if uuid and not uuid.startswith("GPU-") else (uuid or "0"))
    sampler.start()
    barrier(world)
    torch.cuda.synchronize()
    sampler.mark(True)
    if flush is None:
        # a spin on the GPU while the host queues every launch and its events: otherwise a
        # launch shorter than the binding's host-side work would leave the GPU idle between
        # an event and its kernel, and the event pair would time the host
        torch.cuda._sleep(int(2e5 * args.steps))
    for a, b in evs:
        if flush is not None:
            flush.zero_()
        a.record(st)
        w["launch"](w["inputs"], st)
        b.record(st)
    torch.cuda.synchronize()
    sampler.mark(False)
    barrier(world)
    clocks = sampler.stop()
    ms = max_over_ranks(statistics.median(a.elapsed_time(b) for a, b in evs), world)
    if kvc.device_status(st) != kvc.KVC_OK:
        raise SystemExit("device error in the timed region")
    # workloads made of several kernels: time each on its own as well (same loop)
    part_ms = {}
    for part in w.get("parts", ()):
        pev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
               for _ in range(args.steps)]
        torch.cuda.synchronize()
        if flush is None:
            torch.cuda._sleep(int(2e5 * args.steps))
        for a, b in pev:
            if flush is not None:
                flush.zero_()
            a.record(st)
            part["launch"](w["inputs"], st)
            b.record(st)
        torch.cuda.synchronize()
        part_ms[part["name"]] = max_over_ranks(
            statistics.median(a.elapsed_time(b) for a, b in pev), world)
    # e2e: pinned host inputs -> device, the call, outputs -> pinned host
    # inputs the workload keeps resident in device memory (a decode step's KV streams) are
    # not copied; everything else is
    resident = set(w.get("resident", ()))
    host = {k: v.cpu().pin_memory() for k, v in (w.get("e2e_inputs") or w["inputs"]).items()
            if k not in resident}
    houts = [torch.empty(o.shape, dtype=o.dtype).pin_memory() for o in w["outputs"]]
    h2d = sum(v.numel() * v.element_size() for v in host.values())
    d2h = sum(o.numel() * o.element_size() for o in houts)

    def e2e():
        dv = {k: v.to(dev, non_blocking=True) for k, v in host.items()}
        dv.update({k: w["inputs"][k] for k in resident})
        w["launch"](dv, st)
        for ho, o in zip(houts, w["outputs"]):
            ho.copy_(o, non_blocking=True)

    e2e()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    n_e2e = 3
    e0.record(st)
    for _ in range(n_e2e):
        e2e()
    e1.record(st)
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks(e0.elapsed_time(e1), world) / n_e2e
    peak, kind = _peak(w["bound"])
    # the roofline is the dominant kernel's: its own time when the step has several
    rms = part_ms[w["parts"][0]["name"]] if w.get("parts") else ms
    if w["bound"] == "tensor":
        ach, unit = w["units"] / (rms * 1e-3) / 1e12, "TFLOP/s"
    else:
        ach, unit = w["units"] / (rms * 1e-3) / 1e9, "GB/s"
    if rank == 0:
        line = {
            "metric": METRIC, "value": world * w["tokens"] / (ms * 1e-3), "unit": "tokens/s",
            "entries_per_s": world * w["entries"] / (ms * 1e-3), "n_gpus": world,
            "steps": args.steps, "warmup": max(args.warmup, 3), "ms_per_step": ms,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "f32", "data": "synthetic",
            "config": dict(w["config"], l2=w.get("l2") or ("flushed between launches" if w["flush"]
                                                           else "inputs larger than L2")),
            "roofline": {"bound": w["bound"], "kernel": w["kernel"], "achieved": ach,
                         "peak": peak, "unit": unit, "frac": ach / peak, "peak_kind": kind,
                         "frac_of_sustained": (ach / _peak("tensor", True)[0]
                                               if w["bound"] == "tensor" else None),
                         "traffic": _traffic(w["traffic_key"]) if w.get("traffic_key") else None,
                         ("algorithmic_flops" if w["bound"] == "tensor" else "algorithmic_bytes"):
                             w["units"]},
            "gpu_launches": args.steps * max(1, len(w.get("parts", ()))),
            "e2e": {"value": world * w["tokens"] / (e2e_ms * 1e-3), "unit": "tokens/s",
                    "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms},
        }
        line["clocks"] = clocks
        if world == 1 and not args.no_cpu_baseline:
            try:
                cb = cpu_baseline_workload(args.workload)
            except Exception as e:  # the GPU line is printed whatever happens here
                cb = {"error": f"oracle timing failed: {e!r}"}
            if cb is not None:
                line["cpu_baseline"] = cb
        if w.get("parts"):
            line["kernels"] = {}
            for part in w["parts"]:
                pm = part_ms[part["name"]]
                pk, _ = _peak(part["bound"])
                a_ = part["units"] / (pm * 1e-3) / 1e9
                line["kernels"][part["name"]] = {"ms": pm, "GB/s": a_, "frac": a_ / pk}
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist

        dist.destroy_process_group()


def run_profile_case(kind: str, launches: int = 3):
    """A small case of one kernel for Nsight Compute captures (inputs still larger than
    L2 for the streaming kernels; a few hundred MB on the device at most).  Prints one
    line; not a bench value."""
    import torch

    from kv_token_compressor_b200 import kvc, synth

    torch.cuda.set_device(0)
    if kind in ("csa", "hca"):
        n = 1 << 18 if kind == "csa" else 1 << 19  # HCA: enough windows for one per thread
        t = synth.stream_inputs_torch("csa", 1, n, C, M_CSA, "bf16", seed=0, z_row_offset=Z_OFF)
        Bh = torch.randn((M_HCA, C), device="cuda") * float(np.sqrt(0.1))
        for _ in range(launches):
            if kind == "csa":
                kvc.csa_compress(t["Ca"], t["Cb"], t["Za"], t["Zb"], t["Ba"], t["Bb"], m=M_CSA)
            else:
                kvc.hca_compress(t["Ca"], t["Za"], Bh, m=M_HCA)
    elif kind == "hca_n65536":  # the 65536-token HCA workload itself (134 MB, few windows)
        t = synth.stream_inputs_torch("hca", 1, 65536, C, M_HCA, "bf16", seed=0)
        flush = torch.empty(256 << 20, dtype=torch.uint8, device="cuda")
        for _ in range(launches):
            flush.zero_()
            kvc.hca_compress(t["C"], t["Z"], t["B"], m=M_HCA)
    elif kind == "csa_n1024":  # the n = 1024 fp32 CSA workload itself (TMA-fed small-problem kernel)
        t = synth.stream_inputs_torch("csa", 1, 1024, C, M_CSA, "f32", seed=0)
        flush = torch.empty(256 << 20, dtype=torch.uint8, device="cuda")
        for _ in range(launches):
            flush.zero_()
            kvc.csa_compress(t["Ca"], t["Cb"], t["Za"], t["Zb"], t["Ba"], t["Bb"], m=M_CSA)
    elif kind == "indexer_keys":  # CSA at c = 128 (indexer keys), n = 2^18 (268 MB of streams)
        t = synth.stream_inputs_torch("csa", 1, 1 << 18, 128, M_CSA, "bf16", seed=0)
        for _ in range(launches):
            kvc.csa_compress(t["Ca"], t["Cb"], t["Za"], t["Zb"], t["Ba"], t["Bb"], m=M_CSA)
    elif kind == "decode":  # a decode list: 4096 sequences of lengths U[8, 64), newest entry each
        g = torch.Generator(device="cuda")
        g.manual_seed(0)
        lens = torch.randint(8, 64, (4096,), generator=g, device="cuda") // M_CSA * M_CSA
        starts = torch.cumsum(lens, 0) - lens
        t = synth.stream_inputs_torch("csa", 1, int(lens.sum().item()), C, M_CSA, "bf16", seed=0)
        flush = torch.empty(256 << 20, dtype=torch.uint8, device="cuda")
        for _ in range(launches):
            flush.zero_()
            kvc.csa_compress_entries(t["Ca"][0], t["Cb"][0], t["Za"][0], t["Zb"][0], t["Ba"], t["Bb"],
                                     starts, lens, lens // M_CSA - 1, m=M_CSA)
    elif kind == "scalar":  # scalar-logit CSA, n = 2^18 (the scalar workload / 4)
        t = synth.scalar_inputs_torch("csa", 1, 1 << 18, C, M_CSA, "bf16", seed=0)
        for _ in range(launches):
            kvc.csa_compress_scalar_logits(t["Ca"], t["Cb"], t["za"], t["zb"], t["ba"], t["bb"], m=M_CSA)
    elif kind == "cache":  # CSA into the cache layout, n = 2^18 (the cache workload / 4)
        n, r = 1 << 18, 64
        t = synth.stream_inputs_torch("csa", 1, n, C, M_CSA, "bf16", seed=0, z_row_offset=Z_OFF)
        inv = (10000.0 ** (-torch.arange(r // 2, device="cuda", dtype=torch.float64) * 2 / r)).float()
        for _ in range(launches):
            kvc.csa_compress_cache(t["Ca"], t["Cb"], t["Za"], t["Zb"], t["Ba"], t["Bb"], r, inv, 4.0,
                                   1.5, 1.0, m=M_CSA)
    elif kind == "indexer":  # 4 queries x 131072 keys (K 128 MB), top-1024
        T, S = 4, 1 << 17
        t = synth.indexer_inputs_torch(T, 64, T * S, seed=0)
        ks = torch.arange(T, dtype=torch.int64, device="cuda") * S
        nv = torch.full((T,), S, dtype=torch.int64, device="cuda")
        sc = torch.empty((T, S), dtype=torch.float32, device="cuda")
        for _ in range(launches):
            kvc.lightning_indexer_scores(t["q"], t["w"], t["K"], ks, nv, S, scores=sc)
            kvc.indexer_topk(sc, nv, 1024, S)
    elif kind in ("csa_fused", "csa_fused_n32768"):
        # n = 4096: one tile per pair; n = 32768: the fused CSA workload itself (0.5 GB on
        # the device; several tiles per pair, the carried partials between them)
        n, d = (4096 if kind == "csa_fused" else 32768), 7168
        f = synth.fused_inputs_torch("csa", 1, n, d, C, M_CSA, seed=0)
        for _ in range(launches):
            kvc.csa_compress_fused_proj(f["H"], f["W_kva"], f["W_kvb"], f["W_za"], f["W_zb"],
                                        f["Ba"], f["Bb"], 1, n)
    elif kind == "csa_fused_scalar_n32768":  # the scalar-logit fused CSA workload itself
        n, d = 32768, 7168
        f = synth.fused_scalar_inputs_torch("csa", 1, n, d, C, M_CSA, seed=0)
        for _ in range(launches):
            kvc.csa_compress_fused_proj_scalar(f["H"], f["W_kva"], f["W_kvb"], f["w_za"], f["w_zb"],
                                               f["ba"], f["bb"], 1, n)
    elif kind == "hca_fused":
        n, d = 16384, 4096
        f = synth.fused_inputs_torch("hca", 1, n, d, C, M_HCA, seed=0)
        for _ in range(launches):
            kvc.hca_compress_fused_proj(f["H"], f["W_kv"], f["W_z"], f["B"], 1, n)
    else:
        raise SystemExit(f"unknown profile case {kind}")
    torch.cuda.synchronize()
    st = kvc.device_status()
    print(json.dumps({"profile_case": kind, "launches": launches, "device_status": st}))
    if st != kvc.KVC_OK:
        raise SystemExit(1)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=1000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--split", choices=["replicas", "sequence"], default="replicas",
                    help="replicas (default): every rank its own 2^20-token problem; sequence: "
                         "one world x 2^20-token sequence split over the ranks (shard plan)")
    ap.add_argument("--no-fused", action="store_true",
                    help="skip the fused-path kernels timed after the default step")
    ap.add_argument("--workload", default="long",
                    choices=["long", "fused_csa", "fused_csa_cache", "fused_csa_scalar",
                             "fused_hca_scalar", "fused_hca", "hca_n65536",
                             "hca_n65536_prepared", "csa_f32_n1024",
                             "indexer_keys", "fused_indexer_keys", "scalar_long",
                             "decode_entries", "cache_long", "indexer_decode"],
                    help="long (default): CSA + HCA over the 2^20-token streams; the others "
                         "time one kernel on its own workload")
    ap.add_argument("--profile-case", choices=["csa", "hca", "hca_n65536", "csa_n1024", "indexer_keys",
                                               "decode", "scalar", "cache", "indexer", "csa_fused",
                                               "csa_fused_n32768", "csa_fused_scalar_n32768",
                                               "hca_fused"],
                    help="run one kernel on a small case for ncu (no bench line)")
    args = ap.parse_args()
    if args.profile_case:
        run_profile_case(args.profile_case)
    elif args.impl == "reference":
        run_reference(args)
    else:
        if args.split == "sequence":
            run_split(args)
        else:
            run_ours(args) if args.workload == "long" else run_workload(args)


if __name__ == "__main__":
    main()
