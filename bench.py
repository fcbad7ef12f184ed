"""Benchmark of the LCA decode step (one step = one lca_decode over one batch).

  python bench.py [--gpus N] [--steps K] [--warmup W] [--blocks R]
                  [--impl ours|reference|ranks] [--workload v2] [--g G] [--w W]
                  [--no-cpu-baseline] [--no-e2e] [--no-per-config]

Default workload: the DeepSeek-V2-shaped decode (B=32, H=128 heads sharing one
latent, d_c=512, d_r=64, L=65536, g=16, w=2048, bf16 latents, queries
N(0,1)/sqrt(576)) -- the largest workload that fits one GPU -- with synthetic
seeded inputs.  Metric: context tokens per second (B*L per step), whole job
over all ranks, from the median of R timed blocks of K steps each.  Under
torchrun every rank runs its own batch on its own GPU (sequences are
independent: no collective on the data path) and the time is the max over
ranks ("weak" scaling); `--gpus N` without torchrun starts the N ranks itself.
The other benchmark workloads (V2-Lite, needle, the ten sweep points, the tiny
fp32 case) are timed in the same process under "per_config".

Prints one JSON line on rank 0.  `--impl reference` times the CPU oracle on
the host cores instead (rank 0 only), on bounded samples of the same workload.
`--impl ranks` runs only the rank plumbing (gloo, CPU) as a stand-in arm.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402

import workloads  # noqa: E402

METRIC = "LCA decode context tokens/s per GPU; HBM GB/s as % of B200 peak"
UNIT = "context tokens/s"
L2_BYTES = 126 * 1024 * 1024
# committed ncu DRAM-traffic summaries of the main kernel, per workload, and
# the sources of that kernel (a summary counts only while they are unchanged)
_CSRC = "kv_compression_b200/csrc/"
TRAFFIC_FILES = {
    "v2lite": ("profiles/lca_tc_kernel_v2lite_traffic.txt",
               [_CSRC + "tc_kernel.cuh", _CSRC + "ptx.cuh", _CSRC + "checks.cuh", _CSRC + "paged_kernel.cuh"]),
    "v2": ("profiles/lca_pair_kernel_v2_traffic.txt",
           [_CSRC + "pair_kernel.cuh", _CSRC + "ptx.cuh", _CSRC + "checks.cuh", _CSRC + "paged_kernel.cuh"]),
}
MAIN_KERNEL_NAMES = {"tcgen05": "lca_tc_kernel", "tcgen05_pair": "lca_pair_kernel", "simt": "lca_simt_kernel"}


def workload_desc(wl: workloads.Workload) -> str:
    return (f"{wl.name}: B={wl.B} H={wl.H} d_c={wl.d_c} d_r={wl.d_r} L={wl.L} g={wl.g} w={wl.w} "
            f"{wl.dtype} latents, q*{wl.q_scale:.4g}")


def algorithmic_bytes(wl: workloads.Workload) -> int:
    """Cache read once + queries + fp32 output + int32 anchors."""
    es = wl.elem_bytes
    cache = wl.B * wl.L * (wl.d_c + wl.d_r) * es
    q = wl.B * wl.H * (wl.d_c + wl.d_r) * es
    out = wl.B * wl.H * wl.d_c * 4
    anc = wl.B * wl.H * wl.n_groups * 4
    return cache + q + out + anc


def measured_peaks() -> tuple[dict, str]:
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            return json.load(f), "measured"
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}, "fallback"


def kernel_source_sha(sources: list[str]) -> str:
    h = hashlib.sha256()
    for rel in sources:
        with open(os.path.join(ROOT, rel), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def profiled_traffic(wl: workloads.Workload) -> int | None:
    """DRAM bytes per launch of the main kernel from the committed ncu summary
    for this workload, or None when absent, taken at another batch size or on a
    different kernel source."""
    entry = TRAFFIC_FILES.get(wl.name)
    path = os.path.join(ROOT, entry[0]) if entry else None
    if not path or not os.path.exists(path):
        return None
    kv = {}
    with open(path) as f:
        for line in f:
            if ":" in line and not line.startswith("#"):
                k, v = line.split(":", 1)
                kv[k.strip()] = v.strip()
    if kv.get("source_sha256") != kernel_source_sha(entry[1]):
        return None
    if "batch" in kv and int(kv["batch"]) != wl.B:
        return None
    try:
        return int(kv["dram_bytes_per_launch"])
    except (KeyError, ValueError):
        return None


class NvmlSampler:
    """Samples SM clock, power and clock-event reasons of one GPU through NVML
    every few milliseconds from a host thread (read-only queries), so that a
    timed region of a few tens of milliseconds still holds samples."""

    REASONS = (("hw_slowdown", "nvmlClocksEventReasonHwSlowdown", 0x8),
               ("hw_thermal_slowdown", "nvmlClocksEventReasonHwThermalSlowdown", 0x40),
               ("sw_thermal_slowdown", "nvmlClocksEventReasonSwThermalSlowdown", 0x20),
               ("sw_power_cap", "nvmlClocksEventReasonSwPowerCap", 0x4))

    def __init__(self, gpu_uuid: str | None, interval_s: float = 0.002):
        import threading
        self.samples: list[tuple[float, float, int]] = []
        self.sm_max = None
        self.ok = False
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nvml = pynvml
            self.h = (pynvml.nvmlDeviceGetHandleByUUID(gpu_uuid) if gpu_uuid
                      else pynvml.nvmlDeviceGetHandleByIndex(0))
            self.sm_max = float(pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM))
            self.ok = True
        except Exception:  # noqa: BLE001 - no NVML: report no samples
            return
        self.interval = interval_s
        self.stop_evt = threading.Event()
        self.thread = threading.Thread(target=self._run, daemon=True)

    def _one(self) -> None:
        n = self.nvml
        sm = float(n.nvmlDeviceGetClockInfo(self.h, n.NVML_CLOCK_SM))
        pw = n.nvmlDeviceGetPowerUsage(self.h) / 1000.0
        rs = n.nvmlDeviceGetCurrentClocksEventReasons(self.h)
        self.samples.append((sm, pw, int(rs)))

    def _run(self) -> None:
        while True:
            try:
                self._one()
            except Exception:  # noqa: BLE001
                return
            if self.stop_evt.wait(self.interval):
                return

    def start(self) -> None:
        if self.ok:
            self.thread.start()

    def stop(self) -> dict:
        if not self.ok:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0, "source": "none"}
        self.stop_evt.set()
        self.thread.join(timeout=5)
        try:
            self._one()                      # one sample at the end of the region
        except Exception:  # noqa: BLE001
            pass
        reasons = set()
        for name, attr, bit in self.REASONS:
            mask = getattr(self.nvml, attr, bit)
            if any(r & mask for _, _, r in self.samples):
                reasons.add(name)
        sm = [s for s, _, _ in self.samples]
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": self.sm_max,
                "reasons": sorted(reasons), "samples": len(sm),
                "power_w_median": statistics.median([p for _, p, _ in self.samples]) if sm else None,
                "source": f"NVML every {self.interval * 1e3:.0f} ms over the timed region"}


class ClockSampler:
    """nvidia-smi samples (200 ms) of one GPU over the whole run, a cross-check
    of the NVML samples taken over the timed region."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_uuid: str | None):
        self.path = tempfile.mktemp(prefix="lca_clocks_", suffix=".csv")
        self.proc = None
        cmd = ["nvidia-smi", f"--query-gpu=timestamp,{self.FIELDS}", "--format=csv,noheader,nounits",
               "-lms", "200"]
        if gpu_uuid:
            cmd += ["-i", gpu_uuid]
        try:
            self.f = open(self.path, "w")
            self.proc = subprocess.Popen(cmd, stdout=self.f, stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None

    def stop(self) -> dict:
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.f.close()
        sm, smax, power, reasons = [], [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        with open(self.path) as f:
            for line in f:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) < 10:
                    continue
                try:
                    sm.append(float(parts[2])); smax.append(float(parts[3])); power.append(float(parts[4]))
                except ValueError:
                    continue
                for n, v in zip(names, parts[6:10]):
                    if v.lower().startswith("active"):
                        reasons.add(n)
        os.unlink(self.path)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": sorted(reasons), "samples": 0}
        idle = min(power)
        loaded = [s for s, p in zip(sm, power) if p > idle + 50.0] or sm
        return {"sm_mhz": statistics.median(loaded), "sm_max_mhz": max(smax),
                "reasons": sorted(reasons), "samples": len(sm), "samples_under_load": len(loaded)}


def to_device(a, torch):
    if a.dtype == np.uint16:
        return torch.from_numpy(a.view(np.int16)).view(torch.bfloat16).cuda()
    return torch.from_numpy(a).cuda()


def run_cpu_oracle_steps(wl, x, steps: int, budget_s: float, nthreads: int):
    """Time the oracle on bounded samples: one sequence per step, heads cut to fit the budget.
    Returns (context tokens per second, description, threads)."""
    from oracle import oracle
    t0 = time.perf_counter()
    oracle.lca(x.q_c[:, :1], x.q_r[:, :1], x.c_kv, x.k_r, g=wl.g, w=wl.w, rows=[0], nthreads=nthreads)
    per_head = time.perf_counter() - t0
    heads = int(max(1, min(wl.H, budget_s / max(steps, 1) / max(per_head, 1e-6))))
    tok, secs = 0.0, 0.0
    for k in range(steps):
        b = k % wl.B
        t0 = time.perf_counter()
        oracle.lca(x.q_c[:, :heads], x.q_r[:, :heads], x.c_kv, x.k_r, g=wl.g, w=wl.w, rows=[b],
                   nthreads=nthreads)
        secs += time.perf_counter() - t0
        tok += wl.L * heads / wl.H     # context tokens, counted at all H heads per token
    desc = (f"{steps} step(s) of one sequence x {heads}/{wl.H} heads of {wl.name} "
            f"(L={wl.L}, g={wl.g}, w={wl.w}), oracle formulation A, {nthreads} threads")
    return tok / secs, desc, secs


def reference_arm(args) -> None:
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    wl = with_point(workloads.WORKLOADS[args.workload], args)
    x = workloads.generate(wl)
    from oracle import oracle
    oracle.build()
    nthreads = os.cpu_count() or 1
    budget = float(os.environ.get("LCA_REFERENCE_BUDGET_S", "120"))
    if args.warmup > 0:
        run_cpu_oracle_steps(wl, x, min(args.warmup, 1), budget / 10, nthreads)
    value, desc, secs = run_cpu_oracle_steps(wl, x, args.steps, budget, nthreads)
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT,
        "n_gpus": int(os.environ.get("WORLD_SIZE", "1")),
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": secs / max(args.steps, 1) * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic (seeded, workloads/)",
        "config": {"workload": workload_desc(wl), "parallelism": "host threads (OpenMP)"},
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": nthreads, "kind": "oracle",
                         "sample": desc},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def with_point(wl: workloads.Workload, args) -> workloads.Workload:
    """The workload at another (g, w) point of the same inputs (e.g. the sweep grid)."""
    if args.g is not None:
        wl = wl.with_(g=args.g)
    if args.w is not None:
        wl = wl.with_(w=args.w)
    if getattr(args, "batch", None):
        wl = wl.with_(B=args.batch)
    return wl


def rank_workload(wl: workloads.Workload, rank: int) -> workloads.Workload:
    """Each rank decodes its own batch: the same shapes, inputs drawn with seed = rank."""
    return wl.with_(seed=rank)


def max_over_ranks(dist, v: float, device) -> float:
    """The largest of one float over all ranks (every rank must call it); v itself
    when there is no process group."""
    if dist is None:
        return v
    import torch
    t = torch.tensor([v], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_rate(world: int, wl: workloads.Workload, steps: int, t_max: float) -> float:
    """Context tokens per second of the whole job: every rank decodes B * L tokens
    per step, and the job takes as long as its slowest rank."""
    return world * wl.B * wl.L * steps / t_max


def algorithmic_flops(wl: workloads.Workload) -> int:
    """Scores 2 H (d_c + d_r) plus the folded P.C 2 H d_c per context token."""
    return wl.B * wl.L * (2 * wl.H * (wl.d_c + wl.d_r) + 2 * wl.H * wl.d_c)


def spawn_ranks(args) -> int | None:
    """`--gpus N` without torchrun: start N local ranks under torch.distributed.run
    (rendezvous on 127.0.0.1) and return their exit status; None when this
    process already is a rank (WORLD_SIZE set) or N == 1."""
    if args.gpus <= 1 or "WORLD_SIZE" in os.environ:
        return None
    import socket
    with socket.socket(socket.AF_INET, socket.SOCK_STREAM) as sk:
        sk.bind(("127.0.0.1", 0))
        port = sk.getsockname()[1]
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes", "1", "--nproc-per-node",
           str(args.gpus), "--master-addr", "127.0.0.1", "--master-port", str(port),
           os.path.abspath(__file__), *sys.argv[1:]]
    return subprocess.call(cmd)


def ranks_arm(args) -> None:
    """Stand-in for the GPU arm that exercises only the rank plumbing on CPU
    (gloo): every rank joins, the world size and the max over ranks are
    formed exactly as the GPU arm forms them, and rank 0 prints one line."""
    import datetime
    import torch.distributed as dist
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    pg = None
    if world > 1:
        dist.init_process_group("gloo", timeout=datetime.timedelta(seconds=60))
        pg = dist
    t = max_over_ranks(pg, 1.0 + rank, "cpu")
    ranks = [None] * world
    if pg is not None:
        dist.all_gather_object(ranks, rank)
        dist.destroy_process_group()
    else:
        ranks = [0]
    if rank == 0:
        print(json.dumps({"impl": "ranks", "n_gpus": world, "ranks": ranks, "t_max": t}), flush=True)


class Timer:
    """CUDA events on the launching stream."""

    def __init__(self, torch, stream):
        self.torch, self.stream = torch, stream
        self.a = torch.cuda.Event(enable_timing=True)
        self.b = torch.cuda.Event(enable_timing=True)

    def start(self):
        self.a.record(self.stream)

    def stop(self) -> float:
        self.b.record(self.stream)
        self.b.synchronize()
        return self.a.elapsed_time(self.b) * 1e-3


class Runner:
    """One workload resident in HBM with its plan and outputs; `step(k)` is one
    lca_decode over the whole batch (copies of the inputs rotated so that no
    step starts with its cache warm in L2)."""

    def __init__(self, torch, kvc, wl, stream):
        self.torch, self.kvc, self.wl, self.stream = torch, kvc, wl, stream
        self.x = workloads.generate(wl, threads=16)
        self.cache_bytes = self.x.c_kv.nbytes + self.x.k_r.nbytes
        self.copies = 1 if self.cache_bytes >= 4 * L2_BYTES else 2
        self.dev = [(to_device(self.x.q_c, torch), to_device(self.x.q_r, torch),
                     to_device(self.x.c_kv, torch), to_device(self.x.k_r, torch))
                    for _ in range(self.copies)]
        self.plan = kvc.Plan(wl.B, wl.H, wl.d_c, wl.d_r, wl.dtype, wl.L)
        self.nG = wl.n_groups
        self.out = torch.empty(wl.B, wl.H, wl.d_c, dtype=torch.float32, device="cuda")
        self.anc = torch.empty(wl.B, wl.H, max(self.nG, 1), dtype=torch.int32, device="cuda")

    def kernel(self) -> str:
        return self.plan.kernel(self.wl.L, self.wl.g, self.wl.w)

    def step(self, k: int, g=None, w=None) -> None:
        wl = self.wl
        g = wl.g if g is None else g
        w = wl.w if w is None else w
        nG = (wl.L - w) // g if wl.L > w else 0
        q_c, q_r, c_kv, k_r = self.dev[k % self.copies]
        anc = self.anc if nG > 0 else None
        if anc is not None and anc.shape[-1] < nG:
            self.anc = self.torch.empty(wl.B, wl.H, nG, dtype=self.torch.int32, device="cuda")
            anc = self.anc
        self.plan.decode(q_c, q_r, c_kv, k_r, wl.L, g, w, self.out, anc, self.stream)

    def dense(self, k: int) -> None:
        q_c, q_r, c_kv, k_r = self.dev[k % self.copies]
        self.plan.dense(q_c, q_r, c_kv, k_r, self.wl.L, self.out, self.stream)

    def check_device(self) -> None:
        """Raise, naming the workload and the wait site, if a kernel reported an error."""
        st = self.plan.device_error()
        if st != self.kvc.LCA_OK:
            raise RuntimeError(f"device error {st} at site {self.plan.device_error_site():#x} on "
                               f"{workload_desc(self.wl)}")

    def main_kernel_time(self, steps: int, g=None, w=None) -> list[float]:
        """Per-step duration of the main kernel alone: an event recorded on the
        launching stream before the step and, by the library, right after the
        main-kernel launch (before the split combine)."""
        torch = self.torch
        ev_s = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
        ev_m = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
        for e in ev_m:
            e.record(self.stream)
        torch.cuda.synchronize()
        for k in range(steps):
            ev_s[k].record(self.stream)
            self.plan.set_timing_event(ev_m[k])
            self.step(k, g, w)
        torch.cuda.synchronize()
        self.plan.set_timing_event(None)
        self.check_device()
        return [ev_s[k].elapsed_time(ev_m[k]) * 1e-3 for k in range(steps)]

    def free(self) -> None:
        self.plan.close()
        del self.dev, self.out, self.anc
        self.torch.cuda.empty_cache()


def timed_blocks(torch, runner, K: int, blocks: int, sync, fn=None) -> list[float]:
    """`blocks` timed regions of exactly K back-to-back steps, each bracketed by
    barrier + synchronize; returns each region's seconds (max over ranks is
    taken by `sync`'s caller)."""
    fn = fn or runner.step
    times = []
    for _ in range(blocks):
        sync()
        t = Timer(torch, runner.stream)
        t.start()
        for k in range(K):
            fn(k)
        times.append(t.stop())
        sync()
    return times


def stored_leg(torch, kvc, r, K: int, peaks: dict, t_lca: float, t_mla: float) -> dict:
    """The stored, head-shared condensed cache on the same inputs: build it once
    from the full cache (condense every group with this step's query, copy the
    window), then decode over the n_G + |W| stored rows.  Enough copies of the
    stored cache rotate that every step reads it from HBM."""
    wl = r.wl
    R = kvc.stored_rows(wl.L, wl.g, wl.w)
    nG = wl.n_groups
    tdt = torch.bfloat16 if wl.dtype == "bf16" else torch.float32
    row_bytes = (wl.d_c + wl.d_r) * wl.elem_bytes
    store_bytes = wl.B * R * row_bytes
    copies = int(min(20, max(1, math.ceil(4 * L2_BYTES / store_bytes))))
    q_c, q_r, c_kv, k_r = r.dev[0]
    stores = []
    anc = torch.empty(wl.B, max(nG, 1), dtype=torch.int32, device="cuda")
    for _ in range(copies):
        c_st = torch.empty(wl.B, R, wl.d_c, dtype=tdt, device="cuda")
        k_st = torch.empty(wl.B, R, wl.d_r, dtype=tdt, device="cuda")
        r.plan.build_stored(q_c, q_r, c_kv, k_r, wl.L, wl.g, wl.w, c_st, k_st, anc if nG else None)
        stores.append((c_st, k_st))
    torch.cuda.synchronize()
    tb = Timer(torch, r.stream)
    builds = []
    for k in range(3):                      # the build reads the whole cache once (a prefill cost)
        tb.start()
        r.plan.build_stored(*r.dev[k % r.copies], wl.L, wl.g, wl.w, stores[0][0], stores[0][1],
                            anc if nG else None)
        builds.append(tb.stop())
    out = torch.empty(wl.B, wl.H, wl.d_c, dtype=torch.float32, device="cuda")

    def step(k: int) -> None:
        c_st, k_st = stores[k % copies]
        r.plan.decode_stored(q_c, q_r, c_st, k_st, R, nG, 0.0, out, r.stream)

    for k in range(3):
        step(k)
    torch.cuda.synchronize()
    blocks = []
    t = Timer(torch, r.stream)
    for _ in range(5):
        t.start()
        for k in range(K):
            step(k)
        blocks.append(t.stop() / K)
    r.check_device()
    ts = statistics.median(blocks)
    alg = store_bytes + wl.B * wl.H * (wl.d_c + wl.d_r) * wl.elem_bytes + wl.B * wl.H * wl.d_c * 4
    del stores
    torch.cuda.empty_cache()
    return {"ms_per_step": ts * 1e3, "context_tokens_per_s": wl.B * wl.L / ts, "unit": UNIT,
            "stored_rows_per_seq": R, "rows_ratio_vs_full": R / wl.L,
            "bytes_per_step": alg, "hbm_frac": alg / ts / 1e9 / peaks["hbm_gbs"],
            "speedup_vs_lca_decode": t_lca / ts, "speedup_vs_mla_decode": t_mla / ts,
            "build_ms": statistics.median(builds) * 1e3, "copies_rotated": copies,
            "kernel": r.plan.kernel(R, 1, 0),
            "note": "lca_build_stored once (head-mean condensation with this step's query), then "
                    "lca_decode_stored over [stored || window] per step, no bias"}


def paged_leg(torch, kvc, r, K: int, peaks: dict, t_lca: float) -> dict:
    """The same batch through lca_decode_paged: its cache cut into 64-token
    pages placed in a seeded random order in one pool, first at the batch's
    own length (the cost of the block-table path against lca_decode), then
    with lengths drawn uniformly from [L/4, L] per sequence (variable-length
    batch; bytes counted per sequence)."""
    wl = r.wl
    ps = 64
    pages = -(-wl.L // ps)
    q_c, q_r, c_kv, k_r = r.dev[0]
    gen = torch.Generator().manual_seed(1234)
    perm = torch.randperm(wl.B * pages, generator=gen).cuda()
    table = perm.view(wl.B, pages).to(torch.int32).contiguous()
    tdt = c_kv.dtype

    def pool_of(t):
        d = t.shape[-1]
        src = torch.zeros(wl.B, pages * ps, d, dtype=tdt, device="cuda")
        src[:, :wl.L] = t
        pool = torch.empty(wl.B * pages, ps, d, dtype=tdt, device="cuda")
        pool.index_copy_(0, perm, src.view(wl.B * pages, ps, d))
        return pool.view(-1, d)

    c_pool, k_pool = pool_of(c_kv), pool_of(k_r)
    nG_max = wl.n_groups
    out = torch.empty(wl.B, wl.H, wl.d_c, dtype=torch.float32, device="cuda")
    anc = torch.empty(wl.B, wl.H, max(nG_max, 1), dtype=torch.int32, device="cuda")
    full = torch.full((wl.B,), wl.L, dtype=torch.int32, device="cuda")
    lo = max(1, wl.L // 4)
    var_host = torch.randint(lo, wl.L + 1, (wl.B,), generator=gen, dtype=torch.int32)
    var = var_host.cuda()

    def run(lens, steps: int, event=None) -> float:
        t = Timer(torch, r.stream)
        t.start()
        for _ in range(steps):
            r.plan.decode_paged(q_c, q_r, c_pool, k_pool, ps, table, lens, wl.g, wl.w, out,
                                anc if nG_max > 0 else None, r.stream)
        return t.stop() / steps

    res = {}
    for name, lens, toks in (("same_lengths", full, wl.B * wl.L),
                             ("variable_lengths", var, int(var_host.sum()))):
        run(lens, 3)
        torch.cuda.synchronize()
        ts = statistics.median([run(lens, K) for _ in range(5)])
        ev_s = torch.cuda.Event(enable_timing=True)
        ev_m = torch.cuda.Event(enable_timing=True)
        ev_m.record(r.stream)          # torch creates the event at its first record
        torch.cuda.synchronize()
        mains = []
        for _ in range(5):
            ev_s.record(r.stream)
            r.plan.set_timing_event(ev_m)
            run(lens, 1)
            torch.cuda.synchronize()
            mains.append(ev_s.elapsed_time(ev_m) * 1e-3)
        r.plan.set_timing_event(None)
        r.check_device()
        alg = toks * (wl.d_c + wl.d_r) * wl.elem_bytes + wl.B * wl.H * (wl.d_c + wl.d_r) * wl.elem_bytes + \
            wl.B * wl.H * wl.d_c * 4
        tm = statistics.mean(mains)
        res[name] = {"ms_per_step": ts * 1e3, "main_kernel_ms": tm * 1e3,
                     "context_tokens_per_s": toks / ts, "context_tokens_per_step": toks,
                     "hbm_frac_whole_step": alg / ts / 1e9 / peaks["hbm_gbs"],
                     "hbm_frac_main_kernel": alg / tm / 1e9 / peaks["hbm_gbs"]}
    res["same_lengths"]["time_vs_lca_decode"] = res["same_lengths"]["ms_per_step"] / (t_lca * 1e3)
    res.update({"page_size": ps, "pages_per_seq": pages, "kernel": r.kernel(), "unit": UNIT,
                "variable_lengths_range": [lo, wl.L],
                "note": "lca_decode_paged over a pool of 64-token pages in random order; the main-kernel "
                        "time includes the metadata kernel before it"})
    del c_pool, k_pool
    torch.cuda.empty_cache()
    return res


def prefill_leg(torch, kvc, r, K: int, n: int = 64) -> dict:
    """LCA prefill of the last chunk of one sequence of the batch: n queries at
    positions L - n .. L - 1, each condensing its own causal prefix
    (lca_prefill_paged over the sequence's cache as 64-token pages), beside the
    same chunk with nothing condensed (w = L: dense causal attention over each
    prefix, the same kernels).  Queries are seeded N(0, 1) scaled like the
    workload's."""
    wl = r.wl
    ps = 64
    pages = -(-wl.L // ps)
    q_c0, q_r0, c_kv, k_r = r.dev[0]
    c_pool = c_kv[0].contiguous()                 # sequence 0's rows, pages in order
    k_pool = k_r[0].contiguous()
    row = torch.arange(pages, dtype=torch.int32, device="cuda")
    gen = torch.Generator(device="cuda").manual_seed(77)
    tdt = q_c0.dtype
    q_c = (torch.randn(n, wl.H, wl.d_c, generator=gen, device="cuda") * wl.q_scale).to(tdt)
    q_r = (torch.randn(n, wl.H, wl.d_r, generator=gen, device="cuda") * wl.q_scale).to(tdt)
    plan = kvc.Plan(n, wl.H, wl.d_c, wl.d_r, wl.dtype, wl.L)
    out = torch.empty(n, wl.H, wl.d_c, dtype=torch.float32, device="cuda")
    anc = torch.empty(n, wl.H, max(wl.n_groups, 1), dtype=torch.int32, device="cuda")
    pos0 = wl.L - n
    tokens = n * pos0 + n * (n + 1) // 2          # sum of the queries' prefix lengths
    res = {"queries": n, "pos0": pos0, "context_tokens_per_chunk": tokens, "page_size": ps,
           "kernel": plan.kernel(wl.L, wl.g, wl.w), "unit": UNIT}
    for name, w in (("lca", wl.w), ("dense", wl.L)):
        def run(steps: int) -> float:
            t = Timer(torch, r.stream)
            t.start()
            for _ in range(steps):
                plan.prefill_paged(q_c, q_r, c_pool, k_pool, ps, row, pos0, wl.g, w, out,
                                   anc if w < wl.L else None, r.stream)
            return t.stop() / steps
        run(2)
        torch.cuda.synchronize()
        ts = statistics.median([run(K) for _ in range(3)])
        st = plan.device_error()
        if st != kvc.LCA_OK:
            raise RuntimeError(f"device error {st} at site {plan.device_error_site():#x} in the prefill leg")
        res[name] = {"ms_per_chunk": ts * 1e3, "queries_per_s": n / ts, "context_tokens_per_s": tokens / ts}
    res["note"] = ("each query is the decode of its own causal prefix (lengths pos0 + 1 .. L), every query "
                   "reading the sequence's pages; the sequence's cache (" +
                   f"{wl.L * (wl.d_c + wl.d_r) * wl.elem_bytes / 1e6:.0f} MB) is read from L2 after the first query")
    plan.close()
    return res


def gqa_leg(torch, kvc, stream, K: int, peaks: dict) -> dict:
    """GQA LCA decode (lca_decode_gqa) on a Distill-Qwen-7B-shaped batch: B=8,
    28 query heads over 4 KV heads of 128 (keys and values), L=32768, g=16,
    w=1024, bf16 caches N(0, 1) and queries N(0, 1)/sqrt(128) drawn on the device
    (seeded); beside it the same kernels with nothing condensed (w = L)."""
    B, H, H_kv, d, L, g, w = 8, 28, 4, 128, 32768, 16, 1024
    gen = torch.Generator(device="cuda").manual_seed(4242)
    k = torch.randn(B, L, H_kv, d, generator=gen, device="cuda").to(torch.bfloat16)
    v = torch.randn(B, L, H_kv, d, generator=gen, device="cuda").to(torch.bfloat16)
    q = (torch.randn(B, H, d, generator=gen, device="cuda") / math.sqrt(d)).to(torch.bfloat16)
    plan = kvc.Plan(B, H, d, d, "bf16", L)
    nG = kvc.num_groups(L, g, w)
    out = torch.empty(B, H, d, dtype=torch.float32, device="cuda")
    anc = torch.empty(B, H, nG, dtype=torch.int32, device="cuda")
    alg = B * L * H_kv * 2 * d * 2 + B * H * d * 2 + B * H * d * 4
    res = {"workload": f"GQA (Distill-Qwen-7B-shaped): B={B} H={H} H_kv={H_kv} d_k=d_v={d} L={L} g={g} w={w} "
                       "bf16, q*0.0884", "bytes_per_step": alg, "unit": UNIT, "kernel": "lca_gqa_kernel (CUDA cores)"}
    for name, ww in (("lca", w), ("dense", L)):
        def step() -> None:
            plan.decode_gqa(q, k, v, L, H_kv, g, ww, out, anc if ww < L else None, stream)
        for _ in range(3):
            step()
        torch.cuda.synchronize()
        t = Timer(torch, stream)
        blocks = []
        for _ in range(5):
            t.start()
            for _ in range(K):
                step()
            blocks.append(t.stop() / K)
        ev_s = torch.cuda.Event(enable_timing=True)
        ev_m = torch.cuda.Event(enable_timing=True)
        ev_m.record(stream)
        torch.cuda.synchronize()
        mains = []
        for _ in range(5):
            ev_s.record(stream)
            plan.set_timing_event(ev_m)
            step()
            torch.cuda.synchronize()
            mains.append(ev_s.elapsed_time(ev_m) * 1e-3)
        plan.set_timing_event(None)
        st = plan.device_error()
        if st != kvc.LCA_OK:
            raise RuntimeError(f"device error {st} in the GQA leg")
        ts, tm = statistics.median(blocks), statistics.mean(mains)
        res[name] = {"ms_per_step": ts * 1e3, "main_kernel_ms": tm * 1e3, "context_tokens_per_s": B * L / ts,
                     "hbm_frac_whole_step": alg / ts / 1e9 / peaks["hbm_gbs"],
                     "hbm_frac_main_kernel": alg / tm / 1e9 / peaks["hbm_gbs"]}
    plan.close()
    del k, v, q
    torch.cuda.empty_cache()
    return res


def workload_fractions(wl, t_step: float, t_main: float, peaks: dict) -> dict:
    alg = algorithmic_bytes(wl)
    flops = algorithmic_flops(wl)
    return {"ms_per_step": t_step * 1e3, "main_kernel_ms": t_main * 1e3,
            "context_tokens_per_s": wl.B * wl.L / t_step,
            "hbm_frac_whole_step": alg / t_step / 1e9 / peaks["hbm_gbs"],
            "hbm_frac_main_kernel": alg / t_main / 1e9 / peaks["hbm_gbs"],
            "tensor_frac_main_kernel": flops / t_main / 1e12 / peaks["bf16_tflops"]}


def per_config(torch, kvc, stream, names: list[str], peaks: dict, steps: int) -> dict:
    """Every other benchmark workload in the same process: whole-step and
    main-kernel fractions (every (g, w) point of the sweep)."""
    res = {}
    for name in names:
        wl = workloads.WORKLOADS[name]
        r = Runner(torch, kvc, wl, stream)
        points = list(wl.sweep) if wl.sweep else [(wl.g, wl.w)]
        for (g, w) in points:
            wlp = wl.with_(g=g, w=w)
            key = name if not wl.sweep else f"{name} g={g} w={w}"
            for k in range(3):
                r.step(k, g, w)
            torch.cuda.synchronize()
            t = Timer(torch, stream)
            blocks = []
            for _ in range(3):
                t.start()
                for k in range(steps):
                    r.step(k, g, w)
                blocks.append(t.stop() / steps)
            main = r.main_kernel_time(steps, g, w)
            d = workload_fractions(wlp, statistics.median(blocks), statistics.mean(main), peaks)
            d.update({"workload": workload_desc(wlp), "kernel": r.kernel() if not wl.sweep else
                      r.plan.kernel(wl.L, g, w), "steps": steps, "blocks": 3})
            res[key] = d
        r.free()
    return res


def our_arm(args) -> None:
    import torch
    import kv_compression_b200 as kvc

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dist = None
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))

    wl = rank_workload(with_point(workloads.WORKLOADS[args.workload], args), rank)
    stream = torch.cuda.current_stream()
    r = Runner(torch, kvc, wl, stream)
    x = r.x
    kernel = r.kernel()
    nG = wl.n_groups

    props = torch.cuda.get_device_properties(local)
    uuid = ("GPU-" + str(props.uuid)) if getattr(props, "uuid", None) else None
    sampler = ClockSampler(uuid)
    tw = Timer(torch, stream)
    tw.start()
    for k in range(args.warmup):
        r.step(k)
    t_warm = tw.stop() / max(args.warmup, 1)
    r.check_device()

    K = args.steps

    def barrier_sync() -> None:
        torch.cuda.synchronize()
        if dist is not None:
            dist.barrier()
        torch.cuda.synchronize()

    def rank_max(v: float) -> float:
        return max_over_ranks(dist, v, "cuda")

    # Timed regions: blocks of K back-to-back steps exactly as a caller issues them
    # (no event between the main and the combine kernel, so the combine's
    # programmatic dependent launch overlaps the main kernel's tail).  Enough
    # blocks for about half a second of timed work; the median block is reported.
    blocks = args.blocks or int(min(200, max(5, math.ceil(0.5 / max(K * t_warm, 1e-6)))))
    if dist is not None:
        blocks = int(rank_max(float(blocks)))      # every rank runs the same collective steps
    nvml = NvmlSampler(uuid)
    nvml.start()
    block_s = timed_blocks(torch, r, K, blocks, barrier_sync)
    clocks = nvml.stop()
    block_s = [rank_max(t) for t in block_s]
    t_total = statistics.median(block_s)
    r.check_device()

    # The main kernel's own duration (its roofline): events on the launching stream
    # around each main-kernel launch, over a second pass of K steps.
    barrier_sync()
    main_s = r.main_kernel_time(K)
    t_main = rank_max(statistics.mean(main_s))
    clocks["nvidia_smi_whole_run"] = sampler.stop()

    # Dense MLA (mla_decode) on the same inputs: the same bytes, nothing condensed.
    kd = max(1, min(K, 200))
    barrier_sync()
    dense_s = [rank_max(t) for t in timed_blocks(torch, r, kd, 3, barrier_sync, fn=r.dense)]
    t_dense = statistics.median(dense_s)
    r.check_device()

    stored = None
    if not args.no_stored:
        barrier_sync()
        stored = stored_leg(torch, kvc, r, max(5, min(K, 200)), measured_peaks()[0], t_total / K,
                            t_dense / kd)

    paged = None
    if not args.no_paged and rank == 0 and world == 1:
        barrier_sync()
        paged = paged_leg(torch, kvc, r, max(5, min(K, 50)), measured_peaks()[0], t_total / K)
    prefill = None
    if not args.no_prefill and rank == 0 and world == 1:
        barrier_sync()
        prefill = prefill_leg(torch, kvc, r, max(3, min(K, 20)))

    tokens_per_step = world * wl.B * wl.L
    value = whole_job_rate(world, wl, K, t_total * 1.0)
    peaks, peak_kind = measured_peaks()
    alg = algorithmic_bytes(wl)
    achieved = alg / t_main / 1e9
    flops = algorithmic_flops(wl)
    traffic = profiled_traffic(wl)

    e2e = None
    if not args.no_e2e:
        def pinned(a):
            t = torch.from_numpy(a.view(np.int16) if a.dtype == np.uint16 else a)
            return t.pin_memory()
        hq_c, hq_r, hc, hk = pinned(x.q_c), pinned(x.q_r), pinned(x.c_kv), pinned(x.k_r)
        h_out = torch.empty(wl.B, wl.H, wl.d_c, dtype=torch.float32).pin_memory()
        h_anc = torch.empty(wl.B, wl.H, max(nG, 1), dtype=torch.int32).pin_memory()
        ke = max(1, min(K, 10))
        r.plan.decode_host(hq_c, hq_r, hc, hk, wl.L, wl.g, wl.w, h_out, h_anc if nG > 0 else None,
                           stream)
        barrier_sync()
        te_t = Timer(torch, stream)
        te_t.start()
        for _ in range(ke):
            r.plan.decode_host(hq_c, hq_r, hc, hk, wl.L, wl.g, wl.w, h_out,
                               h_anc if nG > 0 else None, stream)
        te = rank_max(te_t.stop())
        h2d = hq_c.numel() * hq_c.element_size() + hq_r.numel() * hq_r.element_size() + \
            hc.numel() * hc.element_size() + hk.numel() * hk.element_size()
        d2h = h_out.numel() * 4 + (wl.B * wl.H * nG * 4)
        e2e = {"value": tokens_per_step * ke / te, "unit": UNIT, "h2d_bytes_per_step": int(h2d),
               "d2h_bytes_per_step": int(d2h), "steps": ke,
               "path": "lca_decode_host (pinned host buffers; copies inside the timed region)"}
        del hq_c, hq_r, hc, hk

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        from oracle import oracle
        nthreads = os.cpu_count() or 1
        # rows 0 and B-1, then more rows until about 10 s of oracle work
        first = oracle.lca(x.q_c, x.q_r, x.c_kv, x.k_r, g=wl.g, w=wl.w, rows=[0], nthreads=nthreads)
        n_rows = int(max(2, min(wl.B, 10.0 / max(first.seconds, 1e-3))))
        rows = sorted({0, wl.B - 1} | set(range(1, n_rows - 1)))
        res = oracle.lca(x.q_c, x.q_r, x.c_kv, x.k_r, g=wl.g, w=wl.w, rows=rows, nthreads=nthreads)
        cpu = {"value": len(rows) * wl.L / res.seconds, "unit": UNIT, "cores": nthreads,
               "kind": "oracle",
               "sample": f"{len(rows)} sequences of the batch (rows {rows[0]}..{rows[-1]}; all "
                         f"{wl.H} heads, L={wl.L}), oracle formulation A, {res.seconds:.1f} s"}

    head_kernel = kernel
    r.free()
    del r, x
    pc = None
    if rank == 0 and world == 1 and not args.no_per_config:
        others = [n for n in ("v2lite", "v2", "needle", "sweep", "tiny_f32") if n != args.workload]
        pc = per_config(torch, kvc, stream, others, peaks, max(5, min(K, 50)))
    gqa = None
    if rank == 0 and world == 1 and not args.no_gqa:
        gqa = gqa_leg(torch, kvc, stream, max(5, min(K, 50)), peaks)

    if dist is not None:
        dist.destroy_process_group()
    if rank != 0:
        return
    tc_peak_s = peaks.get("bf16_tflops_sustained", peaks["bf16_tflops"])
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": K,
        "warmup": args.warmup, "ms_per_step": t_total / K * 1e3, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16" if wl.dtype == "bf16" else "f32",
        "data": "synthetic (seeded, workloads/)",
        "config": {"workload": workload_desc(wl), "kernel": head_kernel, "parallelism": f"replicas x{world}",
                   "l2": (f"inputs {r_cache_mb(wl):.0f} MB per step > 126 MB L2; "
                          f"{1 if r_cache_mb(wl) * 1e6 >= 4 * L2_BYTES else 2} copies rotated, no flush"),
                   "timed_blocks": blocks, "block_ms": [t * 1e3 for t in block_s],
                   "hbm_gbs_whole_step": alg / (t_total / K) / 1e9,
                   "hbm_frac_whole_step": alg / (t_total / K) / 1e9 / peaks["hbm_gbs"]},
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                     "frac": achieved / peaks["hbm_gbs"], "traffic": traffic,
                     "kernel": MAIN_KERNEL_NAMES.get(head_kernel, head_kernel),
                     "algorithmic_bytes_per_launch": alg, "launch_ms": t_main * 1e3,
                     "launch_ms_min": min(main_s) * 1e3, "launch_ms_max": max(main_s) * 1e3,
                     "timing": "CUDA events on the launching stream around each main-kernel launch, "
                               "mean over a second pass of K steps",
                     "peak_kind": f"{peak_kind} hbm_gbs (copy)",
                     "flops_per_launch": flops, "achieved_tflops": flops / t_main / 1e12,
                     "tensor_frac": flops / t_main / 1e12 / peaks["bf16_tflops"],
                     "tensor_frac_sustained": flops / t_main / 1e12 / tc_peak_s,
                     "tensor_peak_kind": f"{peak_kind} bf16_tflops (cuBLAS burst; sustained beside it)"},
        "mla_decode": {"value": whole_job_rate(world, wl, kd, t_dense), "unit": UNIT,
                       "ms_per_step": t_dense / kd * 1e3, "steps": kd,
                       "hbm_frac": alg / (t_dense / kd) / 1e9 / peaks["hbm_gbs"],
                       "note": "dense MLA decode over the same cache (same bytes), same kernels with n_G = 0"},
        "stored_cache": stored,
        "paged": paged,
        "prefill": prefill,
        "gqa": gqa,
        "per_config": pc,
        "cpu_baseline": cpu,
        "e2e": e2e,
        "gpu_launches": 2 * K,
        "gpu_launches_note": "per timed block of K steps: main + combine per step; the instrumented, "
                             "dense, e2e and per-config passes are outside the timed blocks",
        "clocks": clocks,
    }
    print(json.dumps(line), flush=True)


def r_cache_mb(wl: workloads.Workload) -> float:
    return wl.B * wl.L * (wl.d_c + wl.d_r) * wl.elem_bytes / 1e6


def main() -> None:
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--blocks", type=int, default=0,
                    help="timed blocks of --steps steps (0: enough for about 0.5 s)")
    ap.add_argument("--impl", choices=["ours", "reference", "ranks"], default="ours")
    ap.add_argument("--workload", default="v2", choices=sorted(workloads.WORKLOADS))
    ap.add_argument("--g", type=int, default=None, help="group size (default: the workload's)")
    ap.add_argument("--w", type=int, default=None, help="window (default: the workload's)")
    ap.add_argument("--batch", type=int, default=None,
                    help="sequences per step (default: the workload's; smaller for profiling captures)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-per-config", action="store_true")
    ap.add_argument("--no-stored", action="store_true")
    ap.add_argument("--no-paged", action="store_true")
    ap.add_argument("--no-prefill", action="store_true")
    ap.add_argument("--no-gqa", action="store_true")
    args = ap.parse_args()
    rc = spawn_ranks(args)
    if rc is not None:
        sys.exit(rc)
    if args.impl == "reference":
        reference_arm(args)
    elif args.impl == "ranks":
        ranks_arm(args)
    else:
        our_arm(args)


if __name__ == "__main__":
    main()
