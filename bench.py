"""Benchmark: anisotropic-AH search throughput (queries/s at top-10) on B200.

One step = one batched search of the whole hot path (centroid scores -> top-L
leaves -> lookup tables -> 4-bit code scan -> top-R -> exact reorder -> top-k)
over one batch of synthetic queries, through the C ABI.  Default workload: the
largest fixed single-GPU configuration, OpenAI-embedding-shaped IVF-AH
(n = 2,000,000, d = 1,536, dims_per_block = 4, 2,000 leaves, 40 searched,
10,000 queries, k = 10, reorder 300 against a bfloat16 copy); ``--workload``
selects another (tiny, glove, bigann, openai; ``--sweep`` for the sweep).

Single GPU:  python bench.py [--steps K --warmup W]
N GPUs:      python -m torch.distributed.run --nproc-per-node N bench.py --gpus N
             (one process per GPU; every rank holds a replica of the index and
             searches its own query batch; no data-path collective -> weak
             scaling; timing is the max over ranks)
Reference:   python bench.py --impl reference  (the CPU oracle, rank 0 only)

Prints one JSON line (rank 0).
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

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "AH search queries/sec at top-10 (1 B200); code-scan GB/s vs HBM/smem roofline"
L2_BYTES = 126 * 1024 * 1024
SM_COUNT = 148
SMEM_BYTES_PER_CLK = 128          # per SM: 32 banks x 4 B
SM_MAX_MHZ_FALLBACK = 1965.0
# DRAM bytes (read + write) that one ncu capture counted for the scan launches of
# one step (all scan phases), per (workload, table mode) at the workload's default
# batch; None where no capture of the current scan kernel exists.
SCAN_TRAFFIC_BYTES = {("openai", 0): 8.43e9}   # the three phase launches of one step, one ncu pass


def parse():
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=400)
    p.add_argument("--warmup", type=int, default=10)
    p.add_argument("--impl", choices=["ours", "reference"], default="ours")
    p.add_argument("--workload", default=None,
                   help="openai (the default), glove, bigann, tiny, sweep; --encode and --kmeans default to glove")
    p.add_argument("--lut-mode", type=int, default=0, choices=[0, 1])
    p.add_argument("--nq", type=int, default=None)
    p.add_argument("--leaves", type=int, default=None, help="num_leaves_to_search")
    p.add_argument("--n", type=int, default=None,
                   help="reduced point count (profiling captures): means and training sample scale along")
    p.add_argument("--num-leaves", type=int, default=None, help="partition size with --n")
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--cpu-seconds", type=float, default=12.0)
    p.add_argument("--e2e-steps", type=int, default=100)
    p.add_argument("--sweep", action="store_true",
                   help="sweep workload: one JSON line per (batch, leaves) point instead of the single line")
    p.add_argument("--encode", action="store_true",
                   help="index build: time the anisotropic code assignment over the workload's points")
    p.add_argument("--passes", type=int, default=10)
    p.add_argument("--leaf-shards", action="store_true",
                   help="leaf-partitioned search: rank r scans the leaves c with c %% N == r for the whole batch; "
                        "candidates are gathered and merged exactly (strong scaling)")
    p.add_argument("--kmeans", action="store_true",
                   help="index build: time one k-means iteration (assignment + update) over the workload's points")
    args = p.parse_args()
    if args.workload is None:
        args.workload = "glove" if (args.encode or args.kmeans) else "openai"
    if (args.encode or args.kmeans) and "--steps" not in sys.argv:
        args.steps = 20                                  # the index-build lines time whole passes over n points
    return args


def cpu_model() -> str:
    """The host CPU's model name (for the oracle baseline's record)."""
    try:
        with open("/proc/cpuinfo") as f:
            for ln in f:
                if ln.startswith("model name"):
                    return ln.split(":", 1)[1].strip()
    except OSError:
        pass
    return "unknown"


def dist_env():
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return rank, world, local


def init_ranks(world, dev):
    """Process group for N > 1 ranks (NCCL on GPUs, gloo on CPU), with a short
    timeout so ranks waiting for a missing peer end with an error."""
    import torch.distributed as dist
    from datetime import timedelta
    if world <= 1:
        return False
    if dev.type == "cuda":
        dist.init_process_group("nccl", timeout=timedelta(seconds=120), device_id=dev)
    else:
        dist.init_process_group("gloo", timeout=timedelta(seconds=120))
    return True


def max_over_ranks(x, dev, world):
    """The largest of every rank's x (device time: the slowest rank sets the job's time)."""
    if world <= 1:
        return float(x)
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(x)], device=dev, dtype=torch.float64)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(world, nq_per_rank, total_ms, steps):
    """Whole-job queries/s (every rank searches its own batch each step) and ms per step."""
    ms_per_step = total_ms / steps
    return world * nq_per_rank / (ms_per_step * 1e-3), ms_per_step


def rank_workload(w, rank):
    """Rank r searches its own query batch (query seed + 1000 r) over the same index."""
    return w.scaled(query_seed=w.query_seed + 1000 * rank)


class ClockSampler:
    """SM clocks and clock-event (throttle) reasons sampled during the timed
    region, read-only.  NVML is polled in-process every ``period_s`` (1 ms by
    default, so a timed region of a few milliseconds still gets samples);
    without NVML it falls back to ``nvidia-smi -lms 100``."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
    REASON_BITS = {"hw_slowdown": 0x8, "hw_thermal_slowdown": 0x40, "sw_thermal_slowdown": 0x20,
                   "sw_power_cap": 0x4, "hw_power_brake_slowdown": 0x80}

    def __init__(self, device, period_s: float = 0.001):
        self.device = device
        self.period = period_s
        self.proc = None
        self.lines = []
        self.samples = []            # (sm MHz, max MHz, reason bits)
        self.source = None
        self._stop = threading.Event()
        self._t = None
        self._nvml = None
        self._h = None

    def _nvml_handle(self):
        import pynvml
        import torch
        pynvml.nvmlInit()
        self._nvml = pynvml
        idx = self.device.index if hasattr(self.device, "index") else int(self.device)
        p = torch.cuda.get_device_properties(idx or 0)
        bus = f"{p.pci_domain_id:08x}:{p.pci_bus_id:02x}:{p.pci_device_id:02x}.0"
        return pynvml.nvmlDeviceGetHandleByPciBusId(bus)

    def _poll(self):
        nv, h = self._nvml, self._h
        mx = nv.nvmlDeviceGetMaxClockInfo(h, nv.NVML_CLOCK_SM)
        while not self._stop.is_set():
            try:
                sm = nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM)
                rs = nv.nvmlDeviceGetCurrentClocksEventReasons(h)
                self.samples.append((float(sm), float(mx), int(rs)))
            except Exception:
                pass
            self._stop.wait(self.period)

    def __enter__(self):
        try:
            self._h = self._nvml_handle()
            self.source = "nvml"
            self._t = threading.Thread(target=self._poll, daemon=True)
            self._t.start()
            return self
        except Exception:
            self._nvml = None
        try:
            idx = self.device.index if hasattr(self.device, "index") else int(self.device)
            self.proc = subprocess.Popen(["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                                          "-i", str(idx or 0), "-lms", "100"],
                                         stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.source = "nvidia-smi"
            self._t = threading.Thread(target=self._read, daemon=True)
            self._t.start()
        except (FileNotFoundError, OSError):
            self.proc = None
        return self

    def _read(self):
        for ln in self.proc.stdout:
            self.lines.append(ln.strip())

    def __exit__(self, *a):
        self._stop.set()
        if self._nvml is not None and self._t is not None:
            self._t.join(timeout=5)
            try:
                self._nvml.nvmlShutdown()
            except Exception:
                pass
        if self.proc:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self):
        sm, mx, reasons = [], [], set()
        for s, m, bits in self.samples:
            sm.append(s)
            mx.append(m)
            for nm, bit in self.REASON_BITS.items():
                if bits & bit:
                    reasons.add(nm)
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            f = [x.strip() for x in ln.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                mx.append(float(f[2]))
            except ValueError:
                continue
            for nm, v in zip(names, f[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(nm)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0, "source": self.source}
        return {"sm_mhz": statistics.median(sm), "sm_min_mhz": min(sm), "sm_max_mhz": max(mx),
                "reasons": sorted(reasons), "samples": len(sm), "source": self.source}


def workload_spec(args):
    from mips_ivf_centroid_b200 import datagen
    w = datagen.WORKLOADS[args.workload]
    if args.nq:
        w = w.scaled(nq=args.nq)
    if args.leaves:
        w = w.scaled(num_leaves_to_search=args.leaves)
    if args.n:
        nl = args.num_leaves or max(1, w.num_leaves * args.n // w.n)
        w = w.scaled(n=args.n, num_leaves=nl, n_means=max(1, w.n_means * args.n // w.n),
                     training_sample_size=min(w.training_sample_size, args.n))
    return w


def config_dict(w, args):
    return {"workload": f"{w.name}-shaped IVF-AH: n={w.n:,} d={w.d} dims_per_block={w.dims_per_block} "
                        f"num_leaves={w.num_leaves} num_leaves_to_search={w.num_leaves_to_search} nq={w.nq} "
                        f"k={w.k} reorder_num={w.reorder_num} ({w.reorder_dtype} reorder copy)",
            "n": w.n, "d": w.d, "dims_per_block": w.dims_per_block, "num_leaves": w.num_leaves,
            "num_leaves_to_search": w.num_leaves_to_search, "nq": w.nq, "k": w.k, "reorder_num": w.reorder_num,
            "lut_mode": "u8" if args.lut_mode else "f32", "l2_flush_between_steps": True}


def oracle_rate(orc, Q, w, lut_mode, seconds):
    """Queries/s of the oracle on this host, on consecutive query chunks until
    ``seconds`` have elapsed (a bounded sample of the workload)."""
    import oracle
    nthreads = os.cpu_count() or 1
    done, t0, i = 0, time.perf_counter(), 0
    chunk = max(8, nthreads * 2)
    while True:
        qs = Q[(i % Q.shape[0]):(i % Q.shape[0]) + chunk]
        orc.search(qs, w.k, w.num_leaves_to_search, w.reorder_num, lut_mode, nthreads=nthreads, trace=False)
        done += qs.shape[0]
        i += chunk
        el = time.perf_counter() - t0
        if el >= seconds or done >= 50 * Q.shape[0]:
            break
    return done / el, done, el, oracle.max_threads()


def run_reference(args):
    import torch
    rank, world, local = dist_env()
    if rank != 0:
        return
    import oracle
    from mips_ivf_centroid_b200 import datagen
    w = workload_spec(args)
    dev = "cuda" if torch.cuda.is_available() else "cpu"
    X = datagen.make_data(w)
    Q = datagen.make_queries(w)
    arr = datagen.build_index(w, X, dev).numpy()
    del X
    orc = oracle.OracleIndex(arr)
    nthreads = os.cpu_count() or 1
    # calibrate the per-step sample so W + K steps take about 90 s
    t0 = time.perf_counter()
    orc.search(Q[:nthreads], w.k, w.num_leaves_to_search, w.reorder_num, args.lut_mode, nthreads=nthreads, trace=False)
    per_q = (time.perf_counter() - t0) / nthreads
    S = int(max(1, min(w.nq, 90.0 / max(1, args.steps + args.warmup) / max(per_q, 1e-6))))
    times = []
    for s in range(args.warmup + args.steps):
        qs = Q[(s * S) % w.nq:][:S]
        t0 = time.perf_counter()
        orc.search(qs, w.k, w.num_leaves_to_search, w.reorder_num, args.lut_mode, nthreads=nthreads, trace=False)
        if s >= args.warmup:
            times.append((time.perf_counter() - t0, qs.shape[0]))
    tot = sum(t for t, _ in times)
    nqs = sum(n for _, n in times)
    value = nqs / tot
    line = {"metric": METRIC, "value": value, "unit": "queries/s", "n_gpus": args.gpus, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": 1e3 * tot / len(times), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64" if args.lut_mode == 0 else "u8",
            "data": f"synthetic (seeded Gaussian mixture, {w.name}-shaped)", "config": config_dict(w, args),
            "impl": "reference",
            "cpu_baseline": {"value": value, "unit": "queries/s", "cores": oracle.max_threads(), "kind": "oracle", "cpu_model": cpu_model(),
                             "sample": f"{S} of {w.nq} queries per step, {len(times)} steps"},
            "e2e": {"value": value, "unit": "queries/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def run_ours(args):
    import torch
    import torch.distributed as dist
    rank, world, local = dist_env()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    init_ranks(world, dev)

    from mips_ivf_centroid_b200 import Index, build as ahbuild, datagen
    ahbuild.build()
    w = workload_spec(args)
    wq = rank_workload(w, rank)                                    # each rank: its own batch
    X = datagen.make_data(w)
    Q = datagen.make_queries(wq)
    ix = datagen.build_index(w, X, dev)
    del X
    torch.cuda.empty_cache()            # release the index build's temporaries
    index = Index(ix)
    qg = torch.from_numpy(Q).to(dev)
    L, k, R, mode = w.num_leaves_to_search, w.k, w.reorder_num, args.lut_mode
    index.reserve(w.nq, k, L, R, mode)
    stream = torch.cuda.current_stream()
    flush = torch.empty(2 * L2_BYTES // 4, dtype=torch.float32, device=dev)

    # warm-up
    for _ in range(args.warmup):
        index.search(qg, k, L, R, mode)
    index.sync_status()
    _, _, tr = index.search(qg, k, L, R, mode, trace=True)
    scanned = int(tr["scanned"].sum().item())
    leaves = tr["leaf_ids"].cpu().numpy()
    offs = ix.leaf_offsets.cpu().numpy()
    touched = np.unique(leaves)
    unique_code_bytes = int((offs[touched + 1] - offs[touched]).sum()) * w.code_bytes
    index.sync_status()

    # timed region: K steps, L2 flushed before each (outside the step's events);
    # events mark only the scan phases inside a step, so the rest of the
    # kernel chain keeps its overlapped launches
    index.set_profiling(2)
    ev0 = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    ev1 = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    stage_ms = {}
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    with ClockSampler(local) as clk:
        t_wall = time.perf_counter()
        for s in range(args.steps):
            flush.zero_()
            ev0[s].record(stream)
            index.search(qg, k, L, R, mode)
            ev1[s].record(stream)
            # the scan phases' events of every timed step (reading them waits
            # for this step; the next step's flush and launches follow)
            stage_ms.setdefault("scan_timed", []).append(sum(
                v for kname, v in index.stage_times().items() if kname in ("scan", "scan_rest")))
        torch.cuda.synchronize()
        t_wall = time.perf_counter() - t_wall
    # per-stage breakdown (every stage marked), outside the timed region
    index.set_profiling(True)
    for s in range(min(args.steps, 50)):
        flush.zero_()
        index.search(qg, k, L, R, mode)
        for kname, v in index.stage_times().items():
            stage_ms.setdefault(kname, []).append(v)
    index.set_profiling(False)
    index.sync_status()
    step_ms = [a.elapsed_time(b) for a, b in zip(ev0, ev1)]
    dev_ms = sum(step_ms)
    launches = index.last_search_info()["launches"]
    dev_ms = max_over_ranks(dev_ms, dev, world)
    if world > 1:
        dist.barrier()
    value, ms_per_step = job_throughput(world, w.nq, dev_ms, args.steps)

    # e2e through the host entry point: pinned host queries in, host results out
    hq = torch.from_numpy(Q).pin_memory()
    hids = torch.empty((w.nq, k), dtype=torch.int32).pin_memory()
    hsc = torch.empty((w.nq, k), dtype=torch.float32).pin_memory()
    for _ in range(3):
        index.search_host(hq, k, L, R, mode, out_ids=hids, out_scores=hsc)
    e2e_times = []
    if world > 1:
        dist.barrier()
    for _ in range(args.e2e_steps):
        flush.zero_()
        torch.cuda.synchronize()
        t0 = time.perf_counter()
        index.search_host(hq, k, L, R, mode, out_ids=hids, out_scores=hsc)
        e2e_times.append(time.perf_counter() - t0)
    e2e_s = max_over_ranks(sum(e2e_times), dev, world)
    e2e_value = world * w.nq * args.e2e_steps / e2e_s

    if rank == 0:
        med = {kname: statistics.median(v) for kname, v in stage_ms.items() if kname != "scan_timed"}
        scan_ms = statistics.fmean(stage_ms["scan_timed"])       # mean scan time over every timed step
        clocks = clk.summary()
        lookups = scanned * w.blocks
        bytes_per_lookup = 4 if mode == 0 else 1
        lut_bytes = lookups * bytes_per_lookup
        mhz = SM_MAX_MHZ_FALLBACK
        peaks_path = os.path.join(ROOT, "MEASURED_PEAKS.json")
        hbm_peak = None
        if os.path.exists(peaks_path):
            pk = json.load(open(peaks_path))
            mhz = float(pk.get("sm_max_mhz", mhz))
            hbm_peak = pk.get("hbm_gbs")
        smem_peak_gbs = SM_COUNT * SMEM_BYTES_PER_CLK * mhz * 1e6 / 1e9
        achieved = lut_bytes / (scan_ms * 1e-3) / 1e9
        roofline = {"bound": "smem", "achieved": achieved, "peak": smem_peak_gbs, "unit": "GB/s",
                    "frac": achieved / smem_peak_gbs,
                    "traffic": (SCAN_TRAFFIC_BYTES.get((args.workload, mode))
                                if args.nq is None and args.leaves is None else None),
                    "kernel": "scan_kernel", "unit_bytes": f"{bytes_per_lookup} B per table lookup",
                    "lookups_per_launch": lookups,
                    "peak_source": f"derived: {SM_COUNT} SMs x {SMEM_BYTES_PER_CLK} B/clk x {mhz:.0f} MHz",
                    "scan_ms_mean": scan_ms, "scan_steps": len(stage_ms["scan_timed"])}
        if clocks.get("sm_mhz"):
            # the same fraction against the peak at the SM clock sampled during the timed steps
            at_clk = SM_COUNT * SMEM_BYTES_PER_CLK * clocks["sm_mhz"] * 1e6 / 1e9
            roofline["frac_at_sampled_clock"] = achieved / at_clk
            roofline["peak_at_sampled_clock"] = at_clk
        # the step against the sum of its stages' roofline times: centroid GEMM at
        # the SIMT fp32 FMA peak, the scan at the larger of its SMEM-lookup and
        # unique-code HBM times, the reorder gather at the HBM copy rate
        hbm = hbm_peak or 6650.0
        fp32_tflops = SM_COUNT * 128 * 2 * mhz * 1e6 / 1e12
        elt = 2 if w.reorder_dtype == "bf16" else 4
        parts = {"centroid_scores": 2.0 * w.nq * w.num_leaves * w.d / (fp32_tflops * 1e12) * 1e3,
                 "scan": max(lut_bytes / (smem_peak_gbs * 1e9), unique_code_bytes / (hbm * 1e9)) * 1e3,
                 "reorder_gather": (w.nq * w.reorder_num * w.d * elt / (hbm * 1e9) * 1e3) if w.reorder_num else 0.0}
        roof_ms = sum(parts.values())
        step_roofline = {"ms": roof_ms, "frac": roof_ms / ms_per_step, "parts_ms": parts,
                         "peaks": f"fp32 FMA {fp32_tflops:.1f} TFLOP/s derived, SMEM {smem_peak_gbs:.0f} GB/s derived, "
                                  f"HBM {hbm:.0f} GB/s " + ("measured" if hbm_peak else "fallback")}
        line = {"metric": METRIC, "value": value, "unit": "queries/s", "n_gpus": world, "steps": args.steps,
                "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True, "scaling": "weak",
                "vs_baseline": None, "dtype": "f32" if mode == 0 else "u8",
                "data": f"synthetic (seeded Gaussian mixture, {w.name}-shaped; index trained on it)",
                "config": config_dict(w, args),
                "roofline": roofline, "step_roofline": step_roofline,
                "scan": {"ms": scan_ms, "hbm_unique_code_gbs": unique_code_bytes / (scan_ms * 1e-3) / 1e9,
                         "unique_code_bytes": unique_code_bytes, "hbm_peak_gbs": hbm_peak,
                         "lookups_per_s": lookups / (scan_ms * 1e-3)},
                "stages_ms": med,
                "e2e": {"value": e2e_value, "unit": "queries/s", "h2d_bytes_per_step": int(Q.nbytes),
                        "d2h_bytes_per_step": int(w.nq * k * 8)},
                "gpu_launches": launches * args.steps,
                "clocks": clocks, "wall_s_timed": t_wall}
        if not args.no_cpu_baseline and world == 1:
            import oracle
            orc = oracle.OracleIndex(ix.numpy())
            rate, done, el, cores = oracle_rate(orc, Q, w, mode, args.cpu_seconds)
            line["cpu_baseline"] = {"value": rate, "unit": "queries/s", "cores": cores, "kind": "oracle", "cpu_model": cpu_model(),
                                    "sample": f"{done} queries of the batch in {el:.1f} s"}
        print(json.dumps(line), flush=True)
    index.close()
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


def run_sweep(args):
    """Queries/s and scan rates over the sweep grid (batch x leaves searched)."""
    import torch
    from mips_ivf_centroid_b200 import Index, build as ahbuild, datagen
    ahbuild.build()
    w = datagen.WORKLOADS["sweep"]
    dev = torch.device("cuda", 0)
    X = datagen.make_data(w)
    Q = datagen.make_queries(w)
    ix = datagen.build_index(w, X, dev)
    del X
    torch.cuda.empty_cache()
    index = Index(ix)
    offs = ix.leaf_offsets.cpu().numpy()
    flush = torch.empty(2 * L2_BYTES // 4, dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream()
    for L in datagen.SWEEP_LEAVES:
        for nq in datagen.SWEEP_BATCHES:
            qg = torch.from_numpy(Q[:nq]).to(dev)
            index.reserve(nq, w.k, L, w.reorder_num, args.lut_mode)
            for _ in range(3):
                index.search(qg, w.k, L, w.reorder_num, args.lut_mode)
            _, _, tr = index.search(qg, w.k, L, w.reorder_num, args.lut_mode, trace=True)
            scanned = int(tr["scanned"].sum().item())
            touched = np.unique(tr["leaf_ids"].cpu().numpy())
            unique_bytes = int((offs[touched + 1] - offs[touched]).sum()) * w.code_bytes
            index.sync_status()
            # about 1 s of timed work per point, at least 5 steps
            t0 = time.perf_counter()
            index.search(qg, w.k, L, w.reorder_num, args.lut_mode)
            torch.cuda.synchronize()
            est = time.perf_counter() - t0
            steps = int(min(200, max(5, 1.0 / max(est, 1e-4))))
            index.set_profiling(2)          # scan phases marked; the rest of the chain unbroken
            ms, scan, stages = [], [], {}
            for _ in range(steps):
                flush.zero_()
                e0 = torch.cuda.Event(enable_timing=True)
                e1 = torch.cuda.Event(enable_timing=True)
                e0.record(stream)
                index.search(qg, w.k, L, w.reorder_num, args.lut_mode)
                e1.record(stream)
                st = index.stage_times()
                e1.synchronize()
                ms.append(e0.elapsed_time(e1))
                scan.append(st["scan"] + st.get("scan_rest", 0.0))
            index.set_profiling(True)       # per-stage breakdown, a few untimed steps
            for _ in range(min(steps, 10)):
                flush.zero_()
                index.search(qg, w.k, L, w.reorder_num, args.lut_mode)
                for kname, v in index.stage_times().items():
                    stages.setdefault(kname, []).append(v)
            index.set_profiling(False)
            index.sync_status()
            m = statistics.median(ms)
            sc = statistics.median(scan)
            lookups = scanned * w.blocks
            line = {"sweep_point": {"nq": nq, "num_leaves_to_search": L}, "metric": METRIC, "unit": "queries/s",
                    "value": nq / (m * 1e-3), "ms_per_step": m, "steps": steps,
                    "scan_ms": sc, "scan_lookups_per_s": lookups / (sc * 1e-3),
                    "scan_smem_gbs": lookups * (4 if args.lut_mode == 0 else 1) / (sc * 1e-3) / 1e9,
                    "scan_unique_code_gbs": unique_bytes / (sc * 1e-3) / 1e9, "unique_code_bytes": unique_bytes,
                    "points_scanned": scanned, "dtype": "f32" if args.lut_mode == 0 else "u8",
                    "stages_ms": {kname: statistics.median(v) for kname, v in stages.items()},
                    "config": config_dict(w.scaled(nq=nq, num_leaves_to_search=L), args)}
            print(json.dumps(line), flush=True)
    index.close()


def run_encode(args):
    """One JSON line: anisotropic code assignment (ah_encode) of the workload's
    n points against its trained codebook, points/s on the device (inputs
    resident), with the oracle's restatement timed on a sample of points."""
    import torch
    from mips_ivf_centroid_b200 import build as ahbuild, datagen
    ahbuild.build()
    from mips_ivf_centroid_b200 import encode
    import oracle
    w = workload_spec(args)
    T = w.threshold_T or 0.0
    X = datagen.make_data(w)
    ix = datagen.build_index(w, X, "cuda")
    Xg = torch.from_numpy(X).cuda()
    cb = ix.codebook
    stream = torch.cuda.current_stream()
    codes, used = encode(Xg, cb, T, args.passes)
    for _ in range(args.warmup):
        encode(Xg, cb, T, args.passes, out=codes, passes_used=used)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(0) as clk:
        e0.record(stream)
        for _ in range(args.steps):
            encode(Xg, cb, T, args.passes, out=codes, passes_used=used)
        e1.record(stream)
        torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / args.steps
    up = used.cpu().numpy().astype(np.int64)
    B, dpb = w.blocks, w.dims_per_block
    # fp64 operations the descent performs: start (16 centers x dpb x 3 per
    # block), residual sums (dpb x 5 per block), and per pass and block 16
    # centers x (dpb x 6 + 5) plus the current center's dpb x 6
    ops = float(w.n) * (2 * w.d + B * (16 * dpb * 3 + dpb * 5)) + float(up.sum()) * B * (16 * (6 * dpb + 5) + 6 * dpb)
    mhz = SM_MAX_MHZ_FALLBACK
    peak = SM_COUNT * 64 * mhz * 1e6          # fp64 ops per second, one per lane per clock
    # oracle on a sample of points
    ns = min(w.n, 20000)
    t0 = time.perf_counter()
    ocodes, oused = oracle.encode(X[:ns], cb.cpu().numpy(), T, args.passes)
    ot = time.perf_counter() - t0
    same = bool(np.array_equal(ocodes, codes[:ns].cpu().numpy()))
    line = {"metric": "anisotropic code assignment points/s (1 B200)", "value": w.n / (ms * 1e-3),
            "unit": "points/s", "n_gpus": 1, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic (seeded Gaussian mixture; codebook trained on it)",
            "config": {"workload": f"{w.name}-shaped: n={w.n:,} d={w.d} dims_per_block={dpb} T={T} passes<={args.passes}"},
            "passes_mean": float(up.mean()),
            "roofline": {"bound": "alu", "achieved": ops / (ms * 1e-3) / 1e12, "peak": peak / 1e12,
                         "unit": "Tops/s (fp64)", "frac": ops / (ms * 1e-3) / peak, "traffic": None,
                         "peak_source": f"derived: {SM_COUNT} SMs x 64 fp64 lanes x {mhz:.0f} MHz (nominal rate)"},
            "cpu_baseline": {"value": ns / ot, "unit": "points/s", "cores": oracle.max_threads(), "kind": "oracle", "cpu_model": cpu_model(),
                             "sample": f"first {ns} points"},
            "oracle_match_on_sample": same, "clocks": clk.summary(), "gpu_launches": args.steps + args.warmup + 1}
    print(json.dumps(line), flush=True)


def run_kmeans(args):
    """One JSON line: one Lloyd iteration (ah_kmeans_assign + ah_kmeans_update)
    of the workload's n points against its num_leaves centroids, points/s on
    the device, with the oracle timed on a sample of points."""
    import torch
    from mips_ivf_centroid_b200 import build as ahbuild, datagen
    ahbuild.build()
    from mips_ivf_centroid_b200 import kmeans_assign, kmeans_update
    import oracle
    w = workload_spec(args)
    X = datagen.make_data(w)
    rng = np.random.default_rng(1)
    C = X[rng.choice(w.n, size=w.num_leaves, replace=False)].copy()
    Xg, Cg = torch.from_numpy(X).cuda(), torch.from_numpy(C).cuda()
    stream = torch.cuda.current_stream()
    for _ in range(args.warmup):
        a, _ = kmeans_assign(Xg, Cg)
        kmeans_update(Xg, a, Cg)
    torch.cuda.synchronize()
    e0, e1, e2 = (torch.cuda.Event(enable_timing=True) for _ in range(3))
    ta = tu = 0.0
    with ClockSampler(0) as clk:
        for _ in range(args.steps):
            e0.record(stream)
            a, _ = kmeans_assign(Xg, Cg)
            e1.record(stream)
            Cn, cnt = kmeans_update(Xg, a, Cg)
            e2.record(stream)
            torch.cuda.synchronize()
            ta += e0.elapsed_time(e1)
            tu += e1.elapsed_time(e2)
    ta, tu = ta / args.steps, tu / args.steps
    # the anisotropic center update on the same assignment (eta per point from
    # the workload's threshold T, 0.2 where it names none)
    from mips_ivf_centroid_b200 import avq_update
    T_avq = w.threshold_T or 0.2
    for _ in range(max(1, args.warmup)):
        Cv, _, it = avq_update(Xg, a, Cg, T_avq)
    torch.cuda.synchronize()
    e0.record(stream)
    for _ in range(args.steps):
        Cv, _, it = avq_update(Xg, a, Cg, T_avq)
    e1.record(stream)
    torch.cuda.synchronize()
    tv = e0.elapsed_time(e1) / args.steps
    it_np = it.cpu().numpy()
    ops = 3.0 * w.n * w.num_leaves * w.d           # difference, square, sum per (point, centroid, coordinate)
    mhz = SM_MAX_MHZ_FALLBACK
    peak = SM_COUNT * 64 * mhz * 1e6
    ns = min(w.n, 2000)
    t0 = time.perf_counter()
    ao, _ = oracle.kmeans_assign(X[:ns], C)
    ot = time.perf_counter() - t0
    same = bool(np.array_equal(ao, a[:ns].cpu().numpy()))
    line = {"metric": "k-means iteration points/s (1 B200)", "value": w.n / ((ta + tu) * 1e-3), "unit": "points/s",
            "n_gpus": 1, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ta + tu,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic (seeded Gaussian mixture)",
            "config": {"workload": f"{w.name}-shaped: n={w.n:,} d={w.d} centroids={w.num_leaves}"},
            "assign_ms": ta, "update_ms": tu,
            "avq_update": {"ms": tv, "T": T_avq, "cg_steps_mean": float(it_np.mean()), "cg_steps_max": int(it_np.max()),
                           "points_per_s": w.n / (tv * 1e-3),
                           "note": "closed-form anisotropic center update (conjugate gradients, fp64) on the same assignment"},
            "roofline": {"bound": "alu", "kernel": "kmeans_assign", "achieved": ops / (ta * 1e-3) / 1e12,
                         "peak": peak / 1e12, "unit": "Tops/s (fp64)", "frac": ops / (ta * 1e-3) / peak,
                         "traffic": None,
                         "peak_source": f"derived: {SM_COUNT} SMs x 64 fp64 lanes x {mhz:.0f} MHz (nominal rate)"},
            "cpu_baseline": {"value": ns / ot, "unit": "points/s (assignment)", "cores": oracle.max_threads(),
                             "kind": "oracle", "cpu_model": cpu_model(), "sample": f"first {ns} points"},
            "oracle_match_on_sample": same, "clocks": clk.summary(),
            "gpu_launches": 2 * (args.steps + args.warmup) + 4 * (args.steps + max(1, args.warmup))}
    print(json.dumps(line), flush=True)


def run_leaf_shards(args):
    """One JSON line: the leaf-partitioned search.  Every rank holds all
    centroids and the codebook and the points of its own leaves, searches the
    same batch, and the ranks' best R (with exact scores) are gathered and
    merged; value = queries / the slowest rank's device time per step."""
    import torch
    import torch.distributed as dist
    rank, world, local = dist_env()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    init_ranks(world, dev)
    from mips_ivf_centroid_b200 import Index, build as ahbuild, datagen, shard
    ahbuild.build()
    w = workload_spec(args)
    X = datagen.make_data(w)
    Q = datagen.make_queries(w)
    full = datagen.build_index(w, X, dev)
    del X
    sh = shard.shard_arrays(full, world, rank)
    del full
    torch.cuda.empty_cache()
    index = Index(sh)
    qg = torch.from_numpy(Q).to(dev)
    L, k, R, mode = w.num_leaves_to_search, w.k, w.reorder_num, args.lut_mode
    stream = torch.cuda.current_stream()
    flush = torch.empty(2 * L2_BYTES // 4, dtype=torch.float32, device=dev)

    def step():
        local_c = shard.shard_candidates(index, qg, k, L, R, mode)
        g = shard.gather_candidates(local_c) if world > 1 else tuple(
            None if t is None else t.unsqueeze(0).contiguous() for t in local_c)
        return shard.merge_gathered(g, k)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    with ClockSampler(local) as clk:
        for i in range(args.steps):
            flush.zero_()
            ev[i][0].record(stream)
            step()
            ev[i][1].record(stream)
        torch.cuda.synchronize()
    total = max_over_ranks(sum(a.elapsed_time(b) for a, b in ev), dev, world)
    ms = total / args.steps
    if rank == 0:
        line = {"metric": METRIC, "value": w.nq / (ms * 1e-3), "unit": "queries/s", "n_gpus": world,
                "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True,
                "scaling": "strong", "vs_baseline": None, "dtype": "f32" if mode == 0 else "u8",
                "data": "synthetic (seeded Gaussian mixture; index trained on it)",
                "config": dict(config_dict(w, args), parallelism=f"leaf-partitioned x{world}"),
                "clocks": clk.summary()}
        print(json.dumps(line), flush=True)
    index.close()
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


def main():
    args = parse()
    if args.impl == "reference":
        run_reference(args)
    elif args.leaf_shards:
        run_leaf_shards(args)
    elif args.kmeans:
        run_kmeans(args)
    elif args.encode:
        run_encode(args)
    elif args.sweep:
        run_sweep(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
