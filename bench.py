"""Throughput of bipartite prefix-shared attention on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload mixed] [--impl reference]

One step is one pass of the forward over one batch of the named workload (default: the
mixed bipartite batch, 32768 requests, run as the fewest request-disjoint launches that fit
in device memory).  Prints one JSON line on rank 0.  Under torchrun the one batch is split
over the ranks by prefix group (hot prefixes replicated, cold ones on the rank that holds
them, prefixes a rank lacks fetched once from their owner by NCCL send/recv before the timed
steps; no collective inside a step): strong scaling, the step time is the max over ranks of
device time measured with CUDA events.

``--impl reference`` times the fp64 CPU oracle instead (the reference arm): on rank 0 only,
on a bounded sample of the same workload.
"""

from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from workloads import CONFIGS, device_tensors, host_tensors, make_table, split_launches  # noqa: E402

METRIC = "bipartite-attention TFLOP/s and requests/s on 1 B200; % of bf16 tensor roofline"
UNIT = "TFLOP/s"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
L2_BYTES = 126 * 2**20


def load_peaks(path=None):
    """The roofline denominators: each of hbm_gbs, bf16_tflops and bf16_tflops_sustained from
    MEASURED_PEAKS.json when it holds a positive number for it, else the recorded fallback.
    Returns (peaks, kinds) with kinds[key] in {"measured", "fallback"}."""
    p = path or os.path.join(ROOT, "MEASURED_PEAKS.json")
    d = {}
    if os.path.exists(p):
        try:
            d = json.load(open(p))
        except (OSError, ValueError):
            d = {}
    peaks, kinds = {}, {}
    for k, fb in FALLBACK_PEAKS.items():
        v = d.get(k)
        ok = isinstance(v, (int, float)) and not isinstance(v, bool) and v > 0
        peaks[k], kinds[k] = (float(v), "measured") if ok else (fb, "fallback")
    return peaks, kinds


def max_over_ranks(x: float, device) -> float:
    """The largest value over all ranks (every rank calls this, in the same order); x itself
    when no process group is running."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(x)
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def all_ranks(flag: bool, device) -> bool:
    """True only if `flag` holds on every rank (every rank calls this, in the same order)."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return bool(flag)
    t = torch.tensor([1 if flag else 0], dtype=torch.int32, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MIN)
    return bool(t.item())


def whole_job_rate(work_per_rank: float, world: int, steps: int, elapsed_ms: float) -> float:
    """Weak scaling: every rank does `work_per_rank` per step; the job's rate is all ranks' work
    over the slowest rank's time."""
    return work_per_rank * world * steps / (elapsed_ms * 1e-3)


def workload_flops_bytes(tab, H, d, elt):
    from prefix_shared_attention_b200.metrics import algorithmic_bytes, algorithmic_flops
    return (algorithmic_flops(tab.prefix_len, tab.req_prefix, tab.suffix_len, H, d),
            algorithmic_bytes(tab.prefix_len, tab.req_prefix, tab.suffix_len, H, d, elt))


KERNEL_SOURCES = ("bat_attn_tc.cu", "bat_ptx.h", "bat_kernels.h")


def kernel_source_hash():
    """First 16 hex digits of the SHA-256 of the attention kernel's sources, in a fixed order."""
    h = hashlib.sha256()
    for name in KERNEL_SOURCES:
        h.update(open(os.path.join(ROOT, "prefix_shared_attention_b200", "csrc", name), "rb").read())
    return h.hexdigest()[:16]


def traffic_per_launch(workload, alg_bytes_per_launch):
    """DRAM bytes per launch from the committed ncu summary of this workload, if it was taken on
    the current kernel sources; else None.  A capture of a smaller launch of the same workload
    (the first requests and the prefixes they read) is scaled to this launch by algorithmic
    bytes: the ratio of measured to algorithmic traffic is what the capture measures."""
    path = os.path.join(ROOT, "profiles", f"bat_attn_tc_{workload}_traffic.json")
    if not os.path.exists(path):
        return None
    rec = json.load(open(path))
    if rec.get("kernel_sha256_16") != kernel_source_hash():
        return None
    return rec["dram_bytes_per_launch"] / rec["alg_bytes_per_launch"] * alg_bytes_per_launch


class NvmlClockSampler:
    """SM clock and clock-event-reason samples read through NVML (read only) every `period_s`
    while the timed region runs, plus one at its end, so a timed region shorter than a
    polling interval still has a record.  The device is found by its UUID, so the right GPU
    is read whatever CUDA_VISIBLE_DEVICES maps.  `nvml` is the binding module (injectable)."""

    REASONS = (("hw_slowdown", "nvmlClocksEventReasonHwSlowdown"),
               ("hw_thermal_slowdown", "nvmlClocksEventReasonHwThermalSlowdown"),
               ("sw_thermal_slowdown", "nvmlClocksEventReasonSwThermalSlowdown"),
               ("sw_power_cap", "nvmlClocksEventReasonSwPowerCap"))

    def __init__(self, uuid, nvml=None, period_s=0.002):
        self.uuid, self.nvml, self.period = uuid, nvml, period_s
        self.samples = []
        self._stop = threading.Event()
        self.thread = None

    def _sample(self):
        n = self.nvml
        self.samples.append((n.nvmlDeviceGetClockInfo(self.h, n.NVML_CLOCK_SM),
                             n.nvmlDeviceGetMaxClockInfo(self.h, n.NVML_CLOCK_SM),
                             n.nvmlDeviceGetCurrentClocksEventReasons(self.h)))

    def start(self):
        if self.nvml is None:
            import pynvml
            self.nvml = pynvml
        self.nvml.nvmlInit()
        u = self.uuid if self.uuid.startswith("GPU-") else "GPU-" + self.uuid
        self.h = self.nvml.nvmlDeviceGetHandleByUUID(u)
        self._sample()   # the binding works: fail here, before the timed region, if it does not

        def run():
            while not self._stop.wait(self.period):
                self._sample()
        self.samples.clear()
        self.thread = threading.Thread(target=run, daemon=True)
        self.thread.start()

    def stop(self):
        self._stop.set()
        self.thread.join(timeout=2)
        self._sample()
        try:
            self.nvml.nvmlShutdown()
        except Exception:
            pass
        sm = [c for c, _, _ in self.samples]
        reasons = sorted({name for _, _, r in self.samples for name, attr in self.REASONS
                          if r & getattr(self.nvml, attr)})
        return {"sm_mhz": float(np.median(sm)), "sm_max_mhz": max(m for _, m, _ in self.samples),
                "reasons": reasons, "samples": len(sm), "source": "nvml"}


def clock_sampler(dev_index):
    """NVML sampler of this process's GPU, else the nvidia-smi one."""
    import torch
    try:
        s = NvmlClockSampler(str(torch.cuda.get_device_properties(dev_index).uuid))
        s.start()
        s.stop()
        return NvmlClockSampler(s.uuid, s.nvml)
    except Exception:
        return ClockSampler(dev_index)


class ClockSampler:
    """nvidia-smi clock / throttle-reason samples while the timed region runs."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.gpu = gpu_index
        self.proc = None
        self.lines = []

    def start(self):
        try:
            self.proc = subprocess.Popen(["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.FIELDS}",
                                          "--format=csv,noheader,nounits", "-lms", "200"],
                                         stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
        except Exception:
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.thread.join(timeout=2)
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                mx.append(float(parts[2]))
            except ValueError:
                continue
            for n, v in zip(names, parts[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        return {"sm_mhz": float(np.median(sm)) if sm else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": sorted(reasons), "samples": len(sm), "source": "nvidia-smi"}


def fits_launches(tab, spec, free_bytes, elt):
    """Fewest equal request-disjoint launches whose suffix tensors (q, k, v, out) fit next to
    the resident prefix cache in 80 % of free device memory."""
    row = spec.H * spec.d * elt
    cache = 2 * tab.T_cache * row
    budget = 0.80 * free_bytes - cache - (1 << 30)
    for n in range(1, 257):
        if tab.R % n:
            continue
        parts = split_launches(tab, n)
        if 4 * max(p.T_suf for p in parts) * row <= budget:
            return n
    raise RuntimeError("workload does not fit in device memory")


# --------------------------------------------------------------------------------------------
# CPU oracle (reference arm and cpu_baseline): the fp64 oracle as it stands, on a bounded sample

def oracle_sample(workload, target_s=12.0, seed=99, prefix_side=False):
    """Seeded sample of requests (stratified by prefix kind), its host inputs, and its FLOPs."""
    import oracle
    spec = CONFIGS[workload]
    tab = make_table(workload)
    if prefix_side:
        from workloads import prefix_side_table
        tab = prefix_side_table(tab)
    rng = np.random.default_rng(seed)
    order = []
    kinds = np.unique(tab.kind)
    per_kind = [rng.permutation(np.flatnonzero(tab.kind == k)) for k in kinds]
    for i in range(max(len(p) for p in per_kind)):
        for p in per_kind:
            if i < len(p):
                order.append(int(p[i]))
    order = np.array(order)

    def build(reqs):
        sub = tab.subset(reqs)
        used = np.unique(sub.req_prefix[sub.req_prefix >= 0])
        remap = np.full(tab.P, -1, np.int64)
        remap[used] = np.arange(len(used))
        from workloads import RequestTable
        mapped = remap[np.clip(sub.req_prefix, 0, None)] if tab.P else np.zeros_like(sub.req_prefix)
        t = RequestTable(tab.prefix_len[used], np.where(sub.req_prefix >= 0, mapped, -1), sub.suffix_len, sub.kind)
        x = host_tensors(t, spec.H, spec.d, spec.dtype, spec.seed + 5)
        x = {k: v.double().numpy() for k, v in x.items()}
        return t, x

    def run(t, x):
        return oracle.bipartite_attention(x["q"], x["k_suf"], x["v_suf"], x["k_cache"], x["v_cache"],
                                          t.prefix_offsets, t.suffix_offsets, t.req_prefix)

    # Calibrate on one request, then take enough requests for about target_s of CPU work.
    t1, x1 = build(order[:1])
    f1 = workload_flops_bytes(t1, spec.H, spec.d, 2)[0]
    s0 = time.perf_counter()
    run(t1, x1)
    rate = f1 / max(time.perf_counter() - s0, 1e-6)
    n = 1
    flops = f1
    fl_all = [workload_flops_bytes(tab.subset(order[i:i + 1]), spec.H, spec.d, 2)[0] for i in range(min(len(order), 4096))]
    while n < len(fl_all) and flops + fl_all[n] <= rate * target_s:
        flops += fl_all[n]
        n += 1
    t, x = build(order[:n])
    return spec, tab, t, x, run, n


def blas_threads():
    try:
        from threadpoolctl import threadpool_info
        info = [i for i in threadpool_info() if i.get("user_api") == "blas"]
        if info:
            return int(info[0]["num_threads"])
    except Exception:
        pass
    return len(os.sched_getaffinity(0))


def cpu_baseline(workload, target_s=12.0, prefix_side=False):
    spec, tab, t, x, run, n = oracle_sample(workload, target_s, prefix_side=prefix_side)
    flops = workload_flops_bytes(t, spec.H, spec.d, 2)[0]
    s0 = time.perf_counter()
    run(t, x)
    dt = time.perf_counter() - s0
    what = "prefixes (prefix-side step)" if prefix_side else "requests"
    return {"value": flops / dt / 1e12, "unit": UNIT, "cores": blas_threads(), "kind": "oracle",
            "sample": f"{n} of {tab.R} {what} of '{workload}' (stratified by prefix kind), fp64 numpy, "
                      f"{flops / 1e9:.1f} GFLOP in {dt:.2f} s",
            "requests_per_s": n / dt}


def repo_libraries_loaded():
    """Shared objects of this repository mapped into the process (the reference arm must map
    none: it times the oracle alone)."""
    try:
        maps = open("/proc/self/maps").read().splitlines()
    except OSError:
        return []
    return sorted({l.split()[-1] for l in maps if l.split()[-1].startswith(ROOT) and ".so" in l.split()[-1]})


def run_reference(args, rank, world):
    if rank != 0:
        return 0
    spec, tab, t, x, run, n = oracle_sample(args.workload, target_s=max(5.0, 150.0 / max(args.steps + args.warmup, 1)),
                                            prefix_side=args.prefix_side)
    flops = workload_flops_bytes(t, spec.H, spec.d, 2)[0]
    for _ in range(args.warmup):
        run(t, x)
    s0 = time.perf_counter()
    for _ in range(args.steps):
        run(t, x)
    dt = time.perf_counter() - s0
    value = flops * args.steps / dt / 1e12
    cores = blas_threads()
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": dt / args.steps * 1e3,
            "higher_is_better": True, "scaling": "strong", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": args.workload + ("/prefix-side" if args.prefix_side else ""), "sample_requests": n,
                       "requests": tab.R, "H": spec.H, "d": spec.d},
            "requests_per_s": n * args.steps / dt,
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle",
                             "sample": f"{n} of {tab.R} requests per step, fp64 numpy oracle"},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
            "repo_libraries_loaded": [os.path.relpath(p, ROOT) for p in repo_libraries_loaded()]}
    print(json.dumps(line), flush=True)
    return 0


# --------------------------------------------------------------------------------------------
# GPU arm

SECONDARY = ("long-user-history", "item-as-prefix", "user-as-prefix")


def gbla_work(seq_lens, H, d=128):
    """Algorithmic FLOPs and bytes of one GBLA layer: the state (2 T d^2 per head) and the output
    (2 T d^2 per head) contractions; q, k, v, z and the gate logits read once, y written once."""
    T = float(sum(seq_lens))
    return 4.0 * T * d * d * H, (5.0 * T * H * d + T * H) * 2.0


def time_gbla(dev, peaks, reps=10, warmup=3, n_seqs=0):
    """CUDA-event time of the GBLA layer (state, reduce and output kernels) on the long-history
    batch (or its first `n_seqs` histories), L2 flushed before every timed launch, clocks
    sampled meanwhile."""
    import torch
    import prefix_shared_attention_b200 as bat
    from workloads import GBLA_LONG_HISTORY
    from workloads import gbla_tensors
    W = dict(GBLA_LONG_HISTORY)
    if n_seqs:
        W["seq_lens"] = W["seq_lens"][:n_seqs]
        W["description"] = f"first {n_seqs} of: " + W["description"]
    x, so = gbla_tensors(W["seq_lens"], W["H"], W["seed"], device=dev)
    y = torch.empty_like(x["q"])
    flush = torch.empty(2 * L2_BYTES, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream()
    with bat.GblaPlan(so, W["H"]) as plan:
        ws = torch.empty(plan.workspace_bytes, dtype=torch.uint8, device=dev)
        fwd = lambda: bat.bat_gbla_forward(plan, x["q"], x["k"], x["v"], x["a"], x["z"], x["cq"], x["ck"], x["cv"],
                                           x["g"], y=y, workspace=ws, stream=stream)
        for _ in range(warmup):
            fwd()
        torch.cuda.synchronize()
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(reps)]
        clocks = clock_sampler(dev.index)
        clocks.start()
        for a, b in ev:
            flush.zero_()
            a.record(stream)
            fwd()
            b.record(stream)
        torch.cuda.synchronize()
        clk = clocks.stop()
        if bat.bat_get_device_status() != bat.BAT_OK:
            raise RuntimeError(bat.last_error())
        n_chunks = len(plan.chunks())
    ms = sorted(a.elapsed_time(b) for a, b in ev)
    med = ms[len(ms) // 2]
    flops, nbytes = gbla_work(W["seq_lens"], W["H"])
    r = {"workload": W["description"], "ms": med, "tflops": flops / (med * 1e-3) / 1e12,
         "tokens_per_s": float(sum(W["seq_lens"])) / (med * 1e-3), "launches": 3, "chunks": n_chunks, "reps": reps,
         "l2": "flushed before every timed launch", "roofline": roofline_of(flops, nbytes, med * 1e-3, peaks),
         "clocks": clk}
    del x, y, flush, ws
    torch.cuda.empty_cache()
    return r


def shard_batch(full, spec, rank, world, dev):
    """This rank's share of one batch and its local prefix pool.  The pool starts sharded by
    prefix id (every rank draws the whole pool from one seed and keeps the prefixes it owns, so
    a prefix's K/V is the same on every rank); `place` assigns the request groups, and the
    prefixes a rank needs but does not own are fetched from their owners by NCCL send/recv
    (timed with CUDA events, max over ranks).  Returns (local table, pool tensors, fetch record)."""
    import torch
    import torch.distributed as dist
    from prefix_shared_attention_b200.sharding import bat_copy_rows, exchange_prefixes, hash_owner, local_table, place
    owner = hash_owner(full.P, world)
    pl = place(full.prefix_len, full.req_prefix, full.suffix_len, world, spec.H, spec.d, owner=owner)
    everything = device_tensors(full, spec.H, spec.d, spec.dtype, spec.seed, device=dev, which=("k_cache", "v_cache"))
    owned = np.flatnonzero(owner == rank)
    po = full.prefix_offsets
    lens = full.prefix_len[owned]
    dst = np.concatenate([[0], np.cumsum(lens)]).astype(np.int64)
    ok_ = torch.empty((int(dst[-1]), spec.H, spec.d), dtype=everything["k_cache"].dtype, device=dev)
    ov_ = torch.empty_like(ok_)
    bat_copy_rows(everything["k_cache"], everything["v_cache"],
                  [(int(po[p]), int(full.prefix_len[p]), int(dst[i])) for i, p in enumerate(owned) if full.prefix_len[p]],
                  ok_, ov_)
    torch.cuda.synchronize()
    del everything
    torch.cuda.empty_cache()
    dist.barrier()   # a collective before the first point-to-point batch, as NCCL requires
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record()
    k_pool, v_pool, nbytes = exchange_prefixes(pl, rank, world, full.prefix_len, owned, ok_, ov_,
                                               copy_rows=bat_copy_rows)
    b.record()
    torch.cuda.synchronize()
    fetch_ms = max_over_ranks(a.elapsed_time(b), dev)
    del ok_, ov_
    torch.cuda.empty_cache()
    tab, _ = local_table(pl, rank, full)
    total = torch.tensor([float(nbytes), float(len(pl.fetch[rank]))], dtype=torch.float64, device=dev)
    dist.all_reduce(total)
    rec = {"ms": fetch_ms, "bytes": float(total[0].item()), "prefixes": int(total[1].item()),
           "hot_prefixes": int(len(pl.hot)), "load_imbalance": float(pl.load.max() / pl.load.mean()),
           "timed": "once before the forward steps (not inside them)"}
    return tab, {"k_cache": k_pool, "v_cache": v_pool}, rec


def roofline_of(flops, nbytes, kernel_s, peaks):
    """Which roof binds (algorithmic FLOP per byte against the ridge of the measured peaks) and
    the fraction of it reached; tensor-bound work is compared with the burst bf16 figure."""
    ridge = float(peaks["bf16_tflops"]) * 1e12 / (float(peaks["hbm_gbs"]) * 1e9)
    tf = flops / kernel_s / 1e12
    if flops / nbytes < ridge:
        gbs = nbytes / kernel_s / 1e9
        return {"bound": "hbm", "achieved": gbs, "peak": float(peaks["hbm_gbs"]), "unit": "GB/s",
                "frac": gbs / float(peaks["hbm_gbs"]), "tensor_tflops": tf}
    return {"bound": "tensor", "achieved": tf, "peak": float(peaks["bf16_tflops"]), "unit": "TFLOP/s",
            "frac": tf / float(peaks["bf16_tflops"])}


def time_secondary(name, dev, peaks, reps=10, warmup=3):
    """CUDA-event time of one forward of a named workload (one launch), L2 flushed before every
    timed launch, clocks sampled meanwhile.  The same kernel and launch path as the main line."""
    import torch
    import prefix_shared_attention_b200 as bat
    spec = CONFIGS[name]
    tab = make_table(name)
    x = device_tensors(tab, spec.H, spec.d, spec.dtype, spec.seed, device=dev)
    out = torch.empty_like(x["q"])
    flush = torch.empty(2 * L2_BYTES, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream()
    with bat.Plan(tab.req_prefix, tab.suffix_offsets, tab.prefix_offsets, spec.H, spec.d, bat.BAT_BF16) as plan:
        ws = torch.empty(max(plan.workspace_bytes, 16), dtype=torch.uint8, device=dev)

        def fwd():
            bat.bat_attention_forward(plan, x["q"], x["k_suf"], x["v_suf"], x["k_cache"], x["v_cache"], out=out,
                                      workspace=ws, stream=stream)
        for _ in range(warmup):
            fwd()
        torch.cuda.synchronize()
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(reps)]
        clocks = clock_sampler(dev.index)
        clocks.start()
        for a, b in ev:
            flush.zero_()
            a.record(stream)
            fwd()
            b.record(stream)
        torch.cuda.synchronize()
        clk = clocks.stop()
        if bat.bat_get_device_status() != bat.BAT_OK:
            raise RuntimeError(bat.last_error())
        n_launch = 1 + (plan.info().n_merges > 0)
    ms = sorted(a.elapsed_time(b) for a, b in ev)
    med = ms[len(ms) // 2]
    flops, nbytes = workload_flops_bytes(tab, spec.H, spec.d, 2)
    r = {"tflops": flops / (med * 1e-3) / 1e12, "requests_per_s": tab.R / (med * 1e-3), "ms": med,
         "launches": n_launch, "reps": reps, "l2": "flushed before every timed launch",
         "roofline": roofline_of(flops, nbytes, med * 1e-3, peaks), "clocks": clk}
    del x, out, flush, ws
    torch.cuda.empty_cache()
    return r


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=5)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--workload", default="mixed", choices=sorted(CONFIGS))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--e2e-steps", type=int, default=1)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--launches", type=int, default=0, help="override the number of launches per step")
    ap.add_argument("--prefix-side", action="store_true",
                    help="time the prefix-side step instead: every prefix the workload reads attends over "
                         "its own tokens (the outputs of the prefix tokens themselves)")
    ap.add_argument("--subset", type=int, default=0,
                    help="profiling aid: only the first N requests (and the prefixes they read); not a bench line")
    ap.add_argument("--no-secondary", action="store_true",
                    help="skip the one-launch timings of the other bf16 workloads")
    ap.add_argument("--gbla", type=int, default=-1, metavar="N_SEQS",
                    help="profiling aid: time only the GBLA layer on the long-history batch (0: all of its "
                         "histories, else the first N) and print its record; not a bench line")
    args = ap.parse_args()
    assert args.warmup >= 3 or args.impl == "reference" or os.environ.get("BAT_BENCH_ALLOW_SHORT"), \
        "at least 3 warm-up steps"

    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        return run_reference(args, rank, world)

    import torch
    import torch.distributed as dist
    import prefix_shared_attention_b200 as bat

    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=300), device_id=dev)

    if args.gbla >= 0:
        if rank == 0:
            rec = time_gbla(dev, load_peaks()[0], reps=max(args.steps, 1), warmup=args.warmup, n_seqs=args.gbla)
            print(json.dumps(rec), flush=True)
        return 0

    spec = CONFIGS[args.workload]
    assert spec.dtype == "bf16", "the bench times the bf16 tensor-core path"
    elt = 2
    tab = make_table(args.workload)
    if args.subset:
        tab = tab.compact(np.arange(min(args.subset, tab.R)))
    if args.prefix_side:
        from workloads import prefix_side_table
        tab = prefix_side_table(tab)
    full = tab
    seed = spec.seed + 1000 * rank
    fetch = None
    if world > 1:
        # The one batch split over the ranks: hot prefixes replicated, cold ones on the rank that
        # holds them (a pool sharded by prefix id), groups moved off an overloaded owner fetch
        # their prefix from it (point-to-point copies over NVLink).
        tab, cache, fetch = shard_batch(full, spec, rank, world, dev)
    else:
        cache = device_tensors(tab, spec.H, spec.d, spec.dtype, seed, device=dev, which=("k_cache", "v_cache"))
    free, total = torch.cuda.mem_get_info()
    # fits_launches budgets the resident pool itself, which is already allocated here.
    free += sum(t.numel() * t.element_size() for t in cache.values())
    n_launch = args.launches or fits_launches(tab, spec, free, elt)
    parts = split_launches(tab, n_launch)
    rows = max(p.T_suf for p in parts)
    suf = device_tensors(parts[0], spec.H, spec.d, spec.dtype, seed + 1, device=dev, which=("q", "k_suf", "v_suf"),
                         rows=rows)
    out = torch.empty_like(suf["q"])
    t_plan = time.perf_counter()
    plans = [bat.Plan(p.req_prefix, p.suffix_offsets, p.prefix_offsets, spec.H, spec.d, bat.BAT_BF16) for p in parts]
    plan_ms = (time.perf_counter() - t_plan) * 1e3   # host grouping pass + work-list upload, all launches
    ws_bytes = max(pl.workspace_bytes for pl in plans)
    ws = torch.empty(max(ws_bytes, 16), dtype=torch.uint8, device=dev)
    launches_per_step = sum(1 + (pl.info().n_merges > 0) for pl in plans)
    flops_l, bytes_l = zip(*[workload_flops_bytes(p, spec.H, spec.d, elt) for p in parts])
    step_flops, step_bytes = float(sum(flops_l)), float(sum(bytes_l))
    stream = torch.cuda.current_stream()

    def step(events=None):
        for i, (p, pl) in enumerate(zip(parts, plans)):
            T = p.T_suf
            if events is not None:
                events[i][0].record(stream)
            bat.bat_attention_forward(pl, suf["q"][:T], suf["k_suf"][:T], suf["v_suf"][:T], cache["k_cache"],
                                      cache["v_cache"], out=out[:T], workspace=ws, stream=stream)
            if events is not None:
                events[i][1].record(stream)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    if bat.bat_get_device_status() != bat.BAT_OK:
        raise RuntimeError(bat.last_error())

    ev = [[[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in parts] for _ in range(args.steps)]
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    clocks = clock_sampler(local_rank)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    clocks.start()
    t0.record(stream)
    for k in range(args.steps):
        step(ev[k])
    t1.record(stream)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    clk = clocks.stop()
    status = bat.bat_get_device_status()
    if status != bat.BAT_OK:
        raise RuntimeError(bat.last_error())
    elapsed_ms = t0.elapsed_time(t1)
    kernel_ms = [sum(ev[k][i][0].elapsed_time(ev[k][i][1]) for k in range(args.steps)) / args.steps
                 for i in range(len(parts))]
    elapsed_ms = max_over_ranks(elapsed_ms, dev)

    ms_per_step = elapsed_ms / args.steps
    # Every rank serves its share of the one batch: the job's rate is the whole batch's work over
    # the slowest rank's time (strong scaling; at one rank the share is the batch).
    job_flops = workload_flops_bytes(full, spec.H, spec.d, elt)[0]
    value = job_flops * args.steps / (elapsed_ms * 1e-3) / 1e12
    req_s = full.R * args.steps / (elapsed_ms * 1e-3)
    peaks, peak_kinds = load_peaks()
    achieved = step_flops / (sum(kernel_ms) * 1e-3) / 1e12
    # Which roof binds: algorithmic FLOP per byte against the ridge of the measured peaks.
    ridge = float(peaks["bf16_tflops"]) * 1e12 / (float(peaks["hbm_gbs"]) * 1e9)
    hbm_bound = step_flops / step_bytes < ridge
    # The fraction divides by the burst bf16 GEMM figure, the denominator the target is stated
    # against (>= 60 % of it); the sustained figure (the same GEMM back to back for seconds,
    # under the power cap) is reported beside it.
    peak = float(peaks["bf16_tflops"])
    traffic = None if (args.prefix_side or args.subset) else traffic_per_launch(args.workload, step_bytes / n_launch)

    # End to end through the public API with host buffers: every launch's request tokens (q,
    # k, v) go host -> device from pinned memory, the forward runs, the output comes back.  The
    # prefix cache is resident (it is built once per cached prefix, off this path).  As a
    # serving loop would, the launches are pipelined over two device buffer sets and three
    # streams: the copy-in of launch i+1 and the copy-out of launch i-1 overlap the forward of
    # launch i.  Each launch is split in two so that two buffer sets fit beside the cache.
    e2e = None
    row_b = spec.H * spec.d * 2
    if not args.no_e2e:
        for pl in plans:
            pl.close()
        suf = out = None
        torch.cuda.empty_cache()
        parts2 = split_launches(tab, 2 * n_launch)
        rows2 = max(p.T_suf for p in parts2)
        need_host = 4 * rows2 * row_b
        # Every rank on this node pins its own host buffers.
        local_world = int(os.environ.get("LOCAL_WORLD_SIZE", str(world)))
        try:
            import psutil
            host_ok = psutil.virtual_memory().available > 1.5 * need_host * local_world
        except Exception:
            host_ok = True
        free_now, _ = torch.cuda.mem_get_info()
        fits = free_now >= 0.9 * 2 * 4 * rows2 * row_b
        # Every rank takes the same collective steps: agree on whether all ranks run it.
        everyone = all_ranks(host_ok and fits, dev)
        if not host_ok:
            e2e = {"value": None, "unit": UNIT,
                   "skipped": f"needs {need_host * local_world / 1e9:.0f} GB of pinned host memory on this node"}
        elif not fits:
            e2e = {"value": None, "unit": UNIT, "skipped": "two device buffer sets do not fit"}
        elif not everyone:
            e2e = {"value": None, "unit": UNIT, "skipped": "another rank cannot hold its end-to-end buffers"}
        else:
            plans2 = [bat.Plan(p.req_prefix, p.suffix_offsets, p.prefix_offsets, spec.H, spec.d, bat.BAT_BF16)
                      for p in parts2]
            ws2 = torch.empty(max(max(pl.workspace_bytes for pl in plans2), 16), dtype=torch.uint8, device=dev)
            h = {k: torch.empty((rows2, spec.H, spec.d), dtype=torch.bfloat16, pin_memory=True) for k in ("q", "k", "v", "o")}
            sets = [{k: torch.empty((rows2, spec.H, spec.d), dtype=torch.bfloat16, device=dev) for k in ("q", "k", "v", "o")}
                    for _ in range(2)]
            gen = torch.Generator(device=dev)
            gen.manual_seed(seed + 2)
            for k in ("q", "k", "v"):   # N(0,1) request tokens, drawn on the device, kept on the host
                sets[0][k].normal_(generator=gen)
                h[k].copy_(sets[0][k])
            s_in, s_run, s_out = torch.cuda.Stream(), torch.cuda.Stream(), torch.cuda.Stream()

            def e2e_step():
                ev_run = [None, None]
                ev_out = [None, None]
                for i, (p, pl) in enumerate(zip(parts2, plans2)):
                    T, b = p.T_suf, sets[i % 2]
                    with torch.cuda.stream(s_in):
                        # The buffer set is free once launch i-2 has read it and its output left.
                        for ev in (ev_run[i % 2], ev_out[i % 2]):
                            if ev is not None:
                                s_in.wait_event(ev)
                        b["q"][:T].copy_(h["q"][:T], non_blocking=True)
                        b["k"][:T].copy_(h["k"][:T], non_blocking=True)
                        b["v"][:T].copy_(h["v"][:T], non_blocking=True)
                        ev_in = torch.cuda.Event()
                        ev_in.record(s_in)
                    s_run.wait_event(ev_in)
                    bat.bat_attention_forward(pl, b["q"][:T], b["k"][:T], b["v"][:T], cache["k_cache"], cache["v_cache"],
                                              out=b["o"][:T], workspace=ws2, stream=s_run)
                    ev_run[i % 2] = torch.cuda.Event()
                    ev_run[i % 2].record(s_run)
                    with torch.cuda.stream(s_out):
                        s_out.wait_event(ev_run[i % 2])
                        h["o"][:T].copy_(b["o"][:T], non_blocking=True)
                        ev_out[i % 2] = torch.cuda.Event()
                        ev_out[i % 2].record(s_out)
                return ev_out

            e2e_step()
            torch.cuda.synchronize()
            if world > 1:
                dist.barrier()
            a, b_ev = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(s_in)
            for _ in range(args.e2e_steps):
                last = e2e_step()
            for ev in last:
                if ev is not None:
                    s_out.wait_event(ev)
            b_ev.record(s_out)
            torch.cuda.synchronize()
            e_ms = max_over_ranks(a.elapsed_time(b_ev), dev)
            e2e = {"value": job_flops * args.e2e_steps / (e_ms * 1e-3) / 1e12, "unit": UNIT,
                   "h2d_bytes_per_step": int(3 * full.T_suf * row_b), "d2h_bytes_per_step": int(full.T_suf * row_b),
                   "ms_per_step": e_ms / args.e2e_steps, "steps": args.e2e_steps,
                   "pipeline": f"{len(parts2)} launches over 2 buffer sets; copy-in, forward, copy-out on 3 streams"}
            for pl in plans2:
                pl.close()
            del h, sets, ws2
            if bat.bat_get_device_status() != bat.BAT_OK:
                raise RuntimeError(bat.last_error())
    else:
        for pl in plans:
            pl.close()

    suf = cache = out = ws = None
    torch.cuda.empty_cache()
    secondary = None
    if not (args.no_secondary or args.subset or args.prefix_side or args.workload != "mixed"):
        # One launch of each other bf16 workload, on every rank (same steps everywhere).
        if world == 1:
            secondary = {name: time_secondary(name, dev, load_peaks()[0]) for name in SECONDARY}
            # The second workload: one GBLA layer over long user histories (HBM-bound).
            secondary["gbla-long-history"] = time_gbla(dev, load_peaks()[0])

    base = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        base = cpu_baseline(args.workload, prefix_side=args.prefix_side)

    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True, "scaling": "strong",
            "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": {"workload": args.workload + (f"[:{args.subset}]" if args.subset else "")
                                   + ("/prefix-side" if args.prefix_side else ""), "requests": tab.R, "launches": n_launch, "H": spec.H, "d": spec.d,
                       "prefixes_cached": tab.P, "tokens_suffix": tab.T_suf, "tokens_cache": tab.T_cache,
                       "l2": "inputs larger than L2 (%.0f GB per launch)" % (step_bytes / n_launch / 1e9),
                       "parallelism": (f"{world} ranks, one batch split by prefix group (hot replicated, cold "
                                       f"sharded)" if world > 1 else "single")},
            "requests_per_s": req_s,
            "plan_ms": plan_ms,
            "roofline": {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                         "frac": achieved / peak, "traffic": traffic,
                         "peak_source": f"{peak_kinds['bf16_tflops']} bf16_tflops (burst)",
                         "target_frac": 0.60, "target_met": achieved / peak >= 0.60,
                         "frac_of_burst": achieved / float(peaks["bf16_tflops"]),
                         "frac_of_sustained": achieved / float(peaks.get("bf16_tflops_sustained", peak)),
                         "frac_of_spec": achieved / 2250.0,
                         "flop_per_byte": step_flops / step_bytes, "ridge_flop_per_byte": ridge,
                         "kernel": "bat_attn_tc_kernel", "kernel_ms_per_launch": kernel_ms,
                         "alg_gflop_per_launch": [f / 1e9 for f in flops_l],
                         "alg_gb_per_launch": [b / 1e9 for b in bytes_l]},
            "cpu_baseline": base, "e2e": e2e, "gpu_launches": launches_per_step * args.steps, "clocks": clk,
        }
        if secondary is not None:
            line["secondary"] = secondary
        if fetch is not None:
            line["prefix_fetch"] = fetch
        if hbm_bound:
            # Left of the ridge: the bandwidth roof binds; report against the measured copy rate.
            gbs = step_bytes / (sum(kernel_ms) * 1e-3) / 1e9
            line["roofline"].update({"bound": "hbm", "achieved": gbs, "peak": float(peaks["hbm_gbs"]), "unit": "GB/s",
                                     "frac": gbs / float(peaks["hbm_gbs"]),
                                     "peak_source": f"{peak_kinds['hbm_gbs']} hbm_gbs", "tensor_tflops": achieved})
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
