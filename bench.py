#!/usr/bin/env python
"""Benchmark: effective attention TFLOP/s of one fused forward + backward step.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--config NAME] [--impl reference]

A step is one sdpa_fwd + sdpa_bwd over one batch of seeded synthetic inputs
already resident in HBM.  Effective FLOPs count only unmasked (query, key)
pairs P per (batch, query head): forward 4 d P, backward 10 d P (the
recompute of the scores included), 14 d P in total.  Per kernel, the
FLOPs are the matrix products that kernel needs for its own outputs over the
unmasked pairs: forward 4 d P, dQ 6 d P (S, dP, dQ), dK/dV 8 d P (S, dP, dV,
dK).  With N > 1 (torchrun)
every rank runs its own batch (replicas; no collective on the data path) and
rank 0 prints the whole-job rate: all ranks' FLOPs / the slowest rank's time.

--impl reference times the float64 CPU oracle on the host cores instead, on a
bounded sample of the same workload (one KV head group of one batch per step).

--bias-grad (a workload with a bias) times the step with the bias gradient
(sdpa_bwd_bias_grad) beside the plain step on the same inputs, and reports
the gradient's extra cost against its extra HBM traffic.
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

METRIC = "effective attention TFLOP/s fwd+bwd (unmasked FLOPs) and % of B200 BF16 peak"

CONFIGS = {
    "mistral4k": dict(B=4, Hq=32, Hkv=8, L=4096, d=128, causal=True, wl=4096, wr=-1, bias="none"),
    "mistral8k": dict(B=2, Hq=32, Hkv=8, L=8192, d=128, causal=True, wl=4096, wr=-1, bias="none"),
    "t5rpe": dict(B=16, Hq=12, Hkv=12, L=1024, d=64, causal=False, wl=-1, wr=-1, bias="t5"),
    "t5dense": dict(B=16, Hq=12, Hkv=12, L=1024, d=64, causal=False, wl=-1, wr=-1, bias="dense"),
    "tiny": dict(B=1, Hq=2, Hkv=2, L=128, d=64, causal=True, wl=-1, wr=-1, bias="none"),
    # the Mistral GQA shape with an in-kernel ALiBi bias (slopes 2^(-8 (h+1) / 32))
    "alibi_causal_4k": dict(B=4, Hq=32, Hkv=8, L=4096, d=128, causal=True, wl=-1, wr=-1,
                            bias="alibi"),
    # the t5rpe shape at batch 4: the case the bias-gradient ncu capture runs
    # on (its fp32 dS, 200 MB, still larger than L2)
    "t5rpe_small": dict(B=4, Hq=12, Hkv=12, L=1024, d=64, causal=False, wl=-1, wr=-1, bias="t5"),
    # the t5dense shape at batch 4: the case its ncu capture runs on (the
    # fp32 bias, 200 MB, still larger than L2)
    "t5dense_small": dict(B=4, Hq=12, Hkv=12, L=1024, d=64, causal=False, wl=-1, wr=-1,
                          bias="dense"),
    # the mistral4k shape at batch 2: the case the ncu captures run on (inputs
    # still larger than L2, a few hundred MB on the device)
    "mistral4k_small": dict(B=2, Hq=32, Hkv=8, L=4096, d=128, causal=True, wl=4096, wr=-1,
                            bias="none"),
}
# The head-sharing and sequence-length sweep, forward only: Hq 32, d 128,
# causal, Hkv 32 (MHA) / 8 (GQA) / 1 (MQA), B * L = 32768 tokens.
for _hkv, _tag in ((32, "mha"), (8, "gqa"), (1, "mqa")):
    for _L in (512, 2048, 8192, 16384):
        CONFIGS[f"sweep_{_tag}_{_L}"] = dict(B=32768 // _L, Hq=32, Hkv=_hkv, L=_L, d=128,
                                             causal=True, wl=-1, wr=-1, bias="none",
                                             fwd_only=True)

# DRAM bytes per launch of a kernel (dram__bytes_read.sum + dram__bytes_write.sum
# from one ncu capture, divided by the captured batch size), keyed by workload
# shape and kernel, with the hash of the kernel sources the counters were taken
# on.  A bench workload of the same shape reports them scaled to its batch, and
# only while the library is built from exactly those sources.
NCU_TRAFFIC = {
    # mistral4k_small (batch 2) capture, profiles/mistral4k_small_full_capture.md
    ("mistral4k", "fwd"): {"bytes_per_batch": (100771328 + 37383168) / 2,
        "source_hash": "99e2ec3349212877272f08c8b7b1e98abfcf74474ee83ea1a209a2e3e5a6bec4"},
    ("mistral4k", "bwd_dq"): {"bytes_per_batch": (171738624 + 45638144) / 2,
        "source_hash": "99e2ec3349212877272f08c8b7b1e98abfcf74474ee83ea1a209a2e3e5a6bec4"},
    ("mistral4k", "bwd_dkdv"): {"bytes_per_batch": (170260224 + 24276224) / 2,
        "source_hash": "99e2ec3349212877272f08c8b7b1e98abfcf74474ee83ea1a209a2e3e5a6bec4"},
    # t5dense_small (batch 4) capture, profiles/t5dense_small_capture.md
    ("t5dense", "fwd"): {"bytes_per_batch": (233312768 + 5899776) / 4,
        "source_hash": "99e2ec3349212877272f08c8b7b1e98abfcf74474ee83ea1a209a2e3e5a6bec4"},
    ("t5dense", "bwd_dq"): {"bytes_per_batch": (241260288 + 6072064) / 4,
        "source_hash": "99e2ec3349212877272f08c8b7b1e98abfcf74474ee83ea1a209a2e3e5a6bec4"},
    ("t5dense", "bwd_dkdv"): {"bytes_per_batch": (227603456 + 8563200) / 4,
        "source_hash": "99e2ec3349212877272f08c8b7b1e98abfcf74474ee83ea1a209a2e3e5a6bec4"},
}


# DRAM bytes the T5 table gradient adds to one backward, per batch entry:
# (dQ kernel with dS output - plain dQ kernel) + diagonal sums + piece fold +
# bucket sums, each as dram__bytes.sum.per_second x gpu__time_duration of one
# launch from one ncu capture of
#   python bench.py --config t5rpe_small --bias-grad --steps 1 --warmup 1
# under ncu --section SpeedOfLight --section MemoryWorkloadAnalysis
#   -k regex:"bwd_dq_kernel|t5_" -c 6 (batch 4).
BIAS_GRAD_TRAFFIC = {
}


def bias_grad_traffic(config_name, batch):
    """ncu DRAM bytes the bias gradient adds to one step of this workload, else None."""
    from scaled_dot_product_bwd_b200.build import source_hash
    rec = BIAS_GRAD_TRAFFIC.get(config_name.replace("_small", ""))
    if rec is None or rec["source_hash"] != source_hash():
        return None
    return int(round(rec["bytes_per_batch"] * batch))


def traffic_per_launch(config_name, kernel, batch):
    """ncu DRAM bytes of one launch of `kernel` on this workload, else None."""
    from scaled_dot_product_bwd_b200.build import source_hash
    shape = config_name.replace("_small", "")
    rec = NCU_TRAFFIC.get((shape, kernel))
    if rec is None or rec["source_hash"] != source_hash():
        return None
    return int(round(rec["bytes_per_batch"] * batch))


def describe(c):
    mask = "causal" if c["causal"] else "bidirectional"
    if c["wl"] >= 0:
        mask += f" window_left={c['wl']}"
    fwd = ", forward only" if c.get("fwd_only") else ""
    return (f"B={c['B']} Hq={c['Hq']} Hkv={c['Hkv']} L={c['L']} d={c['d']} {mask} "
            f"bias={c['bias']}{fwd}")


def visible_pairs(L, causal, wl, wr):
    """Unmasked (i, j) pairs of one head: sum over rows of the visible key span."""
    i = np.arange(L, dtype=np.int64)
    lo = np.maximum(0, i - wl) if wl >= 0 else np.zeros(L, np.int64)
    hi = np.full(L, L - 1, np.int64)
    if causal:
        hi = np.minimum(hi, i)
    if wr >= 0:
        hi = np.minimum(hi, i + wr)
    return int(np.maximum(0, hi - lo + 1).sum())


def flop_counts(c):
    P = visible_pairs(c["L"], c["causal"], c["wl"], c["wr"])
    heads = c["B"] * c["Hq"]
    d = c["d"]
    return dict(P=P, fwd=4 * d * P * heads, bwd=10 * d * P * heads, bwd_strict=8 * d * P * heads,
                bwd_dq=6 * d * P * heads, bwd_dkdv=8 * d * P * heads)


def kernel_bytes(c):
    """Algorithmic HBM bytes of one launch of each kernel: every input read
    once and every output written once (bf16 tensors, fp32 LSE / D / bias)."""
    B, L, Hq, Hkv, d = c["B"], c["L"], c["Hq"], c["Hkv"], c["d"]
    q = B * L * Hq * d * 2
    kv = B * L * Hkv * d * 2
    vec = B * Hq * L * 4
    bias = B * Hq * L * L * 4 if c["bias"] == "dense" else 0
    return {"fwd": q + 2 * kv + q + vec + bias,
            "bwd_preprocess": 2 * q + vec,
            "bwd_dq": q + 2 * kv + q + 2 * vec + bias + q,
            "bwd_dkdv": q + 2 * kv + q + 2 * vec + bias + 2 * kv}


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            pk = json.load(f)
        return dict(tflops=pk["bf16_tflops"], tflops_sustained=pk.get("bf16_tflops_sustained"),
                    hbm=pk["hbm_gbs"], source="measured")
    return dict(tflops=1590.0, tflops_sustained=1400.0, hbm=6650.0, source="fallback")


class ClockSampler:
    """SM clock and clock-event (throttle) reasons sampled while the timed
    region runs.

    NVML is polled from a thread every ~2 ms on the GPU that CUDA device
    `gpu` is (found by its UUID, so CUDA_VISIBLE_DEVICES cannot point it at
    another GPU); where NVML cannot be used, nvidia-smi's query loop is read
    instead.  Every sample is timestamped.  ready() waits for the first
    sample, so that the timed region, bracketed by mark_start() /
    mark_end(), falls inside the sampled stretch; the report keeps the
    samples taken during the region, or the one nearest to it when the
    region is shorter than the sampling interval.  Only reads settings."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
    NAMES = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")
    PERIOD_S = 0.002

    def __init__(self, gpu: int):
        import threading
        self.proc = None
        self.nvml = None
        self.rows = []           # (monotonic time, sm MHz, max sm MHz, {reasons})
        self.lines = []          # nvidia-smi: (monotonic time, line)
        self.t0 = self.t1 = None
        self.first = threading.Event()
        self.halt = threading.Event()
        self.reader = None
        if self._open_nvml(gpu):
            self.reader = threading.Thread(target=self._poll, daemon=True)
            self.reader.start()
            return
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "50", "-i", str(gpu)],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except (OSError, ValueError):
            self.proc = None
            return
        self.reader = threading.Thread(target=self._read, daemon=True)
        self.reader.start()

    def _open_nvml(self, gpu):
        try:
            import pynvml
            import torch
            uuid = str(torch.cuda.get_device_properties(gpu).uuid)
            pynvml.nvmlInit()
        except Exception:
            return False
        try:
            h = pynvml.nvmlDeviceGetHandleByUUID(uuid if uuid.startswith("GPU-") else "GPU-" + uuid)
            self.max_mhz = float(pynvml.nvmlDeviceGetMaxClockInfo(h, pynvml.NVML_CLOCK_SM))
            self.reasons_of = getattr(pynvml, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
                pynvml.nvmlDeviceGetCurrentClocksThrottleReasons
            self.reasons_of(h)
            pre = ("nvmlClocksEventReason" if hasattr(pynvml, "nvmlClocksEventReasonHwSlowdown")
                   else "nvmlClocksThrottleReason")
            self.bits = {n: getattr(pynvml, pre + b) for n, b in zip(
                self.NAMES, ("HwSlowdown", "HwThermalSlowdown", "SwThermalSlowdown", "SwPowerCap"))}
        except Exception:
            pynvml.nvmlShutdown()
            return False
        self.nvml, self.handle = pynvml, h
        return True

    def _poll(self):
        nv, h = self.nvml, self.handle
        while not self.halt.is_set():
            t = time.monotonic()
            try:
                sm = float(nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM))
                r = int(self.reasons_of(h))
            except Exception:
                break
            self.rows.append((t, sm, self.max_mhz, {n for n, b in self.bits.items() if r & b}))
            self.first.set()
            self.halt.wait(self.PERIOD_S)

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append((time.monotonic(), line))
            self.first.set()

    def ready(self, timeout=5.0):
        if self.reader is not None:
            self.first.wait(timeout)

    def mark_start(self):
        self.t0 = time.monotonic()

    def mark_end(self):
        self.t1 = time.monotonic()

    def stop(self):
        if self.reader is None:
            return None
        if self.nvml is not None:
            self.halt.set()
            self.reader.join(timeout=5)
            self.nvml.nvmlShutdown()
            rows, source = self.rows, "nvml"
        else:
            time.sleep(0.06)
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
                self.proc.wait()
            self.reader.join(timeout=5)
            rows, source = [], "nvidia-smi"
            for t, line in self.lines:
                f = [x.strip() for x in line.split(",")]
                if len(f) < 9:
                    continue
                try:
                    rows.append((t, float(f[1]), float(f[2]),
                                 {n for n, v in zip(self.NAMES, f[5:9])
                                  if v.lower().startswith("active")}))
                except ValueError:
                    continue
        if not rows:
            return None
        t0 = self.t0 if self.t0 is not None else rows[0][0]
        t1 = self.t1 if self.t1 is not None else rows[-1][0]
        # nvidia-smi lines are stamped when read, a little after they were taken
        slack = 0.05 if source == "nvidia-smi" else 0.0
        inside = [r for r in rows if t0 <= r[0] <= t1 + slack]
        if not inside:  # region shorter than the sampling interval: the nearest sample
            mid = 0.5 * (t0 + t1)
            inside = [min(rows, key=lambda r: abs(r[0] - mid))]
        reasons = set().union(*(r[3] for r in inside))
        return {"sm_mhz": statistics.median(r[1] for r in inside),
                "sm_max_mhz": max(r[2] for r in inside), "samples": len(inside),
                "reasons": sorted(reasons), "source": source}


def make_case(c, seed):
    from scaled_dot_product_bwd_b200.inputs import make_inputs
    return make_inputs(c["B"], c["L"], c["Hq"], c["Hkv"], c["d"], seed=seed,
                       t5_buckets=32 if c["bias"] == "t5" else 0,
                       dense_bias=c["bias"] == "dense", alibi=c["bias"] == "alibi")


# ------------------------------------------------------------------ oracle
def oracle_plan(c):
    """Bounded sample of a workload for the float64 oracle: batch 0, KV head 0
    and `heads` of its query heads; for a forward-only workload longer than
    2048, an evenly spaced set of 1024 query rows (the oracle then forms only
    those rows of S).  The sample's effective FLOPs count its unmasked pairs."""
    G = c["Hq"] // c["Hkv"]
    L = c["L"]
    fwd_only = c.get("fwd_only", False)
    heads = min(G, 2) if fwd_only else (G if L <= 4096 else 1)
    rows = None
    if fwd_only and L > 2048:
        rows = np.unique(np.linspace(0, L - 1, 1024).astype(np.int64))
    return heads, rows


def oracle_sample(c, inp, rows):
    """fwd (+ bwd) of the oracle on the sample's slice of the workload."""
    from oracle import attention_backward, attention_forward
    kw = dict(causal=c["causal"], window_left=c["wl"], window_right=c["wr"],
              bias=inp.bias, t5_table=inp.t5_table, alibi_slopes=inp.alibi_slopes)
    attention_forward(inp.q, inp.k, inp.v, query_rows=rows, **kw)
    if not c.get("fwd_only", False):
        attention_backward(inp.q, inp.k, inp.v, inp.do, **kw)


def sample_pairs(c, rows):
    """Unmasked (i, j) pairs of the sampled query rows of one head."""
    L = c["L"]
    i = np.arange(L, dtype=np.int64) if rows is None else np.asarray(rows, dtype=np.int64)
    lo = np.maximum(0, i - c["wl"]) if c["wl"] >= 0 else np.zeros_like(i)
    hi = np.full_like(i, L - 1)
    if c["causal"]:
        hi = np.minimum(hi, i)
    if c["wr"] >= 0:
        hi = np.minimum(hi, i + c["wr"])
    return int(np.maximum(0, hi - lo + 1).sum())


def time_oracle(c, steps, warmup):
    heads, rows = oracle_plan(c)
    sc = dict(c, B=1, Hq=heads, Hkv=1)
    inp = make_case(sc, 0)
    per = 4 if c.get("fwd_only", False) else 14
    total = per * c["d"] * sample_pairs(c, rows) * heads
    for _ in range(warmup):
        oracle_sample(sc, inp, rows)
    t0 = time.perf_counter()
    for _ in range(steps):
        oracle_sample(sc, inp, rows)
    dt = (time.perf_counter() - t0) / steps
    cores = len(os.sched_getaffinity(0))
    what = "fwd" if c.get("fwd_only", False) else "fwd + bwd"
    rows_txt = "all query rows" if rows is None else f"{len(rows)} evenly spaced query rows"
    sample = (f"{what} of batch 0, KV head 0 with {heads} of its query heads, {rows_txt}, "
              f"of {describe(c)}; float64 numpy, explicit score matrices; effective FLOPs of "
              f"the sample's unmasked pairs")
    return dict(value=total / dt / 1e12, seconds_per_sample=dt, cores=cores, sample=sample,
                flops=total)


def run_reference(args, c):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    r = time_oracle(c, max(1, args.steps), args.warmup)
    line = {
        "impl": "reference", "metric": METRIC, "value": r["value"], "unit": "TFLOP/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": r["seconds_per_sample"] * 1e3, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": f"{args.config}: {describe(c)}", "sample": r["sample"]},
        "cpu_baseline": {"value": r["value"], "unit": "TFLOP/s", "cores": r["cores"],
                         "kind": "oracle", "sample": r["sample"]},
        "e2e": {"value": r["value"], "unit": "TFLOP/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


# ------------------------------------------------------- multi-rank plumbing
def max_over_ranks(value: float, device=None) -> float:
    """The slowest rank's time: all_reduce(MAX) when a process group is up."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return value
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_tflops(world: int, flops_per_rank_step: int, ms_per_step: float) -> float:
    """Weak scaling: every rank runs its own batch; all ranks' FLOPs / slowest time."""
    return world * flops_per_rank_step / (ms_per_step * 1e-3) / 1e12


# --------------------------------------------------------------------- GPU
def run_gpu(args, c):
    import torch
    import torch.distributed as dist

    from scaled_dot_product_bwd_b200 import (BWD_DKDV, BWD_DQ, BWD_PREPROCESS, load_library,
                                             sdpa_bwd, sdpa_bwd_workspace_size, sdpa_fwd,
                                             sdpa_read_device_status)

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=dev)
    load_library()

    inp = make_case(c, seed=rank)
    q, k, v, do = (t.to(dev) for t in (inp.q, inp.k, inp.v, inp.do))
    bias = inp.bias.to(dev) if inp.bias is not None else None
    table = inp.t5_table.to(dev) if inp.t5_table is not None else None
    slopes = inp.alibi_slopes.to(dev) if inp.alibi_slopes is not None else None
    kw = dict(causal=c["causal"], window_left=c["wl"], window_right=c["wr"], bias=bias,
              t5_table=table, alibi_slopes=slopes)
    o = torch.empty_like(q)
    lse = torch.empty(c["B"], c["Hq"], c["L"], device=dev, dtype=torch.float32)
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    ws = torch.empty(sdpa_bwd_workspace_size(q, k), device=dev, dtype=torch.uint8)
    stream = torch.cuda.current_stream(dev)

    fwd_only = c.get("fwd_only", False)
    names = ["fwd"] if fwd_only else ["fwd", "bwd_preprocess", "bwd_dq", "bwd_dkdv"]

    def step(ev=None):
        if ev is not None:
            ev[0].record(stream)
        sdpa_fwd(q, k, v, out=o, lse=lse, **kw)
        if ev is not None:
            ev[1].record(stream)
        if fwd_only:
            return
        sdpa_bwd(q, k, v, o, do, lse, dq=dq, dk=dk, dv=dv, workspace=ws,
                 phases=BWD_PREPROCESS, **kw)
        if ev is not None:
            ev[2].record(stream)
        sdpa_bwd(q, k, v, o, do, lse, dq=dq, dk=dk, dv=dv, workspace=ws, phases=BWD_DQ, **kw)
        if ev is not None:
            ev[3].record(stream)
        sdpa_bwd(q, k, v, o, do, lse, dq=dq, dk=dk, dv=dv, workspace=ws, phases=BWD_DKDV, **kw)
        if ev is not None:
            ev[4].record(stream)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize(dev)
    if sdpa_read_device_status() != 0:
        raise RuntimeError("device status reports a timed-out wait during warm-up")

    # ---------------- timed region: K steps, device-timed, max over ranks
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(len(names) + 1)]
           for _ in range(args.steps)]
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize(dev)
    sampler = ClockSampler(local)
    sampler.ready()
    sampler.mark_start()
    start.record(stream)
    for s in range(args.steps):
        step(evs[s])
    end.record(stream)
    torch.cuda.synchronize(dev)
    sampler.mark_end()
    if world > 1:
        dist.barrier()
    clocks = sampler.stop()
    ms_total = start.elapsed_time(end)
    phase_ms = [statistics.fmean(e[i].elapsed_time(e[i + 1]) for e in evs)
                for i in range(len(names))]
    ms_total = max_over_ranks(ms_total, dev)
    status = sdpa_read_device_status()

    # ---------------- end to end: pinned host buffers, copies inside the timed region.
    # Every step copies its inputs up from pinned host memory and its results
    # (O, LSE, dQ, dK, dV) down again.  Steps are pipelined over three streams
    # and two sets of device buffers: step s+1's inputs go up while step s
    # computes and step s-1's results come down (PCIe runs both directions at
    # once); events order each buffer set's reuse.
    hq_, hk_, hv_, hdo_ = (t.pin_memory() for t in (inp.q, inp.k, inp.v, inp.do))
    ho, hlse = torch.empty_like(hq_).pin_memory(), torch.empty(lse.shape).pin_memory()
    hdq, hdk, hdv = (torch.empty_like(t).pin_memory() for t in (hq_, hk_, hv_))
    ups = (("q", hq_), ("k", hk_), ("v", hv_)) + (() if fwd_only else (("do", hdo_),))
    downs = ((ho, "o"), (hlse, "lse")) + (() if fwd_only else ((hdq, "dq"), (hdk, "dk"),
                                                               (hdv, "dv")))
    h2d = sum(h.numel() * h.element_size() for _, h in ups)
    d2h = sum(h.numel() * h.element_size() for h, _ in downs)
    sets = [dict(q=q, k=k, v=v, do=do, o=o, lse=lse, dq=dq, dk=dk, dv=dv, ws=ws)]
    sets.append({n: torch.empty_like(t) for n, t in sets[0].items()})
    s_up, s_cmp, s_down = (torch.cuda.Stream(dev) for _ in range(3))
    up_done, cmp_done, down_done = ([torch.cuda.Event() for _ in range(2)] for _ in range(3))

    def e2e_run(n_steps):
        for s_i in range(n_steps):
            x = s_i % 2
            S = sets[x]
            with torch.cuda.stream(s_up):
                if s_i >= 2:
                    s_up.wait_event(cmp_done[x])  # step s-2 is done reading these inputs
                for d_, h in ups:
                    S[d_].copy_(h, non_blocking=True)
                up_done[x].record(s_up)
            with torch.cuda.stream(s_cmp):
                s_cmp.wait_event(up_done[x])
                if s_i >= 2:
                    s_cmp.wait_event(down_done[x])  # step s-2's results are copied out
                sdpa_fwd(S["q"], S["k"], S["v"], out=S["o"], lse=S["lse"], **kw)
                if not fwd_only:
                    sdpa_bwd(S["q"], S["k"], S["v"], S["o"], S["do"], S["lse"], dq=S["dq"],
                             dk=S["dk"], dv=S["dv"], workspace=S["ws"], **kw)
                cmp_done[x].record(s_cmp)
            with torch.cuda.stream(s_down):
                s_down.wait_event(cmp_done[x])
                for h, d_ in downs:
                    h.copy_(S[d_], non_blocking=True)
                down_done[x].record(s_down)

    e2e_steps = max(2, min(args.steps, 10))
    e2e_run(min(args.warmup, 2))
    torch.cuda.synchronize(dev)
    if world > 1:
        dist.barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(s_up)
    e2e_run(e2e_steps)
    s_down.wait_stream(s_cmp)
    e1.record(s_down)
    torch.cuda.synchronize(dev)
    e2e_ms = e0.elapsed_time(e1) / e2e_steps
    e2e_ms = max_over_ranks(e2e_ms, dev)

    fl = flop_counts(c)
    step_flops = fl["fwd"] + (0 if fwd_only else fl["bwd"])
    ms_step = ms_total / args.steps
    value = whole_job_tflops(world, step_flops, ms_step)
    peaks = load_peaks()
    peak_src = ("measured bf16 burst / copy bandwidth (MEASURED_PEAKS.json)"
                if peaks["source"] == "measured" else "fallback 1.59 PFLOP/s, 6.65 TB/s")

    # Per kernel: algorithmic FLOPs and HBM bytes per launch against the mean
    # event time, as fractions of the tensor and HBM peaks.  The roofline
    # object is the dominant kernel's, bound by whichever roof is nearer.
    algo = {"fwd": fl["fwd"], "bwd_preprocess": 0, "bwd_dq": fl["bwd_dq"],
            "bwd_dkdv": fl["bwd_dkdv"]}
    nbytes = kernel_bytes(c)
    kernels = {}
    for n, t in zip(names, phase_ms):
        tf = algo[n] / (t * 1e-3) / 1e12
        gbs = nbytes[n] / (t * 1e-3) / 1e9
        kernels[n] = {"ms": round(t, 4), "tflops": round(tf, 1),
                      "frac_tensor": round(tf / peaks["tflops"], 4), "gbs": round(gbs, 1),
                      "frac_hbm": round(gbs / peaks["hbm"], 4), "flops": algo[n],
                      "bytes": nbytes[n]}
    dname = max(kernels, key=lambda n: kernels[n]["ms"])
    kd = kernels[dname]
    hbm_bound = kd["frac_hbm"] > kd["frac_tensor"]
    roofline = {"kernel": dname, "bound": "hbm" if hbm_bound else "tensor",
                "achieved": kd["gbs"] if hbm_bound else kd["tflops"],
                "peak": peaks["hbm"] if hbm_bound else peaks["tflops"],
                "unit": "GB/s" if hbm_bound else "TFLOP/s",
                "frac": kd["frac_hbm"] if hbm_bound else kd["frac_tensor"],
                "traffic": traffic_per_launch(args.config, dname, c["B"]),
                "peak_source": peak_src, "flops_per_launch": kd["flops"],
                "bytes_per_launch": kd["bytes"], "ms_per_launch": kd["ms"]}

    line = {
        "metric": METRIC, "value": round(value, 2), "unit": "TFLOP/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms_step, 4),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic",
        "config": {"workload": f"{args.config}: {describe(c)}", "global_batch": c["B"] * world,
                   "seq_len": c["L"], "parallelism": f"replicas x{world} (batch shards)",
                   "l2": "inputs larger than L2: no flush between steps",
                   "flops_per_step": step_flops, "unmasked_pairs_per_head": fl["P"]},
        "pct_of_peak": round(100 * value / world / peaks["tflops"], 2),
        "value_strict": round(world * (fl["fwd"] + (0 if fwd_only else fl["bwd_strict"]))
                              / (ms_step * 1e-3) / 1e12, 2),
        "kernel_ms": {n: round(t, 4) for n, t in zip(names, phase_ms)},
        "kernels": kernels,
        "roofline": roofline,
        "e2e": {"value": round(whole_job_tflops(world, step_flops, e2e_ms), 2), "unit": "TFLOP/s",
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                "ms_per_step": round(e2e_ms, 3),
                "pipelining": "3 streams, 2 device buffer sets: H2D(s+1) | compute(s) | D2H(s-1)"},
        "gpu_launches": len(names) * args.steps,
        "clocks": clocks,
        "device_status": status,
    }
    if world > 1:
        dist.destroy_process_group()
    if rank == 0:
        if world == 1 and not args.no_cpu_baseline:
            r = time_oracle(c, 1, 0)
            line["cpu_baseline"] = {"value": r["value"], "unit": "TFLOP/s", "cores": r["cores"],
                                    "kind": "oracle", "sample": r["sample"]}
        print(json.dumps(line), flush=True)
    return 0


def visited_tile_pairs(c):
    """(query tile, key tile) pairs of one head that hold a visible (i, j)."""
    L, n = c["L"], (c["L"] + 127) // 128
    count = 0
    for mi in range(n):
        i0, i1 = mi * 128, min(L, mi * 128 + 128) - 1
        lo = max(0, i0 - c["wl"]) if c["wl"] >= 0 else 0
        hi = L - 1
        if c["causal"]:
            hi = min(hi, i1)
        if c["wr"] >= 0:
            hi = min(hi, i1 + c["wr"])
        if hi >= lo:
            count += hi // 128 - lo // 128 + 1
    return count


def bias_grad_extra_bytes(c):
    """HBM bytes the bias gradient adds to the backward.  A dense bias: the
    fp32 dS written once (full shape), or written and read back by the
    broadcast reduction.  T5: the dQ kernel's per-bucket sums (8 warps x 32
    buckets per (batch, head, query tile)) written and read back once, then
    the result.  ALiBi: the dQ kernel's
    per-warp sums of |j - i| dS (8 floats per visited tile pair) written and
    read back once, then the result."""
    B, H, L = c["B"], c["Hq"], c["L"]
    if c["bias"] == "t5":
        nt = (L + 127) // 128
        return 2 * B * H * nt * 8 * 32 * 4 + 32 * H * 4
    if c["bias"] == "alibi":
        tiles = B * H * visited_tile_pairs(c)
        return 2 * tiles * 8 * 4 + H * 4
    return B * H * L * L * 4       # a full-shape dense bias: dS goes straight out


def bias_grad_launches(c):
    """Kernels one timed step of the bias-gradient leg launches: the forward,
    preprocess, the dQ kernel (storing dS, its diagonal sums or its |j - i|
    moments) and the dK/dV kernel; a dense bias under a mask adds the zero
    fill of skipped key tiles; T5 adds the per-(bucket, head) sum of the
    per-bucket sums, ALiBi the per-head sum of the moments."""
    n = 4
    if c["bias"] in ("t5", "alibi"):
        return n + 1
    if c["causal"] or c["wl"] >= 0 or c["wr"] >= 0:
        n += 1
    return n


def run_bias_grad(args, c):
    import torch

    from scaled_dot_product_bwd_b200 import (load_library, sdpa_bwd, sdpa_bwd_bias_grad,
                                             sdpa_bwd_bias_grad_workspace_size,
                                             sdpa_bwd_workspace_size, sdpa_fwd,
                                             sdpa_read_device_status)
    if c["bias"] == "none":
        raise SystemExit("--bias-grad needs a workload with a bias")
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    load_library()
    inp = make_case(c, seed=0)
    q, k, v, do = (t.to(dev) for t in (inp.q, inp.k, inp.v, inp.do))
    bias = inp.bias.to(dev) if inp.bias is not None else None
    table = inp.t5_table.to(dev) if inp.t5_table is not None else None
    slopes = inp.alibi_slopes.to(dev) if inp.alibi_slopes is not None else None
    kw = dict(causal=c["causal"], window_left=c["wl"], window_right=c["wr"], bias=bias,
              t5_table=table, alibi_slopes=slopes)
    o = torch.empty_like(q)
    lse = torch.empty(c["B"], c["Hq"], c["L"], device=dev, dtype=torch.float32)
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    ref = next(x for x in (bias, table, slopes) if x is not None)
    dbias = torch.empty_strided(ref.shape, ref.stride(), device=dev, dtype=torch.float32)
    ws = torch.empty(sdpa_bwd_workspace_size(q, k), device=dev, dtype=torch.uint8)
    wsg = torch.empty(max(256, sdpa_bwd_bias_grad_workspace_size(
        q, k, bias=bias, t5_table=table, alibi_slopes=slopes)), device=dev, dtype=torch.uint8)
    stream = torch.cuda.current_stream(dev)

    def step(grad, ev=None):
        if ev is not None:
            ev[0].record(stream)
        sdpa_fwd(q, k, v, out=o, lse=lse, **kw)
        if ev is not None:
            ev[1].record(stream)
        if grad:
            sdpa_bwd_bias_grad(q, k, v, o, do, lse, dq=dq, dk=dk, dv=dv, dbias=dbias,
                               workspace=wsg, **kw)
        else:
            sdpa_bwd(q, k, v, o, do, lse, dq=dq, dk=dk, dv=dv, workspace=ws, **kw)
        if ev is not None:
            ev[2].record(stream)

    res = {}
    for grad in (False, True):
        for _ in range(args.warmup):
            step(grad)
        torch.cuda.synchronize(dev)
        evs = [[torch.cuda.Event(enable_timing=True) for _ in range(3)]
               for _ in range(args.steps)]
        sampler = ClockSampler(0) if grad else None
        if sampler is not None:
            sampler.ready()
            sampler.mark_start()
        for s_i in range(args.steps):
            step(grad, evs[s_i])
        torch.cuda.synchronize(dev)
        if sampler is not None:
            sampler.mark_end()
        clocks = sampler.stop() if sampler is not None else None
        res[grad] = dict(fwd=statistics.fmean(e[0].elapsed_time(e[1]) for e in evs),
                         bwd=statistics.fmean(e[1].elapsed_time(e[2]) for e in evs),
                         clocks=clocks)
    status = sdpa_read_device_status()
    fl = flop_counts(c)
    step_flops = fl["fwd"] + fl["bwd"]
    ms_step = res[True]["fwd"] + res[True]["bwd"]
    extra_ms = res[True]["bwd"] - res[False]["bwd"]
    extra = bias_grad_extra_bytes(c)
    peaks = load_peaks()
    ach = extra / (extra_ms * 1e-3) / 1e9 if extra_ms > 0 else None
    line = {
        "metric": METRIC + ", backward with the bias gradient",
        "value": round(step_flops / (ms_step * 1e-3) / 1e12, 2), "unit": "TFLOP/s", "n_gpus": 1,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms_step, 4),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic",
        "config": {"workload": f"{args.config}: {describe(c)}, with bias gradient",
                   "global_batch": c["B"], "seq_len": c["L"], "parallelism": "replicas x1",
                   "l2": "inputs larger than L2: no flush between steps",
                   "flops_per_step": step_flops},
        "kernel_ms": {"fwd": round(res[True]["fwd"], 4),
                      "bwd_bias_grad": round(res[True]["bwd"], 4),
                      "bwd_plain": round(res[False]["bwd"], 4)},
        "bias_grad_extra_ms": round(extra_ms, 4),
        "roofline": {"kernel": "bias-gradient extra (dS, its partial sums, reductions)", "bound": "hbm",
                     "achieved": None if ach is None else round(ach, 1),
                     "peak": peaks["hbm"], "unit": "GB/s",
                     "frac": None if ach is None else round(ach / peaks["hbm"], 4),
                     "traffic": bias_grad_traffic(args.config, c["B"]), "bytes_per_step": extra,
                     "peak_source": "measured copy bandwidth (MEASURED_PEAKS.json)"
                     if peaks["source"] == "measured" else "fallback 6.65 TB/s"},
        "gpu_launches": args.steps * bias_grad_launches(c),
        "clocks": res[True]["clocks"],
        "device_status": status,
    }
    print(json.dumps(line), flush=True)
    return 0


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=30)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--config", default="mistral4k", choices=sorted(CONFIGS))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--bias-grad", action="store_true")
    args = ap.parse_args()
    c = CONFIGS[args.config]
    if args.impl == "reference":
        return run_reference(args, c)
    if args.bias_grad:
        return run_bias_grad(args, c)
    return run_gpu(args, c)


if __name__ == "__main__":
    sys.exit(main())
