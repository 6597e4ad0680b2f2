#!/usr/bin/env python
"""Benchmark of the AWQ per-layer scale search on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload NAME]

One step is one pass of the whole per-layer path over one synthetic workload:
activation statistic of every distinct layer input -> alpha grid search of
every linear (scale table, per-alpha bf16 operand, the fused tensor-core loss
GEMM, loss reduction + argmin) -> s* = a^alpha* -> final quantise + pack.

The default workload is the 70B-shaped decoder block: seven linears (q/o
8192 x 8192, k/v 8192 x 1024, gate/up 8192 x 28672, down 28672 x 8192) on four
inputs of N = 4096 tokens, 21 alphas, 4-bit g128, all seven searched by one
``awq_search_batched`` call.  ``value`` is alpha-candidates per second over
all linears (7 x 21 per step).  The same line carries one sub-object per other
workload (``configs``: the 512 x 512 layer, the LLaMA-7B attention and MLP
down projections, the bit-width / group sweep), each with its own step time
and roofline.

Multi-GPU (launched with torchrun, one rank per GPU): every rank quantises its
own independent block (different seeds) -- layers are searched independently,
so there is no collective on the data path; `value` is the aggregate
alpha-candidates/s of all ranks, timed as the max over ranks.

--impl reference times the CPU oracle (oracle/) on the host cores, on a bounded
sample of the same workload per step (a few output columns of every linear at
one alpha each); rank 0 alone runs it.

Prints one JSON line (rank 0).
"""
from __future__ import annotations

import argparse
import gc
import hashlib
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time
from dataclasses import dataclass
from typing import List, Tuple

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "AWQ search α-candidates/s per layer; eff. TFLOP/s and % of B200 bf16 peak"
UNIT = "alpha-candidates/s"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
SUB_CONFIGS = ("linear_512_n256", "llama7b_attn_proj", "llama7b_mlp_down", "sweep_4096x11008_n16k")
# kernels per profiled stage: the loss reduction is two launches (column sums, final sum + argmin)
KERNELS_PER_STAGE = {"loss_reduce": 2}


def parse_args():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=("ours", "reference"), default="ours")
    ap.add_argument("--workload", default="llama70b_block")
    ap.add_argument("--flush-mib", type=int, default=512)
    ap.add_argument("--cpu-seconds", type=float, default=15.0,
                    help="target CPU time of the oracle baseline sample")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-configs", action="store_true", help="skip the per-workload sub-objects")
    ap.add_argument("--no-clip", action="store_true", help="skip timing the weight-clipping search")
    ap.add_argument("--no-gram", action="store_true", help="skip timing the Gram form of the search")
    ap.add_argument("--no-w4a16", action="store_true", help="skip timing the W4A16 consumer kernel")
    ap.add_argument("--no-e2e", action="store_true", help="skip the host-to-host measurement")
    ap.add_argument("--loss-form", choices=("error", "reference"), default="error")
    return ap.parse_args()


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def source_hash() -> str:
    h = hashlib.sha1()
    for name in ("search.cu", "ptx.cuh"):
        with open(os.path.join(ROOT, "post_weight_only_b200", "csrc", name), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def committed_traffic(workload: str):
    """DRAM bytes of the search GEMM per step of `workload` from the committed
    ncu summary, if it was taken on the current kernel source (else None)."""
    path = os.path.join(ROOT, "profiles", "search_gemm_traffic.json")
    if not os.path.exists(path):
        return None
    with open(path) as f:
        d = json.load(f)
    if d.get("kernel_source_sha1_16") != source_hash():
        return None
    entry = d.get("workloads", {}).get(workload)
    if entry is None and d.get("workload") == workload:
        entry = d
    return entry


class ClockSampler:
    """nvidia-smi clocks and throttle reasons, sampled every 20 ms around the
    timed region; only the samples taken inside the region (by their
    timestamps against the host clock at its start and end) are reported."""
    FIELDS = ("timestamp,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.path = None
        self.t0 = self.t1 = None

    def start(self):
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.index}", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "20"], stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None
        time.sleep(0.3)

    def mark_start(self):
        self.t0 = time.time()

    def mark_end(self):
        self.t1 = time.time()

    @staticmethod
    def _stamp(text):
        import datetime
        for fmt in ("%Y/%m/%d %H:%M:%S.%f", "%Y/%m/%d %H:%M:%S"):
            try:
                return datetime.datetime.strptime(text, fmt).timestamp()
            except ValueError:
                pass
        return None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        time.sleep(0.1)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        rows = []
        with open(self.path) as f:
            for line in f:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) >= 9:
                    rows.append(parts)
        os.unlink(self.path)

        def num(x):
            try:
                return float(x)
            except ValueError:
                return None
        inside = [r for r in rows if (t := self._stamp(r[0])) is not None and self.t0 is not None
                  and self.t0 - 0.02 <= t <= self.t1 + 0.02]
        use = inside or rows
        sm = [v for r in use if (v := num(r[1])) is not None]
        smax = [v for r in rows if (v := num(r[2])) is not None]
        power = [v for r in use if (v := num(r[3])) is not None]
        names = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")
        reasons = sorted({names[i] for r in use for i in range(4) if r[5 + i].lower().startswith("active")})
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(smax) if smax else None,
                "power_w_max": max(power) if power else None,
                "samples": len(use), "samples_in_timed_region": len(inside),
                "interval_ms": 20, "reasons": reasons}


# ----------------------------------------------------------------------------- workloads as jobs
@dataclass
class Search:
    x: int              # index into Job.xs
    w: int              # index into Job.ws
    bits: int
    group: int
    name: str


@dataclass
class Job:
    """One workload as the bench runs it: its distinct layer inputs, its
    weights, and the searches (input, weight, bits, group) of one step."""
    name: str
    xs: list            # XSpec-backed (N, D_in, spec)
    ws: list            # (D_in, D_out, std, seed)
    searches: List[Search]
    alphas: list        # float alpha grid

    @property
    def A(self) -> int:
        return len(self.alphas)

    def dims(self, s: Search) -> Tuple[int, int, int]:
        N, D_in, _ = self.xs[s.x]
        return N, D_in, self.ws[s.w][1]

    def flops(self) -> float:
        """alpha-GEMM flops of one step (2 N D_in D_out per alpha and linear)."""
        return sum(self.A * 2.0 * n * k * m for n, k, m in (self.dims(s) for s in self.searches))

    def units(self) -> int:
        return self.A * len(self.searches)


def make_job(name: str, rank: int = 0) -> Job:
    """The workload's inputs (seeds offset by 1000 per rank beyond rank 0)."""
    from post_weight_only_b200 import synth
    wl = synth.workload(name)
    off = 1000 * rank
    xs, ws, searches, xkey, wkey = [], [], [], {}, {}

    def x_index(N, D_in, spec):
        key = (spec.kind, spec.seed, spec.n_outlier, N, D_in)
        if key not in xkey:
            xkey[key] = len(xs)
            xs.append((N, D_in, synth.XSpec(spec.kind, spec.n_outlier, spec.lo, spec.hi, spec.seed + off)))
        return xkey[key]

    def w_index(D_in, D_out, std, seed):
        key = (D_in, D_out, std, seed)
        if key not in wkey:
            wkey[key] = len(ws)
            ws.append((D_in, D_out, std, seed + off))
        return wkey[key]

    for bits, group in wl.quant:
        for L in wl.layers:
            searches.append(Search(x_index(L.N, L.D_in, L.x), w_index(L.D_in, L.D_out, L.w_std, L.w_seed),
                                   bits, group, f"{L.name}_b{bits}g{group}"))
    return Job(name, xs, ws, searches, synth.alpha_grid(wl.n_intervals).tolist())


def host_inputs(job: Job):
    """(list of X bf16, list of W fp32) on the CPU, from the seeded generators."""
    from post_weight_only_b200 import synth
    X = [synth.make_x(N, D_in, spec) for N, D_in, spec in job.xs]
    W = [synth.make_w(D_in, D_out, std, seed) for D_in, D_out, std, seed in job.ws]
    return X, W


def stats_bytes(job: Job) -> int:
    return sum(N * D_in * 2 + D_in * 4 for N, D_in, _ in job.xs)


def pack_bytes(job: Job) -> int:
    tot = 0
    for s in job.searches:
        _, D_in, D_out = job.dims(s)
        tot += D_in * D_out * 4 + D_in * 4 + (D_in // 8) * D_out * 4 + (D_in // s.group) * D_out * 4
    return tot


def operand_bytes(job: Job) -> int:
    """W once, s and 1/s per alpha, the bf16 operand per alpha, per search."""
    tot = 0
    for s in job.searches:
        _, D_in, D_out = job.dims(s)
        tot += D_in * D_out * 4 + job.A * D_in * 8 + job.A * D_in * D_out * 2
    return tot


def config_of(job: Job, world: int, loss_form: str = "error"):
    c = {"workload": job.name, "n_alpha": job.A, "loss_form": loss_form,
         "linears": [{"name": s.name, "N": job.dims(s)[0], "D_in": job.dims(s)[1], "D_out": job.dims(s)[2],
                      "bits": s.bits, "group": s.group} for s in job.searches],
         "flops_per_step": job.flops(),
         "parallelism": f"{world} independent workload(s), one per GPU",
         "l2": "flushed between timed steps: 512 MiB write, then a read of it (no dirty lines left)"}
    if len(job.searches) == 1:
        N, D_in, D_out = job.dims(job.searches[0])
        c.update({"N": N, "D_in": D_in, "D_out": D_out, "bits": job.searches[0].bits,
                  "group": job.searches[0].group})
    return c


# ----------------------------------------------------------------------------- the CPU oracle on a sample
def oracle_rate(job: Job, X, W, cols_per_search: int, alphas_per_search: int, step: int = 0):
    """Time the oracle on a sample of the job and extrapolate to the whole job.

    For every search: `cols_per_search` evenly spaced output columns (shifted
    by `step`) at `alphas_per_search` alphas (rotated by `step`), one oracle
    call.  The oracle runs one column per OpenMP thread, so the whole search's
    wall time is the sample's times (D_out / columns) x (A / alphas).
    Returns (alpha-candidates/s of the whole job, sample seconds, whole-job
    estimate seconds)."""
    import numpy as np
    import oracle
    a = [oracle.act_stats(x).astype(np.float32) for x in X]
    sample_s = est_s = 0.0
    alphas = np.array(job.alphas, dtype=np.float32)
    for si, s in enumerate(job.searches):
        _, _, D_out = job.dims(s)
        nc = max(1, min(cols_per_search, D_out))
        cols = (np.arange(nc, dtype=np.int64) * (D_out // nc) + step * 7 + si) % D_out
        na = max(1, min(alphas_per_search, job.A))
        sub = alphas[[(step + si + k) % job.A for k in range(na)]]
        t0 = time.perf_counter()
        oracle.search(X[s.x], W[s.w], a[s.x], sub, s.bits, s.group, cols=np.unique(cols))
        dt = time.perf_counter() - t0
        sample_s += dt
        est_s += dt * (D_out / len(np.unique(cols))) * (job.A / na)
    return job.units() / est_s, sample_s, est_s


def cpu_baseline(job: Job, X, W, target_s: float):
    """The oracle as it stands on a bounded sample of the job on this host's
    cores: one column per thread of every search, as many alphas as fit in
    about target_s seconds."""
    import oracle
    nt = max(1, oracle.num_threads())
    _, probe_s, _ = oracle_rate(job, X, W, nt, 1)
    na = max(1, min(job.A, int(target_s / max(probe_s, 1e-3))))
    value, sample_s, est_s = oracle_rate(job, X, W, nt, na, step=1)
    return {"value": value, "unit": UNIT, "cores": nt, "kind": "oracle",
            "sample": f"{nt} output columns (one per thread) x {na} of {job.A} alphas of each of the "
                      f"{len(job.searches)} searches (full N and D_in), {sample_s:.1f} s; the whole job is "
                      f"extrapolated by columns and alphas to {est_s:.0f} s on {nt} threads"}


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    import oracle
    job = make_job(args.workload)
    X, W = host_inputs(job)
    nt = max(1, oracle.num_threads())
    # size one step so that the whole run stays within a few minutes
    budget = min(4.0, 150.0 / max(1, args.steps + args.warmup))
    _, probe_s, _ = oracle_rate(job, X, W, nt, 1)
    cols = nt if probe_s <= budget else max(1, int(nt * budget / probe_s))
    for k in range(args.warmup):
        oracle_rate(job, X, W, cols, 1, step=k)
    est, times = [], []
    for k in range(args.steps):
        _, dt, e = oracle_rate(job, X, W, cols, 1, step=args.warmup + k)
        times.append(dt)
        est.append(e)
    value = job.units() / (sum(est) / len(est))
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * sum(times) / len(times),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic (seeded; no dataset or weights)", "config": config_of(job, 1),
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": nt, "kind": "oracle",
                         "sample": f"each step: {cols} output columns x 1 alpha (rotating) of each of the "
                                   f"{len(job.searches)} searches (full N and D_in); value extrapolated to "
                                   "whole-job alpha-candidates by columns and alphas"},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


# ----------------------------------------------------------------------------- the CUDA path
class DeviceJob:
    """A job's inputs resident on the device and its one-step pipeline."""

    def __init__(self, job: Job, X, W, dev, form):
        from post_weight_only_b200 import awq
        self.awq = awq
        self.job = job
        self.form = form
        self.xs = [x.to(dev) for x in X]
        self.ws = [w.to(dev) for w in W]
        self.workspace = awq.Workspace()
        # searches grouped by quantiser setting: one call per setting (batched when several)
        self.groups = {}
        for i, s in enumerate(job.searches):
            self.groups.setdefault((s.bits, s.group), []).append(i)

    def step(self):
        """statistic of every input -> search of every linear -> s* -> pack.
        No host synchronisation; returns the per-search results."""
        awq, job = self.awq, self.job
        a = awq.act_stats_batched(self.xs) if len(self.xs) > 1 else [awq.act_stats(self.xs[0])]
        out = [None] * len(job.searches)
        for (bits, group), idx in self.groups.items():
            if len(idx) == 1:
                s = job.searches[idx[0]]
                res = [awq.search(self.xs[s.x], self.ws[s.w], a[s.x], job.alphas, bits, group,
                                  workspace=self.workspace, check_status=False, loss_form=self.form)]
            else:
                res = awq.search_batched([(self.xs[job.searches[i].x], self.ws[job.searches[i].w],
                                           a[job.searches[i].x]) for i in idx], job.alphas, bits, group,
                                         workspace=self.workspace, loss_form=self.form, check_status=False)
            for i, r in zip(idx, res):
                s = job.searches[i]
                s_star = awq.scales(a[s.x], r.alpha_star)
                packed, sc = awq.quantize_pack(self.ws[s.w], s_star, bits, group)
                out[i] = (r, s_star, packed, sc)
        return out

    def check(self, out):
        for r, *_ in out:
            self.awq.check_device_status(r.status)


def timed_steps(dj: DeviceJob, steps: int, warmup: int, flush, flush_sink, barrier=None, clocks=None):
    """Warm up, then time `steps` steps with CUDA events on the launching
    stream, L2 flushed before each; the library's per-stage event timings are
    collected over the same region."""
    import torch
    awq = dj.awq
    out = None
    for _ in range(warmup):
        out = dj.step()
    torch.cuda.synchronize()
    if out is not None:
        dj.check(out)
    if clocks:
        clocks.start()
    awq.profile_enable(True)
    awq.profile_reset()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
    (barrier or torch.cuda.synchronize)()
    if clocks:
        clocks.mark_start()
    for k in range(steps):
        # Evict the inputs from L2 before every step: write a buffer larger
        # than L2, then read it back so that the write-back of its dirty lines
        # happens here and not inside the step.
        flush.zero_()
        flush_sink.add_(flush.amax())
        ev[k][0].record()
        out = dj.step()
        ev[k][1].record()
    (barrier or torch.cuda.synchronize)()
    if clocks:
        clocks.mark_end()
    clk = clocks.stop() if clocks else None
    prof = awq.profile_read()
    awq.profile_enable(False)
    dj.check(out)
    step_ms = [a.elapsed_time(b) for a, b in ev]
    return out, step_ms, prof, clk


SUSTAINED_MS = 500.0


def roofline_of(job: Job, prof, steps: int, timed_ms: float):
    """The search GEMM's roofline over the timed region: the alpha-GEMM flops
    of all its launches over their summed CUDA-event durations.  A region of
    at least half a second of back-to-back GEMMs is the sustained regime (the
    power-capped cuBLAS loop: under the 1 kW cap the clocks settle within tens
    of milliseconds), a shorter one the burst regime."""
    peaks, src = load_peaks()
    gemm_ms, gemm_n = prof["search_gemm"]
    flops = job.flops() * steps
    achieved = flops / (gemm_ms / 1e3) / 1e12
    burst = float(peaks["bf16_tflops"])
    sustained = float(peaks.get("bf16_tflops_sustained", burst))
    regime = "sustained" if timed_ms >= SUSTAINED_MS else "burst"
    peak = sustained if regime == "sustained" else burst
    tr = committed_traffic(job.name)
    launches_per_step = gemm_n / max(steps, 1)
    roof = {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s", "frac": achieved / peak,
            "peak_source": f"{src} bf16 dense, {regime} (cuBLAS), from MEASURED_PEAKS.json" if src == "measured"
            else "fallback 1.59 PFLOP/s burst / 1.4 sustained",
            "frac_of_burst": achieved / burst, "frac_of_sustained": achieved / sustained,
            "regime": regime, "timed_region_ms": timed_ms,
            "kernel": "search_kernel (fused per-alpha loss GEMM)",
            "launches_per_step": launches_per_step,
            "avg_launch_ms": gemm_ms / max(gemm_n, 1),
            "flops_per_launch": job.flops() / max(launches_per_step, 1),
            "traffic": None if tr is None else tr["dram_bytes_per_launch"]}
    if tr is not None:
        roof["traffic_note"] = tr.get("note", "")
    return roof


def hbm_in_step(prof, stage: str, nbytes_per_step: int, steps: int):
    ms, n = prof[stage]
    if n == 0:
        return None
    peaks, _ = load_peaks()
    per_step = ms / steps
    gbs = nbytes_per_step / (per_step / 1e3) / 1e9
    return {"ms_per_step": per_step, "launches_per_step": n / steps, "algorithmic_bytes_per_step": nbytes_per_step,
            "achieved_gbs": gbs, "peak_gbs": float(peaks["hbm_gbs"]), "frac": gbs / float(peaks["hbm_gbs"]),
            "timing": "events around each launch inside the timed steps"}


def launches_of(prof) -> int:
    return sum(n * KERNELS_PER_STAGE.get(name, 1) for name, (_, n) in prof.items())


def measure_job(job: Job, dev, steps: int, warmup: int, flush, flush_sink, form, barrier=None, clocks=None,
                host=None):
    """Device-resident timing of one job; returns (summary dict, DeviceJob, host inputs, last outputs)."""
    X, W = host if host is not None else host_inputs(job)
    dj = DeviceJob(job, X, W, dev, form)
    out, step_ms, prof, clk = timed_steps(dj, steps, warmup, flush, flush_sink, barrier, clocks)
    total = sum(step_ms)
    ms = total / steps
    peaks, _ = load_peaks()
    summary = {
        "ms_per_step": ms, "steps": steps, "warmup": warmup, "value": job.units() / (ms / 1e3), "unit": UNIT,
        "eff_tflops": job.flops() / (ms / 1e3) / 1e12,
        "pct_bf16_peak_step": job.flops() / (ms / 1e3) / 1e12 / float(peaks["bf16_tflops"]),
        "roofline": roofline_of(job, prof, steps, total),
        "hbm_kernels": {"act_stats": hbm_in_step(prof, "act_stats", stats_bytes(job), steps),   # one launch per step
                        "quantize_pack": hbm_in_step(prof, "quantize_pack", pack_bytes(job), steps),
                        "search_operand": hbm_in_step(prof, "search_operand", operand_bytes(job), steps)},
        "kernels": {name: {"total_ms": t, "launches": n} for name, (t, n) in prof.items() if n},
        "gpu_launches": launches_of(prof),
        "alpha_star": {job.searches[i].name: float(r.alpha_star.item()) for i, (r, *_) in enumerate(out)},
    }
    if clk is not None:
        summary["clocks"] = clk
    return summary, dj, (X, W), out


def per_search_times(dj: DeviceJob, reps: int = 3):
    """Each search of the job alone (same inputs, L2 not flushed): the GEMM's
    share per linear, to see which layer shapes leave the tensor pipe idle."""
    import torch
    awq, job = dj.awq, dj.job
    a = [awq.act_stats(x) for x in dj.xs]
    out = {}
    peaks, _ = load_peaks()
    for s in job.searches:
        N, D_in, D_out = job.dims(s)
        awq.search(dj.xs[s.x], dj.ws[s.w], a[s.x], job.alphas, s.bits, s.group, workspace=dj.workspace,
                   check_status=False, loss_form=dj.form)
        torch.cuda.synchronize()
        awq.profile_enable(True)
        awq.profile_reset()
        for _ in range(reps):
            r = awq.search(dj.xs[s.x], dj.ws[s.w], a[s.x], job.alphas, s.bits, s.group, workspace=dj.workspace,
                           check_status=False, loss_form=dj.form)
        prof = awq.profile_read()
        awq.profile_enable(False)
        awq.check_device_status(r.status)
        g_ms = prof["search_gemm"][0] / reps
        flops = job.A * 2.0 * N * D_in * D_out
        out[s.name] = {"gemm_ms": g_ms, "operand_ms": prof["search_operand"][0] / reps,
                       "other_ms": (prof["scale_table"][0] + prof["loss_reduce"][0]) / reps,
                       "gemm_tflops": flops / (g_ms / 1e3) / 1e12,
                       "gemm_frac_of_burst": flops / (g_ms / 1e3) / 1e12 / float(peaks["bf16_tflops"])}
    return out


def e2e_of(job: Job, X, W, dev, steps: int, warmup: int, form, max_over_ranks):
    """The same metric through the public host-to-host calls: pinned host
    inputs in, host results out, copies inside the timed region."""
    import torch
    from post_weight_only_b200 import awq
    Xh = [x.pin_memory() for x in X]
    Wh = [w.pin_memory() for w in W]
    h2d = sum(t.numel() * t.element_size() for t in Xh + Wh)
    times = []
    if len(job.searches) == 1:
        s = job.searches[0]
        ws = awq.Workspace()
        out = None
        for k in range(warmup + steps):
            torch.cuda.synchronize()
            t0 = time.perf_counter()
            out = awq.quantize_layer_host(Xh[s.x], Wh[s.w], job.alphas, s.bits, s.group, device=dev, workspace=ws,
                                          out=out, loss_form=form)
            if k >= warmup:
                times.append((time.perf_counter() - t0) * 1e3)
        d2h = sum(t.numel() * t.element_size() for t in out.values())
        api = "awq.quantize_layer_host"
    elif len({(s.bits, s.group) for s in job.searches}) == 1:
        bits, group = job.searches[0].bits, job.searches[0].group
        layers = [(s.x, Wh[s.w]) for s in job.searches]
        ws = awq.Workspace()
        state = awq.BlockHostState()
        res = None
        for k in range(warmup):
            res = awq.quantize_block_host(Xh, layers, job.alphas, bits, group, device=dev, workspace=ws,
                                          state=state, loss_form=form)
        # The timed steps as one stream of blocks: each call queues the next
        # step's upload (its own copy of the same host inputs) behind its own
        # work; the first timed call uploads its own inputs and the last queues
        # nothing, so the region holds exactly one upload and one download per
        # step.  One wall-clock region from the first call to the last result.
        torch.cuda.synchronize()
        t0 = time.perf_counter()
        for k in range(steps):
            res = awq.quantize_block_host(Xh, layers, job.alphas, bits, group, device=dev, workspace=ws,
                                          state=state, loss_form=form,
                                          prefetch=(Xh, layers) if k + 1 < steps else None)
        torch.cuda.synchronize()
        times.append((time.perf_counter() - t0) * 1e3)
        d2h = sum(t.numel() * t.element_size() for r in res for t in r.values())
        api = ("awq.quantize_block_host, each call queueing the next step's upload behind its own work "
               "(prefetch); copy stream for inputs, per-layer awq_search, result stream")
        del state
    else:
        return None
    per = max_over_ranks(sum(times)) / steps
    return {"value": job.units() / (per / 1e3), "unit": UNIT, "ms_per_step": per, "h2d_bytes_per_step": h2d,
            "d2h_bytes_per_step": d2h, "api": api}


def run_ours(args):
    import torch
    from post_weight_only_b200 import awq, synth

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    dist = None
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300), device_id=dev)

    def barrier():
        if dist is not None:
            dist.barrier()
        torch.cuda.synchronize()

    def max_over_ranks(x: float) -> float:
        if dist is None:
            return x
        t = torch.tensor([x], dtype=torch.float64, device=dev)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        return float(t.item())

    form = awq.LOSS_ERROR if args.loss_form == "error" else awq.LOSS_REFERENCE
    flush = torch.empty(args.flush_mib << 20, dtype=torch.uint8, device=dev)
    flush_sink = torch.zeros((), dtype=torch.uint8, device=dev)

    # ---------------- the headline: device-resident timed region
    job = make_job(args.workload, rank)
    X, W = host_inputs(job)
    clocks = ClockSampler(local)
    head, dj, _, out = measure_job(job, dev, args.steps, args.warmup, flush, flush_sink, form, barrier=barrier,
                                   clocks=clocks, host=(X, W))
    total_ms = max_over_ranks(head["ms_per_step"] * args.steps)
    ms_per_step = total_ms / args.steps
    value = job.units() * world / (ms_per_step / 1e3)
    per_layer = per_search_times(dj) if len(job.searches) > 1 else None
    del dj, out
    torch.cuda.empty_cache()

    # ---------------- end to end: host buffers in, host results out
    e2e = None if args.no_e2e else e2e_of(job, X, W, dev, args.steps, min(args.warmup, 2), form, max_over_ranks)
    if e2e is not None:
        e2e["value"] *= world
    torch.cuda.empty_cache()

    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic (seeded; no dataset or weights)",
        "config": config_of(job, world, args.loss_form),
        "eff_tflops": job.flops() * world / (ms_per_step / 1e3) / 1e12,
        "pct_bf16_peak_step": head["pct_bf16_peak_step"],
        "roofline": head["roofline"],
        "hbm_kernels": head["hbm_kernels"],
        "kernels": head["kernels"],
        "per_linear_search": per_layer,
        "e2e": e2e,
        "gpu_launches": head["gpu_launches"],
        "clocks": head.get("clocks"),
        "alpha_star": head["alpha_star"],
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(job, X, W, args.cpu_seconds)
    del X, W

    # ---------------- the other workloads, one sub-object each
    configs = {}
    if not args.no_configs and world == 1:
        for name in SUB_CONFIGS:
            if name == args.workload:
                continue
            sub = make_job(name, rank)
            if sub.name == "sweep_4096x11008_n16k":
                steps_c, warm_c = 3, 1
            else:
                ms_guess = sub.flops() / 1.2e15 * 1e3 + 0.05
                steps_c, warm_c = max(5, min(50, int(200.0 / ms_guess))), 3
            summary, dj_c, _, _ = measure_job(sub, dev, steps_c, warm_c, flush, flush_sink, form)
            summary["config"] = config_of(sub, 1, args.loss_form)
            if len(sub.searches) > 1:
                summary["per_search"] = per_search_times(dj_c, reps=1)
            configs[name] = summary
            del dj_c
            torch.cuda.empty_cache()
    line["configs"] = configs or None

    # ---------------- the weight-clipping search that follows the scale search
    # (not part of the step): the 4096^2 layer at s*, 21 ratios from 1 down to 0.5
    if not args.no_clip and world == 1:
        line["clip_search"] = clip_section(dev, flush, flush_sink)
    # ---------------- the Gram form of the search on the 16384-token sweep layer
    if not args.no_gram and world == 1:
        line["gram_search"] = gram_section(dev, flush, flush_sink)
    # ---------------- the W4A16 consumer of the pack format
    if not args.no_w4a16 and world == 1:
        line["w4a16"] = w4a16_section(dev, rank)

    if rank == 0:
        print(json.dumps(line), flush=True)
    if dist is not None:
        dist.barrier()
        dist.destroy_process_group()


def clip_section(dev, flush, flush_sink):
    import torch
    from post_weight_only_b200 import awq, synth
    spec = synth.workload("llama7b_attn_proj").layers[0]
    X_cpu, W_cpu = synth.layer_inputs(spec)
    X, W = X_cpu.to(dev), W_cpu.to(dev)
    bits, group = 4, 128
    alphas = synth.alpha_grid(20).tolist()
    r = awq.quantize_layer(X, W, alphas, bits, group)
    cgrid = synth.clip_grid(20).tolist()
    cws = awq.Workspace()
    for _ in range(2):
        awq.clip_search(X, W, r.s_star, cgrid, bits, group, workspace=cws)
    torch.cuda.synchronize()
    reps = 10
    times = []
    # The call is a few short launches: a host-side pause inside the region
    # (a collection of the earlier sections' garbage) would leave the device
    # idle between them, so collection is held off while it is timed and the
    # median call is reported beside the mean.
    gc.collect()
    gc.disable()
    try:
        for _ in range(reps):
            flush.zero_()
            flush_sink.add_(flush.amax())
            ea, eb = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            ea.record()
            cr = awq.clip_search(X, W, r.s_star, cgrid, bits, group, workspace=cws, check_status=False)
            eb.record()
            times.append((ea, eb))
        torch.cuda.synchronize()
    finally:
        gc.enable()
    awq.check_device_status(cr.status)
    per_call = sorted(a_.elapsed_time(b_) for a_, b_ in times)
    call_ms = per_call[reps // 2]
    awq.profile_enable(True)
    awq.profile_reset()
    for _ in range(3):
        awq.clip_search(X, W, r.s_star, cgrid, bits, group, workspace=cws, check_status=False)
    cprof = awq.profile_read()
    awq.profile_enable(False)
    C = len(cgrid)
    op_bytes = C * spec.D_in * spec.D_out * 2
    loss_ms = cprof["clip_loss"][0] / max(cprof["clip_loss"][1], 1)
    hbm = float(load_peaks()[0]["hbm_gbs"])
    return {
        "layer": f"{spec.name} (N={spec.N}, D_in={spec.D_in}, D_out={spec.D_out}), {C} ratios, 4-bit g128",
        "ms_per_call": call_ms, "ms_per_call_mean": sum(per_call) / reps, "ms_per_call_max": per_call[-1],
        "n_clip": C,
        "stages_ms": {k: cprof[k][0] / max(cprof[k][1], 1) for k in ("clip_gram", "clip_operand", "clip_loss")},
        "loss_kernel": {"algorithmic_bytes": op_bytes, "achieved_gbs": op_bytes / (loss_ms / 1e3) / 1e9,
                        "frac_hbm": op_bytes / (loss_ms / 1e3) / 1e9 / hbm,
                        "mma_tflops": 2.0 * group * spec.D_in * spec.D_out * C / (loss_ms / 1e3) / 1e12},
        "mean_ratio": float(cr.clip.mean().item()),
        "frac_clipped": float((cr.idx > 0).float().mean().item()),
    }


def gram_section(dev, flush, flush_sink):
    """L(alpha) = sum_n e_n^T (X^T X) e_n against the direct ||X E||^2, one
    call each on the same 16384-token layer and 41-point grid."""
    import torch
    from post_weight_only_b200 import awq, synth
    gspec = synth.workload("sweep_4096x11008_n16k").layers[1]
    Xg_cpu, Wg_cpu = synth.layer_inputs(gspec)
    Xg, Wg = Xg_cpu.to(dev), Wg_cpu.to(dev)
    ag = awq.act_stats(Xg)
    ggrid = synth.alpha_grid(40).tolist()
    bits, group = 4, 128
    gws = awq.Workspace()
    info = {"layer": f"{gspec.name} (N={gspec.N}, D_in={gspec.D_in}, D_out={gspec.D_out}), 41 alphas, 4-bit g128"}
    results = {}
    for mode in ("direct", "gram"):
        use_gram = mode == "gram"
        awq.search(Xg, Wg, ag, ggrid, bits, group, workspace=gws, gram=use_gram)
        torch.cuda.synchronize()
        times = []
        for _ in range(3):
            flush.zero_()
            flush_sink.add_(flush.amax())
            ea, eb = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            ea.record()
            rr = awq.search(Xg, Wg, ag, ggrid, bits, group, workspace=gws, gram=use_gram, check_status=False)
            eb.record()
            times.append((ea, eb))
        torch.cuda.synchronize()
        awq.check_device_status(rr.status)
        ms = sum(a_.elapsed_time(b_) for a_, b_ in times) / len(times)
        results[mode] = rr
        gemm_flops = 2.0 * (gspec.D_in if use_gram else gspec.N) * gspec.D_in * gspec.D_out * len(ggrid)
        info[mode] = {"ms_per_call": ms, "gemm_flops": gemm_flops, "alpha_star": float(rr.alpha_star.item()),
                      "direct_equivalent_tflops": 2.0 * gspec.N * gspec.D_in * gspec.D_out * len(ggrid)
                                                  / (ms / 1e3) / 1e12}
    Ld, Lg = results["direct"].L.cpu(), results["gram"].L.cpu()
    info["speedup"] = info["direct"]["ms_per_call"] / info["gram"]["ms_per_call"]
    info["max_rel_diff_L"] = float(((Lg - Ld).abs() / Ld).max().item())
    del Xg, Wg, gws, results
    torch.cuda.empty_cache()
    return info


def w4a16_section(dev, rank):
    """The W4A16 consumer of the pack format (not part of the step).  Each
    call is timed as one node group of a CUDA graph of 20 calls (its host cost
    is not measured, so small decode shapes are not host-bound); the packed
    weights rotate over copies larger than L2."""
    import torch
    from post_weight_only_b200 import awq

    def rotating(t):
        n = max(2, -(-(256 << 20) // (t.numel() * t.element_size())))
        return [t.clone() for _ in range(n)]

    def graph_ms(fn, reps=20):
        side = torch.cuda.Stream()
        side.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(side):
            for i in range(3):
                fn(i)
        torch.cuda.current_stream().wait_stream(side)
        gr = torch.cuda.CUDAGraph()
        with torch.cuda.graph(gr):
            for i in range(reps):
                fn(i)
        for _ in range(2):                 # untimed replays: clocks up from an idle GPU
            gr.replay()
        torch.cuda.synchronize()
        best = float("inf")
        for _ in range(5):                 # the best of five timed replays
            ea, eb = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            ea.record()
            gr.replay()
            eb.record()
            eb.synchronize()
            best = min(best, ea.elapsed_time(eb))
        del gr
        return best / reps

    bits, group = 4, 128
    g4 = torch.Generator(device=dev).manual_seed(4321 + rank)
    info = {"timing": "best of 5 replays of a CUDA graph of 20 calls (N <= 8: one GEMV launch whose column-tile splits are "
                      "reduced in a cluster (N = 1-2 on the CUDA cores, 3-8 on mma.sync tiles), or a stream-K GEMV "
                      "and a dependent reduce launch; else a status "
                      "clear, the pre-pass and the GEMM), weights rotated over copies > 256 MiB; synthetic "
                      "packed words and deltas",
            "algorithmic_bytes": "packed words + fp32 deltas + X (bf16) + s + Y (fp32), each once"}
    peaks, _ = load_peaks()
    hbm_peak, bf16_peak = float(peaks["hbm_gbs"]), float(peaks["bf16_tflops"])
    for name, (Dk, Dn, Ns) in (("down_proj_28672x8192", (28672, 8192, (1, 2, 4, 8, 16))),
                                ("attn_proj_4096x4096", (4096, 4096, (1, 4, 16, 4096))),
                                ("square_8192x8192", (8192, 8192, (4096,)))):
        packed_q = torch.randint(-2 ** 31, 2 ** 31 - 1, (Dk // 8, Dn), generator=g4, device=dev,
                                 dtype=torch.int64).to(torch.int32)
        scales_q = torch.rand(Dk // group, Dn, generator=g4, device=dev) * 0.01 + 1e-3
        s_q = torch.rand(Dk, generator=g4, device=dev) + 0.5
        weights = rotating(packed_q)
        w_bytes = Dk * Dn // 2 + (Dk // group) * Dn * 4
        for Nq in Ns:
            Xq = torch.randn(Nq, Dk, generator=g4, device=dev).to(torch.bfloat16)
            ws_q = torch.empty(awq.w4a16_workspace_size(Nq, Dk, Dn), dtype=torch.uint8, device=dev)
            ms = graph_ms(lambda i: awq.w4a16_gemm(Xq, s_q, weights[i % len(weights)], scales_q, bits, group,
                                                   check_status=False, workspace=ws_q))
            nbytes = w_bytes + Nq * Dk * 2 + Nq * Dn * 4 + Dk * 4
            gbs = nbytes / (ms / 1e3) / 1e9
            tf = 2.0 * Nq * Dk * Dn / (ms / 1e3) / 1e12
            info[f"{name}_N{Nq}"] = {
                "path": ("cuda-core GEMV" if Nq <= 2 else "mma.sync GEMV") if Nq <= 8 else "tcgen05 GEMM", "ms": ms, "algorithmic_bytes": nbytes,
                "achieved_gbs": gbs, "frac_hbm": gbs / hbm_peak, "tflops": tf, "frac_bf16": tf / bf16_peak}
        del weights, packed_q
    torch.cuda.empty_cache()
    return info


def main():
    args = parse_args()
    if args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
