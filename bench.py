#!/usr/bin/env python
"""Benchmark of the AWQ per-layer scale search on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload NAME]

One step is one pass of the whole per-layer path over one synthetic layer:
activation statistic -> alpha grid search (scale table, per-alpha bf16 operand, the
fused tensor-core loss GEMM, loss reduction + argmin) -> s* = a^alpha* ->
final quantise + pack.  The default workload is the LLaMA-7B-shaped attention
projection (X 4096 x 4096 bf16, W 4096 x 4096 fp32, 4-bit g128, 21 alphas).

Multi-GPU (launched with torchrun, one rank per GPU): every rank searches its
own independent layer (different seed) -- layers are searched independently,
so there is no collective on the data path; `value` is the aggregate
alpha-candidates/s of all ranks, timed as the max over ranks.

--impl reference times the CPU oracle (oracle/) on the host cores on a bounded
column sample of the same workload; rank 0 alone runs it.

Prints one JSON line (rank 0).
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "AWQ search α-candidates/s per layer; eff. TFLOP/s and % of B200 bf16 peak"
UNIT = "alpha-candidates/s"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def parse_args():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=("ours", "reference"), default="ours")
    ap.add_argument("--workload", default="llama7b_attn_proj")
    ap.add_argument("--flush-mib", type=int, default=512)
    ap.add_argument("--cpu-seconds", type=float, default=15.0,
                    help="target CPU time of the oracle baseline sample")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-clip", action="store_true", help="skip timing the weight-clipping search")
    ap.add_argument("--no-gram", action="store_true", help="skip timing the Gram form of the search")
    ap.add_argument("--no-w4a16", action="store_true", help="skip timing the W4A16 consumer kernel")
    ap.add_argument("--no-at-scale", action="store_true",
                    help="skip timing the statistic and pack kernels on the 70B block's largest operands")
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


def committed_traffic():
    """dram bytes of one search-GEMM launch from the committed ncu summary, if
    it was taken on the current kernel source (else None)."""
    path = os.path.join(ROOT, "profiles", "search_gemm_traffic.json")
    if not os.path.exists(path):
        return None
    with open(path) as f:
        d = json.load(f)
    if d.get("kernel_source_sha1_16") != source_hash():
        return None
    return d


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


def layer_for_rank(wl, rank):
    from post_weight_only_b200 import synth
    L = wl.layers[0]
    if rank == 0:
        return L
    x = synth.XSpec(L.x.kind, L.x.n_outlier, L.x.lo, L.x.hi, L.x.seed + 1000 * rank)
    return synth.LayerSpec(f"{L.name}_r{rank}", L.N, L.D_in, L.D_out, x, L.w_std, L.w_seed + 1000 * rank)


def config_of(wl, layer, bits, group, world, loss_form="error"):
    return {"workload": wl.name, "N": layer.N, "D_in": layer.D_in, "D_out": layer.D_out,
            "n_alpha": wl.n_alpha, "bits": bits, "group": group, "loss_form": loss_form,
            "parallelism": f"{world} independent layer(s), one per GPU",
            "l2": "flushed between timed steps: 512 MiB write, then a read of it (no dirty lines left)"}


def calibrate_columns(oracle, X, W, a, alphas, bits, group, target_s):
    """Number of output columns the oracle handles in about target_s seconds
    (it runs one column per OpenMP thread, so calibrate with one per thread)."""
    import numpy as np
    D_out = W.shape[1]
    nt = max(1, oracle.num_threads())
    probe = np.arange(min(nt, D_out), dtype=np.int64)
    t0 = time.perf_counter()
    oracle.search(X, W, a, alphas, bits, group, cols=probe)
    t1 = max(time.perf_counter() - t0, 1e-3)
    return int(max(1, min(D_out, round(len(probe) * target_s / t1 / nt) * nt)))


def cpu_baseline(X, W, alphas, bits, group, target_s):
    """The oracle as it stands, on a bounded column sample, on this host's cores."""
    import numpy as np
    import oracle
    a = oracle.act_stats(X).astype(np.float32)
    D_out = W.shape[1]
    ncols = calibrate_columns(oracle, X, W, a, alphas, bits, group, target_s)
    cols = np.linspace(0, D_out - 1, ncols).astype(np.int64)
    t0 = time.perf_counter()
    oracle.search(X, W, a, alphas, bits, group, cols=cols)
    dt = time.perf_counter() - t0
    value = len(alphas) * (ncols / D_out) / dt
    return {"value": value, "unit": UNIT, "cores": oracle.num_threads(), "kind": "oracle",
            "sample": f"{ncols} of {D_out} output columns x {len(alphas)} alphas (full N and D_in), "
                      f"{dt:.1f} s; value scaled to whole-layer alpha-candidates"}


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    import numpy as np
    import oracle
    from post_weight_only_b200 import synth
    wl = synth.workload(args.workload)
    layer = wl.layers[0]
    bits, group = wl.quant[0]
    X, W = synth.layer_inputs(layer)
    alphas = synth.alpha_grid(wl.n_intervals).numpy()
    a = oracle.act_stats(X).astype(np.float32)
    # size one step (a column sample) to ~4 s of host CPU work
    ncols = calibrate_columns(oracle, X, W, a, alphas, bits, group, 4.0)
    cols = np.linspace(0, layer.D_out - 1, ncols).astype(np.int64)
    for _ in range(args.warmup):
        oracle.search(X, W, a, alphas, bits, group, cols=cols)
    times = []
    for _ in range(args.steps):
        t0 = time.perf_counter()
        oracle.search(X, W, a, alphas, bits, group, cols=cols)
        times.append(time.perf_counter() - t0)
    per_step = sum(times) / len(times)
    value = len(alphas) * (ncols / layer.D_out) / per_step
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": per_step * 1e3, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic (seeded; no dataset or weights)",
        "config": config_of(wl, layer, bits, group, 1),
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": oracle.num_threads(), "kind": "oracle",
                         "sample": f"each step: {ncols} of {layer.D_out} output columns x {len(alphas)} alphas "
                                   "(full N and D_in); value scaled to whole-layer alpha-candidates"},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def run_ours(args):
    import torch
    from post_weight_only_b200 import synth
    from post_weight_only_b200 import awq

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    dist = None
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)

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

    wl = synth.workload(args.workload)
    layer = layer_for_rank(wl, rank)
    bits, group = wl.quant[0]
    alphas = synth.alpha_grid(wl.n_intervals).tolist()
    A = len(alphas)
    X_cpu, W_cpu = synth.layer_inputs(layer)
    X_h, W_h = X_cpu.pin_memory(), W_cpu.pin_memory()
    X = X_h.to(dev)
    W = W_h.to(dev)
    ws = awq.Workspace()
    flush = torch.empty(args.flush_mib << 20, dtype=torch.uint8, device=dev)
    flush_sink = torch.zeros((), dtype=torch.uint8, device=dev)

    form = awq.LOSS_ERROR if args.loss_form == "error" else awq.LOSS_REFERENCE

    def step():
        return awq.quantize_layer(X, W, alphas, bits, group, workspace=ws, loss_form=form)

    for _ in range(args.warmup):
        r = step()
    torch.cuda.synchronize()
    awq.check_device_status(r.search.status)

    # ---------------- device-resident timed region
    clocks = ClockSampler(local)
    clocks.start()
    awq.profile_enable(True)
    awq.profile_reset()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    barrier()
    clocks.mark_start()
    for k in range(args.steps):
        # Evict X and W from L2 before every step: write a buffer larger than
        # L2, then read it back so that the write-back of its dirty lines
        # happens here and not inside the step.
        flush.zero_()
        flush_sink.add_(flush.amax())
        ev[k][0].record()
        r = step()
        ev[k][1].record()
    barrier()
    clocks.mark_end()
    clk = clocks.stop()
    prof = awq.profile_read()
    awq.profile_enable(False)
    awq.check_device_status(r.search.status)
    step_ms = [a.elapsed_time(b) for a, b in ev]
    total_ms = max_over_ranks(sum(step_ms))
    ms_per_step = total_ms / args.steps
    value = A * world / (ms_per_step / 1e3)

    # ---------------- end to end: host buffers in, host results out
    out = None
    e2e_ms = []
    for k in range(args.warmup + args.steps):
        torch.cuda.synchronize()
        t0 = time.perf_counter()
        out = awq.quantize_layer_host(X_h, W_h, alphas, bits, group, device=dev, workspace=ws, out=out,
                                      loss_form=form)
        if k >= args.warmup:
            e2e_ms.append((time.perf_counter() - t0) * 1e3)
    e2e_total = max_over_ranks(sum(e2e_ms))
    e2e_per_step = e2e_total / args.steps
    h2d = X_h.numel() * X_h.element_size() + W_h.numel() * W_h.element_size()
    d2h = sum(t.numel() * t.element_size() for k_, t in out.items())

    # ---------------- roofline of the dominant kernel (the fused loss GEMM)
    peaks, peak_src = load_peaks()
    gemm_ms, gemm_n = prof["search_gemm"]
    flops = A * 2.0 * layer.N * layer.D_in * layer.D_out       # alpha GEMMs only (reference pass excluded)
    gemm_avg_ms = gemm_ms / max(gemm_n, 1)
    achieved = flops / (gemm_avg_ms / 1e3) / 1e12
    peak = float(peaks["bf16_tflops"])
    traffic = committed_traffic()
    roof = {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s", "frac": achieved / peak,
            "peak_source": f"{peak_src} bf16 dense (burst, cuBLAS) from MEASURED_PEAKS.json"
            if peak_src == "measured" else "fallback 1.59 PFLOP/s",
            "kernel": "search_kernel (fused per-alpha loss GEMM)",
            "avg_launch_ms": gemm_avg_ms,
            "traffic": None if traffic is None else traffic["dram_bytes_per_launch"]}
    if traffic is not None:
        roof["traffic_note"] = traffic.get("note", "")

    # ---------------- the HBM-bound kernels alone: back-to-back launches on
    # rotating copies of their inputs (together larger than L2, so every launch
    # reads from HBM), timed by one pair of events around the loop, so that no
    # per-launch event record is inside a launch's time
    def loop_ms(fn, inputs, reps=40):
        for i in range(3):
            fn(inputs[i % len(inputs)])
        torch.cuda.synchronize()
        ea, eb = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        ea.record()
        for i in range(reps):
            fn(inputs[i % len(inputs)])
        eb.record()
        eb.synchronize()
        return ea.elapsed_time(eb) / reps

    def rotating(t):
        n = max(2, -(-(256 << 20) // (t.numel() * t.element_size())))
        return [t.clone() for _ in range(n)]
    Xs, Ws = rotating(X), rotating(W)
    s_star = r.s_star
    alone_ms = {"act_stats": loop_ms(lambda x: awq.act_stats(x), Xs),
                "quantize_pack": loop_ms(lambda w: awq.quantize_pack(w, s_star, bits, group), Ws)}
    del Xs, Ws

    # The same two kernels on the largest operands of the 70B-shaped block
    # (the down projection's 4096 x 28672 activations, the gate projection's
    # 8192 x 28672 weights), where the fixed cost of a launch is amortised:
    # seeded random data of those shapes, generated on the device.
    at_scale = {}
    if not args.no_at_scale:
        g = torch.Generator(device=dev).manual_seed(1234 + rank)
        Xb = torch.randn(4096, 28672, generator=g, device=dev).to(torch.bfloat16)
        Wb = torch.randn(8192, 28672, generator=g, device=dev) * 0.01
        sb = torch.rand(8192, generator=g, device=dev) + 0.5
        xs_b, ws_b = rotating(Xb), rotating(Wb)
        del Xb, Wb
        for name, ms, nbytes, shape in (
                ("act_stats", loop_ms(lambda x: awq.act_stats(x), xs_b, reps=20),
                 4096 * 28672 * 2 + 28672 * 4, "X 4096 x 28672 bf16"),
                ("quantize_pack", loop_ms(lambda w: awq.quantize_pack(w, sb, bits, group), ws_b, reps=10),
                 8192 * 28672 * 4 + 8192 * 4 + 1024 * 28672 * 4 + (8192 // group) * 28672 * 4,
                 "W 8192 x 28672 fp32")):
            gbs = nbytes / (ms / 1e3) / 1e9
            at_scale[name] = {"shape": shape, "avg_launch_ms": ms, "algorithmic_bytes": nbytes, "achieved_gbs": gbs,
                              "peak_gbs": float(load_peaks()[0]["hbm_gbs"]),
                              "frac": gbs / float(load_peaks()[0]["hbm_gbs"])}
        del xs_b, ws_b
        torch.cuda.empty_cache()

    # ---------------- the weight-clipping search that follows the scale search
    # (not part of the step): the same layer at s*, 21 ratios from 1 down to 0.5
    clip_info = None
    if not args.no_clip:
        cgrid = synth.clip_grid(20).tolist()
        cws = awq.Workspace()
        for _ in range(2):
            awq.clip_search(X, W, r.s_star, cgrid, bits, group, workspace=cws)
        torch.cuda.synchronize()
        reps = 10
        times = []
        for _ in range(reps):
            flush.zero_()
            flush_sink.add_(flush.amax())
            ea, eb = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            ea.record()
            cr = awq.clip_search(X, W, r.s_star, cgrid, bits, group, workspace=cws, check_status=False)
            eb.record()
            times.append((ea, eb))
        torch.cuda.synchronize()
        awq.check_device_status(cr.status)
        call_ms = sum(a_.elapsed_time(b_) for a_, b_ in times) / reps
        awq.profile_enable(True)
        awq.profile_reset()
        for _ in range(3):
            awq.clip_search(X, W, r.s_star, cgrid, bits, group, workspace=cws, check_status=False)
        cprof = awq.profile_read()
        awq.profile_enable(False)
        C = len(cgrid)
        op_bytes = C * layer.D_in * layer.D_out * 2
        loss_ms = cprof["clip_loss"][0] / max(cprof["clip_loss"][1], 1)
        clip_info = {
            "ms_per_call": call_ms, "n_clip": C,
            "stages_ms": {k: cprof[k][0] / max(cprof[k][1], 1) for k in ("clip_gram", "clip_operand", "clip_loss")},
            "loss_kernel": {"algorithmic_bytes": op_bytes, "achieved_gbs": op_bytes / (loss_ms / 1e3) / 1e9,
                            "frac_hbm": op_bytes / (loss_ms / 1e3) / 1e9 / float(load_peaks()[0]["hbm_gbs"]),
                            "mma_tflops": 2.0 * group * layer.D_in * layer.D_out * C / (loss_ms / 1e3) / 1e12},
            "mean_ratio": float(cr.clip.mean().item()),
            "frac_clipped": float((cr.idx > 0).float().mean().item()),
        }

    # ---------------- the Gram form of the search on the 16384-token sweep layer
    # (not part of the step): L(alpha) = sum_n e_n^T (X^T X) e_n against the
    # direct ||X E||^2, one call each on the same layer and 41-point grid.
    gram_info = None
    if not args.no_gram:
        gspec = synth.workload("sweep_4096x11008_n16k").layers[1]
        Xg_cpu, Wg_cpu = synth.layer_inputs(gspec)
        Xg, Wg = Xg_cpu.to(dev), Wg_cpu.to(dev)
        ag = awq.act_stats(Xg)
        ggrid = synth.alpha_grid(40).tolist()
        gws = awq.Workspace()
        gram_info = {"layer": f"{gspec.name} (N={gspec.N}, D_in={gspec.D_in}, D_out={gspec.D_out}), 41 alphas, 4-bit g128"}
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
            gram_info[mode] = {"ms_per_call": ms, "gemm_flops": gemm_flops,
                               "alpha_star": float(rr.alpha_star.item()),
                               "direct_equivalent_tflops": 2.0 * gspec.N * gspec.D_in * gspec.D_out * len(ggrid)
                                                           / (ms / 1e3) / 1e12}
        Ld, Lg = results["direct"].L.cpu(), results["gram"].L.cpu()
        gram_info["speedup"] = gram_info["direct"]["ms_per_call"] / gram_info["gram"]["ms_per_call"]
        gram_info["max_rel_diff_L"] = float(((Lg - Ld).abs() / Ld).max().item())
        del Xg, Wg, gws, results
        torch.cuda.empty_cache()

    # ---------------- the W4A16 consumer of the pack format (not part of the step)
    # Each call is timed as one node group of a CUDA graph of 20 calls (its
    # host cost is not measured, so small decode shapes are not host-bound);
    # the packed weights rotate over copies larger than L2.
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
        gr.replay()
        torch.cuda.synchronize()
        ea, eb = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        ea.record()
        gr.replay()
        eb.record()
        eb.synchronize()
        del gr
        return ea.elapsed_time(eb) / reps

    w4_info = None
    if not args.no_w4a16:
        g4 = torch.Generator(device=dev).manual_seed(4321 + rank)
        w4_info = {"timing": "CUDA graph of 20 calls (status clear, then N <= 4: GEMV + split reduce, else "
                             "pre-pass + GEMM), weights rotated over copies > 256 MiB; synthetic packed words "
                             "and deltas",
                   "algorithmic_bytes": "packed words + fp32 deltas + X (bf16) + s + Y (fp32), each once"}
        hbm_peak = float(load_peaks()[0]["hbm_gbs"])
        bf16_peak = float(load_peaks()[0]["bf16_tflops"])
        for name, (Dk, Dn, Ns) in (("down_proj_28672x8192", (28672, 8192, (1, 4, 16))),
                                    ("attn_proj_4096x4096", (4096, 4096, (1, 16, 4096))),
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
                w4_info[f"{name}_N{Nq}"] = {
                    "path": "cuda-core GEMV" if Nq <= 4 else "tcgen05 GEMM", "ms": ms, "algorithmic_bytes": nbytes, "achieved_gbs": gbs, "frac_hbm": gbs / hbm_peak,
                    "tflops": tf, "frac_bf16": tf / bf16_peak}
            del weights, packed_q
        torch.cuda.empty_cache()

    def hbm(stage, nbytes):
        ms, n = prof[stage]
        if n == 0:
            return None
        in_step = ms / n
        avg = alone_ms.get(stage, in_step)
        gbs = nbytes / (avg / 1e3) / 1e9
        out = {"avg_launch_ms": avg, "in_step_ms": in_step, "algorithmic_bytes": nbytes, "achieved_gbs": gbs,
               "peak_gbs": float(peaks["hbm_gbs"]), "frac": gbs / float(peaks["hbm_gbs"])}
        out["timing"] = ("back-to-back launches on rotating inputs larger than L2" if stage in alone_ms
                         else "events around each launch inside the step")
        return out

    stats_bytes = layer.N * layer.D_in * 2 + layer.D_in * 4
    pack_bytes = layer.D_in * layer.D_out * 4 + layer.D_in * 4 + (layer.D_in // 8) * layer.D_out * 4 + \
        (layer.D_in // group) * layer.D_out * 4
    # W once, s and 1/s per alpha, the bf16 operand per alpha
    operand_bytes = layer.D_in * layer.D_out * 4 + A * layer.D_in * 8 + A * layer.D_in * layer.D_out * 2
    kernels = {name: {"total_ms": ms, "launches": n} for name, (ms, n) in prof.items() if n}
    launches = sum(n for _, n in prof.values())     # the library's launches in the timed region

    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic (seeded; no dataset or weights)",
        "config": config_of(wl, layer, bits, group, world, args.loss_form),
        "eff_tflops": flops * world / (ms_per_step / 1e3) / 1e12,
        "pct_bf16_peak_step": flops / (ms_per_step / 1e3) / 1e12 / peak,
        "roofline": roof,
        "hbm_kernels": {"act_stats": hbm("act_stats", stats_bytes), "quantize_pack": hbm("quantize_pack", pack_bytes),
                        "search_operand": hbm("search_operand", operand_bytes)},
        "hbm_kernels_at_scale": at_scale or None,
        "clip_search": clip_info,
        "gram_search": gram_info,
        "w4a16": w4_info,
        "kernels": kernels,
        "e2e": {"value": A * world / (e2e_per_step / 1e3), "unit": UNIT, "ms_per_step": e2e_per_step,
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h},
        "gpu_launches": launches,
        "clocks": clk,
        "alpha_star": float(r.search.alpha_star.item()),
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        import numpy as np
        line["cpu_baseline"] = cpu_baseline(X_cpu, W_cpu, np.array(alphas, dtype=np.float32), bits, group,
                                            args.cpu_seconds)
    if rank == 0:
        print(json.dumps(line), flush=True)
    if dist is not None:
        dist.barrier()
        dist.destroy_process_group()


def main():
    args = parse_args()
    if args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
