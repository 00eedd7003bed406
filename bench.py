#!/usr/bin/env python3
"""Benchmark of the SmoothQuant W8A8 linear layer on B200.

Workload: a Llama-7B-shaped QKV projection (K=4096 in, N=12288 out, M=2048
runtime tokens, fp16 activations and weights with 0.5% seeded outlier
channels x U(20,100), W ~ N(0, 0.02^2)), calibrated on 64 batches of 512
tokens, alpha=0.5, per-tensor static activation scale, per-row weight scale,
fp16 output.  Synthetic, seeded inputs.

One step = the whole hot path over one batch, all through the C ABI:
  calibration absmax over the 32768 calibration tokens (one launch) ->
  weight column absmax -> smoothing factors + closed-form static scale ->
  weight transform + per-row INT8 -> runtime smooth + INT8 quant of X ->
  tcgen05 INT8 GEMM with the fp16 dequant epilogue.
Under torchrun (N>1) each rank calibrates its own 64 x 512 token shard and
runs its own runtime batch (weak scaling); the per-channel maxima are
combined with one NCCL all-reduce(MAX) of K floats before the smoothing
factors -- the only exchange the method has.

Prints one JSON line (rank 0).  ``--impl reference`` times the CPU oracle
instead, on a bounded sample of the same workload.
"""
from __future__ import annotations

import argparse
import itertools
import json
import os
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "W8A8 linear INT8 TOPS & tokens/s at 1 B200; % of INT8 peak / HBM GB/s"
WORKLOAD = ("Llama-7B QKV projection: K=4096, N=12288, M=2048 tokens, fp16 X/W with 0.5% outlier "
            "channels, 64x512 calibration tokens, alpha=0.5, static per-tensor act scale, per-row "
            "weight scale, fp16 out")
M_TOK, K_IN, N_OUT, CALIB_B, CALIB_R = 2048, 4096, 12288, 64, 512
ALPHA = 0.5


def peaks():
    """Measured roofline denominators (generated file) or the recipe's fallback."""
    src = "measured"
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            mp = json.load(f)
        hbm, bf16, bf16_s = float(mp["hbm_gbs"]), float(mp["bf16_tflops"]), float(mp["bf16_tflops_sustained"])
    except Exception:
        hbm, bf16, bf16_s, src = 6650.0, 1590.0, 1400.0, "fallback"
    # INT8 dense tensor peak = measured bf16 x the nominal dense ratio 4.5 / 2.25
    return {"hbm_gbs": hbm, "int8_tops": bf16 * 2.0, "int8_tops_sustained": bf16_s * 2.0, "source": src}


def gemm_traffic():
    """DRAM bytes per GEMM launch from the committed ncu summary, or None when the
    kernel source changed after the counters were taken."""
    import hashlib
    tf = os.path.join(ROOT, "profiles", "linear_w8a8_qkv7b_traffic.json")
    try:
        d = json.load(open(tf))
        h = hashlib.sha256()
        for f in ("gemm.cuh", "ptx_sm100.cuh", "libsq.cu"):
            h.update(open(os.path.join(ROOT, "w8a8_post_quantization_calib_b200", "csrc", f), "rb").read())
        return d["dram_bytes_per_launch"] if h.hexdigest()[:16] == d["source_sha256_16"] else None
    except Exception:
        return None


class ClockSampler:
    """Polls SM clocks and throttle reasons through NVML from a background thread
    (started before the timed region); summary() keeps the samples taken inside
    the [begin, end] window marked around it."""

    REASONS = {0x8: "hw_slowdown", 0x40: "hw_thermal_slowdown", 0x20: "sw_thermal_slowdown",
               0x4: "sw_power_cap", 0x80: "hw_power_brake_slowdown"}

    def __init__(self, device_index: int):
        self.samples, self.max_mhz = [], None      # (t, mhz, reason bits)
        self.t0 = self.t1 = None
        self._stop = threading.Event()
        self.nv = None
        try:
            import pynvml
            pynvml.nvmlInit()
            uuid = None
            try:
                import torch
                uuid = str(torch.cuda.get_device_properties(device_index).uuid)
            except Exception:
                pass
            h = None
            if uuid:
                for cand in (uuid, "GPU-" + uuid):
                    try:
                        h = pynvml.nvmlDeviceGetHandleByUUID(cand)
                        break
                    except Exception:
                        pass
            self.h = h if h is not None else pynvml.nvmlDeviceGetHandleByIndex(device_index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self.reason_fn = (getattr(pynvml, "nvmlDeviceGetCurrentClocksEventReasons", None)
                              or pynvml.nvmlDeviceGetCurrentClocksThrottleReasons)
            self.nv = pynvml
        except Exception:
            self.nv = None

    def _run(self):
        while not self._stop.is_set():
            try:
                mhz = self.nv.nvmlDeviceGetClockInfo(self.h, self.nv.NVML_CLOCK_SM)
                r = self.reason_fn(self.h)
                self.samples.append((time.perf_counter(), mhz, r))
            except Exception:
                pass
            time.sleep(0.001)

    def start(self):
        if self.nv is not None:
            self.t = threading.Thread(target=self._run, daemon=True)
            self.t.start()
            time.sleep(0.05)
        return self

    def begin(self):
        self.t0 = time.perf_counter()

    def end(self):
        self.t1 = time.perf_counter()

    def stop(self):
        self._stop.set()
        if self.nv is not None:
            self.t.join()

    def summary(self):
        win = [x for x in self.samples if self.t0 is not None and self.t0 <= x[0] <= (self.t1 or x[0])]
        if not win and self.samples and self.t0 is not None:     # region shorter than one poll
            win = [min(self.samples, key=lambda x: abs(x[0] - self.t0))]
        reasons = sorted({name for _, _, r in win for bit, name in self.REASONS.items() if r & bit})
        mhz = statistics.median([m for _, m, _ in win]) if win else None
        return {"sm_mhz": mhz, "sm_max_mhz": self.max_mhz, "reasons": reasons, "samples": len(win)}


# --------------------------------------------------------------------------
# CPU oracle timing (reference arm and cpu_baseline)
# --------------------------------------------------------------------------
def oracle_sample(frac: float, wl=None):
    """Run the oracle's full step on a fraction `frac` of every part of the workload.

    Every part is linear in its row count (calibration rows, weight rows for
    the statistic and the quantisation, runtime token rows for quantisation
    and the INT8 GEMM over all N), so step time ~= sample time / frac.
    Returns (seconds, description).
    """
    import numpy as np
    import oracle
    import synth
    if wl is None:
        wl = synth.qkv_7b()
    calib = np.concatenate(wl.calib)
    rc = max(1, int(round(calib.shape[0] * frac)))
    rw = max(1, int(round(N_OUT * frac)))
    rx = max(1, int(round(M_TOK * frac)))
    t0 = time.perf_counter()
    act_max = np.zeros(K_IN, np.float32)
    oracle.calib_absmax(calib[:rc], synth.F16, act_max)
    w_max = oracle.calib_absmax(wl.w[:rw], synth.F16)
    s = oracle.smooth_scales(act_max, w_max, ALPHA)
    a = oracle.static_scale(act_max, s)
    wq, ws = oracle.quant_weight(wl.w[:rw], s, synth.F16)
    xq, av = oracle.smooth_quant_act(wl.x[:rx], s, oracle.STATIC, a, synth.F16)
    wq_full = np.resize(wq, (N_OUT, K_IN))          # GEMM over all N output channels
    ws_full = np.resize(ws, N_OUT)
    acc = oracle.gemm_s32(xq, wq_full)
    oracle.dequant(acc, av, oracle.STATIC, ws_full, synth.F16)
    dt = time.perf_counter() - t0
    desc = (f"oracle full step on a {frac:.4f} fraction of every part: {rc} calibration rows, {rw} weight rows "
            f"(statistic + quantisation), {rx} runtime tokens (quant + INT8 GEMM over all N={N_OUT}); "
            f"step time extrapolated as sample time / fraction")
    return dt, desc


def cpu_cores():
    n = os.environ.get("OMP_NUM_THREADS")
    return int(n) if n and n.isdigit() else (os.cpu_count() or 1)


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    import oracle
    import synth
    oracle.build()
    wl = synth.qkv_7b()
    ops = 2.0 * M_TOK * N_OUT * K_IN
    # size one step so that warmup + steps stay within ~2 minutes
    t_probe, _ = oracle_sample(1.0 / 512, wl)
    budget = 120.0 / max(1, args.steps + args.warmup)
    frac = min(1.0, max(1.0 / 2048, (1.0 / 512) * budget / max(t_probe, 1e-3)))
    for _ in range(args.warmup):
        oracle_sample(frac, wl)
    times, desc = [], ""
    for _ in range(args.steps):
        t, desc = oracle_sample(frac, wl)
        times.append(t / frac)
    ms = 1e3 * statistics.mean(times)
    value = ops / (ms * 1e-3) / 1e12
    line = {
        "metric": METRIC, "value": value, "unit": "TOPS", "n_gpus": args.gpus, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "s8", "data": "synthetic", "impl": "reference",
        "config": {"workload": WORKLOAD, "M": M_TOK, "K": K_IN, "N": N_OUT, "calib_tokens": CALIB_B * CALIB_R,
                   "parallelism": "host cores"},
        "tokens_per_s": M_TOK / (ms * 1e-3),
        "cpu_baseline": {"value": value, "unit": "TOPS", "cores": cpu_cores(), "kind": "oracle", "sample": desc},
        "e2e": {"value": value, "unit": "TOPS", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


# --------------------------------------------------------------------------
# GPU arm
# --------------------------------------------------------------------------
def run_gpu(args):
    import numpy as np
    import torch
    import torch.distributed as dist

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))

    import synth
    import w8a8_post_quantization_calib_b200 as sq
    from w8a8_post_quantization_calib_b200.dist import allreduce_absmax_

    P = peaks()
    wl = synth.qkv_7b(shard=rank)
    dev = torch.device("cuda", local)

    def up(bits, dt=torch.float16):
        return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(dt)

    calib_h = up(np.concatenate(wl.calib)).pin_memory()
    w_h = up(wl.w).pin_memory()
    x_h = up(wl.x).pin_memory()
    calib = calib_h.to(dev)
    W = w_h.to(dev)
    X = x_h.to(dev)
    stats = torch.zeros(2 * K_IN, dtype=torch.float32, device=dev)    # running maxima, zeroed per step
    act_max, w_max = stats[:K_IN], stats[K_IN:]
    s = torch.empty(K_IN, dtype=torch.float32, device=dev)
    a = torch.empty(1, dtype=torch.float32, device=dev)
    wq = torch.empty(N_OUT, K_IN, dtype=torch.int8, device=dev)
    ws = torch.empty(N_OUT, dtype=torch.float32, device=dev)
    xq = torch.empty(M_TOK, K_IN, dtype=torch.int8, device=dev)
    y = torch.empty(M_TOK, N_OUT, dtype=torch.float16, device=dev)
    y_h = torch.empty(M_TOK, N_OUT, dtype=torch.float16).pin_memory()
    stream = torch.cuda.current_stream()
    names = ["calib_absmax", "weight_absmax", "smooth_scales", "quant_weight", "smooth_quant_act", "linear_w8a8"]
    if world > 1:
        names.insert(1, "allreduce_max")

    def step(evs=None):
        def mark(i):
            if evs is not None and evs[i] is not None:
                evs[i].record()          # the current stream: the capture stream while capturing
        i = 0
        mark(i)
        stats.zero_()                      # both running maxima start from zero each step
        sq.calib_absmax(calib, act_max)
        i += 1
        mark(i)
        if world > 1:
            allreduce_absmax_(act_max)      # the one exchange: per-channel maxima of all token shards
            i += 1
            mark(i)
        sq.calib_absmax(W, w_max)
        i += 1
        mark(i)
        sq.smooth_scales(act_max, w_max, ALPHA, s, a)
        i += 1
        mark(i)
        sq.quant_weight(W, s, wq, ws)
        i += 1
        mark(i)
        sq.smooth_quant_act(X, s, sq.ACT_STATIC, a, xq)
        i += 1
        mark(i)
        sq.linear_w8a8(xq, wq, a, sq.ACT_STATIC, ws, y)
        i += 1
        mark(i)

    def barrier():
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()

    for _ in range(args.warmup):
        step()
    if sq.sync_status() != 0:
        raise RuntimeError("kernel error during warm-up")

    # ---- timed region: K steps captured once into a CUDA graph and launched as one
    # graph.  Inside it, events bracket only each step's GEMM (the dominant kernel, for
    # the roofline): an event between two kernels serialises them and cancels the
    # programmatic-launch overlap, so the other kernels are timed in a second pass.
    nk = len(names)
    gi = names.index("linear_w8a8")

    def capture(ev_sets):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            for k in range(args.steps):
                step(ev_sets[k])
        g.replay()                          # untimed: uploads the graph
        torch.cuda.synchronize()
        return g

    def gemm_only_events():
        e = [None] * (nk + 1)
        e[gi] = torch.cuda.Event(enable_timing=True, external=not args.eager_steps)
        e[gi + 1] = torch.cuda.Event(enable_timing=True, external=not args.eager_steps)
        return e

    ev_t = [gemm_only_events() for _ in range(args.steps)]
    graph = None
    if not args.eager_steps:
        try:
            graph = capture(ev_t)
        except Exception as exc:            # noqa: BLE001
            print(f"graph capture failed ({exc}); timing eager launches", file=sys.stderr)
            graph = None
            torch.cuda.synchronize()
            ev_t = [gemm_only_events() for _ in range(args.steps)]
    stream = torch.cuda.current_stream()
    t_start, t_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    clk = ClockSampler(local).start()
    barrier()
    clk.begin()
    t_start.record(stream)
    if graph is not None:
        graph.replay()
    else:
        for k in range(args.steps):
            step(ev_t[k])
    t_end.record(stream)
    barrier()
    clk.end()
    clk.stop()
    st = sq.sync_status()
    if st != 0:
        raise RuntimeError(f"kernel error in the timed region (status {st})")
    ms_total = t_start.elapsed_time(t_end)
    gemm_ms = statistics.mean(ev_t[k][gi].elapsed_time(ev_t[k][gi + 1]) for k in range(args.steps))
    ms_step = ms_total / args.steps
    if world > 1:
        t = torch.tensor([ms_step], dtype=torch.float64, device=dev)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        ms_step = float(t.item())
    used_graph = graph is not None
    del graph

    # ---- per-kernel breakdown: the same K steps with an event between every two kernels
    ext = not args.eager_steps
    evs = [[torch.cuda.Event(enable_timing=True, external=ext) for _ in range(nk + 1)] for _ in range(args.steps)]
    g2 = None
    if used_graph:
        try:
            g2 = capture(evs)
        except Exception:                   # noqa: BLE001
            g2 = None
            evs = [[torch.cuda.Event(enable_timing=True) for _ in range(nk + 1)] for _ in range(args.steps)]
    barrier()
    t2s, t2e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t2s.record(stream)
    if g2 is not None:
        g2.replay()
    else:
        for k in range(args.steps):
            step(evs[k])
    t2e.record(stream)
    barrier()
    ms_step_serial = t2s.elapsed_time(t2e) / args.steps
    per_kernel = [statistics.mean(evs[k][i].elapsed_time(evs[k][i + 1]) for k in range(args.steps))
                  for i in range(nk)]
    del g2

    ops = 2.0 * M_TOK * N_OUT * K_IN
    value = world * ops / (ms_step * 1e-3) / 1e12
    kt = dict(zip(names, per_kernel))

    # algorithmic bytes / ops per launch
    calib_bytes = CALIB_B * CALIB_R * K_IN * 2
    kern = {
        "calib_absmax": {"ms": kt["calib_absmax"], "bytes": calib_bytes},
        "weight_absmax": {"ms": kt["weight_absmax"], "bytes": N_OUT * K_IN * 2},
        "smooth_scales": {"ms": kt["smooth_scales"], "bytes": K_IN * 4 * 3},
        "quant_weight": {"ms": kt["quant_weight"], "bytes": N_OUT * K_IN * 3 + N_OUT * 4},
        "smooth_quant_act": {"ms": kt["smooth_quant_act"], "bytes": M_TOK * K_IN * 3},
        "linear_w8a8": {"ms": kt["linear_w8a8"], "ops": ops,
                        "bytes": M_TOK * K_IN + N_OUT * K_IN + M_TOK * N_OUT * 2 + N_OUT * 4},
    }
    for k, v in kern.items():
        v["share"] = v["ms"] / ms_step_serial
        if "ops" in v:
            v["tops"] = v["ops"] / (v["ms"] * 1e-3) / 1e12
            v["frac_int8_peak"] = v["tops"] / P["int8_tops"]
        v["gbs"] = v["bytes"] / (v["ms"] * 1e-3) / 1e9
        v["frac_hbm"] = v["gbs"] / P["hbm_gbs"]
    if world > 1:
        kern["allreduce_max"] = {"ms": kt["allreduce_max"], "share": kt["allreduce_max"] / ms_step_serial}

    gemm_tops = ops / (gemm_ms * 1e-3) / 1e12
    traffic = gemm_traffic()
    roofline = {"bound": "tensor", "kernel": "linear_w8a8 (tcgen05 kind::i8 GEMM + dequant)",
                "achieved": gemm_tops, "peak": P["int8_tops"], "unit": "TOPS", "frac": gemm_tops / P["int8_tops"],
                "launch_us": gemm_ms * 1e3,
                "traffic": traffic,
                "peak_note": f"INT8 dense = 2 x {P['source']} bf16 cuBLAS burst (nominal 4.5/2.25 ratio); "
                             f"vs sustained {P['int8_tops_sustained']:.0f}: {gemm_tops / P['int8_tops_sustained']:.3f}; "
                             f"vs the nominal 4500 dense INT8: {gemm_tops / 4500.0:.3f}"}

    # ---- end to end: pinned host buffers, H2D of the step's inputs and D2H of the result in the region
    e2e_steps = max(1, min(args.steps, 5))
    h2d = calib_h.numel() * 2 + w_h.numel() * 2 + x_h.numel() * 2
    d2h = y_h.numel() * 2
    barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(e2e_steps):
        calib.copy_(calib_h, non_blocking=True)
        W.copy_(w_h, non_blocking=True)
        X.copy_(x_h, non_blocking=True)
        step()
        y_h.copy_(y, non_blocking=True)
    e1.record(stream)
    barrier()
    ms_e2e = e0.elapsed_time(e1) / e2e_steps
    if world > 1:
        t = torch.tensor([ms_e2e], dtype=torch.float64, device=dev)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        ms_e2e = float(t.item())
    e2e = {"value": world * ops / (ms_e2e * 1e-3) / 1e12, "unit": "TOPS", "h2d_bytes_per_step": h2d,
           "d2h_bytes_per_step": d2h, "ms_per_step": ms_e2e, "steps": e2e_steps}

    cpu = None
    if world == 1 and not args.no_cpu_baseline:
        import oracle
        oracle.build()
        frac = args.cpu_frac
        t, desc = oracle_sample(frac, wl)
        cpu = {"value": ops / (t / frac) / 1e12, "unit": "TOPS", "cores": cpu_cores(), "kind": "oracle",
               "sample": desc, "sample_seconds": t}

    launches_per_step = 6
    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": "TOPS", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "s8", "data": "synthetic",
            "config": {"workload": WORKLOAD, "M": M_TOK, "K": K_IN, "N": N_OUT, "calib_tokens": CALIB_B * CALIB_R,
                       "alpha": ALPHA, "parallelism": f"dp{world} (token shards; all-reduce MAX of act_max)",
                       "l2": "no flush: every step streams 384 MB of inputs (> 126 MB L2)",
                       "launch": "K steps as one CUDA graph" if used_graph else "eager"},
            "tokens_per_s": world * M_TOK / (ms_step * 1e-3),
            "roofline": roofline,
            "kernels": kern,
            "kernels_note": "per-kernel times from a second pass of the same K steps with an event between every "
                            f"two kernels (serialised: {ms_step_serial:.4f} ms/step); the timed region itself has "
                            "events only around the GEMM, so consecutive kernels overlap their launch "
                            "(programmatic dependent launch)",
            "cpu_baseline": cpu,
            "e2e": e2e,
            "clocks": clk.summary(),
            "gpu_launches": launches_per_step * args.steps,
            "gpu_launches_note": "6 libsq kernels per step (+1 torch fill zeroing the two running maxima)",
            "peaks": P,
        }
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    return 0


# --------------------------------------------------------------------------
# Measurement of the other workloads (one JSON line each; not the bench line)
# --------------------------------------------------------------------------
def _time_ms(fn, iters, warmup=3, graph=True):
    """Mean device time of fn() in ms.  With graph=True, `iters` back-to-back calls
    are captured into one CUDA graph (consecutive kernels overlap launch and
    prologue through programmatic dependent launch, as a chain of layers would)
    and the graph is launched once, so host launch overhead is not counted."""
    import torch
    for _ in range(warmup):
        fn()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if graph:
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            for _ in range(iters):
                fn()
        g.replay()
        torch.cuda.synchronize()
        e0.record()
        g.replay()
        e1.record()
    else:
        e0.record()
        for _ in range(iters):
            fn()
        e1.record()
    torch.cuda.synchronize()
    return e0.elapsed_time(e1) / iters


def _dev16(bits, dt):
    import numpy as np
    import torch
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(dt).cuda()


def run_workload(args):
    import numpy as np
    import torch
    import synth
    import w8a8_post_quantization_calib_b200 as sq

    torch.cuda.set_device(0)
    P = peaks()
    out = {"workload": args.workload, "peaks": P}
    bf16, f16 = torch.bfloat16, torch.float16
    if args.workload == "mlp7b":
        # per-token linear sweep, decode to prefill: the runtime quantisation + GEMM of one step
        lines = []
        for which in args.proj.split(","):
            wl = synth.mlp_7b(which, M=4096, calib_batches=4)
            K, N = wl.K, wl.N
            W = _dev16(wl.w, bf16)
            am = torch.zeros(K, device="cuda")
            sq.calib_absmax(_dev16(np.concatenate(wl.calib), bf16), am)
            wm = torch.zeros(K, device="cuda")
            sq.calib_absmax(W, wm)
            s = torch.empty(K, device="cuda")
            a = torch.empty(1, device="cuda")
            sq.smooth_scales(am, wm, 0.5, s, a)
            wq = torch.empty(N, K, dtype=torch.int8, device="cuda")
            ws = torch.empty(N, device="cuda")
            sq.quant_weight(W, s, wq, ws)
            # a decode step reads each layer's weights once: the timed chain
            # rotates over copies whose total exceeds the 126 MB L2, so every
            # GEMM streams its weights from HBM
            wcopies = [wq] + [wq.clone() for _ in range(max(1, -(-3 * 126 * 2**20 // (N * K))))]
            Xall = _dev16(wl.x, bf16)
            for M in (int(t) for t in args.tokens.split(",")):
                X = Xall[:M]
                xq = torch.empty(M, K, dtype=torch.int8, device="cuda")
                at = torch.empty(M, device="cuda")
                y = torch.empty(M, N, dtype=bf16, device="cuda")
                n = sq.linear_workspace_size(M, N, K)
                work = torch.zeros(max(16, n), dtype=torch.uint8, device="cuda")
                t_q = _time_ms(lambda: sq.smooth_quant_act(X, s, sq.ACT_PER_TOKEN, at, xq), 50)
                ctr = itertools.count()
                t_g = _time_ms(lambda: sq.linear_w8a8(xq, wcopies[next(ctr) % len(wcopies)], at, sq.ACT_PER_TOKEN,
                                                      ws, y, workspace=work), 50)
                # one decode layer step: activation quant followed by the GEMM,
                # chained (programmatic dependent launch overlaps the two)
                ctr2 = itertools.count()

                def pair():
                    sq.smooth_quant_act(X, s, sq.ACT_PER_TOKEN, at, xq)
                    sq.linear_w8a8(xq, wcopies[next(ctr2) % len(wcopies)], at, sq.ACT_PER_TOKEN, ws, y,
                                   workspace=work)
                t_p = _time_ms(pair, 50)
                ops = 2.0 * M * N * K
                wbytes = N * K + N * 4 + M * K + M * N * 2
                lines.append({"proj": which, "M": M, "K": K, "N": N,
                              "act_quant_us": t_q * 1e3, "act_quant_gbs": M * K * 3 / (t_q * 1e-3) / 1e9,
                              "gemm_us": t_g * 1e3, "gemm_tops": ops / (t_g * 1e-3) / 1e12,
                              "gemm_frac_int8_peak": ops / (t_g * 1e-3) / 1e12 / P["int8_tops"],
                              "gemm_gbs": wbytes / (t_g * 1e-3) / 1e9,
                              "gemm_frac_hbm": wbytes / (t_g * 1e-3) / 1e9 / P["hbm_gbs"],
                              "tokens_per_s": M / ((t_q + t_g) * 1e-3),
                              "quant_gemm_chain_us": t_p * 1e3})
        out["lines"] = lines
    elif args.workload == "alpha13b":
        wl = synth.heavy_13b(M=8192)
        K, N, M = wl.K, wl.N, wl.M
        W = _dev16(wl.w, f16)
        am = torch.zeros(K, device="cuda")
        sq.calib_absmax(_dev16(np.concatenate(wl.calib), f16), am)
        wm = torch.zeros(K, device="cuda")
        sq.calib_absmax(W, wm)
        held = _dev16(wl.calib[0], f16)
        work = torch.zeros(sq.alpha_search_workspace_size(held.shape[0], N, K, 4), dtype=torch.uint8, device="cuda")
        best = [None]

        def search():
            best[0] = sq.alpha_search(held, W, am, wm, work)
        t_s = _time_ms(search, 5, warmup=1, graph=False)
        al = best[0][0]
        s = torch.empty(K, device="cuda")
        a = torch.empty(1, device="cuda")
        sq.smooth_scales(am, wm, al, s, a)
        wq = torch.empty(N, K, dtype=torch.int8, device="cuda")
        ws = torch.empty(N, device="cuda")
        sq.quant_weight(W, s, wq, ws)
        X = _dev16(wl.x, f16)
        xq = torch.empty(M, K, dtype=torch.int8, device="cuda")
        y = torch.empty(M, N, dtype=f16, device="cuda")
        t_q = _time_ms(lambda: sq.smooth_quant_act(X, s, sq.ACT_STATIC, a, xq), 20)
        t_g = _time_ms(lambda: sq.linear_w8a8(xq, wq, a, sq.ACT_STATIC, ws, y), 20)
        yr = torch.empty(held.shape[0], N, dtype=f16, device="cuda")
        t_r = _time_ms(lambda: sq.gemm_f16_ref(held, W, yr), 20)
        ops = 2.0 * M * N * K
        ops_h = 2.0 * held.shape[0] * N * K
        out.update({"alpha": al, "mse": best[0][1], "search_ms": t_s,
                    "search_note": "one f16 reference GEMM + 4 x (scales, weight quant, held-batch quant, INT8 GEMM, SSE) + host argmin",
                    "ref_gemm_f16_us": t_r * 1e3, "ref_gemm_f16_tflops": ops_h / (t_r * 1e-3) / 1e12,
                    "ref_gemm_f16_frac_bf16_peak": ops_h / (t_r * 1e-3) / 1e12 / (P["int8_tops"] / 2),
                    "act_quant_us": t_q * 1e3, "act_quant_gbs": M * K * 3 / (t_q * 1e-3) / 1e9,
                    "gemm_us": t_g * 1e3, "gemm_tops": ops / (t_g * 1e-3) / 1e12,
                    "gemm_frac_int8_peak": ops / (t_g * 1e-3) / 1e12 / P["int8_tops"]})
    elif args.workload == "mlp70b":
        blk = synth.mlp_block_70b(calib_batches=1)
        d, f, M = blk.d, blk.f, blk.M
        g = torch.from_numpy(blk.gamma).cuda()
        Wg, Wu, Wd = _dev16(blk.w_gate, bf16), _dev16(blk.w_up, bf16), _dev16(blk.w_down, bf16)
        calib = _dev16(blk.calib[0], bf16)
        am1 = torch.zeros(d, device="cuda")
        t_stat = _time_ms(lambda: sq.rmsnorm_absmax(calib, g, blk.eps, am1), 10)
        wm1 = torch.zeros(d, device="cuda")
        sq.calib_absmax(Wg, wm1)
        sq.calib_absmax(Wu, wm1)
        s1 = torch.empty(d, device="cuda")
        a1 = torch.empty(1, device="cuda")
        sq.smooth_scales(am1, wm1, 0.5, s1, a1)
        wq_gu = torch.empty(2 * f, d, dtype=torch.int8, device="cuda")
        ws_gu = torch.empty(2 * f, device="cuda")
        t_wgu = _time_ms(lambda: sq.quant_weight_gateup(Wg, Wu, s1, wq_gu, ws_gu), 5)
        X = _dev16(blk.x, bf16)
        xq = torch.empty(M, d, dtype=torch.int8, device="cuda")
        h = torch.empty(M, f, dtype=bf16, device="cuda")
        hq = torch.empty(M, f, dtype=torch.int8, device="cuda")
        sq.rmsnorm_quant(X, g, s1, blk.eps, a1, xq)
        sq.linear_w8a8_gateup_silu(xq[:2048], wq_gu, a1, sq.ACT_STATIC, ws_gu, h=h[:2048])
        am2 = torch.zeros(f, device="cuda")
        sq.calib_absmax(h[:2048], am2)
        wm2 = torch.zeros(f, device="cuda")
        sq.calib_absmax(Wd, wm2)
        s2 = torch.empty(f, device="cuda")
        a2 = torch.empty(1, device="cuda")
        sq.smooth_scales(am2, wm2, 0.5, s2, a2)
        wq_d = torch.empty(d, f, dtype=torch.int8, device="cuda")
        ws_d = torch.empty(d, device="cuda")
        sq.quant_weight(Wd, s2, wq_d, ws_d)
        y = torch.empty(M, d, dtype=bf16, device="cuda")
        t_n = _time_ms(lambda: sq.rmsnorm_quant(X, g, s1, blk.eps, a1, xq), 10)
        t_gu = _time_ms(lambda: sq.linear_w8a8_gateup_silu(xq, wq_gu, a1, sq.ACT_STATIC, ws_gu, s2=s2, a2=a2, hq=hq), 5)
        t_gu_h = _time_ms(lambda: sq.linear_w8a8_gateup_silu(xq, wq_gu, a1, sq.ACT_STATIC, ws_gu, h=h), 5)
        t_d = _time_ms(lambda: sq.linear_w8a8(hq, wq_d, a2, sq.ACT_STATIC, ws_d, y), 5)
        ops_gu, ops_d = 2.0 * M * 2 * f * d, 2.0 * M * d * f
        t_blk = t_n + t_gu + t_d
        out.update({"M": M, "d": d, "f": f,
                    "block_ms": t_blk, "block_tokens_per_s": M / (t_blk * 1e-3),
                    "block_tops": (ops_gu + ops_d) / (t_blk * 1e-3) / 1e12,
                    "rmsnorm_quant_us": t_n * 1e3, "rmsnorm_quant_gbs": M * d * 3 / (t_n * 1e-3) / 1e9,
                    "rmsnorm_absmax_us_per_2048_tokens": t_stat * 1e3,
                    "rmsnorm_absmax_gbs": 2048 * d * 2 / (t_stat * 1e-3) / 1e9,
                    "gateup_silu_requant_us": t_gu * 1e3, "gateup_tops": ops_gu / (t_gu * 1e-3) / 1e12,
                    "gateup_frac_int8_peak": ops_gu / (t_gu * 1e-3) / 1e12 / P["int8_tops"],
                    "gateup_silu_bf16_h_us": t_gu_h * 1e3,
                    "down_us": t_d * 1e3, "down_tops": ops_d / (t_d * 1e-3) / 1e12,
                    "down_frac_int8_peak": ops_d / (t_d * 1e-3) / 1e12 / P["int8_tops"],
                    "weight_quant_gateup_us": t_wgu * 1e3,
                    "weight_quant_gateup_gbs": 2 * f * d * 3 / (t_wgu * 1e-3) / 1e9})
    elif args.workload == "rows":
        # the HBM-bound kernels on inputs of 256 MiB (twice the L2), so that
        # every call of a timed chain streams from HBM; bytes = algorithmic
        # reads + writes
        R = 1 << 27                                   # elements per input tensor
        g16 = torch.Generator(device="cuda").manual_seed(7)
        lines = []

        only = set(args.only.split(",")) if args.only else None

        def rec(name, fn, nbytes, shape, dt):
            if only is not None and name not in only:
                return
            t_ms = _time_ms(fn, 10)
            gbs = nbytes / (t_ms * 1e-3) / 1e9
            lines.append({"kernel": name, "shape": shape, "dtype": dt, "us": t_ms * 1e3, "gbs": gbs,
                          "frac_hbm": gbs / P["hbm_gbs"]})
        if only is None or "calib_64_launches" in only:
            # the QKV workload's calibration set (64 batches x 512 tokens, fp16,
            # K = 4096) as 64 launches, one per batch, against the one launch
            # over the concatenated batches
            cb = torch.randn(64 * 512, 4096, generator=g16, device="cuda").to(torch.float16)
            amc = torch.zeros(4096, device="cuda")
            views = [cb[i * 512:(i + 1) * 512] for i in range(64)]

            def per_batch():
                for v in views:
                    sq.calib_absmax(v, amc)
            for name, fn in (("calib_64_launches", per_batch), ("calib_1_launch", lambda: sq.calib_absmax(cb, amc))):
                t_ms = _time_ms(fn, 5)
                gbs = cb.numel() * 2 / (t_ms * 1e-3) / 1e9
                lines.append({"kernel": name, "shape": [64 * 512, 4096], "dtype": "f16", "us": t_ms * 1e3, "gbs": gbs,
                              "frac_hbm": gbs / P["hbm_gbs"]})
            del cb, views
            torch.cuda.empty_cache()
        shapes = ((4096, torch.float16), (8192, torch.bfloat16))
        if args.rows_k:
            shapes = tuple(sh for sh in shapes if sh[0] in {int(k) for k in args.rows_k.split(",")})
        for K, dt in shapes:
            M = R // K
            X = torch.randn(M, K, generator=g16, device="cuda").to(dt)
            name = "f16" if dt == torch.float16 else "bf16"
            am = torch.zeros(K, device="cuda")
            rec("calib_absmax", lambda: sq.calib_absmax(X, am), M * K * 2, [M, K], name)
            s = torch.rand(K, device="cuda") + 0.5
            a = torch.full((1,), 0.05, device="cuda")
            xq = torch.empty(M, K, dtype=torch.int8, device="cuda")
            at = torch.empty(M, device="cuda")
            rec("act_static", lambda: sq.smooth_quant_act(X, s, sq.ACT_STATIC, a, xq), M * K * 3, [M, K], name)
            rec("act_per_token", lambda: sq.smooth_quant_act(X, s, sq.ACT_PER_TOKEN, at, xq),
                M * K * 3 + M * 4, [M, K], name)
            rec("quant_weight", lambda: sq.quant_weight(X, s, xq, at), M * K * 3 + M * 4, [M, K], name)
            gam = torch.rand(K, device="cuda") + 0.5
            rec("rmsnorm_quant", lambda: sq.rmsnorm_quant(X, gam, s, 1e-5, a, xq), M * K * 3, [M, K], name)
            rec("rmsnorm_absmax", lambda: sq.rmsnorm_absmax(X, gam, 1e-5, am), M * K * 2, [M, K], name)
            del X, xq, at
            torch.cuda.empty_cache()
        out["lines"] = lines
    print(json.dumps(out), flush=True)
    return 0


def main():
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=["sq", "reference"], default="sq")
    ap.add_argument("--cpu-frac", type=float, default=0.25,
                    help="fraction of the workload the CPU oracle baseline runs")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--eager-steps", action="store_true",
                    help="launch the timed steps one call at a time instead of as one captured CUDA graph")
    ap.add_argument("--tokens", default="1,16,128,4096",
                    help="mlp7b workload: comma-separated token counts M to sweep")
    ap.add_argument("--proj", default="up,down", help="mlp7b workload: projections to sweep")
    ap.add_argument("--only", default="", help="rows workload: comma-separated kernels to run (default all)")
    ap.add_argument("--rows-k", default="", help="rows workload: row lengths to run, of 4096 (fp16) and 8192 (bf16)")
    ap.add_argument("--workload", choices=["qkv7b", "mlp7b", "alpha13b", "mlp70b", "rows"], default="qkv7b",
                    help="qkv7b is the bench line; the others print per-kernel measurements of the other workloads")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    if args.impl == "reference":
        return run_reference(args)
    if args.workload != "qkv7b":
        return run_workload(args)
    return run_gpu(args)


if __name__ == "__main__":
    sys.exit(main())
