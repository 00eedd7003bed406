#!/usr/bin/env python3
"""Benchmark of the SmoothQuant W8A8 layer on B200.

Bench line (default, ``--workload mlp70b``): the 70B-shaped decoder MLP
block, the largest single-GPU workload.  Inputs: bf16 X [16384, 8192]
(runtime tokens) and 8 x 2048 calibration tokens, both N(0,1) with 41
seeded outlier channels x U(20,100); W_gate, W_up [28672, 8192] and W_down
[8192, 28672] ~ N(0, 0.02^2) bf16; RMSNorm gain 1, eps 1e-5; alpha 0.5.
Synthetic, seeded.

One step = the whole hot path over one batch, all through the C ABI:
  calibration statistic of the normalised input over the 16384
  calibration tokens -> weight column statistics of W_gate, W_up -> smoothing
  factors + static scale -> gate/up weight transform + per-row INT8 ->
  calibration forward (RMSNorm + quant -> gate/up GEMM with SiLU*mul, the
  column max of |h| kept in its epilogue) -> weight statistic of W_down ->
  smoothing factors + static scale of h -> down weight transform -> runtime
  block:
  RMSNorm with 1/s folded into its gain + INT8 quant -> gate/up GEMM with the
  SiLU*mul epilogue and the smooth + requant of h -> down GEMM -> bf16 Y.
Under torchrun (N>1) each rank calibrates on its own token shard and runs its
own runtime tokens (weak scaling); the two per-channel statistics are
combined with one NCCL all-reduce(MAX) each, the only exchanges the method
has.

``--workload qkv7b`` prints the same kind of line for the Llama-7B QKV
projection; the other workloads print per-kernel measurements.  Prints one
JSON line (rank 0).  ``--impl reference`` times the CPU oracle instead, on a
bounded sample of the same workload.
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
from dataclasses import dataclass, field

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "W8A8 linear INT8 TOPS & tokens/s at 1 B200; % of INT8 peak / HBM GB/s"
LINES = ("mlp70b", "qkv7b")
MLP70B_DESC = ("70B decoder MLP block: RMSNorm(d=8192, 1/s folded into the gain) + INT8 quant -> gate/up GEMM "
               "K=8192, N=2x28672 + SiLU*mul + smooth/requant -> down GEMM K=28672, N=8192; M=16384 tokens, "
               "8x2048 calibration tokens (h statistic from the calibration forward), alpha=0.5, static "
               "per-tensor act scales, per-row weight scales, bf16 in/out, outlier channels")
QKV_DESC = ("Llama-7B QKV projection: K=4096, N=12288, M=2048 tokens, fp16 X/W with 0.5% outlier channels, "
            "64x512 calibration tokens, alpha=0.5, static per-tensor act scale, per-row weight scale, fp16 out")


def peaks():
    """Measured HBM and bf16 denominators (generated file) or the recipe's fallback."""
    src = "measured"
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            mp = json.load(f)
        hbm, bf16, bf16_s = float(mp["hbm_gbs"]), float(mp["bf16_tflops"]), float(mp["bf16_tflops_sustained"])
    except Exception:
        hbm, bf16, bf16_s, src = 6650.0, 1590.0, 1400.0, "fallback"
    return {"hbm_gbs": hbm, "bf16_tflops": bf16, "bf16_tflops_sustained": bf16_s, "source": src}


def tensor_peak(kind: str = "i8", clk=None) -> dict:
    """Dense tensor-core peak measured on this GPU now (libsq_peak: the GEMM
    mainloop on shared-memory operands): one ~100 ms launch (burst) and ~2 s of
    back-to-back launches (sustained), with the SM clock sampled over each."""
    from w8a8_post_quantization_calib_b200 import peak
    out = {"kind": kind}
    for name, kw in (("burst", {"ms": 100.0}), ("sustained", {"ms": 100.0, "seconds": 2.0})):
        if clk is not None:
            clk.begin()
        r = peak.measure(kind, **kw)
        if clk is not None:
            clk.end()
            c = clk.summary()
            r["sm_mhz"] = c["sm_mhz"]
            r["reasons"] = c["reasons"]
            if c["sm_mhz"]:
                r["tops_per_mhz"] = r["tops"] / c["sm_mhz"]
        out[name] = r
    return out


def traffic_from_profile(name: str):
    """DRAM bytes per launch of a kernel from a committed ncu summary
    (profiles/<name>.json), or None when the kernel's source files (listed
    there) changed after the counters were taken."""
    import hashlib
    tf = os.path.join(ROOT, "profiles", name + ".json")
    try:
        d = json.load(open(tf))
        h = hashlib.sha256()
        for f in d.get("sources", ("gemm.cuh", "ptx_sm100.cuh", "libsq.cu")):
            h.update(open(os.path.join(ROOT, "w8a8_post_quantization_calib_b200", "csrc", f), "rb").read())
        if h.hexdigest()[:16] != d["source_sha256_16"]:
            return None
        return d["dram_bytes_per_launch"] * d.get("scale_to_bench", 1.0)
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
QKV_M, QKV_K, QKV_N, QKV_CB, QKV_CR = 2048, 4096, 12288, 64, 512


def oracle_sample_qkv(frac: float, wl=None):
    """The oracle's full QKV step on a fraction `frac` of every part of the
    workload: calibration rows, weight rows (statistic and quantisation),
    runtime token rows (quantisation and the INT8 GEMM over all N).  Every
    part is linear in its row count, so step time ~= sample time / frac.
    Returns (seconds, description)."""
    import numpy as np
    import oracle
    import synth
    if wl is None:
        wl = synth.qkv_7b()
    calib = np.concatenate(wl.calib)
    rc = max(1, int(round(calib.shape[0] * frac)))
    rw = max(1, int(round(QKV_N * frac)))
    rx = max(1, int(round(QKV_M * frac)))
    t0 = time.perf_counter()
    act_max = np.zeros(QKV_K, np.float32)
    oracle.calib_absmax(calib[:rc], synth.F16, act_max)
    w_max = oracle.calib_absmax(wl.w[:rw], synth.F16)
    s = oracle.smooth_scales(act_max, w_max, 0.5)
    a = oracle.static_scale(act_max, s)
    wq, ws = oracle.quant_weight(wl.w[:rw], s, synth.F16)
    xq, av = oracle.smooth_quant_act(wl.x[:rx], s, oracle.STATIC, a, synth.F16)
    wq_full = np.resize(wq, (QKV_N, QKV_K))          # GEMM over all N output channels
    ws_full = np.resize(ws, QKV_N)
    acc = oracle.gemm_s32(xq, wq_full)
    oracle.dequant(acc, av, oracle.STATIC, ws_full, synth.F16)
    dt = time.perf_counter() - t0
    desc = (f"oracle QKV step on a {frac:.4f} fraction of every part: {rc} calibration rows, {rw} weight rows "
            f"(statistic + quantisation), {rx} runtime tokens (quant + INT8 GEMM over all N={QKV_N}); "
            f"step time extrapolated as sample time / fraction")
    return dt, desc


def oracle_sample_mlp70b(frac: float, blk=None):
    """The oracle's full 70B MLP-block step on a fraction `frac` of every part:
    calibration token rows (norm statistic, calibration forward through the
    gate/up GEMM over all 2 x 28672 rows, h statistic), weight rows of W_gate,
    W_up and W_down (statistics and quantisation), runtime token rows
    (RMSNorm + quant, gate/up GEMM over all rows, SiLU*mul + requant, down GEMM
    over all 8192 rows).  Step time ~= sample time / frac.  Returns
    (seconds, description)."""
    import numpy as np
    import oracle
    import synth
    BF16 = synth.BF16
    if blk is None:
        blk = synth.mlp_block_70b()
    d, f, eps = blk.d, blk.f, blk.eps
    calib = np.concatenate(blk.calib)
    rc = max(1, int(round(calib.shape[0] * frac)))
    rf = max(32, int(round(f * frac)) // 32 * 32)
    rd = max(1, int(round(d * frac)))
    rx = max(1, int(round(blk.M * frac)))
    one = np.array([1.0], np.float32)

    def silu_h(xq, a, wg, wsg, wu, wsu):
        gv = oracle.dequant_f32(oracle.gemm_s32(xq, wg), np.array([a], np.float32), oracle.STATIC, wsg)
        uv = oracle.dequant_f32(oracle.gemm_s32(xq, wu), np.array([a], np.float32), oracle.STATIC, wsu)
        return oracle.silu_mul_bf16(gv, uv)

    t0 = time.perf_counter()
    am1 = oracle.rmsnorm_absmax(calib[:rc], blk.gamma, eps, BF16)
    wm1 = oracle.calib_absmax(blk.w_gate[:rf], BF16)
    oracle.calib_absmax(blk.w_up[:rf], BF16, wm1)
    s1 = oracle.smooth_scales(am1, wm1, blk.alpha)
    a1 = oracle.static_scale(am1, s1)
    wqg, wsg = oracle.quant_weight(blk.w_gate[:rf], s1, BF16)
    wqu, wsu = oracle.quant_weight(blk.w_up[:rf], s1, BF16)
    wqg, wsg = np.resize(wqg, (f, d)), np.resize(wsg, f)          # GEMMs over all f rows
    wqu, wsu = np.resize(wqu, (f, d)), np.resize(wsu, f)
    xq_c, _ = oracle.rmsnorm_quant(calib[:rc], blk.gamma, s1, eps, a1, BF16)
    am2 = oracle.calib_absmax(silu_h(xq_c, a1, wqg, wsg, wqu, wsu), BF16)
    wm2 = oracle.calib_absmax(blk.w_down[:rd], BF16)
    s2 = oracle.smooth_scales(am2, wm2, blk.alpha)
    a2 = oracle.static_scale(am2, s2)
    wqd, wsd = oracle.quant_weight(blk.w_down[:rd], s2, BF16)
    wqd, wsd = np.resize(wqd, (d, f)), np.resize(wsd, d)
    xq, _ = oracle.rmsnorm_quant(blk.x[:rx], blk.gamma, s1, eps, a1, BF16)
    h = silu_h(xq, a1, wqg, wsg, wqu, wsu)
    hq, _ = oracle.smooth_quant_act(h, s2, oracle.STATIC, a2, BF16)
    oracle.dequant(oracle.gemm_s32(hq, wqd), np.array([a2], np.float32), oracle.STATIC, wsd, BF16)
    del one
    dt = time.perf_counter() - t0
    desc = (f"oracle 70B MLP-block step on a {frac:.5f} fraction of every part (a subset): {rc} calibration "
            f"tokens (norm statistic, calibration forward over all {2 * f} gate/up rows, h statistic), "
            f"{rf}+{rf} gate/up and {rd} down weight rows (statistics + quantisation), {rx} runtime tokens "
            f"(RMSNorm+quant, gate/up over all rows, SiLU*mul+requant, down over all {d} rows); step time "
            f"extrapolated as sample time / fraction")
    return dt, desc


ORACLE_SAMPLE = {"mlp70b": oracle_sample_mlp70b, "qkv7b": oracle_sample_qkv}


def cpu_cores():
    n = os.environ.get("OMP_NUM_THREADS")
    return int(n) if n and n.isdigit() else (os.cpu_count() or 1)


def oracle_baseline(workload: str, target_s: float, data=None):
    """Times the oracle on a sample sized for about target_s seconds of CPU
    work; returns (step seconds extrapolated, description, sample seconds)."""
    fn = ORACLE_SAMPLE[workload]
    probe = 1.0 / 1024
    t_probe, _ = fn(probe, data)
    frac = min(1.0, max(1.0 / 16384, probe * target_s / max(t_probe, 1e-3)))
    t, desc = fn(frac, data)
    return t / frac, desc, t, frac


# --------------------------------------------------------------------------
# GPU arm: one bench line
# --------------------------------------------------------------------------
@dataclass
class Spec:
    """What run_line needs from a workload."""
    workload: str
    config: dict
    ops_per_step: float                 # INT8 tensor-core ops of one step (one rank)
    tokens_per_step: int                # runtime tokens of one step (one rank)
    names: list                         # kernels of a step, in order
    step: object                        # step(mark): mark(i) before kernel i, mark(len(names)) after the last
    dominant: str                       # the kernel the roofline line describes
    work: dict                          # name -> {"bytes": algorithmic bytes, "ops": ops} per launch
    solo: dict                          # name -> callable launching that kernel alone (same buffers)
    host_in: dict                       # name -> pinned host tensor: the step's inputs for the e2e leg
    host_out: dict                      # name -> pinned host tensor: the step's result
    io0: dict                           # name -> device tensor: the inputs and the result the step uses
    alloc_io: object                    # () -> a second device set of the same inputs and result
    make_step: object                   # io -> step(mark) on that set
    launches_per_step: int
    launches_note: str
    traffic: object = None              # callable -> DRAM bytes per launch of the dominant kernel, or None
    data: object = None                 # host-side workload object (for the oracle baseline)
    extra: dict = field(default_factory=dict)


def run_line(args, build):
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
    import w8a8_post_quantization_calib_b200 as sq

    # a created stream: the library's kernels overlap their launches with
    # programmatic dependent launch there (not on the default stream)
    torch.cuda.set_stream(torch.cuda.Stream())
    P = peaks()
    spec = build(args, rank, world)
    names, nk = spec.names, len(spec.names)
    steps = args.steps

    def barrier():
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()

    for _ in range(args.warmup):
        spec.step(lambda i: None)
    if sq.sync_status() != 0:
        raise RuntimeError("kernel error during warm-up")

    clk = ClockSampler(local).start()
    # the INT8 dense tensor-core peak of this GPU, measured now
    barrier()
    tpk = tensor_peak("i8", clk)
    barrier()

    # ---- timed region: the K steps captured once into a CUDA graph and launched
    # as one graph; events bracket only each step's dominant kernel (an event
    # between two kernels serialises them and cancels the programmatic-launch
    # overlap).  The other kernels are timed alone below.
    gi = names.index(spec.dominant)

    def events_for_dominant():
        e = [None] * (nk + 1)
        e[gi] = torch.cuda.Event(enable_timing=True, external=not args.eager_steps)
        e[gi + 1] = torch.cuda.Event(enable_timing=True, external=not args.eager_steps)
        return e

    def run_steps(evsets):
        for k in range(steps):
            ev = evsets[k]

            def mark(i, ev=ev):
                if ev[i] is not None:
                    ev[i].record()
            spec.step(mark)

    ev_t = [events_for_dominant() for _ in range(steps)]
    graph = None
    if not args.eager_steps:
        try:
            graph = torch.cuda.CUDAGraph()
            with torch.cuda.graph(graph):
                run_steps(ev_t)
            graph.replay()                    # untimed: uploads the graph
            torch.cuda.synchronize()
        except Exception as exc:              # noqa: BLE001
            print(f"graph capture failed ({exc}); timing eager launches", file=sys.stderr)
            graph = None
            torch.cuda.synchronize()
            ev_t = [events_for_dominant() for _ in range(steps)]
    stream = torch.cuda.current_stream()
    t_start, t_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier()
    clk.begin()
    t_start.record(stream)
    if graph is not None:
        graph.replay()
    else:
        run_steps(ev_t)
    t_end.record(stream)
    barrier()
    clk.end()
    clocks = clk.summary()
    st = sq.sync_status()
    if st != 0:
        raise RuntimeError(f"kernel error in the timed region (status {st})")
    ms_total = t_start.elapsed_time(t_end)
    dom_ms = statistics.mean(ev_t[k][gi].elapsed_time(ev_t[k][gi + 1]) for k in range(steps))
    ms_step = ms_total / steps
    if world > 1:
        t = torch.tensor([ms_step], dtype=torch.float64, device="cuda")
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        ms_step = float(t.item())
    used_graph = graph is not None
    del graph

    # ---- every kernel alone: back-to-back launches of the same call in one
    # graph (inputs larger than L2 stream from HBM on every launch)
    kern = {}
    for name in names:
        fn = spec.solo.get(name)
        if fn is None:
            continue
        reps = spec.extra.get("solo_reps", {}).get(name, 10)
        time.sleep(0.3)        # let the clocks recover from the power cap of the previous measurement
        ms = _time_ms(fn, reps, warmup=2, graph=not args.eager_steps)
        v = {"ms": ms}
        w = spec.work.get(name, {})
        if "bytes" in w:
            v["gbs"] = w["bytes"] / (ms * 1e-3) / 1e9
            v["frac_hbm"] = v["gbs"] / P["hbm_gbs"]
        if "ops" in w:
            v["tops"] = w["ops"] / (ms * 1e-3) / 1e12
            v["frac_int8_peak"] = v["tops"] / tpk["burst"]["tops"]
        kern[name] = v
    if sq.sync_status() != 0:
        raise RuntimeError("kernel error in the per-kernel pass")

    value = world * spec.ops_per_step / (ms_step * 1e-3) / 1e12
    dw = spec.work[spec.dominant]
    dom_tops = dw["ops"] / (dom_ms * 1e-3) / 1e12
    peak_b, peak_s = tpk["burst"]["tops"], tpk["sustained"]["tops"]
    roofline = {"bound": "tensor", "kernel": spec.dominant, "achieved": dom_tops, "peak": peak_b, "unit": "TOPS",
                "frac": dom_tops / peak_b, "traffic": spec.traffic() if spec.traffic else None,
                "launch_us": dom_ms * 1e3, "ops_per_launch": dw["ops"],
                "peak_note": ("measured on this GPU in this run (libsq_peak: tcgen05 kind::i8 mainloop on "
                              "shared-memory operands, one ~100 ms launch); vs its ~2 s sustained figure "
                              f"{peak_s:.0f}: {dom_tops / peak_s:.3f}; vs 2 x the {P['source']} bf16 cuBLAS burst "
                              f"{2 * P['bf16_tflops']:.0f}: {dom_tops / (2 * P['bf16_tflops']):.3f}; vs the nominal "
                              f"4500 dense INT8: {dom_tops / 4500.0:.3f}")}

    # ---- end to end: pinned host buffers, the H2D copy of every step's inputs
    # and the D2H read of its result inside the region.  Two device sets of
    # inputs and results, so that step k+1's inputs cross PCIe (copy stream)
    # while step k computes (this stream) and step k-1's result returns (a
    # third stream); every step still moves all of its bytes.
    n2 = max(2, args.e2e_steps)
    h2d = sum(h.numel() * h.element_size() for h in spec.host_in.values())
    d2h = sum(h.numel() * h.element_size() for h in spec.host_out.values())
    ios = [spec.io0, spec.alloc_io()]
    steps_fn = [spec.make_step(io) for io in ios]
    copy_s, back_s = torch.cuda.Stream(), torch.cuda.Stream()
    copied = [torch.cuda.Event() for _ in range(n2)]
    done = [torch.cuda.Event() for _ in range(n2)]
    back = [torch.cuda.Event() for _ in range(n2)]
    barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    copy_s.wait_event(e0)
    for k in range(n2):
        b = k & 1
        with torch.cuda.stream(copy_s):
            if k >= 2:
                copy_s.wait_event(done[k - 2])          # set b is free once step k-2 has read it
            for name, hv in spec.host_in.items():
                ios[b][name].copy_(hv, non_blocking=True)
            copied[k].record(copy_s)
        stream.wait_event(copied[k])
        if k >= 2:
            stream.wait_event(back[k - 2])              # step k-2's result has left set b
        steps_fn[b](lambda i: None)
        done[k].record(stream)
        with torch.cuda.stream(back_s):
            back_s.wait_event(done[k])
            for name, hv in spec.host_out.items():
                hv.copy_(ios[b][name], non_blocking=True)
            back[k].record(back_s)
    stream.wait_event(back[n2 - 1])
    e1.record(stream)
    barrier()
    ms_e2e = e0.elapsed_time(e1) / n2
    # the PCIe ceiling of the same copies: the step's host inputs alone,
    # back to back on the copy stream (no compute)
    big = max(spec.host_in.values(), key=lambda h: h.numel() * h.element_size())
    with torch.cuda.stream(copy_s):
        ios[0][next(n for n, h in spec.host_in.items() if h is big)].copy_(big, non_blocking=True)
    c0, c1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    c0.record(copy_s)
    with torch.cuda.stream(copy_s):
        for name, hv in spec.host_in.items():
            ios[0][name].copy_(hv, non_blocking=True)
    c1.record(copy_s)
    torch.cuda.synchronize()
    ms_h2d = c0.elapsed_time(c1)
    del ios, steps_fn
    if world > 1:
        t = torch.tensor([ms_e2e], dtype=torch.float64, device="cuda")
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        ms_e2e = float(t.item())
    clk.stop()
    e2e = {"value": world * spec.ops_per_step / (ms_e2e * 1e-3) / 1e12, "unit": "TOPS",
           "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": ms_e2e, "steps": n2,
           "tokens_per_s": world * spec.tokens_per_step / (ms_e2e * 1e-3),
           "h2d_alone_ms": ms_h2d, "h2d_alone_gbs": h2d / (ms_h2d * 1e-3) / 1e9,
           "note": ("pinned host buffers through the C-ABI calls; every step copies its inputs in and its "
                    "result out; two device sets, so step k+1's inputs cross PCIe while step k computes; "
                    "h2d_alone_ms: the same input copies alone, back to back (the PCIe floor of a step)")}

    cpu = None
    if world == 1 and not args.no_cpu_baseline:
        import oracle
        oracle.build()
        t_step, desc, t_sample, frac = oracle_baseline(spec.workload, args.cpu_seconds, spec.data)
        cpu = {"value": spec.ops_per_step / t_step / 1e12, "unit": "TOPS", "cores": cpu_cores(), "kind": "oracle",
               "sample": desc, "sample_seconds": t_sample, "fraction": frac}

    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": "TOPS", "n_gpus": world, "steps": steps,
            "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "s8", "data": "synthetic (seeded; shapes and laws of the workload)",
            "config": dict(spec.config, parallelism=f"dp{world} (token shards; all-reduce MAX of the statistics)",
                           launch="K steps as one CUDA graph" if used_graph else "eager"),
            "tokens_per_s": world * spec.tokens_per_step / (ms_step * 1e-3),
            "roofline": roofline,
            "kernels": kern,
            "kernels_note": ("each kernel timed alone after a 0.3 s pause: back-to-back launches of the same "
                             "call captured in one CUDA graph (CUDA events), fractions of the measured HBM copy / "
                             "of this run's measured INT8 burst peak; inside the step the GEMMs hold the GPU at "
                             "its power cap and lower clocks"),
            "cpu_baseline": cpu,
            "e2e": e2e,
            "clocks": clocks,
            "int8_peak": tpk,
            "gpu_launches": spec.launches_per_step * steps,
            "gpu_launches_note": spec.launches_note,
            "peaks": P,
        }
        line.update(spec.extra.get("line", {}))
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    return 0


def _pinned16(bits, dt):
    import numpy as np
    import torch
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(dt).pin_memory()


def build_mlp70b(args, rank, world) -> Spec:
    import numpy as np
    import torch
    import synth
    import w8a8_post_quantization_calib_b200 as sq
    from w8a8_post_quantization_calib_b200.dist import allreduce_absmax_

    bf16 = torch.bfloat16
    blk = synth.mlp_block_70b(shard=rank)
    d, f, M, eps, al = blk.d, blk.f, blk.M, blk.eps, blk.alpha
    calib_h = _pinned16(np.concatenate(blk.calib), bf16)
    x_h = _pinned16(blk.x, bf16)
    wg_h, wu_h, wd_h = _pinned16(blk.w_gate, bf16), _pinned16(blk.w_up, bf16), _pinned16(blk.w_down, bf16)
    Mc = calib_h.shape[0]
    dv = torch.device("cuda")
    host_in = {"calib": calib_h, "X": x_h, "Wg": wg_h, "Wu": wu_h, "Wd": wd_h}
    io0 = {k: v.to(dv) for k, v in host_in.items()}
    io0["y"] = torch.empty(M, d, dtype=bf16, device=dv)
    y_h = torch.empty(M, d, dtype=bf16).pin_memory()

    def alloc_io():
        io = {k: torch.empty_like(v, device=dv) for k, v in host_in.items()}
        io["y"] = torch.empty(M, d, dtype=bf16, device=dv)
        return io
    gamma = torch.from_numpy(blk.gamma).to(dv)
    stats = torch.zeros(2 * d + 2 * f, dtype=torch.float32, device=dv)     # running maxima, zeroed each step
    am1, wm1 = stats[:d], stats[d:2 * d]
    am2, wm2 = stats[2 * d:2 * d + f], stats[2 * d + f:]
    s1, s2 = torch.empty(d, device=dv), torch.empty(f, device=dv)
    a1, a2 = torch.empty(1, device=dv), torch.empty(1, device=dv)
    wq_gu = torch.empty(2 * f, d, dtype=torch.int8, device=dv)
    ws_gu = torch.empty(2 * f, device=dv)
    wq_d = torch.empty(d, f, dtype=torch.int8, device=dv)
    ws_d = torch.empty(d, device=dv)
    xq_c = torch.empty(Mc, d, dtype=torch.int8, device=dv)
    xq = torch.empty(M, d, dtype=torch.int8, device=dv)
    hq = torch.empty(M, f, dtype=torch.int8, device=dv)
    S = sq.ACT_STATIC

    def make_calls(io):
        calib, X, Wg, Wu, Wd, y = io["calib"], io["X"], io["Wg"], io["Wu"], io["Wd"], io["y"]
        calls = [
            ("calib_norm_absmax", lambda: sq.rmsnorm_absmax(calib, gamma, eps, am1)),
            ("allreduce_norm_stat", lambda: allreduce_absmax_(am1)),
            ("weight_absmax_gate", lambda: sq.calib_absmax(Wg, wm1)),
            ("weight_absmax_up", lambda: sq.calib_absmax(Wu, wm1)),
            ("smooth_scales_gateup", lambda: sq.smooth_scales(am1, wm1, al, s1, a1)),
            ("quant_weight_gateup", lambda: sq.quant_weight_gateup(Wg, Wu, s1, wq_gu, ws_gu)),
            ("calib_rmsnorm_quant", lambda: sq.rmsnorm_quant(calib, gamma, s1, eps, a1, xq_c)),
            ("calib_gateup_hmax", lambda: sq.linear_w8a8_gateup_silu_absmax(xq_c, wq_gu, a1, S, ws_gu, am2)),
            ("allreduce_h_stat", lambda: allreduce_absmax_(am2)),
            ("weight_absmax_down", lambda: sq.calib_absmax(Wd, wm2)),
            ("smooth_scales_down", lambda: sq.smooth_scales(am2, wm2, al, s2, a2)),
            ("quant_weight_down", lambda: sq.quant_weight(Wd, s2, wq_d, ws_d)),
            ("rmsnorm_quant", lambda: sq.rmsnorm_quant(X, gamma, s1, eps, a1, xq)),
            ("gateup_silu_requant", lambda: sq.linear_w8a8_gateup_silu(xq, wq_gu, a1, S, ws_gu, s2=s2, a2=a2,
                                                                       hq=hq)),
            ("down", lambda: sq.linear_w8a8(hq, wq_d, a2, S, ws_d, y)),
        ]
        if world == 1:
            calls = [c for c in calls if not c[0].startswith("allreduce")]
        return calls

    def make_step(io):
        cl = make_calls(io)

        def step(mark):
            stats.zero_()                    # the running maxima start from zero each step
            for i, (_, fn) in enumerate(cl):
                mark(i)
                fn()
            mark(len(cl))
        return step

    calls = make_calls(io0)
    names = [c[0] for c in calls]
    step = make_step(io0)

    gu_ops = 2.0 * M * 2 * f * d
    work = {
        "calib_norm_absmax": {"bytes": Mc * d * 2},
        "weight_absmax_gate": {"bytes": f * d * 2},
        "weight_absmax_up": {"bytes": f * d * 2},
        "smooth_scales_gateup": {"bytes": d * 12},
        "quant_weight_gateup": {"bytes": 2 * f * d * 3 + 2 * f * 4},
        "calib_rmsnorm_quant": {"bytes": Mc * d * 3},
        "calib_gateup_hmax": {"ops": 2.0 * Mc * 2 * f * d, "bytes": Mc * d + 2 * f * d + f * 4},
        "weight_absmax_down": {"bytes": d * f * 2},
        "smooth_scales_down": {"bytes": f * 12},
        "quant_weight_down": {"bytes": d * f * 3 + d * 4},
        "rmsnorm_quant": {"bytes": M * d * 3},
        "gateup_silu_requant": {"ops": gu_ops, "bytes": M * d + 2 * f * d + M * f},
        "down": {"ops": 2.0 * M * d * f, "bytes": M * f + d * f + M * d * 2},
    }
    solo = {n: fn for n, fn in calls if not n.startswith("allreduce")}
    ops = 2.0 * Mc * 2 * f * d + gu_ops + 2.0 * M * d * f
    nlaunch = len([n for n in names if not n.startswith("allreduce")])
    return Spec(
        workload="mlp70b",
        config=dict(LINE_CONFIG["mlp70b"]),
        ops_per_step=ops, tokens_per_step=M, names=names, step=step, dominant="gateup_silu_requant",
        work=work, solo=solo,
        host_in=host_in, host_out={"y": y_h}, io0=io0, alloc_io=alloc_io, make_step=make_step,
        launches_per_step=nlaunch,
        launches_note=(f"{nlaunch} libsq kernels per step (+1 torch fill zeroing the four running maxima"
                       + (", +2 NCCL all-reduces" if world > 1 else "") + ")"),
        traffic=lambda: traffic_from_profile("linear_w8a8_gateup_mlp70b_traffic"),
        data=blk if world == 1 else None,
        extra={"solo_reps": {"calib_gateup_hmax": 3, "gateup_silu_requant": 3, "down": 3, "quant_weight_gateup": 5},
               "line": {"ops_note": ("ops per step = the calibration forward's gate/up GEMM (16384 calibration "
                                     "tokens) + the runtime gate/up and down GEMMs, 2*M*N*K each")}},
    )


def build_qkv7b(args, rank, world) -> Spec:
    import numpy as np
    import torch
    import synth
    import w8a8_post_quantization_calib_b200 as sq
    from w8a8_post_quantization_calib_b200.dist import allreduce_absmax_

    f16 = torch.float16
    wl = synth.qkv_7b(shard=rank)
    M, K, N = QKV_M, QKV_K, QKV_N
    calib_h, w_h, x_h = _pinned16(np.concatenate(wl.calib), f16), _pinned16(wl.w, f16), _pinned16(wl.x, f16)
    dv = torch.device("cuda")
    host_in = {"calib": calib_h, "W": w_h, "X": x_h}
    io0 = {k: v.to(dv) for k, v in host_in.items()}
    io0["y"] = torch.empty(M, N, dtype=f16, device=dv)
    y_h = torch.empty(M, N, dtype=f16).pin_memory()

    def alloc_io():
        io = {k: torch.empty_like(v, device=dv) for k, v in host_in.items()}
        io["y"] = torch.empty(M, N, dtype=f16, device=dv)
        return io
    stats = torch.zeros(2 * K, dtype=torch.float32, device=dv)
    act_max, w_max = stats[:K], stats[K:]
    s, a = torch.empty(K, device=dv), torch.empty(1, device=dv)
    wq, ws = torch.empty(N, K, dtype=torch.int8, device=dv), torch.empty(N, device=dv)
    xq = torch.empty(M, K, dtype=torch.int8, device=dv)

    def make_calls(io):
        calib, W, X, y = io["calib"], io["W"], io["X"], io["y"]
        calls = [
            ("calib_absmax", lambda: sq.calib_absmax(calib, act_max)),
            ("allreduce_max", lambda: allreduce_absmax_(act_max)),
            ("weight_absmax", lambda: sq.calib_absmax(W, w_max)),
            ("smooth_scales", lambda: sq.smooth_scales(act_max, w_max, 0.5, s, a)),
            ("quant_weight", lambda: sq.quant_weight(W, s, wq, ws)),
            ("smooth_quant_act", lambda: sq.smooth_quant_act(X, s, sq.ACT_STATIC, a, xq)),
            ("linear_w8a8", lambda: sq.linear_w8a8(xq, wq, a, sq.ACT_STATIC, ws, y)),
        ]
        if world == 1:
            calls = [c for c in calls if c[0] != "allreduce_max"]
        return calls

    def make_step(io):
        cl = make_calls(io)

        def step(mark):
            stats.zero_()
            for i, (_, fn) in enumerate(cl):
                mark(i)
                fn()
            mark(len(cl))
        return step

    calls = make_calls(io0)
    names = [c[0] for c in calls]
    step = make_step(io0)

    ops = 2.0 * M * N * K
    Mc = calib_h.shape[0]
    work = {"calib_absmax": {"bytes": Mc * K * 2}, "weight_absmax": {"bytes": N * K * 2},
            "smooth_scales": {"bytes": K * 12}, "quant_weight": {"bytes": N * K * 3 + N * 4},
            "smooth_quant_act": {"bytes": M * K * 3},
            "linear_w8a8": {"ops": ops, "bytes": M * K + N * K + M * N * 2 + N * 4}}
    return Spec(
        workload="qkv7b",
        config=dict(LINE_CONFIG["qkv7b"]),
        ops_per_step=ops, tokens_per_step=M, names=names, step=step, dominant="linear_w8a8", work=work,
        solo={n: fn for n, fn in calls if n != "allreduce_max"},
        host_in=host_in, host_out={"y": y_h}, io0=io0, alloc_io=alloc_io, make_step=make_step,
        launches_per_step=6, launches_note="6 libsq kernels per step (+1 torch fill zeroing the two running maxima)",
        traffic=lambda: traffic_from_profile("linear_w8a8_qkv7b_traffic"),
        data=wl if world == 1 else None,
        extra={"solo_reps": {"linear_w8a8": 20, "calib_absmax": 10}})


BUILDERS = {"mlp70b": build_mlp70b, "qkv7b": build_qkv7b}
# the config of each line, shared by both arms (the reference arm reports the
# same workload; "launch" is the GPU arm's default)
LINE_CONFIG = {
    "mlp70b": {"workload": MLP70B_DESC, "M": 16384, "d": 8192, "f": 28672, "calib_tokens": 16384, "alpha": 0.5,
               "eps": 1e-5, "l2": "no flush: every step streams about 7 GB of inputs, weights and activations "
                                  "(> 126 MB L2)"},
    "qkv7b": {"workload": QKV_DESC, "M": QKV_M, "K": QKV_K, "N": QKV_N, "calib_tokens": QKV_CB * QKV_CR,
              "alpha": 0.5, "l2": "no flush: every step streams 384 MB of inputs (> 126 MB L2)"},
}


def run_reference(args):
    """The reference arm: the CPU oracle as it stands on a bounded sample of the
    line workload, on this machine's host cores (rank 0 only)."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    import oracle
    import synth
    oracle.build()
    wl = args.workload
    if wl == "mlp70b":
        data = synth.mlp_block_70b()
        ops, tokens = 2.0 * 16384 * 2 * 28672 * 8192 * 2 + 2.0 * 16384 * 8192 * 28672, 16384
    else:
        data = synth.qkv_7b()
        ops, tokens = 2.0 * QKV_M * QKV_N * QKV_K, QKV_M
    cfg = LINE_CONFIG[wl]
    fn = ORACLE_SAMPLE[wl]
    # size one step so that warm-up + steps stay within about two minutes
    probe = 1.0 / 2048
    t_probe, _ = fn(probe, data)
    budget = 120.0 / max(1, args.steps + args.warmup)
    frac = min(1.0, max(1.0 / 16384, probe * budget / max(t_probe, 1e-3)))
    for _ in range(args.warmup):
        fn(frac, data)
    times, sdesc = [], ""
    for _ in range(args.steps):
        t, sdesc = fn(frac, data)
        times.append(t / frac)
    ms = 1e3 * statistics.mean(times)
    value = ops / (ms * 1e-3) / 1e12
    line = {
        "metric": METRIC, "value": value, "unit": "TOPS", "n_gpus": args.gpus, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "s8", "data": "synthetic (seeded; shapes and laws of the workload)",
        "impl": "reference",
        "config": dict(cfg, parallelism=f"dp{args.gpus} (token shards; all-reduce MAX of the statistics)",
                       launch="K steps as one CUDA graph"),
        "tokens_per_s": tokens / (ms * 1e-3),
        "cpu_baseline": {"value": value, "unit": "TOPS", "cores": cpu_cores(), "kind": "oracle", "sample": sdesc},
        "e2e": {"value": value, "unit": "TOPS", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
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


def stream_ceiling_ms(bufs, iters=50):
    """Device time of one launch that only reads one of `bufs` (rotated, so
    that every launch streams from HBM): the ceiling of a GEMM that reads
    the same weight bytes once per launch (libsq_peak's streaming read, 4
    blocks of 512 threads per SM)."""
    import torch
    from w8a8_post_quantization_calib_b200 import peak
    sink = torch.zeros(1, dtype=torch.int32, device="cuda")
    blocks = 4 * torch.cuda.get_device_properties(0).multi_processor_count
    ctr = itertools.count()
    return _time_ms(lambda: peak.stream_read(bufs[next(ctr) % len(bufs)], blocks, sink), iters)


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
    torch.cuda.set_stream(torch.cuda.Stream())
    P = peaks()
    P["int8_tops"] = 2.0 * P["bf16_tflops"]        # per-kernel fractions below: 2 x bf16 (nominal ratio)
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
                t_s = stream_ceiling_ms(wcopies)
                ops = 2.0 * M * N * K
                wbytes = N * K + N * 4 + M * K + M * N * 2
                lines.append({"proj": which, "M": M, "K": K, "N": N,
                              "act_quant_us": t_q * 1e3, "act_quant_gbs": M * K * 3 / (t_q * 1e-3) / 1e9,
                              "gemm_us": t_g * 1e3, "gemm_tops": ops / (t_g * 1e-3) / 1e12,
                              "gemm_frac_int8_peak": ops / (t_g * 1e-3) / 1e12 / P["int8_tops"],
                              "gemm_gbs": wbytes / (t_g * 1e-3) / 1e9,
                              "gemm_frac_hbm": wbytes / (t_g * 1e-3) / 1e9 / P["hbm_gbs"],
                              "weight_stream_us": t_s * 1e3,
                              "gemm_frac_weight_stream": t_s / t_g,
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
    elif args.workload == "peak":
        clk = ClockSampler(0).start()
        out["int8"] = tensor_peak("i8", clk)
        out["e4m3"] = tensor_peak("e4m3", clk)
        clk.stop()
        out["nominal_dense_tops"] = 4500.0
    elif args.workload == "fp8":
        # the FP8 (E4M3) linear on the Llama-7B MLP shapes: per-token E4M3
        # activation quant + kind::f8f6f4 GEMM, against the INT8 path
        tpk = tensor_peak("e4m3")
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
            sq.smooth_scales_fp8(am, wm, 0.5, s, a)
            wq8 = torch.empty(N, K, dtype=torch.uint8, device="cuda")
            ws = torch.empty(N, device="cuda")
            sq.quant_weight_fp8(W, s, wq8, ws)
            t_wq = _time_ms(lambda: sq.quant_weight_fp8(W, s, wq8, ws), 10)
            wcopies = [wq8] + [wq8.clone() for _ in range(max(1, -(-3 * 126 * 2**20 // (N * K))))]
            Xall = _dev16(wl.x, bf16)
            for M in (int(t) for t in args.tokens.split(",")):
                X = Xall[:M]
                xq8 = torch.empty(M, K, dtype=torch.uint8, device="cuda")
                at = torch.empty(M, device="cuda")
                y = torch.empty(M, N, dtype=bf16, device="cuda")
                t_q = _time_ms(lambda: sq.smooth_quant_act_fp8(X, s, sq.ACT_PER_TOKEN, at, xq8), 50)
                ctr = itertools.count()
                t_g = _time_ms(lambda: sq.linear_fp8(xq8, wcopies[next(ctr) % len(wcopies)], at, sq.ACT_PER_TOKEN,
                                                     ws, y), 20)
                t_s = stream_ceiling_ms(wcopies)
                ops = 2.0 * M * N * K
                lines.append({"proj": which, "M": M, "K": K, "N": N,
                              "act_quant_us": t_q * 1e3, "act_quant_gbs": M * K * 3 / (t_q * 1e-3) / 1e9,
                              "gemm_us": t_g * 1e3, "gemm_tops": ops / (t_g * 1e-3) / 1e12,
                              "gemm_frac_e4m3_peak": ops / (t_g * 1e-3) / 1e12 / tpk["burst"]["tops"],
                              "weight_stream_us": t_s * 1e3,
                              "gemm_frac_weight_stream": t_s / t_g,
                              "weight_quant_us": t_wq * 1e3,
                              "weight_quant_gbs": N * K * 3 / (t_wq * 1e-3) / 1e9})
        out["e4m3_peak"] = tpk
        out["lines"] = lines
    elif args.workload == "gemm":
        # one GEMM of the bench workloads on seeded INT8 operands, for timing
        # and for targeted profiler captures: gateup (70B block, SiLU*mul +
        # requant epilogue), down (70B block), qkv (Llama-7B QKV, fp16 out)
        g8 = torch.Generator(device="cuda").manual_seed(11)

        def codes(r, c):
            return torch.randint(-127, 128, (r, c), generator=g8, device="cuda", dtype=torch.int8)
        lines = []
        for M in (int(t) for t in args.tokens.split(",")):
            if args.gemm == "gateup":
                d, f = 8192, 28672
                xq, wq = codes(M, d), codes(2 * f, d)
                a = torch.full((1,), 1e-2, device="cuda")
                ws = torch.rand(2 * f, generator=g8, device="cuda") * 1e-3
                s2 = torch.rand(f, generator=g8, device="cuda") + 0.5
                a2 = torch.full((1,), 0.05, device="cuda")
                hq = torch.empty(M, f, dtype=torch.int8, device="cuda")
                fn = lambda: sq.linear_w8a8_gateup_silu(xq, wq, a, sq.ACT_STATIC, ws, s2=s2, a2=a2, hq=hq)
                ops, nb = 2.0 * M * 2 * f * d, M * d + 2 * f * d + M * f
            else:
                K, N, odt = (28672, 8192, bf16) if args.gemm == "down" else (4096, 12288, f16)
                xq, wq = codes(M, K), codes(N, K)
                a = torch.full((1,), 1e-2, device="cuda")
                ws = torch.rand(N, generator=g8, device="cuda") * 1e-3
                y = torch.empty(M, N, dtype=odt, device="cuda")
                fn = lambda: sq.linear_w8a8(xq, wq, a, sq.ACT_STATIC, ws, y)
                ops, nb = 2.0 * M * N * K, M * K + N * K + M * N * 2
            t_ms = _time_ms(fn, args.reps, warmup=3, graph=not args.eager_steps)
            lines.append({"gemm": args.gemm, "M": M, "us": t_ms * 1e3, "tops": ops / (t_ms * 1e-3) / 1e12,
                          "frac_int8_2xbf16": ops / (t_ms * 1e-3) / 1e12 / P["int8_tops"],
                          "algorithmic_bytes": nb})
            del xq, wq
        out["lines"] = lines
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
    ap.add_argument("--steps", type=int, default=None,
                    help="timed steps (default: 20 for mlp70b, 200 for qkv7b)")
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["sq", "reference"], default="sq")
    ap.add_argument("--cpu-seconds", type=float, default=20.0,
                    help="CPU work the oracle baseline's sample is sized for")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--e2e-steps", type=int, default=6)
    ap.add_argument("--eager-steps", action="store_true",
                    help="launch the timed steps one call at a time instead of as one captured CUDA graph")
    ap.add_argument("--tokens", default="1,16,128,4096",
                    help="mlp7b / fp8 workloads: comma-separated token counts M to sweep")
    ap.add_argument("--proj", default="up,down", help="mlp7b / fp8 workloads: projections to sweep")
    ap.add_argument("--only", default="", help="rows workload: comma-separated kernels to run (default all)")
    ap.add_argument("--rows-k", default="", help="rows workload: row lengths to run, of 4096 (fp16) and 8192 (bf16)")
    ap.add_argument("--gemm", choices=["gateup", "down", "qkv"], default="gateup",
                    help="gemm workload: which GEMM of the bench workloads to run")
    ap.add_argument("--reps", type=int, default=10, help="gemm workload: launches in the timed graph")
    ap.add_argument("--workload", choices=list(LINES) + ["mlp7b", "alpha13b", "rows", "peak", "fp8", "gemm"],
                    default="mlp70b",
                    help="mlp70b (default) and qkv7b print a bench line; the others print per-kernel measurements")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    if args.steps is None:
        args.steps = 20 if args.workload == "mlp70b" else 200
    if args.impl == "reference":
        if args.workload not in LINES:
            ap.error("--impl reference times a bench-line workload")
        return run_reference(args)
    if args.workload not in LINES:
        return run_workload(args)
    return run_line(args, BUILDERS[args.workload])


if __name__ == "__main__":
    sys.exit(main())
