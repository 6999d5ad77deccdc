#!/usr/bin/env python
"""Benchmark of the int6 QAT training hot path on B200.

One step = one QAT training step of the tied int8 head (8192 x 512) over the
int6 ReLU^2 MLP 512 -> 2048 -> 512 at 65,536 tokens per GPU: per-row weight
quantization of all three weights, MLP forward (relu^2 fused), logits GEMM,
the STE backward of both (dX and fp32 dW GEMMs, fused 2*relu(pre)), and with
N > 1 GPUs the data-parallel all-reduce of the weight gradients over NCCL.

Prints ONE JSON line (rank 0).  Also measured in the same run and reported as
sub-objects: the export quantizer over the 11-layer d=512 state dict (one
grouped launch) and the 3x3 recurrent core at d=640, 16x1024 tokens, R=3.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
"""
import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "QAT linear/MLP TFLOP/s (% B200 bf16 peak); export quantizer GB/s (% HBM)"
T_TOKENS = 65536
VOCAB, D, H = 8192, 512, 2048

# DRAM bytes (read + write) per launch of the head GEMMs from one ncu capture
# each at 16,384 tokens, scaled by 4 to the 65,536-token launch (the traffic
# grows with the token count), with the hash of the GEMM sources the captures
# were taken on: reported only while the sources still match.
NCU_TRAFFIC = {"kernel_hash": "69143808865586e3",
               "bytes_per_launch": {"logits_fwd": 4 * (25.225472e6 + 214.154496e6),
                                    "head_dW": 4 * (285.239808e6 + 3.235328e6)}}


def gemm_source_hash():
    h = hashlib.sha256()
    for f in ("gemm_sm100.cu", "gemm_sm100.cuh", "sm100_ptx.cuh", "common.cuh"):
        with open(os.path.join(ROOT, "quantization_aware_tiny_b200", "csrc", f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            j = json.load(f)
        return {"hbm_gbs": j["hbm_gbs"], "bf16_tflops": j["bf16_tflops"],
                "bf16_tflops_sustained": j.get("bf16_tflops_sustained", j["bf16_tflops"]),
                "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
            "source": "fallback"}


class ClockSampler:
    """SM clock and throttle-reason samples, each with a host timestamp: NVML
    queries (read-only) from a thread every few milliseconds, else
    nvidia-smi's own loop.  Started before the warm-up (nvidia-smi needs a
    moment to start); summary() keeps the samples inside the window marked
    by begin() / end() around the timed region."""

    FIELDS = ("timestamp,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")
    REASONS = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")

    def __init__(self, index, period_s=0.004):
        self.index, self.period = index, period_s
        self.proc, self.thread = None, None
        self.samples = []  # (host time, sm MHz, max MHz, reasons)
        self.t0 = self.t1 = None
        self.nvml_error = None

    def _nvml_handle(self):
        import pynvml
        pynvml.nvmlInit()
        try:
            p = torch.cuda.get_device_properties(self.index)
            bus = "%08X:%02X:%02X.0" % (p.pci_domain_id, p.pci_bus_id, p.pci_device_id)
            return pynvml, pynvml.nvmlDeviceGetHandleByPciBusId(bus)
        except Exception:
            return pynvml, pynvml.nvmlDeviceGetHandleByIndex(self.index)

    def _nvml_loop(self, nv, h, mx):
        bits = {"hw_slowdown": nv.nvmlClocksEventReasonHwSlowdown,
                "hw_thermal_slowdown": nv.nvmlClocksEventReasonHwThermalSlowdown,
                "sw_thermal_slowdown": nv.nvmlClocksEventReasonSwThermalSlowdown,
                "sw_power_cap": nv.nvmlClocksEventReasonSwPowerCap}
        while not self.stop.is_set():
            try:
                sm = float(nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM))
                try:
                    r = nv.nvmlDeviceGetCurrentClocksEventReasons(h)
                except Exception:
                    r = nv.nvmlDeviceGetCurrentClocksThrottleReasons(h)
                self.samples.append((time.monotonic(), sm, mx,
                                     tuple(n for n, bit in bits.items() if r & bit)))
            except Exception as e:  # keep sampling; report the last failure
                self.nvml_error = "%s: %s" % (type(e).__name__, e)
            self.stop.wait(self.period)

    def __enter__(self):
        import threading
        try:
            nv, h = self._nvml_handle()
            mx = float(nv.nvmlDeviceGetMaxClockInfo(h, nv.NVML_CLOCK_SM))
            self.stop = threading.Event()
            self.thread = threading.Thread(target=self._nvml_loop, args=(nv, h, mx), daemon=True)
            self.thread.start()
            return self
        except Exception as e:
            self.nvml_error = "%s: %s" % (type(e).__name__, e)
            self.thread = None
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.index), "--query-gpu=" + self.FIELDS,
                 "--format=csv,noheader,nounits", "-lms", "20"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.smi_t0 = (time.time(), time.monotonic())
        except OSError:
            self.proc = None
        return self

    def begin(self):
        self.t0 = time.monotonic()

    def end(self):
        self.t1 = time.monotonic()

    def __exit__(self, *a):
        if self.thread is not None:
            self.stop.set()
            self.thread.join(timeout=5)
            return
        out = ""
        if self.proc is not None:
            self.proc.terminate()
            try:
                out, _ = self.proc.communicate(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
                out, _ = self.proc.communicate()
        import datetime
        for line in out.strip().splitlines():
            parts = [x.strip() for x in line.split(",")]
            if len(parts) < 8:
                continue
            try:  # nvidia-smi's wall-clock timestamp mapped onto time.monotonic()
                ts = datetime.datetime.strptime(parts[0], "%Y/%m/%d %H:%M:%S.%f").timestamp()
                sm, mx = float(parts[1]), float(parts[2])
            except ValueError:
                continue
            t = ts - self.smi_t0[0] + self.smi_t0[1]
            self.samples.append((t, sm, mx, tuple(n for n, v in zip(self.REASONS, parts[4:8])
                                                 if v.lower() == "active")))

    def summary(self):
        inside = [x for x in self.samples
                  if self.t0 is not None and self.t1 is not None and self.t0 <= x[0] <= self.t1]
        source = "nvml" if self.thread is not None else "nvidia-smi"
        if not inside:
            out = {"samples": 0, "samples_outside_window": len(self.samples), "source": source}
            if self.nvml_error:
                out["nvml_error"] = self.nvml_error
            return out
        sm = [x[1] for x in inside]
        loaded = [v for v in sm if v > 0.5 * max(sm)] or sm
        reasons = sorted({r for x in inside for r in x[3]})
        out = {"sm_mhz": statistics.median(loaded), "sm_max_mhz": max(x[2] for x in inside),
               "samples": len(inside), "source": source, "reasons": reasons}
        if self.nvml_error:
            out["nvml_error"] = self.nvml_error
        return out


def dist_env():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    return int(os.environ.get("RANK", "0")), ws, int(os.environ.get("LOCAL_RANK", "0"))


def make_inputs(seed, device):
    """Synthetic step inputs of one rank, generated on the host: the weights
    are the same on every rank (seed 0, data-parallel replicas), the token
    shard and its upstream gradient come from the rank's own seed."""
    from quantization_aware_tiny_b200 import synthetic as sy
    c = sy.head_mlp_case(T=T_TOKENS, vocab=VOCAB, d=D, H=H, seed=seed)
    if seed != 0:
        w = sy.head_mlp_case(T=1, vocab=VOCAB, d=D, H=H, seed=0)
        c.update({k: w[k] for k in ("Wemb", "Wfc", "Wproj")})
    return {k: (torch.from_numpy(v) if isinstance(v, np.ndarray) else v) for k, v in c.items()}


def timed_calls(step, X, dL, ev_pairs, stream, on_head_grad=None):
    """One step with CUDA events around each call (the head GEMM calls are
    single kernels; quantize and the MLP calls are the step's other launches).
    on_head_grad() runs between the head's backward and the MLP backward."""
    from quantization_aware_tiny_b200 import qat
    qe, qf, qp = step.q

    def timed(name, fn):
        ev_pairs[name][0].record(stream)
        fn()
        ev_pairs[name][1].record(stream)

    timed("quantize", lambda: step.quantize(stream))
    timed("mlp_fwd", lambda: qat.qat_mlp_fwd(X, step.Z, 6, D, H, qfc=qf, qproj=qp,
                                             pre_save=step.pre, h_save=step.h, stream=stream))
    timed("logits_fwd", lambda: qat.qat_linear_fwd(step.Z, step.logits, 8, qw=qe, stream=stream))
    timed("head_dX", lambda: qat.qat_linear_bwd(step.Z, dL, 8, qw=qe, dX=step.dZ, stream=stream))
    timed("head_dW", lambda: qat.qat_linear_bwd(step.Z, dL, 8, dW=step.dWemb, N=VOCAB, K=D,
                                                stream=stream))
    if on_head_grad is not None:
        on_head_grad()
    timed("mlp_bwd", lambda: qat.qat_mlp_bwd(X, step.pre, step.h, step.dZ, 6, D, H, qfc=qf,
                                             qproj=qp, dX=step.dX, dWfc=step.dWfc,
                                             dWproj=step.dWproj, workspace=step.ws,
                                             stream=stream))


CALLS = ("quantize", "mlp_fwd", "logits_fwd", "head_dX", "head_dW", "mlp_bwd")


def kflops_call(name):
    """Contraction FLOPs of one call of the step (0 for the quantizer)."""
    head = 2.0 * T_TOKENS * VOCAB * D
    mlp = 2.0 * T_TOKENS * D * H
    return {"logits_fwd": head, "head_dX": head, "head_dW": head, "mlp_fwd": 2 * mlp,
            "mlp_bwd": 4 * mlp}.get(name, 0.0)
HEAD_KERNELS = ("logits_fwd", "head_dX", "head_dW")


def run_ours(args):
    from quantization_aware_tiny_b200 import dp, qat, steps
    rank, world, local = dist_env()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    pg = None
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=dev)
        pg = dist
    stream = torch.cuda.current_stream()
    inp = make_inputs(seed=dp.shard_seed(0, rank), device=dev)
    W = {k: inp[k].to(dev) for k in ("Wemb", "Wfc", "Wproj")}
    X, dL = inp["X"].to(dev), inp["dLogits"].to(dev)
    step = steps.HeadMlpStep(W["Wemb"], W["Wfc"], W["Wproj"], T_TOKENS)
    flops_step = step.flops_per_token() * T_TOKENS
    names = CALLS
    per_step_events = []

    sync = dp.GradSync(pg) if pg is not None else None
    # with N > 1 the tied head's gradient is summed while the MLP backward runs;
    # the MLP's gradients follow, and every sum completes within the step
    head_hook = (lambda: sync.start([step.dWemb], stream)) if sync is not None else None

    def one(i, timed):
        if timed:
            ev = {n: (torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
                  for n in names}
            per_step_events.append(ev)
            timed_calls(step, X, dL, ev, stream, head_hook)
        else:
            step.step(X, dL, stream, head_hook)
        if sync is not None:
            sync.start([step.dWfc, step.dWproj], stream)
            sync.wait(stream)

    with ClockSampler(local) as clk:  # started before the warm-up, read over the timed window
        for i in range(args.warmup):
            one(i, False)
        if pg is not None:
            pg.barrier()
        torch.cuda.synchronize()
        n0 = qat.launch_count()
        start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        clk.begin()
        start.record(stream)
        for i in range(args.steps):
            one(i, True)
        end.record(stream)
        torch.cuda.synchronize()
        clk.end()
    if pg is not None:
        pg.barrier()
    launches = qat.launch_count() - n0
    ms = start.elapsed_time(end)
    if pg is not None:
        ms = dp.max_over_ranks(ms, pg, dev)
    err = qat.device_error()
    value = flops_step * world * args.steps / (ms * 1e-3) / 1e12

    # per-kernel durations of the head GEMMs (same stream, inside the timed region)
    kt = {n: statistics.mean(e[n][0].elapsed_time(e[n][1]) for e in per_step_events) for n in names}
    dom = max(HEAD_KERNELS, key=kt.get)
    kflops = {"logits_fwd": 2.0 * T_TOKENS * VOCAB * D, "head_dX": 2.0 * T_TOKENS * VOCAB * D,
              "head_dW": 2.0 * T_TOKENS * VOCAB * D}
    pk = peaks()
    # The burst GEMM peak fits a timed region well under a second (the clocks
    # stay at their maximum); the sustained one, measured over seconds under
    # the power cap, fits a region of seconds.
    peak, peak_kind = ((pk["bf16_tflops"], "burst bf16") if ms < 1000.0 else
                       (pk["bf16_tflops_sustained"], "sustained bf16"))
    achieved = kflops[dom] / (kt[dom] * 1e-3) / 1e12
    traffic = (NCU_TRAFFIC["bytes_per_launch"].get(dom)
               if NCU_TRAFFIC["kernel_hash"] == gemm_source_hash() else None)
    roofline = {"bound": "tensor", "kernel": dom, "achieved": round(achieved, 1),
                "peak": peak, "unit": "TFLOP/s",
                "frac": round(achieved / peak, 4), "traffic": traffic,
                "peak_kind": "%s (%s), timed region %.0f ms" % (peak_kind, pk["source"], ms),
                "call_ms": {k: round(v, 4) for k, v in kt.items()},
                "call_frac": {k: round(kflops_call(k) / (v * 1e-3) / 1e12 / peak, 4)
                              for k, v in kt.items() if kflops_call(k)}}

    out = None
    if rank == 0:
        out = {"metric": METRIC, "value": round(value, 2), "unit": "TFLOP/s", "n_gpus": world,
               "steps": args.steps, "warmup": args.warmup,
               "ms_per_step": round(ms / args.steps, 4), "higher_is_better": True,
               "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
               "data": "synthetic (seeded N(0,0.02) weights, N(0,1) bf16 activations, "
                       "N(0,0.01) bf16 upstream grads)",
               "config": {"workload": "tied int8 head 8192x512 + int6 ReLU^2 MLP 512-2048-512, "
                                      "fwd + STE bwd, 65536 tokens per GPU",
                          "tokens_per_gpu": T_TOKENS, "vocab": VOCAB, "d": D, "mlp_hidden": H,
                          "head_bits": 8, "mlp_bits": 6, "global_batch_tokens": T_TOKENS * world,
                          "parallelism": "dp%d" % world,
                          "l2": "inputs larger than L2 (dLogits 1 GiB per step)"},
               "frac_of_peak": round(value / peak, 4),
               "roofline": roofline, "gpu_launches": launches, "device_error": err}
        out["clocks"] = clk.summary()
    # end-to-end through the C ABI with host buffers (all ranks take the same steps)
    e2e = measure_e2e(step, inp, dev, stream, args, pg, flops_step, world)
    if rank == 0:
        out["e2e"] = e2e
        if world == 1:
            out["export"] = measure_export(dev, stream, pk)
            out["export_pack6"] = measure_export(dev, stream, pk, pack6=True)
            out["export_clip_search"] = measure_export(dev, stream, pk, clip_search=True)
            out["dequantize"] = measure_dequant(dev, stream, pk)
            out["recurrent_core"] = measure_core(dev, stream, pk)
            out["recurrent_core_fwd_bwd"] = measure_core_train(dev, stream, pk)
            out["fused_producer"] = measure_fused_producer(dev, stream, pk)
            out["export_int5_mlp"] = auxiliary(lambda: measure_export(dev, stream, pk, mlp_int5=True))
            out["noisy_operand"] = auxiliary(lambda: measure_noisy(dev, stream, pk))
            out["cpu_baseline"] = cpu_baseline()
        print(json.dumps(out), flush=True)
    if pg is not None:
        pg.barrier()
        pg.destroy_process_group()


def measure_e2e(step, inp, dev, stream, args, pg, flops_step, world):
    """Same step through the public API with its inputs copied from pinned host
    memory and its weight gradients read back to pinned host memory, every step
    inside the timed region.  As a training loop's data prefetch would, the
    host-to-device copy of step i + 1's inputs runs on a copy stream while step i
    computes (two device input buffers), and step i's gradients go back on a
    third stream (PCIe carries both directions at once); step i + 1's kernels
    wait for its inputs, and its backward for the read-back of step i."""
    from quantization_aware_tiny_b200 import dp
    hX = inp["X"].pin_memory()
    hdL = inp["dLogits"].pin_memory()
    Xs = [torch.empty_like(hX, device=dev) for _ in range(2)]
    dLs = [torch.empty_like(hdL, device=dev) for _ in range(2)]
    hg = [torch.empty(g.shape, dtype=g.dtype, pin_memory=True) for g in step.grads()]
    steps_e2e = max(3, min(args.steps, 10))
    h2d_s, d2h_s = torch.cuda.Stream(device=dev), torch.cuda.Stream(device=dev)
    ev = lambda: torch.cuda.Event()
    copied = [ev(), ev()]      # inputs of the step using buffer b are on the device
    consumed = [ev(), ev()]    # the step using buffer b no longer reads it
    computed, read_back = ev(), ev()
    sync = dp.GradSync(pg) if pg is not None else None
    head_hook = (lambda: sync.start([step.dWemb], stream)) if sync is not None else None

    def copy_in(i):
        b = i % 2
        with torch.cuda.stream(h2d_s):
            if i >= 2:
                h2d_s.wait_event(consumed[b])
            Xs[b].copy_(hX, non_blocking=True)
            dLs[b].copy_(hdL, non_blocking=True)
            copied[b].record(h2d_s)

    def run(n):
        copy_in(0)
        for i in range(n):
            b = i % 2
            if i + 1 < n:
                copy_in(i + 1)
            stream.wait_event(copied[b])
            if i > 0:
                stream.wait_event(read_back)  # the previous step's gradients have left
            step.step(Xs[b], dLs[b], stream, head_hook)
            if sync is not None:
                sync.start([step.dWfc, step.dWproj], stream)
                sync.wait(stream)
            consumed[b].record(stream)
            computed.record(stream)
            with torch.cuda.stream(d2h_s):
                d2h_s.wait_event(computed)
                for h, g in zip(hg, step.grads()):
                    h.copy_(g, non_blocking=True)
                read_back.record(d2h_s)
        stream.wait_event(read_back)

    run(2)
    torch.cuda.synchronize()
    if pg is not None:
        pg.barrier()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(stream)
    h2d_s.wait_event(a)  # the first copy starts inside the timed region
    run(steps_e2e)
    b.record(stream)
    torch.cuda.synchronize()
    ms = a.elapsed_time(b)
    if pg is not None:
        ms = dp.max_over_ranks(ms, pg, dev)
    h2d = hX.numel() * 2 + hdL.numel() * 2
    d2h = sum(g.numel() * 4 for g in hg)
    return {"value": round(flops_step * world * steps_e2e / (ms * 1e-3) / 1e12, 2),
            "unit": "TFLOP/s", "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
            "steps": steps_e2e, "ms_per_step": round(ms / steps_e2e, 3),
            "overlap": "next step's host-to-device copy runs during this step's compute"}


def flush_l2(buf, clean):
    """Evict L2: write a buffer larger than L2, then read another one so the
    written lines are already back in DRAM when the timed launch starts."""
    buf.add_(1)
    clean.sum()


def measure_export(dev, stream, pk, pack6=False, clip_search=False, mlp_int5=False):
    """Export quantizer over the 11-layer d=512 state dict: one grouped launch,
    L2 flushed (256 MB write) before every timed launch.  pack6: the int6 codes
    are stored 6-bit packed (3 bytes per 4 codes); clip_search: each row keeps
    the least-error clip of six candidates (compute-bound: six candidate
    quantizations and error sums per element)."""
    from quantization_aware_tiny_b200 import export as qexport
    from quantization_aware_tiny_b200 import qat
    from quantization_aware_tiny_b200 import synthetic as sy
    sd = {k: torch.from_numpy(v).to(dev) for k, v in sy.state_dict_case().items()}
    out = qexport.export_state_dict(sd, pack6=pack6, mlp_int5=mlp_int5)  # allocates outputs once
    fl = qat.QAT_EXPORT_CLIP_SEARCH if clip_search else 0
    descs = []
    algo = 0
    for name, mode in qexport.plan(sd, mlp_int5=mlp_int5):
        t = sd[name]
        o = out[name]
        if mode == qat.QAT_EXPORT_FP16:
            descs.append((t.reshape(-1), mode, o["values"], None))
            algo += t.numel() * (4 + 2)
        elif "packed" in o:
            descs.append((t, mode, o["packed"], o["scale16"], fl | qat.QAT_EXPORT_PACK6))
            algo += t.numel() * 4 + t.numel() * 3 // 4 + t.shape[0] * 2
        else:
            descs.append((t, mode, o["codes"], o["scale16"], fl))
            algo += t.numel() * (4 + 1) + t.shape[0] * 2
    flush = torch.empty(64 * 1024 * 1024, dtype=torch.float32, device=dev)
    clean = torch.zeros(64 * 1024 * 1024, dtype=torch.float32, device=dev)
    arr = qat.export_descs(descs)  # marshalled once: the timed launches carry no Python work
    # The same launch captured once in a CUDA graph and replayed on the timed stream.
    side = torch.cuda.Stream(device=dev)
    side.wait_stream(stream)
    with torch.cuda.stream(side):
        qat.quantize_export_batch(arr, stream=side)
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph, stream=side):
            qat.quantize_export_batch(arr, stream=side)
    stream.wait_stream(side)

    def timed(run):
        events = []
        for i in range(60):
            flush_l2(flush, clean)
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            run()
            b.record(stream)
            events.append((a, b))
        torch.cuda.synchronize()
        return statistics.median(a.elapsed_time(b) for a, b in events[10:])  # 10 warm-up, 50 timed

    ms = timed(lambda: qat.quantize_export_batch(arr, stream=stream))
    with torch.cuda.stream(stream):
        ms_graph = timed(graph.replay)
    del graph
    gbs = algo / (ms * 1e-3) / 1e9
    return {"value": round(gbs, 1), "unit": "GB/s", "ms": round(ms, 4),
            "graph": {"ms": round(ms_graph, 4), "value": round(algo / (ms_graph * 1e-3) / 1e9, 1),
                      "unit": "GB/s"},
            "algorithmic_bytes": algo, "launches_per_export": 1,
            "roofline": {"bound": "hbm", "achieved": round(gbs, 1), "peak": pk["hbm_gbs"],
                         "unit": "GB/s", "frac": round(gbs / pk["hbm_gbs"], 4),
                         "peak_kind": "copy bandwidth (%s)" % pk["source"]},
            "workload": "11 blocks x (Q,K,V,O,fc,proj) d=512 MLP3x int6%s + tied emb 1024x512 "
                        "+ small tensors fp16 passthrough; L2 flushed (256 MB written, 256 MB read) "
                        "before each launch" % ((" 6-bit packed" if pack6 else "") +
                                                (" clip search" if clip_search else "") +
                                                (", MLP weights int5" if mlp_int5 else ""))}


def measure_noisy(dev, stream, pk):
    """Noisy-QAT forward operands of the 3x3 core's shared weights at d=640
    (Q, K, V, O, fc 1920x640, proj 640x1920: 3.69 M weights), one
    qat_noisy_operand call each (six launches), int8 step amax/127, L2
    flushed before each set.  Algorithmic bytes: 4 B read + 2 B bf16 written
    per weight, 4 B per row scale."""
    from quantization_aware_tiny_b200 import qat
    from quantization_aware_tiny_b200 import synthetic as sy
    c = sy.recurrent_core_case(T=8)
    Ws = [torch.from_numpy(c[k]).to(dev) for k in ("Wq", "Wk", "Wv", "Wo", "Wfc", "Wproj")]
    outs = [(torch.empty(w.shape, dtype=torch.bfloat16, device=dev),
             torch.empty(w.shape[0], dtype=torch.float32, device=dev)) for w in Ws]
    algo = sum(w.numel() * 6 + w.shape[0] * 4 for w in Ws)
    flush = torch.empty(64 * 1024 * 1024, dtype=torch.float32, device=dev)
    clean = torch.zeros(64 * 1024 * 1024, dtype=torch.float32, device=dev)
    n0 = qat.launch_count()

    def run(step):
        for i, (w, (op, sc)) in enumerate(zip(Ws, outs)):
            qat.qat_noisy_operand(w, 1234, 6 * step + i, op, sc, stream=stream, bits=8)

    events = []
    for it in range(60):
        flush_l2(flush, clean)
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        run(it)
        b.record(stream)
        events.append((a, b))
    torch.cuda.synchronize()
    ms = statistics.median(a.elapsed_time(b) for a, b in events[10:])
    gbs = algo / (ms * 1e-3) / 1e9
    return {"value": round(gbs, 1), "unit": "GB/s", "ms": round(ms, 4), "algorithmic_bytes": algo,
            "launches_per_set": (qat.launch_count() - n0) // 60,
            "roofline": {"bound": "hbm", "achieved": round(gbs, 1), "peak": pk["hbm_gbs"],
                         "unit": "GB/s", "frac": round(gbs / pk["hbm_gbs"], 4),
                         "peak_kind": "copy bandwidth (%s)" % pk["source"]},
            "device_error": qat.device_error(),
            "workload": "Noisy-QAT bf16 operands (Philox-4x32-10 noise, int8 step) of the 3x3 "
                        "core's six shared weights at d=640, one call per weight; L2 flushed "
                        "(256 MB written, 256 MB read) before each set"}


def auxiliary(fn):
    """A sub-measurement that must not cost the benchmark line: an exception is
    recorded in its place in the line, with nothing else skipped."""
    try:
        return fn()
    except Exception as e:  # recorded, not hidden
        return {"error": "%s: %s" % (type(e).__name__, e)}


def measure_dequant(dev, stream, pk):
    """The roundtrip dequantize of the exported 11-layer d=512 state dict (66
    int6 tensors: codes + fp16 row scales -> fp32) in one dequantize_rows_batch
    launch, L2 flushed before each; beside it the same work as 66 per-tensor
    dequantize_rows calls replayed from a CUDA graph.  Algorithmic bytes: 1 B
    code read + 4 B written per element, 2 B per row scale."""
    from quantization_aware_tiny_b200 import export as qexport
    from quantization_aware_tiny_b200 import qat
    from quantization_aware_tiny_b200 import synthetic as sy
    sd = {k: torch.from_numpy(v).to(dev) for k, v in sy.state_dict_case().items()}
    ex = qexport.export_state_dict(sd)
    items = []
    algo = 0
    for name, e in ex.items():
        if "codes" in e:
            c = e["codes"]
            items.append((c, e["scale16"], torch.empty(c.shape, dtype=torch.float32, device=dev)))
            algo += c.numel() * 5 + c.shape[0] * 2
    arr = qat.dequant_descs(items)  # marshalled once
    flush = torch.empty(64 * 1024 * 1024, dtype=torch.float32, device=dev)
    clean = torch.zeros(64 * 1024 * 1024, dtype=torch.float32, device=dev)

    def per_tensor(st):
        for c, s16, o in items:
            qat.dequantize_rows(c, s16, o, stream=st)

    side = torch.cuda.Stream(device=dev)
    side.wait_stream(stream)
    with torch.cuda.stream(side):
        per_tensor(side)
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph, stream=side):
            per_tensor(side)
    stream.wait_stream(side)

    def timed(fn):
        events = []
        for i in range(60):
            flush_l2(flush, clean)
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            fn()
            b.record(stream)
            events.append((a, b))
        torch.cuda.synchronize()
        return statistics.median(a.elapsed_time(b) for a, b in events[10:])

    ms = timed(lambda: qat.dequantize_rows_batch(arr, stream=stream))
    with torch.cuda.stream(stream):
        ms_graph = timed(graph.replay)
    del graph
    gbs = algo / (ms * 1e-3) / 1e9
    return {"value": round(gbs, 1), "unit": "GB/s", "ms": round(ms, 4), "launches": 1,
            "per_tensor_graph": {"ms": round(ms_graph, 4), "launches": len(items),
                                 "value": round(algo / (ms_graph * 1e-3) / 1e9, 1)},
            "algorithmic_bytes": algo,
            "roofline": {"bound": "hbm", "achieved": round(gbs, 1), "peak": pk["hbm_gbs"],
                         "unit": "GB/s", "frac": round(gbs / pk["hbm_gbs"], 4),
                         "peak_kind": "copy bandwidth (%s)" % pk["source"]},
            "workload": "66 int6 tensors of the exported 11-layer d=512 state dict -> fp32 in one "
                        "grouped launch; L2 flushed before each"}


def measure_fused_producer(dev, stream, pk):
    """The QAT linear forward from fp32 weights two ways: the GEMM that
    quantizes W in its own producer (what qat_linear_fwd does when given no
    workspace: the operand never reaches global memory, one launch) against
    quantizing into a workspace first and then running the GEMM on the
    materialised operand (the default).  Cases: the single int6 CastedLinear
    512->512 at 256 tokens and the int8 tied head 8192x512 at 65,536 tokens.
    Each timed call runs from the host: per-call times include the launch
    path a caller sees."""
    from quantization_aware_tiny_b200 import qat
    g = torch.Generator(device="cpu").manual_seed(7)
    out = {}
    for name, (T, N, K, bits) in (("linear_512x512_T256_int6", (256, 512, 512, 6)),
                                  ("head_8192x512_T65536_int8", (65536, 8192, 512, 8))):
        W = (torch.randn(N, K, generator=g) * 0.02).to(dev)
        X = torch.randn(T, K, generator=g).to(torch.bfloat16).to(dev)
        Y = torch.empty((T, N), dtype=torch.bfloat16, device=dev)
        ws = torch.empty(N * K * 2 + N * 4 + 4096, dtype=torch.uint8, device=dev)
        q = qat.quantize_weight(W, bits)

        def fused():
            qat.qat_linear_fwd(X, Y, bits, W=W, stream=stream)  # no workspace: fused producer

        def materialised():
            qat.qat_quantize_weights(W, bits, q.scales, None, q.operand, stream=stream)
            qat.qat_linear_fwd(X, Y, bits, qw=q, stream=stream)

        res = {}
        for label, fn in (("fused_us", fused), ("materialised_us", materialised)):
            for _ in range(3):
                fn()
            reps = 50 if T <= 4096 else 10
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            for _ in range(reps):
                fn()
            b.record(stream)
            torch.cuda.synchronize()
            res[label] = round(a.elapsed_time(b) * 1000 / reps, 2)
        flops = 2.0 * T * N * K
        res["fused_tflops"] = round(flops / (res["fused_us"] * 1e-6) / 1e12, 1)
        res["materialised_tflops"] = round(flops / (res["materialised_us"] * 1e-6) / 1e12, 1)
        out[name] = res
    out["device_error"] = qat.device_error()
    return out


def _core_setup(dev):
    from quantization_aware_tiny_b200 import steps
    from quantization_aware_tiny_b200 import synthetic as sy
    c = sy.recurrent_core_case(T=16384)
    w = {k: torch.from_numpy(c[k]).to(dev) for k in ("Wq", "Wk", "Wv", "Wo", "Wfc", "Wproj")}
    core = steps.RecurrentCore(w["Wq"], w["Wk"], w["Wv"], w["Wo"], w["Wfc"], w["Wproj"], 6)
    return core, c["X"].to(dev)


def _timed_l2_flushed(fn, prep, stream, dev, warm=10, reps=50):
    """Median CUDA-event time of fn() over reps launches, prep() and an L2
    flush before each (the activations and the weights leave L2)."""
    flush = torch.empty(64 * 1024 * 1024, dtype=torch.float32, device=dev)
    clean = torch.zeros(64 * 1024 * 1024, dtype=torch.float32, device=dev)
    for _ in range(warm):
        prep()
        fn()
    times = []
    for _ in range(reps):
        prep()
        flush_l2(flush, clean)
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        fn()
        b.record(stream)
        torch.cuda.synchronize()
        times.append(a.elapsed_time(b))
    return statistics.median(times)


def measure_core(dev, stream, pk):
    """3x3 recurrent core at d=640 (QKV/O + MLP 1920), 16x1024 tokens, R=3:
    the inference forward (in place, nothing kept)."""
    core, x0 = _core_setup(dev)
    x = x0.clone()
    ms = _timed_l2_flushed(lambda: core.forward(x, 3, stream), lambda: x.copy_(x0), stream, dev)
    tf = core.flops(16384, 3) / (ms * 1e-3) / 1e12
    return {"value": round(tf, 1), "unit": "TFLOP/s", "ms": round(ms, 4),
            "frac": round(tf / pk["bf16_tflops"], 4), "peak_kind": "burst bf16 (%s)" % pk["source"],
            "workload": "3x3 core d=640 8H/4KV hd80, QKV+O+MLP1920, 16384 tokens, R=3, "
                        "weights quantized once; L2 flushed before each timed forward"}


def measure_core_train(dev, stream, pk):
    """The same core for training: the forward keeping every application's
    activations, then the STE backward through the R = 3 applications in
    reverse with the shared weights' gradients summed over the uses.  FLOPs:
    the forward's plus, per application, 8*T*d*H (the MLP's four backward
    GEMMs) and 8*T*d*d (two each for O and Q)."""
    from quantization_aware_tiny_b200 import qat
    from quantization_aware_tiny_b200 import synthetic as sy
    core, x0 = _core_setup(dev)
    dY = sy.act_bf16(np.random.default_rng(13), 16384, 640, std=sy.DY_STD).to(dev)

    def fwd_bwd():
        core.forward_train(x0, 3, stream)
        core.backward(dY, stream)

    core.forward_train(x0, 3, stream)  # buffers allocated before timing
    core.backward(dY, stream)
    torch.cuda.synchronize()
    ms = _timed_l2_flushed(fwd_bwd, lambda: None, stream, dev)
    ms_bwd = _timed_l2_flushed(lambda: core.backward(dY, stream), lambda: None, stream, dev)
    f_fwd, f_bwd = core.flops(16384, 3), core.flops_bwd(16384, 3)
    tf = (f_fwd + f_bwd) / (ms * 1e-3) / 1e12
    tfb = f_bwd / (ms_bwd * 1e-3) / 1e12
    return {"value": round(tf, 1), "unit": "TFLOP/s", "ms": round(ms, 4),
            "frac": round(tf / pk["bf16_tflops"], 4), "peak_kind": "burst bf16 (%s)" % pk["source"],
            "gflop": round((f_fwd + f_bwd) / 1e9, 1),
            "bwd": {"ms": round(ms_bwd, 4), "value": round(tfb, 1), "gflop": round(f_bwd / 1e9, 1),
                    "frac": round(tfb / pk["bf16_tflops"], 4)},
            "device_error": qat.device_error(),
            "workload": "3x3 core d=640, 16384 tokens, R=3: forward keeping activations + STE "
                        "backward over the 3 applications (dW summed); L2 flushed before each"}


def _threads():
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 1) for i in threadpool_info() if i.get("user_api") == "blas"]
        return max(n) if n else 1
    except Exception:
        return os.cpu_count() or 1


def oracle_step_time(T, seed=0):
    """The CPU oracle's version of one step on T tokens (time in seconds)."""
    import oracle as o
    from quantization_aware_tiny_b200 import synthetic as sy
    c = sy.head_mlp_case(T=T, vocab=VOCAB, d=D, H=H, seed=seed)
    X, dL = c["X"].float().numpy(), c["dLogits"].float().numpy()
    t0 = time.perf_counter()
    qe = o.quantize_weight(c["Wemb"], 8)
    qf = o.quantize_weight(c["Wfc"], 6)
    qp = o.quantize_weight(c["Wproj"], 6)
    o.head_mlp_step(qe, qf, qp, X, dL)
    return time.perf_counter() - t0


def cpu_baseline(target_s=12.0):
    """The oracle, as it stands, on a bounded sample of the step's tokens."""
    t_small = oracle_step_time(512)
    T = int(min(T_TOKENS, max(512, 512 * target_s / max(t_small, 1e-3))))
    T = max(512, T // 512 * 512)
    dt = oracle_step_time(T)
    flops = 3 * 2.0 * D * (VOCAB + 2 * H) * T
    return {"value": round(flops / dt / 1e12, 5), "unit": "TFLOP/s", "cores": _threads(),
            "kind": "oracle",
            "sample": "one step on %d of the 65536 tokens (quantize + fwd + STE bwd, numpy "
                      "fp64 GEMMs, scalar C quantizer), %.1f s" % (T, dt)}


def run_reference(args):
    rank, world, _ = dist_env()
    if rank != 0:
        return
    # per-step sample sized so the whole --steps/--warmup run stays within minutes
    t_small = oracle_step_time(256)
    per_step = min(6.0, 150.0 / max(1, args.steps + args.warmup))
    T = int(min(T_TOKENS, max(256, 256 * per_step / max(t_small, 1e-3))))
    T = max(256, T // 256 * 256)
    for i in range(args.warmup):
        oracle_step_time(T, seed=i)
    tot = 0.0
    for i in range(args.steps):
        tot += oracle_step_time(T, seed=100 + i)
    flops = 3 * 2.0 * D * (VOCAB + 2 * H) * T
    value = flops * args.steps / tot / 1e12
    cb = {"value": round(value, 5), "unit": "TFLOP/s", "cores": _threads(), "kind": "oracle",
          "sample": "%d tokens per step of the 65536-token step (quantize + fwd + STE bwd)" % T}
    print(json.dumps({
        "impl": "reference", "metric": METRIC, "value": round(value, 5), "unit": "TFLOP/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(tot / args.steps * 1e3, 2), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": "tied int8 head 8192x512 + int6 ReLU^2 MLP 512-2048-512, "
                               "fwd + STE bwd, 65536 tokens per GPU",
                   "tokens_per_step_sample": T, "parallelism": "dp%d" % world},
        "cpu_baseline": cb,
        "e2e": {"value": round(value, 5), "unit": "TFLOP/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0}}), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=30)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=("ours", "reference"))
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    if args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
