#!/usr/bin/env python
"""Throughput benchmark of the GKA layer library on B200.

Default workload: the chunked forward on B=8, heads=8, T=2048, D=128, bf16,
chunk 64, a=0.5, r=20 (the shape of the paper's solver study), seeded
synthetic inputs.  One step = one gka_forward call over the whole batch.
A second measurement times the recurrent decode step on 256 x 32 heads with
an fp32 state of 1 GiB (HBM-bound) and reports GB/s.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Prints one JSON line on rank 0.  With --impl reference the float64 CPU
oracle is timed on the host cores on a bounded sample of the same workload.
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

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "GKA fwd tokens/s (B8·T2048·H8·D128 bf16) & % bf16 tensor peak; decode GB/s"
WORKLOAD = "bf16_b8h8t2048d128"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
                  "sm_max_mhz": 1965.0}


# DRAM traffic (dram__bytes_read.sum + dram__bytes_write.sum) of one ncu capture per
# kernel, with the SHA-1 of the kernel's source file at capture time: when the
# source has changed since, the figure no longer describes the kernel and the
# bench reports null.  The captures' commands sit beside their summaries.
TRAFFIC = {
    # full-size forward workload (B8 H8 T2048 D128, chunk 64), one launch
    "chunk_solve_tc": {"bytes": 237.094400e6 + 23.277824e6, "workload": "bf16_b8h8t2048d128",
                       "src": "test_ridge_regression_b200/csrc/solve_tc.cuh",
                       "sha1": "bf2266c98c0e6146d6f61891d28cc9b931a90aef"},
    "state_pass_tc": {"bytes": 67.716864e6 + 79.924480e6, "workload": "bf16_b8h8t2048d128",
                      "src": "test_ridge_regression_b200/csrc/state_tc.cuh",
                      "sha1": "557968b9a4b4f6da6d895bc493988a8c16af285f"},
    # backward kernels captured at B2 H8 T2048 (1024 chunks, 16 heads), scaled x4 to the
    # full workload (the row kernel's traffic is per chunk, the adjoint pass's per head)
    "bwd_rows_tc": {"bytes": 4 * (217.798144e6 + 43.793664e6), "workload": "bf16_b8h8t2048d128",
                    "src": "test_ridge_regression_b200/csrc/backward_tc.cuh",
                    "sha1": "ac9c66bdb4db03eca297e2dd0a96931353d9febb"},
    "adjoint_pass_tc": {"bytes": 4 * (117.882624e6 + 38.258432e6), "workload": "bf16_b8h8t2048d128",
                        "src": "test_ridge_regression_b200/csrc/adjoint_tc.cuh",
                        "sha1": "bcd3ef1e1b540648f212e8dd8eb7ac785171869a"},
    # decode captured on 64 x 32 heads (state above L2), scaled x4 to 256 x 32 heads
    "decode_step": {"bytes": 4 * (270.045952e6 + 209.251584e6), "workload": "decode_bf16_b256h32d128",
                    "src": "test_ridge_regression_b200/csrc/decode.cuh",
                    "sha1": "7f7fb0601312f76476c7888b57b106839465129d"},
}

def traffic_of(kernel, workload):
    import hashlib
    t = TRAFFIC.get(kernel)
    if not t or t["workload"] != workload:
        return None
    try:
        with open(os.path.join(ROOT, t["src"]), "rb") as f:
            if hashlib.sha1(f.read()).hexdigest() != t["sha1"]:
                return None
    except OSError:
        return None
    return t["bytes"]


def parse():
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=20)
    p.add_argument("--warmup", type=int, default=5)
    p.add_argument("--impl", choices=["ours", "reference"], default="ours")
    p.add_argument("--workload", default=WORKLOAD)
    p.add_argument("--no-decode", action="store_true")
    p.add_argument("--no-write-gate", action="store_true",
                   help="skip the write-gated forward leg")
    p.add_argument("--no-backward", action="store_true", help="skip the backward leg")
    p.add_argument("--no-solver-study", action="store_true", help="skip the solver-study leg")
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--no-configs", action="store_true",
                   help="skip the legs of the other forward workloads")
    p.add_argument("--decode-steps", type=int, default=None)
    p.add_argument("--decode-batch", type=int, default=None,
                   help="fewer decode sequences (profiling runs); default: the workload's 256")
    return p.parse_args()


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        d["_source"] = "measured"
        return d
    d = dict(FALLBACK_PEAKS)
    d["_source"] = "fallback"
    return d


def flops_per_head_token(D, C, r):
    """Algorithmic flops of the chunk form per (head, token), counting the causal
    C x C products as dense tiles: Chebyshev (r-1)(2D^2+4CD), readout 2D^2+4CD,
    state update 4D^2, norm 2D^2+2CD+2C^2."""
    ch = (r - 1) * (2 * D * D + 4 * C * D)
    out = 2 * D * D + 4 * C * D
    upd = 4 * D * D
    nrm = 2 * D * D + 2 * C * D + 2 * C * C
    return ch, out, upd, nrm


class ClockSampler:
    """Samples the SM clock and the clock-event (throttle) reasons of the bench GPU
    during a timed region: NVML polled every millisecond from a thread (reads
    only), with nvidia-smi at 200 ms as a fallback."""

    REASONS = {0x4: "sw_power_cap", 0x8: "hw_slowdown", 0x20: "sw_thermal_slowdown",
               0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown"}

    def __init__(self, cuda_index: int):
        self.cuda_index = cuda_index
        self.samples = []          # (sm_mhz, reasons bitmask)
        self.max_mhz = None
        self._stop = threading.Event()
        self._thread = None
        self._proc = None

    def _pci_id(self):
        import torch
        p = torch.cuda.get_device_properties(self.cuda_index)
        return f"{p.pci_domain_id:08x}:{p.pci_bus_id:02x}:{p.pci_device_id:02x}.0"

    def __enter__(self):
        try:
            import pynvml
            pynvml.nvmlInit()
            h = pynvml.nvmlDeviceGetHandleByPciBusId(self._pci_id().encode())
            self.max_mhz = float(pynvml.nvmlDeviceGetMaxClockInfo(h, pynvml.NVML_CLOCK_SM))

            def poll():
                while not self._stop.is_set():
                    try:
                        mhz = pynvml.nvmlDeviceGetClockInfo(h, pynvml.NVML_CLOCK_SM)
                        why = pynvml.nvmlDeviceGetCurrentClocksEventReasons(h)
                        self.samples.append((float(mhz), int(why)))
                    except Exception:
                        pass
                    self._stop.wait(0.001)
            self._thread = threading.Thread(target=poll, daemon=True)
            self._thread.start()
        except Exception:
            self._start_smi()
        return self

    def _start_smi(self):
        try:
            self._proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self._pci_id()}",
                 "--query-gpu=clocks.sm,clocks.max.sm,clocks_event_reasons.active",
                 "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)

            def read():
                for line in self._proc.stdout:
                    parts = [x.strip() for x in line.split(",")]
                    try:
                        self.max_mhz = float(parts[1])
                        self.samples.append((float(parts[0]), int(parts[2], 16)))
                    except (ValueError, IndexError):
                        pass
            self._thread = threading.Thread(target=read, daemon=True)
            self._thread.start()
        except Exception:
            self._proc = None

    def __exit__(self, *a):
        self._stop.set()
        if self._proc is not None:
            self._proc.terminate()
            try:
                self._proc.wait(timeout=5)
            except Exception:
                self._proc.kill()
        if self._thread is not None:
            self._thread.join(timeout=2)

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": ["unsampled"]}
        mhz = [m for m, _ in self.samples]
        mask = 0
        for _, w in self.samples:
            mask |= w
        reasons = sorted(name for bit, name in self.REASONS.items() if mask & bit)
        return {"sm_mhz": statistics.median(mhz), "sm_max_mhz": self.max_mhz, "reasons": reasons,
                "samples": len(mhz), "source": "nvml" if self._proc is None else "nvidia-smi"}


def cpu_threads():
    try:
        return len(os.sched_getaffinity(0))
    except Exception:
        return os.cpu_count() or 1


def _heads(x, n, w, with_d=True):
    if with_d:
        return x.reshape(w.B * w.H, w.T, w.D)[:n].reshape(1, n, w.T, w.D)
    return x.reshape(w.B * w.H, w.T)[:n].reshape(1, n, w.T)


def oracle_calibrate(w, budget_s, q, k, v, beta):
    """Number of whole heads the oracle runs in about `budget_s` seconds with
    all host threads (measured on one head per thread)."""
    import oracle
    nth = cpu_threads()
    n0 = max(1, min(nth, w.B * w.H))
    t0 = time.perf_counter()
    oracle.forward(_heads(q, n0, w), _heads(k, n0, w), _heads(v, n0, w),
                   _heads(beta, n0, w, False), w.a, w.r, nthreads=n0)
    t_par = time.perf_counter() - t0
    rounds = max(1, int(budget_s / max(t_par, 1e-3)))
    return max(1, min(w.B * w.H, n0 * rounds))


def oracle_sample(w, nheads, q, k, v, beta):
    """Times the oracle on the first `nheads` whole heads of the workload;
    returns (tokens/s in the metric's unit, seconds, threads)."""
    import oracle
    threads = min(cpu_threads(), nheads)
    args = (_heads(q, nheads, w), _heads(k, nheads, w), _heads(v, nheads, w),
            _heads(beta, nheads, w, False))
    t0 = time.perf_counter()
    oracle.forward(*args, w.a, w.r, nthreads=threads)
    dt = time.perf_counter() - t0
    tokens = nheads * w.T / w.H          # metric tokens: (batch, position) over all heads
    return tokens / dt, dt, threads


def run_reference(args, w, cfg, rank, world):
    """The oracle, timed on the host cores (rank 0 only)."""
    if rank != 0:
        return
    from test_ridge_regression_b200.inputs import workload_inputs
    q, k, v, beta = workload_inputs(w)
    total = args.steps + args.warmup
    budget = min(5.0, max(0.5, 150.0 / max(total, 1)))
    nheads = oracle_calibrate(w, budget, q, k, v, beta)
    vals = []
    info = None
    for i in range(total):
        val, dt, threads = oracle_sample(w, nheads, q, k, v, beta)
        if i >= args.warmup:
            vals.append(val)
            info = (nheads, threads)
    value = statistics.mean(vals) if vals else 0.0
    tok_step = w.B * w.T
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1e3 * tok_step / value if value else None,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "config": cfg,
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": info[1] if info else 0,
                         "kind": "oracle",
                         "sample": f"{info[0]} whole heads x {w.T} tokens of the workload per "
                                   f"step (float64 C oracle, OpenMP over heads)" if info else ""},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


# algorithmic flops per (head, token) of each forward kernel, from the four parts of
# flops_per_head_token: the tensor-core solve also computes the per-token norm (fused)
KERNEL_PARTS = {"chunk_solve_tc": ("ch", "out", "nrm"), "chunk_solve": ("ch", "out"),
                "chunk_norm": ("nrm",), "chunk_delta": ("upd",), "state_pass_tc": ("upd",)}


def kernel_flops_per_head_token(name, D, C, r):
    ch, out, upd, nrm = flops_per_head_token(D, C, r)
    parts = {"ch": ch, "out": out, "upd": upd, "nrm": nrm}
    return sum(parts[x] for x in KERNEL_PARTS.get(name, ()))


def alu_peak_tflops(peaks):
    """fp32 FMA peak: 148 SMs x 128 lanes x 2 flop x max SM clock."""
    return 148 * 128 * 2 * peaks.get("sm_max_mhz", 1965.0) * 1e6 / 1e12


def forward_roofline(w, kt, steps, ms_per_step, peaks):
    """Roofline of the step's dominant kernel (largest summed device time) and the
    whole step's fraction of the bf16 tensor peak."""
    ch, out, upd, nrm = flops_per_head_token(w.D, w.chunk, w.r)
    head_tok = w.B * w.H * w.T
    dom_name, (dom_ms, dom_n) = max(kt.items(), key=lambda kv: kv[1][0])
    per_step_ms = dom_ms / steps
    kernel_flops = kernel_flops_per_head_token(dom_name, w.D, w.chunk, w.r) * head_tok
    if dom_name == "chunk_solve_tc":
        # fp16 operands, fp32 accumulation: the dense fp16 peak equals the bf16 one
        bound, peak = "tensor", peaks["bf16_tflops"]
        peak_note = f"dense bf16/fp16 tensor peak, {peaks['_source']} burst (cuBLAS bf16)"
    else:
        bound, peak = "alu", alu_peak_tflops(peaks)
        peak_note = "fp32 FMA: 148 SMs x 128 lanes x 2 flop x max SM clock"
    achieved = kernel_flops / (per_step_ms / 1e3) / 1e12
    whole_flops = (ch + out + upd + nrm) * head_tok
    tr = traffic_of(dom_name, w.name)
    return {"bound": bound, "kernel": dom_name, "achieved": achieved, "peak": peak,
            "unit": "TFLOP/s", "frac": achieved / peak,
            "traffic": None if tr is None else tr * (dom_n / steps),
            "peak_source": peak_note, "launches_per_step": dom_n / steps,
            "algorithmic_per_step": kernel_flops,
            "algorithmic_parts": "+".join(KERNEL_PARTS.get(dom_name, ())),
            "step_frac_of_bf16_peak": whole_flops / (ms_per_step / 1e3) / 1e12
            / peaks["bf16_tflops"]}


def time_forward(step, steps, warmup, flush, dev, barrier):
    """W warm-up steps, then K steps with L2 flushed before each, CUDA events per
    step on the launch stream and the SM clock sampled meanwhile; then the same K
    steps again under the library's launch profiler (per-kernel device times, kept
    out of the step times).  Returns (per-step ms, kernel times, clock summary)."""
    import torch
    from test_ridge_regression_b200 import gka
    for _ in range(max(warmup, 3)):
        step()
    torch.cuda.synchronize()
    if gka.device_status() != 0:
        raise RuntimeError("device status error after warm-up")
    starts = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
    barrier()
    torch.cuda.synchronize()
    with ClockSampler(dev.index) as clk:
        for i in range(steps):
            flush.fill_(float(i))
            starts[i].record()
            step()
            ends[i].record()
        torch.cuda.synchronize()
    barrier()
    step_ms = [s.elapsed_time(e) for s, e in zip(starts, ends)]
    gka.profiler_read()
    gka.profiler_enable(True)
    barrier()
    torch.cuda.synchronize()
    for i in range(steps):
        flush.fill_(float(i))
        step()
    torch.cuda.synchronize()
    barrier()
    gka.profiler_enable(False)
    kt = gka.profiler_read()
    if gka.device_status() != 0:
        raise RuntimeError("device status error after the timed steps")
    return step_ms, kt, clk.summary()


def bench_config(args, w, dev, peaks, flush):
    """One other forward workload (N = 1): the same timing as the main line, its
    own roofline and step fraction."""
    import torch
    from test_ridge_regression_b200 import gka
    from test_ridge_regression_b200.inputs import workload_inputs
    qd, kd, vd, bd = (t.to(dev) for t in workload_inputs(w))
    od = torch.empty_like(vd)
    ws = gka.alloc_workspace(w.B, w.H, w.T, w.D, w.chunk, w.dtype, dev)

    def step():
        gka.gka_forward(qd, kd, vd, bd, w.a, w.r, w.chunk, o=od, workspace=ws)

    steps = max(1, min(args.steps, 20))
    step_ms, kt, clk = time_forward(step, steps, args.warmup, flush, dev, lambda: None)
    ms = sum(step_ms) / steps
    out = {"workload": w.name, "B": w.B, "heads": w.H, "T": w.T, "D": w.D, "chunk": w.chunk,
           "a": w.a, "r": w.r, "dtype": "bf16" if w.dtype == torch.bfloat16 else "f32",
           "beta": f"sigmoid(N({w.beta_mu},{w.beta_sigma}))", "steps": steps,
           "ms_per_step": ms, "tokens_per_s": w.B * w.T / (ms / 1e3),
           "kernels_ms_per_step": {n: t / steps for n, (t, _) in kt.items()},
           "gpu_launches": sum(n for _, n in kt.values()),
           "roofline": forward_roofline(w, kt, steps, ms, peaks), "clocks": clk}
    del qd, kd, vd, bd, od, ws
    torch.cuda.empty_cache()
    return out


def main():
    args = parse()
    from test_ridge_regression_b200 import dist as gdist
    rank, world, local = gdist.rank_env()
    from test_ridge_regression_b200.inputs import WORKLOADS
    w = WORKLOADS[args.workload]
    cfg = {"workload": w.name, "B": w.B, "heads": w.H, "T": w.T, "D": w.D, "chunk": w.chunk,
           "a": w.a, "r": w.r, "beta": f"sigmoid(N({w.beta_mu},{w.beta_sigma}))",
           "global_batch": w.B * world, "seq_len": w.T, "parallelism": f"dp{world}",
           "l2": "flushed (256 MiB write) before every timed step"}
    if args.impl == "reference":
        run_reference(args, w, cfg, rank, world)
        return

    import torch
    import torch.distributed as dist
    from test_ridge_regression_b200 import build, gka
    from test_ridge_regression_b200.inputs import workload_inputs

    build.build()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        gdist.init("nccl", timeout_s=120, device=dev)

    def barrier():
        if world > 1:
            dist.barrier()

    peaks = load_peaks()
    # every rank runs its own batch (weak scaling over independent sequences)
    from dataclasses import replace as _replace
    q, k, v, beta = workload_inputs(_replace(w, seed=gdist.shard_seed(w.seed, rank)))
    qd, kd, vd, bd = (t.to(dev) for t in (q, k, v, beta))
    od = torch.empty_like(vd)
    ws = gka.alloc_workspace(w.B, w.H, w.T, w.D, w.chunk, w.dtype, dev)
    flush = torch.empty(256 * 1024 * 1024 // 4, dtype=torch.float32, device=dev)

    def step():
        gka.gka_forward(qd, kd, vd, bd, w.a, w.r, w.chunk, o=od, workspace=ws)

    step_ms, kt, clocks = time_forward(step, args.steps, args.warmup, flush, dev, barrier)
    total_ms = gdist.max_over_ranks(sum(step_ms), dev)
    ms_per_step = total_ms / args.steps
    tok_step = w.B * w.T
    value = world * tok_step * args.steps / (total_ms / 1e3)
    launches = sum(n for _, n in kt.values())
    roofline = forward_roofline(w, kt, args.steps, ms_per_step, peaks)

    result = {
        "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_per_step,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic", "config": cfg, "roofline": roofline, "gpu_launches": launches,
        "kernels_ms_per_step": {n: ms / args.steps for n, (ms, _) in kt.items()},
        "clocks": clocks,
    }

    # ---- end to end: the library's host-buffer forward (pinned host buffers; the
    # copies in and out are inside the timed region, overlapped with the compute
    # of other slices of the batch) ----
    qh, kh, vh, bh = (t.pin_memory() for t in (q, k, v, beta))
    oh = torch.empty(q.shape, dtype=q.dtype).pin_memory()
    hws = gka.alloc_host_workspace(w.B, w.H, w.T, w.D, w.chunk, w.dtype, 0, dev)

    def e2e_step():
        gka.gka_forward_host(qh, kh, vh, bh, w.a, w.r, w.chunk, o=oh, workspace=hws)

    e_starts = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    e_ends = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    for _ in range(max(args.warmup, 3)):
        e2e_step()
    torch.cuda.synchronize()
    barrier()
    for i in range(args.steps):
        flush.fill_(float(i))
        e_starts[i].record()
        e2e_step()
        e_ends[i].record()
    torch.cuda.synchronize()
    barrier()
    e_ms = gdist.max_over_ranks(sum(s.elapsed_time(e) for s, e in zip(e_starts, e_ends)), dev)
    h2d = sum(t.numel() * t.element_size() for t in (q, k, v, beta))
    result["e2e"] = {"value": world * tok_step * args.steps / (e_ms / 1e3), "unit": "tokens/s",
                     "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": oh.numel() * oh.element_size(),
                     "api": "gka_forward_host (slices of the batch pipelined over two copy streams)"}
    if gka.device_status() != 0:
        raise RuntimeError("device status error after the end-to-end steps")
    del qh, kh, vh, bh, oh

    # ---- write-gated forward on the same inputs plus a gate ----
    if not args.no_write_gate:
        result["write_gate"] = bench_write_gate(args, w, dev, qd, kd, vd, bd, od, ws, flush,
                                                rank, world, barrier)

    # ---- backward pass (implicit differentiation) on the same inputs ----
    if not args.no_backward:
        result["backward"] = bench_backward(args, w, dev, qd, kd, vd, bd, flush, rank, world,
                                            barrier, peaks)

    # ---- solver study: Chebyshev vs gradient descent, Nesterov, conjugate gradient ----
    if not args.no_solver_study and world == 1:
        result["solver_study"] = bench_solver_study(w, qd, kd, bd, peaks)

    # ---- decode step: HBM-bound, 256 x 32 heads, fp32 state ----
    if not args.no_decode and world == 1:
        result["decode"] = bench_decode(args, dev, peaks)

    # ---- the other forward workloads (N = 1): every config, timed like the main line ----
    if not args.no_configs and world == 1:
        from test_ridge_regression_b200.inputs import WORKLOADS as _W
        result["configs"] = {name: bench_config(args, cw, dev, peaks, flush)
                             for name, cw in _W.items() if name != w.name}

    # ---- CPU baseline: the oracle on a bounded sample (rank 0, N = 1) ----
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        nheads = oracle_calibrate(w, 10.0, q, k, v, beta)
        vals, total, reps = [], 0.0, 0
        while total < 10.0 and reps < 50:   # the whole sample, repeated to about 10 s
            val, dt, threads = oracle_sample(w, nheads, q, k, v, beta)
            vals.append(val)
            total += dt
            reps += 1
        result["cpu_baseline"] = {
            "value": statistics.mean(vals), "unit": "tokens/s", "cores": threads, "kind": "oracle",
            "sample": f"{nheads} whole heads x {w.T} tokens of the workload, {reps} runs, "
                      f"{total:.1f} s (float64 C oracle, OpenMP over heads)"}
    if gka.device_status() != 0:
        raise RuntimeError("device status error")
    if rank == 0:
        print(json.dumps(result), flush=True)
    if world > 1:
        dist.destroy_process_group()


def bench_write_gate(args, w, dev, qd, kd, vd, bd, od, ws, flush, rank, world, barrier):
    """The paper's beta_t-augmented variant (a per-token write gate in [0, 1],
    gka_forward_gated) on the workload's inputs: K steps timed like the main ones,
    then the same K steps under the launch profiler for the per-kernel times."""
    import torch
    from test_ridge_regression_b200 import dist as gdist
    from test_ridge_regression_b200 import gka
    from test_ridge_regression_b200.inputs import make_gate
    gd = make_gate((w.B, w.H, w.T), gdist.shard_seed(w.seed, rank)).to(dev)

    def step():
        gka.gka_forward_gated(qd, kd, vd, bd, gd, w.a, w.r, w.chunk, o=od, workspace=ws)

    for _ in range(max(args.warmup, 3)):
        step()
    starts = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    torch.cuda.synchronize()
    barrier()
    for i in range(args.steps):
        flush.fill_(float(i))
        starts[i].record()
        step()
        ends[i].record()
    torch.cuda.synchronize()
    barrier()
    total_ms = gdist.max_over_ranks(sum(s.elapsed_time(e) for s, e in zip(starts, ends)), dev)
    gka.profiler_read()
    gka.profiler_enable(True)
    for i in range(args.steps):
        flush.fill_(float(i))
        step()
    torch.cuda.synchronize()
    gka.profiler_enable(False)
    kt = gka.profiler_read()
    if gka.device_status() != 0:
        raise RuntimeError("device status error after the write-gated steps")
    return {"gate": "sigmoid(N(0,1.5)) per token, fp32", "ms_per_step": total_ms / args.steps,
            "tokens_per_s": world * w.B * w.T * args.steps / (total_ms / 1e3),
            "kernels_ms_per_step": {n: ms / args.steps for n, (ms, _) in kt.items()},
            "gpu_launches": sum(n for _, n in kt.values())}


BWD_CHUNK = 32


def bwd_flops_per_head_token(D, C, r):
    """Algorithmic flops of each backward kernel per (head, token), causal C x C
    products counted as dense tiles (2 flops per multiply-add)."""
    ch = (r - 1) * (2 * D * D + 4 * C * D)
    return {
        "chunk_solve": ch,                                  # forward iterates, recomputed
        "bwd_solve": (2 * D * D + 4 * C * D) + ch,          # u = M^T g, then the iteration
        "bwd_delta": 6 * D * D,                             # three rank-C products per chunk
        "bwd_rows": 14 * D * D,                             # seven row-times-matrix products
        "bwd_grads": 16 * C * D,                            # four C x C x D dots, four C x C x D sums
        "chunk_delta": 4 * D * D, "chunk_norm": 2 * D * D + 2 * C * D + 2 * C * C,
    }


def bench_backward(args, w, dev, qd, kd, vd, bd, flush, rank, world, barrier, peaks):
    """gka_backward on the workload's inputs with a seeded upstream gradient: K steps
    timed like the forward's, then the same steps under the launch profiler."""
    import torch
    from test_ridge_regression_b200 import dist as gdist
    from test_ridge_regression_b200 import gka
    g = torch.Generator(device=dev).manual_seed(gdist.shard_seed(w.seed, rank) + 77)
    dout = torch.randn(qd.shape, generator=g, device=dev).to(qd.dtype)
    ws = torch.empty(gka.backward_workspace_bytes(w.B, w.H, w.T, w.D, BWD_CHUNK, w.dtype),
                     dtype=torch.uint8, device=dev)
    steps = max(1, min(args.steps, 10))

    def step():
        return gka.gka_backward(qd, kd, vd, bd, dout, w.a, w.r, BWD_CHUNK, workspace=ws)

    for _ in range(max(args.warmup, 3)):
        step()
    starts = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
    torch.cuda.synchronize()
    barrier()
    for i in range(steps):
        flush.fill_(float(i))
        starts[i].record()
        step()
        ends[i].record()
    torch.cuda.synchronize()
    barrier()
    total_ms = gdist.max_over_ranks(sum(s.elapsed_time(e) for s, e in zip(starts, ends)), dev)
    gka.profiler_read()
    gka.profiler_enable(True)
    for i in range(steps):
        flush.fill_(float(i))
        step()
    torch.cuda.synchronize()
    gka.profiler_enable(False)
    kt = gka.profiler_read()
    if gka.device_status() != 0:
        raise RuntimeError("device status error after the backward steps")
    per_kernel = {n: ms / steps for n, (ms, _) in kt.items()}
    fl = bwd_flops_per_head_token(w.D, BWD_CHUNK, w.r)
    head_tok = w.B * w.H * w.T
    # roofline of the largest of the backward's own kernels (the forward recompute's
    # kernels have theirs in the forward leg)
    own = {n: t for n, t in per_kernel.items() if n.startswith("bwd_") or n == "adjoint_scan"}
    dom = max(own or per_kernel, key=(own or per_kernel).get)
    peak = 148 * 128 * 2 * peaks.get("sm_max_mhz", 1965.0) * 1e6 / 1e12
    total_fl = sum(fl[n] for n in per_kernel if n in fl) * head_tok
    tc_path = w.dtype == torch.bfloat16 and w.D == 128 and BWD_CHUNK == 32 and w.T % 64 == 0
    # the tensor-core kernels of the backward are bound by what they must move
    hbm = {}
    if tc_path:
        D, C = w.D, BWD_CHUNK
        # row products: per chunk the fp16 copies of H_s, M_s, E^H, E^M; the k, v, g
        # (bf16) and x, y (fp32) rows in, R1..R4 and the per-token scalars out
        rows_tok = 4 * D * D * 2 / C + 3 * D * 2 + 2 * D * 4 + 4 * D * 4 + 4 * 4
        # adjoint pass: per chunk the two state copies in and the two adjoint copies out
        # (fp16); the y, x (fp32) and k, g (bf16) rows, beta and c in
        adj_tok = 4 * D * D * 2 / C + 2 * D * 4 + 2 * D * 2 + 2 * 4
        for name, per_tok, key in (("bwd_rows", rows_tok, "bwd_rows_tc"),
                                   ("adjoint_scan", adj_tok, "adjoint_pass_tc")):
            if name not in per_kernel:
                continue
            byts = per_tok * head_tok
            ach = byts / (per_kernel[name] / 1e3) / 1e9
            hbm[name] = {"bound": "hbm", "kernel": name, "achieved": ach,
                         "peak": peaks["hbm_gbs"], "unit": "GB/s", "frac": ach / peaks["hbm_gbs"],
                         "traffic": traffic_of(key, w.name),
                         "peak_source": "measured copy bandwidth", "algorithmic_per_step": byts}
    if dom in hbm:
        roof = hbm[dom]
    else:
        achieved = fl.get(dom, 0) * head_tok / (per_kernel[dom] / 1e3) / 1e12
        roof = {"bound": "alu", "kernel": dom, "achieved": achieved, "peak": peak,
                "unit": "TFLOP/s", "frac": achieved / peak, "traffic": None,
                "peak_source": "fp32 FMA: 148 SMs x 128 lanes x 2 flop x max SM clock",
                "algorithmic_per_step": fl.get(dom, 0) * head_tok}
    return {"chunk": BWD_CHUNK, "steps": steps, "ms_per_step": total_ms / steps,
            "tokens_per_s": world * w.B * w.T * steps / (total_ms / 1e3),
            "kernels_ms_per_step": per_kernel,
            "gpu_launches": sum(n for _, n in kt.values()),
            "roofline": roof,
            "hbm_rooflines": hbm,
            "step_frac_of_fp32_peak": total_fl / (total_ms / steps / 1e3) / 1e12 / peak}


def bench_solver_study(w, qd, kd, bd, peaks):
    """Residual histories of the four solvers on every token of the workload (the
    pages' Fig. 1a on its random-regression shape) and the final mean residual for
    several regularisation strengths (Fig. 8); one timed run per solver at the
    workload's a and r."""
    import torch
    from test_ridge_regression_b200 import gka
    chunk = 64
    out = {"chunk": chunk, "r": w.r, "a": w.a, "mean_residual": {}, "ms": {}}
    for solver in gka.SOLVERS:
        gka.gka_solver_study(qd, kd, bd, w.a, w.r, solver, chunk)   # warm-up
        s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        s.record()
        res = gka.gka_solver_study(qd, kd, bd, w.a, w.r, solver, chunk)
        e.record()
        torch.cuda.synchronize()
        out["ms"][solver] = s.elapsed_time(e)
        out["mean_residual"][solver] = [float(x) for x in res.double().mean(dim=(0, 1, 2))]
    sweep = {}
    for a in (0.5, 0.1, 0.05, 0.02):
        sweep[str(a)] = {solver: float(gka.gka_solver_study(qd, kd, bd, a, 30, solver, chunk)
                                       [..., -1].double().mean())
                         for solver in gka.SOLVERS}
    out["a_sweep_final_mean_residual_r30"] = sweep
    # ALU roofline of the study kernel (Chebyshev run): r products A x per token, each
    # 2 D^2 + 4 C D flops in chunk form (CG takes two per step)
    head_tok = w.B * w.H * w.T
    fl = w.r * (2 * w.D * w.D + 4 * chunk * w.D) * head_tok
    peak = 148 * 128 * 2 * peaks.get("sm_max_mhz", 1965.0) * 1e6 / 1e12
    ach = fl / (out["ms"]["chebyshev"] / 1e3) / 1e12
    out["roofline"] = {"bound": "alu", "kernel": "solver_study (chebyshev)", "achieved": ach,
                       "peak": peak, "unit": "TFLOP/s", "frac": ach / peak,
                       "algorithmic_per_run": fl,
                       "peak_source": "fp32 FMA: 148 SMs x 128 lanes x 2 flop x max SM clock"}
    if gka.device_status() != 0:
        raise RuntimeError("device status error after the solver study")
    return out


def bench_decode(args, dev, peaks):
    import torch
    from test_ridge_regression_b200 import gka
    from dataclasses import replace
    from test_ridge_regression_b200.inputs import DECODE as w
    if args.decode_batch:
        w = replace(w, batch=args.decode_batch)
    gen = torch.Generator(device=dev)
    gen.manual_seed(w.seed)

    def draw(b, h, t):
        qq = torch.randn(b, h, t, w.D, generator=gen, device=dev)
        kk = torch.randn(b, h, t, w.D, generator=gen, device=dev)
        vv = torch.randn(b, h, t, w.D, generator=gen, device=dev)
        bb = torch.sigmoid(w.beta_mu + w.beta_sigma * torch.randn(b, h, t, generator=gen,
                                                                   device=dev))
        qq = (qq / qq.norm(dim=-1, keepdim=True)).to(torch.bfloat16)
        kk = (kk / kk.norm(dim=-1, keepdim=True)).to(torch.bfloat16)
        return qq, kk, vv.to(torch.bfloat16), bb.contiguous()

    # prefill through the forward path: the decode state is its final state
    state = torch.empty(w.batch, w.H, 2, w.D, w.D, device=dev)
    pq, pk, pv, pb = draw(w.batch, w.H, w.prefill)
    gka.gka_forward(pq, pk, pv, pb, w.a, w.r, 64, final_state=state)
    del pq, pk, pv, pb
    torch.cuda.empty_cache()
    nsets = 16
    sets = [tuple(x[:, :, 0].contiguous() for x in draw(w.batch, w.H, 1)) for _ in range(nsets)]
    o = torch.empty(w.batch, w.H, w.D, dtype=torch.bfloat16, device=dev)
    steps = args.decode_steps or w.steps
    for i in range(5):
        qq, kk, vv, bb = sets[i % nsets]
        gka.gka_decode_step(state, qq, kk, vv, bb, w.a, w.r, o=o)
    torch.cuda.synchronize()
    gka.profiler_read()
    gka.profiler_enable(True)
    s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(dev.index) as clk:
        s.record()
        for i in range(steps):
            qq, kk, vv, bb = sets[i % nsets]
            gka.gka_decode_step(state, qq, kk, vv, bb, w.a, w.r, o=o)
        e.record()
        torch.cuda.synchronize()
    gka.profiler_enable(False)
    kt = gka.profiler_read()
    ms = s.elapsed_time(e) / steps
    heads = w.batch * w.H
    bytes_step = heads * (4 * w.D * w.D * 4 + 4 * w.D * 2 + 4)
    k_ms, k_n = kt["decode_step"]
    achieved = bytes_step / (k_ms / k_n / 1e3) / 1e9
    return {
        "workload": w.name, "steps": steps, "ms_per_step": ms,
        "tokens_per_s": w.batch / (ms / 1e3), "GB_per_s": bytes_step / (ms / 1e3) / 1e9,
        "roofline": {"bound": "hbm", "kernel": "decode_step", "achieved": achieved,
                     "peak": peaks["hbm_gbs"], "unit": "GB/s",
                     "frac": achieved / peaks["hbm_gbs"],
                     "traffic": traffic_of("decode_step", w.name) if w.batch == 256 else None,
                     "algorithmic_per_launch": bytes_step,
                     "peak_source": f"{peaks['_source']} copy bandwidth"},
        "gpu_launches": k_n, "clocks": clk.summary(),
    }


if __name__ == "__main__":
    main()
