#!/usr/bin/env python
"""Throughput of the exact-attention hot path on B200, one JSON line on rank 0.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

A step is one pass of the whole path over the causal LLM-shape workload
(B=2, H=32, N=4096, d=128, causal; inputs N(0,1)*0.5 in bf16): the forward
kernel (O and logsumexp) followed, when the library has it, by the backward
with recomputation (dQ, dK, dV from Q, K, V, O, dO and L).  Throughput is
TFLOP/s with the usual convention: forward 4*B*H*N^2*d, halved for causal;
backward 2.5x the forward.

Timing: W untimed warm-up steps, then K steps bracketed by a barrier and a
device synchronise; every step is timed with CUDA events on the launching
stream and L2 is flushed (256 MB write) between steps, outside the events.
With N > 1 ranks (torchrun, NCCL) every rank runs its own copy of the
workload (independent heads: weak scaling, no collective on the data path)
and the time is the max over ranks.

--impl reference times the fp64 CPU oracle (the definition of the result,
not a GPU program) on a bounded row-block sample of the same workload.
"""

from __future__ import annotations

import argparse
import datetime
import json
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

WORKLOAD = "causal"          # forward workload; the backward uses the same shape
GRAD_WORKLOAD = "bwd"
# --workload choices: the forward workload and the one whose dO seed the backward uses
BENCH_WORKLOADS = {"causal": ("causal", "bwd"), "long": ("long", "long"), "swa": ("swa", "swa"),
                   "gqa": ("gqa", "gqa"), "decode": ("decode", "decode"), "decode_fp8": ("decode", "decode"),
                   "d256": ("d256", "d256"), "fp8": ("causal", "bwd"), "tiny": ("tiny", "tiny"),
                   "gpt2": ("gpt2", "gpt2")}
# workloads timed as a forward alone (the configurations that name only O and the logsumexp)
FORWARD_ONLY = ("tiny", "gpt2")
FLUSH_BYTES = 256 << 20      # > 126 MB L2
PEAKS_FILE = os.path.join(ROOT, "MEASURED_PEAKS.json")
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def parse_args():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=1000)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--e2e-steps", type=int, default=20)
    ap.add_argument("--cpu-seconds", type=float, default=12.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--workload", choices=sorted(BENCH_WORKLOADS), default="causal",
                    help="causal: B2 H32 N4096 d128 (the default line); gqa: the same with 8 K/V heads; "
                         "long / swa: N32768 with a one- / two-sided window of 4096, FLOPs counted over "
                         "the pairs the band keeps; decode: one new row per query head over 32768 "
                         "cached keys (B8, 64 query heads on 8 K/V heads), forward only, HBM-bound; "
                         "decode_fp8: the same over an E4M3 K/V cache with per-tensor scales; "
                         "d256: B2 H16 N4096 head dimension 256, causal, forward+backward; "
                         "fp8: the causal shape's forward on E4M3 Q, K, V (V transposed); "
                         "tiny: B1 H2 N128 d64 forward (launch/HBM-bound: reported against the HBM "
                         "peak); gpt2: B4 H16 N2048 d64 non-causal forward")
    return ap.parse_args()


# ----------------------------------------------------------------------------- FLOPs
def band_pairs(N, causal, window) -> int:
    """(query, key) pairs a banded mask keeps in N x N self-attention (closed forms)."""
    w = min(window, N)
    if causal:
        return w * (w + 1) // 2 + (N - w) * w
    return N * (2 * w - 1) - w * (w - 1)


def fwd_flops(B, H, N, d, causal, window=0) -> float:
    """4 B H N^2 d, halved if causal; with a window, 4 d per pair the band keeps."""
    if window > 0:
        return 4.0 * B * H * d * band_pairs(N, causal, window)
    f = 4.0 * B * H * N * N * d
    return f / 2 if causal else f


def bwd_flops(B, H, N, d, causal, window=0) -> float:
    return 2.5 * fwd_flops(B, H, N, d, causal, window)


def decode_band(pos, n_k, causal, window):
    """Closed interval of keys a query at key position pos may attend (the mask readings)."""
    lo = max(0, pos - window + 1) if window > 0 else 0
    if causal:
        hi = pos
    elif window > 0:
        hi = min(n_k - 1, pos + window - 1)
    else:
        hi = n_k - 1
    return lo, hi


def decode_pairs(n_q, n_k, causal, window) -> int:
    """(query, key) pairs kept when n_q new rows stand at the last n_q of n_k key positions."""
    total = 0
    for i in range(n_q):
        lo, hi = decode_band(n_k - n_q + i, n_k, causal, window)
        total += hi - lo + 1
    return total


def decode_flops(B, H, n_q, n_k, d, causal, window=0) -> float:
    """4 d per kept (query, key) pair: Q K^T and P V, two flops per multiply-add."""
    return 4.0 * B * H * d * decode_pairs(n_q, n_k, causal, window)


def decode_bytes(B, H, H_kv, n_q, n_k, d, causal, window=0, kv_elem_bytes=2) -> int:
    """Algorithmic HBM bytes of a decode forward: read Q (bf16) and, once, the K and V rows
    of the keys any new row may attend (kv_elem_bytes each: 2 for bf16, 1 for E4M3); write O
    (bf16) and L (fp32)."""
    lo, _ = decode_band(n_k - n_q, n_k, causal, window)
    _, hi = decode_band(n_k - 1, n_k, causal, window)
    keys = hi - lo + 1
    return 2 * B * H * n_q * d * 2 + 2 * B * H_kv * keys * d * kv_elem_bytes + B * H * n_q * 4


def kernel_names(d: int):
    """(forward kernel, backward main kernel) names for head dimension d."""
    if d == 256:
        return "fa_fwd256_kernel", "fa_bwd256_kernel"
    return f"fa_fwd_kernel<{d}>", f"fa_bwd_kernel<{d}>"


def max_over_ranks(values, device=None):
    """Element-wise max of a list of floats over all ranks (identity without a process group).

    Every rank calls it with the same number of values at the same point of the program.
    """
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return list(values)
    t = torch.tensor(list(values), dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return t.tolist()


def job_throughput(world: int, flops_per_rank_step: float, ms_per_step: float) -> float:
    """Whole-job TFLOP/s: every rank processed its own copy of the workload in ms_per_step."""
    return world * flops_per_rank_step / (ms_per_step * 1e-3) / 1e12


def load_peaks():
    try:
        with open(PEAKS_FILE) as f:
            p = json.load(f)
        return p, "measured"
    except Exception:
        return FALLBACK_PEAKS, "fallback"


# A timed region at least this long runs at the clock the 1 kW power cap settles to; a shorter
# one mostly at the boost clock.  The measured peaks come in both regimes.
SUSTAINED_MS = 1000.0


def regime_fields(roofline: dict, clocks: dict, timed_ms: float, kernel_ms: float, peaks: dict, scale: float = 1.0):
    """Add to a tensor-bound roofline the regime of the timed region and the fraction of the other
    regime's peak, and return the clock-normalised figures: the dominant kernel's time scaled to
    the maximum SM clock (time x median MHz / max MHz) and its throughput at that time.  `scale`
    converts the bf16 peaks to the kernel's own type (the FP8 arm)."""
    regime = "sustained" if timed_ms >= SUSTAINED_MS else "burst"
    burst, sustained = peaks["bf16_tflops"] * scale, peaks["bf16_tflops_sustained"] * scale
    roofline["regime"] = regime
    if regime == "sustained":
        roofline["peak"] = round(sustained, 1)
        roofline["frac"] = round(roofline["achieved"] / sustained, 4)
        roofline["peak_source"] = roofline["peak_source"].replace("burst", "sustained")
    roofline["timed_region_ms"] = round(timed_ms, 1)
    roofline["frac_of_burst_peak"] = round(roofline["achieved"] / burst, 4)
    roofline["frac_of_sustained_peak"] = round(roofline["achieved"] / sustained, 4)
    mhz, mhz_max = clocks.get("sm_mhz"), clocks.get("sm_max_mhz")
    if not mhz or not mhz_max:
        return None
    t_norm = kernel_ms * mhz / mhz_max
    return {"sm_mhz_median": mhz, "sm_max_mhz": mhz_max, "samples_in_window": clocks.get("samples"),
            "kernel": roofline["kernel"], "kernel_ms_at_max_clock": round(t_norm, 5),
            "achieved_at_max_clock": round(roofline["achieved"] * kernel_ms / t_norm, 1),
            "frac_at_max_clock": round(roofline["achieved"] * kernel_ms / t_norm / burst, 4)}


# ----------------------------------------------------------------------------- clocks
class ClockSampler:
    """nvidia-smi samples (every 100 ms) of SM clock and throttle reasons."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
    REASONS = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")

    def __init__(self, gpu_id: str):
        self.gpu_id = gpu_id
        self.samples = []
        self.proc = None
        self.thread = None
        self.window = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", self.gpu_id, f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None
            return
        self.thread = threading.Thread(target=self._read, daemon=True)
        self.thread.start()

    def _read(self):
        for line in self.proc.stdout:
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm, smax = float(parts[1]), float(parts[2])
            except ValueError:
                continue
            self.samples.append((time.time(), sm, smax, parts[5:9]))

    def mark(self, t0, t1):
        self.window = (t0, t1)

    def stop(self):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()
        if self.thread is not None:
            self.thread.join(timeout=2)

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        t0, t1 = self.window or (0, float("inf"))
        inside = [s for s in self.samples if t0 - 0.05 <= s[0] <= t1 + 0.05]
        used = inside if inside else self.samples
        reasons = sorted({name for s in used for name, flag in zip(self.REASONS, s[3])
                          if flag.lower() == "active"})
        return {"sm_mhz": statistics.median(s[1] for s in used),
                "sm_max_mhz": max(s[2] for s in used), "reasons": reasons,
                "samples": len(inside), "samples_total": len(self.samples)}


def gpu_id_for(dev_index: int) -> str:
    import torch
    try:
        uuid = str(torch.cuda.get_device_properties(dev_index).uuid)
        return uuid if uuid.startswith("GPU-") else "GPU-" + uuid
    except Exception:
        vis = os.environ.get("CUDA_VISIBLE_DEVICES")
        if vis:
            return vis.split(",")[dev_index]
        return str(dev_index)


# ----------------------------------------------------------------------------- CPU oracle
def oracle_sample(seconds: float, rows_per_block: int = 512, with_bwd: bool = True,
                  max_blocks: int | None = None):
    """Time the fp64 oracle on contiguous query-row blocks of head 0 of the workload.

    Returns (flops credited, seconds, blocks, cores).  A block of R rows is credited
    R/N of one head's conventional forward (+ backward) FLOPs.
    """
    import numpy as np
    from oracle import attention as orc
    from synthetic import WORKLOADS, make_grad_output, make_inputs
    wl = WORKLOADS[WORKLOAD]
    sub = wl.with_(B=1, H=1, H_kv=None)
    q, k, v = (x[0, 0].double().numpy() for x in make_inputs(sub))
    do = None
    if with_bwd:
        do = make_grad_output(WORKLOADS[GRAD_WORKLOAD].with_(B=1, H=1, H_kv=None))[0, 0].double().numpy()
    per_row = fwd_flops(1, 1, wl.N, wl.d, wl.causal, wl.window) / wl.N
    if with_bwd:
        per_row += bwd_flops(1, 1, wl.N, wl.d, wl.causal, wl.window) / wl.N
    t0 = time.perf_counter()
    blocks = 0
    start = 0
    while True:
        rows = np.arange(start, start + rows_per_block) % wl.N
        orc.attention_forward_rows(q, k, v, wl.scale, wl.causal, wl.window, rows=rows)
        if with_bwd:
            orc.attention_backward_rows(q, k, v, do, wl.scale, wl.causal, wl.window, query_rows=rows)
        blocks += 1
        start = (start + rows_per_block) % wl.N
        el = time.perf_counter() - t0
        if el >= seconds or (max_blocks is not None and blocks >= max_blocks):
            break
    return per_row * rows_per_block * blocks, el, blocks, blas_threads()


def blas_threads() -> int:
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 0) for i in threadpool_info() if i.get("user_api") == "blas"]
        if n:
            return int(max(n))
    except Exception:
        pass
    return os.cpu_count() or 1


# ----------------------------------------------------------------------------- GPU arm
def run_ours(args):
    import torch
    import torch.distributed as dist

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        dist.init_process_group("nccl", device_id=dev, timeout=datetime.timedelta(seconds=300))

    import exact_io_aware_77_b200 as fa
    fa.load()                                    # no library, no bench: fails loudly
    from synthetic import WORKLOADS, make_grad_output, make_inputs

    wl = WORKLOADS[WORKLOAD]
    B, H, N, d = wl.B, wl.H, wl.N, wl.d
    names = kernel_names(d)
    has_bwd = hasattr(fa, "backward")
    q_h, k_h, v_h = make_inputs(wl)
    do_h = make_grad_output(WORKLOADS[GRAD_WORKLOAD])
    q, k, v, do = (x.to(dev) for x in (q_h, k_h, v_h, do_h))
    o = torch.empty_like(q)
    lse = torch.empty((B, H, N), dtype=torch.float32, device=dev)
    grads = (torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)) if has_bwd else None
    ws = None
    if has_bwd:
        ws = torch.empty(fa.bwd_workspace_size(B, H, N, d), dtype=torch.uint8, device=dev)
    flush = torch.empty(FLUSH_BYTES, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)

    f_fwd = fwd_flops(B, H, N, d, wl.causal, wl.window)
    f_bwd = bwd_flops(B, H, N, d, wl.causal, wl.window) if has_bwd else 0.0

    def step(ev=None):
        # forward, then the backward as its three phases (exactly fa_bwd) so that the recompute
        # kernel, the dominant one, has events of its own
        if ev:
            ev[0].record(stream)
        fa.forward(q, k, v, wl.scale, wl.causal, wl.window, out=o, lse=lse)
        if ev:
            ev[1].record(stream)
        if has_bwd:
            for i, ph in enumerate((1, 2, 4)):
                fa.backward(q, k, v, o, lse, do, wl.scale, wl.causal, wl.window, grads=grads, workspace=ws,
                            phases=ph)
                if ev:
                    ev[2 + i].record(stream)

    for _ in range(args.warmup):
        flush.zero_()
        step()
    st = fa.check_status(dev)
    if st != 0:
        raise RuntimeError(f"device status after warm-up: {fa.STATUS_NAMES.get(st, st)}")

    sampler = ClockSampler(gpu_id_for(local))
    sampler.start()
    time.sleep(0.3)
    n_ev = 5 if has_bwd else 2
    events = [[torch.cuda.Event(enable_timing=True) for _ in range(n_ev)] for _ in range(args.steps)]
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize(dev)
    wall0 = time.time()
    for i in range(args.steps):
        flush.zero_()
        step(events[i])
    torch.cuda.synchronize(dev)
    wall1 = time.time()
    if world > 1:
        dist.barrier()
    sampler.mark(wall0, wall1)
    time.sleep(0.25)
    sampler.stop()
    st = fa.check_status(dev)
    if st != 0:
        raise RuntimeError(f"device status after timing: {fa.STATUS_NAMES.get(st, st)}")

    fwd_ms = [e[0].elapsed_time(e[1]) for e in events]
    bwd_ms = [e[1].elapsed_time(e[4]) for e in events] if has_bwd else [0.0] * args.steps
    main_ms = [e[2].elapsed_time(e[3]) for e in events] if has_bwd else [0.0] * args.steps
    step_ms_total = sum(f + b for f, b in zip(fwd_ms, bwd_ms))
    fwd_total, bwd_total, main_total = sum(fwd_ms), sum(bwd_ms), sum(main_ms)
    step_ms_total, fwd_total, bwd_total, main_total = max_over_ranks(
        [step_ms_total, fwd_total, bwd_total, main_total], dev)
    ms_per_step = step_ms_total / args.steps
    value = job_throughput(world, f_fwd + f_bwd, ms_per_step)

    # end to end through the public API: pinned host inputs -> device -> path -> host outputs
    e2e = None
    if not args.no_e2e:
        e2e = measure_e2e(fa, torch, wl, dev, stream, q_h, k_h, v_h, do_h, has_bwd, args.e2e_steps,
                          f_fwd + f_bwd, world)

    peaks, peak_kind = load_peaks()
    fwd_ms_avg = fwd_total / args.steps
    bwd_ms_avg = bwd_total / args.steps
    main_ms_avg = main_total / args.steps
    if has_bwd and main_ms_avg > fwd_ms_avg:
        # the backward's conventional FLOPs are all tensor work of the recompute kernel
        dom, dom_flops, dom_ms = names[1], f_bwd, main_ms_avg
    else:
        dom, dom_flops, dom_ms = names[0], f_fwd, fwd_ms_avg
    achieved = dom_flops / (dom_ms * 1e-3) / 1e12
    # a long timed region runs under the power cap: its kernel is compared with the sustained peak
    sustained = step_ms_total >= SUSTAINED_MS
    peak = peaks["bf16_tflops_sustained" if sustained else "bf16_tflops"]
    roofline = {"bound": "tensor", "kernel": dom, "achieved": round(achieved, 1),
                "peak": peak, "unit": "TFLOP/s",
                "frac": round(achieved / peak, 4),
                "peak_source": (f"{peak_kind} {'sustained' if sustained else 'burst'} bf16 (MEASURED_PEAKS.json)"
                                if peak_kind == "measured" else "fallback (1.59 PFLOP/s burst, 1.4 sustained)"),
                # the ncu counters were taken on the default causal workload only
                "traffic": load_traffic(dom) if WORKLOAD == "causal" else None}

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        flops, secs, blocks, cores = oracle_sample(args.cpu_seconds, with_bwd=has_bwd)
        cpu = {"value": round(flops / secs / 1e12, 6), "unit": "TFLOP/s", "cores": cores, "kind": "oracle",
               "sample": f"{blocks} blocks of 512 query rows of head 0 of the {wl.name} workload "
                         f"(B{wl.B} H{wl.H} N{wl.N} d{wl.d}) through the fp64 oracle "
                         f"({'fwd+bwd' if has_bwd else 'fwd'}), {secs:.1f} s, credited rows/N of a "
                         f"head's FLOPs"}

    clocks = sampler.summary()
    clock_norm = regime_fields(roofline, clocks, step_ms_total, dom_ms, peaks)
    line = {
        "metric": "attention fwd/bwd TFLOP/s at 1 B200; % of dense BF16 tensor peak",
        "value": round(value, 2), "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(ms_per_step, 4), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": workload_text(wl, has_bwd),
                   "global_batch": B * world, "seq_len": N, "parallelism": f"replicas{world}",
                   "l2": "flushed (256 MB write) between timed steps, outside the events",
                   "grids": "one CTA per work item, heads in chunks, the costliest items of a chunk first"},
        "fwd_tflops": round(job_throughput(world, f_fwd, fwd_ms_avg), 2),
        "fwd_ms": round(fwd_ms_avg, 4),
        "pct_of_measured_peak": round(100 * value / world / peaks["bf16_tflops"], 2),
        "pct_of_spec_peak_2250": round(100 * value / world / 2250.0, 2),
        "roofline": roofline,
        "cpu_baseline": cpu,
        "e2e": e2e,
        "gpu_launches": args.steps * (1 + (3 if has_bwd else 0)),
        "kernel_ms": {names[0]: round(fwd_ms_avg, 4),
                      "fa_bwd_prep+" + names[1] + "+fa_bwd_dq_final": round(bwd_ms_avg, 4),
                      names[1]: round(main_ms_avg, 4)} if has_bwd else None,
        "clocks": clocks,
        "clock_normalised": clock_norm,
    }
    if has_bwd:
        line["bwd_tflops"] = round(job_throughput(world, f_bwd, bwd_ms_avg), 2)
        line["bwd_ms"] = round(bwd_ms_avg, 4)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(line), flush=True)


def measure_e2e(fa, torch, wl, dev, stream, q_h, k_h, v_h, do_h, has_bwd, steps, flops, world):
    """The step through the public API with its host copies inside the timed region: every step
    copies its inputs from pinned host memory to the device and its results (O, L and, with the
    backward, dQ, dK, dV) back to pinned host memory.

    Pipelined as a training or serving loop runs: two device buffer sets, the host-to-device
    copies on one stream, the compute on the current stream and the device-to-host copies on a
    third, so that step i+1's inputs and step i-1's results cross PCIe while step i computes
    (each copy engine moves one direction).  Should the pipelined form fail, the serial one
    (copy in, compute, copy out on one stream) is measured instead and named in ``mode``."""
    pin = [x.pin_memory() for x in (q_h, k_h, v_h, do_h if has_bwd else q_h[:0])]
    o_h = torch.empty_like(pin[0]).pin_memory()
    l_h = torch.empty((wl.B, wl.H, wl.N), dtype=torch.float32).pin_memory()
    grads_h = tuple(torch.empty_like(pin[i]).pin_memory() for i in range(3)) if has_bwd else ()
    ws = None
    if has_bwd:
        ws = torch.empty(fa.bwd_workspace_size(wl.B, wl.H, wl.N, wl.d), dtype=torch.uint8, device=dev)
    h2d = sum(x.numel() * x.element_size() for x in pin)
    d2h = o_h.numel() * 2 + l_h.numel() * 4 + sum(g.numel() * 2 for g in grads_h)

    def buffers():
        ins = [torch.empty_like(x, device=dev) for x in pin[:3]] + ([torch.empty_like(pin[3], device=dev)]
                                                                   if has_bwd else [])
        outs = [torch.empty_like(ins[0]), torch.empty((wl.B, wl.H, wl.N), dtype=torch.float32, device=dev)]
        if has_bwd:
            outs += [torch.empty_like(ins[0]), torch.empty_like(ins[1]), torch.empty_like(ins[2])]
        return ins, outs

    def copy_in(ins):
        for dst, src in zip(ins, pin):
            dst.copy_(src, non_blocking=True)

    def compute(ins, outs):
        q, k, v = ins[:3]
        fa.forward(q, k, v, wl.scale, wl.causal, wl.window, out=outs[0], lse=outs[1])
        if has_bwd:
            fa.backward(q, k, v, outs[0], outs[1], ins[3], wl.scale, wl.causal, wl.window,
                        grads=tuple(outs[2:5]), workspace=ws)

    def copy_out(outs):
        for h, t in zip((o_h, l_h) + grads_h, outs):
            h.copy_(t, non_blocking=True)

    def timed(run_steps):
        torch.cuda.synchronize(dev)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        run_steps(e0)
        e1.record(stream)
        torch.cuda.synchronize(dev)
        return e0.elapsed_time(e1) / steps

    def pipelined():
        sets = [buffers(), buffers()]
        s_in, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
        in_done, comp_done, out_done = ([torch.cuda.Event() for _ in range(2)] for _ in range(3))
        used = [False, False]

        def step(i):
            b = i % 2
            ins, outs = sets[b]
            with torch.cuda.stream(s_in):
                if used[b]:
                    s_in.wait_event(comp_done[b])      # step i-2's compute has read these inputs
                copy_in(ins)
                in_done[b].record(s_in)
            stream.wait_event(in_done[b])
            if used[b]:
                stream.wait_event(out_done[b])         # step i-2's results have left these outputs
            with torch.cuda.stream(stream):
                compute(ins, outs)
            comp_done[b].record(stream)
            with torch.cuda.stream(s_out):
                s_out.wait_event(comp_done[b])
                copy_out(outs)
                out_done[b].record(s_out)
            used[b] = True
            return b

        for i in range(2):
            step(i)

        def run(e0):
            s_in.wait_event(e0)
            last = 0
            for i in range(steps):
                last = step(i)
            stream.wait_event(out_done[last])          # the last step's results are on the host

        return timed(run)

    def serial():
        ins, outs = buffers()

        def one():
            copy_in(ins)
            compute(ins, outs)
            copy_out(outs)

        for _ in range(2):
            one()

        def run(e0):
            for _ in range(steps):
                one()

        return timed(run)

    mode = "pipelined: step i+1's inputs and step i-1's results copy while step i computes"
    try:
        ms_local = pipelined()
    except Exception as exc:   # the serial form still measures the whole step
        mode = f"serial (the pipelined form raised {type(exc).__name__})"
        torch.cuda.synchronize(dev)
        ms_local = serial()
    ms = max_over_ranks([ms_local], dev)[0]
    return {"value": round(job_throughput(world, flops, ms), 3), "unit": "TFLOP/s",
            "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": round(ms, 3), "mode": mode}


# DRAM bytes per launch (dram__bytes_read.sum + dram__bytes_write.sum) from one ncu capture of
# the workload the bench line times (the causal B2 H32 N4096 d128 one, or the decode one), keyed by kernel, with the SHA-1 of the kernel's sources
# when the counters were taken (profiles/ holds the summaries).  A changed source reports null.
NCU_TRAFFIC = {
    "fa_fwd_kernel<128>": {"bytes": 249242624,
                           "sources": {"fwd_kernel.cuh": "faf4e3c455010476279ab78331d6407948b04090",
                                       "sm100.cuh": "d0155c807bbebb96a598c40bfe5826be5d752097",
                                       "grid_sched.cuh": "d69cc1d77285fb320f5966be935efafc0d37f593"}},
    "fa_bwd_kernel<128>": {"bytes": 625917696,
                           "sources": {"bwd_kernel.cuh": "4ff5578c97f3b087315277901bd12f07653933dd",
                                       "sm100.cuh": "d0155c807bbebb96a598c40bfe5826be5d752097",
                                       "grid_sched.cuh": "d69cc1d77285fb320f5966be935efafc0d37f593"}},
    # the decode workload (B8 H64 with 8 K/V heads, N_q 1, N_k 32768): both kernels of one step
    "fa_decode_kernel<128,false>+fa_decode_merge_kernel<128>": {
        "bytes": 1080936960,
        "sources": {"decode_kernel.cuh": "0b0388b3ae07210bfe25fc0f560b02d870b7b25b",
                    "decode_ops.cuh": "ce1146b0eed95a0cdd62429f8d0ff970bb9bdcf5",
                    "sm100.cuh": "d0155c807bbebb96a598c40bfe5826be5d752097"}},
}


def load_traffic(kernel: str):
    import hashlib
    entry = NCU_TRAFFIC.get(kernel)
    if not entry:
        return None
    csrc = os.path.join(ROOT, "exact_io_aware_77_b200", "csrc")
    for name, sha in entry["sources"].items():
        try:
            with open(os.path.join(csrc, name), "rb") as f:
                if hashlib.sha1(f.read()).hexdigest() != sha:
                    return None
        except OSError:
            return None
    return entry["bytes"]


# ----------------------------------------------------------------------------- decode arm
_INPUT_CACHE = {}


def decode_oracle_sample(seconds: float, max_heads: int | None = None, fp8: bool = False):
    """Time the fp64 oracle's decode forward head by head (batch entry 0) on the decode
    workload (fp8: over its E4M3 K/V cache).  Returns (flops credited, seconds, heads, cores)."""
    from oracle import attention as orc
    from synthetic import WORKLOADS, make_inputs, make_inputs_fp8kv
    wl = WORKLOADS["decode"]
    key = "decode_fp8" if fp8 else "decode"
    if key not in _INPUT_CACHE:
        _INPUT_CACHE[key] = make_inputs_fp8kv(wl) if fp8 else make_inputs(wl)
    if fp8:
        q, k8, v8, s_k, s_v = _INPUT_CACHE[key]
    else:
        q, k, v = _INPUT_CACHE[key]
    g = wl.H // wl.kv_heads
    per_head = decode_flops(1, 1, wl.q_rows, wl.N, wl.d, wl.causal, wl.window)
    t0 = time.perf_counter()
    heads = 0
    while True:
        h = heads % wl.H
        kv = slice(h // g, h // g + 1)
        if fp8:
            orc.attention_forward_decode_fp8kv(q[0:1, h:h + 1], k8[0:1, kv], v8[0:1, kv], s_k, s_v, wl.scale,
                                               wl.causal, wl.window)
        else:
            orc.attention_forward_decode(q[0:1, h:h + 1], k[0:1, kv], v[0:1, kv], wl.scale, wl.causal, wl.window)
        heads += 1
        el = time.perf_counter() - t0
        if el >= seconds or (max_heads is not None and heads >= max_heads):
            break
    return per_head * heads, el, heads, blas_threads()


def decode_workload_text(wl, fp8: bool = False) -> str:
    kv = ("K and V as E4M3 codes with per-tensor scales (max|x|/448)" if fp8 else "bf16")
    return (f"decode forward: B={wl.B} H={wl.H} (K/V heads {wl.kv_heads}) N_q={wl.q_rows} new row(s) at "
            f"the last positions of N_k={wl.N} keys, d={wl.d} {'causal' if wl.causal else 'no mask'}"
            f"{f' window {wl.window}' if wl.window else ''}, inputs N(0,1)*{wl.std:g} bf16 seeded, K/V {kv}")


def run_decode(args, fp8: bool = False):
    import torch
    import torch.distributed as dist

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        dist.init_process_group("nccl", device_id=dev, timeout=datetime.timedelta(seconds=300))

    import exact_io_aware_77_b200 as fa
    fa.load()
    from synthetic import WORKLOADS, make_inputs, make_inputs_fp8kv
    wl = WORKLOADS["decode"]
    B, H, Hkv, Nq, Nk, d = wl.B, wl.H, wl.kv_heads, wl.q_rows, wl.N, wl.d
    s_k = s_v = 1.0
    if fp8:
        q_h, k_h, v_h, s_k, s_v = make_inputs_fp8kv(wl)
    else:
        q_h, k_h, v_h = make_inputs(wl)
    q, k, v = (x.to(dev) for x in (q_h, k_h, v_h))
    o = torch.empty_like(q)
    lse = torch.empty((B, H, Nq), dtype=torch.float32, device=dev)
    need = fa.decode_workspace_size(B, H, Hkv, Nq, Nk, d, wl.causal, wl.window)
    ws = torch.empty(max(need, 16), dtype=torch.uint8, device=dev)
    launches = 2 if need else 1                  # split kernel, then the split merge
    flops = decode_flops(B, H, Nq, Nk, d, wl.causal, wl.window)
    nbytes = decode_bytes(B, H, Hkv, Nq, Nk, d, wl.causal, wl.window, kv_elem_bytes=1 if fp8 else 2)
    stream = torch.cuda.current_stream(dev)

    def run(qq, kk, vv):
        if fp8:
            fa.decode_fp8kv(qq, kk, vv, s_k, s_v, wl.scale, wl.causal, wl.window, out=o, lse=lse, workspace=ws)
        else:
            fa.decode(qq, kk, vv, wl.scale, wl.causal, wl.window, out=o, lse=lse, workspace=ws)

    def step(ev=None):
        if ev:
            ev[0].record(stream)
        run(q, k, v)
        if ev:
            ev[1].record(stream)

    for _ in range(args.warmup):
        step()
    st = fa.check_status(dev)
    if st != 0:
        raise RuntimeError(f"device status after warm-up: {fa.STATUS_NAMES.get(st, st)}")
    sampler = ClockSampler(gpu_id_for(local))
    sampler.start()
    time.sleep(0.3)
    events = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(args.steps)]
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize(dev)
    wall0 = time.time()
    for i in range(args.steps):
        step(events[i])                           # K and V (1.07 GB, or 0.54 GB as E4M3) exceed L2
    torch.cuda.synchronize(dev)
    wall1 = time.time()
    if world > 1:
        dist.barrier()
    sampler.mark(wall0, wall1)
    time.sleep(0.25)
    sampler.stop()
    st = fa.check_status(dev)
    if st != 0:
        raise RuntimeError(f"device status after timing: {fa.STATUS_NAMES.get(st, st)}")
    total = max_over_ranks([sum(e[0].elapsed_time(e[1]) for e in events)], dev)[0]
    ms = total / args.steps
    value = job_throughput(world, flops, ms)

    e2e = None
    if not args.no_e2e:
        pin = [x.pin_memory() for x in (q_h, k_h, v_h)]
        o_h = torch.empty_like(pin[0]).pin_memory()
        l_h = torch.empty((B, H, Nq), dtype=torch.float32).pin_memory()
        qe, ke, ve = (torch.empty_like(x, device=dev) for x in pin)

        def one():
            for dst, src in zip((qe, ke, ve), pin):
                dst.copy_(src, non_blocking=True)
            run(qe, ke, ve)
            o_h.copy_(o, non_blocking=True)
            l_h.copy_(lse, non_blocking=True)

        one()
        torch.cuda.synchronize(dev)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        n_e2e = max(1, min(args.e2e_steps, 3))
        e0.record(stream)
        for _ in range(n_e2e):
            one()
        e1.record(stream)
        torch.cuda.synchronize(dev)
        ms_e2e = max_over_ranks([e0.elapsed_time(e1) / n_e2e], dev)[0]
        e2e = {"value": round(job_throughput(world, flops, ms_e2e), 4), "unit": "TFLOP/s",
               "h2d_bytes_per_step": sum(x.numel() * x.element_size() for x in pin),
               "d2h_bytes_per_step": o_h.numel() * 2 + l_h.numel() * 4, "ms_per_step": round(ms_e2e, 3)}

    peaks, peak_kind = load_peaks()
    achieved = nbytes / (ms * 1e-3) / 1e9
    roofline_kernel = f"fa_decode_kernel<128,{'true' if fp8 else 'false'}>+fa_decode_merge_kernel<128>"
    roofline = {"bound": "hbm", "kernel": roofline_kernel,
                "achieved": round(achieved, 1), "peak": peaks["hbm_gbs"], "unit": "GB/s",
                "frac": round(achieved / peaks["hbm_gbs"], 4),
                "peak_source": f"{peak_kind} copy bandwidth (MEASURED_PEAKS.json)" if peak_kind == "measured"
                else "fallback 6.65 TB/s",
                "algorithmic_bytes": nbytes,
                "traffic": load_traffic(roofline_kernel)}
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        f, secs, heads, cores = decode_oracle_sample(args.cpu_seconds, fp8=fp8)
        cpu = {"value": round(f / secs / 1e12, 6), "unit": "TFLOP/s", "cores": cores, "kind": "oracle",
               "sample": f"{heads} query heads (batch entry 0) of the decode workload through the fp64 "
                         f"oracle, {secs:.1f} s, credited each head's FLOPs"}
    line = {
        "metric": "attention fwd/bwd TFLOP/s at 1 B200; % of dense BF16 tensor peak",
        "value": round(value, 3), "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(ms, 4), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": decode_workload_text(wl, fp8), "global_batch": B * world, "seq_len": Nk,
                   "parallelism": f"replicas{world}",
                   "l2": "not flushed: the K and V read each step (1.07 GB bf16, 0.54 GB E4M3) exceed the 126 MB L2"},
        "hbm_gbs": round(achieved, 1),
        "roofline": roofline,
        "cpu_baseline": cpu,
        "e2e": e2e,
        "gpu_launches": args.steps * launches,
        "clocks": sampler.summary(),
    }
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(line), flush=True)


# ----------------------------------------------------------------------------- FP8 forward arm
FP8_OVER_BF16 = 2.0   # nominal dense E4M3 / bf16 tensor throughput of a B200 (4.5 / 2.25 PFLOP/s)


def fp8_oracle_sample(seconds: float, max_heads: int | None = None):
    """Time the oracle's FP8 forward head by head on the causal workload's E4M3 inputs.
    Returns (flops credited, seconds, heads, cores)."""
    from oracle import attention as orc
    from synthetic import WORKLOADS, make_inputs_fp8
    wl = WORKLOADS["causal"]
    if "fp8" not in _INPUT_CACHE:
        _INPUT_CACHE["fp8"] = make_inputs_fp8(wl.with_(B=1, H=4))
    q8, k8, vt8, s_q, s_k, s_v = _INPUT_CACHE["fp8"]
    per_head = fwd_flops(1, 1, wl.N, wl.d, wl.causal, wl.window)
    t0 = time.perf_counter()
    heads = 0
    while True:
        h = heads % 4
        orc.attention_forward_fp8(q8[:, h:h + 1], k8[:, h:h + 1], vt8[:, h:h + 1], s_q, s_k, s_v, wl.scale,
                                  wl.causal, wl.window)
        heads += 1
        el = time.perf_counter() - t0
        if el >= seconds or (max_heads is not None and heads >= max_heads):
            break
    return per_head * heads, el, heads, blas_threads()


def run_fp8(args):
    import torch
    import torch.distributed as dist

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        dist.init_process_group("nccl", device_id=dev, timeout=datetime.timedelta(seconds=300))
    import exact_io_aware_77_b200 as fa
    fa.load()
    from synthetic import WORKLOADS, make_inputs_fp8
    wl = WORKLOADS["causal"]
    B, H, N, d = wl.B, wl.H, wl.N, wl.d
    q8_h, k8_h, vt8_h, s_q, s_k, s_v = make_inputs_fp8(wl)
    q8, k8, vt8 = (x.to(dev) for x in (q8_h, k8_h, vt8_h))
    o = torch.empty((B, H, N, d), dtype=torch.bfloat16, device=dev)
    lse = torch.empty((B, H, N), dtype=torch.float32, device=dev)
    flush = torch.empty(FLUSH_BYTES, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)
    flops = fwd_flops(B, H, N, d, wl.causal, wl.window)

    def step(ev=None):
        if ev:
            ev[0].record(stream)
        fa.forward_fp8(q8, k8, vt8, s_q, s_k, s_v, wl.scale, wl.causal, wl.window, out=o, lse=lse)
        if ev:
            ev[1].record(stream)

    for _ in range(args.warmup):
        flush.zero_()
        step()
    st = fa.check_status(dev)
    if st != 0:
        raise RuntimeError(f"device status after warm-up: {fa.STATUS_NAMES.get(st, st)}")
    sampler = ClockSampler(gpu_id_for(local))
    sampler.start()
    time.sleep(0.3)
    events = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(args.steps)]
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize(dev)
    wall0 = time.time()
    for i in range(args.steps):
        flush.zero_()
        step(events[i])
    torch.cuda.synchronize(dev)
    wall1 = time.time()
    if world > 1:
        dist.barrier()
    sampler.mark(wall0, wall1)
    time.sleep(0.25)
    sampler.stop()
    st = fa.check_status(dev)
    if st != 0:
        raise RuntimeError(f"device status after timing: {fa.STATUS_NAMES.get(st, st)}")
    total = max_over_ranks([sum(e[0].elapsed_time(e[1]) for e in events)], dev)[0]
    ms = total / args.steps
    value = job_throughput(world, flops, ms)
    e2e = None
    if not args.no_e2e:
        pin = [x.pin_memory() for x in (q8_h, k8_h, vt8_h)]
        o_h = torch.empty((B, H, N, d), dtype=torch.bfloat16).pin_memory()
        l_h = torch.empty((B, H, N), dtype=torch.float32).pin_memory()
        dq, dk, dvt = (torch.empty_like(x, device=dev) for x in pin)

        def one():
            for dst, src in zip((dq, dk, dvt), pin):
                dst.copy_(src, non_blocking=True)
            fa.forward_fp8(dq, dk, dvt, s_q, s_k, s_v, wl.scale, wl.causal, wl.window, out=o, lse=lse)
            o_h.copy_(o, non_blocking=True)
            l_h.copy_(lse, non_blocking=True)

        one()
        torch.cuda.synchronize(dev)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        n_e2e = max(1, args.e2e_steps)
        e0.record(stream)
        for _ in range(n_e2e):
            one()
        e1.record(stream)
        torch.cuda.synchronize(dev)
        ms_e2e = max_over_ranks([e0.elapsed_time(e1) / n_e2e], dev)[0]
        e2e = {"value": round(job_throughput(world, flops, ms_e2e), 3), "unit": "TFLOP/s",
               "h2d_bytes_per_step": sum(x.numel() for x in pin),
               "d2h_bytes_per_step": o_h.numel() * 2 + l_h.numel() * 4, "ms_per_step": round(ms_e2e, 3)}
    peaks, peak_kind = load_peaks()
    peak = peaks["bf16_tflops"] * FP8_OVER_BF16
    roofline = {"bound": "tensor", "kernel": "fa_fwd_fp8_kernel", "achieved": round(value / world, 1),
                "peak": round(peak, 1), "unit": "TFLOP/s", "frac": round(value / world / peak, 4),
                "peak_source": f"{peak_kind} burst bf16 (MEASURED_PEAKS.json) x {FP8_OVER_BF16:g}, the nominal "
                               f"E4M3/bf16 ratio", "traffic": None}
    clocks = sampler.summary()
    clock_norm = regime_fields(roofline, clocks, total, ms, peaks, FP8_OVER_BF16)
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        f, secs, heads, cores = fp8_oracle_sample(args.cpu_seconds)
        cpu = {"value": round(f / secs / 1e12, 6), "unit": "TFLOP/s", "cores": cores, "kind": "oracle",
               "sample": f"{heads} heads of the causal shape's E4M3 inputs through the fp64 oracle, {secs:.1f} s"}
    line = {
        "metric": "attention fwd/bwd TFLOP/s at 1 B200; % of dense BF16 tensor peak",
        "value": round(value, 2), "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(ms, 4), "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "e4m3", "data": "synthetic",
        "config": {"workload": f"FP8 forward: B={B} H={H} N={N} d={d} causal, E4M3 Q, K, V^T with per-tensor "
                               f"scales from N(0,1)*{wl.std:g} inputs",
                   "global_batch": B * world, "seq_len": N, "parallelism": f"replicas{world}",
                   "l2": "flushed (256 MB write) between timed steps, outside the events"},
        "roofline": roofline, "cpu_baseline": cpu, "e2e": e2e, "gpu_launches": args.steps,
        "clocks": clocks, "clock_normalised": clock_norm,
    }
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(line), flush=True)


# ----------------------------------------------------------------------------- forward-only arm
def fwd_hbm_bytes(wl) -> int:
    """Algorithmic bytes of one forward: read Q, K, V once, write O (bf16) and L (fp32)."""
    q_el = wl.B * wl.H * wl.q_rows * wl.d
    kv_el = wl.B * wl.kv_heads * wl.N * wl.d
    return 2 * (2 * q_el + 2 * kv_el) + 4 * wl.B * wl.H * wl.q_rows


def run_forward_only(args):
    """The forward alone (O and the logsumexp) on the tiny or the GPT-2-like workload.

    tiny (B1 H2 N128 d64) is one CTA's work: launch latency and HBM bound, so its roofline is
    the algorithmic bytes over the kernel time against the measured HBM copy bandwidth.  gpt2
    (B4 H16 N2048 d64) is a dense contraction: TFLOP/s against the measured bf16 peak."""
    import torch
    import torch.distributed as dist

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        dist.init_process_group("nccl", device_id=dev, timeout=datetime.timedelta(seconds=300))
    import exact_io_aware_77_b200 as fa
    fa.load()
    from synthetic import WORKLOADS, make_inputs
    wl = WORKLOADS[WORKLOAD]
    B, H, N, d = wl.B, wl.H, wl.N, wl.d
    q_h, k_h, v_h = make_inputs(wl)
    q, k, v = (x.to(dev) for x in (q_h, k_h, v_h))
    o = torch.empty_like(q)
    lse = torch.empty((B, H, N), dtype=torch.float32, device=dev)
    flush = torch.empty(FLUSH_BYTES, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)
    flops = fwd_flops(B, H, N, d, wl.causal, wl.window)
    nbytes = fwd_hbm_bytes(wl)
    kname = kernel_names(d)[0]

    def step(ev=None):
        if ev:
            ev[0].record(stream)
        fa.forward(q, k, v, wl.scale, wl.causal, wl.window, out=o, lse=lse)
        if ev:
            ev[1].record(stream)

    for _ in range(args.warmup):
        flush.zero_()
        step()
    st = fa.check_status(dev)
    if st != 0:
        raise RuntimeError(f"device status after warm-up: {fa.STATUS_NAMES.get(st, st)}")
    sampler = ClockSampler(gpu_id_for(local))
    sampler.start()
    time.sleep(0.3)
    events = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(args.steps)]
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize(dev)
    wall0 = time.time()
    for i in range(args.steps):
        flush.zero_()
        step(events[i])
    torch.cuda.synchronize(dev)
    wall1 = time.time()
    if world > 1:
        dist.barrier()
    sampler.mark(wall0, wall1)
    time.sleep(0.25)
    sampler.stop()
    st = fa.check_status(dev)
    if st != 0:
        raise RuntimeError(f"device status after timing: {fa.STATUS_NAMES.get(st, st)}")
    per_step = [e[0].elapsed_time(e[1]) for e in events]
    total = max_over_ranks([sum(per_step)], dev)[0]
    ms = total / args.steps
    value = job_throughput(world, flops, ms)

    e2e = None
    if not args.no_e2e:
        # through the public API with host buffers: pinned Q, K, V in, O and L out, every step
        pin = [x.pin_memory() for x in (q_h, k_h, v_h)]
        o_h = torch.empty_like(pin[0]).pin_memory()
        l_h = torch.empty((B, H, N), dtype=torch.float32).pin_memory()
        qd, kd, vd = (torch.empty_like(x, device=dev) for x in pin)

        def one():
            for dst, src in zip((qd, kd, vd), pin):
                dst.copy_(src, non_blocking=True)
            fa.forward(qd, kd, vd, wl.scale, wl.causal, wl.window, out=o, lse=lse)
            o_h.copy_(o, non_blocking=True)
            l_h.copy_(lse, non_blocking=True)

        for _ in range(3):
            one()
        torch.cuda.synchronize(dev)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        n_e2e = max(1, args.e2e_steps)
        e0.record(stream)
        for _ in range(n_e2e):
            one()
        e1.record(stream)
        torch.cuda.synchronize(dev)
        ms_e2e = max_over_ranks([e0.elapsed_time(e1) / n_e2e], dev)[0]
        e2e = {"value": round(job_throughput(world, flops, ms_e2e), 4), "unit": "TFLOP/s",
               "h2d_bytes_per_step": sum(x.numel() * x.element_size() for x in pin),
               "d2h_bytes_per_step": o_h.numel() * 2 + l_h.numel() * 4, "ms_per_step": round(ms_e2e, 4),
               "mode": "serial: copy in, forward, copy out on one stream"}

    peaks, peak_kind = load_peaks()
    gbs = nbytes / (ms * 1e-3) / 1e9
    tflops = flops / (ms * 1e-3) / 1e12
    if WORKLOAD == "tiny":
        roofline = {"bound": "hbm", "kernel": kname, "achieved": round(gbs, 1), "peak": peaks["hbm_gbs"],
                    "unit": "GB/s", "frac": round(gbs / peaks["hbm_gbs"], 4),
                    "peak_source": f"{peak_kind} HBM copy (MEASURED_PEAKS.json)", "traffic": None,
                    "bytes_per_launch": nbytes}
    else:
        roofline = {"bound": "tensor", "kernel": kname, "achieved": round(tflops, 1),
                    "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
                    "frac": round(tflops / peaks["bf16_tflops"], 4),
                    "peak_source": f"{peak_kind} burst bf16 (MEASURED_PEAKS.json)", "traffic": None}
    clocks = sampler.summary()
    clock_norm = regime_fields(roofline, clocks, total, ms, peaks) if roofline["bound"] == "tensor" else None
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        f, secs, blocks, cores = oracle_sample(args.cpu_seconds, rows_per_block=min(512, N), with_bwd=False)
        cpu = {"value": round(f / secs / 1e12, 6), "unit": "TFLOP/s", "cores": cores, "kind": "oracle",
               "sample": f"{blocks} blocks of {min(512, N)} query rows of head 0 of the {wl.name} workload "
                         f"(B{B} H{H} N{N} d{d}) through the fp64 oracle (fwd), {secs:.1f} s, credited "
                         f"rows/N of a head's FLOPs"}
    line = {
        "metric": "attention fwd/bwd TFLOP/s at 1 B200; % of dense BF16 tensor peak",
        "value": round(value, 3), "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(ms, 5), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": workload_text(wl, False), "global_batch": B * world, "seq_len": N,
                   "parallelism": f"replicas{world}",
                   "l2": "flushed (256 MB write) between timed steps, outside the events"},
        "fwd_us": round(ms * 1e3, 2), "fwd_gbs": round(gbs, 1),
        "pct_of_measured_peak": round(100 * tflops / peaks["bf16_tflops"], 2),
        "pct_of_spec_peak_2250": round(100 * tflops / 2250.0, 2),
        "pct_of_measured_hbm": round(100 * gbs / peaks["hbm_gbs"], 2),
        "roofline": roofline, "cpu_baseline": cpu, "e2e": e2e, "gpu_launches": args.steps,
        "kernel_ms": {kname: round(ms, 5)}, "clocks": clocks, "clock_normalised": clock_norm,
    }
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(line), flush=True)


# ----------------------------------------------------------------------------- reference arm
def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    from synthetic import WORKLOADS
    wl = WORKLOADS[WORKLOAD]
    if WORKLOAD == "decode":
        return run_decode_reference(args, wl, fp8=args.workload == "decode_fp8")
    if args.workload == "fp8":
        return run_fp8_reference(args, wl)
    import exact_io_aware_77_b200 as fa_pkg   # only to learn whether the path has a backward
    with_bwd = hasattr(fa_pkg, "backward") and args.workload not in FORWARD_ONLY
    times, flops = [], []
    for i in range(args.warmup + args.steps):
        f, s, _, cores = oracle_sample(0.0, rows_per_block=min(128, wl.N), with_bwd=with_bwd, max_blocks=1)
        if i >= args.warmup:
            times.append(s)
            flops.append(f)
    secs = sum(times)
    value = sum(flops) / secs / 1e12
    sample = (f"each step: {min(128, wl.N)} query rows of head 0 of the {wl.name} workload (B{wl.B} H{wl.H} N{wl.N} "
              f"d{wl.d}) through the fp64 oracle ({'fwd+bwd' if with_bwd else 'fwd'}), credited rows/N "
              f"of a head's FLOPs")
    line = {
        "metric": "attention fwd/bwd TFLOP/s at 1 B200; % of dense BF16 tensor peak",
        "value": round(value, 6), "unit": "TFLOP/s", "n_gpus": int(os.environ.get("WORLD_SIZE", "1")),
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(1e3 * secs / args.steps, 3),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "impl": "reference",
        "config": {"workload": workload_text(wl, with_bwd) + " (row-block sample)",
                   "global_batch": wl.B, "seq_len": wl.N, "parallelism": "cpu"},
        "cpu_baseline": {"value": round(value, 6), "unit": "TFLOP/s", "cores": cores, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": round(value, 6), "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def run_decode_reference(args, wl, fp8: bool = False):
    times, flops = [], []
    cores = blas_threads()
    for i in range(args.warmup + args.steps):
        f, secs, _, cores = decode_oracle_sample(0.0, max_heads=1, fp8=fp8)
        if i >= args.warmup:
            times.append(secs)
            flops.append(f)
    secs = sum(times)
    value = sum(flops) / secs / 1e12
    line = {
        "metric": "attention fwd/bwd TFLOP/s at 1 B200; % of dense BF16 tensor peak",
        "value": round(value, 6), "unit": "TFLOP/s", "n_gpus": int(os.environ.get("WORLD_SIZE", "1")),
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(1e3 * secs / args.steps, 3),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "impl": "reference",
        "config": {"workload": decode_workload_text(wl, fp8) + " (one-head sample per step)",
                   "global_batch": wl.B, "seq_len": wl.N, "parallelism": "cpu"},
        "cpu_baseline": {"value": round(value, 6), "unit": "TFLOP/s", "cores": cores, "kind": "oracle",
                         "sample": "each step: query head 0 of batch entry 0 of the decode workload through "
                                   "the fp64 oracle, credited that head's FLOPs"},
        "e2e": {"value": round(value, 6), "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def run_fp8_reference(args, wl):
    times, flops = [], []
    cores = blas_threads()
    for i in range(args.warmup + args.steps):
        f, secs, _, cores = fp8_oracle_sample(0.0, max_heads=1)
        if i >= args.warmup:
            times.append(secs)
            flops.append(f)
    secs = sum(times)
    value = sum(flops) / secs / 1e12
    print(json.dumps({
        "metric": "attention fwd/bwd TFLOP/s at 1 B200; % of dense BF16 tensor peak",
        "value": round(value, 6), "unit": "TFLOP/s", "n_gpus": int(os.environ.get("WORLD_SIZE", "1")),
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(1e3 * secs / args.steps, 3),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "impl": "reference",
        "config": {"workload": f"FP8 forward of the causal shape (B={wl.B} H={wl.H} N={wl.N} d={wl.d}), one head "
                               f"per step", "global_batch": wl.B, "seq_len": wl.N, "parallelism": "cpu"},
        "cpu_baseline": {"value": round(value, 6), "unit": "TFLOP/s", "cores": cores, "kind": "oracle",
                         "sample": "each step: one head of the E4M3 inputs through the fp64 oracle"},
        "e2e": {"value": round(value, 6), "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }), flush=True)


def workload_text(wl, with_bwd: bool) -> str:
    if wl.window:
        band = (f"{'causal' if wl.causal else 'two-sided'} window {wl.window}, FLOPs over the "
                f"{band_pairs(wl.N, wl.causal, wl.window)} kept pairs per head")
        kind = "long-context"
    else:
        kinds = {"tiny": "tiny", "gpt2": "GPT-2-like", "d256": "head dimension 256"}
        band, kind = ("causal" if wl.causal else "no mask"), kinds.get(wl.name, "causal LLM shape")
    heads = f"H={wl.H}" + (f" (K/V heads {wl.kv_heads})" if wl.kv_heads != wl.H else "")
    return (f"{kind} {'forward+backward' if with_bwd else 'forward'}: B={wl.B} {heads} N={wl.N} "
            f"d={wl.d} {band}, inputs N(0,1)*{wl.std:g} bf16 seeded")


def main():
    global WORKLOAD, GRAD_WORKLOAD
    args = parse_args()
    WORKLOAD, GRAD_WORKLOAD = BENCH_WORKLOADS[args.workload]
    if args.impl == "reference":
        run_reference(args)
    elif WORKLOAD == "decode":
        run_decode(args, fp8=args.workload == "decode_fp8")
    elif args.workload == "fp8":
        run_fp8(args)
    elif args.workload in FORWARD_ONLY:
        run_forward_only(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
