"""Benchmark of the KDA hot path on B200: prefill tokens/s and decode state GB/s.

Workloads (H=96, K=V=128, synthetic seeded inputs from ``workloads.py``):

* prefill -- B=1, T=4096, bf16 q/k/v, fp32 decay logits (z ~ N(0,2)), fp32 beta,
  zero initial state, fp32 final state. One step = one ``kda_prefill_logits``
  call: the chunked prefill evaluates the bounded gate from the logits while it
  reads them (-> o, final_state). ``value`` is tokens/s.
* decode -- B=64 kept 128x128 fp32 states (402.7 MB), bf16 q/k/v, z ~ N(0,1).
  One step = one in-place ``kda_decode_step_logits`` call (gate inside the
  step). Reported in the ``decode`` object as state GB/s (2*4*K*V*B*H bytes per
  step) and steps/s.
* varlen, long_kv -- the 16 packed sequences of 512..8192 tokens (H=96, own
  initial states) and the long K != V batch (B=4, T=16384, H=32, V=256, initial
  states), each one ``kda_prefill_logits`` call per step; the ``varlen`` and
  ``long_kv`` objects carry tokens/s, the HBM roofline of their algorithmic
  bytes (states included), e2e and the oracle on a sample of heads.
* softplus, backward -- the prefill workload through Kimi Linear's unbounded
  gate, and the gradients from the logits (their own objects).

Timing: W untimed warm-up steps, then K steps bracketed by a barrier and a
device synchronise, CUDA events on the stream the kernels are launched on,
max over ranks. Every input set is larger than the 126 MB L2, so no flush is
inserted between steps. ``e2e`` repeats the measurement through the public
API with pinned host buffers: each step copies its inputs host->device and
reads its results device->host inside the timed region.

``--impl reference`` times the fp64 CPU oracle on a bounded sample of the same
workload and prints the same line with ``"impl": "reference"``.

Multi-GPU (``torchrun``): every rank runs its own copy of the workload (the
(sequence, head) units are independent, so there is no collective on the data
path); ``value`` = units of all ranks / max-over-ranks time, ``scaling`` weak.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import workloads as W  # noqa: E402

METRIC = "KDA prefill tokens/s & decode state GB/s (H96,K=V=128); % of roofline"
PEAKS_FALLBACK = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


# ------------------------------------------------------------------------------------------------
# Algorithmic work per launch (the units the roofline fractions are computed from)
# ------------------------------------------------------------------------------------------------

def prefill_bytes(B, T, H, K, V, n_states_in, n_states_out, es=2):
    """Minimum HBM bytes of one prefill launch: read q, k (K each), v (V) in the input dtype,
    the decay input (alpha, g or the logits z; K fp32) and beta (fp32) per token-head, write o (V); read/write the
    fp32 states."""
    per_tok_head = 2 * K * es + V * es + 4 * K + 4 + V * es
    return B * T * H * per_tok_head + (n_states_in + n_states_out) * H * K * V * 4


def prefill_flops(B, T, H, K, V, C=64):
    """Dense chunk-form FLOPs at a fixed C = 64 per token-head: 6CK + 4CV + 6KV + C^2/3."""
    return B * T * H * (6 * C * K + 4 * C * V + 6 * K * V + C * C / 3.0)


def decode_bytes(B, H, K, V, es=2):
    """Per step: state read + write (8KV), q, k, v, o in the input dtype, the decay input (K fp32), beta fp32."""
    return B * H * (8 * K * V + (2 * K + 2 * V) * es + 4 * K + 4)


def decode_state_bytes(B, H, K, V):
    return B * H * 2 * 4 * K * V


def gate_bytes(n_elems, es_in=4, es_out=4):
    return n_elems * (es_in + es_out)


# DRAM bytes (read + write) per launch of each step, from one ncu capture of its kernels (dram__bytes_read.sum +
# dram__bytes_write.sum of every kernel the step launches). They hold only for the kernel sources they were
# taken on, so a sha256 of those sources (comments and blank space left out, see source_digest) is kept
# beside them and a mismatch at run time reports null.
MEASURED_TRAFFIC = {
    # chunk_intra_kernel<2> 404.5 + 357.0 MB; chunk_state_kernel 506.6 + 83.7 MB
    "prefill": {"bytes": 1351800000, "files": ['chunk_split.cu', 'chunk_common.cuh', 'gate_math.cuh', 'common.cuh', 'kda_internal.h'],
              "sha256": "93945c09b373a8da39759aa9cdf609f006a5ce122ed041363d97f5658609f158"},
    # decode_bulk_kernel 410.6 + 342.6 MB
    "decode": {"bytes": 753100000, "files": ['decode.cu', 'gate_math.cuh', 'common.cuh', 'kda_internal.h'],
               "sha256": "734d2492590f985a4aad384a7233e845473b4b9a545a6749e1a2ccec3f938b83"},
    # chunk_intra_kernel<3> 405.0 + 357.7 MB; chunk_state_kernel 506.6 + 83.8 MB (the unbounded gate's prefill)
    "softplus": {"bytes": 1353000000, "files": ['chunk_split.cu', 'chunk_common.cuh', 'gate_math.cuh', 'common.cuh', 'kda_internal.h'],
               "sha256": "93945c09b373a8da39759aa9cdf609f006a5ce122ed041363d97f5658609f158"},
    # chunk_intra_kernel<2> 7,937.8 + 7,282.0 MB; chunk_state_kernel 9,227.2 + 1,884.4 MB (16 packed sequences)
    "varlen": {"bytes": 26331400000, "files": ['chunk_split.cu', 'chunk_common.cuh', 'gate_math.cuh', 'common.cuh', 'kda_internal.h'],
             "sha256": "93945c09b373a8da39759aa9cdf609f006a5ce122ed041363d97f5658609f158"},
    # chunk_intra_kernel<2> 2,335.6 + 2,120.8 MB; chunk_state_kernel 3,254.9 + 1,059.7 MB (4 x 16384 x 32, V = 256)
    "long_kv": {"bytes": 8771000000, "files": ['chunk_split.cu', 'chunk_common.cuh', 'gate_math.cuh', 'common.cuh', 'kda_internal.h'],
              "sha256": "93945c09b373a8da39759aa9cdf609f006a5ce122ed041363d97f5658609f158"},
    # bounded_decay_kernel 201.4 + 153.4 MB; scan_backward_kernel 19,322.0 + 27,321.0 MB;
    # bounded_decay_backward_kernel 402.7 + 163.3 MB (one backward step from the logits, exact token adjoint)
    # the chunked backward step (gate, forward kernels P and S, prep, pair, inverse, 16 cuBLAS products, dstate,
    # mask_dgc, dt, da, assemble, gate gradient): 14,730.3 MB read + 6,846.4 MB written
    "backward_chunked": {"bytes": 21576700000,
                         "files": ['backward_chunked.cu', 'chunk_split.cu', 'chunk_common.cuh', 'gate.cu', 'gate_math.cuh',
                                   'common.cuh', 'kda_internal.h'],
                         "sha256": "d699bdefb43595a5b8f949e9df41d52f4a85e740593fda122b6cdf073a328ee6"},
    "backward": {"bytes": 47563800000, "files": ['backward.cu', 'gate.cu', 'gate_math.cuh', 'common.cuh', 'kda_internal.h'],
                 "sha256": "7a7ad8f22444f39b7918104ba5cb3bc16be94cd42d9be45876612e744271116e"},
}


def source_digest(files) -> str:
    """sha256 of the kernel sources with their comments and blank space removed, so that a change of comments
    alone keeps a measurement taken on the same code."""
    import hashlib
    import re
    h = hashlib.sha256()
    for f in files:
        with open(os.path.join(ROOT, "gated_delta_rule_bounded_b200", "csrc", f), "rb") as fh:
            text = fh.read().decode()
        text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
        text = re.sub(r"//[^\n]*", "", text)
        lines = (" ".join(line.split()) for line in text.splitlines())
        h.update("\n".join(line for line in lines if line).encode())
    return h.hexdigest()


def measured_traffic(step: str):
    m = MEASURED_TRAFFIC.get(step)
    if m is None:
        return None
    try:
        digest = source_digest(m["files"])
    except OSError:
        return None
    return m["bytes"] if digest == m["sha256"] else None


# ------------------------------------------------------------------------------------------------
# Environment helpers
# ------------------------------------------------------------------------------------------------

def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return p, "measured"
    except (OSError, ValueError):
        return dict(PEAKS_FALLBACK), "fallback"


class ClockSampler:
    """Samples nvidia-smi clocks and throttle reasons while the timed region runs.

    A reader thread collects the CSV lines. Entering waits for the first sample
    (so the sampler is running before the timed region starts); leaving waits
    for one more sample after it ends, so even a short region is covered."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index: int):
        self.idx = device_index
        self.proc = None
        self.lines = []
        self.thread = None

    def _reader(self):
        for line in self.proc.stdout:
            self.lines.append(line)

    def _wait_lines(self, n, timeout):
        t_end = time.time() + timeout
        while len(self.lines) < n and time.time() < t_end:
            time.sleep(0.01)

    def __enter__(self):
        import threading
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.idx}", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "50"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
            return self
        self.thread = threading.Thread(target=self._reader, daemon=True)
        self.thread.start()
        self._wait_lines(1, 3.0)
        self.first = len(self.lines)
        return self

    def __exit__(self, *exc):
        if self.proc is None:
            return False
        self._wait_lines(len(self.lines) + 1, 1.0)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        if self.thread is not None:
            self.thread.join(timeout=2)
        return False

    def summary(self):
        if not self.lines:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"], "samples": 0}
        sm, smax, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        # samples from just before the timed region to just after it
        for line in self.lines[max(0, self.first - 1):]:
            parts = [x.strip() for x in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                smax = float(parts[2])
            except ValueError:
                continue
            for name, val in zip(names, parts[5:9]):
                if val.lower() == "active":
                    reasons.add(name)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": smax,
                "reasons": sorted(reasons), "samples": len(sm)}


def dist_setup(n_gpus):
    """One process per GPU under torchrun; returns (rank, world, local_rank)."""
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        backend = "nccl" if torch.cuda.is_available() else "gloo"
        if backend == "nccl":
            torch.cuda.set_device(local)
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
    if n_gpus != world and world > 1 and rank == 0:
        print(f"warning: --gpus {n_gpus} but WORLD_SIZE={world}", file=sys.stderr)
    return rank, world, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(x: float, world: int) -> float:
    """Max of a per-rank scalar over all ranks (identity for one rank)."""
    if world == 1:
        return float(x)
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([float(x)], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def weak_scaling_value(units_per_rank: float, local_ms: float, world: int) -> tuple:
    """Whole-job throughput of replicated work: every rank processes `units_per_rank` units in
    `local_ms`; the job takes the slowest rank's time. Returns (units/s, max ms)."""
    slowest = max_over_ranks(local_ms, world)
    return units_per_rank * world / (slowest / 1e3), slowest


def sum_over_ranks(x: float, world: int) -> float:
    if world == 1:
        return float(x)
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([float(x)], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.SUM)
    return float(t.item())


# ------------------------------------------------------------------------------------------------
# GPU arm
# ------------------------------------------------------------------------------------------------

def timed_loop(step_fns, steps, warmup, world, stream, sampler=None):
    """Runs each step fn once per iteration. Returns (total ms over `steps`, per-fn avg ms).

    Each step fn is bracketed by its own events (recorded on `stream`, the stream the
    kernels are launched on), so the per-kernel averages come from the same timed run."""
    for _ in range(warmup):
        for fn in step_fns:
            fn()
    torch.cuda.synchronize()
    barrier(world)
    torch.cuda.synchronize()
    n = len(step_fns)
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(n + 1)] for _ in range(steps)]
    ctx = sampler if sampler is not None else _Null()
    with ctx:
        # About 1 ms of queued device work ahead of the first event, so that the first timed step does not
        # include the host's latency to issue it (the GPU would otherwise sit idle after the event).
        with torch.cuda.stream(stream):
            torch.cuda._sleep(2_000_000)
        start = torch.cuda.Event(enable_timing=True)
        end = torch.cuda.Event(enable_timing=True)
        start.record(stream)
        for s in range(steps):
            ev[s][0].record(stream)
            for i, fn in enumerate(step_fns):
                fn()
                ev[s][i + 1].record(stream)
        end.record(stream)
        torch.cuda.synchronize()
    total = start.elapsed_time(end)
    per_fn = [sum(ev[s][i].elapsed_time(ev[s][i + 1]) for s in range(steps)) / steps for i in range(n)]
    barrier(world)
    return total, per_fn


def pipelined_e2e(host_in, dev_in, host_out, dev_out, run_fn, steps, warmup, world):
    """End-to-end steps through the public API, as a serving loop runs them: each step copies its inputs from
    pinned host memory to the device, calls the library and copies its results back to pinned host memory,
    with the three stages of consecutive steps overlapped on three streams (step i's inputs come in while step
    i-1 computes and step i-2's results go out). Inputs and outputs are double-buffered: dev_in and dev_out are
    two dicts each; run_fn(inputs, outputs) launches on the current stream (the computes run in order on one
    stream). host_in is a dict of pinned tensors, or a list of such dicts taken in turn. Returns the total ms
    over `steps` (first input copy to last result copy, CUDA events)."""
    s_in, s_cmp, s_out = torch.cuda.Stream(), torch.cuda.Stream(), torch.cuda.Stream()
    n = warmup + steps
    ev = {k: [torch.cuda.Event() for _ in range(n)] for k in ("in", "cmp", "out")}
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    barrier(world)
    torch.cuda.synchronize()
    for i in range(n):
        if i == warmup:
            torch.cuda.synchronize()
            start.record(s_in)
        b = i % 2
        with torch.cuda.stream(s_in):
            if i >= 2:
                s_in.wait_event(ev["cmp"][i - 2])  # step i-2 has read these input buffers
            src = host_in[i % len(host_in)] if isinstance(host_in, list) else host_in
            for name, x in src.items():
                dev_in[b][name].copy_(x, non_blocking=True)
            ev["in"][i].record(s_in)
        with torch.cuda.stream(s_cmp):
            s_cmp.wait_event(ev["in"][i])
            if i >= 2:
                s_cmp.wait_event(ev["out"][i - 2])  # step i-2's results have left these output buffers
            run_fn(dev_in[b], dev_out[b])
            ev["cmp"][i].record(s_cmp)
        with torch.cuda.stream(s_out):
            s_out.wait_event(ev["cmp"][i])
            for name, x in host_out.items():
                x.copy_(dev_out[b][name], non_blocking=True)
            ev["out"][i].record(s_out)
    s_out.wait_stream(s_in)
    s_out.wait_stream(s_cmp)
    end.record(s_out)
    torch.cuda.synchronize()
    barrier(world)
    return start.elapsed_time(end)


class _Null:
    def __enter__(self):
        return self

    def __exit__(self, *a):
        return False


def prefill_leg(args, kda, dev, stream, rank, world, hbm, bf16_peak, peak_src):
    w = W.PREFILL
    d = W.make_scan_inputs(w)
    B, T, H, K, V = w.B, w.T, w.H, w.K, w.V
    g = {n: (x.to(dev) if isinstance(x, torch.Tensor) else x) for n, x in d.items()}
    o = torch.empty(B, T, H, V, device=dev, dtype=torch.bfloat16)
    sf = torch.empty(B, H, K, V, device=dev, dtype=torch.float32)
    ws_bytes = kda.prefill_workspace_bytes(B, T, H, K, V, 0, torch.bfloat16)
    ws = torch.empty(max(ws_bytes, 1), device=dev, dtype=torch.uint8)

    # One call: the scan kernels read the decay logits z and evaluate the bounded gate themselves.
    def prefill_fn():
        kda.prefill_logits(g["q"], g["k"], g["v"], g["z"], g["A_log"], w.g_min, g["beta"], None, out=o,
                           final_state=sf, workspace=ws)

    sampler = ClockSampler(dev.index if dev.index is not None else 0) if rank == 0 else None
    total_ms, (pre_ms,) = timed_loop([prefill_fn], args.steps, args.warmup, world, stream, sampler)
    value, total_ms = weak_scaling_value(B * T * args.steps, total_ms, world)
    ms_per_step = total_ms / args.steps
    tokens = B * T * world
    pb = prefill_bytes(B, T, H, K, V, 0, 1)
    achieved = pb / (pre_ms / 1e3) / 1e9
    flops = prefill_flops(B, T, H, K, V)
    tflops = flops / (pre_ms / 1e3) / 1e12
    res = {
        "value": value, "ms_per_step": ms_per_step, "workload": w, "clocks": sampler.summary() if sampler else None,
        "kernels_ms": {"prefill_logits": pre_ms},
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": hbm, "unit": "GB/s",
                     "frac": achieved / hbm, "traffic": measured_traffic("prefill"), "kernel": "kda_prefill_logits",
                     "bytes_per_launch": pb, "ms_per_launch": pre_ms, "peak_source": f"{peak_src} hbm_gbs",
                     "tensor": {"tflops_at_C64_formula": tflops, "peak": bf16_peak,
                                "frac": tflops / bf16_peak, "flops_per_launch": flops}},
        "gpu_launches": 2 * args.steps,  # the operand kernel and the recurrence kernel per call
    }
    if args.no_e2e:
        return res
    # e2e: pinned host inputs -> device, prefill from logits, o and final state -> pinned host, consecutive
    # steps overlapped (the inputs of one step copy in while the previous step computes)
    host = {n: d[n].pin_memory() for n in ("q", "k", "v", "z", "A_log", "beta")}
    host_out = {"o": torch.empty(B, T, H, V, dtype=torch.bfloat16).pin_memory(),
                "sf": torch.empty(B, H, K, V, dtype=torch.float32).pin_memory()}
    dev_in = [{n: torch.empty_like(x, device=dev) for n, x in host.items()} for _ in range(2)]
    dev_out = [{"o": o, "sf": sf}, {"o": torch.empty_like(o), "sf": torch.empty_like(sf)}]
    h2d = sum(x.numel() * x.element_size() for x in host.values())
    d2h = sum(x.numel() * x.element_size() for x in host_out.values())

    def run(i, out):
        kda.prefill_logits(i["q"], i["k"], i["v"], i["z"], i["A_log"], w.g_min, i["beta"], None, out=out["o"],
                           final_state=out["sf"], workspace=ws)  # computes run in order on one stream

    e2e_steps = max(3, min(args.steps, 10))
    e2e_total = pipelined_e2e(host, dev_in, host_out, dev_out, run, e2e_steps, max(1, args.warmup // 2), world)
    e2e_total = max_over_ranks(e2e_total, world)
    res["e2e"] = {"value": tokens / (e2e_total / e2e_steps / 1e3), "unit": "tokens/s",
                  "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h}
    return res


def softplus_leg(args, kda, dev, stream, rank, world, hbm, peak_src):
    """The prefill workload through Kimi Linear's unbounded gate (gate="softplus"): kernel P (with the
    pairwise diagonal tiles of the blocks whose decay leaves the factorisation's range) and kernel S;
    device-timed only."""
    w = W.PREFILL
    d = W.make_scan_inputs(w)
    B, T, H, K, V = w.B, w.T, w.H, w.K, w.V
    g = {n: (x.to(dev) if isinstance(x, torch.Tensor) else x) for n, x in d.items()}
    o = torch.empty(B, T, H, V, device=dev, dtype=torch.bfloat16)
    sf = torch.empty(B, H, K, V, device=dev, dtype=torch.float32)
    ws = torch.empty(max(kda.prefill_workspace_bytes(B, T, H, K, V, 0, torch.bfloat16), 1), device=dev,
                     dtype=torch.uint8)

    def fn():
        kda.prefill_logits(g["q"], g["k"], g["v"], g["z"], g["A_log"], w.g_min, g["beta"], None, gate="softplus",
                           out=o, final_state=sf, workspace=ws)

    steps = max(3, min(args.steps, 20))
    total_ms, (ms,) = timed_loop([fn], steps, args.warmup, world, stream)
    value, total_ms = weak_scaling_value(B * T * steps, total_ms, world)
    pb = prefill_bytes(B, T, H, K, V, 0, 1)
    achieved = pb / (ms / 1e3) / 1e9
    return {
        "workload": w.name + "_softplus_gate", "value": value, "unit": "tokens/s", "ms_per_step": total_ms / steps,
        "steps": steps, "gpu_launches": 2 * steps,  # kernel P, kernel S
        "kernels_ms": {"prefill_logits_softplus": ms},
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": hbm, "unit": "GB/s", "frac": achieved / hbm,
                     "traffic": measured_traffic("softplus"), "kernel": "kda_prefill_logits (KDA_GATE_SOFTPLUS)",
                     "bytes_per_launch": pb, "ms_per_launch": ms, "peak_source": f"{peak_src} hbm_gbs"},
    }


def workload_leg(args, kda, dev, stream, rank, world, hbm, bf16_peak, peak_src, w, cpu_heads, key):
    """Throughput of one more prefill workload through the same call as the headline (kda_prefill_logits,
    two-kernel path, gate from the logits): the 16 packed variable-length sequences with their own initial
    states, or the long K != V batch. tokens/s, the HBM roofline of its algorithmic bytes, e2e through
    pinned host buffers and the oracle on a sample of heads."""
    d = W.make_scan_inputs(w)
    cu = d["cu_seqlens"]
    B, T, H, K, V = d["q"].shape[0], d["q"].shape[1], w.H, w.K, w.V
    N = B if cu is None else cu.numel() - 1
    g = {n: (x.to(dev) if isinstance(x, torch.Tensor) else x) for n, x in d.items()}
    o = torch.empty(B, T, H, V, device=dev, dtype=torch.bfloat16)
    sf = torch.empty(N, H, K, V, device=dev, dtype=torch.float32)
    ws = torch.empty(max(kda.prefill_workspace_bytes(B, T, H, K, V, 0 if cu is None else N, torch.bfloat16), 1),
                     device=dev, dtype=torch.uint8)

    def fn():
        kda.prefill_logits(g["q"], g["k"], g["v"], g["z"], g["A_log"], w.g_min, g["beta"], g["initial_state"],
                           g["cu_seqlens"], out=o, final_state=sf, workspace=ws)

    steps = max(3, min(args.steps, 20))
    sampler = ClockSampler(dev.index if dev.index is not None else 0) if rank == 0 else None
    total_ms, (ms,) = timed_loop([fn], steps, args.warmup, world, stream, sampler)
    value, total_ms = weak_scaling_value(B * T * steps, total_ms, world)
    pb = prefill_bytes(B, T, H, K, V, N, N)
    achieved = pb / (ms / 1e3) / 1e9
    flops = prefill_flops(B, T, H, K, V)
    res = {
        "workload": w.name, "value": value, "unit": "tokens/s", "ms_per_step": total_ms / steps, "steps": steps,
        "tokens_per_step": B * T, "gpu_launches": 2 * steps,  # kernel P, kernel S
        "kernels_ms": {"prefill_logits": ms},
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": hbm, "unit": "GB/s", "frac": achieved / hbm,
                     "traffic": measured_traffic(key), "kernel": "kda_prefill_logits", "bytes_per_launch": pb,
                     "ms_per_launch": ms,
                     "peak_source": f"{peak_src} hbm_gbs",
                     "tensor": {"tflops_at_C64_formula": flops / (ms / 1e3) / 1e12, "peak": bf16_peak,
                                "frac": flops / (ms / 1e3) / 1e12 / bf16_peak, "flops_per_launch": flops}},
        "clocks": sampler.summary() if sampler else None,
    }
    if not args.no_e2e:
        names = ("q", "k", "v", "z", "A_log", "beta", "initial_state")
        host = {n: d[n].pin_memory() for n in names}
        host_out = {"o": torch.empty(B, T, H, V, dtype=torch.bfloat16).pin_memory(),
                    "sf": torch.empty(N, H, K, V, dtype=torch.float32).pin_memory()}
        dev_in = [{n: torch.empty_like(x, device=dev) for n, x in host.items()} for _ in range(2)]
        dev_out = [{"o": o, "sf": sf}, {"o": torch.empty_like(o), "sf": torch.empty_like(sf)}]
        h2d = sum(x.numel() * x.element_size() for x in host.values())
        d2h = sum(x.numel() * x.element_size() for x in host_out.values())

        def run(i, out):
            kda.prefill_logits(i["q"], i["k"], i["v"], i["z"], i["A_log"], w.g_min, i["beta"], i["initial_state"],
                               g["cu_seqlens"], out=out["o"], final_state=out["sf"], workspace=ws)

        e2e_steps = 3
        e2e_total = pipelined_e2e(host, dev_in, host_out, dev_out, run, e2e_steps, 1, world)
        e2e_total = max_over_ranks(e2e_total, world)
        res["e2e"] = {"value": B * T * world / (e2e_total / e2e_steps / 1e3), "unit": "tokens/s",
                      "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h}
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        import oracle
        oracle._load()
        hs = list(range(cpu_heads))
        s0 = d["initial_state"][:, hs] if d["initial_state"] is not None else None
        t_start = time.perf_counter()
        alpha = oracle.bounded_decay(d["z"][:, :, hs], d["A_log"][hs], w.g_min)
        oracle.scan(d["q"][:, :, hs], d["k"][:, :, hs], d["v"][:, :, hs], alpha, d["beta"][:, :, hs], s0, cu)
        dt = time.perf_counter() - t_start
        res["cpu_baseline"] = {"value": B * T * cpu_heads / H / dt, "unit": "tokens/s", "cores": oracle.max_threads(),
                               "kind": "oracle",
                               "sample": f"{w.name}, {cpu_heads} of {H} heads, every token; fp64 gate + "
                                         f"token-by-token scan; {dt:.2f} s; tokens/s scaled to all heads"}
    return res


def backward_bytes(B, T, H, K, V, es=2):
    """Minimum HBM bytes of one backward step from the logits, per token-head: the gate (read z, write g:
    8K), the scan gradients (read q, k, v in the input dtype, g, beta, dL/do in fp32; write dq, dk, dg, dv,
    dbeta in fp32) and the gate's gradient (read z and dg, write dz: 12K)."""
    gate = 8 * K
    scan = (2 * K + V) * es + 4 * K + 4 + 4 * V + 4 * (3 * K + V) + 4
    gate_bwd = 12 * K
    return B * T * H * (gate + scan + gate_bwd)


def backward_leg(args, kda, dev, stream, rank, world, hbm, peak_src):
    """Gradients of the prefill from logits: the log-decay gate, the scan's gradients and
    kda_bounded_decay_backward, on the prefill workload with dL/do ~ N(0, 1). The line's value is the chunked
    backward (kda_scan_backward_chunked, parallel over chunks); the exact token-level adjoint
    (kda_scan_backward) is timed beside it."""
    w = W.PREFILL
    d = W.make_scan_inputs(w)
    B, T, H, K, V = w.B, w.T, w.H, w.K, w.V
    g = {n: (x.to(dev) if isinstance(x, torch.Tensor) else x) for n, x in d.items()}
    d_o = W.make_output_grad(w).to(dev)
    ws = torch.empty(kda.chunked_backward_workspace_bytes(B, T, H, K, V), device=dev, dtype=torch.uint8)

    def chunked_fn():
        lg = kda.bounded_decay(g["z"], g["A_log"], w.g_min, log_decay=True)
        grads = kda.scan_backward_chunked(g["q"], g["k"], g["v"], lg, g["beta"], None, d_o, gate_is_log=True,
                                          workspace=ws)
        kda.bounded_decay_backward(g["z"], g["A_log"], w.g_min, grads["dgate"])

    def exact_fn():
        lg = kda.bounded_decay(g["z"], g["A_log"], w.g_min, log_decay=True)
        grads = kda.scan_backward(g["q"], g["k"], g["v"], lg, g["beta"], None, d_o, gate_is_log=True)
        kda.bounded_decay_backward(g["z"], g["A_log"], w.g_min, grads["dgate"])

    steps = max(3, min(args.steps, 10))
    total_ms, (ms,) = timed_loop([chunked_fn], steps, args.warmup, world, stream)
    _, (ms_exact,) = timed_loop([exact_fn], steps, args.warmup, world, stream)
    value, total_ms = weak_scaling_value(B * T * steps, total_ms, world)
    nb = backward_bytes(B, T, H, K, V)
    achieved = nb / (ms / 1e3) / 1e9
    return {
        "workload": w.name + "_backward", "value": value, "unit": "tokens/s", "ms_per_step": total_ms / steps,
        "steps": steps,
        # per step: gate; forward kernels P and S; prep, pair, inverse, dstate, mask_dgc, dt, da, assemble;
        # gate gradient (the 14 batched products are cuBLAS's)
        "gpu_launches": 12 * steps,
        "kernels_ms": {"backward_from_logits_chunked": ms, "backward_from_logits_exact": ms_exact},
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": hbm, "unit": "GB/s", "frac": achieved / hbm,
                     "traffic": measured_traffic("backward_chunked"),
                     "kernel": "kda_scan_backward_chunked (+ gate and gate gradient)",
                     "bytes_per_launch": nb, "ms_per_launch": ms, "peak_source": f"{peak_src} hbm_gbs",
                     "note": "achieved counts the minimum bytes of the gradients; the chunked path moves fp32 "
                             "per-chunk matrices through HBM between its kernels and cuBLAS products (traffic)"},
        "exact": {"ms_per_step": ms_exact, "value": B * T * world / (ms_exact / 1e3), "unit": "tokens/s",
                  "kernel": "kda_scan_backward (token-serial adjoint, one CTA per head)",
                  "traffic": measured_traffic("backward")},
    }


def cpu_backward_sample(T=1024, n_heads=8):
    """Times the fp64 oracle's gradients (gate and scan through autograd) on a slice of the prefill workload;
    returns tokens/s scaled to all heads of the workload."""
    import time
    import oracle
    w = W.PREFILL
    d = W.make_scan_inputs(w, T=T)
    hs = list(range(n_heads))
    d_o = W.make_output_grad(w, T=T)[:, :, hs].numpy()
    q, k, v = (d[n][:, :, hs] for n in ("q", "k", "v"))
    z, A_log, beta = d["z"][:, :, hs], d["A_log"][hs], d["beta"][:, :, hs]
    t = time.perf_counter()
    alpha = oracle.bounded_decay(z, A_log, w.g_min)
    r = oracle.scan_backward(q, k, v, alpha, beta, None, d_o)
    oracle.bounded_decay_backward(z, A_log, w.g_min, r["alpha"] * alpha)
    dt = time.perf_counter() - t
    return {"value": T * n_heads / dt / w.H, "unit": "tokens/s", "cores": torch.get_num_threads(), "kind": "oracle",
            "sample": f"backward of the prefill workload, {n_heads} of {w.H} heads, first {T} tokens, fp64 autograd; "
                      f"{dt:.2f} s; tokens/s scaled to all heads"}


def decode_leg(args, kda, dev, stream, rank, world, hbm, peak_src):
    dw = W.DECODE
    prm = W.make_decode_params(dw)
    state = prm["state"].to(dev)
    A_dec = prm["A_log"].to(dev)
    n_sets = 4
    sets = [{n: x.to(dev) for n, x in W.make_decode_step(dw, s).items()} for s in range(n_sets)]
    o_dec = torch.empty(dw.B, dw.H, dw.V, device=dev, dtype=torch.bfloat16)
    it = {"i": 0}

    # One call per step: the decode kernel reads the decay logits and evaluates the gate itself.
    def dstep_fn():
        s = sets[it["i"] % n_sets]
        kda.decode_step_logits(s["q"], s["k"], s["v"], s["z"], A_dec, dw.g_min, s["beta"], state, out=o_dec)
        it["i"] += 1

    dsteps = max(args.steps, 20)
    dsampler = ClockSampler(dev.index if dev.index is not None else 0) if rank == 0 else None
    d_total, (dk_ms,) = timed_loop([dstep_fn], dsteps, args.warmup, world, stream, dsampler)
    sbytes = decode_state_bytes(dw.B, dw.H, dw.K, dw.V)
    d_bps, d_total = weak_scaling_value(sbytes * dsteps, d_total, world)
    d_ms = d_total / dsteps
    dbytes = decode_bytes(dw.B, dw.H, dw.K, dw.V)
    d_achieved = dbytes / (dk_ms / 1e3) / 1e9
    res = {
        "workload": dw.name, "value": d_bps / 1e9, "unit": "GB/s (state)",
        "steps_per_s": 1e3 / d_ms, "ms_per_step": d_ms, "steps": dsteps, "gpu_launches": dsteps,
        "kernels_ms": {"decode_step_logits": dk_ms},
        "roofline": {"bound": "hbm", "achieved": d_achieved, "peak": hbm, "unit": "GB/s",
                     "frac": d_achieved / hbm, "traffic": measured_traffic("decode"), "kernel": "kda_decode_step_logits",
                     "bytes_per_launch": dbytes, "ms_per_launch": dk_ms, "peak_source": f"{peak_src} hbm_gbs"},
        "clocks": dsampler.summary() if dsampler is not None else None,
    }
    if args.no_e2e:
        return res
    # e2e: each step's q, k, v, z, beta from pinned host memory, the step on the kept state, o back to the host;
    # consecutive steps overlapped (the state update itself stays in order on one stream)
    # A step's five small inputs travel as one copy: packed into one pinned buffer per input set (256-byte
    # aligned pieces), unpacked on the device as views of one buffer.
    steps_in = [W.make_decode_step(dw, s) for s in range(n_sets)]
    layout, total = {}, 0
    for n, x in steps_in[0].items():
        layout[n] = (total, x.numel() * x.element_size(), x.dtype, tuple(x.shape))
        total += (layout[n][1] + 255) // 256 * 256
    hostd = []
    for st in steps_in:
        buf = torch.zeros(total, dtype=torch.uint8).pin_memory()
        for n, (off, nb, dt, shp) in layout.items():
            buf[off:off + nb].copy_(st[n].contiguous().view(torch.uint8).reshape(-1))
        hostd.append({"buf": buf})
    devd = []
    for _ in range(2):
        dbuf = torch.empty(total, dtype=torch.uint8, device=dev)
        devd.append({"buf": dbuf, **{n: dbuf[off:off + nb].view(dt).view(shp)
                                     for n, (off, nb, dt, shp) in layout.items()}})
    host_out = {"o": torch.empty(dw.B, dw.H, dw.V, dtype=torch.bfloat16).pin_memory()}
    dev_out = [{"o": o_dec}, {"o": torch.empty_like(o_dec)}]
    dh2d = sum(nb for _, nb, _, _ in layout.values())
    dd2h = host_out["o"].numel() * host_out["o"].element_size()

    def drun(i, out):
        kda.decode_step_logits(i["q"], i["k"], i["v"], i["z"], A_dec, dw.g_min, i["beta"], state, out=out["o"])

    de_total = pipelined_e2e(hostd, devd, host_out, dev_out, drun, dsteps, args.warmup, world)
    de_total = max_over_ranks(de_total, world)
    res["e2e"] = {"value": sbytes * world / (de_total / dsteps / 1e3) / 1e9, "unit": "GB/s (state)",
                  "h2d_bytes_per_step": dh2d, "d2h_bytes_per_step": dd2h}
    return res


def gpu_arm(args, rank, world, local):
    import gated_delta_rule_bounded_b200 as kda
    kda.load_library()
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    stream = torch.cuda.current_stream(dev)
    peaks, peak_src = load_peaks()
    hbm = float(peaks["hbm_gbs"])
    bf16_peak = float(peaks.get("bf16_tflops", PEAKS_FALLBACK["bf16_tflops"]))
    pre = dec = None
    if args.workload in ("all", "prefill"):
        pre = prefill_leg(args, kda, dev, stream, rank, world, hbm, bf16_peak, peak_src)
        torch.cuda.empty_cache()
    if args.workload in ("all", "decode"):
        dec = decode_leg(args, kda, dev, stream, rank, world, hbm, peak_src)
        torch.cuda.empty_cache()
    spl = None
    if args.workload in ("all", "softplus"):
        spl = softplus_leg(args, kda, dev, stream, rank, world, hbm, peak_src)
        torch.cuda.empty_cache()
    more = {}
    for key, wl, heads in (("varlen", W.VARLEN, 16), ("long_kv", W.LONG_KV, 4)):
        if args.workload in ("all", key):
            more[key] = workload_leg(args, kda, dev, stream, rank, world, hbm, bf16_peak, peak_src, wl, heads, key)
            torch.cuda.empty_cache()
    bwd = None
    if args.workload in ("all", "backward"):
        bwd = backward_leg(args, kda, dev, stream, rank, world, hbm, peak_src)
        if rank == 0 and world == 1 and not args.no_cpu_baseline:
            bwd["cpu_baseline"] = cpu_backward_sample()
    cpu = cpu_baseline(args) if (rank == 0 and world == 1 and not args.no_cpu_baseline) else None
    if pre is None and dec is None:  # single-leg profiling run
        return {"metric": METRIC, "workload_only": args.workload, "backward": bwd, "softplus": spl, **more}
    if pre is None:  # decode-only profiling run
        return {"metric": METRIC, "workload_only": "decode", "decode": dec}
    w = pre["workload"]
    line = {
        "metric": METRIC,
        "value": pre["value"],
        "unit": "tokens/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": pre["ms_per_step"],
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16",
        "data": "synthetic (seeded; no dataset)",
        "config": {"workload": w.name, "B": w.B, "T": w.T, "H": w.H, "K": w.K, "V": w.V, "g_min": w.g_min,
                   "z_std": w.z_std, "initial_state": "zeros", "step": "prefill from decay logits z (bounded gate evaluated inside the scan kernels)",
                   "l2": "inputs larger than L2 (q/k/v/z ~ 0.5 GB, workspace 0.4 GB); no flush",
                   "parallelism": f"replica per GPU x{world}"},
        "roofline": pre["roofline"],
        "kernels_ms": pre["kernels_ms"],
        "e2e": pre.get("e2e"),
        "gpu_launches": pre["gpu_launches"],
        "clocks": pre["clocks"],
    }
    if dec is not None:
        line["decode"] = dec
    if spl is not None:
        line["softplus"] = spl
    line.update(more)
    if bwd is not None:
        line["backward"] = bwd
    if cpu is not None:
        line["cpu_baseline"] = cpu
    return line


# ------------------------------------------------------------------------------------------------
# CPU oracle (baseline leg and reference arm)
# ------------------------------------------------------------------------------------------------

def oracle_prefill_sample(n_heads, inputs=None, threads=0):
    """Times the fp64 oracle (gate + scan) on `n_heads` heads of the prefill workload.
    Returns (seconds, tokens-equivalent of the full workload processed)."""
    import oracle
    w = W.PREFILL
    d = inputs if inputs is not None else W.make_scan_inputs(w)
    hs = list(range(n_heads))
    sub = {n: d[n][:, :, hs] for n in ("q", "k", "v", "z", "beta")}
    t0 = time.perf_counter()
    alpha = oracle.bounded_decay(sub["z"], d["A_log"][hs], w.g_min)
    oracle.scan(sub["q"], sub["k"], sub["v"], alpha, sub["beta"], None, None, n_threads=threads)
    dt = time.perf_counter() - t0
    return dt, w.B * w.T * n_heads / w.H


def cpu_baseline(args):
    import oracle
    oracle._load()
    cores = oracle.max_threads()
    d = W.make_scan_inputs(W.PREFILL)
    n_heads = max(1, min(W.PREFILL.H, args.cpu_heads or 4 * cores))
    dt, tok = oracle_prefill_sample(n_heads, d)
    return {"value": tok / dt, "unit": "tokens/s", "cores": cores, "kind": "oracle",
            "sample": f"prefill workload, {n_heads} of {W.PREFILL.H} heads, full T={W.PREFILL.T}, "
                      f"fp64 gate + token-by-token scan; {dt:.2f} s; tokens/s scaled to all heads"}


def reference_arm(args, rank, world):
    if rank != 0:
        return None
    import oracle
    oracle._load()
    cores = oracle.max_threads()
    d = W.make_scan_inputs(W.PREFILL)
    n_heads = max(1, min(W.PREFILL.H, args.cpu_heads or cores))
    for _ in range(args.warmup):
        oracle_prefill_sample(n_heads, d)
    times, tok = [], 0.0
    for _ in range(args.steps):
        dt, tok = oracle_prefill_sample(n_heads, d)
        times.append(dt)
    ms = 1e3 * sum(times) / len(times)
    value = tok / (ms / 1e3)
    sample = (f"each step: prefill workload, {n_heads} of {W.PREFILL.H} heads, full T={W.PREFILL.T}, "
              f"fp64 gate + token-by-token scan on {cores} threads; tokens/s scaled to all heads")
    return {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic (seeded; no dataset)",
        "config": {"workload": W.PREFILL.name, "B": W.PREFILL.B, "T": W.PREFILL.T, "H": W.PREFILL.H,
                   "K": W.PREFILL.K, "V": W.PREFILL.V, "g_min": W.PREFILL.g_min},
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": cores, "kind": "oracle", "sample": sample},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
        "gpu_launches": 0,
    }


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["kda", "reference"], default="kda")
    ap.add_argument("--cpu-heads", type=int, default=0, help="heads in the oracle sample (0: auto)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--workload", choices=["all", "prefill", "decode", "softplus", "varlen", "long_kv", "backward"],
                    default="all",
                    help="one leg alone (profiling runs); the JSON line needs 'all'")
    ap.add_argument("--no-e2e", action="store_true", help="skip the host-buffer end-to-end legs")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    rank, world, local = dist_setup(args.gpus)
    try:
        if args.impl == "reference":
            line = reference_arm(args, rank, world)
        else:
            line = gpu_arm(args, rank, world, local)
        if rank == 0 and line is not None:
            print(json.dumps(line), flush=True)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
