#!/usr/bin/env python
"""Throughput of the sparse MoE feed-forward layer (Mixtral 8x7B shapes) on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload prefill|decode|skewed]
                    [--impl ours|reference] [--no-extras]

A step is one full layer (router, permutation, both grouped GEMMs, combine)
over the workload's T tokens, through the C ABI (moe_layer_forward_ex), with
inputs resident in HBM.  Default workload: the prefill layer, T = 4096
tokens, d = 4096, f = 14336, E = 8, top-2, bf16.  With N > 1 (torchrun, one
process per GPU) every rank runs its own T tokens on its own replica of the
weights; the layer needs no exchange between ranks, so there is no
collective on the data path (weak scaling).  Rank 0 prints one JSON line.

Timing: W untimed warm-up steps, then K steps between a barrier and a device
synchronisation on both sides; each step is bracketed by CUDA events on the
launching stream and the L2 is flushed (a 512 MiB write) between steps,
outside the events.  The elapsed time is the max over ranks.

The roofline object is the up-projection GEMM's (the dominant kernel): its
algorithmic flops (bytes at decode) over its CUDA-event launch time, against
the measured bf16 peak of the clock regime the timed steps ran in (the SM
clock is sampled during them): the sustained figure when the power cap held
the clock well below its maximum, the burst figure otherwise; both fractions
are reported.

--impl reference times the fp64 CPU oracle on the host cores (rank 0 only)
on a bounded sample of the same workload.
"""

from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "MoE-layer tokens/sec and TFLOP/s (fraction of bf16 peak / HBM GB/s) on 1 B200"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=300)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--workload", default="prefill", choices=["prefill", "decode", "skewed"])
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-extras", action="store_true", help="skip the decode line and the CPU baseline")
    ap.add_argument("--cpu-sample", type=int, default=4096,
                    help="tokens in the oracle's timed CPU-baseline sample (default: the whole prefill batch)")
    ap.add_argument("--ref-sample", type=int, default=4096,
                    help="tokens per step of --impl reference: by default the whole prefill batch, the same "
                         "sample as the cpu_baseline leg (~4 s per step on 16 cores)")
    ap.add_argument("--e2e-chunks", type=int, default=1,
                    help="pieces the end-to-end leg pipelines host copies and compute in")
    ap.add_argument("--gemm-vs-cublas", action="store_true",
                    help="instead of the layer: time the two expert GEMMs against cuBLAS (torch.matmul) "
                         "on the same shapes and print one JSON line")
    return ap.parse_args()


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return d, "measured"
    return FALLBACK_PEAKS, "fallback"


def clock_regime(clocks):
    """Which measured bf16 peak the timed steps are held to: "sustained" when
    the SM clock sampled during them had a median below 92 % of its maximum
    (the power cap holding it down over a long run), else "burst" (a short
    timed region at full clock; also when no clock was sampled)."""
    if not clocks or not clocks.get("sm_mhz") or not clocks.get("sm_max_mhz"):
        return "burst"
    return "sustained" if clocks["sm_mhz"] < 0.92 * clocks["sm_max_mhz"] else "burst"


def workload_desc(s, n):
    return {"workload": "Mixtral-8x7B MoE FFN layer, %s: T=%d tokens per GPU, d=%d, f=%d, E=%d, top-%d, %s"
                        % (s.name, s.T, s.d, s.f, s.E, s.k, s.dtype),
            "T": s.T, "d": s.d, "f": s.f, "E": s.E, "k": s.k, "routing": "skewed (Zipf log prior, hottest expert 35%)"
            if s.skew else "near-uniform (Wg ~ N(0, 1/d))",
            "global_batch_tokens": s.T * n, "parallelism": "replicas x%d (token-sharded, no collective)" % n,
            "l2": "flushed between timed steps (512 MiB write outside the step events); weights 2.82 GB > L2"}


class ClockSampler:
    """SM clock, power and clock-event reasons of the benchmarked GPU while
    the timed region runs: NVML read every 2 ms from a side thread (read-only
    queries), else `nvidia-smi -lms 200` if NVML cannot be loaded.  The GPU
    is found by its PCI bus id (NVML numbers all GPUs of the host, whatever
    CUDA_VISIBLE_DEVICES says)."""

    FIELDS = ("index,pci.bus_id,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
    REASONS = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")
    PERIOD_S = 0.002

    def __init__(self, bus_id):
        self.bus_id = (bus_id or "").lower()
        self.proc = None
        self.path = None
        self.nvml = None
        self.handle = None
        self.thread = None
        self.halt = threading.Event()
        self.rows = []
        try:
            import pynvml
            pynvml.nvmlInit()
            key = self.bus_id[-5:] + "."  # "bb:dd." of domain:bus:device
            for i in range(pynvml.nvmlDeviceGetCount()):
                h = pynvml.nvmlDeviceGetHandleByIndex(i)
                bid = pynvml.nvmlDeviceGetPciInfo(h).busId
                bid = (bid.decode() if isinstance(bid, bytes) else bid).lower()
                if self.bus_id and key in bid:
                    self.handle = h
                    break
            if self.handle is not None:
                self.nvml = pynvml
        except Exception:
            self.nvml = None

    def _poll(self):
        n = self.nvml
        bits = (n.nvmlClocksEventReasonHwSlowdown, n.nvmlClocksEventReasonHwThermalSlowdown,
                n.nvmlClocksEventReasonSwThermalSlowdown, n.nvmlClocksEventReasonSwPowerCap)
        while not self.halt.is_set():
            try:
                sm = n.nvmlDeviceGetClockInfo(self.handle, n.NVML_CLOCK_SM)
                r = n.nvmlDeviceGetCurrentClocksEventReasons(self.handle)
                w = n.nvmlDeviceGetPowerUsage(self.handle) / 1000.0
                self.rows.append((sm, w, tuple(bool(r & b) for b in bits)))
            except Exception:
                return
            time.sleep(self.PERIOD_S)

    def start(self):
        if self.nvml is not None:
            self.thread = threading.Thread(target=self._poll, daemon=True)
            self.thread.start()
            return
        try:
            fd, self.path = tempfile.mkstemp(suffix=".csv")
            os.close(fd)
            self.proc = subprocess.Popen(["nvidia-smi", "--query-gpu=" + self.FIELDS, "--format=csv,noheader,nounits",
                                          "-lms", "200", "-f", self.path], stdout=subprocess.DEVNULL,
                                         stderr=subprocess.DEVNULL)
            time.sleep(0.5)
        except Exception:
            self.proc = None

    def stop(self):
        if self.thread is not None:
            self.halt.set()
            self.thread.join()
            if not self.rows:
                return None
            n = self.nvml
            try:
                mx = float(n.nvmlDeviceGetMaxClockInfo(self.handle, n.NVML_CLOCK_SM))
            except Exception:
                mx = None
            reasons = sorted({self.REASONS[i] for _, _, f in self.rows for i in range(4) if f[i]})
            sm = [float(r[0]) for r in self.rows]
            return {"sm_mhz": statistics.median(sm), "sm_min_mhz": min(sm), "sm_max_mhz": mx, "reasons": reasons,
                    "samples": len(self.rows), "source": "NVML every %g ms during the timed steps" % (1e3 * self.PERIOD_S),
                    "power_w_max": max(r[1] for r in self.rows)}
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        rows = []
        for line in open(self.path):
            f = [c.strip() for c in line.split(",")]
            if len(f) < 10:
                continue
            if self.bus_id and self.bus_id[-12:] not in f[1].lower():
                continue
            rows.append(f)
        os.unlink(self.path)
        if not rows:
            return None
        sm = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        mx = max(float(r[3]) for r in rows if r[3].replace(".", "").isdigit())
        reasons = sorted({self.REASONS[i] for r in rows for i in range(4) if r[6 + i].lower().startswith("active")})
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": mx, "reasons": reasons,
                "samples": len(rows), "source": "nvidia-smi every 200 ms",
                "power_w_max": max(float(r[4]) for r in rows if r[4].replace(".", "").isdigit())}


def gemm_source_hash():
    p = os.path.join(ROOT, "sparse_mixture_experts_06_b200", "csrc", "gemm_sm100.cu")
    return hashlib.sha256(open(p, "rb").read()).hexdigest()[:16]


def traffic_record(kernel):
    """DRAM bytes per launch from the committed ncu summary, if it was taken on this kernel source."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    d = json.load(open(p)).get(kernel)
    if not d or d.get("source_sha256_16") != gemm_source_hash():
        return None
    return d


# --------------------------------------------------------------------- replicas (N > 1)

def replica_x_seed(rank: int) -> int:
    """Seed of rank `rank`'s tokens: every replica holds the same weights
    (seed 0) and its own T tokens."""
    return 1000 + rank


def max_over_ranks(ms: float, dist, device) -> float:
    """The job's elapsed time: the max of the ranks' device-timed totals.
    A side reduction of one scalar, outside the timed region; the layer
    itself exchanges nothing between ranks."""
    if dist is None:
        return ms
    import torch
    tt = torch.tensor([ms], dtype=torch.float64, device=device)
    dist.all_reduce(tt, op=dist.ReduceOp.MAX)
    return float(tt.item())


def job_tokens_per_s(world: int, T: int, steps: int, total_ms: float) -> float:
    """Whole-job throughput: tokens processed by all ranks / the max elapsed."""
    return world * T * steps / (total_ms * 1e-3)


# --------------------------------------------------------------------- oracle (CPU) side

def oracle_weights_f64(t, E):
    """Host fp64 copies of the weights (input marshalling for the oracle)."""
    import numpy as np
    import synth
    from synth.device import to_host_bits
    out = {}
    for name in ("W1", "W3", "W2"):
        bits = to_host_bits(t[name])
        out[name] = np.stack([synth.bf16_bits_to_f64(bits[e]) for e in range(E)])
    out["Wg"] = synth.bf16_bits_to_f64(to_host_bits(t["Wg"]))
    return out


def time_oracle(w64, x_bits, k):
    """Times oracle.moe_forward on the host rows x_bits (as it stands)."""
    import oracle
    import synth
    from threadpoolctl import threadpool_info
    x64 = synth.bf16_bits_to_f64(x_bits)
    t0 = time.perf_counter()
    oracle.moe_forward(x64, w64["Wg"], w64["W1"], w64["W3"], w64["W2"], k)
    dt = time.perf_counter() - t0
    threads = max([i.get("num_threads", 1) for i in threadpool_info()] + [1])
    return dt, threads


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    import numpy as np
    import torch
    import synth
    from synth.device import device_inputs, to_host_bits
    s = synth.CONFIGS[args.workload]
    t = device_inputs(s, 0)
    w64 = oracle_weights_f64(t, s.E)
    x_bits = to_host_bits(t["x"])
    del t
    torch.cuda.empty_cache()
    n = args.ref_sample
    rng = np.random.default_rng(0)
    times = []
    threads = 1
    for i in range(args.warmup + args.steps):
        rows = np.sort(rng.choice(s.T, size=min(n, s.T), replace=False))
        dt, threads = time_oracle(w64, x_bits[rows], s.k)
        if i >= args.warmup:
            times.append(dt)
    tot = sum(times)
    value = len(times) * min(n, s.T) / tot
    line = {"metric": METRIC, "impl": "reference", "value": value, "unit": "tokens/s", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * tot / len(times),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "config": workload_desc(s, 1),
            "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": threads, "kind": "oracle",
                             "sample": "%d random tokens of the %s workload per step (router, top-k, both "
                                       "experts, combine in fp64; the same sample size as the cpu_baseline "
                                       "leg of the default run, so the two throughputs agree)"
                                       % (min(n, s.T), s.name)},
            "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


# --------------------------------------------------------------------- GPU side

def make_inputs(s, rank, device):
    import torch
    import synth
    from synth.device import device_inputs, normal_tensor
    t = device_inputs(synth.MoEShape(s.name, s.T, s.d, s.f, s.E, s.k, s.dtype, skew=s.skew), 0,
                      device=device, with_x=False)
    t["x"] = normal_tensor((s.T, s.d), replica_x_seed(rank), synth.tensor_id(synth.TENSOR_X), 1.0, s.dtype, device)
    if s.skew:
        t["x"][:, -1] = 1.0
    torch.cuda.synchronize()
    return t


def timed_loop(step, steps, flush, stream):
    """K steps, each between two events on the launching stream; with `flush`
    (a buffer larger than L2) written before each step, outside its events;
    with flush=None the steps run back to back (inputs larger than L2)."""
    import torch
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
    for a, b in evs:
        if flush is not None:
            flush.zero_()
        a.record(stream)
        step()
        b.record(stream)
    return evs


def bench_workload(args, s, rank, world, device, dist, extras_for_decode=False, record_up=True, l2_flush=True):
    import torch
    import sparse_mixture_experts_06_b200 as moe
    t = make_inputs(s, rank, device)
    stream = torch.cuda.current_stream(device)
    y = torch.empty_like(t["x"])
    ws = torch.empty(moe.moe_workspace_size(s.T, s.d, s.f, s.E, s.k, 0), dtype=torch.uint8, device=device)
    flush = torch.empty(512 << 20, dtype=torch.uint8, device=device)

    def step():
        moe.moe_layer_forward_ex(t["x"], t["Wg"], t["W1"], t["W3"], t["W2"], s.k, y=y, workspace=ws, stream=stream)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize(device)
    if dist is not None:
        dist.barrier()
    torch.cuda.synchronize(device)
    # inside the timed steps only the up-projection GEMM (the roofline's kernel)
    # is bracketed by events: events between kernels serialise them (they undo
    # the programmatic-launch overlap with its neighbours) and cost ~50 us per
    # prefill step if every kernel had them; record_up=False times the steps
    # with no event inside at all
    if record_up:
        moe.moe_profile_select(["up_swiglu_gemm"])
        moe.moe_profile_enable(True)
    props = torch.cuda.get_device_properties(device)
    bus = "%04x:%02x:%02x" % (getattr(props, "pci_domain_id", 0), getattr(props, "pci_bus_id", 0),
                              getattr(props, "pci_device_id", 0)) if hasattr(props, "pci_bus_id") else ""
    sampler = ClockSampler(bus) if rank == 0 and not extras_for_decode else None
    if sampler:
        sampler.start()
    evs = timed_loop(step, args.steps, flush if l2_flush else None, stream)
    torch.cuda.synchronize(device)
    if dist is not None:
        dist.barrier()
    torch.cuda.synchronize(device)
    clocks = sampler.stop() if sampler else None
    flushed_ms = None
    if not l2_flush:
        # the same steps with the L2 flush between them, for comparison
        fe = timed_loop(step, args.steps, flush, stream)
        torch.cuda.synchronize(device)
        flushed_ms = [a.elapsed_time(b) for a, b in fe]
    moe.moe_profile_enable(False)
    prof_up = moe.moe_profile_read() if record_up else None
    step_ms = [a.elapsed_time(b) for a, b in evs]
    total_ms = max_over_ranks(sum(step_ms), dist, device)
    # per-stage breakdown: a separate, untimed pass with every stage recorded
    nb = max(5, min(args.steps, 50))
    moe.moe_profile_select(None)
    moe.moe_profile_enable(True)
    timed_loop(step, nb, flush, stream)
    torch.cuda.synchronize(device)
    moe.moe_profile_enable(False)
    prof = moe.moe_profile_read()
    deverr = moe.moe_device_errors()
    res = {"t": t, "y": y, "ws": ws, "total_ms": total_ms, "step_ms": step_ms, "prof_up": prof_up, "prof": prof,
           "flushed_step_ms": flushed_ms,
           "breakdown_steps": nb, "clocks": clocks, "deverr": deverr, "stream": stream}
    return res


def bench_stack(steps, device, pk):
    """The 32-layer stack (T = 8192, 90 GB of per-layer weights, residual
    between layers) as one moe_stack_forward call captured in a CUDA graph."""
    import torch
    import sparse_mixture_experts_06_b200 as moe
    import synth
    from synth.device import device_inputs, normal_tensor
    import dataclasses
    s = synth.CONFIGS["stack"]
    one = dataclasses.replace(s, name="stack-layer", layers=1)
    layers = []
    for l in range(s.layers):
        w = device_inputs(one, 0, layer=l, device=device, with_x=False)
        layers.append((w["Wg"], w["W1"], w["W3"], w["W2"]))
    x = normal_tensor((s.T, s.d), replica_x_seed(0), synth.tensor_id(synth.TENSOR_X), 1.0, s.dtype, device)
    y = torch.empty_like(x)
    scratch = torch.empty_like(x)
    ws = torch.empty(moe.moe_workspace_size(s.T, s.d, s.f, s.E, s.k, 0), dtype=torch.uint8, device=device)
    moe.moe_stack_forward(x, layers, s.k, y=y, scratch=scratch, workspace=ws)  # one-time set-up, uncaptured
    torch.cuda.synchronize(device)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        moe.moe_stack_forward(x, layers, s.k, y=y, scratch=scratch, workspace=ws)
    g.replay()
    torch.cuda.synchronize(device)
    stream = torch.cuda.current_stream(device)
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(stream)
    for _ in range(steps):
        g.replay()
    b.record(stream)
    torch.cuda.synchronize(device)
    ms = a.elapsed_time(b) / steps
    out = {"workload": "32-layer Mixtral-8x7B MoE stack, T=%d tokens, residual between layers, per-layer weights "
                       "(%.1f GB, W2 scaled by 1/4 so the residual stream stays finite), one CUDA graph"
                       % (s.T, s.weight_bytes / 1e9),
           "ms_per_step": ms, "tokens_per_s": s.T / (ms * 1e-3), "tflops": s.flops / (ms * 1e-3) / 1e12,
           "frac_of_bf16_peak": s.flops / (ms * 1e-3) / 1e12 / pk["bf16_tflops"], "ms_per_layer": ms / s.layers,
           "steps": steps, "device_error_flags": moe.moe_device_errors()}
    del g, layers
    return out


def graph_step_ms(r, s, device, steps):
    """The same layer call captured once in a CUDA graph and replayed
    (no per-kernel launch gaps; how a serving loop would run decode)."""
    import torch
    import sparse_mixture_experts_06_b200 as moe
    t, y, ws = r["t"], r["y"], r["ws"]
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        moe.moe_layer_forward_ex(t["x"], t["Wg"], t["W1"], t["W3"], t["W2"], s.k, y=y, workspace=ws)
    for _ in range(3):
        g.replay()
    torch.cuda.synchronize(device)
    stream = torch.cuda.current_stream(device)
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(stream)
    for _ in range(steps):
        g.replay()
    b.record(stream)
    torch.cuda.synchronize(device)
    del g
    return a.elapsed_time(b) / steps


def loop_step_ms(r, s, device, steps):
    """The layer called back to back as a serving loop runs it, one event
    pair around all the steps (no event between two layers, which would
    hold back the next layer's programmatic early launch)."""
    import torch
    import sparse_mixture_experts_06_b200 as moe
    t, y, ws = r["t"], r["y"], r["ws"]
    stream = torch.cuda.current_stream(device)
    for _ in range(3):
        moe.moe_layer_forward_ex(t["x"], t["Wg"], t["W1"], t["W3"], t["W2"], s.k, y=y, workspace=ws)
    torch.cuda.synchronize(device)
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(stream)
    for _ in range(steps):
        moe.moe_layer_forward_ex(t["x"], t["Wg"], t["W1"], t["W3"], t["W2"], s.k, y=y, workspace=ws)
    b.record(stream)
    torch.cuda.synchronize(device)
    return a.elapsed_time(b) / steps


def e2e_leg(args, s, t, device, steps):
    """Same layer through the public host-buffer entry point
    moe_layer_forward_host, as a server calls it back to back: every step
    copies its tokens in from pinned host memory and its output back, inside
    the timed region; the library pipelines those copies with the compute of
    the neighbouring pieces (args.e2e_chunks per step, staging alternating
    across steps; x_ready, since the host tokens are ready at each call, and
    y_async, with one moe_layer_forward_host_wait before the end event).
    All of every step's copies are inside the timed region, so the first
    step's copy in and the last step's copy out, which have no neighbouring
    compute to hide behind (~0.7 ms each at prefill over PCIe), add
    ~1.4 ms / steps to the per-step time."""
    import torch
    import sparse_mixture_experts_06_b200 as moe
    x_h = t["x"].cpu().pin_memory()
    y_h = torch.empty_like(x_h).pin_memory()
    stream = torch.cuda.current_stream(device)

    def step():
        moe.moe_layer_forward_host(x_h, t["Wg"], t["W1"], t["W3"], t["W2"], s.k, y=y_h, chunks=args.e2e_chunks,
                                   x_ready=True, y_async=True, stream=stream)

    for _ in range(3):
        step()
    torch.cuda.synchronize(device)
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(stream)
    for _ in range(steps):
        step()
    moe.moe_layer_forward_host_wait(stream)  # the end event follows the last step's copy out
    b.record(stream)
    torch.cuda.synchronize(device)
    ms = a.elapsed_time(b) / steps
    nbytes = x_h.numel() * x_h.element_size()
    return ms, nbytes, y_h.numel() * y_h.element_size()


def gemm_vs_cublas(args, device):
    """The expert GEMMs of the prefill layer (T = 4096, d = 4096, f = 14336,
    E = 8, k = 2) against cuBLAS through torch.matmul, for context.  Four
    arms, run in turn within every step (so that all see the same clocks
    under the power cap), each after an L2 flush; medians over the steps:
      * cuBLAS on one dense GEMM of all 8192 rows (up: [8192, d] x [d, 2f];
        down: [8192, f] x [f, d]), no SwiGLU or gate: cuBLAS's best case;
      * ours on one expert of 8192 rows (E = k = 1): no expert tails;
      * ours on the router's routing of the prefill batch (its expert row
        counts leave short last row blocks, the tails);
      * ours on a balanced routing (token t -> experts 2t mod 8, 2t+1 mod 8:
        1024 rows per expert, a multiple of the 256-row pair tiles).
    Ours through moe_expert_ffn, the GEMM times from the library's stage
    profiler.  cuBLAS is a measuring stick only; the layer never calls it."""
    import numpy as np
    import torch
    import synth
    import sparse_mixture_experts_06_b200 as moe
    from synth.device import device_inputs

    s = synth.CONFIGS["prefill"]
    M, d, f = s.T * s.k, s.d, s.f
    flush = torch.empty(512 << 20, dtype=torch.uint8, device=device)
    g = torch.Generator(device=device).manual_seed(0)
    x = torch.randn(M, d, device=device, generator=g).to(torch.bfloat16)
    W13 = (torch.randn(2 * f, d, device=device, generator=g) / 64).to(torch.bfloat16)
    h = torch.randn(M, f, device=device, generator=g).to(torch.bfloat16)
    W2 = (torch.randn(d, f, device=device, generator=g) / 120).to(torch.bfloat16)

    def timed(fn):
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        fn()
        b.record()
        b.synchronize()
        return a.elapsed_time(b)

    def cublas():
        up = timed(lambda: x @ W13.t())
        flush.zero_()
        return up, timed(lambda: h @ W2.t())

    def ours(tt, routing, ws, y):
        off, perm, inv, w = routing

        def run():
            moe.moe_profile_select(None)
            moe.moe_profile_enable(True)
            moe.moe_expert_ffn(tt["x"], tt["W1"], tt["W3"], tt["W2"], off, perm, inv, w, y=y, workspace=ws)
            torch.cuda.synchronize()
            pr = moe.moe_profile_read()
            moe.moe_profile_enable(False)
            return pr["up_swiglu_gemm"][0], pr["down_combine_gemm"][0]
        return run

    one = synth.MoEShape("one-expert", M, d, f, 1, 1, "bf16")
    t1 = device_inputs(one, 0, device=device)
    r1 = (*moe.moe_permute(torch.zeros(M, 1, dtype=torch.int32, device=device), 1),
          torch.ones(M, 1, dtype=torch.float32, device=device))
    ws1 = torch.empty(moe.moe_workspace_size(M, d, f, 1, 1, 0), dtype=torch.uint8, device=device)
    tp = make_inputs(s, 0, device)
    idx, w = moe.moe_router_topk(tp["x"], tp["Wg"], s.k)
    rr = (*moe.moe_permute(idx, s.E), w)
    bal = np.stack([(2 * np.arange(s.T)) % s.E, (2 * np.arange(s.T) + 1) % s.E], 1).astype(np.int32)
    rb = (*moe.moe_permute(torch.from_numpy(bal).to(device), s.E), w)
    wsp = torch.empty(moe.moe_workspace_size(s.T, d, f, s.E, s.k, 0), dtype=torch.uint8, device=device)
    y1 = torch.empty(M, d, dtype=torch.bfloat16, device=device)
    yp = torch.empty(s.T, d, dtype=torch.bfloat16, device=device)
    arms = {"cublas_dense": cublas, "ours_one_expert": ours(t1, r1, ws1, y1),
            "ours_router_routing": ours(tp, rr, wsp, yp), "ours_balanced_routing": ours(tp, rb, wsp, yp)}
    for fn in arms.values():
        for _ in range(3):
            flush.zero_()
            torch.cuda.synchronize()
            fn()
    res = {k: [] for k in arms}
    steps = max(10, min(args.steps, 40))
    for i in range(steps):
        for k in (list(arms) if i % 2 == 0 else list(arms)[::-1]):
            flush.zero_()
            torch.cuda.synchronize()
            res[k].append(arms[k]())
    tf = lambda flop, ms: round(flop / ms / 1e9, 1)  # noqa: E731
    out = {"mode": "gemm_vs_cublas", "unit": "TFLOP/s", "rows": M, "d": d, "f": f, "steps": steps,
           "router_counts": np.diff(rr[0].cpu().numpy()).tolist()}
    for k, v in res.items():
        up = statistics.median(a for a, _ in v)
        dn = statistics.median(b for _, b in v)
        out[k] = {"up_ms": round(up, 4), "up": tf(4.0 * M * d * f, up), "down_ms": round(dn, 4),
                  "down": tf(2.0 * M * d * f, dn)}
    print(json.dumps(out))
    return 0


def main():
    args = parse()
    if args.impl == "reference":
        return run_reference(args)
    if args.gemm_vs_cublas:
        import torch
        torch.cuda.set_device(0)
        return gemm_vs_cublas(args, torch.device("cuda", 0))
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    import torch
    torch.cuda.set_device(local)
    device = torch.device("cuda", local)
    dist = None
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=device)
    import synth
    s = synth.CONFIGS[args.workload]
    pk, pk_kind = peaks()

    r = bench_workload(args, s, rank, world, device, dist)
    K = args.steps
    total_s = r["total_ms"] * 1e-3
    value = job_tokens_per_s(world, s.T, K, r["total_ms"])
    tflops = world * s.flops * K / total_s / 1e12

    prof, nb = r["prof"], r["breakdown_steps"]
    up_ms, up_n = r["prof_up"]["up_swiglu_gemm"]  # timed steps
    # the library's kernels per step (one per recorded stage launch) x timed steps
    launches = int(round(sum(n for _, n in prof.values()) / nb * K))
    rows = s.T * s.k
    # dominant kernel: the up-projection GEMM (2/3 of the flops; HBM-bound at decode)
    up_flops = 2.0 * rows * s.d * (2 * s.f)
    up_avg_s = up_ms / max(up_n, 1) * 1e-3
    if s.T * s.k >= 1024:
        tr = traffic_record("up_swiglu_gemm")
        roofline = {"kernel": "up_swiglu_gemm (tcgen05 grouped GEMM, SwiGLU epilogue)", "bound": "tensor",
                    "achieved": up_flops / up_avg_s / 1e12, "peak": pk["bf16_tflops"], "unit": "TFLOP/s",
                    "peak_kind": pk_kind + " bf16 (burst)",
                    "algorithmic_per_launch": up_flops, "avg_launch_ms": up_avg_s * 1e3,
                    "traffic": tr["bytes_per_launch"] if tr else None}
    else:
        up_bytes = 2.0 * s.E * s.f * s.d * 2 + rows * s.d * 2 + rows * s.f * 2
        tr = traffic_record("up_swiglu_gemm_decode")
        roofline = {"kernel": "up_swiglu_gemm (weight streaming)", "bound": "hbm",
                    "achieved": up_bytes / up_avg_s / 1e9, "peak": pk["hbm_gbs"], "unit": "GB/s",
                    "peak_kind": pk_kind, "algorithmic_per_launch": up_bytes, "avg_launch_ms": up_avg_s * 1e3,
                    "traffic": tr["bytes_per_launch"] if tr else None}
    regime = clock_regime(r["clocks"])
    if roofline["bound"] == "tensor" and "bf16_tflops_sustained" in pk:
        # A kernel timed inside a long run, where the power cap holds the clock
        # down, is held to the sustained cuBLAS figure; a short timed region at
        # full clock to the burst one.  The regime is read from the clocks
        # sampled during the timed steps; both fractions are reported.
        roofline["peak_burst"] = pk["bf16_tflops"]
        roofline["frac_of_burst"] = roofline["achieved"] / pk["bf16_tflops"]
        roofline["peak_sustained"] = pk["bf16_tflops_sustained"]
        roofline["frac_of_sustained"] = roofline["achieved"] / pk["bf16_tflops_sustained"]
        if regime == "sustained":
            roofline["peak"] = pk["bf16_tflops_sustained"]
            roofline["peak_kind"] = pk_kind + " bf16 (sustained)"
        clk = r["clocks"] or {}
        roofline["regime"] = "%s: median SM clock %s of max %s MHz during the timed steps" % (
            regime, clk.get("sm_mhz"), clk.get("sm_max_mhz"))
    roofline["frac"] = roofline["achieved"] / roofline["peak"]

    line = {"metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": K,
            "warmup": args.warmup, "ms_per_step": r["total_ms"] / K, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic: seeded counter-based N(0,1) tokens, N(0,1/fan_in) random-init Mixtral-8x7B expert "
                    "and router weights",
            "config": workload_desc(s, world),
            "tflops": tflops, "frac_of_bf16_peak": tflops / world / pk["bf16_tflops"], "peak_kind": pk_kind,
            "roofline": roofline, "gpu_launches": launches,
            "stages_ms_per_step": {k: round(v[0] / nb, 4) for k, v in prof.items() if v[1]},
            "stages_note": "per-stage times from a separate pass of %d steps with events around every kernel "
                           "(those events serialise the kernels; the timed steps record only the up GEMM's)" % nb,
            "device_error_flags": r["deverr"]}
    if r["clocks"]:
        line["clocks"] = r["clocks"]

    # every rank runs the host-buffer path on its own tokens; max over ranks
    if dist is not None:
        dist.barrier()
    e_ms, hb, db = e2e_leg(args, s, r["t"], device, max(10, min(K, 100)))
    e_ms = max_over_ranks(e_ms, dist, device)
    if rank == 0:
        line["e2e"] = {"value": world * s.T / (e_ms * 1e-3), "unit": "tokens/s", "h2d_bytes_per_step": hb,
                       "d2h_bytes_per_step": db, "ms_per_step": e_ms, "steps": max(10, min(K, 100)),
                       "chunks": args.e2e_chunks,
                       "path": "pinned host x -> moe_layer_forward_host (x_ready, y_async; each step's "
                               "copies pipelined with the compute of neighbouring pieces, %d per step) -> "
                               "pinned host y" % args.e2e_chunks}
    del r
    torch.cuda.empty_cache()

    if not args.no_extras and args.workload == "prefill":
        d = synth.CONFIGS["decode"]
        dargs = argparse.Namespace(**vars(args))
        dargs.steps = 200  # ~0.1 s of decode steps whatever K is: a stable mean
        # the timed decode steps carry no events inside (the layer as a caller
        # runs it); the GEMMs' rates come from the breakdown pass
        rd = bench_workload(dargs, d, rank, world, device, dist, extras_for_decode=True, record_up=False,
                            l2_flush=False)
        p, dnb = rd["prof"], rd["breakdown_steps"]
        counts = None
        wbytes = 3.0 * d.E * d.d * d.f * 2  # all 8 experts are touched at T=32 with near-uniform routing
        ups, upn = p["up_swiglu_gemm"]
        dns, dnn = p["down_combine_gemm"]
        # the direct calls and the captured graph, timed the same way, back to back
        dms = loop_step_ms(rd, d, device, dargs.steps)
        gms = graph_step_ms(rd, d, device, dargs.steps)
        fl = rd["flushed_step_ms"]
        line["decode"] = {"workload": workload_desc(d, world)["workload"], "ms_per_step": dms,
                          "timing": "one event pair around %d back-to-back calls (no event between layers)"
                                    % dargs.steps,
                          "ms_per_step_step_events": rd["total_ms"] / dargs.steps,
                          "ms_per_step_median": statistics.median(rd["step_ms"]),
                          "step_events_note": "the same calls with an event pair around every step (an event "
                                              "between two layers holds back the next one's early launch)",
                          "steps": dargs.steps,
                          "l2": "steps back to back: the 2.82 GB of expert weights exceed the 126 MB L2, and each "
                                "step streams all of them, so no step finds another's weights in L2",
                          "ms_per_step_l2_flushed": sum(fl) / len(fl),
                          "frac_of_hbm_l2_flushed": wbytes / (sum(fl) / len(fl) * 1e-3) / 1e9 / pk["hbm_gbs"],
                          "ms_per_step_cuda_graph": gms,
                          "cuda_graph_note": "one captured layer replayed back to back; no L2 flush (the 2.82 GB "
                                             "of weights exceed L2)",
                          "weight_GBps_cuda_graph": wbytes / (gms * 1e-3) / 1e9,
                          "frac_of_hbm_cuda_graph": wbytes / (gms * 1e-3) / 1e9 / pk["hbm_gbs"],
                          "tokens_per_s": world * d.T / (dms * 1e-3),
                          "weight_GBps": wbytes / (dms * 1e-3) / 1e9,
                          "frac_of_hbm": wbytes / (dms * 1e-3) / 1e9 / pk["hbm_gbs"],
                          "up_gemm_GBps": (2.0 * d.E * d.f * d.d * 2) / (ups / upn * 1e-3) / 1e9,
                          "down_gemm_GBps": (1.0 * d.E * d.f * d.d * 2) / (dns / dnn * 1e-3) / 1e9,
                          "gemm_rates_note": "from the breakdown pass (events around every kernel)",
                          "stages_ms_per_step": {k: round(v[0] / dnb, 4) for k, v in p.items() if v[1]},
                          "device_error_flags": rd["deverr"]}
        del rd, counts
        torch.cuda.empty_cache()
        sk = synth.CONFIGS["skewed"]
        sargs = argparse.Namespace(**vars(args))
        sargs.steps = max(10, min(60, K))
        rs = bench_workload(sargs, sk, rank, world, device, dist, extras_for_decode=True, record_up=False)
        sms = rs["total_ms"] / sargs.steps
        line["skewed"] = {"workload": workload_desc(sk, world)["workload"] + ", Zipf-shaped load (hottest expert 35%)",
                          "ms_per_step": sms, "tokens_per_s": world * sk.T / (sms * 1e-3),
                          "tflops": sk.flops / (sms * 1e-3) / 1e12,
                          "frac_of_bf16_peak": sk.flops / (sms * 1e-3) / 1e12 / pk["bf16_tflops"],
                          "stages_ms_per_step": {k: round(v[0] / rs["breakdown_steps"], 4)
                                                 for k, v in rs["prof"].items() if v[1]},
                          "device_error_flags": rs["deverr"]}
        del rs
        torch.cuda.empty_cache()
        if world == 1:
            line["stack"] = bench_stack(max(3, min(10, K)), device, pk)
            torch.cuda.empty_cache()

    if rank == 0 and world == 1 and not args.no_extras:
        import numpy as np
        from synth.device import device_inputs, to_host_bits
        t = make_inputs(s, 0, device)
        w64 = oracle_weights_f64(t, s.E)
        n = min(args.cpu_sample, s.T)
        rows_sel = np.sort(np.random.default_rng(0).choice(s.T, size=n, replace=False))
        x_bits = to_host_bits(t["x"])[rows_sel]
        del t
        dt, threads = time_oracle(w64, x_bits, s.k)
        line["cpu_baseline"] = {"value": n / dt, "unit": "tokens/s", "cores": threads, "kind": "oracle",
                                "sample": "%d random tokens of the %s workload (fp64 router, top-k, both experts "
                                          "and combine; weights pre-widened to fp64 outside the timing), %.1f s"
                                          % (n, s.name, dt)}
    if dist is not None:
        dist.barrier()
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(line), flush=True)
    return 0


if __name__ == "__main__":
    sys.exit(main())
