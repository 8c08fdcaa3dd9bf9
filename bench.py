#!/usr/bin/env python
"""Benchmark: causal linear-attention forward + backward tokens/s on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

One step is one training pass of the attention layer on the timed workload
(causal, B=8, H=16, N=8192, D=64, bf16, phi = elu+1): la_forward, which also
keeps the per-token denominators g and the final state (S, z), followed by
la_backward given o, g and (S, z), through the library's Python binding,
inputs resident in HBM.  The inputs (4 x 128 MiB) are larger than the 126 MB
L2, so consecutive steps cannot serve each other from cache.  W untimed
warm-up steps, then exactly K steps between two barrier + synchronize
points, timed with CUDA events on the launching stream; with several GPUs
each rank runs its own replica (there is no exchange step in this op) and
the max time over ranks is used.

The printed JSON line also carries:
  roofline      the dominant kernel: algorithmic bytes per launch (the
                method's byte budget of the pass when the kernel is that
                whole pass) over its measured launch time (CUDA events the
                library records on its launch stream during the timed steps)
                against the measured HBM copy bandwidth;
  rows          step, forward and backward fractions of the method's byte
                budget (forward 8 N D, backward 14 N D, step 22 N D bytes per
                head in bf16; the slower of bytes at HBM peak and flops at
                the bf16 MMA peak), the split timed with events between the
                two calls;
  kernels       per-kernel launch times and the fraction of each kernel's own
                reads and writes;
  graded        the other full-size workloads, each with its own clocks: the
                long-context causal forward (B1 H32 N131072 D128), 1024
                decode steps (B256 H32 D128, fp32 state in place), the same
                with grouped-query attention (8 key/value heads) and the
                1.4B-parameter LM layer shape forward + backward (B4 H16
                N4096 D128) with both feature maps, and the timed shape with
                a decay factor per head (decayed recurrence);
  e2e           the headline metric with every step's inputs copied from
                pinned host memory and its outputs (o, dq, dk, dv) read back
                inside the timed region, consecutive steps pipelined over two
                copy streams;
  cpu_baseline  the fp64 CPU oracle, as it stands, on a bounded sample;
  clocks        SM clocks and throttle reasons sampled during the timed steps.

``--impl reference`` times the CPU oracle on the same workload instead (this
op has no runnable upstream implementation; the oracle is the reference arm).
"""
from __future__ import annotations

import argparse
import dataclasses
import json
import math
import os
import statistics
import sys
import threading
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

from linear_attention_transformers_b200 import inputs  # noqa: E402

WORKLOAD = inputs.WORKLOADS["causal_fwdbwd_b8h16n8192d64_bf16"]
METRIC = "linear-attn fwd+bwd tokens/s per B200; % of roofline (HBM GB/s, TC util)"
UNIT = "tokens/s"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


# ----------------------------------------------------------------- helpers
def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return p, "measured"
    except Exception:
        return dict(FALLBACK_PEAKS), "fallback"


def method_bytes(w, part: str) -> float:
    """The method's minimum bytes for workload w (the per-head figures of the
    method's byte budget, times heads): forward reads q, k, v and writes o
    (4 tensors); backward reads q, k, v, dO and writes dq, dk, dv (7); the
    step is both (11 tensors; 22 N D bytes per head in bf16)."""
    e = 2 if w.dtype == torch.bfloat16 else 4
    t = w.B * w.H * w.N * w.D * e  # bytes of one [B,H,N,D] tensor
    return float({"forward": 4, "backward": 7, "step": 11}[part] * t)


def method_flops(w, part: str) -> float:
    """The method's multiply-add work: 4 N D^2 per head forward (state update
    and query), 10 N D^2 backward."""
    per = {"forward": 4, "backward": 10, "step": 14}[part]
    return float(per * w.B * w.H * w.N * w.D * w.D)


def own_bytes(kernel: str, w) -> float:
    """Bytes one launch of `kernel` must move for workload w by its own
    design (what it reads and writes), for the per-kernel fractions."""
    e = 2 if w.dtype == torch.bfloat16 else 4
    t = w.B * w.H * w.N * w.D * e
    n = w.B * w.H * w.N * 4  # one float32 per token (g or dg)
    table = {
        "fwd_generic": 4 * t,           # q, k, v -> o
        "bwd_generic": 7 * t,           # q, k, v, dO -> dq, dk, dv
        "chunk_causal": 4 * t + n,      # q, k, v -> o, g (+2t with phi(q), phi(k) stored)
        "bwd_dq": 6 * t + 2 * n,        # phi(q), phi(k), v, dO, o, g -> dq, dg
        "bwd_dkdv": 6 * t + 2 * n,      # phi(q), phi(k), v, dO, g, dg -> dk, dv
        "phi_map": 4 * t,               # q, k -> phi(q), phi(k)
    }
    return float(table.get(kernel, 0.0))


def roofline_of(bytes_, flops, seconds, peaks, sustained=True):
    """Roofline fraction of a timed region: the slower of bytes at the
    measured HBM bandwidth and flops at the measured bf16 MMA rate."""
    hbm = peaks["hbm_gbs"] * 1e9
    tc = peaks["bf16_tflops_sustained" if sustained else "bf16_tflops"] * 1e12
    t_roof = max(bytes_ / hbm, flops / tc)
    return {"bound": "hbm" if bytes_ / hbm >= flops / tc else "tensor",
            "achieved_gbs": bytes_ / seconds / 1e9, "frac": t_roof / seconds,
            "algorithmic_bytes": bytes_, "flops": flops}


# DRAM traffic per launch from one ncu capture (dram__bytes_read.sum +
# dram__bytes_write.sum), per token and head so that it scales to the bench
# workload; valid only while the sources the kernel is built and launched
# from (`files`, under csrc/) hash to `sources`.  Captures run at a smaller
# N (the profiling size rule); these kernels move each token's tiles once,
# so traffic grows in proportion to tokens.
_FWD64_SOURCES = ["la_chunk_fwd64.cuh", "la_chunk_fwd.cuh", "la_tile_ops.cuh", "la_sm100.cuh",
                  "la_common.cuh"]
_BWD64_SOURCES = ["la_chunk_bwd64.cuh", "la_chunk_bwd.cuh", "la_tile_ops.cuh", "la_sm100.cuh",
                  "la_common.cuh"]
MEASURED_TRAFFIC = {
    # one ncu launch each (the fourth of each kernel; DRAM byte counters) at
    # B8 H16 N4096 D64, the timed workload at half its tokens
    "chunk_causal": {"D": 64, "bytes_per_token_head": (201.394944e6 + 155.971072e6) / (8 * 16 * 4096),
                     "files": _FWD64_SOURCES,
                     "sources": "8bcebbcf1ed37f1201997187a0234b234545cea7b36d51bc13516deaf81a4591"},
    "bwd_dq": {"D": 64, "bytes_per_token_head": (337.735168e6 + 49.178368e6) / (8 * 16 * 4096),
               "files": _BWD64_SOURCES,
               "sources": "cf3a81aef51868101c532774411a259712c05b9e423fc79c5ecc8ecef1c6d207"},
    "bwd_dkdv": {"D": 64, "bytes_per_token_head": (272.699392e6 + 96.399872e6) / (8 * 16 * 4096),
                 "files": _BWD64_SOURCES,
                 "sources": "cf3a81aef51868101c532774411a259712c05b9e423fc79c5ecc8ecef1c6d207"},
}


def kernel_sources_hash(files) -> str:
    """sha256 over the named CUDA sources of the library (names and bytes)."""
    import hashlib
    d = os.path.join(ROOT, "linear_attention_transformers_b200", "csrc")
    h = hashlib.sha256()
    for name in sorted(files):
        h.update(name.encode())
        with open(os.path.join(d, name), "rb") as f:
            h.update(f.read())
    return h.hexdigest()


def measured_traffic(kernel: str, w):
    """Per-launch DRAM bytes of `kernel` on workload w, or None when no
    capture exists for it (at w's head size) or its sources changed since."""
    rec = MEASURED_TRAFFIC.get(kernel)
    if rec is None or rec["D"] != w.D or rec["sources"] != kernel_sources_hash(rec["files"]):
        return None
    return rec["bytes_per_token_head"] * w.B * w.H * w.N


class ClockSampler:
    """Samples SM clock and throttle reasons through NVML on a thread."""

    REASONS = {
        "hw_slowdown": 0x8, "hw_thermal_slowdown": 0x40, "sw_thermal_slowdown": 0x20,
        "sw_power_cap": 0x4, "hw_power_brake_slowdown": 0x80, "sync_boost": 0x10,
    }

    def __init__(self, index: int, period_s: float = 0.005):
        self.samples, self.reasons = [], set()
        self.period = period_s
        self.ok = False
        self.max_mhz = None
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByIndex(index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception:
            self.ok = False
        self._stop = threading.Event()
        self._t = None

    def _run(self):
        while not self._stop.is_set():
            try:
                self.samples.append(self.nv.nvmlDeviceGetClockInfo(self.h, self.nv.NVML_CLOCK_SM))
                mask = self.nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
                for name, bit in self.REASONS.items():
                    if mask & bit:
                        self.reasons.add(name)
            except Exception:
                pass
            time.sleep(self.period)

    def __enter__(self):
        if self.ok:
            self._t = threading.Thread(target=self._run, daemon=True)
            self._t.start()
        return self

    def __exit__(self, *exc):
        if self._t:
            self._stop.set()
            self._t.join()

    def summary(self):
        if not self.ok or not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": sorted(self.reasons),
                    "samples": len(self.samples)}
        return {"sm_mhz": statistics.median(self.samples), "sm_max_mhz": self.max_mhz,
                "reasons": sorted(self.reasons), "samples": len(self.samples)}


def dist_setup():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        backend = "nccl" if torch.cuda.is_available() else "gloo"
        if torch.cuda.is_available():
            torch.cuda.set_device(local)
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=300))
    elif torch.cuda.is_available():
        torch.cuda.set_device(local)
    return world, rank, local


def max_over_ranks(x: float, world: int) -> float:
    if world == 1:
        return x
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier(world: int):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


# ---------------------------------------------------------------- CPU oracle
def oracle_sample(w, heads: int, tokens: int, threads: int):
    """Time the oracle's forward+backward on `heads` heads x `tokens` tokens
    of workload w (a bounded sample: the first heads, the first tokens)."""
    import oracle
    q, k, v, dO = inputs.make_tensors(1, heads, tokens, w.D, w.dtype, w.seed + 7,
                                      with_grad_out=True)
    oracle.build()
    oracle.set_threads(threads)
    t0 = time.perf_counter()
    oracle.forward(q, k, v, w.causal, w.phi)
    oracle.backward(q, k, v, dO, w.causal, w.phi)
    dt = time.perf_counter() - t0
    # one workload token covers H heads
    return (heads * tokens / w.H) / dt, dt


def cpu_cores() -> int:
    try:
        return len(os.sched_getaffinity(0))
    except Exception:
        return os.cpu_count() or 1


def cpu_baseline(w, target_s: float = 15.0):
    cores = cpu_cores()
    # calibrate on a short prefix, then take whole heads (full N) until the
    # sample is about target_s of work
    _, dt = oracle_sample(w, cores, 256, cores)
    t_head = dt / 256 * w.N  # seconds for one full head on one core
    heads = int(min(w.B * w.H, max(1, round(target_s * cores / max(t_head, 1e-9)))))
    heads = max(1, (heads // cores) * cores) if heads >= cores else heads
    value, dt = oracle_sample(w, heads, w.N, cores)
    return {"value": value, "unit": UNIT, "cores": min(cores, heads), "kind": "oracle",
            "sample": f"fp64 oracle forward+backward on {heads} of {w.B * w.H} heads x all "
                      f"{w.N} tokens (same shape and distribution, OpenMP over heads), "
                      f"{dt:.1f} s; tokens/s = heads*N/H / time"}


def run_reference(args, world, rank):
    if rank != 0:
        return 0
    w = WORKLOAD
    cores = cpu_cores()
    # each step: the oracle on `cores` heads x `tokens` tokens, sized so the
    # whole (warmup + steps) run stays near two minutes
    budget = 120.0 / max(1, args.steps + args.warmup)
    _, dt = oracle_sample(w, cores, 256, cores)
    tokens = int(max(64, min(w.N, budget / max(dt / 256, 1e-9))))
    for _ in range(args.warmup):
        oracle_sample(w, cores, tokens, cores)
    total = 0.0
    for _ in range(args.steps):
        _, dt = oracle_sample(w, cores, tokens, cores)
        total += dt
    value = (args.steps * cores * tokens / w.H) / total
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT,
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1e3 * total / args.steps, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": config_dict(w, args.gpus),
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle",
                         "sample": f"each step: fp64 oracle forward+backward on {cores} heads x "
                                   f"first {tokens} tokens (one thread per head)"},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def workload_from_args(args):
    """The timed workload, or a reshaped copy of it (--shape B,H,N,D) for
    small profiling runs."""
    if not args.shape:
        return WORKLOAD
    B, H, N, D = (int(x) for x in args.shape.split(","))
    return dataclasses.replace(WORKLOAD, name=f"causal_fwdbwd_b{B}h{H}n{N}d{D}_bf16", B=B, H=H,
                               N=N, D=D)


def config_dict(w, gpus):
    return {"workload": w.name, "B": w.B, "H": w.H, "N": w.N, "D": w.D,
            "causal": w.causal, "phi": "elu1" if w.phi == 0 else "relu_eps",
            "global_batch": w.B * gpus, "seq_len": w.N, "parallelism": f"replicas{gpus}",
            "l2": "inputs larger than L2 (4 x 128 MiB per step)"}


# --------------------------------------------------------------------- ours
def timed_region(fn, steps, stream, dev, world, sampler_index):
    """Run fn() `steps` times between barrier + synchronize points, timed
    with CUDA events on `stream`; returns (max-over-ranks ms, clocks)."""
    sampler = ClockSampler(sampler_index)
    barrier(world)
    torch.cuda.synchronize(dev)
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with sampler:
        ev0.record(stream)
        for _ in range(steps):
            fn()
        ev1.record(stream)
        torch.cuda.synchronize(dev)
    barrier(world)
    return max_over_ranks(ev0.elapsed_time(ev1), world), sampler.summary()


class TrainStep:
    """One forward + backward of workload w through the library's binding,
    with every output and workspace preallocated: la_forward keeps o, the
    denominators g and the final state (S, z) (and the feature maps where the
    backward reads them); la_backward takes them."""

    def __init__(self, api, w, dev, stream, tensors=None):
        self.api, self.w, self.stream = api, w, stream
        q, k, v, dO = tensors if tensors is not None else inputs.make_inputs(
            w, device=dev, with_grad_out=True)
        self.q, self.k, self.v, self.dO = q, k, v, dO
        B, H, N, D = q.shape
        self.o = torch.empty_like(q)
        self.g = torch.empty((B, H, N), dtype=torch.float32, device=dev)
        self.S = torch.empty((B, H, D, D), dtype=torch.float32, device=dev)
        self.z = torch.empty((B, H, D), dtype=torch.float32, device=dev)
        self.pq = self.pk = None
        if api.backward_reads_phi(q.dtype, D):
            self.pq, self.pk = torch.empty_like(q), torch.empty_like(q)
        self.dq, self.dk, self.dv = torch.empty_like(q), torch.empty_like(q), torch.empty_like(q)
        ws_f = api.la_workspace_size(api.LA_OP_FORWARD, B, H, N, D, w.causal, w.dtype)
        ws_b = api.la_workspace_size(api.LA_OP_BACKWARD, B, H, N, D, w.causal, w.dtype)
        self.ws = torch.empty(max(ws_f, ws_b, 256), dtype=torch.uint8, device=dev)

    def forward(self, q=None, k=None, v=None, o=None):
        a, w = self.api, self.w
        a.la_forward(q if q is not None else self.q, k if k is not None else self.k,
                     v if v is not None else self.v, w.causal, w.phi,
                     o=o if o is not None else self.o, workspace=self.ws, stream=self.stream,
                     g=self.g, phi_out=None if self.pq is None else (self.pq, self.pk),
                     state_out=(self.S, self.z))

    def backward(self, q=None, k=None, v=None, dO=None, o=None, grads=None):
        a, w = self.api, self.w
        dq, dk, dv = grads if grads is not None else (self.dq, self.dk, self.dv)
        a.la_backward(q if q is not None else self.q, k if k is not None else self.k,
                      v if v is not None else self.v, dO if dO is not None else self.dO,
                      w.causal, w.phi, dq=dq, dk=dk, dv=dv, workspace=self.ws,
                      stream=self.stream, o=o if o is not None else self.o, g=self.g,
                      phi_q=self.pq, phi_k=self.pk)

    def __call__(self):
        self.forward()
        self.backward()


class DecayTrainStep(TrainStep):
    """TrainStep of the decayed recurrence (one factor per head): the forward
    keeps o and g, the backward takes them."""

    def __init__(self, api, w, dev, stream, gamma):
        super().__init__(api, w, dev, stream)
        self.gamma = gamma
        B, H, N, D = self.q.shape
        need = max(api.la_workspace_size_decay(op, B, H, N, D, w.dtype)
                   for op in (api.LA_OP_FORWARD, api.LA_OP_BACKWARD))
        if need > self.ws.numel():
            self.ws = torch.empty(need, dtype=torch.uint8, device=dev)

    def forward(self, q=None, k=None, v=None, o=None):
        self.api.la_forward_decay(self.q, self.k, self.v, self.gamma, self.w.phi, o=self.o,
                                  workspace=self.ws, stream=self.stream, g=self.g)

    def backward(self, q=None, k=None, v=None, dO=None, o=None, grads=None):
        self.api.la_backward_decay(self.q, self.k, self.v, self.dO, self.gamma, self.w.phi,
                                   dq=self.dq, dk=self.dk, dv=self.dv, workspace=self.ws,
                                   stream=self.stream, o=self.o, g=self.g)


def split_times(step, steps, stream):
    """Forward and backward milliseconds per step, from CUDA events recorded
    between the two calls on the launching stream (a separate, untimed-by-
    the-headline pass over the same steps)."""
    evs = [torch.cuda.Event(enable_timing=True) for _ in range(3 * steps)]
    for i in range(steps):
        evs[3 * i].record(stream)
        step.forward()
        evs[3 * i + 1].record(stream)
        step.backward()
        evs[3 * i + 2].record(stream)
    torch.cuda.synchronize()
    f = sum(evs[3 * i].elapsed_time(evs[3 * i + 1]) for i in range(steps)) / steps
    b = sum(evs[3 * i + 1].elapsed_time(evs[3 * i + 2]) for i in range(steps)) / steps
    return f, b


def graded_train(api, w, dev, stream, world, peaks, steps=20, warmup=5, gamma=None):
    """A forward + backward workload at its full size: ms per step, tokens/s
    and the roofline fractions of the step, the forward and the backward.
    gamma: per-head decay factors (the decayed recurrence)."""
    step = TrainStep(api, w, dev, stream) if gamma is None else \
        DecayTrainStep(api, w, dev, stream, gamma)
    for _ in range(warmup):
        step()
    torch.cuda.synchronize(dev)
    api.la_get_device_error(stream)
    ms, clocks = timed_region(step, steps, stream, dev, world, dev.index or 0)
    f_ms, b_ms = split_times(step, max(3, steps // 2), stream)
    api.la_get_device_error(stream)
    out = {"workload": w.name, "ms_per_step": ms / steps,
           "tokens_per_s": world * w.B * w.N * steps / (ms / 1e3),
           "step": roofline_of(method_bytes(w, "step"), method_flops(w, "step"),
                               ms / steps / 1e3, peaks),
           "forward": dict(ms=f_ms, **roofline_of(method_bytes(w, "forward"),
                                                  method_flops(w, "forward"), f_ms / 1e3, peaks)),
           "backward": dict(ms=b_ms, **roofline_of(method_bytes(w, "backward"),
                                                   method_flops(w, "backward"), b_ms / 1e3,
                                                   peaks)),
           "clocks": clocks}
    del step
    torch.cuda.empty_cache()
    return out


def graded_forward(api, w, dev, stream, world, peaks, steps=10, warmup=3):
    """The causal forward alone at full size (the long-context workload)."""
    q, k, v = inputs.make_inputs(w, device=dev, with_grad_out=False)
    o = torch.empty_like(q)
    B, H, N, D = q.shape
    ws = torch.empty(max(256, api.la_workspace_size(api.LA_OP_FORWARD, B, H, N, D, w.causal,
                                                    w.dtype)), dtype=torch.uint8, device=dev)

    def fwd():
        api.la_forward(q, k, v, w.causal, w.phi, o=o, workspace=ws, stream=stream)

    for _ in range(warmup):
        fwd()
    torch.cuda.synchronize(dev)
    api.la_get_device_error(stream)
    ms, clocks = timed_region(fwd, steps, stream, dev, world, dev.index or 0)
    api.la_get_device_error(stream)
    out = {"workload": w.name, "ms_per_call": ms / steps,
           "tokens_per_s": world * w.B * w.N * steps / (ms / 1e3),
           "forward": roofline_of(method_bytes(w, "forward"), method_flops(w, "forward"),
                                  ms / steps / 1e3, peaks),
           "clocks": clocks}
    del q, k, v, o, ws
    torch.cuda.empty_cache()
    return out


def graded_decode(api, dev, stream, world, peaks, reps=3, warmup=2, grouped=False):
    """`steps` recurrent decode steps at batch B (fp32 state in place), each
    step one la_decode_step over every (b, h); timed over whole runs of all
    steps.  grouped: Hkv key/value heads, each state shared by H/Hkv query
    heads."""
    cfg = inputs.DECODE_GQA if grouped else inputs.DECODE
    B, H, D, steps = cfg["B"], cfg["H"], cfg["D"], cfg["steps"]
    Hkv = cfg.get("Hkv", H)
    if grouped:
        q, k, v = inputs.make_decode_gqa_inputs(B, H, Hkv, D, steps, cfg["seed"], device=dev)
    else:
        q, k, v = inputs.make_decode_inputs(B, H, D, steps, cfg["seed"], device=dev)
    S = torch.zeros(B, Hkv, D, D, device=dev)
    z = torch.zeros(B, Hkv, D, device=dev)
    outs = torch.empty(steps, B, H, D, dtype=q.dtype, device=dev)

    def run():
        for t in range(steps):
            api.la_decode_step(S, z, q[t], k[t], v[t], o=outs[t], stream=stream)

    for _ in range(warmup):
        run()
    torch.cuda.synchronize(dev)
    api.la_get_device_error(stream)
    ms, clocks = timed_region(run, reps, stream, dev, world, dev.index or 0)
    api.la_get_device_error(stream)
    s_step = ms / reps / steps / 1e3
    # per key/value head and step: S and z read and written in float32, k, v
    # read in bf16; per query head q read and o written in bf16
    bytes_step = B * Hkv * (2 * 4 * (D * D + D) + 2 * D * 2) + B * H * 2 * D * 2
    flops_step = B * Hkv * 2 * D * D + B * H * 2 * D * D
    name = f"decode_b{B}h{H}" + (f"kv{Hkv}" if grouped else "") + f"d{D}_x{steps}_bf16"
    out = {"workload": name, "us_per_step": s_step * 1e6,
           "steps_per_s": world / s_step, "tokens_per_s": world * B / s_step,
           "step": roofline_of(bytes_step, flops_step, s_step, peaks), "clocks": clocks}
    del q, k, v, S, z, outs
    torch.cuda.empty_cache()
    return out


def run_ours(args, world, rank, local):
    from linear_attention_transformers_b200 import api
    w = workload_from_args(args)
    dev = torch.device("cuda", local)
    api.load_library()
    stream = torch.cuda.current_stream(dev)
    peaks, peaks_src = load_peaks()
    step = TrainStep(api, w, dev, stream)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize(dev)
    api.la_get_device_error(stream)

    # ---- timed region (the headline)
    api.la_profile_enable(True)
    api.la_profile_collect()
    launches0 = api.la_launch_count()
    ms_max, clocks = timed_region(step, args.steps, stream, dev, world,
                                  dev.index if dev.index is not None else 0)
    launches = api.la_launch_count() - launches0
    prof = api.la_profile_collect()
    api.la_profile_enable(False)
    api.la_get_device_error(stream)
    tokens_per_step = w.B * w.N
    value = world * tokens_per_step * args.steps / (ms_max / 1e3)
    s_step = ms_max / args.steps / 1e3

    # ---- forward / backward split (events between the calls, own pass)
    f_ms, b_ms = split_times(step, min(args.steps, 20), stream)
    rows = {
        "step": roofline_of(method_bytes(w, "step"), method_flops(w, "step"), s_step, peaks),
        "forward": dict(ms=f_ms, **roofline_of(method_bytes(w, "forward"),
                                               method_flops(w, "forward"), f_ms / 1e3, peaks)),
        "backward": dict(ms=b_ms, **roofline_of(method_bytes(w, "backward"),
                                                method_flops(w, "backward"), b_ms / 1e3, peaks)),
    }

    # ---- dominant kernel: the library's own per-launch CUDA events (recorded
    # on its launch stream during the timed steps).  Its algorithmic bytes
    # are the method's byte budget of the pass it belongs to (forward: 4
    # tensors, backward: 7), charged against the summed launch time per step
    # of that pass's kernels; each kernel's own reads and writes are reported
    # apart (kernels.*.own_frac).
    kernels = {}
    for name, (n, tot) in prof.items():
        avg_s = tot / n / 1e3
        ob = own_bytes(name, w)
        kernels[name] = {"launches": n, "total_ms": tot, "share": tot / max(ms_max, 1e-9),
                         "avg_ms": avg_s * 1e3, "own_bytes": ob,
                         "own_frac": (ob / avg_s / 1e9) / peaks["hbm_gbs"] if ob else None}
    roofline = None
    if prof:
        name, (n, tot) = max(prof.items(), key=lambda kv: kv[1][1])
        avg_s = tot / n / 1e3
        backward_kernels = ("bwd_dq", "bwd_dkdv", "bwd_generic")
        part = "backward" if name in backward_kernels else "forward"
        members = [k for k in prof if (k in backward_kernels) == (part == "backward")]
        pass_s = sum(prof[k][1] for k in members) / args.steps / 1e3
        alg = method_bytes(w, part)
        achieved = alg / pass_s / 1e9
        roofline = {"kernel": name, "pass": part, "pass_kernels": members, "bound": "hbm",
                    "achieved": achieved, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                    "frac": achieved / peaks["hbm_gbs"], "traffic": measured_traffic(name, w),
                    "algorithmic_bytes_per_launch": alg,
                    "algorithmic_bytes_basis": (f"method {part}: {7 if part == 'backward' else 4}"
                                                " tensors of B*H*N*D bf16 per step"),
                    "pass_ms_per_step": pass_s * 1e3, "avg_launch_ms": avg_s * 1e3,
                    "peak_source": f"{peaks_src} hbm_gbs (of {peaks_src})",
                    "share_of_step": tot / max(ms_max, 1e-9)}

    # ---- end to end: pinned host inputs in, outputs back, every step.  Steps
    # are pipelined the way a streaming caller runs them: step t's inputs go
    # up on one copy stream while step t-1 computes and step t-2's outputs
    # come down on another (PCIe is full duplex), with two device buffer sets
    # ordered by events.
    e2e = None
    if not args.no_e2e:
        q, k, v, dO = step.q, step.k, step.v, step.dO
        hin = [t.cpu().pin_memory() for t in (q, k, v, dO)]
        hout = [[torch.empty(q.shape, dtype=q.dtype, pin_memory=True) for _ in range(4)]
                for _ in range(2)]
        xin = [[q, k, v, dO], [torch.empty_like(t) for t in (q, k, v, dO)]]
        yout = [[step.o, step.dq, step.dk, step.dv], [torch.empty_like(q) for _ in range(4)]]
        s_in, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
        in_ready = [torch.cuda.Event() for _ in range(2)]
        cmp_done = [torch.cuda.Event() for _ in range(2)]
        out_done = [torch.cuda.Event() for _ in range(2)]
        e2e_steps = max(3, min(args.steps, 10))

        def e2e_step(t):
            b = t % 2
            xq, xk, xv, xdO = xin[b]
            yo, ydq, ydk, ydv = yout[b]
            with torch.cuda.stream(s_in):
                if t >= 2:
                    s_in.wait_event(cmp_done[b])  # step t-2 no longer reads xin[b]
                for dst, src in zip(xin[b], hin):
                    dst.copy_(src, non_blocking=True)
                in_ready[b].record(s_in)
            stream.wait_event(in_ready[b])
            if t >= 2:
                stream.wait_event(out_done[b])  # step t-2's outputs are on the host
            step.forward(xq, xk, xv, o=yo)
            step.backward(xq, xk, xv, xdO, o=yo, grads=(ydq, ydk, ydv))
            cmp_done[b].record(stream)
            with torch.cuda.stream(s_out):
                s_out.wait_event(cmp_done[b])
                for dst, src in zip(hout[b], yout[b]):
                    dst.copy_(src, non_blocking=True)
                out_done[b].record(s_out)

        for t in range(2):
            e2e_step(t)
        torch.cuda.synchronize(dev)
        barrier(world)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(s_in)
        for t in range(e2e_steps):
            e2e_step(t)
        # the last step's outputs are the last work; s_out has waited on all of it
        e1.record(s_out)
        torch.cuda.synchronize(dev)
        barrier(world)
        ems = max_over_ranks(e0.elapsed_time(e1), world)
        nbytes = q.numel() * q.element_size()
        e2e = {"value": world * tokens_per_step * e2e_steps / (ems / 1e3), "unit": UNIT,
               "h2d_bytes_per_step": 4 * nbytes, "d2h_bytes_per_step": 4 * nbytes,
               "steps": e2e_steps, "pipelined": "h2d, compute and d2h of consecutive steps overlap"}
        api.la_get_device_error(stream)
        del hin, hout, xin, yout
    del step
    torch.cuda.empty_cache()

    # ---- the other graded workloads, each at full size with its own clocks
    graded = None
    if not args.no_graded and not args.shape:
        graded = {
            "long_causal_fwd": graded_forward(api, inputs.WORKLOADS[
                "causal_fwd_b1h32n131072d128_bf16"], dev, stream, world, peaks),
            "decode": graded_decode(api, dev, stream, world, peaks),
            "decode_gqa": graded_decode(api, dev, stream, world, peaks, grouped=True),
            "lm_layer_relu": graded_train(api, inputs.WORKLOADS[
                "causal_fwdbwd_b4h16n4096d128_relu_bf16"], dev, stream, world, peaks),
            "lm_layer_elu": graded_train(api, inputs.WORKLOADS[
                "causal_fwdbwd_b4h16n4096d128_elu_bf16"], dev, stream, world, peaks),
            "decay_train": graded_train(api, inputs.DECAY_TRAIN, dev, stream, world, peaks,
                                        gamma=inputs.decay_factors(inputs.DECAY_TRAIN.H)),
        }

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(w)

    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_max / args.steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "bf16", "data": "synthetic",
            "config": config_dict(w, world),
            "roofline": roofline,
            "step_roofline": rows["step"],
            "rows": rows,
            "kernels": kernels,
            "gpu_launches": int(launches),
            "e2e": e2e,
            "cpu_baseline": cpu,
            "clocks": clocks,
            "graded": graded,
        }
        print(json.dumps(line), flush=True)
    return 0


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-graded", action="store_true",
                    help="skip the other full-size workloads (long forward, decode, LM layer)")
    ap.add_argument("--shape", default="", help="B,H,N,D override (profiling runs only)")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        ap.error("--warmup must be at least 3")
    world, rank, local = dist_setup()
    try:
        if args.impl == "reference":
            return run_reference(args, world, rank)
        return run_ours(args, world, rank, local)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    sys.exit(main())
