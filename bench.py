#!/usr/bin/env python
"""Benchmark of the Step-3.5-Flash routed-expert MoE layer on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl native|reference]

One step = one full forward of the layer (routing, dispatch, both grouped expert GEMMs,
combine) over one batch of synthetic tokens with all inputs resident in HBM.  The L2 is
flushed before every timed step, outside the timed events: a 2x-L2 write, then a 2x-L2 read,
so that the write-back of the flush's own dirty lines also happens outside the events (it
would otherwise land in the step: 15 us of a 226 us decode step).  Each step is
timed with CUDA events on the launching stream; the sum over K steps, max over ranks,
gives ``value`` = tokens of all ranks / time.  ``e2e`` repeats the measurement through the
public API with the step's tokens copied from pinned host memory and the output read
back inside the timed region.  Under torchrun each rank runs an independent replica on its
own tokens (the layer shards by tokens; no collective on the data path): weak scaling.

``--impl reference`` times the CPU oracle (plain C, OpenMP) on the host cores instead.
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

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from sparse_mixture_experts_ffn_b200 import inputs  # noqa: E402

METRIC = "MoE-layer tokens/s at T=4…16384; % of HBM or bf16 tensor-core roofline"
UNIT = "tokens/s"
DEFAULT_WORKLOAD = "decode_t4"
DEFAULT_STEPS = {"decode_t4": 2000, "decode_t128": 500, "prefill_t4096": 200,
                 "prefill_t16384_skew": 60, "tiny_f32_t64": 2000}


def log(*a):
    print(*a, file=sys.stderr, flush=True)


# ------------------------------------------------------------------------------------------
# clocks during the timed region
# ------------------------------------------------------------------------------------------
class ClockSampler:
    """SM clock, power and clock-event reasons of one GPU, read through NVML (read-only
    queries) every ``period_s`` in a background thread while the ``with`` block runs.
    Falls back to ``nvidia-smi -lms`` if NVML cannot be loaded."""
    REASONS = {  # NVML clock-event reason bits that the run record names
        0x4: "sw_power_cap", 0x8: "hw_slowdown", 0x20: "sw_thermal_slowdown", 0x40: "hw_thermal_slowdown",
        0x80: "hw_power_brake_slowdown",
    }
    FIELDS = ("clocks.sm", "clocks.max.sm", "power.draw", "clocks_event_reasons.active",
              "clocks_event_reasons.hw_slowdown", "clocks_event_reasons.hw_thermal_slowdown",
              "clocks_event_reasons.sw_thermal_slowdown", "clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index: int, period_s: float = 0.005):
        self.dev = device_index
        self.period = period_s
        self.samples = []  # (sm_mhz, sm_max_mhz, reason names)
        self.proc = None
        self._stop = threading.Event()
        self._t = None
        self.source = None

    def _uuid(self):
        uuid = str(torch.cuda.get_device_properties(self.dev).uuid)
        return uuid if uuid.startswith("GPU-") else f"GPU-{uuid}"

    def __enter__(self):
        try:
            import pynvml
            pynvml.nvmlInit()
            h = pynvml.nvmlDeviceGetHandleByUUID(self._uuid())
            smax = pynvml.nvmlDeviceGetMaxClockInfo(h, pynvml.NVML_CLOCK_SM)

            def poll():
                while not self._stop.is_set():
                    try:
                        sm = pynvml.nvmlDeviceGetClockInfo(h, pynvml.NVML_CLOCK_SM)
                        bits = pynvml.nvmlDeviceGetCurrentClocksEventReasons(h)
                        self.samples.append((float(sm), float(smax),
                                             [n for b, n in self.REASONS.items() if bits & b]))
                    except Exception:  # pragma: no cover - a failed query is skipped
                        pass
                    self._stop.wait(self.period)
            self.source = f"nvml every {self.period * 1e3:.0f} ms"
            self._t = threading.Thread(target=poll, daemon=True)
            self._t.start()
            return self
        except Exception as e:  # pragma: no cover - no NVML on this host
            log("NVML unavailable, falling back to nvidia-smi:", e)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", self._uuid(), "--query-gpu=" + ",".join(self.FIELDS),
                 "--format=csv,noheader,nounits", "-lms", "10"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.source = "nvidia-smi -lms 10"
            self._t = threading.Thread(target=self._read_smi, daemon=True)
            self._t.start()
        except Exception as e:  # pragma: no cover - no nvidia-smi
            log("clock sampler unavailable:", e)
            self.proc = None
        return self

    def _read_smi(self):
        names = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")
        for line in self.proc.stdout:
            parts = [q.strip() for q in line.strip().split(",")]
            if len(parts) != len(self.FIELDS):
                continue
            try:
                self.samples.append((float(parts[0]), float(parts[1]),
                                     [n for n, v in zip(names, parts[4:]) if v.lower() == "active"]))
            except ValueError:
                continue

    def __exit__(self, *exc):
        self._stop.set()
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()
        if self._t is not None:
            self._t.join(timeout=2)

    def summary(self, since: int = 0):
        """Median SM clock, the max clock and every reason seen, over samples[since:]."""
        rows = self.samples[since:]
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0, "source": self.source}
        return {"sm_mhz": statistics.median(r[0] for r in rows), "sm_max_mhz": max(r[1] for r in rows),
                "reasons": sorted({n for r in rows for n in r[2]}), "samples": len(rows), "source": self.source}


# ------------------------------------------------------------------------------------------
# algorithmic bytes / flops
# ------------------------------------------------------------------------------------------
def algorithmic(cfg, counts: np.ndarray, fp8: bool = False):
    """Bytes and FLOPs of the layer and of its gate/up GEMM for one step (no padding).
    fp8: expert weights as E4M3 codes (1 byte) plus one scale byte per 128 x 128 block."""
    es = 2 if cfg.dtype == "bf16" else 4
    H, I, Is, E, T, k = cfg.H, cfg.I, cfg.I_shared, cfg.E, cfg.T, cfg.top_k
    touched = int((counts > 0).sum())
    P = T * k

    def wb(n):  # bytes of n expert weights
        return n + n // (128 * 128) if fp8 else n * es
    layer_bytes = wb(touched * 3 * H * I + 3 * H * Is) + (E * H + 2 * T * H) * es
    layer_flops = 2 * T * E * H + P * 6 * H * I + T * 6 * H * Is
    gu_bytes = wb(touched * 2 * I * H + 2 * Is * H) + (P * H + T * H + P * I + T * Is) * es
    gu_flops = P * 4 * H * I + T * 4 * H * Is
    dn_bytes = wb(touched * H * I + H * Is) + (P * I + T * Is + P * H + T * H) * es
    dn_flops = P * 2 * H * I + T * 2 * H * Is
    return dict(touched=touched, layer_bytes=layer_bytes, layer_flops=layer_flops,
                gate_up_bytes=gu_bytes, gate_up_flops=gu_flops, down_bytes=dn_bytes, down_flops=dn_flops)


def measured_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return dict(hbm_gbs=float(d["hbm_gbs"]), bf16_tflops=float(d["bf16_tflops"]),
                    bf16_tflops_sustained=float(d.get("bf16_tflops_sustained", d["bf16_tflops"])),
                    source="measured")
    except Exception:
        return dict(hbm_gbs=6650.0, bf16_tflops=1590.0, bf16_tflops_sustained=1400.0, source="fallback")


def code_digest(src: bytes) -> str:
    """sha256[:16] of a C/C++/CUDA source with its comments removed and every run of
    whitespace folded to one space: edits to comments or layout keep the digest, any change
    to the code (a token added, removed or altered) moves it.  String and character literals
    are kept as written, so a `//` inside one is not taken for a comment."""
    import hashlib
    t = src.decode("utf-8", "replace")
    out, i, n = [], 0, len(t)
    while i < n:
        c = t[i]
        if c in "\"'":
            j = i + 1
            while j < n and t[j] != c:
                j += 2 if t[j] == "\\" else 1
            out.append(t[i:j + 1])
            i = j + 1
        elif t.startswith("//", i):
            j = t.find("\n", i)
            i = n if j < 0 else j
        elif t.startswith("/*", i):
            j = t.find("*/", i + 2)
            out.append(" ")
            i = n if j < 0 else j + 2
        else:
            out.append(c)
            i += 1
    return hashlib.sha256(" ".join("".join(out).split()).encode()).hexdigest()[:16]


def ncu_traffic(kernel: str, workload: str, algorithmic_bytes: float):
    """DRAM bytes per launch of `kernel` on `workload`, from a committed ncu summary under
    profiles/: a line `traffic-ratio <kernel> <workload> <ratio> <source> <digest>` gives
    the kernel's DRAM bytes over its algorithmic bytes, measured by ncu on a small variant
    of the workload (the ratio carries over: the bytes per weight tile and token row do not
    depend on the number of experts).  <digest> is code_digest() of the kernel source at
    the capture.  None when no summary matches or the kernel's code has changed since."""
    import glob
    for path in sorted(glob.glob(os.path.join(ROOT, "profiles", "*.md"))):
        try:
            lines = open(path).read().splitlines()
        except OSError:
            continue
        for line in lines:
            f = line.strip().strip("`").split()
            if len(f) != 6 or f[0] != "traffic-ratio" or f[1] != kernel or f[2] != workload:
                continue
            try:
                src = open(os.path.join(ROOT, f[4]), "rb").read()
            except OSError:
                return None
            if code_digest(src) != f[5]:
                return None
            return float(f[3]) * algorithmic_bytes
    return None


# ------------------------------------------------------------------------------------------
# ranks: every rank is an independent replica on its own tokens (weak scaling)
# ------------------------------------------------------------------------------------------
def rank_config(cfg, rank: int):
    """Rank r processes its own batch: same shapes and weights, tokens from seed + 1000 r."""
    return inputs.with_sizes(cfg, seed=cfg.seed + 1000 * rank) if rank else cfg


def max_over_ranks(value: float, pg, device) -> float:
    """The largest value over all ranks (the job's elapsed time is the slowest rank's)."""
    if pg is None:
        return value
    t = torch.tensor([value], device=device, dtype=torch.float64)
    pg.all_reduce(t, op=pg.ReduceOp.MAX)
    return float(t.item())


def job_tokens_per_s(tokens_per_rank: int, world: int, steps: int, elapsed_ms: float) -> float:
    return world * tokens_per_rank * steps / (elapsed_ms / 1e3)


# ------------------------------------------------------------------------------------------
# the oracle on the host (cpu baseline and the reference arm)
# ------------------------------------------------------------------------------------------
def host_arrays(d):
    import numpy as _np

    def cv(t):
        if t is None:
            return None
        if isinstance(t, tuple):  # FP8 weights: (codes, scales)
            return tuple(cv(u) for u in t)
        t = t.detach().cpu().contiguous()
        return t.view(torch.int16).numpy().view(_np.uint16) if t.dtype == torch.bfloat16 else t.numpy()
    return {k: cv(v) for k, v in d.items()}


LAYER_DEFAULTS = dict(router="softmax", routed_scaling_factor=1.0, swiglu_limit=0.0, swiglu_limit_shared=0.0)


def layer_options(args) -> dict:
    """Per-layer options of the run (router mode and scale, SwiGLU limits)."""
    return dict(router=args.router, routed_scaling_factor=args.routed_scale,
                swiglu_limit=args.swiglu_limit, swiglu_limit_shared=args.swiglu_limit_shared)


def config_options(args) -> dict:
    """The options as reported in the JSON line's config (empty for the defaults)."""
    o = layer_options(args)
    out = {"layer_options": o} if o != LAYER_DEFAULTS else {}
    if getattr(args, "fp32_router", False):
        out["router_weights"] = "fp32"
    if getattr(args, "weights", "bf16") == "fp8":
        out["expert_weights"] = "fp8: E4M3 codes, one E8M0 scale per 128x128 block (bf16 tensor-core math)"
    return out


def oracle_step(h, cfg, tokens, opts=None):
    """The whole hot path for the listed tokens: exact router over all experts, top-k and
    weights, then the expert FFNs and the combine.  FP8 weights come as (codes, scales)."""
    import oracle
    o = dict(LAYER_DEFAULTS, **(opts or {}))
    x = h["x"][tokens]
    s = oracle.router_scores(x, h["W_router"])
    bias = None if h.get("bias") is None else h["bias"].astype(np.float32)
    idx, w, w64 = oracle.route(s, cfg.top_k, bias, router=o["router"], scale=o["routed_scaling_factor"])
    lim = dict(swiglu_limit=o["swiglu_limit"], swiglu_limit_shared=o["swiglu_limit_shared"])
    if isinstance(h["W_gate_up"], tuple):
        return oracle.moe_tokens_fp8(x, idx, w64, h["W_gate_up"], h["W_down"], h["Ws_gate_up"], h["Ws_down"],
                                     **lim)
    return oracle.moe_tokens(x, idx, w64, h["W_gate_up"], h["W_down"], h["Ws_gate_up"], h["Ws_down"], **lim)


def sample_tokens(cfg) -> list:
    """The bounded token sample that the oracle times: the first min(T, 8) tokens of the
    workload (the whole batch of the T = 4 decode)."""
    return list(range(min(cfg.T, 8)))


def host_inputs(cfg, args, dev):
    """The workload's inputs for the oracle, as host arrays (weights drawn on the GPU when
    there is one, as the CUDA path draws them)."""
    x, Wr, bias = inputs.make_routing_inputs(cfg, router_fp32=args.fp32_router)
    if args.weights == "fp8":
        d = dict(x=x, W_router=Wr, bias=bias, **inputs.make_fp8_expert_weights(cfg, dev))
    else:
        Wgu, Wd, Wsgu, Wsd = inputs.make_expert_weights(cfg, dev)
        d = dict(x=x, W_router=Wr, bias=bias, W_gate_up=Wgu, W_down=Wd, Ws_gate_up=Wsgu, Ws_down=Wsd)
    return host_arrays(d)


def run_reference(args, cfg):
    """The reference arm: the CPU oracle as it stands, timed on the host cores; each step is
    one pass of the whole layer over the workload's bounded token sample."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    import oracle
    oracle.build()
    dev = "cuda" if torch.cuda.is_available() else "cpu"
    h = host_inputs(cfg, args, dev)
    cores = len(os.sched_getaffinity(0))
    tokens = sample_tokens(cfg)
    for _ in range(args.warmup):
        oracle_step(h, cfg, tokens, layer_options(args))
    t0 = time.perf_counter()
    for _ in range(args.steps):
        oracle_step(h, cfg, tokens, layer_options(args))
    dt = time.perf_counter() - t0
    value = len(tokens) * args.steps / dt
    sample = (f"{len(tokens)} tokens of {cfg.name} per step (tokens 0..{len(tokens) - 1}): exact router over "
              f"{cfg.E} experts, top-{cfg.top_k}, routed + shared expert FFNs in fp64")
    line = {"metric": METRIC, "value": value, "unit": UNIT, "impl": "reference", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * dt / args.steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": cfg.dtype,
            "data": "synthetic", "config": {"workload": cfg.name, "T": cfg.T, "H": cfg.H, "E": cfg.E,
                                             "top_k": cfg.top_k, "I": cfg.I, "I_shared": cfg.I_shared,
                                             **config_options(args)},
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle", "sample": sample},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


def cpu_baseline(h, cfg, opts=None, budget_s=8.0):
    """The oracle on the host cores, repeated over the workload's bounded token sample for
    about ``budget_s`` seconds (at least twice)."""
    import oracle
    cores = len(os.sched_getaffinity(0))
    tokens = sample_tokens(cfg)
    oracle_step(h, cfg, tokens, opts)  # warm-up: page in the weights
    n, t0 = 0, time.perf_counter()
    while True:
        oracle_step(h, cfg, tokens, opts)
        n += 1
        if n >= 2 and time.perf_counter() - t0 >= budget_s:
            break
    dt = time.perf_counter() - t0
    return {"value": len(tokens) * n / dt, "unit": UNIT, "cores": cores, "kind": "oracle",
            "sample": f"{len(tokens)} tokens of {cfg.name} (tokens 0..{len(tokens) - 1}) x {n} repetitions "
                      f"({dt:.1f} s): exact router over {cfg.E} experts, top-{cfg.top_k}, routed + shared "
                      f"expert FFNs in fp64"}


# ------------------------------------------------------------------------------------------
# the CUDA path
# ------------------------------------------------------------------------------------------
BF16_WORKLOADS = ("decode_t4", "decode_t128", "prefill_t4096", "prefill_t16384_skew")


def gemms_in_one_launch(cfg, fp8: bool) -> bool:
    """Whether the library runs both expert GEMMs as one launch on this workload: bf16
    weights with 16-token tiles, which it takes when experts hold at most six assignments
    on average (T * top_k <= 6 E).  The gate/up stage then times both GEMMs and the down
    stage is empty."""
    return not fp8 and cfg.T * cfg.top_k <= 6 * cfg.E


def roofline(alg, peaks, gu_ms, fp8, workload, fused=False):
    """Roofline of the dominant kernel, the gate/up GEMM (with 16-token tiles: the one launch
    of both GEMMs): its algorithmic bytes or FLOPs per launch over its average launch time,
    against the measured copy bandwidth when the launch is HBM-bound and the sustained bf16
    tensor peak when it is tensor-bound."""
    tc_peak = peaks["bf16_tflops_sustained"]
    nbytes = alg["gate_up_bytes"] + (alg["down_bytes"] if fused else 0)
    nflops = alg["gate_up_flops"] + (alg["down_flops"] if fused else 0)
    tensor_bound = nflops / (tc_peak * 1e12) > nbytes / (peaks["hbm_gbs"] * 1e9)
    if tensor_bound:
        achieved = nflops / (gu_ms / 1e3) / 1e12
        roof = {"bound": "tensor", "achieved": achieved, "peak": tc_peak, "unit": "TFLOP/s",
                "frac": achieved / tc_peak, "peak_kind": "sustained bf16 (cuBLAS, seconds-long loop)",
                "frac_of_burst": achieved / peaks["bf16_tflops"]}
    else:
        achieved = nbytes / (gu_ms / 1e3) / 1e9
        roof = {"bound": "hbm", "achieved": achieved, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                "frac": achieved / peaks["hbm_gbs"]}
    if fused:
        kernel = "expert_gemm_tc_kernel<gated, 16 tokens, both GEMMs> (gate/up + SiLU*up, then down)"
        key = "gemm_fused"
    else:
        kernel = "expert_gemm_tc_kernel<gated%s> (gate/up GEMM + SiLU*up)" % (", fp8" if fp8 else "")
        key = "gate_up"
    roof.update({"kernel": kernel,
                 "timing": "CUDA events around each launch, stage-timed pass of the same steps",
                 "traffic": ncu_traffic(key, workload + ("+fp8" if fp8 else ""), nbytes),
                 "peak_source": peaks["source"],
                 "ms_per_launch": gu_ms, "algorithmic_bytes": nbytes,
                 "algorithmic_flops": nflops})
    return roof


def layer_roofline(alg, peaks, ms_per_step):
    """The whole step against both roofs: bytes / time, FLOPs / time, and the fraction of the
    attainable time max(bytes / measured HBM bandwidth, FLOPs / sustained bf16 peak)."""
    s = ms_per_step / 1e3
    floor = max(alg["layer_bytes"] / (peaks["hbm_gbs"] * 1e9), alg["layer_flops"] / (peaks["bf16_tflops_sustained"] * 1e12))
    return {"touched_experts": alg["touched"], "algorithmic_bytes": alg["layer_bytes"],
            "algorithmic_flops": alg["layer_flops"],
            "hbm_gbs": alg["layer_bytes"] / s / 1e9, "hbm_frac": alg["layer_bytes"] / s / 1e9 / peaks["hbm_gbs"],
            "hbm_frac_of_8000": alg["layer_bytes"] / s / 1e9 / 8000.0,
            "tflops": alg["layer_flops"] / s / 1e12,
            "tensor_frac_sustained": alg["layer_flops"] / s / 1e12 / peaks["bf16_tflops_sustained"],
            "tensor_frac_burst": alg["layer_flops"] / s / 1e12 / peaks["bf16_tflops"],
            "frac_of_attainable": floor / s}


def measure(cfg, args, dev, pg, world, rank, local, clocks):
    """Everything measured on one workload: the plain timed pass (the value), a stage-timed
    pass (per-kernel durations), the end-to-end pass through host buffers and, on rank 0 at
    N = 1, the oracle's CPU baseline.  Returns the workload's record (rank 0) or None."""
    import sparse_mixture_experts_ffn_b200 as moe
    steps = args.steps if args.steps is not None else DEFAULT_STEPS.get(cfg.name, 100)
    x, Wr, bias = inputs.make_routing_inputs(rank_config(cfg, rank), router_fp32=args.fp32_router)
    fp8 = args.weights == "fp8"
    if fp8:
        W8 = inputs.make_fp8_expert_weights(cfg, dev)
        Wgu, Wd, Wsgu, Wsd = W8["W_gate_up"], W8["W_down"], W8["Ws_gate_up"], W8["Ws_down"]
    else:
        Wgu, Wd, Wsgu, Wsd = inputs.make_expert_weights(cfg, dev)
    x, Wr = x.to(dev), Wr.to(dev)
    bias = None if bias is None else bias.to(dev)
    shape = moe.make_shape(cfg.T, cfg.H, cfg.E, cfg.I, cfg.I_shared, cfg.top_k, cfg.torch_dtype)
    ws = moe.alloc_workspace(shape, dev)
    y = torch.empty_like(x)
    l2 = torch.cuda.get_device_properties(dev).L2_cache_size
    flush_w = torch.empty(max(2 * l2, 256 << 20), dtype=torch.uint8, device=dev)
    flush_r = torch.ones(flush_w.numel() // 4, dtype=torch.int32, device=dev)
    flush_sink = torch.zeros(1, dtype=torch.int64, device=dev)

    def flush():
        # evict everything, then leave the L2 holding clean lines of an unrelated buffer
        flush_w.zero_()
        flush_sink.add_(flush_r.sum())
    stream = torch.cuda.current_stream(dev)

    def step(xin, yout, routing=False):
        if fp8:
            return moe.moe_layer_forward_fp8(xin, Wr, W8, top_k=cfg.top_k, router_bias=bias, y=yout,
                                             workspace=ws, routing=routing, stream=stream, **layer_options(args))
        return moe.moe_layer_forward(xin, Wr, Wgu, Wd, Wsgu, Wsd, top_k=cfg.top_k, router_bias=bias,
                                     y=yout, workspace=ws, routing=routing, stream=stream,
                                     **layer_options(args))

    _, r = step(x, y, routing=True)
    torch.cuda.synchronize()
    status = moe.check_status(ws)
    if status != moe.MOE_OK:
        raise RuntimeError(f"{cfg.name}: device status {moe.status_string(status)}")
    counts = r.counts.cpu().numpy()
    route_stats = moe.route_stats(ws)
    alg = algorithmic(cfg, counts, fp8)

    for _ in range(args.warmup):
        flush()
        step(x, y)
    torch.cuda.synchronize()

    def timed_pass(profile: bool):
        starts = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
        ends = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
        moe.profile_read()
        moe.profile_enable(profile)
        if pg:
            pg.barrier()
        torch.cuda.synchronize()
        launches0 = moe.launch_count()
        since = len(clocks.samples)
        for i in range(steps):
            flush()
            starts[i].record(stream)
            step(x, y)
            ends[i].record(stream)
        torch.cuda.synchronize()
        clk = clocks.summary(since)
        if pg:
            pg.barrier()
        launches = moe.launch_count() - launches0
        moe.profile_enable(False)
        calls, stage_ms = moe.profile_read()
        elapsed = max_over_ranks(sum(s.elapsed_time(e) for s, e in zip(starts, ends)), pg, dev)
        return elapsed, launches, clk, calls, stage_ms

    # pass 1: the step as a user runs it, kernels chained with programmatic launches
    elapsed_ms, launches, clk, _, _ = timed_pass(False)
    # pass 2: the same steps with a CUDA event pair around every stage, for the per-kernel
    # durations (the events end the programmatic overlap between stages, so this pass is slower)
    elapsed_prof_ms, _, _, calls, stage_ms = timed_pass(True)
    status = moe.check_status(ws)

    # ---- end to end through the public API, host buffers ----------------------------------
    x_host = x.cpu().pin_memory()
    y_host = torch.empty(y.shape, dtype=y.dtype).pin_memory()
    x_dev = torch.empty_like(x)
    e_steps = max(3, min(steps, 500))
    es_, ee_ = ([torch.cuda.Event(enable_timing=True) for _ in range(e_steps)] for _ in range(2))
    for _ in range(3):
        x_dev.copy_(x_host, non_blocking=True)
        step(x_dev, y)
        y_host.copy_(y, non_blocking=True)
    torch.cuda.synchronize()
    if pg:
        pg.barrier()
    for i in range(e_steps):
        flush()
        es_[i].record(stream)
        x_dev.copy_(x_host, non_blocking=True)
        step(x_dev, y)
        y_host.copy_(y, non_blocking=True)
        ee_[i].record(stream)
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks(sum(s.elapsed_time(e) for s, e in zip(es_, ee_)), pg, dev)
    if pg:
        pg.barrier()
    rec = None
    if rank == 0:
        peaks = measured_peaks()
        ms_per_step = elapsed_ms / steps
        gu_ms = stage_ms["gate_up"] / max(calls, 1)
        rec = {
            "workload": cfg.name, "T": cfg.T, "steps": steps, "ms_per_step": ms_per_step,
            "value": job_tokens_per_s(cfg.T, world, steps, elapsed_ms), "unit": UNIT,
            "ms_per_step_stage_timed": elapsed_prof_ms / steps,
            "roofline": roofline(alg, peaks, gu_ms, fp8, cfg.name, gemms_in_one_launch(cfg, fp8)),
            "layer": dict(layer_roofline(alg, peaks, ms_per_step),
                          stage_ms_per_step={k: v / max(calls, 1) for k, v in stage_ms.items()},
                          route_stats=route_stats, device_status=moe.status_string(status)),
            "e2e": {"value": job_tokens_per_s(cfg.T, world, e_steps, e2e_ms), "unit": UNIT,
                    "h2d_bytes_per_step": x.numel() * x.element_size(),
                    "d2h_bytes_per_step": y.numel() * y.element_size(), "steps": e_steps},
            "gpu_launches": int(launches),
            "clocks": clk,
        }
    del ws, y, flush_w, flush_r, x_host
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        import oracle
        oracle.build()
        h = host_arrays(dict(x=x, W_router=Wr, bias=bias, W_gate_up=Wgu, W_down=Wd, Ws_gate_up=Wsgu,
                             Ws_down=Wsd))
        del Wgu, Wd, Wsgu, Wsd
        if fp8:
            del W8
        torch.cuda.empty_cache()
        rec["cpu_baseline"] = cpu_baseline(h, cfg, layer_options(args))
    return rec


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=None)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--workload", default=None, choices=sorted(inputs.CONFIGS),
                    help="one workload only (default: the four bf16 workloads, decode_t4 as the headline)")
    ap.add_argument("--impl", default="native", choices=["native", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--T", type=int, default=None, help="profiling variant: override the token count")
    ap.add_argument("--E", type=int, default=None, help="profiling variant: override the expert count")
    ap.add_argument("--router", default="softmax", choices=["softmax", "sigmoid"],
                    help="router mode (sigmoid: the router as configured, bias for the selection only)")
    ap.add_argument("--routed-scale", type=float, default=1.0, help="sigmoid router: routed scaling factor")
    ap.add_argument("--fp32-router", action="store_true", help="fp32 router weights (bf16 tokens and experts)")
    ap.add_argument("--swiglu-limit", type=float, default=0.0, help="SwiGLU limit of the routed experts")
    ap.add_argument("--swiglu-limit-shared", type=float, default=0.0, help="SwiGLU limit of the shared expert")
    ap.add_argument("--weights", default="bf16", choices=["bf16", "fp8"],
                    help="expert weights: bf16, or FP8 E4M3 codes with one E8M0 scale per 128x128 block")
    ap.add_argument("--I", type=int, default=None,
                    help="profiling variant: override both expert widths (small weights, same router)")
    args = ap.parse_args()
    names = [args.workload] if args.workload else list(BF16_WORKLOADS)
    cfgs = []
    for name in names:
        cfg = inputs.CONFIGS[name]
        if args.T is not None or args.E is not None or args.I is not None:
            T = cfg.T if args.T is None else args.T
            E = cfg.E if args.E is None else args.E
            I = cfg.I if args.I is None else args.I
            cfg = inputs.with_sizes(cfg, T=T, E=E, I=I, I_shared=I, name=f"{cfg.name}[T={T},E={E},I={I}]")
        cfgs.append(cfg)
    args.warmup = max(args.warmup, 3)
    if args.impl == "reference":
        if args.steps is None:
            args.steps = 20
        return run_reference(args, cfgs[0])

    import sparse_mixture_experts_ffn_b200 as moe
    from sparse_mixture_experts_ffn_b200 import build
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    pg = None
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)
        pg = dist
    if rank == 0 or world == 1:
        build.build()
    if pg:
        pg.barrier()
    moe.load_library()

    recs = []
    with ClockSampler(local) as clocks:
        for cfg in cfgs:
            recs.append(measure(cfg, args, dev, pg, world, rank, local, clocks))
            torch.cuda.empty_cache()
    if rank == 0:
        head = recs[0]
        cfg = cfgs[0]
        line = {
            "metric": METRIC, "value": head["value"], "unit": UNIT, "n_gpus": world, "steps": head["steps"],
            "warmup": args.warmup, "ms_per_step": head["ms_per_step"],
            "ms_per_step_stage_timed": head["ms_per_step_stage_timed"], "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": cfg.dtype, "data": "synthetic",
            "config": {"workload": cfg.name, "T": cfg.T, "H": cfg.H, "E": cfg.E, "top_k": cfg.top_k,
                       "I": cfg.I, "I_shared": cfg.I_shared, "tokens_per_gpu": cfg.T,
                       **config_options(args),
                       "l2": "flushed before every timed step, outside the events: 2x L2 write, then 2x L2 read",
                       "parallelism": f"replicas x{world}"},
            "roofline": head["roofline"],
            "layer": head["layer"],
            "e2e": head["e2e"],
            "gpu_launches": head["gpu_launches"],
            "clocks": head["clocks"],
        }
        if "cpu_baseline" in head:
            line["cpu_baseline"] = head["cpu_baseline"]
        if len(recs) > 1:
            line["per_workload"] = {r["workload"]: r for r in recs}
            line["clocks_all_workloads"] = clocks.summary()
        print(json.dumps(line), flush=True)
    if pg:
        pg.barrier()
        pg.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
