#!/usr/bin/env python
"""Benchmark of the B200 MoE layer forward pass (biased-sigmoid routing, clipped SwiGLU
experts, shared expert) through the C ABI.

One step = one moe_forward over one batch: router -> permutation -> gather / tile table ->
grouped gate_up GEMM + clipped SwiGLU -> grouped down GEMM + weighted scatter-add.
Default workload: the largest single-GPU configuration, the Step-5-Preview-shaped layer
with skewed routing (T=16384, H=4096, E=352, top-8, I=Is=1536, Zipf-shaped router bias).
Inputs are seeded synthetic tensors drawn on the device; the expert weights (13 GB) are
larger than L2, so every step streams them from HBM. Decode-sized workloads (at most 16
routed rows per expert) also write a 512 MiB buffer between timed steps, outside the
timed intervals, so no step starts with the previous step's weights in L2.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl b200|reference]

Multi-GPU (torchrun, one process per GPU): independent replicas, no collective on the data
path ("replicas only"); value = tokens processed by all ranks / max-over-ranks time.
--impl reference times the CPU oracle on a bounded token sample of the same workload.
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

METRIC = "MoE layer fwd tokens/s on 1 B200; % of BF16 tensor peak / HBM roofline"
UNIT = "tokens/s"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default="step5_skewed")
    ap.add_argument("--impl", default="b200", choices=["b200", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--deterministic", action="store_true")
    ap.add_argument("--routing", default="router", choices=["router", "balanced"],
                    help="router: full layer; balanced: fixed round-robin routing through moe_forward_with_ids "
                         "(fake balanced static expert routing)")
    ap.add_argument("--weights", default="bf16", choices=["bf16", "fp8"],
                    help="routed expert weights: bf16, or FP8 E4M3 with 128x128 block scales (moe_forward_fp8)")
    ap.add_argument("--pass", dest="which", default="forward", choices=["forward", "backward", "router"],
                    help="backward: time moe_backward (all gradients) for the forward's routing; "
                         "router: time moe_router alone (profiling)")
    ap.add_argument("--parallel", default="replicas", choices=["replicas", "ep"],
                    help="ep: expert parallelism, E/N routed experts per rank, T tokens per rank")
    ap.add_argument("--graph", action="store_true",
                    help="also time the forward captured once in a CUDA graph and replayed (key 'graph')")
    ap.add_argument("--tokens", type=int, default=None, help="override T (profiling runs)")
    ap.add_argument("--experts", type=int, default=None, help="override E (profiling runs)")
    return ap.parse_args()


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            p = json.load(f)
        return p, "measured"
    return FALLBACK_PEAKS, "fallback"


class ClockSampler:
    """SM clock and clock-event reasons of this GPU, read through NVML every 5 ms while the
    timed region runs (read-only queries; nvidia-smi at its 200 ms minimum if NVML is
    unavailable)."""

    REASONS = (("hw_slowdown", "nvmlClocksEventReasonHwSlowdown"),
               ("hw_thermal_slowdown", "nvmlClocksEventReasonHwThermalSlowdown"),
               ("sw_thermal_slowdown", "nvmlClocksEventReasonSwThermalSlowdown"),
               ("sw_power_cap", "nvmlClocksEventReasonSwPowerCap"),
               ("hw_power_brake", "nvmlClocksEventReasonHwPowerBrakeSlowdown"),
               # informative only (a clock lock or an application-clock setting shows here)
               ("applications_clocks_setting", "nvmlClocksEventReasonApplicationsClocksSetting"),
               ("sync_boost", "nvmlClocksEventReasonSyncBoost"),
               ("display_clock_setting", "nvmlClocksEventReasonDisplayClockSetting"))
    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_id: str):
        self.gpu_id = gpu_id
        self.samples = []  # (sm_mhz, sm_max_mhz, reasons)
        self.lines = []
        self.proc = None
        self.thread = None
        self.stop_flag = threading.Event()
        self.source = None

    def start(self):
        try:
            import pynvml
            pynvml.nvmlInit()
            handle = pynvml.nvmlDeviceGetHandleByUUID(self.gpu_id)
            smax = float(pynvml.nvmlDeviceGetMaxClockInfo(handle, pynvml.NVML_CLOCK_SM))
            masks = [(name, getattr(pynvml, attr, 0)) for name, attr in self.REASONS]
        except Exception:
            self._start_smi()
            return
        self.source = "nvml 5 ms"

        def poll():
            while not self.stop_flag.is_set():
                try:
                    sm = float(pynvml.nvmlDeviceGetClockInfo(handle, pynvml.NVML_CLOCK_SM))
                    bits = pynvml.nvmlDeviceGetCurrentClocksEventReasons(handle)
                    self.samples.append((sm, smax, {n for n, m in masks if bits & m}))
                except Exception:
                    pass
                time.sleep(0.005)

        self.thread = threading.Thread(target=poll, daemon=True)
        self.thread.start()

    def _start_smi(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits", "-i", self.gpu_id,
                 "-lms", "200"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
            return
        self.source = "nvidia-smi 200 ms"
        self.thread = threading.Thread(target=self._read, daemon=True)
        self.thread.start()

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        self.stop_flag.set()
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
        if self.thread:
            self.thread.join(timeout=5)
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 8:
                continue
            try:
                self.samples.append((float(parts[0]), float(parts[1]),
                                     {n for n, v in zip(names, parts[4:8]) if v.lower() == "active"}))
            except ValueError:
                continue
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no clock samples"], "samples": 0,
                    "source": self.source}
        sm = [x[0] for x in self.samples]
        reasons = set().union(*(x[2] for x in self.samples))
        return {"sm_mhz": statistics.median(sm), "sm_min_mhz": min(sm), "sm_max_mhz": max(x[1] for x in self.samples),
                "reasons": sorted(reasons), "samples": len(sm), "source": self.source}


def max_over_ranks(value: float, device) -> float:
    """Largest value over all ranks (the job's time is its slowest rank's time)."""
    import torch
    import torch.distributed as dist

    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_tokens_per_s(world: int, tokens_per_rank: int, steps: int, max_ms: float) -> float:
    """Whole-job throughput: tokens processed by all ranks over the slowest rank's time."""
    return world * tokens_per_rank * steps / (max_ms / 1e3)


def workload_config(shape, extra=None):
    c = {"workload": shape.name, "T": shape.T, "H": shape.H, "E": shape.E, "k": shape.k, "I": shape.I,
         "Is": shape.Is, "scale": shape.scale, "norm_expert_weight": shape.norm_expert_weight,
         "limit_routed": shape.limit_routed, "limit_shared": shape.limit_shared, "seed": shape.seed,
         "bias": shape.bias_kind}
    if extra:
        c.update(extra)
    return c


def cpu_oracle_sample(shape, inp, target_s: float, max_tokens: int = 4096, start: int = 0):
    """Times the CPU oracle on a token sample of the workload; returns (tokens/s, n, seconds)."""
    import numpy as np
    import oracle
    from sparse_moe_layer_biased_b200.inputs import bf16_bits

    host = {k: v.cpu() for k, v in inp.items() if k in ("Wr", "bias", "Wsh_gate_up", "Wsh_down")}
    gu = inp["W_gate_up"]
    wd = inp["W_down"]
    Wr = bf16_bits(host["Wr"])
    bias = host["bias"].numpy()
    Wsh_gu = bf16_bits(host["Wsh_gate_up"])
    Wsh_d = bf16_bits(host["Wsh_down"])
    cache = {}

    def run(rows):
        x_rows = bf16_bits(inp["x"][rows])
        r = oracle.router(x_rows, Wr, bias, shape.k, shape.scale, shape.norm_expert_weight)
        for e in np.unique(r["idx"]):
            if int(e) not in cache:
                cache[int(e)] = (bf16_bits(gu[int(e)]), bf16_bits(wd[int(e)]))
        experts = {int(e): cache[int(e)] for e in np.unique(r["idx"])}
        t0 = time.perf_counter()
        ref = oracle.forward_tokens(x_rows, Wr, bias, experts, Wsh_gu, Wsh_d, k=shape.k, scale=shape.scale,
                                    norm=shape.norm_expert_weight, limit_routed=shape.limit_routed,
                                    limit_shared=shape.limit_shared)
        return time.perf_counter() - t0, ref

    nthreads = oracle.num_threads()
    n0 = max(1, min(nthreads, shape.T))
    rows = [(start + i) % shape.T for i in range(n0)]
    dt, _ = run(rows)
    per_tok = dt / n0
    n = int(min(max_tokens, shape.T, max(n0, target_s / max(per_tok, 1e-9))))
    # spread the timed sample over the whole batch (every region of the permuted rows)
    step = max(1, shape.T // n)
    rows = sorted({(start + n0 + i * step) % shape.T for i in range(n)})
    dt, ref = run(rows)
    return len(rows) / dt, len(rows), dt, nthreads, rows, ref


def run_reference(args, shape):
    """CPU oracle arm: each step runs the oracle on a bounded token sample."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    import torch
    from sparse_moe_layer_biased_b200.inputs import draw

    dev = "cuda" if torch.cuda.is_available() else "cpu"
    inp = draw(shape, device=dev)
    budget = 150.0 / max(1, args.steps + args.warmup)
    rates, times = [], []
    n_used = None
    threads = None
    for i in range(args.warmup + args.steps):
        rate, n, dt, threads, _, _ = cpu_oracle_sample(shape, inp, target_s=budget, start=i * 97)
        if i >= args.warmup:
            rates.append(rate)
            times.append(dt * 1e3)
            n_used = n
    value = statistics.median(rates)
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": statistics.median(times),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic (seeded; same draw as the b200 arm)",
        "config": workload_config(shape, {"parallelism": "rank 0 only (CPU oracle)"}),
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": threads, "kind": "oracle",
                         "sample": f"{n_used} tokens per step of {shape.name}, oracle forward (router + k routed "
                                   f"+ shared expert MLPs in fp64)"},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


# DRAM traffic (read + write) of one launch of the dominant kernel, as a ratio to the launch's
# algorithmic bytes, from one ncu capture of a reduced case of the same shape per expert (the
# profile named in each entry: T=2048, E=44 for the skewed Step-5 layer; T=1024, E=72 for the
# Step-3.5 prefill layer): the full launch's traffic is that ratio times its own algorithmic
# bytes. A figure holds only for the sources it was taken from: the lookup returns None once
# the code of any file in TRAFFIC_SOURCES changes.
PROFILED_TRAFFIC = {
    ("step5_skewed", "bf16"): {"ratio": (1450539008 + 51255552) / 1205862400,
                               "csrc_sha256": "f5dad4ee22b697d3d812c89b0052aa624b354519758885a58a935909f9ac4fde",
                               "source": "profiles/dram_gate_up_down_step5_skewed_T2048_E44.md"},
    ("step35_prefill", "bf16"): {"ratio": (1623792640 + 23229952) / 1562902528,
                                 "csrc_sha256": "f5dad4ee22b697d3d812c89b0052aa624b354519758885a58a935909f9ac4fde",
                                 "source": "profiles/dram_gate_up_down_step35_prefill_T1024_E72.md"},
}


def _strip_comments(src: str) -> str:
    """C/C++ source without its comments and blank lines (string and character literals kept)."""
    out, i, n = [], 0, len(src)
    while i < n:
        c = src[i]
        if c in "\"'":
            j = i + 1
            while j < n and src[j] != c:
                j += 2 if src[j] == "\\" else 1
            out.append(src[i:j + 1])
            i = j + 1
        elif src.startswith("//", i):
            j = src.find("\n", i)
            i = n if j < 0 else j
        elif src.startswith("/*", i):
            j = src.find("*/", i + 2)
            i = n if j < 0 else j + 2
        else:
            out.append(c)
            i += 1
    return "\n".join(l.strip() for l in "".join(out).splitlines() if l.strip())


# Sources of the BF16 forward path up to and including the grouped GEMMs (launch sequence and
# configuration, permutation and gather, GEMM kernels and their helpers): the files whose
# code decides the gate_up kernel's DRAM traffic. The router, the FP8 kernels and the
# backward pass are not among them.
TRAFFIC_SOURCES = ("moe_api.cu", "internal.h", "permute.cu", "expert_gemm.cu", "expert_gemm_pair.cu",
                   "epilogue.cuh", "gemm_common.cuh", "sm100.cuh")


def csrc_digest() -> str:
    """Digest of the code (comments excluded) of TRAFFIC_SOURCES, which the profiled traffic
    figures are tied to."""
    import hashlib
    d = os.path.join(os.path.dirname(os.path.abspath(__file__)), "sparse_moe_layer_biased_b200", "csrc")
    h = hashlib.sha256()
    for name in sorted(TRAFFIC_SOURCES):
        with open(os.path.join(d, name), encoding="utf-8") as f:
            h.update(name.encode() + b"\0" + _strip_comments(f.read()).encode())
    return h.hexdigest()


def profiled_traffic(shape_name: str, weights: str, algorithmic_bytes: float):
    """Per-launch DRAM traffic of gate_up for this workload (None without a capture of the
    current sources)."""
    e = PROFILED_TRAFFIC.get((shape_name, weights))
    if e is None or e["csrc_sha256"] != csrc_digest():
        return None
    return e["ratio"] * algorithmic_bytes


def kernels_per_step(shape, fp8=False, deterministic=False, router=True):
    """Kernels one forward call launches: router, permute, gather, tile tables, gate_up and
    down (+ combine in deterministic mode; no router with given ids). With FP8 routed experts
    on a prefill-sized call the BF16 shared expert runs on the CTA-pair kernels with its own
    tile tables, gate_up and down."""
    n = 6 + (1 if deterministic else 0) - (0 if router else 1)
    if (fp8 and shape.T * shape.k > 16 * shape.E and shape.I % 128 == 0 and shape.Is % 128 == 0
            and shape.H % 512 == 0):
        n += 3
    return n


def gate_up_bytes(shape, counts, fp8=False):
    """Algorithmic HBM bytes of one gate_up launch: weights of every expert that received
    tokens (2I x H, bf16 or E4M3 codes plus one fp32 scale per 128x128 block) + shared
    gate_up (bf16) + the token rows x, counted once (the method reads each token once;
    the implementation's permuted copy of x is not algorithmic) + the hidden activations
    written (routed and shared rows, bf16)."""
    touched = int((counts[: shape.E] > 0).sum())
    T, H, k, I, Is = shape.T, shape.H, shape.k, shape.I, shape.Is
    per_expert = 2 * I * H + (2 * I // 128) * (H // 128) * 4 if fp8 else 2 * I * H * 2
    w = touched * per_expert + 2 * Is * H * 2
    acts = T * H * 2
    out = T * k * I * 2 + T * Is * 2
    return w + acts + out, touched


def gate_up_flops(shape):
    """Algorithmic FLOPs of one gate_up launch: 2 x (2I x H) per routed row, 2 x (2Is x H) per
    shared row."""
    return 4.0 * shape.H * (shape.I * shape.T * shape.k + shape.Is * shape.T)


def graph_replay(args, shape, step, x, y, flush_buf, stream, world):
    """The step captured once in a CUDA graph (the library only enqueues: no allocation or
    synchronisation inside a call) and replayed K times, each replay between its own CUDA events
    (the L2 flush of decode-sized workloads stays outside them). Returns the per-step time and
    the throughput; the launches of the graph are the step's kernels."""
    import torch

    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, capture_error_mode="relaxed"):
        step(x, y)
    torch.cuda.synchronize()
    for _ in range(max(1, args.warmup)):
        g.replay()
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    torch.cuda.synchronize()
    cur = torch.cuda.current_stream()
    for i in range(args.steps):
        if flush_buf is not None:
            flush_buf.fill_(i & 0xFF)
        evs[i][0].record(cur)
        g.replay()
        evs[i][1].record(cur)
    torch.cuda.synchronize()
    ms = max_over_ranks(sum(a.elapsed_time(b) for a, b in evs), "cuda")
    del g
    return {"value": job_tokens_per_s(world, shape.T, args.steps, ms), "unit": UNIT,
            "ms_per_step": ms / args.steps, "api": "moe_forward captured in one CUDA graph, replayed"}


def gate_up_kernel_name(shape, fp8=False):
    """The gate_up kernel one call launches (the library's configuration choice)."""
    decode = shape.T * shape.k <= 16 * shape.E
    if fp8:
        if decode and shape.H % 256 == 0 and shape.I % 128 == 0 and shape.Is % 128 == 0:
            return "gemm_fp8_mma_kernel<GateUpArgs>"
        return "gemm_fp8_kernel<GateUpArgs>"
    if not decode and shape.I % 128 == 0 and shape.Is % 128 == 0 and shape.H % 512 == 0:
        return "gate_up_pair_kernel"
    return "gate_up_kernel"


def gate_up_roofline(shape, counts, launch_ms, peaks, peak_kind, fp8=False, traffic=None):
    """Roofline block of the dominant kernel (gate_up). The bound is the resource whose
    time floor is longer at the measured peaks: algorithmic bytes / HBM copy bandwidth
    against algorithmic FLOPs / bf16 dense peak (burst). achieved / frac are reported on
    that bound; the other figure is kept beside it for context."""
    nbytes, touched = gate_up_bytes(shape, counts, fp8)
    flops = gate_up_flops(shape)
    t_hbm = nbytes / (peaks["hbm_gbs"] * 1e9)
    t_tc = flops / (peaks["bf16_tflops"] * 1e12)
    gbs = nbytes / (launch_ms / 1e3) / 1e9
    tfs = flops / (launch_ms / 1e3) / 1e12
    kernel = gate_up_kernel_name(shape, fp8)
    common = {"kernel": kernel, "traffic": traffic, "algorithmic_bytes": nbytes, "algorithmic_flops": flops,
              "intensity_flop_per_byte": flops / nbytes,
              "ridge_flop_per_byte": peaks["bf16_tflops"] * 1e12 / (peaks["hbm_gbs"] * 1e9),
              "launch_ms": launch_ms, "touched_experts": touched,
              "hbm": {"achieved": gbs, "peak": peaks["hbm_gbs"], "frac": gbs / peaks["hbm_gbs"]},
              "tensor": {"achieved": tfs, "peak": peaks["bf16_tflops"], "frac": tfs / peaks["bf16_tflops"],
                         "frac_of_sustained": tfs / peaks.get("bf16_tflops_sustained", peaks["bf16_tflops"])}}
    if t_tc >= t_hbm and not fp8:
        head = {"bound": "tensor", "achieved": tfs, "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
                "frac": tfs / peaks["bf16_tflops"], "peak_source": f"{peak_kind} bf16_tflops (burst)"}
    else:
        head = {"bound": "hbm", "achieved": gbs, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                "frac": gbs / peaks["hbm_gbs"], "peak_source": f"{peak_kind} hbm_gbs"}
    head.update(common)
    return head


def decode_sized(shape) -> bool:
    """At most 16 routed rows per expert on average (the decode tiling of the kernels)."""
    return shape.T * shape.k <= 16 * shape.E


def sample_parity(y, idx, w, rows, ref, near_tie=1e-6):
    """Parity of the timed path on the oracle's token sample: expert-id sets equal outside
    near-ties (oracle margin < 1e-6, counted), and the output's relative Frobenius and max
    abs errors against the fp64 oracle over the sampled tokens whose id sets agree (a
    near-tie token routed to another valid set is counted, not compared)."""
    import numpy as np
    import torch

    r = torch.as_tensor(rows, device=y.device)
    yg = y[r].double().cpu().numpy()
    ig = idx[r].cpu().numpy()
    keep = ref["margin"] >= near_tie
    same = (np.sort(ig, 1) == np.sort(ref["idx"], 1)).all(1)
    d = yg[same] - ref["y"][same]
    return {"tokens": int(len(rows)), "near_ties": int((~keep).sum()),
            "ids_equal_outside_near_ties": bool(same[keep].all()),
            "near_tie_tokens_routed_differently": int((~same & ~keep).sum()),
            "rel_fro": float(np.linalg.norm(d) / np.linalg.norm(ref["y"][same])),
            "max_abs": float(np.abs(d).max()), "bar": {"rel_fro": 1e-2, "max_abs": 3e-2}}


def run_b200(args, shape):
    import numpy as np
    import torch
    import torch.distributed as dist

    from sparse_moe_layer_biased_b200 import _abi
    from sparse_moe_layer_biased_b200.inputs import draw, draw_fp8
    from sparse_moe_layer_biased_b200.layer import MoeLayer

    fp8 = args.weights == "fp8"
    if fp8 and args.routing == "balanced":
        raise SystemExit("--routing balanced replays routing through the BF16 entry point only")
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    if world > 1:
        import datetime

        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))

    def barrier():
        if world > 1:
            dist.barrier()

    inp = (draw_fp8 if fp8 else draw)(shape, device="cuda")
    layer = MoeLayer(shape, inp, deterministic=args.deterministic)
    x = inp["x"]
    y = torch.empty((shape.T, shape.H), dtype=torch.float32, device="cuda")
    stream = torch.cuda.current_stream()
    if args.routing == "balanced":
        t = torch.arange(shape.T, device="cuda")[:, None]
        j = torch.arange(shape.k, device="cuda")[None, :]
        fixed_idx = ((t * shape.k + j) % shape.E).to(torch.int32).contiguous()
        fixed_w = torch.full((shape.T, shape.k), shape.scale / shape.k, dtype=torch.float32, device="cuda")
        bdesc = _abi.desc_of(shape, deterministic=args.deterministic)

        def step(xx, yy):
            _abi.moe_forward_with_ids(bdesc, xx, fixed_idx, fixed_w, inp["W_gate_up"], inp["W_down"],
                                      inp["Wsh_gate_up"], inp["Wsh_down"], yy, layer.ws)
    else:
        def step(xx, yy):
            layer.forward(xx, y=yy)

    # warm-up (also yields the routing used for the algorithmic byte count)
    if args.routing == "balanced":
        idx = fixed_idx
        step(x, y)
    else:
        _, idx, _ = layer.forward(x, y=y, routing=True)
    for _ in range(max(0, args.warmup - 1)):
        step(x, y)
    torch.cuda.synchronize()
    _abi.moe_check_device()
    counts = np.bincount(idx.cpu().numpy().ravel(), minlength=shape.E)

    nstage = 7 if args.deterministic else 6
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(nstage)] for _ in range(args.steps)]
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    gpu_name = str(torch.cuda.get_device_properties(local).uuid)
    sampler = ClockSampler("GPU-" + gpu_name if not gpu_name.startswith("GPU-") else gpu_name)
    flush = decode_sized(shape)
    flush_buf = torch.empty(512 << 20, dtype=torch.uint8, device="cuda") if flush else None
    barrier()
    torch.cuda.synchronize()
    sampler.start()
    start.record(stream)
    for i in range(args.steps):
        if flush:
            flush_buf.fill_(i & 0xFF)  # evicts L2 between steps, outside the step's events
        _abi.moe_set_stage_events(evs[i])
        step(x, y)
    end.record(stream)
    torch.cuda.synchronize()
    clocks = sampler.stop()
    _abi.moe_set_stage_events([])
    barrier()
    if flush:  # the steps' own intervals, first to last stage event, flushes excluded
        total = sum(evs[i][0].elapsed_time(evs[i][nstage - 1]) for i in range(args.steps))
    else:
        total = start.elapsed_time(end)
    ms = max_over_ranks(total, "cuda")
    names = ["router", "permute", "gather_tiles", "gate_up", "down", "combine"][: nstage - 1]
    stage_ms = {n: statistics.mean(evs[i][j].elapsed_time(evs[i][j + 1]) for i in range(args.steps))
                for j, n in enumerate(names)}
    _abi.moe_check_device()

    # end to end through the public API with host buffers (pinned), copies inside the timed region
    e2e = None
    if not args.no_e2e and args.routing == "router":
        # moe_forward_host: every step's batch comes from pinned host memory and its output
        # goes back to it; the copies overlap the forward of the neighbouring batch
        per_batch = shape.T * shape.H * 6
        nb = max(2, min(args.steps, (4 << 30) // per_batch))
        x_h = x.cpu()[None].expand(nb, shape.T, shape.H).contiguous().pin_memory()
        y_h = torch.empty((nb, shape.T, shape.H), dtype=torch.float32).pin_memory()
        layer.forward_host(x_h[:2], y_h[:2])
        torch.cuda.synchronize()
        barrier()
        s2, e2 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        s2.record(stream)
        left = args.steps
        while left > 0:
            n = min(nb, left)
            layer.forward_host(x_h[:n], y_h[:n])
            left -= n
        e2.record(stream)
        torch.cuda.synchronize()
        _abi.moe_check_device()
        ms2 = max_over_ranks(s2.elapsed_time(e2), "cuda")
        e2e = {"value": job_tokens_per_s(world, shape.T, args.steps, ms2), "unit": UNIT,
               "h2d_bytes_per_step": shape.T * shape.H * 2, "d2h_bytes_per_step": shape.T * shape.H * 4,
               "api": f"moe_forward_host, {nb} host batches per call"}
    elif not args.no_e2e:
        x_h = x.cpu().pin_memory()
        y_h = torch.empty((shape.T, shape.H), dtype=torch.float32).pin_memory()
        x_d = torch.empty_like(x)
        for _ in range(2):
            x_d.copy_(x_h, non_blocking=True)
            step(x_d, y)
            y_h.copy_(y, non_blocking=True)
        torch.cuda.synchronize()
        barrier()
        s2, e2 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        s2.record(stream)
        for _ in range(args.steps):
            x_d.copy_(x_h, non_blocking=True)
            step(x_d, y)
            y_h.copy_(y, non_blocking=True)
        e2.record(stream)
        torch.cuda.synchronize()
        ms2 = max_over_ranks(s2.elapsed_time(e2), "cuda")
        e2e = {"value": job_tokens_per_s(world, shape.T, args.steps, ms2), "unit": UNIT,
               "h2d_bytes_per_step": shape.T * shape.H * 2, "d2h_bytes_per_step": shape.T * shape.H * 4}

    peaks, peak_kind = load_peaks()
    roofline = gate_up_roofline(shape, counts, stage_ms["gate_up"], peaks, peak_kind, fp8)
    roofline["traffic"] = profiled_traffic(shape.name, args.weights, roofline["algorithmic_bytes"])
    flops = shape.flops_per_token * shape.T
    step_ms = ms / args.steps
    value = job_tokens_per_s(world, shape.T, args.steps, ms)
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": step_ms, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic (seeded draw on device; random-init weights)",
        "config": workload_config(shape, {"parallelism": f"replicas x{world}" if world > 1 else "single GPU",
                                          "l2": ("512 MiB written between timed steps (decode-sized); "
                                                 "expert weights larger than L2") if flush else
                                                "inputs larger than L2 (expert weights streamed every step)",
                                          "routing": args.routing,
                                          "weights": "fp8_e4m3_block128x128" if fp8 else "bf16",
                                          "deterministic": bool(args.deterministic)}),
        "roofline": roofline,
        "tensor": {"achieved_tflops": flops / (step_ms / 1e3) / 1e12,
                   "frac_of_bf16_peak": flops / (step_ms / 1e3) / 1e12 / peaks["bf16_tflops"]},
        "stages_ms": stage_ms,
        "clocks": clocks,
        "e2e": e2e,
        "gpu_launches": kernels_per_step(shape, fp8, args.deterministic, args.routing != "balanced") * args.steps,
    }
    if args.graph:
        line["graph"] = graph_replay(args, shape, step, x, y, flush_buf, stream, world)
    if rank == 0 and world == 1 and not args.no_cpu_baseline and not fp8:
        # one more forward in the timed launch configuration: the oracle's sample doubles
        # as a parity check of the timed path
        _, idx_now, w_now = layer.forward(x, y=y, routing=True)
        torch.cuda.synchronize()
        rate, n, dt, threads, rows, ref = cpu_oracle_sample(shape, inp, target_s=15.0)
        line["cpu_baseline"] = {"value": rate, "unit": UNIT, "cores": threads, "kind": "oracle",
                                "sample": f"{n} tokens of {shape.name} spread over the batch, through the CPU "
                                          f"oracle forward ({dt:.1f} s, fp64)"}
        line["parity"] = sample_parity(y, idx_now, w_now, rows, ref)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(line), flush=True)


def run_ep(args, shape):
    """Expert-parallel layer (EPMoeLayer): N ranks, rank r owns routed experts
    [r*E/N, (r+1)*E/N), each rank routes its own T tokens (weak scaling); dispatch, return and
    combine go through NCCL all-to-alls. At N = 1 the exchanges are copies, which measures
    the cost of the split path against the fused single-GPU forward. Kernel launches per
    step: router, permute, pack, regroup, gather, tile table, gate_up, down (owner side),
    tile table, gate_up, down (shared expert), combine."""
    import datetime

    import torch
    import torch.distributed as dist

    from sparse_moe_layer_biased_b200 import _abi
    from sparse_moe_layer_biased_b200.ep import EPMoeLayer
    from sparse_moe_layer_biased_b200.inputs import draw

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    kw = {"timeout": datetime.timedelta(seconds=120), "device_id": torch.device("cuda", local)}
    if world > 1:
        dist.init_process_group("nccl", **kw)
    else:
        dist.init_process_group("nccl", store=dist.HashStore(), rank=0, world_size=1, **kw)
    inp = draw(shape, device="cuda")
    Er = shape.E // world
    w = {"Wr": inp["Wr"], "bias": inp["bias"], "Wsh_gate_up": inp["Wsh_gate_up"], "Wsh_down": inp["Wsh_down"],
         "W_gate_up": inp["W_gate_up"][rank * Er:(rank + 1) * Er].contiguous(),
         "W_down": inp["W_down"][rank * Er:(rank + 1) * Er].contiguous()}
    del inp["W_gate_up"], inp["W_down"]
    if rank == 0:
        x = inp["x"]
    else:
        g = torch.Generator(device="cuda").manual_seed(shape.seed * 1000 + rank)
        x = (torch.randn((shape.T, shape.H), generator=g, device="cuda") * shape.x_std).to(torch.bfloat16)
    layer = EPMoeLayer(shape, w)
    for _ in range(max(1, args.warmup)):
        layer.forward(x)
    torch.cuda.synchronize()
    _abi.moe_check_device()
    stream = torch.cuda.current_stream()
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    uuid = str(torch.cuda.get_device_properties(local).uuid)
    sampler = ClockSampler(uuid if uuid.startswith("GPU-") else "GPU-" + uuid)
    dist.barrier()
    torch.cuda.synchronize()
    sampler.start()
    start.record(stream)
    for _ in range(args.steps):
        layer.forward(x)
    end.record(stream)
    torch.cuda.synchronize()
    clocks = sampler.stop()
    dist.barrier()
    _abi.moe_check_device()
    ms = max_over_ranks(start.elapsed_time(end), "cuda")
    line = {
        "metric": METRIC, "value": job_tokens_per_s(world, shape.T, args.steps, ms), "unit": UNIT,
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (seeded draw on device; random-init weights)",
        "config": workload_config(shape, {"parallelism": f"ep{world} ({Er} routed experts per rank)",
                                          "l2": "inputs larger than L2 (expert weights streamed every step)",
                                          "routing": "router", "weights": "bf16", "deterministic": True}),
        "roofline": None,
        "clocks": clocks,
        "e2e": None,
        "gpu_launches": 12 * args.steps,
    }
    dist.barrier()
    dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(line), flush=True)


def run_router_only(args, shape):
    """Times moe_router alone on the workload's x, router weights and bias (the same draw as
    the layer; the expert tensors are drawn at I = Is = 64 to keep the device footprint
    small). One GPU; one router_kernel launch per step."""
    import torch

    from sparse_moe_layer_biased_b200 import _abi
    from sparse_moe_layer_biased_b200.inputs import draw

    torch.cuda.set_device(0)
    inp = draw(shape.replace(I=64, Is=64), device="cuda")
    d = _abi.desc_of(shape)
    idx = torch.empty((shape.T, shape.k), dtype=torch.int32, device="cuda")
    w = torch.empty((shape.T, shape.k), dtype=torch.float32, device="cuda")
    for _ in range(max(1, args.warmup)):
        _abi.moe_router(d, inp["x"], inp["Wr"], inp["bias"], idx, w)
    torch.cuda.synchronize()
    _abi.moe_check_device()
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    start.record()
    for _ in range(args.steps):
        _abi.moe_router(d, inp["x"], inp["Wr"], inp["bias"], idx, w)
    end.record()
    torch.cuda.synchronize()
    _abi.moe_check_device()
    ms = start.elapsed_time(end) / args.steps
    print(json.dumps({"metric": "MoE router tokens/s on 1 B200", "value": shape.T / (ms / 1e3), "unit": UNIT,
                      "n_gpus": 1, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
                      "higher_is_better": True, "dtype": "bf16", "data": "synthetic (seeded draw on device)",
                      "config": workload_config(shape, {"pass": "router"}), "gpu_launches": args.steps}),
          flush=True)


def run_backward(args, shape):
    """Times moe_backward (dx, dWr, dW_gate_up, dW_down and the shared expert's gradients) on
    device-resident inputs for the forward's routing; one GPU. Algorithmic FLOPs per routed
    (token, expert) row: recompute 4HI + dgrad 2HI + 4HI + wgrad 2HI + 4HI = 16HI (shared
    rows 16H*Is) + router 4HE-level work not counted."""
    import torch

    from sparse_moe_layer_biased_b200 import _abi
    from sparse_moe_layer_biased_b200.inputs import draw
    from sparse_moe_layer_biased_b200.layer import MoeLayer

    torch.cuda.set_device(0)
    inp = draw(shape, device="cuda")
    _, idx, w = MoeLayer(shape, inp).forward(inp["x"], routing=True)
    dy = torch.randn((shape.T, shape.H), generator=torch.Generator(device="cuda").manual_seed(5), device="cuda")
    d = _abi.desc_of(shape)
    ws = torch.empty(_abi.moe_backward_workspace_size(d), dtype=torch.uint8, device="cuda")
    E, H, I, Is, T = shape.E, shape.H, shape.I, shape.Is, shape.T
    outs = [torch.empty((T, H), device="cuda"), torch.empty((E, H), device="cuda"),
            torch.empty((E, 2 * I, H), device="cuda"), torch.empty((E, H, I), device="cuda"),
            torch.empty((2 * Is, H), device="cuda"), torch.empty((H, Is), device="cuda")]

    def step():
        _abi.moe_backward(d, inp["x"], inp["Wr"], inp["W_gate_up"], inp["W_down"], inp["Wsh_gate_up"],
                          inp["Wsh_down"], idx, w, dy, *outs, ws)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    _abi.moe_check_device()
    s0, s1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    uuid = str(torch.cuda.get_device_properties(0).uuid)
    sampler = ClockSampler(uuid if uuid.startswith("GPU-") else "GPU-" + uuid)
    sampler.start()
    s0.record()
    for _ in range(args.steps):
        step()
    s1.record()
    torch.cuda.synchronize()
    clocks = sampler.stop()
    _abi.moe_check_device()
    ms = s0.elapsed_time(s1) / args.steps
    flops = 16.0 * H * (I * T * shape.k + Is * T)
    wbytes = 4.0 * (E * 3 * I * H + 3 * Is * H)  # fp32 weight gradients written
    peaks, _ = load_peaks()
    line = {"metric": "MoE layer backward tokens/s on 1 B200", "value": T / (ms / 1e3), "unit": UNIT,
            "n_gpus": 1, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True,
            "dtype": "bf16", "data": "synthetic (seeded draw on device; random-init weights)",
            "config": workload_config(shape, {"pass": "backward", "routing": "router"}),
            "tensor": {"achieved_tflops": flops / (ms / 1e3) / 1e12,
                       "frac_of_bf16_peak": flops / (ms / 1e3) / 1e12 / peaks["bf16_tflops"]},
            "weight_grad_bytes": wbytes, "clocks": clocks}
    print(json.dumps(line), flush=True)


def main():
    args = parse()
    from sparse_moe_layer_biased_b200.inputs import WORKLOADS

    shape = WORKLOADS[args.workload]
    if args.tokens or args.experts:
        shape = shape.replace(name=f"{shape.name}_T{args.tokens or shape.T}_E{args.experts or shape.E}",
                              T=args.tokens or shape.T, E=args.experts or shape.E)
    if args.impl == "reference":
        run_reference(args, shape)
    elif args.which == "backward":
        run_backward(args, shape)
    elif args.which == "router":
        run_router_only(args, shape)
    elif args.parallel == "ep":
        run_ep(args, shape)
    else:
        run_b200(args, shape)


if __name__ == "__main__":
    main()
