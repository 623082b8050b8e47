"""Benchmark of the VDN-H3 linear-branch forward on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload 768p] [--impl reference]
    python bench.py --path softmax|hybrid --steps 10 --warmup 3     # the windowed softmax branch / whole layer
    python bench.py --path backward --steps 5 --warmup 3            # gradients of the linear branch

One step is one vdn_branch_forward call over the whole workload (all heads,
all frames) with the inputs resident in HBM.  Prints ONE JSON line (rank 0):
latent tokens/s over all ranks, the roofline of the dominant kernel (live CUDA
event timing per kernel, algorithmic bytes / duration against the measured HBM
copy bandwidth), the whole-path roofline fraction, an end-to-end figure through
the same C ABI with host buffers, clocks sampled during the timed region, and
the float64 oracle timed on the host cores on a bounded sample.

Multi-GPU (torchrun, one rank per GPU): the branch needs no communication, each
rank runs its own clip (seed + 1000 * rank) of the same workload: weak scaling.

--path softmax times vdn_window_softmax_forward (the near-field branch over the
RoPE-side q/k) and --path hybrid times vdn_hybrid_forward (softmax branch plus
linear branch, the whole attention layer) on the same workload; their roofline is
the tensor-core one of the softmax kernel (algorithmic Q K^T and P V FLOPs over
the window's key tokens against the measured sustained bf16 GEMM rate).
"""
from __future__ import annotations

import argparse
import datetime
import hashlib
import json
import os
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import torch  # noqa: E402

from video_diffusion_linear_b200 import shard, synth  # noqa: E402

METRIC = "latent tokens/sec through VDN linear branch fwd (1 B200); % of roofline"
METRIC_PATH = {"backward": "latent tokens/sec through the VDN linear branch backward (forward recompute + "
                           "gradients of every input, 1 B200)",
               "softmax": "latent tokens/sec through the windowed softmax branch fwd (1 B200)",
               "hybrid": "latent tokens/sec through the VDN-H3 hybrid attention layer fwd (softmax + linear branch, 1 B200)",
               "features": "latent tokens/sec through the branch's Step 1 alone (conv, SiLU, L2 norm; 1 B200)"}
DEFAULT_WORKLOAD = "768p"
KERNELS_TC = ["frame_stats", "frame_solve", "scan", "gather", "readout"]
KERNEL_SOURCES = {"frame_stats": "tc_stats.cu", "frame_solve": "solve_gather.cu", "scan": "tc_scan.cu",
                  "gather": "solve_gather.cu", "readout": "tc_readout.cu", "window_softmax": "softmax.cu"}
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
REFERENCE_BUDGET_S = 150.0     # host time of a whole --impl reference run (warm-up + timed steps)


# ----------------------------------------------------------------------------- workload arithmetic
def describe(w: synth.Workload) -> str:
    txt = "with text state" if w.text else "no text state"
    return (f"{w.name}: B={w.B} H={w.H} d={w.d} F={w.F} S={w.S} ({w.tokens} latent tokens), {w.dtype}, "
            f"{w.rule} c={w.c}, chunk {w.chunk}, radius {w.radius}, {txt}")


def algorithmic_bytes(w: synth.Workload) -> dict:
    """Bytes each kernel must move at least once: the tokens it reads or writes once and the
    per-frame matrices (fp32 statistics, operand images, states) it exchanges with its neighbours."""
    d = w.d
    TH = w.B * w.F * w.S * w.H                 # token-heads
    NF = w.B * w.H * w.F                       # (batch, head, frame) triples
    mat = d * d * 4                            # one fp32 d x d matrix
    img = d * d * 2 * 2                        # bf16 hi/lo operand image of N_f
    wimg = d * d * 2                           # fp16 read-out operand image of W_t
    stored = 2 * w.B * w.H * (-(-w.F // w.chunk))   # chunk-boundary states written by the scan
    return {
        "frame_stats": TH * (2 * d * 2 + 4) + NF * 2 * mat,
        "frame_solve": NF * (2 * mat + mat + img),
        "scan": 2 * NF * (img + mat) + stored * mat,
        "gather": NF * (2 * mat + wimg),
        "readout": TH * 3 * d * 2 + NF * wimg,
    }


def path_roofline(w: synth.Workload, peaks: dict) -> dict:
    """Whole-branch roofline: algorithmic bytes (q, k, v, gate, beta in, out once;
    per frame alpha, the per-frame maps written and read once, chunk-boundary
    states) and FLOPs (A, B: 4 d^2 and read-out 2 d^2 per token-head, about
    7 d^3 per frame for the solve and the two scans)."""
    d = w.d
    TH = w.B * w.F * w.S * w.H
    NF = w.B * w.H * w.F
    states = 2 * w.B * w.H * (-(-w.F // w.chunk)) * d * d * 4 * 2
    nbytes = TH * (4 * d * 2 + 4 + d * 2) + NF * (d * 4 + 4 * d * d * 4) + states
    flops = TH * 6 * d * d + NF * 7 * d ** 3
    t_hbm = nbytes / (peaks["hbm_gbs"] * 1e9)
    t_tc = flops / (peaks["bf16_tflops"] * 1e12)
    return {"bytes": nbytes, "flops": flops, "t_roof_us": max(t_hbm, t_tc) * 1e6,
            "bound": "hbm" if t_hbm >= t_tc else "tensor"}


def softmax_flops(w: synth.Workload) -> float:
    """Algorithmic FLOPs of the windowed softmax branch: Q K^T and P V, 2 d each per
    (query, key) pair inside the query's window (exponentials not counted)."""
    pairs = 0
    for t in range(w.F):
        c = t // w.chunk
        lo = max(0, w.chunk * (c - w.radius))
        hi = min(w.F - 1, w.chunk * (c + w.radius + 1) - 1)
        pairs += w.S * (hi - lo + 1) * w.S
    return 4.0 * w.d * pairs * w.B * w.H


BWD_KERNELS = ["forward_recompute", "readout_bwd", "gather_bwd", "scan_bwd", "stats_bwd", "conv_bwd", "finish_bwd"]


def backward_flops(w: synth.Workload) -> dict:
    """Algorithmic FLOPs of the backward kernels that are contractions: the read-out's
    o = W q', dq' = W^T do and dW = sum do q'^T, and the statistics' (dA + dA^T) k',
    dB^T v', dB k' (2 d^2 each per token-head); the adjoint scans' two d x d products
    per frame and direction (2 d^3 each)."""
    TH = w.B * w.F * w.S * w.H
    NF = w.B * w.H * w.F
    return {"readout_bwd": 6.0 * w.d * w.d * TH, "stats_bwd": 6.0 * w.d * w.d * TH,
            "scan_bwd": 2 * 2 * 2.0 * w.d ** 3 * NF}


def backward_bytes(w: synth.Workload) -> dict:
    """Bytes each token-parallel backward kernel must move at least once (tokens and the
    conv-output gradients dk', dv' in the workload's element type, fp32 per-frame matrices):
      readout_bwd: q, gate, dout in, dq, dgate out (5 x d elements per token-head) + W_t in, dW_t out;
      stats_bwd:   k, v, beta in, dk', dv' and d beta out + dA, dB of both scans in;
      conv_bwd:    dk', dv', k, v in, dk, dv out."""
    d = w.d
    el = 2 if w.dtype == "bf16" else 4
    TH = w.B * w.F * w.S * w.H
    NF = w.B * w.H * w.F
    mat = d * d * 4
    return {"readout_bwd": 5 * el * d * TH + 2 * mat * NF,
            "stats_bwd": (2 * el * d + 4 + 2 * el * d + 4) * TH + 4 * mat * NF,
            "conv_bwd": 6 * el * d * TH}


def fp32_peak_tflops(sm_mhz: float) -> float:
    """FP32 FMA rate of the SIMT pipes: 148 SMs x 128 lanes x 2 FLOP per cycle."""
    return 148 * 128 * 2 * sm_mhz * 1e6 / 1e12


def load_peaks() -> tuple[dict, str]:
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            j = json.load(f)
        return {"hbm_gbs": float(j["hbm_gbs"]), "bf16_tflops": float(j["bf16_tflops"]),
                "bf16_tflops_sustained": float(j.get("bf16_tflops_sustained", j["bf16_tflops"]))}, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def source_hash(name: str) -> str:
    path = os.path.join(ROOT, "video_diffusion_linear_b200", "csrc", name)
    with open(path, "rb") as f:
        return hashlib.sha1(f.read()).hexdigest()[:12]


def recorded_traffic(kernel: str):
    """DRAM bytes per launch of `kernel` from the committed ncu summary
    (profiles/dram_traffic.txt: 'kernel workload source_sha1 bytes'), or None when
    absent or when the kernel's source changed since the capture."""
    path = os.path.join(ROOT, "profiles", "dram_traffic.txt")
    if not os.path.exists(path):
        return None
    with open(path) as f:
        for line in f:
            parts = line.split()
            if len(parts) >= 4 and parts[0] == kernel and not line.startswith("#"):
                if parts[2] == source_hash(KERNEL_SOURCES[kernel]):
                    return {"workload": parts[1], "bytes": float(parts[3])}
    return None


# ----------------------------------------------------------------------------- distributed helpers
def dist_env() -> tuple[int, int, int]:
    return int(os.environ.get("RANK", 0)), int(os.environ.get("WORLD_SIZE", 1)), int(os.environ.get("LOCAL_RANK", 0))


def rank_workload(w: synth.Workload, rank: int) -> synth.Workload:
    """Each rank runs its own clip of the workload (weak scaling, no exchange)."""
    return w.replace(seed=w.seed + 1000 * rank)


def rank_inputs(shard_mode: str, w: synth.Workload, world: int, rank: int, *, cotangent: bool = False, **make_kw):
    """The rank's host inputs: its own clip ("clips": weak scaling) or its contiguous share of the
    heads of the job's one clip ("heads": strong scaling; every rank draws the same clip).
    Returns (inputs, the rank's workload, latent tokens the whole job processes per step,
    the JSON line's scaling/global_batch/parallelism)."""
    if shard_mode == "heads":
        if world > w.H:
            raise SystemExit(f"--shard heads needs at most H = {w.H} ranks")
        full = synth.make_inputs(w, **make_kw)
        if cotangent:
            full["dout"] = synth.make_cotangent(w)
        host = shard.shard_inputs(full, world, rank)
        wr = w.replace(H=int(host["q"].shape[2]))
        h0, h1 = shard.head_range(w.H, world, 0)
        return host, wr, w.tokens, {"scaling": "strong", "global_batch": w.B,
                                    "parallelism": f"heads{world}: one clip, its {w.H} heads split across the "
                                                   f"GPUs ({h1 - h0} on the first), no exchange in the branch"}
    wr = rank_workload(w, rank)
    host = synth.make_inputs(wr, **make_kw)
    if cotangent:
        host["dout"] = synth.make_cotangent(wr)
    return host, wr, w.tokens * world, {"scaling": "weak", "global_batch": w.B * world,
                                        "parallelism": f"dp{world}: independent clips per GPU, no collective"}


def reduce_max(value: float, device=None) -> float:
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()):
        return value
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier(device=None):
    import torch.distributed as dist
    if dist.is_available() and dist.is_initialized():
        if device is not None and dist.get_backend() == "nccl":
            dist.barrier(device_ids=[device.index])
        else:
            dist.barrier()


# ----------------------------------------------------------------------------- clocks
class ClockSampler:
    """Samples SM clock and clock-event reasons through NVML every `period` s."""
    REASONS = {0x4: "sw_power_cap", 0x8: "hw_slowdown", 0x20: "sw_thermal_slowdown",
               0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown", 0x2: "applications_clocks_setting"}

    def __init__(self, device_index: int, period: float = 0.01):
        self.period = period
        self.samples = []
        self.reasons = set()
        self.max_mhz = None
        self._stop = threading.Event()
        self._h = None
        try:
            import pynvml
            pynvml.nvmlInit()
            self._nv = pynvml
            uuid = getattr(torch.cuda.get_device_properties(device_index), "uuid", None)
            h = None
            if uuid is not None:
                try:
                    h = pynvml.nvmlDeviceGetHandleByUUID(("GPU-" + str(uuid)).encode())
                except Exception:
                    h = None
            if h is None:
                h = pynvml.nvmlDeviceGetHandleByIndex(device_index)
            self._h = h
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(h, pynvml.NVML_CLOCK_SM)
        except Exception as e:  # NVML missing: report it instead of clocks
            self.error = str(e)

    def _run(self):
        nv = self._nv
        while not self._stop.is_set():
            try:
                self.samples.append(nv.nvmlDeviceGetClockInfo(self._h, nv.NVML_CLOCK_SM))
                fn = getattr(nv, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
                    getattr(nv, "nvmlDeviceGetCurrentClocksThrottleReasons")
                bits = fn(self._h)
                for b, name in self.REASONS.items():
                    if bits & b:
                        self.reasons.add(name)
            except Exception:
                pass
            time.sleep(self.period)

    def __enter__(self):
        if self._h is not None:
            self._t = threading.Thread(target=self._run, daemon=True)
            self._t.start()
        return self

    def __exit__(self, *a):
        if self._h is not None:
            self._stop.set()
            self._t.join()

    def summary(self) -> dict:
        if self._h is None:
            return {"error": getattr(self, "error", "nvml unavailable")}
        med = statistics.median(self.samples) if self.samples else None
        return {"sm_mhz": med, "sm_max_mhz": self.max_mhz, "reasons": sorted(self.reasons),
                "samples": len(self.samples)}


# ----------------------------------------------------------------------------- CPU oracle sample
def oracle_sample(inp: dict, w: synth.Workload, heads) -> tuple[float, int]:
    """Runs the float64 oracle over all frames and tokens of the given heads of
    batch 0; returns (seconds, token-heads processed)."""
    from oracle import vdn_oracle as O
    rms_w = O._f64(inp["rms_w"])
    t0 = time.perf_counter()
    for h in heads:
        st = O.head_state(inp, 0, h, w.F, w.S, w.rule, w.c, w.chunk, w.radius)
        g = O._f64(inp["gate"][0, :, h, :]).reshape(w.F, w.S, w.d)
        for t in range(w.F):
            O.readout(st["W"][t], st["qf"][t], g[t], rms_w)
    return time.perf_counter() - t0, len(heads) * w.F * w.S


def blas_threads() -> int:
    try:
        import threadpoolctl
        info = threadpoolctl.threadpool_info()
        blas = [i for i in info if i.get("user_api") == "blas"]
        if blas:
            return int(blas[0]["num_threads"])
    except Exception:
        pass
    return len(os.sched_getaffinity(0))


def softmax_oracle_sample(inp: dict, w: synth.Workload, n_tokens: int) -> tuple[float, int]:
    """Runs the float64 oracle's windowed softmax for n_tokens query tokens of
    (batch 0, head 0), spread over every frame; returns (seconds, token-heads)."""
    from oracle import vdn_oracle as O
    N = w.F * w.S
    toks = sorted(set(int(x) for x in torch.linspace(0, N - 1, n_tokens).round().tolist()))
    t0 = time.perf_counter()
    O.sampled_window_softmax(inp, w.F, w.S, w.chunk, w.radius, 0, 0, toks)
    return time.perf_counter() - t0, len(toks)


def run_reference(args, w: synth.Workload) -> None:
    rank, world, _ = dist_env()
    if rank != 0:
        return
    if args.path == "backward":
        return run_reference_backward(args, w)
    if args.path != "linear":
        return run_reference_softmax(args, w)
    # Each step runs the oracle over one head of a sub-clip: F_step whole frames (all S tokens each),
    # F_step sized so that all warm-up and timed steps take about REFERENCE_BUDGET_S.  Both parts of
    # the oracle's cost scale with the frames (per-token statistics and read-out, per-frame solves and
    # scan steps; the window gather is negligible), so a sub-clip's tokens/s is the clip's.
    wc = w.replace(H=1, F=min(w.F, 2))
    cal = synth.make_inputs(wc)
    oracle_sample(cal, wc, [0])                                   # first call: imports and allocations
    dt_c, _ = oracle_sample(cal, wc, [0])
    per_step = REFERENCE_BUDGET_S / (args.warmup + args.steps)
    f_step = int(min(w.F, max(1, round(wc.F * per_step / max(dt_c, 1e-6)))))
    ws = w.replace(H=1, F=f_step)
    inp = synth.make_inputs(ws)
    times = []
    th = 0
    for i in range(args.warmup + args.steps):
        dt, th = oracle_sample(inp, ws, [0])
        if i >= args.warmup:
            times.append(dt)
    step = sum(times) / len(times)
    tokens_equiv = th / w.H                    # one head of H: tokens x (1/H)
    value = tokens_equiv / step
    cores = blas_threads()
    sample = (f"one head of {w.H} per step over a {f_step}-frame sub-clip ({f_step} x {w.S} tokens, the same "
              f"distribution; the oracle's cost scales with the frames), batch 0; tokens counted x 1/H")
    print(json.dumps({
        "impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": step * 1e3, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": describe(w)},
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": cores, "kind": "oracle", "sample": sample},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }), flush=True)


def run_reference_softmax(args, w: synth.Workload) -> None:
    inp = synth.make_inputs(w, with_rope_side=True)
    times, th = [], 0
    for i in range(args.warmup + args.steps):
        dt_s, th_s = softmax_oracle_sample(inp, w, args.cpu_tokens)
        dt, th = dt_s, th_s
        if args.path == "hybrid":
            dt_l, th_l = oracle_sample(inp, w, [i % w.H])
            dt = dt_s + dt_l * th_s / th_l     # linear-branch cost of the same token-heads
        if i >= args.warmup:
            times.append(dt)
    step = sum(times) / len(times)
    value = (th / w.H) / step
    cores = blas_threads()
    sample = (f"{th} query tokens of head 0 (of {w.H}), batch 0, spread over all {w.F} frames, per step"
              + (" (+ the linear branch's per-token-head cost from one full head)" if args.path == "hybrid" else "")
              + "; tokens counted x 1/H")
    print(json.dumps({
        "impl": "reference", "metric": METRIC_PATH[args.path], "value": value, "unit": "tokens/s", "n_gpus": 1,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": step * 1e3, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": describe(w)},
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": cores, "kind": "oracle", "sample": sample},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }), flush=True)


def backward_oracle_sample(inp: dict, dout, w: synth.Workload, h: int) -> tuple[float, int]:
    """Runs the float64 backward oracle over one (batch 0, head h): all frames and tokens."""
    from oracle import vdn_backward as BW
    t0 = time.perf_counter()
    BW.head_backward(inp, 0, h, w.F, w.S, w.rule, w.c, w.chunk, w.radius, dout[0, :, h, :])
    return time.perf_counter() - t0, w.F * w.S


def run_reference_backward(args, w: synth.Workload) -> None:
    # one head per step over a sub-clip of whole frames, sized to the run's time budget as for the
    # forward's reference arm (the backward oracle's cost also scales with the frames)
    wc = w.replace(H=1, F=min(w.F, 2))
    cal, dcal = synth.make_inputs(wc), synth.make_cotangent(wc)
    backward_oracle_sample(cal, dcal, wc, 0)
    dt_c, _ = backward_oracle_sample(cal, dcal, wc, 0)
    per_step = REFERENCE_BUDGET_S / (args.warmup + args.steps)
    f_step = int(min(w.F, max(1, round(wc.F * per_step / max(dt_c, 1e-6)))))
    ws = w.replace(H=1, F=f_step)
    inp, dout = synth.make_inputs(ws), synth.make_cotangent(ws)
    times = []
    th = 0
    for i in range(args.warmup + args.steps):
        dt, th = backward_oracle_sample(inp, dout, ws, 0)
        if i >= args.warmup:
            times.append(dt)
    step = sum(times) / len(times)
    value = (th / w.H) / step
    sample = (f"one head of {w.H} per step over a {f_step}-frame sub-clip ({f_step} x {w.S} tokens), batch 0; "
              "tokens counted x 1/H")
    print(json.dumps({
        "impl": "reference", "metric": METRIC_PATH["backward"], "value": value, "unit": "tokens/s", "n_gpus": 1,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": step * 1e3, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": describe(w)},
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": blas_threads(), "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }), flush=True)


# ----------------------------------------------------------------------------- GPU arm
def run_gpu_backward(args, w: synth.Workload) -> None:
    """The branch's backward pass (vdn_branch_backward: forward recompute, then the
    gradients of every input) on one or more GPUs (independent clips per rank)."""
    from video_diffusion_linear_b200 import _lib, api
    rank, world, local = dist_env()
    device = torch.device("cuda", local)
    torch.cuda.set_device(device)
    if world > 1:
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300), device_id=device)
    _lib.load()
    host, wr, job_tokens, split = rank_inputs(args.shard, w, world, rank, cotangent=True)
    if args.shard == "heads" and world > 1:
        split["parallelism"] += "; NCCL all-reduce of the rms_w gradient (shared by every head) per step"
    dev = api.to_device(host, device)
    args_t = api.forward_inputs(dev)
    shape = api.shape_from(dev["q"], w.F, dev["conv_k_w"])
    ws = torch.empty(api.backward_workspace_size(shape, w.rule), dtype=torch.uint8, device=device)
    stream = torch.cuda.current_stream(device)
    # forward kernels + copies of its per-frame export (B, P, Q, W; SIMT also A, N) + backward kernels
    nfwd = api.launch_count(shape)
    launches = nfwd + (4 if nfwd == 5 else 6) + len(BWD_KERNELS) - 1
    grads = api.branch_backward(*args_t, dout=dev["dout"], F=w.F, rule=w.rule, c=w.c, chunk=w.chunk,
                                radius=w.radius, workspace=ws, stream=stream)

    def step(events=None):
        api.branch_backward(*args_t, dout=dev["dout"], F=w.F, rule=w.rule, c=w.c, chunk=w.chunk, radius=w.radius,
                            grads=grads, workspace=ws, stream=stream, events=events)
        if args.shard == "heads" and world > 1:
            shard.reduce_shared_grads(grads)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize(device)
    if api.workspace_status(ws) != 0:
        raise RuntimeError("device-side wait timed out during warm-up")
    nk = len(BWD_KERNELS)
    kev = [[torch.cuda.Event(enable_timing=True) for _ in range(nk + 1)] for _ in range(args.steps)]
    for evs in kev:
        for e in evs:
            e.record(stream)
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize(device)
    barrier(device)
    torch.cuda.synchronize(device)
    with ClockSampler(local) as clk:
        start.record(stream)
        for i in range(args.steps):
            step(kev[i])
        end.record(stream)
        torch.cuda.synchronize(device)
    barrier(device)
    torch.cuda.synchronize(device)
    ms = start.elapsed_time(end)
    ms_max = reduce_max(ms, device)
    value = job_tokens * args.steps / (ms_max / 1e3)
    per = {n: statistics.fmean(kev[i][j].elapsed_time(kev[i][j + 1]) for i in range(args.steps))
           for j, n in enumerate(BWD_KERNELS)}
    flops = backward_flops(wr)
    nbytes = backward_bytes(wr)
    bwd_only = {n: v for n, v in per.items() if n != "forward_recompute"}
    dom = max(bwd_only, key=bwd_only.get)
    csum = clk.summary()
    peaks, peak_src = load_peaks()
    if dom in nbytes:
        # the token-parallel kernels saturate neither the tensor pipe (their contractions are
        # small) nor the FP32 pipes: their bound is the bytes they must move
        achieved = nbytes[dom] / (per[dom] / 1e3) / 1e9
        roof = {"kernel": dom, "bound": "hbm", "achieved": achieved, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                "frac": achieved / peaks["hbm_gbs"], "peak_source": peak_src,
                "algorithmic_bytes_per_launch": nbytes[dom], "traffic": None}
    else:
        peak = fp32_peak_tflops(float(csum.get("sm_max_mhz") or 1965.0))
        achieved = flops[dom] / (per[dom] / 1e3) / 1e12 if dom in flops else None
        roof = {"kernel": dom, "bound": "alu", "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                "frac": achieved / peak if achieved else None,
                "peak_source": "derived: 148 SMs x 128 FP32 lanes x 2 FLOP x max SM clock (fp32 FMA)",
                "algorithmic_flops_per_launch": flops.get(dom), "traffic": None}
    kernels = {n: {"us": per[n] * 1e3, "share": per[n] / sum(per.values()),
                   "tflops": (flops[n] / (per[n] / 1e3) / 1e12) if n in flops else None,
                   "gbs": (nbytes[n] / (per[n] / 1e3) / 1e9) if n in nbytes else None} for n in per}

    e2e = None
    if not args.no_e2e:
        keys = ["q", "k", "v", "beta", "alpha", "gate", "dout"]
        pinned = {k: host[k].pin_memory() for k in keys}
        outs = ["dq", "dk", "dv", "dgate", "dbeta", "dalpha"]
        host_out = {k: torch.empty(grads[k].shape, dtype=grads[k].dtype).pin_memory() for k in outs}
        h2d = sum(pinned[k].numel() * pinned[k].element_size() for k in keys)
        d2h = sum(t.numel() * t.element_size() for t in host_out.values())
        n_e2e = max(1, min(args.steps, args.e2e_steps))
        torch.cuda.synchronize(device)
        barrier(device)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(n_e2e):
            for k in keys:
                dev[k].copy_(pinned[k], non_blocking=True)
            step()
            for k in outs:
                host_out[k].copy_(grads[k], non_blocking=True)
        e1.record(stream)
        torch.cuda.synchronize(device)
        e2e_ms = reduce_max(e0.elapsed_time(e1), device)
        e2e = {"value": job_tokens * n_e2e / (e2e_ms / 1e3), "unit": "tokens/s", "h2d_bytes_per_step": h2d,
               "d2h_bytes_per_step": d2h, "steps": n_e2e}

    cpu = None
    if rank == 0 and not args.no_cpu and world == 1:
        dt, th = backward_oracle_sample(host, host["dout"], w, 0)
        cpu = {"value": (th / w.H) / dt, "unit": "tokens/s", "cores": blas_threads(), "kind": "oracle",
               "sample": f"head 0 of {w.H}, batch 0, all {w.F} frames x {w.S} tokens ({dt:.1f} s); "
                         "tokens counted x 1/H"}

    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()
    if rank != 0:
        return
    print(json.dumps({
        "metric": METRIC_PATH["backward"], "value": value, "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_max / args.steps, "higher_is_better": True,
        "scaling": split["scaling"], "vs_baseline": None, "dtype": "f32 (bf16 inputs and gradients)",
        "data": "synthetic",
        "config": {"workload": describe(w) + ", upstream gradient N(0, 1)", "global_batch": split["global_batch"],
                   "tokens_per_step": job_tokens,
                   "l2": "inputs larger than L2 (q, k, v, gate, dout: %.2f GB per GPU)"
                         % (5 * wr.tokens * wr.H * wr.d * 2 / 1e9),
                   "parallelism": split["parallelism"]},
        "roofline": roof,
        "kernels": kernels,
        "cpu_baseline": cpu,
        "e2e": e2e,
        "gpu_launches": launches * args.steps,
        "clocks": csum,
    }), flush=True)


def run_gpu_softmax(args, w: synth.Workload) -> None:
    """The windowed softmax branch (--path softmax) or the whole hybrid layer
    (--path hybrid) on one or more GPUs (independent clips per rank)."""
    from video_diffusion_linear_b200 import _lib, api
    rank, world, local = dist_env()
    device = torch.device("cuda", local)
    torch.cuda.set_device(device)
    if world > 1:
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300), device_id=device)
    _lib.load()
    host, wr, job_tokens, split = rank_inputs(args.shard, w, world, rank, with_rope_side=True)
    dev = api.to_device(host, device)
    out = torch.empty_like(dev["q"])
    stream = torch.cuda.current_stream(device)
    hybrid = args.path == "hybrid"
    if hybrid:
        args_t = api.forward_inputs(dev)
        shape = api.shape_from(dev["q"], w.F, dev["conv_k_w"])
        ws = api.alloc_workspace(shape, w.rule, "auto", device)
        launches = api.launch_count(shape) + 1
    else:
        ws = torch.empty(256, dtype=torch.uint8, device=device)
        launches = 1

    def step():
        if hybrid:
            api.hybrid_forward(dev["q_rope"], dev["k_rope"], *args_t, F=w.F, rule=w.rule, c=w.c, chunk=w.chunk,
                               radius=w.radius, out=out, workspace=ws, stream=stream)
        else:
            api.window_softmax_forward(dev["q_rope"], dev["k_rope"], dev["v"], F=w.F, chunk=w.chunk,
                                       radius=w.radius, out=out, workspace=ws, stream=stream)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize(device)
    if api.workspace_status(ws) != 0:
        raise RuntimeError("device-side wait timed out during warm-up")
    # the softmax kernel alone, for the roofline of the dominant kernel (same stream, CUDA events)
    kev = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps + 1)]
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize(device)
    barrier(device)
    torch.cuda.synchronize(device)
    with ClockSampler(local) as clk:
        start.record(stream)
        for _ in range(args.steps):
            step()
        end.record(stream)
        torch.cuda.synchronize(device)
        if hybrid:
            kev[0].record(stream)
            for i in range(args.steps):
                api.window_softmax_forward(dev["q_rope"], dev["k_rope"], dev["v"], F=w.F, chunk=w.chunk,
                                           radius=w.radius, out=out, stream=stream)
                kev[i + 1].record(stream)
            torch.cuda.synchronize(device)
    barrier(device)
    torch.cuda.synchronize(device)
    if api.workspace_status(ws) != 0:
        raise RuntimeError("device-side wait timed out during the timed steps")
    ms = start.elapsed_time(end)
    ms_max = reduce_max(ms, device)
    value = job_tokens * args.steps / (ms_max / 1e3)
    soft_ms = (statistics.fmean(kev[i].elapsed_time(kev[i + 1]) for i in range(args.steps)) if hybrid
               else ms / args.steps)
    peaks, peak_src = load_peaks()
    flops = softmax_flops(wr)
    achieved = flops / (soft_ms / 1e3) / 1e12
    peak = peaks["bf16_tflops_sustained"]
    roof = {"kernel": "window_softmax", "bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
            "frac": achieved / peak, "peak_source": peak_src + " (sustained bf16 GEMM: the kernel runs ~0.1 s)",
            "algorithmic_flops_per_launch": flops, "traffic": recorded_traffic("window_softmax"),
            "us_per_launch": soft_ms * 1e3}
    if roof["traffic"] is not None:
        roof["traffic_workload"] = roof["traffic"]["workload"] + ("" if wr.H == w.H else
                                                                  f", scaled by {wr.H}/{w.H} heads")
        roof["traffic"] = roof["traffic"]["bytes"] * wr.H / w.H

    e2e = None
    if not args.no_e2e:
        keys = ["q_rope", "k_rope", "v"] + (["q", "k", "beta", "alpha", "gate"] if hybrid else [])
        pinned = {k: host[k].pin_memory() for k in keys}
        out_host = torch.empty(out.shape, dtype=out.dtype).pin_memory()
        h2d = sum(pinned[k].numel() * pinned[k].element_size() for k in keys)
        d2h = out_host.numel() * out_host.element_size()
        n_e2e = max(1, min(args.steps, args.e2e_steps))
        torch.cuda.synchronize(device)
        barrier(device)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(n_e2e):
            for k in keys:
                dev[k].copy_(pinned[k], non_blocking=True)
            step()
            out_host.copy_(out, non_blocking=True)
        e1.record(stream)
        torch.cuda.synchronize(device)
        e2e_ms = reduce_max(e0.elapsed_time(e1), device)
        e2e = {"value": job_tokens * n_e2e / (e2e_ms / 1e3), "unit": "tokens/s", "h2d_bytes_per_step": h2d,
               "d2h_bytes_per_step": d2h, "steps": n_e2e}

    cpu = None
    if rank == 0 and not args.no_cpu and world == 1:
        dt, th = softmax_oracle_sample(host, w, args.cpu_tokens)
        sample = f"{th} query tokens of head 0 (of {w.H}), batch 0, over all {w.F} frames ({dt:.1f} s)"
        if hybrid:
            dl, tl = oracle_sample(host, w, [0])
            dt += dl * th / tl
            sample += f" + the linear branch's per-token-head cost from head 0 ({dl:.1f} s)"
        cpu = {"value": (th / w.H) / dt, "unit": "tokens/s", "cores": blas_threads(), "kind": "oracle",
               "sample": sample + "; tokens counted x 1/H"}

    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()
    if rank != 0:
        return
    print(json.dumps({
        "metric": METRIC_PATH[args.path], "value": value, "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_max / args.steps, "higher_is_better": True,
        "scaling": split["scaling"], "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": describe(w) + f", softmax window = chunk {w.chunk} +- {w.radius} chunks, "
                   "scale 1/sqrt(d)", "global_batch": split["global_batch"], "tokens_per_step": job_tokens,
                   "l2": "inputs larger than L2 (q_rope, k_rope, v: %.2f GB per GPU)"
                         % (3 * wr.tokens * wr.H * wr.d * 2 / 1e9),
                   "parallelism": split["parallelism"]},
        "roofline": roof,
        "cpu_baseline": cpu,
        "e2e": e2e,
        "gpu_launches": launches * args.steps,
        "clocks": clk.summary(),
    }), flush=True)


def run_gpu_features(args, w: synth.Workload) -> None:
    """Step 1 alone (--path features): vdn_feature_prep over the workload's q, k, v, writing
    q', k', v'.  A streaming kernel: its roofline is HBM, with algorithmic bytes = q, k, v read
    once and q', k', v' written once (6 x d x 2 B per token-head in bf16)."""
    from video_diffusion_linear_b200 import _lib, api
    rank, world, local = dist_env()
    device = torch.device("cuda", local)
    torch.cuda.set_device(device)
    if world > 1:
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300), device_id=device)
    _lib.load()
    host, wr, job_tokens, split = rank_inputs(args.shard, w, world, rank)
    dev = api.to_device(host, device)
    stream = torch.cuda.current_stream(device)
    outs = tuple(torch.empty_like(dev[k]) for k in ("q", "k", "v"))

    def step():
        api.feature_prep(dev["q"], dev["k"], dev["v"], dev["conv_k_w"], dev["conv_v_w"], F=wr.F, stream=stream,
                         out=outs)

    for _ in range(args.warmup):
        step()
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize(device)
    barrier(device)
    torch.cuda.synchronize(device)
    with ClockSampler(local) as clk:
        start.record(stream)
        for _ in range(args.steps):
            step()
        end.record(stream)
        torch.cuda.synchronize(device)
    barrier(device)
    torch.cuda.synchronize(device)
    ms = start.elapsed_time(end)
    ms_max = reduce_max(ms, device)
    value = job_tokens * args.steps / (ms_max / 1e3)
    peaks, peak_src = load_peaks()
    TH = wr.B * wr.F * wr.S * wr.H
    nbytes = 6 * wr.d * (2 if wr.dtype == "bf16" else 4) * TH
    us = ms / args.steps * 1e3
    achieved = nbytes / (us / 1e6) / 1e9
    roof = {"kernel": "feature_prep", "bound": "hbm", "achieved": achieved, "peak": peaks["hbm_gbs"], "unit": "GB/s",
            "frac": achieved / peaks["hbm_gbs"], "peak_source": peak_src, "algorithmic_bytes_per_launch": nbytes,
            "traffic": None, "us_per_launch": us}

    e2e = None
    if not args.no_e2e:
        keys = ["q", "k", "v"]
        pinned = {k: host[k].pin_memory() for k in keys}
        outs_host = tuple(torch.empty(o.shape, dtype=o.dtype).pin_memory() for o in outs)
        h2d = sum(pinned[k].numel() * pinned[k].element_size() for k in keys)
        d2h = sum(o.numel() * o.element_size() for o in outs_host)
        n_e2e = max(1, min(args.steps, args.e2e_steps))
        torch.cuda.synchronize(device)
        barrier(device)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(n_e2e):
            for k in keys:
                dev[k].copy_(pinned[k], non_blocking=True)
            step()
            for oh, o in zip(outs_host, outs):
                oh.copy_(o, non_blocking=True)
        e1.record(stream)
        torch.cuda.synchronize(device)
        e2e_ms = reduce_max(e0.elapsed_time(e1), device)
        e2e = {"value": job_tokens * n_e2e / (e2e_ms / 1e3), "unit": "tokens/s", "h2d_bytes_per_step": h2d,
               "d2h_bytes_per_step": d2h, "steps": n_e2e}

    cpu = None
    if rank == 0 and not args.no_cpu and world == 1:
        from oracle import vdn_oracle as O
        heads = list(range(min(args.cpu_heads, w.H)))
        t0 = time.perf_counter()
        for h in heads:
            O.prepare_features(O._f64(host["q"][0, :, h]), O._f64(host["k"][0, :, h]), O._f64(host["v"][0, :, h]),
                               w.F, w.S, None if host["conv_k_w"] is None else O._f64(host["conv_k_w"][h]),
                               None if host["conv_v_w"] is None else O._f64(host["conv_v_w"][h]))
        dt = time.perf_counter() - t0
        cpu = {"value": len(heads) * w.F * w.S / w.H / dt, "unit": "tokens/s", "cores": blas_threads(),
               "kind": "oracle", "sample": f"heads 0..{len(heads) - 1} of {w.H}, batch 0, all {w.F} frames x {w.S} "
                                           f"tokens ({dt:.1f} s); tokens counted x heads/H"}

    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()
    if rank != 0:
        return
    print(json.dumps({
        "metric": METRIC_PATH["features"], "value": value, "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_max / args.steps, "higher_is_better": True,
        "scaling": split["scaling"], "vs_baseline": None, "dtype": wr.dtype, "data": "synthetic",
        "config": {"workload": describe(w) + "; Step 1 only (conv, SiLU, L2 norm of q and k)",
                   "global_batch": split["global_batch"], "tokens_per_step": job_tokens,
                   "l2": "inputs larger than L2 (q, k, v: %.2f GB per GPU)" % (3 * wr.tokens * wr.H * wr.d * 2 / 1e9),
                   "parallelism": split["parallelism"]},
        "roofline": roof,
        "cpu_baseline": cpu,
        "e2e": e2e,
        "gpu_launches": args.steps,
        "clocks": clk.summary(),
    }), flush=True)


def run_gpu_frames(args, w: synth.Workload) -> None:
    """The linear branch of ONE clip split by frames across the ranks (strong scaling): each rank
    writes the affine maps of its chunks, one all-gather gives every rank every map, and each rank
    folds them, gathers and reads out its own frames (the step shard.frame_sharded_forward runs).
    Per-kernel events are not recorded in this mode: the roofline is the rank's share of the path."""
    from video_diffusion_linear_b200 import _lib, api
    rank, world, local = dist_env()
    device = torch.device("cuda", local)
    torch.cuda.set_device(device)
    if world > 1:
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300), device_id=device)
    _lib.load()
    if world > -(-w.F // w.chunk):
        raise SystemExit(f"--shard frames needs at most {-(-w.F // w.chunk)} ranks (one chunk each)")
    if w.dtype != "bf16" or w.d != 128 or w.chunk > 16:
        raise SystemExit("--shard frames runs the tensor-core path: bf16, d = 128, chunk <= 16")
    host = shard.frame_inputs(synth.make_inputs(w), w.F, world, rank, w.chunk)
    f0, f1 = shard.frame_range(w.F, world, rank, w.chunk)
    wr = w.replace(F=f1 - f0)
    dev = api.to_device(host, device)
    stream = torch.cuda.current_stream(device)
    shape = api.shape_from(dev["q"], wr.F, dev["conv_k_w"])
    ws = torch.empty(api.frames_workspace_size(shape, w.F, world, rank, w.rule, w.chunk), dtype=torch.uint8,
                     device=device)
    nmap = api.frames_map_bytes(shape, w.F, world, rank, w.chunk) // 4
    maps = torch.empty(nmap, dtype=torch.float32, device=device)
    maps_all = torch.empty(world * nmap, dtype=torch.float32, device=device) if world > 1 else maps
    out = torch.empty_like(dev["q"])
    kw = dict(F_total=w.F, world=world, rank=rank, rule=w.rule, c=w.c, chunk=w.chunk, workspace=ws, stream=stream)

    def step():
        api.frames_maps(dev["k"], dev["v"], dev["beta"], dev["alpha"], dev["conv_k_w"], dev["conv_v_w"], maps=maps,
                        **kw)
        if world > 1:
            dist.all_gather_into_tensor(maps_all, maps)
        api.frames_finish(dev["q"], dev["alpha_all"], dev["gate"], dev["rms_w"], dev["text_state"], maps_all,
                          radius=w.radius, out=out, **kw)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize(device)
    if api.workspace_status(ws) != 0:
        raise RuntimeError("device-side wait timed out during warm-up")
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize(device)
    barrier(device)
    torch.cuda.synchronize(device)
    with ClockSampler(local) as clk:
        start.record(stream)
        for _ in range(args.steps):
            step()
        end.record(stream)
        torch.cuda.synchronize(device)
    barrier(device)
    torch.cuda.synchronize(device)
    ms_max = reduce_max(start.elapsed_time(end), device)
    value = w.tokens * args.steps / (ms_max / 1e3)
    peaks, peak_src = load_peaks()
    pr = path_roofline(wr, peaks)
    step_us = ms_max / args.steps * 1e3
    achieved = pr["bytes"] / (step_us / 1e6) / 1e9
    roof = {"kernel": "whole path, this rank's frames (per-kernel events not recorded with --shard frames)",
            "bound": "hbm", "achieved": achieved, "peak": peaks["hbm_gbs"], "unit": "GB/s",
            "frac": achieved / peaks["hbm_gbs"], "peak_source": peak_src,
            "algorithmic_bytes_per_launch": pr["bytes"], "traffic": None}

    e2e = None
    if not args.no_e2e:
        keys = ["q", "k", "v", "beta", "alpha", "alpha_all", "gate"]
        pinned = {k: host[k].pin_memory() for k in keys}
        out_host = torch.empty(out.shape, dtype=out.dtype).pin_memory()
        h2d = sum(pinned[k].numel() * pinned[k].element_size() for k in keys)
        d2h = out_host.numel() * out_host.element_size()
        n_e2e = max(1, min(args.steps, args.e2e_steps))
        torch.cuda.synchronize(device)
        barrier(device)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(n_e2e):
            for k in keys:
                dev[k].copy_(pinned[k], non_blocking=True)
            step()
            out_host.copy_(out, non_blocking=True)
        e1.record(stream)
        torch.cuda.synchronize(device)
        e2e_ms = reduce_max(e0.elapsed_time(e1), device)
        e2e = {"value": w.tokens * n_e2e / (e2e_ms / 1e3), "unit": "tokens/s", "h2d_bytes_per_step": h2d,
               "d2h_bytes_per_step": d2h, "steps": n_e2e}

    if world > 1:
        dist.destroy_process_group()
    if rank != 0:
        return
    print(json.dumps({
        "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_max / args.steps, "higher_is_better": True, "scaling": "strong",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": describe(w), "global_batch": w.B, "tokens_per_step": w.tokens,
                   "l2": "inputs larger than L2 (q, k, v, gate: %.2f GB per step per GPU)"
                         % (4 * wr.tokens * wr.H * wr.d * 2 / 1e9),
                   "parallelism": f"frames{world}: one clip, frames {f0}..{f1 - 1} on rank 0 of {world}, one "
                                  "all-gather of per-chunk maps per step"},
        "roofline": roof,
        "path_roofline": {"t_roof_us": pr["t_roof_us"], "t_step_us": step_us, "frac": pr["t_roof_us"] / step_us,
                          "bound": pr["bound"], "peaks": peaks, "peak_source": peak_src},
        "cpu_baseline": None,
        "e2e": e2e,
        "gpu_launches": 7 * args.steps,
        "clocks": clk.summary(),
    }), flush=True)


def run_gpu(args, w: synth.Workload) -> None:
    from video_diffusion_linear_b200 import _lib, api
    rank, world, local = dist_env()
    device = torch.device("cuda", local)
    torch.cuda.set_device(device)
    if world > 1:
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300), device_id=device)
    _lib.load()
    host, wr, job_tokens, split = rank_inputs(args.shard, w, world, rank)
    dev = api.to_device(host, device)
    args_t = api.forward_inputs(dev)
    shape = api.shape_from(dev["q"], w.F, dev["conv_k_w"])
    ws = api.alloc_workspace(shape, w.rule, "auto", device)
    out = torch.empty_like(dev["q"])
    nl = api.launch_count(shape)
    stream = torch.cuda.current_stream(device)

    def step(events=None):
        if events is None:
            api.branch_forward(*args_t, F=w.F, rule=w.rule, c=w.c, chunk=w.chunk, radius=w.radius, out=out,
                               workspace=ws, stream=stream)
        else:
            api.branch_forward_timed(*args_t, F=w.F, rule=w.rule, c=w.c, chunk=w.chunk, radius=w.radius,
                                     out=out, workspace=ws, stream=stream, events=events)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize(device)
    if api.workspace_status(ws) != 0:
        raise RuntimeError("device-side wait timed out during warm-up")

    # per-kernel events for every timed step (recorded once so their handles exist)
    kev = [[torch.cuda.Event(enable_timing=True) for _ in range(nl + 1)] for _ in range(args.steps)]
    for evs in kev:
        for e in evs:
            e.record(stream)
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize(device)
    barrier(device)
    torch.cuda.synchronize(device)
    with ClockSampler(local) as clk:
        start.record(stream)
        for i in range(args.steps):
            step(kev[i])
        end.record(stream)
        torch.cuda.synchronize(device)
    barrier(device)
    torch.cuda.synchronize(device)
    ms = start.elapsed_time(end)
    ms_max = reduce_max(ms, device)
    tokens = job_tokens * args.steps
    value = tokens / (ms_max / 1e3)

    names = KERNELS_TC if nl == 5 else [f"kernel{i}" for i in range(nl)]
    per = {n: statistics.fmean(kev[i][j].elapsed_time(kev[i][j + 1]) for i in range(args.steps))
           for j, n in enumerate(names)}
    peaks, peak_src = load_peaks()
    alg = algorithmic_bytes(wr)
    dom = max(per, key=per.get)
    dom_ms = per[dom]
    achieved = alg.get(dom, 0) / (dom_ms / 1e3) / 1e9 if dom in alg else None
    traffic = recorded_traffic(dom)
    roof = {"kernel": dom, "bound": "hbm", "achieved": achieved, "peak": peaks["hbm_gbs"], "unit": "GB/s",
            "frac": (achieved / peaks["hbm_gbs"]) if achieved else None, "peak_source": peak_src,
            "algorithmic_bytes_per_launch": alg.get(dom),
            "traffic": traffic["bytes"] * wr.H / w.H if traffic else None,   # units scale with the heads
            "traffic_workload": (traffic["workload"] + ("" if wr.H == w.H else f", scaled by {wr.H}/{w.H} heads"))
                                if traffic else None}
    pr = path_roofline(wr, peaks)
    step_us = ms_max / args.steps * 1e3
    kernels = {n: {"us": per[n] * 1e3, "share": per[n] / sum(per.values()),
                   "gbs": (alg[n] / (per[n] / 1e3) / 1e9) if n in alg else None} for n in per}

    # end to end through the same C ABI: pinned host inputs in, result out, every step
    e2e = None
    if not args.no_e2e:
        keys = ["q", "k", "v", "beta", "alpha", "gate"]
        pinned = {k: host[k].pin_memory() for k in keys}
        out_host = torch.empty(out.shape, dtype=out.dtype).pin_memory()
        h2d = sum(pinned[k].numel() * pinned[k].element_size() for k in keys)
        d2h = out_host.numel() * out_host.element_size()
        n_e2e = max(1, min(args.steps, args.e2e_steps))
        for _ in range(2):
            for k in keys:
                dev[k].copy_(pinned[k], non_blocking=True)
            step()
            out_host.copy_(out, non_blocking=True)
        torch.cuda.synchronize(device)
        barrier(device)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(n_e2e):
            for k in keys:
                dev[k].copy_(pinned[k], non_blocking=True)
            step()
            out_host.copy_(out, non_blocking=True)
        e1.record(stream)
        torch.cuda.synchronize(device)
        e2e_ms = reduce_max(e0.elapsed_time(e1), device)
        e2e = {"value": job_tokens * n_e2e / (e2e_ms / 1e3), "unit": "tokens/s", "h2d_bytes_per_step": h2d,
               "d2h_bytes_per_step": d2h, "steps": n_e2e}

    cpu = None
    if rank == 0 and not args.no_cpu and world == 1:
        heads = list(range(min(w.H, args.cpu_heads)))
        dt, th = oracle_sample(host, w, heads)
        cpu = {"value": (th / w.H) / dt, "unit": "tokens/s", "cores": blas_threads(), "kind": "oracle",
               "sample": f"heads 0..{len(heads) - 1} of {w.H}, batch 0, all {w.F} frames x {w.S} tokens "
                         f"({dt:.1f} s); tokens counted x heads/H"}

    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()
    if rank != 0:
        return
    line = {
        "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_max / args.steps, "higher_is_better": True,
        "scaling": split["scaling"], "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": describe(w), "global_batch": split["global_batch"], "tokens_per_step": job_tokens,
                   "l2": "inputs larger than L2 (q, k, v, gate: %.2f GB per step per GPU)"
                         % (4 * wr.tokens * wr.H * wr.d * 2 / 1e9),
                   "parallelism": split["parallelism"]},
        "roofline": roof,
        "path_roofline": {"t_roof_us": pr["t_roof_us"], "t_step_us": step_us, "frac": pr["t_roof_us"] / step_us,
                          "bound": pr["bound"], "algorithmic_bytes": pr["bytes"], "flops": pr["flops"],
                          "peaks": peaks, "peak_source": peak_src},
        "kernels": kernels,
        "cpu_baseline": cpu,
        "e2e": e2e,
        "gpu_launches": nl * args.steps,
        "clocks": clk.summary(),
    }
    print(json.dumps(line), flush=True)


def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=300)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD, choices=sorted(synth.WORKLOADS))
    ap.add_argument("--rule", default=None)
    ap.add_argument("--c", type=float, default=None)
    ap.add_argument("--impl", default="b200", choices=["b200", "reference"])
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--e2e-steps", type=int, default=5)
    ap.add_argument("--no-cpu", action="store_true")
    ap.add_argument("--cpu-heads", type=int, default=2)
    ap.add_argument("--heads", type=int, default=None, help="override H (smaller profiling captures)")
    ap.add_argument("--path", default="linear", choices=["linear", "softmax", "hybrid", "backward", "features"],
                    help="linear branch (default), windowed softmax branch, the whole hybrid layer, the "
                         "linear branch's backward pass, or its Step 1 alone (vdn_feature_prep)")
    ap.add_argument("--cpu-tokens", type=int, default=256, help="query tokens in the softmax oracle sample")
    ap.add_argument("--shard", default="clips", choices=["clips", "heads", "frames"],
                    help="multi-GPU: independent clips per rank (weak scaling, default), one clip with its "
                         "heads split across the ranks, or (linear path) one clip split by frames (strong scaling)")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        ap.error("--warmup must be at least 3")
    if args.shard != "clips" and args.impl == "reference":
        ap.error("--shard applies to the GPU arm")
    if args.shard == "frames" and args.path != "linear":
        ap.error("--shard frames applies to the linear branch path")
    w = synth.WORKLOADS[args.workload]
    if args.rule:
        w = w.replace(rule=args.rule)
    if args.c is not None:
        w = w.replace(c=args.c)
    if args.heads:
        w = w.replace(H=args.heads)
    if args.path == "features" and (args.impl == "reference" or args.shard == "frames"):
        ap.error("--path features runs the GPU arm with --shard clips or heads")
    if args.impl == "reference":
        run_reference(args, w)
    elif args.path == "features":
        run_gpu_features(args, w)
    elif args.path == "backward":
        run_gpu_backward(args, w)
    elif args.path != "linear":
        run_gpu_softmax(args, w)
    elif args.shard == "frames":
        run_gpu_frames(args, w)
    else:
        run_gpu(args, w)


if __name__ == "__main__":
    main()
