"""Shared helpers of the GPU tests: run the library and the oracle on the same
seeded inputs and compare them."""
from __future__ import annotations

import numpy as np
import torch

from oracle import vdn_oracle as O
from video_diffusion_linear_b200 import api, synth

TOL_F32 = 1e-4     # max |gpu - ref| / max |ref|, fp32 inputs and outputs
TOL_BF16 = 2e-2    # same, bf16 inputs and outputs with fp32 state and accumulation


def rel_err(got, ref) -> float:
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    denom = np.abs(ref).max()
    num = np.abs(got - ref).max()
    if denom == 0:
        return float(num)
    return float(num / denom)


def gpu_forward(w: synth.Workload, inp: dict, rule=None, c=None, impl="auto", debug=False, want=api.DEBUG_FIELDS):
    dev = api.to_device(inp)
    rule = rule or w.rule
    c = w.c if c is None else c
    args = api.forward_inputs(dev)
    if debug:
        out, mats = api.branch_forward_debug(*args, F=w.F, rule=rule, c=c, chunk=w.chunk, radius=w.radius,
                                             impl=impl, want=want)
    else:
        out, mats = api.branch_forward(*args, F=w.F, rule=rule, c=c, chunk=w.chunk, radius=w.radius), {}
    torch.cuda.synchronize()
    return out, mats


def oracle_forward(w: synth.Workload, inp: dict, rule=None, c=None, heads=None, batches=None):
    rule = rule or w.rule
    c = w.c if c is None else c
    return O.branch_forward(inp, w.F, w.S, rule, c, w.chunk, w.radius, heads=heads, batches=batches)


def to_np(t: torch.Tensor) -> np.ndarray:
    return t.detach().float().cpu().numpy().astype(np.float64)
