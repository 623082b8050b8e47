"""Seeded synthetic inputs for the VDN-H3 linear branch.

This module only draws random tensors in the library's argument layout; it holds
none of the branch's arithmetic.  Both the CUDA path (tests, bench) and the CPU
oracle read the same host tensors produced here.

Workload shapes follow the latent grids of the 480p / 768p / 14 s / 1024^2 clips
(VAE 16x spatial, 4x temporal); the distributions are the ones listed with each
workload below.  Every tensor is drawn in float64 from its own counter-addressed
PCG64 streams (one stream per 2^22-element chunk, keyed by (seed, tensor id,
chunk index)), so the values do not depend on how many threads draw them, and
are then rounded once, round-to-nearest-even, to the run dtype.
"""
from __future__ import annotations

import dataclasses
import os
from concurrent.futures import ThreadPoolExecutor

import numpy as np
import torch

# draw order / stream ids
_Q, _K, _V, _BETA, _ALPHA, _GATE, _RMSW, _CONVK, _CONVV, _TEXT, _QR, _KR, _DOUT = range(13)
_CHUNK = 1 << 22

RULE_IDS = {"sana_scaled": 0, "vdn_solve": 1, "vdn_scaled": 2, "additive": 3}


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    B: int
    H: int
    d: int
    F: int
    S: int
    dtype: str            # "f32" or "bf16": element type of q, k, v, gate and out
    alpha_mu: float       # alpha = sigmoid(N(alpha_mu, 1))
    text: bool            # pass a text state
    seed: int
    conv_width: int = 3
    rule: str = "vdn_solve"
    c: float = 1.0
    chunk: int = 5
    radius: int = 1

    @property
    def N(self) -> int:
        return self.F * self.S

    @property
    def tokens(self) -> int:
        return self.B * self.F * self.S

    def replace(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)


WORKLOADS = {
    # B1 H2 d16 F10 S16 fp32; every window spans all 10 frames, so the output is exactly 0
    "tiny": Workload("tiny", 1, 2, 16, 10, 16, "f32", 2.0, False, 0),
    # the same with 20 frames (far field exists), without / with a text state
    "tiny_f20": Workload("tiny_f20", 1, 2, 16, 20, 16, "f32", 2.0, False, 0),
    "tiny_f20_text": Workload("tiny_f20_text", 1, 2, 16, 20, 16, "f32", 2.0, True, 0),
    # 480p 5 s: 31 latent frames of a 30x52 grid
    "480p": Workload("480p", 1, 24, 128, 31, 1560, "bf16", 2.0, True, 1),
    # 768p 5 s: 31 latent frames of a 48x84 grid
    "768p": Workload("768p", 1, 24, 128, 31, 4032, "bf16", 2.0, True, 2),
    # 14 s first/last-frame clip: 85 latent frames of a 30x52 grid, long memory
    "14s": Workload("14s", 1, 24, 128, 85, 1560, "bf16", 3.0, True, 3),
    # 1024^2: batch 2, 31 latent frames of a 64x64 grid (rule sweep workload)
    "1024sq": Workload("1024sq", 2, 24, 128, 31, 4096, "bf16", 2.0, True, 4),
}

# the rule sweep run on the 1024^2 workload: (rule, c, text)
RULE_SWEEP = [(r, c, t) for r in ("sana_scaled", "vdn_scaled") for c in (0.5, 1.0) for t in (False, True)] + \
             [("vdn_solve", 1.0, t) for t in (False, True)]


def _draw_chunk(args):
    seed, tid, idx, n, kind, mu, sd, out_dtype = args
    g = np.random.Generator(np.random.PCG64(np.random.SeedSequence([seed, tid, idx])))
    x = g.standard_normal(n) * sd + mu
    if kind == "sigmoid":
        x = 1.0 / (1.0 + np.exp(-x))
    t = torch.from_numpy(x)
    return t.to(out_dtype)


def _draw(seed: int, tid: int, shape, kind: str, mu: float, sd: float, dtype: torch.dtype,
          pool: ThreadPoolExecutor) -> torch.Tensor:
    n = int(np.prod(shape))
    jobs = [(seed, tid, i, min(_CHUNK, n - i * _CHUNK), kind, mu, sd, dtype)
            for i in range((n + _CHUNK - 1) // _CHUNK)]
    parts = list(pool.map(_draw_chunk, jobs)) if jobs else [torch.empty(0, dtype=dtype)]
    return torch.cat(parts).reshape(shape)


def make_inputs(w: Workload, *, threads: int | None = None, with_text: bool | None = None,
                with_rope_side: bool = False) -> dict:
    """Host (CPU) tensors in the library's argument layout.

    q, k, v, gate: [B, F*S, H, d] in the run dtype (token-major, heads interleaved)
    beta:          [B, F*S, H] float32, sigmoid(N(0,1))
    alpha:         [B, F, H, d] float32, sigmoid(N(alpha_mu, 1))
    rms_w:         [d] float32, 1 + 0.1 N(0,1)
    conv_k_w/v_w:  [H, d, K] float32, N(0, 1/K)   (None when K == 1: identity tap)
    text_state:    [H, d, d] float32, 0.5 * R with R ~ N(0, 0.1^2)   (None without text)
    q_rope, k_rope: [B, F*S, H, d] in the run dtype, N(0, 2^2) and N(0, 1) (only with
                   with_rope_side: the softmax branch's rotated q / k, drawn as independent
                   tensors; scores q.k / sqrt(d) then have standard deviation 2)
    """
    threads = threads or min(32, os.cpu_count() or 1)
    dt = torch.bfloat16 if w.dtype == "bf16" else torch.float32
    f32 = torch.float32
    B, H, d, F, S, N = w.B, w.H, w.d, w.F, w.S, w.N
    K = w.conv_width
    text = w.text if with_text is None else with_text
    with ThreadPoolExecutor(threads) as pool:
        out = {
            "q": _draw(w.seed, _Q, (B, N, H, d), "normal", 0.0, 1.0, dt, pool),
            "k": _draw(w.seed, _K, (B, N, H, d), "normal", 0.0, 1.0, dt, pool),
            "v": _draw(w.seed, _V, (B, N, H, d), "normal", 0.0, 1.0, dt, pool),
            "beta": _draw(w.seed, _BETA, (B, N, H), "sigmoid", 0.0, 1.0, f32, pool),
            "alpha": _draw(w.seed, _ALPHA, (B, F, H, d), "sigmoid", w.alpha_mu, 1.0, f32, pool),
            "gate": _draw(w.seed, _GATE, (B, N, H, d), "sigmoid", 0.0, 1.0, dt, pool),
            "rms_w": _draw(w.seed, _RMSW, (d,), "normal", 1.0, 0.1, f32, pool),
        }
        if K > 1:
            out["conv_k_w"] = _draw(w.seed, _CONVK, (H, d, K), "normal", 0.0, 1.0 / np.sqrt(K), f32, pool)
            out["conv_v_w"] = _draw(w.seed, _CONVV, (H, d, K), "normal", 0.0, 1.0 / np.sqrt(K), f32, pool)
        else:
            out["conv_k_w"] = None
            out["conv_v_w"] = None
        if text:
            out["text_state"] = (0.5 * _draw(w.seed, _TEXT, (H, d, d), "normal", 0.0, 0.1,
                                             torch.float64, pool)).to(f32)
        else:
            out["text_state"] = None
        if with_rope_side:
            out["q_rope"] = _draw(w.seed, _QR, (B, N, H, d), "normal", 0.0, 2.0, dt, pool)
            out["k_rope"] = _draw(w.seed, _KR, (B, N, H, d), "normal", 0.0, 1.0, dt, pool)
    return out


def make_cotangent(w: Workload, *, threads: int | None = None) -> torch.Tensor:
    """Upstream gradient dL/d out for the backward pass: N(0, 1) of the output's shape
    and dtype (the loss L = <dout, out>), from its own stream of the workload's seed."""
    dt = torch.bfloat16 if w.dtype == "bf16" else torch.float32
    with ThreadPoolExecutor(threads) as pool:
        return _draw(w.seed, _DOUT, (w.B, w.N, w.H, w.d), "normal", 0.0, 1.0, dt, pool)
