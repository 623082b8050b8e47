"""Parity of the windowed softmax branch and of the hybrid layer (softmax branch
plus linear branch) with the float64 oracle, through the C ABI: the SIMT path
(fp32, d = 16 and 128) and the tensor-core path (bf16, d = 128), ragged tiles
(S not a multiple of 128), windows clipped at both clip ends, a last chunk
shorter than the others, accumulation into an existing output, run-to-run
determinism, and sampled tokens at the 480p size."""
import numpy as np
import pytest
import torch

from harness import TOL_BF16, TOL_F32, rel_err, to_np
from oracle import vdn_oracle as O
from video_diffusion_linear_b200 import api, synth

pytestmark = pytest.mark.gpu


def _run(w, inp, accumulate=False, base=None, scale=0.0):
    dev = api.to_device(inp)
    out = None
    if accumulate:
        out = torch.from_numpy(np.asarray(base)).to(dev["q_rope"].dtype).cuda()
    ws = torch.empty(256, dtype=torch.uint8, device="cuda")
    out = api.window_softmax_forward(dev["q_rope"], dev["k_rope"], dev["v"], F=w.F, chunk=w.chunk, radius=w.radius,
                                     scale=scale, accumulate=accumulate, out=out, workspace=ws)
    torch.cuda.synchronize()
    assert api.workspace_status(ws) == 0          # no bounded wait expired
    return out


CASES = [
    synth.Workload("sm_tiny", B=1, H=2, d=16, F=10, S=16, dtype="f32", alpha_mu=2.0, text=False, seed=40),
    synth.Workload("sm_f32_d128", B=1, H=2, d=128, F=7, S=40, dtype="f32", alpha_mu=2.0, text=False, seed=41, chunk=3),
    synth.Workload("sm_bf16_ragged", B=2, H=2, d=128, F=12, S=200, dtype="bf16", alpha_mu=2.0, text=False, seed=42),
    synth.Workload("sm_bf16_short_window", B=1, H=3, d=128, F=9, S=24, dtype="bf16", alpha_mu=2.0, text=False, seed=43, chunk=2, radius=0),
    synth.Workload("sm_bf16_wide", B=1, H=1, d=128, F=11, S=128, dtype="bf16", alpha_mu=2.0, text=False, seed=44, chunk=4, radius=2),
]


@pytest.mark.parametrize("w", CASES, ids=[c.name for c in CASES])
def test_window_softmax_matches_oracle(w):
    inp = synth.make_inputs(w, with_rope_side=True)
    got = _run(w, inp)
    ref = O.window_softmax_forward(inp, w.F, w.S, w.chunk, w.radius)
    tol = TOL_F32 if w.dtype == "f32" else TOL_BF16
    assert rel_err(to_np(got), ref) <= tol, (w.name, rel_err(to_np(got), ref))


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_explicit_scale_and_accumulate(dtype):
    w = synth.Workload("sm_acc", B=1, H=2, d=128, F=6, S=64, dtype=dtype, alpha_mu=2.0, text=False, seed=45, chunk=3)
    inp = synth.make_inputs(w, with_rope_side=True)
    rng = np.random.default_rng(0)
    base = rng.normal(size=tuple(inp["q"].shape)).astype(np.float32)
    base_t = torch.from_numpy(base).to(inp["q"].dtype)
    got = _run(w, inp, accumulate=True, base=base_t.float().numpy(), scale=0.05)
    ref = O.window_softmax_forward(inp, w.F, w.S, w.chunk, w.radius, scale=0.05) + base_t.double().numpy()
    tol = TOL_F32 if dtype == "f32" else TOL_BF16
    assert rel_err(to_np(got), ref) <= tol


def test_run_to_run_bitwise():
    w = CASES[2]
    inp = synth.make_inputs(w, with_rope_side=True)
    a = _run(w, inp)
    b = _run(w, inp)
    assert torch.equal(a, b)


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_hybrid_layer_matches_oracle(dtype):
    w = synth.Workload("hyb", B=1, H=2, d=128, F=12, S=48, dtype=dtype, alpha_mu=2.0, seed=46, text=True)
    inp = synth.make_inputs(w, with_rope_side=True)
    dev = api.to_device(inp)
    out = api.hybrid_forward(dev["q_rope"], dev["k_rope"], *api.forward_inputs(dev), F=w.F, rule=w.rule, c=w.c,
                             chunk=w.chunk, radius=w.radius)
    torch.cuda.synchronize()
    ref = O.hybrid_forward(inp, w.F, w.S, w.rule, w.c, w.chunk, w.radius)
    tol = TOL_F32 if dtype == "f32" else TOL_BF16
    assert rel_err(to_np(out), ref) <= tol


def test_480p_sampled_tokens():
    w = synth.WORKLOADS["480p"]
    inp = synth.make_inputs(w, with_rope_side=True)
    got = _run(w, inp)
    rng = np.random.default_rng(w.seed)
    for b, h in [(0, 0), (0, w.H - 1)]:
        toks = []
        for t in range(w.F):
            toks += [t * w.S, t * w.S + w.S - 1] + list(t * w.S + rng.integers(0, w.S, size=3))
        toks = np.array(sorted(set(toks)))
        ref = O.sampled_window_softmax(inp, w.F, w.S, w.chunk, w.radius, b, h, toks)
        g = got[b, torch.as_tensor(toks, device=got.device), h, :].float().cpu().numpy().astype(np.float64)
        assert rel_err(g, ref) <= TOL_BF16, (b, h, rel_err(g, ref))
    assert torch.isfinite(got.float()).all()


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_scores_rising_along_the_window(dtype):
    # key norms grow along the sequence, so a row's running maximum keeps rising from key
    # tile to key tile: the tensor-core path must bring O and the normaliser to each new
    # reference maximum (and stays exact when it does not move)
    w = synth.Workload("sm_rising", B=1, H=2, d=128, F=10, S=96, dtype=dtype, alpha_mu=2.0, text=False, seed=47,
                       chunk=5, radius=1)
    inp = synth.make_inputs(w, with_rope_side=True)
    N = w.F * w.S
    ramp = torch.linspace(0.2, 6.0, N, dtype=torch.float64).view(1, N, 1, 1)
    inp["k_rope"] = (inp["k_rope"].double() * ramp).to(inp["k_rope"].dtype)
    got = _run(w, inp)
    ref = O.window_softmax_forward(inp, w.F, w.S, w.chunk, w.radius)
    tol = TOL_F32 if dtype == "f32" else TOL_BF16
    assert rel_err(to_np(got), ref) <= tol, rel_err(to_np(got), ref)


def test_repeated_full_size_calls_never_time_out():
    # every barrier of the tensor-core kernel has to hold under real scheduling skew between
    # its warps: a lost or doubled arrival shows up as an expired bounded wait (status word)
    # or as a run that differs from the first
    w = synth.WORKLOADS["480p"]
    dev = api.to_device(synth.make_inputs(w, with_rope_side=True))
    ws = torch.empty(256, dtype=torch.uint8, device="cuda")
    first = None
    for _ in range(12):
        out = api.window_softmax_forward(dev["q_rope"], dev["k_rope"], dev["v"], F=w.F, workspace=ws)
        torch.cuda.synchronize()
        assert api.workspace_status(ws) == 0
        if first is None:
            first = out
        else:
            assert torch.equal(out, first)


EDGE = [
    synth.Workload("sm_one_frame", B=1, H=2, d=128, F=1, S=100, dtype="bf16", alpha_mu=2.0, text=False, seed=48),
    synth.Workload("sm_one_chunk", B=1, H=1, d=128, F=4, S=90, dtype="bf16", alpha_mu=2.0, text=False, seed=49,
                   chunk=8, radius=1),
    synth.Workload("sm_window_wider_than_clip", B=2, H=1, d=128, F=6, S=50, dtype="bf16", alpha_mu=2.0, text=False,
                   seed=60, chunk=2, radius=5),
    synth.Workload("sm_d16_one_frame", B=1, H=3, d=16, F=1, S=7, dtype="f32", alpha_mu=2.0, text=False, seed=61),
]


@pytest.mark.parametrize("w", EDGE, ids=[c.name for c in EDGE])
def test_window_softmax_edge_cases(w):
    inp = synth.make_inputs(w, with_rope_side=True)
    got = _run(w, inp)
    ref = O.window_softmax_forward(inp, w.F, w.S, w.chunk, w.radius)
    tol = TOL_F32 if w.dtype == "f32" else TOL_BF16
    assert rel_err(to_np(got), ref) <= tol, (w.name, rel_err(to_np(got), ref))
