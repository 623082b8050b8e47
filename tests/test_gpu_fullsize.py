"""Parity at the full workload sizes, in the launch configuration bench.py times.

The oracle recomputes sampled outputs one by one (a few heads, tokens spread
over every frame including the first and last token of each frame and the
ragged last tile); a property that holds at any size (the RMS of
out / (gate * rms_w) over d is 1 up to eps and bf16 rounding) is checked on
every token."""
import numpy as np
import pytest
import torch

from harness import TOL_BF16, rel_err
from oracle import vdn_oracle as O
from video_diffusion_linear_b200 import api, synth

pytestmark = pytest.mark.gpu


def _sample_tokens(w, rng, per_frame=3):
    toks = []
    for t in range(w.F):
        base = t * w.S
        toks += [base, base + w.S - 1]
        toks += list(base + rng.integers(0, w.S, size=per_frame))
    return np.array(sorted(set(toks)))


def _check(w, inp, out, heads, rule, c, rng):
    for b, h in heads:
        toks = _sample_tokens(w, rng)
        ref = O.sampled_outputs(inp, w.F, w.S, rule, c, w.chunk, w.radius, b, h, toks)
        got = out[b, torch.as_tensor(toks, device=out.device), h, :].float().cpu().numpy().astype(np.float64)
        err = rel_err(got, ref)
        assert err <= TOL_BF16, (w.name, rule, c, b, h, err)


def _rms_property(w, dev, out):
    g = dev["gate"].float() * dev["rms_w"].float()
    r = (out.float() / g).pow(2).mean(dim=-1)
    assert torch.isfinite(out.float()).all()
    lo, hi = r.min().item(), r.max().item()
    assert 0.9 < lo and hi < 1.1, (lo, hi)


@pytest.mark.parametrize("name", ["480p", "768p", "14s"])
def test_full_size_configs(name):
    w = synth.WORKLOADS[name]
    inp = synth.make_inputs(w)
    dev = api.to_device(inp)
    out = api.branch_forward(*api.forward_inputs(dev), F=w.F, rule=w.rule, c=w.c, chunk=w.chunk, radius=w.radius)
    torch.cuda.synchronize()
    rng = np.random.default_rng(w.seed)
    _check(w, inp, out, [(0, 0), (0, w.H - 1)], w.rule, w.c, rng)
    _rms_property(w, dev, out)


def test_rule_sweep_1024sq():
    """sana_scaled and vdn_scaled at c in {0.5, 1.0} and vdn_solve, each with and
    without the text state, on the 1024^2 workload (batch 2)."""
    w = synth.WORKLOADS["1024sq"]
    inp = synth.make_inputs(w, with_text=True)
    dev = api.to_device(inp)
    shape = api.shape_from(dev["q"], w.F, dev["conv_k_w"])
    ws = api.alloc_workspace(shape)
    out = torch.empty_like(dev["q"])
    rng = np.random.default_rng(4)
    for i, (rule, c, text) in enumerate(synth.RULE_SWEEP):
        args = list(api.forward_inputs(dev))
        inp_run = dict(inp)
        if not text:
            args[-1] = None
            inp_run["text_state"] = None
        api.branch_forward(*args, F=w.F, rule=rule, c=c, chunk=w.chunk, radius=w.radius, out=out, workspace=ws)
        torch.cuda.synchronize()
        assert api.workspace_status(ws) == 0
        # both batch elements (the second one's frames sit in other statistics slots), two heads each
        heads = [(b, (7 * i + 11 * b + j * (w.H // 2)) % w.H) for b in range(w.B) for j in range(2)]
        _check(w, inp_run, out, heads, rule, c, rng)
    _rms_property(w, dev, out)
