"""GPU parity of the sharded paths through the C ABI; the ranks run one after another on one GPU
(their calls never wait on one another, and the collectives become concatenations and sums):
  * the frame-sharded branch (vdn_frames_maps, then vdn_frames_finish): the joined output against
    the float64 oracle of the whole clip within the bf16 bound, and against the unsharded call;
  * the head-sharded backward: per-head gradients joined, the rms_w gradient summed."""
import numpy as np
import pytest
import torch

from harness import TOL_BF16, gpu_forward, oracle_forward, rel_err, to_np
from oracle import vdn_backward as BW
from oracle import vdn_oracle as O
from test_gpu_backward import BF16, NAMES, _compare
from video_diffusion_linear_b200 import api, shard, synth

pytestmark = pytest.mark.gpu


def _sharded(w, inp, world):
    """Each rank's two phases share one workspace; its device status word must stay clear after
    phase 1 and after phase 2 (which keeps a phase-1 report)."""
    parts = [api.to_device(shard.frame_inputs(inp, w.F, world, r, w.chunk)) for r in range(world)]
    wss = []
    for r, p in enumerate(parts):
        f0, f1 = shard.frame_range(w.F, world, r, w.chunk)
        shape = api.shape_from(p["k"], f1 - f0, p["conv_k_w"])
        wss.append(torch.empty(api.frames_workspace_size(shape, w.F, world, r, w.rule, w.chunk), dtype=torch.uint8,
                               device=p["k"].device))
    maps = [api.frames_maps(p["k"], p["v"], p["beta"], p["alpha"], p["conv_k_w"], p["conv_v_w"], F_total=w.F,
                            world=world, rank=r, rule=w.rule, c=w.c, chunk=w.chunk, workspace=wss[r])
            for r, p in enumerate(parts)]
    for ws in wss:
        assert api.workspace_status(ws) == 0
    maps_all = torch.cat(maps)
    outs = [api.frames_finish(p["q"], p["alpha_all"], p["gate"], p["rms_w"], p["text_state"], maps_all, F_total=w.F,
                              world=world, rank=r, rule=w.rule, c=w.c, chunk=w.chunk, radius=w.radius,
                              workspace=wss[r])
            for r, p in enumerate(parts)]
    torch.cuda.synchronize()
    for ws in wss:
        assert api.workspace_status(ws) == 0
    return torch.cat(outs, dim=1)


CASES = [
    # 8 chunks of 3 over 3 ranks (3, 3, 2 chunks): windows reach the neighbouring ranks
    (synth.Workload("fr_solve", B=1, H=2, d=128, F=23, S=40, dtype="bf16", alpha_mu=2.0, text=True, seed=70,
                    chunk=3, radius=1), 3),
    # 10 chunks of 2 over 4 ranks, windows of 9 chunks: states come from two ranks away; no text state
    (synth.Workload("fr_sana", B=2, H=1, d=128, F=20, S=33, dtype="bf16", alpha_mu=2.0, text=False, seed=71,
                    chunk=2, radius=4, rule="sana_scaled", c=0.7), 4),
    # the page's chunk 5 / radius 1 on a ragged 31-frame clip over 2 ranks (4 + 3 chunks)
    (synth.Workload("fr_p5", B=1, H=2, d=128, F=31, S=24, dtype="bf16", alpha_mu=2.0, text=True, seed=72), 2),
]


@pytest.mark.parametrize("w,world", CASES, ids=[c[0].name for c in CASES])
def test_frame_sharded_branch_matches_the_whole_clip(w, world):
    inp = synth.make_inputs(w)
    joined = _sharded(w, inp, world)
    assert torch.isfinite(joined.float()).all()
    ref = oracle_forward(w, inp)
    assert rel_err(to_np(joined), ref) <= TOL_BF16
    full, _ = gpu_forward(w, inp)
    assert rel_err(to_np(joined), to_np(full)) <= TOL_BF16


def test_frame_sharded_divergent_sana_stays_finite():
    """sana_scaled at c = 1 on inputs whose per-frame operator I - A has an eigenvalue near
    -0.2 beta S: the float64 scans pass 1e39, beyond fp32.  The chunk maps carry power-of-two
    exponents through the all-gather and the fold, so the frame-sharded output stays finite and
    matches the oracle (the same stress inputs as the whole-clip divergence test)."""
    w = synth.Workload("fr_div", B=1, H=2, d=128, F=40, S=384, dtype="bf16", alpha_mu=3.0, text=True, seed=32,
                       rule="sana_scaled", c=1.0)
    inp = synth.make_inputs(w)
    st = O.head_state(inp, 0, 0, w.F, w.S, "sana_scaled", 1.0, w.chunk, w.radius)
    assert np.abs(st["P"]).max() > 1e39
    joined = _sharded(w, inp, 3)
    assert torch.isfinite(joined.float()).all()
    assert rel_err(to_np(joined), oracle_forward(w, inp)) <= TOL_BF16


def test_shard_frame_sharded_forward_checks_the_status_word():
    """shard.frame_sharded_forward with one rank (no collective) shares a workspace between the
    phases, reads its status word and returns the whole clip's output."""
    w = CASES[2][0]
    inp = synth.make_inputs(w)
    local = api.to_device(shard.frame_inputs(inp, w.F, 1, 0, w.chunk))
    out = shard.frame_sharded_forward(local, w.F, 1, 0, rule=w.rule, c=w.c, chunk=w.chunk, radius=w.radius)
    torch.cuda.synchronize()
    assert rel_err(to_np(out), oracle_forward(w, inp)) <= TOL_BF16


def test_one_rank_equals_the_unsharded_call():
    w = CASES[0][0]
    inp = synth.make_inputs(w)
    joined = _sharded(w, inp, 1)
    full, _ = gpu_forward(w, inp)
    assert rel_err(to_np(joined), to_np(full)) <= 1e-2


@pytest.mark.parametrize("world", [2, 3])
def test_head_sharded_backward_reassembles_the_clip(world):
    """Each rank's backward call on its slice of the heads (run one after another: the calls never
    wait on one another); the per-head gradients join along the head axis and the rms_w gradient,
    which every head shares, is the sum of the ranks' partials (what shard.reduce_shared_grads
    all-reduces across GPUs)."""
    w = BF16[0].replace(name="bw_bf16_shard", H=3)
    inp = synth.make_inputs(w)
    dout = synth.make_cotangent(w)
    full = dict(inp, dout=dout)
    parts = []
    for r in range(world):
        part = shard.shard_inputs(full, world, r)
        dev = api.to_device(part)
        parts.append(api.branch_backward(*api.forward_inputs(dev), dout=dev["dout"], F=w.F, rule=w.rule, c=w.c,
                                         chunk=w.chunk, radius=w.radius))
    torch.cuda.synchronize()
    got = {n: None if parts[0][n] is None else
           (sum(p[n] for p in parts) if n in shard.SHARED_GRADS else
            torch.cat([p[n] for p in parts], dim=shard.PER_HEAD[n])) for n in NAMES}
    ref = BW.branch_backward(inp, dout, w.F, w.S, w.rule, w.c, w.chunk, w.radius)
    _compare(w, got, ref, TOL_BF16)
