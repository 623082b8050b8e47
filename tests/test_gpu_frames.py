"""GPU parity of the frame-sharded branch (vdn_frames_maps, then vdn_frames_finish) through the
C ABI: the ranks run one after another on one GPU (their calls never wait on one another; the
all-gather of the maps is a concatenation here), and the joined output must match the float64
oracle of the whole clip within the bf16 bound, and the unsharded call."""
import numpy as np
import pytest
import torch

from harness import TOL_BF16, gpu_forward, oracle_forward, rel_err, to_np
from video_diffusion_linear_b200 import api, shard, synth

pytestmark = pytest.mark.gpu


def _sharded(w, inp, world):
    parts = [api.to_device(shard.frame_inputs(inp, w.F, world, r, w.chunk)) for r in range(world)]
    maps = [api.frames_maps(p["k"], p["v"], p["beta"], p["alpha"], p["conv_k_w"], p["conv_v_w"], F_total=w.F,
                            world=world, rank=r, rule=w.rule, c=w.c, chunk=w.chunk) for r, p in enumerate(parts)]
    maps_all = torch.cat(maps)
    outs = [api.frames_finish(p["q"], p["alpha_all"], p["gate"], p["rms_w"], p["text_state"], maps_all, F_total=w.F,
                              world=world, rank=r, rule=w.rule, c=w.c, chunk=w.chunk, radius=w.radius)
            for r, p in enumerate(parts)]
    torch.cuda.synchronize()
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


def test_one_rank_equals_the_unsharded_call():
    w = CASES[0][0]
    inp = synth.make_inputs(w)
    joined = _sharded(w, inp, 1)
    full, _ = gpu_forward(w, inp)
    assert rel_err(to_np(joined), to_np(full)) <= 1e-2
