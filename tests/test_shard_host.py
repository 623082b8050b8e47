"""Head sharding (CPU): the balanced partition of the heads across ranks, the per-rank input
slices, and on two gloo ranks that per-rank branch outputs (computed here by the oracle on each
rank's slice) reassemble the whole clip's output exactly, and that per-rank backward gradients,
with the rms_w gradient summed across the ranks by reduce_shared_grads, are the whole clip's."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from oracle import vdn_backward as OB
from oracle import vdn_oracle as O
from video_diffusion_linear_b200 import shard, synth


@pytest.mark.parametrize("H", [0, 1, 2, 3, 7, 24, 25])
@pytest.mark.parametrize("world", [1, 2, 3, 4, 8])
def test_head_ranges_cover_every_head_once_and_balance(H, world):
    ranges = [shard.head_range(H, world, r) for r in range(world)]
    owned = [h for h0, h1 in ranges for h in range(h0, h1)]
    assert owned == list(range(H))                         # contiguous, in rank order, no gap or overlap
    sizes = [h1 - h0 for h0, h1 in ranges]
    assert max(sizes) - min(sizes) <= 1
    assert sizes == sorted(sizes, reverse=True)            # the extra heads go to the first ranks


@pytest.mark.parametrize("H,world,rank", [(4, 0, 0), (4, 2, 2), (4, 2, -1), (-1, 2, 0)])
def test_head_range_rejects_bad_arguments(H, world, rank):
    with pytest.raises(ValueError):
        shard.head_range(H, world, rank)


def test_shard_inputs_slices_per_head_tensors_only():
    w = synth.WORKLOADS["tiny_f20_text"].replace(H=3)
    inp = synth.make_inputs(w)
    parts = [shard.shard_inputs(inp, 2, r) for r in range(2)]
    assert [p["q"].shape[2] for p in parts] == [2, 1]
    for name, axis in shard.PER_HEAD.items():
        if inp.get(name) is None:
            continue
        joined = torch.cat([p[name] for p in parts], dim=axis)
        assert torch.equal(joined, inp[name]), name
        assert all(p[name].is_contiguous() for p in parts)
    for name in inp:
        if name not in shard.PER_HEAD:
            assert all(p[name] is inp[name] for p in parts), name


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


W_SHARD = synth.Workload("shard", B=1, H=3, d=16, F=14, S=9, dtype="f32", alpha_mu=2.0, text=True, seed=31,
                         chunk=3, radius=1)


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        w = W_SHARD
        part = shard.shard_inputs(synth.make_inputs(w), world, rank)   # every rank draws the same clip
        out = torch.from_numpy(O.branch_forward(part, w.F, w.S, w.rule, w.c, w.chunk, w.radius))
        got = [None] * world
        dist.all_gather_object(got, out)
        if rank == 0:
            q.put(torch.cat(got, dim=2).numpy())
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_reassemble_the_whole_output():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    joined = q.get(timeout=180)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    w = W_SHARD
    full = O.branch_forward(synth.make_inputs(w), w.F, w.S, w.rule, w.c, w.chunk, w.radius)
    assert joined.shape == full.shape
    assert np.array_equal(joined, full)                    # the heads never interact: bitwise


W_SHARD_BWD = synth.Workload("shard_bwd", B=2, H=3, d=16, F=8, S=9, dtype="f32", alpha_mu=2.0, text=True, seed=32,
                             chunk=2, radius=1)
GRADS = ("dq", "dk", "dv", "dgate", "dbeta", "dalpha", "dconv_k_w", "dconv_v_w", "dtext_state")


def _bwd_worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        w = W_SHARD_BWD
        full = synth.make_inputs(w)
        full["dout"] = synth.make_cotangent(w)
        part = shard.shard_inputs(full, world, rank)
        g = OB.branch_backward(part, part["dout"], w.F, w.S, w.rule, w.c, w.chunk, w.radius)
        g = {n: None if t is None else torch.from_numpy(np.asarray(t)) for n, t in g.items()}
        local_drms = g["drms_w"].clone()
        shard.reduce_shared_grads(g)
        got = [None] * world
        dist.all_gather_object(got, {n: g[n] for n in GRADS})
        if rank == 0:
            joined = {n: torch.cat([r[n] for r in got], dim=shard.PER_HEAD[n]).numpy() for n in GRADS}
            q.put((joined, g["drms_w"].numpy(), local_drms.numpy()))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_reassemble_the_backward():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_bwd_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    joined, drms, local_drms = q.get(timeout=180)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    w = W_SHARD_BWD
    full = synth.make_inputs(w)
    ref = OB.branch_backward(full, synth.make_cotangent(w), w.F, w.S, w.rule, w.c, w.chunk, w.radius)
    for n in GRADS:
        assert np.array_equal(joined[n], ref[n]), n        # per-head gradients never mix heads: bitwise
    # the shared gradient is a sum over heads: equal up to the order of the additions
    np.testing.assert_allclose(drms, ref["drms_w"], rtol=1e-12, atol=1e-12 * np.abs(ref["drms_w"]).max())
    assert not np.allclose(local_drms, ref["drms_w"])    # rank 0's own heads alone do not give it
