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


# ----------------------------------------------------------------------------- frame sharding
@pytest.mark.parametrize("F,chunk", [(0, 5), (1, 5), (23, 3), (31, 5), (30, 2), (85, 5)])
@pytest.mark.parametrize("world", [1, 2, 3, 8])
def test_frame_ranges_are_whole_chunks_covering_every_frame_once(F, chunk, world):
    ranges = [shard.frame_range(F, world, r, chunk) for r in range(world)]
    assert [f for f0, f1 in ranges for f in range(f0, f1)] == list(range(F))
    assert all(f0 % chunk == 0 for f0, f1 in ranges if f1 > f0)
    nchunks = [-(-(f1 - f0) // chunk) for f0, f1 in ranges]
    assert max(nchunks) - min(nchunks) <= 1


@pytest.mark.parametrize("F,chunk,radius,world", [(23, 3, 1, 3), (30, 2, 6, 3), (31, 5, 1, 4), (31, 5, 2, 2)])
def test_exchange_plan_matches_the_window_geometry(F, chunk, radius, world):
    # brute force from the oracle's window geometry: every state a window reads outside its rank is
    # published by exactly the rank that owns it
    owner = {f: r for r in range(world) for f in range(*shard.frame_range(F, world, r, chunk))}
    need_pre, need_suf = set(), set()
    for r in range(world):
        f0, f1 = shard.frame_range(F, world, r, chunk)
        pre, suf = shard.remote_states(F, chunk, radius, f0, f1)
        want_pre = {lo - 1 for lo, hi in (O.window_bounds(t, F, chunk, radius) for t in range(f0, f1))
                    if lo > 0 and owner[lo - 1] != r}
        want_suf = {hi + 1 for lo, hi in (O.window_bounds(t, F, chunk, radius) for t in range(f0, f1))
                    if hi < F - 1 and owner[hi + 1] != r}
        assert set(pre) == want_pre and set(suf) == want_suf
        need_pre |= want_pre
        need_suf |= want_suf
    pub = [shard.published_states(F, world, r, chunk, radius) for r in range(world)]
    assert sorted(f for p, _ in pub for f in p) == sorted(need_pre)
    assert sorted(f for _, s in pub for f in s) == sorted(need_suf)
    assert all(owner[f] == r for r, (p, s) in enumerate(pub) for f in p + s)


def _frame_worker(rank, world, port, w, q):
    """One rank of the frame-sharded branch, its arithmetic taken from the oracle: local features,
    statistics and per-frame affine maps; an all-gather of each rank's composed maps gives the seeds;
    a local re-scan; an all-gather of the published boundary states; then gather and read-out.
    States the plan does not deliver stay NaN, so a gap in it shows in the output."""
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        inp = synth.make_inputs(w)
        F, S, d, H = w.F, w.S, w.d, w.H
        f0, f1 = shard.frame_range(F, world, rank, w.chunk)
        n = f1 - f0
        eye, zero = np.eye(d), np.zeros((d, d))

        def step(s, f, st):
            return O.rule_step(s, st["A"][f - f0], st["B"][f - f0], st["alpha"][f], w.rule, w.c)

        local = {}
        maps = {}
        for h in range(H):
            sl = slice(f0 * S, f1 * S)
            qf, kf, vf = O.prepare_features(O._f64(inp["q"][0, sl, h]), O._f64(inp["k"][0, sl, h]),
                                            O._f64(inp["v"][0, sl, h]), n, S, O._f64(inp["conv_k_w"][h]),
                                            O._f64(inp["conv_v_w"][h]))
            A, Bm = O.frame_statistics(kf, vf, O._f64(inp["beta"][0, sl, h]).reshape(n, S))
            st = {"qf": qf, "A": A, "B": Bm, "alpha": O._f64(inp["alpha"][0, :, h]),
                  "seed": O.seed_state(O._f64(inp["text_state"][h]), d)}
            local[h] = st
            Gf, Bf = eye, zero                        # frames f0..f1-1, in the prefix scan's order
            for f in range(f0, f1):
                Bp = step(zero, f, st)
                Gf, Bf = Gf @ (step(eye, f, st) - Bp), Bf @ (step(eye, f, st) - Bp) + Bp
            Gb, Bb = eye, zero                        # frames f1-1..f0, in the suffix scan's order
            for f in reversed(range(f0, f1)):
                Bp = step(zero, f, st)
                Gb, Bb = Gb @ (step(eye, f, st) - Bp), Bb @ (step(eye, f, st) - Bp) + Bp
            maps[h] = (Gf, Bf, Gb, Bb)
        all_maps = [None] * world
        dist.all_gather_object(all_maps, maps)

        pub_pre, pub_suf = shard.published_states(F, world, rank, w.chunk, w.radius)
        sent = {}
        for h, st in local.items():
            sp = st["seed"]
            for r in range(rank):
                sp = sp @ all_maps[r][h][0] + all_maps[r][h][1]
            ss = st["seed"]
            for r in reversed(range(rank + 1, world)):
                ss = ss @ all_maps[r][h][2] + all_maps[r][h][3]
            P = np.full((F, d, d), np.nan)
            Q = np.full((F, d, d), np.nan)
            for f in range(f0, f1):
                sp = step(sp, f, st)
                P[f] = sp
            for f in reversed(range(f0, f1)):
                ss = step(ss, f, st)
                Q[f] = ss
            st["P"], st["Q"] = P, Q
            sent[h] = ({f: P[f] for f in pub_pre}, {f: Q[f] for f in pub_suf})
        got = [None] * world
        dist.all_gather_object(got, sent)

        need_pre, need_suf = shard.remote_states(F, w.chunk, w.radius, f0, f1)
        out = np.empty((n * S, H, d))
        rms_w = O._f64(inp["rms_w"])
        for h, st in local.items():
            for r in range(world):
                for f, x in got[r][h][0].items():
                    if f in need_pre:
                        st["P"][f] = x
                for f, x in got[r][h][1].items():
                    if f in need_suf:
                        st["Q"][f] = x
            g = O._f64(inp["gate"][0, f0 * S:f1 * S, h]).reshape(n, S, d)
            for t in range(f0, f1):
                W_t = O.gather_state(st["P"], st["Q"], st["seed"], st["alpha"], t, w.chunk, w.radius)
                out[(t - f0) * S:(t - f0 + 1) * S, h] = O.readout(W_t, st["qf"][t - f0], g[t - f0], rms_w)
        parts = [None] * world
        dist.all_gather_object(parts, out)
        if rank == 0:
            q.put(np.concatenate(parts, axis=0))
    finally:
        dist.destroy_process_group()


FRAME_CASES = [
    # 8 chunks over 3 ranks (3, 3, 2): windows reach the neighbouring ranks
    synth.Workload("fs_solve", B=1, H=2, d=8, F=23, S=7, dtype="f32", alpha_mu=2.0, text=True, seed=33,
                   chunk=3, radius=1),
    # 15 chunks of 2 frames over 3 ranks, windows 12 frames each side: states come from two ranks away
    synth.Workload("fs_sana", B=1, H=1, d=8, F=30, S=5, dtype="f32", alpha_mu=2.0, text=True, seed=34,
                   chunk=2, radius=6, rule="sana_scaled", c=0.7),
]


@pytest.mark.parametrize("w", FRAME_CASES, ids=[c.name for c in FRAME_CASES])
def test_three_gloo_ranks_frame_sharded_branch_matches_the_whole_clip(w):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_frame_worker, args=(r, 3, port, w, q)) for r in range(3)]
    for p in procs:
        p.start()
    joined = q.get(timeout=180)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    ref = O.branch_forward(synth.make_inputs(w), w.F, w.S, w.rule, w.c, w.chunk, w.radius)[0]
    assert np.isfinite(joined).all()
    # composing the maps reorders the arithmetic of the scans: equal to rounding
    np.testing.assert_allclose(joined, ref, rtol=1e-9, atol=1e-11 * np.abs(ref).max())


@pytest.mark.parametrize("rule,c", [("vdn_solve", 1.0), ("vdn_scaled", 0.6), ("sana_scaled", 0.7), ("additive", 1.0)])
@pytest.mark.parametrize("F,chunk", [(11, 3), (10, 5), (7, 2)])
def test_chunk_maps_fold_into_the_scans_chunk_edge_states(rule, c, F, chunk):
    """The device path's exchange, in the oracle's arithmetic: per chunk and direction, O_c is the
    chunk's scan from zero and G_c the scan from the identity with B taken as zero (the linear part);
    folding S <- S G_c + O_c from the seed in scan order gives P at every chunk end and Q at every
    chunk start, as the whole-clip scans do."""
    rng = np.random.default_rng(40 + F + chunk)
    d = 6
    R = rng.normal(size=(F, d, d))
    A = np.einsum("fij,fkj->fik", R, R) / d
    Bm = rng.normal(size=(F, d, d))
    alpha = 1 / (1 + np.exp(-rng.normal(2, 1, size=(F, d))))
    seed = rng.normal(size=(d, d))
    P, Q = O.bidirectional_scan(A, Bm, alpha, seed, rule, c)
    zero = np.zeros((d, d))
    chunks = [list(range(j, min(F, j + chunk))) for j in range(0, F, chunk)]

    def chunk_map(frames):
        s0, s1 = zero, np.eye(d)
        for f in frames:
            s0 = O.rule_step(s0, A[f], Bm[f], alpha[f], rule, c)
            s1 = O.rule_step(s1, A[f], zero, alpha[f], rule, c)
        return s1, s0                                           # (G_c, O_c)

    s = seed
    for fr in chunks[:-1]:                                      # prefix: P at each chunk's last frame
        G, Oc = chunk_map(fr)
        s = s @ G + Oc
        np.testing.assert_allclose(s, P[fr[-1]], rtol=1e-10, atol=1e-10 * np.abs(P).max())
    s = seed
    for fr in reversed(chunks[1:]):                             # suffix: Q at each chunk's first frame
        G, Oc = chunk_map(fr[::-1])
        s = s @ G + Oc
        np.testing.assert_allclose(s, Q[fr[0]], rtol=1e-10, atol=1e-10 * np.abs(Q).max())


# ----------------------------------------------------------------------------- frame-sharded orchestration
def _fake_frames_maps(k, v, beta, alpha, conv_k_w, conv_v_w, *, F_total, world, rank, rule, c, chunk, **_):
    """vdn_frames_maps in the oracle's arithmetic, in the header's layout: the maps
    [B*H][2 directions][nch][G_c | O_c][d][d], nch = ceil(C / world), then one exponent e per
    map (the map is 2^e times the stored matrix; here e puts the largest entry in [0.5, 1)),
    float64 throughout."""
    f0, f1 = shard.frame_range(F_total, world, rank, chunk)
    n = f1 - f0
    B, N, H, d = k.shape
    S = N // n
    nch = -(-(-(-F_total // chunk)) // world)
    maps = np.full((B, H, 2, nch, 2, d, d), np.nan)
    eye, zero = np.eye(d), np.zeros((d, d))
    for b in range(B):
        for h in range(H):
            kh, vh = O._f64(k[b, :, h]), O._f64(v[b, :, h])
            _, kf, vf = O.prepare_features(kh, kh, vh, n, S, O._f64(conv_k_w[h]), O._f64(conv_v_w[h]))
            A, Bm = O.frame_statistics(kf, vf, O._f64(beta[b, :, h]).reshape(n, S))
            al = O._f64(alpha[b, :, h])
            for j, c0 in enumerate(range(0, n, chunk)):
                frames = list(range(c0, min(n, c0 + chunk)))
                for dr, order in ((0, frames), (1, frames[::-1])):
                    g, o = eye, zero
                    for f in order:
                        g = O.rule_step(g, A[f], zero, al[f], rule, c)
                        o = O.rule_step(o, A[f], Bm[f], al[f], rule, c)
                    maps[b, h, dr, j] = g, o
    exps = np.zeros(maps.shape[:-2])
    for idx in np.ndindex(*exps.shape):
        m = np.abs(maps[idx]).max()
        if np.isfinite(m) and m > 0:
            e = np.frexp(m)[1]
            exps[idx] = e
            maps[idx] = np.ldexp(maps[idx], -e)
    return torch.from_numpy(np.concatenate([maps.ravel(), exps.ravel()]))


def _fake_frames_finish(q, alpha_all, gate, rms_w, text_state, maps_all, *, F_total, world, rank, rule, c, chunk,
                        radius, **_):
    """vdn_frames_finish in the oracle's arithmetic: fold every rank's maps (rank-major, as the
    all-gather lays them out) into the chunk-edge states, gather and read out the rank's frames."""
    f0, f1 = shard.frame_range(F_total, world, rank, chunk)
    n = f1 - f0
    B, N, H, d = q.shape
    S = N // n
    C = -(-F_total // chunk)
    nch = -(-C // world)
    buf = maps_all.numpy().reshape(world, -1)
    nm = B * H * 2 * nch * 2 * d * d
    exps = buf[:, nm:].reshape(world, B, H, 2, nch, 2)
    maps = np.ldexp(buf[:, :nm].reshape(world, B, H, 2, nch, 2, d, d), exps[..., None, None].astype(int))
    first = [shard.frame_range(F_total, world, r, chunk)[0] // chunk for r in range(world)]
    owner = lambda ch: max(r for r in range(world) if first[r] <= ch)
    out = np.empty((B, N, H, d))
    for b in range(B):
        for h in range(H):
            seed = O.seed_state(None if text_state is None else O._f64(text_state[h]), d)
            P = np.full((F_total, d, d), np.nan)
            Q = np.full((F_total, d, d), np.nan)
            s = seed
            for ch in range(C - 1):
                r = owner(ch)
                g, o = maps[r, b, h, 0, ch - first[r]]
                s = s @ g + o
                P[(ch + 1) * chunk - 1] = s
            s = seed
            for ch in range(C - 1, 0, -1):
                r = owner(ch)
                g, o = maps[r, b, h, 1, ch - first[r]]
                s = s @ g + o
                Q[ch * chunk] = s
            qh = O._f64(q[b, :, h])
            qf, _, _ = O.prepare_features(qh, qh, qh, n, S)
            g = O._f64(gate[b, :, h]).reshape(n, S, d)
            al = O._f64(alpha_all[b, :, h])
            for t in range(f0, f1):
                W_t = O.gather_state(P, Q, seed, al, t, chunk, radius)
                out[b, (t - f0) * S:(t - f0 + 1) * S, h] = O.readout(W_t, qf[t - f0], g[t - f0], O._f64(rms_w))
    return torch.from_numpy(out)


def _orchestration_worker(rank, world, port, w, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        from video_diffusion_linear_b200 import api
        api.frames_maps, api.frames_finish = _fake_frames_maps, _fake_frames_finish
        local = shard.frame_inputs(synth.make_inputs(w), w.F, world, rank, w.chunk)
        out = shard.frame_sharded_forward(local, w.F, world, rank, rule=w.rule, c=w.c, chunk=w.chunk,
                                          radius=w.radius)
        got = [None] * world
        dist.all_gather_object(got, out)
        if rank == 0:
            q.put(torch.cat(got, dim=1).numpy())
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("w,world", [(FRAME_CASES[0], 3), (FRAME_CASES[1].replace(B=2), 2)],
                         ids=["solve_3", "sana_2"])
def test_frame_sharded_forward_orchestration_on_gloo_ranks(w, world):
    """shard.frame_sharded_forward on gloo ranks, its two device phases stood in for by the oracle
    following the header's map layout: the all-gather's rank order, the padding of the map buffers
    to ceil(C / world) chunks and the frame slicing give the whole clip's output."""
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_orchestration_worker, args=(r, world, port, w, q)) for r in range(world)]
    for p in procs:
        p.start()
    joined = q.get(timeout=180)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    ref = O.branch_forward(synth.make_inputs(w), w.F, w.S, w.rule, w.c, w.chunk, w.radius)
    assert np.isfinite(joined).all()
    np.testing.assert_allclose(joined, ref, rtol=1e-9, atol=1e-11 * np.abs(ref).max())
