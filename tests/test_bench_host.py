"""Host logic of bench.py: roofline arithmetic, the traffic table, and the
multi-rank helpers on two gloo ranks (CPU, 127.0.0.1)."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench
from video_diffusion_linear_b200 import synth


def test_path_roofline_768p():
    w = synth.WORKLOADS["768p"]
    pr = bench.path_roofline(w, {"hbm_gbs": 6546.9, "bf16_tflops": 1590.1})
    assert pr["bound"] == "hbm"
    assert abs(pr["bytes"] / 1e9 - 4.09) < 0.01          # q, k, v, gate, beta in, out, per-frame maps
    assert abs(pr["t_roof_us"] - 625) < 2
    assert abs(pr["flops"] / 1e9 - 305.8) < 0.5


def test_algorithmic_bytes_cover_the_path():
    w = synth.WORKLOADS["768p"]
    alg = bench.algorithmic_bytes(w)
    TH = w.B * w.F * w.S * w.H
    assert alg["frame_stats"] >= TH * 516 and alg["readout"] >= TH * 768
    assert set(alg) == set(bench.KERNELS_TC)


def test_recorded_traffic_tracks_source():
    for k in bench.KERNELS_TC:
        rec = bench.recorded_traffic(k)
        if rec is not None:                      # present only while the kernel source is unchanged
            assert rec["bytes"] > 0 and rec["workload"] == "768p"


def test_rank_workloads_are_distinct_clips():
    w = synth.WORKLOADS["768p"]
    seeds = {bench.rank_workload(w, r).seed for r in range(8)}
    assert len(seeds) == 8
    assert all(bench.rank_workload(w, r).tokens == w.tokens for r in range(8))


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        bench.barrier()
        m = bench.reduce_max(float(10 + rank))
        q.put((rank, m, bench.dist_env()[:2]))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_take_the_max_time():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert [r[1] for r in res] == [11.0, 11.0]
    assert [tuple(r[2]) for r in res] == [(0, 2), (1, 2)]


def test_reduce_max_without_process_group():
    assert bench.reduce_max(3.5) == 3.5


@pytest.mark.parametrize("name", ["480p", "768p", "14s"])
def test_softmax_flops_count_chunk_pairs(name):
    # chunk-aligned windows are symmetric: frame f is in the window of frame t exactly when their chunks
    # differ by at most `radius`, so the (query, key) pairs are sums over chunk pairs
    w = synth.WORKLOADS[name]
    nch = -(-w.F // w.chunk)
    size = [min(w.F, (c + 1) * w.chunk) - c * w.chunk for c in range(nch)]
    pairs = sum(size[a] * size[b] for a in range(nch) for b in range(nch) if abs(a - b) <= w.radius) * w.S * w.S
    assert bench.softmax_flops(w) == 4 * w.d * pairs * w.B * w.H


def test_backward_accounting():
    w = synth.WORKLOADS["768p"]
    TH = w.B * w.F * w.S * w.H
    nb = bench.backward_bytes(w)
    tok = 2 * w.d * TH                                   # one bf16 token tensor
    assert nb["readout_bwd"] >= 5 * tok                  # q, gate, dout in; dq, dgate out
    assert nb["stats_bwd"] >= 2 * tok + 2 * tok          # k, v in; dk', dv' out
    assert nb["conv_bwd"] >= 4 * tok                     # dk', dv' (or more), k, v in; dk, dv out
    fl = bench.backward_flops(w)
    assert fl["readout_bwd"] == fl["stats_bwd"] == 6 * w.d * w.d * TH
    assert set(bench.BWD_KERNELS) >= set(nb) | set(fl)


def test_recorded_traffic_of_the_softmax_kernel():
    rec = bench.recorded_traffic("window_softmax")
    if rec is not None:                                  # present while softmax.cu is unchanged
        w = synth.WORKLOADS["768p"]
        alg = 4 * 2 * w.d * w.B * w.F * w.S * w.H        # q_rope, k_rope, v in, out out
        assert 0.9 * alg <= rec["bytes"] <= 1.2 * alg


@pytest.mark.parametrize("path", ["linear", "softmax", "backward"])
def test_reference_arm_prints_one_contract_line(path, capsys):
    # the oracle arm on the smallest workload: one JSON line with the contract's keys
    import json
    bench.main(["--impl", "reference", "--path", path, "--workload", "tiny", "--steps", "2", "--warmup", "3",
                "--cpu-tokens", "8"])
    lines = [l for l in capsys.readouterr().out.splitlines() if l.startswith("{")]
    assert len(lines) == 1
    j = json.loads(lines[0])
    assert j["impl"] == "reference" and j["value"] > 0 and j["steps"] == 2 and j["warmup"] == 3
    assert j["cpu_baseline"]["kind"] == "oracle" and j["cpu_baseline"]["value"] == j["value"]
    assert j["e2e"]["h2d_bytes_per_step"] == 0 and j["e2e"]["d2h_bytes_per_step"] == 0


def test_rank_inputs_split_heads_or_clips():
    w = synth.WORKLOADS["tiny_f20_text"].replace(H=3)
    parts = [bench.rank_inputs("heads", w, 2, r) for r in range(2)]
    assert [p[1].H for p in parts] == [2, 1]
    assert all(p[2] == w.tokens and p[3]["scaling"] == "strong" and p[3]["global_batch"] == w.B for p in parts)
    full = synth.make_inputs(w)
    assert torch.equal(torch.cat([p[0]["q"] for p in parts], dim=2), full["q"])
    host, wr, job, split = bench.rank_inputs("clips", w, 2, 1, cotangent=True)
    assert wr.seed != w.seed and job == 2 * w.tokens and split["scaling"] == "weak" and "dout" in host
    with pytest.raises(SystemExit):
        bench.rank_inputs("heads", w, 4, 0)


@pytest.mark.parametrize("path", ["linear", "softmax", "backward"])
def test_reference_arm_runs_on_rank_zero_only(path, capsys, monkeypatch):
    # under torchrun every rank but 0 returns at once, printing nothing and running no oracle
    monkeypatch.setenv("RANK", "1")
    monkeypatch.setenv("WORLD_SIZE", "2")
    monkeypatch.setattr(bench, "oracle_sample", lambda *a, **k: pytest.fail("oracle ran on rank 1"))
    bench.main(["--impl", "reference", "--path", path, "--workload", "tiny", "--steps", "2", "--warmup", "3"])
    assert capsys.readouterr().out == ""
