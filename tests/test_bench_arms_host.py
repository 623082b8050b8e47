"""bench.py's GPU arms run through on the CPU with CUDA and the library calls stubbed out (here,
in the test only): every arm and sharding mode assembles the contract's JSON line.  This guards
the code paths that otherwise only run on a GPU machine against Python errors; the numbers are
meaningless."""
import contextlib
import io
import json

import pytest
import torch

import bench
from video_diffusion_linear_b200 import api, synth

KEYS = {"metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better", "scaling",
        "vs_baseline", "dtype", "data", "config", "roofline", "cpu_baseline", "e2e", "gpu_launches", "clocks"}
ROOF = {"bound", "achieved", "peak", "unit", "frac", "traffic"}
E2E = {"value", "unit", "h2d_bytes_per_step", "d2h_bytes_per_step"}


class _Event:
    def __init__(self, *a, **k):
        self.cuda_event = 0

    def record(self, *a):
        pass

    def elapsed_time(self, other):
        return 1.0


class _Clocks:
    def __init__(self, *a):
        pass

    def __enter__(self):
        return self

    def __exit__(self, *a):
        return False

    def summary(self):
        return {"sm_mhz": 1965, "sm_max_mhz": 1965, "reasons": []}


class _Stream:
    cuda_stream = 0


def _grads(q, k, v, beta, alpha, gate, rms_w, conv_k_w=None, conv_v_w=None, text_state=None, *, grads=None, **kw):
    if grads is not None:
        return grads
    f32 = dict(dtype=torch.float32)
    return {"dq": torch.empty_like(q), "dk": torch.empty_like(k), "dv": torch.empty_like(v),
            "dgate": torch.empty_like(gate), "dbeta": torch.empty(beta.shape, **f32),
            "dalpha": torch.empty(alpha.shape, **f32), "drms_w": torch.empty(rms_w.shape, **f32),
            "dconv_k_w": None, "dconv_v_w": None, "dtext_state": None}


@pytest.fixture
def stubbed(monkeypatch):
    empty = torch.empty

    def host_empty(*a, **k):
        if "cuda" in str(k.get("device", "")):
            k.pop("device")
        return empty(*a, **k)

    monkeypatch.setattr(torch, "empty", host_empty)
    monkeypatch.setattr(torch.cuda, "Event", _Event)
    monkeypatch.setattr(torch.cuda, "set_device", lambda *a, **k: None)
    monkeypatch.setattr(torch.cuda, "synchronize", lambda *a, **k: None)
    monkeypatch.setattr(torch.cuda, "current_stream", lambda *a, **k: _Stream())
    monkeypatch.setattr(torch.Tensor, "pin_memory", lambda self: self)
    monkeypatch.setattr(bench, "ClockSampler", _Clocks)
    monkeypatch.setattr(api, "to_device", lambda inp, device="cuda": dict(inp))
    monkeypatch.setattr(api, "alloc_workspace", lambda *a, **k: empty(16, dtype=torch.uint8))
    for name in ("branch_forward", "branch_forward_timed", "window_softmax_forward", "hybrid_forward"):
        monkeypatch.setattr(api, name, lambda *a, **k: k.get("out"))
    monkeypatch.setattr(api, "workspace_status", lambda *a, **k: 0)
    monkeypatch.setattr(api, "branch_backward", _grads)
    monkeypatch.setattr(api, "frames_maps", lambda *a, maps=None, **k: maps)
    monkeypatch.setattr(api, "frames_finish", lambda *a, out=None, **k: out)
    monkeypatch.setattr(api, "feature_prep", lambda *a, out=None, **k: out)
    monkeypatch.setitem(synth.WORKLOADS, "tiny_bf16", synth.Workload("tiny_bf16", 1, 2, 128, 12, 8, "bf16", 2.0,
                                                                     True, 5))


def _line(argv):
    buf = io.StringIO()
    with contextlib.redirect_stdout(buf):
        bench.main(argv)
    return json.loads(buf.getvalue().strip().splitlines()[-1])


@pytest.mark.parametrize("extra", [
    [], ["--shard", "heads"], ["--path", "softmax"], ["--path", "hybrid", "--shard", "heads"],
    ["--path", "backward"], ["--path", "backward", "--shard", "heads"],
    ["--workload", "tiny_bf16", "--shard", "frames"],
    ["--workload", "tiny_bf16", "--path", "features"], ["--workload", "tiny_bf16", "--path", "features",
                                                        "--shard", "heads"],
])
def test_gpu_arms_assemble_the_contract_line(stubbed, extra):
    argv = ["--workload", "tiny_f20_text", "--steps", "2", "--warmup", "3", "--no-cpu"] + extra
    j = _line(argv)
    assert KEYS <= set(j), KEYS - set(j)
    assert ROOF <= set(j["roofline"]) and E2E <= set(j["e2e"])
    assert j["n_gpus"] == 1 and j["steps"] == 2 and j["warmup"] == 3 and j["gpu_launches"] > 0
    assert j["scaling"] == ("weak" if "--shard" not in extra else "strong")
    assert "workload" in j["config"] and "parallelism" in j["config"]


def test_default_arm_carries_the_oracle_baseline(stubbed):
    j = _line(["--workload", "tiny_f20_text", "--steps", "2", "--warmup", "3"])
    assert j["cpu_baseline"]["kind"] == "oracle" and j["cpu_baseline"]["value"] > 0 and j["cpu_baseline"]["cores"] >= 1


def test_features_arm_carries_the_oracle_baseline(stubbed):
    j = _line(["--workload", "tiny_bf16", "--path", "features", "--steps", "2", "--warmup", "3"])
    assert j["roofline"]["kernel"] == "feature_prep" and j["roofline"]["bound"] == "hbm"
    assert j["cpu_baseline"]["kind"] == "oracle" and j["cpu_baseline"]["value"] > 0
