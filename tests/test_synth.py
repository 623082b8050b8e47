"""The seeded input generator: shapes, dtypes, value ranges, determinism."""
import numpy as np
import torch

from video_diffusion_linear_b200 import synth


def test_shapes_and_dtypes():
    w = synth.WORKLOADS["tiny_f20_text"]
    x = synth.make_inputs(w)
    B, N, H, d = w.B, w.N, w.H, w.d
    assert x["q"].shape == (B, N, H, d) and x["q"].dtype == torch.float32
    assert x["beta"].shape == (B, N, H)
    assert x["alpha"].shape == (B, w.F, H, d)
    assert x["conv_k_w"].shape == (H, d, 3)
    assert x["text_state"].shape == (H, d, d)
    assert ((x["beta"] > 0) & (x["beta"] < 1)).all()
    assert ((x["alpha"] > 0) & (x["alpha"] <= 1)).all()


def test_bf16_workload_dtype():
    w = synth.WORKLOADS["480p"].replace(H=2, F=3, S=10)
    x = synth.make_inputs(w)
    assert x["q"].dtype == torch.bfloat16 and x["gate"].dtype == torch.bfloat16
    assert x["beta"].dtype == torch.float32


def test_independent_of_thread_count():
    w = synth.WORKLOADS["480p"].replace(H=3, F=5, S=300)
    a = synth.make_inputs(w, threads=1)
    b = synth.make_inputs(w, threads=7)
    for key in a:
        if a[key] is not None:
            assert torch.equal(a[key], b[key]), key


def test_seed_changes_values():
    w = synth.WORKLOADS["tiny"]
    a = synth.make_inputs(w)
    b = synth.make_inputs(w.replace(seed=5))
    assert not torch.equal(a["q"], b["q"])
