"""The Python binding's argument checks (CPU): host tensors, and tensors whose dtype, shape or
device differ from what vdn.h fixes, are refused before any pointer reaches the library; the
checks accept the inputs the seeded generator makes for every workload."""
import types

import pytest
import torch

from video_diffusion_linear_b200 import api, synth

CUDA = torch.device("cuda", 0)


def _fake(t, device=CUDA, dtype=None, shape=None):
    # stands in for a CUDA tensor: the checks read only device, dtype and shape
    return types.SimpleNamespace(device=device, dtype=dtype or t.dtype, shape=tuple(shape or t.shape))


@pytest.mark.parametrize("name", ["tiny_f20_text", "480p"])
def test_specs_accept_the_generated_inputs(name):
    w = synth.WORKLOADS[name].replace(F=4 if name == "480p" else synth.WORKLOADS[name].F)
    inp = synth.make_inputs(w, with_rope_side=False)
    a = api.forward_inputs(inp)
    specs = api._branch_specs(*a, w.F)
    for n, t, shape, dtype, optional in specs:
        if t is None:
            assert optional, n
            continue
        assert tuple(t.shape) == tuple(shape) and t.dtype == dtype, n
    api._validate([(n, None if t is None else _fake(t), s, d, o) for n, t, s, d, o in specs], CUDA)


def test_host_tensors_are_refused():
    w = synth.WORKLOADS["tiny_f20_text"]
    inp = synth.make_inputs(w)
    with pytest.raises(ValueError, match="CUDA tensors"):
        api.branch_forward(*api.forward_inputs(inp), F=w.F)
    with pytest.raises(ValueError, match="CUDA tensors"):
        api.window_softmax_forward(inp["q"], inp["k"], inp["v"], F=w.F)
    with pytest.raises(ValueError, match="CUDA tensors"):
        api.branch_backward(*api.forward_inputs(inp), dout=inp["q"], F=w.F)


@pytest.mark.parametrize("name,bad", [
    ("beta", dict(dtype=torch.bfloat16)),             # fp32 per vdn.h: read as 4-byte elements
    ("alpha", dict(shape=(1, 19, 2, 16))),            # one frame short
    ("rms_w", dict(shape=(32,))),
    ("k", dict(dtype=torch.bfloat16)),                 # token tensors share q's dtype
    ("conv_v_w", dict(shape=(2, 16, 1))),              # both taps have one width
    ("text_state", dict(device=torch.device("cuda", 1))),
])
def test_mismatched_tensors_are_refused(name, bad):
    w = synth.WORKLOADS["tiny_f20_text"]
    inp = synth.make_inputs(w)
    specs = api._branch_specs(*api.forward_inputs(inp), w.F)
    fakes = [(n, None if t is None else _fake(t, **(bad if n == name else {})), s, d, o) for n, t, s, d, o in specs]
    with pytest.raises(ValueError, match=name):
        api._validate(fakes, CUDA)


def test_missing_required_tensor_and_byte_buffers():
    w = synth.WORKLOADS["tiny_f20_text"]
    inp = synth.make_inputs(w)
    specs = api._branch_specs(*api.forward_inputs(inp), w.F)
    fakes = [(n, None if (t is None or n == "gate") else _fake(t), s, d, o) for n, t, s, d, o in specs]
    with pytest.raises(ValueError, match="gate is required"):
        api._validate(fakes, CUDA)
    with pytest.raises(ValueError, match="workspace"):
        api._bytes("workspace", _fake(inp["beta"]), CUDA)          # fp32, not bytes
    with pytest.raises(ValueError, match="saved"):
        api._bytes("saved", types.SimpleNamespace(device=torch.device("cpu"), dtype=torch.uint8), CUDA)
    api._bytes("workspace", types.SimpleNamespace(device=CUDA, dtype=torch.uint8), CUDA)
