"""Thin Python binding of libvdn (include/vdn.h).

Argument marshalling only: torch supplies device memory and the stream, every
step of the branch runs in the library's CUDA kernels.  Tensors must be CUDA
tensors in the layouts documented in vdn.h.
"""
from __future__ import annotations

import ctypes

import torch

from . import _lib
from ._lib import VDN_DTYPE, VDN_IMPL, VDN_RULE, VdnDebugOut, VdnShape, check

_TORCH_DTYPE = {torch.float32: "f32", torch.bfloat16: "bf16"}


def _ptr(t):
    if t is None:
        return None
    if not t.is_contiguous():
        raise ValueError("tensors passed to libvdn must be contiguous")
    return ctypes.c_void_p(t.data_ptr())


def _validate(specs, device) -> None:
    """Checks (name, tensor, shape, dtype, optional) specs before any pointer reaches the library:
    the kernels read each buffer with the element type and extent vdn.h fixes, so a tensor of
    another dtype, shape or device would be read out of its bounds."""
    if device.type != "cuda":
        raise ValueError(f"libvdn takes CUDA tensors, got a tensor on {device}")
    for name, t, shape, dtype, optional in specs:
        if t is None:
            if optional:
                continue
            raise ValueError(f"{name} is required")
        if t.device != device:
            raise ValueError(f"{name} is on {t.device}, the other tensors on {device}")
        if t.dtype != dtype:
            raise ValueError(f"{name} has dtype {t.dtype}, expected {dtype}")
        if tuple(t.shape) != tuple(shape):
            raise ValueError(f"{name} has shape {tuple(t.shape)}, expected {tuple(shape)}")


def _bytes(name, t, device) -> None:
    """A caller-owned byte buffer (workspace, saved state): a uint8 CUDA tensor on `device`, whose
    numel is the byte count the library is told."""
    if t is None:
        return
    if t.device != device or t.dtype != torch.uint8:
        raise ValueError(f"{name} must be a uint8 tensor on {device}, got {t.dtype} on {t.device}")


def _branch_specs(q, k, v, beta, alpha, gate, rms_w, conv_k_w, conv_v_w, text_state, F, out=None):
    """Specs of the branch's inputs (vdn.h, vdn_branch_forward) for q of shape [B, F*S, H, d]."""
    B, N, H, d = q.shape
    f32 = torch.float32
    K = conv_k_w.shape[-1] if conv_k_w is not None else (conv_v_w.shape[-1] if conv_v_w is not None else 1)
    return [("q", q, (B, N, H, d), q.dtype, False), ("k", k, (B, N, H, d), q.dtype, False),
            ("v", v, (B, N, H, d), q.dtype, False), ("gate", gate, (B, N, H, d), q.dtype, False),
            ("beta", beta, (B, N, H), f32, False), ("alpha", alpha, (B, F, H, d), f32, False),
            ("rms_w", rms_w, (d,), f32, False), ("conv_k_w", conv_k_w, (H, d, K), f32, True),
            ("conv_v_w", conv_v_w, (H, d, K), f32, True), ("text_state", text_state, (H, d, d), f32, True),
            ("out", out, (B, N, H, d), q.dtype, True)]


def _stream_ptr(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def make_shape(B, H, F, S, d, conv_width=3, dtype="bf16") -> VdnShape:
    if isinstance(dtype, torch.dtype):
        dtype = _TORCH_DTYPE[dtype]
    return VdnShape(B, H, F, S, d, conv_width, VDN_DTYPE[dtype])


def shape_from(q: torch.Tensor, F: int, conv_k_w=None) -> VdnShape:
    B, N, H, d = q.shape
    if N % F:
        raise ValueError(f"token count {N} is not a multiple of F={F}")
    K = 1 if conv_k_w is None else conv_k_w.shape[-1]
    return make_shape(B, H, F, N // F, d, K, q.dtype)


def workspace_size(shape: VdnShape, rule="vdn_solve", impl="auto") -> int:
    n = _lib.load().vdn_branch_workspace_size_impl(ctypes.byref(shape), VDN_RULE[rule], VDN_IMPL[impl])
    if n == 0:
        raise _lib.VdnError(_lib.VDN_ERR_INVALID_ARG, "vdn_branch_workspace_size")
    return n


def alloc_workspace(shape: VdnShape, rule="vdn_solve", impl="auto", device="cuda") -> torch.Tensor:
    return torch.empty(workspace_size(shape, rule, impl), dtype=torch.uint8, device=device)


def _forward_args(shape, q, k, v, beta, alpha, gate, rms_w, conv_k_w, conv_v_w, text_state, rule, c, chunk,
                  radius, workspace, out, stream):
    return (ctypes.byref(shape), _ptr(q), _ptr(k), _ptr(v), _ptr(beta), _ptr(alpha), _ptr(gate), _ptr(rms_w),
            _ptr(conv_k_w), _ptr(conv_v_w), _ptr(text_state), VDN_RULE[rule], float(c), int(chunk), int(radius),
            _ptr(workspace), workspace.numel(), _ptr(out), _stream_ptr(stream))


def branch_forward(q, k, v, beta, alpha, gate, rms_w, conv_k_w=None, conv_v_w=None, text_state=None, *,
                   F: int, rule="vdn_solve", c=1.0, chunk=5, radius=1, out=None, workspace=None, stream=None):
    """vdn_branch_forward: the whole branch.  Returns `out` ([B, F*S, H, d], q's dtype)."""
    shape = shape_from(q, F, conv_k_w if conv_k_w is not None else conv_v_w)
    _validate(_branch_specs(q, k, v, beta, alpha, gate, rms_w, conv_k_w, conv_v_w, text_state, F, out), q.device)
    if out is None:
        out = torch.empty_like(q)
    if workspace is None:
        workspace = alloc_workspace(shape, rule, "auto", q.device)
    _bytes("workspace", workspace, q.device)
    st = _lib.load().vdn_branch_forward(*_forward_args(shape, q, k, v, beta, alpha, gate, rms_w, conv_k_w,
                                                       conv_v_w, text_state, rule, c, chunk, radius, workspace,
                                                       out, stream))
    check(st, "vdn_branch_forward")
    return out


def window_softmax_forward(q_rope, k_rope, v, *, F: int, chunk=5, radius=1, scale=0.0, accumulate=False,
                           out=None, workspace=None, stream=None):
    """vdn_window_softmax_forward: the windowed softmax branch (out = or += its
    output).  Returns `out` ([B, F*S, H, d], q_rope's dtype)."""
    shape = shape_from(q_rope, F)
    _validate([(n, t, q_rope.shape, q_rope.dtype, n == "out") for n, t in
               (("q_rope", q_rope), ("k_rope", k_rope), ("v", v), ("out", out))], q_rope.device)
    if out is None:
        out = torch.zeros_like(q_rope) if accumulate else torch.empty_like(q_rope)
    if workspace is None:
        workspace = torch.empty(_lib.load().vdn_window_softmax_workspace_size(ctypes.byref(shape)),
                                dtype=torch.uint8, device=q_rope.device)
    _bytes("workspace", workspace, q_rope.device)
    st = _lib.load().vdn_window_softmax_forward(ctypes.byref(shape), _ptr(q_rope), _ptr(k_rope), _ptr(v), int(chunk),
                                                int(radius), float(scale), int(bool(accumulate)), _ptr(workspace),
                                                workspace.numel(), _ptr(out), _stream_ptr(stream))
    check(st, "vdn_window_softmax_forward")
    return out


def hybrid_forward(q_rope, k_rope, q, k, v, beta, alpha, gate, rms_w, conv_k_w=None, conv_v_w=None,
                   text_state=None, *, F: int, rule="vdn_solve", c=1.0, chunk=5, radius=1, scale=0.0, out=None,
                   workspace=None, stream=None):
    """vdn_hybrid_forward: windowed softmax branch + linear branch.  Returns `out`."""
    shape = shape_from(q, F, conv_k_w if conv_k_w is not None else conv_v_w)
    _validate(_branch_specs(q, k, v, beta, alpha, gate, rms_w, conv_k_w, conv_v_w, text_state, F, out) +
              [("q_rope", q_rope, q.shape, q.dtype, False), ("k_rope", k_rope, q.shape, q.dtype, False)], q.device)
    if out is None:
        out = torch.empty_like(q)
    if workspace is None:
        workspace = alloc_workspace(shape, rule, "auto", q.device)
    _bytes("workspace", workspace, q.device)
    fa = _forward_args(shape, q, k, v, beta, alpha, gate, rms_w, conv_k_w, conv_v_w, text_state, rule, c, chunk,
                       radius, workspace, out, stream)
    st = _lib.load().vdn_hybrid_forward(fa[0], _ptr(q_rope), _ptr(k_rope), *fa[1:15], float(scale), *fa[15:])
    check(st, "vdn_hybrid_forward")
    return out


def launch_count(shape: VdnShape, impl="auto") -> int:
    return _lib.load().vdn_branch_launch_count(ctypes.byref(shape), VDN_IMPL[impl])


def branch_forward_timed(q, k, v, beta, alpha, gate, rms_w, conv_k_w=None, conv_v_w=None, text_state=None, *,
                         F: int, events, rule="vdn_solve", c=1.0, chunk=5, radius=1, out=None, workspace=None,
                         stream=None):
    """vdn_branch_forward_timed: like branch_forward, recording `events` (torch.cuda.Event
    objects with timing enabled, already recorded once so their handles exist) before the
    first kernel and after each kernel."""
    shape = shape_from(q, F, conv_k_w if conv_k_w is not None else conv_v_w)
    _validate(_branch_specs(q, k, v, beta, alpha, gate, rms_w, conv_k_w, conv_v_w, text_state, F, out), q.device)
    if out is None:
        out = torch.empty_like(q)
    if workspace is None:
        workspace = alloc_workspace(shape, rule, "auto", q.device)
    _bytes("workspace", workspace, q.device)
    arr = (ctypes.c_void_p * len(events))(*[e.cuda_event for e in events])
    st = _lib.load().vdn_branch_forward_timed(*_forward_args(shape, q, k, v, beta, alpha, gate, rms_w, conv_k_w,
                                                             conv_v_w, text_state, rule, c, chunk, radius,
                                                             workspace, out, stream), arr, len(events))
    check(st, "vdn_branch_forward_timed")
    return out


DEBUG_FIELDS = ("A", "B", "N", "P", "Q", "W")


def branch_forward_debug(q, k, v, beta, alpha, gate, rms_w, conv_k_w=None, conv_v_w=None, text_state=None, *,
                         F: int, rule="vdn_solve", c=1.0, chunk=5, radius=1, impl="auto", want=DEBUG_FIELDS,
                         out=None, workspace=None, stream=None):
    """vdn_branch_forward_debug: returns (out, {name: fp32 [B, H, F, d, d]}) for the requested intermediates."""
    shape = shape_from(q, F, conv_k_w if conv_k_w is not None else conv_v_w)
    _validate(_branch_specs(q, k, v, beta, alpha, gate, rms_w, conv_k_w, conv_v_w, text_state, F, out), q.device)
    if out is None:
        out = torch.empty_like(q)
    if workspace is None:
        workspace = alloc_workspace(shape, rule, impl, q.device)
    _bytes("workspace", workspace, q.device)
    B, N, H, d = q.shape
    mats = {name: torch.full((B, H, F, d, d), float("nan"), dtype=torch.float32, device=q.device) for name in want}
    dbg = VdnDebugOut(VDN_IMPL[impl], *[mats[n].data_ptr() if n in mats else None for n in DEBUG_FIELDS])
    st = _lib.load().vdn_branch_forward_debug(*_forward_args(shape, q, k, v, beta, alpha, gate, rms_w, conv_k_w,
                                                             conv_v_w, text_state, rule, c, chunk, radius,
                                                             workspace, out, stream), ctypes.byref(dbg))
    check(st, "vdn_branch_forward_debug")
    return out, mats


def feature_prep(q, k, v, conv_k_w=None, conv_v_w=None, *, F: int, stream=None, out=None):
    """vdn_feature_prep: Step 1 alone.  Returns (q', k', v') in q's dtype (into `out`, a tuple
    of three tensors shaped like q, when given)."""
    shape = shape_from(q, F, conv_k_w if conv_k_w is not None else conv_v_w)
    _validate([s for s in _branch_specs(q, k, v, None, None, None, None, conv_k_w, conv_v_w, None, F)
               if s[0] in ("q", "k", "v", "conv_k_w", "conv_v_w")], q.device)
    if out is None:
        qo, ko, vo = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    else:
        qo, ko, vo = out
        _validate([("q_out", qo, q.shape, q.dtype, False), ("k_out", ko, q.shape, q.dtype, False),
                   ("v_out", vo, q.shape, q.dtype, False)], q.device)
    st = _lib.load().vdn_feature_prep(ctypes.byref(shape), _ptr(q), _ptr(k), _ptr(v), _ptr(conv_k_w),
                                      _ptr(conv_v_w), _ptr(qo), _ptr(ko), _ptr(vo), _stream_ptr(stream))
    check(st, "vdn_feature_prep")
    return qo, ko, vo


def window_bounds(t: int, F: int, chunk: int = 5, radius: int = 1):
    lo, hi = ctypes.c_int(), ctypes.c_int()
    check(_lib.load().vdn_window_bounds(t, F, chunk, radius, ctypes.byref(lo), ctypes.byref(hi)),
          "vdn_window_bounds")
    return lo.value, hi.value


def workspace_status(workspace: torch.Tensor, stream=None) -> int:
    return _lib.load().vdn_workspace_status(_ptr(workspace), workspace.numel(), _stream_ptr(stream))


def to_device(inp: dict, device="cuda") -> dict:
    """Copies the host tensors of synth.make_inputs to the device (None stays None)."""
    return {k: (None if t is None else t.to(device)) for k, t in inp.items()}


def saved_size(shape: VdnShape) -> int:
    n = _lib.load().vdn_branch_saved_size(ctypes.byref(shape))
    if n == 0:
        raise _lib.VdnError(_lib.VDN_ERR_INVALID_ARG, "vdn_branch_saved_size")
    return n


def branch_forward_train(q, k, v, beta, alpha, gate, rms_w, conv_k_w=None, conv_v_w=None, text_state=None, *,
                         F: int, rule="vdn_solve", c=1.0, chunk=5, radius=1, out=None, saved=None, workspace=None,
                         stream=None):
    """vdn_branch_forward_train: the branch's output and the per-frame state its backward
    reads.  Returns (out, saved); pass `saved` to branch_backward(..., saved=saved)."""
    shape = shape_from(q, F, conv_k_w if conv_k_w is not None else conv_v_w)
    _validate(_branch_specs(q, k, v, beta, alpha, gate, rms_w, conv_k_w, conv_v_w, text_state, F, out), q.device)
    if out is None:
        out = torch.empty_like(q)
    if saved is None:
        saved = torch.empty(saved_size(shape), dtype=torch.uint8, device=q.device)
    if workspace is None:
        workspace = alloc_workspace(shape, rule, "auto", q.device)
    _bytes("saved", saved, q.device)
    _bytes("workspace", workspace, q.device)
    fa = _forward_args(shape, q, k, v, beta, alpha, gate, rms_w, conv_k_w, conv_v_w, text_state, rule, c, chunk,
                       radius, workspace, out, stream)
    st = _lib.load().vdn_branch_forward_train(*fa[:-1], _ptr(saved), saved.numel(), fa[-1])
    check(st, "vdn_branch_forward_train")
    return out, saved


def backward_workspace_size(shape: VdnShape, rule="vdn_solve", saved=False) -> int:
    if saved:
        n = _lib.load().vdn_branch_backward_saved_workspace_size(ctypes.byref(shape), VDN_RULE[rule])
        if n == 0:
            raise _lib.VdnError(_lib.VDN_ERR_INVALID_ARG, "vdn_branch_backward_saved_workspace_size")
        return n
    n = _lib.load().vdn_branch_backward_workspace_size(ctypes.byref(shape), VDN_RULE[rule])
    if n == 0:
        raise _lib.VdnError(_lib.VDN_ERR_INVALID_ARG, "vdn_branch_backward_workspace_size")
    return n


def branch_backward(q, k, v, beta, alpha, gate, rms_w, conv_k_w=None, conv_v_w=None, text_state=None, *, dout,
                    F: int, rule="vdn_solve", c=1.0, chunk=5, radius=1, grads=None, workspace=None, stream=None,
                    events=None, saved=None):
    """vdn_branch_backward: gradients of <dout, branch_forward(...)> with respect to every
    input.  Returns a dict dq, dk, dv, dgate (q's dtype), dbeta, dalpha, drms_w, and
    dconv_k_w, dconv_v_w, dtext_state (fp32; None where the input is None).  With
    `events` (8 torch.cuda.Event), vdn_branch_backward_timed records them between the
    forward recompute and each backward kernel.  With `saved` (from branch_forward_train),
    vdn_branch_backward_saved runs instead, without the forward recompute."""
    shape = shape_from(q, F, conv_k_w if conv_k_w is not None else conv_v_w)
    dev = q.device
    specs = _branch_specs(q, k, v, beta, alpha, gate, rms_w, conv_k_w, conv_v_w, text_state, F)
    _validate(specs + [("dout", dout, q.shape, q.dtype, False)], dev)
    if grads is None:
        f32 = dict(dtype=torch.float32, device=dev)
        grads = {"dq": torch.empty_like(q), "dk": torch.empty_like(k), "dv": torch.empty_like(v),
                 "dgate": torch.empty_like(gate), "dbeta": torch.empty(beta.shape, **f32),
                 "dalpha": torch.empty(alpha.shape, **f32), "drms_w": torch.empty(rms_w.shape, **f32),
                 "dconv_k_w": None if conv_k_w is None else torch.empty(conv_k_w.shape, **f32),
                 "dconv_v_w": None if conv_v_w is None else torch.empty(conv_v_w.shape, **f32),
                 "dtext_state": None if text_state is None else torch.empty(text_state.shape, **f32)}
    if workspace is None:
        workspace = torch.empty(backward_workspace_size(shape, rule, saved is not None), dtype=torch.uint8,
                                device=dev)
    _bytes("workspace", workspace, dev)
    _bytes("saved", saved, dev)
    # each gradient has its input's shape: q's dtype for the token tensors, fp32 for the rest
    _validate([("d" + n, grads.get("d" + n), shp, dt if n in ("q", "k", "v", "gate") else torch.float32, True)
               for n, _, shp, dt, _ in specs if n != "out"], dev)
    g = grads
    args = (ctypes.byref(shape), _ptr(q), _ptr(k), _ptr(v), _ptr(beta), _ptr(alpha), _ptr(gate), _ptr(rms_w),
            _ptr(conv_k_w), _ptr(conv_v_w), _ptr(text_state), VDN_RULE[rule], float(c), int(chunk), int(radius),
            _ptr(dout), _ptr(workspace), workspace.numel(), _ptr(g["dq"]), _ptr(g["dk"]), _ptr(g["dv"]),
            _ptr(g["dbeta"]), _ptr(g["dalpha"]), _ptr(g["dgate"]), _ptr(g["drms_w"]), _ptr(g["dconv_k_w"]),
            _ptr(g["dconv_v_w"]), _ptr(g["dtext_state"]), _stream_ptr(stream))
    if saved is not None:
        if events is not None:
            raise ValueError("events are recorded by the recomputing backward only")
        st = _lib.load().vdn_branch_backward_saved(*args[:16], _ptr(saved), saved.numel(), *args[16:])
    elif events is None:
        st = _lib.load().vdn_branch_backward(*args)
    else:
        arr = (ctypes.c_void_p * len(events))(*[ctypes.c_void_p(e.cuda_event) for e in events])
        st = _lib.load().vdn_branch_backward_timed(*args, arr, len(events))
    check(st, "vdn_branch_backward")
    return grads


def forward_inputs(dev: dict):
    """Positional tensor arguments of branch_forward from a synth-style dict."""
    return (dev["q"], dev["k"], dev["v"], dev["beta"], dev["alpha"], dev["gate"], dev["rms_w"],
            dev.get("conv_k_w"), dev.get("conv_v_w"), dev.get("text_state"))


# ----------------------------------------------------------------------------- frame sharding
def frame_range(F: int, world: int, rank: int, chunk: int = 5) -> tuple[int, int]:
    """vdn_frame_range: the frames [f0, f1) rank `rank` of `world` owns under frame sharding
    (whole chunks, split as evenly as possible)."""
    f0, f1 = ctypes.c_int(), ctypes.c_int()
    check(_lib.load().vdn_frame_range(F, world, rank, chunk, ctypes.byref(f0), ctypes.byref(f1)), "vdn_frame_range")
    return f0.value, f1.value


def frame_owner(F: int, world: int, frame: int, chunk: int = 5) -> int:
    r = ctypes.c_int()
    check(_lib.load().vdn_frame_owner(F, world, chunk, frame, ctypes.byref(r)), "vdn_frame_owner")
    return r.value


def frames_map_bytes(shape: VdnShape, F_total: int, world: int, rank: int, chunk: int = 5) -> int:
    n = _lib.load().vdn_frames_map_bytes(ctypes.byref(shape), F_total, world, rank, chunk)
    if n == 0:
        raise _lib.VdnError(_lib.VDN_ERR_INVALID_ARG, "vdn_frames_map_bytes")
    return n


def frames_workspace_size(shape: VdnShape, F_total: int, world: int, rank: int, rule="vdn_solve",
                          chunk: int = 5) -> int:
    n = _lib.load().vdn_frames_workspace_size(ctypes.byref(shape), F_total, world, rank, VDN_RULE[rule], chunk)
    if n == 0:
        raise _lib.VdnError(_lib.VDN_ERR_INVALID_ARG, "vdn_frames_workspace_size")
    return n


def frames_maps(k, v, beta, alpha, conv_k_w=None, conv_v_w=None, *, F_total: int, world: int, rank: int,
                rule="vdn_solve", c=1.0, chunk=5, workspace=None, maps=None, stream=None) -> torch.Tensor:
    """vdn_frames_maps, phase 1 of the frame-sharded branch: k, v, beta, alpha hold the rank's
    frames only.  Returns the rank's per-chunk affine maps (flat fp32, frames_map_bytes / 4)."""
    f0, f1 = frame_range(F_total, world, rank, chunk)
    shape = shape_from(k, f1 - f0, conv_k_w if conv_k_w is not None else conv_v_w)
    _validate([s for s in _branch_specs(k, k, v, beta, alpha, k, None, conv_k_w, conv_v_w, None, f1 - f0)
               if s[0] in ("k", "v", "beta", "alpha", "conv_k_w", "conv_v_w")], k.device)
    nb = frames_map_bytes(shape, F_total, world, rank, chunk)
    if maps is None:
        maps = torch.empty(nb // 4, dtype=torch.float32, device=k.device)
    if workspace is None:
        workspace = torch.empty(frames_workspace_size(shape, F_total, world, rank, rule, chunk), dtype=torch.uint8,
                                device=k.device)
    _validate([("maps", maps, (maps.numel(),), torch.float32, False)], k.device)
    _bytes("workspace", workspace, k.device)
    st = _lib.load().vdn_frames_maps(ctypes.byref(shape), F_total, world, rank, _ptr(k), _ptr(v), _ptr(beta),
                                     _ptr(alpha), _ptr(conv_k_w), _ptr(conv_v_w), VDN_RULE[rule], float(c),
                                     int(chunk), _ptr(workspace), workspace.numel(), _ptr(maps),
                                     maps.numel() * maps.element_size(), _stream_ptr(stream))
    check(st, "vdn_frames_maps")
    return maps


def frames_finish(q, alpha_all, gate, rms_w, text_state, maps_all, *, F_total: int, world: int, rank: int,
                  rule="vdn_solve", c=1.0, chunk=5, radius=1, out=None, workspace=None, stream=None):
    """vdn_frames_finish, phase 2: q and gate hold the rank's frames, alpha_all the whole clip's,
    maps_all every rank's maps in rank order.  Returns the branch output of the rank's frames."""
    f0, f1 = frame_range(F_total, world, rank, chunk)
    shape = shape_from(q, f1 - f0)
    B, N, H, d = q.shape
    f32 = torch.float32
    _validate([("q", q, q.shape, q.dtype, False), ("gate", gate, q.shape, q.dtype, False),
               ("out", out, q.shape, q.dtype, True), ("alpha_all", alpha_all, (B, F_total, H, d), f32, False),
               ("rms_w", rms_w, (d,), f32, False), ("text_state", text_state, (H, d, d), f32, True),
               ("maps_all", maps_all, (maps_all.numel(),), f32, False)], q.device)
    if out is None:
        out = torch.empty_like(q)
    if workspace is None:
        workspace = torch.empty(frames_workspace_size(shape, F_total, world, rank, rule, chunk), dtype=torch.uint8,
                                device=q.device)
        workspace[:256].zero_()   # phase 2 keeps the device status word it is given
    _bytes("workspace", workspace, q.device)
    st = _lib.load().vdn_frames_finish(ctypes.byref(shape), F_total, world, rank, _ptr(q), _ptr(alpha_all),
                                       _ptr(gate), _ptr(rms_w), _ptr(text_state), VDN_RULE[rule], float(c),
                                       int(chunk), int(radius), _ptr(maps_all),
                                       maps_all.numel() * maps_all.element_size(), _ptr(workspace),
                                       workspace.numel(), _ptr(out), _stream_ptr(stream))
    check(st, "vdn_frames_finish")
    return out
