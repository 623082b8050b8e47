"""Host-side checks of the C ABI: the library loads, exports every function that
include/vdn.h declares, and rejects bad arguments before any CUDA call (so these
run without a GPU: the pointers below are never dereferenced)."""
import ctypes

import pytest

from oracle import vdn_oracle as O
from video_diffusion_linear_b200 import _lib
from video_diffusion_linear_b200._lib import (VDN_ERR_ALIGNMENT, VDN_ERR_INVALID_ARG, VDN_ERR_UNSUPPORTED,
                                              VDN_ERR_WORKSPACE, VDN_OK, VdnShape)


def test_exports_every_header_symbol(lib):
    names = _lib.header_symbols()
    assert "vdn_branch_forward" in names and len(names) >= 8
    for n in names:
        assert hasattr(lib, n), n


def test_status_strings(lib):
    for s in range(7):
        assert lib.vdn_status_string(s).decode() != "unknown status"
    assert lib.vdn_status_string(99).decode() == "unknown status"


@pytest.mark.parametrize("chunk", [1, 2, 5, 7])
@pytest.mark.parametrize("radius", [0, 1, 3])
def test_window_bounds_matches_oracle(lib, chunk, radius):
    lo, hi = ctypes.c_int(), ctypes.c_int()
    for F in (1, 9, 31, 85):
        for t in range(F):
            assert lib.vdn_window_bounds(t, F, chunk, radius, ctypes.byref(lo), ctypes.byref(hi)) == VDN_OK
            assert (lo.value, hi.value) == O.window_bounds(t, F, chunk, radius)
    assert lib.vdn_window_bounds(5, 5, 5, 1, ctypes.byref(lo), ctypes.byref(hi)) == VDN_ERR_INVALID_ARG
    assert lib.vdn_window_bounds(0, 5, 0, 1, ctypes.byref(lo), ctypes.byref(hi)) == VDN_ERR_INVALID_ARG


def _shape(**kw):
    base = dict(B=1, H=2, F=12, S=100, d=128, conv_width=3, dtype=1)
    base.update(kw)
    return VdnShape(**base)


BASE = 1 << 40      # fake, 4 KiB-aligned device addresses, far apart
GAP = 1 << 34


def _args(shape, ws_bytes=None, **over):
    ptr = {name: BASE + i * GAP for i, name in enumerate(
        ["q", "k", "v", "beta", "alpha", "gate", "rms_w", "conv_k_w", "conv_v_w", "text", "ws", "out"])}
    ptr.update(over)
    if ws_bytes is None:
        ws_bytes = _lib.load().vdn_branch_workspace_size(ctypes.byref(shape), 1)
    P = lambda n: None if ptr[n] is None else ctypes.c_void_p(ptr[n])
    return (ctypes.byref(shape), P("q"), P("k"), P("v"), P("beta"), P("alpha"), P("gate"), P("rms_w"),
            P("conv_k_w"), P("conv_v_w"), P("text"), 1, 1.0, 5, 1, P("ws"), ws_bytes, P("out"), None)


def test_workspace_size(lib):
    s = _shape()
    n = lib.vdn_branch_workspace_size(ctypes.byref(s), 1)
    assert n > 0 and n % 256 == 0
    assert lib.vdn_branch_workspace_size(ctypes.byref(_shape(d=64)), 1) == 0
    assert lib.vdn_branch_workspace_size(ctypes.byref(s), 9) == 0
    assert lib.vdn_branch_workspace_size_impl(ctypes.byref(_shape(dtype=1, d=16)), 1, 0) == 0
    assert lib.vdn_branch_workspace_size_impl(ctypes.byref(_shape(dtype=0, d=16)), 1, 2) == 0
    assert lib.vdn_branch_workspace_size_impl(ctypes.byref(_shape(dtype=0, d=16)), 1, 1) > 0


@pytest.mark.parametrize("case,expect", [
    (dict(shape=dict(d=64)), VDN_ERR_UNSUPPORTED),
    (dict(shape=dict(d=16, dtype=1)), VDN_ERR_UNSUPPORTED),
    (dict(shape=dict(conv_width=5)), VDN_ERR_UNSUPPORTED),
    (dict(shape=dict(S=0)), VDN_ERR_INVALID_ARG),
    (dict(shape=dict(B=-1)), VDN_ERR_INVALID_ARG),
    (dict(shape=dict(dtype=7)), VDN_ERR_INVALID_ARG),
    (dict(ptr=dict(q=None)), VDN_ERR_INVALID_ARG),
    (dict(ptr=dict(out=None)), VDN_ERR_INVALID_ARG),
    (dict(ptr=dict(ws=None)), VDN_ERR_INVALID_ARG),
    (dict(ptr=dict(q=BASE + 8)), VDN_ERR_ALIGNMENT),
    (dict(ptr=dict(beta=BASE + 3 * GAP + 4)), VDN_ERR_ALIGNMENT),
    (dict(ptr=dict(ws=BASE + 10 * GAP + 64)), VDN_ERR_ALIGNMENT),
    (dict(ptr=dict(out=BASE + 64)), VDN_ERR_INVALID_ARG),               # out overlaps q
    (dict(ptr=dict(out=BASE + 10 * GAP + 256)), VDN_ERR_INVALID_ARG),   # out overlaps the workspace
    (dict(ws_bytes=1024), VDN_ERR_WORKSPACE),
])
def test_validation_rejects_before_launch(lib, case, expect):
    s = _shape(**case.get("shape", {}))
    args = _args(s, case.get("ws_bytes", 1 << 40), **case.get("ptr", {}))
    assert lib.vdn_branch_forward(*args) == expect


def test_bad_rule_and_window_args(lib):
    s = _shape()
    args = list(_args(s, 1 << 40))
    for idx, val in ((11, 4), (11, -1), (13, 0), (14, -1), (12, float("nan"))):
        a = list(args)
        a[idx] = val
        assert lib.vdn_branch_forward(*a) == VDN_ERR_INVALID_ARG, (idx, val)


def test_feature_prep_validation(lib):
    s = _shape()
    p = lambda i: ctypes.c_void_p(BASE + i * GAP)
    assert lib.vdn_feature_prep(ctypes.byref(s), p(0), p(1), p(2), None, None, p(0), p(4), p(5), None) == \
        VDN_ERR_INVALID_ARG
    assert lib.vdn_feature_prep(ctypes.byref(s), p(0), p(1), p(2), None, None, p(3), p(3), p(5), None) == \
        VDN_ERR_INVALID_ARG
    assert lib.vdn_feature_prep(ctypes.byref(s), None, p(1), p(2), None, None, p(3), p(4), p(5), None) == \
        VDN_ERR_INVALID_ARG
    assert lib.vdn_feature_prep(ctypes.byref(_shape(d=32)), p(0), p(1), p(2), None, None, p(3), p(4), p(5),
                                None) == VDN_ERR_UNSUPPORTED


def _bwd_args(shape, ws_bytes=1 << 40, **over):
    names = ["q", "k", "v", "beta", "alpha", "gate", "rms_w", "conv_k_w", "conv_v_w", "text", "dout", "ws",
             "dq", "dk", "dv", "dbeta", "dalpha", "dgate", "drms_w", "dconv_k_w", "dconv_v_w", "dtext"]
    ptr = {name: BASE + i * GAP for i, name in enumerate(names)}
    ptr.update(over)
    P = lambda n: None if ptr[n] is None else ctypes.c_void_p(ptr[n])
    return (ctypes.byref(shape), P("q"), P("k"), P("v"), P("beta"), P("alpha"), P("gate"), P("rms_w"),
            P("conv_k_w"), P("conv_v_w"), P("text"), 1, 1.0, 5, 1, P("dout"), P("ws"), ws_bytes, P("dq"), P("dk"),
            P("dv"), P("dbeta"), P("dalpha"), P("dgate"), P("drms_w"), P("dconv_k_w"), P("dconv_v_w"), P("dtext"),
            None)


def test_backward_workspace_size(lib):
    s = _shape()
    n = lib.vdn_branch_backward_workspace_size(ctypes.byref(s), 1)
    assert n > lib.vdn_branch_workspace_size(ctypes.byref(s), 1) and n % 256 == 0
    assert lib.vdn_branch_backward_workspace_size(ctypes.byref(_shape(d=64)), 1) == 0
    assert lib.vdn_branch_backward_workspace_size(ctypes.byref(s), 9) == 0


@pytest.mark.parametrize("case,expect", [
    (dict(ptr=dict(dout=None)), VDN_ERR_INVALID_ARG),
    (dict(ptr=dict(dalpha=None)), VDN_ERR_INVALID_ARG),
    (dict(ptr=dict(dconv_k_w=None)), VDN_ERR_INVALID_ARG),              # taps given, no tap gradient
    (dict(ptr=dict(text=None)), VDN_ERR_INVALID_ARG),                   # text gradient without a text state
    (dict(ptr=dict(dq=BASE + 64)), VDN_ERR_INVALID_ARG),                # dq overlaps q
    (dict(ptr=dict(dk=BASE + 12 * GAP + 512)), VDN_ERR_INVALID_ARG),    # dk overlaps dq
    (dict(ptr=dict(dbeta=BASE + 10 * GAP)), VDN_ERR_INVALID_ARG),       # dbeta overlaps dout
    (dict(ptr=dict(dgate=BASE + 11 * GAP + 4096)), VDN_ERR_INVALID_ARG),  # dgate overlaps the workspace
    (dict(ptr=dict(dalpha=BASE + 16 * GAP + 8)), VDN_ERR_ALIGNMENT),
    (dict(ws_bytes=1 << 20), VDN_ERR_WORKSPACE),
    (dict(shape=dict(d=64)), VDN_ERR_UNSUPPORTED),
])
def test_backward_validation_rejects_before_launch(lib, case, expect):
    s = _shape(**case.get("shape", {}))
    args = _bwd_args(s, case.get("ws_bytes", 1 << 40), **case.get("ptr", {}))
    assert lib.vdn_branch_backward(*args) == expect


def test_saved_state_sizes(lib):
    s = _shape()
    n = lib.vdn_branch_saved_size(ctypes.byref(s))
    assert n > 0 and n % 256 == 0
    w_saved = lib.vdn_branch_backward_saved_workspace_size(ctypes.byref(s), 1)
    assert 0 < w_saved < lib.vdn_branch_backward_workspace_size(ctypes.byref(s), 1)
    assert lib.vdn_branch_saved_size(ctypes.byref(_shape(d=64))) == 0


def _saved_args(shape, saved=BASE + 30 * GAP, saved_bytes=1 << 40, ws=BASE + 11 * GAP):
    args = list(_bwd_args(shape))
    # vdn_branch_backward_saved: ..., dout, saved, saved_bytes, workspace, workspace_bytes, gradients..., stream
    head, tail = args[:16], args[16:]
    tail[0] = ctypes.c_void_p(ws)
    return head + [None if saved is None else ctypes.c_void_p(saved), saved_bytes] + tail


@pytest.mark.parametrize("case,expect", [
    (dict(saved=None), VDN_ERR_INVALID_ARG),
    (dict(saved_bytes=1024), VDN_ERR_WORKSPACE),
    (dict(saved=BASE + 30 * GAP + 16), VDN_ERR_ALIGNMENT),
    (dict(saved=BASE + 11 * GAP + 4096), VDN_ERR_INVALID_ARG),        # saved state overlaps the workspace
    (dict(saved=BASE + 12 * GAP), VDN_ERR_INVALID_ARG),               # saved state overlaps dq
])
def test_backward_saved_validation(lib, case, expect):
    s = _shape()
    assert lib.vdn_branch_backward_saved(*_saved_args(s, **case)) == expect


def test_forward_train_validation(lib):
    s = _shape()
    base = list(_args(s, 1 << 40))
    # vdn_branch_forward_train: forward arguments up to out, then saved, saved_bytes, stream
    def call(saved, nbytes):
        return lib.vdn_branch_forward_train(*base[:-1], None if saved is None else ctypes.c_void_p(saved), nbytes,
                                            None)
    assert call(None, 1 << 40) == VDN_ERR_INVALID_ARG
    assert call(BASE + 30 * GAP, 1024) == VDN_ERR_WORKSPACE
    assert call(BASE + 30 * GAP + 64, 1 << 40) == VDN_ERR_ALIGNMENT
    assert call(BASE + 11 * GAP, 1 << 40) == VDN_ERR_INVALID_ARG       # overlaps the output
    assert call(BASE + 10 * GAP, 1 << 40) == VDN_ERR_INVALID_ARG       # overlaps the workspace


def _soft_args(shape, chunk=5, radius=1, scale=0.0, accumulate=0, ws_bytes=256, **over):
    names = ["q_rope", "k_rope", "v", "ws", "out"]
    ptr = {name: BASE + i * GAP for i, name in enumerate(names)}
    ptr.update(over)
    P = lambda n: None if ptr[n] is None else ctypes.c_void_p(ptr[n])
    return (ctypes.byref(shape), P("q_rope"), P("k_rope"), P("v"), chunk, radius, scale, accumulate, P("ws"),
            ws_bytes, P("out"), None)


@pytest.mark.parametrize("case,expect", [
    (dict(chunk=0), VDN_ERR_INVALID_ARG),
    (dict(radius=-1), VDN_ERR_INVALID_ARG),
    (dict(scale=float("nan")), VDN_ERR_INVALID_ARG),
    (dict(scale=float("inf")), VDN_ERR_INVALID_ARG),
    (dict(accumulate=2), VDN_ERR_INVALID_ARG),
    (dict(q_rope=None), VDN_ERR_INVALID_ARG),
    (dict(out=None), VDN_ERR_INVALID_ARG),
    (dict(ws=None), VDN_ERR_INVALID_ARG),
    (dict(k_rope=BASE + GAP + 8), VDN_ERR_ALIGNMENT),
    (dict(ws=BASE + 3 * GAP + 64), VDN_ERR_ALIGNMENT),
    (dict(ws_bytes=128), VDN_ERR_WORKSPACE),
    (dict(out=BASE + 2 * GAP + 4096), VDN_ERR_INVALID_ARG),            # out overlaps v
    (dict(out=BASE + 3 * GAP), VDN_ERR_INVALID_ARG),                   # out overlaps the status word
])
def test_window_softmax_validation(lib, case, expect):
    s = _shape()
    assert lib.vdn_window_softmax_forward(*_soft_args(s, **case)) == expect


def test_window_softmax_unsupported_shapes(lib):
    assert lib.vdn_window_softmax_forward(*_soft_args(_shape(d=64))) == VDN_ERR_UNSUPPORTED
    assert lib.vdn_window_softmax_forward(*_soft_args(_shape(d=16, dtype=1))) == VDN_ERR_UNSUPPORTED
    assert lib.vdn_window_softmax_workspace_size(ctypes.byref(_shape())) == 256
    assert lib.vdn_window_softmax_workspace_size(ctypes.byref(_shape(d=64))) == 0


def test_hybrid_validation(lib):
    s = _shape()
    fwd = list(_args(s, 1 << 40))
    # vdn_hybrid_forward: shape, q_rope, k_rope, then the forward's tensors, rule, c, chunk, radius, scale,
    # workspace, workspace_bytes, out, stream
    qr, kr = ctypes.c_void_p(BASE + 20 * GAP), ctypes.c_void_p(BASE + 21 * GAP)
    def call(scale=0.0, qr_=qr, out=fwd[17]):
        return lib.vdn_hybrid_forward(fwd[0], qr_, kr, *fwd[1:15], scale, fwd[15], fwd[16], out, None)
    assert call(scale=float("nan")) == VDN_ERR_INVALID_ARG
    assert call(qr_=None) == VDN_ERR_INVALID_ARG
    assert call(qr_=ctypes.c_void_p(BASE + 20 * GAP + 4)) == VDN_ERR_ALIGNMENT
    assert call(out=ctypes.c_void_p(BASE + 21 * GAP + 256)) == VDN_ERR_INVALID_ARG   # out overlaps k_rope
    assert call(out=ctypes.c_void_p(BASE + 64)) == VDN_ERR_INVALID_ARG               # out overlaps q


def test_every_export_is_declared(lib):
    # the boundary is the header: nothing the library exports is left undocumented
    import shutil
    import subprocess
    nm = shutil.which("nm")
    if nm is None:
        pytest.skip("nm not available")
    out = subprocess.run([nm, "-D", "--defined-only", _lib.LIB_PATH], capture_output=True, text=True,
                         check=True).stdout
    exported = {ln.split()[-1] for ln in out.splitlines() if ln.split()[-2:-1] == ["T"]}
    exported = {n for n in exported if n.startswith("vdn_")}
    assert exported and exported <= set(_lib.header_symbols()), exported - set(_lib.header_symbols())


@pytest.mark.parametrize("kw", [
    dict(F=70000, S=40000),              # F*S tokens of one batch element past int32
    dict(B=40000, H=60000, F=1, S=1),    # (batch, head, frame) triples past int32
    dict(B=1 << 20, H=1 << 11, F=1, S=1),   # 2 B H past int32
])
def test_index_ranges_past_int32_are_refused(lib, kw):
    # the kernels index tokens of one batch element and (batch, head, frame) triples in int32:
    # shapes beyond that are refused before any allocation or launch, by every entry point
    s = _shape(**kw)
    assert lib.vdn_branch_workspace_size(ctypes.byref(s), 1) == 0
    assert lib.vdn_branch_forward(*_args(s, ws_bytes=1 << 40)) == VDN_ERR_UNSUPPORTED
    assert lib.vdn_window_softmax_workspace_size(ctypes.byref(s)) == 0
    assert lib.vdn_branch_backward_workspace_size(ctypes.byref(s), 1) == 0


def test_largest_single_gpu_sizes_are_accepted(lib):
    # the 14 s and 1024^2 clips, and a 4x longer clip: sizes only (nothing runs)
    for kw in (dict(F=85, S=1560, H=24), dict(B=2, F=31, S=4096, H=24), dict(F=340, S=1560, H=24)):
        s = _shape(**kw)
        n = lib.vdn_branch_workspace_size(ctypes.byref(s), 1)
        assert 0 < n < 180e9


def test_static_forward_refuses_before_any_cuda_call(lib):
    # without a GPU any CUDA call would fail: a too-large problem must be refused by its size
    # alone (VDN_ERR_WORKSPACE), an invalid shape by the regular validation
    fn = lib.vdn_branch_forward_static
    fn.restype = ctypes.c_int
    fn.argtypes = ([ctypes.POINTER(VdnShape)] + [ctypes.c_void_p] * 10
                   + [ctypes.c_int, ctypes.c_float, ctypes.c_int, ctypes.c_int, ctypes.c_void_p, ctypes.c_void_p])
    big = _shape(H=24, F=31, S=4032)                       # the 768p clip
    assert lib.vdn_branch_workspace_size(ctypes.byref(big), 1) > 64 << 20
    a = _args(big)
    assert fn(*(a[:15] + a[17:])) == VDN_ERR_WORKSPACE
    bad = _shape(H=24, F=31, S=4032, d=64)
    assert fn(*((ctypes.byref(bad),) + a[1:15] + a[17:])) == VDN_ERR_UNSUPPORTED


def test_workspace_status_argument_checks(lib):
    fn = lib.vdn_workspace_status
    fn.restype = ctypes.c_int
    fn.argtypes = [ctypes.c_void_p, ctypes.c_size_t, ctypes.c_void_p]
    assert fn(None, 1 << 20, None) == VDN_ERR_INVALID_ARG
    assert fn(ctypes.c_void_p(BASE), 16, None) == VDN_ERR_INVALID_ARG
