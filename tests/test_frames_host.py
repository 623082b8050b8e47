"""Host-side checks of the frame-sharding entry points (no GPU: every call below is rejected or
answered before any CUDA call, and the pointers are never dereferenced): the partition agrees
with shard.frame_range and the window geometry, the map and workspace sizes, and the argument
validation of both phases."""
import ctypes

import pytest

from oracle import vdn_oracle as O
from video_diffusion_linear_b200 import _lib, api, shard
from video_diffusion_linear_b200._lib import (VDN_ERR_ALIGNMENT, VDN_ERR_INVALID_ARG, VDN_ERR_UNSUPPORTED,
                                              VDN_ERR_WORKSPACE, VDN_OK, VdnShape)


@pytest.fixture(scope="module")
def lib():
    return _lib.load()


@pytest.mark.parametrize("F,chunk", [(1, 5), (5, 5), (23, 3), (30, 2), (31, 5), (85, 5), (100, 16)])
@pytest.mark.parametrize("world", [1, 2, 3, 4, 8])
def test_partition_matches_the_host_plan(lib, F, chunk, world):
    C = -(-F // chunk)
    f0, f1 = ctypes.c_int(), ctypes.c_int()
    if world > C:
        assert lib.vdn_frame_range(F, world, 0, chunk, ctypes.byref(f0), ctypes.byref(f1)) == VDN_ERR_INVALID_ARG
        return
    for r in range(world):
        assert lib.vdn_frame_range(F, world, r, chunk, ctypes.byref(f0), ctypes.byref(f1)) == VDN_OK
        assert (f0.value, f1.value) == shard.frame_range(F, world, r, chunk)
    # the owner rule the fold kernel uses (shared with vdn_frame_owner) agrees with the ranges
    for f in range(F):
        a, b = shard.frame_range(F, world, api.frame_owner(F, world, f, chunk), chunk)
        assert a <= f < b


def test_partition_rejects_bad_arguments(lib):
    f0, f1, r = ctypes.c_int(), ctypes.c_int(), ctypes.c_int()
    for args in [(0, 1, 0, 5), (10, 0, 0, 5), (10, 2, 2, 5), (10, 2, -1, 5), (10, 2, 0, 0)]:
        assert lib.vdn_frame_range(*args, ctypes.byref(f0), ctypes.byref(f1)) == VDN_ERR_INVALID_ARG
    assert lib.vdn_frame_range(10, 2, 0, 5, None, ctypes.byref(f1)) == VDN_ERR_INVALID_ARG
    assert lib.vdn_frame_owner(10, 2, 5, 10, ctypes.byref(r)) == VDN_ERR_INVALID_ARG
    assert lib.vdn_frame_owner(10, 2, 5, -1, ctypes.byref(r)) == VDN_ERR_INVALID_ARG
    assert lib.vdn_frame_owner(10, 3, 5, 0, ctypes.byref(r)) == VDN_ERR_INVALID_ARG   # 2 chunks, 3 ranks


@pytest.mark.parametrize("F,chunk,radius,world", [(23, 3, 1, 3), (30, 2, 6, 3), (31, 5, 1, 4), (20, 2, 4, 4)])
def test_every_chunk_edge_state_a_window_reads_is_folded(F, chunk, radius, world):
    # the fold writes P at the last frame of chunks 0 .. C-2 and Q at the first frame of chunks
    # 1 .. C-1; every state a window of any rank reads is among them
    C = -(-F // chunk)
    p_written = {(c + 1) * chunk - 1 for c in range(C - 1)}
    q_written = {c * chunk for c in range(1, C)}
    assert all(f < F for f in p_written | q_written)
    for t in range(F):
        lo, hi = O.window_bounds(t, F, chunk, radius)
        if lo > 0:
            assert lo - 1 in p_written
        if hi < F - 1:
            assert hi + 1 in q_written


def _shape(**kw):
    base = dict(B=1, H=2, F=9, S=40, d=128, conv_width=3, dtype=1)
    base.update(kw)
    return VdnShape(**base)


def _map_bytes(B, H, nch, d=128):
    """The header's rank buffer: fp32 maps [B*H][2][nch][G | O][d][d], then int32 exponents
    [B*H][2][nch][G | O], padded to 16 bytes."""
    n = B * H * 2 * nch * 2 * d * d * 4 + B * H * 2 * nch * 2 * 4
    return (n + 15) // 16 * 16


def test_map_bytes_and_workspace(lib):
    s = _shape()                                   # rank 0 of 3 over 23 frames in chunks of 3: 9 frames
    assert lib.vdn_frames_map_bytes(ctypes.byref(s), 23, 3, 0, 3) == _map_bytes(1, 2, 3)
    s2 = _shape(F=5)                               # rank 2 owns the last two chunks (3 + 2 frames)
    assert lib.vdn_frames_map_bytes(ctypes.byref(s2), 23, 3, 2, 3) == _map_bytes(1, 2, 3)
    s3 = _shape(B=3, H=1, F=5)                     # an exponent block that is not a multiple of 16 bytes
    assert lib.vdn_frames_map_bytes(ctypes.byref(s3), 23, 3, 2, 3) == _map_bytes(3, 1, 3)
    n = lib.vdn_frames_workspace_size(ctypes.byref(s), 23, 3, 0, 1, 3)
    assert n > 0 and n % 256 == 0
    # the clip-wide chunk-edge banks: two [B, H, F_total, d, d] fp32 regions at least
    assert n >= 2 * 1 * 2 * 23 * 128 * 128 * 4
    for bad in [dict(shape=_shape(dtype=0, d=16)), dict(shape=_shape(dtype=0)), dict(shape=_shape(F=8)),
                dict(chunk=17, shape=_shape(F=17)), dict(world=9)]:
        sh = bad.get("shape", s)
        expect0 = lib.vdn_frames_map_bytes(ctypes.byref(sh), 23, bad.get("world", 3), 0, bad.get("chunk", 3))
        assert expect0 == 0, bad
        assert lib.vdn_frames_workspace_size(ctypes.byref(sh), 23, bad.get("world", 3), 0, 1, bad.get("chunk", 3)) == 0


BASE = 1 << 40
GAP = 1 << 34


def _maps_args(shape, **over):
    names = ["k", "v", "beta", "alpha", "conv_k_w", "conv_v_w", "ws", "maps"]
    ptr = {n: BASE + i * GAP for i, n in enumerate(names)}
    ptr.update(over.pop("ptr", {}))
    lib = _lib.load()
    ws = over.pop("ws_bytes", lib.vdn_frames_workspace_size(ctypes.byref(shape), 23, 3, 0, 1, 3))
    mb = over.pop("map_bytes", 1 << 30)
    P = lambda n: None if ptr[n] is None else ctypes.c_void_p(ptr[n])
    a = dict(F_total=23, world=3, rank=0, rule=1, c=1.0, chunk=3)
    a.update(over)
    return (ctypes.byref(shape), a["F_total"], a["world"], a["rank"], P("k"), P("v"), P("beta"), P("alpha"),
            P("conv_k_w"), P("conv_v_w"), a["rule"], a["c"], a["chunk"], P("ws"), ws, P("maps"), mb, None)


@pytest.mark.parametrize("case,expect", [
    (dict(shape=dict(dtype=0)), VDN_ERR_UNSUPPORTED),
    (dict(shape=dict(F=8)), VDN_ERR_INVALID_ARG),                 # not rank 0's 9 frames
    (dict(rank=3), VDN_ERR_INVALID_ARG),
    (dict(world=9), VDN_ERR_INVALID_ARG),                          # 8 chunks cannot feed 9 ranks
    (dict(rule=7), VDN_ERR_INVALID_ARG),
    (dict(c=float("nan")), VDN_ERR_INVALID_ARG),
    (dict(ptr=dict(k=None)), VDN_ERR_INVALID_ARG),
    (dict(ptr=dict(maps=None)), VDN_ERR_INVALID_ARG),
    (dict(ptr=dict(beta=BASE + 2 * GAP + 4)), VDN_ERR_ALIGNMENT),
    (dict(ptr=dict(ws=BASE + 6 * GAP + 16)), VDN_ERR_ALIGNMENT),
    (dict(ws_bytes=1024), VDN_ERR_WORKSPACE),
    (dict(map_bytes=1024), VDN_ERR_INVALID_ARG),
    (dict(ptr=dict(maps=BASE + 1 * GAP + 64)), VDN_ERR_INVALID_ARG),   # maps inside v
])
def test_maps_validation(lib, case, expect):
    case = dict(case)
    shape = _shape(**case.pop("shape", {}))
    assert lib.vdn_frames_maps(*_maps_args(shape, **case)) == expect


def _finish_args(shape, **over):
    names = ["q", "alpha_all", "gate", "rms_w", "text", "maps_all", "ws", "out"]
    ptr = {n: BASE + i * GAP for i, n in enumerate(names)}
    ptr.update(over.pop("ptr", {}))
    lib = _lib.load()
    ws = over.pop("ws_bytes", lib.vdn_frames_workspace_size(ctypes.byref(shape), 23, 3, 0, 1, 3))
    mb = over.pop("maps_all_bytes", 1 << 30)
    P = lambda n: None if ptr[n] is None else ctypes.c_void_p(ptr[n])
    a = dict(F_total=23, world=3, rank=0, rule=1, c=1.0, chunk=3, radius=1)
    a.update(over)
    return (ctypes.byref(shape), a["F_total"], a["world"], a["rank"], P("q"), P("alpha_all"), P("gate"), P("rms_w"),
            P("text"), a["rule"], a["c"], a["chunk"], a["radius"], P("maps_all"), mb, P("ws"), ws, P("out"), None)


@pytest.mark.parametrize("case,expect", [
    (dict(shape=dict(d=16)), VDN_ERR_UNSUPPORTED),
    (dict(chunk=17, F_total=40, shape=dict(F=17)), VDN_ERR_UNSUPPORTED),
    (dict(shape=dict(F=10)), VDN_ERR_INVALID_ARG),
    (dict(radius=-1), VDN_ERR_INVALID_ARG),
    (dict(ptr=dict(q=None)), VDN_ERR_INVALID_ARG),
    (dict(ptr=dict(alpha_all=None)), VDN_ERR_INVALID_ARG),
    (dict(ptr=dict(out=None)), VDN_ERR_INVALID_ARG),
    (dict(ptr=dict(out=BASE + 7 * GAP + 8)), VDN_ERR_ALIGNMENT),
    (dict(ws_bytes=4096), VDN_ERR_WORKSPACE),
    (dict(maps_all_bytes=3 * 1024), VDN_ERR_INVALID_ARG),         # fewer than world map buffers
    (dict(ptr=dict(out=BASE + 0 * GAP + 256)), VDN_ERR_INVALID_ARG),   # out inside q
    (dict(ptr=dict(out=BASE + 6 * GAP + 4096)), VDN_ERR_INVALID_ARG),  # out inside the workspace
    (dict(ptr=dict(maps_all=BASE + 6 * GAP + 1024)), VDN_ERR_INVALID_ARG),  # maps inside the workspace
])
def test_finish_validation(lib, case, expect):
    case = dict(case)
    shape = _shape(**case.pop("shape", {}))
    assert lib.vdn_frames_finish(*_finish_args(shape, **case)) == expect
