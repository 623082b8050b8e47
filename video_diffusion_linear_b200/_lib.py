"""ctypes loader of libvdn.so: declares the C ABI of include/vdn.h.

Fails loudly when the library is missing; there is no fallback implementation.
"""
from __future__ import annotations

import ctypes
import os
import re

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libvdn.so")
HEADER = os.path.join(os.path.dirname(_HERE), "include", "vdn.h")

VDN_OK, VDN_ERR_INVALID_ARG, VDN_ERR_UNSUPPORTED, VDN_ERR_ALIGNMENT, VDN_ERR_WORKSPACE, VDN_ERR_CUDA, \
    VDN_ERR_TIMEOUT = range(7)
VDN_RULE = {"sana_scaled": 0, "vdn_solve": 1, "vdn_scaled": 2, "additive": 3}
VDN_DTYPE = {"f32": 0, "bf16": 1}
VDN_IMPL = {"auto": 0, "simt": 1, "tc": 2}


class VdnShape(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int), ("H", ctypes.c_int), ("F", ctypes.c_int), ("S", ctypes.c_int),
                ("d", ctypes.c_int), ("conv_width", ctypes.c_int), ("dtype", ctypes.c_int)]


class VdnDebugOut(ctypes.Structure):
    _fields_ = [("impl", ctypes.c_int), ("A", ctypes.c_void_p), ("B", ctypes.c_void_p), ("N", ctypes.c_void_p),
                ("P", ctypes.c_void_p), ("Q", ctypes.c_void_p), ("W", ctypes.c_void_p)]


class VdnError(RuntimeError):
    def __init__(self, status: int, what: str):
        super().__init__(f"{what}: {string(status)} (status {status})")
        self.status = status


_P = ctypes.c_void_p
_FORWARD_ARGS = [ctypes.POINTER(VdnShape), _P, _P, _P, _P, _P, _P, _P, _P, _P, _P,
                 ctypes.c_int, ctypes.c_float, ctypes.c_int, ctypes.c_int, _P, ctypes.c_size_t, _P, _P]

_SIGNATURES = {
    "vdn_branch_workspace_size": (ctypes.c_size_t, [ctypes.POINTER(VdnShape), ctypes.c_int]),
    "vdn_branch_workspace_size_impl": (ctypes.c_size_t, [ctypes.POINTER(VdnShape), ctypes.c_int, ctypes.c_int]),
    "vdn_branch_forward": (ctypes.c_int, _FORWARD_ARGS),
    "vdn_branch_forward_debug": (ctypes.c_int, _FORWARD_ARGS + [ctypes.POINTER(VdnDebugOut)]),
    "vdn_branch_launch_count": (ctypes.c_int, [ctypes.POINTER(VdnShape), ctypes.c_int]),
    "vdn_branch_forward_timed": (ctypes.c_int, _FORWARD_ARGS + [ctypes.POINTER(ctypes.c_void_p), ctypes.c_int]),
    "vdn_feature_prep": (ctypes.c_int, [ctypes.POINTER(VdnShape), _P, _P, _P, _P, _P, _P, _P, _P, _P]),
    "vdn_window_softmax_workspace_size": (ctypes.c_size_t, [ctypes.POINTER(VdnShape)]),
    "vdn_window_softmax_forward": (ctypes.c_int, [ctypes.POINTER(VdnShape), _P, _P, _P, ctypes.c_int, ctypes.c_int,
                                                  ctypes.c_float, ctypes.c_int, _P, ctypes.c_size_t, _P, _P]),
    "vdn_hybrid_forward": (ctypes.c_int, [ctypes.POINTER(VdnShape), _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P,
                                          ctypes.c_int, ctypes.c_float, ctypes.c_int, ctypes.c_int, ctypes.c_float,
                                          _P, ctypes.c_size_t, _P, _P]),
    "vdn_window_bounds": (ctypes.c_int, [ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                         ctypes.POINTER(ctypes.c_int), ctypes.POINTER(ctypes.c_int)]),
    "vdn_branch_backward_workspace_size": (ctypes.c_size_t, [ctypes.POINTER(VdnShape), ctypes.c_int]),
    "vdn_branch_backward": (ctypes.c_int, [ctypes.POINTER(VdnShape), _P, _P, _P, _P, _P, _P, _P, _P, _P, _P,
                                           ctypes.c_int, ctypes.c_float, ctypes.c_int, ctypes.c_int, _P, _P,
                                           ctypes.c_size_t, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P]),
    "vdn_branch_backward_timed": (ctypes.c_int, [ctypes.POINTER(VdnShape), _P, _P, _P, _P, _P, _P, _P, _P, _P,
                                                 _P, ctypes.c_int, ctypes.c_float, ctypes.c_int, ctypes.c_int, _P,
                                                 _P, ctypes.c_size_t, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P,
                                                 ctypes.POINTER(ctypes.c_void_p), ctypes.c_int]),
    "vdn_branch_saved_size": (ctypes.c_size_t, [ctypes.POINTER(VdnShape)]),
    "vdn_branch_backward_saved_workspace_size": (ctypes.c_size_t, [ctypes.POINTER(VdnShape), ctypes.c_int]),
    "vdn_branch_forward_train": (ctypes.c_int, _FORWARD_ARGS[:-2] + [_P, _P, ctypes.c_size_t, _P]),
    "vdn_branch_backward_saved": (ctypes.c_int, [ctypes.POINTER(VdnShape), _P, _P, _P, _P, _P, _P, _P, _P, _P, _P,
                                                 ctypes.c_int, ctypes.c_float, ctypes.c_int, ctypes.c_int, _P, _P,
                                                 ctypes.c_size_t, _P, ctypes.c_size_t, _P, _P, _P, _P, _P, _P, _P,
                                                 _P, _P, _P, _P]),
    "vdn_frame_range": (ctypes.c_int, [ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                       ctypes.POINTER(ctypes.c_int), ctypes.POINTER(ctypes.c_int)]),
    "vdn_frame_owner": (ctypes.c_int, [ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                       ctypes.POINTER(ctypes.c_int)]),
    "vdn_frames_map_bytes": (ctypes.c_size_t, [ctypes.POINTER(VdnShape), ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                               ctypes.c_int]),
    "vdn_frames_workspace_size": (ctypes.c_size_t, [ctypes.POINTER(VdnShape), ctypes.c_int, ctypes.c_int,
                                                    ctypes.c_int, ctypes.c_int, ctypes.c_int]),
    "vdn_frames_maps": (ctypes.c_int, [ctypes.POINTER(VdnShape), ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                       _P, _P, _P, _P, _P, _P, ctypes.c_int, ctypes.c_float, ctypes.c_int,
                                       _P, ctypes.c_size_t, _P, ctypes.c_size_t, _P]),
    "vdn_frames_finish": (ctypes.c_int, [ctypes.POINTER(VdnShape), ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                         _P, _P, _P, _P, _P, ctypes.c_int, ctypes.c_float, ctypes.c_int,
                                         ctypes.c_int, _P, ctypes.c_size_t, _P, ctypes.c_size_t, _P, _P]),
    "vdn_workspace_status": (ctypes.c_int, [_P, ctypes.c_size_t, _P]),
    "vdn_status_string": (ctypes.c_char_p, [ctypes.c_int]),
}

_lib = None


def header_symbols() -> list[str]:
    """Function names declared in include/vdn.h."""
    text = open(HEADER).read()
    return sorted(set(re.findall(r"\b(vdn_[a-z_0-9]+)\s*\(", text)))


def load(path: str = LIB_PATH) -> ctypes.CDLL:
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise RuntimeError(f"libvdn.so not built ({path}); run python -m video_diffusion_linear_b200.build")
    lib = ctypes.CDLL(path)
    for name, (res, args) in _SIGNATURES.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    _lib = lib
    return lib


def string(status: int) -> str:
    try:
        return load().vdn_status_string(status).decode()
    except Exception:
        return "unknown"


def check(status: int, what: str) -> None:
    if status != VDN_OK:
        raise VdnError(status, what)
