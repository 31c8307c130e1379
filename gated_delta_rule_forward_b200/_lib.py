"""ctypes loader for libgdr.so (built in-tree by csrc/build.py).

Loading never falls back to anything: if the shared library is missing or
does not export the ABI, ``lib()`` raises.
"""
from __future__ import annotations

import ctypes
import os
import threading

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libgdr.so")

EXPORTS = (
    "gdr_forward_workspace_size", "gdr_forward_chunked", "gdr_decode_step",
    "gdr_forward_launches", "gdr_forward_kernel_name", "gdr_status_string",
    "gdr_last_error", "gdr_version", "gdr_device_status", "gdr_forward_chunked_noalloc",
    "gdr_forward_plan", "gdr_forward_segment_parts", "gdr_backward_workspace_size", "gdr_backward",
)

STATUS = {0: "GDR_OK", 1: "GDR_ERR_INVALID_ARG", 2: "GDR_ERR_UNSUPPORTED", 3: "GDR_ERR_ALIGNMENT",
          4: "GDR_ERR_CUDA", 5: "GDR_ERR_TIMEOUT", 6: "GDR_ERR_RANGE"}


class FwdArgs(ctypes.Structure):
    """Mirror of gdr_fwd_args_t (include/gdr.h)."""
    _fields_ = [(name, ctypes.c_void_p) for name in (
        "q", "k", "v", "beta", "log_g", "erase_b", "write_w", "initial_state", "final_state", "o")]


class BwdGrads(ctypes.Structure):
    """Mirror of gdr_bwd_grads_t (include/gdr.h)."""
    _fields_ = [(name, ctypes.c_void_p) for name in ("dq", "dk", "dv", "dbeta", "dlog_g", "d_initial_state",
                                                      "d_erase_b", "d_write_w")]


_lock = threading.Lock()
_lib = None


def lib() -> ctypes.CDLL:
    global _lib
    with _lock:
        if _lib is None:
            if not os.path.exists(LIB_PATH):
                raise RuntimeError(
                    f"libgdr.so not found at {LIB_PATH}; build it with "
                    "`python gated_delta_rule_forward_b200/csrc/build.py` (there is no fallback)")
            L = ctypes.CDLL(LIB_PATH)
            i, vp, f, sz = ctypes.c_int, ctypes.c_void_p, ctypes.c_float, ctypes.c_size_t
            L.gdr_forward_workspace_size.argtypes = [i] * 8
            L.gdr_forward_workspace_size.restype = sz
            L.gdr_forward_chunked.argtypes = [i] * 7 + [ctypes.POINTER(FwdArgs), f, f, i, vp, sz, vp]
            L.gdr_forward_chunked.restype = i
            L.gdr_forward_chunked_noalloc.argtypes = [i] * 7 + [ctypes.POINTER(FwdArgs), f, f, vp]
            L.gdr_forward_chunked_noalloc.restype = i
            L.gdr_decode_step.argtypes = [i] * 6 + [vp] * 3 + [vp] * 4 + [vp, vp, f, f, vp]
            L.gdr_decode_step.restype = i
            L.gdr_forward_launches.argtypes = [i] * 8
            L.gdr_forward_launches.restype = i
            L.gdr_forward_plan.argtypes = [i] * 6 + [ctypes.POINTER(i)] * 3
            L.gdr_forward_plan.restype = i
            L.gdr_forward_segment_parts.argtypes = [i] * 6 + [ctypes.POINTER(i)] * 2
            L.gdr_forward_segment_parts.restype = i
            L.gdr_forward_kernel_name.argtypes = [i] * 8
            L.gdr_forward_kernel_name.restype = ctypes.c_char_p
            L.gdr_status_string.argtypes = [i]
            L.gdr_status_string.restype = ctypes.c_char_p
            L.gdr_last_error.argtypes = []
            L.gdr_last_error.restype = ctypes.c_char_p
            L.gdr_device_status.argtypes = [vp]
            L.gdr_device_status.restype = i
            L.gdr_version.argtypes = []
            L.gdr_version.restype = i
            L.gdr_backward_workspace_size.argtypes = [i] * 7
            L.gdr_backward_workspace_size.restype = sz
            L.gdr_backward.argtypes = ([i] * 7 + [ctypes.POINTER(FwdArgs), vp, vp, ctypes.POINTER(BwdGrads), f, f,
                                                 vp, sz, vp])
            L.gdr_backward.restype = i
            _lib = L
        return _lib


class GdrError(RuntimeError):
    def __init__(self, status: int, message: str):
        self.status = status
        super().__init__(f"{STATUS.get(status, status)}: {message}")


def check(status: int) -> None:
    if status != 0:
        raise GdrError(status, lib().gdr_last_error().decode())
