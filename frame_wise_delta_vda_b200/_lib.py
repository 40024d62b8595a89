"""ctypes declarations of libvda.so (the C ABI in include/vda.h).

Argument marshalling only.  Loading fails loudly when the library has not
been built: there is no fallback implementation.
"""

from __future__ import annotations

import ctypes
import os
import re

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libvda.so")
HEADER = os.path.join(os.path.dirname(HERE), "include", "vda.h")

VDA_OK = 0
VDA_ERR_INVALID_ARGUMENT = 1
VDA_ERR_UNSUPPORTED = 2
VDA_ERR_WORKSPACE = 3
VDA_ERR_CUDA = 4
VDA_ERR_TIMEOUT = 5
VDA_BF16 = 0
VDA_F32 = 1
VDA_SCAN_AUTO = 0
VDA_SCAN_FRAMES = 1
VDA_SCAN_CHUNKS = 2
NOALLOC_SCRATCH_BYTES = 16 << 20   # VDA_NOALLOC_SCRATCH_BYTES in include/vda.h

c_int, c_size_t, c_void_p, c_float = ctypes.c_int, ctypes.c_size_t, ctypes.c_void_p, ctypes.c_float
c_float_p = ctypes.POINTER(ctypes.c_float)
c_int_p = ctypes.POINTER(ctypes.c_int)


class VdaArgs(ctypes.Structure):
    """Mirror of `vda_args` in include/vda.h."""
    _fields_ = [
        ("dtype", c_int),
        ("q", c_void_p), ("k", c_void_p), ("v", c_void_p), ("beta", c_void_p), ("gate", c_void_p),
        ("rms_weight", c_void_p), ("S0_fwd", c_void_p), ("S0_rev", c_void_p), ("out", c_void_p),
        ("B", c_int), ("H", c_int), ("T", c_int), ("U", c_int), ("d_k", c_int), ("d_v", c_int),
        ("chunk", c_int), ("window_chunks", c_int),
        ("eps", c_float),
        ("stream", c_void_p),
        ("alpha", c_void_p),
        ("scan_form", c_int),
    ]


class VdaPrepArgs(ctypes.Structure):
    """Mirror of `vda_prep_args` in include/vda.h."""
    _fields_ = [
        ("q_in", c_void_p), ("k_in", c_void_p), ("v_in", c_void_p),
        ("wk_s", c_void_p), ("wk_t", c_void_p), ("wv_s", c_void_p), ("wv_t", c_void_p),
        ("q_out", c_void_p), ("k_out", c_void_p), ("v_out", c_void_p),
        ("B", c_int), ("H", c_int), ("T", c_int), ("Hl", c_int), ("Wl", c_int), ("d", c_int),
        ("eps", c_float),
        ("stream", c_void_p),
    ]


_SIGNATURES = {
    "vda_forward": (c_int, [c_void_p] * 8 + [c_int] * 8 + [c_void_p, c_void_p]),
    "vda_forward_f32": (c_int, [c_void_p] * 8 + [c_int] * 8 + [c_void_p, c_void_p]),
    "vda_workspace_bytes": (c_size_t, [c_int] * 8),
    "vda_forward_ex": (c_int, [ctypes.POINTER(VdaArgs), c_void_p, c_size_t, c_void_p, c_void_p]),
    "vda_text_state_workspace_bytes": (c_size_t, [c_int] * 6),
    "vda_text_state": (c_int, [c_int, c_void_p, c_void_p, c_void_p] + [c_int] * 5
                       + [c_void_p, c_void_p, c_size_t, c_void_p]),
    "vda_forward_host_bytes": (c_size_t, [c_int] * 8),
    "vda_forward_host": (c_int, [ctypes.POINTER(VdaArgs), c_void_p, c_size_t]),
    "vda_forward_noalloc": (c_int, [ctypes.POINTER(VdaArgs)]),
    "vda_device_status": (c_int, [c_void_p]),
    "vda_timing_enable": (c_int, [c_int]),
    "vda_timing_read": (c_int, [c_float_p, c_int, c_int_p]),
    "vda_launches_per_forward": (c_int, [c_int] * 8),
    "vda_status_string": (ctypes.c_char_p, [c_int]),
    "vda_prep": (c_int, [ctypes.POINTER(VdaPrepArgs)]),
    "vda_selftest_wait_timeout": (c_int, [c_int, c_void_p]),
}

_lib = None


class VdaError(RuntimeError):
    def __init__(self, status, where=""):
        self.status = status
        name = lib().vda_status_string(status).decode() if _lib is not None else str(status)
        super().__init__(f"{where}: {name} ({status})" if where else f"{name} ({status})")


def header_symbols():
    """Function names declared in include/vda.h."""
    text = open(HEADER).read()
    return sorted(set(re.findall(r"^\s*VDA_API\s+[\w\s\*]*?\b(vda_\w+)\s*\(", text, re.M)))


def lib():
    """The loaded libvda.so (ctypes.CDLL with argtypes declared)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(
                f"{LIB_PATH} is missing: build it with `python -m frame_wise_delta_vda_b200.build` "
                "(or __graft_entry__.build()); there is no non-CUDA implementation")
        L = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in _SIGNATURES.items():
            fn = getattr(L, name)
            fn.restype = res
            fn.argtypes = args
        _lib = L
    return _lib


def check(status, where=""):
    if status != VDA_OK:
        raise VdaError(status, where)
