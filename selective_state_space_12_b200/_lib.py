"""ctypes view of libssd.so: the C ABI of include/ssd.h, nothing else.

The library is looked up next to this file (built in-tree). Loading fails
loudly when it is missing; there is no fallback implementation.
"""
from __future__ import annotations

import ctypes
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libssd.so")

SSD_OK = 0
SSD_ERR_INVALID_ARG = 1
SSD_ERR_UNSUPPORTED = 2
SSD_ERR_CUDA = 3
SSD_ERR_NO_MEMORY = 4
SSD_ERR_TIMEOUT = 5
STATUS_NAMES = {0: "SSD_OK", 1: "SSD_ERR_INVALID_ARG", 2: "SSD_ERR_UNSUPPORTED",
                3: "SSD_ERR_CUDA", 4: "SSD_ERR_NO_MEMORY", 5: "SSD_ERR_TIMEOUT"}

SSD_F32 = 0
SSD_BF16 = 1


class Dims(ctypes.Structure):
    """struct ssd_dims."""

    _fields_ = [("batch", ctypes.c_int64), ("seqlen", ctypes.c_int64),
                ("nheads", ctypes.c_int64), ("headdim", ctypes.c_int64),
                ("dstate", ctypes.c_int64), ("ngroups", ctypes.c_int64),
                ("dtype", ctypes.c_int32), ("reserved", ctypes.c_int32)]


SSD_DISC_EULER = 0
SSD_DISC_ZOH = 1


class Options(ctypes.Structure):
    """struct ssd_options (all zero: the plain layer)."""

    _fields_ = [("dt_bias", ctypes.c_void_p), ("dt_softplus", ctypes.c_int32),
                ("discretization", ctypes.c_int32), ("dt_min", ctypes.c_float),
                ("dt_max", ctypes.c_float), ("reserved", ctypes.c_int32 * 4)]


class KernelTime(ctypes.Structure):
    """struct ssd_kernel_time."""

    _fields_ = [("name", ctypes.c_char_p), ("launches", ctypes.c_longlong),
                ("total_ms", ctypes.c_double)]


_VP = ctypes.c_void_p
_SIGNATURES = {
    "ssd_forward_workspace_size": (ctypes.c_size_t, [ctypes.POINTER(Dims), ctypes.c_int]),
    "ssd_forward": (ctypes.c_int, [_VP, _VP, _VP, _VP, _VP, _VP, _VP, ctypes.c_int, _VP, _VP,
                                   ctypes.POINTER(Dims), _VP, ctypes.c_size_t, _VP]),
    "ssd_forward_noalloc": (ctypes.c_int, [_VP, _VP, _VP, _VP, _VP, _VP, _VP, ctypes.c_int,
                                           _VP, _VP, ctypes.POINTER(Dims), _VP]),
    "ssd_forward_ex": (ctypes.c_int, [_VP, _VP, _VP, _VP, _VP, _VP, _VP, ctypes.c_int, _VP,
                                      _VP, ctypes.POINTER(Dims), ctypes.POINTER(Options), _VP,
                                      ctypes.c_size_t, _VP]),
    "ssd_step": (ctypes.c_int, [_VP, _VP, _VP, _VP, _VP, _VP, _VP, _VP,
                                ctypes.POINTER(Dims), _VP]),
    "ssd_step_ex": (ctypes.c_int, [_VP, _VP, _VP, _VP, _VP, _VP, _VP, _VP,
                                   ctypes.POINTER(Dims), ctypes.POINTER(Options), _VP]),
    "ssd_forward_state_workspace_size": (ctypes.c_size_t, [ctypes.POINTER(Dims), ctypes.c_int]),
    "ssd_forward_state": (ctypes.c_int, [_VP, _VP, _VP, _VP, ctypes.c_int, _VP, _VP,
                                         ctypes.POINTER(Dims), ctypes.POINTER(Options), _VP,
                                         ctypes.c_size_t, _VP]),
    "ssd_state_chain": (ctypes.c_int, [_VP, _VP, ctypes.c_int, ctypes.c_int, _VP, _VP, _VP,
                                       ctypes.POINTER(Dims), _VP]),
    "ssd_selective_scan": (ctypes.c_int, [_VP, _VP, _VP, _VP, _VP, _VP, _VP, _VP, _VP,
                                          ctypes.POINTER(Dims), ctypes.POINTER(Options), _VP]),
    "ssd_backward_workspace_size": (ctypes.c_size_t, [ctypes.POINTER(Dims)]),
    "ssd_backward": (ctypes.c_int, [_VP] * 16 + [ctypes.POINTER(Dims), _VP, ctypes.c_size_t,
                                                 _VP]),
    "ssd_device_status": (ctypes.c_int, [_VP]),
    "ssd_last_error": (ctypes.c_char_p, []),
    "ssd_set_wait_limit": (None, [ctypes.c_longlong]),
    "ssd_abi_version": (ctypes.c_int, []),
    "ssd_launch_count": (ctypes.c_longlong, []),
    "ssd_profile_begin": (ctypes.c_int, []),
    "ssd_profile_end": (ctypes.c_int, [ctypes.POINTER(KernelTime), ctypes.c_int]),
}

_lib = None


def load():
    """Load libssd.so (once) and declare the ABI's signatures."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise ImportError(
            f"libssd.so not found at {LIB_PATH}; build it with "
            "`python -m selective_state_space_12_b200.build`")
    lib = ctypes.CDLL(LIB_PATH)
    for name, (res, args) in _SIGNATURES.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    _lib = lib
    return lib


def exported_symbols():
    """Names of the ABI functions this module binds."""
    return sorted(_SIGNATURES)


def last_error() -> str:
    return load().ssd_last_error().decode("utf-8", "replace")
