"""ctypes declarations of libmuon.so (include/muon.h).  Argument marshalling
only; every step of the optimizer runs in the library's CUDA kernels."""
from __future__ import annotations

import ctypes
import os

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libmuon.so")

MUON_OK = 0
MUON_ERR_INVALID_ARG = -1
MUON_ERR_UNSUPPORTED = -2
MUON_ERR_CUDA = -3
MUON_ERR_NO_MEMORY = -4
MUON_ERR_TIMEOUT = -5
MUON_ERR_NONFINITE = -6
MUON_ERR_GUARD = -7

MUON_NS_STANDARD = 0
MUON_NS_GRAM = 1
MUON_NS_AUTO = 2
MUON_PREC_FP32 = 0x100

MUON_DTYPE_BF16 = 0
MUON_DTYPE_F32 = 1

MUON_MAX_STEPS = 16
MUON_MAX_SHAPE_SCHEDULES = 64

STATUS_NAMES = {
    MUON_OK: "MUON_OK", MUON_ERR_INVALID_ARG: "MUON_ERR_INVALID_ARG",
    MUON_ERR_UNSUPPORTED: "MUON_ERR_UNSUPPORTED", MUON_ERR_CUDA: "MUON_ERR_CUDA",
    MUON_ERR_NO_MEMORY: "MUON_ERR_NO_MEMORY", MUON_ERR_TIMEOUT: "MUON_ERR_TIMEOUT",
    MUON_ERR_NONFINITE: "MUON_ERR_NONFINITE", MUON_ERR_GUARD: "MUON_ERR_GUARD",
}

# every symbol include/muon.h declares
EXPORTS = (
    "muon_version", "muon_default_config", "muon_set_config", "muon_get_config",
    "muon_set_stream", "muon_last_error", "muon_release_workspace",
    "muon_device_status", "muon_orthogonalize", "muon_step",
    "muon_profile_enable", "muon_profile_read", "muon_profile_reset",
    "muon_launch_count", "muon_normalize_noalloc", "muon_adamw_step",
    "muon_set_shape_coeffs", "muon_get_shape_coeffs", "muon_clear_shape_coeffs",
    "muon_hybrid_step", "muon_step_offload", "muon_offload_chunks", "muon_debug_corrupt_guard",
)


class MuonConfig(ctypes.Structure):
    _fields_ = [
        ("steps", ctypes.c_int),
        ("coeffs", ctypes.c_float * (3 * MUON_MAX_STEPS)),
        ("mode", ctypes.c_int),
        ("restart_mask", ctypes.c_uint),
        ("eps", ctypes.c_float),
        ("momentum_dtype", ctypes.c_int),
        ("param_dtype", ctypes.c_int),
        ("grad_dtype", ctypes.c_int),
        ("soft_threshold", ctypes.c_float),
    ]


class MuonAdamwLane(ctypes.Structure):
    _fields_ = [
        ("params", ctypes.POINTER(ctypes.c_void_p)),
        ("grads", ctypes.POINTER(ctypes.c_void_p)),
        ("exp_avg", ctypes.POINTER(ctypes.c_void_p)),
        ("exp_avg_sq", ctypes.POINTER(ctypes.c_void_p)),
        ("numels", ctypes.POINTER(ctypes.c_longlong)),
        ("count", ctypes.c_int),
        ("lr", ctypes.c_float),
        ("beta1", ctypes.c_float),
        ("beta2", ctypes.c_float),
        ("eps", ctypes.c_float),
        ("weight_decay", ctypes.c_float),
        ("step", ctypes.c_int),
    ]


class MuonKernelStats(ctypes.Structure):
    _fields_ = [
        ("name", ctypes.c_char * 32),
        ("launches", ctypes.c_longlong),
        ("total_ms", ctypes.c_double),
        ("flops", ctypes.c_double),
        ("bytes", ctypes.c_double),
    ]


_LIB = None


def load(path=LIB_PATH):
    """Load libmuon.so; raises ImportError when it has not been built."""
    global _LIB
    if _LIB is not None:
        return _LIB
    if not os.path.exists(path):
        raise ImportError(
            f"{path} is missing: build it with "
            "`python -m matrix_orthogonalizing_optimizer_step_b200.build` "
            "(there is no fallback implementation)")
    lib = ctypes.CDLL(path)
    c_int, c_float, vp = ctypes.c_int, ctypes.c_float, ctypes.c_void_p
    sig = {
        "muon_version": (c_int, []),
        "muon_default_config": (c_int, [ctypes.POINTER(MuonConfig)]),
        "muon_set_config": (c_int, [ctypes.POINTER(MuonConfig)]),
        "muon_get_config": (c_int, [ctypes.POINTER(MuonConfig)]),
        "muon_set_stream": (c_int, [vp]),
        "muon_last_error": (ctypes.c_char_p, []),
        "muon_release_workspace": (c_int, []),
        "muon_device_status": (c_int, [ctypes.POINTER(c_int)]),
        "muon_orthogonalize": (c_int, [c_int, c_int, c_int, vp,
                                       ctypes.POINTER(c_float), c_int, c_int]),
        "muon_step": (c_int, [ctypes.POINTER(vp), ctypes.POINTER(vp),
                              ctypes.POINTER(vp), c_float, c_int, c_float,
                              ctypes.POINTER(c_int), c_int]),
        "muon_profile_enable": (c_int, [c_int]),
        "muon_profile_read": (c_int, [ctypes.POINTER(MuonKernelStats), c_int,
                                      ctypes.POINTER(c_int)]),
        "muon_profile_reset": (c_int, []),
        "muon_launch_count": (ctypes.c_longlong, []),
        "muon_normalize_noalloc": (c_int, [c_int, c_int, c_int, vp, vp, c_int, c_float]),
        "muon_adamw_step": (c_int, [ctypes.POINTER(vp), ctypes.POINTER(vp), ctypes.POINTER(vp),
                                    ctypes.POINTER(vp), ctypes.POINTER(ctypes.c_longlong), c_int,
                                    c_float, c_float, c_float, c_float, c_float, c_int]),
        "muon_set_shape_coeffs": (c_int, [c_int, c_int, ctypes.POINTER(c_float), c_int]),
        "muon_get_shape_coeffs": (c_int, [c_int, c_int, ctypes.POINTER(c_float), ctypes.POINTER(c_int)]),
        "muon_clear_shape_coeffs": (c_int, []),
        "muon_hybrid_step": (c_int, [ctypes.POINTER(vp), ctypes.POINTER(vp), ctypes.POINTER(vp), c_float, c_int,
                                     c_float, ctypes.POINTER(c_int), c_int, ctypes.POINTER(MuonAdamwLane)]),
        "muon_step_offload": (c_int, [ctypes.POINTER(vp), ctypes.POINTER(vp), ctypes.POINTER(vp),
                                      ctypes.POINTER(vp), ctypes.POINTER(vp), c_float, c_int, c_float,
                                      ctypes.POINTER(c_int), c_int, c_int]),
        "muon_offload_chunks": (c_int, [ctypes.POINTER(ctypes.c_longlong), c_int, c_int, ctypes.POINTER(c_int)]),
        "muon_debug_corrupt_guard": (c_int, [c_int]),
    }
    assert set(sig) == set(EXPORTS)
    for name, (res, args) in sig.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    _LIB = lib
    return lib
