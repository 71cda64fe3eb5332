"""ctypes view of libgdelta.so (the C ABI declared in include/gdelta.h).

Argument marshalling only: every step of the mixer runs in the library's CUDA
kernels.  Loading fails loudly when the library is missing; there is no
fallback.
"""
from __future__ import annotations

import ctypes
import os

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libgdelta.so")

GDELTA_OK = 0
STATUS_NAMES = {
    0: "GDELTA_OK",
    1: "GDELTA_ERR_INVALID_ARG",
    2: "GDELTA_ERR_UNSUPPORTED",
    3: "GDELTA_ERR_ALIGNMENT",
    4: "GDELTA_ERR_CUDA",
    5: "GDELTA_ERR_TIMEOUT",
    6: "GDELTA_ERR_WORKSPACE",
    7: "GDELTA_ERR_RANGE",
}
GDELTA_F32, GDELTA_BF16 = 0, 1
PATHS = {"auto": 0, "simt": 1, "tc": 2}
PATH_NAMES = {1: "simt", 2: "tc"}

# Every symbol include/gdelta.h declares.
EXPORTED = (
    "gdelta_abi_version",
    "gdelta_status_string",
    "gdelta_fwd_workspace_bytes",
    "gdelta_fwd_selected_path",
    "gdelta_state_init",
    "gdelta_state_affine",
    "gdelta_fwd_chunked",
    "gdelta_fwd_chunked_noalloc",
    "gdelta_decode_step",
    "gdelta_bwd_workspace_bytes",
    "gdelta_bwd",
    "gdelta_gate_proj_workspace_bytes",
    "gdelta_gate_proj",
    "gdelta_set_wait_limit",
    "gdelta_set_wait_timeout_test",
    "gdelta_get_last_device_error",
)

_vp = ctypes.c_void_p
_fp = ctypes.c_void_p


class FwdArgs(ctypes.Structure):
    _fields_ = [
        ("B", ctypes.c_int32), ("T", ctypes.c_int32), ("H", ctypes.c_int32),
        ("dk", ctypes.c_int32), ("dv", ctypes.c_int32), ("chunk", ctypes.c_int32),
        ("dtype", ctypes.c_int32), ("path", ctypes.c_int32),
        ("q", _vp), ("k", _vp), ("z", _vp), ("b", _vp),
        ("v", _vp), ("w", _vp), ("g", _vp),
        ("log_alpha", _fp), ("gamma_stat", _fp), ("S_in", _fp), ("S_out", _fp),
        ("y", _vp), ("o_raw", _fp), ("eps", ctypes.c_float),
        ("workspace", _vp), ("workspace_bytes", ctypes.c_size_t),
        ("beta", _vp), ("decay_per_token", ctypes.c_int32), ("qk_raw", ctypes.c_int32),
    ]


class DecodeArgs(ctypes.Structure):
    _fields_ = [
        ("B", ctypes.c_int32), ("H", ctypes.c_int32), ("dk", ctypes.c_int32),
        ("dv", ctypes.c_int32), ("dtype", ctypes.c_int32), ("reserved", ctypes.c_int32),
        ("q", _vp), ("k", _vp), ("z", _vp), ("b", _vp),
        ("v", _vp), ("w", _vp), ("g", _vp),
        ("log_alpha", _fp), ("gamma_stat", _fp), ("S", _fp),
        ("y", _vp), ("o_raw", _fp), ("eps", ctypes.c_float),
        ("beta", _vp), ("decay_per_token", ctypes.c_int32), ("qk_raw", ctypes.c_int32),
    ]


class BwdArgs(ctypes.Structure):
    _fields_ = [
        ("B", ctypes.c_int32), ("T", ctypes.c_int32), ("H", ctypes.c_int32),
        ("dk", ctypes.c_int32), ("dv", ctypes.c_int32), ("dtype", ctypes.c_int32),
        ("q", _vp), ("k", _vp), ("z", _vp), ("b", _vp), ("v", _vp), ("w", _vp), ("g", _vp),
        ("log_alpha", _fp), ("gamma_stat", _fp), ("S_in", _fp),
        ("grad_y", _fp), ("grad_S_out", _fp), ("eps", ctypes.c_float),
        ("grad_q", _fp), ("grad_k", _fp), ("grad_z", _fp), ("grad_b", _fp), ("grad_log_alpha", _fp),
        ("grad_v", _fp), ("grad_w", _fp), ("grad_g", _fp),
        ("grad_gamma_stat", _fp), ("grad_S_in", _fp),
        ("workspace", _vp), ("workspace_bytes", ctypes.c_size_t),
    ]


class GateProjArgs(ctypes.Structure):
    _fields_ = [
        ("N", ctypes.c_int32), ("d", ctypes.c_int32), ("ranks", ctypes.c_int32 * 5),
        ("x", _vp), ("w_down", _vp), ("w_up", _vp), ("bias", _fp),
        ("log_alpha", _fp), ("b", _vp), ("g", _vp), ("w", _vp), ("z", _vp),
        ("workspace", _vp), ("workspace_bytes", ctypes.c_size_t),
    ]


_lib = None


def load(path: str = LIB_PATH):
    """Load the library once; raises if it is missing."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise RuntimeError(
            f"libgdelta.so not found at {path}; build it with "
            "`python -m channel_gated_delta_b200.build` (there is no CPU fallback)")
    lib = ctypes.CDLL(path)
    lib.gdelta_abi_version.restype = ctypes.c_int
    lib.gdelta_status_string.restype = ctypes.c_char_p
    lib.gdelta_status_string.argtypes = [ctypes.c_int]
    lib.gdelta_fwd_workspace_bytes.restype = ctypes.c_size_t
    lib.gdelta_fwd_workspace_bytes.argtypes = [ctypes.POINTER(FwdArgs)]
    lib.gdelta_fwd_selected_path.restype = ctypes.c_int
    lib.gdelta_fwd_selected_path.argtypes = [ctypes.POINTER(FwdArgs)]
    lib.gdelta_state_init.restype = ctypes.c_int
    lib.gdelta_state_init.argtypes = [_fp, ctypes.c_int32, ctypes.c_int32, ctypes.c_int32,
                                      ctypes.c_int32, _fp, _vp]
    lib.gdelta_state_affine.restype = ctypes.c_int
    lib.gdelta_state_affine.argtypes = [_fp, _fp, _fp, _fp, ctypes.c_int32, ctypes.c_int32, ctypes.c_int32,
                                        ctypes.c_int32, _vp]
    lib.gdelta_fwd_chunked.restype = ctypes.c_int
    lib.gdelta_fwd_chunked.argtypes = [ctypes.POINTER(FwdArgs), _vp]
    lib.gdelta_fwd_chunked_noalloc.restype = ctypes.c_int
    lib.gdelta_fwd_chunked_noalloc.argtypes = [ctypes.POINTER(FwdArgs), _vp]
    lib.gdelta_bwd_workspace_bytes.restype = ctypes.c_size_t
    lib.gdelta_bwd_workspace_bytes.argtypes = [ctypes.POINTER(BwdArgs)]
    lib.gdelta_bwd.restype = ctypes.c_int
    lib.gdelta_bwd.argtypes = [ctypes.POINTER(BwdArgs), _vp]
    lib.gdelta_decode_step.restype = ctypes.c_int
    lib.gdelta_decode_step.argtypes = [ctypes.POINTER(DecodeArgs), _vp]
    lib.gdelta_gate_proj_workspace_bytes.restype = ctypes.c_size_t
    lib.gdelta_gate_proj_workspace_bytes.argtypes = [ctypes.POINTER(GateProjArgs)]
    lib.gdelta_gate_proj.restype = ctypes.c_int
    lib.gdelta_gate_proj.argtypes = [ctypes.POINTER(GateProjArgs), _vp]
    lib.gdelta_set_wait_limit.restype = ctypes.c_int
    lib.gdelta_set_wait_limit.argtypes = [ctypes.c_uint32]
    lib.gdelta_set_wait_timeout_test.restype = ctypes.c_int
    lib.gdelta_set_wait_timeout_test.argtypes = [ctypes.c_int32]
    lib.gdelta_get_last_device_error.restype = ctypes.c_int
    lib.gdelta_get_last_device_error.argtypes = [_vp]
    _lib = lib
    return lib
