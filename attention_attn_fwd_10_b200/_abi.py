"""ctypes view of libattn.so: the C entry points of include/attn.h, same names.

Argument marshalling only.  Loading fails loudly when the library is missing:
there is no fallback implementation anywhere in this package.
"""
from __future__ import annotations

import ctypes
import os

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libattn.so")

ATTN_OK = 0
STATUS_NAMES = {
    0: "ATTN_OK",
    1: "ATTN_ERR_INVALID_ARG",
    2: "ATTN_ERR_UNSUPPORTED",
    3: "ATTN_ERR_MISALIGNED",
    4: "ATTN_ERR_CUDA",
    5: "ATTN_ERR_DEVICE_TIMEOUT",
    6: "ATTN_ERR_SCRATCH_TOO_SMALL",
}

# Every symbol include/attn.h declares (tests check the library exports all of them).
EXPORTED = (
    "attn_abi_version",
    "attn_status_string",
    "attn_fwd",
    "attn_fwd_default_options",
    "attn_fwd_ex",
    "attn_fwd_qk8",
    "attn_fwd_qkv8",
    "attn_fwd_split",
    "attn_fwd_split_qk8",
    "attn_fwd_split_count",
    "attn_fwd_split_workspace_size",
    "attn_bwd_workspace_size",
    "attn_bwd",
    "attn_bwd_ex",
    "attn_bwd_noalloc",
    "attn_device_status",
    "attn_set_wait_limit_ns",
    "attn_exp2_poly_eval",
    "attn_read_probe",
)


class FwdOptions(ctypes.Structure):
    """attn_fwd_options_t"""

    _fields_ = [
        ("rescale_threshold", ctypes.c_float),
        ("poly_exp_every", ctypes.c_int),
        ("rescale_count", ctypes.c_void_p),
        ("persistent", ctypes.c_int),
    ]


class BwdOptions(ctypes.Structure):
    """attn_bwd_options_t"""

    _fields_ = [("main_pass_start", ctypes.c_void_p), ("main_pass_stop", ctypes.c_void_p),
                ("deterministic", ctypes.c_int), ("cta_mode", ctypes.c_int)]


_vp = ctypes.c_void_p
_i = ctypes.c_int
_f = ctypes.c_float

_SIGNATURES = {
    "attn_abi_version": (_i, []),
    "attn_status_string": (ctypes.c_char_p, [_i]),
    "attn_fwd": (_i, [_vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _i, _i, _f, _vp]),
    "attn_fwd_default_options": (None, [ctypes.POINTER(FwdOptions)]),
    "attn_fwd_ex": (_i, [_vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _i, _i, _f,
                         ctypes.POINTER(FwdOptions), _vp]),
    "attn_fwd_qk8": (_i, [_vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _i, _i, _f,
                          ctypes.POINTER(FwdOptions), _vp]),
    "attn_fwd_qkv8": (_i, [_vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _i, _i, _f,
                           ctypes.POINTER(FwdOptions), _vp]),
    "attn_fwd_split": (_i, [_vp] * 6 + [_i, _i, _i, _i, _i, _i, _i, _f, _i, _vp]),
    "attn_fwd_split_qk8": (_i, [_vp] * 6 + [_i, _i, _i, _i, _i, _i, _i, _f, _i, _vp]),
    "attn_fwd_split_count": (_i, [_i, _i, _i, _i, _i, _i]),
    "attn_fwd_split_workspace_size": (ctypes.c_size_t, [_i, _i, _i, _i, _i]),
    "attn_bwd_workspace_size": (ctypes.c_size_t, [_i, _i, _i, _i]),
    "attn_bwd": (_i, [_vp] * 10 + [_i, _i, _i, _i, _i, _i, _i, _f, _vp]),
    "attn_bwd_ex": (_i, [_vp] * 10 + [_i, _i, _i, _i, _i, _i, _i, _f, ctypes.POINTER(BwdOptions), _vp]),
    "attn_bwd_noalloc": (_i, [_vp] * 9 + [_i, _i, _i, _i, _i, _i, _i, _f, _vp]),
    "attn_device_status": (_i, [_vp]),
    "attn_set_wait_limit_ns": (None, [ctypes.c_ulonglong]),
    "attn_exp2_poly_eval": (_i, [_vp, _vp, ctypes.c_longlong, _vp]),
    "attn_read_probe": (_i, [_vp, ctypes.c_longlong, _vp, _vp]),
}

_lib = None


def load(path: str = LIB_PATH) -> ctypes.CDLL:
    """Load libattn.so once; raise if it is missing (build it with attention_attn_fwd_10_b200.build)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise RuntimeError(f"{path} is missing: run `python -m attention_attn_fwd_10_b200.build` first")
    lib = ctypes.CDLL(path)
    for name, (res, args) in _SIGNATURES.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    _lib = lib
    return lib


def status_string(code: int) -> str:
    return load().attn_status_string(code).decode()


def check(code: int, what: str) -> None:
    if code != ATTN_OK:
        raise RuntimeError(f"{what} failed: {status_string(code)}")
