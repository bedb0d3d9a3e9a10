"""ctypes view of libmls (include/mls.h).  Argument marshalling only.

The functions here carry the C names and take raw device pointers (ints).
The library must be built (``python -m lm_head_loss_junction_b200.build``);
loading fails loudly otherwise -- there is no fallback implementation.
"""
from __future__ import annotations

import ctypes
import os

PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(PKG, "libmls.so")

MLS_F32 = 0
MLS_BF16 = 1
MLS_DEVFLAG_BAD_ID = 1
MLS_DEVFLAG_TIMEOUT = 2
MLS_JUNCTION_STANDARD = 0
MLS_JUNCTION_NO_RESCALE = 1
MLS_JUNCTION_ZERO_FILL = 2
MLS_JUNCTION_STOP_GRAD = 4

STATUS_NAMES = {
    0: "MLS_OK", 1: "MLS_ERR_INVALID_ARG", 2: "MLS_ERR_UNSUPPORTED", 3: "MLS_ERR_WORKSPACE",
    4: "MLS_ERR_CUDA", 5: "MLS_ERR_BAD_ID", 6: "MLS_ERR_DEVICE_TIMEOUT", 7: "MLS_ERR_NO_DEVICE",
}

_vp = ctypes.c_void_p
_i64 = ctypes.c_int64
_i32 = ctypes.c_int32
_int = ctypes.c_int
_f32 = ctypes.c_float
_sz = ctypes.c_size_t
_u32 = ctypes.c_uint32

class LossOptions(ctypes.Structure):
    """mls_loss_options"""
    _fields_ = [("exit_weights", ctypes.POINTER(ctypes.c_float)), ("distill", ctypes.c_int),
                ("teacher_grad", ctypes.c_int)]


# name -> (restype, argtypes), in the order of include/mls.h
PROTOTYPES = {
    "mls_junction_fwd": (_int, [_vp, _i64, _vp, _i64, _vp, _i64, _i64, _vp, _vp, _int, _vp, _vp]),
    "mls_junction_bwd": (_int, [_vp, _i64, _vp, _i64, _vp, _i64, _i64, _vp, _vp, _vp, _vp, _int,
                                _vp, _sz, _int, _vp, _vp]),
    "mls_junction_fwd_variant": (_int, [_vp, _i64, _vp, _i64, _vp, _i64, _i64, _vp, _vp, _u32, _int, _vp, _vp]),
    "mls_junction_bwd_variant": (_int, [_vp, _i64, _vp, _i64, _vp, _i64, _i64, _vp, _vp, _vp, _vp, _int,
                                        _vp, _sz, _u32, _int, _vp, _vp]),
    "mls_junction_bwd_workspace": (_int, [_i64, _i64, ctypes.POINTER(_sz)]),
    "mls_junction_fwd_multi": (_int, [_vp, _i64, _i64, _int, ctypes.POINTER(_i64), ctypes.POINTER(_vp),
                                      ctypes.POINTER(_vp), ctypes.POINTER(_vp), ctypes.POINTER(_vp), _int, _vp, _vp]),
    "mls_junction_bwd_multi_workspace": (_int, [_i64, _i64, _int, ctypes.POINTER(_sz)]),
    "mls_junction_bwd_multi": (_int, [_vp, _i64, _i64, _int, ctypes.POINTER(_i64), ctypes.POINTER(_vp),
                                      ctypes.POINTER(_vp), ctypes.POINTER(_vp), ctypes.POINTER(_vp),
                                      ctypes.POINTER(_vp), ctypes.POINTER(_vp), _int, _vp, _sz, _int, _vp, _vp]),
    "mls_junction_bwd_noalloc": (_int, [_vp, _i64, _vp, _i64, _vp, _i64, _i64, _vp, _vp, _vp, _vp, _int,
                                        _int, _vp, _vp]),
    "mls_multiexit_loss_workspace": (_int, [_int, _i64, ctypes.POINTER(_i64), _i64, _int,
                                            ctypes.POINTER(_sz), ctypes.POINTER(_sz)]),
    "mls_multiexit_loss_bwd_plan": (_int, [_int, _i64, ctypes.POINTER(_i64), _i64, _int, _sz,
                                           ctypes.POINTER(_i64), ctypes.POINTER(_i64), ctypes.POINTER(_sz)]),
    "mls_multiexit_loss_fwd": (_int, [_int, _i64, _i64, ctypes.POINTER(_i64), _vp,
                                      ctypes.POINTER(_vp), ctypes.POINTER(_vp), _f32, _int,
                                      _vp, _vp, _vp, _sz, _vp, _vp]),
    "mls_multiexit_loss_bwd": (_int, [_int, _i64, _i64, ctypes.POINTER(_i64), _vp,
                                      ctypes.POINTER(_vp), ctypes.POINTER(_vp), _f32, _int,
                                      _vp, _f32, ctypes.POINTER(_vp), ctypes.POINTER(_vp), _int,
                                      _vp, _sz, _vp, _vp]),
    "mls_multiexit_loss_fwd_opts": (_int, [_int, _i64, _i64, ctypes.POINTER(_i64), _vp,
                                           ctypes.POINTER(_vp), ctypes.POINTER(_vp), _f32, _int,
                                           _vp, _vp, _vp, _sz, ctypes.POINTER(LossOptions), _vp, _vp]),
    "mls_multiexit_loss_bwd_opts": (_int, [_int, _i64, _i64, ctypes.POINTER(_i64), _vp,
                                           ctypes.POINTER(_vp), ctypes.POINTER(_vp), _f32, _int,
                                           _vp, _f32, ctypes.POINTER(_vp), ctypes.POINTER(_vp), _int,
                                           _vp, _sz, ctypes.POINTER(LossOptions), _vp, _vp]),
    "mls_exit_agreement_workspace": (_int, [_int, _i64, ctypes.POINTER(_i64), _i64, _int, ctypes.POINTER(_sz)]),
    "mls_exit_agreement": (_int, [_int, _i64, _i64, ctypes.POINTER(_i64), ctypes.POINTER(_vp), ctypes.POINTER(_vp),
                                  _int, _vp, _vp, _vp, _vp, _vp, _sz, _vp, _vp]),
    "mls_selftest_wait_timeout": (_int, [_int, _i64, _i64, ctypes.POINTER(_i64), _vp, ctypes.POINTER(_vp),
                                         ctypes.POINTER(_vp), _vp, _vp, _vp, _sz, ctypes.c_uint64, _vp, _vp]),
    "mls_status_read": (_int, [_vp, _vp, ctypes.POINTER(_i32)]),
    "mls_status_string": (ctypes.c_char_p, [_int]),
    "mls_version": (_int, []),
    "mls_kernel_launches": (ctypes.c_uint64, []),
}


class MLSError(RuntimeError):
    def __init__(self, fn: str, code: int):
        self.code = code
        super().__init__(f"{fn} failed: {STATUS_NAMES.get(code, code)}")


_LIB = None


def lib() -> ctypes.CDLL:
    global _LIB
    if _LIB is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(
                f"{LIB_PATH} is not built; run `python -m lm_head_loss_junction_b200.build` "
                "(the CUDA library is the only implementation)")
        handle = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in PROTOTYPES.items():
            fn = getattr(handle, name)
            fn.restype = res
            fn.argtypes = args
        _LIB = handle
    return _LIB


def check(fn: str, code: int) -> None:
    if code != 0:
        raise MLSError(fn, code)


def ptr_array(ptrs):
    arr = (_vp * len(ptrs))()
    for i, p in enumerate(ptrs):
        arr[i] = p
    return arr


def i64_array(vals):
    arr = (_i64 * len(vals))()
    for i, v in enumerate(vals):
        arr[i] = int(v)
    return arr


MLS_DISTILL = {"ce": 0, "reverse_kl": 1, "js": 2, "accept": 3}


def loss_options(exit_weights=None, distill="ce", teacher_grad=False):
    """ctypes options struct (and the buffer it points to), or None for defaults."""
    if exit_weights is None and distill == "ce" and not teacher_grad:
        return None
    if exit_weights is None:
        opts = LossOptions(None, MLS_DISTILL[distill], int(bool(teacher_grad)))
        opts._buf = None
        return opts
    buf = (ctypes.c_float * len(exit_weights))(*[float(w) for w in exit_weights])
    opts = LossOptions(ctypes.cast(buf, ctypes.POINTER(ctypes.c_float)), MLS_DISTILL[distill],
                       int(bool(teacher_grad)))
    opts._buf = buf          # keep the weights alive with the struct
    return opts
