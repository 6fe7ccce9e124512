"""ctypes binding of libfa_b200.so (argument marshalling only).

Every entry point of include/fa.h is bound with its C signature.  Loading
fails loudly when the library has not been built; there is no fallback.
"""

from __future__ import annotations

import ctypes
import os

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libfa_b200.so")

FA_OK = 0
FA_ERR_ARG = -1
FA_ERR_UNSUPPORTED = -2
FA_ERR_ALIGN = -3
FA_ERR_CUDA = -4
FA_ERR_TIMEOUT = -5

FA_FP16, FA_BF16, FA_E4M3 = 0, 1, 2
FA_MASK_BOOL, FA_MASK_ADD = 1, 2

_c_int, _c_float, _vp = ctypes.c_int, ctypes.c_float, ctypes.c_void_p
_fp = ctypes.POINTER(ctypes.c_float)

class FwdArgs(ctypes.Structure):
    """fa_fwd_args (include/fa.h), field for field."""
    _fields_ = [("q", _vp), ("k", _vp), ("v", _vp), ("out", _vp), ("lse", _vp),
                ("B", _c_int), ("N_q", _c_int), ("N_k", _c_int), ("H", _c_int), ("H_kv", _c_int), ("D", _c_int),
                ("scale", _c_float), ("causal", _c_int), ("window_left", _c_int), ("window_right", _c_int),
                ("dtype", _c_int), ("q_descale", _c_float), ("k_descale", _c_float), ("v_descale", _c_float),
                ("cu_seqlens_q", _vp), ("cu_seqlens_k", _vp), ("total_q", _c_int), ("total_k", _c_int),
                ("dropout_p", _c_float), ("seed", ctypes.c_ulonglong), ("offset", ctypes.c_uint)]


class BwdArgs(ctypes.Structure):
    """fa_bwd_args (include/fa.h), field for field."""
    _fields_ = [("q", _vp), ("k", _vp), ("v", _vp), ("out", _vp), ("dout", _vp), ("lse", _vp),
                ("dq", _vp), ("dk", _vp), ("dv", _vp),
                ("B", _c_int), ("N_q", _c_int), ("N_k", _c_int), ("H", _c_int), ("H_kv", _c_int), ("D", _c_int),
                ("scale", _c_float), ("causal", _c_int), ("window_left", _c_int), ("window_right", _c_int),
                ("dtype", _c_int), ("cu_seqlens_q", _vp), ("cu_seqlens_k", _vp), ("total_q", _c_int),
                ("total_k", _c_int), ("dropout_p", _c_float), ("seed", ctypes.c_ulonglong), ("offset", ctypes.c_uint),
                ("workspace", _vp), ("workspace_bytes", ctypes.c_size_t)]


SIGNATURES = {
    "fa_fwd": (_c_int, [_vp, _vp, _vp, _vp, _vp, _c_int, _c_int, _c_int, _c_int, _c_int, _c_float,
                        _c_int, _c_int, _c_int, _vp]),
    "fa_fwd_fp8": (_c_int, [_vp, _vp, _vp, _vp, _vp, _c_int, _c_int, _c_int, _c_int, _c_int, _c_float,
                            _c_int, _c_int, _c_float, _c_float, _c_float, _vp]),
    "fa_fwd_gqa": (_c_int, [_vp, _vp, _vp, _vp, _vp, _c_int, _c_int, _c_int, _c_int, _c_int, _c_int, _c_float,
                            _c_int, _c_int, _c_int, _c_float, _c_float, _c_float, _vp]),
    "fa_fwd_window": (_c_int, [_vp, _vp, _vp, _vp, _vp, _c_int, _c_int, _c_int, _c_int, _c_int, _c_int, _c_float,
                               _c_int, _c_int, _c_int, _c_int, _c_float, _c_float, _c_float, _vp]),
    "fa_fwd_splitkv_workspace_bytes": (ctypes.c_size_t, [_c_int, _c_int, _c_int, _c_int, _c_int, _c_int]),
    "fa_fwd_splitkv": (_c_int, [_vp, _vp, _vp, _vp, _vp, _c_int, _c_int, _c_int, _c_int, _c_int, _c_int, _c_float,
                                _c_int, _c_int, _c_int, _c_float, _c_float, _c_float, _c_int, _vp, ctypes.c_size_t,
                                _vp]),
    "fa_fwd_mask": (_c_int, [_vp, _vp, _vp, _vp, _vp, _c_int, _c_int, _c_int, _c_int, _c_int, _c_int, _c_float,
                             _c_int, _c_int, _c_int, _c_float, _c_float, _c_float, _vp, _c_int,
                             ctypes.c_longlong, ctypes.c_longlong, ctypes.c_longlong, _vp]),
    "fa_fwd_varlen": (_c_int, [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _c_int, _c_int, _c_int, _c_int, _c_int, _c_int,
                               _c_int, _c_int, _c_float, _c_int, _c_int, _c_int, _c_float, _c_float, _c_float, _vp]),
    "fa_fwd_dropout": (_c_int, [_vp, _vp, _vp, _vp, _vp, _c_int, _c_int, _c_int, _c_int, _c_int, _c_int,
                                _c_float, _c_int, _c_int, _c_int, _c_float, ctypes.c_ulonglong, ctypes.c_uint, _vp]),
    "fa_fwd_host": (_c_int, [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _c_int, _c_int, _c_int,
                             _c_int, _c_int, _c_float, _c_int, _c_int, _c_int, _c_float, _c_float,
                             _c_float, _vp]),
    "fa_fwd_host_async": (_c_int, [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _c_int, _c_int, _c_int,
                                   _c_int, _c_int, _c_float, _c_int, _c_int, _c_int, _c_float, _c_float,
                                   _c_float, _vp]),
    "fa_fwd_noalloc": (_c_int, [_vp, _vp, _vp, _vp, _vp, _c_int, _c_int, _c_int, _c_int, _c_int, _c_float,
                                _c_int, _c_int, _c_int, _c_float, _c_float, _c_float, _vp]),
    "fa_bwd_workspace_bytes": (ctypes.c_size_t, [_c_int, _c_int, _c_int, _c_int]),
    "fa_bwd": (_c_int, [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _c_int, _c_int, _c_int, _c_int, _c_int,
                        _c_float, _c_int, _c_int, _c_int, _vp, ctypes.c_size_t, _vp]),
    "fa_bwd_gqa": (_c_int, [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _c_int, _c_int, _c_int, _c_int, _c_int,
                            _c_int, _c_float, _c_int, _c_int, _c_int, _vp, ctypes.c_size_t, _vp]),
    "fa_bwd_window": (_c_int, [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _c_int, _c_int, _c_int, _c_int,
                               _c_int, _c_int, _c_float, _c_int, _c_int, _c_int, _c_int, _vp, ctypes.c_size_t, _vp]),
    "fa_bwd_varlen": (_c_int, [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _c_int, _c_int, _c_int, _c_int,
                               _c_int, _c_int, _c_int, _c_int, _c_float, _c_int, _c_int, _c_int, _vp, ctypes.c_size_t,
                               _vp]),
    "fa_bwd_dropout": (_c_int, [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _c_int, _c_int, _c_int, _c_int,
                                _c_int, _c_int, _c_float, _c_int, _c_int, _c_int, _c_float, ctypes.c_ulonglong,
                                ctypes.c_uint, _vp, ctypes.c_size_t, _vp]),
    "fa_fwd_ex": (_c_int, [ctypes.POINTER(FwdArgs), _vp]),
    "fa_bwd_ex": (_c_int, [ctypes.POINTER(BwdArgs), _vp]),
    "fa_device_status": (_c_int, [_vp, ctypes.POINTER(ctypes.c_int)]),
    "fa_set_wait_limit_ns": (None, [ctypes.c_ulonglong]),
    "fa_wait_probe": (_c_int, [ctypes.c_ulonglong, _vp]),
    "fa_exp2_check": (_c_int, [_vp, _vp, _vp, _c_int, _c_int, _vp]),
    "fa_status_string": (ctypes.c_char_p, [_c_int]),
    "fa_version": (ctypes.c_char_p, []),
}

_lib = None


class FAError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__(f"{what}: {status_string(status)} ({status})")


def lib() -> ctypes.CDLL:
    """The loaded library (loaded once).  Raises if it was never built."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(
                f"{LIB_PATH} is missing: build it with `python -m exact_attention_136_b200.build` "
                "(there is no CPU or PyTorch fallback)")
        handle = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in SIGNATURES.items():
            fn = getattr(handle, name)
            fn.restype = res
            fn.argtypes = args
        _lib = handle
    return _lib


def status_string(status: int) -> str:
    return lib().fa_status_string(int(status)).decode()


def check(status: int, what: str) -> None:
    if status != FA_OK:
        raise FAError(status, what)
