"""ctypes loader for the in-tree CUDA library ``libdiffattn.so``.

Loading fails loudly when the library has not been built: there is no other
implementation behind these calls.
"""
from __future__ import annotations

import ctypes
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libdiffattn.so")
# the bounds-checked build (same entry points; kernels record DIFFATTN_ERR_BOUNDS)
DEBUG_LIB_PATH = os.path.join(_HERE, "libdiffattn_debug.so")

_handles = {}
_active = LIB_PATH

# name -> (restype, argtypes); mirrors include/diffattn.h
_c_int, _c_float, _c_size, _vp, _c_ll = ctypes.c_int, ctypes.c_float, ctypes.c_size_t, ctypes.c_void_p, ctypes.c_longlong
SIGNATURES = {
    "diffattn_lambda": (_c_int, [_vp, _vp, _vp, _vp, _c_int, _c_float, _vp, _vp]),
    "diffattn_fwd": (_c_int, [_vp, _vp, _vp, _vp, _c_int, _c_int, _c_int, _c_int, _c_int, _c_int,
                              _vp, _c_float, _vp, _c_float, _vp]),
    "diffattn_fwd_mode": (_c_int, [_vp, _vp, _vp, _vp, _c_int, _c_int, _c_int, _c_int, _c_int, _c_int,
                                   _vp, _c_float, _vp, _c_float, _c_int, _vp]),
    "diffattn_quantize_qk": (_c_int, [_vp, _c_int, _c_int, _c_int, _c_int, _vp, _vp, _vp]),
    "diffattn_fwd_qk8": (_c_int, [_vp, _vp, _vp, _vp, _vp, _vp, _c_int, _c_int, _c_int, _c_int, _c_int,
                                  _vp, _c_float, _vp, _c_float, _c_int, _vp]),
    "diffattn_quantize_qk4": (_c_int, [_vp, _c_int, _c_int, _c_int, _c_int, _vp, _vp, _vp]),
    "diffattn_fwd_qk4": (_c_int, [_vp, _vp, _vp, _vp, _vp, _vp, _c_int, _c_int, _c_int, _c_int, _c_int,
                                  _vp, _c_float, _vp, _c_float, _c_int, _vp]),
    "diffattn_bwd_workspace_size": (_c_size, [_c_int, _c_int, _c_int, _c_int]),
    "diffattn_bwd": (_c_int, [_vp, _vp, _vp, _vp, _c_int, _c_int, _c_int, _c_int, _c_int, _c_int, _vp, _c_float,
                              _vp, _c_float, _c_int, _vp, _vp, _vp, _vp, _vp, _vp, _c_size, _vp]),
    "diffattn_bwd_tc_workspace_size": (_c_size, [_c_int, _c_int, _c_int, _c_int]),
    "diffattn_bwd_tc": (_c_int, [_vp, _vp, _vp, _vp, _c_int, _c_int, _c_int, _c_int, _c_int, _vp, _c_float,
                                 _vp, _c_float, _c_int, _vp, _vp, _vp, _vp, _vp, _vp, _c_size, _vp]),
    "diffattn_fwd_train": (_c_int, [_vp, _vp, _vp, _vp, _c_int, _c_int, _c_int, _c_int, _c_int, _vp, _c_float, _vp,
                                    _c_float, _c_int, _vp, _c_size, _vp]),
    "diffattn_bwd_tc_saved": (_c_int, [_vp, _vp, _vp, _vp, _c_int, _c_int, _c_int, _c_int, _c_int, _vp, _c_float,
                                       _vp, _c_float, _c_int, _vp, _vp, _vp, _vp, _vp, _vp, _c_size, _vp]),
    "diffattn_rope_table": (_c_int, [_c_int, _c_int, ctypes.c_double, _vp, _vp]),
    "diffattn_qkv_proj": (_c_int, [_vp, _vp, _c_int, _c_int, _c_int, _c_int, _c_int, _vp, _vp, _vp, _vp, _vp]),
    "diffattn_out_proj": (_c_int, [_vp, _vp, _c_int, _c_int, _c_int, _vp, _vp]),
    "diffattn_lambda_bwd": (_c_int, [_vp, _vp, _vp, _vp, _c_int, _vp, _vp, _vp, _vp, _vp, _vp]),
    "diffattn_decode_workspace_size": (_c_size, [_c_int, _c_int, _c_int, _c_int]),
    "diffattn_decode": (_c_int, [_vp, _vp, _vp, _vp, _c_int, _vp, _c_int, _c_int, _c_int, _vp, _c_float,
                                 _vp, _c_float, _vp, _c_size, _vp]),
    "diffattn_decode_mode": (_c_int, [_vp, _vp, _vp, _vp, _c_int, _vp, _c_int, _c_int, _c_int, _vp, _c_float,
                                      _vp, _c_float, _c_int, _vp, _c_size, _vp]),
    "diffattn_decode_noalloc": (_c_int, [_vp, _vp, _vp, _vp, _c_int, _vp, _c_int, _c_int, _c_int, _vp,
                                         _c_float, _vp, _c_float, _vp]),
    "diffattn_device_status": (_c_int, [ctypes.POINTER(_c_int)]),
    "diffattn_set_wait_limit_ns": (_c_int, [_c_ll]),
    "diffattn_status_string": (ctypes.c_char_p, [_c_int]),
    "diffattn_version": (_c_int, []),
}


def _load(path: str) -> ctypes.CDLL:
    if path not in _handles:
        if not os.path.exists(path):
            raise RuntimeError(
                f"{path} is missing: build it with `python -m differential_attention_04_b200.build`"
                + (" --debug" if path == DEBUG_LIB_PATH else ""))
        handle = ctypes.CDLL(path)
        for name, (res, args) in SIGNATURES.items():
            fn = getattr(handle, name)
            fn.restype = res
            fn.argtypes = args
        _handles[path] = handle
    return _handles[path]


def lib() -> ctypes.CDLL:
    """Load (once) and return the active library with typed entry points."""
    return _load(_active)


def use_debug_library(on: bool = True) -> None:
    """Route every binding call to the bounds-checked build (on) or back to the release one.

    The two are separate libraries, each with its own device status word."""
    global _active
    _active = DEBUG_LIB_PATH if on else LIB_PATH
    _load(_active)
