"""ctypes loader for the in-tree CUDA library ``libdiffattn.so``.

Loading fails loudly when the library has not been built: there is no other
implementation behind these calls.
"""
from __future__ import annotations

import ctypes
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libdiffattn.so")

_lib = None

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


def lib() -> ctypes.CDLL:
    """Load (once) and return the library with typed entry points."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(
                f"{LIB_PATH} is missing: build it with `python -m differential_attention_04_b200.build`")
        handle = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in SIGNATURES.items():
            fn = getattr(handle, name)
            fn.restype = res
            fn.argtypes = args
        _lib = handle
    return _lib
