"""Differential-attention forward for NVIDIA B200 (sm_100a).

The computation lives in the CUDA library ``libdiffattn.so`` (C ABI in
``include/diffattn.h``); this package is its thin Python binding plus the
seeded input generators.
"""
from .api import (  # noqa: F401
    BF16,
    F32,
    DiffAttnError,
    decode_workspace_size,
    device_status,
    diffattn_decode,
    diffattn_fwd,
    diffattn_lambda,
    set_wait_limit_ns,
)
