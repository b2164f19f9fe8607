"""Differential-attention forward for NVIDIA B200 (sm_100a).

The computation lives in the CUDA library ``libdiffattn.so`` (C ABI in
``include/diffattn.h``); this package is its thin Python binding plus the
seeded input generators.
"""
from .api import (  # noqa: F401
    BF16,
    ERR_CUDA,
    ERR_INVALID_ARG,
    ERR_TIMEOUT,
    ERR_UNSUPPORTED,
    ERR_WORKSPACE,
    F32,
    MODE_DIFF,
    MODE_LAMBDA_ZERO,
    MODE_SUM,
    OK,
    DiffAttnError,
    bwd_tc_workspace_size,
    bwd_workspace_size,
    decode_workspace_size,
    device_status,
    diffattn_bwd,
    diffattn_bwd_tc,
    diffattn_bwd_tc_saved,
    diffattn_decode,
    diffattn_decode_noalloc,
    diffattn_fwd,
    diffattn_fwd_qk4,
    diffattn_fwd_qk8,
    diffattn_fwd_train,
    diffattn_lambda,
    diffattn_lambda_bwd,
    out_proj,
    qkv_proj,
    quantize_qk,
    quantize_qk4,
    rope_table,
    set_wait_limit_ns,
)
