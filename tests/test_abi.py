"""The C-ABI library loads and exports every entry point declared in
include/*.h; host-side validation rejects bad arguments before any CUDA call
(no GPU needed)."""
import ctypes
import glob
import os
import re

import pytest

from differential_attention_04_b200 import _lib, api
from differential_attention_04_b200.build import build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def L():
    build()
    return _lib.lib()


def _declared():
    names = set()
    for h in glob.glob(os.path.join(ROOT, "include", "*.h")):
        txt = open(h).read()
        txt = re.sub(r"/\*.*?\*/", "", txt, flags=re.S)
        names |= set(re.findall(r"\b(diffattn_\w+)\s*\(", txt))
    return names


def test_every_declared_symbol_is_exported(L):
    declared = _declared()
    assert {"diffattn_lambda", "diffattn_fwd", "diffattn_decode"} <= declared
    for name in sorted(declared):
        assert hasattr(L, name), f"{name} declared in include/ but not exported"


def test_binding_covers_header(L):
    assert _declared() == set(_lib.SIGNATURES)


def test_status_strings_and_version(L):
    assert L.diffattn_version() >= 100
    for code in range(6):
        assert L.diffattn_status_string(code)
    assert L.diffattn_status_string(99) == b"unknown status"


def test_validation_without_gpu(L):
    # every case below is rejected before the library touches CUDA
    nul = None
    assert L.diffattn_lambda(nul, nul, nul, nul, 64, 0.5, nul, nul) == api.ERR_INVALID_ARG
    fake = ctypes.c_void_p(4096)
    assert L.diffattn_lambda(fake, fake, fake, fake, 0, 0.5, fake, nul) == api.ERR_INVALID_ARG
    # prefill: bad sizes, bad dtype, null and misaligned pointers
    args = lambda q, dt, B, N, H, d, eps=1e-5: L.diffattn_fwd(q, q, q, q, dt, B, N, H, d, 1, q, 0.5, q, eps, nul)
    assert args(fake, api.BF16, 0, 16, 2, 128) == api.ERR_INVALID_ARG
    assert args(fake, api.BF16, 1, -1, 2, 128) == api.ERR_INVALID_ARG
    assert args(fake, 7, 1, 16, 2, 128) == api.ERR_INVALID_ARG
    assert args(fake, api.BF16, 1, 16, 2, 128, eps=-1.0) == api.ERR_INVALID_ARG
    assert args(nul, api.BF16, 1, 16, 2, 128) == api.ERR_INVALID_ARG
    assert args(ctypes.c_void_p(4100), api.BF16, 1, 16, 2, 128) == api.ERR_INVALID_ARG
    assert args(fake, api.BF16, 1, 16, 2, 96) == api.ERR_UNSUPPORTED
    assert args(fake, api.F32, 1, 16, 2, 129) == api.ERR_UNSUPPORTED
    assert args(fake, api.BF16, 1 << 16, 1 << 16, 2, 128) == api.ERR_INVALID_ARG  # > 2^31 elements
    assert args(nul, api.BF16, 1, 0, 2, 128) == api.OK  # N = 0 is a no-op
    # prefill with a combination mode: unknown modes are rejected
    margs = lambda q, mode: L.diffattn_fwd_mode(q, q, q, q, api.BF16, 1, 16, 2, 128, 1, q, 0.5, q, 1e-5, mode, nul)
    for bad in (-1, 3, 7):
        assert margs(fake, bad) == api.ERR_INVALID_ARG
    assert margs(nul, api.MODE_SUM) == api.ERR_INVALID_ARG
    assert L.diffattn_fwd_mode(nul, nul, nul, nul, api.BF16, 1, 0, 2, 128, 1, nul, 0.5, nul, 1e-5,
                               api.MODE_LAMBDA_ZERO, nul) == api.OK
    # e4m3 queries/keys: quantiser and forward
    qz = lambda x, N, d, B=1, H=2: L.diffattn_quantize_qk(x, B, N, H, d, x, x, nul)
    assert qz(fake, 16, 12) == api.ERR_INVALID_ARG      # d not a multiple of 8
    assert qz(fake, 0, 128) == api.ERR_INVALID_ARG
    assert qz(nul, 16, 128) == api.ERR_INVALID_ARG
    assert qz(fake, 16, 128, B=1 << 15, H=2) == api.ERR_UNSUPPORTED  # B*H*2 > 65535 groups
    f8 = lambda x, N, d, mode=0: L.diffattn_fwd_qk8(x, x, x, x, x, x, 1, N, 2, d, 1, x, 0.5, x, 1e-5, mode, nul)
    assert f8(fake, 16, 64) == api.ERR_UNSUPPORTED
    assert f8(fake, 16, 128, mode=5) == api.ERR_INVALID_ARG
    assert f8(nul, 16, 128) == api.ERR_INVALID_ARG
    assert f8(nul, 0, 128) == api.OK
    # e2m1 queries/keys: same checks, and the codes must be 32-byte aligned
    qz4 = lambda x, N, d, B=1, H=2: L.diffattn_quantize_qk4(x, B, N, H, d, x, x, nul)
    assert qz4(fake, 16, 12) == api.ERR_INVALID_ARG
    assert qz4(nul, 16, 128) == api.ERR_INVALID_ARG
    assert qz4(fake, 16, 128, B=1 << 15, H=2) == api.ERR_UNSUPPORTED
    f4 = lambda x, c, N, d, mode=0: L.diffattn_fwd_qk4(c, x, c, x, x, x, 1, N, 2, d, 1, x, 0.5, x, 1e-5, mode, nul)
    assert f4(fake, fake, 16, 64) == api.ERR_UNSUPPORTED
    assert f4(fake, fake, 16, 128, mode=5) == api.ERR_INVALID_ARG
    assert f4(fake, ctypes.c_void_p(4096 + 16), 16, 128) == api.ERR_INVALID_ARG  # 16- but not 32-byte aligned
    assert f4(nul, nul, 16, 128) == api.ERR_INVALID_ARG
    assert f4(nul, nul, 0, 128) == api.OK
    # backward
    bw = lambda x, N, d, ws, wsb, mode=0: L.diffattn_bwd(x, x, x, x, api.F32, 1, N, 2, d, 1, x, 0.5, x, 1e-5, mode,
                                                         x, x, x, x, x, ws, wsb, nul)
    assert bw(fake, 16, 129, fake, 1 << 30) == api.ERR_UNSUPPORTED
    assert bw(fake, 16, 64, nul, 1 << 30) == api.ERR_WORKSPACE
    assert bw(fake, 16, 64, fake, 16) == api.ERR_WORKSPACE
    assert bw(nul, 16, 64, fake, 1 << 30) == api.ERR_INVALID_ARG
    assert bw(fake, 16, 64, fake, 1 << 30, mode=9) == api.ERR_INVALID_ARG
    assert bw(fake, 0, 64, fake, 1 << 30) == api.ERR_INVALID_ARG
    assert L.diffattn_bwd_workspace_size(1, 16, 2, 64) == 4 * 16 * 2 * 128 + 16 * 16 * 2
    assert L.diffattn_bwd_workspace_size(0, 16, 2, 64) == 0
    assert L.diffattn_lambda_bwd(nul, nul, nul, nul, 8, nul, nul, nul, nul, nul, nul) == api.ERR_INVALID_ARG
    # tensor-core backward: d in {64, 128}, aligned pointers, enough workspace
    tc = lambda x, N, d, ws, wsb, mode=0: L.diffattn_bwd_tc(x, x, x, x, 1, N, 2, d, 1, x, 0.5, x, 1e-5, mode,
                                                            x, x, x, x, x, ws, wsb, nul)
    assert tc(fake, 16, 96, fake, 1 << 30) == api.ERR_UNSUPPORTED
    assert tc(fake, 16, 32, fake, 1 << 30) == api.ERR_UNSUPPORTED
    assert tc(fake, 16, 128, nul, 1 << 30) == api.ERR_WORKSPACE
    assert tc(fake, 16, 128, fake, 16) == api.ERR_WORKSPACE
    assert tc(nul, 16, 128, fake, 1 << 30) == api.ERR_INVALID_ARG
    assert tc(ctypes.c_void_p(4104), 16, 128, fake, 1 << 30) == api.ERR_INVALID_ARG
    assert tc(fake, 16, 128, fake, 1 << 30, mode=4) == api.ERR_INVALID_ARG
    assert tc(fake, 0, 128, fake, 1 << 30) == api.ERR_INVALID_ARG
    # per map A_i V (float32), dO (bf16), 16 bytes per (b, h, n) with n rounded up to 128; 256-byte sections
    up = lambda x: (x + 255) // 256 * 256
    assert L.diffattn_bwd_tc_workspace_size(1, 16, 2, 64) == up(4 * 16 * 2 * 2 * 128) + up(2 * 16 * 2 * 128) + \
        up(16 * 2 * 128)
    assert L.diffattn_bwd_tc_workspace_size(2, 300, 3, 128) == up(4 * 600 * 3 * 2 * 256) + up(2 * 600 * 3 * 256) + \
        up(16 * 2 * 3 * 384)
    assert L.diffattn_bwd_tc_workspace_size(1, 0, 2, 64) == 0
    # training pair
    ft = lambda x, d, ws, wsb, mode=0: L.diffattn_fwd_train(x, x, x, x, 1, 16, 2, d, 1, x, 0.5, x, 1e-5, mode, ws, wsb,
                                                            nul)
    assert ft(fake, 96, fake, 1 << 30) == api.ERR_UNSUPPORTED
    assert ft(fake, 128, nul, 1 << 30) == api.ERR_WORKSPACE
    assert ft(fake, 128, fake, 16) == api.ERR_WORKSPACE
    assert ft(nul, 128, fake, 1 << 30) == api.ERR_INVALID_ARG
    assert ft(fake, 128, fake, 1 << 30, mode=3) == api.ERR_INVALID_ARG
    ts = lambda x, d, ws, wsb: L.diffattn_bwd_tc_saved(x, x, x, x, 1, 16, 2, d, 1, x, 0.5, x, 1e-5, 0,
                                                       x, x, x, x, x, ws, wsb, nul)
    assert ts(fake, 96, fake, 1 << 30) == api.ERR_UNSUPPORTED
    assert ts(fake, 128, fake, 16) == api.ERR_WORKSPACE
    assert ts(nul, 128, fake, 1 << 30) == api.ERR_INVALID_ARG
    # projections: sizes, multiples, pointers
    assert L.diffattn_rope_table(0, 64, 1e4, fake, nul) == api.ERR_INVALID_ARG
    assert L.diffattn_rope_table(16, 7, 1e4, fake, nul) == api.ERR_INVALID_ARG
    assert L.diffattn_rope_table(16, 64, -1.0, fake, nul) == api.ERR_INVALID_ARG
    assert L.diffattn_rope_table(16, 64, 1e4, nul, nul) == api.ERR_INVALID_ARG
    qp = lambda x, dm, d, rope=None: L.diffattn_qkv_proj(x, x, 2, 16, dm, 2, d, rope, x, x, x, nul)
    assert qp(fake, 96, 64) == api.ERR_UNSUPPORTED     # d_model not a multiple of 64
    assert qp(fake, 128, 48) == api.ERR_UNSUPPORTED    # d not a multiple of 32
    assert qp(nul, 128, 64) == api.ERR_INVALID_ARG
    assert qp(ctypes.c_void_p(4104), 128, 64) == api.ERR_INVALID_ARG
    assert qp(fake, 128, 64, rope=ctypes.c_void_p(4100)) == api.ERR_INVALID_ARG
    assert L.diffattn_qkv_proj(fake, fake, 0, 16, 128, 2, 64, nul, fake, fake, fake, nul) == api.ERR_INVALID_ARG
    op = lambda x, M, K, n: L.diffattn_out_proj(x, x, M, K, n, x, nul)
    assert op(fake, 16, 96, 64) == api.ERR_UNSUPPORTED
    assert op(fake, 16, 128, 48) == api.ERR_UNSUPPORTED
    assert op(fake, 0, 128, 64) == api.ERR_INVALID_ARG
    assert op(nul, 16, 128, 64) == api.ERR_INVALID_ARG
    # decode
    dec = lambda q, d, ws, wsb, S=4: L.diffattn_decode(q, q, q, q, 100, q, S, 2, d, q, 0.5, q, 1e-5, ws, wsb, nul)
    assert dec(nul, 128, fake, 1 << 30) == api.ERR_INVALID_ARG
    assert dec(fake, 64, fake, 1 << 30) == api.ERR_UNSUPPORTED
    assert dec(fake, 128, nul, 1 << 30) == api.ERR_WORKSPACE
    assert dec(fake, 128, fake, 16) == api.ERR_WORKSPACE
    assert dec(fake, 128, fake, 1 << 30, S=0) == api.ERR_INVALID_ARG
    decm = lambda mode: L.diffattn_decode_mode(fake, fake, fake, fake, 100, fake, 4, 2, 128, fake, 0.5, fake, 1e-5,
                                               mode, fake, 1 << 30, nul)
    assert decm(3) == api.ERR_INVALID_ARG and decm(-1) == api.ERR_INVALID_ARG


def test_workspace_size(L):
    assert L.diffattn_decode_workspace_size(0, 12, 128, 100) == 0
    assert L.diffattn_decode_workspace_size(4, 12, 64, 100) == 0
    # one record per (key chunk of up to 512 keys, head): m1, l1, m2, l2 and two
    # 256-wide partial outputs in float32, then the S + 1 chunk offsets (int32)
    rec = (4 + 2 * 256) * 4
    one = L.diffattn_decode_workspace_size(1, 1, 128, 1)
    assert one % 16 == 0 and one >= rec + 2 * 4
    many = L.diffattn_decode_workspace_size(3, 5, 128, 1)
    assert many % 16 == 0 and many >= 15 * rec + 4 * 4
    # grows with the number of key chunks per sequence
    long = L.diffattn_decode_workspace_size(1, 1, 128, 100000)
    assert long % 16 == 0 and long >= 196 * rec


def test_wait_limit_setter(L):
    assert L.diffattn_set_wait_limit_ns(-1) == api.ERR_INVALID_ARG
    assert L.diffattn_set_wait_limit_ns(0) == api.OK


def test_package_exports_every_binding():
    import inspect

    import differential_attention_04_b200 as pkg

    public = {n for n, f in inspect.getmembers(api, inspect.isfunction)
              if f.__module__ == api.__name__ and not n.startswith("_")}
    assert public, "no binding functions found"
    missing = sorted(n for n in public if not hasattr(pkg, n))
    assert not missing, f"not exported from the package: {missing}"
