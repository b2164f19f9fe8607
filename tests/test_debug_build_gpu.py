"""The bounds-checked debug build (libdiffattn_debug.so, -DDIFFATTN_DEBUG).

Its kernels check every global index and tensor-map coordinate before use,
skip an access out of range (never trap) and record DIFFATTN_ERR_BOUNDS in the
device status word.  Checked through the C ABI:
  * the parity cases of the release library (prefill bf16 and fp32, decode,
    low-bit queries and keys, the projections, the tensor-core backward) give
    the same results against the float64 oracle, and the status stays OK;
  * the full-size prefill configurations, the decode workload, and the
    backward and projections at the 3B-like shapes pass every check (status
    OK) and give the release library's results (bit for bit where each
    output element is written once);
  * a decode whose cu_seqlens gives a sequence more keys than max_seqlen (a
    host-built input that stays inside the cache: the kernels only ever read
    the first max_seqlen keys of a sequence) sets DIFFATTN_ERR_BOUNDS in the
    debug build, and leaves the status OK in the release build, which cuts
    the sequence silently.
"""
import numpy as np
import pytest
import torch

import oracle.bwd_ref as bwd_ref
import oracle.diffattn_ref as ref
import oracle.proj_ref as proj_ref
import oracle.qk8_ref as q8
from differential_attention_04_b200 import _lib, api
from differential_attention_04_b200 import workloads as wl

pytestmark = pytest.mark.gpu

BF16_REL, BF16_ABS = 5e-3, 2e-2
F32_TOL = 1e-5
f = wl.to_f64


@pytest.fixture(scope="module", autouse=True)
def _debug_library():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from differential_attention_04_b200.build import build
    build()
    build(debug=True)
    torch.cuda.set_device(0)
    _lib.use_debug_library(True)
    assert api.device_status() == api.OK
    yield
    _lib.use_debug_library(False)


def _close(y, want, fp32=False):
    y = f(y) if isinstance(y, torch.Tensor) else np.asarray(y)
    assert np.isfinite(y).all()
    rel = np.linalg.norm(y - want) / np.linalg.norm(want)
    mx = np.abs(y - want).max()
    tol = (F32_TOL, F32_TOL) if fp32 else (BF16_REL, BF16_ABS)
    assert rel <= tol[0] and mx <= tol[1], f"rel {rel:.3e} max-abs {mx:.3e}"


def _lam(inp):
    return ref.lambda_reparam(f(inp.lq1), f(inp.lk1), f(inp.lq2), f(inp.lk2), inp.lambda_init)


@pytest.mark.parametrize("N,d,causal", [(1, 128, True), (517, 128, True), (300, 64, False), (384, 128, False)])
def test_prefill_bf16_under_debug_build(N, d, causal):
    inp = wl.make_prefill(2, N, 3, d, causal=causal, dtype="bf16", seed=N + d, device="cuda")
    lam = api.diffattn_lambda(inp.lq1, inp.lk1, inp.lq2, inp.lk2, inp.lambda_init)
    y = api.diffattn_fwd(inp.q, inp.k, inp.v, lam, inp.lambda_init, inp.rms_w, inp.eps, causal)
    torch.cuda.synchronize()
    want = ref.diffattn_fwd(f(inp.q), f(inp.k), f(inp.v), _lam(inp), inp.lambda_init, f(inp.rms_w), inp.eps, causal)
    _close(y, want)
    assert api.device_status() == api.OK


def test_prefill_fp32_under_debug_build():
    inp = wl.make_prefill_case("tiny_fp32", device="cuda")
    lam = api.diffattn_lambda(inp.lq1, inp.lk1, inp.lq2, inp.lk2, inp.lambda_init)
    y = api.diffattn_fwd(inp.q, inp.k, inp.v, lam, inp.lambda_init, inp.rms_w, inp.eps, True)
    torch.cuda.synchronize()
    want = ref.diffattn_fwd(f(inp.q), f(inp.k), f(inp.v), _lam(inp), inp.lambda_init, f(inp.rms_w), inp.eps, True)
    _close(y, want, fp32=True)
    assert api.device_status() == api.OK


def _oracle_decode(inp):
    return ref.diffattn_decode(f(inp.q), f(inp.k_cache), f(inp.v_cache), inp.cu_seqlens.cpu().numpy(), _lam(inp),
                               inp.lambda_init, f(inp.rms_w), inp.eps)


def test_decode_under_debug_build():
    inp = wl.make_decode(5, 3, 128, 0, 0, seqlens=[1, 511, 512, 513, 1700], seed=7, device="cuda")
    lam = api.diffattn_lambda(inp.lq1, inp.lk1, inp.lq2, inp.lk2, inp.lambda_init)
    y = api.diffattn_decode(inp.q, inp.k_cache, inp.v_cache, inp.cu_seqlens, inp.max_seqlen, lam, inp.lambda_init,
                            inp.rms_w, inp.eps)
    torch.cuda.synchronize()
    _close(y, _oracle_decode(inp))
    assert api.device_status() == api.OK


def test_lowbit_under_debug_build():
    inp = wl.make_prefill(1, 300, 2, 128, causal=True, dtype="bf16", seed=11, device="cuda")
    lam = api.diffattn_lambda(inp.lq1, inp.lk1, inp.lq2, inp.lk2, inp.lambda_init)
    qc, qs = api.quantize_qk(inp.q)
    kc, ks = api.quantize_qk(inp.k)
    y = api.diffattn_fwd_qk8(qc, qs, kc, ks, inp.v, lam, inp.lambda_init, inp.rms_w, inp.eps, True)
    torch.cuda.synchronize()
    want = q8.diffattn_fwd_qk8(inp.q.float().cpu().numpy(), inp.k.float().cpu().numpy(), f(inp.v), _lam(inp),
                               inp.lambda_init, f(inp.rms_w), inp.eps, True)
    _close(y, want)
    assert api.device_status() == api.OK


def test_projections_under_debug_build():
    pj = wl.make_proj(1, 100, 128, 2, 64, seed=2, device="cuda")
    q, k, v = api.qkv_proj(pj.x, pj.w_qkv, 1, 100, 2, 64, api.rope_table(100, 64))
    torch.cuda.synchronize()
    for got, want in zip((q, k, v), proj_ref.qkv_proj(f(pj.x), f(pj.w_qkv), 1, 100, 2, 64)):
        rel = np.linalg.norm(f(got) - want) / np.linalg.norm(want)
        assert rel <= BF16_REL
    assert api.device_status() == api.OK


def test_backward_under_debug_build():
    inp = wl.make_prefill(1, 200, 2, 64, causal=True, dtype="bf16", seed=5, device="cuda")
    g = torch.Generator(device="cuda").manual_seed(3)
    dy = torch.randn(inp.v.shape, generator=g, device="cuda").to(torch.bfloat16)
    lam = api.diffattn_lambda(inp.lq1, inp.lk1, inp.lq2, inp.lk2, inp.lambda_init)
    grads = api.diffattn_bwd_tc(inp.q, inp.k, inp.v, dy, lam, inp.lambda_init, inp.rms_w, inp.eps, True)
    grads32 = api.diffattn_bwd(inp.q, inp.k, inp.v, dy, lam, inp.lambda_init, inp.rms_w, inp.eps, True)
    torch.cuda.synchronize()
    want = bwd_ref.diffattn_bwd(f(inp.q), f(inp.k), f(inp.v), f(dy), _lam(inp), inp.lambda_init, f(inp.rms_w),
                                inp.eps, True)
    for got in (grads, grads32):
        for x, w in zip(got[:3], want[:3]):
            assert np.linalg.norm(f(x) - w) / np.linalg.norm(w) <= 1e-2
    assert api.device_status() == api.OK


def _release(fn):
    """fn() run on the release library (the debug one is restored after)."""
    _lib.use_debug_library(False)
    try:
        out = fn()
        torch.cuda.synchronize()
        assert api.device_status() == api.OK
        return out
    finally:
        _lib.use_debug_library(True)


@pytest.mark.parametrize("case", ["prefill_3b", "prefill_64k_needle", "prefill_13b_causal", "prefill_13b_nomask"])
def test_full_size_prefill_under_debug_build(case):
    # every tile, tail and grid position of the full-size launches passes the
    # debug build's bounds checks, and the checks change no result
    inp = wl.make_prefill_case(case, device="cuda")
    lam = api.diffattn_lambda(inp.lq1, inp.lk1, inp.lq2, inp.lk2, inp.lambda_init)

    def run():
        return api.diffattn_fwd(inp.q, inp.k, inp.v, lam, inp.lambda_init, inp.rms_w, inp.eps, inp.causal)

    y = run()
    torch.cuda.synchronize()
    assert api.device_status() == api.OK
    assert torch.equal(y, _release(run))


def test_full_size_decode_under_debug_build():
    inp = wl.make_decode_case("decode_64x12", device="cuda")
    lam = api.diffattn_lambda(inp.lq1, inp.lk1, inp.lq2, inp.lk2, inp.lambda_init)

    def run():
        return api.diffattn_decode(inp.q, inp.k_cache, inp.v_cache, inp.cu_seqlens, inp.max_seqlen, lam,
                                   inp.lambda_init, inp.rms_w, inp.eps)

    y = run()
    torch.cuda.synchronize()
    assert api.device_status() == api.OK
    assert torch.equal(y, _release(run))


def test_full_size_backward_and_projections_under_debug_build():
    # the tensor-core backward and both projection GEMMs at the 3B-like shapes:
    # the checks pass and change nothing (dq, dk, dv and the projections are
    # each written once, so bit for bit; dlambda and the norm weight's gradient
    # are sums of per-CTA atomics, whose order varies)
    inp = wl.make_prefill_case("prefill_3b", device="cuda")
    g = torch.Generator(device="cuda").manual_seed(3)
    dy = torch.randn(inp.v.shape, generator=g, device="cuda").to(torch.bfloat16)
    lam = api.diffattn_lambda(inp.lq1, inp.lk1, inp.lq2, inp.lk2, inp.lambda_init)

    def bwd():
        return api.diffattn_bwd_tc(inp.q, inp.k, inp.v, dy, lam, inp.lambda_init, inp.rms_w, inp.eps, True)

    got = bwd()
    torch.cuda.synchronize()
    assert api.device_status() == api.OK
    want = _release(bwd)
    for x, w in zip(got[:3], want[:3]):
        assert torch.equal(x, w)
    for x, w in zip(got[3:], want[3:]):
        assert torch.allclose(x, w, rtol=1e-4, atol=1e-6)
    del got, want, inp, dy
    pj = wl.make_proj_case("proj_3b", device="cuda")
    table = api.rope_table(pj.N, pj.d)

    def proj():
        q, k, v = api.qkv_proj(pj.x, pj.w_qkv, pj.B, pj.N, pj.H, pj.d, table)
        return q, k, v, api.out_proj(v, pj.w_o)

    got = proj()
    torch.cuda.synchronize()
    assert api.device_status() == api.OK
    for x, w in zip(got, _release(proj)):
        assert torch.equal(x, w)


def _overlong_decode():
    """Sequence 1 holds 600 cached keys but max_seqlen says 512: every kernel
    reads at most the first 512 of them, all inside the cache."""
    inp = wl.make_decode(2, 2, 128, 0, 0, seqlens=[100, 600], seed=9, device="cuda")
    lam = api.diffattn_lambda(inp.lq1, inp.lk1, inp.lq2, inp.lk2, inp.lambda_init)
    y = api.diffattn_decode(inp.q, inp.k_cache, inp.v_cache, inp.cu_seqlens, 512, lam, inp.lambda_init, inp.rms_w,
                            inp.eps)
    torch.cuda.synchronize()
    return inp, y


def test_overlong_sequence_is_flagged_by_debug_build():
    inp, y = _overlong_decode()
    assert api.device_status() == api.ERR_BOUNDS
    # the sequence was cut to its first 512 keys: sequence 0 is untouched
    _close(y[:1], _oracle_decode(inp)[:1])
    assert api.device_status() == api.OK  # reading the status cleared it


def test_overlong_sequence_is_cut_silently_by_release_build():
    _lib.use_debug_library(False)
    try:
        _overlong_decode()
        assert api.device_status() == api.OK
    finally:
        _lib.use_debug_library(True)
