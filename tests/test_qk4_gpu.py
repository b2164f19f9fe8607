"""GPU parity of the e2m1 (FP4) query/key path against its CPU oracle
(oracle/qk4_ref.py).

The packed codes and the scales are exact decisions taken in float32 on both
sides, so they must match bit for bit.  The scores of 4-bit codes are exact
in the tensor cores' fp32 accumulation (every product is a multiple of 1/4 of
magnitude at most 36), so the forward is compared with the oracle's float64
result on the dequantised queries and keys with the same bf16 tolerance as
the other prefill tests.
"""
import numpy as np
import pytest
import torch

import oracle.qk4_ref as q4
from differential_attention_04_b200 import api
from differential_attention_04_b200 import workloads as wl

from test_parity_gpu import assert_close, oracle_lambda
from test_qk8_gpu import _quant_inputs

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("B,N,H,d", [(1, 1, 1, 8), (2, 37, 3, 64), (1, 300, 2, 128), (2, 517, 12, 128),
                                     (1, 4096, 4, 128)])
def test_quantize4_bit_exact(B, N, H, d):
    x = _quant_inputs(B, N, H, d, seed=B * 2000 + N + d)
    codes, scales = api.quantize_qk4(x)
    torch.cuda.synchronize()
    want_codes, want_scales = q4.quantize_qk(x.float().cpu().numpy())
    got_scales = scales.cpu().numpy()
    assert np.array_equal(got_scales.view(np.uint32), want_scales.view(np.uint32))
    got = codes.cpu().numpy()
    want = q4.pack(want_codes)
    assert got.shape == want.shape
    bad = np.argwhere(got != want)
    assert bad.size == 0, f"{len(bad)} bytes differ, first at {bad[0].tolist()}"


def _run_qk4(inp, mode=api.MODE_DIFF):
    lam = api.diffattn_lambda(inp.lq1, inp.lk1, inp.lq2, inp.lk2, inp.lambda_init)
    qc, qs = api.quantize_qk4(inp.q)
    kc, ks = api.quantize_qk4(inp.k)
    y = api.diffattn_fwd_qk4(qc, qs, kc, ks, inp.v, lam, inp.lambda_init, inp.rms_w, inp.eps, inp.causal, mode=mode)
    torch.cuda.synchronize()
    return y


def _oracle_qk4(inp, mode="diff", rows=None, heads=None):
    f = wl.to_f64
    return q4.diffattn_fwd_qk4(inp.q.float().cpu().numpy(), inp.k.float().cpu().numpy(), f(inp.v),
                               oracle_lambda(inp), inp.lambda_init, f(inp.rms_w), inp.eps, inp.causal,
                               rows=rows, heads=heads, mode=mode)


@pytest.mark.parametrize("causal", [True, False])
@pytest.mark.parametrize("N", [1, 128, 200, 517])
def test_fwd_qk4_parity(N, causal):
    inp = wl.make_prefill(2, N, 3, 128, causal=causal, dtype="bf16", lambda_init=0.5, w="normal", seed=161 + N,
                          device="cuda")
    assert_close(wl.to_f64(_run_qk4(inp)), _oracle_qk4(inp))


@pytest.mark.parametrize("mode,name", [(api.MODE_LAMBDA_ZERO, "lambda_zero"), (api.MODE_SUM, "sum")])
def test_fwd_qk4_modes(mode, name):
    inp = wl.make_prefill(1, 300, 2, 128, causal=True, dtype="bf16", lambda_init=0.6, w="normal", seed=171,
                          device="cuda")
    assert_close(wl.to_f64(_run_qk4(inp, mode)), _oracle_qk4(inp, name))


def test_fwd_qk4_large_scores():
    # scaled queries/keys: the rescale paths with 4-bit scores
    inp = wl.make_prefill(1, 640, 2, 128, causal=True, dtype="bf16", lambda_init=0.5, seed=173, device="cuda")
    ramp = torch.linspace(1.0, 24.0, 640, device="cuda").view(1, 640, 1, 1, 1)
    inp.k.copy_((inp.k.float() * ramp).to(inp.k.dtype))
    inp.q.mul_(4)
    y = _run_qk4(inp)
    assert torch.isfinite(y.float()).all()
    assert_close(wl.to_f64(y), _oracle_qk4(inp))


def test_fwd_qk4_full_size_sampled():
    # the 3B-like prefill workload (B4 H12 N4096 causal); sampled rows of three heads
    inp = wl.make_prefill_case("prefill_3b", seed=5, device="cuda")
    y = _run_qk4(inp)
    rows = [0, 1, 127, 128, 2047, 4000, 4095]
    heads = [(0, 0), (1, 7), (3, 11)]
    want = _oracle_qk4(inp, rows=rows, heads=heads)
    yf = wl.to_f64(y)
    for b, h in heads:
        assert_close(yf[b, rows, h], want[b, :, h])


def test_qk4_further_from_bf16_than_qk8():
    # 4-bit scores perturb the result more than 8-bit ones, and both stay near the bf16 path
    inp = wl.make_prefill(1, 512, 4, 128, causal=True, dtype="bf16", lambda_init=0.5, w="normal", seed=179,
                          device="cuda")
    lam = api.diffattn_lambda(inp.lq1, inp.lk1, inp.lq2, inp.lk2, inp.lambda_init)
    y16 = wl.to_f64(api.diffattn_fwd(inp.q, inp.k, inp.v, lam, inp.lambda_init, inp.rms_w, inp.eps, True))
    qc, qs = api.quantize_qk(inp.q)
    kc, ks = api.quantize_qk(inp.k)
    y8 = wl.to_f64(api.diffattn_fwd_qk8(qc, qs, kc, ks, inp.v, lam, inp.lambda_init, inp.rms_w, inp.eps, True))
    y4 = wl.to_f64(_run_qk4(inp))
    rel8 = np.linalg.norm(y8 - y16) / np.linalg.norm(y16)
    rel4 = np.linalg.norm(y4 - y16) / np.linalg.norm(y16)
    assert rel8 < rel4 < 0.5, (rel8, rel4)


def test_qk4_rejects():
    inp = wl.make_prefill(1, 16, 1, 64, causal=True, dtype="bf16", seed=1, device="cuda")
    lam = api.diffattn_lambda(inp.lq1, inp.lk1, inp.lq2, inp.lk2, inp.lambda_init)
    qc, qs = api.quantize_qk4(inp.q)
    with pytest.raises(api.DiffAttnError) as e:  # d = 64
        api.diffattn_fwd_qk4(qc, qs, qc, qs, inp.v, lam, inp.lambda_init, inp.rms_w, inp.eps, True)
    assert e.value.status == api.ERR_UNSUPPORTED
    inp = wl.make_prefill(1, 16, 1, 128, causal=True, dtype="bf16", seed=2, device="cuda")
    qc, qs = api.quantize_qk4(inp.q)
    buf = torch.zeros(qc.numel() + 64, dtype=torch.uint8, device="cuda")
    off = buf[16:16 + qc.numel()].view(qc.shape)  # 16- but not 32-byte aligned
    off.copy_(qc)
    with pytest.raises(api.DiffAttnError) as e:
        api.diffattn_fwd_qk4(off, qs, qc, qs, inp.v, lam, inp.lambda_init, inp.rms_w, inp.eps, True)
    assert e.value.status == api.ERR_INVALID_ARG
