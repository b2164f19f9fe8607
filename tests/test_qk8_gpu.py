"""GPU parity of the e4m3 query/key path against its CPU oracle (oracle/qk8_ref.py).

The codes and scales are integer/exact decisions taken in float32 on both
sides, so they must match bit for bit; the forward is compared with the
oracle's float64 result on the dequantised queries and keys, with the bf16
tolerance of the other prefill tests.
"""
import numpy as np
import pytest
import torch

import oracle.diffattn_ref as ref
import oracle.qk8_ref as q8
from differential_attention_04_b200 import api
from differential_attention_04_b200 import workloads as wl

from test_parity_gpu import BF16_ABS, BF16_REL, assert_close, oracle_lambda

pytestmark = pytest.mark.gpu


def _quant_inputs(B, N, H, d, seed):
    g = torch.Generator(device="cuda").manual_seed(seed)
    x = torch.randn((B, N, H, 2, d), generator=g, device="cuda")
    # a different scale per (batch, head, map), a zero group and a huge value
    x *= torch.exp(2 * torch.randn((B, 1, H, 2, 1), generator=g, device="cuda"))
    if B * H > 1:
        x[0, :, 0, 1] = 0
    x[-1, N // 2, H - 1, 0, d - 1] = 3.0e4
    return x.to(torch.bfloat16)


@pytest.mark.parametrize("B,N,H,d", [(1, 1, 1, 8), (2, 37, 3, 64), (1, 300, 2, 128), (2, 517, 12, 128),
                                     (1, 4096, 4, 128)])
def test_quantize_bit_exact(B, N, H, d):
    x = _quant_inputs(B, N, H, d, seed=B * 1000 + N + d)
    codes, scales = api.quantize_qk(x)
    torch.cuda.synchronize()
    want_codes, want_scales = q8.quantize_qk(x.float().cpu().numpy())
    got_scales = scales.cpu().numpy()
    assert np.array_equal(got_scales.view(np.uint32), want_scales.view(np.uint32))
    got = codes.cpu().numpy()
    bad = np.argwhere(got != want_codes)
    assert bad.size == 0, f"{len(bad)} codes differ, first at {bad[0].tolist()}"


def _run_qk8(inp, mode=api.MODE_DIFF):
    lam = api.diffattn_lambda(inp.lq1, inp.lk1, inp.lq2, inp.lk2, inp.lambda_init)
    qc, qs = api.quantize_qk(inp.q)
    kc, ks = api.quantize_qk(inp.k)
    y = api.diffattn_fwd_qk8(qc, qs, kc, ks, inp.v, lam, inp.lambda_init, inp.rms_w, inp.eps, inp.causal, mode=mode)
    torch.cuda.synchronize()
    return y


def _oracle_qk8(inp, mode="diff", rows=None, heads=None):
    f = wl.to_f64
    return q8.diffattn_fwd_qk8(inp.q.float().cpu().numpy(), inp.k.float().cpu().numpy(), f(inp.v),
                               oracle_lambda(inp), inp.lambda_init, f(inp.rms_w), inp.eps, inp.causal,
                               rows=rows, heads=heads, mode=mode)


@pytest.mark.parametrize("causal", [True, False])
@pytest.mark.parametrize("N", [1, 128, 200, 517])
def test_fwd_qk8_parity(N, causal):
    inp = wl.make_prefill(2, N, 3, 128, causal=causal, dtype="bf16", lambda_init=0.5, w="normal", seed=61 + N,
                          device="cuda")
    assert_close(wl.to_f64(_run_qk8(inp)), _oracle_qk8(inp))


@pytest.mark.parametrize("mode,name", [(api.MODE_LAMBDA_ZERO, "lambda_zero"), (api.MODE_SUM, "sum")])
def test_fwd_qk8_modes(mode, name):
    inp = wl.make_prefill(1, 300, 2, 128, causal=True, dtype="bf16", lambda_init=0.6, w="normal", seed=71,
                          device="cuda")
    assert_close(wl.to_f64(_run_qk8(inp, mode)), _oracle_qk8(inp, name))


def test_fwd_qk8_large_scores():
    # scaled queries/keys: the rescale paths with e4m3 scores
    inp = wl.make_prefill(1, 640, 2, 128, causal=True, dtype="bf16", lambda_init=0.5, seed=73, device="cuda")
    ramp = torch.linspace(1.0, 24.0, 640, device="cuda").view(1, 640, 1, 1, 1)
    inp.k.copy_((inp.k.float() * ramp).to(inp.k.dtype))
    inp.q.mul_(4)
    y = _run_qk8(inp)
    assert torch.isfinite(y.float()).all()
    assert_close(wl.to_f64(y), _oracle_qk8(inp))


def test_fwd_qk8_full_size_sampled():
    # the bench workload (B4 H12 N4096 causal); sampled rows of three heads
    inp = wl.make_prefill_case("prefill_3b", seed=5, device="cuda")
    y = _run_qk8(inp)
    rows = [0, 1, 127, 128, 2047, 4000, 4095]
    heads = [(0, 0), (1, 7), (3, 11)]
    want = _oracle_qk8(inp, rows=rows, heads=heads)
    yf = wl.to_f64(y)
    for b, h in heads:
        assert_close(yf[b, rows, h], want[b, :, h])


def test_qk8_close_to_bf16_path():
    # the e4m3 scores only perturb the result by the quantisation error
    inp = wl.make_prefill(1, 512, 4, 128, causal=True, dtype="bf16", lambda_init=0.5, w="normal", seed=79,
                          device="cuda")
    y8 = wl.to_f64(_run_qk8(inp))
    lam = api.diffattn_lambda(inp.lq1, inp.lk1, inp.lq2, inp.lk2, inp.lambda_init)
    y16 = wl.to_f64(api.diffattn_fwd(inp.q, inp.k, inp.v, lam, inp.lambda_init, inp.rms_w, inp.eps, True))
    rel = np.linalg.norm(y8 - y16) / np.linalg.norm(y16)
    assert 1e-4 < rel < 0.1, rel


def test_qk8_rejects_unsupported():
    inp = wl.make_prefill(1, 16, 1, 64, causal=True, dtype="bf16", seed=1, device="cuda")
    lam = api.diffattn_lambda(inp.lq1, inp.lk1, inp.lq2, inp.lk2, inp.lambda_init)
    qc, qs = api.quantize_qk(inp.q)
    with pytest.raises(api.DiffAttnError) as e:
        api.diffattn_fwd_qk8(qc, qs, qc, qs, inp.v, lam, inp.lambda_init, inp.rms_w, inp.eps, True)
    assert e.value.status == api.ERR_UNSUPPORTED
