"""GPU parity of the backward pass against its float64 oracle (oracle/bwd_ref.py).

The kernels compute in float32 on CUDA cores from the exact input values, so
the comparison is against float32 rounding: a normwise relative error of at
most 2e-5 and a max-abs error of at most 1e-4 of the largest gradient entry
(a few thousand fp32 accumulations with exp at about 1e-7 each), dlambda and
the norm weight's gradient to 1e-4 relative.  Gradients that vanish in exact
arithmetic (dq and dk when a row sees a single key) are held to an absolute
floor of 1e-5 of the largest dv entry: float32 leaves noise of about 1e-7
there.
"""
import numpy as np
import pytest
import torch

import oracle.bwd_ref as bwd
from differential_attention_04_b200 import api
from differential_attention_04_b200 import workloads as wl

from test_parity_gpu import oracle_lambda

pytestmark = pytest.mark.gpu

MODES = {api.MODE_DIFF: "diff", api.MODE_LAMBDA_ZERO: "lambda_zero", api.MODE_SUM: "sum"}


def _close(got, want, name, rel_norm=2e-5, rel_max=1e-4, scale_floor=0.0):
    """Errors relative to the gradient's own size, or to scale_floor where that is larger."""
    got, want = np.asarray(got, dtype=np.float64), np.asarray(want, dtype=np.float64)
    scale = max(float(np.max(np.abs(want))), scale_floor, 1e-30)
    norm_ref = max(float(np.linalg.norm(want)), scale_floor * np.sqrt(want.size), 1e-30)
    norm = float(np.linalg.norm(got - want)) / norm_ref
    mx = float(np.max(np.abs(got - want))) / scale
    assert norm <= rel_norm and mx <= rel_max, f"{name}: normwise {norm:.2e}, max {mx:.2e}"


def _check(inp, mode=api.MODE_DIFF, seed=0):
    g = torch.Generator(device="cuda").manual_seed(seed)
    dy = torch.randn(inp.v.shape, generator=g, device="cuda").to(inp.v.dtype)
    lam = api.diffattn_lambda(inp.lq1, inp.lk1, inp.lq2, inp.lk2, inp.lambda_init)
    dq, dk, dv, dlam, dw = api.diffattn_bwd(inp.q, inp.k, inp.v, dy, lam, inp.lambda_init, inp.rms_w, inp.eps,
                                            inp.causal, mode)
    torch.cuda.synchronize()
    f = wl.to_f64
    want = bwd.diffattn_bwd(f(inp.q), f(inp.k), f(inp.v), f(dy), oracle_lambda(inp), inp.lambda_init,
                            f(inp.rms_w), inp.eps, inp.causal, MODES[mode])
    floor = 0.1 * float(np.max(np.abs(want[2])))  # allows 1e-5 of the largest dv entry where dq, dk vanish
    for name, got, w in zip(("dq", "dk", "dv"), (dq, dk, dv), want[:3]):
        _close(got.cpu().numpy(), w, name, scale_floor=floor)
    if mode != api.MODE_LAMBDA_ZERO:
        assert abs(float(dlam) - want[3]) <= 1e-4 * max(1.0, abs(want[3])), (float(dlam), want[3])
    else:
        assert float(dlam) == 0.0
        assert not dq[..., 1, :].any() and not dk[..., 1, :].any()
    _close(dw.cpu().numpy(), want[4], "dw", 1e-4, 1e-4)


@pytest.mark.parametrize("causal", [True, False])
@pytest.mark.parametrize("N,d", [(1, 8), (37, 7), (130, 64), (100, 128)])
def test_bwd_fp32(N, d, causal):
    inp = wl.make_prefill(2, N, 2, d, causal=causal, dtype="f32", lambda_init=0.3, w="normal", seed=N + d,
                          device="cuda")
    _check(inp, seed=N)


@pytest.mark.parametrize("mode", [api.MODE_LAMBDA_ZERO, api.MODE_SUM])
def test_bwd_modes(mode):
    inp = wl.make_prefill(1, 90, 3, 32, causal=True, dtype="f32", lambda_init=0.5, w="normal", seed=5,
                          device="cuda")
    _check(inp, mode)


@pytest.mark.parametrize("causal", [True, False])
def test_bwd_bf16_inputs(causal):
    inp = wl.make_prefill(1, 300, 2, 128, causal=causal, dtype="bf16", lambda_init=0.5, w="normal", seed=9,
                          device="cuda")
    _check(inp, seed=3)


def test_bwd_longer_sequence():
    inp = wl.make_prefill(1, 1024, 2, 128, causal=True, dtype="bf16", lambda_init=0.65, w="normal", seed=11,
                          device="cuda")
    _check(inp, seed=4)


def test_lambda_bwd():
    inp = wl.make_prefill(1, 4, 1, 64, causal=True, dtype="f32", seed=13, device="cuda")
    dlam = torch.tensor([1.37], device="cuda")
    got = api.diffattn_lambda_bwd(inp.lq1, inp.lk1, inp.lq2, inp.lk2, dlam)
    torch.cuda.synchronize()
    f = wl.to_f64
    want = bwd.lambda_reparam_bwd(f(inp.lq1), f(inp.lk1), f(inp.lq2), f(inp.lk2), 1.37)
    for g_, w_ in zip(got, want):
        np.testing.assert_allclose(g_.cpu().numpy(), w_, rtol=1e-5, atol=1e-6)


def test_bwd_rejects_bad_workspace():
    inp = wl.make_prefill(1, 16, 1, 32, causal=True, dtype="f32", seed=1, device="cuda")
    lam = api.diffattn_lambda(inp.lq1, inp.lk1, inp.lq2, inp.lk2, inp.lambda_init)
    small = torch.empty(64, dtype=torch.uint8, device="cuda")
    with pytest.raises(api.DiffAttnError) as e:
        api.diffattn_bwd(inp.q, inp.k, inp.v, inp.v, lam, inp.lambda_init, inp.rms_w, inp.eps, True, workspace=small)
    assert e.value.status == api.ERR_WORKSPACE
