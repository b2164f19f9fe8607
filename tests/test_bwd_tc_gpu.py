"""GPU parity of the tensor-core backward (diffattn_bwd_tc) against the float64
oracle (oracle/bwd_ref.py).

The kernels take P, dO = G and dS as bf16 operands of tcgen05 products with
float32 accumulation, and the per-map outputs A_i V from a prefill whose P
is bf16 as well.  Each gradient entry is a sum over keys (or queries) of
products in which one or two factors carry a bf16 rounding (relative error
at most 2^-9 each, of random sign), so the error of a sum grows like
2^-9 times the root of the sum of its squared terms; with the cancellation
of signed G and dS entries that root is of the order of the sum itself.
Normwise that is a few 2^-9 = 1.95e-3: the bound is 1e-2, and the largest
single error at most 4e-2 of the largest entry (which is 15 to 20
standard deviations of a sum of that kind).  dlambda and the norm weight's
gradient are sums in float32 of the statistics pass's outputs: 1e-2
relative for dw.  dlambda = -<G, A_2 V> is a cancelling sum: the RMSNorm
backward makes G nearly orthogonal to O = A_1 V + c A_2 V in every row, so
|dlambda| is far below the size of its terms, and the statistics pass's
A_2 V carries the bf16 rounding of P (relative 2^-9 per term, independent
from term to term).  Its error is a random walk of about
2^-9 ||G * A_2 V||_F (elementwise product): the bound is four times that,
plus 1e-3 of |dlambda|.  Gradients that vanish in exact arithmetic (dq, dk
when a row sees a single key) are held against a floor of 0.1 of the
largest dv entry.
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
REL_NORM, REL_MAX, REL_SCALAR = 1e-2, 4e-2, 1e-2


def _err(got, want, scale_floor=0.0):
    got, want = np.asarray(got, dtype=np.float64), np.asarray(want, dtype=np.float64)
    scale = max(float(np.max(np.abs(want))), scale_floor, 1e-30)
    norm_ref = max(float(np.linalg.norm(want)), scale_floor * np.sqrt(want.size), 1e-30)
    return float(np.linalg.norm(got - want)) / norm_ref, float(np.max(np.abs(got - want))) / scale


def _close(got, want, name, scale_floor=0.0):
    norm, mx = _err(got, want, scale_floor)
    assert norm <= REL_NORM and mx <= REL_MAX, f"{name}: normwise {norm:.2e}, max {mx:.2e}"


def _dlam_noise_scale(q, k, v, dy, lam, lambda_init, w, eps, causal, mode):
    """||G * (A_2 V)||_F over all rows, from the oracle's own pieces (float64)."""
    B, N, H, _, d = q.shape
    c, _ = bwd.mode_coefficient(lam, mode)
    tot = 0.0
    for b in range(B):
        for h in range(H):
            a1 = bwd._masked_softmax(q[b, :, h, 0], k[b, :, h, 0], 1 / np.sqrt(d), causal)
            a2 = bwd._masked_softmax(q[b, :, h, 1], k[b, :, h, 1], 1 / np.sqrt(d), causal)
            o2 = a2 @ v[b, :, h]
            g, _ = bwd.rmsnorm_bwd(a1 @ v[b, :, h] + c * o2, dy[b, :, h], w, eps, lambda_init)
            tot += float(np.sum((g * o2) ** 2))
    return np.sqrt(tot)


def _run(inp, mode, seed):
    g = torch.Generator(device="cuda").manual_seed(seed)
    dy = torch.randn(inp.v.shape, generator=g, device="cuda").to(torch.bfloat16)
    lam = api.diffattn_lambda(inp.lq1, inp.lk1, inp.lq2, inp.lk2, inp.lambda_init)
    out = api.diffattn_bwd_tc(inp.q, inp.k, inp.v, dy, lam, inp.lambda_init, inp.rms_w, inp.eps, inp.causal, mode)
    torch.cuda.synchronize()
    assert api.device_status() == api.OK
    return dy, out


def _check(inp, mode=api.MODE_DIFF, seed=0):
    dy, (dq, dk, dv, dlam, dw) = _run(inp, mode, seed)
    f = wl.to_f64
    want = bwd.diffattn_bwd(f(inp.q), f(inp.k), f(inp.v), f(dy), oracle_lambda(inp), inp.lambda_init,
                            f(inp.rms_w), inp.eps, inp.causal, MODES[mode])
    floor = 0.1 * float(np.max(np.abs(want[2])))
    for name, got, w in zip(("dq", "dk", "dv"), (dq, dk, dv), want[:3]):
        _close(got.cpu().numpy(), w, name, scale_floor=floor)
    if mode != api.MODE_LAMBDA_ZERO:
        args = (f(inp.q), f(inp.k), f(inp.v), f(dy), oracle_lambda(inp), inp.lambda_init, f(inp.rms_w), inp.eps,
                inp.causal, MODES[mode])
        tol = 4 * 2.0 ** -9 * _dlam_noise_scale(*args) + 1e-3 * abs(want[3])
        assert abs(float(dlam) - want[3]) <= tol, (float(dlam), want[3], tol)
    else:
        assert float(dlam) == 0.0
        assert not dq[..., 1, :].any() and not dk[..., 1, :].any()
    norm, mx = _err(dw.cpu().numpy(), want[4])
    assert norm <= REL_SCALAR and mx <= REL_SCALAR, f"dw: normwise {norm:.2e}, max {mx:.2e}"


@pytest.mark.parametrize("causal", [True, False])
@pytest.mark.parametrize("B,N,H,d", [(1, 1, 2, 128), (2, 37, 2, 64), (1, 130, 2, 128), (1, 300, 2, 128),
                                     (2, 517, 3, 64)])
def test_bwd_tc_shapes(B, N, H, d, causal):
    inp = wl.make_prefill(B, N, H, d, causal=causal, dtype="bf16", lambda_init=0.5, w="normal", seed=N + d,
                          device="cuda")
    _check(inp, seed=N)


@pytest.mark.parametrize("mode", [api.MODE_LAMBDA_ZERO, api.MODE_SUM])
def test_bwd_tc_modes(mode):
    inp = wl.make_prefill(1, 200, 2, 128, causal=True, dtype="bf16", lambda_init=0.5, w="normal", seed=5,
                          device="cuda")
    _check(inp, mode)


def test_bwd_tc_longer_sequence():
    inp = wl.make_prefill(1, 1024, 2, 128, causal=True, dtype="bf16", lambda_init=0.65, w="normal", seed=11,
                          device="cuda")
    _check(inp, seed=4)


def test_bwd_tc_deterministic():
    """dq, dk and dv are written once per row, without atomics: bitwise equal across runs."""
    inp = wl.make_prefill(1, 384, 2, 128, causal=True, dtype="bf16", seed=21, device="cuda")
    _, a = _run(inp, api.MODE_DIFF, 1)
    _, b = _run(inp, api.MODE_DIFF, 1)
    for x, y in zip(a[:3], b[:3]):
        assert torch.equal(x, y)


def test_bwd_tc_full_size_sampled_heads():
    """The 3B-like prefill's shape (B=4, N=4096, H=12, d=128, causal) in one call,
    with dq, dk and dv of two (batch, head) pairs checked against the oracle
    run on those heads alone (the gradients of one head depend on its own
    q, k, v and dy, lambda and the norm weight only)."""
    inp = wl.make_prefill_case("prefill_3b", seed=0, device="cuda")
    dy, (dq, dk, dv, _, _) = _run(inp, api.MODE_DIFF, 7)
    f = wl.to_f64
    lam = oracle_lambda(inp)
    for b, h in [(0, 0), (3, 11)]:
        sl = (slice(b, b + 1), slice(None), slice(h, h + 1))
        want = bwd.diffattn_bwd(f(inp.q[sl]), f(inp.k[sl]), f(inp.v[sl]), f(dy[sl]), lam, inp.lambda_init,
                                f(inp.rms_w), inp.eps, True, "diff")
        floor = 0.1 * float(np.max(np.abs(want[2])))
        for name, got, w in zip(("dq", "dk", "dv"), (dq[sl], dk[sl], dv[sl]), want[:3]):
            _close(got.cpu().numpy(), w, f"{name}[{b},{h}]", scale_floor=floor)


def test_bwd_tc_rejects():
    inp = wl.make_prefill(1, 16, 1, 32, causal=True, dtype="bf16", seed=1, device="cuda")
    lam = api.diffattn_lambda(inp.lq1, inp.lk1, inp.lq2, inp.lk2, inp.lambda_init)
    with pytest.raises(api.DiffAttnError) as e:
        api.diffattn_bwd_tc(inp.q, inp.k, inp.v, inp.v, lam, inp.lambda_init, inp.rms_w, inp.eps, True)
    assert e.value.status == api.ERR_UNSUPPORTED
    inp = wl.make_prefill(1, 16, 1, 64, causal=True, dtype="bf16", seed=1, device="cuda")
    small = torch.empty(64, dtype=torch.uint8, device="cuda")
    with pytest.raises(api.DiffAttnError) as e:
        api.diffattn_bwd_tc(inp.q, inp.k, inp.v, inp.v, lam, inp.lambda_init, inp.rms_w, inp.eps, True,
                            workspace=small)
    assert e.value.status == api.ERR_WORKSPACE


@pytest.mark.parametrize("B,N,H,d,causal,mode", [(1, 300, 2, 128, True, api.MODE_DIFF), (2, 130, 3, 64, False, api.MODE_SUM),
                                                  (1, 517, 2, 128, True, api.MODE_LAMBDA_ZERO)])
def test_train_forward_and_saved_backward(B, N, H, d, causal, mode):
    """The training pair equals the separate calls: diffattn_fwd_train's output is bitwise the forward's,
    and diffattn_bwd_tc_saved (statistics from the training forward) bitwise the backward that
    recomputes them (dq, dk, dv; dlambda and dw are atomic sums, equal up to the order of the additions)."""
    inp = wl.make_prefill(B, N, H, d, causal=causal, dtype="bf16", lambda_init=0.5, w="normal", seed=N + d,
                          device="cuda")
    g = torch.Generator(device="cuda").manual_seed(11)
    dy = torch.randn(inp.v.shape, generator=g, device="cuda").to(torch.bfloat16)
    lam = api.diffattn_lambda(inp.lq1, inp.lk1, inp.lq2, inp.lk2, inp.lambda_init)
    y_ref = api.diffattn_fwd(inp.q, inp.k, inp.v, lam, inp.lambda_init, inp.rms_w, inp.eps, causal, mode=mode)
    y, ws = api.diffattn_fwd_train(inp.q, inp.k, inp.v, lam, inp.lambda_init, inp.rms_w, inp.eps, causal, mode)
    saved = api.diffattn_bwd_tc_saved(inp.q, inp.k, inp.v, dy, lam, inp.lambda_init, inp.rms_w, inp.eps, causal, mode,
                                      ws)
    fresh = api.diffattn_bwd_tc(inp.q, inp.k, inp.v, dy, lam, inp.lambda_init, inp.rms_w, inp.eps, causal, mode)
    torch.cuda.synchronize()
    assert api.device_status() == api.OK
    assert torch.equal(y, y_ref)
    for a, b in zip(saved[:3], fresh[:3]):
        assert torch.equal(a, b)
    # dlambda and dw add per-CTA partial sums with float atomics in the order the CTAs finish: reordering
    # changes a sum of a few hundred fp32 partials by at most a few hundred roundings of the largest one
    for a, b in zip(saved[3:], fresh[3:]):
        assert (a - b).abs().max() <= 1e-4 * max(1.0, float(b.abs().max()))
