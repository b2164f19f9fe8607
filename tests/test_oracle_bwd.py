"""Pins for the float64 backward oracle (no GPU).

The hand-derived gradients are pinned to torch.autograd on an independent
float64 torch forward (a library routine does the differentiation), to
central finite differences, and to two structural facts of the control modes.
The mutation test plants plausible mistakes on the CPU and checks that some
pin fails for each.
"""
import math

import numpy as np
import pytest
import torch

import oracle.bwd_ref as bwd
import oracle.diffattn_ref as ref


def _case(seed, B=1, N=7, H=2, d=4, scale=1.0):
    rng = np.random.default_rng(seed)
    q = rng.standard_normal((B, N, H, 2, d)) * scale
    k = rng.standard_normal((B, N, H, 2, d)) * scale
    v = rng.standard_normal((B, N, H, 2 * d))
    dy = rng.standard_normal((B, N, H, 2 * d))
    w = 1 + 0.2 * rng.standard_normal(2 * d)
    return q, k, v, dy, w


def _torch_grads(q, k, v, dy, lam, lambda_init, w, eps, causal, mode):
    t = lambda a: torch.tensor(a, dtype=torch.float64, requires_grad=True)
    qt, kt, vt, wt, lt = t(q), t(k), t(v), t(w), t(lam)
    d = q.shape[-1]
    n = q.shape[1]
    s1 = torch.einsum("bnhd,bmhd->bhnm", qt[..., 0, :], kt[..., 0, :]) / math.sqrt(d)
    s2 = torch.einsum("bnhd,bmhd->bhnm", qt[..., 1, :], kt[..., 1, :]) / math.sqrt(d)
    if causal:
        mask = torch.triu(torch.ones(n, n, dtype=torch.bool), 1)
        s1 = s1.masked_fill(mask, float("-inf"))
        s2 = s2.masked_fill(mask, float("-inf"))
    a1, a2 = torch.softmax(s1, -1), torch.softmax(s2, -1)
    c = {"diff": -lt, "lambda_zero": 0 * lt, "sum": lt}[mode]
    o = torch.einsum("bhnm,bmhc->bnhc", a1 + c * a2, vt)
    y = (1 - lambda_init) * wt * o / torch.sqrt(torch.mean(o * o, -1, keepdim=True) + eps)
    y.backward(torch.tensor(dy, dtype=torch.float64))
    return qt.grad.numpy(), kt.grad.numpy(), vt.grad.numpy(), float(lt.grad), wt.grad.numpy()


def _close(a, b, tol=1e-10):
    a, b = np.asarray(a, dtype=np.float64), np.asarray(b, dtype=np.float64)
    return np.max(np.abs(a - b)) <= tol * max(1.0, float(np.max(np.abs(b))))


def pin_autograd():
    for seed, causal, mode, lam in [(1, True, "diff", 0.4), (2, False, "diff", -0.3), (3, True, "sum", 0.7),
                                    (4, False, "lambda_zero", 0.5)]:
        q, k, v, dy, w = _case(seed)
        got = bwd.diffattn_bwd(q, k, v, dy, lam, 0.3, w, 1e-5, causal, mode)
        want = _torch_grads(q, k, v, dy, lam, 0.3, w, 1e-5, causal, mode)
        for name, g, t in zip(("dq", "dk", "dv", "dlam", "dw"), got, want):
            assert _close(g, t), (seed, name)


def pin_finite_differences():
    q, k, v, dy, w = _case(5, N=5, H=1, d=3)
    lam, li, eps = 0.35, 0.2, 1e-5
    base = dict(q=q, k=k, v=v, w=w)
    loss = lambda a, lam_=lam: float(np.sum(ref.diffattn_fwd(a["q"], a["k"], a["v"], lam_, li, a["w"], eps, True) * dy))
    dq, dk, dv, dlam, dw = bwd.diffattn_bwd(q, k, v, dy, lam, li, w, eps, True)
    grads = dict(q=dq, k=dk, v=dv, w=dw)
    h = 1e-6
    rng = np.random.default_rng(0)
    for name in ("q", "k", "v", "w"):
        for _ in range(4):
            idx = tuple(int(rng.integers(0, n)) for n in base[name].shape)
            plus, minus = dict(base), dict(base)
            plus[name] = base[name].copy()
            minus[name] = base[name].copy()
            plus[name][idx] += h
            minus[name][idx] -= h
            fd = (loss(plus) - loss(minus)) / (2 * h)
            assert abs(fd - grads[name][idx]) <= 1e-6 * max(1.0, abs(fd)), (name, idx, fd, grads[name][idx])
    fd = (loss(base, lam + h) - loss(base, lam - h)) / (2 * h)
    assert abs(fd - dlam) <= 1e-6 * max(1.0, abs(fd))


def pin_lambda_zero_leaves_map2():
    q, k, v, dy, w = _case(6)
    dq, dk, dv, dlam, dw = bwd.diffattn_bwd(q, k, v, dy, 0.9, 0.3, w, 1e-5, True, "lambda_zero")
    assert np.all(dq[..., 1, :] == 0) and np.all(dk[..., 1, :] == 0) and dlam == 0.0
    assert np.any(dq[..., 0, :] != 0)


def pin_sum_is_diff_of_negated_lambda():
    q, k, v, dy, w = _case(7)
    s = bwd.diffattn_bwd(q, k, v, dy, 0.45, 0.3, w, 1e-5, True, "sum")
    dd = bwd.diffattn_bwd(q, k, v, dy, -0.45, 0.3, w, 1e-5, True, "diff")
    for a, b in zip(s[:3] + s[4:], dd[:3] + dd[4:]):
        assert _close(a, b, 1e-13)
    assert abs(s[3] + dd[3]) <= 1e-12 * max(1.0, abs(s[3]))


def pin_lambda_reparam_bwd():
    rng = np.random.default_rng(8)
    vecs = [0.3 * rng.standard_normal(6) for _ in range(4)]
    dlam = 1.7
    got = bwd.lambda_reparam_bwd(*vecs, dlam)
    h = 1e-7
    for i in range(4):
        for j in range(6):
            p = [a.copy() for a in vecs]
            m = [a.copy() for a in vecs]
            p[i][j] += h
            m[i][j] -= h
            fd = dlam * (ref.lambda_reparam(*p, 0.1) - ref.lambda_reparam(*m, 0.1)) / (2 * h)
            assert abs(fd - got[i][j]) <= 1e-6 * max(1.0, abs(fd))


PINS = [pin_autograd, pin_finite_differences, pin_lambda_zero_leaves_map2, pin_sum_is_diff_of_negated_lambda,
        pin_lambda_reparam_bwd]


@pytest.mark.parametrize("pin", PINS, ids=[p.__name__ for p in PINS])
def test_pin(pin):
    pin()


# ------------------------------------------------------------ mutations ----

_orig_bwd = bwd.diffattn_bwd
_orig_softmax_bwd = bwd.softmax_bwd
_orig_rms_bwd = bwd.rmsnorm_bwd


def _mut_softmax_no_rowsum(A, dA):
    return A * dA


def _mut_softmax_rowsum_of_dA(A, dA):
    return A * (dA - np.sum(dA, axis=-1, keepdims=True))


def _mut_dlam_sign(*a, **kw):
    dq, dk, dv, dlam, dw = _orig_bwd(*a, **kw)
    return dq, dk, dv, -dlam, dw


def _mut_norm_diagonal_only(O, dy, w, eps, lambda_init):
    g = 1.0 - float(lambda_init)
    r = 1.0 / np.sqrt(np.mean(O * O, axis=-1, keepdims=True) + float(eps))
    return g * r * (w * dy), np.sum(g * r * O * dy, axis=0)


def _mut_norm_without_g_in_dw(O, dy, w, eps, lambda_init):
    dO, dw = _orig_rms_bwd(O, dy, w, eps, lambda_init)
    return dO, dw / (1.0 - float(lambda_init))


def _mut_dk_not_transposed(dS, q, k, scale):
    return dS @ k * scale, dS @ q * scale


def _mut_reparam_swap(lq1, lk1, lq2, lk2, dlam):
    e1 = math.exp(float(np.dot(lq1, lk1)))
    e2 = math.exp(float(np.dot(lq2, lk2)))
    return dlam * e1 * lq1, dlam * e1 * lk1, -dlam * e2 * lk2, -dlam * e2 * lq2


MUTANTS = {
    "softmax_bwd_without_row_sum": ("softmax_bwd", _mut_softmax_no_rowsum),
    "softmax_bwd_row_sum_of_dA_only": ("softmax_bwd", _mut_softmax_rowsum_of_dA),
    "dlambda_sign": ("diffattn_bwd", _mut_dlam_sign),
    "norm_jacobian_diagonal_only": ("rmsnorm_bwd", _mut_norm_diagonal_only),
    "dw_without_scale": ("rmsnorm_bwd", _mut_norm_without_g_in_dw),
    "dk_not_transposed": ("score_grads", _mut_dk_not_transposed),
    "reparam_grads_swapped": ("lambda_reparam_bwd", _mut_reparam_swap),
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_pins_catch_mutant(name, monkeypatch):
    attr, fn = MUTANTS[name]
    monkeypatch.setattr(bwd, attr, fn)
    caught = []
    for pin in PINS:
        try:
            with np.errstate(all="ignore"):
                pin()
        except (AssertionError, FloatingPointError, ValueError):
            caught.append(pin.__name__)
    assert caught, f"no pin catches mutant {name}"


from hypothesis import given, settings  # noqa: E402
from hypothesis import strategies as st  # noqa: E402


@settings(max_examples=30, deadline=None)
@given(B=st.integers(1, 2), N=st.integers(1, 6), H=st.integers(1, 2), d=st.integers(1, 4), causal=st.booleans(),
       mode=st.sampled_from(["diff", "lambda_zero", "sum"]), lam=st.floats(-1.5, 1.5),
       lam_init=st.floats(0.0, 0.9), eps=st.sampled_from([1e-5, 0.1]), scale=st.sampled_from([0.3, 1.0, 3.0]),
       seed=st.integers(0, 2 ** 31 - 1))
def test_autograd_on_random_shapes(B, N, H, d, causal, mode, lam, lam_init, eps, scale, seed):
    # pin_autograd over drawn shapes (one token and one channel included), masks, modes and lambda
    q, k, v, dy, w = _case(seed, B=B, N=N, H=H, d=d, scale=scale)
    got = bwd.diffattn_bwd(q, k, v, dy, lam, lam_init, w, eps, causal, mode)
    want = _torch_grads(q, k, v, dy, lam, lam_init, w, eps, causal, mode)
    for name, g, t in zip(("dq", "dk", "dv", "dlam", "dw"), got, want):
        assert _close(g, t, tol=1e-8), name
