"""Plain float64 CPU oracle for the backward pass of the prefill (training).

TEST INFRASTRUCTURE ONLY, like ``diffattn_ref``: nothing on the product path
imports this module, and it shares no code with the CUDA library.

It differentiates the forward that ``diffattn_ref.diffattn_fwd`` defines --
the DiffAttn equation (page "Differential Transformer: Canceling Context Noise
with Differential Attention", "Cancelling Context Noise Through Attention Map
Subtraction"; peer review "Differential Transformer", Summary, Eq. 1), then
the headwise RMSNorm and the (1 - lambda_init) scale (Eq. 3) -- with respect to
q, k, v, lambda and the RMSNorm weight w, for an upstream gradient dy.  The
lambda re-parameterisation (Eq. 2) is differentiated separately
(``lambda_reparam_bwd``).  The pages train this model (peer review, Summary:
the scaling and long-context training runs), so the path needs its gradients.

Per head, with both maps materialised (no tiling, no recomputation tricks):

    S_i = Q_i K_i^T / sqrt(d) (masked),  A_i = softmax(S_i)
    O = A_1 V + c A_2 V               c = -lambda, 0 or +lambda (the mode)
    r = 1 / sqrt(mean_c O^2 + eps),   y = g w O r,   g = 1 - lambda_init

    dw     = sum over rows of g r O dy
    G = dO = g r (w dy) - O g r^3 / (2d) * sum_c (w dy O)
    dV     = A_1^T G + c A_2^T G
    dA_1   = G V^T,   dA_2 = c G V^T
    dlambda = (dc/dlambda) <G, A_2 V>,  dc/dlambda = -1, 0 or +1
    dS_i   = A_i * (dA_i - rowsum(dA_i * A_i))       (softmax backward)
    dQ_i   = dS_i K_i / sqrt(d),   dK_i = dS_i^T Q_i / sqrt(d)

Pins (tests/test_oracle_bwd.py): torch.autograd on a float64 torch forward,
central finite differences, the lambda = 0 mode leaving map 2 without
gradient, and sum(lambda) = diff(-lambda) with dlambda changing sign.
"""
from __future__ import annotations

import math

import numpy as np

from . import diffattn_ref as ref

__all__ = ["mode_coefficient", "softmax_bwd", "rmsnorm_bwd", "score_grads", "diffattn_bwd", "lambda_reparam_bwd"]


def mode_coefficient(lam: float, mode: str):
    """(c, dc/dlambda) of map 2 in O = A_1 V + c A_2 V for a combination mode."""
    if mode == "diff":
        return -float(lam), -1.0
    if mode == "lambda_zero":
        return 0.0, 0.0
    if mode == "sum":
        return float(lam), 1.0
    raise ValueError(f"mode must be one of {ref.MODES}")


def _masked_softmax(q, k, scale, causal):
    n = q.shape[0]
    S = (q @ k.T) * scale
    if causal:
        S = np.where(np.arange(n)[None, :] > np.arange(n)[:, None], -np.inf, S)
    return ref.softmax_rows(S)


def softmax_bwd(A, dA):
    """dS for A = softmax(S) row-wise: A * (dA - rowsum(dA * A))."""
    return A * (dA - np.sum(dA * A, axis=-1, keepdims=True))


def rmsnorm_bwd(O, dy, w, eps: float, lambda_init: float):
    """(dO, dw) of y = g w O r, r = 1 / sqrt(mean_c O^2 + eps), g = 1 - lambda_init,
    over the last axis (dw summed over the rows)."""
    g = 1.0 - float(lambda_init)
    n = O.shape[-1]
    r = 1.0 / np.sqrt(np.mean(O * O, axis=-1, keepdims=True) + float(eps))
    t = np.sum(w * dy * O, axis=-1, keepdims=True)
    dO = g * r * (w * dy) - O * (g * r ** 3 / n) * t
    return dO, np.sum(g * r * O * dy, axis=0)


def score_grads(dS, q, k, scale: float):
    """(dQ, dK) of S = Q K^T * scale."""
    return dS @ k * scale, dS.T @ q * scale


def diffattn_bwd(q, k, v, dy, lam: float, lambda_init: float, w, eps: float, causal: bool, mode: str = "diff"):
    """Gradients of ``diffattn_ref.diffattn_fwd`` for the upstream gradient dy.

    q, k : [B, N, H, 2, d]; v, dy : [B, N, H, 2d].  Returns
    (dq, dk, dv, dlambda, dw) with the shapes of q, k, v, a float and [2d].
    """
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    dy = np.asarray(dy, dtype=np.float64)
    w = np.asarray(w, dtype=np.float64)
    B, N, H, two, d = q.shape
    scale = 1.0 / math.sqrt(d)
    c, dc = mode_coefficient(lam, mode)
    dq = np.zeros_like(q)
    dk = np.zeros_like(k)
    dvv = np.zeros_like(v)
    dw = np.zeros(2 * d, dtype=np.float64)
    dlam = 0.0
    for b in range(B):
        for h in range(H):
            q1, q2 = q[b, :, h, 0], q[b, :, h, 1]
            k1, k2 = k[b, :, h, 0], k[b, :, h, 1]
            vh, dyh = v[b, :, h], dy[b, :, h]
            A1 = _masked_softmax(q1, k1, scale, causal)
            A2 = _masked_softmax(q2, k2, scale, causal)
            O2 = A2 @ vh
            O = A1 @ vh + c * O2
            G, dw_h = rmsnorm_bwd(O, dyh, w, eps, lambda_init)
            dw += dw_h
            dvv[b, :, h] = A1.T @ G + c * (A2.T @ G)
            dlam += dc * float(np.sum(G * O2))
            dS1 = softmax_bwd(A1, G @ vh.T)
            dS2 = softmax_bwd(A2, c * (G @ vh.T))
            dq[b, :, h, 0], dk[b, :, h, 0] = score_grads(dS1, q1, k1, scale)
            dq[b, :, h, 1], dk[b, :, h, 1] = score_grads(dS2, q2, k2, scale)
    return dq, dk, dvv, dlam, dw


def lambda_reparam_bwd(lq1, lk1, lq2, lk2, dlam: float):
    """Gradients of lambda = exp(lq1 . lk1) - exp(lq2 . lk2) + lambda_init
    (page "Differential Transformer: Canceling Context Noise with Differential
    Attention", the same section as the DiffAttn equation; peer review Eq. 2)."""
    lq1, lk1, lq2, lk2 = (np.asarray(a, dtype=np.float64) for a in (lq1, lk1, lq2, lk2))
    e1 = math.exp(float(np.dot(lq1, lk1)))
    e2 = math.exp(float(np.dot(lq2, lk2)))
    return dlam * e1 * lk1, dlam * e1 * lq1, -dlam * e2 * lk2, -dlam * e2 * lq2
