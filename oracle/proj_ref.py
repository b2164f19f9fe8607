"""Plain float64 CPU oracle for the steps either side of the attention path:
the query/key/value projection with rotary position embedding in front of it,
and the output projection after it.

TEST INFRASTRUCTURE ONLY, like ``diffattn_ref``: nothing on the product path
imports this module, and it shares no code with the CUDA library.

What it computes, and where the pages define it
-----------------------------------------------
* Projections (page "Differential attention", section "How it's wired (and
  why it's nearly free)"): each head's query and key projections are split
  into two halves, Q1, K1 and Q2, K2, and the layer drops into a standard
  transformer block in place of ordinary attention.  With the token
  activations X [M, d_model] and weights stored as a linear layer's, one row
  per output feature:

      [Q | K | V] = X W^T,   W = [W_q; W_k; W_v],   W_q, W_k: [H * 2 * d, d_model],
                                                   W_v: [H * 2d, d_model]

  Q's columns are ordered (head h, map i, channel c), so that Q reshaped to
  [.., H, 2, d] gives Q_i of head h at [.., h, i, :] (and likewise K); V's
  columns are (head h, channel c) for the value width 2d.  The output
  projection maps the heads' concatenated outputs back: Y = O W_o^T with
  W_o: [d_model, H * 2d].
* Rotary position embedding: the pages cite RoFormer (page "Differential
  Transformer", "Builds on") and give no formula.  The reading here is
  RoFormer's rotation of consecutive channel pairs: for a d-wide vector x at
  position n, with theta_j = base^(-2j / d), j = 0 .. d/2 - 1,

      (x'_{2j}, x'_{2j+1}) = (x_{2j} cos(n theta_j) - x_{2j+1} sin(n theta_j),
                              x_{2j} sin(n theta_j) + x_{2j+1} cos(n theta_j))

  applied to each of Q1, Q2, K1, K2 of every head (V is not rotated); the
  position of row m of X is m mod N (rows are [B, N] flattened).

Pins (tests/test_oracle_proj.py): a worked 2-d rotation, the identity at
position 0, norm preservation, RoFormer's relative-position property
(<R_m q, R_n k> depends on m - n only), explicit loops for the projections on
tiny shapes, and planted mistakes that some pin must catch.
"""
from __future__ import annotations

import numpy as np

__all__ = ["rope_angles", "apply_rope", "qkv_proj", "out_proj"]


def rope_angles(positions, d: int, base: float = 10000.0):
    """Angles n * theta_j, float64 [len(positions), d / 2]."""
    if d % 2:
        raise ValueError("d must be even")
    j = np.arange(d // 2, dtype=np.float64)
    theta = float(base) ** (-2.0 * j / d)
    return np.asarray(positions, dtype=np.float64)[:, None] * theta[None, :]


def apply_rope(x, positions, base: float = 10000.0):
    """Rotate consecutive channel pairs of x [..., n, d] by the angles of the
    positions [n] (broadcast over leading axes)."""
    x = np.asarray(x, dtype=np.float64)
    d = x.shape[-1]
    ang = rope_angles(positions, d, base)  # [n, d/2]
    c, s = np.cos(ang), np.sin(ang)
    ev, od = x[..., 0::2], x[..., 1::2]
    out = np.empty_like(x)
    out[..., 0::2] = ev * c - od * s
    out[..., 1::2] = ev * s + od * c
    return out


def qkv_proj(x, w_qkv, B: int, N: int, H: int, d: int, rope_base: float | None = 10000.0):
    """x [B*N, d_model], w_qkv [H*2*d + H*2*d + H*2d, d_model] -> q, k [B, N, H, 2, d],
    v [B, N, H, 2d] (float64); RoPE on q and k unless rope_base is None."""
    x = np.asarray(x, dtype=np.float64)
    w = np.asarray(w_qkv, dtype=np.float64)
    y = x @ w.T
    hq = H * 2 * d
    q = y[:, :hq].reshape(B, N, H, 2, d)
    k = y[:, hq:2 * hq].reshape(B, N, H, 2, d)
    v = y[:, 2 * hq:].reshape(B, N, H, 2 * d)
    if rope_base is not None:
        pos = np.arange(N)
        # rotate along the token axis: move it next to the channels
        q = np.moveaxis(apply_rope(np.moveaxis(q, 1, -2), pos, rope_base), -2, 1)
        k = np.moveaxis(apply_rope(np.moveaxis(k, 1, -2), pos, rope_base), -2, 1)
    return q, k, v


def out_proj(o, w_o):
    """o [M, H*2d], w_o [d_model, H*2d] -> o W_o^T [M, d_model] (float64)."""
    return np.asarray(o, dtype=np.float64) @ np.asarray(w_o, dtype=np.float64).T
