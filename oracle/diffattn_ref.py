"""Plain float64 CPU oracle for the differential-attention forward.

TEST INFRASTRUCTURE ONLY.  Nothing on the product path imports this module:
only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline /
reference arm may call it.  It shares no code with the CUDA library.

What it computes, and where the pages define it
-----------------------------------------------
* DiffAttn for one head (page "Differential Transformer: Canceling Context
  Noise with Differential Attention", section "Cancelling Context Noise Through
  Attention Map Subtraction", the DiffAttn equation; the same equation on page
  "Differential attention", section "The noise-canceling idea"; Eq. 1 in the
  peer review "Differential Transformer", Summary):

      DiffAttn = (softmax(Q1 K1^T / sqrt(d)) - lambda * softmax(Q2 K2^T / sqrt(d))) V

* The lambda re-parameterisation (same section of the first page; Eq. 2 of the
  peer review's Summary):

      lambda = exp(lq1 . lk1) - exp(lq2 . lk2) + lambda_init

* Headwise normalisation, then the fixed (1 - lambda_init) scale (peer review
  "Differential Transformer", Summary, Eq. 3).  The pages name
  "GroupNorm/RMSNorm"; this oracle uses RMSNorm over the 2d channels of each
  (token, head): y = (1 - lambda_init) * w * o / sqrt(mean(o^2) + eps).
* The row max is subtracted before exponentiating (the softmax in the worked
  example on page "Differential attention", "The noise-canceling idea").

Readings where the pages are silent:
  d in sqrt(d) is the per-map query/key width; eps sits inside the square
  root; w is one fp32 vector of length 2d shared by all heads; the scale uses
  lambda_init (not the learned lambda) and is applied after w; causal means key
  j is visible to query i iff j <= i (prefill, equal query/key lengths); a
  decode query sees every cached key of its sequence.

Every function materialises both softmax maps explicitly; there is no tiling,
fusion or reordering beyond what the definitions state.  Inputs are upcast to
float64 (for bf16 inputs: the exact bf16 values the GPU receives).

Layouts (the same as the library's):
  prefill  q, k : [B, N, H, 2, d]   (Q1 = q[..., 0, :], Q2 = q[..., 1, :])
           v    : [B, N, H, 2d]     -> y : [B, N, H, 2d]
  decode   q    : [S, H, 2, d]; k_cache : [T, H, 2, d]; v_cache : [T, H, 2d]
           cu_seqlens : int[S + 1], sequence s owns cache rows
           cu_seqlens[s] .. cu_seqlens[s+1]-1 (its own token included)
           -> y : [S, H, 2d]

Pins (tests/test_oracle.py): the pages' six-key worked example, the row-sum
invariant 1 - lambda, lambda = 0 against torch's scaled_dot_product_attention
(a library routine), map 2 alone against the same routine, Q2=Q1/K2=K1 giving
(1 - lambda) times single-map attention, the single visible key of causal row
0, hand-computed RMSNorm and lambda values, brute-force loops on tiny shapes,
decode == last prefill row, and for the two control modes (lambda = 0:
one map; "+lambda": the maps added) torch's attention per map.
"""
from __future__ import annotations

import math

import numpy as np

__all__ = [
    "lambda_reparam",
    "MODES",
    "map_weights",
    "softmax_rows",
    "diff_weights",
    "diffattn_head_prenorm",
    "headwise_rmsnorm",
    "diffattn_fwd",
    "decode_head_prenorm",
    "diffattn_decode",
]


def lambda_reparam(lq1, lk1, lq2, lk2, lambda_init: float) -> float:
    """lambda = exp(lq1 . lk1) - exp(lq2 . lk2) + lambda_init.

    Page "Differential Transformer: Canceling Context Noise with Differential
    Attention", section "Cancelling Context Noise Through Attention Map
    Subtraction" (the re-parameterisation); peer review "Differential
    Transformer", Summary, Eq. 2.  One scalar per call, shared by every head.
    """
    lq1 = np.asarray(lq1, dtype=np.float64)
    lk1 = np.asarray(lk1, dtype=np.float64)
    lq2 = np.asarray(lq2, dtype=np.float64)
    lk2 = np.asarray(lk2, dtype=np.float64)
    return float(np.exp(np.dot(lq1, lk1)) - np.exp(np.dot(lq2, lk2)) + float(lambda_init))


def softmax_rows(S: np.ndarray) -> np.ndarray:
    """Row-wise softmax with the row max subtracted first.

    The softmax of the worked example on page "Differential attention",
    section "The noise-canceling idea".  Entries equal to -inf (masked keys)
    get weight exactly 0.  Every row must have at least one finite entry.
    """
    S = np.asarray(S, dtype=np.float64)
    m = S.max(axis=-1, keepdims=True)
    E = np.exp(S - m)
    return E / E.sum(axis=-1, keepdims=True)


def diff_weights(S1: np.ndarray, S2: np.ndarray, lam: float) -> np.ndarray:
    """The differential map softmax(S1) - lambda * softmax(S2).

    DiffAttn equation, page "Differential attention", "The noise-canceling
    idea" (the ``diff`` line of its worked example).  Each row sums to
    1 - lambda and may hold negative entries (peer review "Differential
    Transformer", Weaknesses, first bullet).
    """
    return softmax_rows(S1) - float(lam) * softmax_rows(S2)


# Combination of the two maps, D = softmax(S1) + c * softmax(S2):
#   "diff"        c = -lambda : the DiffAttn equation (the method itself)
#   "lambda_zero" c = 0       : the peer review's lambda = 0 control (Questions,
#                               first bullet; Weaknesses, second bullet): the same
#                               architecture with a single softmax map
#   "sum"         c = +lambda : the review's "+lambda" control, two maps added
#                               rather than subtracted (same bullets)
MODES = ("diff", "lambda_zero", "sum")


def map_weights(S1: np.ndarray, S2: np.ndarray, lam: float, mode: str = "diff") -> np.ndarray:
    """softmax(S1) + c * softmax(S2) with c given by ``mode`` (see MODES).

    "lambda_zero" uses softmax(S1) alone (S2 is not looked at).
    """
    if mode == "diff":
        return diff_weights(S1, S2, lam)
    if mode == "lambda_zero":
        return softmax_rows(S1)
    if mode == "sum":
        return softmax_rows(S1) + float(lam) * softmax_rows(S2)
    raise ValueError(f"mode must be one of {MODES}")


def _causal_scores(q: np.ndarray, k: np.ndarray, scale: float, q_pos, causal: bool) -> np.ndarray:
    """Scores q k^T * scale for the query positions ``q_pos`` against all keys.

    With ``causal`` the key j is hidden (-inf) from the query at position i
    when j > i.
    """
    S = (q @ k.T) * scale
    if causal:
        j = np.arange(k.shape[0])[None, :]
        i = np.asarray(q_pos)[:, None]
        S = np.where(j > i, -np.inf, S)
    return S


def diffattn_head_prenorm(q1, k1, q2, k2, v, lam: float, causal: bool, rows=None, mode: str = "diff") -> np.ndarray:
    """DiffAttn for one head, before the headwise norm.

    q1, q2 : [N, d]   k1, k2 : [N, d]   v : [N, 2d]   ->   O : [len(rows), 2d]

    ``rows`` (default: all N) selects the query positions whose output rows are
    computed; each selected row is still computed against every key, so a
    sampled row equals the corresponding row of the full result.
    DiffAttn equation (page "Differential Transformer: Canceling Context Noise
    with Differential Attention", "Cancelling Context Noise Through Attention
    Map Subtraction"; peer review Eq. 1), with d = the per-map width (the
    peer review's lambda=0 control: query/key width d = 128, value width 2d).
    ``mode`` selects the combination of the two maps (see MODES).
    """
    q1 = np.asarray(q1, dtype=np.float64)
    q2 = np.asarray(q2, dtype=np.float64)
    k1 = np.asarray(k1, dtype=np.float64)
    k2 = np.asarray(k2, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    n, d = q1.shape
    if rows is None:
        rows = np.arange(n)
    rows = np.asarray(rows)
    scale = 1.0 / math.sqrt(d)
    S1 = _causal_scores(q1[rows], k1, scale, rows, causal)
    S2 = _causal_scores(q2[rows], k2, scale, rows, causal)
    D = map_weights(S1, S2, lam, mode)
    return D @ v


def headwise_rmsnorm(O: np.ndarray, w, eps: float, lambda_init: float) -> np.ndarray:
    """(1 - lambda_init) * w * O / sqrt(mean(O^2) + eps) over the last axis.

    Peer review "Differential Transformer", Summary, Eq. 3: each head's output
    is normalised on its own, then multiplied by the fixed (1 - lambda_init).
    RMSNorm (no mean subtraction), eps inside the square root, w applied per
    channel before the scale.
    """
    O = np.asarray(O, dtype=np.float64)
    w = np.asarray(w, dtype=np.float64)
    ms = np.mean(O * O, axis=-1, keepdims=True)
    return (1.0 - float(lambda_init)) * w * O / np.sqrt(ms + float(eps))


def diffattn_fwd(q, k, v, lam: float, lambda_init: float, w, eps: float, causal: bool,
                 rows=None, heads=None, mode: str = "diff") -> np.ndarray:
    """Prefill: normalised DiffAttn output for every (batch, head).

    q, k : [B, N, H, 2, d]; v : [B, N, H, 2d].  Returns y : [B, R, H, 2d] where
    R = N, or the query positions in ``rows``.  ``heads`` (optional) is a list
    of (b, h) pairs to compute; the others are left as NaN.  ``mode`` selects
    the combination of the two maps (see MODES).
    """
    q = np.asarray(q)
    k = np.asarray(k)
    v = np.asarray(v)
    B, N, H, two, d = q.shape
    assert two == 2 and k.shape == q.shape and v.shape == (B, N, H, 2 * d)
    R = N if rows is None else len(rows)
    y = np.full((B, R, H, 2 * d), np.nan, dtype=np.float64)
    pairs = [(b, h) for b in range(B) for h in range(H)] if heads is None else heads
    for b, h in pairs:
        O = diffattn_head_prenorm(q[b, :, h, 0, :], k[b, :, h, 0, :],
                                  q[b, :, h, 1, :], k[b, :, h, 1, :],
                                  v[b, :, h, :], lam, causal, rows, mode)
        y[b, :, h, :] = headwise_rmsnorm(O, w, eps, lambda_init)
    return y


def decode_head_prenorm(q1, q2, k1, k2, v, lam: float, mode: str = "diff") -> np.ndarray:
    """DiffAttn for one query (length-1 decode) against L cached keys.

    q1, q2 : [d]; k1, k2 : [L, d]; v : [L, 2d]  ->  O : [2d].  The query sees
    all L keys (its own included), so no mask applies.  ``mode`` selects the
    combination of the two maps (see MODES).
    """
    q1 = np.asarray(q1, dtype=np.float64)[None, :]
    q2 = np.asarray(q2, dtype=np.float64)[None, :]
    k1 = np.asarray(k1, dtype=np.float64)
    k2 = np.asarray(k2, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    scale = 1.0 / math.sqrt(q1.shape[1])
    D = map_weights((q1 @ k1.T) * scale, (q2 @ k2.T) * scale, lam, mode)
    return (D @ v)[0]


def diffattn_decode(q, k_cache, v_cache, cu_seqlens, lam: float, lambda_init: float, w,
                    eps: float, pairs=None, mode: str = "diff") -> np.ndarray:
    """Decode over a packed KV cache: normalised output per (sequence, head).

    q : [S, H, 2, d]; k_cache : [T, H, 2, d]; v_cache : [T, H, 2d];
    cu_seqlens : [S + 1].  Returns y : [S, H, 2d]; with ``pairs`` (a list of
    (s, h)) only those rows are computed and the rest are NaN.
    """
    q = np.asarray(q)
    S, H, two, d = q.shape
    cu = np.asarray(cu_seqlens, dtype=np.int64)
    y = np.full((S, H, 2 * d), np.nan, dtype=np.float64)
    todo = [(s, h) for s in range(S) for h in range(H)] if pairs is None else pairs
    for s, h in todo:
        lo, hi = int(cu[s]), int(cu[s + 1])
        kc = np.asarray(k_cache[lo:hi, h], dtype=np.float64)
        vc = np.asarray(v_cache[lo:hi, h], dtype=np.float64)
        O = decode_head_prenorm(q[s, h, 0], q[s, h, 1], kc[:, 0], kc[:, 1], vc, lam, mode)
        y[s, h] = headwise_rmsnorm(O, w, eps, lambda_init)
    return y
