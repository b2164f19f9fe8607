"""Property tests of the float64 oracle against pure-Python loops (no GPU).

The brute-force pin in test_oracle.py fixes one shape and one lambda; here
hypothesis draws the shapes (including a single token and a single channel),
the mask, lambda over both signs and beyond 1, lambda_init, eps, the
combination mode and the scale of the inputs, and every draw must agree with
loops that restate the method directly: two softmax maps per head (the DiffAttn
equation of page "Differential Transformer: Canceling Context Noise with
Differential Attention", section "Cancelling Context Noise Through Attention
Map Subtraction"), combined with coefficient -lambda, 0 or +lambda (the peer
review's controls), then RMSNorm over the head's 2d channels with eps inside
the root and the (1 - lambda_init) scale (peer review, Eq. 3).  The decode
test does the same for one query per sequence over a packed cache of random
lengths, each query seeing its whole sequence.
"""
import math

import numpy as np
from hypothesis import given, settings
from hypothesis import strategies as st

import oracle.diffattn_ref as ref

COEF = {"diff": -1.0, "lambda_zero": 0.0, "sum": 1.0}


def _loops(q, k, v, lam, lam_init, w, eps, causal, mode, shape):
    B, N, H, d = shape
    out = [[[None] * H for _ in range(N)] for _ in range(B)]
    c = COEF[mode] * lam
    for b in range(B):
        for h in range(H):
            for i in range(N):
                keys = [j for j in range(N) if not causal or j <= i]
                maps = []
                for m in (0, 1):
                    s = [sum(q[b][i][h][m][t] * k[b][j][h][m][t] for t in range(d)) / math.sqrt(d) for j in keys]
                    top = max(s)
                    e = [math.exp(x - top) for x in s]
                    z = sum(e)
                    maps.append([x / z for x in e])
                wts = [a + c * bb for a, bb in zip(maps[0], maps[1])]
                o = [sum(wts[n] * v[b][j][h][ch] for n, j in enumerate(keys)) for ch in range(2 * d)]
                ms = sum(x * x for x in o) / (2 * d)
                if ms + eps == 0.0:  # a head output of exact zeros with eps = 0: 0 / 0
                    out[b][i][h] = [math.nan] * (2 * d)
                else:
                    out[b][i][h] = [(1 - lam_init) * w[ch] * o[ch] / math.sqrt(ms + eps) for ch in range(2 * d)]
    return out


@settings(max_examples=60, deadline=None)
@given(B=st.integers(1, 2), N=st.integers(1, 6), H=st.integers(1, 2), d=st.integers(1, 4),
       causal=st.booleans(), mode=st.sampled_from(sorted(COEF)),
       lam=st.floats(-1.5, 1.5), lam_init=st.floats(0.0, 0.9), eps=st.sampled_from([0.0, 1e-5, 0.5]),
       scale=st.sampled_from([0.1, 1.0, 8.0]), seed=st.integers(0, 2 ** 31 - 1))
def test_oracle_matches_loops(B, N, H, d, causal, mode, lam, lam_init, eps, scale, seed):
    rng = np.random.default_rng(seed)
    q = rng.standard_normal((B, N, H, 2, d)) * scale
    k = rng.standard_normal((B, N, H, 2, d)) * scale
    v = rng.standard_normal((B, N, H, 2 * d))
    w = 1 + 0.1 * rng.standard_normal(2 * d)
    with np.errstate(invalid="ignore"):
        y = ref.diffattn_fwd(q, k, v, lam, lam_init, w, eps, causal, mode=mode)
    want = np.array(_loops(q.tolist(), k.tolist(), v.tolist(), lam, lam_init, w.tolist(), eps, causal, mode,
                           (B, N, H, d)))
    # the loops and numpy sum in different orders; the outputs are normalised (of order one), so an
    # absolute bound far above float64 rounding and far below any formula error fits every draw
    np.testing.assert_allclose(y, want, rtol=1e-9, atol=1e-9, equal_nan=True)


def _decode_loops(q, kc, vc, cu, lam, lam_init, w, eps, mode, S, H, d):
    c = COEF[mode] * lam
    out = []
    for s in range(S):
        row = []
        for h in range(H):
            keys = range(cu[s], cu[s + 1])  # the sequence's whole cache, its own token included
            maps = []
            for m in (0, 1):
                sc = [sum(q[s][h][m][t] * kc[j][h][m][t] for t in range(d)) / math.sqrt(d) for j in keys]
                top = max(sc)
                e = [math.exp(x - top) for x in sc]
                z = sum(e)
                maps.append([x / z for x in e])
            wts = [a + c * b for a, b in zip(maps[0], maps[1])]
            o = [sum(wts[n] * vc[j][h][ch] for n, j in enumerate(keys)) for ch in range(2 * d)]
            ms = sum(x * x for x in o) / (2 * d)
            row.append([math.nan] * (2 * d) if ms + eps == 0.0 else
                       [(1 - lam_init) * w[ch] * o[ch] / math.sqrt(ms + eps) for ch in range(2 * d)])
        out.append(row)
    return out


@settings(max_examples=40, deadline=None)
@given(lens=st.lists(st.integers(1, 6), min_size=1, max_size=4), H=st.integers(1, 2), d=st.integers(1, 4),
       mode=st.sampled_from(sorted(COEF)), lam=st.floats(-1.5, 1.5), lam_init=st.floats(0.0, 0.9),
       eps=st.sampled_from([0.0, 1e-5]), seed=st.integers(0, 2 ** 31 - 1))
def test_decode_oracle_matches_loops(lens, H, d, mode, lam, lam_init, eps, seed):
    rng = np.random.default_rng(seed)
    S = len(lens)
    cu = [0]
    for n in lens:
        cu.append(cu[-1] + n)
    T = cu[-1]
    q = rng.standard_normal((S, H, 2, d))
    kc = rng.standard_normal((T, H, 2, d))
    vc = rng.standard_normal((T, H, 2 * d))
    w = 1 + 0.1 * rng.standard_normal(2 * d)
    with np.errstate(invalid="ignore"):
        y = ref.diffattn_decode(q, kc, vc, cu, lam, lam_init, w, eps, mode=mode)
    want = np.array(_decode_loops(q.tolist(), kc.tolist(), vc.tolist(), cu, lam, lam_init, w.tolist(), eps, mode,
                                  S, H, d))
    np.testing.assert_allclose(y, want, rtol=1e-9, atol=1e-9, equal_nan=True)
