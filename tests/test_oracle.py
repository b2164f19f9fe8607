"""Pins for the float64 CPU oracle (no GPU).

Each pin ties the oracle to something other than itself: the printed worked
example of page "Differential attention" ("The noise-canceling idea"), the
row-sum invariant of the peer review "Differential Transformer" (Weaknesses,
first bullet), torch's scaled_dot_product_attention (a library routine) for
the cases that reduce to ordinary attention, hand-computed closed forms, and
brute-force loops on tiny shapes.  The mutation test at the end plants
plausible mistakes in the oracle (on the CPU) and checks that some pin fails
for each of them.
"""
import math
import os

import numpy as np
import pytest
import torch
import torch.nn.functional as F

import oracle.diffattn_ref as ref

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "worked_example.txt")


def _load_golden(path=GOLDEN):
    vals = {}
    with open(path) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            key, rhs = [t.strip() for t in line.split("=", 1)]
            nums = [float(t) for t in rhs.split()]
            vals[key] = nums if len(nums) > 1 else nums[0]
    return vals


def _sdpa(q, k, v, causal):
    """torch's attention on float64 CPU tensors: softmax(q k^T / sqrt(width)) v."""
    t = lambda a: torch.from_numpy(np.ascontiguousarray(a, dtype=np.float64))[None, None]
    return F.scaled_dot_product_attention(t(q), t(k), t(v), is_causal=causal)[0, 0].numpy()


def _rand_head(rng, n, d):
    q1, k1, q2, k2 = (rng.standard_normal((n, d)) for _ in range(4))
    v = rng.standard_normal((n, 2 * d))
    return q1, k1, q2, k2, v


# ----------------------------------------------------------------- pins ----

def pin_worked_example():
    g = _load_golden()
    tol = g["tolerance"]
    s1 = np.array(g["s1"])[None, :]
    s2 = np.array(g["s2"])[None, :]
    irr = [int(i) for i in g["irrelevant"]]
    a1 = ref.softmax_rows(s1)[0]
    assert np.allclose(a1, g["softmax_s1"], atol=tol, rtol=0)
    assert abs(a1[irr].sum() - g["softmax_irrelevant_sum"]) <= tol
    diff = ref.diff_weights(s1, s2, g["lambda"])[0]
    assert np.allclose(diff, g["diff"], atol=tol, rtol=0)
    assert abs(diff[irr].sum() - g["diff_irrelevant_sum"]) <= tol
    # The same example through the decode path: d = 1 (so 1/sqrt(d) = 1),
    # query 1, keys = the scores; value column 0 marks the relevant key and
    # column 1 the irrelevant ones, so O = [diff[1], sum of diff on irrelevant].
    n = len(g["s1"])
    v = np.zeros((n, 2))
    v[1, 0] = 1.0
    v[irr, 1] = 1.0
    O = ref.decode_head_prenorm([1.0], [1.0], np.array(g["s1"])[:, None],
                                np.array(g["s2"])[:, None], v, g["lambda"])
    assert abs(O[0] - g["diff"][1]) <= tol
    assert abs(O[1] - g["diff_irrelevant_sum"]) <= tol


def pin_large_scores():
    # softmax is shift-invariant: scores near 1000 (exp would overflow) give
    # the same weights as scores near 0: [1, 3] / 4 for a gap of ln 3.
    a = ref.softmax_rows(np.array([[1000.0, 1000.0 + math.log(3.0)]]))
    assert np.allclose(a, [[0.25, 0.75]], atol=1e-15)


def pin_row_sums():
    rng = np.random.default_rng(1)
    for lam in (0.5, -0.7, 1.3, 0.0):
        S1 = rng.standard_normal((9, 13)) * 3
        S2 = rng.standard_normal((9, 13)) * 3
        D = ref.diff_weights(S1, S2, lam)
        assert np.allclose(D.sum(axis=1), 1.0 - lam, atol=1e-12)
        # through the full head: V of ones gives (1 - lambda) in every channel
        for causal in (False, True):
            q1, k1, q2, k2, _ = _rand_head(rng, 11, 4)
            O = ref.diffattn_head_prenorm(q1, k1, q2, k2, np.ones((11, 8)), lam, causal)
            assert np.allclose(O, 1.0 - lam, atol=1e-12)


def pin_lambda_zero_is_attention():
    rng = np.random.default_rng(2)
    for causal in (False, True):
        q1, k1, q2, k2, v = _rand_head(rng, 37, 8)
        O = ref.diffattn_head_prenorm(q1, k1, q2, k2, v, 0.0, causal)
        assert np.allclose(O, _sdpa(q1, k1, v, causal), atol=1e-12)


def pin_map2_alone():
    # Q1 = K1 = 0 makes map 1 uniform over the visible keys, which is what
    # the library routine gives for all-zero queries and keys.
    rng = np.random.default_rng(3)
    for causal in (False, True):
        _, _, q2, k2, v = _rand_head(rng, 29, 8)
        z = np.zeros_like(q2)
        lam = 0.37
        O = ref.diffattn_head_prenorm(z, z, q2, k2, v, lam, causal)
        want = _sdpa(z, z, v, causal) - lam * _sdpa(q2, k2, v, causal)
        assert np.allclose(O, want, atol=1e-12)


def pin_equal_maps():
    rng = np.random.default_rng(4)
    for causal in (False, True):
        q1, k1, _, _, v = _rand_head(rng, 23, 8)
        lam = 0.8
        O = ref.diffattn_head_prenorm(q1, k1, q1, k1, v, lam, causal)
        assert np.allclose(O, (1 - lam) * _sdpa(q1, k1, v, causal), atol=1e-12)


def pin_causal_row0():
    rng = np.random.default_rng(5)
    q1, k1, q2, k2, v = _rand_head(rng, 16, 8)
    lam = 0.6
    O = ref.diffattn_head_prenorm(q1, k1, q2, k2, v, lam, True)
    assert np.allclose(O[0], (1 - lam) * v[0], atol=1e-12)
    # after the norm (eps = 0): (1 - lambda_init) * w * v0 / rms(v0), the sign of 1 - lambda kept
    w = rng.standard_normal(16)
    y = ref.headwise_rmsnorm(O[:1], w, 0.0, 0.2)[0]
    rms_v0 = math.sqrt(sum(x * x for x in v[0]) / 16)
    assert np.allclose(y, 0.8 * w * v[0] / rms_v0, atol=1e-12)


def pin_rmsnorm_hand():
    w = np.array([1.0, 2.0, 3.0, 4.0])
    o = np.array([[1.0, -1.0, 1.0, -1.0]])          # mean square 1
    assert np.allclose(ref.headwise_rmsnorm(o, w, 0.0, 0.25), [[0.75, -1.5, 2.25, -3.0]], atol=1e-15)
    # eps = 3 sits inside the root: sqrt(1 + 3) = 2
    assert np.allclose(ref.headwise_rmsnorm(o, w, 3.0, 0.25), [[0.375, -0.75, 1.125, -1.5]], atol=1e-15)
    o2 = np.array([[3.0, 4.0, 0.0, 0.0]])           # mean square 25/4, rms 2.5
    assert np.allclose(ref.headwise_rmsnorm(o2, w, 0.0, 0.5), [[0.6, 1.6, 0.0, 0.0]], atol=1e-15)


def pin_lambda_hand():
    # exp(0.5) - exp(0.2) + 0.3 = 1.6487212707 - 1.2214027582 + 0.3
    lam = ref.lambda_reparam([1, 0, 0], [0.5, 7, 0], [0, 2, 0], [0, 0.1, 9], 0.3)
    assert abs(lam - 0.7273185125) < 1e-9
    z = np.zeros(64)
    assert ref.lambda_reparam(z, z, z, z, 0.65) == pytest.approx(0.65, abs=1e-15)


def _brute_head(q1, k1, q2, k2, v, lam, causal):
    """Pure-Python loops (no numpy) over one head, before the norm."""
    n, d = len(q1), len(q1[0])
    out = []
    for i in range(n):
        keys = [j for j in range(n) if (not causal or j <= i)]
        rows = []
        for q, k in ((q1, k1), (q2, k2)):
            s = [sum(q[i][c] * k[j][c] for c in range(d)) / math.sqrt(d) for j in keys]
            mx = max(s)
            e = [math.exp(x - mx) for x in s]
            tot = sum(e)
            rows.append([x / tot for x in e])
        wts = [a - lam * b for a, b in zip(rows[0], rows[1])]
        out.append([sum(wts[t] * v[j][c] for t, j in enumerate(keys)) for c in range(len(v[0]))])
    return out


def pin_brute_force():
    rng = np.random.default_rng(6)
    B, N, H, d = 2, 7, 3, 4
    q = rng.standard_normal((B, N, H, 2, d))
    k = rng.standard_normal((B, N, H, 2, d))
    v = rng.standard_normal((B, N, H, 2 * d))
    w = 1 + 0.1 * rng.standard_normal(2 * d)
    lam, lam_init, eps = 0.45, 0.3, 1e-5
    for causal in (False, True):
        y = ref.diffattn_fwd(q, k, v, lam, lam_init, w, eps, causal)
        for b in range(B):
            for h in range(H):
                O = _brute_head(q[b, :, h, 0].tolist(), k[b, :, h, 0].tolist(),
                                q[b, :, h, 1].tolist(), k[b, :, h, 1].tolist(),
                                v[b, :, h].tolist(), lam, causal)
                for i in range(N):
                    ms = sum(x * x for x in O[i]) / (2 * d)
                    yi = [(1 - lam_init) * w[c] * O[i][c] / math.sqrt(ms + eps) for c in range(2 * d)]
                    assert np.allclose(y[b, i, h], yi, atol=1e-12, rtol=0)


def pin_decode_is_last_prefill_row():
    rng = np.random.default_rng(7)
    H, d = 2, 8
    lens = [5, 1, 12]
    cu = np.concatenate([[0], np.cumsum(lens)])
    T = int(cu[-1])
    kc = rng.standard_normal((T, H, 2, d))
    vc = rng.standard_normal((T, H, 2 * d))
    qs = rng.standard_normal((len(lens), H, 2, d))
    w = 1 + 0.1 * rng.standard_normal(2 * d)
    lam, lam_init, eps = 0.31, 0.5, 1e-5
    qp = [rng.standard_normal((1, L, H, 2, d)) for L in lens]
    for mode in ref.MODES:  # in every combination mode
        y = ref.diffattn_decode(qs, kc, vc, cu, lam, lam_init, w, eps, mode=mode)
        for s, L in enumerate(lens):
            lo = cu[s]
            q = qp[s].copy()
            q[0, L - 1] = qs[s]
            yp = ref.diffattn_fwd(q, kc[None, lo:lo + L], vc[None, lo:lo + L], lam, lam_init, w, eps, True,
                                  mode=mode)
            assert np.allclose(y[s], yp[0, L - 1], atol=1e-12)


def pin_sampled_rows():
    rng = np.random.default_rng(8)
    q = rng.standard_normal((1, 20, 2, 2, 4))
    k = rng.standard_normal((1, 20, 2, 2, 4))
    v = rng.standard_normal((1, 20, 2, 8))
    w = np.ones(8)
    rows = [0, 7, 19]
    for causal in (False, True):
        full = ref.diffattn_fwd(q, k, v, 0.4, 0.2, w, 1e-5, causal)
        part = ref.diffattn_fwd(q, k, v, 0.4, 0.2, w, 1e-5, causal, rows=rows)
        assert np.allclose(full[:, rows], part, atol=1e-13)


def _hand_rmsnorm(O, w, eps, lambda_init):
    out = np.empty_like(O)
    for i in range(O.shape[0]):
        ms = sum(float(x) * float(x) for x in O[i]) / O.shape[1]
        out[i] = (1.0 - lambda_init) * w * O[i] / math.sqrt(ms + eps)
    return out


def pin_mode_lambda_zero():
    # the review's lambda = 0 control: one softmax map (map 1), whatever map 2
    # and lambda are; torch's attention on map 1, then the headwise norm
    rng = np.random.default_rng(21)
    n, d = 9, 4
    q1, k1, q2, k2, v = _rand_head(rng, n, d)
    w = 1 + 0.1 * rng.standard_normal(2 * d)
    q = np.stack([q1, q2], 1)[None, :, None]
    k = np.stack([k1, k2], 1)[None, :, None]
    for causal in (False, True):
        y = ref.diffattn_fwd(q, k, v[None, :, None], 0.7, 0.3, w, 1e-5, causal, mode="lambda_zero")[0, :, 0]
        want = _hand_rmsnorm(_sdpa(q1, k1, v, causal), w, 1e-5, 0.3)
        assert np.allclose(y, want, atol=1e-12)
        q[0, :, 0, 1] = rng.standard_normal((n, d))  # map 2 changes: the output does not
        y2 = ref.diffattn_fwd(q, k, v[None, :, None], -1.3, 0.3, w, 1e-5, causal, mode="lambda_zero")[0, :, 0]
        assert np.array_equal(y, y2)


def pin_mode_sum():
    # the review's "+lambda" control: the two maps added; against torch's
    # attention per map, the row sums 1 + lambda, and sum(lambda) = diff(-lambda)
    rng = np.random.default_rng(22)
    n, d = 10, 4
    q1, k1, q2, k2, v = _rand_head(rng, n, d)
    lam = 0.45
    for causal in (False, True):
        O = ref.diffattn_head_prenorm(q1, k1, q2, k2, v, lam, causal, mode="sum")
        want = _sdpa(q1, k1, v, causal) + lam * _sdpa(q2, k2, v, causal)
        assert np.allclose(O, want, atol=1e-12)
        O_neg = ref.diffattn_head_prenorm(q1, k1, q2, k2, v, -lam, causal, mode="diff")
        assert np.allclose(O, O_neg, atol=1e-13)
    S1, S2 = q1 @ k1.T / 2.0, q2 @ k2.T / 2.0
    assert np.allclose(ref.map_weights(S1, S2, lam, "sum").sum(axis=1), 1.0 + lam, atol=1e-13)
    try:
        ref.map_weights(S1, S2, lam, "difference")
    except ValueError:
        pass
    else:
        raise AssertionError("an unknown mode was accepted")


PINS = [pin_worked_example, pin_large_scores, pin_row_sums, pin_lambda_zero_is_attention, pin_map2_alone,
        pin_equal_maps, pin_causal_row0, pin_rmsnorm_hand, pin_lambda_hand, pin_brute_force,
        pin_decode_is_last_prefill_row, pin_sampled_rows, pin_mode_lambda_zero, pin_mode_sum]


@pytest.mark.parametrize("pin", PINS, ids=[p.__name__ for p in PINS])
def test_pin(pin):
    pin()


# ------------------------------------------------------------ mutations ----

def _mut_sign(S1, S2, lam):
    return ref.softmax_rows(S1) + float(lam) * ref.softmax_rows(S2)


def _mut_no_max(S):
    E = np.exp(np.asarray(S, dtype=np.float64))
    return E / E.sum(axis=-1, keepdims=True)


def _mut_scale_d(q, k, scale, q_pos, causal):
    S = (q @ k.T) * (scale * scale)
    if causal:
        S = np.where(np.arange(k.shape[0])[None, :] > np.asarray(q_pos)[:, None], -np.inf, S)
    return S


def _mut_mask_dir(q, k, scale, q_pos, causal):
    S = (q @ k.T) * scale
    if causal:
        S = np.where(np.arange(k.shape[0])[None, :] < np.asarray(q_pos)[:, None], -np.inf, S)
    return S


def _mut_strict_mask(q, k, scale, q_pos, causal):
    S = (q @ k.T) * scale
    if causal:
        S = np.where(np.arange(k.shape[0])[None, :] >= np.asarray(q_pos)[:, None], -1e30, S)
    return S


def _mut_transpose(q, k, scale, q_pos, causal):
    S = (k @ q.T) * scale if q.shape[0] == k.shape[0] else (q @ k.T) * scale
    if causal:
        S = np.where(np.arange(k.shape[0])[None, :] > np.asarray(q_pos)[:, None], -np.inf, S)
    return S


def _mut_eps_outside(O, w, eps, lambda_init):
    O = np.asarray(O, dtype=np.float64)
    return (1.0 - lambda_init) * np.asarray(w) * O / (np.sqrt(np.mean(O * O, axis=-1, keepdims=True)) + eps)


def _mut_no_scale(O, w, eps, lambda_init):
    O = np.asarray(O, dtype=np.float64)
    return np.asarray(w) * O / np.sqrt(np.mean(O * O, axis=-1, keepdims=True) + eps)


def _mut_mean_sub(O, w, eps, lambda_init):
    O = np.asarray(O, dtype=np.float64)
    O = O - O.mean(axis=-1, keepdims=True)
    return (1.0 - lambda_init) * np.asarray(w) * O / np.sqrt(np.mean(O * O, axis=-1, keepdims=True) + eps)


def _mut_lambda_sign(lq1, lk1, lq2, lk2, lambda_init):
    return float(np.exp(np.dot(lq1, lk1)) + np.exp(np.dot(lq2, lk2)) + lambda_init)


def _mut_head_swap(q1, k1, q2, k2, v, lam, causal, rows=None, mode="diff"):
    return _orig_head(q1, k2, q2, k1, v, lam, causal, rows, mode)


def _mut_sum_subtracts(S1, S2, lam, mode="diff"):
    if mode == "lambda_zero":
        return ref.softmax_rows(S1)
    return ref.softmax_rows(S1) - float(lam) * ref.softmax_rows(S2)


def _mut_zero_keeps_map2(S1, S2, lam, mode="diff"):
    if mode == "sum":
        return ref.softmax_rows(S1) + float(lam) * ref.softmax_rows(S2)
    return ref.softmax_rows(S1) - float(lam) * ref.softmax_rows(S2)


def _mut_decode_maps(q1, q2, k1, k2, v, lam, mode="diff"):
    return _orig_decode(q1, q2, k1, k1, v, lam, mode)


_orig_head = ref.diffattn_head_prenorm
_orig_decode = ref.decode_head_prenorm
_orig_fwd = ref.diffattn_fwd
_orig_norm = ref.headwise_rmsnorm


def _mut_norm_over_tokens(O, w, eps, lambda_init):
    O = np.asarray(O, dtype=np.float64)
    ms = np.mean(O * O, axis=0, keepdims=True)  # over the rows instead of the head's channels
    return (1.0 - float(lambda_init)) * np.asarray(w, dtype=np.float64) * O / np.sqrt(ms + float(eps))


def _mut_weight_reversed(O, w, eps, lambda_init):
    return _orig_norm(O, np.asarray(w)[::-1], eps, lambda_init)


def _mut_v_next_head(q, k, v, lam, lambda_init, w, eps, causal, rows=None, heads=None, mode="diff"):
    return _orig_fwd(q, k, np.roll(np.asarray(v), -1, axis=2), lam, lambda_init, w, eps, causal, rows, heads, mode)


def _mut_query_maps_swapped(q, k, v, lam, lambda_init, w, eps, causal, rows=None, heads=None, mode="diff"):
    return _orig_fwd(np.asarray(q)[:, :, :, ::-1, :], k, v, lam, lambda_init, w, eps, causal, rows, heads, mode)


def _mut_rows_lose_positions(q1, k1, q2, k2, v, lam, causal, rows=None, mode="diff"):
    if rows is None:
        return _orig_head(q1, k1, q2, k2, v, lam, causal, rows, mode)
    q1, q2 = np.asarray(q1, np.float64), np.asarray(q2, np.float64)
    rows = np.asarray(rows)
    scale = 1.0 / math.sqrt(q1.shape[1])
    pos = np.arange(len(rows))  # the sampled rows masked as if they were rows 0, 1, ...
    S1 = ref._causal_scores(q1[rows], np.asarray(k1, np.float64), scale, pos, causal)
    S2 = ref._causal_scores(q2[rows], np.asarray(k2, np.float64), scale, pos, causal)
    return ref.map_weights(S1, S2, lam, mode) @ np.asarray(v, np.float64)


def _mut_scale_value_width(q1, k1, q2, k2, v, lam, causal, rows=None, mode="diff"):
    f = math.sqrt(0.5)  # 1/sqrt(2d): the value width instead of the per-map width
    return _orig_head(np.asarray(q1, np.float64) * f, k1, np.asarray(q2, np.float64) * f, k2, v, lam, causal, rows,
                      mode)

MUTANTS = {
    "plus_lambda": ("diff_weights", _mut_sign),
    "no_max_subtraction_overflow": ("softmax_rows", _mut_no_max),
    "scale_1_over_d": ("_causal_scores", _mut_scale_d),
    "mask_direction": ("_causal_scores", _mut_mask_dir),
    "mask_hides_diagonal": ("_causal_scores", _mut_strict_mask),
    "transposed_scores": ("_causal_scores", _mut_transpose),
    "eps_outside_root": ("headwise_rmsnorm", _mut_eps_outside),
    "dropped_1_minus_lambda_init": ("headwise_rmsnorm", _mut_no_scale),
    "groupnorm_mean_subtraction": ("headwise_rmsnorm", _mut_mean_sub),
    "lambda_reparam_sign": ("lambda_reparam", _mut_lambda_sign),
    "keys_of_maps_swapped": ("diffattn_head_prenorm", _mut_head_swap),
    "decode_map2_uses_k1": ("decode_head_prenorm", _mut_decode_maps),
    "sum_mode_subtracts": ("map_weights", _mut_sum_subtracts),
    "lambda_zero_keeps_map2": ("map_weights", _mut_zero_keeps_map2),
    "norm_over_tokens": ("headwise_rmsnorm", _mut_norm_over_tokens),
    "norm_weight_reversed": ("headwise_rmsnorm", _mut_weight_reversed),
    "values_of_next_head": ("diffattn_fwd", _mut_v_next_head),
    "query_maps_swapped": ("diffattn_fwd", _mut_query_maps_swapped),
    "sampled_rows_lose_positions": ("diffattn_head_prenorm", _mut_rows_lose_positions),
    "scale_1_over_sqrt_value_width": ("diffattn_head_prenorm", _mut_scale_value_width),
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_pins_catch_mutant(name, monkeypatch):
    attr, fn = MUTANTS[name]
    monkeypatch.setattr(ref, attr, fn)
    caught = []
    for pin in PINS:
        try:
            with np.errstate(all="ignore"):
                pin()
        except (AssertionError, FloatingPointError, ValueError):
            caught.append(pin.__name__)
    assert caught, f"no pin catches mutant {name}"
