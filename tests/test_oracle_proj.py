"""Pins for the projection / rotary-embedding oracle (no GPU).

RoPE is pinned to a rotation worked by hand, to the identity at position 0,
to norm preservation and to RoFormer's relative-position property; the
projections to explicit loops.  The mutation test plants plausible mistakes
(rotating the two halves instead of consecutive pairs, a flipped sine, a
wrong frequency exponent, a transposed weight, swapped maps) on the CPU and
checks that some pin fails for each.
"""
import math

import numpy as np
import pytest

import oracle.proj_ref as pr


def pin_worked_rotation():
    # d = 4, position 1, base 100: theta = (1, 100^-1/2 = 0.1)
    x = np.array([[1.0, 2.0, 3.0, -1.0]])
    got = pr.apply_rope(x, [1], base=100.0)[0]
    c0, s0, c1, s1 = math.cos(1.0), math.sin(1.0), math.cos(0.1), math.sin(0.1)
    want = [1 * c0 - 2 * s0, 1 * s0 + 2 * c0, 3 * c1 + 1 * s1, 3 * s1 - 1 * c1]
    assert np.allclose(got, want, rtol=0, atol=1e-15)


def pin_position_zero_is_identity():
    x = np.random.default_rng(1).standard_normal((3, 5, 8))
    assert np.array_equal(pr.apply_rope(x[:, :1], [0])[:, 0], x[:, 0])


def pin_norm_of_each_pair():
    rng = np.random.default_rng(2)
    x = rng.standard_normal((7, 16))
    y = pr.apply_rope(x, np.arange(7) * 37)
    assert np.allclose(x[:, 0::2] ** 2 + x[:, 1::2] ** 2, y[:, 0::2] ** 2 + y[:, 1::2] ** 2, atol=1e-12)


def pin_relative_position():
    rng = np.random.default_rng(3)
    q, k = rng.standard_normal(32), rng.standard_normal(32)
    dots = []
    for m, n in [(5, 2), (105, 102), (3, 0), (1003, 1000)]:
        qm = pr.apply_rope(q[None], [m])[0]
        kn = pr.apply_rope(k[None], [n])[0]
        dots.append(float(qm @ kn))
    assert np.allclose(dots, dots[0], atol=1e-9)
    # and it does change with the offset
    q7 = pr.apply_rope(q[None], [7])[0]
    assert abs(float(q7 @ pr.apply_rope(k[None], [0])[0]) - dots[0]) > 1e-3


def pin_projection_loops():
    rng = np.random.default_rng(4)
    B, N, H, d, dm = 2, 3, 2, 4, 5
    x = rng.standard_normal((B * N, dm))
    w = rng.standard_normal((3 * H * 2 * d, dm))
    q, k, v = pr.qkv_proj(x, w, B, N, H, d, rope_base=None)
    for b in range(B):
        for n in range(N):
            row = b * N + n
            for h in range(H):
                for i in range(2):
                    for c in range(d):
                        fq = (h * 2 + i) * d + c
                        assert abs(q[b, n, h, i, c] - sum(x[row, t] * w[fq, t] for t in range(dm))) < 1e-12
                        fk = H * 2 * d + fq
                        assert abs(k[b, n, h, i, c] - sum(x[row, t] * w[fk, t] for t in range(dm))) < 1e-12
                for c in range(2 * d):
                    fv = 2 * H * 2 * d + h * 2 * d + c
                    assert abs(v[b, n, h, c] - sum(x[row, t] * w[fv, t] for t in range(dm))) < 1e-12
    o = rng.standard_normal((B * N, H * 2 * d))
    wo = rng.standard_normal((dm, H * 2 * d))
    y = pr.out_proj(o, wo)
    for r in range(B * N):
        for f in range(dm):
            assert abs(y[r, f] - sum(o[r, t] * wo[f, t] for t in range(H * 2 * d))) < 1e-12


def pin_rope_in_projection():
    # the rotated projection equals the plain one rotated per token position,
    # head and map (positions restart for every batch row)
    rng = np.random.default_rng(5)
    B, N, H, d, dm = 2, 6, 2, 8, 12
    x = rng.standard_normal((B * N, dm))
    w = rng.standard_normal((3 * H * 2 * d, dm))
    q0, k0, v0 = pr.qkv_proj(x, w, B, N, H, d, rope_base=None)
    q, k, v = pr.qkv_proj(x, w, B, N, H, d, rope_base=500.0)
    assert np.array_equal(v, v0)
    for b in range(B):
        for n in range(N):
            for h in range(H):
                for i in range(2):
                    assert np.allclose(q[b, n, h, i], pr.apply_rope(q0[b, n, h, i][None], [n], 500.0)[0], atol=1e-12)
                    assert np.allclose(k[b, n, h, i], pr.apply_rope(k0[b, n, h, i][None], [n], 500.0)[0], atol=1e-12)
    assert np.array_equal(q[:, 0], q0[:, 0])


PINS = [pin_worked_rotation, pin_position_zero_is_identity, pin_norm_of_each_pair, pin_relative_position,
        pin_projection_loops, pin_rope_in_projection]


@pytest.mark.parametrize("pin", PINS, ids=[p.__name__ for p in PINS])
def test_pin(pin):
    pin()


# ------------------------------------------------------------ mutations ----

_orig_apply = pr.apply_rope
_orig_angles = pr.rope_angles
_orig_qkv = pr.qkv_proj


def _mut_half_split(x, positions, base=10000.0):
    x = np.asarray(x, dtype=np.float64)
    d = x.shape[-1]
    ang = _orig_angles(positions, d, base)
    c, s = np.cos(ang), np.sin(ang)
    a, b = x[..., : d // 2], x[..., d // 2:]
    return np.concatenate([a * c - b * s, a * s + b * c], axis=-1)


def _mut_sine_sign(x, positions, base=10000.0):
    x = np.asarray(x, dtype=np.float64)
    ang = _orig_angles(positions, x.shape[-1], base)
    c, s = np.cos(ang), np.sin(ang)
    out = np.empty_like(x)
    out[..., 0::2] = x[..., 0::2] * c + x[..., 1::2] * s
    out[..., 1::2] = -x[..., 0::2] * s + x[..., 1::2] * c
    return out


def _mut_exponent(positions, d, base=10000.0):
    j = np.arange(d // 2, dtype=np.float64)
    return np.asarray(positions, dtype=np.float64)[:, None] * (float(base) ** (-j / d))[None, :]


def _mut_transposed_weight(x, w_qkv, B, N, H, d, rope_base=10000.0):
    w = np.asarray(w_qkv, dtype=np.float64)
    hq = H * 2 * d
    # the output features read as (map, head) instead of (head, map)
    wq = w[:hq].reshape(H, 2, d, -1).transpose(1, 0, 2, 3).reshape(hq, -1)
    return _orig_qkv(x, np.concatenate([wq, w[hq:]]), B, N, H, d, rope_base)


def _mut_positions_global(x, w_qkv, B, N, H, d, rope_base=10000.0):
    # positions run over the flattened rows instead of restarting per batch row
    q, k, v = _orig_qkv(x, w_qkv, B, N, H, d, None)
    if rope_base is not None:
        pos = np.arange(B * N)
        q = _orig_apply(q.reshape(B * N, H * 2, d).transpose(1, 0, 2), pos, rope_base).transpose(1, 0, 2)
        k = _orig_apply(k.reshape(B * N, H * 2, d).transpose(1, 0, 2), pos, rope_base).transpose(1, 0, 2)
        q, k = q.reshape(B, N, H, 2, d), k.reshape(B, N, H, 2, d)
    return q, k, v


MUTANTS = {
    "rope_half_split_pairs": ("apply_rope", _mut_half_split),
    "rope_sine_sign": ("apply_rope", _mut_sine_sign),
    "rope_frequency_exponent": ("rope_angles", _mut_exponent),
    "qkv_maps_and_heads_swapped": ("qkv_proj", _mut_transposed_weight),
    "rope_positions_not_per_sequence": ("qkv_proj", _mut_positions_global),
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_pins_catch_mutant(name, monkeypatch):
    attr, fn = MUTANTS[name]
    monkeypatch.setattr(pr, attr, fn)
    caught = []
    for pin in PINS:
        try:
            pin()
        except (AssertionError, ValueError, IndexError):
            caught.append(pin.__name__)
    assert caught, f"no pin catches mutant {name}"


from hypothesis import given, settings  # noqa: E402
from hypothesis import strategies as st  # noqa: E402


@settings(max_examples=25, deadline=None)
@given(B=st.integers(1, 2), N=st.integers(1, 5), H=st.integers(1, 2), half=st.integers(1, 3), dm=st.integers(1, 6),
       base=st.sampled_from([100.0, 10000.0]), seed=st.integers(0, 2 ** 31 - 1))
def test_projection_with_rope_matches_loops(B, N, H, half, dm, base, seed):
    # the fused projection + rotation over drawn shapes, against loops that rotate each
    # consecutive channel pair of Q1, Q2, K1, K2 by n * base^(-2j/d), n the token's position
    d = 2 * half
    rng = np.random.default_rng(seed)
    x = rng.standard_normal((B * N, dm))
    w = rng.standard_normal((3 * H * 2 * d, dm))
    q, k, v = pr.qkv_proj(x, w, B, N, H, d, rope_base=base)
    for b in range(B):
        for n in range(N):
            row = b * N + n
            feat = [sum(x[row, t] * w[f, t] for t in range(dm)) for f in range(w.shape[0])]
            for h in range(H):
                for i in range(2):
                    for part, got in ((0, q), (1, k)):
                        f0 = part * H * 2 * d + (h * 2 + i) * d
                        for j in range(half):
                            a, c = feat[f0 + 2 * j], feat[f0 + 2 * j + 1]
                            ang = n * base ** (-2.0 * j / d)
                            want = (a * math.cos(ang) - c * math.sin(ang), a * math.sin(ang) + c * math.cos(ang))
                            assert abs(got[b, n, h, i, 2 * j] - want[0]) < 1e-9
                            assert abs(got[b, n, h, i, 2 * j + 1] - want[1]) < 1e-9
                for c2 in range(2 * d):
                    assert abs(v[b, n, h, c2] - feat[2 * H * 2 * d + h * 2 * d + c2]) < 1e-9
