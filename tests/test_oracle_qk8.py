"""Pins for the e4m3 query/key oracle (no GPU).

The codec is pinned to hand-decoded codes of the OCP FP8 E4M3 format, to an
independent round-to-nearest-even formula, and to its ties, saturation and
subnormal edge; the quantiser to the absmax element landing on 448 and to the
half-ulp error bound; the forward to the bf16-path oracle on inputs that the
quantisation leaves unchanged.  The mutation test plants plausible mistakes on
the CPU and checks that some pin fails for each.
"""
import math

import numpy as np
import pytest

import oracle.diffattn_ref as ref
import oracle.qk8_ref as q8


def _rne_formula(x):
    """Round |x| to 3 mantissa bits (exponent at least -6, so the subnormal step
    is 2^-9), ties to even, clamp at 448; the sign is kept."""
    x = np.asarray(x, dtype=np.float64)
    mag = np.minimum(np.abs(x), 448.0)
    out = np.zeros_like(mag)
    nz = mag > 0
    e = np.maximum(np.floor(np.log2(mag[nz])), -6.0)
    step = 2.0 ** (e - 3)
    out[nz] = np.round(mag[nz] / step) * step  # numpy rounds half to even
    return np.copysign(np.minimum(out, 448.0), x)


def pin_decoded_codes():
    t = q8.e4m3_table()
    hand = {0x00: 0.0, 0x01: 2.0 ** -9, 0x07: 7 * 2.0 ** -9, 0x08: 2.0 ** -6, 0x38: 1.0, 0x39: 1.125,
            0x3F: 1.875, 0x40: 2.0, 0x7E: 448.0, 0xB8: -1.0, 0xFE: -448.0}
    for c, v in hand.items():
        assert t[c] == v, (hex(c), t[c], v)
    assert np.isnan(t[0x7F]) and np.isnan(t[0xFF])
    assert np.signbit(t[0x80]) and t[0x80] == 0.0
    assert np.nanmax(t) == 448.0 and np.sum(np.isnan(t)) == 2


def pin_encoder_matches_formula():
    rng = np.random.default_rng(3)
    x = np.concatenate([rng.standard_normal(20000) * s for s in (1e-3, 0.05, 1.0, 30.0, 300.0)]).astype(np.float32)
    got = q8.e4m3_table()[q8.e4m3_encode(x)]
    assert np.array_equal(got, _rne_formula(x))


def pin_ties_saturation_subnormals():
    enc = lambda v: int(q8.e4m3_encode(np.array([v], np.float32))[0])
    assert enc(1.0625) == 0x38 and enc(1.1875) == 0x3A       # ties to the even code
    assert enc(2.0 ** -10) == 0x00 and enc(3 * 2.0 ** -10) == 0x02
    assert enc(500.0) == 0x7E and enc(1e30) == 0x7E and enc(-1e30) == 0xFE
    assert enc(-1e-6) == 0x80
    finite = [c for c in range(256) if not np.isnan(q8.e4m3_table()[c])]
    assert all(enc(q8.e4m3_table()[c]) == c for c in finite)  # every value encodes to its own code


def pin_absmax_lands_on_448():
    rng = np.random.default_rng(4)
    t = (rng.standard_normal((2, 33, 3, 2, 16)) * rng.uniform(0.1, 10, (2, 1, 3, 2, 1))).astype(np.float32)
    codes, s = q8.quantize_qk(t)
    assert s.shape == (2, 3, 2) and s.dtype == np.float32
    for b in range(2):
        for h in range(3):
            for i in range(2):
                g = t[b, :, h, i]
                assert s[b, h, i] == np.float32(np.abs(g).max() / np.float32(448.0))
                c = codes[b, :, h, i]
                assert (c & 0x7F).max() == 0x7E                       # the absmax element
                assert ((c & 0x7F) <= 0x7E).all()                     # no NaN codes
    z = np.zeros((1, 4, 1, 2, 8), np.float32)
    zc, zs = q8.quantize_qk(z)
    assert (zs == 1.0).all() and (zc == 0).all()


def pin_error_bound():
    rng = np.random.default_rng(5)
    t = rng.standard_normal((1, 64, 2, 2, 32)).astype(np.float32)
    codes, s = q8.quantize_qk(t)
    deq = q8.dequantize(codes, s)
    scale = s[:, None, :, :, None].astype(np.float64)
    bound = np.maximum(np.abs(t) * 2.0 ** -4, scale * 2.0 ** -10) * (1 + 1e-6)
    assert (np.abs(deq - t) <= bound).all()


def pin_lossless_inputs_give_bf16_result():
    # every group holds +-448 * 2^p and otherwise e4m3 values * 2^p: quantisation is exact
    rng = np.random.default_rng(6)
    B, N, H, d = 1, 24, 2, 8
    tab = q8.e4m3_table()
    finite = np.array([c for c in range(256) if not np.isnan(tab[c])])

    def exact(p):
        t = tab[rng.choice(finite, (B, N, H, 2, d))] * 2.0 ** p
        t[:, 0, :, :, 0] = 448.0 * 2.0 ** p
        return t.astype(np.float32)

    q, k = exact(-7), exact(-6)
    v = rng.standard_normal((B, N, H, 2 * d))
    w = 1 + 0.1 * rng.standard_normal(2 * d)
    for causal in (True, False):
        y8 = q8.diffattn_fwd_qk8(q, k, v, 0.4, 0.3, w, 1e-5, causal)
        y = ref.diffattn_fwd(q.astype(np.float64), k.astype(np.float64), v, 0.4, 0.3, w, 1e-5, causal)
        assert np.array_equal(y8, y)


def pin_groups_are_per_batch_head_map():
    # scaling one (batch, head, map) group changes its scale only
    rng = np.random.default_rng(7)
    t = rng.standard_normal((2, 10, 2, 2, 8)).astype(np.float32)
    _, s0 = q8.quantize_qk(t)
    t2 = t.copy()
    t2[1, :, 0, 1] *= 8.0
    c2, s2 = q8.quantize_qk(t2)
    changed = s2 != s0
    assert changed[1, 0, 1] and changed.sum() == 1
    assert s2[1, 0, 1] == np.float32(s0[1, 0, 1] * 8)


PINS = [pin_decoded_codes, pin_encoder_matches_formula, pin_ties_saturation_subnormals, pin_absmax_lands_on_448,
        pin_error_bound, pin_lossless_inputs_give_bf16_result, pin_groups_are_per_batch_head_map]


@pytest.mark.parametrize("pin", PINS, ids=[p.__name__ for p in PINS])
def test_pin(pin):
    pin()


# ------------------------------------------------------------ mutations ----

_orig_encode = q8.e4m3_encode
_orig_table = q8.e4m3_table


def _mut_ties_up(x):
    x32 = np.asarray(x, dtype=np.float32)
    mag = np.minimum(np.abs(x32.astype(np.float64)), 448.0)
    vals = q8._POS_VALS
    hi = np.clip(np.searchsorted(vals, mag, side="left"), 0, len(vals) - 1)
    lo = np.clip(hi - 1, 0, len(vals) - 1)
    code = np.where(vals[hi] - mag <= mag - vals[lo], hi, lo).astype(np.uint8)
    return np.where(np.signbit(x32), code | np.uint8(0x80), code).astype(np.uint8)


def _mut_no_saturation(x):
    x32 = np.asarray(x, dtype=np.float32)
    c = _orig_encode(x32)
    return np.where(np.abs(x32) > 448.0, np.uint8(0x7F) | (c & np.uint8(0x80)), c).astype(np.uint8)


def _mut_bias8():
    t = _orig_table()
    return t / 2.0


def _mut_scale_240(t):
    t = np.asarray(t, dtype=np.float32)
    amax = np.abs(t).max(axis=(1, 4))
    return np.where(amax > 0, (amax / np.float32(240.0)).astype(np.float32), np.float32(1.0)).astype(np.float32)


def _mut_per_tensor(t):
    t = np.asarray(t, dtype=np.float32)
    amax = np.abs(t).max()
    return np.full((t.shape[0], t.shape[2], 2), amax / np.float32(448.0), np.float32)


def _mut_truncate(x):
    x32 = np.asarray(x, dtype=np.float32)
    mag = np.minimum(np.abs(x32.astype(np.float64)), 448.0)
    idx = np.clip(np.searchsorted(q8._POS_VALS, mag, side="right") - 1, 0, len(q8._POS_VALS) - 1)
    code = q8._POS_CODES[idx].astype(np.uint8)
    return np.where(np.signbit(x32), code | np.uint8(0x80), code).astype(np.uint8)


MUTANTS = {
    "ties_away_from_zero": ("e4m3_encode", _mut_ties_up),
    "no_saturation": ("e4m3_encode", _mut_no_saturation),
    "exponent_bias_8": ("e4m3_table", _mut_bias8),
    "scale_to_240": ("absmax_scales", _mut_scale_240),
    "per_tensor_scale": ("absmax_scales", _mut_per_tensor),
    "truncating_encoder": ("e4m3_encode", _mut_truncate),
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_pins_catch_mutant(name, monkeypatch):
    attr, fn = MUTANTS[name]
    monkeypatch.setattr(q8, attr, fn)
    if attr == "e4m3_table":
        monkeypatch.setattr(q8, "_TABLE", fn())
    caught = []
    for pin in PINS:
        try:
            with np.errstate(all="ignore"):
                pin()
        except (AssertionError, FloatingPointError, ValueError, IndexError):
            caught.append(pin.__name__)
    assert caught, f"no pin catches mutant {name}"
