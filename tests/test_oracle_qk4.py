"""Pins for the e2m1 (FP4) query/key oracle (no GPU).

The codec is pinned to the value table of the OCP Microscaling Formats
specification's FP4 E2M1 type, to an independent round-to-nearest-even
formula, and to its ties, saturation and sign of zero; the packing to a row
packed by hand; the quantiser to the absmax element landing on 6 and to the
half-step error bound; the forward to the unquantised oracle on inputs that
the quantisation leaves unchanged.  The mutation test plants plausible
mistakes on the CPU and checks that some pin fails for each.
"""
import numpy as np
import pytest

import oracle.diffattn_ref as ref
import oracle.qk4_ref as q4


def _rne_formula(x):
    """Round |x| to 1 mantissa bit (exponent at least 0, so the subnormal step
    is 1/2), ties to even, clamp at 6; the sign is kept."""
    x = np.asarray(x, dtype=np.float64)
    mag = np.minimum(np.abs(x), 6.0)
    out = np.zeros_like(mag)
    nz = mag > 0
    e = np.maximum(np.floor(np.log2(mag[nz])), 0.0)
    step = 2.0 ** (e - 1)
    out[nz] = np.round(mag[nz] / step) * step  # numpy rounds half to even
    return np.copysign(np.minimum(out, 6.0), x)


def pin_spec_values():
    t = q4.e2m1_table()
    spec = [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]
    assert list(t[:8]) == spec
    assert list(t[8:]) == [-v for v in spec]
    assert np.signbit(t[8]) and not np.signbit(t[0])


def pin_encoder_matches_formula():
    rng = np.random.default_rng(13)
    x = np.concatenate([rng.standard_normal(20000) * s for s in (0.05, 0.5, 1.0, 2.5, 10.0)]).astype(np.float32)
    got = q4.e2m1_table()[q4.e2m1_encode(x)]
    assert np.array_equal(got, _rne_formula(x))


def pin_ties_saturation_sign():
    enc = lambda v: int(q4.e2m1_encode(np.array([v], np.float32))[0])
    ties = {0.25: 0, 0.75: 2, 1.25: 2, 1.75: 4, 2.5: 4, 3.5: 6, 5.0: 6}  # to the even code
    for v, c in ties.items():
        assert enc(v) == c, (v, enc(v), c)
        assert enc(-v) == c | 0x8, (-v, enc(-v))
    assert enc(6.5) == 0x7 and enc(1e30) == 0x7 and enc(-1e30) == 0xF
    assert enc(-0.1) == 0x8 and enc(0.1) == 0x0
    assert all(enc(q4.e2m1_table()[c]) == c for c in range(16))  # every value encodes to its own code


def pin_absmax_lands_on_6():
    rng = np.random.default_rng(14)
    t = (rng.standard_normal((2, 33, 3, 2, 16)) * rng.uniform(0.1, 10, (2, 1, 3, 2, 1))).astype(np.float32)
    codes, s = q4.quantize_qk(t)
    assert s.shape == (2, 3, 2) and s.dtype == np.float32
    assert codes.dtype == np.uint8 and codes.shape == t.shape and codes.max() <= 0xF
    for b in range(2):
        for h in range(3):
            for i in range(2):
                g = t[b, :, h, i]
                assert s[b, h, i] == np.float32(np.abs(g).max() / np.float32(6.0))
                assert (codes[b, :, h, i] & 0x7).max() == 0x7  # the absmax element
    z = np.zeros((1, 4, 1, 2, 8), np.float32)
    zc, zs = q4.quantize_qk(z)
    assert (zs == 1.0).all() and (zc == 0).all()


def pin_nibble_order():
    assert q4.pack(np.array([[1, 2, 3, 15]], np.uint8)).tolist() == [[0x21, 0xF3]]
    assert q4.unpack(np.array([0x21, 0xF3], np.uint8)).tolist() == [1, 2, 3, 15]
    c = np.random.default_rng(15).integers(0, 16, (3, 5, 2, 2, 32)).astype(np.uint8)
    p = q4.pack(c)
    assert p.shape == (3, 5, 2, 2, 16)
    assert np.array_equal(q4.unpack(p), c)


def pin_error_bound():
    rng = np.random.default_rng(16)
    t = rng.standard_normal((1, 64, 2, 2, 32)).astype(np.float32)
    codes, s = q4.quantize_qk(t)
    deq = q4.dequantize(codes, s)
    scale = s[:, None, :, :, None].astype(np.float64)
    bound = np.maximum(np.abs(t) / 4.0, scale / 4.0) * (1 + 1e-6)
    assert (np.abs(deq - t) <= bound).all()


def pin_lossless_inputs_give_unquantised_result():
    # every group holds +-6 * 2^p and otherwise e2m1 values * 2^p: quantisation is exact
    rng = np.random.default_rng(17)
    B, N, H, d = 1, 24, 2, 8
    tab = q4.e2m1_table()

    def exact(p):
        t = tab[rng.integers(0, 16, (B, N, H, 2, d))] * 2.0 ** p
        t[:, 0, :, :, 0] = 6.0 * 2.0 ** p
        return t.astype(np.float32)

    q, k = exact(-3), exact(-2)
    v = rng.standard_normal((B, N, H, 2 * d))
    w = 1 + 0.1 * rng.standard_normal(2 * d)
    for causal in (True, False):
        y4 = q4.diffattn_fwd_qk4(q, k, v, 0.4, 0.3, w, 1e-5, causal)
        y = ref.diffattn_fwd(q.astype(np.float64), k.astype(np.float64), v, 0.4, 0.3, w, 1e-5, causal)
        assert np.array_equal(y4, y)


def pin_groups_are_per_batch_head_map():
    # scaling one (batch, head, map) group changes its scale only
    rng = np.random.default_rng(18)
    t = rng.standard_normal((2, 10, 2, 2, 8)).astype(np.float32)
    c0, s0 = q4.quantize_qk(t)
    t2 = t.copy()
    t2[1, :, 0, 1] *= 8.0
    c2, s2 = q4.quantize_qk(t2)
    changed = s2 != s0
    assert changed[1, 0, 1] and changed.sum() == 1
    assert s2[1, 0, 1] == np.float32(s0[1, 0, 1] * 8)
    assert np.array_equal(c2, c0)  # a power-of-two rescale leaves the codes as they were


PINS = [pin_spec_values, pin_encoder_matches_formula, pin_ties_saturation_sign, pin_absmax_lands_on_6,
        pin_nibble_order, pin_error_bound, pin_lossless_inputs_give_unquantised_result,
        pin_groups_are_per_batch_head_map]


@pytest.mark.parametrize("pin", PINS, ids=[p.__name__ for p in PINS])
def test_pin(pin):
    pin()


# ------------------------------------------------------------ mutations ----

_orig_encode = q4.e2m1_encode
_orig_table = q4.e2m1_table
_orig_pack = q4.pack
_POS = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0])


def _mut_ties_up(x):
    x32 = np.asarray(x, dtype=np.float32)
    mag = np.minimum(np.abs(x32.astype(np.float64)), 6.0)
    hi = np.clip(np.searchsorted(_POS, mag, side="left"), 0, 7)
    lo = np.clip(hi - 1, 0, 7)
    code = np.where(_POS[hi] - mag <= mag - _POS[lo], hi, lo).astype(np.uint8)
    return np.where(np.signbit(x32), code | np.uint8(0x8), code).astype(np.uint8)


def _mut_truncate(x):
    x32 = np.asarray(x, dtype=np.float32)
    mag = np.minimum(np.abs(x32.astype(np.float64)), 6.0)
    code = np.clip(np.searchsorted(_POS, mag, side="right") - 1, 0, 7).astype(np.uint8)
    return np.where(np.signbit(x32), code | np.uint8(0x8), code).astype(np.uint8)


def _mut_sign_dropped(x):
    return _orig_encode(np.abs(np.asarray(x, dtype=np.float32)))


def _mut_bias2():
    return _orig_table() / 2.0


def _mut_scale_448(t):
    t = np.asarray(t, dtype=np.float32)
    amax = np.abs(t).max(axis=(1, 4))
    return np.where(amax > 0, (amax / np.float32(448.0)).astype(np.float32), np.float32(1.0)).astype(np.float32)


def _mut_per_tensor(t):
    t = np.asarray(t, dtype=np.float32)
    return np.full((t.shape[0], t.shape[2], 2), np.abs(t).max() / np.float32(6.0), np.float32)


def _mut_nibbles_swapped(codes):
    c = np.asarray(codes, dtype=np.uint8)
    return ((c[..., 0::2] & 0xF) << 4) | (c[..., 1::2] & 0xF)


MUTANTS = {
    "ties_away_from_zero": ("e2m1_encode", _mut_ties_up),
    "truncating_encoder": ("e2m1_encode", _mut_truncate),
    "sign_dropped": ("e2m1_encode", _mut_sign_dropped),
    "exponent_bias_2": ("e2m1_table", _mut_bias2),
    "scale_to_448": ("absmax_scales", _mut_scale_448),
    "per_tensor_scale": ("absmax_scales", _mut_per_tensor),
    "nibbles_swapped": ("pack", _mut_nibbles_swapped),
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_pins_catch_mutant(name, monkeypatch):
    attr, fn = MUTANTS[name]
    monkeypatch.setattr(q4, attr, fn)
    caught = []
    for pin in PINS:
        try:
            with np.errstate(all="ignore"):
                pin()
        except (AssertionError, FloatingPointError, ValueError, IndexError):
            caught.append(pin.__name__)
    assert caught, f"no pin catches mutant {name}"
