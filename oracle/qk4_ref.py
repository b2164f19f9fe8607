"""Plain CPU oracle for the 4-bit (FP4 e2m1) query/key variant of the prefill.

TEST INFRASTRUCTURE ONLY, like ``diffattn_ref``: nothing on the product path
imports this module, and it shares no code with the CUDA library.

What it computes
----------------
The peer review "Differential Transformer" (Strengths, the activation-outlier
bullet) cites 4-bit attention-logit quantisation (Fig. 8 of the paper) as
pointing at low-bit attention kernels, and its Questions ask whether absmax
quantisation is applied per logit map and per head.  This variant takes the
same reading as the 8-bit one (``qk8_ref``), with 4-bit codes:

* For every (batch b, head h, map i) the queries Q_i[b, :, h, :] (all N tokens,
  all d channels) share one absmax scale, and so do the keys K_i[b, :, h, :]:

      amax  = max |x| over the group            (float32, exact)
      scale = amax / 6     (float32 division)   (1 when amax = 0)
      code  = e2m1(x / scale)                   (x / scale in float32, then
                                                 the nearest e2m1 value,
                                                 ties to the even code,
                                                 saturating at +-6)

  6 is the largest e2m1 magnitude, so the group's absmax lands on it.
* The scores use the dequantised values, code value * scale; everything after
  the scores is the float64 DiffAttn of ``diffattn_ref``.

The e2m1 format (OCP Microscaling Formats specification v1.0, the FP4 E2M1
element type): bit 3 sign, bits 2..1 exponent with bias 1, bit 0 mantissa;
exponent 0 holds the subnormals m * 2^-1.  The eight magnitudes are
0, 0.5, 1, 1.5, 2, 3, 4, 6; there is no infinity and no NaN.  The encoder here
is the plain definition: the nearest value of the 16-entry table, ties to the
even code, magnitudes beyond 6 clamped, the sign kept (so negative values that
round to zero give the code of -0).

Storage: two codes per byte along the channel axis, channel 2j in the low
nibble and channel 2j + 1 in the high nibble, so a [.., d] row of codes takes
d / 2 bytes (``pack`` / ``unpack``).

Pins (tests/test_oracle_qk4.py): the specification's value table, an
independent round-to-nearest-even formula for the encoder, ties, saturation
and the sign of zero, the absmax element landing on 6, the nibble order of a
hand-packed row, lossless inputs giving the unquantised result, and the
dequantised error bound.  Planted mistakes must fail at least one pin.
"""
from __future__ import annotations

import numpy as np

from . import diffattn_ref as ref

E2M1_MAX = 6.0

__all__ = ["E2M1_MAX", "e2m1_table", "e2m1_encode", "absmax_scales", "quantize_qk", "pack", "unpack",
           "dequantize", "diffattn_fwd_qk4"]


def e2m1_table() -> np.ndarray:
    """The value of each of the 16 codes (float64)."""
    vals = np.empty(16, dtype=np.float64)
    for c in range(16):
        s = -1.0 if c & 0x8 else 1.0
        e = (c >> 1) & 0x3
        m = c & 0x1
        if e == 0:
            vals[c] = s * m * 0.5
        else:
            vals[c] = s * (1.0 + m / 2.0) * 2.0 ** (e - 1)
    return vals


def _pos():
    table = e2m1_table()
    codes = np.arange(8)  # 0x0 .. 0x7: the non-negative values, ascending
    return codes, table[codes]


def e2m1_encode(x) -> np.ndarray:
    """Nearest e2m1 code (uint8, 0..15) for each element of x (float32
    values): ties to the even code, magnitudes beyond 6 saturate to +-6, the
    sign is kept."""
    pos_codes, pos_vals = _pos()
    x = np.asarray(x, dtype=np.float32).astype(np.float64)
    mag = np.minimum(np.abs(x), E2M1_MAX)
    hi = np.clip(np.searchsorted(pos_vals, mag, side="left"), 0, len(pos_vals) - 1)  # first value >= mag
    lo = np.clip(hi - 1, 0, len(pos_vals) - 1)
    d_lo = mag - pos_vals[lo]
    d_hi = pos_vals[hi] - mag
    pick_hi = (d_hi < d_lo) | ((d_hi == d_lo) & (pos_codes[hi] % 2 == 0) & (hi != lo))
    code = np.where(pick_hi, pos_codes[hi], pos_codes[lo]).astype(np.uint8)
    return np.where(np.signbit(x), code | np.uint8(0x8), code).astype(np.uint8)


def absmax_scales(t) -> np.ndarray:
    """float32 scales [B, H, 2] of t [B, N, H, 2, d]: absmax of each (b, h, map)
    group divided by 6 in float32 (1 for an all-zero group)."""
    t = np.asarray(t, dtype=np.float32)
    amax = np.abs(t).max(axis=(1, 4))
    scale = (amax / np.float32(E2M1_MAX)).astype(np.float32)
    return np.where(amax > 0, scale, np.float32(1.0)).astype(np.float32)


def quantize_qk(t):
    """(codes uint8 [B, N, H, 2, d], one code 0..15 per element; scales
    float32 [B, H, 2]) for t [B, N, H, 2, d]."""
    t = np.asarray(t, dtype=np.float32)
    s = absmax_scales(t)
    ratio = (t / s[:, None, :, :, None]).astype(np.float32)  # float32 division
    return e2m1_encode(ratio), s


def pack(codes) -> np.ndarray:
    """Two codes per byte along the last axis: [.., d] -> [.., d / 2] uint8,
    element 2j in the low nibble, 2j + 1 in the high nibble."""
    c = np.asarray(codes, dtype=np.uint8)
    if c.shape[-1] % 2:
        raise ValueError("the last axis must have even length")
    return (c[..., 0::2] & 0xF) | ((c[..., 1::2] & 0xF) << 4)


def unpack(packed) -> np.ndarray:
    """Inverse of ``pack``: [.., d / 2] uint8 -> [.., d] codes."""
    p = np.asarray(packed, dtype=np.uint8)
    out = np.empty(p.shape[:-1] + (2 * p.shape[-1],), dtype=np.uint8)
    out[..., 0::2] = p & 0xF
    out[..., 1::2] = p >> 4
    return out


def dequantize(codes, scales) -> np.ndarray:
    """float64 values code * scale, [B, N, H, 2, d] (codes unpacked)."""
    return e2m1_table()[np.asarray(codes)] * np.asarray(scales, dtype=np.float64)[:, None, :, :, None]


def diffattn_fwd_qk4(q, k, v, lam: float, lambda_init: float, w, eps: float, causal: bool,
                     rows=None, heads=None, mode: str = "diff") -> np.ndarray:
    """The prefill with queries and keys quantised to e2m1 per (batch, head, map).

    q, k : [B, N, H, 2, d] (the bf16 values the library receives); v : [B, N, H, 2d].
    Same output as ``diffattn_ref.diffattn_fwd`` on the dequantised q and k.
    """
    qc, qs = quantize_qk(q)
    kc, ks = quantize_qk(k)
    return ref.diffattn_fwd(dequantize(qc, qs), dequantize(kc, ks), v, lam, lambda_init, w, eps, causal,
                            rows=rows, heads=heads, mode=mode)
