"""Plain CPU oracle for the low-bit (FP8 e4m3) query/key variant of the prefill.

TEST INFRASTRUCTURE ONLY, like ``diffattn_ref``: nothing on the product path
imports this module, and it shares no code with the CUDA library.

What it computes
----------------
The peer review "Differential Transformer" (Strengths, the activation-outlier
bullet; Questions, the quantisation bullet) points at low-bit attention
kernels and asks whether absmax quantisation is applied per logit map and per
head.  This variant takes that reading for the inputs of the two logit maps:

* For every (batch b, head h, map i) the queries Q_i[b, :, h, :] (all N tokens,
  all d channels) share one absmax scale, and so do the keys K_i[b, :, h, :]:

      amax  = max |x| over the group            (float32, exact)
      scale = amax / 448   (float32 division)   (1 when amax = 0)
      code  = e4m3(x / scale)                   (x / scale in float32, then
                                                 round to nearest e4m3 value,
                                                 ties to even, saturating at
                                                 +-448)

  448 is the largest finite e4m3 value, so the group's absmax lands on it.
* The scores use the dequantised values, code value * scale; everything after
  the scores (both softmax maps, the difference with lambda, the value
  product, the headwise RMSNorm and the (1 - lambda_init) scale) is the
  float64 DiffAttn of ``diffattn_ref``.

The e4m3 format (OCP 8-bit floating point, the FP8 E4M3 encoding): bit 7 sign,
bits 6..3 exponent with bias 7, bits 2..0 mantissa; exponent 0 holds the
subnormals m * 2^-9; exponent 15 with mantissa 7 is NaN; there is no infinity.
The encoder here is the plain definition: the nearest finite value of the
256-entry table, ties to the even code, magnitudes beyond 448 clamped.

Pins (tests/test_oracle_qk8.py): hand-decoded codes, an independent
round-to-nearest-even formula for the encoder, ties, saturation and the
subnormal edge, the absmax element landing on 448, lossless inputs giving the
bf16-path result exactly, and the dequantised error bound.
"""
from __future__ import annotations

import numpy as np

from . import diffattn_ref as ref

E4M3_MAX = 448.0

__all__ = ["E4M3_MAX", "e4m3_table", "e4m3_encode", "absmax_scales", "quantize_qk", "dequantize",
           "diffattn_fwd_qk8"]


def e4m3_table() -> np.ndarray:
    """The value of each of the 256 codes (float64; NaN for the two NaN codes)."""
    vals = np.empty(256, dtype=np.float64)
    for c in range(256):
        s = -1.0 if c & 0x80 else 1.0
        e = (c >> 3) & 0xF
        m = c & 0x7
        if e == 0xF and m == 0x7:
            vals[c] = np.nan
        elif e == 0:
            vals[c] = s * m * 2.0 ** -9
        else:
            vals[c] = s * (1.0 + m / 8.0) * 2.0 ** (e - 7)
    return vals


_TABLE = e4m3_table()
_POS_CODES = np.arange(0x7F)            # 0x00 .. 0x7E: the non-negative finite values, ascending
_POS_VALS = _TABLE[_POS_CODES]


def e4m3_encode(x) -> np.ndarray:
    """Nearest e4m3 code for each element of x (float32 values): ties to the
    even code, magnitudes beyond 448 saturate to +-448, the sign is kept (so
    negative values that round to zero give the code of -0)."""
    x = np.asarray(x, dtype=np.float32).astype(np.float64)
    mag = np.minimum(np.abs(x), E4M3_MAX)
    hi = np.searchsorted(_POS_VALS, mag, side="left")          # first value >= mag
    hi = np.clip(hi, 0, len(_POS_VALS) - 1)
    lo = np.clip(hi - 1, 0, len(_POS_VALS) - 1)
    d_lo = mag - _POS_VALS[lo]
    d_hi = _POS_VALS[hi] - mag
    pick_hi = (d_hi < d_lo) | ((d_hi == d_lo) & (_POS_CODES[hi] % 2 == 0) & (hi != lo))
    code = np.where(pick_hi, _POS_CODES[hi], _POS_CODES[lo]).astype(np.uint8)
    neg = np.signbit(x)
    return np.where(neg, code | np.uint8(0x80), code).astype(np.uint8)


def absmax_scales(t) -> np.ndarray:
    """float32 scales [B, H, 2] of t [B, N, H, 2, d]: absmax of each (b, h, map)
    group divided by 448 in float32 (1 for an all-zero group)."""
    t = np.asarray(t, dtype=np.float32)
    amax = np.abs(t).max(axis=(1, 4))                          # [B, H, 2]
    scale = (amax / np.float32(E4M3_MAX)).astype(np.float32)
    return np.where(amax > 0, scale, np.float32(1.0)).astype(np.float32)


def quantize_qk(t):
    """(codes uint8 [B, N, H, 2, d], scales float32 [B, H, 2]) for t [B, N, H, 2, d]."""
    t = np.asarray(t, dtype=np.float32)
    s = absmax_scales(t)
    ratio = (t / s[:, None, :, :, None]).astype(np.float32)  # float32 division, as the kernel does
    return e4m3_encode(ratio), s


def dequantize(codes, scales) -> np.ndarray:
    """float64 values code * scale, [B, N, H, 2, d]."""
    return _TABLE[np.asarray(codes)] * np.asarray(scales, dtype=np.float64)[:, None, :, :, None]


def diffattn_fwd_qk8(q, k, v, lam: float, lambda_init: float, w, eps: float, causal: bool,
                     rows=None, heads=None, mode: str = "diff") -> np.ndarray:
    """The prefill with queries and keys quantised to e4m3 per (batch, head, map).

    q, k : [B, N, H, 2, d] (the bf16 values the library receives); v : [B, N, H, 2d].
    Same output as ``diffattn_ref.diffattn_fwd`` on the dequantised q and k.
    """
    qc, qs = quantize_qk(q)
    kc, ks = quantize_qk(k)
    return ref.diffattn_fwd(dequantize(qc, qs), dequantize(kc, ks), v, lam, lambda_init, w, eps, causal,
                            rows=rows, heads=heads, mode=mode)
