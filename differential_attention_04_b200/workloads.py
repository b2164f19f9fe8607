"""Seeded synthetic inputs for the prefill and decode workloads.

This module only draws random inputs; it holds none of the method's
arithmetic.  Both the CUDA path and the float64 oracle are fed from it.

Distributions (the shapes of the pages' 3B-13B, up-to-64K-context workloads;
no dataset or trained weight is used):
  * Q, K, V entries i.i.d. N(0, 1), drawn in float32 with ``torch.randn`` from
    a ``torch.Generator`` seeded with ``seed`` on the target device, then
    rounded (round-to-nearest-even) to the storage dtype.  RoPE is treated as
    already applied.
  * lambda vectors lq1, lk1, lq2, lk2: i.i.d. N(0, 0.1) (0.1 = standard
    deviation), float32.
  * RMSNorm weight: all ones ("ones") or N(1, 0.02) ("normal"), float32[2d].
  * Needle (long-context case): for every head h of every batch b, at a seeded
    position p < N-1, K1[b, p, h] = 4 * Q1[b, N-1, h] / |Q1[b, N-1, h]|
    (computed in float32 from the stored query, then rounded); K2 stays noise.
  * Projections (the steps either side of the path): token activations X
    i.i.d. N(0, 1) [B*N, d_model]; weights i.i.d. N(0, 1/d_model) (so the
    projected entries have unit variance), drawn like Q, K, V and rounded to
    bf16: W_qkv [3 * H * 2d, d_model], W_o [d_model, H * 2d].  The 3B-like
    model: d_model = 3072, H = 12, d = 128.
  * Decode: per-sequence KV length L_s ~ U{lmin .. lmax} from
    ``numpy.random.default_rng(seed).integers(lmin, lmax + 1, S)``; sequences
    packed back to back; the cache includes the current token.
"""
from __future__ import annotations

from dataclasses import dataclass

import numpy as np
import torch

# The five workloads: sizes and constants per case.
PREFILL_CASES = {
    "tiny_fp32": dict(B=1, H=2, N=128, d=64, causal=True, dtype="f32", lambda_init=0.2, w="ones"),
    "prefill_3b": dict(B=4, H=12, N=4096, d=128, causal=True, dtype="bf16", lambda_init=0.5, w="normal"),
    "prefill_64k_needle": dict(B=1, H=12, N=65536, d=128, causal=True, dtype="bf16", lambda_init=0.8,
                               w="normal", needle=True),
    "prefill_13b_causal": dict(B=2, H=20, N=8192, d=128, causal=True, dtype="bf16", lambda_init=0.65,
                               w="normal"),
    "prefill_13b_nomask": dict(B=2, H=20, N=8192, d=128, causal=False, dtype="bf16", lambda_init=0.65,
                               w="normal"),
}
DECODE_CASES = {
    "decode_64x12": dict(S=64, H=12, d=128, lmin=1024, lmax=32768, lambda_init=0.5, w="normal"),
}
EPS = 1e-5

_DT = {"bf16": torch.bfloat16, "f32": torch.float32}


@dataclass
class PrefillInputs:
    q: torch.Tensor
    k: torch.Tensor
    v: torch.Tensor
    lq1: torch.Tensor
    lk1: torch.Tensor
    lq2: torch.Tensor
    lk2: torch.Tensor
    rms_w: torch.Tensor
    lambda_init: float
    eps: float
    causal: bool
    needle_pos: list | None = None


@dataclass
class DecodeInputs:
    q: torch.Tensor
    k_cache: torch.Tensor
    v_cache: torch.Tensor
    cu_seqlens: torch.Tensor
    seqlens: np.ndarray
    max_seqlen: int
    lq1: torch.Tensor
    lk1: torch.Tensor
    lq2: torch.Tensor
    lk2: torch.Tensor
    rms_w: torch.Tensor
    lambda_init: float
    eps: float


def _randn(shape, gen, device, dtype, chunk_elems=1 << 28):
    """N(0,1) float32 draws rounded to ``dtype``, generated in chunks to bound temporaries."""
    out = torch.empty(shape, dtype=dtype, device=device)
    flat = out.view(-1)
    n = flat.numel()
    for s in range(0, n, chunk_elems):
        e = min(n, s + chunk_elems)
        flat[s:e] = torch.randn(e - s, generator=gen, device=device, dtype=torch.float32).to(dtype)
    return out


def _lambda_and_w(gen, device, d, w_kind):
    lam = [torch.randn(d, generator=gen, device=device, dtype=torch.float32) * 0.1 for _ in range(4)]
    if w_kind == "ones":
        w = torch.ones(2 * d, dtype=torch.float32, device=device)
    else:
        w = 1.0 + 0.02 * torch.randn(2 * d, generator=gen, device=device, dtype=torch.float32)
    return lam, w


def make_prefill(B, N, H, d, causal=True, dtype="bf16", lambda_init=0.5, w="normal", needle=False,
                 eps=EPS, seed=0, device="cpu") -> PrefillInputs:
    gen = torch.Generator(device=device)
    gen.manual_seed(seed)
    dt = _DT[dtype]
    q = _randn((B, N, H, 2, d), gen, device, dt)
    k = _randn((B, N, H, 2, d), gen, device, dt)
    v = _randn((B, N, H, 2 * d), gen, device, dt)
    lam, wv = _lambda_and_w(gen, device, d, w)
    pos = None
    if needle and N >= 2:
        rng = np.random.default_rng(seed + 1)
        pos = [[int(x) for x in rng.integers(0, N - 1, H)] for _ in range(B)]
        for b in range(B):
            for h in range(H):
                ql = q[b, N - 1, h, 0].float()
                k[b, pos[b][h], h, 0] = (4.0 * ql / ql.norm()).to(dt)
    return PrefillInputs(q, k, v, *lam, wv, float(lambda_init), float(eps), bool(causal), pos)


def make_prefill_case(name: str, seed=0, device="cpu", **override) -> PrefillInputs:
    cfg = dict(PREFILL_CASES[name])
    cfg.update(override)
    return make_prefill(seed=seed, device=device, **cfg)


def make_decode(S, H, d, lmin, lmax, lambda_init=0.5, w="normal", eps=EPS, seed=0, device="cpu",
                seqlens=None) -> DecodeInputs:
    if seqlens is None:
        seqlens = np.random.default_rng(seed).integers(lmin, lmax + 1, S)
    seqlens = np.asarray(seqlens, dtype=np.int64)
    cu = np.concatenate([[0], np.cumsum(seqlens)]).astype(np.int32)
    T = int(cu[-1])
    gen = torch.Generator(device=device)
    gen.manual_seed(seed)
    q = _randn((S, H, 2, d), gen, device, torch.bfloat16)
    kc = _randn((T, H, 2, d), gen, device, torch.bfloat16)
    vc = _randn((T, H, 2 * d), gen, device, torch.bfloat16)
    lam, wv = _lambda_and_w(gen, device, d, w)
    return DecodeInputs(q, kc, vc, torch.from_numpy(cu).to(device), seqlens, int(seqlens.max()), *lam, wv,
                        float(lambda_init), float(eps))


def make_decode_case(name: str, seed=0, device="cpu", **override) -> DecodeInputs:
    cfg = dict(DECODE_CASES[name])
    cfg.update(override)
    return make_decode(seed=seed, device=device, **cfg)


def to_f64(t: torch.Tensor) -> np.ndarray:
    """Exact float64 copy (on the host) of a float32/bf16 tensor."""
    return t.detach().to("cpu", torch.float64).numpy()


PROJ_CASES = {
    "proj_3b": dict(B=4, N=4096, d_model=3072, H=12, d=128),
}


@dataclass
class ProjInputs:
    x: torch.Tensor      # [B*N, d_model]
    w_qkv: torch.Tensor  # [3 * H * 2d, d_model]
    w_o: torch.Tensor    # [d_model, H * 2d]
    B: int
    N: int
    H: int
    d: int


def make_proj(B, N, d_model, H, d, seed=0, device="cpu") -> ProjInputs:
    gen = torch.Generator(device=device)
    gen.manual_seed(seed)
    x = _randn((B * N, d_model), gen, device, torch.bfloat16)
    w_qkv = _randn((3 * H * 2 * d, d_model), gen, device, torch.float32)
    w_qkv = (w_qkv / float(np.sqrt(d_model))).to(torch.bfloat16)
    w_o = _randn((d_model, H * 2 * d), gen, device, torch.float32)
    w_o = (w_o / float(np.sqrt(H * 2 * d))).to(torch.bfloat16)
    return ProjInputs(x, w_qkv, w_o, B, N, H, d)


def make_proj_case(name: str, seed=0, device="cpu") -> ProjInputs:
    return make_proj(seed=seed, device=device, **PROJ_CASES[name])
