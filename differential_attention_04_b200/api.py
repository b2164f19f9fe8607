"""Python binding of the C ABI in include/diffattn.h.

Argument marshalling only: every step of the computation runs in the CUDA
library.  Tensors are passed by device pointer on the current torch stream;
the functions return immediately (stream-ordered), like the C calls.
"""
from __future__ import annotations

import ctypes

import torch

from ._lib import lib

OK, ERR_INVALID_ARG, ERR_UNSUPPORTED, ERR_CUDA, ERR_TIMEOUT, ERR_WORKSPACE, ERR_BOUNDS = range(7)
F32, BF16 = 0, 1
# how the two maps are combined: softmax(S1) + c softmax(S2), c = -lambda, 0, +lambda
MODE_DIFF, MODE_LAMBDA_ZERO, MODE_SUM = 0, 1, 2


class DiffAttnError(RuntimeError):
    def __init__(self, fn: str, status: int):
        msg = lib().diffattn_status_string(status).decode()
        super().__init__(f"{fn} failed: {msg} (status {status})")
        self.status = status


def _check(fn: str, status: int) -> None:
    if status != OK:
        raise DiffAttnError(fn, status)


def _ptr(t: torch.Tensor | None) -> int | None:
    return None if t is None else t.data_ptr()


def _dev(*ts: torch.Tensor) -> torch.device:
    """The one CUDA device all of `ts` live on (every tensor contiguous)."""
    dev = None
    for t in ts:
        if not t.is_cuda:
            raise ValueError("all tensors must be CUDA tensors")
        if not t.is_contiguous():
            raise ValueError("all tensors must be contiguous")
        if dev is None:
            dev = t.device
        elif t.device != dev:
            raise ValueError(f"all tensors must be on one device (found {dev} and {t.device})")
    return dev


def _launch(name: str, tensors, *args) -> None:
    """Call the C entry point `name` with `args` and the current stream of the
    device that `tensors` (every tensor the call reads or writes) live on, with
    that device current: the library launches on the current device."""
    dev = _dev(*tensors)
    with torch.cuda.device(dev):
        status = getattr(lib(), name)(*args, torch.cuda.current_stream(dev).cuda_stream)
    _check(name, status)


# Shape and dtype checks run before the device check, so that every tensor the
# kernels index is known to be large enough before its pointer is passed on.
def _need(cond: bool, msg: str) -> None:
    if not cond:
        raise ValueError(msg)


def _scalar_f32(name: str, t: torch.Tensor) -> None:
    _need(t.dtype == torch.float32 and t.numel() >= 1, f"{name} must be a float32 device scalar")


def _f32(name: str, t: torch.Tensor, n: int) -> None:
    _need(t.dtype == torch.float32 and t.numel() == n, f"{name} must be float32 with {n} elements")


def _like(name: str, t: torch.Tensor, shape, dtype) -> None:
    _need(tuple(t.shape) == tuple(shape) and t.dtype == dtype, f"{name} must be {dtype} of shape {tuple(shape)}")


def _qkv(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, dy: torch.Tensor | None = None):
    """(B, N, H, d) of q, k [B, N, H, 2, d] and v (and dy) [B, N, H, 2d]."""
    _need(q.dim() == 5 and q.shape[3] == 2 and k.shape == q.shape,
          "q and k must be [B, N, H, 2, d] of one shape")
    B, N, H, _, d = q.shape
    _need(tuple(v.shape) == (B, N, H, 2 * d), "v must be [B, N, H, 2d]")
    _need(dy is None or dy.shape == v.shape, "dy must have v's shape")
    return B, N, H, d


def diffattn_lambda(lq1: torch.Tensor, lk1: torch.Tensor, lq2: torch.Tensor, lk2: torch.Tensor,
                    lambda_init: float, out: torch.Tensor | None = None) -> torch.Tensor:
    """lambda = exp(lq1 . lk1) - exp(lq2 . lk2) + lambda_init, as a device fp32 scalar (shape [1])."""
    for name, t in (("lq1", lq1), ("lk1", lk1), ("lq2", lq2), ("lk2", lk2)):
        _f32(name, t, lq1.numel())
    if out is None:
        out = torch.empty(1, dtype=torch.float32, device=lq1.device)
    _scalar_f32("out", out)
    _launch("diffattn_lambda", (lq1, lk1, lq2, lk2, out),
            _ptr(lq1), _ptr(lk1), _ptr(lq2), _ptr(lk2), lq1.numel(), float(lambda_init), _ptr(out))
    return out


def diffattn_fwd(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, lam: torch.Tensor, lambda_init: float,
                 rms_w: torch.Tensor, eps: float = 1e-5, causal: bool = True,
                 out: torch.Tensor | None = None, mode: int = MODE_DIFF) -> torch.Tensor:
    """Prefill.  q, k: [B, N, H, 2, d]; v: [B, N, H, 2d]; lam: device fp32 scalar; rms_w: fp32 [2d].

    ``mode`` (MODE_DIFF, MODE_LAMBDA_ZERO, MODE_SUM) picks the combination of
    the two maps; MODE_DIFF is the differential attention itself."""
    B, N, H, d = _qkv(q, k, v)
    if q.dtype == torch.bfloat16:
        dt = BF16
    elif q.dtype == torch.float32:
        dt = F32
    else:
        raise ValueError("dtype must be bfloat16 or float32")
    if k.dtype != q.dtype or v.dtype != q.dtype:
        raise ValueError("q, k, v must share one dtype")
    _scalar_f32("lam", lam)
    _f32("rms_w", rms_w, 2 * d)
    if out is None:
        out = torch.empty_like(v)
    _like("out", out, v.shape, v.dtype)
    ts = (q, k, v, lam, rms_w, out)
    if mode == MODE_DIFF:
        _launch("diffattn_fwd", ts, _ptr(q), _ptr(k), _ptr(v), _ptr(out), dt, B, N, H, d, int(bool(causal)),
                _ptr(lam), float(lambda_init), _ptr(rms_w), float(eps))
    else:
        _launch("diffattn_fwd_mode", ts, _ptr(q), _ptr(k), _ptr(v), _ptr(out), dt, B, N, H, d, int(bool(causal)),
                _ptr(lam), float(lambda_init), _ptr(rms_w), float(eps), int(mode))
    return out


def quantize_qk(x: torch.Tensor, codes: torch.Tensor | None = None,
                scales: torch.Tensor | None = None) -> tuple[torch.Tensor, torch.Tensor]:
    """e4m3 codes (uint8, x's shape) and float32 scales [B, H, 2] of a bf16 q or k [B, N, H, 2, d]:
    one absmax scale per (batch, head, map)."""
    if x.dtype != torch.bfloat16 or x.dim() != 5 or x.shape[3] != 2:
        raise ValueError("x must be bfloat16 [B, N, H, 2, d]")
    B, N, H, _, d = x.shape
    if codes is None:
        codes = torch.empty(x.shape, dtype=torch.uint8, device=x.device)
    if scales is None:
        scales = torch.empty((B, H, 2), dtype=torch.float32, device=x.device)
    if codes.shape != x.shape or codes.dtype != torch.uint8 or scales.numel() != B * H * 2 or \
            scales.dtype != torch.float32:
        raise ValueError("codes must be uint8 like x and scales float32 [B, H, 2]")
    _launch("diffattn_quantize_qk", (x, codes, scales),
            _ptr(x), B, N, H, d, _ptr(codes), _ptr(scales))
    return codes, scales


def _lowbit_rest(B, N, H, d, q_scales, k_scales, v, lam, rms_w) -> None:
    _f32("q_scales", q_scales, B * H * 2)
    _f32("k_scales", k_scales, B * H * 2)
    _like("v", v, (B, N, H, 2 * d), torch.bfloat16)
    _scalar_f32("lam", lam)
    _f32("rms_w", rms_w, 2 * d)


def diffattn_fwd_qk8(q_codes: torch.Tensor, q_scales: torch.Tensor, k_codes: torch.Tensor, k_scales: torch.Tensor,
                     v: torch.Tensor, lam: torch.Tensor, lambda_init: float, rms_w: torch.Tensor, eps: float = 1e-5,
                     causal: bool = True, out: torch.Tensor | None = None, mode: int = MODE_DIFF) -> torch.Tensor:
    """Prefill with e4m3 queries and keys (as quantize_qk returns them); v, out: bf16 [B, N, H, 2d]."""
    if q_codes.dtype != torch.uint8 or k_codes.dtype != torch.uint8 or k_codes.shape != q_codes.shape or \
            q_codes.dim() != 5 or q_codes.shape[3] != 2:
        raise ValueError("q_codes, k_codes must be uint8 [B, N, H, 2, d]")
    B, N, H, _, d = q_codes.shape
    _lowbit_rest(B, N, H, d, q_scales, k_scales, v, lam, rms_w)
    if out is None:
        out = torch.empty_like(v)
    _like("out", out, v.shape, torch.bfloat16)
    _launch("diffattn_fwd_qk8", (q_codes, q_scales, k_codes, k_scales, v, lam, rms_w, out),
            _ptr(q_codes), _ptr(q_scales), _ptr(k_codes), _ptr(k_scales), _ptr(v), _ptr(out), B, N, H, d,
            int(bool(causal)), _ptr(lam), float(lambda_init), _ptr(rms_w), float(eps), int(mode))
    return out


def quantize_qk4(x: torch.Tensor, codes: torch.Tensor | None = None,
                 scales: torch.Tensor | None = None) -> tuple[torch.Tensor, torch.Tensor]:
    """e2m1 codes, two per byte (uint8 [B, N, H, 2, d / 2], channel 2j in the low nibble), and float32
    scales [B, H, 2] of a bf16 q or k [B, N, H, 2, d]: one absmax scale per (batch, head, map)."""
    if x.dtype != torch.bfloat16 or x.dim() != 5 or x.shape[3] != 2:
        raise ValueError("x must be bfloat16 [B, N, H, 2, d]")
    B, N, H, _, d = x.shape
    if d % 8:
        raise ValueError("d must be a multiple of 8")
    shape = (B, N, H, 2, d // 2)
    if codes is None:
        codes = torch.empty(shape, dtype=torch.uint8, device=x.device)
    if scales is None:
        scales = torch.empty((B, H, 2), dtype=torch.float32, device=x.device)
    if tuple(codes.shape) != shape or codes.dtype != torch.uint8 or scales.numel() != B * H * 2 or \
            scales.dtype != torch.float32:
        raise ValueError("codes must be uint8 [B, N, H, 2, d / 2] and scales float32 [B, H, 2]")
    _launch("diffattn_quantize_qk4", (x, codes, scales),
            _ptr(x), B, N, H, d, _ptr(codes), _ptr(scales))
    return codes, scales


def diffattn_fwd_qk4(q_codes: torch.Tensor, q_scales: torch.Tensor, k_codes: torch.Tensor, k_scales: torch.Tensor,
                     v: torch.Tensor, lam: torch.Tensor, lambda_init: float, rms_w: torch.Tensor, eps: float = 1e-5,
                     causal: bool = True, out: torch.Tensor | None = None, mode: int = MODE_DIFF) -> torch.Tensor:
    """Prefill with e2m1 queries and keys (as quantize_qk4 returns them, [B, N, H, 2, d / 2]);
    v, out: bf16 [B, N, H, 2d]."""
    if q_codes.dtype != torch.uint8 or k_codes.dtype != torch.uint8 or k_codes.shape != q_codes.shape or \
            q_codes.dim() != 5 or q_codes.shape[3] != 2:
        raise ValueError("q_codes, k_codes must be uint8 [B, N, H, 2, d / 2]")
    B, N, H, _, half = q_codes.shape
    d = 2 * half
    _lowbit_rest(B, N, H, d, q_scales, k_scales, v, lam, rms_w)
    if out is None:
        out = torch.empty_like(v)
    _like("out", out, v.shape, torch.bfloat16)
    _launch("diffattn_fwd_qk4", (q_codes, q_scales, k_codes, k_scales, v, lam, rms_w, out),
            _ptr(q_codes), _ptr(q_scales), _ptr(k_codes), _ptr(k_scales), _ptr(v), _ptr(out), B, N, H, d,
            int(bool(causal)), _ptr(lam), float(lambda_init), _ptr(rms_w), float(eps), int(mode))
    return out


def bwd_workspace_size(B: int, N: int, H: int, d: int) -> int:
    return int(lib().diffattn_bwd_workspace_size(B, N, H, d))


def diffattn_bwd(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, dy: torch.Tensor, lam: torch.Tensor,
                 lambda_init: float, rms_w: torch.Tensor, eps: float = 1e-5, causal: bool = True,
                 mode: int = MODE_DIFF, workspace: torch.Tensor | None = None):
    """Backward of the prefill: (dq, dk, dv, dlambda, drms_w), float32, for the upstream gradient dy
    (shaped like v).  q, k, v, dy share one dtype (bfloat16 or float32)."""
    B, N, H, d = _qkv(q, k, v, dy)
    dt = BF16 if q.dtype == torch.bfloat16 else F32 if q.dtype == torch.float32 else None
    if dt is None or any(t.dtype != q.dtype for t in (k, v, dy)):
        raise ValueError("q, k, v, dy must share one dtype, bfloat16 or float32")
    _scalar_f32("lam", lam)
    _f32("rms_w", rms_w, 2 * d)
    _dev(q, k, v, dy, lam, rms_w)
    f32 = dict(dtype=torch.float32, device=q.device)
    dq, dk, dv = torch.empty(q.shape, **f32), torch.empty(k.shape, **f32), torch.empty(v.shape, **f32)
    dlam, dw = torch.empty(1, **f32), torch.empty(2 * d, **f32)
    need = bwd_workspace_size(B, N, H, d)
    if workspace is None:
        workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
    _launch("diffattn_bwd", (q, k, v, dy, lam, rms_w, dq, dk, dv, dlam, dw, workspace),
            _ptr(q), _ptr(k), _ptr(v), _ptr(dy), dt, B, N, H, d, int(bool(causal)), _ptr(lam), float(lambda_init),
            _ptr(rms_w), float(eps), int(mode), _ptr(dq), _ptr(dk), _ptr(dv), _ptr(dlam), _ptr(dw), _ptr(workspace),
            workspace.numel() * workspace.element_size())
    return dq, dk, dv, dlam, dw


def _grads_out(out, q: torch.Tensor, v: torch.Tensor, d: int):
    """The five float32 gradient outputs (dq, dk, dv, dlambda, drms_w), allocated when `out` is None."""
    f32 = dict(dtype=torch.float32, device=q.device)
    if out is None:
        return (torch.empty(q.shape, **f32), torch.empty(q.shape, **f32), torch.empty(v.shape, **f32),
                torch.empty(1, **f32), torch.empty(2 * d, **f32))
    _need(len(out) == 5, "out must hold (dq, dk, dv, dlambda, drms_w)")
    dq, dk, dv, dlam, dw = out
    _like("dq", dq, q.shape, torch.float32)
    _like("dk", dk, q.shape, torch.float32)
    _like("dv", dv, v.shape, torch.float32)
    _scalar_f32("dlambda", dlam)
    _f32("drms_w", dw, 2 * d)
    _dev(dq, dk, dv, dlam, dw)
    return out


def bwd_tc_workspace_size(B: int, N: int, H: int, d: int) -> int:
    return int(lib().diffattn_bwd_tc_workspace_size(B, N, H, d))


def diffattn_bwd_tc(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, dy: torch.Tensor, lam: torch.Tensor,
                    lambda_init: float, rms_w: torch.Tensor, eps: float = 1e-5, causal: bool = True,
                    mode: int = MODE_DIFF, workspace: torch.Tensor | None = None, out=None):
    """Tensor-core backward of the prefill: (dq, dk, dv, dlambda, drms_w), float32, for bfloat16 q, k, v and
    upstream gradient dy (shaped like v), d = 64 or 128.  `out` may hold preallocated outputs in that order."""
    B, N, H, d = _qkv(q, k, v, dy)
    if any(t.dtype != torch.bfloat16 for t in (q, k, v, dy)):
        raise ValueError("q, k, v, dy must be bfloat16")
    _scalar_f32("lam", lam)
    _f32("rms_w", rms_w, 2 * d)
    dq, dk, dv, dlam, dw = _grads_out(out, q, v, d)
    _dev(q, k, v, dy, lam, rms_w)
    if workspace is None:
        workspace = torch.empty(bwd_tc_workspace_size(B, N, H, d), dtype=torch.uint8, device=q.device)
    _launch("diffattn_bwd_tc", (q, k, v, dy, lam, rms_w, dq, dk, dv, dlam, dw, workspace),
            _ptr(q), _ptr(k), _ptr(v), _ptr(dy), B, N, H, d, int(bool(causal)), _ptr(lam), float(lambda_init),
            _ptr(rms_w), float(eps), int(mode), _ptr(dq), _ptr(dk), _ptr(dv), _ptr(dlam), _ptr(dw), _ptr(workspace),
            workspace.numel() * workspace.element_size())
    return dq, dk, dv, dlam, dw


def diffattn_fwd_train(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, lam: torch.Tensor, lambda_init: float,
                       rms_w: torch.Tensor, eps: float = 1e-5, causal: bool = True, mode: int = MODE_DIFF,
                       workspace: torch.Tensor | None = None, out: torch.Tensor | None = None):
    """Training forward: (o, workspace).  o as diffattn_fwd; the workspace (bwd_tc_workspace_size bytes) holds
    what diffattn_bwd_tc_saved needs for the same q, k, v, lambda and mask."""
    B, N, H, d = _qkv(q, k, v)
    if any(t.dtype != torch.bfloat16 for t in (q, k, v)):
        raise ValueError("q, k, v must be bfloat16")
    _scalar_f32("lam", lam)
    _f32("rms_w", rms_w, 2 * d)
    if out is None:
        out = torch.empty_like(v)
    _like("out", out, v.shape, torch.bfloat16)
    if workspace is None:
        workspace = torch.empty(bwd_tc_workspace_size(B, N, H, d), dtype=torch.uint8, device=q.device)
    _launch("diffattn_fwd_train", (q, k, v, lam, rms_w, out, workspace),
            _ptr(q), _ptr(k), _ptr(v), _ptr(out), B, N, H, d, int(bool(causal)), _ptr(lam), float(lambda_init),
            _ptr(rms_w), float(eps), int(mode), _ptr(workspace), workspace.numel() * workspace.element_size())
    return out, workspace


def diffattn_bwd_tc_saved(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, dy: torch.Tensor, lam: torch.Tensor,
                          lambda_init: float, rms_w: torch.Tensor, eps: float, causal: bool, mode: int,
                          workspace: torch.Tensor, out=None):
    """diffattn_bwd_tc using the statistics diffattn_fwd_train left in `workspace`."""
    B, N, H, d = _qkv(q, k, v, dy)
    if any(t.dtype != torch.bfloat16 for t in (q, k, v, dy)):
        raise ValueError("q, k, v, dy must be bfloat16")
    _scalar_f32("lam", lam)
    _f32("rms_w", rms_w, 2 * d)
    dq, dk, dv, dlam, dw = _grads_out(out, q, v, d)
    _launch("diffattn_bwd_tc_saved", (q, k, v, dy, lam, rms_w, dq, dk, dv, dlam, dw, workspace),
            _ptr(q), _ptr(k), _ptr(v), _ptr(dy), B, N, H, d, int(bool(causal)), _ptr(lam), float(lambda_init),
            _ptr(rms_w), float(eps), int(mode), _ptr(dq), _ptr(dk), _ptr(dv), _ptr(dlam), _ptr(dw), _ptr(workspace),
            workspace.numel() * workspace.element_size())
    return dq, dk, dv, dlam, dw


def rope_table(N: int, d: int, base: float = 10000.0, device=None) -> torch.Tensor:
    """(cos, sin) of n * base^(-2j/d) for n < N, j < d/2: float32 [N, d/2, 2] on the device."""
    t = torch.empty((N, d // 2, 2), dtype=torch.float32, device=device or torch.device("cuda"))
    _launch("diffattn_rope_table", (t,), int(N), int(d), float(base), _ptr(t))
    return t


def qkv_proj(x: torch.Tensor, w_qkv: torch.Tensor, B: int, N: int, H: int, d: int, rope: torch.Tensor | None = None,
             out=None):
    """[Q | K | V] = x w_qkv^T with RoPE (from rope_table) on Q and K: q, k [B, N, H, 2, d], v [B, N, H, 2d],
    bfloat16.  x: bfloat16 [B*N, d_model]; w_qkv: bfloat16 [3*H*2d, d_model] (W_q; W_k; W_v)."""
    dm = x.shape[-1]
    if x.dtype != torch.bfloat16 or w_qkv.dtype != torch.bfloat16 or x.numel() != B * N * dm:
        raise ValueError("x must be bfloat16 [B*N, d_model]")
    if tuple(w_qkv.shape) != (3 * H * 2 * d, dm):
        raise ValueError("w_qkv must be bfloat16 [3*H*2d, d_model]")
    if rope is not None and (rope.dtype != torch.float32 or rope.dim() != 3 or rope.shape[0] < N or
                             rope.shape[1] * 2 != d or rope.shape[2] != 2):
        raise ValueError("rope must come from rope_table(>= N, d)")
    if out is None:
        bf = dict(dtype=torch.bfloat16, device=x.device)
        out = (torch.empty((B, N, H, 2, d), **bf), torch.empty((B, N, H, 2, d), **bf), torch.empty((B, N, H, 2 * d), **bf))
    _need(len(out) == 3, "out must hold (q, k, v)")
    q, k, v = out
    _like("q", q, (B, N, H, 2, d), torch.bfloat16)
    _like("k", k, (B, N, H, 2, d), torch.bfloat16)
    _like("v", v, (B, N, H, 2 * d), torch.bfloat16)
    _launch("diffattn_qkv_proj", (x, w_qkv, q, k, v, *(() if rope is None else (rope,))),
            _ptr(x), _ptr(w_qkv), B, N, dm, H, d, _ptr(rope) if rope is not None else None, _ptr(q), _ptr(k), _ptr(v))
    return q, k, v


def out_proj(o: torch.Tensor, w_o: torch.Tensor, out: torch.Tensor | None = None) -> torch.Tensor:
    """y = o w_o^T: o bfloat16 [M, K] (or [B, N, H, 2d]), w_o bfloat16 [n_out, K] -> y bfloat16 [M, n_out]."""
    if w_o.dim() != 2 or o.dtype != torch.bfloat16 or w_o.dtype != torch.bfloat16 or o.numel() % w_o.shape[1]:
        raise ValueError("o and w_o must be bfloat16 with o's rows of width w_o.shape[1]")
    K = w_o.shape[1]
    M, n_out = o.numel() // K, w_o.shape[0]
    if out is None:
        out = torch.empty((M, n_out), dtype=torch.bfloat16, device=o.device)
    _like("out", out, (M, n_out), torch.bfloat16)
    _launch("diffattn_out_proj", (o, w_o, out),
            _ptr(o), _ptr(w_o), M, K, n_out, _ptr(out))
    return out


def diffattn_lambda_bwd(lq1: torch.Tensor, lk1: torch.Tensor, lq2: torch.Tensor, lk2: torch.Tensor,
                        dlam: torch.Tensor):
    """Gradients (dlq1, dlk1, dlq2, dlk2) of the lambda re-parameterisation for a device dlambda."""
    for name, t in (("lq1", lq1), ("lk1", lk1), ("lq2", lq2), ("lk2", lk2)):
        _f32(name, t, lq1.numel())
    _scalar_f32("dlam", dlam)
    _dev(lq1, lk1, lq2, lk2, dlam)
    outs = [torch.empty_like(t) for t in (lq1, lk1, lq2, lk2)]
    _launch("diffattn_lambda_bwd", (lq1, lk1, lq2, lk2, dlam, *outs),
            _ptr(lq1), _ptr(lk1), _ptr(lq2), _ptr(lk2), lq1.numel(), _ptr(dlam), *[_ptr(t) for t in outs])
    return tuple(outs)


def _decode_shapes(q, k_cache, v_cache, cu_seqlens, lam, rms_w):
    """(S, H, d) of a decode call; checks every shape and dtype the kernels rely on (the offsets in
    cu_seqlens are device data: the caller keeps them within the cache)."""
    _need(q.dim() == 4 and q.shape[2] == 2, "q must be [S, H, 2, d]")
    S, H, _, d = q.shape
    _need(k_cache.dim() == 4 and tuple(k_cache.shape[1:]) == (H, 2, d) and k_cache.dtype == q.dtype,
          "k_cache must be [T, H, 2, d] of q's dtype")
    _like("v_cache", v_cache, (k_cache.shape[0], H, 2 * d), q.dtype)
    _need(cu_seqlens.dtype == torch.int32 and cu_seqlens.numel() == S + 1,
          "cu_seqlens must be int32 with S + 1 entries")
    _scalar_f32("lam", lam)
    _f32("rms_w", rms_w, 2 * d)
    _dev(q, k_cache, v_cache, cu_seqlens, lam, rms_w)
    return S, H, d


def decode_workspace_size(S: int, H: int, d: int, max_seqlen: int) -> int:
    return int(lib().diffattn_decode_workspace_size(S, H, d, max_seqlen))


def diffattn_decode(q: torch.Tensor, k_cache: torch.Tensor, v_cache: torch.Tensor, cu_seqlens: torch.Tensor,
                    max_seqlen: int, lam: torch.Tensor, lambda_init: float, rms_w: torch.Tensor,
                    eps: float = 1e-5, workspace: torch.Tensor | None = None,
                    out: torch.Tensor | None = None, mode: int = MODE_DIFF) -> torch.Tensor:
    """Decode.  q: [S, H, 2, d]; k_cache: [T, H, 2, d]; v_cache: [T, H, 2d]; cu_seqlens: int32 [S + 1].
    ``mode`` as in diffattn_fwd."""
    S, H, d = _decode_shapes(q, k_cache, v_cache, cu_seqlens, lam, rms_w)
    need = decode_workspace_size(S, H, d, max_seqlen)
    if workspace is None:
        workspace = torch.empty(max(need, 16), dtype=torch.uint8, device=q.device)
    if out is None:
        out = torch.empty((S, H, 2 * d), dtype=q.dtype, device=q.device)
    _like("out", out, (S, H, 2 * d), q.dtype)
    ts = (q, k_cache, v_cache, cu_seqlens, lam, rms_w, workspace, out)
    ws_bytes = workspace.numel() * workspace.element_size()
    if mode == MODE_DIFF:
        _launch("diffattn_decode", ts, _ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(cu_seqlens), int(max_seqlen),
                _ptr(out), S, H, d, _ptr(lam), float(lambda_init), _ptr(rms_w), float(eps), _ptr(workspace), ws_bytes)
    else:
        _launch("diffattn_decode_mode", ts, _ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(cu_seqlens),
                int(max_seqlen), _ptr(out), S, H, d, _ptr(lam), float(lambda_init), _ptr(rms_w), float(eps),
                int(mode), _ptr(workspace), ws_bytes)
    return out


NOALLOC_SCRATCH_BYTES = 16 << 20  # DIFFATTN_DECODE_NOALLOC_SCRATCH_BYTES


def diffattn_decode_noalloc(q: torch.Tensor, k_cache: torch.Tensor, v_cache: torch.Tensor,
                            cu_seqlens: torch.Tensor, max_seqlen: int, lam: torch.Tensor, lambda_init: float,
                            rms_w: torch.Tensor, eps: float = 1e-5, out: torch.Tensor | None = None) -> torch.Tensor:
    """Decode without a workspace, for callers that may not allocate device memory.

    The library's built-in 16 MiB device scratch replaces the workspace; calls
    that overlap on the GPU share it and race.  Pass ``out`` to keep this call
    free of allocations on the Python side as well.
    """
    S, H, d = _decode_shapes(q, k_cache, v_cache, cu_seqlens, lam, rms_w)
    if out is None:
        out = torch.empty((S, H, 2 * d), dtype=q.dtype, device=q.device)
    _like("out", out, (S, H, 2 * d), q.dtype)
    _launch("diffattn_decode_noalloc", (q, k_cache, v_cache, cu_seqlens, lam, rms_w, out),
            _ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(cu_seqlens), int(max_seqlen), _ptr(out), S, H, d,
            _ptr(lam), float(lambda_init), _ptr(rms_w), float(eps))
    return out


def device_status() -> int:
    """Synchronise the device and return (and clear) the kernels' status word."""
    v = ctypes.c_int(0)
    _check("diffattn_device_status", lib().diffattn_device_status(ctypes.byref(v)))
    return v.value


def set_wait_limit_ns(limit_ns: int) -> None:
    _check("diffattn_set_wait_limit_ns", lib().diffattn_set_wait_limit_ns(int(limit_ns)))
