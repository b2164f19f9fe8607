"""The Python binding checks every shape and dtype the kernels index before
any pointer reaches the library (no GPU needed).

Valid call patterns -- those of the GPU tests, the bench and the smoke run,
built on the CPU by the same generators -- must pass every check and stop
only at the device check; each kind of bad argument (a short weight vector,
a mis-shaped output, too few scales, a half-precision lambda, a cache of the
wrong width) must be rejected with a message naming it.
"""
import pytest
import torch

from differential_attention_04_b200 import api
from differential_attention_04_b200 import workloads as wl

ON_DEVICE = "must be CUDA tensors"


def _cpu_only(fn, *a, **k):
    with pytest.raises(ValueError, match=ON_DEVICE):
        fn(*a, **k)


def _rejects(match, fn, *a, **k):
    with pytest.raises(ValueError, match=match):
        fn(*a, **k)


@pytest.fixture(scope="module")
def pre():
    return wl.make_prefill(2, 40, 3, 64, causal=True, dtype="bf16", seed=1, device="cpu")


def _lam():
    return torch.zeros(1, dtype=torch.float32)


def test_valid_patterns_reach_the_device_check(pre):
    B, N, H, _, d = pre.q.shape
    lam = _lam()
    f32 = dict(dtype=torch.float32)
    _cpu_only(api.diffattn_lambda, pre.lq1, pre.lk1, pre.lq2, pre.lk2, 0.5)
    _cpu_only(api.diffattn_lambda, pre.lq1, pre.lk1, pre.lq2, pre.lk2, 0.5, out=lam)
    _cpu_only(api.diffattn_fwd, pre.q, pre.k, pre.v, lam, 0.5, pre.rms_w, 1e-5, True)
    _cpu_only(api.diffattn_fwd, pre.q, pre.k, pre.v, lam, 0.5, pre.rms_w, 1e-5, True, out=torch.empty_like(pre.v),
              mode=api.MODE_SUM)
    _cpu_only(api.quantize_qk, pre.q)
    _cpu_only(api.quantize_qk4, pre.q)
    codes8 = torch.zeros(pre.q.shape, dtype=torch.uint8)
    codes4 = torch.zeros(pre.q.shape[:-1] + (d // 2,), dtype=torch.uint8)
    sc = torch.ones((B, H, 2), **f32)
    _cpu_only(api.diffattn_fwd_qk8, codes8, sc, codes8, sc, pre.v, lam, 0.5, pre.rms_w, 1e-5, True,
              out=torch.empty_like(pre.v))
    _cpu_only(api.diffattn_fwd_qk4, codes4, sc, codes4, sc, pre.v, lam, 0.5, pre.rms_w, 1e-5, True)
    _cpu_only(api.quantize_qk, pre.q, codes8, sc)  # into the caller's buffers, as the bench loop does
    _cpu_only(api.quantize_qk4, pre.q, codes4, sc)
    _cpu_only(api.diffattn_fwd_qk4, codes4, sc, codes4, sc, pre.v, lam, 0.5, pre.rms_w, 1e-5, True,
              out=torch.empty_like(pre.v))
    dy = torch.zeros_like(pre.v)
    _cpu_only(api.diffattn_bwd, pre.q, pre.k, pre.v, dy, lam, 0.5, pre.rms_w)
    _cpu_only(api.diffattn_bwd, pre.q, pre.k, pre.v, dy, lam, 0.5, pre.rms_w, 1e-5, True,
              workspace=torch.empty(64, dtype=torch.uint8))
    f32in = wl.make_prefill(1, 12, 2, 48, causal=False, dtype="f32", seed=3, device="cpu")
    _cpu_only(api.diffattn_fwd, f32in.q, f32in.k, f32in.v, lam, 0.5, f32in.rms_w, 1e-5, False)
    _cpu_only(api.diffattn_bwd, f32in.q, f32in.k, f32in.v, torch.zeros_like(f32in.v), lam, 0.5, f32in.rms_w)
    outs = (torch.empty(pre.q.shape, **f32), torch.empty(pre.k.shape, **f32), torch.empty(pre.v.shape, **f32),
            torch.empty(1, **f32), torch.empty(2 * d, **f32))
    ws = torch.empty(64, dtype=torch.uint8)
    _cpu_only(api.diffattn_bwd_tc, pre.q, pre.k, pre.v, dy, lam, 0.5, pre.rms_w, 1e-5, True, workspace=ws, out=outs)
    _cpu_only(api.diffattn_fwd_train, pre.q, pre.k, pre.v, lam, 0.5, pre.rms_w, 1e-5, True, workspace=ws,
              out=torch.empty_like(pre.v))
    _cpu_only(api.diffattn_bwd_tc_saved, pre.q, pre.k, pre.v, dy, lam, 0.5, pre.rms_w, 1e-5, True, api.MODE_DIFF,
              ws, out=outs)
    _cpu_only(api.diffattn_lambda_bwd, pre.lq1, pre.lk1, pre.lq2, pre.lk2, torch.tensor([1.37]))
    pj = wl.make_proj(1, 24, 96, 2, 16, seed=2, device="cpu")
    rope = torch.zeros((24, 8, 2), **f32)
    _cpu_only(api.qkv_proj, pj.x, pj.w_qkv, 1, 24, 2, 16, rope)
    _cpu_only(api.qkv_proj, pj.x, pj.w_qkv, 1, 24, 2, 16, None)
    v = torch.zeros((1, 24, 2, 32), dtype=torch.bfloat16)
    _cpu_only(api.out_proj, v, pj.w_o, out=torch.empty((24, 96), dtype=torch.bfloat16))
    dec = wl.make_decode(3, 2, 128, 0, 0, seqlens=[1, 60, 110], seed=1, device="cpu")
    _cpu_only(api.diffattn_decode, dec.q, dec.k_cache, dec.v_cache, dec.cu_seqlens, dec.max_seqlen, lam, 0.5,
              dec.rms_w, 1e-5, workspace=torch.empty(16, dtype=torch.uint8),
              out=torch.empty((3, 2, 256), dtype=torch.bfloat16))
    _cpu_only(api.diffattn_decode_noalloc, dec.q, dec.k_cache, dec.v_cache, dec.cu_seqlens, dec.max_seqlen, lam,
              0.5, dec.rms_w)
    # a single query row against its own prefix as a cache, as the decode-vs-prefill test does
    _cpu_only(api.diffattn_decode, pre.q[0, 9:10].contiguous(), pre.k[0].contiguous(), pre.v[0].contiguous(),
              torch.tensor([0, 10], dtype=torch.int32), 10, lam, 0.5, pre.rms_w)


def test_bad_arguments_are_named(pre):
    B, N, H, _, d = pre.q.shape
    lam = _lam()
    f32 = dict(dtype=torch.float32)
    short_w = pre.rms_w[:d].clone()
    _rejects("rms_w", api.diffattn_fwd, pre.q, pre.k, pre.v, lam, 0.5, short_w)
    _rejects("lam", api.diffattn_fwd, pre.q, pre.k, pre.v, lam.to(torch.bfloat16), 0.5, pre.rms_w)
    _rejects("out", api.diffattn_fwd, pre.q, pre.k, pre.v, lam, 0.5, pre.rms_w,
             out=torch.empty((B, N, H, d), dtype=torch.bfloat16))
    _rejects("out", api.diffattn_fwd, pre.q, pre.k, pre.v, lam, 0.5, pre.rms_w,
             out=torch.empty(pre.v.shape, dtype=torch.float32))
    _rejects("v must be", api.diffattn_fwd, pre.q, pre.k, pre.v[..., :d].contiguous(), lam, 0.5, pre.rms_w)
    _rejects("q and k", api.diffattn_fwd, pre.q, pre.k[:, :-1].contiguous(), pre.v, lam, 0.5, pre.rms_w)
    _rejects("lq2", api.diffattn_lambda, pre.lq1, pre.lk1, pre.lq2[:-1].clone(), pre.lk2, 0.5)
    codes4 = torch.zeros(pre.q.shape[:-1] + (d // 2,), dtype=torch.uint8)
    sc = torch.ones((B, H, 2), **f32)
    _rejects("k_scales", api.diffattn_fwd_qk4, codes4, sc, codes4, sc[:1].clone(), pre.v, lam, 0.5, pre.rms_w)
    _rejects("q_scales", api.diffattn_fwd_qk8, torch.zeros(pre.q.shape, dtype=torch.uint8), sc.double(),
             torch.zeros(pre.q.shape, dtype=torch.uint8), sc, pre.v, lam, 0.5, pre.rms_w)
    _rejects("codes", api.quantize_qk4, pre.q, codes=torch.zeros(pre.q.shape, dtype=torch.uint8))
    dy = torch.zeros_like(pre.v)
    bad_outs = (torch.empty(pre.q.shape, **f32), torch.empty(pre.k.shape, **f32), torch.empty(pre.q.shape, **f32),
                torch.empty(1, **f32), torch.empty(2 * d, **f32))
    _rejects("dv", api.diffattn_bwd_tc, pre.q, pre.k, pre.v, dy, lam, 0.5, pre.rms_w, out=bad_outs)
    _rejects("dy", api.diffattn_bwd, pre.q, pre.k, pre.v, dy[:, :-1].contiguous(), lam, 0.5, pre.rms_w)
    pj = wl.make_proj(1, 24, 96, 2, 16, seed=2, device="cpu")
    _rejects("rope", api.qkv_proj, pj.x, pj.w_qkv, 1, 24, 2, 16, torch.zeros((12, 8, 2), **f32))
    bf = dict(dtype=torch.bfloat16)
    small = (torch.empty((1, 24, 2, 2, 16), **bf), torch.empty((1, 24, 2, 2, 16), **bf), torch.empty((1, 24, 2, 16), **bf))
    _rejects("v must be", api.qkv_proj, pj.x, pj.w_qkv, 1, 24, 2, 16, None, out=small)
    _rejects("out", api.out_proj, torch.zeros((24, 64), **bf), pj.w_o, out=torch.empty((24, 64), **bf))
    dec = wl.make_decode(3, 2, 128, 0, 0, seqlens=[1, 60, 110], seed=1, device="cpu")
    _rejects("v_cache", api.diffattn_decode, dec.q, dec.k_cache, dec.v_cache[..., :128].contiguous(),
             dec.cu_seqlens, dec.max_seqlen, lam, 0.5, dec.rms_w)
    _rejects("k_cache", api.diffattn_decode, dec.q, dec.k_cache.float(), dec.v_cache, dec.cu_seqlens,
             dec.max_seqlen, lam, 0.5, dec.rms_w)
    _rejects("cu_seqlens", api.diffattn_decode_noalloc, dec.q, dec.k_cache, dec.v_cache, dec.cu_seqlens.long(),
             dec.max_seqlen, lam, 0.5, dec.rms_w)


class _FakeCuda:
    """Stands in for a CUDA tensor on a given device: only what the binding's device check reads."""

    is_cuda = True

    def __init__(self, index: int):
        self.device = torch.device("cuda", index)

    def is_contiguous(self):
        return True


def test_tensors_on_two_devices_are_rejected_before_any_launch(monkeypatch):
    # the library would launch on whichever device is current; tensors that
    # live on two devices must never reach it
    def no_launch(*a, **k):
        raise AssertionError("the library was reached")

    monkeypatch.setattr(api, "lib", no_launch)
    with pytest.raises(ValueError, match="one device"):
        api._dev(_FakeCuda(0), _FakeCuda(0), _FakeCuda(1))
    with pytest.raises(ValueError, match="one device"):
        api._launch("diffattn_fwd", (_FakeCuda(1), _FakeCuda(0)), 0)
    assert api._dev(_FakeCuda(1), _FakeCuda(1)) == torch.device("cuda", 1)
