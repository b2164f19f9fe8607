"""The allocation-free decode entry point (diffattn_decode_noalloc).

It serves callers that may not call cudaMalloc (for instance a plugin in an
engine that owns all device memory), by using the library's built-in device
scratch array instead of a caller workspace.  Checked through the C ABI on two
calls in a row with different problems (the second call reuses the scratch
the first one left behind):
  * bit for bit against the workspace-based diffattn_decode, which runs the
    same kernels on the same inputs;
  * against the float64 oracle, within the bf16 tolerance of the parity tests.
The Python wrapper, given its output buffer, is checked to allocate no device
memory.  The file is named so that pytest collects it last.
"""
import numpy as np
import pytest
import torch

import oracle.diffattn_ref as ref
from differential_attention_04_b200 import _lib, api
from differential_attention_04_b200 import workloads as wl

pytestmark = pytest.mark.gpu

BF16_REL, BF16_ABS = 5e-3, 2e-2


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from differential_attention_04_b200.build import build
    build()
    torch.cuda.set_device(0)


def _close_to_oracle(got, inp):
    f = wl.to_f64
    lam = ref.lambda_reparam(f(inp.lq1), f(inp.lk1), f(inp.lq2), f(inp.lk2), inp.lambda_init)
    want = ref.diffattn_decode(f(inp.q), f(inp.k_cache), f(inp.v_cache), inp.cu_seqlens.cpu().numpy(), lam,
                               inp.lambda_init, f(inp.rms_w), inp.eps)
    a = f(got)
    assert np.isfinite(a).all()
    rel = np.linalg.norm(a - want) / np.linalg.norm(want)
    assert rel <= BF16_REL and np.abs(a - want).max() <= BF16_ABS, f"rel {rel:.3e}"


def _noalloc_call(inp, lam, out):
    L = _lib.lib()
    S, H, _, d = inp.q.shape
    return L.diffattn_decode_noalloc(inp.q.data_ptr(), inp.k_cache.data_ptr(), inp.v_cache.data_ptr(),
                                     inp.cu_seqlens.data_ptr(), inp.max_seqlen, out.data_ptr(), S, H, d,
                                     lam.data_ptr(), inp.lambda_init, inp.rms_w.data_ptr(), inp.eps,
                                     torch.cuda.current_stream().cuda_stream)


def test_noalloc_matches_workspace_decode_twice():
    problems = [
        wl.make_decode(6, 4, 128, 0, 0, seqlens=[1, 300, 511, 512, 1025, 2500], seed=31, device="cuda"),
        wl.make_decode(3, 12, 128, 0, 0, seqlens=[700, 2, 129], seed=32, device="cuda"),
    ]
    for i, inp in enumerate(problems):
        lam = api.diffattn_lambda(inp.lq1, inp.lk1, inp.lq2, inp.lk2, inp.lambda_init)
        want = api.diffattn_decode(inp.q, inp.k_cache, inp.v_cache, inp.cu_seqlens, inp.max_seqlen, lam,
                                   inp.lambda_init, inp.rms_w, inp.eps)
        out = torch.full_like(want, float("nan"))
        assert _noalloc_call(inp, lam, out) == api.OK
        torch.cuda.synchronize()
        # the same kernels on the same inputs: identical bits
        assert torch.equal(out, want)
        if i == 0:
            _close_to_oracle(out, inp)
    assert api.device_status() == api.OK


def test_noalloc_wrapper_allocates_nothing():
    inp = wl.make_decode(4, 3, 128, 0, 0, seqlens=[9, 513, 1, 1200], seed=34, device="cuda")
    lam = api.diffattn_lambda(inp.lq1, inp.lk1, inp.lq2, inp.lk2, inp.lambda_init)
    out = torch.empty((4, 3, 256), dtype=torch.bfloat16, device="cuda")
    api.diffattn_decode_noalloc(inp.q, inp.k_cache, inp.v_cache, inp.cu_seqlens, inp.max_seqlen, lam,
                                inp.lambda_init, inp.rms_w, inp.eps, out=out)  # set-up call
    torch.cuda.synchronize()
    alloc, reserved = torch.cuda.memory_allocated(), torch.cuda.memory_reserved()
    for _ in range(3):
        api.diffattn_decode_noalloc(inp.q, inp.k_cache, inp.v_cache, inp.cu_seqlens, inp.max_seqlen, lam,
                                    inp.lambda_init, inp.rms_w, inp.eps, out=out)
    torch.cuda.synchronize()
    assert torch.cuda.memory_allocated() == alloc and torch.cuda.memory_reserved() == reserved
    _close_to_oracle(out, inp)


def test_noalloc_rejects_problems_beyond_its_scratch():
    inp = wl.make_decode(2, 2, 128, 0, 0, seqlens=[5, 7], seed=33, device="cuda")
    lam = api.diffattn_lambda(inp.lq1, inp.lk1, inp.lq2, inp.lk2, inp.lambda_init)
    out = torch.empty((2, 2, 256), dtype=torch.bfloat16, device="cuda")
    L = _lib.lib()
    # S = 64, H = 12 and max_seqlen = 32768 need far more than the 16 MiB scratch
    assert L.diffattn_decode_workspace_size(64, 12, 128, 32768) > api.NOALLOC_SCRATCH_BYTES
    big = L.diffattn_decode_noalloc(inp.q.data_ptr(), inp.k_cache.data_ptr(), inp.v_cache.data_ptr(),
                                    inp.cu_seqlens.data_ptr(), 32768, out.data_ptr(), 64, 12, 128,
                                    lam.data_ptr(), 0.5, inp.rms_w.data_ptr(), 1e-5, None)
    assert big == api.ERR_WORKSPACE
