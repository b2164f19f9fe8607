"""Failure detection without a GPU fault: every pipeline wait inside the
prefill kernel is bounded.  With the limit forced down to 1 ns the waits run
out at once; the kernel records DIFFATTN_ERR_TIMEOUT in the device status
word, drains its copies and tensor-core work, frees its tensor memory and
returns, and the context stays usable for a normal, correct call."""
import numpy as np
import pytest
import torch

import oracle.diffattn_ref as ref
from differential_attention_04_b200 import api
from differential_attention_04_b200 import workloads as wl

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from differential_attention_04_b200.build import build
    build()
    torch.cuda.set_device(0)
    api.set_wait_limit_ns(0)
    yield
    api.set_wait_limit_ns(0)


def _run(inp):
    lam = api.diffattn_lambda(inp.lq1, inp.lk1, inp.lq2, inp.lk2, inp.lambda_init)
    y = api.diffattn_fwd(inp.q, inp.k, inp.v, lam, inp.lambda_init, inp.rms_w, inp.eps, inp.causal)
    torch.cuda.synchronize()
    return y


def test_forced_timeout_is_reported_and_context_survives():
    inp = wl.make_prefill(1, 640, 2, 128, causal=True, dtype="bf16", seed=5, device="cuda")
    assert api.device_status() == api.OK
    api.set_wait_limit_ns(1)
    try:
        _run(inp)
    finally:
        api.set_wait_limit_ns(0)
    assert api.device_status() == api.ERR_TIMEOUT
    assert api.device_status() == api.OK  # reading clears the word
    # the context is intact: the same call with the default limit is correct
    y = _run(inp)
    f = wl.to_f64
    lam = ref.lambda_reparam(f(inp.lq1), f(inp.lk1), f(inp.lq2), f(inp.lk2), inp.lambda_init)
    want = ref.diffattn_fwd(f(inp.q), f(inp.k), f(inp.v), lam, inp.lambda_init, f(inp.rms_w), inp.eps, True)
    got = f(y)
    rel = np.linalg.norm(got - want) / np.linalg.norm(want)
    assert rel <= 5e-3 and np.abs(got - want).max() <= 2e-2
    assert api.device_status() == api.OK
