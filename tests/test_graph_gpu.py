"""CUDA-graph capture of the library's calls.

Every call is stream-ordered and neither allocates device memory nor
synchronises, so a whole step (lambda, the prefill, the low-bit prefill with
its quantisers, decode with a workspace and without one) can be captured
once and replayed: the replay must give the same bits as the same calls made
eagerly, and must pick up new input values written into the captured
buffers.  Every kernel here is deterministic: each output element is
computed by a fixed sequence of operations, whatever CTA runs it.
"""
import pytest
import torch

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
    assert api.device_status() == api.OK


def _buffers():
    inp = wl.make_prefill(2, 300, 3, 128, causal=True, dtype="bf16", lambda_init=0.5, w="normal", seed=21,
                          device="cuda")
    dec = wl.make_decode(5, 3, 128, 0, 0, seqlens=[1, 600, 513, 2048, 77], seed=22, device="cuda")
    S, H, _, d = dec.q.shape
    bf = dict(dtype=torch.bfloat16, device="cuda")
    b = dict(
        lam=torch.empty(1, device="cuda"), lam_d=torch.empty(1, device="cuda"),
        y=torch.empty_like(inp.v), y8=torch.empty_like(inp.v),
        qc=torch.empty(inp.q.shape, dtype=torch.uint8, device="cuda"),
        kc=torch.empty(inp.k.shape, dtype=torch.uint8, device="cuda"),
        qs=torch.empty((2, 3, 2), device="cuda"), ks=torch.empty((2, 3, 2), device="cuda"),
        ws=torch.empty(api.decode_workspace_size(S, H, d, dec.max_seqlen), dtype=torch.uint8, device="cuda"),
        yd=torch.empty((S, H, 2 * d), **bf), yn=torch.empty((S, H, 2 * d), **bf),
    )
    return inp, dec, b


def _step(inp, dec, b):
    api.diffattn_lambda(inp.lq1, inp.lk1, inp.lq2, inp.lk2, inp.lambda_init, out=b["lam"])
    api.diffattn_fwd(inp.q, inp.k, inp.v, b["lam"], inp.lambda_init, inp.rms_w, inp.eps, True, out=b["y"])
    api.quantize_qk(inp.q, b["qc"], b["qs"])
    api.quantize_qk(inp.k, b["kc"], b["ks"])
    api.diffattn_fwd_qk8(b["qc"], b["qs"], b["kc"], b["ks"], inp.v, b["lam"], inp.lambda_init, inp.rms_w, inp.eps,
                         True, out=b["y8"])
    api.diffattn_lambda(dec.lq1, dec.lk1, dec.lq2, dec.lk2, dec.lambda_init, out=b["lam_d"])
    api.diffattn_decode(dec.q, dec.k_cache, dec.v_cache, dec.cu_seqlens, dec.max_seqlen, b["lam_d"],
                        dec.lambda_init, dec.rms_w, dec.eps, workspace=b["ws"], out=b["yd"])
    api.diffattn_decode_noalloc(dec.q, dec.k_cache, dec.v_cache, dec.cu_seqlens, dec.max_seqlen, b["lam_d"],
                                dec.lambda_init, dec.rms_w, dec.eps, out=b["yn"])


OUTS = ("y", "y8", "yd", "yn")


def test_step_replays_bit_exact_and_follows_its_inputs():
    inp, dec, b = _buffers()
    # eager run on a side stream (as graph capture wants): the reference, and
    # the first use of every per-device table the library fills lazily
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        _step(inp, dec, b)
    torch.cuda.current_stream().wait_stream(side)
    torch.cuda.synchronize()
    want = {k: b[k].clone() for k in OUTS}
    for k in OUTS:
        b[k].zero_()
    torch.cuda.synchronize()

    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        _step(inp, dec, b)
    for _ in range(3):
        g.replay()
    torch.cuda.synchronize()
    for k in OUTS:
        assert torch.equal(b[k], want[k]), k
    assert torch.equal(b["yd"], b["yn"])

    # new values in the captured input buffers: the replay computes with them
    inp.q.mul_(0.5)
    dec.q.mul_(-1.0)
    g.replay()
    torch.cuda.synchronize()
    got = {k: b[k].clone() for k in OUTS}
    _step(inp, dec, b)
    torch.cuda.synchronize()
    for k in OUTS:
        assert torch.equal(got[k], b[k]), k
    assert not torch.equal(got["y"], want["y"])
    del g
