"""GPU parity of the projections either side of the path (qkv_proj with its
fused rotary embedding, out_proj) and of the cos/sin table, against the
float64 oracle (oracle/proj_ref.py) on the same bf16 inputs.

Bounds.  The table is float32 rounding of double-precision cos/sin: at most
2^-25 of 1 plus the double routines' error, so 6e-8 absolute.  A projected
entry is a float32 sum of d_model bf16 x bf16 products (each product exact in
float32; the sum's rounding error at most about d_model * 2^-24 of the sum of
|products|, well below 1e-4 of the largest entry here), rotated in float32
with the float32 table, then rounded once to bf16 (relative error at most
2^-9): |got - ref| <= 2^-8 |ref| + 1e-4 max|ref|.
"""
import numpy as np
import pytest
import torch

import oracle.proj_ref as pr
from differential_attention_04_b200 import api
from differential_attention_04_b200 import workloads as wl

pytestmark = pytest.mark.gpu


def _close(got, want, name):
    got = got.float().cpu().numpy().astype(np.float64)
    want = np.asarray(want, dtype=np.float64)
    tol = 2.0 ** -8 * np.abs(want) + 1e-4 * float(np.max(np.abs(want)))
    bad = np.abs(got - want) > tol
    assert not bad.any(), f"{name}: {int(bad.sum())} entries out of bound, worst {float(np.max(np.abs(got - want) - tol)):.3e}"


@pytest.mark.parametrize("N,d,base", [(1, 64, 10000.0), (300, 128, 10000.0), (4096, 128, 10000.0),
                                      (65536, 128, 500000.0)])
def test_rope_table(N, d, base):
    t = api.rope_table(N, d, base)
    torch.cuda.synchronize()
    ang = pr.rope_angles(np.arange(N), d, base)
    got = t.cpu().numpy().astype(np.float64)
    assert np.max(np.abs(got[..., 0] - np.cos(ang))) <= 6e-8
    assert np.max(np.abs(got[..., 1] - np.sin(ang))) <= 6e-8


@pytest.mark.parametrize("rope", [True, False])
@pytest.mark.parametrize("B,N,dm,H,d", [(1, 1, 64, 1, 32), (2, 37, 128, 2, 64), (1, 300, 256, 3, 128),
                                        (2, 129, 192, 2, 32), (1, 200, 512, 4, 128)])
def test_qkv_proj(B, N, dm, H, d, rope):
    inp = wl.make_proj(B, N, dm, H, d, seed=N + dm, device="cuda")
    table = api.rope_table(N, d) if rope else None
    q, k, v = api.qkv_proj(inp.x, inp.w_qkv, B, N, H, d, table)
    torch.cuda.synchronize()
    assert api.device_status() == api.OK
    f = wl.to_f64
    wq, wk, wv = pr.qkv_proj(f(inp.x), f(inp.w_qkv), B, N, H, d, 10000.0 if rope else None)
    _close(q, wq, "q")
    _close(k, wk, "k")
    _close(v, wv, "v")


@pytest.mark.parametrize("M,K,n_out", [(1, 64, 32), (37, 128, 96), (300, 256, 512), (1000, 512, 288),
                                       (129, 3072, 256)])
def test_out_proj(M, K, n_out):
    g = torch.Generator(device="cuda").manual_seed(M + K)
    o = torch.randn((M, K), generator=g, device="cuda").to(torch.bfloat16)
    w = (torch.randn((n_out, K), generator=g, device="cuda") / K ** 0.5).to(torch.bfloat16)
    y = api.out_proj(o, w)
    torch.cuda.synchronize()
    _close(y, pr.out_proj(wl.to_f64(o), wl.to_f64(w)), "y")


def test_qkv_proj_full_size_sampled_rows():
    """The 3B-like model's projection (B=4, N=4096, d_model=3072, H=12, d=128)
    in one call; 24 rows (sequence starts, ends and interior positions) checked
    in every column against the oracle run on those rows alone."""
    inp = wl.make_proj_case("proj_3b", seed=0, device="cuda")
    B, N, H, d = inp.B, inp.N, inp.H, inp.d
    table = api.rope_table(N, d)
    q, k, v = api.qkv_proj(inp.x, inp.w_qkv, B, N, H, d, table)
    torch.cuda.synchronize()
    rows = [0, 1, 127, 128, 4095, 4096, 4097, 8191, 12287, 16383] + list(range(5000, 16384, 997))
    x = wl.to_f64(inp.x[rows])
    w = wl.to_f64(inp.w_qkv)
    y = x @ w.T
    hq = H * 2 * d
    for i, m in enumerate(rows):
        b, n = divmod(m, N)
        wq = pr.apply_rope(y[i, :hq].reshape(H * 2, 1, d), [n])[:, 0].reshape(H, 2, d)
        wk = pr.apply_rope(y[i, hq:2 * hq].reshape(H * 2, 1, d), [n])[:, 0].reshape(H, 2, d)
        _close(q[b, n], wq, f"q row {m}")
        _close(k[b, n], wk, f"k row {m}")
        _close(v[b, n], y[i, 2 * hq:].reshape(H, 2 * d), f"v row {m}")
