"""GPU parity: the CUDA library (through the C ABI) against the float64 oracle.

Tolerances (from the arithmetic the kernels are asked to match):
  bf16 inputs, fp32 accumulation, bf16 output: relative Frobenius error
  <= 5e-3 and max-abs error <= 2e-2; fp32 inputs: both <= 1e-5.
Small shapes are compared element by element over the whole output (several
128-row tiles plus a ragged tail); the full-size workloads are compared on
sampled (batch, head, row) outputs that the oracle computes one by one.
"""
import math

import numpy as np
import pytest
import torch

import oracle.diffattn_ref as ref
from differential_attention_04_b200 import api
from differential_attention_04_b200 import workloads as wl

pytestmark = pytest.mark.gpu

BF16_REL, BF16_ABS = 5e-3, 2e-2
F32_TOL = 1e-5


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


def errs(y, yref):
    y = np.asarray(y, dtype=np.float64)
    yref = np.asarray(yref, dtype=np.float64)
    assert np.isfinite(y).all(), "non-finite output"
    rel = np.linalg.norm(y - yref) / np.linalg.norm(yref)
    mx = np.abs(y - yref).max()
    return rel, mx


def assert_close(y, yref, fp32=False):
    rel, mx = errs(y, yref)
    if fp32:
        assert rel <= F32_TOL and mx <= F32_TOL, f"rel {rel:.3e} max-abs {mx:.3e}"
    else:
        assert rel <= BF16_REL and mx <= BF16_ABS, f"rel {rel:.3e} max-abs {mx:.3e}"


def oracle_lambda(inp):
    f = wl.to_f64
    return ref.lambda_reparam(f(inp.lq1), f(inp.lk1), f(inp.lq2), f(inp.lk2), inp.lambda_init)


def run_prefill(inp):
    lam = api.diffattn_lambda(inp.lq1, inp.lk1, inp.lq2, inp.lk2, inp.lambda_init)
    y = api.diffattn_fwd(inp.q, inp.k, inp.v, lam, inp.lambda_init, inp.rms_w, inp.eps, inp.causal)
    torch.cuda.synchronize()
    return y, lam


def oracle_prefill(inp, heads=None, rows=None):
    f = wl.to_f64
    lam = oracle_lambda(inp)
    if heads is None:
        return ref.diffattn_fwd(f(inp.q), f(inp.k), f(inp.v), lam, inp.lambda_init, f(inp.rms_w), inp.eps,
                                inp.causal, rows=rows)
    out = {}
    for b, h in heads:
        qh = f(inp.q[b:b + 1, :, h:h + 1])
        kh = f(inp.k[b:b + 1, :, h:h + 1])
        vh = f(inp.v[b:b + 1, :, h:h + 1])
        out[(b, h)] = ref.diffattn_fwd(qh, kh, vh, lam, inp.lambda_init, f(inp.rms_w), inp.eps, inp.causal,
                                       rows=rows)[0, :, 0]
    return out


# ------------------------------------------------------------------ lambda --

@pytest.mark.parametrize("d", [1, 64, 128, 1000])
def test_lambda(d):
    g = torch.Generator(device="cuda").manual_seed(d)
    vecs = [torch.randn(d, generator=g, device="cuda") * 0.3 for _ in range(4)]
    lam = api.diffattn_lambda(*vecs, 0.37).item()
    want = ref.lambda_reparam(*[wl.to_f64(t) for t in vecs], 0.37)
    assert abs(lam - want) <= 1e-6 * max(1.0, abs(want))


def test_lambda_zero_vectors_give_lambda_init():
    z = torch.zeros(128, device="cuda")
    assert api.diffattn_lambda(z, z, z, z, 0.65).item() == pytest.approx(0.65, abs=1e-7)


# ------------------------------------------------------------- fp32 prefill --

def test_tiny_fp32_case():
    inp = wl.make_prefill_case("tiny_fp32", device="cuda")
    y, _ = run_prefill(inp)
    assert_close(wl.to_f64(y), oracle_prefill(inp), fp32=True)


@pytest.mark.parametrize("N,d,causal", [(1, 8, True), (37, 7, True), (200, 32, False), (130, 100, True),
                                        (65, 128, False)])
def test_fp32_shapes(N, d, causal):
    inp = wl.make_prefill(2, N, 3, d, causal=causal, dtype="f32", lambda_init=0.3, w="normal", seed=N + d,
                          device="cuda")
    y, _ = run_prefill(inp)
    assert_close(wl.to_f64(y), oracle_prefill(inp), fp32=True)


# ------------------------------------------------------------- bf16 prefill --

@pytest.mark.parametrize("d", [128, 64])
@pytest.mark.parametrize("causal", [True, False])
@pytest.mark.parametrize("N", [1, 100, 128, 200, 384, 517])
def test_bf16_small_full(N, d, causal):
    inp = wl.make_prefill(2, N, 2, d, causal=causal, dtype="bf16", lambda_init=0.5, w="normal", seed=N,
                          device="cuda")
    y, _ = run_prefill(inp)
    assert_close(wl.to_f64(y), oracle_prefill(inp))


@pytest.mark.parametrize("e1,e2,lambda_init,want", [(3.0, 1.0, 0.2, 2.2), (1.0, 2.5, 0.8, -0.7),
                                                    (1.0, 1.0, 0.0, 0.0)])
def test_bf16_lambda_range(e1, e2, lambda_init, want):
    # lambda outside (0, 1) and lambda = 0: constant lambda vectors with
    # lq1 . lk1 = ln(e1) and lq2 . lk2 = ln(e2), so lambda = e1 - e2 + lambda_init.
    d = 128
    inp = wl.make_prefill(1, 300, 3, d, causal=True, dtype="bf16", lambda_init=lambda_init, seed=11,
                          device="cuda")
    inp.lq1.fill_(math.sqrt(math.log(e1) / d))
    inp.lk1.copy_(inp.lq1)
    inp.lq2.fill_(math.sqrt(math.log(e2) / d))
    inp.lk2.copy_(inp.lq2)
    y, lam = run_prefill(inp)
    # the float32 lambda vectors hold ln(e)/d only to float32 precision
    assert abs(oracle_lambda(inp) - want) < 1e-6
    assert abs(lam.item() - oracle_lambda(inp)) <= 1e-6 * max(1.0, abs(want))
    assert_close(wl.to_f64(y), oracle_prefill(inp))


def test_bf16_equal_maps_reduce():
    # Q2 = Q1 and K2 = K1: the output is the normalised single-map attention
    # (the factor 1 - lambda cancels in the RMSNorm when lambda < 1).
    inp = wl.make_prefill(1, 256, 2, 128, causal=True, dtype="bf16", lambda_init=0.5, seed=5, device="cuda")
    inp.q[:, :, :, 1] = inp.q[:, :, :, 0]
    inp.k[:, :, :, 1] = inp.k[:, :, :, 0]
    y, _ = run_prefill(inp)
    assert_close(wl.to_f64(y), oracle_prefill(inp))


def test_bf16_large_scores():
    # scaled-up inputs give scores far from 0 and exercise the lazy rescale of O
    inp = wl.make_prefill(1, 640, 2, 128, causal=True, dtype="bf16", lambda_init=0.5, seed=9, device="cuda")
    inp.q.mul_(4)
    inp.k.mul_(4)
    y, _ = run_prefill(inp)
    assert_close(wl.to_f64(y), oracle_prefill(inp))


def test_bf16_score_jumps():
    # keys scaled up along the sequence: the running maximum climbs by far
    # more than 2^64 (log2 units) between key tiles, which takes the
    # overflow-guard path (rescale O first, then recompute P) as well as the
    # lazy rescale after PV
    inp = wl.make_prefill(1, 640, 2, 128, causal=True, dtype="bf16", lambda_init=0.5, seed=11, device="cuda")
    ramp = torch.linspace(1.0, 24.0, 640, device="cuda").view(1, 640, 1, 1, 1)
    inp.k.copy_((inp.k.float() * ramp).to(inp.k.dtype))
    inp.q.mul_(4)
    y, _ = run_prefill(inp)
    assert torch.isfinite(y.float()).all()
    assert_close(wl.to_f64(y), oracle_prefill(inp))


MODE_NAMES = {api.MODE_LAMBDA_ZERO: "lambda_zero", api.MODE_SUM: "sum"}


def _oracle_mode(inp, mode):
    f = wl.to_f64
    return ref.diffattn_fwd(f(inp.q), f(inp.k), f(inp.v), oracle_lambda(inp), inp.lambda_init, f(inp.rms_w),
                            inp.eps, inp.causal, mode=MODE_NAMES[mode])


@pytest.mark.parametrize("mode", sorted(MODE_NAMES))
@pytest.mark.parametrize("d", [128, 64])
@pytest.mark.parametrize("causal", [True, False])
def test_bf16_control_modes(mode, d, causal):
    # the review's controls: lambda fixed to 0 (one map) and the maps added
    inp = wl.make_prefill(1, 200, 2, d, causal=causal, dtype="bf16", lambda_init=0.5, w="normal", seed=31 + d,
                          device="cuda")
    lam = api.diffattn_lambda(inp.lq1, inp.lk1, inp.lq2, inp.lk2, inp.lambda_init)
    y = api.diffattn_fwd(inp.q, inp.k, inp.v, lam, inp.lambda_init, inp.rms_w, inp.eps, causal, mode=mode)
    torch.cuda.synchronize()
    assert_close(wl.to_f64(y), _oracle_mode(inp, mode))


@pytest.mark.parametrize("mode", sorted(MODE_NAMES))
def test_fp32_control_modes(mode):
    inp = wl.make_prefill(2, 70, 3, 32, causal=True, dtype="f32", lambda_init=0.3, w="normal", seed=41,
                          device="cuda")
    lam = api.diffattn_lambda(inp.lq1, inp.lk1, inp.lq2, inp.lk2, inp.lambda_init)
    y = api.diffattn_fwd(inp.q, inp.k, inp.v, lam, inp.lambda_init, inp.rms_w, inp.eps, True, mode=mode)
    torch.cuda.synchronize()
    assert_close(wl.to_f64(y), _oracle_mode(inp, mode), fp32=True)


def test_lambda_zero_ignores_map2():
    inp = wl.make_prefill(1, 300, 2, 128, causal=True, dtype="bf16", seed=43, device="cuda")
    lam = api.diffattn_lambda(inp.lq1, inp.lk1, inp.lq2, inp.lk2, inp.lambda_init)
    y1 = api.diffattn_fwd(inp.q, inp.k, inp.v, lam, inp.lambda_init, inp.rms_w, inp.eps, True,
                          mode=api.MODE_LAMBDA_ZERO)
    inp.q[:, :, :, 1].normal_()
    inp.k[:, :, :, 1].mul_(3.0)
    y2 = api.diffattn_fwd(inp.q, inp.k, inp.v, lam, inp.lambda_init, inp.rms_w, inp.eps, True,
                          mode=api.MODE_LAMBDA_ZERO)
    torch.cuda.synchronize()
    assert torch.equal(y1, y2)


def test_output_only_written_in_bounds():
    inp = wl.make_prefill(1, 200, 2, 128, causal=True, dtype="bf16", seed=3, device="cuda")
    lam = api.diffattn_lambda(inp.lq1, inp.lk1, inp.lq2, inp.lk2, inp.lambda_init)
    big = torch.full((1, 256, 2, 256), 7.0, dtype=torch.bfloat16, device="cuda")
    out = big[:, :200]  # contiguous prefix of a larger buffer
    api.diffattn_fwd(inp.q, inp.k, inp.v, lam, inp.lambda_init, inp.rms_w, inp.eps, True, out=out)
    torch.cuda.synchronize()
    assert torch.all(big[:, 200:] == 7.0)


# ------------------------------------------------ full-size prefill (sampled) --

def _sample_rows(N, extra=(), n_random=24, seed=0):
    rng = np.random.default_rng(seed)
    rows = {0, 1, 127, 128, N // 2, N - 129, N - 2, N - 1} | set(int(x) for x in extra)
    rows |= set(int(x) for x in rng.integers(0, N, n_random))
    return sorted(r for r in rows if 0 <= r < N)


@pytest.mark.parametrize("case", ["prefill_3b", "prefill_13b_causal", "prefill_13b_nomask"])
def test_full_size_sampled(case):
    inp = wl.make_prefill_case(case, device="cuda")
    y, _ = run_prefill(inp)
    B, N, H = inp.q.shape[:3]
    heads = [(0, 0), (B - 1, H - 1), (B // 2, H // 2)]
    rows = _sample_rows(N)
    want = oracle_prefill(inp, heads=heads, rows=rows)
    for (b, h), yr in want.items():
        assert_close(wl.to_f64(y[b, rows, h]), yr)
    # every output is finite
    assert torch.isfinite(y.float()).all()


def test_full_size_64k_needle_sampled():
    inp = wl.make_prefill_case("prefill_64k_needle", device="cuda")
    y, _ = run_prefill(inp)
    N, H = inp.q.shape[1], inp.q.shape[2]
    for h in (0, 5, H - 1):
        p = inp.needle_pos[0][h]
        rows = _sample_rows(N, extra=(p, p + 1, p - 1), n_random=12, seed=h)
        want = oracle_prefill(inp, heads=[(0, h)], rows=rows)[(0, h)]
        assert_close(wl.to_f64(y[0, rows, h]), want)
    assert torch.isfinite(y.float()).all()


def _oracle_full_head(inp, b, h, block=1024):
    """Every output row of one (batch, head), computed by the oracle in
    blocks of query rows (the rows are independent: each block still scores
    its queries against every key)."""
    f = wl.to_f64
    N = inp.q.shape[1]
    lam = oracle_lambda(inp)
    qh, kh, vh = (f(t[b:b + 1, :, h:h + 1]) for t in (inp.q, inp.k, inp.v))
    w = f(inp.rms_w)
    parts = [ref.diffattn_fwd(qh, kh, vh, lam, inp.lambda_init, w, inp.eps, inp.causal,
                              rows=np.arange(r0, min(N, r0 + block)))[0, :, 0]
             for r0 in range(0, N, block)]
    return np.concatenate(parts, axis=0)


@pytest.mark.parametrize("case,head", [("prefill_64k_needle", (0, 0)), ("prefill_13b_causal", (1, 19)),
                                       ("prefill_13b_nomask", (0, 7))])
def test_full_size_one_head_complete(case, head):
    # one whole head of each long configuration, element by element: all N
    # query rows against all keys (the 64K case takes the head whose needle
    # key the last query aligns with)
    inp = wl.make_prefill_case(case, device="cuda")
    y, _ = run_prefill(inp)
    b, h = head
    got = wl.to_f64(y[b, :, h])
    del y
    torch.cuda.empty_cache()
    assert_close(got, _oracle_full_head(inp, b, h))


# ------------------------------------------------------------------ decode --

def run_decode(inp, mode=api.MODE_DIFF):
    lam = api.diffattn_lambda(inp.lq1, inp.lk1, inp.lq2, inp.lk2, inp.lambda_init)
    y = api.diffattn_decode(inp.q, inp.k_cache, inp.v_cache, inp.cu_seqlens, inp.max_seqlen, lam,
                            inp.lambda_init, inp.rms_w, inp.eps, mode=mode)
    torch.cuda.synchronize()
    return y


def oracle_decode(inp, pairs, mode="diff"):
    f = wl.to_f64
    lam = ref.lambda_reparam(f(inp.lq1), f(inp.lk1), f(inp.lq2), f(inp.lk2), inp.lambda_init)
    cu = inp.cu_seqlens.cpu().numpy()
    out = {}
    for s, h in pairs:
        lo, hi = int(cu[s]), int(cu[s + 1])
        kc = f(inp.k_cache[lo:hi, h:h + 1])
        vc = f(inp.v_cache[lo:hi, h:h + 1])
        out[(s, h)] = ref.diffattn_decode(f(inp.q[s:s + 1, h:h + 1]), kc, vc, [0, hi - lo], lam,
                                          inp.lambda_init, f(inp.rms_w), inp.eps, mode=mode)[0, 0]
    return out


def test_decode_small_full():
    inp = wl.make_decode(7, 3, 128, 0, 0, seqlens=[1, 2, 7, 511, 512, 513, 1500], seed=4, device="cuda")
    y = run_decode(inp)
    want = oracle_decode(inp, [(s, h) for s in range(7) for h in range(3)])
    got = np.stack([wl.to_f64(y[s, h]) for (s, h) in want])
    assert_close(got, np.stack(list(want.values())))


@pytest.mark.parametrize("mode,name", [(1, "lambda_zero"), (2, "sum")])
def test_decode_control_modes(mode, name):
    inp = wl.make_decode(5, 3, 128, 0, 0, seqlens=[1, 33, 512, 513, 1300], seed=6, device="cuda")
    y = run_decode(inp, mode)
    want = oracle_decode(inp, [(s, h) for s in range(5) for h in range(3)], name)
    got = np.stack([wl.to_f64(y[s, h]) for (s, h) in want])
    assert_close(got, np.stack(list(want.values())))


def test_decode_is_last_prefill_row():
    # a decode step over a sequence equals the last row of a causal prefill over it
    L, H = 300, 2
    pre = wl.make_prefill(1, L, H, 128, causal=True, dtype="bf16", lambda_init=0.5, seed=21, device="cuda")
    y_pre, lam = run_prefill(pre)
    cu = torch.tensor([0, L], dtype=torch.int32, device="cuda")
    y_dec = api.diffattn_decode(pre.q[0, L - 1:L].contiguous(), pre.k[0].contiguous(), pre.v[0].contiguous(), cu,
                                L, lam, pre.lambda_init, pre.rms_w, pre.eps)
    torch.cuda.synchronize()
    rel, mx = errs(wl.to_f64(y_dec[0]), wl.to_f64(y_pre[0, L - 1]))
    assert rel <= 2 * BF16_REL and mx <= 2 * BF16_ABS


def test_decode_full_size_sampled():
    inp = wl.make_decode_case("decode_64x12", device="cuda")
    y = run_decode(inp)
    rng = np.random.default_rng(1)
    S, H = inp.q.shape[:2]
    longest = int(np.argmax(inp.seqlens))
    shortest = int(np.argmin(inp.seqlens))
    pairs = [(longest, 0), (shortest, H - 1)] + [(int(s), int(h)) for s, h in
                                                  zip(rng.integers(0, S, 14), rng.integers(0, H, 14))]
    want = oracle_decode(inp, pairs)
    got = np.stack([wl.to_f64(y[s, h]) for (s, h) in want])
    assert_close(got, np.stack(list(want.values())))
    assert torch.isfinite(y.float()).all()
