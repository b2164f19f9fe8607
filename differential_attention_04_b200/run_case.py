"""Run one prefill or decode case a few times (e.g. under a profiler).

  python -m differential_attention_04_b200.run_case prefill --B 2 --N 4096 --H 12 --d 128 --causal 1 --iters 3
  python -m differential_attention_04_b200.run_case prefill --qk8 1 ...   (e4m3 queries/keys: quantise + forward;
                                                                          2: forward only; 3: quantise only)
  python -m differential_attention_04_b200.run_case prefill --qk8 1 --bits 4 ...   (the same with e2m1 codes)
  python -m differential_attention_04_b200.run_case bwd --tc 1 ...   (tensor-core backward; 0: CUDA cores)
  python -m differential_attention_04_b200.run_case proj --B 1 --N 4096 --H 12 --d 128 --dmodel 3072 --iters 3
                                                                          (QKV projection + RoPE, then output projection)
  python -m differential_attention_04_b200.run_case decode --S 64 --H 12 --lmin 1024 --lmax 4096 --iters 3

Inputs come from the seeded generators in ``workloads``; the output is not
checked here (the tests do that).  Prints the CUDA-event time of each launch.
"""
from __future__ import annotations

import argparse

import torch

from . import api
from . import workloads as wl
from .build import build


def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("kind", choices=["prefill", "decode", "bwd", "proj"])
    ap.add_argument("--B", type=int, default=2)
    ap.add_argument("--N", type=int, default=4096)
    ap.add_argument("--H", type=int, default=12)
    ap.add_argument("--d", type=int, default=128)
    ap.add_argument("--causal", type=int, default=1)
    ap.add_argument("--dtype", default="bf16")
    ap.add_argument("--qk8", type=int, default=0)
    ap.add_argument("--bits", type=int, default=8, choices=[8, 4])
    ap.add_argument("--tc", type=int, default=1)
    ap.add_argument("--dmodel", type=int, default=3072)
    ap.add_argument("--S", type=int, default=64)
    ap.add_argument("--lmin", type=int, default=1024)
    ap.add_argument("--lmax", type=int, default=4096)
    ap.add_argument("--iters", type=int, default=3)
    ap.add_argument("--seed", type=int, default=0)
    a = ap.parse_args(argv)
    build()
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    if a.kind == "prefill":
        inp = wl.make_prefill(a.B, a.N, a.H, a.d, causal=bool(a.causal), dtype=a.dtype, seed=a.seed, device=dev)
        lam = api.diffattn_lambda(inp.lq1, inp.lk1, inp.lq2, inp.lk2, inp.lambda_init)
        y = torch.empty_like(inp.v)
        if a.qk8:
            quantize = api.quantize_qk if a.bits == 8 else api.quantize_qk4
            forward = api.diffattn_fwd_qk8 if a.bits == 8 else api.diffattn_fwd_qk4
            qc, qs = quantize(inp.q)
            kc, ks = quantize(inp.k)

            def run():  # --qk8 1: quantise and forward; 2: forward only; 3: quantise only
                if a.qk8 != 2:
                    quantize(inp.q, qc, qs)
                    quantize(inp.k, kc, ks)
                if a.qk8 != 3:
                    forward(qc, qs, kc, ks, inp.v, lam, inp.lambda_init, inp.rms_w, inp.eps, inp.causal, out=y)
        else:
            run = lambda: api.diffattn_fwd(inp.q, inp.k, inp.v, lam, inp.lambda_init, inp.rms_w, inp.eps,
                                           inp.causal, out=y)
    elif a.kind == "bwd":
        inp = wl.make_prefill(a.B, a.N, a.H, a.d, causal=bool(a.causal), dtype=a.dtype, seed=a.seed, device=dev)
        lam = api.diffattn_lambda(inp.lq1, inp.lk1, inp.lq2, inp.lk2, inp.lambda_init)
        dy = torch.randn(inp.v.shape, device=dev).to(inp.v.dtype)
        if a.tc:
            ws = torch.empty(api.bwd_tc_workspace_size(a.B, a.N, a.H, a.d), dtype=torch.uint8, device=dev)
            run = lambda: api.diffattn_bwd_tc(inp.q, inp.k, inp.v, dy, lam, inp.lambda_init, inp.rms_w, inp.eps,
                                              inp.causal, workspace=ws)
        else:
            ws = torch.empty(api.bwd_workspace_size(a.B, a.N, a.H, a.d), dtype=torch.uint8, device=dev)
            run = lambda: api.diffattn_bwd(inp.q, inp.k, inp.v, dy, lam, inp.lambda_init, inp.rms_w, inp.eps,
                                           inp.causal, workspace=ws)
    elif a.kind == "proj":
        inp = wl.make_proj(a.B, a.N, a.dmodel, a.H, a.d, seed=a.seed, device=dev)
        table = api.rope_table(a.N, a.d)
        qkv = api.qkv_proj(inp.x, inp.w_qkv, a.B, a.N, a.H, a.d, table)
        y = torch.empty((a.B * a.N, a.dmodel), dtype=torch.bfloat16, device=dev)

        def run():
            api.qkv_proj(inp.x, inp.w_qkv, a.B, a.N, a.H, a.d, table, out=qkv)
            api.out_proj(qkv[2], inp.w_o, out=y)
    else:
        inp = wl.make_decode(a.S, a.H, a.d, a.lmin, a.lmax, seed=a.seed, device=dev)
        lam = api.diffattn_lambda(inp.lq1, inp.lk1, inp.lq2, inp.lk2, inp.lambda_init)
        ws = torch.empty(api.decode_workspace_size(a.S, a.H, a.d, inp.max_seqlen), dtype=torch.uint8, device=dev)
        y = torch.empty((a.S, a.H, 2 * a.d), dtype=torch.bfloat16, device=dev)
        run = lambda: api.diffattn_decode(inp.q, inp.k_cache, inp.v_cache, inp.cu_seqlens, inp.max_seqlen, lam,
                                          inp.lambda_init, inp.rms_w, inp.eps, workspace=ws, out=y)
    torch.cuda.synchronize()
    for i in range(a.iters):
        s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        s.record()
        run()
        e.record()
        torch.cuda.synchronize()
        print(f"{a.kind} iter {i}: {s.elapsed_time(e):.3f} ms")
    status = api.device_status()
    if status != api.OK:
        raise SystemExit(f"kernel status {status}")


if __name__ == "__main__":
    main()
