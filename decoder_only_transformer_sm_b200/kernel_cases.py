"""Run single kernels of the training step on chosen shapes, through the
kernel-level C ABI, and print their CUDA-event times. Used to time kernels in
isolation and as the target command of ncu captures.

  python -m decoder_only_transformer_sm_b200.kernel_cases gemm --layout NT \
      --M 16384 --N 3072 --K 768 --epilogue bias_gelu --reps 3
  python -m decoder_only_transformer_sm_b200.kernel_cases attention \
      --B 16 --T 1024 --H 12 --hd 64 --engine 1 --reps 3
"""
from __future__ import annotations

import argparse
import json


def _events(torch, fn, reps: int):
    times = []
    for _ in range(reps):
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        fn()
        b.record()
        torch.cuda.synchronize()
        times.append(a.elapsed_time(b))
    return times


def gemm_case(args):
    import torch
    from . import native
    M, N, K = args.M, args.N, args.K
    g = torch.Generator().manual_seed(0)
    if args.layout == "NT":
        A, B = torch.randn((M, K), generator=g), torch.randn((N, K), generator=g)
    elif args.layout == "NN":
        A, B = torch.randn((M, K), generator=g), torch.randn((K, N), generator=g)
    else:
        A, B = torch.randn((K, M), generator=g), torch.randn((K, N), generator=g)
    A, B = A.to(torch.bfloat16).cuda(), B.to(torch.bfloat16).cuda()
    ep = args.epilogue
    f32_out = ep in ("bias_resid", "accum_f32")
    out = torch.zeros((M, N), dtype=torch.float32 if f32_out else torch.bfloat16, device="cuda")
    out2 = torch.empty((M, N), dtype=torch.bfloat16, device="cuda") if ep == "bias_gelu" else None
    bias = torch.randn(N, device="cuda") if ep.startswith("bias") else None
    resid = torch.randn((M, N), device="cuda") if ep == "bias_resid" else None
    aux = torch.randn((M, N), device="cuda").to(torch.bfloat16) if ep == "mul" else None
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    fn = lambda: native.matmul_bf16(args.layout, A, B, M, N, K, ep, out, out2=out2, bias=bias,  # noqa: E731
                                    resid=resid, aux=aux, beta=1.0, engine="tc" if args.engine else "simt",
                                    status=st)
    fn()
    torch.cuda.synchronize()
    t = _events(torch, fn, args.reps)
    best = min(t)
    print(json.dumps({"case": "gemm", "layout": args.layout, "M": M, "N": N, "K": K, "epilogue": ep,
                      "ms": t, "tflops_best": 2.0 * M * N * K / best / 1e9, "status": int(st.item())}))


def attention_case(args):
    import torch
    from . import native
    B, T, H, hd = args.B, args.T, args.H, args.hd
    C = H * hd
    g = torch.Generator().manual_seed(0)
    qkv = torch.randn((B, T, 3 * C), generator=g).to(torch.bfloat16).cuda()
    dout = torch.randn((B, T, C), generator=g).to(torch.bfloat16).cuda()
    out = torch.empty((B, T, C), dtype=torch.bfloat16, device="cuda")
    lse = torch.empty((B, H, T), dtype=torch.float32, device="cuda")
    dqkv = torch.empty_like(qkv)
    ws = torch.empty(B * H * T, dtype=torch.float32, device="cuda")
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    fwd = lambda: native.attention_fwd(qkv, out, lse, B, T, H, hd, engine=args.engine, status=st)  # noqa: E731
    bwd = lambda: native.attention_bwd(qkv, out, dout, lse, dqkv, B, T, H, hd, ws,  # noqa: E731
                                       engine=args.engine, status=st)
    fwd()
    bwd()
    torch.cuda.synchronize()
    tf = _events(torch, fwd, args.reps)
    tb = _events(torch, bwd, args.reps)
    flops = 2.0 * B * H * T * (T + 1) * hd
    print(json.dumps({"case": "attention", "B": B, "T": T, "H": H, "hd": hd, "fwd_ms": tf, "bwd_ms": tb,
                      "fwd_tflops_best": flops / min(tf) / 1e9, "bwd_tflops_best": 2.5 * flops / min(tb) / 1e9,
                      "status": int(st.item())}))


def main():
    ap = argparse.ArgumentParser()
    sub = ap.add_subparsers(dest="case", required=True)
    g = sub.add_parser("gemm")
    g.add_argument("--layout", default="NT", choices=["NT", "NN", "TN"])
    g.add_argument("--M", type=int, default=16384)
    g.add_argument("--N", type=int, default=3072)
    g.add_argument("--K", type=int, default=768)
    g.add_argument("--epilogue", default="store")
    g.add_argument("--engine", type=int, default=1)
    g.add_argument("--reps", type=int, default=3)
    a = sub.add_parser("attention")
    a.add_argument("--B", type=int, default=16)
    a.add_argument("--T", type=int, default=1024)
    a.add_argument("--H", type=int, default=12)
    a.add_argument("--hd", type=int, default=64)
    a.add_argument("--engine", type=int, default=1)
    a.add_argument("--reps", type=int, default=3)
    args = ap.parse_args()
    {"gemm": gemm_case, "attention": attention_case}[args.case](args)


if __name__ == "__main__":
    main()
