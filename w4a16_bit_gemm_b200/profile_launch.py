"""A few launches of one libwq operation on one seeded workload, for profilers.

    python -m w4a16_bit_gemm_b200.profile_launch linear --N 4096 --K 4096 --M 1
    python -m w4a16_bit_gemm_b200.profile_launch quantize --N 4096 --K 4096
    python -m w4a16_bit_gemm_b200.profile_launch dequantize --N 4096 --K 4096
    python -m w4a16_bit_gemm_b200.profile_launch gemm --N 8192 --K 8192 --M 2048
    python -m w4a16_bit_gemm_b200.profile_launch linear_w8 --N 4096 --K 4096 --M 1

Each run quantizes one N(0, 0.02) weight matrix (group 128, asymmetric unless
--sym; linear_w8: symmetric INT8 per channel unless --g is given), keeps
--copies packed copies so that consecutive launches read different memory
(copies x artifact bytes > L2 at the default sizes), and issues --iters
launches of the operation eagerly on the current stream, then
checks the device status.  Under `ncu -k regex:<kernel> -s <skip> -c 1` one of
the later launches is captured; the launch sequence and the inputs are the
same as those of the benchmark's sweep of that shape.
"""
from __future__ import annotations

import argparse
import sys

import torch


def main(argv=None) -> int:
    ap = argparse.ArgumentParser()
    ap.add_argument("op", choices=["linear", "quantize", "dequantize", "gemm", "linear_w8"])
    ap.add_argument("--N", type=int, default=4096)
    ap.add_argument("--K", type=int, default=4096)
    ap.add_argument("--M", type=int, default=1)
    ap.add_argument("--g", type=int, default=None, help="group size (default 128; per-channel for linear_w8)")
    ap.add_argument("--sym", action="store_true")
    ap.add_argument("--copies", type=int, default=8)
    ap.add_argument("--iters", type=int, default=16)
    args = ap.parse_args(argv)

    from w4a16_bit_gemm_b200 import binding as b
    from w4a16_bit_gemm_b200 import synthetic as syn

    W = syn.weight(args.N, args.K, 0.02, 0x5EED0000 + 2, 0, "cuda")
    if args.op == "linear_w8":
        p8 = b.quantize_w8(W, args.g)
        packs = [b.PackedLinearW8(p8.qweight.clone(), p8.scales.clone(), p8.d_out, p8.d_in, p8.group_size)
                 for _ in range(args.copies)]
    else:
        g = args.g or 128
        p0 = b.quantize_rtn(W, g, args.sym)
        packs = [b.PackedLinear(p0.qweight.clone(), p0.scales.clone(), None if p0.zeros is None else p0.zeros.clone(),
                                args.N, args.K, g, args.sym) for _ in range(args.copies)]
    X = syn.activations(args.M, args.K, 0x5EED0000 + 2, 77, "cuda")
    Y = torch.empty(args.M, args.N, dtype=torch.bfloat16, device="cuda")
    Wh = torch.empty(args.N, args.K, dtype=torch.bfloat16, device="cuda")
    for i in range(args.iters):
        p = packs[i % args.copies]
        if args.op in ("linear", "gemm"):
            b.linear_w4a16(X, p, out=Y)
        elif args.op == "linear_w8":
            b.linear_w8a16(X, p, out=Y)
        elif args.op == "quantize":
            b.quantize_rtn(W, args.g or 128, args.sym, out=p)
        else:
            b.dequantize(p, out=Wh)
    torch.cuda.synchronize()
    st, flags = b.device_error()
    print(f"{args.op} N={args.N} K={args.K} M={args.M}: {args.iters} launches, status {st} flags {flags}")
    return 0 if st == b.WQ_OK else 1


if __name__ == "__main__":
    sys.exit(main())
