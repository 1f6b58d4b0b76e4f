"""Small, self-contained invocations of one library call for a profiler to capture.

    python -m free_weight_quantization_b200.profile_cases gemm --batch 16
    python -m free_weight_quantization_b200.profile_cases gemv
    python -m free_weight_quantization_b200.profile_cases dequant
    python -m free_weight_quantization_b200.profile_cases quantize

Each quantizes the 4096x4096 4-bit group-64 workload matrix once on cuda:0 (one launch chain),
then runs the named call `--calls` times (3 by default) on its codes and synchronizes.  A
profiler that skips the quantize chain's launches captures the named call on warm code paths;
the inputs (a few tens of MB) are far below the device's memory, so every capture stays small.
"""
from __future__ import annotations

import argparse
import os
import sys

sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))


def main() -> None:
    ap = argparse.ArgumentParser()
    ap.add_argument("call", choices=["gemm", "gemv", "dequant", "quantize"])
    ap.add_argument("--batch", type=int, default=16)
    ap.add_argument("--calls", type=int, default=3)
    args = ap.parse_args()

    import torch

    from free_weight_quantization_b200 import hqq
    from free_weight_quantization_b200 import workloads as wl

    c = wl.ATTN
    W = torch.from_numpy(c.make()).to("cuda:0")
    q = hqq.hqq_quantize(W, c.nbits, c.group_size, c.axis)
    torch.cuda.synchronize()
    if args.call == "gemm":
        X = torch.randn(args.batch, c.cols, device="cuda:0").to(torch.float16)
        for _ in range(args.calls):
            out = hqq.hqq_gemm(q, X)
    elif args.call == "gemv":
        x = torch.randn(c.cols, device="cuda:0").to(torch.float16)
        for _ in range(args.calls):
            out = hqq.hqq_gemv(q, x)
    elif args.call == "dequant":
        for _ in range(args.calls):
            out = hqq.hqq_dequantize(q)
    else:
        for _ in range(args.calls):
            out = hqq.hqq_quantize(W, c.nbits, c.group_size, c.axis, out=q).packed
    torch.cuda.synchronize()
    print(f"ok {args.call}: {float(out.float().abs().sum()):.6g}")


if __name__ == "__main__":
    main()
