"""Run one libbsq kernel a few times at a given shape, for profiler captures.

    python profile_case.py w4a4 --m 4096 --n 17408 --k 5120 --iters 3

Inputs are random codes in device memory (the kernel's cost does not depend
on their values beyond power); nothing is checked.  Kinds: w4a4 (M <= 128
runs the few-row kernel), fp8gemm, int8gemm, int8gemm_ws (with the
tail-splitting workspace), gemv, gemv_bs (block-scaled),
quant_nvfp4, quant_rowfp8, quant_int8, requant_w, requant_block.
"""
from __future__ import annotations

import argparse
import os
import sys

import torch

sys.path.insert(0, os.path.dirname(os.path.abspath(__file__)))

import int8_gemm_gemv_b200 as bsq


def main():
    p = argparse.ArgumentParser()
    p.add_argument("kind")
    p.add_argument("--m", type=int, default=4096)
    p.add_argument("--n", type=int, default=17408)
    p.add_argument("--k", type=int, default=5120)
    p.add_argument("--iters", type=int, default=3)
    a = p.parse_args()
    m, n, k = a.m, a.n, a.k
    dev = "cuda"
    g = torch.Generator(device=dev)
    g.manual_seed(0)

    def u8(shape, lo=0, hi=256):
        return torch.randint(lo, hi, shape, dtype=torch.uint8, device=dev, generator=g)

    def bf16(shape, std=1.0):
        return (torch.randn(shape, device=dev, generator=g) * std).to(torch.bfloat16)

    out = torch.empty((m, n), dtype=torch.int16, device=dev) if a.kind in ("w4a4", "fp8gemm", "int8gemm", "int8gemm_ws", "gemv",
                                                                          "gemv_bs") else None
    if a.kind == "w4a4":
        ap, asf, wp, wsf = u8((m, k // 2)), u8((m, k // 16), 0x30, 0x40), u8((n, k // 2)), u8((n, k // 16), 0x30, 0x40)
        fn = lambda: bsq.w4a4_gemm(ap, asf, wp, wsf, out, 1.0, 1.0, m, n, k)
    elif a.kind == "fp8gemm":
        x, w = u8((m, k), 0, 0x7F), u8((n, k), 0, 0x7F)
        sa, sw = torch.rand(m, device=dev), torch.rand(n, device=dev)
        fn = lambda: bsq.fp8_gemm_rowscale(x, sa, w, sw, out, m, n, k)
    elif a.kind in ("int8gemm", "int8gemm_ws"):
        x = torch.randint(-127, 128, (m, k), dtype=torch.int8, device=dev)
        w = torch.randint(-127, 128, (n, k), dtype=torch.int8, device=dev)
        sa, sw = torch.rand(m, k // 32, device=dev), torch.rand(n, k // 32, device=dev)
        if a.kind == "int8gemm":
            fn = lambda: bsq.int8_blockscaled_gemm(x, w, sa, sw, out, m, n, k)
        else:
            nb = bsq.int8_gemm_workspace_bytes()
            ws = torch.zeros(nb, dtype=torch.uint8, device=dev)
            fn = lambda: bsq.int8_blockscaled_gemm_ws(x, w, sa, sw, out, ws, nb, m, n, k)
    elif a.kind == "gemv_bs":
        x, w = bf16((m, k)), u8((n, k), 0, 0x7F)
        S = torch.rand(n // 128, k // 128, device=dev)
        fn = lambda: bsq.fp8_gemv_blockscaled(x, w, S, out, m, n, k)
    elif a.kind == "gemv":
        x, w, s = bf16((m, k)), u8((n, k), 0, 0x7F), torch.rand(n, device=dev)
        fn = lambda: bsq.fp8_gemv_rowscale(x, w, s, out, m, n, k)
    elif a.kind == "quant_nvfp4":
        x = bf16((m, k))
        p_, s_ = u8((m, k // 2)), u8((m, k // 16))
        fn = lambda: bsq.quantize_bf16_to_nvfp4(x, p_, s_, 1.0, m, k)
    elif a.kind == "quant_rowfp8":
        x = bf16((m, k))
        q, s = u8((m, k)), torch.empty(m, device=dev)
        fn = lambda: bsq.quant_rowwise_fp8(x, q, s, m, k)
    elif a.kind == "quant_int8":
        x = bf16((m, k))
        q, s = torch.empty((m, k), dtype=torch.int8, device=dev), torch.empty((m, k // 32), device=dev)
        fn = lambda: bsq.quant_act_int8_per32(x, q, s, m, k)
    elif a.kind == "requant_w":
        wp, wsf = u8((n, k // 2)), u8((n, k // 16), 0x30, 0x40)
        q, s = torch.empty((n, k), dtype=torch.int8, device=dev), torch.empty((n, k // 32), device=dev)
        fn = lambda: bsq.requant_w_nvfp4_int8(wp, wsf, 1e-3, q, s, n, k)
    elif a.kind == "requant_block":
        w, S = u8((n, k), 0, 0x7F), torch.rand(n // 128, k // 128, device=dev)
        q, s = u8((n, k)), torch.empty(n, device=dev)
        fn = lambda: bsq.requant_blockfp8_to_rowwise(bsq.BSQ_FP8_BLOCK_SCALED, w, S, n, k, q, s)
    else:
        raise SystemExit(f"unknown kind {a.kind}")
    for _ in range(a.iters):
        fn()
    torch.cuda.synchronize()
    t = bsq.debug_take_timeouts()
    if t:
        raise SystemExit(f"kernel wait timeouts: {t:#x}")


if __name__ == "__main__":
    main()
