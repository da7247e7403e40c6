"""Small, self-contained cases of each kernel for profilers (ncu): each sets up its
inputs once, then calls one entry point `--iters` times.  Inputs are larger than
the 126 MB L2 but hold at most a few GB on the device.

  python profile_cases.py --case gemm_prefill --iters 3
  python profile_cases.py --case quant_prefill --iters 30 --time-cold write
cases: gemm_prefill (8192 x 14336 x 4096 NVFP4, 16-wide rotation), gemm_mxfp4,
gemm_decode (16 x 14336 x 4096), quant_prefill (8192 x 4096 rotated, dynamic
scale; _static: the tensor scale given; _static_h0: given, no rotation),
kv_load (8 x 8 x 32768 x 128 cache to FP8; --kv-batch sets the 8 sequences), kv_store, kv_attention (decode
attention over the same 8 x 8 caches, G = 4), quant_mse (the 14336 x 4096 weight,
MSE-optimal scales), gemm_quant (the prefill GEMM with its output NVFP4-encoded),
linear_decode (16 x 14336 x 4096 with the activation quantiser inside the GEMM),
gptq (MR-GPTQ of the 14336 x 4096 weight, NVFP4, 16-wide rotation).
"""
from __future__ import annotations

import argparse
import os
import sys

import numpy as np
import torch

sys.path.insert(0, os.path.dirname(os.path.abspath(__file__)))

import mxfp4_microscaled_bit_b200 as fl  # noqa: E402
import synthetic_inputs as si  # noqa: E402


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--case", required=True,
                    choices=["gemm_prefill", "gemm_mxfp4", "gemm_decode", "quant_prefill", "quant_prefill_static",
                             "quant_prefill_static_h0", "kv_load", "kv_store", "kv_attention", "quant_mse",
                             "gemm_quant", "linear_decode", "gptq"])
    ap.add_argument("--iters", type=int, default=3)
    ap.add_argument("--kv-batch", type=int, default=8,
                    help="sequences in the kv_* cases' cache (8 x 8 x 32768 x 128 by default)")
    ap.add_argument("--time-cold", choices=["write", "read"], default=None,
                    help="time each call with CUDA events after flushing the L2 by writing (or reading) "
                         "512 MiB; print the mean")
    a = ap.parse_args()
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    if a.case == "gptq":
        W = si.prefill_W().to(dev)
        K = W.shape[1]
        u = fl.gptq_hessian_factor(torch.from_numpy(si.gptq_calibration(7, 2 * K, K)).to(dev), 16)
        ws = torch.empty(int(fl.lib().gptq_workspace_bytes(W.shape[0], K)), dtype=torch.uint8, device=dev)
        fn = lambda: fl.gptq_quantize(W, u, "nvfp4", 16, workspace=ws)  # noqa: E731
    elif a.case == "linear_decode":
        M, N, K = 16, 14336, 4096
        w = fl.prepare_weight(si.decode_W(N, K).to(dev), "nvfp4", 0)
        x = si.decode_A(M, K).to(dev)
        y = torch.empty(M, N, dtype=torch.bfloat16, device=dev)
        g = torch.empty(1, dtype=torch.float32, device=dev)
        ws = torch.empty(int(fl.lib().nvfp4_linear_decode_workspace_bytes(M, N, K)), dtype=torch.uint8, device=dev)
        fn = lambda: fl.nvfp4_linear_decode(x, w.codes, w.scales, w.g, g_a=g, compute_global_scale=True,  # noqa: E731
                                            out=y, workspace=ws)
    elif a.case == "quant_mse":
        W = si.prefill_W().to(dev)
        fn = lambda: fl.nvfp4_quantize(W, 16, mse=True)  # noqa: E731
    elif a.case in ("gemm_prefill", "gemm_mxfp4", "quant_prefill", "quant_prefill_static",
                    "quant_prefill_static_h0", "gemm_quant"):
        A = si.prefill_A().to(dev)
        if a.case == "quant_prefill":
            fn = lambda: fl.nvfp4_quantize(A, 16)  # noqa: E731
        elif a.case.startswith("quant_prefill_static"):
            had = 0 if a.case.endswith("h0") else 16
            c, s, g = fl.nvfp4_quantize(A, had)  # the tensor scale, then reused as a static one
            fn = lambda: fl.nvfp4_quantize(A, had, g, codes=c, scales=s)  # noqa: E731
        elif a.case == "gemm_quant":
            w = fl.prepare_weight(si.prefill_W().to(dev), "nvfp4", 16)
            ca, sa, ga = fl.nvfp4_quantize(A, 16)
            y = fl.nvfp4_gemm(ca, sa, ga, w.codes, w.scales, w.g)
            _, _, gy = fl.nvfp4_quantize(y, 16)
            del y
            yc = torch.empty(A.shape[0], w.N // 2, dtype=torch.uint8, device=dev)
            ys = torch.empty(fl.scale_bytes(A.shape[0], w.N // 16), dtype=torch.uint8, device=dev)
            fn = lambda: fl.nvfp4_gemm_quant(ca, sa, ga, w.codes, w.scales, w.g, gy, hadamard=16,  # noqa: E731
                                             write_y=False, y_codes=yc, y_scales=ys, workspace=False)
        else:
            fmt, had = ("nvfp4", 16) if a.case == "gemm_prefill" else ("mxfp4", 32)
            w = fl.prepare_weight(si.prefill_W().to(dev), fmt, had)
            if fmt == "nvfp4":
                ca, sa, ga = fl.nvfp4_quantize(A, 16)
                y = torch.empty(A.shape[0], w.N, dtype=torch.bfloat16, device=dev)
                fn = lambda: fl.nvfp4_gemm(ca, sa, ga, w.codes, w.scales, w.g, out=y)  # noqa: E731
            else:
                ca, sa = fl.mxfp4_quantize(A, 32)
                y = torch.empty(A.shape[0], w.N, dtype=torch.bfloat16, device=dev)
                fn = lambda: fl.mxfp4_gemm(ca, sa, w.codes, w.scales, out=y)  # noqa: E731
    elif a.case == "gemm_decode":
        A = si.decode_A(16, 4096).to(dev)
        w = fl.prepare_weight(si.decode_W(14336, 4096).to(dev), "nvfp4", 0)
        ca, sa, ga = fl.nvfp4_quantize(A)
        fn = lambda: fl.nvfp4_gemm(ca, sa, ga, w.codes, w.scales, w.g)  # noqa: E731
    else:
        B, H, L, D = a.kv_batch, 8, si.KVCACHE["L"], si.KVCACHE["D"]
        x = torch.empty(B, H, L, D, dtype=torch.bfloat16)
        for b in range(B):
            for h in range(H):
                x[b, h] = si.kv_slice_bf16("k", b, h)
        g = torch.tensor([np.float32(x.abs().max().float().item()) / np.float32(2688.0)], device=dev)
        codes = torch.empty(B, H, L, D // 2, dtype=torch.uint8, device=dev)
        scales = torch.empty(B, H, L, D // 16, dtype=torch.uint8, device=dev)
        xd = x.to(dev)
        fl.kv_nvfp4_store(xd, torch.zeros(B, dtype=torch.int32, device=dev), g, codes, scales)
        if a.case == "kv_load":
            out = torch.empty(B, H, L, D, dtype=torch.uint8, device=dev)
            fn = lambda: fl.kv_nvfp4_load_fp8(codes, scales, g, L, out=out)  # noqa: E731
        elif a.case == "kv_attention":
            G = 4
            q = si.normal_bf16(7, B * H * G, D).reshape(B, H * G, D).to(dev)
            out = torch.empty(B, H * G, D, dtype=torch.float32, device=dev)
            cache = (codes, scales, g)  # K and V: the same cache, read twice as K and as V
            fn = lambda: fl.kv_nvfp4_attention(q, cache, cache, L, out=out)  # noqa: E731
        else:
            new = xd[:, :, :1].contiguous()
            pos = torch.full((B,), L - 1, dtype=torch.int32, device=dev)
            fn = lambda: fl.kv_nvfp4_store(new, pos, g, codes, scales)  # noqa: E731
    if a.time_cold:
        flush = torch.empty(512 * 2**20, dtype=torch.uint8, device=dev)
        fn()
        total = 0.0
        for _ in range(a.iters):
            if a.time_cold == "write":
                flush.zero_()
            else:
                flush.view(torch.int64).sum()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            fn()
            e1.record()
            e1.synchronize()
            total += e0.elapsed_time(e1)
        assert fl.device_status() == 0
        print(f"{a.case}: {total / a.iters * 1e3:.1f} us per call (mean of {a.iters}, L2 flushed by {a.time_cold})")
        return
    for _ in range(a.iters):
        fn()
    torch.cuda.synchronize()
    assert fl.device_status() == 0
    print(f"{a.case}: {a.iters} iterations ok")


if __name__ == "__main__":
    main()
