#!/usr/bin/env python
"""Benchmark of the B200 NVFP4 W4A4 linear layer and NVFP4 KV cache.

One step is one pass of the whole hot path over one batch of synthetic input:
  * the prefill linear layer, M=8192 tokens, K=4096, N=14336: online NVFP4
    quantisation of the bf16 activations with the 16-wide blockwise Hadamard
    rotation and a dynamic FP32 tensor scale, then the block-scaled tcgen05 GEMM
    against pre-rotated, pre-quantised NVFP4 weights, bf16 out;
  * the KV-cache decode step on a 64 x 8 x 32768 x 128 cache: append one new
    K and one new V row per sequence in NVFP4 and dequantise both whole caches
    to FP8 E4M3 for attention.
`value` is the layer's TFLOP/s (2*M*N*K over the layer's device time); the
per-kernel rooflines, the KV and quantiser bandwidths, the MXFP4 variant and the
CPU oracle baseline are reported beside it.  Usage:

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference]

With N > 1 it runs one rank per GPU under torch.distributed.run: either the
caller launches it so (WORLD_SIZE must then equal N), or, when WORLD_SIZE is
unset, bench.py re-launches itself that way.  Each rank runs the same workload on
its own GPU (replicas: the path has no exchange step), and times are the maximum
over ranks.
"""
from __future__ import annotations

import argparse
import datetime
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import synthetic_inputs as si  # noqa: E402

FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
FP4_PER_BF16 = 4.0  # nominal dense FP4 : BF16 tensor throughput (9 : 2.25 PFLOP/s)

# DRAM bytes (read + write) per step for a kernel, from one ncu capture of the current build
# (summarised under profiles/); None where no capture covers the kernel as it stands.
NCU_TRAFFIC = {
    "gemm": 308.7e6,          # the 8192x14336x4096 prefill GEMM (CTA-pair kernel), one launch
    "mxfp4_gemm": 293.7e6,    # the same product in MXFP4 (CTA-pair kernel), one launch
    "kv_load_fp8": 6.511e9,   # 1627.6 MB per 32x8x32768x128 cache, x 2 (64 sequences) x 2 (K, V)
    "quantize": None,         # the capture covers the quantise pass only, not the amax pass
    "kv_store": None,
}
# How each traffic figure was taken, where it is not a full-size launch.
NCU_TRAFFIC_NOTE = {
    "kv_load_fp8": "DRAM bytes of a 32x8x32768x128 capture (reads 604.0 MB = the codes and scales once) scaled "
                   "x4 by the units processed; ~50 MB of that launch's writes were still in L2 when it ended "
                   "(written back after it), so the figure reads 3% below the 6.711 GB algorithmic bytes",
}
METRIC = "NVFP4 GEMM TFLOP/s (% dense FP4 peak); quantize/KV GB/s (% of HBM)"


# ------------------------------------------------------------------ distributed plumbing
def dist_env():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    return int(os.environ.get("RANK", "0")), int(os.environ.get("LOCAL_RANK", "0")), ws


def dist_init(backend: str):
    rank, local, ws = dist_env()
    if ws > 1 and not torch.distributed.is_initialized():
        torch.distributed.init_process_group(backend, timeout=datetime.timedelta(seconds=180))
    return rank, local, ws


def max_over_ranks(x: float, device="cpu") -> float:
    """Maximum of a per-rank number over all ranks (identity when not distributed)."""
    if not (torch.distributed.is_available() and torch.distributed.is_initialized()):
        return float(x)
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def barrier():
    if torch.distributed.is_available() and torch.distributed.is_initialized():
        torch.distributed.barrier()


def free_port() -> int:
    import socket
    with socket.socket() as sk:
        sk.bind(("127.0.0.1", 0))
        return sk.getsockname()[1]


def relaunch(n: int, argv: list[str]) -> int:
    """Run this script again under torch.distributed.run with n ranks on this node (127.0.0.1);
    rank 0's JSON line reaches our stdout.  Returns the launcher's exit status."""
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", f"--nproc-per-node={n}",
           "--master-addr", "127.0.0.1", "--master-port", str(free_port()), os.path.abspath(__file__), *argv]
    return subprocess.call(cmd)


def launch_check() -> int:
    """The launch alone, on CPU: join the process group over gloo, take the maximum of the rank
    numbers over all ranks, rank 0 prints it."""
    rank, _, ws = dist_init("gloo")
    m = max_over_ranks(float(rank))
    barrier()
    if rank == 0:
        print(json.dumps({"launch_check": True, "n_gpus": ws, "max_rank": m}), flush=True)
    if torch.distributed.is_initialized():
        torch.distributed.destroy_process_group()
    return 0


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return {k: float(d[k]) for k in FALLBACK_PEAKS}, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


# ------------------------------------------------------------------ clocks
class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.path = None

    def start(self):
        try:
            fd, self.path = tempfile.mkstemp(suffix=".csv")
            os.close(fd)
            self.out = open(self.path, "w")
            self.proc = subprocess.Popen(["nvidia-smi", f"--id={self.index}", f"--query-gpu={self.FIELDS}",
                                          "--format=csv,noheader,nounits", "-lms", "200"],
                                         stdout=self.out, stderr=subprocess.DEVNULL)
        except (OSError, FileNotFoundError):
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"], "samples": 0}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.out.close()
        rows = []
        with open(self.path) as f:
            for line in f:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) >= 9:
                    rows.append(parts)
        os.unlink(self.path)
        sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        mx = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({n for r in rows for n, v in zip(names, r[5:9]) if v.lower() == "active"})
        loaded = [s for s in sm if s > 500] or sm
        return {"sm_mhz": statistics.median(loaded) if loaded else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": reasons, "samples": len(rows),
                "power_w_max": max((float(r[3]) for r in rows if r[3].replace(".", "").isdigit()), default=None)}


# ------------------------------------------------------------------ workload
class Workload:
    """Device-resident inputs and outputs of one step (nothing is allocated while timing)."""

    def __init__(self, fl, dev, with_kv=True):
        P = si.PREFILL
        self.M, self.N, self.K = P["M"], P["N"], P["K"]
        self.fl, self.dev = fl, dev
        t0 = time.time()
        self.A_host = si.prefill_A().pin_memory()
        W = si.prefill_W()
        self.A = self.A_host.to(dev)
        self.W_bf16 = W.to(dev)  # kept for the bf16 context number
        self.w = fl.prepare_weight(self.W_bf16, "nvfp4", hadamard=16)  # offline: rotated + quantised once
        self.w_mx = fl.prepare_weight(self.W_bf16, "mxfp4", hadamard=32)
        del W
        M, K = self.M, self.K
        self.a_codes = torch.empty(M, K // 2, dtype=torch.uint8, device=dev)
        self.a_scales = torch.empty(fl.scale_bytes(M, K // 16), dtype=torch.uint8, device=dev)
        self.a_scales_mx = torch.empty(fl.scale_bytes(M, K // 32), dtype=torch.uint8, device=dev)
        self.g_a = torch.empty(1, dtype=torch.float32, device=dev)
        self.q_ws = torch.empty(1024, dtype=torch.float32, device=dev)
        self.y = torch.empty(M, self.N, dtype=torch.bfloat16, device=dev)
        self.y_host = torch.empty(M, self.N, dtype=torch.bfloat16).pin_memory()
        self.setup_s = {"layer": time.time() - t0}
        self.with_kv = with_kv
        if with_kv:
            self._setup_kv()

    def _setup_kv(self):
        fl, dev = self.fl, self.dev
        C = si.KVCACHE
        B, H, L, D = C["B"], C["H"], C["L"], C["D"]
        self.B, self.H, self.L, self.D = B, H, L, D
        t0 = time.time()
        self.cache = {}
        self.kv_new_host = {}
        self.kv_new = {}
        self.kv_g = {}
        for which in ("k", "v"):
            host = torch.empty(B, H, L, D, dtype=torch.bfloat16).pin_memory()

            def fill(bh):
                b, h = divmod(bh, H)
                host[b, h] = si.to_bf16(si.kv_slice(which, b, h))
                return float(host[b, h].abs().max().float())

            from concurrent.futures import ThreadPoolExecutor
            with ThreadPoolExecutor(max(1, min(32, os.cpu_count() or 1))) as ex:
                amax = max(ex.map(fill, range(B * H)))
            # static FP32 scale of the whole tensor from its bf16 values (calibration at setup, not timed)
            g = np.float32(amax) / np.float32(2688.0)
            codes = torch.empty(B, H, L, D // 2, dtype=torch.uint8, device=dev)
            scales = torch.empty(B, H, L, D // 16, dtype=torch.uint8, device=dev)
            gt = torch.tensor([g], dtype=torch.float32, device=dev)
            x = host.to(dev)
            # prefill: the first L-1 tokens through the store path
            fl.kv_nvfp4_store(x[:, :, :L - 1].contiguous(), torch.zeros(B, dtype=torch.int32, device=dev), gt,
                              codes, scales)
            self.kv_new_host[which] = host[:, :, L - 1:L].contiguous().pin_memory()
            self.kv_new[which] = x[:, :, L - 1:L].contiguous()
            del x, host
            out = torch.empty(B, H, L, D, dtype=torch.uint8, device=dev)
            osc = torch.empty(1, dtype=torch.float32, device=dev)
            self.cache[which] = (codes, scales, out, osc)
            self.kv_g[which] = gt
        self.pos = torch.full((B,), L - 1, dtype=torch.int32, device=dev)
        torch.cuda.synchronize()
        assert self.fl.device_status() == 0
        self.setup_s["kv"] = time.time() - t0

    def step(self, ev=None, A=None, y=None, kv_new=None):
        """One pass of the hot path; `ev` (5 CUDA events) brackets its four parts.  A, y, kv_new:
        other buffers of the same shapes in place of the workload's own."""
        fl = self.fl
        A = self.A if A is None else A
        y = self.y if y is None else y
        kv_new = self.kv_new if kv_new is None else kv_new
        if ev is not None:
            ev[0].record()
        fl.nvfp4_quantize(A, 16, self.g_a, compute_global_scale=True, codes=self.a_codes,
                          scales=self.a_scales, workspace=self.q_ws)
        if ev is not None:
            ev[1].record()
        fl.nvfp4_gemm(self.a_codes, self.a_scales, self.g_a, self.w.codes, self.w.scales, self.w.g, out=y,
                      workspace=False)
        if ev is not None:
            ev[2].record()
        if self.with_kv:
            for which in ("k", "v"):
                codes, scales, _, _ = self.cache[which]
                fl.kv_nvfp4_store(kv_new[which], self.pos, self.kv_g[which], codes, scales)
            if ev is not None:
                ev[3].record()
            for which in ("k", "v"):
                codes, scales, out, osc = self.cache[which]
                fl.kv_nvfp4_load_fp8(codes, scales, self.kv_g[which], self.L, out=out, out_scale=osc)
            if ev is not None:
                ev[4].record()

    LAUNCHES_PER_STEP = 7  # amax + quantise + GEMM + 2 KV stores + 2 KV loads

    def mxfp4_layer(self, ev=None):
        fl = self.fl
        if ev is not None:
            ev[0].record()
        fl.mxfp4_quantize(self.A, 32, codes=self.a_codes, scales=self.a_scales_mx)
        if ev is not None:
            ev[1].record()
        fl.mxfp4_gemm(self.a_codes, self.a_scales_mx, self.w_mx.codes, self.w_mx.scales, out=self.y,
                      workspace=False)
        if ev is not None:
            ev[2].record()

    # the layer's output as the next layer's NVFP4 input (static tensor scale, 16-wide rotation)
    def chained_setup(self):
        fl = self.fl
        self.step()
        _, _, self.g_y = fl.nvfp4_quantize(self.y, 16)  # computed once, as a calibrated static scale
        self.y_codes = torch.empty(self.M, self.N // 2, dtype=torch.uint8, device=self.dev)
        self.y_scales = torch.empty(fl.scale_bytes(self.M, self.N // 16), dtype=torch.uint8, device=self.dev)

    def gemm_then_quantize(self):
        fl = self.fl
        fl.nvfp4_gemm(self.a_codes, self.a_scales, self.g_a, self.w.codes, self.w.scales, self.w.g, out=self.y,
                      workspace=False)
        fl.nvfp4_quantize(self.y, 16, self.g_y, compute_global_scale=False, codes=self.y_codes,
                          scales=self.y_scales)

    def gemm_quant_fused(self):
        self.fl.nvfp4_gemm_quant(self.a_codes, self.a_scales, self.g_a, self.w.codes, self.w.scales, self.w.g,
                                 self.g_y, hadamard=16, write_y=False, y_codes=self.y_codes,
                                 y_scales=self.y_scales, workspace=False)

    def decode_setup(self, M=16, N=14336, K=4096, hadamard=0):
        """The decode linear layer (M activation rows, dynamic tensor scale) as two CUDA
        graphs of `copies` calls each, every call against its own copy of the weights (together
        larger than L2, so each call streams its weights from HBM): quantise then GEMM, and the
        GEMM that quantises the activations itself.  -> (unfused, fused, calls per replay)."""
        fl, dev = self.fl, self.dev
        w0 = fl.prepare_weight(si.decode_W(N, K).to(dev), "nvfp4", hadamard)
        copies = int(300e6 // (N * K * (0.5 + 1 / 16))) + 1
        Ws = [(w0.codes.clone(), w0.scales.clone(), w0.g.clone()) for _ in range(copies)]
        x = si.decode_A(M, K).to(dev)
        y = torch.empty(M, N, dtype=torch.bfloat16, device=dev)
        g = torch.empty(1, dtype=torch.float32, device=dev)
        c = torch.empty(M, K // 2, dtype=torch.uint8, device=dev)
        sc = torch.empty(fl.scale_bytes(M, K // 16), dtype=torch.uint8, device=dev)
        qws = torch.empty(1024, dtype=torch.float32, device=dev)
        gws = torch.empty(max(16, fl.gemm_workspace_bytes(M, N, K)), dtype=torch.uint8, device=dev)
        dws = torch.empty(max(16, fl.lib().nvfp4_linear_decode_workspace_bytes(M, N, K)), dtype=torch.uint8,
                          device=dev)

        def unfused(st):
            for wc, wsc, wg in Ws:
                fl.nvfp4_quantize(x, hadamard, g, compute_global_scale=True, codes=c, scales=sc, workspace=qws,
                                  stream=st)
                fl.nvfp4_gemm(c, sc, g, wc, wsc, wg, out=y, workspace=gws, stream=st)

        def fused(st):
            for wc, wsc, wg in Ws:
                fl.nvfp4_linear_decode(x, wc, wsc, wg, hadamard=hadamard, g_a=g, compute_global_scale=True, out=y,
                                       workspace=dws, stream=st)

        st = torch.cuda.Stream()
        graphs = []
        with torch.cuda.stream(st):
            for fn in (unfused, fused):
                fn(st)  # warm: kernel attributes set outside the capture
                st.synchronize()
                gr = torch.cuda.CUDAGraph()
                with torch.cuda.graph(gr, stream=st):
                    fn(st)
                graphs.append(gr)
        torch.cuda.synchronize()
        self.decode_shape = (M, N, K)
        self.decode_launches = {"unfused": 3 + (fl.gemm_workspace_bytes(M, N, K) > 0),
                                "fused": 2 + (fl.lib().nvfp4_linear_decode_workspace_bytes(M, N, K) > 4096)}
        return graphs[0].replay, graphs[1].replay, copies

    def decode_bytes(self):
        M, N, K = self.decode_shape
        return N * K * (0.5 + 1 / 16) + M * K * 2 + M * N * 2  # weights once, bf16 x in, bf16 y out

    def gptq_setup(self):
        """MR-GPTQ of the prefill weight (NVFP4, 16-wide rotation) against the damped Hessian of
        seeded calibration activations; 64 further rows of the same draw are held out to
        measure the layer's output error.  -> (callable, error ratio GPTQ / plain rounding)."""
        fl, dev = self.fl, self.dev
        N, K = self.N, self.K
        x = torch.from_numpy(si.gptq_calibration(7, 2 * K + 64, K)).to(dev)
        self.gptq_u = fl.gptq_hessian_factor(x[:2 * K], 16)
        ws = torch.empty(int(fl.lib().gptq_workspace_bytes(N, K)), dtype=torch.uint8, device=dev)
        codes = torch.empty(N, K // 2, dtype=torch.uint8, device=dev)
        scales = torch.empty(fl.scale_bytes(N, K // 16), dtype=torch.uint8, device=dev)
        g = torch.empty(1, dtype=torch.float32, device=dev)
        fn = lambda: fl.gptq_quantize(self.W_bf16, self.gptq_u, "nvfp4", 16, g, compute_global_scale=True,  # noqa: E731
                                      codes=codes, scales=scales, workspace=ws)
        fn()
        wq = fl.QuantizedWeight("nvfp4", codes, scales, g, 16, N, K)
        xh = x[2 * K:].to(torch.bfloat16)
        ref = xh.double() @ self.W_bf16.double().T
        ratio = float((fl.nvfp4_linear(xh, wq).double() - ref).norm() / (fl.nvfp4_linear(xh, self.w).double() - ref).norm())
        return fn, ratio

    def gptq_fmas(self):
        return self.N * self.K * (self.K - 1) / 2  # one multiply-add per (row, j < k)

    def attention_setup(self, G):
        """-> a callable running kv_nvfp4_attention over the decode step's caches."""
        fl = self.fl
        gen = torch.Generator(device=self.dev).manual_seed(5)
        q = torch.randn(self.B, self.H * G, self.D, generator=gen, device=self.dev).to(torch.bfloat16)
        out = torch.empty(self.B, self.H * G, self.D, dtype=torch.float32, device=self.dev)
        ws = torch.empty(fl.lib().kv_attention_workspace_bytes(self.B, self.H, G, self.L, self.D),
                         dtype=torch.uint8, device=self.dev)
        k = (self.cache["k"][0], self.cache["k"][1], self.kv_g["k"])
        v = (self.cache["v"][0], self.cache["v"][1], self.kv_g["v"])
        self.attn_G = G
        return lambda: fl.kv_nvfp4_attention(q, k, v, self.L, out=out, workspace=ws)

    def attention_bytes(self):
        return 2 * self.B * self.H * self.L * self.D * (0.5 + 1 / 16)  # K and V codes + scales, once

    # algorithmic work
    def flops(self):
        return 2.0 * self.M * self.N * self.K

    def quant_bytes(self):
        return self.M * self.K * (2 + 0.5 + 1 / 16)  # one read of A, codes + scales written

    def gemm_min_bytes(self):
        M, N, K = self.M, self.N, self.K
        return (M + N) * K * (0.5 + 1 / 16) + 2.0 * M * N

    def kv_load_bytes(self):
        return 2 * self.B * self.H * self.L * self.D * (0.5 + 1 / 16 + 1.0)  # K and V

    def kv_store_bytes(self):
        return 2 * self.B * self.H * self.D * (2 + 0.5 + 1 / 16)


def time_loop(fn, steps, stream):
    """CUDA-event time (ms) of `steps` calls of fn on `stream`."""
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(steps):
        fn()
    e1.record(stream)
    e1.synchronize()
    return e0.elapsed_time(e1)


# ------------------------------------------------------------------ CPU oracle baseline
class OracleLayer:
    """The oracle as it stands, on this host's cores: the prefill layer on a sample of rows."""

    def __init__(self):
        import oracle
        oracle.lib()
        self.o = oracle
        W = si.prefill_W()
        wc, ws, wg = oracle.nvfp4_quantize(W, 16)  # weight preparation is offline, as on the GPU
        self.Wd = oracle.dequant(wc, ws, "nvfp4", wg)

    def run(self, rows: int):
        """Quantise rows 0..rows-1 of the activations (H16 rotation, tensor scale of the sample) and
        multiply them against all weight rows in fp64; returns (TFLOP/s, seconds)."""
        o = self.o
        A = si.prefill_A(0, rows)
        t0 = time.perf_counter()
        ac, as_, ag = o.nvfp4_quantize(A, 16)
        y, _ = o.gemm_abt(o.dequant(ac, as_, "nvfp4", ag), self.Wd)
        dt = time.perf_counter() - t0
        return 2.0 * rows * si.PREFILL["N"] * si.PREFILL["K"] / dt / 1e12, dt

    def describe(self, rows, dt):
        return {"cores": self.o.num_threads(), "kind": "oracle",
                "sample": f"prefill layer, activation rows 0..{rows - 1} of 8192 quantised with the H16 rotation "
                          f"and multiplied in fp64 against all 14336 pre-quantised weight rows ({dt:.2f} s)"}


def cpu_baseline(rows: int = 1024):
    ol = OracleLayer()
    v, dt = ol.run(rows)
    return {"value": v, "unit": "TFLOP/s", **ol.describe(rows, dt)}


def reference_arm(args):
    """The reference arm: the oracle timed on the host cores, one bounded sample per step."""
    rank, _, ws = dist_env()
    if rank != 0:
        return 0
    ol = OracleLayer()
    # about 8 ms of fp64 work per row on 8-16 cores: keep the whole run under a couple of minutes
    rows = int(min(256, max(8, round(45.0 / max(1, args.steps + args.warmup) / 0.008))))
    for _ in range(args.warmup):
        ol.run(rows)
    vals, secs = [], []
    for _ in range(max(1, args.steps)):
        v, dt = ol.run(rows)
        vals.append(v)
        secs.append(dt)
    v = statistics.median(vals)
    d = ol.describe(rows, statistics.median(secs))
    line = {"metric": METRIC, "value": v, "unit": "TFLOP/s", "n_gpus": ws, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": 1e3 * statistics.median(secs), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "impl": "reference", "config": config_dict(),
            "cpu_baseline": {"value": v, "unit": "TFLOP/s", **d},
            "e2e": {"value": v, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


def config_dict():
    P, C = si.PREFILL, si.KVCACHE
    return {"workload": f"prefill NVFP4 W4A4 linear layer M={P['M']} K={P['K']} N={P['N']}, 16-wide Hadamard "
                        f"rotation, dynamic tensor scale (Student-t nu=3 activations, N(0,0.02^2) weights) + "
                        f"NVFP4 KV decode step B={C['B']} H={C['H']} L={C['L']} D={C['D']}",
            "M": P["M"], "N": P["N"], "K": P["K"], "hadamard": 16,
            "kv": [C["B"], C["H"], C["L"], C["D"]],
            "l2": "inputs larger than L2: every step streams 6.7 GB of KV cache after the layer, so no layer "
                  "operand is L2-resident when the next step starts",
            "parallelism": "replicas"}


# ------------------------------------------------------------------ main
def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=1000)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--e2e-steps", type=int, default=10)
    ap.add_argument("--cpu-rows", type=int, default=1024)
    ap.add_argument("--launch-check", action="store_true",
                    help="only start the N ranks, join them over gloo and report (no GPU work)")
    args = ap.parse_args()
    args.warmup = max(3, args.warmup)
    if args.gpus < 1:
        print(f"bench.py: --gpus must be >= 1, not {args.gpus}", file=sys.stderr)
        return 2
    if args.gpus > 1 and "WORLD_SIZE" not in os.environ:
        return relaunch(args.gpus, sys.argv[1:])
    if dist_env()[2] != args.gpus:
        print(f"bench.py: --gpus {args.gpus} but WORLD_SIZE={dist_env()[2]}: launch one rank per GPU",
              file=sys.stderr)
        return 2
    if args.launch_check:
        return launch_check()

    if args.impl == "reference":
        return reference_arm(args)

    rank, local, ws = dist_init("nccl")
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    import mxfp4_microscaled_bit_b200 as fl
    fl.lib()
    peaks, peak_src = load_peaks()
    stream = torch.cuda.current_stream()

    w = Workload(fl, dev)
    torch.cuda.synchronize()
    # warm-up (untimed)
    for _ in range(args.warmup):
        w.step()
    torch.cuda.synchronize()
    assert fl.device_status() == 0

    # ---- timed region: exactly `steps` steps, barrier + synchronize on both sides
    nparts = 5
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(nparts)] for _ in range(args.steps)]
    clocks = ClockSampler(torch.cuda.current_device())
    clocks.start()
    time.sleep(0.3)
    barrier()
    torch.cuda.synchronize()
    t_start, t_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t_start.record(stream)
    for i in range(args.steps):
        w.step(evs[i])
    t_end.record(stream)
    torch.cuda.synchronize()
    barrier()
    clk = clocks.stop()
    assert fl.device_status() == 0
    total_ms = t_start.elapsed_time(t_end)
    parts = np.array([[e[j].elapsed_time(e[j + 1]) for j in range(nparts - 1)] for e in evs])  # ms
    q_ms, gemm_ms, st_ms, ld_ms = (float(np.mean(parts[:, j])) for j in range(4))
    layer_ms = q_ms + gemm_ms

    total_ms_max = max_over_ranks(total_ms, dev)
    layer_ms_max = max_over_ranks(layer_ms, dev)
    gemm_ms_max = max_over_ranks(gemm_ms, dev)

    # ---- MXFP4 variant of the same layer (reported, not part of the step): quantise + GEMM, the
    #      GEMM's own time from events around it
    for _ in range(3):
        w.mxfp4_layer()
    mx_ev = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(20)]
    for e in mx_ev:
        w.mxfp4_layer(e)
    torch.cuda.synchronize()
    mx_ms = float(np.mean([e[0].elapsed_time(e[2]) for e in mx_ev]))
    mx_gemm_ms = float(np.mean([e[1].elapsed_time(e[2]) for e in mx_ev]))

    # ---- the MXFP4 comparison on the prefill shape: relative Frobenius error of each format's layer
    #      output (with and without rotation) against the float64 product of the unquantised
    #      operands, on the first 128 activation rows (every weight row)
    def rel_frobenius():
        rows = 128
        exact = w.A[:rows].double() @ w.W_bf16.double().T
        out = {}
        for name, fmt, had in (("nvfp4_h16", "nvfp4", 16), ("nvfp4", "nvfp4", 0), ("mxfp4_h32", "mxfp4", 32),
                               ("mxfp4", "mxfp4", 0)):
            wq = w.w if (fmt, had) == ("nvfp4", 16) else (w.w_mx if (fmt, had) == ("mxfp4", 32)
                                                          else fl.prepare_weight(w.W_bf16, fmt, had))
            lin = fl.nvfp4_linear if fmt == "nvfp4" else fl.mxfp4_linear
            y = lin(w.A, wq)[:rows].double()
            out[name] = float((y - exact).norm() / exact.norm())
            del wq
        return out

    c3_err = rel_frobenius()
    assert fl.device_status() == 0

    # ---- the output handed to a next NVFP4 layer: GEMM then quantiser vs the fused epilogue
    w.chained_setup()
    for _ in range(3):
        w.gemm_then_quantize()
        w.gemm_quant_fused()
    unfused_ms = time_loop(w.gemm_then_quantize, 20, stream) / 20
    fused_ms = time_loop(w.gemm_quant_fused, 20, stream) / 20
    assert fl.device_status() == 0

    # ---- context: cuBLAS bf16 on the same prefill product (torch.matmul of the unquantised operands)
    a_bf = w.A
    w_bf = w.W_bf16
    y_bf = torch.empty_like(w.y)
    mm = lambda: torch.matmul(a_bf, w_bf.t(), out=y_bf)
    for _ in range(3):
        mm()
    bf16_ms = time_loop(mm, 10, stream) / 10
    del w_bf, y_bf

    # ---- the decode linear layer: quantise then GEMM vs the GEMM that quantises its input
    dec_unfused, dec_fused, dec_calls = w.decode_setup()
    for _ in range(3):
        dec_unfused()
        dec_fused()
    dec_unfused_us = time_loop(dec_unfused, 10, stream) / (10 * dec_calls) * 1e3
    dec_fused_us = time_loop(dec_fused, 10, stream) / (10 * dec_calls) * 1e3
    assert fl.device_status() == 0

    # ---- MR-GPTQ of the prefill weight (offline weight preparation; reported, not part of the step)
    gptq_fn, gptq_ratio = w.gptq_setup()
    for _ in range(2):
        gptq_fn()
    gptq_ms = time_loop(gptq_fn, 3, stream) / 3
    assert fl.device_status() == 0

    # ---- decode attention straight from the NVFP4 caches (G = 4 query heads per kv head)
    attn = w.attention_setup(4)
    for _ in range(3):
        attn()
    attn_ms = time_loop(attn, 10, stream) / 10
    assert fl.device_status() == 0

    # ---- end to end through the public API with host buffers: H2D of A and the new K/V rows,
    #      the step, D2H of y and the FP8 output scales
    def e2e_step():
        w.A.copy_(w.A_host, non_blocking=True)
        for which in ("k", "v"):
            w.kv_new[which].copy_(w.kv_new_host[which], non_blocking=True)
        w.step()
        w.y_host.copy_(w.y, non_blocking=True)
        osc = [w.cache[k][3] for k in ("k", "v")]
        return osc

    e2e_osc_host = torch.empty(2, dtype=torch.float32).pin_memory()

    def e2e_full():
        osc = e2e_step()
        e2e_osc_host[0:1].copy_(osc[0], non_blocking=True)
        e2e_osc_host[1:2].copy_(osc[1], non_blocking=True)

    for _ in range(2):
        e2e_full()
    torch.cuda.synchronize()
    barrier()
    e2e_serial_ms = time_loop(e2e_full, args.e2e_steps, stream) / args.e2e_steps
    e2e_serial_ms = max_over_ranks(e2e_serial_ms, dev)

    # ---- the same, pipelined as a serving loop would run it: two sets of device buffers; each
    #      step's copies in (A, the new K/V rows) and out (y, the FP8 output scales) run on copy
    #      streams, overlapping the neighbouring steps' compute; every copy stays in the timed region
    A_dev = [w.A, torch.empty_like(w.A)]
    y_dev = [w.y, torch.empty_like(w.y)]
    kv_dev = [w.kv_new, {k: torch.empty_like(v) for k, v in w.kv_new.items()}]
    y_host = [w.y_host, torch.empty(w.y.shape, dtype=w.y.dtype, pin_memory=True)]
    osc_host = [torch.empty(2, dtype=torch.float32, pin_memory=True) for _ in range(2)]
    s_in, s_out = torch.cuda.Stream(), torch.cuda.Stream()
    ev_in, ev_done, ev_out = ([torch.cuda.Event() for _ in range(2)] for _ in range(3))

    def e2e_pipelined(n):
        s_in.wait_stream(stream)
        for i in range(n):
            b = i & 1
            with torch.cuda.stream(s_in):
                if i >= 2:
                    s_in.wait_event(ev_done[b])  # buffers b were read by step i - 2
                A_dev[b].copy_(w.A_host, non_blocking=True)
                for which in ("k", "v"):
                    kv_dev[b][which].copy_(w.kv_new_host[which], non_blocking=True)
                ev_in[b].record(s_in)
            stream.wait_event(ev_in[b])
            if i >= 2:
                stream.wait_event(ev_out[b])  # y of step i - 2 has left the device
            w.step(A=A_dev[b], y=y_dev[b], kv_new=kv_dev[b])
            ev_done[b].record(stream)
            with torch.cuda.stream(s_out):
                s_out.wait_event(ev_done[b])
                y_host[b].copy_(y_dev[b], non_blocking=True)
                osc_host[b][0:1].copy_(w.cache["k"][3], non_blocking=True)
                osc_host[b][1:2].copy_(w.cache["v"][3], non_blocking=True)
                ev_out[b].record(s_out)
        stream.wait_stream(s_out)

    e2e_pipelined(2)
    torch.cuda.synchronize()
    barrier()
    e2e_ms = time_loop(lambda: e2e_pipelined(args.e2e_steps), 1, stream) / args.e2e_steps
    e2e_ms = max_over_ranks(e2e_ms, dev)
    h2d = w.A.numel() * 2 + sum(w.kv_new[k].numel() * 2 for k in ("k", "v"))
    d2h = w.y.numel() * 2 + 8

    # ---- results
    flops = w.flops()
    sustained_fp4 = peaks["bf16_tflops_sustained"] * FP4_PER_BF16
    burst_fp4 = peaks["bf16_tflops"] * FP4_PER_BF16
    hbm = peaks["hbm_gbs"]
    fp32_fma_peak = 148 * 128 * float(clk.get("sm_mhz") or 1965.0) * 1e6 / 1e12  # TFMA/s

    def hbm_roof(bytes_, ms):
        gbs = bytes_ / (ms * 1e-3) / 1e9
        return {"bound": "hbm", "achieved": gbs, "peak": hbm, "unit": "GB/s", "frac": gbs / hbm,
                "traffic": None, "algorithmic_bytes": bytes_, "ms": ms}

    gemm_tf = flops / (gemm_ms * 1e-3) / 1e12
    # the FP4 tensor pipe's own rate at the sampled clock: one 128x256x64 block-scaled MMA per SM
    # every 128 cycles (measured with a stream of MMAs and no other work), 148 SMs
    clock_fp4 = 148 * (2 * 128 * 256 * 64 / 128) * float(clk.get("sm_mhz") or 1965.0) * 1e6 / 1e12
    mx_gemm_tf = flops / (mx_gemm_ms * 1e-3) / 1e12
    rooflines = {
        "gemm": {"bound": "tensor", "achieved": gemm_tf, "peak": burst_fp4, "unit": "TFLOP/s",
                 "frac": gemm_tf / burst_fp4, "traffic": None, "ms": gemm_ms,
                 "peak_basis": f"{peak_src} bf16 burst x {FP4_PER_BF16:g} (dense FP4 : BF16); the step's GEMMs "
                               f"run in a short region at full clock",
                 "frac_of_sustained_fp4": gemm_tf / sustained_fp4, "frac_of_clock_fp4": gemm_tf / clock_fp4,
                 "clock_fp4_tflops": clock_fp4, "frac_of_datasheet_9pf": gemm_tf / 9000.0},
        "mxfp4_gemm": {"bound": "tensor", "achieved": mx_gemm_tf, "peak": burst_fp4, "unit": "TFLOP/s",
                       "frac": mx_gemm_tf / burst_fp4, "traffic": None, "ms": mx_gemm_ms,
                       "frac_of_clock_fp4": mx_gemm_tf / clock_fp4},
        "kv_load_fp8": hbm_roof(w.kv_load_bytes(), ld_ms),
        "quantize": hbm_roof(w.quant_bytes(), q_ms),
        "kv_store": hbm_roof(w.kv_store_bytes(), st_ms),
    }
    for k, r in rooflines.items():
        r["traffic"] = NCU_TRAFFIC.get(k)
        if k in NCU_TRAFFIC_NOTE:
            r["traffic_note"] = NCU_TRAFFIC_NOTE[k]
    rooflines["quantize"]["note"] = ("2.5625 B/element (one read of A); the dynamic tensor scale reads A twice: "
                                     "frac_of_bytes_moved counts the 4.5625 B/element the two passes move")
    q_moved = w.quant_bytes() + 2.0 * w.M * w.K  # plus the second read of A
    rooflines["quantize"]["frac_of_bytes_moved"] = q_moved / (q_ms * 1e-3) / 1e9 / hbm
    rooflines["kv_load_fp8"]["frac_of_8tbs"] = rooflines["kv_load_fp8"]["achieved"] / 8000.0
    shares = {"quantize": q_ms, "gemm": gemm_ms, "kv_store": st_ms, "kv_load_fp8": ld_ms}
    dominant = max(shares, key=shares.get)
    roof = dict(rooflines[dominant])
    roof["kernel"] = dominant
    # every timed kernel's roofline in brief, beside the dominant one's
    roof["kernels"] = {k: {"achieved": r["achieved"], "peak": r["peak"], "unit": r["unit"], "frac": r["frac"],
                           "ms": r["ms"]} for k, r in rooflines.items()}
    roof["kernels"]["gemm"]["frac_of_clock_fp4"] = gemm_tf / clock_fp4
    roof["kernels"]["quantize"]["frac_of_bytes_moved"] = rooflines["quantize"]["frac_of_bytes_moved"]
    roof["kernels"]["mxfp4_gemm"]["frac_of_clock_fp4"] = mx_gemm_tf / clock_fp4
    roof["kernels"]["mxfp4_gemm"]["layer_tflops"] = flops / (mx_ms * 1e-3) / 1e12
    roof["kernels"]["mxfp4_gemm"]["rel_frobenius_error"] = c3_err

    layer_tf = ws * flops / (layer_ms_max * 1e-3) / 1e12
    line = {
        "metric": METRIC,
        "value": layer_tf,
        "unit": "TFLOP/s",
        "n_gpus": ws,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": total_ms_max / args.steps,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "nvfp4",
        "data": "synthetic",
        "config": config_dict(),
        "roofline": roof,
        "rooflines": rooflines,
        "step_ms": {"quantize": q_ms, "gemm": gemm_ms, "kv_store": st_ms, "kv_load_fp8": ld_ms,
                    "layer": layer_ms, "share": {k: v / sum(shares.values()) for k, v in shares.items()}},
        "metrics": {"layer_tflops": layer_tf, "gemm_tflops": gemm_tf,
                    "gemm_frac_dense_fp4": gemm_tf / burst_fp4,
                    "quantize_gbs": rooflines["quantize"]["achieved"],
                    "kv_load_gbs": rooflines["kv_load_fp8"]["achieved"],
                    "kv_store_us": st_ms * 1e3,
                    "mxfp4_layer_tflops": flops / (mx_ms * 1e-3) / 1e12,
                    "mxfp4_vs_nvfp4": {"layer_tflops": {"nvfp4_h16": layer_tf, "mxfp4_h32": flops / (mx_ms * 1e-3) / 1e12},
                                       "rel_frobenius_error": c3_err,
                                       "note": "prefill shape; errors of the layer output on activation rows "
                                               "0..127 against the float64 product of the unquantised bf16 "
                                               "operands"},
                    "bf16_matmul_context": {"ms": bf16_ms, "tflops": flops / (bf16_ms * 1e-3) / 1e12,
                                            "layer_speedup": bf16_ms / layer_ms, "gemm_speedup": bf16_ms / gemm_ms,
                                            "note": "torch.matmul (cuBLAS) bf16 on the unquantised prefill "
                                                    "operands, back-to-back calls"},
                    "kv_attention": {
                        "ms": attn_ms, "G": w.attn_G,
                        "gbs": w.attention_bytes() / (attn_ms * 1e-3) / 1e9,
                        "frac_hbm": w.attention_bytes() / (attn_ms * 1e-3) / 1e9 / hbm,
                        "kv_load_fp8_ms": ld_ms,
                        "note": "decode attention over the NVFP4 caches with the FP8 values formed on chip; "
                                "kv_load_fp8_ms is the step's FP8 load of the same caches, which an FP8 "
                                "attention kernel would then read back"},
                    "decode_layer": {
                        "shape_mnk": list(w.decode_shape), "unfused_us": dec_unfused_us, "fused_us": dec_fused_us,
                        "speedup": dec_unfused_us / dec_fused_us,
                        "fused_gbs": w.decode_bytes() / (dec_fused_us * 1e-6) / 1e9,
                        "fused_frac_hbm": w.decode_bytes() / (dec_fused_us * 1e-6) / 1e9 / hbm,
                        "launches": w.decode_launches,
                        "note": "decode config (no rotation), dynamic tensor scale; nvfp4_quantize + nvfp4_gemm vs "
                                "nvfp4_linear_decode (amax pass + the GEMM that encodes its input + split-K "
                                "reduction); CUDA-graph replay, each call on its own weight copy (> L2)"},
                    "gptq": {
                        "ms": gptq_ms, "shape_nk": [w.N, w.K],
                        "tfma_per_s": w.gptq_fmas() / (gptq_ms * 1e-3) / 1e12,
                        "roofline": {"bound": "alu", "unit": "TFMA/s",
                                     "achieved": w.gptq_fmas() / (gptq_ms * 1e-3) / 1e12,
                                     "peak": fp32_fma_peak, "frac": w.gptq_fmas() / (gptq_ms * 1e-3) / 1e12 / fp32_fma_peak,
                                     "peak_basis": "148 SMs x 128 binary32 FMA lanes x the median SM clock under load"},
                        "output_error_vs_rounding": gptq_ratio,
                        "note": "NVFP4, 16-wide rotation, binary32 sweep; output error on 64 held-out rows of "
                                "the calibration draw, GPTQ weights / plainly rounded weights, same layer"},
                    "next_layer_input": {
                        "gemm_then_quantize_ms": unfused_ms, "gemm_quant_fused_ms": fused_ms,
                        "speedup": unfused_ms / fused_ms,
                        "note": "y handed on as NVFP4 (static g_y, H16): nvfp4_gemm + nvfp4_quantize vs "
                                "nvfp4_gemm_quant without bf16 y; back-to-back calls, operands L2-warm"}},
        "e2e": {"value": ws * flops / (e2e_ms * 1e-3) / 1e12, "unit": "TFLOP/s", "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms,
                "serial_ms_per_step": e2e_serial_ms,
                "note": "public API, pinned host buffers; copies of step i+1 in and step i-1 out overlap step i "
                        "(two device buffer sets); serial_ms_per_step: the same with copy, step, copy in sequence"},
        "gpu_launches": Workload.LAUNCHES_PER_STEP * args.steps,
        "clocks": clk,
        "peaks": {**peaks, "source": peak_src},
        "setup_s": w.setup_s,
    }
    if rank == 0 and ws == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(args.cpu_rows)
    if rank == 0:
        print(json.dumps(line), flush=True)
    barrier()
    if torch.distributed.is_initialized():
        torch.distributed.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
