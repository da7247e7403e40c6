"""Shared helpers of the GPU parity tests (CUDA path vs the oracle)."""
import numpy as np
import torch

import mxfp4_microscaled_bit_b200 as fl

DEV = "cuda"


def status_ok():
    st = fl.device_status()
    assert st == 0, f"device status {st}"


def gpu_nvfp4(x_cpu, hadamard=0, g=None):
    """Quantise on the GPU into poisoned buffers; returns numpy (codes, scale bytes, g)."""
    x = x_cpu.to(DEV)
    rows, cols = x.shape
    codes = torch.full((rows, cols // 2), 0xAA, dtype=torch.uint8, device=DEV)
    scales = torch.full((fl.scale_bytes(rows, cols // 16),), 0xFF, dtype=torch.uint8, device=DEV)
    gt = None if g is None else torch.tensor([g], dtype=torch.float32, device=DEV)
    c, s, gg = fl.nvfp4_quantize(x, hadamard, gt, codes=codes, scales=scales)
    status_ok()
    return c, s, gg


def gpu_mxfp4(x_cpu, hadamard=0):
    x = x_cpu.to(DEV)
    rows, cols = x.shape
    codes = torch.full((rows, cols // 2), 0xAA, dtype=torch.uint8, device=DEV)
    scales = torch.full((fl.scale_bytes(rows, cols // 32),), 0xFF, dtype=torch.uint8, device=DEV)
    c, s = fl.mxfp4_quantize(x, hadamard, codes=codes, scales=scales)
    status_ok()
    return c, s


def assert_bytes_equal(got, ref, what):
    got = np.asarray(got)
    ref = np.asarray(ref)
    assert got.shape == ref.shape, (what, got.shape, ref.shape)
    bad = np.nonzero(got.reshape(-1) != ref.reshape(-1))[0]
    assert bad.size == 0, f"{what}: {bad.size} mismatches, first at {bad[:8]}: got {got.reshape(-1)[bad[:8]]} want {ref.reshape(-1)[bad[:8]]}"


def check_nvfp4(orc, x_cpu, hadamard=0, g=None):
    """GPU vs oracle, bit for bit: codes, every scale byte (padding included), tensor scale."""
    c, s, gg = gpu_nvfp4(x_cpu, hadamard, g)
    oc, osl, og = orc.nvfp4_quantize(x_cpu, hadamard, g)
    gpu_g = gg.cpu().numpy().astype(np.float32)
    assert gpu_g.view(np.uint32)[0] == np.float32(og).view(np.uint32), (gpu_g[0], og)
    assert_bytes_equal(c.cpu().numpy(), oc, "codes")
    assert_bytes_equal(s.cpu().numpy(), orc.tc_scale_layout(osl), "scales")
    return c, s, gg, oc, osl, og


def check_mxfp4(orc, x_cpu, hadamard=0):
    c, s = gpu_mxfp4(x_cpu, hadamard)
    oc, osl = orc.mxfp4_quantize(x_cpu, hadamard)
    assert_bytes_equal(c.cpu().numpy(), oc, "codes")
    assert_bytes_equal(s.cpu().numpy(), orc.tc_scale_layout(osl), "scales")
    return c, s, oc, osl


def bf16_window(orc, y_ref, s, rel=1e-4):
    """[lo, hi] bf16 values allowed by |y - y_ref| <= rel * sum|a b| before the bf16 rounding
    (round-to-nearest is monotone, so rounding both ends gives the exact window)."""
    lo = orc.bf16_bits_to_f64(orc.bf16_rn(y_ref - rel * s))
    hi = orc.bf16_bits_to_f64(orc.bf16_rn(y_ref + rel * s))
    return lo, hi


def check_gemm_values(orc, y_gpu, y_ref, s, what, rel=1e-4):
    y = np.asarray(y_gpu, dtype=np.float64)
    lo, hi = bf16_window(orc, y_ref, s, rel)
    bad = np.nonzero((y < lo) | (y > hi))
    err = np.abs(y - y_ref) / np.maximum(s, 1e-300)
    assert bad[0].size == 0, (f"{what}: {bad[0].size} of {y.size} outside the window; worst rel err "
                              f"{err.max():.3e}; first {list(zip(*[b[:5] for b in bad]))}")
    return float(err.max())
