"""The allocation-free entry point nvfp4_quantize_noalloc, called through the C ABI.

Some callers cannot allocate device memory (plug-ins whose host framework owns the
whole device memory pool, latency-critical loops where a cudaMalloc/cudaFree would
synchronise the device).  For them the library keeps the tensor-scale partials of the
quantiser in its own fixed 4 KB array.  This test checks that two calls in a row give
the same codes, scales and tensor scale, byte for byte, as nvfp4_quantize with a
caller workspace.  It sits in a file of its own that pytest collects last, and passes
both alone in a fresh process and after the other tests.
"""
import ctypes

import numpy as np
import pytest
import torch

import mxfp4_microscaled_bit_b200 as fl
import synthetic_inputs as si

pytestmark = pytest.mark.gpu

DEV = "cuda"


def _with_workspace(x, hadamard):
    return fl.nvfp4_quantize(x, hadamard)  # compute_global_scale with a workspace it allocates


def _no_alloc(x, hadamard):
    rows, cols = x.shape
    codes = torch.full((rows, cols // 2), 0xAA, dtype=torch.uint8, device=DEV)
    scales = torch.full((fl.scale_bytes(rows, cols // 16),), 0xFF, dtype=torch.uint8, device=DEV)
    g = torch.full((1,), -1.0, dtype=torch.float32, device=DEV)
    st = fl.lib().nvfp4_quantize_noalloc(
        ctypes.c_void_p(x.data_ptr()), rows, cols, x.stride(0), hadamard, ctypes.c_void_p(g.data_ptr()),
        ctypes.c_void_p(codes.data_ptr()), ctypes.c_void_p(scales.data_ptr()),
        ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert st == 0, st
    return codes, scales, g


@pytest.mark.parametrize("hadamard", [0, 16])
def test_no_alloc_matches_workspace_entry_point(hadamard):
    # two calls in a row on different tensors: the shared array keeps the first call's
    # partials, and the second call must not see them
    first = si.student_t_bf16(71, 1000, 1024).to(DEV)
    second = (si.normal_bf16(72, 129, 4096, std=0.01)).to(DEV)  # a much smaller tensor scale
    for x in (first, second):
        c, s, g = _no_alloc(x, hadamard)
        rc, rs, rg = _with_workspace(x, hadamard)
        assert fl.device_status() == 0
        assert torch.equal(c, rc)
        assert torch.equal(s, rs)
        assert g.cpu().numpy().view(np.uint32)[0] == rg.cpu().numpy().view(np.uint32)[0]


def test_no_alloc_prefill_activations():
    x = si.prefill_A().to(DEV)
    c, s, g = _no_alloc(x, 16)
    rc, rs, rg = _with_workspace(x, 16)
    assert fl.device_status() == 0
    assert torch.equal(c, rc) and torch.equal(s, rs) and torch.equal(g, rg)


def test_python_wrapper_matches_c_abi_call():
    # the binding's nvfp4_quantize_noalloc (argument checks, then the same C call) gives the
    # bytes of the direct C-ABI call
    x = si.student_t_bf16(73, 257, 2048).to(DEV)
    c, s, g = _no_alloc(x, 16)
    wc = torch.full_like(c, 0x55)
    ws = torch.full_like(s, 0x11)
    wg = torch.full((1,), -2.0, dtype=torch.float32, device=DEV)
    fl.nvfp4_quantize_noalloc(x, 16, wg, wc, ws)
    assert fl.device_status() == 0
    assert torch.equal(wc, c) and torch.equal(ws, s) and torch.equal(wg, g)
    with pytest.raises(ValueError):
        fl.nvfp4_quantize_noalloc(x, 16, wg, wc[:-1], ws)  # a short codes buffer never reaches the C call


def test_no_alloc_rejects_bad_arguments():
    L = fl.lib()
    P = 0x10000
    assert L.nvfp4_quantize_noalloc(P, 4, 96, 96, 0, P, P, P, None) == 2   # cols not a multiple of 64
    assert L.nvfp4_quantize_noalloc(P, 4, 128, 128, 8, P, P, P, None) == 1  # rotation size
    assert L.nvfp4_quantize_noalloc(P, 4, 128, 128, 0, None, P, P, None) == 1
