"""The C ABI without a GPU: the library builds and loads, exports every entry point
include/fp4lin.h declares, and its host-side checks return the documented status
without launching anything (fake device pointers are never dereferenced)."""
import ctypes
import os
import re

import pytest

import mxfp4_microscaled_bit_b200 as fl

HEADER = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include", "fp4lin.h")

OK, INVALID, SHAPE, MISALIGNED, WORKSPACE = 0, 1, 2, 3, 7
P = 0x10000  # a 16-byte aligned fake device address; never dereferenced on these paths


def header_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"^\s*(?:int|int64_t|size_t)\s+(\w+)\s*\(", src, flags=re.M)))


def test_every_declared_symbol_is_exported():
    names = header_functions()
    assert len(names) == 31, names
    L = fl.lib()
    for n in names:
        assert hasattr(L, n), n
    assert set(names) == set(fl.EXPORTS)


def test_library_has_no_driver_dependency():
    # the runtime is linked statically and the driver is reached through an entry-point query,
    # so the library loads on a host without libcuda
    out = os.popen(f"ldd {fl.library_path()}").read()
    assert "libcuda.so" not in out and "libcudart.so" not in out


def test_sizes():
    L = fl.lib()
    assert L.fp4lin_version() == 100
    assert L.fp4lin_scale_bytes(1, 1) == 512
    assert L.fp4lin_scale_bytes(128, 4) == 512
    assert L.fp4lin_scale_bytes(129, 8) == 2048
    assert L.fp4lin_scale_bytes(8192, 256) == 8192 * 256
    assert L.nvfp4_quantize_workspace_bytes(8192, 4096) == 4096
    # prefill shape needs no split; decode shapes split K over the SMs
    assert L.fp4lin_gemm_workspace_bytes(8192, 14336, 4096) == 0
    assert L.fp4lin_gemm_workspace_bytes(16, 4096, 4096) > 0


def quant_call(x=P, rows=16, cols=128, ld=128, had=0, dyn=0, g=P, codes=P, scales=P, ws=P, wsb=4096, fn="nvfp4_quantize"):
    return getattr(fl.lib(), fn)(x, rows, cols, ld, had, dyn, g, codes, scales, ws, wsb, None)


@pytest.mark.parametrize("fn", ["nvfp4_quantize", "nvfp4_quantize_mse"])
def test_nvfp4_quantize_argument_checks(fn):
    def q(**kw):
        return quant_call(fn=fn, **kw)

    assert q(x=None) == INVALID
    assert q(codes=None) == INVALID
    assert q(g=None) == INVALID
    assert q(rows=0) == INVALID
    assert q(ld=64) == INVALID
    assert q(had=8) == INVALID
    assert q(dyn=2) == INVALID
    assert q(cols=96, ld=96) == SHAPE
    assert q(ld=132) == SHAPE
    assert q(x=P + 8) == MISALIGNED
    assert q(scales=P + 4) == MISALIGNED
    assert q(dyn=1, ws=None) == WORKSPACE
    assert q(dyn=1, wsb=100) == WORKSPACE


@pytest.mark.parametrize("fn", ["mxfp4_quantize", "mxfp4_quantize_nearest"])
def test_mxfp4_quantize_argument_checks(fn):
    f = getattr(fl.lib(), fn)
    assert f(P, 4, 128, 128, 16, P, P, None) == INVALID
    assert f(P, 4, 96, 96, 0, P, P, None) == SHAPE
    assert f(P + 2, 4, 128, 128, 0, P, P, None) == MISALIGNED


def g(M=16, N=64, K=128, ldy=64, a=P, y=P, ga=P):
    return fl.lib().nvfp4_gemm(a, P, ga, P, P, P, y, M, N, K, ldy, None, 0, None)


def test_gemm_argument_checks():
    assert g(a=None) == INVALID
    assert g(ga=None) == INVALID
    assert g(M=0) == INVALID
    assert g(ldy=32) == INVALID
    assert g(K=96) == SHAPE
    assert g(ldy=68, N=66) == SHAPE
    assert g(y=P + 2) == MISALIGNED
    L = fl.lib()
    assert L.mxfp4_gemm(P, P, P, P, P, 16, 64, 96, 64, None, 0, None) == SHAPE


def test_kv_argument_checks():
    L = fl.lib()
    assert L.kv_nvfp4_store(P, P, P, P, P, 2, 2, 1, 8, 24, None) == SHAPE
    assert L.kv_nvfp4_store(P, P, P, P, P, 0, 2, 1, 8, 128, None) == INVALID
    assert L.kv_nvfp4_store(P, P + 2, P, P, P, 2, 2, 1, 8, 128, None) == MISALIGNED
    assert L.kv_nvfp4_load_fp8(P, P, P, 9, P, P, 2, 2, 8, 128, None) == INVALID  # L > Lcap
    assert L.kv_nvfp4_load_fp8(P, P, P, 8, P + 1, P, 2, 2, 8, 128, None) == MISALIGNED
    assert L.fp4lin_convert_selftest(P, P, P, 0, None) == INVALID
    # the wait diagnostic: limit outside [1 us, 100 ms], arrive not 0/1, no result buffer
    assert L.fp4lin_wait_selftest(999, 0, P, None) == INVALID
    assert L.fp4lin_wait_selftest(100000001, 0, P, None) == INVALID
    assert L.fp4lin_wait_selftest(10000, 2, P, None) == INVALID
    assert L.fp4lin_wait_selftest(10000, 0, None, None) == INVALID
    assert L.fp4lin_wait_selftest(10000, 0, P + 4, None) == MISALIGNED


def d(M=16, K=128, ldx=128, had=0, dyn=0, ga=P, x=P, y=P, N=64, ldy=64, ws=P, wsb=8192):
    return fl.lib().nvfp4_linear_decode(x, M, K, ldx, had, dyn, ga, P, P, P, y, N, ldy, ws, wsb, None)


def test_gptq_argument_checks():
    L = fl.lib()
    ws = L.gptq_workspace_bytes(64, 128)
    assert ws == (64 * 128 + 2 * 256 * 64 + 1024) * 4

    def q(w=P, N=64, K=128, ldw=128, had=0, u=P, ldu=128, dyn=0, g=P, wsp=P, wsb=ws):
        return L.nvfp4_gptq_quantize(w, N, K, ldw, had, u, ldu, dyn, g, P, P, wsp, wsb, None)

    assert q(w=None) == INVALID
    assert q(u=None) == INVALID
    assert q(g=None) == INVALID
    assert q(had=32) == INVALID
    assert q(ldu=64) == INVALID
    assert q(K=96, ldw=96, ldu=96) == SHAPE
    assert q(u=P + 4) == MISALIGNED
    assert q(ldu=130) == SHAPE
    assert q(wsb=ws - 1) == WORKSPACE
    assert q(wsp=None) == INVALID
    assert L.mxfp4_gptq_quantize(P, 64, 128, 128, 16, P, 128, P, P, P, ws, None) == INVALID  # 32 or 0
    assert L.mxfp4_gptq_quantize(P, 64, 96, 96, 32, P, 96, P, P, P, ws, None) == SHAPE


def test_hessian_factor_argument_checks():
    L = fl.lib()
    ws = L.gptq_hessian_workspace_bytes(200, 128)
    assert ws == 8 * (200 * 128 + 2 * 128 * 128 + 128 * 128)
    assert L.gptq_hessian_workspace_bytes(200, 96) == 0  # K not a multiple of 64

    def h(x=P, T=200, K=128, ldx=128, had=16, damp=0.01, u=P, ldu=128, wsp=P, wsb=ws):
        return L.gptq_hessian_factor(x, T, K, ldx, had, damp, u, ldu, wsp, wsb, None)

    assert h(x=None) == INVALID
    assert h(u=None) == INVALID
    assert h(wsp=None) == INVALID
    assert h(T=0) == INVALID
    assert h(ldx=127) == INVALID
    assert h(ldu=64) == INVALID
    assert h(had=8) == INVALID
    assert h(damp=-0.5) == INVALID
    assert h(damp=float("nan")) == INVALID
    assert h(K=96, ldx=96, ldu=96, wsb=10 ** 9) == SHAPE
    assert h(x=P + 4) == MISALIGNED
    assert h(u=P + 2) == MISALIGNED
    assert h(wsb=ws - 1) == WORKSPACE


def test_tiled_weight_checks():
    L = fl.lib()
    assert L.fp4lin_tiled_weight_bytes(200, 320) == 256 * 256  # rows to 128, K to 256 values
    assert L.fp4lin_tiled_weight_bytes(0, 64) == 0
    assert L.fp4lin_tile_weights(None, 16, 64, P, None) == INVALID
    assert L.fp4lin_tile_weights(P, 16, 96, P, None) == SHAPE
    assert L.fp4lin_tile_weights(P, 16, 64, P + 8, None) == MISALIGNED
    assert L.nvfp4_gemm_tiled(P, P, P, P, P, P, P, 17, 64, 128, 64, None, 0, None) == SHAPE  # decode sizes only
    assert L.nvfp4_linear_decode_tiled(P, 17, 128, 128, 0, 0, P, P, P, P, P, 64, 64, P, 8192, None) == SHAPE


def test_linear_decode_argument_checks():
    assert d(x=None) == INVALID
    assert d(ga=None) == INVALID
    assert d(M=0) == INVALID
    assert d(had=32) == INVALID
    assert d(dyn=3) == INVALID
    assert d(ldx=64) == INVALID
    assert d(M=17) == SHAPE  # decode sizes only
    assert d(K=96, ldx=96) == SHAPE
    assert d(ldy=68, N=66) == SHAPE
    assert d(x=P + 8) == MISALIGNED
    assert d(dyn=1, ws=None) == WORKSPACE
    assert d(dyn=1, wsb=1000) == WORKSPACE
    L = fl.lib()
    assert L.nvfp4_linear_decode_workspace_bytes(17, 64, 128) == 0
    assert L.nvfp4_linear_decode_workspace_bytes(16, 4096, 4096) >= 4096


@pytest.mark.parametrize("fn", ["nvfp4_quantize", "mxfp4_quantize", "nvfp4_gemm", "mxfp4_gemm",
                                "kv_nvfp4_store", "kv_nvfp4_load_fp8", "nvfp4_linear_decode", "nvfp4_gemm_quant",
                                "kv_nvfp4_attention"])
def test_binding_names_match_abi(fn):
    assert callable(getattr(fl, fn))
