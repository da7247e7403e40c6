"""The oracle: a plain, slow CPU reference for the NVFP4 / MXFP4 W4A4 linear layer
and the NVFP4 KV cache (numpy in, numpy out, over the C library built from
``oracle/oracle.c``).

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and
``bench.py``'s CPU-baseline / reference legs import this package.  It shares no
code with the CUDA library and never imports it.

Every function follows the format statements of the source pages (cited in
``oracle.c``'s header by page title and section) and the readings R1-R8 listed
there.  Parity is pinned by ``tests/test_oracle_*.py`` against library
conversions (ml_dtypes, torch), scipy's Hadamard matrix, numpy fp64 matmul,
closed forms and brute force.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
_lock = threading.Lock()
_lib = None

CFLAGS = ["-O2", "-ffp-contract=off", "-fno-fast-math", "-fopenmp", "-std=c11",
          "-shared", "-fPIC", "-Wall", "-Wno-unknown-pragmas"]


def build(force: bool = False) -> str:
    """Compile oracle.c with gcc into oracle/liboracle.so (skipped when up to date)."""
    if (not force and os.path.exists(_LIB)
            and os.path.getmtime(_LIB) >= os.path.getmtime(_SRC)):
        return _LIB
    tmp = _LIB + f".tmp{os.getpid()}"
    subprocess.run(["gcc", *CFLAGS, "-o", tmp, _SRC, "-lm"], check=True)
    os.replace(tmp, _LIB)
    return _LIB


def _p(a: np.ndarray, ctype):
    return a.ctypes.data_as(ctypes.POINTER(ctype))


def lib() -> ctypes.CDLL:
    global _lib
    with _lock:
        if _lib is None:
            build()
            L = ctypes.CDLL(_LIB)
            i64, u8p, u16p = ctypes.c_int64, ctypes.POINTER(ctypes.c_uint8), ctypes.POINTER(ctypes.c_uint16)
            f64p, i8p, i32p = ctypes.POINTER(ctypes.c_double), ctypes.POINTER(ctypes.c_int8), ctypes.POINTER(ctypes.c_int32)
            f32p = ctypes.POINTER(ctypes.c_float)
            sig = {
                "oracle_e2m1_decode": (ctypes.c_double, [ctypes.c_uint8]),
                "oracle_e2m1_encode": (ctypes.c_uint8, [ctypes.c_float]),
                "oracle_e4m3_decode": (ctypes.c_double, [ctypes.c_uint8]),
                "oracle_e4m3_encode": (ctypes.c_uint8, [ctypes.c_float]),
                "oracle_e8m0_decode": (ctypes.c_double, [ctypes.c_uint8]),
                "oracle_bf16_rn": (ctypes.c_uint16, [ctypes.c_double]),
                "oracle_hadamard_matrix": (None, [ctypes.c_int, i8p]),
                "oracle_hadamard_norm": (ctypes.c_float, [ctypes.c_int]),
                "oracle_fwht": (None, [f32p, ctypes.c_int]),
                "oracle_nvfp4_tensor_scale": (ctypes.c_float, [u16p, i64, i64, i64, ctypes.c_int]),
                "oracle_nvfp4_quantize": (None, [u16p, i64, i64, i64, ctypes.c_int, ctypes.c_float, u8p, u8p]),
                "oracle_mxfp4_quantize": (None, [u16p, i64, i64, i64, ctypes.c_int, u8p, u8p]),
                "oracle_nvfp4_quantize_mse": (None, [u16p, i64, i64, i64, ctypes.c_int, ctypes.c_float, u8p, u8p]),
                "oracle_mxfp4_quantize_nearest": (None, [u16p, i64, i64, i64, ctypes.c_int, u8p, u8p]),
                "oracle_tc_scale_bytes": (i64, [i64, i64]),
                "oracle_tc_scale_layout": (None, [u8p, i64, i64, u8p]),
                "oracle_dequant": (None, [u8p, u8p, i64, i64, ctypes.c_int, ctypes.c_int, ctypes.c_double, f64p]),
                "oracle_gemm_abt": (None, [f64p, f64p, i64, i64, i64, f64p, f64p]),
                "oracle_num_threads": (ctypes.c_int, []),
                "oracle_kv_store": (None, [u16p, i32p, ctypes.c_float, u8p, u8p, ctypes.c_int, ctypes.c_int,
                                           ctypes.c_int, i64, ctypes.c_int]),
                "oracle_kv_load_fp8": (None, [u8p, u8p, i64, ctypes.c_int, ctypes.c_int, i64, ctypes.c_int, u8p]),
                "oracle_gptq": (None, [u16p, i64, i64, i64, ctypes.c_int, ctypes.c_int, f32p, ctypes.c_float, u8p,
                                       u8p, f32p]),
                "oracle_gptq_mse": (None, [u16p, i64, i64, i64, ctypes.c_int, f32p, ctypes.c_float, u8p, u8p, f32p]),
                "oracle_kv_attention": (None, [u16p, u8p, u8p, ctypes.c_float, u8p, u8p, ctypes.c_float, i64,
                                               ctypes.c_int, ctypes.c_int, ctypes.c_int, i64, ctypes.c_int, f64p]),
            }
            for name, (res, args) in sig.items():
                fn = getattr(L, name)
                fn.restype, fn.argtypes = res, args
            _lib = L
    return _lib


def _bits(x) -> np.ndarray:
    """bf16 input (torch bf16 tensor or uint16 ndarray) -> C-contiguous uint16 ndarray."""
    if hasattr(x, "view") and hasattr(x, "dtype") and str(x.dtype) == "torch.bfloat16":
        import torch
        x = x.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)
    return np.ascontiguousarray(x, dtype=np.uint16)


# ------------------------------------------------------------ scalar formats
def e2m1_decode(codes) -> np.ndarray:
    L = lib()
    c = np.asarray(codes, dtype=np.uint8)
    return np.vectorize(lambda v: L.oracle_e2m1_decode(int(v)), otypes=[np.float64])(c)


def e2m1_encode(v) -> np.ndarray:
    L = lib()
    a = np.asarray(v, dtype=np.float32)
    return np.vectorize(lambda x: L.oracle_e2m1_encode(float(x)), otypes=[np.uint8])(a)


def e4m3_decode(b) -> np.ndarray:
    L = lib()
    return np.vectorize(lambda v: L.oracle_e4m3_decode(int(v)), otypes=[np.float64])(np.asarray(b, dtype=np.uint8))


def e4m3_encode(v) -> np.ndarray:
    L = lib()
    return np.vectorize(lambda x: L.oracle_e4m3_encode(float(x)), otypes=[np.uint8])(np.asarray(v, dtype=np.float32))


def e8m0_decode(b) -> np.ndarray:
    L = lib()
    return np.vectorize(lambda v: L.oracle_e8m0_decode(int(v)), otypes=[np.float64])(np.asarray(b, dtype=np.uint8))


def bf16_rn(v) -> np.ndarray:
    """float64 values -> bf16 bit patterns (uint16), one rounding to nearest even."""
    L = lib()
    return np.vectorize(lambda x: L.oracle_bf16_rn(float(x)), otypes=[np.uint16])(np.asarray(v, dtype=np.float64))


def bf16_bits_to_f64(bits) -> np.ndarray:
    b = np.asarray(bits, dtype=np.uint16).astype(np.uint32) << 16
    return b.view(np.float32).astype(np.float64)


# ------------------------------------------------------------ rotation
def hadamard_matrix(b: int) -> np.ndarray:
    H = np.zeros((b, b), dtype=np.int8)
    lib().oracle_hadamard_matrix(b, _p(H, ctypes.c_int8))
    return H


def hadamard_norm(b: int) -> np.float32:
    return np.float32(lib().oracle_hadamard_norm(b))


def fwht(x, b: int) -> np.ndarray:
    """Blockwise rotation of the last axis (a multiple of b) in blocks of b."""
    a = np.array(x, dtype=np.float32, copy=True)
    flat = np.ascontiguousarray(a.reshape(-1, b))
    L = lib()
    for i in range(flat.shape[0]):
        row = flat[i]
        L.oracle_fwht(_p(row, ctypes.c_float), b)
    return flat.reshape(a.shape)


# ------------------------------------------------------------ quantisers
def nvfp4_tensor_scale(x, hadamard: int = 0) -> np.float32:
    xb = _bits(x)
    rows, cols = xb.shape
    return np.float32(lib().oracle_nvfp4_tensor_scale(_p(xb, ctypes.c_uint16), rows, cols, cols, hadamard))


def nvfp4_quantize(x, hadamard: int = 0, g=None):
    """-> (codes uint8 [rows, cols/2], sf uint8 [rows, cols/16] row-major, g float32)."""
    xb = _bits(x)
    rows, cols = xb.shape
    if g is None:
        g = nvfp4_tensor_scale(xb, hadamard)
    codes = np.zeros((rows, cols // 2), dtype=np.uint8)
    sf = np.zeros((rows, cols // 16), dtype=np.uint8)
    lib().oracle_nvfp4_quantize(_p(xb, ctypes.c_uint16), rows, cols, cols, hadamard, float(g),
                                _p(codes, ctypes.c_uint8), _p(sf, ctypes.c_uint8))
    return codes, sf, np.float32(g)


def nvfp4_quantize_mse(x, hadamard: int = 0, g=None):
    """NVFP4 with the MSE-optimal block scale (reading R9): brute force over all 127
    non-negative finite E4M3 scales per block.  Same outputs as nvfp4_quantize."""
    xb = _bits(x)
    rows, cols = xb.shape
    if g is None:
        g = nvfp4_tensor_scale(xb, hadamard)
    codes = np.zeros((rows, cols // 2), dtype=np.uint8)
    sf = np.zeros((rows, cols // 16), dtype=np.uint8)
    lib().oracle_nvfp4_quantize_mse(_p(xb, ctypes.c_uint16), rows, cols, cols, hadamard, float(g),
                                    _p(codes, ctypes.c_uint8), _p(sf, ctypes.c_uint8))
    return codes, sf, np.float32(g)


def mxfp4_quantize(x, hadamard: int = 0, nearest: bool = False):
    """-> (codes uint8 [rows, cols/2], sf uint8 [rows, cols/32] row-major E8M0).
    nearest: the nearest-power-of-two scale (reading R10) instead of the OCP rule (R4)."""
    xb = _bits(x)
    rows, cols = xb.shape
    codes = np.zeros((rows, cols // 2), dtype=np.uint8)
    sf = np.zeros((rows, cols // 32), dtype=np.uint8)
    fn = lib().oracle_mxfp4_quantize_nearest if nearest else lib().oracle_mxfp4_quantize
    fn(_p(xb, ctypes.c_uint16), rows, cols, cols, hadamard, _p(codes, ctypes.c_uint8), _p(sf, ctypes.c_uint8))
    return codes, sf


def gptq(w, u: np.ndarray, fmt: str = "nvfp4", hadamard: int = 0, g=None, want_err: bool = False,
         mse: bool = False):
    """MR-GPTQ (reading R12) of bf16 weights w [N, K] with the inverse-Hessian factor u
    (fp32 [K, K], upper triangle read).  -> (codes [N, K/2], sf [N, K/G] row-major, g
    (NVFP4; None for MXFP4)[, err fp32 [N, K]]).  NVFP4's g defaults to the rotated w's
    tensor scale, as nvfp4_quantize computes it.  mse (NVFP4): block scales by R9."""
    wb = _bits(w)
    N, K = wb.shape
    uu = np.ascontiguousarray(u, dtype=np.float32)
    assert uu.shape == (K, K)
    group = 16 if fmt == "nvfp4" else 32
    if fmt == "nvfp4" and g is None:
        g = nvfp4_tensor_scale(wb, hadamard)
    codes = np.zeros((N, K // 2), dtype=np.uint8)
    sf = np.zeros((N, K // group), dtype=np.uint8)
    err = np.zeros((N, K), dtype=np.float32) if want_err else None
    if mse:
        assert fmt == "nvfp4"
        lib().oracle_gptq_mse(_p(wb, ctypes.c_uint16), N, K, K, hadamard, _p(uu, ctypes.c_float), float(g),
                              _p(codes, ctypes.c_uint8), _p(sf, ctypes.c_uint8),
                              _p(err, ctypes.c_float) if want_err else None)
    else:
        lib().oracle_gptq(_p(wb, ctypes.c_uint16), N, K, K, group, hadamard, _p(uu, ctypes.c_float),
                          float(g) if fmt == "nvfp4" else 1.0, _p(codes, ctypes.c_uint8), _p(sf, ctypes.c_uint8),
                          _p(err, ctypes.c_float) if want_err else None)
    out = (codes, sf, np.float32(g) if fmt == "nvfp4" else None)
    return out + (err,) if want_err else out


def gptq_hessian_factor(x: np.ndarray, hadamard: int = 0, damp: float = 0.01) -> np.ndarray:
    """The input GPTQ needs (reading R12), in binary64: the calibration activations x [T, K]
    rotated blockwise by H_b / sqrt(b) (b = hadamard, 0 = none), H = x'^T x' + damp *
    mean(diag) * I, and U upper triangular with H^-1 = U^T U; returned as float32."""
    x = np.asarray(x, dtype=np.float64)
    T, K = x.shape
    if hadamard:
        R = hadamard_matrix(hadamard).astype(np.float64) / np.sqrt(hadamard)
        x = (x.reshape(T, K // hadamard, hadamard) @ R.T).reshape(T, K)
    H = x.T @ x
    H[np.diag_indices(K)] += damp * np.mean(np.diag(H))
    Hinv = np.linalg.inv(H)
    L = np.linalg.cholesky((Hinv + Hinv.T) / 2)
    return np.ascontiguousarray(L.T, dtype=np.float32)


def tc_scale_bytes(rows: int, sf_cols: int) -> int:
    return int(lib().oracle_tc_scale_bytes(rows, sf_cols))


def tc_scale_layout(sf_lin: np.ndarray) -> np.ndarray:
    """Row-major [rows, sf_cols] scale bytes -> flat tensor-core layout (padding 0)."""
    s = np.ascontiguousarray(sf_lin, dtype=np.uint8)
    rows, sfc = s.shape
    out = np.zeros(tc_scale_bytes(rows, sfc), dtype=np.uint8)
    lib().oracle_tc_scale_layout(_p(s, ctypes.c_uint8), rows, sfc, _p(out, ctypes.c_uint8))
    return out


# ------------------------------------------------------------ GEMM reference
def dequant(codes: np.ndarray, sf_lin: np.ndarray, fmt: str, g: float = 1.0) -> np.ndarray:
    """Exact fp64 values of a packed operand; fmt 'nvfp4' (16, E4M3, times g) or 'mxfp4' (32, E8M0)."""
    c = np.ascontiguousarray(codes, dtype=np.uint8)
    s = np.ascontiguousarray(sf_lin, dtype=np.uint8)
    rows, cols = c.shape[0], c.shape[1] * 2
    out = np.empty((rows, cols), dtype=np.float64)
    block, kind = (16, 0) if fmt == "nvfp4" else (32, 1)
    lib().oracle_dequant(_p(c, ctypes.c_uint8), _p(s, ctypes.c_uint8), rows, cols, block, kind,
                         float(g) if fmt == "nvfp4" else 1.0, _p(out, ctypes.c_double))
    return out


def gemm_abt(A: np.ndarray, W: np.ndarray):
    """-> (y = A W^T, s = sum_k |a_k w_k|), both fp64 [M, N]."""
    A = np.ascontiguousarray(A, dtype=np.float64)
    W = np.ascontiguousarray(W, dtype=np.float64)
    M, K = A.shape
    N = W.shape[0]
    y = np.empty((M, N), dtype=np.float64)
    s = np.empty((M, N), dtype=np.float64)
    lib().oracle_gemm_abt(_p(A, ctypes.c_double), _p(W, ctypes.c_double), M, N, K,
                          _p(y, ctypes.c_double), _p(s, ctypes.c_double))
    return y, s


def num_threads() -> int:
    return int(lib().oracle_num_threads())


# ------------------------------------------------------------ KV cache
def kv_store(kv_new, pos: np.ndarray, g: float, cache_codes: np.ndarray, cache_sf: np.ndarray) -> None:
    """In place: quantise kv_new bf16 [B,H,T,D] into the cache at positions pos[b] + t."""
    xb = _bits(kv_new)
    B, H, T, D = xb.shape
    Lcap = cache_codes.shape[2]
    p = np.ascontiguousarray(pos, dtype=np.int32)
    assert cache_codes.flags.c_contiguous and cache_sf.flags.c_contiguous
    lib().oracle_kv_store(_p(xb, ctypes.c_uint16), _p(p, ctypes.c_int32), float(g),
                          _p(cache_codes, ctypes.c_uint8), _p(cache_sf, ctypes.c_uint8), B, H, T, Lcap, D)


def kv_load_fp8(cache_codes: np.ndarray, cache_sf: np.ndarray, L: int) -> np.ndarray:
    """-> FP8 E4M3 bytes [B,H,L,D] of the first L positions."""
    c = np.ascontiguousarray(cache_codes, dtype=np.uint8)
    s = np.ascontiguousarray(cache_sf, dtype=np.uint8)
    B, H, Lcap, D2 = c.shape
    D = D2 * 2
    out = np.empty((B, H, L, D), dtype=np.uint8)
    lib().oracle_kv_load_fp8(_p(c, ctypes.c_uint8), _p(s, ctypes.c_uint8), L, B, H, Lcap, D,
                             _p(out, ctypes.c_uint8))
    return out


def kv_attention(q, k_codes, k_sf, gk: float, v_codes, v_sf, gv: float, L: int) -> np.ndarray:
    """Decode attention (reading R11) over the first L cached positions.  q: bf16 [B, H*G, D];
    caches as kv_store.  -> float64 [B, H*G, D]."""
    qb = _bits(q)
    B, HG, D = qb.shape
    kc, ks = np.ascontiguousarray(k_codes, dtype=np.uint8), np.ascontiguousarray(k_sf, dtype=np.uint8)
    vc, vs = np.ascontiguousarray(v_codes, dtype=np.uint8), np.ascontiguousarray(v_sf, dtype=np.uint8)
    H, Lcap = kc.shape[1], kc.shape[2]
    G = HG // H
    out = np.empty((B, HG, D), dtype=np.float64)
    lib().oracle_kv_attention(_p(qb, ctypes.c_uint16), _p(kc, ctypes.c_uint8), _p(ks, ctypes.c_uint8), float(gk),
                              _p(vc, ctypes.c_uint8), _p(vs, ctypes.c_uint8), float(gv), L, B, H, G, Lcap, D,
                              _p(out, ctypes.c_double))
    return out
