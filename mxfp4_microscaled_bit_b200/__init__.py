"""Python binding of libfp4lin.so, the B200 (sm_100a) NVFP4 / MXFP4 W4A4 linear
layer and NVFP4 KV cache.

Argument marshalling only: every step runs in the library's CUDA kernels.
PyTorch supplies device memory and the current stream.  There is no CPU or
PyTorch fallback -- if the library cannot be built or loaded, the first call
raises.

Entry points (same names as the C ABI in include/fp4lin.h):
  nvfp4_quantize, nvfp4_gemm, mxfp4_quantize, mxfp4_gemm,
  kv_nvfp4_store, kv_nvfp4_load_fp8, kv_nvfp4_attention, nvfp4_gemm_quant,
  nvfp4_linear_decode, nvfp4_gemm_tiled, gptq_quantize
plus helpers: scale_bytes, gemm_workspace_bytes, tile_weights, device_status,
convert_selftest, wait_selftest, prepare_weight, prepare_weight_gptq,
gptq_hessian_factor, nvfp4_linear, mxfp4_linear.

Errors: a caller-supplied tensor of the wrong dtype raises TypeError; one in host
memory, on another device, in a layout the call cannot take, or smaller than the
call reads or writes raises ValueError -- all before anything is launched.  A
status other than OK from the library raises Fp4LinError.  Timeouts and
out-of-range KV positions found on the device are reported by device_status().
"""
from __future__ import annotations

import ctypes
import os
import threading
from dataclasses import dataclass

import torch

from . import build as _build

__all__ = [
    "Fp4LinError", "lib", "nvfp4_quantize", "nvfp4_gemm", "mxfp4_quantize", "mxfp4_gemm",
    "kv_nvfp4_store", "kv_nvfp4_load_fp8", "scale_bytes", "gemm_workspace_bytes",
    "device_status", "convert_selftest", "wait_selftest", "QuantizedWeight", "prepare_weight", "nvfp4_linear",
    "mxfp4_linear", "nvfp4_linear_decode", "tile_weights", "nvfp4_gemm_tiled", "gptq_quantize", "gptq_hessian_factor", "prepare_weight_gptq",
    "EXPORTS",
]

STATUS = {0: "OK", 1: "INVALID_ARGUMENT", 2: "UNSUPPORTED_SHAPE", 3: "MISALIGNED", 4: "CUDA",
          5: "TIMEOUT", 6: "DEVICE", 7: "WORKSPACE", 8: "OUT_OF_RANGE", 9: "NUMERIC"}

_i64, _sz, _vp, _int = ctypes.c_int64, ctypes.c_size_t, ctypes.c_void_p, ctypes.c_int
EXPORTS = {
    "fp4lin_version": (_int, []),
    "fp4lin_scale_bytes": (_i64, [_i64, _i64]),
    "nvfp4_quantize_workspace_bytes": (_sz, [_i64, _i64]),
    "fp4lin_gemm_workspace_bytes": (_sz, [_i64, _i64, _i64]),
    "nvfp4_quantize": (_int, [_vp, _i64, _i64, _i64, _int, _int, _vp, _vp, _vp, _vp, _sz, _vp]),
    "nvfp4_gemm": (_int, [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _i64, _i64, _i64, _i64, _vp, _sz, _vp]),
    "mxfp4_quantize": (_int, [_vp, _i64, _i64, _i64, _int, _vp, _vp, _vp]),
    "mxfp4_gemm": (_int, [_vp, _vp, _vp, _vp, _vp, _i64, _i64, _i64, _i64, _vp, _sz, _vp]),
    "kv_nvfp4_store": (_int, [_vp, _vp, _vp, _vp, _vp, _int, _int, _int, _i64, _int, _vp]),
    "kv_nvfp4_load_fp8": (_int, [_vp, _vp, _vp, _i64, _vp, _vp, _int, _int, _i64, _int, _vp]),
    "fp4lin_device_status": (_int, [_vp]),
    "fp4lin_convert_selftest": (_int, [_vp, _vp, _vp, _i64, _vp]),
    "fp4lin_wait_selftest": (_int, [ctypes.c_uint64, _int, _vp, _vp]),
    "nvfp4_quantize_noalloc": (_int, [_vp, _i64, _i64, _i64, _int, _vp, _vp, _vp, _vp]),
    "nvfp4_quantize_mse": (_int, [_vp, _i64, _i64, _i64, _int, _int, _vp, _vp, _vp, _vp, _sz, _vp]),
    "mxfp4_quantize_nearest": (_int, [_vp, _i64, _i64, _i64, _int, _vp, _vp, _vp]),
    "kv_attention_workspace_bytes": (_sz, [_int, _int, _int, _i64, _int]),
    "kv_nvfp4_attention": (_int, [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _i64, _vp, _int, _int, _int, _i64, _int, _vp,
                                  _sz, _vp]),
    "nvfp4_gemm_quant": (_int, [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _i64, _int, _vp, _vp, _vp, _i64, _i64, _i64,
                                _vp, _sz, _vp]),
    "nvfp4_linear_decode_workspace_bytes": (_sz, [_i64, _i64, _i64]),
    "gptq_workspace_bytes": (_sz, [_i64, _i64]),
    "fp4lin_tiled_weight_bytes": (_sz, [_i64, _i64]),
    "fp4lin_tile_weights": (_int, [_vp, _i64, _i64, _vp, _vp]),
    "nvfp4_gemm_tiled": (_int, [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _i64, _i64, _i64, _i64, _vp, _sz, _vp]),
    "nvfp4_linear_decode_tiled": (_int, [_vp, _i64, _i64, _i64, _int, _int, _vp, _vp, _vp, _vp, _vp, _i64, _i64,
                                         _vp, _sz, _vp]),
    "nvfp4_gptq_quantize": (_int, [_vp, _i64, _i64, _i64, _int, _vp, _i64, _int, _vp, _vp, _vp, _vp, _sz, _vp]),
    "nvfp4_gptq_quantize_mse": (_int, [_vp, _i64, _i64, _i64, _int, _vp, _i64, _int, _vp, _vp, _vp, _vp, _sz, _vp]),
    "mxfp4_gptq_quantize": (_int, [_vp, _i64, _i64, _i64, _int, _vp, _i64, _vp, _vp, _vp, _sz, _vp]),
    "nvfp4_linear_decode": (_int, [_vp, _i64, _i64, _i64, _int, _int, _vp, _vp, _vp, _vp, _vp, _i64, _i64, _vp, _sz,
                                   _vp]),
    "gptq_hessian_workspace_bytes": (_sz, [_i64, _i64]),
    "gptq_hessian_factor": (_int, [_vp, _i64, _i64, _i64, _int, ctypes.c_double, _vp, _i64, _vp, _sz, _vp]),
}

_lock = threading.Lock()
_lib = None


class Fp4LinError(RuntimeError):
    def __init__(self, fn: str, status: int):
        super().__init__(f"{fn} failed: FP4LIN_ERR_{STATUS.get(status, status)} ({status})")
        self.status = status


def lib() -> ctypes.CDLL:
    """Load (building first if needed) the CUDA library; raises if that is impossible."""
    global _lib
    with _lock:
        if _lib is None:
            path = _build.build()
            L = ctypes.CDLL(path)
            for name, (res, args) in EXPORTS.items():
                fn = getattr(L, name)
                fn.restype, fn.argtypes = res, args
            _lib = L
    return _lib


def library_path() -> str:
    return _build.LIB


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream))


def _check(name: str, st: int) -> None:
    if st != 0:
        raise Fp4LinError(name, st)


# ------------------------------------------------------------------ argument checks
# The library takes every pointer as memory of the current CUDA device, laid out as its header
# states.  These checks run before a pointer crosses the C ABI, so a host tensor, a wrong dtype
# or a buffer smaller than the call reads or writes raises here instead of reaching a kernel.
_BF16, _U8, _F32, _I32 = torch.bfloat16, torch.uint8, torch.float32, torch.int32


def _arg(fn: str, name: str, t, dtype, nbytes: int = 0, rows: bool = False) -> None:
    """t: a `dtype` tensor (any dtype when None) on the current CUDA device holding at least
    nbytes.  rows: a 2-D view with unit stride along its rows and a row stride of at least the
    row length (the calls that take a leading dimension); otherwise t must be contiguous."""
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{fn}: {name} must be a torch.Tensor, not {type(t).__name__}")
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"{fn}: {name} must be {dtype}, not {t.dtype}")
    if rows:
        if t.dim() != 2 or (t.size(1) > 1 and t.stride(1) != 1) or (t.size(0) > 1 and t.stride(0) < t.size(1)):
            raise ValueError(f"{fn}: {name} must be 2-D with unit stride along its rows")
        span = ((t.size(0) - 1) * t.stride(0) + t.size(1)) * t.element_size() if t.numel() else 0
    else:
        if not t.is_contiguous():
            raise ValueError(f"{fn}: {name} must be contiguous")
        span = t.numel() * t.element_size()
    if t.device.type != "cuda":
        raise ValueError(f"{fn}: {name} must be a CUDA tensor, not on {t.device}")
    cur = torch.cuda.current_device()
    if t.device.index != cur:
        raise ValueError(f"{fn}: {name} is on {t.device}; the library works on the current device cuda:{cur}")
    if span < nbytes:
        raise ValueError(f"{fn}: {name} holds {span} bytes, the call needs {nbytes}")


def _ws_arg(fn: str, workspace) -> int:
    """Bytes of an optional contiguous workspace tensor (0 when None)."""
    if workspace is None:
        return 0
    _arg(fn, "workspace", workspace, None)
    return workspace.numel() * workspace.element_size()


def _rows_span(t: torch.Tensor, nrows: int, ncols: int) -> int:
    """Bytes a call touches in a row-strided 2-D view for nrows rows of ncols elements."""
    return ((nrows - 1) * t.stride(0) + ncols) * t.element_size() if nrows > 0 and ncols > 0 else 0


def scale_bytes(rows: int, sf_cols: int) -> int:
    return int(lib().fp4lin_scale_bytes(rows, sf_cols))


def gemm_workspace_bytes(M: int, N: int, K: int) -> int:
    return int(lib().fp4lin_gemm_workspace_bytes(M, N, K))


def device_status(stream=None) -> int:
    """Synchronise the stream, return and clear the device status word (0 = OK)."""
    return int(lib().fp4lin_device_status(_stream(stream)))


# ------------------------------------------------------------------ quantisers
def nvfp4_quantize(x: torch.Tensor, hadamard: int = 0, g: torch.Tensor | None = None, *,
                   compute_global_scale: bool | None = None, codes: torch.Tensor | None = None,
                   scales: torch.Tensor | None = None, workspace: torch.Tensor | None = None, stream=None,
                   mse: bool = False):
    """NVFP4-quantise bf16 x [rows, cols] (row stride x.stride(0)).

    By default the FP32 tensor scale is computed when g is None (returned as a new 1-element
    device tensor) and used as given otherwise.  compute_global_scale=True with a g tensor
    writes the computed scale into that tensor.  mse=True chooses every block scale by the
    least squared error over all E4M3 scales (nvfp4_quantize_mse) instead of amax/6.
    Returns (codes uint8 [rows, cols/2], scales uint8 [scale_bytes], g).
    """
    name = "nvfp4_quantize_mse" if mse else "nvfp4_quantize"
    _arg(name, "x", x, _BF16, rows=True)
    rows, cols = x.shape
    dev = x.device
    dynamic = (g is None) if compute_global_scale is None else bool(compute_global_scale)
    if g is None:
        g = torch.empty(1, dtype=torch.float32, device=dev)
    else:
        _arg(name, "g", g, _F32, 4)
    if dynamic:
        if workspace is None:
            workspace = torch.empty(int(lib().nvfp4_quantize_workspace_bytes(rows, cols)) // 4,
                                    dtype=torch.float32, device=dev)
    if codes is None:
        codes = torch.empty(rows, cols // 2, dtype=torch.uint8, device=dev)
    else:
        _arg(name, "codes", codes, _U8, rows * (cols // 2))
    if scales is None:
        scales = torch.empty(scale_bytes(rows, cols // 16), dtype=torch.uint8, device=dev)
    else:
        _arg(name, "scales", scales, _U8, scale_bytes(rows, cols // 16))
    ws_bytes = _ws_arg(name, workspace)
    _check(name, getattr(lib(), name)(
        _ptr(x), rows, cols, x.stride(0), hadamard, 1 if dynamic else 0, _ptr(g), _ptr(codes), _ptr(scales),
        _ptr(workspace), ws_bytes, _stream(stream)))
    return codes, scales, g


def nvfp4_quantize_noalloc(x: torch.Tensor, hadamard: int, g: torch.Tensor, codes: torch.Tensor,
                           scales: torch.Tensor, stream=None) -> None:
    """nvfp4_quantize with the computed tensor scale, without any device allocation: the library's
    own 4 KB array holds the tensor-scale partials (see include/fp4lin.h).  The caller passes every
    output buffer; concurrent calls on one device must not overlap on the GPU."""
    fn = "nvfp4_quantize_noalloc"
    _arg(fn, "x", x, _BF16, rows=True)
    rows, cols = x.shape
    _arg(fn, "g", g, _F32, 4)
    _arg(fn, "codes", codes, _U8, rows * (cols // 2))
    _arg(fn, "scales", scales, _U8, scale_bytes(rows, cols // 16))
    _check("nvfp4_quantize_noalloc", lib().nvfp4_quantize_noalloc(
        _ptr(x), rows, cols, x.stride(0), hadamard, _ptr(g), _ptr(codes), _ptr(scales), _stream(stream)))


def mxfp4_quantize(x: torch.Tensor, hadamard: int = 0, *, codes: torch.Tensor | None = None,
                   scales: torch.Tensor | None = None, stream=None, nearest: bool = False):
    """MXFP4-quantise bf16 x [rows, cols] -> (codes uint8 [rows, cols/2], scales uint8 [scale_bytes]).
    nearest=True rounds each scale to the nearest power of two (mxfp4_quantize_nearest)."""
    name = "mxfp4_quantize_nearest" if nearest else "mxfp4_quantize"
    _arg(name, "x", x, _BF16, rows=True)
    rows, cols = x.shape
    if codes is None:
        codes = torch.empty(rows, cols // 2, dtype=torch.uint8, device=x.device)
    else:
        _arg(name, "codes", codes, _U8, rows * (cols // 2))
    if scales is None:
        scales = torch.empty(scale_bytes(rows, cols // 32), dtype=torch.uint8, device=x.device)
    else:
        _arg(name, "scales", scales, _U8, scale_bytes(rows, cols // 32))
    _check(name, getattr(lib(), name)(_ptr(x), rows, cols, x.stride(0), hadamard, _ptr(codes), _ptr(scales),
                                      _stream(stream)))
    return codes, scales


# ------------------------------------------------------------------ GEMMs
def _operand(fn: str, side: str, codes, scales, nrows: int, K: int, blk: int, g=None, codes_bytes=None) -> None:
    """One GEMM operand: codes [nrows, K/2] (or a flat tile-order buffer of codes_bytes), its
    tensor-core-layout scales and, for NVFP4, its FP32 tensor scale."""
    if codes_bytes is None:
        _arg(fn, f"{side}_codes", codes, _U8, nrows * (K // 2))
    else:
        _arg(fn, f"{side}_codes", codes, _U8, codes_bytes)
    _arg(fn, f"{side}_scales", scales, _U8, scale_bytes(nrows, K // blk))
    if g is not None:
        _arg(fn, f"g_{side}", g, _F32, 4)


def _codes_shape(fn: str, name: str, codes) -> tuple[int, int]:
    """(rows, K) of a 2-D codes tensor [rows, K/2]."""
    if not isinstance(codes, torch.Tensor) or codes.dim() != 2:
        raise ValueError(f"{fn}: {name} must be a 2-D codes tensor [rows, K/2]")
    return codes.shape[0], codes.shape[1] * 2


def _gemm_out(M, N, out, dev):
    return torch.empty(M, N, dtype=torch.bfloat16, device=dev) if out is None else out


def _gemm_ws(M, N, K, workspace, dev):
    if workspace is False:  # explicitly none: the GEMM then runs without splitting K
        return None, 0
    if workspace is None:
        need = gemm_workspace_bytes(M, N, K)
        workspace = torch.empty(max(need, 16), dtype=torch.uint8, device=dev) if need else None
    return workspace, (0 if workspace is None else workspace.numel() * workspace.element_size())


def nvfp4_gemm(a_codes, a_scales, g_a, w_codes, w_scales, g_w, *, out=None, workspace=None, stream=None):
    """y [M, N] bf16 = (A_q W_q^T) * g_a * g_w for NVFP4 operands (codes [rows, K/2])."""
    fn = "nvfp4_gemm"
    M, K = _codes_shape(fn, "a_codes", a_codes)
    N = _codes_shape(fn, "w_codes", w_codes)[0]
    _operand(fn, "a", a_codes, a_scales, M, K, 16, g_a)
    _operand(fn, "w", w_codes, w_scales, N, K, 16, g_w)
    if out is not None:
        _arg(fn, "out", out, _BF16, _rows_span(out, M, N), rows=True)
    y = _gemm_out(M, N, out, a_codes.device)
    if workspace is not None and workspace is not False:
        _ws_arg(fn, workspace)
    ws, wsb = _gemm_ws(M, N, K, workspace, a_codes.device)
    _check("nvfp4_gemm", lib().nvfp4_gemm(_ptr(a_codes), _ptr(a_scales), _ptr(g_a), _ptr(w_codes), _ptr(w_scales),
                                          _ptr(g_w), _ptr(y), M, N, K, y.stride(0), _ptr(ws), wsb, _stream(stream)))
    return y


def kv_nvfp4_attention(q, k_cache, v_cache, L: int, *, out=None, workspace=None, stream=None):
    """Decode attention from the NVFP4 caches.  q: bf16 [B, H*G, D]; k_cache, v_cache: (codes
    [B,H,Lcap,D/2], scales [B,H,Lcap,D/16], g) as kv_nvfp4_store fills them.
    Returns float32 [B, H*G, D]."""
    fn = "kv_nvfp4_attention"
    kc, ks, gk = k_cache
    vc, vs, gv = v_cache
    B, H, Lcap, D2 = kc.shape
    D = 2 * D2
    G = q.shape[1] // H
    dev = q.device
    _arg(fn, "q", q, _BF16, B * H * G * D * 2)
    for side, (c, sc, gg) in (("k", k_cache), ("v", v_cache)):
        if tuple(c.shape) != (B, H, Lcap, D2):
            raise ValueError(f"{fn}: the K and V caches must have the same shape")
        _arg(fn, f"{side}_codes", c, _U8, B * H * Lcap * D2)
        _arg(fn, f"{side}_scales", sc, _U8, B * H * Lcap * (D // 16))
        _arg(fn, f"g_{side}", gg, _F32, 4)
    if out is None:
        out = torch.empty(B, H * G, D, dtype=torch.float32, device=dev)
    else:
        _arg(fn, "out", out, _F32, B * H * G * D * 4)
    if workspace is None:
        need = int(lib().kv_attention_workspace_bytes(B, H, G, L, D))
        workspace = torch.empty(max(need, 16), dtype=torch.uint8, device=dev)
    else:
        _ws_arg(fn, workspace)
    _check("kv_nvfp4_attention", lib().kv_nvfp4_attention(
        _ptr(q), _ptr(kc), _ptr(ks), _ptr(gk), _ptr(vc), _ptr(vs), _ptr(gv), L, _ptr(out), B, H, G, Lcap, D,
        _ptr(workspace), workspace.numel() * workspace.element_size(), _stream(stream)))
    return out


def nvfp4_gemm_quant(a_codes, a_scales, g_a, w_codes, w_scales, g_w, g_y, *, hadamard: int = 0,
                     out=None, write_y: bool = True, y_codes=None, y_scales=None, workspace=None, stream=None):
    """nvfp4_gemm with the output also NVFP4-quantised (static tensor scale g_y, 16-wide rotation
    when hadamard=16) for the next layer.  Returns (y or None, y_codes [M, N/2], y_scales)."""
    fn = "nvfp4_gemm_quant"
    M, K = _codes_shape(fn, "a_codes", a_codes)
    N = _codes_shape(fn, "w_codes", w_codes)[0]
    _operand(fn, "a", a_codes, a_scales, M, K, 16, g_a)
    _operand(fn, "w", w_codes, w_scales, N, K, 16, g_w)
    _arg(fn, "g_y", g_y, _F32, 4)
    dev = a_codes.device
    if write_y and out is not None:
        _arg(fn, "out", out, _BF16, _rows_span(out, M, N), rows=True)
    y = _gemm_out(M, N, out, dev) if write_y else None
    if y_codes is None:
        y_codes = torch.empty(M, N // 2, dtype=torch.uint8, device=dev)
    else:
        _arg(fn, "y_codes", y_codes, _U8, M * (N // 2))
    if y_scales is None:
        y_scales = torch.empty(scale_bytes(M, N // 16), dtype=torch.uint8, device=dev)
    else:
        _arg(fn, "y_scales", y_scales, _U8, scale_bytes(M, N // 16))
    if workspace is not None and workspace is not False:
        _ws_arg(fn, workspace)
    ws, wsb = _gemm_ws(M, N, K, workspace, dev)
    _check("nvfp4_gemm_quant", lib().nvfp4_gemm_quant(
        _ptr(a_codes), _ptr(a_scales), _ptr(g_a), _ptr(w_codes), _ptr(w_scales), _ptr(g_w), _ptr(y),
        y.stride(0) if y is not None else N, hadamard, _ptr(g_y), _ptr(y_codes), _ptr(y_scales), M, N, K, _ptr(ws),
        wsb, _stream(stream)))
    return y, y_codes, y_scales


def tile_weights(codes: torch.Tensor, *, stream=None) -> torch.Tensor:
    """Weight codes [N, K/2] -> the decode GEMM's tile order (flat uint8, see include/fp4lin.h)."""
    N, K = _codes_shape("fp4lin_tile_weights", "codes", codes)
    _arg("fp4lin_tile_weights", "codes", codes, _U8, N * (K // 2))
    tiled = torch.empty(int(lib().fp4lin_tiled_weight_bytes(N, K)), dtype=torch.uint8, device=codes.device)
    _check("fp4lin_tile_weights", lib().fp4lin_tile_weights(_ptr(codes), N, K, _ptr(tiled), _stream(stream)))
    return tiled


def nvfp4_gemm_tiled(a_codes, a_scales, g_a, w_tiled, w_scales, g_w, N: int, *, out=None, workspace=None,
                     stream=None):
    """nvfp4_gemm for M <= 16 with the weights' codes in tile order (tile_weights)."""
    fn = "nvfp4_gemm_tiled"
    M, K = _codes_shape(fn, "a_codes", a_codes)
    _operand(fn, "a", a_codes, a_scales, M, K, 16, g_a)
    _operand(fn, "w", w_tiled, w_scales, N, K, 16, g_w, codes_bytes=int(lib().fp4lin_tiled_weight_bytes(N, K)))
    if out is not None:
        _arg(fn, "out", out, _BF16, _rows_span(out, M, N), rows=True)
    y = _gemm_out(M, N, out, a_codes.device)
    if workspace is not None and workspace is not False:
        _ws_arg(fn, workspace)
    ws, wsb = _gemm_ws(M, N, K, workspace, a_codes.device)
    _check("nvfp4_gemm_tiled", lib().nvfp4_gemm_tiled(
        _ptr(a_codes), _ptr(a_scales), _ptr(g_a), _ptr(w_tiled), _ptr(w_scales), _ptr(g_w), _ptr(y), M, N, K,
        y.stride(0), _ptr(ws), wsb, _stream(stream)))
    return y


def nvfp4_linear_decode(x, w_codes, w_scales, g_w, *, hadamard: int = 0, g_a=None,
                        compute_global_scale: bool | None = None, out=None, workspace=None, stream=None,
                        tiled_n: int | None = None):
    """Decode-sized (M <= 16) y = x W^T with the activation quantiser inside the GEMM: bit-equal to
    nvfp4_quantize(x, hadamard, g_a, compute_global_scale=...) then nvfp4_gemm.  The activations'
    tensor scale is computed (amax / 2688) when g_a is None or compute_global_scale is True (then
    written into g_a), else taken from g_a.  tiled_n: w_codes is the tile-order buffer of a
    weight with tiled_n rows (tile_weights).  Returns (y, g_a)."""
    fn = "nvfp4_linear_decode" if tiled_n is None else "nvfp4_linear_decode_tiled"
    _arg(fn, "x", x, _BF16, rows=True)
    M, K = x.shape
    if tiled_n is None:
        N = _codes_shape(fn, "w_codes", w_codes)[0]
        _operand(fn, "w", w_codes, w_scales, N, K, 16, g_w)
    else:
        N = tiled_n
        _operand(fn, "w", w_codes, w_scales, N, K, 16, g_w, codes_bytes=int(lib().fp4lin_tiled_weight_bytes(N, K)))
    dev = x.device
    if out is not None:
        _arg(fn, "out", out, _BF16, _rows_span(out, M, N), rows=True)
    y = _gemm_out(M, N, out, dev)
    dynamic = (g_a is None) if compute_global_scale is None else bool(compute_global_scale)
    if g_a is None:
        g_a = torch.empty(1, dtype=torch.float32, device=dev)
    else:
        _arg(fn, "g_a", g_a, _F32, 4)
    if workspace is None:
        need = lib().nvfp4_linear_decode_workspace_bytes(M, N, K)
        workspace = torch.empty(max(need, 16), dtype=torch.uint8, device=dev)
    elif workspace is False:
        workspace = None
    wsb = _ws_arg(fn, workspace)
    _check(fn, getattr(lib(), fn)(
        _ptr(x), M, K, x.stride(0), hadamard, int(dynamic), _ptr(g_a), _ptr(w_codes), _ptr(w_scales), _ptr(g_w),
        _ptr(y), N, y.stride(0), _ptr(workspace), wsb, _stream(stream)))
    return y, g_a


def mxfp4_gemm(a_codes, a_scales, w_codes, w_scales, *, out=None, workspace=None, stream=None):
    """y [M, N] bf16 = A_q W_q^T for MXFP4 operands."""
    fn = "mxfp4_gemm"
    M, K = _codes_shape(fn, "a_codes", a_codes)
    N = _codes_shape(fn, "w_codes", w_codes)[0]
    _operand(fn, "a", a_codes, a_scales, M, K, 32)
    _operand(fn, "w", w_codes, w_scales, N, K, 32)
    if out is not None:
        _arg(fn, "out", out, _BF16, _rows_span(out, M, N), rows=True)
    y = _gemm_out(M, N, out, a_codes.device)
    if workspace is not None and workspace is not False:
        _ws_arg(fn, workspace)
    ws, wsb = _gemm_ws(M, N, K, workspace, a_codes.device)
    _check("mxfp4_gemm", lib().mxfp4_gemm(_ptr(a_codes), _ptr(a_scales), _ptr(w_codes), _ptr(w_scales), _ptr(y),
                                          M, N, K, y.stride(0), _ptr(ws), wsb, _stream(stream)))
    return y


# ------------------------------------------------------------------ KV cache
def kv_nvfp4_store(kv_new, pos, g, cache_codes, cache_scales, *, stream=None) -> None:
    """Quantise kv_new bf16 [B, H, T, D] into cache_codes [B, H, Lcap, D/2] / cache_scales [B, H, Lcap, D/16]
    at positions pos[b] + t (pos: int32 device [B]; g: float32 device [1])."""
    fn = "kv_nvfp4_store"
    B, H, T, D = kv_new.shape
    Lcap = cache_codes.shape[2]
    _arg(fn, "kv_new", kv_new, _BF16, B * H * T * D * 2)
    _arg(fn, "pos", pos, _I32, B * 4)
    _arg(fn, "g", g, _F32, 4)
    _arg(fn, "cache_codes", cache_codes, _U8, B * H * Lcap * (D // 2))
    _arg(fn, "cache_scales", cache_scales, _U8, B * H * Lcap * (D // 16))
    _check("kv_nvfp4_store", lib().kv_nvfp4_store(_ptr(kv_new), _ptr(pos), _ptr(g), _ptr(cache_codes),
                                                  _ptr(cache_scales), B, H, T, Lcap, D, _stream(stream)))


def kv_nvfp4_load_fp8(cache_codes, cache_scales, g, L: int, *, out=None, out_scale=None, stream=None):
    """Dequantise positions [0, L) to FP8 E4M3 bytes [B, H, L, D]; returns (out, out_scale = 8 g)."""
    fn = "kv_nvfp4_load_fp8"
    B, H, Lcap, D2 = cache_codes.shape
    D = D2 * 2
    dev = cache_codes.device
    _arg(fn, "cache_codes", cache_codes, _U8, B * H * Lcap * D2)
    _arg(fn, "cache_scales", cache_scales, _U8, B * H * Lcap * (D // 16))
    _arg(fn, "g", g, _F32, 4)
    if out is None:
        out = torch.empty(B, H, L, D, dtype=torch.uint8, device=dev)
    else:
        _arg(fn, "out", out, _U8, B * H * max(L, 0) * D)
    if out_scale is None:
        out_scale = torch.empty(1, dtype=torch.float32, device=dev)
    else:
        _arg(fn, "out_scale", out_scale, _F32, 4)
    _check("kv_nvfp4_load_fp8", lib().kv_nvfp4_load_fp8(_ptr(cache_codes), _ptr(cache_scales), _ptr(g), L,
                                                        _ptr(out), _ptr(out_scale), B, H, Lcap, D, _stream(stream)))
    return out, out_scale


def convert_selftest(x: torch.Tensor, stream=None):
    """The library's E2M1 and E4M3 conversions of float32 device tensor x (diagnostic)."""
    _arg("fp4lin_convert_selftest", "x", x, _F32)
    n = x.numel()
    e2 = torch.empty(n, dtype=torch.uint8, device=x.device)
    e4 = torch.empty(n, dtype=torch.uint8, device=x.device)
    _check("fp4lin_convert_selftest", lib().fp4lin_convert_selftest(_ptr(x), _ptr(e2), _ptr(e4), n, _stream(stream)))
    return e2, e4


def wait_selftest(limit_ns: int, arrive: bool, device=None, stream=None) -> torch.Tensor:
    """Run the device-side bounded wait (diagnostic): two barrier waits in one CTA, the
    second limited to limit_ns.  Without `arrive` nothing completes them, so the second
    expires and records TIMEOUT in the device status, and the first gives up after it.
    Returns the int64 tensor [done0, done1, ns0, ns1] on the device."""
    dev = torch.device(device) if device is not None else torch.device("cuda", torch.cuda.current_device())
    r = torch.full((4,), -1, dtype=torch.int64, device=dev)
    _check("fp4lin_wait_selftest", lib().fp4lin_wait_selftest(int(limit_ns), 1 if arrive else 0, _ptr(r),
                                                               _stream(stream)))
    return r


# ------------------------------------------------------------------ layer helpers
@dataclass
class QuantizedWeight:
    """A pre-quantised weight [N, K]: codes, tensor-core-layout scales and (NVFP4) the FP32 scale."""
    fmt: str
    codes: torch.Tensor
    scales: torch.Tensor
    g: torch.Tensor | None
    hadamard: int
    N: int
    K: int
    tiled: torch.Tensor | None = None  # NVFP4 codes in the decode GEMM's tile order (optional)


def prepare_weight(w: torch.Tensor, fmt: str = "nvfp4", hadamard: int = 0, tiled: bool = False) -> QuantizedWeight:
    """Quantise a bf16 weight [N, K] once, offline; with hadamard the rotation is folded into it,
    so y = (x H)(W H)^T = x W^T needs only the online rotation of the activations.  tiled
    (NVFP4): also keep the codes in tile order, which decode-sized calls then stream."""
    if fmt == "nvfp4":
        c, s, g = nvfp4_quantize(w, hadamard)
        return QuantizedWeight("nvfp4", c, s, g, hadamard, w.shape[0], w.shape[1], tile_weights(c) if tiled else None)
    c, s = mxfp4_quantize(w, hadamard)
    return QuantizedWeight("mxfp4", c, s, None, hadamard, w.shape[0], w.shape[1])


# ------------------------------------------------------------------ MR-GPTQ (offline weights)
def gptq_hessian_factor(x: torch.Tensor, hadamard: int = 0, damp: float = 0.01, *, out=None, workspace=None,
                        stream=None) -> torch.Tensor:
    """GPTQ's input from calibration activations x [T, K] (float64, on the current device): the
    library's gptq_hessian_factor -- x rotated blockwise by H_b / sqrt(b) (b = hadamard), the damped
    Hessian H = x'^T x' + damp * mean(diag) I, and the upper factor U with H^-1 = U^T U, in
    binary64.  Returns U as float32 [K, K] (out, if given).  A Hessian that is not positive
    definite is reported by device_status() as NUMERIC (9)."""
    fn = "gptq_hessian_factor"
    _arg(fn, "x", x, torch.float64, rows=True)
    T, K = x.shape
    dev = x.device
    if out is None:
        out = torch.empty(K, K, dtype=torch.float32, device=dev)
    else:
        _arg(fn, "out", out, _F32, _rows_span(out, K, K), rows=True)
    if workspace is None:
        workspace = torch.empty(max(16, int(lib().gptq_hessian_workspace_bytes(T, K))), dtype=torch.uint8,
                                device=dev)
    wsb = _ws_arg(fn, workspace)
    _check(fn, lib().gptq_hessian_factor(_ptr(x), T, K, x.stride(0), hadamard, float(damp), _ptr(out), out.stride(0),
                                         _ptr(workspace), wsb, _stream(stream)))
    return out


def gptq_quantize(w: torch.Tensor, u: torch.Tensor, fmt: str = "nvfp4", hadamard: int = 0, g=None, *,
                  compute_global_scale: bool | None = None, codes=None, scales=None, workspace=None, stream=None,
                  mse: bool = False):
    """MR-GPTQ of bf16 weights w [N, K] with the inverse-Hessian factor u [K, K] (float32).
    Returns (codes [N, K/2], scales, g) -- g None for MXFP4 -- ready for nvfp4_gemm /
    mxfp4_gemm against activations rotated the same way.  mse (NVFP4): block scales of least
    squared error (nvfp4_gptq_quantize_mse)."""
    if fmt not in ("nvfp4", "mxfp4"):
        raise ValueError(f"gptq_quantize: fmt must be 'nvfp4' or 'mxfp4', not {fmt!r}")
    fn = ("nvfp4_gptq_quantize_mse" if mse else "nvfp4_gptq_quantize") if fmt == "nvfp4" else "mxfp4_gptq_quantize"
    _arg(fn, "w", w, _BF16, rows=True)
    N, K = w.shape
    _arg(fn, "u", u, _F32, _rows_span(u, K, K), rows=True)
    dev = w.device
    G = 16 if fmt == "nvfp4" else 32
    if codes is None:
        codes = torch.empty(N, K // 2, dtype=torch.uint8, device=dev)
    else:
        _arg(fn, "codes", codes, _U8, N * (K // 2))
    if scales is None:
        scales = torch.empty(scale_bytes(N, K // G), dtype=torch.uint8, device=dev)
    else:
        _arg(fn, "scales", scales, _U8, scale_bytes(N, K // G))
    if workspace is None:
        workspace = torch.empty(int(lib().gptq_workspace_bytes(N, K)), dtype=torch.uint8, device=dev)
    wsb = _ws_arg(fn, workspace)
    if fmt == "nvfp4":
        dynamic = (g is None) if compute_global_scale is None else bool(compute_global_scale)
        if g is None:
            g = torch.empty(1, dtype=torch.float32, device=dev)
        else:
            _arg(fn, "g", g, _F32, 4)
        _check(fn, getattr(lib(), fn)(
            _ptr(w), N, K, w.stride(0), hadamard, _ptr(u), u.stride(0), int(dynamic), _ptr(g), _ptr(codes),
            _ptr(scales), _ptr(workspace), wsb, _stream(stream)))
        return codes, scales, g
    _check("mxfp4_gptq_quantize", lib().mxfp4_gptq_quantize(
        _ptr(w), N, K, w.stride(0), hadamard, _ptr(u), u.stride(0), _ptr(codes), _ptr(scales), _ptr(workspace),
        wsb, _stream(stream)))
    return codes, scales, None


def prepare_weight_gptq(w: torch.Tensor, u: torch.Tensor, fmt: str = "nvfp4", hadamard: int = 0) -> "QuantizedWeight":
    """prepare_weight with MR-GPTQ in place of plain rounding (u from gptq_hessian_factor of the
    layer's calibration inputs with the same hadamard)."""
    c, s, g = gptq_quantize(w, u, fmt, hadamard)
    return QuantizedWeight(fmt, c, s, g, hadamard, w.shape[0], w.shape[1])


def nvfp4_linear(x: torch.Tensor, w: QuantizedWeight, *, out=None, stream=None) -> torch.Tensor:
    """y = x W^T: online (rotated) NVFP4 quantisation of x, then the block-scaled GEMM (for M <= 16
    one fused launch that quantises inside the GEMM; the same result)."""
    if x.shape[0] <= 16 and x.shape[1] % 64 == 0:
        if w.tiled is not None:
            return nvfp4_linear_decode(x, w.tiled, w.scales, w.g, hadamard=w.hadamard, out=out, stream=stream,
                                       tiled_n=w.N)[0]
        return nvfp4_linear_decode(x, w.codes, w.scales, w.g, hadamard=w.hadamard, out=out, stream=stream)[0]
    c, s, g = nvfp4_quantize(x, w.hadamard, stream=stream)
    return nvfp4_gemm(c, s, g, w.codes, w.scales, w.g, out=out, stream=stream)


def mxfp4_linear(x: torch.Tensor, w: QuantizedWeight, *, out=None, stream=None) -> torch.Tensor:
    c, s = mxfp4_quantize(x, w.hadamard, stream=stream)
    return mxfp4_gemm(c, s, w.codes, w.scales, out=out, stream=stream)
