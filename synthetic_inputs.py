"""Seeded synthetic inputs for the NVFP4 / MXFP4 W4A4 linear layer and the NVFP4 KV cache.

This module draws random numbers and nothing else: it applies each workload's
distribution and outlier pattern and rounds the result to bf16 (round to
nearest even, done by torch's float32 -> bfloat16 cast).  It holds none of the
quantisation arithmetic, so the oracle and the CUDA path can both take their
inputs from here without sharing any of the method.

Every draw comes from a Philox generator keyed by (seed, tensor id, chunk id),
so any row block (or, for the KV cache, any (batch, head) slice) can be
regenerated on its own without materialising the whole tensor.

Workloads (the five synthetic configurations of the linear layer and the cache):

* ``tiny``    seed 0: A bf16 [16,128] ~ N(0,1); W bf16 [64,128] ~ N(0, 0.02^2)
  with round(1% of 64*128) = 82 entries, drawn without replacement, times 20.
* ``decode``  seed 1: A bf16 [M,K] ~ N(0,1), M in {1,4,16}, with round(0.5% of K)
  columns (channels) times 30; W bf16 [N,K] ~ N(0, 0.02^2);
  (N,K) in {(4096,4096), (14336,4096), (4096,14336)}.
* ``prefill`` seed 2: A bf16 [8192,4096] Student-t with 3 degrees of freedom;
  W bf16 [14336,4096] ~ N(0, 0.02^2).  The MXFP4 comparison uses these same tensors.
* ``kvcache`` seed 4: K and V bf16 [64,8,32768,128] ~ N(0,1) times one scale per
  (tensor, kv head), the 16 scales log-uniform on [0.1, 10].
* ``gptq_calibration``: calibration activations for a GPTQ Hessian, float64 [T,K]:
  Z M / sqrt(K/4) + 0.3 E with Z [T,K/4], M [K/4,K], E [T,K] ~ N(0,1) (correlated
  channels), then K/64 channels (drawn without replacement) times 8.
"""
from __future__ import annotations

import os
from concurrent.futures import ThreadPoolExecutor

import numpy as np
import torch

# tensor ids used in the generator keys
_T_A, _T_W, _T_K, _T_V, _T_HEADSCALE, _T_OUTLIER, _T_CALIB = 1, 2, 3, 4, 5, 6, 7

ROW_CHUNK = 256  # rows per independently keyed chunk

TINY = dict(M=16, N=64, K=128, seed=0)
DECODE_M = (1, 4, 16)
DECODE_NK = ((4096, 4096), (14336, 4096), (4096, 14336))
PREFILL = dict(M=8192, N=14336, K=4096, seed=2)
KVCACHE = dict(B=64, H=8, L=32768, D=128, seed=4)


def _rng(*key: int) -> np.random.Generator:
    return np.random.Generator(np.random.Philox(np.random.SeedSequence([int(k) for k in key])))


def _threads() -> int:
    return max(1, min(32, os.cpu_count() or 1))


def to_bf16(x: np.ndarray) -> torch.Tensor:
    """float32 ndarray -> contiguous CPU bf16 tensor (round to nearest even)."""
    return torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).to(torch.bfloat16)


def bf16_bits(t: torch.Tensor) -> np.ndarray:
    """CPU bf16 tensor -> its raw bit patterns as a uint16 ndarray (no copy when contiguous)."""
    return t.contiguous().view(torch.int16).numpy().view(np.uint16)


def _rows(seed: int, tid: int, extra: tuple, r0: int, r1: int, cols: int, draw) -> np.ndarray:
    """Rows [r0, r1) of a chunk-keyed float32 matrix; ``draw(rng, n_rows, cols)`` makes one chunk."""
    c0, c1 = r0 // ROW_CHUNK, (r1 + ROW_CHUNK - 1) // ROW_CHUNK
    out = np.empty((r1 - r0, cols), dtype=np.float32)

    def one(c: int) -> None:
        rows_c = ROW_CHUNK
        blk = draw(_rng(seed, tid, *extra, c), rows_c, cols)
        lo, hi = max(r0, c * ROW_CHUNK), min(r1, (c + 1) * ROW_CHUNK)
        out[lo - r0:hi - r0] = blk[lo - c * ROW_CHUNK:hi - c * ROW_CHUNK]

    if c1 - c0 > 4:
        with ThreadPoolExecutor(_threads()) as ex:
            list(ex.map(one, range(c0, c1)))
    else:
        for c in range(c0, c1):
            one(c)
    return out


def _normal(std: float):
    def draw(g, n, k):
        x = g.standard_normal((n, k), dtype=np.float32)
        return x * np.float32(std) if std != 1.0 else x
    return draw


def _student_t3(g, n, k):
    return g.standard_t(3.0, size=(n, k)).astype(np.float32)


# ---------------------------------------------------------------- tiny layer
def tiny() -> dict:
    """The tiny NVFP4 layer: A [16,128] ~ N(0,1), W [64,128] ~ N(0,0.02^2) with 82 outliers x20."""
    s, M, N, K = TINY["seed"], TINY["M"], TINY["N"], TINY["K"]
    a = _rows(s, _T_A, (), 0, M, K, _normal(1.0))
    w = _rows(s, _T_W, (), 0, N, K, _normal(0.02))
    n_out = int(round(0.01 * N * K))
    idx = _rng(s, _T_OUTLIER).choice(N * K, size=n_out, replace=False)
    w.reshape(-1)[idx] *= np.float32(20.0)
    return dict(A=to_bf16(a), W=to_bf16(w), M=M, N=N, K=K)


# ---------------------------------------------------------------- decode GEMMs
def decode_outlier_channels(K: int) -> np.ndarray:
    n = int(round(0.005 * K))
    return np.sort(_rng(1, _T_OUTLIER, K).choice(K, size=n, replace=False))


def decode_A(M: int, K: int) -> torch.Tensor:
    """Decode activations [M,K] ~ N(0,1), 0.5% of the K channels times 30 (rows nest across M)."""
    a = _rows(1, _T_A, (K,), 0, M, K, _normal(1.0))
    a[:, decode_outlier_channels(K)] *= np.float32(30.0)
    return to_bf16(a)


def decode_W(N: int, K: int, r0: int = 0, r1: int | None = None) -> torch.Tensor:
    r1 = N if r1 is None else r1
    return to_bf16(_rows(1, _T_W, (N, K), r0, r1, K, _normal(0.02)))


# ---------------------------------------------------------------- prefill layer
def prefill_A(r0: int = 0, r1: int | None = None) -> torch.Tensor:
    """Prefill activations rows [r0,r1) of [8192,4096], Student-t (nu = 3)."""
    r1 = PREFILL["M"] if r1 is None else r1
    return to_bf16(_rows(PREFILL["seed"], _T_A, (), r0, r1, PREFILL["K"], _student_t3))


def prefill_W(r0: int = 0, r1: int | None = None) -> torch.Tensor:
    """Prefill weights rows [r0,r1) of [14336,4096] ~ N(0, 0.02^2)."""
    r1 = PREFILL["N"] if r1 is None else r1
    return to_bf16(_rows(PREFILL["seed"], _T_W, (), r0, r1, PREFILL["K"], _normal(0.02)))


# ---------------------------------------------------------------- KV cache
def kv_head_scales() -> np.ndarray:
    """[2, H] float32: one scale per (tensor K/V, kv head), log-uniform on [0.1, 10]."""
    u = _rng(KVCACHE["seed"], _T_HEADSCALE).uniform(-1.0, 1.0, size=(2, KVCACHE["H"]))
    return (10.0 ** u).astype(np.float32)


def kv_slice(which: str, b: int, h: int, t0: int = 0, t1: int | None = None,
             L: int | None = None, D: int | None = None) -> np.ndarray:
    """float32 [t1-t0, D] rows of the K ('k') or V ('v') cache slice (b, h) before the bf16 cast.

    The slice for (b, h) is keyed by (seed, tensor, b, h, row chunk), so any token range can be
    regenerated alone.  ``L`` and ``D`` default to the full cache shape.
    """
    L = KVCACHE["L"] if L is None else L
    D = KVCACHE["D"] if D is None else D
    t1 = L if t1 is None else t1
    tid = _T_K if which == "k" else _T_V
    s = kv_head_scales()[0 if which == "k" else 1, h]
    x = _rows(KVCACHE["seed"], tid, (b, h), t0, t1, D, _normal(1.0))
    return x * s


def kv_slice_bf16(which: str, b: int, h: int, t0: int = 0, t1: int | None = None,
                  L: int | None = None, D: int | None = None) -> torch.Tensor:
    return to_bf16(kv_slice(which, b, h, t0, t1, L, D))


# ---------------------------------------------------------------- generic
def normal_bf16(seed: int, rows: int, cols: int, std: float = 1.0, tag: int = 99) -> torch.Tensor:
    """A generic seeded N(0, std^2) bf16 matrix for edge-case tests."""
    return to_bf16(_rows(seed, tag, (rows, cols), 0, rows, cols, _normal(std)))


def student_t_bf16(seed: int, rows: int, cols: int, tag: int = 98) -> torch.Tensor:
    return to_bf16(_rows(seed, tag, (rows, cols), 0, rows, cols, _student_t3))


# ---------------------------------------------------------------- GPTQ calibration
def gptq_calibration(seed: int, T: int, K: int) -> np.ndarray:
    """Calibration activations [T, K] (float64): a rank-K/4 mix of normal draws plus
    independent noise, with K/64 outlier channels times 8."""
    g = _rng(seed, _T_CALIB, T, K)
    z = g.standard_normal((T, K // 4))
    m = g.standard_normal((K // 4, K)) / np.sqrt(K // 4)
    x = z @ m + 0.3 * g.standard_normal((T, K))
    x[:, g.choice(K, size=max(1, K // 64), replace=False)] *= 8.0
    return x
