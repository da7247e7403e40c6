"""Pins of the oracle's number formats and rotation against things other than itself:
library conversions (ml_dtypes, torch), scipy's Hadamard matrix, hand-worked values,
closed forms and invariants.  CPU only."""
from decimal import Decimal, getcontext

import ml_dtypes
import numpy as np
import pytest
import scipy.linalg
import torch

from conftest import golden


# ------------------------------------------------------------------ E2M1
def test_e2m1_decode_matches_grid_and_library(orc):
    g = golden("e2m1_grid.json")["magnitudes"]
    dec = orc.e2m1_decode(np.arange(16))
    assert list(dec[:8]) == g
    assert list(dec[8:]) == [-v for v in g]
    assert np.signbit(dec[8])  # code 8 is -0
    lib = np.arange(16, dtype=np.uint8).view(ml_dtypes.float4_e2m1fn).astype(np.float64)
    assert np.array_equal(dec, lib) and np.array_equal(np.signbit(dec), np.signbit(lib))


def _e2m1_probe_values():
    grid = np.array([0, 0.5, 1, 1.5, 2, 3, 4, 6], dtype=np.float64)
    mids = (grid[1:] + grid[:-1]) / 2
    v = [grid, mids, np.linspace(-8, 8, 40001), [6.0001, 7, 100, 1e30, 3.4e38, 1e-30, 1e-45, 0.25000003, 0.24999999]]
    v = np.concatenate([np.asarray(a, dtype=np.float64).ravel() for a in v])
    v = np.concatenate([v, -v]).astype(np.float32)
    # every float32 around each tie point, to catch an off-by-one-ulp tie rule
    near = []
    for m in mids:
        up = dn = np.float32(m)
        near.append(up)
        for _ in range(3):
            up = np.nextafter(up, np.float32(np.inf))
            dn = np.nextafter(dn, np.float32(-np.inf))
            near += [up, dn]
    rng = np.random.default_rng(7)
    rand = rng.uniform(-7, 7, 20000).astype(np.float32)
    return np.concatenate([v, np.array(near, dtype=np.float32), -np.array(near, dtype=np.float32), rand])


def test_e2m1_encode_matches_ml_dtypes(orc):
    v = _e2m1_probe_values()
    ours = orc.e2m1_encode(v)
    ref = v.astype(ml_dtypes.float4_e2m1fn).view(np.uint8) & 0xF
    bad = np.nonzero(ours != ref)[0]
    assert bad.size == 0, list(zip(v[bad][:10], ours[bad][:10], ref[bad][:10]))


def test_e2m1_encode_decode_roundtrip(orc):
    codes = np.arange(16, dtype=np.uint8)
    assert np.array_equal(orc.e2m1_encode(orc.e2m1_decode(codes).astype(np.float32)), codes)


# ------------------------------------------------------------------ E4M3
def test_e4m3_decode_matches_torch(orc):
    b = np.arange(256, dtype=np.uint8)
    ours = orc.e4m3_decode(b)
    ref = torch.from_numpy(b).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    nan = np.isnan(ref)
    assert list(np.nonzero(nan)[0]) == [0x7F, 0xFF]
    assert np.array_equal(np.isnan(ours), nan)
    assert np.array_equal(ours[~nan], ref[~nan])
    assert orc.e4m3_decode([0x7E])[0] == 448.0 and orc.e4m3_decode([1])[0] == 2.0 ** -9


def test_e4m3_encode_matches_torch_inside_range(orc):
    finite = orc.e4m3_decode(np.arange(127, dtype=np.uint8))
    mids = (finite[1:] + finite[:-1]) / 2
    rng = np.random.default_rng(11)
    v = np.concatenate([finite, mids, rng.uniform(0, 448, 30000), 2.0 ** rng.uniform(-14, 8.8, 30000),
                        [2.0 ** -10, 2.0 ** -10 * 1.0000001, 2.0 ** -11, 1e-20, 0.0, 460.0, 463.9]])
    v = np.concatenate([v, -v]).astype(np.float32)
    ours = orc.e4m3_encode(v)
    ref = torch.from_numpy(v).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    bad = np.nonzero(ours != ref)[0]
    assert bad.size == 0, list(zip(v[bad][:10], ours[bad][:10], ref[bad][:10]))


def test_e4m3_encode_saturates(orc):
    # satfinite: everything above the largest finite value maps to 448 (torch would give NaN)
    v = np.array([449, 464, 470, 480, 1e6, 3.4e38], dtype=np.float32)
    assert list(orc.e4m3_encode(v)) == [0x7E] * 6
    assert list(orc.e4m3_encode(-v)) == [0xFE] * 6


def test_e8m0_decode_matches_torch(orc):
    b = np.arange(255, dtype=np.uint8)
    ours = orc.e8m0_decode(b)
    ref = torch.from_numpy(b).view(torch.float8_e8m0fnu).to(torch.float64).numpy()
    assert np.array_equal(ours, ref)
    assert np.isnan(orc.e8m0_decode([255])[0])
    assert orc.e8m0_decode([127])[0] == 1.0


# ------------------------------------------------------------------ bf16 rounding
def test_bf16_rn_hand_cases(orc):
    for v, bits in golden("bf16_rounding.json")["cases"]:
        assert int(orc.bf16_rn([v])[0]) == bits, (v, bits)


def test_bf16_rn_matches_torch_on_float_inputs(orc):
    # for inputs that are already binary32 a single rounding is what torch's cast does
    rng = np.random.default_rng(3)
    v = np.concatenate([rng.standard_normal(20000) * 10.0 ** rng.uniform(-30, 30, 20000),
                        rng.standard_normal(2000) * 1e-39]).astype(np.float32)
    ref = torch.from_numpy(v).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(orc.bf16_rn(v.astype(np.float64)), ref)


# ------------------------------------------------------------------ Hadamard rotation
@pytest.mark.parametrize("b", [2, 4, 8, 16, 32])
def test_hadamard_matrix_is_sylvester(orc, b):
    H = orc.hadamard_matrix(b).astype(np.int64)
    assert np.array_equal(H, scipy.linalg.hadamard(b))
    assert np.array_equal(H @ H.T, b * np.eye(b, dtype=np.int64))


def test_hadamard_norm_is_correctly_rounded(orc):
    assert orc.hadamard_norm(16) == np.float32(0.25)
    c = orc.hadamard_norm(32)
    getcontext().prec = 60
    exact = Decimal(1) / Decimal(32).sqrt()
    below, above = np.nextafter(c, np.float32(0)), np.nextafter(c, np.float32(1))
    err = abs(Decimal(float(c)) - exact)
    assert err <= abs(Decimal(float(below)) - exact) and err <= abs(Decimal(float(above)) - exact)


@pytest.mark.parametrize("b", [16, 32])
def test_fwht_matches_matrix_product(orc, b):
    rng = np.random.default_rng(b)
    x = rng.standard_t(3, size=(200, b)).astype(np.float32)
    y = orc.fwht(x, b).astype(np.float64)
    H = scipy.linalg.hadamard(b).astype(np.float64)
    ref = x.astype(np.float64) @ H.T / np.sqrt(b)
    # butterflies in binary32: log2(b) additions plus one multiply, each off by at most half an ulp
    tol = (np.log2(b) + 2) * 2.0 ** -24 * (np.abs(x).astype(np.float64) @ np.abs(H).T / np.sqrt(b))
    assert np.all(np.abs(y - ref) <= tol + 1e-30)
    # Parseval: the rotation preserves the Euclidean norm of each block
    assert np.allclose(np.linalg.norm(y, axis=1), np.linalg.norm(x.astype(np.float64), axis=1), rtol=1e-5)


def test_fwht_exact_on_small_integers(orc):
    # small integer inputs: every butterfly sum is exact, and 1/sqrt(16) = 0.25 is exact
    rng = np.random.default_rng(5)
    x = rng.integers(-100, 100, size=(50, 16)).astype(np.float32)
    ref = (x.astype(np.int64) @ scipy.linalg.hadamard(16).T).astype(np.float64) / 4.0
    assert np.array_equal(orc.fwht(x, 16).astype(np.float64), ref)


def test_rotation_preserves_products(orc):
    # (A H/sqrt b)(W H/sqrt b)^T = A W^T: rotating both operands keeps the layer's result
    rng = np.random.default_rng(9)
    A = rng.standard_normal((8, 64)).astype(np.float32)
    W = rng.standard_normal((12, 64)).astype(np.float32)
    for b in (16, 32):
        Ar, Wr = orc.fwht(A, b).astype(np.float64), orc.fwht(W, b).astype(np.float64)
        assert np.allclose(Ar @ Wr.T, A.astype(np.float64) @ W.astype(np.float64).T, atol=1e-4)


# ------------------------------------------------------------------ storage ratios
def test_storage_ratios():
    # about 4.5 bits per value for NVFP4; 3.5x smaller than FP16 and about 1.8x smaller than FP8
    # (page "FP8, NVFP4 czy AWQ?", section "Czym roznia sie FP8, NVFP4, MXFP4 i AWQ?")
    nv_bytes = 0.5 + 1 / 16
    mx_bytes = 0.5 + 1 / 32
    assert nv_bytes * 8 == 4.5 and mx_bytes * 8 == 4.25
    assert round(2 / nv_bytes, 2) == 3.56 and round(1 / nv_bytes, 2) == 1.78
