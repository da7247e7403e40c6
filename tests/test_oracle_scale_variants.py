"""Pins of the oracle's scale-choice variants (page "FP4 auf Blackwell", section "Was NVFP4
von frueheren 4-Bit-Formaten unterscheidet"): the NVFP4 block scale that minimises the
squared error over the block (reading R9), and the MXFP4 scale rounded to the nearest power
of two (reading R10).  Each check recomputes the result another way: a float64 brute force
written here with ml_dtypes, exact rationals, or blocks whose optimum is known."""
from fractions import Fraction

import ml_dtypes
import numpy as np
import pytest
import torch

import synthetic_inputs as si

E4M3_VALUES = np.arange(127, dtype=np.uint8).view(ml_dtypes.float8_e4m3fn).astype(np.float64)  # codes 0..126


def _e2m1_rne(v):
    """E2M1 round to nearest even with saturation at 6, float64 in -> float64 value out."""
    return np.clip(v, -6.0, 6.0).astype(ml_dtypes.float4_e2m1fn).astype(np.float64)


def _bf16_to_f64(x):
    return x.float().numpy().astype(np.float64)


def _errors64(block, g):
    """Squared error of the block under every candidate scale code 0..126, in float64."""
    d = E4M3_VALUES * float(g)
    out = np.empty(127)
    for c in range(127):
        q = _e2m1_rne(block / d[c]) if d[c] > 0 else np.zeros_like(block)
        out[c] = np.sum((block - q * d[c]) ** 2)
    return out


@pytest.mark.parametrize("seed,dist", [(3, "normal"), (4, "student"), (5, "wide")])
def test_mse_scale_is_the_float64_minimum(orc, seed, dist):
    rows, cols = 24, 256
    if dist == "normal":
        x = si.normal_bf16(seed, rows, cols)
    elif dist == "student":
        x = si.student_t_bf16(seed, rows, cols)
    else:
        x = si.normal_bf16(seed, rows, cols) * torch.logspace(-3, 3, rows).to(torch.bfloat16)[:, None]
    codes, sf, g = orc.nvfp4_quantize_mse(x)
    dcodes, dsf, dg = orc.nvfp4_quantize(x)
    assert dg == g
    xv = _bf16_to_f64(x)
    got = orc.dequant(codes, sf, "nvfp4", g)
    dflt = orc.dequant(dcodes, dsf, "nvfp4", g)
    for r in range(rows):
        for k in range(cols // 16):
            blk = xv[r, 16 * k:16 * k + 16]
            e = _errors64(blk, g)
            chosen = np.sum((blk - got[r, 16 * k:16 * k + 16]) ** 2)
            # the oracle decides in binary32: its pick is the float64 minimum up to rounding
            assert chosen <= e.min() * (1 + 1e-4) + 1e-30, (r, k, chosen, e.min(), int(sf[r, k]), int(np.argmin(e)))
            assert abs(chosen - e[sf[r, k]]) <= 1e-6 * max(chosen, 1e-30), "codes are not E2M1 of x under that scale"
            # never worse than the amax/6 rule
            assert chosen <= np.sum((blk - dflt[r, 16 * k:16 * k + 16]) ** 2) * (1 + 1e-6) + 1e-30


def test_mse_scale_finds_exact_blocks(orc):
    # blocks that are exactly e2m1 values times an E4M3 scale (g = 1): zero error, exact round trip
    rng = np.random.default_rng(11)
    rows, cols = 8, 128
    mags = np.array([0, 0.5, 1, 1.5, 2, 3, 4, 6])
    x = np.zeros((rows, cols))
    for r in range(rows):
        for k in range(cols // 16):
            s = E4M3_VALUES[rng.integers(40, 80)]
            v = mags[rng.integers(0, 8, 16)] * np.where(rng.random(16) < 0.5, -1.0, 1.0)
            v[rng.integers(0, 16)] = 6.0  # the block maximum sits on the largest code
            x[r, 16 * k:16 * k + 16] = v * s
    xb = torch.from_numpy(x).to(torch.bfloat16)
    assert np.array_equal(_bf16_to_f64(xb), x)  # the construction is bf16-exact
    codes, sf, g = orc.nvfp4_quantize_mse(xb, 0, 1.0)
    assert np.array_equal(orc.dequant(codes, sf, "nvfp4", np.float32(1.0)), x)


def test_mse_scale_tie_takes_the_smallest_code(orc):
    # [6, 0, ..., 0] with g = 1 is exact under the scales 1, 1.5, 2, 3, 4, 6, 12 (and more):
    # the tie goes to the smallest code, E4M3 1.0 = 0x38, with the element on code 6 (0x7)
    x = torch.zeros(1, 64, dtype=torch.bfloat16)
    x[0, 0] = 6.0
    codes, sf, _ = orc.nvfp4_quantize_mse(x, 0, 1.0)
    assert sf[0, 0] == 0x38 and codes[0, 0] == 0x07 and not codes[0, 1:8].any()
    assert (sf[0, 1:] == 0).all()  # all-zero blocks: every scale gives error 0, the smallest code is 0


def test_mse_scale_zero_tensor(orc):
    codes, sf, g = orc.nvfp4_quantize_mse(torch.zeros(3, 64, dtype=torch.bfloat16))
    assert g == 1.0 and not codes.any() and not sf.any()


# ------------------------------------------------------------------ MXFP4, nearest power of two
def _floor_log2(q: Fraction) -> int:
    k = q.numerator.bit_length() - q.denominator.bit_length()
    while Fraction(2) ** k > q:
        k -= 1
    while Fraction(2) ** (k + 1) <= q:
        k += 1
    return k


def _nearest_byte(amax: Fraction) -> int:
    if amax == 0:
        return 0
    u = amax / 6
    k = _floor_log2(u)
    lo, hi = Fraction(2) ** k, Fraction(2) ** (k + 1)
    X = k + 1 if hi - u <= u - lo else k  # nearer by value, ties upward
    return min(max(X + 127, 0), 254)


@pytest.mark.parametrize("amax,byte", [(6.0, 127), (6.5, 127), (8.875, 127), (9.0, 128), (4.375, 126),
                                       (4.5, 127), (12.0, 128), (0.75, 124)])
def test_nearest_power_of_two_closed_form(orc, amax, byte):
    # amax/6 = 1 -> 2^0; 8.875/6 = 1.479 -> 2^0 (amax clips to 6); 9/6 = 1.5 -> tie upward, 2^1;
    # 4.375/6 = 0.729 -> 2^-1; 0.75/6 = 0.125 -> 2^-3
    x = torch.zeros(1, 64, dtype=torch.bfloat16)
    x[0, 3] = amax
    x[0, 40] = -amax
    assert float(x[0, 3]) == amax
    _, sf = orc.mxfp4_quantize(x, 0, nearest=True)
    assert sf[0, 0] == byte and sf[0, 1] == byte
    assert sf[0, 0] == _nearest_byte(Fraction(amax))


def test_nearest_power_of_two_matches_exact_rationals(orc):
    rows, cols = 40, 256
    x = si.student_t_bf16(21, rows, cols) * torch.logspace(-30, 30, rows).to(torch.bfloat16)[:, None]
    x[3, :32] = 0
    codes, sf = orc.mxfp4_quantize(x, 0, nearest=True)
    _, sf_ocp = orc.mxfp4_quantize(x, 0)
    xv = _bf16_to_f64(x)
    for r in range(rows):
        for k in range(cols // 32):
            blk = xv[r, 32 * k:32 * k + 32]
            amax = Fraction(float(np.max(np.abs(blk))))
            b = _nearest_byte(amax)
            assert sf[r, k] == b, (r, k, float(amax), int(sf[r, k]), b)
            assert b in (int(sf_ocp[r, k]), int(sf_ocp[r, k]) - 1) or sf_ocp[r, k] == 0
            want = _e2m1_rne(blk * 2.0 ** (127 - b))
            got = orc.dequant(codes[r:r + 1, 16 * k:16 * k + 16], sf[r:r + 1, k:k + 1], "mxfp4")[0] * 2.0 ** (127 - b)
            assert np.array_equal(got, want), (r, k)


def test_nearest_scale_loses_to_ocp_only_by_clipping(orc):
    # the nearest rule picks the lower power of two exactly when amax in [2^e, 1.125 * 2^e):
    # then amax / 2^X lies in [8, 9) and saturates to 6
    x = si.normal_bf16(22, 64, 1024)
    _, sf_n = orc.mxfp4_quantize(x, 0, nearest=True)
    _, sf_o = orc.mxfp4_quantize(x, 0)
    xv = np.abs(_bf16_to_f64(x)).reshape(64, 32, 32).max(axis=2)
    e = np.floor(np.log2(xv))
    lower = xv < 1.125 * 2.0 ** e
    assert np.array_equal(sf_n.astype(int), sf_o.astype(int) - lower.astype(int))
