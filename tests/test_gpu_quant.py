"""GPU parity of the quantisers against the oracle: codes, scale bytes (padding
included) and the FP32 tensor scale must match bit for bit."""
from concurrent.futures import ThreadPoolExecutor

import ml_dtypes
import numpy as np
import pytest
import torch

import mxfp4_microscaled_bit_b200 as fl
import synthetic_inputs as si
from gpu_util import DEV, check_mxfp4, check_nvfp4, status_ok

pytestmark = pytest.mark.gpu


# ------------------------------------------------------------------ element conversions
def _ref_e2m1(x):
    return x.astype(ml_dtypes.float4_e2m1fn).view(np.uint8) & 0xF


def _ref_e4m3(x):
    r = x.astype(ml_dtypes.float8_e4m3fn).view(np.uint8).copy()
    big = np.abs(x) > 448.0
    r[big] = np.where(np.signbit(x[big]), 0xFE, 0x7E)  # satfinite
    return r


def _chunk(lo, hi, step=1):
    bits = np.arange(lo, hi, step, dtype=np.uint64).astype(np.uint32)
    x = bits.view(np.float32)
    e2, e4 = fl.convert_selftest(torch.from_numpy(x).to(DEV))
    status_ok()
    e2, e4 = e2.cpu().numpy(), e4.cpu().numpy()
    with ThreadPoolExecutor(8) as ex:
        parts = list(ex.map(lambda sl: (_ref_e2m1(x[sl]), _ref_e4m3(x[sl])),
                            [slice(i, i + (1 << 22)) for i in range(0, x.size, 1 << 22)]))
    r2 = np.concatenate([p[0] for p in parts])
    r4 = np.concatenate([p[1] for p in parts])
    b2, b4 = np.nonzero(e2 != r2)[0], np.nonzero(e4 != r4)[0]
    assert b2.size == 0, ("e2m1", x[b2[:8]], e2[b2[:8]], r2[b2[:8]])
    assert b4.size == 0, ("e4m3", x[b4[:8]], e4[b4[:8]], r4[b4[:8]])


@pytest.mark.slow
def test_conversions_exhaustive_nonnegative():
    # every non-negative binary32 below 512 (all of E2M1's and E4M3's rounding decisions), then
    # +inf-side saturation on a stride; E2M1/E4M3 round to nearest even with saturation
    top = 0x44000000
    for lo in range(0, top, 1 << 28):
        _chunk(lo, min(top, lo + (1 << 28)))
    _chunk(top, 0x7F800000, 997)


def test_conversions_negative_sample():
    _chunk(0x80000000, 0xC4000000, 61)


def test_conversions_oracle_sample(orc):
    # the oracle agrees with the library conversions on values around every cut point
    grid = np.array([0, 0.5, 1, 1.5, 2, 3, 4, 6])
    mids = (grid[1:] + grid[:-1]) / 2
    x = np.concatenate([mids, np.nextafter(mids, 0), np.nextafter(mids, 9), [0.0, -0.0, -0.1, 7, 448, 449, 1e9]])
    x = np.concatenate([x, -x]).astype(np.float32)
    e2, e4 = fl.convert_selftest(torch.from_numpy(x).to(DEV))
    assert np.array_equal(e2.cpu().numpy(), orc.e2m1_encode(x))
    assert np.array_equal(e4.cpu().numpy(), orc.e4m3_encode(x))


# ------------------------------------------------------------------ NVFP4
def test_nvfp4_tiny_layer(orc):
    d = si.tiny()
    check_nvfp4(orc, d["A"])
    check_nvfp4(orc, d["W"])


@pytest.mark.parametrize("M", si.DECODE_M)
@pytest.mark.parametrize("K", [4096, 14336])
def test_nvfp4_decode_activations(orc, M, K):
    check_nvfp4(orc, si.decode_A(M, K))


@pytest.mark.parametrize("N,K", si.DECODE_NK)
def test_nvfp4_decode_weights(orc, N, K):
    check_nvfp4(orc, si.decode_W(N, K))


@pytest.mark.slow
def test_nvfp4_prefill_activations_rotated(orc):
    check_nvfp4(orc, si.prefill_A(), hadamard=16)


@pytest.mark.slow
def test_nvfp4_prefill_weights_rotated(orc):
    check_nvfp4(orc, si.prefill_W(), hadamard=16)


@pytest.mark.parametrize("rows", [1, 17, 129, 200, 257])
@pytest.mark.parametrize("cols", [64, 192, 320])
@pytest.mark.parametrize("hadamard", [0, 16])
def test_nvfp4_ragged(orc, rows, cols, hadamard):
    check_nvfp4(orc, si.student_t_bf16(rows * 1000 + cols, rows, cols), hadamard)


def test_nvfp4_strided_rows(orc):
    big = si.normal_bf16(5, 40, 512 + 64)
    x = big[:, :512]  # row stride 576 > cols
    assert x.stride(0) == 576
    c, s, gg = check_nvfp4(orc, x.contiguous(), 16)[:3]
    c2, s2, g2 = fl.nvfp4_quantize(big.to(DEV)[:, :512], 16)
    assert torch.equal(c2.cpu(), c.cpu()) and torch.equal(s2.cpu(), s.cpu()) and torch.equal(g2.cpu(), gg.cpu())


@pytest.mark.parametrize("g", [1.0, 1e-3, 7.5e-2])
def test_nvfp4_static_scale(orc, g):
    # small static scales push the block scales into E4M3 saturation and the codes into clipping
    check_nvfp4(orc, si.student_t_bf16(77, 64, 256), 0, g)
    check_nvfp4(orc, si.student_t_bf16(78, 64, 256), 16, g)


@pytest.mark.parametrize("k", [0, 3, 7])
def test_nvfp4_block_scale_near_e4m3_midpoints(orc, k):
    # Block j has maximum 1536 * 2^-j (exact in bf16), so (amax/6)/g = 256/g * 2^-j exactly
    # (barring underflow).  g is chosen so that 256/g lands within +-40 binary32 units of the
    # E4M3 rounding midpoint (1 + (2k+1)/16) * 2^8; every block then carries the same offset
    # from a midpoint into its own binade, through the normal, subnormal and zero range of
    # E4M3.  Both sides of each midpoint must round as the two-division definition does.
    mid = 1.0 + (2 * k + 1) / 16.0
    rows, cols = 8, 64  # 32 blocks
    j = np.arange(32, dtype=np.float64)
    amax = 1536.0 * 2.0 ** -j
    frac = np.array([1.0] + [((-1) ** i) * i / 16.0 for i in range(1, 16)])
    x = (amax[:, None] * frac[None, :]).astype(np.float32).reshape(rows, cols)
    xb = si.to_bf16(x)
    assert torch.equal(xb.float().abs().reshape(32, 16).amax(1), torch.from_numpy(amax.astype(np.float32)))
    for d in range(-40, 41):
        g = float(np.float32(1.0 / (mid * (1.0 + d * 2.0 ** -23))))
        check_nvfp4(orc, xb, 0, g)
    status_ok()


def test_nvfp4_zero_and_tiny_tensors(orc):
    check_nvfp4(orc, torch.zeros(3, 64, dtype=torch.bfloat16))
    tiny = si.normal_bf16(9, 5, 128, std=1e-30)
    check_nvfp4(orc, tiny)
    mixed = si.normal_bf16(10, 8, 128)
    mixed[3] *= 1e-20  # blocks whose scale underflows to zero relative to the tensor scale
    check_nvfp4(orc, mixed, 16)


# ------------------------------------------------------------------ MXFP4
@pytest.mark.slow
@pytest.mark.parametrize("hadamard", [0, 32])
def test_mxfp4_prefill_activations(orc, hadamard):
    check_mxfp4(orc, si.prefill_A(), hadamard)


@pytest.mark.parametrize("rows", [1, 17, 130])
@pytest.mark.parametrize("cols", [64, 128, 320])
@pytest.mark.parametrize("hadamard", [0, 32])
def test_mxfp4_ragged(orc, rows, cols, hadamard):
    # cols 64 and 320 leave half-empty scale atoms: their padding must be written 0
    check_mxfp4(orc, si.student_t_bf16(rows * 7 + cols, rows, cols), hadamard)


def test_mxfp4_extreme_exponents(orc):
    x = si.normal_bf16(11, 6, 128)
    x[0] *= 1e30
    x[1] *= 1e-30
    x[2, :32] = 0
    x[3, :] = 1e-39
    check_mxfp4(orc, x)
    check_mxfp4(orc, x, 32)


@pytest.mark.parametrize("hadamard", [0, 16])
def test_nvfp4_narrow_load_path(orc, hadamard):
    # base only 16-byte aligned and a row stride of 600 elements: no 256-bit loads
    big = si.student_t_bf16(12, 40, 600)
    x = big.to(DEV)[:, 8:8 + 512]
    assert x.data_ptr() % 32 == 16 and x.stride(0) == 600
    c, s, g = fl.nvfp4_quantize(x, hadamard)
    status_ok()
    oc, osl, og = orc.nvfp4_quantize(big[:, 8:8 + 512].contiguous(), hadamard)
    assert np.array_equal(c.cpu().numpy(), oc)
    assert np.array_equal(s.cpu().numpy(), orc.tc_scale_layout(osl))
    assert g.item() == float(og)


@pytest.mark.parametrize("hadamard", [0, 32])
def test_mxfp4_narrow_load_path(orc, hadamard):
    big = si.student_t_bf16(13, 33, 1048)
    x = big.to(DEV)[:, 8:8 + 1024]
    assert x.data_ptr() % 32 == 16
    c, s = fl.mxfp4_quantize(x, hadamard)
    status_ok()
    oc, osl = orc.mxfp4_quantize(big[:, 8:8 + 1024].contiguous(), hadamard)
    assert np.array_equal(c.cpu().numpy(), oc)
    assert np.array_equal(s.cpu().numpy(), orc.tc_scale_layout(osl))
