"""GPU parity of the scale-choice variants against the oracle, bit for bit: the NVFP4
quantiser whose block scales minimise each block's squared error (nvfp4_quantize_mse) and
the MXFP4 quantiser with nearest-power-of-two scales (mxfp4_quantize_nearest).  Codes,
every scale byte (padding included) and the tensor scale must match."""
import numpy as np
import pytest
import torch

import mxfp4_microscaled_bit_b200 as fl
import synthetic_inputs as si
from gpu_util import DEV, assert_bytes_equal, status_ok

pytestmark = pytest.mark.gpu


def _gpu_mse(x_cpu, hadamard=0, g=None):
    x = x_cpu.to(DEV)
    rows, cols = x.shape
    codes = torch.full((rows, cols // 2), 0xAA, dtype=torch.uint8, device=DEV)
    scales = torch.full((fl.scale_bytes(rows, cols // 16),), 0xFF, dtype=torch.uint8, device=DEV)
    gt = None if g is None else torch.tensor([g], dtype=torch.float32, device=DEV)
    c, s, gg = fl.nvfp4_quantize(x, hadamard, gt, codes=codes, scales=scales, mse=True)
    status_ok()
    return c.cpu().numpy(), s.cpu().numpy(), np.float32(gg.item())


def _check_mse(orc, x_cpu, hadamard=0, g=None):
    c, s, gg = _gpu_mse(x_cpu, hadamard, g)
    oc, osl, og = orc.nvfp4_quantize_mse(x_cpu, hadamard, g)
    assert gg.view(np.uint32) == np.float32(og).view(np.uint32), (gg, og)
    assert_bytes_equal(s, orc.tc_scale_layout(osl), "mse scales")
    assert_bytes_equal(c, oc, "mse codes")
    return oc, osl, og


@pytest.mark.parametrize("rows,cols", [(1, 64), (17, 192), (130, 320), (256, 1024)])
@pytest.mark.parametrize("hadamard", [0, 16])
def test_mse_ragged(orc, rows, cols, hadamard):
    _check_mse(orc, si.student_t_bf16(rows * 31 + cols, rows, cols), hadamard)


@pytest.mark.parametrize("g", [1.0, 1e-3, 2.5e-2])
def test_mse_static_scale(orc, g):
    # small static scales push many candidates into E4M3 and E2M1 saturation
    _check_mse(orc, si.normal_bf16(41, 64, 256), 0, g)
    _check_mse(orc, si.student_t_bf16(42, 64, 256), 16, g)


def test_mse_wide_range_and_zero_rows(orc):
    x = si.normal_bf16(43, 48, 512) * torch.logspace(-12, 12, 48).to(torch.bfloat16)[:, None]
    x[5] = 0
    x[6, :16] = 0
    _check_mse(orc, x, 16)


def test_mse_decode_weight_and_error(orc):
    # a decode weight: the MSE choice must not lose to amax/6 in relative Frobenius error
    W = si.decode_W(4096, 1024)
    oc, osl, og = _check_mse(orc, W)
    dc, dsl, dg = orc.nvfp4_quantize(W)
    ref = W.double().numpy()
    e_mse = np.linalg.norm(orc.dequant(oc, osl, "nvfp4", og) - ref) / np.linalg.norm(ref)
    e_def = np.linalg.norm(orc.dequant(dc, dsl, "nvfp4", dg) - ref) / np.linalg.norm(ref)
    print(f"relative Frobenius error: amax/6 {e_def:.5f}, MSE-optimal {e_mse:.5f}")
    assert e_mse < e_def


@pytest.mark.slow
def test_mse_prefill_weight_sampled(orc):
    # the full prefill weight (14336 x 4096, rotated) on the GPU; rows sampled for the oracle,
    # with the tensor scale of the whole tensor
    W = si.prefill_W()
    c, s, gg = _gpu_mse(W, 16)
    og = orc.nvfp4_tensor_scale(W, 16)
    assert gg == og
    rows = np.unique(np.concatenate([[0, 127, 128, W.shape[0] - 1], np.random.default_rng(5).integers(0, W.shape[0], 60)]))
    oc, osl, _ = orc.nvfp4_quantize_mse(W[torch.from_numpy(rows)], 16, og)
    assert_bytes_equal(c[rows], oc, "mse codes (sampled rows)")
    lin = s  # tensor-core layout of all rows: pick the sampled rows' bytes
    katoms = (W.shape[1] // 16 + 3) // 4
    r = rows[:, None]
    k = np.arange(W.shape[1] // 16)[None, :]
    off = ((r >> 7) * katoms + (k >> 2)) * 512 + (r & 31) * 16 + ((r >> 5) & 3) * 4 + (k & 3)
    assert_bytes_equal(lin[off], osl, "mse scales (sampled rows)")


# ------------------------------------------------------------------ MXFP4, nearest power of two
def _check_nearest(orc, x_cpu, hadamard=0):
    x = x_cpu.to(DEV)
    rows, cols = x.shape
    codes = torch.full((rows, cols // 2), 0xAA, dtype=torch.uint8, device=DEV)
    scales = torch.full((fl.scale_bytes(rows, cols // 32),), 0xFF, dtype=torch.uint8, device=DEV)
    c, s = fl.mxfp4_quantize(x, hadamard, codes=codes, scales=scales, nearest=True)
    status_ok()
    oc, osl = orc.mxfp4_quantize(x_cpu, hadamard, nearest=True)
    assert_bytes_equal(c.cpu().numpy(), oc, "nearest codes")
    assert_bytes_equal(s.cpu().numpy(), orc.tc_scale_layout(osl), "nearest scales")


@pytest.mark.parametrize("rows,cols", [(1, 64), (17, 128), (130, 320), (512, 2048)])
@pytest.mark.parametrize("hadamard", [0, 32])
def test_nearest_ragged(orc, rows, cols, hadamard):
    _check_nearest(orc, si.student_t_bf16(rows * 37 + cols, rows, cols), hadamard)


def test_nearest_extreme_exponents(orc):
    x = si.normal_bf16(44, 8, 128)
    x[0] *= 1e30
    x[1] *= 1e-30
    x[2, :32] = 0
    x[3, :] = 1e-39
    x[4, :] = 8.875  # amax / 6 = 1.479: the lower power of two, values clip to 6
    x[5, :] = 9.0    # amax / 6 = 1.5: the tie goes to the upper power of two
    _check_nearest(orc, x)
    _check_nearest(orc, x, 32)


@pytest.mark.slow
def test_nearest_prefill_activations(orc):
    _check_nearest(orc, si.prefill_A(), 32)
