"""GEMM with the output NVFP4-quantised for the next layer (nvfp4_gemm_quant).  The codes and
scales must equal the oracle's NVFP4 quantisation (static tensor scale, optional 16-wide
rotation) of the GPU's own bf16 output, bit for bit, on every path that can produce them:
the 128x256 and 128x64 tile epilogues, the split-K reduction and the decode (swapped) epilogue.
The bf16 output itself must equal plain nvfp4_gemm's."""
import numpy as np
import pytest
import torch

import mxfp4_microscaled_bit_b200 as fl
import synthetic_inputs as si
from gpu_util import DEV, assert_bytes_equal, status_ok

pytestmark = pytest.mark.gpu

CASES = [
    (300, 1024, 1024, False),   # 128x256 tiles, one CTA per tile, no K split
    (300, 1024, 1024, "auto"),  # few tiles: K split, the reduction encodes
    (100, 512, 512, False),     # M <= 128: 128x64 tiles
    (257, 320, 320, "auto"),
    (16, 4096, 4096, False),    # decode: swapped operands, the epilogue encodes across lanes
    (16, 4096, 4096, "auto"),   # decode with a K split
    (1, 640, 256, False),
    (4, 14336, 512, "auto"),
]


def _operands(M, N, K, seed):
    ca, sa, ga = fl.nvfp4_quantize(si.student_t_bf16(seed, M, K).to(DEV), 16)
    cw, sw, gw = fl.nvfp4_quantize(si.normal_bf16(seed + 1, N, K, std=0.02).to(DEV), 16)
    return ca, sa, ga, cw, sw, gw


@pytest.mark.parametrize("M,N,K,ws", CASES)
@pytest.mark.parametrize("hadamard", [0, 16])
def test_output_quantisation_matches_oracle(orc, M, N, K, ws, hadamard):
    ca, sa, ga, cw, sw, gw = _operands(M, N, K, M + N + K)
    kw = {} if ws == "auto" else {"workspace": ws}
    y_ref = fl.nvfp4_gemm(ca, sa, ga, cw, sw, gw, **kw)
    status_ok()
    g_y = np.float32(orc.nvfp4_tensor_scale(y_ref.cpu(), hadamard))
    gy = torch.tensor([g_y], dtype=torch.float32, device=DEV)
    scales = torch.full((fl.scale_bytes(M, N // 16),), 0xFF, dtype=torch.uint8, device=DEV)
    codes = torch.full((M, N // 2), 0xAA, dtype=torch.uint8, device=DEV)
    y, c, s = fl.nvfp4_gemm_quant(ca, sa, ga, cw, sw, gw, gy, hadamard=hadamard, y_codes=codes, y_scales=scales,
                                  **kw)
    status_ok()
    assert torch.equal(y.view(torch.int16), y_ref.view(torch.int16)), "bf16 output differs from nvfp4_gemm"
    oc, osl, _ = orc.nvfp4_quantize(y.cpu(), hadamard, g_y)
    assert_bytes_equal(c.cpu().numpy(), oc, "output codes")
    assert_bytes_equal(s.cpu().numpy(), orc.tc_scale_layout(osl), "output scales")
    # without the bf16 output: the same encoding
    _, c2, s2 = fl.nvfp4_gemm_quant(ca, sa, ga, cw, sw, gw, gy, hadamard=hadamard, write_y=False, **kw)
    status_ok()
    assert torch.equal(c2, c) and torch.equal(s2, s)


def test_output_quantisation_saturating_scale(orc):
    # a static scale far too small: block scales saturate at 448 and codes at 6
    M, N, K = 64, 256, 512
    ca, sa, ga, cw, sw, gw = _operands(M, N, K, 7)
    gy = torch.tensor([1e-6], dtype=torch.float32, device=DEV)
    y, c, s = fl.nvfp4_gemm_quant(ca, sa, ga, cw, sw, gw, gy, hadamard=16, workspace=False)
    status_ok()
    oc, osl, _ = orc.nvfp4_quantize(y.cpu(), 16, np.float32(1e-6))
    assert_bytes_equal(c.cpu().numpy(), oc, "output codes")
    assert_bytes_equal(s.cpu().numpy(), orc.tc_scale_layout(osl), "output scales")


def test_output_quantisation_rejects_bad_shapes():
    M, N, K = 16, 96, 128  # N not a multiple of 64
    ca, sa, ga, cw, sw, gw = _operands(M, N, K, 9)
    gy = torch.ones(1, dtype=torch.float32, device=DEV)
    with pytest.raises(fl.Fp4LinError):
        fl.nvfp4_gemm_quant(ca, sa, ga, cw, sw, gw, gy)
    with pytest.raises(fl.Fp4LinError):
        ca2, sa2, ga2, cw2, sw2, gw2 = _operands(16, 128, 128, 10)
        fl.nvfp4_gemm_quant(ca2, sa2, ga2, cw2, sw2, gw2, gy, hadamard=8)
