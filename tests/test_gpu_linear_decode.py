"""Decode linear layer with the activation quantiser inside the GEMM (nvfp4_linear_decode).
The GEMM's own warps encode the bf16 activations, so the result must equal, bit for bit, the
two-launch path nvfp4_quantize then nvfp4_gemm (whose parity against the oracle is checked
elsewhere), and the computed tensor scale must equal the quantiser's.  One case per form is
also checked against the oracle directly: the oracle quantises x, dequantises both operands
and takes the fp64 product; y must lie in the bf16 window of that product."""
import numpy as np
import pytest
import torch

import mxfp4_microscaled_bit_b200 as fl
import synthetic_inputs as si
from gpu_util import DEV, check_gemm_values, status_ok

pytestmark = pytest.mark.gpu


def _weights(N, K, hadamard, seed):
    return fl.nvfp4_quantize(si.normal_bf16(seed, N, K, std=0.02).to(DEV), hadamard)


def _bits(y):
    return y.view(torch.int16)


# up to 16384 activation values every CTA takes the amax itself; above, a separate amax pass
SHAPES = [(1, 640, 256), (4, 4096, 4096), (5, 320, 1088), (16, 14336, 512), (16, 4096, 4096), (3, 128, 64),
          (16, 512, 8192), (11, 1024, 14336)]


@pytest.mark.parametrize("M,N,K", SHAPES)
@pytest.mark.parametrize("hadamard", [0, 16])
@pytest.mark.parametrize("dynamic", [True, False])
def test_fused_equals_two_launch_path(M, N, K, hadamard, dynamic):
    x = si.student_t_bf16(M * 7 + K, M, K).to(DEV)
    cw, sw, gw = _weights(N, K, hadamard, N + K)
    g_in = None if dynamic else torch.tensor([float(x.abs().max()) / 2000.0], dtype=torch.float32, device=DEV)
    ca, sa, ga = fl.nvfp4_quantize(x, hadamard, g_in)
    y_ref = fl.nvfp4_gemm(ca, sa, ga, cw, sw, gw)
    status_ok()
    for ws in (None, False):  # with the planned K split, and unsplit
        if dynamic and ws is False:
            continue  # the amax partials need a workspace
        g_arg = None if dynamic else g_in.clone()
        y, g = fl.nvfp4_linear_decode(x, cw, sw, gw, hadamard=hadamard, g_a=g_arg, workspace=ws)
        status_ok()
        assert torch.equal(_bits(y), _bits(y_ref)), (M, N, K, hadamard, dynamic, ws)
        assert g.view(torch.int32).item() == ga.view(torch.int32).item()


def test_fused_strided_input_and_output():
    # x and y as row slices of wider buffers
    M, N, K = 7, 1024, 512
    big = si.student_t_bf16(11, M, K + 64).to(DEV)
    x = big[:, 32:32 + K]
    cw, sw, gw = _weights(N, K, 16, 12)
    ybig = torch.full((M, N + 64), 7.0, dtype=torch.bfloat16, device=DEV)
    y, g = fl.nvfp4_linear_decode(x, cw, sw, gw, hadamard=16, out=ybig[:, :N])
    status_ok()
    ca, sa, ga = fl.nvfp4_quantize(x.contiguous(), 16)
    y_ref = fl.nvfp4_gemm(ca, sa, ga, cw, sw, gw)
    assert torch.equal(_bits(ybig[:, :N]), _bits(y_ref))
    assert torch.all(ybig[:, N:] == 7.0), "wrote outside y"


def test_fused_zero_activations():
    # amax 0: the quantiser's tensor scale falls back to 1 and every code is 0
    M, N, K = 2, 256, 256
    x = torch.zeros(M, K, dtype=torch.bfloat16, device=DEV)
    cw, sw, gw = _weights(N, K, 0, 13)
    y, g = fl.nvfp4_linear_decode(x, cw, sw, gw)
    status_ok()
    assert float(g) == 1.0
    assert torch.all(y == 0)


@pytest.mark.parametrize("M,N,K,hadamard", [(16, 1024, 1024, 16), (3, 384, 320, 0)])
def test_fused_matches_oracle(orc, M, N, K, hadamard):
    xc = si.student_t_bf16(21 + M, M, K)
    wc = si.normal_bf16(22 + N, N, K, std=0.02)
    cw, sw, gw = fl.nvfp4_quantize(wc.to(DEV), hadamard)
    y, g = fl.nvfp4_linear_decode(xc.to(DEV), cw, sw, gw, hadamard=hadamard)
    status_ok()
    oca, osa, oga = orc.nvfp4_quantize(xc, hadamard)
    ocw, osw, ogw = orc.nvfp4_quantize(wc, hadamard)
    assert np.float32(g.item()).view(np.uint32) == np.float32(oga).view(np.uint32)
    yr, s = orc.gemm_abt(orc.dequant(oca, osa, "nvfp4", oga), orc.dequant(ocw, osw, "nvfp4", ogw))
    check_gemm_values(orc, y.float().cpu().numpy(), yr, s, "fused decode layer")


def test_linear_routes_decode_sizes_through_fused_path():
    M, N, K = 9, 512, 512
    x = si.student_t_bf16(30, M, K).to(DEV)
    w = fl.prepare_weight(si.normal_bf16(31, N, K, std=0.02).to(DEV), "nvfp4", 16)
    y = fl.nvfp4_linear(x, w)
    status_ok()
    ca, sa, ga = fl.nvfp4_quantize(x, 16)
    assert torch.equal(_bits(y), _bits(fl.nvfp4_gemm(ca, sa, ga, w.codes, w.scales, w.g)))


# ---------------------------------------------------------------- weights in tile order
def _tile_reference(codes: np.ndarray) -> np.ndarray:
    """The documented tile order, built with numpy: tile (mt, kt) = rows 128 mt.., code bytes
    128 kt.., 16-byte chunk c of row r at position c ^ (r % 8); zero padding."""
    N, KB = codes.shape
    nm, nk = (N + 127) // 128, (KB + 127) // 128
    pad = np.zeros((nm * 128, nk * 128), dtype=np.uint8)
    pad[:N, :KB] = codes
    t = pad.reshape(nm, 128, nk, 8, 16).transpose(0, 2, 1, 3, 4)  # [mt, kt, r, c, 16]
    out = np.empty_like(t)
    for r in range(128):
        for c in range(8):
            out[:, :, r, c ^ (r % 8)] = t[:, :, r, c]
    return out.reshape(-1)


@pytest.mark.parametrize("N,K", [(200, 320), (128, 256), (1, 64), (4096, 1088)])
def test_tile_order_matches_documented_layout(N, K):
    codes = torch.randint(0, 256, (N, K // 2), dtype=torch.uint8, device=DEV)
    tiled = fl.tile_weights(codes)
    status_ok()
    assert np.array_equal(tiled.cpu().numpy(), _tile_reference(codes.cpu().numpy()))


@pytest.mark.parametrize("M,N,K", [(1, 640, 256), (5, 320, 1088), (16, 14336, 512), (16, 4096, 4096), (4, 136, 64),
                                   (16, 4096, 14336)])
@pytest.mark.parametrize("hadamard", [0, 16])
def test_tiled_weights_give_the_same_bits(M, N, K, hadamard):
    x = si.student_t_bf16(M * 5 + K, M, K).to(DEV)
    cw, sw, gw = _weights(N, K, hadamard, N + 2 * K)
    tiled = fl.tile_weights(cw)
    ca, sa, ga = fl.nvfp4_quantize(x, hadamard)
    y_ref = fl.nvfp4_gemm(ca, sa, ga, cw, sw, gw)
    status_ok()
    y_t = fl.nvfp4_gemm_tiled(ca, sa, ga, tiled, sw, gw, N)
    y_f, g = fl.nvfp4_linear_decode(x, tiled, sw, gw, hadamard=hadamard, tiled_n=N)
    status_ok()
    assert torch.equal(_bits(y_t), _bits(y_ref))
    assert torch.equal(_bits(y_f), _bits(y_ref))
    assert torch.equal(g, ga)
    y_u, _ = fl.nvfp4_linear_decode(x, tiled, sw, gw, hadamard=hadamard, tiled_n=N, workspace=False,
                                    g_a=ga.clone())  # unsplit, static scale
    status_ok()
    assert torch.equal(_bits(y_u), _bits(y_ref))


def test_linear_uses_tiled_weights():
    M, N, K = 3, 1024, 512
    x = si.student_t_bf16(60, M, K).to(DEV)
    wt = fl.prepare_weight(si.normal_bf16(61, N, K, std=0.02).to(DEV), "nvfp4", 16, tiled=True)
    assert wt.tiled is not None
    y = fl.nvfp4_linear(x, wt)
    status_ok()
    ca, sa, ga = fl.nvfp4_quantize(x, 16)
    assert torch.equal(_bits(y), _bits(fl.nvfp4_gemm(ca, sa, ga, wt.codes, wt.scales, wt.g)))
