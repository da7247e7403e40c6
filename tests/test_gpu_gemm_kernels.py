"""Both GEMM kernels -- one CTA per 128 x 256 tile, and the CTA pair (cta_group::2) per
256 x 256 tile -- against the oracle, forced in turn through FP4LIN_GEMM_KERNEL and run
without a K split.  Shapes leave ragged M, N and K tails, odd numbers of 128-row tiles
(the second CTA of a pair then reads only zero rows) and more tiles than resident
CTAs, so the persistent loop wraps its stage ring across tiles."""
import numpy as np
import pytest
import torch

import mxfp4_microscaled_bit_b200 as fl
import synthetic_inputs as si
from gpu_util import DEV, check_gemm_values, check_mxfp4, check_nvfp4, status_ok

pytestmark = pytest.mark.gpu

KERNELS = ["single", "pair"]


@pytest.fixture(params=KERNELS)
def kernel(request, monkeypatch):
    monkeypatch.setenv("FP4LIN_GEMM_KERNEL", request.param)
    return request.param


def _tc(orc, sf_lin):
    return torch.from_numpy(orc.tc_scale_layout(sf_lin)).to(DEV)


@pytest.mark.parametrize("M,N,K", [(256, 256, 256), (257, 264, 320), (520, 304, 1088), (640, 1024, 4096)])
def test_unit_scales_exact(orc, kernel, M, N, K):
    # unit scales: every partial sum is a multiple of 1/4 and exact in fp32, so y = bf16(exact)
    rng = np.random.default_rng(7 * M + N + K)
    ca = rng.integers(0, 256, size=(M, K // 2), dtype=np.uint8)
    cw = rng.integers(0, 256, size=(N, K // 2), dtype=np.uint8)
    one = np.float32(1.0)
    yr, _ = orc.gemm_abt(orc.dequant(ca, np.full((M, K // 16), 0x38, np.uint8), "nvfp4", one),
                         orc.dequant(cw, np.full((N, K // 16), 0x38, np.uint8), "nvfp4", one))
    want = orc.bf16_rn(yr)
    g = torch.ones(1, dtype=torch.float32, device=DEV)
    dca, dcw = torch.from_numpy(ca).to(DEV), torch.from_numpy(cw).to(DEV)
    y = fl.nvfp4_gemm(dca, _tc(orc, np.full((M, K // 16), 0x38, np.uint8)), g,
                      dcw, _tc(orc, np.full((N, K // 16), 0x38, np.uint8)), g, workspace=False)
    status_ok()
    got = y.cpu().view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(got, want), f"nvfp4 {kernel}: {np.count_nonzero(got != want)} of {got.size} differ"
    y8 = fl.mxfp4_gemm(dca, _tc(orc, np.full((M, K // 32), 127, np.uint8)),
                       dcw, _tc(orc, np.full((N, K // 32), 127, np.uint8)), workspace=False)
    status_ok()
    got8 = y8.cpu().view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(got8, want), f"mxfp4 {kernel}: {np.count_nonzero(got8 != want)} of {got8.size} differ"


@pytest.mark.parametrize("M,N,K", [(300, 520, 1024), (513, 776, 1216), (2048, 4096, 1024)])
def test_random_nvfp4(orc, kernel, M, N, K):
    A = si.student_t_bf16(11 * M + K, M, K)
    W = si.normal_bf16(13 * N + K, N, K, std=0.02)
    ca, sa, ga, oca, osa, oga = check_nvfp4(orc, A, 16)
    cw, sw, gw, ocw, osw, ogw = check_nvfp4(orc, W, 16)
    y = fl.nvfp4_gemm(ca, sa, ga, cw, sw, gw, workspace=False)
    status_ok()
    yr, s = orc.gemm_abt(orc.dequant(oca, osa, "nvfp4", oga), orc.dequant(ocw, osw, "nvfp4", ogw))
    check_gemm_values(orc, y.float().cpu().numpy(), yr, s, f"nvfp4 {kernel} {M}x{N}x{K}")


@pytest.mark.parametrize("M,N,K", [(300, 520, 1024), (513, 776, 1216)])
def test_random_mxfp4(orc, kernel, M, N, K):
    A = si.student_t_bf16(17 * M + K, M, K)
    W = si.normal_bf16(19 * N + K, N, K, std=0.02)
    ca, sa, oca, osa = check_mxfp4(orc, A, 32)
    cw, sw, ocw, osw = check_mxfp4(orc, W, 32)
    y = fl.mxfp4_gemm(ca, sa, cw, sw, workspace=False)
    status_ok()
    yr, s = orc.gemm_abt(orc.dequant(oca, osa, "mxfp4"), orc.dequant(ocw, osw, "mxfp4"))
    check_gemm_values(orc, y.float().cpu().numpy(), yr, s, f"mxfp4 {kernel} {M}x{N}x{K}")


def test_kernels_agree_bitwise(monkeypatch):
    # the two kernels issue the same K-ordered sequence of 64-deep block-scaled MMAs per output
    # element, so their outputs agree bit for bit
    M, N, K = 1000, 1304, 2112
    ca, sa, ga = fl.nvfp4_quantize(si.student_t_bf16(23, M, K).to(DEV), 16)
    cw, sw, gw = fl.nvfp4_quantize(si.normal_bf16(29, N, K, std=0.02).to(DEV), 16)
    out = {}
    for k in KERNELS:
        monkeypatch.setenv("FP4LIN_GEMM_KERNEL", k)
        out[k] = fl.nvfp4_gemm(ca, sa, ga, cw, sw, gw, workspace=False)
        status_ok()
    diff = (out["single"].view(torch.int16) != out["pair"].view(torch.int16)).sum().item()
    assert diff == 0, f"{diff} elements differ between the kernels"


# ---------------------------------------------------------------- the decode GEMM on CTA pairs
DECODE_CASES = [(1, 64, 64), (16, 256, 256), (5, 320, 1088), (16, 4096, 4096), (4, 14336, 4096), (16, 4096, 14336),
                (9, 4224, 512)]


@pytest.mark.parametrize("M,N,K", DECODE_CASES)
@pytest.mark.parametrize("fmt", ["nvfp4", "mxfp4"])
def test_decode_pair_matches_single_and_oracle(orc, monkeypatch, M, N, K, fmt):
    # the pair issues, per output element, the same K-ordered 64-deep MMAs as the one-CTA
    # decode form (M = 256 instead of 128 on the weight side): the same bits, split or not
    A = si.student_t_bf16(M + N, M, K)
    W = si.normal_bf16(N + K, N, K, std=0.02)
    out = {}
    for kernel in ("single", "pair"):
        monkeypatch.setenv("FP4LIN_DECODE_KERNEL", kernel)
        for ws in ("auto", False):
            kw = {} if ws == "auto" else {"workspace": ws}
            if fmt == "nvfp4":
                ca, sa, ga = fl.nvfp4_quantize(A.to(DEV), 16)
                cw, sw, gw = fl.nvfp4_quantize(W.to(DEV), 16)
                out[kernel, ws] = fl.nvfp4_gemm(ca, sa, ga, cw, sw, gw, **kw)
            else:
                ca, sa = fl.mxfp4_quantize(A.to(DEV), 32)
                cw, sw = fl.mxfp4_quantize(W.to(DEV), 32)
                out[kernel, ws] = fl.mxfp4_gemm(ca, sa, cw, sw, **kw)
            status_ok()
    for ws in ("auto", False):
        assert torch.equal(out["pair", ws].view(torch.int16), out["single", ws].view(torch.int16)), ws
    # and against the oracle's product (the unsplit pair output)
    if fmt == "nvfp4":
        oca, osa, oga = orc.nvfp4_quantize(A, 16)
        ocw, osw, ogw = orc.nvfp4_quantize(W, 16)
        yr, s = orc.gemm_abt(orc.dequant(oca, osa, "nvfp4", oga), orc.dequant(ocw, osw, "nvfp4", ogw))
    else:
        oca, osa = orc.mxfp4_quantize(A, 32)
        ocw, osw = orc.mxfp4_quantize(W, 32)
        yr, s = orc.gemm_abt(orc.dequant(oca, osa, "mxfp4"), orc.dequant(ocw, osw, "mxfp4"))
    check_gemm_values(orc, out["pair", False].float().cpu().numpy(), yr, s, f"decode pair {fmt} {M}x{N}x{K}")
