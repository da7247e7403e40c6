"""GPU parity of the block-scaled GEMMs against the oracle's fp64 product of the
dequantised operands: every element within |y - y_ref| <= 1e-4 * sum|a_i b_i|
(applied before the bf16 rounding), exact where the exact result is known."""
import numpy as np
import pytest
import torch

import mxfp4_microscaled_bit_b200 as fl
import synthetic_inputs as si
from gpu_util import DEV, check_gemm_values, check_mxfp4, check_nvfp4, status_ok

pytestmark = pytest.mark.gpu


def _nv_layer(orc, A, W, hadamard=0, sample=None, workspace="auto"):
    ca, sa, ga, oca, osa, oga = check_nvfp4(orc, A, hadamard)
    cw, sw, gw, ocw, osw, ogw = check_nvfp4(orc, W, hadamard)
    kw = {} if workspace == "auto" else {"workspace": workspace}
    y = fl.nvfp4_gemm(ca, sa, ga, cw, sw, gw, **kw)
    status_ok()
    y = y.float().cpu().numpy()
    rows, cols = (slice(None), slice(None)) if sample is None else sample
    Ad = orc.dequant(oca[rows], osa[rows], "nvfp4", oga)
    Wd = orc.dequant(ocw[cols], osw[cols], "nvfp4", ogw)
    yr, s = orc.gemm_abt(Ad, Wd)
    return y[rows][:, cols], yr, s


def _mx_layer(orc, A, W, hadamard=0, sample=None):
    ca, sa, oca, osa = check_mxfp4(orc, A, hadamard)
    cw, sw, ocw, osw = check_mxfp4(orc, W, hadamard)
    y = fl.mxfp4_gemm(ca, sa, cw, sw)
    status_ok()
    y = y.float().cpu().numpy()
    rows, cols = (slice(None), slice(None)) if sample is None else sample
    yr, s = orc.gemm_abt(orc.dequant(oca[rows], osa[rows], "mxfp4"), orc.dequant(ocw[cols], osw[cols], "mxfp4"))
    return y[rows][:, cols], yr, s


# ------------------------------------------------------------------ exact cases
def _tc(orc, sf_lin):
    return torch.from_numpy(orc.tc_scale_layout(sf_lin)).to(DEV)


@pytest.mark.parametrize("M,N,K", [(16, 64, 128), (128, 256, 256), (200, 320, 512), (300, 520, 1024)])
def test_unit_scales_exact(orc, M, N, K):
    # with unit scales every product is a multiple of 1/4 and every partial sum is exact in fp32,
    # so y must equal bf16(exact sum): this pins the operand layouts, swizzle and descriptors
    rng = np.random.default_rng(M + N + K)
    ca = rng.integers(0, 256, size=(M, K // 2), dtype=np.uint8)
    cw = rng.integers(0, 256, size=(N, K // 2), dtype=np.uint8)
    one = np.float32(1.0)
    sa = np.full((M, K // 16), 0x38, np.uint8)
    sw = np.full((N, K // 16), 0x38, np.uint8)
    g = torch.ones(1, dtype=torch.float32, device=DEV)
    y = fl.nvfp4_gemm(torch.from_numpy(ca).to(DEV), _tc(orc, sa), g, torch.from_numpy(cw).to(DEV), _tc(orc, sw), g)
    status_ok()
    yr, _ = orc.gemm_abt(orc.dequant(ca, sa, "nvfp4", one), orc.dequant(cw, sw, "nvfp4", one))
    want = orc.bf16_rn(yr)
    got = y.cpu().view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(got, want), f"{np.count_nonzero(got != want)} of {got.size} differ"
    # the same with MXFP4 unit scales (E8M0 127)
    sa8 = np.full((M, K // 32), 127, np.uint8)
    sw8 = np.full((N, K // 32), 127, np.uint8)
    y8 = fl.mxfp4_gemm(torch.from_numpy(ca).to(DEV), _tc(orc, sa8), torch.from_numpy(cw).to(DEV), _tc(orc, sw8))
    status_ok()
    got8 = y8.cpu().view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(got8, want)


def test_scales_select_blocks(orc):
    # one nonzero scale per row in a different K block: y picks exactly that block's partial sum
    M, N, K = 64, 128, 512
    rng = np.random.default_rng(3)
    ca = rng.integers(0, 256, size=(M, K // 2), dtype=np.uint8)
    cw = rng.integers(0, 256, size=(N, K // 2), dtype=np.uint8)
    sa = np.zeros((M, K // 16), np.uint8)
    sa[np.arange(M), np.arange(M) % (K // 16)] = 0x40  # E4M3 2.0
    sw = rng.integers(0x30, 0x48, size=(N, K // 16), dtype=np.uint8)
    g = torch.ones(1, dtype=torch.float32, device=DEV)
    y = fl.nvfp4_gemm(torch.from_numpy(ca).to(DEV), _tc(orc, sa), g, torch.from_numpy(cw).to(DEV), _tc(orc, sw), g)
    status_ok()
    yr, s = orc.gemm_abt(orc.dequant(ca, sa, "nvfp4", 1.0), orc.dequant(cw, sw, "nvfp4", 1.0))
    check_gemm_values(orc, y.float().cpu().numpy(), yr, s, "block select")


# ------------------------------------------------------------------ the workloads
def test_tiny_layer(orc):
    d = si.tiny()
    y, yr, s = _nv_layer(orc, d["A"], d["W"])
    print("tiny max rel err", check_gemm_values(orc, y, yr, s, "tiny"))


@pytest.mark.parametrize("M", si.DECODE_M)
@pytest.mark.parametrize("N,K", si.DECODE_NK)
def test_decode_shapes(orc, M, N, K):
    A, W = si.decode_A(M, K), si.decode_W(N, K)
    y, yr, s = _nv_layer(orc, A, W)
    print(f"decode M={M} N={N} K={K} max rel err", check_gemm_values(orc, y, yr, s, "decode"))


def test_decode_without_workspace_matches(orc):
    A, W = si.decode_A(16, 4096), si.decode_W(4096, 4096)
    y1, yr, s = _nv_layer(orc, A, W, workspace=False)  # no workspace: K is not split
    check_gemm_values(orc, y1, yr, s, "decode, no split")


def _sample(M, N, rng, n=48):
    rows = np.unique(np.concatenate([[0, 127, 128, M - 1], rng.integers(0, M, n)]))
    cols = np.unique(np.concatenate([[0, 255, 256, N - 1], rng.integers(0, N, n)]))
    return rows, cols


@pytest.mark.slow
def test_prefill_rotated_sampled(orc):
    M, N, K = si.PREFILL["M"], si.PREFILL["N"], si.PREFILL["K"]
    rows, cols = _sample(M, N, np.random.default_rng(2))
    y, yr, s = _nv_layer(orc, si.prefill_A(), si.prefill_W(), 16, sample=(rows, cols))
    print("prefill max rel err", check_gemm_values(orc, y, yr, s, "prefill"))


@pytest.mark.slow
@pytest.mark.parametrize("hadamard", [0, 32])
def test_prefill_mxfp4_sampled(orc, hadamard):
    M, N = si.PREFILL["M"], si.PREFILL["N"]
    rows, cols = _sample(M, N, np.random.default_rng(3))
    y, yr, s = _mx_layer(orc, si.prefill_A(), si.prefill_W(), hadamard, sample=(rows, cols))
    print("prefill mxfp4 max rel err", check_gemm_values(orc, y, yr, s, "prefill mxfp4"))


@pytest.mark.parametrize("M,N,K", [(1, 64, 64), (17, 72, 128), (129, 200, 320), (200, 320, 576),
                                   (257, 264, 1024), (300, 520, 4096), (4, 1000, 1216)])
@pytest.mark.parametrize("hadamard", [0, 16])
def test_ragged_nvfp4(orc, M, N, K, hadamard):
    A = si.student_t_bf16(M + K, M, K)
    W = si.normal_bf16(N + K, N, K, std=0.02)
    y, yr, s = _nv_layer(orc, A, W, hadamard)
    check_gemm_values(orc, y, yr, s, f"ragged {M}x{N}x{K}")


@pytest.mark.parametrize("M,N,K", [(1, 64, 64), (17, 72, 192), (129, 200, 320), (257, 264, 1024)])
@pytest.mark.parametrize("hadamard", [0, 32])
def test_ragged_mxfp4(orc, M, N, K, hadamard):
    A = si.student_t_bf16(M + K + 1, M, K)
    W = si.normal_bf16(N + K + 1, N, K, std=0.02)
    y, yr, s = _mx_layer(orc, A, W, hadamard)
    check_gemm_values(orc, y, yr, s, f"ragged mx {M}x{N}x{K}")


def test_output_row_stride(orc):
    d = si.tiny()
    ca, sa, ga = fl.nvfp4_quantize(d["A"].to(DEV))
    cw, sw, gw = fl.nvfp4_quantize(d["W"].to(DEV))
    big = torch.full((16, 80), 7.0, dtype=torch.bfloat16, device=DEV)
    fl.nvfp4_gemm(ca, sa, ga, cw, sw, gw, out=big[:, :64])
    ref = fl.nvfp4_gemm(ca, sa, ga, cw, sw, gw)
    status_ok()
    assert torch.equal(big[:, :64], ref) and bool((big[:, 64:] == 7.0).all())


def test_nvfp4_beats_mxfp4_error(orc):
    # relative Frobenius error against the fp64 product of the unquantised operands: NVFP4's finer
    # scaling beats MXFP4, and the 32-wide rotation helps MXFP4 on heavy-tailed activations
    M, N, K = 256, 256, 1024
    A = si.student_t_bf16(501, M, K)
    W = si.normal_bf16(502, N, K, std=0.02)
    exact = A.double().numpy() @ W.double().numpy().T
    errs = {}
    for name, fn in [("nv", lambda: _nv_layer(orc, A, W)), ("nv_h", lambda: _nv_layer(orc, A, W, 16)),
                     ("mx", lambda: _mx_layer(orc, A, W)), ("mx_h", lambda: _mx_layer(orc, A, W, 32))]:
        y = fn()[0]
        errs[name] = np.linalg.norm(y - exact) / np.linalg.norm(exact)
    print("relative Frobenius errors", errs)
    assert errs["nv"] < errs["mx"] and errs["nv_h"] < errs["mx_h"]


def test_binding_refuses_undersized_buffers():
    # a caller-supplied buffer smaller than what the call writes raises before any launch
    x = si.normal_bf16(3, 32, 128).to(DEV)
    codes = torch.full((32, 64), 0xAA, dtype=torch.uint8, device=DEV)
    small = torch.full((100,), 0xAA, dtype=torch.uint8, device=DEV)  # the layout needs 512 bytes
    with pytest.raises(ValueError, match="scales holds 100 bytes"):
        fl.nvfp4_quantize(x, 0, codes=codes, scales=small)
    torch.cuda.synchronize()
    assert bool((codes == 0xAA).all()) and bool((small == 0xAA).all())
    c, s, g = fl.nvfp4_quantize(x)
    y_small = torch.full((16, 32), 7.0, dtype=torch.bfloat16, device=DEV)  # 32 rows are written
    with pytest.raises(ValueError, match="out holds"):
        fl.nvfp4_gemm(c, s, g, c, s, g, out=y_small)
    torch.cuda.synchronize()
    assert bool((y_small == 7.0).all())
    with pytest.raises(ValueError, match="out_scale must be contiguous|out holds"):
        kc = torch.zeros(1, 1, 8, 64, dtype=torch.uint8, device=DEV)
        ks = torch.full((1, 1, 8, 8), 0x38, dtype=torch.uint8, device=DEV)
        fl.kv_nvfp4_load_fp8(kc, ks, torch.ones(1, device=DEV), 8, out=torch.empty(1, 1, 4, 128, dtype=torch.uint8,
                                                                                     device=DEV))
    status_ok()
