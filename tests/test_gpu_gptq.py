"""MR-GPTQ on the GPU (nvfp4_gptq_quantize / mxfp4_gptq_quantize) against the oracle's sweep
(reading R12), bit for bit: codes, every scale byte in the tensor-core layout (padding
included) and the computed tensor scale.  Both sides take the same inverse-Hessian factor U,
computed by the oracle from seeded calibration activations; the sweep is binary32 in a fixed
order on both sides, so every quantisation decision must agree."""
import numpy as np
import pytest
import torch

import mxfp4_microscaled_bit_b200 as fl
import synthetic_inputs as si
from gpu_util import DEV, assert_bytes_equal, status_ok

pytestmark = pytest.mark.gpu

FORMS = [("nvfp4", 0), ("nvfp4", 16), ("mxfp4", 0), ("mxfp4", 32)]


def _case(orc, N, K, had, seed):
    w = si.normal_bf16(seed, N, K, std=0.02)
    u = orc.gptq_hessian_factor(si.gptq_calibration(seed + 1, 2 * K, K), had)
    return w, u


def _gpu(w, u, fmt, had, g=None):
    N, K = w.shape
    G = 16 if fmt == "nvfp4" else 32
    codes = torch.full((N, K // 2), 0xAA, dtype=torch.uint8, device=DEV)
    scales = torch.full((fl.scale_bytes(N, K // G),), 0xFF, dtype=torch.uint8, device=DEV)
    gt = None if g is None else torch.tensor([g], dtype=torch.float32, device=DEV)
    c, s, gg = fl.gptq_quantize(w.to(DEV), torch.from_numpy(u).to(DEV), fmt, had, gt, codes=codes, scales=scales)
    status_ok()
    return c.cpu().numpy(), s.cpu().numpy(), (None if gg is None else np.float32(gg.item()))


@pytest.mark.parametrize("fmt,had", FORMS)
@pytest.mark.parametrize("N,K", [(24, 128), (200, 320), (130, 1024), (1, 64), (257, 192)])
def test_gptq_matches_oracle(orc, fmt, had, N, K):
    w, u = _case(orc, N, K, had, N + K)
    c, s, g = _gpu(w, u, fmt, had)
    oc, osf, og = orc.gptq(w, u, fmt, had)
    if fmt == "nvfp4":
        assert np.float32(g).view(np.uint32) == np.float32(og).view(np.uint32), (g, og)
    assert_bytes_equal(c, oc, "codes")
    assert_bytes_equal(s, orc.tc_scale_layout(osf), "scales")


@pytest.mark.parametrize("had", [0, 16])
@pytest.mark.parametrize("N,K", [(24, 128), (200, 320), (1, 64), (130, 512)])
def test_gptq_mse_matches_oracle(orc, had, N, K):
    w, u = _case(orc, N, K, had, 3 * N + K)
    codes = torch.full((N, K // 2), 0xAA, dtype=torch.uint8, device=DEV)
    scales = torch.full((fl.scale_bytes(N, K // 16),), 0xFF, dtype=torch.uint8, device=DEV)
    c, s, g = fl.gptq_quantize(w.to(DEV), torch.from_numpy(u).to(DEV), "nvfp4", had, codes=codes, scales=scales,
                               mse=True)
    status_ok()
    oc, osf, og = orc.gptq(w, u, "nvfp4", had, mse=True)
    assert np.float32(g.item()).view(np.uint32) == np.float32(og).view(np.uint32)
    assert_bytes_equal(c.cpu().numpy(), oc, "codes")
    assert_bytes_equal(s.cpu().numpy(), orc.tc_scale_layout(osf), "scales")


def test_gptq_static_scale(orc):
    N, K = 64, 256
    w, u = _case(orc, N, K, 16, 5)
    g = np.float32(3e-6)  # small: block scales saturate
    c, s, gg = _gpu(w, u, "nvfp4", 16, g)
    oc, osf, _ = orc.gptq(w, u, "nvfp4", 16, g)
    assert gg == g
    assert_bytes_equal(c, oc, "codes")
    assert_bytes_equal(s, orc.tc_scale_layout(osf), "scales")


@pytest.mark.parametrize("fmt,had", [("nvfp4", 16), ("mxfp4", 32)])
def test_identity_factor_is_the_quantiser(fmt, had):
    # no error feedback: GPTQ must reproduce the plain quantiser's bytes
    N, K = 300, 512
    w = si.normal_bf16(9, N, K, std=0.02).to(DEV)
    u = torch.eye(K, dtype=torch.float32, device=DEV)
    c, s, g = fl.gptq_quantize(w, u, fmt, had)
    status_ok()
    if fmt == "nvfp4":
        rc, rs, rg = fl.nvfp4_quantize(w, had)
        assert torch.equal(g, rg)
    else:
        rc, rs = fl.mxfp4_quantize(w, had)
    status_ok()
    assert torch.equal(c, rc) and torch.equal(s, rs)


def test_gptq_weights_in_the_gemm(orc):
    # the GPTQ weights feed the block-scaled GEMM as they are; on held-out rows of the
    # calibration draw their weight error costs the output less than plain rounding's
    N, K, M = 256, 512, 64
    had = 16
    w = si.normal_bf16(41, N, K, std=0.02)
    xall = si.gptq_calibration(42, 2 * K + M, K)  # one draw: 2K rows build H, M held-out rows test
    u = torch.from_numpy(orc.gptq_hessian_factor(xall[:2 * K], had)).to(DEV)
    wq = fl.prepare_weight_gptq(w.to(DEV), u, "nvfp4", had)
    wr = fl.prepare_weight(w.to(DEV), "nvfp4", had)
    status_ok()
    x64 = xall[2 * K:]
    R = orc.hadamard_matrix(had).astype(np.float64) / np.sqrt(had)
    xr = (x64.reshape(M, K // had, had) @ R.T).reshape(M, K)
    w_rot = orc.fwht(w.float().numpy(), had).astype(np.float64)

    def weight_err(q):
        d = w_rot - orc.dequant(q.codes.cpu().numpy(), orc_sf(q), "nvfp4", float(q.g.item()))
        return np.linalg.norm(xr @ d.T)

    def orc_sf(q):  # tensor-core layout back to row-major [N, K/16]
        flat = q.scales.cpu().numpy()
        katoms = (K // 16 + 3) // 4
        out = np.empty((N, K // 16), dtype=np.uint8)
        for r in range(N):
            for c in range(K // 16):
                out[r, c] = flat[((r // 128) * katoms + c // 4) * 512 + (r % 32) * 16 + ((r % 128) // 32) * 4 + c % 4]
        return out

    assert weight_err(wq) < 0.8 * weight_err(wr)
    # and through the GEMM (activations quantised online, identical on both sides)
    x = torch.from_numpy(x64.astype(np.float32)).to(torch.bfloat16).to(DEV)
    ref = x.double() @ w.to(DEV).double().T
    e_gptq = (fl.nvfp4_linear(x, wq).double() - ref).norm()
    e_rtn = (fl.nvfp4_linear(x, wr).double() - ref).norm()
    status_ok()
    assert e_gptq < e_rtn, (float(e_gptq), float(e_rtn))


def _definition_hinv(x, b, damp=0.01):
    """H^-1 of the blockwise-rotated x in binary64, written out from the definition (scipy's
    Sylvester Hadamard matrix, an explicit inverse)."""
    import scipy.linalg
    x = np.asarray(x, np.float64)
    T, K = x.shape
    if b:
        x = x @ np.kron(np.eye(K // b), scipy.linalg.hadamard(b) / np.sqrt(b)).T
    return np.linalg.inv(x.T @ x + damp * np.mean(np.sum(x * x, axis=0)) * np.eye(K))


@pytest.mark.parametrize("K,T", [(64, 128), (256, 512), (320, 100), (1024, 2048 + 37)])
@pytest.mark.parametrize("had", [0, 16, 32])
def test_hessian_factor_matches_oracle(orc, K, T, had):
    # the library's binary64 preparation of U against the oracle's, to 1e-5 max|U|; T < K (a
    # rank-deficient Gram made definite by the damping) and a ragged T included; u is written
    # into a poisoned buffer with a row stride wider than K
    x = si.gptq_calibration(51 + K + had, T, K)
    u = torch.full((K, K + 8), float("nan"), dtype=torch.float32, device=DEV)
    got = fl.gptq_hessian_factor(torch.from_numpy(x).to(DEV), had, out=u[:, :K])
    status_ok()
    got = got.cpu().numpy()
    assert np.all(np.isnan(u[:, K:].cpu().numpy()))  # nothing written past the row
    ref = orc.gptq_hessian_factor(x, had)
    assert np.all(np.tril(got, -1) == 0) and np.all(np.diag(got) > 0)
    assert np.abs(got - ref).max() <= 1e-5 * np.abs(ref).max()
    hinv = _definition_hinv(x, had)
    g64 = got.astype(np.float64)
    assert np.abs(g64.T @ g64 - hinv).max() <= 1e-5 * np.abs(hinv).max()


@pytest.mark.slow
def test_hessian_factor_prefill_size(orc):
    # the size the bench prepares: K = 4096 with 8192 calibration tokens, H16
    K = si.PREFILL["K"]
    x = si.gptq_calibration(7, 2 * K, K)
    got = fl.gptq_hessian_factor(torch.from_numpy(x).to(DEV), 16).cpu().numpy()
    status_ok()
    ref = orc.gptq_hessian_factor(x, 16)
    assert np.abs(got - ref).max() <= 1e-5 * np.abs(ref).max()


def test_hessian_factor_reports_a_singular_hessian():
    # all-zero activations without damping: H = 0 has no Cholesky factor
    x = torch.zeros(128, 64, dtype=torch.float64, device=DEV)
    fl.gptq_hessian_factor(x, 16, damp=0.0)
    assert fl.device_status() == 9  # FP4LIN_ERR_NUMERIC
    assert fl.device_status() == 0


def test_hessian_factor_feeds_gptq_like_the_oracle_factor(orc):
    # the whole MR-GPTQ path through the library: the library's U is the oracle's to 1e-5 max|U|,
    # and GPTQ with it gives the oracle's GPTQ codes for that same U, byte for byte
    K, N = 128, 64
    x = si.gptq_calibration(61, 2 * K, K)
    w = si.normal_bf16(62, N, K, std=0.02)
    u_lib = fl.gptq_hessian_factor(torch.from_numpy(x).to(DEV), 16)
    u_orc = orc.gptq_hessian_factor(x, 16)
    c, s, g = fl.gptq_quantize(w.to(DEV), u_lib, "nvfp4", 16)
    status_ok()
    oc, osf, og = orc.gptq(w, u_lib.cpu().numpy(), "nvfp4", 16)
    assert_bytes_equal(c.cpu().numpy(), oc, "codes with the library's U")
    assert np.abs(u_lib.cpu().numpy() - u_orc).max() <= 1e-5 * np.abs(u_orc).max()


@pytest.mark.slow
@pytest.mark.parametrize("fmt,had", [("nvfp4", 16), ("mxfp4", 32)])
def test_gptq_prefill_weight_sampled_rows(orc, fmt, had):
    # the 14336 x 4096 prefill weight with a 4096-wide Hessian; rows are independent in the
    # sweep, so the oracle checks a sample of them
    N, K = si.PREFILL["N"], si.PREFILL["K"]
    w = si.prefill_W()
    u = orc.gptq_hessian_factor(si.gptq_calibration(7, 2 * K, K), had)
    c, s, g = _gpu(w, u, fmt, had)
    G = 16 if fmt == "nvfp4" else 32
    rows = [0, 1, 127, 128, 4097, 9000, N - 1]
    oc, osf, og = orc.gptq(w[rows], u, fmt, had, g if fmt == "nvfp4" else None)
    if fmt == "nvfp4":
        assert g == orc.nvfp4_tensor_scale(w, had)
    assert_bytes_equal(c[rows], oc, "codes")
    katoms = (K // G + 3) // 4
    for i, r in enumerate(rows):
        for col in range(K // G):
            off = ((r // 128) * katoms + col // 4) * 512 + (r % 32) * 16 + ((r % 128) // 32) * 4 + col % 4
            assert s[off] == osf[i, col], (r, col)
