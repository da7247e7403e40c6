"""Pins of the oracle's MR-GPTQ (reading R12) to things other than itself:
- with U = I there is no error feedback, and GPTQ must reduce to the plain quantiser
  (the oracle's own RTN, itself pinned elsewhere);
- the classic optimal-brain-surgeon form of GPTQ, written here in numpy binary64 from H
  itself (inverse Hessian updated by eliminating each quantised column, no Cholesky
  factor), must pick the same codes and scales;
- the algebraic identity of the sweep: W' - Q = E U column by column (the error of every
  column is the sum of the corrections it received plus its own rounding), with a
  deliberately planted wrong index shown to break it;
- on correlated inputs GPTQ lowers the Hessian-weighted output error against plain rounding.
"""
import numpy as np
import pytest

import synthetic_inputs as si


def _rotated_f32(orc, w_bf16, b):
    """The oracle's fp32 rotation of every row (the same values the GPTQ sweep starts from)."""
    w = w_bf16.float().numpy().astype(np.float32)
    if not b:
        return w
    out = w.copy()
    for r in range(out.shape[0]):
        for k in range(0, out.shape[1], b):
            blk = np.ascontiguousarray(out[r, k:k + b])
            out[r, k:k + b] = orc.fwht(blk, b)
    return out


@pytest.mark.parametrize("fmt,had", [("nvfp4", 0), ("nvfp4", 16), ("mxfp4", 0), ("mxfp4", 32)])
def test_identity_hessian_is_plain_rounding(orc, fmt, had):
    N, K = 24, 128
    w = si.normal_bf16(3, N, K, std=0.02)
    u = np.eye(K, dtype=np.float32)
    codes, sf, g = orc.gptq(w, u, fmt, had)
    if fmt == "nvfp4":
        rc, rs, rg = orc.nvfp4_quantize(w, had, g)
    else:
        rc, rs = orc.mxfp4_quantize(w, had)
    assert np.array_equal(codes, rc) and np.array_equal(sf, rs)


def _quant_dequant_f32(orc, v, fmt, scale_state):
    """One value by the format's rule with its block scale fixed in scale_state (binary32
    steps; the scalar E2M1 conversions are the oracle's, pinned on their own)."""
    f32 = np.float32
    mul, back = scale_state
    c = int(orc.e2m1_encode(np.array([f32(v) * mul], dtype=np.float32))[0])
    return c, f32(orc.e2m1_decode(np.array([c], dtype=np.uint8))[0]) * back


def _scale(block, fmt, g, orc):
    f32 = np.float32
    amax = f32(np.max(np.abs(block)))
    if fmt == "nvfp4":
        s = int(orc.e4m3_encode(np.array([(amax / f32(6.0)) / g], dtype=np.float32))[0])
        d = f32(orc.e4m3_decode(np.array([s], dtype=np.uint8))[0]) * g
        return s, (f32(1.0) / d if d > 0 else f32(0.0), d)
    byte = 0
    if amax > 0:
        e = np.frexp(np.float64(amax))[1]
        byte = int(np.clip(e - 1 - 2 + 127, 0, 254))
    return byte, (np.ldexp(f32(1.0), 127 - byte).astype(np.float32), np.ldexp(f32(1.0), byte - 127).astype(np.float32))


def _gptq_obs(orc, w_rot, H, fmt, g):
    """GPTQ in its optimal-brain-surgeon form (binary64 updates from H^-1 itself)."""
    G = 16 if fmt == "nvfp4" else 32
    N, K = w_rot.shape
    W = w_rot.astype(np.float64).copy()
    Hinv = np.linalg.inv(H)
    codes = np.zeros((N, K), dtype=np.int64)
    sf = np.zeros((N, K // G), dtype=np.int64)
    state = [None] * N
    for j in range(K):
        for n in range(N):
            if j % G == 0:
                sf[n, j // G], state[n] = _scale(W[n, j:j + G].astype(np.float32), fmt, g, orc)
            c, q = _quant_dequant_f32(orc, np.float32(W[n, j]), fmt, state[n])
            codes[n, j] = c
            err = (W[n, j] - float(q)) / Hinv[j, j]
            W[n, j + 1:] -= err * Hinv[j, j + 1:]
        Hinv = Hinv - np.outer(Hinv[:, j], Hinv[j, :]) / Hinv[j, j]
    packed = (codes[:, 0::2] | (codes[:, 1::2] << 4)).astype(np.uint8)
    return packed, sf.astype(np.uint8)


@pytest.mark.parametrize("fmt,had", [("nvfp4", 0), ("nvfp4", 16), ("mxfp4", 32)])
def test_matches_optimal_brain_surgeon_form(orc, fmt, had):
    N, K = 5, 64
    w = si.normal_bf16(11, N, K, std=0.02)
    x = si.gptq_calibration(12, 4 * K, K)
    u = orc.gptq_hessian_factor(x, had)
    codes, sf, g = orc.gptq(w, u, fmt, had)
    # the same damped Hessian of the rotated inputs, in binary64, without the factor
    xr = x
    if had:
        R = orc.hadamard_matrix(had).astype(np.float64) / np.sqrt(had)
        xr = (x.reshape(x.shape[0], K // had, had) @ R.T).reshape(x.shape)
    H = xr.T @ xr
    H[np.diag_indices(K)] += 0.01 * np.mean(np.diag(H))
    oc, osf = _gptq_obs(orc, _rotated_f32(orc, w, had), H, fmt, np.float32(g) if g is not None else None)
    assert np.array_equal(osf, sf), "scales differ from the surgeon form"
    assert np.array_equal(oc, codes), "codes differ from the surgeon form"


def _sweep_identity_residual(orc, w_rot, codes, sf, g, fmt, err, u):
    """max | (W' - Q) - E U | over the upper-triangular product, relative to max |W'|."""
    G = 16 if fmt == "nvfp4" else 32
    Q = orc.dequant(codes, sf, fmt, g if g is not None else 1.0)
    lhs = w_rot.astype(np.float64) - Q
    rhs = err.astype(np.float64) @ np.triu(u.astype(np.float64))
    return np.abs(lhs - rhs).max() / np.abs(w_rot).max()


@pytest.mark.parametrize("fmt,had", [("nvfp4", 16), ("mxfp4", 0)])
def test_sweep_identity(orc, fmt, had):
    N, K = 16, 128
    w = si.normal_bf16(21, N, K, std=0.02)
    u = orc.gptq_hessian_factor(si.gptq_calibration(22, 3 * K, K), had)
    codes, sf, g, err = orc.gptq(w, u, fmt, had, want_err=True)
    w_rot = _rotated_f32(orc, w, had)
    res = _sweep_identity_residual(orc, w_rot, codes, sf, g, fmt, err, u)
    assert res < 1e-4, res
    # a planted mistake (the feedback read from the transposed factor) must break the identity
    bad, bsf, bg, berr = orc.gptq(w, np.ascontiguousarray(u.T), fmt, had, want_err=True)
    assert _sweep_identity_residual(orc, w_rot, bad, bsf, bg, fmt, berr, u) > 1e-2


@pytest.mark.parametrize("fmt,had", [("nvfp4", 16), ("mxfp4", 32), ("mxfp4", 0)])
def test_gptq_beats_rounding_on_correlated_inputs(orc, fmt, had):
    N, K = 64, 256
    w = si.normal_bf16(31, N, K, std=0.02)
    x = si.gptq_calibration(32, 4 * K, K)
    u = orc.gptq_hessian_factor(x, had)
    codes, sf, g = orc.gptq(w, u, fmt, had)
    if fmt == "nvfp4":
        rc, rs, _ = orc.nvfp4_quantize(w, had, g)
    else:
        rc, rs = orc.mxfp4_quantize(w, had)
    xr = x
    if had:
        R = orc.hadamard_matrix(had).astype(np.float64) / np.sqrt(had)
        xr = (x.reshape(x.shape[0], K // had, had) @ R.T).reshape(x.shape)
    w_rot = _rotated_f32(orc, w, had).astype(np.float64)
    gg = g if g is not None else 1.0

    def out_err(c, s):
        d = w_rot - orc.dequant(c, s, fmt, gg)
        return np.linalg.norm(xr @ d.T)

    e_gptq, e_rtn = out_err(codes, sf), out_err(rc, rs)
    assert e_gptq < 0.8 * e_rtn, (e_gptq, e_rtn)


# ---------------------------------------------------------------- the MSE-scale variant (R12 with R9)
@pytest.mark.parametrize("had", [0, 16])
def test_mse_variant_identity_hessian_is_the_mse_quantiser(orc, had):
    N, K = 16, 128
    w = si.normal_bf16(4, N, K, std=0.02)
    codes, sf, g = orc.gptq(w, np.eye(K, dtype=np.float32), "nvfp4", had, mse=True)
    rc, rs, _ = orc.nvfp4_quantize_mse(w, had, g)
    assert np.array_equal(codes, rc) and np.array_equal(sf, rs)


def test_mse_variant_sweep_identity(orc):
    N, K = 12, 128
    w = si.normal_bf16(23, N, K, std=0.02)
    u = orc.gptq_hessian_factor(si.gptq_calibration(24, 3 * K, K), 16)
    codes, sf, g, err = orc.gptq(w, u, "nvfp4", 16, want_err=True, mse=True)
    assert _sweep_identity_residual(orc, _rotated_f32(orc, w, 16), codes, sf, g, "nvfp4", err, u) < 1e-4


def test_mse_variant_lowers_output_error(orc):
    N, K = 64, 256
    w = si.normal_bf16(33, N, K, std=0.02)
    x = si.gptq_calibration(34, 4 * K, K)
    u = orc.gptq_hessian_factor(x, 16)
    R = orc.hadamard_matrix(16).astype(np.float64) / 4.0
    xr = (x.reshape(x.shape[0], K // 16, 16) @ R.T).reshape(x.shape)
    w_rot = _rotated_f32(orc, w, 16).astype(np.float64)

    def out_err(c, s, g):
        return np.linalg.norm(xr @ (w_rot - orc.dequant(c, s, "nvfp4", g)).T)

    c0, s0, g0 = orc.gptq(w, u, "nvfp4", 16)
    c1, s1, g1 = orc.gptq(w, u, "nvfp4", 16, mse=True)
    assert out_err(c1, s1, g1) < out_err(c0, s0, g0)
