"""GPTQ's input on the CPU: the oracle's upper factor U of the inverse damped Hessian of the
rotated calibration activations, H^-1 = U^T U, checked against the definition, with the
rotation built from scipy's Sylvester Hadamard matrix.  (The library computes the same factor
on the GPU: tests/test_gpu_gptq.py compares it with this oracle.)"""
import numpy as np
import pytest
import scipy.linalg
import synthetic_inputs as si


def definition(x, b, damp=0.01):
    """H^-1 of the blockwise-rotated x, in binary64, written out from the definition."""
    x = np.asarray(x, np.float64)
    T, K = x.shape
    if b:
        R = np.kron(np.eye(K // b), scipy.linalg.hadamard(b) / np.sqrt(b))  # block-diagonal rotation
        x = x @ R.T
    H = x.T @ x + damp * np.mean(np.sum(x * x, axis=0)) * np.eye(K)
    return np.linalg.inv(H)


@pytest.mark.parametrize("b", [0, 16, 32])
def test_factor_reproduces_the_inverse_hessian(orc, b):
    K = 128
    x = si.gptq_calibration(3, 2 * K, K)
    hinv = definition(x, b)
    scale = np.abs(hinv).max()
    for u in (orc.gptq_hessian_factor(x, b),):
        assert u.dtype == np.float32 and u.shape == (K, K)
        assert np.all(np.tril(u, -1) == 0)  # upper triangular
        assert np.all(np.diag(u) > 0)
        uu = u.astype(np.float64)
        assert np.abs(uu.T @ uu - hinv).max() <= 1e-5 * scale
