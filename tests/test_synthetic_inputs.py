"""The seeded input generators keep their stated recipe: the same draws every time, row blocks
and KV slices that regenerate alone and equal the corresponding part of the whole, the stated
outlier patterns, and the distributions' tell-tale statistics. The parity tests and the bench
rely on all of this (a sampled row of a full-size case is regenerated on its own)."""
import numpy as np
import torch

import synthetic_inputs as si


def test_draws_are_deterministic():
    a, b = si.tiny(), si.tiny()
    assert torch.equal(a["A"], b["A"]) and torch.equal(a["W"], b["W"])
    assert torch.equal(si.decode_A(16, 4096), si.decode_A(16, 4096))
    assert np.array_equal(si.gptq_calibration(7, 64, 128), si.gptq_calibration(7, 64, 128))
    assert not torch.equal(si.normal_bf16(1, 8, 64), si.normal_bf16(2, 8, 64))


def test_row_blocks_regenerate_alone():
    # a block that straddles the 256-row chunk boundary equals the same rows of a larger draw
    whole = si.prefill_W(0, 768)
    assert torch.equal(si.prefill_W(200, 600), whole[200:600])
    assert torch.equal(si.decode_W(4096, 4096, 250, 260), si.decode_W(4096, 4096, 0, 512)[250:260])
    k = si.kv_slice("k", 3, 5, 0, 1024, L=32768, D=128)
    assert np.array_equal(si.kv_slice("k", 3, 5, 500, 700, L=32768, D=128), k[500:700])


def test_decode_rows_nest_and_carry_the_outlier_channels():
    a16, a4 = si.decode_A(16, 4096), si.decode_A(4, 4096)
    assert torch.equal(a16[:4], a4)
    ch = si.decode_outlier_channels(4096)
    assert ch.size == round(0.005 * 4096) and np.unique(ch).size == ch.size
    x = a16.float().numpy()
    others = np.setdiff1d(np.arange(4096), ch)
    # the scaled channels carry ~30x the spread of the others
    assert 20 < np.abs(x[:, ch]).mean() / np.abs(x[:, others]).mean() < 45


def test_tiny_weight_outliers():
    w = si.tiny()["W"].float().numpy()
    assert w.shape == (64, 128)
    # N(0, 0.02^2) entries beyond 0.2 (10 sigma) exist only among the 82 entries times 20
    big = np.count_nonzero(np.abs(w) > 0.2)
    assert 40 < big <= 82


def test_distribution_statistics():
    a = si.prefill_A(0, 256).float().numpy().astype(np.float64)
    w = si.prefill_W(0, 256).float().numpy().astype(np.float64)
    # Student-t with 3 degrees of freedom: variance 3, heavy tails (far more mass beyond 10)
    assert 2.0 < a.var() < 4.5
    assert np.mean(np.abs(a) > 10) > 1e-3
    assert abs(w.std() - 0.02) < 0.001 and np.mean(np.abs(w) > 0.1) < 1e-5
    s = si.kv_head_scales()
    assert s.shape == (2, 8) and np.all((s >= 0.1) & (s <= 10))
    k = si.kv_slice("v", 0, 2, 0, 2048, L=32768, D=128)
    assert abs(k.std() / s[1, 2] - 1) < 0.02


def test_calibration_channels_are_correlated_with_outliers():
    x = si.gptq_calibration(5, 4096, 256)
    c = np.corrcoef(x, rowvar=False)
    off = np.abs(c[~np.eye(256, dtype=bool)])
    assert off.mean() > 0.05  # the rank-K/4 mix correlates channels
    sd = x.std(axis=0)
    assert np.count_nonzero(sd > 4 * np.median(sd)) == 256 // 64
