"""Pins of the oracle's decode attention over the NVFP4 KV cache (reading R11): against
torch's scaled_dot_product_attention in float64 on the FP8 values the load path produces,
and closed forms (one position: the output is that value row; equal keys: the mean)."""
import ml_dtypes
import numpy as np
import pytest
import torch

import synthetic_inputs as si


def _cache(orc, B, H, L, D, seed, g):
    Lcap = L + 3
    codes = np.zeros((B, H, Lcap, D // 2), np.uint8)
    sf = np.zeros((B, H, Lcap, D // 16), np.uint8)
    x = si.normal_bf16(seed, B * H * L, D).reshape(B, H, L, D)
    orc.kv_store(x, np.zeros(B, np.int32), g, codes, sf)
    return codes, sf


def _fp8_values(orc, codes, sf, L, g):
    b = orc.kv_load_fp8(codes, sf, L)
    return b.view(ml_dtypes.float8_e4m3fn).astype(np.float64) * (8.0 * float(np.float32(g)))


@pytest.mark.parametrize("B,H,G,L", [(2, 2, 4, 37), (1, 3, 1, 200), (2, 1, 8, 64)])
def test_attention_matches_torch_sdpa(orc, B, H, G, L):
    D = 128
    gk, gv = np.float32(0.0031), np.float32(0.0017)
    kc, ks = _cache(orc, B, H, L, D, 5, gk)
    vc, vs = _cache(orc, B, H, L, D, 6, gv)
    q = si.normal_bf16(7, B * H * G, D).reshape(B, H * G, D)
    out = orc.kv_attention(q, kc, ks, gk, vc, vs, gv, L)
    k = torch.from_numpy(_fp8_values(orc, kc, ks, L, gk)).repeat_interleave(G, dim=1)
    v = torch.from_numpy(_fp8_values(orc, vc, vs, L, gv)).repeat_interleave(G, dim=1)
    ref = torch.nn.functional.scaled_dot_product_attention(q.double().unsqueeze(2), k, v).squeeze(2).numpy()
    np.testing.assert_allclose(out, ref, rtol=1e-11, atol=1e-13)


def test_attention_single_position_is_the_value_row(orc):
    B, H, G, L, D = 1, 2, 2, 1, 128
    kc, ks = _cache(orc, B, H, L, D, 8, 0.01)
    vc, vs = _cache(orc, B, H, L, D, 9, 0.02)
    q = si.normal_bf16(10, B * H * G, D).reshape(B, H * G, D)
    out = orc.kv_attention(q, kc, ks, 0.01, vc, vs, 0.02, L)
    v = _fp8_values(orc, vc, vs, L, 0.02)
    for h in range(H):
        for j in range(G):
            assert np.array_equal(out[0, h * G + j], v[0, h, 0])


def test_attention_equal_keys_average_the_values(orc):
    B, H, G, L, D = 1, 1, 3, 50, 128
    kc, ks = _cache(orc, B, H, L, D, 11, 0.01)
    kc[:, :, :L] = kc[:, :, :1]
    ks[:, :, :L] = ks[:, :, :1]
    vc, vs = _cache(orc, B, H, L, D, 12, 0.02)
    q = si.normal_bf16(13, B * H * G, D).reshape(B, H * G, D)
    out = orc.kv_attention(q, kc, ks, 0.01, vc, vs, 0.02, L)
    mean = _fp8_values(orc, vc, vs, L, 0.02)[0, 0].mean(axis=0)
    for j in range(G):
        np.testing.assert_allclose(out[0, j], mean, rtol=1e-13, atol=1e-15)
