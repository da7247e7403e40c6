"""Decode attention straight from the NVFP4 KV cache (kv_nvfp4_attention) against the oracle's
attention over the FP8 values (reading R11).  Tolerance, from the arithmetic: scores are binary32
dot products of 128 terms, the chunk sums run over at most 256 positions and the merge over the
chunks (at most 128 of them here), so the error is at most ~(128 + 256 + 128) * 2^-24 = 3.1e-5
of the largest |v| of the head; the check allows 1e-4 of it."""
import ml_dtypes
import numpy as np
import pytest
import torch

import mxfp4_microscaled_bit_b200 as fl
import synthetic_inputs as si
from gpu_util import DEV, status_ok

pytestmark = pytest.mark.gpu

TOL = 1e-4


def _store(x, Lcap):
    """x: bf16 [B, H, L, D] on the GPU -> (codes, scales, g) with the static g = amax / 2688."""
    B, H, L, D = x.shape
    g = torch.tensor([float(x.abs().max().float()) / 2688.0], dtype=torch.float32, device=DEV)
    codes = torch.zeros(B, H, Lcap, D // 2, dtype=torch.uint8, device=DEV)
    scales = torch.zeros(B, H, Lcap, D // 16, dtype=torch.uint8, device=DEV)
    fl.kv_nvfp4_store(x, torch.zeros(B, dtype=torch.int32, device=DEV), g, codes, scales)
    status_ok()
    return codes, scales, g


def _check(orc, q, kcache, vcache, L, bh=None):
    out = fl.kv_nvfp4_attention(q, kcache, vcache, L)
    status_ok()
    kc, ks, gk = (t.cpu() for t in kcache)
    vc, vs, gv = (t.cpu() for t in vcache)
    B, H = kc.shape[:2]
    G = q.shape[1] // H
    pairs = [(b, h) for b in range(B) for h in range(H)] if bh is None else bh
    worst = 0.0
    for b, h in pairs:
        ref = orc.kv_attention(q[b:b + 1, h * G:(h + 1) * G].cpu(), kc[b:b + 1, h:h + 1].numpy(),
                               ks[b:b + 1, h:h + 1].numpy(), float(gk), vc[b:b + 1, h:h + 1].numpy(),
                               vs[b:b + 1, h:h + 1].numpy(), float(gv), L)[0]
        got = out[b, h * G:(h + 1) * G].double().cpu().numpy()
        fp8 = orc.kv_load_fp8(vc[b:b + 1, h:h + 1].numpy(), vs[b:b + 1, h:h + 1].numpy(), L)
        vmax = np.abs(fp8.view(ml_dtypes.float8_e4m3fn).astype(np.float64)).max() * 8.0 * float(gv)
        err = np.abs(got - ref).max()
        worst = max(worst, err / max(vmax, 1e-30))
        assert err <= TOL * vmax, (b, h, err, TOL * vmax)
    print(f"max |out - ref| / max|v| = {worst:.2e}")


def _kv(B, H, L, Lcap, seed):
    """K and V caches of the decode-step distribution (normal times one scale per kv head);
    batch index offset by seed so the cases draw different slices."""
    def tensor(which):
        return torch.stack([torch.stack([si.kv_slice_bf16(which, seed + b, h, 0, L) for h in range(H)])
                            for b in range(B)]).to(DEV)
    return _store(tensor("k"), Lcap), _store(tensor("v"), Lcap)


@pytest.mark.parametrize("B,H,G,L", [(2, 2, 4, 1), (2, 2, 4, 255), (1, 3, 4, 256), (2, 2, 4, 257), (2, 2, 4, 511),
                                     (1, 3, 4, 512), (2, 2, 4, 513),
                                     (1, 2, 1, 1000), (1, 2, 8, 1500), (2, 1, 3, 77)])
def test_attention_matches_oracle(orc, B, H, G, L):
    kcache, vcache = _kv(B, H, L, L + 5, 0)
    q = si.normal_bf16(31 + L, B * H * G, 128).reshape(B, H * G, 128).to(DEV)
    _check(orc, q, kcache, vcache, L)


def test_attention_full_capacity(orc):
    # L = Lcap, and a second call with a shorter L on the same caches
    B, H, G, L = 1, 2, 4, 1024
    kcache, vcache = _kv(B, H, L, L, 1)
    q = si.normal_bf16(32, B * H * G, 128).reshape(B, H * G, 128).to(DEV)
    _check(orc, q, kcache, vcache, L)
    _check(orc, q, kcache, vcache, 700)


def test_attention_argument_checks():
    kcache, vcache = _kv(1, 1, 16, 16, 2)
    q = torch.zeros(1, 4, 128, dtype=torch.bfloat16, device=DEV)
    with pytest.raises(fl.Fp4LinError):
        fl.kv_nvfp4_attention(q, kcache, vcache, 17)  # L > Lcap
    with pytest.raises(fl.Fp4LinError):
        fl.kv_nvfp4_attention(torch.zeros(1, 9, 128, dtype=torch.bfloat16, device=DEV), kcache, vcache, 16)  # G = 9


@pytest.mark.slow
def test_attention_full_cache_sampled(orc):
    # the 64 x 8 x 32768 x 128 cache of the decode step (device-generated normal data times one
    # scale per kv head), G = 4; (b, h) slices sampled for the oracle
    B, H, L, D, G = 64, 8, 32768, 128, 4
    gen = torch.Generator(device=DEV).manual_seed(4)
    scales = torch.from_numpy(si.kv_head_scales()).to(DEV)
    caches = []
    for t in range(2):
        x = (torch.randn(B, H, L, D, generator=gen, device=DEV) * scales[t][None, :, None, None]).to(torch.bfloat16)
        caches.append(_store(x, L))
        del x
    q = torch.randn(B, H * G, D, generator=gen, device=DEV).to(torch.bfloat16)
    _check(orc, q, caches[0], caches[1], L, bh=[(0, 0), (17, 3), (63, 7), (40, 5)])
