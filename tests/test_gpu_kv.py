"""GPU parity of the NVFP4 KV cache (store of new K/V rows, dequantisation to FP8)
against the oracle, bit for bit."""
import os
from concurrent.futures import ThreadPoolExecutor

import numpy as np
import pytest
import torch

import mxfp4_microscaled_bit_b200 as fl
import synthetic_inputs as si
from gpu_util import DEV, assert_bytes_equal, status_ok

pytestmark = pytest.mark.gpu


def _g_of(x_cpu):
    return np.float32(np.abs(x_cpu.float().numpy()).max()) / np.float32(2688.0)


def test_kv_small_store_and_load(orc):
    B, H, Lcap, D = 3, 2, 48, 128
    rng = np.random.default_rng(4)
    prefill = si.to_bf16(rng.standard_normal((B, H, 30, D)).astype(np.float32) * 2)
    step = si.to_bf16(rng.standard_normal((B, H, 1, D)).astype(np.float32) * 5)  # exceeds the static scale
    g = _g_of(prefill)
    gt = torch.tensor([g], dtype=torch.float32, device=DEV)
    codes = torch.zeros(B, H, Lcap, D // 2, dtype=torch.uint8, device=DEV)
    scales = torch.zeros(B, H, Lcap, D // 16, dtype=torch.uint8, device=DEV)
    oc = np.zeros((B, H, Lcap, D // 2), np.uint8)
    osf = np.zeros((B, H, Lcap, D // 16), np.uint8)
    pos0 = np.zeros(B, np.int32)
    fl.kv_nvfp4_store(prefill.to(DEV), torch.from_numpy(pos0).to(DEV), gt, codes, scales)
    orc.kv_store(prefill, pos0, g, oc, osf)
    pos1 = np.array([30, 35, 47], np.int32)  # sequences at different lengths, one at the last slot
    fl.kv_nvfp4_store(step.to(DEV), torch.from_numpy(pos1).to(DEV), gt, codes, scales)
    orc.kv_store(step, pos1, g, oc, osf)
    status_ok()
    assert_bytes_equal(codes.cpu().numpy(), oc, "cache codes")
    assert_bytes_equal(scales.cpu().numpy(), osf, "cache scales")
    for L in (1, 31, 48):
        out = torch.full((B, H, L, D), 0x7F, dtype=torch.uint8, device=DEV)
        o, osc = fl.kv_nvfp4_load_fp8(codes, scales, gt, L, out=out)
        status_ok()
        assert_bytes_equal(o.cpu().numpy(), orc.kv_load_fp8(oc, osf, L), f"fp8 L={L}")
        assert osc.item() == np.float32(8.0) * g


def test_kv_out_of_range_position_is_reported():
    B, H, Lcap, D = 2, 1, 8, 32
    x = torch.ones(B, H, 1, D, dtype=torch.bfloat16, device=DEV)
    codes = torch.zeros(B, H, Lcap, D // 2, dtype=torch.uint8, device=DEV)
    scales = torch.zeros(B, H, Lcap, D // 16, dtype=torch.uint8, device=DEV)
    pos = torch.tensor([3, 8], dtype=torch.int32, device=DEV)  # 8 == Lcap: outside the cache
    g = torch.tensor([1.0], dtype=torch.float32, device=DEV)
    fl.kv_nvfp4_store(x, pos, g, codes, scales)
    assert fl.device_status() == 8  # FP4LIN_ERR_OUT_OF_RANGE, nothing written for batch 1
    assert fl.device_status() == 0  # cleared by the read
    assert codes[0, 0, 3].any() and not codes[1].any()


def _oracle_fp8_table(orc):
    """The oracle's FP8 byte for every (scale byte, code nibble) pair: a one-block-per-row cache
    whose row s has scale byte s and the 16 codes 0..15, dequantised by oracle.kv_load_fp8.
    The dequantisation is a function of that pair alone, so T[sf, code] is the oracle's answer
    for any cache element."""
    codes = np.tile(np.array([0x10, 0x32, 0x54, 0x76, 0x98, 0xBA, 0xDC, 0xFE], np.uint8), (256, 1))
    sf = np.arange(256, dtype=np.uint8).reshape(256, 1)
    return orc.kv_load_fp8(codes.reshape(1, 1, 256, 8), sf.reshape(1, 1, 256, 1), 256)[0, 0]


def _fp8_by_table(table, codes, sf):
    """FP8 bytes [L, D] of one cache slice (codes [L, D/2], scales [L, D/16]) through the table."""
    nib = np.empty((codes.shape[0], codes.shape[1] * 2), np.uint8)
    nib[:, 0::2] = codes & 0x0F
    nib[:, 1::2] = codes >> 4
    return table[np.repeat(sf, 16, axis=1), nib]


@pytest.mark.slow
def test_kv_full_cache_every_byte(orc):
    """The full cache workload (64 x 8 x 32768 x 128): prefill 32767 tokens, append one per
    sequence, dequantise all 32768 into an output pre-filled with 0x7F (an E4M3 NaN, which a
    valid output byte never is).  Every (b, h) slice is checked against the oracle byte for
    byte: the cache's codes and scales against oracle.kv_store of that slice, and every FP8
    byte against the oracle's dequantisation of that element (oracle.kv_load_fp8 tabulated
    over all scale-byte / code pairs; the table path is first shown equal to the direct
    oracle call on one whole slice)."""
    B, H, L, D = si.KVCACHE["B"], si.KVCACHE["H"], si.KVCACHE["L"], si.KVCACHE["D"]
    which = "k"
    host = torch.empty(B, H, L, D, dtype=torch.bfloat16).pin_memory()
    for b in range(B):
        for h in range(H):
            host[b, h] = si.to_bf16(si.kv_slice(which, b, h))
    g = np.float32(host.float().abs().max().item()) / np.float32(2688.0)
    gt = torch.tensor([g], dtype=torch.float32, device=DEV)
    codes = torch.full((B, H, L, D // 2), 0xAA, dtype=torch.uint8, device=DEV)
    scales = torch.full((B, H, L, D // 16), 0xFF, dtype=torch.uint8, device=DEV)
    dev_x = host.to(DEV, non_blocking=True)
    fl.kv_nvfp4_store(dev_x[:, :, :L - 1].contiguous(), torch.zeros(B, dtype=torch.int32, device=DEV), gt,
                      codes, scales)
    fl.kv_nvfp4_store(dev_x[:, :, L - 1:].contiguous(), torch.full((B,), L - 1, dtype=torch.int32, device=DEV), gt,
                      codes, scales)
    del dev_x
    out = torch.full((B, H, L, D), 0x7F, dtype=torch.uint8, device=DEV)
    fl.kv_nvfp4_load_fp8(codes, scales, gt, L, out=out)
    status_ok()
    assert not bool(((out == 0x7F) | (out == 0xFF)).any()), "an output byte was not written"

    table = _oracle_fp8_table(orc)

    def oracle_slice(b, h):
        oc = np.zeros((1, 1, L, D // 2), np.uint8)
        osf = np.zeros((1, 1, L, D // 16), np.uint8)
        orc.kv_store(host[b:b + 1, h:h + 1], np.zeros(1, np.int32), g, oc, osf)
        return oc[0, 0], osf[0, 0]

    oc, osf = oracle_slice(0, 0)
    direct = orc.kv_load_fp8(oc.reshape(1, 1, L, D // 2), osf.reshape(1, 1, L, D // 16), L)[0, 0]
    assert np.array_equal(_fp8_by_table(table, oc, osf), direct)

    def check(b, h, c, s, o):
        oc, osf = oracle_slice(b, h)
        bad = []
        if not np.array_equal(c, oc):
            bad.append(f"codes ({b},{h}): {int((c != oc).sum())} bytes differ")
        if not np.array_equal(s, osf):
            bad.append(f"scales ({b},{h}): {int((s != osf).sum())} bytes differ")
        ref = _fp8_by_table(table, oc, osf)
        if not np.array_equal(o, ref):
            bad.append(f"fp8 ({b},{h}): {int((o != ref).sum())} bytes differ")
        return bad

    problems = []
    with ThreadPoolExecutor(max_workers=max(1, os.cpu_count() or 1)) as ex:
        for b in range(B):
            cb, sb, ob = codes[b].cpu().numpy(), scales[b].cpu().numpy(), out[b].cpu().numpy()
            for f in [ex.submit(check, b, h, cb[h], sb[h], ob[h]) for h in range(H)]:
                problems += f.result()
    assert not problems, problems[:8]


@pytest.mark.parametrize("D,Lcap,L", [(16, 37, 37), (48, 21, 20), (128, 9, 5)])
def test_kv_odd_slice_alignment(orc, D, Lcap, L):
    # slices whose base is not 16-byte aligned (Lcap * D/16 odd) and odd block counts take the
    # narrow-load path; both must match the oracle byte for byte
    B, H = 2, 3
    rng = np.random.default_rng(D + Lcap)
    x = si.to_bf16(rng.standard_normal((B, H, Lcap, D)).astype(np.float32))
    g = _g_of(x)
    gt = torch.tensor([g], dtype=torch.float32, device=DEV)
    codes = torch.zeros(B, H, Lcap, D // 2, dtype=torch.uint8, device=DEV)
    scales = torch.zeros(B, H, Lcap, D // 16, dtype=torch.uint8, device=DEV)
    fl.kv_nvfp4_store(x.to(DEV), torch.zeros(B, dtype=torch.int32, device=DEV), gt, codes, scales)
    oc = np.zeros((B, H, Lcap, D // 2), np.uint8)
    osf = np.zeros((B, H, Lcap, D // 16), np.uint8)
    orc.kv_store(x, np.zeros(B, np.int32), g, oc, osf)
    out, _ = fl.kv_nvfp4_load_fp8(codes, scales, gt, L)
    status_ok()
    assert_bytes_equal(out.cpu().numpy(), orc.kv_load_fp8(oc, osf, L), "fp8")
