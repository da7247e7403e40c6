"""Pins of the oracle's quantisers, scale layout, GEMM reference and KV path against
hand-worked fixtures, library conversions, closed forms, invariants and brute force.
CPU only."""
import ml_dtypes
import numpy as np
import pytest
import torch

import synthetic_inputs as si
from conftest import golden

E2M1_MAG = np.array([0, 0.5, 1, 1.5, 2, 3, 4, 6], dtype=np.float64)


def _bf16(x):
    return si.to_bf16(np.asarray(x, dtype=np.float32))


def _unpack(codes):
    codes = np.asarray(codes, dtype=np.uint8)
    out = np.empty(codes.shape[:-1] + (codes.shape[-1] * 2,), dtype=np.uint8)
    out[..., 0::2] = codes & 15
    out[..., 1::2] = codes >> 4
    return out


# ------------------------------------------------------------------ hand-worked fixtures
@pytest.mark.parametrize("case", golden("nvfp4_worked.json")["cases"], ids=lambda c: c["name"])
def test_nvfp4_worked_blocks(orc, case):
    x = _bf16([case["x"]])
    assert np.array_equal(x.float().numpy()[0], np.float32(case["x"]))  # inputs exact in bf16
    codes, sf, g = orc.nvfp4_quantize(x, hadamard=case["hadamard"], g=case["g"])
    assert list(sf[0]) == case["sf"]
    assert list(codes[0]) == case["codes"]


@pytest.mark.parametrize("case", golden("nvfp4_worked.json")["tensor_cases"], ids=lambda c: c["name"])
def test_nvfp4_worked_tensor_scale(orc, case):
    x = _bf16([case["x"]])
    codes, sf, g = orc.nvfp4_quantize(x, hadamard=case["hadamard"])
    assert g == np.float32(case["g"])
    assert list(sf[0]) == case["sf"] and list(codes[0]) == case["codes"]


@pytest.mark.parametrize("case", golden("mxfp4_worked.json")["cases"], ids=lambda c: c["name"])
def test_mxfp4_worked_blocks(orc, case):
    row = np.zeros(32, dtype=np.float32)
    row[:len(case["x_head"])] = case["x_head"]
    x = _bf16([row])
    assert np.array_equal(x.float().numpy()[0], row)
    codes, sf = orc.mxfp4_quantize(x, hadamard=case["hadamard"])
    assert int(sf[0, 0]) == case["sf"]
    head = case["codes_head"]
    assert list(codes[0, :len(head)]) == head
    assert not codes[0, len(head):].any()


def test_mxfp4_subnormal_block(orc):
    # amax below 2^-126: X = floor(log2 amax) - 2 is far below -127, so the byte clamps to 0
    row = np.zeros(32, dtype=np.float32)
    row[0] = 1e-39
    codes, sf = orc.mxfp4_quantize(_bf16([row]))
    assert sf[0, 0] == 0 and not codes.any()


# ------------------------------------------------------------------ NVFP4 properties
def _representable_nvfp4(rng, rows, cols, g_exp):
    """x = e2m1(c) * dec(sf) * g exactly, g a power of two, each block holding a +-6."""
    nb = cols // 16
    c = rng.integers(0, 16, size=(rows, cols)).astype(np.uint8)
    c[:, ::16] = np.where(rng.random((rows, nb)) < 0.5, 7, 15)  # one +-6 per block
    sf = rng.integers(0x08, 0x7F, size=(rows, nb)).astype(np.uint8)  # normal E4M3 scales
    mag = E2M1_MAG[c & 7] * np.where(c & 8, -1.0, 1.0)
    dec_sf = torch.from_numpy(sf).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    x = mag * np.repeat(dec_sf, 16, axis=1) * 2.0 ** g_exp
    return x.astype(np.float32), c, sf


@pytest.mark.parametrize("g_exp", [0, -7, 5])
def test_nvfp4_idempotent_on_representable(orc, g_exp):
    rng = np.random.default_rng(20 + g_exp)
    x, c, sf = _representable_nvfp4(rng, 8, 256, g_exp)
    xb = _bf16(x)
    assert np.array_equal(xb.float().numpy(), x)  # 2 + 4 significant bits fit in bf16
    codes, sf2, _ = orc.nvfp4_quantize(xb, g=2.0 ** g_exp)
    assert np.array_equal(sf2, sf)
    # -0 elements carry code 8 on input; the quantiser maps x=-0 back to code 8 as well
    assert np.array_equal(_unpack(codes), c)


def test_nvfp4_codes_are_nearest_grid_points(orc):
    # brute force: every element's code is a nearest E2M1 point of v = x * r (ties excluded), and
    # the block's largest element lands on 6 whenever its scale is a normal E4M3 value
    x = si.student_t_bf16(31, 64, 512)
    codes, sf, g = orc.nvfp4_quantize(x, hadamard=16)
    xr = orc.fwht(x.float().numpy(), 16).reshape(64, 32, 16).astype(np.float64)
    d = torch.from_numpy(sf).view(torch.float8_e4m3fn).to(torch.float64).numpy()[..., None] * float(g)
    v = xr / d
    mag = E2M1_MAG[_unpack(codes).reshape(64, 32, 16) & 7]
    dist = np.abs(np.abs(v)[..., None] - E2M1_MAG).min(axis=-1)
    chosen = np.abs(np.minimum(np.abs(v), 6.0) - mag)
    assert np.all(chosen <= dist + 1e-6 * np.abs(v) + 1e-12)
    normal = sf >= 0x08
    top = mag.max(axis=-1)
    assert np.all(top[normal] == 6.0)


def test_nvfp4_tensor_scale_closed_form(orc):
    x = si.student_t_bf16(32, 40, 256)
    amax = np.abs(x.float().numpy()).max()
    assert orc.nvfp4_tensor_scale(x) == np.float32(amax) / np.float32(2688.0)
    xr = orc.fwht(x.float().numpy(), 16)
    assert orc.nvfp4_tensor_scale(x, 16) == np.float32(np.abs(xr).max()) / np.float32(2688.0)
    assert orc.nvfp4_tensor_scale(torch.zeros(4, 32, dtype=torch.bfloat16)) == 1.0


def test_nvfp4_block_error_bound(orc):
    # |x - dequant(x)| <= half the local grid spacing * d, plus the clip above 6*d
    x = si.normal_bf16(33, 32, 1024, std=3.0)
    codes, sf, g = orc.nvfp4_quantize(x)
    xd = orc.dequant(codes, sf, "nvfp4", g)
    xf = x.float().numpy().astype(np.float64)
    d = np.repeat(torch.from_numpy(sf).view(torch.float8_e4m3fn).to(torch.float64).numpy(), 16, axis=1) * float(g)
    v = np.abs(xf) / d
    half_gap = np.select([v < 2, v < 4], [0.25, 0.5], 1.0)
    err = np.abs(xf - xd)
    assert np.all(err <= half_gap * d * (1 + 1e-6) + np.maximum(np.abs(xf) - 6 * d, 0))


# ------------------------------------------------------------------ MXFP4 properties
def test_mxfp4_scale_exponent_closed_form(orc):
    x = si.student_t_bf16(34, 32, 1024)
    codes, sf = orc.mxfp4_quantize(x)
    amax = np.abs(x.float().numpy().astype(np.float64)).reshape(32, 32, 32).max(axis=-1)
    X = np.floor(np.log2(amax)) - 2
    assert np.array_equal(sf.astype(np.int64), (X + 127).astype(np.int64))
    # every element: |x| * 2^-X is within half a grid gap of its code, or clipped at 6
    v = np.abs(x.float().numpy().astype(np.float64)).reshape(32, 32, 32) * 2.0 ** -X[..., None]
    mag = E2M1_MAG[_unpack(codes).reshape(32, 32, 32) & 7]
    half_gap = np.select([v < 2, v < 4], [0.25, 0.5], 1.0)
    assert np.all(np.abs(np.minimum(v, 6) - mag) <= half_gap)


def test_mxfp4_error_larger_than_nvfp4(orc):
    # NVFP4's finer blocks and fractional scales fit better than MXFP4's power-of-two 32-blocks
    # (page "FP8, NVFP4 czy AWQ?", section "Czym roznia sie FP8, NVFP4, MXFP4 i AWQ?")
    x = si.student_t_bf16(35, 64, 1024)
    xf = x.float().numpy().astype(np.float64)
    c1, s1, g = orc.nvfp4_quantize(x)
    c2, s2 = orc.mxfp4_quantize(x)
    e_nv = np.linalg.norm(orc.dequant(c1, s1, "nvfp4", g) - xf)
    e_mx = np.linalg.norm(orc.dequant(c2, s2, "mxfp4") - xf)
    assert e_nv < e_mx


# ------------------------------------------------------------------ scale layout
def test_scale_layout_hand_positions(orc):
    gl = golden("scale_layout_positions.json")
    rows, sfc = gl["rows"], gl["sf_cols"]
    for r, c, off in gl["positions"]:
        lin = np.zeros((rows, sfc), dtype=np.uint8)
        lin[r, c] = 1
        out = orc.tc_scale_layout(lin)
        assert list(np.nonzero(out)[0]) == [off], (r, c)


@pytest.mark.parametrize("rows,sfc", [(128, 4), (200, 8), (1, 2), (257, 10), (16, 8)])
def test_scale_layout_is_a_bijection(orc, rows, sfc):
    lin = (np.arange(rows * sfc, dtype=np.int64) % 251 + 1).astype(np.uint8).reshape(rows, sfc)
    out = orc.tc_scale_layout(lin)
    rp, cp = -(-rows // 128) * 128, -(-sfc // 4) * 4
    assert out.size == rp * cp == orc.tc_scale_bytes(rows, sfc)
    # independent construction: pad, then view as [row tile, col atom, r%32, (r%128)/32, c%4]
    pad = np.zeros((rp, cp), dtype=np.uint8)
    pad[:rows, :sfc] = lin
    ref = pad.reshape(rp // 128, 4, 32, cp // 4, 4).transpose(0, 3, 2, 1, 4).reshape(-1)
    assert np.array_equal(out, ref)


# ------------------------------------------------------------------ GEMM reference
def test_gemm_abt_matches_numpy(orc):
    rng = np.random.default_rng(40)
    A, W = rng.standard_normal((17, 96)), rng.standard_normal((23, 96))
    y, s = orc.gemm_abt(A, W)
    assert np.allclose(y, A @ W.T, rtol=0, atol=1e-12 * s.max())
    assert np.allclose(s, np.abs(A) @ np.abs(W).T, rtol=1e-13)


def test_dequant_unit_scales_is_the_code_table(orc):
    rng = np.random.default_rng(41)
    codes = rng.integers(0, 256, size=(5, 32)).astype(np.uint8)
    sf = np.full((5, 4), 0x38, dtype=np.uint8)  # E4M3 1.0
    ref = _unpack(codes).view(ml_dtypes.float4_e2m1fn).astype(np.float64)
    assert np.array_equal(orc.dequant(codes, sf, "nvfp4", 1.0), ref)
    sf8 = np.full((5, 2), 127, dtype=np.uint8)  # E8M0 1.0
    assert np.array_equal(orc.dequant(codes, sf8, "mxfp4"), ref)


def test_gemm_exact_on_unit_scales(orc):
    # products of E2M1 values are multiples of 1/4, so with unit scales the sum is exact
    rng = np.random.default_rng(42)
    ca = rng.integers(0, 256, size=(9, 64)).astype(np.uint8)
    cw = rng.integers(0, 256, size=(11, 64)).astype(np.uint8)
    one = lambda r: np.full((r, 8), 0x38, dtype=np.uint8)
    A = orc.dequant(ca, one(9), "nvfp4", 1.0)
    W = orc.dequant(cw, one(11), "nvfp4", 1.0)
    y, _ = orc.gemm_abt(A, W)
    ia = (_unpack(ca).view(ml_dtypes.float4_e2m1fn).astype(np.float64) * 2).astype(np.int64)
    iw = (_unpack(cw).view(ml_dtypes.float4_e2m1fn).astype(np.float64) * 2).astype(np.int64)
    assert np.array_equal(y * 4, (ia @ iw.T).astype(np.float64))


def test_gemm_one_hot_rows_select_weight_rows(orc):
    rng = np.random.default_rng(43)
    cw = rng.integers(0, 256, size=(6, 16)).astype(np.uint8)  # 32 values per row
    sw = rng.integers(0x20, 0x50, size=(6, 2)).astype(np.uint8)
    W = orc.dequant(cw, sw, "nvfp4", 0.5)
    A = np.zeros((32, 32))
    A[np.arange(32), np.arange(32)] = 1.0
    y, _ = orc.gemm_abt(A, W)
    assert np.array_equal(y, W.T)


# ------------------------------------------------------------------ KV cache
def test_kv_store_then_load_composition(orc):
    B, H, Lcap, D, T = 2, 3, 12, 128, 2
    rng = np.random.default_rng(44)
    kv = si.to_bf16(rng.standard_normal((B, H, T, D)).astype(np.float32) * 3.0)
    g = np.float32(np.abs(kv.float().numpy()).max()) / np.float32(2688.0)
    codes = np.zeros((B, H, Lcap, D // 2), dtype=np.uint8)
    sfs = np.zeros((B, H, Lcap, D // 16), dtype=np.uint8)
    pos = np.array([3, 9], dtype=np.int32)
    orc.kv_store(kv, pos, g, codes, sfs)
    for b in range(B):
        for h in range(H):
            c, s, _ = orc.nvfp4_quantize(kv[b, h], g=g)
            assert np.array_equal(codes[b, h, pos[b]:pos[b] + T], c)
            assert np.array_equal(sfs[b, h, pos[b]:pos[b] + T], s)
            untouched = np.ones(Lcap, bool)
            untouched[pos[b]:pos[b] + T] = False
            assert not codes[b, h, untouched].any() and not sfs[b, h, untouched].any()
    out = orc.kv_load_fp8(codes, sfs, Lcap)
    # library pin of the FP8 step: e2m1 * dec(sf) / 8 is exact in fp64 and below 448, so torch's
    # round-to-nearest-even E4M3 cast is the whole step
    e2 = _unpack(codes).view(ml_dtypes.float4_e2m1fn).astype(np.float64)
    dsf = np.repeat(torch.from_numpy(sfs).view(torch.float8_e4m3fn).to(torch.float64).numpy(), 16, axis=-1)
    ref = torch.from_numpy((e2 * dsf / 8).astype(np.float32)).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(out, ref)


def test_kv_bytes_ratio():
    # NVFP4 KV: 0.5 B codes + 1/16 B scale per value against 1 B for FP8 (the KV-cache story's memory claim)
    assert (0.5 + 1 / 16) / 1.0 == 0.5625
