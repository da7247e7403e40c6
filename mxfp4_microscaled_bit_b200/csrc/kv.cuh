// kv.cuh -- NVFP4 KV cache: quantise appended K/V rows into the cache, and
// dequantise the cache to FP8 E4M3 for attention.  Source: the NVFP4 KV-cache
// story (hyper.ai/de/stories/e1307393ec176dd2b0276468adeec3f9), a single
// untitled paragraph; the passage used is its statement that new K/V vectors
// are written to the cache in NVFP4 while the KV tensors are dequantised to
// FP8 before the attention computation.
#pragma once

#include "common.cuh"

namespace fp4lin {

constexpr int KV_THREADS = 256;

struct KvStoreShape {
    const __nv_bfloat16 *x;  // [B, H, T, D]
    const int32_t *pos;      // [B]
    const float *g;
    uint8_t *codes, *scales; // [B, H, Lcap, D/2], [B, H, Lcap, D/16]
    int B, H, T, D;
    int64_t Lcap;
    int64_t total_chunks;    // B*H*T*D/8
};

// One lane per 8 values, a lane pair per 16-value block (as the NVFP4
// quantiser, without rotation and with the static tensor scale).
__global__ void __launch_bounds__(KV_THREADS) kv_store_kernel(KvStoreShape s)
{
    const int lane = threadIdx.x & 31;
    const bool upper = lane & 1;
    const float g = *s.g;
    const int64_t cpr = s.D / 8;
    const int64_t stride = (int64_t)gridDim.x * KV_THREADS;
    for (int64_t w0 = (int64_t)blockIdx.x * KV_THREADS + (threadIdx.x & ~31); w0 < s.total_chunks; w0 += stride) {
        const int64_t i = w0 + lane;
        const bool valid = i < s.total_chunks;
        int64_t row = 0, c8 = 0;
        uint4 raw = make_uint4(0, 0, 0, 0);
        if (valid) {
            row = i / cpr;
            c8 = i - row * cpr;
            raw = ld_nc_v4(s.x + row * s.D + c8 * 8);
        }
        float v[8];
        bf16x8_to_f32(raw, v);
        float amax = 0.0f;
#pragma unroll
        for (int j = 0; j < 8; ++j)
            amax = fmaxf(amax, fabsf(v[j]));
        amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 1));
        float rcp;
        const uint32_t sf = nvfp4_block_scale(amax, g, rcp);
#pragma unroll
        for (int j = 0; j < 8; ++j)
            v[j] = __fmul_rn(v[j], rcp);
        const uint32_t packed = pack_e2m1x8(v);
        if (valid) {
            const int64_t t_idx = row % s.T, bh = row / s.T, b = bh / s.H;
            const int64_t p = (int64_t)s.pos[b] + t_idx;
            if (p < 0 || p >= s.Lcap) {
                if (c8 == 0)
                    report_error(FP4LIN_ERR_OUT_OF_RANGE);
                continue;
            }
            const int64_t dst = bh * s.Lcap + p;
            *reinterpret_cast<uint32_t *>(s.codes + dst * (s.D / 2) + c8 * 4) = packed;
            if (!upper)
                s.scales[dst * (s.D / 16) + (c8 >> 1)] = (uint8_t)sf;
        }
    }
}

struct KvLoadShape {
    const uint8_t *codes, *scales;
    const float *g;
    uint8_t *out;
    float *out_scale;
    int64_t L, Lcap, bpr;  // bpr: 16-value blocks per row (D/16)
};

// 16 FP8 bytes of one 16-value block: e2m1 * (dec(sf) / 8) is formed in
// f16x2, where both factors and the product are exact (at most 6 significant
// bits, magnitudes in [2^-13, 336]), so the E4M3 rounding of the f16 product
// is the single rounding.
__device__ __forceinline__ uint4 kv_block_fp8(uint2 c, uint32_t sf)
{
    const __half2 s2 = __float2half2_rn(__fmul_rn(e4m3_value(sf), 0.125f));
    const uint32_t s2u = *reinterpret_cast<const uint32_t *>(&s2);
    uint32_t out[4];
    const uint32_t cw[2] = {c.x, c.y};
#pragma unroll
    for (int w = 0; w < 2; ++w) {
        uint32_t h[4];
        asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\t"
            "mov.b32 {b0, b1, b2, b3}, %4;\n\t"
            "cvt.rn.f16x2.e2m1x2 %0, b0;\n\t"
            "cvt.rn.f16x2.e2m1x2 %1, b1;\n\t"
            "cvt.rn.f16x2.e2m1x2 %2, b2;\n\t"
            "cvt.rn.f16x2.e2m1x2 %3, b3;\n\t}"
            : "=r"(h[0]), "=r"(h[1]), "=r"(h[2]), "=r"(h[3]) : "r"(cw[w]));
        uint16_t q[4];
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            uint32_t p;
            asm("mul.rn.f16x2 %0, %1, %2;" : "=r"(p) : "r"(h[k]), "r"(s2u));
            asm("cvt.rn.satfinite.e4m3x2.f16x2 %0, %1;" : "=h"(q[k]) : "r"(p));
        }
        out[2 * w] = (uint32_t)q[0] | ((uint32_t)q[1] << 16);
        out[2 * w + 1] = (uint32_t)q[2] | ((uint32_t)q[3] << 16);
    }
    return make_uint4(out[0], out[1], out[2], out[3]);
}

// Wide path: a thread takes 8 consecutive blocks -- 64 code bytes (two 256-bit
// loads), 8 scale bytes (one 64-bit load), 128 FP8 bytes out (four 256-bit
// stores) -- and keeps KV_WIDE_INFLIGHT such groups in flight.  Taken when the
// slice's block count and every base are aligned for it (see kv_load_fp8_wide_ok).
// Four groups (120 registers, two CTAs per SM) keep more loads in flight per SM
// than two (73 registers, three CTAs) or one (32 registers, eight CTAs).
constexpr int KV_WIDE_INFLIGHT = 4;
__device__ __forceinline__ void kv_load_group8(const uint8_t *codes, const uint8_t *scales, uint8_t *out, int64_t grp,
                                               uint32_t *c, uint2 &sf)
{
    ld_nc_v8(codes + grp * 64, c);
    ld_nc_v8(codes + grp * 64 + 32, c + 8);
    sf = ld_nc_v2(scales + grp * 8);
    (void)out;
}

__global__ void __launch_bounds__(KV_THREADS) kv_load_fp8_wide_kernel(KvLoadShape s)
{
    if (blockIdx.x == 0 && blockIdx.y == 0 && threadIdx.x == 0)
        *s.out_scale = __fmul_rn(8.0f, *s.g);
    const int64_t bh = blockIdx.y;
    const int64_t nblk = s.L * s.bpr, ngrp = nblk / 8;
    const uint8_t *codes = s.codes + bh * s.Lcap * s.bpr * 8;
    const uint8_t *scales = s.scales + bh * s.Lcap * s.bpr;
    uint8_t *out = s.out + bh * nblk * 16;
    const int64_t stride = (int64_t)gridDim.x * KV_THREADS;
    for (int64_t g0 = (int64_t)blockIdx.x * KV_THREADS + threadIdx.x; g0 < ngrp; g0 += KV_WIDE_INFLIGHT * stride) {
        uint32_t c[KV_WIDE_INFLIGHT][16];
        uint2 sf[KV_WIDE_INFLIGHT];
#pragma unroll
        for (int u = 0; u < KV_WIDE_INFLIGHT; ++u) {
            const int64_t grp = g0 + u * stride;
            if (grp < ngrp)
                kv_load_group8(codes, scales, out, grp, c[u], sf[u]);
        }
#pragma unroll
        for (int u = 0; u < KV_WIDE_INFLIGHT; ++u) {
            const int64_t grp = g0 + u * stride;
            if (grp >= ngrp)
                continue;
            const uint32_t sw[2] = {sf[u].x, sf[u].y};
#pragma unroll
            for (int h = 0; h < 4; ++h) {  // two blocks per 256-bit store
                uint32_t o[8];
#pragma unroll
                for (int b = 0; b < 2; ++b) {
                    const int blk = 2 * h + b;
                    const uint4 f = kv_block_fp8(make_uint2(c[u][2 * blk], c[u][2 * blk + 1]),
                                                 (sw[blk >> 2] >> (8 * (blk & 3))) & 0xFFu);
                    o[4 * b] = f.x;
                    o[4 * b + 1] = f.y;
                    o[4 * b + 2] = f.z;
                    o[4 * b + 3] = f.w;
                }
                st_v8(out + grp * 128 + h * 32, o);
            }
        }
    }
}

// CTA row y = one (batch, head) slice.  The slice's first L cache rows are
// contiguous, so block j of the slice sits at code byte 8j and scale byte j
// and its FP8 output at byte 16j: a flat index, no division.  A thread takes
// a pair of blocks (16 code bytes) per step, two pairs in flight.
__global__ void __launch_bounds__(KV_THREADS) kv_load_fp8_kernel(KvLoadShape s)
{
    if (blockIdx.x == 0 && blockIdx.y == 0 && threadIdx.x == 0)
        *s.out_scale = __fmul_rn(8.0f, *s.g);
    const int64_t bh = blockIdx.y;
    const int64_t nblk = s.L * s.bpr;
    const uint8_t *codes = s.codes + bh * s.Lcap * s.bpr * 8;
    const uint8_t *scales = s.scales + bh * s.Lcap * s.bpr;
    uint8_t *out = s.out + bh * nblk * 16;
    const bool vec = ((s.Lcap * s.bpr) & 1) == 0;  // slice base 16-byte aligned
    const int64_t npair = (nblk + 1) / 2;
    const int64_t stride = (int64_t)gridDim.x * KV_THREADS;
    for (int64_t p0 = (int64_t)blockIdx.x * KV_THREADS + threadIdx.x; p0 < npair; p0 += 2 * stride) {
        uint2 c[4];
        uint32_t sf[4];
#pragma unroll
        for (int u = 0; u < 2; ++u) {
            const int64_t p = p0 + u * stride, j = 2 * p;
            c[2 * u] = c[2 * u + 1] = make_uint2(0, 0);
            sf[2 * u] = sf[2 * u + 1] = 0;
            if (p < npair) {
                if (vec && j + 1 < nblk) {
                    const uint4 v = ld_nc_v4(codes + j * 8);
                    c[2 * u] = make_uint2(v.x, v.y);
                    c[2 * u + 1] = make_uint2(v.z, v.w);
                } else {
                    c[2 * u] = ld_nc_v2(codes + j * 8);
                    if (j + 1 < nblk)
                        c[2 * u + 1] = ld_nc_v2(codes + j * 8 + 8);
                }
                sf[2 * u] = scales[j];
                if (j + 1 < nblk)
                    sf[2 * u + 1] = scales[j + 1];
            }
        }
#pragma unroll
        for (int u = 0; u < 2; ++u) {
            const int64_t p = p0 + u * stride, j = 2 * p;
            if (p < npair) {
                st_v4(out + j * 16, kv_block_fp8(c[2 * u], sf[2 * u]));
                if (j + 1 < nblk)
                    st_v4(out + j * 16 + 16, kv_block_fp8(c[2 * u + 1], sf[2 * u + 1]));
            }
        }
    }
}

}  // namespace fp4lin
