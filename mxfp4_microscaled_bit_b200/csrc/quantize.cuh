// quantize.cuh -- NVFP4 and MXFP4 quantisers with the blockwise Hadamard
// rotation fused in (HBM-bound kernels).
//
// Formats: E2M1 elements in 16-value blocks with an E4M3 block scale and an
// FP32 tensor scale (NVFP4), or 32-value blocks with an E8M0 power-of-two
// scale (MXFP4) -- page "FP4 auf Blackwell: Was NVFP4 fuer lokale KI
// wirklich aendert", section "Was NVFP4 von frueheren 4-Bit-Formaten
// unterscheidet", and page "FP8, NVFP4 czy AWQ?", section "Czym roznia sie
// FP8, NVFP4, MXFP4 i AWQ?".  The rotation is the online activation side of
// the blockwise Hadamard transform of the MR-GPTQ abstract.
//
// Work mapping: one lane owns 8 consecutive bf16 (one 16-byte load).  A
// 16-value NVFP4 block is a lane pair, a 32-value MXFP4 block a lane quad;
// the last Hadamard stages and the block maxima cross lanes with shuffles.
// A warp reads 512 contiguous bytes of one row per load and writes 128
// contiguous code bytes per store.  Requires cols % 64 == 0, so no block is
// cut by the end of a row.
#pragma once

#include "common.cuh"

namespace fp4lin {

constexpr int QTHREADS = 256;          // 8 warps
constexpr int QWARPS = QTHREADS / 32;
constexpr int QUNROLL = 4;             // rows per warp per pass: four 16-byte loads in flight per lane
constexpr int QROWS = QWARPS * QUNROLL;  // rows covered by one CTA in one pass (32)
constexpr int AMAX_MAX_BLOCKS = 1024;

// Mapping: CTA (bx, by) covers the 256-value row segment bx of rows
// [by*QROWS, by*QROWS + QROWS); warp w handles rows by*QROWS + w + QWARPS*u,
// lane l the 8 values at column 8*(32*bx + l).  No integer division.
struct QuantShape {
    const __nv_bfloat16 *x;
    int64_t rows, cols, ld;
    uint8_t *codes, *scales;
    int64_t chunks_per_row;  // cols / 8
    int64_t sf_cols;         // cols / block
    int64_t katoms;          // ceil(sf_cols / 4)
    int64_t pad_items;       // padding bytes of the scale layout
};

// Byte offset of scale (r, c) in the tensor-core layout (128 x 4 atoms).
__device__ __forceinline__ int64_t tc_offset(int64_t r, int64_t c, int64_t katoms)
{
    return ((r >> 7) * katoms + (c >> 2)) * 512 + (r & 31) * 16 + ((r >> 5) & 3) * 4 + (c & 3);
}

// Butterflies with strides 1, 2, 4 on the lane's 8 consecutive values.
__device__ __forceinline__ void fwht8(float *v)
{
#pragma unroll
    for (int h = 1; h < 8; h <<= 1)
#pragma unroll
        for (int i = 0; i < 8; ++i)
            if ((i & h) == 0) {
                float u = v[i], w = v[i + h];
                v[i] = __fadd_rn(u, w);
                v[i + h] = __fsub_rn(u, w);
            }
}

// One butterfly stage across the lane pair (lane, lane ^ mask): the lower
// lane holds u and keeps u + w, the upper lane holds w and keeps u - w.
__device__ __forceinline__ void fwht_cross(float *v, int mask, bool upper)
{
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        float o = __shfl_xor_sync(0xffffffffu, v[i], mask);
        v[i] = upper ? __fsub_rn(o, v[i]) : __fadd_rn(v[i], o);
    }
}

__device__ __forceinline__ float abs_max8(const float *v)
{
    float m = 0.0f;
#pragma unroll
    for (int i = 0; i < 8; ++i)
        m = fmaxf(m, fabsf(v[i]));
    return m;
}

// Rotated (when HAD) values of a lane's chunk of a 16-value block.
template <bool HAD>
__device__ __forceinline__ void nvfp4_lane_values(uint4 raw, bool upper, float *v)
{
    bf16x8_to_f32(raw, v);
    if (HAD) {
        fwht8(v);
        fwht_cross(v, 1, upper);
#pragma unroll
        for (int j = 0; j < 8; ++j)
            v[j] = __fmul_rn(v[j], 0.25f);  // 1/sqrt(16), exact
    }
}

template <bool HAD>
__device__ __forceinline__ void mxfp4_lane_values(uint4 raw, int lane, float *v)
{
    bf16x8_to_f32(raw, v);
    if (HAD) {
        fwht8(v);
        fwht_cross(v, 1, lane & 1);
        fwht_cross(v, 2, lane & 2);
#pragma unroll
        for (int j = 0; j < 8; ++j)
            v[j] = __fmul_rn(v[j], 0x1.6a09e6p-3f);  // 1/sqrt(32) rounded to binary32
    }
}

// Zero the padding bytes of a tensor-core scale buffer (rows past `rows`,
// scale columns past `sf_cols`); item j of pad_items.
__device__ __forceinline__ void zero_scale_padding(const QuantShape &q, int64_t j)
{
    const int64_t rows_pad = (q.rows + 127) / 128 * 128, sfc_pad = q.katoms * 4;
    const int64_t tail_rows_items = (rows_pad - q.rows) * sfc_pad;
    int64_t r, c;
    if (j < tail_rows_items) {
        r = q.rows + j / sfc_pad;
        c = j % sfc_pad;
    } else {
        j -= tail_rows_items;
        const int64_t w = sfc_pad - q.sf_cols;
        r = j / w;
        c = q.sf_cols + j % w;
    }
    q.scales[tc_offset(r, c, q.katoms)] = 0;
}

// -------------------------------------------------------------------------
// Pass 1 of the dynamic tensor scale: per-CTA maxima of |x'| into partials[].
// Grid-strided over segments (x) and row groups (y); at most AMAX_MAX_BLOCKS CTAs.
template <bool HAD>
__global__ void __launch_bounds__(QTHREADS) nvfp4_amax_kernel(QuantShape q, float *partials)
{
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const bool upper = lane & 1;
    float m = 0.0f;
    for (int64_t seg = blockIdx.x; seg * 32 < q.chunks_per_row; seg += gridDim.x) {
        const int64_t c8 = seg * 32 + lane;
        const bool col_ok = c8 < q.chunks_per_row;
        for (int64_t r0 = (int64_t)blockIdx.y * QROWS; r0 < q.rows; r0 += (int64_t)gridDim.y * QROWS) {
            uint4 raw[QUNROLL];
#pragma unroll
            for (int u = 0; u < QUNROLL; ++u) {
                const int64_t r = r0 + warp + QWARPS * u;
                raw[u] = (col_ok && r < q.rows) ? ld_nc_v4(q.x + r * q.ld + c8 * 8) : make_uint4(0, 0, 0, 0);
            }
#pragma unroll
            for (int u = 0; u < QUNROLL; ++u) {
                float v[8];
                nvfp4_lane_values<HAD>(raw[u], upper, v);
                m = fmaxf(m, abs_max8(v));
            }
        }
    }
#pragma unroll
    for (int o = 16; o; o >>= 1)
        m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    __shared__ float red[QWARPS];
    if (lane == 0)
        red[warp] = m;
    __syncthreads();
    if (threadIdx.x == 0) {
        float b = 0.0f;
        for (int k = 0; k < QWARPS; ++k)
            b = fmaxf(b, red[k]);
        partials[blockIdx.y * gridDim.x + blockIdx.x] = b;
    }
}

// Zero the padding bytes of a tensor-core scale buffer (launched only when there are any).
__global__ void __launch_bounds__(QTHREADS) scale_padding_kernel(QuantShape q)
{
    for (int64_t j = (int64_t)blockIdx.x * QTHREADS + threadIdx.x; j < q.pad_items; j += (int64_t)gridDim.x * QTHREADS)
        zero_scale_padding(q, j);
}

// Pass 2: quantise.  DYNAMIC: g = max(partials) / (6*448) (1 if not > 0),
// written to g_io by CTA (0,0); otherwise g is read from g_io.
template <bool HAD, bool DYNAMIC>
__global__ void __launch_bounds__(QTHREADS)
    nvfp4_quant_kernel(QuantShape q, float *g_io, const float *partials, int n_partials)
{
    __shared__ float s_g;
    __shared__ float red[QWARPS];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int64_t c8 = (int64_t)blockIdx.x * 32 + lane;
    const bool col_ok = c8 < q.chunks_per_row;
    const int64_t r0 = (int64_t)blockIdx.y * QROWS + warp;
    // issue the loads first; the tensor-scale reduction overlaps them
    uint4 raw[QUNROLL];
#pragma unroll
    for (int u = 0; u < QUNROLL; ++u) {
        const int64_t r = r0 + QWARPS * u;
        raw[u] = (col_ok && r < q.rows) ? ld_nc_v4(q.x + r * q.ld + c8 * 8) : make_uint4(0, 0, 0, 0);
    }
    if (DYNAMIC) {
        float m = 0.0f;
        for (int k = threadIdx.x; k < n_partials; k += QTHREADS)
            m = fmaxf(m, partials[k]);
#pragma unroll
        for (int o = 16; o; o >>= 1)
            m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
        if (lane == 0)
            red[warp] = m;
        __syncthreads();
        if (threadIdx.x == 0) {
            float b = 0.0f;
            for (int k = 0; k < QWARPS; ++k)
                b = fmaxf(b, red[k]);
            float g = __fdiv_rn(b, 2688.0f);  // 6 * 448: E2M1 max times E4M3 max
            if (!(g > 0.0f))
                g = 1.0f;
            s_g = g;
            if (blockIdx.x == 0 && blockIdx.y == 0)
                *g_io = g;
        }
    } else if (threadIdx.x == 0) {
        s_g = *g_io;
    }
    __syncthreads();
    const float g = s_g;
    const bool upper = lane & 1;
#pragma unroll
    for (int u = 0; u < QUNROLL; ++u) {
        const int64_t r = r0 + QWARPS * u;
        float v[8];
        nvfp4_lane_values<HAD>(raw[u], upper, v);
        float amax = abs_max8(v);
        amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 1));
        const float t = __fdiv_rn(__fdiv_rn(amax, 6.0f), g);
        const uint32_t sf = cvt_e4m3(t);
        const float d = __fmul_rn(e4m3_value(sf), g);
        const float rcp = d > 0.0f ? __fdiv_rn(1.0f, d) : 0.0f;
#pragma unroll
        for (int j = 0; j < 8; ++j)
            v[j] = __fmul_rn(v[j], rcp);
        const uint32_t packed = pack_e2m1x8(v);
        if (col_ok && r < q.rows) {
            *reinterpret_cast<uint32_t *>(q.codes + r * (q.cols / 2) + c8 * 4) = packed;
            if (!upper)
                q.scales[tc_offset(r, c8 >> 1, q.katoms)] = (uint8_t)sf;
        }
    }
}

// MXFP4: E8M0 byte = max(E - 2, 0) where E is the biased binary32 exponent
// of the block maximum (= clamp(floor(log2 amax) - 2 + 127, 0, 254) for
// finite inputs); elements are scaled by 2^(127 - byte), an exact product.
template <bool HAD>
__global__ void __launch_bounds__(QTHREADS) mxfp4_quant_kernel(QuantShape q)
{
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int64_t c8 = (int64_t)blockIdx.x * 32 + lane;
    const bool col_ok = c8 < q.chunks_per_row;
    const int64_t r0 = (int64_t)blockIdx.y * QROWS + warp;
    uint4 raw[QUNROLL];
#pragma unroll
    for (int u = 0; u < QUNROLL; ++u) {
        const int64_t r = r0 + QWARPS * u;
        raw[u] = (col_ok && r < q.rows) ? ld_nc_v4(q.x + r * q.ld + c8 * 8) : make_uint4(0, 0, 0, 0);
    }
#pragma unroll
    for (int u = 0; u < QUNROLL; ++u) {
        const int64_t r = r0 + QWARPS * u;
        float v[8];
        mxfp4_lane_values<HAD>(raw[u], lane, v);
        float amax = abs_max8(v);
        amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 1));
        amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 2));
        const uint32_t E = (__float_as_uint(amax) >> 23) & 0xFFu;
        const uint32_t byte = E >= 2u ? E - 2u : 0u;
        const float s = __uint_as_float((254u - byte) << 23);  // 2^(127 - byte)
#pragma unroll
        for (int j = 0; j < 8; ++j)
            v[j] = __fmul_rn(v[j], s);
        const uint32_t packed = pack_e2m1x8(v);
        if (col_ok && r < q.rows) {
            *reinterpret_cast<uint32_t *>(q.codes + r * (q.cols / 2) + c8 * 4) = packed;
            if ((lane & 3) == 0)
                q.scales[tc_offset(r, c8 >> 2, q.katoms)] = (uint8_t)byte;
        }
    }
}

// Element conversions exactly as the quantisers use them (diagnostic export).
__global__ void convert_selftest_kernel(const float *in, uint8_t *e2m1, uint8_t *e4m3, int64_t n)
{
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (int64_t)gridDim.x * blockDim.x) {
        const float x = in[i];
        e2m1[i] = (uint8_t)(cvt_e2m1x2(x, 0.0f) & 0xFu);
        e4m3[i] = (uint8_t)cvt_e4m3(x);
    }
}

}  // namespace fp4lin
