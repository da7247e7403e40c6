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
// Work mapping: one lane owns one whole block -- 16 bf16 (32 bytes, one
// 256-bit load) for NVFP4, 32 bf16 (two loads) for MXFP4 -- so the Hadamard
// butterflies, the block maximum and the scale arithmetic all stay in the
// lane's registers and run once per block.  A warp covers 32 consecutive
// blocks of one row: 1 KB (NVFP4) or 2 KB (MXFP4) of contiguous input and
// 256 / 512 contiguous code bytes.  Requires cols % 64 == 0.
#pragma once

#include "common.cuh"

namespace fp4lin {

constexpr int QTHREADS = 256;            // 8 warps
constexpr int QWARPS = QTHREADS / 32;
constexpr int QUNROLL = 4;               // rows per warp per pass: four blocks in flight per lane
constexpr int QROWS = QWARPS * QUNROLL;  // rows covered by one CTA (32)
constexpr int AMAX_MAX_BLOCKS = 1024;

// Mapping: CTA (bx, by) covers blocks 32*bx .. 32*bx+31 of rows
// [by*QROWS, by*QROWS + QROWS); warp w handles rows by*QROWS + w + QWARPS*u,
// lane l block 32*bx + l.  No integer division.
struct QuantShape {
    const __nv_bfloat16 *x;
    int64_t rows, cols, ld;
    uint8_t *codes, *scales;
    int64_t blocks_per_row;  // cols / block
    int64_t sf_cols;         // = blocks_per_row
    int64_t katoms;          // ceil(sf_cols / 4)
    int64_t pad_items;       // padding bytes of the scale layout
    bool wide;               // x and every row start are 32-byte aligned: 256-bit loads
};

// Byte offset of scale (r, c) in the tensor-core layout (128 x 4 atoms).
__device__ __forceinline__ int64_t tc_offset(int64_t r, int64_t c, int64_t katoms)
{
    return ((r >> 7) * katoms + (c >> 2)) * 512 + (r & 31) * 16 + ((r >> 5) & 3) * 4 + (c & 3);
}

// In-place blockwise Hadamard butterflies on B values, strides 1, 2, 4, ...:
// the pair (u, w) becomes (u + w, u - w).
template <int B>
__device__ __forceinline__ void fwht(float *v)
{
#pragma unroll
    for (int h = 1; h < B; h <<= 1)
#pragma unroll
        for (int i = 0; i < B; ++i)
            if ((i & h) == 0) {
                const float u = v[i], w = v[i + h];
                v[i] = __fadd_rn(u, w);
                v[i + h] = __fsub_rn(u, w);
            }
}

// The same butterflies on the packed binary32 pipe: stride 1 pairs neighbours and runs
// scalar; every stride h >= 2 pairs element 2m with 2m+h and 2m+1 with 2m+1+h, so the
// pairs (v[2m], v[2m+1]) move together through add/sub.f32x2 -- the same IEEE operations
// in the same order, two per instruction.  The 1/sqrt(B) scaling `s` is packed too.
template <int B, bool SCALE = true>
__device__ __forceinline__ void fwht_scaled_packed(float *v, float s)
{
#pragma unroll
    for (int i = 0; i < B; i += 2) {
        const float u = v[i], w = v[i + 1];
        v[i] = __fadd_rn(u, w);
        v[i + 1] = __fsub_rn(u, w);
    }
    uint64_t P[B / 2];
#pragma unroll
    for (int m = 0; m < B / 2; ++m)
        P[m] = f2_pack(v[2 * m], v[2 * m + 1]);
#pragma unroll
    for (int h2 = 1; h2 < B / 2; h2 <<= 1)
#pragma unroll
        for (int m = 0; m < B / 2; ++m)
            if ((m & h2) == 0) {
                const uint64_t a = P[m], b = P[m + h2];
                P[m] = f2_add(a, b);
                P[m + h2] = f2_sub(a, b);
            }
    if constexpr (SCALE) {
        const uint64_t ss = f2_pack(s, s);
#pragma unroll
        for (int m = 0; m < B / 2; ++m)
            f2_unpack(f2_mul(P[m], ss), v[2 * m], v[2 * m + 1]);
    } else {
#pragma unroll
        for (int m = 0; m < B / 2; ++m)
            f2_unpack(P[m], v[2 * m], v[2 * m + 1]);
    }
}

// v[j] = RN(v[j] * s) for B values, two per packed instruction.
template <int B>
__device__ __forceinline__ void scale_packed(float *v, float s)
{
    const uint64_t ss = f2_pack(s, s);
#pragma unroll
    for (int m = 0; m < B / 2; ++m)
        f2_unpack(f2_mul(f2_pack(v[2 * m], v[2 * m + 1]), ss), v[2 * m], v[2 * m + 1]);
}

// max(a, b, c) in one instruction (the three-input form of max.f32; like fmaxf, a NaN input
// is ignored).
__device__ __forceinline__ float max3f(float a, float b, float c)
{
    float r;
    asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
    return r;
}

// max |v[i]| over B values: for B a multiple of 16 by three-input maxima (8 per 16 values).
template <int B>
__device__ __forceinline__ float abs_max(const float *v)
{
    float m = 0.0f;
    if constexpr (B % 16 != 0) {
#pragma unroll
        for (int i = 0; i < B; ++i)
            m = fmaxf(m, fabsf(v[i]));
        return m;
    }
#pragma unroll
    for (int i = 0; i < B; i += 16) {
        const float a = max3f(fabsf(v[i + 0]), fabsf(v[i + 1]), fabsf(v[i + 2]));
        const float b = max3f(fabsf(v[i + 3]), fabsf(v[i + 4]), fabsf(v[i + 5]));
        const float c = max3f(fabsf(v[i + 6]), fabsf(v[i + 7]), fabsf(v[i + 8]));
        const float d = max3f(fabsf(v[i + 9]), fabsf(v[i + 10]), fabsf(v[i + 11]));
        const float e = max3f(fabsf(v[i + 12]), fabsf(v[i + 13]), fabsf(v[i + 14]));
        m = max3f(m, max3f(a, b, c), max3f(d, e, fabsf(v[i + 15])));
    }
    return m;
}

// The (rotated, when HAD) values of one NVFP4 block: 16 bf16 in `raw`.  SCALE false leaves
// out the rotation's final exact factor 1/4 (for a maximum, which can take it afterwards).
template <bool HAD, bool SCALE = true>
__device__ __forceinline__ void nvfp4_block_values(const uint32_t *raw, float *v)
{
    bf16x8_to_f32(make_uint4(raw[0], raw[1], raw[2], raw[3]), v);
    bf16x8_to_f32(make_uint4(raw[4], raw[5], raw[6], raw[7]), v + 8);
    if (HAD)
        fwht_scaled_packed<16, SCALE>(v, 0.25f);  // 1/sqrt(16), exact
}

// The (rotated, when HAD) values of one MXFP4 block: 32 bf16 in `raw`.
template <bool HAD>
__device__ __forceinline__ void mxfp4_block_values(const uint32_t *raw, float *v)
{
#pragma unroll
    for (int k = 0; k < 4; ++k)
        bf16x8_to_f32(make_uint4(raw[4 * k], raw[4 * k + 1], raw[4 * k + 2], raw[4 * k + 3]), v + 8 * k);
    if (HAD)
        fwht_scaled_packed<32>(v, 0x1.6a09e6p-3f);  // 1/sqrt(32) rounded to binary32
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

// Zero the padding bytes of a tensor-core scale buffer (launched only when there are any).
__global__ void __launch_bounds__(QTHREADS) scale_padding_kernel(QuantShape q)
{
    for (int64_t j = (int64_t)blockIdx.x * QTHREADS + threadIdx.x; j < q.pad_items; j += (int64_t)gridDim.x * QTHREADS)
        zero_scale_padding(q, j);
}

// -------------------------------------------------------------------------
// Pass 1 of the dynamic tensor scale: per-CTA maxima of |x'| into partials[].
// Grid-strided over block segments (x) and row groups (y); at most
// AMAX_MAX_BLOCKS CTAs.
template <bool HAD>
__global__ void __launch_bounds__(QTHREADS) nvfp4_amax_kernel(QuantShape q, float *partials)
{
    pdl_trigger();  // a fused decode GEMM may start streaming its weights meanwhile
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    float m = 0.0f;
    for (int64_t seg = blockIdx.x; seg * 32 < q.blocks_per_row; seg += gridDim.x) {
        const int64_t c = seg * 32 + lane;
        const bool col_ok = c < q.blocks_per_row;
        for (int64_t r0 = (int64_t)blockIdx.y * QROWS; r0 < q.rows; r0 += (int64_t)gridDim.y * QROWS) {
            uint32_t raw[QUNROLL][8];
#pragma unroll
            for (int u = 0; u < QUNROLL; ++u) {
                const int64_t r = r0 + warp + QWARPS * u;
                if (col_ok && r < q.rows)
                    ld_nc_32B(q.x + r * q.ld + c * 16, q.wide, raw[u]);
                else
#pragma unroll
                    for (int j = 0; j < 8; ++j)
                        raw[u][j] = 0;
            }
#pragma unroll
            for (int u = 0; u < QUNROLL; ++u) {
                float v[16];
                nvfp4_block_values<HAD, false>(raw[u], v);
                m = fmaxf(m, abs_max<16>(v));
            }
        }
    }
    // the rotation's factor 1/4 on the maximum instead of on every value: x -> RN(x / 4) is
    // non-decreasing and odd, so the maximum of the scaled magnitudes is the scaled maximum
    if (HAD)
        m = __fmul_rn(m, 0.25f);
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

// Pass 2: quantise.  DYNAMIC: g = max(partials) / (6*448) (1 if not > 0),
// written to g_io by CTA (0,0); otherwise g is read from g_io.
// Per block: t = (amax/6)/g, sf = E4M3(t), d = dec(sf)*g, r = d > 0 ? 1/d : 0,
// codes = E2M1(x'*r).  sf comes from nvfp4_scale_code_fast (one product, the two divisions
// only where that product could round differently) and r from a per-CTA table over the 256
// scale bytes: the same bytes and codes as nvfp4_block_scale.
template <bool HAD, bool DYNAMIC>
__global__ void __launch_bounds__(QTHREADS, 4)  // four CTAs per SM: at most 64 registers
    nvfp4_quant_kernel(QuantShape q, float *g_io, const float *partials, int n_partials)
{
    __shared__ float s_g;
    __shared__ float red[QWARPS];
    __shared__ float s_rcp[256];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int64_t c = (int64_t)blockIdx.x * 32 + lane;
    const bool col_ok = c < q.blocks_per_row;
    const int64_t r0 = (int64_t)blockIdx.y * QROWS + warp;
    static_assert(QROWS == 32 && QWARPS == 8, "a CTA's rows are one 32-row group of the scale layout");
    // issue the loads first; the tensor-scale reduction overlaps them
    uint32_t raw[QUNROLL][8];
#pragma unroll
    for (int u = 0; u < QUNROLL; ++u) {
        const int64_t r = r0 + QWARPS * u;
        if (col_ok && r < q.rows)
            ld_nc_32B(q.x + r * q.ld + c * 16, q.wide, raw[u]);
        else
#pragma unroll
            for (int j = 0; j < 8; ++j)
                raw[u][j] = 0;
    }
    if (DYNAMIC) {
        pdl_wait();  // launched under the amax pass: its partials are complete past this point
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
    // 1/(dec(sf)*g) for every scale byte, once per CTA instead of once per block
    static_assert(QTHREADS == 256, "one table entry per thread");
    s_rcp[threadIdx.x] = nvfp4_block_rcp(threadIdx.x, g);
    __syncthreads();
    const float c6 = nvfp4_fast_c6(g);
    // the QUNROLL rows of a thread share their 32-row group: scale bytes 128 apart
    const int64_t sbase = tc_offset(r0, c, q.katoms);
#pragma unroll
    for (int u = 0; u < QUNROLL; ++u) {
        const int64_t r = r0 + QWARPS * u;
        if (!(col_ok && r < q.rows))
            continue;
        float v[16];
        nvfp4_block_values<HAD>(raw[u], v);
        const uint32_t sf = nvfp4_scale_code_fast(abs_max<16>(v), g, c6);
        scale_packed<16>(v, s_rcp[sf]);
        *reinterpret_cast<uint2 *>(q.codes + r * (q.cols / 2) + c * 8) = make_uint2(pack_e2m1x8(v), pack_e2m1x8(v + 8));
        q.scales[sbase + 128 * u] = (uint8_t)sf;
    }
}

// MXFP4: E8M0 byte = max(E - 2, 0) where E is the biased binary32 exponent
// of the block maximum (= clamp(floor(log2 amax) - 2 + 127, 0, 254) for
// finite inputs); elements are scaled by 2^(127 - byte), an exact product.
// NEAREST: the scale amax/6 rounded to the nearer power of two by value, ties
// upward (page "FP4 auf Blackwell", section "Was NVFP4 von frueheren
// 4-Bit-Formaten unterscheidet": E8M0 rounds the scale to the nearest power of
// two): one step lower than the rule above exactly when amax < 1.125 * 2^(E-127),
// i.e. when the stored mantissa is below 2^20.
template <bool HAD, bool NEAREST = false>
__global__ void __launch_bounds__(QTHREADS) mxfp4_quant_kernel(QuantShape q)
{
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int64_t c = (int64_t)blockIdx.x * 32 + lane;
    const bool col_ok = c < q.blocks_per_row;
    const int64_t r0 = (int64_t)blockIdx.y * QROWS + warp;
    constexpr int U = QUNROLL / 2;  // a block is 64 bytes: two rows in flight per pass
#pragma unroll
    for (int half = 0; half < 2; ++half) {
        uint32_t raw[U][16];
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const int64_t r = r0 + QWARPS * (u + U * half);
            if (col_ok && r < q.rows) {
                const __nv_bfloat16 *p = q.x + r * q.ld + c * 32;
                ld_nc_32B(p, q.wide, raw[u]);
                ld_nc_32B(p + 16, q.wide, raw[u] + 8);
            } else {
#pragma unroll
                for (int j = 0; j < 16; ++j)
                    raw[u][j] = 0;
            }
        }
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const int64_t r = r0 + QWARPS * (u + U * half);
            if (!(col_ok && r < q.rows))
                continue;
            float v[32];
            mxfp4_block_values<HAD>(raw[u], v);
            const float amax = abs_max<32>(v);
            const uint32_t bits = __float_as_uint(amax);
            const uint32_t E = (bits >> 23) & 0xFFu;
            const uint32_t lower = (NEAREST && (bits & 0x7FFFFFu) < 0x100000u) ? 1u : 0u;
            const uint32_t byte = E >= 2u + lower ? E - 2u - lower : 0u;
            const float s = __uint_as_float((254u - byte) << 23);  // 2^(127 - byte)
            scale_packed<32>(v, s);
            st_v4(q.codes + r * (q.cols / 2) + c * 16,
                  make_uint4(pack_e2m1x8(v), pack_e2m1x8(v + 8), pack_e2m1x8(v + 16), pack_e2m1x8(v + 24)));
            q.scales[tc_offset(r, c, q.katoms)] = (uint8_t)byte;
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
