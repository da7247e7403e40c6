// gptq.cuh -- MR-GPTQ weight quantisation (offline): GPTQ's column sweep on the
// blockwise-Hadamard-rotated weights (the MR-GPTQ abstract, hyper.ai/de/papers/2509.23202,
// "Abstract": GPTQ adapted to FP4 through blockwise Hadamard transforms; page "FP8, NVFP4
// czy AWQ?", section "Czym roznia sie FP8, NVFP4, MXFP4 i AWQ?": GPTQ quantises weights
// layer by layer with error correction).
//
// The sweep, for every row of W' = W R independently: at the first column of each block
// (16 NVFP4 / 32 MXFP4 values) fix the block's scale from the row's current values with the
// format's rule; quantise column j; e = (w_j - q_j) / U[j][j]; w_k <- fma(-e, U[j][k], w_k)
// for all k > j, so every value receives its corrections one at a time in increasing j.
// U (upper triangular, H^-1 = U^T U for the damped Hessian of the rotated inputs) is an
// input.
//
// GPU form (GPTQ's lazy batches, two levels deep, in the same arithmetic order):
//  * gptq_rotate_kernel: bf16 W -> binary32 W' in the workspace (the quantisers' rotation).
//  * per superblock of 256 columns [s0, s0+256), per 64-column block [c0, c0+64) in it:
//      gptq_block_kernel: one thread per row holds the 64 values in registers and sweeps
//      them, reading the 64x64 triangle of U from shared memory (every thread reads the same
//      word: a broadcast); writes the codes, the scales and the negated errors -e of its
//      row into E^T [256][N] (transposed: the update kernel copies it as it stands);
//      gptq_update_kernel over [c0+64, s0+256): the block's corrections to the rest of the
//      superblock, so the next block sweeps current values;
//    then gptq_update_kernel over [s0+256, K) with all 256 corrections of the superblock.
//    Each value still receives its corrections one at a time in increasing j; W' beyond the
//    superblock is read and written once per 256 columns instead of once per 64.
//  The update is a 128x128-tile binary32 product accumulated straight into W', its E and U
//  chunks streamed through a double-buffered cp.async ring.
// The tensor cores are not used: their products round differently, and the quantisation
// decisions downstream must see exactly the binary32 values the sweep defines.
#pragma once

#include "scale_search.cuh"

namespace fp4lin {

constexpr int GQ_B = 64;         // columns per lazy block
constexpr int GQ_SB = 256;       // columns per superblock (the E^T buffer's height)
constexpr int GQ_ROWS = 128;     // rows (threads) per CTA of the block kernel
constexpr int GQ_TILE = 128;     // update kernel: 128 x 128 tile of W', 256 threads, 8 x 8 each
constexpr int GQ_CJ = 32;                                        // values of j per staged chunk
constexpr int GQ_CHUNK_FLOATS = GQ_CJ * GQ_TILE;                 // one 32 x 128 operand chunk
constexpr int GQ_UPD_SMEM = 2 * 2 * GQ_CHUNK_FLOATS * 4;          // two stages of (E^T chunk, U chunk): 64 KB

struct GptqArgs {
    float *wr;            // W' [N, K] binary32, row stride K (workspace)
    float *et;            // -e of the current superblock, transposed: [256][np] (workspace)
    int64_t np;           // row stride of et: N rounded up to a multiple of 4
    const float *u;       // U [K, K], row stride ld_u; entries with row > column are not read
    int64_t N, K, ld_u;
    const float *g;       // NVFP4 tensor scale (device)
    uint8_t *codes;       // [N, K/2]
    uint8_t *scales;      // tensor-core layout of [N, K/16] (NVFP4) or [N, K/32] (MXFP4)
    int64_t katoms;       // scale atoms along K
};

// bf16 W [N, K] (row stride ld) -> W' [N, K] binary32 (row stride K): each BW-value block
// rotated by H_BW / sqrt(BW) when HAD, with the quantisers' own arithmetic.
template <int BW, bool HAD>
__global__ void __launch_bounds__(256) gptq_rotate_kernel(const __nv_bfloat16 *w, int64_t N, int64_t K, int64_t ld,
                                                          float *wr)
{
    const int64_t nb = K / BW, total = N * nb;
    for (int64_t i = (int64_t)blockIdx.x * 256 + threadIdx.x; i < total; i += (int64_t)gridDim.x * 256) {
        const int64_t r = i / nb, b = i - r * nb;
        const __nv_bfloat16 *src = w + r * ld + b * BW;
        uint32_t raw[BW / 2];
#pragma unroll
        for (int q = 0; q < BW / 8; ++q) {
            const uint4 t = ld_nc_v4(src + 8 * q);
            raw[4 * q] = t.x;
            raw[4 * q + 1] = t.y;
            raw[4 * q + 2] = t.z;
            raw[4 * q + 3] = t.w;
        }
        float v[BW];
        if constexpr (BW == 16)
            nvfp4_block_values<HAD>(raw, v);
        else
            mxfp4_block_values<HAD>(raw, v);
        float4 *dst = reinterpret_cast<float4 *>(wr + r * K + b * BW);
#pragma unroll
        for (int q = 0; q < BW / 4; ++q)
            dst[q] = make_float4(v[4 * q], v[4 * q + 1], v[4 * q + 2], v[4 * q + 3]);
    }
}

// g = max(partials) / 2688 (1 when not > 0): the quantiser's dynamic tensor scale.
__global__ void gptq_tensor_scale_kernel(const float *partials, int n, float *g)
{
    __shared__ float red[8];
    float m = 0.0f;
    for (int k = threadIdx.x; k < n; k += 256)
        m = fmaxf(m, partials[k]);
#pragma unroll
    for (int o = 16; o; o >>= 1)
        m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    if ((threadIdx.x & 31) == 0)
        red[threadIdx.x >> 5] = m;
    __syncthreads();
    if (threadIdx.x == 0) {
        float b = 0.0f;
        for (int k = 0; k < 8; ++k)
            b = fmaxf(b, red[k]);
        float v = __fdiv_rn(b, 2688.0f);
        *g = (v > 0.0f) ? v : 1.0f;
    }
}

// Exact binary32 value of one E2M1 code (low nibble of c).
__device__ __forceinline__ float e2m1_value(uint32_t c)
{
    uint32_t h;
    asm("{\n\t.reg .b8 b;\n\tcvt.u8.u32 b, %1;\n\tcvt.rn.f16x2.e2m1x2 %0, b;\n\t}" : "=r"(h) : "r"(c & 0xFu));
    return __half2float(__ushort_as_half((unsigned short)(h & 0xFFFFu)));
}

// 2^(byte - 127), exact (byte 0 is the subnormal 2^-127).
__device__ __forceinline__ float e8m0_value(uint32_t byte)
{
    return __uint_as_float(byte ? byte << 23 : 0x00400000u);
}

// Column J of a row's 64-value block: the block scale at the first column of each format
// block, the code, the error, and the corrections of the later columns.  A template over J
// so that every index into the register arrays is a constant.
template <bool NV, bool MSE, int J>
struct GptqColumn {
    static __device__ __forceinline__ void run(float (&w)[GQ_B], const float (&us)[GQ_B][GQ_B], float g, float &mul,
                                               float &back, uint32_t (&code_words)[GQ_B / 8], uint32_t &sf_word,
                                               float *ecol, int64_t np)
    {
        constexpr int G = NV ? 16 : 32;
        if constexpr (J % G == 0) {
            float amax = 0.0f;
#pragma unroll
            for (int i = 0; i < G; ++i)
                amax = fmaxf(amax, fabsf(w[J + i]));
            uint32_t sf;
            if constexpr (NV && MSE) {  // the least squared error over all 127 E4M3 codes (ties: smaller)
                float best = block_sq_error(&w[J], 0u, g);
                sf = 0u;
                for (uint32_t cand = 1; cand <= 126; ++cand) {
                    const float e = block_sq_error(&w[J], cand, g);
                    if (e < best) {
                        best = e;
                        sf = cand;
                    }
                }
                back = __fmul_rn(e4m3_value(sf), g);
                mul = back > 0.0f ? __fdiv_rn(1.0f, back) : 0.0f;
            } else if constexpr (NV) {
                sf = nvfp4_block_scale(amax, g, mul);
                back = __fmul_rn(e4m3_value(sf), g);
            } else {
                const uint32_t E = (__float_as_uint(amax) >> 23) & 0xFFu;
                sf = E >= 2u ? E - 2u : 0u;
                mul = __uint_as_float((254u - sf) << 23);  // 2^(127 - byte)
                back = e8m0_value(sf);
            }
            sf_word |= sf << (8 * (J / G));
        }
        const uint32_t c = cvt_e2m1x2(__fmul_rn(w[J], mul), 0.0f) & 0xFu;
        const float q = __fmul_rn(e2m1_value(c), back);
        if constexpr (J % 8 == 0)
            code_words[J / 8] = c;
        else
            code_words[J / 8] |= c << (4 * (J % 8));
        const float e = __fdiv_rn(__fsub_rn(w[J], q), us[J][J]);
        ecol[J * np] = -e;
#pragma unroll
        for (int k = J + 1; k < GQ_B; ++k)
            w[k] = __fmaf_rn(-e, us[J][k], w[k]);
        if constexpr (J + 1 < GQ_B)
            GptqColumn<NV, MSE, J + 1>::run(w, us, g, mul, back, code_words, sf_word, ecol, np);
    }
};

// One 64-column block of the sweep for every row.  NV: NVFP4 (16-value blocks, E4M3 scales
// relative to *g; MSE: the scale of least squared error over all 127 E4M3 codes, as
// nvfp4_quant_mse_kernel picks it); else MXFP4 (32-value blocks, E8M0 by the OCP rule).
template <bool NV, bool MSE = false>
__global__ void __launch_bounds__(GQ_ROWS) gptq_block_kernel(GptqArgs a, int64_t c0, int64_t s0)
{
    __shared__ float us[GQ_B][GQ_B];
    for (int i = threadIdx.x; i < GQ_B * GQ_B; i += GQ_ROWS) {
        const int j = i / GQ_B, k = i % GQ_B;
        us[j][k] = k >= j ? a.u[(c0 + j) * a.ld_u + c0 + k] : 0.0f;
    }
    __syncthreads();
    const int64_t n = (int64_t)blockIdx.x * GQ_ROWS + threadIdx.x;
    if (n >= a.N)
        return;
    float w[GQ_B];
    const float4 *src = reinterpret_cast<const float4 *>(a.wr + n * a.K + c0);
#pragma unroll
    for (int q = 0; q < GQ_B / 4; ++q) {
        const float4 t = src[q];
        w[4 * q] = t.x;
        w[4 * q + 1] = t.y;
        w[4 * q + 2] = t.z;
        w[4 * q + 3] = t.w;
    }
    const float g = NV ? *a.g : 1.0f;
    float mul = 0.0f, back = 0.0f;  // x -> code scale and code -> value scale of the current block
    uint32_t code_words[GQ_B / 8];
    uint32_t sf_word = 0;
    GptqColumn<NV, MSE, 0>::run(w, us, g, mul, back, code_words, sf_word, a.et + (c0 - s0) * a.np + n, a.np);
    uint4 *dst = reinterpret_cast<uint4 *>(a.codes + n * (a.K / 2) + c0 / 2);
    dst[0] = make_uint4(code_words[0], code_words[1], code_words[2], code_words[3]);
    dst[1] = make_uint4(code_words[4], code_words[5], code_words[6], code_words[7]);
    if constexpr (NV)  // scale columns c0/16 .. c0/16 + 3: the 4 bytes of one atom word
        *reinterpret_cast<uint32_t *>(a.scales + tc_offset(n, c0 / 16, a.katoms)) = sf_word;
    else               // scale columns c0/32, c0/32 + 1
        *reinterpret_cast<uint16_t *>(a.scales + tc_offset(n, c0 / 32, a.katoms)) = (uint16_t)sf_word;
}

__device__ __forceinline__ void cp_async16(void *smem, const void *gmem, uint32_t src_bytes)
{
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(smem_u32(smem)), "l"(gmem), "r"(src_bytes)
                 : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait1() { asm volatile("cp.async.wait_group 1;" ::: "memory"); }

// W'[:, k0 : k1) receives the corrections of columns j0 .. j0+nj-1 (nj a multiple of 64),
// element by element in increasing j: w = fma(-e_j, U[j][k], w).  -e_j comes from row
// jo + (j - j0) of E^T.  CTA tile 128 rows x 128 columns; thread (ty, tx) of 16 x 16 holds
// rows 8 ty + i (i < 8) and columns 4 tx + 64 h + l (h < 2, l < 4), so a step j is four
// 128-bit shared loads (8 multipliers, 8 U values) and 64 scalar fmas.  (The packed
// fma.rn.f32x2 form holds the FMA pipe two cycles per instruction and measured slower.)
__global__ void __launch_bounds__(256, 2)
    gptq_update_kernel(GptqArgs a, int64_t j0, int nj, int64_t jo, int64_t k0, int64_t k1)
{
    extern __shared__ __align__(16) float gq_smem[];
    const int64_t row0 = (int64_t)blockIdx.y * GQ_TILE, col0 = k0 + (int64_t)blockIdx.x * GQ_TILE;
    const int t = threadIdx.x, tx = t & 15, ty = t >> 4;
    // chunk q (32 values of j) into stage b: es[j][r] = -e of row row0 + r, us[j][c] = U[j][col0 + c]
    auto stage = [&](int q, int b) {
        float *es = gq_smem + b * 2 * GQ_CHUNK_FLOATS, *us = es + GQ_CHUNK_FLOATS;
#pragma unroll
        for (int x = 0; x < GQ_CHUNK_FLOATS / 4 / 256; ++x) {
            const int c = t + 256 * x, j = c >> 5, q4 = (c & 31) * 4;  // 32 16-byte pieces per row
            const int64_t n = row0 + q4;
            const int64_t nv = a.N - n;  // rows of this piece inside E^T's live part
            const uint32_t eb = nv >= 4 ? 16u : nv > 0 ? (uint32_t)nv * 4u : 0u;
            const float *esrc = a.et + (jo + GQ_CJ * q + j) * a.np + (eb ? n : 0);
            cp_async16(es + j * GQ_TILE + q4, esrc, eb);
            const int64_t k = col0 + q4;
            const uint32_t ub = k < k1 ? 16u : 0u;  // k1 - col0 is a multiple of 64: whole pieces
            const float *usrc = a.u + (j0 + GQ_CJ * q + j) * a.ld_u + (ub ? k : 0);
            cp_async16(us + j * GQ_TILE + q4, usrc, ub);
        }
    };
    const int nq = nj / GQ_CJ;
    stage(0, 0);
    cp_async_commit();
    float acc[8][8];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        const int64_t n = row0 + 8 * ty + i;
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            const int64_t k = col0 + 4 * tx + 64 * h;
            float4 v = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
            if (n < a.N && k < k1)
                v = *reinterpret_cast<const float4 *>(a.wr + n * a.K + k);
            acc[i][4 * h] = v.x;
            acc[i][4 * h + 1] = v.y;
            acc[i][4 * h + 2] = v.z;
            acc[i][4 * h + 3] = v.w;
        }
    }
    for (int q = 0; q < nq; ++q) {
        if (q + 1 < nq)
            stage(q + 1, (q + 1) & 1);
        cp_async_commit();  // possibly empty: the wait below always leaves one group in flight
        cp_async_wait1();
        __syncthreads();
        const float *es = gq_smem + (q & 1) * 2 * GQ_CHUNK_FLOATS, *us = es + GQ_CHUNK_FLOATS;
#pragma unroll 2
        for (int j = 0; j < GQ_CJ; ++j) {
            const float4 e0 = *reinterpret_cast<const float4 *>(es + j * GQ_TILE + 8 * ty);
            const float4 e1 = *reinterpret_cast<const float4 *>(es + j * GQ_TILE + 8 * ty + 4);
            const float4 u0 = *reinterpret_cast<const float4 *>(us + j * GQ_TILE + 4 * tx);
            const float4 u1 = *reinterpret_cast<const float4 *>(us + j * GQ_TILE + 64 + 4 * tx);
            const float ev[8] = {e0.x, e0.y, e0.z, e0.w, e1.x, e1.y, e1.z, e1.w};
            const float uv[8] = {u0.x, u0.y, u0.z, u0.w, u1.x, u1.y, u1.z, u1.w};
#pragma unroll
            for (int i = 0; i < 8; ++i)
#pragma unroll
                for (int l = 0; l < 8; ++l)
                    acc[i][l] = __fmaf_rn(ev[i], uv[l], acc[i][l]);
        }
        __syncthreads();  // stage q & 1 is refilled by the next iteration
    }
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        const int64_t n = row0 + 8 * ty + i;
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            const int64_t k = col0 + 4 * tx + 64 * h;
            if (n < a.N && k < k1)
                *reinterpret_cast<float4 *>(a.wr + n * a.K + k) =
                    make_float4(acc[i][4 * h], acc[i][4 * h + 1], acc[i][4 * h + 2], acc[i][4 * h + 3]);
        }
    }
}

}  // namespace fp4lin
