// kv_attention.cuh -- decode attention straight from the NVFP4 KV cache.  The
// cached K and V rows are dequantised to the FP8 values the load path
// (kv_nvfp4_load_fp8) would write -- page "NVFP4 KV cache" story: new K/V rows
// stored in NVFP4, dequantised to FP8 before attention -- but in registers,
// so the 4.3 GB FP8 copy of the 64 x 8 x 32768 x 128 cache is never written
// or read back: the cache's 2.4 GB are read once.
//
// Attention (a reading; the pages name no details): G query heads per kv
// head, query head j uses kv head j / G; s_l = (q . k_l) / sqrt(D) with k_l
// the FP8 value times 8 g_k; softmax over l < L; o = sum_l p_l v_l with v_l
// the FP8 value times 8 g_v.  binary32 arithmetic, D = 128.
//
// Split over L (flash-decoding): CTA (s, bh) takes positions [s*chunk,
// min(L, (s+1)*chunk)) of kv head bh for all G query heads (each K/V byte is
// read once per group).  Pass 1: one thread per position forms the G scores
// (q from shared memory, broadcast reads).  Pass 2: a half-warp per position,
// lane l of a half owns dimensions 8l..8l+7.  The chunk's maximum, sum and unnormalised
// output go to the workspace; kv_attn_merge_kernel combines the chunks.
#pragma once

#include "common.cuh"

namespace fp4lin {

constexpr int KA_D = 128;          // head dimension
constexpr int KA_THREADS = 256;
constexpr int KA_WARPS = KA_THREADS / 32;
constexpr int KA_CHUNK = 512;      // positions per CTA
constexpr int KA_GMAX = 8;         // query heads per kv head

struct KvAttnShape {
    const __nv_bfloat16 *q;        // [B, H*G, D]
    const uint8_t *kc, *ks, *vc, *vs;  // [B, H, Lcap, D/2] codes, [B, H, Lcap, D/16] scales
    const float *gk, *gv;
    float *ws;                     // [B*H, S, G, D + 2]: unnormalised output, chunk max, chunk sum
    float *out;                    // [B, H*G, D]
    int64_t L, Lcap;
    int H, S;
};

// Eight E2M1 codes (one code word, element 2i in the low nibble of byte i) times the block
// scale / 8, rounded to E4M3 and back: the FP8 values of kv_nvfp4_load_fp8 as four f16x2
// (low half = even element).  Every step is exact except the one E4M3 rounding.
__device__ __forceinline__ void kv_fp8_word(uint32_t w, uint32_t s2u, uint32_t *h)
{
    asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\t.reg .b32 t0, t1, t2, t3;\n\t.reg .b16 e0, e1, e2, e3;\n\t"
        "mov.b32 {b0, b1, b2, b3}, %4;\n\t"
        "cvt.rn.f16x2.e2m1x2 t0, b0;\n\t"
        "cvt.rn.f16x2.e2m1x2 t1, b1;\n\t"
        "cvt.rn.f16x2.e2m1x2 t2, b2;\n\t"
        "cvt.rn.f16x2.e2m1x2 t3, b3;\n\t"
        "mul.rn.f16x2 t0, t0, %5;\n\t"
        "mul.rn.f16x2 t1, t1, %5;\n\t"
        "mul.rn.f16x2 t2, t2, %5;\n\t"
        "mul.rn.f16x2 t3, t3, %5;\n\t"
        "cvt.rn.satfinite.e4m3x2.f16x2 e0, t0;\n\t"
        "cvt.rn.satfinite.e4m3x2.f16x2 e1, t1;\n\t"
        "cvt.rn.satfinite.e4m3x2.f16x2 e2, t2;\n\t"
        "cvt.rn.satfinite.e4m3x2.f16x2 e3, t3;\n\t"
        "cvt.rn.f16x2.e4m3x2 %0, e0;\n\t"
        "cvt.rn.f16x2.e4m3x2 %1, e1;\n\t"
        "cvt.rn.f16x2.e4m3x2 %2, e2;\n\t"
        "cvt.rn.f16x2.e4m3x2 %3, e3;\n\t}"
        : "=r"(h[0]), "=r"(h[1]), "=r"(h[2]), "=r"(h[3])
        : "r"(w), "r"(s2u));
}

// The block scale / 8 as an f16x2 bit pattern (exact in f16); bit conversions only, no
// type punning through pointers.
__device__ __forceinline__ uint32_t kv_scale_half2(uint32_t sf)
{
    const uint32_t u = __half_as_ushort(__float2half_rn(__fmul_rn(e4m3_value(sf), 0.125f)));
    return u | (u << 16);
}

__device__ __forceinline__ float2 half2_to_float2(uint32_t h)
{
    return make_float2(__half2float(__ushort_as_half((unsigned short)(h & 0xFFFFu))),
                       __half2float(__ushort_as_half((unsigned short)(h >> 16))));
}

template <int G>
__global__ void __launch_bounds__(KA_THREADS) kv_attn_split_kernel(KvAttnShape a)
{
    __shared__ __align__(16) float s_q[G * KA_D];
    // pass 1: scores [chunk][G]; after pass 2: the warps' partial outputs [warps][G][D]
    __shared__ __align__(16) float s_buf[(KA_CHUNK > KA_WARPS * KA_D ? KA_CHUNK : KA_WARPS * KA_D) * G];
    __shared__ float s_red[KA_WARPS][G];
    __shared__ float s_m[G], s_sum[G];

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int64_t bh = blockIdx.y, b = bh / a.H, h = bh - b * a.H;
    const int64_t l0 = (int64_t)blockIdx.x * KA_CHUNK;
    const int n = (int)min((int64_t)KA_CHUNK, a.L - l0);
    const float kscale = __fmul_rn(__fmul_rn(*a.gk, 8.0f), 0.08838834764831845f);  // 8 g_k / sqrt(128)

    const __nv_bfloat16 *qp = a.q + ((b * a.H + h) * G) * KA_D;
    for (int i = tid; i < G * KA_D; i += KA_THREADS)
        s_q[i] = __bfloat162float(qp[i]);
    __syncthreads();

    // ---- pass 1: scores, one thread per position
    const int64_t row0 = bh * a.Lcap + l0;
    float mloc[G];
#pragma unroll
    for (int j = 0; j < G; ++j)
        mloc[j] = -INFINITY;
    for (int t = tid; t < n; t += KA_THREADS) {
        const uint8_t *crow = a.kc + (row0 + t) * (KA_D / 2);
        const uint2 sc = ld_nc_v2(a.ks + (row0 + t) * (KA_D / 16));
        float acc[G];
#pragma unroll
        for (int j = 0; j < G; ++j)
            acc[j] = 0.0f;
#pragma unroll
        for (int hb = 0; hb < 4; ++hb) {  // 16 code bytes = two 16-value blocks
            const uint4 cw = ld_nc_v4(crow + 16 * hb);
            const uint32_t words[4] = {cw.x, cw.y, cw.z, cw.w};
#pragma unroll
            for (int wi = 0; wi < 4; ++wi) {
                const int blk = 2 * hb + (wi >> 1);
                const uint32_t sfb = ((blk < 4 ? sc.x : sc.y) >> (8 * (blk & 3))) & 0xFFu;
                const uint32_t s2u = kv_scale_half2(sfb);
                uint32_t hv[4];
                kv_fp8_word(words[wi], s2u, hv);
                float kv[8];
#pragma unroll
                for (int bi = 0; bi < 4; ++bi) {
                    const float2 f = half2_to_float2(hv[bi]);
                    kv[2 * bi] = f.x;
                    kv[2 * bi + 1] = f.y;
                }
                const int d = 32 * hb + 8 * wi;  // the word's first dimension
#pragma unroll
                for (int j = 0; j < G; ++j) {
                    const float4 q0 = *reinterpret_cast<const float4 *>(&s_q[j * KA_D + d]);
                    const float4 q1 = *reinterpret_cast<const float4 *>(&s_q[j * KA_D + d + 4]);
                    acc[j] = fmaf(q0.x, kv[0], acc[j]);
                    acc[j] = fmaf(q0.y, kv[1], acc[j]);
                    acc[j] = fmaf(q0.z, kv[2], acc[j]);
                    acc[j] = fmaf(q0.w, kv[3], acc[j]);
                    acc[j] = fmaf(q1.x, kv[4], acc[j]);
                    acc[j] = fmaf(q1.y, kv[5], acc[j]);
                    acc[j] = fmaf(q1.z, kv[6], acc[j]);
                    acc[j] = fmaf(q1.w, kv[7], acc[j]);
                }
            }
        }
#pragma unroll
        for (int j = 0; j < G; ++j) {
            const float sj = __fmul_rn(acc[j], kscale);
            s_buf[t * G + j] = sj;
            mloc[j] = fmaxf(mloc[j], sj);
        }
    }
    // chunk maximum per query head
#pragma unroll
    for (int j = 0; j < G; ++j) {
        float m = mloc[j];
#pragma unroll
        for (int o = 16; o; o >>= 1)
            m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
        if (lane == 0)
            s_red[warp][j] = m;
    }
    __syncthreads();
    if (tid < G) {
        float m = s_red[0][tid];
        for (int w = 1; w < KA_WARPS; ++w)
            m = fmaxf(m, s_red[w][tid]);
        s_m[tid] = m;
    }
    __syncthreads();
    // weights p = exp(s - m) in place, and their sum per query head
    float sloc[G];
#pragma unroll
    for (int j = 0; j < G; ++j)
        sloc[j] = 0.0f;
    for (int t = tid; t < n; t += KA_THREADS)
#pragma unroll
        for (int j = 0; j < G; ++j) {
            const float p = expf(s_buf[t * G + j] - s_m[j]);
            s_buf[t * G + j] = p;
            sloc[j] += p;
        }
#pragma unroll
    for (int j = 0; j < G; ++j) {
        float sj = sloc[j];
#pragma unroll
        for (int o = 16; o; o >>= 1)
            sj += __shfl_xor_sync(0xffffffffu, sj, o);
        if (lane == 0)
            s_red[warp][j] = sj;
    }
    __syncthreads();
    if (tid < G) {
        float sj = 0.0f;
        for (int w = 0; w < KA_WARPS; ++w)
            sj += s_red[w][tid];
        s_sum[tid] = sj;
    }

    // ---- pass 2: o = sum_l p_l v_l.  A warp takes two positions per step, a half-warp each;
    // lane l of a half owns dimensions 8l..8l+7 (one 32-bit code word, scale byte l/2)
    const int hl = lane & 15;
    float o[G][8];
#pragma unroll
    for (int j = 0; j < G; ++j)
#pragma unroll
        for (int i = 0; i < 8; ++i)
            o[j][i] = 0.0f;
    for (int t0 = 2 * warp; t0 < n; t0 += 2 * KA_WARPS) {
        const int t = t0 + (lane >> 4);
        if (t < n) {
            const int64_t row = row0 + t;
            const uint32_t w = *reinterpret_cast<const uint32_t *>(a.vc + row * (KA_D / 2) + 4 * hl);
            const uint32_t s2u = kv_scale_half2(a.vs[row * (KA_D / 16) + (hl >> 1)]);
            uint32_t hv[4];
            kv_fp8_word(w, s2u, hv);
            float v[8];
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                const float2 f = half2_to_float2(hv[k]);
                v[2 * k] = f.x;
                v[2 * k + 1] = f.y;
            }
#pragma unroll
            for (int j = 0; j < G; ++j) {
                const float p = s_buf[t * G + j];
#pragma unroll
                for (int i = 0; i < 8; ++i)
                    o[j][i] = fmaf(p, v[i], o[j][i]);
            }
        }
    }
    // the two halves hold the same dimensions for different positions
#pragma unroll
    for (int j = 0; j < G; ++j)
#pragma unroll
        for (int i = 0; i < 8; ++i)
            o[j][i] += __shfl_xor_sync(0xffffffffu, o[j][i], 16);
    __syncthreads();  // every thread has read the weights: reuse s_buf for the warps' outputs
    if (lane < 16)
#pragma unroll
        for (int j = 0; j < G; ++j)
#pragma unroll
            for (int i = 0; i < 8; ++i)
                s_buf[(warp * G + j) * KA_D + 8 * hl + i] = o[j][i];
    __syncthreads();
    float *dst = a.ws + ((bh * a.S + blockIdx.x) * G) * (KA_D + 2);
    for (int i = tid; i < G * KA_D; i += KA_THREADS) {
        const int j = i / KA_D, d = i - j * KA_D;
        float sum = 0.0f;
        for (int w = 0; w < KA_WARPS; ++w)  // fixed order: deterministic
            sum += s_buf[(w * G + j) * KA_D + d];
        dst[j * (KA_D + 2) + d] = sum;
    }
    if (tid < G) {
        dst[tid * (KA_D + 2) + KA_D] = s_m[tid];
        dst[tid * (KA_D + 2) + KA_D + 1] = s_sum[tid];
    }
}

// out[b, h*G + j, d] = 8 g_v * sum_s e^(m_s - M) o_s[d] / sum_s e^(m_s - M) l_s, M = max_s m_s.
__global__ void __launch_bounds__(KA_D) kv_attn_merge_kernel(KvAttnShape a, int G)
{
    const int64_t bhj = blockIdx.x, bh = bhj / G, j = bhj - bh * G;
    const int d = threadIdx.x;
    const float *src = a.ws + (bh * a.S * G + j) * (KA_D + 2);
    const int64_t step = (int64_t)G * (KA_D + 2);
    float M = -INFINITY;
    for (int s = 0; s < a.S; ++s)
        M = fmaxf(M, src[s * step + KA_D]);
    float num = 0.0f, den = 0.0f;
    for (int s = 0; s < a.S; ++s) {
        const float e = expf(src[s * step + KA_D] - M);
        num = fmaf(e, src[s * step + d], num);
        den = fmaf(e, src[s * step + KA_D + 1], den);
    }
    const float gv8 = __fmul_rn(*a.gv, 8.0f);
    a.out[bhj * KA_D + d] = __fmul_rn(__fdiv_rn(num, den), gv8);
}

}  // namespace fp4lin
