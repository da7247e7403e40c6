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
// read once per group), staging the chunk in shared memory with bulk async
// copies; scores and the weighted sum of values run on the tensor cores
// (kv_attn_tc_kernel).  The chunk's maximum, sum and unnormalised output go to
// the workspace; kv_attn_merge_kernel combines the chunks.
#pragma once

#include "gemm_sm100.cuh"  // mbarrier, bulk-copy and bounded-wait helpers

namespace fp4lin {

constexpr int KA_D = 128;          // head dimension
constexpr int KA_THREADS = 128;  // four warps: four CTAs share an SM, so one loads while others compute
constexpr int KA_WARPS = KA_THREADS / 32;
constexpr int KA_CHUNK = 256;      // positions per CTA
constexpr int KA_GMAX = 8;         // query heads per kv head
constexpr int KA_SBUF = KA_CHUNK > KA_WARPS * KA_D ? KA_CHUNK : KA_WARPS * KA_D;  // score / output floats per head

// Dynamic shared memory of kv_attn_tc_kernel<G>: the chunk's K and V codes and scales, the
// score buffer, two mbarriers and an abort flag.
constexpr int ka_tc_smem(int G)
{
    return KA_CHUNK * (KA_D / 2) * 2 + KA_CHUNK * (KA_D / 16) * 2 + KA_SBUF * G * 4 + 2 * 8 + 16;
}

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

// The block scale / 8 in both halves of an f16x2, from a 16-bit word holding the scale byte
// twice: the hardware's E4M3 -> f16 conversion (exact: E4M3 is a subset of f16) and an exact
// multiply by 1/8 (the smallest result, 2^-12, is still a normal f16).
__device__ __forceinline__ uint32_t kv_scale_pair(uint32_t sf_twice)
{
    uint32_t h;
    asm("{\n\t.reg .b16 p;\n\tcvt.u16.u32 p, %1;\n\tcvt.rn.f16x2.e4m3x2 %0, p;\n\tmul.rn.f16x2 %0, %0, %2;\n\t}"
        : "=r"(h)
        : "r"(sf_twice), "r"(0x30003000u));  // 0x3000: 0.125 in f16
    return h;
}

__device__ __forceinline__ float2 half2_to_float2(uint32_t h)
{
    return make_float2(__half2float(__ushort_as_half((unsigned short)(h & 0xFFFFu))),
                       __half2float(__ushort_as_half((unsigned short)(h >> 16))));
}

// ------------------------------------------------------------------ tensor-core form
// D[16 x 8] += A[16 x 16] B[16 x 8], f16 operands, binary32 accumulation (the warp-level
// MMA: one side of these products is at most 8 query heads, too small for tcgen05).
// Fragments, with g = lane / 4, t = lane % 4: a0 = A[g][2t, 2t+1], a1 = A[g+8][2t, 2t+1],
// a2 = A[g][2t+8, 2t+9], a3 = A[g+8][2t+8, 2t+9]; b0 = B[2t, 2t+1][g], b1 = B[2t+8, 2t+9][g];
// d0, d1 = D[g][2t, 2t+1], d2, d3 = D[g+8][2t, 2t+1].
__device__ __forceinline__ void mma_16816x(float *d, uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3, uint32_t b0,
                                           uint32_t b1)
{
    asm volatile("mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
                 "{%0,%1,%2,%3};"
                 : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
                 : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// f16x2 bit pattern of two floats (round to nearest).
__device__ __forceinline__ uint32_t f16x2_bits(float lo, float hi)
{
    return (uint32_t)__half_as_ushort(__float2half_rn(lo)) | ((uint32_t)__half_as_ushort(__float2half_rn(hi)) << 16);
}

// Tensor-core form of the split kernel (same workspace output).  The CTA first stages its
// chunk in shared memory: the K and V code rows (contiguous per kv head) by one bulk async
// copy each, the scale rows by cooperative 8-byte loads, so every byte of the chunk is in
// flight at once and V arrives while pass 1 runs.
// Pass 1: scores^T by mma_16816x, A = K (16 positions as rows), B = q^T (8 heads as columns,
// G used), one 16-dimension slice per MMA.  A common permutation of the dimensions leaves
// the dot products unchanged; it is chosen so that a lane converts whole 32-bit code words:
// word 4r + t (dimensions 32r + 8t .. +7) feeds slice 2r with its first four dimensions and
// slice 2r+1 with its last four, and q is loaded in the same order.
// Pass 2: o += p v by mma_16816x, A = the weights of 16 positions for 8 heads in rows 0..7
// and the f16 rounding of what the f16 weights leave out in rows 8..15 (so p keeps ~22
// bits and one MMA accumulates both), B = V with the output dimensions permuted so that a
// lane needs 16 contiguous dimensions (8 code bytes, one scale) of each of its 4 rows; the
// code nibbles of two rows are interleaved before the conversion, so each converted pair is
// already a fragment register (one row per half).
template <int G>
__global__ void __launch_bounds__(KA_THREADS, 4) kv_attn_tc_kernel(KvAttnShape a)
{
    extern __shared__ __align__(128) uint8_t ka_smem[];
    uint8_t *s_kc = ka_smem;
    uint8_t *s_vc = s_kc + KA_CHUNK * (KA_D / 2);
    uint8_t *s_ks = s_vc + KA_CHUNK * (KA_D / 2);
    uint8_t *s_vs = s_ks + KA_CHUNK * (KA_D / 16);
    float *s_buf = reinterpret_cast<float *>(s_vs + KA_CHUNK * (KA_D / 16));  // [KA_SBUF * G]
    uint64_t *bars = reinterpret_cast<uint64_t *>(s_buf + KA_SBUF * G);
    volatile int *abort = reinterpret_cast<volatile int *>(bars + 2);
    __shared__ float s_red[KA_WARPS][G];
    __shared__ float s_m[G], s_sum[G];

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5, gq = lane >> 2, tg = lane & 3;
    const int64_t bh = blockIdx.y, b = bh / a.H, h = bh - b * a.H;
    const int64_t l0 = (int64_t)blockIdx.x * KA_CHUNK;
    const int n = (int)min((int64_t)KA_CHUNK, a.L - l0);
    const float kscale = __fmul_rn(__fmul_rn(*a.gk, 8.0f), 0.08838834764831845f);  // 8 g_k / sqrt(128)
    const int64_t row0 = bh * a.Lcap + l0;

    if (tid == 0) {
        mbar_init(&bars[0], 1);
        mbar_init(&bars[1], 1);
        *abort = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    __syncthreads();
    if (tid == 0) {
        const uint32_t bytes = (uint32_t)n * (KA_D / 2);  // a multiple of 64
        mbar_expect_tx(&bars[0], bytes);
        bulk_load(s_kc, a.kc + row0 * (KA_D / 2), bytes, &bars[0]);
        mbar_expect_tx(&bars[1], bytes);
        bulk_load(s_vc, a.vc + row0 * (KA_D / 2), bytes, &bars[1]);
    }
    for (int t = tid; t < n; t += KA_THREADS) {  // scale rows: 8-byte aligned only
        *reinterpret_cast<uint2 *>(s_ks + t * 8) = ld_nc_v2(a.ks + (row0 + t) * (KA_D / 16));
        *reinterpret_cast<uint2 *>(s_vs + t * 8) = ld_nc_v2(a.vs + (row0 + t) * (KA_D / 16));
    }
    // q^T as B fragments in the permuted dimension order (zero columns for heads >= G)
    uint32_t qb[8][2];
#pragma unroll
    for (int r = 0; r < 4; ++r) {
        if (gq < G) {
            const uint4 u = ld_nc_v4(a.q + ((b * a.H + h) * G + gq) * KA_D + 32 * r + 8 * tg);
            float f[8];
            bf16x8_to_f32(u, f);
            qb[2 * r][0] = f16x2_bits(f[0], f[1]);
            qb[2 * r][1] = f16x2_bits(f[2], f[3]);
            qb[2 * r + 1][0] = f16x2_bits(f[4], f[5]);
            qb[2 * r + 1][1] = f16x2_bits(f[6], f[7]);
        } else {
            qb[2 * r][0] = qb[2 * r][1] = qb[2 * r + 1][0] = qb[2 * r + 1][1] = 0u;
        }
    }
    wait_bar(&bars[0], 0, abort);
    __syncthreads();
    const bool ok = *abort == 0;

    // ---- pass 1: blocks of 16 positions; this lane loads positions t16 + gq and t16 + gq + 8
    float mloc[2] = {-INFINITY, -INFINITY};  // heads 2tg, 2tg + 1
    for (int t16 = warp * 16; ok && t16 < n; t16 += KA_WARPS * 16) {
        const int pa = t16 + gq, pb = pa + 8;
        uint32_t wa[4] = {0u, 0u, 0u, 0u}, wb[4] = {0u, 0u, 0u, 0u};
        uint2 sa = make_uint2(0u, 0u), sb = make_uint2(0u, 0u);
        if (pa < n) {
#pragma unroll
            for (int r = 0; r < 4; ++r)
                wa[r] = *reinterpret_cast<const uint32_t *>(s_kc + pa * (KA_D / 2) + 4 * (4 * r + tg));
            sa = *reinterpret_cast<const uint2 *>(s_ks + pa * 8);
        }
        if (pb < n) {
#pragma unroll
            for (int r = 0; r < 4; ++r)
                wb[r] = *reinterpret_cast<const uint32_t *>(s_kc + pb * (KA_D / 2) + 4 * (4 * r + tg));
            sb = *reinterpret_cast<const uint2 *>(s_ks + pb * 8);
        }
        float sc[4] = {0.0f, 0.0f, 0.0f, 0.0f};
#pragma unroll
        for (int r = 0; r < 4; ++r) {
            const uint32_t dup = (uint32_t)(2 * r + (tg >> 1)) * 0x11u;  // scale byte of dimensions 32r + 8t .., twice
            uint32_t ha[4], hb[4];
            kv_fp8_word(wa[r], kv_scale_pair(__byte_perm(sa.x, sa.y, dup)), ha);
            kv_fp8_word(wb[r], kv_scale_pair(__byte_perm(sb.x, sb.y, dup)), hb);
            mma_16816x(sc, ha[0], hb[0], ha[1], hb[1], qb[2 * r][0], qb[2 * r][1]);
            mma_16816x(sc, ha[2], hb[2], ha[3], hb[3], qb[2 * r + 1][0], qb[2 * r + 1][1]);
        }
        // sc[0], sc[1]: position pa, heads 2t, 2t+1; sc[2], sc[3]: position pb, same heads
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const int hd = 2 * tg + (e & 1), pos = (e < 2) ? pa : pb;
            if (hd < G && pos < n) {
                const float sj = __fmul_rn(sc[e], kscale);
                s_buf[pos * G + hd] = sj;
                mloc[e & 1] = fmaxf(mloc[e & 1], sj);
            }
        }
    }
    // chunk maximum per head: the 8 lanes holding a head (same t), then the warps
#pragma unroll
    for (int e = 0; e < 2; ++e) {
        float m = mloc[e];
        m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 4));
        m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 8));
        m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 16));
        if (gq == 0 && 2 * tg + e < G)
            s_red[warp][2 * tg + e] = m;
    }
    __syncthreads();
    if (tid < G) {
        float m = s_red[0][tid];
        for (int w = 1; w < KA_WARPS; ++w)
            m = fmaxf(m, s_red[w][tid]);
        s_m[tid] = m;
    }
    __syncthreads();
    // weights p = exp(s - m) in place, and their sum per head
    float sloc[G];
#pragma unroll
    for (int j = 0; j < G; ++j)
        sloc[j] = 0.0f;
    for (int t = tid; ok && t < n; t += KA_THREADS)
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
    wait_bar(&bars[1], 0, abort);
    __syncthreads();  // weights written, V landed
    if (tid < G) {
        float sj = 0.0f;
        for (int w = 0; w < KA_WARPS; ++w)
            sj += s_red[w][tid];
        s_sum[tid] = sj;
    }
    const bool ok2 = *abort == 0;

    // ---- pass 2: blocks of 16 positions; n-tile u of the output holds dimension 16c + u in
    // column c, so lane (gq, t) accumulates head gq at dimensions 32t + u and 32t + 16 + u
    // (rows gq: the f16 weights' part, rows gq + 8: the rest's part)
    float o[16][4];
#pragma unroll
    for (int u = 0; u < 16; ++u)
        o[u][0] = o[u][1] = o[u][2] = o[u][3] = 0.0f;
    for (int t16 = warp * 16; ok2 && t16 < n; t16 += KA_WARPS * 16) {
        const int rp[4] = {t16 + 2 * tg, t16 + 2 * tg + 1, t16 + 2 * tg + 8, t16 + 2 * tg + 9};
        float p4[4];
#pragma unroll
        for (int e = 0; e < 4; ++e)
            p4[e] = (gq < G && rp[e] < n) ? s_buf[rp[e] * G + gq] : 0.0f;
        const uint32_t ah0 = f16x2_bits(p4[0], p4[1]), ah2 = f16x2_bits(p4[2], p4[3]);
        const float2 b01 = half2_to_float2(ah0), b23 = half2_to_float2(ah2);
        const uint32_t al0 = f16x2_bits(__fsub_rn(p4[0], b01.x), __fsub_rn(p4[1], b01.y));
        const uint32_t al2 = f16x2_bits(__fsub_rn(p4[2], b23.x), __fsub_rn(p4[3], b23.y));
        // rows rp[0..3]: their code words (dimensions 16gq .. 16gq + 15) and scale bytes
        uint2 c[4];
        uint32_t sfb[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            c[e] = make_uint2(0u, 0u);
            sfb[e] = 0u;
            if (rp[e] < n) {
                c[e] = *reinterpret_cast<const uint2 *>(s_vc + rp[e] * (KA_D / 2) + 8 * gq);
                sfb[e] = s_vs[rp[e] * 8 + gq];
            }
        }
        // B fragments: for dimension 16gq + u, (row 2t, row 2t+1) in bv[0][u], (row 2t+8, row 2t+9) in
        // bv[1][u].  The two rows' code nibbles are interleaved first -- byte j of `ev` holds dimension
        // 2j of both rows, of `od` dimension 2j+1 -- so each conversion yields such a pair directly,
        // scaled by the two rows' own scales (low half: the first row).
        uint32_t bv[2][16];
#pragma unroll
        for (int pr = 0; pr < 2; ++pr) {
            const uint32_t s2u = kv_scale_pair(sfb[2 * pr] | (sfb[2 * pr + 1] << 8));
#pragma unroll
            for (int hw = 0; hw < 2; ++hw) {  // dimensions 0..7, then 8..15
                const uint32_t x0 = hw ? c[2 * pr].y : c[2 * pr].x, x1 = hw ? c[2 * pr + 1].y : c[2 * pr + 1].x;
                const uint32_t ev = (x0 & 0x0F0F0F0Fu) | ((x1 & 0x0F0F0F0Fu) << 4);
                const uint32_t od = ((x0 >> 4) & 0x0F0F0F0Fu) | (x1 & 0xF0F0F0F0u);
                uint32_t he[4], ho[4];
                kv_fp8_word(ev, s2u, he);
                kv_fp8_word(od, s2u, ho);
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    bv[pr][8 * hw + 2 * j] = he[j];
                    bv[pr][8 * hw + 2 * j + 1] = ho[j];
                }
            }
        }
#pragma unroll
        for (int u = 0; u < 16; ++u)
            mma_16816x(o[u], ah0, al0, ah2, al2, bv[0][u], bv[1][u]);
    }
    __syncthreads();  // every thread has read the weights: reuse s_buf for the warps' outputs
    if (gq < G)
#pragma unroll
        for (int u = 0; u < 16; ++u) {
            s_buf[(warp * G + gq) * KA_D + 32 * tg + u] = o[u][0] + o[u][2];
            s_buf[(warp * G + gq) * KA_D + 32 * tg + 16 + u] = o[u][1] + o[u][3];
        }
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
