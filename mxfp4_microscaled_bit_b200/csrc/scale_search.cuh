// scale_search.cuh -- NVFP4 quantisation with the block scale chosen to minimise
// the block's squared error (page "FP4 auf Blackwell: Was NVFP4 fuer lokale KI
// wirklich aendert", section "Was NVFP4 von frueheren 4-Bit-Formaten
// unterscheidet": the scaling algorithm picks the factor with the least mean
// squared error over the 16 values of a block).  An offline step for weights.
//
// The search is exhaustive: all 127 non-negative finite E4M3 scale codes.  For
// code c the scale is d = RN32(dec(c) * g), the reciprocal r = RN32(1/d) (0 when
// d = 0), the codes q_i = E2M1(RN32(x_i * r)), and the error the binary32 sum,
// in order i = 0..15, of RN32(RN32(x_i - RN32(e2m1(q_i) * d))^2).  The least
// error wins, ties to the smaller code.  Every step is explicitly rounded, so
// the choice -- an integer decided by floating point -- is the same one a
// binary32 evaluation of those formulas makes anywhere.
//
// Mapping: one warp per block; lane l evaluates the codes l, l+32, l+64, l+96
// (up to 126) and a butterfly takes the (error, code) minimum.  Every lane
// loads the same 32 bytes (one L1 transaction) and rotates them itself.
// Compute-bound: ~140 instructions per candidate (16 products, 8 E2M1 encodes,
// 4 f16x2 decodes, 16 f16-to-f32, 64 for the error sum), 127 candidates.
#pragma once

#include "quantize.cuh"

namespace fp4lin {

// Exact values of the 8 E2M1 codes of one code word (element 2i in the low nibble
// of byte i): each byte to f16x2 (low nibble -> low half), then each half to
// binary32; both conversions are exact, code 8 gives -0.
__device__ __forceinline__ void e2m1x8_values(uint32_t w, float *out)
{
    uint32_t h[4];
    asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\t"
        "mov.b32 {b0, b1, b2, b3}, %4;\n\t"
        "cvt.rn.f16x2.e2m1x2 %0, b0;\n\t"
        "cvt.rn.f16x2.e2m1x2 %1, b1;\n\t"
        "cvt.rn.f16x2.e2m1x2 %2, b2;\n\t"
        "cvt.rn.f16x2.e2m1x2 %3, b3;\n\t}"
        : "=r"(h[0]), "=r"(h[1]), "=r"(h[2]), "=r"(h[3]) : "r"(w));
#pragma unroll
    for (int k = 0; k < 4; ++k) {
        out[2 * k] = __half2float(__ushort_as_half((unsigned short)(h[k] & 0xFFFFu)));
        out[2 * k + 1] = __half2float(__ushort_as_half((unsigned short)(h[k] >> 16)));
    }
}

// Squared error of the 16 values v under E4M3 scale code c and tensor scale g.
__device__ __forceinline__ float block_sq_error(const float *v, uint32_t c, float g)
{
    const float d = __fmul_rn(e4m3_value(c), g);
    const float r = d > 0.0f ? __fdiv_rn(1.0f, d) : 0.0f;
    float err = 0.0f;
#pragma unroll
    for (int h = 0; h < 16; h += 8) {
        float p[8], e[8];
#pragma unroll
        for (int i = 0; i < 8; ++i)
            p[i] = __fmul_rn(v[h + i], r);
        e2m1x8_values(pack_e2m1x8(p), e);
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const float t = __fsub_rn(v[h + i], __fmul_rn(e[i], d));
            err = __fadd_rn(err, __fmul_rn(t, t));
        }
    }
    return err;
}

template <bool HAD, bool DYNAMIC>
__global__ void __launch_bounds__(QTHREADS)
    nvfp4_quant_mse_kernel(QuantShape q, float *g_io, const float *partials, int n_partials)
{
    __shared__ float s_g;
    __shared__ float red[QWARPS];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
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
            float g = __fdiv_rn(b, 2688.0f);  // 6 * 448, as the amax/6 quantiser
            if (!(g > 0.0f))
                g = 1.0f;
            s_g = g;
            if (blockIdx.x == 0)
                *g_io = g;
        }
    } else if (threadIdx.x == 0) {
        s_g = *g_io;
    }
    __syncthreads();
    const float g = s_g;
    const int64_t nblocks = q.rows * q.blocks_per_row;
    for (int64_t b = (int64_t)blockIdx.x * QWARPS + warp; b < nblocks; b += (int64_t)gridDim.x * QWARPS) {
        const int64_t r = b / q.blocks_per_row, c = b - r * q.blocks_per_row;
        uint32_t raw[8];
        ld_nc_32B(q.x + r * q.ld + c * 16, q.wide, raw);
        float v[16];
        nvfp4_block_values<HAD>(raw, v);
        float best = block_sq_error(v, (uint32_t)lane, g);
        uint32_t bc = (uint32_t)lane;
#pragma unroll
        for (int j = 1; j < 4; ++j) {
            const uint32_t cand = (uint32_t)(lane + 32 * j);
            if (cand <= 126u) {
                const float e = block_sq_error(v, cand, g);
                if (e < best) {  // candidates rise within a lane: strict keeps the smaller code
                    best = e;
                    bc = cand;
                }
            }
        }
#pragma unroll
        for (int o = 16; o; o >>= 1) {
            const float oe = __shfl_xor_sync(0xffffffffu, best, o);
            const uint32_t oc = __shfl_xor_sync(0xffffffffu, bc, o);
            if (oe < best || (oe == best && oc < bc)) {
                best = oe;
                bc = oc;
            }
        }
        if (lane == 0) {
            const float d = __fmul_rn(e4m3_value(bc), g);
            const float rr = d > 0.0f ? __fdiv_rn(1.0f, d) : 0.0f;
#pragma unroll
            for (int i = 0; i < 16; ++i)
                v[i] = __fmul_rn(v[i], rr);
            *reinterpret_cast<uint2 *>(q.codes + r * (q.cols / 2) + c * 8) =
                make_uint2(pack_e2m1x8(v), pack_e2m1x8(v + 8));
            q.scales[tc_offset(r, c, q.katoms)] = (uint8_t)bc;
        }
    }
}

}  // namespace fp4lin
