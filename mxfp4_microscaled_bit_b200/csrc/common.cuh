// common.cuh -- device helpers shared by the quantiser, KV and GEMM kernels
// (sm_100a only).  Every floating-point step that decides a code uses the
// explicitly rounded intrinsics (__fmul_rn, __fdiv_rn, __fadd_rn, __fsub_rn),
// so no multiply-add contraction can change a result.
#pragma once

#include <cstdint>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "../../include/fp4lin.h"

namespace fp4lin {

// One status word per device: the first device-side error since it was last
// read (FP4LIN_ERR_TIMEOUT, FP4LIN_ERR_OUT_OF_RANGE).  Read and cleared by
// fp4lin_device_status().
__device__ unsigned int g_device_status;

__device__ __forceinline__ void report_error(unsigned int code)
{
    atomicCAS(&g_device_status, 0u, code);
}

// ------------------------------------------------------------------ loads
// Programmatic dependent launch.  pdl_trigger: this CTA lets the next kernel in the stream
// (launched with programmatic stream serialisation) start early.  pdl_wait: block until the
// preceding kernel has completed and its writes are visible (returns at once when this
// kernel was launched without the attribute).
__device__ __forceinline__ void pdl_trigger() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

__device__ __forceinline__ uint4 ld_nc_v4(const void *p)
{
    uint4 r;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w) : "l"(p));
    return r;
}

// 32 bytes in one 256-bit load (p must be 32-byte aligned).
__device__ __forceinline__ void ld_nc_v8(const void *p, uint32_t *r)
{
    asm volatile("ld.global.nc.L1::no_allocate.v8.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7])
                 : "l"(p));
}

// 32 bytes as one 256-bit load when `wide` (32-byte aligned), else as two 128-bit loads.
__device__ __forceinline__ void ld_nc_32B(const void *p, bool wide, uint32_t *r)
{
    if (wide) {
        ld_nc_v8(p, r);
    } else {
        const uint4 a = ld_nc_v4(p), b = ld_nc_v4(static_cast<const uint8_t *>(p) + 16);
        r[0] = a.x; r[1] = a.y; r[2] = a.z; r[3] = a.w;
        r[4] = b.x; r[5] = b.y; r[6] = b.z; r[7] = b.w;
    }
}

__device__ __forceinline__ uint2 ld_nc_v2(const void *p)
{
    uint2 r;
    asm volatile("ld.global.nc.L1::no_allocate.v2.u32 {%0,%1}, [%2];" : "=r"(r.x), "=r"(r.y) : "l"(p));
    return r;
}

// 32 bytes in one 256-bit store (p must be 32-byte aligned).
__device__ __forceinline__ void st_v8(void *p, const uint32_t *v)
{
    asm volatile("st.global.v8.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8};" ::"l"(p), "r"(v[0]), "r"(v[1]), "r"(v[2]),
                 "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7])
                 : "memory");
}

__device__ __forceinline__ void st_v4(void *p, uint4 v)
{
    asm volatile("st.global.v4.u32 [%0], {%1,%2,%3,%4};" ::"l"(p), "r"(v.x), "r"(v.y), "r"(v.z), "r"(v.w)
                 : "memory");
}

// Eight bf16 (one 16-byte load) -> eight floats, exact.
__device__ __forceinline__ void bf16x8_to_f32(uint4 u, float *v)
{
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        v[2 * i] = __uint_as_float(w[i] << 16);
        v[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
    }
}

// ------------------------------------------------------------------ conversions
// E2M1 pair: round to nearest even, saturate at +-6, sign kept; `lo` goes to
// the low nibble (the even element), `hi` to the high nibble.
__device__ __forceinline__ uint32_t cvt_e2m1x2(float lo, float hi)
{
    uint32_t r;
    asm("{\n\t.reg .b8 t;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 t, %2, %1;\n\t"
        "cvt.u32.u8 %0, t;\n\t}"
        : "=r"(r) : "f"(lo), "f"(hi));
    return r;
}

// Eight floats -> four code bytes (element 0 in the lowest nibble).
__device__ __forceinline__ uint32_t pack_e2m1x8(const float *v)
{
    return cvt_e2m1x2(v[0], v[1]) | (cvt_e2m1x2(v[2], v[3]) << 8) | (cvt_e2m1x2(v[4], v[5]) << 16) |
           (cvt_e2m1x2(v[6], v[7]) << 24);
}

// E4M3 byte of a float: round to nearest even, saturate at +-448.
__device__ __forceinline__ uint32_t cvt_e4m3(float x)
{
    uint16_t r;
    asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(0.0f), "f"(x));
    return r & 0xFFu;
}

// Exact value of an E4M3 byte (finite codes; the scale path never makes NaN).
__device__ __forceinline__ float e4m3_value(uint32_t b)
{
    uint32_t e = (b >> 3) & 15u, m = b & 7u;
    float mag = e ? __uint_as_float(((e + 120u) << 23) | (m << 20)) : __fmul_rn((float)m, 0x1p-9f);
    return (b & 0x80u) ? -mag : mag;
}

// NVFP4 block scale from the block maximum and the FP32 tensor scale g:
// t = (amax/6)/g, sf = E4M3(t), d = dec(sf)*g, rcp = 1/d (0 when d is not positive).
// The one arithmetic every NVFP4 encoder in this library uses (nvfp4_block_scale below).

// 1/d for scale byte sf, d = dec(sf)*g; 0 when d is not positive.
__device__ __forceinline__ float nvfp4_block_rcp(uint32_t sf, float g)
{
    const float d = __fmul_rn(e4m3_value(sf), g);
    return d > 0.0f ? __fdiv_rn(1.0f, d) : 0.0f;
}


// The scale byte of nvfp4_block_scale, E4M3((amax/6)/g), from one product where that gives
// the same byte.  c6 = nvfp4_fast_c6(g) approximates 1/(6g) within 2 rounding errors, so
// ta = amax*c6 is within 3 relative rounding errors of amax/(6g) and the two-division
// quotient within 2: the two differ by less than 6 units in the last place of ta's binade.
// Rounding to E4M3 keeps mantissa bits 22..20 and rounds on bits 19..0; its midpoints are
// bits 19..0 = 0x80000.  So where ta is in the normal E4M3 range (>= 2^-6), finite, and more
// than 32 units from such a midpoint, both round to the same byte (near a power of two,
// where the two may sit in adjacent binades, both round to that power).  Everything else
// (midpoint neighbourhoods, the subnormal range, non-finite values, g outside the range
// nvfp4_fast_c6 accepts) takes the two divisions.
__device__ __forceinline__ float nvfp4_fast_c6(float g)
{
    return (g >= 0x1p-100f && g <= 0x1p+100f) ? __fdiv_rn(1.0f, __fmul_rn(6.0f, g)) : __int_as_float(0x7fc00000);
}

__device__ __forceinline__ uint32_t nvfp4_scale_code_fast(float amax, float g, float c6)
{
    const float ta = __fmul_rn(amax, c6);
    const int off = (int)(__float_as_uint(ta) & 0xFFFFFu) - 0x80000;
    if (ta >= 0x1p-6f && ta <= 0x1.fffffep+127f && (off > 32 || off < -32))
        return cvt_e4m3(ta);
    if (amax == 0.0f && c6 > 0.0f)  // (0/6)/g = 0 for a finite positive g
        return 0u;
    return cvt_e4m3(__fdiv_rn(__fdiv_rn(amax, 6.0f), g));
}

// NVFP4 block scale byte and rcp as defined above.  Callers that encode many blocks with one
// g get nvfp4_fast_c6(g) computed once (the compiler hoists it out of their loops).
__device__ __forceinline__ uint32_t nvfp4_block_scale(float amax, float g, float &rcp)
{
    const uint32_t sf = nvfp4_scale_code_fast(amax, g, nvfp4_fast_c6(g));
    rcp = nvfp4_block_rcp(sf, g);
    return sf;
}

// ------------------------------------------------------------------ packed binary32 pairs
// sm_100a executes two binary32 operations per instruction on register pairs (.f32x2); each
// half is the IEEE operation rounded to nearest, exactly as the scalar form.
__device__ __forceinline__ uint64_t f2_pack(float lo, float hi)
{
    uint64_t r;
    asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
    return r;
}

__device__ __forceinline__ void f2_unpack(uint64_t v, float &lo, float &hi)
{
    asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
}

__device__ __forceinline__ uint64_t f2_fma(uint64_t a, uint64_t b, uint64_t c)
{
    uint64_t d;
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
    return d;
}

__device__ __forceinline__ uint64_t f2_add(uint64_t a, uint64_t b)
{
    uint64_t d;
    asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
    return d;
}

__device__ __forceinline__ uint64_t f2_sub(uint64_t a, uint64_t b)
{
    uint64_t d;
    asm("sub.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
    return d;
}

__device__ __forceinline__ uint64_t f2_mul(uint64_t a, uint64_t b)
{
    uint64_t d;
    asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
    return d;
}

// ------------------------------------------------------------------ misc
__device__ __forceinline__ unsigned long long globaltimer_ns()
{
    unsigned long long t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

__device__ __forceinline__ uint32_t smem_u32(const void *p)
{
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

}  // namespace fp4lin
