// gemm_sm100.cuh -- y = A W^T for NVFP4 / MXFP4 operands on the sm_100a
// block-scaled tensor cores (tcgen05.mma kind::mxf4nvf4 / kind::mxf4).
//
// The W4A4 layer runs its matrix products on the low-precision tensor cores
// (page "FP8, NVFP4 czy AWQ?", section "Dlaczego W8A8 i W4A16 to nie to
// samo?"); Blackwell's 5th-generation tensor cores apply the two-level NVFP4
// scaling natively (page "FP4 auf Blackwell", section "Was NVFP4 von
// frueheren 4-Bit-Formaten unterscheidet").
//
// Design (one CTA per SM, persistent over output tiles):
//   warp 0      TMA producer: code tiles by cp.async.bulk.tensor (128-byte
//               swizzle), scale atoms by cp.async.bulk, into a STAGES-deep
//               ring of shared-memory stages guarded by mbarriers.
//   warp 1      owns TMEM; the whole warp runs the issue loop (converged) and one
//               elected lane issues each instruction: the copies of a stage's
//               scale atoms into TMEM (tcgen05.cp 32x128b.warpx4) and the
//               block-scaled MMAs (128 x BN x 64 each) into a TMEM accumulator.
//               It waits on no mbarrier itself: between tensor-core instructions
//               such a wait stalls the issue far longer than a named barrier.
//   warps 2..9  epilogue: tcgen05.ld the accumulator into registers, release
//               it at once, then scale by g_a*g_w, round to bf16 and store
//               (256-bit stores; fp32 partials when K is split across CTAs).
//   warp 10     waiter: polls the accumulator and stage barriers in the MMA
//               warp's order, one step ahead of it, and meets it at a named
//               barrier after each, passing on a wait that gave up.
// Every mbarrier wait is bounded (WAIT_LIMIT_NS); on expiry the kernel
// records FP4LIN_ERR_TIMEOUT, raises a CTA abort flag, waits (bounded) for
// its own copies and MMAs, frees TMEM and returns.
#pragma once

#include <cuda.h>

#include "common.cuh"
#include "quantize.cuh"  // fwht, abs_max, tc_offset: the output quantisation encodes as the quantiser does

namespace fp4lin {

constexpr unsigned long long WAIT_LIMIT_NS = 1000000000ull;  // 1 s; a tile takes microseconds

// ------------------------------------------------------------------ PTX wrappers
__device__ __forceinline__ void mbar_init(uint64_t *bar, uint32_t count)
{
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}

__device__ __forceinline__ void mbar_expect_tx(uint64_t *bar, uint32_t bytes)
{
    asm volatile("mbarrier.arrive.expect_tx.release.cta.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)),
                 "r"(bytes)
                 : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t *bar)
{
    asm volatile("mbarrier.arrive.release.cta.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t *bar, uint32_t parity)
{
    uint32_t ok;
    asm volatile("{\n\t.reg .pred p;\n\t"
                 "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
                 "selp.u32 %0, 1, 0, p;\n\t}"
                 : "=r"(ok)
                 : "r"(smem_u32(bar)), "r"(parity)
                 : "memory");
    return ok != 0;
}

// Wait for the phase of `bar` with parity `parity`.  Returns false if it gave
// up: after limit_ns (records a timeout and raises *abort), or, when
// honor_abort, as soon as another role has raised *abort.
__device__ __noinline__ bool wait_bounded(uint64_t *bar, uint32_t parity, volatile int *abort, bool honor_abort,
                                          unsigned long long limit_ns = WAIT_LIMIT_NS)
{
    if (mbar_try_wait(bar, parity))
        return true;
    const unsigned long long t0 = globaltimer_ns();
    for (uint32_t it = 1;; ++it) {
        if (mbar_try_wait(bar, parity))
            return true;
        if ((it & 7u) == 0u) {
            if (honor_abort && *abort)
                return false;
            if (globaltimer_ns() - t0 > limit_ns) {
                report_error(FP4LIN_ERR_TIMEOUT);
                *abort = 1;
                return false;
            }
        }
    }
}

// One try_wait that may suspend the thread for up to 20 us while the phase is
// incomplete; it returns as soon as the phase completes.
__device__ __forceinline__ bool mbar_try_wait_hint(uint64_t *bar, uint32_t parity)
{
    uint32_t ok;
    asm volatile("{\n\t.reg .pred p;\n\t"
                 "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
                 "selp.u32 %0, 1, 0, p;\n\t}"
                 : "=r"(ok)
                 : "r"(smem_u32(bar)), "r"(parity), "r"(20000u)
                 : "memory");
    return ok != 0;
}

// Single-thread wait: the common case inline, the bounded slow path out of line.
__device__ __forceinline__ bool wait_bar(uint64_t *bar, uint32_t parity, volatile int *abort)
{
    if (mbar_try_wait_hint(bar, parity))
        return true;
    return wait_bounded(bar, parity, abort, true);
}

// Lane 0 waits, the warp learns the outcome.
__device__ __forceinline__ bool warp_wait(uint64_t *bar, uint32_t parity, volatile int *abort, int lane)
{
    int ok = 0;
    if (lane == 0)
        ok = wait_bar(bar, parity, abort) ? 1 : 0;
    return __shfl_sync(0xffffffffu, ok, 0) != 0;
}

// Wait for the phase of `bar` with parity `parity` with every lane of the warp polling it (no
// suspend hint): the form for warps that issue tcgen05 instructions as a converged warp and for
// the epilogue's accumulator wait.  Every lane sees the same barrier state, the same clock and
// the same flag, so the lanes stay together and agree on the outcome; lane 0 records a timeout.
// Returns false when the wait gave up (after WAIT_LIMIT_NS, or once another role raised *abort).
__device__ __forceinline__ bool warp_poll(uint64_t *bar, uint32_t parity, volatile int *abort, int lane)
{
    if (mbar_try_wait(bar, parity))
        return true;
    const unsigned long long t0 = globaltimer_ns();
    for (uint32_t it = 1;; ++it) {
        if (mbar_try_wait(bar, parity))
            return true;
        if ((it & 7u) == 0u) {
            if (*abort)
                return false;
            if (globaltimer_ns() - t0 > WAIT_LIMIT_NS) {
                if (lane == 0) {
                    report_error(FP4LIN_ERR_TIMEOUT);
                    *abort = 1;
                }
                return false;
            }
        }
    }
}

// The MMA warp and its waiter warp meet at named barrier 2 (64 threads); the result is true
// when either side passed true (a wait that gave up).  A named barrier costs the issuing warp
// far less than an mbarrier wait of its own between its tensor-core instructions.
__device__ __forceinline__ bool meet_or(bool fail)
{
    uint32_t r;
    asm volatile("{\n\t.reg .pred p, q;\n\tsetp.ne.u32 q, %1, 0;\n\tbar.red.or.pred p, 2, 64, q;\n\t"
                 "selp.u32 %0, 1, 0, p;\n\t}"
                 : "=r"(r)
                 : "r"((uint32_t)fail)
                 : "memory");
    return r != 0;
}

// Diagnostic of the expiry path of wait_bounded, the wait every pipeline role
// uses.  Two single-arrival barriers; lane 0 of warp w waits on barrier w.
// Warp 1 waits with limit_ns, warp 0 with the kernel limit but honouring the
// CTA abort flag, as the GEMM's roles do.  With arrive != 0 each barrier gets
// its arrival first and both waits succeed.  Without it nothing ever arrives:
// warp 1's wait expires (records FP4LIN_ERR_TIMEOUT, raises the flag) and
// warp 0's gives up on seeing the flag.  Every loop ends by the clock.
// result[w] = 1 if warp w's wait saw the phase complete, else 0;
// result[2 + w] = nanoseconds warp w spent waiting.
__global__ void __launch_bounds__(64, 1)
    wait_selftest_kernel(unsigned long long limit_ns, int arrive, unsigned long long *result)
{
    __shared__ __align__(8) uint64_t bars[2];
    __shared__ int abort_flag;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (threadIdx.x == 0) {
        mbar_init(&bars[0], 1);
        mbar_init(&bars[1], 1);
        abort_flag = 0;
    }
    __syncthreads();
    if (lane != 0)
        return;
    if (arrive)
        mbar_arrive(&bars[warp]);
    const unsigned long long t0 = globaltimer_ns();
    const bool ok = wait_bounded(&bars[warp], 0, &abort_flag, warp == 0, warp == 1 ? limit_ns : WAIT_LIMIT_NS);
    result[2 + warp] = globaltimer_ns() - t0;
    result[warp] = ok ? 1ull : 0ull;
}

__device__ __forceinline__ void tma_load_2d(void *dst, const CUtensorMap *map, uint64_t *bar, int x, int y)
{
    asm volatile("cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
                 " [%0], [%1, {%3, %4}], [%2];" ::"r"(smem_u32(dst)),
                 "l"(map), "r"(smem_u32(bar)), "r"(x), "r"(y)
                 : "memory");
}

__device__ __forceinline__ void bulk_load(void *dst, const void *src, uint32_t bytes, uint64_t *bar)
{
    asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
                     smem_u32(dst)),
                 "l"(src), "r"(bytes), "r"(smem_u32(bar))
                 : "memory");
}

__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

__device__ __forceinline__ void tc_commit(uint64_t *bar)
{
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_u32(bar))
                 : "memory");
}

__device__ __forceinline__ void tc_cp_atom(uint32_t taddr, uint64_t sdesc)
{
    asm volatile("tcgen05.cp.cta_group::1.32x128b.warpx4 [%0], %1;" ::"r"(taddr), "l"(sdesc) : "memory");
}

// The same three instructions for a converged warp: every lane executes the call with the
// same operands and one lane, chosen by elect.sync inside the asm, issues the instruction.
// Issued this way the scale copies cost the tensor pipe almost nothing (a 128 x 256 x 64 MMA
// with its three copies takes ~132 cycles, against ~225 when one lane of an otherwise idle
// warp issues the same sequence: the operands then reach the issue unit through per-thread
// registers).  Every lane of the warp must make the call.
__device__ __forceinline__ void tc_cp_atom_w(uint32_t taddr, uint64_t sdesc)
{
    asm volatile("{\n\t.reg .pred e;\n\telect.sync _|e, 0xffffffff;\n\t"
                 "@e tcgen05.cp.cta_group::1.32x128b.warpx4 [%0], %1;\n\t}" ::"r"(taddr),
                 "l"(sdesc)
                 : "memory");
}

__device__ __forceinline__ void tc_commit_w(uint64_t *bar)
{
    asm volatile("{\n\t.reg .pred e;\n\telect.sync _|e, 0xffffffff;\n\t"
                 "@e tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];\n\t}" ::"r"(
                     smem_u32(bar))
                 : "memory");
}

template <bool NV>
__device__ __forceinline__ void tc_mma_w(uint32_t d, uint64_t a, uint64_t b, uint32_t idesc, uint32_t sfa,
                                         uint32_t sfb, uint32_t acc)
{
    if constexpr (NV) {
        asm volatile("{\n\t.reg .pred p, e;\n\tsetp.ne.b32 p, %4, 0;\n\telect.sync _|e, 0xffffffff;\n\t"
                     "@e tcgen05.mma.cta_group::1.kind::mxf4nvf4.block_scale.block16 [%0], %1, %2, %3, [%5], [%6], p;\n\t}" ::"r"(
                         d),
                     "l"(a), "l"(b), "r"(idesc), "r"(acc), "r"(sfa), "r"(sfb)
                     : "memory");
    } else {
        asm volatile("{\n\t.reg .pred p, e;\n\tsetp.ne.b32 p, %4, 0;\n\telect.sync _|e, 0xffffffff;\n\t"
                     "@e tcgen05.mma.cta_group::1.kind::mxf4.block_scale.block32 [%0], %1, %2, %3, [%5], [%6], p;\n\t}" ::"r"(
                         d),
                     "l"(a), "l"(b), "r"(idesc), "r"(acc), "r"(sfa), "r"(sfb)
                     : "memory");
    }
}

template <bool NV>
__device__ __forceinline__ void tc_mma(uint32_t d, uint64_t a, uint64_t b, uint32_t idesc, uint32_t sfa, uint32_t sfb,
                                       uint32_t acc)
{
    if constexpr (NV) {
        asm volatile("{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
                     "tcgen05.mma.cta_group::1.kind::mxf4nvf4.block_scale.block16 [%0], %1, %2, %3, [%5], [%6], p;\n\t}" ::"r"(
                         d),
                     "l"(a), "l"(b), "r"(idesc), "r"(acc), "r"(sfa), "r"(sfb)
                     : "memory");
    } else {
        asm volatile("{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
                     "tcgen05.mma.cta_group::1.kind::mxf4.block_scale.block32 [%0], %1, %2, %3, [%5], [%6], p;\n\t}" ::"r"(
                         d),
                     "l"(a), "l"(b), "r"(idesc), "r"(acc), "r"(sfa), "r"(sfb)
                     : "memory");
    }
}

// 32 consecutive accumulator columns of this thread's TMEM lane, waited for
// inside the same asm so no register is read early.
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, float *v)
{
    uint32_t r[32];
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x32.b32 "
                 "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
                 "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];\n\t"
                 "tcgen05.wait::ld.sync.aligned;"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
                   "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]),
                   "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]),
                   "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]),
                   "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
                 : "r"(taddr)
                 : "memory");
#pragma unroll
    for (int i = 0; i < 32; ++i)
        v[i] = __uint_as_float(r[i]);
}

// 8 consecutive accumulator columns of this thread's TMEM lane.
__device__ __forceinline__ void tmem_ld8(uint32_t taddr, float *v)
{
    uint32_t r[8];
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];\n\t"
                 "tcgen05.wait::ld.sync.aligned;"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7])
                 : "r"(taddr)
                 : "memory");
#pragma unroll
    for (int i = 0; i < 8; ++i)
        v[i] = __uint_as_float(r[i]);
}

// Shared-memory matrix descriptor, K-major with the 128-byte swizzle: rows of
// 128 bytes, 8-row groups 1024 bytes apart (stride byte offset), version 1.
__device__ __forceinline__ uint64_t desc_sw128(uint32_t saddr)
{
    return (uint64_t)((saddr & 0x3FFFFu) >> 4) | ((uint64_t)1 << 16) | ((uint64_t)(1024 >> 4) << 32) |
           ((uint64_t)1 << 46) | ((uint64_t)2 << 61);
}

// Descriptor of one 512-byte scale atom as the tcgen05.cp source: 32 rows of
// 16 bytes, no swizzle, 8-row core matrices 128 bytes apart.
__device__ __forceinline__ uint64_t desc_sf_atom(uint32_t saddr)
{
    return (uint64_t)((saddr & 0x3FFFFu) >> 4) | ((uint64_t)(128 >> 4) << 32) | ((uint64_t)1 << 46);
}

// ------------------------------------------------------------------ configuration
// SWAP: the MMA computes y^T = W A^T -- its M operand is W (128 rows per tile), its N
// operand the few activation rows (BN = 16) -- and the epilogue writes y transposed.  For
// decode-sized M every tile then streams 128 weight rows instead of padding M to 128.
// FUSEQ (decode, with SWAP): the activations arrive as bf16 and the epilogue warps quantise
// them into each stage themselves (NVFP4, the quantiser's arithmetic), instead of TMA loading
// codes and scales a separate quantiser wrote.
template <int BN_, bool NV_, bool SWAP_ = false, bool FUSEQ_ = false>
struct GemmCfg {
    static constexpr int BN = BN_;
    static constexpr bool NV = NV_;                       // NVFP4 (16-blocks, E4M3) or MXFP4 (32-blocks, E8M0)
    static constexpr bool SWAP = SWAP_;
    static constexpr bool FUSEQ = FUSEQ_;
    static constexpr int BM = 128;
    static constexpr int BK = 256;                        // elements per stage (128 code bytes per row)
    static constexpr int MMA_K = 64;
    static constexpr int APK = NV ? BK / 64 : BK / 128;   // scale atoms per 128 rows per stage
    // 128-row scale tiles per B stage: a tile of BN rows starting at row BN * nt meets at most
    // this many of the weight scale layout's 128-row tiles
    static constexpr int RT = BN <= 128 ? 1 : (BN + 127) / 128;
    static constexpr int A_BYTES = BM * 128;
    static constexpr int B_BYTES = BN * 128;
    static constexpr int SFA_BYTES = APK * 512;
    static constexpr int SFB_BYTES = RT * APK * 512;
    static constexpr int STAGE_BYTES = A_BYTES + B_BYTES + SFA_BYTES + SFB_BYTES;
    static constexpr int STAGES = (220 * 1024) / STAGE_BYTES > 8 ? 8 : (220 * 1024) / STAGE_BYTES;
    static constexpr int NUM_ACC = BN >= 256 ? 1 : 2;
    static constexpr int SFA_COLS = APK * 4, SFB_COLS = RT * APK * 4;
    static constexpr int SF_COLS = SFA_COLS + SFB_COLS;          // one stage's scales
    static constexpr int TMEM_USED = NUM_ACC * BN + 2 * SF_COLS;  // scales double-buffered across k-tiles
    static constexpr int TMEM_COLS = TMEM_USED <= 32 ? 32 : TMEM_USED <= 64 ? 64 : TMEM_USED <= 128 ? 128
                                   : TMEM_USED <= 256 ? 256 : 512;
    static constexpr int EPI_WARPS = 8;
    static constexpr int WAITER_WARP = 2 + EPI_WARPS;    // waits on the MMA warp's barriers
    static constexpr int THREADS = 64 + EPI_WARPS * 32 + 32;
    static constexpr int COLS_PER_WARP = BN / 2;
    static constexpr int BAR_BYTES = 256;
    static constexpr int SMEM_BYTES = STAGES * STAGE_BYTES + BAR_BYTES + 1024;
    // instruction descriptor: A/B E2M1 (1), dense, K-major, N>>3, scale type, M>>4
    static constexpr uint32_t IDESC = (1u << 7) | (1u << 10) | ((uint32_t)(BN >> 3) << 17) |
                                      ((NV ? 0u : 1u) << 23) | ((uint32_t)(BM >> 4) << 24);
    static_assert(TMEM_USED <= 512, "TMEM overflow");
    static_assert(SMEM_BYTES <= 232448, "shared memory overflow");
    static_assert(STAGES >= 2, "pipeline too shallow");
    static_assert(!SWAP || BN == 16, "the swapped form serves at most 16 activation rows");
    static_assert(!FUSEQ || (SWAP && NV), "the fused activation quantiser is the NVFP4 decode form's");
    static_assert(SWAP || COLS_PER_WARP % 32 == 0, "epilogue loads 32 columns at a time");
};

struct GemmParams {
    int raster;                 // m-tiles per raster group (num_mt: plain m-fastest order)
    const uint8_t *sfa, *sfb;   // tensor-core scale layouts of A [M, K/blk] and W [N, K/blk]
    const float *g_a, *g_w;     // NVFP4 tensor scales (null for MXFP4)
    __nv_bfloat16 *y;
    float *ws;                  // split-K partials [splits, M, ldw] (splits > 1)
    int64_t M, N, K, ldy, ldw;
    int64_t katoms;             // scale atoms per 128-row tile along K
    int64_t sfb_rtiles;         // 128-row tiles of the B scale buffer (ceil(N / 128))
    int num_mt, num_nt, nk, kps, splits;
    int64_t work;               // num_mt * num_nt * splits
    // Optional NVFP4 quantisation of the bf16 output for the next layer (qc null: off):
    // codes [M, N/2], scales tensor-core layout of [M, N/16] (qkatoms = N/64 atoms per
    // row tile), static tensor scale *qg, 16-wide rotation when qhad.  y may then be null.
    uint8_t *qc, *qs;
    const float *qg;
    int qhad;
    int64_t qkatoms;
    // FUSEQ: the bf16 activations [p.N rows, K] (row stride ld_xa), rotated by H_16/4 when
    // xhad.  Their tensor scale is *g_w (xnpart == 0: static; the swapped form's activation
    // slot), or amax / 2688 written to g_a_out by CTA 0, the amax taken over the xnpart partial
    // maxima at xpart (xnpart > 0) or by every CTA over all the activations (xnpart < 0).
    const __nv_bfloat16 *xa;
    int64_t ld_xa;
    // A operand in tile order (non-null: loaded by plain bulk copies instead of TMA): tile
    // (mt, kt) -- 128 rows x 128 code bytes, already in the 128-byte-swizzled image the MMA
    // reads -- is the 16 KB at ((mt * nk + kt) * 16384).  For decode weights, prepared once.
    const uint8_t *a_tiled;
    int xhad;
    const float *xpart;
    int xnpart;
    float *g_a_out;
};

// NVFP4-encode 16 consecutive output values of one row held by this thread (already
// rounded to bf16): rotation, block scale, codes -- the quantiser's arithmetic.
__device__ __forceinline__ void quantize_out_block(const float *y16, int64_t m, int64_t nb, uint8_t *qc,
                                                   uint8_t *qs, float g, bool had, int64_t N, int64_t katoms)
{
    float w[16];
#pragma unroll
    for (int j = 0; j < 16; ++j)
        w[j] = y16[j];
    if (had) {
        fwht<16>(w);
#pragma unroll
        for (int j = 0; j < 16; ++j)
            w[j] = __fmul_rn(w[j], 0.25f);
    }
    float rcp;
    const uint32_t sf = nvfp4_block_scale(abs_max<16>(w), g, rcp);
#pragma unroll
    for (int j = 0; j < 16; ++j)
        w[j] = __fmul_rn(w[j], rcp);
    *reinterpret_cast<uint2 *>(qc + m * (N / 2) + nb / 2) = make_uint2(pack_e2m1x8(w), pack_e2m1x8(w + 8));
    qs[tc_offset(m, nb / 16, katoms)] = (uint8_t)sf;
}

// The 16-point rotation of a block spread over L lanes (16/L consecutive values per lane,
// lanes of a block consecutive): butterfly strides 1, 2, ... in order, the pair (u, w)
// becoming (u + w, u - w); strides >= 16/L pair values of lanes lane ^ (stride / (16/L)).
template <int L>
__device__ __forceinline__ void fwht16_lanes(float *w)
{
    constexpr int E = 16 / L;  // values per lane
#pragma unroll
    for (int h = 1; h < E; h <<= 1)
#pragma unroll
        for (int i = 0; i < E; ++i)
            if ((i & h) == 0) {
                const float u = w[i], x = w[i + h];
                w[i] = __fadd_rn(u, x);
                w[i + h] = __fsub_rn(u, x);
            }
    const int lane = threadIdx.x & 31;
#pragma unroll
    for (int h = 1; h < L; h <<= 1) {
        const bool upper = (lane & h) != 0;
#pragma unroll
        for (int i = 0; i < E; ++i) {
            const float o = __shfl_xor_sync(0xffffffffu, w[i], h);
            w[i] = upper ? __fsub_rn(o, w[i]) : __fadd_rn(w[i], o);  // upper: (lower u) - (own w)
        }
    }
}

// MMAs (64 values of K each) in k-tile kt: 4, or fewer in a last partial tile.
template <class C>
__device__ __forceinline__ int stage_mmas(int64_t K, int kt)
{
    const int64_t left = (K - (int64_t)kt * C::BK) / C::MMA_K;
    return left < C::BK / C::MMA_K ? (int)left : C::BK / C::MMA_K;
}

// Work item w -> (m tile, n tile, K split).  Tiles are walked in groups of
// `raster` m-tiles: inside a group m runs fastest, then n, so the CTAs that
// run at the same time share a few A and B tiles in L2 instead of one B tile
// being read by every CTA at once.
__device__ __forceinline__ void tile_coords(const GemmParams &p, int64_t w, int &mt, int &nt, int &sp)
{
    const int64_t tiles_mn = (int64_t)p.num_mt * p.num_nt;
    sp = (int)(w / tiles_mn);
    const int64_t t = w - (int64_t)sp * tiles_mn;
    const int64_t group = (int64_t)p.raster * p.num_nt;
    const int64_t g = t / group, idx = t - g * group;
    const int64_t m0 = g * p.raster;
    const int64_t rows = min((int64_t)p.raster, (int64_t)p.num_mt - m0);
    mt = (int)(m0 + idx % rows);
    nt = (int)(idx / rows);
}

// FUSEQ: one epilogue thread (et = 0..255) owns activation block (row et / 16, block et % 16)
// of every k-tile.  fuseq_load fetches its 16 bf16 values (nothing outside the activations);
// fuseq_store quantises them into the stage: the 8 code bytes at their place in the
// 128-byte-swizzled 16-row operand tile (16-byte chunk index XOR row % 8), the scale byte at
// its place in the row's scale lines (fuseq_store); blocks outside the activations get
// zeros.  The same arithmetic as nvfp4_quant_kernel, so the codes and scales are those it
// would write.
struct FuseRaw {
    uint4 u0, u1;
};

__device__ __forceinline__ bool fuseq_valid(const GemmParams &p, int kt, int et)
{
    return (et >> 4) < p.N && (int64_t)kt * 256 + 16 * (et & 15) < p.K;
}

__device__ __forceinline__ void fuseq_load(const GemmParams &p, int kt, int et, FuseRaw &r)
{
    if (fuseq_valid(p, kt, et)) {
        const __nv_bfloat16 *src = p.xa + (et >> 4) * p.ld_xa + (int64_t)kt * 256 + 16 * (et & 15);
        r.u0 = ld_nc_v4(src);
        r.u1 = ld_nc_v4(src + 8);
    }
}

__device__ __forceinline__ void fuseq_store(const GemmParams &p, uint8_t *sB, uint8_t *sSFB, int kt, int et,
                                            const FuseRaw &x, float xg, float c6, const float *s_rcp)
{
    const int r = et >> 4, c = et & 15;
    uint32_t lo = 0u, hi = 0u, sf = 0u;
    if (fuseq_valid(p, kt, et)) {
        const uint32_t raw[8] = {x.u0.x, x.u0.y, x.u0.z, x.u0.w, x.u1.x, x.u1.y, x.u1.z, x.u1.w};
        float v[16];
        if (p.xhad)
            nvfp4_block_values<true>(raw, v);
        else
            nvfp4_block_values<false>(raw, v);
        // nvfp4_block_scale's byte and multiplier without a division: c6 and the table of
        // 1/(dec(sf) xg) over the 256 scale bytes are computed once per CTA
        sf = nvfp4_scale_code_fast(abs_max<16>(v), xg, c6);
        scale_packed<16>(v, s_rcp[sf]);
        lo = pack_e2m1x8(v);
        hi = pack_e2m1x8(v + 8);
    }
    *reinterpret_cast<uint2 *>(sB + r * 128 + (((c >> 1) ^ (r & 7)) << 4) + ((c & 1) << 3)) = make_uint2(lo, hi);
    // two k-blocks' scales per 16-byte line of row r: k-blocks 2h and 2h+1 at bytes 0..3 and
    // 8..11 of line r of the 512-byte region h, so one copy serves two MMAs, which read their
    // scales at TMEM column offsets 0 and 2 of it (offsets the 64-row B tiles use as well)
    const int kb = c >> 2;
    sSFB[(kb >> 1) * 512 + r * 16 + (kb & 1) * 8 + (c & 3)] = (uint8_t)sf;
}

// k-tiles whose activations are fetched ahead of the one being encoded
constexpr int FUSEQ_PREFETCH = 3;

template <class C>
__global__ void __launch_bounds__(C::THREADS, 1)
    fp4_gemm_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB, GemmParams p)
{
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
    uint8_t *bar_area = smem + C::STAGES * C::STAGE_BYTES;
    uint64_t *full = reinterpret_cast<uint64_t *>(bar_area);
    uint64_t *empty = full + C::STAGES;
    uint64_t *acc_full = empty + C::STAGES;
    uint64_t *acc_empty = acc_full + C::NUM_ACC;
    uint64_t *done_bar = acc_empty + C::NUM_ACC;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(done_bar + 1);
    volatile int *abort = reinterpret_cast<volatile int *>(tmem_slot + 1);
    volatile int *epi_ok = abort + 1;  // [2]: outcome of the accumulator wait, per tile parity

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        pdl_trigger();  // the split-K reduction may launch now; it waits for this grid to finish
        for (int s = 0; s < C::STAGES; ++s) {
            mbar_init(&full[s], C::FUSEQ ? 1 + C::EPI_WARPS : 1);
            mbar_init(&empty[s], 1);
        }
        for (int a = 0; a < C::NUM_ACC; ++a) {
            mbar_init(&acc_full[a], 1);
            mbar_init(&acc_empty[a], C::EPI_WARPS);
        }
        mbar_init(done_bar, 1);
        *abort = 0;
        epi_ok[2] = 0;  // the epilogue warps' failure flag
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (warp == 1) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tmem_slot)),
                     "r"((uint32_t)C::TMEM_COLS)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;

    if (warp == 0) {
        // ---------------------------------------------------------------- producer (one thread)
        if (lane == 0) {
            int stage = 0;
            uint32_t phase = 0;
            uint32_t armed = 0, armed_phase = 0;  // bit s: stage s armed at least once / parity of its last arm
            bool ok = true;
            for (int64_t w = blockIdx.x; w < p.work && ok; w += gridDim.x) {
                int mt, nt, sp;
                tile_coords(p, w, mt, nt, sp);
                const int kt0 = sp * p.kps, kt1 = min(p.nk, kt0 + p.kps);
                const int64_t brt0 = ((int64_t)nt * C::BN) / 128;
                for (int kt = kt0; kt < kt1; ++kt) {
                    if (!(ok = wait_bar(&empty[stage], phase ^ 1u, abort)))
                        break;
                    const int mmas = stage_mmas<C>(p.K, kt);
                    const int atoms = C::NV ? mmas : (mmas + 1) / 2;
                    uint8_t *sA = smem + stage * C::STAGE_BYTES;
                    uint8_t *sB = sA + C::A_BYTES;
                    uint8_t *sSFA = sB + C::B_BYTES;
                    uint8_t *sSFB = sSFA + C::SFA_BYTES;
                    // B scale row-tiles of this stage that exist (the last tile may reach past them)
                    const int rts = (int)min((int64_t)C::RT, p.sfb_rtiles - brt0);
                    if constexpr (C::FUSEQ)  // the activation half of the stage comes from the epilogue warps
                        mbar_expect_tx(&full[stage], C::A_BYTES + atoms * 512);
                    else
                        mbar_expect_tx(&full[stage], C::A_BYTES + C::B_BYTES + atoms * 512 * (1 + rts));
                    armed |= 1u << stage;
                    armed_phase = (armed_phase & ~(1u << stage)) | (phase << stage);
                    if (p.a_tiled)
                        bulk_load(sA, p.a_tiled + ((int64_t)mt * p.nk + kt) * C::A_BYTES, C::A_BYTES, &full[stage]);
                    else
                        tma_load_2d(sA, &tmA, &full[stage], kt * 128, mt * C::BM);
                    const int64_t ka = (int64_t)kt * C::APK;
                    bulk_load(sSFA, p.sfa + ((int64_t)mt * p.katoms + ka) * 512, atoms * 512, &full[stage]);
                    if constexpr (!C::FUSEQ) {
                        tma_load_2d(sB, &tmB, &full[stage], kt * 128, nt * C::BN);
#pragma unroll
                        for (int rt = 0; rt < C::RT; ++rt)
                            if (rt < rts)
                                bulk_load(sSFB + rt * C::APK * 512, p.sfb + ((brt0 + rt) * p.katoms + ka) * 512,
                                          atoms * 512, &full[stage]);
                    }
                    if (++stage == C::STAGES) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
            }
            // drain: every copy this CTA started has landed before shared memory is released
            for (int s = 0; s < C::STAGES; ++s)
                if (armed & (1u << s))
                    wait_bounded(&full[s], (armed_phase >> s) & 1u, abort, false);
        }
        __syncwarp();
    } else if (warp == 1) {
        // ---------------------------------------------------------------- MMA issuer (one warp)
        // The whole warp runs the loop on warp-uniform values and one elected lane issues each
        // tcgen05 instruction.  The waiter warp does the barrier waits; this warp meets it at
        // named barrier 2 before each tile and each k-tile.
        {
            const uint32_t tm_sf = tmem_base + C::NUM_ACC * C::BN;
            int stage = 0;
            uint32_t phase = 0, sfsel = 0;  // sfsel alternates the scale region every k-tile
            int it = 0;
            bool ok = true;
            for (int64_t w = blockIdx.x; w < p.work && ok; w += gridDim.x, ++it) {
                int mt, nt, sp;
                tile_coords(p, w, mt, nt, sp);
                const int kt0 = sp * p.kps, kt1 = min(p.nk, kt0 + p.kps);
                const int acc = it % C::NUM_ACC;
                const uint32_t acc_phase = (uint32_t)(it / C::NUM_ACC) & 1u;
                if (!(ok = !meet_or(false)))  // the waiter saw the accumulator free
                    break;
                tc_fence_after();  // order the epilogue's TMEM reads before these MMAs
                const uint32_t d_tmem = tmem_base + acc * C::BN;
                // a B tile starting 64 rows into a 128-row scale atom (BN = 64) reads its scales
                // from the atom's column +2: 32 rows per TMEM column of the atom
                const uint32_t sfb_off = (uint32_t)((((int64_t)nt * C::BN) & 127) >> 5);
                for (int kt = kt0; kt < kt1; ++kt) {
                    if (!(ok = !meet_or(false)))  // the waiter saw the stage full
                        break;
                    const int mmas = stage_mmas<C>(p.K, kt);
                    uint8_t *sA = smem + stage * C::STAGE_BYTES;
                    uint8_t *sB = sA + C::A_BYTES;
                    uint8_t *sSFA = sB + C::B_BYTES;
                    uint8_t *sSFB = sSFA + C::SFA_BYTES;
                    const uint32_t tm_sfa = tm_sf + sfsel * C::SF_COLS;
                    sfsel ^= 1u;
                    const uint32_t tm_sfb = tm_sfa + C::SFA_COLS;
                    const uint64_t dA = desc_sw128(smem_u32(sA)), dB = desc_sw128(smem_u32(sB));
#pragma unroll
                    for (int kb = 0; kb < C::BK / C::MMA_K; ++kb) {
                        if (kb >= mmas)
                            break;
                        // copy an atom's scales just before the first MMA that reads them, so the
                        // copies of k-block kb+1 overlap the MMA of k-block kb
                        const int a = C::NV ? kb : kb >> 1;
                        if (C::NV || (kb & 1) == 0) {
                            tc_cp_atom_w(tm_sfa + a * 4, desc_sf_atom(smem_u32(sSFA + a * 512)));
                            if constexpr (C::FUSEQ) {  // one copy per two k-blocks (see fuseq_store)
                                if ((kb & 1) == 0)
                                    tc_cp_atom_w(tm_sfb + (kb >> 1) * 4,
                                                 desc_sf_atom(smem_u32(sSFB + (kb >> 1) * 512)));
                            } else {
#pragma unroll
                                for (int rt = 0; rt < C::RT; ++rt)
                                    tc_cp_atom_w(tm_sfb + a * C::RT * 4 + rt * 4,
                                                 desc_sf_atom(smem_u32(sSFB + (rt * C::APK + a) * 512)));
                            }
                        }
                        uint32_t sfa, sfb, idesc;
                        if (C::NV) {
                            sfa = tm_sfa + kb * 4;
                            // rows n < 32 of B read their scales at lane n, column 0 of the address:
                            // k-block kb's scales sit at column 4 (kb / 2) + 2 (kb % 2)
                            sfb = C::FUSEQ ? tm_sfb + (kb >> 1) * 4 + (kb & 1) * 2
                                           : tm_sfb + kb * C::RT * 4 + sfb_off;
                            idesc = C::IDESC;
                        } else {
                            const uint32_t byte = (uint32_t)(kb & 1) * 2u;  // second MMA of an atom: scale bytes 2..3
                            sfa = (tm_sfa + a * 4) | (byte << 30);
                            sfb = (tm_sfb + a * C::RT * 4 + sfb_off) | (byte << 30);
                            idesc = C::IDESC | (byte << 29) | (byte << 4);
                        }
                        // advance 64 FP4 values = 32 bytes inside the swizzled rows
                        tc_mma_w<C::NV>(d_tmem, dA + (uint64_t)(kb * 2), dB + (uint64_t)(kb * 2), idesc, sfa, sfb,
                                        (kt > kt0 || kb > 0) ? 1u : 0u);
                    }
                    tc_commit_w(&empty[stage]);
                    if (++stage == C::STAGES) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
                if (!ok)
                    break;
                tc_commit_w(&acc_full[acc]);
            }
            // every MMA this CTA issued has completed before TMEM is freed
            tc_commit_w(done_bar);
            if (lane == 0)
                wait_bounded(done_bar, 0, abort, false);
        }
        __syncwarp();
    } else if (warp == C::WAITER_WARP) {
        // ---------------------------------------------------------------- waiter (one warp)
        // Walks the MMA warp's sequence of barrier waits -- per tile the accumulator, per k-tile
        // the stage -- one step ahead of it, and meets it after each (named barrier 2, which also
        // carries a failed wait to it).  Both leave at the same meeting.
        int stage = 0;
        uint32_t phase = 0;
        int it = 0;
        bool ok = true;
        for (int64_t w = blockIdx.x; w < p.work && ok; w += gridDim.x, ++it) {
            int mt, nt, sp;
            tile_coords(p, w, mt, nt, sp);
            const int kt0 = sp * p.kps, kt1 = min(p.nk, kt0 + p.kps);
            const int acc = it % C::NUM_ACC;
            const uint32_t acc_phase = (uint32_t)(it / C::NUM_ACC) & 1u;
            if (meet_or(!warp_poll(&acc_empty[acc], acc_phase ^ 1u, abort, lane))) {
                ok = false;
                break;
            }
            for (int kt = kt0; kt < kt1; ++kt) {
                if (meet_or(!warp_poll(&full[stage], phase, abort, lane))) {
                    ok = false;
                    break;
                }
                if (++stage == C::STAGES) {
                    stage = 0;
                    phase ^= 1u;
                }
            }
        }
    } else {
        // ---------------------------------------------------------------- epilogue
        const int quad = warp & 3;                       // TMEM lanes this warp may access
        const int half = (warp - 2) >> 2;                // which half of the tile's columns
        const int et = threadIdx.x - 64;                 // 0..255 over the epilogue warps
        float gg = C::NV ? __fmul_rn(*p.g_a, *p.g_w) : 1.0f;
        float xg = 0.0f;                                 // FUSEQ: the activations' tensor scale
        __shared__ float s_xred[C::EPI_WARPS];
        __shared__ float s_xg;
        __shared__ float s_rcp[C::FUSEQ ? 256 : 1];  // FUSEQ: 1/(dec(sf) xg) per scale byte
        float c6 = 0.0f;
        if constexpr (C::FUSEQ) {
            if (p.xnpart != 0) {  // the computed tensor scale: amax / 2688
                float m = 0.0f;
                if (p.xnpart > 0) {  // over the amax pass's partial maxima
                    pdl_wait();  // this grid may have started before the amax pass finished
                    for (int k = et; k < p.xnpart; k += C::EPI_WARPS * 32)
                        m = fmaxf(m, p.xpart[k]);
                } else {  // over all of the (few) activations, in this CTA
                    constexpr int U = 4, T = C::EPI_WARPS * 32;
                    const int nbk = (int)(p.K >> 4), nb = (int)p.N * nbk;
                    for (int b0 = et; b0 < nb; b0 += U * T) {
                        FuseRaw buf[U];
#pragma unroll
                        for (int j = 0; j < U; ++j) {
                            const int b = b0 + j * T;
                            if (b < nb) {
                                const int r = b / nbk;
                                const __nv_bfloat16 *src = p.xa + r * p.ld_xa + 16 * (b - r * nbk);
                                buf[j].u0 = ld_nc_v4(src);
                                buf[j].u1 = ld_nc_v4(src + 8);
                            }
                        }
#pragma unroll
                        for (int j = 0; j < U; ++j) {
                            if (b0 + j * T < nb) {
                                const uint32_t raw[8] = {buf[j].u0.x, buf[j].u0.y, buf[j].u0.z, buf[j].u0.w,
                                                         buf[j].u1.x, buf[j].u1.y, buf[j].u1.z, buf[j].u1.w};
                                float v[16];
                                if (p.xhad)
                                    nvfp4_block_values<true>(raw, v);
                                else
                                    nvfp4_block_values<false>(raw, v);
                                m = fmaxf(m, abs_max<16>(v));
                            }
                        }
                    }
                }
#pragma unroll
                for (int o = 16; o; o >>= 1)
                    m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
                if (lane == 0)
                    s_xred[warp - 2] = m;
                asm volatile("bar.sync 1, %0;" ::"r"(C::EPI_WARPS * 32) : "memory");
                if (et == 0) {
                    float b = 0.0f;
                    for (int k = 0; k < C::EPI_WARPS; ++k)
                        b = fmaxf(b, s_xred[k]);
                    float g = __fdiv_rn(b, 2688.0f);  // 6 * 448, as the quantiser
                    if (!(g > 0.0f))
                        g = 1.0f;
                    s_xg = g;
                    if (blockIdx.x == 0)
                        *p.g_a_out = g;
                }
                asm volatile("bar.sync 1, %0;" ::"r"(C::EPI_WARPS * 32) : "memory");
                xg = s_xg;
            } else {
                xg = *p.g_w;  // swapped form: g_w is the activations' slot, g_a the weights'
            }
            gg = __fmul_rn(xg, *p.g_a);
            c6 = nvfp4_fast_c6(xg);
            for (int i = et; i < 256; i += C::EPI_WARPS * 32)
                s_rcp[i] = nvfp4_block_rcp((uint32_t)i, xg);
            // scale-atom rows past the 16 activation rows: zero once in every stage
            for (int s = 0; s < C::STAGES; ++s) {
                uint8_t *sfb = smem + s * C::STAGE_BYTES + C::A_BYTES + C::B_BYTES + C::SFA_BYTES;
                for (int i = et; i < C::SFB_BYTES / 16; i += C::EPI_WARPS * 32)
                    *reinterpret_cast<uint4 *>(sfb + 16 * i) = make_uint4(0u, 0u, 0u, 0u);
            }
            asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
            asm volatile("bar.sync 1, %0;" ::"r"(C::EPI_WARPS * 32) : "memory");  // zeros before any fill
        }
        volatile int *epi_fail = epi_ok + 2;
        int qstage = 0;
        uint32_t qphase = 0;
        // FUSEQ: fill the activation operand of item w's stages, as the producer fills the
        // weights; the k-tile's values are fetched FUSEQ_PREFETCH k-tiles ahead of their encoding.
        // Returns false (all epilogue warps agree) when a wait gave up.
        auto fill_item = [&](int64_t w) -> bool {
            int mt, nt, sp;
            tile_coords(p, w, mt, nt, sp);
            const int kt0 = sp * p.kps, kt1 = min(p.nk, kt0 + p.kps);
            FuseRaw buf[FUSEQ_PREFETCH];
#pragma unroll
            for (int j = 0; j < FUSEQ_PREFETCH; ++j)
                if (kt0 + j < kt1)
                    fuseq_load(p, kt0 + j, et, buf[j]);
            bool okq = true;
            for (int base = kt0; okq && base < kt1; base += FUSEQ_PREFETCH) {
#pragma unroll
                for (int j = 0; j < FUSEQ_PREFETCH; ++j) {
                    const int kt = base + j;
                    if (kt >= kt1)
                        break;
                    const FuseRaw cur = buf[j];
                    if (kt + FUSEQ_PREFETCH < kt1)
                        fuseq_load(p, kt + FUSEQ_PREFETCH, et, buf[j]);
                    if (!(okq = warp_wait(&empty[qstage], qphase ^ 1u, abort, lane)))
                        break;
                    uint8_t *sB = smem + qstage * C::STAGE_BYTES + C::A_BYTES;
                    fuseq_store(p, sB, sB + C::B_BYTES + C::SFA_BYTES, kt, et, cur, xg, c6, s_rcp);
                    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");  // visible to the tensor core
                    __syncwarp();
                    if (lane == 0)
                        mbar_arrive(&full[qstage]);
                    if (++qstage == C::STAGES) {
                        qstage = 0;
                        qphase ^= 1u;
                    }
                }
            }
            if (!okq && lane == 0)
                *epi_fail = 1;
            asm volatile("bar.sync 1, %0;" ::"r"(C::EPI_WARPS * 32) : "memory");  // agree before going on
            return *epi_fail == 0;
        };
        if constexpr (C::FUSEQ) {
            if (blockIdx.x < p.work)
                (void)fill_item(blockIdx.x);
        }
        int it = 0;
        for (int64_t w = blockIdx.x; w < p.work; w += gridDim.x, ++it) {
            int mt, nt, sp;
            tile_coords(p, w, mt, nt, sp);
            if constexpr (C::FUSEQ) {
                // the next item's operand first, so its MMAs can start while this item drains
                if (*epi_fail || (w + gridDim.x < p.work && !fill_item(w + gridDim.x)))
                    break;
            }
            const int acc = it % C::NUM_ACC;
            const uint32_t acc_phase = (uint32_t)(it / C::NUM_ACC) & 1u;
            // one warp polls the accumulator barrier; the others sleep in a named barrier (they
            // issue nothing meanwhile, so the MMA-issuing warp keeps the SM's issue slots)
            if (warp == 2) {
                const bool okw = warp_poll(&acc_full[acc], acc_phase, abort, lane);
                if (lane == 0)
                    epi_ok[it & 1] = okw ? 1 : 0;
            }
            asm volatile("bar.sync 1, %0;" ::"r"(C::EPI_WARPS * 32) : "memory");
            if (!epi_ok[it & 1])
                break;
            tc_fence_after();
            float v[C::COLS_PER_WARP];
            const uint32_t taddr = tmem_base + ((uint32_t)(quad * 32) << 16) + acc * C::BN + half * C::COLS_PER_WARP;
            if constexpr (C::SWAP) {
                tmem_ld8(taddr, v);
            } else {
#pragma unroll
                for (int c = 0; c < C::COLS_PER_WARP; c += 32)
                    tmem_ld32(taddr + c, v + c);
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0)
                mbar_arrive(&acc_empty[acc]);  // this warp's part of the accumulator is free

            if constexpr (C::SWAP) {
                // accumulator row = weight row n, column = activation row m: y[m, n]
                const int64_t n = (int64_t)mt * C::BM + quad * 32 + lane;
                if (p.splits == 1 && p.qc) {
                    // output quantisation: a 16-column block of row m lies on 16 lanes; with
                    // N % 64 == 0 the warp's 32 columns are all inside or all outside N
                    if ((int64_t)mt * C::BM + quad * 32 < p.M) {
                        const float qg = *p.qg;
#pragma unroll
                        for (int c = 0; c < C::COLS_PER_WARP; ++c) {
                            const int64_t m = (int64_t)nt * C::BN + half * C::COLS_PER_WARP + c;
                            if (m >= p.N)
                                break;
                            const __nv_bfloat16 yb = __float2bfloat16_rn(__fmul_rn(v[c], gg));
                            if (p.y)
                                p.y[m * p.ldy + n] = yb;
                            float w = __bfloat162float(yb);
                            if (p.qhad) {
                                fwht16_lanes<16>(&w);
                                w = __fmul_rn(w, 0.25f);
                            }
                            float a = fabsf(w);
#pragma unroll
                            for (int o = 1; o < 16; o <<= 1)
                                a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, o));
                            float rcp;
                            const uint32_t sf = nvfp4_block_scale(a, qg, rcp);
                            const float wv = __fmul_rn(w, rcp);
                            const float wn = __shfl_xor_sync(0xffffffffu, wv, 1);
                            if ((lane & 1) == 0)  // even column: low nibble, its odd neighbour: high
                                p.qc[m * (p.M / 2) + n / 2] = (uint8_t)cvt_e2m1x2(wv, wn);
                            if ((lane & 15) == 0)
                                p.qs[tc_offset(m, n / 16, p.qkatoms)] = (uint8_t)sf;
                        }
                    }
                    continue;
                }
                if (n < p.M) {
#pragma unroll
                    for (int c = 0; c < C::COLS_PER_WARP; ++c) {
                        const int64_t m = (int64_t)nt * C::BN + half * C::COLS_PER_WARP + c;
                        if (m < p.N) {
                            if (p.splits == 1)
                                p.y[m * p.ldy + n] = __float2bfloat16_rn(__fmul_rn(v[c], gg));
                            else
                                p.ws[((int64_t)sp * p.N + m) * p.ldw + n] = v[c];
                        }
                    }
                }
                continue;
            }

            const int64_t m = (int64_t)mt * C::BM + quad * 32 + lane;
            const int64_t n0 = (int64_t)nt * C::BN + half * C::COLS_PER_WARP;
            if (m < p.M) {
                if (p.splits == 1) {
#pragma unroll
                    for (int c = 0; c < C::COLS_PER_WARP; ++c)
                        v[c] = __fmul_rn(v[c], gg);
                    if (p.qc) {
                        // round once to bf16, in place: the stored y and the quantised y agree
#pragma unroll
                        for (int c = 0; c < C::COLS_PER_WARP; ++c)
                            v[c] = __bfloat162float(__float2bfloat16_rn(v[c]));
                    }
                    if (p.y) {
                        __nv_bfloat16 *yr = p.y + m * p.ldy;
                        // 16 columns per 256-bit store where the row segment is 32-byte aligned
                        const bool w32 = (reinterpret_cast<uintptr_t>(yr + n0) & 31) == 0;
#pragma unroll
                        for (int c = 0; c < C::COLS_PER_WARP; c += 16) {
                            const int64_t n = n0 + c;
                            if (w32 && n + 16 <= p.N) {
                                uint32_t w8[8];
#pragma unroll
                                for (int j = 0; j < 8; ++j) {
                                    __nv_bfloat162 b2 = __floats2bfloat162_rn(v[c + 2 * j], v[c + 2 * j + 1]);
                                    w8[j] = *reinterpret_cast<uint32_t *>(&b2);
                                }
                                st_v8(yr + n, w8);
                                continue;
                            }
#pragma unroll
                            for (int h = 0; h < 16; h += 8) {
                                if (n + h + 8 <= p.N) {
                                    uint32_t w4[4];
#pragma unroll
                                    for (int j = 0; j < 4; ++j) {
                                        __nv_bfloat162 b2 =
                                            __floats2bfloat162_rn(v[c + h + 2 * j], v[c + h + 2 * j + 1]);
                                        w4[j] = *reinterpret_cast<uint32_t *>(&b2);
                                    }
                                    st_v4(yr + n + h, make_uint4(w4[0], w4[1], w4[2], w4[3]));
                                } else {
                                    for (int j = 0; j < 8; ++j)
                                        if (n + h + j < p.N)
                                            yr[n + h + j] = __float2bfloat16_rn(v[c + h + j]);
                                }
                            }
                        }
                    }
                    if (p.qc) {
                        const float qg = *p.qg;
#pragma unroll
                        for (int c = 0; c < C::COLS_PER_WARP; c += 16)
                            if (n0 + c < p.N)  // N % 64 == 0: whole blocks
                                quantize_out_block(v + c, m, n0 + c, p.qc, p.qs, qg, p.qhad != 0, p.N, p.qkatoms);
                    }
                } else {
                    float *wr = p.ws + ((int64_t)sp * p.M + m) * p.ldw;
#pragma unroll
                    for (int c = 0; c < C::COLS_PER_WARP; c += 4) {
                        const int64_t n = n0 + c;
                        if (n + 4 <= p.N) {
                            st_v4(wr + n, make_uint4(__float_as_uint(v[c]), __float_as_uint(v[c + 1]),
                                                     __float_as_uint(v[c + 2]), __float_as_uint(v[c + 3])));
                        } else {
                            for (int j = 0; j < 4; ++j)
                                if (n + j < p.N)
                                    wr[n + j] = v[c + j];
                        }
                    }
                }
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem_base),
                     "r"((uint32_t)C::TMEM_COLS)
                     : "memory");
    }
}

// Output quantisation arguments of the split-K reduction (qc null: off); see GemmParams.
struct QuantOut {
    uint8_t *qc, *qs;
    const float *qg;
    int qhad;
    int64_t qkatoms;
};

// y = bf16(g_a * g_w * sum_s ws[s]) in split order (deterministic), and optionally its NVFP4
// encoding.  Every lane of a warp runs the same iterations: with N % 64 == 0 a 16-column
// block of the output is 4 consecutive lanes, which share its maximum and rotation by shuffles.
__global__ void __launch_bounds__(256) splitk_reduce_kernel(const float *ws, int splits, int64_t M, int64_t N,
                                                            int64_t ldw, const float *g_a, const float *g_w,
                                                            __nv_bfloat16 *y, int64_t ldy, QuantOut qo)
{
    pdl_wait();  // launched while the GEMM still runs
    const float gg = (g_a && g_w) ? __fmul_rn(*g_a, *g_w) : 1.0f;
    const float qg = qo.qc ? *qo.qg : 1.0f;
    const int64_t nq = (N + 3) / 4, total = M * nq;
    const int lane = threadIdx.x & 31;
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    for (int64_t base = (int64_t)blockIdx.x * blockDim.x + (threadIdx.x & ~31); base < total; base += stride) {
        const int64_t i = base + lane;
        const bool valid = i < total;
        int64_t m = 0, n = 0;
        float s[4] = {0.f, 0.f, 0.f, 0.f};
        if (valid) {
            m = i / nq;
            n = (i - m * nq) * 4;
            for (int k = 0; k < splits; ++k) {
                const float *src = ws + ((int64_t)k * M + m) * ldw + n;
                if (n + 4 <= N) {
                    const float4 f = *reinterpret_cast<const float4 *>(src);
                    s[0] = __fadd_rn(s[0], f.x);
                    s[1] = __fadd_rn(s[1], f.y);
                    s[2] = __fadd_rn(s[2], f.z);
                    s[3] = __fadd_rn(s[3], f.w);
                } else {
                    for (int j = 0; j < 4 && n + j < N; ++j)
                        s[j] = __fadd_rn(s[j], src[j]);
                }
            }
        }
        if (!qo.qc) {
            if (!valid)
                continue;
            __nv_bfloat16 *dst = y + m * ldy + n;
            if (n + 4 <= N) {
                __nv_bfloat162 lo = __floats2bfloat162_rn(__fmul_rn(s[0], gg), __fmul_rn(s[1], gg));
                __nv_bfloat162 hi = __floats2bfloat162_rn(__fmul_rn(s[2], gg), __fmul_rn(s[3], gg));
                uint2 u = make_uint2(*reinterpret_cast<uint32_t *>(&lo), *reinterpret_cast<uint32_t *>(&hi));
                *reinterpret_cast<uint2 *>(dst) = u;
            } else {
                for (int j = 0; j < 4 && n + j < N; ++j)
                    dst[j] = __float2bfloat16_rn(__fmul_rn(s[j], gg));
            }
            continue;
        }
        // output quantisation (N % 64 == 0: four whole columns per lane)
        float w[4];
#pragma unroll
        for (int j = 0; j < 4; ++j)
            w[j] = __bfloat162float(__float2bfloat16_rn(__fmul_rn(s[j], gg)));
        if (valid && y) {
            __nv_bfloat162 lo = __floats2bfloat162_rn(w[0], w[1]), hi = __floats2bfloat162_rn(w[2], w[3]);
            *reinterpret_cast<uint2 *>(y + m * ldy + n) =
                make_uint2(*reinterpret_cast<uint32_t *>(&lo), *reinterpret_cast<uint32_t *>(&hi));
        }
        if (qo.qhad) {
            fwht16_lanes<4>(w);
#pragma unroll
            for (int j = 0; j < 4; ++j)
                w[j] = __fmul_rn(w[j], 0.25f);
        }
        float a = abs_max<4>(w);
        a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, 1));
        a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, 2));
        float rcp;
        const uint32_t sf = nvfp4_block_scale(a, qg, rcp);
        if (valid) {
            const uint32_t c01 = cvt_e2m1x2(__fmul_rn(w[0], rcp), __fmul_rn(w[1], rcp));
            const uint32_t c23 = cvt_e2m1x2(__fmul_rn(w[2], rcp), __fmul_rn(w[3], rcp));
            *reinterpret_cast<uint16_t *>(qo.qc + m * (N / 2) + n / 2) = (uint16_t)(c01 | (c23 << 8));
            if ((lane & 3) == 0)
                qo.qs[tc_offset(m, n / 16, qo.qkatoms)] = (uint8_t)sf;
        }
    }
}

// Weights [N, K/2] codes -> tile order for the decode GEMM: tile (mt, kt) holds rows
// 128 mt .. +127, code bytes 128 kt .. +127, as the 128-byte-swizzled image (16-byte chunk c
// of row r at chunk c ^ (r % 8)); rows past N and bytes past K/2 are zero.  One thread per
// 16-byte chunk of the output.
__global__ void __launch_bounds__(256) weight_tile_kernel(const uint8_t *codes, int64_t N, int64_t K, uint8_t *tiled,
                                                          int64_t chunks)
{
    const int64_t nk = (K + 255) / 256;
    for (int64_t o = (int64_t)blockIdx.x * 256 + threadIdx.x; o < chunks; o += (int64_t)gridDim.x * 256) {
        const int64_t tile = o >> 10, within = o & 1023;
        const int r = (int)(within >> 3), c = (int)(within & 7) ^ (r & 7);
        const int64_t mt = tile / nk, kt = tile - mt * nk;
        const int64_t row = mt * 128 + r, byte = kt * 128 + c * 16;
        uint4 v = make_uint4(0u, 0u, 0u, 0u);
        if (row < N && byte < K / 2)  // K % 64 == 0: a 16-byte chunk is all in or all out
            v = ld_nc_v4(codes + row * (K / 2) + byte);
        reinterpret_cast<uint4 *>(tiled)[o] = v;
    }
}

}  // namespace fp4lin
