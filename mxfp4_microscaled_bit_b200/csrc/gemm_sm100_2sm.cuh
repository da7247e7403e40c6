// gemm_sm100_2sm.cuh -- the prefill GEMM on CTA pairs: tcgen05.mma.cta_group::2
// computes a 256 x 256 tile across two SMs of a cluster.  Each CTA holds 128
// rows of A and 128 rows (N) of B in its shared memory and 128 x 256 of the
// accumulator in its TMEM; the pair's tensor cores read both halves of B, so
// per SM the operand traffic per FLOP drops by a third against the one-CTA
// 128 x 256 tile, and a stage shrinks from 54 KB to 38 KB (five stages).
// Both kernels issue their tcgen05 instructions from a converged warp (see tc_mma_w) and
// give the same results bit for bit.  On the 8192 x 14336 x 4096 prefill product the pair
// takes 212 us (NVFP4) and 189 us (MXFP4), the one-CTA kernel 228 and 206 us, so the pair
// runs every GEMM of 256-column tiles without a K split once M >= 256
// (FP4LIN_GEMM_KERNEL=single or =pair forces either).
//
// Roles (352 threads per CTA, both CTAs):
//   warp 0 lane 0   producer: TMA loads of this CTA's A half, B half, scale A
//                   (its 128 rows) and scale B (all 256 N rows -- every CTA's
//                   TMEM needs them), all completing on the LEADER's `full`
//                   barrier (cta_group::2 form, peer bit of the address cleared);
//   warp 1          TMEM (cta_group::2 alloc/dealloc in both CTAs); in the
//                   leader, the converged warp issues (one elected lane) the scale
//                   copies and MMAs for the pair and commits, multicast to both
//                   CTAs' barriers;
//   warps 2..9      epilogue of this CTA's 128 accumulator rows; they release
//                   the accumulator by arriving on the leader's `acc_empty`;
//   warp 10         in the leader, waits on the barriers for the MMA warp and
//                   meets it at a named barrier (as in the one-CTA kernel).
// All waits are bounded as in the one-CTA kernel.  No load uses multicast.
#pragma once

#include "gemm_sm100.cuh"

namespace fp4lin {

__device__ __forceinline__ uint32_t cluster_ctarank()
{
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}

__device__ __forceinline__ void cluster_sync_all()
{
    asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}

// Shared::cluster address of the same shared-memory object in the leader CTA (rank 0).
__device__ __forceinline__ uint32_t leader_addr(uint32_t cta_addr)
{
    uint32_t r;
    asm volatile("mapa.shared::cluster.u32 %0, %1, 0;" : "=r"(r) : "r"(cta_addr));
    return r;
}

// TMA tile load into this CTA's shared memory whose bytes complete on the
// leader's mbarrier (the .cta_group::2 form; no multicast).
__device__ __forceinline__ void tma_load_2d_pair(void *dst, const CUtensorMap *map, uint64_t *bar, int x, int y)
{
    asm volatile("cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes"
                 " [%0], [%1, {%3, %4}], [%2];" ::"r"(smem_u32(dst)),
                 "l"(map), "r"(leader_addr(smem_u32(bar))), "r"(x), "r"(y)
                 : "memory");
}

// Arrive on the leader's copy of `bar` (release at cluster scope).
__device__ __forceinline__ void mbar_arrive_leader(uint64_t *bar)
{
    asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(leader_addr(smem_u32(bar)))
                 : "memory");
}

__device__ __forceinline__ bool mbar_try_wait_cluster(uint64_t *bar, uint32_t parity)
{
    uint32_t ok;
    asm volatile("{\n\t.reg .pred p;\n\t"
                 "mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2, %3;\n\t"
                 "selp.u32 %0, 1, 0, p;\n\t}"
                 : "=r"(ok)
                 : "r"(smem_u32(bar)), "r"(parity), "r"(20000u)
                 : "memory");
    return ok != 0;
}

// Bounded wait with cluster-scope acquire (arrivals come from the peer CTA too).
__device__ __noinline__ bool wait_bounded_cluster(uint64_t *bar, uint32_t parity, volatile int *abort)
{
    const unsigned long long t0 = globaltimer_ns();
    for (uint32_t it = 0;; ++it) {
        if (mbar_try_wait_cluster(bar, parity))
            return true;
        if ((it & 7u) == 7u) {
            if (*abort)
                return false;
            if (globaltimer_ns() - t0 > WAIT_LIMIT_NS) {
                report_error(FP4LIN_ERR_TIMEOUT);
                *abort = 1;
                return false;
            }
        }
    }
}

// Commit this thread's prior tcgen05 operations to `bar` in both CTAs of the pair.
__device__ __forceinline__ void tc_commit_pair(uint64_t *bar)
{
    asm volatile("tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], %1;" ::"r"(
                     smem_u32(bar)),
                 "h"((uint16_t)3)
                 : "memory");
}

__device__ __forceinline__ void tc_cp_atom_pair(uint32_t taddr, uint64_t sdesc)
{
    asm volatile("tcgen05.cp.cta_group::2.32x128b.warpx4 [%0], %1;" ::"r"(taddr), "l"(sdesc) : "memory");
}

// Converged-warp forms (every lane of the issuing warp makes the call, one elected lane issues;
// see tc_mma_w in gemm_sm100.cuh).
__device__ __forceinline__ void tc_commit_pair_w(uint64_t *bar)
{
    asm volatile("{\n\t.reg .pred e;\n\telect.sync _|e, 0xffffffff;\n\t"
                 "@e tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], %1;\n\t}" ::"r"(
                     smem_u32(bar)),
                 "h"((uint16_t)3)
                 : "memory");
}

__device__ __forceinline__ void tc_cp_atom_pair_w(uint32_t taddr, uint64_t sdesc)
{
    asm volatile("{\n\t.reg .pred e;\n\telect.sync _|e, 0xffffffff;\n\t"
                 "@e tcgen05.cp.cta_group::2.32x128b.warpx4 [%0], %1;\n\t}" ::"r"(taddr),
                 "l"(sdesc)
                 : "memory");
}

template <bool NV>
__device__ __forceinline__ void tc_mma_pair_w(uint32_t d, uint64_t a, uint64_t b, uint32_t idesc, uint32_t sfa,
                                              uint32_t sfb, uint32_t acc)
{
    if constexpr (NV) {
        asm volatile("{\n\t.reg .pred p, e;\n\tsetp.ne.b32 p, %4, 0;\n\telect.sync _|e, 0xffffffff;\n\t"
                     "@e tcgen05.mma.cta_group::2.kind::mxf4nvf4.block_scale.block16 [%0], %1, %2, %3, [%5], [%6], p;\n\t}" ::"r"(
                         d),
                     "l"(a), "l"(b), "r"(idesc), "r"(acc), "r"(sfa), "r"(sfb)
                     : "memory");
    } else {
        asm volatile("{\n\t.reg .pred p, e;\n\tsetp.ne.b32 p, %4, 0;\n\telect.sync _|e, 0xffffffff;\n\t"
                     "@e tcgen05.mma.cta_group::2.kind::mxf4.block_scale.block32 [%0], %1, %2, %3, [%5], [%6], p;\n\t}" ::"r"(
                         d),
                     "l"(a), "l"(b), "r"(idesc), "r"(acc), "r"(sfa), "r"(sfb)
                     : "memory");
    }
}

// warp_poll with cluster-scope acquire (the barrier's arrivals come from the peer CTA too).
__device__ __forceinline__ bool warp_poll_cluster(uint64_t *bar, uint32_t parity, volatile int *abort, int lane)
{
    const unsigned long long t0 = globaltimer_ns();
    for (uint32_t it = 0;; ++it) {
        uint32_t ok;
        asm volatile("{\n\t.reg .pred p;\n\t"
                     "mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2;\n\t"
                     "selp.u32 %0, 1, 0, p;\n\t}"
                     : "=r"(ok)
                     : "r"(smem_u32(bar)), "r"(parity)
                     : "memory");
        if (ok)
            return true;
        if ((it & 7u) == 7u) {
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

template <bool NV>
__device__ __forceinline__ void tc_mma_pair(uint32_t d, uint64_t a, uint64_t b, uint32_t idesc, uint32_t sfa,
                                            uint32_t sfb, uint32_t acc)
{
    if constexpr (NV) {
        asm volatile("{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
                     "tcgen05.mma.cta_group::2.kind::mxf4nvf4.block_scale.block16 [%0], %1, %2, %3, [%5], [%6], p;\n\t}" ::"r"(
                         d),
                     "l"(a), "l"(b), "r"(idesc), "r"(acc), "r"(sfa), "r"(sfb)
                     : "memory");
    } else {
        asm volatile("{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
                     "tcgen05.mma.cta_group::2.kind::mxf4.block_scale.block32 [%0], %1, %2, %3, [%5], [%6], p;\n\t}" ::"r"(
                         d),
                     "l"(a), "l"(b), "r"(idesc), "r"(acc), "r"(sfa), "r"(sfb)
                     : "memory");
    }
}

template <bool NV_>
struct Gemm2Cfg {
    static constexpr bool NV = NV_;
    static constexpr int BM = 256, BN = 256;               // pair tile
    static constexpr int CM = 128, CN = 128;               // rows of A / B in each CTA
    static constexpr int BK = 256, MMA_K = 64;
    static constexpr int APK = NV ? BK / 64 : BK / 128;    // scale atoms per 128 rows per stage
    static constexpr int SF_BOX_ROWS = APK * 2;            // the atoms as rows of 256 bytes
    static constexpr int A_BYTES = CM * 128, B_BYTES = CN * 128;
    static constexpr int SFA_BYTES = APK * 512, SFB_BYTES = 2 * APK * 512;  // B scales: all 256 N rows
    static constexpr int STAGE_BYTES = A_BYTES + B_BYTES + SFA_BYTES + SFB_BYTES;
    static constexpr int STAGES = (225 * 1024) / STAGE_BYTES > 8 ? 8 : (225 * 1024) / STAGE_BYTES;
    static constexpr int TX_BYTES = 2 * STAGE_BYTES;       // both CTAs' bytes land on the leader's barrier
    static constexpr int SFA_COLS = APK * 4, SFB_COLS = 2 * APK * 4, SF_COLS = SFA_COLS + SFB_COLS;
    static constexpr int TMEM_USED = BN + 2 * SF_COLS;
    static constexpr int TMEM_COLS = 512;
    static constexpr int EPI_WARPS = 8;
    static constexpr int WAITER_WARP = 2 + EPI_WARPS;    // the leader's barrier waits for its MMA warp
    static constexpr int THREADS = 64 + EPI_WARPS * 32 + 32;
    static constexpr int COLS_PER_WARP = BN / 2;
    static constexpr int BAR_BYTES = 256;
    static constexpr int SMEM_BYTES = STAGES * STAGE_BYTES + BAR_BYTES + 1024;
    // instruction descriptor: A/B E2M1, K-major, N = 256, M = 256 (the pair)
    static constexpr uint32_t IDESC = (1u << 7) | (1u << 10) | ((uint32_t)(BN >> 3) << 17) |
                                      ((NV ? 0u : 1u) << 23) | ((uint32_t)(BM >> 4) << 24);
    static_assert(TMEM_USED <= 512, "TMEM overflow");
    static_assert(SMEM_BYTES <= 232448, "shared memory overflow");
    static_assert(STAGE_BYTES % 1024 == 0, "stages must keep the 1024-byte alignment of the swizzled tiles");
    static_assert(STAGES >= 3, "pipeline too shallow");
};

struct Gemm2Params {
    const float *g_a, *g_w;
    __nv_bfloat16 *y;
    int64_t M, N, K, ldy;
    int64_t katoms;             // scale atoms per 128-row tile along K
    int num_mt, num_nt, nk;     // pair tiles of 256 x 256, k-tiles of 256
    int raster;
    int64_t work;
};

// Pair tile w -> (m tile, n tile), walked in groups of `raster` m-tiles.
__device__ __forceinline__ void pair_tile_coords(const Gemm2Params &p, int64_t w, int &mt, int &nt)
{
    const int64_t group = (int64_t)p.raster * p.num_nt;
    const int64_t g = w / group, idx = w - g * group;
    const int64_t m0 = g * p.raster;
    const int64_t rows = min((int64_t)p.raster, (int64_t)p.num_mt - m0);
    mt = (int)(m0 + idx % rows);
    nt = (int)(idx / rows);
}

template <class C>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(C::THREADS, 1)
    fp4_gemm_pair_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                         const __grid_constant__ CUtensorMap tmSFA, const __grid_constant__ CUtensorMap tmSFB,
                         Gemm2Params p)
{
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
    uint8_t *bar_area = smem + C::STAGES * C::STAGE_BYTES;
    uint64_t *full = reinterpret_cast<uint64_t *>(bar_area);   // leader's copy counts both CTAs' bytes
    uint64_t *empty = full + C::STAGES;                          // both CTAs: stage consumed by the pair's MMAs
    uint64_t *acc_full = empty + C::STAGES;                      // both CTAs: accumulator complete
    uint64_t *acc_empty = acc_full + 1;                          // leader: both CTAs' epilogues have read it
    uint64_t *done_bar = acc_empty + 1;                          // both CTAs: every MMA of the pair completed
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(done_bar + 1);
    volatile int *abort = reinterpret_cast<volatile int *>(tmem_slot + 1);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t rank = cluster_ctarank();
    const int64_t pair = blockIdx.x >> 1, npairs = gridDim.x >> 1;

    if (threadIdx.x == 0) {
        for (int s = 0; s < C::STAGES; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        mbar_init(acc_full, 1);
        mbar_init(acc_empty, 2 * C::EPI_WARPS);
        mbar_init(done_bar, 1);
        *abort = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (warp == 1) {
        // the pair allocates the same TMEM columns on both SMs
        asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tmem_slot)),
                     "r"((uint32_t)C::TMEM_COLS)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
    }
    tc_fence_before();
    cluster_sync_all();  // barriers of both CTAs initialised and TMEM allocated before any remote use
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;

    if (warp == 0) {
        // ---------------------------------------------------------------- producer (one thread per CTA)
        if (lane == 0) {
            int stage = 0;
            uint32_t phase = 0;
            uint32_t armed = 0, armed_phase = 0;
            bool ok = true;
            for (int64_t w = pair; w < p.work && ok; w += npairs) {
                int mt, nt;
                pair_tile_coords(p, w, mt, nt);
                const int a_row = mt * C::BM + (int)rank * C::CM;
                const int b_row = nt * C::BN + (int)rank * C::CN;
                const int64_t sfa_tile = (int64_t)mt * 2 + rank, sfb_tile = (int64_t)nt * 2;
                for (int kt = 0; kt < p.nk; ++kt) {
                    if (!(ok = wait_bar(&empty[stage], phase ^ 1u, abort)))
                        break;
                    uint8_t *sA = smem + stage * C::STAGE_BYTES;
                    uint8_t *sB = sA + C::A_BYTES;
                    uint8_t *sSFA = sB + C::B_BYTES;
                    uint8_t *sSFB = sSFA + C::SFA_BYTES;
                    if (rank == 0)
                        mbar_expect_tx(&full[stage], C::TX_BYTES);
                    armed |= 1u << stage;
                    armed_phase = (armed_phase & ~(1u << stage)) | (phase << stage);
                    const int64_t ka = (int64_t)kt * C::APK;
                    tma_load_2d_pair(sA, &tmA, &full[stage], kt * 128, a_row);
                    tma_load_2d_pair(sB, &tmB, &full[stage], kt * 128, b_row);
                    // scale atoms as rows of 256 bytes: atom j of row tile t starts at row 2 (t katoms + j)
                    tma_load_2d_pair(sSFA, &tmSFA, &full[stage], 0, (int)((sfa_tile * p.katoms + ka) * 2));
                    tma_load_2d_pair(sSFB, &tmSFB, &full[stage], 0, (int)((sfb_tile * p.katoms + ka) * 2));
                    tma_load_2d_pair(sSFB + C::APK * 512, &tmSFB, &full[stage], 0,
                                     (int)(((sfb_tile + 1) * p.katoms + ka) * 2));
                    if (++stage == C::STAGES) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
            }
            // drain: the pair's MMAs have consumed (so the copies have landed in) every stage this CTA filled
            for (int s = 0; s < C::STAGES; ++s)
                if (armed & (1u << s))
                    wait_bounded(&empty[s], (armed_phase >> s) & 1u, abort, false);
        }
        __syncwarp();
    } else if (warp == 1) {
        // ---------------------------------------------------------------- MMA issuer (leader, one warp)
        // The whole warp polls the barriers and runs the loop; one elected lane issues.
        if (rank == 0) {
            const uint32_t tm_sf = tmem_base + C::BN;
            int stage = 0;
            uint32_t phase = 0, sfsel = 0;
            int it = 0;
            bool ok = true;
            for (int64_t w = pair; w < p.work && ok; w += npairs, ++it) {
                if (!(ok = !meet_or(false)))  // the waiter saw both CTAs' epilogues release the accumulator
                    break;
                tc_fence_after();
                for (int kt = 0; kt < p.nk; ++kt) {
                    if (!(ok = !meet_or(false)))  // the waiter saw both CTAs' stage bytes land
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
                        const int a = C::NV ? kb : kb >> 1;
                        if (C::NV || (kb & 1) == 0) {
                            // each CTA copies its own scale A atom and both 128-row scale B atoms
                            tc_cp_atom_pair_w(tm_sfa + a * 4, desc_sf_atom(smem_u32(sSFA + a * 512)));
                            tc_cp_atom_pair_w(tm_sfb + a * 8, desc_sf_atom(smem_u32(sSFB + a * 512)));
                            tc_cp_atom_pair_w(tm_sfb + a * 8 + 4, desc_sf_atom(smem_u32(sSFB + (C::APK + a) * 512)));
                        }
                        uint32_t sfa, sfb, idesc;
                        if (C::NV) {
                            sfa = tm_sfa + kb * 4;
                            sfb = tm_sfb + kb * 8;
                            idesc = C::IDESC;
                        } else {
                            const uint32_t byte = (uint32_t)(kb & 1) * 2u;
                            sfa = (tm_sfa + a * 4) | (byte << 30);
                            sfb = (tm_sfb + a * 8) | (byte << 30);
                            idesc = C::IDESC | (byte << 29) | (byte << 4);
                        }
                        tc_mma_pair_w<C::NV>(tmem_base, dA + (uint64_t)(kb * 2), dB + (uint64_t)(kb * 2), idesc, sfa,
                                             sfb, (kt > 0 || kb > 0) ? 1u : 0u);
                    }
                    tc_commit_pair_w(&empty[stage]);
                    if (++stage == C::STAGES) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
                if (!ok)
                    break;
                tc_commit_pair_w(acc_full);
            }
            tc_commit_pair_w(done_bar);
        }
        // both CTAs: every MMA of the pair has completed before TMEM or shared memory is released
        if (lane == 0)
            wait_bounded(done_bar, 0, abort, false);
        __syncwarp();
    } else if (warp == C::WAITER_WARP) {
        // ---------------------------------------------------------------- waiter (leader, one warp)
        // The MMA warp's barrier waits, one step ahead of it, each followed by a meeting at
        // named barrier 2 that passes on a wait that gave up.
        if (rank == 0) {
            int stage = 0;
            uint32_t phase = 0;
            int it = 0;
            bool ok = true;
            for (int64_t w = pair; w < p.work && ok; w += npairs, ++it) {
                if (meet_or(!warp_poll_cluster(acc_empty, ((uint32_t)it & 1u) ^ 1u, abort, lane))) {
                    ok = false;
                    break;
                }
                for (int kt = 0; kt < p.nk; ++kt) {
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
        }
    } else {
        // ---------------------------------------------------------------- epilogue (both CTAs)
        const int quad = warp & 3;
        const int half = (warp - 2) >> 2;
        const float gg = C::NV ? __fmul_rn(*p.g_a, *p.g_w) : 1.0f;
        int it = 0;
        for (int64_t w = pair; w < p.work; w += npairs, ++it) {
            int mt, nt;
            pair_tile_coords(p, w, mt, nt);
            if (!warp_poll(acc_full, (uint32_t)it & 1u, abort, lane))
                break;
            tc_fence_after();
            float v[C::COLS_PER_WARP];
            const uint32_t taddr = tmem_base + ((uint32_t)(quad * 32) << 16) + half * C::COLS_PER_WARP;
#pragma unroll
            for (int c = 0; c < C::COLS_PER_WARP; c += 32)
                tmem_ld32(taddr + c, v + c);
            tc_fence_before();
            __syncwarp();
            if (lane == 0)
                mbar_arrive_leader(acc_empty);  // this warp's part of the accumulator is free

            const int64_t m = (int64_t)mt * C::BM + rank * C::CM + quad * 32 + lane;
            const int64_t n0 = (int64_t)nt * C::BN + half * C::COLS_PER_WARP;
            if (m < p.M) {
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
                            __nv_bfloat162 b2 = __floats2bfloat162_rn(__fmul_rn(v[c + 2 * j], gg),
                                                                      __fmul_rn(v[c + 2 * j + 1], gg));
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
                                __nv_bfloat162 b2 = __floats2bfloat162_rn(__fmul_rn(v[c + h + 2 * j], gg),
                                                                          __fmul_rn(v[c + h + 2 * j + 1], gg));
                                w4[j] = *reinterpret_cast<uint32_t *>(&b2);
                            }
                            st_v4(yr + n + h, make_uint4(w4[0], w4[1], w4[2], w4[3]));
                        } else {
                            for (int j = 0; j < 8; ++j)
                                if (n + h + j < p.N)
                                    yr[n + h + j] = __float2bfloat16_rn(__fmul_rn(v[c + h + j], gg));
                        }
                    }
                }
            }
        }
    }

    tc_fence_before();
    cluster_sync_all();  // no CTA frees TMEM or leaves while its peer may still signal or read it
    if (warp == 1) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(tmem_base),
                     "r"((uint32_t)C::TMEM_COLS)
                     : "memory");
    }
    cluster_sync_all();
}

}  // namespace fp4lin
