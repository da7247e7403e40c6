// gemm_sm100_2sm_decode.cuh -- the decode-sized GEMM (M <= 16 activation rows) on CTA pairs.
//
// The decode form computes y^T = W A^T: the weights are the MMA's M side, the few activation
// rows its N side (N = 16).  On one CTA every 128 weight rows cost the issuing thread a scale
// copy for the weights, one for the activations and one MMA per 64 values of K, and that
// thread, not DRAM, bounds the decode GEMM.  A CTA pair runs tcgen05.mma.cta_group::2 with
// M = 256: the leader issues one scale-A copy (each CTA copies its own 128 rows), one scale-B
// copy and one MMA for 256 weight rows -- half the instructions per weight row.
//
// Measured, it is slower than the one-CTA form (16x14336x4096: 18.5 against 15.8 us, both
// issuing from a converged warp with a waiter warp): the pair's completions on the leader's
// barriers and its cluster-wide hand-offs cost more than the instructions it saves, so it
// runs only when FP4LIN_DECODE_KERNEL=pair asks for it.  Its results are the same, bit for bit.
//
// Roles (352 threads per CTA, both CTAs of the pair):
//   warp 0 lane 0   producer: TMA loads of this CTA's 128 weight rows, its 8 of the 16
//                   activation rows, its weight scale atoms and all activation scale atoms
//                   (every CTA's TMEM needs them), completing on the LEADER's `full` barrier;
//   warp 1          TMEM (cta_group::2 alloc/dealloc); in the leader the converged warp issues
//                   (one elected lane) the pair's copies and MMAs and commits, multicast to
//                   both CTAs' barriers;
//   warps 2..9      epilogue of this CTA's 128 weight rows: y (transposed) or, with a K split,
//                   binary32 partial sums for splitk_reduce_kernel;
//   warp 10         in the leader, waits on the barriers for the MMA warp and meets it at a
//                   named barrier.
// Two accumulators (16 columns each) let a pair start its next item while the previous one
// drains.  All waits are bounded.  No load uses multicast.
#pragma once

#include "gemm_sm100_2sm.cuh"

namespace fp4lin {

template <bool NV_>
struct GemmDecodePairCfg {
    static constexpr bool NV = NV_;
    static constexpr bool FUSEQ = false;
    static constexpr int BM = 256, BN = 16;                 // pair tile: weight rows x activation rows
    static constexpr int CM = 128, CN = 8;                  // rows of A / B in each CTA
    static constexpr int BK = 256, MMA_K = 64;
    static constexpr int APK = NV ? BK / 64 : BK / 128;
    static constexpr int SF_BOX_ROWS = APK * 2;
    static constexpr int A_BYTES = CM * 128, B_BYTES = 1024;  // 8 rows x 128 B: one 1024-byte swizzle atom
    static constexpr int SFA_BYTES = APK * 512, SFB_BYTES = APK * 512;
    static constexpr int STAGE_BYTES = A_BYTES + B_BYTES + SFA_BYTES + SFB_BYTES;
    static constexpr int STAGES = 8;
    static constexpr int TX_BYTES = 2 * STAGE_BYTES;
    static constexpr int NUM_ACC = 2;
    static constexpr int SFA_COLS = APK * 4, SFB_COLS = APK * 4, SF_COLS = SFA_COLS + SFB_COLS;
    static constexpr int TMEM_USED = NUM_ACC * BN + 2 * SF_COLS;
    static constexpr int TMEM_COLS = TMEM_USED <= 64 ? 64 : TMEM_USED <= 128 ? 128 : 256;
    static constexpr int EPI_WARPS = 8;
    static constexpr int WAITER_WARP = 2 + EPI_WARPS;    // the leader's barrier waits for its MMA warp
    static constexpr int THREADS = 64 + EPI_WARPS * 32 + 32;
    static constexpr int COLS_PER_WARP = BN / 2;
    static constexpr int BAR_BYTES = 256;
    static constexpr int SMEM_BYTES = STAGES * STAGE_BYTES + BAR_BYTES + 1024;
    static constexpr uint32_t IDESC = (1u << 7) | (1u << 10) | ((uint32_t)(BN >> 3) << 17) |
                                      ((NV ? 0u : 1u) << 23) | ((uint32_t)(BM >> 4) << 24);
    static_assert(TMEM_USED <= 256, "TMEM overflow");
    static_assert(SMEM_BYTES <= 232448, "shared memory overflow");
    static_assert(STAGE_BYTES % 1024 == 0, "stages must keep the 1024-byte alignment of the swizzled tiles");
};

struct GemmDecodePairParams {
    const float *g_a, *g_w;     // swapped slots: g_a the weights' scale, g_w the activations'
    __nv_bfloat16 *y;           // [Mact, ldy] (y[m, n], n the weight row)
    float *ws;                  // split partials [splits, Mact, ldw]
    int64_t Nw, Mact, K, ldy, ldw;
    int64_t katoms;             // weight scale atoms per 128-row tile along K
    int64_t katoms_act;         // activation scale atoms per 128-row tile along K
    int num_mt, nk, kps, splits;
    int64_t work;               // num_mt * splits
};

template <class C>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(C::THREADS, 1)
    fp4_gemm_decode_pair_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                                const __grid_constant__ CUtensorMap tmSFA, const __grid_constant__ CUtensorMap tmSFB,
                                GemmDecodePairParams p)
{
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
    uint8_t *bar_area = smem + C::STAGES * C::STAGE_BYTES;
    uint64_t *full = reinterpret_cast<uint64_t *>(bar_area);  // leader's copy counts both CTAs' bytes
    uint64_t *empty = full + C::STAGES;                         // both CTAs: stage consumed by the pair's MMAs
    uint64_t *acc_full = empty + C::STAGES;                     // both CTAs: accumulator complete [NUM_ACC]
    uint64_t *acc_empty = acc_full + C::NUM_ACC;                // leader: both CTAs' epilogues have read it
    uint64_t *done_bar = acc_empty + C::NUM_ACC;                // both CTAs: every MMA of the pair completed
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(done_bar + 1);
    volatile int *abort = reinterpret_cast<volatile int *>(tmem_slot + 1);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t rank = cluster_ctarank();
    const int64_t pair = blockIdx.x >> 1, npairs = gridDim.x >> 1;

    if (threadIdx.x == 0) {
        pdl_trigger();  // the split-K reduction may launch now; it waits for this grid to finish
        for (int s = 0; s < C::STAGES; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        for (int a = 0; a < C::NUM_ACC; ++a) {
            mbar_init(&acc_full[a], 1);
            mbar_init(&acc_empty[a], 2 * C::EPI_WARPS);
        }
        mbar_init(done_bar, 1);
        *abort = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (warp == 1) {
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
                const int mt = (int)(w % p.num_mt), sp = (int)(w / p.num_mt);
                const int kt0 = sp * p.kps, kt1 = min(p.nk, kt0 + p.kps);
                const int a_row = mt * C::BM + (int)rank * C::CM;
                const int64_t sfa_tile = (int64_t)mt * 2 + rank;
                for (int kt = kt0; kt < kt1; ++kt) {
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
                    tma_load_2d_pair(sB, &tmB, &full[stage], kt * 128, (int)rank * C::CN);
                    // scale atoms as rows of 256 bytes: atom j of row tile t starts at row 2 (t katoms + j)
                    tma_load_2d_pair(sSFA, &tmSFA, &full[stage], 0, (int)((sfa_tile * p.katoms + ka) * 2));
                    tma_load_2d_pair(sSFB, &tmSFB, &full[stage], 0, (int)(ka * 2));  // row tile 0: the 16 rows
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
        // The converged warp runs the loop and one elected lane issues; the waiter warp does the
        // barrier waits and meets this warp at named barrier 2 (as in the prefill kernels).
        if (rank == 0) {
            const uint32_t tm_sf = tmem_base + C::NUM_ACC * C::BN;
            int stage = 0;
            uint32_t phase = 0, sfsel = 0;
            int it = 0;
            bool ok = true;
            for (int64_t w = pair; w < p.work && ok; w += npairs, ++it) {
                const int sp = (int)(w / p.num_mt);
                const int kt0 = sp * p.kps, kt1 = min(p.nk, kt0 + p.kps);
                const int acc = it & 1;
                if (!(ok = !meet_or(false)))  // the waiter saw both CTAs' epilogues release the accumulator
                    break;
                tc_fence_after();
                const uint32_t d_tmem = tmem_base + acc * C::BN;
                for (int kt = kt0; kt < kt1; ++kt) {
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
                            // each CTA copies its own weight scale atom and the activation scale atom
                            tc_cp_atom_pair_w(tm_sfa + a * 4, desc_sf_atom(smem_u32(sSFA + a * 512)));
                            tc_cp_atom_pair_w(tm_sfb + a * 4, desc_sf_atom(smem_u32(sSFB + a * 512)));
                        }
                        uint32_t sfa, sfb, idesc;
                        if (C::NV) {
                            sfa = tm_sfa + kb * 4;
                            sfb = tm_sfb + kb * 4;
                            idesc = C::IDESC;
                        } else {
                            const uint32_t byte = (uint32_t)(kb & 1) * 2u;
                            sfa = (tm_sfa + a * 4) | (byte << 30);
                            sfb = (tm_sfb + a * 4) | (byte << 30);
                            idesc = C::IDESC | (byte << 29) | (byte << 4);
                        }
                        tc_mma_pair_w<C::NV>(d_tmem, dA + (uint64_t)(kb * 2), dB + (uint64_t)(kb * 2), idesc, sfa,
                                             sfb, (kt > kt0 || kb > 0) ? 1u : 0u);
                    }
                    tc_commit_pair_w(&empty[stage]);
                    if (++stage == C::STAGES) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
                if (!ok)
                    break;
                tc_commit_pair_w(&acc_full[acc]);
            }
            tc_commit_pair_w(done_bar);
        }
        // both CTAs: every MMA of the pair has completed before TMEM or shared memory is released
        if (lane == 0)
            wait_bounded(done_bar, 0, abort, false);
        __syncwarp();
    } else if (warp == C::WAITER_WARP) {
        // ---------------------------------------------------------------- waiter (leader, one warp)
        if (rank == 0) {
            int stage = 0;
            uint32_t phase = 0;
            int it = 0;
            bool ok = true;
            for (int64_t w = pair; w < p.work && ok; w += npairs, ++it) {
                const int sp = (int)(w / p.num_mt);
                const int kt0 = sp * p.kps, kt1 = min(p.nk, kt0 + p.kps);
                const int acc = it & 1;
                if (meet_or(!warp_poll_cluster(&acc_empty[acc], ((uint32_t)(it >> 1) & 1u) ^ 1u, abort, lane))) {
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
        }
    } else {
        // ---------------------------------------------------------------- epilogue (both CTAs)
        const int quad = warp & 3;
        const int half = (warp - 2) >> 2;
        const float gg = C::NV ? __fmul_rn(*p.g_a, *p.g_w) : 1.0f;
        int it = 0;
        for (int64_t w = pair; w < p.work; w += npairs, ++it) {
            const int mt = (int)(w % p.num_mt), sp = (int)(w / p.num_mt);
            const int acc = it & 1;
            if (!warp_wait(&acc_full[acc], (uint32_t)(it >> 1) & 1u, abort, lane))
                break;
            tc_fence_after();
            float v[C::COLS_PER_WARP];
            tmem_ld8(tmem_base + ((uint32_t)(quad * 32) << 16) + acc * C::BN + half * C::COLS_PER_WARP, v);
            tc_fence_before();
            __syncwarp();
            if (lane == 0)
                mbar_arrive_leader(&acc_empty[acc]);  // this warp's part of the accumulator is free
            // accumulator row = weight row n, column = activation row m: y[m, n]
            const int64_t n = (int64_t)mt * C::BM + rank * C::CM + quad * 32 + lane;
            if (n < p.Nw) {
#pragma unroll
                for (int c = 0; c < C::COLS_PER_WARP; ++c) {
                    const int64_t m = half * C::COLS_PER_WARP + c;
                    if (m < p.Mact) {
                        if (p.splits == 1)
                            p.y[m * p.ldy + n] = __float2bfloat16_rn(__fmul_rn(v[c], gg));
                        else
                            p.ws[((int64_t)sp * p.Mact + m) * p.ldw + n] = v[c];
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
