// Grouped GEMM on CTA pairs (tcgen05 cta_group::2): the same computation as grouped_gemm_kernel (see
// gemm.cuh), with 256-row tiles computed by the two CTAs of a cluster as one M=256 MMA.
//
// Why: with one CTA per tile every SM must pull a 128 x 64 A block and a BN x 64 B block per K step,
// 96 bytes per clock at full tensor rate. A pair shares B: each CTA loads its own 128 A rows and half of
// the B rows (BN/2), 64 bytes per clock, so the shared-memory ring can be deeper (6 stages) for the same
// bytes and the L2 -> SM traffic per FLOP drops by a third.
//
// Roles (192 threads per CTA, both CTAs of the pair):
//   warp 0     TMA producer of this CTA's A rows and B half; completion is counted on the pair leader's
//              full[stage] (the leader alone arms it with both CTAs' bytes); each CTA waits on its own
//              empty[stage], which the leader's MMA thread releases in both CTAs at once.
//   warp 1     TMEM allocation (mirrored in both CTAs). In the leader, one lane issues
//              tcgen05.mma.cta_group::2 M=256 N=BN K=16 x4 per stage and signals tmem_full in both CTAs.
//   warps 2-5  epilogue of this CTA's 128 rows (its TMEM lanes), as in the single-CTA kernel; they release
//              the accumulator by arriving on the leader's tmem_empty (8 arrivals: 4 warps x 2 CTAs).
// Gate|up: the leader's B half holds the BN/2 gate rows and the peer's the matching up rows, so the
// accumulator of both CTAs holds [gate | up] for their own rows, exactly as in the single-CTA layout.
// No load uses multicast; each CTA reads its own data.
#pragma once
#include "common.cuh"
#include "gemm.cuh"

namespace moe {

constexpr int GP_BM = 256;  // rows per pair tile (128 per CTA)

// SUB: 64-wide K blocks per ring stage. Two halve the barrier round trips per FLOP (8 MMAs per stage); measured
// faster for gate|up from K = 2048 on.
template <int BN, int STAGES, bool GATEUP, int SUB = 1>
struct GemmPairShape {
    static_assert(BN % 32 == 0 || (!GATEUP && BN % 16 == 0), "tile width");
    static_assert(BN >= 64 && BN <= 256, "UMMA N for M=256 (cta_group::2) is a multiple of 16 up to 256");
    static_assert(!GATEUP || (BN / 2) % 32 == 0, "gate|up halves must be whole 32-column TMEM loads");
    static_assert((BN / 2) % 8 == 0, "each CTA's B half must be whole 8-row swizzle atoms");
    static constexpr int A_BYTES = 128 * GG_BK * 2;
    static constexpr int B_BYTES = (BN / 2) * GG_BK * 2;
    static constexpr int SUB_BYTES = A_BYTES + B_BYTES;
    static constexpr int STAGE_BYTES = SUB * SUB_BYTES;
    static_assert(SUB_BYTES % 1024 == 0, "sub-block bases stay 1024-byte aligned");
    static constexpr int OUT_COLS = GATEUP ? BN / 2 : BN;
    static constexpr int TMEM_COLS = 2 * BN <= 128 ? 128 : (2 * BN <= 256 ? 256 : 512);
    static constexpr int BAR_BYTES = 256;
    static constexpr int TABLE_BYTES = (2 * (GG_MAX_GROUPS + 1) * 4 + 127) / 128 * 128;
    static constexpr int EPI_BYTES = 4 * 2 * 2048;  // per epilogue warp, two store staging buffers
    static_assert((STAGES * STAGE_BYTES) % 1024 == 0, "staging buffers (after the ring) stay 1024-byte aligned");
    static constexpr int SMEM_BYTES = 1024 + STAGES * STAGE_BYTES + EPI_BYTES + BAR_BYTES + TABLE_BYTES;
    static_assert(SMEM_BYTES <= 232448, "shared memory");
    static_assert((2 * STAGES + 6) * 8 + 8 <= BAR_BYTES, "barrier area");
};

template <int BN, int STAGES, bool GATEUP, int SUB = 1>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(GG_THREADS, 1)
    grouped_gemm_pair_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                             const __grid_constant__ CUtensorMap tmO, const GemmArgs args, int weights_streamed_once) {
    // tmO: the output [M][n_out], 32 x 32 boxes, 64-byte swizzle (TMA stores of whole epilogue blocks)
    using S = GemmPairShape<BN, STAGES, GATEUP, SUB>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    uint8_t* stages = smem;
    uint8_t* epi_stage = smem + STAGES * S::STAGE_BYTES;  // [4 warps][2][2048]
    uint64_t* full_bar = reinterpret_cast<uint64_t*>(smem + STAGES * S::STAGE_BYTES + S::EPI_BYTES);  // leader
    uint64_t* empty_bar = full_bar + STAGES;
    uint64_t* tfull_bar = empty_bar + STAGES;
    uint64_t* tempty_bar = tfull_bar + 2;  // used in the leader
    uint64_t* final_bar = tempty_bar + 2;
    uint64_t* never_bar = final_bar + 1;  // nothing arrives on it (test_stall)
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(never_bar + 1);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
    int32_t* s_off = reinterpret_cast<int32_t*>(smem + STAGES * S::STAGE_BYTES + S::EPI_BYTES + S::BAR_BYTES);
    int32_t* s_tp = s_off + (GG_MAX_GROUPS + 1);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t rank = cluster_ctarank();
    const bool leader = rank == 0;
    const int cluster = blockIdx.x >> 1, n_clusters = gridDim.x >> 1;
    const int G = args.G;
    const int KB = (args.K + GG_BK * SUB - 1) / (GG_BK * SUB);  // ring stages per tile

    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(&full_bar[s], 1);
            mbar_init(&empty_bar[s], 1);
        }
        for (int a = 0; a < 2; ++a) {
            mbar_init(&tfull_bar[a], 1);
            mbar_init(&tempty_bar[a], 8);
        }
        mbar_init(final_bar, 1);
        mbar_init(never_bar, 1);
        *abort_flag = 0;
        fence_mbar_init();
        tma_prefetch_desc(&tmA);
        tma_prefetch_desc(&tmB);
        tma_prefetch_desc(&tmO);
    }
    if (warp == 1) {
        tmem_alloc_pair(tmem_slot, S::TMEM_COLS);
        tmem_relinquish_pair();
    }
    grid_dep_wait();  // inputs below come from earlier kernels in the stream
    grid_dep_trigger();
    for (int g = threadIdx.x; g <= G; g += GG_THREADS) {
        int v = args.group_offsets[g];
        if (v < 0 || v > args.M) {
            flag_error(MOE_DEVERR_GROUP_RANGE);
            v = min(max(v, 0), args.M);
        }
        s_off[g] = v;
    }
    __syncthreads();
    if (warp == 0) {  // tile prefix over groups: tiles(g) = ceil(rows / 256) * n_tiles
        const int per = (G + 31) / 32;
        const int g0 = lane * per, g1 = min(g0 + per, G);
        int local = 0;
        for (int g = g0; g < g1; ++g) {
            const int rows = s_off[g + 1] - s_off[g];
            if (rows < 0) flag_error(MOE_DEVERR_GROUP_RANGE);
            local += (max(rows, 0) + GP_BM - 1) / GP_BM * args.n_tiles;
        }
        int incl = local;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int v = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += v;
        }
        int run = incl - local;
        for (int g = g0; g < g1; ++g) {
            s_tp[g] = run;
            run += (max(s_off[g + 1] - s_off[g], 0) + GP_BM - 1) / GP_BM * args.n_tiles;
        }
        if (lane == 31) s_tp[G] = incl;
    }
    tc_fence_before_sync();
    __syncthreads();
    cluster_sync();  // both CTAs' barriers are initialised before any cross-CTA arrive or TMA signal
    tc_fence_after_sync();
    const uint32_t tmem_base = *tmem_slot;
    const int total = s_tp[G];

    auto locate = [&](int tile, int& g, int& nb, int& mb) {
        int lo = 0, hi = G - 1;
        while (lo < hi) {
            const int mid = (lo + hi + 1) >> 1;
            if (s_tp[mid] <= tile)
                lo = mid;
            else
                hi = mid - 1;
        }
        g = lo;
        const int mt = (max(s_off[g + 1] - s_off[g], 0) + GP_BM - 1) / GP_BM;
        const int local = tile - s_tp[g];
        nb = local / mt;
        mb = local - nb * mt;
    };

    if (warp == 0) {
        // ---------------- TMA producer (both CTAs) ----------------
        const uint64_t pol_a = l2_policy_evict_last();
        const uint64_t pol_b = weights_streamed_once ? l2_policy_evict_first() : l2_policy_evict_normal();
        int stage = 0;
        uint32_t phase = 0;
        long issued = 0;
        bool ok = true;
        for (int tile = cluster; tile < total && ok; tile += n_clusters) {
            int g, nb, mb;
            locate(tile, g, nb, mb);
            const int row0 = s_off[g] + mb * GP_BM + (int)rank * 128;
            int brow;
            if constexpr (GATEUP)
                brow = (rank ? args.f : 0) + nb * (BN / 2);
            else
                brow = nb * BN + (int)rank * (BN / 2);
            for (int kb = 0; kb < KB; ++kb) {
                if (lane == 0) ok = mbar_wait_bounded(&empty_bar[stage], phase ^ 1u, abort_flag);
                ok = __shfl_sync(0xffffffffu, ok, 0);
                if (!ok) break;
                if (lane == 0) {
                    uint8_t* sa = stages + stage * S::STAGE_BYTES;
                    const uint32_t bar = mapa_shared(smem_u32(&full_bar[stage]), 0);
                    if (leader) mbar_arrive_expect_tx(&full_bar[stage], 2 * S::STAGE_BYTES);
#pragma unroll
                    for (int sb = 0; sb < SUB; ++sb) {  // K past the end arrives as zeros
                        const int kc = (kb * SUB + sb) * GG_BK;
                        tma_load_2d_pair(sa + sb * S::SUB_BYTES, &tmA, bar, kc, row0, pol_a);
                        tma_load_3d_pair(sa + sb * S::SUB_BYTES + S::A_BYTES, &tmB, bar, kc, brow, g, pol_b);
                    }
                }
                ++issued;
                if (++stage == STAGES) {
                    stage = 0;
                    phase ^= 1u;
                }
            }
        }
        // the leader's full barriers count both CTAs' copies: it waits for the last ones (bounded)
        if (lane == 0 && leader) {
            for (long n = issued > STAGES ? issued - STAGES : 0; n < issued; ++n)
                mbar_wait_drain(&full_bar[n % STAGES], (uint32_t)((n / STAGES) & 1));
        }
        __syncwarp();
    } else if (warp == 1) {
        // ---------------- MMA issuer (leader only) ----------------
        if (leader) {
            constexpr uint32_t IDESC = idesc_bf16_f32(GP_BM, BN);
            int stage = 0, acc = 0;
            uint32_t phase = 0, acc_phase = 0;
            bool ok = true;
            if (lane == 0) ok = test_stall(never_bar, abort_flag);
            ok = __shfl_sync(0xffffffffu, ok, 0);
            for (int tile = cluster; tile < total && ok; tile += n_clusters) {
                if (lane == 0) ok = mbar_wait_bounded(&tempty_bar[acc], acc_phase ^ 1u, abort_flag);
                ok = __shfl_sync(0xffffffffu, ok, 0);
                if (!ok) break;
                tc_fence_after_sync();
                const uint32_t d_tmem = tmem_base + (uint32_t)(acc * BN);
                for (int kb = 0; kb < KB; ++kb) {
                    if (lane == 0) ok = mbar_wait_bounded(&full_bar[stage], phase, abort_flag);
                    ok = __shfl_sync(0xffffffffu, ok, 0);
                    if (!ok) break;
                    tc_fence_after_sync();
                    if (lane == 0) {
#pragma unroll
                        for (int sb = 0; sb < SUB; ++sb) {
                            const uint32_t sa = smem_u32(stages + stage * S::STAGE_BYTES + sb * S::SUB_BYTES);
                            const uint64_t adesc = smem_desc_sw128(sa);
                            const uint64_t bdesc = smem_desc_sw128(sa + S::A_BYTES);
#pragma unroll
                            for (int k = 0; k < GG_BK / 16; ++k)
                                umma_bf16_ss_pair(d_tmem, adesc + 2 * k, bdesc + 2 * k, IDESC,
                                                  (kb | sb | k) != 0 ? 1u : 0u);
                        }
                        umma_commit_pair_multicast(&empty_bar[stage], 0x3);
                    }
                    __syncwarp();
                    if (++stage == STAGES) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
                if (!ok) break;
                if (lane == 0) umma_commit_pair_multicast(&tfull_bar[acc], 0x3);
                __syncwarp();
                acc ^= 1;
                if (acc == 0) acc_phase ^= 1u;
            }
            if (lane == 0) umma_commit_pair(final_bar);
            __syncwarp();
        }
    } else {
        // ---------------- epilogue (warps 2-5, both CTAs) ----------------
        const int q = warp & 3;
        const uint32_t tempty_leader0 = mapa_shared(smem_u32(&tempty_bar[0]), 0);
        const uint32_t tempty_leader1 = mapa_shared(smem_u32(&tempty_bar[1]), 0);
        int acc = 0;
        uint32_t acc_phase = 0;
        bool ok = true;
        uint32_t blocks = 0;  // output blocks this warp has staged (alternating buffers)
        for (int tile = cluster; tile < total; tile += n_clusters) {
            int g, nb, mb;
            locate(tile, g, nb, mb);
            const int row_end = s_off[g + 1];
            const int row_base = s_off[g] + mb * GP_BM + (int)rank * 128 + q * 32;  // row of lane 0
            const bool rows_whole = row_base + 32 <= row_end;  // this warp's 32 rows all belong to the group
            if (lane == 0) ok = mbar_wait_bounded(&tfull_bar[acc], acc_phase, abort_flag);
            ok = __shfl_sync(0xffffffffu, ok, 0);
            if (!ok) break;
            tc_fence_after_sync();
            const uint32_t t_row = tmem_base + ((uint32_t)(q * 32) << 16) + (uint32_t)(acc * BN);
            const int col_base = nb * S::OUT_COLS;
#pragma unroll 1
            for (int c0 = 0; c0 < S::OUT_COLS; c0 += 32) {
                const int col0 = col_base + c0;
                if (col0 >= args.n_out) break;  // warp-uniform
                uint32_t pk[16];
                if constexpr (GATEUP) {
                    uint32_t gv[32], uv[32];
                    tmem_load_32cols(t_row + c0, gv);
                    tmem_load_32cols(t_row + BN / 2 + c0, uv);
#pragma unroll
                    for (int i = 0; i < 16; ++i) {
                        const float g0 = __uint_as_float(gv[2 * i]), g1 = __uint_as_float(gv[2 * i + 1]);
                        const float u0 = __uint_as_float(uv[2 * i]), u1 = __uint_as_float(uv[2 * i + 1]);
                        pk[i] = pack_bf16x2(swiglu(g0, u0), swiglu(g1, u1));
                    }
                } else {
                    uint32_t v[32];
                    tmem_load_32cols(t_row + c0, v);
#pragma unroll
                    for (int i = 0; i < 16; ++i)
                        pk[i] = pack_bf16x2(__uint_as_float(v[2 * i]), __uint_as_float(v[2 * i + 1]));
                }
                uint8_t* my_stage = epi_stage + ((warp - 2) * 2 + (int)(blocks & 1u)) * 2048;
                ++blocks;
                if (lane == 0) bulk_wait_group_read<1>();  // the TMA store that last read this buffer is done
                __syncwarp();
                if (rows_whole && S::OUT_COLS - c0 >= 32)
                    store_warp_block_tma(my_stage, pk, lane, &tmO, row_base, col0);
                else {
                    store_warp_rows_32cols(my_stage, pk, lane, args.out, args.n_out, row_base, row_end, col0,
                                           args.n_out, S::OUT_COLS - c0);
                    if (lane == 0) bulk_commit_group();  // an empty group: one group per staged block
                }
            }
            tc_fence_before_sync();
            __syncwarp();
            if (lane == 0) mbar_arrive_cluster(acc ? tempty_leader1 : tempty_leader0);
            acc ^= 1;
            if (acc == 0) acc_phase ^= 1u;
        }
        if (lane == 0) bulk_wait_all();  // the output stores have landed before the CTA leaves
        __syncwarp();
    }

    tc_fence_before_sync();
    __syncthreads();
    if (warp == 1 && leader) {
        if (lane == 0) mbar_wait_drain(final_bar, 0);  // the pair's MMAs have finished
        __syncwarp();
    }
    cluster_sync();  // no CTA leaves while its peer may still signal its barriers or read its smem
    tc_fence_after_sync();
    if (warp == 1) tmem_dealloc_pair(tmem_base, S::TMEM_COLS);
}

}  // namespace moe
