// Grouped GEMM on CTA pairs with 2*NH-wide tiles: the same computation as grouped_gemm_pair_kernel (see
// gemm_pair.cuh) with half the A traffic per FLOP.
//
// Why: one A block (128 rows x 64 of this CTA) feeds two tcgen05.mma.cta_group::2 of N = NH each, into two
// TMEM accumulators, so a K step moves A 16 KB + B NH*128 bytes per CTA for twice the FLOPs of a 256 x 256 pair
// tile, and each barrier round trip of the shared-memory ring covers 8 MMAs instead of 4. The price: the two
// accumulators fill TMEM (2*NH <= 512 columns), so the epilogue of a tile cannot overlap the next tile's
// mainloop; it is spread over 8 warps to keep it short. Measured on B200: faster than the double-buffered pair
// tile on long reductions, slower on short ones, which is how the host chooses (gate|up from K = 8192, the
// down projection from K = 2048).
//
// Column mapping. Each CTA's B buffer holds NH rows; MMA a (a = 0, 1) reads rows [a*NH/2, (a+1)*NH/2) of
// both CTAs' buffers (the leader's first, then the peer's), so accumulator a, column c = h*NH/2 + cc
// (h = 0 leader half, 1 peer half) holds:
//   gate|up: h = 0 -> gate column a*NH/2 + cc of the tile, h = 1 -> the matching up column (the leader loads
//            NH gate rows, the peer the NH up rows), so the tile produces NH columns of silu(gate) * up;
//   down:    output column h*NH + a*NH/2 + cc of the tile's 2*NH columns (leader rows = the first NH output
//            columns, peer rows = the next NH).
//
// Roles (320 threads per CTA, both CTAs): warp 0 TMA producer (this CTA's A rows + its NH B rows, counted
// on the leader's full barrier), warp 1 TMEM allocation and, in the leader, the MMA issuer; warps 2-9 the
// epilogue: warps 2-5 drain accumulator 0, warps 6-9 accumulator 1, each warp its 32 TMEM lanes.
// No load uses multicast.
#pragma once
#include "common.cuh"
#include "gemm.cuh"
#include "gemm_pair.cuh"

namespace moe {

constexpr int GW_THREADS = 320;

template <int NH, int STAGES, bool GATEUP>
struct GemmWideShape {
    static_assert(NH % 16 == 0 && NH >= 64 && NH <= 256, "UMMA N for M=256 (cta_group::2)");
    static_assert((NH / 2) % 8 == 0, "each MMA's B rows must be whole 8-row swizzle atoms");
    static constexpr int A_BYTES = 128 * GG_BK * 2;
    static constexpr int B_BYTES = NH * GG_BK * 2;
    static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
    static_assert(STAGE_BYTES % 1024 == 0, "stage bases stay 1024-byte aligned");
    static constexpr int OUT_COLS = GATEUP ? NH : 2 * NH;  // output columns per tile
    static constexpr int TMEM_COLS = 512;
    static_assert(2 * NH <= TMEM_COLS, "two accumulators");
    static constexpr int BAR_BYTES = 256;
    static constexpr int TABLE_BYTES = (2 * (GG_MAX_GROUPS + 1) * 4 + 127) / 128 * 128;
    static constexpr int EPI_BYTES = 8 * 2048;  // per-epilogue-warp store staging
    static_assert((STAGES * STAGE_BYTES + BAR_BYTES + TABLE_BYTES) % 128 == 0, "staging buffer alignment");
    static constexpr int SMEM_BYTES = 1024 + STAGES * STAGE_BYTES + BAR_BYTES + TABLE_BYTES + EPI_BYTES;
    static_assert(SMEM_BYTES <= 232448, "shared memory");
    static_assert((2 * STAGES + 5) * 8 + 8 <= BAR_BYTES, "barrier area");
};

// As store_warp_rows_32cols (gemm.cuh), but each 8-column piece u of the chunk has its own destination column
// piece_col[u] (or -1 when the piece is outside the tile).
__device__ __forceinline__ void store_warp_rows_pieces(uint8_t* stage, const uint32_t (&pk)[16], int lane,
                                                       __nv_bfloat16* out, int ld_out, int row_base, int row_end,
                                                       const int (&piece_col)[4], int n_out) {
#pragma unroll
    for (int v = 0; v < 4; ++v)
        *reinterpret_cast<uint4*>(stage + lane * 64 + ((v ^ ((lane >> 1) & 3)) << 4)) =
            make_uint4(pk[4 * v], pk[4 * v + 1], pk[4 * v + 2], pk[4 * v + 3]);
    __syncwarp();
    const int u = lane & 3;
    const int col = u == 0 ? piece_col[0] : (u == 1 ? piece_col[1] : (u == 2 ? piece_col[2] : piece_col[3]));
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const int row = i * 8 + (lane >> 2);
        const uint4 val = *reinterpret_cast<const uint4*>(stage + row * 64 + ((u ^ ((row >> 1) & 3)) << 4));
        const int grow = row_base + row;
        if (grow < row_end && col >= 0 && col < n_out)
            *reinterpret_cast<uint4*>(out + (size_t)grow * ld_out + col) = val;
    }
    __syncwarp();
}

template <int NH, int STAGES, bool GATEUP>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(GW_THREADS, 1)
    grouped_gemm_wide_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                             const GemmArgs args, int weights_streamed_once) {
    using S = GemmWideShape<NH, STAGES, GATEUP>;
    constexpr int HALF = NH / 2;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    uint8_t* stages = smem;
    uint64_t* full_bar = reinterpret_cast<uint64_t*>(smem + STAGES * S::STAGE_BYTES);  // used in the leader
    uint64_t* empty_bar = full_bar + STAGES;
    uint64_t* tfull_bar = empty_bar + STAGES;  // [1]
    uint64_t* tempty_bar = tfull_bar + 1;      // [1], used in the leader
    uint64_t* final_bar = tempty_bar + 1;
    uint64_t* never_bar = final_bar + 1;  // nothing arrives on it (test_stall)
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(never_bar + 1);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
    int32_t* s_off = reinterpret_cast<int32_t*>(smem + STAGES * S::STAGE_BYTES + S::BAR_BYTES);
    int32_t* s_tp = s_off + (GG_MAX_GROUPS + 1);
    uint8_t* epi_stage = smem + STAGES * S::STAGE_BYTES + S::BAR_BYTES + S::TABLE_BYTES;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t rank = cluster_ctarank();
    const bool leader = rank == 0;
    const int cluster = blockIdx.x >> 1, n_clusters = gridDim.x >> 1;
    const int G = args.G;
    const int KB = (args.K + GG_BK - 1) / GG_BK;

    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(&full_bar[s], 1);
            mbar_init(&empty_bar[s], 1);
        }
        mbar_init(tfull_bar, 1);
        mbar_init(tempty_bar, 16);  // 8 epilogue warps x 2 CTAs
        mbar_init(final_bar, 1);
        mbar_init(never_bar, 1);
        *abort_flag = 0;
        fence_mbar_init();
        tma_prefetch_desc(&tmA);
        tma_prefetch_desc(&tmB);
    }
    if (warp == 1) {
        tmem_alloc_pair(tmem_slot, S::TMEM_COLS);
        tmem_relinquish_pair();
    }
    grid_dep_wait();  // inputs below come from earlier kernels in the stream
    grid_dep_trigger();
    for (int g = threadIdx.x; g <= G; g += GW_THREADS) {
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
    cluster_sync();
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
            // gate|up: the leader loads NH gate rows, the peer the NH matching up rows; down: the leader
            // the tile's first NH output rows of W_down, the peer the next NH
            const int brow = GATEUP ? (rank ? args.f : 0) + nb * NH : nb * 2 * NH + (int)rank * NH;
            for (int kb = 0; kb < KB; ++kb) {
                if (lane == 0) ok = mbar_wait_bounded(&empty_bar[stage], phase ^ 1u, abort_flag);
                ok = __shfl_sync(0xffffffffu, ok, 0);
                if (!ok) break;
                if (lane == 0) {
                    uint8_t* sa = stages + stage * S::STAGE_BYTES;
                    const uint32_t bar = mapa_shared(smem_u32(&full_bar[stage]), 0);
                    if (leader) mbar_arrive_expect_tx(&full_bar[stage], 2 * S::STAGE_BYTES);
                    tma_load_2d_pair(sa, &tmA, bar, kb * GG_BK, row0, pol_a);
                    tma_load_3d_pair(sa + S::A_BYTES, &tmB, bar, kb * GG_BK, brow, g, pol_b);
                }
                ++issued;
                if (++stage == STAGES) {
                    stage = 0;
                    phase ^= 1u;
                }
            }
        }
        if (lane == 0 && leader) {
            for (long n = issued > STAGES ? issued - STAGES : 0; n < issued; ++n)
                mbar_wait_drain(&full_bar[n % STAGES], (uint32_t)((n / STAGES) & 1));
        }
        __syncwarp();
    } else if (warp == 1) {
        // ---------------- MMA issuer (leader only) ----------------
        if (leader) {
            constexpr uint32_t IDESC = idesc_bf16_f32(GP_BM, NH);
            int stage = 0;
            uint32_t phase = 0, tphase = 0;
            bool ok = true;
            if (lane == 0) ok = test_stall(never_bar, abort_flag);
            ok = __shfl_sync(0xffffffffu, ok, 0);
            for (int tile = cluster; tile < total && ok; tile += n_clusters) {
                if (lane == 0) ok = mbar_wait_bounded(tempty_bar, tphase ^ 1u, abort_flag);
                ok = __shfl_sync(0xffffffffu, ok, 0);
                if (!ok) break;
                tc_fence_after_sync();
                for (int kb = 0; kb < KB; ++kb) {
                    if (lane == 0) ok = mbar_wait_bounded(&full_bar[stage], phase, abort_flag);
                    ok = __shfl_sync(0xffffffffu, ok, 0);
                    if (!ok) break;
                    tc_fence_after_sync();
                    if (lane == 0) {
                        const uint32_t sa = smem_u32(stages + stage * S::STAGE_BYTES);
                        const uint64_t adesc = smem_desc_sw128(sa);
                        const uint64_t bdesc0 = smem_desc_sw128(sa + S::A_BYTES);
                        const uint64_t bdesc1 = smem_desc_sw128(sa + S::A_BYTES + HALF * GG_BK * 2);
                        // all K steps of one accumulator, then the other (measured faster than alternating)
#pragma unroll
                        for (int k = 0; k < GG_BK / 16; ++k)
                            umma_bf16_ss_pair(tmem_base, adesc + 2 * k, bdesc0 + 2 * k, IDESC, (kb | k) != 0 ? 1u : 0u);
#pragma unroll
                        for (int k = 0; k < GG_BK / 16; ++k)
                            umma_bf16_ss_pair(tmem_base + NH, adesc + 2 * k, bdesc1 + 2 * k, IDESC,
                                              (kb | k) != 0 ? 1u : 0u);
                        umma_commit_pair_multicast(&empty_bar[stage], 0x3);
                    }
                    __syncwarp();
                    if (++stage == STAGES) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
                if (!ok) break;
                if (lane == 0) umma_commit_pair_multicast(tfull_bar, 0x3);
                __syncwarp();
                tphase ^= 1u;
            }
            if (lane == 0) umma_commit_pair(final_bar);
            __syncwarp();
        }
    } else {
        // ---------------- epilogue (warps 2-9, both CTAs) ----------------
        const int q = warp & 3;          // TMEM lanes 32q .. 32q+31
        const int a = (warp - 2) >> 2;   // accumulator drained by this warp
        const uint32_t tempty_leader = mapa_shared(smem_u32(tempty_bar), 0);
        uint8_t* my_stage = epi_stage + (warp - 2) * 2048;
        uint32_t tphase = 0;
        bool ok = true;
        for (int tile = cluster; tile < total; tile += n_clusters) {
            int g, nb, mb;
            locate(tile, g, nb, mb);
            const int row_end = s_off[g + 1];
            const int row_base = s_off[g] + mb * GP_BM + (int)rank * 128 + q * 32;
            if (lane == 0) ok = mbar_wait_bounded(tfull_bar, tphase, abort_flag);
            ok = __shfl_sync(0xffffffffu, ok, 0);
            if (!ok) break;
            tc_fence_after_sync();
            const uint32_t t_acc = tmem_base + ((uint32_t)(q * 32) << 16) + (uint32_t)(a * NH);
            const int tile_col = nb * S::OUT_COLS;
            if constexpr (GATEUP) {
                // h columns tile_col + a*HALF + jj, jj < HALF: gate at accumulator column jj, up at HALF + jj
#pragma unroll 1
                for (int c0 = 0; c0 < HALF; c0 += 32) {
                    if (tile_col + a * HALF + c0 >= args.n_out) break;  // warp-uniform
                    uint32_t gv[32], uv[32], pk[16];
                    tmem_load_32cols(t_acc + c0, gv);
                    tmem_load_32cols(t_acc + HALF + c0, uv);
#pragma unroll
                    for (int i = 0; i < 16; ++i) {
                        const float g0 = __uint_as_float(gv[2 * i]), g1 = __uint_as_float(gv[2 * i + 1]);
                        const float u0 = __uint_as_float(uv[2 * i]), u1 = __uint_as_float(uv[2 * i + 1]);
                        pk[i] = pack_bf16x2(swiglu(g0, u0), swiglu(g1, u1));
                    }
                    int pc[4];
#pragma unroll
                    for (int u = 0; u < 4; ++u) {
                        const int jj = c0 + 8 * u;
                        pc[u] = jj < HALF ? tile_col + a * HALF + jj : -1;
                    }
                    store_warp_rows_pieces(my_stage, pk, lane, args.out, args.n_out, row_base, row_end, pc,
                                           args.n_out);
                }
            } else {
                // accumulator column c = h*HALF + cc -> output column tile_col + h*NH + a*HALF + cc
#pragma unroll 1
                for (int c0 = 0; c0 < NH; c0 += 32) {
                    uint32_t v[32], pk[16];
                    tmem_load_32cols(t_acc + c0, v);
#pragma unroll
                    for (int i = 0; i < 16; ++i)
                        pk[i] = pack_bf16x2(__uint_as_float(v[2 * i]), __uint_as_float(v[2 * i + 1]));
                    int pc[4];
#pragma unroll
                    for (int u = 0; u < 4; ++u) {
                        const int c = c0 + 8 * u;
                        const int h = c >= HALF ? 1 : 0;
                        pc[u] = c < NH ? tile_col + h * NH + a * HALF + (c - h * HALF) : -1;
                    }
                    store_warp_rows_pieces(my_stage, pk, lane, args.out, args.n_out, row_base, row_end, pc,
                                           args.n_out);
                }
            }
            tc_fence_before_sync();
            __syncwarp();
            if (lane == 0) mbar_arrive_cluster(tempty_leader);
            tphase ^= 1u;
        }
    }

    tc_fence_before_sync();
    __syncthreads();
    if (warp == 1 && leader) {
        if (lane == 0) mbar_wait_drain(final_bar, 0);
        __syncwarp();
    }
    cluster_sync();
    tc_fence_after_sync();
    if (warp == 1) tmem_dealloc_pair(tmem_base, S::TMEM_COLS);
}

}  // namespace moe
