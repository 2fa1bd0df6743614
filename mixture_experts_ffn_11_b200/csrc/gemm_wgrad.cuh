// Weight gradients of the grouped projections: a GEMM grouped over the reduction axis.
//
//   out[g][p][q] = sum_{r in group g} a[r][p] * b[r][q]       (dW[g] = a_g^T b_g, fp32)
//
// The training path of the blog post "Mixture of Experts (MoEs) in Transformers" (section "Training MoEs with
// Transformers") runs through the same grouped expert backend; for an expert's weight gradient the reduction runs
// over the rows routed to it. The operands come transposed and per-group zero-padded (transpose_pad_kernel):
// aT [P][cap] and bT [Q][cap] with group g's rows at columns [pad_off[g], pad_off[g+1]), a multiple of 64 long,
// so every K block of a group is whole and the padding adds zeros. Each output tile is computed by one CTA pair
// over its group's whole K range (no split-K, no atomics: deterministic), M = 256 rows of aT per pair, N = 256 rows
// of bT, accumulators in TMEM, fp32 results sent by TMA stores of 32 x 32 blocks (128-byte swizzle). An empty group
// gets zeros. Roles as in the CTA-pair grouped GEMM (gemm_pair.cuh); no load uses multicast.
#pragma once
#include "common.cuh"
#include "gemm.cuh"

namespace moe {

constexpr int WG_THREADS = 192;
constexpr int WG_TILE = 256;

struct GemmWgradShape {
    static constexpr int STAGES = 5;
    static constexpr int A_BYTES = 128 * GG_BK * 2;
    static constexpr int B_BYTES = 128 * GG_BK * 2;
    static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
    static constexpr int TMEM_COLS = 512;  // two accumulators of 256 fp32 columns
    static constexpr int EPI_BYTES = 4 * 2 * 4096;  // per epilogue warp two 32 x 32 fp32 staging blocks
    static constexpr int BAR_BYTES = 256;
    static constexpr int TABLE_BYTES = ((GG_MAX_GROUPS + 1) * 4 + 127) / 128 * 128;
    static constexpr int SMEM_BYTES = 1024 + STAGES * STAGE_BYTES + EPI_BYTES + BAR_BYTES + TABLE_BYTES;
    static_assert(SMEM_BYTES <= 232448, "shared memory");
    static_assert((2 * STAGES + 6) * 8 + 8 <= BAR_BYTES, "barrier area");
};

struct WgradArgs {
    const int32_t* pad_off;  // [G+1], device
    int G, P, Q;
};

// tmA: aT [P][cap] bf16, box {64, 128}; tmB: bT [Q][cap] bf16, box {64, 128}; tmO: out [G][P][Q] fp32, box
// {32, 32, 1}, 128-byte swizzle.
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(WG_THREADS, 1)
    grouped_wgrad_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                         const __grid_constant__ CUtensorMap tmO, const WgradArgs args) {
    using S = GemmWgradShape;
    constexpr int STAGES = S::STAGES;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    uint8_t* stages = smem;
    uint8_t* epi = smem + STAGES * S::STAGE_BYTES;
    uint64_t* full_bar = reinterpret_cast<uint64_t*>(epi + S::EPI_BYTES);  // used in the leader
    uint64_t* empty_bar = full_bar + STAGES;
    uint64_t* tfull_bar = empty_bar + STAGES;  // [2]
    uint64_t* tempty_bar = tfull_bar + 2;      // [2], used in the leader
    uint64_t* final_bar = tempty_bar + 2;
    uint64_t* never_bar = final_bar + 1;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(never_bar + 1);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
    int32_t* s_pad = reinterpret_cast<int32_t*>(epi + S::EPI_BYTES + S::BAR_BYTES);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t rank = cluster_ctarank();
    const bool leader = rank == 0;
    const int cluster = blockIdx.x >> 1, n_clusters = gridDim.x >> 1;
    const int G = args.G;
    const int MB = (args.P + WG_TILE - 1) / WG_TILE, NB = (args.Q + WG_TILE - 1) / WG_TILE;
    const int total = G * MB * NB;

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
    grid_dep_wait();
    grid_dep_trigger();
    for (int g = threadIdx.x; g <= G; g += WG_THREADS) s_pad[g] = args.pad_off[g];
    tc_fence_before_sync();
    __syncthreads();
    cluster_sync();
    tc_fence_after_sync();
    const uint32_t tmem_base = *tmem_slot;

    // tile -> group, M block, N block; K blocks of the group (0 for an empty group)
    auto locate = [&](int tile, int& g, int& mb, int& nb, int& k0, int& kblocks) {
        g = tile / (MB * NB);
        const int rem = tile - g * (MB * NB);
        mb = rem / NB;
        nb = rem - mb * NB;
        k0 = s_pad[g];
        const int len = s_pad[g + 1] - k0;
        kblocks = len > 0 ? len / GG_BK : 0;
    };

    if (warp == 0) {
        // ---------------- TMA producer (both CTAs) ----------------
        const uint64_t pol = l2_policy_evict_normal();
        int stage = 0;
        uint32_t phase = 0;
        long issued = 0;
        bool ok = true;
        for (int tile = cluster; tile < total && ok; tile += n_clusters) {
            int g, mb, nb, k0, KB;
            locate(tile, g, mb, nb, k0, KB);
            const int arow = mb * WG_TILE + (int)rank * 128, brow = nb * WG_TILE + (int)rank * 128;
            for (int kb = 0; kb < KB; ++kb) {
                if (lane == 0) ok = mbar_wait_bounded(&empty_bar[stage], phase ^ 1u, abort_flag);
                ok = __shfl_sync(0xffffffffu, ok, 0);
                if (!ok) break;
                if (lane == 0) {
                    uint8_t* sa = stages + stage * S::STAGE_BYTES;
                    const uint32_t bar = mapa_shared(smem_u32(&full_bar[stage]), 0);
                    if (leader) mbar_arrive_expect_tx(&full_bar[stage], 2 * S::STAGE_BYTES);
                    tma_load_2d_pair(sa, &tmA, bar, k0 + kb * GG_BK, arow, pol);
                    tma_load_2d_pair(sa + S::A_BYTES, &tmB, bar, k0 + kb * GG_BK, brow, pol);
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
            constexpr uint32_t IDESC = idesc_bf16_f32(256, WG_TILE);
            int stage = 0, acc = 0;
            uint32_t phase = 0, acc_phase = 0;
            bool ok = true;
            if (lane == 0) ok = test_stall(never_bar, abort_flag);
            ok = __shfl_sync(0xffffffffu, ok, 0);
            for (int tile = cluster; tile < total && ok; tile += n_clusters) {
                int g, mb, nb, k0, KB;
                locate(tile, g, mb, nb, k0, KB);
                if (lane == 0) ok = mbar_wait_bounded(&tempty_bar[acc], acc_phase ^ 1u, abort_flag);
                ok = __shfl_sync(0xffffffffu, ok, 0);
                if (!ok) break;
                tc_fence_after_sync();
                const uint32_t d_tmem = tmem_base + (uint32_t)(acc * WG_TILE);
                for (int kb = 0; kb < KB; ++kb) {
                    if (lane == 0) ok = mbar_wait_bounded(&full_bar[stage], phase, abort_flag);
                    ok = __shfl_sync(0xffffffffu, ok, 0);
                    if (!ok) break;
                    tc_fence_after_sync();
                    if (lane == 0) {
                        const uint32_t sa = smem_u32(stages + stage * S::STAGE_BYTES);
                        const uint64_t adesc = smem_desc_sw128(sa);
                        const uint64_t bdesc = smem_desc_sw128(sa + S::A_BYTES);
#pragma unroll
                        for (int k = 0; k < GG_BK / 16; ++k)
                            umma_bf16_ss_pair(d_tmem, adesc + 2 * k, bdesc + 2 * k, IDESC, (kb | k) != 0 ? 1u : 0u);
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
        uint8_t* stage_base = epi + (warp - 2) * 8192;
        int acc = 0;
        uint32_t acc_phase = 0;
        uint32_t blocks = 0;
        bool ok = true;
        for (int tile = cluster; tile < total; tile += n_clusters) {
            int g, mb, nb, k0, KB;
            locate(tile, g, mb, nb, k0, KB);
            const int row0 = mb * WG_TILE + (int)rank * 128 + q * 32;  // output row of lane 0
            if (lane == 0) ok = mbar_wait_bounded(&tfull_bar[acc], acc_phase, abort_flag);
            ok = __shfl_sync(0xffffffffu, ok, 0);
            if (!ok) break;
            tc_fence_after_sync();
            const uint32_t t_row = tmem_base + ((uint32_t)(q * 32) << 16) + (uint32_t)(acc * WG_TILE);
#pragma unroll 1
            for (int c0 = 0; c0 < WG_TILE; c0 += 32) {
                const int col0 = nb * WG_TILE + c0;
                if (col0 >= args.Q || row0 >= args.P) break;  // warp-uniform: nothing of this block is in range
                uint32_t v[32];
                if (KB > 0) {
                    tmem_load_32cols(t_row + (uint32_t)c0, v);
                } else {
#pragma unroll
                    for (int i = 0; i < 32; ++i) v[i] = 0u;
                }
                uint8_t* st = stage_base + (int)(blocks & 1u) * 4096;
                ++blocks;
                if (lane == 0) bulk_wait_group_read<1>();
                __syncwarp();
#pragma unroll
                for (int u = 0; u < 8; ++u)  // row = lane, 16-byte unit u at u ^ (row % 8) (128-byte swizzle)
                    *reinterpret_cast<uint4*>(st + lane * 128 + ((u ^ (lane & 7)) << 4)) =
                        make_uint4(v[4 * u], v[4 * u + 1], v[4 * u + 2], v[4 * u + 3]);
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) {  // the tensor map clips the block at the edges of out
                    tma_store_3d(&tmO, st, col0, row0, g);
                    bulk_commit_group();
                }
            }
            tc_fence_before_sync();
            __syncwarp();
            if (lane == 0) mbar_arrive_cluster(acc ? tempty_leader1 : tempty_leader0);
            acc ^= 1;
            if (acc == 0) acc_phase ^= 1u;
        }
        if (lane == 0) bulk_wait_all();
        __syncwarp();
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
