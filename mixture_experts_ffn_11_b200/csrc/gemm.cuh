// Persistent grouped GEMM on the 5th-generation tensor cores (tcgen05, accumulators in TMEM, operands
// staged by TMA), one group per expert: the grouped_mm strategy of the blog post "Mixture of Experts
// (MoEs) in Transformers", section "Expert Backend" (sort by expert, group, one grouped GEMM).
//
//   out[r][n] = epilogue( sum_k A[r][k] * B[g][n][k] )   for r in [off[g], off[g+1])
//
// Two instantiations:
//   gate|up (GATEUP = true): B is the packed gate_up_proj slab of expert g ([2f][d], gate rows then up
//     rows, section "Dynamic Weight Loading with WeightConverter"). A tile computes BN/2 gate columns
//     and the matching BN/2 up columns in one BN-wide accumulator; the epilogue writes
//     h = silu(gate) * up in bf16, so the 2f-wide intermediate never reaches memory.
//   down (GATEUP = false): B is the down_proj slab [d][f]; the epilogue writes bf16.
//
// CTA organisation (192 threads, one CTA per SM, persistent over tiles):
//   warp 0     TMA producer: A box [128 x 64] and B box(es) [BN x 64] per K step into a STAGES-deep
//              ring of 128-byte-swizzled shared-memory buffers, completion on full[stage]
//   warp 1     MMA issuer: allocates TMEM (2 accumulators of BN fp32 columns), issues
//              tcgen05.mma M=128 N=BN K=16 x4 per stage, frees the stage with tcgen05.commit ->
//              empty[stage], and signals a finished tile with tcgen05.commit -> tmem_full[acc]
//   warps 2-5  epilogue: tcgen05.ld of their 32-lane quarter of the accumulator, math, bf16 stores
//              masked to the group's rows; then release the accumulator (tmem_empty[acc]) so the
//              next-but-one tile can reuse it while this tile's epilogue overlapped the next mainloop
// Tiles are numbered group-major, then N-block, then M-block (M fastest), so CTAs running at the same
// time share the expert's weight slab in L2. Group row counts are read on the device from the offsets,
// so ragged and empty groups need no host synchronisation. Tail tiles may read rows of the next group
// or past the end (TMA fills zeros there); those rows are never stored.
//
// Every wait is bounded (see mbar_wait_bounded): on a timeout the CTA raises an error bit, all roles
// leave their loops, in-flight copies and MMAs are waited for (bounded), and TMEM is released.
#pragma once
#include "common.cuh"

namespace moe {

constexpr int GG_BM = 128;
constexpr int GG_BK = 64;  // 64 bf16 = 128 bytes = one swizzle row
constexpr int GG_THREADS = 192;
constexpr int GG_MAX_GROUPS = 1024;

struct GemmArgs {
    const int32_t* group_offsets;  // [G+1], device
    int G;
    int M;        // rows allocated in A and out
    int K;        // reduction length
    int n_out;    // output columns
    int f;        // gate|up: first up row inside an expert's [2f][d] slab
    int n_tiles;  // N-blocks per group
    __nv_bfloat16* out;  // [M][n_out]
    __nv_bfloat16* out2 = nullptr;     // gate|up saving its pre-activations: [M][2f]
    const int32_t* row_src = nullptr;  // gathering kernels: A row r is row row_src[r] of a [src_rows][K] tensor
    int src_rows = 0;
};

// silu(g) * u, silu(g) = g / (1 + e^-g), with the fast exponential and the fast divide: a few fp32 ulp, far
// below the bf16 rounding of h, and fewer instructions on the epilogue warps, which share their SM sub-partitions
// with the TMA and MMA issuing warps (measured: gate|up -2..4%). For g < -88, e^-g is past the divide's range and
// silu(g) evaluates to 0 (its true magnitude is below 1e-36).
__device__ __forceinline__ float swiglu(float g, float u) { return __fdividef(g, 1.f + __expf(-g)) * u; }

// Epilogue store of one warp's 32 rows x 32 bf16 columns (thread = row, 16 packed words per thread).
// A thread's own row is 64 contiguous bytes, but a warp-wide store of one 16-byte piece per row touches
// 32 rows and only half of each 32-byte sector; L2 then has to fetch the rest of every sector from DRAM.
// So the rows go through a 2 KB per-warp staging buffer (16-byte units XOR-swizzled by row, which keeps
// both the write and the read at the minimum of four shared-memory wavefronts) and leave it as
// 8 rows x 64 contiguous bytes per instruction: whole sectors, masked per row and column.
// The same 32 x 32 block sent by one TMA store when it lies whole inside the rows and columns this tile owns
// (no masking needed). The staging layout above is the TMA engine's 64-byte swizzle (the 16-byte unit of a
// 64-byte row is XORed with row / 2), so the tensor map (box 32 x 32, SWIZZLE_64B) reads it as written; the
// buffer must be 512-byte aligned. Lane 0 issues the store and commits it as a bulk group: the caller waits
// (bulk_wait_group_read) before writing this buffer again.
__device__ __forceinline__ void store_warp_block_tma(uint8_t* stage, const uint32_t (&pk)[16], int lane,
                                                     const CUtensorMap* tm_out, int row_base, int col0) {
#pragma unroll
    for (int v = 0; v < 4; ++v)
        *reinterpret_cast<uint4*>(stage + lane * 64 + ((v ^ ((lane >> 1) & 3)) << 4)) =
            make_uint4(pk[4 * v], pk[4 * v + 1], pk[4 * v + 2], pk[4 * v + 3]);
    fence_proxy_async_smem();  // generic writes -> the TMA engine
    __syncwarp();
    if (lane == 0) {
        tma_store_2d(tm_out, stage, col0, row_base);
        bulk_commit_group();
    }
}

__device__ __forceinline__ void store_warp_rows_32cols(uint8_t* stage, const uint32_t (&pk)[16], int lane,
                                                       __nv_bfloat16* out, int ld_out, int row_base, int row_end,
                                                       int col0, int n_out, int cols_in_tile) {
#pragma unroll
    for (int v = 0; v < 4; ++v)
        *reinterpret_cast<uint4*>(stage + lane * 64 + ((v ^ ((lane >> 1) & 3)) << 4)) =
            make_uint4(pk[4 * v], pk[4 * v + 1], pk[4 * v + 2], pk[4 * v + 3]);
    __syncwarp();
    const int u = lane & 3;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const int row = i * 8 + (lane >> 2);
        const uint4 val = *reinterpret_cast<const uint4*>(stage + row * 64 + ((u ^ ((row >> 1) & 3)) << 4));
        const int grow = row_base + row, col = col0 + u * 8;
        if (grow < row_end && u * 8 < cols_in_tile && col < n_out)
            *reinterpret_cast<uint4*>(out + (size_t)grow * ld_out + col) = val;
    }
    __syncwarp();
}

template <int BN, int STAGES, bool GATEUP>
struct GemmShape {
    static_assert(BN % 16 == 0 && BN >= 32 && BN <= 256, "UMMA N for M=128 is a multiple of 16 up to 256");
    static_assert(!GATEUP || (BN / 2) % 32 == 0, "gate|up halves must be whole 32-column TMEM loads");
    static constexpr int A_BYTES = GG_BM * GG_BK * 2;
    static constexpr int B_BYTES = BN * GG_BK * 2;
    static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
    static constexpr int OUT_COLS = GATEUP ? BN / 2 : BN;
    static constexpr int TMEM_COLS = 2 * BN <= 64 ? 64 : (2 * BN <= 128 ? 128 : (2 * BN <= 256 ? 256 : 512));
    static constexpr int BAR_BYTES = 256;
    static constexpr int TABLE_BYTES = (2 * (GG_MAX_GROUPS + 1) * 4 + 127) / 128 * 128;  // keeps what follows 128-B aligned
    static constexpr int EPI_BYTES = 4 * 2048;  // per-epilogue-warp store staging
    static_assert((STAGES * STAGE_BYTES + BAR_BYTES + TABLE_BYTES) % 128 == 0, "staging buffer alignment");
    static constexpr int SMEM_BYTES = 1024 + STAGES * STAGE_BYTES + BAR_BYTES + TABLE_BYTES + EPI_BYTES;
    static_assert((2 * STAGES + 6) * 8 + 8 <= BAR_BYTES, "barrier area");
    static_assert(SMEM_BYTES <= 232448, "shared memory");
};

template <int BN, int STAGES, bool GATEUP>
__global__ void __launch_bounds__(GG_THREADS, 1)
    grouped_gemm_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                        const GemmArgs args, int weights_streamed_once) {
    using S = GemmShape<BN, STAGES, GATEUP>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    uint8_t* stages = smem;
    uint64_t* full_bar = reinterpret_cast<uint64_t*>(smem + STAGES * S::STAGE_BYTES);
    uint64_t* empty_bar = full_bar + STAGES;
    uint64_t* tfull_bar = empty_bar + STAGES;
    uint64_t* tempty_bar = tfull_bar + 2;
    uint64_t* final_bar = tempty_bar + 2;
    uint64_t* never_bar = final_bar + 1;  // nothing arrives on it (test_stall)
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(never_bar + 1);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
    int32_t* s_off = reinterpret_cast<int32_t*>(smem + STAGES * S::STAGE_BYTES + S::BAR_BYTES);
    int32_t* s_tp = s_off + (GG_MAX_GROUPS + 1);
    uint8_t* epi_stage = smem + STAGES * S::STAGE_BYTES + S::BAR_BYTES + S::TABLE_BYTES;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int G = args.G;
    const int KB = (args.K + GG_BK - 1) / GG_BK;

    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(&full_bar[s], 1);
            mbar_init(&empty_bar[s], 1);
        }
        for (int a = 0; a < 2; ++a) {
            mbar_init(&tfull_bar[a], 1);
            mbar_init(&tempty_bar[a], 4);
        }
        mbar_init(final_bar, 1);
        mbar_init(never_bar, 1);
        *abort_flag = 0;
        fence_mbar_init();
        tma_prefetch_desc(&tmA);
        tma_prefetch_desc(&tmB);
    }
    if (warp == 1) {
        tmem_alloc(tmem_slot, S::TMEM_COLS);
        tmem_relinquish();
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
    if (warp == 0) {  // tile prefix over groups: tiles(g) = ceil(rows / 128) * n_tiles
        const int per = (G + 31) / 32;
        const int g0 = lane * per, g1 = min(g0 + per, G);
        int local = 0;
        for (int g = g0; g < g1; ++g) {
            const int rows = s_off[g + 1] - s_off[g];
            if (rows < 0) flag_error(MOE_DEVERR_GROUP_RANGE);
            local += (max(rows, 0) + GG_BM - 1) / GG_BM * args.n_tiles;
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
            run += (max(s_off[g + 1] - s_off[g], 0) + GG_BM - 1) / GG_BM * args.n_tiles;
        }
        if (lane == 31) s_tp[G] = incl;
    }
    tc_fence_before_sync();
    __syncthreads();
    tc_fence_after_sync();
    const uint32_t tmem_base = *tmem_slot;
    const int total = s_tp[G];

    // tile -> (group, N-block, M-block); the last group whose first tile is <= tile is never empty
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
        const int mt = (max(s_off[g + 1] - s_off[g], 0) + GG_BM - 1) / GG_BM;
        const int local = tile - s_tp[g];
        nb = local / mt;
        mb = local - nb * mt;
    };

    if (warp == 0) {
        // ---------------- TMA producer ----------------
        // activations are re-read by every N-block; weights are re-read by the M-blocks of their group unless
        // each group fits one M-block, in which case they are streamed once and should not displace anything
        const uint64_t pol_a = l2_policy_evict_last();
        const uint64_t pol_b = weights_streamed_once ? l2_policy_evict_first() : l2_policy_evict_normal();
        int stage = 0;
        uint32_t phase = 0;
        long issued = 0;
        bool ok = true;
        for (int tile = blockIdx.x; tile < total && ok; tile += gridDim.x) {
            int g, nb, mb;
            locate(tile, g, nb, mb);
            const int row0 = s_off[g] + mb * GG_BM;
            for (int kb = 0; kb < KB; ++kb) {
                if (lane == 0) ok = mbar_wait_bounded(&empty_bar[stage], phase ^ 1u, abort_flag);
                ok = __shfl_sync(0xffffffffu, ok, 0);
                if (!ok) break;
                if (lane == 0) {
                    uint8_t* sa = stages + stage * S::STAGE_BYTES;
                    uint8_t* sb = sa + S::A_BYTES;
                    mbar_arrive_expect_tx(&full_bar[stage], S::STAGE_BYTES);
                    tma_load_2d(sa, &tmA, &full_bar[stage], kb * GG_BK, row0, pol_a);
                    if constexpr (GATEUP) {
                        tma_load_3d(sb, &tmB, &full_bar[stage], kb * GG_BK, nb * (BN / 2), g, pol_b);
                        tma_load_3d(sb + (BN / 2) * GG_BK * 2, &tmB, &full_bar[stage], kb * GG_BK,
                                    args.f + nb * (BN / 2), g, pol_b);
                    } else {
                        tma_load_3d(sb, &tmB, &full_bar[stage], kb * GG_BK, nb * BN, g, pol_b);
                    }
                }
                ++issued;
                if (++stage == STAGES) {
                    stage = 0;
                    phase ^= 1u;
                }
            }
        }
        // copies still in flight complete by themselves; wait for them (bounded) before leaving
        if (lane == 0) {
            for (long n = issued > STAGES ? issued - STAGES : 0; n < issued; ++n)
                mbar_wait_drain(&full_bar[n % STAGES], (uint32_t)((n / STAGES) & 1));
        }
        __syncwarp();
    } else if (warp == 1) {
        // ---------------- MMA issuer ----------------
        constexpr uint32_t IDESC = idesc_bf16_f32(GG_BM, BN);
        int stage = 0, acc = 0;
        uint32_t phase = 0, acc_phase = 0;
        bool ok = true;
        if (lane == 0) ok = test_stall(never_bar, abort_flag);
        ok = __shfl_sync(0xffffffffu, ok, 0);
        for (int tile = blockIdx.x; tile < total && ok; tile += gridDim.x) {
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
                    const uint32_t sa = smem_u32(stages + stage * S::STAGE_BYTES);
                    const uint64_t adesc = smem_desc_sw128(sa);
                    const uint64_t bdesc = smem_desc_sw128(sa + S::A_BYTES);
#pragma unroll
                    for (int k = 0; k < GG_BK / 16; ++k)  // +32 bytes along K per step
                        umma_bf16_ss(d_tmem, adesc + 2 * k, bdesc + 2 * k, IDESC, (kb | k) != 0 ? 1u : 0u);
                    umma_commit(&empty_bar[stage]);
                }
                __syncwarp();
                if (++stage == STAGES) {
                    stage = 0;
                    phase ^= 1u;
                }
            }
            if (!ok) break;
            if (lane == 0) umma_commit(&tfull_bar[acc]);
            __syncwarp();
            acc ^= 1;
            if (acc == 0) acc_phase ^= 1u;
        }
        if (lane == 0) umma_commit(final_bar);  // arrives once all MMAs issued above have finished
        __syncwarp();
    } else {
        // ---------------- epilogue (warps 2-5) ----------------
        const int q = warp & 3;  // this warp may access TMEM lanes 32q .. 32q+31
        int acc = 0;
        uint32_t acc_phase = 0;
        bool ok = true;
        for (int tile = blockIdx.x; tile < total; tile += gridDim.x) {
            int g, nb, mb;
            locate(tile, g, nb, mb);
            const int row_end = s_off[g + 1];
            const int row_base = s_off[g] + mb * GG_BM + q * 32;  // global row of this warp's lane 0
            if (lane == 0) ok = mbar_wait_bounded(&tfull_bar[acc], acc_phase, abort_flag);
            ok = __shfl_sync(0xffffffffu, ok, 0);
            if (!ok) break;
            tc_fence_after_sync();
            const uint32_t t_row = tmem_base + ((uint32_t)(q * 32) << 16) + (uint32_t)(acc * BN);
            const int col_base = nb * S::OUT_COLS;
            uint8_t* my_stage = epi_stage + (warp - 2) * 2048;
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
                store_warp_rows_32cols(my_stage, pk, lane, args.out, args.n_out, row_base, row_end, col0, args.n_out,
                                       S::OUT_COLS - c0);
            }
            tc_fence_before_sync();
            __syncwarp();
            if (lane == 0) mbar_arrive(&tempty_bar[acc]);
            acc ^= 1;
            if (acc == 0) acc_phase ^= 1u;
        }
    }

    tc_fence_before_sync();
    __syncthreads();
    tc_fence_after_sync();
    if (warp == 1) {
        if (lane == 0) mbar_wait_drain(final_bar, 0);
        __syncwarp();
        tmem_dealloc(tmem_base, S::TMEM_COLS);
    }
}

}  // namespace moe
