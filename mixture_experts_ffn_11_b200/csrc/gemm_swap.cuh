// Grouped GEMM on CTA pairs with the expert weights as the MMA's M dimension and the group's token rows as its
// N dimension ("swap AB"): the same results as the pair kernel (gemm_pair.cuh), with far less padding.
//
// Why: an expert's rows come in ragged counts (gpt-oss-shaped prefill: 447-569 rows per expert). With token rows
// as M, a CTA pair computes 256 of them at a time, so a group's last tile is on average half padding (22% of the
// tensor work on that workload). With token rows as N, a tile takes any multiple of 16 rows up to 256: a group of
// n rows is cut into full tiles of 256 rows and one last tile of the remaining rows rounded up to 16, so the
// padding falls to a few rows per group. The weight rows (M = 256 per pair, 128 per CTA) are the expert's output
// columns, whose count is fixed by the model and mostly a multiple of 128.
//
//   out[r][c] = epilogue( sum_k A[r][k] * W[g][c][k] )   for r in [off[g], off[g+1])
//
// computed as D[c][r] = W[g][c][:] . A[r][:] with D in tensor memory: TMEM lane = output column, TMEM column =
// token row. Per pair tile (one group g, one block of weight rows, one block of at most 256 token rows):
//   down   (GATEUP = false): CTA `rank` holds weight rows (= output columns) c0 + 128*rank + [0, 128).
//   gate|up (GATEUP = true): the tile covers 128 columns j0 + [0, 128) of h; CTA `rank` holds the 64 gate rows
//          j0 + 64*rank + [0, 64) in TMEM lanes 0-63 and the matching 64 up rows (f + j) in lanes 64-127 (one
//          TMA box of the weights viewed as [G][2][f][K]), so one accumulator holds both factors of
//          silu(gate) * up for its columns. A warp may read TMEM only in its own lane quarter, so the warps of
//          lanes 0-63 (warps 4 and 5, which share their SM sub-partitions with the TMA and MMA issuing warps)
//          pass their gate values through shared memory (bounded mbarrier hand-off) to the warps of lanes
//          64-127 (warps 2 and 3), which compute and store h.
// The token rows of the tile are split between the pair as the MMA's B operand: the leader loads the first N/2,
// the peer the next N/2 (one TMA box of 128, 64, 32, 16 or 8 rows, the smallest that holds N/2), and both
// accumulators hold all N columns.
//
// Roles (192 threads per CTA, both CTAs):
//   warp 0     TMA producer: per 64-wide K block, this CTA's 128 weight rows (one box) and its token rows (one
//              box), SUB K blocks per ring stage; completion counted on the leader's full[stage].
//   warp 1     TMEM allocation (512 columns: two accumulators of up to 256 token columns) and, in the leader,
//              the MMA issuer: tcgen05.mma.cta_group::2 M=256 N=tile rows (runtime instruction descriptor).
//   warps 2-5  epilogue: tcgen05.ld of the lane quarter, transpose through shared memory (thread = output
//              column, 32 token rows per block) into the output's row-major layout, TMA store of whole 32 x 32
//              blocks, masked stores at group and column edges.
// Tiles are numbered group-major, then weight block, then token block, so the token blocks of one weight block
// run side by side (sharing it in L2) and all tiles of a group share its token rows. No load uses multicast.
#pragma once
#include "common.cuh"
#include "gemm.cuh"
#include "gemm_pair.cuh"

namespace moe {

constexpr int GS_THREADS = 192;
constexpr int GS_MAX_N = 256;  // token rows per tile (UMMA N for M = 256, a multiple of 16)

// Stage layout: the SUB K blocks of this CTA's weight rows, then the SUB K blocks of its token rows:
//   [W k0 | W k1 | ... | X k0 | X k1 | ...], W blocks 16 KB apart, X blocks (rows per CTA) * 128 bytes apart.
// BIGBOX: the operands are read through tensor maps that view [rows][K] as [K/64][rows][64] (K a multiple of 64),
// so one TMA box brings the SUB K blocks of a stage at once (a 32 KB box moves faster than two 16 KB ones).
template <bool GATEUP, int SUB, int STAGES, bool SAVE = false>
struct GemmSwapShape {
    static constexpr int W_BYTES = 128 * GG_BK * 2;  // this CTA's 128 weight rows of one K block
    static constexpr int X_BYTES = 128 * GG_BK * 2;  // room for this CTA's share of the token rows (<= 128)
    static constexpr int SUB_BYTES = W_BYTES + X_BYTES;
    static constexpr int STAGE_BYTES = SUB * SUB_BYTES;
    static constexpr int X_OFF = SUB * W_BYTES;  // token blocks start here in a stage
    static constexpr int TILE_W = GATEUP ? 128 : 256;  // output columns per pair tile
    static constexpr int TMEM_COLS = 512;
    static constexpr int BAR_BYTES = 256;
    static constexpr int TABLE_BYTES = (2 * (GG_MAX_GROUPS + 1) * 4 + 127) / 128 * 128;
    // 4 x two 2 KB staging blocks (down); gate|up: two storing warps' staging blocks + two 4 KB hand-off buffers;
    // SAVE: one more 2 KB block per epilogue warp for the pre-activations
    static constexpr int EPI_BYTES = 4 * 2 * 2048 + (SAVE ? 4 * 2048 : 0);
    static constexpr int SMEM_BYTES = 1024 + STAGES * STAGE_BYTES + EPI_BYTES + BAR_BYTES + TABLE_BYTES;
    static_assert(SUB_BYTES % 1024 == 0, "sub-block bases stay 1024-byte aligned");
    static_assert(SMEM_BYTES <= 232448, "shared memory");
    static_assert((2 * STAGES + 4 + 1 + 4 + 1) * 8 + 8 <= BAR_BYTES, "barrier area");
};

// Write one warp's 32 output columns (thread = column) x 32 token rows (v[t], fp32) into a 2 KB staging block in
// the output's row-major order: row t holds the 32 columns as 64 bytes, its 16-byte units XOR-swizzled by
// (t / 2) % 4 (the TMA engine's 64-byte swizzle, as store_warp_block_tma expects). For a fixed row the warp
// writes 64 contiguous bytes: one shared-memory wavefront per row.
__device__ __forceinline__ void stage_transposed(uint8_t* stage, const float (&v)[32], int lane) {
    const int unit = lane >> 3, sub = (lane & 7) * 2;
#pragma unroll
    for (int t = 0; t < 32; t += 2) {
        const uint32_t pk = pack_bf16x2(v[t], v[t + 1]);
        *reinterpret_cast<uint16_t*>(stage + t * 64 + ((unit ^ ((t >> 1) & 3)) << 4) + sub) = (uint16_t)(pk & 0xffffu);
        *reinterpret_cast<uint16_t*>(stage + (t + 1) * 64 + ((unit ^ (((t + 1) >> 1) & 3)) << 4) + sub) =
            (uint16_t)(pk >> 16);
    }
}

// Send a staged block (rows row0 .. row0+31, columns col0 .. col0+31 of out [M][ld]): one TMA store when the
// whole block belongs to this tile, else 16-byte stores masked to rows < row_end and columns < col_end.
__device__ __forceinline__ void flush_staged_block(uint8_t* stage, int lane, const CUtensorMap* tm_out,
                                                   __nv_bfloat16* out, int ld, int row0, int row_end, int col0,
                                                   int col_end) {
    if (row0 + 32 <= row_end && col0 + 32 <= col_end) {
        fence_proxy_async_smem();  // generic writes -> the TMA engine
        __syncwarp();
        if (lane == 0) {
            tma_store_2d(tm_out, stage, col0, row0);
            bulk_commit_group();
        }
        return;
    }
    __syncwarp();
    const int u = lane & 3;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const int row = i * 8 + (lane >> 2);
        const uint4 val = *reinterpret_cast<const uint4*>(stage + row * 64 + ((u ^ ((row >> 1) & 3)) << 4));
        const int col = col0 + u * 8;
        if (row0 + row < row_end && col < col_end)
            *reinterpret_cast<uint4*>(out + (size_t)(row0 + row) * ld + col) = val;
    }
    if (lane == 0) bulk_commit_group();  // an empty group keeps one group per staged block
    __syncwarp();
}

// The weighted combine fused into the down GEMM (COMBINE): "apply the routing weights and then collect and
// reorder the results" (blog post "Mixture of Experts (MoEs) in Transformers", section "Expert Backend"),
//   y[t][c] = sum_{j<k} w[t][j] * y_perm[inv_perm[t*k+j]][c] (+ shared[t][c]),  fp32 in slot order, bf16 out,
// the arithmetic of the stand-alone combine kernel. The k rows of a token come from k groups, computed by
// different tiles in any order, so no tile can sum them as it goes without fixing an order by waiting. Instead
// each epilogue warp, once its y_perm rows of a tile are stored, counts one arrival per row on a counter of
// (token, 32-column block); the warp whose arrival is the k-th reads the k rows back (from L2, just written)
// and sums them in slot order. The sum is the same whoever finishes last: deterministic, no waiting.
struct CombineArgs {
    const int32_t* perm_src = nullptr;      // [M] grouped row -> token
    const int32_t* inv_perm = nullptr;      // [T*k] assignment -> grouped row
    const float* topk_w = nullptr;          // [T*k]
    const __nv_bfloat16* shared = nullptr;  // [T][n_out] or null
    __nv_bfloat16* y = nullptr;             // [T][n_out]
    int* counters = nullptr;                // [T][ceil(n_out / 32)], zero when the kernel starts
    int T = 0, k = 0;
};

// Sum one token's k slot rows over the 32 columns [c0, c0 + 32) (those below n_out) into y[t].
__device__ __noinline__ void combine_token_columns(const CombineArgs& ca, const __nv_bfloat16* y_perm, int M,
                                                   int n_out, int t, int c0) {
    const int nunit = min(4, (n_out - c0) >> 3);  // 16-byte units (8 columns) inside the output
    float acc[32];
#pragma unroll
    for (int i = 0; i < 32; ++i) acc[i] = 0.f;
#pragma unroll 4
    for (int j = 0; j < ca.k; ++j) {
        const int row = __ldg(ca.inv_perm + (size_t)t * ca.k + j);
        const float w = __ldg(ca.topk_w + (size_t)t * ca.k + j);
        if (row < 0 || row >= M) {
            flag_error(MOE_DEVERR_ROW_RANGE);
            continue;
        }
        // written by other CTAs in this kernel: read through L2 (ld.global.cg), after the acquire fence
        const uint4* src = reinterpret_cast<const uint4*>(y_perm + (size_t)row * n_out + c0);
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            if (u < nunit) {
                const uint4 q = __ldcg(src + u);
                const uint32_t uq[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const float2 f = unpack_bf16x2(uq[i]);
                    acc[8 * u + 2 * i] = fmaf(w, f.x, acc[8 * u + 2 * i]);
                    acc[8 * u + 2 * i + 1] = fmaf(w, f.y, acc[8 * u + 2 * i + 1]);
                }
            }
        }
    }
#pragma unroll
    for (int u = 0; u < 4; ++u) {
        if (u >= nunit) continue;
        if (ca.shared) {
            const uint4 q = __ldg(reinterpret_cast<const uint4*>(ca.shared + (size_t)t * n_out + c0) + u);
            const uint32_t uq[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const float2 f = unpack_bf16x2(uq[i]);
                acc[8 * u + 2 * i] += f.x;
                acc[8 * u + 2 * i + 1] += f.y;
            }
        }
        uint4 o;
        o.x = pack_bf16x2(acc[8 * u + 0], acc[8 * u + 1]);
        o.y = pack_bf16x2(acc[8 * u + 2], acc[8 * u + 3]);
        o.z = pack_bf16x2(acc[8 * u + 4], acc[8 * u + 5]);
        o.w = pack_bf16x2(acc[8 * u + 6], acc[8 * u + 7]);
        reinterpret_cast<uint4*>(ca.y + (size_t)t * n_out + c0)[u] = o;
    }
}

// After a warp has stored its 32 columns [c0, c0 + 32) of the tile's rows r0 .. r0 + rows - 1 of y_perm: publish
// them, count one arrival per row, and finish the tokens whose last slot this was.
__device__ __forceinline__ void combine_after_tile(const CombineArgs& ca, const __nv_bfloat16* y_perm, int M,
                                                   int n_out, int r0, int rows, int c0, int lane) {
    if (lane == 0) {
        bulk_wait_all();             // this warp's TMA stores of the tile have landed
        fence_proxy_async_global();  // ... and are ordered before the generic release below
    }
    __syncwarp();
    __threadfence();  // release: the rows (and the masked edge stores) before the arrivals
    const int ncb = (n_out + 31) >> 5;
    const int cb = c0 >> 5;
    int tok[GS_MAX_N / 32], old[GS_MAX_N / 32];
#pragma unroll
    for (int i = 0; i < GS_MAX_N / 32; ++i) {
        const int rr = lane + 32 * i;
        int t = -1;
        if (rr < rows) {
            t = __ldg(ca.perm_src + r0 + rr);
            if (t < 0 || t >= ca.T) {
                flag_error(MOE_DEVERR_ROW_RANGE);
                t = -1;
            }
        }
        tok[i] = t;
    }
#pragma unroll
    for (int i = 0; i < GS_MAX_N / 32; ++i)
        old[i] = tok[i] >= 0 ? atomicAdd(ca.counters + (size_t)tok[i] * ncb + cb, 1) : -1;
    __threadfence();  // acquire: the other slots' rows, published before their arrivals
#pragma unroll 1
    for (int i = 0; i < GS_MAX_N / 32; ++i)
        if (tok[i] >= 0 && old[i] == ca.k - 1) combine_token_columns(ca, y_perm, M, n_out, tok[i], c0);
}

// tmX[i]: the token rows [M][K] with boxes of 128 >> i rows (i = 0..4).
struct SwapMaps {
    CUtensorMap x[5];
};

// Map index of the smallest token box holding `half` rows (half a multiple of 8, 8..128).
__device__ __forceinline__ int swap_box_index(int half) {
    return half > 64 ? 0 : (half > 32 ? 1 : (half > 16 ? 2 : (half > 8 ? 3 : 4)));
}

// tmW: the weights, K-major, 128-byte swizzle: gate|up as [G][2][f][K] with box {64, 64, 2, 1} (64 gate rows
// and the matching 64 up rows), down as [G][d][K] with box {64, 128, 1}; with BIGBOX the same views with a K-block
// dimension {64, rows.., K/64} boxing SUB K blocks. tmX: the token rows, [M][K] (or [K/64][M][64] with BIGBOX).
// tmO: the output [M][n_out], 32 x 32 boxes, 64-byte swizzle.
// RAW (gate|up only): no SwiGLU; every warp stores its own lanes, gate rows to columns [0, f) and up rows to
// columns [f, 2f) of an [M][2f] output (the pre-activations a backward pass needs).
// GATHER: token row r of the tile is row args.row_src[r] of x [src_rows][K] (the dispatch of the blog post's
// expert backend folded into the operand load): tmX.x[0] views x with a one-row box, and each producer lane brings
// four of the CTA's rows per K block with one TMA gather4 into the places a tile box would fill, so the MMA and
// the epilogue are unchanged and no permuted copy of x is written.
// COMBINE (down only): after each tile, the weighted combine of the tokens completed by it (CombineArgs).
// SAVE (gate|up with SwiGLU): h as usual, and the pre-activations g | u into args.out2 [M][2f] (gate in columns
// [0, f), up in [f, 2f); tmG its map), the values the RAW mode stores: the gate warps store theirs after handing
// them off, the up warps theirs before computing h. A training forward keeps them for the backward pass.
template <bool GATEUP, int SUB, int STAGES, bool BIGBOX, bool RAW = false, bool GATHER = false, bool COMBINE = false,
          bool SAVE = false>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(GS_THREADS, 1)
    grouped_gemm_swap_kernel(const __grid_constant__ CUtensorMap tmW, const __grid_constant__ SwapMaps tmX,
                             const __grid_constant__ CUtensorMap tmO, const __grid_constant__ CUtensorMap tmG,
                             const GemmArgs args, int weights_streamed_once, const __grid_constant__ CombineArgs cargs) {
    static_assert(!COMBINE || !GATEUP, "the combine follows the down projection");
    static_assert(!SAVE || (GATEUP && !RAW), "saved pre-activations come with the SwiGLU epilogue");
    using S = GemmSwapShape<GATEUP, SUB, STAGES, SAVE>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    uint8_t* stages = smem;
    uint8_t* epi = smem + STAGES * S::STAGE_BYTES;  // 16 KB
    uint64_t* full_bar = reinterpret_cast<uint64_t*>(epi + S::EPI_BYTES);  // used in the leader
    uint64_t* empty_bar = full_bar + STAGES;
    uint64_t* tfull_bar = empty_bar + STAGES;  // [2]
    uint64_t* tempty_bar = tfull_bar + 2;      // [2], used in the leader
    uint64_t* final_bar = tempty_bar + 2;
    uint64_t* xfull_bar = final_bar + 1;   // [2] gate|up: gate values of a block are in xbuf[p]
    uint64_t* xempty_bar = xfull_bar + 2;  // [2] gate|up: xbuf[p] has been read
    uint64_t* never_bar = xempty_bar + 2;  // nothing arrives on it (test_stall)
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(never_bar + 1);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
    int32_t* s_off = reinterpret_cast<int32_t*>(epi + S::EPI_BYTES + S::BAR_BYTES);
    int32_t* s_tp = s_off + (GG_MAX_GROUPS + 1);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t rank = cluster_ctarank();
    const bool leader = rank == 0;
    const int cluster = blockIdx.x >> 1, n_clusters = gridDim.x >> 1;
    const int G = args.G;
    const int KBS = (args.K + GG_BK - 1) / GG_BK;  // 64-wide K blocks
    const int KB = (KBS + SUB - 1) / SUB;          // ring stages per tile
    const int wblocks = args.n_tiles;              // weight blocks (TILE_W output columns each)

    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(&full_bar[s], 1);
            mbar_init(&empty_bar[s], 1);
        }
        for (int a = 0; a < 2; ++a) {
            mbar_init(&tfull_bar[a], 1);
            mbar_init(&tempty_bar[a], 8);
            mbar_init(&xfull_bar[a], 32);
            mbar_init(&xempty_bar[a], 32);
        }
        mbar_init(final_bar, 1);
        mbar_init(never_bar, 1);
        *abort_flag = 0;
        fence_mbar_init();
        tma_prefetch_desc(&tmW);
        tma_prefetch_desc(&tmO);
#pragma unroll
        for (int i = 0; i < 5; ++i) tma_prefetch_desc(&tmX.x[i]);
    }
    if (warp == 1) {
        tmem_alloc_pair(tmem_slot, S::TMEM_COLS);
        tmem_relinquish_pair();
    }
    grid_dep_wait();  // inputs below come from earlier kernels in the stream
    grid_dep_trigger();
    for (int g = threadIdx.x; g <= G; g += GS_THREADS) {
        int v = args.group_offsets[g];
        if (v < 0 || v > args.M) {
            flag_error(MOE_DEVERR_GROUP_RANGE);
            v = min(max(v, 0), args.M);
        }
        s_off[g] = v;
    }
    __syncthreads();
    if (warp == 0) {  // tile prefix over groups: tiles(g) = ceil(rows / 256) * wblocks
        const int per = (G + 31) / 32;
        const int g0 = lane * per, g1 = min(g0 + per, G);
        int local = 0;
        for (int g = g0; g < g1; ++g) {
            const int n = s_off[g + 1] - s_off[g];
            if (n < 0) flag_error(MOE_DEVERR_GROUP_RANGE);
            local += (max(n, 0) + GS_MAX_N - 1) / GS_MAX_N * wblocks;
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
            run += (max(s_off[g + 1] - s_off[g], 0) + GS_MAX_N - 1) / GS_MAX_N * wblocks;
        }
        if (lane == 31) s_tp[G] = incl;
    }
    tc_fence_before_sync();
    __syncthreads();
    cluster_sync();  // both CTAs' barriers are initialised before any cross-CTA arrive or TMA signal
    tc_fence_after_sync();
    const uint32_t tmem_base = *tmem_slot;
    const int total = s_tp[G];

    // tile -> group g, weight block wb, first token row r0 (absolute), rows in the tile (<= 256)
    auto locate = [&](int tile, int& g, int& wb, int& r0, int& rows) {
        int lo = 0, hi = G - 1;
        while (lo < hi) {
            const int mid = (lo + hi + 1) >> 1;
            if (s_tp[mid] <= tile)
                lo = mid;
            else
                hi = mid - 1;
        }
        g = lo;
        const int n = s_off[g + 1] - s_off[g];
        const int tt = (n + GS_MAX_N - 1) / GS_MAX_N;
        const int local = tile - s_tp[g];
        wb = local / tt;
        const int ti = local - wb * tt;
        r0 = s_off[g] + ti * GS_MAX_N;
        rows = min(GS_MAX_N, n - ti * GS_MAX_N);
    };

    if (warp == 0) {
        // ---------------- TMA producer (both CTAs) ----------------
        const uint64_t pol_x = l2_policy_evict_last();
        const uint64_t pol_w = weights_streamed_once ? l2_policy_evict_first() : l2_policy_evict_normal();
        int stage = 0;
        uint32_t phase = 0;
        long issued = 0;
        bool ok = true;
        for (int tile = cluster; tile < total && ok; tile += n_clusters) {
            int g, wb, r0, rows;
            locate(tile, g, wb, r0, rows);
            const int half = ((rows + 15) / 16) * 8;  // token rows per CTA (N / 2)
            const int bi = swap_box_index(half);
            const int xrow0 = r0 + (int)rank * half;
            const int wrow = GATEUP ? wb * 128 + 64 * (int)rank : wb * 256 + 128 * (int)rank;
            const uint32_t sub_tx = (uint32_t)(S::W_BYTES + (128 >> bi) * GG_BK * 2);
            // GATHER: this lane's four token rows (4 * lane .. 4 * lane + 3 of the CTA's share) as rows of x
            int src0 = 0, src1 = 0, src2 = 0, src3 = 0;
            if constexpr (GATHER) {
                int v[4] = {0, 0, 0, 0};
                if (4 * lane < half) {
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        const int r = xrow0 + 4 * lane + i;  // rows past the tile (padding) are never stored
                        int src = r < args.M ? __ldg(args.row_src + r) : 0;
                        if (src < 0 || src >= args.src_rows) {
                            flag_error(MOE_DEVERR_ROW_RANGE);
                            src = 0;
                        }
                        v[i] = src;
                    }
                }
                src0 = v[0];
                src1 = v[1];
                src2 = v[2];
                src3 = v[3];
            }
            for (int kb = 0; kb < KB; ++kb) {
                if (lane == 0) ok = mbar_wait_bounded(&empty_bar[stage], phase ^ 1u, abort_flag);
                ok = __shfl_sync(0xffffffffu, ok, 0);
                if (!ok) break;
                if constexpr (GATHER) {
                    const int nsub = min(SUB, KBS - kb * SUB);
                    uint8_t* sa = stages + stage * S::STAGE_BYTES;
                    const uint32_t bar = mapa_shared(smem_u32(&full_bar[stage]), 0);
                    if (lane == 0) {
                        const uint32_t w_tx = (uint32_t)((BIGBOX ? SUB : nsub) * S::W_BYTES);
                        if (leader)
                            mbar_arrive_expect_tx(&full_bar[stage], 2u * (w_tx + (uint32_t)(nsub * half * GG_BK * 2)));
                        if constexpr (BIGBOX) {
                            if constexpr (GATEUP)
                                tma_load_5d_pair(sa, &tmW, bar, 0, wrow, 0, kb * SUB, g, pol_w);
                            else
                                tma_load_4d_pair(sa, &tmW, bar, 0, wrow, kb * SUB, g, pol_w);
                        } else {
                            for (int sb = 0; sb < nsub; ++sb) {
                                const int kc = (kb * SUB + sb) * GG_BK;
                                if constexpr (GATEUP)
                                    tma_load_4d_pair(sa + sb * S::W_BYTES, &tmW, bar, kc, wrow, 0, g, pol_w);
                                else
                                    tma_load_3d_pair(sa + sb * S::W_BYTES, &tmW, bar, kc, wrow, g, pol_w);
                            }
                        }
                    }
                    if (4 * lane < half) {
                        for (int sb = 0; sb < nsub; ++sb)
                            tma_gather4_pair(sa + S::X_OFF + sb * (128 >> bi) * GG_BK * 2 + lane * 4 * GG_BK * 2,
                                             &tmX.x[0], bar, (kb * SUB + sb) * GG_BK, src0, src1, src2, src3, pol_x);
                    }
                    __syncwarp();
                } else if (lane == 0) {
                    uint8_t* sa = stages + stage * S::STAGE_BYTES;
                    const uint32_t bar = mapa_shared(smem_u32(&full_bar[stage]), 0);
                    if constexpr (BIGBOX) {  // one box per operand: SUB K blocks (past the end: zeros)
                        if (leader) mbar_arrive_expect_tx(&full_bar[stage], 2u * (uint32_t)SUB * sub_tx);
                        if constexpr (GATEUP)
                            tma_load_5d_pair(sa, &tmW, bar, 0, wrow, 0, kb * SUB, g, pol_w);
                        else
                            tma_load_4d_pair(sa, &tmW, bar, 0, wrow, kb * SUB, g, pol_w);
                        tma_load_3d_pair(sa + S::X_OFF, &tmX.x[bi], bar, 0, xrow0, kb * SUB, pol_x);
                    } else {
                        const int nsub = min(SUB, KBS - kb * SUB);
                        if (leader) mbar_arrive_expect_tx(&full_bar[stage], 2u * (uint32_t)nsub * sub_tx);
                        for (int sb = 0; sb < nsub; ++sb) {  // K past the end arrives as zeros
                            const int kc = (kb * SUB + sb) * GG_BK;
                            uint8_t* sw = sa + sb * S::W_BYTES;
                            if constexpr (GATEUP)
                                tma_load_4d_pair(sw, &tmW, bar, kc, wrow, 0, g, pol_w);
                            else
                                tma_load_3d_pair(sw, &tmW, bar, kc, wrow, g, pol_w);
                            tma_load_2d_pair(sa + S::X_OFF + sb * (128 >> bi) * GG_BK * 2, &tmX.x[bi], bar, kc,
                                             xrow0, pol_x);
                        }
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
            int stage = 0, acc = 0;
            uint32_t phase = 0, acc_phase = 0;
            bool ok = true;
            if (lane == 0) ok = test_stall(never_bar, abort_flag);
            ok = __shfl_sync(0xffffffffu, ok, 0);
            for (int tile = cluster; tile < total && ok; tile += n_clusters) {
                int g, wb, r0, rows;
                locate(tile, g, wb, r0, rows);
                const uint32_t idesc = idesc_bf16_f32(256, (rows + 15) / 16 * 16);
                const uint32_t xstride = (uint32_t)(128 >> swap_box_index((rows + 15) / 16 * 8)) * GG_BK * 2;
                if (lane == 0) ok = mbar_wait_bounded(&tempty_bar[acc], acc_phase ^ 1u, abort_flag);
                ok = __shfl_sync(0xffffffffu, ok, 0);
                if (!ok) break;
                tc_fence_after_sync();
                const uint32_t d_tmem = tmem_base + (uint32_t)(acc * GS_MAX_N);
                for (int kb = 0; kb < KB; ++kb) {
                    if (lane == 0) ok = mbar_wait_bounded(&full_bar[stage], phase, abort_flag);
                    ok = __shfl_sync(0xffffffffu, ok, 0);
                    if (!ok) break;
                    tc_fence_after_sync();
                    if (lane == 0) {
                        const int nsub = min(SUB, KBS - kb * SUB);
                        for (int sb = 0; sb < nsub; ++sb) {
                            const uint32_t sa = smem_u32(stages + stage * S::STAGE_BYTES);
                            const uint64_t wdesc = smem_desc_sw128(sa + sb * S::W_BYTES);
                            const uint64_t xdesc = smem_desc_sw128(sa + S::X_OFF + sb * xstride);
#pragma unroll
                            for (int k = 0; k < GG_BK / 16; ++k)
                                umma_bf16_ss_pair(d_tmem, wdesc + 2 * k, xdesc + 2 * k, idesc,
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
        const int q = warp & 3;  // TMEM lanes 32q .. 32q+31
        const uint32_t tempty_leader0 = mapa_shared(smem_u32(&tempty_bar[0]), 0);
        const uint32_t tempty_leader1 = mapa_shared(smem_u32(&tempty_bar[1]), 0);
        // gate|up: the warps of lanes 0-63 (q = 0, 1: gate rows) hand their values to the warps of lanes 64-127
        // (q = 2, 3: up rows), which compute and store h
        const bool ferry = GATEUP && !RAW && q < 2;
        const int p = q & 1;  // hand-off pair (gate|up)
        uint8_t* xbuf = epi + 8192 + p * 4096;
        uint8_t* stage_base = epi + ((GATEUP && !RAW) ? p : (warp - 2)) * 4096;
        uint8_t* save_buf = epi + 16384 + p * 4096 + (ferry ? 0 : 2048);  // SAVE: g (gate warps) or u
        // output row stride and this warp's column limit: RAW gate|up stores gate rows below f, up rows from f on
        const int ld_out = RAW ? 2 * args.f : args.n_out;
        const int col_off = (RAW && q >= 2) ? args.f : 0;
        const int col_end = RAW ? col_off + args.f : args.n_out;
        int acc = 0;
        uint32_t acc_phase = 0;
        uint32_t blocks = 0;  // blocks staged (alternating buffers) or handed off by this warp
        bool ok = true;
        for (int tile = cluster; tile < total; tile += n_clusters) {
            int g, wb, r0, rows;
            locate(tile, g, wb, r0, rows);
            const int row_end = r0 + rows;
            if (lane == 0) ok = mbar_wait_bounded(&tfull_bar[acc], acc_phase, abort_flag);
            ok = __shfl_sync(0xffffffffu, ok, 0);
            if (!ok) break;
            tc_fence_after_sync();
            const uint32_t t_acc = tmem_base + ((uint32_t)(q * 32) << 16) + (uint32_t)(acc * GS_MAX_N);
            // output columns of this warp's lanes
            const int col0 = col_off + (GATEUP ? wb * 128 + 64 * (int)rank + 32 * p : wb * 256 + 128 * (int)rank + 32 * q);
#pragma unroll 1
            for (int c0 = 0; c0 < rows && ok; c0 += 32) {
                uint32_t raw[32];
                tmem_load_32cols(t_acc + (uint32_t)c0, raw);
                float v[32];
                if constexpr (GATEUP && !RAW) {
                    const uint32_t par = blocks & 1u;
                    if (ferry) {
                        // hand off: thread = gate row, 32 token values as eight 16-byte units, XOR-swizzled by lane
                        if (blocks > 0) {
                            ok = mbar_wait_bounded(&xempty_bar[p], par ^ 1u, abort_flag);
                            ok = __all_sync(0xffffffffu, ok);
                            if (!ok) break;
                        }
#pragma unroll
                        for (int u = 0; u < 8; ++u)
                            *reinterpret_cast<uint4*>(xbuf + lane * 128 + ((u ^ (lane & 7)) << 4)) =
                                make_uint4(raw[4 * u], raw[4 * u + 1], raw[4 * u + 2], raw[4 * u + 3]);
                        mbar_arrive(&xfull_bar[p]);
                        if constexpr (SAVE) {  // g of this warp's 32 columns (single buffer: one group per block)
#pragma unroll
                            for (int t = 0; t < 32; ++t) v[t] = __uint_as_float(raw[t]);
                            if (lane == 0) bulk_wait_group_read<0>();
                            __syncwarp();
                            stage_transposed(save_buf, v, lane);
                            flush_staged_block(save_buf, lane, &tmG, args.out2, 2 * args.f, r0 + c0, row_end, col0,
                                               args.f);
                        }
                        ++blocks;
                        continue;
                    }
                    ok = mbar_wait_bounded(&xfull_bar[p], par, abort_flag);
                    ok = __all_sync(0xffffffffu, ok);
                    if (!ok) break;
                    uint32_t gt[32];
#pragma unroll
                    for (int u = 0; u < 8; ++u) {
                        const uint4 w4 = *reinterpret_cast<const uint4*>(xbuf + lane * 128 + ((u ^ (lane & 7)) << 4));
                        gt[4 * u] = w4.x;
                        gt[4 * u + 1] = w4.y;
                        gt[4 * u + 2] = w4.z;
                        gt[4 * u + 3] = w4.w;
                    }
                    mbar_arrive(&xempty_bar[p]);
                    if constexpr (SAVE) {  // u of these columns; groups per block: u, then h
#pragma unroll
                        for (int t = 0; t < 32; ++t) v[t] = __uint_as_float(raw[t]);
                        if (lane == 0) bulk_wait_group_read<1>();  // the previous block's u store (h after it)
                        __syncwarp();
                        stage_transposed(save_buf, v, lane);
                        flush_staged_block(save_buf, lane, &tmG, args.out2, 2 * args.f, r0 + c0, row_end,
                                           args.f + col0, 2 * args.f);
                    }
#pragma unroll
                    for (int t = 0; t < 32; ++t) v[t] = swiglu(__uint_as_float(gt[t]), __uint_as_float(raw[t]));
                } else {
#pragma unroll
                    for (int t = 0; t < 32; ++t) v[t] = __uint_as_float(raw[t]);
                }
                uint8_t* my_stage = stage_base + (int)(blocks & 1u) * 2048;
                ++blocks;
                // the TMA store that last read this buffer is done (SAVE: two blocks back, three groups since)
                if (lane == 0) bulk_wait_group_read<SAVE ? 3 : 1>();
                __syncwarp();
                stage_transposed(my_stage, v, lane);
                flush_staged_block(my_stage, lane, &tmO, args.out, ld_out, r0 + c0, row_end, col0, col_end);
            }
            if (!ok) break;
            tc_fence_before_sync();
            __syncwarp();
            if (lane == 0) mbar_arrive_cluster(acc ? tempty_leader1 : tempty_leader0);
            acc ^= 1;
            if (acc == 0) acc_phase ^= 1u;
            if constexpr (COMBINE) {
                if (col0 < args.n_out) combine_after_tile(cargs, args.out, args.M, args.n_out, r0, rows, col0, lane);
            }
        }
        if (ferry && ok && blocks > 0) {  // the last hand-off has been read before the buffer goes away
            mbar_wait_bounded(&xempty_bar[p], (blocks & 1u) ^ 1u, abort_flag);
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
