// Router on the tensor cores, for large token counts, with top-k fused into the epilogue.
//
// logits[t][e] = sum_i x[t][i] * W_r[e][i] + bias[e] with x bf16 and W_r fp32. The fp32 weights are split
// into three bf16 pieces, W_r = hi + mid + lo (hi = w truncated to bf16, mid = (w - hi) truncated, lo =
// bf16(w - hi - mid); the differences are exact, and for normal weights so is the sum: 24 significand bits
// are 8 + 8 + 8), so the product is three bf16 MMAs x*hi + x*mid + x*lo. bf16*bf16 products are exact in
// fp32. The pieces are either written once beforehand (PRESPLIT, router_split_kernel) and loaded by TMA, or
// made in every call by converter warps.
//
// The tensor core's fp32 accumulator drops low-order bits when it adds (a bias toward zero that grows
// with the number of accumulation steps and the size of the running sum; on a 3 x 4096-long reduction it
// reaches ~1e-5 of the logit). So each 64-wide K block is accumulated on its own, in one of NBUF TMEM
// buffers (as many as fit, up to 8, so the round trip MMA -> drain -> reuse is not on the critical
// path), and CUDA-core threads add the block partials into fp32 registers with IEEE round-to-nearest.
// When 3 * BNR <= 256 the three pieces sit one after another as the rows of a single B operand, so one MMA
// per 16-wide K step (N = 3 * BNR) gives the three partial products side by side in TMEM and the drain adds
// them: 4 MMAs per K block instead of 12 (small-N MMAs cost about as much to issue as large ones).
//
// Split K across a cluster: a 128-token tile is processed by a cluster of CS CTAs (1, 2 or 4), each taking a
// contiguous range of K blocks; the partial sums go through shared memory and the cluster's first CTA adds its
// peers' partials over DSMEM in rank order (deterministic) and runs the epilogue. Small expert counts leave
// few 128-token tiles, so without the split most SMs would idle.
//
// Per CTA (320 threads):
//   warp 0     TMA of the x tile [128 x 64] bf16 per K block into a STAGES-deep ring, with (PRESPLIT) the
//              three pieces [3 x BNR x 64] bf16 in one box, or (BNR <= 64) the W_r block [BNR x 64] fp32
//              (unswizzled, 256 bytes per expert row)
//   warp 1     TMEM allocation; one lane issues the K block's tcgen05.mma (M=128; 4 of N = 3*BNR, or 3 x 4 of
//              N = BNR) into accumulator buffer (kb % NBUF), starting it afresh
//   warps 2-5  (not PRESPLIT) convert the W_r block (staged, or read from L2 when BNR = 128) into the three
//              bf16 pieces, stored in the 128-byte-swizzled K-major layout the TMA engine writes, then signal
//              conv[stage]
//   warps 6-9  drain: add each finished block partial of their 32 TMEM lanes into registers
// Epilogue (the cluster's first CTA), top-k by insertion into a sorted list of 8 (descending, equal logits keep
// the lower expert id first), then the routing weights of the mode:
//   BNR <= 32, k <= 8: each drain thread routes its own token from its registers (the unrolled insertion is
//              short for so few experts), storing its logits row itself;
//   otherwise: the sums + bias go to shared memory; warps 4-9 store the logits row by row (coalesced) while
//              threads 0-127 route one token each with a loop over the experts that skips logits not above the
//              current k-th (k > 8: one warp per token runs warp_route_select, the stand-alone top-k code).
#pragma once
#include "common.cuh"
#include "route.cuh"

namespace moe {

constexpr int RTC_BM = 128, RTC_BK = 64, RTC_THREADS = 320, RTC_KMAX = 32, RTC_KINS = 8;
constexpr int RTC_RED_LD = RTC_BM + 1;  // row stride of the [expert][token] sums in shared memory (odd: no bank conflicts)

// PRESPLIT: the three bf16 pieces of W_r were written once by router_split_kernel ([3][E][d], as the weights do
// not change between calls) and arrive with the x tile by TMA; the converter warps then have nothing to do.
template <int BNR, bool PRESPLIT = false>
struct RouterTcShape {
    static_assert(BNR % 16 == 0 && BNR >= 16 && BNR <= 128, "UMMA N (and the drain's register budget)");
    static constexpr int A_BYTES = RTC_BM * RTC_BK * 2;  // x tile, bf16
    // BNR = 128: the converters read their W_r values from global memory (L2; loads issued before the stage
    // wait) instead of a TMA-staged fp32 block, which leaves room for a 3-stage ring (64 KB stages, not 96 KB)
    static constexpr bool W_DIRECT = BNR > 64 && !PRESPLIT;
    static constexpr int W_BYTES = (W_DIRECT || PRESPLIT) ? 0 : BNR * RTC_BK * 4;  // W_r block, fp32 as loaded
    static constexpr int P_BYTES = BNR * RTC_BK * 2;     // one bf16 piece
    static constexpr int STAGE_BYTES = A_BYTES + W_BYTES + 3 * P_BYTES;
    static_assert(STAGE_BYTES % 1024 == 0, "stage bases stay 1024-byte aligned");
    static constexpr int STAGES = (200 * 1024) / STAGE_BYTES > 8 ? 8 : (200 * 1024) / STAGE_BYTES;
    static_assert(STAGES >= 2, "ring depth");
    static constexpr bool JOINT = 3 * BNR <= 256;                // one MMA over [hi; mid; lo] per K step
    static constexpr int ACC_COLS = JOINT ? 3 * BNR : BNR;           // TMEM columns of one K block's result
    static constexpr int ACC_STRIDE = ACC_COLS <= 64 ? 64 : (ACC_COLS <= 128 ? 128 : 256);
    static constexpr int NBUF = 512 / ACC_STRIDE >= 8 ? 8 : 512 / ACC_STRIDE;  // partial-sum buffers in TMEM
    static constexpr int TMEM_COLS = NBUF * ACC_STRIDE <= 256 ? 256 : 512;
    static constexpr int BAR_BYTES = 512;
    static constexpr int SMEM_BYTES = 1024 + STAGES * STAGE_BYTES + BAR_BYTES;
    static_assert(SMEM_BYTES <= 232448, "shared memory");
    static_assert((3 * STAGES + 2 * NBUF + 1) * 8 + 8 <= BAR_BYTES, "barrier area");
    static_assert(BNR * RTC_RED_LD * 4 <= STAGES * STAGE_BYTES, "epilogue sums reuse the ring");
};

// Exact three-way split of two fp32 weights into bf16 pieces, packed in pairs: hi = w truncated to bf16
// (its top 16 bits), mid = (w - hi) truncated likewise, lo = bf16(w - hi - mid) rounded to nearest; the two
// subtractions are exact, so hi + mid + lo equals w to ~2^-25 relative.
__device__ __forceinline__ void split3_pair(float w0, float w1, uint32_t& hi, uint32_t& mid, uint32_t& lo) {
    const uint32_t u0 = __float_as_uint(w0), u1 = __float_as_uint(w1);
    const float r0 = w0 - __uint_as_float(u0 & 0xffff0000u), r1 = w1 - __uint_as_float(u1 & 0xffff0000u);
    const uint32_t v0 = __float_as_uint(r0), v1 = __float_as_uint(r1);
    const float s0 = r0 - __uint_as_float(v0 & 0xffff0000u), s1 = r1 - __uint_as_float(v1 & 0xffff0000u);
    hi = __byte_perm(u0, u1, 0x7632);  // upper halves: element 0 in the low 16 bits
    mid = __byte_perm(v0, v1, 0x7632);
    lo = pack_bf16x2(s0, s1);
}

// Routing weights of the first k entries of a sorted selection (tv descending, te the expert ids):
//   sigmoid_topk_norm    sigmoid(v_j) / sum of the selected sigmoids
//   topk_softmax         softmax over the selected logits
//   softmax_topk_renorm  softmax over all E logits (zall = sum_e exp(v_e - v_max)), renormalised over the selection
__device__ __forceinline__ void route_weights(const float (&tv)[RTC_KINS], const int (&te)[RTC_KINS], int k, int mode,
                                              float zall, int32_t* __restrict__ idx_row, float* __restrict__ w_row) {
    float wv[RTC_KINS];
    float z = 0.f;
    if (mode == MOE_ROUTE_SIGMOID_TOPK_NORM) {
#pragma unroll
        for (int j = 0; j < RTC_KINS; ++j)
            if (j < k) {
                wv[j] = 1.f / (1.f + expf(-tv[j]));
                z += wv[j];
            }
    } else {
#pragma unroll
        for (int j = 0; j < RTC_KINS; ++j)
            if (j < k) {
                wv[j] = expf(tv[j] - tv[0]);
                z += wv[j];
            }
        if (mode == MOE_ROUTE_SOFTMAX_TOPK_RENORM) {
            float zp = 0.f;
#pragma unroll
            for (int j = 0; j < RTC_KINS; ++j)
                if (j < k) {
                    wv[j] = wv[j] / zall;
                    zp += wv[j];
                }
            z = zp;
        }
    }
#pragma unroll
    for (int j = 0; j < RTC_KINS; ++j)
        if (j < k) {
            idx_row[j] = te[j];
            w_row[j] = wv[j] / z;
        }
}

// Routes one token from its E logits at col[e * RTC_RED_LD] (shared memory), k <= RTC_KINS: tv/te hold the
// RTC_KINS largest so far in the order (descending value, lower expert id first); a new logit bubbles down from
// the top, taking the first slot it beats strictly, so an equal value stays behind the earlier (lower) id.
// Logits not above the current k-th are skipped (they cannot reach the first k slots).
__device__ __forceinline__ void route_token_insertion(const float* col, int E, int k, int mode,
                                                      int32_t* __restrict__ idx_row, float* __restrict__ w_row) {
    float tv[RTC_KINS];
    int te[RTC_KINS];
#pragma unroll
    for (int i = 0; i < RTC_KINS; ++i) {
        tv[i] = 0.f;
        te[i] = INT_MAX;
    }
    int filled = 0;  // min(experts seen, k)
    float kth = 0.f;  // tv[k-1] once filled == k
#pragma unroll 4
    for (int e = 0; e < E; ++e) {
        float cv = col[e * RTC_RED_LD];
        if (filled == k && !(cv > kth)) continue;
        int ce = e;
#pragma unroll
        for (int i = 0; i < RTC_KINS; ++i) {
            if (te[i] == INT_MAX || cv > tv[i]) {
                const float tf = tv[i];
                const int ti = te[i];
                tv[i] = cv;
                te[i] = ce;
                cv = tf;
                ce = ti;
            }
        }
        if (filled < k) ++filled;
#pragma unroll
        for (int i = 0; i < RTC_KINS; ++i)
            if (i == k - 1) kth = tv[i];
    }
    float zall = 0.f;  // softmax over all E logits, relative to the largest (renormalising mode only)
    if (mode == MOE_ROUTE_SOFTMAX_TOPK_RENORM)
        for (int e = 0; e < E; ++e) zall += expf(col[e * RTC_RED_LD] - tv[0]);
    route_weights(tv, te, k, mode, zall, idx_row, w_row);
}

// Converter thread ct's share of one 64-wide K block of W_r, read from global memory: item it is expert row
// (ct + 128*it) / 8, columns col0 + 8*((ct + 128*it) % 8) .. +8; rows past E and columns past d are zeros (d is a
// multiple of 8, so a chunk is all in or all out).
template <int ITEMS, int N>
__device__ __forceinline__ void router_load_w_chunks(float4 (&wv)[N][2], const float* __restrict__ w_router, int ct,
                                                     int col0, int E, int d) {
#pragma unroll
    for (int it = 0; it < ITEMS; ++it) {
        const int item = ct + 128 * it;
        const int r = item >> 3, col = col0 + (item & 7) * 8;
        if (r < E && col < d) {
            const float4* src = reinterpret_cast<const float4*>(w_router + (size_t)r * d + col);
            wv[it][0] = __ldg(src);
            wv[it][1] = __ldg(src + 1);
        } else {
            wv[it][0] = wv[it][1] = make_float4(0.f, 0.f, 0.f, 0.f);
        }
    }
}

template <int BNR, bool PRESPLIT = false>
__global__ void __launch_bounds__(RTC_THREADS, 1)
    router_tc_kernel(const __grid_constant__ CUtensorMap tmX, const __grid_constant__ CUtensorMap tmW,
                     const __grid_constant__ CUtensorMap tmP, const float* __restrict__ w_router,
                     const float* __restrict__ bias, int T, int d, int E, int k, int mode, int fuse_topk,
                     float* __restrict__ logits, int32_t* __restrict__ topk_idx, float* __restrict__ topk_w) {
    using S = RouterTcShape<BNR, PRESPLIT>;
    // tmP (PRESPLIT): the pieces [3][E][d] bf16, boxes of 64 x BNR x 3 (all three pieces of a K block at once)
    constexpr int STAGES = S::STAGES;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    uint64_t* full_bar = reinterpret_cast<uint64_t*>(smem + STAGES * S::STAGE_BYTES);  // TMA landed
    uint64_t* conv_bar = full_bar + STAGES;                                            // pieces written
    uint64_t* empty_bar = conv_bar + STAGES;                                           // MMA done
    constexpr int NBUF = S::NBUF;
    uint64_t* tfull_bar = empty_bar + STAGES;  // [NBUF]
    uint64_t* tempty_bar = tfull_bar + NBUF;   // [NBUF]
    uint64_t* final_bar = tempty_bar + NBUF;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(final_bar + 1);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t rank = cluster_ctarank(), cs = cluster_nctarank();
    const int m0 = (int)(blockIdx.x / cs) * RTC_BM;
    const int KB_all = (d + RTC_BK - 1) / RTC_BK;
    const int kb0 = (int)(rank * KB_all / cs);                          // this CTA's K blocks
    const int KB = (int)((rank + 1) * KB_all / cs) - kb0;              // (count; the host keeps it >= 1)

    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(&full_bar[s], 1);
            mbar_init(&conv_bar[s], 128);  // every converter thread
            mbar_init(&empty_bar[s], 1);
        }
        for (int a = 0; a < NBUF; ++a) {
            mbar_init(&tfull_bar[a], 1);
            mbar_init(&tempty_bar[a], 4);  // lane 0 of each drain warp
        }
        mbar_init(final_bar, 1);
        *abort_flag = 0;
        fence_mbar_init();
        tma_prefetch_desc(&tmX);
        tma_prefetch_desc(PRESPLIT ? &tmP : &tmW);
    }
    if (warp == 1) {
        tmem_alloc(tmem_slot, S::TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before_sync();
    __syncthreads();
    tc_fence_after_sync();
    const uint32_t tmem_base = *tmem_slot;
    grid_dep_wait();  // x, W_r and the outputs' earlier readers: everything below follows earlier kernels
    grid_dep_trigger();
    // drain warps (6-9): this thread's row of the tile
    const int q = warp & 3;  // TMEM lanes 32q .. 32q+31
    const bool is_drain = warp >= 6;
    bool drain_ok = false;
    // [BNR][RTC_RED_LD] row sums, expert-major, over the ring once the last K block is drained (the ring is then
    // idle: every TMA copy, conversion and MMA of this CTA has completed)
    float* red = reinterpret_cast<float*>(smem);

    if (warp == 0) {
        // ---------------- TMA: x tile ----------------
        int stage = 0;
        uint32_t phase = 0;
        int issued = 0;
        bool ok = true;
        const uint64_t pol = l2_policy_evict_first();      // x: read once per tile
        const uint64_t pol_w = l2_policy_evict_last();     // W_r: read by every tile
        for (int kb = 0; kb < KB; ++kb) {
            if (lane == 0) ok = mbar_wait_bounded(&empty_bar[stage], phase ^ 1u, abort_flag);
            ok = __shfl_sync(0xffffffffu, ok, 0);
            if (!ok) break;
            if (lane == 0) {
                uint8_t* sa = smem + stage * S::STAGE_BYTES;
                mbar_arrive_expect_tx(&full_bar[stage], S::A_BYTES + (PRESPLIT ? 3 * S::P_BYTES : S::W_BYTES));
                tma_load_2d(sa, &tmX, &full_bar[stage], (kb0 + kb) * RTC_BK, m0, pol);
                if (PRESPLIT)  // hi, mid, lo land as the three consecutive piece blocks the MMA reads
                    tma_load_3d(sa + S::A_BYTES, &tmP, &full_bar[stage], (kb0 + kb) * RTC_BK, 0, 0, pol_w);
                else if (!S::W_DIRECT)
                    tma_load_2d(sa + S::A_BYTES, &tmW, &full_bar[stage], (kb0 + kb) * RTC_BK, 0, pol_w);
            }
            ++issued;
            if (++stage == STAGES) {
                stage = 0;
                phase ^= 1u;
            }
        }
        if (lane == 0)
            for (int n = issued > STAGES ? issued - STAGES : 0; n < issued; ++n)
                mbar_wait_drain(&full_bar[n % STAGES], (uint32_t)((n / STAGES) & 1));
        __syncwarp();
    } else if (warp == 1) {
        // ---------------- MMA: one fresh accumulation per K block ----------------
        constexpr uint32_t IDESC = idesc_bf16_f32(RTC_BM, S::ACC_COLS);
        int stage = 0;
        uint32_t phase = 0;
        bool ok = true;
        for (int kb = 0; kb < KB; ++kb) {
            const int acc = kb % NBUF;
            if (lane == 0) ok = mbar_wait_bounded(&tempty_bar[acc], ((kb / NBUF) & 1) ^ 1u, abort_flag);
            ok = __shfl_sync(0xffffffffu, ok, 0);
            if (!ok) break;
            if (lane == 0) ok = (PRESPLIT || mbar_wait_bounded(&conv_bar[stage], phase, abort_flag)) &&
                                mbar_wait_bounded(&full_bar[stage], phase, abort_flag);
            ok = __shfl_sync(0xffffffffu, ok, 0);
            if (!ok) break;
            tc_fence_after_sync();
            if (lane == 0) {
                const uint32_t sa = smem_u32(smem + stage * S::STAGE_BYTES);
                const uint64_t adesc = smem_desc_sw128(sa);
                const uint32_t d_tmem = tmem_base + (uint32_t)(acc * S::ACC_STRIDE);
                if constexpr (S::JOINT) {  // the pieces are consecutive row blocks: one B operand of 3*BNR rows
                    const uint64_t bdesc = smem_desc_sw128(sa + S::A_BYTES + S::W_BYTES);
#pragma unroll
                    for (int kk = 0; kk < RTC_BK / 16; ++kk)
                        umma_bf16_ss(d_tmem, adesc + 2 * kk, bdesc + 2 * kk, IDESC, kk != 0 ? 1u : 0u);
                } else {
#pragma unroll
                    for (int p = 0; p < 3; ++p) {
                        const uint64_t bdesc = smem_desc_sw128(sa + S::A_BYTES + S::W_BYTES + p * S::P_BYTES);
#pragma unroll
                        for (int kk = 0; kk < RTC_BK / 16; ++kk)
                            umma_bf16_ss(d_tmem, adesc + 2 * kk, bdesc + 2 * kk, IDESC, (p | kk) != 0 ? 1u : 0u);
                    }
                }
                umma_commit(&empty_bar[stage]);
                umma_commit(&tfull_bar[acc]);
            }
            __syncwarp();
            if (++stage == STAGES) {
                stage = 0;
                phase ^= 1u;
            }
        }
        if (lane == 0) umma_commit(final_bar);
        __syncwarp();
    } else if (warp < 6) {
        // ---------------- converters: W_r block (fp32) -> hi/mid/lo bf16 pieces (idle if PRESPLIT) ----------------
        const int ct = threadIdx.x - 64;  // 0..127
        int stage = 0;
        uint32_t phase = 0;
        bool ok = true;
        constexpr int ITEMS = BNR * (RTC_BK / 8) / 128;  // 16-byte output chunks per thread per piece
        for (int kb = 0; kb < (PRESPLIT ? 0 : KB); ++kb) {
            float4 wv[S::W_DIRECT ? ITEMS : 1][2];  // W_DIRECT: this K block's chunks, in flight during the wait
            if constexpr (S::W_DIRECT) router_load_w_chunks<ITEMS>(wv, w_router, ct, (kb0 + kb) * RTC_BK, E, d);
            if (lane == 0) ok = mbar_wait_bounded(&full_bar[stage], phase, abort_flag);
            ok = __shfl_sync(0xffffffffu, ok, 0);
            if (!ok) break;
            const uint8_t* wbase = smem + stage * S::STAGE_BYTES + S::A_BYTES;
            uint8_t* pbase = smem + stage * S::STAGE_BYTES + S::A_BYTES + S::W_BYTES;
#pragma unroll
            for (int it = 0; it < ITEMS; ++it) {
                const int item = ct + 128 * it;
                const int r = item >> 3, c = item & 7;  // expert row, 8-element chunk of the 64-wide block
                float4 v0, v1;  // rows past E and columns past d are zeros
                if constexpr (S::W_DIRECT) {
                    v0 = wv[it][0];
                    v1 = wv[it][1];
                } else {
                    const float4* src = reinterpret_cast<const float4*>(wbase + r * (RTC_BK * 4) + c * 32);
                    v0 = src[0];
                    v1 = src[1];
                }
                const float w8[8] = {v0.x, v0.y, v0.z, v0.w, v1.x, v1.y, v1.z, v1.w};
                uint32_t hi[4], mi[4], lo[4];
#pragma unroll
                for (int j = 0; j < 4; ++j) split3_pair(w8[2 * j], w8[2 * j + 1], hi[j], mi[j], lo[j]);
                const int off = r * 128 + ((c ^ (r & 7)) << 4);
                *reinterpret_cast<uint4*>(pbase + off) = make_uint4(hi[0], hi[1], hi[2], hi[3]);
                *reinterpret_cast<uint4*>(pbase + S::P_BYTES + off) = make_uint4(mi[0], mi[1], mi[2], mi[3]);
                *reinterpret_cast<uint4*>(pbase + 2 * S::P_BYTES + off) = make_uint4(lo[0], lo[1], lo[2], lo[3]);
            }
            asm volatile("fence.proxy.async.shared::cta;" ::: "memory");  // generic writes -> tensor core
            mbar_arrive(&conv_bar[stage]);
            if (++stage == STAGES) {
                stage = 0;
                phase ^= 1u;
            }
        }
    } else {
        // ---------------- drain (warps 6-9) ----------------
        const uint32_t t_row = tmem_base + ((uint32_t)(q * 32) << 16);
        float sum[BNR];  // this thread's row: running fp32 sums of the K-block partials
#pragma unroll
        for (int j = 0; j < BNR; ++j) sum[j] = 0.f;
        bool ok = true;
        for (int kb = 0; kb < KB; ++kb) {
            const int acc = kb % NBUF;
            if (lane == 0) ok = mbar_wait_bounded(&tfull_bar[acc], (kb / NBUF) & 1, abort_flag);
            ok = __shfl_sync(0xffffffffu, ok, 0);
            if (!ok) break;
            tc_fence_after_sync();
            const uint32_t t_acc = t_row + (uint32_t)(acc * S::ACC_STRIDE);
            if constexpr (S::JOINT && BNR == 16) {
                uint32_t h[16], m[16], l[16];
                tmem_load_16cols(t_acc, h);
                tmem_load_16cols(t_acc + 16, m);
                tmem_load_16cols(t_acc + 32, l);
#pragma unroll
                for (int j = 0; j < 16; ++j)
                    sum[j] += (__uint_as_float(h[j]) + __uint_as_float(m[j])) + __uint_as_float(l[j]);
            } else if constexpr (S::JOINT) {
#pragma unroll
                for (int c0 = 0; c0 < BNR; c0 += 32) {
                    if (c0 < E) {
                        uint32_t h[32], m[32], l[32];
                        tmem_load_32cols(t_acc + c0, h);
                        tmem_load_32cols(t_acc + BNR + c0, m);
                        tmem_load_32cols(t_acc + 2 * BNR + c0, l);
#pragma unroll
                        for (int j = 0; j < 32; ++j)
                            sum[c0 + j] += (__uint_as_float(h[j]) + __uint_as_float(m[j])) + __uint_as_float(l[j]);
                    }
                }
            } else {
#pragma unroll
                for (int c0 = 0; c0 < BNR; c0 += 32) {
                    if (c0 < E) {
                        uint32_t v[32];
                        tmem_load_32cols(t_acc + c0, v);
#pragma unroll
                        for (int j = 0; j < 32; ++j) sum[c0 + j] += __uint_as_float(v[j]);
                    }
                }
            }
            tc_fence_before_sync();
            __syncwarp();
            if (lane == 0) mbar_arrive(&tempty_bar[acc]);
        }
        drain_ok = ok;
        if (ok) {
#pragma unroll
            for (int j = 0; j < BNR; ++j) red[j * RTC_RED_LD + q * 32 + lane] = sum[j];
        }
    }

    // ---- split-K reduction over the cluster, then the epilogue in the cluster's first CTA ----
    tc_fence_before_sync();
    __syncthreads();  // all roles done, every partial sum is in red
    if (cs > 1) {
        cluster_sync();
        if (rank == 0 && is_drain) {  // own partial, then the peers' in rank order: deterministic
            const uint32_t base = smem_u32(red);
            float v[BNR];
#pragma unroll
            for (int j = 0; j < BNR; ++j) v[j] = red[j * RTC_RED_LD + q * 32 + lane];
            for (uint32_t r = 1; r < cs; ++r) {
                const uint32_t peer = mapa_shared(base, r);
#pragma unroll
                for (int j = 0; j < BNR; ++j)  // independent remote loads, all in flight
                    v[j] += ld_shared_cluster_f32(peer + (uint32_t)((j * RTC_RED_LD + q * 32 + lane) * 4));
            }
#pragma unroll
            for (int j = 0; j < BNR; ++j) red[j * RTC_RED_LD + q * 32 + lane] = v[j];
        }
        cluster_sync();  // no CTA leaves while the first one may still read its shared memory
        // (a CTA whose pipeline wait gave up has already set the device error word)
    }
    if (rank == 0 && BNR <= 32 && fuse_topk && k <= RTC_KINS) {
        if (is_drain && drain_ok && !*abort_flag) {
            const int row = m0 + q * 32 + lane;
            float* lrow = logits + (size_t)(row < T ? row : 0) * E;
            float sum[BNR];
#pragma unroll
            for (int j = 0; j < BNR; ++j) sum[j] = red[j * RTC_RED_LD + q * 32 + lane];
            float tv[RTC_KINS];
            int te[RTC_KINS];
#pragma unroll
            for (int i = 0; i < RTC_KINS; ++i) {
                tv[i] = 0.f;
                te[i] = INT_MAX;
            }
#pragma unroll
            for (int e = 0; e < BNR; ++e) {
                if (e < E) {
                    sum[e] += bias ? __ldg(bias + e) : 0.f;
                    if (row < T) lrow[e] = sum[e];
                    float cv = sum[e];
                    int ce = e;
#pragma unroll
                    for (int i = 0; i < RTC_KINS; ++i) {
                        if (te[i] == INT_MAX || cv > tv[i]) {
                            const float tf = tv[i];
                            const int ti = te[i];
                            tv[i] = cv;
                            te[i] = ce;
                            cv = tf;
                            ce = ti;
                        }
                    }
                }
            }
            if (row < T) {
                float zall = 0.f;  // softmax over all E logits, relative to the largest (renormalising mode only)
                if (mode == MOE_ROUTE_SOFTMAX_TOPK_RENORM) {
#pragma unroll
                    for (int e = 0; e < BNR; ++e)
                        if (e < E) zall += expf(sum[e] - tv[0]);
                }
                route_weights(tv, te, k, mode, zall, topk_idx + (size_t)row * k, topk_w + (size_t)row * k);
            }
        }
    } else if (rank == 0) {
        if (is_drain) {
#pragma unroll
            for (int j = 0; j < BNR; ++j)
                if (j < E) red[j * RTC_RED_LD + q * 32 + lane] += bias ? __ldg(bias + j) : 0.f;
        }
        __syncthreads();
        if (!*abort_flag) {
            if (warp >= 4) {  // logits, row by row
                for (int r = warp - 4; r < RTC_BM && m0 + r < T; r += RTC_THREADS / 32 - 4) {
                    float* lrow = logits + (size_t)(m0 + r) * E;
                    for (int e = lane; e < E; e += 32) lrow[e] = red[e * RTC_RED_LD + r];
                }
            } else if (fuse_topk && k <= RTC_KINS) {
                const int r = threadIdx.x;  // one token per thread
                if (m0 + r < T) route_token_insertion(red + r, E, k, mode, topk_idx + (size_t)(m0 + r) * k,
                                                      topk_w + (size_t)(m0 + r) * k);
            }
            if (fuse_topk && k > RTC_KINS) {
                __syncthreads();  // warps 4-9 join once the logits are out
                for (int r = warp; r < RTC_BM && m0 + r < T; r += RTC_THREADS / 32) {
                    const float* col = red + r;
                    warp_route_select([=](int e) { return col[e * RTC_RED_LD]; }, E, k, mode,
                                      topk_idx + (size_t)(m0 + r) * k, topk_w + (size_t)(m0 + r) * k);
                }
            }
        }
    }

    tc_fence_after_sync();
    if (warp == 1) {
        if (lane == 0) mbar_wait_drain(final_bar, 0);
        __syncwarp();
        tmem_dealloc(tmem_base, S::TMEM_COLS);
    }
}

// The three bf16 pieces of W_r ([E][d] fp32 -> hi, mid, lo planes of [E][d] bf16, split3_pair on each pair of
// weights): written once, read by router_tc_kernel<.., true> on every call.
__global__ void __launch_bounds__(256) router_split_kernel(const float* __restrict__ w, long n_pairs,
                                                           uint32_t* __restrict__ hi, uint32_t* __restrict__ mid,
                                                           uint32_t* __restrict__ lo) {
    grid_dep_wait();
    grid_dep_trigger();
    for (long i = (long)blockIdx.x * 256 + threadIdx.x; i < n_pairs; i += (long)gridDim.x * 256) {
        const float2 v = reinterpret_cast<const float2*>(w)[i];
        uint32_t h, m, l;
        split3_pair(v.x, v.y, h, m, l);
        hi[i] = h;
        mid[i] = m;
        lo[i] = l;
    }
}

// ---- small token counts: logits on CUDA cores, parallel over experts -----------------------------------
// Block b handles experts [b*EPB, b*EPB + EPB) (EPB <= 4) for every token. W_r rows of the block's experts are
// staged in shared memory; each warp then takes RS_TPW tokens at a time and walks d in 16-byte vectors of x,
// so RS_TPW independent loads per lane are in flight; dot products are reduced across lanes with shuffles
// in a fixed order (deterministic).
constexpr int RS_THREADS = 256, RS_TPW = 8;

__global__ void __launch_bounds__(RS_THREADS) router_logits_small_kernel(const __nv_bfloat16* __restrict__ x,
                                                                         const float* __restrict__ w_router,
                                                                         const float* __restrict__ bias, int T,
                                                                         int d, int E, int epb,
                                                                         float* __restrict__ logits) {
    extern __shared__ float wsm[];  // [epb][d]
    grid_dep_wait();
    grid_dep_trigger();
    const int e0 = blockIdx.x * epb;
    const int ne = min(epb, E - e0);
    {
        const float4* src = reinterpret_cast<const float4*>(w_router + (size_t)e0 * d);
        float4* dst = reinterpret_cast<float4*>(wsm);
        const int n4 = ne * d / 4;
#pragma unroll 4
        for (int i = threadIdx.x; i < n4; i += RS_THREADS) dst[i] = __ldg(src + i);
    }
    __syncthreads();
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int nvec = d / 8;
    for (int t0 = warp * RS_TPW; t0 < T; t0 += (RS_THREADS / 32) * RS_TPW) {
        float acc[RS_TPW][4];
#pragma unroll
        for (int i = 0; i < RS_TPW; ++i)
#pragma unroll
            for (int e = 0; e < 4; ++e) acc[i][e] = 0.f;
#pragma unroll 2
        for (int v = lane; v < nvec; v += 32) {
            uint4 q[RS_TPW];
#pragma unroll
            for (int i = 0; i < RS_TPW; ++i)
                q[i] = t0 + i < T ? __ldg(reinterpret_cast<const uint4*>(x + (size_t)(t0 + i) * d) + v)
                                  : make_uint4(0, 0, 0, 0);
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                if (e < ne) {
                    const float4* wr = reinterpret_cast<const float4*>(wsm + (size_t)e * d + v * 8);
                    const float4 a = wr[0], b = wr[1];
#pragma unroll
                    for (int i = 0; i < RS_TPW; ++i) {
                        const float2 x01 = unpack_bf16x2(q[i].x), x23 = unpack_bf16x2(q[i].y);
                        const float2 x45 = unpack_bf16x2(q[i].z), x67 = unpack_bf16x2(q[i].w);
                        float s = acc[i][e];
                        s = fmaf(x01.x, a.x, s);
                        s = fmaf(x01.y, a.y, s);
                        s = fmaf(x23.x, a.z, s);
                        s = fmaf(x23.y, a.w, s);
                        s = fmaf(x45.x, b.x, s);
                        s = fmaf(x45.y, b.y, s);
                        s = fmaf(x67.x, b.z, s);
                        s = fmaf(x67.y, b.w, s);
                        acc[i][e] = s;
                    }
                }
            }
        }
#pragma unroll
        for (int i = 0; i < RS_TPW; ++i)
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                float s = acc[i][e];
#pragma unroll
                for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
                if (lane == 0 && e < ne && t0 + i < T)
                    logits[(size_t)(t0 + i) * E + e0 + e] = s + (bias ? bias[e0 + e] : 0.f);
            }
    }
}

}  // namespace moe
