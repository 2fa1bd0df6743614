// MXFP4 grouped GEMM for a few rows per expert (decode), on warp-level MMAs in f16.
//
// Decode streams each active expert's weights once for a handful of token rows, so the kernel must turn 4-bit
// codes into MMA operands at the HBM rate (about 44 weights per clock per SM on B200). The tensor-memory kernel
// (gemm_fp4.cuh) is held below that by the narrow tcgen05 MMA (M = 128 weight rows, N = 16 tokens, K = 16 per
// instruction). Here each warp owns 16 weight rows and runs mma.sync m16n8k16 (N = 8 tokens), which costs next to
// nothing at these sizes, so the limit becomes instruction issue, and decoding is cut to one conversion
// instruction per code pair:
//   - the hardware's E2M1 -> f16 conversion (cvt.rn.f16x2.e2m1x2) turns one byte (two codes) into an f16 pair,
//     exactly, with no scale applied;
//   - every MMA covers 16 codes of one 32-element scale block, so the block's scale 2^(s - 127) multiplies the
//     MMA's fp32 partial sums (two MMAs per block, one fused multiply-add per accumulator element);
//   - the activations are f16 too: each token row is scaled by a power of two 2^-e (its largest magnitude lands in
//     [16, 32)) so that its bf16 values convert to f16 exactly (f16 has three more mantissa bits than bf16; only
//     values 2^-18 below the row maximum fall into f16's subnormal range), and the outputs are multiplied back by
//     2^e.
// The sums are those of the bf16 path up to fp32 rounding order: products of exact weights and exact activations,
// fp32 accumulation.
//
// Operand order inside an MMA. The 16 "K columns" of an MMA need not be 16 consecutive k: any assignment works if
// A and B use the same one. A thread of the m16n8k16 layout holds, for each of its two weight rows, the columns
// (2t, 2t+1) and (2t+8, 2t+9) (t = lane % 4). The code layout puts elements 8t' + {0,2,4,6} in bytes 0, 1 and
// 8t' + {1,3,5,7} in bytes 2, 3 of the 32-bit word t' of a 16-byte block; so thread t reads word t of its rows'
// block (one 32-bit shared-memory load per row) and feeds bytes 0, 1 to the block's first MMA and bytes 2, 3 to its
// second: both MMAs then draw their 16 codes from the one scale block. The activations are stored to match: per
// token, block and t, 16 bytes of f16 in the order x0 x2 x4 x6 x1 x3 x5 x7 (x_i = element 32b + 8t + i), one
// 16-byte load giving the B fragments of both MMAs. (A byte's low code goes to the low half of the f16 pair.)
//
// CTA (544 threads, one per SM, persistent over its range of units): warps 0-15 compute, warp 16 is the TMA producer.
// Work unit = (group g, block of 8 token rows, one weight block: 256 rows for down; 128 gate rows and the matching
// 128 up rows for gate|up), numbered group by group, token block by token block, weight block by weight block.
// Every unit streams the same bytes, so CTA b takes the contiguous range [U b / grid, U (b + 1) / grid) of the U
// units (balanced to one unit whatever U; a fixed tile size left up to half an SM wave idle at the end). A range
// splits into segments, one per token block it touches (usually two or three), and the token rows are loaded and
// converted once per segment. Per segment the producer loads the 8 token rows whole (one box per row) and then
// streams, per weight block, stages of K = 256: codes [128 rows x 128 bytes] (128-byte swizzle) and scales [8 x 128]
// per projection. Warps 0-7 scale and convert the token rows in place once per segment (warp w takes row w). Warps w and
// w + 8 compute weight rows 16w .. 16w+15 of each block, w the even and w + 8 the odd 32-element blocks of every
// stage (four warps per SM sub-partition hide the MMA and load latencies); at the end of a weight block warp w + 8
// hands its partial sums to warp w through shared memory, which adds them to its own (always in that order) and
// stores the outputs. Every wait is bounded.
#pragma once
#include "common.cuh"
#include "gemm.cuh"
#include "gemm_fp4.cuh"
#include <cuda_fp16.h>

namespace moe {

constexpr int FW_NT = 8;                      // token rows per token block (the MMA's N)
constexpr int FW_WARPS = 16;                  // compute warps
constexpr int FW_THREADS = (FW_WARPS + 1) * 32;
constexpr int FW_KS = GF_KS;                  // K per stage: 256 (128 bytes of codes per row)
constexpr int FW_MAX_K = 8192;                // one TMA box per token row: K / 32 <= 256
constexpr int FW_BAR_BYTES = 512;

// gate|up: blocks of 128 weight rows (and the matching 128 up rows), two warps per 16 rows (even / odd K blocks);
// down: blocks of 256 rows, one warp per 16 rows over all of K (no hand-off; K is short: d x f = 7168 x 2048)
template <bool GATEUP>
struct GemmFp4WarpShape {
    static constexpr int RW = GATEUP ? 8 : 16;         // row warps, 16 weight rows each
    static constexpr int KSPL = FW_WARPS / RW;         // warps per 16 rows
    static constexpr int BM = 16 * RW;                 // weight rows per block
    static constexpr int BLOCKS = GATEUP ? 2 : 1;
    static constexpr int Q_BYTES = BM * (FW_KS / 2);   // codes of one projection block (16 or 32 KB)
    static constexpr int S_BYTES = (FW_KS / 32) * BM;  // its scales
    static constexpr int RED_BYTES = KSPL > 1 ? RW * 32 * 8 * 4 : 0;  // partial sums handed from warp w + RW to w
    // down: the block scales through a 256-entry table of 2^(s - 127) in shared memory (a load instead of a shift
    // and a max on the busier integer pipe; measured: down 0.465 -> 0.448 ms on the decode layer, while gate|up,
    // whose ring has no room to spare, ran 1.5% slower with it)
    static constexpr bool SCALE_LUT = !GATEUP;
    static constexpr int LUT_BYTES = SCALE_LUT ? 1024 : 0;
    static constexpr int STAGE_BYTES = BLOCKS * (Q_BYTES + S_BYTES);
    __host__ __device__ static int table_bytes(int G) { return (2 * (G + 1) * 4 + 127) / 128 * 128; }
    static_assert(STAGE_BYTES % 1024 == 0, "stages start on 1024-byte atoms");
    // token row stride in shared memory: K rounded up to 64 elements (the odd rows' 32-element blocks are stored
    // swapped in pairs), in bytes
    __host__ __device__ static int row_bytes(int K) { return (K + 63) / 64 * 64 * 2; }
    __host__ __device__ static int b_bytes(int K) { return FW_NT * row_bytes(K); }
    // smem: [token rows][ring][barriers, token scales][partial sums][group tables], the first two 1024-aligned
    __host__ __device__ static int ring_offset(int K) { return (b_bytes(K) + 1023) / 1024 * 1024; }
    __host__ __device__ static int smem_bytes(int K, int stages, int G) {
        return 1024 + ring_offset(K) + stages * STAGE_BYTES + FW_BAR_BYTES + RED_BYTES + LUT_BYTES + table_bytes(G);
    }
    static constexpr int MAX_SMEM = 232448;
    // deepest ring (at most 8 stages) that fits beside the token rows
    __host__ __device__ static int stages_for(int K, int G) {
        int s = 8;
        while (s > 0 && smem_bytes(K, s, G) > MAX_SMEM) --s;
        return s;
    }
};

// the four code pairs of a 32-bit word as four f16 pairs (bytes 0..3 in order): the hardware's exact E2M1 -> f16
// conversion, low code to the low half. The bytes come from one unpacking move, which the compiler turns into byte
// selects of the conversions themselves (measured: gate|up 0.806 -> 0.720 ms, down 0.450 -> 0.402 ms on the decode
// layer, against a shift in front of every conversion)
__device__ __forceinline__ void e2m1x8_to_f16x2x4(uint32_t w, uint32_t& o0, uint32_t& o1, uint32_t& o2, uint32_t& o3) {
    asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\tmov.b32 {b0, b1, b2, b3}, %4;\n\t"
        "cvt.rn.f16x2.e2m1x2 %0, b0;\n\tcvt.rn.f16x2.e2m1x2 %1, b1;\n\t"
        "cvt.rn.f16x2.e2m1x2 %2, b2;\n\tcvt.rn.f16x2.e2m1x2 %3, b3;\n\t}"
        : "=r"(o0), "=r"(o1), "=r"(o2), "=r"(o3)
        : "r"(w));
}

__device__ __forceinline__ void mma_f16_m16n8k16(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
        "{%0, %1, %2, %3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

__device__ __forceinline__ uint32_t pack_f16x2(float lo, float hi) {
    __half2 v = __floats2half2_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&v);
}

// E8M0 scale code -> 2^(s - 127) as fp32 (s = 0: 2^-127, the subnormal 0x00400000; every s >= 1 gives bits above it)
__device__ __forceinline__ float e8m0_to_f32(uint32_t s) {
    return __uint_as_float(max(s << 23, 0x00400000u));
}

// 8 bf16 (one 16-byte chunk, elements 0..7 in order) times 2^-e as f16, in the order 0 2 4 6 1 3 5 7
__device__ __forceinline__ uint4 bf16x8_to_f16_permuted(const uint4 v, float inv) {
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
    float f[8];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        f[2 * i] = __uint_as_float(w[i] << 16) * inv;
        f[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u) * inv;
    }
    uint4 o;
    o.x = pack_f16x2(f[0], f[2]);
    o.y = pack_f16x2(f[4], f[6]);
    o.z = pack_f16x2(f[1], f[3]);
    o.w = pack_f16x2(f[5], f[7]);
    return o;
}

template <bool GATEUP>
__global__ void __launch_bounds__(FW_THREADS, 1)
    grouped_gemm_fp4_warp_kernel(const __grid_constant__ CUtensorMap tmX, const __grid_constant__ CUtensorMap tmQ,
                                 const __grid_constant__ CUtensorMap tmS, const GemmArgs args,
                                 int weights_streamed_once, int stages_n) {
    using S = GemmFp4WarpShape<GATEUP>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    const int K = args.K;
    const int row_bytes = S::row_bytes(K);
    uint8_t* brows = smem;                               // [8][row_bytes] token rows
    uint8_t* ring = smem + S::ring_offset(K);
    uint64_t* full_bar = reinterpret_cast<uint64_t*>(ring + stages_n * S::STAGE_BYTES);
    uint64_t* empty_bar = full_bar + 8;
    uint64_t* bfull_bar = empty_bar + 8;
    uint64_t* bempty_bar = bfull_bar + 1;
    uint64_t* bconv_bar = bempty_bar + 1;  // every token row of the segment converted
    uint64_t* red_full = bconv_bar + 1;  // [8] (two warps per rows) partial sums of warp w + RW are in red[w]
    uint64_t* red_empty = red_full + 8;  // [8] red[w] has been read
    volatile int* abort_flag = reinterpret_cast<volatile int*>(red_empty + 8);
    float* tok_scale = reinterpret_cast<float*>(ring + stages_n * S::STAGE_BYTES + 384);  // [8]
    float* red = reinterpret_cast<float*>(ring + stages_n * S::STAGE_BYTES + FW_BAR_BYTES);  // [RW][32][8]
    float* scale_lut = reinterpret_cast<float*>(ring + stages_n * S::STAGE_BYTES + FW_BAR_BYTES + S::RED_BYTES);
    int32_t* s_off =
        reinterpret_cast<int32_t*>(ring + stages_n * S::STAGE_BYTES + FW_BAR_BYTES + S::RED_BYTES + S::LUT_BYTES);
    int32_t* s_tp = s_off + (args.G + 1);  // tables sized by G (table_bytes)

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int G = args.G;
    const int KB32 = K / 32;                    // scale blocks per row
    const int KS = (K + FW_KS - 1) / FW_KS;     // stages per weight block
    const int wblocks = args.n_tiles;           // weight blocks of S::BM output columns

    if (threadIdx.x == 0) {
        for (int s = 0; s < stages_n; ++s) {
            mbar_init(&full_bar[s], 1);
            mbar_init(&empty_bar[s], FW_WARPS);
        }
        mbar_init(bfull_bar, 1);
        mbar_init(bempty_bar, FW_WARPS);
        mbar_init(bconv_bar, FW_WARPS);
        for (int w = 0; w < 8; ++w) {
            mbar_init(&red_full[w], 32);
            mbar_init(&red_empty[w], 32);
        }
        *abort_flag = 0;
        fence_mbar_init();
        tma_prefetch_desc(&tmX);
        tma_prefetch_desc(&tmQ);
        tma_prefetch_desc(&tmS);
    }
    if constexpr (S::SCALE_LUT) {
        for (int i = threadIdx.x; i < 256; i += FW_THREADS) scale_lut[i] = e8m0_to_f32((uint32_t)i);
    }
    grid_dep_wait();
    grid_dep_trigger();
    for (int g = threadIdx.x; g <= G; g += FW_THREADS) {
        int v = args.group_offsets[g];
        if (v < 0 || v > args.M) {
            flag_error(MOE_DEVERR_GROUP_RANGE);
            v = min(max(v, 0), args.M);
        }
        s_off[g] = v;
    }
    __syncthreads();
    if (warp == 0) {  // unit prefix over groups: units(g) = ceil(rows / 8) * wblocks
        const int per = (G + 31) / 32;
        const int g0 = lane * per, g1 = min(g0 + per, G);
        int local = 0;
        for (int g = g0; g < g1; ++g) {
            const int rows = s_off[g + 1] - s_off[g];
            if (rows < 0) flag_error(MOE_DEVERR_GROUP_RANGE);
            local += (max(rows, 0) + FW_NT - 1) / FW_NT * wblocks;
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
            run += (max(s_off[g + 1] - s_off[g], 0) + FW_NT - 1) / FW_NT * wblocks;
        }
        if (lane == 31) s_tp[G] = incl;
    }
    __syncthreads();
    const int total = s_tp[G];
    const int u_begin = (int)((long)total * blockIdx.x / gridDim.x);
    const int u_end = (int)((long)total * (blockIdx.x + 1) / gridDim.x);

    // the segment that starts at unit u: group g, token block tb, weight blocks [wb0, wb1) (up to the end of the
    // token block or of this CTA's range)
    auto segment = [&](int u, int& g, int& tb, int& wb0, int& wb1) {
        int lo = 0, hi = G - 1;
        while (lo < hi) {
            const int mid = (lo + hi + 1) >> 1;
            if (s_tp[mid] <= u)
                lo = mid;
            else
                hi = mid - 1;
        }
        g = lo;
        const int local = u - s_tp[g];
        tb = local / wblocks;
        wb0 = local - tb * wblocks;
        wb1 = min(wblocks, wb0 + (u_end - u));
    };

    if (warp == FW_WARPS) {
        // ---------------- TMA producer ----------------
        const uint64_t pol_x = l2_policy_evict_last();
        const uint64_t pol_w = weights_streamed_once ? l2_policy_evict_first() : l2_policy_evict_normal();
        int stage = 0;
        uint32_t phase = 0, bphase = 0;
        long issued = 0;
        bool ok = true;
        int segs_done = 0;
        int g, tb, wb0, wb1;
        for (int u = u_begin; u < u_end && ok; u += wb1 - wb0) {
            segment(u, g, tb, wb0, wb1);
            const int row0 = s_off[g] + tb * FW_NT;
            // the token rows: after the compute warps are done with the previous segment's
            if (lane == 0) {
                ok = mbar_wait_bounded(bempty_bar, bphase ^ 1u, abort_flag);
                if (ok) {
                    mbar_arrive_expect_tx(bfull_bar, (uint32_t)(FW_NT * K * 2));
                    for (int r = 0; r < FW_NT; ++r)  // rows past M arrive as zeros
                        tma_load_3d(brows + r * row_bytes, &tmX, bfull_bar, 0, 0, row0 + r, pol_x);
                }
            }
            bphase ^= 1u;
            ok = __shfl_sync(0xffffffffu, ok, 0);
            if (!ok) break;
            ++segs_done;  // its token rows are in flight (drained below even if a later wait gives up)
            for (int wb = wb0; wb < wb1 && ok; ++wb) {
                const int wrow = wb * S::BM;
                for (int ks = 0; ks < KS; ++ks) {
                    if (lane == 0) ok = mbar_wait_bounded(&empty_bar[stage], phase ^ 1u, abort_flag);
                    ok = __shfl_sync(0xffffffffu, ok, 0);
                    if (!ok) break;
                    if (lane == 0) {
                        uint8_t* st = ring + stage * S::STAGE_BYTES;
                        const int k0 = ks * FW_KS;
                        mbar_arrive_expect_tx(&full_bar[stage], S::STAGE_BYTES);
                        tma_load_3d(st, &tmQ, &full_bar[stage], k0 / 2, wrow, g, pol_w);
                        tma_load_3d(st + S::BLOCKS * S::Q_BYTES, &tmS, &full_bar[stage], wrow, k0 / 32, g, pol_w);
                        if constexpr (GATEUP) {
                            tma_load_3d(st + S::Q_BYTES, &tmQ, &full_bar[stage], k0 / 2, args.f + wrow, g, pol_w);
                            tma_load_3d(st + S::BLOCKS * S::Q_BYTES + S::S_BYTES, &tmS, &full_bar[stage],
                                        args.f + wrow, k0 / 32, g, pol_w);
                        }
                    }
                    ++issued;
                    if (++stage == stages_n) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
            }
        }
        // copies still in flight land before the CTA leaves (bounded)
        if (lane == 0) {
            for (long n = issued > stages_n ? issued - stages_n : 0; n < issued; ++n)
                mbar_wait_drain(&full_bar[n % stages_n], (uint32_t)((n / stages_n) & 1));
            if (segs_done > 0) mbar_wait_drain(bfull_bar, (uint32_t)((segs_done - 1) & 1));
        }
        __syncwarp();
    } else {
        // ---------------- compute warps 0-15 ----------------
        const int gq = lane >> 2, t = lane & 3;
        const int rw = warp % S::RW, kw = warp / S::RW;  // row group; K part (two per rows: even, odd blocks)
        const int ra = rw * 16 + gq, rb = ra + 8;        // this thread's weight rows within the block
        // byte offsets in a stage's code block of word t of 16-byte unit `kw` of rows ra, rb (128-byte swizzle: unit
        // u of row r sits at u ^ (r % 8)); unit kw + KSPL * i is then offset ^ ((KSPL * i) << 4)
        const uint32_t qa = (uint32_t)(ra * 128 + ((kw ^ (ra & 7)) << 4) + 4 * t);
        const uint32_t qb = (uint32_t)(rb * 128 + ((kw ^ (rb & 7)) << 4) + 4 * t);
        const int nchunk = K / 8;                     // 16-byte chunks of a token row
        const int npairs = 4 * ((nchunk + 7) / 8);    // (chunk, chunk + 4) pairs, per 64 elements
        int stage = 0;
        uint32_t phase = 0, bphase = 0, rphase = 0;
        bool ok = true;
        int g, tb, wb0, wb1;
        for (int u = u_begin; u < u_end && ok; u += wb1 - wb0) {
            segment(u, g, tb, wb0, wb1);
            const int row0 = s_off[g] + tb * FW_NT;
            const int rows = min(FW_NT, s_off[g + 1] - row0);
            if (lane == 0) ok = mbar_wait_bounded(bfull_bar, bphase, abort_flag);
            ok = __shfl_sync(0xffffffffu, ok, 0);
            bphase ^= 1u;
            if (!ok) break;
            if (warp < FW_NT) {  // token row `warp`: largest magnitude, scale exponent, conversion to permuted f16
                uint8_t* row = brows + warp * row_bytes;
                uint32_t mx = 0;
                for (int c = lane; c < nchunk; c += 32) {
                    const uint4 v = *reinterpret_cast<const uint4*>(row + c * 16);
                    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
                    for (int i = 0; i < 4; ++i) mx = max(mx, max(w[i] & 0x7fffu, (w[i] >> 16) & 0x7fffu));
                }
#pragma unroll
                for (int o = 16; o; o >>= 1) mx = max(mx, __shfl_xor_sync(0xffffffffu, mx, o));
                int e = 0;  // the row times 2^-e has its largest magnitude in [16, 32)
                if (mx != 0) {
                    const int ef = (int)(mx >> 7);
                    const int fl = ef ? ef - 127 : (31 - __clz((int)mx)) - 133;  // floor(log2 max)
                    e = max(fl - 4, -126);
                }
                const float inv = __uint_as_float((uint32_t)(127 - e) << 23);  // 2^-e, e in [-126, 123]
                if (lane == 0) tok_scale[warp] = __uint_as_float((uint32_t)(127 + e) << 23);
                // odd rows keep each pair of 32-element blocks swapped (16-byte units u -> u ^ 4), so that the
                // B loads of two neighbouring tokens fall in different banks
                const bool odd = (warp & 1) != 0;
                for (int p = lane; p < npairs; p += 32) {
                    const int c0 = (p >> 2) * 8 + (p & 3), c1 = c0 + 4;
                    const uint4 v0 = *reinterpret_cast<const uint4*>(row + c0 * 16);
                    const uint4 v1 = *reinterpret_cast<const uint4*>(row + c1 * 16);  // padding past K: unused
                    const uint4 o0 = bf16x8_to_f16_permuted(v0, inv), o1 = bf16x8_to_f16_permuted(v1, inv);
                    *reinterpret_cast<uint4*>(row + (odd ? c1 : c0) * 16) = o0;
                    *reinterpret_cast<uint4*>(row + (odd ? c0 : c1) * 16) = o1;
                }
            }
            // every token row converted (a bounded wait on a barrier, not a hardware barrier: a warp that gave up
            // on a wait leaves without blocking the others)
            __syncwarp();
            if (lane == 0) {
                mbar_arrive(bconv_bar);
                ok = mbar_wait_bounded(bconv_bar, bphase ^ 1u, abort_flag);
            }
            ok = __shfl_sync(0xffffffffu, ok, 0);
            if (!ok) break;
            const float tsc0 = tok_scale[2 * t], tsc1 = tok_scale[2 * t + 1];
            // token row gq, unit 4 kb + t of block kb = 8 ks + KSPL i + kw, stored at block kb ^ (gq % 2): with two
            // warps per rows that is 8 ks + 2 i + (kw ^ (gq % 2)); with one, 8 ks + (i ^ (gq % 2)), i.e. +i for even
            // i and i - 2 (gq % 2) for odd i
            const int par = gq & 1;
            const uint8_t* bx0 = brows + gq * row_bytes + (((S::KSPL > 1 ? (kw ^ par) : par) * 4 + t) << 4);
            const uint8_t* bx1 = bx0 - (S::KSPL > 1 ? 0 : 2 * par * 64);  // odd i, one warp per rows
            for (int wb = wb0; wb < wb1 && ok; ++wb) {
                float acc_g[4] = {0.f, 0.f, 0.f, 0.f}, acc_u[4] = {0.f, 0.f, 0.f, 0.f};
                for (int ks = 0; ks < KS; ++ks) {
                    if (lane == 0) ok = mbar_wait_bounded(&full_bar[stage], phase, abort_flag);
                    ok = __shfl_sync(0xffffffffu, ok, 0);
                    if (!ok) break;
                    const uint8_t* st = ring + stage * S::STAGE_BYTES;
                    const uint8_t* sc = st + S::BLOCKS * S::Q_BYTES + kw * S::BM;
                    const int nb = KB32 - ks * (FW_KS / 32);  // blocks of this stage inside K (>= 8: all)
#pragma unroll
                    for (int i = 0; i < FW_KS / 32 / S::KSPL; ++i) {
                        if (S::KSPL * i + kw >= nb) break;
                        const uint8_t* bx = (S::KSPL > 1 || (i & 1) == 0) ? bx0 : bx1;
                        const uint4 xv = *reinterpret_cast<const uint4*>(bx + ks * (FW_KS * 2) + i * (S::KSPL * 64));
#pragma unroll
                        for (int blk = 0; blk < S::BLOCKS; ++blk) {
                            const uint8_t* q = st + blk * S::Q_BYTES;
                            const uint32_t sw = (uint32_t)((S::KSPL * i) << 4);
                            const uint32_t wa = *reinterpret_cast<const uint32_t*>(q + (qa ^ sw));
                            const uint32_t wbv = *reinterpret_cast<const uint32_t*>(q + (qb ^ sw));
                            const uint32_t ca = sc[blk * S::S_BYTES + S::KSPL * i * S::BM + ra];
                            const uint32_t cb = sc[blk * S::S_BYTES + S::KSPL * i * S::BM + rb];
                            const float sa = S::SCALE_LUT ? scale_lut[ca] : e8m0_to_f32(ca);
                            const float sb = S::SCALE_LUT ? scale_lut[cb] : e8m0_to_f32(cb);
                            uint32_t a0[4], a1[4];
                            e2m1x8_to_f16x2x4(wa, a0[0], a0[2], a1[0], a1[2]);
                            e2m1x8_to_f16x2x4(wbv, a0[1], a0[3], a1[1], a1[3]);
                            float d[4] = {0.f, 0.f, 0.f, 0.f};
                            mma_f16_m16n8k16(d, a0, xv.x, xv.y);
                            mma_f16_m16n8k16(d, a1, xv.z, xv.w);
                            float* acc = blk == 0 ? acc_g : acc_u;
                            acc[0] = fmaf(d[0], sa, acc[0]);
                            acc[1] = fmaf(d[1], sa, acc[1]);
                            acc[2] = fmaf(d[2], sb, acc[2]);
                            acc[3] = fmaf(d[3], sb, acc[3]);
                        }
                    }
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&empty_bar[stage]);
                    if (++stage == stages_n) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
                if (!ok) break;
                if constexpr (S::KSPL > 1) {
                    float4* slot = reinterpret_cast<float4*>(red + (rw * 32 + lane) * 8);
                    if (kw == 1) {  // partial sums of the odd blocks to warp rw
                        ok = mbar_wait_bounded(&red_empty[rw], rphase ^ 1u, abort_flag);
                        ok = __all_sync(0xffffffffu, ok);
                        if (!ok) break;
                        slot[0] = make_float4(acc_g[0], acc_g[1], acc_g[2], acc_g[3]);
                        slot[1] = make_float4(acc_u[0], acc_u[1], acc_u[2], acc_u[3]);
                        mbar_arrive(&red_full[rw]);
                        rphase ^= 1u;
                        continue;
                    }
                    ok = mbar_wait_bounded(&red_full[rw], rphase, abort_flag);
                    ok = __all_sync(0xffffffffu, ok);
                    if (!ok) break;
                    const float4 og = slot[0], ou = slot[1];
                    mbar_arrive(&red_empty[rw]);
                    rphase ^= 1u;
                    acc_g[0] += og.x;
                    acc_g[1] += og.y;
                    acc_g[2] += og.z;
                    acc_g[3] += og.w;
                    acc_u[0] += ou.x;
                    acc_u[1] += ou.y;
                    acc_u[2] += ou.z;
                    acc_u[3] += ou.w;
                }
                // outputs: weight rows ra, rb (output columns) x tokens 2t, 2t+1
                const int ca = wb * S::BM + ra, cb = wb * S::BM + rb;
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    const int tok = 2 * t + (j & 1);
                    const int col = (j < 2) ? ca : cb;
                    if (tok >= rows || col >= args.n_out) continue;
                    const float ts = (j & 1) ? tsc1 : tsc0;
                    const float v = GATEUP ? swiglu(acc_g[j] * ts, acc_u[j] * ts) : acc_g[j] * ts;
                    args.out[(size_t)(row0 + tok) * args.n_out + col] = __float2bfloat16_rn(v);
                }
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(bempty_bar);  // this warp is done with the token rows
        }
    }
    __syncthreads();
}

}  // namespace moe
