// MXFP4 expert weights: the encoder, and the grouped GEMMs that stream 4-bit weights for a few rows per expert.
//
// The blog post "Mixture of Experts (MoEs) in Transformers" (section "From Dense to Sparse: What Are MoEs?")
// estimates generation speed as memory bandwidth over the bytes of the active parameters, and notes that
// kernels for gpt-oss's native mxfp4 quantization would be faster still. Decode is that case: each expert sees a
// handful of rows, so the layer time is the time to stream its weights. MXFP4 (OCP Microscaling Formats v1.0)
// stores a weight in 4 bits plus an 8-bit scale per 32, 4.25 bits instead of bf16's 16.
//
// Format (the library's layout; the specification fixes the encoding, not the memory order):
//   codes  [G][N][K/2] bytes: each little-endian 32-bit word holds 8 consecutive elements of a row, nibble i
//          (bits 4i..4i+3) being element 2i for i < 4 and element 2(i-4)+1 for i >= 4: even elements in the low
//          half, odd elements in the high half. A code is E2M1: sign, two exponent bits (bias 1), one mantissa bit.
//   scales [G][K/32][N] bytes, E8M0: the block of 32 elements of row n starting at 32b has scale 2^(s - 127).
//
// The GEMM keeps the activations in bf16 and the arithmetic of the bf16 path (bf16 products, fp32
// accumulation): the weights are decoded on the fly, exactly, into bf16.
//
// Layout of the computation ("swap AB"): the weight rows are the MMA's M dimension (128 per accumulator, one
// per TMEM lane) and the group's rows are its N dimension (NT = 16, 32 or 64 per tile). A decode group of two
// rows then costs an N = 16 MMA instead of a 128-row tile that is 98% padding. The decoded weights go straight
// from registers into tensor memory (tcgen05.st) and the MMA reads its A operand from there, so shared memory
// only carries the 4-bit codes, the scales and the small activation tile: decoding does not compete with the
// MMA for shared-memory bandwidth.
//
// CTA organisation (448 threads, one CTA per SM, persistent over tiles):
//   warp 0      TMA producer: per stage (K = 256) the codes [128 rows x 128 bytes] of the tile's weight block(s)
//               (SWIZZLE_128B), their scales [8 x 128], and the activation rows [NT x 256] as 4 boxes
//   warp 1      TMEM allocator and MMA issuer: tcgen05.mma M=128 N=NT K=16 with A from TMEM
//   warps 2-9   decoders: two groups of four warps, each thread one TMEM lane (one weight row). For gate|up,
//               group 0 decodes the gate rows and group 1 the matching up rows; for down, the two groups take
//               alternate 64-element halves of each 128-element slot. A slot (64 TMEM columns) is filled with
//               tcgen05.st and handed to the MMA warp through afull[slot]; the MMA's commit frees it.
//   warps 10-13 epilogue: tcgen05.ld of the accumulator(s), silu(gate) * up or the plain sum, bf16 stores
//               masked to the group's rows and the output columns
// Tiles are numbered group-major, then weight block, then token block, so token blocks of one weight block run
// side by side and share its codes in L2. Every wait is bounded as in the bf16 grouped GEMM.
#pragma once
#include "common.cuh"
#include "gemm.cuh"

namespace moe {

// ---- encoder ------------------------------------------------------------------------------------------

// E2M1 magnitude code of p = |v| / scale (0 <= p < 8): round to the nearest of 0, 0.5, 1, 1.5, 2, 3, 4, 6, a tie
// going to the value whose mantissa bit is 0, and p above 6 clamped to 6. The code counts the rounding
// thresholds (midpoints) that p passes; at a midpoint whose upper neighbour has mantissa bit 0 the comparison
// is >=, otherwise >.
__device__ __forceinline__ uint32_t e2m1_code_of(float p) {
    return (uint32_t)(p > 0.25f) + (uint32_t)(p >= 0.75f) + (uint32_t)(p > 1.25f) + (uint32_t)(p >= 1.75f) +
           (uint32_t)(p > 2.5f) + (uint32_t)(p >= 3.5f) + (uint32_t)(p > 5.0f);
}

// One thread per block of 32 weights (row-major, blocks of a row consecutive): 64 bytes in, 16 bytes of codes
// and one scale byte out. Scale = 2^(floor(log2 max|v|) - 2), the exponent of the block's largest magnitude
// minus that of E2M1's largest value (6 = 1.5 * 2^2), clamped to the E8M0 range; an all-zero block gets code 0.
__global__ void __launch_bounds__(256) mxfp4_quantize_kernel(const __nv_bfloat16* __restrict__ w, long rows, int N,
                                                           int K, uint8_t* __restrict__ q, uint8_t* __restrict__ s) {
    grid_dep_wait();
    grid_dep_trigger();
    const int nb = K / 32;
    const long total = rows * nb;
    for (long i = (long)blockIdx.x * blockDim.x + threadIdx.x; i < total; i += (long)gridDim.x * blockDim.x) {
        const long row = i / nb;
        const int b = (int)(i - row * nb);
        const uint4* src = reinterpret_cast<const uint4*>(w + row * K + (long)b * 32);
        uint32_t v[16];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const uint4 u = src[j];
            v[4 * j] = u.x;
            v[4 * j + 1] = u.y;
            v[4 * j + 2] = u.z;
            v[4 * j + 3] = u.w;
        }
        // for finite bf16, |a| <= |b| exactly when (a & 0x7fff) <= (b & 0x7fff)
        uint32_t amax = 0;
#pragma unroll
        for (int j = 0; j < 16; ++j) amax = max(amax, max(v[j] & 0x7fffu, (v[j] >> 16) & 0x7fffu));
        int shared = -127;
        if (amax != 0) {
            const int ef = (int)(amax >> 7);
            const int fl = ef ? ef - 127 : (31 - __clz((int)amax)) - 133;  // floor(log2 max|v|); subnormal: m * 2^-133
            shared = min(max(fl - 2, -127), 127);
        }
        // |v| / 2^shared by a power-of-two multiply: shared <= 125 for finite bf16, so the factor is a normal float
        const float inv = __int_as_float((127 - shared) << 23);
        uint32_t word[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            uint32_t wd = 0;
#pragma unroll
            for (int i2 = 0; i2 < 4; ++i2) {
                const uint32_t pr = v[4 * j + i2];  // elements 8j + 2*i2 (low half) and 8j + 2*i2 + 1 (high half)
                const uint32_t lo = pr & 0xffffu, hi = pr >> 16;
                const uint32_t clo = e2m1_code_of(__uint_as_float((lo & 0x7fffu) << 16) * inv) | ((lo >> 12) & 8u);
                const uint32_t chi = e2m1_code_of(__uint_as_float((hi & 0x7fffu) << 16) * inv) | ((hi >> 12) & 8u);
                wd |= clo << (4 * i2);
                wd |= chi << (16 + 4 * i2);
            }
            word[j] = wd;
        }
        *reinterpret_cast<uint4*>(q + row * (K / 2) + (long)b * 16) = make_uint4(word[0], word[1], word[2], word[3]);
        const long g = row / N, n = row - g * N;
        s[(g * nb + b) * (long)N + n] = (uint8_t)(shared + 127);
    }
}

// ---- decoder ------------------------------------------------------------------------------------------

__device__ __forceinline__ uint32_t bf16x2_mul(uint32_t a, uint32_t b) {
    uint32_t d;
    asm("mul.rn.bf16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
    return d;
}

// bf16x2 holding 2^e in both halves, e in [-126, 127]
__device__ __forceinline__ uint32_t bf16x2_pow2(int e) {
    const uint32_t h = (uint32_t)(e + 127) << 7;
    return h | (h << 16);
}

// 32 codes (one 16-byte unit of the layout: elements 0..31 of a block) with scale code sc -> 16 bf16x2 words in
// K order. An E2M1 code's magnitude bits e1 e0 m placed at bf16 bits 8..6 (exponent field e1e0, mantissa top
// bit m) and its sign at bit 15 form a bf16 whose value is the code's value times 2^-126 (the exponent bias
// 127 against E2M1's 1; exponent field 0 is the subnormal 0 or 2^-127, i.e. 0 or 0.5 * 2^-126). One multiply by
// 2^(126 + sc - 127) = 2^(sc - 1) then gives the weight exactly; for sc > 128 that factor is not a bf16 number
// and the multiply is split in two. The word layout puts element 2i in nibble i and element 2i+1 in nibble
// i+4, so the pair (2i, 2i+1) needs the same shift for both halves of the output word.
__device__ __forceinline__ void mxfp4_decode_patterns(const uint4 c, uint32_t* out) {
    constexpr uint32_t MAG = 0x01C001C0u, SGN = 0x80008000u;
    const uint32_t xs[4] = {c.x, c.y, c.z, c.w};
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        const uint32_t x = xs[j];
        out[4 * j + 0] = ((x << 6) & MAG) | ((x << 12) & SGN);
        out[4 * j + 1] = ((x << 2) & MAG) | ((x << 8) & SGN);
        out[4 * j + 2] = ((x >> 2) & MAG) | ((x << 4) & SGN);
        out[4 * j + 3] = ((x >> 6) & MAG) | (x & SGN);
    }
}

__device__ __forceinline__ void mxfp4_decode_unit(const uint4 c, int sc, uint32_t* out) {
    mxfp4_decode_patterns(c, out);
    if (sc <= 128) {  // one branch per 32 weights, uniform across the warp for realistic scales
        const uint32_t f1 = bf16x2_pow2(sc - 1);
#pragma unroll
        for (int i = 0; i < 16; ++i) out[i] = bf16x2_mul(out[i], f1);
    } else {
        const uint32_t f1 = bf16x2_pow2(126), f2 = bf16x2_pow2(sc - 127);
#pragma unroll
        for (int i = 0; i < 16; ++i) out[i] = bf16x2_mul(bf16x2_mul(out[i], f1), f2);
    }
}

// ---- grouped GEMM -------------------------------------------------------------------------------------

constexpr int GF_BM = 128;          // weight rows per block (TMEM lanes)
constexpr int GF_KS = 256;          // K per shared-memory stage: 128 bytes of codes per row
constexpr int GF_THREADS = 448;     // 14 warps
constexpr int GF_SLOTS = 4;         // A-operand slots in TMEM columns [0, 256)
constexpr int GF_SLOT_COLS = 64;    // columns per slot: 128 K of bf16
constexpr int GF_ACC_BASE = 256;    // accumulators in TMEM columns [256, 512)
constexpr int GF_ACC_COLS = 256;
constexpr int GF_TMEM_COLS = 512;

template <int NT, bool GATEUP>
struct GemmFp4Shape {
    static_assert(NT == 16 || NT == 32 || NT == 64, "token tile: UMMA N for M = 128, 16 columns per epilogue load");
    static constexpr int BLOCKS = GATEUP ? 2 : 1;             // weight row blocks per tile (gate, up)
    static constexpr int Q_BYTES = GF_BM * (GF_KS / 2);       // codes of one block
    static constexpr int S_BYTES = (GF_KS / 32) * GF_BM;      // scales of one block
    static constexpr int XBOX_BYTES = NT * 128;               // {64 K, NT rows} of bf16
    static constexpr int X_BYTES = (GF_KS / 64) * XBOX_BYTES;
    static constexpr int STAGE_BYTES = BLOCKS * Q_BYTES + X_BYTES + BLOCKS * S_BYTES;
    static_assert(STAGE_BYTES % 1024 == 0 && XBOX_BYTES % 1024 == 0, "swizzled boxes start on 1024-byte atoms");
    static constexpr int SLOTS_PER_STAGE = GATEUP ? 4 : 2;    // a slot holds 64 K of gate and up, or 128 K
    static constexpr int ACC_COLS = GATEUP ? 2 * NT : NT;     // one accumulator buffer
    static_assert(2 * ACC_COLS <= GF_ACC_COLS, "two accumulator buffers above the slots");
    static constexpr int BAR_BYTES = 256;
    static constexpr int TABLE_BYTES = (2 * (GG_MAX_GROUPS + 1) * 4 + 127) / 128 * 128;
    static constexpr int FIXED = 1024 + BAR_BYTES + TABLE_BYTES;
    static constexpr int STAGES_FIT = (232448 - FIXED) / STAGE_BYTES;
    static constexpr int STAGES = STAGES_FIT > 8 ? 8 : STAGES_FIT;
    static_assert(STAGES >= 2, "pipeline depth");
    static constexpr int SMEM_BYTES = FIXED + STAGES * STAGE_BYTES;
    static_assert((2 * STAGES + 2 * GF_SLOTS + 5) * 8 + 8 <= BAR_BYTES, "barrier area");
};

template <int NT, bool GATEUP>
__global__ void __launch_bounds__(GF_THREADS, 1)
    grouped_gemm_fp4_kernel(const __grid_constant__ CUtensorMap tmX, const __grid_constant__ CUtensorMap tmQ,
                            const __grid_constant__ CUtensorMap tmS, const GemmArgs args, int weights_streamed_once) {
    using S = GemmFp4Shape<NT, GATEUP>;
    constexpr int STAGES = S::STAGES;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    uint8_t* stages = smem;
    uint64_t* full_bar = reinterpret_cast<uint64_t*>(smem + STAGES * S::STAGE_BYTES);
    uint64_t* empty_bar = full_bar + STAGES;
    uint64_t* afull_bar = empty_bar + STAGES;
    uint64_t* aempty_bar = afull_bar + GF_SLOTS;
    uint64_t* tfull_bar = aempty_bar + GF_SLOTS;
    uint64_t* tempty_bar = tfull_bar + 2;
    uint64_t* final_bar = tempty_bar + 2;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(final_bar + 1);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
    int32_t* s_off = reinterpret_cast<int32_t*>(smem + STAGES * S::STAGE_BYTES + S::BAR_BYTES);
    int32_t* s_tp = s_off + (GG_MAX_GROUPS + 1);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int G = args.G;
    const int KS = (args.K + GF_KS - 1) / GF_KS;

    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(&full_bar[s], 1);
            mbar_init(&empty_bar[s], 9);  // the 8 decoder warps and the MMA warp's commit (activations)
        }
        for (int s = 0; s < GF_SLOTS; ++s) {
            mbar_init(&afull_bar[s], 8);
            mbar_init(&aempty_bar[s], 1);
        }
        for (int a = 0; a < 2; ++a) {
            mbar_init(&tfull_bar[a], 1);
            mbar_init(&tempty_bar[a], 4);
        }
        mbar_init(final_bar, 1);
        *abort_flag = 0;
        fence_mbar_init();
        tma_prefetch_desc(&tmX);
        tma_prefetch_desc(&tmQ);
        tma_prefetch_desc(&tmS);
    }
    if (warp == 1) {
        tmem_alloc(tmem_slot, GF_TMEM_COLS);
        tmem_relinquish();
    }
    grid_dep_wait();
    grid_dep_trigger();
    for (int g = threadIdx.x; g <= G; g += GF_THREADS) {
        int v = args.group_offsets[g];
        if (v < 0 || v > args.M) {
            flag_error(MOE_DEVERR_GROUP_RANGE);
            v = min(max(v, 0), args.M);
        }
        s_off[g] = v;
    }
    __syncthreads();
    if (warp == 0) {  // tile prefix over groups: tiles(g) = ceil(rows / NT) * n_tiles
        const int per = (G + 31) / 32;
        const int g0 = lane * per, g1 = min(g0 + per, G);
        int local = 0;
        for (int g = g0; g < g1; ++g) {
            const int rows = s_off[g + 1] - s_off[g];
            if (rows < 0) flag_error(MOE_DEVERR_GROUP_RANGE);
            local += (max(rows, 0) + NT - 1) / NT * args.n_tiles;
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
            run += (max(s_off[g + 1] - s_off[g], 0) + NT - 1) / NT * args.n_tiles;
        }
        if (lane == 31) s_tp[G] = incl;
    }
    tc_fence_before_sync();
    __syncthreads();
    tc_fence_after_sync();
    const uint32_t tmem_base = *tmem_slot;
    const int total = s_tp[G];

    // tile -> (group, weight block, token block)
    auto locate = [&](int tile, int& g, int& wb, int& tb) {
        int lo = 0, hi = G - 1;
        while (lo < hi) {
            const int mid = (lo + hi + 1) >> 1;
            if (s_tp[mid] <= tile)
                lo = mid;
            else
                hi = mid - 1;
        }
        g = lo;
        const int mt = (max(s_off[g + 1] - s_off[g], 0) + NT - 1) / NT;
        const int local = tile - s_tp[g];
        wb = local / mt;
        tb = local - wb * mt;
    };

    if (warp == 0) {
        // ---------------- TMA producer ----------------
        const uint64_t pol_x = l2_policy_evict_last();
        const uint64_t pol_w = weights_streamed_once ? l2_policy_evict_first() : l2_policy_evict_normal();
        int stage = 0;
        uint32_t phase = 0;
        long issued = 0;
        bool ok = true;
        for (int tile = blockIdx.x; tile < total && ok; tile += gridDim.x) {
            int g, wb, tb;
            locate(tile, g, wb, tb);
            const int row0 = s_off[g] + tb * NT;
            const int wrow = wb * GF_BM;
            for (int ks = 0; ks < KS; ++ks) {
                if (lane == 0) ok = mbar_wait_backoff(&empty_bar[stage], phase ^ 1u, abort_flag, 64);
                ok = __shfl_sync(0xffffffffu, ok, 0);
                if (!ok) break;
                if (lane == 0) {
                    uint8_t* st = stages + stage * S::STAGE_BYTES;
                    uint8_t* sx = st + S::BLOCKS * S::Q_BYTES;
                    uint8_t* ss = sx + S::X_BYTES;
                    const int k0 = ks * GF_KS;
                    mbar_arrive_expect_tx(&full_bar[stage], S::STAGE_BYTES);
                    tma_load_3d(st, &tmQ, &full_bar[stage], k0 / 2, wrow, g, pol_w);
                    tma_load_3d(ss, &tmS, &full_bar[stage], wrow, k0 / 32, g, pol_w);
                    if constexpr (GATEUP) {
                        tma_load_3d(st + S::Q_BYTES, &tmQ, &full_bar[stage], k0 / 2, args.f + wrow, g, pol_w);
                        tma_load_3d(ss + S::S_BYTES, &tmS, &full_bar[stage], args.f + wrow, k0 / 32, g, pol_w);
                    }
#pragma unroll
                    for (int i = 0; i < GF_KS / 64; ++i)
                        tma_load_2d(sx + i * S::XBOX_BYTES, &tmX, &full_bar[stage], k0 + 64 * i, row0, pol_x);
                }
                ++issued;
                if (++stage == STAGES) {
                    stage = 0;
                    phase ^= 1u;
                }
            }
        }
        if (lane == 0) {
            for (long n = issued > STAGES ? issued - STAGES : 0; n < issued; ++n)
                mbar_wait_drain(&full_bar[n % STAGES], (uint32_t)((n / STAGES) & 1));
        }
        __syncwarp();
    } else if (warp == 1) {
        // ---------------- MMA issuer ----------------
        constexpr uint32_t IDESC = idesc_bf16_f32(GF_BM, NT);
        int stage = 0, slot = 0, acc = 0;
        uint32_t phase = 0, slot_phase = 0, acc_phase = 0;
        bool ok = true;
        for (int tile = blockIdx.x; tile < total && ok; tile += gridDim.x) {
            if (lane == 0) ok = mbar_wait_backoff(&tempty_bar[acc], acc_phase ^ 1u, abort_flag, 64);
            ok = __shfl_sync(0xffffffffu, ok, 0);
            if (!ok) break;
            tc_fence_after_sync();
            const uint32_t d0 = tmem_base + (uint32_t)(GF_ACC_BASE + acc * S::ACC_COLS);  // gate, or the output
            const uint32_t d1 = d0 + NT;                                      // up (gate|up)
            for (int ks = 0; ks < KS && ok; ++ks) {
                if (lane == 0) ok = mbar_wait_bounded(&full_bar[stage], phase, abort_flag);
                ok = __shfl_sync(0xffffffffu, ok, 0);
                if (!ok) break;
                tc_fence_after_sync();
                const uint32_t sx = smem_u32(stages + stage * S::STAGE_BYTES + S::BLOCKS * S::Q_BYTES);
                for (int j = 0; j < S::SLOTS_PER_STAGE; ++j) {
                    if (lane == 0) ok = mbar_wait_bounded(&afull_bar[slot], slot_phase, abort_flag);
                    ok = __shfl_sync(0xffffffffu, ok, 0);
                    if (!ok) break;
                    tc_fence_after_sync();
                    if (lane == 0) {
                        const uint32_t a = tmem_base + (uint32_t)(slot * GF_SLOT_COLS);
                        if constexpr (GATEUP) {
#pragma unroll
                            for (int t = 0; t < 4; ++t) {  // K = 64j + 16t of the stage: box j, +32 bytes per t
                                const uint64_t bd = smem_desc_sw128(sx + j * S::XBOX_BYTES) + 2 * t;
                                const uint32_t accf = (ks | j | t) != 0 ? 1u : 0u;
                                umma_bf16_ts(d0, a + 8 * t, bd, IDESC, accf);
                                umma_bf16_ts(d1, a + 32 + 8 * t, bd, IDESC, accf);
                            }
                        } else {
#pragma unroll
                            for (int t = 0; t < 8; ++t) {  // K = 128j + 16t: box 2j + t/4
                                const uint64_t bd = smem_desc_sw128(sx + (2 * j + (t >> 2)) * S::XBOX_BYTES) + 2 * (t & 3);
                                umma_bf16_ts(d0, a + 8 * t, bd, IDESC, (ks | j | t) != 0 ? 1u : 0u);
                            }
                        }
                        umma_commit(&aempty_bar[slot]);
                    }
                    __syncwarp();
                    if (++slot == GF_SLOTS) {
                        slot = 0;
                        slot_phase ^= 1u;
                    }
                }
                if (!ok) break;
                if (lane == 0) umma_commit(&empty_bar[stage]);
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
        if (lane == 0) umma_commit(final_bar);
        __syncwarp();
    } else if (warp < 10) {
        // ---------------- decoders (warps 2-9) ----------------
        const int grp = (warp - 2) >> 2;  // 0: warps 2-5, 1: warps 6-9
        const int q = warp & 3;           // TMEM lanes 32q .. 32q+31
        const int r = q * 32 + lane;      // weight row within the block
        const int blk = GATEUP ? grp : 0;
        const uint32_t t_lane = tmem_base + ((uint32_t)(q * 32) << 16) + (uint32_t)(grp * 32);
        int stage = 0, slot = 0;
        uint32_t phase = 0, slot_phase = 0;
        bool ok = true;
        for (int tile = blockIdx.x; tile < total && ok; tile += gridDim.x) {
            for (int ks = 0; ks < KS && ok; ++ks) {
                if (lane == 0) ok = mbar_wait_bounded(&full_bar[stage], phase, abort_flag);
                ok = __shfl_sync(0xffffffffu, ok, 0);
                if (!ok) break;
                const uint8_t* st = stages + stage * S::STAGE_BYTES;
                const uint8_t* qrow = st + blk * S::Q_BYTES + r * 128;
                const uint8_t* srow = st + S::BLOCKS * S::Q_BYTES + S::X_BYTES + blk * S::S_BYTES + r;
                for (int j = 0; j < S::SLOTS_PER_STAGE; ++j) {
                    const int ch = GATEUP ? j : 2 * j + grp;  // 64-element chunk of the stage: units 2ch, 2ch+1
                    const uint4 c0 = *reinterpret_cast<const uint4*>(qrow + (((2 * ch) ^ (r & 7)) << 4));
                    const uint4 c1 = *reinterpret_cast<const uint4*>(qrow + (((2 * ch + 1) ^ (r & 7)) << 4));
                    const int s0 = srow[(2 * ch) * GF_BM], s1 = srow[(2 * ch + 1) * GF_BM];
                    uint32_t a[32];
                    mxfp4_decode_unit(c0, s0, a);
                    mxfp4_decode_unit(c1, s1, a + 16);
                    if (lane == 0) ok = mbar_wait_bounded(&aempty_bar[slot], slot_phase ^ 1u, abort_flag);
                    ok = __shfl_sync(0xffffffffu, ok, 0);
                    if (!ok) break;
                    tc_fence_after_sync();
                    tmem_store_32cols(t_lane + (uint32_t)(slot * GF_SLOT_COLS), a);
                    tmem_wait_st();
                    tc_fence_before_sync();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&afull_bar[slot]);
                    if (++slot == GF_SLOTS) {
                        slot = 0;
                        slot_phase ^= 1u;
                    }
                }
                if (!ok) break;
                __syncwarp();
                if (lane == 0) mbar_arrive(&empty_bar[stage]);
                if (++stage == STAGES) {
                    stage = 0;
                    phase ^= 1u;
                }
            }
        }
    } else {
        // ---------------- epilogue (warps 10-13) ----------------
        const int q = warp & 3;
        const int r = q * 32 + lane;
        int acc = 0;
        uint32_t acc_phase = 0;
        bool ok = true;
        for (int tile = blockIdx.x; tile < total; tile += gridDim.x) {
            int g, wb, tb;
            locate(tile, g, wb, tb);
            const int row0 = s_off[g] + tb * NT;
            const int rows = min(NT, s_off[g + 1] - row0);
            const int n = wb * GF_BM + r;  // output column of this thread
            if (lane == 0) ok = mbar_wait_backoff(&tfull_bar[acc], acc_phase, abort_flag, 256);
            ok = __shfl_sync(0xffffffffu, ok, 0);
            if (!ok) break;
            tc_fence_after_sync();
            const uint32_t t0 = tmem_base + ((uint32_t)(q * 32) << 16) + (uint32_t)(GF_ACC_BASE + acc * S::ACC_COLS);
            const bool col_ok = n < args.n_out;
#pragma unroll
            for (int c = 0; c < NT / 16; ++c) {
                uint32_t v[16];
                tmem_load_16cols(t0 + 16 * c, v);
                if constexpr (GATEUP) {
                    uint32_t u[16];
                    tmem_load_16cols(t0 + NT + 16 * c, u);
#pragma unroll
                    for (int i = 0; i < 16; ++i) {
                        const int jrow = 16 * c + i;
                        if (col_ok && jrow < rows)
                            args.out[(size_t)(row0 + jrow) * args.n_out + n] =
                                __float2bfloat16_rn(swiglu(__uint_as_float(v[i]), __uint_as_float(u[i])));
                    }
                } else {
#pragma unroll
                    for (int i = 0; i < 16; ++i) {
                        const int jrow = 16 * c + i;
                        if (col_ok && jrow < rows)
                            args.out[(size_t)(row0 + jrow) * args.n_out + n] = __float2bfloat16_rn(__uint_as_float(v[i]));
                    }
                }
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
        tmem_dealloc(tmem_base, GF_TMEM_COLS);
    }
}

}  // namespace moe
