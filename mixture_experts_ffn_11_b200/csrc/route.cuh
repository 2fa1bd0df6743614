// Router: fp32 logits x . W_r^T (+bias) and top-k selection with routing weights.
// Blog post "Mixture of Experts (MoEs) in Transformers", section "From Dense to Sparse": for each
// token a router selects a small subset of experts from the token's hidden representation.
#pragma once
#include "common.cuh"

namespace moe {

// ---- logits: a small fp32 GEMM [T,d] x [d,E] -----------------------------------------------------
// Tile: 64 tokens x 32 experts per block of 128 threads, K chunks of 32. Each thread owns a 4x4 block
// of outputs. x rows (bf16) and W_r rows (fp32) are both K-contiguous; they are transposed into
// shared memory so the inner loop is an outer product of two float4 vectors.
constexpr int RT_TOK = 64, RT_EXP = 32, RT_K = 32, RT_THREADS = 128;

__global__ void __launch_bounds__(RT_THREADS) router_logits_kernel(const __nv_bfloat16* __restrict__ x,
                                                                   const float* __restrict__ w_router,
                                                                   const float* __restrict__ bias, int T, int d,
                                                                   int E, float* __restrict__ logits) {
    __shared__ __align__(16) float xs[RT_K][RT_TOK + 4];
    __shared__ __align__(16) float ws[RT_K][RT_EXP + 4];
    grid_dep_wait();
    grid_dep_trigger();
    const int t0 = blockIdx.x * RT_TOK, e0 = blockIdx.y * RT_EXP;
    const int tid = threadIdx.x;
    const int ty = tid / 8, tx = tid % 8;  // 16 x 8 threads, 4 tokens x 4 experts each
    float acc[4][4];
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = 0.f;

    for (int k0 = 0; k0 < d; k0 += RT_K) {
        // x tile: 64 rows x 32 bf16 = 256 vectors of 8 elements (d is a multiple of 8)
        for (int i = tid; i < RT_TOK * RT_K / 8; i += RT_THREADS) {
            const int row = i / (RT_K / 8), kc = (i % (RT_K / 8)) * 8;
            const int t = t0 + row;
            uint4 v = make_uint4(0, 0, 0, 0);
            if (t < T && k0 + kc < d) v = *reinterpret_cast<const uint4*>(x + (size_t)t * d + k0 + kc);
            const uint32_t u[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                float2 f = unpack_bf16x2(u[j]);
                xs[kc + 2 * j][row] = f.x;
                xs[kc + 2 * j + 1][row] = f.y;
            }
        }
        // W_r tile: 32 rows x 32 fp32 = 256 float4
        for (int i = tid; i < RT_EXP * RT_K / 4; i += RT_THREADS) {
            const int row = i / (RT_K / 4), kc = (i % (RT_K / 4)) * 4;
            const int e = e0 + row;
            float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
            if (e < E && k0 + kc < d) v = *reinterpret_cast<const float4*>(w_router + (size_t)e * d + k0 + kc);
            ws[kc + 0][row] = v.x;
            ws[kc + 1][row] = v.y;
            ws[kc + 2][row] = v.z;
            ws[kc + 3][row] = v.w;
        }
        __syncthreads();
#pragma unroll 8
        for (int kk = 0; kk < RT_K; ++kk) {
            const float4 a = *reinterpret_cast<const float4*>(&xs[kk][ty * 4]);
            const float4 b = *reinterpret_cast<const float4*>(&ws[kk][tx * 4]);
            const float av[4] = {a.x, a.y, a.z, a.w}, bv[4] = {b.x, b.y, b.z, b.w};
#pragma unroll
            for (int i = 0; i < 4; ++i)
#pragma unroll
                for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(av[i], bv[j], acc[i][j]);
        }
        __syncthreads();
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const int t = t0 + ty * 4 + i;
        if (t >= T) continue;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int e = e0 + tx * 4 + j;
            if (e < E) logits[(size_t)t * E + e] = acc[i][j] + (bias ? bias[e] : 0.f);
        }
    }
}

// ---- top-k selection + weights: one warp per token ------------------------------------------------
// Lane l owns experts l, l+32, ... (E <= 1024, so at most 32 each, tracked by a bitmask). k rounds of
// a warp arg-max: the larger logit wins, equal logits go to the lower expert id, which is exactly the
// order "descending logit, lower id first". Lane j keeps the j-th selection (k <= 32).
struct Cand {
    float v;
    int e;  // INT_MAX when the lane has nothing left
};

__device__ __forceinline__ bool cand_better(const Cand& a, const Cand& b) {
    if (a.e == INT_MAX) return false;
    if (b.e == INT_MAX) return true;
    return a.v > b.v || (a.v == b.v && a.e < b.e);
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

// One warp routes one token: selects its k largest logits (descending; equal values keep the lower expert id
// first) and computes the routing weights of `mode`. get(e) returns logit e; lane j < k writes slot j of
// idx_row / w_row. k <= 32.
template <class Get>
__device__ __forceinline__ void warp_route_select(Get get, int E, int k, int mode, int32_t* __restrict__ idx_row,
                                                  float* __restrict__ w_row) {
    const int lane = threadIdx.x & 31;
    const int per = (E + 31) / 32;
    // E <= 256: the token's logits stay in registers (8 per lane) across the k rounds
    constexpr int RPER = 8;
    float rv[RPER];
    if (per <= RPER) {
#pragma unroll
        for (int s = 0; s < RPER; ++s) {
            const int e = s * 32 + lane;
            rv[s] = (s < per && e < E) ? get(e) : 0.f;
        }
    }
    uint32_t taken = 0;
    float my_v = 0.f;
    int my_e = -1;
    for (int j = 0; j < k; ++j) {
        Cand c{0.f, INT_MAX};
        if (per <= RPER) {
#pragma unroll
            for (int s = 0; s < RPER; ++s) {
                const int e = s * 32 + lane;
                if (s >= per || e >= E || (taken >> s) & 1u) continue;
                if (c.e == INT_MAX || rv[s] > c.v) c = Cand{rv[s], e};  // ascending e: strict '>' keeps the lower id
            }
        } else {
            for (int s = 0; s < per; ++s) {
                const int e = s * 32 + lane;
                if (e >= E || (taken >> s) & 1u) continue;
                const float v = get(e);
                if (c.e == INT_MAX || v > c.v) c = Cand{v, e};
            }
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            Cand other{__shfl_xor_sync(0xffffffffu, c.v, o), __shfl_xor_sync(0xffffffffu, c.e, o)};
            if (cand_better(other, c)) c = other;
        }
        // every lane now holds the same winner
        if ((c.e & 31) == lane) taken |= 1u << (c.e >> 5);
        if (lane == j) {
            my_v = c.v;
            my_e = c.e;
        }
    }
    const bool mine = lane < k;
    const float vmax = __shfl_sync(0xffffffffu, my_v, 0);
    float w = 0.f;
    if (mode == MOE_ROUTE_SIGMOID_TOPK_NORM) {
        const float s = mine ? 1.f / (1.f + expf(-my_v)) : 0.f;
        w = s / warp_sum(s);
    } else {
        const float ex = mine ? expf(my_v - vmax) : 0.f;
        const float zsel = warp_sum(ex);
        if (mode == MOE_ROUTE_SOFTMAX_TOPK_RENORM) {
            float part = 0.f;
            for (int s = 0; s < per; ++s) {
                const int e = s * 32 + lane;
                if (e < E) part += expf(get(e) - vmax);
            }
            const float zall = warp_sum(part);
            const float p = ex / zall;  // probability under the full softmax
            w = p / warp_sum(p);
        } else {
            w = ex / zsel;
        }
    }
    if (mine) {
        idx_row[lane] = my_e;
        w_row[lane] = w;
    }
}

constexpr int TOPK_WARPS = 8;

__global__ void __launch_bounds__(TOPK_WARPS * 32) topk_kernel(const float* __restrict__ logits, int T, int E,
                                                                 int k, int mode, int32_t* __restrict__ topk_idx,
                                                                 float* __restrict__ topk_w) {
    grid_dep_wait();
    grid_dep_trigger();
    const int t = blockIdx.x * TOPK_WARPS + (threadIdx.x >> 5);
    if (t >= T) return;
    const float* l = logits + (size_t)t * E;
    warp_route_select([=](int e) { return l[e]; }, E, k, mode, topk_idx + (size_t)t * k, topk_w + (size_t)t * k);
}

}  // namespace moe
