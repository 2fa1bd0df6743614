// Backward pass of the MoE feed-forward layer: the kernels that are not GEMMs.
//
// The blog post "Mixture of Experts (MoEs) in Transformers" (section "Training MoEs with Transformers") trains
// MoE layers through the same grouped expert backend as inference. The gradients of one layer call, with the
// top-k selection held fixed (it is piecewise constant in the router logits):
//   dy_perm[r]   = w[t,j] * dy[t]                       for the row r of assignment (t, j)
//   dw[t,j]      = <dy[t], y_perm[r]>                   gradient of the routing weight
//   dh           = dy_perm W_down[e]                    (grouped GEMM, weights transposed)
//   dg, du       = dh * u * silu'(g), dh * silu(g)      (this file: swiglu_backward_kernel)
//   dx_perm      = [dg | du] W_gateup[e]                (grouped GEMM, weights transposed)
//   dx[t]        = sum_j dx_perm[r(t,j)] + router share (the combine with unit weights)
//   dW_down[e]   = sum_{r in e} dy_perm[r]^T h[r],  dW_gateup[e] = sum_{r in e} [dg|du][r]^T x_perm[r]
//   router: dlogits from dw through the routing-weight formula, dW_r[e] = sum_t dlogit[t,e] x[t],
//           dbias[e] = sum_t dlogit[t,e], dx[t] += sum_j dlogit[t,j] W_r[e_j]
// Every reduction here runs in a fixed order (no atomics), so the results are deterministic.
#pragma once
#include "common.cuh"

namespace moe {

// ---- SwiGLU derivative ----------------------------------------------------------------------------------
// dg = dh * u * s * (1 + g * (1 - s)), du = dh * g * s, with s = 1 / (1 + e^-g) (IEEE divide; s -> 0 or 1 in the
// tails, where the products stay finite). gu holds g in columns [0, f) and u in [f, 2f); so does dgu.
__global__ void __launch_bounds__(256) swiglu_backward_kernel(const __nv_bfloat16* __restrict__ dh,
                                                              const __nv_bfloat16* __restrict__ gu, long M, int f,
                                                              __nv_bfloat16* __restrict__ dgu) {
    grid_dep_wait();
    grid_dep_trigger();
    const int vpr = f / 8;  // 8-element vectors per row of dh
    const long total = M * vpr;
    for (long i = (long)blockIdx.x * blockDim.x + threadIdx.x; i < total; i += (long)gridDim.x * blockDim.x) {
        const long row = i / vpr;
        const int c = (int)(i - row * vpr) * 8;
        const uint4 vh = *reinterpret_cast<const uint4*>(dh + row * f + c);
        const uint4 vg = *reinterpret_cast<const uint4*>(gu + row * 2 * f + c);
        const uint4 vu = *reinterpret_cast<const uint4*>(gu + row * 2 * f + f + c);
        const uint32_t hh[4] = {vh.x, vh.y, vh.z, vh.w}, gg[4] = {vg.x, vg.y, vg.z, vg.w},
                       uu[4] = {vu.x, vu.y, vu.z, vu.w};
        uint32_t og[4], ou[4];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const float2 h2 = unpack_bf16x2(hh[q]), g2 = unpack_bf16x2(gg[q]), u2 = unpack_bf16x2(uu[q]);
            float dg[2], du[2];
            const float hv[2] = {h2.x, h2.y}, gv[2] = {g2.x, g2.y}, uv[2] = {u2.x, u2.y};
#pragma unroll
            for (int e = 0; e < 2; ++e) {
                const float s = 1.0f / (1.0f + expf(-gv[e]));
                du[e] = hv[e] * gv[e] * s;
                dg[e] = hv[e] * uv[e] * s * (1.0f + gv[e] * (1.0f - s));
            }
            og[q] = pack_bf16x2(dg[0], dg[1]);
            ou[q] = pack_bf16x2(du[0], du[1]);
        }
        *reinterpret_cast<uint4*>(dgu + row * 2 * f + c) = make_uint4(og[0], og[1], og[2], og[3]);
        *reinterpret_cast<uint4*>(dgu + row * 2 * f + f + c) = make_uint4(ou[0], ou[1], ou[2], ou[3]);
    }
}

// ---- gradient of the combine -------------------------------------------------------------------------------
// One warp per assignment a = t*k + j (row r = inv_perm[a]): dy_perm[r] = bf16(w[a] * dy[t]) and
// dw[a] = sum_c dy[t][c] * y_perm[r][c] in fp32 (lane-strided partial sums, then a fixed shuffle tree).
constexpr int PB_WARPS = 8;
__global__ void __launch_bounds__(PB_WARPS * 32) permute_backward_kernel(
    const __nv_bfloat16* __restrict__ dy, const int32_t* __restrict__ inv_perm, const float* __restrict__ topk_w,
    const __nv_bfloat16* __restrict__ y_perm, int T, int d, int k, __nv_bfloat16* __restrict__ dy_perm,
    float* __restrict__ dw) {
    grid_dep_wait();
    grid_dep_trigger();
    const int lane = threadIdx.x & 31;
    const long R = (long)T * k;
    for (long a = (long)blockIdx.x * PB_WARPS + (threadIdx.x >> 5); a < R; a += (long)gridDim.x * PB_WARPS) {
        const long t = a / k;
        const int r = inv_perm[a];
        if (r < 0 || r >= R) {
            if (lane == 0) {
                flag_error(MOE_DEVERR_ROW_RANGE);
                dw[a] = 0.f;
            }
            continue;
        }
        const float w = topk_w[a];
        float dot = 0.f;
        for (int c = lane * 8; c < d; c += 256) {
            const uint4 g4 = *reinterpret_cast<const uint4*>(dy + t * d + c);
            const uint4 y4 = *reinterpret_cast<const uint4*>(y_perm + (long)r * d + c);
            const uint32_t gg[4] = {g4.x, g4.y, g4.z, g4.w}, yy[4] = {y4.x, y4.y, y4.z, y4.w};
            uint32_t o[4];
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                const float2 g2 = unpack_bf16x2(gg[q]), y2 = unpack_bf16x2(yy[q]);
                dot = fmaf(g2.x, y2.x, dot);
                dot = fmaf(g2.y, y2.y, dot);
                o[q] = pack_bf16x2(w * g2.x, w * g2.y);
            }
            *reinterpret_cast<uint4*>(dy_perm + (long)r * d + c) = make_uint4(o[0], o[1], o[2], o[3]);
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) dot += __shfl_xor_sync(0xffffffffu, dot, o);
        if (lane == 0) dw[a] = dot;
    }
}

// ---- transposes ---------------------------------------------------------------------------------------------
// dst[g][c][r] = src[g][r][c] for every group, 32 x 32 tiles through shared memory (bf16).
__global__ void __launch_bounds__(256) transpose_kernel(const __nv_bfloat16* __restrict__ src, int rows, int cols,
                                                        __nv_bfloat16* __restrict__ dst) {
    __shared__ __nv_bfloat16 tile[32][33];
    grid_dep_wait();
    grid_dep_trigger();
    const long g = blockIdx.z;
    const int r0 = blockIdx.y * 32, c0 = blockIdx.x * 32;
    const __nv_bfloat16* s = src + g * (long)rows * cols;
    __nv_bfloat16* o = dst + g * (long)rows * cols;
    const int tx = threadIdx.x & 31, ty = threadIdx.x >> 5;  // 32 x 8 threads
#pragma unroll
    for (int i = 0; i < 32; i += 8) {
        const int r = r0 + ty + i, c = c0 + tx;
        if (r < rows && c < cols) tile[ty + i][tx] = s[(long)r * cols + c];
    }
    __syncthreads();
#pragma unroll
    for (int i = 0; i < 32; i += 8) {
        const int c = c0 + ty + i, r = r0 + tx;
        if (r < rows && c < cols) o[(long)c * rows + r] = tile[tx][ty + i];
    }
}

// Group g's rows padded to a multiple of 64: pad_off[g] = sum_{i<g} roundup64(rows_i), pad_off[G] the total.
// One block of 1024 threads (G <= 1024).
constexpr int WG_PAD = 64;
__global__ void __launch_bounds__(1024) pad_offsets_kernel(const int32_t* __restrict__ offsets, int G, int M,
                                                           int32_t* __restrict__ pad_off) {
    __shared__ int warp_sums[32];
    grid_dep_wait();
    grid_dep_trigger();
    const int g = threadIdx.x, lane = g & 31, w = g >> 5;
    int v = 0;
    if (g < G) {
        int a = offsets[g], b = offsets[g + 1];
        if (a < 0 || b > M || b < a) {
            flag_error(MOE_DEVERR_GROUP_RANGE);
            a = min(max(a, 0), M);
            b = min(max(b, a), M);
        }
        v = (b - a + WG_PAD - 1) / WG_PAD * WG_PAD;
    }
    int incl = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int u = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += u;
    }
    if (lane == 31) warp_sums[w] = incl;
    __syncthreads();
    if (w == 0) {
        int s = warp_sums[lane];
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int u = __shfl_up_sync(0xffffffffu, s, o);
            if (lane >= o) s += u;
        }
        warp_sums[lane] = s;  // inclusive sums of the warps
    }
    __syncthreads();
    const int excl = incl - v + (w > 0 ? warp_sums[w - 1] : 0);
    if (g < G) pad_off[g] = excl;
    if (g == G - 1) pad_off[G] = excl + v;
}

// dst[c][q] for padded positions q in [0, pad_cap): q in group g (pad_off[g] <= q < pad_off[g+1]) at row
// q - pad_off[g] < rows_g holds src[offsets[g] + q - pad_off[g]][c]; the rest of the group's padding is zero.
// Positions at or past pad_off[G] are not written (never read). 64 x 64 tiles: each thread loads 16 bytes (8
// columns) of a source row and stores 16 bytes (8 positions) of a destination row; the tile goes through shared
// memory as 32-bit words with a padded pitch. cols a multiple of 8.
constexpr int TP_TILE = 64;
__global__ void __launch_bounds__(256) transpose_pad_kernel(const __nv_bfloat16* __restrict__ src,
                                                            const int32_t* __restrict__ offsets,
                                                            const int32_t* __restrict__ pad_off, int G, int M,
                                                            int cols, long pad_cap, __nv_bfloat16* __restrict__ dst) {
    __shared__ uint16_t tile[TP_TILE][TP_TILE + 2];  // [q][c], pitch 66 halves
    __shared__ int src_row[TP_TILE];
    grid_dep_wait();
    grid_dep_trigger();
    const long q0 = (long)blockIdx.y * TP_TILE;
    const int c0 = blockIdx.x * TP_TILE;
    const int total = pad_off[G];
    if (q0 >= total) return;
    if (threadIdx.x < TP_TILE) {
        const long q = q0 + threadIdx.x;
        int sr = -1;
        if (q < total) {
            int lo = 0, hi = G - 1;  // last group with pad_off[g] <= q
            while (lo < hi) {
                const int mid = (lo + hi + 1) >> 1;
                if (pad_off[mid] <= q)
                    lo = mid;
                else
                    hi = mid - 1;
            }
            const int a = min(max(offsets[lo], 0), M), b = min(max(offsets[lo + 1], a), M);
            const long i = q - pad_off[lo];
            if (i < b - a) sr = a + (int)i;
        }
        src_row[threadIdx.x] = sr;
    }
    __syncthreads();
    // load: 64 rows x 8 pieces of 8 columns, 256 threads -> 2 rounds
#pragma unroll
    for (int it = 0; it < 2; ++it) {
        const int idx = threadIdx.x + it * 256;
        const int r = idx >> 3, piece = idx & 7;
        const int c = c0 + piece * 8;
        const int sr = src_row[r];
        uint4 v = make_uint4(0, 0, 0, 0);
        if (sr >= 0 && c < cols) v = *reinterpret_cast<const uint4*>(src + (long)sr * cols + c);
        const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            tile[r][piece * 8 + 2 * j] = (uint16_t)(w[j] & 0xffffu);
            tile[r][piece * 8 + 2 * j + 1] = (uint16_t)(w[j] >> 16);
        }
    }
    __syncthreads();
    // store: 64 columns (destination rows) x 8 pieces of 8 positions
#pragma unroll
    for (int it = 0; it < 2; ++it) {
        const int idx = threadIdx.x + it * 256;
        const int cc = idx >> 3, piece = idx & 7;
        const int c = c0 + cc;
        const long q = q0 + piece * 8;
        if (c >= cols || q >= total) continue;
        uint32_t w[4];
#pragma unroll
        for (int j = 0; j < 4; ++j)
            w[j] = (uint32_t)tile[piece * 8 + 2 * j][cc] | ((uint32_t)tile[piece * 8 + 2 * j + 1][cc] << 16);
        *reinterpret_cast<uint4*>(dst + (long)c * pad_cap + q) = make_uint4(w[0], w[1], w[2], w[3]);
    }
}

// ---- router --------------------------------------------------------------------------------------------------
// dlogits of the k selected experts of each token, from dw (the routing weights' gradient), with the selection
// held fixed. Softmax over the selected logits (also the softmax-then-renormalise mode, the same function of
// them): dl_j = w_j (dw_j - sum_i w_i dw_i). Sigmoid normalised: with s_i = sigma(l_i), S = sum s_i,
// dl_i = (dw_i - sum_j w_j dw_j) / S * s_i (1 - s_i). Written per assignment (dl_tk) and per grouped row (dl_perm).
__global__ void __launch_bounds__(256) router_dlogits_kernel(const float* __restrict__ logits,
                                                             const int32_t* __restrict__ topk_idx,
                                                             const float* __restrict__ topk_w,
                                                             const float* __restrict__ dw,
                                                             const int32_t* __restrict__ inv_perm, int T, int E,
                                                             int k, int mode, float* __restrict__ dl_tk,
                                                             float* __restrict__ dl_perm) {
    grid_dep_wait();
    grid_dep_trigger();
    const long R = (long)T * k;
    for (long t = (long)blockIdx.x * blockDim.x + threadIdx.x; t < T; t += (long)gridDim.x * blockDim.x) {
        const float* w = topk_w + t * k;
        const float* g = dw + t * k;
        float wdw = 0.f;
        for (int j = 0; j < k; ++j) wdw = fmaf(w[j], g[j], wdw);
        float S = 0.f;
        if (mode == MOE_ROUTE_SIGMOID_TOPK_NORM) {
            for (int j = 0; j < k; ++j) {
                const int e = topk_idx[t * k + j];
                const float l = (e >= 0 && e < E) ? logits[t * E + e] : 0.f;
                S += 1.0f / (1.0f + expf(-l));
            }
        }
        for (int j = 0; j < k; ++j) {
            float dl;
            if (mode == MOE_ROUTE_SIGMOID_TOPK_NORM) {
                const int e = topk_idx[t * k + j];
                const float l = (e >= 0 && e < E) ? logits[t * E + e] : 0.f;
                const float s = 1.0f / (1.0f + expf(-l));
                dl = (g[j] - wdw) / S * s * (1.0f - s);
            } else {
                dl = w[j] * (g[j] - wdw);
            }
            dl_tk[t * k + j] = dl;
            const int r = inv_perm[t * k + j];
            if (r >= 0 && r < R)
                dl_perm[r] = dl;
            else
                flag_error(MOE_DEVERR_ROW_RANGE);
        }
    }
}

// dW_r[e][c] = sum over the rows r of expert e (in grouped order) of dl_perm[r] * x[perm_src[r]][c], and
// dbias[e] = sum of the same dl_perm[r], in two deterministic passes: each expert's rows are cut into chunks of
// RB_ROWS (chunk_prefix[e] = chunks before expert e, router_chunk_prefix_kernel); router_chunk_partial_kernel sums
// one chunk per block and 256-column slice into partial[chunk][c]; router_chunk_reduce_kernel adds an expert's
// chunk partials in chunk order.
constexpr int RB_COLS = 256;
constexpr int RB_ROWS = 256;
__global__ void __launch_bounds__(1024) router_chunk_prefix_kernel(const int32_t* __restrict__ offsets, int E, int R,
                                                                   int32_t* __restrict__ chunk_prefix) {
    __shared__ int warp_sums[32];
    grid_dep_wait();
    grid_dep_trigger();
    const int e = threadIdx.x, lane = e & 31, w = e >> 5;
    int v = 0;
    if (e < E) {
        const int a = min(max(offsets[e], 0), R), b = min(max(offsets[e + 1], a), R);
        v = (b - a + RB_ROWS - 1) / RB_ROWS;
    }
    int incl = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int u = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += u;
    }
    if (lane == 31) warp_sums[w] = incl;
    __syncthreads();
    if (w == 0) {
        int sm = warp_sums[lane];
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int u = __shfl_up_sync(0xffffffffu, sm, o);
            if (lane >= o) sm += u;
        }
        warp_sums[lane] = sm;
    }
    __syncthreads();
    const int excl = incl - v + (w > 0 ? warp_sums[w - 1] : 0);
    if (e < E) chunk_prefix[e] = excl;
    if (e == E - 1) chunk_prefix[E] = excl + v;
}

__global__ void __launch_bounds__(RB_COLS) router_chunk_partial_kernel(
    const __nv_bfloat16* __restrict__ x, const int32_t* __restrict__ perm_src, const int32_t* __restrict__ offsets,
    const int32_t* __restrict__ chunk_prefix, const float* __restrict__ dl_perm, int T, int d, int E, int R,
    float* __restrict__ partial, float* __restrict__ pbias) {
    grid_dep_wait();
    grid_dep_trigger();
    const int chunk = blockIdx.y;
    if (chunk >= chunk_prefix[E]) return;
    int lo = 0, hi = E - 1;  // the last expert whose first chunk is <= chunk
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (chunk_prefix[mid] <= chunk)
            lo = mid;
        else
            hi = mid - 1;
    }
    const int e = lo;
    const int a = min(max(offsets[e], 0), R), b = min(max(offsets[e + 1], a), R);
    const int r0 = a + (chunk - chunk_prefix[e]) * RB_ROWS, r1 = min(r0 + RB_ROWS, b);
    const int c = blockIdx.x * RB_COLS + threadIdx.x;
    float acc = 0.f, bsum = 0.f;
    for (int r = r0; r < r1; ++r) {
        const float dl = dl_perm[r];
        const int t = perm_src[r];
        bsum += dl;
        if (c < d && t >= 0 && t < T) acc = fmaf(dl, __bfloat162float(x[(long)t * d + c]), acc);
    }
    if (c < d) partial[(long)chunk * d + c] = acc;
    if (blockIdx.x == 0 && threadIdx.x == 0) pbias[chunk] = bsum;
}

__global__ void __launch_bounds__(RB_COLS) router_chunk_reduce_kernel(const int32_t* __restrict__ chunk_prefix,
                                                                      const float* __restrict__ partial,
                                                                      const float* __restrict__ pbias, int d, int E,
                                                                      float* __restrict__ dw_router,
                                                                      float* __restrict__ dbias) {
    grid_dep_wait();
    grid_dep_trigger();
    const int e = blockIdx.y;
    const int c = blockIdx.x * RB_COLS + threadIdx.x;
    const int k0 = chunk_prefix[e], k1 = chunk_prefix[e + 1];
    float acc = 0.f;
    if (c < d) {
        for (int ch = k0; ch < k1; ++ch) acc += partial[(long)ch * d + c];
        dw_router[(long)e * d + c] = acc;
    }
    if (dbias && blockIdx.x == 0 && threadIdx.x == 0) {
        float bs = 0.f;
        for (int ch = k0; ch < k1; ++ch) bs += pbias[ch];
        dbias[e] = bs;
    }
}

// dx_router[t][c] = sum_j dl_tk[t][j] * W_r[e_j][c] (+ addend[t][c]), fp32 sum in slot order, rounded to bf16.
// One warp per token, 8 columns per lane per step.
__global__ void __launch_bounds__(256) router_input_grad_kernel(const int32_t* __restrict__ topk_idx,
                                                                const float* __restrict__ dl_tk,
                                                                const float* __restrict__ w_router,
                                                                const __nv_bfloat16* __restrict__ addend, int T, int d,
                                                                int E, int k, __nv_bfloat16* __restrict__ dx) {
    grid_dep_wait();
    grid_dep_trigger();
    const int lane = threadIdx.x & 31;
    for (long t = (long)blockIdx.x * 8 + (threadIdx.x >> 5); t < T; t += (long)gridDim.x * 8) {
        for (int c = lane * 8; c < d; c += 256) {
            float acc[8];
            if (addend) {
                const uint4 a4 = *reinterpret_cast<const uint4*>(addend + t * d + c);
                const uint32_t aa[4] = {a4.x, a4.y, a4.z, a4.w};
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    const float2 v = unpack_bf16x2(aa[q]);
                    acc[2 * q] = v.x;
                    acc[2 * q + 1] = v.y;
                }
            } else {
#pragma unroll
                for (int q = 0; q < 8; ++q) acc[q] = 0.f;
            }
            for (int j = 0; j < k; ++j) {
                const int e = topk_idx[t * k + j];
                if (e < 0 || e >= E) continue;
                const float dl = dl_tk[t * k + j];
                const float4 w0 = *reinterpret_cast<const float4*>(w_router + (long)e * d + c);
                const float4 w1 = *reinterpret_cast<const float4*>(w_router + (long)e * d + c + 4);
                acc[0] = fmaf(dl, w0.x, acc[0]);
                acc[1] = fmaf(dl, w0.y, acc[1]);
                acc[2] = fmaf(dl, w0.z, acc[2]);
                acc[3] = fmaf(dl, w0.w, acc[3]);
                acc[4] = fmaf(dl, w1.x, acc[4]);
                acc[5] = fmaf(dl, w1.y, acc[5]);
                acc[6] = fmaf(dl, w1.z, acc[6]);
                acc[7] = fmaf(dl, w1.w, acc[7]);
            }
            *reinterpret_cast<uint4*>(dx + t * d + c) =
                make_uint4(pack_bf16x2(acc[0], acc[1]), pack_bf16x2(acc[2], acc[3]), pack_bf16x2(acc[4], acc[5]),
                           pack_bf16x2(acc[6], acc[7]));
        }
    }
}

}  // namespace moe
