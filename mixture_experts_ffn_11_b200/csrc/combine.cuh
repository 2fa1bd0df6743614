// Weighted combine back to token order: "apply the routing weights and then collect and reorder the
// results" (blog post "Mixture of Experts (MoEs) in Transformers", section "Expert Backend").
// y[t] = sum_{j<k} w[t][j] * y_perm[inv_perm[t*k+j]] (+ shared[t]), fp32 in slot order, bf16 out.
// Warps over (token, column chunk), 16-byte vectors along d; deterministic (no atomics).
#pragma once
#include "common.cuh"

namespace moe {

// Work item = (token, chunk of CB_CHUNK_VEC 16-byte vectors); a warp handles one item with each lane on
// CB_VPL vectors, and the k slot loads of a vector are unrolled in groups of CB_KU so several are in flight.
// Two vectors per lane (items of 1 KB per slot row) rather than four: more, smaller items fill the grid's last wave
// (measured: gpt-oss-shaped combine 33 -> 30 µs, zipf-128e 117-121 -> 109 µs).
constexpr int CB_VPL = 2, CB_CHUNK_VEC = 32 * CB_VPL, CB_KU = 8;

__global__ void __launch_bounds__(256) combine_kernel(const __nv_bfloat16* __restrict__ y_perm,
                                                      const int32_t* __restrict__ inv_perm,
                                                      const float* __restrict__ topk_w,
                                                      const __nv_bfloat16* __restrict__ shared, int T, int d, int k,
                                                      int R, __nv_bfloat16* __restrict__ y) {
    grid_dep_wait();
    grid_dep_trigger();
    const int lane = threadIdx.x & 31;
    const int nvec = d / 8;
    const int nchunk = (nvec + CB_CHUNK_VEC - 1) / CB_CHUNK_VEC;
    const long items = (long)T * nchunk;
    const long nwarps = (long)gridDim.x * (blockDim.x / 32);
    for (long it = (long)blockIdx.x * (blockDim.x / 32) + (threadIdx.x >> 5); it < items; it += nwarps) {
        const long t = it / nchunk;
        const int chunk = (int)(it - t * nchunk);
        int my_row = -1;
        float my_w = 0.f;
        if (lane < k) {
            my_row = inv_perm[t * k + lane];
            my_w = topk_w[t * k + lane];
            if (my_row < 0 || my_row >= R) {
                flag_error(MOE_DEVERR_ROW_RANGE);
                my_row = -1;
            }
        }
        float acc[CB_VPL][8];
#pragma unroll
        for (int u = 0; u < CB_VPL; ++u)
#pragma unroll
            for (int i = 0; i < 8; ++i) acc[u][i] = 0.f;
        for (int j0 = 0; j0 < k; j0 += CB_KU) {
#pragma unroll
            for (int jj = 0; jj < CB_KU; ++jj) {
                const int j = j0 + jj;
                const int row = __shfl_sync(0xffffffffu, my_row, j & 31);
                const float w = __shfl_sync(0xffffffffu, my_w, j & 31);
                if (j >= k || row < 0) continue;
                const uint4* src = reinterpret_cast<const uint4*>(y_perm + (size_t)row * d);
#pragma unroll
                for (int u = 0; u < CB_VPL; ++u) {
                    const int v = chunk * CB_CHUNK_VEC + u * 32 + lane;
                    if (v < nvec) {
                        const uint4 q = __ldg(src + v);
                        const uint32_t uq[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
                        for (int i = 0; i < 4; ++i) {
                            const float2 f = unpack_bf16x2(uq[i]);
                            acc[u][2 * i] = fmaf(w, f.x, acc[u][2 * i]);
                            acc[u][2 * i + 1] = fmaf(w, f.y, acc[u][2 * i + 1]);
                        }
                    }
                }
            }
        }
#pragma unroll
        for (int u = 0; u < CB_VPL; ++u) {
            const int v = chunk * CB_CHUNK_VEC + u * 32 + lane;
            if (v >= nvec) continue;
            if (shared) {
                const uint4 q = __ldg(reinterpret_cast<const uint4*>(shared + (size_t)t * d) + v);
                const uint32_t uq[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const float2 f = unpack_bf16x2(uq[i]);
                    acc[u][2 * i] += f.x;
                    acc[u][2 * i + 1] += f.y;
                }
            }
            uint4 o;
            o.x = pack_bf16x2(acc[u][0], acc[u][1]);
            o.y = pack_bf16x2(acc[u][2], acc[u][3]);
            o.z = pack_bf16x2(acc[u][4], acc[u][5]);
            o.w = pack_bf16x2(acc[u][6], acc[u][7]);
            reinterpret_cast<uint4*>(y + (size_t)t * d)[v] = o;
        }
    }
}

}  // namespace moe
