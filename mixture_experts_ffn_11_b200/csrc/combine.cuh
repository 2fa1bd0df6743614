// Weighted combine back to token order: "apply the routing weights and then collect and reorder the
// results" (blog post "Mixture of Experts (MoEs) in Transformers", section "Expert Backend").
// y[t] = sum_{j<k} w[t][j] * y_perm[inv_perm[t*k+j]] (+ shared[t]), fp32 in slot order, bf16 out.
// One warp per token, 16-byte vectors along d; deterministic (no atomics).
#pragma once
#include "common.cuh"

namespace moe {

__global__ void __launch_bounds__(256) combine_kernel(const __nv_bfloat16* __restrict__ y_perm,
                                                      const int32_t* __restrict__ inv_perm,
                                                      const float* __restrict__ topk_w,
                                                      const __nv_bfloat16* __restrict__ shared, int T, int d, int k,
                                                      int R, __nv_bfloat16* __restrict__ y) {
    const int lane = threadIdx.x & 31;
    const int nvec = d / 8;
    const long nwarps = (long)gridDim.x * (blockDim.x / 32);
    for (long t = (long)blockIdx.x * (blockDim.x / 32) + (threadIdx.x >> 5); t < T; t += nwarps) {
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
        for (int v = lane; v < nvec; v += 32) {
            float acc[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) acc[i] = 0.f;
            for (int j = 0; j < k; ++j) {
                const int row = __shfl_sync(0xffffffffu, my_row, j);
                const float w = __shfl_sync(0xffffffffu, my_w, j);
                if (row < 0) continue;
                const uint4 q = __ldg(reinterpret_cast<const uint4*>(y_perm + (size_t)row * d) + v);
                const uint32_t u[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const float2 f = unpack_bf16x2(u[i]);
                    acc[2 * i] = fmaf(w, f.x, acc[2 * i]);
                    acc[2 * i + 1] = fmaf(w, f.y, acc[2 * i + 1]);
                }
            }
            if (shared) {
                const uint4 q = __ldg(reinterpret_cast<const uint4*>(shared + (size_t)t * d) + v);
                const uint32_t u[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const float2 f = unpack_bf16x2(u[i]);
                    acc[2 * i] += f.x;
                    acc[2 * i + 1] += f.y;
                }
            }
            uint4 o;
            o.x = pack_bf16x2(acc[0], acc[1]);
            o.y = pack_bf16x2(acc[2], acc[3]);
            o.z = pack_bf16x2(acc[4], acc[5]);
            o.w = pack_bf16x2(acc[6], acc[7]);
            reinterpret_cast<uint4*>(y + (size_t)t * d)[v] = o;
        }
    }
}

}  // namespace moe
