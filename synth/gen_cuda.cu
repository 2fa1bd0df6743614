/*
 * Seeded synthetic inputs for the MoE feed-forward layer: GPU implementation.
 *
 * The definition is the one stated at the top of gen.c (SplitMix64 draws,
 * Irwin-Hall sum of twelve 32-bit uniforms, one fp64 multiply by sigma, fp32
 * then bf16 round-to-nearest-even). Only integer operations, an exact
 * int64->fp64 conversion, one correctly rounded fp64 multiply and correctly
 * rounded conversions are used, so the output is bit-identical to the host's.
 * It exists so that multi-gigabyte weight tensors can be filled directly in
 * device memory. It holds no part of the layer's arithmetic.
 */
#include <cstdint>
#include <cuda_runtime.h>

#define GAMMA 0x9e3779b97f4a7c15ULL

__host__ __device__ static inline uint64_t mix64(uint64_t z) {
    z ^= z >> 30; z *= 0xbf58476d1ce4e5b9ULL;
    z ^= z >> 27; z *= 0x94d049bb133111ebULL;
    z ^= z >> 31;
    return z;
}

__device__ static inline double irwin_hall12(uint64_t key, uint64_t i) {
    uint64_t s = 0;
#pragma unroll
    for (int j = 0; j < 6; ++j) {
        uint64_t r = mix64(key + (6 * i + (uint64_t)j + 1) * GAMMA);
        s += (r & 0xffffffffULL) + (r >> 32);
    }
    long long c = (long long)s - (long long)(6ULL << 32);
    return __dmul_rn(__ll2double_rn(c), 1.0 / 4294967296.0);
}

__device__ static inline uint16_t f32_to_bf16_rne(float v) {
    uint32_t u = __float_as_uint(v);
    if ((u & 0x7f800000u) == 0x7f800000u) return (uint16_t)(u >> 16);
    uint32_t lsb = (u >> 16) & 1u;
    u += 0x7fffu + lsb;
    return (uint16_t)(u >> 16);
}

__global__ void synth_normal_kernel(uint64_t key, uint64_t first, uint64_t count, double sigma, void* out,
                                    int kind) {
    uint64_t stride = (uint64_t)gridDim.x * blockDim.x;
    for (uint64_t i = (uint64_t)blockIdx.x * blockDim.x + threadIdx.x; i < count; i += stride) {
        float v = __double2float_rn(__dmul_rn(irwin_hall12(key, first + i), sigma));
        if (kind == 0)
            ((uint16_t*)out)[i] = f32_to_bf16_rne(v);
        else
            ((float*)out)[i] = v;
    }
}

static uint64_t stream_key(uint64_t seed, uint64_t tensor_id) { return mix64(mix64(seed) + tensor_id * GAMMA); }

static int launch(uint64_t seed, uint64_t tensor_id, uint64_t first, uint64_t count, double sigma, void* out,
                  int kind, cudaStream_t stream) {
    if (count == 0) return 0;
    if (out == nullptr) return 1;
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    uint64_t want = (count + 255) / 256;
    uint64_t cap = (uint64_t)sms * 16;
    unsigned grid = (unsigned)(want < cap ? want : cap);
    synth_normal_kernel<<<grid, 256, 0, stream>>>(stream_key(seed, tensor_id), first, count, sigma, out, kind);
    return cudaGetLastError() == cudaSuccess ? 0 : 2;
}

extern "C" {
/* Fill out[0..count) (device memory) with elements [first, first+count) of the
 * bf16 tensor (seed, tensor_id, sigma). Returns 0 on success. Asynchronous. */
int synth_normal_bf16_device(uint64_t seed, uint64_t tensor_id, uint64_t first, uint64_t count, double sigma,
                             void* out, void* stream) {
    return launch(seed, tensor_id, first, count, sigma, out, 0, (cudaStream_t)stream);
}
/* Same draws as fp32. */
int synth_normal_f32_device(uint64_t seed, uint64_t tensor_id, uint64_t first, uint64_t count, double sigma,
                            void* out, void* stream) {
    return launch(seed, tensor_id, first, count, sigma, out, 1, (cudaStream_t)stream);
}
}
