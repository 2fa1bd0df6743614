/*
 * Seeded synthetic inputs for the MoE feed-forward layer: host implementation.
 *
 * This file holds no part of the layer's arithmetic. It only draws numbers.
 * The same generator is implemented for the GPU in gen_cuda.cu; both follow
 * the definition below, use only integer operations and IEEE-754 correctly
 * rounded conversions/multiplies, and therefore agree bit for bit.
 *
 * Definition
 *   mix64(z)      the SplitMix64 output function (Steele, Lea & Flood,
 *                 "Fast splittable pseudorandom number generators", OOPSLA 2014):
 *                 z ^= z >> 30; z *= 0xbf58476d1ce4e5b9;
 *                 z ^= z >> 27; z *= 0x94d049bb133111eb; z ^= z >> 31.
 *   key(s, id)    mix64(mix64(s) + id * GAMMA), GAMMA = 0x9e3779b97f4a7c15
 *   draw(s,id,n)  mix64(key(s,id) + (n + 1) * GAMMA)   (the n-th SplitMix64
 *                 output of the stream that starts at key(s,id))
 *   normal(i)     Irwin-Hall sum of twelve 32-bit uniforms taken from draws
 *                 6i .. 6i+5 (low half, then high half of each draw):
 *                 S = sum of the twelve uint32 values (exact, in uint64),
 *                 z = (double)(S - 6 * 2^32) * 2^-32      (exact),
 *                 which has mean ~0 and variance 1 and lies in [-6, 6].
 *   value(i)      (float)(z * sigma)   [one fp64 multiply, then fp64->fp32 RNE]
 *   bf16 value    round-to-nearest-even of the fp32 value to bfloat16.
 *   uniform64(n)  draw(s, id, n) itself, for permutations and the like.
 *
 * Element i of a tensor is its flat row-major index.
 */
#include <stdint.h>
#include <string.h>
#include <pthread.h>

#define GAMMA 0x9e3779b97f4a7c15ULL

static inline uint64_t mix64(uint64_t z) {
    z ^= z >> 30; z *= 0xbf58476d1ce4e5b9ULL;
    z ^= z >> 27; z *= 0x94d049bb133111ebULL;
    z ^= z >> 31;
    return z;
}

uint64_t synth_stream_key(uint64_t seed, uint64_t tensor_id) {
    return mix64(mix64(seed) + tensor_id * GAMMA);
}

uint64_t synth_draw(uint64_t key, uint64_t n) { return mix64(key + (n + 1) * GAMMA); }

static inline double irwin_hall12(uint64_t key, uint64_t i) {
    uint64_t s = 0;
    for (int j = 0; j < 6; ++j) {
        uint64_t r = mix64(key + (6 * i + (uint64_t)j + 1) * GAMMA);
        s += (r & 0xffffffffULL) + (r >> 32);
    }
    int64_t c = (int64_t)s - (int64_t)(6ULL << 32);
    return (double)c * (1.0 / 4294967296.0);
}

static inline uint16_t f32_to_bf16_rne(float v) {
    uint32_t u;
    memcpy(&u, &v, 4);
    if ((u & 0x7f800000u) == 0x7f800000u) return (uint16_t)(u >> 16); /* inf/nan: not produced here */
    uint32_t lsb = (u >> 16) & 1u;
    u += 0x7fffu + lsb;
    return (uint16_t)(u >> 16);
}

typedef struct {
    uint64_t key, first, count;
    double sigma;
    void* out;
    int kind; /* 0 bf16, 1 f32 */
} job_t;

static void* run_job(void* p) {
    job_t* j = (job_t*)p;
    if (j->kind == 0) {
        uint16_t* o = (uint16_t*)j->out;
        for (uint64_t i = 0; i < j->count; ++i) {
            float v = (float)(irwin_hall12(j->key, j->first + i) * j->sigma);
            o[i] = f32_to_bf16_rne(v);
        }
    } else {
        float* o = (float*)j->out;
        for (uint64_t i = 0; i < j->count; ++i)
            o[i] = (float)(irwin_hall12(j->key, j->first + i) * j->sigma);
    }
    return NULL;
}

static void run_parallel(uint64_t key, uint64_t first, uint64_t count, double sigma, void* out, int kind,
                         int nthreads) {
    if (nthreads < 1) nthreads = 1;
    if (nthreads > 256) nthreads = 256;
    if (count < (uint64_t)nthreads * 4096) nthreads = 1;
    pthread_t th[256];
    job_t jobs[256];
    uint64_t per = (count + (uint64_t)nthreads - 1) / (uint64_t)nthreads;
    int started = 0;
    for (int t = 0; t < nthreads; ++t) {
        uint64_t b = (uint64_t)t * per;
        if (b >= count) break;
        uint64_t n = count - b < per ? count - b : per;
        jobs[t].key = key; jobs[t].first = first + b; jobs[t].count = n; jobs[t].sigma = sigma;
        jobs[t].kind = kind;
        jobs[t].out = kind == 0 ? (void*)((uint16_t*)out + b) : (void*)((float*)out + b);
        if (nthreads == 1) { run_job(&jobs[t]); started = 0; break; }
        if (pthread_create(&th[t], NULL, run_job, &jobs[t]) != 0) { run_job(&jobs[t]); continue; }
        started = t + 1;
    }
    for (int t = 0; t < started; ++t) pthread_join(th[t], NULL);
}

/* Elements [first, first+count) of a N(0, sigma^2)-like tensor, as bf16 bits. */
void synth_normal_bf16(uint64_t seed, uint64_t tensor_id, uint64_t first, uint64_t count, double sigma,
                       uint16_t* out, int nthreads) {
    run_parallel(synth_stream_key(seed, tensor_id), first, count, sigma, out, 0, nthreads);
}

/* Same draws, kept as fp32. */
void synth_normal_f32(uint64_t seed, uint64_t tensor_id, uint64_t first, uint64_t count, double sigma,
                      float* out, int nthreads) {
    run_parallel(synth_stream_key(seed, tensor_id), first, count, sigma, out, 1, nthreads);
}

/* Raw 64-bit draws n = first .. first+count-1 of a stream. */
void synth_uniform_u64(uint64_t seed, uint64_t tensor_id, uint64_t first, uint64_t count, uint64_t* out) {
    uint64_t key = synth_stream_key(seed, tensor_id);
    for (uint64_t i = 0; i < count; ++i) out[i] = synth_draw(key, first + i);
}
