/*
 * CPU oracle for the sparse MoE feed-forward layer.
 *
 * TEST INFRASTRUCTURE ONLY. This code proves the CUDA path correct; it is not
 * part of the product. Only the tests, the smoke check and the benchmark's CPU
 * baseline leg may load it. It shares no code, header, table or helper with
 * the CUDA path.
 *
 * What it computes follows the blog post "Mixture of Experts (MoEs) in
 * Transformers":
 *   - section "From Dense to Sparse": a router picks a small subset of experts
 *     per token; each expert is a learnable sub-network that replaces the
 *     dense feed-forward block;
 *   - section "Expert Backend": the runtime dispatches tokens to their
 *     selected experts, runs the projections, applies the routing weights and
 *     collects the results back in token order; the "eager" backend, a plain
 *     loop over the selected experts, is the correctness reference. This file
 *     is that loop, written per token;
 *   - section "Dynamic Weight Loading with WeightConverter": the packed
 *     gate_up_proj tensor stacks experts on dim 0 and concatenates w1 (gate)
 *     then w3 (up) on dim 1, so expert e's rows [0,f) are gate and [f,2f) are
 *     up, each row of length d; down_proj stacks the experts' w2 on dim 0,
 *     each [d, f] (output row c, input column n).
 *   - "sort tokens by expert ID, group them" (grouped_mm, section "Expert
 *     Backend"): the grouping is a stable counting sort by expert id.
 * The pages do not state the router formula or the expert activation; the
 * layer descriptions this library serves fix them: fp32 logits x.W_r^T (+bias),
 * top-k on the logits (descending, lower expert id first on ties), weights by
 * one of three modes, and a SwiGLU expert silu(gate)*up followed by down.
 *
 * Precision: every sum is accumulated in fp64 from the bf16/fp32 inputs, and
 * the SwiGLU intermediate is kept in fp64. The only rounding to fp32 is of
 * the router logits, because top-k selection (an integer decision) is taken
 * in fp32 on both sides.
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

enum { ORACLE_TOPK_SOFTMAX = 0, ORACLE_SOFTMAX_TOPK_RENORM = 1, ORACLE_SIGMOID_TOPK_NORM = 2 };

static double bf16_to_double(uint16_t b) {
    uint32_t u = (uint32_t)b << 16;
    float v;
    memcpy(&v, &u, 4);
    return (double)v;
}

/* Router logits: l[t][e] = sum_i x[t][i] * W_r[e][i] (+ bias[e]), in fp64. */
void oracle_router_logits(const uint16_t* x, const float* w_router, const float* bias, int T, int d, int E,
                          double* logits) {
    for (int t = 0; t < T; ++t) {
        for (int e = 0; e < E; ++e) {
            double s = 0.0;
            for (int i = 0; i < d; ++i) s += bf16_to_double(x[(size_t)t * d + i]) * (double)w_router[(size_t)e * d + i];
            if (bias) s += (double)bias[e];
            logits[(size_t)t * E + e] = s;
        }
    }
}

/* Top-k selection and routing weights from fp32 logits [T][E].
 * idx[t][j]: the j-th largest logit's expert (ties: lower expert id first).
 * w[t][j]:   routing weight of that expert, by mode, in fp64.
 * Returns 0, or -1 on bad arguments. */
int oracle_topk(const float* logits, int T, int E, int k, int mode, int32_t* idx, double* w) {
    if (T < 0 || E <= 0 || k <= 0 || k > E) return -1;
    if (mode < 0 || mode > 2) return -1;
    char* taken = (char*)malloc((size_t)E);
    if (!taken) return -1;
    for (int t = 0; t < T; ++t) {
        const float* l = logits + (size_t)t * E;
        memset(taken, 0, (size_t)E);
        /* k passes of "largest not yet taken"; strict '>' keeps the lower id on ties. */
        for (int j = 0; j < k; ++j) {
            int best = -1;
            for (int e = 0; e < E; ++e) {
                if (taken[e]) continue;
                if (best < 0 || l[e] > l[best]) best = e;
            }
            taken[best] = 1;
            idx[(size_t)t * k + j] = best;
        }
        double* wt = w + (size_t)t * k;
        const int32_t* it = idx + (size_t)t * k;
        if (mode == ORACLE_TOPK_SOFTMAX) {
            /* softmax over the k selected logits (max-subtracted) */
            double m = (double)l[it[0]];
            double z = 0.0;
            for (int j = 0; j < k; ++j) { wt[j] = exp((double)l[it[j]] - m); z += wt[j]; }
            for (int j = 0; j < k; ++j) wt[j] /= z;
        } else if (mode == ORACLE_SOFTMAX_TOPK_RENORM) {
            /* softmax over all E logits, keep the selected probabilities, divide by their sum */
            double m = (double)l[it[0]];
            double zall = 0.0;
            for (int e = 0; e < E; ++e) zall += exp((double)l[e] - m);
            double zsel = 0.0;
            for (int j = 0; j < k; ++j) { wt[j] = exp((double)l[it[j]] - m) / zall; zsel += wt[j]; }
            for (int j = 0; j < k; ++j) wt[j] /= zsel;
        } else {
            /* sigmoid scores of the selected experts, divided by their sum */
            double z = 0.0;
            for (int j = 0; j < k; ++j) { wt[j] = 1.0 / (1.0 + exp(-(double)l[it[j]])); z += wt[j]; }
            for (int j = 0; j < k; ++j) wt[j] /= z;
        }
    }
    free(taken);
    return 0;
}

/* Margin between the k-th and (k+1)-th largest fp64 logits of each token
 * (INFINITY when k == E). Tokens with a tiny margin are near-ties whose
 * selection depends on summation order. */
int oracle_topk_margin(const double* logits, int T, int E, int k, double* margin) {
    if (k <= 0 || k > E) return -1;
    double* v = (double*)malloc(sizeof(double) * (size_t)(k + 1));
    if (!v) return -1;
    for (int t = 0; t < T; ++t) {
        if (k == E) { margin[t] = INFINITY; continue; }
        const double* l = logits + (size_t)t * E;
        /* keep the k+1 largest values in descending order (insertion) */
        int n = 0;
        for (int e = 0; e < E; ++e) {
            double x = l[e];
            if (n == k + 1 && x <= v[k]) continue;
            int p = n < k + 1 ? n++ : k;
            while (p > 0 && v[p - 1] < x) { v[p] = v[p - 1]; --p; }
            v[p] = x;
        }
        margin[t] = v[k - 1] - v[k];
    }
    free(v);
    return 0;
}

/* Grouping by expert id: a stable counting sort of the T*k assignments.
 * Assignment a = t*k + j goes to expert idx[a].
 * counts[e]    number of assignments to expert e
 * offsets[e]   exclusive prefix sum of counts; offsets[E] = T*k
 * perm_src[r]  token of the assignment placed at row r (rows sorted by expert,
 *              then by a)
 * inv_perm[a]  row at which assignment a is placed
 * Returns 0, or -1 if an index is out of range. */
int oracle_permute(const int32_t* idx, int T, int E, int k, int32_t* counts, int32_t* offsets, int32_t* perm_src,
                   int32_t* inv_perm) {
    long R = (long)T * k;
    for (int e = 0; e < E; ++e) counts[e] = 0;
    for (long a = 0; a < R; ++a) {
        if (idx[a] < 0 || idx[a] >= E) return -1;
        counts[idx[a]]++;
    }
    offsets[0] = 0;
    for (int e = 0; e < E; ++e) offsets[e + 1] = offsets[e] + counts[e];
    int32_t* cursor = (int32_t*)malloc(sizeof(int32_t) * (size_t)(E > 0 ? E : 1));
    if (!cursor) return -1;
    for (int e = 0; e < E; ++e) cursor[e] = offsets[e];
    for (long a = 0; a < R; ++a) {
        int32_t r = cursor[idx[a]]++;
        perm_src[r] = (int32_t)(a / k);
        inv_perm[a] = r;
    }
    free(cursor);
    return 0;
}

/* ---- expert MLP + weighted combine, per token -------------------------------------------------- */

typedef struct {
    const uint16_t* x;
    int T, d, f, E, k, fs;
    const uint16_t* const* wgu; /* E pointers to [2f][d] (NULL where not needed) */
    const uint16_t* const* wd;  /* E pointers to [d][f] */
    const int32_t* idx;
    const double* w;
    const uint16_t* wgu_s; /* shared expert [2fs][d] or NULL */
    const uint16_t* wd_s;  /* shared expert [d][fs] or NULL */
    const int32_t* tokens;
    int n_tokens;
    double* out;
    int first, last;
    int status;
} tok_job_t;

/* acc[c] += scale * sum_n h[n] * Wd[c][n], h[n] = silu(g[n]) * u[n],
 * g[n] = sum_i x[i] Wgu[n][i], u[n] = sum_i x[i] Wgu[f+n][i]. */
static void swiglu_expert(const uint16_t* xt, int d, int f, const uint16_t* wgu, const uint16_t* wd, double scale,
                          double* h, double* acc) {
    for (int n = 0; n < f; ++n) {
        const uint16_t* gr = wgu + (size_t)n * d;
        const uint16_t* ur = wgu + (size_t)(f + n) * d;
        double g = 0.0, u = 0.0;
        for (int i = 0; i < d; ++i) {
            double xi = bf16_to_double(xt[i]);
            g += xi * bf16_to_double(gr[i]);
            u += xi * bf16_to_double(ur[i]);
        }
        h[n] = g / (1.0 + exp(-g)) * u;
    }
    for (int c = 0; c < d; ++c) {
        const uint16_t* dr = wd + (size_t)c * f;
        double s = 0.0;
        for (int n = 0; n < f; ++n) s += h[n] * bf16_to_double(dr[n]);
        acc[c] += scale * s;
    }
}

static void* tok_worker(void* p) {
    tok_job_t* J = (tok_job_t*)p;
    int hf = J->f > J->fs ? J->f : J->fs;
    double* h = (double*)malloc(sizeof(double) * (size_t)(hf > 0 ? hf : 1));
    if (!h) { J->status = -1; return NULL; }
    for (int q = J->first; q < J->last; ++q) {
        int t = J->tokens[q];
        const uint16_t* xt = J->x + (size_t)t * J->d;
        double* acc = J->out + (size_t)q * J->d;
        for (int c = 0; c < J->d; ++c) acc[c] = 0.0;
        for (int j = 0; j < J->k; ++j) {
            int e = J->idx[(size_t)t * J->k + j];
            if (e < 0 || e >= J->E || !J->wgu[e] || !J->wd[e]) { J->status = -2; free(h); return NULL; }
            swiglu_expert(xt, J->d, J->f, J->wgu[e], J->wd[e], J->w[(size_t)t * J->k + j], h, acc);
        }
        if (J->wgu_s && J->wd_s) swiglu_expert(xt, J->d, J->fs, J->wgu_s, J->wd_s, 1.0, h, acc);
    }
    free(h);
    return NULL;
}

/* out[q][c] for the listed tokens q: sum over the token's selected experts of
 * w * down(silu(gate) * up), plus the shared expert (weight 1) when given.
 * wgu/wd are arrays of E per-expert pointers; only the experts the listed
 * tokens select must be non-NULL. Runs on nthreads threads (tokens split into
 * contiguous chunks). Returns 0, -1 on allocation failure, -2 on a missing
 * expert or bad index. */
int oracle_moe_tokens(const uint16_t* x, int T, int d, int f, int E, int k, const uint16_t* const* wgu,
                      const uint16_t* const* wd, const int32_t* idx, const double* w, const uint16_t* wgu_shared,
                      const uint16_t* wd_shared, int f_shared, const int32_t* tokens, int n_tokens, double* out,
                      int nthreads) {
    if (nthreads < 1) nthreads = 1;
    if (nthreads > n_tokens) nthreads = n_tokens > 0 ? n_tokens : 1;
    if (nthreads > 512) nthreads = 512;
    for (int q = 0; q < n_tokens; ++q)
        if (tokens[q] < 0 || tokens[q] >= T) return -2;
    tok_job_t* jobs = (tok_job_t*)calloc((size_t)nthreads, sizeof(tok_job_t));
    pthread_t* th = (pthread_t*)calloc((size_t)nthreads, sizeof(pthread_t));
    char* started = (char*)calloc((size_t)nthreads, 1);
    if (!jobs || !th || !started) { free(jobs); free(th); free(started); return -1; }
    int per = (n_tokens + nthreads - 1) / nthreads;
    for (int i = 0; i < nthreads; ++i) {
        tok_job_t* J = &jobs[i];
        J->x = x; J->T = T; J->d = d; J->f = f; J->E = E; J->k = k;
        J->fs = (wgu_shared && wd_shared) ? f_shared : 0;
        J->wgu = wgu; J->wd = wd; J->idx = idx; J->w = w;
        J->wgu_s = wgu_shared; J->wd_s = wd_shared;
        J->tokens = tokens; J->n_tokens = n_tokens; J->out = out;
        J->first = i * per;
        J->last = (i + 1) * per < n_tokens ? (i + 1) * per : n_tokens;
        if (J->first >= J->last) continue;
        if (nthreads == 1 || pthread_create(&th[i], NULL, tok_worker, J) != 0)
            tok_worker(J);
        else
            started[i] = 1;
    }
    int status = 0;
    for (int i = 0; i < nthreads; ++i) {
        if (started[i]) pthread_join(th[i], NULL);
        if (jobs[i].status) status = jobs[i].status;
    }
    free(jobs); free(th); free(started);
    return status;
}

/*
 * MXFP4 expert weights. The blog post's section "From Dense to Sparse: What Are MoEs?" estimates gpt-oss-20b's
 * generation speed as memory bandwidth over the bytes of its active parameters, and notes that kernels for the
 * model's native mxfp4 quantization would be faster still: fewer bytes per weight. The format is the OCP
 * Microscaling Formats (MX) v1.0 one: blocks of 32 consecutive elements along the reduction axis share one
 * E8M0 scale (an 8-bit power-of-two exponent, bias 127), and each element is an FP4 E2M1 code (sign bit, two
 * exponent bits with bias 1, one mantissa bit; exponent field 0 holds the subnormals 0 and 0.5).
 *
 * Readings taken where the specification leaves a choice open:
 *   - a block whose elements are all zero gets scale code 0 (its codes are all zero whatever the scale);
 *   - the shared exponent is clamped to the E8M0 range [-127, 127]; code 255 (NaN) is never written;
 *   - the sign bit of every code is the sign bit of the input, also when the magnitude rounds to 0;
 *   - inputs must be finite.
 * Memory layout (this library's, the specification fixes none): codes [G][N][K/2] bytes, each little-endian
 * 32-bit word holding 8 consecutive elements k0..k0+7 of one row, nibble i (bits 4i..4i+3) being element
 * k0+2i for i < 4 and element k0+2(i-4)+1 for i >= 4 (even elements in the low half, odd ones in the high
 * half); scales [G][K/32][N] bytes (the scale of row n's block b at [g][b][n]).
 */

/* Value of an FP4 E2M1 code, from the element format's definition. */
double oracle_e2m1_value(int code) {
    const int sign = (code >> 3) & 1, e = (code >> 1) & 3, m = code & 1;
    const double mag = e == 0 ? 0.5 * m : ldexp(1.0 + 0.5 * m, e - 1);
    return sign ? -mag : mag;
}

/* Nearest E2M1 magnitude code (0..7) to p >= 0, ties to the code with mantissa bit 0 (round to nearest even);
   beyond the largest magnitude (6) the nearest is 6, which is the clamp the conversion asks for. */
static int e2m1_nearest(double p) {
    int best = 0;
    double bestd = fabs(p - oracle_e2m1_value(0));
    for (int c = 1; c < 8; ++c) {
        const double dist = fabs(p - oracle_e2m1_value(c));
        if (dist < bestd || (dist == bestd && (c & 1) == 0 && (best & 1) == 1)) {
            best = c;
            bestd = dist;
        }
    }
    return best;
}

/* Rows [first, last) of a [G*N][K] weight tensor, shared by the threads that encode or decode it. */
typedef struct {
    const uint16_t* w;
    uint16_t* w_out;
    const uint8_t* qin;
    const uint8_t* sin;
    uint8_t* q;
    uint8_t* s;
    int N, K;
    long first, last;
    int status;
} mx_job_t;

static void* mx_quantize_rows(void* p) {
    mx_job_t* J = (mx_job_t*)p;
    const int N = J->N, K = J->K, nb = K / 32;
    for (long row = J->first; row < J->last; ++row) {
        const long g = row / N, n = row % N;
        for (int b = 0; b < nb; ++b) {
            const uint16_t* v = J->w + (size_t)row * K + (size_t)b * 32;
            double amax = 0.0;
            for (int i = 0; i < 32; ++i) amax = fmax(amax, fabs(bf16_to_double(v[i])));
            int shared = -127;
            if (amax > 0.0) {
                int ex;
                frexp(amax, &ex); /* amax = m * 2^ex, m in [0.5, 1): floor(log2(amax)) = ex - 1 */
                shared = ex - 1 - 2;
                if (shared < -127) shared = -127;
                if (shared > 127) shared = 127;
            }
            int code[32];
            for (int i = 0; i < 32; ++i) {
                const double p = fabs(bf16_to_double(v[i])) / ldexp(1.0, shared);
                code[i] = e2m1_nearest(p) | ((v[i] >> 15) ? 8 : 0);
            }
            uint8_t* out = J->q + (size_t)row * (size_t)(K / 2) + (size_t)b * 16;
            for (int j = 0; j < 4; ++j) {
                uint32_t word = 0;
                for (int i = 0; i < 4; ++i) {
                    word |= (uint32_t)code[8 * j + 2 * i] << (4 * i);
                    word |= (uint32_t)code[8 * j + 2 * i + 1] << (16 + 4 * i);
                }
                for (int byte = 0; byte < 4; ++byte) out[4 * j + byte] = (uint8_t)(word >> (8 * byte));
            }
            J->s[((size_t)g * nb + b) * N + n] = (uint8_t)(shared + 127);
        }
    }
    return NULL;
}

static void* mx_dequantize_rows(void* p) {
    mx_job_t* J = (mx_job_t*)p;
    const int N = J->N, K = J->K, nb = K / 32;
    for (long row = J->first; row < J->last; ++row) {
        const long g = row / N, n = row % N;
        for (int k = 0; k < K; ++k) {
            const int b = k / 32, j = (k % 32) / 8, e = k % 8;
            const uint8_t* blk = J->qin + (size_t)row * (size_t)(K / 2) + (size_t)b * 16 + 4 * j;
            const uint32_t word = (uint32_t)blk[0] | ((uint32_t)blk[1] << 8) | ((uint32_t)blk[2] << 16) |
                                  ((uint32_t)blk[3] << 24);
            const int nib = (e % 2 == 0) ? e / 2 : 4 + e / 2;
            const int code = (int)((word >> (4 * nib)) & 15u);
            const int sc = J->sin[((size_t)g * nb + b) * N + n];
            if (sc == 255) { J->status = -1; return NULL; }
            const double val = oracle_e2m1_value(code) * ldexp(1.0, sc - 127);
            const float fv = (float)val;
            if ((double)fv != val || isinf(fv)) { J->status = -1; return NULL; }
            uint32_t u;
            memcpy(&u, &fv, 4);
            if (u & 0xFFFFu) { J->status = -1; return NULL; }
            J->w_out[(size_t)row * K + k] = (uint16_t)(u >> 16);
        }
    }
    return NULL;
}

/* Split rows over host threads (the arithmetic per row is the same whatever the split). */
static int mx_run(void* (*fn)(void*), mx_job_t proto, long rows, int nthreads) {
    if (nthreads < 1) nthreads = 1;
    if (nthreads > 256) nthreads = 256;
    if (nthreads > rows) nthreads = rows > 0 ? (int)rows : 1;
    mx_job_t jobs[256];
    pthread_t th[256];
    char started[256];
    const long per = (rows + nthreads - 1) / nthreads;
    for (int i = 0; i < nthreads; ++i) {
        jobs[i] = proto;
        jobs[i].first = i * per;
        jobs[i].last = (i + 1) * per < rows ? (i + 1) * per : rows;
        jobs[i].status = 0;
        started[i] = 0;
        if (jobs[i].first >= jobs[i].last) continue;
        if (nthreads == 1 || pthread_create(&th[i], NULL, fn, &jobs[i]) != 0)
            fn(&jobs[i]);
        else
            started[i] = 1;
    }
    int status = 0;
    for (int i = 0; i < nthreads; ++i) {
        if (started[i]) pthread_join(th[i], NULL);
        if (jobs[i].status) status = jobs[i].status;
    }
    return status;
}

/* w [G][N][K] bf16 -> codes q [G][N][K/2], scales s [G][K/32][N]. Per block of 32: the shared exponent is
   floor(log2(max |v|)) minus 2 (the exponent of E2M1's largest magnitude, 6 = 1.5 * 2^2), each element is
   v / 2^shared rounded to the nearest E2M1 value. Returns 0, or -1 when K is not a multiple of 32. */
int oracle_mxfp4_quantize(const uint16_t* w, int G, int N, int K, uint8_t* q, uint8_t* s, int nthreads) {
    if (K % 32 != 0 || G < 0 || N < 0) return -1;
    mx_job_t J = {0};
    J.w = w; J.q = q; J.s = s; J.N = N; J.K = K;
    return mx_run(mx_quantize_rows, J, (long)G * N, nthreads);
}

/* Codes and scales -> the weights they encode, as bf16 bits: code value * 2^(scale - 127). Every such value
   with scale <= 252 is exactly a bf16 number; returns -1 for a value that is not (overflow, scale 255),
   -2 for a bad K. */
int oracle_mxfp4_dequantize(const uint8_t* q, const uint8_t* s, int G, int N, int K, uint16_t* w, int nthreads) {
    if (K % 32 != 0 || G < 0 || N < 0) return -2;
    mx_job_t J = {0};
    J.qin = q; J.sin = s; J.w_out = w; J.N = N; J.K = K;
    return mx_run(mx_dequantize_rows, J, (long)G * N, nthreads);
}

/*
 * Backward pass (training). The blog post's section "Training MoEs with Transformers" trains through the same
 * grouped_mm expert backend; the gradients below are those of the per-token eager loop above, differentiated by
 * hand, in fp64. Given dy[t] = d loss / d out[t]:
 *   for each selected expert e of token t, routing weight w_tj:
 *     g = Wg x, u = Wu x, a = silu(g), h = a * u, y_e = Wd h
 *     dw[t][j]      = <dy[t], y_e>
 *     dye           = w_tj * dy[t]
 *     dh[n]         = sum_c dye[c] * Wd[c][n]
 *     dWd[e][c][n] += dye[c] * h[n]
 *     dg[n]         = dh[n] * u[n] * silu'(g[n]),  silu'(g) = s * (1 + g * (1 - s)),  s = 1 / (1 + e^-g)
 *     du[n]         = dh[n] * a[n]
 *     dx[t][i]     += sum_n dg[n] * Wg[n][i] + du[n] * Wu[n][i]
 *     dWg[e][n][i] += dg[n] * x[i];  dWu[e][n][i] += du[n] * x[i]
 *   the shared expert the same with weight 1 and no routing-weight gradient.
 * Single-threaded (weight gradients accumulate over tokens); meant for small problems.
 */
static void swiglu_expert_backward(const uint16_t* xt, int d, int f, const uint16_t* wgu, const uint16_t* wd,
                                   double scale, const double* dyt, double* dxt, double* dwgu, double* dwd,
                                   double* dwt, double* g, double* u, double* h, double* dh) {
    for (int n = 0; n < f; ++n) {
        const uint16_t* gr = wgu + (size_t)n * d;
        const uint16_t* ur = wgu + (size_t)(f + n) * d;
        double gs = 0.0, us = 0.0;
        for (int i = 0; i < d; ++i) {
            const double xi = bf16_to_double(xt[i]);
            gs += xi * bf16_to_double(gr[i]);
            us += xi * bf16_to_double(ur[i]);
        }
        g[n] = gs;
        u[n] = us;
        h[n] = gs / (1.0 + exp(-gs)) * us;
    }
    if (dwt) { /* <dy, y_e>, y_e = Wd h */
        double s = 0.0;
        for (int c = 0; c < d; ++c) {
            const uint16_t* dr = wd + (size_t)c * f;
            double yc = 0.0;
            for (int n = 0; n < f; ++n) yc += bf16_to_double(dr[n]) * h[n];
            s += dyt[c] * yc;
        }
        *dwt = s;
    }
    for (int n = 0; n < f; ++n) dh[n] = 0.0;
    for (int c = 0; c < d; ++c) {
        const uint16_t* dr = wd + (size_t)c * f;
        const double dyc = scale * dyt[c];
        for (int n = 0; n < f; ++n) {
            dh[n] += dyc * bf16_to_double(dr[n]);
            if (dwd) dwd[(size_t)c * f + n] += dyc * h[n];
        }
    }
    for (int n = 0; n < f; ++n) {
        const double s = 1.0 / (1.0 + exp(-g[n]));
        const double a = g[n] * s;
        const double dg = dh[n] * u[n] * (s * (1.0 + g[n] * (1.0 - s)));
        const double du = dh[n] * a;
        const uint16_t* gr = wgu + (size_t)n * d;
        const uint16_t* ur = wgu + (size_t)(f + n) * d;
        double* dgr = dwgu ? dwgu + (size_t)n * d : NULL;
        double* dur = dwgu ? dwgu + (size_t)(f + n) * d : NULL;
        for (int i = 0; i < d; ++i) {
            const double xi = bf16_to_double(xt[i]);
            dxt[i] += dg * bf16_to_double(gr[i]) + du * bf16_to_double(ur[i]);
            if (dgr) {
                dgr[i] += dg * xi;
                dur[i] += du * xi;
            }
        }
    }
}

/* dx [T][d], dwgu: E pointers to [2f][d], dwd: E pointers to [d][f] (all fp64, zeroed here; NULL pointers for
   experts no token selects; dwgu and dwd themselves NULL when no weight gradient is wanted), dw [T][k];
   shared-expert gradients dwgu_s [2fs][d], dwd_s [d][fs] when given. Returns 0, -1 on a bad argument or
   allocation failure, -2 when a selected expert has no weights (or no gradient arrays, when they are wanted). */
int oracle_moe_backward(const uint16_t* x, int T, int d, int f, int E, int k, const uint16_t* const* wgu,
                        const uint16_t* const* wd, const int32_t* idx, const double* w, const double* dy,
                        const uint16_t* wgu_s, const uint16_t* wd_s, int fs, double* dx, double* const* dwgu,
                        double* const* dwd, double* dw, double* dwgu_s, double* dwd_s) {
    if (T < 0 || d <= 0 || f <= 0 || E <= 0 || k <= 0 || k > E) return -1;
    const int hf = f > fs ? f : fs;
    double* g = (double*)malloc(sizeof(double) * (size_t)hf);
    double* u = (double*)malloc(sizeof(double) * (size_t)hf);
    double* h = (double*)malloc(sizeof(double) * (size_t)hf);
    double* dh = (double*)malloc(sizeof(double) * (size_t)hf);
    if (!g || !u || !h || !dh) { free(g); free(u); free(h); free(dh); return -1; }
    memset(dx, 0, sizeof(double) * (size_t)T * d);
    const int wgrad = dwgu != NULL && dwd != NULL;
    if (wgrad)
        for (int e = 0; e < E; ++e) {
            if (dwgu[e]) memset(dwgu[e], 0, sizeof(double) * (size_t)2 * f * d);
            if (dwd[e]) memset(dwd[e], 0, sizeof(double) * (size_t)d * f);
        }
    const int shared = wgu_s && wd_s && fs > 0;
    if (shared && dwgu_s && dwd_s) {
        memset(dwgu_s, 0, sizeof(double) * (size_t)2 * fs * d);
        memset(dwd_s, 0, sizeof(double) * (size_t)d * fs);
    }
    int status = 0;
    for (int t = 0; t < T && !status; ++t) {
        const uint16_t* xt = x + (size_t)t * d;
        const double* dyt = dy + (size_t)t * d;
        double* dxt = dx + (size_t)t * d;
        for (int j = 0; j < k; ++j) {
            const int e = idx[(size_t)t * k + j];
            if (e < 0 || e >= E || !wgu[e] || !wd[e] || (wgrad && (!dwgu[e] || !dwd[e]))) { status = -2; break; }
            swiglu_expert_backward(xt, d, f, wgu[e], wd[e], w[(size_t)t * k + j], dyt, dxt,
                                   wgrad ? dwgu[e] : NULL, wgrad ? dwd[e] : NULL, &dw[(size_t)t * k + j], g, u, h, dh);
        }
        if (shared && !status)
            swiglu_expert_backward(xt, d, fs, wgu_s, wd_s, 1.0, dyt, dxt, dwgu_s, dwd_s, NULL, g, u, h, dh);
    }
    free(g); free(u); free(h); free(dh);
    return status;
}

/* Router backward, the selection held fixed (top-k is piecewise constant in the logits, so no gradient flows
   through it). From dw[t][j] = d loss / d w[t][j], with the weights w the forward computed from the fp32 logits:
     top-k softmax and softmax -> top-k -> renorm (the same function of the selected logits):
         dl[t][e_j] = w_j * (dw_j - sum_i w_i dw_i)
     sigmoid -> top-k -> norm, s_j = sigmoid(l_j), S = sum_i s_i:
         dl[t][e_j] = s_j * (1 - s_j) / S * (dw_j - sum_i w_i dw_i)
     unselected experts: 0.
   Then through l = x W_r^T + b: dW_r[e][i] = sum_t dl[t][e] x[t][i], dbias[e] = sum_t dl[t][e],
   dx[t][i] = sum_e dl[t][e] W_r[e][i]. Outputs fp64, zeroed here. */
int oracle_router_backward(const uint16_t* x, const float* w_router, const float* logits, int T, int d, int E, int k,
                           int mode, const int32_t* idx, const double* w, const double* dw, double* dlogits,
                           double* dw_router, double* dbias, double* dx) {
    if (T < 0 || d <= 0 || E <= 0 || k <= 0 || k > E || mode < 0 || mode > 2) return -1;
    memset(dlogits, 0, sizeof(double) * (size_t)T * E);
    memset(dw_router, 0, sizeof(double) * (size_t)E * d);
    memset(dbias, 0, sizeof(double) * (size_t)E);
    memset(dx, 0, sizeof(double) * (size_t)T * d);
    for (int t = 0; t < T; ++t) {
        const int32_t* it = idx + (size_t)t * k;
        const double* wt = w + (size_t)t * k;
        const double* dwt = dw + (size_t)t * k;
        double dot = 0.0;
        for (int j = 0; j < k; ++j) dot += wt[j] * dwt[j];
        double S = 0.0;
        if (mode == ORACLE_SIGMOID_TOPK_NORM)
            for (int j = 0; j < k; ++j) S += 1.0 / (1.0 + exp(-(double)logits[(size_t)t * E + it[j]]));
        for (int j = 0; j < k; ++j) {
            const int e = it[j];
            if (e < 0 || e >= E) return -2;
            double g;
            if (mode == ORACLE_SIGMOID_TOPK_NORM) {
                const double s = 1.0 / (1.0 + exp(-(double)logits[(size_t)t * E + e]));
                g = s * (1.0 - s) / S * (dwt[j] - dot);
            } else {
                g = wt[j] * (dwt[j] - dot);
            }
            dlogits[(size_t)t * E + e] = g;
        }
        for (int e = 0; e < E; ++e) {
            const double g = dlogits[(size_t)t * E + e];
            if (g == 0.0) continue;
            dbias[e] += g;
            for (int i = 0; i < d; ++i) {
                dw_router[(size_t)e * d + i] += g * bf16_to_double(x[(size_t)t * d + i]);
                dx[(size_t)t * d + i] += g * (double)w_router[(size_t)e * d + i];
            }
        }
    }
    return 0;
}

/* Selected entries of one expert's weight gradients, summed over every (token, slot) that selects expert e: the
   sums oracle_moe_backward accumulates, restricted to the asked entries so that full-size layers stay cheap.
     kind 0 (down):    out[q] = dWd[a[q]][b[q]] = sum w_tj * dy[t][c] * h_t[n],          c = a[q], n = b[q]
     kind 1 (gate|up): out[q] = dWgu[a[q]][b[q]], row m = a[q] in [0, 2f), column i = b[q]:
                       sum dg_t[m] * x_t[i] for m < f,  sum du_t[m - f] * x_t[i] for m >= f
   with h, dg, du as in oracle_moe_backward. Returns 0, or -1 on a bad argument or allocation failure. */
int oracle_weight_grad_entries(const uint16_t* x, int T, int d, int f, int k, const uint16_t* wgu, const uint16_t* wd,
                               int e, const int32_t* idx, const double* w, const double* dy, int kind,
                               const int32_t* a, const int32_t* b, int n_entries, double* out) {
    if (T < 0 || d <= 0 || f <= 0 || k <= 0 || (kind != 0 && kind != 1)) return -1;
    for (int q = 0; q < n_entries; ++q) {
        if (kind == 0 && (a[q] < 0 || a[q] >= d || b[q] < 0 || b[q] >= f)) return -1;
        if (kind == 1 && (a[q] < 0 || a[q] >= 2 * f || b[q] < 0 || b[q] >= d)) return -1;
        out[q] = 0.0;
    }
    double* g = (double*)malloc(sizeof(double) * (size_t)f);
    double* u = (double*)malloc(sizeof(double) * (size_t)f);
    double* h = (double*)malloc(sizeof(double) * (size_t)f);
    double* dh = (double*)malloc(sizeof(double) * (size_t)f);
    if (!g || !u || !h || !dh) { free(g); free(u); free(h); free(dh); return -1; }
    for (int t = 0; t < T; ++t)
        for (int j = 0; j < k; ++j) {
            if (idx[(size_t)t * k + j] != e) continue;
            const uint16_t* xt = x + (size_t)t * d;
            const double wt = w[(size_t)t * k + j];
            const double* dyt = dy + (size_t)t * d;
            for (int n = 0; n < f; ++n) {
                double gs = 0.0, us = 0.0;
                for (int i = 0; i < d; ++i) {
                    const double xi = bf16_to_double(xt[i]);
                    gs += xi * bf16_to_double(wgu[(size_t)n * d + i]);
                    us += xi * bf16_to_double(wgu[(size_t)(f + n) * d + i]);
                }
                g[n] = gs;
                u[n] = us;
                h[n] = gs / (1.0 + exp(-gs)) * us;
            }
            if (kind == 0) {
                for (int q = 0; q < n_entries; ++q) out[q] += wt * dyt[a[q]] * h[b[q]];
                continue;
            }
            for (int n = 0; n < f; ++n) {
                double s = 0.0;
                for (int c = 0; c < d; ++c) s += wt * dyt[c] * bf16_to_double(wd[(size_t)c * f + n]);
                dh[n] = s;
            }
            for (int q = 0; q < n_entries; ++q) {
                const int m = a[q], i = b[q];
                const int n = m < f ? m : m - f;
                const double sg = 1.0 / (1.0 + exp(-g[n]));
                const double coef = m < f ? dh[n] * u[n] * (sg * (1.0 + g[n] * (1.0 - sg))) : dh[n] * g[n] * sg;
                out[q] += coef * bf16_to_double(xt[i]);
            }
        }
    free(g); free(u); free(h); free(dh);
    return 0;
}
