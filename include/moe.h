/*
 * moe.h — C-ABI of the B200 (sm_100a) sparse mixture-of-experts feed-forward layer.
 *
 * The layer replaces a dense feed-forward block by E expert networks and a
 * router that sends each token to a small subset of them (blog post "Mixture
 * of Experts (MoEs) in Transformers", section "From Dense to Sparse"). At run
 * time it must dispatch tokens to their selected experts, run the expert
 * projections, apply the routing weights and collect the results back in
 * token order (same post, section "Expert Backend"). This library does it the
 * grouped_mm way described there: sort tokens by expert id, group them, and
 * run one grouped GEMM over all experts. One layer call is:
 *
 *   moe_route_topk          logits, top-k expert ids and routing weights
 *   moe_permute             expert histogram, exclusive scan, stable scatter,
 *                           gather of x rows into expert-contiguous order
 *   moe_grouped_gemm_gateup h = silu(x_perm Wg^T) * (x_perm Wu^T), per expert
 *                           (moe_grouped_gemm_gateup_gather: the same with
 *                           the gather folded into the GEMM's operand load)
 *   moe_grouped_gemm_down   y_perm = h Wd^T, per expert
 *   moe_unpermute_combine   y[t] = sum_j w[t,j] * y_perm[row of (t,j)] (+ shared[t])
 *                           (moe_grouped_gemm_down_combine: down and combine
 *                           in one call, the combine in the GEMM's epilogue)
 *
 * With MXFP4 expert weights (encoded once by moe_mxfp4_quantize) the two
 * grouped GEMMs are moe_grouped_gemm_gateup_mxfp4 / moe_grouped_gemm_down_mxfp4.
 *
 * Conventions (all entry points):
 *  - Every pointer argument is a DEVICE pointer to memory the caller allocated
 *    and owns, unless stated otherwise. The library allocates no device memory
 *    and frees nothing; it holds no state besides per-device attributes it
 *    caches (SM count, kernel attributes) and a device-side error word.
 *  - bf16 tensors are passed as moe_bf16_t (the raw 16-bit pattern of a
 *    bfloat16). All tensors are dense and row-major (last index fastest).
 *  - Pointers must be 16-byte aligned. d and f must be multiples of 8 (rows of
 *    bf16 then start on 16-byte boundaries, as the TMA engine requires).
 *  - Calls are asynchronous on `stream`. They never synchronise and never
 *    read device memory from the host, except moe_get_device_error().
 *  - Argument errors are reported before anything is launched (outputs are
 *    left untouched): MOE_ERR_INVALID_ARG. A launch failure returns
 *    MOE_ERR_CUDA; moe_last_error_string() describes it.
 *  - Anomalies found on the device (an expert id or a group offset out of
 *    range, a pipeline wait that timed out) never fault: the kernel skips the
 *    offending access, sets a bit in a device error word and returns. Read and
 *    clear it with moe_get_device_error().
 *  - Integer sizes are int; T*k, T*d and T*E must fit in int32, group row
 *    counts M in int32.
 */
#ifndef MOE_H
#define MOE_H

#include <stddef.h>
#include <stdint.h>
#include <cuda_runtime_api.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef uint16_t moe_bf16_t;

typedef enum {
    MOE_OK = 0,
    MOE_ERR_INVALID_ARG = 1, /* null/misaligned pointer, bad size, k > E, unsupported mode */
    MOE_ERR_UNSUPPORTED = 2, /* current device is not sm_100 */
    MOE_ERR_WORKSPACE = 3,   /* workspace missing or smaller than the *_workspace_size() figure */
    MOE_ERR_CUDA = 4,        /* a CUDA call or launch failed; see moe_last_error_string() */
    MOE_ERR_DEVICE = 5       /* returned by moe_get_device_error() when the error word was set */
} moe_status_t;

/* Empty problems: a call with T = 0 (router, top-k, permute, combine) or
 * M = 0 (grouped GEMMs) launches nothing and returns MOE_OK once its sizes
 * check out; pointers to arrays that are then empty may be NULL. moe_permute
 * still writes its [E] counts and [E+1] offsets (all zero). */

/* Bits of the device error word. */
#define MOE_DEVERR_WAIT_TIMEOUT 0x1u  /* a pipeline wait in a GEMM gave up after its time limit */
#define MOE_DEVERR_EXPERT_RANGE 0x2u  /* an expert id outside [0, E) reached moe_permute */
#define MOE_DEVERR_GROUP_RANGE 0x4u   /* group offsets not non-decreasing within [0, M] */
#define MOE_DEVERR_ROW_RANGE 0x8u     /* a permutation entry outside its range */

/* Routing weight modes. Selection is always the k largest logits in
 * descending order, the lower expert id first on ties. Weights of the k
 * selected experts of a token:
 *   MOE_ROUTE_TOPK_SOFTMAX         softmax over the k selected logits
 *   MOE_ROUTE_SOFTMAX_TOPK_RENORM  softmax over all E logits, keep the k
 *                                  selected probabilities, divide by their sum
 *   MOE_ROUTE_SIGMOID_TOPK_NORM    sigmoid of each selected logit, divided by
 *                                  the sum of the k sigmoids
 * The blog post names the router but not its formula ("From Dense to Sparse");
 * these are the three variants used by the model families it lists. */
typedef enum {
    MOE_ROUTE_TOPK_SOFTMAX = 0,
    MOE_ROUTE_SOFTMAX_TOPK_RENORM = 1,
    MOE_ROUTE_SIGMOID_TOPK_NORM = 2
} moe_route_mode_t;

/* Router: logits[t][e] = sum_i x[t][i] * w_router[e][i] + bias[e] in fp32,
 * then top-k selection and routing weights (section "From Dense to Sparse":
 * "a router selects a small subset of experts" per token).
 *   x          [T][d] bf16
 *   w_router   [E][d] fp32
 *   bias       [E] fp32, or NULL for none (added before selection and weights)
 *   logits_out [T][E] fp32, written (required: the selection reads it back)
 *   topk_idx   [T][k] int32, expert ids, descending logit order
 *   topk_w     [T][k] fp32, routing weights per `mode`
 * Limits: 1 <= E <= 1024, 1 <= k <= min(E, 32), T >= 0 (T == 0 launches
 * nothing). */
moe_status_t moe_route_topk(const moe_bf16_t* x, const float* w_router, const float* bias, int T, int d, int E,
                            int k, moe_route_mode_t mode, float* logits_out, int32_t* topk_idx, float* topk_w,
                            cudaStream_t stream);

/* The router's fp32 weights as three bf16 pieces, written once and then
 * reused by moe_route_topk_split: w = hi + mid + lo with hi = w truncated to
 * bf16, mid = (w - hi) truncated, lo = bf16(w - hi - mid) rounded to nearest
 * (the tensor-core router multiplies x by the three pieces, carrying ~24
 * bits of w). Router weights do not change between forward calls, so the
 * split belongs with loading them (the blog post converts checkpoint
 * tensors into the layout its kernels want at load time: "Dynamic Weight
 * Loading with WeightConverter").
 *   w_router  [E][d] fp32
 *   w_pieces  [3][E][d] bf16, written: plane 0 hi, 1 mid, 2 lo
 * Limits: 1 <= E <= 1024, d >= 8 a multiple of 8. */
moe_status_t moe_router_split_weights(const float* w_router, int E, int d, moe_bf16_t* w_pieces,
                                      cudaStream_t stream);

/* moe_route_topk with the pieces written by moe_router_split_weights for
 * this w_router: the same results, bit for bit, without re-splitting W_r in
 * every call (the tensor-core router loads the pieces by TMA). w_router is
 * still read where the router runs on CUDA cores (T < 2048 or E > 128).
 * Arguments and limits otherwise as moe_route_topk; w_pieces must not be
 * NULL. */
moe_status_t moe_route_topk_split(const moe_bf16_t* x, const float* w_router, const moe_bf16_t* w_pieces,
                                  const float* bias, int T, int d, int E, int k, moe_route_mode_t mode,
                                  float* logits_out, int32_t* topk_idx, float* topk_w, cudaStream_t stream);

/* Top-k selection and routing weights from given fp32 logits [T][E] (bias, if
 * any, already included). Same outputs and limits as moe_route_topk. */
moe_status_t moe_topk_from_logits(const float* logits, int T, int E, int k, moe_route_mode_t mode,
                                  int32_t* topk_idx, float* topk_w, cudaStream_t stream);

/* Bytes of device workspace moe_permute needs for these sizes (a multiple of
 * 256; 0 when T*k == 0). */
size_t moe_permute_workspace_size(int T, int E, int k);

/* Group the T*k (token, slot) assignments by expert: "sort tokens by expert
 * ID, group them" (section "Expert Backend", grouped_mm). Assignment a = t*k+j
 * goes to expert topk_idx[a]. The sort is stable: rows of one expert keep
 * increasing a, so the result is unique and deterministic.
 *   expert_counts  [E]   assignments per expert
 *   expert_offsets [E+1] exclusive prefix sum of counts; [E] = T*k
 *   perm_src       [T*k] token whose row sits at each grouped row
 *   inv_perm       [T*k] grouped row of assignment a
 *   x, x_perm      [T][d] and [T*k][d] bf16: x_perm[r] = x[perm_src[r]];
 *                  pass both NULL to skip the gather (then d is ignored)
 *   ws, ws_bytes   workspace of at least moe_permute_workspace_size(T,E,k)
 *                  bytes, 256-byte aligned; its contents need not be
 *                  initialised and are scratch after the call.
 * Expert ids outside [0,E) are skipped and flagged (MOE_DEVERR_EXPERT_RANGE);
 * the outputs are then incomplete. Limits: 1 <= E <= 1024,
 * 1 <= k <= min(E, 32). */
moe_status_t moe_permute(const moe_bf16_t* x, const int32_t* topk_idx, int T, int d, int E, int k,
                         int32_t* expert_counts, int32_t* expert_offsets, int32_t* perm_src, int32_t* inv_perm,
                         moe_bf16_t* x_perm, void* ws, size_t ws_bytes, cudaStream_t stream);

/* Allocation-free variant of moe_permute. The blog post has no counterpart to
 * this call; it exists for callers that cannot supply device scratch memory.
 * Some callers cannot hand this library a workspace: they reach it through a
 * fixed interface with no workspace argument and have no device allocator of
 * their own, or they must not call cudaMalloc at run time (it can block the
 * whole device, and it fails once a memory pool has reserved the device).
 * This call does exactly what moe_permute does, with the same arguments minus
 * the workspace; its scratch is a file-scope array of
 * MOE_PERMUTE_STATIC_WS_BYTES bytes inside the library, which every GPU that
 * loads the library holds until the process exits. It allocates nothing.
 *  - Sizes whose moe_permute_workspace_size(T, E, k) exceeds
 *    MOE_PERMUTE_STATIC_WS_BYTES are rejected with MOE_ERR_WORKSPACE before
 *    anything is launched (the scratch is 4 bytes per expert per block of
 *    1024 assignments: E = 128 allows up to 2,097,152 assignments T*k,
 *    E = 1024 up to 262,144).
 *  - The first call on a device looks up the array's device address (a
 *    one-time set-up per device); make that first call before capturing a
 *    stream. The address is kept for the life of the process: a device
 *    reset (cudaDeviceReset, or tearing down the primary context) is not
 *    supported while the library stays loaded.
 *  - All calls on a device share the one array. Its contents persist between
 *    calls, and each call rewrites every byte it reads before reading it, so
 *    nothing has to be cleared. Calls that can overlap on the GPU (different
 *    streams without ordering between them) race on the array and must be
 *    serialised by the caller. */
#define MOE_PERMUTE_STATIC_WS_BYTES (1u << 20)
moe_status_t moe_permute_static_ws(const moe_bf16_t* x, const int32_t* topk_idx, int T, int d, int E, int k,
                                   int32_t* expert_counts, int32_t* expert_offsets, int32_t* perm_src,
                                   int32_t* inv_perm, moe_bf16_t* x_perm, cudaStream_t stream);

/* Grouped gate|up projection with fused SwiGLU, one expert per group:
 * for every group g and row r in [group_offsets[g], group_offsets[g+1]):
 *   h[r][n] = silu(sum_i a[r][i] * w[g][n][i]) * (sum_i a[r][i] * w[g][f+n][i]),  n < f,
 * with silu(v) = v / (1 + exp(-v)), fp32 accumulation, h rounded to bf16.
 * w is the packed gate_up_proj tensor [G][2f][d]: per expert, the gate rows
 * (w1) then the up rows (w3), concatenated on dim 1 (section "Dynamic Weight
 * Loading with WeightConverter").
 *   a              [M][d] bf16 (rows grouped by expert, e.g. x_perm)
 *   group_offsets  [G+1] int32, DEVICE memory, non-decreasing, [G] <= M;
 *                  rows at or past group_offsets[G] are not written
 *   h              [M][f] bf16
 * M is the number of rows the caller allocated (T*k after moe_permute, T for
 * a shared expert with G = 1 and offsets {0, T}). Limits: 1 <= G <= 1024
 * (the other grouped GEMMs below share it), d, f >= 8, multiples of 8. */
moe_status_t moe_grouped_gemm_gateup(const moe_bf16_t* a, const moe_bf16_t* w_gateup, const int32_t* group_offsets,
                                     int G, int M, int d, int f, moe_bf16_t* h, cudaStream_t stream);

/* Bytes of workspace moe_grouped_gemm_gateup_gather needs: 0 when the groups
 * average 128 rows or more (M >= 128*G), else M*d*2 rounded up to 256. */
size_t moe_grouped_gemm_gateup_gather_workspace_size(int G, int M, int d);

/* moe_grouped_gemm_gateup with the dispatch folded in (section "Expert
 * Backend": tokens are dispatched to their experts' weights, here without a
 * grouped copy of x): row r of the GEMM's A operand is x[row_src[r]], e.g.
 * row_src = perm_src of moe_permute called with x = x_perm = NULL. Same sums
 * and the same h bits as moe_permute's gather followed by
 * moe_grouped_gemm_gateup.
 *   x        [T][d] bf16, 16-byte aligned
 *   row_src  [M] int32, DEVICE memory, entries in [0, T); an entry outside it
 *            is flagged (MOE_DEVERR_ROW_RANGE) and the h row it feeds is
 *            unspecified (no out-of-range read is made)
 *   ws       workspace of moe_grouped_gemm_gateup_gather_workspace_size(G,
 *            M, d) bytes, 16-byte aligned (may be NULL when that is 0):
 *            with fewer than 128 rows per group on average the rows are
 *            gathered there first and the GEMM runs on the copy.
 * Other arguments and limits as moe_grouped_gemm_gateup. The kernel family
 * hook (moe_set_gemm_kernel) applies only to the workspace path. */
moe_status_t moe_grouped_gemm_gateup_gather(const moe_bf16_t* x, const int32_t* row_src, int T,
                                            const moe_bf16_t* w_gateup, const int32_t* group_offsets, int G, int M,
                                            int d, int f, moe_bf16_t* h, void* ws, size_t ws_bytes,
                                            cudaStream_t stream);

/* out[r] = x[row_src[r]] for r < R: the gather of moe_permute on its own.
 *   x [T][d], out [R][d] bf16, 16-byte aligned; row_src [R] int32 in [0, T)
 *   (an entry outside it is flagged, MOE_DEVERR_ROW_RANGE, and its row
 *   zeroed). d a positive multiple of 8. */
moe_status_t moe_gather_rows(const moe_bf16_t* x, const int32_t* row_src, int T, int d, int R, moe_bf16_t* out,
                             cudaStream_t stream);

/* Grouped down projection: y[r][c] = sum_n h[r][n] * w[g][c][n] (fp32
 * accumulation, rounded to bf16) for r in group g. w is the packed down_proj
 * tensor [G][d][f] (experts' w2 stacked on dim 0, same section).
 *   h [M][f] bf16, y [M][d] bf16, group_offsets as above. */
moe_status_t moe_grouped_gemm_down(const moe_bf16_t* h, const moe_bf16_t* w_down, const int32_t* group_offsets,
                                   int G, int M, int d, int f, moe_bf16_t* y, cudaStream_t stream);

/* Bytes of workspace moe_grouped_gemm_down_combine needs: T * ceil(d/32) * 4
 * rounded up to 256 (arrival counters). */
size_t moe_grouped_gemm_down_combine_workspace_size(int T, int d);

/* moe_grouped_gemm_down followed by moe_unpermute_combine in one call, with
 * the collect step (section "Expert Backend": apply the routing weights, then
 * collect and reorder) folded into the GEMM when the groups average 128 rows
 * or more (M >= 128*G): as each tile's y_perm rows are stored, one arrival
 * per row is counted on a counter of (token, 32-column block), and the tile
 * that brings a token's k-th arrival for a block sums the token's k rows of
 * that block in slot order. Writes y_perm (as moe_grouped_gemm_down) and y (as
 * moe_unpermute_combine), with the same bits as those two calls.
 *   h, w_down, group_offsets, G, M, d, f   as moe_grouped_gemm_down; M = T*k
 *   perm_src, inv_perm  [T*k] int32 of moe_permute (one the inverse of the
 *                       other: a row of group g holds assignment a of token
 *                       perm_src[row] with inv_perm[a] = row)
 *   topk_w [T][k] fp32, shared [T][d] bf16 or NULL, y_perm [M][d], y [T][d]
 *   ws, ws_bytes        workspace of
 *                       moe_grouped_gemm_down_combine_workspace_size(T, d)
 *                       bytes, 16-byte aligned; need not be initialised
 *                       (the call clears what it uses).
 * Entries of perm_src or inv_perm out of range are flagged
 * (MOE_DEVERR_ROW_RANGE); a pair that is not mutually inverse leaves rows of
 * y unspecified. The kernel family hook (moe_set_gemm_kernel) applies only
 * when the groups are smaller (then the two calls run one after the other).
 * Limits: those of both calls. */
moe_status_t moe_grouped_gemm_down_combine(const moe_bf16_t* h, const moe_bf16_t* w_down,
                                           const int32_t* group_offsets, int G, int M, int d, int f,
                                           const int32_t* perm_src, const int32_t* inv_perm, const float* topk_w,
                                           const moe_bf16_t* shared, int T, int k, moe_bf16_t* y_perm, moe_bf16_t* y,
                                           void* ws, size_t ws_bytes, cudaStream_t stream);

/* ---- MXFP4 expert weights ----
 * The blog post's section "From Dense to Sparse: What Are MoEs?" estimates
 * generation speed as memory bandwidth over the bytes of the active
 * parameters and notes that kernels for gpt-oss's native mxfp4 quantization
 * would be faster. MXFP4 is the OCP Microscaling Formats (MX) v1.0 format:
 * along the reduction axis (K), blocks of 32 elements share one E8M0 scale
 * (value 2^(s-127)) and each element is an FP4 E2M1 code (sign bit, two
 * exponent bits with bias 1, one mantissa bit: magnitudes 0, 0.5, 1, 1.5, 2,
 * 3, 4, 6). Layout of a [G][N][K] weight tensor (this library's; the format
 * fixes no memory order):
 *   q [G][N][K/2] uint8: each little-endian 32-bit word holds 8 consecutive
 *     elements k0..k0+7 of a row; nibble i (bits 4i..4i+3) is element k0+2i
 *     for i < 4 and element k0+2(i-4)+1 for i >= 4 (even elements in the low
 *     16 bits, odd ones in the high 16 bits);
 *   s [G][K/32][N] uint8: the scale of row n's block b is s[g][b][n].
 * A gate|up tensor [G][2f][d] is encoded along d, a down tensor [G][d][f]
 * along f. */

/* Encode bf16 weights w [G][N][K] as MXFP4 codes q and scales s (layout
 * above). Per block of 32: the scale exponent is floor(log2(max |v|)) - 2
 * (2 being the exponent of E2M1's largest magnitude 6), clamped to
 * [-127, 127]; an all-zero block gets s = 0. Every v / 2^(s-127) is rounded
 * to the nearest E2M1 magnitude, ties to the one with mantissa bit 0, values
 * above 6 clamped to 6; the sign bit is w's, also for a magnitude of 0.
 * Inputs must be finite. Deterministic and exact (integer decisions only).
 *   w 16-byte aligned; q 16-byte aligned; K a positive multiple of 32;
 *   G = 0 or N = 0 is an empty no-op. */
moe_status_t moe_mxfp4_quantize(const moe_bf16_t* w, int G, int N, int K, uint8_t* q, uint8_t* s,
                                cudaStream_t stream);

/* moe_grouped_gemm_gateup with MXFP4 weights: the same h, computed with the
 * weights the codes encode (decoded exactly to bf16; bf16 products, fp32
 * accumulation, h rounded to bf16).
 *   wq_gateup [G][2f][d/2], ws_gateup [G][d/32][2f] (gate rows, then up rows,
 *   as in moe_grouped_gemm_gateup), encoded along d.
 * Built for few rows per expert (decode), where streaming the weights is the
 * cost: weight rows are the MMA's M dimension and the group's rows its N
 * dimension (16, 32 or 64 per tile, chosen from M / G); groups larger than the
 * tile are covered by several tiles, each decoding the weights again.
 * Limits: d, f positive multiples of 32; all pointers 16-byte aligned; the
 * other arguments as for moe_grouped_gemm_gateup. Scale codes above 252 are
 * not supported (the decoded weight would overflow bf16). */
moe_status_t moe_grouped_gemm_gateup_mxfp4(const moe_bf16_t* a, const uint8_t* wq_gateup, const uint8_t* ws_gateup,
                                           const int32_t* group_offsets, int G, int M, int d, int f, moe_bf16_t* h,
                                           cudaStream_t stream);

/* moe_grouped_gemm_down with MXFP4 weights wq_down [G][d][f/2],
 * ws_down [G][f/32][d] (encoded along f); limits as above. */
moe_status_t moe_grouped_gemm_down_mxfp4(const moe_bf16_t* h, const uint8_t* wq_down, const uint8_t* ws_down,
                                         const int32_t* group_offsets, int G, int M, int d, int f, moe_bf16_t* y,
                                         cudaStream_t stream);

/* Apply the routing weights and return to token order ("apply the routing
 * weights and then collect and reorder the results", section "Expert
 * Backend"): y[t][c] = sum_{j<k} topk_w[t][j] * y_perm[inv_perm[t*k+j]][c]
 * (+ shared[t][c]), summed in fp32 in slot order j, rounded to bf16. No
 * atomics: the result is deterministic.
 *   y_perm [T*k][d] bf16, inv_perm [T*k] int32, topk_w [T][k] fp32,
 *   shared [T][d] bf16 or NULL (an always-on expert added with weight 1),
 *   y [T][d] bf16 (must not alias the inputs). */
moe_status_t moe_unpermute_combine(const moe_bf16_t* y_perm, const int32_t* inv_perm, const float* topk_w,
                                   const moe_bf16_t* shared, int T, int d, int k, moe_bf16_t* y,
                                   cudaStream_t stream);

/* ---- Backward pass (training) ----
 * The blog post trains MoE layers through the same grouped expert backend
 * ("Training MoEs with Transformers"). With the top-k selection held fixed (it
 * is piecewise constant in the router logits), the gradients of one layer
 * call y = combine(down(swiglu(gateup(x_perm)))) for an upstream gradient dy:
 *   moe_permute_backward            dy_perm[r] = w[t,j] dy[t], dw[t,j] = <dy[t], y_perm[r]>
 *   moe_grouped_gemm_down           dh = dy_perm W_down[e]        (weights transposed: W_down^T [E][f][d])
 *   moe_grouped_gemm_gateup_preact  g | u of the forward, recomputed [M][2f] (or kept by a
 *                                   forward that ran moe_grouped_gemm_gateup_save)
 *   moe_swiglu_backward             dg = dh u silu'(g), du = dh silu(g)
 *   moe_grouped_gemm_down           dx_perm = [dg|du] W_gateup[e] (weights transposed: W_gateup^T [E][d][2f])
 *   moe_unpermute_combine           dx = sum over slots of dx_perm (unit weights) + the router's share
 *   moe_grouped_weight_grad         dW_down[e] = dy_perm_e^T h_e, dW_gateup[e] = [dg|du]_e^T x_perm_e
 *   moe_router_backward             dlogits, dW_r, dbias and the router's share of dx
 * Every reduction runs in a fixed order (no atomics): the results are
 * deterministic. moe_transpose_weights makes the transposed weight copies
 * once per weight update. */

/* Pre-activations of the gate|up projection: gu[r][n] = sum_i a[r][i] w[g][n][i]
 * for n < 2f (columns [0, f) the gate, [f, 2f) the up projection), fp32
 * accumulation rounded to bf16; the same sums as moe_grouped_gemm_gateup before
 * its SwiGLU. Arguments and limits as moe_grouped_gemm_gateup; gu [M][2f]. */
moe_status_t moe_grouped_gemm_gateup_preact(const moe_bf16_t* a, const moe_bf16_t* w_gateup,
                                            const int32_t* group_offsets, int G, int M, int d, int f, moe_bf16_t* gu,
                                            cudaStream_t stream);

/* A training forward's gate|up projection: h exactly as moe_grouped_gemm_gateup
 * and, from the same sums, gu exactly as moe_grouped_gemm_gateup_preact (gate
 * in columns [0, f), up in [f, 2f)), so that the backward pass need not
 * recompute them. With 128 rows or more per group on average one kernel
 * writes both (the epilogue stores g and u beside h: 2f more bf16 values per
 * row, no second pass over the weights); otherwise the two calls run one after
 * the other. Arguments and limits as moe_grouped_gemm_gateup; gu [M][2f],
 * 16-byte aligned. */
moe_status_t moe_grouped_gemm_gateup_save(const moe_bf16_t* a, const moe_bf16_t* w_gateup,
                                          const int32_t* group_offsets, int G, int M, int d, int f, moe_bf16_t* h,
                                          moe_bf16_t* gu, cudaStream_t stream);

/* SwiGLU derivative: with s = 1 / (1 + exp(-g)), for every row and n < f
 *   dgu[r][n] = dh[r][n] * u * s * (1 + g * (1 - s)),  dgu[r][f + n] = dh[r][n] * g * s,
 * g = gu[r][n], u = gu[r][f + n]; fp32 arithmetic, bf16 in and out.
 *   dh [M][f], gu [M][2f], dgu [M][2f]; f a positive multiple of 8. */
moe_status_t moe_swiglu_backward(const moe_bf16_t* dh, const moe_bf16_t* gu, int M, int f, moe_bf16_t* dgu,
                                 cudaStream_t stream);

/* Gradient of moe_unpermute_combine: for assignment a = t*k+j and its row
 * r = inv_perm[a], dy_perm[r] = bf16(topk_w[a] * dy[t]) and dw[a] = sum_c
 * dy[t][c] * y_perm[r][c] (fp32, fixed order).
 *   dy [T][d], y_perm [T*k][d] (the forward's), dy_perm [T*k][d] bf16; dw [T][k] fp32.
 * Limits as moe_unpermute_combine. */
moe_status_t moe_permute_backward(const moe_bf16_t* dy, const int32_t* inv_perm, const float* topk_w,
                                  const moe_bf16_t* y_perm, int T, int d, int k, moe_bf16_t* dy_perm, float* dw,
                                  cudaStream_t stream);

/* wt[g][c][r] = w[g][r][c]: per-expert transposed copies of the weights, for the
 * backward GEMMs (W_down [E][d][f] -> [E][f][d], W_gateup [E][2f][d] -> [E][d][2f]).
 * Not in place. G <= 65535, rows <= 2,097,120. */
moe_status_t moe_transpose_weights(const moe_bf16_t* w, int G, int rows, int cols, moe_bf16_t* wt,
                                   cudaStream_t stream);

/* Bytes of workspace moe_grouped_weight_grad needs (a multiple of 256). */
size_t moe_grouped_weight_grad_workspace_size(int M, int G, int P, int Q);

/* Weight gradient of a grouped projection, a GEMM grouped over its reduction
 * axis: dw[g][p][q] = sum over rows r of group g of a[r][p] * b[r][q], fp32
 * (bf16 products, fp32 accumulation in row order blocks of 64), one output tile
 * per CTA pair over the group's whole range (deterministic). An empty group
 * gets zeros.
 *   a [M][P], b [M][Q] bf16 (rows grouped by group_offsets [G+1], device)
 *   dw [G][P][Q] fp32
 *   ws, ws_bytes   workspace of moe_grouped_weight_grad_workspace_size(M, G, P, Q)
 *                  bytes, 256-byte aligned (the transposed, per-group
 *                  zero-padded operands)
 * Limits: 1 <= G <= 1024, P and Q positive multiples of 8. */
moe_status_t moe_grouped_weight_grad(const moe_bf16_t* a, const moe_bf16_t* b, const int32_t* group_offsets, int G,
                                     int M, int P, int Q, float* dw, void* ws, size_t ws_bytes, cudaStream_t stream);

/* Bytes of workspace moe_router_backward needs. */
size_t moe_router_backward_workspace_size(int T, int d, int E, int k);

/* Router backward, the top-k selection held fixed. From dw (the routing
 * weights' gradient, moe_permute_backward) the gradient of each selected
 * logit: softmax over the selected logits (also SOFTMAX_TOPK_RENORM, the same
 * function of them) dl_j = w_j (dw_j - sum_i w_i dw_i); sigmoid normalised,
 * with s_i = sigmoid(l_i) and S = sum s_i, dl_i = (dw_i - sum_j w_j dw_j) / S *
 * s_i (1 - s_i). Then
 *   dw_router[e][c] = sum over tokens t selecting e of dl * x[t][c]   (fp32)
 *   dbias[e]        = sum over tokens t selecting e of dl             (fp32; NULL: skipped)
 *   dx[t][c]        = dx_addend[t][c] + sum_j dl_j * w_router[e_j][c] (bf16; dx_addend may be NULL)
 * The sums over tokens run over the grouped rows (perm_src, expert_offsets of
 * moe_permute): per expert in chunks of 256 rows, then the chunks in order
 * (deterministic).
 *   logits [T][E] fp32 (the forward's), topk_idx / topk_w / dw [T][k],
 *   perm_src / inv_perm [T*k], expert_offsets [E+1], ws of
 *   moe_router_backward_workspace_size(T, d, E, k) bytes, 256-byte aligned.
 * Limits as moe_route_topk, and T*k / 256 + E <= 65535. */
moe_status_t moe_router_backward(const moe_bf16_t* x, const float* w_router, const float* logits,
                                 const int32_t* topk_idx, const float* topk_w, const float* dw,
                                 const int32_t* perm_src, const int32_t* inv_perm, const int32_t* expert_offsets,
                                 int T, int d, int E, int k, moe_route_mode_t mode, const moe_bf16_t* dx_addend,
                                 moe_bf16_t* dx, float* dw_router, float* dbias, void* ws, size_t ws_bytes,
                                 cudaStream_t stream);

/* ---- Measurement and test hook ----
 * The bf16 grouped GEMMs (moe_grouped_gemm_gateup / _down) pick one of
 * several kernel families from the problem's shape. All of them compute the
 * same sums in the same order per output element (bf16 products, fp32
 * accumulation over K in ascending 16-element steps), so their results are
 * identical; they differ in tile shape and speed:
 *   MOE_GEMM_SINGLE  one CTA per 128-row tile (few rows per expert)
 *   MOE_GEMM_PAIR    CTA pairs, 256 token rows per tile
 *   MOE_GEMM_WIDE    CTA pairs, 256 token rows x two accumulators per tile
 *   MOE_GEMM_SWAP    CTA pairs, the weight rows as the MMA's M dimension
 *                    and tiles of any multiple of 16 token rows
 * moe_set_gemm_kernel forces one family for every later call in the process
 * (on every device), so that a test can reach each of them and a benchmark
 * can compare them; MOE_GEMM_AUTO restores the library's own choice. The
 * setting is process-wide and not tied to a stream: do not change it while
 * another thread is calling the GEMMs. Not needed for normal use. */
typedef enum {
    MOE_GEMM_AUTO = 0,
    MOE_GEMM_SINGLE = 1,
    MOE_GEMM_PAIR = 2,
    MOE_GEMM_WIDE = 3,
    MOE_GEMM_SWAP = 4
} moe_gemm_kernel_t;
moe_status_t moe_set_gemm_kernel(moe_gemm_kernel_t kind);

/* Test hook for the kernels' failure path. Every pipeline wait inside the
 * grouped GEMMs is bounded: when it runs out, the kernel sets
 * MOE_DEVERR_WAIT_TIMEOUT, every role leaves its loop, copies and MMAs still
 * in flight are waited for (each wait bounded again), tensor memory is freed
 * and the kernel returns; the CUDA context stays usable. This call sets, on
 * the current device, the wait limit in nanoseconds (0 restores the default
 * of 2 s) and, with stall != 0, makes the MMA-issuing warp of every bf16
 * grouped GEMM first wait on a barrier that nothing arrives on, so that a
 * test can run the timeout path on purpose. It synchronises the device first.
 * Results of GEMMs launched while stall is set are undefined; the device
 * error word reports the timeout. Not for normal use. */
moe_status_t moe_test_set_wait(unsigned long long limit_ns, int stall);

/* Synchronise `stream`, copy the device error word of the current device to
 * *out (0 = no anomaly) and clear it. Returns MOE_OK when the word was 0,
 * MOE_ERR_DEVICE when a bit was set, MOE_ERR_CUDA when the copy failed. */
moe_status_t moe_get_device_error(unsigned int* out, cudaStream_t stream);

/* Text of the last MOE_ERR_CUDA / MOE_ERR_INVALID_ARG on the calling thread
 * ("" if none). The string is owned by the library, valid until the next call
 * on that thread. */
const char* moe_last_error_string(void);

#ifdef __cplusplus
}
#endif

#endif /* MOE_H */
