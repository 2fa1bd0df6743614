// C-ABI entry points of the MoE feed-forward layer library (declared in include/moe.h).
// Every kernel of the library is in this one translation unit (the headers below), so the device
// error word has a single definition.
#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <atomic>
#include <cstdarg>
#include <cstdio>
#include <mutex>
#include <string>

#include "moe.h"
#include "common.cuh"
#include "route.cuh"
#include "route_tc.cuh"
#include "permute.cuh"
#include "gemm.cuh"
#include "gemm_pair.cuh"
#include "gemm_wide.cuh"
#include "gemm_swap.cuh"
#include "gemm_fp4.cuh"
#include "gemm_fp4_mma.cuh"
#include "gemm_wgrad.cuh"
#include "backward.cuh"
#include "combine.cuh"

using namespace moe;

namespace {

thread_local std::string t_last_error;

moe_status_t fail(moe_status_t st, const char* fmt, ...) {
    char buf[512];
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(buf, sizeof buf, fmt, ap);
    va_end(ap);
    t_last_error = buf;
    return st;
}

// launch_err: what the launch call returned (the error state is read as well)
moe_status_t check_launch(const char* what, cudaError_t launch_err = cudaSuccess) {
    const cudaError_t e = launch_err != cudaSuccess ? launch_err : cudaGetLastError();
    if (e != cudaSuccess) return fail(MOE_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
    return MOE_OK;
}

// Every kernel is launched with programmatic stream serialization: the next kernel in the stream may be
// launched before this one ends, runs its prologue, and waits in grid_dep_wait (common.cuh) for the data.
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t stream,
                       Args&&... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

// The backward pass's elementwise, gather and transpose kernels are launched without programmatic stream
// serialization: they start after the previous kernel ends. Measured on B200: the SwiGLU-derivative kernel launched
// early as a programmatic dependent (of the pre-activation GEMM or of the combine) and followed by the CTA-pair
// dx_perm GEMM stalled the stream within a few hundred layer steps; launched plainly it did not (thousands of steps).
template <typename... KArgs, typename... Args>
cudaError_t launch_plain(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t stream,
                         Args&&... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cfg.numAttrs = 0;
    return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Grouped-GEMM configurations compiled into the library:
//   single CTA, BN 256 (4 stages) or 64 (8 stages): few rows per group (decode) or few tiles
//   CTA pair, BN 256 (6 stages), and BN 240 for the down projection when d is a multiple of 240
using Single256GU = GemmShape<256, 4, true>;
using Single256DN = GemmShape<256, 4, false>;
using Single64GU = GemmShape<64, 8, true>;
using Single64DN = GemmShape<64, 8, false>;
using Pair256GU = GemmPairShape<256, 6, true>;
using Pair256DN = GemmPairShape<256, 6, false>;
using Pair240DN = GemmPairShape<240, 6, false>;
using Pair256GU2 = GemmPairShape<256, 3, true, 2>;  // two K blocks per stage, for K >= kSub2MinK
// measured (interleaved A/B): gate|up K=2048 -6%, K=2880 -3%, K=4096 -8..10%; down K=768 +1% (not used)
constexpr int kSub2MinK = 2048;
//   CTA pair with two accumulators (2*NH-wide tiles, NH 256 or 240) when K is long
using Wide256GU = GemmWideShape<256, 4, true>;
using Wide240GU = GemmWideShape<240, 4, true>;
using Wide256DN = GemmWideShape<256, 4, false>;
using Wide240DN = GemmWideShape<240, 4, false>;
// The wide tile's epilogue is not overlapped with the next tile's MMAs, so it paid off on long reductions only
// (interleaved A/B against the 256-wide pair tile: gate|up K=2880 -8%, K=14336 +10%; down K=768 -25%, K=14336
// +10%). The pair and wide families are now reached only through moe_set_gemm_kernel.
//   CTA pair with the weights as M and the token rows as N (tiles of any multiple of 16 rows)
using SwapGU = GemmSwapShape<true, 2, 3>;
using SwapDN = GemmSwapShape<false, 2, 3>;

// Kernel family forced by moe_set_gemm_kernel (MOE_GEMM_AUTO: the library's choice).
std::atomic<int> g_gemm_kernel{MOE_GEMM_AUTO};

cudaError_t set_gemm_attributes() {
    const cudaFuncAttribute a = cudaFuncAttributeMaxDynamicSharedMemorySize;
    cudaError_t e = cudaFuncSetAttribute(grouped_gemm_kernel<256, 4, true>, a, Single256GU::SMEM_BYTES);
    if (e == cudaSuccess) e = cudaFuncSetAttribute(grouped_gemm_kernel<256, 4, false>, a, Single256DN::SMEM_BYTES);
    if (e == cudaSuccess) e = cudaFuncSetAttribute(grouped_gemm_kernel<64, 8, true>, a, Single64GU::SMEM_BYTES);
    if (e == cudaSuccess) e = cudaFuncSetAttribute(grouped_gemm_kernel<64, 8, false>, a, Single64DN::SMEM_BYTES);
    if (e == cudaSuccess) e = cudaFuncSetAttribute(grouped_gemm_pair_kernel<256, 6, true>, a, Pair256GU::SMEM_BYTES);
    if (e == cudaSuccess) e = cudaFuncSetAttribute(grouped_gemm_pair_kernel<256, 6, false>, a, Pair256DN::SMEM_BYTES);
    if (e == cudaSuccess) e = cudaFuncSetAttribute(grouped_gemm_pair_kernel<240, 6, false>, a, Pair240DN::SMEM_BYTES);
    if (e == cudaSuccess)
        e = cudaFuncSetAttribute(grouped_gemm_pair_kernel<256, 3, true, 2>, a, Pair256GU2::SMEM_BYTES);
    if (e == cudaSuccess) e = cudaFuncSetAttribute(grouped_gemm_wide_kernel<256, 4, true>, a, Wide256GU::SMEM_BYTES);
    if (e == cudaSuccess) e = cudaFuncSetAttribute(grouped_gemm_wide_kernel<240, 4, true>, a, Wide240GU::SMEM_BYTES);
    if (e == cudaSuccess) e = cudaFuncSetAttribute(grouped_gemm_wide_kernel<256, 4, false>, a, Wide256DN::SMEM_BYTES);
    if (e == cudaSuccess) e = cudaFuncSetAttribute(grouped_gemm_wide_kernel<240, 4, false>, a, Wide240DN::SMEM_BYTES);
    if (e == cudaSuccess) e = cudaFuncSetAttribute(grouped_gemm_swap_kernel<true, 2, 3, false>, a, SwapGU::SMEM_BYTES);
    if (e == cudaSuccess) e = cudaFuncSetAttribute(grouped_gemm_swap_kernel<false, 2, 3, false>, a, SwapDN::SMEM_BYTES);
    if (e == cudaSuccess) e = cudaFuncSetAttribute(grouped_gemm_swap_kernel<true, 2, 3, true>, a, SwapGU::SMEM_BYTES);
    if (e == cudaSuccess) e = cudaFuncSetAttribute(grouped_gemm_swap_kernel<false, 2, 3, true>, a, SwapDN::SMEM_BYTES);
    if (e == cudaSuccess)
        e = cudaFuncSetAttribute(grouped_gemm_swap_kernel<true, 2, 3, false, true>, a, SwapGU::SMEM_BYTES);
    if (e == cudaSuccess)
        e = cudaFuncSetAttribute(grouped_gemm_swap_kernel<true, 2, 3, true, true>, a, SwapGU::SMEM_BYTES);
    if (e == cudaSuccess)  // row gather in the operand load
        e = cudaFuncSetAttribute(grouped_gemm_swap_kernel<true, 2, 3, false, false, true>, a, SwapGU::SMEM_BYTES);
    if (e == cudaSuccess)
        e = cudaFuncSetAttribute(grouped_gemm_swap_kernel<true, 2, 3, true, false, true>, a, SwapGU::SMEM_BYTES);
    if (e == cudaSuccess)  // pre-activations saved beside h
        e = cudaFuncSetAttribute(grouped_gemm_swap_kernel<true, 2, 3, false, false, false, false, true>, a,
                                 GemmSwapShape<true, 2, 3, true>::SMEM_BYTES);
    if (e == cudaSuccess)
        e = cudaFuncSetAttribute(grouped_gemm_swap_kernel<true, 2, 3, true, false, false, false, true>, a,
                                 GemmSwapShape<true, 2, 3, true>::SMEM_BYTES);
    if (e == cudaSuccess)  // combine in the epilogue
        e = cudaFuncSetAttribute(grouped_gemm_swap_kernel<false, 2, 3, false, false, false, true>, a,
                                 SwapDN::SMEM_BYTES);
    if (e == cudaSuccess)
        e = cudaFuncSetAttribute(grouped_gemm_swap_kernel<false, 2, 3, true, false, false, true>, a,
                                 SwapDN::SMEM_BYTES);
    if (e == cudaSuccess) e = cudaFuncSetAttribute(grouped_wgrad_kernel, a, GemmWgradShape::SMEM_BYTES);
    if (e == cudaSuccess)
        e = cudaFuncSetAttribute(grouped_gemm_fp4_warp_kernel<true>, a, GemmFp4WarpShape<true>::MAX_SMEM);
    if (e == cudaSuccess)
        e = cudaFuncSetAttribute(grouped_gemm_fp4_warp_kernel<false>, a, GemmFp4WarpShape<false>::MAX_SMEM);
    if (e == cudaSuccess) e = cudaFuncSetAttribute(grouped_gemm_fp4_kernel<16, true>, a, GemmFp4Shape<16, true>::SMEM_BYTES);
    if (e == cudaSuccess) e = cudaFuncSetAttribute(grouped_gemm_fp4_kernel<32, true>, a, GemmFp4Shape<32, true>::SMEM_BYTES);
    if (e == cudaSuccess) e = cudaFuncSetAttribute(grouped_gemm_fp4_kernel<64, true>, a, GemmFp4Shape<64, true>::SMEM_BYTES);
    if (e == cudaSuccess) e = cudaFuncSetAttribute(grouped_gemm_fp4_kernel<16, false>, a, GemmFp4Shape<16, false>::SMEM_BYTES);
    if (e == cudaSuccess) e = cudaFuncSetAttribute(grouped_gemm_fp4_kernel<32, false>, a, GemmFp4Shape<32, false>::SMEM_BYTES);
    if (e == cudaSuccess) e = cudaFuncSetAttribute(grouped_gemm_fp4_kernel<64, false>, a, GemmFp4Shape<64, false>::SMEM_BYTES);
    return e;
}

constexpr int kRouterSmallMaxSmem = 200 * 1024;  // W_r rows staged by the small-T router kernel
constexpr int kRouterTcMinT = 2048;               // token count from which the tensor-core router pays off

template <int BNR>
cudaError_t set_router_tc_attr() {
    cudaError_t e = cudaFuncSetAttribute(router_tc_kernel<BNR, false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         RouterTcShape<BNR, false>::SMEM_BYTES);
    if (e == cudaSuccess)
        e = cudaFuncSetAttribute(router_tc_kernel<BNR, true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 RouterTcShape<BNR, true>::SMEM_BYTES);
    return e;
}

cudaError_t set_router_attributes() {
    cudaError_t e = set_router_tc_attr<16>();
    if (e == cudaSuccess) e = set_router_tc_attr<32>();
    if (e == cudaSuccess) e = set_router_tc_attr<64>();
    if (e == cudaSuccess) e = set_router_tc_attr<128>();
    if (e == cudaSuccess)
        e = cudaFuncSetAttribute(router_logits_small_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 kRouterSmallMaxSmem);
    return e;
}

struct DeviceInfo {
    bool ready = false;
    bool sm100 = false;
    int sms = 0;
};
constexpr int kMaxDevices = 64;
std::mutex g_mu;
DeviceInfo g_dev[kMaxDevices];

moe_status_t device_info(DeviceInfo& out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return fail(MOE_ERR_CUDA, "cudaGetDevice: %s", cudaGetErrorString(e));
    if (dev < 0 || dev >= kMaxDevices) return fail(MOE_ERR_UNSUPPORTED, "device ordinal %d out of range", dev);
    std::lock_guard<std::mutex> lock(g_mu);
    DeviceInfo& di = g_dev[dev];
    if (!di.ready) {
        int major = 0, minor = 0, sms = 0;
        if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
            return fail(MOE_ERR_CUDA, "cudaDeviceGetAttribute failed on device %d", dev);
        di.sm100 = (major == 10 && minor == 0);
        di.sms = sms;
        if (di.sm100) {
            e = set_gemm_attributes();
            if (e == cudaSuccess) e = set_router_attributes();
            if (e != cudaSuccess)
                return fail(MOE_ERR_CUDA, "cudaFuncSetAttribute: %s", cudaGetErrorString(e));
        }
        di.ready = true;
    }
    out = di;
    if (!di.sm100) return fail(MOE_ERR_UNSUPPORTED, "device %d is not sm_100 (this library is built for sm_100a)", dev);
    return MOE_OK;
}

// cuTensorMapEncodeTiled through the runtime's driver entry point (no link against libcuda).
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
    });
    return fn;
}

// Tiled tensor map; dims/strides innermost first, strides in bytes for dims >= 1. bf16 maps use the
// 128-byte swizzle the UMMA descriptors expect; the fp32 router-weight map is unswizzled.
moe_status_t make_tmap(CUtensorMap* map, const void* base, int rank, const cuuint64_t* dims,
                       const cuuint64_t* strides, const cuuint32_t* box,
                       CUtensorMapDataType dtype = CU_TENSOR_MAP_DATA_TYPE_BFLOAT16,
                       CUtensorMapSwizzle swizzle = CU_TENSOR_MAP_SWIZZLE_128B) {
    EncodeTiledFn enc = encode_fn();
    if (!enc) return fail(MOE_ERR_CUDA, "cuTensorMapEncodeTiled is unavailable");
    const cuuint32_t elem_strides[5] = {1, 1, 1, 1, 1};
    const CUresult r = enc(map, dtype, (cuuint32_t)rank, const_cast<void*>(base), dims, strides, box, elem_strides,
                           CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                           CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return fail(MOE_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", (int)r);
    return MOE_OK;
}

struct GemmProblem {
    const void* a;
    const void* w;
    const int32_t* offsets;
    int G, M, K, n_out, f;
    void* out;
    const int32_t* row_src = nullptr;  // gathering gate|up: A row r is row row_src[r] of a [src_rows][K] tensor
    int src_rows = 0;
    void* out2 = nullptr;  // gate|up saving its pre-activations [M][2f]
};

// Tensor maps: A [M][K] in 128-row x 64 boxes; B slabs [G][rows][K] (rows = 2f for gate|up, n_out for
// down) in b_rows x 64 boxes.
moe_status_t make_gemm_maps(const GemmProblem& p, bool gateup, int b_rows, CUtensorMap* ta, CUtensorMap* tb) {
    const cuuint64_t adims[2] = {(cuuint64_t)p.K, (cuuint64_t)p.M};
    const cuuint64_t astr[1] = {(cuuint64_t)p.K * 2};
    const cuuint32_t abox[2] = {GG_BK, GG_BM};
    moe_status_t st = make_tmap(ta, p.a, 2, adims, astr, abox);
    if (st != MOE_OK) return st;
    const cuuint64_t rows = gateup ? (cuuint64_t)2 * p.f : (cuuint64_t)p.n_out;
    const cuuint64_t bdims[3] = {(cuuint64_t)p.K, rows, (cuuint64_t)p.G};
    const cuuint64_t bstr[2] = {(cuuint64_t)p.K * 2, rows * (cuuint64_t)p.K * 2};
    const cuuint32_t bbox[3] = {GG_BK, (cuuint32_t)b_rows, 1};
    return make_tmap(tb, p.w, 3, bdims, bstr, bbox);
}

// Output [M][n_out] for TMA stores of 32 x 32 epilogue blocks (64-byte swizzle, as the staging layout).
moe_status_t make_out_map(const GemmProblem& p, CUtensorMap* to) {
    const cuuint64_t dims[2] = {(cuuint64_t)p.n_out, (cuuint64_t)p.M};
    const cuuint64_t strides[1] = {(cuuint64_t)p.n_out * 2};
    const cuuint32_t box[2] = {32, 32};
    return make_tmap(to, p.out, 2, dims, strides, box, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, CU_TENSOR_MAP_SWIZZLE_64B);
}

GemmArgs gemm_args(const GemmProblem& p, int out_cols) {
    GemmArgs args;
    args.group_offsets = p.offsets;
    args.G = p.G;
    args.M = p.M;
    args.K = p.K;
    args.n_out = p.n_out;
    args.f = p.f;
    args.n_tiles = (p.n_out + out_cols - 1) / out_cols;
    args.out = reinterpret_cast<__nv_bfloat16*>(p.out);
    args.row_src = p.row_src;
    args.src_rows = p.src_rows;
    args.out2 = reinterpret_cast<__nv_bfloat16*>(p.out2);
    return args;
}

template <int BN, int STAGES, bool GATEUP>
moe_status_t launch_single(const GemmProblem& p, int sms, cudaStream_t stream) {
    using S = GemmShape<BN, STAGES, GATEUP>;
    CUtensorMap ta, tb;
    moe_status_t st = make_gemm_maps(p, GATEUP, GATEUP ? BN / 2 : BN, &ta, &tb);
    if (st != MOE_OK) return st;
    const GemmArgs args = gemm_args(p, S::OUT_COLS);
    const long upper = ((long)p.M / GG_BM + p.G) * (long)args.n_tiles;  // >= the real tile count
    const int grid = (int)(upper < sms ? upper : sms);
    const int streamed_once = (long)p.M <= (long)p.G * GG_BM ? 1 : 0;
    const cudaError_t e = launch_pdl(grouped_gemm_kernel<BN, STAGES, GATEUP>, dim3(grid), dim3(GG_THREADS),
                                     S::SMEM_BYTES, stream, ta, tb, args, streamed_once);
    return check_launch(GATEUP ? "grouped_gemm_gateup" : "grouped_gemm_down", e);
}

template <int BN, int STAGES, bool GATEUP, int SUB = 1>
moe_status_t launch_pair(const GemmProblem& p, int sms, cudaStream_t stream) {
    using S = GemmPairShape<BN, STAGES, GATEUP, SUB>;
    CUtensorMap ta, tb, to;
    moe_status_t st = make_gemm_maps(p, GATEUP, BN / 2, &ta, &tb);
    if (st == MOE_OK) st = make_out_map(p, &to);
    if (st != MOE_OK) return st;
    const GemmArgs args = gemm_args(p, S::OUT_COLS);
    const long upper = ((long)p.M / GP_BM + p.G) * (long)args.n_tiles;
    const int clusters = (int)(upper < sms / 2 ? upper : sms / 2);
    const int streamed_once = (long)p.M <= (long)p.G * GP_BM ? 1 : 0;
    const cudaError_t e = launch_pdl(grouped_gemm_pair_kernel<BN, STAGES, GATEUP, SUB>, dim3(2 * clusters),
                                     dim3(GG_THREADS), S::SMEM_BYTES, stream, ta, tb, to, args, streamed_once);
    return check_launch(GATEUP ? "grouped_gemm_gateup (pair)" : "grouped_gemm_down (pair)", e);
}

template <int NH, int STAGES, bool GATEUP>
moe_status_t launch_wide(const GemmProblem& p, int sms, cudaStream_t stream) {
    using S = GemmWideShape<NH, STAGES, GATEUP>;
    CUtensorMap ta, tb;
    moe_status_t st = make_gemm_maps(p, GATEUP, NH, &ta, &tb);
    if (st != MOE_OK) return st;
    const GemmArgs args = gemm_args(p, S::OUT_COLS);
    const long upper = ((long)p.M / GP_BM + p.G) * (long)args.n_tiles;
    const int clusters = (int)(upper < sms / 2 ? upper : sms / 2);
    const int streamed_once = (long)p.M <= (long)p.G * GP_BM ? 1 : 0;
    const cudaError_t e = launch_pdl(grouped_gemm_wide_kernel<NH, STAGES, GATEUP>, dim3(2 * clusters),
                                     dim3(GW_THREADS), S::SMEM_BYTES, stream, ta, tb, args, streamed_once);
    return check_launch(GATEUP ? "grouped_gemm_gateup (wide pair)" : "grouped_gemm_down (wide pair)", e);
}

template <bool GATEUP, int SUB, int STAGES, bool BIGBOX, bool RAW = false, bool GATHER = false, bool COMBINE = false,
          bool SAVE = false>
moe_status_t launch_swap(const GemmProblem& p, int sms, cudaStream_t stream, const CombineArgs& ca = CombineArgs()) {
    using S = GemmSwapShape<GATEUP, SUB, STAGES, SAVE>;
    CUtensorMap tw, to, tg;
    SwapMaps tx;
    moe_status_t st;
    const cuuint64_t K = (cuuint64_t)p.K, f = (cuuint64_t)p.f, G = (cuuint64_t)p.G, n_out = (cuuint64_t)p.n_out;
    const cuuint64_t KBS = (K + GG_BK - 1) / GG_BK;
    if (BIGBOX) {  // K-block views: [rows][K] read as [K/64][rows][64] (K a multiple of 64), SUB K blocks per box
        if (GATEUP) {  // [G][K/64][2][f][64]
            const cuuint64_t wdims[5] = {GG_BK, f, 2, KBS, G};
            const cuuint64_t wstr[4] = {K * 2, f * K * 2, GG_BK * 2, 2 * f * K * 2};
            const cuuint32_t wbox[5] = {GG_BK, 64, 2, SUB, 1};
            st = make_tmap(&tw, p.w, 5, wdims, wstr, wbox);
        } else {  // [G][K/64][d][64]
            const cuuint64_t wdims[4] = {GG_BK, n_out, KBS, G};
            const cuuint64_t wstr[3] = {K * 2, GG_BK * 2, n_out * K * 2};
            const cuuint32_t wbox[4] = {GG_BK, 128, SUB, 1};
            st = make_tmap(&tw, p.w, 4, wdims, wstr, wbox);
        }
        const cuuint64_t xdims[3] = {GG_BK, (cuuint64_t)p.M, KBS};
        const cuuint64_t xstr[2] = {K * 2, GG_BK * 2};
        for (int i = 0; i < 5 && st == MOE_OK; ++i) {
            const cuuint32_t xbox[3] = {GG_BK, (cuuint32_t)(128 >> i), SUB};
            st = make_tmap(&tx.x[i], p.a, 3, xdims, xstr, xbox);
        }
    } else {
        if (GATEUP) {  // [G][2][f][K]: one box = 64 gate rows and the matching 64 up rows
            const cuuint64_t wdims[4] = {K, f, 2, G};
            const cuuint64_t wstr[3] = {K * 2, f * K * 2, 2 * f * K * 2};
            const cuuint32_t wbox[4] = {GG_BK, 64, 2, 1};
            st = make_tmap(&tw, p.w, 4, wdims, wstr, wbox);
        } else {  // [G][d][K]
            const cuuint64_t wdims[3] = {K, n_out, G};
            const cuuint64_t wstr[2] = {K * 2, n_out * K * 2};
            const cuuint32_t wbox[3] = {GG_BK, 128, 1};
            st = make_tmap(&tw, p.w, 3, wdims, wstr, wbox);
        }
        const cuuint64_t xdims[2] = {K, (cuuint64_t)p.M};
        const cuuint64_t xstr[1] = {K * 2};
        for (int i = 0; i < 5 && st == MOE_OK; ++i) {
            const cuuint32_t xbox[2] = {GG_BK, (cuuint32_t)(128 >> i)};
            st = make_tmap(&tx.x[i], p.a, 2, xdims, xstr, xbox);
        }
    }
    if (GATHER && st == MOE_OK) {  // the source rows [src_rows][K], one row per box (TMA gather4)
        const cuuint64_t gdims[2] = {K, (cuuint64_t)p.src_rows};
        const cuuint64_t gstr[1] = {K * 2};
        const cuuint32_t gbox[2] = {GG_BK, 1};
        st = make_tmap(&tx.x[0], p.a, 2, gdims, gstr, gbox);
        for (int i = 1; i < 5; ++i) tx.x[i] = tx.x[0];
    }
    if (st == MOE_OK) {
        if (RAW) {  // [M][2f] pre-activations: gate in columns [0, f), up in [f, 2f)
            GemmProblem q = p;
            q.n_out = 2 * p.f;
            st = make_out_map(q, &to);
        } else {
            st = make_out_map(p, &to);
        }
    }
    if (st != MOE_OK) return st;
    tg = to;
    if (SAVE) {  // [M][2f] pre-activations
        GemmProblem q = p;
        q.n_out = 2 * p.f;
        q.out = p.out2;
        if ((st = make_out_map(q, &tg)) != MOE_OK) return st;
    }
    const GemmArgs args = gemm_args(p, S::TILE_W);
    const long upper = ((long)p.M / GS_MAX_N + p.G) * (long)args.n_tiles;  // >= the real tile count
    const int clusters = (int)(upper < sms / 2 ? upper : sms / 2);
    const int streamed_once = (long)p.M <= (long)p.G * GS_MAX_N ? 1 : 0;
    const cudaError_t e = launch_pdl(grouped_gemm_swap_kernel<GATEUP, SUB, STAGES, BIGBOX, RAW, GATHER, COMBINE, SAVE>,
                                     dim3(2 * clusters), dim3(GS_THREADS), S::SMEM_BYTES, stream, tw, tx, to, tg, args,
                                     streamed_once, ca);
    return check_launch(RAW ? "grouped_gemm_gateup_preact (swap pair)"
                            : (GATEUP ? "grouped_gemm_gateup (swap pair)"
                                      : (COMBINE ? "grouped_gemm_down_combine (swap pair)"
                                                 : "grouped_gemm_down (swap pair)")), e);
}

template <bool GATEUP>
moe_status_t launch_swap_auto(const GemmProblem& p, int sms, cudaStream_t stream) {
    if (p.K % GG_BK == 0) return launch_swap<GATEUP, 2, 3, true>(p, sms, stream);
    return launch_swap<GATEUP, 2, 3, false>(p, sms, stream);
}

// A kernel family chosen with moe_set_gemm_kernel.
moe_status_t launch_forced(int kind, const GemmProblem& p, bool gateup, int sms, cudaStream_t stream) {
    const bool sub2 = p.K >= kSub2MinK;
    const bool w240 = (long)(p.n_out + 239) / 240 * 240 < (long)(p.n_out + 255) / 256 * 256;
    switch (kind) {
        case MOE_GEMM_SINGLE:
            return gateup ? launch_single<256, 4, true>(p, sms, stream) : launch_single<256, 4, false>(p, sms, stream);
        case MOE_GEMM_PAIR:
            if (gateup) return sub2 ? launch_pair<256, 3, true, 2>(p, sms, stream) : launch_pair<256, 6, true>(p, sms, stream);
            return w240 ? launch_pair<240, 6, false>(p, sms, stream) : launch_pair<256, 6, false>(p, sms, stream);
        case MOE_GEMM_WIDE: {
            const long span = gateup ? 1 : 2;
            const bool wide240 = (long)(p.n_out + 240 * span - 1) / (240 * span) * (240 * span) <
                                 (long)(p.n_out + 256 * span - 1) / (256 * span) * (256 * span);
            if (gateup)
                return wide240 ? launch_wide<240, 4, true>(p, sms, stream) : launch_wide<256, 4, true>(p, sms, stream);
            return wide240 ? launch_wide<240, 4, false>(p, sms, stream) : launch_wide<256, 4, false>(p, sms, stream);
        }
        default:
            return gateup ? launch_swap_auto<true>(p, sms, stream) : launch_swap_auto<false>(p, sms, stream);
    }
}

// Kernel choice. Groups averaging at least 128 rows (prefill) run on CTA pairs with the weights as the MMA's M
// dimension (gemm_swap.cuh): tiles of any multiple of 16 token rows, so ragged groups cost almost no padding;
// measured faster than the 256-row pair tiles and the two-accumulator tiles on every prefill workload (gpt-oss
// gate|up -9%, Mixtral gate|up -5%, zipf-128e -8%). Otherwise (a few rows per expert, decode) a single CTA per
// 128-row tile streams the weights, 256 wide unless that leaves SMs idle (e.g. one small group), then 64 wide.
moe_status_t launch_grouped_gemm(const GemmProblem& p, bool gateup, int sms, cudaStream_t stream) {
    const int forced = g_gemm_kernel.load(std::memory_order_relaxed);
    if (forced != MOE_GEMM_AUTO && sms >= 2) return launch_forced(forced, p, gateup, sms, stream);
    if ((long)p.M >= (long)p.G * GG_BM && sms >= 2)
        return gateup ? launch_swap_auto<true>(p, sms, stream) : launch_swap_auto<false>(p, sms, stream);
    const long row_tiles = std::max<long>((p.M + GG_BM - 1) / GG_BM, std::min<long>(p.G, p.M));
    const long wide_tiles = row_tiles * ((p.n_out + (gateup ? 127 : 255)) / (gateup ? 128 : 256));
    if (wide_tiles >= sms)
        return gateup ? launch_single<256, 4, true>(p, sms, stream) : launch_single<256, 4, false>(p, sms, stream);
    return gateup ? launch_single<64, 8, true>(p, sms, stream) : launch_single<64, 8, false>(p, sms, stream);
}

// ---- MXFP4 weights ----
struct Fp4Problem {
    const void* a;        // activations [M][K] bf16
    const uint8_t* q;     // codes [G][rows][K/2]
    const uint8_t* s;     // scales [G][K/32][rows]
    const int32_t* offsets;
    int G, M, K, n_out, f, rows;  // rows: weight rows per group (2f for gate|up, d for down)
    void* out;
};

template <int NT, bool GATEUP>
moe_status_t launch_fp4(const Fp4Problem& p, int sms, cudaStream_t stream) {
    using S = GemmFp4Shape<NT, GATEUP>;
    CUtensorMap tx, tq, ts;
    const cuuint64_t xdims[2] = {(cuuint64_t)p.K, (cuuint64_t)p.M};
    const cuuint64_t xstr[1] = {(cuuint64_t)p.K * 2};
    const cuuint32_t xbox[2] = {64, (cuuint32_t)NT};
    moe_status_t st = make_tmap(&tx, p.a, 2, xdims, xstr, xbox);
    if (st != MOE_OK) return st;
    const cuuint64_t qdims[3] = {(cuuint64_t)p.K / 2, (cuuint64_t)p.rows, (cuuint64_t)p.G};
    const cuuint64_t qstr[2] = {(cuuint64_t)p.K / 2, (cuuint64_t)p.rows * (p.K / 2)};
    const cuuint32_t qbox[3] = {GF_KS / 2, GF_BM, 1};
    if ((st = make_tmap(&tq, p.q, 3, qdims, qstr, qbox, CU_TENSOR_MAP_DATA_TYPE_UINT8)) != MOE_OK) return st;
    const cuuint64_t sdims[3] = {(cuuint64_t)p.rows, (cuuint64_t)p.K / 32, (cuuint64_t)p.G};
    const cuuint64_t sstr[2] = {(cuuint64_t)p.rows, (cuuint64_t)p.rows * (p.K / 32)};
    const cuuint32_t sbox[3] = {GF_BM, GF_KS / 32, 1};
    if ((st = make_tmap(&ts, p.s, 3, sdims, sstr, sbox, CU_TENSOR_MAP_DATA_TYPE_UINT8, CU_TENSOR_MAP_SWIZZLE_NONE)) !=
        MOE_OK)
        return st;
    GemmArgs args;
    args.group_offsets = p.offsets;
    args.G = p.G;
    args.M = p.M;
    args.K = p.K;
    args.n_out = p.n_out;
    args.f = p.f;
    args.n_tiles = (p.n_out + GF_BM - 1) / GF_BM;
    args.out = reinterpret_cast<__nv_bfloat16*>(p.out);
    const long upper = ((long)p.M / NT + p.G) * (long)args.n_tiles;  // >= the real tile count
    const int grid = (int)(upper < sms ? upper : sms);
    const int streamed_once = (long)p.M <= (long)p.G * NT ? 1 : 0;
    const cudaError_t e = launch_pdl(grouped_gemm_fp4_kernel<NT, GATEUP>, dim3(grid), dim3(GF_THREADS), S::SMEM_BYTES,
                                     stream, tx, tq, ts, args, streamed_once);
    return check_launch(GATEUP ? "grouped_gemm_gateup_mxfp4" : "grouped_gemm_down_mxfp4", e);
}

// Warp-MMA kernel (gemm_fp4_mma.cuh): 8-row token blocks, an equal share of the units per CTA.
template <bool GATEUP>
moe_status_t launch_fp4_warp(const Fp4Problem& p, int sms, cudaStream_t stream) {
    using S = GemmFp4WarpShape<GATEUP>;
    const int stages = S::stages_for(p.K, p.G);
    CUtensorMap tx, tq, ts;
    // token rows as [M][K/32][32]: one box = one whole row
    const cuuint64_t xdims[3] = {32, (cuuint64_t)p.K / 32, (cuuint64_t)p.M};
    const cuuint64_t xstr[2] = {64, (cuuint64_t)p.K * 2};
    const cuuint32_t xbox[3] = {32, (cuuint32_t)(p.K / 32), 1};
    moe_status_t st = make_tmap(&tx, p.a, 3, xdims, xstr, xbox, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16,
                                CU_TENSOR_MAP_SWIZZLE_NONE);
    if (st != MOE_OK) return st;
    const cuuint64_t qdims[3] = {(cuuint64_t)p.K / 2, (cuuint64_t)p.rows, (cuuint64_t)p.G};
    const cuuint64_t qstr[2] = {(cuuint64_t)p.K / 2, (cuuint64_t)p.rows * (p.K / 2)};
    const cuuint32_t qbox[3] = {FW_KS / 2, S::BM, 1};
    if ((st = make_tmap(&tq, p.q, 3, qdims, qstr, qbox, CU_TENSOR_MAP_DATA_TYPE_UINT8)) != MOE_OK) return st;
    const cuuint64_t sdims[3] = {(cuuint64_t)p.rows, (cuuint64_t)p.K / 32, (cuuint64_t)p.G};
    const cuuint64_t sstr[2] = {(cuuint64_t)p.rows, (cuuint64_t)p.rows * (p.K / 32)};
    const cuuint32_t sbox[3] = {S::BM, FW_KS / 32, 1};
    if ((st = make_tmap(&ts, p.s, 3, sdims, sstr, sbox, CU_TENSOR_MAP_DATA_TYPE_UINT8, CU_TENSOR_MAP_SWIZZLE_NONE)) !=
        MOE_OK)
        return st;
    GemmArgs args;
    args.group_offsets = p.offsets;
    args.G = p.G;
    args.M = p.M;
    args.K = p.K;
    args.n_out = p.n_out;
    args.f = p.f;
    args.n_tiles = (p.n_out + S::BM - 1) / S::BM;
    args.out = reinterpret_cast<__nv_bfloat16*>(p.out);
    // one CTA per SM, each with an equal share of the (token block, weight block) units
    const long upper = ((long)p.M / FW_NT + p.G) * (long)args.n_tiles;  // >= the unit count
    const int grid = (int)(upper < sms ? upper : sms);
    const int streamed_once = (long)p.M <= (long)p.G * FW_NT ? 1 : 0;
    const cudaError_t e = launch_pdl(grouped_gemm_fp4_warp_kernel<GATEUP>, dim3(grid), dim3(FW_THREADS),
                                     (size_t)S::smem_bytes(p.K, stages, p.G), stream, tx, tq, ts, args, streamed_once,
                                     stages);
    return check_launch(GATEUP ? "grouped_gemm_gateup_mxfp4 (warp MMA)" : "grouped_gemm_down_mxfp4 (warp MMA)", e);
}

// A few rows per expert (at most 8 on average: decode) and K <= 8192: the warp-MMA kernel. Otherwise the
// tensor-memory kernel with the smallest token tile of 16, 32, 64 that holds an average group (a shared expert:
// all T rows in one group; measured: on the decode layer's side stream the warp kernel took its 64 rows in 108
// instead of 128 µs but, on every SM, slowed the routing and grouping beside it by as much). Larger groups take
// several token tiles.
template <bool GATEUP>
moe_status_t launch_fp4_nt(const Fp4Problem& p, int sms, cudaStream_t stream) {
    if ((long)p.M <= 8L * p.G && p.K <= FW_MAX_K && GemmFp4WarpShape<GATEUP>::stages_for(p.K, p.G) >= 2)
        return launch_fp4_warp<GATEUP>(p, sms, stream);
    if ((long)p.M <= 8L * p.G) return launch_fp4<16, GATEUP>(p, sms, stream);
    if ((long)p.M <= 24L * p.G) return launch_fp4<32, GATEUP>(p, sms, stream);
    return launch_fp4<64, GATEUP>(p, sms, stream);
}

moe_status_t check_fp4_args(const void* a, const uint8_t* q, const uint8_t* s, const int32_t* offsets, int G, int M,
                            int d, int f, const void* out) {
    if (!q || !s || !offsets || (M > 0 && (!a || !out))) return fail(MOE_ERR_INVALID_ARG, "null pointer argument");
    if (!aligned16(a) || !aligned16(q) || !aligned16(s) || !aligned16(out))
        return fail(MOE_ERR_INVALID_ARG, "activation, code, scale and output pointers must be 16-byte aligned");
    if ((reinterpret_cast<uintptr_t>(offsets) & 3u) != 0) return fail(MOE_ERR_INVALID_ARG, "offsets misaligned");
    if (G < 1 || G > GG_MAX_GROUPS) return fail(MOE_ERR_INVALID_ARG, "G=%d outside [1, %d]", G, GG_MAX_GROUPS);
    if (M < 0) return fail(MOE_ERR_INVALID_ARG, "M=%d < 0", M);
    if (d < 32 || f < 32 || d % 32 || f % 32)
        return fail(MOE_ERR_INVALID_ARG, "d=%d and f=%d must be positive multiples of 32 (MXFP4 blocks)", d, f);
    return MOE_OK;
}

template <int BNR, bool PRESPLIT>
moe_status_t launch_router_tc(const CUtensorMap& tm, const CUtensorMap& tw, const CUtensorMap& tp,
                              const float* w_router, const float* bias, int T, int d, int E, int k, int mode,
                              int fuse, float* logits, int32_t* idx, float* w, int tiles, int cs,
                              cudaStream_t stream) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)(tiles * cs));
    cfg.blockDim = dim3(RTC_THREADS);
    cfg.dynamicSmemBytes = RouterTcShape<BNR, PRESPLIT>::SMEM_BYTES;
    cfg.stream = stream;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = (unsigned)cs;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;  // as launch_pdl
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 2;
    const cudaError_t e = cudaLaunchKernelEx(&cfg, router_tc_kernel<BNR, PRESPLIT>, tm, tw, tp, w_router, bias, T, d,
                                             E, k, mode, fuse, logits, idx, w);
    if (e != cudaSuccess) return fail(MOE_ERR_CUDA, "router_tc launch: %s", cudaGetErrorString(e));
    return MOE_OK;
}

// With M = 0 the activation and output arrays are empty and their pointers may be null.
moe_status_t check_gemm_args(const void* a, const void* w, const int32_t* offsets, int G, int M, int d, int f,
                             const void* out) {
    if (!w || !offsets || (M > 0 && (!a || !out))) return fail(MOE_ERR_INVALID_ARG, "null pointer argument");
    if (!aligned16(a) || !aligned16(w) || !aligned16(out))
        return fail(MOE_ERR_INVALID_ARG, "activation, weight and output pointers must be 16-byte aligned");
    if ((reinterpret_cast<uintptr_t>(offsets) & 3u) != 0) return fail(MOE_ERR_INVALID_ARG, "offsets misaligned");
    if (G < 1 || G > GG_MAX_GROUPS) return fail(MOE_ERR_INVALID_ARG, "G=%d outside [1, %d]", G, GG_MAX_GROUPS);
    if (M < 0) return fail(MOE_ERR_INVALID_ARG, "M=%d < 0", M);
    if (d < 8 || f < 8 || d % 8 || f % 8)
        return fail(MOE_ERR_INVALID_ARG, "d=%d and f=%d must be positive multiples of 8", d, f);
    return MOE_OK;
}

moe_status_t check_route_sizes(int T, int E, int k) {
    if (T < 0) return fail(MOE_ERR_INVALID_ARG, "T=%d < 0", T);
    if (E < 1 || E > 1024) return fail(MOE_ERR_INVALID_ARG, "E=%d outside [1, 1024]", E);
    if (k < 1 || k > E || k > 32) return fail(MOE_ERR_INVALID_ARG, "k=%d outside [1, min(E, 32)]", k);
    if ((long)T * E > 0x7fffffffL || (long)T * k > 0x7fffffffL)
        return fail(MOE_ERR_INVALID_ARG, "T*E or T*k exceeds int32");
    return MOE_OK;
}

int grid_cap(long want, int sms, int per_sm) {
    const long cap = (long)sms * per_sm;
    if (want < 1) want = 1;
    return (int)(want < cap ? want : cap);
}

}  // namespace

// Scratch of moe_permute_static_ws: one array per device, part of the loaded module (nothing is
// allocated). Host code must not pass this symbol to a kernel (on the host it is only a stand-in); the
// device address comes from cudaGetSymbolAddress, looked up once per device.
static __device__ __align__(256) unsigned char g_permute_static_ws[MOE_PERMUTE_STATIC_WS_BYTES];

namespace {
void* g_static_ws_addr[kMaxDevices] = {};

moe_status_t static_ws_address(void** out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return fail(MOE_ERR_CUDA, "cudaGetDevice: %s", cudaGetErrorString(e));
    if (dev < 0 || dev >= kMaxDevices) return fail(MOE_ERR_UNSUPPORTED, "device ordinal %d out of range", dev);
    std::lock_guard<std::mutex> lock(g_mu);
    if (!g_static_ws_addr[dev]) {
        void* p = nullptr;
        e = cudaGetSymbolAddress(&p, g_permute_static_ws);
        if (e != cudaSuccess || !p)
            return fail(MOE_ERR_CUDA, "cudaGetSymbolAddress(static permute scratch): %s", cudaGetErrorString(e));
        g_static_ws_addr[dev] = p;
    }
    *out = g_static_ws_addr[dev];
    return MOE_OK;
}
}  // namespace

namespace {

template <bool PRESPLIT>
moe_status_t launch_router_tc_bnr(int bnr, const CUtensorMap& tm, const CUtensorMap& tw, const CUtensorMap& tp,
                                  const float* w_router, const float* bias, int T, int d, int E, int k, int mode,
                                  int fuse, float* logits, int32_t* idx, float* w, int tiles, int cs,
                                  cudaStream_t stream) {
    switch (bnr) {
        case 16:
            return launch_router_tc<16, PRESPLIT>(tm, tw, tp, w_router, bias, T, d, E, k, mode, fuse, logits, idx, w,
                                                  tiles, cs, stream);
        case 32:
            return launch_router_tc<32, PRESPLIT>(tm, tw, tp, w_router, bias, T, d, E, k, mode, fuse, logits, idx, w,
                                                  tiles, cs, stream);
        case 64:
            return launch_router_tc<64, PRESPLIT>(tm, tw, tp, w_router, bias, T, d, E, k, mode, fuse, logits, idx, w,
                                                  tiles, cs, stream);
        default:
            return launch_router_tc<128, PRESPLIT>(tm, tw, tp, w_router, bias, T, d, E, k, mode, fuse, logits, idx,
                                                   w, tiles, cs, stream);
    }
}

// moe_route_topk and moe_route_topk_split; w_pieces (nullable): the [3][E][d] bf16 split of w_router
moe_status_t route_impl(const moe_bf16_t* x, const float* w_router, const moe_bf16_t* w_pieces, const float* bias,
                        int T, int d, int E, int k, moe_route_mode_t mode, float* logits_out, int32_t* topk_idx,
                        float* topk_w, cudaStream_t stream) {
    moe_status_t st = check_route_sizes(T, E, k);
    if (st != MOE_OK) return st;
    if (mode < MOE_ROUTE_TOPK_SOFTMAX || mode > MOE_ROUTE_SIGMOID_TOPK_NORM)
        return fail(MOE_ERR_INVALID_ARG, "unknown routing mode %d", (int)mode);
    if (d < 8 || d % 8) return fail(MOE_ERR_INVALID_ARG, "d=%d must be a positive multiple of 8", d);
    if (T == 0) return MOE_OK;  // nothing to route (the empty arrays' pointers may be null)
    if (!x || !w_router || !logits_out || !topk_idx || !topk_w) return fail(MOE_ERR_INVALID_ARG, "null pointer");
    if (!aligned16(x) || !aligned16(w_router) || !aligned16(w_pieces))
        return fail(MOE_ERR_INVALID_ARG, "x / w_router / w_pieces not 16-byte aligned");
    DeviceInfo di;
    if ((st = device_info(di)) != MOE_OK) return st;
    const __nv_bfloat16* xb = reinterpret_cast<const __nv_bfloat16*>(x);
    if (E <= 128 && T >= kRouterTcMinT) {
        // tensor cores, W_r as three bf16 pieces (split here, or given); top-k fused (any k <= 32)
        CUtensorMap tm, tw, tp;
        const cuuint64_t dims[2] = {(cuuint64_t)d, (cuuint64_t)T};
        const cuuint64_t strides[1] = {(cuuint64_t)d * 2};
        const cuuint32_t box[2] = {RTC_BK, RTC_BM};
        if ((st = make_tmap(&tm, x, 2, dims, strides, box)) != MOE_OK) return st;
        const int bnr = E <= 16 ? 16 : (E <= 32 ? 32 : (E <= 64 ? 64 : 128));
        const cuuint64_t wdims[2] = {(cuuint64_t)d, (cuuint64_t)E};
        const cuuint64_t wstrides[1] = {(cuuint64_t)d * 4};
        const cuuint32_t wbox[2] = {RTC_BK, (cuuint32_t)bnr};
        if ((st = make_tmap(&tw, w_router, 2, wdims, wstrides, wbox, CU_TENSOR_MAP_DATA_TYPE_FLOAT32,
                            CU_TENSOR_MAP_SWIZZLE_NONE)) != MOE_OK)
            return st;
        if (w_pieces) {  // [3][E][d] bf16: one box brings a K block of all three pieces
            const cuuint64_t pdims[3] = {(cuuint64_t)d, (cuuint64_t)E, 3};
            const cuuint64_t pstrides[2] = {(cuuint64_t)d * 2, (cuuint64_t)E * d * 2};
            const cuuint32_t pbox[3] = {RTC_BK, (cuuint32_t)bnr, 3};
            if ((st = make_tmap(&tp, w_pieces, 3, pdims, pstrides, pbox)) != MOE_OK) return st;
        } else {
            tp = tw;  // unused
        }
        const int fuse = k <= RTC_KMAX ? 1 : 0;
        const int tiles = (T + RTC_BM - 1) / RTC_BM;
        const int kblocks = (d + RTC_BK - 1) / RTC_BK;
        // split K over a cluster when there are few 128-token tiles (keeps >= 2 K blocks per CTA)
        int cs = 1;
        if (tiles * 4 <= di.sms && kblocks >= 8)
            cs = 4;
        else if (tiles * 2 <= di.sms && kblocks >= 4)
            cs = 2;
        st = w_pieces ? launch_router_tc_bnr<true>(bnr, tm, tw, tp, w_router, bias, T, d, E, k, (int)mode, fuse,
                                                   logits_out, topk_idx, topk_w, tiles, cs, stream)
                      : launch_router_tc_bnr<false>(bnr, tm, tw, tp, w_router, bias, T, d, E, k, (int)mode, fuse,
                                                    logits_out, topk_idx, topk_w, tiles, cs, stream);
        if (st != MOE_OK) return st;
        if ((st = check_launch("router_tc")) != MOE_OK) return st;
        if (fuse) return MOE_OK;
    } else if ((size_t)d * sizeof(float) <= (size_t)kRouterSmallMaxSmem) {
        // few tokens: CUDA cores, parallel over experts so every SM streams part of W_r
        int epb = E >= 2 * di.sms ? 4 : (E >= di.sms ? 2 : 1);
        while (epb > 1 && (size_t)epb * d * sizeof(float) > (size_t)kRouterSmallMaxSmem) --epb;
        const int grid = (E + epb - 1) / epb;
        const cudaError_t e = launch_pdl(router_logits_small_kernel, dim3(grid), dim3(RS_THREADS),
                                         (size_t)epb * d * sizeof(float), stream, xb, w_router, bias, T, d, E, epb,
                                         logits_out);
        if ((st = check_launch("router_logits_small", e)) != MOE_OK) return st;
    } else {
        dim3 grid((T + RT_TOK - 1) / RT_TOK, (E + RT_EXP - 1) / RT_EXP);
        const cudaError_t e = launch_pdl(router_logits_kernel, dim3(grid), dim3(RT_THREADS), 0, stream, xb, w_router,
                                         bias, T, d, E, logits_out);
        if ((st = check_launch("router_logits", e)) != MOE_OK) return st;
    }
    const cudaError_t e = launch_pdl(topk_kernel, dim3((T + TOPK_WARPS - 1) / TOPK_WARPS), dim3(TOPK_WARPS * 32), 0,
                                     stream, logits_out, T, E, k, (int)mode, topk_idx, topk_w);
    return check_launch("topk", e);
}

}  // namespace

extern "C" {

moe_status_t moe_route_topk(const moe_bf16_t* x, const float* w_router, const float* bias, int T, int d, int E,
                            int k, moe_route_mode_t mode, float* logits_out, int32_t* topk_idx, float* topk_w,
                            cudaStream_t stream) {
    return route_impl(x, w_router, nullptr, bias, T, d, E, k, mode, logits_out, topk_idx, topk_w, stream);
}

moe_status_t moe_router_split_weights(const float* w_router, int E, int d, moe_bf16_t* w_pieces,
                                      cudaStream_t stream) {
    if (E < 1 || E > 1024) return fail(MOE_ERR_INVALID_ARG, "E=%d outside [1, 1024]", E);
    if (d < 8 || d % 8) return fail(MOE_ERR_INVALID_ARG, "d=%d must be a positive multiple of 8", d);
    if (!w_router || !w_pieces) return fail(MOE_ERR_INVALID_ARG, "null pointer");
    if (!aligned16(w_router) || !aligned16(w_pieces))
        return fail(MOE_ERR_INVALID_ARG, "w_router / w_pieces not 16-byte aligned");
    DeviceInfo di;
    moe_status_t st = device_info(di);
    if (st != MOE_OK) return st;
    const long pairs = (long)E * d / 2;
    uint32_t* base = reinterpret_cast<uint32_t*>(w_pieces);
    const int grid = grid_cap((pairs + 255) / 256, di.sms, 8);
    const cudaError_t e = launch_pdl(router_split_kernel, dim3(grid), dim3(256), 0, stream, w_router, pairs, base,
                                     base + pairs, base + 2 * pairs);
    return check_launch("router_split", e);
}

moe_status_t moe_route_topk_split(const moe_bf16_t* x, const float* w_router, const moe_bf16_t* w_pieces,
                                  const float* bias, int T, int d, int E, int k, moe_route_mode_t mode,
                                  float* logits_out, int32_t* topk_idx, float* topk_w, cudaStream_t stream) {
    if (!w_pieces) return fail(MOE_ERR_INVALID_ARG, "w_pieces is required (moe_route_topk takes none)");
    return route_impl(x, w_router, w_pieces, bias, T, d, E, k, mode, logits_out, topk_idx, topk_w, stream);
}

moe_status_t moe_topk_from_logits(const float* logits, int T, int E, int k, moe_route_mode_t mode,
                                  int32_t* topk_idx, float* topk_w, cudaStream_t stream) {
    moe_status_t st = check_route_sizes(T, E, k);
    if (st != MOE_OK) return st;
    if (mode < MOE_ROUTE_TOPK_SOFTMAX || mode > MOE_ROUTE_SIGMOID_TOPK_NORM)
        return fail(MOE_ERR_INVALID_ARG, "unknown routing mode %d", (int)mode);
    if (T == 0) return MOE_OK;
    if (!logits || !topk_idx || !topk_w) return fail(MOE_ERR_INVALID_ARG, "null pointer");
    DeviceInfo di;
    if ((st = device_info(di)) != MOE_OK) return st;
    const cudaError_t e = launch_pdl(topk_kernel, dim3((T + TOPK_WARPS - 1) / TOPK_WARPS), dim3(TOPK_WARPS * 32), 0,
                                     stream, logits, T, E, k, (int)mode, topk_idx, topk_w);
    return check_launch("topk", e);
}

size_t moe_permute_workspace_size(int T, int E, int k) {
    if (T <= 0 || E <= 0 || k <= 0) return 0;
    const size_t bytes = (size_t)perm_num_segments((long)T * k) * (size_t)E * sizeof(int32_t);
    return (bytes + 255) / 256 * 256;
}

moe_status_t moe_permute(const moe_bf16_t* x, const int32_t* topk_idx, int T, int d, int E, int k,
                         int32_t* expert_counts, int32_t* expert_offsets, int32_t* perm_src, int32_t* inv_perm,
                         moe_bf16_t* x_perm, void* ws, size_t ws_bytes, cudaStream_t stream) {
    moe_status_t st = check_route_sizes(T, E, k);
    if (st != MOE_OK) return st;
    if (!expert_counts || !expert_offsets) return fail(MOE_ERR_INVALID_ARG, "null pointer");
    if (T == 0) {  // no assignments: counts and offsets all zero (the empty arrays' pointers may be null)
        DeviceInfo di;
        if ((st = device_info(di)) != MOE_OK) return st;
        cudaError_t e = cudaMemsetAsync(expert_counts, 0, sizeof(int32_t) * E, stream);
        if (e == cudaSuccess) e = cudaMemsetAsync(expert_offsets, 0, sizeof(int32_t) * (E + 1), stream);
        if (e != cudaSuccess) return fail(MOE_ERR_CUDA, "cudaMemsetAsync: %s", cudaGetErrorString(e));
        return MOE_OK;
    }
    if (!topk_idx || !perm_src || !inv_perm) return fail(MOE_ERR_INVALID_ARG, "null pointer");
    if ((x == nullptr) != (x_perm == nullptr)) return fail(MOE_ERR_INVALID_ARG, "x and x_perm: give both or neither");
    if (x) {
        if (d < 8 || d % 8) return fail(MOE_ERR_INVALID_ARG, "d=%d must be a positive multiple of 8", d);
        if (!aligned16(x) || !aligned16(x_perm)) return fail(MOE_ERR_INVALID_ARG, "x / x_perm not 16-byte aligned");
        if ((long)T * k * (long)d > 0x7fffffffffffL) return fail(MOE_ERR_INVALID_ARG, "x_perm too large");
    }
    const size_t need = moe_permute_workspace_size(T, E, k);
    if (need && (!ws || ws_bytes < need))
        return fail(MOE_ERR_WORKSPACE, "workspace of %zu bytes needed, %zu given", need, ws ? ws_bytes : (size_t)0);
    if (ws && (reinterpret_cast<uintptr_t>(ws) & 255u)) return fail(MOE_ERR_WORKSPACE, "workspace not 256-byte aligned");
    DeviceInfo di;
    if ((st = device_info(di)) != MOE_OK) return st;
    const int R = T * k;
    int32_t* seg = reinterpret_cast<int32_t*>(ws);
    const int nseg = perm_num_segments(R);
    cudaError_t e = launch_pdl(permute_hist_kernel, dim3(nseg), dim3(PERM_THREADS), E * sizeof(int32_t), stream,
                               topk_idx, R, E, seg);
    if ((st = check_launch("permute_hist", e)) != MOE_OK) return st;
    e = launch_pdl(permute_scan_kernel, dim3(1), dim3(1024), 0, stream, seg, nseg, E, expert_counts, expert_offsets);
    if ((st = check_launch("permute_scan", e)) != MOE_OK) return st;
    e = launch_pdl(permute_scatter_kernel, dim3(nseg), dim3(PERM_THREADS), PERM_WARPS * E * sizeof(int32_t), stream,
                   topk_idx, R, E, k, seg, perm_src, inv_perm);
    if ((st = check_launch("permute_scatter", e)) != MOE_OK) return st;
    if (x) {
        const int grid = grid_cap((R + 7) / 8, di.sms, 16);
        e = launch_pdl(gather_rows_kernel, dim3(grid), dim3(256), 0, stream, reinterpret_cast<const __nv_bfloat16*>(x),
                       perm_src, R, T, d, reinterpret_cast<__nv_bfloat16*>(x_perm));
        if ((st = check_launch("gather_rows", e)) != MOE_OK) return st;
    }
    return MOE_OK;
}

moe_status_t moe_permute_static_ws(const moe_bf16_t* x, const int32_t* topk_idx, int T, int d, int E, int k,
                                   int32_t* expert_counts, int32_t* expert_offsets, int32_t* perm_src,
                                   int32_t* inv_perm, moe_bf16_t* x_perm, cudaStream_t stream) {
    moe_status_t st = check_route_sizes(T, E, k);
    if (st != MOE_OK) return st;
    const size_t need = moe_permute_workspace_size(T, E, k);
    if (need > MOE_PERMUTE_STATIC_WS_BYTES)
        return fail(MOE_ERR_WORKSPACE,
                    "T=%d, E=%d, k=%d need %zu bytes of scratch; the library's static array holds %u (use moe_permute "
                    "with a workspace for larger sizes)",
                    T, E, k, need, (unsigned)MOE_PERMUTE_STATIC_WS_BYTES);
    void* ws = nullptr;
    if ((st = static_ws_address(&ws)) != MOE_OK) return st;
    return moe_permute(x, topk_idx, T, d, E, k, expert_counts, expert_offsets, perm_src, inv_perm, x_perm, ws,
                       MOE_PERMUTE_STATIC_WS_BYTES, stream);
}

moe_status_t moe_grouped_gemm_gateup(const moe_bf16_t* a, const moe_bf16_t* w_gateup, const int32_t* group_offsets,
                                     int G, int M, int d, int f, moe_bf16_t* h, cudaStream_t stream) {
    moe_status_t st = check_gemm_args(a, w_gateup, group_offsets, G, M, d, f, h);
    if (st != MOE_OK) return st;
    DeviceInfo di;
    if ((st = device_info(di)) != MOE_OK) return st;
    if (M == 0) return MOE_OK;
    const GemmProblem p{a, w_gateup, group_offsets, G, M, d, f, f, h};
    return launch_grouped_gemm(p, true, di.sms, stream);
}

size_t moe_grouped_gemm_gateup_gather_workspace_size(int G, int M, int d) {
    if (G < 1 || M <= 0 || d <= 0 || (long)M >= (long)G * GG_BM) return 0;
    return ((size_t)M * (size_t)d * 2 + 255) / 256 * 256;
}

moe_status_t moe_grouped_gemm_gateup_gather(const moe_bf16_t* x, const int32_t* row_src, int T,
                                            const moe_bf16_t* w_gateup, const int32_t* group_offsets, int G, int M,
                                            int d, int f, moe_bf16_t* h, void* ws, size_t ws_bytes,
                                            cudaStream_t stream) {
    moe_status_t st = check_gemm_args(x, w_gateup, group_offsets, G, M, d, f, h);
    if (st != MOE_OK) return st;
    if (T < 0 || (M > 0 && (T == 0 || !row_src))) return fail(MOE_ERR_INVALID_ARG, "x rows T=%d / row_src", T);
    if ((reinterpret_cast<uintptr_t>(row_src) & 3u) != 0) return fail(MOE_ERR_INVALID_ARG, "row_src misaligned");
    if ((long)T * (long)d > 0x7fffffffffffL) return fail(MOE_ERR_INVALID_ARG, "x too large");
    const size_t need = moe_grouped_gemm_gateup_gather_workspace_size(G, M, d);
    if (need && (!ws || ws_bytes < need))
        return fail(MOE_ERR_WORKSPACE, "workspace of %zu bytes needed, %zu given", need, ws ? ws_bytes : (size_t)0);
    if (need && !aligned16(ws)) return fail(MOE_ERR_WORKSPACE, "workspace not 16-byte aligned");
    DeviceInfo di;
    if ((st = device_info(di)) != MOE_OK) return st;
    if (M == 0) return MOE_OK;
    if (need == 0) {  // groups of 128 rows or more on average: the gather rides in the operand load
        if (di.sms < 2) return fail(MOE_ERR_UNSUPPORTED, "the gathering GEMM needs CTA pairs");
        GemmProblem p{x, w_gateup, group_offsets, G, M, d, f, f, h};
        p.row_src = row_src;
        p.src_rows = T;
        if (d % GG_BK == 0) return launch_swap<true, 2, 3, true, false, true>(p, di.sms, stream);
        return launch_swap<true, 2, 3, false, false, true>(p, di.sms, stream);
    }
    // a few rows per expert: gather the rows into the workspace, then the GEMM the shape calls for
    const int grid = grid_cap((M + 7) / 8, di.sms, 16);
    const cudaError_t e = launch_pdl(gather_rows_kernel, dim3(grid), dim3(256), 0, stream,
                                     reinterpret_cast<const __nv_bfloat16*>(x), row_src, M, T, d,
                                     reinterpret_cast<__nv_bfloat16*>(ws));
    if ((st = check_launch("gather_rows", e)) != MOE_OK) return st;
    const GemmProblem p{ws, w_gateup, group_offsets, G, M, d, f, f, h};
    return launch_grouped_gemm(p, true, di.sms, stream);
}

moe_status_t moe_gather_rows(const moe_bf16_t* x, const int32_t* row_src, int T, int d, int R, moe_bf16_t* out,
                             cudaStream_t stream) {
    if (T < 0 || R < 0) return fail(MOE_ERR_INVALID_ARG, "T=%d, R=%d must be >= 0", T, R);
    if (d < 8 || d % 8) return fail(MOE_ERR_INVALID_ARG, "d=%d must be a positive multiple of 8", d);
    if (R == 0) return MOE_OK;
    if (!x || !row_src || !out || T == 0) return fail(MOE_ERR_INVALID_ARG, "null pointer or T = 0");
    if (!aligned16(x) || !aligned16(out)) return fail(MOE_ERR_INVALID_ARG, "x / out not 16-byte aligned");
    if ((reinterpret_cast<uintptr_t>(row_src) & 3u) != 0) return fail(MOE_ERR_INVALID_ARG, "row_src misaligned");
    DeviceInfo di;
    moe_status_t st = device_info(di);
    if (st != MOE_OK) return st;
    const int grid = grid_cap((R + 7) / 8, di.sms, 16);
    const cudaError_t e = launch_pdl(gather_rows_kernel, dim3(grid), dim3(256), 0, stream,
                                     reinterpret_cast<const __nv_bfloat16*>(x), row_src, R, T, d,
                                     reinterpret_cast<__nv_bfloat16*>(out));
    return check_launch("gather_rows", e);
}

moe_status_t moe_grouped_gemm_down(const moe_bf16_t* h, const moe_bf16_t* w_down, const int32_t* group_offsets,
                                   int G, int M, int d, int f, moe_bf16_t* y, cudaStream_t stream) {
    moe_status_t st = check_gemm_args(h, w_down, group_offsets, G, M, d, f, y);
    if (st != MOE_OK) return st;
    DeviceInfo di;
    if ((st = device_info(di)) != MOE_OK) return st;
    if (M == 0) return MOE_OK;
    const GemmProblem p{h, w_down, group_offsets, G, M, f, d, f, y};
    return launch_grouped_gemm(p, false, di.sms, stream);
}

moe_status_t moe_mxfp4_quantize(const moe_bf16_t* w, int G, int N, int K, uint8_t* q, uint8_t* s,
                                cudaStream_t stream) {
    if (G < 0 || N < 0) return fail(MOE_ERR_INVALID_ARG, "G=%d, N=%d must be >= 0", G, N);
    if (K < 32 || K % 32) return fail(MOE_ERR_INVALID_ARG, "K=%d must be a positive multiple of 32", K);
    if (G == 0 || N == 0) return MOE_OK;
    if (!w || !q || !s) return fail(MOE_ERR_INVALID_ARG, "null pointer");
    if (!aligned16(w) || !aligned16(q)) return fail(MOE_ERR_INVALID_ARG, "w and q must be 16-byte aligned");
    DeviceInfo di;
    moe_status_t st = device_info(di);
    if (st != MOE_OK) return st;
    const long rows = (long)G * N;
    const long blocks = rows * (K / 32);
    const int grid = grid_cap((blocks + 255) / 256, di.sms, 8);
    const cudaError_t e = launch_pdl(mxfp4_quantize_kernel, dim3(grid), dim3(256), 0, stream,
                                     reinterpret_cast<const __nv_bfloat16*>(w), rows, N, K, q, s);
    return check_launch("mxfp4_quantize", e);
}

moe_status_t moe_grouped_gemm_gateup_mxfp4(const moe_bf16_t* a, const uint8_t* wq_gateup, const uint8_t* ws_gateup,
                                           const int32_t* group_offsets, int G, int M, int d, int f, moe_bf16_t* h,
                                           cudaStream_t stream) {
    moe_status_t st = check_fp4_args(a, wq_gateup, ws_gateup, group_offsets, G, M, d, f, h);
    if (st != MOE_OK) return st;
    DeviceInfo di;
    if ((st = device_info(di)) != MOE_OK) return st;
    if (M == 0) return MOE_OK;
    const Fp4Problem p{a, wq_gateup, ws_gateup, group_offsets, G, M, d, f, f, 2 * f, h};
    return launch_fp4_nt<true>(p, di.sms, stream);
}

moe_status_t moe_grouped_gemm_down_mxfp4(const moe_bf16_t* h, const uint8_t* wq_down, const uint8_t* ws_down,
                                         const int32_t* group_offsets, int G, int M, int d, int f, moe_bf16_t* y,
                                         cudaStream_t stream) {
    moe_status_t st = check_fp4_args(h, wq_down, ws_down, group_offsets, G, M, d, f, y);
    if (st != MOE_OK) return st;
    DeviceInfo di;
    if ((st = device_info(di)) != MOE_OK) return st;
    if (M == 0) return MOE_OK;
    const Fp4Problem p{h, wq_down, ws_down, group_offsets, G, M, f, d, f, d, y};
    return launch_fp4_nt<false>(p, di.sms, stream);
}

moe_status_t moe_unpermute_combine(const moe_bf16_t* y_perm, const int32_t* inv_perm, const float* topk_w,
                                   const moe_bf16_t* shared, int T, int d, int k, moe_bf16_t* y,
                                   cudaStream_t stream) {
    if (T < 0 || k < 1 || k > 32) return fail(MOE_ERR_INVALID_ARG, "T=%d, k=%d (need T >= 0, 1 <= k <= 32)", T, k);
    if (d < 8 || d % 8) return fail(MOE_ERR_INVALID_ARG, "d=%d must be a positive multiple of 8", d);
    if (T == 0) return MOE_OK;  // nothing to combine (the empty arrays' pointers may be null)
    if (!y_perm || !inv_perm || !topk_w || !y) return fail(MOE_ERR_INVALID_ARG, "null pointer");
    if (!aligned16(y_perm) || !aligned16(y) || (shared && !aligned16(shared)))
        return fail(MOE_ERR_INVALID_ARG, "bf16 tensors must be 16-byte aligned");
    if ((long)T * k > 0x7fffffffL) return fail(MOE_ERR_INVALID_ARG, "T*k exceeds int32");
    DeviceInfo di;
    moe_status_t st = device_info(di);
    if (st != MOE_OK) return st;
    const long items = (long)T * ((d / 8 + CB_CHUNK_VEC - 1) / CB_CHUNK_VEC);
    const int grid = grid_cap((items + 7) / 8, di.sms, 16);
    const cudaError_t e = launch_pdl(combine_kernel, dim3(grid), dim3(256), 0, stream,
                                     reinterpret_cast<const __nv_bfloat16*>(y_perm), inv_perm, topk_w,
                                     reinterpret_cast<const __nv_bfloat16*>(shared), T, d, k, T * k,
                                     reinterpret_cast<__nv_bfloat16*>(y));
    return check_launch("unpermute_combine", e);
}

size_t moe_grouped_gemm_down_combine_workspace_size(int T, int d) {
    if (T <= 0 || d <= 0) return 0;
    return ((size_t)T * (size_t)((d + 31) / 32) * sizeof(int32_t) + 255) / 256 * 256;
}

moe_status_t moe_grouped_gemm_down_combine(const moe_bf16_t* h, const moe_bf16_t* w_down,
                                           const int32_t* group_offsets, int G, int M, int d, int f,
                                           const int32_t* perm_src, const int32_t* inv_perm, const float* topk_w,
                                           const moe_bf16_t* shared, int T, int k, moe_bf16_t* y_perm, moe_bf16_t* y,
                                           void* ws, size_t ws_bytes, cudaStream_t stream) {
    moe_status_t st = check_gemm_args(h, w_down, group_offsets, G, M, d, f, y_perm);
    if (st != MOE_OK) return st;
    if (T < 0 || k < 1 || k > 32) return fail(MOE_ERR_INVALID_ARG, "T=%d, k=%d (need T >= 0, 1 <= k <= 32)", T, k);
    if ((long)T * k != (long)M) return fail(MOE_ERR_INVALID_ARG, "M=%d must be T*k=%ld", M, (long)T * k);
    if (T == 0) return MOE_OK;
    if (!perm_src || !inv_perm || !topk_w || !y) return fail(MOE_ERR_INVALID_ARG, "null pointer");
    if (!aligned16(y) || (shared && !aligned16(shared)))
        return fail(MOE_ERR_INVALID_ARG, "bf16 tensors must be 16-byte aligned");
    const size_t need = moe_grouped_gemm_down_combine_workspace_size(T, d);
    if (!ws || ws_bytes < need)
        return fail(MOE_ERR_WORKSPACE, "workspace of %zu bytes needed, %zu given", need, ws ? ws_bytes : (size_t)0);
    if ((reinterpret_cast<uintptr_t>(ws) & 15u) != 0) return fail(MOE_ERR_WORKSPACE, "workspace not 16-byte aligned");
    DeviceInfo di;
    if ((st = device_info(di)) != MOE_OK) return st;
    const GemmProblem p{h, w_down, group_offsets, G, M, f, d, f, y_perm};
    if ((long)M >= (long)G * GG_BM && di.sms >= 2) {  // prefill: the combine runs in the GEMM's epilogue
        cudaError_t e = cudaMemsetAsync(ws, 0, need, stream);  // arrival counters
        if (e != cudaSuccess) return fail(MOE_ERR_CUDA, "cudaMemsetAsync: %s", cudaGetErrorString(e));
        CombineArgs ca;
        ca.perm_src = perm_src;
        ca.inv_perm = inv_perm;
        ca.topk_w = topk_w;
        ca.shared = reinterpret_cast<const __nv_bfloat16*>(shared);
        ca.y = reinterpret_cast<__nv_bfloat16*>(y);
        ca.counters = reinterpret_cast<int*>(ws);
        ca.T = T;
        ca.k = k;
        if (f % GG_BK == 0) return launch_swap<false, 2, 3, true, false, false, true>(p, di.sms, stream, ca);
        return launch_swap<false, 2, 3, false, false, false, true>(p, di.sms, stream, ca);
    }
    // a few rows per expert: the GEMM the shape calls for, then the stand-alone combine
    if ((st = launch_grouped_gemm(p, false, di.sms, stream)) != MOE_OK) return st;
    return moe_unpermute_combine(y_perm, inv_perm, topk_w, shared, T, d, k, y, stream);
}

// ---- backward ----

moe_status_t moe_grouped_gemm_gateup_preact(const moe_bf16_t* a, const moe_bf16_t* w_gateup,
                                            const int32_t* group_offsets, int G, int M, int d, int f, moe_bf16_t* gu,
                                            cudaStream_t stream) {
    moe_status_t st = check_gemm_args(a, w_gateup, group_offsets, G, M, d, f, gu);
    if (st != MOE_OK) return st;
    DeviceInfo di;
    if ((st = device_info(di)) != MOE_OK) return st;
    if (M == 0) return MOE_OK;
    if (di.sms < 2) return fail(MOE_ERR_UNSUPPORTED, "the pre-activation GEMM needs CTA pairs");
    const GemmProblem p{a, w_gateup, group_offsets, G, M, d, f, f, gu};
    if (d % GG_BK == 0) return launch_swap<true, 2, 3, true, true>(p, di.sms, stream);
    return launch_swap<true, 2, 3, false, true>(p, di.sms, stream);
}

moe_status_t moe_grouped_gemm_gateup_save(const moe_bf16_t* a, const moe_bf16_t* w_gateup, const int32_t* group_offsets,
                                          int G, int M, int d, int f, moe_bf16_t* h, moe_bf16_t* gu,
                                          cudaStream_t stream) {
    moe_status_t st = check_gemm_args(a, w_gateup, group_offsets, G, M, d, f, h);
    if (st != MOE_OK) return st;
    if (M > 0 && !gu) return fail(MOE_ERR_INVALID_ARG, "null pointer argument");
    if (!aligned16(gu)) return fail(MOE_ERR_INVALID_ARG, "gu must be 16-byte aligned");
    DeviceInfo di;
    if ((st = device_info(di)) != MOE_OK) return st;
    if (M == 0) return MOE_OK;
    if (di.sms < 2) return fail(MOE_ERR_UNSUPPORTED, "the gate|up GEMM with saved pre-activations needs CTA pairs");
    GemmProblem p{a, w_gateup, group_offsets, G, M, d, f, f, h};
    if ((long)M >= (long)G * GG_BM) {  // prefill: one kernel writes h and g | u
        p.out2 = gu;
        if (d % GG_BK == 0) return launch_swap<true, 2, 3, true, false, false, false, true>(p, di.sms, stream);
        return launch_swap<true, 2, 3, false, false, false, false, true>(p, di.sms, stream);
    }
    // a few rows per expert: h as moe_grouped_gemm_gateup, then the pre-activation GEMM
    if ((st = launch_grouped_gemm(p, true, di.sms, stream)) != MOE_OK) return st;
    return moe_grouped_gemm_gateup_preact(a, w_gateup, group_offsets, G, M, d, f, gu, stream);
}

moe_status_t moe_swiglu_backward(const moe_bf16_t* dh, const moe_bf16_t* gu, int M, int f, moe_bf16_t* dgu,
                                 cudaStream_t stream) {
    if (M < 0 || f < 8 || f % 8) return fail(MOE_ERR_INVALID_ARG, "M=%d, f=%d (f a positive multiple of 8)", M, f);
    if (M == 0) return MOE_OK;
    if (!dh || !gu || !dgu) return fail(MOE_ERR_INVALID_ARG, "null pointer");
    if (!aligned16(dh) || !aligned16(gu) || !aligned16(dgu)) return fail(MOE_ERR_INVALID_ARG, "pointers must be 16-byte aligned");
    DeviceInfo di;
    moe_status_t st = device_info(di);
    if (st != MOE_OK) return st;
    const long items = (long)M * (f / 8);
    const cudaError_t e = launch_plain(swiglu_backward_kernel, dim3(grid_cap((items + 255) / 256, di.sms, 8)), dim3(256),
                                     0, stream, reinterpret_cast<const __nv_bfloat16*>(dh),
                                     reinterpret_cast<const __nv_bfloat16*>(gu), (long)M, f,
                                     reinterpret_cast<__nv_bfloat16*>(dgu));
    return check_launch("swiglu_backward", e);
}

moe_status_t moe_permute_backward(const moe_bf16_t* dy, const int32_t* inv_perm, const float* topk_w,
                                  const moe_bf16_t* y_perm, int T, int d, int k, moe_bf16_t* dy_perm, float* dw,
                                  cudaStream_t stream) {
    if (T < 0 || k < 1 || k > 32) return fail(MOE_ERR_INVALID_ARG, "T=%d, k=%d (need T >= 0, 1 <= k <= 32)", T, k);
    if (d < 8 || d % 8) return fail(MOE_ERR_INVALID_ARG, "d=%d must be a positive multiple of 8", d);
    if ((long)T * k > 0x7fffffffL) return fail(MOE_ERR_INVALID_ARG, "T*k exceeds int32");
    if (T == 0) return MOE_OK;
    if (!dy || !inv_perm || !topk_w || !y_perm || !dy_perm || !dw) return fail(MOE_ERR_INVALID_ARG, "null pointer");
    if (!aligned16(dy) || !aligned16(y_perm) || !aligned16(dy_perm))
        return fail(MOE_ERR_INVALID_ARG, "bf16 tensors must be 16-byte aligned");
    DeviceInfo di;
    moe_status_t st = device_info(di);
    if (st != MOE_OK) return st;
    const long R = (long)T * k;
    const cudaError_t e = launch_plain(permute_backward_kernel, dim3(grid_cap((R + PB_WARPS - 1) / PB_WARPS, di.sms, 16)),
                                     dim3(PB_WARPS * 32), 0, stream, reinterpret_cast<const __nv_bfloat16*>(dy),
                                     inv_perm, topk_w, reinterpret_cast<const __nv_bfloat16*>(y_perm), T, d, k,
                                     reinterpret_cast<__nv_bfloat16*>(dy_perm), dw);
    return check_launch("permute_backward", e);
}

moe_status_t moe_transpose_weights(const moe_bf16_t* w, int G, int rows, int cols, moe_bf16_t* wt,
                                   cudaStream_t stream) {
    if (G < 0 || rows < 0 || cols < 0 || G > 65535) return fail(MOE_ERR_INVALID_ARG, "G=%d, rows=%d, cols=%d", G, rows, cols);
    if (G == 0 || rows == 0 || cols == 0) return MOE_OK;
    if (!w || !wt) return fail(MOE_ERR_INVALID_ARG, "null pointer");
    if (w == wt) return fail(MOE_ERR_INVALID_ARG, "the transpose cannot be done in place");
    DeviceInfo di;
    moe_status_t st = device_info(di);
    if (st != MOE_OK) return st;
    const dim3 grid((cols + 31) / 32, (rows + 31) / 32, G);
    if (grid.y > 65535) return fail(MOE_ERR_INVALID_ARG, "rows=%d too large", rows);
    const cudaError_t e = launch_plain(transpose_kernel, grid, dim3(256), 0, stream,
                                     reinterpret_cast<const __nv_bfloat16*>(w), rows, cols,
                                     reinterpret_cast<__nv_bfloat16*>(wt));
    return check_launch("transpose", e);
}

namespace {
long wgrad_cap(int M, int G) { return ((long)M + (long)(WG_PAD - 1) * G + WG_PAD - 1) / WG_PAD * WG_PAD; }
size_t round256(size_t b) { return (b + 255) / 256 * 256; }
}  // namespace

size_t moe_grouped_weight_grad_workspace_size(int M, int G, int P, int Q) {
    if (M <= 0 || G <= 0 || P <= 0 || Q <= 0) return 0;
    const long cap = wgrad_cap(M, G);
    return round256((size_t)(G + 1) * 4) + round256((size_t)P * cap * 2) + round256((size_t)Q * cap * 2);
}

moe_status_t moe_grouped_weight_grad(const moe_bf16_t* a, const moe_bf16_t* b, const int32_t* group_offsets, int G,
                                     int M, int P, int Q, float* dw, void* ws, size_t ws_bytes, cudaStream_t stream) {
    if (G < 1 || G > GG_MAX_GROUPS) return fail(MOE_ERR_INVALID_ARG, "G=%d outside [1, %d]", G, GG_MAX_GROUPS);
    if (M < 0) return fail(MOE_ERR_INVALID_ARG, "M=%d < 0", M);
    if (P < 8 || Q < 8 || P % 8 || Q % 8) return fail(MOE_ERR_INVALID_ARG, "P=%d and Q=%d must be positive multiples of 8", P, Q);
    if (!group_offsets || !dw || (M > 0 && (!a || !b))) return fail(MOE_ERR_INVALID_ARG, "null pointer");
    if (!aligned16(a) || !aligned16(b) || !aligned16(dw)) return fail(MOE_ERR_INVALID_ARG, "pointers must be 16-byte aligned");
    if ((reinterpret_cast<uintptr_t>(group_offsets) & 3u) != 0) return fail(MOE_ERR_INVALID_ARG, "offsets misaligned");
    const int Mw = M > 0 ? M : 1;
    const size_t need = moe_grouped_weight_grad_workspace_size(Mw, G, P, Q);
    if (!ws || ws_bytes < need)
        return fail(MOE_ERR_WORKSPACE, "workspace of %zu bytes needed, %zu given", need, ws ? ws_bytes : (size_t)0);
    if (reinterpret_cast<uintptr_t>(ws) & 255u) return fail(MOE_ERR_WORKSPACE, "workspace not 256-byte aligned");
    DeviceInfo di;
    moe_status_t st = device_info(di);
    if (st != MOE_OK) return st;
    if (di.sms < 2) return fail(MOE_ERR_UNSUPPORTED, "the weight-gradient GEMM needs CTA pairs");
    const long cap = wgrad_cap(Mw, G);
    uint8_t* base = reinterpret_cast<uint8_t*>(ws);
    int32_t* pad_off = reinterpret_cast<int32_t*>(base);
    __nv_bfloat16* aT = reinterpret_cast<__nv_bfloat16*>(base + round256((size_t)(G + 1) * 4));
    __nv_bfloat16* bT = reinterpret_cast<__nv_bfloat16*>(reinterpret_cast<uint8_t*>(aT) + round256((size_t)P * cap * 2));
    cudaError_t e = launch_plain(pad_offsets_kernel, dim3(1), dim3(1024), 0, stream, group_offsets, G, M, pad_off);
    if ((st = check_launch("pad_offsets", e)) != MOE_OK) return st;
    if (M > 0) {
        if (cap / TP_TILE > 65535) return fail(MOE_ERR_INVALID_ARG, "M=%d too large for the weight-gradient transpose", M);
        e = launch_plain(transpose_pad_kernel, dim3((P + TP_TILE - 1) / TP_TILE, (unsigned)(cap / TP_TILE)), dim3(256), 0, stream,
                       reinterpret_cast<const __nv_bfloat16*>(a), group_offsets, (const int32_t*)pad_off, G, M, P, cap, aT);
        if ((st = check_launch("transpose_pad", e)) != MOE_OK) return st;
        e = launch_plain(transpose_pad_kernel, dim3((Q + TP_TILE - 1) / TP_TILE, (unsigned)(cap / TP_TILE)), dim3(256), 0, stream,
                       reinterpret_cast<const __nv_bfloat16*>(b), group_offsets, (const int32_t*)pad_off, G, M, Q, cap, bT);
        if ((st = check_launch("transpose_pad", e)) != MOE_OK) return st;
    }
    CUtensorMap ta, tb, to;
    const cuuint64_t adims[2] = {(cuuint64_t)cap, (cuuint64_t)P};
    const cuuint64_t astr[1] = {(cuuint64_t)cap * 2};
    const cuuint32_t box[2] = {GG_BK, 128};
    if ((st = make_tmap(&ta, aT, 2, adims, astr, box)) != MOE_OK) return st;
    const cuuint64_t bdims[2] = {(cuuint64_t)cap, (cuuint64_t)Q};
    if ((st = make_tmap(&tb, bT, 2, bdims, astr, box)) != MOE_OK) return st;
    const cuuint64_t odims[3] = {(cuuint64_t)Q, (cuuint64_t)P, (cuuint64_t)G};
    const cuuint64_t ostr[2] = {(cuuint64_t)Q * 4, (cuuint64_t)P * Q * 4};
    const cuuint32_t obox[3] = {32, 32, 1};
    if ((st = make_tmap(&to, dw, 3, odims, ostr, obox, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, CU_TENSOR_MAP_SWIZZLE_128B)) !=
        MOE_OK)
        return st;
    WgradArgs args;
    args.pad_off = pad_off;
    args.G = G;
    args.P = P;
    args.Q = Q;
    const long tiles = (long)G * ((P + WG_TILE - 1) / WG_TILE) * ((Q + WG_TILE - 1) / WG_TILE);
    const int clusters = (int)(tiles < di.sms / 2 ? tiles : di.sms / 2);
    e = launch_pdl(grouped_wgrad_kernel, dim3(2 * clusters), dim3(WG_THREADS), GemmWgradShape::SMEM_BYTES, stream, ta,
                   tb, to, args);
    return check_launch("grouped_weight_grad", e);
}

namespace {
// router backward workspace: dl_tk [T*k] | dl_perm [T*k] | chunk_prefix [E+1] | pbias [chunks] | partial [chunks][d]
long router_chunks_cap(int T, int E, int k) { return ((long)T * k + RB_ROWS - 1) / RB_ROWS + E; }
}  // namespace

size_t moe_router_backward_workspace_size(int T, int d, int E, int k) {
    if (T <= 0 || k <= 0 || E <= 0 || d <= 0) return 0;
    const long chunks = router_chunks_cap(T, E, k);
    return round256((size_t)T * k * 4) * 2 + round256((size_t)(E + 1) * 4) + round256((size_t)chunks * 4) +
           round256((size_t)chunks * d * 4);
}

moe_status_t moe_router_backward(const moe_bf16_t* x, const float* w_router, const float* logits,
                                 const int32_t* topk_idx, const float* topk_w, const float* dw,
                                 const int32_t* perm_src, const int32_t* inv_perm, const int32_t* expert_offsets,
                                 int T, int d, int E, int k, moe_route_mode_t mode, const moe_bf16_t* dx_addend,
                                 moe_bf16_t* dx, float* dw_router, float* dbias, void* ws, size_t ws_bytes,
                                 cudaStream_t stream) {
    moe_status_t st = check_route_sizes(T, E, k);
    if (st != MOE_OK) return st;
    if (mode < MOE_ROUTE_TOPK_SOFTMAX || mode > MOE_ROUTE_SIGMOID_TOPK_NORM)
        return fail(MOE_ERR_INVALID_ARG, "unknown routing mode %d", (int)mode);
    if (d < 8 || d % 8) return fail(MOE_ERR_INVALID_ARG, "d=%d must be a positive multiple of 8", d);
    if (!dw_router || !expert_offsets) return fail(MOE_ERR_INVALID_ARG, "null pointer");
    DeviceInfo di;
    if ((st = device_info(di)) != MOE_OK) return st;
    if (T == 0) {  // no tokens: the router's weight gradient (and the bias gradient) is zero
        cudaError_t e = cudaMemsetAsync(dw_router, 0, sizeof(float) * (size_t)E * d, stream);
        if (e == cudaSuccess && dbias) e = cudaMemsetAsync(dbias, 0, sizeof(float) * (size_t)E, stream);
        if (e != cudaSuccess) return fail(MOE_ERR_CUDA, "cudaMemsetAsync: %s", cudaGetErrorString(e));
        return MOE_OK;
    }
    if (!x || !w_router || !logits || !topk_idx || !topk_w || !dw || !perm_src || !inv_perm || !dx)
        return fail(MOE_ERR_INVALID_ARG, "null pointer");
    if (!aligned16(x) || !aligned16(w_router) || !aligned16(dx) || (dx_addend && !aligned16(dx_addend)))
        return fail(MOE_ERR_INVALID_ARG, "x, w_router, dx and dx_addend must be 16-byte aligned");
    const size_t need = moe_router_backward_workspace_size(T, d, E, k);
    if (!ws || ws_bytes < need)
        return fail(MOE_ERR_WORKSPACE, "workspace of %zu bytes needed, %zu given", need, ws ? ws_bytes : (size_t)0);
    if (reinterpret_cast<uintptr_t>(ws) & 255u) return fail(MOE_ERR_WORKSPACE, "workspace not 256-byte aligned");
    const long chunks = router_chunks_cap(T, E, k);
    if (chunks > 65535) return fail(MOE_ERR_INVALID_ARG, "T*k=%ld too large for the router backward", (long)T * k);
    uint8_t* base = reinterpret_cast<uint8_t*>(ws);
    float* dl_tk = reinterpret_cast<float*>(base);
    base += round256((size_t)T * k * 4);
    float* dl_perm = reinterpret_cast<float*>(base);
    base += round256((size_t)T * k * 4);
    int32_t* chunk_prefix = reinterpret_cast<int32_t*>(base);
    base += round256((size_t)(E + 1) * 4);
    float* pbias = reinterpret_cast<float*>(base);
    base += round256((size_t)chunks * 4);
    float* partial = reinterpret_cast<float*>(base);
    const int R = T * k;
    cudaError_t e = launch_plain(router_dlogits_kernel, dim3(grid_cap((T + 255) / 256, di.sms, 4)), dim3(256), 0,
                               stream, logits, topk_idx, topk_w, dw, inv_perm, T, E, k, (int)mode, dl_tk, dl_perm);
    if ((st = check_launch("router_dlogits", e)) != MOE_OK) return st;
    e = launch_plain(router_chunk_prefix_kernel, dim3(1), dim3(1024), 0, stream, expert_offsets, E, R, chunk_prefix);
    if ((st = check_launch("router_chunk_prefix", e)) != MOE_OK) return st;
    e = launch_plain(router_chunk_partial_kernel, dim3((d + RB_COLS - 1) / RB_COLS, (unsigned)chunks), dim3(RB_COLS), 0,
                     stream, reinterpret_cast<const __nv_bfloat16*>(x), perm_src, expert_offsets,
                     (const int32_t*)chunk_prefix, (const float*)dl_perm, T, d, E, R, partial, pbias);
    if ((st = check_launch("router_chunk_partial", e)) != MOE_OK) return st;
    e = launch_plain(router_chunk_reduce_kernel, dim3((d + RB_COLS - 1) / RB_COLS, E), dim3(RB_COLS), 0, stream,
                     (const int32_t*)chunk_prefix, (const float*)partial, (const float*)pbias, d, E, dw_router, dbias);
    if ((st = check_launch("router_chunk_reduce", e)) != MOE_OK) return st;
    e = launch_plain(router_input_grad_kernel, dim3(grid_cap((T + 7) / 8, di.sms, 16)), dim3(256), 0, stream, topk_idx,
                   (const float*)dl_tk, w_router, reinterpret_cast<const __nv_bfloat16*>(dx_addend), T, d, E, k,
                   reinterpret_cast<__nv_bfloat16*>(dx));
    return check_launch("router_input_grad", e);
}

moe_status_t moe_set_gemm_kernel(moe_gemm_kernel_t kind) {
    if (kind < MOE_GEMM_AUTO || kind > MOE_GEMM_SWAP) return fail(MOE_ERR_INVALID_ARG, "unknown GEMM kernel %d", (int)kind);
    g_gemm_kernel.store((int)kind, std::memory_order_relaxed);
    return MOE_OK;
}

moe_status_t moe_test_set_wait(unsigned long long limit_ns, int stall) {
    if (limit_ns == 0) limit_ns = kWaitLimitNs;
    DeviceInfo di;
    moe_status_t st = device_info(di);
    if (st != MOE_OK) return st;
    const int flag = stall ? 1 : 0;
    cudaError_t e = cudaDeviceSynchronize();  // no kernel of this device is waiting while the values change
    if (e == cudaSuccess) e = cudaMemcpyToSymbol(g_wait_limit_ns, &limit_ns, sizeof limit_ns);
    if (e == cudaSuccess) e = cudaMemcpyToSymbol(g_wait_stall, &flag, sizeof flag);
    if (e != cudaSuccess) return fail(MOE_ERR_CUDA, "setting the wait limit: %s", cudaGetErrorString(e));
    return MOE_OK;
}

moe_status_t moe_get_device_error(unsigned int* out, cudaStream_t stream) {
    if (!out) return fail(MOE_ERR_INVALID_ARG, "null pointer");
    cudaError_t e = cudaStreamSynchronize(stream);
    unsigned int v = 0;
    if (e == cudaSuccess) e = cudaMemcpyFromSymbol(&v, g_device_error, sizeof v);
    const unsigned int zero = 0;
    if (e == cudaSuccess) e = cudaMemcpyToSymbol(g_device_error, &zero, sizeof zero);
    if (e != cudaSuccess) return fail(MOE_ERR_CUDA, "reading the device error word: %s", cudaGetErrorString(e));
    *out = v;
    return v ? MOE_ERR_DEVICE : MOE_OK;
}

const char* moe_last_error_string(void) { return t_last_error.c_str(); }

}  // extern "C"
