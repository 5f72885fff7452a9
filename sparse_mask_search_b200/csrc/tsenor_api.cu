// Host side of the C ABI declared in include/tsenor.h: argument checks,
// dispatch on M and dtype, stream-ordered launches, the failure counter.
#include <cstdio>
#include <cstring>
#include <mutex>
#include <new>
#include <type_traits>

#include <cudaTypedefs.h>

#include "../../include/tsenor.h"
#include "common.cuh"
#include "dykstra.cuh"
#include "round_warp.cuh"
#include "round_group.cuh"
#include "fused.cuh"
#include "objective.cuh"

namespace tsenor {
namespace {

thread_local char g_last_error[256] = "";

tsenor_status cuda_fail(cudaError_t e, const char* what) {
    std::snprintf(g_last_error, sizeof(g_last_error), "%s: %s", what, cudaGetErrorString(e));
    return TSENOR_ERR_CUDA;
}

bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

tsenor_status check_common(const void* W, int dtype, int64_t rows, int64_t cols, int N, int M) {
    if (M != 4 && M != 8 && M != 16 && M != 32 && M != 64) return TSENOR_ERR_UNSUPPORTED_M;
    if (dtype != TSENOR_F32 && dtype != TSENOR_BF16) return TSENOR_ERR_ARG;
    if (N < 1 || N > M) return TSENOR_ERR_ARG;
    if (rows < 0 || cols < 0 || rows % M || cols % M) return TSENOR_ERR_SHAPE;
    if (rows > (int64_t(1) << 31) || cols > (int64_t(1) << 31)) return TSENOR_ERR_SHAPE;
    if (rows == 0 || cols == 0) return TSENOR_OK;
    if (!W || !aligned(W, 16)) return TSENOR_ERR_ARG;
    return TSENOR_OK;
}

// EXT = warm start / stop rule / potentials export (tsenor_mask_warm, tsenor_plan_warm).
// Tensor map of W for the TMA tile copies: a rows x cols row-major matrix of
// T::storage, box M x M.  cuTensorMapEncodeTiled is fetched from the driver
// once (no link against the driver library).
PFN_cuTensorMapEncodeTiled g_encode_tiled = nullptr;
std::once_flag g_encode_once;

template <typename T>
cudaError_t encode_w_map(CUtensorMap* map, const void* W, int64_t rows, int64_t cols, int M) {
    std::call_once(g_encode_once, [] {
        void* fn = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            g_encode_tiled = reinterpret_cast<PFN_cuTensorMapEncodeTiled>(fn);
    });
    if (!g_encode_tiled) return cudaErrorNotSupported;
    constexpr size_t es = sizeof(typename T::storage);
    const cuuint64_t dims[2] = {cuuint64_t(cols), cuuint64_t(rows)};
    const cuuint64_t strides[1] = {cuuint64_t(cols) * es};          // bytes, a multiple of 16 (cols % 16 == 0)
    const cuuint32_t box[2] = {cuuint32_t(M), cuuint32_t(M)};       // inner box M * es bytes, a multiple of 16
    const cuuint32_t estr[2] = {1, 1};
    const CUtensorMapDataType dt = std::is_same<T, BF16>::value ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16
                                                                : CU_TENSOR_MAP_DATA_TYPE_FLOAT32;
    const CUresult r = g_encode_tiled(map, dt, 2, const_cast<void*>(W), dims, strides, box, estr,
                                      CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
                                      CU_TENSOR_MAP_L2_PROMOTION_L2_128B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

template <int M, typename T, bool EXT>
cudaError_t launch_plan(const void* W, int64_t rows, int64_t cols, int N, float tau, int iters,
                        float* plan, cudaStream_t st, const DykstraExt& ext) {
    const int64_t nb = (rows / M) * (cols / M);
    const auto* w = static_cast<const typename T::storage*>(W);
    if constexpr (M <= 8) {
        const int64_t grid = (nb + 127) / 128;
        constexpr size_t smem = sizeof(float) * 128 * thread_y0_stride<M>();
        static_assert(smem <= 48 * 1024, "default dynamic shared memory limit");
        dykstra_thread_kernel<M, T, EXT><<<dim3(unsigned(grid)), 128, smem, st>>>(w, cols, nb, N, tau, iters, plan,
                                                                                   ext);
    } else {
        CUtensorMap map;
        cudaError_t e = encode_w_map<T>(&map, W, rows, cols, M);
        if (e != cudaSuccess) return e;
        constexpr size_t smem = dykstra_tile_smem<M, T>();
        e = cudaFuncSetAttribute(dykstra_tile_kernel<M, T, EXT>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 int(smem));
        if (e != cudaSuccess) return e;
        const int64_t grid = (nb + TileCfg<M>::BPC - 1) / TileCfg<M>::BPC;
        dykstra_tile_kernel<M, T, EXT><<<dim3(unsigned(grid)), TileCfg<M>::THREADS, smem, st>>>(
            map, cols, nb, N, tau, iters, plan, ext);
    }
    return cudaGetLastError();
}

template <int M, typename T>
cudaError_t launch_round(const float* plan, const void* W, int64_t rows, int64_t cols, int N,
                         int sweeps, uint32_t* mask, cudaStream_t st) {
    const int64_t nb = (rows / M) * (cols / M);
    const int64_t wpr = (cols + 31) / 32;
    if (M == 4 || ((M == 8 || M == 16) && cols % 32)) {
        // rows narrower than a word: zero first so padding bits are 0 (and M = 4 can OR)
        cudaError_t e = cudaMemsetAsync(mask, 0, size_t(rows) * size_t(wpr) * 4, st);
        if (e != cudaSuccess) return e;
    }
    if constexpr (M <= 8) {
        constexpr size_t smem = round_group_smem<M>();
        constexpr int64_t bpc = 4 * GroupRound<M>::BPW;
        cudaError_t e = cudaFuncSetAttribute(round_group_kernel<M, T>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             int(smem));
        if (e != cudaSuccess) return e;
        round_group_kernel<M, T><<<dim3(unsigned((nb + bpc - 1) / bpc)), 128, smem, st>>>(
            plan, static_cast<const typename T::storage*>(W), cols, nb, N, sweeps, mask, wpr);
    } else if constexpr (M == 64) {
        constexpr size_t smem = sizeof(Round64Smem<typename KeyOf<T>::type>);
        cudaError_t e = cudaFuncSetAttribute(round_cta64_kernel<T>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             int(smem));
        if (e != cudaSuccess) return e;
        round_cta64_kernel<T><<<dim3(unsigned(nb)), 128, smem, st>>>(
            plan, static_cast<const typename T::storage*>(W), cols, nb, N, sweeps, mask, wpr);
    } else {
        constexpr size_t smem = round_warp_smem<M>();
        cudaError_t e = cudaFuncSetAttribute(round_warp_kernel<M, T>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             int(smem));
        if (e != cudaSuccess) return e;
        const int64_t grid = (nb + 3) / 4;
        round_warp_kernel<M, T><<<dim3(unsigned(grid)), 128, smem, st>>>(
            plan, static_cast<const typename T::storage*>(W), cols, nb, N, sweeps, mask, wpr);
    }
    return cudaGetLastError();
}

// Whole path in one kernel (M = 16, 32, 64): no workspace.
template <int M, typename T, bool EXT>
cudaError_t launch_fused(const void* W, int64_t rows, int64_t cols, int N, float tau, int iters, int sweeps,
                         uint32_t* mask, cudaStream_t st, const DykstraExt& ext) {
    const int64_t nb = (rows / M) * (cols / M);
    const int64_t wpr = (cols + 31) / 32;
    cudaError_t e = cudaSuccess;
    if constexpr (M <= 8) {
        if (M == 4 || cols % 32) {
            // sub-word rows: zero first so padding bits are 0 (and M = 4 can OR)
            e = cudaMemsetAsync(mask, 0, size_t(rows) * size_t(wpr) * 4, st);
            if (e != cudaSuccess) return e;
        }
        constexpr size_t smem = FusedSmallCfg<M>::bytes;
        e = cudaFuncSetAttribute(fused_kernel_small<M, T, EXT>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 int(smem));
        if (e != cudaSuccess) return e;
        constexpr int64_t bpc = FusedSmallCfg<M>::THREADS;
        fused_kernel_small<M, T, EXT><<<dim3(unsigned((nb + bpc - 1) / bpc)), FusedSmallCfg<M>::THREADS, smem, st>>>(
            static_cast<const typename T::storage*>(W), cols, nb, N, tau, iters, sweeps, mask, wpr, ext);
    } else if constexpr (M == 32) {
        CUtensorMap map;
        e = encode_w_map<T>(&map, W, rows, cols, M);
        if (e != cudaSuccess) return e;
        constexpr size_t smem = fused32_smem();
        e = cudaFuncSetAttribute(fused_kernel32<T, EXT>, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem));
        if (e != cudaSuccess) return e;
        fused_kernel32<T, EXT><<<dim3(unsigned((nb + 3) / 4)), 128, smem, st>>>(map, cols, nb, N, tau, iters, sweeps,
                                                                               mask, wpr, ext);
    } else if constexpr (M == 16) {
        CUtensorMap w;
        e = encode_w_map<T>(&w, W, rows, cols, M);
        if (e != cudaSuccess) return e;
        if (cols % 32) {
            e = cudaMemsetAsync(mask, 0, size_t(rows) * size_t(wpr) * 4, st);   // padding bits
            if (e != cudaSuccess) return e;
        }
        constexpr size_t smem = fused16_smem();
        e = cudaFuncSetAttribute(fused_kernel16<T, EXT>, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem));
        if (e != cudaSuccess) return e;
        fused_kernel16<T, EXT><<<dim3(unsigned((nb + 15) / 16)), 128, smem, st>>>(w, cols, nb, N, tau, iters, sweeps,
                                                                                 mask, wpr, ext);
    } else {
        CUtensorMap w;
        e = encode_w_map<T>(&w, W, rows, cols, M);
        if (e != cudaSuccess) return e;
        constexpr size_t smem = sizeof(Round64Smem<typename KeyOf<T>::type>);
        e = cudaFuncSetAttribute(fused_kernel64<T, EXT>, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem));
        if (e != cudaSuccess) return e;
        fused_kernel64<T, EXT><<<dim3(unsigned(nb)), 128, smem, st>>>(w, cols, nb, N, tau, iters, sweeps, mask, wpr,
                                                                     ext);
    }
    return cudaGetLastError();
}

// ext == nullptr: the plain solve; otherwise the EXT kernels with *ext.
template <typename T, bool EXT>
cudaError_t dispatch_fused_m(int M, const void* W, int64_t rows, int64_t cols, int N, float tau, int iters,
                             int sweeps, uint32_t* mask, cudaStream_t st, const DykstraExt& ext) {
    switch (M) {
        case 4: return launch_fused<4, T, EXT>(W, rows, cols, N, tau, iters, sweeps, mask, st, ext);
        case 8: return launch_fused<8, T, EXT>(W, rows, cols, N, tau, iters, sweeps, mask, st, ext);
        case 16: return launch_fused<16, T, EXT>(W, rows, cols, N, tau, iters, sweeps, mask, st, ext);
        case 32: return launch_fused<32, T, EXT>(W, rows, cols, N, tau, iters, sweeps, mask, st, ext);
        default: return launch_fused<64, T, EXT>(W, rows, cols, N, tau, iters, sweeps, mask, st, ext);
    }
}

template <typename T>
cudaError_t dispatch_fused(int M, const void* W, int64_t rows, int64_t cols, int N, float tau, int iters, int sweeps,
                           uint32_t* mask, cudaStream_t st, const DykstraExt* ext = nullptr) {
    return ext ? dispatch_fused_m<T, true>(M, W, rows, cols, N, tau, iters, sweeps, mask, st, *ext)
               : dispatch_fused_m<T, false>(M, W, rows, cols, N, tau, iters, sweeps, mask, st, DykstraExt{});
}

template <typename T, bool EXT>
cudaError_t dispatch_plan_m(int M, const void* W, int64_t rows, int64_t cols, int N, float tau, int iters,
                            float* plan, cudaStream_t st, const DykstraExt& ext) {
    switch (M) {
        case 4: return launch_plan<4, T, EXT>(W, rows, cols, N, tau, iters, plan, st, ext);
        case 8: return launch_plan<8, T, EXT>(W, rows, cols, N, tau, iters, plan, st, ext);
        case 16: return launch_plan<16, T, EXT>(W, rows, cols, N, tau, iters, plan, st, ext);
        case 32: return launch_plan<32, T, EXT>(W, rows, cols, N, tau, iters, plan, st, ext);
        default: return launch_plan<64, T, EXT>(W, rows, cols, N, tau, iters, plan, st, ext);
    }
}

template <typename T>
cudaError_t dispatch_plan(int M, const void* W, int64_t rows, int64_t cols, int N, float tau, int iters,
                          float* plan, cudaStream_t st, const DykstraExt* ext = nullptr) {
    return ext ? dispatch_plan_m<T, true>(M, W, rows, cols, N, tau, iters, plan, st, *ext)
               : dispatch_plan_m<T, false>(M, W, rows, cols, N, tau, iters, plan, st, DykstraExt{});
}

template <typename T>
cudaError_t dispatch_round(int M, const float* plan, const void* W, int64_t rows, int64_t cols, int N,
                           int sweeps, uint32_t* mask, cudaStream_t st) {
    switch (M) {
        case 4: return launch_round<4, T>(plan, W, rows, cols, N, sweeps, mask, st);
        case 8: return launch_round<8, T>(plan, W, rows, cols, N, sweeps, mask, st);
        case 16: return launch_round<16, T>(plan, W, rows, cols, N, sweeps, mask, st);
        case 32: return launch_round<32, T>(plan, W, rows, cols, N, sweeps, mask, st);
        default: return launch_round<64, T>(plan, W, rows, cols, N, sweeps, mask, st);
    }
}

cudaError_t run_plan(int dtype, int M, const void* W, int64_t rows, int64_t cols, int N, float tau,
                     int iters, float* plan, cudaStream_t st, const DykstraExt* ext = nullptr) {
    return dtype == TSENOR_BF16 ? dispatch_plan<BF16>(M, W, rows, cols, N, tau, iters, plan, st, ext)
                                : dispatch_plan<F32>(M, W, rows, cols, N, tau, iters, plan, st, ext);
}

cudaError_t run_round(int dtype, int M, const float* plan, const void* W, int64_t rows, int64_t cols,
                      int N, int sweeps, uint32_t* mask, cudaStream_t st) {
    return dtype == TSENOR_BF16 ? dispatch_round<BF16>(M, plan, W, rows, cols, N, sweeps, mask, st)
                                : dispatch_round<F32>(M, plan, W, rows, cols, N, sweeps, mask, st);
}

bool solver_params_ok(float tau, int iters) {
    return tau > 0.f && tau <= kMaxTau && iters >= 1;
}

// Arguments of the warm-start entry points beyond the plain ones.
bool warm_params_ok(float tol, int warm, const float* potentials, const int32_t* iters_used) {
    if (!(tol >= 0.f) || tol > 3.0e38f) return false;            // NaN, negative or infinite
    if (warm && !potentials) return false;
    if (potentials && !aligned(potentials, 4)) return false;
    if (iters_used && !aligned(iters_used, 4)) return false;
    return true;
}

}  // namespace
}  // namespace tsenor

using namespace tsenor;

extern "C" tsenor_status tsenor_plan(const void* W, tsenor_dtype dtype, int64_t rows, int64_t cols, int N,
                                     int M, float tau, int iters, float* plan_out, tsenor_stream_t stream) {
    tsenor_status s = check_common(W, dtype, rows, cols, N, M);
    if (s != TSENOR_OK) return s;
    if (!solver_params_ok(tau, iters)) return TSENOR_ERR_ARG;
    if (rows == 0 || cols == 0) return TSENOR_OK;
    if (!plan_out || !aligned(plan_out, 16)) return TSENOR_ERR_ARG;
    cudaError_t e = run_plan(dtype, M, W, rows, cols, N, tau, iters, plan_out, (cudaStream_t)stream);
    return e == cudaSuccess ? TSENOR_OK : cuda_fail(e, "tsenor_plan launch");
}

extern "C" tsenor_status tsenor_round(const float* plan, const void* W, tsenor_dtype dtype, int64_t rows,
                                      int64_t cols, int N, int M, int sweeps, uint32_t* mask_out,
                                      tsenor_stream_t stream) {
    tsenor_status s = check_common(W, dtype, rows, cols, N, M);
    if (s != TSENOR_OK) return s;
    if (sweeps < 0) return TSENOR_ERR_ARG;
    if (rows == 0 || cols == 0) return TSENOR_OK;
    if (!plan || !aligned(plan, 16) || !mask_out || !aligned(mask_out, 8)) return TSENOR_ERR_ARG;
    cudaError_t e = run_round(dtype, M, plan, W, rows, cols, N, sweeps, mask_out, (cudaStream_t)stream);
    return e == cudaSuccess ? TSENOR_OK : cuda_fail(e, "tsenor_round launch");
}

extern "C" tsenor_status tsenor_mask(const void* W, tsenor_dtype dtype, int64_t rows, int64_t cols, int N,
                                     int M, float tau, int iters, int sweeps, uint32_t* mask_out,
                                     tsenor_stream_t stream) {
    tsenor_status s = check_common(W, dtype, rows, cols, N, M);
    if (s != TSENOR_OK) return s;
    if (!solver_params_ok(tau, iters) || sweeps < 0) return TSENOR_ERR_ARG;
    if (rows == 0 || cols == 0) return TSENOR_OK;
    if (!mask_out || !aligned(mask_out, 8)) return TSENOR_ERR_ARG;
    cudaStream_t st = (cudaStream_t)stream;
    cudaError_t e = dtype == TSENOR_BF16 ? dispatch_fused<BF16>(M, W, rows, cols, N, tau, iters, sweeps, mask_out, st)
                                         : dispatch_fused<F32>(M, W, rows, cols, N, tau, iters, sweeps, mask_out, st);
    return e == cudaSuccess ? TSENOR_OK : cuda_fail(e, "tsenor_mask launch");
}

extern "C" tsenor_status tsenor_mask_scores(const float* scores, int64_t rows, int64_t cols, int N, int M, float tau,
                                            int iters, int sweeps, uint32_t* mask_out, tsenor_stream_t stream) {
    return tsenor_mask(scores, TSENOR_F32, rows, cols, N, M, tau, iters, sweeps, mask_out, stream);
}

extern "C" tsenor_status tsenor_mask_warm(const void* W, tsenor_dtype dtype, int64_t rows, int64_t cols, int N,
                                          int M, float tau, int iters, int sweeps, float tol, int warm,
                                          float* potentials, int32_t* iters_used, uint32_t* mask_out,
                                          tsenor_stream_t stream) {
    tsenor_status s = check_common(W, dtype, rows, cols, N, M);
    if (s != TSENOR_OK) return s;
    if (!solver_params_ok(tau, iters) || sweeps < 0) return TSENOR_ERR_ARG;
    if (!warm_params_ok(tol, warm, potentials, iters_used)) return TSENOR_ERR_ARG;
    if (rows == 0 || cols == 0) return TSENOR_OK;
    if (!mask_out || !aligned(mask_out, 8)) return TSENOR_ERR_ARG;
    cudaStream_t st = (cudaStream_t)stream;
    const DykstraExt ext{potentials, iters_used, tol * kLog2e, warm != 0};
    cudaError_t e = dtype == TSENOR_BF16
                        ? dispatch_fused<BF16>(M, W, rows, cols, N, tau, iters, sweeps, mask_out, st, &ext)
                        : dispatch_fused<F32>(M, W, rows, cols, N, tau, iters, sweeps, mask_out, st, &ext);
    return e == cudaSuccess ? TSENOR_OK : cuda_fail(e, "tsenor_mask_warm launch");
}

extern "C" tsenor_status tsenor_plan_warm(const void* W, tsenor_dtype dtype, int64_t rows, int64_t cols, int N,
                                          int M, float tau, int iters, float tol, int warm, float* potentials,
                                          int32_t* iters_used, float* plan_out, tsenor_stream_t stream) {
    tsenor_status s = check_common(W, dtype, rows, cols, N, M);
    if (s != TSENOR_OK) return s;
    if (!solver_params_ok(tau, iters)) return TSENOR_ERR_ARG;
    if (!warm_params_ok(tol, warm, potentials, iters_used)) return TSENOR_ERR_ARG;
    if (rows == 0 || cols == 0) return TSENOR_OK;
    if (!plan_out || !aligned(plan_out, 16)) return TSENOR_ERR_ARG;
    const DykstraExt ext{potentials, iters_used, tol * kLog2e, warm != 0};
    cudaError_t e = run_plan(dtype, M, W, rows, cols, N, tau, iters, plan_out, (cudaStream_t)stream, &ext);
    return e == cudaSuccess ? TSENOR_OK : cuda_fail(e, "tsenor_plan_warm launch");
}

// ---------------------------------------------------------------------------
// The context current on the calling thread (driver entry point fetched once
// through the runtime): resources cached across calls are keyed by it, so a
// new primary context after cudaDeviceReset gets fresh ones.  *ctx is null
// while the runtime has not yet made a context current on this thread.
namespace {
constexpr int kMaxDevices = 64;
PFN_cuCtxGetCurrent g_ctx_current = nullptr;
std::once_flag g_ctx_once;

cudaError_t current_context(CUcontext* ctx) {
    std::call_once(g_ctx_once, [] {
        void* fn = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &fn, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            g_ctx_current = reinterpret_cast<PFN_cuCtxGetCurrent>(fn);
    });
    if (!g_ctx_current) return cudaErrorNotSupported;
    *ctx = nullptr;
    return g_ctx_current(ctx) == CUDA_SUCCESS ? cudaSuccess : cudaErrorDeviceUninitialized;
}
}  // namespace

// ---------------------------------------------------------------------------
// tsenor_mask_host: row chunks of a host matrix pipelined through two device
// slots.  Copies run on an internal stream X, solves alternate between the
// caller's stream and a second internal stream (so that one chunk's tail
// overlaps the next chunk's head).  X first uploads chunks 0 and 1; then per
// chunk k, slot s = k % 2:
//   compute stream: wait h2d[k]; tsenor_mask on dW[s] -> dmask[s]; event comp[k]
//   X: wait comp[k]; copy dmask[s] -> host mask chunk k; upload chunk k+2
//      into dW[s] (free: chunk k's solve is done); event h2d[k+2]
// so each upload overlaps the solve of the chunk before it.  The caller's
// stream then waits for X's last copy.
// The two internal streams and the events are created on a host thread's
// first call on a device (and context) and kept for its later calls:
// creating and destroying them took most of a call's host time, and the
// first upload waited for it (the 16:32 workload's call spent about 0.5 ms
// on the host before).  An event is recorded once per call, and every wait
// on it is enqueued in the same call, after that record, so reuse across
// calls is safe; calls of one thread share the streams and so run in order.
// They are never destroyed: they go with the context.
namespace {
constexpr int kHostMaxChunks = 64;
constexpr int kHostEvents = 2 * kHostMaxChunks + 2;

struct HostPipeRes {
    CUcontext ctx = nullptr;
    cudaStream_t x = nullptr, c2 = nullptr;
    cudaEvent_t ev[kHostEvents] = {};
};
thread_local HostPipeRes* tl_pipe[kMaxDevices];   // allocated on first use, never freed

// This thread's streams and events on the current device and context.
cudaError_t host_pipe_res(HostPipeRes** out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
    CUcontext ctx = nullptr;
    e = current_context(&ctx);
    if (e != cudaSuccess) return e;
    if (!tl_pipe[dev]) tl_pipe[dev] = new (std::nothrow) HostPipeRes();
    if (!tl_pipe[dev]) return cudaErrorMemoryAllocation;
    HostPipeRes& r = *tl_pipe[dev];
    if (!r.x || !ctx || r.ctx != ctx) {
        HostPipeRes fresh;                           // a stale context's handles are dropped, not destroyed
        e = cudaStreamCreateWithFlags(&fresh.x, cudaStreamNonBlocking);
        if (e == cudaSuccess) e = cudaStreamCreateWithFlags(&fresh.c2, cudaStreamNonBlocking);
        for (int i = 0; i < kHostEvents && e == cudaSuccess; ++i)
            e = cudaEventCreateWithFlags(&fresh.ev[i], cudaEventDisableTiming);
        if (e == cudaSuccess) e = current_context(&fresh.ctx);
        if (e == cudaSuccess && !fresh.ctx) e = cudaErrorDeviceUninitialized;
        if (e != cudaSuccess) {
            for (int i = 0; i < kHostEvents; ++i)
                if (fresh.ev[i]) cudaEventDestroy(fresh.ev[i]);
            if (fresh.x) cudaStreamDestroy(fresh.x);
            if (fresh.c2) cudaStreamDestroy(fresh.c2);
            return e;
        }
        r = fresh;
    }
    *out = &r;
    return cudaSuccess;
}

struct HostPipe {
    cudaStream_t x = nullptr, c2 = nullptr;
    cudaEvent_t* ev = nullptr;
    int nev = 0;
    void* dW[2] = {nullptr, nullptr};
    uint32_t* dm[2] = {nullptr, nullptr};
    cudaEvent_t event() { return nev < kHostEvents ? ev[nev++] : nullptr; }
    void release(cudaStream_t st) {
        for (int s = 0; s < 2; ++s) {
            if (dW[s]) cudaFreeAsync(dW[s], st);
            if (dm[s]) cudaFreeAsync(dm[s], st);
        }
    }
};
}  // namespace

extern "C" tsenor_status tsenor_mask_host(const void* W_host, tsenor_dtype dtype, int64_t rows, int64_t cols, int N,
                                          int M, float tau, int iters, int sweeps, uint32_t* mask_host,
                                          tsenor_stream_t stream) {
    if (M != 4 && M != 8 && M != 16 && M != 32 && M != 64) return TSENOR_ERR_UNSUPPORTED_M;
    if (dtype != TSENOR_F32 && dtype != TSENOR_BF16) return TSENOR_ERR_ARG;
    if (N < 1 || N > M || !solver_params_ok(tau, iters) || sweeps < 0) return TSENOR_ERR_ARG;
    if (rows < 0 || cols < 0 || rows % M || cols % M) return TSENOR_ERR_SHAPE;
    if (rows > (int64_t(1) << 31) || cols > (int64_t(1) << 31)) return TSENOR_ERR_SHAPE;
    if (rows == 0 || cols == 0) return TSENOR_OK;
    if (!W_host || !mask_host) return TSENOR_ERR_ARG;
    cudaStream_t st = (cudaStream_t)stream;
    const size_t es = dtype == TSENOR_BF16 ? 2 : 4;
    const int64_t wpr = (cols + 31) / 32;
    // one chunk per ~8 MB of W, between 1 and 8 chunks, each a multiple of M rows
    const int64_t bytes = rows * cols * int64_t(es);
    int64_t want = bytes / (int64_t(8) << 20);
    want = want < 1 ? 1 : (want > 8 ? 8 : want);
    int64_t chunk = ((rows + want - 1) / want + M - 1) / M * M;
    const int64_t nchunks = (rows + chunk - 1) / chunk;

    HostPipe p;
    HostPipeRes* res = nullptr;
    cudaError_t e = host_pipe_res(&res);
    if (e != cudaSuccess) return cuda_fail(e, "tsenor_mask_host streams");
    p.x = res->x;
    p.c2 = res->c2;
    p.ev = res->ev;
    for (int s = 0; s < 2 && e == cudaSuccess; ++s) {
        e = cudaMallocAsync(&p.dW[s], size_t(chunk) * size_t(cols) * es, st);
        if (e == cudaSuccess)
            e = cudaMallocAsync(reinterpret_cast<void**>(&p.dm[s]), size_t(chunk) * size_t(wpr) * 4, st);
    }
    cudaEvent_t start = e == cudaSuccess ? p.event() : nullptr;
    if (e == cudaSuccess && !start) e = cudaErrorMemoryAllocation;
    // everything below is ordered after the caller's earlier work and the allocations
    if (e == cudaSuccess) e = cudaEventRecord(start, st);
    if (e == cudaSuccess) e = cudaStreamWaitEvent(p.x, start, 0);
    if (e == cudaSuccess) e = cudaStreamWaitEvent(p.c2, start, 0);
    tsenor_status s = TSENOR_OK;
    cudaEvent_t h2d[kHostMaxChunks] = {};
    auto rows_of = [&](int64_t k) { return rows - k * chunk < chunk ? rows - k * chunk : chunk; };
    auto upload = [&](int64_t k) -> cudaError_t {        // on X: W chunk k into slot k % 2
        h2d[k] = p.event();
        if (!h2d[k]) return cudaErrorMemoryAllocation;
        cudaError_t r = cudaMemcpyAsync(p.dW[k % 2],
                                        static_cast<const char*>(W_host) + size_t(k * chunk) * size_t(cols) * es,
                                        size_t(rows_of(k)) * size_t(cols) * es, cudaMemcpyHostToDevice, p.x);
        return r == cudaSuccess ? cudaEventRecord(h2d[k], p.x) : r;
    };
    for (int64_t k = 0; k < 2 && k < nchunks && e == cudaSuccess; ++k) e = upload(k);
    for (int64_t k = 0; k < nchunks && e == cudaSuccess && s == TSENOR_OK; ++k) {
        const int slot = int(k % 2);
        const int64_t r0 = k * chunk, nr = rows_of(k);
        cudaStream_t cs = slot == 0 ? st : p.c2;
        cudaEvent_t comp = p.event();
        if (!comp) { e = cudaErrorMemoryAllocation; break; }
        e = cudaStreamWaitEvent(cs, h2d[k], 0);
        if (e != cudaSuccess) break;
        s = tsenor_mask(p.dW[slot], dtype, nr, cols, N, M, tau, iters, sweeps, p.dm[slot], (tsenor_stream_t)cs);
        if (s != TSENOR_OK) break;
        e = cudaEventRecord(comp, cs);
        if (e == cudaSuccess) e = cudaStreamWaitEvent(p.x, comp, 0);
        if (e == cudaSuccess)
            e = cudaMemcpyAsync(mask_host + size_t(r0) * size_t(wpr), p.dm[slot], size_t(nr) * size_t(wpr) * 4,
                                cudaMemcpyDeviceToHost, p.x);
        if (e == cudaSuccess && k + 2 < nchunks) e = upload(k + 2);
    }
    // the caller's stream waits for the last copy (and with it every chunk)
    cudaEvent_t done = p.event();
    cudaError_t e2 = done ? cudaEventRecord(done, p.x) : cudaErrorMemoryAllocation;
    if (e2 == cudaSuccess) e2 = cudaStreamWaitEvent(st, done, 0);
    p.release(st);
    if (s != TSENOR_OK) return s;
    if (e != cudaSuccess) return cuda_fail(e, "tsenor_mask_host");
    if (e2 != cudaSuccess) return cuda_fail(e2, "tsenor_mask_host join");
    return TSENOR_OK;
}

extern "C" tsenor_status tsenor_mask_safeguard(const void* W, tsenor_dtype dtype, int64_t rows, int64_t cols,
                                               int N, int M, float tau, int iters, int sweeps,
                                               const uint32_t* prev_mask, uint32_t* mask_out,
                                               unsigned long long* kept_out, tsenor_stream_t stream) {
    tsenor_status s = check_common(W, dtype, rows, cols, N, M);
    if (s != TSENOR_OK) return s;
    if (!solver_params_ok(tau, iters) || sweeps < 0) return TSENOR_ERR_ARG;
    if (rows == 0 || cols == 0) return TSENOR_OK;
    if (!prev_mask || !aligned(prev_mask, 8) || prev_mask == mask_out) return TSENOR_ERR_ARG;
    if (kept_out && !aligned(kept_out, 8)) return TSENOR_ERR_ARG;
    s = tsenor_mask(W, dtype, rows, cols, N, M, tau, iters, sweeps, mask_out, stream);
    if (s != TSENOR_OK) return s;
    cudaError_t e = launch_safeguard(dtype == TSENOR_BF16, W, rows, cols, prev_mask, mask_out, N, M, kept_out,
                                     (cudaStream_t)stream);
    return e == cudaSuccess ? TSENOR_OK : cuda_fail(e, "tsenor_mask_safeguard launch");
}

extern "C" tsenor_status tsenor_mask_padded(const void* W, tsenor_dtype dtype, int64_t rows, int64_t cols, int N,
                                            int M, float tau, int iters, int sweeps, uint32_t* mask_out,
                                            tsenor_stream_t stream) {
    if (M != 4 && M != 8 && M != 16 && M != 32 && M != 64) return TSENOR_ERR_UNSUPPORTED_M;
    if (dtype != TSENOR_F32 && dtype != TSENOR_BF16) return TSENOR_ERR_ARG;
    if (N < 1 || N > M || !solver_params_ok(tau, iters) || sweeps < 0) return TSENOR_ERR_ARG;
    if (rows < 0 || cols < 0 || rows > (int64_t(1) << 31) || cols > (int64_t(1) << 31)) return TSENOR_ERR_SHAPE;
    if (rows == 0 || cols == 0) return TSENOR_OK;
    if (!W || !mask_out || !aligned(mask_out, 4)) return TSENOR_ERR_ARG;
    if (rows % M == 0 && cols % M == 0 && aligned(W, 16) && aligned(mask_out, 8))
        return tsenor_mask(W, dtype, rows, cols, N, M, tau, iters, sweeps, mask_out, stream);
    cudaStream_t st = (cudaStream_t)stream;
    const size_t es = dtype == TSENOR_BF16 ? 2 : 4;
    const int64_t rp = (rows + M - 1) / M * M, cp = (cols + M - 1) / M * M;
    const int64_t wpr = (cols + 31) / 32, wprp = (cp + 31) / 32;
    void* Wp = nullptr;
    uint32_t* mp = nullptr;
    cudaError_t e = cudaMallocAsync(&Wp, size_t(rp) * size_t(cp) * es, st);
    if (e == cudaSuccess) e = cudaMallocAsync(reinterpret_cast<void**>(&mp), size_t(rp) * size_t(wprp) * 4, st);
    if (e == cudaSuccess) e = cudaMemsetAsync(Wp, 0, size_t(rp) * size_t(cp) * es, st);
    if (e == cudaSuccess)
        e = cudaMemcpy2DAsync(Wp, size_t(cp) * es, W, size_t(cols) * es, size_t(cols) * es, size_t(rows),
                              cudaMemcpyDeviceToDevice, st);
    tsenor_status s = TSENOR_OK;
    if (e == cudaSuccess) s = tsenor_mask(Wp, dtype, rp, cp, N, M, tau, iters, sweeps, mp, stream);
    if (e == cudaSuccess && s == TSENOR_OK) {
        const int64_t n = rows * wpr;
        crop_mask_kernel<<<unsigned((n + 255) / 256), 256, 0, st>>>(mp, wprp, mask_out, wpr, rows, cols);
        e = cudaGetLastError();
    }
    cudaError_t e2 = Wp ? cudaFreeAsync(Wp, st) : cudaSuccess;
    cudaError_t e3 = mp ? cudaFreeAsync(mp, st) : cudaSuccess;
    if (e != cudaSuccess) return cuda_fail(e, "tsenor_mask_padded");
    if (s != TSENOR_OK) return s;
    if (e2 != cudaSuccess) return cuda_fail(e2, "tsenor_mask_padded free");
    if (e3 != cudaSuccess) return cuda_fail(e3, "tsenor_mask_padded free");
    return TSENOR_OK;
}

extern "C" tsenor_status tsenor_objective(const void* W, tsenor_dtype dtype, int64_t rows, int64_t cols,
                                          const uint32_t* mask, int N, int M, double* out,
                                          tsenor_stream_t stream) {
    tsenor_status s = check_common(W, dtype, rows, cols, N, M);
    if (s != TSENOR_OK) return s;
    if (rows == 0 || cols == 0) return TSENOR_OK;
    if (!mask || !out || !aligned(mask, 4) || !aligned(out, 8)) return TSENOR_ERR_ARG;
    cudaError_t e = launch_objective(dtype == TSENOR_BF16, W, rows, cols, mask, N, M, out, (cudaStream_t)stream);
    return e == cudaSuccess ? TSENOR_OK : cuda_fail(e, "tsenor_objective launch");
}

extern "C" tsenor_status tsenor_error_count(tsenor_stream_t stream, int64_t* count_out) {
    if (!count_out) return TSENOR_ERR_ARG;
    cudaStream_t st = (cudaStream_t)stream;
    unsigned long long v = 0;
    const unsigned long long zero = 0;
    cudaError_t e = cudaMemcpyFromSymbolAsync(&v, g_block_failures, sizeof(v), 0, cudaMemcpyDeviceToHost, st);
    if (e == cudaSuccess) e = cudaMemcpyToSymbolAsync(g_block_failures, &zero, sizeof(zero), 0, cudaMemcpyHostToDevice, st);
    if (e == cudaSuccess) e = cudaStreamSynchronize(st);
    if (e != cudaSuccess) return cuda_fail(e, "tsenor_error_count");
    *count_out = int64_t(v);
    return v ? TSENOR_ERR_DEVICE : TSENOR_OK;
}

extern "C" const char* tsenor_status_string(int status) {
    switch (status) {
        case TSENOR_OK: return "ok";
        case TSENOR_ERR_ARG: return "invalid argument";
        case TSENOR_ERR_SHAPE: return "rows/cols not a non-negative multiple of M";
        case TSENOR_ERR_UNSUPPORTED_M: return "M must be 4, 8, 16, 32 or 64";
        case TSENOR_ERR_CUDA: return "CUDA runtime error";
        case TSENOR_ERR_DEVICE: return "blocks failed on the device (non-finite input or no repair move); see the count";
        case TSENOR_ERR_TOO_LARGE: return "rows*cols exceeds TSENOR_NOALLOC_MAX_PARAMS (16777216) of tsenor_mask_noalloc";
        default: return "unknown status";
    }
}

extern "C" const char* tsenor_last_error(void) { return tsenor::g_last_error; }

// ---------------------------------------------------------------------------
// tsenor_mask_noalloc: the plan + round kernels with the plan between them
// in a file-scope device array, so that the call allocates nothing (see
// include/tsenor.h).  Host code must not hand `g_noalloc_plan` itself to a
// kernel: on the host that name is only a stand-in for the symbol, not a
// device address.  The device address is looked up with
// cudaGetSymbolAddress once per device and context: the cache is keyed by
// the context that is current on the device, so a new primary context
// (after cudaDeviceReset) gets a fresh lookup.

static __device__ __align__(256) float g_noalloc_plan[TSENOR_NOALLOC_MAX_PARAMS];

namespace {
std::mutex g_noalloc_mutex;
float* g_noalloc_ptr[kMaxDevices] = {};
CUcontext g_noalloc_ctx[kMaxDevices] = {};

// Device address of g_noalloc_plan on the current device and context.
cudaError_t noalloc_plan_ptr(float** out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
    // no current context yet on this thread (the runtime makes the primary
    // context current lazily): the symbol lookup below does that first
    CUcontext ctx = nullptr;
    e = current_context(&ctx);
    if (e != cudaSuccess) return e;
    std::lock_guard<std::mutex> lock(g_noalloc_mutex);
    if (!g_noalloc_ptr[dev] || !ctx || g_noalloc_ctx[dev] != ctx) {
        void* p = nullptr;
        e = cudaGetSymbolAddress(&p, g_noalloc_plan);
        if (e != cudaSuccess) return e;
        e = current_context(&ctx);
        if (e != cudaSuccess) return e;
        if (!ctx) return cudaErrorDeviceUninitialized;
        g_noalloc_ptr[dev] = static_cast<float*>(p);
        g_noalloc_ctx[dev] = ctx;
    }
    *out = g_noalloc_ptr[dev];
    return cudaSuccess;
}
}  // namespace

extern "C" tsenor_status tsenor_mask_noalloc(const void* W, tsenor_dtype dtype, int64_t rows, int64_t cols, int N,
                                             int M, float tau, int iters, int sweeps, uint32_t* mask_out,
                                             tsenor_stream_t stream) {
    tsenor_status s = check_common(W, dtype, rows, cols, N, M);
    if (s != TSENOR_OK) return s;
    if (!solver_params_ok(tau, iters) || sweeps < 0) return TSENOR_ERR_ARG;
    if (rows == 0 || cols == 0) return TSENOR_OK;
    if (!mask_out || !aligned(mask_out, 8)) return TSENOR_ERR_ARG;
    if (rows * cols > TSENOR_NOALLOC_MAX_PARAMS) return TSENOR_ERR_TOO_LARGE;
    cudaStream_t st = (cudaStream_t)stream;
    float* plan = nullptr;
    cudaError_t e = noalloc_plan_ptr(&plan);
    if (e != cudaSuccess) return cuda_fail(e, "tsenor_mask_noalloc device array address");
    e = run_plan(dtype, M, W, rows, cols, N, tau, iters, plan, st);
    if (e == cudaSuccess) e = run_round(dtype, M, plan, W, rows, cols, N, sweeps, mask_out, st);
    if (e != cudaSuccess) return cuda_fail(e, "tsenor_mask_noalloc launch");
    return TSENOR_OK;
}
