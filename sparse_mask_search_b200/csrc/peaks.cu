// Throughput probes for the roofline denominators of the mask solver: the
// FP32 FMA pipe and the MUFU (special-function) pipe, the two pipes the
// Dykstra iterations load.  Each kernel runs independent dependency chains so
// that the pipe, not latency, limits it; the caller times a launch with CUDA
// events and divides the operation count by the time.  Not part of the
// solver: only the benchmark uses this library.
#include <cuda_runtime.h>

namespace {

constexpr int kChains = 8;

// kChains fma chains per thread: x <- x * a + b, with |a| < 1 so that the
// values stay bounded; one FP32 operation per fma.
__global__ void __launch_bounds__(256) peak_fma_kernel(int iters, float a, float b, float* out) {
    float x[kChains];
#pragma unroll
    for (int c = 0; c < kChains; ++c) x[c] = float(threadIdx.x + c);
#pragma unroll 1
    for (int i = 0; i < iters; ++i) {
#pragma unroll
        for (int u = 0; u < 16; ++u)
#pragma unroll
            for (int c = 0; c < kChains; ++c) x[c] = fmaf(x[c], a, b);
    }
    float s = 0.f;
#pragma unroll
    for (int c = 0; c < kChains; ++c) s += x[c];
    if (s == 1234.5f) out[blockIdx.x] = s;          // keeps the chains live; practically never stored
}

// kChains chains of the hardware base-2 exponential: x <- 2^-x stays in
// [0.5, 1] for x in [0, 1]; one MUFU operation per step (the negation is an
// operand modifier).
__global__ void __launch_bounds__(256) peak_mufu_kernel(int iters, float* out) {
    float x[kChains];
#pragma unroll
    for (int c = 0; c < kChains; ++c) x[c] = 0.001f * float((threadIdx.x + c) & 511);
#pragma unroll 1
    for (int i = 0; i < iters; ++i) {
#pragma unroll
        for (int u = 0; u < 16; ++u)
#pragma unroll
            for (int c = 0; c < kChains; ++c) asm volatile("ex2.approx.ftz.f32 %0, %1;" : "=f"(x[c]) : "f"(-x[c]));
    }
    float s = 0.f;
#pragma unroll
    for (int c = 0; c < kChains; ++c) s += x[c];
    if (s == 1234.5f) out[blockIdx.x] = s;
}

}  // namespace

// Operations one launch performs: blocks * threads * iters * 16 * kChains.
extern "C" long long tsenor_peak_ops(int blocks, int threads, int iters) {
    return static_cast<long long>(blocks) * threads * iters * 16 * kChains;
}

// kind 0: FP32 fma, kind 1: MUFU ex2.  threads <= 256.  out: `blocks` floats
// of device memory (never written in practice).  Returns a cudaError_t value.
extern "C" int tsenor_peak_launch(int kind, int blocks, int threads, int iters, float* out, cudaStream_t stream) {
    if (blocks < 1 || threads < 1 || threads > 256 || iters < 1 || !out) return int(cudaErrorInvalidValue);
    if (kind == 0) peak_fma_kernel<<<blocks, threads, 0, stream>>>(iters, 0.999f, 0.001f, out);
    else peak_mufu_kernel<<<blocks, threads, 0, stream>>>(iters, out);
    return int(cudaGetLastError());
}
