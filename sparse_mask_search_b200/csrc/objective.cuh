// Kept mass and validity of a mask, one warp per block (the block objective of
// the TSENOR review's "Core claim": sum of |W| over the kept entries).
#pragma once

#include "common.cuh"

namespace tsenor {

template <int M, typename T>
__global__ void __launch_bounds__(128)
objective_kernel(const typename T::storage* __restrict__ W, int64_t cols, int64_t n_blocks,
                 const uint32_t* __restrict__ mask, int64_t wpr, int N, double* __restrict__ out) {
    const int lane = threadIdx.x & 31;
    const int64_t b = int64_t(blockIdx.x) * 4 + (threadIdx.x >> 5);
    if (b >= n_blocks) return;
    const int64_t nbc = cols / M;
    const int64_t r0 = (b / nbc) * M, c0 = (b % nbc) * M;
    double acc = 0.0;
    bool valid = true;
    int colcnt[(M + 31) / 32] = {};
    for (int i = 0; i < M; ++i) {
        const uint32_t* row = mask + (r0 + i) * wpr;
        int rowcnt = 0;
        for (int jb = 0; jb < M; jb += 32) {
            const int j = jb + lane;
            const int64_t col = c0 + j;
            const bool in = j < M && ((row[col / 32] >> (col % 32)) & 1u);
            if (in) acc += double(T::load1(W + (r0 + i) * cols + col));
            if (in) colcnt[jb / 32] += 1;
            rowcnt += __popc(__ballot_sync(kFullMask, in));
        }
        valid = valid && rowcnt == N;
    }
    for (int jb = 0; jb < M; jb += 32)
        if (jb + lane < M) valid = valid && colcnt[jb / 32] == N;
    valid = __all_sync(kFullMask, valid);
#pragma unroll
    for (int s = 16; s >= 1; s >>= 1) acc += __shfl_xor_sync(kFullMask, acc, s);
    if (lane == 0) out[b] = valid ? acc : __longlong_as_double(0x7ff8000000000000ll);
}

// Monotonicity safeguard: one thread per block; both kept sums in fp64,
// row-major within the block (the order the CPU reference sums in), so the
// keep / replace decision is reproducible bit for bit.
template <int M, typename T>
__global__ void __launch_bounds__(128)
safeguard_kernel(const typename T::storage* __restrict__ W, int64_t cols, int64_t n_blocks,
                 const uint32_t* __restrict__ prev, uint32_t* __restrict__ mask, int64_t wpr, int N,
                 unsigned long long* kept) {
    const int64_t b = int64_t(blockIdx.x) * blockDim.x + threadIdx.x;
    if (b >= n_blocks) return;
    const int64_t nbc = cols / M;
    const int64_t r0 = (b / nbc) * M, c0 = (b % nbc) * M;
    double op = 0.0, on = 0.0;
    bool valid = true;
    int cc[M];
#pragma unroll
    for (int j = 0; j < M; ++j) cc[j] = 0;
    for (int i = 0; i < M; ++i) {
        int rcnt = 0;
        for (int j = 0; j < M; ++j) {
            const int64_t col = c0 + j, w = (r0 + i) * wpr + col / 32;
            const int sh = int(col % 32);
            const bool bp = (prev[w] >> sh) & 1u, bn = (mask[w] >> sh) & 1u;
            if (bp || bn) {
                const double a = double(T::load1(W + (r0 + i) * cols + col));
                if (bp) { op += a; ++rcnt; ++cc[j]; }
                if (bn) on += a;
            }
        }
        valid = valid && rcnt == N;
    }
#pragma unroll
    for (int j = 0; j < M; ++j) valid = valid && cc[j] == N;
    if (!(valid && op > on)) return;
    if (kept) atomicAdd(kept, 1ull);
    for (int i = 0; i < M; ++i) {
        for (int j0 = 0; j0 < M; j0 += 32) {
            const int64_t col = c0 + j0, w = (r0 + i) * wpr + col / 32;
            const int sh = int(col % 32);
            const int width = M - j0 < 32 ? M - j0 : 32;
            const uint32_t bm = (width == 32 ? 0xffffffffu : ((1u << width) - 1u)) << sh;
            if (bm == 0xffffffffu) {
                mask[w] = prev[w];
            } else {                                     // other blocks own the other bits of the word
                atomicAnd(&mask[w], ~bm);
                atomicOr(&mask[w], prev[w] & bm);
            }
        }
    }
}

template <int M>
cudaError_t launch_safeguard_m(bool bf16, const void* W, int64_t rows, int64_t cols, const uint32_t* prev,
                               uint32_t* mask, int N, unsigned long long* kept, cudaStream_t st) {
    const int64_t nb = (rows / M) * (cols / M);
    const int64_t wpr = (cols + 31) / 32;
    const unsigned grid = unsigned((nb + 127) / 128);
    if (bf16)
        safeguard_kernel<M, BF16><<<grid, 128, 0, st>>>(static_cast<const uint16_t*>(W), cols, nb, prev, mask, wpr,
                                                        N, kept);
    else
        safeguard_kernel<M, F32><<<grid, 128, 0, st>>>(static_cast<const float*>(W), cols, nb, prev, mask, wpr, N,
                                                       kept);
    return cudaGetLastError();
}

inline cudaError_t launch_safeguard(bool bf16, const void* W, int64_t rows, int64_t cols, const uint32_t* prev,
                                    uint32_t* mask, int N, int M, unsigned long long* kept, cudaStream_t st) {
    switch (M) {
        case 4: return launch_safeguard_m<4>(bf16, W, rows, cols, prev, mask, N, kept, st);
        case 8: return launch_safeguard_m<8>(bf16, W, rows, cols, prev, mask, N, kept, st);
        case 16: return launch_safeguard_m<16>(bf16, W, rows, cols, prev, mask, N, kept, st);
        case 32: return launch_safeguard_m<32>(bf16, W, rows, cols, prev, mask, N, kept, st);
        default: return launch_safeguard_m<64>(bf16, W, rows, cols, prev, mask, N, kept, st);
    }
}

// Rows of a mask of padded width into a narrower one; bits at or past `cols` cleared.
__global__ void crop_mask_kernel(const uint32_t* __restrict__ src, int64_t src_wpr, uint32_t* __restrict__ dst,
                                 int64_t dst_wpr, int64_t rows, int64_t cols) {
    const int64_t k = int64_t(blockIdx.x) * blockDim.x + threadIdx.x;
    if (k >= rows * dst_wpr) return;
    const int64_t r = k / dst_wpr, w = k % dst_wpr;
    uint32_t v = src[r * src_wpr + w];
    const int64_t valid = cols - w * 32;
    if (valid < 32) v &= (1u << valid) - 1u;
    dst[k] = v;
}

template <int M>
cudaError_t launch_objective_m(bool bf16, const void* W, int64_t rows, int64_t cols, const uint32_t* mask,
                               int N, double* out, cudaStream_t st) {
    const int64_t nb = (rows / M) * (cols / M);
    const int64_t wpr = (cols + 31) / 32;
    const unsigned grid = unsigned((nb + 3) / 4);
    if (bf16)
        objective_kernel<M, BF16><<<grid, 128, 0, st>>>(static_cast<const uint16_t*>(W), cols, nb, mask, wpr, N, out);
    else
        objective_kernel<M, F32><<<grid, 128, 0, st>>>(static_cast<const float*>(W), cols, nb, mask, wpr, N, out);
    return cudaGetLastError();
}

inline cudaError_t launch_objective(bool bf16, const void* W, int64_t rows, int64_t cols, const uint32_t* mask,
                                    int N, int M, double* out, cudaStream_t st) {
    switch (M) {
        case 4: return launch_objective_m<4>(bf16, W, rows, cols, mask, N, out, st);
        case 8: return launch_objective_m<8>(bf16, W, rows, cols, mask, N, out, st);
        case 16: return launch_objective_m<16>(bf16, W, rows, cols, mask, N, out, st);
        case 32: return launch_objective_m<32>(bf16, W, rows, cols, mask, N, out, st);
        default: return launch_objective_m<64>(bf16, W, rows, cols, mask, N, out, st);
    }
}

}  // namespace tsenor
