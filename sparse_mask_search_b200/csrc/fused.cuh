// The whole hot path for one block in one warp (M = 32): Dykstra plan kept in
// registers, sort keys formed from it directly, rounding, packed mask.  No
// plan ever reaches device memory.  The keys are bit-identical to what the
// plan kernel writes (same arithmetic), so the result equals rounding the
// exported plan.
#pragma once

#include "dykstra.cuh"
#include "round_warp.cuh"

namespace tsenor {

template <typename T>
__global__ void __launch_bounds__(128)
fused_kernel32(const typename T::storage* __restrict__ W, int64_t cols, int64_t n_blocks, int N, float tau,
               int iters, int sweeps, uint32_t* __restrict__ mask, int64_t wpr) {
    constexpr int M = 32;
    using C = TileCfg<M>;
    using Key = typename KeyOf<T>::type;
    static_assert(C::TPB == 32 && C::BPC == 4, "one warp per block");
    constexpr int TS = M + 1;                       // tile row stride (conflict-free column access)
    extern __shared__ float fused_smem[];
    const TileThread<M> th;
    float* tile = fused_smem + th.blk * M * TS;
    RoundShared<M>* shs = reinterpret_cast<RoundShared<M>*>(fused_smem + C::BPC * M * TS);
    const int64_t b = int64_t(blockIdx.x) * C::BPC + th.blk;
    const bool active = b < n_blocks;
    const int64_t nbc = cols / M;
    const int64_t r0 = active ? (b / nbc) * M : 0, c0 = active ? (b % nbc) * M : 0;

    float y[C::P][C::Q];
    const bool finite = dykstra_tile_solve<M, T, TS>(W, cols, r0, c0, active, N, tau, iters, tile, nullptr, th, y);
    if (!active) return;                              // no CTA-wide barrier follows

    Key key[C::P * C::Q];
#pragma unroll
    for (int k = 0; k < C::P; ++k)
#pragma unroll
        for (int c = 0; c < C::Q; ++c) {
            const int e = th.row(k) * M + th.col(c);
            key[k * C::Q + c] = Key::make(plan_value(y[k][c]), tile[th.row(k) * TS + th.col(c)], e);
        }
    bool ok = finite;                                 // one block per warp: uniform
    if (ok) ok = round_block_warp<M, Key>(key, tile, shs[th.blk], N, sweeps, th.lane);
    if (!ok && th.lane == 0) atomicAdd(&g_block_failures, 1ull);
    __syncwarp();
    write_mask_rows<M>(mask, wpr, r0, c0, shs[th.blk].rowbits, ok, th.lane);
}

constexpr size_t fused32_smem() {
    return sizeof(float) * TileCfg<32>::BPC * 32 * 33 + sizeof(RoundShared<32>) * TileCfg<32>::BPC;
}

}  // namespace tsenor
