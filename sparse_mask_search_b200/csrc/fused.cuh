// The whole hot path in one kernel (M = 16, 32, 64): Dykstra, sort keys from
// the final state, rounding, packed mask.  No plan ever reaches device
// memory.  The keys are bit-identical to what the plan kernel writes (same
// arithmetic), so the result equals rounding the exported plan.
//  - M = 32: one warp per block; keys straight from the registers.
//  - M = 16: one warp solves four blocks (8 threads each), writes their plans
//    to shared memory and rounds them one after another.
//  - M = 64: one CTA of 4 warps per block; the CTA sorts, warp 0 runs the
//    greedy and the repair, all 128 threads the local search.
// EXT instances add the warm start, the stop rule and the potentials export
// of dykstra_tile_solve.  M = 16, 32 and 64 stage the W tiles by TMA.
#pragma once

#include <type_traits>

#include "dykstra.cuh"
#include "round_group.cuh"
#include "round_warp.cuh"

namespace tsenor {

// bf16: registers capped at 96, five CTAs per SM (shared memory would admit
// six): 4.01 ms against 4.06 ms with the 80-register cap of six CTAs on the
// 4096x11008 16:32 workload (an earlier solver); at the cap of four CTAs (128
// registers, no spill) the current kernel takes 3.60 ms against 3.57.  The
// fp32 key needs more registers.
// W tiles are staged by TMA into the block's rounding space (free during the
// solve), with the mbarrier in its row-count array.  A/B on the same workload
// against 16-byte loads by the block's threads: 3.488 / 3.495 ms against
// 3.490 ms (2.750 against 2.766 ms without the local search); with both paths
// compiled into one kernel either one took about 3.56 ms.
template <typename T, bool EXT = false>
__global__ void __launch_bounds__(128, std::is_same<T, BF16>::value ? 5 : 4)
fused_kernel32(const __grid_constant__ CUtensorMap wmap, int64_t cols, int64_t n_blocks, int N, float tau, int iters,
               int sweeps, uint32_t* __restrict__ mask, int64_t wpr, DykstraExt ext = {}) {
    constexpr int M = 32;
    using C = TileCfg<M>;
    using Key = typename KeyOf<T>::type;
    static_assert(C::TPB == 32 && C::BPC == 4, "one warp per block");
    constexpr int TS = M + 1;                       // tile row stride (conflict-free column access)
    static_assert((C::BPC * M * TS * 4) % 128 == 0 && sizeof(RoundShared<M>) % 128 == 0, "TMA staging alignment");
    static_assert(sizeof(RoundShared<M>::G) >= M * M * sizeof(typename T::storage), "TMA staging size");
    extern __shared__ __align__(128) unsigned char fused32_raw[];
    const TileThread<M> th;
    float* tile = reinterpret_cast<float*>(fused32_raw) + th.blk * M * TS;
    RoundShared<M>* shs = reinterpret_cast<RoundShared<M>*>(reinterpret_cast<float*>(fused32_raw) + C::BPC * M * TS);
    const int64_t b = int64_t(blockIdx.x) * C::BPC + th.blk;
    const bool active = b < n_blocks;
    const int64_t nbc = cols / M;
    const int64_t r0 = active ? (b / nbc) * M : 0, c0 = active ? (b % nbc) * M : 0;

    float S[C::P][C::Q];                      // plan of this thread's entries
    const TileSource<T> src{&wmap, reinterpret_cast<typename T::storage*>(shs[th.blk].G),
                            reinterpret_cast<uint64_t*>(shs[th.blk].rc), nullptr, 0};
    const bool finite = dykstra_tile_solve<M, T, TS, EXT>(src, r0, c0, active, N, tau, iters, tile, nullptr, th, S,
                                                          ext, b);
    if (!active) return;                              // no CTA-wide barrier follows
    // the tile's copy has landed and every lane has waited for it: the barrier's
    // row-count slots are handed back to the rounding (a block whose copy did not
    // land is failed and never rounded)
    if (finite && th.lane == 0) mbar_inval(reinterpret_cast<uint64_t*>(shs[th.blk].rc));
    __syncwarp();

    Key key[C::P * C::Q];
#pragma unroll
    for (int k = 0; k < C::P; ++k)
#pragma unroll
        for (int c = 0; c < C::Q; ++c) {
            const int e = th.row(k) * M + th.col(c);
            key[k * C::Q + c] = Key::make(S[k][c], tile[th.row(k) * TS + th.col(c)], e);
        }
    bool ok = finite;                                 // one block per warp: uniform
    if (ok) ok = round_block_warp<M, Key>(key, tile, shs[th.blk].view(), N, sweeps, th.lane);
    if (!ok && th.lane == 0) atomicAdd(&g_block_failures, 1ull);
    __syncwarp();
    write_mask_rows<M>(mask, wpr, r0, c0, shs[th.blk].rowbits, ok, th.lane);
}

constexpr size_t fused32_smem() {
    return sizeof(float) * TileCfg<32>::BPC * 32 * 33 + sizeof(RoundShared<32>) * TileCfg<32>::BPC;
}

// M = 16: a warp holds 4 blocks of 8 threads each.
template <typename T, bool EXT = false>
__global__ void __launch_bounds__(128, 5)
fused_kernel16(const __grid_constant__ CUtensorMap wmap, int64_t cols, int64_t n_blocks, int N, float tau,
               int iters, int sweeps, uint32_t* __restrict__ mask, int64_t wpr, DykstraExt ext = {}) {
    constexpr int M = 16, TS = M + 1, E = M * M;
    using C = TileCfg<M>;
    using Key = typename KeyOf<T>::type;
    constexpr int BPW = C::BPW, R = WarpRound<M>::R;
    static_assert(C::TPB == 8 && BPW == 4 && C::BPC == 16, "four blocks per warp");
    static_assert((C::BPC * M * TS * 4) % 128 == 0 && (E * 4) % 128 == 0, "TMA staging alignment");
    extern __shared__ __align__(128) unsigned char fused16_raw[];
    float* atiles = reinterpret_cast<float*>(fused16_raw);   // [BPC][M * TS] |W|
    float* ptiles = atiles + C::BPC * M * TS;                 // [BPC][M * M]  plan (first: TMA staging of W)
    RoundShared<M>* shs = reinterpret_cast<RoundShared<M>*>(ptiles + C::BPC * E);   // one per warp
    int* flags = reinterpret_cast<int*>(shs + 4);             // [BPC] finite
    uint64_t* bars = reinterpret_cast<uint64_t*>(flags + C::BPC);
    const TileThread<M> th;
    float* tile = atiles + th.blk * M * TS;
    const int64_t b = int64_t(blockIdx.x) * C::BPC + th.blk;
    const bool active = b < n_blocks;
    const int64_t nbc = cols / M;
    const int64_t r0 = active ? (b / nbc) * M : 0, c0 = active ? (b % nbc) * M : 0;

    float S[C::P][C::Q];                      // plan of this thread's entries
    const TileSource<T> src{&wmap, reinterpret_cast<typename T::storage*>(ptiles + th.blk * E), bars + th.blk,
                            nullptr, 0};
    const bool finite = dykstra_tile_solve<M, T, TS, EXT>(src, r0, c0, active, N, tau, iters, tile, nullptr, th, S,
                                                          ext, b);
    float* ptile = ptiles + th.blk * E;
#pragma unroll
    for (int k = 0; k < C::P; ++k)
#pragma unroll
        for (int c = 0; c < C::Q; ++c) ptile[th.row(k) * M + th.col(c)] = S[k][c];
    if (th.t == 0) flags[th.blk] = finite;
    __syncwarp();

    const int lane = th.lane, warp = th.warp;
    for (int s = 0; s < BPW; ++s) {
        const int slot = warp * BPW + s;
        const int64_t bb = int64_t(blockIdx.x) * C::BPC + slot;
        if (bb >= n_blocks) break;                           // uniform over the warp
        const int64_t rr = (bb / nbc) * M, cc = (bb % nbc) * M;
        const float* at = atiles + slot * M * TS;
        const float* pt = ptiles + slot * E;
        Key key[R];
#pragma unroll
        for (int r = 0; r < R; ++r) {
            const int e = r * 32 + lane;
            key[r] = Key::make(pt[e], at[(e / M) * TS + (e % M)], e);
        }
        bool ok = flags[slot] != 0;
        if (ok) ok = round_block_warp<M, Key>(key, at, shs[warp].view(), N, sweeps, lane);
        if (!ok && lane == 0) atomicAdd(&g_block_failures, 1ull);
        __syncwarp();
        write_mask_rows<M>(mask, wpr, rr, cc, shs[warp].rowbits, ok, lane);
        __syncwarp();
    }
}

constexpr size_t fused16_smem() {
    return sizeof(float) * 16 * (16 * 17 + 16 * 16) + sizeof(RoundShared<16>) * 4 + sizeof(int) * 16 +
           sizeof(uint64_t) * 16;
}
static_assert((sizeof(float) * 16 * (16 * 17 + 16 * 16) + sizeof(RoundShared<16>) * 4 + sizeof(int) * 16) % 8 == 0,
              "barrier alignment");

// M = 4, 8: a CTA of 64 threads solves 64 blocks, one per thread (the whole
// block in registers, as dykstra_thread_kernel), stages the plans in shared
// memory, then groups of M lanes of each warp round that warp's 32 blocks
// (round_group.cuh), each group several in turn; |W| for the keys is read
// again (from L2).
template <int M>
struct FusedSmallCfg {
    static constexpr int THREADS = 64;                         // = blocks per CTA
    static constexpr int SS = M * M + 4;                       // plan row stride (floats; conflict-free stores)
    static constexpr int NG = THREADS / M;                     // groups per CTA
    static constexpr size_t plan_bytes = sizeof(float) * THREADS * SS;
    static constexpr size_t group_off = plan_bytes;
    static constexpr size_t flags_off = group_off + sizeof(RoundGroupSmem<M>) * NG;
    static constexpr size_t bytes = flags_off + sizeof(int) * THREADS;
};

template <int M, typename T, bool EXT = false>
__global__ void __maxnreg__(128)
fused_kernel_small(const typename T::storage* __restrict__ W, int64_t cols, int64_t n_blocks, int N, float tau,
                   int iters, int sweeps, uint32_t* __restrict__ mask, int64_t wpr, DykstraExt ext = {}) {
    using Cfg = FusedSmallCfg<M>;
    using Key = typename KeyOf<T>::type;
    constexpr int AS = M + 1;
    extern __shared__ __align__(16) unsigned char fused_small_raw[];
    float* plans = reinterpret_cast<float*>(fused_small_raw);
    RoundGroupSmem<M>* groups = reinterpret_cast<RoundGroupSmem<M>*>(fused_small_raw + Cfg::group_off);
    int* flags = reinterpret_cast<int*>(fused_small_raw + Cfg::flags_off);
    const int t = threadIdx.x;
    const int64_t nbc = cols / M;
    {
        const int64_t b = int64_t(blockIdx.x) * Cfg::THREADS + t;
        if (b < n_blocks) {
            const int64_t r0 = (b / nbc) * M, c0 = (b % nbc) * M;
            float S[M][M];                                    // plan of the block
            float* dst = plans + t * Cfg::SS;                 // y0 during the solve, then the plan
            const bool finite = dykstra_thread_solve<M, T, EXT>(W, cols, b, r0, c0, N, tau, iters, ext, S, dst);
#pragma unroll
            for (int i = 0; i < M; ++i)
#pragma unroll
                for (int v = 0; v < M / 4; ++v)
                    reinterpret_cast<float4*>(dst + i * M)[v] =
                        make_float4(S[i][4 * v], S[i][4 * v + 1], S[i][4 * v + 2], S[i][4 * v + 3]);
            flags[t] = finite;
        }
    }
    // each warp rounds the 32 blocks its own lanes solved: no CTA-wide barrier,
    // so warps drift apart and one warp's rounding overlaps another's solve
    __syncwarp();

    const int lane = t & 31, gl = lane % M, g = t / M;
    const unsigned gmask = ((1u << M) - 1u) << (lane - gl);
    RoundGroupSmem<M>& sm = groups[g];
    const RoundView<M> sh = sm.sh.view();
    const int wbase = t - lane;                               // first block slot of this warp
    for (int s = wbase + lane / M; s < wbase + 32; s += 32 / M) {
        const int64_t b = int64_t(blockIdx.x) * Cfg::THREADS + s;
        if (b >= n_blocks) break;                             // uniform per group
        const int64_t r0 = (b / nbc) * M, c0 = (b % nbc) * M;
        const float* src = plans + s * Cfg::SS;
        Key key[M];
#pragma unroll
        for (int r = 0; r < M; ++r) {
            const int e = r * M + gl;                         // row r, column gl
            const float a = T::load1(W + (r0 + r) * cols + c0 + gl);
            sm.a[r * AS + gl] = a;
            key[r] = Key::make(src[e], a, e);
        }
        __syncwarp(gmask);
        bool ok = flags[s] != 0;
        if (ok) ok = round_block_group<M, Key>(key, sm.a, sh, N, sweeps, lane, gl, gmask);
        if (!ok && gl == 0) atomicAdd(&g_block_failures, 1ull);
        __syncwarp(gmask);
        write_group_row<M>(mask, wpr, r0, c0, ok ? static_cast<unsigned>(sh.rowbits[gl]) : 0u, gl);
        __syncwarp(gmask);                                    // the group's arrays are reused by its next block
    }
}

// M = 64: one CTA of 4 warps per block; Round64Smem's colbuf serves the
// Dykstra phase's cross-warp column sums.
static_assert(Round64Smem<KeyB>::kColbufFloats >= 2 * 4 * 32 * TileCfg<64>::CO, "column-sum buffer");

template <typename T, bool EXT = false>
__global__ void __launch_bounds__(128, std::is_same<T, BF16>::value ? 4 : 1)
fused_kernel64(const __grid_constant__ CUtensorMap wmap, int64_t cols, int64_t n_blocks, int N, float tau,
               int iters, int sweeps, uint32_t* __restrict__ mask, int64_t wpr, DykstraExt ext = {}) {
    constexpr int M = 64, TS = M + 1;
    using C = TileCfg<M>;
    using Key = typename KeyOf<T>::type;
    static_assert(C::TPB == 128 && C::BPC == 1, "one block per CTA");
    static_assert(sizeof(Round64Smem<Key>::u) >= M * M * sizeof(typename T::storage), "TMA staging size");
    extern __shared__ __align__(128) unsigned char fused64_raw[];
    Round64Smem<Key>& sm = *reinterpret_cast<Round64Smem<Key>*>(fused64_raw);
    const TileThread<M> th;
    const int64_t b = blockIdx.x;
    if (b >= n_blocks) return;                         // uniform per CTA
    const int64_t nbc = cols / M;
    const int64_t r0 = (b / nbc) * M, c0 = (b % nbc) * M;

    float S[C::P][C::Q];                      // plan of this thread's entries
    // the raw W tile is staged in the sort exchange space
    const TileSource<T> src{&wmap, reinterpret_cast<typename T::storage*>(&sm.u), &sm.tma_bar, nullptr, 0};
    const bool finite = dykstra_tile_solve<M, T, TS, EXT>(src, r0, c0, true, N, tau, iters, sm.a, sm.v.colbuf, th, S,
                                                          ext, b);
    Key key[C::P * C::Q];
#pragma unroll
    for (int k = 0; k < C::P; ++k)
#pragma unroll
        for (int c = 0; c < C::Q; ++c) {
            const int row = th.row(k), col = th.col(c);
            key[k * C::Q + c] = Key::make(S[k][c], sm.a[row * TS + col], row * M + col);
        }
    bool ok = finite;                                   // uniform over the CTA
    if (ok) ok = round_block_cta64(key, sm, N, sweeps, th.tid);
    if (!ok && th.tid == 0) atomicAdd(&g_block_failures, 1ull);
    write_mask_rows<M>(mask, wpr, r0, c0, sm.v.rb.rowbits, ok, th.tid, 128);
}

}  // namespace tsenor
