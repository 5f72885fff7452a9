// Rounding for small blocks (M = 4, 8): a group of M lanes per block, one lane
// per block row, 32/M blocks per warp.  Same steps, order and fp32 decisions
// as the warp-per-block rounding of round_warp.cuh ("What carries the
// argument" and the Fig. 2 caption of the TSENOR review):
//   1. bitonic sort of the block's M*M keys, M per lane (in-lane
//      compare-exchanges below distance M, shuffles inside the group above);
//   2. greedy over M sorted entries at a time with the exact conflict
//      resolution of greedy_and_repair, on group-masked votes;
//   3. repair by group argmax over the 2-in/1-out candidates;
//   4. local search with the cached gain table, lane y serving row y.
// A warp-per-block rounding leaves most lanes idle at these sizes (M = 8:
// 64 entries, 8 rows); the groups keep every lane busy.
#pragma once

#include "round_warp.cuh"

namespace tsenor {

template <int M>
struct GroupRound {
    static_assert(M == 4 || M == 8, "group rounding serves M = 4 and 8");
    static constexpr int G = M;                  // lanes per block
    static constexpr int R = M;                  // keys per lane
    static constexpr int E = M * M;
    static constexpr int BPW = 32 / G;           // blocks per warp
    static constexpr int AS = M + 1;             // row stride of |W| and of the gain table
};

// Argmax over the group (larger value, then lower index).
template <int G>
__device__ __forceinline__ void group_argmax(float& v, int& i, unsigned gmask) {
#pragma unroll
    for (int s = G / 2; s >= 1; s >>= 1) {
        const float ov = __shfl_xor_sync(gmask, v, s);
        const int oi = __shfl_xor_sync(gmask, i, s);
        if (ov > v || (ov == v && oi < i)) { v = ov; i = oi; }
    }
}

// Bitonic sort of G*R keys, R per lane (position gl*R + r), earliest first.
template <int R, int G, typename Key>
__device__ __forceinline__ void group_bitonic_sort(Key (&key)[R], int gl, unsigned gmask) {
    constexpr int EP = G * R;
    bitonic_local<R, 2>(key, gl);
#pragma unroll
    for (int k = 2 * R; k <= EP; k <<= 1) {
        const bool up = ((gl * R) & k) == 0;
#pragma unroll
        for (int j = k >> 1; j >= R; j >>= 1) {
            const int m = j / R;
            const bool take_earlier = ((gl & m) == 0) == up;
#pragma unroll
            for (int r = 0; r < R; ++r) {
                const Key x = key[r];
                Key y;
                y.k = __shfl_xor_sync(gmask, x.k, m);
                if constexpr (sizeof(Key) > 8) y.idx = __shfl_xor_sync(gmask, x.idx, m);
                key[r] = (y.before(x) == take_earlier) ? y : x;
            }
        }
        bitonic_regs_down<R, R / 2>(key, up);
    }
}

// Greedy and repair for one block by its group (see greedy_and_repair).
template <int M>
__device__ bool group_greedy_and_repair(const float* a, const RoundView<M>& sh, int N, int lane, int gl,
                                        unsigned gmask) {
    using Bits = typename WarpRound<M>::Bits;
    constexpr int E = M * M, G = M, AS = M + 1;
    sh.rc[gl] = 0;
    sh.cc[gl] = 0;
    sh.rowbits[gl] = 0;
    __syncwarp(gmask);
    const int target = N * M;
    const int gbase = lane - gl;
    const unsigned lt = ((1u << lane) - 1u) & gmask;
    int taken = 0;
    for (int base = 0; base < E && taken < target; base += G) {
        const int e = sh.order[base + gl];
        const int i = e / M, j = e % M;
        const unsigned mr = __match_any_sync(gmask, i);
        const unsigned mc = __match_any_sync(gmask, j);
        const int r0c = sh.rc[i], c0c = sh.cc[j];
        unsigned acc = 0u;
        unsigned und = __ballot_sync(gmask, r0c < N && c0c < N);
        {   // first pass: nothing accepted yet, so the lower bound rejects no lane
            const bool mine = (und >> lane) & 1u;
            const int ru = r0c + __popc(mr & lt & und), cu = c0c + __popc(mc & lt & und);
            acc = __ballot_sync(gmask, mine && ru < N && cu < N);
            und &= ~acc;
        }
        while (und) {
            const bool mine = (und >> lane) & 1u;
            const unsigned maybe = acc | und;
            const int ru = r0c + __popc(mr & lt & maybe), cu = c0c + __popc(mc & lt & maybe);
            const int rl = r0c + __popc(mr & lt & acc), cl = c0c + __popc(mc & lt & acc);
            const unsigned A = __ballot_sync(gmask, mine && ru < N && cu < N);
            const unsigned Rj = __ballot_sync(gmask, mine && (rl >= N || cl >= N));
            acc |= A;
            und &= ~(A | Rj);
        }
        if ((acc >> lane) & 1u) atomicOr(&sh.rowbits[i], Bits(1) << j);
        const unsigned ga = mr & acc, gc = mc & acc;
        if (ga && __ffs(ga) - 1 == lane) sh.rc[i] = r0c + __popc(ga);   // the counts read at the chunk's start
        if (gc && __ffs(gc) - 1 == lane) sh.cc[j] = c0c + __popc(gc);
        taken += __popc(acc);
        __syncwarp(gmask);
    }

    for (int guard = 0; guard <= target; ++guard) {
        const unsigned shortR = (__ballot_sync(gmask, sh.rc[gl] < N) & gmask) >> gbase;
        const unsigned shortC = (__ballot_sync(gmask, sh.cc[gl] < N) & gmask) >> gbase;
        if (!shortR) return true;
        if (!shortC || guard == target) return false;
        const int i = __ffs(shortR) - 1, j = __ffs(shortC) - 1;
        const Bits Oi = sh.rowbits[i];
        float best = -INFINITY;
        int bflat = INT_MAX;
        {
            const int ip = gl;
            const Bits Op = sh.rowbits[ip];
            if (!((Op >> j) & 1)) {
                Bits cand = Op & ~Oi;
                while (cand) {
                    const int jp = lowest_bit(cand);
                    cand &= cand - 1;
                    const float sigma = __fsub_rn(__fadd_rn(a[i * AS + jp], a[ip * AS + j]), a[ip * AS + jp]);
                    const int flat = ip * M + jp;
                    if (sigma > best || (sigma == best && flat < bflat)) { best = sigma; bflat = flat; }
                }
            }
        }
        group_argmax<G>(best, bflat, gmask);
        if (bflat == INT_MAX) return false;
        if (gl == 0) {
            const int ip = bflat / M, jp = bflat % M;
            sh.rowbits[i] |= Bits(1) << jp;
            sh.rowbits[ip] = (sh.rowbits[ip] | (Bits(1) << j)) & ~(Bits(1) << jp);
            sh.rc[i] += 1;
            sh.cc[j] += 1;
        }
        __syncwarp(gmask);
    }
    return false;
}

// Local search for one block by its group, lane gl serving row gl (see local_search).
template <int M>
__device__ void group_local_search(const float* a, const RoundView<M>& sh, int sweeps, int gl, unsigned gmask) {
    using Bits = typename WarpRound<M>::Bits;
    constexpr int AS = M + 1, GS = M + 1, G = M;
    const int y = gl;
    float ay[M];
#pragma unroll
    for (int jj = 0; jj < M; ++jj) ay[jj] = a[y * AS + jj];
    {
        const Bits Oy = sh.rowbits[y];
        sh.G[y * GS + y] = -INFINITY;                      // no partner of itself (rescan_row)
#pragma unroll 1
        for (int d = 1; d <= M / 2; ++d) {
            const int x = (y + d) & (M - 1);
            float txy = -INFINITY, tyx = -INFINITY;
            pair_pieces<M, M, Bits>(ay, a + x * AS, sh.rowbits[x], Oy, 0, txy, tyx);
            if (!(d == M / 2 && y >= M / 2)) {
                const float g = __fadd_rn(txy, tyx);
                sh.G[x * GS + y] = g;
                sh.G[y * GS + x] = g;
            }
        }
    }
    __syncwarp(gmask);
    rescan_row<M>(sh, y);
    __syncwarp(gmask);

    int quiet = 0;
    for (int sw = 0; sw < sweeps && quiet < M; ++sw) {
        for (int i = 0; i < M && quiet < M; ++i) {
            {   // skip anchors with no positive best gain (fixed between swaps)
                const unsigned P = (__ballot_sync(gmask, sh.bestv[gl] > 0.f) & gmask) >> (__ffs(gmask) - 1);
                const unsigned ahead = P & (~0u << i);
                if (!ahead) { quiet += M - i; break; }
                const int nxt = __ffs(ahead) - 1;
                quiet += nxt - i;
                i = nxt;
                if (quiet >= M) break;
            }
            const float best = sh.bestv[i];
            const int bp = sh.bestp[i];
            if (!(best > 0.f)) { ++quiet; continue; }
            const Bits Oi = sh.rowbits[i], Ob = sh.rowbits[bp];
            float v1 = -INFINITY, v2 = -INFINITY;
            int j1 = INT_MAX, j2 = INT_MAX;
            {
                const int jj = gl;
                const bool in_i = (Oi >> jj) & 1, in_p = (Ob >> jj) & 1;
                if (in_i && !in_p) { v1 = __fsub_rn(a[bp * AS + jj], a[i * AS + jj]); j1 = jj; }
                if (!in_i && in_p) { v2 = __fsub_rn(a[i * AS + jj], a[bp * AS + jj]); j2 = jj; }
            }
            group_argmax<G>(v1, j1, gmask);
            group_argmax<G>(v2, j2, gmask);
            if (j1 >= M || j2 >= M) { ++quiet; continue; }   // unreachable: a positive gain needs both sets
            quiet = 0;
            const Bits Oi2 = (Oi & ~(Bits(1) << j1)) | (Bits(1) << j2);
            const Bits Ob2 = (Ob & ~(Bits(1) << j2)) | (Bits(1) << j1);
            const Bits Oy = (y == i) ? Oi2 : (y == bp) ? Ob2 : sh.rowbits[y];
            __syncwarp(gmask);                            // everyone has read the old rows
            if (gl == 0) {
                sh.rowbits[i] = Oi2;
                sh.rowbits[bp] = Ob2;
            }
            float t1i = -INFINITY, t2i = -INFINITY, t1b = -INFINITY, t2b = -INFINITY;
            pair_pieces<M, M, Bits>(ay, a + i * AS, Oi2, Oy, 0, t1i, t2i);
            pair_pieces<M, M, Bits>(ay, a + bp * AS, Ob2, Oy, 0, t1b, t2b);
            const float gi = __fadd_rn(t1i, t2i), gb = __fadd_rn(t1b, t2b);
            if (y != i) { sh.G[i * GS + y] = gi; sh.G[y * GS + i] = gi; }
            if (y != i && y != bp) { sh.G[bp * GS + y] = gb; sh.G[y * GS + bp] = gb; }
            __syncwarp(gmask);                            // gain table and rows complete
            const int op = sh.bestp[y];
            if (y == i || y == bp || op == i || op == bp) {
                rescan_row<M>(sh, y);
            } else {
                float bv = sh.bestv[y];
                int b2 = op;
                const int c1 = i < bp ? i : bp, c2 = i < bp ? bp : i;
                const float g1 = c1 == i ? gi : gb, g2 = c2 == i ? gi : gb;
                if (g1 > bv || (g1 == bv && c1 < b2)) { bv = g1; b2 = c1; }
                if (g2 > bv || (g2 == bv && c2 < b2)) { bv = g2; b2 = c2; }
                sh.bestv[y] = bv;
                sh.bestp[y] = b2;
            }
            __syncwarp(gmask);                            // row bests complete
        }
    }
}

// Steps 1-4 for one block by its group: `key` holds lane gl's keys (entry
// r*M + gl in register r), `a` the block's |W| (row stride M+1, shared
// memory).  Returns false when the block could not be made feasible; the
// row bitmasks are in sh.rowbits.
template <int M, typename Key>
__device__ __forceinline__ bool round_block_group(Key (&key)[M], const float* a, const RoundView<M>& sh, int N,
                                                  int sweeps, int lane, int gl, unsigned gmask) {
    group_bitonic_sort<M, M>(key, gl, gmask);
#pragma unroll
    for (int r = 0; r < M; ++r) sh.order[gl * M + r] = static_cast<uint16_t>(key[r].index());
    __syncwarp(gmask);
    if (!group_greedy_and_repair<M>(a, sh, N, lane, gl, gmask)) return false;
    if (sweeps > 0) {
        __syncwarp(gmask);
        group_local_search<M>(a, sh, sweeps, gl, gmask);
    }
    return true;
}

// Row gl of a block's mask: a byte (M = 8) or a nibble OR-ed into a zeroed
// mask (M = 4).
template <int M>
__device__ __forceinline__ void write_group_row(uint32_t* mask, int64_t wpr, int64_t r0, int64_t c0, unsigned bits,
                                                int gl) {
    uint32_t* row = mask + (r0 + gl) * wpr;
    if constexpr (M == 8) {
        reinterpret_cast<uint8_t*>(row)[c0 / 8] = static_cast<uint8_t>(bits);
    } else {
        if (bits) atomicOr(&row[c0 / 32], bits << (c0 % 32));
    }
}

// Rounding of a given plan, M lanes per block (M = 4, 8).  Entry e = r*M + gl
// of the block goes to lane gl's register r: register r holds block row r,
// so a group reads whole block rows and the groups of a warp read
// neighbouring blocks.
template <int M>
struct RoundGroupSmem {
    float a[M * (M + 1)];           // |W|, row stride M+1
    RoundShared<M> sh;
};

template <int M, typename T>
__global__ void __launch_bounds__(128)
round_group_kernel(const float* __restrict__ plan, const typename T::storage* __restrict__ W, int64_t cols,
                   int64_t n_blocks, int N, int sweeps, uint32_t* __restrict__ mask, int64_t wpr) {
    using Key = typename KeyOf<T>::type;
    using Cfg = GroupRound<M>;
    constexpr int G = Cfg::G, R = Cfg::R, BPC = 4 * Cfg::BPW, AS = M + 1;
    extern __shared__ __align__(16) unsigned char round_group_raw[];
    const int lane = threadIdx.x & 31, gl = lane % G, slot = threadIdx.x / G;
    const unsigned gmask = ((1u << G) - 1u) << (lane - gl);
    RoundGroupSmem<M>& sm = reinterpret_cast<RoundGroupSmem<M>*>(round_group_raw)[slot];
    const int64_t b = int64_t(blockIdx.x) * BPC + slot;
    if (b >= n_blocks) return;                       // uniform per group; groups never wait on each other
    const int64_t nbc = cols / M;
    const int64_t r0 = (b / nbc) * M, c0 = (b % nbc) * M;

    Key key[R];
    bool ok = true;
#pragma unroll
    for (int r = 0; r < R; ++r) {
        const int e = r * M + gl;                    // row r, column gl
        const float s = fabsf(plan[(r0 + r) * cols + c0 + gl]);
        const float a = T::load1(W + (r0 + r) * cols + c0 + gl);
        ok = ok && (s <= 3.402823466e38f) && (a <= 3.402823466e38f);
        sm.a[r * AS + gl] = a;
        key[r] = Key::make(s, a, e);
    }
    ok = __all_sync(gmask, ok);
    __syncwarp(gmask);
    const RoundView<M> sh = sm.sh.view();
    if (ok) ok = round_block_group<M, Key>(key, sm.a, sh, N, sweeps, lane, gl, gmask);
    if (!ok && gl == 0) atomicAdd(&g_block_failures, 1ull);
    __syncwarp(gmask);
    write_group_row<M>(mask, wpr, r0, c0, ok ? static_cast<unsigned>(sh.rowbits[gl]) : 0u, gl);
}

template <int M>
constexpr size_t round_group_smem() { return sizeof(RoundGroupSmem<M>) * 4 * GroupRound<M>::BPW; }

}  // namespace tsenor
