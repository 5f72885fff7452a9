// Rounding of the fractional plan into a transposable N:M mask, one warp per
// block ("What carries the argument" and the Fig. 2 caption of the TSENOR
// review; referee comment 3 on the rounding stage).
//
// Order of work per block:
//   1. keys (plan, |W|, flat index) into shared memory; bitonic sort so that
//      position 0 holds the entry taken first (plan desc, |W| desc, index asc);
//   2. greedy: entries in sorted order are taken while their row and column
//      budgets N remain.  The warp decides 32 consecutive entries at a time;
//      a lane is settled as soon as an upper bound (all undecided earlier
//      lanes of its row/column taken) keeps it within budget, or a lower bound
//      (only accepted earlier lanes) exhausts it.  The first undecided lane is
//      always settled, so the result is exactly the sequential greedy;
//   3. repair: while a row is short, the lowest short row i and lowest short
//      column j get the 2-in/1-out move (i,j'),(i',j) in, (i',j') out with the
//      best score (a_ij' + a_i'j) - a_i'j' of any sign (ties: lowest i'*M+j');
//   4. local search: anchors i = 0..M-1 per sweep; the partner i' with the
//      best net gain max_{j in O_i\O_i'}(a_i'j - a_ij) + max_{j' in O_i'\O_i}
//      (a_ij' - a_i'j') is swapped when that gain is positive.  The gain of a
//      row pair depends on those two rows only and is symmetric, so it is
//      cached in an M x M table and only the two rows touched by a swap are
//      recomputed; once M anchors in a row found nothing the state is a fixed
//      point and the remaining sweeps are skipped (they would change nothing);
//   5. row bitmasks to the packed mask.
// All comparisons that decide an integer use fp32 values evaluated in the
// order written above.
#pragma once

#include <climits>

#include "common.cuh"

namespace tsenor {

__device__ unsigned long long g_block_failures;   // blocks that could not be rounded

template <int M>
struct RoundCfg {
    static constexpr int E = M * M;
    static constexpr int WARPS = (M == 64) ? 1 : 4;      // warps (= blocks) per CTA
    using Bits = typename std::conditional<(M > 32), unsigned long long, uint32_t>::type;
};

template <int M>
struct RoundSmem {
    static constexpr int E = M * M;
    union {
        struct { unsigned long long key[E]; uint16_t idx[E]; } s;
        float G[E];
    } u;
    float a[E];
    unsigned long long rowbits[M];
    int rc[M];
    int cc[M];
};

template <int M>
__device__ __forceinline__ void warp_argmax(float& v, int& i) {
#pragma unroll
    for (int s = 16; s >= 1; s >>= 1) {
        const float ov = __shfl_xor_sync(kFullMask, v, s);
        const int oi = __shfl_xor_sync(kFullMask, i, s);
        if (ov > v || (ov == v && oi < i)) { v = ov; i = oi; }
    }
}

// Net gain of exchanging one entry between rows i and ip (see item 4 above).
template <int M>
__device__ __forceinline__ float pair_gain(const RoundSmem<M>& sm, int i, int ip) {
    const unsigned long long Oi = sm.rowbits[i], Op = sm.rowbits[ip];
    unsigned long long d1 = Oi & ~Op, d2 = Op & ~Oi;
    if (!d1) return -INFINITY;
    float t1 = -INFINITY, t2 = -INFINITY;
    while (d1) {
        const int j = __ffsll((long long)d1) - 1;
        d1 &= d1 - 1;
        t1 = fmaxf(t1, __fsub_rn(sm.a[ip * M + j], sm.a[i * M + j]));
    }
    while (d2) {
        const int j = __ffsll((long long)d2) - 1;
        d2 &= d2 - 1;
        t2 = fmaxf(t2, __fsub_rn(sm.a[i * M + j], sm.a[ip * M + j]));
    }
    return __fadd_rn(t1, t2);
}

// mask_mode: 0 = plain stores of whole bytes/halves/words (M >= 8),
//            1 = atomicOr into a zeroed mask (M = 4, two blocks share a byte).
template <int M, typename T>
__global__ void __launch_bounds__(RoundCfg<M>::WARPS * 32)
round_kernel(const float* __restrict__ plan, const typename T::storage* __restrict__ W,
             int64_t cols, int64_t n_blocks, int N, int sweeps, uint32_t* __restrict__ mask,
             int64_t wpr) {
    using Cfg = RoundCfg<M>;
    constexpr int E = Cfg::E;
    extern __shared__ __align__(16) unsigned char round_smem_raw[];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    RoundSmem<M>& sm = reinterpret_cast<RoundSmem<M>*>(round_smem_raw)[warp];
    const int64_t b = int64_t(blockIdx.x) * Cfg::WARPS + warp;
    if (b >= n_blocks) return;                       // uniform per warp
    const int64_t nbc = cols / M;
    const int64_t r0 = (b / nbc) * M, c0 = (b % nbc) * M;

    // ---- 1. keys
    bool ok = true;
    for (int e = lane; e < E; e += 32) {
        const int i = e / M, j = e % M;
        const float s = fabsf(plan[(r0 + i) * cols + c0 + j]);
        const float a = T::load1(W + (r0 + i) * cols + c0 + j);
        ok = ok && (s <= 3.402823466e38f) && (a <= 3.402823466e38f);
        sm.u.s.key[e] = (static_cast<unsigned long long>(__float_as_uint(s)) << 32) | __float_as_uint(a);
        sm.u.s.idx[e] = static_cast<uint16_t>(e);
        sm.a[e] = a;
    }
    for (int r = lane; r < M; r += 32) { sm.rc[r] = 0; sm.cc[r] = 0; sm.rowbits[r] = 0ull; }
    ok = __all_sync(kFullMask, ok);
    __syncwarp();

    if (ok) {
        // bitonic sort, descending in the rounding order
        for (int k = 2; k <= E; k <<= 1) {
            for (int j = k >> 1; j > 0; j >>= 1) {
                for (int u = lane; u < E / 2; u += 32) {
                    const int p = ((u & ~(j - 1)) << 1) | (u & (j - 1));
                    const int q = p | j;
                    const SortKey kp{sm.u.s.key[p], sm.u.s.idx[p]};
                    const SortKey kq{sm.u.s.key[q], sm.u.s.idx[q]};
                    const bool up = (p & k) == 0;
                    const bool swap = up ? key_before(kq, kp) : key_before(kp, kq);
                    if (swap) {
                        sm.u.s.key[p] = kq.k; sm.u.s.idx[p] = static_cast<uint16_t>(kq.idx);
                        sm.u.s.key[q] = kp.k; sm.u.s.idx[q] = static_cast<uint16_t>(kp.idx);
                    }
                }
                __syncwarp();
            }
        }

        // ---- 2. greedy, 32 sorted entries per step
        const int target = N * M;
        int taken = 0;
        for (int base = 0; base < E && taken < target; base += 32) {
            const int pos = base + lane;
            const bool valid = pos < E;
            const int e = valid ? sm.u.s.idx[pos] : 0;
            const int i = e / M, j = e % M;
            const unsigned mr = __match_any_sync(kFullMask, valid ? i : 4096 + lane);
            const unsigned mc = __match_any_sync(kFullMask, valid ? j : 8192 + lane);
            const unsigned lt = (1u << lane) - 1u;
            const int r0c = valid ? sm.rc[i] : N, c0c = valid ? sm.cc[j] : N;
            unsigned acc = 0u;
            unsigned und = __ballot_sync(kFullMask, valid && r0c < N && c0c < N);
            while (und) {
                const bool mine = (und >> lane) & 1u;
                const unsigned maybe = acc | und;
                const int ru = r0c + __popc(mr & lt & maybe), cu = c0c + __popc(mc & lt & maybe);
                const int rl = r0c + __popc(mr & lt & acc), cl = c0c + __popc(mc & lt & acc);
                const unsigned A = __ballot_sync(kFullMask, mine && ru < N && cu < N);
                const unsigned R = __ballot_sync(kFullMask, mine && (rl >= N || cl >= N));
                acc |= A;
                und &= ~(A | R);
            }
            if ((acc >> lane) & 1u) atomicOr(&sm.rowbits[i], 1ull << j);
            // row / column counts: the lowest accepted lane of each group adds the group's count
            if (((acc >> lane) & 1u) && (__ffs(mr & acc) - 1 == lane)) sm.rc[i] += __popc(mr & acc);
            if (((acc >> lane) & 1u) && (__ffs(mc & acc) - 1 == lane)) sm.cc[j] += __popc(mc & acc);
            taken += __popc(acc);
            __syncwarp();
        }

        // ---- 3. repair
        for (int guard = 0; guard <= target; ++guard) {
            unsigned long long shortR, shortC;
            if constexpr (M <= 32) {
                shortR = __ballot_sync(kFullMask, lane < M && sm.rc[lane] < N);
                shortC = __ballot_sync(kFullMask, lane < M && sm.cc[lane] < N);
            } else {
                shortR = __ballot_sync(kFullMask, sm.rc[lane] < N) |
                         (static_cast<unsigned long long>(__ballot_sync(kFullMask, sm.rc[lane + 32] < N)) << 32);
                shortC = __ballot_sync(kFullMask, sm.cc[lane] < N) |
                         (static_cast<unsigned long long>(__ballot_sync(kFullMask, sm.cc[lane + 32] < N)) << 32);
            }
            if (!shortR) break;
            if (!shortC || guard == target) { ok = false; break; }
            const int i = __ffsll((long long)shortR) - 1, j = __ffsll((long long)shortC) - 1;
            const unsigned long long Oi = sm.rowbits[i];
            float best = -INFINITY;
            int bflat = INT_MAX;
            for (int ip = lane; ip < M; ip += 32) {
                const unsigned long long Op = sm.rowbits[ip];
                if ((Op >> j) & 1ull) continue;
                unsigned long long cand = Op & ~Oi;
                while (cand) {
                    const int jp = __ffsll((long long)cand) - 1;
                    cand &= cand - 1;
                    const float sigma = __fsub_rn(__fadd_rn(sm.a[i * M + jp], sm.a[ip * M + j]), sm.a[ip * M + jp]);
                    const int flat = ip * M + jp;
                    if (sigma > best || (sigma == best && flat < bflat)) { best = sigma; bflat = flat; }
                }
            }
            warp_argmax<M>(best, bflat);
            if (bflat == INT_MAX) { ok = false; break; }
            if (lane == 0) {
                const int ip = bflat / M, jp = bflat % M;
                sm.rowbits[i] |= 1ull << jp;
                sm.rowbits[ip] = (sm.rowbits[ip] | (1ull << j)) & ~(1ull << jp);
                sm.rc[i] += 1;
                sm.cc[j] += 1;
            }
            __syncwarp();
        }
    }

    if (ok && sweeps > 0) {
        // ---- 4. local search with the cached symmetric gain table
        __syncwarp();
        for (int i = 0; i < M; ++i)
            for (int ip = i + 1 + lane; ip < M; ip += 32) {
                const float g = pair_gain<M>(sm, i, ip);
                sm.u.G[i * M + ip] = g;
                sm.u.G[ip * M + i] = g;
            }
        __syncwarp();
        int quiet = 0;                                   // anchors in a row without a swap
        for (int sw = 0; sw < sweeps && quiet < M; ++sw) {
            for (int i = 0; i < M && quiet < M; ++i) {
                float best = -INFINITY;
                int bp = INT_MAX;
                for (int ip = lane; ip < M; ip += 32) {
                    const float g = ip == i ? -INFINITY : sm.u.G[i * M + ip];
                    if (ip != i && (g > best || bp == INT_MAX)) { best = g; bp = ip; }
                }
                warp_argmax<M>(best, bp);
                if (!(best > 0.f)) { ++quiet; continue; }
                quiet = 0;
                // entries to exchange: lowest index on ties
                const unsigned long long Oi = sm.rowbits[i], Op = sm.rowbits[bp];
                float v1 = -INFINITY, v2 = -INFINITY;
                int j1 = INT_MAX, j2 = INT_MAX;
                for (int jj = lane; jj < M; jj += 32) {
                    const bool in_i = (Oi >> jj) & 1ull, in_p = (Op >> jj) & 1ull;
                    if (in_i && !in_p) {
                        const float d = __fsub_rn(sm.a[bp * M + jj], sm.a[i * M + jj]);
                        if (d > v1 || j1 == INT_MAX) { v1 = d; j1 = jj; }
                    }
                    if (!in_i && in_p) {
                        const float d = __fsub_rn(sm.a[i * M + jj], sm.a[bp * M + jj]);
                        if (d > v2 || j2 == INT_MAX) { v2 = d; j2 = jj; }
                    }
                }
                warp_argmax<M>(v1, j1);
                warp_argmax<M>(v2, j2);
                __syncwarp();
                if (j1 >= M || j2 >= M) { ++quiet; continue; }   // unreachable: best > 0 needs both sets
                if (lane == 0) {
                    sm.rowbits[i] = (Oi & ~(1ull << j1)) | (1ull << j2);
                    sm.rowbits[bp] = (Op & ~(1ull << j2)) | (1ull << j1);
                }
                __syncwarp();
                for (int ip = lane; ip < M; ip += 32) {
                    if (ip != i) {
                        const float g = pair_gain<M>(sm, i, ip);
                        sm.u.G[i * M + ip] = g;
                        sm.u.G[ip * M + i] = g;
                    }
                    if (ip != bp && ip != i) {
                        const float g = pair_gain<M>(sm, bp, ip);
                        sm.u.G[bp * M + ip] = g;
                        sm.u.G[ip * M + bp] = g;
                    }
                }
                __syncwarp();
            }
        }
    }
    __syncwarp();

    // ---- 5. packed mask rows
    if (!ok && lane == 0) atomicAdd(&g_block_failures, 1ull);
    for (int r = lane; r < M; r += 32) {
        const unsigned long long bits = ok ? sm.rowbits[r] : 0ull;
        uint32_t* row = mask + (r0 + r) * wpr;
        if constexpr (M == 64) {
            row[c0 / 32] = static_cast<uint32_t>(bits);
            row[c0 / 32 + 1] = static_cast<uint32_t>(bits >> 32);
        } else if constexpr (M == 32) {
            row[c0 / 32] = static_cast<uint32_t>(bits);
        } else if constexpr (M == 16) {
            reinterpret_cast<uint16_t*>(row)[c0 / 16] = static_cast<uint16_t>(bits);
        } else if constexpr (M == 8) {
            reinterpret_cast<uint8_t*>(row)[c0 / 8] = static_cast<uint8_t>(bits);
        } else {
            if (bits) atomicOr(&row[c0 / 32], static_cast<uint32_t>(bits) << (c0 % 32));
        }
    }
}

template <int M>
constexpr size_t round_smem() { return sizeof(RoundSmem<M>) * RoundCfg<M>::WARPS; }

}  // namespace tsenor
