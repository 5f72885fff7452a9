// Rounding of one block's fractional plan into a transposable N:M mask by one
// warp ("What carries the argument" and the Fig. 2 caption of the TSENOR
// review; referee comment 3 on the rounding stage).
//
//   1. sort: each lane holds R = E/32 keys in registers (E = M*M, padded to
//      32 for M = 4); a bitonic network orders them so that position
//      p = lane*R + r holds the p-th entry of the rounding order (plan desc,
//      |W| desc, flat index asc).  Distances below R are compare-exchanges
//      inside a lane, larger ones are shuffles between lanes;
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
//   5. the caller writes the row bitmasks.
// Every comparison that decides an integer uses fp32 values evaluated in the
// order written above.
#pragma once

#include <climits>
#include <type_traits>

#include "common.cuh"

namespace tsenor {

__device__ unsigned long long g_block_failures;   // blocks that could not be rounded

// Sort keys.  KeyB (bf16 input): the low 16 bits of |W| are zero, so one
// 64-bit word holds plan bits, |W| bits and the complemented index:
// a larger word is earlier in the rounding order.  KeyF (fp32 input): plan and
// |W| bits in one word, the index in a second one.
struct KeyB {
    unsigned long long k;
    __device__ __forceinline__ static KeyB make(float s, float a, int idx) {
        return KeyB{(static_cast<unsigned long long>(__float_as_uint(s)) << 32) |
                    (__float_as_uint(a) & 0xffff0000u) | (0xffffu - static_cast<unsigned>(idx))};
    }
    __device__ __forceinline__ static KeyB sentinel() { return KeyB{0ull}; }
    __device__ __forceinline__ int index() const { return int(0xffffu - unsigned(k & 0xffffu)); }
    __device__ __forceinline__ bool before(const KeyB& o) const { return k > o.k; }
    __device__ __forceinline__ KeyB shfl_xor(int m) const {
        return KeyB{__shfl_xor_sync(kFullMask, k, m)};
    }
};

struct KeyF {
    unsigned long long k;
    unsigned idx;
    __device__ __forceinline__ static KeyF make(float s, float a, int idx) {
        return KeyF{(static_cast<unsigned long long>(__float_as_uint(s)) << 32) | __float_as_uint(a),
                    static_cast<unsigned>(idx)};
    }
    __device__ __forceinline__ static KeyF sentinel() { return KeyF{0ull, 0xffffffffu}; }
    __device__ __forceinline__ int index() const { return int(idx); }
    __device__ __forceinline__ bool before(const KeyF& o) const { return k > o.k || (k == o.k && idx < o.idx); }
    __device__ __forceinline__ KeyF shfl_xor(int m) const {
        return KeyF{__shfl_xor_sync(kFullMask, k, m), __shfl_xor_sync(kFullMask, idx, m)};
    }
};

template <typename T> struct KeyOf;
template <> struct KeyOf<BF16> { using type = KeyB; };
template <> struct KeyOf<F32> { using type = KeyF; };

template <int M>
struct WarpRound {
    static constexpr int E = M * M;
    static constexpr int EP = E < 32 ? 32 : E;     // padded entry count
    static constexpr int R = EP / 32;              // keys per lane (M <= 32)
    static constexpr int AS = M + 1;               // row stride of |W| and of the gain table in smem
    using Bits = typename std::conditional<(M > 32), unsigned long long, unsigned>::type;   // one row
};

template <typename Bits>
__device__ __forceinline__ int lowest_bit(Bits x) {
    if constexpr (sizeof(Bits) == 8) return __ffsll(static_cast<long long>(x)) - 1;
    else return __ffs(static_cast<int>(x)) - 1;
}

// Where the rounding steps after the sort keep one block's state (shared
// memory).  A view of pointers, so that M = 64 can overlay the arrays of
// different steps (see Round64Smem).
template <int M>
struct RoundView {
    using Bits = typename WarpRound<M>::Bits;
    float* G;                           // cached pair gains (local search), row stride M+1
    uint16_t* order;                    // sorted flat indices
    Bits* rowbits;                      // row bitmasks of the mask being built
    float* bestv;                       // best gain of each row over its partners ...
    int* bestp;                         // ... and that partner (lowest index on ties)
    int* rc;                            // row counts (greedy, repair)
    int* cc;                            // column counts
    float* sc;                          // M <= 32: 4*M floats, 16-byte aligned (local search)
};

// Per-block shared memory of the rounding steps after the sort (M <= 32).
// The sorted order is read by the greedy only and the gain table is first
// written by the local search, after the greedy and the repair: they share
// their space.
template <int M>
struct RoundShared {
    using Bits = typename WarpRound<M>::Bits;
    static constexpr int GS = M + 1;
    union {
        float G[M * GS];
        uint16_t order[WarpRound<M>::EP];
    };
    Bits rowbits[M];
    float bestv[M];
    int bestp[M];
    int rc[M];
    int cc[M];
    float sc[4 * M];                    // local search: C and Bn of the two rows of the last swap
    __device__ __forceinline__ RoundView<M> view() { return RoundView<M>{G, order, rowbits, bestv, bestp, rc, cc, sc}; }
};

// Bitonic compare-exchange of registers r and r|J of this lane: the pair ends
// earliest-first when `up`.  The order is strict (no two keys of a block are
// equal), so one comparison decides either direction.
template <int R, int J, typename Key>
__device__ __forceinline__ void bitonic_regs(Key (&key)[R], bool up) {
#pragma unroll
    for (int r = 0; r < R; ++r) {
        if (r & J) continue;
        const Key x = key[r], y = key[r | J];
        const bool sw = y.before(x) == up;
        key[r] = sw ? y : x;
        key[r | J] = sw ? x : y;
    }
}

// In-register stages j = J, J/2, ..., 1 with a direction that is constant
// over this lane's registers.
template <int R, int J, typename Key>
__device__ __forceinline__ void bitonic_regs_down(Key (&key)[R], bool up) {
    if constexpr (J >= 1) {
        bitonic_regs<R, J>(key, up);
        bitonic_regs_down<R, J / 2>(key, up);
    }
}

// Phase 1 of the sort: each lane's R registers (positions lane*R + r) become a
// sorted run, earliest-first on even lanes and latest-first on odd lanes.
template <int R, int K, typename Key>
__device__ __forceinline__ void bitonic_local(Key (&key)[R], int lane) {
    if constexpr (K <= R) {
#pragma unroll
        for (int j = K / 2; j >= 1; j >>= 1) {
#pragma unroll
            for (int r = 0; r < R; ++r) {
                if (r & j) continue;
                const bool up = K < R ? ((r & K) == 0) : ((lane & 1) == 0);
                const Key x = key[r], y = key[r | j];
                const bool sw = y.before(x) == up;
                key[r] = sw ? y : x;
                key[r | j] = sw ? x : y;
            }
        }
        bitonic_local<R, K * 2>(key, lane);
    }
}

// Cross-lane stage: pair lane with lane ^ m, same register.
template <int R, typename Key>
__device__ __forceinline__ void bitonic_shfl(Key (&key)[R], int m, bool take_earlier) {
#pragma unroll
    for (int r = 0; r < R; ++r) {
        const Key x = key[r];
        const Key y = x.shfl_xor(m);
        key[r] = (y.before(x) == take_earlier) ? y : x;
    }
}

// Bitonic sort of 32*R keys held R per lane (position p = lane*R + r),
// earliest first.  Distances below R are compare-exchanges inside a lane,
// larger ones pair lane with lane ^ (j/R) through shuffles.
template <int R, typename Key>
__device__ __forceinline__ void warp_bitonic_sort(Key (&key)[R], int lane) {
    constexpr int EP = 32 * R;
    bitonic_local<R, 2>(key, lane);
#pragma unroll 1
    for (int k = 2 * R; k <= EP; k <<= 1) {
        const bool up = ((lane * R) & k) == 0;       // same for all of this lane's positions
#pragma unroll 1
        for (int j = k >> 1; j >= R; j >>= 1) {
            const int m = j / R;
            bitonic_shfl<R>(key, m, ((lane & m) == 0) == up);
        }
        bitonic_regs_down<R, R / 2>(key, up);
    }
}

// Bitonic sort of 4096 keys over a CTA of 4 warps (M = 64): 32 keys per
// thread at position t*32 + r (t = warp*32 + lane).  Distances of a warp's
// 1024 positions or more go through shared memory (xbuf: 4*32*32 keys).
template <typename Key>
__device__ void cta_bitonic_sort64(Key (&key)[32], Key* xbuf, int warp, int lane) {
    constexpr int R = 32, EP = 4096;
    const int t = warp * 32 + lane;
    bitonic_local<R, 2>(key, lane);
#pragma unroll 1
    for (int k = 2 * R; k <= EP; k <<= 1) {
        const bool up = ((t * R) & k) == 0;
#pragma unroll 1
        for (int j = k >> 1; j >= R; j >>= 1) {
            if (j >= 32 * R) {
                const int mw = j / (32 * R);
#pragma unroll
                for (int r = 0; r < R; ++r) xbuf[(warp * R + r) * 32 + lane] = key[r];
                __syncthreads();
                const bool take_earlier = ((warp & mw) == 0) == up;
#pragma unroll
                for (int r = 0; r < R; ++r) {
                    const Key x = key[r];
                    const Key y = xbuf[((warp ^ mw) * R + r) * 32 + lane];
                    key[r] = (y.before(x) == take_earlier) ? y : x;
                }
                __syncthreads();
            } else {
                const int m = j / R;
                bitonic_shfl<R>(key, m, ((lane & m) == 0) == up);
            }
        }
        bitonic_regs_down<R, R / 2>(key, up);
    }
}

// Integer image of a float that orders like the float (no NaN): the sign
// bit flips the order of the negative half.  -0 is first made +0 (x + 0 in
// round-to-nearest), so that the two zeros stay equal as in a float compare.
__device__ __forceinline__ int ordered_bits(float f) {
    const int b = __float_as_int(f + 0.f);
    return b >= 0 ? b : b ^ 0x7fffffff;
}
__device__ __forceinline__ float from_ordered_bits(int k) { return __int_as_float(k >= 0 ? k : k ^ 0x7fffffff); }

// Warp-wide (largest v, lowest i among the lanes holding it), returned to
// every lane: two warp reductions (redux.sync) instead of a shuffle butterfly.
__device__ __forceinline__ void warp_argmax(float& v, int& i) {
    const int k = ordered_bits(v);
    const int km = __reduce_max_sync(kFullMask, k);
    i = static_cast<int>(__reduce_min_sync(kFullMask, k == km ? static_cast<unsigned>(i) : 0xffffffffu));
    v = from_ordered_bits(km);
}

// Sorted keys of one warp into sh.order.
template <int M, typename Key>
__device__ __forceinline__ void keys_to_order(const Key (&key)[WarpRound<M>::R], const RoundView<M>& sh, int lane) {
    constexpr int R = WarpRound<M>::R, E = M * M;
#pragma unroll
    for (int r = 0; r < R; ++r) {
        const int idx = key[r].index();
        sh.order[lane * R + r] = static_cast<uint16_t>(idx < E ? idx : 0xffff);
    }
}

// Steps 2-3 (greedy, repair) for one block by one warp, from sh.order.
// Returns false when the block could not be made feasible.
template <int M, int EP>
__device__ bool greedy_and_repair(const float* a, const RoundView<M>& sh, int N, int lane) {
    using Bits = typename WarpRound<M>::Bits;
    constexpr int E = M * M, AS = M + 1;
    for (int r = lane; r < M; r += 32) { sh.rc[r] = 0; sh.cc[r] = 0; sh.rowbits[r] = 0; }
    __syncwarp();
    const int target = N * M;
    int taken = 0;
    const unsigned lt = (1u << lane) - 1u;
    // the next chunk's entries and row/column groups do not depend on this
    // chunk's decisions: they are fetched one chunk ahead
    int e_next = sh.order[lane];
    unsigned mr_next = __match_any_sync(kFullMask, e_next < E ? e_next / M : 4096 + lane);
    unsigned mc_next = __match_any_sync(kFullMask, e_next < E ? e_next % M : 8192 + lane);
    for (int base = 0; base < EP && taken < target; base += 32) {
        const int e = e_next;
        const unsigned mr = mr_next, mc = mc_next;
        if (base + 32 < EP) {
            e_next = sh.order[base + 32 + lane];
            mr_next = __match_any_sync(kFullMask, e_next < E ? e_next / M : 4096 + lane);
            mc_next = __match_any_sync(kFullMask, e_next < E ? e_next % M : 8192 + lane);
        }
        const bool valid = e < E;
        const int i = valid ? e / M : 0, j = valid ? e % M : 0;
        const int r0c = valid ? sh.rc[i] : N, c0c = valid ? sh.cc[j] : N;
        unsigned acc = 0u;
        unsigned und = __ballot_sync(kFullMask, valid && r0c < N && c0c < N);
        {   // first pass: nothing accepted yet, so the lower bound rejects no lane
            const bool mine = (und >> lane) & 1u;
            const int ru = r0c + __popc(mr & lt & und), cu = c0c + __popc(mc & lt & und);
            acc = __ballot_sync(kFullMask, mine && ru < N && cu < N);
            und &= ~acc;
        }
        while (und) {
            const bool mine = (und >> lane) & 1u;
            const unsigned maybe = acc | und;
            const int ru = r0c + __popc(mr & lt & maybe), cu = c0c + __popc(mc & lt & maybe);
            const int rl = r0c + __popc(mr & lt & acc), cl = c0c + __popc(mc & lt & acc);
            const unsigned A = __ballot_sync(kFullMask, mine && ru < N && cu < N);
            const unsigned Rj = __ballot_sync(kFullMask, mine && (rl >= N || cl >= N));
            acc |= A;
            und &= ~(A | Rj);
        }
        const bool mine_acc = (acc >> lane) & 1u;
        // accepted entries set their bit (32-bit shared atomics); the lowest
        // accepted lane of each row (column) group adds the group's count
        if (mine_acc) atomicOr(reinterpret_cast<unsigned*>(&sh.rowbits[i]) + (j >> 5), 1u << (j & 31));
        const unsigned ga = mr & acc, gc = mc & acc;
        if (ga && __ffs(ga) - 1 == lane) sh.rc[i] = r0c + __popc(ga);   // the counts read at the chunk's start
        if (gc && __ffs(gc) - 1 == lane) sh.cc[j] = c0c + __popc(gc);
        taken += __popc(acc);
        __syncwarp();
    }

    for (int guard = 0; guard <= target; ++guard) {
        unsigned long long shortR, shortC;
        if constexpr (M <= 32) {
            shortR = __ballot_sync(kFullMask, lane < M && sh.rc[lane] < N);
            shortC = __ballot_sync(kFullMask, lane < M && sh.cc[lane] < N);
        } else {
            shortR = __ballot_sync(kFullMask, sh.rc[lane] < N) |
                     (static_cast<unsigned long long>(__ballot_sync(kFullMask, sh.rc[lane + 32] < N)) << 32);
            shortC = __ballot_sync(kFullMask, sh.cc[lane] < N) |
                     (static_cast<unsigned long long>(__ballot_sync(kFullMask, sh.cc[lane + 32] < N)) << 32);
        }
        if (!shortR) return true;
        if (!shortC || guard == target) return false;
        const int i = __ffsll((long long)shortR) - 1, j = __ffsll((long long)shortC) - 1;
        const Bits Oi = sh.rowbits[i];
        float best = -INFINITY;
        int bflat = INT_MAX;
        for (int ip = lane; ip < M; ip += 32) {
            const Bits Op = sh.rowbits[ip];
            if ((Op >> j) & 1) continue;
            Bits cand = Op & ~Oi;
            while (cand) {
                const int jp = lowest_bit(cand);
                cand &= cand - 1;
                const float sigma = __fsub_rn(__fadd_rn(a[i * AS + jp], a[ip * AS + j]), a[ip * AS + jp]);
                const int flat = ip * M + jp;
                if (sigma > best || (sigma == best && flat < bflat)) { best = sigma; bflat = flat; }
            }
        }
        warp_argmax(best, bflat);
        if (bflat == INT_MAX) return false;
        if (lane == 0) {
            const int ip = bflat / M, jp = bflat % M;
            sh.rowbits[i] |= Bits(1) << jp;
            sh.rowbits[ip] = (sh.rowbits[ip] | (Bits(1) << j)) & ~(Bits(1) << jp);
            sh.rc[i] += 1;
            sh.cc[j] += 1;
        }
        __syncwarp();
    }
    return false;
}

// Thread layout of the local search: NT threads (one warp for M <= 32, a CTA
// of 4 warps for M = 64); thread tid serves partner row y = tid / CH and
// columns [h*CPT, (h+1)*CPT) of it, h = tid % CH.  Each thread keeps those
// |W| values of its row in registers.
// 3-input maximum (sm_100).
__device__ __forceinline__ float max3f(float a, float b, float c) {
    float d;
    asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
    return d;
}

template <int M>
struct LsCfg {
    static constexpr int NT = M <= 32 ? 32 : 128;
    static constexpr int CH = M <= 32 ? 1 : 2;      // threads per row
    static constexpr int CPT = M / CH;              // columns per thread
};

template <int NT>
__device__ __forceinline__ void ls_barrier() {
    if constexpr (NT == 32) __syncwarp(); else __syncthreads();
}

// Pair gain pieces of row y against row x over this thread's columns:
// txy = max over j in O_x \ O_y of (a_yj - a_xj), tyx = max over j in O_y \ O_x
// of (a_xj - a_yj); the net gain of the exchange is txy + tyx (item 4 above).
template <int M, int CPT, typename Bits>
__device__ __forceinline__ void pair_pieces(const float (&ay)[CPT], const float* ax, Bits Ox, Bits Oy, int j0,
                                            float& txy, float& tyx) {
    const Bits m1 = Ox & ~Oy, m2 = Oy & ~Ox;
#pragma unroll
    for (int jj = 0; jj < CPT; ++jj) {
        const int j = j0 + jj;
        const float d = __fsub_rn(ay[jj], ax[j]);
        if ((m1 >> j) & 1) txy = fmaxf(txy, d);
        if ((m2 >> j) & 1) tyx = fmaxf(tyx, -d);
    }
}

template <int CH>
__device__ __forceinline__ float row_max(float t) {
#pragma unroll
    for (int s = 1; s < CH; s <<= 1) t = fmaxf(t, __shfl_xor_sync(kFullMask, t, s));
    return t;
}

// Best partner of row x over the cached gains (lowest partner index on ties).
// The diagonal G[x][x] holds -inf (set with the table), so it never beats a
// partner: with N < M every row has a partner of finite gain (two rows with
// the same support in every pair would put M ones in those columns); with
// N = M every gain is -inf and no swap ever happens, whichever index is kept.
// Quads are reduced independently, then merged in index order.  rescan_row_val
// returns the best, rescan_row stores it in sh.bestv / sh.bestp.
template <int M>
__device__ __forceinline__ void rescan_row_val(const RoundView<M>& sh, int x, float& best_v, int& best_p) {
    constexpr int GS = M + 1;
    static_assert(M % 4 == 0, "quads");
    const float* row = sh.G + x * GS;
    float bv = -INFINITY;
    int bp = -1;
#pragma unroll
    for (int q = 0; q < M / 4; ++q) {
        const float g0 = row[4 * q], g1 = row[4 * q + 1], g2 = row[4 * q + 2], g3 = row[4 * q + 3];
        const bool s01 = g1 > g0, s23 = g3 > g2;
        const float v01 = s01 ? g1 : g0, v23 = s23 ? g3 : g2;
        const int i01 = 4 * q + (s01 ? 1 : 0), i23 = 4 * q + (s23 ? 3 : 2);
        const bool s = v23 > v01;
        const float vq = s ? v23 : v01;
        const int iq = s ? i23 : i01;
        if (q == 0 || vq > bv) { bv = vq; bp = iq; }
    }
    best_v = bv;
    best_p = bp;
}
template <int M>
__device__ __forceinline__ void rescan_row(const RoundView<M>& sh, int x) {
    float bv;
    int bp;
    rescan_row_val<M>(sh, x, bv, bp);
    sh.bestv[x] = bv;
    sh.bestp[x] = bp;
}

// Step 4 for one block by LsCfg<M>::NT threads: the gain table, the row
// bests, then the sweeps.  `a`: |W| with row stride M+1.
template <int M>
__device__ void local_search(const float* a, const RoundView<M>& sh, int sweeps, int tid) {
    using L = LsCfg<M>;
    using Bits = typename WarpRound<M>::Bits;
    constexpr int AS = M + 1, GS = M + 1, NT = L::NT, CH = L::CH, CPT = L::CPT;
    const int lane = tid & 31;
    const int y = tid / CH, h = tid % CH, j0 = h * CPT;
    const bool row_thread = y < M;
    float ay[CPT];
#pragma unroll
    for (int jj = 0; jj < CPT; ++jj) ay[jj] = row_thread ? a[y * AS + j0 + jj] : 0.f;

    // gain table: row y with rows y+1 .. y+M/2 (mod M), every unordered pair once
    {
        const Bits Oy = row_thread ? sh.rowbits[y] : Bits(0);
        if (row_thread && h == 0) sh.G[y * GS + y] = -INFINITY;   // no partner of itself (rescan_row)
#pragma unroll 1
        for (int d = 1; d <= M / 2; ++d) {
            const int x = (y + d) & (M - 1);
            float txy = -INFINITY, tyx = -INFINITY;
            if (row_thread) pair_pieces<M, CPT, Bits>(ay, a + x * AS, sh.rowbits[x], Oy, j0, txy, tyx);
            txy = row_max<CH>(txy);
            tyx = row_max<CH>(tyx);
            if (row_thread && h == 0 && !(d == M / 2 && y >= M / 2)) {
                const float g = __fadd_rn(txy, tyx);
                sh.G[x * GS + y] = g;
                sh.G[y * GS + x] = g;
            }
        }
    }
    ls_barrier<NT>();
    // each row's best partner and gain: M = 32 keeps them in the row's lane
    // (reg_bests), M = 16 in shared memory
    constexpr bool reg_bests = M == 32;
    float my_bv = -INFINITY;
    int my_bp = 0;
    if constexpr (reg_bests) rescan_row_val<M>(sh, y, my_bv, my_bp);
    else if (row_thread && h == 0) rescan_row<M>(sh, y);

    // The sweeps compute pair gains in max-plus form: with C_x[j] = a_xj off
    // row x's support (-inf on it) and Bn_x[j] = a_xj on it (+inf off it),
    // max over j in O_x \ O_y of (a_yj - a_xj) = max_j (C_y[j] - Bn_x[j]) and
    // max over j in O_y \ O_x of (a_xj - a_yj) = max_j (C_x[j] - Bn_y[j]):
    // the same fp32 differences, with no per-column tests.  Each lane keeps
    // its own row in that form; after a swap the two changed rows are written
    // to sh.sc, where every lane reads them.
    static_assert(NT == 32 && CH == 1 && M % 4 == 0, "one row per lane");
    constexpr int M2 = M / 2;
    float2 Cy[M2], Bny[M2];
    {
        const Bits Oy = row_thread ? sh.rowbits[y] : Bits(0);
#pragma unroll
        for (int c = 0; c < M2; ++c) {
            const bool in0 = (Oy >> (2 * c)) & 1, in1 = (Oy >> (2 * c + 1)) & 1;
            Cy[c] = make_float2(in0 ? -INFINITY : ay[2 * c], in1 ? -INFINITY : ay[2 * c + 1]);
            Bny[c] = make_float2(in0 ? ay[2 * c] : INFINITY, in1 ? ay[2 * c + 1] : INFINITY);
        }
    }
    ls_barrier<NT>();

    int quiet = 0;                                   // anchors in a row without a swap
    for (int sw = 0; sw < sweeps && quiet < M; ++sw) {
        for (int i = 0; i < M && quiet < M; ++i) {
            {   // skip anchors with no positive best gain (fixed between swaps)
                const Bits P = __ballot_sync(kFullMask, lane < M && (reg_bests ? my_bv : sh.bestv[lane]) > 0.f);
                const Bits ahead = P & (~Bits(0) << i);
                if (!ahead) { quiet += M - i; break; }
                const int nxt = lowest_bit(ahead);
                quiet += nxt - i;
                i = nxt;
                if (quiet >= M) break;
            }
            const float best = reg_bests ? __shfl_sync(kFullMask, my_bv, i) : sh.bestv[i];
            const int bp = reg_bests ? __shfl_sync(kFullMask, my_bp, i) : sh.bestp[i];
            if (!(best > 0.f)) { ++quiet; continue; }
            const Bits Oi = sh.rowbits[i], Ob = sh.rowbits[bp];
            // entries to exchange (every lane finds the same pair): lowest index on ties
            float v1 = -INFINITY, v2 = -INFINITY;
            int j1 = INT_MAX, j2 = INT_MAX;
            const float ai = row_thread ? a[i * AS + lane] : 0.f, ab = row_thread ? a[bp * AS + lane] : 0.f;
            if (row_thread) {
                const bool in_i = (Oi >> lane) & 1, in_p = (Ob >> lane) & 1;
                if (in_i && !in_p) { v1 = __fsub_rn(ab, ai); j1 = lane; }
                if (!in_i && in_p) { v2 = __fsub_rn(ai, ab); j2 = lane; }
            }
            warp_argmax(v1, j1);
            warp_argmax(v2, j2);
            if (j1 >= M || j2 >= M) { ++quiet; continue; }   // unreachable: a positive gain needs both sets
            quiet = 0;
            const Bits Oi2 = (Oi & ~(Bits(1) << j1)) | (Bits(1) << j2);
            const Bits Ob2 = (Ob & ~(Bits(1) << j2)) | (Bits(1) << j1);
            // sc was last read before the previous swap's final barrier, so it
            // is written at once; the row masks after the next barrier, when
            // every lane has read the old ones
            if (row_thread) {                        // rows i and bp after the swap: C, Bn, C, Bn
                const bool ni = (Oi2 >> lane) & 1, nb = (Ob2 >> lane) & 1;
                sh.sc[lane] = ni ? -INFINITY : ai;
                sh.sc[M + lane] = ni ? ai : INFINITY;
                sh.sc[2 * M + lane] = nb ? -INFINITY : ab;
                sh.sc[3 * M + lane] = nb ? ab : INFINITY;
            }
            ls_barrier<NT>();
            if (tid == 0) {
                sh.rowbits[i] = Oi2;
                sh.rowbits[bp] = Ob2;
            }
            if (y == i || y == bp) {                 // this lane's own row changed
                const float* src = sh.sc + (y == i ? 0 : 2 * M);
#pragma unroll
                for (int q = 0; q < M / 4; ++q) {
                    const float4 c4 = *reinterpret_cast<const float4*>(src + 4 * q);
                    const float4 b4 = *reinterpret_cast<const float4*>(src + M + 4 * q);
                    Cy[2 * q] = make_float2(c4.x, c4.y);
                    Cy[2 * q + 1] = make_float2(c4.z, c4.w);
                    Bny[2 * q] = make_float2(b4.x, b4.y);
                    Bny[2 * q + 1] = make_float2(b4.z, b4.w);
                }
            }
            // new gains g(i, y) and g(bp, y) of partner row y
            float t1i0 = -INFINITY, t1i1 = -INFINITY, t2i0 = -INFINITY, t2i1 = -INFINITY;
            float t1b0 = -INFINITY, t1b1 = -INFINITY, t2b0 = -INFINITY, t2b1 = -INFINITY;
#pragma unroll
            for (int q = 0; q < M / 4; ++q) {
                const float4 ci = *reinterpret_cast<const float4*>(sh.sc + 4 * q);
                const float4 bi = *reinterpret_cast<const float4*>(sh.sc + M + 4 * q);
                const float4 cb = *reinterpret_cast<const float4*>(sh.sc + 2 * M + 4 * q);
                const float4 bb = *reinterpret_cast<const float4*>(sh.sc + 3 * M + 4 * q);
                float2 d;
                d = sub2(Cy[2 * q], make_float2(bi.x, bi.y));     t1i0 = max3f(t1i0, d.x, d.y);
                d = sub2(Cy[2 * q + 1], make_float2(bi.z, bi.w)); t1i1 = max3f(t1i1, d.x, d.y);
                d = sub2(make_float2(ci.x, ci.y), Bny[2 * q]);     t2i0 = max3f(t2i0, d.x, d.y);
                d = sub2(make_float2(ci.z, ci.w), Bny[2 * q + 1]); t2i1 = max3f(t2i1, d.x, d.y);
                d = sub2(Cy[2 * q], make_float2(bb.x, bb.y));     t1b0 = max3f(t1b0, d.x, d.y);
                d = sub2(Cy[2 * q + 1], make_float2(bb.z, bb.w)); t1b1 = max3f(t1b1, d.x, d.y);
                d = sub2(make_float2(cb.x, cb.y), Bny[2 * q]);     t2b0 = max3f(t2b0, d.x, d.y);
                d = sub2(make_float2(cb.z, cb.w), Bny[2 * q + 1]); t2b1 = max3f(t2b1, d.x, d.y);
            }
            const float gi = __fadd_rn(fmaxf(t1i0, t1i1), fmaxf(t2i0, t2i1));
            const float gb = __fadd_rn(fmaxf(t1b0, t1b1), fmaxf(t2b0, t2b1));
            if (row_thread) {
                if (y != i) { sh.G[i * GS + y] = gi; sh.G[y * GS + i] = gi; }
                if (y != i && y != bp) { sh.G[bp * GS + y] = gb; sh.G[y * GS + bp] = gb; }
            }
            ls_barrier<NT>();                        // gain table and rows complete
            {
                // rows i and bp, and rows whose best partner was one of them, are
                // rescanned: for M = 32 by the whole warp, one row at a time (a
                // warp argmax over the row's cached gains: lowest partner on ties,
                // the diagonal is -inf; rows i and bp from the new gains in the
                // lanes' registers), for M = 16 each by its own lane (a row of 16
                // gains); every other row compares its best with its new
                // g(i, y), g(bp, y).  A/B: 16:32 3.499 -> 3.444 ms per call with
                // the warp rescans, 8:16 1.125 -> 1.139 (so M = 16 keeps its own)
                // A row whose best partner was i (bp) needs no rescan while its new
                // gain with that partner has not fallen below the old best: every
                // other partner's gain is unchanged and at most that value, and one
                // equal to it has a higher index; the compare below then gives
                // the same best as a rescan.  M = 16 rescans such rows anyway (its
                // own-lane rescans are short: 8:16 1.067 -> 1.073 ms with the test,
                // 16:32 3.286 -> 3.188 ms with it and the direct bests below).
                const int op = reg_bests ? my_bp : (row_thread ? sh.bestp[y] : 0);
                const float ov = reg_bests ? my_bv : (row_thread ? sh.bestv[y] : 0.f);
                const bool mine = y == i || y == bp;
                const bool fell = M < 32 || (op == i ? gi : gb) < ov;
                const bool need = row_thread && (mine || ((op == i || op == bp) && fell));
                if constexpr (M < 32) {
                    if (need) rescan_row<M>(sh, y);
                }
                if (row_thread && !need) {
                    float bv = ov;
                    int b2 = op;
                    const int c1 = i < bp ? i : bp, c2 = i < bp ? bp : i;
                    const float g1 = c1 == i ? gi : gb, g2 = c2 == i ? gi : gb;
                    if (g1 > bv || (g1 == bv && c1 < b2)) { bv = g1; b2 = c1; }
                    if (g2 > bv || (g2 == bv && c2 < b2)) { bv = g2; b2 = c2; }
                    if constexpr (reg_bests) {
                        my_bv = bv;
                        my_bp = b2;
                    } else {
                        sh.bestv[y] = bv;
                        sh.bestp[y] = b2;
                    }
                }
                if constexpr (M == 32) {
                    // rows i and bp: their new gains are this warp's gi and gb (the
                    // diagonal -inf; lane i's gb = g(bp, i) is lane bp's gi with
                    // the two terms added in the other order, the same value)
                    float vi = y == i ? -INFINITY : gi, vb = y == bp ? -INFINITY : gb;
                    int pi = y, pb = y;
                    warp_argmax(vi, pi);
                    warp_argmax(vb, pb);
                    if (lane == i) { my_bv = vi; my_bp = pi; }
                    if (lane == bp) { my_bv = vb; my_bp = pb; }
                }
                unsigned rows = M < 32 ? 0u : __ballot_sync(kFullMask, need && !mine);
                while (rows) {
                    const int x = __ffs(static_cast<int>(rows)) - 1;
                    rows &= rows - 1;
                    float g = lane < M ? sh.G[x * GS + lane] : -INFINITY;
                    int p = lane;
                    warp_argmax(g, p);
                    if (lane == x) {                    // M = 32: reg_bests
                        my_bv = g;
                        my_bp = p;
                    }
                }
            }
            ls_barrier<NT>();                        // row bests complete
        }
    }
}

// ---------------------------------------------------------------------------
// Sorting on 32-bit keys (bf16 inputs, blocks of E = M*M >= 256 entries).
// The rounding order is (plan desc, |W| desc, flat index asc), a 64-bit key
// (KeyB).  A 32-bit key orders all but a few entries the same way and halves
// the work of every compare-exchange and shuffle.  Its IB = log2 E low bits
// hold E-1-idx, the 32-IB bits above them a bucket of the plan:
//   - plan exactly 1 (clipped): nibble 15, then the |W| bits: exact among
//     the clipped entries and above every other bucket;
//   - plan in [2^-14, 1): nibble e-112 (e the biased exponent, 113..126),
//     then the MB = 28-IB upper mantissa bits;
//   - plan below 2^-14: nibble 0, then the plan's bits shifted right so that
//     they fit the MB bits (monotone, coarse).
// The 4-bit exponent window spends the key's bits on the binades the plans
// occupy (on the synthetic 32:64 workload, tau = 30, every plan lies in
// [2^-8, 1]), so that 4096-entry blocks keep 16 mantissa bits (A/B against
// the plan's upper bits without the window, 4096x11008 16:32 workload: 3.413
// -> 3.289 ms per call).  After sorting on it, runs of
// adjacent entries in the same bucket (near-ties, usually of two) are ordered
// by the full key with a few passes of odd-even transposition; a block that
// has not settled after kFixPasses passes (long runs of equal plans, as in a
// constant block) is sorted again on the 64-bit keys.
// ---------------------------------------------------------------------------
struct Key32 {
    unsigned k;
    __device__ __forceinline__ bool before(const Key32& o) const { return k > o.k; }
    __device__ __forceinline__ Key32 shfl_xor(int m) const { return Key32{__shfl_xor_sync(kFullMask, k, m)}; }
};

template <int E>
struct Key32Fmt {
    static constexpr int IB = E == 256 ? 8 : E == 1024 ? 10 : 12;
    static_assert((1 << IB) == E, "E = 256, 1024 or 4096");
    static constexpr int MB = 28 - IB;                // mantissa bits of a bucket
    static constexpr unsigned kIdx = E - 1;
    static constexpr unsigned kOne = 0x3F800000u;     // bits of 1.0f
    static constexpr unsigned kLowExp = 112;          // biased exponents up to this share nibble 0
    __device__ __forceinline__ static unsigned make(unsigned long long kb) {
        const unsigned s = static_cast<unsigned>(kb >> 32);
        const unsigned inv = static_cast<unsigned>(kb) & kIdx;                  // E-1-idx
        const unsigned ex = s >> 23;
        const unsigned bucket =
            s >= kOne ? ((15u << MB) | (static_cast<unsigned>(kb >> 16) & 0xffffu))
            : ex > kLowExp ? (((ex - kLowExp) << MB) | ((s >> (23 - MB)) & ((1u << MB) - 1u)))
                           : (s >> (30 - MB));
        return (bucket << IB) | inv;
    }
    __device__ __forceinline__ static bool clipped(unsigned k) { return (k >> 28) == 15u; }
    __device__ __forceinline__ static int index(unsigned k) { return static_cast<int>(kIdx - (k & kIdx)); }
};

constexpr int kFixPasses = 8;

// Adjacent sorted keys x (earlier) and y: true when the full key puts y first.
// Only entries below 1 in the same bucket can be out of order;
// their full keys are compared out of line (rare, and it keeps the unrolled
// passes short: the fused kernels' code competes for the instruction cache).
// sbits: plan bits by flat index; a: |W| with row stride M+1.
template <int M>
__device__ __noinline__ bool fix_swap_full(unsigned x, unsigned y, const unsigned* sbits, const float* a) {
    using F = Key32Fmt<M * M>;
    const int ix = F::index(x), iy = F::index(y);
    const unsigned long long kx = (static_cast<unsigned long long>(sbits[ix]) << 32) |
                                  (__float_as_uint(a[(ix / M) * (M + 1) + ix % M]) & 0xffff0000u) |
                                  (0xffffu - static_cast<unsigned>(ix));
    const unsigned long long ky = (static_cast<unsigned long long>(sbits[iy]) << 32) |
                                  (__float_as_uint(a[(iy / M) * (M + 1) + iy % M]) & 0xffff0000u) |
                                  (0xffffu - static_cast<unsigned>(iy));
    return ky > kx;
}
template <int M>
__device__ __forceinline__ bool fix_swap(unsigned x, unsigned y, const unsigned* sbits, const float* a) {
    using F = Key32Fmt<M * M>;
    if (F::clipped(x) || ((x ^ y) & ~F::kIdx)) return false;
    return fix_swap_full<M>(x, y, sbits, a);
}

// Odd-even transposition over the warp's sorted keys (position lane*R + r)
// with the full key; returns whether a full pass made no exchange.
template <int M, int R>
__device__ bool fix_near_ties(Key32 (&k)[R], const unsigned* sbits, const float* a, int lane) {
    static_assert(R % 2 == 0, "pairs (2m, 2m+1) within a lane");
#pragma unroll 1
    for (int pass = 0; pass < kFixPasses; ++pass) {
        bool moved = false;
#pragma unroll
        for (int r = 0; r < R; r += 2)
            if (fix_swap<M>(k[r].k, k[r + 1].k, sbits, a)) { const Key32 t = k[r]; k[r] = k[r + 1]; k[r + 1] = t; moved = true; }
#pragma unroll
        for (int r = 1; r + 1 < R; r += 2)
            if (fix_swap<M>(k[r].k, k[r + 1].k, sbits, a)) { const Key32 t = k[r]; k[r] = k[r + 1]; k[r + 1] = t; moved = true; }
        // the pair across the lane boundary: both lanes take the same decision
        const unsigned nxt = __shfl_down_sync(kFullMask, k[0].k, 1);
        const unsigned prv = __shfl_up_sync(kFullMask, k[R - 1].k, 1);
        const bool down = lane < 31 && fix_swap<M>(k[R - 1].k, nxt, sbits, a);
        const bool up = lane > 0 && fix_swap<M>(prv, k[0].k, sbits, a);
        if (down) k[R - 1].k = nxt;
        if (up) k[0].k = prv;
        moved = moved || down || up;
        if (!__any_sync(kFullMask, moved)) return true;
    }
    return false;
}

// The 64-bit sort of a block whose 32-bit keys did not settle, from the plan
// bits (sbits, by flat index), |W| and the index: out of line, so that this
// rarely taken path does not enlarge the fused kernels' loops (the
// instruction cache of an SM holds the code of warps in every phase).
template <int M>
__device__ __noinline__ void sort_to_order_full(const unsigned* sbits, const float* a, const RoundView<M>& sh,
                                                int lane) {
    constexpr int R = WarpRound<M>::R;
    KeyB kb[R];
#pragma unroll
    for (int r = 0; r < R; ++r) {
        const int e = lane * R + r;                  // any assignment of entries to positions
        kb[r] = KeyB::make(__uint_as_float(sbits[e]), a[(e / M) * (M + 1) + e % M], e);
    }
    warp_bitonic_sort<R>(kb, lane);
    __syncwarp();                                    // sbits read by every lane before the order overlays it
    keys_to_order<M>(kb, sh, lane);
}

// Step 1 for bf16 keys: sort on Key32, settle the near-ties, write the order;
// a block that does not settle is sorted on its 64-bit keys.  sbits: E words
// of shared memory that the order does not need until this returns (the gain
// table's space).
template <int M>
__device__ void sort_to_order(KeyB (&key)[WarpRound<M>::R], const float* a, const RoundView<M>& sh,
                              unsigned* sbits, int lane) {
    constexpr int R = WarpRound<M>::R, E = M * M;
    using F = Key32Fmt<E>;
    static_assert(E % 32 == 0 && E >= 256, "no padding keys");
    Key32 k[R];
    bool above_one = false;                          // a given plan above 1: only the 64-bit keys order it
#pragma unroll
    for (int r = 0; r < R; ++r) {
        const unsigned sb = static_cast<unsigned>(key[r].k >> 32);
        sbits[key[r].index()] = sb;
        above_one = above_one || sb > F::kOne;
        k[r] = Key32{F::make(key[r].k)};
    }
    __syncwarp();
    bool fast = !__any_sync(kFullMask, above_one);
    if (fast) {
        warp_bitonic_sort<R>(k, lane);
        fast = fix_near_ties<M, R>(k, sbits, a, lane);
    }
    if (fast) {
        __syncwarp();                                // sbits read by every lane before the order overlays it
#pragma unroll
        for (int r = 0; r < R; ++r) sh.order[lane * R + r] = static_cast<uint16_t>(F::index(k[r].k));
    } else {
        sort_to_order_full<M>(sbits, a, sh, lane);
    }
}

// Steps 1-4 for one block (M <= 32).  `key` holds this lane's keys (any
// assignment of the block's entries to positions; padding positions hold
// Key::sentinel()), `a` the block's |W| (row stride M+1, shared memory).
// Returns false when the block could not be made feasible (never expected,
// see the repair proof); the final row bitmasks are in sh.rowbits.
template <int M, typename Key>
__device__ bool round_block_warp(Key (&key)[WarpRound<M>::R], const float* a, const RoundView<M>& sh, int N,
                                 int sweeps, int lane) {
    constexpr int R = WarpRound<M>::R;
    if constexpr (std::is_same<Key, KeyB>::value && M >= 16) {
        sort_to_order<M>(key, a, sh, reinterpret_cast<unsigned*>(sh.G), lane);
    } else {
        warp_bitonic_sort<R>(key, lane);
        keys_to_order<M>(key, sh, lane);
    }
    __syncwarp();
    if (!greedy_and_repair<M, WarpRound<M>::EP>(a, sh, N, lane)) return false;
    if (sweeps <= 0) return true;
    __syncwarp();
    local_search<M>(a, sh, sweeps, lane);
    return true;
}

// Row bitmasks of one block into the packed mask as whole words or halves
// (M = 16, 32, 64; the small-block kernels write their rows themselves).
template <int M>
__device__ __forceinline__ void write_mask_rows(uint32_t* mask, int64_t wpr, int64_t r0, int64_t c0,
                                                const typename WarpRound<M>::Bits* rowbits, bool ok, int lane,
                                                int nthreads = 32) {
    static_assert(M == 16 || M == 32 || M == 64, "whole halves or words per row");
    for (int r = lane; r < M; r += nthreads) {
        const unsigned long long bits = ok ? static_cast<unsigned long long>(rowbits[r]) : 0ull;
        uint32_t* row = mask + (r0 + r) * wpr;
        if constexpr (M == 64) {
            row[c0 / 32] = static_cast<uint32_t>(bits);
            row[c0 / 32 + 1] = static_cast<uint32_t>(bits >> 32);
        } else if constexpr (M == 32) {
            row[c0 / 32] = static_cast<uint32_t>(bits);
        } else {
            reinterpret_cast<uint16_t*>(row)[c0 / 16] = static_cast<uint16_t>(bits);
        }
    }
}

}  // namespace tsenor

namespace tsenor {

// Rounding of a given plan, one warp per block (M = 16, 32).  Entry e = r*32 + lane
// of the block (row-major flat index) goes to this lane's register r, so the
// loads of plan and W are coalesced along block rows.
template <int M>
struct RoundWarpSmem {
    float a[M * (M + 1)];           // |W|, row stride M+1
    RoundShared<M> sh;
};

template <int M, typename T>
__global__ void __launch_bounds__(128)
round_warp_kernel(const float* __restrict__ plan, const typename T::storage* __restrict__ W, int64_t cols,
                  int64_t n_blocks, int N, int sweeps, uint32_t* __restrict__ mask, int64_t wpr) {
    using Key = typename KeyOf<T>::type;
    constexpr int E = M * M, R = WarpRound<M>::R;
    extern __shared__ __align__(16) unsigned char round_warp_raw[];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    RoundWarpSmem<M>& sm = reinterpret_cast<RoundWarpSmem<M>*>(round_warp_raw)[warp];
    const int64_t b = int64_t(blockIdx.x) * 4 + warp;
    if (b >= n_blocks) return;                       // uniform per warp
    const int64_t nbc = cols / M;
    const int64_t r0 = (b / nbc) * M, c0 = (b % nbc) * M;

    Key key[R];
    bool ok = true;
#pragma unroll
    for (int r = 0; r < R; ++r) {
        const int e = r * 32 + lane;
        if (e < E) {
            const int i = e / M, j = e % M;
            const float s = fabsf(plan[(r0 + i) * cols + c0 + j]);
            const float a = T::load1(W + (r0 + i) * cols + c0 + j);
            ok = ok && (s <= 3.402823466e38f) && (a <= 3.402823466e38f);
            sm.a[i * (M + 1) + j] = a;
            key[r] = Key::make(s, a, e);
        } else {
            key[r] = Key::sentinel();
        }
    }
    ok = __all_sync(kFullMask, ok);
    __syncwarp();
    if (ok) ok = round_block_warp<M, Key>(key, sm.a, sm.sh.view(), N, sweeps, lane);
    if (!ok && lane == 0) atomicAdd(&g_block_failures, 1ull);
    __syncwarp();
    write_mask_rows<M>(mask, wpr, r0, c0, sm.sh.rowbits, ok, lane);
}

template <int M>
constexpr size_t round_warp_smem() { return sizeof(RoundWarpSmem<M>) * 4; }

// ---------------------------------------------------------------------------
// M = 64: one CTA of 4 warps per block.  The 4096 keys are sorted by the
// whole CTA (32 per thread); greedy and repair run on warp 0; the local
// search runs on all 128 threads (two per row) in max-plus form:
//   B_x[j] = -a_xj for j in O_x, else -inf;  C_x[j] = a_xj for j not in O_x,
//   else -inf;  g(x, y) = max_j (C_y[j] + B_x[j]) + max_j (C_x[j] + B_y[j]).
// C_y[j] + B_x[j] is a_yj - a_xj exactly (IEEE a - b is a + (-b)) where j is
// in O_x \ O_y and -inf elsewhere, so g is the same fp32 value as the
// bit-tested form used for M <= 32, with no per-column tests.
// ---------------------------------------------------------------------------


// B and C rows in shared memory (row stride M floats) keep their 16-byte
// chunks XOR-swizzled: logical chunk c of row r is stored at chunk
// c ^ (r % 16) ^ (4 if c >= 8).  The row term puts chunk c of different rows
// in different bank groups (the gain table setup, where the threads read
// different rows); the last term does the same for chunks c and c + 8 of one
// row, which the two threads of a row read together (the sweeps, where every
// thread reads the same row): without it the two fall in the same bank group
// (ncu on 1024x8192 32:64: 43.8 M -> 2.5 M shared-load bank conflicts; 33.82
// -> 32.41 ms per 8192x28672 call).
template <int M>
__device__ __forceinline__ int bc_index(int r, int j) {
    return r * M + ((((j >> 2) ^ r ^ ((j >> 5) << 2)) & (M / 4 - 1)) << 2) + (j & 3);
}

// max_j (u[j] + v[j]) over this thread's CPT columns (logical chunks c0 ..
// c0 + CPT/4 - 1) of row r of a swizzled B or C array.
template <int M, int CPT>
__device__ __forceinline__ float max_plus(const float (&u)[CPT], const float* arr, int r, int c0) {
    float t0 = -INFINITY, t1 = -INFINITY;
    const float* row = arr + r * M;
#pragma unroll
    for (int q = 0; q < CPT / 4; ++q) {
        const int c = c0 + q;                        // logical chunk; stored as bc_index places it
        const float4 w = *reinterpret_cast<const float4*>(row + (((c ^ r ^ ((c >> 3) << 2)) & (M / 4 - 1)) << 2));
        const float2 s0 = add2(make_float2(u[4 * q], u[4 * q + 1]), make_float2(w.x, w.y));
        const float2 s1 = add2(make_float2(u[4 * q + 2], u[4 * q + 3]), make_float2(w.z, w.w));
        t0 = max3f(t0, s0.x, s0.y);
        t1 = max3f(t1, s1.x, s1.y);
    }
    return fmaxf(t0, t1);
}

// Best partner of row x (lowest partner index on ties) by the two threads of
// row x, each scanning half of the cached gains; both threads must call it.
template <int M>
__device__ __forceinline__ void rescan_row_pair(const RoundView<M>& sh, int x, int h, int lane) {
    constexpr int GS = M + 1, HALF = M / 2;
    float g[HALF];
#pragma unroll
    for (int k = 0; k < HALF; ++k) g[k] = sh.G[x * GS + h * HALF + k];
    float bv = -INFINITY;
    int bp = -1;
#pragma unroll
    for (int k = 0; k < HALF; ++k) {
        const int y = h * HALF + k;
        if (y == x) continue;
        if (bp < 0 || g[k] > bv) { bv = g[k]; bp = y; }
    }
    const unsigned pair = 3u << (lane & 30);
    const float ov = __shfl_xor_sync(pair, bv, 1);
    const int op = __shfl_xor_sync(pair, bp, 1);
    // the lower half's candidate wins ties (lower partner index)
    if (h == 0 ? (ov > bv) : !(bv > ov)) { bv = ov; bp = op; }
    if (h == 0) {
        sh.bestv[x] = bv;
        sh.bestp[x] = bp;
    }
}

// Step 4 for one M = 64 block by 128 threads.  `a`: |W| (row stride M+1),
// read only until the B/C arrays are built; sh.G may overlay it.  Bm, Cm:
// M x M floats each (swizzled rows, bc_index), 16-byte aligned; xj: two ints
// of shared memory (the pair of each swap).
template <int M>
__device__ void local_search_mp(const float* a, float* Bm, float* Cm, const RoundView<M>& sh, int* xj, int sweeps,
                                int tid) {
    using L = LsCfg<M>;
    using Bits = typename WarpRound<M>::Bits;
    constexpr int AS = M + 1, GS = M + 1, CH = L::CH, CPT = L::CPT;
    static_assert(L::NT == 2 * M && CH == 2, "two threads per row");
    const int lane = tid & 31;
    const int y = tid / CH, h = tid % CH, j0 = h * CPT;
    float By[CPT], Cy[CPT];                          // this thread's columns of B_y and C_y
    {
        const Bits Oy = sh.rowbits[y];
#pragma unroll
        for (int jj = 0; jj < CPT; ++jj) {
            const float v = a[y * AS + j0 + jj];
            const bool in = (Oy >> (j0 + jj)) & 1;
            By[jj] = in ? -v : -INFINITY;
            Cy[jj] = in ? -INFINITY : v;
        }
#pragma unroll
        for (int q = 0; q < CPT / 4; ++q) {
            const int e = bc_index<M>(y, j0 + 4 * q);
            *reinterpret_cast<float4*>(Bm + e) = make_float4(By[4 * q], By[4 * q + 1], By[4 * q + 2], By[4 * q + 3]);
            *reinterpret_cast<float4*>(Cm + e) = make_float4(Cy[4 * q], Cy[4 * q + 1], Cy[4 * q + 2], Cy[4 * q + 3]);
        }
    }
    __syncthreads();                                 // B, C complete; |W| is not read again (G may overlay it)

    // gain table: row y with rows y+1 .. y+M/2 (mod M), every unordered pair once
#pragma unroll 1
    for (int d = 1; d <= M / 2; ++d) {
        const int x = (y + d) & (M - 1);
        const float txy = row_max<CH>(max_plus<M, CPT>(Cy, Bm, x, j0 / 4));   // j in O_x \ O_y: a_yj - a_xj
        const float tyx = row_max<CH>(max_plus<M, CPT>(By, Cm, x, j0 / 4));   // j in O_y \ O_x: a_xj - a_yj
        if (h == 0 && !(d == M / 2 && y >= M / 2)) {
            const float g = __fadd_rn(txy, tyx);
            sh.G[x * GS + y] = g;
            sh.G[y * GS + x] = g;
        }
    }
    __syncthreads();
    rescan_row_pair<M>(sh, y, h, lane);
    __syncthreads();

    int quiet = 0;                                   // anchors in a row without a swap
    for (int sw = 0; sw < sweeps && quiet < M; ++sw) {
        for (int i = 0; i < M && quiet < M; ++i) {
            {   // skip anchors with no positive best gain (fixed between swaps)
                const Bits P = (static_cast<Bits>(__ballot_sync(kFullMask, sh.bestv[lane + 32] > 0.f)) << 32) |
                               __ballot_sync(kFullMask, sh.bestv[lane] > 0.f);
                const Bits ahead = P & (~Bits(0) << i);
                if (!ahead) { quiet += M - i; break; }
                const int nxt = lowest_bit(ahead);
                quiet += nxt - i;
                i = nxt;
                if (quiet >= M) break;
            }
            const float best = sh.bestv[i];
            const int bp = sh.bestp[i];
            if (!(best > 0.f)) { ++quiet; continue; }
            // entries to exchange, by warp 0 alone (lowest index on ties), which
            // also applies the swap: since the last barrier no other warp has
            // read rows i and bp, and the next barrier publishes the result
            if (tid < 32) {
                float v1 = -INFINITY, v2 = -INFINITY;
                int j1 = INT_MAX, j2 = INT_MAX;
#pragma unroll
                for (int jj = lane; jj < M; jj += 32) {
                    const int ei = bc_index<M>(i, jj), eb = bc_index<M>(bp, jj);
                    const float d1 = Cm[eb] + Bm[ei];                  // j in O_i \ O_bp: a_bp,j - a_ij
                    if (d1 > -INFINITY && (j1 == INT_MAX || d1 > v1)) { v1 = d1; j1 = jj; }
                    const float d2 = Cm[ei] + Bm[eb];                  // j in O_bp \ O_i: a_ij - a_bp,j
                    if (d2 > -INFINITY && (j2 == INT_MAX || d2 > v2)) { v2 = d2; j2 = jj; }
                }
                warp_argmax(v1, j1);
                warp_argmax(v2, j2);
                __syncwarp();                        // the warp has read rows i and bp
                if (j1 < M && j2 < M) {              // always: a positive gain needs both sets
                    if (tid < 4) {
                        // j1 leaves row i for row bp, j2 leaves row bp for row i: one entry per thread
                        const int r = tid < 2 ? i : bp;
                        const int j = (tid == 0 || tid == 3) ? j1 : j2;
                        const int e = bc_index<M>(r, j);
                        const bool leaves = (tid & 1) == 0;   // (i, j1) and (bp, j2) leave their rows
                        const float b = Bm[e], c = Cm[e];
                        Bm[e] = leaves ? -INFINITY : -c;
                        Cm[e] = leaves ? -b : -INFINITY;
                    } else if (tid == 4) {
                        const Bits Oi = sh.rowbits[i], Ob = sh.rowbits[bp];
                        sh.rowbits[i] = (Oi & ~(Bits(1) << j1)) | (Bits(1) << j2);
                        sh.rowbits[bp] = (Ob & ~(Bits(1) << j2)) | (Bits(1) << j1);
                    }
                }
                if (tid == 0) { xj[0] = j1; xj[1] = j2; }
            }
            __syncthreads();                         // rows i and bp updated, the pair published
            if (xj[0] >= M || xj[1] >= M) {          // unreachable (uniform)
                __syncthreads();                     // xj read by all before warp 0 writes it again
                ++quiet;
                continue;
            }
            quiet = 0;
            if (y == i || y == bp) {
#pragma unroll
                for (int q = 0; q < CPT / 4; ++q) {
                    const int e = bc_index<M>(y, j0 + 4 * q);
                    const float4 wb = *reinterpret_cast<const float4*>(Bm + e);
                    const float4 wc = *reinterpret_cast<const float4*>(Cm + e);
                    By[4 * q] = wb.x; By[4 * q + 1] = wb.y; By[4 * q + 2] = wb.z; By[4 * q + 3] = wb.w;
                    Cy[4 * q] = wc.x; Cy[4 * q + 1] = wc.y; Cy[4 * q + 2] = wc.z; Cy[4 * q + 3] = wc.w;
                }
            }
            // new gains g(i, y) and g(bp, y) of partner row y
            const float t1i = row_max<CH>(max_plus<M, CPT>(Cy, Bm, i, j0 / 4));
            const float t2i = row_max<CH>(max_plus<M, CPT>(By, Cm, i, j0 / 4));
            const float t1b = row_max<CH>(max_plus<M, CPT>(Cy, Bm, bp, j0 / 4));
            const float t2b = row_max<CH>(max_plus<M, CPT>(By, Cm, bp, j0 / 4));
            const float gi = __fadd_rn(t1i, t2i), gb = __fadd_rn(t1b, t2b);
            if (h == 0) {
                if (y != i) { sh.G[i * GS + y] = gi; sh.G[y * GS + i] = gi; }
                if (y != i && y != bp) { sh.G[bp * GS + y] = gb; sh.G[y * GS + bp] = gb; }
            }
            __syncthreads();                         // gain table and rows complete
            {
                // rows i and bp, and rows whose best partner was one of them: each
                // warp rescans those of its 16 rows one at a time (a warp argmax
                // over the row's 64 cached gains, lowest partner on ties; the
                // diagonal, which holds no gain, is skipped); every other row
                // compares its best with its new g(i, y), g(bp, y)
                // (a row whose best partner was i or bp and whose gain with it has
                // not fallen keeps a best among i and bp, as in local_search)
                const int op = sh.bestp[y];
                const float ov = sh.bestv[y];
                const bool need = y == i || y == bp ||
                                  ((op == i || op == bp) && (op == i ? gi : gb) < ov);   // same for both threads of row y
                if (!need && h == 0) {
                    float bv = ov;
                    int b2 = op;
                    const int c1 = i < bp ? i : bp, c2 = i < bp ? bp : i;
                    const float g1 = c1 == i ? gi : gb, g2 = c2 == i ? gi : gb;
                    if (g1 > bv || (g1 == bv && c1 < b2)) { bv = g1; b2 = c1; }
                    if (g2 > bv || (g2 == bv && c2 < b2)) { bv = g2; b2 = c2; }
                    sh.bestv[y] = bv;
                    sh.bestp[y] = b2;
                }
                unsigned rows = __ballot_sync(kFullMask, need && h == 0);   // bit 2k: row 16 * warp + k
                while (rows) {
                    const int x = (tid >> 5) * 16 + (__ffs(static_cast<int>(rows)) - 1) / 2;
                    rows &= rows - 1;
                    const float g0 = lane == x ? -INFINITY : sh.G[x * GS + lane];
                    const float g1 = lane + 32 == x ? -INFINITY : sh.G[x * GS + lane + 32];
                    const bool hi = g1 > g0;                  // lower column on ties
                    float g = hi ? g1 : g0;
                    int p = (hi ? lane + 32 : lane) == x ? 0x7fff : (hi ? lane + 32 : lane);
                    warp_argmax(g, p);
                    if (lane == 0) {
                        sh.bestv[x] = g;
                        sh.bestp[x] = p;
                    }
                }
            }
            __syncthreads();                         // row bests complete
        }
    }
}

// Shared memory of one M = 64 block; the arrays of successive steps overlay.
template <typename Key>
struct Round64Smem {
    union {
        Key xbuf[4096];                              // sort exchange between warps
        struct {
            uint16_t order[4096];                    // sorted flat indices
            int rc[64], cc[64];
        } gr;                                        // greedy and repair
        float bc[2 * 64 * 64];                       // local search: B, then C (row stride 64)
    } u;
    float a[64 * 65];                                // |W| (row stride 65); the gain table G in the local search
    static constexpr int kColbufFloats = 512;
    union {
        float colbuf[kColbufFloats];                 // Dykstra phase of the fused kernel: cross-warp column sums
        struct {
            unsigned long long rowbits[64];
            float bestv[64];
            int bestp[64];
        } rb;
    } v;
    int ok;
    int xj[2];                                       // local search: the entries of the current swap
    unsigned bnd[8];                                 // 32-bit sort: first and last key of each warp
    uint64_t tma_bar;                                // fused kernel: completion of the W tile copy
    __device__ __forceinline__ RoundView<64> view() {
        return RoundView<64>{a, u.gr.order, v.rb.rowbits, v.rb.bestv, v.rb.bestp, u.gr.rc, u.gr.cc, nullptr};
    }
};

// Odd-even transposition over the CTA's 4096 sorted 32-bit keys (position
// t*32 + r, t = warp*32 + lane) with the full key, as fix_near_ties; the
// pairs across warps go through sm.bnd.  Returns whether a full pass made
// no exchange (uniform over the CTA).
__device__ bool cta_fix_near_ties64(Key32 (&k)[32], const unsigned* sbits, const float* a, unsigned* bnd, int warp,
                                    int lane) {
    constexpr int R = 32, M = 64;
#pragma unroll 1
    for (int pass = 0; pass < kFixPasses; ++pass) {
        bool moved = false;
#pragma unroll
        for (int r = 0; r < R; r += 2)
            if (fix_swap<M>(k[r].k, k[r + 1].k, sbits, a)) { const Key32 t = k[r]; k[r] = k[r + 1]; k[r + 1] = t; moved = true; }
#pragma unroll
        for (int r = 1; r + 1 < R; r += 2)
            if (fix_swap<M>(k[r].k, k[r + 1].k, sbits, a)) { const Key32 t = k[r]; k[r] = k[r + 1]; k[r + 1] = t; moved = true; }
        unsigned nxt = __shfl_down_sync(kFullMask, k[0].k, 1);
        unsigned prv = __shfl_up_sync(kFullMask, k[R - 1].k, 1);
        if (lane == 0) bnd[warp] = k[0].k;
        if (lane == 31) bnd[4 + warp] = k[R - 1].k;
        __syncthreads();
        if (lane == 31 && warp < 3) nxt = bnd[warp + 1];
        if (lane == 0 && warp > 0) prv = bnd[4 + warp - 1];
        // both threads of a pair take the same decision from the same two keys
        const bool down = (lane < 31 || warp < 3) && fix_swap<M>(k[R - 1].k, nxt, sbits, a);
        const bool up = (lane > 0 || warp > 0) && fix_swap<M>(prv, k[0].k, sbits, a);
        if (down) k[R - 1].k = nxt;
        if (up) k[0].k = prv;
        moved = moved || down || up;
        if (!__syncthreads_or(moved)) return true;   // also orders this pass's bnd reads before the next writes
    }
    return false;
}

// The 64-bit sort of an M = 64 block whose 32-bit keys did not settle (or
// that holds a plan above 1), from the plan bits (sbits, by flat index) and
// |W|; out of line, as sort_to_order_full.
__device__ __noinline__ void cta_sort_to_order64_full(const unsigned* sbits, Round64Smem<KeyB>& sm, int warp,
                                                      int lane) {
    constexpr int M = 64, R = 32;
    const int t = warp * 32 + lane;
    KeyB kb[R];
#pragma unroll
    for (int r = 0; r < R; ++r) {
        const int e = t * R + r;                     // any assignment of entries to positions
        kb[r] = KeyB::make(__uint_as_float(sbits[e]), sm.a[(e / M) * (M + 1) + e % M], e);
    }
    __syncthreads();                                 // sbits read by all before the exchange space is reused
    cta_bitonic_sort64(kb, sm.u.xbuf, warp, lane);
    __syncthreads();
#pragma unroll
    for (int r = 0; r < R; ++r) sm.u.gr.order[t * R + r] = static_cast<uint16_t>(kb[r].index());
}

// Step 1 for one M = 64 block of bf16 keys by the CTA: sort on Key32 (the
// exchange buffer in the first 16 KB of the block's exchange space, the plan
// bits by flat index in the second), settle the near-ties, write the order;
// a block that does not settle is sorted on its 64-bit keys.  Every thread
// calls it.  A/B against the 64-bit sort, 8192x28672 32:64 workload: 34.99 ->
// 34.05 ms per call (a bucket of the plan's upper 20 bits, without the
// exponent window, had left too many near-ties: 35.00 -> 35.42 ms).
__device__ void cta_sort_to_order64(KeyB (&key)[32], Round64Smem<KeyB>& sm, int warp, int lane) {
    constexpr int R = 32, E = 4096;
    using F = Key32Fmt<E>;
    static_assert(sizeof(sm.u) >= 2 * E * sizeof(unsigned), "exchange space: keys and plan bits");
    static_assert(sizeof(uint16_t) * E + sizeof(int) * 128 <= sizeof(unsigned) * E, "the order stays clear of sbits");
    Key32* xbuf = reinterpret_cast<Key32*>(&sm.u);
    unsigned* sbits = reinterpret_cast<unsigned*>(&sm.u) + E;
    const int t = warp * 32 + lane;
    Key32 k[R];
    bool above_one = false;                          // a given plan above 1: only the 64-bit keys order it
#pragma unroll
    for (int r = 0; r < R; ++r) {
        const unsigned sb = static_cast<unsigned>(key[r].k >> 32);
        sbits[key[r].index()] = sb;
        above_one = above_one || sb > F::kOne;
        k[r] = Key32{F::make(key[r].k)};
    }
    bool fast = !__syncthreads_or(above_one);        // also publishes sbits
    if (fast) {
        cta_bitonic_sort64(k, xbuf, warp, lane);     // ends with a barrier after its last exchange
        fast = cta_fix_near_ties64(k, sbits, sm.a, sm.bnd, warp, lane);
    }
    if (fast) {
        // the order overlays the key exchange buffer (no longer read), not sbits
#pragma unroll
        for (int r = 0; r < R; ++r) sm.u.gr.order[t * R + r] = static_cast<uint16_t>(F::index(k[r].k));
    } else {
        cta_sort_to_order64_full(sbits, sm, warp, lane);
    }
}

// Steps 1-4 for one M = 64 block by a CTA of 4 warps (every thread calls it;
// the result is uniform over the CTA).  `key`: this thread's 32 keys; sm.a:
// the block's |W|.  The final row bitmasks are in sm.v.rb.rowbits.
template <typename Key>
__device__ bool round_block_cta64(Key (&key)[32], Round64Smem<Key>& sm, int N, int sweeps, int tid) {
    constexpr int M = 64;
    const int lane = tid & 31, warp = tid >> 5;
    const RoundView<M> sh = sm.view();
    if constexpr (std::is_same<Key, KeyB>::value) {
        cta_sort_to_order64(key, sm, warp, lane);
    } else {
        cta_bitonic_sort64(key, sm.u.xbuf, warp, lane);
        __syncthreads();
#pragma unroll
        for (int r = 0; r < 32; ++r) sh.order[tid * 32 + r] = static_cast<uint16_t>(key[r].index());
    }
    __syncthreads();
    if (warp == 0) {
        const bool g = greedy_and_repair<M, 4096>(sm.a, sh, N, lane);
        if (lane == 0) sm.ok = g;
    }
    __syncthreads();
    const bool ok = sm.ok;
    if (ok && sweeps > 0) {
        local_search_mp<M>(sm.a, sm.u.bc, sm.u.bc + M * M, sh, sm.xj, sweeps, tid);
        __syncthreads();
    }
    return ok;
}

template <typename T>
__global__ void __launch_bounds__(128)
round_cta64_kernel(const float* __restrict__ plan, const typename T::storage* __restrict__ W, int64_t cols,
                   int64_t n_blocks, int N, int sweeps, uint32_t* __restrict__ mask, int64_t wpr) {
    constexpr int M = 64, AS = 65;
    using Key = typename KeyOf<T>::type;
    extern __shared__ __align__(16) unsigned char round64_raw[];
    Round64Smem<Key>& sm = *reinterpret_cast<Round64Smem<Key>*>(round64_raw);
    const int tid = threadIdx.x;
    const int64_t b = blockIdx.x;
    if (b >= n_blocks) return;                       // uniform per CTA
    const int64_t nbc = cols / M;
    const int64_t r0 = (b / nbc) * M, c0 = (b % nbc) * M;

    Key key[32];
    bool ok = true;
#pragma unroll
    for (int r = 0; r < 32; ++r) {
        const int e = r * 128 + tid;
        const int i = e / M, j = e % M;
        const float s = fabsf(plan[(r0 + i) * cols + c0 + j]);
        const float a = T::load1(W + (r0 + i) * cols + c0 + j);
        ok = ok && (s <= 3.402823466e38f) && (a <= 3.402823466e38f);
        sm.a[i * AS + j] = a;
        key[r] = Key::make(s, a, e);
    }
    ok = __syncthreads_and(ok);
    if (ok) ok = round_block_cta64(key, sm, N, sweeps, tid);
    if (!ok && tid == 0) atomicAdd(&g_block_failures, 1ull);
    write_mask_rows<M>(mask, wpr, r0, c0, sm.v.rb.rowbits, ok, tid, 128);
}

}  // namespace tsenor
