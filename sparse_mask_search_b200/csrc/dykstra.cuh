// Dykstra's algorithm for the entropic capacitated transport relaxation of
// every MxM block ("What carries the argument" and "Core claim" of the TSENOR
// review; minor comment 2 on Algorithm 1).
//
// Math used by every kernel here (exact in real arithmetic):
//  * State in base-2 log units.  After a clip, x = min(y, 0) and the Dykstra
//    correction is logQ = max(y, 0) for y = x + logQ, so one number y per
//    entry carries both.  Starting from y0 = (x0 - tau) * log2(e) keeps
//    y0 <= 0 (so logQ0 = 0) and changes nothing: the first row step is blind
//    to a constant shift of a row.
//  * One iteration with e_ij = 2^min(y_ij, 0):
//        R_i = sum_j e_ij          r_i = log2 N - log2 R_i     (row step)
//        C_j = sum_i e_ij N / R_i  c_j = log2 N - log2 C_j     (column step,
//                                  reusing the row step's exponentials)
//        y_ij += r_i + c_j                                     (clip folded in)
//    Written this way it takes one exponential per entry and iteration; the
//    kernels below carry E = 2^y instead (row factors as clip thresholds,
//    column factors on E) and rebuild it only at anchor points, as
//    E = 2^y0 * 2^U_i * 2^V_j, see dykstra_tile_solve.
//  * The plan is S = 2^min(y, 0) = min(E, 1) after the last iteration.
//  * Since y only ever gains r_i + c_j, y = y0 + U_i + V_j with U, V the
//    potentials accumulated so far: the 2M numbers (U, V) are the whole
//    state of a block.  The EXT kernels start from given (U, V) (warm
//    start), export the final ones, and may stop a block early once every
//    |r_i| and |c_j| of an iteration is at most a tolerance.  The review fixes
//    T with no convergence test ("Assumptions & free parameters"); this is
//    the library's extension, and U = V = 0 with no tolerance is exactly the
//    plain solve.
#pragma once

#include <type_traits>

#include "../../include/tsenor.h"
#include "common.cuh"
#include "tma.cuh"

namespace tsenor {

constexpr float kLog2e = 1.4426950408889634f;
constexpr double kLog2eD = 1.4426950408889634;
constexpr double kLn2D = 0.6931471805599453;

// Warm start / adaptive stopping arguments of the EXT kernels.
struct DykstraExt {
    float* potentials;      // [n_blocks][2M]: U_0..U_{M-1}, V_0..V_{M-1} (nats); in when warm, always out
    int32_t* iters_used;    // [n_blocks] iterations run, or null
    float tol2;             // stop tolerance on |r_i|, |c_j| in log2 units; 0 = run all iterations
    int warm;               // nonzero: start from `potentials`
};

// Iterations between two anchor points of the linear-form exponentials
// (see dykstra_tile_solve).
constexpr int kAnchorEvery = 64;

// Largest tau the kernels accept (TSENOR_MAX_TAU; the host rejects larger
// ones): E0 = 2^y0 spans 2^-tau2 .. 1 within a block (tau2 = tau * log2(e)),
// which must stay inside the normal fp32 range; at tau = 80, tau2 = 115.4.
constexpr float kMaxTau = TSENOR_MAX_TAU;

// 2^y for a double y in [-126, 126] (clamped), as fp32, to within the
// hardware exponential's error: y = n + f with n the nearest integer (the
// 1.5 * 2^52 shift leaves n in the low word of the sum) and |f| <= 1/2, so
// the fp32 rounding of f costs at most 2^-26 in the exponent, and 2^n is an
// exact scaling.  Used where the exponent is large but its result must be
// good to a few ulps: E0 = 2^y0 and the potentials' factors 2^U, 2^V.
__device__ __forceinline__ float exp2_wide(double y) {
    y = fmin(fmax(y, -126.0), 126.0);
    constexpr double kShift = 6755399441055744.0;    // 1.5 * 2^52
    const double s = y + kShift;
    const int n = __double2loint(s);
    const float f = __double2float_rn(y - (s - kShift));
    return ex2(f) * __int_as_float((n + 127) << 23);
}


// ---------------------------------------------------------------------------
// M = 4, 8: one thread holds a whole block in registers.  Rows are streamed:
// the exponentials of one row live only until its column contributions are
// added, so no cross-thread traffic is needed at all.
// ---------------------------------------------------------------------------
// Shared-memory load of a float4 that the compiler may not move out of a loop.
__device__ __forceinline__ float4 lds4_keep(const float* p) {
    float4 v;
    asm volatile("ld.shared.v4.f32 {%0, %1, %2, %3}, [%4];"
                 : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w)
                 : "r"(static_cast<unsigned>(__cvta_generic_to_shared(p))));
    return v;
}

// Dykstra for block b (rows r0.., columns c0..) by one thread, in the form of
// dykstra_tile_solve: the state is y = y0 + U_i + V_j, E = 2^y = F / TH_i is
// carried in linear form between anchor points (the row step sets the row's
// clip threshold TH_i, the column step multiplies F by N / C_j) and
// recomputed every kAnchorEvery iterations as (E0_ij * 2^U_i) * 2^V_j with
// E0 = 2^y0, when the logarithms of the thresholds and of the column factors'
// products are added to U and V (fp32), so the potentials follow the very
// factors applied.  y0s: this thread's M*M floats of shared memory (16-byte
// aligned), which hold E0 during the iterations.  On return `s` holds the plan
// 2^min(y, 0); returns whether the block's W is finite.
template <int M, typename T, bool EXT = false>
__device__ __forceinline__ bool dykstra_thread_solve(const typename T::storage* __restrict__ W, int64_t cols,
                                                     int64_t b, int64_t r0, int64_t c0, int N, float tau,
                                                     int iters, const DykstraExt& ext, float (&s)[M][M],
                                                     float* y0s) {
    float (&y)[M][M] = s;                            // |W|, then y0, then the plan
#pragma unroll
    for (int i = 0; i < M; ++i) {
        const typename T::storage* src = W + (r0 + i) * cols + c0;
        if constexpr (M * sizeof(typename T::storage) >= 16) {
#pragma unroll
            for (int v = 0; v < M / T::kVec; ++v) T::load16(src + v * T::kVec, &y[i][v * T::kVec]);
        } else {
#pragma unroll
            for (int j = 0; j < M; ++j) y[i][j] = T::load1(src + j);
        }
    }
    float m = 0.f;
    bool finite = true;
#pragma unroll
    for (int i = 0; i < M; ++i)
#pragma unroll
        for (int j = 0; j < M; ++j) {
            finite = finite && (y[i][j] <= 3.402823466e38f);   // false for NaN and Inf
            m = fmaxf(m, y[i][j]);
        }
    // y0 in fp64 (as the oracle's x0), kept as E0 = 2^y0
    const double tau2d = double(tau) * kLog2eD;
    const double inv_m = m > 0.f ? 1.0 / double(m) : 0.0;
#pragma unroll
    for (int i = 0; i < M; ++i) {
#pragma unroll
        for (int j = 0; j < M; ++j) y[i][j] = exp2_wide(fma(tau2d, double(y[i][j]) * inv_m, -tau2d));
#pragma unroll
        for (int v = 0; v < M / 4; ++v)
            reinterpret_cast<float4*>(y0s + i * M)[v] = make_float4(y[i][4 * v], y[i][4 * v + 1], y[i][4 * v + 2],
                                                                    y[i][4 * v + 3]);
        // one row's fp64 temporaries at a time: with the rows interleaved the
        // compiler kept many of them live and spilled the solver's registers
        asm volatile("" ::: "memory");
    }
    const float fN = float(N);

    // potentials (log2 units) as of the last anchor point; since then each
    // row's scaling lives in its clip threshold TH (E = F / TH, see
    // dykstra_tile_solve) and the column scalings multiply F, their products
    // kept in PV; both are added to U and V at the next anchor point
    const float invN = 1.f / float(N);
    float U[M], V[M], TH[M], PV[M];
    int used = 0;
    {
        const float* uv = nullptr;
        if constexpr (EXT) uv = ext.warm ? ext.potentials + 2 * M * b : nullptr;
#pragma unroll
        for (int k = 0; k < M; ++k) {
            U[k] = uv ? float(double(uv[k]) * kLog2eD) : 0.f;
            V[k] = uv ? float(double(uv[M + k]) * kLog2eD) : 0.f;
            TH[k] = 1.f;
            PV[k] = 1.f;
        }
    }
    auto flush = [&]() {
#pragma unroll
        for (int k = 0; k < M; ++k) {
            U[k] -= lg2(TH[k]);
            V[k] += lg2(PV[k]);
            PV[k] = 1.f;
        }
    };
    // column pairs (j, j+1) as packed fp32x2 values
    constexpr int M2 = M / 2;
    float2 E2[M][M2];                                // F
    // F = 2^(y0 + U_i + V_j) = (E0_ij * 2^U_i) * 2^V_j, so that the rounding
    // of the large potentials is common to a row or a column.  The factors
    // stay in the fp32 range while every |U_i|, |V_j| is below 124 (from a
    // cold start they stay within about tau * log2(e) + log2(M) <= 122); a
    // warm start from potentials beyond that takes the exponent
    // lg2(E0) + U_i + V_j per entry instead.
    auto anchor = [&]() {
        flush();
        float span = 0.f;
#pragma unroll
        for (int k = 0; k < M; ++k) {
            TH[k] = 1.f;
            span = fmaxf(span, fmaxf(fabsf(U[k]), fabsf(V[k])));
        }
        if (span < 124.f) {
            float2 Q2v[M2];
#pragma unroll
            for (int c = 0; c < M2; ++c) Q2v[c] = make_float2(ex2(V[2 * c]), ex2(V[2 * c + 1]));
#pragma unroll
            for (int i = 0; i < M; ++i) {
                const float p = ex2(U[i]);
                const float2 p2 = make_float2(p, p);
#pragma unroll
                for (int v = 0; v < M / 4; ++v) {
                    const float4 q = lds4_keep(y0s + i * M + 4 * v);
                    E2[i][2 * v] = mul2(mul2(make_float2(q.x, q.y), p2), Q2v[2 * v]);
                    E2[i][2 * v + 1] = mul2(mul2(make_float2(q.z, q.w), p2), Q2v[2 * v + 1]);
                }
            }
        } else {
#pragma unroll
            for (int i = 0; i < M; ++i)
#pragma unroll
                for (int v = 0; v < M / 4; ++v) {
                    const float4 q = lds4_keep(y0s + i * M + 4 * v);
                    E2[i][2 * v] = make_float2(ex2(lg2(q.x) + (U[i] + V[4 * v])), ex2(lg2(q.y) + (U[i] + V[4 * v + 1])));
                    E2[i][2 * v + 1] = make_float2(ex2(lg2(q.z) + (U[i] + V[4 * v + 2])),
                                                   ex2(lg2(q.w) + (U[i] + V[4 * v + 3])));
                }
        }
    };
    // one call site, at the top of each anchor period: with a second call
    // before the loop the compiler laid the loop out slower (A/B: one 4:8
    // matrix 0.93 -> 1.00 ms, the 16:32 plan kernel 2.11 -> 2.64 ms); the
    // result is unused for a non-finite block, which runs no period
    bool stop = !finite;
#pragma unroll 1
    for (int t0 = 0; t0 < iters && !stop; t0 += kAnchorEvery) {
        anchor();
        const int t1 = min(iters, t0 + kAnchorEvery);
#pragma unroll 1
        for (int t = t0; t < t1; ++t) {
            float delta = 0.f;                         // largest |r_i|, |c_j| of this iteration (EXT)
            float2 C2[M2];
#pragma unroll
            for (int c = 0; c < M2; ++c) C2[c] = make_float2(0.f, 0.f);
#pragma unroll
            for (int i = 0; i < M; ++i) {
                float2 e2[M2];
#pragma unroll
                for (int c = 0; c < M2; ++c) e2[c] = make_float2(fminf(E2[i][c].x, TH[i]), fminf(E2[i][c].y, TH[i]));
                float2 acc = e2[0];
#pragma unroll
                for (int c = 1; c < M2; ++c) acc = add2(acc, e2[c]);
                const float S = acc.x + acc.y;
                const float w = fN * rcp(S);             // weight of min(F, TH) in the column step
                const float2 w2 = make_float2(w, w);
#pragma unroll
                for (int c = 0; c < M2; ++c) C2[c] = fma2(e2[c], w2, C2[c]);
                const float tn = S * invN;               // threshold after the row step
                if constexpr (EXT) {
                    if (ext.tol2 > 0.f) delta = fmaxf(delta, fabsf(lg2(TH[i]) - lg2(tn)));
                }
                TH[i] = tn;
            }
#pragma unroll
            for (int c = 0; c < M2; ++c) {
                const float2 u2 = make_float2(fN * rcp(C2[c].x), fN * rcp(C2[c].y));   // N / C_j = 2^c_j
#pragma unroll
                for (int i = 0; i < M; ++i) E2[i][c] = mul2(E2[i][c], u2);
                PV[2 * c] *= u2.x;
                PV[2 * c + 1] *= u2.y;
                if constexpr (EXT) {
                    if (ext.tol2 > 0.f) delta = fmaxf(delta, fmaxf(fabsf(lg2(u2.x)), fabsf(lg2(u2.y))));
                }
            }
            used = t + 1;
            if constexpr (EXT) {
                if (ext.tol2 > 0.f && delta <= ext.tol2) { stop = true; break; }
            }
        }
    }
#pragma unroll
    for (int i = 0; i < M; ++i) {
        const float rho = rcp(TH[i]);
#pragma unroll
        for (int c = 0; c < M2; ++c) {
            y[i][2 * c] = fminf(E2[i][c].x * rho, 1.f);
            y[i][2 * c + 1] = fminf(E2[i][c].y * rho, 1.f);
        }
    }
    if constexpr (EXT) {
        if (ext.potentials) {
            flush();
            float* uv = ext.potentials + 2 * M * b;
#pragma unroll
            for (int k = 0; k < M; ++k) {
                uv[k] = finite ? float(double(U[k]) * kLn2D) : __int_as_float(0x7fc00000);
                uv[M + k] = finite ? float(double(V[k]) * kLn2D) : __int_as_float(0x7fc00000);
            }
        }
        if (ext.iters_used) ext.iters_used[b] = finite ? used : 0;
    }
    return finite;
}

// Per-thread y0 space of dykstra_thread_kernel (floats; padded so that the
// threads' 16-byte accesses do not share banks).
template <int M>
__host__ __device__ constexpr int thread_y0_stride() { return M * M + 4; }

template <int M, typename T, bool EXT = false>
__global__ void __launch_bounds__(128, 4)
dykstra_thread_kernel(const typename T::storage* __restrict__ W, int64_t cols, int64_t n_blocks,
                      int N, float tau, int iters, float* __restrict__ plan, DykstraExt ext = {}) {
    extern __shared__ __align__(16) float thread_y0[];
    const int64_t b = int64_t(blockIdx.x) * blockDim.x + threadIdx.x;
    if (b >= n_blocks) return;
    const int64_t nbc = cols / M;
    const int64_t r0 = (b / nbc) * M, c0 = (b % nbc) * M;
    float S[M][M];
    const bool finite = dykstra_thread_solve<M, T, EXT>(W, cols, b, r0, c0, N, tau, iters, ext, S,
                                                        thread_y0 + threadIdx.x * thread_y0_stride<M>());
#pragma unroll
    for (int i = 0; i < M; ++i) {
        float* dst = plan + (r0 + i) * cols + c0;
#pragma unroll
        for (int v = 0; v < M / 4; ++v)
            reinterpret_cast<float4*>(dst)[v] =
                finite ? make_float4(S[i][4 * v], S[i][4 * v + 1], S[i][4 * v + 2], S[i][4 * v + 3])
                       : make_float4(__int_as_float(0x7fc00000), __int_as_float(0x7fc00000),
                                     __int_as_float(0x7fc00000), __int_as_float(0x7fc00000));
    }
}

// ---------------------------------------------------------------------------
// M = 16, 32, 64: a block is spread over M*M/32 threads, each holding a
// P x Q = 4 x 8 sub-tile.  Threads of one block: t = rg * CG + cg with
// cg in [0, CG = M/8) (lowest lane bits: the threads that share rows) and
// rg in [0, RG = M/4) (the threads that share columns).
//
// Row and column sums are formed by a shuffle reduce-scatter in which every
// thread keeps its registers in an order permuted by XOR with its own group
// index; with that order every level of the butterfly sends the upper half
// of the live registers to the partner and keeps the lower half, with no
// lane-dependent selects.  The matching all-gather returns the row and
// column potentials in the same permuted order.
// ---------------------------------------------------------------------------
template <int M>
struct TileCfg {
    static constexpr int P = 4, Q = 8;
    static constexpr int CG = M / Q;                 // threads sharing a row
    static constexpr int RG = M / P;                 // threads sharing a column
    static constexpr int TPB = CG * RG;              // threads per block
    static constexpr int BPW = TPB < 32 ? 32 / TPB : 1;   // blocks per warp
    static constexpr int RSR = CG < P ? CG : P;      // lanes in the row reduce-scatter
    static constexpr int ARR = CG / RSR;             // lanes in the row all-reduce after it
    static constexpr int RO = P / RSR;               // rows owned per thread
    static constexpr int CW = (RG < 32 / CG) ? RG : 32 / CG;   // column sharers inside a warp
    static constexpr int RSC = CW < Q ? CW : Q;      // lanes in the column reduce-scatter
    static constexpr int CO = Q / RSC;               // columns owned per thread
    static constexpr int WC = RG / CW;               // warps sharing a column
    static constexpr int THREADS = 128;              // CTA size
    static constexpr int BPC = THREADS / TPB;        // blocks per CTA
    static_assert(P * Q == 32, "sub-tile of 32 entries");
    static_assert(TPB <= THREADS, "block larger than a CTA");
    static_assert(CG * RSC == 32 || WC == 1, "cross-warp columns need full warps");
};

// Identity of a thread inside its block's tile, and the permuted local row /
// column that its register k / c holds.
template <int M>
struct TileThread {
    using C = TileCfg<M>;
    int tid, lane, warp, blk, t, cg, rg, gr, gc;
    __device__ __forceinline__ TileThread() {
        tid = threadIdx.x;
        lane = tid & 31;
        warp = tid >> 5;
        blk = tid / C::TPB;            // block slot within the CTA
        t = tid % C::TPB;              // thread within the block
        cg = t % C::CG;
        rg = t / C::CG;
        gr = cg % C::RSR;              // index in the row reduce-scatter group
        gc = rg % C::RSC;              // index in the column reduce-scatter group
    }
    __device__ __forceinline__ int lrow(int k) const { return ((k / C::RO) ^ gr) * C::RO + (k % C::RO); }
    __device__ __forceinline__ int lcol(int c) const { return ((c / C::CO) ^ gc) * C::CO + (c % C::CO); }
    __device__ __forceinline__ int row(int k) const { return C::P * rg + lrow(k); }   // row within the block
    __device__ __forceinline__ int col(int c) const { return C::Q * cg + lcol(c); }   // column within the block
};

// Where a block's W tile comes from.  With a tensor map (`map` non-null) the
// tile (rows r0.., columns c0..) is copied by TMA into `raw` (M*M elements,
// 128-byte aligned, shared memory) on the barrier `bar` and then widened to
// |W|; otherwise the block's threads read it from `W` (row stride `cols`)
// with 16-byte loads.
template <typename T>
struct TileSource {
    const CUtensorMap* map;
    typename T::storage* raw;
    uint64_t* bar;
    const typename T::storage* W;
    int64_t cols;
};

// Dykstra for one block spread over its TPB threads.  On return `out` holds the
// plan S = 2^min(y, 0) of this thread's sub-tile.  The tile (M x M floats in
// shared memory, row stride TS) holds the initial state y0 during the
// iterations; with RESTORE it holds the block's |W| again on return.
// Contains CTA-wide barriers: every thread of the CTA must call it.  Returns
// whether the block's W is finite (false too when its tile copy did not
// complete in time).
//
// The iteration is the log-space one (state y = x + log Q, base 2), kept in
// the form y = y0 + U_i + V_j: the accumulated row and column potentials U, V
// (fp64, in the threads that own the row or column after the reduce-scatters)
// are the whole state.  The clipped exponentials e = 2^min(y, 0) are not
// taken afresh every iteration: E = 2^y is carried from one iteration to the
// next by the same update in linear form, E <- E * 2^r_i * 2^c_j (the
// exponential of y += r_i + c_j, 2^r_i = N / R_i and 2^c_j = N / C_j).  The
// row factor is not applied entry by entry: E_ij = F_ij / th_i, the clip
// min(E, 1) = min(F, th_i) / th_i, and the row step replaces th_i by S_i / N
// (S_i = sum_j min(F_ij, th_i)), which is the same as multiplying row i of E
// by N / R_i; the column step multiplies F by N / C_j (hardware reciprocal),
// so one multiply per entry and iteration remains.  Every kAnchorEvery
// iterations log2 of the threshold and of the column factors' product are
// added to U and V, and E is re-anchored to 2^(y0 + U + V) (th = 1), so that
// an entry that underflowed for a while recovers and the rounding of the
// products never builds up.  The anchor is taken as the product
// (E0_ij * 2^U_i) * 2^V_j, E0 = 2^y0 computed once from an fp64 y0: y0 and
// U + V are each of size up to tau * log2(e) and cancel, so their fp32 sum
// would put an error of about |y0| * 2^-24 into every entry, which the
// iterations do not remove; in the product form each entry carries a few
// ulps, and the rounding of a potential is common to its row or column.

// EXT: warm start from / export to ext.potentials of block b, stop rule
// ext.tol2, iteration count to ext.iters_used.
template <int M, typename T, int TS = M, bool EXT = false, bool RESTORE = true>
__device__ __forceinline__ bool dykstra_tile_solve(const TileSource<T>& src, int64_t r0, int64_t c0, bool active,
                                                   int N, float tau, int iters, float* tile, float* colbuf,
                                                   const TileThread<M>& th, float (&out)[4][8],
                                                   const DykstraExt& ext = DykstraExt{}, int64_t b = 0) {
    using C = TileCfg<M>;
    constexpr int P = C::P, Q = C::Q, Q2 = Q / 2;
    float (&y)[P][Q] = out;                          // |W| of this thread's entries, then the plan
    const int lane = th.lane, warp = th.warp;

    bool loaded = true;
    // |W| of the block into the tile: 16-byte loads from W, or the TMA-staged
    // raw tile widened (zeros for an inactive block or a copy that did not land)
    auto fill_abs = [&]() {
        if (!src.map) {
            constexpr int V = T::kVec;
            constexpr int CPR = M / V;                 // 16-byte chunks per tile row
            for (int q = th.t; q < M * CPR; q += C::TPB) {
                const int i = q / CPR, v = q % CPR;
                float tmp[V];
                if (active) T::load16(src.W + (r0 + i) * src.cols + c0 + v * V, tmp);
                else {
#pragma unroll
                    for (int u = 0; u < V; ++u) tmp[u] = 0.f;
                }
#pragma unroll
                for (int u = 0; u < V; ++u) tile[i * TS + v * V + u] = tmp[u];
            }
        } else {
            constexpr int V = 16 / int(sizeof(typename T::storage));   // elements per 16-byte chunk
            constexpr int CPR = M / V;                                  // chunks per tile row
            for (int q = th.t; q < M * CPR; q += C::TPB) {
                const int i = q / CPR, v = q % CPR;
                float tmp[V];
                if (active && loaded) T::smem16(src.raw + i * M + v * V, tmp);
                else {
#pragma unroll
                    for (int u = 0; u < V; ++u) tmp[u] = 0.f;
                }
#pragma unroll
                for (int u = 0; u < V; ++u) tile[i * TS + v * V + u] = tmp[u];
            }
        }
    };
    auto block_sync = [&]() {
        if constexpr (C::TPB <= 32) __syncwarp(); else __syncthreads();
    };

    if (src.map) {
        // ---- stage the block's W tile in shared memory by TMA
        typename T::storage* raw = src.raw;
        uint64_t* bar = src.bar;
        // a staging address off the 128-byte grid is never handed to the copy
        // engine: the block is reported as failed instead
        const bool staged = (smem_u32(raw) & 127u) == 0 && (smem_u32(bar) & 7u) == 0;
        if (active && staged && th.t == 0) {
            mbar_init(bar, 1);
            mbar_init_fence();
        }
        block_sync();                                  // barrier initialised before any poll
        if (active && staged && th.t == 0) {
            mbar_arrive_expect_tx(bar, unsigned(M * M * sizeof(typename T::storage)));
            tma_load_2d(raw, src.map, int(c0), int(r0), bar);
        }
        if (active) {
            loaded = staged && mbar_wait_bounded(bar, 0);
            // a copy that did not land in time may still arrive: wait once more before the space is reused
            if (staged && !loaded) mbar_wait_bounded(bar, 0);
        }
    }
    fill_abs();
    __syncthreads();

    float m = 0.f;
    bool finite = loaded;
#pragma unroll
    for (int k = 0; k < P; ++k)
#pragma unroll
        for (int c = 0; c < Q; ++c) {
            const float a = tile[th.row(k) * TS + th.col(c)];
            y[k][c] = a;
            finite = finite && (a <= 3.402823466e38f);
            m = fmaxf(m, a);
        }
    // block max and finiteness over the block's threads
    if constexpr (C::TPB <= 32) {
#pragma unroll
        for (int s = 1; s < C::TPB; s <<= 1) {
            m = fmaxf(m, __shfl_xor_sync(kFullMask, m, s));
            finite = __shfl_xor_sync(kFullMask, int(finite), s) && finite;
        }
    } else {
#pragma unroll
        for (int s = 1; s < 32; s <<= 1) {
            m = fmaxf(m, __shfl_xor_sync(kFullMask, m, s));
            finite = __shfl_xor_sync(kFullMask, int(finite), s) && finite;
        }
        __shared__ float red_m[4];
        __shared__ int red_f[4];
        if (lane == 0) { red_m[warp] = m; red_f[warp] = finite; }
        __syncthreads();
        m = fmaxf(fmaxf(red_m[0], red_m[1]), fmaxf(red_m[2], red_m[3]));
        finite = red_f[0] && red_f[1] && red_f[2] && red_f[3];
    }
    // y0 = (x0 - tau) log2 e with x0 = tau |W| / max|W|, taken in fp64 (as
    // the oracle's x0); kept in the tile for the anchor points as E0 = 2^y0:
    // column pair (k, c) of thread t at float2 slot
    // (k * Q/2 + c) * TPB + t (consecutive threads, consecutive slots)
    block_sync();                                    // every thread has read its |W|
    const double tau2d = double(tau) * kLog2eD;
    const double inv_m = m > 0.f ? 1.0 / double(m) : 0.0;
    float2* y0t = reinterpret_cast<float2*>(tile) + th.t;
    static_assert(P * Q * C::TPB <= M * TS, "y0 fits the tile");
#pragma unroll
    for (int k = 0; k < P; ++k)
#pragma unroll
        for (int c = 0; c < Q2; ++c) {
            const double y0a = fma(tau2d, double(y[k][2 * c]) * inv_m, -tau2d);
            const double y0b = fma(tau2d, double(y[k][2 * c + 1]) * inv_m, -tau2d);
            y0t[(k * Q2 + c) * C::TPB] = make_float2(exp2_wide(y0a), exp2_wide(y0b));
        }
    const float fN = float(N);

    // potentials of the owned rows (register k < RO holds row(k)) and columns
    // (c < CO holds col(c)) as of the last anchor point (EXT may start them
    // from ext.potentials, nats).  Since then: each row's scaling lives in
    // its clip threshold thr[k] (E_ij = F_ij / th_i, so min(E, 1) is
    // min(F, th_i) / th_i and the row step sets th_i = S_i / N with
    // S_i = sum_j min(F_ij, th_i)), which makes the row's potential step
    // log2(th_old / th_new); the column scalings multiply F, and the owners
    // keep their products.  Both are added to U and V at the next anchor point.
    const float invN = 1.f / float(N);
    double ua[C::RO], va[C::CO];
    float thr[P], pv[C::CO];
#pragma unroll
    for (int k = 0; k < P; ++k) thr[k] = 1.f;
#pragma unroll
    for (int lo = 0; lo < C::CO; ++lo) pv[lo] = 1.f;
    auto flush = [&]() {
#pragma unroll
        for (int lo = 0; lo < C::RO; ++lo) ua[lo] -= double(lg2(thr[lo]));
#pragma unroll
        for (int lo = 0; lo < C::CO; ++lo) { va[lo] += double(lg2(pv[lo])); pv[lo] = 1.f; }
    };
    {
        const float* uv = nullptr;
        if constexpr (EXT) uv = (ext.warm && active) ? ext.potentials + 2 * M * b : nullptr;
#pragma unroll
        for (int lo = 0; lo < C::RO; ++lo) ua[lo] = uv ? double(uv[th.row(lo)]) * kLog2eD : 0.0;
#pragma unroll
        for (int lo = 0; lo < C::CO; ++lo) va[lo] = uv ? double(uv[M + th.col(lo)]) * kLog2eD : 0.0;
    }
    // F = E = 2^(y0 + U_i + V_j) = (E0_ij * 2^U_i) * 2^V_j over this thread's
    // entries and th = 1, the factors taken from the fp64 potentials by their
    // owners and all-gathered into the permuted register order; the
    // potentials' large magnitudes (up to about tau2) never meet in an fp32
    // sum, so each entry carries only a few ulps of rounding, and an error in
    // a factor is common to a whole row or column.
    float2 F2[P][Q2];                                // column pairs packed
    auto anchor = [&]() {
        flush();
#pragma unroll
        for (int k = 0; k < P; ++k) thr[k] = 1.f;
        float U[P], V[Q];                            // 2^U_i, 2^V_j
#pragma unroll
        for (int lo = 0; lo < C::RO; ++lo) U[lo] = exp2_wide(ua[lo]);
#pragma unroll
        for (int s = 1; s < C::RSR; s <<= 1)
#pragma unroll
            for (int hi = 0; hi < s; ++hi)
#pragma unroll
                for (int lo = 0; lo < C::RO; ++lo)
                    U[(hi + s) * C::RO + lo] = __shfl_xor_sync(kFullMask, U[hi * C::RO + lo], s);
#pragma unroll
        for (int lo = 0; lo < C::CO; ++lo) V[lo] = exp2_wide(va[lo]);
#pragma unroll
        for (int s = 1; s < C::RSC; s <<= 1)
#pragma unroll
            for (int hi = 0; hi < s; ++hi)
#pragma unroll
                for (int lo = 0; lo < C::CO; ++lo)
                    V[(hi + s) * C::CO + lo] = __shfl_xor_sync(kFullMask, V[hi * C::CO + lo], s * C::CG);
#pragma unroll
        for (int k = 0; k < P; ++k)
#pragma unroll
            for (int c = 0; c < Q2; ++c)
                F2[k][c] = mul2(mul2(lds_keep(y0t + (k * Q2 + c) * C::TPB), make_float2(U[k], U[k])),
                                make_float2(V[2 * c], V[2 * c + 1]));
    };
    bool done = !finite;                             // EXT: this block has stopped
    int used = 0;

    // Blocks of one warp (M = 16) may differ in finiteness; all lanes run the
    // loop so that the shuffles stay converged, and a non-finite block's
    // result is discarded by the caller.
    const bool run = (C::TPB <= 32) ? (__any_sync(kFullMask, finite) != 0) : finite;
    bool stop = !run;
#pragma unroll 1
    for (int it0 = 0; it0 < iters && !stop; it0 += kAnchorEvery) {
        anchor();                                    // one call site (see dykstra_thread_solve)
        const int it1 = min(iters, it0 + kAnchorEvery);
#pragma unroll 1
        for (int it = it0; it < it1; ++it) {
            float2 e2[P][Q2];
            float rs[P];
#pragma unroll
            for (int k = 0; k < P; ++k) {
#pragma unroll
                for (int c = 0; c < Q2; ++c) e2[k][c] = make_float2(fminf(F2[k][c].x, thr[k]), fminf(F2[k][c].y, thr[k]));
                const float2 acc = add2(add2(e2[k][0], e2[k][1]), add2(e2[k][2], e2[k][3]));
                rs[k] = acc.x + acc.y;
            }
            // row reduce-scatter over RSR lanes, then all-reduce over ARR
#pragma unroll
            for (int s = C::RSR / 2; s >= 1; s >>= 1)
#pragma unroll
                for (int hi = 0; hi < s; ++hi)
#pragma unroll
                    for (int lo = 0; lo < C::RO; ++lo)
                        rs[hi * C::RO + lo] += __shfl_xor_sync(kFullMask, rs[(hi + s) * C::RO + lo], s);
#pragma unroll
            for (int s = C::RSR; s < C::CG; s <<= 1)
#pragma unroll
                for (int lo = 0; lo < C::RO; ++lo)
                    rs[lo] += __shfl_xor_sync(kFullMask, rs[lo], s);
            // owned rows: column-step weight N / S (= e's scale N / R over th) and
            // the next threshold S / N
            float wv[P], tn[P];
#pragma unroll
            for (int lo = 0; lo < C::RO; ++lo) {
                wv[lo] = fN * rcp(rs[lo]);
                tn[lo] = rs[lo] * invN;
            }
            // all-gather of the scales back into the permuted register order
#pragma unroll
            for (int s = 1; s < C::RSR; s <<= 1)
#pragma unroll
                for (int hi = 0; hi < s; ++hi)
#pragma unroll
                    for (int lo = 0; lo < C::RO; ++lo)
                    {
                        wv[(hi + s) * C::RO + lo] = __shfl_xor_sync(kFullMask, wv[hi * C::RO + lo], s);
                        tn[(hi + s) * C::RO + lo] = __shfl_xor_sync(kFullMask, tn[hi * C::RO + lo], s);
                    }
            // column partial sums of e * w
            float cs[Q];
#pragma unroll
            for (int c = 0; c < Q2; ++c) {
                float2 acc = mul2(e2[0][c], make_float2(wv[0], wv[0]));
#pragma unroll
                for (int k = 1; k < P; ++k) acc = fma2(e2[k][c], make_float2(wv[k], wv[k]), acc);
                cs[2 * c] = acc.x;
                cs[2 * c + 1] = acc.y;
            }
#pragma unroll
            for (int s = C::RSC / 2; s >= 1; s >>= 1)
#pragma unroll
                for (int hi = 0; hi < s; ++hi)
#pragma unroll
                    for (int lo = 0; lo < C::CO; ++lo)
                        cs[hi * C::CO + lo] += __shfl_xor_sync(kFullMask, cs[(hi + s) * C::CO + lo], s * C::CG);
            if constexpr (C::WC > 1) {
                float* buf = colbuf + (it & 1) * (4 * 32 * C::CO);
#pragma unroll
                for (int lo = 0; lo < C::CO; ++lo) buf[(warp * 32 + lane) * C::CO + lo] = cs[lo];
                __syncthreads();
#pragma unroll
                for (int lo = 0; lo < C::CO; ++lo) {
                    float acc = buf[(0 * 32 + lane) * C::CO + lo];
#pragma unroll
                    for (int w2 = 1; w2 < C::WC; ++w2) acc += buf[(w2 * 32 + lane) * C::CO + lo];
                    cs[lo] = acc;
                }
            }
            // owned columns: scale u = N / C = 2^c
            float uv[Q];
#pragma unroll
            for (int lo = 0; lo < C::CO; ++lo) uv[lo] = fN * rcp(cs[lo]);
#pragma unroll
            for (int s = 1; s < C::RSC; s <<= 1)
#pragma unroll
                for (int hi = 0; hi < s; ++hi)
#pragma unroll
                    for (int lo = 0; lo < C::CO; ++lo)
                        uv[(hi + s) * C::CO + lo] = __shfl_xor_sync(kFullMask, uv[hi * C::CO + lo], s * C::CG);
            float delta = 0.f;                       // EXT: largest |r_i|, |c_j| of the owned ones
            if constexpr (EXT) {
                if (ext.tol2 > 0.f) {
#pragma unroll
                    for (int lo = 0; lo < C::RO; ++lo) delta = fmaxf(delta, fabsf(lg2(thr[lo]) - lg2(tn[lo])));
#pragma unroll
                    for (int lo = 0; lo < C::CO; ++lo) delta = fmaxf(delta, fabsf(lg2(uv[lo])));
                }
                // a stopped block of a shared warp (M = 16) keeps its state
                if (done) {
#pragma unroll
                    for (int k = 0; k < P; ++k) tn[k] = thr[k];
#pragma unroll
                    for (int c = 0; c < Q; ++c) uv[c] = 1.f;
                }
            }
            // y += r_i + c_j: the row part through the thresholds, the column part on F
#pragma unroll
            for (int k = 0; k < P; ++k) {
                thr[k] = tn[k];
#pragma unroll
                for (int c = 0; c < Q2; ++c) F2[k][c] = mul2(F2[k][c], make_float2(uv[2 * c], uv[2 * c + 1]));
            }
#pragma unroll
            for (int lo = 0; lo < C::CO; ++lo) pv[lo] *= uv[lo];
            if constexpr (EXT) {
                if (!done) used = it + 1;
                if (ext.tol2 > 0.f) {
                    const bool small = delta <= ext.tol2;
                    bool all_small;
                    if constexpr (C::TPB < 32) {
                        const unsigned bal = __ballot_sync(kFullMask, small);
                        const unsigned gm = ((1u << C::TPB) - 1u) << ((lane / C::TPB) * C::TPB);
                        all_small = (bal & gm) == gm;
                    } else if constexpr (C::TPB == 32) {
                        all_small = __all_sync(kFullMask, small);
                    } else {
                        all_small = __syncthreads_and(small);
                    }
                    done = done || all_small;
                    stop = (C::TPB <= 32) ? (__all_sync(kFullMask, done) != 0) : done;
                    if (stop) break;
                }
            }
        }
    }
#pragma unroll
    for (int k = 0; k < P; ++k)
#pragma unroll
        for (int c = 0; c < Q2; ++c) {
            const float rho = rcp(thr[k]);
            y[k][2 * c] = fminf(F2[k][c].x * rho, 1.f);
            y[k][2 * c + 1] = fminf(F2[k][c].y * rho, 1.f);
        }
    if constexpr (EXT) {
        flush();
        if (active) {
            if (ext.potentials) {
                float* uv = ext.potentials + 2 * M * b;
                const float nan = __int_as_float(0x7fc00000);
                if (th.cg < C::RSR)
#pragma unroll
                    for (int lo = 0; lo < C::RO; ++lo) uv[th.row(lo)] = finite ? float(ua[lo] * kLn2D) : nan;
                if (th.rg < C::RSC)
#pragma unroll
                    for (int lo = 0; lo < C::CO; ++lo) uv[M + th.col(lo)] = finite ? float(va[lo] * kLn2D) : nan;
            }
            if (ext.iters_used && th.t == 0) ext.iters_used[b] = finite ? used : 0;
        }
    }
    if constexpr (RESTORE) {
        block_sync();                                // every thread has read its y0
        fill_abs();
        block_sync();
    }
    return finite;
}

// Shared memory of dykstra_tile_kernel: TMA staging of the raw W tiles, the
// |W| tiles, the cross-warp column buffer, one barrier per block slot.
template <int M, typename T>
struct PlanSmem {
    using C = TileCfg<M>;
    static constexpr size_t raw_bytes = size_t(C::BPC) * M * M * sizeof(typename T::storage);
    static constexpr size_t tile_off = (raw_bytes + 127) / 128 * 128;
    static constexpr size_t colbuf_off = tile_off + sizeof(float) * C::BPC * M * M;
    static constexpr size_t bar_off = colbuf_off + sizeof(float) * (C::WC > 1 ? 2 * 4 * 32 * C::CO : 0);
    static constexpr size_t bytes = bar_off + sizeof(uint64_t) * C::BPC;
};

template <int M, typename T, bool EXT = false>
__global__ void __launch_bounds__(128, 5)
dykstra_tile_kernel(const __grid_constant__ CUtensorMap wmap, int64_t cols, int64_t n_blocks,
                    int N, float tau, int iters, float* __restrict__ plan, DykstraExt ext = {}) {
    using C = TileCfg<M>;
    using L = PlanSmem<M, T>;
    extern __shared__ __align__(128) unsigned char plan_raw[];
    const TileThread<M> th;
    auto* raw = reinterpret_cast<typename T::storage*>(plan_raw) + th.blk * M * M;
    float* tile = reinterpret_cast<float*>(plan_raw + L::tile_off) + th.blk * M * M;
    float* colbuf = reinterpret_cast<float*>(plan_raw + L::colbuf_off);   // [2][warps][32][CO]
    uint64_t* bar = reinterpret_cast<uint64_t*>(plan_raw + L::bar_off) + th.blk;
    const int64_t b = int64_t(blockIdx.x) * C::BPC + th.blk;
    const bool active = b < n_blocks;
    const int64_t nbc = cols / M;
    const int64_t r0 = active ? (b / nbc) * M : 0, c0 = active ? (b % nbc) * M : 0;

    float S[C::P][C::Q];                      // plan of this thread's entries
    const TileSource<T> src{&wmap, raw, bar, nullptr, 0};
    const bool finite = dykstra_tile_solve<M, T, M, EXT, false>(src, r0, c0, active, N, tau, iters, tile, colbuf, th, S, ext,
                                                         b);

    // ---- plan via the smem tile, then 16-byte coalesced stores
    __syncthreads();
#pragma unroll
    for (int k = 0; k < C::P; ++k)
#pragma unroll
        for (int c = 0; c < C::Q; ++c)
            tile[th.row(k) * M + th.col(c)] = finite ? S[k][c] : __int_as_float(0x7fc00000);
    __syncthreads();
    if (active) {
        constexpr int CPR = M / 4;
        for (int q = th.t; q < M * CPR; q += C::TPB) {
            const int i = q / CPR, v = q % CPR;
            const float4 val = *reinterpret_cast<const float4*>(tile + i * M + 4 * v);
            *reinterpret_cast<float4*>(plan + (r0 + i) * cols + c0 + 4 * v) = val;
        }
    }
}

template <int M, typename T>
constexpr size_t dykstra_tile_smem() { return PlanSmem<M, T>::bytes; }

}  // namespace tsenor
