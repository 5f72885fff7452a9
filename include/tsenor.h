/*
 * tsenor.h -- C ABI of the B200 transposable N:M mask solver.
 *
 * The method is TSENOR, as described in "Pith review of TSENOR:
 * Highly-Efficient Algorithm for Finding Transposable N:M Sparse Masks"
 * (pith.science/paper/2505.23949):
 *   - the problem ("Core claim"): split W into MxM blocks and, per block, find
 *     a 0/1 mask with exactly N ones in every row and every column that
 *     maximises the kept sum of |W|;
 *   - the solver ("What carries the argument"): entropy-regularised
 *     capacitated transport relaxation solved by Dykstra's alternating KL
 *     projections in log space (row normalisation, column normalisation,
 *     clip at 1 with a correction term), then rounding by a descending sort
 *     with greedy row/column budgets, a feasibility repair and the
 *     2-in/1-out swap local search;
 *   - the free parameters ("Assumptions & free parameters"): tau, the
 *     iteration count T and the local-search length L.
 * The review prints no interface or code; this ABI is this library's own.
 *
 * Common conventions for every entry point:
 *  - Pointers to W, the plan, the mask and the objective are DEVICE pointers
 *    owned by the caller; the library keeps none of them after the call.
 *    W and the plan must be 16-byte aligned; the mask 8-byte aligned.
 *  - W is row-major, rows x cols, of the element type `dtype`; only |W| is
 *    used, so any matrix of importance scores (for example |W_ij| times the
 *    norm of input feature j, as layer-wise pruning methods use) can be
 *    passed in its place.  rows and cols must be multiples of M (the review leaves other
 *    shapes open, "Assumptions & free parameters"); rows == 0 or cols == 0
 *    is a valid empty call that does nothing.
 *  - Supported M: 4, 8, 16, 32, 64.  1 <= N <= M.  0 < tau <= TSENOR_MAX_TAU,
 *    iters >= 1, sweeps >= 0.
 *  - The kernel of block b is x0_ij = tau * |W_ij| / max(|W| over b)
 *    (x0 = 0 for an all-zero block); one iteration is a row step, a column
 *    step and a clip.
 *  - Mask layout: row-major, words_per_row = ceil(cols / 32) uint32 words
 *    per row; bit k of word w of row r is column 32*w + k (least significant
 *    bit first); bits past the last column are written as 0.
 *  - All calls are asynchronous and ordered on `stream` (a cudaStream_t;
 *    NULL is the legacy default stream).  Argument errors are detected on
 *    the host before anything is enqueued and return at once.
 *  - A block whose W holds NaN or Inf gets an all-zero mask and bumps the
 *    device failure counter read by tsenor_error_count; the other blocks of
 *    the call are unaffected.
 *  - The library is not re-entrant across host threads for the same device
 *    failure counter: concurrent calls add into one counter.
 */
#ifndef TSENOR_H
#define TSENOR_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

struct CUstream_st;
typedef struct CUstream_st* tsenor_stream_t;   /* same type as cudaStream_t */

typedef enum { TSENOR_F32 = 0, TSENOR_BF16 = 1 } tsenor_dtype;

/*
 * Largest tau accepted (larger values return TSENOR_ERR_ARG).  The kernels
 * carry the exponentials of the Dykstra state in fp32, and a block's kernel
 * exp(tau * |W| / max|W|) spans a factor 2^(tau * log2 e) between its
 * smallest and largest entry; at tau = 80 that is 2^115, inside the normal
 * fp32 range with room for the potentials.  The review's default
 * temperature, 0.005 * max|W| ("Assumptions & free parameters"), corresponds
 * to tau = 200 in this convention and is outside it.
 */
#define TSENOR_MAX_TAU 80.0f

typedef enum {
    TSENOR_OK = 0,
    TSENOR_ERR_ARG = -1,             /* null pointer, bad dtype, N/tau/iters/sweeps out of range (tau: see TSENOR_MAX_TAU), misaligned pointer */
    TSENOR_ERR_SHAPE = -2,           /* rows or cols negative or not a multiple of M */
    TSENOR_ERR_UNSUPPORTED_M = -3,   /* M not in {4, 8, 16, 32, 64} */
    TSENOR_ERR_CUDA = -4,            /* a CUDA runtime call failed; see tsenor_last_error() */
    TSENOR_ERR_DEVICE = -5,          /* tsenor_error_count: blocks failed on the device (count in *count_out) */
    TSENOR_ERR_TOO_LARGE = -6        /* tsenor_mask_noalloc: rows*cols above TSENOR_NOALLOC_MAX_PARAMS */
} tsenor_status;

/*
 * Transposable N:M mask of W (the whole hot path: Dykstra plan, sort, greedy,
 * repair, local search, bit packing).
 *   mask_out: rows x words_per_row uint32, written completely.
 *   sweeps:   local-search sweeps L; one sweep visits every anchor row once.
 * One fused kernel per call (every M), no workspace: the plan never leaves
 * the chip.
 */
tsenor_status tsenor_mask(const void* W, tsenor_dtype dtype, int64_t rows, int64_t cols,
                          int N, int M, float tau, int iters, int sweeps,
                          uint32_t* mask_out, tsenor_stream_t stream);

/*
 * The fractional transport plan only: S = exp(x) after the clip of the last
 * Dykstra iteration ("What carries the argument"), fp32, rows x cols,
 * row-major, every block at its place in W.  0 <= S <= 1.  A block with
 * non-finite W gets NaN.
 */
tsenor_status tsenor_plan(const void* W, tsenor_dtype dtype, int64_t rows, int64_t cols,
                          int N, int M, float tau, int iters, float* plan_out,
                          tsenor_stream_t stream);

/*
 * The rounding only, from a given plan (keys): per block, sort entries by
 * (plan desc, |W| desc, flat index i*M+j asc), greedy with row/column
 * budgets N, feasibility repair by 2-in/1-out moves, then `sweeps` sweeps of
 * the swap local search, then bit packing into mask_out.
 * plan: rows x cols fp32 (non-negative; a block holding NaN fails).
 */
tsenor_status tsenor_round(const float* plan, const void* W, tsenor_dtype dtype,
                           int64_t rows, int64_t cols, int N, int M, int sweeps,
                           uint32_t* mask_out, tsenor_stream_t stream);

/*
 * Kept mass per block: out[b] = sum over block b of |W_ij| * mask_ij in fp64,
 * or NaN when a row or a column of block b does not hold exactly N ones.
 * Blocks are numbered row-major over the block grid: b = (r/M)*(cols/M) + c/M.
 *   out: (rows/M)*(cols/M) doubles (device).
 */
tsenor_status tsenor_objective(const void* W, tsenor_dtype dtype, int64_t rows, int64_t cols,
                               const uint32_t* mask, int N, int M, double* out,
                               tsenor_stream_t stream);

/*
 * Synchronises `stream`, then returns in *count_out the number of blocks that
 * failed on this device (non-finite input, or a rounding step that found no
 * move) since the previous call, and resets the counter.  Returns TSENOR_OK
 * when that number is 0 and TSENOR_ERR_DEVICE when it is not (the count is
 * written in both cases); TSENOR_ERR_ARG for a null count_out, TSENOR_ERR_CUDA
 * when the copy or the synchronisation fails.
 */
tsenor_status tsenor_error_count(tsenor_stream_t stream, int64_t* count_out);

/*
 * tsenor_mask with the monotonicity safeguard of the review's "Assumptions &
 * free parameters" (Assumption 1 of Theorem 1; referee comment 2): inside an
 * outer loop (an ADMM mask update) the new mask must not lower the block
 * objective below the previous mask's.  Per block: the new mask is computed
 * as by tsenor_mask; when prev_mask's block is a valid N:M block whose kept
 * sum of |W| is strictly larger, prev_mask's block is written instead.  Both
 * sums are taken in fp64 in row-major order within the block.
 *   prev_mask: rows x words_per_row uint32 (device), same layout as mask_out;
 *              it may not alias mask_out.
 *   kept_out:  optional device counter (may be NULL); the number of blocks that
 *              kept prev_mask is ADDED to it.
 */
tsenor_status tsenor_mask_safeguard(const void* W, tsenor_dtype dtype, int64_t rows, int64_t cols,
                                    int N, int M, float tau, int iters, int sweeps,
                                    const uint32_t* prev_mask, uint32_t* mask_out,
                                    unsigned long long* kept_out, tsenor_stream_t stream);

/*
 * tsenor_mask for shapes that are not multiples of M.  The review leaves
 * such shapes open ("Assumptions & free parameters": the partition into MxM
 * blocks "with no remainder or with padding"); this entry point takes the
 * padding reading: W is extended with zeros to ceil(rows/M)*M x
 * ceil(cols/M)*M, every block of the extended matrix is solved, and mask_out
 * receives the rows x cols part (words_per_row = ceil(cols/32), bits past
 * cols are 0).  In a full block every row and column keeps exactly N entries;
 * in an edge block a real row or column keeps at most N.
 *   W: rows x cols, row-major, no alignment requirement.
 * Uses stream-ordered workspaces (cudaMallocAsync / cudaFreeAsync) for the
 * padded copy of W and its mask.
 */
tsenor_status tsenor_mask_padded(const void* W, tsenor_dtype dtype, int64_t rows, int64_t cols,
                                 int N, int M, float tau, int iters, int sweeps,
                                 uint32_t* mask_out, tsenor_stream_t stream);

/*
 * tsenor_mask with warm start and adaptive stopping of the Dykstra loop.
 *
 * The review fixes the iteration count T and gives no convergence test
 * ("Assumptions & free parameters"); inside an outer pruning loop the same
 * layer is solved again and again for a slowly changing W.  This entry point
 * lets such calls resume from the previous solution and stop each block once
 * it has converged.  It rests on one identity: the row and column steps add
 * potentials r_i = ln N - LSE_j(x_ij) and c_j = ln N - LSE_i(x_ij) to x, and
 * the clip only moves an amount between x and its correction term, so after
 * every iteration
 *     x_ij + logQ_ij = (x0_ij - tau) + U_i + V_j,  x = min(that, 0),
 * with U, V the potentials accumulated so far.  The 2M numbers (U, V) of a
 * block are its whole Dykstra state.
 *   potentials: (rows/M)*(cols/M) blocks x 2M fp32 (device), block b (row-major
 *               over the block grid) at offset 2M*b: U_0..U_{M-1}, then
 *               V_0..V_{M-1}, natural-log units.  warm != 0: read as the
 *               starting state.  warm == 0: the start is U = V = 0 and the
 *               array is only written (may be NULL then).  When non-NULL it is
 *               overwritten with the final potentials (NaN for a block with
 *               non-finite W).  The same array may be passed back on the next
 *               call.
 *   tol:        >= 0 and finite.  tol > 0: a block stops after the first
 *               iteration whose potentials all satisfy |r_i| <= tol and
 *               |c_j| <= tol (natural-log units; at most `iters`
 *               iterations).  tol == 0: every block runs exactly `iters`.
 *   iters_used: optional (rows/M)*(cols/M) int32 (device, may be NULL): the
 *               iterations each block ran (0 for a non-finite block).
 * With warm == 0 and tol == 0 the mask equals tsenor_mask's bit for bit.
 * The stop decision is taken in fp32 on log2-scaled potentials, so a block
 * whose largest step lies within about 1e-6 of tol may stop one iteration
 * earlier or later than an exact evaluation would.
 * Workspace as tsenor_mask.  The review has no counterpart of this call.
 */
tsenor_status tsenor_mask_warm(const void* W, tsenor_dtype dtype, int64_t rows, int64_t cols,
                               int N, int M, float tau, int iters, int sweeps, float tol, int warm,
                               float* potentials, int32_t* iters_used, uint32_t* mask_out,
                               tsenor_stream_t stream);

/*
 * The plan of tsenor_mask_warm (same state, stop rule and outputs), written
 * as tsenor_plan writes it.  Test hook and building block.
 */
tsenor_status tsenor_plan_warm(const void* W, tsenor_dtype dtype, int64_t rows, int64_t cols,
                               int N, int M, float tau, int iters, float tol, int warm,
                               float* potentials, int32_t* iters_used, float* plan_out,
                               tsenor_stream_t stream);

/*
 * tsenor_mask on an importance-score matrix instead of weights.  Layer-wise
 * pruning methods hand the solver scores rather than |W| (the review names
 * Wanda, SparseGPT and ALPS: "Core claim", "What carries the argument"), for
 * example |W_ij| times the norm of input feature j.
 *   scores: rows x cols fp32 (device, 16-byte aligned); the magnitude of each
 *           score is used, so non-negative scores are taken as they are.
 * Same result as tsenor_mask(scores, TSENOR_F32, ...), same errors.
 */
tsenor_status tsenor_mask_scores(const float* scores, int64_t rows, int64_t cols, int N, int M, float tau,
                                 int iters, int sweeps, uint32_t* mask_out, tsenor_stream_t stream);

/*
 * tsenor_mask for W and the mask in HOST memory, with the transfers
 * overlapped with the solve: W is cut into row chunks (multiples of M rows);
 * chunk k+1 is copied to the device while chunk k is solved, and each
 * chunk's mask is copied back as soon as it is ready.  Results are those of
 * tsenor_mask on the whole matrix (blocks are independent).
 *   W_host:    rows x cols, row-major, host memory; page-locked memory
 *              (cudaHostAlloc / cudaHostRegister) lets the copies overlap,
 *              pageable memory works but serialises them.
 *   mask_host: rows x words_per_row uint32, host memory (page-locked for
 *              overlap); written completely.
 *   stream:    every copy and kernel is ordered after the work already on
 *              `stream`, and `stream` waits for all of them before its later
 *              work (the library uses two internal streams in between).  The
 *              host buffers must stay valid until then.
 * Uses stream-ordered device workspaces for two W chunks and two mask chunks
 * (cudaMallocAsync / cudaFreeAsync).  The two internal streams and their
 * events are created on a host thread's first call on a device (and context)
 * and reused by that thread's later calls (whose copies therefore queue
 * behind the earlier calls' copies); they are never destroyed (they go with
 * the context).  Errors as tsenor_mask; TSENOR_ERR_ARG
 * also for a null host pointer.  The review has no counterpart of this call.
 */
tsenor_status tsenor_mask_host(const void* W_host, tsenor_dtype dtype, int64_t rows, int64_t cols, int N, int M,
                               float tau, int iters, int sweeps, uint32_t* mask_host, tsenor_stream_t stream);

/* Static description of a status code. */
const char* tsenor_status_string(int status);

/* Message of the last TSENOR_ERR_CUDA on the calling host thread ("" if none). */
const char* tsenor_last_error(void);

/*
 * tsenor_mask_noalloc -- the two-kernel plan + round path with its plan in
 * a fixed array inside the library, for callers that cannot allocate.
 *
 * The TSENOR review has no counterpart of this entry point.  Running the
 * plan and the rounding as two kernels (tsenor_plan, then tsenor_round) needs
 * a rows x cols fp32 plan buffer between them, and some callers cannot
 * allocate one at call time:
 *  - processes whose device memory is already reserved by another allocator
 *    (for example a framework's caching allocator holding most of the GPU),
 *    where a fresh cudaMalloc can fail with out-of-memory although the
 *    caller still has free space in its own pool;
 *  - services that run under a fixed device-memory budget and must not grow
 *    their footprint, or wait on an allocation, while they are serving.
 * This entry point runs those two kernels with the plan in a file-scope
 * device array of TSENOR_NOALLOC_MAX_PARAMS floats (64 MiB).  That array
 * exists on every GPU that loads the library and stays allocated until the
 * process exits.  The call itself allocates nothing: no cudaMalloc,
 * cudaMallocAsync, cudaFree or allocating library routine.
 *
 * Arguments, results and error behaviour are those of tsenor_mask, and the
 * masks are equal bit for bit: tsenor_mask is one fused kernel that builds
 * the same keys on chip (and allocates nothing either), so it is the faster
 * call; this one takes the plan through device memory and back.
 *
 *  - rows * cols must not exceed TSENOR_NOALLOC_MAX_PARAMS; larger calls
 *    return TSENOR_ERR_TOO_LARGE before anything is enqueued.
 *  - The first call on a device looks up the array's device address on that
 *    device (cudaGetSymbolAddress, with the device current) and keeps it for
 *    later calls; it is looked up again when the device's current context
 *    has changed (after a cudaDeviceReset, for example).  Make the first call
 *    on each device before any stream capture.
 *  - Every call on a device shares the one array, and the array keeps the
 *    last call's contents.  Nothing in it needs to start at zero: each call
 *    writes the whole plan region it later reads.  Calls whose work overlaps
 *    on the GPU (different streams without ordering between them, or several
 *    host threads) race on the array and corrupt each other's masks; order
 *    them on one stream or with events.
 */
#define TSENOR_NOALLOC_MAX_PARAMS (16LL * 1024 * 1024)
tsenor_status tsenor_mask_noalloc(const void* W, tsenor_dtype dtype, int64_t rows, int64_t cols,
                                  int N, int M, float tau, int iters, int sweeps,
                                  uint32_t* mask_out, tsenor_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* TSENOR_H */
