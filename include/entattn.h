/*
 * entattn.h -- C ABI of the B200 fused alpha-entmax attention library
 * (libentattn.so).  Forward and backward of
 *
 *     s = Q K^T / sqrt(d),   P = alpha-entmax(s) row-wise,   O = P V,
 *
 * with alpha-entmax p_j = [(alpha-1) s_j - tau]_+^(1/(alpha-1)), tau such that
 * sum_j p_j = 1 (support strict: p_j > 0 iff (alpha-1) s_j > tau).
 *
 * Defining passages (AdaSplash web pages, by title and section):
 *  - "AdaSplash: Adaptive Sparse Flash Attention" (ICML 2025 talk summary):
 *      Background -- alpha-entmax, alpha = 1 softmax, alpha = 2 sparsemax;
 *      Technical Deep Dive / Accelerated Alpha-Entmax Transformation -- tau as
 *        the root of f(tau) = 0, Halley-bisection;
 *      Technical Deep Dive / AdaSplash: Fused GPU Kernel for Attention -- the
 *        Q tile stays on chip, K tiles stream for the tau passes, a final pass
 *        streams K and V and accumulates O = P V without materialising S or P;
 *      Technical Deep Dive / Exploiting Sparsity -- all-zero tiles of P skip
 *        their K/V loads and compute, in the forward and the backward;
 *      Experimental Setup & Results / Backward Pass -- the backward skips the
 *        same zero tiles.
 *  - "AdaSplash-2: The Transformer Revolution We Didn't See Coming",
 *      Sparse Attention Makes Waves -- a coarse on-chip histogram of the
 *      scores starts the tau iteration (typically 1-2 further iterations).
 *
 * Conventions shared by every entry point:
 *  - Tensors are contiguous row-major [B][H][N][d] (q, k, v, o, dout, dq, dk,
 *    dv), all of one dtype: ENT_F32 (float) or ENT_BF16 (bfloat16 bits).
 *  - All tensor pointers are DEVICE pointers owned by the caller; the library
 *    allocates no memory.  Pointers must be 16-byte aligned.
 *  - The scale is fixed at 1/sqrt(d).  A score temperature beta is applied by
 *    the caller pre-scaling q.
 *  - tau is float32 [B][H][N], in units of x = (alpha-1) s (absolute, not
 *    shifted by the row maximum).
 *  - block_mask is uint8 [B][H][T][T], T = ceil(N/128): entry (t, b) is 1 iff
 *    the 128x128 block of P for query tile t and key block b holds a nonzero
 *    (blocks above the diagonal are 0 when causal).  The forward writes it;
 *    the backward reads it and skips exactly the 0 blocks.
 *  - Supported: 1 < alpha <= 2, d in {32, 64, 128}, 1 <= N <= 130944 (any N; the
 *    last tile may be ragged), B, H >= 0, B*H <= 65535.  B*H == 0 or N == 0 is a no-op returning ENT_OK.
 *  - Work is enqueued asynchronously on `stream` (a cudaStream_t; NULL is the
 *    legacy default stream).  Argument errors return synchronously before any
 *    work is enqueued.  No exception crosses the ABI.
 *  - ws / ws_bytes: caller-owned device workspace of at least the size that
 *    the matching *_workspace_size() returns.  The library zeroes what it
 *    needs on `stream`; its first 256 bytes hold a status word and counters
 *    (see ent_attn_read_status).
 *  - Device waits are bounded: a wait that gives up sets the status word in
 *    ws; ent_attn_read_status then reports ENT_ETIMEOUT.
 */
#ifndef ENTATTN_H
#define ENTATTN_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    ENT_OK = 0,
    ENT_EINVAL = 1,        /* a bad argument (null pointer, bad size, alpha out of range) */
    ENT_EUNSUPPORTED = 2,  /* a valid request the library does not implement (e.g. d = 96) */
    ENT_ECUDA = 3,         /* a CUDA runtime call failed; see ent_attn_last_error() */
    ENT_ETIMEOUT = 4       /* a bounded device wait gave up (reported by ent_attn_read_status) */
} ent_status;

typedef enum { ENT_F32 = 0, ENT_BF16 = 1 } ent_dtype;

/* Query/key tile edge of the block mask (128). */
int ent_attn_block_size(void);

/*
 * Bytes of device workspace the forward / backward need for this shape.
 * The forward's (bf16) holds the centroid bounds of the statistics pass, the list
 * of query tiles to solve again and, for N of at least 64 query tiles, the scores
 * of 8 sampled query rows per head (B*H*8*N floats) for the calibrated start.
 * The backward's is the 256-byte header plus delta, one float per query row:
 * 256 + round_up(B*H*N*4, 256).  A negative size gives 0.
 */
size_t ent_attn_fwd_workspace_size(int B, int H, int N, int d, int dtype);
size_t ent_attn_bwd_workspace_size(int B, int H, int N, int d, int dtype);

/*
 * Forward.  Inputs q, k, v [B,H,N,d].  Outputs: o [B,H,N,d] (same dtype),
 * tau float [B,H,N], block_mask uint8 [B,H,T,T] (all required) and iters
 * uint8 [B,H,N] (nullable): the number of tau-solver passes each row took
 * after the statistics pass.  Per 128-row query tile the kernel runs one
 * statistics pass (row max, per-block maxima, and the score histogram when
 * the histogram start is selected), solver passes until every row of the
 * tile has converged, and one P.V pass over the live key blocks.  A row stops
 * when |f(tau)| <= 1e-5 (bf16; 1e-6 float32), when its next step is below
 * 1e-6 (4e-7) * max(1, |tau|), or after 24 passes.  The bf16 path also stops
 * on a Halley step it does not evaluate when the step is at most 1e-2 and the
 * elements that can cross the support boundary within it change f by at most
 * 5e-5 upward (all leaving elements together: F2 h^2 for gamma >= 2, F1 h
 * below) or 3e-5 per entering element downward (h^min(gamma,2));
 * the P.V pass then checks |sum_j p_ij - 1| <= 1e-4 at the returned tau, and
 * every query tile with a row that fails the check is solved again with
 * evaluated stops only, by the CTAs of the same launch that are free.  The block mask is
 * written from p > 0 at the returned tau, so it is exact for that tau.
 * Environment switches read at each call, for ablations: ENTATTN_ACCEPT=0 (no
 * unevaluated stops), ENTATTN_VERIFY_TOL (the check's tolerance; negative:
 * solve every such tile again), ENTATTN_BOUND=0 (no centroid bound pass),
 * ENTATTN_SPEC=0 (no speculative first job: by default the K blocks of a score
 * pass's first job are loaded and multiplied again before the decision that
 * ends the pass, and used if the next pass starts with the same job).
 * bf16 inputs start every row's solver inside the plain bracket [m-1, m - n^(1-alpha)]
 * (measured faster on B200 than the histogram start, whose inserts cost more than
 * the passes they save): at its midpoint, or, for N of at least 64 query tiles, at
 * m - g, g = m - tau of the nearest of 8 query rows per head that two small kernels
 * solve exactly before the forward (ENTATTN_CALIB=0: the midpoint always).  The environment variable ENTATTN_HIST_BUDGET, read at each
 * call, selects the histogram start of the statistics pass instead: a tile builds
 * the histogram until it has made that many inserts after its first block (a
 * negative value: no limit).  float32 inputs always use the histogram start.  The
 * result is the same to the solver's stop rule either way.
 */
ent_status ent_attn_fwd(const void *q, const void *k, const void *v,
                        int B, int H, int N, int d, int dtype,
                        float alpha, int causal,
                        void *o, float *tau, uint8_t *block_mask, uint8_t *iters,
                        void *ws, size_t ws_bytes, void *stream);

/*
 * Backward.  Inputs q, k, v, o, dout [B,H,N,d]; tau and block_mask as the
 * forward wrote them.  Outputs dq, dk, dv [B,H,N,d] (same dtype), computed
 * with g = (x - tau)_+^(1/(alpha-1) - 1), delta_i = sum_j g_ij dP_ij /
 * sum_j g_ij, dS = g (dP - delta), dP = dO V^T:
 *     dQ = dS K / sqrt(d),  dK = dS^T Q / sqrt(d),  dV = P^T dO,
 * visiting only blocks whose block_mask entry is 1.  `o` is accepted for
 * interface symmetry and may be NULL (entmax has no O-based shortcut for
 * delta; it is recomputed from the live blocks).
 */
ent_status ent_attn_bwd(const void *q, const void *k, const void *v, const void *o,
                        const void *dout, const float *tau, const uint8_t *block_mask,
                        int B, int H, int N, int d, int dtype, float alpha, int causal,
                        void *dq, void *dk, void *dv,
                        void *ws, size_t ws_bytes, void *stream);

/*
 * Forward that also returns otilde, float32 [B,H,N,d] (caller-owned, 16-byte
 * aligned): the g-weighted mean of the value rows at the returned tau,
 *     otilde_i = sum_j g_ij v_j / sum_j g_ij,   g = (x - tau)_+^(1/(alpha-1) - 1).
 * Everything else is ent_attn_fwd's (same outputs, same workspace size).  The
 * backward's delta_i = sum_j g_ij dP_ij / sum_j g_ij equals dO_i . otilde_i
 * because dP = dO V^T (derived from the definition), so ent_attn_bwd_otilde
 * needs no delta pass over the keys.  The P.V pass then also accumulates G V
 * (one more 128x128xd block product per live block, counter [5]); on the
 * bf16 path g is rounded to bf16 for that product, as P is.  A null otilde is
 * ENT_EINVAL.
 */
ent_status ent_attn_fwd_otilde(const void *q, const void *k, const void *v,
                               int B, int H, int N, int d, int dtype,
                               float alpha, int causal,
                               void *o, float *tau, uint8_t *block_mask, uint8_t *iters,
                               float *otilde, void *ws, size_t ws_bytes, void *stream);

/*
 * Backward given otilde from ent_attn_fwd_otilde of the same q, k, v (with
 * the tau and block_mask of that call): delta_i = dO_i . otilde_i, then dq,
 * dk, dv exactly as ent_attn_bwd computes them, without the delta pass (two
 * block products per live block fewer).  Same workspace size as
 * ent_attn_bwd.  A null otilde is ENT_EINVAL.
 */
ent_status ent_attn_bwd_otilde(const void *q, const void *k, const void *v, const float *otilde,
                               const void *dout, const float *tau, const uint8_t *block_mask,
                               int B, int H, int N, int d, int dtype, float alpha, int causal,
                               void *dq, void *dk, void *dv,
                               void *ws, size_t ws_bytes, void *stream);

/*
 * Support lists: the forward pair for rows with few nonzeros ("AdaSplash: Adaptive
 * Sparse Flash Attention", Technical Deep Dive / Exploiting Sparsity -- skipping the
 * zeros of P, here at the grain of single keys instead of 128x128 blocks).
 *
 * ent_attn_fwd_lists is ent_attn_fwd (same outputs, workspace, limits) that also
 * records, for every query row, the keys j with p_ij > 0 and u_ij = x_ij - tau_i:
 *   list_key int32 [B,H,N,cap], list_u float [B,H,N,cap] (cap = ent_attn_list_cap(),
 *   16): entries 0 .. list_n-1 of the row, in no particular order (the rest of the
 *   row is not written);
 *   list_n uint8 [B,H,N]: the number of entries, or 255 when the row has more than
 *   cap nonzeros (its list is then incomplete and must not be used).
 * All three are caller-owned device buffers, required (NULL is ENT_EINVAL).  bf16
 * inputs only (float32: ENT_EUNSUPPORTED).
 *
 * ent_attn_bwd_lists is ent_attn_bwd given those lists (and the tau and block_mask of
 * the same forward): every query tile whose rows all have lists (list_n != 255) is
 * done from its lists alone -- per listed key, dP = dO_i . v_j, then delta, dS and
 * the dQ, dK, dV contributions, with no score recomputation -- and the remaining
 * tiles by the block kernels of ent_attn_bwd.  Same outputs as ent_attn_bwd (up to
 * fp32 summation order: dK and dV collect the list contributions by atomic adds).
 * Its workspace: ent_attn_bwd_lists_workspace_size (ent_attn_bwd's plus one byte per
 * query tile and two float [B,H,N,d] accumulators).  The list kernel runs on a
 * library-owned non-blocking stream (one per device) forked from `stream` by an
 * event and joined back into it before the last kernel, so the work is ordered
 * after everything enqueued on `stream` before the call and complete when `stream`
 * passes the call (stream capture sees the same fork and join).
 */
int ent_attn_list_cap(void);
size_t ent_attn_bwd_lists_workspace_size(int B, int H, int N, int d, int dtype);
ent_status ent_attn_fwd_lists(const void *q, const void *k, const void *v,
                              int B, int H, int N, int d, int dtype,
                              float alpha, int causal,
                              void *o, float *tau, uint8_t *block_mask, uint8_t *iters,
                              int32_t *list_key, float *list_u, uint8_t *list_n,
                              void *ws, size_t ws_bytes, void *stream);
ent_status ent_attn_bwd_lists(const void *q, const void *k, const void *v,
                              const int32_t *list_key, const float *list_u,
                              const uint8_t *list_n, const void *dout, const float *tau,
                              const uint8_t *block_mask,
                              int B, int H, int N, int d, int dtype, float alpha, int causal,
                              void *dq, void *dk, void *dv,
                              void *ws, size_t ws_bytes, void *stream);

/*
 * Backward without a workspace argument.  The pages have no counterpart: this
 * is a library convenience.  It computes exactly what ent_attn_bwd computes
 * (same kernels, same arguments minus ws / ws_bytes) for callers that cannot
 * allocate device memory when they run the backward -- stacks that plan all
 * device memory ahead of time and forbid later cudaMalloc calls (an
 * allocation can synchronise the device and fragments a fixed pool), or plain
 * C code with no device allocator to size and own a workspace.
 *  - Scratch: a fixed 4 MiB device array inside the library (a 256-byte header
 *    plus one float per query row), held on every GPU that loads the library
 *    until the process exits.  B*H*N above 1,048,512 rows returns
 *    ENT_EUNSUPPORTED with a message; use ent_attn_bwd then.
 *  - The first call on each device looks up the array's device address
 *    (cudaGetSymbolAddress, with that device current) and caches it; make that
 *    first call before any stream capture.
 *  - All calls share the one array, and it keeps the previous call's contents
 *    (the call clears the header itself): calls whose work overlaps on the GPU
 *    (concurrent streams, or other host threads) race and must be ordered by
 *    the caller.
 *  - A bounded device wait that gives up sets the status word in the array's
 *    header; ent_attn_noalloc_read_status reads it (and the counters) back.
 * Allocates nothing: no cudaMalloc, cudaFree or allocating library call.
 */
ent_status ent_attn_bwd_noalloc(const void *q, const void *k, const void *v, const void *o,
                                const void *dout, const float *tau, const uint8_t *block_mask,
                                int B, int H, int N, int d, int dtype, float alpha, int causal,
                                void *dq, void *dk, void *dv, void *stream);

/*
 * Status of the last ent_attn_bwd_noalloc call on the current device: the
 * same as ent_attn_read_status on a workspace (synchronises `stream`, copies
 * the header to the host, fills counters when non-null, returns ENT_ETIMEOUT
 * if a bounded wait gave up), read from the library's fixed array.  The array
 * is shared, so the answer belongs to whichever ent_attn_bwd_noalloc call
 * last wrote it; order the calls.  Returns ENT_EINVAL if no
 * ent_attn_bwd_noalloc call has looked up the array on this device yet.
 * Allocates nothing.
 */
ent_status ent_attn_noalloc_read_status(long long *counters, void *stream);

/*
 * Synchronises `stream` and reads the status word and the work counters of a
 * workspace that a forward or backward used.  counters (nullable, 8 entries):
 *   [0] block products (128x128xd, 2*128*128*d flops each) in the forward's
 *       statistics and solver passes (one S block per visited block and pass,
 *       plus the blocks of speculative first jobs that were not used),
 *   [1] live blocks in the forward P.V pass (two block products each: S, P V),
 *   [2] solver passes summed over query tiles,
 *   [3] query tiles processed,
 *   [4] block products issued by the backward kernels (all of them),
 *   [5] G.V block products of ent_attn_fwd_otilde (one per live block),
 *   [6] key blocks a forward left out of its statistics pass because a centroid
 *       bound rules them out for every row of the query tile (bf16 path; the
 *       bound's own products, one per 128 centroids, are counted in [0]),
 *   [7] support-list entries the backward of ent_attn_bwd_lists handled (8*d flops
 *       each: the dP, dQ, dK and dV terms of one nonzero).
 * Executed flops of a call = 2*128*128*d * ([0] + 2*[1] + [4] + [5]) + 8*d*[7].
 * Returns ENT_OK, ENT_ETIMEOUT if a bounded wait gave up, ENT_ECUDA on a
 * CUDA error.
 */
ent_status ent_attn_read_status(const void *ws, long long *counters, void *stream);

/* Thread-local message describing the last non-OK status of this thread. */
const char *ent_attn_last_error(void);

/*
 * Row-wise alpha-entmax of a score matrix, without attention ("AdaSplash:
 * Adaptive Sparse Flash Attention", Background and Technical Deep Dive /
 * Accelerated Alpha-Entmax Transformation; "AdaSplash-2: ...", Sparse Attention
 * Makes Waves): for each row of z [rows][n] (row-major, contiguous),
 *     p_j = ((alpha-1) z_j - tau)_+^(1/(alpha-1)),   sum_j p_j = 1,
 * with tau the root of f(tau) = sum_j ((alpha-1) z_j - tau)_+^gamma - 1, in units of
 * (alpha-1) z.  `method` picks the root finder (same stop rule as the attention
 * forward: |f| <= 1e-6 (float32) / 1e-5 (bf16), or a step below 4e-7 / 1e-6 of
 * max(1,|tau|), or the pass cap):
 *   ENT_SOLVE_HIST    Halley-bisection from the bracket and start of a 64-bin
 *                     histogram of the row (the attention path's solver);
 *   ENT_SOLVE_HALLEY  Halley-bisection from the plain bracket
 *                     [m - 1, m - n^(1-alpha)] (m = row max), midpoint start;
 *   ENT_SOLVE_BISECT  bisection on the plain bracket (pass cap 48).
 * Outputs (device, caller-owned): p [rows][n] in the dtype of z, tau float
 * [rows], iters uint8 [rows] (nullable; solver passes per row).  Supported:
 * 1 < alpha <= 2, 1 <= n <= ent_entmax_rows_max_n() (ENT_EUNSUPPORTED above);
 * rows = 0 or n = 0 is a no-op.  No workspace; asynchronous on `stream`.
 * Returns ENT_EINVAL for a bad argument (checked before any work is queued),
 * ENT_ECUDA if a launch fails.
 */
#define ENT_SOLVE_HIST 0
#define ENT_SOLVE_HALLEY 1
#define ENT_SOLVE_BISECT 2
int ent_entmax_rows_max_n(void);
ent_status ent_entmax_rows_fwd(const void *z, int rows, int n, int dtype, float alpha,
                               int method, void *p, float *tau, uint8_t *iters, void *stream);

/*
 * Vector-Jacobian product of ent_entmax_rows_fwd (derived from the definition):
 * dz_j = g_j (dp_j - delta), g_j = ((alpha-1) z_j - tau)_+^(gamma-1) (0 off the
 * support), delta = sum_j g_j dp_j / sum_j g_j.  z, dp, dz [rows][n] in one dtype;
 * tau float [rows] as the forward returned it.  Same limits and errors as the
 * forward.
 */
ent_status ent_entmax_rows_bwd(const void *z, const float *tau, const void *dp, int rows, int n,
                               int dtype, float alpha, void *dz, void *stream);

#ifdef __cplusplus
}
#endif
#endif /* ENTATTN_H */
