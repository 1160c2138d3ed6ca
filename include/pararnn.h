/*
 * pararnn.h -- C ABI of the B200 (sm_100a) ParaGRU / ParaLSTM Newton-scan
 * solver.
 *
 * The problem (from "Параллельность RNN?", §1.1): given the initial state s_0
 * and the inputs, the states s_1..s_T of the recurrence s_t = f(s_{t-1}, x_t)
 * are the unique root of the residual r_t = s_t - f(s_{t-1}, x_t).  The
 * solvers find it by Newton iterations (§1.2) whose linear systems have a
 * block-bidiagonal Jacobian (§1.3); each system is the linear recurrence
 * ds_t = A_t ds_{t-1} - r_t, solved by an associative scan over affine pairs
 * (A, b) (§1.3, "Уровень 2").  The cells have diagonal recurrent weights, so
 * A_t is diagonal for ParaGRU and 2x2 block-diagonal per channel for ParaLSTM
 * ("Apple научила классические RNN масштабироваться до 7B параметров...",
 * "Что именно сделали технически", item 3).  The interface mirrors the
 * pages' step signature recurrence_step(h, x, system_parameters) ("Как
 * запустить"): x is the precomputed gate input projection u, the system
 * parameters are the diagonal weights a and the biases.
 *
 * Cells (every product is elementwise; sig = logistic sigmoid):
 *   ParaGRU  gates (z, r, c):
 *     z = sig(a_z h + u_z + b_z)   r = sig(a_r h + u_r + b_r)
 *     c = tanh(a_c (r h) + u_c + b_c)          h' = (1 - z) h + z c
 *   ParaLSTM gates (i, f, g, o), state (c, h):
 *     i = sig(a_i h + u_i + b_i)   f = sig(a_f h + u_f + b_f)
 *     g = tanh(a_g h + u_g + b_g)  o = sig(a_o h + u_o + b_o)
 *     c' = f c + i g               h' = o tanh(c')
 *
 * Layouts (row-major, channel index d fastest, all contiguous):
 *   u        [B][T][G][D]  G = 3 (GRU) or 4 (LSTM); bf16 or fp32
 *   a, bias  [G][D]        fp32
 *   h0, c0   [B][D]        fp32
 *   h, c     [B][T][D]     fp32, state after step t at index t-1
 *   dLdh     [B][T][D]     fp32
 *   du       [B][T][G][D]  fp32
 *   da,dbias [G][D]        fp32
 *
 * Conventions shared by every entry point:
 *   - All array pointers are DEVICE pointers owned by the caller.  The library
 *     allocates no memory and keeps no global state.
 *   - Calls are asynchronous on `stream` (a cudaStream_t; NULL = legacy
 *     default stream).  Device-written results (states, stats, status) are
 *     valid once the stream reaches that point; reading them is the caller's
 *     synchronisation.
 *   - Host-detectable errors return a negative PARARNN_ERR_* code before any
 *     work is enqueued.  Outcomes decided on the device go to a status word.
 *   - Requirements: B, T, D >= 1; D % 8 == 0; u, h, c, du, dLdh 16-byte
 *     aligned; a, bias, h0, c0, da, dbias, dc0, dh0 4-byte aligned.
 *   - The workspace: size from pararnn_workspace_size(); it must be
 *     zero-filled once before its first use (pararnn_workspace_init), after
 *     which the library keeps it consistent across calls (each call bumps an
 *     epoch counter stored in it).  One call at a time may use a workspace.
 *   - No entry point traps, asserts or waits without bound on the device:
 *     every cross-block wait gives up after opts.timeout_us microseconds and
 *     reports PARARNN_STATUS_TIMEOUT.
 */
#ifndef PARARNN_H
#define PARARNN_H

#include <stddef.h>

#ifdef __cplusplus
extern "C" {
#endif

/* cudaStream_t without including CUDA headers */
typedef struct CUstream_st* pararnn_stream_t;

/* element type of u */
enum { PARARNN_F32 = 0, PARARNN_BF16 = 1 };
/* cell selector */
enum { PARARNN_GRU = 0, PARARNN_LSTM = 1 };

/* host return codes */
#define PARARNN_OK 0
#define PARARNN_ERR_INVALID_ARG (-1)
#define PARARNN_ERR_UNSUPPORTED_DTYPE (-2)
#define PARARNN_ERR_WORKSPACE_TOO_SMALL (-3)
#define PARARNN_ERR_CUDA (-4)
#define PARARNN_ERR_MISALIGNED (-5)
#define PARARNN_ERR_TOO_LARGE (-6)

/* device status word values (pararnn_stats.status, adjoint *status) */
#define PARARNN_STATUS_CONVERGED 0
#define PARARNN_STATUS_NOT_CONVERGED 1
#define PARARNN_STATUS_NONFINITE 2
#define PARARNN_STATUS_TIMEOUT 3

/* opts.flags */
#define PARARNN_FLAG_INJECT_WITHHOLD 1u /* testing: a part of the solve's
                                           exchange is withheld so that the
                                           bounded waits for it run out
                                           (TIMEOUT): in the chunked forward
                                           solves cluster chunk inject_chunk
                                           never publishes its look-back
                                           record; in the row solves the CTA
                                           of cluster rank inject_chunk
                                           withholds its exchange at the
                                           residual-only evaluation of the
                                           cap (use max_iters to reach it);
                                           in the segment-queue solve item
                                           inject_chunk (segment-major:
                                           segment * tiles + tile) never
                                           publishes its states to the next
                                           segment; for the adjoint see
                                           pararnn_adjoint_ex */
#define PARARNN_FLAG_FORCE_CHUNKED 2u   /* use the chunked (cluster + decoupled
                                           look-back) solve where the
                                           whole-sequence row kernels would
                                           run: ParaGRU with T <= 4096 (bf16 or
                                           fp32 u) or longer with at least one
                                           8-channel tile per SM, ParaLSTM with
                                           bf16 u and T <= 4096 (segmented as
                                           the solves' comments say) */
#define PARARNN_FLAG_DENSE_SIMT 8u      /* pararnn_dense_gru_solve: fp32
                                           products on CUDA cores (exact
                                           Newton steps, D <= 128) instead of
                                           tf32 tensor-core products */
#define PARARNN_FLAG_FORCE_ROW 4u       /* bf16 u: the whole-sequence (row)
                                           kernels, launched segment by
                                           segment, where the one-launch
                                           segment-queue solves (forward of
                                           both cells, ParaGRU adjoint) would
                                           run (kept for comparison) */
#define PARARNN_FLAG_EXACT_STEPS 16u    /* every Newton evaluation exact.
                                           Without it the segment-queue
                                           solves (both cells) and the
                                           ParaGRU row kernels evaluate the
                                           cell with the one-instruction tanh
                                           (gates within about 2^-11
                                           relative) while the item's max |r|
                                           is above 0.1, and decide
                                           convergence on exact evaluations
                                           only: the converged states are
                                           the same, the iterates before that
                                           are inexact Newton iterates.  With
                                           it, a solve capped at n updates
                                           returns the n-th exact iterate. */

typedef struct {
  float tol;          /* stop when max|r| < tol; <= 0 -> 1e-6 */
  int max_iters;      /* cap on Newton updates; <= 0 -> 64 (the workspace is
                         sized for this value) */
  unsigned flags;     /* PARARNN_FLAG_* */
  int inject_chunk;   /* chunk index for PARARNN_FLAG_INJECT_WITHHOLD */
  unsigned timeout_us;/* bound on any cross-block wait; 0 -> 2,000,000 */
  int max_cluster;    /* cap on CTAs per thread-block cluster (2..16);
                         0 -> the largest the device can keep resident */
  int* chan_iters;    /* fused forward solves only: device int [B][D] or NULL.
                         Receives each (b, d) channel's iteration index, the
                         input of iter_hist: the number of updates applied
                         before the first evaluation from which the channel's
                         own max_t |r_t| stays below tol (max_iters + 1 if it
                         never got there).  Where the sequence is solved in
                         segments, the largest index over the segments.  An
                         inexact evaluation (see PARARNN_FLAG_EXACT_STEPS)
                         never counts as below tol.
                         4-byte aligned; the call overwrites every entry. */
} pararnn_opts;

/* Device-resident solve statistics (written by the solve; zeroed by it at
 * the start of the call). */
typedef struct {
  int iters;          /* Newton updates applied (max over sequence chunks) */
  float max_residual; /* max|r| at the last evaluated iterate, before the
                         final update (max over chunks) */
  int status;         /* PARARNN_STATUS_* (max over chunks) */
  int evals;          /* cell evaluations per element (max over chunks) */
} pararnn_stats;

/* Bytes of workspace a call needs.  `adjoint` = 0 for the forward solves,
 * 1 for pararnn_adjoint.  max_iters as in pararnn_opts (<= 0 -> default).
 * Returns 0 on invalid sizes. */
size_t pararnn_workspace_size(int cell, int B, int T, int D, int max_iters,
                              int adjoint);

/* Zero-fill a workspace (stream-ordered).  Needed once before first use. */
int pararnn_workspace_init(void* workspace, size_t ws_bytes,
                           pararnn_stream_t stream);

/* ParaGRU forward solve.
 * In:  u [B][T][3][D] (z, r, c projections; dtype u_dtype), a [3][D],
 *      bias [3][D] or NULL (zeros), h0 [B][D] or NULL (zeros).
 * Out: h [B][T][D] states; *stats (device); iter_hist [max_iters+2] or NULL:
 *      iter_hist[k], k <= max_iters, counts the (b, d) channels whose own
 *      max_t |r_t| is below tol from evaluation k onwards (k = updates applied
 *      before that evaluation); iter_hist[max_iters+1] counts channels that
 *      never got there within the cap.
 * Newton starts from h = 0 at every t, applies the page's update until the
 * residual of an iterate is below tol everywhere upstream (and then applies
 * that last update), or until max_iters updates have been applied.  The
 * segment-queue and whole-sequence solves evaluate only the residual of an
 * iterate reached by an exact step from a residual at most sqrt(tol), and
 * return that iterate itself when it is below tol.  Channels are
 * independent; each 8-channel tile stops on its own.  With bf16 u and at
 * least one 8-channel tile per resident CTA of the segment-queue solve
 * (B * D / 8 >= 4 * SMs), one launch solves every 512-step segment of every
 * tile, each segment from the state the one before it converged to (stats
 * and iter_hist take the maximum over the segments).  Otherwise a sequence of
 * up to 4096 steps is held by a cluster of k CTAs of 1024 steps per tile; when a
 * smaller cluster of k' CTAs already gives two CTAs per SM
 * (k' * B * D / 8 >= 2 * SMs), it is solved in segments of k' * 1024 steps.
 * A longer sequence with at least one 8-channel tile (B * D / 8) per SM is
 * solved in 4096-step segments.  Each segment starts from the state the one
 * before it converged to; stats and iter_hist then take the maximum over the
 * segments.  Shorter-tiled long sequences use one solve over the whole
 * sequence (cluster chunks joined by decoupled look-back). */
int pararnn_gru_solve(const void* u, int u_dtype, const float* a,
                      const float* bias, const float* h0, float* h, int B,
                      int T, int D, const pararnn_opts* opts,
                      pararnn_stats* stats, int* iter_hist, void* workspace,
                      size_t ws_bytes, pararnn_stream_t stream);

/* ParaLSTM forward solve.  As pararnn_gru_solve with u [B][T][4][D]
 * (i, f, g, o), a/bias [4][D], initial cell state c0 (NULL = zeros) and both
 * state trajectories out: c [B][T][D], h [B][T][D].  The residual norm is the
 * max over both components.  With bf16 u and at least one 8-channel tile per
 * resident CTA of the segment-queue solve (B * D / 8 >= 4 * SMs), one launch
 * solves every 128-step segment of every tile (any T), each segment from the
 * (c, h) the one before it converged to.  Otherwise, with bf16 u and
 * T <= 4096, a tile's sequence is held by a cluster of k CTAs of 512 steps
 * each; when a smaller cluster of k' CTAs already puts one CTA on every SM
 * (k' * B * D / 8 >= SMs), the sequence is solved in segments of k' * 512
 * steps instead, each starting from the (c, h) the one before it converged
 * to; stats and iter_hist then take the maximum over the segments.  The
 * segment-queue and whole-sequence solves check an iterate reached by an
 * exact step from a residual at most sqrt(tol / 2) by its residual alone and
 * return it when that is below tol / 2 (a margin for the fp32 rounding of a
 * cell state, which is not bounded). */
int pararnn_lstm_solve(const void* u, int u_dtype, const float* a,
                       const float* bias, const float* c0, const float* h0,
                       float* c, float* h, int B, int T, int D,
                       const pararnn_opts* opts, pararnn_stats* stats,
                       int* iter_hist, void* workspace, size_t ws_bytes,
                       pararnn_stream_t stream);

/* Adjoint (backward) of a solved trajectory: the reverse scan
 *   lambda_t = g_t + A_{t+1}^T lambda_{t+1},  lambda_T = g_T
 * on the transposed Jacobians (Jacobian structure from "Параллельность
 * RNN?", §1.3), with g_t = dL/dh_t (dL/dc_t = 0 for ParaLSTM).  Outputs
 *   du_t = (df_t/du_t)^T lambda_t                [B][T][G][D]
 *   da   = sum_{b,t} (df_t/da)^T lambda_t        [G][D]
 *   dbias= sum_{b,t} du_t  (NULL to skip)        [G][D]
 *   dh0  = d L / d h0, dc0 = d L / d c0 (LSTM; NULL to skip) [B][D]
 * c0 and c must be NULL for ParaGRU and non-NULL for ParaLSTM.  The sums over
 * (b, t) are reduced in a fixed order (bitwise reproducible).
 * *status (device int) receives PARARNN_STATUS_CONVERGED (0) on success,
 * NONFINITE or TIMEOUT otherwise. */
int pararnn_adjoint(int cell, const void* u, int u_dtype, const float* a,
                    const float* bias, const float* c0, const float* h0,
                    const float* c, const float* h, const float* dLdh,
                    float* du, float* da, float* dbias, float* dc0, float* dh0,
                    int B, int T, int D, int* status, void* workspace,
                    size_t ws_bytes, pararnn_stream_t stream);

/* pararnn_adjoint with options: opts->timeout_us bounds every cross-block
 * wait (0 or NULL opts: 2 s); with PARARNN_FLAG_INJECT_WITHHOLD in
 * opts->flags, for testing, a part of the exchange is withheld so that the
 * waits for it run out and *status becomes PARARNN_STATUS_TIMEOUT: in the
 * look-back adjoint (fp32 u or T > 4096) the chunk whose ticket is
 * opts->inject_chunk (the tile's chunks take tickets last first) publishes
 * no records; in the whole-sequence adjoint (bf16 u, T <= 4096) the CTA of
 * cluster rank opts->inject_chunk withholds its map in its cluster's last
 * tile; in the queue adjoints item opts->inject_chunk (r * tiles + tile for
 * the segment r from the end) never publishes its carry.  With
 * PARARNN_FLAG_FORCE_ROW in opts->flags the whole-sequence kernels run where
 * the queue adjoint would.  Other opts fields are ignored.  NULL opts =
 * pararnn_adjoint.
 * Kernels: bf16 u with at least one tile per resident CTA of the queue
 * adjoint takes the queue adjoint (every segment of every tile in one launch,
 * last segments first, each segment's carry from the segment after it):
 * 32-channel tiles in 128-step segments, one 16-warp CTA per SM (so at
 * least 148 tiles of 32 channels on a B200).  Other bf16
 * problems with T <= 4096 the
 * whole-sequence kernels (a cluster of CTAs per tile); the rest the chunked
 * look-back adjoint.  The first two stage the rows of a, bias, h0 and c0 by
 * 1-D bulk copies and are taken only when those pointers are 16-byte aligned
 * (4-byte aligned rows take the look-back adjoint: same results within
 * rounding, slower). */
int pararnn_adjoint_ex(int cell, const void* u, int u_dtype, const float* a,
                       const float* bias, const float* c0, const float* h0,
                       const float* c, const float* h, const float* dLdh,
                       float* du, float* da, float* dbias, float* dc0,
                       float* dh0, int B, int T, int D, int* status,
                       void* workspace, size_t ws_bytes,
                       const pararnn_opts* opts, pararnn_stream_t stream);

/* Adjoint without a caller-supplied workspace.  (The pages have no
 * counterpart; this is a library convenience.)  For callers that cannot hand
 * the library scratch memory -- because an allocator they do not control owns
 * the device memory, or because cudaMalloc's latency and implicit
 * synchronisation are not acceptable on their path.  Same arguments and
 * results as pararnn_adjoint minus the workspace: the scratch is a fixed
 * PARARNN_NOALLOC_SCRATCH_BYTES array inside the library, held in device
 * memory by every GPU that loads the library until the process exits.  The
 * call allocates nothing.  The first call on a device looks the array's
 * address up (cudaGetSymbolAddress) and clears the array with a memset on
 * `stream`, ordered before that call's kernels; make that first call before
 * any stream capture.  All calls on a device share the array, which keeps
 * what the last call left in it (nothing that can mislead the next call):
 * calls that overlap on the GPU race and must not be made.  Problems that need more scratch than the
 * array holds (pararnn_workspace_size(cell, B, T, D, 0, 1) above the limit:
 * about 13000 ParaGRU chunks of 32 channels x 128 steps, i.e.
 * B*ceil(D/32)*ceil(T/128), or about 6500 ParaLSTM chunks of 32 x 64) return
 * PARARNN_ERR_WORKSPACE_TOO_SMALL without launching anything. */
#define PARARNN_NOALLOC_SCRATCH_BYTES (16u << 20)
int pararnn_adjoint_noalloc(int cell, const void* u, int u_dtype,
                            const float* a, const float* bias,
                            const float* c0, const float* h0, const float* c,
                            const float* h, const float* dLdh, float* du,
                            float* da, float* dbias, float* dc0, float* dh0,
                            int B, int T, int D, int* status,
                            pararnn_stream_t stream);

/* Naive step-by-step GPU evaluation (one thread per (b, d) channel looping
 * over t) -- the sequential baseline the parallel solve is compared with.
 * c0/c must be NULL for ParaGRU.  No workspace. */
int pararnn_seq_baseline(int cell, const void* u, int u_dtype, const float* a,
                         const float* bias, const float* c0, const float* h0,
                         float* c, float* h, int B, int T, int D,
                         pararnn_stream_t stream);

/* Unfused Newton solve: the "CUDA-accelerated" tier of the pages' three
 * ("Apple научила классические RNN масштабироваться...", "Три уровня
 * производительности"), kept as an ablation against the fused solves.  Each
 * iteration ("Параллельность RNN?", §1.2-§1.3) runs one kernel that writes
 * the Jacobian blocks A_t and the right-hand sides -r_t of every element to
 * the workspace, three kernels that solve ds_t = A_t ds_{t-1} - r_t by a
 * chunked scan and add ds to the iterate, and a host check of the residual.
 * cell: PARARNN_GRU (c0 and c NULL) or PARARNN_LSTM; u, a, bias, c0, h0, c, h
 * as for pararnn_gru_solve / pararnn_lstm_solve.  Stopping is global: the
 * update of the first iteration whose max|r| over the whole problem is below
 * opts->tol is applied and the solve ends; the cap ends with a residual-only
 * evaluation and NOT_CONVERGED.  *stats as for the fused solves; there is no
 * iteration histogram.
 * Blocking: the host reads the residual after every iteration, so the call
 * synchronises `stream` and returns when the solve is done.
 * Workspace: pararnn_unfused_workspace_size(cell, B, T, D) bytes, 256-byte
 * aligned, no initialisation (4 B per element for each Jacobian entry and
 * right-hand side: 8 B per element for ParaGRU, 24 B for ParaLSTM, plus the
 * scan's chunk maps).  Alignment: u 2 B (bf16) or 4 B (fp32), the float
 * arrays 4 B.  Errors as for the fused solves. */
size_t pararnn_unfused_workspace_size(int cell, int B, int T, int D);
int pararnn_solve_unfused(int cell, const void* u, int u_dtype, const float* a,
                          const float* bias, const float* c0,
                          const float* h0, float* c, float* h, int B, int T,
                          int D, const pararnn_opts* opts,
                          pararnn_stats* stats, void* workspace,
                          size_t ws_bytes, pararnn_stream_t stream);

/* Newton solve for a general cell with a dense D x D Jacobian: the GRU with
 * full recurrent matrices ("Параллельность RNN?", §1.3: the block-bidiagonal
 * Jacobian with full blocks -df/ds below the identities):
 *   z = sig(W_z h + u_z + b_z), r = sig(W_r h + u_r + b_r),
 *   c = tanh(u_c + b_c + r (W_c h)), h' = (1 - z) h + z c.
 * With diagonal W_g it is the ParaGRU cell.  In: u [B][T][3][D] (dtype
 * u_dtype), W [3][D][D] row-major (row i of W_g feeds unit i), bias [3][D]
 * or NULL, h0 [B][D] or NULL.  Out: h [B][T][D], *stats (device).  Each
 * iteration writes the blocks J_t and -r_t to the workspace, solves
 * ds_t = J_t ds_{t-1} - r_t by a chunked scan of D x D maps and checks the
 * residual on the host: stopping is global, as for pararnn_solve_unfused,
 * and the call synchronises `stream`.  The contractions (the recurrent
 * pre-activations, and the products of blocks that compose 16-step chunk
 * maps, a tree of four levels) run on the tensor cores with tf32 inputs and
 * fp32 accumulation: each Newton step is then inexact (about 1e-3 relative
 * in the chunk maps) while the residual, evaluated in fp32, still defines the
 * fixed point.  opts->flags PARARNN_FLAG_DENSE_SIMT takes fp32 products on
 * CUDA cores instead (exact steps).  D a multiple of 8, at most 512 (128 with
 * PARARNN_FLAG_DENSE_SIMT).  W, h and h0 16-byte aligned.  Status TIMEOUT if
 * a tensor-core product's bounded wait ran out.
 * Workspace: pararnn_dense_workspace_size(B, T, D) bytes (about 8 D^2 + 32 D
 * bytes per (b, t) with T rounded up to 16, plus 12 D^2 for W^T), 256-byte
 * aligned, no initialisation; 0 means the shape is not supported.  Errors as
 * for the other solves. */
size_t pararnn_dense_workspace_size(int B, int T, int D);
/* The tensor-core contraction of pararnn_dense_gru_solve, exposed so that it
 * can be checked on its own: C[z] = A[z] B[z]^T for z < Z, with A[z] M x K
 * and B[z] N x K row-major fp32 (A[z] at A + z M K, B[z] at Bm + z N K),
 * tf32 products (tcgen05.mma kind::tf32) accumulated in fp32.  C[z] at
 * C + z M N: row-major M x N (store_mode 0), transposed N x M (1),
 * row-major for odd z and transposed for even z (2), or row-major with the
 * product added to what C holds (3).  Launches with at least one 128 x 256
 * output tile per SM run a persistent kernel (one CTA per SM, 128 x 256
 * tiles, two accumulators in tensor memory), smaller ones one CTA per
 * 128 x 128 tile.  K a multiple of 4; A,
 * Bm, C 16-byte aligned.  *err (device int) is set to 1 if a bounded wait ran
 * out (the affected tiles are not written); it is not cleared. */
int pararnn_dense_matmul(const float* A, const float* Bm, float* C, int M,
                         int N, int K, int Z, int store_mode, int* err,
                         pararnn_stream_t stream);
int pararnn_dense_gru_solve(const void* u, int u_dtype, const float* W,
                            const float* bias, const float* h0, float* h,
                            int B, int T, int D, const pararnn_opts* opts,
                            pararnn_stats* stats, void* workspace,
                            size_t ws_bytes, pararnn_stream_t stream);

/* Sequence sharding: the time axis split over processes (GPUs).  Shard r of
 * W holds steps [T_r, T_{r+1}) of every (b, d) channel: its slice of u
 * ([B][Ts][G][D], Ts = T_{r+1} - T_r) and of the iterate.  The page's linear
 * system of a Newton iteration ("Параллельность RNN?", §1.3) couples a shard
 * to the shards before it only through the delta entering its first step,
 * and the scan's operator is associative ("Уровень 2"), so long sequences
 * can be cut into chunks solved apart and joined ("ParaRNN：解锁非线性RNN并行
 * 训练的革命性框架", on long sequences).  One Newton iteration of the
 * sharded solve is
 *   1. pararnn_shard_eval on every shard: residual and Jacobians at the
 *      iterate, the shard's system solved from a zero incoming delta, its map
 *      ds_out = P ds_in + d and its last state(s) before the update, max|r|;
 *   2. an exchange of every shard's map, last states and max|r| (all-gather
 *      and all-reduce over the processes: NCCL between GPUs);
 *   3. pararnn_shard_combine on every shard: the delta entering it (the maps
 *      of the shards before it, composed in order) and its new initial state
 *      for the next iteration (the previous shard's last state plus that
 *      delta; shard 0 keeps the true initial state);
 *   4. pararnn_shard_apply: the local solution plus P_t ds_in added to the
 *      iterate.
 * These are the Newton iterates of the whole sequence (with the stopping
 * rule of pararnn_solve_unfused applied to the global max|r|), so the result
 * does not depend on how T is split.  The loop and the exchange run on the
 * host (nonlinear_rnn_paragru_b200.shard).  cell PARARNN_GRU or PARARNN_LSTM;
 * for ParaGRU the c arguments are NULL.
 *
 * Workspace: pararnn_shard_workspace_size(cell, B, Ts, D) bytes, 256-byte
 * aligned, no initialisation; it carries the Jacobians and chunk maps from
 * pararnn_shard_eval to pararnn_shard_apply of the same iteration. */
size_t pararnn_shard_workspace_size(int cell, int B, int Ts, int D);
/* In:  u, a, bias as for the solves (u a shard's slice); c_bound, h_bound
 *      [B][D] the states before the shard's first step (NULL = zeros); c, h
 *      [B][Ts][D] the shard's iterate (not changed).
 * Out: agg [NA][B][D] the shard's map, NA = 2 (ParaGRU: P, d) or 6
 *      (ParaLSTM: P00, P01, P10, P11, d0, d1 for the state order c, h);
 *      last [S][B][D] the iterate's last state(s), S = 1 (h) or 2 (c, h);
 *      *rmax (device float) max|r| over the shard (NaN if any is NaN).
 * Alignment 4 bytes (u: 2 for bf16), workspace 256. */
int pararnn_shard_eval(int cell, const void* u, int u_dtype, const float* a,
                       const float* bias, const float* c_bound,
                       const float* h_bound, const float* c, const float* h,
                       int B, int Ts, int D, float* agg, float* last,
                       float* rmax, void* workspace, size_t ws_bytes,
                       pararnn_stream_t stream);
/* In:  aggs [W][NA][B][D] and lasts [W][S][B][D], every shard's agg and last
 *      in shard order; r this shard's index.
 * Out: din [S][B][D] the delta entering shard r; for r > 0, bound [S][B][D]
 *      its initial state for the next iteration (bound may be NULL for r = 0,
 *      whose initial state is the true one). */
int pararnn_shard_combine(int cell, const float* aggs, const float* lasts,
                          int W, int r, int B, int D, float* din, float* bound,
                          pararnn_stream_t stream);
/* Adds the Newton update to the shard's iterate c, h [B][Ts][D] (c NULL for
 * ParaGRU), given din from pararnn_shard_combine and the workspace of this
 * iteration's pararnn_shard_eval. */
int pararnn_shard_apply(int cell, const float* din, float* c, float* h, int B,
                        int Ts, int D, void* workspace, size_t ws_bytes,
                        pararnn_stream_t stream);

/* One recurrence step, for autoregressive decoding.  Generating a token
 * costs one update of the hidden state whatever the context length
 * ("Apple научила классические RNN масштабироваться...", "Инференс быстрее и
 * стабильнее по длине контекста", Figure 8); this applies the cell of
 * pararnn_gru_solve once to a batch of states.
 * In:  u_t [B][3][D] (the step's z, r, c projections; dtype u_dtype), a [3][D],
 *      bias [3][D] or NULL (zeros), h_prev [B][D] or NULL (zeros).
 * Out: h_next [B][D].  h_next may be h_prev itself (in-place update: every
 *      element is read before it is written); other overlaps are not allowed.
 * D must be a multiple of 8, as for the solves.  Stream-ordered, no
 * workspace, no synchronisation.  Returns PARARNN_ERR_INVALID_ARG /
 * _UNSUPPORTED_DTYPE / _MISALIGNED (4 B for float arrays, 2 B for bf16 u_t)
 * without launching, PARARNN_ERR_CUDA if the launch fails. */
int pararnn_gru_step(const void* u_t, int u_dtype, const float* a,
                     const float* bias, const float* h_prev, float* h_next,
                     int B, int D, pararnn_stream_t stream);

/* ParaLSTM step: u_t [B][4][D] (i, f, g, o), a/bias [4][D], c_prev/h_prev
 * [B][D] or NULL (zeros) -> c_next, h_next [B][D].  c_next and h_next must
 * be distinct; each may be the matching *_prev array (in-place update). */
int pararnn_lstm_step(const void* u_t, int u_dtype, const float* a,
                      const float* bias, const float* c_prev,
                      const float* h_prev, float* c_next, float* h_next,
                      int B, int D, pararnn_stream_t stream);

/* Human-readable text for a return code. */
const char* pararnn_strerror(int code);

#ifdef __cplusplus
}
#endif
#endif /* PARARNN_H */
