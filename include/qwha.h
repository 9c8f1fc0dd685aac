/*
 * qwha.h -- C ABI of the B200 (sm_100a) implementation of the Walsh-Hadamard
 * adapter (WHA) layer on a group-quantized linear layer.
 *
 * The layer, after "QWHA: Quantization-Aware Walsh-Hadamard Adaptation for
 * Parameter-Efficient Fine-Tuning on Large Language Models" (papernotes.org,
 * section 整体框架 and 关键设计 1; gist.science, section 2.1 Adapter Design):
 *
 *     Y = X W_Q^T + alpha * X (F H^-1)^T
 *
 * W_Q is the frozen quantized base weight [d_out, d_in]; H is the frozen
 * Walsh-Hadamard matrix over d_in; F = Scatter(c, E) is a sparse [d_out, d_in]
 * matrix with p nonzeros whose values c are the only trained parameters.
 * This library takes H to be the Sylvester-ordered matrix normalised to be
 * orthonormal, H_n[i][j] = (-1)^popcount(i & j) / sqrt(n), so H^-1 = H = H^T;
 * when d_in is not a power of two, H is block-diagonal with d_in / had_block
 * equal blocks H_had_block. Then
 *
 *     Z    = X H                               (fast transform, no multiply)
 *     Y    = X W_Q^T + alpha * Z F^T           (forward)
 *     dc_j = alpha * sum_t dY[t, r_j] Z[t, k_j]  (backward, E = {(r_j, k_j)})
 *     dX   = dY W_Q + alpha * (dY F) H
 *
 * Conventions for every call:
 *   - Matrices are dense, row-major, with no padding between rows.
 *   - Pointers named d_* or documented as "device" are CUDA device pointers;
 *     the library reads them on `stream` and never frees or keeps them.
 *   - `stream` is a cudaStream_t (NULL = the legacy default stream). Every call
 *     only enqueues work on it and returns without synchronising, except
 *     qwha_validate_plan and qwha_check_stream_status, which synchronise it.
 *   - Device buffers must be 16-byte aligned (QWHA_ERR_MISALIGNED otherwise).
 *   - The caller owns all memory. Calls that need scratch take `ws` (device,
 *     256-byte aligned) and `ws_bytes`; qwha_workspace_size gives the need.
 *   - Errors are returned as qwha_status; nothing is thrown across the ABI.
 *     qwha_last_error() gives a message for the last failing call of the
 *     calling thread. Arguments are checked on the host before any launch; a
 *     failed check launches nothing.
 */
#ifndef QWHA_H
#define QWHA_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  QWHA_OK = 0,
  QWHA_ERR_INVALID_ARG = 1, /* a shape, size, pointer or enum value is out of range */
  QWHA_ERR_MISALIGNED = 2,  /* a device buffer is not 16-byte aligned */
  QWHA_ERR_UNSUPPORTED = 3, /* a valid combination this build does not implement */
  QWHA_ERR_WORKSPACE = 4,   /* ws is NULL or ws_bytes is below qwha_workspace_size */
  QWHA_ERR_CUDA = 5,        /* a CUDA runtime call or launch failed */
  QWHA_ERR_TIMEOUT = 6      /* a bounded device-side wait gave up (see qwha_check_stream_status) */
} qwha_status;

typedef enum { QWHA_F32 = 0, QWHA_BF16 = 1 } qwha_dtype;

/* Where the rounding remainder of the AdaAlloc budget goes: one extra
 * coefficient each to the least-allocated channels (the rule the pages state,
 * papernotes.org 关键设计 2) or to the channels of largest error. */
typedef enum { QWHA_REM_FEWEST_ALLOC = 0, QWHA_REM_LARGEST_ERROR = 1 } qwha_remainder;

/* How qwha_adapter_fwd/bwd compute the adapter terms. Both give the same
 * results up to rounding order.
 *   QWHA_ALGO_SPARSE: the sparse kernels on the FMA units -- the product
 *     Z F^T over the CSR rows, the coefficient gradient over the tile view,
 *     the transposed gather over the CSC view -- with the adapter terms added
 *     in fp32 in the base GEMM's epilogue. Any dtype.
 *   QWHA_ALGO_DENSE: the adapter folded into the tensor-core GEMMs.
 *     W_eff = W_Q + alpha F H is built in bf16 (one transform of F's rows),
 *     Y = X W_eff^T and dX = dY W_eff are single GEMMs, and dc is gathered at
 *     E from the dense G = dY^T Z (fp32). bf16 only. */
typedef enum { QWHA_ALGO_SPARSE = 0, QWHA_ALGO_DENSE = 1 } qwha_algo;

/* Edge of the square blocks of F into which the coefficient-gradient kernel
 * tiles the nonzeros (the tile view built by qwha_plan_build). */
#define QWHA_TILE 256

/* The sparse coefficient matrix F = Scatter(c, E) and its index views. All
 * arrays are device memory owned by the caller.
 *   row_ptr [d_out+1], col_idx [p], coef [p]: CSR by output channel; within a
 *       row col_idx is strictly increasing (qwha_init_alloc writes this form).
 *   col_ptr [d_in+1], row_idx [p], perm [p]: CSC view; for column k the
 *       nonzeros in increasing CSR position; perm[q] is the CSR position of CSC
 *       entry q and row_idx[q] its row.
 *   tile_ptr [n_tiles+1], tile_pos [p], tile_rk [p]: the nonzeros grouped by
 *       QWHA_TILE x QWHA_TILE block of F (block (rb, kb) has id
 *       kb * ceil(d_out/QWHA_TILE) + rb), in CSC order inside a block;
 *       tile_pos is the CSR position, tile_rk packs (r mod QWHA_TILE) << 16 |
 *       (k mod QWHA_TILE).
 * The views are written by qwha_plan_build and depend on E only; the forward
 * needs the CSR arrays only; the sparse backward needs all three views, the
 * dense backward the CSR arrays only. */
typedef struct {
  int32_t d_in, d_out, had_block;
  int32_t algo; /* qwha_algo; 0 (sparse) for a zero-initialised struct */
  int64_t p;
  const int32_t *row_ptr, *col_idx;
  const float *coef;
  const int32_t *col_ptr, *row_idx, *perm;
  const int32_t *tile_ptr, *tile_pos, *tile_rk;
  /* Optional (dense algorithm): bf16 [d_out, d_in] device buffer for
   * W_eff = W_Q + alpha F H. When set, qwha_adapter_fwd writes W_eff there and
   * qwha_adapter_bwd reads it as it stands instead of rebuilding it, like a
   * tensor saved for the backward: the caller must run the forward after every
   * change of coef, the base weight or alpha. NULL: each call builds its own
   * copy in the workspace. */
  void *weff;
  /* Nonzero: Z_out of this forward call already holds X H for the same X and
   * had_block (written by the forward of another layer that reads the same
   * input, e.g. q, k and v of an attention block, or gate and up of an MLP);
   * the forward reads it instead of computing it. The backward is unaffected.
   * 0 (default): the forward computes Z_out. */
  int32_t z_given;
} qwha_adapter;

/* The frozen quantized base weight W_Q [d_out, d_in], device memory.
 * Code q[i][k] (0 <= q < 2^bits) is bits [bits*k, bits*k + bits) of row i's
 * little-endian bit stream, qweight holds d_out rows of d_in*bits/8 bytes;
 * W_Q[i][k] = scales[i][k/group] * (q[i][k] - zeros[i][k/group]) in fp32;
 * scales fp32 and zeros u8 are [d_out, d_in/group]. bits in {2, 3, 4}; group a
 * multiple of 8 that divides d_in. The tensor cores consume W_Q rounded to
 * bf16. (The pages start from an already quantized model, papernotes.org
 * 整体框架; this format is the library's own.) */
typedef struct {
  int32_t bits, group;
  const uint8_t *qweight;
  const float *scales;
  const uint8_t *zeros;
} qwha_qweight;

/* Operations for qwha_workspace_size. */
typedef enum {
  QWHA_OP_FWD = 0,       /* qwha_adapter_fwd, algo sparse */
  QWHA_OP_BWD = 1,       /* qwha_adapter_bwd, algo sparse */
  QWHA_OP_INIT = 2,      /* qwha_init_alloc */
  QWHA_OP_PLAN = 3,      /* qwha_plan_build */
  QWHA_OP_FWD_DENSE = 4, /* qwha_adapter_fwd, algo dense */
  QWHA_OP_BWD_DENSE = 5, /* qwha_adapter_bwd, algo dense */
  QWHA_OP_SELECT_GLOBAL = 6, /* qwha_init_select_global */
  QWHA_OP_REFINE = 7,        /* qwha_refine_values */
  QWHA_OP_ENERGY = 8,        /* qwha_energy_stats */
  QWHA_OP_PATTERN = 9        /* qwha_pattern_stats */
} qwha_op;

/* Z = X H row by row: x and z are [rows, n] of dtype dt (device), each row
 * transformed by the block-diagonal orthonormal Hadamard matrix with blocks
 * of had_block. had_block is a power of two in [2, 32768] dividing n; x and z
 * must not overlap. Arithmetic in fp32.
 * (papernotes.org 关键设计 1 and gist.science 2.1: the +-1 kernel turns the
 * transform into a recursion of sums and differences.) */
qwha_status qwha_fwht(qwha_dtype dt, const void *x, void *z, int64_t rows, int32_t n,
                      int32_t had_block, void *stream);

/* Forward of the adapted layer (gist.science 2.1; papernotes.org 整体框架):
 *   Z_out = X H                 [T, d_in], dtype dt (kept for the backward)
 *   Y     = X W_Q^T + alpha Z F^T  [T, d_out], dtype dt
 * wq == NULL computes the adapter alone (Y = alpha Z F^T). With wq, or with
 * a->algo == QWHA_ALGO_DENSE, dt must be QWHA_BF16. X, Z_out, Y are device
 * buffers; a->row_ptr/col_idx/coef are required, the other views are not
 * read. T >= 0 (T = 0 does nothing). ws: qwha_workspace_size(QWHA_OP_FWD,
 * ...) bytes for the sparse algorithm (it holds the entries of E in the order
 * the SpMM reads them, 8 bytes each with the padding of the groups of
 * segments, the segments' ranking by length, and with wq the fp32 adapter
 * term and the dequantized weight), QWHA_OP_FWD_DENSE for the dense one
 * (W_eff, unless a->weff is given). */
qwha_status qwha_adapter_fwd(const qwha_adapter *a, const qwha_qweight *wq, qwha_dtype dt,
                             const void *X, int64_t T, float alpha, void *Z_out, void *Y,
                             void *ws, size_t ws_bytes, void *stream);

/* Backward with only c trained (papernotes.org 整体框架 and 训练策略):
 *   dc[j] = alpha * sum_t dY[t, r_j] Z[t, k_j]   fp32 [p], CSR order
 *   dX    = dY W_Q + alpha (dY F) H              [T, d_in], dtype dt
 * Z is the Z_out of the matching forward. dc is overwritten (not accumulated).
 * The sparse algorithm needs all views of `a` (qwha_plan_build). dX may be
 * NULL to skip it, and dc may be NULL to skip the coefficient gradient (a
 * data-parallel caller computes dc first, starts its all-reduce, then dX; the
 * results are the same as from one call). Every reduction runs in a fixed
 * order: results are bitwise reproducible. ws: qwha_workspace_size(QWHA_OP_BWD
 * or QWHA_OP_BWD_DENSE, ...) bytes (for the sparse algorithm: the partial sums
 * of dc, the transposed dY and Z of the coefficient gradient, which dZ reuses
 * afterwards, and the gather's entries). */
qwha_status qwha_adapter_bwd(const qwha_adapter *a, const qwha_qweight *wq, qwha_dtype dt,
                             const void *dY, const void *Z, int64_t T, float alpha, float *dc,
                             void *dX, void *ws, size_t ws_bytes, void *stream);

/* AdaAlloc initialisation from the quantization error dW_Q = W0 - W_Q
 * (papernotes.org 关键设计 2 and 3; gist.science 2.2). dWq fp32 [d_out, d_in]
 * device. Per channel i:
 *   e_i = ||dWq[i,:]||_2 (fp64 squares, pairwise sum in index order);
 *   budget_i = min_per_row + floor(pool * e_i / sum e), pool = p -
 *       min_per_row * d_out; a channel above d_in is capped and the others
 *       re-share the rest; the remainder p - sum(budget) goes one each in the
 *       order given by `mode`;
 *   V = dWq[i,:] H_unnormalised (fp64 butterflies, stages h = 1, 2, 4, ...);
 *   E row i = the budget_i largest |V| (ties to the lower index), ascending;
 *   c = float(V * 1/sqrt(had_block)) (the dense solution values).
 * Outputs (device): budgets [d_out], row_ptr [d_out+1], col_idx [p], coef [p].
 * Requires min_per_row*d_out <= p <= d_in*d_out, p < 2^31, d_in <= 16384.
 * Budgets and E are bitwise deterministic. */
qwha_status qwha_init_alloc(const float *dWq, int32_t d_out, int32_t d_in, int32_t had_block,
                            int64_t p, int32_t min_per_row, qwha_remainder mode,
                            int32_t *budgets, int32_t *row_ptr, int32_t *col_idx, float *coef,
                            void *ws, size_t ws_bytes, void *stream);

/* The three steps of qwha_init_alloc as separate calls, for AdaAlloc sharded
 * by output rows over data-parallel ranks: each rank computes the norms of its
 * rows (qwha_init_norms), the ranks exchange them so that every rank holds all
 * d_out norms, every rank computes the same budgets from them
 * (qwha_init_budgets; bitwise identical, as the norms are), each rank selects
 * E and c for its rows (qwha_init_select), and the ranks exchange their CSR
 * slices. Run over all rows in one process, the three calls give bit for bit
 * the outputs of qwha_init_alloc. Same requirements as qwha_init_alloc; all
 * pointers are device memory. */
/* e[i] = ||dWq[i,:]||_2 for the `rows` rows of dWq [rows, d_in] fp32 (fp64
 * squares, pairwise sum in index order); e fp64 [rows]. */
qwha_status qwha_init_norms(const float *dWq, int32_t rows, int32_t d_in, double *e, void *stream);
/* budgets [d_out] and row_ptr [d_out+1] from all d_out norms e (fp64) by the
 * rule of qwha_init_alloc. ws: qwha_workspace_size(QWHA_OP_INIT, ...) bytes. */
qwha_status qwha_init_budgets(const double *e, int32_t d_out, int32_t d_in, int64_t p,
                              int32_t min_per_row, qwha_remainder mode, int32_t *budgets,
                              int32_t *row_ptr, void *ws, size_t ws_bytes, void *stream);
/* E and c of `rows` consecutive rows: dWq [rows, d_in] fp32 holds those rows,
 * budgets [rows] and row_ptr [rows+1] are the matching slices of the global
 * budgets and row_ptr (row_ptr need not start at 0). Row i's entries go to
 * col_idx / coef [row_ptr[i] - row_ptr[0], + budgets[i]); p_local =
 * row_ptr[rows] - row_ptr[0] is the capacity of col_idx and coef. */
qwha_status qwha_init_select(const float *dWq, int32_t rows, int32_t d_in, int32_t had_block,
                             const int32_t *budgets, const int32_t *row_ptr, int64_t p_local,
                             int32_t *col_idx, float *coef, void *stream);

/* Selection rules the pages compare AdaAlloc with (papernotes.org 消融实验,
 * table 4; gist.science 2.2 notes that they may crowd the parameters into a few
 * channels): E is chosen over the whole d_out x d_in matrix, not per channel. */
typedef enum {
  QWHA_SEL_MAGNITUDE = 0, /* the p largest |V|, V = dWq H_unnormalised as in qwha_init_alloc */
  QWHA_SEL_RANDOM = 1     /* p positions uniformly at random (seeded) */
} qwha_selection;

/* E and c by a whole-matrix rule. Flat index j = i * d_in + k; key_j is the
 * magnitude (largest |V| first) or, for QWHA_SEL_RANDOM, output j + 1 of the
 * SplitMix64 generator seeded with `seed` (smallest first); E = the p first
 * keys, equal keys in increasing j; c = float(V * 1/sqrt(had_block)) at E
 * (the dense solution). Outputs (device) as qwha_init_alloc: budgets [d_out]
 * (E's count per row, no minimum), row_ptr [d_out+1], col_idx [p] ascending
 * within a row, coef [p]. Requires 0 <= p <= d_in*d_out, p < 2^31,
 * d_in <= 16384; ws: qwha_workspace_size(QWHA_OP_SELECT_GLOBAL, ...) bytes
 * (V in fp64 for every entry, plus a few arrays of d_out). Deterministic. */
qwha_status qwha_init_select_global(const float *dWq, int32_t d_out, int32_t d_in, int32_t had_block,
                                    int64_t p, qwha_selection sel, uint64_t seed, int32_t *budgets,
                                    int32_t *row_ptr, int32_t *col_idx, float *coef, void *ws,
                                    size_t ws_bytes, void *stream);

/* Selection diagnostics: the two measurements the pages use to argue for
 * the WHT and for AdaAlloc (papernotes.org 关键设计 1 and 2; gist.science
 * 2.2). Both compute what the pages describe rather than a step of the
 * training path.
 *
 * qwha_energy_stats: energy concentration of the transform coefficients of
 * the quantization error. The pages fit the coefficient magnitudes with a
 * Pareto law and compare transforms by its Hill exponent eta (the smaller,
 * the steeper the tail and the more error energy a fixed number of
 * coefficients reconstructs); they give no formula, and this library takes
 * Hill's estimate over the k largest magnitudes a = |V|, V = dWq
 * H_unnormalised (fp64, as in qwha_init_alloc), sorted a_(1) >= a_(2) >= ...:
 *   xi = (1/k) sum_{i=1..k} ln(a_(i) / a_(k+1)),  eta = 1 / xi.
 * stats (device fp64 [4]): [0] eta (NaN when a_(k+1) = 0 or xi = 0), [1] the
 * fraction of sum a^2 held by the k largest (the cumulative energy at k; NaN
 * for an all-zero dWq), [2] a_(k+1) (unnormalised), [3] sum a^2
 * (= had_block * ||dWq||_F^2). dWq fp32 [d_out, d_in]; 1 <= k < d_out * d_in,
 * k < 2^31, d_in <= 16384. ws: qwha_workspace_size(QWHA_OP_ENERGY, d_out,
 * d_in, 0, 0, 0) bytes. Deterministic: a fixed-order reduction.
 *
 * qwha_pattern_stats: how E spreads over rows and columns. F is full rank with
 * high probability once rows and columns average more than two entries, and
 * an empty row or column cannot add to rank(F); a whole-matrix magnitude
 * selection crowds the entries into a few channels. From the CSR row_ptr
 * [d_out+1] and col_idx [p] (device) it writes col_counts (device int32
 * [d_in], entries per column) and stats (device int64 [8]): [0] rows without
 * entries, [1] columns without entries, [2] fewest entries in a row, [3] most
 * in a row, [4] fewest in a column, [5] most in a column, [6] min(d_out - [0],
 * d_in - [1]), an upper bound on rank(F), [7] the fewest rows that together
 * hold at least ceil(p / 2) entries. Entries with col_idx outside [0, d_in)
 * are not counted. ws: qwha_workspace_size(QWHA_OP_PATTERN, d_out, d_in, p,
 * 0, 0) bytes. Exact (integer arithmetic). */
qwha_status qwha_energy_stats(const float *dWq, int32_t d_out, int32_t d_in, int32_t had_block, int64_t k,
                              double *stats, void *ws, size_t ws_bytes, void *stream);
qwha_status qwha_pattern_stats(int32_t d_out, int32_t d_in, int64_t p, const int32_t *row_ptr,
                               const int32_t *col_idx, int32_t *col_counts, int64_t *stats, void *ws,
                               size_t ws_bytes, void *stream);

/* Calibration Hessian for Value Refinement: S = X^T X, fp32 [d_in, d_in]
 * (device), from calibration rows X bf16 [T, d_in] (device, T >= 1, d_in a
 * multiple of 8), on the tensor cores with fp32 accumulation. */
qwha_status qwha_calib_hessian(const void *X, int64_t T, int32_t d_in, float *S, void *stream);

/* Value Refinement (papernotes.org 关键设计 3): for a fixed E (CSR row_ptr,
 * col_idx, p entries; e.g. from qwha_init_alloc) the values that minimise each
 * channel's layer-output error for the calibration Hessian S fp32
 * [d_in, d_in] (symmetric, from qwha_calib_hessian). The page keeps the
 * per-channel problem min ||v - x B'|| (v = dWq[i,:] R, B = H^-1 R,
 * R R^T = S) and loses its closed form; this is its least-squares solution
 *   c[E_i] = u_i[E_i] (G[E_i, E_i])^-1,  G = H S H,  u_i = dWq[i,:] S H,
 * with S first damped by damp * mean(diag S) (damp >= 0; G[E_i, E_i] must be
 * positive definite). With S = I it returns the dense solution of
 * qwha_init_alloc. dWq fp32 [d_out, d_in]; coef fp32 [p] written (device).
 * Channels with more than min(d_in, 1024) entries are not solved: their
 * coef become NaN and qwha_check_stream_status reports it.
 * ws: qwha_workspace_size(QWHA_OP_REFINE, ...) bytes. */
qwha_status qwha_refine_values(const float *dWq, int32_t d_out, int32_t d_in, int32_t had_block,
                               const float *S, float damp, const int32_t *row_ptr,
                               const int32_t *col_idx, int64_t p, float *coef, void *ws,
                               size_t ws_bytes, void *stream);

/* Index views of E for the backward (E stays fixed while c trains,
 * papernotes.org 整体框架): from the CSR row_ptr/col_idx (device) write the
 * CSC view (col_ptr [d_in+1], row_idx [p], perm [p]) and the tile view
 * (tile_ptr [qwha_plan_tiles(d_out, d_in) + 1], tile_pos [p], tile_rk [p]).
 * col_idx must be within [0, d_in); duplicates inside a row are not checked
 * here (qwha_validate_plan does). */
qwha_status qwha_plan_build(int32_t d_out, int32_t d_in, int64_t p, const int32_t *row_ptr,
                            const int32_t *col_idx, int32_t *col_ptr, int32_t *row_idx,
                            int32_t *perm, int32_t *tile_ptr, int32_t *tile_pos,
                            int32_t *tile_rk, void *ws, size_t ws_bytes, void *stream);

/* Size of the library's own static device scratch used by
 * qwha_coef_grad_noalloc (16 MiB, held on every GPU that loads the library
 * until the process exits). */
#define QWHA_NOALLOC_SCRATCH_BYTES (16u << 20)

/* The coefficient gradient dc of qwha_adapter_bwd, for callers that cannot
 * allocate device memory and cannot pass a workspace: for example a custom-op
 * slot of a host framework that hands the op only its inputs and outputs, or
 * a step that must not call cudaMalloc (it may synchronise the device and can
 * fail under a fixed memory budget). There is no counterpart on the pages; it
 * is an engineering variant of the backward's first stage.
 *   dc[j] = alpha * sum_t dY[t, r_j] Z[t, k_j]   fp32 [p], CSR order
 * Same arguments and result as the dc of qwha_adapter_bwd (tile view of `a`
 * required; dX is not computed). The partial sums live in one static array of
 * QWHA_NOALLOC_SCRATCH_BYTES inside the library: chunks x p x 4 bytes, where
 * the number of token chunks is chosen from T, the tile count and the
 * device's SM count (the q_proj layer, p = 524288 at 8192 tokens, takes 4
 * chunks, 8.4 MB, on a 148-SM B200). A call needing more returns
 * QWHA_ERR_WORKSPACE and launches nothing. Nothing is allocated. All calls on
 * a device share that array: calls whose work overlaps on the GPU race and
 * must be serialised by the caller; each call clears the partial sums it
 * uses. The first call in a CUDA context (for runtime users: the first call
 * on a device) looks up the array's device address with that context
 * current, so it must come before any stream capture; the lookup is cached
 * per context, so a context created later, e.g. after cudaDeviceReset, gets
 * a fresh one. The result is bit for bit the dc of qwha_adapter_bwd with the
 * sparse algorithm: for bf16 with 16-byte aligned rows that call feeds its
 * kernel with transposed copies of dY and Z kept in its workspace, while this
 * entry point stages and transposes the slices inside its kernel; the two
 * kernels share the multiply-add code, the tiles, chunks and summation order. */
qwha_status qwha_coef_grad_noalloc(const qwha_adapter *a, qwha_dtype dt, const void *dY, const void *Z,
                                   int64_t T, float alpha, float *dc, void *stream);

/* Number of QWHA_TILE x QWHA_TILE blocks of F. */
int64_t qwha_plan_tiles(int32_t d_out, int32_t d_in);

/* Scratch bytes a call needs (0 if none). T is the token count for FWD/BWD,
 * with_base is 1 when a qwha_qweight is passed. */
size_t qwha_workspace_size(qwha_op op, int32_t d_out, int32_t d_in, int64_t p, int64_t T,
                           int32_t with_base);

/* Check E and its views on the device: row_ptr non-decreasing from 0 to p,
 * col_idx in range and strictly increasing per row, and, if present, the CSC
 * and tile views consistent with it. Synchronises the stream.
 * QWHA_ERR_INVALID_ARG names the first failure in qwha_last_error(). */
qwha_status qwha_validate_plan(const qwha_adapter *a, void *stream);

/* Synchronise `stream` and report a device-side error word set by a bounded
 * wait (QWHA_ERR_TIMEOUT) or a CUDA error (QWHA_ERR_CUDA); clears the word. */
qwha_status qwha_check_stream_status(void *stream);

/* Tracing aid: per-stage device time of the library's own kernels. While
 * enabled (off by default), every stage a call runs (the kernels of one step
 * of the path, e.g. the forward transform or the base GEMM) is bracketed by a
 * pair of CUDA events recorded on the call's stream. qwha_stage_report waits
 * for those events and fills, for each stage i < qwha_stage_count(), the
 * number of stage executions calls[i], the kernels they launched launches[i]
 * and their total device time ms[i] since the previous report; then it
 * resets the counters. Arrays are host memory of qwha_stage_count() entries.
 * Not for use inside CUDA graph capture. */
void qwha_stage_timing(int32_t enable);
int32_t qwha_stage_count(void);
const char *qwha_stage_name(int32_t i);
qwha_status qwha_stage_report(int64_t *calls, int64_t *launches, double *ms);

/* Test and fault-injection hooks. They change process-wide state of the
 * library and exist so that the error paths can be exercised without a GPU
 * fault; production code does not call them.
 *
 * qwha_debug_wait_limit_ns sets the bound, in ns, of the main-loop waits of
 * the row-transform kernel (the bulk-copy ring that qwha_fwht and the sparse
 * algorithm's transforms run on) and returns the previous bound (default
 * 2000000000, i.e. 2 s). A wait that gives up sets the device error word and
 * its CTA exits after letting its own copies already in flight land (those
 * drain waits keep the fixed 2 s bound); the call's output is then incomplete
 * and qwha_check_stream_status reports QWHA_ERR_TIMEOUT. A bound of 0 makes
 * every such wait give up at once, without polling, so the give-up path runs
 * whatever the timing. Not thread-safe with respect to calls in flight on
 * other threads.
 *
 * qwha_debug_fail_cuda_checks(n) makes the next n checks of a successful CUDA
 * runtime result inside the library (launches, memsets, copies) report
 * QWHA_ERR_CUDA with "injected failure" in qwha_last_error(), as though that
 * call had failed; the work itself was enqueued. n <= 0 disarms it. */
uint64_t qwha_debug_wait_limit_ns(uint64_t ns);
void qwha_debug_fail_cuda_checks(int32_t n);

const char *qwha_status_string(qwha_status s);
const char *qwha_last_error(void);
const char *qwha_version(void);

#ifdef __cplusplus
}
#endif

#endif /* QWHA_H */
