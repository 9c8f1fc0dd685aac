// Internal launchers of libqwha (not part of the C ABI). Each enqueues its
// kernels on `s` and returns the launch status; argument checks live in api.cu.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "qwha.h"

namespace qwha {

// W_eff rows for Hadamard blocks of 2^logn, 7 <= logn <= 12 (fwht.cu).
bool weff_rows_supported(int logn);
cudaError_t launch_weff_rows(const int32_t *row_ptr, const int32_t *col_idx, const float *coef, int64_t p, int d_in,
                             int64_t n_rows, int logn, float scale, int bits, int group, const uint8_t *qw,
                             const float *scales, const uint8_t *zeros, void *out, cudaStream_t s);

// Transform `blocks` consecutive blocks of 2^logn elements; out = H_unnorm(in) * scale.
cudaError_t launch_fwht(qwha_dtype din, qwha_dtype dout, const void *x, void *z, int64_t blocks,
                        int logn, float scale, cudaStream_t s);

}  // namespace qwha

namespace qwha {

// Upper bound on the token chunks of the coefficient-gradient kernel (its
// partial sums take kSddmmMaxChunks * p floats of workspace at most).
constexpr int kSddmmMaxChunks = 16;

// out[t, i] = alpha * sum_{j in [seg_ptr[i], seg_ptr[i+1])} v_j * in[t, idx[j]], with
// v_j = val[perm[j]] when perm is given (the CSC view), else val[j]. scratch
// (256-byte aligned) holds the entries in the order the kernel reads them;
// spmm_scratch_bytes(nnz, n_seg, W_in) bytes always suffice. *launched (if
// given) receives the number of kernels enqueued.
size_t spmm_scratch_bytes(int64_t p, int n_seg, int W_in);
cudaError_t launch_seg_spmm(qwha_dtype din, qwha_dtype dout, const void *in, int64_t T, int W_in,
                            const int32_t *seg_ptr, const int32_t *idx, const float *val, const int32_t *perm,
                            int64_t nnz, int n_seg, float alpha, void *scratch, size_t scratch_bytes, void *out,
                            cudaStream_t s, int *launched = nullptr);

int sddmm_chunks(int64_t T, int32_t d_out, int32_t d_in);

// Bytes of the transposed copies of dY and Z that launch_sddmm can use (bf16).
size_t sddmm_transposed_bytes(int64_t T, int32_t d_out, int32_t d_in);

// dc[j] = alpha * sum_t dY[t, r_j] Z[t, k_j] through the tile view; partial is
// workspace of sddmm_chunks(...) * p floats. tscratch (16-byte aligned, at
// least sddmm_transposed_bytes(...)) lets bf16 inputs take the path that
// transposes dY and Z once and feeds the kernel by tensor copies; nullptr, or
// shapes that path does not take (fp32, d_out or d_in not a multiple of 8),
// keep the kernel that stages and transposes its own tiles. Both give
// bitwise the same dc. *launched (if given) receives the number of kernels
// enqueued.
cudaError_t launch_sddmm(qwha_dtype dt, const void *dY, const void *Z, int64_t T, int32_t d_out, int32_t d_in,
                         const int32_t *tile_ptr, const int32_t *tile_pos, const int32_t *tile_rk, int64_t p,
                         float alpha, float *partial, float *dc, cudaStream_t s, void *tscratch = nullptr,
                         int *launched = nullptr);

// A tensor map over a bf16 matrix of rows x cols with a row stride of ld
// elements (ld * 2 a multiple of 16, ptr 16-byte aligned), box box_cols x
// box_rows, no swizzle (gemm.cu).
bool make_map_rows(CUtensorMap *m, const void *ptr, int64_t rows, int64_t cols, int64_t ld, uint32_t box_cols,
                   uint32_t box_rows);

size_t plan_workspace(int32_t d_out, int32_t d_in);
int plan_max_row_blocks();
cudaError_t launch_plan_build(int32_t d_out, int32_t d_in, int64_t p, const int32_t *row_ptr,
                              const int32_t *col_idx, int32_t *col_ptr, int32_t *row_idx, int32_t *perm,
                              int32_t *tile_ptr, int32_t *tile_pos, int32_t *tile_rk, void *ws,
                              cudaStream_t s);

}  // namespace qwha

namespace qwha {

// AdaAlloc (init.cu)
size_t init_workspace(int32_t d_out, int32_t d_in);
int init_max_din();
// Value Refinement (refine.cu)
int refine_cap(int32_t d_in);
size_t refine_workspace(int32_t d_out, int32_t d_in);
cudaError_t launch_calib_hessian(const void *X, int64_t T, int32_t d_in, float *S, cudaStream_t s);
cudaError_t launch_refine(const float *dWq, int32_t d_out, int32_t d_in, int32_t had_block, const float *S,
                          float damp, const int32_t *row_ptr, const int32_t *col_idx, int64_t p, float *coef,
                          void *ws, cudaStream_t s);
size_t select_global_workspace(int32_t d_out, int32_t d_in);
cudaError_t launch_select_global(const float *dW, int32_t d_out, int32_t d_in, int32_t had_block, int64_t p, int sel,
                                 uint64_t seed, int32_t *budgets, int32_t *row_ptr, int32_t *col_idx, float *coef,
                                 void *ws, cudaStream_t s);
// Selection diagnostics (init.cu, diag.cu).
size_t energy_stats_workspace(int32_t d_out, int32_t d_in);
cudaError_t launch_energy_stats(const float *dW, int32_t d_out, int32_t d_in, int32_t had_block, int64_t k,
                                double *out, void *ws, cudaStream_t s);
size_t pattern_stats_workspace(int32_t d_in);
cudaError_t launch_pattern_stats(int32_t d_out, int32_t d_in, int64_t p, const int32_t *row_ptr,
                                 const int32_t *col_idx, int32_t *col_counts, int64_t *stats, void *ws,
                                 cudaStream_t s);
cudaError_t launch_init_norms(const float *dW, int32_t rows, int32_t d_in, double *e, cudaStream_t s);
cudaError_t launch_init_budgets(const double *e, int32_t d_out, int32_t d_in, int64_t p, int32_t min_per_row, int mode,
                                int32_t *budgets, int32_t *row_ptr, void *ws, cudaStream_t s);
cudaError_t launch_init_select(const float *dW, int32_t rows, int32_t d_in, int32_t had_block, const int32_t *budgets,
                               const int32_t *row_ptr, int64_t p, int32_t *col_idx, float *coef, cudaStream_t s);
cudaError_t launch_init_alloc(const float *dW, int32_t d_out, int32_t d_in, int32_t had_block, int64_t p,
                              int32_t min_per_row, int mode, int32_t *budgets, int32_t *row_ptr, int32_t *col_idx,
                              float *coef, void *ws, cudaStream_t s);

// Base weight (dequant.cu): bf16 W_Q [d_out, d_in].
size_t wdeq_bytes(int32_t d_out, int32_t d_in);
cudaError_t launch_dequant(int bits, int group, int32_t d_out, int32_t d_in, const uint8_t *qw, const float *scales,
                           const uint8_t *zeros, void *out, cudaStream_t s);

// Base GEMM with fp32 addend in the epilogue (gemm.cu).
cudaError_t launch_gemm_fwd(const void *X, const void *wdeq, const float *y_ad, void *Y, int64_t T, int32_t d_out,
                            int32_t d_in, cudaStream_t s);
// out[M, N] = A[M, K] B[N, K]^T (+ addend), A and B bf16 K-major, out fp32 or bf16.
cudaError_t launch_gemm_nt(const void *A, const void *B, const float *addend, void *out, bool f32_out, int64_t M,
                           int64_t N, int64_t K, cudaStream_t s);
// dc[j] = alpha * (A B^T)[r_j, col_idx[j]] for the CSR entries of E, written
// by the GEMM epilogue (no dense output).
// Forward GEMM Y = X W^T (bf16, K-major) whose launch also writes Z = X H
// (bf16, Hadamard blocks of 2^logn, times scale) from extra warps.
bool gemm_fused_fwht_supported(int64_t M, int logn);
cudaError_t launch_gemm_fwd_fused(const void *X, const void *W, void *Y, int64_t T, int32_t d_out, int32_t d_in,
                                  void *Z, int logn, float scale, cudaStream_t s);
cudaError_t launch_gemm_sampled(const void *A, bool a_mn, const void *B, bool b_mn, int64_t M, int64_t N, int64_t K,
                                const int32_t *row_ptr, const int32_t *col_idx, int64_t p, float alpha, float *dc,
                                cudaStream_t s);
// Same with either operand MN-major: A [K, M] when a_mn, B [K, N] when b_mn.
cudaError_t launch_gemm_any(const void *A, bool a_mn, const void *B, bool b_mn, const float *addend, void *out,
                            bool f32_out, int64_t M, int64_t N, int64_t K, cudaStream_t s);

// Device error word and plan validation (misc.cu).
cudaError_t read_and_clear_error_word(unsigned int *word, cudaStream_t s);
const char *validate_message(unsigned int code);
cudaError_t launch_validate(const qwha_adapter *a, cudaStream_t s, uint32_t *code, int64_t *where);

}  // namespace qwha

namespace qwha {

// Dense formulation (dense.cu).
size_t weff_smem(int32_t d_in);
// out = bf16(dequant(W_Q) + alpha * (F H)) [d_out, d_in]; wq may be NULL (adapter alone).
cudaError_t launch_weff(const qwha_adapter *a, const qwha_qweight *wq, float alpha, void *out, cudaStream_t s);

}  // namespace qwha
