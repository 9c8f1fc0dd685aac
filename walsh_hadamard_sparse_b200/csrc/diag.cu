// Selection diagnostics: row and column counts of E (the pages' rank argument
// for AdaAlloc: "QWHA", papernotes.org, 关键设计 1 and 2).
//
// An empty row or column of F = Scatter(c, E) cannot add to rank(F), so
// min(non-empty rows, non-empty columns) bounds the rank; the fewest rows that
// hold half of the entries shows how far a selection crowds the budget into a
// few channels. Every result is an integer computed with integer atomics and
// scans, so it is exact and independent of scheduling.

#include <limits.h>

#include <algorithm>

#include "common.cuh"
#include "kernels.h"

namespace qwha {
namespace {

constexpr int kDiagThreads = 256;
constexpr int kFinishThreads = 1024;

__global__ void __launch_bounds__(kDiagThreads) diag_clear_kernel(int32_t *__restrict__ col_counts, int d_in,
                                                                   int32_t *__restrict__ hist) {
  const int stride = gridDim.x * blockDim.x;
  for (int i = blockIdx.x * blockDim.x + threadIdx.x; i <= d_in; i += stride) {
    if (i < d_in) col_counts[i] = 0;
    hist[i] = 0;
  }
}

// hist[c] = number of rows with c entries (c clamped to [0, d_in]).
__global__ void __launch_bounds__(kDiagThreads) diag_rows_kernel(const int32_t *__restrict__ row_ptr, int d_out,
                                                                  int d_in, int32_t *__restrict__ hist) {
  const int stride = gridDim.x * blockDim.x;
  for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < d_out; i += stride) {
    int c = row_ptr[i + 1] - row_ptr[i];
    c = c < 0 ? 0 : (c > d_in ? d_in : c);
    atomicAdd(&hist[c], 1);
  }
}

// col_counts[k] = entries in column k (indices outside [0, d_in) are skipped).
__global__ void __launch_bounds__(kDiagThreads) diag_cols_kernel(const int32_t *__restrict__ col_idx, int64_t p,
                                                                  int d_in, int32_t *__restrict__ col_counts) {
  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  for (int64_t j = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; j < p; j += stride) {
    const int k = col_idx[j];
    if ((unsigned)k < (unsigned)d_in) atomicAdd(&col_counts[k], 1);
  }
}

// op over the block; `id` is op's identity (pads the slots of absent warps).
template <typename T, typename Op>
__device__ T block_reduce(T v, T *sh, Op op, T id) {
  const int t = threadIdx.x, lane = t & 31, nw = blockDim.x >> 5;
#pragma unroll
  for (int off = 16; off; off >>= 1) v = op(v, __shfl_xor_sync(0xffffffffu, v, off));
  if (lane == 0) sh[t >> 5] = v;
  __syncthreads();
  if (t < 32) {
    T x = t < nw ? sh[t] : id;
#pragma unroll
    for (int off = 16; off; off >>= 1) x = op(x, __shfl_xor_sync(0xffffffffu, x, off));
    if (t == 0) sh[32] = x;
  }
  __syncthreads();
  const T r = sh[32];
  __syncthreads();
  return r;
}

// Exclusive prefix of v over the block; *tot receives the total.
__device__ long long block_excl_scan(long long v, long long *sh, long long *tot) {
  const int t = threadIdx.x, lane = t & 31, nw = blockDim.x >> 5;
  long long incl = v;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const long long o = __shfl_up_sync(0xffffffffu, incl, off);
    if (lane >= off) incl += o;
  }
  if (lane == 31) sh[t >> 5] = incl;
  __syncthreads();
  if (t < 32) {
    long long w = t < nw ? sh[t] : 0;
    long long wi = w;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const long long o = __shfl_up_sync(0xffffffffu, wi, off);
      if (lane >= off) wi += o;
    }
    if (t < nw) sh[t] = wi - w;  // exclusive prefix of the warps' totals
    if (t == 31) sh[32] = wi;
  }
  __syncthreads();
  const long long r = sh[t >> 5] + incl - v;
  *tot = sh[32];
  __syncthreads();
  return r;
}

// One CTA: the eight statistics (see qwha_pattern_stats).
__global__ void __launch_bounds__(kFinishThreads)
    diag_finish_kernel(const int32_t *__restrict__ col_counts, const int32_t *__restrict__ hist, int d_out, int d_in,
                       int64_t p, int64_t *__restrict__ stats) {
  __shared__ long long shl[33];
  __shared__ int shi[33];
  const int t = threadIdx.x;
  auto add = [](long long a, long long b) { return a + b; };
  auto mn = [](int a, int b) { return a < b ? a : b; };
  auto mx = [](int a, int b) { return a > b ? a : b; };

  long long empty = 0;
  int cmin = INT_MAX, cmax = 0;
  for (int k = t; k < d_in; k += blockDim.x) {
    const int c = col_counts[k];
    empty += c == 0;
    cmin = c < cmin ? c : cmin;
    cmax = c > cmax ? c : cmax;
  }
  const long long empty_c = block_reduce(empty, shl, add, 0LL);
  cmin = block_reduce(cmin, shi, mn, INT_MAX);
  cmax = block_reduce(cmax, shi, mx, 0);

  int lo = INT_MAX, hi = -1;
  for (int b = t; b <= d_in; b += blockDim.x)
    if (hist[b]) {
      lo = b < lo ? b : lo;
      hi = b > hi ? b : hi;
    }
  lo = block_reduce(lo, shi, mn, INT_MAX);
  hi = block_reduce(hi, shi, mx, -1);

  // The fewest rows holding ceil(p / 2) entries: the histogram's bins from the
  // fullest down, in contiguous runs per thread, prefix sums of their entries
  // and rows; the thread whose run reaches the target finishes inside its run.
  const long long target = (p + 1) / 2;
  const int nbins = d_in + 1;
  const int chunk = (nbins + (int)blockDim.x - 1) / (int)blockDim.x;
  const int q0 = t * chunk, q1 = q0 + chunk < nbins ? q0 + chunk : nbins;
  long long ent = 0, rows = 0;
  for (int q = q0; q < q1; ++q) {
    const int b = d_in - q;
    ent += (long long)b * hist[b];
    rows += hist[b];
  }
  long long tot_e = 0, tot_r = 0;
  const long long ent0 = block_excl_scan(ent, shl, &tot_e);
  const long long rows0 = block_excl_scan(rows, shl, &tot_r);
  if (t == 0 && target == 0) stats[7] = 0;
  if (target > 0 && ent0 < target && ent0 + ent >= target) {
    long long cum = ent0, m = rows0;
    for (int q = q0; q < q1; ++q) {
      const int b = d_in - q;
      const long long h = hist[b];
      if (b > 0 && cum + (long long)b * h >= target) {
        m += (target - cum + b - 1) / b;
        break;
      }
      cum += (long long)b * h;
      m += h;
    }
    stats[7] = m;
  }
  if (t == 0) {
    const long long empty_r = hist[0];
    stats[0] = empty_r;
    stats[1] = empty_c;
    stats[2] = lo;
    stats[3] = hi;
    stats[4] = cmin;
    stats[5] = cmax;
    const long long nr = d_out - empty_r, nc = d_in - empty_c;
    stats[6] = nr < nc ? nr : nc;
  }
}

}  // namespace

size_t pattern_stats_workspace(int32_t d_in) { return align_up(((size_t)d_in + 1) * 4, 256); }

cudaError_t launch_pattern_stats(int32_t d_out, int32_t d_in, int64_t p, const int32_t *row_ptr,
                                 const int32_t *col_idx, int32_t *col_counts, int64_t *stats, void *ws,
                                 cudaStream_t s) {
  int32_t *hist = static_cast<int32_t *>(ws);
  const int cap = sm_count() * 8;
  auto grid = [&](int64_t n) { return (unsigned)std::max<int64_t>(1, std::min<int64_t>(cdiv(n, kDiagThreads), cap)); };
  diag_clear_kernel<<<grid(d_in + 1), kDiagThreads, 0, s>>>(col_counts, d_in, hist);
  diag_rows_kernel<<<grid(d_out), kDiagThreads, 0, s>>>(row_ptr, d_out, d_in, hist);
  if (p > 0) diag_cols_kernel<<<grid(p), kDiagThreads, 0, s>>>(col_idx, p, d_in, col_counts);
  diag_finish_kernel<<<1, kFinishThreads, 0, s>>>(col_counts, hist, d_out, d_in, p, stats);
  return cudaGetLastError();
}

}  // namespace qwha
