// Device error word for bounded waits, and the on-device check of E and its
// index views (qwha_validate_plan).

#include <cuda_runtime.h>

#include "common.cuh"
#include "kernels.h"

namespace qwha {

namespace {

__device__ unsigned int g_error_word;

struct ValidateResult {
  unsigned int code;
  unsigned int pad;
  long long where;
};
__device__ ValidateResult g_validate;

__device__ void report(unsigned int code, long long where) {
  if (atomicCAS(&g_validate.code, 0u, code) == 0u) g_validate.where = where;
}

// Row of CSR position j (row_ptr non-decreasing).
__device__ int row_of(const int32_t *row_ptr, int d_out, int64_t j) {
  int lo = 0, hi = d_out;  // row_ptr[lo] <= j < row_ptr[hi]
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (row_ptr[mid] <= j) lo = mid;
    else hi = mid;
  }
  return lo;
}

__global__ void validate_csr_kernel(const int32_t *__restrict__ row_ptr, const int32_t *__restrict__ col_idx,
                                    int d_out, int d_in, int64_t p) {
  const int64_t tid = blockIdx.x * (int64_t)blockDim.x + threadIdx.x, stride = (int64_t)gridDim.x * blockDim.x;
  if (tid == 0 && row_ptr[0] != 0) report(1, 0);
  if (tid == 0 && row_ptr[d_out] != p) report(2, d_out);
  for (int64_t r = tid; r < d_out; r += stride) {
    const int64_t b = row_ptr[r], e = row_ptr[r + 1];
    if (e < b || b < 0 || e > p) {
      report(3, r);
      continue;
    }
    for (int64_t j = b; j < e; ++j) {
      const int k = col_idx[j];
      if (k < 0 || k >= d_in) report(4, j);
      else if (j > b && col_idx[j - 1] >= k) report(5, j);
    }
  }
}

__global__ void validate_csc_kernel(const int32_t *__restrict__ row_ptr, const int32_t *__restrict__ col_idx,
                                    const int32_t *__restrict__ col_ptr, const int32_t *__restrict__ row_idx,
                                    const int32_t *__restrict__ perm, int d_out, int d_in, int64_t p) {
  const int64_t tid = blockIdx.x * (int64_t)blockDim.x + threadIdx.x, stride = (int64_t)gridDim.x * blockDim.x;
  if (tid == 0 && (col_ptr[0] != 0 || col_ptr[d_in] != p)) report(6, 0);
  for (int64_t k = tid; k < d_in; k += stride) {
    const int64_t b = col_ptr[k], e = col_ptr[k + 1];
    if (e < b || b < 0 || e > p) {
      report(6, k);
      continue;
    }
    for (int64_t q = b; q < e; ++q) {
      const int64_t j = perm[q];
      if (j < 0 || j >= p) {
        report(7, q);
        continue;
      }
      if (col_idx[j] != k) report(8, q);
      if (row_idx[q] != row_of(row_ptr, d_out, j)) report(9, q);
      if (q > b && perm[q - 1] >= j) report(10, q);
    }
  }
}

__global__ void validate_tile_kernel(const int32_t *__restrict__ row_ptr, const int32_t *__restrict__ col_idx,
                                     const int32_t *__restrict__ tile_ptr, const int32_t *__restrict__ tile_pos,
                                     const int32_t *__restrict__ tile_rk, int d_out, int d_in, int64_t p) {
  const int n_rb = (d_out + QWHA_TILE - 1) / QWHA_TILE, n_kb = (d_in + QWHA_TILE - 1) / QWHA_TILE;
  const int64_t n_tiles = (int64_t)n_rb * n_kb;
  const int64_t tid = blockIdx.x * (int64_t)blockDim.x + threadIdx.x, stride = (int64_t)gridDim.x * blockDim.x;
  if (tid == 0 && (tile_ptr[0] != 0 || tile_ptr[n_tiles] != p)) report(11, 0);
  for (int64_t t = tid; t < n_tiles; t += stride) {
    const int64_t b = tile_ptr[t], e = tile_ptr[t + 1];
    if (e < b || b < 0 || e > p) {
      report(11, t);
      continue;
    }
    const int rb = (int)(t % n_rb), kb = (int)(t / n_rb);
    for (int64_t q = b; q < e; ++q) {
      const int64_t j = tile_pos[q];
      if (j < 0 || j >= p) {
        report(12, q);
        continue;
      }
      const int r = row_of(row_ptr, d_out, j), k = col_idx[j];
      const int want = ((r % QWHA_TILE) << 16) | (k % QWHA_TILE);
      if (r / QWHA_TILE != rb || k / QWHA_TILE != kb || tile_rk[q] != want) report(13, q);
    }
  }
}

}  // namespace

unsigned int *device_error_word() {
  static unsigned int *ptrs[64] = {nullptr};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 0 || dev >= 64) return nullptr;
  if (!ptrs[dev]) {
    void *p = nullptr;
    if (cudaGetSymbolAddress(&p, g_error_word) != cudaSuccess) return nullptr;
    ptrs[dev] = static_cast<unsigned int *>(p);
  }
  return ptrs[dev];
}

cudaError_t read_and_clear_error_word(unsigned int *word, cudaStream_t s) {
  unsigned int *d = device_error_word();
  if (!d) return cudaErrorInvalidDevicePointer;
  cudaError_t e = cudaMemcpyAsync(word, d, sizeof(unsigned int), cudaMemcpyDeviceToHost, s);
  if (e == cudaSuccess) e = cudaStreamSynchronize(s);
  if (e == cudaSuccess) e = cudaMemsetAsync(d, 0, sizeof(unsigned int), s);
  if (e == cudaSuccess) e = cudaStreamSynchronize(s);
  return e;
}

const char *validate_message(unsigned int code) {
  switch (code) {
    case 1: return "row_ptr[0] != 0";
    case 2: return "row_ptr[d_out] != p";
    case 3: return "row_ptr decreases or leaves [0, p] at row";
    case 4: return "col_idx out of [0, d_in) at position";
    case 5: return "col_idx not strictly increasing within a row at position";
    case 6: return "col_ptr inconsistent at column";
    case 7: return "perm out of range at CSC entry";
    case 8: return "col_idx[perm[q]] differs from the column of CSC entry";
    case 9: return "row_idx differs from the row of perm at CSC entry";
    case 10: return "perm not increasing within a column at CSC entry";
    case 11: return "tile_ptr inconsistent at tile";
    case 12: return "tile_pos out of range at entry";
    case 13: return "tile entry outside its block or tile_rk wrong at entry";
  }
  return "unknown";
}

cudaError_t launch_validate(const qwha_adapter *a, cudaStream_t s, uint32_t *code, int64_t *where) {
  ValidateResult zero = {0, 0, 0};
  cudaError_t e = cudaMemcpyToSymbolAsync(g_validate, &zero, sizeof(zero), 0, cudaMemcpyHostToDevice, s);
  if (e != cudaSuccess) return e;
  const int sm = sm_count();
  validate_csr_kernel<<<sm * 2, 256, 0, s>>>(a->row_ptr, a->col_idx, a->d_out, a->d_in, a->p);
  ValidateResult r;
  e = cudaMemcpyFromSymbolAsync(&r, g_validate, sizeof(r), 0, cudaMemcpyDeviceToHost, s);
  if (e == cudaSuccess) e = cudaStreamSynchronize(s);
  if (e != cudaSuccess) return e;
  if (r.code == 0 && a->col_ptr && a->row_idx && a->perm) {
    validate_csc_kernel<<<sm * 2, 256, 0, s>>>(a->row_ptr, a->col_idx, a->col_ptr, a->row_idx, a->perm, a->d_out,
                                               a->d_in, a->p);
    e = cudaMemcpyFromSymbolAsync(&r, g_validate, sizeof(r), 0, cudaMemcpyDeviceToHost, s);
    if (e == cudaSuccess) e = cudaStreamSynchronize(s);
    if (e != cudaSuccess) return e;
  }
  if (r.code == 0 && a->tile_ptr && a->tile_pos && a->tile_rk) {
    validate_tile_kernel<<<sm * 2, 256, 0, s>>>(a->row_ptr, a->col_idx, a->tile_ptr, a->tile_pos, a->tile_rk,
                                                a->d_out, a->d_in, a->p);
    e = cudaMemcpyFromSymbolAsync(&r, g_validate, sizeof(r), 0, cudaMemcpyDeviceToHost, s);
    if (e == cudaSuccess) e = cudaStreamSynchronize(s);
    if (e != cudaSuccess) return e;
  }
  *code = r.code;
  *where = r.where;
  return cudaGetLastError();
}

}  // namespace qwha
