// Index views of the sparse pattern E (fixed while c trains: "QWHA",
// papernotes.org 整体框架): the CSC view used by the transposed gather of the
// backward, and the tile view used by the coefficient-gradient kernel.
//
// Both are stable counting sorts done without atomics in the placement step,
// so the output is bitwise deterministic:
//   CSC: rows are cut into chunks of kChunkRows; a per-(chunk, column)
//        histogram (atomics only count) is scanned down each column, then one
//        warp per chunk walks its rows in order and places the nonzeros (a
//        row's columns are distinct, so its lanes touch distinct counters).
//   tiles: one CTA per column block of QWHA_TILE columns partitions that
//        block's CSC range by row block with per-thread counts and a scan.
// Indices outside [0, d_in) are skipped (the result is then incomplete but no
// access leaves its buffer); qwha_validate_plan reports such input.

#include "common.cuh"
#include "kernels.h"

namespace qwha {
namespace {

constexpr int kChunkRows = 32;
constexpr int kTileThreads = 64;
constexpr int kMaxRowBlocks = 128;  // d_out <= 128 * QWHA_TILE

__global__ void chunk_hist_kernel(const int32_t *__restrict__ row_ptr, const int32_t *__restrict__ col_idx,
                                  int d_out, int d_in, int64_t p, int32_t *__restrict__ hist) {
  for (int64_t r = blockIdx.x * (int64_t)blockDim.y + threadIdx.y; r < d_out; r += (int64_t)gridDim.x * blockDim.y) {
    int64_t b = row_ptr[r], e = row_ptr[r + 1];
    if (b < 0) b = 0;
    if (e > p) e = p;
    int32_t *h = hist + (r / kChunkRows) * (int64_t)d_in;
    for (int64_t j = b + threadIdx.x; j < e; j += blockDim.x) {
      const int k = col_idx[j];
      if ((unsigned)k < (unsigned)d_in) atomicAdd(h + k, 1);
    }
  }
}

// Per column: exclusive scan of the chunk counts (in place) and the column total.
__global__ void column_scan_kernel(int32_t *__restrict__ hist, int n_chunks, int d_in, int32_t *__restrict__ total) {
  for (int k = blockIdx.x * blockDim.x + threadIdx.x; k < d_in; k += gridDim.x * blockDim.x) {
    int32_t run = 0;
    for (int c = 0; c < n_chunks; ++c) {
      int32_t *h = hist + (int64_t)c * d_in + k;
      const int32_t v = *h;
      *h = run;
      run += v;
    }
    total[k] = run;
  }
}

// out[0] = 0, out[i+1] = out[i] + in[i]; one CTA, any length.
__global__ void exclusive_scan_kernel(const int32_t *__restrict__ in, int n, int32_t *__restrict__ out) {
  __shared__ int32_t s[1024];
  __shared__ int32_t carry;
  if (threadIdx.x == 0) {
    carry = 0;
    out[0] = 0;
  }
  __syncthreads();
  for (int base = 0; base < n; base += 1024) {
    const int i = base + threadIdx.x;
    s[threadIdx.x] = i < n ? in[i] : 0;
    __syncthreads();
    for (int off = 1; off < 1024; off <<= 1) {
      const int32_t v = threadIdx.x >= off ? s[threadIdx.x - off] : 0;
      __syncthreads();
      s[threadIdx.x] += v;
      __syncthreads();
    }
    if (i < n) out[i + 1] = carry + s[threadIdx.x];
    __syncthreads();
    if (threadIdx.x == 1023) carry += s[1023];
    __syncthreads();
  }
}

__global__ void csc_place_kernel(const int32_t *__restrict__ row_ptr, const int32_t *__restrict__ col_idx,
                                 int d_out, int d_in, int64_t p, int32_t *__restrict__ hist,
                                 const int32_t *__restrict__ col_ptr, int32_t *__restrict__ row_idx,
                                 int32_t *__restrict__ perm) {
  const int warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  const int n_chunks = (d_out + kChunkRows - 1) / kChunkRows;
  if (warp >= n_chunks) return;
  int32_t *h = hist + (int64_t)warp * d_in;
  const int r_end = min(d_out, (warp + 1) * kChunkRows);
  for (int r = warp * kChunkRows; r < r_end; ++r) {
    int64_t b = row_ptr[r], e = row_ptr[r + 1];
    if (b < 0) b = 0;
    if (e > p) e = p;
    for (int64_t j = b + lane; j < e; j += 32) {
      const int k = col_idx[j];
      if ((unsigned)k >= (unsigned)d_in) continue;
      const int32_t pos = col_ptr[k] + h[k];
      h[k] += 1;
      if ((uint64_t)pos < (uint64_t)p) {
        row_idx[pos] = r;
        perm[pos] = (int32_t)j;
      }
    }
    __syncwarp();
  }
}

// One CTA per column block kb: stable partition of its CSC range by row block.
__global__ void __launch_bounds__(kTileThreads)
    tile_place_kernel(const int32_t *__restrict__ col_ptr, const int32_t *__restrict__ row_idx,
                      const int32_t *__restrict__ perm, const int32_t *__restrict__ col_idx, int d_out,
                      int d_in, int64_t p, int32_t *__restrict__ tile_ptr, int32_t *__restrict__ tile_pos,
                      int32_t *__restrict__ tile_rk) {
  __shared__ int32_t cnt[kMaxRowBlocks][kTileThreads + 1];
  __shared__ int32_t tile_start[kMaxRowBlocks];
  const int n_rb = (d_out + QWHA_TILE - 1) / QWHA_TILE;
  const int n_kb = (d_in + QWHA_TILE - 1) / QWHA_TILE;
  const int kb = blockIdx.x;
  const int k0 = kb * QWHA_TILE, k1 = min(d_in, k0 + QWHA_TILE);
  int64_t s0 = col_ptr[k0], s1 = col_ptr[k1];
  if (s0 < 0) s0 = 0;
  if (s1 > p) s1 = p;
  if (s1 < s0) s1 = s0;
  const int64_t len = s1 - s0;
  const int64_t per = (len + kTileThreads - 1) / kTileThreads;
  const int t = threadIdx.x;
  for (int rb = 0; rb < n_rb; ++rb) cnt[rb][t] = 0;
  const int64_t a = s0 + t * per, b = min(s1, a + per);
  for (int64_t q = a; q < b; ++q) {
    const int r = row_idx[q];
    if ((unsigned)r < (unsigned)d_out) cnt[r / QWHA_TILE][t]++;
  }
  __syncthreads();
  if (t < n_rb) {  // exclusive scan over threads for row block t
    int32_t run = 0;
    for (int i = 0; i < kTileThreads; ++i) {
      const int32_t v = cnt[t][i];
      cnt[t][i] = run;
      run += v;
    }
    cnt[t][kTileThreads] = run;
  }
  __syncthreads();
  if (t == 0) {
    int32_t run = (int32_t)s0;
    for (int rb = 0; rb < n_rb; ++rb) {
      tile_start[rb] = run;
      tile_ptr[kb * n_rb + rb] = run;
      run += cnt[rb][kTileThreads];
    }
    if (kb == n_kb - 1) tile_ptr[n_kb * n_rb] = run;
  }
  __syncthreads();
  int32_t local[kMaxRowBlocks];
  for (int rb = 0; rb < n_rb; ++rb) local[rb] = tile_start[rb] + cnt[rb][t];
  for (int64_t q = a; q < b; ++q) {
    const int r = row_idx[q];
    const int j = perm[q];
    if ((unsigned)r >= (unsigned)d_out || (uint64_t)j >= (uint64_t)p) continue;
    const int k = col_idx[j];
    const int32_t pos = local[r / QWHA_TILE]++;
    if ((uint64_t)pos < (uint64_t)p) {
      tile_pos[pos] = j;
      tile_rk[pos] = ((r % QWHA_TILE) << 16) | (k % QWHA_TILE);
    }
  }
}

}  // namespace

size_t plan_workspace(int32_t d_out, int32_t d_in) {
  const int64_t n_chunks = cdiv(d_out, kChunkRows);
  return align_up((size_t)n_chunks * d_in * 4, 256) + align_up((size_t)d_in * 4, 256);
}

int plan_max_row_blocks() { return kMaxRowBlocks; }

cudaError_t launch_plan_build(int32_t d_out, int32_t d_in, int64_t p, const int32_t *row_ptr,
                              const int32_t *col_idx, int32_t *col_ptr, int32_t *row_idx, int32_t *perm,
                              int32_t *tile_ptr, int32_t *tile_pos, int32_t *tile_rk, void *ws,
                              cudaStream_t s) {
  const int n_chunks = (int)cdiv(d_out, kChunkRows);
  int32_t *hist = static_cast<int32_t *>(ws);
  int32_t *total = reinterpret_cast<int32_t *>(static_cast<char *>(ws) +
                                               align_up((size_t)n_chunks * d_in * 4, 256));
  cudaError_t e = cudaMemsetAsync(hist, 0, (size_t)n_chunks * d_in * 4, s);
  if (e != cudaSuccess) return e;
  const int sm = sm_count();
  chunk_hist_kernel<<<sm * 4, dim3(32, 8), 0, s>>>(row_ptr, col_idx, d_out, d_in, p, hist);
  column_scan_kernel<<<(int)cdiv(d_in, 256), 256, 0, s>>>(hist, n_chunks, d_in, total);
  exclusive_scan_kernel<<<1, 1024, 0, s>>>(total, d_in, col_ptr);
  csc_place_kernel<<<(int)cdiv((int64_t)n_chunks * 32, 256), 256, 0, s>>>(row_ptr, col_idx, d_out, d_in, p,
                                                                            hist, col_ptr, row_idx, perm);
  const int n_kb = (int)cdiv(d_in, QWHA_TILE);
  tile_place_kernel<<<n_kb, kTileThreads, 0, s>>>(col_ptr, row_idx, perm, col_idx, d_out, d_in, p, tile_ptr,
                                                  tile_pos, tile_rk);
  return cudaGetLastError();
}

}  // namespace qwha
