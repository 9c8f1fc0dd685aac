// Group dequantization of the frozen base weight to bf16 for the tensor cores.
//   W_Q[i][k] = scales[i][k/group] * (q[i][k] - zeros[i][k/group])   (fp32)
// rounded once to bf16. q[i][k] is bits [b*k, b*k+b) of row i's little-endian
// bit stream. Eight consecutive codes share a group (group % 8 == 0) and span
// exactly b bytes, so a thread dequantizes one 8-code run from one word.
// out[i][k] is [d_out, d_in]: the K-major B operand of Y = X W_Q^T and, read
// MN-major, the B operand of dX = dY W_Q.

#include <algorithm>

#include "common.cuh"
#include "kernels.h"

namespace qwha {
namespace {

// The b bytes holding codes k0 .. k0+7 of a row (k0 a multiple of 8), as one
// little-endian word: a single aligned load for 2- and 4-bit codes.
__device__ __forceinline__ uint32_t code_word(const uint8_t *__restrict__ row, int bits, int k0) {
  const uint8_t *p = row + (k0 / 8) * bits;
  if (bits == 4) return *reinterpret_cast<const uint32_t *>(p);
  if (bits == 2) return *reinterpret_cast<const uint16_t *>(p);
  uint32_t w = 0;
  for (int b = 0; b < bits; ++b) w |= (uint32_t)p[b] << (8 * b);
  return w;
}

// Grid-stride over blocks of kRuns x 256 runs of 8 codes (a run never crosses
// a row: d_in is a multiple of 8). A thread issues the loads of its kRuns runs
// (code word, scale, zero point) before using any of them, so each thread keeps
// several independent DRAM requests in flight; stores are 16 bytes.
constexpr int kDeqThreads = 256;
constexpr int kRuns = 4;

__global__ void __launch_bounds__(kDeqThreads) dequant_kernel(const uint8_t *__restrict__ qw,
                                                              const float *__restrict__ scales,
                                                              const uint8_t *__restrict__ zeros, int bits, int group,
                                                              int d_out, int d_in, __nv_bfloat16 *__restrict__ out) {
  const int runs_per_row = d_in / 8;
  const int64_t total = (int64_t)d_out * runs_per_row;
  const int64_t row_bytes = (int64_t)d_in * bits / 8;
  const int ng = d_in / group;
  const uint32_t mask = (1u << bits) - 1u;
  for (int64_t base = (int64_t)blockIdx.x * kDeqThreads * kRuns; base < total;
       base += (int64_t)gridDim.x * kDeqThreads * kRuns) {
    uint32_t w[kRuns];
    float sc[kRuns], z[kRuns];
    int64_t off[kRuns];
#pragma unroll
    for (int u = 0; u < kRuns; ++u) {
      const int64_t r = base + u * kDeqThreads + threadIdx.x;
      off[u] = -1;
      w[u] = 0;
      sc[u] = 0.f;
      z[u] = 0.f;
      if (r < total) {
        const int i = (int)r / runs_per_row, k0 = ((int)r - i * runs_per_row) * 8;  // total < 2^31
        const int g = k0 / group;
        w[u] = code_word(qw + i * row_bytes, bits, k0);
        sc[u] = scales[(int64_t)i * ng + g];
        z[u] = (float)zeros[(int64_t)i * ng + g];
        off[u] = (int64_t)i * d_in + k0;
      }
    }
#pragma unroll
    for (int u = 0; u < kRuns; ++u) {
      if (off[u] < 0) continue;
      float v[8];
#pragma unroll
      for (int q = 0; q < 8; ++q) v[q] = sc[u] * ((float)((w[u] >> (bits * q)) & mask) - z[u]);
      *reinterpret_cast<uint4 *>(out + off[u]) = io<__nv_bfloat16>::pack(v);
    }
  }
}

}  // namespace

size_t wdeq_bytes(int32_t d_out, int32_t d_in) { return (size_t)d_out * d_in * 2; }

cudaError_t launch_dequant(int bits, int group, int32_t d_out, int32_t d_in, const uint8_t *qw, const float *scales,
                           const uint8_t *zeros, void *out, cudaStream_t s) {
  const int64_t total = (int64_t)d_out * (d_in / 8);
  if (total > 0x7fffffff) return cudaErrorInvalidValue;  // run indices are 32-bit
  const int64_t grid = std::min<int64_t>(cdiv(total, (int64_t)kDeqThreads * kRuns), (int64_t)sm_count() * 8);
  dequant_kernel<<<(unsigned)grid, kDeqThreads, 0, s>>>(qw, scales, zeros, bits, group, d_out, d_in,
                                                static_cast<__nv_bfloat16 *>(out));
  return cudaGetLastError();
}

}  // namespace qwha
