// Group dequantization of the frozen base weight to bf16 for the tensor cores.
//   W_Q[i][k] = scales[i][k/group] * (q[i][k] - zeros[i][k/group])   (fp32)
// rounded once to bf16. q[i][k] is bits [b*k, b*k+b) of row i's little-endian
// bit stream. Eight consecutive codes share a group (group % 8 == 0) and span
// exactly b bytes, so a thread dequantizes one 8-code run from b byte loads.
// out[i][k] is [d_out, d_in]: the K-major B operand of Y = X W_Q^T and, read
// MN-major, the B operand of dX = dY W_Q.

#include <algorithm>

#include "common.cuh"
#include "kernels.h"

namespace qwha {
namespace {

__device__ __forceinline__ void dequant8(const uint8_t *__restrict__ row, int bits, int k0, float s, float z,
                                         float *o) {
  const uint8_t *p = row + (int64_t)k0 * bits / 8;
  uint32_t w = 0;
  for (int b = 0; b < bits; ++b) w |= (uint32_t)p[b] << (8 * b);
  const uint32_t mask = (1u << bits) - 1u;
#pragma unroll
  for (int i = 0; i < 8; ++i) o[i] = s * ((float)((w >> (bits * i)) & mask) - z);
}

__global__ void dequant_kernel(const uint8_t *__restrict__ qw, const float *__restrict__ scales,
                               const uint8_t *__restrict__ zeros, int bits, int group, int d_out, int d_in,
                               __nv_bfloat16 *__restrict__ out) {
  const int64_t runs_per_row = d_in / 8;
  const int64_t total = (int64_t)d_out * runs_per_row;
  const int64_t row_bytes = (int64_t)d_in * bits / 8;
  const int ng = d_in / group;
  for (int64_t r = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; r < total; r += (int64_t)gridDim.x * blockDim.x) {
    const int64_t i = r / runs_per_row;
    const int k0 = (int)(r % runs_per_row) * 8;
    const int g = k0 / group;
    float v[8];
    dequant8(qw + i * row_bytes, bits, k0, scales[i * ng + g], (float)zeros[i * ng + g], v);
    *reinterpret_cast<uint4 *>(out + i * d_in + k0) = io<__nv_bfloat16>::pack(v);
  }
}

}  // namespace

size_t wdeq_bytes(int32_t d_out, int32_t d_in) { return (size_t)d_out * d_in * 2; }

cudaError_t launch_dequant(int bits, int group, int32_t d_out, int32_t d_in, const uint8_t *qw, const float *scales,
                           const uint8_t *zeros, void *out, cudaStream_t s) {
  const int64_t total = (int64_t)d_out * (d_in / 8);
  const int64_t grid = std::min<int64_t>(cdiv(total, 256), (int64_t)sm_count() * 16);
  dequant_kernel<<<(unsigned)grid, 256, 0, s>>>(qw, scales, zeros, bits, group, d_out, d_in,
                                                static_cast<__nv_bfloat16 *>(out));
  return cudaGetLastError();
}

}  // namespace qwha
