// Dense tensor-core formulation of the adapter (the same results as the
// sparse kernels, computed as dense contractions on tcgen05).
//
// Because H is fixed, the adapter's weight update dW = F H is a dense matrix
// that costs one transform of F's rows to build ("QWHA", papernotes.org
// 关键设计 1: the update is F times the inverse transform). Folding it into the
// base weight,
//     W_eff = W_Q + alpha * F H,
// makes the forward Y = X W_eff^T and the input gradient dX = dY W_eff plain
// GEMMs: the adapter costs nothing in either. The coefficient gradient is the
// sampled product dc_j = alpha * (dY^T Z)[r_j, k_j]: one dense GEMM over
// tokens whose epilogue keeps only the entries of E.
//
// Kernels here: weff_kernel (one CTA per row of W_eff: scatter the row of F
// into shared memory, fp32 butterflies per Hadamard block, add the dequantized
// base row, one bf16 rounding; used for Hadamard blocks outside 128..4096).
// Blocks of 128..4096 take the kernels in fwht.cu that share the transform's
// register layout (weff_ring_kernel for blocks of 2048 and 4096 with a base
// weight, weff_pipe_kernel and weff_rows_kernel otherwise). The GEMMs read
// dY, Z and W_eff as stored (MN-major operands), so nothing is transposed,
// and the coefficient gradient is written by the sampled epilogue of the
// dY^T Z GEMM (gemm.cu), so G never reaches memory.

#include <algorithm>

#include "common.cuh"
#include "kernels.h"

namespace qwha {
namespace {

constexpr int kWeffThreads = 512;

__global__ void __launch_bounds__(kWeffThreads)
    weff_kernel(const int32_t *__restrict__ row_ptr, const int32_t *__restrict__ col_idx,
                const float *__restrict__ coef, int64_t p, int d_in, int logn, float scale, int bits, int group,
                const uint8_t *__restrict__ qw, const float *__restrict__ scales, const uint8_t *__restrict__ zeros,
                __nv_bfloat16 *__restrict__ out) {
  extern __shared__ __align__(16) float row[];
  const int64_t r = blockIdx.x;
  for (int k = threadIdx.x; k < d_in; k += blockDim.x) row[k] = 0.f;
  __syncthreads();
  int64_t b = row_ptr[r], e = row_ptr[r + 1];
  if (b < 0) b = 0;
  if (e > p) e = p;
  for (int64_t j = b + threadIdx.x; j < e; j += blockDim.x) {
    const int k = col_idx[j];
    if ((unsigned)k < (unsigned)d_in) row[k] = coef[j];
  }
  __syncthreads();
  // butterflies on index bits [0, logn): per block of 2^logn, three stages per pass
  butterflies_smem_f32(row, d_in, logn);
  // + dequantized base row, one rounding to bf16, 8 values per thread
  const int64_t row_bytes = (int64_t)d_in * bits / 8;
  const int ng = qw ? d_in / group : 0;
  for (int k0 = threadIdx.x * 8; k0 < d_in; k0 += blockDim.x * 8) {
    float f[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) f[i] = scale * row[k0 + i];
    if (qw) {
      const uint8_t *src = qw + r * row_bytes + (int64_t)k0 * bits / 8;
      uint32_t w = 0;
      for (int bb = 0; bb < bits; ++bb) w |= (uint32_t)src[bb] << (8 * bb);
      const uint32_t mask = (1u << bits) - 1u;
      const float sc = scales[r * ng + k0 / group], z = (float)zeros[r * ng + k0 / group];
#pragma unroll
      for (int i = 0; i < 8; ++i) f[i] += sc * ((float)((w >> (bits * i)) & mask) - z);
    }
    *reinterpret_cast<uint4 *>(out + r * d_in + k0) = io<__nv_bfloat16>::pack(f);
  }
}

}  // namespace

size_t weff_smem(int32_t d_in) { return (size_t)d_in * sizeof(float); }

cudaError_t launch_weff(const qwha_adapter *a, const qwha_qweight *wq, float alpha, void *out, cudaStream_t s) {
  const int logn = ilog2(a->had_block);
  const float scale = (float)(alpha / sqrt((double)a->had_block));
  if (weff_rows_supported(logn))
    return launch_weff_rows(a->row_ptr, a->col_idx, a->coef, a->p, a->d_in, a->d_out, logn, scale,
                            wq ? wq->bits : 0, wq ? wq->group : 1, wq ? wq->qweight : nullptr,
                            wq ? wq->scales : nullptr, wq ? wq->zeros : nullptr, out, s);
  const size_t smem = weff_smem(a->d_in);
  cudaError_t e = cudaFuncSetAttribute(weff_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  weff_kernel<<<a->d_out, kWeffThreads, smem, s>>>(a->row_ptr, a->col_idx, a->coef, a->p, a->d_in, logn, scale,
                                                   wq ? wq->bits : 0, wq ? wq->group : 1, wq ? wq->qweight : nullptr,
                                                   wq ? wq->scales : nullptr, wq ? wq->zeros : nullptr,
                                                   static_cast<__nv_bfloat16 *>(out));
  return cudaGetLastError();
}

}  // namespace qwha
