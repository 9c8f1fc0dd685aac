// Value Refinement ("QWHA", papernotes.org 关键设计 3): least-squares values of
// the coefficients at a fixed E for a calibration Hessian S = X^T X.
//
// For channel i the page states min_x ||v - x B'||^2 with v = dW_Q[i,:] R,
// B = H^-1 R, R R^T = S, x non-zero only at E_i. With H orthonormal and
// symmetric its least-squares solution is
//     x* = u_i[E_i] (G[E_i, E_i])^-1,   G = H S H,   u_i = dW_Q[i,:] S H,
// (x* = x0 = (dW_Q H)[i, E_i] when S = I). Steps on the device:
//   1. S is damped: S + damp * mean(diag S) * I (fp32).
//   2. G^T = ((S H)^T) H: the row transform, a tiled transpose, the row
//      transform again (G is symmetric; its transpose is read with the
//      indices swapped).
//   3. P = dW_Q S on the tensor cores with fp32-accurate products: both
//      operands split into bf16 high and low parts, P = Wh Sh + Wh Sl + Wl Sh
//      accumulated in fp32 (the dropped Wl Sl term is ~2^-16 relative), then
//      U = P H by the row transform.
//   4. One CTA per channel at a time (persistent, one CTA per SM): gather
//      G[E_i, E_i] in fp64 into the CTA's slab of global memory, blocked
//      Cholesky with 32 x 32 blocks staged in shared memory, the two
//      triangular solves, c = float(x*).

#include <algorithm>
#include <cmath>

#include "common.cuh"
#include "kernels.h"

namespace qwha {
namespace {

constexpr int kCholThreads = 256;
constexpr int kCB = 32;  // Cholesky block edge

__global__ void damp_kernel(const float *__restrict__ S, int d, float damp, float *__restrict__ out) {
  __shared__ double sh[1024];
  double t = 0;
  for (int k = threadIdx.x; k < d; k += blockDim.x) t += (double)S[(int64_t)k * d + k];
  sh[threadIdx.x] = t;
  __syncthreads();
  for (int w = blockDim.x / 2; w > 0; w >>= 1) {
    if ((int)threadIdx.x < w) sh[threadIdx.x] += sh[threadIdx.x + w];
    __syncthreads();
  }
  const float lam = (float)(damp * sh[0] / d);
  for (int k = threadIdx.x; k < d; k += blockDim.x) out[(int64_t)k * d + k] += lam;
}

__global__ void copy_f32_kernel(const float *__restrict__ a, float *__restrict__ b, int64_t n) {
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < n; i += (int64_t)gridDim.x * blockDim.x)
    b[i] = a[i];
}

// out [C, R] = in [R, C]^T, 32 x 32 tiles through shared memory.
__global__ void transpose_kernel(const float *__restrict__ in, int R, int C, float *__restrict__ out) {
  __shared__ float t[32][33];
  const int c0 = blockIdx.x * 32, r0 = blockIdx.y * 32;
  for (int y = threadIdx.y; y < 32; y += blockDim.y) {
    const int r = r0 + y, c = c0 + threadIdx.x;
    if (r < R && c < C) t[y][threadIdx.x] = in[(int64_t)r * C + c];
  }
  __syncthreads();
  for (int y = threadIdx.y; y < 32; y += blockDim.y) {
    const int c = c0 + y, r = r0 + threadIdx.x;
    if (r < R && c < C) out[(int64_t)c * R + r] = t[threadIdx.x][y];
  }
}

// x = hi + lo with hi = bf16(x), lo = bf16(x - hi).
__global__ void split_bf16_kernel(const float *__restrict__ x, int64_t n, __nv_bfloat16 *__restrict__ hi,
                                  __nv_bfloat16 *__restrict__ lo) {
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < n; i += (int64_t)gridDim.x * blockDim.x) {
    const float v = x[i];
    const __nv_bfloat16 h = __float2bfloat16_rn(v);
    hi[i] = h;
    lo[i] = __float2bfloat16_rn(v - __bfloat162float(h));
  }
}

// Per channel: M = G[E, E] (fp64, padded with the identity to a multiple of
// 32) in this CTA's slab, blocked Cholesky M = L L^T in place (lower), then
// L z = u[E], L^T x = z. Channels with more than `cap` entries get NaN and
// the error word.
__global__ void __launch_bounds__(kCholThreads, 1)
    refine_solve_kernel(const float *__restrict__ Gt, const float *__restrict__ U, int d_out, int d_in,
                        const int32_t *__restrict__ row_ptr, const int32_t *__restrict__ col_idx, int64_t p, int cap,
                        double *__restrict__ slabs, float *__restrict__ coef, unsigned int *err) {
  extern __shared__ __align__(16) double dsm[];
  double *rhs = dsm;                 // [cap]
  double *ta = rhs + cap;            // [32][33] block
  double *tb = ta + kCB * (kCB + 1);  // [32][33] block
  double *panel = tb + kCB * (kCB + 1);  // [kCholThreads][33]: one panel row per thread
  __shared__ int s_cols[1024];
  double *M = slabs + (int64_t)blockIdx.x * cap * cap;
  const int tid = threadIdx.x;
  for (int i = blockIdx.x; i < d_out; i += gridDim.x) {
    int64_t b0 = row_ptr[i], b1 = row_ptr[i + 1];
    if (b0 < 0) b0 = 0;
    if (b1 > p) b1 = p;
    const int m = (int)(b1 - b0);
    if (m <= 0) continue;
    if (m > cap) {
      for (int r = tid; r < m; r += blockDim.x) coef[b0 + r] = __int_as_float(0x7fc00000);
      if (tid == 0) atomicOr(err, 0x100u);
      continue;
    }
    const int mp = (m + kCB - 1) / kCB * kCB, nb = mp / kCB;
    __syncthreads();
    for (int r = tid; r < m; r += blockDim.x) {
      const int k = col_idx[b0 + r];
      s_cols[r] = (unsigned)k < (unsigned)d_in ? k : 0;
    }
    __syncthreads();
    // lower triangle of M and the right-hand side (G[a][b] = Gt[b][a])
    for (int64_t e = tid; e < (int64_t)mp * mp; e += blockDim.x) {
      const int r = (int)(e / mp), c = (int)(e % mp);
      if (c > r) continue;
      double v;
      if (r < m && c < m) v = (double)Gt[(int64_t)s_cols[c] * d_in + s_cols[r]];
      else v = r == c ? 1.0 : 0.0;
      M[(int64_t)r * mp + c] = v;
    }
    for (int r = tid; r < mp; r += blockDim.x) rhs[r] = r < m ? (double)U[(int64_t)i * d_in + s_cols[r]] : 0.0;
    __syncthreads();
    for (int k = 0; k < nb; ++k) {
      const int k0 = k * kCB;
      // 1. factor the diagonal block in shared memory (warp 0, lane = row)
      for (int e = tid; e < kCB * kCB; e += blockDim.x) {
        const int r = e / kCB, c = e % kCB;
        ta[r * (kCB + 1) + c] = c <= r ? M[(int64_t)(k0 + r) * mp + k0 + c] : 0.0;
      }
      __syncthreads();
      if (tid < 32) {
        const int r = tid;
        for (int j = 0; j < kCB; ++j) {
          if (r == j) {
            const double d = ta[j * (kCB + 1) + j];
            ta[j * (kCB + 1) + j] = d > 0 ? sqrt(d) : __longlong_as_double(0x7ff8000000000000ll);
          }
          __syncwarp();
          const double djj = ta[j * (kCB + 1) + j];
          if (r > j) ta[r * (kCB + 1) + j] /= djj;
          __syncwarp();
          if (r > j) {
            const double lrj = ta[r * (kCB + 1) + j];
            for (int c = j + 1; c <= r; ++c) ta[r * (kCB + 1) + c] -= lrj * ta[c * (kCB + 1) + j];
          }
          __syncwarp();
        }
      }
      __syncthreads();
      for (int e = tid; e < kCB * kCB; e += blockDim.x) {
        const int r = e / kCB, c = e % kCB;
        if (c <= r) M[(int64_t)(k0 + r) * mp + k0 + c] = ta[r * (kCB + 1) + c];
      }
      // 2. panel below: rows r >= k0 + 32 solve x L_kk^T = M[r, k0:k0+32],
      //    one row per thread, the row staged in shared memory
      for (int r = k0 + kCB + tid; r < mp; r += blockDim.x) {
        double *x = panel + tid * (kCB + 1);
        for (int c = 0; c < kCB; ++c) x[c] = M[(int64_t)r * mp + k0 + c];
        for (int c = 0; c < kCB; ++c) {
          const double xc = x[c] / ta[c * (kCB + 1) + c];
          x[c] = xc;
          for (int t = c + 1; t < kCB; ++t) x[t] -= xc * ta[t * (kCB + 1) + c];
        }
        for (int c = 0; c < kCB; ++c) M[(int64_t)r * mp + k0 + c] = x[c];
      }
      __syncthreads();
      // 3. trailing update of the lower triangle: M_ij -= L_ik L_jk^T, i >= j > k
      for (int jb = k + 1; jb < nb; ++jb) {
        for (int e = tid; e < kCB * kCB; e += blockDim.x) {
          const int r = e / kCB, c = e % kCB;
          tb[r * (kCB + 1) + c] = M[(int64_t)(jb * kCB + r) * mp + k0 + c];  // L_jk
        }
        for (int ib = jb; ib < nb; ++ib) {
          __syncthreads();
          for (int e = tid; e < kCB * kCB; e += blockDim.x) {
            const int r = e / kCB, c = e % kCB;
            ta[r * (kCB + 1) + c] = M[(int64_t)(ib * kCB + r) * mp + k0 + c];  // L_ik
          }
          __syncthreads();
          for (int e = tid; e < kCB * kCB; e += blockDim.x) {
            const int r = e / kCB, c = e % kCB;
            if (ib == jb && c > r) continue;
            double v = 0;
#pragma unroll 8
            for (int t = 0; t < kCB; ++t) v += ta[r * (kCB + 1) + t] * tb[c * (kCB + 1) + t];
            M[(int64_t)(ib * kCB + r) * mp + jb * kCB + c] -= v;
          }
        }
        __syncthreads();
      }
      __syncthreads();
    }
    // L z = rhs (column-oriented), then L^T x = z
    for (int j = 0; j < mp; ++j) {
      const double zj = rhs[j] / M[(int64_t)j * mp + j];
      __syncthreads();
      if (tid == 0) rhs[j] = zj;
      for (int r = j + 1 + tid; r < mp; r += blockDim.x) rhs[r] -= M[(int64_t)r * mp + j] * zj;
      __syncthreads();
    }
    for (int j = mp - 1; j >= 0; --j) {
      const double xj = rhs[j] / M[(int64_t)j * mp + j];
      __syncthreads();
      if (tid == 0) rhs[j] = xj;
      for (int r = tid; r < j; r += blockDim.x) rhs[r] -= M[(int64_t)j * mp + r] * xj;
      __syncthreads();
    }
    for (int r = tid; r < m; r += blockDim.x) coef[b0 + r] = (float)rhs[r];
    __syncthreads();
  }
}

size_t al(size_t x) { return (x + 255) & ~(size_t)255; }

}  // namespace

int refine_cap(int32_t d_in) { return std::min(((d_in + kCB - 1) / kCB) * kCB, 1024); }

size_t refine_workspace(int32_t d_out, int32_t d_in) {
  const size_t dd = (size_t)d_in * d_in, od = (size_t)d_out * d_in;
  const size_t cap = (size_t)refine_cap(d_in);
  return 3 * al(dd * 4) + 2 * al(dd * 2) + 2 * al(od * 2) + 2 * al(od * 4) + al((size_t)sm_count() * cap * cap * 8);
}

cudaError_t launch_calib_hessian(const void *X, int64_t T, int32_t d_in, float *S, cudaStream_t s) {
  return launch_gemm_any(X, true, X, true, nullptr, S, true, d_in, d_in, T, s);
}

cudaError_t launch_refine(const float *dWq, int32_t d_out, int32_t d_in, int32_t had_block, const float *S,
                          float damp, const int32_t *row_ptr, const int32_t *col_idx, int64_t p, float *coef,
                          void *ws, cudaStream_t s) {
  const size_t dd = (size_t)d_in * d_in, od = (size_t)d_out * d_in;
  char *w = static_cast<char *>(ws);
  float *A0 = reinterpret_cast<float *>(w);
  w += al(dd * 4);
  float *A1 = reinterpret_cast<float *>(w);
  w += al(dd * 4);
  float *Gt = reinterpret_cast<float *>(w);
  w += al(dd * 4);
  __nv_bfloat16 *Sh = reinterpret_cast<__nv_bfloat16 *>(w);
  w += al(dd * 2);
  __nv_bfloat16 *Sl = reinterpret_cast<__nv_bfloat16 *>(w);
  w += al(dd * 2);
  __nv_bfloat16 *Wh = reinterpret_cast<__nv_bfloat16 *>(w);
  w += al(od * 2);
  __nv_bfloat16 *Wl = reinterpret_cast<__nv_bfloat16 *>(w);
  w += al(od * 2);
  float *P0 = reinterpret_cast<float *>(w);
  w += al(od * 4);
  float *P1 = reinterpret_cast<float *>(w);
  w += al(od * 4);
  double *slabs = reinterpret_cast<double *>(w);
  const int logn = ilog2(had_block);
  const float inv = (float)(1.0 / sqrt((double)had_block));
  const int64_t blocks_dd = (int64_t)d_in * (d_in / had_block), blocks_od = (int64_t)d_out * (d_in / had_block);
  const unsigned g1 = (unsigned)std::min<int64_t>(cdiv((int64_t)dd, 256), (int64_t)sm_count() * 8);
  const unsigned g2 = (unsigned)std::min<int64_t>(cdiv((int64_t)od, 256), (int64_t)sm_count() * 8);
  // 1. damped S
  copy_f32_kernel<<<g1, 256, 0, s>>>(S, A0, (int64_t)dd);
  damp_kernel<<<1, 1024, 0, s>>>(S, d_in, damp, A0);
  cudaError_t e = cudaGetLastError();
  // 2. G^T = ((S H)^T) H
  if (e == cudaSuccess) e = launch_fwht(QWHA_F32, QWHA_F32, A0, A1, blocks_dd, logn, inv, s);
  if (e == cudaSuccess) {
    const dim3 grid((unsigned)cdiv(d_in, 32), (unsigned)cdiv(d_in, 32));
    transpose_kernel<<<grid, dim3(32, 8), 0, s>>>(A1, d_in, d_in, Gt);
    e = cudaGetLastError();
  }
  if (e == cudaSuccess) e = launch_fwht(QWHA_F32, QWHA_F32, Gt, A1, blocks_dd, logn, inv, s);
  float *G_t = A1;
  // 3. U = (dW_Q S) H with split-bf16 tensor-core products
  if (e == cudaSuccess) {
    split_bf16_kernel<<<g1, 256, 0, s>>>(A0, (int64_t)dd, Sh, Sl);
    split_bf16_kernel<<<g2, 256, 0, s>>>(dWq, (int64_t)od, Wh, Wl);
    e = cudaGetLastError();
  }
  // P[i][b] = sum_a W[i][a] S[b][a] (S symmetric): B is S as stored, K-major
  if (e == cudaSuccess) e = launch_gemm_any(Wh, false, Sh, false, nullptr, P0, true, d_out, d_in, d_in, s);
  if (e == cudaSuccess) e = launch_gemm_any(Wh, false, Sl, false, P0, P1, true, d_out, d_in, d_in, s);
  if (e == cudaSuccess) e = launch_gemm_any(Wl, false, Sh, false, P1, P0, true, d_out, d_in, d_in, s);
  if (e == cudaSuccess) e = launch_fwht(QWHA_F32, QWHA_F32, P0, P1, blocks_od, logn, inv, s);
  if (e != cudaSuccess) return e;
  // 4. per-channel solves
  const int cap = refine_cap(d_in);
  const size_t smem = ((size_t)cap + (2 + kCholThreads / kCB) * kCB * (kCB + 1)) * sizeof(double);
  e = cudaFuncSetAttribute(refine_solve_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  const int grid = std::min(sm_count(), d_out);
  refine_solve_kernel<<<grid, kCholThreads, smem, s>>>(G_t, P1, d_out, d_in, row_ptr, col_idx, p, cap, slabs, coef,
                                                       device_error_word());
  return cudaGetLastError();
}

}  // namespace qwha
