// Sparse products of the adapter with F = Scatter(c, E) ("QWHA",
// papernotes.org 整体框架; gist.science 2.1).
//
// seg_spmm: out[t, i] = alpha * sum_{j in segment i} val[j] * in[t, idx[j]].
//   Forward (segments = rows of F, CSR):  Y_ad = alpha Z F^T.
//   Backward (segments = columns of F, CSC, val through perm): dZ = alpha dY F.
//   One CTA owns TT tokens: their input rows are staged transposed in shared
//   memory as s_in[k][TT] (a column of the tile is TT contiguous values), then
//   every thread runs one segment for G = min(TT, 8) tokens: per nonzero one
//   broadcast load of (idx, val) and one 16-byte shared load of G inputs.
//   The segment arrays stream from L2 once per token tile.
//
// sddmm: partial[c, j] = sum_{t in chunk c} dY[t, r_j] * Z[t, k_j] over the
//   tile view of E (QWHA_TILE x QWHA_TILE blocks of F). Grid = tiles x token
//   chunks; a CTA stages dY[:, row block] and Z[:, column block] for TT tokens
//   at a time, transposed, and each thread accumulates a run of consecutive
//   tile entries (same column mostly: the Z vector is reloaded only when the
//   column changes).
// sddmm_reduce: dc[j] = alpha * sum_c partial[c, j] in increasing c (fixed
//   order: the result is bitwise reproducible).

#include <algorithm>

#include "common.cuh"
#include "kernels.h"

namespace qwha {
namespace {

constexpr int kSpmmThreads = 256;
constexpr size_t kSpmmSmemCap = 160 * 1024;

template <typename T>
__device__ __forceinline__ void load_vals(const T *p, float *o, int n);

// Load n (<= 8, power of two) consecutive values from shared memory as floats.
template <>
__device__ __forceinline__ void load_vals<__nv_bfloat16>(const __nv_bfloat16 *p, float *o, int n) {
  if (n == 8) {
    const uint4 w = *reinterpret_cast<const uint4 *>(p);
    io<__nv_bfloat16>::unpack(w, o);
  } else if (n == 4) {
    const uint2 w = *reinterpret_cast<const uint2 *>(p);
    o[0] = bf16_lo(w.x), o[1] = bf16_hi(w.x), o[2] = bf16_lo(w.y), o[3] = bf16_hi(w.y);
  } else if (n == 2) {
    const uint32_t w = *reinterpret_cast<const uint32_t *>(p);
    o[0] = bf16_lo(w), o[1] = bf16_hi(w);
  } else {
    o[0] = __bfloat162float(*p);
  }
}

template <>
__device__ __forceinline__ void load_vals<float>(const float *p, float *o, int n) {
  if (n == 8) {
    const float4 a = *reinterpret_cast<const float4 *>(p), b = *reinterpret_cast<const float4 *>(p + 4);
    o[0] = a.x, o[1] = a.y, o[2] = a.z, o[3] = a.w, o[4] = b.x, o[5] = b.y, o[6] = b.z, o[7] = b.w;
  } else if (n == 4) {
    const float4 a = *reinterpret_cast<const float4 *>(p);
    o[0] = a.x, o[1] = a.y, o[2] = a.z, o[3] = a.w;
  } else if (n == 2) {
    const float2 a = *reinterpret_cast<const float2 *>(p);
    o[0] = a.x, o[1] = a.y;
  } else {
    o[0] = *p;
  }
}

// Stage rows [t0, t0+TT) of in[T, W] into s[k * TT + t] (zeros past T).
template <typename T, int TT>
__device__ __forceinline__ void stage_transposed(const T *__restrict__ in, int64_t T_, int W, int64_t t0,
                                                 int k_off, int k_len, int64_t ld, T *s) {
  // One item = one token x 16 bytes along k; consecutive threads take
  // consecutive tokens so that the scattered 2/4-byte stores spread over banks.
  constexpr int V = 16 / (int)sizeof(T);
  const int chunks = k_len / V;
  for (int it = threadIdx.x; it < chunks * TT; it += blockDim.x) {
    const int t = it % TT;
    const int c = it / TT;
    const int64_t tg = t0 + t;
    float v[V];
    if (tg < T_) {
      io<T>::unpack(*reinterpret_cast<const uint4 *>(in + tg * ld + k_off + c * V), v);
    } else {
#pragma unroll
      for (int i = 0; i < V; ++i) v[i] = 0.f;
    }
#pragma unroll
    for (int i = 0; i < V; ++i) io<T>::store1(s + (int64_t)(c * V + i) * TT + t, v[i]);
  }
  (void)W;
}

template <typename Tin, typename Tout, int TT>
__global__ void __launch_bounds__(kSpmmThreads)
    seg_spmm_kernel(const Tin *__restrict__ in, int64_t T, int W_in, const int32_t *__restrict__ seg_ptr,
                    const int32_t *__restrict__ idx, const float *__restrict__ val,
                    const int32_t *__restrict__ val_perm, int64_t nnz, int n_seg, float alpha,
                    Tout *__restrict__ out) {
  constexpr int G = TT < 8 ? TT : 8;  // tokens per thread
  constexpr int NG = TT / G;          // threads per segment
  extern __shared__ __align__(16) unsigned char smem_raw[];
  Tin *s_in = reinterpret_cast<Tin *>(smem_raw);
  const int64_t t0 = (int64_t)blockIdx.x * TT;
  stage_transposed<Tin, TT>(in, T, W_in, t0, 0, W_in, W_in, s_in);
  __syncthreads();

  const int g = threadIdx.x % NG;
  for (int seg = threadIdx.x / NG; seg < n_seg; seg += kSpmmThreads / NG) {
    int64_t b = seg_ptr[seg], e = seg_ptr[seg + 1];
    if (b < 0) b = 0;
    if (e > nnz) e = nnz;
    float acc[G];
#pragma unroll
    for (int i = 0; i < G; ++i) acc[i] = 0.f;
    for (int64_t j = b; j < e; ++j) {
      const int k = __ldg(idx + j);
      const float v = __ldg(val + (val_perm ? __ldg(val_perm + j) : j));
      if ((unsigned)k >= (unsigned)W_in) continue;
      float x[G];
      load_vals<Tin>(s_in + (int64_t)k * TT + g * G, x, G);
#pragma unroll
      for (int i = 0; i < G; ++i) acc[i] = fmaf(v, x[i], acc[i]);
    }
#pragma unroll
    for (int i = 0; i < G; ++i) {
      const int64_t t = t0 + g * G + i;
      if (t < T) io<Tout>::store1(out + t * n_seg + seg, alpha * acc[i]);
    }
  }
}

template <typename Tin, typename Tout, int TT>
cudaError_t run_spmm(const void *in, int64_t T, int W_in, const int32_t *seg_ptr, const int32_t *idx,
                     const float *val, const int32_t *val_perm, int64_t nnz, int n_seg, float alpha, void *out,
                     cudaStream_t s) {
  const size_t smem = (size_t)W_in * TT * sizeof(Tin);
  auto k = seg_spmm_kernel<Tin, Tout, TT>;
  cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  const int64_t grid = cdiv(T, TT);
  k<<<(unsigned)grid, kSpmmThreads, smem, s>>>(static_cast<const Tin *>(in), T, W_in, seg_ptr, idx, val, val_perm,
                                              nnz, n_seg, alpha, static_cast<Tout *>(out));
  return cudaGetLastError();
}

template <typename Tin, typename Tout>
cudaError_t pick_spmm(const void *in, int64_t T, int W_in, const int32_t *seg_ptr, const int32_t *idx,
                      const float *val, const int32_t *val_perm, int64_t nnz, int n_seg, float alpha, void *out,
                      cudaStream_t s) {
  const size_t row = (size_t)W_in * sizeof(Tin);
  if (row * 16 <= kSpmmSmemCap)
    return run_spmm<Tin, Tout, 16>(in, T, W_in, seg_ptr, idx, val, val_perm, nnz, n_seg, alpha, out, s);
  if (row * 8 <= kSpmmSmemCap)
    return run_spmm<Tin, Tout, 8>(in, T, W_in, seg_ptr, idx, val, val_perm, nnz, n_seg, alpha, out, s);
  if (row * 4 <= kSpmmSmemCap)
    return run_spmm<Tin, Tout, 4>(in, T, W_in, seg_ptr, idx, val, val_perm, nnz, n_seg, alpha, out, s);
  if (row * 2 <= kSpmmSmemCap)
    return run_spmm<Tin, Tout, 2>(in, T, W_in, seg_ptr, idx, val, val_perm, nnz, n_seg, alpha, out, s);
  return run_spmm<Tin, Tout, 1>(in, T, W_in, seg_ptr, idx, val, val_perm, nnz, n_seg, alpha, out, s);
}

// ---------------------------------------------------------------- SDDMM

constexpr int kSddmmThreads = 512;
constexpr int kSddmmEPT = 16;  // tile entries per thread per pass

// tokens per staged sub-tile: 2 x QWHA_TILE x TT values stay within 32 KB
template <typename T>
constexpr int sddmm_tt() {
  return sizeof(T) == 2 ? 16 : 8;
}

template <typename T>
__global__ void __launch_bounds__(kSddmmThreads)
    sddmm_kernel(const T *__restrict__ dY, const T *__restrict__ Z, int64_t T_, int d_out, int d_in,
                 const int32_t *__restrict__ tile_ptr, const int32_t *__restrict__ tile_pos,
                 const int32_t *__restrict__ tile_rk, int n_rb, int64_t chunk_tokens, int64_t p,
                 float *__restrict__ partial) {
  constexpr int TT = sddmm_tt<T>();
  __shared__ __align__(16) T s_dy[QWHA_TILE * TT];
  __shared__ __align__(16) T s_z[QWHA_TILE * TT];
  const int tile = blockIdx.x;
  const int rb = tile % n_rb, kb = tile / n_rb;
  const int r0 = rb * QWHA_TILE, k0 = kb * QWHA_TILE;
  const int r_len = min(QWHA_TILE, d_out - r0), k_len = min(QWHA_TILE, d_in - k0);
  int64_t e_begin = tile_ptr[tile], e_end = tile_ptr[tile + 1];
  if (e_begin < 0) e_begin = 0;
  if (e_end > p) e_end = p;
  const int64_t c = blockIdx.y;
  const int64_t ta = c * chunk_tokens, tb = (ta + chunk_tokens < T_) ? ta + chunk_tokens : T_;
  float *part = partial + c * p;

  for (int64_t eb = e_begin; eb < e_end; eb += (int64_t)kSddmmThreads * kSddmmEPT) {
    const int64_t my0 = eb + (int64_t)threadIdx.x * kSddmmEPT;
    const int64_t left = e_end - my0;
    const int n_mine = left <= 0 ? 0 : (left < kSddmmEPT ? (int)left : kSddmmEPT);
    int32_t rk[kSddmmEPT];
    float acc[kSddmmEPT];
#pragma unroll
    for (int q = 0; q < kSddmmEPT; ++q) {
      rk[q] = q < n_mine ? tile_rk[my0 + q] : 0;
      acc[q] = 0.f;
    }
    for (int64_t t0 = ta; t0 < tb; t0 += TT) {
      __syncthreads();
      stage_transposed<T, TT>(dY, tb, d_out, t0, r0, r_len, d_out, s_dy);
      stage_transposed<T, TT>(Z, tb, d_in, t0, k0, k_len, d_in, s_z);
      __syncthreads();
      int cur_k = -1;
      float zv[TT];
#pragma unroll
      for (int q = 0; q < kSddmmEPT; ++q) {
        if (q < n_mine) {
          const int rl = (rk[q] >> 16) & 0xffff, kl = rk[q] & 0xffff;
          if (rl < r_len && kl < k_len) {
            if (kl != cur_k) {
#pragma unroll
              for (int u = 0; u < TT; u += 8) load_vals<T>(s_z + kl * TT + u, zv + u, 8);
              cur_k = kl;
            }
            float yv[TT];
#pragma unroll
            for (int u = 0; u < TT; u += 8) load_vals<T>(s_dy + rl * TT + u, yv + u, 8);
            float a = acc[q];
#pragma unroll
            for (int i = 0; i < TT; ++i) a = fmaf(yv[i], zv[i], a);
            acc[q] = a;
          }
        }
      }
    }
#pragma unroll
    for (int q = 0; q < kSddmmEPT; ++q)
      if (q < n_mine) {
        const int j = tile_pos[my0 + q];
        if ((uint64_t)j < (uint64_t)p) part[j] = acc[q];
      }
  }
}

__global__ void sddmm_reduce_kernel(const float *__restrict__ partial, int n_chunks, int64_t p, float alpha,
                                    float *__restrict__ dc) {
  for (int64_t j = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; j < p; j += (int64_t)gridDim.x * blockDim.x) {
    float s = 0.f;
    for (int c = 0; c < n_chunks; ++c) s += partial[(int64_t)c * p + j];
    dc[j] = alpha * s;
  }
}

}  // namespace

cudaError_t launch_seg_spmm(qwha_dtype din, qwha_dtype dout, const void *in, int64_t T, int W_in,
                            const int32_t *seg_ptr, const int32_t *idx, const float *val, const int32_t *val_perm,
                            int64_t nnz, int n_seg, float alpha, void *out, cudaStream_t s) {
  if (T <= 0 || n_seg <= 0) return cudaSuccess;
  using bf = __nv_bfloat16;
  if (din == QWHA_BF16) {
    if (dout == QWHA_BF16) return pick_spmm<bf, bf>(in, T, W_in, seg_ptr, idx, val, val_perm, nnz, n_seg, alpha, out, s);
    return pick_spmm<bf, float>(in, T, W_in, seg_ptr, idx, val, val_perm, nnz, n_seg, alpha, out, s);
  }
  if (dout == QWHA_BF16) return pick_spmm<float, bf>(in, T, W_in, seg_ptr, idx, val, val_perm, nnz, n_seg, alpha, out, s);
  return pick_spmm<float, float>(in, T, W_in, seg_ptr, idx, val, val_perm, nnz, n_seg, alpha, out, s);
}

int sddmm_chunks(int64_t T, int32_t d_out, int32_t d_in) {
  const int64_t tiles = cdiv(d_out, QWHA_TILE) * cdiv(d_in, QWHA_TILE);
  int64_t want = cdiv(2 * (int64_t)sm_count(), tiles);
  const int64_t max_by_tokens = cdiv(T, 16);
  if (want > max_by_tokens) want = max_by_tokens;
  if (want > kSddmmMaxChunks) want = kSddmmMaxChunks;
  if (want < 1) want = 1;
  return (int)want;
}

cudaError_t launch_sddmm(qwha_dtype dt, const void *dY, const void *Z, int64_t T, int32_t d_out, int32_t d_in,
                         const int32_t *tile_ptr, const int32_t *tile_pos, const int32_t *tile_rk, int64_t p,
                         float alpha, float *partial, float *dc, cudaStream_t s) {
  if (p <= 0) return cudaSuccess;
  const int n_rb = (int)cdiv(d_out, QWHA_TILE);
  const int64_t tiles = n_rb * cdiv(d_in, QWHA_TILE);
  const int n_chunks = sddmm_chunks(T, d_out, d_in);
  const int64_t chunk_tokens = cdiv(cdiv(T, n_chunks), 16) * 16;
  cudaError_t e = cudaMemsetAsync(partial, 0, (size_t)n_chunks * p * sizeof(float), s);
  if (e != cudaSuccess) return e;
  if (T > 0) {
    dim3 grid((unsigned)tiles, (unsigned)n_chunks);
    if (dt == QWHA_BF16)
      sddmm_kernel<__nv_bfloat16><<<grid, kSddmmThreads, 0, s>>>(
          static_cast<const __nv_bfloat16 *>(dY), static_cast<const __nv_bfloat16 *>(Z), T, d_out, d_in, tile_ptr,
          tile_pos, tile_rk, n_rb, chunk_tokens, p, partial);
    else
      sddmm_kernel<float><<<grid, kSddmmThreads, 0, s>>>(static_cast<const float *>(dY),
                                                         static_cast<const float *>(Z), T, d_out, d_in, tile_ptr,
                                                         tile_pos, tile_rk, n_rb, chunk_tokens, p, partial);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  sddmm_reduce_kernel<<<(unsigned)std::min<int64_t>(cdiv(p, 256), (int64_t)sm_count() * 8), 256, 0, s>>>(partial, n_chunks, p,
                                                                                         alpha, dc);
  return cudaGetLastError();
}

}  // namespace qwha
