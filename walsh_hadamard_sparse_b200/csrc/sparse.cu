// Sparse products of the adapter with F = Scatter(c, E) ("QWHA",
// papernotes.org 整体框架; gist.science 2.1).
//
// seg_spmm: out[t, i] = alpha * sum_{j in segment i} val[j] * in[t, idx[j]].
//   Forward (segments = rows of F, CSR):  Y_ad = alpha Z F^T.
//   Backward (segments = columns of F, CSC, val through perm): dZ = alpha dY F.
//   One CTA owns TT tokens: their input rows are staged transposed in shared
//   memory as s_in[k][TT] (a column of the tile is TT contiguous values), then
//   each warp runs one segment at a time (see seg_spmm_kernel). The segment
//   arrays stream from L2 once per token tile. The backward passes the
//   coefficients already permuted to CSC order (permute_kernel).
//
// sddmm: partial[c, j] = sum_{t in chunk c} dY[t, r_j] * Z[t, k_j] over the
//   tile view of E (QWHA_TILE x QWHA_TILE blocks of F). Grid = tiles x token
//   chunks; a CTA stages dY[:, row block] and Z[:, column block] for TT tokens
//   at a time, transposed, with the next sub-tile's global loads issued into
//   registers before the current one is consumed; each thread accumulates a
//   run of consecutive tile entries (same column mostly: the Z vector is
//   reloaded only when the column changes).
// sddmm_reduce: dc[j] = alpha * sum_c partial[c, j] in increasing c (fixed
//   order: the result is bitwise reproducible).

#include <algorithm>

#include "common.cuh"
#include "kernels.h"

namespace qwha {
namespace {

constexpr int kSpmmThreads = 512;
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

// One warp per segment at a time. A lane holds 4 consecutive tokens of the
// tile (Q = TT/4 lanes cover the tile) for one of NSLOT = 32/Q nonzero slots:
// lane = q + Q * slot. The slots walk the segment's nonzeros 8 or 16 at a time
// (coalesced index/value loads, each nonzero's 4-token vector is one 8- or
// 16-byte shared load); a shuffle tree over the slots ends the segment and the
// Q lanes of slot 0 write its TT outputs.
template <typename Tin, typename Tout, int TT>
__global__ void __launch_bounds__(kSpmmThreads)
    seg_spmm_kernel(const Tin *__restrict__ in, int64_t T, int W_in, const int32_t *__restrict__ seg_ptr,
                    const int32_t *__restrict__ idx, const float *__restrict__ val, int64_t nnz, int n_seg,
                    float alpha, Tout *__restrict__ out) {
  constexpr int Q = TT / 4;        // lanes per nonzero (4 tokens each)
  constexpr int NSLOT = 32 / Q;    // nonzeros in flight per warp
  extern __shared__ __align__(16) unsigned char smem_raw[];
  Tin *s_in = reinterpret_cast<Tin *>(smem_raw);
  const int64_t t0 = (int64_t)blockIdx.x * TT;
  stage_transposed<Tin, TT>(in, T, W_in, t0, 0, W_in, W_in, s_in);
  __syncthreads();

  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int q = lane % Q, slot = lane / Q;
  constexpr int kWarps = kSpmmThreads / 32;
  for (int seg = warp; seg < n_seg; seg += kWarps) {
    int64_t b = seg_ptr[seg], e = seg_ptr[seg + 1];
    if (b < 0) b = 0;
    if (e > nnz) e = nnz;
    float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll 4
    for (int64_t j = b + slot; j < e; j += NSLOT) {
      const int k = __ldg(idx + j);
      const float v = __ldg(val + j);
      if ((unsigned)k < (unsigned)W_in) {
        float x[4];
        load_vals<Tin>(s_in + (int64_t)k * TT + 4 * q, x, 4);
#pragma unroll
        for (int i = 0; i < 4; ++i) acc[i] = fmaf(v, x[i], acc[i]);
      }
    }
#pragma unroll
    for (int off = Q; off < 32; off <<= 1)
#pragma unroll
      for (int i = 0; i < 4; ++i) acc[i] += __shfl_xor_sync(0xffffffffu, acc[i], off);
    if (slot == 0) {
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int64_t t = t0 + 4 * q + i;
        if (t < T) io<Tout>::store1(out + t * n_seg + seg, alpha * acc[i]);
      }
    }
  }
}

template <typename Tin, typename Tout, int TT>
cudaError_t run_spmm(const void *in, int64_t T, int W_in, const int32_t *seg_ptr, const int32_t *idx,
                     const float *val, int64_t nnz, int n_seg, float alpha, void *out, cudaStream_t s) {
  const size_t smem = (size_t)W_in * TT * sizeof(Tin);
  auto k = seg_spmm_kernel<Tin, Tout, TT>;
  cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  const int64_t grid = cdiv(T, TT);
  k<<<(unsigned)grid, kSpmmThreads, smem, s>>>(static_cast<const Tin *>(in), T, W_in, seg_ptr, idx, val, nnz, n_seg,
                                              alpha, static_cast<Tout *>(out));
  return cudaGetLastError();
}

template <typename Tin, typename Tout>
cudaError_t pick_spmm(const void *in, int64_t T, int W_in, const int32_t *seg_ptr, const int32_t *idx,
                      const float *val, int64_t nnz, int n_seg, float alpha, void *out, cudaStream_t s) {
  const size_t row = (size_t)W_in * sizeof(Tin);
  if (row * 16 <= kSpmmSmemCap)
    return run_spmm<Tin, Tout, 16>(in, T, W_in, seg_ptr, idx, val, nnz, n_seg, alpha, out, s);
  if (row * 8 <= kSpmmSmemCap)
    return run_spmm<Tin, Tout, 8>(in, T, W_in, seg_ptr, idx, val, nnz, n_seg, alpha, out, s);
  return run_spmm<Tin, Tout, 4>(in, T, W_in, seg_ptr, idx, val, nnz, n_seg, alpha, out, s);
}

__global__ void permute_kernel(const float *__restrict__ src, const int32_t *__restrict__ perm, int64_t p,
                               float *__restrict__ dst) {
  for (int64_t q = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; q < p; q += (int64_t)gridDim.x * blockDim.x) {
    const int32_t j = perm[q];
    dst[q] = (uint64_t)j < (uint64_t)p ? src[j] : 0.f;
  }
}

// ---------------------------------------------------------------- SDDMM

constexpr int kSddmmThreads = 512;
constexpr int kSddmmEPT = 16;  // tile entries per thread per pass

// tokens per staged sub-tile: 2 x QWHA_TILE x TT values = 64 KB
template <typename T>
__host__ __device__ constexpr int sddmm_tt() {
  return sizeof(T) == 2 ? 32 : 16;
}

// Per thread: the 16-byte global vectors of one sub-tile it stages (dY slice
// and Z slice), held in registers so that the next sub-tile's loads overlap
// the current sub-tile's arithmetic.
template <typename T, int TT>
struct SubTile {
  static constexpr int V = 16 / (int)sizeof(T);                       // values per vector
  static constexpr int ITEMS = 2 * (QWHA_TILE / V) * TT / kSddmmThreads;  // vectors per thread
  uint4 v[ITEMS];

  // item it -> (operand, token, vector c along the row/column block)
  __device__ __forceinline__ void load(const T *dY, const T *Z, int64_t tb, int d_out, int d_in, int64_t t0, int r0,
                                       int r_len, int k0, int k_len) {
#pragma unroll
    for (int u = 0; u < ITEMS; ++u) {
      const int it = threadIdx.x + u * kSddmmThreads;
      const int half = (QWHA_TILE / V) * TT;
      const int which = it >= half;
      const int w = it - which * half;
      const int t = w % TT, c = w / TT;
      const int64_t tg = t0 + t;
      const int len = which ? k_len : r_len;
      v[u] = make_uint4(0, 0, 0, 0);
      if (tg < tb && c * V < len) {
        const T *src = which ? Z + tg * d_in + k0 + c * V : dY + tg * d_out + r0 + c * V;
        v[u] = *reinterpret_cast<const uint4 *>(src);
      }
    }
  }
  __device__ __forceinline__ void store(T *s_dy, T *s_z) const {
#pragma unroll
    for (int u = 0; u < ITEMS; ++u) {
      const int it = threadIdx.x + u * kSddmmThreads;
      const int half = (QWHA_TILE / V) * TT;
      const int which = it >= half;
      const int w = it - which * half;
      const int t = w % TT, c = w / TT;
      float f[V];
      io<T>::unpack(v[u], f);
      T *dst = which ? s_z : s_dy;
#pragma unroll
      for (int i = 0; i < V; ++i) io<T>::store1(dst + (c * V + i) * TT + t, f[i]);
    }
  }
};

template <typename T>
__global__ void __launch_bounds__(kSddmmThreads)
    sddmm_kernel(const T *__restrict__ dY, const T *__restrict__ Z, int64_t T_, int d_out, int d_in,
                 const int32_t *__restrict__ tile_ptr, const int32_t *__restrict__ tile_pos,
                 const int32_t *__restrict__ tile_rk, int n_rb, int64_t chunk_tokens, int64_t p,
                 float *__restrict__ partial) {
  constexpr int TT = sddmm_tt<T>();
  extern __shared__ __align__(16) unsigned char smem_raw[];
  T *s_dy = reinterpret_cast<T *>(smem_raw);
  T *s_z = s_dy + QWHA_TILE * TT;
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
    int rk[kSddmmEPT];  // (row << 16 | column) inside the tile, -1 when unused
    float acc[kSddmmEPT];
#pragma unroll
    for (int q = 0; q < kSddmmEPT; ++q) {
      const int v = q < n_mine ? tile_rk[my0 + q] : -1;
      const int r_ = (v >> 16) & 0xffff, k_ = v & 0xffff;
      rk[q] = (q < n_mine && r_ < r_len && k_ < k_len) ? v : -1;
      acc[q] = 0.f;
    }
    SubTile<T, TT> nxt;
    if (ta < tb) nxt.load(dY, Z, tb, d_out, d_in, ta, r0, r_len, k0, k_len);
    for (int64_t t0 = ta; t0 < tb; t0 += TT) {
      __syncthreads();  // the previous sub-tile is consumed
      nxt.store(s_dy, s_z);
      __syncthreads();
      if (t0 + TT < tb) nxt.load(dY, Z, tb, d_out, d_in, t0 + TT, r0, r_len, k0, k_len);
      int cur_k = -2;
      float zv[TT];
#pragma unroll
      for (int q = 0; q < kSddmmEPT; ++q) {
        if (rk[q] < 0) continue;
        const int kq = rk[q] & 0xffff, rq = rk[q] >> 16;
        if (kq != cur_k) {
#pragma unroll
          for (int u = 0; u < TT; u += 8) load_vals<T>(s_z + kq * TT + u, zv + u, 8);
          cur_k = kq;
        }
        float a = acc[q];
#pragma unroll
        for (int u = 0; u < TT; u += 8) {
          float yv[8];
          load_vals<T>(s_dy + rq * TT + u, yv, 8);
#pragma unroll
          for (int i = 0; i < 8; ++i) a = fmaf(yv[i], zv[u + i], a);
        }
        acc[q] = a;
      }
    }
#pragma unroll
    for (int q = 0; q < kSddmmEPT; ++q)
      if (q < n_mine) {
        const int j = tile_pos[my0 + q];
        if ((uint64_t)j < (uint64_t)p) part[j] = acc[q];
      }
    __syncthreads();
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
                            const int32_t *seg_ptr, const int32_t *idx, const float *val, int64_t nnz, int n_seg,
                            float alpha, void *out, cudaStream_t s) {
  if (T <= 0 || n_seg <= 0) return cudaSuccess;
  using bf = __nv_bfloat16;
  if (din == QWHA_BF16) {
    if (dout == QWHA_BF16) return pick_spmm<bf, bf>(in, T, W_in, seg_ptr, idx, val, nnz, n_seg, alpha, out, s);
    return pick_spmm<bf, float>(in, T, W_in, seg_ptr, idx, val, nnz, n_seg, alpha, out, s);
  }
  if (dout == QWHA_BF16) return pick_spmm<float, bf>(in, T, W_in, seg_ptr, idx, val, nnz, n_seg, alpha, out, s);
  return pick_spmm<float, float>(in, T, W_in, seg_ptr, idx, val, nnz, n_seg, alpha, out, s);
}

cudaError_t launch_permute(const float *src, const int32_t *perm, int64_t p, float *dst, cudaStream_t s) {
  if (p <= 0) return cudaSuccess;
  const int64_t grid = std::min<int64_t>(cdiv(p, 256), (int64_t)sm_count() * 8);
  permute_kernel<<<(unsigned)grid, 256, 0, s>>>(src, perm, p, dst);
  return cudaGetLastError();
}

int sddmm_chunks(int64_t T, int32_t d_out, int32_t d_in) {
  const int64_t tiles = cdiv(d_out, QWHA_TILE) * cdiv(d_in, QWHA_TILE);
  int64_t want = cdiv(2 * (int64_t)sm_count(), tiles);
  const int64_t max_by_tokens = cdiv(T, 32);
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
  const int64_t chunk_tokens = cdiv(cdiv(T, n_chunks), 32) * 32;
  cudaError_t e = cudaMemsetAsync(partial, 0, (size_t)n_chunks * p * sizeof(float), s);
  if (e != cudaSuccess) return e;
  if (T > 0) {
    dim3 grid((unsigned)tiles, (unsigned)n_chunks);
    const size_t smem = 64 * 1024;
    if (dt == QWHA_BF16) {
      auto k = sddmm_kernel<__nv_bfloat16>;
      e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
      if (e != cudaSuccess) return e;
      k<<<grid, kSddmmThreads, smem, s>>>(static_cast<const __nv_bfloat16 *>(dY),
                                          static_cast<const __nv_bfloat16 *>(Z), T, d_out, d_in, tile_ptr, tile_pos,
                                          tile_rk, n_rb, chunk_tokens, p, partial);
    } else {
      auto k = sddmm_kernel<float>;
      e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
      if (e != cudaSuccess) return e;
      k<<<grid, kSddmmThreads, smem, s>>>(static_cast<const float *>(dY), static_cast<const float *>(Z), T, d_out,
                                          d_in, tile_ptr, tile_pos, tile_rk, n_rb, chunk_tokens, p, partial);
    }
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  sddmm_reduce_kernel<<<(unsigned)std::min<int64_t>(cdiv(p, 256), (int64_t)sm_count() * 8), 256, 0, s>>>(partial, n_chunks, p,
                                                                                         alpha, dc);
  return cudaGetLastError();
}

}  // namespace qwha
