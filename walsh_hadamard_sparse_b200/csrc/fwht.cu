// Row-wise fast Walsh-Hadamard transform (Sylvester order, orthonormal).
//
// The adapter's transform is the +-1 Walsh-Hadamard matrix, computed as a
// recursion of sums and differences with no multiplications ("QWHA",
// papernotes.org 关键设计 1; gist.science 2.1). Each block of n = 2^m
// consecutive elements of a row is replaced by its transform times `scale`
// (1/sqrt(n) for the orthonormal H, times alpha where the adapter folds it).
//
// Layout of the main kernel (128 <= n <= 4096). The m index bits of an element
// are split into three fields: low (LV bits, one 16-byte vector of the narrow
// I/O type), middle (PB bits) and high (HB bits).
//   phase A: a thread holds the low and high fields in registers (R = 2^RB
//            values) and the middle field is its index inside the row's
//            P = 2^PB threads; its input vectors come from a shared-memory
//            ring that bulk copies fill. All RB register bits get their
//            butterflies.
//   phase B: after a transpose through an fp32 shared-memory buffer, a thread
//            holds the middle field (plus, for odd m, one high bit as a batch
//            bit) and does the remaining butterflies; it writes the scaled
//            results, in the output type, into per-segment staging that bulk
//            copies send to global memory.
// The transpose buffer is padded (Geo::phys, fwht_body.cuh) so that both
// phases' accesses are free of bank conflicts. Arithmetic is fp32 whatever the I/O
// type. fwht_body.cuh holds the same arithmetic for the fused forward GEMM and
// the W_eff kernels below.

#include "common.cuh"
#include "fwht_body.cuh"
#include "bulk.cuh"
#include "kernels.h"

namespace qwha {
namespace {

constexpr int kThreads = 256;
constexpr int kRingSlots = 2;  // ring depth of the transform kernel (measured best of 2, 3, 4)

// Row transform for contiguous rows of 128 <= n <= 4096: a CTA is one worker
// of RW = max(P, 64) threads (RW / P rows per iteration) that streams its rows
// through an S-slot shared-memory ring filled by bulk copies (the TMA engine,
// one copy per iteration, issued S iterations ahead), so loads are always in
// flight without costing the threads issue slots or registers, and the CTA's
// barriers span only its own warps. Results leave through bulk stores of
// staged segments. Requires x and z 16-byte aligned.
template <int LOGN, int V>
struct RingGeo {
  using G = Geo<LOGN, V>;
  static constexpr int RW = G::P < 64 ? 64 : G::P;  // threads of the worker
  static constexpr int RPW = RW / G::P;             // rows per iteration
  // output staging: a segment per (row, high field) value holds the SEGE
  // contiguous output elements of that value, segp() elements apart: one
  // vector (V elements) of padding moves each segment by as many banks as a
  // vector spans, so the phase-B lanes of one store meet distinct banks
  // (two-way for fp32 output at n = 128 and 512)
  static constexpr int SEGE = 1 << (G::LV + G::PB);
  template <typename T>
  __host__ __device__ static constexpr int segp() { return SEGE + V; }
  // the exchange buffer (RPW rows of Geo::NP floats) and the output staging, which
  // reuses it: the larger of the two, rounded to 128 bytes
  template <typename T>
  __host__ __device__ static constexpr int buf_bytes() {
    const int a = RPW * G::NP * 4, b = RPW * (1 << G::HB) * segp<T>() * (int)sizeof(T);
    return ((a > b ? a : b) + 127) & ~127;
  }
};

template <int LOGN, int V, typename Tin, typename Tout, int S>
__global__ void __launch_bounds__(RingGeo<LOGN, V>::RW) fwht_ring_kernel(const Tin *__restrict__ x,
                                                                         Tout *__restrict__ z, int64_t rows,
                                                                         float scale, unsigned int *err,
                                                                         uint64_t wait_ns) {
  using G = Geo<LOGN, V>;
  using RG = RingGeo<LOGN, V>;
  constexpr int RPW = RG::RPW;
  constexpr int SLOT = RPW * G::N * (int)sizeof(Tin);  // bytes, a multiple of 16
  constexpr int BUF = RG::template buf_bytes<Tout>();

  extern __shared__ __align__(128) unsigned char smem_raw[];
  float *buf = reinterpret_cast<float *>(smem_raw);
  unsigned char *ring = smem_raw + BUF;
  uint64_t *full = reinterpret_cast<uint64_t *>(ring + S * SLOT);
  const int tid = threadIdx.x;
  const int rl = tid / G::P, t = tid % G::P;
  const int64_t stride = (int64_t)gridDim.x * RPW;
  const int64_t first = (int64_t)blockIdx.x * RPW;
  const int64_t iters = first < rows ? (rows - first + stride - 1) / stride : 0;
  float *rb = buf + rl * G::NP;  // this row's part of the transpose buffer

  auto issue = [&](int64_t it) {  // thread 0: copy iteration it's rows into its slot
    const int64_t r0 = first + it * stride;
    const int64_t left = rows - r0;
    const uint32_t bytes = (uint32_t)((left < RPW ? left : RPW) * G::N * (int64_t)sizeof(Tin));
    const int s = (int)(it % S);
    bulk::fence_proxy();
    bulk::load(bulk::saddr(ring + s * SLOT), x + r0 * G::N, bytes, bulk::saddr(full + s));
  };

  if (tid == 0) {
#pragma unroll
    for (int s = 0; s < S; ++s) bulk::init(bulk::saddr(full + s), 1);
    bulk::fence_init();
  }
  __syncthreads();
  if (tid == 0)
    for (int64_t it = 0; it < S && it < iters; ++it) issue(it);

  for (int64_t it = 0; it < iters; ++it) {
    const int s = (int)(it % S);
    const int64_t row = first + it * stride + rl;
    const bool active = row < rows;
    // wait_ns bounds this wait (the library's limit, lowered only by a test hook); the drain below always
    // keeps the fixed limit, so that no copy is still landing in shared memory when the CTA exits
    const bool ok = bulk::wait(bulk::saddr(full + s), (uint32_t)((it / S) & 1), wait_ns);
    if (tid == 0) bulk::wait_stores_read();  // the last iteration's output copies have read buf
    // every thread has left the previous iteration's output reads of buf
    if (__syncthreads_or(!ok)) {
      if (tid == 0) {
        atomicOr(err, 0x200u);
        // let the copies already issued land (bounded) before the CTA exits
        for (int64_t j = it; j < iters && j < it + S; ++j)
          (void)bulk::wait(bulk::saddr(full + (int)(j % S)), (uint32_t)((j / S) & 1));
      }
      return;
    }
    float v[G::R];
    if (active) {
      const Tin *xr = reinterpret_cast<const Tin *>(ring + s * SLOT) + rl * G::N;
#pragma unroll
      for (int h = 0; h < (1 << G::HB); ++h) {
        const Tin *src = xr + G::eA(t, h << G::LV);
#pragma unroll
        for (int u = 0; u < V; u += io<Tin>::kVec)
          io<Tin>::unpack(*reinterpret_cast<const uint4 *>(src + u), v + h * V + u);
      }
    } else {
#pragma unroll
      for (int q = 0; q < G::R; ++q) v[q] = 0.f;
    }
    butterflies_x2<G::R, 0, G::RB, 0>(v);
#pragma unroll
    for (int h = 0; h < (1 << G::HB); ++h) {
#pragma unroll
      for (int u = 0; u < V; u += 4)
        *reinterpret_cast<float4 *>(rb + G::phys(G::eA(t, h << G::LV) + u)) =
            make_float4(v[h * V + u], v[h * V + u + 1], v[h * V + u + 2], v[h * V + u + 3]);
    }
    __syncthreads();  // phase A is in buf and slot s is consumed: refill it
    if (tid == 0 && it + S < iters) issue(it + S);
#pragma unroll
    for (int q = 0; q < G::R; ++q) v[q] = rb[G::phys(G::eB(t, q))];
    butterflies_x2<G::R, 0, G::PB, (G::NB ? G::PB : 0)>(v);
    __syncthreads();  // all phase-B reads done before the buffer is reused
    // results straight from phase B into the buffer in the output type, one
    // padded segment per (row, high field) value, written to global memory by
    // bulk copies from one thread, so no thread re-reads them
    Tout *ob = reinterpret_cast<Tout *>(smem_raw) + (rl * (1 << G::HB) + (t >> G::LV)) * RG::template segp<Tout>() +
               (t & (V - 1));
#pragma unroll
    for (int q = 0; q < G::R; ++q)
      io<Tout>::store1(ob + (q >> G::PB) * (1 << (G::HB - G::NB)) * RG::template segp<Tout>() +
                           ((q & (G::P - 1)) << G::LV),
                       v[q] * scale);
    bulk::fence_proxy();  // these writes before the copy engine's reads
    __syncthreads();
    if (tid == 0) {
      const int64_t r0 = first + it * stride;
      const int nrow = rows - r0 < RPW ? (int)(rows - r0) : RPW;
      for (int r = 0; r < nrow; ++r)
        for (int hh = 0; hh < (1 << G::HB); ++hh)
          bulk::store(z + (r0 + r) * G::N + hh * RG::SEGE,
                      bulk::saddr(reinterpret_cast<Tout *>(smem_raw) + (r * (1 << G::HB) + hh) * RG::template segp<Tout>()),
                      RG::SEGE * (int)sizeof(Tout));
      bulk::commit();
    }
  }
  if (tid == 0) bulk::wait_stores_read();  // the buffer stays valid until the last copy has read it
}

// n <= 64: one thread per block, all in registers.
template <int LOGN, typename Tin, typename Tout>
__global__ void __launch_bounds__(kThreads) fwht_small_kernel(const Tin *__restrict__ x,
                                                              Tout *__restrict__ z, int64_t rows,
                                                              float scale) {
  constexpr int N = 1 << LOGN;
  for (int64_t row = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; row < rows;
       row += (int64_t)gridDim.x * blockDim.x) {
    float v[N];
#pragma unroll
    for (int i = 0; i < N; ++i) v[i] = io<Tin>::load1(x + row * N + i);
    butterflies<N, 0, LOGN>(v);
#pragma unroll
    for (int i = 0; i < N; ++i) io<Tout>::store1(z + row * N + i, v[i] * scale);
  }
}

// 8192 <= n <= 32768: one CTA per block, the block in shared memory, three
// stages per pass over groups of 8 elements.
template <typename Tin, typename Tout>
__global__ void __launch_bounds__(512) fwht_large_kernel(const Tin *__restrict__ x,
                                                         Tout *__restrict__ z, int64_t rows,
                                                         int logn, float scale) {
  extern __shared__ __align__(16) float smem[];
  const int N = 1 << logn;
  for (int64_t row = blockIdx.x; row < rows; row += gridDim.x) {
    __syncthreads();
    for (int i = threadIdx.x; i < N; i += blockDim.x) smem[i] = io<Tin>::load1(x + row * N + i);
    __syncthreads();
    butterflies_smem_f32(smem, N, logn);
    for (int i = threadIdx.x; i < N; i += blockDim.x) io<Tout>::store1(z + row * N + i, smem[i] * scale);
  }
}

// W_eff block rows: for block b of row r (n = 2^LOGN columns starting at
// blk * n), scatter that row's coefficients into the padded buffer, run the
// two butterfly phases, then in phase-A layout (8 consecutive columns per
// vector) add the dequantized base weight in fp32 and store one bf16 rounding:
//   out[r, k] = bf16( W_Q[r, k] + scale * (sum_j c_j H_unnorm[k_j, k]) ).
template <int LOGN>
__global__ void __launch_bounds__(kThreads)
    weff_rows_kernel(const int32_t *__restrict__ row_ptr, const int32_t *__restrict__ col_idx,
                     const float *__restrict__ coef, int64_t p, int d_in, int64_t n_rows, float scale, int bits,
                     int group, const uint8_t *__restrict__ qw, const float *__restrict__ scales,
                     const uint8_t *__restrict__ zeros, __nv_bfloat16 *__restrict__ out) {
  using G = Geo<LOGN, 8>;
  constexpr int RPC = kThreads / G::P;
  extern __shared__ __align__(16) float smem[];
  const int rl = threadIdx.x / G::P;
  const int t = threadIdx.x % G::P;
  float *buf = smem + rl * G::NP;
  const int nb = d_in >> LOGN;
  const int64_t blocks = n_rows * nb;
  const int64_t row_bytes = (int64_t)d_in * bits / 8;
  const int ng = qw ? d_in / group : 0;

  for (int64_t base = (int64_t)blockIdx.x * RPC; base < blocks; base += (int64_t)gridDim.x * RPC) {
    const int64_t bi = base + rl;
    const bool active = bi < blocks;
    const int64_t r = active ? bi / nb : 0;
    const int k0 = active ? (int)(bi % nb) << LOGN : 0;
    __syncthreads();  // the previous iteration's readers are done with buf
    for (int i = t; i < G::NP; i += G::P) buf[i] = 0.f;
    __syncthreads();
    if (active) {
      int64_t b = row_ptr[r], e = row_ptr[r + 1];
      if (b < 0) b = 0;
      if (e > p) e = p;
      for (int64_t j = b + t; j < e; j += G::P) {
        const int k = col_idx[j] - k0;
        if ((unsigned)k < (unsigned)G::N) buf[G::phys(k)] = coef[j];
      }
    }
    __syncthreads();
    float v[G::R];
#pragma unroll
    for (int h = 0; h < (1 << G::HB); ++h) {
#pragma unroll
      for (int u = 0; u < 8; u += 4) {
        const float4 f = *reinterpret_cast<const float4 *>(buf + G::phys(G::eA(t, h << G::LV) + u));
        v[h * 8 + u] = f.x, v[h * 8 + u + 1] = f.y, v[h * 8 + u + 2] = f.z, v[h * 8 + u + 3] = f.w;
      }
    }
    butterflies_x2<G::R, 0, G::RB, 0>(v);
    __syncthreads();
#pragma unroll
    for (int h = 0; h < (1 << G::HB); ++h) {
#pragma unroll
      for (int u = 0; u < 8; u += 4)
        *reinterpret_cast<float4 *>(buf + G::phys(G::eA(t, h << G::LV) + u)) = make_float4(v[h * 8 + u], v[h * 8 + u + 1], v[h * 8 + u + 2], v[h * 8 + u + 3]);
    }
    __syncthreads();
#pragma unroll
    for (int q = 0; q < G::R; ++q) v[q] = buf[G::phys(G::eB(t, q))];
    butterflies_x2<G::R, 0, G::PB, (G::NB ? G::PB : 0)>(v);
    __syncthreads();
#pragma unroll
    for (int q = 0; q < G::R; ++q) buf[G::phys(G::eB(t, q))] = v[q] * scale;
    __syncthreads();
    if (active) {
#pragma unroll
      for (int h = 0; h < (1 << G::HB); ++h) {
        const int e = G::eA(t, h << G::LV);
        float f[8];
#pragma unroll
        for (int u = 0; u < 8; u += 4) {
          const float4 a = *reinterpret_cast<const float4 *>(buf + G::phys(e + u));
          f[u] = a.x, f[u + 1] = a.y, f[u + 2] = a.z, f[u + 3] = a.w;
        }
        const int k = k0 + e;
        if (qw) {
          const uint8_t *cp = qw + r * row_bytes + (int64_t)k * bits / 8;
          uint32_t w = 0;
          for (int bb = 0; bb < bits; ++bb) w |= (uint32_t)cp[bb] << (8 * bb);
          const uint32_t mask = (1u << bits) - 1u;
          const float sc = scales[r * ng + k / group], z = (float)zeros[r * ng + k / group];
#pragma unroll
          for (int i = 0; i < 8; ++i) f[i] += sc * ((float)((w >> (bits * i)) & mask) - z);
        }
        st_stream(out + r * d_in + k, io<__nv_bfloat16>::pack(f));
      }
    }
  }
}

// Same result as weff_rows_kernel, software-pipelined: while the butterflies of
// the current row blocks run, cp.async copies the next row blocks' inputs into
// shared memory: their CSR slice (column, coefficient; up to kWeffCsrCap
// entries per row, the rest is read directly) and their block of base-weight
// codes, scales and zero points (double-buffered, as the current block's are
// still needed by the final add). The row_ptr pair of the block after that is
// loaded into registers one iteration ahead. So no global-memory latency sits
// between the arithmetic phases. Requires 16-byte aligned code blocks and
// scales, 4-byte aligned zero points (checked by the launcher).
template <int LOGN>
constexpr int weff_csr_cap() {
  return (1 << LOGN) < 512 ? (1 << LOGN) : 512;
}

__host__ __device__ constexpr int round16(int x) { return (x + 15) & ~15; }

template <int LOGN>
__global__ void __launch_bounds__(kThreads, 2)
    weff_pipe_kernel(const int32_t *__restrict__ row_ptr, const int32_t *__restrict__ col_idx,
                     const float *__restrict__ coef, int64_t p, int d_in, int64_t n_rows, float scale, int bits,
                     int group, const uint8_t *__restrict__ qw, const float *__restrict__ scales,
                     const uint8_t *__restrict__ zeros, __nv_bfloat16 *__restrict__ out, int dq_stride) {
  using G = Geo<LOGN, 8>;
  constexpr int RPC = kThreads / G::P;
  constexpr int CAP = weff_csr_cap<LOGN>();
  extern __shared__ __align__(16) float smem[];
  const int rl = threadIdx.x / G::P;
  const int t = threadIdx.x % G::P;
  float *buf = smem + rl * G::NP;
  int32_t *my_k = reinterpret_cast<int32_t *>(smem + RPC * G::NP) + rl * CAP;
  float *my_v = reinterpret_cast<float *>(smem + RPC * G::NP + RPC * CAP) + rl * CAP;
  uint8_t *dq = reinterpret_cast<uint8_t *>(smem + RPC * G::NP + 2 * RPC * CAP);
  const int nb = d_in >> LOGN;
  const int64_t blocks = n_rows * nb;
  const int64_t row_bytes = (int64_t)d_in * bits / 8;
  const int ng = qw ? d_in / group : 0;
  const int gpb = qw ? G::N / group : 0;  // quantization groups per block
  const int qb = G::N * bits / 8;         // code bytes per block
  const int64_t stride = (int64_t)gridDim.x * RPC;

  auto row_range = [&](int64_t bi, int64_t &b, int64_t &e) {
    b = 0;
    e = 0;
    if (bi < blocks) {
      const int64_t r = bi / nb;
      b = row_ptr[r];
      e = row_ptr[r + 1];
      if (b < 0) b = 0;
      if (e > p) e = p;
      if (e < b) e = b;
    }
  };
  // this thread's share of the copies of block bi's inputs into row slot rl
  auto prefetch = [&](int64_t bi, int64_t b, int64_t e, int d) {
    if (bi < blocks) {
      const int n = (int)(e - b < CAP ? e - b : CAP);
      for (int j = t; j < n; j += G::P) {
        cp_async4(my_k + j, col_idx + b + j);
        cp_async4(my_v + j, coef + b + j);
      }
      if (qw) {
        const int64_t r = bi / nb;
        const int blk = (int)(bi % nb);
        uint8_t *dst = dq + ((size_t)d * RPC + rl) * dq_stride;
        const uint8_t *qsrc = qw + r * row_bytes + (int64_t)blk * qb;
        for (int c = t; c < qb / 16; c += G::P) cp_async16(dst + 16 * c, qsrc + 16 * c);
        const uint8_t *ssrc = reinterpret_cast<const uint8_t *>(scales + r * ng + (int64_t)blk * gpb);
        uint8_t *sdst = dst + round16(qb);
        for (int c = t; c < gpb / 4; c += G::P) cp_async16(sdst + 16 * c, ssrc + 16 * c);
        const uint8_t *zsrc = zeros + r * ng + (int64_t)blk * gpb;
        uint8_t *zdst = sdst + round16(gpb * 4);
        for (int c = t; c < gpb / 4; c += G::P) cp_async4(zdst + 4 * c, zsrc + 4 * c);
      }
    }
    cp_async_commit();
  };

  int64_t bi = (int64_t)blockIdx.x * RPC + rl;
  int64_t b, e, b_next, e_next;
  row_range(bi, b, e);
  prefetch(bi, b, e, 0);
  row_range(bi + stride, b_next, e_next);
  int d = 0;
  for (int64_t base = (int64_t)blockIdx.x * RPC; base < blocks; base += stride, d ^= 1) {
    const bool active = bi < blocks;
    const int64_t r = active ? bi / nb : 0;
    const int k0 = active ? (int)(bi % nb) << LOGN : 0;
    cp_async_wait_all();
    __syncthreads();  // this block's inputs are staged; the previous iteration is done with buf
    for (int i = 4 * t; i < G::NP; i += 4 * G::P) *reinterpret_cast<float4 *>(buf + i) = make_float4(0.f, 0.f, 0.f, 0.f);
    __syncthreads();
    if (active) {
      const int n = (int)(e - b < CAP ? e - b : CAP);
      for (int j = t; j < n; j += G::P) {
        const int k = my_k[j] - k0;
        if ((unsigned)k < (unsigned)G::N) buf[G::phys(k)] = my_v[j];
      }
      for (int64_t j = b + CAP + t; j < e; j += G::P) {  // entries beyond the staged ones
        const int k = col_idx[j] - k0;
        if ((unsigned)k < (unsigned)G::N) buf[G::phys(k)] = coef[j];
      }
    }
    __syncthreads();  // the staged CSR slice is consumed: copy the next block's inputs
    const int64_t bi_next = bi + stride;
    prefetch(bi_next, b_next, e_next, d ^ 1);
    bi = bi_next;
    b = b_next;
    e = e_next;
    row_range(bi + stride, b_next, e_next);  // used one iteration from now

    float v[G::R];
#pragma unroll
    for (int h = 0; h < (1 << G::HB); ++h) {
#pragma unroll
      for (int u = 0; u < 8; u += 4) {
        const float4 f = *reinterpret_cast<const float4 *>(buf + G::phys(G::eA(t, h << G::LV) + u));
        v[h * 8 + u] = f.x, v[h * 8 + u + 1] = f.y, v[h * 8 + u + 2] = f.z, v[h * 8 + u + 3] = f.w;
      }
    }
    butterflies_x2<G::R, 0, G::RB, 0>(v);
    __syncthreads();
#pragma unroll
    for (int h = 0; h < (1 << G::HB); ++h) {
#pragma unroll
      for (int u = 0; u < 8; u += 4)
        *reinterpret_cast<float4 *>(buf + G::phys(G::eA(t, h << G::LV) + u)) = make_float4(v[h * 8 + u], v[h * 8 + u + 1], v[h * 8 + u + 2], v[h * 8 + u + 3]);
    }
    __syncthreads();
#pragma unroll
    for (int q = 0; q < G::R; ++q) v[q] = buf[G::phys(G::eB(t, q))];
    butterflies_x2<G::R, 0, G::PB, (G::NB ? G::PB : 0)>(v);
    __syncthreads();
#pragma unroll
    for (int q = 0; q < G::R; ++q) buf[G::phys(G::eB(t, q))] = v[q] * scale;
    __syncthreads();
    if (active) {
      const uint8_t *dqc = dq + ((size_t)d * RPC + rl) * dq_stride;
      const float *s_sc = reinterpret_cast<const float *>(dqc + round16(qb));
      const uint8_t *s_z = dqc + round16(qb) + round16(gpb * 4);
#pragma unroll
      for (int h = 0; h < (1 << G::HB); ++h) {
        const int el = G::eA(t, h << G::LV);
        float f[8];
#pragma unroll
        for (int u = 0; u < 8; u += 4) {
          const float4 a = *reinterpret_cast<const float4 *>(buf + G::phys(el + u));
          f[u] = a.x, f[u + 1] = a.y, f[u + 2] = a.z, f[u + 3] = a.w;
        }
        if (qw) {
          const uint8_t *cp = dqc + el * bits / 8;
          uint32_t w;
          if (bits == 4) {
            w = *reinterpret_cast<const uint32_t *>(cp);
          } else if (bits == 2) {
            w = *reinterpret_cast<const uint16_t *>(cp);
          } else {
            w = 0;
            for (int bb = 0; bb < bits; ++bb) w |= (uint32_t)cp[bb] << (8 * bb);
          }
          const uint32_t mask = (1u << bits) - 1u;
          const int g = el / group;
          const float sc = s_sc[g], z = (float)s_z[g];
#pragma unroll
          for (int i = 0; i < 8; ++i) f[i] += sc * ((float)((w >> (bits * i)) & mask) - z);
        }
        st_stream(out + r * d_in + k0 + el, io<__nv_bfloat16>::pack(f));
      }
    }
  }
  cp_async_wait_all();  // no copy is left in flight when the CTA exits
}

// W_eff blocks of 2048 or 4096 columns, ring-fed like fwht_ring_kernel: a CTA
// of 64 threads takes 64/P blocks per iteration; one thread copies each
// block's code block, scales, zero points and a 16-byte aligned window of its
// row's CSR slice (column, coefficient) into an S-slot shared-memory ring with
// bulk copies, S - 1 iterations ahead (a slot is refilled once its codes have
// been used by the final add). The row_ptr pair of the block to copy next is
// loaded one iteration before it is needed. Entries past the window (rows of
// more than kWeffWin - 8 entries, or the last entries of the arrays) are read
// directly. Arithmetic as weff_pipe_kernel: scatter into the padded buffer,
// two butterfly phases, base weight added in fp32 in phase-A layout, one bf16
// rounding. Needs the 16-byte alignments checked by run_weff.
constexpr int kWeffWin = 520;  // CSR window entries per block (a multiple of 4)

struct WeffRingLayout {
  int qb, gpb;         // code bytes and quantization groups per block
  int o_sc, o_z, o_k;  // byte offsets of scales, zero points and the CSR window in a block's part of a slot
  int blk;             // bytes of a block's part of a slot
  __host__ __device__ WeffRingLayout(int n, int bits, int group) {
    qb = n * bits / 8;
    gpb = n / group;
    o_sc = round16(qb);
    o_z = o_sc + round16(gpb * 4);
    o_k = o_z + round16(gpb);
    blk = o_k + 2 * kWeffWin * 4;
  }
};

template <int LOGN, int S>
__global__ void __launch_bounds__(64) weff_ring_kernel(const int32_t *__restrict__ row_ptr,
                                                       const int32_t *__restrict__ col_idx,
                                                       const float *__restrict__ coef, int64_t p, int d_in,
                                                       int64_t n_rows, float scale, int bits, int group,
                                                       const uint8_t *__restrict__ qw, const float *__restrict__ scales,
                                                       const uint8_t *__restrict__ zeros,
                                                       __nv_bfloat16 *__restrict__ out, unsigned int *err) {
  using G = Geo<LOGN, 8>;
  static_assert(G::P >= 32, "one warp or more per block");
  constexpr int RW = 64, RPW = RW / G::P;
  extern __shared__ __align__(128) unsigned char smem_raw[];
  float *buf_all = reinterpret_cast<float *>(smem_raw);
  const WeffRingLayout L(G::N, bits, group);
  const int slot_bytes = RPW * L.blk;
  unsigned char *ring = smem_raw + ((RPW * G::NP * 4 + 127) & ~127);
  uint64_t *full = reinterpret_cast<uint64_t *>(ring + S * slot_bytes);
  int *meta = reinterpret_cast<int *>(full + S);  // per slot and block: b, e, a0, a1
  const int tid = threadIdx.x, rl = tid / G::P, t = tid % G::P;
  float *buf = buf_all + rl * G::NP;
  const int nb = d_in >> LOGN;
  const int64_t blocks = n_rows * nb;
  const int64_t row_bytes = (int64_t)d_in * bits / 8;
  const int ng = d_in / group;
  const int64_t stride = (int64_t)gridDim.x * RPW;
  const int64_t first = (int64_t)blockIdx.x * RPW;
  const int64_t iters = first < blocks ? (blocks - first + stride - 1) / stride : 0;
  const int64_t p4 = p & ~(int64_t)3;

  // thread 0: copy the inputs of iteration it (row_ptr pairs in rp) into its slot
  auto issue = [&](int64_t it, const int *rp) {
    const int s = (int)(it % S);
    unsigned char *sl = ring + s * slot_bytes;
    uint32_t bytes = 0;
    int a[RPW][2];
    for (int q = 0; q < RPW; ++q) {
      const int64_t bi = first + it * stride + q;
      int b = 0, e = 0, a0 = 0, a1 = 0;
      if (bi < blocks) {
        b = rp[2 * q];
        e = rp[2 * q + 1];
        if (b < 0) b = 0;
        if (e > p) e = (int)p;
        if (e < b) e = b;
        a0 = b & ~3;
        int64_t hi = ((int64_t)e + 3) & ~(int64_t)3;
        if (hi > p4) hi = p4;
        if (hi > a0 + kWeffWin) hi = a0 + kWeffWin;
        a1 = hi > a0 ? (int)hi : a0;
        bytes += L.qb + L.gpb * 4 + L.gpb + 8 * (a1 - a0);
      }
      int *m = meta + 4 * (s * RPW + q);
      m[0] = b, m[1] = e, m[2] = a0, m[3] = a1;
      a[q][0] = a0, a[q][1] = a1;
    }
    bulk::fence_proxy();
    const uint32_t bar = bulk::saddr(full + s);
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes) : "memory");
    for (int q = 0; q < RPW; ++q) {
      const int64_t bi = first + it * stride + q;
      if (bi >= blocks) continue;
      const int64_t r = bi / nb;
      const int kb = (int)(bi % nb);
      unsigned char *d = sl + q * L.blk;
      bulk::copy(bulk::saddr(d), qw + r * row_bytes + (int64_t)kb * L.qb, L.qb, bar);
      bulk::copy(bulk::saddr(d + L.o_sc), scales + r * ng + (int64_t)kb * L.gpb, L.gpb * 4, bar);
      bulk::copy(bulk::saddr(d + L.o_z), zeros + r * ng + (int64_t)kb * L.gpb, L.gpb, bar);
      const int a0 = a[q][0], a1 = a[q][1];
      if (a1 > a0) {
        bulk::copy(bulk::saddr(d + L.o_k), col_idx + a0, 4 * (a1 - a0), bar);
        bulk::copy(bulk::saddr(d + L.o_k + 4 * kWeffWin), coef + a0, 4 * (a1 - a0), bar);
      }
    }
  };
  auto load_rp = [&](int64_t it, int *rp) {  // row_ptr pairs of iteration it's blocks
    for (int q = 0; q < RPW; ++q) {
      const int64_t bi = first + it * stride + q;
      rp[2 * q] = rp[2 * q + 1] = 0;
      if (it < iters && bi < blocks) {
        const int64_t r = bi / nb;
        rp[2 * q] = row_ptr[r];
        rp[2 * q + 1] = row_ptr[r + 1];
      }
    }
  };

  int rp_next[2 * RPW];
  if (tid == 0) {
#pragma unroll
    for (int s = 0; s < S; ++s) bulk::init(bulk::saddr(full + s), 1);
    bulk::fence_init();
  }
  __syncthreads();
  if (tid == 0) {
    for (int64_t it = 0; it < S && it < iters; ++it) {
      load_rp(it, rp_next);
      issue(it, rp_next);
    }
  }

  for (int64_t it = 0; it < iters; ++it) {
    const int s = (int)(it % S);
    if (tid == 0) load_rp(it + S, rp_next);  // consumed at the end of this iteration
    const bool ok = bulk::wait(bulk::saddr(full + s), (uint32_t)((it / S) & 1));
    if (__syncthreads_or(!ok)) {
      if (tid == 0) {
        atomicOr(err, 0x400u);
        for (int64_t j = it; j < iters && j < it + S; ++j)
          (void)bulk::wait(bulk::saddr(full + (int)(j % S)), (uint32_t)((j / S) & 1));
      }
      return;
    }
    const unsigned char *sl = ring + s * slot_bytes + rl * L.blk;
    const int64_t bi = first + it * stride + rl;
    const bool active = bi < blocks;
    const int64_t r = active ? bi / nb : 0;
    const int k0 = active ? (int)(bi % nb) << LOGN : 0;
    for (int i = 4 * tid; i < RPW * G::NP; i += 4 * RW)
      *reinterpret_cast<float4 *>(buf_all + i) = make_float4(0.f, 0.f, 0.f, 0.f);
    __syncthreads();
    if (active) {
      const int *m = meta + 4 * (s * RPW + rl);
      const int b = m[0], e = m[1], a0 = m[2], a1 = m[3];
      const int32_t *wk = reinterpret_cast<const int32_t *>(sl + L.o_k);
      const float *wv = reinterpret_cast<const float *>(sl + L.o_k + 4 * kWeffWin);
      for (int j = b + t; j < e; j += G::P) {
        const bool in_win = j < a1;
        const int k = (in_win ? wk[j - a0] : col_idx[j]) - k0;
        if ((unsigned)k < (unsigned)G::N) buf[G::phys(k)] = in_win ? wv[j - a0] : coef[j];
      }
    }
    __syncthreads();
    float v[G::R];
#pragma unroll
    for (int h = 0; h < (1 << G::HB); ++h) {
#pragma unroll
      for (int u = 0; u < 8; u += 4) {
        const float4 f = *reinterpret_cast<const float4 *>(buf + G::phys(G::eA(t, h << G::LV) + u));
        v[h * 8 + u] = f.x, v[h * 8 + u + 1] = f.y, v[h * 8 + u + 2] = f.z, v[h * 8 + u + 3] = f.w;
      }
    }
    butterflies_x2<G::R, 0, G::RB, 0>(v);
#pragma unroll
    for (int h = 0; h < (1 << G::HB); ++h) {
#pragma unroll
      for (int u = 0; u < 8; u += 4)
        *reinterpret_cast<float4 *>(buf + G::phys(G::eA(t, h << G::LV) + u)) =
            make_float4(v[h * 8 + u], v[h * 8 + u + 1], v[h * 8 + u + 2], v[h * 8 + u + 3]);
    }
    __syncthreads();
#pragma unroll
    for (int q = 0; q < G::R; ++q) v[q] = buf[G::phys(G::eB(t, q))];
    butterflies_x2<G::R, 0, G::PB, (G::NB ? G::PB : 0)>(v);
    __syncthreads();
#pragma unroll
    for (int q = 0; q < G::R; ++q) buf[G::phys(G::eB(t, q))] = v[q] * scale;
    __syncthreads();
    if (active) {
      const uint8_t *cq = sl;
      const float *s_sc = reinterpret_cast<const float *>(sl + L.o_sc);
      const uint8_t *s_z = sl + L.o_z;
      const uint32_t mask = (1u << bits) - 1u;
#pragma unroll
      for (int h = 0; h < (1 << G::HB); ++h) {
        const int el = G::eA(t, h << G::LV);
        float f[8];
#pragma unroll
        for (int u = 0; u < 8; u += 4) {
          const float4 a = *reinterpret_cast<const float4 *>(buf + G::phys(el + u));
          f[u] = a.x, f[u + 1] = a.y, f[u + 2] = a.z, f[u + 3] = a.w;
        }
        const uint8_t *cp = cq + el * bits / 8;
        uint32_t w;
        if (bits == 4) {
          w = *reinterpret_cast<const uint32_t *>(cp);
        } else if (bits == 2) {
          w = *reinterpret_cast<const uint16_t *>(cp);
        } else {
          w = 0;
          for (int bb = 0; bb < bits; ++bb) w |= (uint32_t)cp[bb] << (8 * bb);
        }
        const int g = el / group;
        const float sc = s_sc[g], z = (float)s_z[g];
#pragma unroll
        for (int i = 0; i < 8; ++i) f[i] += sc * ((float)((w >> (bits * i)) & mask) - z);
        st_stream(out + r * d_in + k0 + el, io<__nv_bfloat16>::pack(f));
      }
    }
    __syncthreads();  // slot s and the buffer are free
    if (tid == 0 && it + S < iters) issue(it + S, rp_next);
  }
}

constexpr int kWeffRingSlots = 3;

template <int LOGN>
cudaError_t run_weff_ring(const int32_t *row_ptr, const int32_t *col_idx, const float *coef, int64_t p, int d_in,
                          int64_t n_rows, float scale, int bits, int group, const uint8_t *qw, const float *scales,
                          const uint8_t *zeros, __nv_bfloat16 *out, cudaStream_t s) {
  using G = Geo<LOGN, 8>;
  constexpr int S = kWeffRingSlots, RPW = 64 / G::P;
  const WeffRingLayout L(G::N, bits, group);
  const size_t smem = (((size_t)RPW * G::NP * 4 + 127) & ~(size_t)127) + (size_t)S * RPW * L.blk + (size_t)S * 8 +
                      (size_t)S * RPW * 16;
  auto k = weff_ring_kernel<LOGN, S>;
  cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  int occ = 0;
  e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, k, 64, smem);
  if (e != cudaSuccess) return e;
  if (occ < 1) occ = 1;
  const int64_t blocks = n_rows * (d_in >> LOGN);
  const int64_t need = cdiv(blocks, RPW), cap = (int64_t)sm_count() * occ;
  k<<<(unsigned)(need < cap ? need : cap), 64, smem, s>>>(row_ptr, col_idx, coef, p, d_in, n_rows, scale, bits, group,
                                                         qw, scales, zeros, out, device_error_word());
  return cudaGetLastError();
}

template <int LOGN>
cudaError_t run_weff(const int32_t *row_ptr, const int32_t *col_idx, const float *coef, int64_t p, int d_in,
                     int64_t n_rows, float scale, int bits, int group, const uint8_t *qw, const float *scales,
                     const uint8_t *zeros, __nv_bfloat16 *out, cudaStream_t s) {
  using G = Geo<LOGN, 8>;
  if constexpr (LOGN >= 11) {
    // the ring-fed kernel copies every per-block input with 16-byte aligned bulk copies
    const int gpb = G::N / group, ng = d_in / group;
    const bool ring = qw && (int64_t)G::N * bits % 128 == 0 && (int64_t)d_in * bits % 128 == 0 && gpb % 16 == 0 &&
                      ng % 16 == 0 && aligned16(qw) && aligned16(scales) && aligned16(zeros) && aligned16(col_idx) &&
                      aligned16(coef);
    if (ring)
      return run_weff_ring<LOGN>(row_ptr, col_idx, coef, p, d_in, n_rows, scale, bits, group, qw, scales, zeros, out,
                                 s);
  }
  constexpr int RPC = kThreads / G::P;
  const int64_t blocks = n_rows * (d_in >> LOGN);
  // the pipelined kernel copies code blocks and scales in 16-byte pieces and
  // zero points in 4-byte pieces
  bool pipe = true;
  int dq_stride = 0;
  if (qw) {
    const int64_t qb = (int64_t)G::N * bits / 8, row_bytes = (int64_t)d_in * bits / 8;
    const int gpb = G::N / group, ng = d_in / group;
    pipe = qb % 16 == 0 && row_bytes % 16 == 0 && gpb % 4 == 0 && ng % 4 == 0 &&
           reinterpret_cast<uintptr_t>(qw) % 16 == 0 && reinterpret_cast<uintptr_t>(scales) % 16 == 0 &&
           reinterpret_cast<uintptr_t>(zeros) % 4 == 0;
    dq_stride = round16((int)qb) + round16(gpb * 4) + round16(gpb);
  }
  if (pipe) {
    const size_t smem = (size_t)RPC * G::NP * sizeof(float) + 2ull * RPC * weff_csr_cap<LOGN>() * 4 +
                        2ull * RPC * dq_stride;
    auto k = weff_pipe_kernel<LOGN>;
    cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    int occ = 0;
    e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, k, kThreads, smem);
    if (e != cudaSuccess) return e;
    if (occ < 1) occ = 1;
    const int64_t need = cdiv(blocks, RPC);
    const int64_t cap = (int64_t)sm_count() * occ;
    k<<<(unsigned)(need < cap ? need : cap), kThreads, smem, s>>>(row_ptr, col_idx, coef, p, d_in, n_rows, scale,
                                                                 bits, group, qw, scales, zeros, out, dq_stride);
    return cudaGetLastError();
  }
  const size_t smem = (size_t)RPC * G::NP * sizeof(float);
  auto k = weff_rows_kernel<LOGN>;
  cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  int occ = 0;
  e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, k, kThreads, smem);
  if (e != cudaSuccess) return e;
  if (occ < 1) occ = 1;
  const int64_t need = cdiv(blocks, RPC);
  const int64_t cap = (int64_t)sm_count() * occ;
  k<<<(unsigned)(need < cap ? need : cap), kThreads, smem, s>>>(row_ptr, col_idx, coef, p, d_in, n_rows, scale, bits,
                                                               group, qw, scales, zeros, out);
  return cudaGetLastError();
}

template <int LOGN, typename Tin, typename Tout, int S>
cudaError_t run_ring(const Tin *x, Tout *z, int64_t rows, float scale, cudaStream_t s) {
  constexpr int V = (sizeof(Tin) == 2 || sizeof(Tout) == 2) ? 8 : 4;
  using G = Geo<LOGN, V>;
  using RG = RingGeo<LOGN, V>;
  const size_t smem = (size_t)RG::template buf_bytes<Tout>() + (size_t)S * RG::RPW * G::N * sizeof(Tin) + (size_t)S * 8;
  auto k = fwht_ring_kernel<LOGN, V, Tin, Tout, S>;
  static bool attr_done[64] = {};  // per instantiation and device
  const int slot = device_slot();
  if (!attr_done[slot]) {
    cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    attr_done[slot] = true;
  }
  int occ = 0;
  cudaError_t e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, k, RG::RW, smem);
  if (e != cudaSuccess) return e;
  if (occ < 1) occ = 1;
  const int64_t need = cdiv(rows, RG::RPW);
  const int64_t cap = (int64_t)sm_count() * occ;
  const int grid = (int)(need < cap ? need : cap);
  k<<<grid, RG::RW, smem, s>>>(x, z, rows, scale, device_error_word(), ring_wait_ns());
  return cudaGetLastError();
}

template <int LOGN, typename Tin, typename Tout>
cudaError_t run_small(const Tin *x, Tout *z, int64_t rows, float scale, cudaStream_t s) {
  const int64_t need = cdiv(rows, kThreads);
  const int64_t cap = (int64_t)sm_count() * 8;
  fwht_small_kernel<LOGN, Tin, Tout><<<(int)(need < cap ? need : cap), kThreads, 0, s>>>(x, z, rows, scale);
  return cudaGetLastError();
}

template <typename Tin, typename Tout>
cudaError_t run_large(const Tin *x, Tout *z, int64_t rows, int logn, float scale, cudaStream_t s) {
  const size_t smem = sizeof(float) << logn;
  auto k = fwht_large_kernel<Tin, Tout>;
  cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  const int64_t cap = (int64_t)sm_count() * 2;
  k<<<(int)(rows < cap ? rows : cap), 512, smem, s>>>(x, z, rows, logn, scale);
  return cudaGetLastError();
}

template <typename Tin, typename Tout>
cudaError_t dispatch(const void *xv, void *zv, int64_t rows, int logn, float scale, cudaStream_t s) {
  const Tin *x = static_cast<const Tin *>(xv);
  Tout *z = static_cast<Tout *>(zv);
  switch (logn) {
    case 1: return run_small<1>(x, z, rows, scale, s);
    case 2: return run_small<2>(x, z, rows, scale, s);
    case 3: return run_small<3>(x, z, rows, scale, s);
    case 4: return run_small<4>(x, z, rows, scale, s);
    case 5: return run_small<5>(x, z, rows, scale, s);
    case 6: return run_small<6>(x, z, rows, scale, s);
    case 7: return run_ring<7, Tin, Tout, kRingSlots>(x, z, rows, scale, s);
    case 8: return run_ring<8, Tin, Tout, kRingSlots>(x, z, rows, scale, s);
    case 9: return run_ring<9, Tin, Tout, kRingSlots>(x, z, rows, scale, s);
    case 10: return run_ring<10, Tin, Tout, kRingSlots>(x, z, rows, scale, s);
    case 11: return run_ring<11, Tin, Tout, kRingSlots>(x, z, rows, scale, s);
    case 12: return run_ring<12, Tin, Tout, kRingSlots>(x, z, rows, scale, s);
    default: return run_large(x, z, rows, logn, scale, s);
  }
}

}  // namespace

cudaError_t launch_fwht(qwha_dtype din, qwha_dtype dout, const void *x, void *z, int64_t blocks,
                        int logn, float scale, cudaStream_t s) {
  if (blocks <= 0) return cudaSuccess;
  using bf = __nv_bfloat16;
  if (din == QWHA_F32 && dout == QWHA_F32) return dispatch<float, float>(x, z, blocks, logn, scale, s);
  if (din == QWHA_BF16 && dout == QWHA_BF16) return dispatch<bf, bf>(x, z, blocks, logn, scale, s);
  if (din == QWHA_F32 && dout == QWHA_BF16) return dispatch<float, bf>(x, z, blocks, logn, scale, s);
  return dispatch<bf, float>(x, z, blocks, logn, scale, s);
}

}  // namespace qwha

namespace qwha {

bool weff_rows_supported(int logn) { return logn >= 7 && logn <= 12; }

cudaError_t launch_weff_rows(const int32_t *row_ptr, const int32_t *col_idx, const float *coef, int64_t p, int d_in,
                             int64_t n_rows, int logn, float scale, int bits, int group, const uint8_t *qw,
                             const float *scales, const uint8_t *zeros, void *out, cudaStream_t s) {
  __nv_bfloat16 *o = static_cast<__nv_bfloat16 *>(out);
  switch (logn) {
    case 7: return run_weff<7>(row_ptr, col_idx, coef, p, d_in, n_rows, scale, bits, group, qw, scales, zeros, o, s);
    case 8: return run_weff<8>(row_ptr, col_idx, coef, p, d_in, n_rows, scale, bits, group, qw, scales, zeros, o, s);
    case 9: return run_weff<9>(row_ptr, col_idx, coef, p, d_in, n_rows, scale, bits, group, qw, scales, zeros, o, s);
    case 10: return run_weff<10>(row_ptr, col_idx, coef, p, d_in, n_rows, scale, bits, group, qw, scales, zeros, o, s);
    case 11: return run_weff<11>(row_ptr, col_idx, coef, p, d_in, n_rows, scale, bits, group, qw, scales, zeros, o, s);
    case 12: return run_weff<12>(row_ptr, col_idx, coef, p, d_in, n_rows, scale, bits, group, qw, scales, zeros, o, s);
  }
  return cudaErrorInvalidValue;
}

}  // namespace qwha
