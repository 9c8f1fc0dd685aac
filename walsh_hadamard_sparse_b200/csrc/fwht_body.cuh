// Register/shared-memory row Walsh-Hadamard transform shared by the
// standalone transform kernels (fwht.cu) and the forward GEMM, whose extra
// warps transform X while the tensor cores run (gemm.cu). See fwht.cu for the
// layout (phase A / phase B index maps, padded transpose buffer).
#pragma once

#include "common.cuh"

namespace qwha {

template <int LOGN, int V>
struct Geo {
  static constexpr int N = 1 << LOGN;
  static constexpr int LV = V == 8 ? 3 : 2;
  static constexpr int RB = (LOGN + 1) / 2;
  static constexpr int R = 1 << RB;
  static constexpr int PB = LOGN - RB;
  static constexpr int P = 1 << PB;
  static constexpr int NB = 2 * RB - LOGN;  // batch bits in phase B (0 or 1)
  static constexpr int HB = RB - LV;        // high bits in phase-A registers
  // Transpose-buffer row: blocks of 4P floats, one per (high field, 16-byte
  // half u of a narrow vector), each followed by 4 padding floats; rows that
  // share a warp (P < 32) are further padded so that they start P banks apart.
  static constexpr int BLK = 4 * P + 4;
  static constexpr int RP = P < 32 ? ((P - V * (1 << HB)) & 31) : 0;
  static constexpr int NP = N + V * (1 << HB) + RP;  // floats per row
  static_assert(HB >= NB && HB >= 0 && PB >= LV && P >= 8, "row too short for this layout");

  // element index of register q of thread t, phase A
  __device__ __forceinline__ static int eA(int t, int q) {
    return (q & (V - 1)) | (t << LV) | ((q >> LV) << (LV + PB));
  }
  // element index of register q of thread t, phase B
  __device__ __forceinline__ static int eB(int t, int q) {
    return (t & (V - 1)) | ((q & (P - 1)) << LV) | ((t >> LV) << (LV + PB)) |
           ((q >> PB) << (LV + PB + HB - NB));
  }
  // Position of element e in its row of the transpose buffer. The low field
  // splits into i (the 4 floats of a 16-byte access) and u (which 16-byte half
  // of a narrow vector); u and the high field select the block, the middle
  // field m the 16-byte slot in it. Phase-A 16-byte accesses (fixed h, u;
  // lanes = consecutive m) cover 128 contiguous bytes per quarter warp;
  // phase-B scalar accesses (fixed m; lanes = i, u, high bits, rows) meet 32
  // distinct banks thanks to the padding. Every position is a per-thread base
  // plus a compile-time offset in both phases.
  __device__ __forceinline__ static int phys(int e) {
    const int i = e & 3, m = (e >> LV) & (P - 1), ub = ((e & (V - 1)) >> 2) | ((e >> (LV + PB)) << (LV - 2));
    return i + 4 * m + BLK * ub;
  }
};

template <typename T, int V>
__device__ __forceinline__ void store_group(T *p, const float *i) {
  constexpr int NU = V * (int)sizeof(T) / 16;
#pragma unroll
  for (int u = 0; u < NU; ++u) st_stream(p + u * io<T>::kVec, io<T>::pack(i + u * io<T>::kVec));
}

// Butterflies on register-index bits [B0, B0 + NBITS) of v[0..R).
template <int R, int B0, int NBITS>
__device__ __forceinline__ void butterflies(float *v) {
#pragma unroll
  for (int b = B0; b < B0 + NBITS; ++b) {
    const int h = 1 << b;
#pragma unroll
    for (int q = 0; q < R; ++q)
      if (!(q & h)) {
        const float a = v[q], c = v[q + h];
        v[q] = a + c;
        v[q + h] = a - c;
      }
  }
}

// Two butterflies at once with the packed fp32x2 add/sub of sm_100:
// (a0, a1), (b0, b1) <- (a0 + b0, a1 + b1), (a0 - b0, a1 - b1).
__device__ __forceinline__ void bfly2(float &a0, float &a1, float &b0, float &b1) {
  unsigned long long a, b, sum, dif;
  asm("mov.b64 %0, {%1, %2};" : "=l"(a) : "f"(a0), "f"(a1));
  asm("mov.b64 %0, {%1, %2};" : "=l"(b) : "f"(b0), "f"(b1));
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(sum) : "l"(a), "l"(b));
  asm("sub.rn.f32x2 %0, %1, %2;" : "=l"(dif) : "l"(a), "l"(b));
  asm("mov.b64 {%0, %1}, %2;" : "=f"(a0), "=f"(a1) : "l"(sum));
  asm("mov.b64 {%0, %1}, %2;" : "=f"(b0), "=f"(b1) : "l"(dif));
}

// Same result as butterflies<R, B0, NBITS>, registers paired along index bit PB:
// stages on other bits run two butterflies per packed add and sub; a stage on
// PB itself (if in range) runs scalar.
template <int R, int B0, int NBITS, int PB>
__device__ __forceinline__ void butterflies_x2(float *v) {
  constexpr int P = 1 << PB;
#pragma unroll
  for (int b = B0; b < B0 + NBITS; ++b) {
    const int h = 1 << b;
    if (b == PB) {
#pragma unroll
      for (int q = 0; q < R; ++q)
        if (!(q & h)) {
          const float a = v[q], c = v[q + h];
          v[q] = a + c;
          v[q + h] = a - c;
        }
    } else {
#pragma unroll
      for (int q = 0; q < R; ++q)
        if (!(q & h) && !(q & P)) bfly2(v[q], v[q + P], v[q + h], v[q + h + P]);
    }
  }
}

__device__ __forceinline__ void cp_async16(void *smem_dst, const void *gmem_src) {
  const uint32_t d = static_cast<uint32_t>(__cvta_generic_to_shared(smem_dst));
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(d), "l"(gmem_src) : "memory");
}
__device__ __forceinline__ void cp_async4(void *smem_dst, const void *gmem_src) {
  const uint32_t d = static_cast<uint32_t>(__cvta_generic_to_shared(smem_dst));
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(d), "l"(gmem_src) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_group 0;" ::: "memory"); }

// The row transform run by a group of NT threads (tid in [0, NT)) that
// synchronise with `bar` (the whole CTA, or a named barrier when the group is
// part of a larger CTA). The group is number `cta` of `n_cta` such groups and
// takes rows cta*RPC, (cta + n_cta)*RPC, ... The input rows of the next
// iteration are copied into a shared-memory staging buffer with cp.async while
// the current rows are transformed; phase A then reads its 16-byte vectors
// from shared memory. smem: NT/P rows x (Geo::NP floats + n input values).
template <int LOGN, int V, typename Tin, typename Tout, int NT, typename Bar>
__device__ __forceinline__ void fwht_rows_body(const Tin *__restrict__ x, Tout *__restrict__ z, int64_t rows,
                                               float scale, float *smem, int tid, int cta, int n_cta,
                                               Bar bar) {
  using G = Geo<LOGN, V>;
  static_assert(G::P <= NT, "row too long for this group of threads");
  constexpr int RPC = NT / G::P;  // rows per group iteration
  constexpr int ROW_CHUNKS = G::N * (int)sizeof(Tin) / 16;
  const int rl = tid / G::P;
  const int t = tid % G::P;
  float *buf = smem + rl * G::NP;
  Tin *stage = reinterpret_cast<Tin *>(smem + RPC * G::NP);

  auto prefetch = [&](int64_t first) {
    const int64_t left = rows - first;
    const int nrow = left < RPC ? (int)left : RPC;
    const char *src = reinterpret_cast<const char *>(x + first * G::N);
    char *dst = reinterpret_cast<char *>(stage);
    for (int c = tid; c < nrow * ROW_CHUNKS; c += NT) cp_async16(dst + 16 * c, src + 16 * (int64_t)c);
    cp_async_commit();
  };

  int64_t base = (int64_t)cta * RPC;
  if (base < rows) prefetch(base);
  for (; base < rows; base += (int64_t)n_cta * RPC) {
    const int64_t row = base + rl;
    const bool active = row < rows;
    cp_async_wait_all();
    bar();  // this iteration's rows are staged; last iteration's readers of buf are done
    float v[G::R];
    if (active) {
      const Tin *xr = stage + rl * G::N;
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
        *reinterpret_cast<float4 *>(buf + G::phys(G::eA(t, h << G::LV) + u)) =
            make_float4(v[h * V + u], v[h * V + u + 1], v[h * V + u + 2], v[h * V + u + 3]);
    }
    bar();  // phase A is in buf, and every thread has read its staged input: fetch the next rows
    if (base + (int64_t)n_cta * RPC < rows) prefetch(base + (int64_t)n_cta * RPC);
#pragma unroll
    for (int q = 0; q < G::R; ++q) v[q] = buf[G::phys(G::eB(t, q))];
    butterflies_x2<G::R, 0, G::PB, (G::NB ? G::PB : 0)>(v);
    bar();  // all phase-B reads done before the buffer is reused

    // scaled fp32 back through the buffer (the phase-B pattern is conflict-free),
    // then phase-A vectors are packed once into the output type
#pragma unroll
    for (int q = 0; q < G::R; ++q) buf[G::phys(G::eB(t, q))] = v[q] * scale;
    bar();
    if (active) {
      Tout *zr = z + row * G::N;
#pragma unroll
      for (int h = 0; h < (1 << G::HB); ++h) {
        const int e = G::eA(t, h << G::LV);
        float o[V];
#pragma unroll
        for (int u = 0; u < V; u += 4) {
          const float4 f = *reinterpret_cast<const float4 *>(buf + G::phys(e + u));
          o[u] = f.x, o[u + 1] = f.y, o[u + 2] = f.z, o[u + 3] = f.w;
        }
        store_group<Tout, V>(zr + e, o);
      }
    }
  }
}

}  // namespace qwha
