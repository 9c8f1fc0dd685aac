// Internal helpers shared by the CUDA translation units of libqwha.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "qwha.h"

namespace qwha {

// Record a message for qwha_last_error() of this thread and return `s`.
qwha_status fail(qwha_status s, const char *fmt, ...);

// Map a CUDA error from a launch or runtime call to QWHA_ERR_CUDA.
qwha_status cuda_status(cudaError_t e, const char *what);

inline bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
inline bool is_pow2(int64_t v) { return v > 0 && (v & (v - 1)) == 0; }
inline int ilog2(int64_t v) {
  int r = 0;
  while ((int64_t(1) << r) < v) ++r;
  return r;
}
inline int64_t cdiv(int64_t a, int64_t b) { return (a + b - 1) / b; }
inline size_t align_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

int sm_count();  // multiprocessors of the current device
int device_slot();  // index of the current device in [0, 64) (0 if unreadable), for per-device caches

// Device error word for bounded waits (set by kernels, read by
// qwha_check_stream_status). One per device, in __device__ memory.
unsigned int *device_error_word();

// Limit of the row-transform kernel's main-loop waits, in ns (2 s unless a
// test lowered it through qwha_debug_wait_limit_ns).
uint64_t ring_wait_ns();

// ---------------------------------------------------------------- device side

__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }

// Two floats to a packed bf16x2 word (round to nearest even); `a` in the low half.
__device__ __forceinline__ uint32_t pack_bf16x2(float a, float b) {
  __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
  return *reinterpret_cast<uint32_t *>(&h);
}

template <typename T>
struct io;

template <>
struct io<float> {
  static constexpr int kVec = 4;  // elements per 16-byte vector
  __device__ __forceinline__ static void unpack(const uint4 &v, float *o) {
    o[0] = __uint_as_float(v.x);
    o[1] = __uint_as_float(v.y);
    o[2] = __uint_as_float(v.z);
    o[3] = __uint_as_float(v.w);
  }
  __device__ __forceinline__ static uint4 pack(const float *i) {
    return make_uint4(__float_as_uint(i[0]), __float_as_uint(i[1]), __float_as_uint(i[2]),
                      __float_as_uint(i[3]));
  }
  __device__ __forceinline__ static float load1(const float *p) { return *p; }
  __device__ __forceinline__ static void store1(float *p, float v) { *p = v; }
};

template <>
struct io<__nv_bfloat16> {
  static constexpr int kVec = 8;
  __device__ __forceinline__ static void unpack(const uint4 &v, float *o) {
    o[0] = bf16_lo(v.x);
    o[1] = bf16_hi(v.x);
    o[2] = bf16_lo(v.y);
    o[3] = bf16_hi(v.y);
    o[4] = bf16_lo(v.z);
    o[5] = bf16_hi(v.z);
    o[6] = bf16_lo(v.w);
    o[7] = bf16_hi(v.w);
  }
  __device__ __forceinline__ static uint4 pack(const float *i) {
    return make_uint4(pack_bf16x2(i[0], i[1]), pack_bf16x2(i[2], i[3]), pack_bf16x2(i[4], i[5]),
                      pack_bf16x2(i[6], i[7]));
  }
  __device__ __forceinline__ static float load1(const __nv_bfloat16 *p) { return __bfloat162float(*p); }
  __device__ __forceinline__ static void store1(__nv_bfloat16 *p, float v) { *p = __float2bfloat16_rn(v); }
};

__device__ __forceinline__ uint4 ld_stream(const void *p) {
  uint4 v;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}

__device__ __forceinline__ void st_stream(void *p, const uint4 &v) {
  asm volatile("st.global.cs.v4.u32 [%0], {%1,%2,%3,%4};" ::"l"(p), "r"(v.x), "r"(v.y), "r"(v.z),
               "r"(v.w)
               : "memory");
}

// One pass of NB butterfly stages (h = 2^s .. 2^(s+NB-1)) over v[0..d) of
// fp32 values in shared memory: each thread takes aligned groups of 2^NB
// elements into registers (compile-time indices, no local memory).
template <int NB>
__device__ __forceinline__ void butterfly_pass_f32(float *v, int d, int s) {
  constexpr int GS = 1 << NB;
  for (int g = threadIdx.x; g < (d >> NB); g += blockDim.x) {
    const int lo = g & ((1 << s) - 1);
    const int base = ((g >> s) << (s + NB)) | lo;
    float x[GS];
#pragma unroll
    for (int i = 0; i < GS; ++i) x[i] = v[base + (i << s)];
#pragma unroll
    for (int b = 0; b < NB; ++b)
#pragma unroll
      for (int i = 0; i < GS; ++i)
        if (!(i & (1 << b))) {
          const float a = x[i], c = x[i + (1 << b)];
          x[i] = a + c;
          x[i + (1 << b)] = a - c;
        }
#pragma unroll
    for (int i = 0; i < GS; ++i) v[base + (i << s)] = x[i];
  }
}

// All logn stages, three per pass (the last pass one or two), with a block
// barrier after each pass.
__device__ __forceinline__ void butterflies_smem_f32(float *v, int d, int logn) {
  for (int s = 0; s < logn; s += 3) {
    const int nb = (logn - s) < 3 ? (logn - s) : 3;
    if (nb == 3) butterfly_pass_f32<3>(v, d, s);
    else if (nb == 2) butterfly_pass_f32<2>(v, d, s);
    else butterfly_pass_f32<1>(v, d, s);
    __syncthreads();
  }
}

}  // namespace qwha
