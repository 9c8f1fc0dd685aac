// AdaAlloc initialisation of the adapter ("QWHA", papernotes.org 关键设计 2 and
// 3; gist.science 2.2): a per-channel budget proportional to the channel's
// quantization error, then inside each channel the largest coefficients of
// the transformed error dW_Q H, valued by the dense solution.
//
// Every rounding that decides an integer is fixed so that budgets and E are
// reproducible bit for bit by an independent implementation:
//   * e_i = sqrt(sum_k dW[i,k]^2): squares in fp64 (exact for fp32 inputs),
//     summed by the pairwise tree in index order over the zero-padded
//     power-of-two length (any larger padding gives the same value: the extra
//     leaves are exact zeros). A thread sums an aligned run with a stack of
//     partial sums (a binary counter), threads combine level by level.
//   * budget_i = min + floor(fl(pool * e_i) / S) with IEEE fp64 multiply and
//     divide, capped at d_in with the pool re-shared among the rest.
//   * the rank key is |V| of the unnormalised transform, fp64 butterflies in
//     the textbook stage order h = 1, 2, 4, ... (pure adds: no contraction).
//   * top-b by a most-significant-digit radix select on the fp64 bit patterns,
//     equal keys taken in increasing index.
//   * c = float(V * (1/sqrt(n))), one fp64 multiply then one rounding.
//
// Kernels: row_norm (one CTA per row), budget (one CTA), select (one CTA per
// row: butterflies in shared memory, radix select, ordered compaction).

#include <algorithm>

#include "common.cuh"
#include "kernels.h"

namespace qwha {
namespace {

constexpr int kNormThreads = 256;
constexpr int kBudgetThreads = 1024;
constexpr int kSelThreads = 256;
constexpr int kMaxInitDin = 16384;

__device__ __forceinline__ int next_pow2(int v) {
  int m = 1;
  while (m < v) m <<= 1;
  return m;
}

// Pairwise sum of v[0..L) (L a power of two) in the canonical tree, by a
// stack of partial sums keyed by level.
template <typename F>
__device__ double run_pairwise(int L, F value) {
  double st[17];
  int lv[17];
  int top = 0;
  for (int i = 0; i < L; ++i) {
    double s = value(i);
    int l = 0;
    while (top > 0 && lv[top - 1] == l) {
      s = __dadd_rn(st[top - 1], s);
      --top;
      ++l;
    }
    st[top] = s;
    lv[top] = l;
    ++top;
  }
  return st[0];
}

// Canonical tree over the per-thread sums held in sh[0..blockDim) (a power of two).
__device__ double block_pairwise(double mine, double *sh) {
  const int t = threadIdx.x;
  sh[t] = mine;
  __syncthreads();
  for (int w = blockDim.x; w > 1; w >>= 1) {
    double v = 0;
    if (t < w / 2) v = __dadd_rn(sh[2 * t], sh[2 * t + 1]);
    __syncthreads();
    if (t < w / 2) sh[t] = v;
    __syncthreads();
  }
  const double r = sh[0];
  __syncthreads();
  return r;
}

template <typename T>
__device__ T block_sum(T v, T *sh) {
  const int t = threadIdx.x;
  sh[t] = v;
  __syncthreads();
  for (int w = blockDim.x / 2; w > 0; w >>= 1) {
    if (t < w) sh[t] += sh[t + w];
    __syncthreads();
  }
  const T r = sh[0];
  __syncthreads();
  return r;
}

// Exclusive prefix over threads of v (blockDim a power of two); returns the total in *tot.
__device__ int64_t block_excl_scan(int64_t v, int64_t *sh, int64_t *tot) {
  const int t = threadIdx.x;
  sh[t] = v;
  __syncthreads();
  for (int off = 1; off < (int)blockDim.x; off <<= 1) {
    const int64_t a = t >= off ? sh[t - off] : 0;
    __syncthreads();
    sh[t] += a;
    __syncthreads();
  }
  const int64_t incl = sh[t];
  *tot = sh[blockDim.x - 1];
  __syncthreads();
  return incl - v;
}

// Pairwise sum of the squares of w[base .. base + L) (zero past d_in), the
// canonical tree of an aligned run of L (a power of two), in registers.
template <int L>
__device__ __forceinline__ double tree_sq(const float *__restrict__ w, int base, int d_in) {
  double x[L];
#pragma unroll
  for (int i = 0; i < L; ++i) {
    const int k = base + i;
    const double v = k < d_in ? (double)w[k] : 0.0;
    x[i] = __dmul_rn(v, v);
  }
#pragma unroll
  for (int h = 1; h < L; h <<= 1)
#pragma unroll
    for (int i = 0; i < L; i += 2 * h) x[i] = __dadd_rn(x[i], x[i + h]);
  return x[0];
}

// e[row] = sqrt of the canonical pairwise sum of squares over the zero-padded
// power-of-two length m: thread t sums the aligned run [t*L, t*L + L) with
// L = m / blockDim (runs of 16 in registers, longer runs as a tree of those),
// then the threads' sums meet in the block-level tree.
__global__ void __launch_bounds__(kNormThreads) row_norm_kernel(const float *__restrict__ dW, int d_in,
                                                                double *__restrict__ e) {
  __shared__ double sh[kNormThreads];
  const int64_t row = blockIdx.x;
  const float *w = dW + row * d_in;
  int m = next_pow2(d_in);
  const int L = m > kNormThreads ? m / kNormThreads : 1;
  const int base = threadIdx.x * L;
  double mine;
  switch (L) {
    case 1: mine = tree_sq<1>(w, base, d_in); break;
    case 2: mine = tree_sq<2>(w, base, d_in); break;
    case 4: mine = tree_sq<4>(w, base, d_in); break;
    case 8: mine = tree_sq<8>(w, base, d_in); break;
    case 16: mine = tree_sq<16>(w, base, d_in); break;
    default: mine = run_pairwise(L / 16, [&](int c) { return tree_sq<16>(w, base + 16 * c, d_in); }); break;
  }
  const double s = block_pairwise(mine, sh);
  if (threadIdx.x == 0) e[row] = __dsqrt_rn(s);
}

// Radix select over `n` keys produced by key(i) (eligible when ok(i)): the
// `want`-th smallest key K and how many keys equal to K are to be taken.
// Eight passes of 8 bits, most significant first. The histogram adds one
// count per distinct digit per warp (the leading bytes of fp64 patterns are
// shared by nearly all keys, so per-key atomics would serialise), and warp 0
// finds the digit holding the `need`-th key with a shuffle scan over the 256
// bins (8 per lane).
constexpr int kCandCap = 1024;  // candidate list of the radix select (indices)

template <typename KeyF, typename OkF>
__device__ void radix_select_smallest(int n, int64_t want, KeyF key, OkF ok, uint32_t *hist, uint64_t *K_out,
                                      int64_t *need_out) {
  __shared__ int sel_digit;
  __shared__ int64_t sel_need;
  // Once the keys that still match the prefix are at most kCandCap, the next
  // pass also lists their indices, and the passes after it scan that list
  // instead of all n keys (the digits found are the same).
  __shared__ int cand[kCandCap];
  __shared__ int cand_n;
  __shared__ uint32_t match_count;  // keys matching the prefix after the last pass
  uint64_t prefix = 0;
  int64_t need = want;
  const int lane = threadIdx.x & 31;
  bool listing = false, listed = false;
  if (threadIdx.x == 0) {
    cand_n = 0;
    match_count = 0xffffffffu;
  }
  __syncthreads();
  for (int shift = 56; shift >= 0; shift -= 8) {
    for (int i = threadIdx.x; i < 256; i += blockDim.x) hist[i] = 0;
    listing = !listed && match_count <= (uint32_t)kCandCap;
    __syncthreads();
    const uint64_t hi_mask = shift == 56 ? 0 : (~0ull << (shift + 8));
    const int m = listed ? cand_n : n;
    const int m_round = (m + blockDim.x - 1) / blockDim.x * blockDim.x;  // whole warps iterate together
    for (int it = threadIdx.x; it < m_round; it += blockDim.x) {
      int bin = 256;  // no count
      if (it < m) {
        const int i = listed ? cand[it] : it;
        if (listed || ok(i)) {
          const uint64_t k = key(i);
          if ((k & hi_mask) == (prefix & hi_mask)) {
            bin = (int)((k >> shift) & 255);
            if (listing) cand[atomicAdd(&cand_n, 1)] = i;
          }
        }
      }
      const unsigned peers = __match_any_sync(0xffffffffu, bin);
      if (bin < 256 && lane == __ffs(peers) - 1) atomicAdd(&hist[bin], (uint32_t)__popc(peers));
    }
    __syncthreads();
    if (listing) listed = true;
    if (threadIdx.x < 32) {
      uint32_t c[8];
      uint32_t mine = 0;
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        c[j] = hist[8 * lane + j];
        mine += c[j];
      }
      uint32_t incl = mine;  // inclusive scan over lanes
#pragma unroll
      for (int off = 1; off < 32; off <<= 1) {
        const uint32_t o = __shfl_up_sync(0xffffffffu, incl, off);
        if (lane >= off) incl += o;
      }
      const int64_t excl = (int64_t)(incl - mine);
      const bool hit = (excl < need && (int64_t)incl >= need) || (lane == 0 && need <= 0);
      const unsigned who = __ballot_sync(0xffffffffu, hit);
      if (hit) {
        int64_t cum = excl;
        int d = 8 * lane + 7;
        uint32_t cnt = c[7];
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          if (cum + c[j] >= need) {
            d = 8 * lane + j;
            cnt = c[j];
            break;
          }
          cum += c[j];
        }
        sel_digit = d;
        sel_need = need - cum;
        match_count = cnt;
      } else if (who == 0 && lane == 31) {  // fewer eligible keys than wanted: past the last digit
        sel_digit = 255;
        sel_need = need - (int64_t)incl;
        match_count = c[7];
      }
    }
    __syncthreads();
    prefix |= (uint64_t)sel_digit << shift;
    need = sel_need;
    __syncthreads();
  }
  *K_out = prefix;
  *need_out = need;
}

// Mark, in increasing index order, every eligible key < K and the first `need`
// keys == K; calls take(i) for each, in an order-preserving compaction whose
// output slot is passed too.
template <typename KeyF, typename OkF, typename TakeF>
__device__ void ordered_take(int n, uint64_t K, int64_t need, KeyF key, OkF ok, TakeF take, int64_t *sh64) {
  const int per = (n + blockDim.x - 1) / blockDim.x;
  const int a = threadIdx.x * per, b = min(n, a + per);
  int64_t eq = 0;
  for (int i = a; i < b; ++i)
    if (ok(i) && key(i) == K) ++eq;
  int64_t tot;
  const int64_t eq_before = block_excl_scan(eq, sh64, &tot);
  int64_t cnt = 0;
  {
    int64_t e_seen = eq_before;
    for (int i = a; i < b; ++i) {
      if (!ok(i)) continue;
      const uint64_t k = key(i);
      if (k < K || (k == K && e_seen++ < need)) ++cnt;
    }
  }
  const int64_t slot0 = block_excl_scan(cnt, sh64, &tot);
  int64_t slot = slot0, e_seen = eq_before;
  for (int i = a; i < b; ++i) {
    if (!ok(i)) continue;
    const uint64_t k = key(i);
    if (k < K || (k == K && e_seen++ < need)) take(i, slot++);
  }
}

__global__ void __launch_bounds__(kBudgetThreads)
    budget_kernel(const double *__restrict__ e, int d_out, int d_in, int64_t p, int min_per_row, int mode,
                  int32_t *__restrict__ budgets, int32_t *__restrict__ row_ptr, unsigned char *__restrict__ capped) {
  __shared__ double shd[kBudgetThreads];
  __shared__ int64_t sh64[kBudgetThreads];
  __shared__ uint32_t hist[256];
  __shared__ int any_new;
  const int t = threadIdx.x;
  for (int i = t; i < d_out; i += blockDim.x) capped[i] = 0;
  __syncthreads();
  double pool = (double)(p - (int64_t)min_per_row * d_out);
  const int m = next_pow2(d_out);
  const int L = m > kBudgetThreads ? m / kBudgetThreads : 1;
  for (;;) {
    const double mine = run_pairwise(L, [&](int i) {
      const int r = t * L + i;
      return (r < d_out && !capped[r]) ? e[r] : 0.0;
    });
    const double S = block_pairwise(mine, shd);
    int64_t na = 0;
    for (int i = t; i < d_out; i += blockDim.x) na += !capped[i];
    const int64_t n_active = block_sum<int64_t>(na, sh64);
    if (n_active == 0) break;
    if (t == 0) any_new = 0;
    __syncthreads();
    for (int i = t; i < d_out; i += blockDim.x) {
      if (capped[i]) continue;
      const double share = S > 0.0 ? floor(__ddiv_rn(__dmul_rn(pool, e[i]), S)) : floor(__ddiv_rn(pool, (double)n_active));
      const int64_t b = (int64_t)min_per_row + (int64_t)share;
      budgets[i] = (int32_t)(b > d_in ? d_in + 1 : b);  // d_in + 1 marks "over"
      if (b > d_in) any_new = 1;
    }
    __syncthreads();
    if (!any_new) break;
    int64_t nc = 0;
    for (int i = t; i < d_out; i += blockDim.x)
      if (!capped[i] && budgets[i] > d_in) {
        budgets[i] = d_in;
        capped[i] = 1;
        ++nc;
      }
    const int64_t newly = block_sum<int64_t>(nc, sh64);
    pool -= (double)newly * (double)(d_in - min_per_row);
    __syncthreads();
  }
  int64_t mysum = 0;
  for (int i = t; i < d_out; i += blockDim.x) mysum += budgets[i];
  int64_t R = p - block_sum<int64_t>(mysum, sh64);
  // remainder: one each, in the mode's order, to rows below d_in
  while (R > 0) {
    int64_t el = 0;
    for (int i = t; i < d_out; i += blockDim.x) el += budgets[i] < d_in;
    const int64_t n_el = block_sum<int64_t>(el, sh64);
    if (n_el == 0) break;  // cannot happen for p <= d_in * d_out
    if (R >= n_el) {
      for (int i = t; i < d_out; i += blockDim.x)
        if (budgets[i] < d_in) budgets[i] += 1;
      R -= n_el;
      __syncthreads();
      continue;
    }
    auto ok = [&](int i) { return budgets[i] < d_in; };
    auto key = [&](int i) -> uint64_t {
      return mode == 0 ? (uint64_t)budgets[i] : ~(uint64_t)__double_as_longlong(e[i]);
    };
    uint64_t K;
    int64_t need;
    radix_select_smallest(d_out, R, key, ok, hist, &K, &need);
    __syncthreads();
    // mark first, then add: the keys must not change while being read
    ordered_take(d_out, K, need, key, ok, [&](int i, int64_t) { capped[i] = 2; }, sh64);
    __syncthreads();
    for (int i = t; i < d_out; i += blockDim.x)
      if (capped[i] == 2) {
        budgets[i] += 1;
        capped[i] = 1;
      }
    R = 0;
    __syncthreads();
  }
  __syncthreads();
  // row_ptr = exclusive scan of budgets, in chunks of blockDim
  int64_t carry = 0;
  if (t == 0) row_ptr[0] = 0;
  for (int base = 0; base < d_out; base += blockDim.x) {
    const int i = base + t;
    const int64_t v = i < d_out ? budgets[i] : 0;
    int64_t tot;
    const int64_t ex = block_excl_scan(v, sh64, &tot);
    if (i < d_out) row_ptr[i + 1] = (int32_t)(carry + ex + v);
    carry += tot;
  }
}

// One pass of NB butterfly stages (h = 2^s .. 2^(s+NB-1)) over v[0..d) in
// shared memory: each thread takes aligned groups of 2^NB elements into
// registers (compile-time indices), textbook order inside the group.
template <int NB>
__device__ __forceinline__ void butterfly_pass_fp64(double *v, int d, int s) {
  constexpr int GS = 1 << NB;
  for (int g = threadIdx.x; g < (d >> NB); g += blockDim.x) {
    const int lo = g & ((1 << s) - 1);
    const int base = ((g >> s) << (s + NB)) | lo;
    double x[GS];
#pragma unroll
    for (int i = 0; i < GS; ++i) x[i] = v[base + (i << s)];
#pragma unroll
    for (int b = 0; b < NB; ++b)
#pragma unroll
      for (int i = 0; i < GS; ++i)
        if (!(i & (1 << b))) {
          const double a = x[i], c = x[i + (1 << b)];
          x[i] = __dadd_rn(a, c);
          x[i + (1 << b)] = __dsub_rn(a, c);
        }
#pragma unroll
    for (int i = 0; i < GS; ++i) v[base + (i << s)] = x[i];
  }
}

// v[0..d_in) = w[0..d_in) H_unnormalised per block of n, fp64 butterflies in
// the textbook stage order (three stages per pass over aligned groups of 8,
// the last pass one or two when log2 n is not a multiple of 3); v is shared
// memory, every thread of the block takes part.
__device__ void row_transform_fp64(const float *__restrict__ w, int d_in, int n, double *v) {
  for (int k = threadIdx.x; k < d_in; k += blockDim.x) v[k] = (double)w[k];
  __syncthreads();
  const int logn = 31 - __clz(n);
  for (int s = 0; s < logn; s += 3) {
    const int nb = min(3, logn - s);
    if (nb == 3) butterfly_pass_fp64<3>(v, d_in, s);
    else if (nb == 2) butterfly_pass_fp64<2>(v, d_in, s);
    else butterfly_pass_fp64<1>(v, d_in, s);
    __syncthreads();
  }
}

__global__ void __launch_bounds__(kSelThreads)
    select_kernel(const float *__restrict__ dW, int d_in, int n, const int32_t *__restrict__ budgets,
                  const int32_t *__restrict__ row_ptr, int64_t p, int32_t *__restrict__ col_idx,
                  float *__restrict__ coef) {
  extern __shared__ __align__(16) double v[];  // d_in values of the row
  __shared__ uint32_t hist[256];
  __shared__ int64_t sh64[kSelThreads];
  const int64_t row = blockIdx.x;
  row_transform_fp64(dW + row * d_in, d_in, n, v);
  const int b = budgets[row];
  int64_t start = (int64_t)row_ptr[row] - row_ptr[0];  // row_ptr may be a slice of a longer one
  if (b <= 0 || start < 0 || start + b > p) return;
  const double inv = __ddiv_rn(1.0, __dsqrt_rn((double)n));
  // largest |V| = smallest complemented magnitude bits
  auto key = [&](int k) -> uint64_t { return ~((uint64_t)__double_as_longlong(v[k]) & 0x7fffffffffffffffull); };
  auto ok = [&](int) { return true; };
  uint64_t K;
  int64_t need;
  radix_select_smallest(d_in, b, key, ok, hist, &K, &need);
  __syncthreads();
  ordered_take(d_in, K, need, key, ok,
               [&](int k, int64_t slot) {
                 if (slot < b) {
                   col_idx[start + slot] = k;
                   coef[start + slot] = __double2float_rn(__dmul_rn(v[k], inv));
                 }
               },
               sh64);
}

// ------------------------------------------------------------ selection over the whole matrix
//
// E = the p smallest keys over all d_out x d_in entries, equal keys taken in
// increasing flat index j = i * d_in + k: magnitude selection (key = the
// complemented magnitude bits of V, so the largest |V| come first) or random
// selection (key = SplitMix64 output j + 1 for the seed: Steele, Lea and
// Flood, 2014). V (fp64, unnormalised transform) is kept in the workspace: the
// magnitude keys read it in every pass and c = float(V / sqrt(n)) at E.

constexpr int kGselThreads = 256;

struct GselState {
  unsigned long long prefix;  // digits of K fixed so far
  long long need;             // how many keys equal to the prefix are still to be taken
  uint32_t hist[256];
};

__device__ __forceinline__ uint64_t splitmix64_at(uint64_t seed, uint64_t n) {
  uint64_t z = seed + n * 0x9E3779B97F4A7C15ull;
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
  return z ^ (z >> 31);
}

__device__ __forceinline__ uint64_t gsel_key(const double *__restrict__ V, int64_t j, int sel, uint64_t seed) {
  if (sel == 0) return ~((uint64_t)__double_as_longlong(V[j]) & 0x7fffffffffffffffull);
  return splitmix64_at(seed, (uint64_t)j + 1);
}

__global__ void __launch_bounds__(kSelThreads)
    gsel_transform_kernel(const float *__restrict__ dW, int d_in, int n, double *__restrict__ V) {
  extern __shared__ __align__(16) double v[];
  const int64_t row = blockIdx.x;
  row_transform_fp64(dW + row * d_in, d_in, n, v);
  for (int k = threadIdx.x; k < d_in; k += blockDim.x) V[row * d_in + k] = v[k];
}

__global__ void gsel_init_kernel(GselState *st, int64_t p) {
  if (threadIdx.x == 0) {
    st->prefix = 0;
    st->need = p;
  }
  for (int i = threadIdx.x; i < 256; i += blockDim.x) st->hist[i] = 0;
}

// Histogram of digit `shift` over the keys that match the prefix so far.
__global__ void __launch_bounds__(kGselThreads)
    gsel_hist_kernel(const double *__restrict__ V, int64_t N, int sel, uint64_t seed, int shift, GselState *st) {
  __shared__ uint32_t hist[256];
  for (int i = threadIdx.x; i < 256; i += blockDim.x) hist[i] = 0;
  __syncthreads();
  const uint64_t prefix = st->prefix;
  const uint64_t hi_mask = shift == 56 ? 0 : (~0ull << (shift + 8));
  const int lane = threadIdx.x & 31;
  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  const int64_t n_round = (N + stride - 1) / stride * stride;  // whole warps iterate together
  for (int64_t j = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; j < n_round; j += stride) {
    int bin = 256;
    if (j < N) {
      const uint64_t k = gsel_key(V, j, sel, seed);
      if ((k & hi_mask) == (prefix & hi_mask)) bin = (int)((k >> shift) & 255);
    }
    const unsigned peers = __match_any_sync(0xffffffffu, bin);
    if (bin < 256 && lane == __ffs(peers) - 1) atomicAdd(&hist[bin], (uint32_t)__popc(peers));
  }
  __syncthreads();
  for (int i = threadIdx.x; i < 256; i += blockDim.x)
    if (hist[i]) atomicAdd(&st->hist[i], hist[i]);
}

// One warp: the digit that holds the need-th key, then clear the histogram.
__global__ void gsel_pick_kernel(GselState *st, int shift) {
  const int lane = threadIdx.x;
  const long long need = st->need;
  uint32_t c[8];
  uint32_t mine = 0;
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    c[j] = st->hist[8 * lane + j];
    mine += c[j];
  }
  uint32_t incl = mine;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const uint32_t o = __shfl_up_sync(0xffffffffu, incl, off);
    if (lane >= off) incl += o;
  }
  const long long excl = (long long)(incl - mine);
  const bool hit = (excl < need && (long long)incl >= need) || (lane == 0 && need <= 0);
  const unsigned who = __ballot_sync(0xffffffffu, hit);
  if (hit) {
    long long cum = excl;
    int d = 8 * lane + 7;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      if (cum + c[j] >= need) {
        d = 8 * lane + j;
        break;
      }
      cum += c[j];
    }
    st->prefix |= (unsigned long long)d << shift;
    st->need = need - cum;
  } else if (who == 0 && lane == 31) {
    st->prefix |= 255ull << shift;
    st->need = need - (long long)incl;
  }
  __syncwarp();
#pragma unroll
  for (int j = 0; j < 8; ++j) st->hist[8 * lane + j] = 0;
}

// Per row: keys below K and keys equal to K.
__global__ void __launch_bounds__(kGselThreads)
    gsel_count_kernel(const double *__restrict__ V, int d_in, int sel, uint64_t seed, const GselState *st,
                      int32_t *__restrict__ lt, int32_t *__restrict__ eq) {
  __shared__ int32_t sh[kGselThreads];
  const uint64_t K = st->prefix;
  const int64_t row = blockIdx.x;
  int a = 0, b = 0;
  for (int k = threadIdx.x; k < d_in; k += blockDim.x) {
    const uint64_t key = gsel_key(V, row * d_in + k, sel, seed);
    a += key < K;
    b += key == K;
  }
  const int la = block_sum(a, sh), lb = block_sum(b, sh);
  if (threadIdx.x == 0) {
    lt[row] = la;
    eq[row] = lb;
  }
}

// One CTA: rows take all their keys below K and, in row order, the first
// `need` keys equal to K; budgets and row_ptr follow.
__global__ void __launch_bounds__(kBudgetThreads)
    gsel_budget_kernel(const int32_t *__restrict__ lt, const int32_t *__restrict__ eq, int d_out, const GselState *st,
                       int32_t *__restrict__ take_eq, int32_t *__restrict__ budgets, int32_t *__restrict__ row_ptr) {
  __shared__ int64_t sh64[kBudgetThreads];
  const int t = threadIdx.x;
  const int64_t need = st->need;
  int64_t eq_carry = 0, b_carry = 0;
  if (t == 0) row_ptr[0] = 0;
  for (int base = 0; base < d_out; base += blockDim.x) {
    const int i = base + t;
    const int64_t e = i < d_out ? eq[i] : 0;
    int64_t tot;
    const int64_t before = eq_carry + block_excl_scan(e, sh64, &tot);
    eq_carry += tot;
    int64_t take = need - before;
    take = take < 0 ? 0 : (take > e ? e : take);
    const int64_t bud = i < d_out ? lt[i] + take : 0;
    const int64_t ex = block_excl_scan(bud, sh64, &tot);
    if (i < d_out) {
      take_eq[i] = (int32_t)take;
      budgets[i] = (int32_t)bud;
      row_ptr[i + 1] = (int32_t)(b_carry + ex + bud);
    }
    b_carry += tot;
  }
}

// Per row: the selected columns in increasing order, with c = float(V / sqrt(n)).
__global__ void __launch_bounds__(kSelThreads)
    gsel_take_kernel(const double *__restrict__ V, int d_in, int n, int sel, uint64_t seed, const GselState *st,
                     const int32_t *__restrict__ take_eq, const int32_t *__restrict__ row_ptr, int64_t p,
                     int32_t *__restrict__ col_idx, float *__restrict__ coef) {
  extern __shared__ __align__(16) double v[];
  __shared__ int64_t sh64[kSelThreads];
  const int64_t row = blockIdx.x;
  for (int k = threadIdx.x; k < d_in; k += blockDim.x) v[k] = V[row * d_in + k];
  __syncthreads();
  const int64_t start = row_ptr[row];
  const int64_t cnt = (int64_t)row_ptr[row + 1] - start;
  if (cnt <= 0 || start < 0 || start + cnt > p) return;
  const uint64_t K = st->prefix;
  const double inv = __ddiv_rn(1.0, __dsqrt_rn((double)n));
  auto key = [&](int k) -> uint64_t {
    if (sel == 0) return ~((uint64_t)__double_as_longlong(v[k]) & 0x7fffffffffffffffull);
    return splitmix64_at(seed, (uint64_t)(row * d_in + k) + 1);
  };
  auto ok = [&](int) { return true; };
  ordered_take(d_in, K, take_eq[row], key, ok,
               [&](int k, int64_t slot) {
                 if (slot < cnt) {
                   col_idx[start + slot] = k;
                   coef[start + slot] = __double2float_rn(__dmul_rn(v[k], inv));
                 }
               },
               sh64);
}

}  // namespace

size_t init_workspace(int32_t d_out, int32_t d_in) {
  (void)d_in;
  return align_up((size_t)d_out * 8, 256) + align_up((size_t)d_out, 256);
}

int init_max_din() { return kMaxInitDin; }

cudaError_t launch_init_alloc(const float *dW, int32_t d_out, int32_t d_in, int32_t had_block, int64_t p,
                              int32_t min_per_row, int mode, int32_t *budgets, int32_t *row_ptr, int32_t *col_idx,
                              float *coef, void *ws, cudaStream_t s) {
  double *e = static_cast<double *>(ws);
  unsigned char *capped = static_cast<unsigned char *>(ws) + align_up((size_t)d_out * 8, 256);
  row_norm_kernel<<<d_out, kNormThreads, 0, s>>>(dW, d_in, e);
  budget_kernel<<<1, kBudgetThreads, 0, s>>>(e, d_out, d_in, p, min_per_row, mode, budgets, row_ptr, capped);
  const size_t smem = (size_t)d_in * sizeof(double);
  cudaError_t err = cudaFuncSetAttribute(select_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (err != cudaSuccess) return err;
  if (p > 0) select_kernel<<<d_out, kSelThreads, smem, s>>>(dW, d_in, had_block, budgets, row_ptr, p, col_idx, coef);
  return cudaGetLastError();
}

size_t select_global_workspace(int32_t d_out, int32_t d_in) {
  return align_up((size_t)d_out * d_in * 8, 256) + align_up(sizeof(GselState), 256) + 3 * align_up((size_t)d_out * 4, 256);
}

cudaError_t launch_select_global(const float *dW, int32_t d_out, int32_t d_in, int32_t had_block, int64_t p, int sel,
                                 uint64_t seed, int32_t *budgets, int32_t *row_ptr, int32_t *col_idx, float *coef,
                                 void *ws, cudaStream_t s) {
  char *w = static_cast<char *>(ws);
  double *V = reinterpret_cast<double *>(w);
  w += align_up((size_t)d_out * d_in * 8, 256);
  GselState *st = reinterpret_cast<GselState *>(w);
  w += align_up(sizeof(GselState), 256);
  int32_t *lt = reinterpret_cast<int32_t *>(w);
  w += align_up((size_t)d_out * 4, 256);
  int32_t *eq = reinterpret_cast<int32_t *>(w);
  w += align_up((size_t)d_out * 4, 256);
  int32_t *take = reinterpret_cast<int32_t *>(w);
  const size_t smem = (size_t)d_in * sizeof(double);
  cudaError_t e = cudaFuncSetAttribute(gsel_transform_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(gsel_take_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  const int64_t N = (int64_t)d_out * d_in;
  gsel_transform_kernel<<<d_out, kSelThreads, smem, s>>>(dW, d_in, had_block, V);
  gsel_init_kernel<<<1, 256, 0, s>>>(st, p);
  const int64_t grid = std::min<int64_t>(cdiv(N, (int64_t)kGselThreads), (int64_t)sm_count() * 8);
  for (int shift = 56; shift >= 0; shift -= 8) {
    gsel_hist_kernel<<<(unsigned)grid, kGselThreads, 0, s>>>(V, N, sel, seed, shift, st);
    gsel_pick_kernel<<<1, 32, 0, s>>>(st, shift);
  }
  gsel_count_kernel<<<d_out, kGselThreads, 0, s>>>(V, d_in, sel, seed, st, lt, eq);
  gsel_budget_kernel<<<1, kBudgetThreads, 0, s>>>(lt, eq, d_out, st, take, budgets, row_ptr);
  if (p > 0)
    gsel_take_kernel<<<d_out, kSelThreads, smem, s>>>(V, d_in, had_block, sel, seed, st, take, row_ptr, p, col_idx,
                                                      coef);
  return cudaGetLastError();
}

cudaError_t launch_init_norms(const float *dW, int32_t rows, int32_t d_in, double *e, cudaStream_t s) {
  if (rows <= 0) return cudaSuccess;
  row_norm_kernel<<<rows, kNormThreads, 0, s>>>(dW, d_in, e);
  return cudaGetLastError();
}

cudaError_t launch_init_budgets(const double *e, int32_t d_out, int32_t d_in, int64_t p, int32_t min_per_row, int mode,
                                int32_t *budgets, int32_t *row_ptr, void *ws, cudaStream_t s) {
  unsigned char *capped = static_cast<unsigned char *>(ws) + align_up((size_t)d_out * 8, 256);
  budget_kernel<<<1, kBudgetThreads, 0, s>>>(e, d_out, d_in, p, min_per_row, mode, budgets, row_ptr, capped);
  return cudaGetLastError();
}

cudaError_t launch_init_select(const float *dW, int32_t rows, int32_t d_in, int32_t had_block, const int32_t *budgets,
                               const int32_t *row_ptr, int64_t p, int32_t *col_idx, float *coef, cudaStream_t s) {
  if (rows <= 0 || p <= 0) return cudaSuccess;
  const size_t smem = (size_t)d_in * sizeof(double);
  cudaError_t err = cudaFuncSetAttribute(select_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (err != cudaSuccess) return err;
  select_kernel<<<rows, kSelThreads, smem, s>>>(dW, d_in, had_block, budgets, row_ptr, p, col_idx, coef);
  return cudaGetLastError();
}

}  // namespace qwha
