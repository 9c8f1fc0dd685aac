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

// Position of entry k of a row's fp64 values in shared memory: one padding
// double after every 16, so the butterfly passes (aligned groups of 8 at any
// stride) and the coalesced sweeps meet distinct banks.
__host__ __device__ __forceinline__ int vpos(int k) { return k + (k >> 4); }
__host__ __device__ __forceinline__ size_t vbytes(int d_in) { return (size_t)vpos(d_in) * sizeof(double); }

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

// Canonical tree over the per-thread values `mine` (blockDim a power of two,
// at most 1024): levels inside a warp by shuffles (the left operand is always
// the lower-index subtree), then the warps' sums through sh[0..32) by warp 0.
__device__ double block_pairwise(double mine, double *sh) {
  const int t = threadIdx.x, lane = t & 31;
  const int width = blockDim.x < 32 ? (int)blockDim.x : 32;
  for (int h = 1; h < width; h <<= 1) {
    const double o = __shfl_down_sync(0xffffffffu, mine, h);
    if ((lane & (2 * h - 1)) == 0) mine = __dadd_rn(mine, o);
  }
  const int nw = (int)blockDim.x / 32;
  if (nw > 1) {
    if (lane == 0) sh[t >> 5] = mine;
    __syncthreads();
    if (t < 32) {
      double x = t < nw ? sh[t] : 0.0;
      for (int h = 1; h < nw; h <<= 1) {
        const double o = __shfl_down_sync(0xffffffffu, x, h);
        if ((lane & (2 * h - 1)) == 0) x = __dadd_rn(x, o);
      }
      if (t == 0) sh[32] = x;
    }
  } else if (t == 0) {
    sh[32] = mine;
  }
  __syncthreads();
  const double r = sh[32];
  __syncthreads();
  return r;
}

// Sum over the block (integers: any order); sh holds 33 entries.
template <typename T>
__device__ T block_sum(T v, T *sh) {
  const int t = threadIdx.x, lane = t & 31;
#pragma unroll
  for (int off = 16; off; off >>= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
  if (lane == 0) sh[t >> 5] = v;
  __syncthreads();
  if (t < 32) {
    T x = t < (int)(blockDim.x >> 5) ? sh[t] : T(0);
#pragma unroll
    for (int off = 16; off; off >>= 1) x += __shfl_xor_sync(0xffffffffu, x, off);
    if (t == 0) sh[32] = x;
  }
  __syncthreads();
  const T r = sh[32];
  __syncthreads();
  return r;
}

// Exclusive prefix over threads of v (blockDim a multiple of 32); returns the
// total in *tot. Warp scans by shuffles, the warps' totals scanned by warp 0.
__device__ int64_t block_excl_scan(int64_t v, int64_t *sh, int64_t *tot) {
  const int t = threadIdx.x, lane = t & 31, nw = (int)blockDim.x >> 5;
  int64_t incl = v;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const int64_t o = __shfl_up_sync(0xffffffffu, incl, off);
    if (lane >= off) incl += o;
  }
  if (lane == 31) sh[t >> 5] = incl;
  __syncthreads();
  if (t < 32) {
    const int64_t w = t < nw ? sh[t] : 0;
    int64_t x = w;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const int64_t o = __shfl_up_sync(0xffffffffu, x, off);
      if (lane >= off) x += o;
    }
    sh[32 + t] = x - w;  // exclusive over warps
    if (t == 31) sh[64] = x;
  }
  __syncthreads();
  const int64_t r = sh[32 + (t >> 5)] + incl - v;
  *tot = sh[64];
  __syncthreads();
  return r;
}

// Pairwise sum of the squares of w[base .. base + L) (zero past d_in), the
// canonical tree of an aligned run of L (a power of two), in registers.
template <int L>
__device__ __forceinline__ double tree_sq(const float *__restrict__ w, int base, int d_in) {
  double x[L];
  if (L % 4 == 0 && base + L <= d_in && (reinterpret_cast<uintptr_t>(w + base) & 15u) == 0) {
#pragma unroll
    for (int i = 0; i < L; i += 4) {  // 16-byte loads where the run is inside the row and aligned
      const float4 f = *reinterpret_cast<const float4 *>(w + base + i);
      x[i] = __dmul_rn((double)f.x, (double)f.x);
      x[i + 1] = __dmul_rn((double)f.y, (double)f.y);
      x[i + 2] = __dmul_rn((double)f.z, (double)f.z);
      x[i + 3] = __dmul_rn((double)f.w, (double)f.w);
    }
  } else {
#pragma unroll
    for (int i = 0; i < L; ++i) {
      const int k = base + i;
      const double v = k < d_in ? (double)w[k] : 0.0;
      x[i] = __dmul_rn(v, v);
    }
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
// `want`-th smallest key K and how many keys equal to K are to be taken
// (want minus the number of keys below K).
//  * A first sweep finds the bits that all eligible keys share (AND and OR
//    of the keys): the digits start right below them, so no pass is spent on
//    the leading bytes that fp64 magnitudes of similar size have in common.
//  * Pass 1 takes a kHistBins-wide (10-bit) digit, later passes 8 bits. The
//    histogram adds one count per distinct digit per warp (__match_any_sync),
//    and warp 0 finds the digit holding the need-th key by a shuffle scan.
//  * Once the keys left are at most kCandCap, one sweep lists their indices
//    and later passes read only the list; once they are at most 32, warp 0
//    ranks them against each other and K follows directly.
// hist holds kHistBins entries.
constexpr int kCandCap = 1024;  // candidate list of the radix select (indices)
constexpr int kHistBins = 1024;

// Warp 0 of a block: among the candidates cand[0..cand_n) whose keys match
// `pm` under `hi_mask` (at most 32 of them), the need-th smallest key and how
// many keys equal to it are to be taken; one lane stores them to *K and
// *need_out and sets *done. The matching keys are staged in fk[0..32) (shared)
// and every lane ranks its own against all of them.
template <typename KeyF>
__device__ __forceinline__ void warp_rank_finish(KeyF key, const int *cand, int cand_n, uint64_t hi_mask, uint64_t pm,
                                                 int64_t need, unsigned long long *fk, unsigned long long *K,
                                                 long long *need_out, int *done) {
  const int lane = threadIdx.x & 31;
  const unsigned below = (1u << lane) - 1u;
  int have = 0;
  for (int c0 = 0; c0 < cand_n; c0 += 32) {
    const int c = c0 + lane;
    uint64_t k = 0;
    bool m = false;
    if (c < cand_n) {
      k = key(cand[c]);
      m = (k & hi_mask) == pm;
    }
    const unsigned mm = __ballot_sync(0xffffffffu, m);
    if (m && have + __popc(mm & below) < 32) fk[have + __popc(mm & below)] = k;
    have += __popc(mm);
  }
  __syncwarp();
  if (have > 32) have = 32;  // cannot happen: the caller checked the count
  const uint64_t mine = lane < have ? fk[lane] : ~0ull;
  int less = 0, eq = 0;
  for (int src = 0; src < have; ++src) {
    const uint64_t ks = fk[src];
    less += ks < mine;
    eq += ks == mine;
  }
  const bool hit = lane < have && less < need && need <= less + eq;
  const unsigned who = __ballot_sync(0xffffffffu, hit);
  if (who && lane == __ffs(who) - 1) {
    *K = mine;
    *need_out = need - less;
    *done = 1;
  }
}

template <bool AGG, typename KeyF, typename OkF>
__device__ void radix_select_smallest(int n, int64_t want, KeyF key, OkF ok, uint32_t *hist, uint64_t *K_out,
                                      int64_t *need_out) {
  __shared__ int sel_digit;
  __shared__ int64_t sel_need;
  __shared__ int cand[kCandCap];
  __shared__ int cand_n;
  __shared__ uint32_t match_count;  // keys matching the prefix after the last pass
  __shared__ unsigned long long s_and, s_or, s_K, fk[32];
  __shared__ long long sel_need_ll;
  __shared__ int s_cnt, s_done;
  const int lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    cand_n = 0;
    s_and = ~0ull;
    s_or = 0ull;
    s_cnt = 0;
    s_done = 0;
  }
  __syncthreads();
  {
    uint64_t ka = ~0ull, ko = 0ull;
    int c = 0;
    for (int i = threadIdx.x; i < n; i += blockDim.x)
      if (ok(i)) {
        const uint64_t k = key(i);
        ka &= k;
        ko |= k;
        ++c;
      }
    const uint32_t alo = __reduce_and_sync(0xffffffffu, (uint32_t)ka);
    const uint32_t ahi = __reduce_and_sync(0xffffffffu, (uint32_t)(ka >> 32));
    const uint32_t olo = __reduce_or_sync(0xffffffffu, (uint32_t)ko);
    const uint32_t ohi = __reduce_or_sync(0xffffffffu, (uint32_t)(ko >> 32));
    c = __reduce_add_sync(0xffffffffu, c);
    if (lane == 0) {
      atomicAnd(&s_and, ((unsigned long long)ahi << 32) | alo);
      atomicOr(&s_or, ((unsigned long long)ohi << 32) | olo);
      atomicAdd(&s_cnt, c);
    }
  }
  __syncthreads();
  const uint64_t kand = s_and, kor = s_or;
  const int cnt = s_cnt;
  if (want <= 0 || want > cnt || kand == kor) {
    // nothing to take; everything; or all eligible keys equal: K needs no pass
    *K_out = want <= 0 ? 0ull : (want > cnt ? ~0ull : kand);
    *need_out = want;
    return;
  }
  const int hb = 63 - __clzll((long long)(kand ^ kor));  // highest bit where eligible keys differ
  uint64_t prefix = hb == 63 ? 0ull : (kand & ~((2ull << hb) - 1ull));
  int64_t need = want;
  int bits = hb + 1 < 10 ? hb + 1 : 10;
  int shift = hb + 1 - bits;
  bool listed = false;
  if (threadIdx.x == 0) match_count = (uint32_t)cnt;
  __syncthreads();
  for (;;) {
    const uint64_t hi_mask = shift + bits >= 64 ? 0ull : ~((1ull << (shift + bits)) - 1ull);
    const int bins = 1 << bits;
    if (!listed && match_count <= (uint32_t)kCandCap) {
      // list the keys that match the prefix (no histogram in this sweep)
      const int n_round = (n + blockDim.x - 1) / blockDim.x * blockDim.x;
      for (int i = threadIdx.x; i < n_round; i += blockDim.x) {
        bool m = false;
        if (i < n && ok(i)) m = (key(i) & hi_mask) == (prefix & hi_mask);
        const unsigned mm = __ballot_sync(0xffffffffu, m);
        int base = 0;
        if (lane == 0 && mm) base = atomicAdd(&cand_n, __popc(mm));
        base = __shfl_sync(0xffffffffu, base, 0);
        if (m) cand[base + __popc(mm & ((1u << lane) - 1u))] = i;
      }
      listed = true;
      __syncthreads();
    }
    if (listed && match_count <= 32u) {
      // warp 0 ranks the (at most 32) keys that match the prefix
      if (threadIdx.x < 32)
        warp_rank_finish(key, cand, cand_n, hi_mask, prefix & hi_mask, need, fk, &s_K, &sel_need_ll, &s_done);
      __syncthreads();
      if (s_done) {
        *K_out = s_K;
        *need_out = sel_need_ll;
        return;
      }
    }
    for (int i = threadIdx.x; i < bins; i += blockDim.x) hist[i] = 0;
    __syncthreads();
    const int m = listed ? cand_n : n;
    const int m_round = (m + blockDim.x - 1) / blockDim.x * blockDim.x;  // whole warps iterate together
    for (int it = threadIdx.x; it < m_round; it += blockDim.x) {
      int bin = kHistBins;  // no count
      if (it < m) {
        const int i = listed ? cand[it] : it;
        if (listed || ok(i)) {
          const uint64_t k = key(i);
          if ((k & hi_mask) == (prefix & hi_mask)) bin = (int)((k >> shift) & (uint64_t)(bins - 1));
        }
      }
      if (AGG) {  // one count per distinct digit per warp: for keys with many duplicates
        const unsigned peers = __match_any_sync(0xffffffffu, bin);
        if (bin < kHistBins && lane == __ffs(peers) - 1) atomicAdd(&hist[bin], (uint32_t)__popc(peers));
      } else if (bin < kHistBins) {
        atomicAdd(&hist[bin], 1u);
      }
    }
    __syncthreads();
    if (threadIdx.x < 32) {
      const int per = (bins + 31) / 32;  // bins per lane
      uint32_t mine = 0;
      for (int j = 0; j < per; ++j) {
        const int bb = lane * per + j;
        mine += bb < bins ? hist[bb] : 0u;
      }
      uint32_t incl = mine;  // inclusive scan over lanes
#pragma unroll
      for (int off = 1; off < 32; off <<= 1) {
        const uint32_t o = __shfl_up_sync(0xffffffffu, incl, off);
        if (lane >= off) incl += o;
      }
      const int64_t excl = (int64_t)(incl - mine);
      const bool hit = excl < need && (int64_t)incl >= need;
      if (hit) {
        int64_t cum = excl;
        for (int j = 0; j < per; ++j) {
          const int bb = lane * per + j;
          const uint32_t c = bb < bins ? hist[bb] : 0u;
          if (cum + c >= need) {
            sel_digit = bb;
            sel_need = need - cum;
            match_count = c;
            break;
          }
          cum += c;
        }
      }
    }
    __syncthreads();
    prefix |= (uint64_t)sel_digit << shift;
    need = sel_need;
    __syncthreads();
    if (shift == 0) break;
    bits = shift < 8 ? shift : 8;
    shift -= bits;
  }
  *K_out = prefix;
  *need_out = need;
}

// Mark, in increasing index order, every eligible key < K and the first `need`
// keys == K; calls take(i, slot) for each, slot being its place in the
// order-preserving compaction. Each warp takes a contiguous range of indices in
// rounds of 32 consecutive ones (coalesced key reads): a first sweep counts the
// keys < K and == K per warp, a scan over the warps places the ranges, and in
// the second sweep ballots rank the marked keys inside a round. sh64 holds at
// least 2 * (blockDim / 32) entries.
template <typename KeyF, typename OkF, typename TakeF>
__device__ void ordered_take(int n, uint64_t K, int64_t need, KeyF key, OkF ok, TakeF take, int64_t *sh64) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
  const int per = (((n + nw - 1) / nw) + 31) & ~31;
  const int a = warp * per, b = min(n, a + per);
  int lt = 0, eq = 0;
  for (int i = a + lane; i < b; i += 32)
    if (ok(i)) {
      const uint64_t k = key(i);
      lt += k < K;
      eq += k == K;
    }
#pragma unroll
  for (int off = 16; off; off >>= 1) {
    lt += __shfl_xor_sync(0xffffffffu, lt, off);
    eq += __shfl_xor_sync(0xffffffffu, eq, off);
  }
  int64_t *s_eq = sh64, *s_take = sh64 + nw;
  if (lane == 0) s_eq[warp] = eq;
  __syncthreads();
  int64_t eq_before = 0;
  for (int w = 0; w < warp; ++w) eq_before += s_eq[w];
  int64_t eq_take = need - eq_before;
  eq_take = eq_take < 0 ? 0 : (eq_take > eq ? eq : eq_take);
  if (lane == 0) s_take[warp] = lt + eq_take;
  __syncthreads();
  int64_t slot = 0;
  for (int w = 0; w < warp; ++w) slot += s_take[w];
  int64_t e_seen = eq_before;
  const unsigned below = (1u << lane) - 1u;
  for (int i0 = a; i0 < b; i0 += 32) {  // warp-uniform rounds
    const int i = i0 + lane;
    bool is_lt = false, is_eq = false;
    if (i < b && ok(i)) {
      const uint64_t k = key(i);
      is_lt = k < K;
      is_eq = k == K;
    }
    const unsigned m_eq = __ballot_sync(0xffffffffu, is_eq);
    const bool t = is_lt || (is_eq && e_seen + __popc(m_eq & below) < need);
    const unsigned m_t = __ballot_sync(0xffffffffu, t);
    if (t) take(i, slot + __popc(m_t & below));
    slot += __popc(m_t);
    e_seen += __popc(m_eq);
  }
  __syncthreads();  // the caller reuses sh64
}

__global__ void __launch_bounds__(kBudgetThreads)
    budget_kernel(const double *__restrict__ e, int d_out, int d_in, int64_t p, int min_per_row, int mode,
                  int32_t *__restrict__ budgets, int32_t *__restrict__ row_ptr, unsigned char *__restrict__ capped) {
  __shared__ double shd[kBudgetThreads];
  __shared__ int64_t sh64[kBudgetThreads];
  __shared__ uint32_t hist[kHistBins];
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
    radix_select_smallest<true>(d_out, R, key, ok, hist, &K, &need);
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
    for (int i = 0; i < GS; ++i) x[i] = v[vpos(base + (i << s))];
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
    for (int i = 0; i < GS; ++i) v[vpos(base + (i << s))] = x[i];
  }
}

// v[0..d_in) = w[0..d_in) H_unnormalised per block of n, fp64 butterflies in
// the textbook stage order (three stages per pass over aligned groups of 8,
// the last pass one or two when log2 n is not a multiple of 3); v is shared
// memory at the padded positions vpos(k), every thread of the block takes part.
__device__ void row_transform_fp64(const float *__restrict__ w, int d_in, int n, double *v) {
  for (int k = threadIdx.x; k < d_in; k += blockDim.x) v[vpos(k)] = (double)w[k];
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

// NT threads per row: 256, or 1024 for long rows, whose buffer leaves room for
// one CTA per SM only.
template <int NT>
__global__ void __launch_bounds__(NT)
    select_kernel(const float *__restrict__ dW, int d_in, int n, const int32_t *__restrict__ budgets,
                  const int32_t *__restrict__ row_ptr, int64_t p, int32_t *__restrict__ col_idx,
                  float *__restrict__ coef) {
  extern __shared__ __align__(16) double v[];  // d_in values of the row
  __shared__ uint32_t hist[kHistBins];
  __shared__ int64_t sh64[128];
  const int64_t row = blockIdx.x;
  row_transform_fp64(dW + row * d_in, d_in, n, v);
  const int b = budgets[row];
  int64_t start = (int64_t)row_ptr[row] - row_ptr[0];  // row_ptr may be a slice of a longer one
  if (b <= 0 || start < 0 || start + b > p) return;
  const double inv = __ddiv_rn(1.0, __dsqrt_rn((double)n));
  // largest |V| = smallest complemented magnitude bits
  auto key = [&](int k) -> uint64_t { return ~((uint64_t)__double_as_longlong(v[vpos(k)]) & 0x7fffffffffffffffull); };
  auto ok = [&](int) { return true; };
  uint64_t K;
  int64_t need;
  radix_select_smallest<false>(d_in, b, key, ok, hist, &K, &need);
  __syncthreads();
  ordered_take(d_in, K, need, key, ok,
               [&](int k, int64_t slot) {
                 if (slot < b) {
                   col_idx[start + slot] = k;
                   coef[start + slot] = __double2float_rn(__dmul_rn(v[vpos(k)], inv));
                 }
               },
               sh64);
}

// Rows of exactly 4096 entries (every workload shape but down_proj): the same
// selection with the row in registers. 256 threads x 16 values; the 12
// butterfly stages run in three register phases of 4 stages (textbook order,
// so the fp64 results are those of row_transform_fp64 bit for bit):
//   phase 1: thread t holds entries 16t + j       (stages h = 1 .. 8)
//   phase 2: entries (t % 16) + 16 j + 256 (t / 16) (h = 16 .. 128)
//   phase 3: entries t + 256 j                      (h = 256 .. 2048)
// with two exchanges through the padded shared buffer (conflict-free for all
// four access patterns). Stages at or above the Hadamard block are skipped.
// The values then stay in registers (and, for the candidate lists, in the
// buffer): the common-prefix sweep, one 10-bit histogram pass, a listing sweep
// and the warp-level finish of radix_select_smallest, then the ordered
// compaction in index order (index 256 j + t: rounds j, warps in order inside
// a round).
constexpr int kRow4k = 4096;

__device__ __forceinline__ void bfly16(double *x, int b0, int logn) {
#pragma unroll
  for (int b = 0; b < 4; ++b) {
    if (b0 + b >= logn) break;
    const int h = 1 << b;
#pragma unroll
    for (int j = 0; j < 16; ++j)
      if (!(j & h)) {
        const double a = x[j], c = x[j + h];
        x[j] = __dadd_rn(a, c);
        x[j + h] = __dsub_rn(a, c);
      }
  }
}

__global__ void __launch_bounds__(kSelThreads, 3)
    select4k_kernel(const float *__restrict__ dW, int n, const int32_t *__restrict__ budgets,
                    const int32_t *__restrict__ row_ptr, int64_t p, int32_t *__restrict__ col_idx,
                    float *__restrict__ coef) {
  extern __shared__ __align__(16) double v[];  // vpos(4096) doubles
  __shared__ uint32_t hist[kHistBins];
  __shared__ int cand[kCandCap];
  __shared__ int cand_n;
  __shared__ unsigned long long s_and, s_or, s_K, fk[32];
  __shared__ int s_digit, s_done;
  __shared__ long long s_need;
  __shared__ uint32_t s_match;
  __shared__ int s_cnt[2][16][8];  // per (round j, warp): keys < K, keys == K
  __shared__ int s_base[16][8];    // output slot of each (round, warp)
  __shared__ int s_eqb[16][8];     // keys == K before each (round, warp)
  const int t = threadIdx.x, lane = t & 31, warp = t >> 5;
  const int64_t row = blockIdx.x;
  const int logn = 31 - __clz(n);
  const int b = budgets[row];
  const int64_t start = (int64_t)row_ptr[row] - row_ptr[0];  // row_ptr may be a slice of a longer one
  if (b <= 0 || start < 0 || start + b > p) return;

  double x[16];
  {
    const float4 *src = reinterpret_cast<const float4 *>(dW + row * kRow4k + 16 * t);
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const float4 f = src[q];
      x[4 * q] = (double)f.x, x[4 * q + 1] = (double)f.y, x[4 * q + 2] = (double)f.z, x[4 * q + 3] = (double)f.w;
    }
  }
  bfly16(x, 0, logn);
#pragma unroll
  for (int j = 0; j < 16; ++j) v[vpos(16 * t + j)] = x[j];
  __syncthreads();
  const int e2 = (t & 15) + 256 * (t >> 4);
#pragma unroll
  for (int j = 0; j < 16; ++j) x[j] = v[vpos(e2 + 16 * j)];
  bfly16(x, 4, logn);
  // each thread rewrites only the positions it has just read: no barrier
#pragma unroll
  for (int j = 0; j < 16; ++j) v[vpos(e2 + 16 * j)] = x[j];
  __syncthreads();
#pragma unroll
  for (int j = 0; j < 16; ++j) x[j] = v[vpos(t + 256 * j)];
  bfly16(x, 8, logn);
  // the final values back in place (own positions again), for the candidate lists
#pragma unroll
  for (int j = 0; j < 16; ++j) v[vpos(t + 256 * j)] = x[j];

  // keys: largest |V| = smallest complemented magnitude bits
  auto kx = [](double d) -> uint64_t { return ~((uint64_t)__double_as_longlong(d) & 0x7fffffffffffffffull); };
  if (t == 0) {
    s_and = ~0ull;
    s_or = 0ull;
    cand_n = 0;
    s_done = 0;
  }
  __syncthreads();
  {
    uint64_t ka = ~0ull, ko = 0ull;
#pragma unroll
    for (int j = 0; j < 16; ++j) {
      ka &= kx(x[j]);
      ko |= kx(x[j]);
    }
    const uint32_t alo = __reduce_and_sync(0xffffffffu, (uint32_t)ka);
    const uint32_t ahi = __reduce_and_sync(0xffffffffu, (uint32_t)(ka >> 32));
    const uint32_t olo = __reduce_or_sync(0xffffffffu, (uint32_t)ko);
    const uint32_t ohi = __reduce_or_sync(0xffffffffu, (uint32_t)(ko >> 32));
    if (lane == 0) {
      atomicAnd(&s_and, ((unsigned long long)ahi << 32) | alo);
      atomicOr(&s_or, ((unsigned long long)ohi << 32) | olo);
    }
  }
  __syncthreads();
  const uint64_t kand = s_and, kor = s_or;
  uint64_t K;
  int64_t need = b;
  if (b >= kRow4k || kand == kor) {
    K = b >= kRow4k ? ~0ull : kand;  // everything, or all keys equal
  } else {
    const int hb = 63 - __clzll((long long)(kand ^ kor));
    uint64_t prefix = hb == 63 ? 0ull : (kand & ~((2ull << hb) - 1ull));
    int bits = hb + 1 < 10 ? hb + 1 : 10;
    int shift = hb + 1 - bits;
    uint32_t match = kRow4k;
    bool listed = false;
    for (;;) {
      const uint64_t hi_mask = shift + bits >= 64 ? 0ull : ~((1ull << (shift + bits)) - 1ull);
      const uint64_t pm = prefix & hi_mask;
      const int bins = 1 << bits;
      if (!listed && match <= (uint32_t)kCandCap) {
#pragma unroll
        for (int j = 0; j < 16; ++j) {
          const bool m = (kx(x[j]) & hi_mask) == pm;
          const unsigned mm = __ballot_sync(0xffffffffu, m);
          int base = 0;
          if (lane == 0 && mm) base = atomicAdd(&cand_n, __popc(mm));
          base = __shfl_sync(0xffffffffu, base, 0);
          if (m) cand[base + __popc(mm & ((1u << lane) - 1u))] = t + 256 * j;
        }
        listed = true;
        __syncthreads();
      }
      if (listed && match <= 32u) {
        if (warp == 0)
          warp_rank_finish([&](int e) { return kx(v[vpos(e)]); }, cand, cand_n, hi_mask, pm, need, fk, &s_K, &s_need,
                           &s_done);
        __syncthreads();
        if (s_done) {
          prefix = s_K;
          need = s_need;
          break;
        }
      }
      for (int i = t; i < bins; i += kSelThreads) hist[i] = 0;
      __syncthreads();
      if (listed) {
        const int m_round = (cand_n + kSelThreads - 1) / kSelThreads * kSelThreads;
        for (int it = t; it < m_round; it += kSelThreads) {
          int bin = kHistBins;
          if (it < cand_n) {
            const uint64_t kc = kx(v[vpos(cand[it])]);
            if ((kc & hi_mask) == pm) bin = (int)((kc >> shift) & (uint64_t)(bins - 1));
          }
          if (bin < kHistBins) atomicAdd(&hist[bin], 1u);
        }
      } else {
#pragma unroll
        for (int j = 0; j < 16; ++j) {
          const uint64_t kj = kx(x[j]);
          const int bin = (kj & hi_mask) == pm ? (int)((kj >> shift) & (uint64_t)(bins - 1)) : kHistBins;
          if (bin < kHistBins) atomicAdd(&hist[bin], 1u);
        }
      }
      __syncthreads();
      if (warp == 0) {
        const int per = (bins + 31) / 32;
        uint32_t mine = 0;
        for (int j = 0; j < per; ++j) {
          const int bb = lane * per + j;
          mine += bb < bins ? hist[bb] : 0u;
        }
        uint32_t incl = mine;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
          const uint32_t o = __shfl_up_sync(0xffffffffu, incl, off);
          if (lane >= off) incl += o;
        }
        const int64_t excl = (int64_t)(incl - mine);
        if (excl < need && (int64_t)incl >= need) {
          int64_t cum = excl;
          for (int j = 0; j < per; ++j) {
            const int bb = lane * per + j;
            const uint32_t c = bb < bins ? hist[bb] : 0u;
            if (cum + c >= need) {
              s_digit = bb;
              s_need = need - cum;
              s_match = c;
              break;
            }
            cum += c;
          }
        }
      }
      __syncthreads();
      prefix |= (uint64_t)s_digit << shift;
      need = s_need;
      match = s_match;
      __syncthreads();
      if (shift == 0) break;
      bits = shift < 8 ? shift : 8;
      shift -= bits;
    }
    K = prefix;
  }

  // ordered compaction: index 256 j + t, rounds j, warps in order inside a round
#pragma unroll
  for (int j = 0; j < 16; ++j) {
    const unsigned m_lt = __ballot_sync(0xffffffffu, kx(x[j]) < K);
    const unsigned m_eq = __ballot_sync(0xffffffffu, kx(x[j]) == K);
    if (lane == 0) {
      s_cnt[0][j][warp] = __popc(m_lt);
      s_cnt[1][j][warp] = __popc(m_eq);
    }
  }
  __syncthreads();
  if (warp == 0) {
    // 128 chunks in index order (chunk c = 8 j + w), four per lane
    int lt4[4], eq4[4];
    int lt_s = 0, eq_s = 0;
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const int c = 4 * lane + q;
      lt4[q] = s_cnt[0][c >> 3][c & 7];
      eq4[q] = s_cnt[1][c >> 3][c & 7];
      lt_s += lt4[q];
      eq_s += eq4[q];
    }
    int lt_x = lt_s, eq_x = eq_s;  // inclusive scans over lanes
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const int a = __shfl_up_sync(0xffffffffu, lt_x, off), e = __shfl_up_sync(0xffffffffu, eq_x, off);
      if (lane >= off) {
        lt_x += a;
        eq_x += e;
      }
    }
    int lt_before = lt_x - lt_s, eq_before = eq_x - eq_s;
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const int c = 4 * lane + q;
      // keys < K before the chunk, plus the keys == K taken before it
      s_base[c >> 3][c & 7] = lt_before + (int)(need < eq_before ? need : eq_before);
      s_eqb[c >> 3][c & 7] = eq_before;
      lt_before += lt4[q];
      eq_before += eq4[q];
    }
  }
  __syncthreads();
  const double inv = __ddiv_rn(1.0, __dsqrt_rn((double)n));
  const unsigned below = (1u << lane) - 1u;
#pragma unroll
  for (int j = 0; j < 16; ++j) {
    const uint64_t kj = kx(x[j]);
    const bool is_lt = kj < K, is_eq = kj == K;
    const unsigned m_eq = __ballot_sync(0xffffffffu, is_eq);
    const bool take = is_lt || (is_eq && s_eqb[j][warp] + __popc(m_eq & below) < need);
    const unsigned m_t = __ballot_sync(0xffffffffu, take);
    if (take) {
      const int slot = s_base[j][warp] + __popc(m_t & below);
      if (slot < b) {
        col_idx[start + slot] = t + 256 * j;
        coef[start + slot] = __double2float_rn(__dmul_rn(x[j], inv));
      }
    }
  }
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
  unsigned long long prefix;  // digits of K fixed so far (all of K once `listed`)
  long long need;             // how many keys equal to the prefix are still to be taken
  uint32_t hist[256];
  unsigned long long cand_n;  // keys in the candidate list
  uint32_t match;             // keys that match the prefix after the last pass
  int want_list;              // the keys matching the prefix fit the list: list them
  int listed;                 // K and need are final; later passes do nothing
};

// Once the keys that match the prefix number at most kGselCap, one pass copies
// them into a list in the workspace and a single CTA finishes the selection on
// the list (the remaining passes over all keys are skipped).
constexpr int kGselCap = 1 << 16;

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
  for (int k = threadIdx.x; k < d_in; k += blockDim.x) V[row * d_in + k] = v[vpos(k)];
}

__global__ void gsel_init_kernel(GselState *st, int64_t p) {
  if (threadIdx.x == 0) {
    st->prefix = 0;
    st->need = p;
    st->cand_n = 0;
    st->match = 0xffffffffu;
    st->want_list = 0;
    st->listed = 0;
  }
  for (int i = threadIdx.x; i < 256; i += blockDim.x) st->hist[i] = 0;
}

// Histogram of digit `shift` over the keys that match the prefix so far.
__global__ void __launch_bounds__(kGselThreads)
    gsel_hist_kernel(const double *__restrict__ V, int64_t N, int sel, uint64_t seed, int shift, GselState *st) {
  if (st->listed) return;
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
  if (st->listed) return;
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
    st->prefix |= (unsigned long long)d << shift;
    st->need = need - cum;
    st->match = cnt;
    st->want_list = need - cum > 0 && cnt <= (uint32_t)kGselCap;
  } else if (who == 0 && lane == 31) {
    st->prefix |= 255ull << shift;
    st->need = need - (long long)incl;
  }
  __syncwarp();
#pragma unroll
  for (int j = 0; j < 8; ++j) st->hist[8 * lane + j] = 0;
}

// The keys that match the prefix after pass `shift` (at most kGselCap) into cand.
__global__ void __launch_bounds__(kGselThreads)
    gsel_list_kernel(const double *__restrict__ V, int64_t N, int sel, uint64_t seed, int shift, GselState *st,
                     unsigned long long *__restrict__ cand) {
  if (st->listed || !st->want_list) return;
  const uint64_t prefix = st->prefix;
  const uint64_t mask = ~0ull << shift;
  const int lane = threadIdx.x & 31;
  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  const int64_t n_round = (N + stride - 1) / stride * stride;
  for (int64_t j = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; j < n_round; j += stride) {
    uint64_t k = 0;
    bool m = false;
    if (j < N) {
      k = gsel_key(V, j, sel, seed);
      m = (k & mask) == (prefix & mask);
    }
    const unsigned mm = __ballot_sync(0xffffffffu, m);
    unsigned long long base = 0;
    if (lane == 0 && mm) base = atomicAdd(&st->cand_n, (unsigned long long)__popc(mm));
    base = __shfl_sync(0xffffffffu, base, 0);
    const unsigned long long at = base + __popc(mm & ((1u << lane) - 1u));
    if (m && at < (unsigned long long)kGselCap) cand[at] = k;
  }
}

// One CTA: K and its need from the candidate list (the radix select of the
// per-row selection, over the list); the remaining passes then do nothing.
__global__ void __launch_bounds__(1024) gsel_finish_kernel(GselState *st, const unsigned long long *__restrict__ cand) {
  if (st->listed || !st->want_list) return;
  __shared__ uint32_t hist[kHistBins];
  const unsigned long long n64 = st->cand_n;
  const int n = (int)(n64 < (unsigned long long)kGselCap ? n64 : (unsigned long long)kGselCap);
  uint64_t K;
  int64_t need;
  radix_select_smallest<false>(n, st->need, [&](int i) -> uint64_t { return cand[i]; }, [](int) { return true; },
                               hist, &K, &need);
  __syncthreads();
  if (threadIdx.x == 0) {
    st->prefix = K;
    st->need = need;
    st->listed = 1;
  }
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
  for (int k = threadIdx.x; k < d_in; k += blockDim.x) v[vpos(k)] = V[row * d_in + k];
  __syncthreads();
  const int64_t start = row_ptr[row];
  const int64_t cnt = (int64_t)row_ptr[row + 1] - start;
  if (cnt <= 0 || start < 0 || start + cnt > p) return;
  const uint64_t K = st->prefix;
  const double inv = __ddiv_rn(1.0, __dsqrt_rn((double)n));
  auto key = [&](int k) -> uint64_t {
    if (sel == 0) return ~((uint64_t)__double_as_longlong(v[vpos(k)]) & 0x7fffffffffffffffull);
    return splitmix64_at(seed, (uint64_t)(row * d_in + k) + 1);
  };
  auto ok = [&](int) { return true; };
  ordered_take(d_in, K, take_eq[row], key, ok,
               [&](int k, int64_t slot) {
                 if (slot < cnt) {
                   col_idx[start + slot] = k;
                   coef[start + slot] = __double2float_rn(__dmul_rn(v[vpos(k)], inv));
                 }
               },
               sh64);
}

// ---------------------------------------------------------------- energy concentration (selection diagnostics)
//
// Hill's estimate over the k largest coefficient magnitudes a = |V| and the
// energy they hold, from the (k+1)-th largest magnitude thr = a_(k+1) found by
// the radix select above (with need = k + 1):
//   sum_{i<=k} ln(a_(i) / thr) = sum over a > thr of ln(a / thr)   (ties add 0)
//   sum_{i<=k} a_(i)^2 = sum over a > thr of a^2 + (k - #{a > thr}) thr^2
// Per-CTA partial sums (fixed thread-to-element map and tree), then one CTA
// adds them in a fixed order: the result does not depend on scheduling.

constexpr int kEnergyMaxParts = 2048;

struct EnergyPart {
  double hill, top2, all2;
  long long gt;
};

__device__ __forceinline__ double magnitude_of_key(uint64_t key) {
  return __longlong_as_double((long long)(~key & 0x7fffffffffffffffull));
}

__global__ void __launch_bounds__(kGselThreads)
    energy_part_kernel(const double *__restrict__ V, int64_t N, const GselState *st, EnergyPart *__restrict__ part) {
  __shared__ double shd[33];
  __shared__ long long shl[33];
  const double thr = magnitude_of_key(st->prefix);
  double hill = 0.0, top2 = 0.0, all2 = 0.0;
  long long gt = 0;
  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  for (int64_t j = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; j < N; j += stride) {
    const double a = fabs(V[j]);
    all2 += a * a;
    if (a > thr) {
      if (thr > 0.0) hill += log(a / thr);
      top2 += a * a;
      ++gt;
    }
  }
  hill = block_sum(hill, shd);
  top2 = block_sum(top2, shd);
  all2 = block_sum(all2, shd);
  gt = block_sum(gt, shl);
  if (threadIdx.x == 0) part[blockIdx.x] = EnergyPart{hill, top2, all2, gt};
}

__global__ void __launch_bounds__(kGselThreads)
    energy_finish_kernel(const EnergyPart *__restrict__ part, int nparts, int64_t k, const GselState *st,
                         double *__restrict__ out) {
  __shared__ double shd[33];
  __shared__ long long shl[33];
  double hill = 0.0, top2 = 0.0, all2 = 0.0;
  long long gt = 0;
  for (int i = threadIdx.x; i < nparts; i += blockDim.x) {
    hill += part[i].hill;
    top2 += part[i].top2;
    all2 += part[i].all2;
    gt += part[i].gt;
  }
  hill = block_sum(hill, shd);
  top2 = block_sum(top2, shd);
  all2 = block_sum(all2, shd);
  gt = block_sum(gt, shl);
  if (threadIdx.x == 0) {
    const double thr = magnitude_of_key(st->prefix);
    const double top = top2 + (double)(k - gt) * thr * thr;
    const double xi = hill / (double)k;
    out[0] = (thr > 0.0 && xi > 0.0) ? 1.0 / xi : __longlong_as_double(0x7ff8000000000000ll);
    out[1] = all2 > 0.0 ? top / all2 : __longlong_as_double(0x7ff8000000000000ll);
    out[2] = thr;
    out[3] = all2;
  }
}

}  // namespace

size_t init_workspace(int32_t d_out, int32_t d_in) {
  (void)d_in;
  return align_up((size_t)d_out * 8, 256) + align_up((size_t)d_out, 256);
}

int init_max_din() { return kMaxInitDin; }

// The per-row selection: rows of 4096 entries in registers, others through
// the generic shared-memory kernel.
cudaError_t launch_select_rows(const float *dW, int32_t rows, int32_t d_in, int32_t had_block, const int32_t *budgets,
                               const int32_t *row_ptr, int64_t p, int32_t *col_idx, float *coef, cudaStream_t s) {
  const size_t smem = vbytes(d_in);
  if (d_in == kRow4k && aligned16(dW)) {
    auto k = select4k_kernel;
    cudaError_t err = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (err != cudaSuccess) return err;
    k<<<rows, kSelThreads, smem, s>>>(dW, had_block, budgets, row_ptr, p, col_idx, coef);
    return cudaGetLastError();
  }
  const bool wide = smem > 64 * 1024;
  auto k = wide ? select_kernel<1024> : select_kernel<kSelThreads>;
  cudaError_t err = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (err != cudaSuccess) return err;
  k<<<rows, wide ? 1024 : kSelThreads, smem, s>>>(dW, d_in, had_block, budgets, row_ptr, p, col_idx, coef);
  return cudaGetLastError();
}

cudaError_t launch_init_alloc(const float *dW, int32_t d_out, int32_t d_in, int32_t had_block, int64_t p,
                              int32_t min_per_row, int mode, int32_t *budgets, int32_t *row_ptr, int32_t *col_idx,
                              float *coef, void *ws, cudaStream_t s) {
  double *e = static_cast<double *>(ws);
  unsigned char *capped = static_cast<unsigned char *>(ws) + align_up((size_t)d_out * 8, 256);
  row_norm_kernel<<<d_out, kNormThreads, 0, s>>>(dW, d_in, e);
  budget_kernel<<<1, kBudgetThreads, 0, s>>>(e, d_out, d_in, p, min_per_row, mode, budgets, row_ptr, capped);
  if (p > 0) return launch_select_rows(dW, d_out, d_in, had_block, budgets, row_ptr, p, col_idx, coef, s);
  return cudaGetLastError();
}

size_t select_global_workspace(int32_t d_out, int32_t d_in) {
  return align_up((size_t)d_out * d_in * 8, 256) + align_up(sizeof(GselState), 256) + 3 * align_up((size_t)d_out * 4, 256) +
         (size_t)kGselCap * 8;
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
  w += align_up((size_t)d_out * 4, 256);
  unsigned long long *cand = reinterpret_cast<unsigned long long *>(w);
  const size_t smem = vbytes(d_in);
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
    if (shift > 0) {  // after the last pass the prefix is K itself
      gsel_list_kernel<<<(unsigned)grid, kGselThreads, 0, s>>>(V, N, sel, seed, shift, st, cand);
      gsel_finish_kernel<<<1, 1024, 0, s>>>(st, cand);
    }
  }
  gsel_count_kernel<<<d_out, kGselThreads, 0, s>>>(V, d_in, sel, seed, st, lt, eq);
  gsel_budget_kernel<<<1, kBudgetThreads, 0, s>>>(lt, eq, d_out, st, take, budgets, row_ptr);
  if (p > 0)
    gsel_take_kernel<<<d_out, kSelThreads, smem, s>>>(V, d_in, had_block, sel, seed, st, take, row_ptr, p, col_idx,
                                                      coef);
  return cudaGetLastError();
}

size_t energy_stats_workspace(int32_t d_out, int32_t d_in) {
  return select_global_workspace(d_out, d_in) + align_up((size_t)kEnergyMaxParts * sizeof(EnergyPart), 256);
}

cudaError_t launch_energy_stats(const float *dW, int32_t d_out, int32_t d_in, int32_t had_block, int64_t k,
                                double *out, void *ws, cudaStream_t s) {
  char *w = static_cast<char *>(ws);
  double *V = reinterpret_cast<double *>(w);
  w += align_up((size_t)d_out * d_in * 8, 256);
  GselState *st = reinterpret_cast<GselState *>(w);
  w += align_up(sizeof(GselState), 256);
  w += 3 * align_up((size_t)d_out * 4, 256);
  unsigned long long *cand = reinterpret_cast<unsigned long long *>(w);
  w += (size_t)kGselCap * 8;
  EnergyPart *part = reinterpret_cast<EnergyPart *>(w);
  const size_t smem = vbytes(d_in);
  cudaError_t e = cudaFuncSetAttribute(gsel_transform_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  const int64_t N = (int64_t)d_out * d_in;
  gsel_transform_kernel<<<d_out, kSelThreads, smem, s>>>(dW, d_in, had_block, V);
  gsel_init_kernel<<<1, 256, 0, s>>>(st, k + 1);  // the (k+1)-th largest magnitude
  const int64_t grid = std::min<int64_t>(cdiv(N, (int64_t)kGselThreads), (int64_t)sm_count() * 8);
  for (int shift = 56; shift >= 0; shift -= 8) {
    gsel_hist_kernel<<<(unsigned)grid, kGselThreads, 0, s>>>(V, N, 0, 0, shift, st);
    gsel_pick_kernel<<<1, 32, 0, s>>>(st, shift);
    if (shift > 0) {
      gsel_list_kernel<<<(unsigned)grid, kGselThreads, 0, s>>>(V, N, 0, 0, shift, st, cand);
      gsel_finish_kernel<<<1, 1024, 0, s>>>(st, cand);
    }
  }
  const int parts = (int)std::min<int64_t>(grid, kEnergyMaxParts);
  energy_part_kernel<<<parts, kGselThreads, 0, s>>>(V, N, st, part);
  energy_finish_kernel<<<1, kGselThreads, 0, s>>>(part, parts, k, st, out);
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
  return launch_select_rows(dW, rows, d_in, had_block, budgets, row_ptr, p, col_idx, coef, s);
}

}  // namespace qwha
