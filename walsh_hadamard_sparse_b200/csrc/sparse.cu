// Sparse products of the adapter with F = Scatter(c, E) ("QWHA",
// papernotes.org 整体框架; gist.science 2.1).
//
// SpMM: out[t, i] = alpha * sum_{j in segment i} val[j] * in[t, idx[j]].
//   Forward (segments = rows of F, CSR):  Y_ad = alpha Z F^T.
//   Backward (segments = columns of F, CSC, val through perm): dZ = alpha dY F.
//   A CTA owns TT tokens: their input rows are staged transposed in shared
//   memory (a column of the tile is TT contiguous values). The segment
//   entries stream from L2 once per token tile, as packed (staged-row,
//   value) words that a preparation kernel writes first, ordered so that the
//   rows one shared-memory wavefront gathers sit on distinct banks as far as
//   the indices allow, with the CSC permutation applied to the coefficients
//   for the backward.
//   sell_spmm_kernel (the sliced layout, see the section that defines it): a
//   slot owns a whole segment; segments are ranked by length within windows
//   of output columns, whose results the CTA writes as whole rows.
//   seg_spmm_kernel (shapes the sliced layout does not take): a warp spreads
//   one segment at a time over its slots and reduces across them at the end.
//
// sddmm: partial[c, j] = sum_{t in chunk c} dY[t, r_j] * Z[t, k_j] over the
//   tile view of E (QWHA_TILE x QWHA_TILE blocks of F). Grid = tiles x token
//   chunks; a CTA multiplies dY[:, row block] and Z[:, column block] held
//   transposed in shared memory, 64 (bf16) or 32 (fp32) tokens at a time. For
//   bf16, sdd_transpose_kernel transposes dY and Z once into the layout the
//   CTAs read and sddmm_t_kernel feeds itself by tensor copies; the other
//   kernels stage and transpose their own slices (see Sdd16Slot and
//   sddmm_kernel for the lane layouts).
// sddmm_reduce: dc[j] = alpha * sum_c partial[c, j] in increasing c (fixed
//   order: the result is bitwise reproducible).

#include <algorithm>
#include <type_traits>

#include "bulk.cuh"
#include "common.cuh"
#include "kernels.h"

namespace qwha {
namespace {

constexpr int kSpmmThreads = 1024;

// For a kernel that runs one CTA per SM over `units` independent CTAs: the
// smallest factor s <= max_split by which to subdivide each unit so that the
// last wave is at least 95% full (else the factor with the fullest last wave).
int wave_split(int64_t units, int max_split) {
  const int64_t slots = sm_count();
  int best = 1;
  double best_eff = 0.0;
  for (int s = 1; s <= max_split; ++s) {
    const int64_t n = units * s;
    const double eff = (double)n / (double)(cdiv(n, slots) * slots);
    if (eff >= 0.95) return s;
    if (eff > best_eff + 1e-9) {
      best_eff = eff;
      best = s;
    }
  }
  return best;
}
constexpr size_t kSpmmSmemCap = 220 * 1024;

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

// d = a * b + c with a, b bf16 (the low or high half of a 32-bit word) and
// c, d fp32: the product of two bf16 values is exact in fp32, so this is an
// fp32 FMA on the widened operands without the widening instructions.
__device__ __forceinline__ float fma_bf16_lo(uint32_t a2, uint32_t b2, float c) {
  float d;
  asm("{\n\t.reg .b16 al, ah, bl, bh;\n\tmov.b32 {al, ah}, %1;\n\tmov.b32 {bl, bh}, %2;\n\t"
      "fma.rn.f32.bf16 %0, al, bl, %3;\n\t}"
      : "=f"(d)
      : "r"(a2), "r"(b2), "f"(c));
  return d;
}
__device__ __forceinline__ float fma_bf16_hi(uint32_t a2, uint32_t b2, float c) {
  float d;
  asm("{\n\t.reg .b16 al, ah, bl, bh;\n\tmov.b32 {al, ah}, %1;\n\tmov.b32 {bl, bh}, %2;\n\t"
      "fma.rn.f32.bf16 %0, ah, bh, %3;\n\t}"
      : "=f"(d)
      : "r"(a2), "r"(b2), "f"(c));
  return d;
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

// Gather order. The SpMM stages the token tile transposed, one row of
// R = TT * sizeof(Tin) bytes per input column (32 bytes for 16 bf16 tokens),
// so a 128-byte bank line holds M = 128 / R rows and column k lands at line
// position k mod M. One shared-memory wavefront of the gather serves the
// lanes of M consecutive entries of a segment (counted from the segment
// start): two of them with equal k mod M and different k are a bank
// conflict. arrange_kernel (one warp per segment) orders the entries by
// (rank within their residue class, residue), round robin over the classes:
// an aligned group of M entries then holds M distinct residues until the
// smaller classes run out. The entry of residue m and rank q goes to
//   start + sum_m' min(cnt[m'], q) + #{m' < m : cnt[m'] > q},
// a bijection onto the segment. It writes (index, value bits) pairs, the
// value taken through perm when there is one. The order only changes the
// fp32 summation order, and it depends on E and R alone (not on T), so the
// results are repeatable.
template <int M>
__global__ void __launch_bounds__(256)
    arrange_kernel(const int32_t *__restrict__ seg_ptr, int n_seg, const int32_t *__restrict__ idx,
                   const float *__restrict__ val, const int32_t *__restrict__ perm, int64_t nnz64,
                   int2 *__restrict__ ent) {
  static_assert(M >= 1 && M <= 32 && (M & (M - 1)) == 0, "residue classes");
  const int lane = threadIdx.x & 31;
  const int nnz = (int)nnz64;
  const unsigned below = (1u << lane) - 1u;
  const int warps = (int)gridDim.x * (int)(blockDim.x >> 5);
  for (int seg = (int)blockIdx.x * (int)(blockDim.x >> 5) + (int)(threadIdx.x >> 5); seg < n_seg;
       seg += warps) {
    // the segment as the SpMM reads it: both ends clamped to [0, nnz]
    int s = seg_ptr[seg], e = seg_ptr[seg + 1];
    s = s < 0 ? 0 : (s > nnz ? nnz : s);
    e = e < s ? s : (e > nnz ? nnz : e);
    int cnt[M];
#pragma unroll
    for (int m = 0; m < M; ++m) cnt[m] = 0;
    for (int j = s + lane; j < e; j += 32) {
      const int r = __ldg(idx + j) & (M - 1);
#pragma unroll
      for (int m = 0; m < M; ++m) cnt[m] += r == m ? 1 : 0;
    }
#pragma unroll
    for (int m = 0; m < M; ++m)
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) cnt[m] += __shfl_xor_sync(0xffffffffu, cnt[m], off);
    int run[M];  // entries of each class in earlier 32-entry chunks
#pragma unroll
    for (int m = 0; m < M; ++m) run[m] = 0;
    for (int b = s; b < e; b += 32) {
      const int j = b + lane;
      int k = 0, r = -1;
      float v = 0.f;
      if (j < e) {
        k = __ldg(idx + j);
        r = k & (M - 1);
        if (perm) {
          const int32_t src = __ldg(perm + j);
          v = (unsigned)src < (unsigned)nnz ? __ldg(val + src) : 0.f;
        } else {
          v = __ldg(val + j);
        }
      }
      int q = 0;
#pragma unroll
      for (int m = 0; m < M; ++m) {
        const unsigned bal = __ballot_sync(0xffffffffu, r == m);
        if (r == m) q = run[m] + __popc(bal & below);
        run[m] += __popc(bal);
      }
      if (j < e) {
        int pos = s;
#pragma unroll
        for (int m = 0; m < M; ++m) pos += (cnt[m] < q ? cnt[m] : q) + (m < r && cnt[m] > q ? 1 : 0);
        ent[pos] = make_int2(k, __float_as_int(v));
      }
    }
  }
}

// One warp per segment at a time. A lane holds G = min(TT, 8) consecutive
// tokens of the tile (Q = TT/G lanes cover it) for one of NSLOT = 32/Q nonzero
// slots: lane = q + Q * slot. A segment is cut into blocks of NSLOT * kUnroll
// nonzeros; slot s takes nonzeros base + s + NSLOT * u. Entries past the
// segment end, or with a column outside the tile, get index 0 and value 0.
// The next block's (index, value) loads go into the other register set while
// the current block is multiplied (the two sets alternate roles: no copies).
// bf16 tiles multiply with fma.rn.f32.bf16 (coefficient rounded to bf16, exact
// product, fp32 accumulation). At a segment's end a reduce-scatter over the
// slots leaves each token's sum in one lane. A warp takes segments in groups
// of kSegGroup consecutive ones: each result is parked in the warp's slice of
// shared memory, and at the group's end the warp writes, for every token, the
// group's kSegGroup consecutive outputs as one vector (a full 32-byte sector
// for fp32) instead of one scattered 4-byte store per segment. The shared
// loads and products of a step u whose slots all lie past the segment end
// are skipped (a warp-uniform test).
constexpr int kUnroll = 8;
constexpr int kSegGroup = 8;

// shared bytes of the per-warp output slices
template <typename Tout>
constexpr size_t spmm_obuf_bytes(int TT) {
  return (size_t)(kSpmmThreads / 32) * kSegGroup * TT * sizeof(float);
}

// N consecutive outputs from fp32 values, one vector store (the address is
// aligned to N outputs).
template <typename Tout, int N>
__device__ __forceinline__ void store_vec(Tout *o, const float *v) {
  if constexpr (std::is_same<Tout, float>::value) {
    if constexpr (N == 4) *reinterpret_cast<float4 *>(o) = make_float4(v[0], v[1], v[2], v[3]);
    else if constexpr (N == 2) *reinterpret_cast<float2 *>(o) = make_float2(v[0], v[1]);
    else o[0] = v[0];
  } else {
    if constexpr (N == 4) {
      const __nv_bfloat162 a = __floats2bfloat162_rn(v[0], v[1]), b = __floats2bfloat162_rn(v[2], v[3]);
      uint2 w;
      w.x = *reinterpret_cast<const uint32_t *>(&a);
      w.y = *reinterpret_cast<const uint32_t *>(&b);
      *reinterpret_cast<uint2 *>(o) = w;
    } else if constexpr (N == 2) {
      *reinterpret_cast<__nv_bfloat162 *>(o) = __floats2bfloat162_rn(v[0], v[1]);
    } else {
      o[0] = __float2bfloat16_rn(v[0]);
    }
  }
}

// acc[i] += v * row[i] for the G tokens (4 or 8) a lane holds.
template <int G>
__device__ __forceinline__ void mac_tokens(const __nv_bfloat16 *row, float v, float *acc) {
  const __nv_bfloat162 vb2 = __floats2bfloat162_rn(v, v);
  const uint32_t vv = *reinterpret_cast<const uint32_t *>(&vb2);
  uint32_t w[G / 2];
  if constexpr (G == 8) {
    const uint4 t = *reinterpret_cast<const uint4 *>(row);
    w[0] = t.x, w[1] = t.y, w[2] = t.z, w[3] = t.w;
  } else {
    const uint2 t = *reinterpret_cast<const uint2 *>(row);
    w[0] = t.x, w[1] = t.y;
  }
#pragma unroll
  for (int i = 0; i < G / 2; ++i) {
    acc[2 * i] = fma_bf16_lo(w[i], vv, acc[2 * i]);
    acc[2 * i + 1] = fma_bf16_hi(w[i], vv, acc[2 * i + 1]);
  }
}

template <int G>
__device__ __forceinline__ void mac_tokens(const float *row, float v, float *acc) {
#pragma unroll
  for (int h = 0; h < G / 4; ++h) {
    const float4 a = *reinterpret_cast<const float4 *>(row + 4 * h);
    acc[4 * h + 0] = fmaf(v, a.x, acc[4 * h + 0]);
    acc[4 * h + 1] = fmaf(v, a.y, acc[4 * h + 1]);
    acc[4 * h + 2] = fmaf(v, a.z, acc[4 * h + 2]);
    acc[4 * h + 3] = fmaf(v, a.w, acc[4 * h + 3]);
  }
}

template <typename Tin, typename Tout, int TT>
__global__ void __launch_bounds__(kSpmmThreads)
    seg_spmm_kernel(const Tin *__restrict__ in, int64_t T, int W_in, const int32_t *__restrict__ seg_ptr,
                    const int2 *__restrict__ ent, int64_t nnz64, int n_seg, float alpha,
                    Tout *__restrict__ out) {
  static_assert(TT == 4 || TT == 8 || TT == 16, "token tile");
  constexpr int G = TT < 8 ? TT : 8;  // tokens per lane
  constexpr int LV = G == 8 ? 3 : 2;  // reduce-scatter levels (log2 G)
  constexpr int Q = TT / G;           // lanes per nonzero
  constexpr int NSLOT = 32 / Q;    // slots per warp
  constexpr int BLOCK = NSLOT * kUnroll;
  constexpr int kWarps = kSpmmThreads / 32;
  constexpr int SG = kSegGroup;
  extern __shared__ __align__(16) unsigned char smem_raw[];
  Tin *s_in = reinterpret_cast<Tin *>(smem_raw);
  const size_t in_bytes = (size_t)W_in * TT * sizeof(Tin);
  int32_t *s_ptr = reinterpret_cast<int32_t *>(smem_raw + in_bytes);
  const int nnz = (int)nnz64;
  const int64_t t0 = (int64_t)blockIdx.x * TT;
  // this CTA's share of the segment groups (blockIdx.y of gridDim.y equal parts)
  const int n_grp = (n_seg + SG - 1) / SG;
  const int g_begin = (int)((int64_t)blockIdx.y * n_grp / gridDim.y);
  const int g_end = (int)((int64_t)(blockIdx.y + 1) * n_grp / gridDim.y);
  for (int i = threadIdx.x; i <= n_seg; i += kSpmmThreads) {
    const int v = seg_ptr[i];
    s_ptr[i] = v < 0 ? 0 : (v > nnz ? nnz : v);
  }
  stage_transposed<Tin, TT>(in, T, W_in, t0, 0, W_in, W_in, s_in);
  __syncthreads();

  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int q = lane % Q, slot = lane / Q;
  const Tin *s_q = s_in + G * q;
  // this warp's output slice: obuf[i * TT + token] for segment i of the current group
  float *obuf = reinterpret_cast<float *>(smem_raw + ((in_bytes + ((size_t)n_seg + 1) * 4 + 15) & ~(size_t)15)) +
                (size_t)warp * SG * TT;

  int grp = g_begin + warp, seg = grp * SG, pos = 0, end = 0;
  if (grp < g_end) {
    pos = s_ptr[seg];
    end = s_ptr[seg + 1];
  }
  auto load_block = [&](int p0, int e, int *kk, float *vv) {
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      const int j = p0 + slot + NSLOT * u;
      kk[u] = W_in;  // marks "no entry"
      vv[u] = 0.f;
      if (j < e) {
        const int2 w = __ldg(ent + j);
        kk[u] = w.x;
        vv[u] = __int_as_float(w.y);
      }
    }
  };
  int ka[kUnroll], kb[kUnroll];
  float va[kUnroll], vb[kUnroll];
  float acc[G];
#pragma unroll
  for (int i = 0; i < G; ++i) acc[i] = 0.f;

  auto step = [&](const int *kc, const float *vc, int *kn, float *vn) {
    int ngrp = grp, nseg = seg, npos = pos + BLOCK, nend = end;
    const bool last_of_seg = npos >= end;
    const int gend = min((grp + 1) * SG, n_seg);  // one past the group's last segment
    if (last_of_seg) {
      if (seg + 1 < gend) {
        nseg = seg + 1;
      } else {
        ngrp = grp + kWarps;
        nseg = ngrp * SG;
      }
      if (ngrp < g_end) {
        npos = s_ptr[nseg];
        nend = s_ptr[nseg + 1];
      }
    }
    if (ngrp < g_end) load_block(npos, nend, kn, vn);
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      if (pos + NSLOT * u >= end) break;  // no slot of this or later u holds an entry (warp-uniform)
      // an empty slot (past the segment's end) reads row 0 and adds zero products: cheaper than a
      // divergent branch around the shared load (measured: 896 against 866 us on q_proj)
      const bool ok = (unsigned)kc[u] < (unsigned)W_in;
      mac_tokens<G>(s_q + (ok ? kc[u] : 0) * TT, ok ? vc[u] : 0.f, acc);
    }
    if (last_of_seg) {
      // reduce-scatter over the top LV slot bits of the lane (16, 8[, 4]):
      // each level keeps half of the values and adds the partner's other half
      float r[G];
#pragma unroll
      for (int i = 0; i < G; ++i) r[i] = acc[i];
      int ti = 0;  // token (within the lane's G) that r[0] ends up holding
#pragma unroll
      for (int lvl = 0; lvl < LV; ++lvl) {
        const int off = 16 >> lvl;
        const int n = G >> (lvl + 1);
        const bool upper = (lane & off) != 0;
        if (upper) ti += n;
#pragma unroll
        for (int i = 0; i < n; ++i) {
          const float keep = upper ? r[i + n] : r[i];
          const float send = upper ? r[i] : r[i + n];
          r[i] = keep + __shfl_xor_sync(0xffffffffu, send, off);
        }
      }
      // the slot bits below those: a plain butterfly sum
      constexpr int kLow = 32 >> LV;
#pragma unroll
      for (int off = Q; off < kLow; off <<= 1) r[0] += __shfl_xor_sync(0xffffffffu, r[0], off);
      if ((lane & (kLow - 1) & ~(Q - 1)) == 0) obuf[(seg - grp * SG) * TT + G * q + ti] = alpha * r[0];
#pragma unroll
      for (int i = 0; i < G; ++i) acc[i] = 0.f;
      if (seg + 1 == gend) {
        // the group's outputs: lane = (token, part); a part is SG * TT / 32 consecutive segments
        constexpr int PARTS = 32 / TT, PER = SG / PARTS;
        __syncwarp();
        const int tt = lane / PARTS, s0 = (lane % PARTS) * PER;
        const int64_t t = t0 + tt;
        const int cnt = gend - grp * SG;
        if (t < T && s0 < cnt) {
          float v[PER];
#pragma unroll
          for (int i = 0; i < PER; ++i) v[i] = obuf[(s0 + i) * TT + tt];
          Tout *o = out + t * n_seg + grp * SG + s0;
          if (s0 + PER <= cnt && (n_seg % SG) == 0) {
            store_vec<Tout, PER>(o, v);
          } else {
            for (int i = 0; i < PER && s0 + i < cnt; ++i) io<Tout>::store1(o + i, v[i]);
          }
        }
        __syncwarp();  // the slice is read before the next group's results land in it
      }
    }
    grp = ngrp;
    seg = nseg;
    pos = npos;
    end = nend;
  };
  if (grp < g_end) load_block(pos, end, ka, va);
  while (grp < g_end) {
    step(ka, va, kb, vb);
    if (grp >= g_end) break;
    step(kb, vb, ka, va);
  }
}

// ---------------------------------------------------------------- sliced SpMM
//
// The same product with one segment per slot. Segments are ranked by length
// (longest first, ties by index) and cut into groups of NSLOT consecutive
// ranks; a group's entries are stored step-major, two steps of a slot next
// to each other: entry step t of the slot s of group g sits at
//   goff[g] + (t / 2) * 2 * NSLOT + 2 * s + (t & 1),
// padded with empty entries (offset 0, value 0) to the group's longest
// segment rounded up to an even count. A slot then runs its own segment
// start to end with no reduction across lanes, and the warp's steps stay
// full: on the q_proj pattern the padding is 0.3% of the entries, against 46%
// for groups of consecutive rows. Inside a segment the entries are ordered
// round robin over the residues of their column modulo M (the staged rows in
// one 128-byte bank line), starting at residue s mod M, so that the slots that
// share one shared-memory wavefront read rows on distinct banks until the
// smaller classes run out. An entry holds the byte offset of its staged row
// and the value, as a bf16 pair (v, v) for bf16 input (the products are
// those of seg_spmm_kernel) or as fp32 bits.
//
// Scratch (spmm_scratch_bytes): entries, then srank [n_seg], sseg [groups *
// NSLOT] (rank -> segment, -1 past the end), goff [groups + 1].
struct SellLayout {
  int n_grp;
  size_t ent_cap;  // entries
  size_t ent_off, srank_off, sseg_off, goff_off, total;
};

__host__ __device__ inline SellLayout sell_layout(int64_t p, int n_seg, int W_in, int nslot) {
  SellLayout L;
  L.n_grp = (n_seg + nslot - 1) / nslot;
  // p entries, plus padding: at most nslot times the longest segment (<= W_in) and one step a group
  L.ent_cap = (size_t)(p > 0 ? p : 0) + (size_t)nslot * ((size_t)W_in + 2) + (size_t)L.n_grp * nslot;
  auto up = [](size_t v) { return (v + 255) / 256 * 256; };
  L.ent_off = 0;
  L.srank_off = up(L.ent_cap * 8);
  L.sseg_off = L.srank_off + up((size_t)n_seg * 4);
  L.goff_off = L.sseg_off + up((size_t)L.n_grp * nslot * 4);
  L.total = L.goff_off + up(((size_t)L.n_grp + 1) * 4);
  return L;
}

// Rank of every segment within its window of ws consecutive segments (ws a
// power of two and a multiple of the group size): window * ws plus the
// number of segments of the window whose key (length descending, index
// ascending) is smaller, summed over chunks of kRankChunk keys (grid.y) with
// integer atomics on a zeroed srank, so the result does not depend on the
// order in which the chunks finish. Keys are unique (the index is part of
// them), so the ranks are a permutation that keeps every window in place.
constexpr int kRankChunk = 256;  // keys per chunk: 4096 segments in 1024-wide windows give 64 busy CTAs
__device__ __forceinline__ uint32_t sell_key(const int32_t *__restrict__ seg_ptr, int i, int nnz) {
  int a = seg_ptr[i], b = seg_ptr[i + 1];
  a = a < 0 ? 0 : (a > nnz ? nnz : a);
  b = b < a ? a : (b > nnz ? nnz : b);
  const int len = b - a < 65535 ? b - a : 65535;
  return ((uint32_t)(65535 - len) << 16) | (uint32_t)i;
}

__global__ void __launch_bounds__(256)
    sell_rank_kernel(const int32_t *__restrict__ seg_ptr, int n_seg, int64_t nnz64, int ws,
                     int32_t *__restrict__ srank) {
  __shared__ __align__(16) uint32_t keys[kRankChunk];
  const int nnz = (int)nnz64;
  const int c0 = (int)blockIdx.y * kRankChunk;
  const int n = n_seg - c0 < kRankChunk ? n_seg - c0 : kRankChunk;
  for (int j = threadIdx.x; j < kRankChunk; j += 256) keys[j] = j < n ? sell_key(seg_ptr, c0 + j, nnz) : 0xffffffffu;
  __syncthreads();
  const int i = (int)blockIdx.x * 256 + (int)threadIdx.x;
  if (i >= n_seg) return;
  const int w0 = i / ws * ws;  // this segment's window [w0, w0 + ws)
  const int lo = (w0 > c0 ? w0 : c0) - c0, hi = (w0 + ws < c0 + n ? w0 + ws : c0 + n) - c0;
  if (lo >= hi) return;  // the window does not meet this chunk
  const uint32_t mine = sell_key(seg_ptr, i, nnz);
  int cnt = 0;
  // lo is a multiple of 4; the keys past n up to (hi + 3) / 4 * 4 are padding and compare false
  for (int j = lo / 4; j < (hi + 3) / 4; ++j) {
    const uint4 k = reinterpret_cast<const uint4 *>(keys)[j];
    cnt += (k.x < mine) + (k.y < mine) + (k.z < mine) + (k.w < mine);
  }
  // the window's base, added by the chunk that holds the window's start (which always meets it)
  if (blockIdx.y == (unsigned)(w0 / kRankChunk)) cnt += w0;
  if (cnt) atomicAdd(srank + i, cnt);
}

// sseg[srank[i]] = i, and -1 for the positions past n_seg of the last group.
__global__ void sell_place_kernel(const int32_t *__restrict__ srank, int n_seg, int n_pad,
                                  int32_t *__restrict__ sseg) {
  const int i = (int)blockIdx.x * (int)blockDim.x + (int)threadIdx.x;
  if (i < n_seg) {
    const int r = srank[i];
    if ((unsigned)r < (unsigned)n_seg) sseg[r] = i;
  } else if (i < n_pad) {
    sseg[i] = -1;
  }
}

// goff[g] = nslot * sum over earlier groups of their step count (the length of
// the group's first, longest, segment, at most W_in, rounded up to even). One
// CTA.
__global__ void __launch_bounds__(1024)
    sell_offsets_kernel(const int32_t *__restrict__ seg_ptr, const int32_t *__restrict__ sseg, int n_grp,
                        int64_t nnz64, int nslot, int W_in, int32_t *__restrict__ goff) {
  __shared__ int32_t part[32];
  __shared__ int32_t carry;
  const int nnz = (int)nnz64;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  if (threadIdx.x == 0) carry = 0;
  __syncthreads();
  for (int g0 = 0; g0 < n_grp; g0 += 1024) {
    const int g = g0 + (int)threadIdx.x;
    int steps = 0;
    if (g < n_grp) {
      const int seg = sseg[(size_t)g * nslot];  // the group's first rank: its longest segment
      int a = seg_ptr[seg], b = seg_ptr[seg + 1];
      a = a < 0 ? 0 : (a > nnz ? nnz : a);
      b = b < a ? a : (b > nnz ? nnz : b);
      // a segment has at most W_in distinct columns; the cap keeps the layout within its scratch
      // even for a malformed one (whose entries past W_in are then left out)
      steps = ((b - a < W_in ? b - a : W_in) + 1) & ~1;
    }
    int v = steps;  // inclusive scan over the CTA
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const int u = __shfl_up_sync(0xffffffffu, v, off);
      if (lane >= off) v += u;
    }
    if (lane == 31) part[warp] = v;
    __syncthreads();
    if (warp == 0) {
      int w = part[lane];
#pragma unroll
      for (int off = 1; off < 32; off <<= 1) {
        const int u = __shfl_up_sync(0xffffffffu, w, off);
        if (lane >= off) w += u;
      }
      part[lane] = w;
    }
    __syncthreads();
    const int incl = v + (warp > 0 ? part[warp - 1] : 0) + carry;
    if (g < n_grp) goff[g] = (incl - steps) * nslot;
    __syncthreads();
    if (threadIdx.x == 1023) carry = incl;
    __syncthreads();
  }
  if (threadIdx.x == 0) goff[n_grp] = carry * nslot;
}

// Staged row of input column k in the sliced kernel: k with its low log2(M)
// bits XORed with bits 8 and up. The bank line position of a staged row is
// its index modulo M, and the columns a segment selects are not spread evenly
// over k mod M (on q_proj a row's largest residue class holds 34% of its
// entries, against 30% for random columns); mixing in the higher bits makes
// the classes as even as random ones (29%), so the round-robin order below
// meets fewer bank conflicts (CPU model of q_proj: 1.48 -> 1.25 wavefronts per
// conflict-free one). A bijection within each aligned block of M rows.
template <int M>
__host__ __device__ __forceinline__ int sell_row(int k) {
  return k ^ ((k >> 8) & (M - 1));
}

// stage_transposed with rows placed by sell_row<M>: s[sell_row(k) * TT + t].
template <typename T, int TT, int M>
__device__ __forceinline__ void stage_sliced(const T *__restrict__ in, int64_t T_, int W, int64_t t0, T *s) {
  constexpr int V = 16 / (int)sizeof(T);
  static_assert(256 % V == 0 && M <= 256, "the V columns of a chunk share their bits 8 and up");
  const int chunks = W / V;
  for (int it = threadIdx.x; it < chunks * TT; it += blockDim.x) {
    const int t = it % TT;
    const int c = it / TT;
    const int64_t tg = t0 + t;
    float v[V];
    if (tg < T_) {
      io<T>::unpack(*reinterpret_cast<const uint4 *>(in + tg * W + c * V), v);
    } else {
#pragma unroll
      for (int i = 0; i < V; ++i) v[i] = 0.f;
    }
    const int x = ((c * V) >> 8) & (M - 1);  // the same for the chunk's V columns
#pragma unroll
    for (int i = 0; i < V; ++i) io<T>::store1(s + (int64_t)((c * V + i) ^ x) * TT + t, v[i]);
  }
}

// One warp per segment: its entries in the rotated round-robin order at the
// positions of its slot, then the padding of the group. The slots of the last
// group past n_seg (ranks n_seg .. n_pad - 1) are written as empty segments.
template <typename Tin, int TT, int M, int NSLOT>
__global__ void __launch_bounds__(256)
    sell_arrange_kernel(const int32_t *__restrict__ seg_ptr, int n_seg, const int32_t *__restrict__ idx,
                        const float *__restrict__ val, const int32_t *__restrict__ perm, int64_t nnz64, int W_in,
                        const int32_t *__restrict__ srank, const int32_t *__restrict__ goff, int2 *__restrict__ ent) {
  static_assert(M >= 1 && M <= 32 && (M & (M - 1)) == 0, "residue classes");
  const int lane = threadIdx.x & 31;
  const int nnz = (int)nnz64;
  const unsigned below = (1u << lane) - 1u;
  const int warps = (int)gridDim.x * (int)(blockDim.x >> 5);
  const int n_pad = (n_seg + NSLOT - 1) / NSLOT * NSLOT;
  for (int seg = (int)blockIdx.x * (int)(blockDim.x >> 5) + (int)(threadIdx.x >> 5); seg < n_pad;
       seg += warps) {
    const bool real = seg < n_seg;
    int s = real ? seg_ptr[seg] : 0, e = real ? seg_ptr[seg + 1] : 0;
    s = s < 0 ? 0 : (s > nnz ? nnz : s);
    e = e < s ? s : (e > nnz ? nnz : e);
    const int rk = real ? srank[seg] : seg;
    const int g = rk / NSLOT, slot = rk % NSLOT;
    const int r0 = slot & (M - 1);  // the class this slot starts with
    const int base = goff[g], steps = (goff[g + 1] - base) / NSLOT;
    int2 *dst = ent + base + 2 * slot;
    auto at = [&](int t) { return dst + (t >> 1) * (2 * NSLOT) + (t & 1); };
    int cnt[M];
#pragma unroll
    for (int m = 0; m < M; ++m) cnt[m] = 0;
    for (int j = s + lane; j < e; j += 32) {
      const int r = (sell_row<M>(__ldg(idx + j)) - r0) & (M - 1);
#pragma unroll
      for (int m = 0; m < M; ++m) cnt[m] += r == m ? 1 : 0;
    }
#pragma unroll
    for (int m = 0; m < M; ++m)
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) cnt[m] += __shfl_xor_sync(0xffffffffu, cnt[m], off);
    int run[M];
#pragma unroll
    for (int m = 0; m < M; ++m) run[m] = 0;
    for (int b = s; b < e; b += 32) {
      const int j = b + lane;
      int k = 0, r = -1;
      float v = 0.f;
      if (j < e) {
        k = __ldg(idx + j);
        r = (sell_row<M>(k) - r0) & (M - 1);
        if (perm) {
          const int32_t src = __ldg(perm + j);
          v = (unsigned)src < (unsigned)nnz ? __ldg(val + src) : 0.f;
        } else {
          v = __ldg(val + j);
        }
      }
      int q = 0;
#pragma unroll
      for (int m = 0; m < M; ++m) {
        const unsigned bal = __ballot_sync(0xffffffffu, r == m);
        if (r == m) q = run[m] + __popc(bal & below);
        run[m] += __popc(bal);
      }
      if (j < e) {
        int t = 0;
#pragma unroll
        for (int m = 0; m < M; ++m) t += (cnt[m] < q ? cnt[m] : q) + (m < r && cnt[m] > q ? 1 : 0);
        const bool ok = (unsigned)k < (unsigned)W_in && t < steps;
        int vb;
        if constexpr (sizeof(Tin) == 2) vb = (int)pack_bf16x2(v, v);
        else vb = __float_as_int(v);
        if (t < steps) *at(t) = ok ? make_int2(sell_row<M>(k) * TT * (int)sizeof(Tin), vb) : make_int2(0, 0);
      }
    }
    for (int t = e - s + lane; t < steps; t += 32) *at(t) = make_int2(0, 0);  // none if e - s >= steps
  }
}

// acc[i] += v * row[i] for the G tokens a lane holds, v as stored in a sliced entry.
template <int G>
__device__ __forceinline__ void mac_sliced(const __nv_bfloat16 *row, int vbits, float *acc) {
  const uint32_t vv = (uint32_t)vbits;
  uint32_t w[G / 2];
  if constexpr (G == 8) {
    const uint4 t = *reinterpret_cast<const uint4 *>(row);
    w[0] = t.x, w[1] = t.y, w[2] = t.z, w[3] = t.w;
  } else {
    const uint2 t = *reinterpret_cast<const uint2 *>(row);
    w[0] = t.x, w[1] = t.y;
  }
#pragma unroll
  for (int i = 0; i < G / 2; ++i) {
    acc[2 * i] = fma_bf16_lo(w[i], vv, acc[2 * i]);
    acc[2 * i + 1] = fma_bf16_hi(w[i], vv, acc[2 * i + 1]);
  }
}
template <int G>
__device__ __forceinline__ void mac_sliced(const float *row, int vbits, float *acc) {
  mac_tokens<G>(row, __int_as_float(vbits), acc);
}

constexpr int kSellPairs = 4;  // step pairs per load batch (8 entries a slot)

// Output staging of the sliced kernel: the CTA's window of ws output columns
// for its TT tokens, fp32, row t at t * ws; a slot's two lanes (tokens t and
// t + 8) would meet the same bank, so rows with bit 3 of t set have their
// columns XORed with 16 (whole 16-byte chunks stay in place).
__device__ __forceinline__ int sell_out_col(int t, int c) { return c ^ (((t >> 3) & 1) << 4); }

template <typename Tin, typename Tout, int TT>
__global__ void __launch_bounds__(kSpmmThreads)
    sell_spmm_kernel(const Tin *__restrict__ in, int64_t T, int W_in, const int4 *__restrict__ ent,
                     const int32_t *__restrict__ sseg, const int32_t *__restrict__ goff, int n_grp, int n_seg,
                     int ws, float alpha, Tout *__restrict__ out) {
  static_assert(TT == 4 || TT == 8 || TT == 16, "token tile");
  constexpr int G = TT < 8 ? TT : 8;  // tokens per lane
  constexpr int Q = TT / G;           // lanes per slot
  constexpr int NSLOT = 32 / Q;
  constexpr int kWarps = kSpmmThreads / 32;
  constexpr int U = kSellPairs;
  constexpr int M = 128 / (TT * (int)sizeof(Tin));
  extern __shared__ __align__(16) unsigned char smem_raw[];
  Tin *s_in = reinterpret_cast<Tin *>(smem_raw);
  const size_t in_bytes = ((((size_t)W_in + M - 1) / M * M) * TT * sizeof(Tin) + 15) & ~(size_t)15;
  float *s_out = reinterpret_cast<float *>(smem_raw + in_bytes);
  const int64_t t0 = (int64_t)blockIdx.x * TT;
  const int w0 = (int)blockIdx.y * ws;  // this CTA's output columns [w0, w1)
  const int w1 = w0 + ws < n_seg ? w0 + ws : n_seg;
  const int g0 = w0 / NSLOT, g1 = (w1 + NSLOT - 1) / NSLOT;
  stage_sliced<Tin, TT, M>(in, T, W_in, t0, s_in);
  __syncthreads();
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int q = lane % Q, slot = lane / Q;
  const unsigned char *s_q = reinterpret_cast<const unsigned char *>(s_in) + (size_t)G * q * sizeof(Tin);
  // the window's groups (longest first) go to the warps in snake order (round j: warp w, then warp
  // kWarps - 1 - w), which evens out the warps' total steps
  for (int j = 0;; ++j) {
    const int local = (j & 1) ? kWarps - 1 - warp : warp;
    const int g = g0 + kWarps * j + local;
    if (g >= g1) break;
    const int base = goff[g];
    const int npair = (goff[g + 1] - base) / (2 * NSLOT);
    // pair i of this slot: ent[(base / 2) + i * NSLOT + slot] as (offset, value) x 2
    const int4 *e = ent + base / 2 + slot;
    float acc[G];
#pragma unroll
    for (int i = 0; i < G; ++i) acc[i] = 0.f;
    int4 cur[U], nxt[U];
#pragma unroll
    for (int u = 0; u < U; ++u) cur[u] = u < npair ? __ldg(e + (size_t)u * NSLOT) : make_int4(0, 0, 0, 0);
    for (int i0 = 0; i0 < npair; i0 += U) {
#pragma unroll
      for (int u = 0; u < U; ++u)
        nxt[u] = i0 + U + u < npair ? __ldg(e + (size_t)(i0 + U + u) * NSLOT) : make_int4(0, 0, 0, 0);
#pragma unroll
      for (int u = 0; u < U; ++u) {
        if (i0 + u >= npair) break;  // warp-uniform
        mac_sliced<G>(reinterpret_cast<const Tin *>(s_q + cur[u].x), cur[u].y, acc);
        mac_sliced<G>(reinterpret_cast<const Tin *>(s_q + cur[u].z), cur[u].w, acc);
      }
#pragma unroll
      for (int u = 0; u < U; ++u) cur[u] = nxt[u];
    }
    const int seg = sseg[(size_t)g * NSLOT + slot];
    if (seg >= w0 && seg < w1) {
      const int c = seg - w0;
#pragma unroll
      for (int i = 0; i < G; ++i) {
        const int t = G * q + i;
        s_out[t * ws + sell_out_col(t, c)] = alpha * acc[i];
      }
    }
  }
  __syncthreads();
  // the window's rows leave as 16-byte vectors (n_seg and ws are multiples of 8)
  const int nv = (w1 - w0) / 4;  // 4-column chunks per row
  for (int it = threadIdx.x; it < TT * nv; it += kSpmmThreads) {
    const int t = it / nv, c4 = it % nv;
    const int64_t tg = t0 + t;
    if (tg >= T) continue;
    const float4 v = *reinterpret_cast<const float4 *>(s_out + t * ws + sell_out_col(t, 4 * c4));
    Tout *o = out + tg * n_seg + w0 + 4 * c4;
    const float f[4] = {v.x, v.y, v.z, v.w};
    store_vec<Tout, 4>(o, f);
  }
}

// Output window of the sliced kernel: the largest power of two ws (>= 32, and
// not beyond n_seg rounded up to a power of two) whose fp32 staging for TT
// tokens fits in the shared memory left after the token tile; 0 if none.
template <typename Tin, int TT>
int sell_window(int W_in, int n_seg) {
  constexpr int M = 128 / (TT * (int)sizeof(Tin));
  const size_t in_bytes = ((((size_t)W_in + M - 1) / M * M) * TT * sizeof(Tin) + 15) & ~(size_t)15;
  if (in_bytes >= kSpmmSmemCap) return 0;
  const size_t room = (kSpmmSmemCap - in_bytes) / (TT * sizeof(float));
  int ws = 32;
  if ((size_t)ws > room) return 0;
  while ((size_t)ws * 2 <= room && ws < n_seg) ws *= 2;
  return ws;
}

template <typename Tin, typename Tout, int TT>
cudaError_t run_spmm_sliced(const void *in, int64_t T, int W_in, const int32_t *seg_ptr, const int32_t *idx,
                            const float *val, const int32_t *perm, int64_t nnz, int n_seg, float alpha,
                            void *scratch, int ws, void *out, cudaStream_t s) {
  constexpr int G = TT < 8 ? TT : 8;
  constexpr int NSLOT = 32 / (TT / G);
  constexpr int M = 128 / (TT * (int)sizeof(Tin));  // staged rows per bank line
  const SellLayout L = sell_layout(nnz, n_seg, W_in, NSLOT);
  char *base = static_cast<char *>(scratch);
  int2 *ent = reinterpret_cast<int2 *>(base + L.ent_off);
  int32_t *srank = reinterpret_cast<int32_t *>(base + L.srank_off);
  int32_t *sseg = reinterpret_cast<int32_t *>(base + L.sseg_off);
  int32_t *goff = reinterpret_cast<int32_t *>(base + L.goff_off);
  const int n_pad = L.n_grp * NSLOT;
  cudaError_t e = cudaMemsetAsync(srank, 0, (size_t)n_seg * 4, s);
  if (e != cudaSuccess) return e;
  sell_rank_kernel<<<dim3((unsigned)cdiv(n_seg, 256), (unsigned)cdiv(n_seg, kRankChunk)), 256, 0, s>>>(seg_ptr, n_seg,
                                                                                                      nnz, ws, srank);
  sell_place_kernel<<<(unsigned)cdiv(n_pad, 256), 256, 0, s>>>(srank, n_seg, n_pad, sseg);
  sell_offsets_kernel<<<1, 1024, 0, s>>>(seg_ptr, sseg, L.n_grp, nnz, NSLOT, W_in, goff);
  {
    const int64_t grid = std::min<int64_t>(cdiv(n_pad, 256 / 32), (int64_t)sm_count() * 8);
    sell_arrange_kernel<Tin, TT, M, NSLOT><<<(unsigned)grid, 256, 0, s>>>(seg_ptr, n_seg, idx, val, perm, nnz, W_in,
                                                                          srank, goff, ent);
  }
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  // rows rounded up to a whole block of M (sell_row may place a column of a partial last block past
  // W_in), then the output window
  const size_t smem = ((((size_t)W_in + M - 1) / M * M) * TT * sizeof(Tin) + 15 & ~(size_t)15) +
                      (size_t)TT * ws * sizeof(float);
  auto k = sell_spmm_kernel<Tin, Tout, TT>;
  static bool attr_done[64] = {};
  const int slot = device_slot();
  if (!attr_done[slot]) {
    e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSpmmSmemCap);
    if (e != cudaSuccess) return e;
    attr_done[slot] = true;
  }
  const dim3 grid((unsigned)cdiv(T, TT), (unsigned)cdiv(n_seg, ws));
  k<<<grid, kSpmmThreads, smem, s>>>(static_cast<const Tin *>(in), T, W_in, reinterpret_cast<const int4 *>(ent), sseg,
                                     goff, L.n_grp, n_seg, ws, alpha, static_cast<Tout *>(out));
  return cudaGetLastError();
}

template <typename Tin, typename Tout, int TT>
cudaError_t run_spmm(const void *in, int64_t T, int W_in, const int32_t *seg_ptr, const int32_t *idx,
                     const float *val, const int32_t *perm, int64_t nnz, int n_seg, float alpha, int2 *ent,
                     void *out, cudaStream_t s) {
  constexpr int M = 128 / (TT * (int)sizeof(Tin));  // staged rows per bank line
  {
    const int64_t grid = std::min<int64_t>(cdiv(n_seg, 256 / 32), (int64_t)sm_count() * 8);
    arrange_kernel<M><<<(unsigned)grid, 256, 0, s>>>(seg_ptr, n_seg, idx, val, perm, nnz, ent);
    const cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  const size_t smem = (((size_t)W_in * TT * sizeof(Tin) + ((size_t)n_seg + 1) * sizeof(int32_t) + 15) & ~(size_t)15) +
                      spmm_obuf_bytes<Tout>(TT);
  auto k = seg_spmm_kernel<Tin, Tout, TT>;
  cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  const int64_t tiles = cdiv(T, TT);
  // one CTA per SM: split the segments so that the token tiles fill whole waves
  const dim3 grid((unsigned)tiles, (unsigned)wave_split(tiles, n_seg >= 4 * kSpmmThreads / 32 ? 4 : 1));
  k<<<grid, kSpmmThreads, smem, s>>>(static_cast<const Tin *>(in), T, W_in, seg_ptr, ent, nnz, n_seg, alpha,
                                     static_cast<Tout *>(out));
  return cudaGetLastError();
}

bool sliced_ok(int64_t nnz, int n_seg, int W_in, int nslot, size_t scratch_bytes) {
  // 16-bit length and index fields of the rank keys
  return n_seg <= 65536 && W_in <= 65535 && nnz < ((int64_t)1 << 30) &&
         sell_layout(nnz, n_seg, W_in, nslot).total <= scratch_bytes;
}

template <typename Tin, typename Tout>
cudaError_t pick_spmm(const void *in, int64_t T, int W_in, const int32_t *seg_ptr, const int32_t *idx,
                      const float *val, const int32_t *perm, int64_t nnz, int n_seg, float alpha, void *scratch,
                      size_t scratch_bytes, void *out, cudaStream_t s, int *launched) {
  const size_t row = (size_t)W_in * sizeof(Tin);
  // the sliced kernel stages the token tile and an output window (5 kernels: rank, place, offsets,
  // arrange, product); the widest token tile with a window of at least 256 columns (or all of them)
  *launched = 5;
  auto fits = [&](int ws) { return ws >= 256 || (ws > 0 && ws >= n_seg); };
  if (const int ws = sell_window<Tin, 16>(W_in, n_seg); fits(ws) && sliced_ok(nnz, n_seg, W_in, 16, scratch_bytes))
    return run_spmm_sliced<Tin, Tout, 16>(in, T, W_in, seg_ptr, idx, val, perm, nnz, n_seg, alpha, scratch, ws, out,
                                          s);
  if (const int ws = sell_window<Tin, 8>(W_in, n_seg); fits(ws) && sliced_ok(nnz, n_seg, W_in, 32, scratch_bytes))
    return run_spmm_sliced<Tin, Tout, 8>(in, T, W_in, seg_ptr, idx, val, perm, nnz, n_seg, alpha, scratch, ws, out,
                                         s);
  if (const int ws = sell_window<Tin, 4>(W_in, n_seg); fits(ws) && sliced_ok(nnz, n_seg, W_in, 32, scratch_bytes))
    return run_spmm_sliced<Tin, Tout, 4>(in, T, W_in, seg_ptr, idx, val, perm, nnz, n_seg, alpha, scratch, ws, out,
                                         s);
  *launched = 2;  // arrange, product
  if (scratch_bytes < (size_t)(nnz > 0 ? nnz : 1) * 8) return cudaErrorInvalidValue;
  int2 *ent = static_cast<int2 *>(scratch);
  const size_t ptrs = ((size_t)n_seg + 1) * sizeof(int32_t) + 16;
  const size_t cap = kSpmmSmemCap > ptrs ? kSpmmSmemCap - ptrs : 0;
  if (row * 16 + spmm_obuf_bytes<Tout>(16) <= cap)
    return run_spmm<Tin, Tout, 16>(in, T, W_in, seg_ptr, idx, val, perm, nnz, n_seg, alpha, ent, out, s);
  if (row * 8 + spmm_obuf_bytes<Tout>(8) <= cap)
    return run_spmm<Tin, Tout, 8>(in, T, W_in, seg_ptr, idx, val, perm, nnz, n_seg, alpha, ent, out, s);
  if (row * 4 + spmm_obuf_bytes<Tout>(4) <= cap)
    return run_spmm<Tin, Tout, 4>(in, T, W_in, seg_ptr, idx, val, perm, nnz, n_seg, alpha, ent, out, s);
  return cudaErrorInvalidValue;  // rows too long for one staged token tile
}

// ---------------------------------------------------------------- SDDMM

constexpr int kSddmmThreads = 512;
constexpr int kSddmmTT = 32;                    // tokens per staged sub-tile
constexpr int kSddmmSlots = kSddmmThreads / 4;  // 4 lanes per slot, each two 16-byte chunks (8 tokens)
// shared memory: the fp32 dY and Z sub-tiles plus two raw staging buffers
template <typename T>
constexpr size_t sddmm_smem() {
  return 2ull * QWHA_TILE * kSddmmTT * sizeof(float) + 2 * (2ull * QWHA_TILE * kSddmmTT * sizeof(T));
}

// entries per slot and pass (the per-entry accumulators and offsets live in registers)
template <typename T>
__host__ __device__ constexpr int sddmm_entries() {
  return sizeof(T) == 2 ? 18 : 12;
}

// Staged sub-tiles are fp32 s[row][token], 32 tokens (128 B) per row; the
// 16-byte chunk c (tokens 4c .. 4c+3) of row r sits at chunk c ^ ((r & 3) << 1)
// (a permutation that keeps the chunk's parity). A staging write (a warp
// covers the 32 tokens of one row) is free of bank conflicts; so is a read:
// the 8 lanes of a quarter warp are two slots of 4 lanes, the even slot
// reads even chunks and the odd slot odd ones, so they meet 8 distinct chunk
// positions whatever their rows.
__device__ __forceinline__ int sdd_phys(int r, int t) {
  return r * kSddmmTT + ((((t >> 2) ^ ((r & 3) << 1)) << 2) | (t & 3));
}

// A sub-tile of dY and Z (32 tokens x QWHA_TILE rows each, as stored) is
// copied raw into a double-buffered staging area with cp.async (16-byte
// pieces; rows or tokens past the edge are zero-filled), then widened to fp32
// into the swizzled layout. A thread moves vectors of V consecutive rows at
// one token; the lanes of a warp take 32 consecutive tokens.
template <typename T>
struct SddStage {
  static constexpr int V = 16 / (int)sizeof(T);
  static constexpr int HALF = (QWHA_TILE / V) * kSddmmTT;  // vectors per operand
  static constexpr int ITEMS = 2 * HALF / kSddmmThreads;    // vectors per thread
  static constexpr size_t kRawBytes = 2ull * QWHA_TILE * kSddmmTT * sizeof(T);  // one buffer, both operands

  static __device__ __forceinline__ void copy(T *raw, const T *dY, const T *Z, int64_t tb, int d_out, int d_in,
                                              int64_t t0, int r0, int r_len, int k0, int k_len) {
#pragma unroll
    for (int u = 0; u < ITEMS; ++u) {
      const int it = threadIdx.x + u * kSddmmThreads;
      const int which = it >= HALF;
      const int w = it - which * HALF;
      const int t = w % kSddmmTT, c = w / kSddmmTT;
      const int64_t tg = t0 + t;
      const int len = which ? k_len : r_len;
      const bool in = tg < tb && c * V < len;
      const T *src = in ? (which ? Z + tg * d_in + k0 + c * V : dY + tg * d_out + r0 + c * V) : dY;
      const uint32_t dst = static_cast<uint32_t>(__cvta_generic_to_shared(raw + (size_t)it * V));
      asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(in ? 16 : 0)
                   : "memory");
    }
    asm volatile("cp.async.commit_group;" ::: "memory");
  }
  static __device__ __forceinline__ void widen(const T *raw, float *s_dy, float *s_z) {
#pragma unroll
    for (int u = 0; u < ITEMS; ++u) {
      const int it = threadIdx.x + u * kSddmmThreads;
      const int which = it >= HALF;
      const int w = it - which * HALF;
      const int t = w % kSddmmTT, c = w / kSddmmTT;
      float f[V];
      io<T>::unpack(*reinterpret_cast<const uint4 *>(raw + (size_t)it * V), f);
      float *dst = which ? s_z : s_dy;
#pragma unroll
      for (int i = 0; i < V; ++i) dst[sdd_phys(c * V + i, t)] = f[i];
    }
  }
};

__device__ __forceinline__ unsigned long long ffma2(unsigned long long a, unsigned long long b, unsigned long long c) {
  unsigned long long d;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
  return d;
}

// One CTA per (QWHA_TILE x QWHA_TILE tile of F, token chunk). A warp is 8
// slots of 4 lanes; lane q of a slot holds tokens 8q .. 8q+7 of the staged
// sub-tile (chunks 2q and 2q+1, whose swizzled offsets differ in bit 2).
// Slot s of the CTA owns E consecutive tile entries (CSC order inside the
// tile: mostly one column, whose Z chunks are reloaded only when it changes).
// Per entry and sub-tile a lane does two 16-byte shared loads of dY and four
// packed fp32x2 FMAs; at the end of the chunk the 4 lanes of a slot are summed
// by shuffles and the sum is written to the chunk's partial sums.
template <typename T>
__global__ void __launch_bounds__(kSddmmThreads, 1)
    sddmm_kernel(const T *__restrict__ dY, const T *__restrict__ Z, int64_t T_, int d_out, int d_in,
                 const int32_t *__restrict__ tile_ptr, const int32_t *__restrict__ tile_pos,
                 const int32_t *__restrict__ tile_rk, int n_rb, int64_t chunk_tokens, int64_t p,
                 float *__restrict__ partial) {
  constexpr int E = sddmm_entries<T>();
  constexpr int kPass = kSddmmSlots * E;
  extern __shared__ __align__(16) float sdd_smem[];
  float *s_dy = sdd_smem;
  float *s_z = sdd_smem + QWHA_TILE * kSddmmTT;
  T *raw = reinterpret_cast<T *>(sdd_smem + 2 * QWHA_TILE * kSddmmTT);  // two staging buffers
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
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int q = lane & 3, slot = warp * 8 + (lane >> 2);

  for (int64_t eb = e_begin; eb < e_end; eb += kPass) {
    const int64_t my0 = eb + (int64_t)slot * E;
    // per entry, fixed over the token range: the shared offsets of this lane's
    // dY and Z chunks (dY high half, Z low half; an unused entry reads row 0
    // and is not stored), whether its column differs from the previous one's,
    // and whether it is in use
    uint32_t off[E];
    uint32_t newcol = 0, valid = 0;
    float acc[E];
#pragma unroll
    for (int i = 0; i < E; ++i) {
      const int64_t e = my0 + i;
      const int v = e < e_end ? tile_rk[e] : -1;
      const int r_ = (v >> 16) & 0xffff, k_ = v & 0xffff;
      const bool ok = e < e_end && v >= 0 && r_ < r_len && k_ < k_len;
      const int rr = ok ? r_ : 0, kk = ok ? k_ : 0;
      // this lane's tokens 8q .. 8q+7 are chunks 2q and 2q+1; it starts with the one of its slot's parity
      const int t_first = 8 * q + 4 * (slot & 1);
      off[i] = ((uint32_t)sdd_phys(rr, t_first) << 16) | (uint32_t)sdd_phys(kk, t_first);
      if (i == 0 || (off[i] & 0xffffu) != (off[i - 1] & 0xffffu)) newcol |= 1u << i;
      if (ok) valid |= 1u << i;
      acc[i] = 0.f;
    }
    using St = SddStage<T>;
    if (ta < tb) St::copy(raw, dY, Z, tb, d_out, d_in, ta, r0, r_len, k0, k_len);
    int buf = 0;
    for (int64_t t0 = ta; t0 < tb; t0 += kSddmmTT, buf ^= 1) {
      asm volatile("cp.async.wait_all;" ::: "memory");
      __syncthreads();  // this sub-tile is staged; the previous one is consumed
      St::widen(raw + buf * (St::kRawBytes / sizeof(T)), s_dy, s_z);
      __syncthreads();
      if (t0 + kSddmmTT < tb)  // the other buffer was widened one iteration ago
        St::copy(raw + (buf ^ 1) * (St::kRawBytes / sizeof(T)), dY, Z, tb, d_out, d_in, t0 + kSddmmTT, r0, r_len,
                 k0, k_len);
      ulonglong2 z0 = make_ulonglong2(0ull, 0ull), z1 = z0;
#pragma unroll
      for (int i = 0; i < E; ++i) {
        if (newcol & (1u << i)) {
          const uint32_t oz = off[i] & 0xffffu;
          z0 = *reinterpret_cast<const ulonglong2 *>(s_z + oz);
          z1 = *reinterpret_cast<const ulonglong2 *>(s_z + (oz ^ 4u));
        }
        const uint32_t oy = off[i] >> 16;
        const ulonglong2 y0 = *reinterpret_cast<const ulonglong2 *>(s_dy + oy);
        const ulonglong2 y1 = *reinterpret_cast<const ulonglong2 *>(s_dy + (oy ^ 4u));
        unsigned long long t2 = ffma2(y0.x, z0.x, 0ull);
        t2 = ffma2(y0.y, z0.y, t2);
        t2 = ffma2(y1.x, z1.x, t2);
        t2 = ffma2(y1.y, z1.y, t2);
        acc[i] += __uint_as_float((uint32_t)t2) + __uint_as_float((uint32_t)(t2 >> 32));
      }
    }
#pragma unroll
    for (int i = 0; i < E; ++i) {
      float s = acc[i];
      s += __shfl_xor_sync(0xffffffffu, s, 1);
      s += __shfl_xor_sync(0xffffffffu, s, 2);
      if (q == 0 && (valid & (1u << i))) {
        const int j = tile_pos[my0 + i];
        if ((uint64_t)j < (uint64_t)p) part[j] = s;
      }
    }
    __syncthreads();
  }
}

// ---------------------------------------------------------------- SDDMM, bf16 activations
//
// The bf16 path keeps the staged sub-tiles in bf16: 64 tokens (128 B) per row
// of s[row][token], half the shared bytes per product of a widened fp32 tile,
// and multiplies with fma.rn.f32.bf16 (bf16 x bf16 -> fp32 accumulate; the
// product of two bf16 values is exact in fp32, so only the summation order
// differs from the fp32 kernel). The 16-byte chunk c (tokens 8c .. 8c+7) of
// row r sits at chunk position c ^ ((r & 3) << 1), which keeps the chunk's
// parity. Lane q of a slot holds tokens 16q .. 16q+15 (chunks 2q, 2q+1) and
// reads the chunk of its slot's parity first: the two slots of a quarter warp
// then meet 8 distinct chunk positions whatever their rows, and so do their
// second reads. Staging: cp.async copies the sub-tile raw (16-byte pieces,
// [operand][row chunk][token], zero-filled past the edges); once it has landed
// every thread transposes its pieces into the swizzled layout (a warp writes
// 64 contiguous bytes of one row per store), and the copy of the next
// sub-tile is issued into the raw buffer while this one is multiplied.
constexpr int kSdd16TT = 64;  // tokens per staged sub-tile (bf16)
constexpr int kSdd16E = 18;   // entries per slot and pass

constexpr size_t sddmm16_smem() {
  return 2ull * QWHA_TILE * kSdd16TT * 2 /* transposed dY, Z */ + 2ull * QWHA_TILE * kSdd16TT * 2 /* raw */;
}

// byte offset of (row r, token t) in a transposed operand
__device__ __forceinline__ uint32_t sdd16_off(int r, int t) {
  return (uint32_t)r * (kSdd16TT * 2) + ((uint32_t)((t >> 3) ^ ((r & 3) << 1)) << 4) + (uint32_t)(t & 7) * 2;
}

__device__ __forceinline__ float dot8_bf16(const uint4 y, const uint4 z, float acc) {
  acc = fma_bf16_lo(y.x, z.x, acc);
  acc = fma_bf16_hi(y.x, z.x, acc);
  acc = fma_bf16_lo(y.y, z.y, acc);
  acc = fma_bf16_hi(y.y, z.y, acc);
  acc = fma_bf16_lo(y.z, z.z, acc);
  acc = fma_bf16_hi(y.z, z.z, acc);
  acc = fma_bf16_lo(y.w, z.w, acc);
  acc = fma_bf16_hi(y.w, z.w, acc);
  return acc;
}

// The per-slot part of the bf16 coefficient gradient, shared by both kernels
// below so that they do the same arithmetic in the same order. A slot (4
// lanes, lane q) owns E consecutive entries of the tile from my0 on and
// multiplies them over every staged 64-token sub-tile.
struct Sdd16Slot {
  uint32_t off[kSdd16E];  // byte offsets of the lane's first dY chunk (high half) and Z chunk (low half)
  uint32_t newcol = 0;    // bit i: entry i's column differs from entry i-1's
  uint32_t valid = 0;     // bit i: entry i exists
  float acc[kSdd16E];

  // per entry, fixed over the token range (an unused entry reads row 0 and is not stored)
  __device__ __forceinline__ void setup(const int32_t *__restrict__ tile_rk, int64_t my0, int64_t e_end, int r_len,
                                        int k_len, int q, int par) {
    newcol = 0;
    valid = 0;
#pragma unroll
    for (int i = 0; i < kSdd16E; ++i) {
      const int64_t e = my0 + i;
      const int v = e < e_end ? tile_rk[e] : -1;
      const int r_ = (v >> 16) & 0xffff, k_ = v & 0xffff;
      const bool ok = e < e_end && v >= 0 && r_ < r_len && k_ < k_len;
      const int rr = ok ? r_ : 0, kk = ok ? k_ : 0;
      const int t_first = 16 * q + 8 * par;
      off[i] = (sdd16_off(rr, t_first) << 16) | sdd16_off(kk, t_first);
      if (i == 0 || (off[i] & 0xffffu) != (off[i - 1] & 0xffffu)) newcol |= 1u << i;
      if (ok) valid |= 1u << i;
      acc[i] = 0.f;
    }
  }
  // one staged sub-tile: s_dy and s_z hold QWHA_TILE rows of 64 tokens each (layout sdd16_off)
  __device__ __forceinline__ void mac(const unsigned char *s_dy, const unsigned char *s_z) {
    uint4 z0 = make_uint4(0, 0, 0, 0), z1 = z0;
#pragma unroll
    for (int i = 0; i < kSdd16E; ++i) {
      if (newcol & (1u << i)) {
        const uint32_t oz = off[i] & 0xffffu;
        z0 = *reinterpret_cast<const uint4 *>(s_z + oz);
        z1 = *reinterpret_cast<const uint4 *>(s_z + (oz ^ 16u));  // the lane's other chunk: parity flipped
      }
      const uint32_t oy = off[i] >> 16;
      const uint4 y0 = *reinterpret_cast<const uint4 *>(s_dy + oy);
      const uint4 y1 = *reinterpret_cast<const uint4 *>(s_dy + (oy ^ 16u));
      acc[i] = dot8_bf16(y1, z1, dot8_bf16(y0, z0, acc[i]));
    }
  }
  __device__ __forceinline__ void store(const int32_t *__restrict__ tile_pos, int64_t my0, int64_t p, int q,
                                        float *__restrict__ part) {
#pragma unroll
    for (int i = 0; i < kSdd16E; ++i) {
      float sum = acc[i];
      sum += __shfl_xor_sync(0xffffffffu, sum, 1);
      sum += __shfl_xor_sync(0xffffffffu, sum, 2);
      if (q == 0 && (valid & (1u << i))) {
        const int j = tile_pos[my0 + i];
        if ((uint64_t)j < (uint64_t)p) part[j] = sum;
      }
    }
  }
};

__global__ void __launch_bounds__(kSddmmThreads, 1)
    sddmm_bf16_kernel(const __nv_bfloat16 *__restrict__ dY, const __nv_bfloat16 *__restrict__ Z, int64_t T_,
                      int d_out, int d_in, const int32_t *__restrict__ tile_ptr, const int32_t *__restrict__ tile_pos,
                      const int32_t *__restrict__ tile_rk, int n_rb, int64_t chunk_tokens, int64_t p,
                      float *__restrict__ partial) {
  constexpr int E = kSdd16E;
  constexpr int kPass = kSddmmSlots * E;
  constexpr int kRowBytes = kSdd16TT * 2;
  constexpr int kOpBytes = QWHA_TILE * kRowBytes;      // one transposed operand
  constexpr int kPieces = QWHA_TILE / 8 * kSdd16TT;    // 16-byte raw pieces per operand
  constexpr int kItems = 2 * kPieces / kSddmmThreads;  // pieces per thread and sub-tile
  extern __shared__ __align__(16) unsigned char sdd16_smem[];
  unsigned char *s_dy = sdd16_smem;
  unsigned char *s_z = sdd16_smem + kOpBytes;
  uint4 *raw = reinterpret_cast<uint4 *>(sdd16_smem + 2 * kOpBytes);  // [operand][row chunk][token]
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
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int q = lane & 3, slot = warp * 8 + (lane >> 2);
  const int par = slot & 1;

  // Raw piece position p = operand * kPieces + ch * 64 + (t & 1) * 32 + t / 2: the two pieces of the
  // token pair (t, t + 1) sit 32 pieces apart, so both the copy's writes (consecutive threads,
  // consecutive positions) and the transpose's reads (consecutive threads, consecutive pairs) cover
  // contiguous 16-byte pieces.
  auto copy = [&](int64_t t0) {
#pragma unroll 2
    for (int u = 0; u < kItems; ++u) {
      const int it = threadIdx.x + u * kSddmmThreads;
      const int which = it >= kPieces;
      const int w = it - which * kPieces;
      const int r = w % kSdd16TT, ch = w / kSdd16TT;
      const int t = 2 * (r & 31) + (r >> 5);
      const int64_t tg = t0 + t;
      const int len = which ? k_len : r_len;
      const bool in = tg < tb && ch * 8 < len;
      const __nv_bfloat16 *src = in ? (which ? Z + tg * d_in + k0 + ch * 8 : dY + tg * d_out + r0 + ch * 8) : dY;
      const uint32_t dst = static_cast<uint32_t>(__cvta_generic_to_shared(raw + it));
      asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(in ? 16 : 0)
                   : "memory");
    }
    asm volatile("cp.async.commit_group;" ::: "memory");
  };
  // Each thread takes the pieces of two adjacent tokens (same rows) and writes, per row, the two
  // tokens as one 4-byte word: a warp's store then fills one whole 128-byte row.
  auto transpose = [&]() {
#pragma unroll
    for (int u = 0; u < kItems / 2; ++u) {
      const int pi = threadIdx.x + u * kSddmmThreads;  // token pair
      const int which = pi >= kPieces / 2;
      const int w = pi - which * (kPieces / 2);
      const int tp = w % (kSdd16TT / 2), ch = w / (kSdd16TT / 2);
      const int t = 2 * tp;
      const int at = which * kPieces + ch * kSdd16TT + tp;
      const uint4 a = raw[at], b = raw[at + kSdd16TT / 2];
      unsigned char *dst = which ? s_z : s_dy;
      const uint32_t wa[4] = {a.x, a.y, a.z, a.w}, wb[4] = {b.x, b.y, b.z, b.w};
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        *reinterpret_cast<uint32_t *>(dst + sdd16_off(ch * 8 + 2 * i, t)) = __byte_perm(wa[i], wb[i], 0x5410);
        *reinterpret_cast<uint32_t *>(dst + sdd16_off(ch * 8 + 2 * i + 1, t)) = __byte_perm(wa[i], wb[i], 0x7632);
      }
    }
  };

  for (int64_t eb = e_begin; eb < e_end; eb += kPass) {
    const int64_t my0 = eb + (int64_t)slot * E;
    Sdd16Slot sl;
    sl.setup(tile_rk, my0, e_end, r_len, k_len, q, par);
    if (ta < tb) copy(ta);
    for (int64_t t0 = ta; t0 < tb; t0 += kSdd16TT) {
      asm volatile("cp.async.wait_all;" ::: "memory");
      __syncthreads();  // this sub-tile's raw pieces have landed; the previous one is multiplied
      transpose();
      __syncthreads();
      if (t0 + kSdd16TT < tb) copy(t0 + kSdd16TT);  // the raw buffer is free again
      sl.mac(s_dy, s_z);
    }
    sl.store(tile_pos, my0, p, q, part);
    __syncthreads();
  }
}

// dY and Z transposed once for the whole gradient: out[f, t] = in[t, f] for
// f < d and t < ld (ld = T rounded up to 64; zeros past T), with the 16-byte
// chunks of every 64-token block of a row f permuted as sdd16_off permutes
// them in shared memory (chunk j at j ^ ((f & 3) << 1)). A plain 2-D tensor
// copy of QWHA_TILE rows x 64 tokens then lands exactly in the layout the
// gradient kernel reads. One CTA transposes 64 tokens x 64 features through
// shared memory: each thread packs the same feature of two adjacent tokens
// into one word, and word slots are XOR-swizzled so that both the writes and
// the 16-byte reads of the exchange are free of bank conflicts. Requires
// d % 8 == 0 and 16-byte aligned rows.
__device__ __forceinline__ int sdd_xpose_swz(int c) { return 4 * ((c + (c >> 3)) & 7); }

__global__ void __launch_bounds__(256) sdd_transpose_kernel(const __nv_bfloat16 *__restrict__ in, int64_t T_, int d,
                                                            int64_t ld, __nv_bfloat16 *__restrict__ out) {
  __shared__ __align__(16) uint32_t sw[64 * 32];  // [feature][token pair], 128 B a feature
  const int64_t t0 = (int64_t)blockIdx.x * 64;
  const int f0 = blockIdx.y * 64;
  const int tid = threadIdx.x;
  {
    const int tp = tid >> 3, ch = tid & 7;
    const int64_t t = t0 + 2 * tp;
    const int f = f0 + 8 * ch;
    uint4 a = make_uint4(0, 0, 0, 0), b = a;
    if (f < d) {  // d % 8 == 0: the 8 features are all in range
      if (t < T_) a = ld_stream(in + t * d + f);
      if (t + 1 < T_) b = ld_stream(in + (t + 1) * d + f);
    }
    const uint32_t wa[4] = {a.x, a.y, a.z, a.w}, wb[4] = {b.x, b.y, b.z, b.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int c = 8 * ch + 2 * i;
      sw[c * 32 + (tp ^ sdd_xpose_swz(c))] = __byte_perm(wa[i], wb[i], 0x5410);
      sw[(c + 1) * 32 + (tp ^ sdd_xpose_swz(c + 1))] = __byte_perm(wa[i], wb[i], 0x7632);
    }
  }
  __syncthreads();
  const int c = tid >> 2, g = tid & 3;
  const int f = f0 + c;
  if (f < d) {
    const int z = sdd_xpose_swz(c);
    const uint4 lo = *reinterpret_cast<const uint4 *>(sw + c * 32 + ((8 * g) ^ z));
    const uint4 hi = *reinterpret_cast<const uint4 *>(sw + c * 32 + ((8 * g + 4) ^ z));
    const int pos = (2 * g) ^ ((f & 3) << 1);  // even: the chunk pair stays adjacent
    __nv_bfloat16 *o = out + (int64_t)f * ld + t0 + 8 * pos;
    st_stream(o, lo);
    st_stream(o + 8, hi);
  }
}

constexpr int kSddTStages = 3;  // sub-tiles in flight per CTA
constexpr int kSddTOpBytes = QWHA_TILE * kSdd16TT * 2;
constexpr size_t sddmm_t_smem() { return (size_t)kSddTStages * 2 * kSddTOpBytes + 1024 + kSddTStages * 8; }

__device__ __forceinline__ void sdd_tma_load(uint32_t dst, const CUtensorMap *map, uint32_t bar, int x, int y) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4}], [%2];" ::"r"(
          dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(bar), "r"(x), "r"(y)
      : "memory");
}

// The bf16 gradient fed by tensor copies of the transposed operands (layout of
// sdd_transpose_kernel): the CTA's sub-tiles (dY rows of its row block and Z
// rows of its column block, 64 tokens each) stream through a ring of
// kSddTStages slots that one thread refills, one CTA barrier per sub-tile.
// Same tile, chunk, pass and slot structure, and the same Sdd16Slot
// arithmetic, as sddmm_bf16_kernel. Every wait is bounded; on a timeout the
// CTA records 0x800 in the error word, lets the copies it issued land and
// exits.
__global__ void __launch_bounds__(kSddmmThreads, 1)
    sddmm_t_kernel(const __grid_constant__ CUtensorMap tmY, const __grid_constant__ CUtensorMap tmZ, int64_t T_,
                   int d_out, int d_in, const int32_t *__restrict__ tile_ptr, const int32_t *__restrict__ tile_pos,
                   const int32_t *__restrict__ tile_rk, int n_rb, int64_t chunk_tokens, int64_t p,
                   float *__restrict__ partial, unsigned int *err) {
  constexpr int E = kSdd16E;
  constexpr int kPass = kSddmmSlots * E;
  constexpr int S = kSddTStages;
  extern __shared__ unsigned char sddt_smem[];
  unsigned char *ring = reinterpret_cast<unsigned char *>((reinterpret_cast<uintptr_t>(sddt_smem) + 1023) & ~uintptr_t(1023));
  uint64_t *full = reinterpret_cast<uint64_t *>(ring + S * 2 * kSddTOpBytes);
  const int tile = blockIdx.x;
  const int rb = tile % n_rb, kb = tile / n_rb;
  const int r0 = rb * QWHA_TILE, k0 = kb * QWHA_TILE;
  const int r_len = min(QWHA_TILE, d_out - r0), k_len = min(QWHA_TILE, d_in - k0);
  int64_t e_begin = tile_ptr[tile], e_end = tile_ptr[tile + 1];
  if (e_begin < 0) e_begin = 0;
  if (e_end > p) e_end = p;
  const int64_t c = blockIdx.y;
  const int64_t ta = c * chunk_tokens, tb = (ta + chunk_tokens < T_) ? ta + chunk_tokens : T_;
  const int64_t n_sub = ta < tb ? (tb - ta + kSdd16TT - 1) / kSdd16TT : 0;
  const int64_t n_pass = e_end > e_begin ? (e_end - e_begin + kPass - 1) / kPass : 0;
  const int64_t total = n_sub * n_pass;  // ring steps
  if (total == 0) return;                // the same for every thread of the CTA
  float *part = partial + c * p;
  const int tid = threadIdx.x;
  const int lane = tid & 31, warp = tid >> 5;
  const int q = lane & 3, slot = warp * 8 + (lane >> 2);
  const int par = slot & 1;

  auto issue = [&](int64_t g) {  // thread 0: sub-tile g % n_sub into slot g % S
    const int s = (int)(g % S);
    const int x = (int)(ta + (g % n_sub) * kSdd16TT);
    const uint32_t bar = bulk::saddr(full + s);
    const uint32_t dst = bulk::saddr(ring + s * 2 * kSddTOpBytes);
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(2 * kSddTOpBytes)
                 : "memory");
    sdd_tma_load(dst, &tmY, bar, x, r0);
    sdd_tma_load(dst + kSddTOpBytes, &tmZ, bar, x, k0);
  };
  if (tid == 0) {
#pragma unroll
    for (int s = 0; s < S; ++s) bulk::init(bulk::saddr(full + s), 1);
    bulk::fence_init();
  }
  __syncthreads();
  if (tid == 0)
    for (int64_t g = 0; g < S && g < total; ++g) issue(g);

  int64_t g = 0;
  for (int64_t pass = 0; pass < n_pass; ++pass) {
    const int64_t my0 = e_begin + pass * kPass + (int64_t)slot * E;
    Sdd16Slot sl;
    sl.setup(tile_rk, my0, e_end, r_len, k_len, q, par);
    for (int64_t sub = 0; sub < n_sub; ++sub, ++g) {
      const int s = (int)(g % S);
      const bool ok = bulk::wait(bulk::saddr(full + s), (uint32_t)((g / S) & 1));
      // also: every thread has finished step g - 1, so its slot can be refilled
      if (__syncthreads_or(!ok)) {
        if (tid == 0) {
          atomicOr(err, 0x800u);
          // issued and not yet consumed: steps g .. S - 1 at the first step, else g .. g + S - 2
          const int64_t last = g == 0 ? S : g + S - 1;
          for (int64_t j = g; j < total && j < last; ++j)
            (void)bulk::wait(bulk::saddr(full + (int)(j % S)), (uint32_t)((j / S) & 1));
        }
        return;
      }
      if (tid == 0 && g >= 1 && g - 1 + S < total) {
        bulk::fence_proxy();
        issue(g - 1 + S);
      }
      const unsigned char *st = ring + s * 2 * kSddTOpBytes;
      sl.mac(st, st + kSddTOpBytes);
    }
    sl.store(tile_pos, my0, p, q, part);
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

size_t spmm_scratch_bytes(int64_t p, int n_seg, int W_in) {
  const size_t a = sell_layout(p, n_seg, W_in, 16).total, b = sell_layout(p, n_seg, W_in, 32).total;
  const size_t c = align_up((size_t)(p > 0 ? p : 1) * 8, 256);
  return std::max(std::max(a, b), c);
}

cudaError_t launch_seg_spmm(qwha_dtype din, qwha_dtype dout, const void *in, int64_t T, int W_in,
                            const int32_t *seg_ptr, const int32_t *idx, const float *val, const int32_t *perm,
                            int64_t nnz, int n_seg, float alpha, void *scratch, size_t scratch_bytes, void *out,
                            cudaStream_t s, int *launched) {
  int dummy = 0;
  int *nk = launched ? launched : &dummy;
  *nk = 0;
  if (T <= 0 || n_seg <= 0) return cudaSuccess;
  if (reinterpret_cast<uintptr_t>(scratch) & 255) return cudaErrorMisalignedAddress;
  using bf = __nv_bfloat16;
  if (din == QWHA_BF16) {
    if (dout == QWHA_BF16)
      return pick_spmm<bf, bf>(in, T, W_in, seg_ptr, idx, val, perm, nnz, n_seg, alpha, scratch, scratch_bytes, out, s,
                               nk);
    return pick_spmm<bf, float>(in, T, W_in, seg_ptr, idx, val, perm, nnz, n_seg, alpha, scratch, scratch_bytes, out,
                                s, nk);
  }
  if (dout == QWHA_BF16)
    return pick_spmm<float, bf>(in, T, W_in, seg_ptr, idx, val, perm, nnz, n_seg, alpha, scratch, scratch_bytes, out,
                                s, nk);
  return pick_spmm<float, float>(in, T, W_in, seg_ptr, idx, val, perm, nnz, n_seg, alpha, scratch, scratch_bytes, out,
                                 s, nk);
}

int sddmm_chunks(int64_t T, int32_t d_out, int32_t d_in) {
  // at least two waves of CTAs (one per SM), the last one nearly full
  const int64_t tiles = cdiv(d_out, QWHA_TILE) * cdiv(d_in, QWHA_TILE);
  const int64_t max_by_tokens = cdiv(T, 32);
  int64_t cap = kSddmmMaxChunks < max_by_tokens ? kSddmmMaxChunks : max_by_tokens;
  if (cap < 1) cap = 1;
  int64_t lo = cdiv(2 * (int64_t)sm_count(), tiles);
  if (lo > cap) lo = cap;
  if (lo < 1) lo = 1;
  int64_t want = lo;
  double best = -1.0;
  for (int64_t c = lo; c <= cap; ++c) {
    const int64_t n = tiles * c, slots = sm_count();
    const double eff = (double)n / (double)(cdiv(n, slots) * slots);
    if (eff >= 0.95) {
      want = c;
      break;
    }
    if (eff > best + 1e-9) {
      best = eff;
      want = c;
    }
  }
  return (int)want;
}

size_t sddmm_transposed_bytes(int64_t T, int32_t d_out, int32_t d_in) {
  const int64_t ld = cdiv(T > 0 ? T : 1, kSdd16TT) * kSdd16TT;
  return align_up((size_t)d_out * ld * 2, 256) + align_up((size_t)d_in * ld * 2, 256);
}

cudaError_t launch_sddmm(qwha_dtype dt, const void *dY, const void *Z, int64_t T, int32_t d_out, int32_t d_in,
                         const int32_t *tile_ptr, const int32_t *tile_pos, const int32_t *tile_rk, int64_t p,
                         float alpha, float *partial, float *dc, cudaStream_t s, void *tscratch, int *launched) {
  int dummy = 0;
  int *nk = launched ? launched : &dummy;
  *nk = 0;
  if (p <= 0) return cudaSuccess;
  const int n_rb = (int)cdiv(d_out, QWHA_TILE);
  const int64_t tiles = n_rb * cdiv(d_in, QWHA_TILE);
  const int n_chunks = sddmm_chunks(T, d_out, d_in);
  const int64_t chunk_tokens = cdiv(cdiv(T, n_chunks), 64) * 64;
  cudaError_t e = cudaMemsetAsync(partial, 0, (size_t)n_chunks * p * sizeof(float), s);
  if (e != cudaSuccess) return e;
  if (T > 0) {
    dim3 grid((unsigned)tiles, (unsigned)n_chunks);
    const int64_t ld = cdiv(T, kSdd16TT) * kSdd16TT;
    __nv_bfloat16 *yt = static_cast<__nv_bfloat16 *>(tscratch);
    __nv_bfloat16 *zt = yt ? yt + align_up((size_t)d_out * ld * 2, 256) / 2 : nullptr;
    CUtensorMap tmY, tmZ;
    const bool transposed = dt == QWHA_BF16 && yt && aligned16(yt) && d_out % 8 == 0 && d_in % 8 == 0 &&
                            aligned16(dY) && aligned16(Z) && ld / kSdd16TT <= 0x7fffffff &&
                            make_map_rows(&tmY, yt, d_out, ld, ld, kSdd16TT, QWHA_TILE) &&
                            make_map_rows(&tmZ, zt, d_in, ld, ld, kSdd16TT, QWHA_TILE);
    if (transposed) {
      const dim3 gy((unsigned)(ld / 64), (unsigned)cdiv(d_out, 64)), gz((unsigned)(ld / 64), (unsigned)cdiv(d_in, 64));
      sdd_transpose_kernel<<<gy, 256, 0, s>>>(static_cast<const __nv_bfloat16 *>(dY), T, d_out, ld, yt);
      sdd_transpose_kernel<<<gz, 256, 0, s>>>(static_cast<const __nv_bfloat16 *>(Z), T, d_in, ld, zt);
      e = cudaGetLastError();
      if (e != cudaSuccess) return e;
      const size_t smem = sddmm_t_smem();
      static bool attr_done[64] = {};
      const int slot = device_slot();
      if (!attr_done[slot]) {
        e = cudaFuncSetAttribute(sddmm_t_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
        attr_done[slot] = true;
      }
      sddmm_t_kernel<<<grid, kSddmmThreads, smem, s>>>(tmY, tmZ, T, d_out, d_in, tile_ptr, tile_pos, tile_rk, n_rb,
                                                        chunk_tokens, p, partial, device_error_word());
      *nk += 3;
    } else {
      const size_t smem = dt == QWHA_BF16 ? sddmm16_smem() : sddmm_smem<float>();
      e = cudaFuncSetAttribute(dt == QWHA_BF16 ? (const void *)sddmm_bf16_kernel : (const void *)sddmm_kernel<float>,
                               cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
      if (e != cudaSuccess) return e;
      if (dt == QWHA_BF16)
        sddmm_bf16_kernel<<<grid, kSddmmThreads, smem, s>>>(
            static_cast<const __nv_bfloat16 *>(dY), static_cast<const __nv_bfloat16 *>(Z), T, d_out, d_in, tile_ptr,
            tile_pos, tile_rk, n_rb, chunk_tokens, p, partial);
      else
        sddmm_kernel<float><<<grid, kSddmmThreads, smem, s>>>(static_cast<const float *>(dY),
                                                           static_cast<const float *>(Z), T, d_out, d_in, tile_ptr,
                                                           tile_pos, tile_rk, n_rb, chunk_tokens, p, partial);
      *nk += 1;
    }
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  sddmm_reduce_kernel<<<(unsigned)std::min<int64_t>(cdiv(p, 256), (int64_t)sm_count() * 8), 256, 0, s>>>(partial, n_chunks, p,
                                                                                         alpha, dc);
  *nk += 1;
  return cudaGetLastError();
}

}  // namespace qwha
