// Dense contractions of the adapted layer on the 5th-generation tensor cores:
//   out[M, N] = A[M, K] . B[N, K]^T (+ addend[M, N]), out bf16 or fp32
// with A, B bf16 K-major (row-major with K contiguous) and addend fp32.
//   forward:  Y  = X W_Q^T + Y_adapter   (A = X, B = W_Q, K = d_in)
//   backward: dX = dY W_Q + dX_adapter   (A = dY, B = W_Q read MN-major, K = d_out)
// The adapter term rides in the epilogue, so it costs one fp32 read.
//
// Structure (persistent; one CTA per SM, or one CTA pair per two SMs):
//   warp 0, one thread : TMA producer. Tensor copies (128B swizzle, no
//                        multicast) of A and B k-blocks of 64 into a shared-
//                        memory ring, completion counted in bytes on the
//                        stage's "full" mbarrier. An operand may be K-major
//                        (one 2-D box of rows x 64 K) or MN-major: one 3-D
//                        box that fills the stage's 64 x 64 slabs along MN
//                        at once (the operand seen as 64 MN elements x K x
//                        MN / 64 slabs), or, when MN is not a multiple of
//                        64, one 2-D box per slab. Fewer, larger copies keep
//                        the tensor pipe fed: the measured cost of an
//                        MN-major operand fell from ~10% to nothing. The
//                        UMMA descriptors and the instruction descriptor's
//                        major bits follow the layout.
//   warp 1, one thread : MMA issuer. tcgen05.mma kind::f16 (bf16 x bf16 ->
//                        fp32), K=16 per instruction, accumulator in TMEM;
//                        tcgen05.commit frees the stage ("empty") and, after
//                        the tile's last k-block, publishes the accumulator.
//                        Warp 1 also owns the TMEM allocation (512 columns:
//                        two accumulators, so the epilogue of tile i overlaps
//                        the main loop of tile i+1).
//   warps 2..5         : epilogue. tcgen05.ld 32 lanes x 32 columns at a
//                        time (warp w reads TMEM lanes 32*(w%4)..+31), add
//                        the fp32 addend (if any), store bf16 or fp32.
// Two variants of the same kernel:
//   CG = 1: one CTA computes a 128 x 256 tile (M = 128 MMA), 48 KB per stage,
//           4 stages.
//   CG = 2: a cluster of two CTAs on two SMs computes a 256 x 256 tile with
//           cta_group::2 MMAs (M = 256) issued by the even CTA. Each CTA loads
//           its own 128 rows of A and its own 128 rows (half) of B, 32 KB per
//           stage, 6 stages; both CTAs' copies complete on the even CTA's
//           "full" barrier, the MMA commits arrive on the barriers of both
//           CTAs (stage free, accumulator ready), and the odd CTA's epilogue
//           reports a drained accumulator on the even CTA's barrier. Every SM
//           then streams 2/3 of the operand bytes of the CG = 1 tile for the
//           same MMA work.
// Every mbarrier wait is bounded by time: on expiry the thread records a code
// in the library's device error word, the CTA stops issuing work, drains what
// it issued, frees TMEM and exits.

#include <cuda.h>

#include <cmath>

#include "common.cuh"
#include "fwht_body.cuh"
#include "kernels.h"

namespace qwha {
namespace {

constexpr int BM = 128, BN = 256;  // accumulator rows per CTA, tile columns
constexpr uint32_t TMEM_COLS = 2 * BN;
// Columns (relative to the tile) of a row's entries that the sampled epilogue
// fetches before the tile's accumulator is ready: one byte each, packed in
// registers.
constexpr int kSelMax = 16;
static_assert(BN <= 256, "prefetched columns are bytes relative to the tile");
// bf16 output: each epilogue warp stages its 32 x 32 block (2 KB) before the coalesced stores
constexpr size_t kEpiBf16Smem = 4 * 2048;

enum { kOutBf16 = 0, kOutF32 = 1, kOutSampled = 2 };

// Epilogue warps per CTA: one per TMEM lane quarter, or, for the sampled
// output, two, each draining half of the tile's columns (its per-entry work
// makes its epilogue the longest, and the last tile's is hidden behind no MMA:
// 186.8 -> 182.6 us on q_proj). Two per quarter slowed the other outputs (the
// fused forward by 3 us; the bf16 output with an fp32 addend by 18 us).
template <int kMode>
constexpr int epi_warps() { return kMode == kOutSampled ? 8 : 4; }

// Extra warps of the fused forward: they transform rows of X (Z = X H, bf16,
// blocks of 2^kZ) while the other warps run the GEMM. Two warps (one 4096-point
// row at a time) keep up with the GEMM on q_proj and leave room for three
// 128-deep stages: 182.8 us against 184.9 us with four warps and five 64-deep
// stages (two 128-deep stages with four warps: 225 us).
constexpr int kZThreads = 64;
template <int kZ>
constexpr size_t z_smem() {
  if constexpr (kZ == 0) return 0;
  else
    return (size_t)(kZThreads / Geo<kZ, 8>::P) *
           ((size_t)Geo<kZ, 8>::NP * sizeof(float) + (size_t)(1u << kZ) * sizeof(__nv_bfloat16));
}

// How an operand's stage is filled (64-wide slabs of 128-byte rows, 128B swizzle):
enum {
  kLdK2d = 0,   // K-major, one 2-D box of rows x 64 K per slab of K (BK / 64 copies)
  kLdMn2d = 1,  // MN-major, one 2-D box of BK x 64 MN per slab of MN
  kLdMn3d = 2,  // MN-major, one 3-D box (64 MN, BK, slabs): the whole stage in one copy (MN % 64 == 0)
  kLdK3d = 3    // K-major, one 3-D box (64 K, rows, BK / 64 slabs): the whole stage in one copy (K % 64 == 0)
};
__host__ __device__ constexpr bool ld_mn(int mode) { return mode == kLdMn2d || mode == kLdMn3d; }

template <int CG, int kMode = kOutBf16, int kZ = 0>
struct Cfg {
  // k-block depth: 128 for the CTA pair (half the copies and barrier rounds per MMA of 64), 64 when the single
  // CTA's 256-row B leaves room for too few 128-deep stages
  static constexpr int BK = CG == 2 ? 128 : 64;
  static constexpr int kStages = CG == 1 ? 4 : 3;
  static constexpr uint32_t kABytes = BM * BK * 2;
  static constexpr int kBRows = BN / CG;  // rows of B this CTA loads
  static constexpr uint32_t kBBytes = kBRows * BK * 2;
  static constexpr uint32_t kStageBytes = kABytes + kBBytes;
  static constexpr size_t kEpiBytes = kMode == kOutBf16 ? kEpiBf16Smem : 0;
  static constexpr size_t kZOffset = (size_t)kStages * kStageBytes + 256 + kEpiBytes;  // from the aligned base
  static constexpr size_t kSmem = kZOffset + 1024 + z_smem<kZ>();
  static constexpr int kEpiWarps = epi_warps<kMode>();
  static constexpr int kGemmThreads = 64 + 32 * kEpiWarps;  // producer warp, MMA warp, epilogue warps
  static constexpr int kThreads = kGemmThreads + (kZ ? kZThreads : 0);
  // Instruction descriptor, kind::f16: D fp32 (bits 4-5 = 1), A bf16 (7-9 = 1),
  // B bf16 (10-12 = 1), both K-major (bits 15, 16 = 0), N >> 3 at bit 17,
  // M >> 4 at bit 24 (M = 128 per CTA of the group).
  static constexpr uint32_t kIdesc = (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(BN >> 3) << 17) |
                                     ((uint32_t)((BM * CG) >> 4) << 24);
};

// The transform the fused forward runs beside the GEMM.
struct ZArgs {
  const __nv_bfloat16 *x;
  __nv_bfloat16 *z;
  int64_t rows;  // rows of 2^kZ values
  float scale;
};

// Sampled output: dc[j] (+)= alpha * D[r_j, k_j] for the CSR entries of E.
struct SampleArgs {
  const int32_t *row_ptr;
  const int32_t *col_idx;
  float *dc;
  float alpha;
  int64_t p;
};
constexpr uint64_t kWaitNs = 2000000000ull;  // 2 s

__device__ __forceinline__ uint32_t smem_u32(const void *p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ uint64_t now_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}

__device__ __forceinline__ void mbar_expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes) : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}

// Wait for the phase with the given parity to complete; false after kWaitNs.
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = now_ns();
  for (;;) {
#pragma unroll 1
    for (int i = 0; i < 32; ++i)
      if (mbar_try_wait(bar, parity)) return true;
    if (now_ns() - t0 > kWaitNs) return false;
  }
}

// 2-D tensor copy into this CTA's shared memory. With CG = 2 the completion
// may be counted on the mbarrier of the other CTA of the pair (bar is then a
// shared::cluster address). No multicast.
template <int CG>
__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap *map, uint32_t bar, int x, int y) {
  if constexpr (CG == 1) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4}], [%2];" ::
            "r"(dst),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(bar), "r"(x), "r"(y)
        : "memory");
  } else {
    asm volatile(
        "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%3, "
        "%4}], [%2];" ::"r"(dst),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(bar), "r"(x), "r"(y)
        : "memory");
  }
}

// 3-D tensor copy (same rules as tma_load_2d): fills box[0] x box[1] x box[2]
// elements, the last dimension slowest, in shared memory.
template <int CG>
__device__ __forceinline__ void tma_load_3d(uint32_t dst, const CUtensorMap *map, uint32_t bar, int x, int y, int z) {
  if constexpr (CG == 1) {
    asm volatile(
        "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4, %5}], [%2];" ::
            "r"(dst),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(bar), "r"(x), "r"(y), "r"(z)
        : "memory");
  } else {
    asm volatile(
        "cp.async.bulk.tensor.3d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%3, "
        "%4, %5}], [%2];" ::"r"(dst),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(bar), "r"(x), "r"(y), "r"(z)
        : "memory");
  }
}

// One k-block of an operand into its stage (see the kLd* modes): `rows`
// M or N rows starting at `row`, K from kb * BK.
template <int CG, int BK>
__device__ __forceinline__ void load_stage(uint32_t dst, const CUtensorMap *map, uint32_t bar, int mode, int row,
                                           int rows, int kb) {
  if (mode == kLdK3d) {
    tma_load_3d<CG>(dst, map, bar, 0, row, kb * (BK / 64));
  } else if (mode == kLdMn3d) {
    tma_load_3d<CG>(dst, map, bar, 0, kb * BK, row / 64);
  } else if (mode == kLdMn2d) {
    for (int h = 0; h < rows / 64; ++h) tma_load_2d<CG>(dst + h * (BK * 128), map, bar, row + 64 * h, kb * BK);
  } else {
#pragma unroll
    for (int s = 0; s < BK / 64; ++s) tma_load_2d<CG>(dst + s * (rows * 128), map, bar, kb * BK + 64 * s, row);
  }
}

__device__ __forceinline__ uint32_t cluster_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}

// Address of the same shared variable in CTA `rank` of the cluster.
__device__ __forceinline__ uint32_t peer_addr(uint32_t saddr, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(saddr), "r"(rank));
  return r;
}

__device__ __forceinline__ void mbar_arrive_remote(uint32_t cluster_addr) {
  asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(cluster_addr) : "memory");
}

// All threads of both CTAs of the cluster (the non-.aligned form: lanes of a
// warp may arrive at different times).
__device__ __forceinline__ void cluster_sync() {
  asm volatile("barrier.cluster.arrive.release;\n\tbarrier.cluster.wait.acquire;" ::: "memory");
}

__device__ __forceinline__ uint64_t sw128_desc(uint32_t saddr) {
  // K-major: start >> 4 | LBO 16 B (unused for swizzled K-major) | SBO 1024 B
  // (8 rows of 128 B) | descriptor version 1 | layout SWIZZLE_128B (2)
  return (uint64_t)((saddr & 0x3FFFFu) >> 4) | ((uint64_t)1 << 16) | ((uint64_t)(1024 >> 4) << 32) |
         ((uint64_t)1 << 46) | ((uint64_t)2 << 61);
}

template <int BK>
__device__ __forceinline__ uint64_t sw128_desc_mn(uint32_t saddr) {
  // MN-major: the stage holds slabs of 64(MN) x BK(K), rows of 128 B along MN,
  // one slab after the other along MN. LBO = BK x 128 B (next 64 MN elements),
  // SBO = 1024 B (next 8 K rows), version 1, SWIZZLE_128B.
  return (uint64_t)((saddr & 0x3FFFFu) >> 4) | ((uint64_t)((BK * 128) >> 4) << 16) |
         ((uint64_t)(1024 >> 4) << 32) | ((uint64_t)1 << 46) | ((uint64_t)2 << 61);
}

template <int CG>
__device__ __forceinline__ void umma_bf16(uint32_t d_tmem, uint64_t a, uint64_t b, uint32_t idesc, uint32_t acc) {
  if constexpr (CG == 1) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(a), "l"(b), "r"(idesc), "r"(acc)
        : "memory");
  } else {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(a), "l"(b), "r"(idesc), "r"(acc)
        : "memory");
  }
}

// Arrive on `bar` (same offset) in every CTA of the group once the MMAs issued
// so far have completed.
template <int CG>
__device__ __forceinline__ void umma_commit_all(uint32_t bar) {
  if constexpr (CG == 1) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar)
                 : "memory");
  } else {
    asm volatile("tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], %1;" ::
                     "r"(bar),
                 "h"((unsigned short)3)
                 : "memory");
  }
}

// Arrive on this CTA's `bar` once the MMAs issued so far have completed.
template <int CG>
__device__ __forceinline__ void umma_commit_local(uint32_t bar) {
  if constexpr (CG == 1) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar)
                 : "memory");
  } else {
    asm volatile("tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar)
                 : "memory");
  }
}

template <int CG>
__device__ __forceinline__ void tmem_alloc(uint32_t slot, uint32_t cols) {
  if constexpr (CG == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(slot), "r"(cols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  } else {
    asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(slot), "r"(cols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
  }
}

template <int CG>
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t cols) {
  if constexpr (CG == 1)
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(cols) : "memory");
  else
    asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(cols) : "memory");
}

__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t *r) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, "
      "%15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
        "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
        "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

// r[k] for a run-time k in [0, 32): a tree of selects over the index bits, so
// the registers are only indexed at compile time (no local or shared memory).
__device__ __forceinline__ uint32_t pick32(const uint32_t (&r)[32], int k) {
  uint32_t a[16], b[8], c[4], d[2];
#pragma unroll
  for (int i = 0; i < 16; ++i) a[i] = (k & 1) ? r[2 * i + 1] : r[2 * i];
#pragma unroll
  for (int i = 0; i < 8; ++i) b[i] = (k & 2) ? a[2 * i + 1] : a[2 * i];
#pragma unroll
  for (int i = 0; i < 4; ++i) c[i] = (k & 4) ? b[2 * i + 1] : b[2 * i];
#pragma unroll
  for (int i = 0; i < 2; ++i) d[i] = (k & 8) ? c[2 * i + 1] : c[2 * i];
  return (k & 16) ? d[1] : d[0];
}

// kF32Out: write fp32 D (no rounding); otherwise bf16. addend may be NULL.
// a_ld / b_ld: how the operand's stage is filled (kLd*): K-major in global
// memory ([M or N rows][K contiguous]) or MN-major ([K rows][M or N
// contiguous]); a stage holds slabs of 128-byte rows (64 K per slab along K
// for K-major, BK K rows per slab of 64 MN for MN-major), filled by one 3-D
// copy when the slab dimension divides evenly, else by one 2-D copy per slab.
// k_splits > 1 (sampled output only): each tile's K range is cut into that
// many parts, each part a separate work unit adding its share into dc. Units
// are numbered part-major (unit = part * tiles + tile), so the units running
// at the same time read the same part of K and share it in L2.
template <int kMode, int CG, int kZ>
__global__ void __launch_bounds__(Cfg<CG, kMode, kZ>::kThreads, 1)
    gemm_bf16_tcgen05_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                             const float *__restrict__ addend, void *__restrict__ out_v, int M, int N, int K,
                             int a_ld, int b_ld, int group_m, int k_splits, SampleArgs sa_args, ZArgs za,
                             unsigned int *err) {
  using C = Cfg<CG, kMode, kZ>;
  constexpr int STAGES = C::kStages;
  constexpr int BK = C::BK;
  const bool a_mn = kZ ? false : ld_mn(a_ld), b_mn = kZ ? false : ld_mn(b_ld);
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint32_t base = smem_u32(smem_raw);
  const uint32_t pad = (1024u - (base & 1023u)) & 1023u;
  uint8_t *smem = smem_raw + pad;
  base += pad;
  uint64_t *bars = reinterpret_cast<uint64_t *>(smem + STAGES * C::kStageBytes);
  const uint32_t bar0 = smem_u32(bars);
  auto full = [&](int s) { return bar0 + 8u * s; };
  auto empty = [&](int s) { return bar0 + 8u * (STAGES + s); };
  auto tfull = [&](int b) { return bar0 + 8u * (2 * STAGES + b); };
  auto tempty = [&](int b) { return bar0 + 8u * (2 * STAGES + 2 + b); };
  const uint32_t done_bar = bar0 + 8u * (2 * STAGES + 4);
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + 2 * STAGES + 5);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);
  float *epi_stage = reinterpret_cast<float *>(smem + STAGES * C::kStageBytes + 256);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = CG == 2 ? cluster_rank() : 0u;  // position in the CTA pair
  const bool leader = rank == 0;
  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(full(s), 1);
      mbar_init(empty(s), 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(tfull(b), 1);
      mbar_init(tempty(b), C::kEpiWarps * CG);  // the epilogue warps of every CTA of the group
    }
    mbar_init(done_bar, 1);
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  }
  if (warp == 1) tmem_alloc<CG>(smem_u32(tmem_slot), TMEM_COLS);
  __syncwarp();
  tc_fence_before();
  if constexpr (CG == 2) cluster_sync();  // the peer's barriers and TMEM exist before any copy or MMA
  else __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  constexpr int TM = BM * CG;  // tile rows
  const int m_tiles = (M + TM - 1) / TM, n_tiles = (N + BN - 1) / BN;
  const int k_blocks = (K + BK - 1) / BK;
  const int kb_per_split = (k_blocks + k_splits - 1) / k_splits;
  const int num_tiles = m_tiles * n_tiles;
  const int num_units = num_tiles * k_splits;
  const int group_id = blockIdx.x / CG, n_groups = gridDim.x / CG;
  // Tile order: groups of group_m row blocks; inside a group, the row block
  // changes fastest and the column block slowest, so the tiles in flight share
  // a few row blocks of A and a run of column blocks of B in L2.
  auto tile_coords = [&](int tile, int &m_blk, int &n_blk) {
    const int gsize = group_m * n_tiles;
    const int g = tile / gsize, rem = tile % gsize;
    const int gm = min(group_m, m_tiles - g * group_m);
    m_blk = g * group_m + rem % gm;
    n_blk = rem / gm;
  };

  auto give_up = [&](unsigned code) {
    atomicOr(err, code);
    *abort_flag = 1;
  };

  if (warp == 0 && lane == 0) {
    // ------------------------------------------------ TMA producer (every CTA)
    int stage = 0;
    uint32_t phase = 0;
    int last_parity[STAGES];
    for (int s = 0; s < STAGES; ++s) last_parity[s] = -1;
    for (int unit = group_id; unit < num_units && !*abort_flag; unit += n_groups) {
      const int tile = unit % num_tiles, split = unit / num_tiles;
      int m_blk, n_blk;
      tile_coords(tile, m_blk, n_blk);
      const int a_row = m_blk * TM + (int)rank * BM;
      const int b_row = n_blk * BN + (int)rank * C::kBRows;
      const int kb0 = split * kb_per_split, kb1 = min(k_blocks, kb0 + kb_per_split);
      for (int kb = kb0; kb < kb1; ++kb) {
        if (!mbar_wait(empty(stage), phase ^ 1)) {
          give_up(0x1u);
          break;
        }
        if (*abort_flag) break;
        // both CTAs' bytes complete on the leader's barrier; only the leader arrives
        if (leader) mbar_expect_tx(full(stage), C::kStageBytes * CG);
        const uint32_t fb = CG == 2 ? peer_addr(full(stage), 0) : full(stage);
        const uint32_t sa = base + stage * C::kStageBytes, sb = sa + C::kABytes;
        if constexpr (kZ != 0) {
          // The fused forward reads both operands K-major, each stage in one 3-D copy. Its binary
          // holds only this path: with the generic one compiled in as well, the launch (four warp
          // roles, the transform's unrolled butterflies among them) ran ~10% slower.
          tma_load_3d<CG>(sa, &tmA, fb, 0, a_row, kb * (BK / 64));
          tma_load_3d<CG>(sb, &tmB, fb, 0, b_row, kb * (BK / 64));
        } else {
          load_stage<CG, BK>(sa, &tmA, fb, a_ld, a_row, BM, kb);
          load_stage<CG, BK>(sb, &tmB, fb, b_ld, b_row, C::kBRows, kb);
        }
        last_parity[stage] = (int)phase;
        if (++stage == STAGES) {
          stage = 0;
          phase ^= 1;
        }
      }
    }
    // drain: every copy of the group has landed before the CTAs exit (the
    // leader's barriers count the copies of both CTAs of a pair)
    if (leader)
      for (int s = 0; s < STAGES; ++s)
        if (last_parity[s] >= 0 && !mbar_wait(full(s), (uint32_t)last_parity[s])) give_up(0x2u);
  } else if (warp == 1 && lane == 0 && leader) {
    // ------------------------------------------------ MMA issuer (leader CTA)
    int stage = 0;
    uint32_t phase = 0;
    int it = 0;
    for (int unit = group_id; unit < num_units && !*abort_flag; unit += n_groups, ++it) {
      const int split = unit / num_tiles;
      const int kb0 = split * kb_per_split, kb1 = min(k_blocks, kb0 + kb_per_split);
      const int buf = it & 1;
      const uint32_t use = (uint32_t)(it >> 1);
      if (!mbar_wait(tempty(buf), (use & 1) ^ 1)) {
        give_up(0x4u);
        break;
      }
      tc_fence_after();
      const uint32_t d_tmem = tmem_base + (uint32_t)(buf * BN);
      bool ok = true;
      for (int kb = kb0; kb < kb1; ++kb) {
        if (!mbar_wait(full(stage), phase)) {
          give_up(0x8u);
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t sa = base + stage * C::kStageBytes, sb = sa + C::kABytes;
        // The descriptors of the stage once; the k-th MMA adds a constant to the start-address field
        // (address >> 4, 14 bits: shared addresses stay below 256 KB, so nothing carries out of it):
        // K-major +32 B per 16 of K inside the 128 B rows and the next slab (rows x 128 B) every 64 of K;
        // MN-major +2 KB (16 rows of 128 B) per 16 of K.
        const uint64_t da = a_mn ? sw128_desc_mn<BK>(sa) : sw128_desc(sa);
        const uint64_t db = b_mn ? sw128_desc_mn<BK>(sb) : sw128_desc(sb);
        const uint32_t idesc = C::kIdesc | ((uint32_t)a_mn << 15) | ((uint32_t)b_mn << 16);
#pragma unroll
        for (int k = 0; k < BK / 16; ++k) {
          const uint64_t oa = a_mn ? 128ull * k : (uint64_t)((k >> 2) * (BM * 128 / 16) + 2 * (k & 3));
          const uint64_t ob = b_mn ? 128ull * k : (uint64_t)((k >> 2) * (C::kBRows * 128 / 16) + 2 * (k & 3));
          umma_bf16<CG>(d_tmem, da + oa, db + ob, idesc, (kb > kb0 || k > 0) ? 1u : 0u);
        }
        umma_commit_all<CG>(empty(stage));
        if (++stage == STAGES) {
          stage = 0;
          phase ^= 1;
        }
      }
      if (!ok) break;
      umma_commit_all<CG>(tfull(buf));
    }
    // drain: all issued MMAs complete before TMEM is released
    umma_commit_local<CG>(done_bar);
    if (!mbar_wait(done_bar, 0)) give_up(0x10u);
  } else if (kZ && warp >= C::kGemmThreads / 32) {
    // ------------------------------------------------ fused transform Z = X H (every CTA)
    if constexpr (kZ != 0) {
      float *zs = reinterpret_cast<float *>(smem + C::kZOffset);
      fwht_rows_body<kZ, 8, __nv_bfloat16, __nv_bfloat16, kZThreads>(
          za.x, za.z, za.rows, za.scale, zs, (int)threadIdx.x - C::kGemmThreads, blockIdx.x, gridDim.x,
          [] { asm volatile("bar.sync 1, %0;" ::"n"(kZThreads) : "memory"); });
    }
  } else if (warp >= 2) {
    // ------------------------------------------------ epilogue (every CTA)
    const int q = warp & 3;  // TMEM lane quarter this warp may access
    // which half of the tile's columns this warp drains (warps 2-5 and 6-9 cover the four quarters)
    const int half = (warp - 2) / 4;
    constexpr int kChunks = BN / 32 / (C::kEpiWarps / 4);  // 32-column chunks per warp
    static_assert(C::kEpiWarps == 4 || C::kEpiWarps == 8, "one or two warps per lane quarter");
    int it = 0;
    float *my_stage = epi_stage + (warp - 2) * 512;
    for (int unit = group_id; unit < num_units; unit += n_groups, ++it) {
      const int tile = unit % num_tiles;
      const int buf = it & 1;
      const uint32_t use = (uint32_t)(it >> 1);
      int m_blk, n_blk;
      tile_coords(tile, m_blk, n_blk);
      const int row = m_blk * TM + (int)rank * BM + q * 32 + lane;
      // Sampled output: this row's CSR entries with column in [n0, n0 + BN), found while the tile's
      // MMAs still run (the search and the column loads are dependent global reads): j is the first
      // of them, and the columns of up to kSelMax of them, relative to n0, are packed four to a
      // register in selw (nsel of them; when all kSelMax fall in the tile, `more` says the ones after
      // are read in the chunk loop). The epilogue then touches no shared memory, whose bandwidth the
      // copies and the MMAs of the next tile are using.
      int64_t j = 0, j_end = 0;
      int nsel = 0;
      bool more = false;
      uint32_t selw[kSelMax / 4] = {};
      if (kMode == kOutSampled && row < M) {
        const int n0 = n_blk * BN;                 // offsets stay relative to the tile
        const int c0 = half * kChunks * 32;        // this warp's columns: [n0 + c0, n0 + c0 + 32 kChunks)
        j = sa_args.row_ptr[row];
        j_end = sa_args.row_ptr[row + 1];
        if (j < 0) j = 0;
        if (j_end > sa_args.p) j_end = sa_args.p;
        int64_t hi = j_end;  // first entry with column >= n0 + c0 (columns ascend within a row)
        while (j < hi) {
          const int64_t mid = (j + hi) >> 1;
          if (sa_args.col_idx[mid] < n0 + c0) j = mid + 1;
          else hi = mid;
        }
        int cols[kSelMax];
#pragma unroll
        for (int i = 0; i < kSelMax; ++i) cols[i] = j + i < j_end ? sa_args.col_idx[j + i] - n0 : BN;
#pragma unroll
        for (int i = 0; i < kSelMax; ++i) {
          const bool in = (unsigned)(cols[i] - c0) < (unsigned)(32 * kChunks);
          selw[i / 4] |= (in ? (uint32_t)cols[i] : 255u) << (8 * (i % 4));
          nsel += in ? 1 : 0;
        }
        more = nsel == kSelMax;
      }
      if (*abort_flag) break;
      if (!mbar_wait(tfull(buf), use & 1)) {
        give_up(0x20u);
        break;
      }
      tc_fence_after();
      int sel = 0;  // entries of the row already written: CSR positions j .. j + sel - 1
      for (int c = half * kChunks; c < (half + 1) * kChunks; ++c) {
        uint32_t r[32];
        tmem_ld32(tmem_base + ((uint32_t)(q * 32) << 16) + (uint32_t)(buf * BN + c * 32), r);
        const int col0 = n_blk * BN + c * 32;
        if (kMode == kOutSampled) {
          const int hi = 32 * (c + 1);  // chunk c covers tile columns [32 c, hi)
          auto put = [&](int o) {
            const float v = sa_args.alpha * __uint_as_float(pick32(r, o & 31));
            if (k_splits > 1) atomicAdd(sa_args.dc + j + sel, v);
            else sa_args.dc[j + sel] = v;
          };
          for (; sel < nsel; ++sel) {
            const uint32_t w = sel < 8 ? (sel < 4 ? selw[0] : selw[1]) : (sel < 12 ? selw[2] : selw[3]);
            const int o = (int)((w >> (8 * (sel & 3))) & 255u);
            if (o >= hi) break;
            put(o);
          }
          if (more && sel >= nsel) {  // past the prefetched entries: the rest from global memory
            for (; j + sel < j_end; ++sel) {
              const int o = sa_args.col_idx[j + sel] - n_blk * BN;
              if (o >= hi) break;
              put(o);
            }
          }
          continue;
        }
        if (kMode == kOutBf16 && !addend && col0 + 32 <= N) {
          // Through shared memory, so that a store instruction writes 8 rows x 64 B
          // (whole sectors) rather than 32 rows x 16 B. Rows are 64 B apart and the
          // 16-byte segment s of row r sits at s ^ ((r >> 1) & 3): both the
          // row-per-lane writes and the transposed reads are free of bank conflicts.
          unsigned char *st = reinterpret_cast<unsigned char *>(my_stage);
          float f[32];
#pragma unroll
          for (int j = 0; j < 32; ++j) f[j] = __uint_as_float(r[j]);
#pragma unroll
          for (int v = 0; v < 4; ++v)
            *reinterpret_cast<uint4 *>(st + lane * 64 + ((v ^ ((lane >> 1) & 3)) << 4)) =
                io<__nv_bfloat16>::pack(f + 8 * v);
          __syncwarp();
          const int row0 = row - lane;
#pragma unroll
          for (int v = 0; v < 4; ++v) {
            const int rr = 8 * v + (lane >> 2), sg = lane & 3;
            const uint4 w = *reinterpret_cast<const uint4 *>(st + rr * 64 + ((sg ^ ((rr >> 1) & 3)) << 4));
            if (row0 + rr < M)
              *reinterpret_cast<uint4 *>(static_cast<__nv_bfloat16 *>(out_v) + (int64_t)(row0 + rr) * N + col0 + 8 * sg) = w;
          }
          __syncwarp();  // the next chunk reuses the staging
          continue;
        }
        if (row < M && col0 < N) {
          const int64_t off = (int64_t)row * N + col0;
          float f[32];
#pragma unroll
          for (int j = 0; j < 32; ++j) f[j] = __uint_as_float(r[j]);
          if (addend) {
            const float *ad = addend + off;
            if (col0 + 32 <= N) {
#pragma unroll
              for (int v = 0; v < 8; ++v) {
                const float4 a4 = *reinterpret_cast<const float4 *>(ad + 4 * v);
                f[4 * v] += a4.x, f[4 * v + 1] += a4.y, f[4 * v + 2] += a4.z, f[4 * v + 3] += a4.w;
              }
            } else {
#pragma unroll
              for (int j = 0; j < 32; ++j)
                if (col0 + j < N) f[j] += ad[j];
            }
          }
          if (kMode == kOutF32) {
            float *o = static_cast<float *>(out_v) + off;
            if (col0 + 32 <= N) {
#pragma unroll
              for (int v = 0; v < 8; ++v)
                *reinterpret_cast<float4 *>(o + 4 * v) = make_float4(f[4 * v], f[4 * v + 1], f[4 * v + 2], f[4 * v + 3]);
            } else {
#pragma unroll
              for (int j = 0; j < 32; ++j)
                if (col0 + j < N) o[j] = f[j];
            }
          } else {
            __nv_bfloat16 *o = static_cast<__nv_bfloat16 *>(out_v) + off;
            if (col0 + 32 <= N) {
#pragma unroll
              for (int v = 0; v < 4; ++v) *reinterpret_cast<uint4 *>(o + 8 * v) = io<__nv_bfloat16>::pack(f + 8 * v);
            } else {
#pragma unroll
              for (int j = 0; j < 32; ++j)
                if (col0 + j < N) o[j] = __float2bfloat16_rn(f[j]);
            }
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        // the accumulator half in this CTA's TMEM is drained: tell the MMA issuer
        if constexpr (CG == 2) mbar_arrive_remote(peer_addr(tempty(buf), 0));
        else mbar_arrive(tempty(buf));
      }
    }
  }
  __syncwarp();
  tc_fence_before();
  // no CTA of a pair leaves (or frees TMEM) while the other may still signal
  // its barriers or the leader's MMAs may still use its memory
  if constexpr (CG == 2) cluster_sync();
  else __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc<CG>(tmem_base, TMEM_COLS);
  }
}

typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                  const cuuint64_t *, const cuuint32_t *, const cuuint32_t *, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  if (!fn) {
    void *p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  }
  return fn;
}

// rows x cols bf16 row-major, box = box_rows x 64 columns, 128-byte swizzle.
bool make_map(CUtensorMap *m, const void *ptr, int64_t rows, int64_t cols, uint32_t box_rows) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  const cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
  const cuuint64_t strides[1] = {(cuuint64_t)cols * 2};
  const cuuint32_t box[2] = {64u, box_rows};
  const cuuint32_t estr[2] = {1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(ptr), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// A K-major operand [rows, K] seen as a 3-D tensor (64 K elements, rows,
// K / 64 slabs of 128 B), box (64, box_rows, nslab): one copy fills nslab
// slabs of box_rows x 128 B, one after the other. Requires K % 64 == 0.
bool make_map_k3d(CUtensorMap *m, const void *ptr, int64_t rows, int64_t K, uint32_t box_rows, uint32_t nslab) {
  EncodeTiledFn fn = encode_fn();
  if (!fn || K % 64) return false;
  const cuuint64_t dims[3] = {64u, (cuuint64_t)rows, (cuuint64_t)(K / 64)};
  const cuuint64_t strides[2] = {(cuuint64_t)K * 2, 128u};
  const cuuint32_t box[3] = {64u, box_rows, nslab};
  const cuuint32_t estr[3] = {1, 1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(ptr), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// An MN-major operand [K, MN] seen as a 3-D tensor (64 MN elements, K rows,
// MN / 64 slabs of 128 B), box (64, bk, nslab): one copy fills nslab slabs of
// bk x 128 B (one after the other). Requires MN % 64 == 0.
bool make_map_mn3d(CUtensorMap *m, const void *ptr, int64_t K, int64_t MN, uint32_t bk, uint32_t nslab) {
  EncodeTiledFn fn = encode_fn();
  if (!fn || MN % 64) return false;
  const cuuint64_t dims[3] = {64u, (cuuint64_t)K, (cuuint64_t)(MN / 64)};
  const cuuint64_t strides[2] = {(cuuint64_t)MN * 2, 128u};
  const cuuint32_t box[3] = {64u, bk, nslab};
  const cuuint32_t estr[3] = {1, 1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(ptr), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Co-resident CTA groups of the CG variant (one CTA per SM; pairs need two SMs
// of one cluster slot).
template <int kMode, int CG, int kZ>
int resident_groups() {
  static int cached[64] = {};  // per device
  int &n = cached[device_slot()];
  if (n) return n;
  using C = Cfg<CG, kMode, kZ>;
  const int sms = sm_count();
  if (CG == 1) return n = sms;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)(sms - sms % CG));
  cfg.blockDim = dim3(C::kThreads);
  cfg.dynamicSmemBytes = C::kSmem;
  cudaLaunchAttribute at[1];
  at[0].id = cudaLaunchAttributeClusterDimension;
  at[0].val.clusterDim.x = CG;
  at[0].val.clusterDim.y = 1;
  at[0].val.clusterDim.z = 1;
  cfg.attrs = at;
  cfg.numAttrs = 1;
  int clusters = 0;
  if (cudaOccupancyMaxActiveClusters(&clusters, gemm_bf16_tcgen05_kernel<kMode, CG, kZ>, &cfg) != cudaSuccess ||
      clusters < 1) {
    (void)cudaGetLastError();
    clusters = sms / CG;
  }
  return n = clusters;
}

// A is [M, K] (K-major) or, with a_mn, [K, M]; B is [N, K] or, with b_mn, [K, N].
// With kZ, the launch also transforms za.rows rows of za.x into za.z.
template <int kMode, int CG, int kZ = 0>
cudaError_t launch_gemm_cg(const void *A, const void *B, const float *addend, void *out, int64_t M, int64_t N,
                           int64_t K, bool a_mn, bool b_mn, const SampleArgs &sa, cudaStream_t s,
                           const ZArgs &za = ZArgs{}) {
  using C = Cfg<CG, kMode, kZ>;
  CUtensorMap ta, tb;
  constexpr int BK = C::BK;
  // one 3-D copy per operand and stage where the slab dimension divides evenly, else one 2-D copy per slab
  auto mode = [&](bool mn, int64_t MN) {
    if (mn) return MN % 64 == 0 ? (int)kLdMn3d : (int)kLdMn2d;
    return (BK > 64 && K % 64 == 0) ? (int)kLdK3d : (int)kLdK2d;
  };
  const int a_ld = mode(a_mn, M), b_ld = mode(b_mn, N);
  auto map = [&](CUtensorMap *t, const void *P, int ld, int64_t MN, uint32_t rows) {
    switch (ld) {
      case kLdK3d: return make_map_k3d(t, P, MN, K, rows, BK / 64);
      case kLdMn3d: return make_map_mn3d(t, P, K, MN, BK, rows / 64);
      case kLdMn2d: return make_map(t, P, K, MN, BK);
      default: return make_map(t, P, MN, K, rows);
    }
  };
  // the fused forward's producer issues only 3-D K-major copies (its K, d_in, is a whole number of 2048-point
  // blocks)
  if (kZ && (a_ld != kLdK3d || b_ld != kLdK3d)) return cudaErrorNotSupported;
  if (!map(&ta, A, a_ld, M, BM) || !map(&tb, B, b_ld, N, C::kBRows)) return cudaErrorInvalidValue;
  auto kern = gemm_bf16_tcgen05_kernel<kMode, CG, kZ>;
  static bool attr[64] = {};  // per device
  bool &attr_done = attr[device_slot()];
  if (!attr_done) {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)C::kSmem);
    if (e != cudaSuccess) return e;
    attr_done = true;
  }
  const int64_t m_tiles = cdiv(M, (int64_t)BM * CG), n_tiles = cdiv(N, BN);
  const int64_t tiles = m_tiles * n_tiles;
  // Rows of A per group: all column blocks of B for one row block at a time
  // when B fits comfortably in L2 (it is then read from DRAM once); otherwise
  // enough row blocks that the tiles in flight span a bounded slice of B.
  const int64_t b_bytes = N * K * 2;
  int64_t group_m = 1;
  if (b_bytes > (48ll << 20)) {
    group_m = 8 / CG;
    if (group_m > m_tiles) group_m = m_tiles;
  }
  const int groups = resident_groups<kMode, CG, kZ>();
  // Sampled output: split K in two when the tiles alone would leave the last
  // wave of groups mostly idle (each dc then receives exactly two additions
  // onto zero, whose result does not depend on their order).
  int k_splits = 1;
  if (kMode == kOutSampled && cdiv(K, BK) >= 4) {
    const double waves1 = (double)tiles / groups, waves2 = 2.0 * tiles / groups;
    const double eff1 = waves1 / std::ceil(waves1), eff2 = waves2 / std::ceil(waves2);
    if (eff2 > eff1 + 0.02) k_splits = 2;
  }
  if (kMode == kOutSampled) {
    cudaError_t e = k_splits > 1 ? cudaMemsetAsync(sa.dc, 0, (size_t)sa.p * sizeof(float), s) : cudaSuccess;
    if (e != cudaSuccess) return e;
  }
  const int64_t units = tiles * k_splits;
  // the fused transform runs in every CTA: launch all resident groups even when there are fewer tiles
  const int64_t n_launch = kZ ? groups : (units < groups ? units : groups);
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)(n_launch * CG));
  cfg.blockDim = dim3(C::kThreads);
  cfg.dynamicSmemBytes = C::kSmem;
  cfg.stream = s;
  cudaLaunchAttribute at[1];
  at[0].id = cudaLaunchAttributeClusterDimension;
  at[0].val.clusterDim.x = CG;
  at[0].val.clusterDim.y = 1;
  at[0].val.clusterDim.z = 1;
  cfg.attrs = at;
  cfg.numAttrs = CG > 1 ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, kern, ta, tb, addend, out, (int)M, (int)N, (int)K, a_ld, b_ld,
                            (int)group_m, k_splits, sa, za, device_error_word());
}

// The pair variant once there are at least two 128-row blocks of output.
template <int kMode>
cudaError_t launch_gemm_t(const void *A, const void *B, const float *addend, void *out, int64_t M, int64_t N,
                          int64_t K, bool a_mn, bool b_mn, const SampleArgs &sa, cudaStream_t s) {
  if (M <= 0 || N <= 0) return cudaSuccess;
  if (M > BM) return launch_gemm_cg<kMode, 2>(A, B, addend, out, M, N, K, a_mn, b_mn, sa, s);
  return launch_gemm_cg<kMode, 1>(A, B, addend, out, M, N, K, a_mn, b_mn, sa, s);
}

cudaError_t launch_gemm(const void *A, const void *B, const float *addend, void *out, int64_t M, int64_t N,
                        int64_t K, cudaStream_t s) {
  return launch_gemm_t<kOutBf16>(A, B, addend, out, M, N, K, false, false, SampleArgs{}, s);
}

}  // namespace

cudaError_t launch_gemm_fwd(const void *X, const void *wdeq, const float *y_ad, void *Y, int64_t T, int32_t d_out,
                            int32_t d_in, cudaStream_t s) {
  return launch_gemm(X, wdeq, y_ad, Y, T, d_out, d_in, s);
}

cudaError_t launch_gemm_nt(const void *A, const void *B, const float *addend, void *out, bool f32_out, int64_t M,
                           int64_t N, int64_t K, cudaStream_t s) {
  return f32_out ? launch_gemm_t<kOutF32>(A, B, addend, out, M, N, K, false, false, SampleArgs{}, s)
                 : launch_gemm_t<kOutBf16>(A, B, addend, out, M, N, K, false, false, SampleArgs{}, s);
}

cudaError_t launch_gemm_any(const void *A, bool a_mn, const void *B, bool b_mn, const float *addend, void *out,
                            bool f32_out, int64_t M, int64_t N, int64_t K, cudaStream_t s) {
  return f32_out ? launch_gemm_t<kOutF32>(A, B, addend, out, M, N, K, a_mn, b_mn, SampleArgs{}, s)
                 : launch_gemm_t<kOutBf16>(A, B, addend, out, M, N, K, a_mn, b_mn, SampleArgs{}, s);
}

bool gemm_fused_fwht_supported(int64_t M, int logn) { return M > BM && (logn == 11 || logn == 12); }

cudaError_t launch_gemm_fwd_fused(const void *X, const void *W, void *Y, int64_t T, int32_t d_out, int32_t d_in,
                                  void *Z, int logn, float scale, cudaStream_t s) {
  if (T <= 0 || d_out <= 0) return cudaSuccess;
  if (!gemm_fused_fwht_supported(T, logn)) return cudaErrorNotSupported;
  ZArgs za{static_cast<const __nv_bfloat16 *>(X), static_cast<__nv_bfloat16 *>(Z), T * (d_in >> logn), scale};
  if (logn == 12)
    return launch_gemm_cg<kOutBf16, 2, 12>(X, W, nullptr, Y, T, d_out, d_in, false, false, SampleArgs{}, s, za);
  return launch_gemm_cg<kOutBf16, 2, 11>(X, W, nullptr, Y, T, d_out, d_in, false, false, SampleArgs{}, s, za);
}

bool make_map_rows(CUtensorMap *m, const void *ptr, int64_t rows, int64_t cols, int64_t ld, uint32_t box_cols,
                   uint32_t box_rows) {
  EncodeTiledFn fn = encode_fn();
  if (!fn || (ld * 2) % 16 || (reinterpret_cast<uintptr_t>(ptr) & 15)) return false;
  const cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
  const cuuint64_t strides[1] = {(cuuint64_t)ld * 2};
  const cuuint32_t box[2] = {box_cols, box_rows};
  const cuuint32_t estr[2] = {1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(ptr), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

cudaError_t launch_gemm_sampled(const void *A, bool a_mn, const void *B, bool b_mn, int64_t M, int64_t N, int64_t K,
                                const int32_t *row_ptr, const int32_t *col_idx, int64_t p, float alpha, float *dc,
                                cudaStream_t s) {
  SampleArgs sa{row_ptr, col_idx, dc, alpha, p};
  return launch_gemm_t<kOutSampled>(A, B, nullptr, nullptr, M, N, K, a_mn, b_mn, sa, s);
}

}  // namespace qwha
