// C ABI of libqwha: argument checks, workspace carving and launch sequencing.
// Every entry point validates on the host and launches nothing on failure.

#include <math.h>
#include <stdarg.h>
#include <stdio.h>

#include <algorithm>
#include <atomic>
#include <mutex>
#include <vector>

#include "common.cuh"
#include "kernels.h"

namespace qwha {

namespace {
thread_local char g_msg[512] = "";
}

qwha_status fail(qwha_status s, const char *fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_msg, sizeof(g_msg), fmt, ap);
  va_end(ap);
  return s;
}

namespace {
std::atomic<uint64_t> g_ring_wait_ns{2000000000ull};
std::atomic<int32_t> g_injected_failures{0};
}  // namespace

uint64_t ring_wait_ns() { return g_ring_wait_ns.load(std::memory_order_relaxed); }

qwha_status cuda_status(cudaError_t e, const char *what) {
  if (e == cudaSuccess) {
    // test hook: report an armed number of successful results as failures
    int32_t n = g_injected_failures.load();
    while (n > 0 && !g_injected_failures.compare_exchange_weak(n, n - 1)) {
    }
    if (n <= 0) return QWHA_OK;
    return fail(QWHA_ERR_CUDA, "%s: injected failure (qwha_debug_fail_cuda_checks)", what);
  }
  return fail(QWHA_ERR_CUDA, "%s: %s (cudaError %d)", what, cudaGetErrorString(e), (int)e);
}

int sm_count() {
  static int counts[64] = {0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 148;
  if (counts[dev] == 0) {
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) n = 148;
    counts[dev] = n;
  }
  return counts[dev];
}

int device_slot() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 0;
  return dev;
}

}  // namespace qwha

using namespace qwha;

namespace {

const char *dtype_name(qwha_dtype d) { return d == QWHA_F32 ? "f32" : d == QWHA_BF16 ? "bf16" : "?"; }

bool valid_dtype(qwha_dtype d) { return d == QWHA_F32 || d == QWHA_BF16; }

// A second stream per device on which the dense forward computes Z = X H while
// the caller's stream builds W_eff and runs the GEMM (they do not depend on each
// other). Fork and join go through events, so the work stays ordered with the
// caller's stream and is captured with it in a CUDA graph.
struct Fork {
  cudaStream_t aux = nullptr;
  cudaEvent_t fork = nullptr, join = nullptr;
};

std::mutex g_fork_mu;
Fork g_fork[64];

cudaError_t get_fork(Fork **out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  Fork &f = g_fork[dev];
  if (!f.aux) {
    e = cudaStreamCreateWithFlags(&f.aux, cudaStreamNonBlocking);
    if (e == cudaSuccess) e = cudaEventCreateWithFlags(&f.fork, cudaEventDisableTiming);
    if (e == cudaSuccess) e = cudaEventCreateWithFlags(&f.join, cudaEventDisableTiming);
    if (e != cudaSuccess) return e;
  }
  *out = &f;
  return cudaSuccess;
}

qwha_status check_hadamard(int32_t n, int32_t had_block) {
  if (n <= 0) return fail(QWHA_ERR_INVALID_ARG, "row length %d must be positive", n);
  if (had_block < 2 || had_block > 32768 || !is_pow2(had_block))
    return fail(QWHA_ERR_INVALID_ARG, "had_block %d must be a power of two in [2, 32768]", had_block);
  if (n % had_block)
    return fail(QWHA_ERR_INVALID_ARG, "had_block %d does not divide the row length %d", had_block, n);
  return QWHA_OK;
}

#define QWHA_CHECK_PTR(p, name)                                                        \
  do {                                                                                 \
    if (!(p)) return fail(QWHA_ERR_INVALID_ARG, "%s is NULL", name);                   \
    if (!aligned16(p)) return fail(QWHA_ERR_MISALIGNED, "%s is not 16-byte aligned", name); \
  } while (0)

}  // namespace

// ---------------------------------------------------------------- stage timing

namespace {

enum Stage {
  ST_FWHT_FWD,
  ST_SPMM_FWD,
  ST_DEQUANT,
  ST_GEMM_FWD,
  ST_SDDMM,
  ST_GATHER_BWD,
  ST_FWHT_BWD,
  ST_GEMM_BWD,
  ST_INIT,
  ST_PLAN,
  ST_FWHT,
  ST_WEFF,
  ST_GEMM_DC,
  ST_COUNT
};
const char *kStageNames[ST_COUNT] = {"fwht_fwd",   "spmm_fwd",   "dequant",  "gemm_fwd",  "sddmm_dc",
                                     "gather_bwd", "fwht_bwd",   "gemm_bwd", "init_alloc",
                                     "plan_build", "fwht",       "weff",      "gemm_dc"};

struct StageRec {
  int stage, kernels;
  cudaEvent_t a, b;
};

std::mutex g_prof_mu;
bool g_prof_on = false;
std::vector<StageRec> g_pending;
std::vector<cudaEvent_t> g_pool;
int64_t g_calls[ST_COUNT], g_launches[ST_COUNT];
double g_ms[ST_COUNT];

cudaEvent_t take_event() {
  if (!g_pool.empty()) {
    cudaEvent_t e = g_pool.back();
    g_pool.pop_back();
    return e;
  }
  cudaEvent_t e = nullptr;
  if (cudaEventCreate(&e) != cudaSuccess) return nullptr;
  return e;
}

// Brackets one stage with events when timing is on; counts launches always-on cheaply.
struct StageScope {
  int stage, kernels;
  cudaStream_t s;
  cudaEvent_t a = nullptr;
  StageScope(int st, int k, cudaStream_t str) : stage(st), kernels(k), s(str) {
    std::lock_guard<std::mutex> g(g_prof_mu);
    if (!g_prof_on) return;
    a = take_event();
    if (a) cudaEventRecord(a, s);
  }
  ~StageScope() {
    std::lock_guard<std::mutex> g(g_prof_mu);
    if (!g_prof_on || !a) return;
    cudaEvent_t b = take_event();
    if (!b) return;
    cudaEventRecord(b, s);
    g_pending.push_back({stage, kernels, a, b});
  }
};

}  // namespace

extern "C" {

void qwha_stage_timing(int32_t enable) {
  std::lock_guard<std::mutex> g(g_prof_mu);
  g_prof_on = enable != 0;
}

int32_t qwha_stage_count(void) { return ST_COUNT; }

const char *qwha_stage_name(int32_t i) { return (i >= 0 && i < ST_COUNT) ? kStageNames[i] : ""; }

qwha_status qwha_stage_report(int64_t *calls, int64_t *launches, double *ms) {
  std::lock_guard<std::mutex> g(g_prof_mu);
  qwha_status st = QWHA_OK;
  for (const StageRec &r : g_pending) {
    float t = 0.f;
    cudaError_t e = cudaEventSynchronize(r.b);
    if (e == cudaSuccess) e = cudaEventElapsedTime(&t, r.a, r.b);
    if (e != cudaSuccess && st == QWHA_OK) st = cuda_status(e, "stage events");
    g_calls[r.stage] += 1;
    g_launches[r.stage] += r.kernels;
    g_ms[r.stage] += t;
    g_pool.push_back(r.a);
    g_pool.push_back(r.b);
  }
  g_pending.clear();
  for (int i = 0; i < ST_COUNT; ++i) {
    if (calls) calls[i] = g_calls[i];
    if (launches) launches[i] = g_launches[i];
    if (ms) ms[i] = g_ms[i];
    g_calls[i] = g_launches[i] = 0;
    g_ms[i] = 0.0;
  }
  return st;
}

}  // extern "C"

extern "C" {

const char *qwha_status_string(qwha_status s) {
  switch (s) {
    case QWHA_OK: return "ok";
    case QWHA_ERR_INVALID_ARG: return "invalid argument";
    case QWHA_ERR_MISALIGNED: return "misaligned buffer";
    case QWHA_ERR_UNSUPPORTED: return "unsupported";
    case QWHA_ERR_WORKSPACE: return "workspace too small";
    case QWHA_ERR_CUDA: return "CUDA error";
    case QWHA_ERR_TIMEOUT: return "device wait timed out";
  }
  return "unknown status";
}

const char *qwha_last_error(void) { return g_msg; }

uint64_t qwha_debug_wait_limit_ns(uint64_t ns) { return g_ring_wait_ns.exchange(ns); }

void qwha_debug_fail_cuda_checks(int32_t n) { g_injected_failures.store(n > 0 ? n : 0); }

const char *qwha_version(void) { return "qwha-b200 0.1 (sm_100a)"; }

qwha_status qwha_fwht(qwha_dtype dt, const void *x, void *z, int64_t rows, int32_t n,
                      int32_t had_block, void *stream) {
  if (!valid_dtype(dt)) return fail(QWHA_ERR_INVALID_ARG, "dtype %d", (int)dt);
  qwha_status st = check_hadamard(n, had_block);
  if (st != QWHA_OK) return st;
  if (rows < 0) return fail(QWHA_ERR_INVALID_ARG, "rows %lld < 0", (long long)rows);
  if (rows == 0) return QWHA_OK;
  QWHA_CHECK_PTR(x, "x");
  QWHA_CHECK_PTR(z, "z");
  const size_t esz = dt == QWHA_F32 ? 4 : 2;
  const char *xb = static_cast<const char *>(x), *zb = static_cast<const char *>(z);
  const size_t bytes = (size_t)rows * n * esz;
  if (xb < zb + bytes && zb < xb + bytes) return fail(QWHA_ERR_INVALID_ARG, "x and z overlap");
  const int logn = ilog2(had_block);
  const float scale = (float)(1.0 / sqrt((double)had_block));
  (void)dtype_name;
  StageScope sc(ST_FWHT, 1, (cudaStream_t)stream);
  return cuda_status(launch_fwht(dt, dt, x, z, rows * (n / had_block), logn, scale, (cudaStream_t)stream),
                     "fwht launch");
}

}  // extern "C"

// ---------------------------------------------------------------- adapter

namespace {

struct Carver {  // hands out 256-byte aligned slices of the caller's workspace
  char *base;
  size_t off = 0;
  explicit Carver(void *b) : base(static_cast<char *>(b)) {}
  void *take(size_t bytes) {
    void *p = base ? base + off : nullptr;
    off += align_up(bytes, 256);
    return p;
  }
};


qwha_status check_adapter_shape(const qwha_adapter *a) {
  if (!a) return fail(QWHA_ERR_INVALID_ARG, "adapter is NULL");
  if (a->d_in <= 0 || a->d_out <= 0 || a->d_in % 8 || a->d_out % 8)
    return fail(QWHA_ERR_INVALID_ARG, "d_in %d and d_out %d must be positive multiples of 8", a->d_in, a->d_out);
  qwha_status st = check_hadamard(a->d_in, a->had_block);
  if (st != QWHA_OK) return st;
  if (a->p < 0 || a->p > (int64_t)a->d_in * a->d_out || a->p > 2147483647LL)
    return fail(QWHA_ERR_INVALID_ARG, "p = %lld out of range", (long long)a->p);
  if (a->algo != QWHA_ALGO_SPARSE && a->algo != QWHA_ALGO_DENSE)
    return fail(QWHA_ERR_INVALID_ARG, "algo %d", (int)a->algo);
  if (a->algo == QWHA_ALGO_DENSE && weff_smem(a->d_in) > 200 * 1024)
    return fail(QWHA_ERR_UNSUPPORTED, "dense algorithm: d_in %d above 51200", a->d_in);
  if (a->weff && !aligned16(a->weff)) return fail(QWHA_ERR_MISALIGNED, "weff is not 16-byte aligned");
  QWHA_CHECK_PTR(a->row_ptr, "row_ptr");
  if (a->p > 0) {
    QWHA_CHECK_PTR(a->col_idx, "col_idx");
    QWHA_CHECK_PTR(a->coef, "coef");
  }
  return QWHA_OK;
}

qwha_status check_views(const qwha_adapter *a) {
  QWHA_CHECK_PTR(a->col_ptr, "col_ptr");
  QWHA_CHECK_PTR(a->tile_ptr, "tile_ptr");
  if (a->p > 0) {
    QWHA_CHECK_PTR(a->row_idx, "row_idx");
    QWHA_CHECK_PTR(a->perm, "perm");
    QWHA_CHECK_PTR(a->tile_pos, "tile_pos");
    QWHA_CHECK_PTR(a->tile_rk, "tile_rk");
  }
  if (cdiv(a->d_out, QWHA_TILE) > plan_max_row_blocks())
    return fail(QWHA_ERR_UNSUPPORTED, "d_out %d above %d", a->d_out, plan_max_row_blocks() * QWHA_TILE);
  return QWHA_OK;
}

qwha_status check_qweight(const qwha_qweight *wq, int32_t d_out, int32_t d_in, qwha_dtype dt) {
  if (!wq) return QWHA_OK;
  if (dt != QWHA_BF16) return fail(QWHA_ERR_UNSUPPORTED, "the base GEMM needs dtype bf16");
  if (wq->bits < 2 || wq->bits > 4) return fail(QWHA_ERR_INVALID_ARG, "bits %d not in {2,3,4}", wq->bits);
  if (wq->group <= 0 || wq->group % 8 || d_in % wq->group)
    return fail(QWHA_ERR_INVALID_ARG, "group %d must be a multiple of 8 dividing d_in %d", wq->group, d_in);
  QWHA_CHECK_PTR(wq->qweight, "qweight");
  QWHA_CHECK_PTR(wq->scales, "scales");
  QWHA_CHECK_PTR(wq->zeros, "zeros");
  (void)d_out;
  return QWHA_OK;
}

qwha_status check_ws(void *ws, size_t ws_bytes, size_t need) {
  if (need == 0) return QWHA_OK;
  if (!ws || ws_bytes < need)
    return fail(QWHA_ERR_WORKSPACE, "workspace %zu bytes, need %zu", ws ? ws_bytes : (size_t)0, need);
  if (reinterpret_cast<uintptr_t>(ws) & 255) return fail(QWHA_ERR_MISALIGNED, "workspace not 256-byte aligned");
  return QWHA_OK;
}

// packed (index, value) entries of the SpMM in gather order
// Scratch of the SpMM for both directions: the forward over rows (segments
// d_out, width d_in) and the backward gather over columns.
size_t ent_bytes(int64_t p, int32_t d_out, int32_t d_in) {
  return std::max(spmm_scratch_bytes(p, d_out, d_in), spmm_scratch_bytes(p, d_in, d_out));
}

size_t fwd_ws(int32_t d_out, int32_t d_in, int64_t p, int64_t T, bool base) {
  const size_t n = ent_bytes(p, d_out, d_in);
  if (!base) return n;
  return n + align_up((size_t)T * d_out * 4, 256) + align_up(wdeq_bytes(d_out, d_in), 256);
}

size_t fwd_dense_ws(int32_t d_out, int32_t d_in) { return align_up((size_t)d_out * d_in * 2, 256); }


size_t bwd_dense_ws(int32_t d_out, int32_t d_in, int64_t T) {
  (void)T;
  return align_up((size_t)d_out * d_in * 2, 256);  // W_eff (unless the adapter carries one)
}

// The sparse backward's dZ buffer, which first holds the transposed dY and Z
// of the coefficient gradient (the gather writes dZ after the gradient has run).
size_t dz_region(int32_t d_out, int32_t d_in, int64_t T) {
  return std::max(align_up((size_t)T * d_in * 4, 256), sddmm_transposed_bytes(T, d_out, d_in));
}

size_t bwd_ws(int32_t d_out, int32_t d_in, int64_t p, int64_t T, bool base) {
  size_t n = align_up((size_t)kSddmmMaxChunks * (size_t)(p > 0 ? p : 1) * 4, 256);
  n += dz_region(d_out, d_in, T);  // dZ, and before it the transposed dY and Z of the gradient
  n += ent_bytes(p, d_out, d_in);  // CSC entries in gather order
  if (base) n += align_up((size_t)T * d_in * 4, 256) + align_up(wdeq_bytes(d_out, d_in), 256);
  return n;
}

// Dense backward: W_eff, dX = dY W_eff (W_eff read MN-major), and dc = alpha *
// (dY^T Z) sampled at E by the GEMM epilogue (both operands read MN-major as
// stored).
qwha_status dense_bwd(const qwha_adapter *a, const qwha_qweight *wq, const void *dY, const void *Z, int64_t T,
                      float alpha, float *dc, void *dX, void *ws, cudaStream_t s) {
  Carver cv(ws);
  void *weff = a->weff ? a->weff : cv.take((size_t)a->d_out * a->d_in * 2);
  cudaError_t e = cudaSuccess;
  if (dX && T > 0) {
    if (!a->weff) {  // otherwise the forward's W_eff is used as it stands
      StageScope sc(ST_WEFF, 1, s);
      e = launch_weff(a, wq, alpha, weff, s);
    }
    if (e != cudaSuccess) return cuda_status(e, "W_eff");
    {
      StageScope sc(ST_GEMM_BWD, 1, s);
      e = launch_gemm_any(dY, false, weff, true, nullptr, dX, false, T, a->d_in, a->d_out, s);
    }
    if (e != cudaSuccess) return cuda_status(e, "GEMM dX");
  }
  if (a->p == 0 || !dc) return QWHA_OK;
  if (T == 0) return cuda_status(cudaMemsetAsync(dc, 0, (size_t)a->p * 4, s), "dc = 0");
  // the coefficient gradient as a sampled dense product: the tcgen05 GEMM's
  // epilogue writes alpha * (dY^T Z)[r_j, k_j] for the entries of E only
  StageScope sc(ST_GEMM_DC, 1, s);
  return cuda_status(launch_gemm_sampled(dY, true, Z, true, a->d_out, a->d_in, T, a->row_ptr, a->col_idx, a->p, alpha,
                                         dc, s),
                     "sampled GEMM dY^T Z");
}

}  // namespace

extern "C" {

int64_t qwha_plan_tiles(int32_t d_out, int32_t d_in) {
  if (d_out <= 0 || d_in <= 0) return 0;
  return cdiv(d_out, QWHA_TILE) * cdiv(d_in, QWHA_TILE);
}

size_t qwha_workspace_size(qwha_op op, int32_t d_out, int32_t d_in, int64_t p, int64_t T, int32_t with_base) {
  if (d_out <= 0 || d_in <= 0 || T < 0 || p < 0) return 0;
  switch (op) {
    case QWHA_OP_FWD: return fwd_ws(d_out, d_in, p, T, with_base != 0);
    case QWHA_OP_BWD: return bwd_ws(d_out, d_in, p, T, with_base != 0);
    case QWHA_OP_INIT: return init_workspace(d_out, d_in);
    case QWHA_OP_PLAN: return plan_workspace(d_out, d_in);
    case QWHA_OP_FWD_DENSE: return fwd_dense_ws(d_out, d_in);
    case QWHA_OP_BWD_DENSE: return bwd_dense_ws(d_out, d_in, T);
    case QWHA_OP_SELECT_GLOBAL: return select_global_workspace(d_out, d_in);
    case QWHA_OP_REFINE: return refine_workspace(d_out, d_in);
    case QWHA_OP_ENERGY: return energy_stats_workspace(d_out, d_in);
    case QWHA_OP_PATTERN: return pattern_stats_workspace(d_in);
  }
  return 0;
}

qwha_status qwha_adapter_fwd(const qwha_adapter *a, const qwha_qweight *wq, qwha_dtype dt, const void *X,
                             int64_t T, float alpha, void *Z_out, void *Y, void *ws, size_t ws_bytes,
                             void *stream) {
  qwha_status st = check_adapter_shape(a);
  if (st != QWHA_OK) return st;
  if (!valid_dtype(dt)) return fail(QWHA_ERR_INVALID_ARG, "dtype %d", (int)dt);
  if ((st = check_qweight(wq, a->d_out, a->d_in, dt)) != QWHA_OK) return st;
  if (T < 0) return fail(QWHA_ERR_INVALID_ARG, "T %lld < 0", (long long)T);
  if (T == 0) return QWHA_OK;
  QWHA_CHECK_PTR(X, "X");
  QWHA_CHECK_PTR(Z_out, "Z_out");
  QWHA_CHECK_PTR(Y, "Y");
  const bool dense = a->algo == QWHA_ALGO_DENSE;
  if (dense && dt != QWHA_BF16) return fail(QWHA_ERR_UNSUPPORTED, "the dense algorithm needs dtype bf16");
  const size_t need = dense ? fwd_dense_ws(a->d_out, a->d_in) : fwd_ws(a->d_out, a->d_in, a->p, T, wq != nullptr);
  if ((st = check_ws(ws, ws_bytes, need)) != QWHA_OK) return st;
  cudaStream_t s = (cudaStream_t)stream;
  const int logn = ilog2(a->had_block);
  const float inv = (float)(1.0 / sqrt((double)a->had_block));
  cudaError_t e = cudaSuccess;
  if (dense && a->z_given) {  // Z_out is an input: W_eff and the GEMM only
    void *weff = a->weff ? a->weff : ws;
    {
      StageScope sc(ST_WEFF, 1, s);
      e = launch_weff(a, wq, alpha, weff, s);
    }
    if (e != cudaSuccess) return cuda_status(e, "W_eff");
    StageScope sc(ST_GEMM_FWD, 1, s);
    return cuda_status(launch_gemm_nt(X, weff, nullptr, Y, false, T, a->d_out, a->d_in, s), "GEMM");
  }
  if (dense && gemm_fused_fwht_supported(T, logn)) {
    // W_eff, then one launch for Y = X W_eff^T whose extra warps write Z = X H
    // (kept for the backward) while the tensor cores run the GEMM.
    void *weff = a->weff ? a->weff : ws;
    {
      StageScope sc(ST_WEFF, 1, s);
      e = launch_weff(a, wq, alpha, weff, s);
    }
    if (e != cudaSuccess) return cuda_status(e, "W_eff");
    StageScope sc(ST_GEMM_FWD, 1, s);
    return cuda_status(launch_gemm_fwd_fused(X, weff, Y, T, a->d_out, a->d_in, Z_out, logn, inv, s),
                       "GEMM + transform");
  }
  if (dense) {
    // Z = X H (kept for the backward) on the auxiliary stream, concurrently
    // with W_eff and Y = X W_eff^T on the caller's stream.
    std::lock_guard<std::mutex> g(g_fork_mu);
    Fork *f = nullptr;
    e = get_fork(&f);
    if (e == cudaSuccess) e = cudaEventRecord(f->fork, s);
    if (e == cudaSuccess) e = cudaStreamWaitEvent(f->aux, f->fork, 0);
    if (e != cudaSuccess) return cuda_status(e, "fork");
    {
      StageScope sc(ST_FWHT_FWD, 1, f->aux);
      e = launch_fwht(dt, dt, X, Z_out, T * (a->d_in / a->had_block), logn, inv, f->aux);
    }
    if (e == cudaSuccess) e = cudaEventRecord(f->join, f->aux);
    if (e != cudaSuccess) return cuda_status(e, "fwht");
    void *weff = a->weff ? a->weff : ws;
    {
      StageScope sc(ST_WEFF, 1, s);
      e = launch_weff(a, wq, alpha, weff, s);
    }
    if (e == cudaSuccess) {
      StageScope sc(ST_GEMM_FWD, 1, s);
      e = launch_gemm_nt(X, weff, nullptr, Y, false, T, a->d_out, a->d_in, s);
    }
    const cudaError_t ej = cudaStreamWaitEvent(s, f->join, 0);  // join even after a failed launch
    if (e != cudaSuccess) return cuda_status(e, "W_eff / GEMM");
    return cuda_status(ej, "join");
  }
  if (!a->z_given) {
    StageScope sc(ST_FWHT_FWD, 1, s);
    e = launch_fwht(dt, dt, X, Z_out, T * (a->d_in / a->had_block), logn, inv, s);
  }
  if (e != cudaSuccess) return cuda_status(e, "fwht");
  Carver cv(ws);
  const size_t ent_n = ent_bytes(a->p, a->d_out, a->d_in);
  void *ent = cv.take(ent_n);
  if (!wq) {
    StageScope sc(ST_SPMM_FWD, 0, s);
    e = launch_seg_spmm(dt, dt, Z_out, T, a->d_in, a->row_ptr, a->col_idx, a->coef, nullptr, a->p, a->d_out, alpha,
                        ent, ent_n, Y, s, &sc.kernels);
    return cuda_status(e, "spmm");
  }
  float *y_ad = static_cast<float *>(cv.take((size_t)T * a->d_out * 4));
  void *wdeq = cv.take(wdeq_bytes(a->d_out, a->d_in));
  {
    StageScope sc(ST_SPMM_FWD, 0, s);
    e = launch_seg_spmm(dt, QWHA_F32, Z_out, T, a->d_in, a->row_ptr, a->col_idx, a->coef, nullptr, a->p, a->d_out,
                        alpha, ent, ent_n, y_ad, s, &sc.kernels);
  }
  if (e != cudaSuccess) return cuda_status(e, "spmm");
  {
    StageScope sc(ST_DEQUANT, 1, s);
    e = launch_dequant(wq->bits, wq->group, a->d_out, a->d_in, wq->qweight, wq->scales, wq->zeros, wdeq, s);
  }
  if (e != cudaSuccess) return cuda_status(e, "dequant");
  StageScope sc(ST_GEMM_FWD, 1, s);
  return cuda_status(launch_gemm_fwd(X, wdeq, y_ad, Y, T, a->d_out, a->d_in, s), "base GEMM");
}

qwha_status qwha_adapter_bwd(const qwha_adapter *a, const qwha_qweight *wq, qwha_dtype dt, const void *dY,
                             const void *Z, int64_t T, float alpha, float *dc, void *dX, void *ws,
                             size_t ws_bytes, void *stream) {
  qwha_status st = check_adapter_shape(a);
  if (st != QWHA_OK) return st;
  const bool dense = a->algo == QWHA_ALGO_DENSE;
  if (!dense && (st = check_views(a)) != QWHA_OK) return st;
  if (!valid_dtype(dt)) return fail(QWHA_ERR_INVALID_ARG, "dtype %d", (int)dt);
  if (dense && dt != QWHA_BF16) return fail(QWHA_ERR_UNSUPPORTED, "the dense algorithm needs dtype bf16");
  if ((st = check_qweight(wq, a->d_out, a->d_in, dt)) != QWHA_OK) return st;
  if (T < 0) return fail(QWHA_ERR_INVALID_ARG, "T %lld < 0", (long long)T);
  if (a->p > 0 && dc) QWHA_CHECK_PTR(dc, "dc");
  if (T > 0) {
    QWHA_CHECK_PTR(dY, "dY");
    QWHA_CHECK_PTR(Z, "Z");
    if (dX) QWHA_CHECK_PTR(dX, "dX");
  }
  const size_t need = dense ? bwd_dense_ws(a->d_out, a->d_in, T) : bwd_ws(a->d_out, a->d_in, a->p, T, wq != nullptr);
  if ((st = check_ws(ws, ws_bytes, need)) != QWHA_OK) return st;
  cudaStream_t s = (cudaStream_t)stream;
  if (dense) return dense_bwd(a, wq, dY, Z, T, alpha, dc, dX, ws, s);
  Carver cv(ws);
  float *partial = static_cast<float *>(cv.take((size_t)kSddmmMaxChunks * (size_t)(a->p > 0 ? a->p : 1) * 4));
  float *dz = static_cast<float *>(cv.take(dz_region(a->d_out, a->d_in, T)));
  const size_t ent_n = ent_bytes(a->p, a->d_out, a->d_in);
  void *ent = cv.take(ent_n);
  cudaError_t e = cudaSuccess;
  if (dc) {
    StageScope sc(ST_SDDMM, 0, s);
    e = launch_sddmm(dt, dY, Z, T, a->d_out, a->d_in, a->tile_ptr, a->tile_pos, a->tile_rk, a->p, alpha, partial, dc,
                     s, dz, &sc.kernels);
  }
  if (e != cudaSuccess) return cuda_status(e, "sddmm");
  if (!dX || T == 0) return QWHA_OK;
  {
    StageScope sc(ST_GATHER_BWD, 0, s);
    e = launch_seg_spmm(dt, QWHA_F32, dY, T, a->d_out, a->col_ptr, a->row_idx, a->coef, a->perm, a->p, a->d_in, alpha,
                        ent, ent_n, dz, s, &sc.kernels);
  }
  if (e != cudaSuccess) return cuda_status(e, "gather");
  const int logn = ilog2(a->had_block);
  const float inv = (float)(1.0 / sqrt((double)a->had_block));
  const int64_t blocks = T * (a->d_in / a->had_block);
  if (!wq) {
    StageScope sc(ST_FWHT_BWD, 1, s);
    return cuda_status(launch_fwht(QWHA_F32, dt, dz, dX, blocks, logn, inv, s), "fwht");
  }
  float *dx_ad = static_cast<float *>(cv.take((size_t)T * a->d_in * 4));
  void *wdeq = cv.take(wdeq_bytes(a->d_out, a->d_in));
  {
    StageScope sc(ST_FWHT_BWD, 1, s);
    e = launch_fwht(QWHA_F32, QWHA_F32, dz, dx_ad, blocks, logn, inv, s);
  }
  if (e != cudaSuccess) return cuda_status(e, "fwht");
  {
    StageScope sc(ST_DEQUANT, 1, s);
    e = launch_dequant(wq->bits, wq->group, a->d_out, a->d_in, wq->qweight, wq->scales, wq->zeros, wdeq, s);
  }
  if (e != cudaSuccess) return cuda_status(e, "dequant");
  StageScope sc(ST_GEMM_BWD, 1, s);
  // dX = dY W_Q + dX_adapter: W_Q [d_out, d_in] is the MN-major B operand as stored
  return cuda_status(launch_gemm_any(dY, false, wdeq, true, dx_ad, dX, false, T, a->d_in, a->d_out, s),
                     "base GEMM (dX)");
}

qwha_status qwha_plan_build(int32_t d_out, int32_t d_in, int64_t p, const int32_t *row_ptr, const int32_t *col_idx,
                            int32_t *col_ptr, int32_t *row_idx, int32_t *perm, int32_t *tile_ptr,
                            int32_t *tile_pos, int32_t *tile_rk, void *ws, size_t ws_bytes, void *stream) {
  if (d_out <= 0 || d_in <= 0) return fail(QWHA_ERR_INVALID_ARG, "d_out %d, d_in %d", d_out, d_in);
  if (cdiv(d_out, QWHA_TILE) > plan_max_row_blocks())
    return fail(QWHA_ERR_UNSUPPORTED, "d_out %d above %d", d_out, plan_max_row_blocks() * QWHA_TILE);
  if (p < 0 || p > (int64_t)d_in * d_out || p > 2147483647LL)
    return fail(QWHA_ERR_INVALID_ARG, "p = %lld out of range", (long long)p);
  QWHA_CHECK_PTR(row_ptr, "row_ptr");
  QWHA_CHECK_PTR(col_ptr, "col_ptr");
  QWHA_CHECK_PTR(tile_ptr, "tile_ptr");
  if (p > 0) {
    QWHA_CHECK_PTR(col_idx, "col_idx");
    QWHA_CHECK_PTR(row_idx, "row_idx");
    QWHA_CHECK_PTR(perm, "perm");
    QWHA_CHECK_PTR(tile_pos, "tile_pos");
    QWHA_CHECK_PTR(tile_rk, "tile_rk");
  }
  qwha_status st = check_ws(ws, ws_bytes, plan_workspace(d_out, d_in));
  if (st != QWHA_OK) return st;
  StageScope sc(ST_PLAN, 5, (cudaStream_t)stream);
  return cuda_status(launch_plan_build(d_out, d_in, p, row_ptr, col_idx, col_ptr, row_idx, perm, tile_ptr, tile_pos,
                                       tile_rk, ws, (cudaStream_t)stream),
                     "plan_build");
}

qwha_status qwha_validate_plan(const qwha_adapter *a, void *stream) {
  qwha_status st = check_adapter_shape(a);
  if (st != QWHA_OK) return st;
  uint32_t code = 0;
  int64_t where = 0;
  cudaError_t e = launch_validate(a, (cudaStream_t)stream, &code, &where);
  if (e != cudaSuccess) return cuda_status(e, "validate");
  if (code) return fail(QWHA_ERR_INVALID_ARG, "%s (at %lld)", validate_message(code), (long long)where);
  return QWHA_OK;
}

qwha_status qwha_check_stream_status(void *stream) {
  cudaError_t e = cudaStreamSynchronize((cudaStream_t)stream);
  if (e != cudaSuccess) return cuda_status(e, "stream");
  unsigned int word = 0;
  e = read_and_clear_error_word(&word, (cudaStream_t)stream);
  if (e != cudaSuccess) return cuda_status(e, "error word");
  if (word) return fail(QWHA_ERR_TIMEOUT, "device wait gave up (code 0x%x)", word);
  return QWHA_OK;
}

qwha_status qwha_init_alloc(const float *dWq, int32_t d_out, int32_t d_in, int32_t had_block, int64_t p,
                            int32_t min_per_row, qwha_remainder mode, int32_t *budgets, int32_t *row_ptr,
                            int32_t *col_idx, float *coef, void *ws, size_t ws_bytes, void *stream) {
  if (d_out <= 0 || d_in <= 0) return fail(QWHA_ERR_INVALID_ARG, "d_out %d, d_in %d", d_out, d_in);
  qwha_status st = check_hadamard(d_in, had_block);
  if (st != QWHA_OK) return st;
  if (d_in > init_max_din()) return fail(QWHA_ERR_UNSUPPORTED, "d_in %d above %d", d_in, init_max_din());
  if (min_per_row < 0 || min_per_row > d_in) return fail(QWHA_ERR_INVALID_ARG, "min_per_row %d", min_per_row);
  if (p < (int64_t)min_per_row * d_out || p > (int64_t)d_in * d_out || p > 2147483647LL)
    return fail(QWHA_ERR_INVALID_ARG, "p = %lld outside [%lld, %lld]", (long long)p,
                (long long)min_per_row * d_out, (long long)d_in * d_out);
  if (mode != QWHA_REM_FEWEST_ALLOC && mode != QWHA_REM_LARGEST_ERROR)
    return fail(QWHA_ERR_INVALID_ARG, "remainder mode %d", (int)mode);
  QWHA_CHECK_PTR(dWq, "dWq");
  QWHA_CHECK_PTR(budgets, "budgets");
  QWHA_CHECK_PTR(row_ptr, "row_ptr");
  if (p > 0) {
    QWHA_CHECK_PTR(col_idx, "col_idx");
    QWHA_CHECK_PTR(coef, "coef");
  }
  if ((st = check_ws(ws, ws_bytes, init_workspace(d_out, d_in))) != QWHA_OK) return st;
  StageScope sc(ST_INIT, 3, (cudaStream_t)stream);
  return cuda_status(launch_init_alloc(dWq, d_out, d_in, had_block, p, min_per_row, (int)mode, budgets, row_ptr,
                                       col_idx, coef, ws, (cudaStream_t)stream),
                     "init_alloc");
}

qwha_status qwha_init_select_global(const float *dWq, int32_t d_out, int32_t d_in, int32_t had_block, int64_t p,
                                    qwha_selection sel, uint64_t seed, int32_t *budgets, int32_t *row_ptr,
                                    int32_t *col_idx, float *coef, void *ws, size_t ws_bytes, void *stream) {
  if (d_out <= 0 || d_in <= 0) return fail(QWHA_ERR_INVALID_ARG, "d_out %d, d_in %d", d_out, d_in);
  qwha_status st = check_hadamard(d_in, had_block);
  if (st != QWHA_OK) return st;
  if (d_in > init_max_din()) return fail(QWHA_ERR_UNSUPPORTED, "d_in %d above %d", d_in, init_max_din());
  if (p < 0 || p > (int64_t)d_in * d_out || p > 2147483647LL)
    return fail(QWHA_ERR_INVALID_ARG, "p = %lld outside [0, %lld]", (long long)p, (long long)d_in * d_out);
  if (sel != QWHA_SEL_MAGNITUDE && sel != QWHA_SEL_RANDOM) return fail(QWHA_ERR_INVALID_ARG, "selection %d", (int)sel);
  QWHA_CHECK_PTR(dWq, "dWq");
  QWHA_CHECK_PTR(budgets, "budgets");
  QWHA_CHECK_PTR(row_ptr, "row_ptr");
  if (p > 0) {
    QWHA_CHECK_PTR(col_idx, "col_idx");
    QWHA_CHECK_PTR(coef, "coef");
  }
  if ((st = check_ws(ws, ws_bytes, select_global_workspace(d_out, d_in))) != QWHA_OK) return st;
  StageScope sc(ST_INIT, 21, (cudaStream_t)stream);
  return cuda_status(launch_select_global(dWq, d_out, d_in, had_block, p, (int)sel, seed, budgets, row_ptr, col_idx,
                                          coef, ws, (cudaStream_t)stream),
                     "init_select_global");
}

qwha_status qwha_energy_stats(const float *dWq, int32_t d_out, int32_t d_in, int32_t had_block, int64_t k,
                              double *stats, void *ws, size_t ws_bytes, void *stream) {
  if (d_out <= 0 || d_in <= 0) return fail(QWHA_ERR_INVALID_ARG, "d_out %d, d_in %d", d_out, d_in);
  qwha_status st = check_hadamard(d_in, had_block);
  if (st != QWHA_OK) return st;
  if (d_in > init_max_din()) return fail(QWHA_ERR_UNSUPPORTED, "d_in %d above %d", d_in, init_max_din());
  if (k < 1 || k >= (int64_t)d_in * d_out || k >= 2147483647LL)
    return fail(QWHA_ERR_INVALID_ARG, "k = %lld outside [1, %lld)", (long long)k, (long long)d_in * d_out);
  QWHA_CHECK_PTR(dWq, "dWq");
  QWHA_CHECK_PTR(stats, "stats");
  if ((st = check_ws(ws, ws_bytes, energy_stats_workspace(d_out, d_in))) != QWHA_OK) return st;
  StageScope sc(ST_INIT, 20, (cudaStream_t)stream);
  return cuda_status(launch_energy_stats(dWq, d_out, d_in, had_block, k, stats, ws, (cudaStream_t)stream),
                     "energy_stats");
}

qwha_status qwha_pattern_stats(int32_t d_out, int32_t d_in, int64_t p, const int32_t *row_ptr, const int32_t *col_idx,
                               int32_t *col_counts, int64_t *stats, void *ws, size_t ws_bytes, void *stream) {
  if (d_out <= 0 || d_in <= 0) return fail(QWHA_ERR_INVALID_ARG, "d_out %d, d_in %d", d_out, d_in);
  if (p < 0 || p > (int64_t)d_in * d_out || p > 2147483647LL)
    return fail(QWHA_ERR_INVALID_ARG, "p = %lld outside [0, %lld]", (long long)p, (long long)d_in * d_out);
  QWHA_CHECK_PTR(row_ptr, "row_ptr");
  if (p > 0) QWHA_CHECK_PTR(col_idx, "col_idx");
  QWHA_CHECK_PTR(col_counts, "col_counts");
  QWHA_CHECK_PTR(stats, "stats");
  qwha_status st = check_ws(ws, ws_bytes, pattern_stats_workspace(d_in));
  if (st != QWHA_OK) return st;
  StageScope sc(ST_INIT, 4, (cudaStream_t)stream);
  return cuda_status(launch_pattern_stats(d_out, d_in, p, row_ptr, col_idx, col_counts, stats, ws,
                                          (cudaStream_t)stream),
                     "pattern_stats");
}

qwha_status qwha_calib_hessian(const void *X, int64_t T, int32_t d_in, float *S, void *stream) {
  if (T < 1 || d_in <= 0 || d_in % 8) return fail(QWHA_ERR_INVALID_ARG, "T %lld, d_in %d (a multiple of 8)", (long long)T, d_in);
  QWHA_CHECK_PTR(X, "X");
  QWHA_CHECK_PTR(S, "S");
  if ((uintptr_t)X % 16 || (uintptr_t)S % 16) return fail(QWHA_ERR_MISALIGNED, "X and S must be 16-byte aligned");
  StageScope sc(ST_INIT, 1, (cudaStream_t)stream);
  return cuda_status(launch_calib_hessian(X, T, d_in, S, (cudaStream_t)stream), "calib_hessian");
}

qwha_status qwha_refine_values(const float *dWq, int32_t d_out, int32_t d_in, int32_t had_block, const float *S,
                               float damp, const int32_t *row_ptr, const int32_t *col_idx, int64_t p, float *coef,
                               void *ws, size_t ws_bytes, void *stream) {
  if (d_out <= 0 || d_in <= 0 || d_in % 8) return fail(QWHA_ERR_INVALID_ARG, "d_out %d, d_in %d (a multiple of 8)", d_out, d_in);
  qwha_status st = check_hadamard(d_in, had_block);
  if (st != QWHA_OK) return st;
  if (!(damp >= 0.0f)) return fail(QWHA_ERR_INVALID_ARG, "damp %g", (double)damp);
  if (p < 0 || p > (int64_t)d_in * d_out || p > 2147483647LL) return fail(QWHA_ERR_INVALID_ARG, "p %lld", (long long)p);
  if (p == 0) return QWHA_OK;
  QWHA_CHECK_PTR(dWq, "dWq");
  QWHA_CHECK_PTR(S, "S");
  QWHA_CHECK_PTR(row_ptr, "row_ptr");
  QWHA_CHECK_PTR(col_idx, "col_idx");
  QWHA_CHECK_PTR(coef, "coef");
  if ((uintptr_t)dWq % 16 || (uintptr_t)S % 16) return fail(QWHA_ERR_MISALIGNED, "dWq and S must be 16-byte aligned");
  if ((st = check_ws(ws, ws_bytes, refine_workspace(d_out, d_in))) != QWHA_OK) return st;
  StageScope sc(ST_INIT, 14, (cudaStream_t)stream);
  return cuda_status(launch_refine(dWq, d_out, d_in, had_block, S, damp, row_ptr, col_idx, p, coef, ws,
                                   (cudaStream_t)stream),
                     "refine_values");
}

qwha_status qwha_init_norms(const float *dWq, int32_t rows, int32_t d_in, double *e, void *stream) {
  if (rows < 0 || d_in <= 0) return fail(QWHA_ERR_INVALID_ARG, "rows %d, d_in %d", rows, d_in);
  if (rows == 0) return QWHA_OK;
  QWHA_CHECK_PTR(dWq, "dWq");
  QWHA_CHECK_PTR(e, "e");
  StageScope sc(ST_INIT, 1, (cudaStream_t)stream);
  return cuda_status(launch_init_norms(dWq, rows, d_in, e, (cudaStream_t)stream), "init_norms");
}

qwha_status qwha_init_budgets(const double *e, int32_t d_out, int32_t d_in, int64_t p, int32_t min_per_row,
                              qwha_remainder mode, int32_t *budgets, int32_t *row_ptr, void *ws, size_t ws_bytes,
                              void *stream) {
  if (d_out <= 0 || d_in <= 0) return fail(QWHA_ERR_INVALID_ARG, "d_out %d, d_in %d", d_out, d_in);
  if (min_per_row < 0 || min_per_row > d_in) return fail(QWHA_ERR_INVALID_ARG, "min_per_row %d", min_per_row);
  if (p < (int64_t)min_per_row * d_out || p > (int64_t)d_in * d_out || p > 2147483647LL)
    return fail(QWHA_ERR_INVALID_ARG, "p = %lld outside [%lld, %lld]", (long long)p,
                (long long)min_per_row * d_out, (long long)d_in * d_out);
  if (mode != QWHA_REM_FEWEST_ALLOC && mode != QWHA_REM_LARGEST_ERROR)
    return fail(QWHA_ERR_INVALID_ARG, "remainder mode %d", (int)mode);
  QWHA_CHECK_PTR(e, "e");
  QWHA_CHECK_PTR(budgets, "budgets");
  QWHA_CHECK_PTR(row_ptr, "row_ptr");
  qwha_status st = check_ws(ws, ws_bytes, init_workspace(d_out, d_in));
  if (st != QWHA_OK) return st;
  StageScope sc(ST_INIT, 1, (cudaStream_t)stream);
  return cuda_status(launch_init_budgets(e, d_out, d_in, p, min_per_row, (int)mode, budgets, row_ptr, ws,
                                         (cudaStream_t)stream),
                     "init_budgets");
}

qwha_status qwha_init_select(const float *dWq, int32_t rows, int32_t d_in, int32_t had_block, const int32_t *budgets,
                             const int32_t *row_ptr, int64_t p_local, int32_t *col_idx, float *coef, void *stream) {
  if (rows < 0) return fail(QWHA_ERR_INVALID_ARG, "rows %d", rows);
  qwha_status st = check_hadamard(d_in, had_block);
  if (st != QWHA_OK) return st;
  if (d_in > init_max_din()) return fail(QWHA_ERR_UNSUPPORTED, "d_in %d above %d", d_in, init_max_din());
  if (p_local < 0 || p_local > 2147483647LL) return fail(QWHA_ERR_INVALID_ARG, "p_local %lld", (long long)p_local);
  if (rows == 0 || p_local == 0) return QWHA_OK;
  QWHA_CHECK_PTR(dWq, "dWq");
  QWHA_CHECK_PTR(budgets, "budgets");
  QWHA_CHECK_PTR(row_ptr, "row_ptr");
  QWHA_CHECK_PTR(col_idx, "col_idx");
  QWHA_CHECK_PTR(coef, "coef");
  StageScope sc(ST_INIT, 1, (cudaStream_t)stream);
  return cuda_status(launch_init_select(dWq, rows, d_in, had_block, budgets, row_ptr, p_local, col_idx, coef,
                                        (cudaStream_t)stream),
                     "init_select");
}

}  // extern "C"
