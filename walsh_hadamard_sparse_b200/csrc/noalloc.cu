// Coefficient gradient without any device allocation by the library or the
// caller: the scratch of the gradient's chunked partial sums lives in a
// file-scope device array that is part of the loaded library.
//
// Who needs this: a caller that can hand the library only its inputs and
// outputs. Examples are a custom-op slot in a host framework that offers no
// workspace hook, and code that must not call cudaMalloc in the middle of a
// step (cudaMalloc can synchronize the whole device and can fail under a fixed
// memory budget). qwha_adapter_bwd needs caller-provided scratch; this entry
// point does not.
//
// Rules that follow from a single shared array:
//   * the array holds QWHA_NOALLOC_SCRATCH_BYTES on every GPU that loads the
//     library, for the life of the process;
//   * every call on a device uses the same array, so two calls whose work
//     overlaps on the GPU (different streams, or graph replays in flight at
//     once) race; serialize them (one stream, or events);
//   * the partial sums are cleared at the start of every call, so nothing
//     left by an earlier call leaks into the result.
// In host code the array's name is only a host-side stand-in, so its device
// address is looked up with cudaGetSymbolAddress, once per CUDA context, on
// the first call made with that context current (for ordinary runtime users:
// once per device, in its primary context). That first call must therefore
// come before any stream capture. The cache is keyed on the context's
// process-unique id, so a context created later (after cudaDeviceReset, or a
// driver-API context of the caller's own) gets its own lookup instead of a
// stale address.

#include <cuda.h>

#include <mutex>

#include "common.cuh"
#include "kernels.h"

namespace qwha {
namespace {

static __device__ __align__(256) unsigned char g_noalloc_scratch[QWHA_NOALLOC_SCRATCH_BYTES];

// Driver entry points reached through the runtime, so the library needs no
// link against libcuda.
using CtxGetCurrentFn = CUresult (*)(CUcontext *);
using CtxGetIdFn = CUresult (*)(CUcontext, unsigned long long *);

struct CachedAddress {
  unsigned long long ctx_id;
  void *addr;
};
constexpr int kMaxContexts = 64;
std::mutex g_mu;
CachedAddress g_cache[kMaxContexts];
int g_cached = 0, g_next_evict = 0;
CtxGetCurrentFn g_ctx_get_current = nullptr;
CtxGetIdFn g_ctx_get_id = nullptr;

qwha_status driver_entry_points() {
  if (g_ctx_get_current && g_ctx_get_id) return QWHA_OK;
  void *f0 = nullptr, *f1 = nullptr;
  cudaDriverEntryPointQueryResult q0 = cudaDriverEntryPointSymbolNotFound, q1 = q0;
  cudaError_t e = cudaGetDriverEntryPoint("cuCtxGetCurrent", &f0, cudaEnableDefault, &q0);
  if (e != cudaSuccess || q0 != cudaDriverEntryPointSuccess || !f0)
    return e != cudaSuccess ? cuda_status(e, "cudaGetDriverEntryPoint(cuCtxGetCurrent)")
                            : fail(QWHA_ERR_CUDA, "cuCtxGetCurrent not found");
  e = cudaGetDriverEntryPoint("cuCtxGetId", &f1, cudaEnableDefault, &q1);
  if (e != cudaSuccess || q1 != cudaDriverEntryPointSuccess || !f1)
    return e != cudaSuccess ? cuda_status(e, "cudaGetDriverEntryPoint(cuCtxGetId)")
                            : fail(QWHA_ERR_CUDA, "cuCtxGetId not found (driver older than CUDA 12.0)");
  g_ctx_get_current = reinterpret_cast<CtxGetCurrentFn>(f0);
  g_ctx_get_id = reinterpret_cast<CtxGetIdFn>(f1);
  return QWHA_OK;
}

// Device address of the scratch array in the current context (looked up on
// the first call in that context).
qwha_status scratch_address(void **out) {
  std::lock_guard<std::mutex> g(g_mu);
  qwha_status st = driver_entry_points();
  if (st != QWHA_OK) return st;
  CUcontext ctx = nullptr;
  if (g_ctx_get_current(&ctx) != CUDA_SUCCESS) return fail(QWHA_ERR_CUDA, "cuCtxGetCurrent failed");
  void *p = nullptr;
  if (!ctx) {
    // No context is current yet: the runtime makes the current device's
    // primary context current on its first call that needs one, this lookup.
    cudaError_t e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess) return cuda_status(e, "cudaGetSymbolAddress(scratch)");
    if (g_ctx_get_current(&ctx) != CUDA_SUCCESS || !ctx) return fail(QWHA_ERR_CUDA, "no current CUDA context");
  }
  unsigned long long id = 0;
  if (g_ctx_get_id(ctx, &id) != CUDA_SUCCESS) return fail(QWHA_ERR_CUDA, "cuCtxGetId failed");
  for (int i = 0; i < g_cached; ++i)
    if (g_cache[i].ctx_id == id) {
      *out = g_cache[i].addr;
      return QWHA_OK;
    }
  if (!p) {
    cudaError_t e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess) return cuda_status(e, "cudaGetSymbolAddress(scratch)");
  }
  const int slot = g_cached < kMaxContexts ? g_cached++ : (g_next_evict++ % kMaxContexts);
  g_cache[slot] = {id, p};
  *out = p;
  return QWHA_OK;
}

}  // namespace
}  // namespace qwha

using namespace qwha;

extern "C" qwha_status qwha_coef_grad_noalloc(const qwha_adapter *a, qwha_dtype dt, const void *dY, const void *Z,
                                              int64_t T, float alpha, float *dc, void *stream) {
  if (!a) return fail(QWHA_ERR_INVALID_ARG, "adapter is NULL");
  if (dt != QWHA_F32 && dt != QWHA_BF16) return fail(QWHA_ERR_INVALID_ARG, "dtype %d", (int)dt);
  if (a->d_in <= 0 || a->d_out <= 0 || a->d_in % 8 || a->d_out % 8)
    return fail(QWHA_ERR_INVALID_ARG, "d_in %d and d_out %d must be positive multiples of 8", a->d_in, a->d_out);
  if (a->p < 0 || a->p > (int64_t)a->d_in * a->d_out || a->p > 2147483647LL)
    return fail(QWHA_ERR_INVALID_ARG, "p = %lld out of range", (long long)a->p);
  if (T < 0) return fail(QWHA_ERR_INVALID_ARG, "T %lld < 0", (long long)T);
  if (cdiv(a->d_out, QWHA_TILE) > plan_max_row_blocks())
    return fail(QWHA_ERR_UNSUPPORTED, "d_out %d above %d", a->d_out, plan_max_row_blocks() * QWHA_TILE);
  if (a->p == 0) return QWHA_OK;
  if (!a->tile_ptr || !a->tile_pos || !a->tile_rk || !dc || (T > 0 && (!dY || !Z)))
    return fail(QWHA_ERR_INVALID_ARG, "a required pointer is NULL (tile view, dc, dY, Z)");
  if (!aligned16(a->tile_ptr) || !aligned16(a->tile_pos) || !aligned16(a->tile_rk) || !aligned16(dc) ||
      (T > 0 && (!aligned16(dY) || !aligned16(Z))))
    return fail(QWHA_ERR_MISALIGNED, "a device buffer is not 16-byte aligned");
  const size_t need = (size_t)sddmm_chunks(T, a->d_out, a->d_in) * (size_t)a->p * sizeof(float);
  if (need > QWHA_NOALLOC_SCRATCH_BYTES)
    return fail(QWHA_ERR_WORKSPACE,
                "qwha_coef_grad_noalloc: %zu bytes of partial sums needed, the static scratch holds %u; "
                "use qwha_adapter_bwd with a caller workspace",
                need, (unsigned)QWHA_NOALLOC_SCRATCH_BYTES);
  void *scratch = nullptr;
  qwha_status st = scratch_address(&scratch);
  if (st != QWHA_OK) return st;
  return cuda_status(launch_sddmm(dt, dY, Z, T, a->d_out, a->d_in, a->tile_ptr, a->tile_pos, a->tile_rk, a->p, alpha,
                                  static_cast<float *>(scratch), dc, (cudaStream_t)stream),
                     "coefficient gradient (static scratch)");
}
