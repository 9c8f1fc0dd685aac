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
// address is looked up with cudaGetSymbolAddress, once per device, on the
// first call made with that device current. That first call must therefore
// come before any stream capture.

#include <mutex>

#include "common.cuh"
#include "kernels.h"

namespace qwha {
namespace {

static __device__ __align__(256) unsigned char g_noalloc_scratch[QWHA_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
void *g_addr[kMaxDevices] = {nullptr};

// Device address of the scratch array for the current device (set-up on first use).
qwha_status scratch_address(void **out) {
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_status(e, "cudaGetDevice");
  if (dev < 0 || dev >= kMaxDevices) return fail(QWHA_ERR_UNSUPPORTED, "device ordinal %d", dev);
  std::lock_guard<std::mutex> g(g_mu);
  if (!g_addr[dev]) {
    void *p = nullptr;
    e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess) return cuda_status(e, "cudaGetSymbolAddress(scratch)");
    g_addr[dev] = p;
  }
  *out = g_addr[dev];
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
