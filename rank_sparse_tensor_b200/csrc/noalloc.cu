// Top-k selection with scratch in a fixed device array (no allocation).
//
// For callers that hold only their input and output buffers and cannot
// allocate device memory. The selection is the one of tgd_topk_select; its
// scratch space (digit histograms, selection state, per-block counts) lives
// in `g_topk_scratch` below instead of a caller workspace.

#include <string>

#include "common.cuh"
#include "kernels.h"

namespace {

// One copy per device, allocated with the module and kept until exit.
static __device__ __align__(256) unsigned char g_topk_scratch[TGD_TOPK_STATIC_SCRATCH_BYTES];

tgd_status fail(tgd_status st, const std::string& msg) {
  tgd::set_global_error(msg);
  return st;
}

}  // namespace

extern "C" tgd_status tgd_topk_select_static(const void* grad, tgd_dtype dtype, int64_t n, int64_t k,
                                             int64_t* omega_out, float* val_out, void* stream) {
  if (dtype < TGD_R32 || dtype > TGD_R16) return fail(TGD_ERR_INVALID_ARG, "unknown dtype");
  if (n < 0 || k < 0 || k > n) return fail(TGD_ERR_INVALID_ARG, "need 0 <= k <= n");
  if (n > TGD_TOPK_STATIC_MAX_N)
    return fail(TGD_ERR_INVALID_ARG, "n exceeds TGD_TOPK_STATIC_MAX_N (" +
                                         std::to_string((long long)TGD_TOPK_STATIC_MAX_N) +
                                         "), the size the fixed scratch array supports");
  if (tgd::select_workspace_bytes(n) > TGD_TOPK_STATIC_SCRATCH_BYTES)
    return fail(TGD_ERR_INVALID_ARG, "scratch array too small for n");
  if (k == 0) return TGD_OK;
  if (!grad || !omega_out) return fail(TGD_ERR_INVALID_ARG, "grad or omega_out is NULL");
  // The array's device address in the current device's context, looked up
  // on every call (a host-side query): nothing stale survives a device reset
  // or a change of the current device.
  void* ws = nullptr;
  cudaError_t e = cudaGetSymbolAddress(&ws, g_topk_scratch);
  if (e != cudaSuccess || !ws)
    return fail(TGD_ERR_CUDA, std::string("cudaGetSymbolAddress: ") + cudaGetErrorString(e));
  // The selection clears its histograms and initialises its state on the
  // stream before use, so the array's previous contents do not matter.
  e = tgd::select_topk(grad, dtype, n, k, omega_out, val_out, ws, (cudaStream_t)stream);
  if (e != cudaSuccess) return fail(TGD_ERR_CUDA, std::string("tgd_topk_select_static: ") + cudaGetErrorString(e));
  return TGD_OK;
}
