// Tensor-core (tcgen05) path of the TensorGRaD step for fp32 gradients and
// weights (real fp32, complex64).
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "step_tc.h"

namespace tgd {

struct Tc32Plan {
  bool ready = false;
  void* impl = nullptr;  // owned by step_tc32.cu
};

// fp32 gradients and weights of one kind (both real or both complex), at least
// one projected mode, projected modes of at most 256 entries.
// proj_mask: bit n set = mode n is projected (see tc_supported).
bool tc32_supported(int nd, const int64_t* shape, const int64_t* ranks, uint32_t proj_mask, int gdt, int wdt);
bool tc32_plan(Tc32Plan& p, int nd, const int64_t* shape, const int64_t* ranks, uint32_t proj_mask, int64_t k,
               int gdt, AllocFn alloc, void* ctx);
void tc32_release(Tc32Plan& p);
// Omega's per-word ranks and the factor images (after every refresh).
cudaError_t tc32_rebuild(Tc32Plan& p, const int64_t* omega, int64_t k, const float* const* U,
                         cudaStream_t s);
// The core buffer (canonical row-major r_1 x ... x r_d, fp32 (re, im) pairs
// for complex) and the buffer the sparse AdamW writes lambda S~ into.
float* tc32_core(Tc32Plan& p);
float* tc32_sparse_update(Tc32Plan& p);
// C = R x_n U_n^H into the core buffer (R = G with Omega zeroed by `bits`).
cudaError_t tc32_project(Tc32Plan& p, const void* grad, const uint32_t* bits, int* d_err, cudaStream_t s,
                         TimerHook hook, void* hook_ctx);
// Delta = C~ x_n U_n, lambda S~ added on Omega, W <- W decay - lr Delta.
cudaError_t tc32_expand_update(Tc32Plan& p, void* w, const uint32_t* bits, float decay, float lr, int* d_err,
                               cudaStream_t s, TimerHook hook, void* hook_ctx);

}  // namespace tgd
