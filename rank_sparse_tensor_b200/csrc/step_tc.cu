// Tensor-core (tcgen05) path: placeholder until the kernels land.
#include "common.cuh"
#include "step_tc.h"

namespace tgd {

bool tc_supported(int, const int64_t*, const int64_t*, int, int) { return false; }
bool tc_plan(TcPlan&, int, const int64_t*, const int64_t*, int64_t, int, int, AllocFn, void*) {
  return false;
}
void tc_release(TcPlan&) {}
cudaError_t tc_rebuild(TcPlan&, const int64_t*, int64_t, const float* const*, cudaStream_t) {
  return cudaErrorNotSupported;
}
cudaError_t tc_step(TcPlan&, const void*, void*, float*, float*, float*, float*, const AdamConst&,
                    const AdamConst&, float, float, int*, cudaStream_t) {
  return cudaErrorNotSupported;
}
cudaError_t tc_core_to_canonical(const TcPlan&, const float*, int, float*) {
  return cudaErrorNotSupported;
}
cudaError_t tc_core_from_canonical(const TcPlan&, const float*, int, float*) {
  return cudaErrorNotSupported;
}

}  // namespace tgd
