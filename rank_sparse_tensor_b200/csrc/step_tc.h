// Tensor-core (tcgen05) path of the TensorGRaD step for complex fp16 tensors.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

namespace tgd {

struct AdamConst;

typedef bool (*AllocFn)(void* ctx, void** p, size_t bytes);
// Called before (phase 0) and after (phase 1) each kernel launch, for timing.
typedef void (*TimerHook)(void* ctx, int phase, const char* name, cudaStream_t s);

// Geometry and device buffers of the tensor-core path (see step_tc.cu).
struct TcPlan {
  int d = 0;
  int64_t I[8] = {}, r[8] = {};
  int64_t N = 0, k = 0, ncore = 0;
  int gdt = 0, wdt = 0;
  int sm_budget = 0;  // > 0: the persistent kernels use at most this many CTAs
  uint64_t wait_ns = 0;      // limit of each projection wait; 0: the default (2 s)
  int skip_first_copy = 0;   // test only: the projection's CTA 0 skips its first tile copy
  bool ready = false;
  void* impl = nullptr;  // owned by step_tc.cu (host-side description)
};

// proj_mask: bit n set = mode n is projected (normally ranks[n] < shape[n];
// a mode-0 shard of a split tensor is projected even when r_0 >= its rows).
bool tc_supported(int nd, const int64_t* shape, const int64_t* ranks, uint32_t proj_mask, int gdt, int wdt);
bool tc_plan(TcPlan& p, int nd, const int64_t* shape, const int64_t* ranks, uint32_t proj_mask, int64_t k,
             int gdt, int wdt, AllocFn alloc, void* ctx);
void tc_release(TcPlan& p);
cudaError_t tc_rebuild(TcPlan& p, const int64_t* omega, int64_t k, const float* const* U,
                       cudaStream_t s);
cudaError_t tc_step(TcPlan& p, const void* g, void* w, float* sp_m, float* sp_v, float* core_m,
                    float* core_v, const AdamConst& asp, const AdamConst& acore, float decay,
                    float lr, int* d_err, cudaStream_t s, TimerHook hook, void* hook_ctx);
// The step in two halves: the sparse AdamW and the projection into the core
// buffer (tc_core, fp32 (re, im) pairs in this path's layout), then the core
// AdamW, the expansion and the weight update.
cudaError_t tc_step_project(TcPlan& p, const void* grad, float* sp_m, float* sp_v, const AdamConst& asp,
                            int* d_err, cudaStream_t s, TimerHook hook, void* hook_ctx);
// recon false: stop before the reconstruction stream (run it with tc_recon).
cudaError_t tc_step_finish(TcPlan& p, void* w, float* core_m, float* core_v, const AdamConst& acore,
                           float decay, float lr, int* d_err, cudaStream_t s, TimerHook hook,
                           void* hook_ctx, bool recon = true);
// The reconstruction stream alone, over tiles [tile0, tile0 + tiles) of the
// weights (tile_elems elements each, the last one possibly partial), after
// tc_step_finish's earlier stages; tc_step_finish runs it over all tiles.
cudaError_t tc_recon(TcPlan& p, void* w, int64_t tile0, int64_t tiles, float decay, float lr, int* d_err,
                     cudaStream_t s, TimerHook hook, void* hook_ctx);
int64_t tc_tiles(TcPlan& p);
int64_t tc_tile_elems(TcPlan& p);
float* tc_core(TcPlan& p);
// Core moments are stored in the path's internal layout; these convert
// to/from the canonical row-major r_1 x ... x r_d layout (host buffers).
cudaError_t tc_core_to_canonical(const TcPlan& p, const float* dev, int comps, float* host_out);
cudaError_t tc_core_from_canonical(const TcPlan& p, const float* host_in, int comps, float* dev);

}  // namespace tgd
