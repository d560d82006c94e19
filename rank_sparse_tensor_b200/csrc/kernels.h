// Host-side launchers shared between the library's translation units.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include <string>

#include "../../include/tgd.h"

namespace tgd {

struct AdamConst;

// Sets the message tgd_last_error(NULL) returns.
void set_global_error(const std::string& msg);

// ---- select.cu: Omega selection and index structures
size_t select_workspace_bytes(int64_t n);
cudaError_t select_topk(const void* g, int dt, int64_t n, int64_t k, int64_t* out_idx,
                        float* out_val, void* ws, cudaStream_t s);
cudaError_t select_random(uint64_t seed, uint64_t ordinal, const void* g, int dt, int64_t n,
                          int64_t k, int64_t* out_idx, float* out_val, void* ws,
                          cudaStream_t s);
cudaError_t build_mask_bits(const int64_t* omega, int64_t k, int64_t n, uint32_t* bits,
                            cudaStream_t s);
cudaError_t build_tile_index(const int64_t* omega, int64_t k, int64_t tile_elems,
                             int64_t n_tiles, int64_t* tile_off, uint16_t* loc, cudaStream_t s);

// ---- gram_eig.cu: refresh of the factors
// Gram of mode n of the masked gradient (shape dims[0..nd), storage dtype dt,
// Omega bitmask `bits`), accumulated in fp32 partials and summed in fp64
// into gram (I_n x I_n complex, interleaved doubles).
size_t gram_partial_bytes(int nd, const int64_t* dims, int n);
// Modes with I_n <= 128 run on the tensor cores; err is the device error word
// a bounded wait sets when it gives up. max_ctas > 0 caps the tensor-core
// Gram's CTAs (one per SM), leaving SMs free for work on another stream.
cudaError_t mode_gram(const void* g, int dt, const uint32_t* bits, int nd, const int64_t* dims,
                      int n, float* partial, double* gram, int* err, cudaStream_t s, int max_ctas = 0);

struct EigJob {
  const double* gram;  // n x n complex (interleaved doubles)
  double* work;        // eig_work_doubles(n) doubles of global scratch
  float* U;            // out: n x r complex fp32, row-major
  double* evals;       // out: n eigenvalues, descending
  double* vprev;       // n x n complex: a unitary basis to start from (rows = vectors), and
                       // out: the eigenvectors found (n <= 128; any order)
  int n, r;
  int warm;            // 1: start from vprev, 0: from the identity
};
// The jobs of one batched launch, passed to the kernel by value (no copy
// from host memory on the stream).
struct EigJobs {
  EigJob j[TGD_MAX_NDIM];
};
size_t eig_work_doubles(int n);
cudaError_t batched_eigh(const EigJob* jobs_host, int njobs, cudaStream_t s);
// DCT basis instead of eigenvectors: U = the r columns of the orthonormal DCT
// matrix most aligned with the Gram (evals: the alignments, descending).
cudaError_t batched_dct_select(const EigJob* jobs_host, int njobs, cudaStream_t s);

// ---- step_generic.cu: CUDA-core path of the step
// L (optional, fp32 like the chain buffers): Adam on G[Omega] - L[Omega].
cudaError_t sparse_adam(const void* g, int dt, const int64_t* omega, int64_t k, float* m,
                        float* v, const AdamConst& a, float* upd, cudaStream_t s,
                        const float* L = nullptr);
// L <- G - L over n elements (fp32; float2 for complex dtypes).
cudaError_t residual_in_place(const void* g, int dt, float* L, int64_t n, cudaStream_t s);
// Y = X x_n M: X (A, K, B), M (J x K) row-major complex or real, Y (A, J, B).
// src_dt >= 0: X is the storage-typed gradient, masked by `bits`; src_dt < 0:
// X is fp32 (float2 when cplx).
cudaError_t mode_product(const void* X, int src_dt, const uint32_t* bits, bool cplx, int64_t A,
                         int64_t K, int64_t B, const float* M, int64_t J, float* Y,
                         cudaStream_t s);
cudaError_t masked_copy(const void* g, int dt, const uint32_t* bits, int64_t n, float* out,
                        cudaStream_t s);
cudaError_t core_adam(float* c, int64_t n, float* m, float* v, const AdamConst& a,
                      cudaStream_t s);
cudaError_t scatter_add(float* L, bool cplx, const int64_t* omega, int64_t k, const float* upd,
                        cudaStream_t s);
cudaError_t weight_update(void* w, int dt, const float* L, int64_t n, float decay, float lr,
                          cudaStream_t s);
// Projection (r x I, conj(U)^T) and expansion (I x r, U) coefficient matrices
// from U (I x r, complex fp32); real tensors get real matrices.
cudaError_t coef_matrices(const float* U, int64_t I, int64_t r, bool cplx, float* P, float* E,
                          cudaStream_t s);

}  // namespace tgd
