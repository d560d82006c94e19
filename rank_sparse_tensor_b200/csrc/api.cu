// Host runtime behind include/tgd.h: argument checks, state ownership, the
// refresh schedule and the launch sequence of one TensorGRaD step.
//
// Schedule (nullthought.net TensorGRaD summary, section 三; Pith review, "What
// carries the argument"): the index set Omega and the factors U_n are
// re-selected every T steps and reused in between; here a refresh runs before
// the step whenever auto-refresh is on, T > 0 and t % T == 0 (t counts steps
// since create), on that step's gradient. Adam bias correction uses s = t + 1.

#include <algorithm>
#include <cmath>
#include <cstring>
#include <new>
#include <string>
#include <vector>

#include "common.cuh"
#include "kernels.h"
#include "step_tc.h"
#include "step_tc32.h"

using namespace tgd;

struct tgd_ctx {
  int d = 0;
  int64_t I[TGD_MAX_NDIM] = {}, r[TGD_MAX_NDIM] = {};
  int64_t N = 0, k = 0, ncore = 0;
  int gdt = 0, wdt = 0;
  bool cplx = false;
  int mc = 1, vc = 1;
  float lr = 0, b1 = 0, b2 = 0, eps = 0, wd = 0;
  double rho = 0;
  int64_t T = 0;
  tgd_options opt{};
  int path = TGD_PATH_GENERIC;
  uint32_t proj = 0;          // bit n: mode n is projected
  int64_t mode0_total = 0;    // > 0: this handle holds a block of rows of mode 0
  bool pending = false;       // tgd_step_begin has run, tgd_step_end has not
  float* core_ptr = nullptr;  // the core buffer of the step in progress (generic path)
  int64_t t = 0, refreshes = 0;
  bool has_subspace = false;
  int device = 0;
  // state
  int64_t* omega = nullptr;
  float* omega_val = nullptr;
  float* U[TGD_MAX_NDIM] = {};
  float* core_m = nullptr;
  float* core_v = nullptr;
  float* sp_m = nullptr;
  float* sp_v = nullptr;
  uint32_t* bits = nullptr;
  // refresh scratch
  void* sel_ws = nullptr;
  float* gram_part = nullptr;
  double* gram[TGD_MAX_NDIM] = {};
  double* evals[TGD_MAX_NDIM] = {};
  double* eig_work[TGD_MAX_NDIM] = {};
  double* eig_v[TGD_MAX_NDIM] = {};  // each mode's eigenvectors of the last refresh
  bool eig_warm = false;             // eig_v holds them (every projected mode <= 128)
  std::vector<EigJob> jobs;
  // the refresh runs each mode's eigensolve on one of two side streams beside
  // the next modes' Grams (fork and join by events)
  cudaStream_t side[2] = {};
  cudaEvent_t ev_fork = nullptr, ev_join[2] = {};
  int num_sms = 0;
  // generic step scratch
  float* P[TGD_MAX_NDIM] = {};  // projection coefficients (r x I)
  float* E[TGD_MAX_NDIM] = {};  // expansion coefficients (I x r)
  float* bufA = nullptr;
  float* bufB = nullptr;
  float* sp_upd = nullptr;
  float* core_buf = nullptr;  // low-rank-first order: the core kept across the L rebuild
  // tensor-core paths: complex fp16 gradients (tc), fp32 gradients (tc32)
  TcPlan tc;
  Tc32Plan tc32;
  bool use_tc32 = false;
  // errors
  int* d_err = nullptr;
  // host-buffer step
  void* stage_g = nullptr;
  void* stage_w = nullptr;
  // the tensor-core path's host-buffer step moves the weights in chunks of
  // tiles on two copy streams (in, out), overlapped with the reconstruction
  cudaStream_t cin = nullptr, cout = nullptr;
  cudaEvent_t hev[2 * 8 + 2] = {};
  std::vector<void*> allocs;
  size_t bytes = 0;
  std::string last_error;
  // per-kernel timing
  bool prof_on = false;
  std::vector<cudaEvent_t> ev_pool;
  size_t ev_used = 0;
  std::vector<std::pair<std::string, std::pair<cudaEvent_t, cudaEvent_t>>> prof;
  cudaEvent_t hook_start = nullptr;
};

namespace {

thread_local std::string g_last_error;

cudaEvent_t next_event(tgd_ctx* h) {
  if (h->ev_used == h->ev_pool.size()) {
    cudaEvent_t e;
    if (cudaEventCreate(&e) != cudaSuccess) return nullptr;
    h->ev_pool.push_back(e);
  }
  return h->ev_pool[h->ev_used++];
}

// Brackets one launch with events on its stream when timing is on.
struct KTimer {
  tgd_ctx* h;
  cudaStream_t s;
  const char* name;
  cudaEvent_t a = nullptr;
  KTimer(tgd_ctx* h_, cudaStream_t s_, const char* n) : h(h_), s(s_), name(n) {
    if (h->prof_on && (a = next_event(h))) cudaEventRecord(a, s);
  }
  ~KTimer() {
    if (!a) return;
    cudaEvent_t b = next_event(h);
    if (!b) return;
    cudaEventRecord(b, s);
    h->prof.push_back({name, {a, b}});
  }
};
// Timing hook for launch sequences that live in other translation units.
void timer_hook(void* ctx, int phase, const char* name, cudaStream_t s) {
  tgd_ctx* h = (tgd_ctx*)ctx;
  if (!h->prof_on) return;
  if (phase == 0) {
    h->hook_start = next_event(h);
    if (h->hook_start) cudaEventRecord(h->hook_start, s);
  } else if (h->hook_start) {
    cudaEvent_t b = next_event(h);
    if (b) {
      cudaEventRecord(b, s);
      h->prof.push_back({name, {h->hook_start, b}});
    }
    h->hook_start = nullptr;
  }
}

#define TGD_CAT2(a, b) a##b
#define TGD_CAT(a, b) TGD_CAT2(a, b)
#define TIMED(h, s, name) KTimer TGD_CAT(kt_, __LINE__)((h), (s), (name))

size_t dt_bytes(int dt) {
  switch (dt) {
    case TGD_R32: return 4;
    case TGD_C64: return 8;
    case TGD_C32H: return 4;
    case TGD_R16: return 2;
  }
  return 0;
}
bool dt_valid(int dt) { return dt >= TGD_R32 && dt <= TGD_R16; }
bool dt_cplx(int dt) { return dt == TGD_C64 || dt == TGD_C32H; }

tgd_status fail(tgd_ctx* h, tgd_status st, const std::string& msg) {
  if (h)
    h->last_error = msg;
  else
    g_last_error = msg;
  return st;
}

tgd_status cuda_fail(tgd_ctx* h, cudaError_t e, const char* where) {
  return fail(h, TGD_ERR_CUDA, std::string(where) + ": " + cudaGetErrorString(e));
}

#define TGD_CUDA(h, call)                                   \
  do {                                                      \
    cudaError_t e_ = (call);                                \
    if (e_ != cudaSuccess) return cuda_fail((h), e_, #call); \
  } while (0)

bool dalloc(tgd_ctx* h, void** p, size_t bytes) {
  *p = nullptr;
  if (bytes == 0) return true;
  bytes = (bytes + 255) & ~(size_t)255;
  if (cudaMalloc(p, bytes) != cudaSuccess) {
    *p = nullptr;
    cudaGetLastError();
    return false;
  }
  h->allocs.push_back(*p);
  h->bytes += bytes;
  return true;
}

template <class T>
bool dalloc_t(tgd_ctx* h, T** p, size_t count) {
  return dalloc(h, (void**)p, count * sizeof(T));
}

void free_all(tgd_ctx* h) {
  tc_release(h->tc);
  tc32_release(h->tc32);
  if (h->ev_fork) cudaEventDestroy(h->ev_fork);
  h->ev_fork = nullptr;
  for (cudaEvent_t& e : h->hev) {
    if (e) cudaEventDestroy(e);
    e = nullptr;
  }
  if (h->cin) cudaStreamDestroy(h->cin);
  if (h->cout) cudaStreamDestroy(h->cout);
  h->cin = h->cout = nullptr;
  for (int i = 0; i < 2; ++i) {
    if (h->ev_join[i]) cudaEventDestroy(h->ev_join[i]);
    if (h->side[i]) cudaStreamDestroy(h->side[i]);
    h->ev_join[i] = nullptr;
    h->side[i] = nullptr;
  }
  for (cudaEvent_t e : h->ev_pool) cudaEventDestroy(e);
  h->ev_pool.clear();
  for (void* p : h->allocs) cudaFree(p);
  h->allocs.clear();
}

AdamConst adam_const(const tgd_ctx* h, double scale) {
  double s = (double)(h->t + 1);
  double bc1 = 1.0 - std::pow((double)h->b1, s), bc2 = 1.0 - std::pow((double)h->b2, s);
  AdamConst a;
  a.b1 = h->b1;
  a.b2 = h->b2;
  a.omb1 = (float)(1.0 - (double)h->b1);
  a.omb2 = (float)(1.0 - (double)h->b2);
  a.inv_bc1 = (float)(1.0 / bc1);
  a.inv_bc2 = (float)(1.0 / bc2);
  a.eps = h->eps;
  a.scale = (float)scale;
  a.cplx = h->cplx ? 1 : 0;
  a.cmode = h->opt.complex_adam;
  return a;
}

bool mode_active(const tgd_ctx* h, int n) { return ((h->proj >> n) & 1u) != 0; }

// The block eigensolver (every projected mode of at most 128 entries) keeps
// each mode's eigenvectors, and the next refresh starts from them.
bool eig_keeps_vectors(const tgd_ctx* h) {
  for (int n = 0; n < h->d; ++n)
    if (mode_active(h, n) && h->I[n] > 128) return false;
  return true;
}

// Derived device data that depends on Omega and U: the Omega bitmask, the
// coefficient matrices of the generic path and the tensor-core operands.
tgd_status rebuild_derived(tgd_ctx* h, cudaStream_t s) {
  TGD_CUDA(h, build_mask_bits(h->omega, h->k, h->N, h->bits, s));
  if (h->path == TGD_PATH_GENERIC) {
    for (int n = 0; n < h->d; ++n)
      if (mode_active(h, n)) TGD_CUDA(h, coef_matrices(h->U[n], h->I[n], h->r[n], h->cplx, h->P[n], h->E[n], s));
  } else if (h->use_tc32) {
    TGD_CUDA(h, tc32_rebuild(h->tc32, h->omega, h->k, (const float* const*)h->U, s));
  } else {
    TGD_CUDA(h, tc_rebuild(h->tc, h->omega, h->k, (const float* const*)h->U, s));
  }
  return TGD_OK;
}

// The fp32 tensor-core step: sparse AdamW into lambda S~, the projection
// chain into the core, core AdamW in place, the expansion chain whose last
// product updates the weights with lambda S~ added on Omega.
tgd_status tc32_begin(tgd_ctx* h, const void* g, cudaStream_t s) {
  AdamConst asp = adam_const(h, h->opt.sparse_scale);
  {
    TIMED(h, s, "sparse_adam");
    TGD_CUDA(h, sparse_adam(g, h->gdt, h->omega, h->k, h->sp_m, h->sp_v, asp, tc32_sparse_update(h->tc32), s));
  }
  TGD_CUDA(h, tc32_project(h->tc32, g, h->bits, h->d_err, s, timer_hook, h));
  return TGD_OK;
}

tgd_status tc32_end(tgd_ctx* h, void* w, cudaStream_t s) {
  AdamConst acore = adam_const(h, 1.0);
  {
    TIMED(h, s, "core_adam");
    TGD_CUDA(h, core_adam(tc32_core(h->tc32), h->ncore, h->core_m, h->core_v, acore, s));
  }
  const float decay = (float)(1.0 - (double)h->lr * (double)h->wd);
  TGD_CUDA(h, tc32_expand_update(h->tc32, w, h->bits, decay, h->lr, h->d_err, s, timer_hook, h));
  return TGD_OK;
}

// ------------------------------------------------ low-rank-first order
// The decomposition order reversed (the method's free parameter "decomposition
// order" in the Pith review; sparse-first is the chosen order): the low-rank
// part of the whole gradient comes first and Omega is selected on what it
// leaves. CUDA-core kernels only.

float* other_buf(tgd_ctx* h, const float* c) { return c == h->bufA ? h->bufB : h->bufA; }

// C = G x_n U_n^H over the projected modes (last mode first), read from the
// storage-typed gradient without a mask; *out is the buffer holding C (G
// itself, copied to fp32, when no mode is projected). dims follows the shape.
tgd_status project_all(tgd_ctx* h, const void* g, int64_t* dims, float** out, cudaStream_t s) {
  float* cur = nullptr;
  for (int n = h->d - 1; n >= 0; --n) {
    if (!mode_active(h, n)) continue;
    int64_t A = 1, B = 1;
    for (int q = 0; q < n; ++q) A *= dims[q];
    for (int q = n + 1; q < h->d; ++q) B *= dims[q];
    float* o = other_buf(h, cur);
    TIMED(h, s, "mode_product");
    if (cur == nullptr)
      TGD_CUDA(h, mode_product(g, h->gdt, nullptr, h->cplx, A, dims[n], B, h->P[n], h->r[n], o, s));
    else
      TGD_CUDA(h, mode_product(cur, -1, nullptr, h->cplx, A, dims[n], B, h->P[n], h->r[n], o, s));
    cur = o;
    dims[n] = h->r[n];
  }
  if (cur == nullptr) {
    TIMED(h, s, "masked_copy");
    TGD_CUDA(h, masked_copy(g, h->gdt, nullptr, h->N, h->bufA, s));
    cur = h->bufA;
  }
  *out = cur;
  return TGD_OK;
}

// X x_n U_n over the projected modes, from src (never written); *out holds the
// result (src itself when no mode is projected).
tgd_status expand_all(tgd_ctx* h, float* src, int64_t* dims, float** out, cudaStream_t s) {
  float* cur = src;
  for (int n = 0; n < h->d; ++n) {
    if (!mode_active(h, n)) continue;
    int64_t A = 1, B = 1;
    for (int q = 0; q < n; ++q) A *= dims[q];
    for (int q = n + 1; q < h->d; ++q) B *= dims[q];
    float* o = other_buf(h, cur);
    TIMED(h, s, "mode_product");
    TGD_CUDA(h, mode_product(cur, -1, nullptr, h->cplx, A, dims[n], B, h->E[n], h->I[n], o, s));
    cur = o;
    dims[n] = h->I[n];
  }
  *out = cur;
  return TGD_OK;
}

// Refresh: U_n from the Grams of G itself, L = G x_n U_n U_n^H, Omega = top-k
// (or the random draw) of E = G - L in fp32; Omega's values are E there.
tgd_status do_refresh_lowrank_first(tgd_ctx* h, const void* g, cudaStream_t s) {
  h->jobs.clear();
  for (int n = 0; n < h->d; ++n) {
    if (!mode_active(h, n)) continue;
    TIMED(h, s, "mode_gram");
    TGD_CUDA(h, mode_gram(g, h->gdt, nullptr, h->d, h->I, n, h->gram_part, h->gram[n], h->d_err, s));
    EigJob j;
    j.gram = h->gram[n];
    j.work = h->eig_work[n];
    j.U = h->U[n];
    j.evals = h->evals[n];
    j.vprev = h->eig_v[n];
    j.warm = h->eig_warm ? 1 : 0;
    j.n = (int)h->I[n];
    j.r = (int)h->r[n];
    h->jobs.push_back(j);
  }
  {
    TIMED(h, s, "eigh");
    TGD_CUDA(h, batched_eigh(h->jobs.data(), (int)h->jobs.size(), s));
    h->eig_warm = eig_keeps_vectors(h);
  }
  for (int n = 0; n < h->d; ++n)
    if (mode_active(h, n)) TGD_CUDA(h, coef_matrices(h->U[n], h->I[n], h->r[n], h->cplx, h->P[n], h->E[n], s));
  int64_t dims[TGD_MAX_NDIM];
  for (int n = 0; n < h->d; ++n) dims[n] = h->I[n];
  float *C = nullptr, *L = nullptr;
  tgd_status st = project_all(h, g, dims, &C, s);
  if (st != TGD_OK) return st;
  st = expand_all(h, C, dims, &L, s);
  if (st != TGD_OK) return st;
  TGD_CUDA(h, residual_in_place(g, h->gdt, L, h->N, s));
  const int edt = h->cplx ? TGD_C64 : TGD_R32;
  if (h->k > 0) {
    KTimer kt(h, s, "select");
    if (h->opt.omega_mode == 0)
      TGD_CUDA(h, select_topk(L, edt, h->N, h->k, h->omega, h->omega_val, h->sel_ws, s));
    else
      TGD_CUDA(h, select_random(h->opt.seed, (uint64_t)h->refreshes, L, edt, h->N, h->k, h->omega,
                                h->omega_val, h->sel_ws, s));
  }
  st = rebuild_derived(h, s);
  if (st != TGD_OK) return st;
  if (h->opt.moments_on_refresh == 1) {
    TGD_CUDA(h, cudaMemsetAsync(h->core_m, 0, sizeof(float) * h->ncore * h->mc, s));
    TGD_CUDA(h, cudaMemsetAsync(h->core_v, 0, sizeof(float) * h->ncore * h->vc, s));
    TGD_CUDA(h, cudaMemsetAsync(h->sp_m, 0, sizeof(float) * h->k * h->mc, s));
    TGD_CUDA(h, cudaMemsetAsync(h->sp_v, 0, sizeof(float) * h->k * h->vc, s));
  }
  h->has_subspace = true;
  h->refreshes += 1;
  return TGD_OK;
}

// Step: C = G x_n U_n^H (the whole gradient), L = C x_n U_n from the pre-Adam
// core, sparse Adam on E[Omega] = G[Omega] - L[Omega], core Adam, Delta =
// C~ x_n U_n with lambda S~ scattered in, the AdamW weight update.
tgd_status step_lowrank_first(tgd_ctx* h, const void* g, void* w, cudaStream_t s) {
  AdamConst asp = adam_const(h, h->opt.sparse_scale);
  AdamConst acore = adam_const(h, 1.0);
  int64_t dims[TGD_MAX_NDIM], ldims[TGD_MAX_NDIM];
  for (int n = 0; n < h->d; ++n) dims[n] = h->I[n];
  float *C = nullptr, *L = nullptr, *D = nullptr;
  tgd_status st = project_all(h, g, dims, &C, s);
  if (st != TGD_OK) return st;
  TGD_CUDA(h, cudaMemcpyAsync(h->core_buf, C, sizeof(float) * h->ncore * h->mc,
                              cudaMemcpyDeviceToDevice, s));
  for (int n = 0; n < h->d; ++n) ldims[n] = dims[n];
  st = expand_all(h, C, ldims, &L, s);
  if (st != TGD_OK) return st;
  {
    TIMED(h, s, "sparse_adam");
    TGD_CUDA(h, sparse_adam(g, h->gdt, h->omega, h->k, h->sp_m, h->sp_v, asp, h->sp_upd, s, L));
  }
  {
    TIMED(h, s, "core_adam");
    TGD_CUDA(h, core_adam(h->core_buf, h->ncore, h->core_m, h->core_v, acore, s));
  }
  st = expand_all(h, h->core_buf, dims, &D, s);
  if (st != TGD_OK) return st;
  {
    TIMED(h, s, "scatter_add");
    TGD_CUDA(h, scatter_add(D, h->cplx, h->omega, h->k, h->sp_upd, s));
  }
  float decay = (float)(1.0 - (double)h->lr * (double)h->wd);
  TIMED(h, s, "weight_update");
  TGD_CUDA(h, weight_update(w, h->wdt, D, h->N, decay, h->lr, s));
  return TGD_OK;
}

tgd_status do_refresh(tgd_ctx* h, const void* g, cudaStream_t s) {
  if (h->opt.order == 1) return do_refresh_lowrank_first(h, g, s);
  if (h->k > 0) {
    KTimer kt(h, s, "select");
    if (h->opt.omega_mode == 0)
      TGD_CUDA(h, select_topk(g, h->gdt, h->N, h->k, h->omega, h->omega_val, h->sel_ws, s));
    else
      TGD_CUDA(h, select_random(h->opt.seed, (uint64_t)h->refreshes, g, h->gdt, h->N, h->k,
                                h->omega, h->omega_val, h->sel_ws, s));
  }
  TGD_CUDA(h, build_mask_bits(h->omega, h->k, h->N, h->bits, s));
  h->jobs.clear();
  // Each mode's eigensolve (one CTA, latency-bound) starts on a side stream
  // (the two in turn) as soon as its Gram is done and runs beside the next
  // modes' Grams, which leave two SMs free for them; the main stream waits
  // for both. Not for a handle given an SM budget: it shares the GPU with
  // other streams.
  const bool overlap = h->opt.basis != 1 && h->side[1] && h->num_sms > 2 && h->opt.sm_budget == 0;
  int nside = 0;
  for (int n = 0; n < h->d; ++n) {
    if (!mode_active(h, n)) continue;
    {
      TIMED(h, s, "mode_gram");
      TGD_CUDA(h, mode_gram(g, h->gdt, h->bits, h->d, h->I, n, h->gram_part, h->gram[n], h->d_err, s,
                            overlap ? h->num_sms - 2 : 0));
    }
    EigJob j;
    j.gram = h->gram[n];
    j.work = h->eig_work[n];
    j.U = h->U[n];
    j.evals = h->evals[n];
    j.vprev = h->eig_v[n];
    j.warm = h->eig_warm ? 1 : 0;
    j.n = (int)h->I[n];
    j.r = (int)h->r[n];
    h->jobs.push_back(j);
    if (overlap) {
      cudaStream_t ss = h->side[nside & 1];
      ++nside;
      TGD_CUDA(h, cudaEventRecord(h->ev_fork, s));
      TGD_CUDA(h, cudaStreamWaitEvent(ss, h->ev_fork, 0));
      TIMED(h, ss, "eigh");
      TGD_CUDA(h, batched_eigh(&h->jobs.back(), 1, ss));
    }
  }
  if (overlap) {
    for (int i = 0; i < 2; ++i) {
      TGD_CUDA(h, cudaEventRecord(h->ev_join[i], h->side[i]));
      TGD_CUDA(h, cudaStreamWaitEvent(s, h->ev_join[i], 0));
    }
    h->eig_warm = eig_keeps_vectors(h);
  } else if (h->opt.basis == 1) {
    TIMED(h, s, "dct_select");
    TGD_CUDA(h, batched_dct_select(h->jobs.data(), (int)h->jobs.size(), s));
  } else {
    TIMED(h, s, "eigh");
    TGD_CUDA(h, batched_eigh(h->jobs.data(), (int)h->jobs.size(), s));
    h->eig_warm = eig_keeps_vectors(h);
  }
  tgd_status st = rebuild_derived(h, s);
  if (st != TGD_OK) return st;
  if (h->opt.moments_on_refresh == 1) {
    TGD_CUDA(h, cudaMemsetAsync(h->core_m, 0, sizeof(float) * h->ncore * h->mc, s));
    TGD_CUDA(h, cudaMemsetAsync(h->core_v, 0, sizeof(float) * h->ncore * h->vc, s));
    TGD_CUDA(h, cudaMemsetAsync(h->sp_m, 0, sizeof(float) * h->k * h->mc, s));
    TGD_CUDA(h, cudaMemsetAsync(h->sp_v, 0, sizeof(float) * h->k * h->vc, s));
  }
  h->has_subspace = true;
  h->refreshes += 1;
  return TGD_OK;
}

// The generic step, first half: sparse AdamW, then the projection chain; the
// core is left in h->core_ptr.
tgd_status generic_begin(tgd_ctx* h, const void* g, cudaStream_t s) {
  AdamConst asp = adam_const(h, h->opt.sparse_scale);
  {
    TIMED(h, s, "sparse_adam");
    TGD_CUDA(h, sparse_adam(g, h->gdt, h->omega, h->k, h->sp_m, h->sp_v, asp, h->sp_upd, s));
  }
  int64_t dims[TGD_MAX_NDIM];
  for (int n = 0; n < h->d; ++n) dims[n] = h->I[n];
  float* cur = nullptr;
  auto other = [&](float* c) { return c == h->bufA ? h->bufB : h->bufA; };
  for (int n = h->d - 1; n >= 0; --n) {
    if (!mode_active(h, n)) continue;
    int64_t A = 1, B = 1;
    for (int q = 0; q < n; ++q) A *= dims[q];
    for (int q = n + 1; q < h->d; ++q) B *= dims[q];
    float* out = other(cur);
    TIMED(h, s, "mode_product");
    if (cur == nullptr)
      TGD_CUDA(h, mode_product(g, h->gdt, h->bits, h->cplx, A, dims[n], B, h->P[n], h->r[n], out, s));
    else
      TGD_CUDA(h, mode_product(cur, -1, nullptr, h->cplx, A, dims[n], B, h->P[n], h->r[n], out, s));
    cur = out;
    dims[n] = h->r[n];
  }
  if (cur == nullptr) {
    TIMED(h, s, "masked_copy");
    TGD_CUDA(h, masked_copy(g, h->gdt, h->bits, h->N, h->bufA, s));
    cur = h->bufA;
  }
  h->core_ptr = cur;
  return TGD_OK;
}

// Second half: core AdamW, the expansion chain, the scatter of lambda S~ and
// the weight update.
tgd_status generic_end(tgd_ctx* h, void* w, cudaStream_t s) {
  AdamConst acore = adam_const(h, 1.0);
  float* cur = h->core_ptr;
  auto other = [&](float* c) { return c == h->bufA ? h->bufB : h->bufA; };
  {
    TIMED(h, s, "core_adam");
    TGD_CUDA(h, core_adam(cur, h->ncore, h->core_m, h->core_v, acore, s));
  }
  int64_t dims[TGD_MAX_NDIM];
  for (int n = 0; n < h->d; ++n) dims[n] = mode_active(h, n) ? h->r[n] : h->I[n];
  for (int n = 0; n < h->d; ++n) {
    if (!mode_active(h, n)) continue;
    int64_t A = 1, B = 1;
    for (int q = 0; q < n; ++q) A *= dims[q];
    for (int q = n + 1; q < h->d; ++q) B *= dims[q];
    float* out = other(cur);
    TIMED(h, s, "mode_product");
    TGD_CUDA(h, mode_product(cur, -1, nullptr, h->cplx, A, dims[n], B, h->E[n], h->I[n], out, s));
    cur = out;
    dims[n] = h->I[n];
  }
  {
    TIMED(h, s, "scatter_add");
    TGD_CUDA(h, scatter_add(cur, h->cplx, h->omega, h->k, h->sp_upd, s));
  }
  float decay = (float)(1.0 - (double)h->lr * (double)h->wd);
  TIMED(h, s, "weight_update");
  TGD_CUDA(h, weight_update(w, h->wdt, cur, h->N, decay, h->lr, s));
  return TGD_OK;
}

// The two halves on the handle's kernel path.
tgd_status step_begin(tgd_ctx* h, const void* g, cudaStream_t s) {
  tgd_status st = TGD_OK;
  if (h->path == TGD_PATH_GENERIC) {
    st = generic_begin(h, g, s);
  } else if (h->use_tc32) {
    st = tc32_begin(h, g, s);
  } else {
    AdamConst asp = adam_const(h, h->opt.sparse_scale);
    cudaError_t e = tc_step_project(h->tc, g, h->sp_m, h->sp_v, asp, h->d_err, s, timer_hook, h);
    if (e != cudaSuccess) st = cuda_fail(h, e, "tensor-core projection");
  }
  if (st == TGD_OK) h->pending = true;
  return st;
}

tgd_status step_end(tgd_ctx* h, void* w, cudaStream_t s) {
  tgd_status st = TGD_OK;
  if (h->path == TGD_PATH_GENERIC) {
    st = generic_end(h, w, s);
  } else if (h->use_tc32) {
    st = tc32_end(h, w, s);
  } else {
    AdamConst acore = adam_const(h, 1.0);
    float decay = (float)(1.0 - (double)h->lr * (double)h->wd);
    cudaError_t e = tc_step_finish(h->tc, w, h->core_m, h->core_v, acore, decay, h->lr, h->d_err, s, timer_hook, h);
    if (e != cudaSuccess) st = cuda_fail(h, e, "tensor-core reconstruction");
  }
  if (st != TGD_OK) return st;
  h->pending = false;
  h->t += 1;
  return TGD_OK;
}

// The core buffer between the halves: device pointer and float count.
float* core_buffer(tgd_ctx* h) {
  if (h->path == TGD_PATH_GENERIC) return h->core_ptr;
  return h->use_tc32 ? tc32_core(h->tc32) : tc_core(h->tc);
}

tgd_status check_device_error(tgd_ctx* h, cudaStream_t s, bool wait) {
  if (wait) TGD_CUDA(h, cudaStreamSynchronize(s));
  int v = 0;
  TGD_CUDA(h, cudaMemcpy(&v, h->d_err, sizeof(int), cudaMemcpyDeviceToHost));
  if (v != 0) {
    TGD_CUDA(h, cudaMemset(h->d_err, 0, sizeof(int)));
    return fail(h, TGD_ERR_TIMEOUT, "a device-side wait gave up (error bits " + std::to_string(v) + ")");
  }
  return TGD_OK;
}

// Identity factors for full-rank modes (U_n = I, R6 of the readings).
__global__ void identity_kernel(float2* U, int64_t n) {
  for (int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; e < n * n;
       e += (int64_t)gridDim.x * blockDim.x)
    U[e] = make_float2((e / n) == (e % n) ? 1.f : 0.f, 0.f);
}

}  // namespace

// Global (handle-less) error message, shared with other translation units.
void tgd::set_global_error(const std::string& msg) { g_last_error = msg; }

extern "C" {

void tgd_default_options(tgd_options* opt) {
  if (!opt) return;
  opt->omega_mode = 0;
  opt->seed = 0;
  opt->sparse_scale = 1.0f;
  opt->complex_adam = 0;
  opt->moments_on_refresh = 0;
  opt->auto_refresh = 1;
  opt->path = TGD_PATH_AUTO;
  opt->sm_budget = 0;
  opt->order = 0;
  opt->basis = 0;
  opt->wait_limit_ms = 0;
  opt->test_stall = 0;
  opt->sparse_k = -1;
  opt->mode0_total = 0;
}

tgd_status tgd_create(tgd_handle* out, int ndim, const int64_t* shape, const int64_t* ranks,
                      double sparse_ratio, int64_t T, float lr, float beta1, float beta2, float eps,
                      float wd, tgd_dtype grad_dtype, tgd_dtype weight_dtype,
                      const tgd_options* opt) {
  if (!out) return fail(nullptr, TGD_ERR_INVALID_ARG, "out is NULL");
  *out = nullptr;
  if (ndim < 2 || ndim > TGD_MAX_NDIM) return fail(nullptr, TGD_ERR_INVALID_ARG, "ndim must be in [2, 8]");
  if (!shape || !ranks) return fail(nullptr, TGD_ERR_INVALID_ARG, "shape or ranks is NULL");
  if (!dt_valid(grad_dtype) || !dt_valid(weight_dtype))
    return fail(nullptr, TGD_ERR_INVALID_ARG, "unknown dtype");
  if (dt_cplx(grad_dtype) != dt_cplx(weight_dtype))
    return fail(nullptr, TGD_ERR_INVALID_ARG, "grad and weight must both be real or both complex");
  if (!(sparse_ratio >= 0.0 && sparse_ratio <= 1.0))
    return fail(nullptr, TGD_ERR_INVALID_ARG, "sparse_ratio must be in [0, 1]");
  if (T < 0) return fail(nullptr, TGD_ERR_INVALID_ARG, "T must be >= 0");
  if (!(beta1 >= 0.f && beta1 < 1.f) || !(beta2 >= 0.f && beta2 < 1.f) || !(eps >= 0.f) ||
      !std::isfinite(lr) || !std::isfinite(wd))
    return fail(nullptr, TGD_ERR_INVALID_ARG, "bad AdamW hyper-parameter");
  tgd_options o;
  tgd_default_options(&o);
  if (opt) o = *opt;
  if (o.omega_mode < 0 || o.omega_mode > 1 || o.complex_adam < 0 || o.complex_adam > 1 ||
      o.moments_on_refresh < 0 || o.moments_on_refresh > 1 || o.path < 0 || o.path > 2 ||
      o.sm_budget < 0 || !std::isfinite(o.sparse_scale) || o.order < 0 || o.order > 1 ||
      o.basis < 0 || o.basis > 1 || o.wait_limit_ms < 0 || o.test_stall < 0 || o.test_stall > 1 ||
      o.sparse_k < -1 || o.mode0_total < 0)
    return fail(nullptr, TGD_ERR_INVALID_ARG, "bad option value");
  if (o.mode0_total > 0 && (o.order != 0 || (o.auto_refresh && T > 0)))
    return fail(nullptr, TGD_ERR_INVALID_ARG,
                "a block of mode-0 rows takes its factors and index set from tgd_set_state: "
                "set T = 0 or auto_refresh = 0, and the sparse-first order");
  if (o.order == 1 && o.path == TGD_PATH_TCGEN05)
    return fail(nullptr, TGD_ERR_UNSUPPORTED, "the low-rank-first order runs on the CUDA-core path");
  int64_t N = 1, ncore = 1;
  uint32_t proj = 0;
  for (int n = 0; n < ndim; ++n) {
    // a block of mode-0 rows: the mode's full size is mode0_total
    const int64_t full = (n == 0 && o.mode0_total > 0) ? o.mode0_total : shape[n];
    if (shape[n] < 1 || ranks[n] < 1 || ranks[n] > full || shape[n] > full)
      return fail(nullptr, TGD_ERR_INVALID_ARG, "need 1 <= ranks[n] <= shape[n] (mode 0 of a block: "
                                                "ranks[0], shape[0] <= mode0_total)");
    if (full > 256 && ranks[n] < full)
      return fail(nullptr, TGD_ERR_UNSUPPORTED, "projected modes are limited to 256 entries");
    if (N > ((int64_t)1 << 40) / shape[n]) return fail(nullptr, TGD_ERR_INVALID_ARG, "tensor too large");
    if (ranks[n] < full) proj |= 1u << n;
    N *= shape[n];
    ncore *= ranks[n];
  }
  if (o.sparse_k > N) return fail(nullptr, TGD_ERR_INVALID_ARG, "sparse_k exceeds the element count");
  tgd_ctx* h = new (std::nothrow) tgd_ctx;
  if (!h) return fail(nullptr, TGD_ERR_OOM, "host allocation failed");
  h->d = ndim;
  for (int n = 0; n < ndim; ++n) {
    h->I[n] = shape[n];
    h->r[n] = ranks[n];
  }
  h->N = N;
  h->ncore = ncore;
  h->rho = sparse_ratio;
  h->k = o.sparse_k >= 0 ? o.sparse_k : (int64_t)std::floor(sparse_ratio * (double)N);
  h->proj = proj;
  h->mode0_total = o.mode0_total;
  h->T = T;
  h->lr = lr;
  h->b1 = beta1;
  h->b2 = beta2;
  h->eps = eps;
  h->wd = wd;
  h->gdt = grad_dtype;
  h->wdt = weight_dtype;
  h->cplx = dt_cplx(grad_dtype);
  h->opt = o;
  h->mc = h->cplx ? 2 : 1;
  h->vc = (h->cplx && o.complex_adam == 1) ? 2 : 1;
  // Path: the tensor-core kernels need complex fp16 gradients and tiles that
  // fit the trailing two modes.
  const bool tc16_ok = tc_supported(ndim, shape, ranks, proj, grad_dtype, weight_dtype);
  const bool tc32_ok = tc32_supported(ndim, shape, ranks, proj, grad_dtype, weight_dtype);
  const bool tc_ok = tc16_ok || tc32_ok;
  if (o.path == TGD_PATH_TCGEN05 && !tc_ok) {
    delete h;
    return fail(nullptr, TGD_ERR_UNSUPPORTED, "tensor-core path: needs complex fp16 gradients with d >= 3, "
                                              "a power-of-two I_{d-1} <= 128, I_d <= 120 and ranks below the "
                                              "modes; or fp32 gradients and weights of one kind with a "
                                              "projected mode");
  }
  h->path = (o.path == TGD_PATH_GENERIC || !tc_ok || o.order == 1) ? TGD_PATH_GENERIC
                                                                    : TGD_PATH_TCGEN05;
  h->use_tc32 = h->path == TGD_PATH_TCGEN05 && !tc16_ok;
  cudaError_t ce = cudaGetDevice(&h->device);
  if (ce != cudaSuccess) {
    delete h;
    cudaGetLastError();
    return fail(nullptr, TGD_ERR_CUDA, std::string("no CUDA device: ") + cudaGetErrorString(ce));
  }
  bool ok = true;
  ok &= dalloc_t(h, &h->omega, std::max<int64_t>(h->k, 1));
  ok &= dalloc_t(h, &h->omega_val, std::max<int64_t>(h->k, 1) * h->mc);
  for (int n = 0; n < ndim; ++n) ok &= dalloc_t(h, &h->U[n], (size_t)shape[n] * ranks[n] * 2);
  ok &= dalloc_t(h, &h->core_m, ncore * h->mc);
  ok &= dalloc_t(h, &h->core_v, ncore * h->vc);
  ok &= dalloc_t(h, &h->sp_m, std::max<int64_t>(h->k, 1) * h->mc);
  ok &= dalloc_t(h, &h->sp_v, std::max<int64_t>(h->k, 1) * h->vc);
  ok &= dalloc_t(h, &h->bits, (size_t)ceil_div(N, 32));
  ok &= dalloc(h, &h->sel_ws, select_workspace_bytes(N));
  size_t gp = 0;
  for (int n = 0; n < ndim; ++n)
    if (ranks[n] < shape[n] && o.mode0_total == 0) {
      gp = std::max(gp, gram_partial_bytes(ndim, shape, n));
      ok &= dalloc_t(h, &h->gram[n], (size_t)shape[n] * shape[n] * 2);
      ok &= dalloc_t(h, &h->evals[n], (size_t)shape[n]);
      ok &= dalloc_t(h, &h->eig_work[n], eig_work_doubles((int)shape[n]));
      ok &= dalloc_t(h, &h->eig_v[n], (size_t)2 * shape[n] * shape[n]);
    }
  ok &= dalloc(h, (void**)&h->gram_part, gp);
  ok &= dalloc_t(h, &h->d_err, 1);
  if (ok && h->path == TGD_PATH_GENERIC) {
    for (int n = 0; n < ndim; ++n)
      if ((proj >> n) & 1u) {
        ok &= dalloc_t(h, &h->P[n], (size_t)shape[n] * ranks[n] * h->mc);
        ok &= dalloc_t(h, &h->E[n], (size_t)shape[n] * ranks[n] * h->mc);
      }
    ok &= dalloc_t(h, &h->bufA, (size_t)N * h->mc);
    ok &= dalloc_t(h, &h->bufB, (size_t)N * h->mc);
    ok &= dalloc_t(h, &h->sp_upd, std::max<int64_t>(h->k, 1) * h->mc);
    if (o.order == 1) ok &= dalloc_t(h, &h->core_buf, ncore * h->mc);
  }
  if (ok && h->use_tc32) {
    auto alloc_fn = [](void* ctx, void** p, size_t b) { return dalloc((tgd_ctx*)ctx, p, b); };
    ok &= tc32_plan(h->tc32, ndim, shape, ranks, proj, h->k, grad_dtype, alloc_fn, h);
  }
  if (ok && h->path == TGD_PATH_TCGEN05 && !h->use_tc32) {
    auto alloc_fn = [](void* ctx, void** p, size_t b) { return dalloc((tgd_ctx*)ctx, p, b); };
    h->tc.sm_budget = o.sm_budget;
    h->tc.wait_ns = (uint64_t)o.wait_limit_ms * 1000000ull;
    h->tc.skip_first_copy = o.test_stall;
    ok &= tc_plan(h->tc, ndim, shape, ranks, proj, h->k, grad_dtype, weight_dtype, alloc_fn, h);
  }
  if (!ok) {
    free_all(h);
    delete h;
    return fail(nullptr, TGD_ERR_OOM, "device allocation failed");
  }
  {
    // the refresh's side streams (see do_refresh); without them the refresh
    // runs on the caller's stream alone
    bool have = false;
    for (int n = 0; n < ndim; ++n) have |= h->gram[n] != nullptr;
    bool made = have && cudaDeviceGetAttribute(&h->num_sms, cudaDevAttrMultiProcessorCount, h->device) == cudaSuccess &&
                cudaEventCreateWithFlags(&h->ev_fork, cudaEventDisableTiming) == cudaSuccess;
    for (int i = 0; i < 2; ++i)
      made = made && cudaStreamCreateWithFlags(&h->side[i], cudaStreamNonBlocking) == cudaSuccess &&
             cudaEventCreateWithFlags(&h->ev_join[i], cudaEventDisableTiming) == cudaSuccess;
    if (!made) {
      if (h->ev_fork) cudaEventDestroy(h->ev_fork);
      h->ev_fork = nullptr;
      for (int i = 0; i < 2; ++i) {
        if (h->ev_join[i]) cudaEventDestroy(h->ev_join[i]);
        if (h->side[i]) cudaStreamDestroy(h->side[i]);
        h->ev_join[i] = nullptr;
        h->side[i] = nullptr;
      }
      cudaGetLastError();
    }
  }
  cudaStream_t s = 0;
  cudaError_t e = cudaSuccess;
  e = cudaMemsetAsync(h->core_m, 0, sizeof(float) * ncore * h->mc, s);
  if (e == cudaSuccess) e = cudaMemsetAsync(h->core_v, 0, sizeof(float) * ncore * h->vc, s);
  if (e == cudaSuccess) e = cudaMemsetAsync(h->sp_m, 0, sizeof(float) * std::max<int64_t>(h->k, 1) * h->mc, s);
  if (e == cudaSuccess) e = cudaMemsetAsync(h->sp_v, 0, sizeof(float) * std::max<int64_t>(h->k, 1) * h->vc, s);
  if (e == cudaSuccess) e = cudaMemsetAsync(h->omega, 0, sizeof(int64_t) * std::max<int64_t>(h->k, 1), s);
  if (e == cudaSuccess) e = cudaMemsetAsync(h->d_err, 0, sizeof(int), s);
  for (int n = 0; n < ndim && e == cudaSuccess; ++n) {
    if (!((proj >> n) & 1u)) {
      identity_kernel<<<(unsigned)std::min<int64_t>(ceil_div(shape[n] * shape[n], 256), 1024), 256, 0, s>>>(
          (float2*)h->U[n], shape[n]);
      e = cudaGetLastError();
    } else {
      e = cudaMemsetAsync(h->U[n], 0, sizeof(float) * 2 * shape[n] * ranks[n], s);
    }
  }
  if (e == cudaSuccess) e = cudaStreamSynchronize(s);
  if (e != cudaSuccess) {
    free_all(h);
    delete h;
    return fail(nullptr, TGD_ERR_CUDA, std::string("initialisation failed: ") + cudaGetErrorString(e));
  }
  *out = h;
  return TGD_OK;
}

tgd_status tgd_refresh(tgd_handle h, const void* grad, void* stream) {
  if (!h) return fail(nullptr, TGD_ERR_INVALID_ARG, "NULL handle");
  if (!grad) return fail(h, TGD_ERR_INVALID_ARG, "grad is NULL");
  if (h->mode0_total > 0)
    return fail(h, TGD_ERR_UNSUPPORTED, "a block of mode-0 rows is not refreshed on its own: set its "
                                        "factors and index set with tgd_set_state");
  if (h->pending) return fail(h, TGD_ERR_STATE, "tgd_step_begin is waiting for tgd_step_end");
  return do_refresh(h, grad, (cudaStream_t)stream);
}

tgd_status tgd_step(tgd_handle h, const void* grad, void* weight, void* stream) {
  if (!h) return fail(nullptr, TGD_ERR_INVALID_ARG, "NULL handle");
  if (!grad || !weight) return fail(h, TGD_ERR_INVALID_ARG, "grad or weight is NULL");
  cudaStream_t s = (cudaStream_t)stream;
  if (h->pending) return fail(h, TGD_ERR_STATE, "tgd_step_begin is waiting for tgd_step_end");
  if (h->mode0_total > 0)
    return fail(h, TGD_ERR_STATE, "a block of mode-0 rows steps with tgd_step_begin, a sum of the "
                                  "blocks' cores, and tgd_step_end");
  if (h->opt.auto_refresh && h->T > 0 && h->t % h->T == 0) {
    tgd_status st = do_refresh(h, grad, s);
    if (st != TGD_OK) return st;
  }
  if (!h->has_subspace) return fail(h, TGD_ERR_STATE, "no refresh has run: call tgd_refresh first");
  if (h->opt.order == 1) {
    tgd_status st = step_lowrank_first(h, grad, weight, s);
    if (st != TGD_OK) return st;
    h->t += 1;
    return TGD_OK;
  }
  tgd_status st = step_begin(h, grad, s);
  if (st != TGD_OK) return st;
  return step_end(h, weight, s);
}

tgd_status tgd_step_begin(tgd_handle h, const void* grad, void* stream) {
  if (!h) return fail(nullptr, TGD_ERR_INVALID_ARG, "NULL handle");
  if (!grad) return fail(h, TGD_ERR_INVALID_ARG, "grad is NULL");
  if (h->pending) return fail(h, TGD_ERR_STATE, "tgd_step_begin is waiting for tgd_step_end");
  if (h->opt.order == 1)
    return fail(h, TGD_ERR_UNSUPPORTED, "the low-rank-first order has no split step");
  cudaStream_t s = (cudaStream_t)stream;
  if (h->mode0_total == 0 && h->opt.auto_refresh && h->T > 0 && h->t % h->T == 0) {
    tgd_status st = do_refresh(h, grad, s);
    if (st != TGD_OK) return st;
  }
  if (!h->has_subspace) return fail(h, TGD_ERR_STATE, "no refresh has run: call tgd_refresh first");
  return step_begin(h, grad, s);
}

tgd_status tgd_core_buffer(tgd_handle h, float** core, int64_t* count) {
  if (!h || !core || !count) return fail(h, TGD_ERR_INVALID_ARG, "NULL argument");
  if (!h->pending) return fail(h, TGD_ERR_STATE, "no tgd_step_begin is waiting for tgd_step_end");
  *core = core_buffer(h);
  *count = h->ncore * h->mc;
  return TGD_OK;
}

tgd_status tgd_step_end(tgd_handle h, void* weight, void* stream) {
  if (!h) return fail(nullptr, TGD_ERR_INVALID_ARG, "NULL handle");
  if (!weight) return fail(h, TGD_ERR_INVALID_ARG, "weight is NULL");
  if (!h->pending) return fail(h, TGD_ERR_STATE, "tgd_step_end without tgd_step_begin");
  return step_end(h, weight, (cudaStream_t)stream);
}

// The host-buffer step of the tensor-core path (complex fp16): G in on the
// caller's stream; W in, in HC chunks of whole tiles, on the input copy
// stream behind G; the projection, the core AdamW and the expansions on the
// caller's stream while W arrives; then per chunk the reconstruction stream
// over its tiles once they have landed, and the chunk back to the host on the
// output copy stream while the next chunks are still coming in (the link
// carries both directions at once).
constexpr int HC = 8;
tgd_status step_host_tc(tgd_ctx* h, const void* grad_host, void* weight_host, cudaStream_t s) {
  const size_t gb = (size_t)h->N * dt_bytes(h->gdt), ws = dt_bytes(h->wdt);
  TGD_CUDA(h, cudaMemcpyAsync(h->stage_g, grad_host, gb, cudaMemcpyHostToDevice, s));
  cudaEvent_t* ev_w = h->hev;           // [HC] chunk i of W landed
  cudaEvent_t* ev_r = h->hev + HC;      // [HC] chunk i of W updated
  cudaEvent_t ev_g = h->hev[2 * HC], ev_out = h->hev[2 * HC + 1];
  TGD_CUDA(h, cudaEventRecord(ev_g, s));
  TGD_CUDA(h, cudaStreamWaitEvent(h->cin, ev_g, 0));
  const int64_t T = tc_tiles(h->tc), te = tc_tile_elems(h->tc);
  const int C = (int)std::min<int64_t>(HC, T);
  auto tile_of = [&](int i) { return T * i / C; };
  auto elem_of = [&](int64_t t) { return std::min<int64_t>(t * te, h->N); };
  for (int i = 0; i < C; ++i) {
    const int64_t e0 = elem_of(tile_of(i)), e1 = elem_of(tile_of(i + 1));
    TGD_CUDA(h, cudaMemcpyAsync((uint8_t*)h->stage_w + e0 * ws, (const uint8_t*)weight_host + e0 * ws,
                                (size_t)(e1 - e0) * ws, cudaMemcpyHostToDevice, h->cin));
    TGD_CUDA(h, cudaEventRecord(ev_w[i], h->cin));
  }
  if (h->opt.auto_refresh && h->T > 0 && h->t % h->T == 0) {
    tgd_status st = do_refresh(h, h->stage_g, s);
    if (st != TGD_OK) return st;
  }
  if (!h->has_subspace) return fail(h, TGD_ERR_STATE, "no refresh has run: call tgd_refresh first");
  tgd_status st = step_begin(h, h->stage_g, s);
  if (st != TGD_OK) return st;
  AdamConst acore = adam_const(h, 1.0);
  const float decay = (float)(1.0 - (double)h->lr * (double)h->wd);
  cudaError_t e = tc_step_finish(h->tc, h->stage_w, h->core_m, h->core_v, acore, decay, h->lr, h->d_err, s,
                                 timer_hook, h, false);
  if (e != cudaSuccess) return cuda_fail(h, e, "tensor-core reconstruction");
  for (int i = 0; i < C; ++i) {
    const int64_t t0 = tile_of(i), t1 = tile_of(i + 1);
    const int64_t e0 = elem_of(t0), e1 = elem_of(t1);
    TGD_CUDA(h, cudaStreamWaitEvent(s, ev_w[i], 0));
    e = tc_recon(h->tc, h->stage_w, t0, t1 - t0, decay, h->lr, h->d_err, s, timer_hook, h);
    if (e != cudaSuccess) return cuda_fail(h, e, "tensor-core reconstruction");
    TGD_CUDA(h, cudaEventRecord(ev_r[i], s));
    TGD_CUDA(h, cudaStreamWaitEvent(h->cout, ev_r[i], 0));
    TGD_CUDA(h, cudaMemcpyAsync((uint8_t*)weight_host + e0 * ws, (const uint8_t*)h->stage_w + e0 * ws,
                                (size_t)(e1 - e0) * ws, cudaMemcpyDeviceToHost, h->cout));
  }
  TGD_CUDA(h, cudaEventRecord(ev_out, h->cout));
  TGD_CUDA(h, cudaStreamWaitEvent(s, ev_out, 0));
  h->pending = false;
  h->t += 1;
  return check_device_error(h, s, true);
}

tgd_status tgd_step_host(tgd_handle h, const void* grad_host, void* weight_host, void* stream) {
  if (!h) return fail(nullptr, TGD_ERR_INVALID_ARG, "NULL handle");
  if (!grad_host || !weight_host) return fail(h, TGD_ERR_INVALID_ARG, "grad or weight is NULL");
  cudaStream_t s = (cudaStream_t)stream;
  size_t gb = (size_t)h->N * dt_bytes(h->gdt), wb = (size_t)h->N * dt_bytes(h->wdt);
  if (!h->stage_g && !dalloc(h, &h->stage_g, gb)) return fail(h, TGD_ERR_OOM, "staging allocation failed");
  if (!h->stage_w && !dalloc(h, &h->stage_w, wb)) return fail(h, TGD_ERR_OOM, "staging allocation failed");
  if (h->pending) return fail(h, TGD_ERR_STATE, "tgd_step_begin is waiting for tgd_step_end");
  if (h->path == TGD_PATH_TCGEN05 && !h->use_tc32 && h->opt.order == 0 && h->mode0_total == 0) {
    if (!h->cin) {
      bool made = cudaStreamCreateWithFlags(&h->cin, cudaStreamNonBlocking) == cudaSuccess &&
                  cudaStreamCreateWithFlags(&h->cout, cudaStreamNonBlocking) == cudaSuccess;
      for (cudaEvent_t& ev : h->hev) made = made && cudaEventCreateWithFlags(&ev, cudaEventDisableTiming) == cudaSuccess;
      if (!made) {
        for (cudaEvent_t& ev : h->hev) {
          if (ev) cudaEventDestroy(ev);
          ev = nullptr;
        }
        if (h->cin) cudaStreamDestroy(h->cin);
        if (h->cout) cudaStreamDestroy(h->cout);
        h->cin = h->cout = nullptr;
        cudaGetLastError();
      }
    }
    if (h->cin) return step_host_tc(h, grad_host, weight_host, s);
  }
  TGD_CUDA(h, cudaMemcpyAsync(h->stage_g, grad_host, gb, cudaMemcpyHostToDevice, s));
  TGD_CUDA(h, cudaMemcpyAsync(h->stage_w, weight_host, wb, cudaMemcpyHostToDevice, s));
  tgd_status st = tgd_step(h, h->stage_g, h->stage_w, stream);
  if (st != TGD_OK) return st;
  TGD_CUDA(h, cudaMemcpyAsync(weight_host, h->stage_w, wb, cudaMemcpyDeviceToHost, s));
  return check_device_error(h, s, true);
}

tgd_status tgd_sync(tgd_handle h, void* stream) {
  if (!h) return fail(nullptr, TGD_ERR_INVALID_ARG, "NULL handle");
  return check_device_error(h, (cudaStream_t)stream, true);
}

tgd_status tgd_destroy(tgd_handle h) {
  if (!h) return TGD_OK;
  cudaDeviceSynchronize();
  free_all(h);
  delete h;
  return TGD_OK;
}

tgd_status tgd_query(tgd_handle h, tgd_info* info) {
  if (!h || !info) return fail(h, TGD_ERR_INVALID_ARG, "NULL argument");
  std::memset(info, 0, sizeof(*info));
  info->ndim = h->d;
  for (int n = 0; n < h->d; ++n) {
    info->shape[n] = h->I[n];
    info->ranks[n] = h->r[n];
  }
  info->N = h->N;
  info->k = h->k;
  info->ncore = h->ncore;
  info->core_m_len = h->ncore * h->mc;
  info->core_v_len = h->ncore * h->vc;
  info->sparse_m_len = h->k * h->mc;
  info->sparse_v_len = h->k * h->vc;
  info->path = h->path;
  info->device_bytes = h->bytes;
  info->t = h->t;
  info->refreshes = h->refreshes;
  info->has_subspace = h->has_subspace ? 1 : 0;
  return TGD_OK;
}

tgd_status tgd_state_memory(int ndim, const int64_t* shape, const int64_t* ranks,
                            double sparse_ratio, tgd_dtype grad_dtype, int complex_adam,
                            tgd_memory* out) {
  if (!out || !shape || !ranks) return fail(nullptr, TGD_ERR_INVALID_ARG, "NULL argument");
  if (ndim < 1 || ndim > TGD_MAX_NDIM) return fail(nullptr, TGD_ERR_INVALID_ARG, "bad ndim");
  if (!(sparse_ratio >= 0.0 && sparse_ratio <= 1.0))
    return fail(nullptr, TGD_ERR_INVALID_ARG, "sparse_ratio must be in [0, 1]");
  if (grad_dtype < TGD_R32 || grad_dtype > TGD_R16 || complex_adam < 0 || complex_adam > 1)
    return fail(nullptr, TGD_ERR_INVALID_ARG, "bad dtype or complex_adam");
  int64_t N = 1, ncore = 1, nfac = 0;
  for (int n = 0; n < ndim; ++n) {
    if (shape[n] < 1 || ranks[n] < 1 || ranks[n] > shape[n])
      return fail(nullptr, TGD_ERR_INVALID_ARG, "need 1 <= ranks[n] <= shape[n]");
    if (N > ((int64_t)1 << 40) / shape[n]) return fail(nullptr, TGD_ERR_INVALID_ARG, "tensor too large");
    N *= shape[n];
    ncore *= ranks[n];
    if (ranks[n] < shape[n]) nfac += shape[n] * ranks[n];
  }
  const bool cplx = grad_dtype == TGD_C64 || grad_dtype == TGD_C32H;
  const int64_t mb = cplx ? 8 : 4, vb = cplx && complex_adam ? 8 : 4, ub = cplx ? 8 : 4;
  const int64_t k = (int64_t)std::floor(sparse_ratio * (double)N);
  tgd_memory m;
  m.N = N;
  m.k = k;
  m.core_elems = ncore;
  m.factor_elems = nfac;
  m.adamw_bytes = N * (mb + vb);
  m.core_bytes = ncore * (mb + vb);
  m.factor_bytes = nfac * ub;
  m.sparse_bytes = k * (8 + mb + vb);
  m.total_bytes = m.core_bytes + m.factor_bytes + m.sparse_bytes;
  *out = m;
  return TGD_OK;
}

tgd_status tgd_get_state(tgd_handle h, tgd_state_view* out, void* stream) {
  if (!h || !out) return fail(h, TGD_ERR_INVALID_ARG, "NULL argument");
  cudaStream_t s = (cudaStream_t)stream;
  TGD_CUDA(h, cudaStreamSynchronize(s));
  out->t = h->t;
  out->refreshes = h->refreshes;
  out->has_subspace = h->has_subspace ? 1 : 0;
  if (out->omega && h->k > 0)
    TGD_CUDA(h, cudaMemcpy(out->omega, h->omega, sizeof(int64_t) * h->k, cudaMemcpyDeviceToHost));
  if (out->omega_val && h->k > 0)
    TGD_CUDA(h, cudaMemcpy(out->omega_val, h->omega_val, sizeof(float) * h->k * h->mc, cudaMemcpyDeviceToHost));
  for (int n = 0; n < h->d; ++n)
    if (out->U[n])
      TGD_CUDA(h, cudaMemcpy(out->U[n], h->U[n], sizeof(float) * 2 * h->I[n] * h->r[n], cudaMemcpyDeviceToHost));
  if (h->path == TGD_PATH_TCGEN05 && !h->use_tc32) {
    if (out->core_m) TGD_CUDA(h, tc_core_to_canonical(h->tc, h->core_m, h->mc, out->core_m));
    if (out->core_v) TGD_CUDA(h, tc_core_to_canonical(h->tc, h->core_v, h->vc, out->core_v));
  } else {
    if (out->core_m)
      TGD_CUDA(h, cudaMemcpy(out->core_m, h->core_m, sizeof(float) * h->ncore * h->mc, cudaMemcpyDeviceToHost));
    if (out->core_v)
      TGD_CUDA(h, cudaMemcpy(out->core_v, h->core_v, sizeof(float) * h->ncore * h->vc, cudaMemcpyDeviceToHost));
  }
  if (out->sparse_m && h->k > 0)
    TGD_CUDA(h, cudaMemcpy(out->sparse_m, h->sp_m, sizeof(float) * h->k * h->mc, cudaMemcpyDeviceToHost));
  if (out->sparse_v && h->k > 0)
    TGD_CUDA(h, cudaMemcpy(out->sparse_v, h->sp_v, sizeof(float) * h->k * h->vc, cudaMemcpyDeviceToHost));
  return TGD_OK;
}

tgd_status tgd_set_state(tgd_handle h, const tgd_state_view* in, void* stream) {
  if (!h || !in) return fail(h, TGD_ERR_INVALID_ARG, "NULL argument");
  if (in->t < 0 || in->refreshes < 0) return fail(h, TGD_ERR_INVALID_ARG, "negative counters");
  if (in->omega) {
    for (int64_t j = 0; j < h->k; ++j) {
      if (in->omega[j] < 0 || in->omega[j] >= h->N || (j > 0 && in->omega[j] <= in->omega[j - 1]))
        return fail(h, TGD_ERR_INVALID_ARG, "omega must be strictly ascending and in range");
    }
  }
  cudaStream_t s = (cudaStream_t)stream;
  TGD_CUDA(h, cudaStreamSynchronize(s));
  if (in->omega && h->k > 0)
    TGD_CUDA(h, cudaMemcpy(h->omega, in->omega, sizeof(int64_t) * h->k, cudaMemcpyHostToDevice));
  if (in->omega_val && h->k > 0)
    TGD_CUDA(h, cudaMemcpy(h->omega_val, in->omega_val, sizeof(float) * h->k * h->mc, cudaMemcpyHostToDevice));
  for (int n = 0; n < h->d; ++n)
    if (in->U[n])
      TGD_CUDA(h, cudaMemcpy(h->U[n], in->U[n], sizeof(float) * 2 * h->I[n] * h->r[n], cudaMemcpyHostToDevice));
  if (h->path == TGD_PATH_TCGEN05 && !h->use_tc32) {
    if (in->core_m) TGD_CUDA(h, tc_core_from_canonical(h->tc, in->core_m, h->mc, h->core_m));
    if (in->core_v) TGD_CUDA(h, tc_core_from_canonical(h->tc, in->core_v, h->vc, h->core_v));
  } else {
    if (in->core_m)
      TGD_CUDA(h, cudaMemcpy(h->core_m, in->core_m, sizeof(float) * h->ncore * h->mc, cudaMemcpyHostToDevice));
    if (in->core_v)
      TGD_CUDA(h, cudaMemcpy(h->core_v, in->core_v, sizeof(float) * h->ncore * h->vc, cudaMemcpyHostToDevice));
  }
  if (in->sparse_m && h->k > 0)
    TGD_CUDA(h, cudaMemcpy(h->sp_m, in->sparse_m, sizeof(float) * h->k * h->mc, cudaMemcpyHostToDevice));
  if (in->sparse_v && h->k > 0)
    TGD_CUDA(h, cudaMemcpy(h->sp_v, in->sparse_v, sizeof(float) * h->k * h->vc, cudaMemcpyHostToDevice));
  h->t = in->t;
  h->refreshes = in->refreshes;
  h->has_subspace = in->has_subspace != 0;
  tgd_status st = rebuild_derived(h, s);
  if (st != TGD_OK) return st;
  TGD_CUDA(h, cudaStreamSynchronize(s));
  return TGD_OK;
}

size_t tgd_topk_workspace_bytes(int64_t n) { return select_workspace_bytes(n); }

tgd_status tgd_topk_select(const void* grad, tgd_dtype dtype, int64_t n, int64_t k,
                           int64_t* omega_out, float* val_out, void* workspace,
                           size_t workspace_bytes, void* stream) {
  if (!dt_valid(dtype)) return fail(nullptr, TGD_ERR_INVALID_ARG, "unknown dtype");
  if (n < 0 || k < 0 || k > n) return fail(nullptr, TGD_ERR_INVALID_ARG, "need 0 <= k <= n");
  if (k == 0) return TGD_OK;
  if (!grad || !omega_out) return fail(nullptr, TGD_ERR_INVALID_ARG, "grad or omega_out is NULL");
  if (k < n && (!workspace || workspace_bytes < select_workspace_bytes(n)))
    return fail(nullptr, TGD_ERR_INVALID_ARG, "workspace too small");
  cudaError_t e = select_topk(grad, dtype, n, k, omega_out, val_out, workspace, (cudaStream_t)stream);
  if (e != cudaSuccess) return cuda_fail(nullptr, e, "tgd_topk_select");
  return TGD_OK;
}

tgd_status tgd_profile(tgd_handle h, int enable) {
  if (!h) return fail(nullptr, TGD_ERR_INVALID_ARG, "NULL handle");
  if (enable) {
    h->prof.clear();
    h->ev_used = 0;
  }
  h->prof_on = enable != 0;
  return TGD_OK;
}

tgd_status tgd_profile_read(tgd_handle h, tgd_kernel_time* out, int capacity, int* count) {
  if (!h || !count) return fail(h, TGD_ERR_INVALID_ARG, "NULL argument");
  std::vector<tgd_kernel_time> acc;
  for (auto& rec : h->prof) {
    TGD_CUDA(h, cudaEventSynchronize(rec.second.second));
    float ms = 0.f;
    TGD_CUDA(h, cudaEventElapsedTime(&ms, rec.second.first, rec.second.second));
    tgd_kernel_time* slot = nullptr;
    for (auto& a : acc)
      if (rec.first == a.name) slot = &a;
    if (!slot) {
      acc.push_back(tgd_kernel_time{});
      slot = &acc.back();
      std::strncpy(slot->name, rec.first.c_str(), sizeof(slot->name) - 1);
    }
    slot->launches += 1;
    slot->total_ms += ms;
  }
  *count = (int)acc.size();
  for (int i = 0; i < (int)acc.size() && i < capacity && out; ++i) out[i] = acc[i];
  return TGD_OK;
}

const char* tgd_last_error(tgd_handle h) {
  return h ? h->last_error.c_str() : g_last_error.c_str();
}

}  // extern "C"
