/*
 * tgd.h - C ABI of the TensorGRaD optimizer step on one NVIDIA B200.
 *
 * The method (TensorGRaD: robust low-rank + sparse decomposition of tensor
 * gradients) is defined on these pages:
 *   [S1] "TensorGRaD" summary, nullthought.net/?p=5973, section 三 (method
 *        implementation details);
 *   [S2] Pith review of TensorGRaD, pith.science/paper/2501.02379, "What
 *        carries the argument" and "Assumptions & free parameters";
 *   [S3] the same review's appended paper text, Theorem 2 (Tensor low-rank
 *        convergence) and Appendix K (tensor operations and notation).
 *
 * One step on an N-way gradient G (shape I_1 x ... x I_d, row-major, last
 * index fastest) and the weight W of the same shape:
 *   1. (every T steps) refresh: Omega = the k = floor(rho * N) entries of
 *      largest magnitude (or k uniformly random entries), R = G with zeros on
 *      Omega, U_n = leading r_n eigenvectors of the mode-n Gram R_(n) R_(n)^H.
 *   2. g_s = G[Omega]; R = G - S (G with zeros on Omega).
 *   3. C = R x_1 U_1^H ... x_d U_d^H.
 *   4. C~ = Adam(C), S~ = lambda * Adam(g_s), FP32 moments, bias-corrected.
 *   5. Delta = C~ x_1 U_1 ... x_d U_d; Delta[Omega] += S~ (in place).
 *   6. W <- W * (1 - lr * wd) - lr * Delta, rounded once to W's dtype.
 * A mode with r_n == I_n uses U_n = I. Complex tensors use the conjugate
 * transpose; "complex Adam" keeps m complex and v = EMA(|g|^2) by default.
 *
 * Conventions for every entry point:
 *  - Device pointers are plain CUDA device addresses (for example a torch
 *    tensor's data_ptr()), contiguous, row-major, 16-byte aligned. Host
 *    pointers are ordinary (preferably pinned) host memory.
 *  - `stream` is a cudaStream_t passed as void*; NULL is the legacy default
 *    stream. Work is enqueued on it and the call returns without waiting,
 *    except where a function says it synchronises.
 *  - Arguments are checked before any work is enqueued; a bad argument
 *    returns TGD_ERR_INVALID_ARG and changes nothing. Errors found on the
 *    device (a bounded wait that ran out) set an error word in the handle;
 *    the calls that synchronise (tgd_sync, tgd_step_host) read it, return
 *    TGD_ERR_TIMEOUT and clear it. The asynchronous calls do not read it.
 *  - A handle is not thread-safe. It owns all optimizer state (allocated at
 *    tgd_create, freed at tgd_destroy); the caller owns grad and weight.
 */
#ifndef TGD_H
#define TGD_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define TGD_MAX_NDIM 8

#if defined(__GNUC__)
#define TGD_API __attribute__((visibility("default")))
#else
#define TGD_API
#endif

typedef struct tgd_ctx* tgd_handle;

typedef enum {
  TGD_OK = 0,
  TGD_ERR_INVALID_ARG = 1,  /* a shape, rank, ratio, dtype or pointer is out of range */
  TGD_ERR_UNSUPPORTED = 2,  /* valid, but not supported by the chosen kernel path */
  TGD_ERR_OOM = 3,          /* device or pinned host allocation failed */
  TGD_ERR_CUDA = 4,         /* a CUDA runtime call failed (no device, launch error, ...) */
  TGD_ERR_TIMEOUT = 5,      /* a bounded device-side wait gave up */
  TGD_ERR_STATE = 6,        /* step before any refresh with auto-refresh off, bad state view */
  TGD_ERR_NONFINITE = 7     /* reserved: non-finite input detected */
} tgd_status;

/* Storage type of gradients and weights. Complex types interleave (re, im). */
typedef enum {
  TGD_R32 = 0,   /* real fp32 */
  TGD_C64 = 1,   /* complex, fp32 re and im */
  TGD_C32H = 2,  /* complex, fp16 re and im (mixed-precision recipe of [S1]) */
  TGD_R16 = 3    /* real fp16 */
} tgd_dtype;

/* Kernel path. AUTO picks TCGEN05 where the tensor-core kernels apply, GENERIC
 * (CUDA cores) otherwise. TCGEN05 covers complex fp16 gradients whose trailing
 * modes fit its streaming tiles (fp16 or fp32 weights), and fp32 gradients
 * with fp32 weights (real or complex) whose projected modes have at most 256
 * entries. */
typedef enum { TGD_PATH_AUTO = 0, TGD_PATH_GENERIC = 1, TGD_PATH_TCGEN05 = 2 } tgd_path;

typedef struct {
  int omega_mode;         /* 0: top-k magnitude (default); 1: random sampling [S2] */
  uint64_t seed;          /* random sampling seed */
  float sparse_scale;     /* lambda, the sparse update scale of [S2]'s free parameters; default 1 */
  int complex_adam;       /* 0: m complex, v = EMA |g|^2 (default); 1: re and im as separate reals */
  int moments_on_refresh; /* 0: keep moments across a refresh (default); 1: reset to zero */
  int auto_refresh;       /* 1 (default): tgd_step refreshes first when T > 0 and t % T == 0 */
  int path;               /* tgd_path */
  int sm_budget;          /* 0 (default): the stream kernels spread over every SM; n > 0: over at
                             most n SMs, so that several tensors stepped on separate streams run
                             side by side (tensor-core path; results do not change) */
  int order;              /* decomposition order, a free parameter of the method [S2]:
                             0 (default) sparse part first, the low-rank part on the residual;
                             1 low-rank part first (the ablated order): U_n from the Gram of G
                             itself, Omega = top-k of E = G - L (L = G x_n U_n U_n^H, E in fp32),
                             each step's sparse values E at Omega with L from that step's core.
                             Order 1 runs on the CUDA-core path. */
  int basis;              /* factors at a refresh: 0 (default) HOSVD, the leading eigenvectors
                             of each mode-n Gram [S2]; 1 the r_n columns q_j of the orthonormal
                             DCT matrix (sqrt(2/n) cos(k (2j+1) pi / 2n), row 0 / sqrt 2) with
                             the largest alignment q_j^T Gram q_j, ties to the lower column (the
                             dynamic column selection of the Trion / DCT-AdamW page); no
                             eigensolver runs */
  int wait_limit_ms;      /* limit of each bounded wait inside the projection kernel of the
                             tensor-core path, in milliseconds; 0 (default) = 2000. A wait that
                             runs out makes the kernel stop its work and return, and the next
                             synchronising call (tgd_sync, tgd_step_host) reports
                             TGD_ERR_TIMEOUT */
  int test_stall;         /* test hook, 0 (default) = off. 1: in every step, the projection
                             kernel's first CTA skips the load of its first tile, so one of its
                             bounded waits runs out after wait_limit_ms (failure detection
                             without a fault); the step's results are then undefined */
  int64_t sparse_k;       /* -1 (default): k = floor(sparse_ratio * N) entries in Omega [S1
                             section 三]; >= 0: exactly this many (a block of a split tensor
                             holds its share of the whole tensor's index set) */
  int64_t mode0_total;    /* 0 (default): the handle holds a whole tensor. > 0: it holds a
                             contiguous block of rows of mode 0 of a tensor whose mode 0 has
                             mode0_total entries (shape[0] = the block's rows; ranks[0] may
                             exceed shape[0]). Mode 0 is projected when ranks[0] < mode0_total,
                             with U_0 = this block's rows of the whole factor (shape[0] x
                             ranks[0]). Such a handle steps only through tgd_step_begin /
                             tgd_step_end with the blocks' partial cores summed in between, and
                             takes its factors and index set from tgd_set_state (no refresh of
                             its own: T = 0 or auto_refresh = 0) */
} tgd_options;

/* Fills `opt` with the defaults listed above. */
TGD_API void tgd_default_options(tgd_options* opt);

/* Creates an optimizer for one tensor [S1 section 三; S2 free parameters].
 *  ndim in [2, 8]; shape[n] >= 1; 1 <= ranks[n] <= shape[n] (== means U_n = I);
 *  sparse_ratio rho in [0, 1], k = floor(rho * N); T >= 0 refresh period
 *  (0 = never refresh automatically); lr, beta1, beta2, eps, wd: AdamW.
 *  grad_dtype and weight_dtype must both be real or both complex.
 *  opt may be NULL (defaults). Allocates all device state on the current
 *  device with cudaMalloc and zeroes the moments; *out receives the handle.
 *  Returns INVALID_ARG, UNSUPPORTED (path TCGEN05 forced on shapes it cannot
 *  tile), OOM or CUDA on failure, with *out set to NULL. */
TGD_API tgd_status tgd_create(tgd_handle* out, int ndim, const int64_t* shape, const int64_t* ranks,
                      double sparse_ratio, int64_t T, float lr, float beta1, float beta2, float eps,
                      float wd, tgd_dtype grad_dtype, tgd_dtype weight_dtype,
                      const tgd_options* opt);

/* One optimizer step (steps 1-6 above) [S1 section 三; S2; S3 Theorem 2].
 *  grad: device, N elements of grad_dtype, read only. weight: device, N
 *  elements of weight_dtype, updated in place. Refreshes first when
 *  auto-refresh is on, T > 0 and t % T == 0. Advances t by one.
 *  Returns STATE if no refresh has happened and none is due. */
TGD_API tgd_status tgd_step(tgd_handle h, const void* grad, void* weight, void* stream);

/* Refresh Omega and the factors U_n from `grad` (device, read only) [S2].
 *  Does not advance t and does not touch weights or moments (unless
 *  moments_on_refresh == 1). Increments the refresh ordinal, which seeds the
 *  random-sampling variant. */
TGD_API tgd_status tgd_refresh(tgd_handle h, const void* grad, void* stream);

/* The same step as tgd_step with host buffers: copies grad (host, N elements)
 *  and weight (host, N elements) to the device, steps, copies weight back.
 *  Synchronises the stream before returning, then returns any device-side
 *  error recorded since the last check (TIMEOUT) as tgd_sync does. Lazily
 *  allocates device staging for both tensors on first use. On the tensor-core
 *  path the weights move in chunks of tiles on two copy streams of the
 *  handle's own, overlapped with the reconstruction of earlier chunks; pinned
 *  host buffers let those copies run asynchronously. */
TGD_API tgd_status tgd_step_host(tgd_handle h, const void* grad_host, void* weight_host, void* stream);

/* Waits for the handle's work on `stream` and returns any device-side error
 *  recorded since the last check (TIMEOUT), else OK. */
TGD_API tgd_status tgd_sync(tgd_handle h, void* stream);

/* Frees everything the handle owns. NULL is allowed. Synchronises the device. */
TGD_API tgd_status tgd_destroy(tgd_handle h);

/* Sizes of the handle's state, for tgd_get_state / tgd_set_state buffers. */
typedef struct {
  int ndim;
  int64_t shape[TGD_MAX_NDIM], ranks[TGD_MAX_NDIM];
  int64_t N;            /* elements of the tensor */
  int64_t k;            /* |Omega| */
  int64_t ncore;        /* prod(ranks) */
  int64_t core_m_len;   /* floats in core m: ncore * (2 if complex else 1) */
  int64_t core_v_len;   /* floats in core v: ncore * (2 if complex_adam == 1 else 1) */
  int64_t sparse_m_len; /* k * (2 if complex else 1) */
  int64_t sparse_v_len; /* k * (2 if complex_adam == 1 else 1) */
  int path;             /* resolved tgd_path (GENERIC or TCGEN05) */
  size_t device_bytes;  /* device memory the handle holds */
  int64_t t, refreshes;
  int has_subspace;
} tgd_info;

TGD_API tgd_status tgd_query(tgd_handle h, tgd_info* info);

/* Optimizer-state memory of the method for one tensor, next to AdamW's
 * (host arithmetic only; no handle, no device). The count follows [S3]'s
 * comparison of matrix and tensor low-rank state (its equations (9) and
 * (10)): the tensor low-rank branch keeps the core, prod r_n entries, and a
 * factor U_n of I_n x r_n entries for every projected mode; a mode with
 * r_n == I_n needs no factor (U_n = I). [S1] section 3 adds the sparse part:
 * a COO index per entry of Omega and Adam moments on its values, and keeps
 * all moments in FP32.
 *
 * Bytes per element: m = 8 complex / 4 real; v = 4, or 8 for complex tensors
 * with complex_adam == 1 (two second moments, view-as-real); a factor entry
 * 8 complex / 4 real; an Omega index 8 (int64). k = floor(sparse_ratio * N).
 * AdamW's figure is N * (m + v) with the same m and v.
 *
 * Arguments are checked as tgd_create checks them (1 <= ranks[n] <= shape[n],
 * 0 <= sparse_ratio <= 1, N <= 2^40, 1 <= ndim <= TGD_MAX_NDIM, complex_adam 0
 * or 1); a bad argument returns TGD_ERR_INVALID_ARG and leaves *out untouched.
 * The caller owns out. */
typedef struct {
  int64_t N;              /* elements of the tensor */
  int64_t k;              /* |Omega| */
  int64_t core_elems;     /* prod r_n */
  int64_t factor_elems;   /* sum of I_n r_n over modes with r_n < I_n */
  int64_t adamw_bytes;    /* N (m + v) */
  int64_t core_bytes;     /* core_elems (m + v) */
  int64_t factor_bytes;   /* factor_elems x (8 complex, 4 real) */
  int64_t sparse_bytes;   /* k (8 + m + v) */
  int64_t total_bytes;    /* core_bytes + factor_bytes + sparse_bytes */
} tgd_memory;

TGD_API tgd_status tgd_state_memory(int ndim, const int64_t* shape, const int64_t* ranks,
                                    double sparse_ratio, tgd_dtype grad_dtype, int complex_adam,
                                    tgd_memory* out);

/* Host copy of the optimizer state (checkpoint / resume, and teacher-forced
 *  testing). Any pointer may be NULL to skip that part. Layouts:
 *   omega     int64[k], ascending linear indices (complex elements counted once)
 *   omega_val float[k * c], G[Omega] at the last refresh (c = 2 for complex)
 *   U[n]      float[I_n * r_n * 2], row-major I_n x r_n, interleaved (re, im)
 *   core_m    float[core_m_len], canonical row-major r_1 x ... x r_d order
 *   core_v    float[core_v_len], same order
 *   sparse_m  float[sparse_m_len], sparse_v float[sparse_v_len], in Omega order */
typedef struct {
  int64_t t;
  int64_t refreshes;
  int has_subspace;
  int64_t* omega;
  float* omega_val;
  float* U[TGD_MAX_NDIM];
  float* core_m;
  float* core_v;
  float* sparse_m;
  float* sparse_v;
} tgd_state_view;

/* The step in two halves, for one tensor split across GPUs along mode 0
 *  (each GPU holds a block of rows; see tgd_options.mode0_total). The mode-0
 *  product of the projection is a sum over mode 0's rows [S2 Appendix K: the
 *  mode-n product sums over i_n], so each block's projection is a partial
 *  core and the whole core is their sum; the core AdamW, the expansion with
 *  the block's rows of U_0, the sparse part and the weight update are local.
 *  - tgd_step_begin: refresh when due (whole tensors only), the sparse AdamW
 *    and the projection of this block into the handle's core buffer.
 *  - tgd_core_buffer: the core buffer's device address and its length in
 *    floats (fp32; (re, im) pairs for complex tensors, in the kernel path's
 *    own element order, the same on every block of one configuration). The
 *    caller sums the blocks' buffers elementwise in place on every block
 *    (for example with an all-reduce over the GPUs, ordered on `stream`).
 *  - tgd_step_end: the core AdamW on the summed core, the expansion, the
 *    scatter-add of the sparse update and the weight update; t advances.
 *  tgd_step equals begin + end on a whole tensor. Out of order calls return
 *  TGD_ERR_STATE; the low-rank-first order has no split (UNSUPPORTED). */
TGD_API tgd_status tgd_step_begin(tgd_handle h, const void* grad, void* stream);
TGD_API tgd_status tgd_core_buffer(tgd_handle h, float** core, int64_t* count);
TGD_API tgd_status tgd_step_end(tgd_handle h, void* weight, void* stream);

/* Copies the state to host buffers. Synchronises `stream`. */
TGD_API tgd_status tgd_get_state(tgd_handle h, tgd_state_view* out, void* stream);

/* Replaces the state from host buffers (NULL parts are left unchanged; t,
 *  refreshes and has_subspace are always taken). Omega must be strictly
 *  ascending and in range, else INVALID_ARG and nothing changes. Derived
 *  device data (index tiles, masks, kernel operands) is rebuilt. Synchronises. */
TGD_API tgd_status tgd_set_state(tgd_handle h, const tgd_state_view* in, void* stream);

/* Standalone top-k selection [S1 section 二; S2]: the k entries of `grad`
 *  (device, n elements of dtype) with the largest magnitude key (real:
 *  fp32 |g|; complex: fp32 fma(re, re, im*im)), ties to the lower index,
 *  written ascending as COO: omega_out (device int64[k]) and val_out (device
 *  float[k * c], fp32 values, c = 2 for complex; may be NULL). workspace is
 *  device memory of at least tgd_topk_workspace_bytes(n) bytes owned by the
 *  caller; its contents on entry do not matter. */
TGD_API size_t tgd_topk_workspace_bytes(int64_t n);
TGD_API tgd_status tgd_topk_select(const void* grad, tgd_dtype dtype, int64_t n, int64_t k,
                           int64_t* omega_out, float* val_out, void* workspace,
                           size_t workspace_bytes, void* stream);

/* Top-k selection that allocates nothing (no counterpart in the paper: an
 *  interface for callers that cannot allocate device memory). The same
 *  selection and output as tgd_topk_select, but its scratch space is a
 *  fixed array compiled into the library instead of a caller workspace, so
 *  a caller that only holds its input and output buffers can use it: for
 *  example a plugin inside a framework whose allocator owns all device
 *  memory, or a loop that must not call cudaMalloc because cudaMalloc may
 *  synchronise the device.
 *  - n must not exceed TGD_TOPK_STATIC_MAX_N, else TGD_ERR_INVALID_ARG.
 *  - The array (TGD_TOPK_STATIC_SCRATCH_BYTES bytes) exists once per GPU
 *    that loads the library and stays allocated until the process exits.
 *  - Every call looks up the array's device address on the current device
 *    (a host-side query, no stream work), so calls may be captured into a
 *    CUDA graph, and a device reset leaves nothing stale behind.
 *  - All calls share the array: calls whose work overlaps on the GPU (on
 *    different streams, or from different threads) race and give wrong
 *    results. Calls in one stream are ordered and safe; the array keeps the
 *    last call's contents, and every call clears what it needs itself. */
#define TGD_TOPK_STATIC_MAX_N ((int64_t)1 << 28)
#define TGD_TOPK_STATIC_SCRATCH_BYTES ((size_t)2 << 20)
TGD_API tgd_status tgd_topk_select_static(const void* grad, tgd_dtype dtype, int64_t n, int64_t k,
                                          int64_t* omega_out, float* val_out, void* stream);

/* Per-kernel timing with CUDA events recorded on the launching stream around
 *  every kernel the handle launches (no effect on results). enable = 1 clears
 *  the record and starts timing; enable = 0 stops it. */
TGD_API tgd_status tgd_profile(tgd_handle h, int enable);

typedef struct {
  char name[40];
  int64_t launches;
  double total_ms;
} tgd_kernel_time;

/* Waits for the recorded events and writes up to `capacity` per-kernel totals
 *  (launch count and summed duration) to `out`; *count receives the number
 *  of distinct kernels. */
TGD_API tgd_status tgd_profile_read(tgd_handle h, tgd_kernel_time* out, int capacity, int* count);

/* Message for the last error on this handle (or a global message for NULL). */
TGD_API const char* tgd_last_error(tgd_handle h);

#ifdef __cplusplus
}
#endif
#endif /* TGD_H */
