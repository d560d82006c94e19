// CUDA-core path of the TensorGRaD step, for every dtype and shape.
//
// The steps follow the nullthought.net TensorGRaD summary, section 三 (sparse
// part first, Tucker low-rank part on the residual, separate Adam updates,
// sparse update scatter-added in place into the rebuilt low-rank tensor) and
// Theorem 2 of the paper text appended to the Pith review (project with U^H
// mode by mode, update the optimizer state on the core, project back with U):
//   sparse_adam   g_s = G[Omega]; S~ = lambda * Adam(g_s)        (COO values)
//   mode_product  C = R x_n U_n^H, reading R as G masked on Omega (first
//                 contraction) and fp32 intermediates afterwards
//   core_adam     C~ = Adam(C) in place
//   mode_product  Delta = C~ x_n U_n
//   scatter_add   Delta[Omega] += S~
//   weight_update W = W (1 - lr wd) - lr Delta, one rounding to W's dtype
// fp32 arithmetic throughout (FFMA); the tensor-core path for complex fp16
// tensors lives in step_tc.cu.

#include "common.cuh"
#include "kernels.h"

namespace tgd {
namespace {

int grid_for(int64_t n, int threads = 256) {
  int64_t b = ceil_div(n, threads);
  int64_t cap = 148 * 16;
  return (int)(b < 1 ? 1 : (b > cap ? cap : b));
}

// Adam on the k values at Omega: G[Omega], or G[Omega] - L[Omega] when L (the
// low-rank part, fp32) is given (the low-rank-first order).
template <int DT>
__global__ void sparse_adam_kernel(const void* g, const float* L, const int64_t* omega, int64_t k,
                                   float* m, float* v, AdamConst a, float* upd) {
  const int mc = a.cplx ? 2 : 1, vc = (a.cplx && a.cmode == 1) ? 2 : 1;
  for (int64_t j = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; j < k;
       j += (int64_t)gridDim.x * blockDim.x) {
    float2 gv = load_elem<DT>(g, omega[j]);
    if (L) {
      const float2 l = a.cplx ? ((const float2*)L)[omega[j]] : make_float2(L[omega[j]], 0.f);
      gv = make_float2(gv.x - l.x, gv.y - l.y);
    }
    float mm[2], vv[2];
    for (int c = 0; c < mc; ++c) mm[c] = m[j * mc + c];
    for (int c = 0; c < vc; ++c) vv[c] = v[j * vc + c];
    float2 u = adam_elem(gv, mm, vv, a);
    for (int c = 0; c < mc; ++c) m[j * mc + c] = mm[c];
    for (int c = 0; c < vc; ++c) v[j * vc + c] = vv[c];
    if (a.cplx)
      ((float2*)upd)[j] = u;
    else
      upd[j] = u.x;
  }
}

__global__ void core_adam_kernel(float* c, int64_t n, float* m, float* v, AdamConst a) {
  const int mc = a.cplx ? 2 : 1, vc = (a.cplx && a.cmode == 1) ? 2 : 1;
  for (int64_t j = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; j < n;
       j += (int64_t)gridDim.x * blockDim.x) {
    float2 gv = a.cplx ? ((float2*)c)[j] : make_float2(c[j], 0.f);
    float mm[2], vv[2];
    for (int q = 0; q < mc; ++q) mm[q] = m[j * mc + q];
    for (int q = 0; q < vc; ++q) vv[q] = v[j * vc + q];
    float2 u = adam_elem(gv, mm, vv, a);
    for (int q = 0; q < mc; ++q) m[j * mc + q] = mm[q];
    for (int q = 0; q < vc; ++q) v[j * vc + q] = vv[q];
    if (a.cplx)
      ((float2*)c)[j] = u;
    else
      c[j] = u.x;
  }
}

// Source of the first contraction: the storage-typed gradient with zeros on
// Omega; later contractions read fp32 (complex: float2) intermediates.
template <int DT, bool CPLX>
struct Src {
  const void* p;
  const uint32_t* bits;
  __device__ __forceinline__ float2 operator()(int64_t i) const {
    if constexpr (DT >= 0) {
      if (bits && mask_bit(bits, i)) return make_float2(0.f, 0.f);
      return load_elem<DT>(p, i);
    } else if constexpr (CPLX) {
      return __ldg((const float2*)p + i);
    } else {
      return make_float2(__ldg((const float*)p + i), 0.f);
    }
  }
};

constexpr int TJ = 32, TC = 64, TK = 16, MT = 256;

// Y[a][j][b] = sum_k M[j][k] * X[a][k][b]. Output columns c = a * B + b.
// A 32 (j) x 64 (c) tile per block, 8 outputs per thread, k in steps of 16.
template <class S, bool CPLX>
__global__ void __launch_bounds__(MT) mode_product_kernel(S src, int64_t A, int64_t K, int64_t B,
                                                          const float* M, int64_t J, float* Y) {
  __shared__ float2 Ms[TJ][TK + 1];
  __shared__ float2 Xs[TK][TC + 1];
  const int64_t ncol = A * B;
  const int64_t c0 = (int64_t)blockIdx.x * TC;
  const int64_t j0 = (int64_t)blockIdx.y * TJ;
  const int ty = threadIdx.x >> 4, tx = threadIdx.x & 15;
  float2 acc[2][4];
  for (int u = 0; u < 2; ++u)
    for (int q = 0; q < 4; ++q) acc[u][q] = make_float2(0.f, 0.f);
  const bool b_unit = (B == 1);
  for (int64_t k0 = 0; k0 < K; k0 += TK) {
    for (int e = threadIdx.x; e < TJ * TK; e += MT) {
      int jj = e / TK, kk = e % TK;
      int64_t j = j0 + jj, k = k0 + kk;
      float2 v = make_float2(0.f, 0.f);
      if (j < J && k < K) {
        if (CPLX)
          v = ((const float2*)M)[j * K + k];
        else
          v.x = M[j * K + k];
      }
      Ms[jj][kk] = v;
    }
    for (int e = threadIdx.x; e < TK * TC; e += MT) {
      int kk, cc;
      if (b_unit) {
        cc = e / TK;
        kk = e % TK;
      } else {
        kk = e / TC;
        cc = e % TC;
      }
      int64_t c = c0 + cc, k = k0 + kk;
      float2 v = make_float2(0.f, 0.f);
      if (c < ncol && k < K) {
        int64_t a = c / B, b = c - a * B;
        v = src((a * K + k) * B + b);
      }
      Xs[kk][cc] = v;
    }
    __syncthreads();
#pragma unroll
    for (int kk = 0; kk < TK; ++kk) {
      float2 m0 = Ms[ty][kk], m1 = Ms[ty + 16][kk];
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        float2 x = Xs[kk][tx + 16 * q];
        if (CPLX) {
          acc[0][q] = cfma(m0, x, acc[0][q]);
          acc[1][q] = cfma(m1, x, acc[1][q]);
        } else {
          acc[0][q].x = __fmaf_rn(m0.x, x.x, acc[0][q].x);
          acc[1][q].x = __fmaf_rn(m1.x, x.x, acc[1][q].x);
        }
      }
    }
    __syncthreads();
  }
  for (int u = 0; u < 2; ++u) {
    int64_t j = j0 + ty + 16 * u;
    if (j >= J) continue;
    for (int q = 0; q < 4; ++q) {
      int64_t c = c0 + tx + 16 * q;
      if (c >= ncol) continue;
      int64_t a = c / B, b = c - a * B;
      int64_t o = (a * J + j) * B + b;
      if (CPLX)
        ((float2*)Y)[o] = acc[u][q];
      else
        Y[o] = acc[u][q].x;
    }
  }
}

// Y = X x_n M for coefficient matrices of at most SP_MAXMK entries (the modes
// of FNO-sized tensors): one thread per column (a, b) of the unfolding reads
// its K values (stride B: coalesced across threads when B > 1, from cache
// when B == 1) once per block of SP_J outputs, M is broadcast from shared
// memory and the outputs stay in registers. The sum over k runs in the same
// order as in mode_product_kernel, so both give the same bits.
constexpr int SP_T = 256, SP_J = 16, SP_MAXMK = 4096;

template <class S, bool CPLX>
__global__ void __launch_bounds__(SP_T) mode_product_small_kernel(S src, int64_t A, int64_t K,
                                                                  int64_t B, const float* M,
                                                                  int64_t J, float* Y) {
  __shared__ float2 Ms[SP_MAXMK];
  for (int64_t e = threadIdx.x; e < J * K; e += SP_T)
    Ms[e] = CPLX ? ((const float2*)M)[e] : make_float2(M[e], 0.f);
  __syncthreads();
  const int64_t ncol = A * B;
  for (int64_t c = (int64_t)blockIdx.x * SP_T + threadIdx.x; c < ncol;
       c += (int64_t)gridDim.x * SP_T) {
    const int64_t a = c / B, b = c - a * B;
    const int64_t xb = a * K * B + b, yb = a * J * B + b;
    for (int64_t j0 = 0; j0 < J; j0 += SP_J) {
      float2 acc[SP_J];
#pragma unroll
      for (int u = 0; u < SP_J; ++u) acc[u] = make_float2(0.f, 0.f);
      for (int64_t k = 0; k < K; ++k) {
        const float2 x = src(xb + k * B);
        const float2* mk = Ms + j0 * K + k;
#pragma unroll
        for (int u = 0; u < SP_J; ++u) {
          if (j0 + u < J) {
            const float2 m = mk[u * K];
            if (CPLX)
              acc[u] = cfma(m, x, acc[u]);
            else
              acc[u].x = __fmaf_rn(m.x, x.x, acc[u].x);
          }
        }
      }
#pragma unroll
      for (int u = 0; u < SP_J; ++u) {
        if (j0 + u < J) {
          const int64_t o = yb + (j0 + u) * B;
          if (CPLX)
            ((float2*)Y)[o] = acc[u];
          else
            Y[o] = acc[u].x;
        }
      }
    }
  }
}

template <int DT>
__global__ void masked_copy_kernel(const void* g, const uint32_t* bits, int64_t n, float* out) {
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n;
       i += (int64_t)gridDim.x * blockDim.x) {
    float2 v = bits && mask_bit(bits, i) ? make_float2(0.f, 0.f) : load_elem<DT>(g, i);
    if (Dt<DT>::cplx)
      ((float2*)out)[i] = v;
    else
      out[i] = v.x;
  }
}

// L <- G - L (fp32, in place): the residual after the low-rank part.
template <int DT>
__global__ void residual_kernel(const void* g, float* L, int64_t n) {
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n;
       i += (int64_t)gridDim.x * blockDim.x) {
    const float2 x = load_elem<DT>(g, i);
    if (Dt<DT>::cplx) {
      const float2 l = ((const float2*)L)[i];
      ((float2*)L)[i] = make_float2(x.x - l.x, x.y - l.y);
    } else {
      L[i] = x.x - L[i];
    }
  }
}

template <bool CPLX>
__global__ void scatter_add_kernel(float* L, const int64_t* omega, int64_t k, const float* upd) {
  for (int64_t j = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; j < k;
       j += (int64_t)gridDim.x * blockDim.x) {
    int64_t i = omega[j];
    if (CPLX) {
      float2 u = ((const float2*)upd)[j];
      float2* p = (float2*)L + i;
      float2 x = *p;
      *p = make_float2(x.x + u.x, x.y + u.y);
    } else {
      L[i] += upd[j];
    }
  }
}

template <int DT>
__global__ void weight_update_kernel(void* w, const float* L, int64_t n, float decay, float lr) {
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n;
       i += (int64_t)gridDim.x * blockDim.x) {
    float2 wv = load_rw<DT>(w, i);
    float2 d = Dt<DT>::cplx ? ((const float2*)L)[i] : make_float2(L[i], 0.f);
    float2 nv = make_float2(__fmaf_rn(-lr, d.x, wv.x * decay), __fmaf_rn(-lr, d.y, wv.y * decay));
    store_elem<DT>(w, i, nv);
  }
}

// Coefficient matrices of the mode products from U (I x r, complex fp32):
//   P (r x I): P[j][i] = conj(U[i][j])   (projection, X x_n U^H)
//   E (I x r): E[i][j] = U[i][j]         (expansion,  X x_n U)
// Real tensors get real (float) matrices holding the real parts.
__global__ void coef_kernel(const float2* U, int64_t I, int64_t r, bool cplx, float* P, float* E) {
  for (int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; e < I * r;
       e += (int64_t)gridDim.x * blockDim.x) {
    int64_t j = e / I, i = e - j * I;
    float2 u = U[i * r + j];
    float2 w = U[e];
    if (cplx) {
      ((float2*)P)[e] = make_float2(u.x, -u.y);
      ((float2*)E)[e] = w;
    } else {
      P[e] = u.x;
      E[e] = w.x;
    }
  }
}

// The small-matrix kernel when M fits its shared memory, else the tiled one.
template <class S, bool CPLX>
void launch_product(S src, int64_t A, int64_t K, int64_t B, const float* M, int64_t J, float* Y,
                    cudaStream_t s, dim3 grid) {
  if (J * K <= SP_MAXMK)
    mode_product_small_kernel<S, CPLX><<<grid_for(A * B, SP_T), SP_T, 0, s>>>(src, A, K, B, M, J, Y);
  else
    mode_product_kernel<S, CPLX><<<grid, MT, 0, s>>>(src, A, K, B, M, J, Y);
}

template <int DT>
cudaError_t launch_first(const void* X, const uint32_t* bits, int64_t A, int64_t K, int64_t B,
                         const float* M, int64_t J, float* Y, cudaStream_t s, dim3 grid) {
  Src<DT, Dt<DT>::cplx> src{X, bits};
  launch_product<Src<DT, Dt<DT>::cplx>, Dt<DT>::cplx>(src, A, K, B, M, J, Y, s, grid);
  return cudaGetLastError();
}

}  // namespace

cudaError_t sparse_adam(const void* g, int dt, const int64_t* omega, int64_t k, float* m,
                        float* v, const AdamConst& a, float* upd, cudaStream_t s, const float* L) {
  if (k <= 0) return cudaSuccess;
  int grid = grid_for(k);
  switch (dt) {
    case TGD_R32: sparse_adam_kernel<TGD_R32><<<grid, 256, 0, s>>>(g, L, omega, k, m, v, a, upd); break;
    case TGD_C64: sparse_adam_kernel<TGD_C64><<<grid, 256, 0, s>>>(g, L, omega, k, m, v, a, upd); break;
    case TGD_C32H: sparse_adam_kernel<TGD_C32H><<<grid, 256, 0, s>>>(g, L, omega, k, m, v, a, upd); break;
    case TGD_R16: sparse_adam_kernel<TGD_R16><<<grid, 256, 0, s>>>(g, L, omega, k, m, v, a, upd); break;
    default: return cudaErrorInvalidValue;
  }
  return cudaGetLastError();
}

cudaError_t residual_in_place(const void* g, int dt, float* L, int64_t n, cudaStream_t s) {
  int grid = grid_for(n);
  switch (dt) {
    case TGD_R32: residual_kernel<TGD_R32><<<grid, 256, 0, s>>>(g, L, n); break;
    case TGD_C64: residual_kernel<TGD_C64><<<grid, 256, 0, s>>>(g, L, n); break;
    case TGD_C32H: residual_kernel<TGD_C32H><<<grid, 256, 0, s>>>(g, L, n); break;
    case TGD_R16: residual_kernel<TGD_R16><<<grid, 256, 0, s>>>(g, L, n); break;
    default: return cudaErrorInvalidValue;
  }
  return cudaGetLastError();
}

cudaError_t mode_product(const void* X, int src_dt, const uint32_t* bits, bool cplx, int64_t A,
                         int64_t K, int64_t B, const float* M, int64_t J, float* Y,
                         cudaStream_t s) {
  dim3 grid((unsigned)ceil_div(A * B, TC), (unsigned)ceil_div(J, TJ));
  switch (src_dt) {
    case TGD_R32: return launch_first<TGD_R32>(X, bits, A, K, B, M, J, Y, s, grid);
    case TGD_C64: return launch_first<TGD_C64>(X, bits, A, K, B, M, J, Y, s, grid);
    case TGD_C32H: return launch_first<TGD_C32H>(X, bits, A, K, B, M, J, Y, s, grid);
    case TGD_R16: return launch_first<TGD_R16>(X, bits, A, K, B, M, J, Y, s, grid);
    default:
      break;
  }
  if (cplx)
    launch_product<Src<-1, true>, true>(Src<-1, true>{X, nullptr}, A, K, B, M, J, Y, s, grid);
  else
    launch_product<Src<-1, false>, false>(Src<-1, false>{X, nullptr}, A, K, B, M, J, Y, s, grid);
  return cudaGetLastError();
}

cudaError_t masked_copy(const void* g, int dt, const uint32_t* bits, int64_t n, float* out,
                        cudaStream_t s) {
  int grid = grid_for(n);
  switch (dt) {
    case TGD_R32: masked_copy_kernel<TGD_R32><<<grid, 256, 0, s>>>(g, bits, n, out); break;
    case TGD_C64: masked_copy_kernel<TGD_C64><<<grid, 256, 0, s>>>(g, bits, n, out); break;
    case TGD_C32H: masked_copy_kernel<TGD_C32H><<<grid, 256, 0, s>>>(g, bits, n, out); break;
    case TGD_R16: masked_copy_kernel<TGD_R16><<<grid, 256, 0, s>>>(g, bits, n, out); break;
    default: return cudaErrorInvalidValue;
  }
  return cudaGetLastError();
}

cudaError_t core_adam(float* c, int64_t n, float* m, float* v, const AdamConst& a,
                      cudaStream_t s) {
  core_adam_kernel<<<grid_for(n), 256, 0, s>>>(c, n, m, v, a);
  return cudaGetLastError();
}

cudaError_t scatter_add(float* L, bool cplx, const int64_t* omega, int64_t k, const float* upd,
                        cudaStream_t s) {
  if (k <= 0) return cudaSuccess;
  if (cplx)
    scatter_add_kernel<true><<<grid_for(k), 256, 0, s>>>(L, omega, k, upd);
  else
    scatter_add_kernel<false><<<grid_for(k), 256, 0, s>>>(L, omega, k, upd);
  return cudaGetLastError();
}

cudaError_t weight_update(void* w, int dt, const float* L, int64_t n, float decay, float lr,
                          cudaStream_t s) {
  int grid = grid_for(n);
  switch (dt) {
    case TGD_R32: weight_update_kernel<TGD_R32><<<grid, 256, 0, s>>>(w, L, n, decay, lr); break;
    case TGD_C64: weight_update_kernel<TGD_C64><<<grid, 256, 0, s>>>(w, L, n, decay, lr); break;
    case TGD_C32H: weight_update_kernel<TGD_C32H><<<grid, 256, 0, s>>>(w, L, n, decay, lr); break;
    case TGD_R16: weight_update_kernel<TGD_R16><<<grid, 256, 0, s>>>(w, L, n, decay, lr); break;
    default: return cudaErrorInvalidValue;
  }
  return cudaGetLastError();
}

cudaError_t coef_matrices(const float* U, int64_t I, int64_t r, bool cplx, float* P, float* E,
                          cudaStream_t s) {
  coef_kernel<<<grid_for(I * r), 256, 0, s>>>((const float2*)U, I, r, cplx, P, E);
  return cudaGetLastError();
}

}  // namespace tgd
