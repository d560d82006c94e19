// Refresh of the Tucker factors: mode-n Gram matrices of the residual and a
// batched Hermitian eigensolver.
//
// The Pith review of TensorGRaD ("What carries the argument") computes the
// factors U^(n) with a higher-order SVD of the residual R = G - S and reuses
// them for T steps. Plain HOSVD takes U_n as the leading r_n left singular
// vectors of the mode-n unfolding R_(n) (the review's appended Appendix K
// defines the unfolding), i.e. the leading eigenvectors of the Hermitian
// positive semidefinite Gram R_(n) R_(n)^H.
//
// Gram: fp32 products accumulated per block over a slice of the unfolding's
// columns (deterministic split), the partial sums added in fp64 in a fixed
// order. The residual is never stored: the gradient is read in its storage
// type and entries of Omega (a bitmask) read as zero.
//
// Eigensolver: two-sided Jacobi in fp64 with the round-robin parallel
// ordering (n/2 disjoint rotations per round), one thread block per matrix,
// matrices in shared memory when n <= 64 and in global scratch otherwise.
// Output: eigenvalues descending (ties to the lower index) and the leading
// r_n eigenvectors, each scaled by a unit phase that makes its largest-
// magnitude entry (ties to the lowest row) real and positive.

#include "common.cuh"
#include "kernels.h"

namespace tgd {
namespace {

constexpr int TI = 32;   // Gram tile edge
constexpr int CC = 32;   // columns per Gram chunk
constexpr int GT = 256;  // threads per Gram block

struct GramGeom {
  int64_t A, I, B, ncol;
  int nti, npairs, nsplit;
  int64_t cols_per_split;
};

GramGeom gram_geom(int nd, const int64_t* dims, int n) {
  GramGeom g;
  g.A = 1;
  g.B = 1;
  for (int q = 0; q < n; ++q) g.A *= dims[q];
  for (int q = n + 1; q < nd; ++q) g.B *= dims[q];
  g.I = dims[n];
  g.ncol = g.A * g.B;
  g.nti = (int)ceil_div(g.I, TI);
  g.npairs = g.nti * (g.nti + 1) / 2;
  int target = 148 * 4;
  int64_t ns = ceil_div(target, g.npairs);
  int64_t max_ns = ceil_div(g.ncol, 64);
  if (ns > max_ns) ns = max_ns;
  if (ns < 1) ns = 1;
  g.nsplit = (int)ns;
  g.cols_per_split = ceil_div(ceil_div(g.ncol, g.nsplit), CC) * CC;
  return g;
}

template <int DT>
__device__ __forceinline__ float2 masked_elem(const void* g, const uint32_t* bits, int64_t idx) {
  if (bits && mask_bit(bits, idx)) return make_float2(0.f, 0.f);
  return load_elem<DT>(g, idx);
}

template <int DT>
__global__ void __launch_bounds__(GT) gram_partial_kernel(const void* g, const uint32_t* bits,
                                                          GramGeom geo, float2* partial) {
  __shared__ float2 Xi[TI][CC + 1];
  __shared__ float2 Xj[TI][CC + 1];
  // tile pair (ti <= tj) from the linear pair index
  int pr = blockIdx.x, ti = 0;
  while (pr >= geo.nti - ti) {
    pr -= geo.nti - ti;
    ++ti;
  }
  const int tj = ti + pr;
  const int split = blockIdx.y;
  const int64_t c_begin = (int64_t)split * geo.cols_per_split;
  int64_t c_end = c_begin + geo.cols_per_split;
  if (c_end > geo.ncol) c_end = geo.ncol;
  const int il = threadIdx.x >> 3;  // 0..31
  const int jl = threadIdx.x & 7;   // + 8q
  float2 acc[4];
  for (int q = 0; q < 4; ++q) acc[q] = make_float2(0.f, 0.f);
  const bool col_fast = geo.B >= CC;
  for (int64_t c0 = c_begin; c0 < c_end; c0 += CC) {
    for (int e = threadIdx.x; e < TI * CC; e += GT) {
      int row, col;
      if (col_fast) {
        row = e / CC;
        col = e % CC;
      } else {
        col = e / TI;
        row = e % TI;
      }
      int64_t c = c0 + col;
      int64_t ri = (int64_t)ti * TI + row, rj = (int64_t)tj * TI + row;
      float2 vi = make_float2(0.f, 0.f), vj = vi;
      if (c < c_end) {
        int64_t a = c / geo.B, b = c - a * geo.B;
        int64_t base = a * geo.I * geo.B + b;
        if (ri < geo.I) vi = masked_elem<DT>(g, bits, base + ri * geo.B);
        if (rj < geo.I) vj = masked_elem<DT>(g, bits, base + rj * geo.B);
      }
      Xi[row][col] = vi;
      Xj[row][col] = vj;
    }
    __syncthreads();
#pragma unroll 8
    for (int cc = 0; cc < CC; ++cc) {
      float2 a = Xi[il][cc];
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        float2 b = Xj[jl + 8 * q][cc];
        // a * conj(b)
        acc[q].x = __fmaf_rn(a.x, b.x, __fmaf_rn(a.y, b.y, acc[q].x));
        acc[q].y = __fmaf_rn(a.y, b.x, __fmaf_rn(-a.x, b.y, acc[q].y));
      }
    }
    __syncthreads();
  }
  const int64_t I = geo.I;
  int64_t gi = (int64_t)ti * TI + il;
  float2* out = partial + (int64_t)split * I * I;
  for (int q = 0; q < 4; ++q) {
    int64_t gj = (int64_t)tj * TI + jl + 8 * q;
    if (gi < I && gj < I) out[gi * I + gj] = acc[q];
  }
}

__global__ void gram_reduce_kernel(const float2* partial, GramGeom geo, double2* gram) {
  const int64_t I = geo.I;
  for (int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; e < I * I;
       e += (int64_t)gridDim.x * blockDim.x) {
    int64_t i = e / I, j = e - i * I;
    bool upper = (i / TI) <= (j / TI);
    int64_t src = upper ? i * I + j : j * I + i;
    double sx = 0, sy = 0;
    for (int s = 0; s < geo.nsplit; ++s) {
      float2 v = partial[(int64_t)s * I * I + src];
      sx += (double)v.x;
      sy += (double)v.y;
    }
    gram[e] = upper ? make_double2(sx, sy) : make_double2(sx, -sy);
  }
}

// ------------------------------------------------------------- eigensolver
__device__ __forceinline__ double2 zmul(double2 a, double2 b) {
  return make_double2(a.x * b.x - a.y * b.y, a.x * b.y + a.y * b.x);
}
__device__ __forceinline__ double zabs2(double2 a) { return a.x * a.x + a.y * a.y; }

constexpr int ET = 512;  // threads per eigensolver block
constexpr int MAXN = 256;

__device__ double block_sum(double v, double* red) {
  for (int o = 16; o; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = v;
  __syncthreads();
  double t = 0;
  for (int w = 0; w < (int)(blockDim.x >> 5); ++w) t += red[w];
  __syncthreads();
  return t;
}

__global__ void __launch_bounds__(ET) eig_kernel(const EigJob* jobs) {
  const EigJob J = jobs[blockIdx.x];
  const int n = J.n;
  extern __shared__ double2 dyn[];
  __shared__ int rp[MAXN / 2], rq[MAXN / 2];
  __shared__ double rcs[MAXN / 2], rsn[MAXN / 2];
  __shared__ double2 rph[MAXN / 2];
  __shared__ double red[ET / 32];
  __shared__ double ev[MAXN];
  __shared__ int col_of_rank[MAXN];
  double2* A;
  double2* V;
  if (n <= 64) {
    A = dyn;
    V = dyn + n * n;
  } else {
    A = (double2*)J.work;
    V = A + (int64_t)n * n;
  }
  const double2* G = (const double2*)J.gram;
  for (int e = threadIdx.x; e < n * n; e += blockDim.x) {
    A[e] = G[e];
    V[e] = make_double2((e / n) == (e % n) ? 1.0 : 0.0, 0.0);
  }
  __syncthreads();
  double fro_part = 0;
  for (int e = threadIdx.x; e < n * n; e += blockDim.x) fro_part += zabs2(A[e]);
  const double fro = block_sum(fro_part, red);
  const int m = n + (n & 1);
  const int npairs = m / 2;
  for (int sweep = 0; sweep < 40; ++sweep) {
    double off_part = 0;
    for (int e = threadIdx.x; e < n * n; e += blockDim.x) {
      int i = e / n, j = e - i * n;
      if (i < j) off_part += zabs2(A[e]);
    }
    double off = block_sum(off_part, red);
    if (off <= 1e-24 * fro || off == 0.0) break;
    for (int round = 0; round < m - 1; ++round) {
      for (int k = threadIdx.x; k < npairs; k += blockDim.x) {
        int p, q;
        if (k == 0) {
          p = round;
          q = m - 1;
        } else {
          p = (round + k) % (m - 1);
          q = (round - k + (m - 1)) % (m - 1);
        }
        if (p > q) {
          int t = p;
          p = q;
          q = t;
        }
        rp[k] = -1;
        if (q < n) {
          double2 apq = A[p * n + q];
          double r = sqrt(zabs2(apq));
          if (r > 0.0) {
            double app = A[p * n + p].x, aqq = A[q * n + q].x;
            double tau = (aqq - app) / (2.0 * r);
            double t = (tau >= 0 ? 1.0 : -1.0) / (fabs(tau) + sqrt(1.0 + tau * tau));
            double c = 1.0 / sqrt(1.0 + t * t);
            rp[k] = p;
            rq[k] = q;
            rcs[k] = c;
            rsn[k] = t * c;
            rph[k] = make_double2(apq.x / r, apq.y / r);  // e = apq / |apq|
          }
        }
      }
      __syncthreads();
      // A <- A J and V <- V J: columns p, q of every row.
      for (int w = threadIdx.x; w < n * npairs; w += blockDim.x) {
        int i = w / npairs, k = w - i * npairs;
        int p = rp[k];
        if (p < 0) continue;
        int q = rq[k];
        double c = rcs[k], s = rsn[k];
        double2 ec = make_double2(rph[k].x, -rph[k].y);
        double2 xp = A[i * n + p], xq = zmul(A[i * n + q], ec);
        A[i * n + p] = make_double2(c * xp.x - s * xq.x, c * xp.y - s * xq.y);
        A[i * n + q] = make_double2(s * xp.x + c * xq.x, s * xp.y + c * xq.y);
        xp = V[i * n + p];
        xq = zmul(V[i * n + q], ec);
        V[i * n + p] = make_double2(c * xp.x - s * xq.x, c * xp.y - s * xq.y);
        V[i * n + q] = make_double2(s * xp.x + c * xq.x, s * xp.y + c * xq.y);
      }
      __syncthreads();
      // A <- J^H A: rows p, q of every column.
      for (int w = threadIdx.x; w < npairs * n; w += blockDim.x) {
        int k = w / n, j = w - k * n;
        int p = rp[k];
        if (p < 0) continue;
        int q = rq[k];
        double c = rcs[k], s = rsn[k];
        double2 xp = A[p * n + j], xq = zmul(A[q * n + j], rph[k]);
        A[p * n + j] = make_double2(c * xp.x - s * xq.x, c * xp.y - s * xq.y);
        A[q * n + j] = make_double2(s * xp.x + c * xq.x, s * xp.y + c * xq.y);
      }
      __syncthreads();
      for (int k = threadIdx.x; k < npairs; k += blockDim.x) {
        int p = rp[k];
        if (p < 0) continue;
        int q = rq[k];
        A[p * n + q] = make_double2(0.0, 0.0);
        A[q * n + p] = make_double2(0.0, 0.0);
        A[p * n + p].y = 0.0;
        A[q * n + q].y = 0.0;
      }
      __syncthreads();
    }
  }
  for (int i = threadIdx.x; i < n; i += blockDim.x) ev[i] = A[i * n + i].x;
  __syncthreads();
  for (int i = threadIdx.x; i < n; i += blockDim.x) {
    double li = ev[i];
    int rank = 0;
    for (int j = 0; j < n; ++j) rank += (ev[j] > li) || (ev[j] == li && j < i);
    col_of_rank[rank] = i;
    J.evals[rank] = li;
  }
  __syncthreads();
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5, nw = blockDim.x >> 5;
  for (int rr = wid; rr < J.r; rr += nw) {
    int c = col_of_rank[rr];
    double best = -1.0;
    int bi = 0;
    for (int row = lane; row < n; row += 32) {
      double mg = zabs2(V[row * n + c]);
      if (mg > best) {
        best = mg;
        bi = row;
      }
    }
    for (int o = 16; o; o >>= 1) {
      double ob = __shfl_xor_sync(0xffffffffu, best, o);
      int oi = __shfl_xor_sync(0xffffffffu, bi, o);
      if (ob > best || (ob == best && oi < bi)) {
        best = ob;
        bi = oi;
      }
    }
    double2 piv = V[bi * n + c];
    double pm = sqrt(zabs2(piv));
    double2 ph = pm > 0 ? make_double2(piv.x / pm, -piv.y / pm) : make_double2(1.0, 0.0);
    for (int row = lane; row < n; row += 32) {
      double2 u = zmul(V[row * n + c], ph);
      ((float2*)J.U)[(int64_t)row * J.r + rr] = make_float2((float)u.x, (float)u.y);
    }
  }
}

}  // namespace

size_t gram_partial_bytes(int nd, const int64_t* dims, int n) {
  GramGeom g = gram_geom(nd, dims, n);
  return sizeof(float2) * (size_t)g.nsplit * g.I * g.I;
}

cudaError_t mode_gram(const void* g, int dt, const uint32_t* bits, int nd, const int64_t* dims,
                      int n, float* partial, double* gram, cudaStream_t s) {
  GramGeom geo = gram_geom(nd, dims, n);
  dim3 grid(geo.npairs, geo.nsplit);
  switch (dt) {
    case TGD_R32:
      gram_partial_kernel<TGD_R32><<<grid, GT, 0, s>>>(g, bits, geo, (float2*)partial);
      break;
    case TGD_C64:
      gram_partial_kernel<TGD_C64><<<grid, GT, 0, s>>>(g, bits, geo, (float2*)partial);
      break;
    case TGD_C32H:
      gram_partial_kernel<TGD_C32H><<<grid, GT, 0, s>>>(g, bits, geo, (float2*)partial);
      break;
    case TGD_R16:
      gram_partial_kernel<TGD_R16><<<grid, GT, 0, s>>>(g, bits, geo, (float2*)partial);
      break;
    default:
      return cudaErrorInvalidValue;
  }
  int64_t cells = geo.I * geo.I;
  int blocks = (int)ceil_div(cells, 256);
  gram_reduce_kernel<<<blocks, 256, 0, s>>>((const float2*)partial, geo, (double2*)gram);
  return cudaGetLastError();
}

size_t eig_work_doubles(int n) { return n > 64 ? (size_t)4 * n * n : 0; }

cudaError_t batched_eigh(const EigJob* jobs_host, int njobs, EigJob* jobs_dev, cudaStream_t s) {
  if (njobs <= 0) return cudaSuccess;
  int smem_n = 0;
  for (int j = 0; j < njobs; ++j) {
    if (jobs_host[j].n > MAXN || jobs_host[j].r > jobs_host[j].n) return cudaErrorInvalidValue;
    if (jobs_host[j].n <= 64 && jobs_host[j].n > smem_n) smem_n = jobs_host[j].n;
  }
  size_t smem = (size_t)2 * smem_n * smem_n * sizeof(double2);
  cudaError_t e = cudaFuncSetAttribute(eig_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)(smem > 0 ? smem : 1));
  if (e != cudaSuccess) return e;
  e = cudaMemcpyAsync(jobs_dev, jobs_host, sizeof(EigJob) * njobs, cudaMemcpyHostToDevice, s);
  if (e != cudaSuccess) return e;
  eig_kernel<<<njobs, ET, smem, s>>>(jobs_dev);
  return cudaGetLastError();
}

}  // namespace tgd
