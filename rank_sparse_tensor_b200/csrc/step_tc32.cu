// Tensor-core (tcgen05, sm_100a) path of the TensorGRaD step for fp32
// gradients and weights (real fp32 and complex64).
//
// The step is the one of the nullthought.net TensorGRaD summary (section 三:
// sparse part first, Tucker part on the residual, separate Adam updates, the
// sparse update scatter-added in place into the rebuilt tensor) and of
// Theorem 2 in the paper text appended to the Pith review (project with the
// conjugate-transposed factors, Adam on the core, project back):
//
//   sparse_adam   S~ = lambda Adam(G[Omega]) (CUDA cores, in Omega order)
//   mode_gemm32   C = R x_n U_n^H for every projected mode, last mode first;
//                 the first contraction reads G itself with Omega zeroed
//                 through the index set's bit mask (R is never stored)
//   core_adam     C~ = Adam(C) in place
//   mode_gemm32   C~ x_n U_n for every projected mode, first mode first; the
//                 last one does not store Delta: its epilogue adds lambda S~
//                 where the output index is in Omega and writes
//                 W <- W (1 - lr wd) - lr (Delta + lambda S~), one rounding
//
// Every mode product is one tcgen05 GEMM per 128 unfolding rows (a, b) of
// the tensor X[a][k][b]: A = the rows' K values gathered by the threads
// (coalesced across threads when b varies fastest), B = the factor's
// embedding (complex products as real 2 x 2 blocks, as in step_tc.cu),
// accumulators in TMEM. fp32 operands are split into three bf16 parts, x =
// h + m + l with h = bf16(x), m = bf16(x - h), l = bf16(x - h - m), and the
// six products hh, hm, mh, hl, lh, mm are accumulated in fp32; the dropped
// products (ml, lm, ll) and the rounding of l are below 2^-24 of |x||u|, the
// accuracy of an fp32 FMA, against 2^-9 for one bf16 operand.
// Every wait is bounded and reports TGD_ERR_TIMEOUT.

#include <algorithm>
#include <vector>

#include "common.cuh"
#include "kernels.h"
#include "step_tc32.h"
#include "tc_ptx.cuh"

namespace tgd {
namespace {

using namespace ptx;

constexpr int G32T = 128;                    // threads = GEMM rows per CTA
constexpr uint32_t G32_LBO = 2048;           // A tile: 128 rows x 16 B between K core matrices
constexpr int G32_KMAX = 64;                 // bf16 K values per chunk at most
constexpr uint64_t G32_WAIT_NS = 2000000000ull;

__host__ __device__ __forceinline__ uint32_t kmaj(uint32_t row, uint32_t k, uint32_t lbo) {
  return (row & 7u) * 16u + (row >> 3) * 128u + (k >> 3) * lbo + (k & 7u) * 2u;
}

__device__ __forceinline__ uint16_t bf16_bits(float x) {
  __nv_bfloat16 h = __float2bfloat16_rn(x);
  return *reinterpret_cast<uint16_t*>(&h);
}
__device__ __forceinline__ float bf16_val(uint16_t b) { return __uint_as_float((uint32_t)b << 16); }
// x = h + m + l (+ a remainder below 2^-24 |x|): the three bf16 parts of two
// neighbouring K values, packed in pairs (lo half = even K)
__device__ __forceinline__ uint32_t bf2_bits(float x, float y) {  // (x lo, y hi), each rounded to nearest
  __nv_bfloat162 h = __floats2bfloat162_rn(x, y);
  return *reinterpret_cast<uint32_t*>(&h);
}
__device__ __forceinline__ void split3(float x, float y, uint32_t& h, uint32_t& m, uint32_t& l) {
  h = bf2_bits(x, y);
  const float rx = x - __uint_as_float(h << 16), ry = y - __uint_as_float(h & 0xffff0000u);
  m = bf2_bits(rx, ry);
  l = bf2_bits(rx - __uint_as_float(m << 16), ry - __uint_as_float(m & 0xffff0000u));
}

struct MG32Args {
  const float* X;         // [a][k][b] fp32 values (re, im interleaved when complex)
  const uint32_t* bits;   // Omega's bit mask when X is the gradient (zeros there), else null
  int64_t rows, K, B;     // rows = A * B unfolding rows; K entries along the mode
  float* Y;               // [a][j][b] output (unused when the epilogue updates W)
  int64_t J;
  const uint8_t* img;     // B operand blocks [n block][k chunk][h, m, l], NT x kp bf16 each
  int NT, nkc, nstage;
  int kp;                 // bf16 K values per chunk: a multiple of 16, at most 64
  uint32_t tmem_cols;
  // epilogue of the last expansion: the weight update
  float* W;               // the weights, the full tensor (Y's layout)
  const float* S;         // lambda S~ in Omega order
  const int64_t* wrank;   // Omega entries before each 32-element word of the mask
  const uint32_t* wbits;  // Omega's bit mask for the update
  float decay, lr;
  // B == 1 (the innermost mode): a CTA's rows of X, and of Y or W, are one
  // contiguous range each; they then move by bulk copy through shared memory
  // at these offsets (0: not staged)
  uint32_t xs_off, os_off;
  // ... and Omega's mask words over those ranges (with the output range's
  // word ranks when the weights are updated), by cp.async (0: not staged)
  uint32_t xm_off, om_off;
  int64_t tile0;          // first 128-row tile of the launch (the grid's x counts from it)
  // the factor itself (I x ur, complex pairs or reals) for the CUDA-core
  // innermost-mode kernel: M = conj(U) (ukind 0) or U^T (ukind 1)
  const float* Uf;
  int ur, ukind;
  int* err;
};

// Asynchronous 4- and 8-byte copies global -> shared.
__device__ __forceinline__ void cpa4(void* dst, const void* src) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(smem_u32(dst)), "l"(src) : "memory");
}
__device__ __forceinline__ void cpa8(void* dst, const void* src) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 8;" ::"r"(smem_u32(dst)), "l"(src) : "memory");
}
__device__ __forceinline__ void cpa_wait_all() {
  asm volatile("cp.async.commit_group;\n\tcp.async.wait_group 0;" ::: "memory");
}

// Y[a][j][b] = sum_k X[a][k][b] M[k][j] over one 128-row block of the
// unfolding and one NT-wide block of (j, re/im) columns. K advances in chunks
// of kp real values (kp / 2 complex; kp = 64, or the whole K rounded up to 16
// when it fits one chunk), in two stages when there are several
// chunks: the chunk's operand image arrives by bulk copy while the threads
// split and store their rows' values, and the next chunk's values are loaded
// while its MMAs run.
// WUPD: instead of storing Y, W[o] <- W[o] decay - lr (Y[o] + S~[o in Omega]).
template <bool CPLX, bool WUPD>
__global__ void __launch_bounds__(G32T) mode_gemm32_kernel(const MG32Args p) {
  extern __shared__ __align__(1024) uint8_t smem[];
  const int kq = p.kp / 8;                       // K core matrices per chunk
  const uint32_t atile = (uint32_t)kq * G32_LBO;  // one part of A: 128 rows x kp bf16
  const uint32_t b_bytes = (uint32_t)p.NT * p.kp * 2;
  const uint32_t stage_bytes = 3 * atile + 3 * b_bytes;
  // stage s: A parts h, m, l, then B parts h, m, l
  auto Apart = [&](int s, int part) { return smem + (uint32_t)s * stage_bytes + (uint32_t)part * atile; };
  auto Bpart = [&](int s, int part) {
    return smem + (uint32_t)s * stage_bytes + 3 * atile + (uint32_t)part * b_bytes;
  };
  // [0,1] MMAs done, [2,3] B landed, [4] staged rows landed
  uint64_t* bars = (uint64_t*)(smem + (uint32_t)p.nstage * stage_bytes);
  uint32_t* tslot = (uint32_t*)(bars + 5);
  __shared__ int s_abort;
  const int tid = threadIdx.x, warp = tid >> 5;
  const uint32_t lane_base = (uint32_t)(warp * 32) << 16;
  const int64_t tile = p.tile0 + blockIdx.x;
  const int64_t rho = tile * G32T + tid;
  const bool valid = rho < p.rows;
  const int64_t a = valid ? rho / p.B : 0, b = valid ? rho - a * p.B : 0;
  const int64_t xbase = a * p.K * p.B + b;  // element index of (a, k = 0, b)
  // staging applies to CTAs whose 128 rows all exist
  const bool full_cta = (tile + 1) * G32T <= p.rows;
  const bool st_in = p.xs_off != 0 && full_cta;
  const bool st_out = p.os_off != 0 && full_cta;
  constexpr int ESZ = CPLX ? 8 : 4;
  float* xs = (float*)(smem + p.xs_off);
  float* os = (float*)(smem + p.os_off);
  const int64_t a0 = tile * G32T;  // first row (B == 1 when staged)
  if (tid == 0) {
    s_abort = 0;
    for (int i = 0; i < 5; ++i) mbar_init(&bars[i], 1);
    fence_mbar_init();
    // the staged rows: X (and W, whose update happens in shared memory)
    const uint32_t xb = st_in ? (uint32_t)(G32T * p.K * ESZ) : 0u;
    const uint32_t wb = (st_out && WUPD) ? (uint32_t)(G32T * p.J * ESZ) : 0u;
    if (xb + wb) {
      mbar_expect_tx(&bars[4], xb + wb);
      if (xb) bulk_g2s(xs, (const uint8_t*)p.X + a0 * p.K * ESZ, xb, &bars[4]);
      if (wb) bulk_g2s(os, (const uint8_t*)p.W + a0 * p.J * ESZ, wb, &bars[4]);
    }
  }
  // Omega's words over the staged ranges (the CTA's rows are contiguous)
  const bool xm = p.xm_off != 0 && st_in && p.bits;
  const bool om = p.om_off != 0 && st_out && WUPD;
  const int64_t xw0 = (a0 * p.K) >> 5, ow0 = (a0 * p.J) >> 5;
  uint32_t* xmw = (uint32_t*)(smem + p.xm_off);
  uint32_t* omw = (uint32_t*)(smem + p.om_off);
  const int onw = (int)((((a0 + G32T) * p.J - 1) >> 5) - ow0 + 1);
  int64_t* omr = (int64_t*)(omw + ((onw + 1) & ~1));
  if (xm) {
    const int nw = (int)((((a0 + G32T) * p.K - 1) >> 5) - xw0 + 1);
    for (int w = tid; w < nw; w += G32T) cpa4(xmw + w, p.bits + xw0 + w);
  }
  if (om)
    for (int w = tid; w < onw; w += G32T) {
      cpa4(omw + w, p.wbits + ow0 + w);
      cpa8(omr + w, p.wrank + ow0 + w);
    }
  if (xm || om) cpa_wait_all();
  __syncthreads();
  if (warp == 0) tmem_alloc(tslot, p.tmem_cols);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t dt = *tslot;
  const uint32_t lbo_b = (uint32_t)(p.NT / 8) * 128;
  const uint32_t idesc = idesc_f16(1, 128, p.NT);
  const uint8_t* img = p.img + (int64_t)blockIdx.y * p.nkc * 3 * b_bytes;
  uint32_t issued[2] = {0, 0}, waited[2] = {0, 0}, bloaded[2] = {0, 0};
  constexpr int KE = CPLX ? G32_KMAX / 2 : G32_KMAX;  // entries per chunk at most
  constexpr int NV = G32_KMAX;                        // fp32 values per chunk and row
  const int ke = CPLX ? p.kp / 2 : p.kp;              // entries per chunk
  auto wait_all = [&](uint64_t* bar, uint32_t parity) -> bool {
    if (tid == 0 && !mbar_wait(bar, parity, G32_WAIT_NS)) {
      atomicOr(p.err, DEV_ERR_TIMEOUT);
      s_abort = 1;
    }
    __syncthreads();
    return s_abort == 0;
  };
  // every thread waits (bounded) for the staged rows: the data of a bulk copy
  // is visible to the threads that observe its barrier phase complete
  auto wait_staged = [&]() -> bool {
    if (!mbar_wait(&bars[4], 0, G32_WAIT_NS)) {
      atomicOr(p.err, DEV_ERR_TIMEOUT);
      s_abort = 1;
    }
    __syncthreads();
    return s_abort == 0;
  };
  float v[NV];
  // this row's values from the staged rows (one chunk: K <= 32 complex / 64 real)
  auto load_x_staged = [&]() {
#pragma unroll
    for (int i = 0; i < KE; ++i) {
      if (i >= ke) break;
      float2 x = make_float2(0.f, 0.f);
      if (i < p.K) {
        const int64_t idx = xbase + i;
        const uint32_t word = !p.bits ? 0u : (xm ? xmw[(idx >> 5) - xw0] : __ldg(p.bits + (idx >> 5)));
        if (!((word >> (idx & 31)) & 1u)) {
          if (CPLX)
            x = ((const float2*)xs)[tid * p.K + i];
          else
            x.x = xs[tid * p.K + i];
        }
      }
      if (CPLX) {
        v[2 * i] = x.x;
        v[2 * i + 1] = x.y;
      } else {
        v[i] = x.x;
      }
    }
  };
  auto load_x = [&](int kc) {
#pragma unroll
    for (int i = 0; i < KE; ++i) {
      if (i >= ke) break;
      const int64_t k = (int64_t)kc * ke + i;
      float2 x = make_float2(0.f, 0.f);
      if (valid && k < p.K) {
        const int64_t idx = xbase + k * p.B;
        if (!(p.bits && ((__ldg(p.bits + (idx >> 5)) >> (idx & 31)) & 1u))) {
          if (CPLX)
            x = __ldg((const float2*)p.X + idx);
          else
            x.x = __ldg(p.X + idx);
        }
      }
      if (CPLX) {
        v[2 * i] = x.x;
        v[2 * i + 1] = x.y;
      } else {
        v[i] = x.x;
      }
    }
  };
  bool staged_waited = false;
  if (st_in) {
    staged_waited = true;
    if (wait_staged()) load_x_staged();
  } else {
    load_x(0);
  }
  const int ns = p.nstage;
  // (s_abort is read right after barriers only, where every thread sees the
  // same value)
  for (int kc = 0; kc < p.nkc && !s_abort; ++kc) {
    const int s = kc % ns;
    if (kc >= ns) {
      const bool ok = wait_all(&bars[s], waited[s] & 1u);
      waited[s]++;
      if (!ok) break;
      tc_fence_after();
    }
    if (tid == 0) {
      mbar_expect_tx(&bars[2 + s], 3 * b_bytes);
      bulk_g2s(Bpart(s, 0), img + (int64_t)kc * 3 * b_bytes, 3 * b_bytes, &bars[2 + s]);
      bloaded[s]++;
    }
    // this row's 64 K values -> the h, m and l A tiles (8 core matrices each)
#pragma unroll
    for (int q = 0; q < G32_KMAX / 8; ++q) {
      if (q >= kq) break;
      uint32_t h[4], m[4], l[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) split3(v[8 * q + 2 * u], v[8 * q + 2 * u + 1], h[u], m[u], l[u]);
      *(uint4*)(Apart(s, 0) + q * G32_LBO + tid * 16) = make_uint4(h[0], h[1], h[2], h[3]);
      *(uint4*)(Apart(s, 1) + q * G32_LBO + tid * 16) = make_uint4(m[0], m[1], m[2], m[3]);
      *(uint4*)(Apart(s, 2) + q * G32_LBO + tid * 16) = make_uint4(l[0], l[1], l[2], l[3]);
    }
    if (kc + 1 < p.nkc) load_x(kc + 1);
    // the chunk's operand image has landed (checked before the barrier, so
    // that every thread reads the same abort flag after it)
    if (tid == 0 && !mbar_wait(&bars[2 + s], (bloaded[s] - 1) & 1u, G32_WAIT_NS)) {
      atomicOr(p.err, DEV_ERR_TIMEOUT);
      s_abort = 1;
    }
    fence_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (s_abort) break;
    if (tid == 0) {
      {
        const uint32_t a0 = smem_u32(Apart(s, 0)), b0 = smem_u32(Bpart(s, 0));
        for (int kk = 0; kk < kq / 2; ++kk) {
          // (A part, B part): hh, hm, mh, hl, lh, mm
#pragma unroll
          for (int pr = 0; pr < 6; ++pr) {
            const uint32_t pa = (0x120100u >> (4 * pr)) & 0xFu, pb = (0x102010u >> (4 * pr)) & 0xFu;
            const uint64_t da = sdesc(a0 + pa * atile + kk * 2 * G32_LBO, G32_LBO, 128);
            const uint64_t db = sdesc(b0 + pb * b_bytes + kk * 2 * lbo_b, lbo_b, 128);
            mma_f16(dt, da, db, idesc, (kc > 0 || kk > 0 || pr > 0) ? 1u : 0u);
          }
        }
        mma_commit(&bars[s]);
        issued[s]++;
      }
    }
  }
  __syncthreads();
  if (!s_abort) {
    const int s = (p.nkc - 1) % ns;
    wait_all(&bars[s], waited[s] & 1u);
    waited[s]++;
    tc_fence_after();
  }
  if (!s_abort && st_out && WUPD && !staged_waited) {
    staged_waited = true;
    wait_staged();
  }
  if (!s_abort && st_out) {
    // rows staged in shared memory: Y written there, or W updated in place
    // (row-major [row][j], the layout of the contiguous range), then one bulk
    // store of the range
    for (int c0 = 0; c0 < p.NT; c0 += 16) {
      float y[16];
      tmem_ld16(dt + lane_base + c0, y);
      constexpr int PER = CPLX ? 8 : 16;
#pragma unroll
      for (int u = 0; u < PER; ++u) {
        const int64_t j = (CPLX ? c0 / 2 : c0) + u;
        if (j >= p.J) continue;
        const int64_t so = (int64_t)tid * p.J + j;
        float dr = CPLX ? y[2 * u] : y[u], di = CPLX ? y[2 * u + 1] : 0.f;
        if (!WUPD) {
          if (CPLX)
            ((float2*)os)[so] = make_float2(dr, di);
          else
            os[so] = dr;
        } else {
          const int64_t o = (a0 + tid) * p.J + j;
          const uint32_t word = om ? omw[(o >> 5) - ow0] : __ldg(p.wbits + (o >> 5));
          const uint32_t bit = (uint32_t)(o & 31);
          if ((word >> bit) & 1u) {
            const int64_t e = (om ? omr[(o >> 5) - ow0] : __ldg(p.wrank + (o >> 5))) + __popc(word & ((1u << bit) - 1u));
            if (CPLX) {
              const float2 sv = __ldg((const float2*)p.S + e);
              dr += sv.x;
              di += sv.y;
            } else {
              dr += __ldg(p.S + e);
            }
          }
          if (CPLX) {
            const float2 w = ((float2*)os)[so];
            ((float2*)os)[so] = make_float2(__fmaf_rn(-p.lr, dr, w.x * p.decay), __fmaf_rn(-p.lr, di, w.y * p.decay));
          } else {
            os[so] = __fmaf_rn(-p.lr, dr, os[so] * p.decay);
          }
        }
      }
    }
    fence_async_smem();
    __syncthreads();
    if (tid == 0) {
      uint8_t* dst = WUPD ? (uint8_t*)p.W : (uint8_t*)p.Y;
      bulk_s2g(dst + a0 * p.J * ESZ, os, (uint32_t)(G32T * p.J * ESZ));
      bulk_commit();
      bulk_wait_read0();  // the source read; the writes complete with the kernel
    }
  } else if (!s_abort) {
    const int64_t j0 = (int64_t)blockIdx.y * (CPLX ? p.NT / 2 : p.NT);
    for (int c0 = 0; c0 < p.NT; c0 += 16) {
      float y[16];
      tmem_ld16(dt + lane_base + c0, y);
      constexpr int PER = CPLX ? 8 : 16;  // outputs per 16 columns
#pragma unroll
      for (int u = 0; u < PER; ++u) {
        const int64_t j = j0 + (CPLX ? c0 / 2 : c0) + u;
        if (!valid || j >= p.J) continue;
        const int64_t o = (a * p.J + j) * p.B + b;
        float dr = CPLX ? y[2 * u] : y[u], di = CPLX ? y[2 * u + 1] : 0.f;
        if (!WUPD) {
          if (CPLX)
            ((float2*)p.Y)[o] = make_float2(dr, di);
          else
            p.Y[o] = dr;
        } else {
          const uint32_t word = __ldg(p.wbits + (o >> 5));
          const uint32_t bit = (uint32_t)(o & 31);
          if ((word >> bit) & 1u) {
            const int64_t e = __ldg(p.wrank + (o >> 5)) + __popc(word & ((1u << bit) - 1u));
            if (CPLX) {
              const float2 sv = __ldg((const float2*)p.S + e);
              dr += sv.x;
              di += sv.y;
            } else {
              dr += __ldg(p.S + e);
            }
          }
          if (CPLX) {
            float2* wp = (float2*)p.W + o;
            const float2 w = *wp;
            *wp = make_float2(__fmaf_rn(-p.lr, dr, w.x * p.decay), __fmaf_rn(-p.lr, di, w.y * p.decay));
          } else {
            float* wp = p.W + o;
            *wp = __fmaf_rn(-p.lr, dr, *wp * p.decay);
          }
        }
      }
    }
  } else if (tid == 0) {
    // bounded waits for the copies and MMAs still in flight
    for (int s = 0; s < 2; ++s) {
      if (issued[s] > waited[s]) mbar_wait(&bars[s], (issued[s] - 1) & 1u, G32_WAIT_NS / 4);
      if (bloaded[s] > 0) mbar_wait(&bars[2 + s], (bloaded[s] - 1) & 1u, G32_WAIT_NS / 4);
    }
    if (st_in || (st_out && WUPD)) mbar_wait(&bars[4], 0, G32_WAIT_NS / 4);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) tmem_dealloc(dt, p.tmem_cols);
}

// B operand of y = x M for one mode, M from U (I x r, complex fp32 pairs; the
// real part only for real tensors): kind 0 projection M = conj(U) (Kc = I,
// Jc = r), kind 1 expansion M = U^T (Kc = r, Jc = I). Complex M as the real
// embedding E[(kk,0)][(j,0)] = Mr, E[(kk,1)][(j,0)] = -Mi, E[(kk,0)][(j,1)] =
// Mi, E[(kk,1)][(j,1)] = Mr; real M as itself. Zero padded to Np x Kp, stored
// as [n block][k chunk][h, m, l] blocks of NT x 64 (the three bf16 parts of
// each fp32 entry), each K-major no-swizzle with 8-row groups 128 B apart and
// K core matrices NT / 8 * 128 B apart.
__global__ void embed32_kernel(const float2* U, int I, int r, int kind, int cplx, int Np, int Kp, int NT,
                               int kp, uint16_t* img) {
  const int nkb = Kp / kp;
  const int Kc = kind == 0 ? I : r, Jc = kind == 0 ? r : I;
  for (int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; e < (int64_t)Np * Kp;
       e += (int64_t)gridDim.x * blockDim.x) {
    const int n = (int)(e / Kp), k = (int)(e - (int64_t)n * Kp);
    float val = 0.f;
    if (cplx) {
      const int j = n >> 1, cp = n & 1, kk = k >> 1, c = k & 1;
      if (j < Jc && kk < Kc) {
        const float2 u = kind == 0 ? U[(int64_t)kk * r + j] : U[(int64_t)j * r + kk];
        const float mr = u.x, mi = kind == 0 ? -u.y : u.y;
        val = (c == 0) ? (cp == 0 ? mr : mi) : (cp == 0 ? -mi : mr);
      }
    } else if (n < Jc && k < Kc) {
      val = kind == 0 ? U[(int64_t)k * r + n].x : U[(int64_t)n * r + k].x;
    }
    const uint16_t h = bf16_bits(val);
    const float r = val - bf16_val(h);
    const uint16_t m = bf16_bits(r), l = bf16_bits(r - bf16_val(m));
    const int nb = n / NT, nl = n - nb * NT, kb = k / kp, kl = k - kb * kp;
    const int64_t base = ((int64_t)nb * nkb + kb) * 3 * NT * kp;
    const uint32_t off = kmaj((uint32_t)nl, (uint32_t)kl, (uint32_t)(NT / 8) * 128u) / 2;
    img[base + off] = h;
    img[base + (int64_t)NT * kp + off] = m;
    img[base + 2 * (int64_t)NT * kp + off] = l;
  }
}

// wrank[w] = number of Omega entries below 32 w (Omega ascending).
__global__ void word_rank_kernel(const int64_t* omega, int64_t k, int64_t nwords, int64_t* wrank) {
  for (int64_t w = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; w < nwords;
       w += (int64_t)gridDim.x * blockDim.x) {
    const int64_t target = w * 32;
    int64_t lo = 0, hi = k;
    while (lo < hi) {
      const int64_t mid = (lo + hi) >> 1;
      if (omega[mid] < target)
        lo = mid + 1;
      else
        hi = mid;
    }
    wrank[w] = lo;
  }
}

struct Mode32 {
  int n = 0;
  int64_t I = 0, r = 0;
  bool active = false;
  uint16_t* img_p = nullptr;  // projection image
  uint16_t* img_e = nullptr;  // expansion image
  const float* U = nullptr;   // the factor (the caller's buffer, refreshed in place)
  int NTp = 0, nntp = 0, nkcp = 0, NTe = 0, nnte = 0, nkce = 0;
  int kpp = 64, kpe = 64;     // bf16 K values per chunk
};

struct Tc32Impl {
  int d = 0;
  bool cplx = false;
  int64_t N = 0, k = 0, ncore = 0, nwords = 0;
  std::vector<Mode32> modes;
  float* X0 = nullptr;
  float* X1 = nullptr;
  float* C = nullptr;
  float* S = nullptr;     // lambda S~, Omega order
  int64_t* wrank = nullptr;
  int num_sms = 148;
};

int r16i(int x) { return (x + 15) / 16 * 16; }
int pow2_cols32(int n) {
  int c = 32;
  while (c < n) c <<= 1;
  return c;
}
// stages x (three A tiles + three B blocks) + barriers
// The innermost mode (B = 1, one K chunk, one column block): a persistent
// version of mode_gemm32_kernel. Each CTA takes whole 128-row tiles t =
// blockIdx.x, + gridDim.x, ...; a tile's rows of X (and of W when the
// weights are updated) are one contiguous range each and arrive by bulk copy,
// Omega's mask words (and word ranks) by cp.async, into a ring of NB buffers,
// NB - 1 tiles ahead of the one whose rows are split into bf16 parts,
// multiplied and written back (one bulk store per tile). The operand image
// of the mode is loaded once per CTA.
struct Inner32Layout {
  uint32_t bimg, xs, os, xm, om, bars;  // offsets; buffer 1 of each at + its size
  uint32_t xs_size, os_size, xm_size, om_size, total;
};
__host__ __device__ inline uint32_t al128u(uint32_t x) { return (x + 127u) / 128u * 128u; }
constexpr int I32_NB_MAX = 4;
__host__ __device__ inline Inner32Layout inner32_layout(int NT, int kp, int64_t K, int64_t J, int esz, bool masked,
                                                        bool wupd, int nb) {
  Inner32Layout L;
  const uint32_t atile = (uint32_t)(kp / 8) * G32_LBO;
  L.bimg = 3 * atile;
  L.xs = al128u(L.bimg + 3u * (uint32_t)NT * (uint32_t)kp * 2u);
  L.xs_size = al128u((uint32_t)(G32T * K * esz));
  L.os = L.xs + nb * L.xs_size;
  L.os_size = al128u((uint32_t)(G32T * J * esz));
  L.xm = L.os + nb * L.os_size;
  L.xm_size = masked ? al128u(4u * (uint32_t)(G32T * K / 32 + 2)) : 0u;
  L.om = L.xm + nb * L.xm_size;
  const uint32_t nw = (uint32_t)(G32T * J / 32 + 2);
  L.om_size = wupd ? al128u(4u * (nw + 1) + 8u * nw) : 0u;
  L.bars = L.om + nb * L.om_size;
  L.total = L.bars + 8 * (I32_NB_MAX + 2) + 16;
  return L;
}

template <bool CPLX, bool WUPD>
__global__ void __launch_bounds__(G32T) inner32_kernel(const MG32Args p, const int64_t ntiles, const int NB) {
  extern __shared__ __align__(1024) uint8_t smem[];
  constexpr int ESZ = CPLX ? 8 : 4;
  const int kq = p.kp / 8;
  const uint32_t atile = (uint32_t)kq * G32_LBO;
  const uint32_t b_bytes = (uint32_t)p.NT * p.kp * 2;
  const Inner32Layout L = inner32_layout(p.NT, p.kp, p.K, p.J, ESZ, p.bits != nullptr, WUPD, NB);
  uint64_t* full = (uint64_t*)(smem + L.bars);  // [NB] a tile's rows (and mask words) landed
  uint64_t* mbar = full + I32_NB_MAX;          // the tile's MMAs done
  uint64_t* bbar = mbar + 1;                   // the operand image landed
  uint32_t* tslot = (uint32_t*)(bbar + 1);
  __shared__ int s_abort;
  const int tid = threadIdx.x, warp = tid >> 5;
  const uint32_t lane_base = (uint32_t)(warp * 32) << 16;
  const bool masked = p.bits != nullptr;
  if (tid == 0) {
    s_abort = 0;
    for (int i = 0; i < I32_NB_MAX + 2; ++i) mbar_init(&full[i], 1);
    fence_mbar_init();
  }
  if (warp == 0) tmem_alloc(tslot, p.tmem_cols);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t dt = *tslot;
  const int64_t nloc = ntiles > blockIdx.x ? (ntiles - blockIdx.x + gridDim.x - 1) / gridDim.x : 0;
  if (tid == 0) {
    mbar_expect_tx(bbar, 3 * b_bytes);
    bulk_g2s(smem + L.bimg, p.img, 3 * b_bytes, bbar);
  }
  // the rows of local tile it into buffer bf: mask words by every thread,
  // then (after a barrier, so that their pending arrivals are counted first)
  // the bulk copies
  auto issue = [&](int64_t it, int bf) {
    const int64_t a0 = ((int64_t)blockIdx.x + it * gridDim.x) * G32T;
    if (masked) {
      uint32_t* xm = (uint32_t*)(smem + L.xm + bf * L.xm_size);
      const int64_t w0 = (a0 * p.K) >> 5, nw = (((a0 + G32T) * p.K - 1) >> 5) - w0 + 1;
      for (int w = tid; w < nw; w += G32T) cpa4(xm + w, p.bits + w0 + w);
    }
    if (WUPD) {
      uint32_t* om = (uint32_t*)(smem + L.om + bf * L.om_size);
      const int64_t w0 = (a0 * p.J) >> 5, nw = (((a0 + G32T) * p.J - 1) >> 5) - w0 + 1;
      int64_t* orank = (int64_t*)(om + ((nw + 1) & ~1ll));
      for (int w = tid; w < nw; w += G32T) {
        cpa4(om + w, p.wbits + w0 + w);
        cpa8(orank + w, p.wrank + w0 + w);
      }
    }
    asm volatile("cp.async.mbarrier.arrive.shared::cta.b64 [%0];" ::"r"(smem_u32(&full[bf])) : "memory");
    __syncthreads();
    if (tid == 0) {
      const uint32_t xb = (uint32_t)(G32T * p.K * ESZ), wb = WUPD ? (uint32_t)(G32T * p.J * ESZ) : 0u;
      mbar_expect_tx(&full[bf], xb + wb);
      bulk_g2s(smem + L.xs + bf * L.xs_size, (const uint8_t*)p.X + a0 * p.K * ESZ, xb, &full[bf]);
      if (WUPD) bulk_g2s(smem + L.os + bf * L.os_size, (const uint8_t*)p.W + a0 * p.J * ESZ, wb, &full[bf]);
    }
  };
  auto wait_bar = [&](uint64_t* bar, uint32_t parity) -> bool {
    if (!mbar_wait(bar, parity, G32_WAIT_NS)) {
      atomicOr(p.err, DEV_ERR_TIMEOUT);
      s_abort = 1;
    }
    __syncthreads();
    return s_abort == 0;
  };
  int64_t issued = 0;
  for (; issued < NB - 1 && issued < nloc; ++issued) issue(issued, (int)issued);
  bool ok = nloc == 0 || wait_bar(bbar, 0);
  const uint32_t idesc = idesc_f16(1, 128, p.NT);
  const uint32_t lbo_b = (uint32_t)(p.NT / 8) * 128;
  constexpr int KE = CPLX ? G32_KMAX / 2 : G32_KMAX;
  const int ke = CPLX ? p.kp / 2 : p.kp;
  for (int64_t it = 0; ok && it < nloc; ++it) {
    const int bf = (int)(it % NB);
    const int64_t a0 = ((int64_t)blockIdx.x + it * gridDim.x) * G32T;
    if (it + NB - 1 < nloc) {
      // the buffer of tile it + NB - 1 held tile it - 1: its store must have
      // read it out
      if (tid == 0) bulk_wait_read0();
      issue(it + NB - 1, (int)((it + NB - 1) % NB));
      issued = it + NB;
    }
    if (!wait_bar(&full[bf], (uint32_t)((it / NB) & 1))) break;
    // this row's K values (Omega's entries zero) -> the h, m, l A tiles
    {
      const float* xs = (const float*)(smem + L.xs + bf * L.xs_size);
      const uint32_t* xm = (const uint32_t*)(smem + L.xm + bf * L.xm_size);
      const int64_t w0 = (a0 * p.K) >> 5;
      float v[G32_KMAX];
#pragma unroll
      for (int i = 0; i < KE; ++i) {
        if (i >= ke) break;
        float2 x = make_float2(0.f, 0.f);
        if (i < p.K) {
          const int64_t idx = (a0 + tid) * p.K + i;
          const uint32_t word = masked ? xm[(idx >> 5) - w0] : 0u;
          if (!((word >> (idx & 31)) & 1u)) {
            if (CPLX)
              x = ((const float2*)xs)[tid * p.K + i];
            else
              x.x = xs[tid * p.K + i];
          }
        }
        if (CPLX) {
          v[2 * i] = x.x;
          v[2 * i + 1] = x.y;
        } else {
          v[i] = x.x;
        }
      }
#pragma unroll
      for (int q = 0; q < G32_KMAX / 8; ++q) {
        if (q >= kq) break;
        uint32_t h[4], m[4], l[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) split3(v[8 * q + 2 * u], v[8 * q + 2 * u + 1], h[u], m[u], l[u]);
        *(uint4*)(smem + 0 * atile + q * G32_LBO + tid * 16) = make_uint4(h[0], h[1], h[2], h[3]);
        *(uint4*)(smem + 1 * atile + q * G32_LBO + tid * 16) = make_uint4(m[0], m[1], m[2], m[3]);
        *(uint4*)(smem + 2 * atile + q * G32_LBO + tid * 16) = make_uint4(l[0], l[1], l[2], l[3]);
      }
    }
    fence_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (tid == 0) {
      const uint32_t a_base = smem_u32(smem), b_base = smem_u32(smem + L.bimg);
      for (int kk = 0; kk < kq / 2; ++kk) {
        // (A part, B part): hh, hm, mh, hl, lh, mm
#pragma unroll
        for (int pr = 0; pr < 6; ++pr) {
          const uint32_t pa = (0x120100u >> (4 * pr)) & 0xFu, pb = (0x102010u >> (4 * pr)) & 0xFu;
          const uint64_t da = sdesc(a_base + pa * atile + kk * 2 * G32_LBO, G32_LBO, 128);
          const uint64_t db = sdesc(b_base + pb * b_bytes + kk * 2 * lbo_b, lbo_b, 128);
          mma_f16(dt, da, db, idesc, (kk > 0 || pr > 0) ? 1u : 0u);
        }
      }
      mma_commit(mbar);
    }
    if (!wait_bar(mbar, (uint32_t)(it & 1))) break;
    tc_fence_after();
    // the tile's rows of Y, or W updated in place, in buffer bf
    {
      float* os = (float*)(smem + L.os + bf * L.os_size);
      const uint32_t* omw = (const uint32_t*)(smem + L.om + bf * L.om_size);
      const int64_t ow0 = (a0 * p.J) >> 5;
      const int onw = (int)((((a0 + G32T) * p.J - 1) >> 5) - ow0 + 1);
      const int64_t* omr = (const int64_t*)(omw + ((onw + 1) & ~1));
      for (int c0 = 0; c0 < p.NT; c0 += 16) {
        constexpr int PER = CPLX ? 8 : 16;
        // the block's S~ values first (independent loads, in flight together)
        float2 sv[PER];
        if (WUPD) {
#pragma unroll
          for (int u = 0; u < PER; ++u) {
            sv[u] = make_float2(0.f, 0.f);
            const int64_t j = (CPLX ? c0 / 2 : c0) + u;
            if (j >= p.J) continue;
            const int64_t o = (a0 + tid) * p.J + j;
            const uint32_t word = omw[(o >> 5) - ow0];
            const uint32_t bit = (uint32_t)(o & 31);
            if ((word >> bit) & 1u) {
              const int64_t e = omr[(o >> 5) - ow0] + __popc(word & ((1u << bit) - 1u));
              if (CPLX)
                sv[u] = __ldg((const float2*)p.S + e);
              else
                sv[u].x = __ldg(p.S + e);
            }
          }
        }
        float y[16];
        tmem_ld16(dt + lane_base + c0, y);
#pragma unroll
        for (int u = 0; u < PER; ++u) {
          const int64_t j = (CPLX ? c0 / 2 : c0) + u;
          if (j >= p.J) continue;
          const int64_t so = (int64_t)tid * p.J + j;
          float dr = CPLX ? y[2 * u] : y[u], di = CPLX ? y[2 * u + 1] : 0.f;
          if (!WUPD) {
            if (CPLX)
              ((float2*)os)[so] = make_float2(dr, di);
            else
              os[so] = dr;
          } else {
            dr += sv[u].x;
            di += sv[u].y;
            if (CPLX) {
              const float2 w = ((float2*)os)[so];
              ((float2*)os)[so] = make_float2(__fmaf_rn(-p.lr, dr, w.x * p.decay), __fmaf_rn(-p.lr, di, w.y * p.decay));
            } else {
              os[so] = __fmaf_rn(-p.lr, dr, os[so] * p.decay);
            }
          }
        }
      }
      fence_async_smem();
      tc_fence_before();
      __syncthreads();
      if (tid == 0) {
        uint8_t* dst = WUPD ? (uint8_t*)p.W : (uint8_t*)p.Y;
        bulk_s2g(dst + a0 * p.J * ESZ, os, (uint32_t)(G32T * p.J * ESZ));
        bulk_commit();
      }
    }
  }
  if (tid == 0) {
    bulk_wait_read0();  // no store still reads this CTA's shared memory
    if (s_abort) {
      // bounded waits for copies still in flight
      for (int64_t i = issued > NB ? issued - NB : 0; i < issued; ++i)
        mbar_wait(&full[i % NB], (uint32_t)((i / NB) & 1), G32_WAIT_NS / 4);
      mbar_wait(bbar, 0, G32_WAIT_NS / 4);
      mbar_wait(mbar, 0, G32_WAIT_NS / 4);
      mbar_wait(mbar, 1, G32_WAIT_NS / 4);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) tmem_dealloc(dt, p.tmem_cols);
}

// The innermost mode on CUDA cores, for factors small enough that the
// product is bound by the rows' bytes (4 K J fp32 FMAs per complex row: 340
// for K = 17, J = 5, against 136 + 40 bytes): the staging ring of
// inner32_kernel (whole 128-row tiles, rows and Omega's words arriving NB - 1
// tiles ahead, one bulk store per tile), with y = x M computed per thread in
// fp32 FMAs from the masked row in registers and M (K x J, from U) in shared
// memory. M[k][j] = conj(U[k][j]) for a projection (ukind 0, K = I, J = r),
// U[j][k] for an expansion (ukind 1, K = r, J = I).
__host__ __device__ inline Inner32Layout ffma32_layout(int64_t K, int64_t J, int esz, bool masked, bool wupd,
                                                       int nb) {
  Inner32Layout L;
  L.bimg = 0;  // M
  L.xs = al128u((uint32_t)(K * ((J + 7) / 8 * 8) * esz));  // M, rows padded to 8 outputs
  L.xs_size = al128u((uint32_t)(G32T * K * esz));
  L.os = L.xs + nb * L.xs_size;
  L.os_size = al128u((uint32_t)(G32T * J * esz));
  L.xm = L.os + nb * L.os_size;
  L.xm_size = masked ? al128u(4u * (uint32_t)(G32T * K / 32 + 2)) : 0u;
  L.om = L.xm + nb * L.xm_size;
  const uint32_t nw = (uint32_t)(G32T * J / 32 + 2);
  L.om_size = wupd ? al128u(4u * (nw + 1) + 8u * nw) : 0u;
  L.bars = L.om + nb * L.om_size;
  L.total = L.bars + 8 * (I32_NB_MAX + 2) + 16;
  return L;
}
constexpr int F32_KMAX = 32;  // K entries of a row held in registers
constexpr int F32_JMAX = 32;  // outputs of a row

template <bool CPLX, bool WUPD>
__global__ void __launch_bounds__(G32T) inner32_ffma_kernel(const MG32Args p, const int64_t ntiles, const int NB) {
  extern __shared__ __align__(1024) uint8_t smem[];
  constexpr int ESZ = CPLX ? 8 : 4;
  const Inner32Layout L = ffma32_layout(p.K, p.J, ESZ, p.bits != nullptr, WUPD, NB);
  uint64_t* full = (uint64_t*)(smem + L.bars);  // [NB] a tile's rows (and mask words) landed
  __shared__ int s_abort;
  const int tid = threadIdx.x;
  const bool masked = p.bits != nullptr;
  const int K = (int)p.K, J = (int)p.J;
  if (tid == 0) {
    s_abort = 0;
    for (int i = 0; i < I32_NB_MAX; ++i) mbar_init(&full[i], 1);
    fence_mbar_init();
  }
  // M from U (I x ur, complex pairs or reals), rows of Jp (J rounded up to
  // 8) outputs, zero padded: eight outputs of a row are 16-byte aligned
  const int Jp = (J + 7) / 8 * 8;
  for (int e = tid; e < K * Jp; e += G32T) {
    const int k = e / Jp, j = e - k * Jp;
    const int64_t ui = p.ukind == 0 ? (int64_t)k * p.ur + j : (int64_t)j * p.ur + k;
    if (CPLX) {
      const float2 u = j < J ? ((const float2*)p.Uf)[ui] : make_float2(0.f, 0.f);
      ((float2*)(smem + L.bimg))[e] = make_float2(u.x, p.ukind == 0 ? -u.y : u.y);
    } else {
      ((float*)(smem + L.bimg))[e] = j < J ? p.Uf[2 * ui] : 0.f;
    }
  }
  __syncthreads();
  const int64_t nloc = ntiles > blockIdx.x ? (ntiles - blockIdx.x + gridDim.x - 1) / gridDim.x : 0;
  auto issue = [&](int64_t it, int bf) {
    const int64_t a0 = ((int64_t)blockIdx.x + it * gridDim.x) * G32T;
    if (masked) {
      uint32_t* xm = (uint32_t*)(smem + L.xm + bf * L.xm_size);
      const int64_t w0 = (a0 * p.K) >> 5, nw = (((a0 + G32T) * p.K - 1) >> 5) - w0 + 1;
      for (int w = tid; w < nw; w += G32T) cpa4(xm + w, p.bits + w0 + w);
    }
    if (WUPD) {
      uint32_t* om = (uint32_t*)(smem + L.om + bf * L.om_size);
      const int64_t w0 = (a0 * p.J) >> 5, nw = (((a0 + G32T) * p.J - 1) >> 5) - w0 + 1;
      int64_t* orank = (int64_t*)(om + ((nw + 1) & ~1ll));
      for (int w = tid; w < nw; w += G32T) {
        cpa4(om + w, p.wbits + w0 + w);
        cpa8(orank + w, p.wrank + w0 + w);
      }
    }
    asm volatile("cp.async.mbarrier.arrive.shared::cta.b64 [%0];" ::"r"(smem_u32(&full[bf])) : "memory");
    __syncthreads();
    if (tid == 0) {
      const uint32_t xb = (uint32_t)(G32T * p.K * ESZ), wb = WUPD ? (uint32_t)(G32T * p.J * ESZ) : 0u;
      mbar_expect_tx(&full[bf], xb + wb);
      bulk_g2s(smem + L.xs + bf * L.xs_size, (const uint8_t*)p.X + a0 * p.K * ESZ, xb, &full[bf]);
      if (WUPD) bulk_g2s(smem + L.os + bf * L.os_size, (const uint8_t*)p.W + a0 * p.J * ESZ, wb, &full[bf]);
    }
  };
  auto wait_bar = [&](uint64_t* bar, uint32_t parity) -> bool {
    if (!mbar_wait(bar, parity, G32_WAIT_NS)) {
      atomicOr(p.err, DEV_ERR_TIMEOUT);
      s_abort = 1;
    }
    __syncthreads();
    return s_abort == 0;
  };
  int64_t issued = 0;
  for (; issued < NB - 1 && issued < nloc; ++issued) issue(issued, (int)issued);
  const float2* M2 = (const float2*)(smem + L.bimg);
  const float* M1 = (const float*)(smem + L.bimg);
  for (int64_t it = 0; it < nloc; ++it) {
    const int bf = (int)(it % NB);
    const int64_t a0 = ((int64_t)blockIdx.x + it * gridDim.x) * G32T;
    if (it + NB - 1 < nloc) {
      // the buffer of tile it + NB - 1 held tile it - 1: its store must have
      // read it out
      if (tid == 0) bulk_wait_read0();
      issue(it + NB - 1, (int)((it + NB - 1) % NB));
      issued = it + NB;
    }
    if (!wait_bar(&full[bf], (uint32_t)((it / NB) & 1))) break;
    // this row's K values, Omega's entries zero
    float2 v[F32_KMAX];
    {
      const float* xs = (const float*)(smem + L.xs + bf * L.xs_size);
      const uint32_t* xm = (const uint32_t*)(smem + L.xm + bf * L.xm_size);
      const int64_t w0 = (a0 * p.K) >> 5;
#pragma unroll
      for (int i = 0; i < F32_KMAX; ++i) {
        if (i >= K) break;
        float2 x = make_float2(0.f, 0.f);
        const int64_t idx = (a0 + tid) * p.K + i;
        const uint32_t word = masked ? xm[(idx >> 5) - w0] : 0u;
        if (!((word >> (idx & 31)) & 1u)) {
          if (CPLX)
            x = ((const float2*)xs)[tid * K + i];
          else
            x.x = xs[tid * K + i];
        }
        v[i] = x;
      }
    }
    // the row's outputs, then its rows of Y or W updated in place, in buffer bf
    {
      float* os = (float*)(smem + L.os + bf * L.os_size);
      const uint32_t* omw = (const uint32_t*)(smem + L.om + bf * L.om_size);
      const int64_t ow0 = (a0 * p.J) >> 5;
      const int onw = (int)((((a0 + G32T) * p.J - 1) >> 5) - ow0 + 1);
      const int64_t* omr = (const int64_t*)(omw + ((onw + 1) & ~1));
      // eight outputs at a time; for the update their S~ values are loaded
      // first (independent loads, in flight together)
#pragma unroll 1
      for (int j0 = 0; j0 < J; j0 += 8) {
        float2 sv[8];
        if (WUPD) {
#pragma unroll
          for (int u = 0; u < 8; ++u) {
            sv[u] = make_float2(0.f, 0.f);
            const int j = j0 + u;
            if (j >= J) continue;
            const int64_t o = (a0 + tid) * p.J + j;
            const uint32_t word = omw[(o >> 5) - ow0];
            const uint32_t bit = (uint32_t)(o & 31);
            if ((word >> bit) & 1u) {
              const int64_t e = omr[(o >> 5) - ow0] + __popc(word & ((1u << bit) - 1u));
              if (CPLX)
                sv[u] = __ldg((const float2*)p.S + e);
              else
                sv[u].x = __ldg(p.S + e);
            }
          }
        }
        // the block's eight outputs together: per K entry, one row of M
        // (four 16-byte loads) and eight independent accumulations
        float ar[8], ai[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) ar[u] = ai[u] = 0.f;
#pragma unroll
        for (int i = 0; i < F32_KMAX; ++i) {
          if (i >= K) break;
          if (CPLX) {
            const float4* mr = (const float4*)(M2 + i * Jp + j0);
#pragma unroll
            for (int h = 0; h < 4; ++h) {
              const float4 m = mr[h];
              ar[2 * h] = __fmaf_rn(v[i].x, m.x, __fmaf_rn(-v[i].y, m.y, ar[2 * h]));
              ai[2 * h] = __fmaf_rn(v[i].x, m.y, __fmaf_rn(v[i].y, m.x, ai[2 * h]));
              ar[2 * h + 1] = __fmaf_rn(v[i].x, m.z, __fmaf_rn(-v[i].y, m.w, ar[2 * h + 1]));
              ai[2 * h + 1] = __fmaf_rn(v[i].x, m.w, __fmaf_rn(v[i].y, m.z, ai[2 * h + 1]));
            }
          } else {
            const float4* mr = (const float4*)(M1 + i * Jp + j0);
#pragma unroll
            for (int h = 0; h < 2; ++h) {
              const float4 m = mr[h];
              ar[4 * h] = __fmaf_rn(v[i].x, m.x, ar[4 * h]);
              ar[4 * h + 1] = __fmaf_rn(v[i].x, m.y, ar[4 * h + 1]);
              ar[4 * h + 2] = __fmaf_rn(v[i].x, m.z, ar[4 * h + 2]);
              ar[4 * h + 3] = __fmaf_rn(v[i].x, m.w, ar[4 * h + 3]);
            }
          }
        }
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          const int j = j0 + u;
          if (j >= J) break;
          float dr = ar[u], di = ai[u];
          const int64_t so = (int64_t)tid * p.J + j;
          if (!WUPD) {
            if (CPLX)
              ((float2*)os)[so] = make_float2(dr, di);
            else
              os[so] = dr;
          } else {
            dr += sv[u].x;
            di += sv[u].y;
            if (CPLX) {
              const float2 w = ((float2*)os)[so];
              ((float2*)os)[so] = make_float2(__fmaf_rn(-p.lr, dr, w.x * p.decay), __fmaf_rn(-p.lr, di, w.y * p.decay));
            } else {
              os[so] = __fmaf_rn(-p.lr, dr, os[so] * p.decay);
            }
          }
        }
      }
      fence_async_smem();
      __syncthreads();
      if (tid == 0) {
        uint8_t* dst = WUPD ? (uint8_t*)p.W : (uint8_t*)p.Y;
        bulk_s2g(dst + a0 * p.J * ESZ, os, (uint32_t)(G32T * p.J * ESZ));
        bulk_commit();
      }
    }
  }
  if (tid == 0) {
    bulk_wait_read0();  // no store still reads this CTA's shared memory
    if (s_abort) {
      // bounded waits for copies still in flight
      for (int64_t i = issued > NB ? issued - NB : 0; i < issued; ++i)
        mbar_wait(&full[i % NB], (uint32_t)((i / NB) & 1), G32_WAIT_NS / 4);
    }
  }
  __syncthreads();
}

size_t g32_smem(int NT, int nstage, int kp) {
  return (size_t)nstage * (3 * (size_t)(kp / 8) * G32_LBO + 3 * (size_t)NT * kp * 2) + 64;
}
constexpr size_t G32_SMEM_LIMIT = 227 * 1024 - 1024;
size_t al128(size_t x) { return (x + 127) / 128 * 128; }

Tc32Impl* impl32(Tc32Plan& p) { return (Tc32Impl*)p.impl; }

// Geometry of one mode's GEMM: N = 2 Jc (complex) or Jc columns in blocks of
// at most 128 (two stages of three A tiles and three B blocks fit shared
// memory); K in chunks of 64 real values (32 complex), or one chunk of K
// rounded up to 16 when it fits.
void mode_geom(int64_t Kc, int64_t Jc, bool cplx, int& NT, int& nnt, int& nkc, int& kp) {
  const int Np = r16i((int)(cplx ? 2 * Jc : Jc));
  NT = Np <= 128 ? Np : 128;
  nnt = (int)ceil_div(Np, NT);
  const int64_t kreal = cplx ? 2 * Kc : Kc;
  nkc = (int)ceil_div(kreal, G32_KMAX);
  kp = nkc == 1 ? r16i((int)kreal) : G32_KMAX;
}

// Staging of the contiguous row ranges of an innermost-mode product (B == 1):
// the input when its K fits one chunk, the output when it is one N block;
// both only where the addresses allow bulk copies and shared memory suffices.
template <bool CPLX, bool WUPD>
cudaError_t launch32(MG32Args a, int nnt, cudaStream_t s) {
  const size_t esz = CPLX ? 8 : 4;
  a.tile0 = 0;
  // the innermost mode with one K chunk and one column block: the persistent
  // kernel over the whole 128-row tiles, this kernel for a ragged last tile
  const void* outp = WUPD ? (const void*)a.W : (const void*)a.Y;
  int dev = 0, nsm = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev);
  // a small factor (K, J <= 32, K J <= 512): CUDA cores over whole tiles
  // (at most 4 K J fp32 FMAs per complex row, bound by the rows' bytes), this
  // kernel for a ragged last tile
  bool tiles_done = false;
  if (a.B == 1 && a.Uf && a.K <= F32_KMAX && a.J <= F32_JMAX && a.K * a.J <= 512 && a.rows >= G32T &&
      ((uintptr_t)a.X % 16) == 0 && ((uintptr_t)outp % 16) == 0) {
    int nb = 0, cps = 0;
    Inner32Layout L{};
    for (int b = 2; b <= I32_NB_MAX; ++b) {
      const Inner32Layout Lb = ffma32_layout(a.K, a.J, (int)esz, a.bits != nullptr, WUPD, b);
      if (Lb.total > G32_SMEM_LIMIT) break;
      const int c = std::min(8, (int)(232448 / (Lb.total + 1024)));
      if (c >= cps) {
        nb = b;
        cps = c;
        L = Lb;
      }
    }
    if (nb > 0) {
      const int64_t ntiles = a.rows / G32T;
      const int64_t grid = std::min<int64_t>(ntiles, (int64_t)nsm * cps);
      cudaError_t e = cudaFuncSetAttribute(inner32_ffma_kernel<CPLX, WUPD>,
                                           cudaFuncAttributeMaxDynamicSharedMemorySize, (int)L.total);
      if (e != cudaSuccess) return e;
      inner32_ffma_kernel<CPLX, WUPD><<<(unsigned)grid, G32T, L.total, s>>>(a, ntiles, nb);
      e = cudaGetLastError();
      if (e != cudaSuccess || a.rows % G32T == 0) return e;
      a.tile0 = ntiles;
      tiles_done = true;
    }
  }
  if (!tiles_done && a.B == 1 && a.nkc == 1 && nnt == 1 && a.rows >= G32T && ((uintptr_t)a.X % 16) == 0 &&
      ((uintptr_t)outp % 16) == 0) {
    // the most CTAs per SM (a tile's latency chain bounds each CTA), then the
    // deepest ring those leave room for
    int nb = 0, cps = 0;
    Inner32Layout L{};
    for (int b = 2; b <= I32_NB_MAX; ++b) {
      const Inner32Layout Lb = inner32_layout(a.NT, a.kp, a.K, a.J, (int)esz, a.bits != nullptr, WUPD, b);
      if (Lb.total > G32_SMEM_LIMIT) break;
      const int c = std::min(4, (int)(232448 / (Lb.total + 1024)));
      if (c >= cps) {
        nb = b;
        cps = c;
        L = Lb;
      }
    }
    if (nb > 0) {
      const int64_t ntiles = a.rows / G32T;
      const int64_t grid = std::min<int64_t>(ntiles, (int64_t)nsm * cps);
      cudaError_t e = cudaFuncSetAttribute(inner32_kernel<CPLX, WUPD>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                           (int)L.total);
      if (e != cudaSuccess) return e;
      inner32_kernel<CPLX, WUPD><<<(unsigned)grid, G32T, L.total, s>>>(a, ntiles, nb);
      e = cudaGetLastError();
      if (e != cudaSuccess || a.rows % G32T == 0) return e;
      a.tile0 = ntiles;
    }
  }
  size_t sm = g32_smem(a.NT, a.nstage, a.kp);
  a.xs_off = 0;
  a.os_off = 0;
  a.xm_off = 0;
  a.om_off = 0;
  if (a.B == 1) {
    size_t off = al128(sm);
    if (a.nkc == 1 && ((uintptr_t)a.X % 16) == 0) {
      const size_t need = off + al128((size_t)G32T * a.K * esz);
      if (need <= G32_SMEM_LIMIT) {
        a.xs_off = (uint32_t)off;
        off = need;
      }
    }
    const void* out = WUPD ? (const void*)a.W : (const void*)a.Y;
    if (nnt == 1 && ((uintptr_t)out % 16) == 0) {
      const size_t need = off + al128((size_t)G32T * a.J * esz);
      if (need <= G32_SMEM_LIMIT) {
        a.os_off = (uint32_t)off;
        off = need;
      }
    }
    // mask words of a staged range: at most 128 K / 32 + 2 (X), and for the
    // update that many words and as many 8-byte ranks (output)
    if (a.xs_off && a.bits) {
      const size_t need = off + al128(4 * ((size_t)G32T * a.K / 32 + 2));
      if (need <= G32_SMEM_LIMIT) {
        a.xm_off = (uint32_t)off;
        off = need;
      }
    }
    if (a.os_off && WUPD) {
      const size_t nw = (size_t)G32T * a.J / 32 + 2;
      const size_t need = off + al128(4 * (nw + 1) + 8 * nw);
      if (need <= G32_SMEM_LIMIT) {
        a.om_off = (uint32_t)off;
        off = need;
      }
    }
    sm = off;
  }
  cudaError_t e = cudaFuncSetAttribute(mode_gemm32_kernel<CPLX, WUPD>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm);
  if (e != cudaSuccess) return e;
  dim3 grid((unsigned)(ceil_div(a.rows, G32T) - a.tile0), (unsigned)nnt);
  mode_gemm32_kernel<CPLX, WUPD><<<grid, G32T, sm, s>>>(a);
  return cudaGetLastError();
}

cudaError_t launch_mode32(bool cplx, bool wupd, const MG32Args& a, int nnt, cudaStream_t s) {
  // (a is copied: the launcher fills in the staging offsets)
  if (cplx) return wupd ? launch32<true, true>(a, nnt, s) : launch32<true, false>(a, nnt, s);
  return wupd ? launch32<false, true>(a, nnt, s) : launch32<false, false>(a, nnt, s);
}

}  // namespace

bool tc32_supported(int nd, const int64_t* shape, const int64_t* ranks, uint32_t proj_mask, int gdt, int wdt) {
  if (!((gdt == TGD_C64 && wdt == TGD_C64) || (gdt == TGD_R32 && wdt == TGD_R32))) return false;
  bool any = false;
  for (int n = 0; n < nd; ++n) {
    if ((proj_mask >> n) & 1u) {
      any = true;
      if (shape[n] > 256 || ranks[n] > 256) return false;
    }
  }
  return any;
}

bool tc32_plan(Tc32Plan& p, int nd, const int64_t* shape, const int64_t* ranks, uint32_t proj_mask, int64_t k,
               int gdt, AllocFn alloc, void* ctx) {
  Tc32Impl* g = new Tc32Impl;
  p.impl = g;
  g->d = nd;
  g->cplx = gdt == TGD_C64;
  g->N = 1;
  g->ncore = 1;
  for (int n = 0; n < nd; ++n) {
    g->N *= shape[n];
    g->ncore *= ranks[n];
  }
  g->k = k;
  g->nwords = ceil_div(g->N, 32);
  int dev = 0;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&g->num_sms, cudaDevAttrMultiProcessorCount, dev);
  const int comps = g->cplx ? 2 : 1;
  auto A = [&](void** ptr, size_t bytes) { return alloc(ctx, ptr, bytes); };
  bool ok = true;
  // intermediates: the largest tensor of either chain short of the full one
  // (the expansion chain passes through the same sizes in reverse)
  int64_t maxe = 1, cur = g->N;
  int first = -1;
  for (int n = nd - 1; n >= 0; --n) {
    if (!((proj_mask >> n) & 1u)) continue;
    if (first < 0) first = n;
    cur = cur / shape[n] * ranks[n];
    maxe = std::max(maxe, cur);
  }
  g->modes.clear();
  for (int n = 0; n < nd; ++n) {
    Mode32 m;
    m.n = n;
    m.I = shape[n];
    m.r = ranks[n];
    m.active = ((proj_mask >> n) & 1u) != 0;
    if (m.active) {
      mode_geom(m.I, m.r, g->cplx, m.NTp, m.nntp, m.nkcp, m.kpp);
      mode_geom(m.r, m.I, g->cplx, m.NTe, m.nnte, m.nkce, m.kpe);
      ok &= A((void**)&m.img_p, (size_t)m.nntp * m.nkcp * 3 * m.NTp * m.kpp * 2);
      ok &= A((void**)&m.img_e, (size_t)m.nnte * m.nkce * 3 * m.NTe * m.kpe * 2);
    }
    g->modes.push_back(m);
  }
  ok &= A((void**)&g->X0, sizeof(float) * comps * maxe);
  ok &= A((void**)&g->X1, sizeof(float) * comps * maxe);
  ok &= A((void**)&g->C, sizeof(float) * comps * g->ncore);
  ok &= A((void**)&g->S, sizeof(float) * comps * std::max<int64_t>(k, 1));
  ok &= A((void**)&g->wrank, sizeof(int64_t) * (g->nwords + 1));
  p.ready = ok;
  return ok;
}

void tc32_release(Tc32Plan& p) {
  delete impl32(p);
  p.impl = nullptr;
  p.ready = false;
}

float* tc32_core(Tc32Plan& p) { return impl32(p) ? impl32(p)->C : nullptr; }
float* tc32_sparse_update(Tc32Plan& p) { return impl32(p) ? impl32(p)->S : nullptr; }

cudaError_t tc32_rebuild(Tc32Plan& p, const int64_t* omega, int64_t k, const float* const* U,
                         cudaStream_t s) {
  Tc32Impl* g = impl32(p);
  if (!g) return cudaErrorNotReady;
  auto blocks = [](int64_t n) { return (unsigned)std::min<int64_t>(ceil_div(n, 256), 4096); };
  word_rank_kernel<<<blocks(g->nwords), 256, 0, s>>>(omega, k, g->nwords, g->wrank);
  for (auto& m : g->modes) {
    if (!m.active) continue;
    m.U = U[m.n];
    const float2* Un = (const float2*)U[m.n];
    int Np = m.nntp * m.NTp, Kp = m.nkcp * m.kpp;
    embed32_kernel<<<blocks((int64_t)Np * Kp), 256, 0, s>>>(Un, (int)m.I, (int)m.r, 0, g->cplx ? 1 : 0, Np, Kp,
                                                            m.NTp, m.kpp, m.img_p);
    Np = m.nnte * m.NTe;
    Kp = m.nkce * m.kpe;
    embed32_kernel<<<blocks((int64_t)Np * Kp), 256, 0, s>>>(Un, (int)m.I, (int)m.r, 1, g->cplx ? 1 : 0, Np, Kp,
                                                            m.NTe, m.kpe, m.img_e);
  }
  return cudaGetLastError();
}

cudaError_t tc32_project(Tc32Plan& p, const void* grad, const uint32_t* bits, int* d_err, cudaStream_t s,
                         TimerHook hook, void* hook_ctx) {
  Tc32Impl* g = impl32(p);
  if (!g) return cudaErrorNotReady;
  const int d = g->d;
  int64_t dims[TGD_MAX_NDIM];
  for (int n = 0; n < d; ++n) dims[n] = g->modes[n].I;
  int first_active = -1;
  for (int n = 0; n < d; ++n)
    if (g->modes[n].active) {
      first_active = n;
      break;
    }
  const float* cur = (const float*)grad;
  bool from_grad = true;
  float* bufs[2] = {g->X0, g->X1};
  int which = 0;
  for (int n = d - 1; n >= 0; --n) {
    Mode32& m = g->modes[n];
    if (!m.active) continue;
    int64_t A = 1, B = 1;
    for (int q = 0; q < n; ++q) A *= dims[q];
    for (int q = n + 1; q < d; ++q) B *= dims[q];
    float* out = n == first_active ? g->C : bufs[which];
    MG32Args a{};
    a.X = cur;
    a.bits = from_grad ? bits : nullptr;
    a.rows = A * B;
    a.K = m.I;
    a.B = B;
    a.Y = out;
    a.J = m.r;
    a.img = (const uint8_t*)m.img_p;
    a.NT = m.NTp;
    a.nkc = m.nkcp;
    a.kp = m.kpp;
    a.nstage = m.nkcp > 1 ? 2 : 1;
    a.tmem_cols = (uint32_t)pow2_cols32(m.NTp);
    a.Uf = m.U;
    a.ur = (int)m.r;
    a.ukind = 0;
    a.err = d_err;
    if (hook) hook(hook_ctx, 0, "mode_gemm32", s);
    cudaError_t e = launch_mode32(g->cplx, false, a, m.nntp, s);
    if (hook) hook(hook_ctx, 1, "mode_gemm32", s);
    if (e != cudaSuccess) return e;
    dims[n] = m.r;
    cur = out;
    from_grad = false;
    which ^= 1;
  }
  return cudaSuccess;
}

cudaError_t tc32_expand_update(Tc32Plan& p, void* w, const uint32_t* bits, float decay, float lr, int* d_err,
                               cudaStream_t s, TimerHook hook, void* hook_ctx) {
  Tc32Impl* g = impl32(p);
  if (!g) return cudaErrorNotReady;
  const int d = g->d;
  int64_t dims[TGD_MAX_NDIM];
  for (int n = 0; n < d; ++n) dims[n] = g->modes[n].r;
  int last_active = -1;
  for (int n = 0; n < d; ++n)
    if (g->modes[n].active) last_active = n;
  const float* cur = g->C;
  float* bufs[2] = {g->X0, g->X1};
  int which = 0;
  for (int n = 0; n < d; ++n) {
    Mode32& m = g->modes[n];
    if (!m.active) continue;
    int64_t A = 1, B = 1;
    for (int q = 0; q < n; ++q) A *= dims[q];
    for (int q = n + 1; q < d; ++q) B *= dims[q];
    const bool last = n == last_active;
    MG32Args a{};
    a.X = cur;
    a.bits = nullptr;
    a.rows = A * B;
    a.K = m.r;
    a.B = B;
    a.Y = last ? nullptr : bufs[which];
    a.J = m.I;
    a.img = (const uint8_t*)m.img_e;
    a.NT = m.NTe;
    a.nkc = m.nkce;
    a.kp = m.kpe;
    a.nstage = m.nkce > 1 ? 2 : 1;
    a.tmem_cols = (uint32_t)pow2_cols32(m.NTe);
    a.Uf = m.U;
    a.ur = (int)m.r;
    a.ukind = 1;
    a.W = (float*)w;
    a.S = g->S;
    a.wrank = g->wrank;
    a.wbits = bits;
    a.decay = decay;
    a.lr = lr;
    a.err = d_err;
    if (hook) hook(hook_ctx, 0, last ? "expand_update32" : "mode_gemm32", s);
    cudaError_t e = launch_mode32(g->cplx, last, a, m.nnte, s);
    if (hook) hook(hook_ctx, 1, last ? "expand_update32" : "mode_gemm32", s);
    if (e != cudaSuccess) return e;
    dims[n] = m.I;
    if (!last) {
      cur = bufs[which];
      which ^= 1;
    }
  }
  return cudaSuccess;
}

}  // namespace tgd
