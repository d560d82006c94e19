// Tensor-core (tcgen05, sm_100a) path of the TensorGRaD step for complex fp16
// gradients, fused so that the gradient and the weights each cross HBM once.
//
// The step is the one of the nullthought.net TensorGRaD summary (section 三:
// sparse part first, Tucker part on the residual, separate Adam updates, the
// sparse update scatter-added in place into the rebuilt tensor, FP32
// optimizer states with FP16 weights and gradients) and of Theorem 2 in the
// paper text appended to the Pith review (project with the transposed
// factors, Adam on the core, project back). With a = d-2 and b = d-1 the
// last two modes, a "slab" is one (I_a x I_b) plane and a "tile" is the 128
// rows (i_a) of 128 / I_a consecutive slabs:
//
//  proj_stream  (one pass over G) per tile: bulk-copy the raw tile to shared
//     memory; on Omega's entries gather g_s, zero the entry (residual) and
//     run the sparse AdamW update (S~ kept as fp16 for the reconstruction);
//     GEMM1  P = X conj(U_b)        M = 128 rows (i_a), K = 2 I_b, N = 2 r_b
//     GEMM2  Y = (U_a^H P)^T        M = 128 rows (slab, j_b), K = 2 I_a, N = 2 r_a
//     over groups of slabs; Y (bf16) is 1/16 of G for the default shapes.
//  mode_gemm    the remaining modes n < a, contracted on Y in place of each
//     other: rows = 128 consecutive inner positions, K = 2 I_n (or 2 r_n),
//     N = 2 r_n (or 2 I_n); the last projection writes the core C in fp32.
//  core_adam    C~ = Adam(C) with FP32 moments, written as bf16.
//  recon_stream (one pass over W) per tile: bulk-copy W and Y';
//     GEMM1  P' = U_a Y'^T          M = 128 rows (slab, i_a), K = 2 r_a per slab
//                                    (block-diagonal over the tile's slabs), N = 2 r_b
//     GEMM2  Delta = P' U_b^T       M = 128 rows, K = 2 r_b, N = 2 I_b
//     epilogue: Delta += lambda S~ on Omega (in place), W <- W (1 - lr wd)
//     - lr Delta rounded once, bulk-copy W back.
//
// Complex products run as real GEMMs on an embedding: for y = x M with x a
// complex row (interleaved re, im along K), the K x N real matrix
// [[Mr, Mi], [-Mi, Mr]] (per complex entry) gives y interleaved along N. All
// operands are K-major in the no-swizzle canonical layout (8-row x 16-byte
// core matrices); accumulators live in TMEM (fp32) and are read back with
// tcgen05.ld. Every wait is bounded and reports TGD_ERR_TIMEOUT.

#include <algorithm>
#include <vector>

#include "common.cuh"
#include "kernels.h"
#include "step_tc.h"
#include "tc_ptx.cuh"

namespace tgd {
namespace {

using namespace ptx;

__device__ __forceinline__ float2 h2_to_f2(uint32_t u) {
  __half2 h = *reinterpret_cast<__half2*>(&u);
  return __half22float2(h);
}
__device__ __forceinline__ uint32_t f2_to_h2(float2 v) {
  __half2 h = __floats2half2_rn(v.x, v.y);
  return *reinterpret_cast<uint32_t*>(&h);
}
__device__ __forceinline__ float2 bf2_to_f2(uint32_t u) {
  __nv_bfloat162 h = *reinterpret_cast<__nv_bfloat162*>(&u);
  return __bfloat1622float2(h);
}
__device__ __forceinline__ uint32_t f2_to_bf2(float x, float y) {
  __nv_bfloat162 h = __floats2bfloat162_rn(x, y);
  return *reinterpret_cast<uint32_t*>(&h);
}

// Byte offset of element (row, k) of a 16-bit K-major no-swizzle operand with
// 8-row groups 128 bytes apart and K core matrices `lbo` bytes apart.
__host__ __device__ __forceinline__ uint32_t kmaj_off(uint32_t row, uint32_t k, uint32_t lbo) {
  return (row & 7u) * 16u + (row >> 3) * 128u + (k >> 3) * lbo + (k & 7u) * 2u;
}

constexpr uint32_t LBO_M128 = 2048;         // 128 rows: 16 groups x 128 B
constexpr uint32_t LBO_M128_PAD = 2048 + 16; // the same plus 16 B: spreads banks
constexpr uint64_t WAIT_NS = 2000000000ull;  // 2 s per wait

// ----------------------------------------------------------- projection
constexpr int P1T = 128;
constexpr int PF = 4;

struct P1Args {
  const uint32_t* G;
  int64_t N, n_slabs, n_tiles, n_groups, tile_elems;
  int Ia, Ib, ra, rb, spb, q, sg;
  int K1, N1, K2, N2;
  const int64_t* tile_off;
  const uint16_t* loc;
  float* sp_m;
  float* sp_v;
  uint32_t* sp_upd;
  AdamConst asp;
  const uint8_t* B1img;
  const uint8_t* B2img;
  void* Y;
  int y_f32;
  int* err;
  uint32_t off_stage0, off_stage1, off_A1, off_A2, off_B1, off_B2, off_bar;
};

__global__ void __launch_bounds__(P1T, 1) proj_stream_kernel(const P1Args p) {
  extern __shared__ __align__(1024) uint8_t smem[];
  uint8_t* stage[2] = {smem + p.off_stage0, smem + p.off_stage1};
  uint8_t* A1 = smem + p.off_A1;
  uint8_t* A2 = smem + p.off_A2;
  uint8_t* B1 = smem + p.off_B1;
  uint8_t* B2 = smem + p.off_B2;
  uint64_t* bars = (uint64_t*)(smem + p.off_bar);  // 0 factors, 1-2 stages, 3 gemm1, 4 gemm2
  uint32_t* tslot = (uint32_t*)(bars + 8);
  __shared__ int s_abort;
  const int tid = threadIdx.x, warp = tid >> 5;
  const uint32_t lane_base = (uint32_t)(warp * 32) << 16;

  const int64_t my_groups =
      p.n_groups > (int64_t)blockIdx.x ? (p.n_groups - 1 - blockIdx.x) / gridDim.x + 1 : 0;
  int64_t n_it = my_groups * p.q;
  if (my_groups > 0) {
    int64_t last_g = blockIdx.x + (my_groups - 1) * gridDim.x;
    int64_t last_tiles = p.n_tiles - last_g * p.q;
    if (last_tiles < p.q) n_it -= p.q - last_tiles;
  }
  auto tile_at = [&](int64_t it) -> int64_t {
    return (blockIdx.x + (it / p.q) * gridDim.x) * p.q + it % p.q;
  };
  auto group_at = [&](int64_t it) -> int64_t { return blockIdx.x + (it / p.q) * gridDim.x; };
  auto is_last = [&](int64_t it) -> bool { return (it % p.q == p.q - 1) || (it == n_it - 1); };
  auto tile_bytes = [&](int64_t t) -> uint32_t {
    int64_t rem = p.N - t * p.tile_elems;
    return (uint32_t)((rem < p.tile_elems ? rem : p.tile_elems) * 4);
  };

  if (tid == 0) {
    s_abort = 0;
    for (int i = 0; i < 5; ++i) mbar_init(&bars[i], 1);
    fence_mbar_init();
  }
  {
    const uint32_t a1b = (uint32_t)(p.K1 / 8) * LBO_M128, a2b = (uint32_t)(p.K2 / 8) * LBO_M128_PAD;
    for (uint32_t i = tid; i < a1b / 16; i += P1T) ((uint4*)A1)[i] = make_uint4(0, 0, 0, 0);
    for (uint32_t i = tid; i < a2b / 16; i += P1T) ((uint4*)A2)[i] = make_uint4(0, 0, 0, 0);
  }
  __syncthreads();
  if (warp == 0) tmem_alloc(tslot, 512);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tslot;
  const uint32_t d1 = tmem, d2 = tmem + 256;

  // thread 0's record of outstanding asynchronous work, for a bounded drain
  uint32_t ld_issued[2] = {0, 0}, ld_waited[2] = {0, 0};
  uint32_t m1_issued = 0, m2_issued = 0;
  if (tid == 0) {
    uint32_t b1 = (uint32_t)(p.N1 * p.K1 * 2), b2 = (uint32_t)(p.N2 * p.K2 * 2);
    mbar_expect_tx(&bars[0], b1 + b2);
    bulk_g2s(B1, p.B1img, b1, &bars[0]);
    bulk_g2s(B2, p.B2img, b2, &bars[0]);
    for (int s = 0; s < 2 && s < n_it; ++s) {
      int64_t t = tile_at(s);
      uint32_t nb = tile_bytes(t);
      mbar_expect_tx(&bars[1 + s], nb);
      bulk_g2s(stage[s], p.G + t * p.tile_elems, nb, &bars[1 + s]);
      ld_issued[s]++;
    }
  }
  // Every wait is bounded; the abort decision is made uniform by a barrier so
  // that warp-collective tcgen05 instructions never run in a divergent warp.
  auto wait_all = [&](uint64_t* bar, uint32_t parity) -> bool {
    if (!mbar_wait(bar, parity, WAIT_NS)) {
      atomicOr(p.err, DEV_ERR_TIMEOUT);
      s_abort = 1;
    }
    __syncthreads();
    return s_abort == 0;
  };
  wait_all(&bars[0], 0);

  const uint32_t lbo_b1 = (uint32_t)(p.N1 / 8) * 128, lbo_b2 = (uint32_t)(p.N2 / 8) * 128;
  const uint32_t id1 = idesc_f16(0, 128, p.N1), id2 = idesc_f16(1, 128, p.N2);
  const uint32_t sA1 = smem_u32(A1), sA2 = smem_u32(A2), sB1 = smem_u32(B1), sB2 = smem_u32(B2);
  const int vc = p.asp.cmode == 1 ? 2 : 1;

  // Omega entries of the next tile, prefetched into registers one tile ahead.
  int64_t pf_e0 = 0, pf_e1 = 0;
  uint32_t pf_loc[PF];
  float2 pf_m[PF], pf_v[PF];
  auto load_pf = [&](int64_t t) {
    pf_e0 = p.tile_off[t];
    pf_e1 = p.tile_off[t + 1];
#pragma unroll
    for (int j = 0; j < PF; ++j) {
      int64_t e = pf_e0 + tid + (int64_t)P1T * j;
      if (e < pf_e1) {
        pf_loc[j] = p.loc[e];
        pf_m[j] = ((const float2*)p.sp_m)[e];
        pf_v[j] = vc == 2 ? ((const float2*)p.sp_v)[e] : make_float2(p.sp_v[e], 0.f);
      }
    }
  };
  auto apply_sparse = [&](uint32_t* sw, int64_t e, uint32_t l, float2 m, float2 v) {
    uint32_t u = sw[l];
    sw[l] = 0u;
    float mm[2] = {m.x, m.y}, vv[2] = {v.x, v.y};
    float2 upd = adam_elem(h2_to_f2(u), mm, vv, p.asp);
    ((float2*)p.sp_m)[e] = make_float2(mm[0], mm[1]);
    if (vc == 2)
      ((float2*)p.sp_v)[e] = make_float2(vv[0], vv[1]);
    else
      p.sp_v[e] = vv[0];
    p.sp_upd[e] = f2_to_h2(upd);
  };

  auto epilogue1 = [&](int64_t it) {
    const int64_t t = tile_at(it);
    const int i = (int)(it % p.q);
    const int m = tid, sl = m / p.Ia, ia = m - sl * p.Ia;
    const bool valid = t * p.spb + sl < p.n_slabs;
    const int m2base = (i * p.spb + sl) * p.rb;
    for (int c0 = 0; c0 < p.N1; c0 += 16) {
      float v[16];
      tmem_ld16(d1 + lane_base + c0, v);
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        int jb = c0 / 2 + u;
        if (valid && jb < p.rb) {
          uint32_t off = kmaj_off((uint32_t)(m2base + jb), (uint32_t)(2 * ia), LBO_M128_PAD);
          *(uint32_t*)(A2 + off) = f2_to_bf2(v[2 * u], v[2 * u + 1]);
        }
      }
    }
  };
  auto epilogue2 = [&](int64_t g) {
    const int m2 = tid, sb = m2 / p.rb, jb = m2 - sb * p.rb;
    const int64_t slab = g * p.sg + sb;
    const bool valid = m2 < p.sg * p.rb && slab < p.n_slabs;
    const int64_t ybase = (slab * p.rb + jb) * p.ra;
    for (int c0 = 0; c0 < p.N2; c0 += 16) {
      float v[16];
      tmem_ld16(d2 + lane_base + c0, v);
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        int ja = c0 / 2 + u;
        if (valid && ja < p.ra) {
          if (p.y_f32)
            ((float2*)p.Y)[ybase + ja] = make_float2(v[2 * u], v[2 * u + 1]);
          else
            ((uint32_t*)p.Y)[ybase + ja] = f2_to_bf2(v[2 * u], v[2 * u + 1]);
        }
      }
    }
  };
  auto issue_gemm1 = [&]() {
    for (int kk = 0; kk < p.K1 / 16; ++kk)
      mma_f16(d1, sdesc(sA1 + kk * 2 * LBO_M128, LBO_M128, 128),
              sdesc(sB1 + kk * 2 * lbo_b1, lbo_b1, 128), id1, kk > 0);
    mma_commit(&bars[3]);
  };
  auto issue_gemm2 = [&]() {
    for (int kk = 0; kk < p.K2 / 16; ++kk)
      mma_f16(d2, sdesc(sA2 + kk * 2 * LBO_M128_PAD, LBO_M128_PAD, 128),
              sdesc(sB2 + kk * 2 * lbo_b2, lbo_b2, 128), id2, kk > 0);
    mma_commit(&bars[4]);
  };

  uint32_t m1_waited = 0, m2_waited = 0;
  if (n_it > 0 && !s_abort) load_pf(tile_at(0));
  __syncthreads();
  for (int64_t it = 0; it < n_it && !s_abort; ++it) {
    const int s = (int)(it & 1);
    const int64_t t = tile_at(it);
    uint32_t* sw = (uint32_t*)stage[s];
    const bool got = wait_all(&bars[1 + s], (uint32_t)((it >> 1) & 1));
    if (tid == 0) ld_waited[s]++;
    if (!got) break;
    {
      // sparse pass: gather, residual, sparse AdamW
      const int64_t e0 = pf_e0, e1 = pf_e1;
#pragma unroll
      for (int j = 0; j < PF; ++j) {
        int64_t e = e0 + tid + (int64_t)P1T * j;
        if (e < e1) apply_sparse(sw, e, pf_loc[j], pf_m[j], pf_v[j]);
      }
      for (int64_t e = e0 + (int64_t)P1T * PF + tid; e < e1; e += P1T) {
        float2 m = ((const float2*)p.sp_m)[e];
        float2 v = vc == 2 ? ((const float2*)p.sp_v)[e] : make_float2(p.sp_v[e], 0.f);
        apply_sparse(sw, e, p.loc[e], m, v);
      }
      if (it + 1 < n_it) load_pf(tile_at(it + 1));
    }
    if (it > 0) {
      const bool ok1 = wait_all(&bars[3], (uint32_t)((it - 1) & 1));
      m1_waited++;
      if (!ok1) break;
      tc_fence_after();
      epilogue1(it - 1);
    } else {
      __syncthreads();
    }
    // residual tile -> GEMM1's A operand (row = i_a of a slab, K = (i_b, re/im))
    {
      const int m = tid, sl = m / p.Ia;
      const bool valid = t * p.spb + sl < p.n_slabs;
      const uint32_t* src = sw + (int64_t)m * p.Ib;
      for (int kc = 0; kc < p.K1 / 8; ++kc) {
        uint32_t v[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          int ib = 4 * kc + u;
          v[u] = (valid && ib < p.Ib) ? src[ib] : 0u;
        }
        *(uint4*)(A1 + kc * LBO_M128 + m * 16) = make_uint4(v[0], v[1], v[2], v[3]);
      }
    }
    fence_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (s_abort) break;
    const bool prev_last = it > 0 && is_last(it - 1);
    if (tid == 0) {
      if (it + 2 < n_it) {
        int64_t t2 = tile_at(it + 2);
        uint32_t nb = tile_bytes(t2);
        mbar_expect_tx(&bars[1 + s], nb);
        bulk_g2s(stage[s], p.G + t2 * p.tile_elems, nb, &bars[1 + s]);
        ld_issued[s]++;
      }
      if (prev_last) {
        issue_gemm2();
        m2_issued++;
      }
      issue_gemm1();
      m1_issued++;
    }
    if (prev_last) {
      const bool ok2 = wait_all(&bars[4], m2_waited & 1u);
      m2_waited++;
      if (!ok2) break;
      tc_fence_after();
      epilogue2(group_at(it - 1));
      tc_fence_before();
      __syncthreads();
      tc_fence_after();
    }
  }
  __syncthreads();
  if (n_it > 0 && !s_abort) {
    const bool ok1 = wait_all(&bars[3], (uint32_t)((n_it - 1) & 1));
    m1_waited++;
    if (ok1) {
      tc_fence_after();
      epilogue1(n_it - 1);
      fence_async_smem();
      tc_fence_before();
      __syncthreads();
      tc_fence_after();
      if (tid == 0) {
        issue_gemm2();
        m2_issued++;
      }
      const bool ok2 = wait_all(&bars[4], m2_waited & 1u);
      m2_waited++;
      if (ok2) {
        tc_fence_after();
        epilogue2(group_at(n_it - 1));
      }
    }
  }
  // Bounded drain of anything still in flight (only after a timeout).
  if (tid == 0 && s_abort) {
    for (int s = 0; s < 2; ++s)
      while (ld_waited[s] < ld_issued[s]) {
        mbar_wait(&bars[1 + s], ld_waited[s] & 1u, WAIT_NS / 4);
        ld_waited[s]++;
      }
    if (m1_issued > m1_waited) mbar_wait(&bars[3], (m1_issued - 1) & 1u, WAIT_NS / 4);
    if (m2_issued > m2_waited) mbar_wait(&bars[4], (m2_issued - 1) & 1u, WAIT_NS / 4);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) tmem_dealloc(tmem, 512);
}

// ------------------------------------------------------- inner-mode GEMM
constexpr int MGT = 128;

struct MGArgs {
  const uint32_t* X;
  int64_t rows, K, B, in_bs;
  void* Y;
  int y_f32;
  int64_t J, out_bs;
  const uint8_t* img;
  int NT, nkc;
  uint32_t tmem_cols;
  int* err;
};

// Y[a][j][b] = sum_k X[a][k][b] M[k][j] (complex, bf16 in, fp32 accumulate).
// Rows of the GEMM are 128 consecutive (a, b) positions; each thread gathers
// its row's K values (coalesced across threads), so any mode is contracted
// without a transpose in memory.
__global__ void __launch_bounds__(MGT) mode_gemm_kernel(const MGArgs p) {
  extern __shared__ __align__(1024) uint8_t smem[];
  const uint32_t a_bytes = 8 * LBO_M128;               // 128 rows x 64 K
  const uint32_t b_bytes = (uint32_t)p.NT * 64 * 2;
  uint8_t* As[2] = {smem, smem + a_bytes};
  uint8_t* Bs[2] = {smem + 2 * a_bytes, smem + 2 * a_bytes + b_bytes};
  uint64_t* bars = (uint64_t*)(smem + 2 * a_bytes + 2 * b_bytes);
  uint32_t* tslot = (uint32_t*)(bars + 4);
  __shared__ int s_abort;
  const int tid = threadIdx.x, warp = tid >> 5;
  const uint32_t lane_base = (uint32_t)(warp * 32) << 16;
  const int64_t rho = (int64_t)blockIdx.x * MGT + tid;
  const bool valid = rho < p.rows;
  const int64_t a = valid ? rho / p.B : 0, b = valid ? rho - a * p.B : 0;
  const uint32_t* xrow = p.X + a * p.K * p.in_bs + b;
  if (tid == 0) {
    s_abort = 0;
    mbar_init(&bars[0], 1);
    mbar_init(&bars[1], 1);
    fence_mbar_init();
  }
  __syncthreads();
  if (warp == 0) tmem_alloc(tslot, p.tmem_cols);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t dt = *tslot;
  const uint32_t lbo_b = (uint32_t)(p.NT / 8) * 128;
  const uint32_t idesc = idesc_f16(1, 128, p.NT);
  const uint8_t* img = p.img + (int64_t)blockIdx.y * p.nkc * b_bytes;
  uint32_t issued[2] = {0, 0}, waited[2] = {0, 0};
  auto wait_all = [&](uint64_t* bar, uint32_t parity) -> bool {
    if (!mbar_wait(bar, parity, WAIT_NS)) {
      atomicOr(p.err, DEV_ERR_TIMEOUT);
      s_abort = 1;
    }
    __syncthreads();
    return s_abort == 0;
  };
  for (int kc = 0; kc < p.nkc; ++kc) {
    const int s = kc & 1;
    if (kc >= 2) {
      const bool ok = wait_all(&bars[s], waited[s] & 1u);
      waited[s]++;
      if (!ok) break;
      tc_fence_after();
    }
#pragma unroll
    for (int q = 0; q < 8; ++q) {
      uint32_t v[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        int64_t k = (int64_t)kc * 32 + 4 * q + u;
        v[u] = (valid && k < p.K) ? __ldg(xrow + k * p.in_bs) : 0u;
      }
      *(uint4*)(As[s] + q * LBO_M128 + tid * 16) = make_uint4(v[0], v[1], v[2], v[3]);
    }
    const uint4* src = (const uint4*)(img + (int64_t)kc * b_bytes);
    for (uint32_t i = tid; i < b_bytes / 16; i += MGT) ((uint4*)Bs[s])[i] = __ldg(src + i);
    fence_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (s_abort) break;
    if (tid == 0) {
      const uint32_t sa = smem_u32(As[s]), sb = smem_u32(Bs[s]);
      for (int kk = 0; kk < 4; ++kk)
        mma_f16(dt, sdesc(sa + kk * 2 * LBO_M128, LBO_M128, 128), sdesc(sb + kk * 2 * lbo_b, lbo_b, 128),
                idesc, (kc > 0 || kk > 0) ? 1u : 0u);
      mma_commit(&bars[s]);
    }
    issued[s]++;
  }
  __syncthreads();
  if (!s_abort) {
    const int s = (p.nkc - 1) & 1;
    wait_all(&bars[s], waited[s] & 1u);
    waited[s]++;
    tc_fence_after();
  }
  if (!s_abort) {
    const int64_t j0 = (int64_t)blockIdx.y * (p.NT / 2);
    for (int c0 = 0; c0 < p.NT; c0 += 16) {
      float v[16];
      tmem_ld16(dt + lane_base + c0, v);
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        int64_t j = j0 + c0 / 2 + u;
        if (valid && j < p.J) {
          int64_t o = (a * p.J + j) * p.out_bs + b;
          if (p.y_f32)
            ((float2*)p.Y)[o] = make_float2(v[2 * u], v[2 * u + 1]);
          else
            ((uint32_t*)p.Y)[o] = f2_to_bf2(v[2 * u], v[2 * u + 1]);
        }
      }
    }
  } else if (tid == 0) {
    for (int s = 0; s < 2; ++s)
      if (issued[s] > waited[s]) mbar_wait(&bars[s], (issued[s] - 1) & 1u, WAIT_NS / 4);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) tmem_dealloc(dt, p.tmem_cols);
}

// ------------------------------------------------------------ core Adam
// C~ = Adam(C) on the core (fp32 in, bf16 out). Element j of the core lands
// at (j / blk) * out_bs + j % blk, which pads the innermost (j_b, j_a) block
// when the output is the reconstruction's slab input.
__global__ void core_adam_tc_kernel(const float2* C, int64_t n, int64_t blk, int64_t out_bs,
                                    float* m, float* v, AdamConst a, uint32_t* out) {
  const int vc = a.cmode == 1 ? 2 : 1;
  for (int64_t j = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; j < n;
       j += (int64_t)gridDim.x * blockDim.x) {
    float mm[2] = {m[2 * j], m[2 * j + 1]}, vv[2];
    for (int q = 0; q < vc; ++q) vv[q] = v[j * vc + q];
    float2 u = adam_elem(C[j], mm, vv, a);
    m[2 * j] = mm[0];
    m[2 * j + 1] = mm[1];
    for (int q = 0; q < vc; ++q) v[j * vc + q] = vv[q];
    out[(j / blk) * out_bs + j % blk] = f2_to_bf2(u.x, u.y);
  }
}

// ------------------------------------------------------- reconstruction
constexpr int R3T = 256;

struct R3Args {
  const uint32_t* Yp;
  int64_t yp_bs;  // u32 (complex) per slab in Y'
  void* W;
  int w_c64;
  int64_t N, n_slabs, n_tiles, tile_elems;
  int Ia, Ib, ra, rb, spb;
  int K1, N1, K2, N2;
  const int64_t* tile_off;
  const uint16_t* loc;
  const uint32_t* sp_upd;
  const uint8_t* A1img;
  const uint8_t* B2img;
  float decay, lr;
  int* err;
  int nstage, cap;
  uint32_t w_tile_bytes, y_tile_bytes;
  uint32_t off_w, off_y, off_A1, off_B1, off_A2, off_B2, off_lloc, off_lval, off_bar;
};

__global__ void __launch_bounds__(R3T, 1) recon_stream_kernel(const R3Args p) {
  extern __shared__ __align__(1024) uint8_t smem[];
  uint8_t* A1 = smem + p.off_A1;
  uint8_t* B1 = smem + p.off_B1;
  uint8_t* A2 = smem + p.off_A2;
  uint8_t* B2 = smem + p.off_B2;
  uint16_t* lloc = (uint16_t*)(smem + p.off_lloc);
  uint32_t* lval = (uint32_t*)(smem + p.off_lval);
  uint64_t* bars = (uint64_t*)(smem + p.off_bar);  // 0..2 stages, 3 operands, 4 gemm1, 5 gemm2
  uint32_t* tslot = (uint32_t*)(bars + 8);
  __shared__ int s_abort;
  const int tid = threadIdx.x, warp = tid >> 5;
  const uint32_t lane_base = (uint32_t)((warp & 3) * 32) << 16;
  const int64_t n_it =
      p.n_tiles > (int64_t)blockIdx.x ? (p.n_tiles - 1 - blockIdx.x) / gridDim.x + 1 : 0;
  auto tile_at = [&](int64_t it) -> int64_t { return blockIdx.x + it * gridDim.x; };
  auto wst = [&](int s) { return smem + p.off_w + (uint32_t)s * p.w_tile_bytes; };
  auto yst = [&](int s) { return smem + p.off_y + (uint32_t)s * p.y_tile_bytes; };
  const int wb = p.w_c64 ? 8 : 4;
  auto tile_wbytes = [&](int64_t t) -> uint32_t {
    int64_t rem = p.N - t * p.tile_elems;
    return (uint32_t)((rem < p.tile_elems ? rem : p.tile_elems) * wb);
  };
  auto tile_ybytes = [&](int64_t t) -> uint32_t {
    int64_t rem = p.n_slabs - t * p.spb;
    return (uint32_t)((rem < p.spb ? rem : p.spb) * p.yp_bs * 4);
  };
  if (tid == 0) {
    s_abort = 0;
    for (int i = 0; i < 6; ++i) mbar_init(&bars[i], 1);
    fence_mbar_init();
  }
  {
    const uint32_t b1b = (uint32_t)(p.N1 * p.K1 * 2), a2b = (uint32_t)(p.K2 / 8) * LBO_M128;
    for (uint32_t i = tid; i < b1b / 16; i += R3T) ((uint4*)B1)[i] = make_uint4(0, 0, 0, 0);
    for (uint32_t i = tid; i < a2b / 16; i += R3T) ((uint4*)A2)[i] = make_uint4(0, 0, 0, 0);
  }
  __syncthreads();
  if (warp == 0) tmem_alloc(tslot, 512);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tslot;
  const uint32_t d1 = tmem, d2 = tmem + 256;
  uint32_t ld_issued[3] = {0, 0, 0}, ld_waited[3] = {0, 0, 0};
  auto issue_loads = [&](int64_t it) {
    const int s = (int)(it % p.nstage);
    const int64_t t = tile_at(it);
    const uint32_t nw = tile_wbytes(t), ny = tile_ybytes(t);
    mbar_expect_tx(&bars[s], nw + ny);
    bulk_g2s(wst(s), (const uint8_t*)p.W + t * p.tile_elems * wb, nw, &bars[s]);
    bulk_g2s(yst(s), p.Yp + t * p.spb * p.yp_bs, ny, &bars[s]);
    ld_issued[s]++;
  };
  if (tid == 0) {
    const uint32_t a1b = (uint32_t)(p.K1 / 8) * LBO_M128, b2b = (uint32_t)(p.N2 * p.K2 * 2);
    mbar_expect_tx(&bars[3], a1b + b2b);
    bulk_g2s(A1, p.A1img, a1b, &bars[3]);
    bulk_g2s(B2, p.B2img, b2b, &bars[3]);
    for (int64_t it = 0; it < p.nstage - 1 && it < n_it; ++it) issue_loads(it);
  }
  auto wait_all = [&](uint64_t* bar, uint32_t parity) -> bool {
    if (!mbar_wait(bar, parity, WAIT_NS)) {
      atomicOr(p.err, DEV_ERR_TIMEOUT);
      s_abort = 1;
    }
    __syncthreads();
    return s_abort == 0;
  };
  wait_all(&bars[3], 0);
  const uint32_t lbo_b1 = (uint32_t)(p.N1 / 8) * 128, lbo_b2 = (uint32_t)(p.N2 / 8) * 128;
  const uint32_t id1 = idesc_f16(1, 128, p.N1), id2 = idesc_f16(1, 128, p.N2);
  const uint32_t sA1 = smem_u32(A1), sB1 = smem_u32(B1), sA2 = smem_u32(A2), sB2 = smem_u32(B2);
  const int blk = p.rb * p.ra;
  uint32_t m1_waited = 0, m2_waited = 0, m1_issued = 0, m2_issued = 0;
  __syncthreads();
  for (int64_t it = 0; it < n_it && !s_abort; ++it) {
    const int s = (int)(it % p.nstage);
    const int64_t t = tile_at(it);
    const bool got = wait_all(&bars[s], (uint32_t)((it / p.nstage) & 1));
    if (tid == 0) ld_waited[s]++;
    if (!got) break;
    const int64_t e0 = p.tile_off[t], e1 = p.tile_off[t + 1];
    const int cnt = (int)(e1 - e0);
    // GEMM1's B operand: the tile's Y' slabs in the embedding [[Yr, Yi], [-Yi, Yr]]
    {
      const uint32_t* ys = (const uint32_t*)yst(s);
      const int64_t vslabs = p.n_slabs - t * p.spb;
      for (int e = tid; e < p.spb * blk; e += R3T) {
        const int sl = e / blk, r2 = e - sl * blk, jb = r2 / p.ra, ja = r2 - jb * p.ra;
        float2 y = sl < vslabs ? bf2_to_f2(ys[sl * p.yp_bs + r2]) : make_float2(0.f, 0.f);
        const uint32_t k = (uint32_t)(sl * 2 * p.ra + 2 * ja);
        *(uint32_t*)(B1 + kmaj_off((uint32_t)(2 * jb), k, lbo_b1)) = f2_to_bf2(y.x, -y.y);
        *(uint32_t*)(B1 + kmaj_off((uint32_t)(2 * jb + 1), k, lbo_b1)) = f2_to_bf2(y.y, y.x);
      }
    }
    // Omega entries of the tile (local index and fp16 S~) into shared memory
    if (cnt <= p.cap) {
      for (int j = tid; j < cnt; j += R3T) {
        lloc[j] = p.loc[e0 + j];
        lval[j] = p.sp_upd[e0 + j];
      }
    }
    fence_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (s_abort) break;
    if (tid == 0) {
      for (int kk = 0; kk < p.K1 / 16; ++kk)
        mma_f16(d1, sdesc(sA1 + kk * 2 * LBO_M128, LBO_M128, 128),
                sdesc(sB1 + kk * 2 * lbo_b1, lbo_b1, 128), id1, kk > 0);
      mma_commit(&bars[4]);
      m1_issued++;
      if (it + p.nstage - 1 < n_it) {
        bulk_wait_read0();  // the stage being refilled was last stored from
        issue_loads(it + p.nstage - 1);
      }
    }
    const bool ok1 = wait_all(&bars[4], m1_waited & 1u);
    m1_waited++;
    if (!ok1) break;
    tc_fence_after();
    if (warp < 4) {
      // P' row (this thread's i_a) -> GEMM2's A operand
      for (int c0 = 0; c0 < p.N1; c0 += 16) {
        float v[16];
        tmem_ld16(d1 + lane_base + c0, v);
        uint32_t w[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) w[u] = f2_to_bf2(v[2 * u], v[2 * u + 1]);
        *(uint4*)(A2 + (c0 / 8) * LBO_M128 + tid * 16) = make_uint4(w[0], w[1], w[2], w[3]);
        *(uint4*)(A2 + (c0 / 8 + 1) * LBO_M128 + tid * 16) = make_uint4(w[4], w[5], w[6], w[7]);
      }
    }
    fence_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (s_abort) break;
    if (tid == 0) {
      for (int kk = 0; kk < p.K2 / 16; ++kk)
        mma_f16(d2, sdesc(sA2 + kk * 2 * LBO_M128, LBO_M128, 128),
                sdesc(sB2 + kk * 2 * lbo_b2, lbo_b2, 128), id2, kk > 0);
      mma_commit(&bars[5]);
      m2_issued++;
    }
    const bool ok2 = wait_all(&bars[5], m2_waited & 1u);
    m2_waited++;
    if (!ok2) break;
    tc_fence_after();
    {
      // Delta row + lambda S~ on Omega, then the AdamW weight update in place.
      const int m = tid & 127, h = tid >> 7;
      const int sl = m / p.Ia;
      const bool valid = t * p.spb + sl < p.n_slabs;
      const int nch = p.N2 / 16, nch0 = (nch + 1) / 2;
      const int c_lo = h ? nch0 : 0, c_hi = h ? nch : nch0;
      const uint32_t erow = (uint32_t)m * p.Ib;
      const uint16_t* L = cnt <= p.cap ? lloc : p.loc + e0;
      const uint32_t* V = cnt <= p.cap ? lval : p.sp_upd + e0;
      int lo = 0, hi = cnt;
      const uint32_t first = erow + (uint32_t)c_lo * 8;
      while (lo < hi) {
        int mid = (lo + hi) >> 1;
        if ((uint32_t)L[mid] < first)
          lo = mid + 1;
        else
          hi = mid;
      }
      int ptr = lo;
      uint8_t* ws = wst(s);
      for (int c = c_lo; c < c_hi; ++c) {
        float v[16];
        tmem_ld16(d2 + lane_base + c * 16, v);
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          const int ib = c * 8 + u;
          if (valid && ib < p.Ib) {
            const uint32_t le = erow + (uint32_t)ib;
            float dx = v[2 * u], dy = v[2 * u + 1];
            while (ptr < cnt && (uint32_t)L[ptr] == le) {
              float2 su = h2_to_f2(V[ptr]);
              dx += su.x;
              dy += su.y;
              ++ptr;
            }
            if (p.w_c64) {
              float2* wp = (float2*)ws + le;
              float2 w = *wp;
              *wp = make_float2(__fmaf_rn(-p.lr, dx, w.x * p.decay), __fmaf_rn(-p.lr, dy, w.y * p.decay));
            } else {
              uint32_t* wp = (uint32_t*)ws + le;
              float2 w = h2_to_f2(*wp);
              *wp = f2_to_h2(make_float2(__fmaf_rn(-p.lr, dx, w.x * p.decay),
                                         __fmaf_rn(-p.lr, dy, w.y * p.decay)));
            }
          }
        }
      }
    }
    fence_async_smem();
    __syncthreads();
    if (s_abort) break;
    if (tid == 0) {
      bulk_s2g((uint8_t*)p.W + t * p.tile_elems * wb, wst(s), tile_wbytes(t));
      bulk_commit();
    }
  }
  __syncthreads();
  if (tid == 0) {
    if (s_abort) {
      for (int s = 0; s < p.nstage; ++s)
        while (ld_waited[s] < ld_issued[s]) {
          mbar_wait(&bars[s], ld_waited[s] & 1u, WAIT_NS / 4);
          ld_waited[s]++;
        }
      if (m1_issued > m1_waited) mbar_wait(&bars[4], (m1_issued - 1) & 1u, WAIT_NS / 4);
      if (m2_issued > m2_waited) mbar_wait(&bars[5], (m2_issued - 1) & 1u, WAIT_NS / 4);
    }
    bulk_wait_all0();
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) tmem_dealloc(tmem, 512);
}

// ----------------------------------------------------- operand images
// Embedding of the complex matrix M (Kc x Jc) for y = x M as a real B operand
// (rows n = (j, re/im), columns k = (kk, re/im)):
//   E[(kk,0)][(j,0)] = Mr, E[(kk,1)][(j,0)] = -Mi, E[(kk,0)][(j,1)] = Mi, E[(kk,1)][(j,1)] = Mr.
// M comes from U (I x r): kind 0: M = conj(U) (Kc = I, Jc = r, projection);
// kind 1: M = U^T (Kc = r, Jc = I, expansion). Zero padded to Np x Kp and
// stored as (NT x KCH) blocks, [n-block][k-block], each block in the K-major
// no-swizzle layout with 8-row groups 128 B apart and LBO = NT / 8 * 128 B.
__global__ void embed_image_kernel(const float2* U, int I, int r, int kind, int Np, int Kp, int NT,
                                   int KCH, int as_fp16, uint16_t* img) {
  const int nkb = Kp / KCH;
  const int Kc = kind == 0 ? I : r, Jc = kind == 0 ? r : I;
  for (int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; e < (int64_t)Np * Kp;
       e += (int64_t)gridDim.x * blockDim.x) {
    const int n = (int)(e / Kp), k = (int)(e - (int64_t)n * Kp);
    const int j = n >> 1, cp = n & 1, kk = k >> 1, c = k & 1;
    float val = 0.f;
    if (j < Jc && kk < Kc) {
      float2 u = kind == 0 ? U[(int64_t)kk * r + j] : U[(int64_t)j * r + kk];
      float mr = u.x, mi = kind == 0 ? -u.y : u.y;
      val = (c == 0) ? (cp == 0 ? mr : mi) : (cp == 0 ? -mi : mr);
    }
    const int nb = n / NT, nl = n - nb * NT, kb = k / KCH, kl = k - kb * KCH;
    const int64_t base = ((int64_t)nb * nkb + kb) * NT * KCH;
    const uint32_t off = kmaj_off((uint32_t)nl, (uint32_t)kl, (uint32_t)(NT / 8) * 128u) / 2;
    uint16_t bits;
    if (as_fp16) {
      __half hv = __float2half_rn(val);
      bits = *reinterpret_cast<uint16_t*>(&hv);
    } else {
      __nv_bfloat16 bv = __float2bfloat16_rn(val);
      bits = *reinterpret_cast<uint16_t*>(&bv);
    }
    img[base + off] = bits;
  }
}

// A operand of the reconstruction's first GEMM: 128 rows (slab sl, i_a),
// K = (slab sl', j_a, re/im); block-diagonal over the tile's slabs with
// entries Ur (re column) and Ui (im column) of U_a[i_a][j_a]. K-major,
// no-swizzle, LBO = 2048 B.
__global__ void blockdiag_image_kernel(const float2* U, int Ia, int ra, int spb, int Kp,
                                       uint16_t* img) {
  for (int e = blockIdx.x * blockDim.x + threadIdx.x; e < 128 * Kp; e += gridDim.x * blockDim.x) {
    const int m = e / Kp, k = e - m * Kp;
    const int sl = m / Ia, ia = m - sl * Ia;
    const int slk = k / (2 * ra), rem = k - slk * 2 * ra, ja = rem >> 1, c = rem & 1;
    float val = 0.f;
    if (sl == slk && slk < spb) {
      float2 u = U[(int64_t)ia * ra + ja];
      val = c == 0 ? u.x : u.y;
    }
    __nv_bfloat16 bv = __float2bfloat16_rn(val);
    img[kmaj_off((uint32_t)m, (uint32_t)k, LBO_M128) / 2] = *reinterpret_cast<uint16_t*>(&bv);
  }
}

// ------------------------------------------------------------ host side
int r16(int x) { return (x + 15) / 16 * 16; }
int pow2_cols(int n) {
  int c = 32;
  while (c < n) c <<= 1;
  return c;
}

struct InnerMode {
  int n = 0;
  int64_t I = 0, r = 0;
  bool active = false;
  uint16_t* img_p = nullptr;  // projection (kind 0)
  uint16_t* img_e = nullptr;  // expansion (kind 1)
  int NTp = 0, nntp = 0, nkcp = 0, NTe = 0, nnte = 0, nkce = 0;
};

struct TcImpl {
  int d = 0, Ia = 0, Ib = 0, ra = 0, rb = 0, spb = 0, q = 0, sg = 0;
  int64_t n_slabs = 0, n_tiles = 0, n_groups = 0, tile_elems = 0, blk = 0, bs_pad = 0;
  int K1 = 0, N1 = 0, K2 = 0, N2 = 0;
  int rK1 = 0, rN1 = 0, rK2 = 0, rN2 = 0;
  int wdt = 0;
  std::vector<InnerMode> inner;
  int64_t* tile_off = nullptr;
  uint16_t* loc = nullptr;
  uint32_t* sp_upd = nullptr;
  uint32_t* Y = nullptr;
  uint32_t* X0 = nullptr;
  uint32_t* X1 = nullptr;
  float* C = nullptr;
  uint32_t* Ct = nullptr;
  uint32_t* Yp = nullptr;
  uint16_t *B1img = nullptr, *B2img = nullptr, *rA1img = nullptr, *rB2img = nullptr;
  P1Args p1{};
  R3Args r3{};
  size_t p1_smem = 0, r3_smem = 0, mg_smem_max = 0;
  int num_sms = 148;
  const float* U[8] = {};
};

size_t p1_smem_bytes(int Ib, int K1, int K2, int N1, int N2, P1Args* a) {
  size_t off = 0;
  auto take = [&](size_t b) {
    size_t o = off;
    off += (b + 127) / 128 * 128;
    return (uint32_t)o;
  };
  size_t tile = (size_t)128 * Ib * 4;
  uint32_t s0 = take(tile), s1 = take(tile);
  uint32_t a1 = take((size_t)(K1 / 8) * LBO_M128), a2 = take((size_t)(K2 / 8) * LBO_M128_PAD);
  uint32_t b1 = take((size_t)N1 * K1 * 2), b2 = take((size_t)N2 * K2 * 2);
  uint32_t bar = take(128);
  if (a) {
    a->off_stage0 = s0;
    a->off_stage1 = s1;
    a->off_A1 = a1;
    a->off_A2 = a2;
    a->off_B1 = b1;
    a->off_B2 = b2;
    a->off_bar = bar;
  }
  return off;
}

size_t r3_smem_bytes(int Ib, int spb, int64_t yp_bs, int wbytes, int nstage, int K1, int N1, int K2,
                     int N2, int cap, R3Args* a) {
  size_t off = 0;
  auto take = [&](size_t b) {
    size_t o = off;
    off += (b + 127) / 128 * 128;
    return (uint32_t)o;
  };
  size_t wt = (size_t)128 * Ib * wbytes, yt = (size_t)spb * yp_bs * 4;
  wt = (wt + 127) / 128 * 128;
  yt = (yt + 127) / 128 * 128;
  uint32_t w = take(wt * nstage), y = take(yt * nstage);
  uint32_t a1 = take((size_t)(K1 / 8) * LBO_M128), b1 = take((size_t)N1 * K1 * 2);
  uint32_t a2 = take((size_t)(K2 / 8) * LBO_M128), b2 = take((size_t)N2 * K2 * 2);
  uint32_t ll = take((size_t)cap * 2), lv = take((size_t)cap * 4), bar = take(128);
  if (a) {
    a->w_tile_bytes = (uint32_t)wt;
    a->y_tile_bytes = (uint32_t)yt;
    a->off_w = w;
    a->off_y = y;
    a->off_A1 = a1;
    a->off_B1 = b1;
    a->off_A2 = a2;
    a->off_B2 = b2;
    a->off_lloc = ll;
    a->off_lval = lv;
    a->off_bar = bar;
  }
  return off;
}

constexpr size_t SMEM_LIMIT = 227 * 1024;
constexpr size_t ONE_CTA_SMEM = 120 * 1024;
constexpr int R3_CAP = 2048;

bool geometry(TcImpl& g, int nd, const int64_t* shape, const int64_t* ranks, int wdt) {
  if (nd < 3) return false;
  g.d = nd;
  g.Ia = (int)shape[nd - 2];
  g.Ib = (int)shape[nd - 1];
  g.ra = (int)ranks[nd - 2];
  g.rb = (int)ranks[nd - 1];
  if (g.Ia < 8 || g.Ia > 128 || (g.Ia & (g.Ia - 1))) return false;
  if (g.Ib < 1 || g.Ib > 120) return false;
  if (g.rb > g.Ia) return false;
  g.spb = 128 / g.Ia;
  g.q = std::max(1, 128 / (g.rb * g.spb));
  g.sg = g.spb * g.q;
  g.n_slabs = 1;
  for (int n = 0; n < nd - 2; ++n) g.n_slabs *= shape[n];
  g.tile_elems = (int64_t)128 * g.Ib;
  g.n_tiles = ceil_div(g.n_slabs, g.spb);
  g.n_groups = ceil_div(g.n_tiles, g.q);
  g.K1 = r16(2 * g.Ib);
  g.N1 = r16(2 * g.rb);
  g.K2 = 2 * g.Ia;
  g.N2 = r16(2 * g.ra);
  g.rK1 = r16(g.spb * 2 * g.ra);
  g.rN1 = r16(2 * g.rb);
  g.rK2 = g.rN1;
  g.rN2 = r16(2 * g.Ib);
  if (g.K1 > 256 || g.N1 > 256 || g.N2 > 256 || g.rK1 > 256 || g.rN2 > 256) return false;
  g.blk = (int64_t)g.rb * g.ra;
  g.bs_pad = (g.blk + 3) / 4 * 4;
  g.wdt = wdt;
  g.p1_smem = p1_smem_bytes(g.Ib, g.K1, g.K2, g.N1, g.N2, nullptr);
  if (g.p1_smem > SMEM_LIMIT) return false;
  int wbytes = wdt == TGD_C64 ? 8 : 4;
  size_t r3a = r3_smem_bytes(g.Ib, g.spb, g.bs_pad, wbytes, 3, g.rK1, g.rN1, g.rK2, g.rN2, R3_CAP, nullptr);
  size_t r3b = r3_smem_bytes(g.Ib, g.spb, g.bs_pad, wbytes, 2, g.rK1, g.rN1, g.rK2, g.rN2, R3_CAP, nullptr);
  g.r3_smem = r3a <= SMEM_LIMIT ? r3a : r3b;
  if (g.r3_smem > SMEM_LIMIT) return false;
  g.inner.clear();
  for (int n = 0; n < nd - 2; ++n) {
    InnerMode m;
    m.n = n;
    m.I = shape[n];
    m.r = ranks[n];
    m.active = ranks[n] < shape[n];
    int Np = r16(2 * (int)m.r), Kp = (int)ceil_div(2 * m.I, 64) * 64;
    m.NTp = Np <= 256 ? Np : 256;
    m.nntp = (int)ceil_div(Np, m.NTp);
    m.nkcp = Kp / 64;
    Np = r16(2 * (int)m.I);
    Kp = (int)ceil_div(2 * m.r, 64) * 64;
    m.NTe = Np <= 256 ? Np : 256;
    m.nnte = (int)ceil_div(Np, m.NTe);
    m.nkce = Kp / 64;
    g.inner.push_back(m);
  }
  // Y' pads each slab's (j_b, j_a) block to a multiple of 4 entries; the last
  // expansion writes that stride only when it is the innermost inner mode.
  bool any = false;
  for (auto& m : g.inner) any |= m.active;
  if (g.bs_pad != g.blk && any && !g.inner.back().active) return false;
  return true;
}

size_t mg_smem(int NT) { return 2 * (size_t)8 * LBO_M128 + 2 * (size_t)NT * 64 * 2 + 64; }

TcImpl* impl_of(TcPlan& p) { return (TcImpl*)p.impl; }
const TcImpl* impl_of(const TcPlan& p) { return (const TcImpl*)p.impl; }

cudaError_t launch_mode_gemm(const uint32_t* X, int64_t A, int64_t K, int64_t B, int64_t in_bs, void* Y,
                             int y_f32, int64_t J, int64_t out_bs, const uint16_t* img, int NT, int nnt,
                             int nkc, int* err, cudaStream_t s) {
  MGArgs a;
  a.X = X;
  a.rows = A * B;
  a.K = K;
  a.B = B;
  a.in_bs = in_bs;
  a.Y = Y;
  a.y_f32 = y_f32;
  a.J = J;
  a.out_bs = out_bs;
  a.img = (const uint8_t*)img;
  a.NT = NT;
  a.nkc = nkc;
  a.tmem_cols = (uint32_t)pow2_cols(NT);
  a.err = err;
  size_t sm = mg_smem(NT);
  cudaError_t e = cudaFuncSetAttribute(mode_gemm_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm);
  if (e != cudaSuccess) return e;
  dim3 grid((unsigned)ceil_div(a.rows, 128), (unsigned)nnt);
  mode_gemm_kernel<<<grid, MGT, sm, s>>>(a);
  return cudaGetLastError();
}

}  // namespace

bool tc_supported(int nd, const int64_t* shape, const int64_t* ranks, int gdt, int wdt) {
  if (gdt != TGD_C32H || (wdt != TGD_C32H && wdt != TGD_C64)) return false;
  TcImpl g;
  return geometry(g, nd, shape, ranks, wdt);
}

bool tc_plan(TcPlan& p, int nd, const int64_t* shape, const int64_t* ranks, int64_t k, int gdt,
             int wdt, AllocFn alloc, void* ctx) {
  TcImpl* g = new TcImpl;
  if (!geometry(*g, nd, shape, ranks, wdt)) {
    delete g;
    return false;
  }
  p.impl = g;
  p.d = nd;
  p.N = 1;
  p.ncore = 1;
  for (int n = 0; n < nd; ++n) {
    p.I[n] = shape[n];
    p.r[n] = ranks[n];
    p.N *= shape[n];
    p.ncore *= ranks[n];
  }
  p.k = k;
  p.gdt = gdt;
  p.wdt = wdt;
  int dev = 0;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&g->num_sms, cudaDevAttrMultiProcessorCount, dev);
  auto A = [&](void** ptr, size_t bytes) { return alloc(ctx, ptr, bytes); };
  bool ok = true;
  ok &= A((void**)&g->tile_off, sizeof(int64_t) * (g->n_tiles + 1));
  ok &= A((void**)&g->loc, sizeof(uint16_t) * std::max<int64_t>(k, 1));
  ok &= A((void**)&g->sp_upd, sizeof(uint32_t) * std::max<int64_t>(k, 1));
  // chain buffers: the largest intermediate of the inner-mode contractions
  int64_t cur = g->n_slabs * g->blk, maxe = cur;
  for (int n = nd - 3; n >= 0; --n) {
    if (!g->inner[n].active) continue;
    cur = cur / shape[n] * ranks[n];
    maxe = std::max(maxe, cur);
  }
  ok &= A((void**)&g->Y, sizeof(uint32_t) * g->n_slabs * g->blk);
  ok &= A((void**)&g->X0, sizeof(uint32_t) * maxe);
  ok &= A((void**)&g->X1, sizeof(uint32_t) * maxe);
  ok &= A((void**)&g->C, sizeof(float2) * p.ncore);
  ok &= A((void**)&g->Ct, sizeof(uint32_t) * p.ncore);
  ok &= A((void**)&g->Yp, sizeof(uint32_t) * g->n_slabs * g->bs_pad);
  ok &= A((void**)&g->B1img, (size_t)g->N1 * g->K1 * 2);
  ok &= A((void**)&g->B2img, (size_t)g->N2 * g->K2 * 2);
  ok &= A((void**)&g->rA1img, (size_t)128 * g->rK1 * 2);
  ok &= A((void**)&g->rB2img, (size_t)g->rN2 * g->rK2 * 2);
  for (auto& m : g->inner) {
    if (!m.active) continue;
    ok &= A((void**)&m.img_p, (size_t)m.nntp * m.NTp * m.nkcp * 64 * 2);
    ok &= A((void**)&m.img_e, (size_t)m.nnte * m.NTe * m.nkce * 64 * 2);
    g->mg_smem_max = std::max(g->mg_smem_max, std::max(mg_smem(m.NTp), mg_smem(m.NTe)));
  }
  p.ready = ok;
  return ok;
}

void tc_release(TcPlan& p) {
  delete impl_of(p);
  p.impl = nullptr;
  p.ready = false;
}

cudaError_t tc_rebuild(TcPlan& p, const int64_t* omega, int64_t k, const float* const* U,
                       cudaStream_t s) {
  TcImpl* g = impl_of(p);
  if (!g) return cudaErrorNotReady;
  cudaError_t e = cudaSuccess;
  if (k > 0) {
    e = build_tile_index(omega, k, g->tile_elems, g->n_tiles, g->tile_off, g->loc, s);
  } else {
    e = cudaMemsetAsync(g->tile_off, 0, sizeof(int64_t) * (g->n_tiles + 1), s);
  }
  if (e != cudaSuccess) return e;
  const int d = p.d;
  const float2* Ua = (const float2*)U[d - 2];
  const float2* Ub = (const float2*)U[d - 1];
  auto blocks = [](int64_t n) { return (unsigned)std::min<int64_t>(ceil_div(n, 256), 4096); };
  embed_image_kernel<<<blocks((int64_t)g->N1 * g->K1), 256, 0, s>>>(Ub, g->Ib, g->rb, 0, g->N1, g->K1,
                                                                      g->N1, g->K1, 1, g->B1img);
  embed_image_kernel<<<blocks((int64_t)g->N2 * g->K2), 256, 0, s>>>(Ua, g->Ia, g->ra, 0, g->N2, g->K2,
                                                                      g->N2, g->K2, 0, g->B2img);
  blockdiag_image_kernel<<<blocks((int64_t)128 * g->rK1), 256, 0, s>>>(Ua, g->Ia, g->ra, g->spb, g->rK1,
                                                                        g->rA1img);
  embed_image_kernel<<<blocks((int64_t)g->rN2 * g->rK2), 256, 0, s>>>(Ub, g->Ib, g->rb, 1, g->rN2,
                                                                        g->rK2, g->rN2, g->rK2, 0, g->rB2img);
  for (auto& m : g->inner) {
    if (!m.active) continue;
    const float2* Un = (const float2*)U[m.n];
    int Np = m.nntp * m.NTp, Kp = m.nkcp * 64;
    embed_image_kernel<<<blocks((int64_t)Np * Kp), 256, 0, s>>>(Un, (int)m.I, (int)m.r, 0, Np, Kp, m.NTp,
                                                                  64, 0, m.img_p);
    Np = m.nnte * m.NTe;
    Kp = m.nkce * 64;
    embed_image_kernel<<<blocks((int64_t)Np * Kp), 256, 0, s>>>(Un, (int)m.I, (int)m.r, 1, Np, Kp, m.NTe,
                                                                  64, 0, m.img_e);
  }
  return cudaGetLastError();
}

cudaError_t tc_step(TcPlan& p, const void* grad, void* w, float* sp_m, float* sp_v, float* core_m,
                    float* core_v, const AdamConst& asp, const AdamConst& acore, float decay, float lr,
                    int* d_err, cudaStream_t s, TimerHook hook, void* hook_ctx) {
  TcImpl* g = impl_of(p);
  if (!g) return cudaErrorNotReady;
  auto H = [&](int ph, const char* name) {
    if (hook) hook(hook_ctx, ph, name, s);
  };
  const int d = p.d;
  int last_active = -1, first_active = -1;
  for (int n = 0; n < d - 2; ++n)
    if (g->inner[n].active) {
      if (first_active < 0) first_active = n;
      last_active = n;
    }
  // ---- projection stream over G
  P1Args& a = g->p1;
  p1_smem_bytes(g->Ib, g->K1, g->K2, g->N1, g->N2, &a);
  a.G = (const uint32_t*)grad;
  a.N = p.N;
  a.n_slabs = g->n_slabs;
  a.n_tiles = g->n_tiles;
  a.n_groups = g->n_groups;
  a.tile_elems = g->tile_elems;
  a.Ia = g->Ia;
  a.Ib = g->Ib;
  a.ra = g->ra;
  a.rb = g->rb;
  a.spb = g->spb;
  a.q = g->q;
  a.sg = g->sg;
  a.K1 = g->K1;
  a.N1 = g->N1;
  a.K2 = g->K2;
  a.N2 = g->N2;
  a.tile_off = g->tile_off;
  a.loc = g->loc;
  a.sp_m = sp_m;
  a.sp_v = sp_v;
  a.sp_upd = g->sp_upd;
  a.asp = asp;
  a.B1img = (const uint8_t*)g->B1img;
  a.B2img = (const uint8_t*)g->B2img;
  const bool no_inner = first_active < 0;
  a.Y = no_inner ? (void*)g->C : (void*)g->Y;
  a.y_f32 = no_inner ? 1 : 0;
  a.err = d_err;
  // At least half the shared memory of an SM, so one CTA (and its 512 TMEM
  // columns) per SM.
  const size_t p1_launch_smem = std::max(g->p1_smem, ONE_CTA_SMEM);
  cudaError_t e = cudaFuncSetAttribute(proj_stream_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)p1_launch_smem);
  if (e != cudaSuccess) return e;
  H(0, "proj_stream");
  proj_stream_kernel<<<(unsigned)std::min<int64_t>(g->n_groups, g->num_sms), P1T, p1_launch_smem, s>>>(a);
  H(1, "proj_stream");
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  // ---- inner modes, innermost first; dims of the current tensor
  int64_t dims[8];
  for (int n = 0; n < d - 2; ++n) dims[n] = p.I[n];
  const uint32_t* cur = g->Y;
  uint32_t* bufs[2] = {g->X0, g->X1};
  int which = 0;
  for (int n = d - 3; n >= 0; --n) {
    InnerMode& m = g->inner[n];
    if (!m.active) continue;
    int64_t A = 1, B = g->blk;
    for (int q = 0; q < n; ++q) A *= dims[q];
    for (int q = n + 1; q < d - 2; ++q) B *= dims[q];
    const bool last = n == first_active;
    void* out = last ? (void*)g->C : (void*)bufs[which];
    H(0, "mode_gemm");
    e = launch_mode_gemm(cur, A, m.I, B, B, out, last ? 1 : 0, m.r, B, m.img_p, m.NTp, m.nntp, m.nkcp,
                         d_err, s);
    H(1, "mode_gemm");
    if (e != cudaSuccess) return e;
    dims[n] = m.r;
    if (!last) {
      cur = bufs[which];
      which ^= 1;
    }
  }
  // ---- Adam on the core; C~ (bf16) feeds the expansion chain, or Y' directly
  {
    const bool direct = no_inner;
    H(0, "core_adam");
    int64_t nc = p.ncore;
    unsigned blocks = (unsigned)std::min<int64_t>(ceil_div(nc, 256), g->num_sms * 8);
    core_adam_tc_kernel<<<blocks, 256, 0, s>>>((const float2*)g->C, nc, g->blk, direct ? g->bs_pad : g->blk,
                                               core_m, core_v, acore, direct ? g->Yp : g->Ct);
    H(1, "core_adam");
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
  }
  // ---- expansion of the inner modes, outermost first; the last writes Y'
  cur = g->Ct;
  which = 0;
  for (int n = 0; n < d - 2; ++n) {
    InnerMode& m = g->inner[n];
    if (!m.active) continue;
    int64_t A = 1, B = g->blk;
    for (int q = 0; q < n; ++q) A *= dims[q];
    for (int q = n + 1; q < d - 2; ++q) B *= dims[q];
    const bool last = n == last_active;
    // Y' pads each slab's (j_b, j_a) block to bs_pad entries: with the slab
    // index outermost, that is an inner stride only for the innermost mode.
    const int64_t out_bs = last ? (B / g->blk) * g->bs_pad : B;
    uint32_t* out = last ? g->Yp : bufs[which];
    H(0, "mode_gemm");
    e = launch_mode_gemm(cur, A, m.r, B, B, out, 0, m.I, out_bs, m.img_e, m.NTe, m.nnte, m.nkce, d_err, s);
    H(1, "mode_gemm");
    if (e != cudaSuccess) return e;
    dims[n] = m.I;
    cur = out;
    which ^= 1;
  }
  // ---- reconstruction stream over W
  R3Args& r = g->r3;
  const int wbytes = g->wdt == TGD_C64 ? 8 : 4;
  size_t need3 = r3_smem_bytes(g->Ib, g->spb, g->bs_pad, wbytes, 3, g->rK1, g->rN1, g->rK2, g->rN2, R3_CAP, nullptr);
  r.nstage = need3 <= SMEM_LIMIT ? 3 : 2;
  r3_smem_bytes(g->Ib, g->spb, g->bs_pad, wbytes, r.nstage, g->rK1, g->rN1, g->rK2, g->rN2, R3_CAP, &r);
  r.cap = R3_CAP;
  r.Yp = g->Yp;
  r.yp_bs = g->bs_pad;
  r.W = w;
  r.w_c64 = g->wdt == TGD_C64 ? 1 : 0;
  r.N = p.N;
  r.n_slabs = g->n_slabs;
  r.n_tiles = g->n_tiles;
  r.tile_elems = g->tile_elems;
  r.Ia = g->Ia;
  r.Ib = g->Ib;
  r.ra = g->ra;
  r.rb = g->rb;
  r.spb = g->spb;
  r.K1 = g->rK1;
  r.N1 = g->rN1;
  r.K2 = g->rK2;
  r.N2 = g->rN2;
  r.tile_off = g->tile_off;
  r.loc = g->loc;
  r.sp_upd = g->sp_upd;
  r.A1img = (const uint8_t*)g->rA1img;
  r.B2img = (const uint8_t*)g->rB2img;
  r.decay = decay;
  r.lr = lr;
  r.err = d_err;
  const size_t r3_launch_smem = std::max(g->r3_smem, ONE_CTA_SMEM);
  e = cudaFuncSetAttribute(recon_stream_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)r3_launch_smem);
  if (e != cudaSuccess) return e;
  H(0, "recon_stream");
  recon_stream_kernel<<<(unsigned)std::min<int64_t>(g->n_tiles, g->num_sms), R3T, r3_launch_smem, s>>>(r);
  H(1, "recon_stream");
  return cudaGetLastError();
}

// Core layout of this path: the canonical order with the last two modes
// swapped (..., j_b, j_a).
cudaError_t tc_core_to_canonical(const TcPlan& p, const float* dev, int comps, float* host_out) {
  const TcImpl* g = impl_of(p);
  std::vector<float> tmp((size_t)p.ncore * comps);
  cudaError_t e = cudaMemcpy(tmp.data(), dev, sizeof(float) * tmp.size(), cudaMemcpyDeviceToHost);
  if (e != cudaSuccess) return e;
  const int64_t lead = p.ncore / g->blk;
  for (int64_t l = 0; l < lead; ++l)
    for (int jb = 0; jb < g->rb; ++jb)
      for (int ja = 0; ja < g->ra; ++ja)
        for (int c = 0; c < comps; ++c)
          host_out[((l * g->ra + ja) * g->rb + jb) * comps + c] = tmp[((l * g->rb + jb) * g->ra + ja) * comps + c];
  return cudaSuccess;
}

cudaError_t tc_core_from_canonical(const TcPlan& p, const float* host_in, int comps, float* dev) {
  const TcImpl* g = impl_of(p);
  std::vector<float> tmp((size_t)p.ncore * comps);
  const int64_t lead = p.ncore / g->blk;
  for (int64_t l = 0; l < lead; ++l)
    for (int jb = 0; jb < g->rb; ++jb)
      for (int ja = 0; ja < g->ra; ++ja)
        for (int c = 0; c < comps; ++c)
          tmp[((l * g->rb + jb) * g->ra + ja) * comps + c] = host_in[((l * g->ra + ja) * g->rb + jb) * comps + c];
  return cudaMemcpy(dev, tmp.data(), sizeof(float) * tmp.size(), cudaMemcpyHostToDevice);
}

}  // namespace tgd
