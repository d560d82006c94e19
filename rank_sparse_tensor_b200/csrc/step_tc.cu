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
//     memory; on Omega's entries gather g_s (stored in Omega order) and zero
//     the entry (residual); the residual rows go to TMEM as GEMM1's A;
//     GEMM1  P = X conj(U_b)        M = 128 rows (i_a), K = 2 I_b, N = 2 r_b
//     GEMM2  Y = (U_a^H P)^T        M = 128 rows (slab, j_b), K = 2 I_a, N = 2 r_a
//     over groups of slabs; Y (bf16) is 1/16 of G for the default shapes.
//  sparse_adam  S~ = lambda Adam(g_s) with FP32 moments, in place over g_s
//     (fp16, the precision S~ is kept in for the reconstruction).
//  mode_gemm    the remaining modes n < a, contracted on Y in place of each
//     other: rows = 128 consecutive inner positions, K = 2 I_n (or 2 r_n),
//     N = 2 r_n (or 2 I_n); the last projection writes the core C in fp32.
//  core_adam    C~ = Adam(C) with FP32 moments, written as bf16.
//  recon_stream (one pass over W) per tile: bulk-copy W and Y';
//     GEMM1  P' = U_a Y'^T          M = 128 rows (slab, i_a), K = 2 r_a per slab
//                                    (block-diagonal over the tile's slabs), N = 2 r_b
//     GEMM2  Delta = P' U_b^T       M = 128 rows, K = 2 r_b, N = 2 I_b
//     (both A operands in TMEM); epilogue: Delta += lambda S~ on Omega,
//     W <- W (1 - lr wd) - lr Delta rounded once, bulk-copy W back.
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
constexpr uint64_t WAIT_NS = 2000000000ull;  // 2 s per wait

// ----------------------------------------------------------- projection
// Bounded wait for one thread. Gives up when another role has aborted or
// after WAIT_NS, setting the CTA's abort flag and the device error word.
__device__ __forceinline__ bool wait1(uint64_t* bar, uint32_t parity, volatile int* abort, int* err,
                                      uint64_t limit_ns = WAIT_NS) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = global_ns();
  // sleep in the barrier (no issue slots) until the phase completes
  while (!mbar_try_wait_sleep(bar, parity, 100000u)) {
    if (*abort) return false;
    if (global_ns() - t0 > limit_ns) {
      *abort = 1;
      atomicOr(err, DEV_ERR_TIMEOUT);
      return false;
    }
  }
  return true;
}
// The same for a whole warp: lane 0 polls, the warp re-converges after.
__device__ __forceinline__ bool waitw(uint64_t* bar, uint32_t parity, volatile int* abort, int* err,
                                      uint64_t limit_ns = WAIT_NS) {
  int ok = 1;
  if ((threadIdx.x & 31) == 0) ok = wait1(bar, parity, abort, err, limit_ns) ? 1 : 0;
  ok = __shfl_sync(0xffffffffu, ok, 0);
  __syncwarp();
  return ok != 0;
}
__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}
__device__ __forceinline__ void named_sync(int id, int nthreads) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}

constexpr int P1T = 512;
constexpr int PF = 4;     // Omega indices per converter thread prefetched for the next tile
constexpr int P1_NS_MAX = 4;
constexpr int P1_CONV_UNROLL = 5;  // 8-column chunks a converter loads before storing

struct P1Args {
  const uint32_t* G;
  int64_t N, n_slabs, n_tiles, n_groups, tile_elems;
  int Ia, Ib, ra, rb, spb, q, sg, log2Ia;
  int K1, N1, K2, N2;
  uint32_t lbo_a2;  // GEMM2's A: 64 or 128 physical rows (see geometry)
  uint32_t d1_col[2], d2_col[2], a1_col[2];  // TMEM columns
  const int64_t* tile_off;
  const uint16_t* loc;
  uint32_t* gs;  // out: g_s = G[Omega] (fp16 pairs), Omega order
  const uint8_t* B1img;
  const uint8_t* B2img;
  void* Y;
  int y_f32, y_vec;  // fp32 (else bf16) Y; rows 16-byte aligned (ra % 4 == 0, or even for fp32)
  int* err;
  int nstage;  // load stages
  uint32_t stage_bytes, off_stage, off_A2, off_B1, off_B2, off_bar;
  uint64_t wait_ns;     // limit of each wait (normally WAIT_NS)
  int skip_first_copy;  // test only: CTA 0 never loads its first tile, so a wait runs out
};

// Position in this CTA's tile sequence: groups blockIdx.x, +gridDim.x, ...,
// q tiles each; advanced incrementally (no divisions).
struct TileCursor {
  int64_t g;
  int i;
  __device__ __forceinline__ int64_t tile(int q) const { return g * q + i; }
  __device__ __forceinline__ void next(int q) {
    if (++i == q) {
      i = 0;
      g += gridDim.x;
    }
  }
};

// Warp-specialised projection stream, one CTA per SM, persistent over groups
// of q tiles (a tile = 128 rows (slab, i_a) x I_b, contiguous in G):
//   warp 0   producer: bulk copies of G tiles into a ring of stages;
//   warps 4-11  converters: gather Omega's values (g_s, written out for
//            the sparse AdamW) and zero them in the staged tile (R = G - S),
//            then write the residual rows into TMEM as GEMM1's A operand
//            (tcgen05.st), two buffers;
//   warp 1   MMA issuer: GEMM1(t) = A1[t & 1] (TMEM) x B1 -> D1[t & 1];
//            per group g GEMM2 = A2[g & 1] x B2 -> D2[g & 1];
//   warps 12-15 epilogue: P(t) from D1 into the group's GEMM2 operand; Y
//            of group g from D2 once the first tile of group g + 1 is
//            drained (so the wait for GEMM2 never stalls the D1 drain).
// Roles hand off through mbarriers.
__global__ void __launch_bounds__(P1T, 1) proj_stream_kernel(const P1Args p) {
  extern __shared__ __align__(1024) uint8_t smem[];
  const uint32_t a2_bytes = (uint32_t)(p.K2 / 8) * p.lbo_a2;
  auto A2b = [&](int64_t g) { return smem + p.off_A2 + (uint32_t)(g & 1) * a2_bytes; };
  uint8_t* B1 = smem + p.off_B1;
  uint8_t* B2 = smem + p.off_B2;
  uint64_t* bars = (uint64_t*)(smem + p.off_bar);
  uint64_t* full = bars;          // [4] stage loaded (1 + tx)
  uint64_t* sempty = bars + 4;    // [4] stage consumed (256)
  uint64_t* a1full = bars + 8;    // [2] A1 written to TMEM (256)
  uint64_t* a1empty = bars + 10;  // [2] GEMM1 done reading A1 (commit)
  uint64_t* d1full = bars + 12;   // [2] (commit)
  uint64_t* d1empty = bars + 14;  // [2] (128)
  uint64_t* opnd = bars + 16;     // B1 + B2 loaded
  uint64_t* a2full = bars + 17;   // [2] (128)
  uint64_t* d2full = bars + 19;   // [2] (commit)
  uint64_t* d2empty = bars + 21;  // [2] (128)
  uint32_t* tslot = (uint32_t*)(bars + 23);
  __shared__ int s_abort_storage;
  volatile int* s_abort = &s_abort_storage;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int q = p.q, ns = p.nstage;

  const int64_t my_groups =
      p.n_groups > (int64_t)blockIdx.x ? (p.n_groups - 1 - blockIdx.x) / gridDim.x + 1 : 0;
  int64_t n_it = my_groups * q;
  if (my_groups > 0) {
    int64_t last_g = blockIdx.x + (my_groups - 1) * gridDim.x;
    int64_t last_tiles = p.n_tiles - last_g * q;
    if (last_tiles < q) n_it -= q - last_tiles;
  }
  auto stage = [&](int s) { return smem + p.off_stage + (uint32_t)s * p.stage_bytes; };

  if (tid == 0) {
    *s_abort = 0;
    for (int i = 0; i < P1_NS_MAX; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&sempty[i], 256);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&a1full[b], 256);
      mbar_init(&a1empty[b], 1);
      mbar_init(&d1full[b], 1);
      mbar_init(&d1empty[b], 128);
    }
    mbar_init(opnd, 1);
    for (int b = 0; b < 2; ++b) {
      mbar_init(&a2full[b], 128);
      mbar_init(&d2full[b], 1);
      mbar_init(&d2empty[b], 128);
    }
    fence_mbar_init();
  }
  {
    for (uint32_t i = tid; i < 2 * a2_bytes / 16; i += P1T) ((uint4*)(smem + p.off_A2))[i] = make_uint4(0, 0, 0, 0);
    fence_async_smem();
  }
  __syncthreads();
  if (warp == 0) tmem_alloc(tslot, 512);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tslot;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      uint32_t b1 = (uint32_t)(p.N1 * p.K1 * 2), b2 = (uint32_t)(p.N2 * p.K2 * 2);
      mbar_expect_tx(opnd, b1 + b2);
      bulk_g2s(B1, p.B1img, b1, opnd);
      bulk_g2s(B2, p.B2img, b2, opnd);
      TileCursor c{(int64_t)blockIdx.x, 0};
      int s = 0;
      uint32_t ph = 0;
      int64_t issued = 0;
      const bool skip0 = p.skip_first_copy && blockIdx.x == 0;
      for (int64_t it = 0; it < n_it; ++it) {
        if (!wait1(&sempty[s], ph ^ 1u, s_abort, p.err, p.wait_ns)) break;
        const int64_t t = c.tile(q);
        const int64_t rem = p.N - t * p.tile_elems;
        const uint32_t nb = (uint32_t)((rem < p.tile_elems ? rem : p.tile_elems) * 4);
        if (!(skip0 && it == 0)) {
          mbar_expect_tx(&full[s], nb);
          bulk_g2s(stage(s), p.G + t * p.tile_elems, nb, &full[s]);
        }
        ++issued;
        c.next(q);
        if (++s == ns) {
          s = 0;
          ph ^= 1u;
        }
      }
      // wait (bounded) for the operand copies and for tile copies still in
      // flight before the CTA exits: the last copy into each stage (earlier
      // phases of a stage's barrier have completed before it was reused)
      mbar_wait(opnd, 0, WAIT_NS / 4);
      for (int64_t it = issued > ns ? issued - ns : 0; it < issued; ++it) {
        if (skip0 && it == 0) continue;
        mbar_wait(&full[it % ns], (uint32_t)((it / ns) & 1), WAIT_NS / 4);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      const uint32_t lbo_b1 = (uint32_t)(p.N1 / 8) * 128, lbo_b2 = (uint32_t)(p.N2 / 8) * 128;
      const uint32_t id1 = idesc_f16(0, 128, p.N1), id2 = idesc_f16(1, 128, p.N2);
      const uint32_t sB1 = smem_u32(B1), sB2 = smem_u32(B2);
      bool ok = wait1(opnd, 0, s_abort, p.err, p.wait_ns);
      TileCursor c{(int64_t)blockIdx.x, 0};
      int64_t it = 0, g2_issued = 0;
      bool pending = false;  // a group whose GEMM1s are all issued awaits its GEMM2
      auto gemm2 = [&]() -> bool {
        const int gb = (int)(g2_issued & 1);
        const uint32_t gpar = (uint32_t)((g2_issued >> 1) & 1);
        if (!wait1(&a2full[gb], gpar, s_abort, p.err, p.wait_ns) || !wait1(&d2empty[gb], gpar ^ 1u, s_abort, p.err, p.wait_ns))
          return false;
        tc_fence_after();
        const uint32_t sA2 = smem_u32(A2b(gb));
        for (int kk = 0; kk < p.K2 / 16; ++kk)
          mma_f16(tmem + p.d2_col[gb], sdesc(sA2 + kk * 2 * p.lbo_a2, p.lbo_a2, 128),
                  sdesc(sB2 + kk * 2 * lbo_b2, lbo_b2, 128), id2, kk > 0);
        mma_commit(&d2full[gb]);
        ++g2_issued;
        return true;
      };
      // Fixed issue order with sleeping waits: GEMM1 of every tile; a
      // group's GEMM2 right after the next group's first GEMM1 (its
      // operand is complete about when that tile's D1 buffer frees up).
      for (; ok && it < n_it; ++it) {
        const int b = (int)(it & 1);
        const uint32_t par = (uint32_t)((it >> 1) & 1);
        if (!wait1(&a1full[b], par, s_abort, p.err, p.wait_ns) || !wait1(&d1empty[b], par ^ 1u, s_abort, p.err, p.wait_ns)) {
          ok = false;
          break;
        }
        tc_fence_after();
        // A from TMEM: 16 K values = 8 columns per MMA
        for (int kk = 0; kk < p.K1 / 16; ++kk)
          mma_f16_ts(tmem + p.d1_col[b], tmem + p.a1_col[b] + kk * 8, sdesc(sB1 + kk * 2 * lbo_b1, lbo_b1, 128),
                     id1, kk > 0);
        mma_commit(&d1full[b]);
        mma_commit(&a1empty[b]);
        if (pending) {
          pending = false;
          if (!gemm2()) {
            ok = false;
            ++it;
            break;
          }
        }
        if (c.i == q - 1 || it == n_it - 1) pending = true;
        c.next(q);
      }
      if (ok && pending) ok = gemm2();
      if (*s_abort) {
        // bounded wait for the last MMAs before TMEM is released
        if (it > 0) mbar_wait(&d1full[(it - 1) & 1], (uint32_t)(((it - 1) >> 1) & 1), WAIT_NS / 4);
        if (g2_issued > 0)
          mbar_wait(&d2full[(g2_issued - 1) & 1], (uint32_t)(((g2_issued - 1) >> 1) & 1), WAIT_NS / 4);
      }
    }
  } else if (warp >= 4 && warp < 12) {
    // ------------------------------------------------------------ converters
    const int ct = tid - 128;  // 0..255
    const int row = ct & 127, half = ct >> 7;
    const int sl_row = row >> p.log2Ia;
    const uint32_t lane_base = (uint32_t)((warp & 3) * 32) << 16;
    const int Ib = p.Ib;
    // GEMM1's A row in TMEM: K1 / 2 columns (one complex fp16 pair each) in
    // chunks of 8; the two halves of the converters take alternate ranges
    const int nch = p.K1 / 16, nch0 = (nch + 1) / 2;
    const int ch_lo = half ? nch0 : 0, ch_hi = half ? nch : nch0;
    int64_t cur_e0 = 0, cur_e1 = 0, nx_e0 = 0, nx_e1 = 0, nn_e0 = 0, nn_e1 = 0;
    uint32_t pf_loc[PF];
    auto load_entries = [&](int64_t e0, int64_t e1) {
#pragma unroll
      for (int j = 0; j < PF; ++j) {
        const int64_t e = e0 + ct + 256 * j;
        if (e >= e1) break;
        pf_loc[j] = p.loc[e];
      }
    };
    TileCursor cur{(int64_t)blockIdx.x, 0}, ahead{(int64_t)blockIdx.x, 0};
    if (n_it > 0) {
      int64_t t0 = cur.tile(q);
      cur_e0 = p.tile_off[t0];
      cur_e1 = p.tile_off[t0 + 1];
      ahead.next(q);
      if (n_it > 1) {
        int64_t t1 = ahead.tile(q);
        nx_e0 = p.tile_off[t1];
        nx_e1 = p.tile_off[t1 + 1];
      }
      ahead.next(q);
      load_entries(cur_e0, cur_e1);
    }
    int s = 0;
    uint32_t ph = 0;
    // After an abort a warp still takes every named barrier of the remaining
    // tiles (and no other work), so no converter warp waits there forever.
    int64_t dead_from = n_it;
    for (int64_t it = 0; it < n_it; ++it) {
      if (it >= dead_from) {
        named_sync(1, 256);
        continue;
      }
      const int64_t t = cur.tile(q);
      const int b = (int)(it & 1);
      const uint32_t par = (uint32_t)((it >> 1) & 1);
      if (it + 2 < n_it) {
        const int64_t t2 = ahead.tile(q);
        nn_e0 = p.tile_off[t2];
        nn_e1 = p.tile_off[t2 + 1];
      }
      if (!waitw(&full[s], ph, s_abort, p.err, p.wait_ns)) {
        named_sync(1, 256);
        dead_from = it + 1;
        continue;
      }
      uint32_t* sw = (uint32_t*)stage(s);
      // gather g_s (coalesced stores, Omega order) and zero it in the tile
      // (R = G - S)
      const int cnt = (int)(cur_e1 - cur_e0);
      {
        uint32_t u[PF];
#pragma unroll
        for (int j = 0; j < PF; ++j)
          if (ct + 256 * j < cnt) u[j] = sw[pf_loc[j]];
#pragma unroll
        for (int j = 0; j < PF; ++j) {
          const int jj = ct + 256 * j;
          if (jj < cnt) {
            sw[pf_loc[j]] = 0u;
            p.gs[cur_e0 + jj] = u[j];
          }
        }
      }
      for (int jj = 256 * PF + ct; jj < cnt; jj += 256) {
        const int64_t e = cur_e0 + jj;
        const uint32_t l = p.loc[e];
        p.gs[e] = sw[l];
        sw[l] = 0u;
      }
      if (it + 1 < n_it) load_entries(nx_e0, nx_e1);
      named_sync(1, 256);  // every zeroed entry is in place before conversion
      if (!waitw(&a1empty[b], par ^ 1u, s_abort, p.err, p.wait_ns)) {
        dead_from = it + 1;
        continue;
      }
      tc_fence_after();
      // residual row -> TMEM (K = (i_b, re/im): one complex pair per column)
      const bool valid = t * p.spb + sl_row < p.n_slabs;
      const uint32_t* src = sw + row * Ib;
      const uint32_t taddr = tmem + lane_base + p.a1_col[b];
      // all loads of up to P1_CONV_UNROLL chunks before their stores
      for (int ch0 = ch_lo; ch0 < ch_hi; ch0 += P1_CONV_UNROLL) {
        const int nc = ch_hi - ch0 < P1_CONV_UNROLL ? ch_hi - ch0 : P1_CONV_UNROLL;
        uint32_t v[8 * P1_CONV_UNROLL];
#pragma unroll
        for (int i = 0; i < P1_CONV_UNROLL; ++i) {
#pragma unroll
          for (int u = 0; u < 8; ++u) {
            const int cc = 8 * (ch0 + i) + u;
            v[8 * i + u] = i < nc && valid && cc < Ib ? src[cc] : 0u;
          }
        }
#pragma unroll
        for (int i = 0; i < P1_CONV_UNROLL; ++i)
          if (i < nc) tmem_st8(taddr + 8 * (ch0 + i), v + 8 * i);  // nc is warp-uniform
      }
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(&a1full[b]);
      mbar_arrive(&sempty[s]);
      // move to the next tile's ranges at the end of the tile, well after
      // the loads of the one two ahead were issued
      cur_e0 = nx_e0;
      cur_e1 = nx_e1;
      nx_e0 = nn_e0;
      nx_e1 = nn_e1;
      cur.next(q);
      ahead.next(q);
      if (++s == ns) {
        s = 0;
        ph ^= 1u;
      }
    }
  } else if (warp >= 12) {
    // ------------------------------------------------------------ epilogue
    const int row = tid & 127;
    const uint32_t lane_base = (uint32_t)((warp & 3) * 32) << 16;
    const int sl_row = row >> p.log2Ia, ia_row = row & (p.Ia - 1);
    TileCursor c{(int64_t)blockIdx.x, 0};
    int64_t g_done = 0;        // groups whose Y has been written
    int64_t g_pending = -1;    // group (index in this CTA) whose Y is ready to read
    int64_t g_pending_abs = 0; // its group number
    // Y of one group from D2[gi & 1] (row = (slab in group, j_b)), j_a contiguous
    auto write_y = [&](int64_t gi, int64_t gabs) -> bool {
      const int gb = (int)(gi & 1);
      if (!waitw(&d2full[gb], (uint32_t)((gi >> 1) & 1), s_abort, p.err, p.wait_ns)) return false;
      tc_fence_after();
      const int sb = row / p.rb, jb = row - sb * p.rb;
      const int64_t slab = gabs * p.sg + sb;
      const bool yvalid = row < p.sg * p.rb && slab < p.n_slabs;
      const int64_t ybase = (slab * p.rb + jb) * p.ra;
      for (int c0 = 0; c0 < p.N2; c0 += 32) {
        float v[32];
        if (c0 + 32 <= p.N2)
          tmem_ld32(tmem + p.d2_col[gb] + lane_base + c0, v);
        else
          tmem_ld16(tmem + p.d2_col[gb] + lane_base + c0, v);
        // a thread owns one Y row: 16-byte stores where the row allows
        // them (one warp store touches 32 rows, so wider is cheaper)
        if (yvalid && p.y_vec && c0 / 2 + 16 <= p.ra) {
          if (p.y_f32) {
            float4* y4 = (float4*)((float2*)p.Y + ybase + c0 / 2);
#pragma unroll
            for (int u = 0; u < 8; ++u) y4[u] = make_float4(v[4 * u], v[4 * u + 1], v[4 * u + 2], v[4 * u + 3]);
          } else {
            uint4* y4 = (uint4*)((uint32_t*)p.Y + ybase + c0 / 2);
#pragma unroll
            for (int u = 0; u < 4; ++u)
              y4[u] = make_uint4(f2_to_bf2(v[8 * u], v[8 * u + 1]), f2_to_bf2(v[8 * u + 2], v[8 * u + 3]),
                                 f2_to_bf2(v[8 * u + 4], v[8 * u + 5]), f2_to_bf2(v[8 * u + 6], v[8 * u + 7]));
          }
        } else if (yvalid) {
#pragma unroll
          for (int u = 0; u < 16; ++u) {
            int ja = c0 / 2 + u;
            if (ja < p.ra) {
              if (p.y_f32)
                ((float2*)p.Y)[ybase + ja] = make_float2(v[2 * u], v[2 * u + 1]);
              else
                ((uint32_t*)p.Y)[ybase + ja] = f2_to_bf2(v[2 * u], v[2 * u + 1]);
            }
          }
        }
      }
      tc_fence_before();
      mbar_arrive(&d2empty[gb]);
      return true;
    };
    bool ok = true;
    int64_t gi = 0;  // index of the current group in this CTA
    for (int64_t it = 0; it < n_it; ++it) {
      const int b = (int)(it & 1);
      const uint32_t par = (uint32_t)((it >> 1) & 1);
      const int64_t t = c.tile(q);
      if (!waitw(&d1full[b], par, s_abort, p.err, p.wait_ns)) {
        ok = false;
        break;
      }
      tc_fence_after();
      // P (fp32, TMEM) -> GEMM2's A operand (bf16), rows (slab in group,
      // j_b), K = (i_a, re/im)
      uint8_t* A2 = A2b(gi);
      const bool valid = t * p.spb + sl_row < p.n_slabs;
      const int m2base = (c.i * p.spb + sl_row) * p.rb;
      for (int c0 = 0; c0 < p.N1; c0 += 32) {
        float v[32];
        if (c0 + 32 <= p.N1)
          tmem_ld32(tmem + p.d1_col[b] + lane_base + c0, v);
        else
          tmem_ld16(tmem + p.d1_col[b] + lane_base + c0, v);
        const int jb0 = m2base + c0 / 2;
        if (valid && (jb0 & 7) == 0 && c0 / 2 + 16 <= p.rb) {
          // 16 whole rows from an 8-row boundary: offsets from one base
          uint8_t* dst = A2 + kmaj_off((uint32_t)jb0, (uint32_t)(2 * ia_row), p.lbo_a2);
#pragma unroll
          for (int u = 0; u < 16; ++u)
            *(uint32_t*)(dst + (u & 7) * 16 + (u >> 3) * 128) = f2_to_bf2(v[2 * u], v[2 * u + 1]);
        } else if (valid) {
#pragma unroll
          for (int u = 0; u < 16; ++u) {
            int jb = c0 / 2 + u;
            if (jb < p.rb) {
              uint32_t off = kmaj_off((uint32_t)(m2base + jb), (uint32_t)(2 * ia_row), p.lbo_a2);
              *(uint32_t*)(A2 + off) = f2_to_bf2(v[2 * u], v[2 * u + 1]);
            }
          }
        }
      }
      tc_fence_before();
      mbar_arrive(&d1empty[b]);
      // the previous group's Y, now that this tile's D1 is drained
      if (g_pending >= 0) {
        if (!write_y(g_pending, g_pending_abs)) {
          ok = false;
          break;
        }
        g_pending = -1;
        ++g_done;
      }
      const bool last = c.i == q - 1 || it == n_it - 1;
      if (last) {
        fence_async_smem();
        mbar_arrive(&a2full[gi & 1]);
        g_pending = gi;
        g_pending_abs = c.g;
        ++gi;
      }
      c.next(q);
    }
    if (ok && g_pending >= 0) write_y(g_pending, g_pending_abs);
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
// without a transpose in memory. K advances in chunks of 32 complex values:
// the next chunk's values are loaded into registers while the current
// chunk's MMAs run, and the operand image chunk arrives by bulk copy.
__global__ void __launch_bounds__(MGT) mode_gemm_kernel(const MGArgs p) {
  extern __shared__ __align__(1024) uint8_t smem[];
  const uint32_t a_bytes = 8 * LBO_M128;               // 128 rows x 64 K
  const uint32_t b_bytes = (uint32_t)p.NT * 64 * 2;
  uint8_t* As[2] = {smem, smem + a_bytes};
  uint8_t* Bs[2] = {smem + 2 * a_bytes, smem + 2 * a_bytes + b_bytes};
  uint64_t* bars = (uint64_t*)(smem + 2 * a_bytes + 2 * b_bytes);  // [0,1] MMA done, [2,3] B landed
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
    for (int i = 0; i < 4; ++i) mbar_init(&bars[i], 1);
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
  uint32_t issued[2] = {0, 0}, waited[2] = {0, 0}, bloaded[2] = {0, 0};
  // One thread waits (bounded), the rest sleep in the barrier.
  auto wait_all = [&](uint64_t* bar, uint32_t parity) -> bool {
    if (tid == 0 && !mbar_wait(bar, parity, WAIT_NS)) {
      atomicOr(p.err, DEV_ERR_TIMEOUT);
      s_abort = 1;
    }
    __syncthreads();
    return s_abort == 0;
  };
  // two register sets: chunk kc + 2 is in flight while chunk kc is stored
  // and its MMAs run
  uint32_t va[32], vb[32];
  auto load_x = [&](uint32_t(&v)[32], int kc) {
#pragma unroll
    for (int i = 0; i < 32; ++i) {
      const int64_t k = (int64_t)kc * 32 + i;
      v[i] = (valid && k < p.K) ? __ldg(xrow + k * p.in_bs) : 0u;
    }
  };
  // one K chunk: buffers free, operand image by bulk copy, X from registers
  // (then the registers are refilled with chunk kc + 2), MMAs
  auto chunk = [&](uint32_t(&v)[32], int kc) -> bool {
    const int s = kc & 1;
    if (kc >= 2) {
      const bool ok = wait_all(&bars[s], waited[s] & 1u);
      waited[s]++;
      if (!ok) return false;
      tc_fence_after();
    }
    if (tid == 0) {
      mbar_expect_tx(&bars[2 + s], b_bytes);
      bulk_g2s(Bs[s], img + (int64_t)kc * b_bytes, b_bytes, &bars[2 + s]);
      bloaded[s]++;
    }
#pragma unroll
    for (int q = 0; q < 8; ++q)
      *(uint4*)(As[s] + q * LBO_M128 + tid * 16) = make_uint4(v[4 * q], v[4 * q + 1], v[4 * q + 2], v[4 * q + 3]);
    if (kc + 2 < p.nkc) load_x(v, kc + 2);
    // the operand image has landed (checked before the barrier, so that
    // every thread reads the same abort flag after it)
    if (tid == 0 && !mbar_wait(&bars[2 + s], (bloaded[s] - 1) & 1u, WAIT_NS)) {
      atomicOr(p.err, DEV_ERR_TIMEOUT);
      s_abort = 1;
    }
    fence_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (s_abort) return false;
    if (tid == 0) {
      {
        const uint32_t sa = smem_u32(As[s]), sb = smem_u32(Bs[s]);
        for (int kk = 0; kk < 4; ++kk)
          mma_f16(dt, sdesc(sa + kk * 2 * LBO_M128, LBO_M128, 128), sdesc(sb + kk * 2 * lbo_b, lbo_b, 128),
                  idesc, (kc > 0 || kk > 0) ? 1u : 0u);
        mma_commit(&bars[s]);
        issued[s]++;
      }
    }
    return true;
  };
  load_x(va, 0);
  if (p.nkc > 1) load_x(vb, 1);
  for (int kc = 0; kc < p.nkc; kc += 2) {
    if (!chunk(va, kc)) break;
    if (kc + 1 < p.nkc && !chunk(vb, kc + 1)) break;
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
      float y[16];
      tmem_ld16(dt + lane_base + c0, y);
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        int64_t j = j0 + c0 / 2 + u;
        if (valid && j < p.J) {
          int64_t o = (a * p.J + j) * p.out_bs + b;
          if (p.y_f32)
            ((float2*)p.Y)[o] = make_float2(y[2 * u], y[2 * u + 1]);
          else
            ((uint32_t*)p.Y)[o] = f2_to_bf2(y[2 * u], y[2 * u + 1]);
        }
      }
    }
  } else if (tid == 0) {
    // bounded waits for the copies and MMAs still in flight
    for (int s = 0; s < 2; ++s) {
      if (issued[s] > waited[s]) mbar_wait(&bars[s], (issued[s] - 1) & 1u, WAIT_NS / 4);
      if (bloaded[s] > 0) mbar_wait(&bars[2 + s], (bloaded[s] - 1) & 1u, WAIT_NS / 4);
    }
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

// S~ = lambda * Adam(g_s), in place of the gathered g_s (fp16 pairs in and
// out; fp32 moments: m complex, v one or two floats). A plain stream over
// the k entries in Omega order.
__global__ void sparse_adam_tc_kernel(uint32_t* gs, int64_t k, float* m, float* v, AdamConst a) {
  const int vc = a.cmode == 1 ? 2 : 1;
  for (int64_t j = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; j < k;
       j += (int64_t)gridDim.x * blockDim.x) {
    const float2 m2 = ((const float2*)m)[j];
    const float2 v2 = vc == 2 ? ((const float2*)v)[j] : make_float2(v[j], 0.f);
    float mm[2] = {m2.x, m2.y}, vv[2] = {v2.x, v2.y};
    const float2 u = adam_elem(h2_to_f2(gs[j]), mm, vv, a);
    ((float2*)m)[j] = make_float2(mm[0], mm[1]);
    if (vc == 2)
      ((float2*)v)[j] = make_float2(vv[0], vv[1]);
    else
      v[j] = vv[0];
    gs[j] = f2_to_h2(u);
  }
}

// ------------------------------------------------------- reconstruction
__device__ __forceinline__ float2 wload(const __half2* p) { return __half22float2(*p); }
__device__ __forceinline__ void wstore(__half2* p, float x, float y) { *p = __floats2half2_rn(x, y); }
__device__ __forceinline__ float2 wload(const float2* p) { return *p; }
__device__ __forceinline__ void wstore(float2* p, float x, float y) { *p = make_float2(x, y); }
// v + d for an fp16 pair d by mixed-precision adds (no separate conversion;
// the same value as converting d and adding in fp32)
__device__ __forceinline__ float2 add_f2_h2(float2 v, uint32_t d) {
  float2 x;
  asm("{\n\t.reg .b16 lo, hi;\n\tmov.b32 {lo, hi}, %2;\n\t"
      "add.rn.f32.f16 %0, lo, %3;\n\tadd.rn.f32.f16 %1, hi, %4;\n\t}"
      : "=f"(x.x), "=f"(x.y)
      : "r"(d), "f"(v.x), "f"(v.y));
  return x;
}
// a * b + c on a pair (packed fp32: two fmaf_rn in one instruction)
__device__ __forceinline__ float2 ffma2(float2 a, float2 b, float2 c) {
  float2 d;
  asm("{\n\t.reg .b64 ra, rb, rc, rd;\n\tmov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\t"
      "mov.b64 rc, {%6, %7};\n\tfma.rn.f32x2 rd, ra, rb, rc;\n\tmov.b64 {%0, %1}, rd;\n\t}"
      : "=f"(d.x), "=f"(d.y)
      : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y), "f"(c.x), "f"(c.y));
  return d;
}
__device__ __forceinline__ float2 fmul2(float2 a, float2 b) {
  float2 d;
  asm("{\n\t.reg .b64 ra, rb, rd;\n\tmov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\t"
      "mul.rn.f32x2 rd, ra, rb;\n\tmov.b64 {%0, %1}, rd;\n\t}"
      : "=f"(d.x), "=f"(d.y)
      : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
  return d;
}

constexpr int R3T = 512;
constexpr int PREP_ITEMS = 2;  // B1 items per prep thread whose addressing is precomputed
constexpr int R3_NS_MAX = 6;  // W stages
constexpr int EPF = 4;  // Omega entries per epilogue thread prefetched for the next tile

struct R3Args {
  const uint32_t* Yp;
  int64_t yp_bs;  // u32 (complex) per slab in Y'
  void* W;
  int w_c64;
  int64_t N, n_slabs, n_tiles, tile_elems;
  int64_t tile0, tiles;  // this launch: tiles [tile0, tile0 + tiles)
  int Ia, Ib, ra, rb, spb, log2Ia;
  int K1, N1, K2, N2;
  uint32_t d1_col[2], d2_col[2], a1_col, a2_col[2];  // TMEM columns
  const int64_t* tile_off;
  const uint16_t* loc;
  const uint32_t* sp_upd;
  const uint8_t* A1img;
  const uint8_t* B2img;
  float decay, lr;
  int* err;
  int nstage;
  uint32_t lbo_b1;  // GEMM1's B: K-adjacent core matrices N1 / 8 * 128 + 16 B apart
  uint32_t w_tile_bytes, y_tile_bytes;
  uint32_t off_w, off_y, off_B1, off_B2, off_ds, off_bar;
};

// Warp-specialised reconstruction stream, one CTA per SM, persistent over
// tiles (t = blockIdx.x, +gridDim.x, ...):
//   warp 0   producer: bulk copies W(t), Y'(t) into a ring of stages, and
//            bulk-stores each W tile once its epilogue is done;
//   warp 1   MMA issuer: GEMM1(t) = A1 x B1(t) -> D1[t&1], GEMM2(t) =
//            A2(t) x B2 -> D2[t&1]; both A operands live in TMEM (A1 the
//            constant U_a image, written once; A2 = P'(t), two buffers), so
//            shared memory holds up to six W stages;
//   warps 4-7   prep: B1(t+1) from Y'(t+1), the tile's Omega list and
//            per-row start table, then P'(t) from D1 into A2[t&1];
//   warps 8-15  epilogue: Delta(t) from D2 + lambda S~ on Omega, AdamW on
//            the staged W tile (column halves per warpgroup).
// Roles hand off through mbarriers; operands, lists and accumulators are
// double-buffered, so consecutive tiles overlap.
// UNIT_DECAY: lr * wd == 0, so W (1 - lr wd) is W itself (no multiply).
template <class WT, bool UNIT_DECAY>
__global__ void __launch_bounds__(R3T, 1) recon_stream_kernel(const R3Args p) {
  extern __shared__ __align__(1024) uint8_t smem[];
  uint8_t* B2 = smem + p.off_B2;
  uint64_t* bars = (uint64_t*)(smem + p.off_bar);
  // barrier map
  uint64_t* full = bars;           // [6] stage loaded
  uint64_t* wdone = bars + 6;      // [6] W tile updated (256 arrivals)
  uint64_t* opnd = bars + 12;      // B2 loaded
  uint64_t* b1full = bars + 13;    // [2] (128)
  uint64_t* b1empty = bars + 15;   // [2] (commit)
  uint64_t* d1full = bars + 17;    // [2] (commit)
  uint64_t* d1empty = bars + 19;   // [2] (128)
  uint64_t* a2full = bars + 21;    // [2] (128)
  uint64_t* a2empty = bars + 23;   // [2] (commit)
  uint64_t* d2full = bars + 25;    // [2] (commit)
  uint64_t* d2empty = bars + 27;   // [2] (256)
  uint32_t* tslot = (uint32_t*)(bars + 29);
  __shared__ int s_abort_storage;
  volatile int* s_abort = &s_abort_storage;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int64_t n_it = p.tiles > (int64_t)blockIdx.x ? (p.tiles - 1 - blockIdx.x) / gridDim.x + 1 : 0;
  const int64_t tb = p.tile0 + blockIdx.x;  // this CTA's first tile
  const int64_t G = gridDim.x;
  const int ns = p.nstage;
  auto wst = [&](int s) { return smem + p.off_w + (uint32_t)s * p.w_tile_bytes; };
  auto yst = [&](int s) { return smem + p.off_y + (uint32_t)s * p.y_tile_bytes; };
  auto B1b = [&](int b) { return smem + p.off_B1 + (uint32_t)b * (uint32_t)(p.K1 / 8) * p.lbo_b1; };
  const int wb = (int)sizeof(WT);
  auto tile_wbytes = [&](int64_t t) -> uint32_t {
    int64_t rem = p.N - t * p.tile_elems;
    return (uint32_t)((rem < p.tile_elems ? rem : p.tile_elems) * wb);
  };
  auto tile_ybytes = [&](int64_t t) -> uint32_t {
    int64_t rem = p.n_slabs - t * p.spb;
    return (uint32_t)((rem < p.spb ? rem : p.spb) * p.yp_bs * 4);
  };

  if (tid == 0) {
    *s_abort = 0;
    for (int i = 0; i < R3_NS_MAX; ++i) mbar_init(&full[i], 1);
    for (int i = 0; i < R3_NS_MAX; ++i) mbar_init(&wdone[i], 256);
    mbar_init(opnd, 1);
    for (int b = 0; b < 2; ++b) {
      mbar_init(&b1full[b], 128);
      mbar_init(&b1empty[b], 1);
      mbar_init(&d1full[b], 1);
      mbar_init(&d1empty[b], 128);
      mbar_init(&a2full[b], 128);
      mbar_init(&a2empty[b], 1);
      mbar_init(&d2full[b], 1);
      mbar_init(&d2empty[b], 256);
    }
    fence_mbar_init();
  }
  {
    const uint32_t b1b = (uint32_t)(2 * (p.K1 / 8)) * p.lbo_b1;
    for (uint32_t i = tid; i < b1b / 16; i += R3T) ((uint4*)(smem + p.off_B1))[i] = make_uint4(0, 0, 0, 0);
  }
  __syncthreads();
  if (warp == 0) tmem_alloc(tslot, 512);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tslot;
  if (warp >= 4 && warp < 8) {
    // GEMM1's A (the U_a image, K-major in global memory) -> TMEM, row per lane
    const int row = tid - 128;
    const uint32_t taddr = tmem + ((uint32_t)((warp & 3) * 32) << 16) + p.a1_col;
    for (int kc = 0; kc < p.K1 / 8; kc += 2) {
      const uint4 x = __ldg((const uint4*)(p.A1img + kmaj_off((uint32_t)row, (uint32_t)(8 * kc), LBO_M128)));
      const uint4 y = __ldg((const uint4*)(p.A1img + kmaj_off((uint32_t)row, (uint32_t)(8 * kc + 8), LBO_M128)));
      const uint32_t w[8] = {x.x, x.y, x.z, x.w, y.x, y.y, y.z, y.w};
      tmem_st8(taddr + 4 * kc, w);
    }
    tmem_wait_st();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      const uint32_t b2b = (uint32_t)(p.N2 * p.K2 * 2);
      mbar_expect_tx(opnd, b2b);
      bulk_g2s(B2, p.B2img, b2b, opnd);
      auto load = [&](int64_t it) {
        const int s = (int)(it % ns);
        const int64_t t = tb + it * G;
        const uint32_t nw = tile_wbytes(t), ny = tile_ybytes(t);
        mbar_expect_tx(&full[s], nw + ny);
        bulk_g2s(wst(s), (const uint8_t*)p.W + t * p.tile_elems * wb, nw, &full[s]);
        bulk_g2s(yst(s), p.Yp + t * p.spb * p.yp_bs, ny, &full[s]);
      };
      int64_t loaded = 0;
      for (; loaded < ns && loaded < n_it; ++loaded) load(loaded);
      int s = 0;
      uint32_t ph = 0;
      for (int64_t it = 0; it < n_it; ++it) {
        if (!wait1(&wdone[s], ph, s_abort, p.err)) break;
        const int64_t t = tb + it * G;
        bulk_s2g((uint8_t*)p.W + t * p.tile_elems * wb, wst(s), tile_wbytes(t));
        bulk_commit();
        if (loaded < n_it) {
          bulk_wait_read0();  // the stage's last store has been read out
          load(loaded++);
        }
        if (++s == ns) {
          s = 0;
          ph ^= 1u;
        }
      }
      // wait (bounded) for loads still in flight before the CTA exits: the
      // last load into each stage (earlier phases completed before reuse)
      for (int64_t it = loaded > ns ? loaded - ns : 0; it < loaded; ++it)
        mbar_wait(&full[it % ns], (uint32_t)((it / ns) & 1), WAIT_NS / 4);
      bulk_wait_all0();
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      const uint32_t lbo_b1 = p.lbo_b1, lbo_b2 = (uint32_t)(p.N2 / 8) * 128;
      const uint32_t id1 = idesc_f16(1, 128, p.N1), id2 = idesc_f16(1, 128, p.N2);
      const uint32_t sB2 = smem_u32(B2);
      bool ok = wait1(opnd, 0, s_abort, p.err);
      auto gemm1 = [&](int64_t it) -> bool {
        const int b = (int)(it & 1);
        const uint32_t par = (uint32_t)((it >> 1) & 1);
        if (!wait1(&b1full[b], par, s_abort, p.err)) return false;
        if (!wait1(&d1empty[b], par ^ 1u, s_abort, p.err)) return false;
        tc_fence_after();
        const uint32_t sB1 = smem_u32(B1b(b));
        for (int kk = 0; kk < p.K1 / 16; ++kk)
          mma_f16_ts(tmem + p.d1_col[b], tmem + p.a1_col + kk * 8, sdesc(sB1 + kk * 2 * lbo_b1, lbo_b1, 128),
                     id1, kk > 0);
        mma_commit(&d1full[b]);
        mma_commit(&b1empty[b]);
        return true;
      };
      int64_t g1_done = 0, g2_done = 0;
      if (ok && n_it > 0) {
        ok = gemm1(0);
        if (ok) g1_done = 1;
      }
      for (int64_t it = 0; ok && it < n_it; ++it) {
        if (it + 1 < n_it) {
          if (!gemm1(it + 1)) break;
          g1_done = it + 2;
        }
        const int b = (int)(it & 1);
        const uint32_t par = (uint32_t)((it >> 1) & 1);
        if (!wait1(&a2full[b], par, s_abort, p.err)) break;
        if (!wait1(&d2empty[b], par ^ 1u, s_abort, p.err)) break;
        tc_fence_after();
        for (int kk = 0; kk < p.K2 / 16; ++kk)
          mma_f16_ts(tmem + p.d2_col[b], tmem + p.a2_col[b] + kk * 8, sdesc(sB2 + kk * 2 * lbo_b2, lbo_b2, 128),
                     id2, kk > 0);
        mma_commit(&d2full[b]);
        mma_commit(&a2empty[b]);
        g2_done = it + 1;
      }
      if (*s_abort) {
        // bounded wait for the last MMAs before TMEM is released
        if (g1_done > 0) mbar_wait(&d1full[(g1_done - 1) & 1], (uint32_t)(((g1_done - 1) >> 1) & 1), WAIT_NS / 4);
        if (g2_done > 0) mbar_wait(&d2full[(g2_done - 1) & 1], (uint32_t)(((g2_done - 1) >> 1) & 1), WAIT_NS / 4);
      }
    }
  } else if (warp >= 4 && warp < 8) {
    // ------------------------------------------------------------ prep
    const int row = tid - 128;  // 0..127, TMEM lane of warps 4-7
    const uint32_t lane_base = (uint32_t)((warp & 3) * 32) << 16;
    const int nkc = p.K1 / 8;  // 16-byte K chunks of a B1 row (4 complex j_a each)
    const bool vec = (p.ra & 3) == 0;  // a chunk's 4 j_a lie in one slab, 16-byte aligned
    bool ok = true;
    // Where each B1 item of this thread reads Y' in a stage and writes B1: the
    // same for every tile, so the divisions are done once (for the first
    // PREP_ITEMS items of the thread; further items, on large ranks, per tile).
    const int n_items = p.rb * nkc;
    auto item_addr = [&](int e, int (&src)[4], int (&sl)[4], uint32_t& dst) {
      const int kc = e % nkc, jb = e / nkc;
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int kp = 4 * kc + u;
        sl[u] = kp / p.ra;
        src[u] = sl[u] * (int)p.yp_bs + jb * p.ra + (kp - sl[u] * p.ra);
      }
      dst = kmaj_off((uint32_t)(2 * jb), (uint32_t)(8 * kc), p.lbo_b1);
    };
    int it_src[PREP_ITEMS][4], it_sl[PREP_ITEMS][4];
    uint32_t it_dst[PREP_ITEMS];
#pragma unroll
    for (int q = 0; q < PREP_ITEMS; ++q)
      if (row + 128 * q < n_items) item_addr(row + 128 * q, it_src[q], it_sl[q], it_dst[q]);
    auto build = [&](int64_t it) -> bool {
      const int b = (int)(it & 1), s = (int)(it % ns);
      const uint32_t par = (uint32_t)((it >> 1) & 1);
      const int64_t t = tb + it * G;
      if (!waitw(&full[s], (uint32_t)((it / ns) & 1), s_abort, p.err)) return false;
      if (!waitw(&b1empty[b], par ^ 1u, s_abort, p.err)) return false;
      // B1: rows (j_b, re/im), K = (slab, j_a, re/im), entries [[Yr, -Yi], [Yi, Yr]];
      // one item = one K chunk of rows 2 j_b and 2 j_b + 1 (two 16-byte stores)
      uint8_t* B1 = B1b(b);
      const uint32_t* ys = (const uint32_t*)yst(s);
      const int64_t vs = p.n_slabs - t * p.spb;
      const int vslabs = vs < p.spb ? (int)vs : p.spb;
      auto item = [&](const int (&src)[4], const int (&sl)[4], uint32_t dst) {
        uint32_t yv[4];
        if (vec) {
          uint4 y4 = make_uint4(0, 0, 0, 0);
          if (sl[0] < vslabs) y4 = *(const uint4*)(ys + src[0]);
          yv[0] = y4.x;
          yv[1] = y4.y;
          yv[2] = y4.z;
          yv[3] = y4.w;
        } else {
#pragma unroll
          for (int u = 0; u < 4; ++u) yv[u] = sl[u] < vslabs ? ys[src[u]] : 0u;
        }
        uint32_t lo[4], hi[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const float2 y = bf2_to_f2(yv[u]);
          lo[u] = f2_to_bf2(y.x, -y.y);
          hi[u] = f2_to_bf2(y.y, y.x);
        }
        // rows 2 j_b and 2 j_b + 1 sit in one 8-row group, 16 bytes apart
        *(uint4*)(B1 + dst) = make_uint4(lo[0], lo[1], lo[2], lo[3]);
        *(uint4*)(B1 + dst + 16) = make_uint4(hi[0], hi[1], hi[2], hi[3]);
      };
#pragma unroll
      for (int q = 0; q < PREP_ITEMS; ++q)
        if (row + 128 * q < n_items) item(it_src[q], it_sl[q], it_dst[q]);
      for (int e = row + 128 * PREP_ITEMS; e < n_items; e += 128) {
        int src[4], sl[4];
        uint32_t dst;
        item_addr(e, src, sl, dst);
        item(src, sl, dst);
      }
      fence_async_smem();
      mbar_arrive(&b1full[b]);
      return true;
    };
    if (n_it > 0) ok = build(0);
    for (int64_t it = 0; ok && it < n_it; ++it) {
      if (it + 1 < n_it && !build(it + 1)) break;
      // P'(t): D1 -> A2 (rows (slab, i_a), K = (j_b, re/im))
      const int b = (int)(it & 1);
      const uint32_t par = (uint32_t)((it >> 1) & 1);
      if (!waitw(&d1full[b], par, s_abort, p.err)) break;
      if (!waitw(&a2empty[b], par ^ 1u, s_abort, p.err)) break;
      tc_fence_after();
      // P' row (bf16 pairs) -> TMEM, the A operand of GEMM2
      for (int c0 = 0; c0 < p.N1; c0 += 16) {
        float v[16];
        tmem_ld16(tmem + p.d1_col[b] + lane_base + c0, v);
        uint32_t w[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) w[u] = f2_to_bf2(v[2 * u], v[2 * u + 1]);
        tmem_st8(tmem + p.a2_col[b] + lane_base + c0 / 2, w);
      }
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(&d1empty[b]);
      mbar_arrive(&a2full[b]);
    }
  } else if (warp >= 8) {
    // ------------------------------------------------------------ epilogue
    // lambda S~ of the tile is scattered into a zeroed tile-sized buffer
    // (fp16 pairs, the precision S~ is kept in), so the weight pass is dense
    // and branch-free: W <- W (1 - lr wd) - lr (Delta + S), one rounding.
    const int et = tid - 256;  // 0..255
    const int row = et & 127, half = et >> 7;
    const uint32_t lane_base = (uint32_t)((warp & 3) * 32) << 16;
    // column halves of Delta in chunks of 8 complex values (the first half
    // takes the larger share of whole chunks; the partial last chunk, with
    // its per-element bounds, falls to the second)
    const int nch = p.N2 / 16, nch0 = (nch + 1) / 2;
    const int c_lo = half ? nch0 : 0, c_hi = half ? nch : nch0;
    const int sl_row = row >> p.log2Ia;
    const uint32_t erow = (uint32_t)row * p.Ib;
    const float nlr = -p.lr, decay = p.decay;
    const int Ib = p.Ib;
    uint32_t* ds = (uint32_t*)(smem + p.off_ds);
    // Omega ranges two tiles ahead, entries one tile ahead (registers)
    int64_t cur_e0 = 0, cur_e1 = 0, nx_e0 = 0, nx_e1 = 0, nn_e0 = 0, nn_e1 = 0;
    uint32_t pf_loc[EPF], pf_val[EPF];
    auto load_entries = [&](int64_t e0, int64_t e1) {
#pragma unroll
      for (int j = 0; j < EPF; ++j) {
        int64_t e = e0 + et + 256 * j;
        if (e < e1) {
          pf_loc[j] = p.loc[e];
          pf_val[j] = p.sp_upd[e];
        }
      }
    };
    if (n_it > 0) {
      cur_e0 = p.tile_off[tb];
      cur_e1 = p.tile_off[tb + 1];
      if (n_it > 1) {
        nx_e0 = p.tile_off[tb + G];
        nx_e1 = p.tile_off[tb + G + 1];
      }
      load_entries(cur_e0, cur_e1);
    }
    for (uint32_t i = et; i < (uint32_t)(128 * Ib); i += 256) ds[i] = 0u;
    named_sync(2, 256);
    int s = 0;
    uint32_t sph = 0;
    // After an abort a warp still takes every named barrier of the remaining
    // tiles (and no other work), so no epilogue warp waits there forever.
    int64_t dead_from = n_it;
    for (int64_t it = 0; it < n_it; ++it) {
      if (it >= dead_from) {
        named_sync(2, 256);
        named_sync(2, 256);
        named_sync(2, 256);
        continue;
      }
      const int b = (int)(it & 1);
      const uint32_t par = (uint32_t)((it >> 1) & 1);
      const int64_t t = tb + it * G;
      if (it + 2 < n_it) {
        nn_e0 = p.tile_off[t + 2 * G];
        nn_e1 = p.tile_off[t + 2 * G + 1];
      }
      // scatter lambda S~ of this tile
#pragma unroll
      for (int j = 0; j < EPF; ++j) {
        int64_t e = cur_e0 + et + 256 * j;
        if (e < cur_e1) ds[pf_loc[j]] = pf_val[j];
      }
      for (int64_t e = cur_e0 + 256 * EPF + et; e < cur_e1; e += 256) ds[p.loc[e]] = p.sp_upd[e];
      // the next tile's entries, a whole tile ahead of their use
      uint32_t zl[EPF];
#pragma unroll
      for (int j = 0; j < EPF; ++j) zl[j] = pf_loc[j];
      if (it + 1 < n_it) load_entries(nx_e0, nx_e1);
      named_sync(2, 256);
      if (!waitw(&d2full[b], par, s_abort, p.err) || !waitw(&full[s], sph, s_abort, p.err)) {
        named_sync(2, 256);
        named_sync(2, 256);
        dead_from = it + 1;
        continue;
      }
      tc_fence_after();
      const bool valid = t * p.spb + sl_row < p.n_slabs;
      WT* wrow = (WT*)wst(s) + erow;
      const uint32_t* drow = ds + erow;
      const uint32_t dbase = tmem + p.d2_col[b] + lane_base;
      for (int c = c_lo; c < c_hi; ++c) {
        float v[16];
        tmem_ld16(dbase + c * 16, v);
        if (!valid) continue;
        const int ib0 = c * 8;
        if (ib0 + 8 <= Ib) {
          float2 w[8];
          uint32_t d[8];
#pragma unroll
          for (int u = 0; u < 8; ++u) {
            w[u] = wload(wrow + ib0 + u);
            d[u] = drow[ib0 + u];
          }
          const float2 nlr2 = make_float2(nlr, nlr), dec2 = make_float2(decay, decay);
#pragma unroll
          for (int u = 0; u < 8; ++u) {
            const float2 x = add_f2_h2(make_float2(v[2 * u], v[2 * u + 1]), d[u]);
            const float2 y = ffma2(nlr2, x, UNIT_DECAY ? w[u] : fmul2(w[u], dec2));
            wstore(wrow + ib0 + u, y.x, y.y);
          }
        } else {
#pragma unroll
          for (int u = 0; u < 8; ++u) {
            if (ib0 + u < Ib) {
              float2 w = wload(wrow + ib0 + u), d = h2_to_f2(drow[ib0 + u]);
              wstore(wrow + ib0 + u, __fmaf_rn(nlr, v[2 * u] + d.x, w.x * decay),
                     __fmaf_rn(nlr, v[2 * u + 1] + d.y, w.y * decay));
            }
          }
        }
      }
      tc_fence_before();
      fence_async_smem();
      mbar_arrive(&d2empty[b]);
      mbar_arrive(&wdone[s]);
      named_sync(2, 256);  // every read of the scattered buffer is done
      // zero the scattered slots again, then move to the next tile's entries
#pragma unroll
      for (int j = 0; j < EPF; ++j) {
        int64_t e = cur_e0 + et + 256 * j;
        if (e < cur_e1) ds[zl[j]] = 0u;
      }
      for (int64_t e = cur_e0 + 256 * EPF + et; e < cur_e1; e += 256) ds[p.loc[e]] = 0u;
      named_sync(2, 256);  // zeroed before the next tile scatters
      cur_e0 = nx_e0;
      cur_e1 = nx_e1;
      nx_e0 = nn_e0;
      nx_e1 = nn_e1;
      if (++s == ns) {
        s = 0;
        sph ^= 1u;
      }
    }
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
  int a2_rows = 128;
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
  int r3_nstage = 3, p1_nstage = 3;
  int num_sms = 148;
  const float* U[8] = {};
};

// Projection shared memory: nstage tile stages, A2 twice, B1, B2, barriers.
size_t p1_smem_bytes(int Ib, int ns, int K2, int K1, int N1, int N2, uint32_t lbo_a2, P1Args* a) {
  size_t off = 0;
  auto take = [&](size_t b) {
    size_t o = off;
    off += (b + 127) / 128 * 128;
    return (uint32_t)o;
  };
  const size_t tile = ((size_t)128 * Ib * 4 + 127) / 128 * 128;
  uint32_t st = take(tile * ns), a2 = take((size_t)2 * (K2 / 8) * lbo_a2);
  uint32_t b1 = take((size_t)N1 * K1 * 2), b2 = take((size_t)N2 * K2 * 2);
  uint32_t bar = take(256);
  if (a) {
    a->nstage = ns;
    a->stage_bytes = (uint32_t)tile;
    a->lbo_a2 = lbo_a2;
    a->off_stage = st;
    a->off_A2 = a2;
    a->off_B1 = b1;
    a->off_B2 = b2;
    a->off_bar = bar;
  }
  return off;
}

size_t r3_smem_bytes(int Ib, int spb, int64_t yp_bs, int wbytes, int nstage, int K1, int N1, int K2,
                     int N2, R3Args* a) {
  size_t off = 0;
  auto take = [&](size_t b) {
    size_t o = off;
    off += (b + 127) / 128 * 128;
    return (uint32_t)o;
  };
  size_t wt = (size_t)128 * Ib * wbytes, yt = (size_t)spb * yp_bs * 4;
  wt = (wt + 127) / 128 * 128;
  yt = (yt + 127) / 128 * 128;
  const uint32_t lbo_b1 = (uint32_t)(N1 / 8) * 128 + 16;
  uint32_t w = take(wt * nstage), y = take(yt * nstage);
  uint32_t b1 = take((size_t)2 * (K1 / 8) * lbo_b1), b2 = take((size_t)N2 * K2 * 2);
  uint32_t dsb = take((size_t)128 * Ib * 4), bar = take(256);
  (void)K2;
  if (a) {
    a->lbo_b1 = lbo_b1;
    a->w_tile_bytes = (uint32_t)wt;
    a->y_tile_bytes = (uint32_t)yt;
    a->off_w = w;
    a->off_y = y;
    a->off_B1 = b1;
    a->off_B2 = b2;
    a->off_ds = dsb;
    a->off_bar = bar;
  }
  return off;
}

constexpr size_t SMEM_LIMIT = 227 * 1024 - 1024;
constexpr size_t ONE_CTA_SMEM = 120 * 1024;

bool geometry(TcImpl& g, int nd, const int64_t* shape, const int64_t* ranks, uint32_t proj_mask, int wdt) {
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
  // GEMM2 groups at most 64 valid rows when a slab's rows allow it; its A
  // operand then holds 64 physical rows and the MMA's rows 64-127 read
  // in-bounds shared memory whose results are never used.
  if (g.rb * g.spb <= 64) {
    g.q = 64 / (g.rb * g.spb);
    g.a2_rows = 64;
  } else {
    g.q = 1;
    g.a2_rows = 128;
  }
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
  const uint32_t lbo_a2 = (uint32_t)(g.a2_rows / 8) * 128 + 16;
  // Projection shared memory: as many load stages as fit.
  for (g.p1_nstage = P1_NS_MAX; g.p1_nstage >= 2; --g.p1_nstage) {
    g.p1_smem = p1_smem_bytes(g.Ib, g.p1_nstage, g.K2, g.K1, g.N1, g.N2, lbo_a2, nullptr);
    if (g.p1_smem <= SMEM_LIMIT) break;
  }
  if (g.p1_smem > SMEM_LIMIT) return false;
  // TMEM (512 columns): P1 holds D1 twice, D2 twice and GEMM1's A twice
  // (K1 / 2 columns each); R3 holds D1 and D2 twice, its GEMM1's A once and its
  // GEMM2's A twice.
  auto r32 = [](int x) { return (x + 31) / 32 * 32; };
  if (2 * r32(g.N1) + 2 * r32(g.N2) + 2 * r32(g.K1 / 2) > 512) return false;
  if (2 * r32(g.rN1) + 2 * r32(g.rN2) + r32(g.rK1 / 2) + 2 * r32(g.rK2 / 2) > 512) return false;
  // Reconstruction: as many W stages as fit (it is bound by the bytes it
  // keeps in flight), at least three.
  int wbytes = wdt == TGD_C64 ? 8 : 4;
  for (g.r3_nstage = R3_NS_MAX; g.r3_nstage >= 3; --g.r3_nstage) {
    g.r3_smem = r3_smem_bytes(g.Ib, g.spb, g.bs_pad, wbytes, g.r3_nstage, g.rK1, g.rN1, g.rK2, g.rN2, nullptr);
    if (g.r3_smem <= SMEM_LIMIT) break;
  }
  if (g.r3_smem > SMEM_LIMIT) return false;
  g.inner.clear();
  for (int n = 0; n < nd - 2; ++n) {
    InnerMode m;
    m.n = n;
    m.I = shape[n];
    m.r = ranks[n];
    m.active = ((proj_mask >> n) & 1u) != 0;
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

bool tc_supported(int nd, const int64_t* shape, const int64_t* ranks, uint32_t proj_mask, int gdt, int wdt) {
  if (gdt != TGD_C32H || (wdt != TGD_C32H && wdt != TGD_C64)) return false;
  TcImpl g;
  return geometry(g, nd, shape, ranks, proj_mask, wdt);
}

bool tc_plan(TcPlan& p, int nd, const int64_t* shape, const int64_t* ranks, uint32_t proj_mask, int64_t k,
             int gdt, int wdt, AllocFn alloc, void* ctx) {
  TcImpl* g = new TcImpl;
  if (!geometry(*g, nd, shape, ranks, proj_mask, wdt)) {
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
  if (p.sm_budget > 0 && p.sm_budget < g->num_sms) g->num_sms = p.sm_budget;
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

float* tc_core(TcPlan& p) {
  TcImpl* g = impl_of(p);
  return g ? g->C : nullptr;
}

cudaError_t tc_step(TcPlan& p, const void* grad, void* w, float* sp_m, float* sp_v, float* core_m,
                    float* core_v, const AdamConst& asp, const AdamConst& acore, float decay, float lr,
                    int* d_err, cudaStream_t s, TimerHook hook, void* hook_ctx) {
  cudaError_t e = tc_step_project(p, grad, sp_m, sp_v, asp, d_err, s, hook, hook_ctx);
  if (e != cudaSuccess) return e;
  return tc_step_finish(p, w, core_m, core_v, acore, decay, lr, d_err, s, hook, hook_ctx);
}

cudaError_t tc_step_project(TcPlan& p, const void* grad, float* sp_m, float* sp_v, const AdamConst& asp,
                            int* d_err, cudaStream_t s, TimerHook hook, void* hook_ctx) {
  TcImpl* g = impl_of(p);
  if (!g) return cudaErrorNotReady;
  auto H = [&](int ph, const char* name) {
    if (hook) hook(hook_ctx, ph, name, s);
  };
  const int d = p.d;
  int first_active = -1;
  for (int n = 0; n < d - 2; ++n)
    if (g->inner[n].active && first_active < 0) first_active = n;
  // ---- projection stream over G
  P1Args& a = g->p1;
  p1_smem_bytes(g->Ib, g->p1_nstage, g->K2, g->K1, g->N1, g->N2, (uint32_t)(g->a2_rows / 8) * 128 + 16, &a);
  {
    // TMEM columns: D1 x2, D2 x2, GEMM1's A x2 (each 32-column aligned)
    const uint32_t n1 = (uint32_t)((g->N1 + 31) / 32 * 32), n2 = (uint32_t)((g->N2 + 31) / 32 * 32);
    const uint32_t na = (uint32_t)((g->K1 / 2 + 31) / 32 * 32);
    a.d1_col[0] = 0;
    a.d1_col[1] = n1;
    a.d2_col[0] = 2 * n1;
    a.d2_col[1] = 2 * n1 + n2;
    a.a1_col[0] = 2 * n1 + 2 * n2;
    a.a1_col[1] = 2 * n1 + 2 * n2 + na;
  }
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
  a.log2Ia = __builtin_ctz((unsigned)g->Ia);
  a.q = g->q;
  a.sg = g->sg;
  a.K1 = g->K1;
  a.N1 = g->N1;
  a.K2 = g->K2;
  a.N2 = g->N2;
  a.tile_off = g->tile_off;
  a.loc = g->loc;
  a.gs = g->sp_upd;  // g_s, replaced in place by S~ below
  a.B1img = (const uint8_t*)g->B1img;
  a.B2img = (const uint8_t*)g->B2img;
  const bool no_inner = first_active < 0;
  a.Y = no_inner ? (void*)g->C : (void*)g->Y;
  a.y_f32 = no_inner ? 1 : 0;
  a.y_vec = a.y_f32 ? (g->ra % 2 == 0) : (g->ra % 4 == 0);
  a.err = d_err;
  a.wait_ns = p.wait_ns ? p.wait_ns : WAIT_NS;
  a.skip_first_copy = p.skip_first_copy;
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
  if (p.k > 0) {
    H(0, "sparse_adam");
    const unsigned blocks = (unsigned)std::min<int64_t>(ceil_div(p.k, 256), (int64_t)g->num_sms * 8);
    sparse_adam_tc_kernel<<<blocks, 256, 0, s>>>(g->sp_upd, p.k, sp_m, sp_v, asp);
    H(1, "sparse_adam");
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
  }
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
  return cudaSuccess;
}

cudaError_t tc_step_finish(TcPlan& p, void* w, float* core_m, float* core_v, const AdamConst& acore,
                           float decay, float lr, int* d_err, cudaStream_t s, TimerHook hook,
                           void* hook_ctx, bool recon) {
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
  const bool no_inner = first_active < 0;
  int64_t dims[8];
  for (int n = 0; n < d - 2; ++n) dims[n] = g->inner[n].active ? p.r[n] : p.I[n];
  const uint32_t* cur = nullptr;
  uint32_t* bufs[2] = {g->X0, g->X1};
  int which = 0;
  cudaError_t e = cudaSuccess;
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
  if (!recon) return cudaSuccess;
  return tc_recon(p, w, 0, g->n_tiles, decay, lr, d_err, s, hook, hook_ctx);
}

int64_t tc_tiles(TcPlan& p) {
  TcImpl* g = impl_of(p);
  return g ? g->n_tiles : 0;
}
int64_t tc_tile_elems(TcPlan& p) {
  TcImpl* g = impl_of(p);
  return g ? g->tile_elems : 0;
}

cudaError_t tc_recon(TcPlan& p, void* w, int64_t tile0, int64_t tiles, float decay, float lr, int* d_err,
                     cudaStream_t s, TimerHook hook, void* hook_ctx) {
  TcImpl* g = impl_of(p);
  if (!g) return cudaErrorNotReady;
  if (tile0 < 0 || tiles < 1 || tile0 + tiles > g->n_tiles) return cudaErrorInvalidValue;
  auto H = [&](int ph, const char* name) {
    if (hook) hook(hook_ctx, ph, name, s);
  };
  cudaError_t e = cudaSuccess;
  // ---- reconstruction stream over W
  R3Args& r = g->r3;
  const int wbytes = g->wdt == TGD_C64 ? 8 : 4;
  r.nstage = g->r3_nstage;
  {
    // TMEM columns: D1 x2, D2 x2, A1 (the U_a image), A2 x2; 32-column aligned
    auto r32c = [](int x) { return (uint32_t)((x + 31) / 32 * 32); };
    const uint32_t n1 = r32c(g->rN1), n2 = r32c(g->rN2), na1 = r32c(g->rK1 / 2), na2 = r32c(g->rK2 / 2);
    r.d1_col[0] = 0;
    r.d1_col[1] = n1;
    r.d2_col[0] = 2 * n1;
    r.d2_col[1] = 2 * n1 + n2;
    r.a1_col = 2 * n1 + 2 * n2;
    r.a2_col[0] = r.a1_col + na1;
    r.a2_col[1] = r.a1_col + na1 + na2;
  }
  r3_smem_bytes(g->Ib, g->spb, g->bs_pad, wbytes, r.nstage, g->rK1, g->rN1, g->rK2, g->rN2, &r);
  r.Yp = g->Yp;
  r.yp_bs = g->bs_pad;
  r.W = w;
  r.w_c64 = g->wdt == TGD_C64 ? 1 : 0;
  r.N = p.N;
  r.n_slabs = g->n_slabs;
  r.n_tiles = g->n_tiles;
  r.tile0 = tile0;
  r.tiles = tiles;
  r.tile_elems = g->tile_elems;
  r.Ia = g->Ia;
  r.Ib = g->Ib;
  r.ra = g->ra;
  r.rb = g->rb;
  r.spb = g->spb;
  r.log2Ia = __builtin_ctz((unsigned)g->Ia);
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
  const unsigned r3_grid = (unsigned)std::min<int64_t>(tiles, g->num_sms);
  auto launch_r3 = [&](auto kern) -> cudaError_t {
    cudaError_t err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)r3_launch_smem);
    if (err != cudaSuccess) return err;
    H(0, "recon_stream");
    kern<<<r3_grid, R3T, r3_launch_smem, s>>>(r);
    return cudaSuccess;
  };
  const bool unit = decay == 1.0f;
  if (r.w_c64)
    e = unit ? launch_r3(recon_stream_kernel<float2, true>) : launch_r3(recon_stream_kernel<float2, false>);
  else
    e = unit ? launch_r3(recon_stream_kernel<__half2, true>) : launch_r3(recon_stream_kernel<__half2, false>);
  if (e != cudaSuccess) return e;
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
