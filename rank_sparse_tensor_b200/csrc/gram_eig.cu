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
// type and entries of Omega (a bitmask) read as zero. A block owns one output
// tile of edge TI = 4 nb (the smallest multiple of 4 >= I_n, at most 64;
// upper tile pairs when I_n > 64); each thread keeps a 4 x 4 block of complex
// sums in registers, and when the tile is small several thread groups take
// interleaved columns of a chunk and their sums are added in group order.
//
// Eigensolver: two-sided Jacobi in fp64 with the round-robin parallel
// ordering (n/2 disjoint rotations per round), one thread block per matrix,
// matrices in shared memory when n <= 64 and in global scratch otherwise.
// Output: eigenvalues descending (ties to the lower index) and the leading
// r_n eigenvectors, each scaled by a unit phase that makes its largest-
// magnitude entry (ties to the lowest row) real and positive.

#include <cuda.h>
#include <cuda_bf16.h>

#include <cstring>

#include "common.cuh"
#include "kernels.h"
#include "tc_ptx.cuh"

namespace tgd {
namespace {

constexpr int GCC = 32;    // columns of one sub-chunk (one per loader lane)
constexpr int GMAXT = 256; // threads per Gram block, at most
constexpr int GEPT = 16;   // elements one loader lane carries per chunk, at most

struct GramGeom {
  int64_t A, I, B, ncol;
  int TI;      // tile edge, 4 * nb
  int nb;      // thread grid edge: thread (ty, tx) owns rows ty + nb p, columns tx + nb q
  int ng;      // thread groups; group g takes chunk columns g, g + ng, ...
  int nthr;    // ng * nb * nb
  int nsub;    // sub-chunks of GCC columns per chunk
  int col_fast;  // loader lanes run along columns (B >= 4) or along rows
  int nti, npairs, nsplit;
  int64_t cols_per_split;
};

// Loader units of one chunk: (tile, sub-chunk, row) along columns, or
// (tile, sub-chunk, row half, column) along rows.
int gram_units(const GramGeom& g, int ntile, int nsub) {
  const int nrh = (g.TI + 31) / 32;
  return g.col_fast ? ntile * nsub * g.TI : ntile * nsub * nrh * GCC;
}

GramGeom gram_geom(int nd, const int64_t* dims, int n) {
  GramGeom g;
  g.A = 1;
  g.B = 1;
  for (int q = 0; q < n; ++q) g.A *= dims[q];
  for (int q = n + 1; q < nd; ++q) g.B *= dims[q];
  g.I = dims[n];
  g.ncol = g.A * g.B;
  g.nb = g.I > 64 ? 16 : (int)ceil_div(g.I, 4);
  g.TI = 4 * g.nb;
  g.ng = g.I > 64 ? 1 : std::min(64, GMAXT / (g.nb * g.nb));
  g.nthr = g.ng * g.nb * g.nb;
  g.col_fast = g.B >= 4;
  g.nti = (int)ceil_div(g.I, g.TI);
  g.npairs = g.nti * (g.nti + 1) / 2;
  const int ntile = g.nti > 1 ? 2 : 1;
  const int nwl = g.nthr / 32;
  g.nsub = std::max(1, 64 / g.TI);
  while (g.nsub > 1 && ceil_div(gram_units(g, ntile, g.nsub), nwl) > GEPT) --g.nsub;
  const int64_t chunk = (int64_t)GCC * g.nsub;
  // about six blocks per SM over all tile pairs; the partial sums stay under
  // 32 MB and every split gets at least two chunks
  int64_t ns = ceil_div(148 * 6, g.npairs);
  ns = std::min<int64_t>(ns, std::max<int64_t>(1, (32 << 20) / (8 * g.I * g.I)));
  ns = std::min<int64_t>(ns, std::max<int64_t>(1, ceil_div(g.ncol, 2 * chunk)));
  g.cols_per_split = ceil_div(ceil_div(g.ncol, ns), chunk) * chunk;
  g.nsplit = (int)ceil_div(g.ncol, g.cols_per_split);
  return g;
}

size_t gram_smem_bytes(const GramGeom& g) {
  const int ntile = g.nti > 1 ? 2 : 1;
  const size_t x = sizeof(float2) * (size_t)ntile * GCC * g.nsub * (g.TI + 1);
  const size_t red = sizeof(float2) * (size_t)g.ng * g.TI * g.TI;
  return std::max(x, red) + sizeof(int64_t) * 2 * GCC * g.nsub;
}

template <int DT>
__device__ __forceinline__ float2 masked_elem(const void* g, const uint32_t* bits, int64_t idx) {
  if (bits && mask_bit(bits, idx)) return make_float2(0.f, 0.f);
  return load_elem<DT>(g, idx);
}

// One (tile pair, column split) of the mode-n Gram R_(n) R_(n)^H. Column c of
// the unfolding is (a, b) = (c / B, c mod B); its row i sits at a I B + i B + b.
// Shared memory: X[tile][chunk column][row] (row stride TI + 1), reused for the
// group sums at the end, then the start offsets of the chunk's columns (two
// slots: the next chunk's are written while this one is read).
template <int DT>
__global__ void __launch_bounds__(GMAXT, 2) gram_partial_kernel(const void* g, const uint32_t* bits,
                                                                GramGeom geo, float2* partial) {
  extern __shared__ __align__(16) unsigned char gram_smem[];
  const int TI = geo.TI, nb = geo.nb, ng = geo.ng, LD = TI + 1;
  const int CCt = GCC * geo.nsub;
  const int ntile_max = geo.nti > 1 ? 2 : 1;
  float2* X = (float2*)gram_smem;
  const size_t x_elems = (size_t)ntile_max * CCt * LD, red_elems = (size_t)ng * TI * TI;
  int64_t* colbase = (int64_t*)(X + (x_elems > red_elems ? x_elems : red_elems));
  // tile pair (ti <= tj) from the linear pair index
  int pr = blockIdx.x, ti = 0;
  while (pr >= geo.nti - ti) {
    pr -= geo.nti - ti;
    ++ti;
  }
  const int tj = ti + pr;
  const int ntile = ti == tj ? 1 : 2;
  const int tid = threadIdx.x, lane = tid & 31, w = tid >> 5, nwl = geo.nthr >> 5;
  const int nrh = (TI + 31) >> 5;
  const int nunits = geo.col_fast ? ntile * geo.nsub * TI : ntile * geo.nsub * nrh * GCC;
  const int64_t c_begin = (int64_t)blockIdx.y * geo.cols_per_split;
  const int64_t c_end = c_begin + geo.cols_per_split < geo.ncol ? c_begin + geo.cols_per_split : geo.ncol;
  const int64_t IB = geo.I * geo.B;
  auto set_colbase = [&](int slot, int64_t c0) {
    for (int j = tid; j < CCt; j += geo.nthr) {
      const int64_t c = c0 + j;
      int64_t off = -1;
      if (c < c_end) {
        const int64_t a = c / geo.B;
        off = a * IB + (c - a * geo.B);
      }
      colbase[slot * CCt + j] = off;
    }
  };
  // Loader unit k of this lane, decoded once (the mapping is the same for
  // every chunk) and packed: bits 0-12 the X index, 13-21 the chunk column,
  // 22-31 the matrix row (1023: outside the matrix, store zero); all ones: no
  // unit.
  uint32_t upk[GEPT];
#pragma unroll
  for (int k = 0; k < GEPT; ++k) {
    const int u = w + nwl * k;
    upk[k] = ~0u;
    if (w < nwl && u < nunits) {
      int t, col, row;
      if (geo.col_fast) {
        const int sub_t = u / TI;  // (tile, sub-chunk)
        row = u - sub_t * TI;
        t = sub_t / geo.nsub;
        col = (sub_t - t * geo.nsub) * GCC + lane;
      } else {
        const int cc = u & (GCC - 1), th = u >> 5;  // th = (tile, sub-chunk, row half)
        const int h = nrh == 2 ? (th & 1) : 0, ts = nrh == 2 ? (th >> 1) : th;
        t = ts / geo.nsub;
        col = (ts - t * geo.nsub) * GCC + cc;
        row = lane + 32 * h;
      }
      const int grow = (t ? tj : ti) * TI + row;
      const uint32_t xi = (uint32_t)((t * CCt + col) * LD + row);
      if (row < TI)
        upk[k] = xi | ((uint32_t)col << 13) | ((uint32_t)(grow < geo.I ? grow : 1023) << 22);
    }
  }
  float2 pre[GEPT];
  auto load = [&](int slot) {
#pragma unroll
    for (int k = 0; k < GEPT; ++k) {
      float2 v = make_float2(0.f, 0.f);
      const uint32_t pk = upk[k];
      const uint32_t grow = pk >> 22;
      if (pk != ~0u && grow != 1023u) {
        const int64_t cb = colbase[slot * CCt + ((pk >> 13) & 511u)];
        if (cb >= 0) v = masked_elem<DT>(g, bits, cb + (int64_t)grow * geo.B);
      }
      pre[k] = v;
    }
  };
  auto store = [&]() {
#pragma unroll
    for (int k = 0; k < GEPT; ++k)
      if (upk[k] != ~0u) X[upk[k] & 8191u] = pre[k];
  };
  const int grp = tid / (nb * nb), l = tid - grp * nb * nb, ty = l / nb, tx = l - ty * nb;
  const float2* Xa = X + ty;
  const float2* Xb = X + (size_t)(ntile - 1) * CCt * LD + tx;
  float2 acc[4][4];
#pragma unroll
  for (int p = 0; p < 4; ++p)
#pragma unroll
    for (int q = 0; q < 4; ++q) acc[p][q] = make_float2(0.f, 0.f);

  set_colbase(0, c_begin);
  __syncthreads();
  load(0);
  int slot = 0;
  for (int64_t c0 = c_begin; c0 < c_end; c0 += CCt) {
    store();
    set_colbase(slot ^ 1, c0 + CCt);
    __syncthreads();
    if (c0 + CCt < c_end) load(slot ^ 1);
#pragma unroll 4
    for (int col = grp; col < CCt; col += ng) {
      float2 a[4], b[4];
#pragma unroll
      for (int p = 0; p < 4; ++p) a[p] = Xa[(size_t)col * LD + nb * p];
#pragma unroll
      for (int q = 0; q < 4; ++q) b[q] = Xb[(size_t)col * LD + nb * q];
#pragma unroll
      for (int p = 0; p < 4; ++p)
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          // a * conj(b)
          acc[p][q].x = __fmaf_rn(a[p].x, b[q].x, acc[p][q].x);
          if constexpr (Dt<DT>::cplx) {
            acc[p][q].x = __fmaf_rn(a[p].y, b[q].y, acc[p][q].x);
            acc[p][q].y = __fmaf_rn(a[p].y, b[q].x, __fmaf_rn(-a[p].x, b[q].y, acc[p][q].y));
          }
        }
    }
    __syncthreads();
    slot ^= 1;
  }
  // group sums in group order, then the tile's rows inside the matrix
  float2* red = X;
#pragma unroll
  for (int p = 0; p < 4; ++p)
#pragma unroll
    for (int q = 0; q < 4; ++q) red[((size_t)grp * TI + ty + nb * p) * TI + tx + nb * q] = acc[p][q];
  __syncthreads();
  float2* out = partial + (int64_t)blockIdx.y * geo.I * geo.I;
  for (int e = tid; e < TI * TI; e += geo.nthr) {
    const int r = e / TI, cl = e - r * TI;
    float2 sum = red[e];
    for (int gg = 1; gg < ng; ++gg) {
      const float2 v = red[(size_t)gg * TI * TI + e];
      sum.x += v.x;
      sum.y += v.y;
    }
    const int64_t gi = (int64_t)ti * TI + r, gj = (int64_t)tj * TI + cl;
    if (gi < geo.I && gj < geo.I) out[gi * geo.I + gj] = sum;
  }
}

// fp64 sum of the split partials: a block takes RC cells, its RS thread rows
// take interleaved splits, and the RS slices are added in slice order. Lower
// tiles come from the upper partials, conjugated.
constexpr int RC = 32, RS = 8;
__global__ void __launch_bounds__(RC * RS) gram_reduce_kernel(const float2* partial, GramGeom geo,
                                                              double2* gram) {
  __shared__ double2 part[RS][RC];
  const int64_t I = geo.I;
  const int cl = threadIdx.x % RC, sl = threadIdx.x / RC;
  const int64_t e = (int64_t)blockIdx.x * RC + cl;
  double sx = 0, sy = 0;
  bool upper = true;
  if (e < I * I) {
    const int64_t i = e / I, j = e - i * I;
    upper = (i / geo.TI) <= (j / geo.TI);
    const int64_t src = upper ? i * I + j : j * I + i;
#pragma unroll 4
    for (int s = sl; s < geo.nsplit; s += RS) {
      const float2 v = partial[(int64_t)s * I * I + src];
      sx += (double)v.x;
      sy += (double)v.y;
    }
  }
  part[sl][cl] = make_double2(sx, sy);
  __syncthreads();
  if (sl == 0 && e < I * I) {
    double tx = 0, ty = 0;
    for (int q = 0; q < RS; ++q) {
      tx += part[q][cl].x;
      ty += part[q][cl].y;
    }
    gram[e] = upper ? make_double2(tx, ty) : make_double2(tx, -ty);
  }
}

// ------------------------------------------------ tensor-core Gram (I_n <= 128)
// The Gram as tcgen05 GEMMs over chunks of at most 32 unfolding columns
// (K = (column, re/im) pairs: 64 bf16 values). Each fp32 value is split into
// three bf16 parts h + m + l (each the bf16 rounding of what the earlier
// parts leave); the Gram is the sum of the part products, of which hh, hm,
// mh, hl, lh and mm (and, where they come free, ml, lm, ll) are formed,
// which keeps about fp32 accuracy.
//
// For part p a K-major tile holds the rows x_i and J x_i, where J maps each
// (re, im) pair of a column to (-im, re). With Y = [x_h; x_m; x_l] (3I rows,
// the B operand), the product of [x_p; J x_p] with Y gives, in column block
// q of D, Re sum_c x_ic conj(y_jc) in the x rows and -Im sum_c x_ic conj(y_jc)
// in the J x rows. An MMA costs about the same below N = 128 whatever its
// N, so the parts are packed as densely as the 128 rows of an A tile allow:
// P_A = min(3, 64 / I) parts per A tile (one MMA per K step for I <= 21,
// two for I <= 32, three for I <= 64), each A tile multiplied with the part
// blocks of Y it needs. Every product lands in D at the row of its A part
// and the column block of its B part; the epilogue adds the column blocks
// and the stacked part rows in a fixed order.
//
// The unfolding is viewed as [A][I][B] (A, B the products of the dimensions
// before and after mode n), column c = a B + b. One CTA per SM owns a range
// of chunks and runs a pipeline whose roles hand stages over through
// mbarriers:
// - a producer warp brings each chunk into a ring of TG_NS shared-memory
//   stages: when B is a multiple of 32, a chunk is 32 columns of one slab a,
//   fetched by one TMA tensor copy of its I x 32 box (TG_ROWS); when B < 32,
//   a chunk is floor(32 / B) whole slabs, one contiguous bulk copy
//   (TG_SLABS); any other layout goes element by element (TG_ELEMS). The
//   words of Omega's bitmask the chunk needs (two per row, or the block's)
//   come by asynchronous copies beside it (TG_ELEMS, the fallback, reads the
//   bits where it converts);
// - two groups of eight converter warps take alternate chunks, each group
//   turning its chunk into the bf16 tiles of its own tile set (one thread:
//   one row, four columns), the entries of Omega read as zero (the
//   residual);
// - one thread issues the chunk's MMAs and commits them to the tile set's
//   free barrier.
constexpr int TG_CONV_WARPS = 16;
constexpr int TG_GROUP_WARPS = 8;           // converter warps per tile set
constexpr int TG_PROD_WARP = TG_CONV_WARPS;
constexpr int TG_MMA_WARP = TG_CONV_WARPS + 1;
constexpr int TG_THREADS = 32 * (TG_CONV_WARPS + 2);
constexpr int TG_COLS = 32;                 // columns of a TG_ROWS / TG_ELEMS chunk
constexpr int TG_KC_MAX = 64;               // column capacity of a chunk (TG_SLABS may take 64)
constexpr int TG_NS_MAX = 4;                // staging stages
constexpr uint32_t TG_LBO_A = 2048;         // A tile: 128 rows x 16 B between K core matrices
constexpr int TG_MASK_WORDS = 256;          // two per row, or a block of <= 4096 bits + 1
constexpr uint64_t TG_WAIT_NS = 2000000000ull;

enum TgMode { TG_ROWS = 0, TG_SLABS = 1, TG_ELEMS = 2 };

struct TcGramArgs {
  const void* g;
  const uint32_t* bits;
  int64_t A, I, B;            // the unfolding as [A][I][B]
  int64_t nchunk;             // chunks of the whole unfolding
  int64_t chunks_per_split;
  int mode;                   // TgMode
  int slabs;                  // slabs per chunk (TG_SLABS)
  int kc;                     // column capacity of a chunk: 16, 32, or 64 (TG_SLABS)
  int ns;                     // staging stages
  int parts;                  // bf16 parts per value: 3, or 2 for 16-bit inputs (I > 64)
  float* partial;             // [split][I][I] complex, interleaved
  int* err;
};

// What the converters need of a staged chunk besides its elements.
struct TgMeta {
  int ncols;                  // valid columns
  int rs;                     // staged stride between rows (elements)
  int sh;                     // bit offset in its first word: of the block (TG_SLABS), of row 0 (TG_ROWS)
  int bsh;                    // TG_ROWS: B mod 32 (row i's offset is sh + i bsh, mod 32)
  int colofs[TG_KC_MAX];      // staged offset of each column's row 0 (elements)
  int64_t gcol[TG_COLS];      // TG_ELEMS: element index of each column's row 0
  uint32_t wm[TG_MASK_WORDS]; // Omega's words: two per row (TG_ROWS), the block's (TG_SLABS)
};

// Parts per A tile for mode size I, and the number of A tiles.
// Byte offset of element (i, col) in a TG_ROWS / TG_ELEMS stage. 8- and
// 4-byte elements: rows of 128 bytes (a box of 16, or of 32, columns; 8-byte
// elements fill two boxes, each starting on a 1024-byte boundary), the
// 16-byte units of row i permuted by XOR with i mod 8 (the TMA 128-byte
// swizzle), so that eight consecutive rows read or written at one column
// fall in different banks; 2-byte elements: plain 64-byte rows.
template <int ES>
__host__ __device__ __forceinline__ uint32_t tg_soff(int i, int col, uint32_t boxb) {
  if constexpr (ES == 8) {
    const uint32_t byte = (uint32_t)(col & 15) * 8;
    return (uint32_t)(col >> 4) * boxb + (uint32_t)i * 128 + ((((byte >> 4) ^ (uint32_t)(i & 7)) << 4) | (byte & 15));
  } else if constexpr (ES == 4) {
    const uint32_t byte = (uint32_t)col * 4;
    return (uint32_t)i * 128 + ((((byte >> 4) ^ (uint32_t)(i & 7)) << 4) | (byte & 15));
  } else {
    return (uint32_t)i * 64 + (uint32_t)col * 2;
  }
}
__host__ __device__ constexpr uint32_t tg_boxb(int I) { return ((uint32_t)I * 128 + 1023) / 1024 * 1024; }

__host__ __device__ constexpr int tg_parts_per_a(int I) { return I <= 21 ? 3 : (I <= 32 ? 2 : 1); }
__host__ __device__ constexpr int tg_a_tiles(int I) { return (3 + tg_parts_per_a(I) - 1) / tg_parts_per_a(I); }
// MMA N of A tile a: the Y part blocks its parts need (p + q <= 2 for the
// tile's first part p), rounded up to 16.
__host__ __device__ constexpr int tg_n_of(int I, int a) { return ((3 - a * tg_parts_per_a(I)) * I + 15) / 16 * 16; }

// Shared-memory layout for mode size I, chunk capacity kc and element size
// es: a tile set holds the A tiles (128 rows x 2 kc bf16 values each) and Y
// (N0 rows); a stage holds a chunk (the swizzled boxes, or a block).
// For 64 < I <= 128 (wide) a tile set holds, per part, an x tile and (for
// complex values) a J x tile of 128 rows each, and no Y (the x tile of part q
// is the B operand).
struct TgLayout {
  uint32_t tile_a, lbo_b, set, stage;
};
__host__ __device__ inline TgLayout tg_layout(int I, int kc, int es, int parts, bool cplx) {
  TgLayout L;
  const uint32_t kg = (uint32_t)kc / 4;
  L.tile_a = kg * TG_LBO_A;
  if (I > 64) {
    L.lbo_b = 0;
    L.set = (cplx ? 2u : 1u) * parts * L.tile_a;
  } else {
    L.lbo_b = (uint32_t)tg_n_of(I, 0) * 16;
    L.set = (uint32_t)tg_a_tiles(I) * L.tile_a + kg * L.lbo_b;
  }
  uint32_t st = (uint32_t)kc * I * es;
  if (es == 8 && ((uint32_t)kc / 16) * tg_boxb(I) > st) st = ((uint32_t)kc / 16) * tg_boxb(I);
  L.stage = (st + 1023) / 1024 * 1024;
  return L;
}

// x = h + m + l (bf16 parts, each the rounding of what the earlier leave).
// The three parts of x and y at once, packed as bf16 pairs (x in the low
// half); each part the rounding to nearest of what the earlier parts leave.
__device__ __forceinline__ uint32_t bf2_bits(float x, float y) {
  __nv_bfloat162 h = __floats2bfloat162_rn(x, y);
  return *reinterpret_cast<uint32_t*>(&h);
}
__device__ __forceinline__ void split3_pair(float x, float y, uint32_t& h, uint32_t& m, uint32_t& l) {
  h = bf2_bits(x, y);
  const float rx = x - __uint_as_float(h << 16), ry = y - __uint_as_float(h & 0xffff0000u);
  m = bf2_bits(rx, ry);
  l = bf2_bits(rx - __uint_as_float(m << 16), ry - __uint_as_float(m & 0xffff0000u));
}

// One element of ES bytes global -> shared: asynchronous for 4 and 8 bytes
// (cp.async), a plain copy for 2-byte elements (below cp.async's minimum).
template <int ES>
__device__ __forceinline__ void cp_async_elem(void* dst, const void* src) {
  if constexpr (ES == 8)
    asm volatile("cp.async.ca.shared.global [%0], [%1], 8;" ::"r"(ptx::smem_u32(dst)), "l"(src) : "memory");
  else if constexpr (ES == 4)
    asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(ptx::smem_u32(dst)), "l"(src) : "memory");
  else
    *(uint16_t*)dst = __ldg((const unsigned short*)src);
}
// The mbarrier gets one more pending arrival, made when this thread's
// earlier cp.async copies have landed.
__device__ __forceinline__ void cp_async_arrive(uint64_t* bar) {
  asm volatile("cp.async.mbarrier.arrive.shared::cta.b64 [%0];" ::"r"(ptx::smem_u32(bar)) : "memory");
}
__device__ __forceinline__ void tg_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(ptx::smem_u32(bar)) : "memory");
}
// TMA copy of the box at (x, y, z) of a 3-D tensor map into shared memory,
// completion counted in bytes on `bar`.
__device__ __forceinline__ void tma_load_3d(void* dst, const CUtensorMap* map, int x, int y, int z, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3, %4}], [%5];" ::"r"(
          ptx::smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(z), "r"(ptx::smem_u32(bar))
      : "memory");
}
// Lane 0 waits (bounded) for the phase, the warp learns the outcome; on
// expiry the error is recorded and the abort flag raised.
__device__ __forceinline__ bool tg_waitw(uint64_t* bar, uint32_t parity, volatile int* abort, int* err) {
  int ok = 1;
  if ((threadIdx.x & 31) == 0) {
    if (*abort) {
      ok = 0;
    } else if (!ptx::mbar_wait(bar, parity, TG_WAIT_NS)) {
      atomicOr(err, DEV_ERR_TIMEOUT);
      *abort = 1;
      ok = 0;
    }
  }
  ok = __shfl_sync(0xffffffffu, ok, 0);
  __syncwarp();
  return ok != 0;
}

// Element (re, im) of storage type DT from raw staged bytes.
template <int DT>
__device__ __forceinline__ float2 staged_elem(const uint8_t* p) {
  if constexpr (DT == TGD_R32) {
    return make_float2(*(const float*)p, 0.f);
  } else if constexpr (DT == TGD_C64) {
    return *(const float2*)p;
  } else if constexpr (DT == TGD_C32H) {
    return __half22float2(*(const __half2*)p);
  } else {
    return make_float2(__half2float(*(const __half*)p), 0.f);
  }
}

template <int DT>
__global__ void __launch_bounds__(TG_THREADS, 1)
    gram_tc_kernel(const TcGramArgs p, const __grid_constant__ CUtensorMap rows_map) {
  constexpr int ES = Dt<DT>::bytes;
  constexpr bool CPLX = DT == TGD_C64 || DT == TGD_C32H;
  const TgLayout L = tg_layout((int)p.I, p.kc, ES, p.parts, CPLX);
  const int NS = p.ns;
  const uint32_t STAGE = L.stage;
  extern __shared__ __align__(1024) uint8_t smem[];
  uint8_t* tiles = smem;                                        // [2] tile sets
  uint8_t* stage = smem + 2 * L.set;                            // [NS] staged chunks
  TgMeta* meta = (TgMeta*)(stage + NS * STAGE);                 // [NS]
  uint64_t* full = (uint64_t*)(meta + NS);                      // [NS] chunk staged
  uint64_t* sfree = full + TG_NS_MAX;                           // [NS] stage read
  uint64_t* tfull = sfree + TG_NS_MAX;                              // [2] tile set written
  uint64_t* tfree = tfull + 2;                                  // [2] tile set's MMAs done
  int* tks = (int*)(tfree + 2);                                 // [2] K steps of the set's chunk
  uint32_t* tslot = (uint32_t*)(tks + 2);
  __shared__ int s_abort;
  volatile int* abort = &s_abort;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int I = (int)p.I;
  const bool wide = I > 64;
  const int P = p.parts;
  const int PA = tg_parts_per_a(I), NA = tg_a_tiles(I);
  // D: narrow, 128 lanes x N0 columns; wide, the x rows' block at column 0
  // and the J x rows' block at column 128, N = I rounded up to 16 each
  const int N0 = wide ? (I + 15) / 16 * 16 : tg_n_of(I, 0);
  const uint32_t tmem_cols = wide ? 256u : (N0 <= 32 ? 32u : (N0 <= 64 ? 64u : (N0 <= 128 ? 128u : 256u)));
  const int64_t IB = p.I * p.B;
  const int64_t q_begin = (int64_t)blockIdx.x * p.chunks_per_split;
  const int64_t q_end = q_begin + p.chunks_per_split < p.nchunk ? q_begin + p.chunks_per_split : p.nchunk;
  const int nch = q_end > q_begin ? (int)(q_end - q_begin) : 0;
  const bool masked = p.bits != nullptr;
  // rows no part uses stay zero in every tile
  for (uint32_t o = tid * 16; o < 2 * L.set; o += TG_THREADS * 16) *(uint4*)(tiles + o) = make_uint4(0, 0, 0, 0);
  if (tid == 0) {
    s_abort = 0;
    for (int s = 0; s < NS; ++s) {
      ptx::mbar_init(&full[s], 1);
      ptx::mbar_init(&sfree[s], TG_GROUP_WARPS);
    }
    for (int t = 0; t < 2; ++t) {
      ptx::mbar_init(&tfull[t], TG_GROUP_WARPS);
      ptx::mbar_init(&tfree[t], 1);
    }
    ptx::fence_mbar_init();
  }
  if (warp == 0) ptx::tmem_alloc(tslot, tmem_cols);
  ptx::fence_async_smem();
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t dt_base = *tslot;
  const uint8_t* gb = (const uint8_t*)p.g;

  if (warp == TG_PROD_WARP) {
    // ------------------------------------------------------------ producer
    int issued = 0;
    // TG_SLABS: staged offset of column lane (and lane + 32) of a block
    const int co_lo = (int)((lane / p.B) * IB + lane % p.B);
    const int co_hi = (int)(((lane + 32) / p.B) * IB + (lane + 32) % p.B);
    for (int kc = 0; kc < nch; ++kc) {
      const int slot = kc % NS;
      if (kc >= NS && !tg_waitw(&sfree[slot], (uint32_t)((kc / NS - 1) & 1), abort, p.err)) break;
      TgMeta* m = &meta[slot];
      uint8_t* st = stage + slot * STAGE;
      const int64_t q = q_begin + kc;
      if (p.mode == TG_SLABS) {
        const int64_t a0 = q * p.slabs;
        const int64_t a1 = a0 + p.slabs < p.A ? a0 + p.slabs : p.A;
        const int ncols = (int)((a1 - a0) * p.B);
        const int64_t blk = a0 * IB, nel = (a1 - a0) * IB;
        if (masked) {
          const int64_t w0 = blk >> 5, nw = ((blk + nel - 1) >> 5) - w0 + 1;
          for (int w = lane; w < nw; w += 32) cp_async_elem<4>(&m->wm[w], p.bits + w0 + w);
        }
        m->colofs[lane] = co_lo;
        m->colofs[lane + 32] = co_hi;
        if (lane == 0) {
          m->ncols = ncols;
          m->rs = (int)p.B;
          m->sh = (int)(blk & 31);
        }
        cp_async_arrive(&full[slot]);
        __syncwarp();
        if (lane == 0) {
          const uint32_t bytes = (uint32_t)((nel * ES + 15) / 16 * 16);
          ptx::mbar_expect_tx(&full[slot], bytes);
          ptx::bulk_g2s(st, gb + blk * ES, bytes, &full[slot]);
        }
      } else if (p.mode == TG_ROWS) {
        const int64_t c0 = q * p.kc;
        const int64_t a = c0 / p.B;
        const int64_t b0 = c0 - a * p.B;
        const int64_t base0 = a * IB + b0;
        if (masked)
          for (int i = lane; i < I; i += 32) {
            // row i's 32 bits start at bit rb: its word and, unless rb is a
            // word boundary, the next
            const int64_t rb = base0 + (int64_t)i * p.B;
            cp_async_elem<4>(&m->wm[2 * i], p.bits + (rb >> 5));
            if (rb & 31) cp_async_elem<4>(&m->wm[2 * i + 1], p.bits + (rb >> 5) + 1);
          }
        m->colofs[lane] = lane;
        if (lane == 0) {
          m->ncols = p.kc;
          m->rs = TG_COLS;
          m->sh = (int)(base0 & 31);
          m->bsh = (int)(p.B & 31);
        }
        cp_async_arrive(&full[slot]);
        __syncwarp();
        if (lane == 0) {
          ptx::mbar_expect_tx(&full[slot], (uint32_t)(I * p.kc * ES));
          // the I rows x kc columns at column b0 of slab a; 8-byte elements
          // are addressed as pairs of 4-byte ones, in boxes of 16 columns
          if constexpr (ES == 8) {
            tma_load_3d(st, &rows_map, (int)(2 * b0), 0, (int)a, &full[slot]);
            if (p.kc == 32) tma_load_3d(st + tg_boxb(I), &rows_map, (int)(2 * b0 + 32), 0, (int)a, &full[slot]);
          } else {
            tma_load_3d(st, &rows_map, (int)b0, 0, (int)a, &full[slot]);
          }
        }
      } else {
        const int64_t c0 = q * p.kc;
        const int64_t ncol = p.A * p.B;
        const int ncols = (int)(ncol - c0 < p.kc ? ncol - c0 : p.kc);
        const bool valid = lane < ncols;
        int64_t cb = 0;
        if (valid) {
          const int64_t c = c0 + lane, a = c / p.B;
          cb = a * IB + (c - a * p.B);
        }
        if (valid)
          for (int i = 0; i < I; ++i)
            cp_async_elem<ES>(st + tg_soff<ES>(i, lane, tg_boxb(I)), gb + (cb + (int64_t)i * p.B) * ES);
        m->colofs[lane] = lane;
        m->gcol[lane] = cb;
        if (lane == 0) {
          m->ncols = ncols;
          m->rs = TG_COLS;
          m->sh = 0;
        }
        cp_async_arrive(&full[slot]);
        __syncwarp();
        if (lane == 0) tg_arrive(&full[slot]);
      }
      issued = kc + 1;
    }
    // no copy may still target this CTA's shared memory at exit
    if (lane == 0)
      for (int kc = issued > NS ? issued - NS : 0; kc < issued; ++kc)
        ptx::mbar_wait(&full[kc % NS], (uint32_t)((kc / NS) & 1), TG_WAIT_NS / 4);
    __syncwarp();
  } else if (warp == TG_MMA_WARP) {
    // ------------------------------------------------------------ MMA issuer
    uint32_t idesc[3];
#pragma unroll
    for (int a = 0; a < 3; ++a) idesc[a] = ptx::idesc_f16(1, 128, a < NA ? tg_n_of(I, a) : 16);
    // descriptors of set 0's first A tile and of its Y tile; the others by
    // adding to the start address field, which counts 16-byte units
    const uint64_t da_base = ptx::sdesc(ptx::smem_u32(tiles), TG_LBO_A, 128);
    const uint64_t dy_base = ptx::sdesc(ptx::smem_u32(tiles + NA * L.tile_a), L.lbo_b, 128);
    int issued[2] = {0, 0};
    for (int kc = 0; kc < nch; ++kc) {
      const int t = kc & 1;
      if (!tg_waitw(&tfull[t], (uint32_t)((kc >> 1) & 1), abort, p.err)) break;
      ptx::tc_fence_after();
      if (lane == 0) {
        const int nks = tks[t];
        const uint32_t set = (uint32_t)t * L.set;
        if (wide) {
          // every product (part pa of A, part qb of the x tile as B, pa + qb
          // <= 2) into one block: the x rows' at column 0, the J x rows' at 128
          const uint32_t idw = ptx::idesc_f16(1, 128, N0);
          for (int kk = 0; kk < nks; ++kk) {
            const uint32_t koff = set + kk * 2 * TG_LBO_A;
#pragma unroll
            for (int xj = 0; xj < (CPLX ? 2 : 1); ++xj) {
              int np = 0;
#pragma unroll
              for (int pa = 0; pa < 3; ++pa)
#pragma unroll
                for (int qb = 0; qb < 3; ++qb) {
                  if (pa >= P || qb >= P || pa + qb > 2) continue;
                  ptx::mma_f16(dt_base + xj * 128, da_base + ((koff + (xj * P + pa) * L.tile_a) >> 4),
                               da_base + ((koff + qb * L.tile_a) >> 4), idw, (kc > 0 || kk > 0 || np > 0) ? 1u : 0u);
                  ++np;
                }
            }
          }
        } else {
          for (int kk = 0; kk < nks; ++kk) {
            const uint64_t dy = dy_base + ((set + kk * 2 * L.lbo_b) >> 4);
#pragma unroll
            for (int a = 0; a < 3; ++a)
              if (a < NA)
                ptx::mma_f16(dt_base, da_base + ((set + a * L.tile_a + kk * 2 * TG_LBO_A) >> 4), dy, idesc[a],
                             (kc > 0 || kk > 0 || a > 0) ? 1u : 0u);
          }
        }
        ptx::mma_commit(&tfree[t]);
      }
      __syncwarp();
      issued[t] = (kc >> 1) + 1;
    }
    // every committed MMA has finished before TMEM is read or freed
    if (lane == 0)
      for (int t = 0; t < 2; ++t)
        if (issued[t] > 0 && !ptx::mbar_wait(&tfree[t], (uint32_t)((issued[t] - 1) & 1), TG_WAIT_NS)) {
          atomicOr(p.err, DEV_ERR_TIMEOUT);
          *abort = 1;
        }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ converters
    // group g converts the chunks kc = g, g + 2, ... into tile set g; a warp
    // item is 8 rows x 16 columns, lane = (row, group of four columns), so
    // that a tile store of the warp covers 8 consecutive rows (128 bytes) of
    // four K groups
    const int grp = warp / TG_GROUP_WARPS, gw = warp % TG_GROUP_WARPS;
    const int rb_n = (I + 7) / 8;
    const uint32_t boxb = tg_boxb(I);
    uint8_t* set = tiles + (size_t)grp * L.set;
    for (int kc = grp; kc < nch; kc += 2) {
      const int slot = kc % NS;
      if (!tg_waitw(&full[slot], (uint32_t)((kc / NS) & 1), abort, p.err)) break;
      if (kc >= 2 && !tg_waitw(&tfree[grp], (uint32_t)(((kc >> 1) - 1) & 1), abort, p.err)) break;
      ptx::tc_fence_after();
      const TgMeta* m = &meta[slot];
      const uint8_t* st = stage + slot * STAGE;
      const int ncols = m->ncols, rs = m->rs, sh = m->sh, bsh = m->bsh;
      const int nks = (ncols + 7) / 8, ngroups = 2 * nks;
      const int halves = (ngroups + 3) / 4;
      for (int it = gw; it < rb_n * halves; it += TG_GROUP_WARPS) {
        const int i = (it % rb_n) * 8 + (lane & 7);
        const int g = (it / rb_n) * 4 + (lane >> 3);
        if (i >= I || g >= ngroups) continue;
        const int col0 = 4 * g;
        // the four elements and their Omega bits, loaded before any use
        float2 x[4];
        uint32_t zbits = 0;
        if (p.mode != TG_SLABS && col0 + 3 < ncols) {
          if constexpr (ES == 8) {
            // columns col0..col0+3: two 16-byte units of row i in box g / 4
            const uint8_t* rowp = st + (uint32_t)(g >> 2) * boxb + (uint32_t)i * 128;
            const uint32_t c0 = 2u * (uint32_t)(g & 3), sw = (uint32_t)(i & 7);
            const float4 v0 = *(const float4*)(rowp + ((c0 ^ sw) << 4));
            const float4 v1 = *(const float4*)(rowp + (((c0 + 1) ^ sw) << 4));
            x[0] = make_float2(v0.x, v0.y);
            x[1] = make_float2(v0.z, v0.w);
            x[2] = make_float2(v1.x, v1.y);
            x[3] = make_float2(v1.z, v1.w);
          } else {
#pragma unroll
            for (int u = 0; u < 4; ++u) x[u] = staged_elem<DT>(st + tg_soff<ES>(i, col0 + u, boxb));
          }
        } else {
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            const int col = col0 + u;
            const bool v = col < ncols;
            if (p.mode == TG_SLABS) {
              const int off = (v ? m->colofs[col] : 0) + i * rs;
              x[u] = v ? staged_elem<DT>(st + (size_t)off * ES) : make_float2(0.f, 0.f);
              if (masked) {
                const int pos = sh + off;
                zbits |= ((m->wm[pos >> 5] >> (pos & 31)) & 1u) << u;
              }
            } else {
              x[u] = v ? staged_elem<DT>(st + tg_soff<ES>(i, col, boxb)) : make_float2(0.f, 0.f);
            }
          }
        }
        if (masked) {
          if (p.mode == TG_ROWS) {
            const uint32_t rowbits = __funnelshift_r(m->wm[2 * i], m->wm[2 * i + 1], (uint32_t)(sh + i * bsh) & 31u);
            zbits = (rowbits >> col0) & 0xFu;
          } else if (p.mode == TG_ELEMS) {
#pragma unroll
            for (int u = 0; u < 4; ++u)
              if (col0 + u < ncols) zbits |= (uint32_t)mask_bit(p.bits, m->gcol[col0 + u] + (int64_t)i * p.B) << u;
          }
        }
        uint32_t xr[3][4], jr[3][4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const float2 v = (zbits >> u) & 1u ? make_float2(0.f, 0.f) : x[u];
          // x row: (re, im), the three parts of both in packed pairs (the low
          // half holds the even K); J x row: (-im, re), the halves swapped and
          // the new low half negated
          split3_pair(v.x, v.y, xr[0][u], xr[1][u], xr[2][u]);
#pragma unroll
          for (int part = 0; part < 3; ++part) jr[part][u] = __byte_perm(xr[part][u], 0u, 0x1032) ^ 0x8000u;
        }
        if (wide) {
          // part p: x row i of tile p, J x row i of tile P + p
#pragma unroll
          for (int part = 0; part < 3; ++part) {
            if (part >= P) break;
            uint8_t* xp = set + (size_t)part * L.tile_a + (uint32_t)g * TG_LBO_A + (uint32_t)i * 16;
            uint8_t* jp = set + (size_t)(P + part) * L.tile_a + (uint32_t)g * TG_LBO_A + (uint32_t)i * 16;
            const uint4 vx = part == 0 ? make_uint4(xr[0][0], xr[0][1], xr[0][2], xr[0][3])
                             : part == 1 ? make_uint4(xr[1][0], xr[1][1], xr[1][2], xr[1][3])
                                         : make_uint4(xr[2][0], xr[2][1], xr[2][2], xr[2][3]);
            const uint4 vj = part == 0 ? make_uint4(jr[0][0], jr[0][1], jr[0][2], jr[0][3])
                             : part == 1 ? make_uint4(jr[1][0], jr[1][1], jr[1][2], jr[1][3])
                                         : make_uint4(jr[2][0], jr[2][1], jr[2][2], jr[2][3]);
            *(uint4*)xp = vx;
            if (CPLX) *(uint4*)jp = vj;
          }
          continue;
        }
#pragma unroll
        for (int part = 0; part < 3; ++part) {
          const int at = part / PA, arow = 2 * I * (part % PA);
          uint8_t* ap = set + (size_t)at * L.tile_a + (uint32_t)g * TG_LBO_A;
          *(uint4*)(ap + (uint32_t)(arow + i) * 16) = make_uint4(xr[part][0], xr[part][1], xr[part][2], xr[part][3]);
          *(uint4*)(ap + (uint32_t)(arow + I + i) * 16) = make_uint4(jr[part][0], jr[part][1], jr[part][2], jr[part][3]);
          uint8_t* yp = set + NA * L.tile_a + (uint32_t)g * L.lbo_b;
          *(uint4*)(yp + (uint32_t)(part * I + i) * 16) = make_uint4(xr[part][0], xr[part][1], xr[part][2], xr[part][3]);
        }
      }
      ptx::fence_async_smem();
      ptx::tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        if (gw == 0) tks[grp] = nks;
        tg_arrive(&tfull[grp]);
        tg_arrive(&sfree[slot]);
      }
    }
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  const bool ok = !*abort;
  float* out = p.partial + (size_t)blockIdx.x * p.I * p.I * 2;
  if (wide) {
    // lane = row i: the real part in the x block, the negated imaginary
    // part in the J x block
    if (warp < 4) {
      const uint32_t lane_base = (uint32_t)(warp * 32) << 16;
      const int row = tid;
      for (int c0 = 0; c0 < N0; c0 += 16) {
        float yx[16], yj[16];
        ptx::tmem_ld16(dt_base + lane_base + c0, yx);
        if (CPLX) {
          ptx::tmem_ld16(dt_base + lane_base + 128 + c0, yj);
        } else {
#pragma unroll
          for (int u = 0; u < 16; ++u) yj[u] = 0.f;
        }
        if (row < I) {
#pragma unroll
          for (int u = 0; u < 16; ++u) {
            const int j = c0 + u;
            if (j < I) {
              out[((int64_t)row * I + j) * 2] = ok && nch > 0 ? yx[u] : 0.f;
              out[((int64_t)row * I + j) * 2 + 1] = ok && nch > 0 ? -yj[u] : 0.f;
            }
          }
        }
      }
    }
    ptx::tc_fence_before();
    __syncthreads();
    if (warp == 0) ptx::tmem_dealloc(dt_base, tmem_cols);
    return;
  }
  // D (128 lanes x N0 columns) -> shared memory S over the tile sets, which
  // no MMA reads any more; warp w reads TMEM lanes 32w..32w+31
  const int SP = N0 + 1;  // S row pitch (floats)
  float* S = (float*)tiles;
  if (warp < 4) {
    const uint32_t lane_base = (uint32_t)(warp * 32) << 16;
    for (int c0 = 0; c0 < N0; c0 += 16) {
      float y[16];
      ptx::tmem_ld16(dt_base + lane_base + c0, y);
#pragma unroll
      for (int u = 0; u < 16; ++u) S[tid * SP + c0 + u] = y[u];
    }
  }
  __syncthreads();
  // stacked row r < 2I (x rows: the real part of row r; J x rows: the
  // negated imaginary part of row r - I), column j < I: the sum over the A
  // tile's part slots s and Y's column blocks q, in that order
  for (int e = tid; e < 2 * I * I; e += TG_THREADS) {
    const int r = e / I, j = e % I;
    float v = 0.f;
    if (ok && nch > 0)
      for (int s = 0; s < PA; ++s)
        for (int q = 0; q < 3; ++q) v += S[(2 * I * s + r) * SP + q * I + j];
    const bool re = r < I;
    out[((int64_t)(re ? r : r - I) * I + j) * 2 + (re ? 0 : 1)] = re ? v : -v;
  }
  ptx::tc_fence_before();
  __syncthreads();
  if (warp == 0) ptx::tmem_dealloc(dt_base, tmem_cols);
}

size_t tg_smem_bytes(int I, int kc, int es, int ns, int parts, bool cplx) {
  const TgLayout L = tg_layout(I, kc, es, parts, cplx);
  return 2 * (size_t)L.set + (size_t)ns * (L.stage + sizeof(TgMeta)) + (2 * TG_NS_MAX + 4) * sizeof(uint64_t) +
         2 * sizeof(int) + 16;
}

struct TcGramGeom {
  int64_t A, I, B, nchunk, chunks_per_split;
  int nsplit, mode, slabs, kc, ns, parts;
};

constexpr int TG_MAX_SPLITS = 148;  // one CTA per SM
constexpr size_t TG_SMEM_LIMIT = 227 * 1024 - 1024;  // the opt-in maximum less the static part

// How mode n's unfolding is staged (see gram_tc_kernel) and split over CTAs:
// the mode, the chunk capacity (64 columns for blocks of whole slabs when it
// fits and I <= 32, 16 for 8-byte elements when I > 64, else 32), the bf16
// parts per value (two represent a 16-bit input exactly; used when I > 64)
// and the most stages (up to four) that fit.
TcGramGeom tc_gram_geom(int nd, const int64_t* dims, int n, int dt, bool aligned16, int max_splits) {
  const int es = dt == TGD_C64 ? 8 : (dt == TGD_R16 ? 2 : 4);
  TcGramGeom g;
  g.A = 1;
  g.B = 1;
  for (int q = 0; q < n; ++q) g.A *= dims[q];
  for (int q = n + 1; q < nd; ++q) g.B *= dims[q];
  g.I = dims[n];
  g.slabs = 1;
  const int I = (int)g.I;
  const bool wide = I > 64;
  g.parts = wide && (dt == TGD_C32H || dt == TGD_R16) ? 2 : 3;
  g.kc = wide && es == 8 ? 16 : TG_COLS;
  const int64_t total_bytes = g.A * g.I * g.B * es;
  // TMA coordinates are 32-bit: the column (in 4-byte units for 8-byte
  // elements) and the slab
  const bool tma_ok = g.A < (1ll << 31) && 2 * g.B < (1ll << 31);
  auto slabs_ok = [&](int kc) {
    return aligned16 && g.B < kc && (kc / g.B) * g.I * g.B * es % 16 == 0 && total_bytes % 16 == 0;
  };
  const bool cplx = dt == TGD_C64 || dt == TGD_C32H;
  auto fits = [&](int kc, int ns) { return tg_smem_bytes(I, kc, es, ns, g.parts, cplx) <= TG_SMEM_LIMIT; };
  // (a 64-column block of I <= 32 rows needs at most 65 of the mask words)
  if (I <= 32 && g.B < TG_COLS && slabs_ok(TG_KC_MAX) && fits(TG_KC_MAX, 2)) {
    g.mode = TG_SLABS;
    g.kc = TG_KC_MAX;
  } else if (slabs_ok(g.kc)) {
    g.mode = TG_SLABS;
  } else if (aligned16 && tma_ok && g.B % g.kc == 0) {
    g.mode = TG_ROWS;
  } else {
    g.mode = TG_ELEMS;
  }
  if (g.mode == TG_SLABS) {
    g.slabs = (int)(g.kc / g.B);
    g.nchunk = ceil_div(g.A, (int64_t)g.slabs);
  } else if (g.mode == TG_ROWS) {
    g.nchunk = g.A * g.B / g.kc;
  } else {
    g.nchunk = ceil_div(g.A * g.B, (int64_t)g.kc);
  }
  g.ns = TG_NS_MAX;
  while (g.ns > 2 && !fits(g.kc, g.ns)) --g.ns;
  const int cap = max_splits > 0 && max_splits < TG_MAX_SPLITS ? max_splits : TG_MAX_SPLITS;
  const int64_t ns = std::max<int64_t>(1, std::min<int64_t>(cap, g.nchunk));
  g.chunks_per_split = ceil_div(g.nchunk, ns);
  g.nsplit = (int)ceil_div(g.nchunk, g.chunks_per_split);
  return g;
}

// ------------------------------------------------------------- eigensolver
__device__ __forceinline__ double2 zmul(double2 a, double2 b) {
  return make_double2(a.x * b.x - a.y * b.y, a.x * b.y + a.y * b.x);
}
__device__ __forceinline__ double zabs2(double2 a) { return a.x * a.x + a.y * a.y; }

constexpr int ET = 1024;  // threads per eigensolver block
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

// Block-wide maximum (every thread gets it); red as for block_sum.
__device__ double block_max(double v, double* red) {
  for (int o = 16; o; o >>= 1) v = fmax(v, __shfl_xor_sync(0xffffffffu, v, o));
  __syncthreads();
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = v;
  __syncthreads();
  double m = -INFINITY;
  for (int w = 0; w < (int)(blockDim.x >> 5); ++w) m = fmax(m, red[w]);
  __syncthreads();
  return m;
}

// Hermitian Jacobi for n <= 256: two-sided rotations in the round-robin
// parallel ordering (n/2 disjoint pairs per round). A and the eigenvector
// rows Vt are both whole, with an odd row pitch (a column walk by 32 lanes
// touches 32 different banks), in shared memory for n <= 64 and in the job's
// global scratch above that. A round applies its rotations to A on 2 x 2
// blocks of pairs, a thread per block (each entry is read and written once,
// the mirror half from the upper one), and to V a warp per pair.
constexpr int ES_MAXN = MAXN;
// Off-diagonal mass, relative to |A|_F^2, below which the rotations stop:
// entries under 1e-9 |A|_F move the eigenvectors by less than the Gram's own
// error (fp32 accumulation, ~1e-7 relative), and the eigenvalues by their
// square.
constexpr double JAC_TOL = 1e-18;
constexpr int ES_SMEM_MAXN = 64;

__global__ void __launch_bounds__(ET) eig_small_kernel(const EigJobs jobs) {
  const EigJob J = jobs.j[blockIdx.x];
  const int n = J.n;
  if (n > ES_MAXN) return;
  const int NP = n + 1 + (n & 1);  // odd row pitch
  extern __shared__ double2 dyn[];
  const bool in_smem = n <= ES_SMEM_MAXN;
  double2* scratch = (double2*)J.work;
  double2* A = in_smem ? dyn : scratch;                            // [n][NP]
  double2* Vt = in_smem ? dyn + n * NP : scratch + (size_t)n * NP;  // [n][NP]: row k = eigenvector k
  __shared__ int rp[ES_MAXN / 2], rq[ES_MAXN / 2], rrot[ES_MAXN / 2];
  __shared__ double rcs[ES_MAXN / 2], rsn[ES_MAXN / 2];
  __shared__ double2 rph[ES_MAXN / 2];
  __shared__ double red[ET / 32];
  __shared__ double ev[ES_MAXN];
  __shared__ int col_of_rank[ES_MAXN];
  __shared__ uint8_t lead[ES_MAXN];
  __shared__ uint8_t bk1[ES_MAXN / 2 * (ES_MAXN / 2 + 1) / 2], bk2[ES_MAXN / 2 * (ES_MAXN / 2 + 1) / 2];
  const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5, nw = blockDim.x >> 5;
  const double2* G = (const double2*)J.gram;
  if (J.warm) {
    // Start from the previous refresh's eigenvectors V (rows of Vt): A =
    // V^H G V is nearly diagonal when the subspaces move little between
    // refreshes. Jacobi converges from any unitary start.
    const double2* Vp = (const double2*)J.vprev;
    double2* W = scratch + (size_t)2 * n * NP;  // W = G V (n x n)
    for (int e = tid; e < n * n; e += blockDim.x) {
      const int k = e / n, i = e - k * n;
      Vt[k * NP + i] = Vp[e];
    }
    __syncthreads();
    for (int e = tid; e < n * n; e += blockDim.x) {
      const int i = e / n, l = e - i * n;
      double2 acc = make_double2(0.0, 0.0);
      for (int j = 0; j < n; ++j) {
        const double2 g = G[i * n + j], v = Vt[l * NP + j];
        acc.x += g.x * v.x - g.y * v.y;
        acc.y += g.x * v.y + g.y * v.x;
      }
      W[e] = acc;
    }
    __syncthreads();
    for (int e = tid; e < n * n; e += blockDim.x) {
      const int k = e / n, l = e - k * n;
      if (l < k) continue;
      double2 acc = make_double2(0.0, 0.0);  // sum_i conj(V[i][k]) W[i][l]
      for (int i = 0; i < n; ++i) {
        const double2 v = Vt[k * NP + i], w = W[i * n + l];
        acc.x += v.x * w.x + v.y * w.y;
        acc.y += v.x * w.y - v.y * w.x;
      }
      if (l == k) acc.y = 0.0;  // Hermitian: a real diagonal
      A[k * NP + l] = acc;
      A[l * NP + k] = make_double2(acc.x, -acc.y);
    }
  } else {
    for (int e = tid; e < n * n; e += blockDim.x) {
      const int i = e / n, j = e - i * n;
      // the upper triangle of G, mirrored (G is Hermitian up to rounding)
      const double2 g = i <= j ? G[i * n + j] : G[j * n + i];
      A[i * NP + j] = i <= j ? g : make_double2(g.x, -g.y);
      if (i == j) A[i * NP + j].y = 0.0;
      Vt[i * NP + j] = make_double2(i == j ? 1.0 : 0.0, 0.0);
    }
  }
  __syncthreads();
  double part = 0;
  for (int e = tid; e < n * n; e += blockDim.x) {
    const int i = e / n, j = e - i * n;
    part += zabs2(A[i * NP + j]);
  }
  const double fro = block_sum(part, red);
  const int m = n + (n & 1);
  const int npairs = m / 2;
  // the 2 x 2 blocks of pairs (k1 <= k2), row by row
  const int nblk = npairs * (npairs + 1) / 2;
  for (int b = tid; b < nblk; b += blockDim.x) {
    int k1 = 0, rr = b;
    while (rr >= npairs - k1) {
      rr -= npairs - k1;
      ++k1;
    }
    bk1[b] = (uint8_t)k1;
    bk2[b] = (uint8_t)(k1 + rr);
  }
  __syncthreads();
  const int r = J.r;
  for (int sweep = 0; sweep < 40; ++sweep) {
    // Stop when A is diagonal to JAC_TOL of its squared Frobenius norm, or
    // when the r rows of the largest diagonal entries are (their off-diagonal
    // mass below the same bound: those diagonal entries and rows of Vt are
    // eigenpairs) and a Gershgorin bound puts every eigenvalue of the other
    // rows' block below the smallest of them (so they are the r leading).
    for (int i = tid; i < n; i += blockDim.x) {
      const double di = A[i * NP + i].x;
      int rank = 0;
      for (int j = 0; j < n; ++j) {
        const double dj = A[j * NP + j].x;
        rank += (dj > di) || (dj == di && j < i);
      }
      lead[i] = rank < r;
    }
    __syncthreads();
    double off_part = 0, lead_part = 0, ger_part = -INFINITY, low_part = INFINITY;
    for (int i = wid; i < n; i += nw) {
      double row = 0, rad = 0;
      for (int j = lane; j < n; j += 32) {
        if (j == i) continue;
        const double a2 = zabs2(A[i * NP + j]);
        row += a2;
        if (!lead[j]) rad += sqrt(a2);
      }
      for (int o = 16; o; o >>= 1) {
        row += __shfl_xor_sync(0xffffffffu, row, o);
        rad += __shfl_xor_sync(0xffffffffu, rad, o);
      }
      if (lane == 0) {
        const double di = A[i * NP + i].x;
        off_part += row;
        if (lead[i]) {
          lead_part += row;
          low_part = fmin(low_part, di);
        } else {
          ger_part = fmax(ger_part, di + rad);
        }
      }
    }
    const double off = block_sum(off_part, red);
    const double lead_off = block_sum(lead_part, red);
    const double ger = block_max(ger_part, red);
    const double low = -block_max(-low_part, red);
    if (off <= JAC_TOL * fro || off == 0.0) break;
    // (the rows' coupling, at most sqrt(lead_off), moves no eigenvalue further)
    if (r < n && lead_off <= JAC_TOL * fro && ger + 2.0 * sqrt(lead_off) < low) break;
    for (int round = 0; round < m - 1; ++round) {
      // the round's disjoint pairs (round-robin) and their rotations
      for (int k = tid; k < npairs; k += blockDim.x) {
        int p, q;
        if (k == 0) {
          p = round;
          q = m - 1;
        } else {
          p = (round + k) % (m - 1);
          q = (round - k + (m - 1)) % (m - 1);
        }
        if (p > q) {
          const int t = p;
          p = q;
          q = t;
        }
        rp[k] = p;
        rq[k] = q;
        rrot[k] = 0;
        if (q < n) {  // the dummy index of odd n is absent
          const double2 apq = A[p * NP + q];
          const double r2 = zabs2(apq);
          if (r2 > 0.0) {
            // the same rotation with one reciprocal square root per quantity:
            // 1/r, then t = sign(tau) / (|tau| + sqrt(1 + tau^2)), c = 1/sqrt(1 + t^2)
            const double app = A[p * NP + p].x, aqq = A[q * NP + q].x;
            const double rinv = rsqrt(r2);
            const double tau = (aqq - app) * 0.5 * rinv;
            const double t = (tau >= 0 ? 1.0 : -1.0) / (fabs(tau) + sqrt(1.0 + tau * tau));
            const double c = rsqrt(1.0 + t * t);
            rrot[k] = 1;
            rcs[k] = c;
            rsn[k] = t * c;
            rph[k] = make_double2(apq.x * rinv, apq.y * rinv);
          }
        }
      }
      __syncthreads();
      // A <- J^H A J on 2 x 2 blocks of pairs (k1 <= k2): a thread reads the
      // block's four entries once, applies J_k2 to its columns and J_k1^H to
      // its rows, and writes it and its mirror (A is Hermitian); the diagonal
      // blocks come out with (p, q) zero and a real diagonal
      for (int b = tid; b < nblk; b += blockDim.x) {
        const int k1 = bk1[b], k2 = bk2[b];
        const bool rot1 = rrot[k1], rot2 = rrot[k2];
        if (!rot1 && !rot2) continue;
        const int p1 = rp[k1], q1 = rq[k1], p2 = rp[k2], q2 = rq[k2];
        const bool h1 = q1 < n, h2 = q2 < n;  // the dummy index of odd n is absent
        const double2 z = make_double2(0.0, 0.0);
        double2 b00 = A[p1 * NP + p2], b01 = h2 ? A[p1 * NP + q2] : z;
        double2 b10 = h1 ? A[q1 * NP + p2] : z, b11 = h1 && h2 ? A[q1 * NP + q2] : z;
        if (rot2) {
          const double c = rcs[k2], s = rsn[k2];
          const double2 ec = make_double2(rph[k2].x, -rph[k2].y);
          double2 xp = b00, xq = zmul(b01, ec);
          b00 = make_double2(c * xp.x - s * xq.x, c * xp.y - s * xq.y);
          b01 = make_double2(s * xp.x + c * xq.x, s * xp.y + c * xq.y);
          xp = b10;
          xq = zmul(b11, ec);
          b10 = make_double2(c * xp.x - s * xq.x, c * xp.y - s * xq.y);
          b11 = make_double2(s * xp.x + c * xq.x, s * xp.y + c * xq.y);
        }
        if (rot1) {
          const double c = rcs[k1], s = rsn[k1];
          const double2 e = rph[k1];
          double2 xp = b00, xq = zmul(b10, e);
          b00 = make_double2(c * xp.x - s * xq.x, c * xp.y - s * xq.y);
          b10 = make_double2(s * xp.x + c * xq.x, s * xp.y + c * xq.y);
          xp = b01;
          xq = zmul(b11, e);
          b01 = make_double2(c * xp.x - s * xq.x, c * xp.y - s * xq.y);
          b11 = make_double2(s * xp.x + c * xq.x, s * xp.y + c * xq.y);
        }
        if (k1 == k2) {
          A[p1 * NP + p1] = make_double2(b00.x, 0.0);
          if (h1) {
            A[p1 * NP + q1] = z;
            A[q1 * NP + p1] = z;
            A[q1 * NP + q1] = make_double2(b11.x, 0.0);
          }
        } else {
          A[p1 * NP + p2] = b00;
          A[p2 * NP + p1] = make_double2(b00.x, -b00.y);
          if (h2) {
            A[p1 * NP + q2] = b01;
            A[q2 * NP + p1] = make_double2(b01.x, -b01.y);
          }
          if (h1) {
            A[q1 * NP + p2] = b10;
            A[p2 * NP + q1] = make_double2(b10.x, -b10.y);
          }
          if (h1 && h2) {
            A[q1 * NP + q2] = b11;
            A[q2 * NP + q1] = make_double2(b11.x, -b11.y);
          }
        }
      }
      // V <- V J on the rows of Vt, a warp per pair
      for (int k = wid; k < npairs; k += nw) {
        if (!rrot[k]) continue;
        const int p = rp[k], q = rq[k];
        const double c = rcs[k], s = rsn[k];
        const double2 ec = make_double2(rph[k].x, -rph[k].y);
        for (int i = lane; i < n; i += 32) {
          const double2 xp = Vt[p * NP + i], xq = zmul(Vt[q * NP + i], ec);
          Vt[p * NP + i] = make_double2(c * xp.x - s * xq.x, c * xp.y - s * xq.y);
          Vt[q * NP + i] = make_double2(s * xp.x + c * xq.x, s * xp.y + c * xq.y);
        }
      }
      __syncthreads();
    }
  }
  for (int i = tid; i < n; i += blockDim.x) ev[i] = A[i * NP + i].x;
  __syncthreads();
  for (int i = tid; i < n; i += blockDim.x) {
    const double li = ev[i];
    int rank = 0;
    for (int j = 0; j < n; ++j) rank += (ev[j] > li) || (ev[j] == li && j < i);
    col_of_rank[rank] = i;
    J.evals[rank] = li;
  }
  __syncthreads();
  // the leading r vectors, each scaled by the unit phase that makes its
  // largest-magnitude entry (ties to the lowest row) real and positive
  for (int rr = wid; rr < J.r; rr += nw) {
    const int c = col_of_rank[rr];
    double best = -1.0;
    int bi = 0;
    for (int row = lane; row < n; row += 32) {
      const double mg = zabs2(Vt[c * NP + row]);
      if (mg > best) {
        best = mg;
        bi = row;
      }
    }
    for (int o = 16; o; o >>= 1) {
      const double ob = __shfl_xor_sync(0xffffffffu, best, o);
      const int oi = __shfl_xor_sync(0xffffffffu, bi, o);
      if (ob > best || (ob == best && oi < bi)) {
        best = ob;
        bi = oi;
      }
    }
    const double2 piv = Vt[c * NP + bi];
    const double pm = sqrt(zabs2(piv));
    const double2 ph = pm > 0 ? make_double2(piv.x / pm, -piv.y / pm) : make_double2(1.0, 0.0);
    for (int row = lane; row < n; row += 32) {
      const double2 u = zmul(Vt[c * NP + row], ph);
      ((float2*)J.U)[(int64_t)row * J.r + rr] = make_float2((float)u.x, (float)u.y);
    }
  }
  // the eigenvectors, the start of the next refresh
  if (J.vprev)
    for (int e = tid; e < n * n; e += blockDim.x) {
      const int k = e / n, i = e - k * n;
      ((double2*)J.vprev)[e] = Vt[k * NP + i];
    }
}

// ------------------------------------------------------- DCT column selection
// The dynamic column selection of the Trion / DCT-AdamW page as a factor
// basis: thread j holds column q_j of the orthonormal DCT matrix (entry (k, j)
// = sqrt(2/n) cos(k (2j+1) pi / (2n)), row 0 divided by sqrt 2) and forms its
// alignment q_j^T Re(Gram) q_j in fp64; the columns are ranked by descending
// alignment (ties to the lower column) and the first r written to U.
constexpr int DCT_MAXN = 256;

__global__ void __launch_bounds__(DCT_MAXN) dct_select_kernel(const EigJobs jobs) {
  const EigJob J = jobs.j[blockIdx.x];
  const int n = J.n;
  __shared__ double score[DCT_MAXN];
  __shared__ int col_of_rank[DCT_MAXN];
  const int j = threadIdx.x;
  const double2* G = (const double2*)J.gram;
  if (j < n) {
    double q[DCT_MAXN];
    const double theta = (2.0 * j + 1.0) * M_PI / (2.0 * n);
    for (int k = 0; k < n; ++k) q[k] = sqrt((k == 0 ? 1.0 : 2.0) / n) * cos(k * theta);
    double sc = 0;
    for (int a = 0; a < n; ++a) {
      double t = 0;
      for (int b = 0; b < n; ++b) t += G[(int64_t)a * n + b].x * q[b];
      sc += q[a] * t;
    }
    score[j] = sc;
  }
  __syncthreads();
  if (j < n) {
    const double sj = score[j];
    int rank = 0;
    for (int i = 0; i < n; ++i) rank += (score[i] > sj) || (score[i] == sj && i < j);
    col_of_rank[rank] = j;
    J.evals[rank] = sj;
  }
  __syncthreads();
  for (int e = threadIdx.x; e < n * J.r; e += blockDim.x) {
    const int row = e / J.r, c = e - row * J.r;
    const int col = col_of_rank[c];
    const double v = sqrt((row == 0 ? 1.0 : 2.0) / n) * cos(row * (2.0 * col + 1.0) * M_PI / (2.0 * n));
    ((float2*)J.U)[e] = make_float2((float)v, 0.f);
  }
}

}  // namespace

cudaError_t batched_dct_select(const EigJob* jobs_host, int njobs, cudaStream_t s) {
  if (njobs <= 0) return cudaSuccess;
  if (njobs > TGD_MAX_NDIM) return cudaErrorInvalidValue;
  EigJobs jobs{};
  for (int j = 0; j < njobs; ++j) {
    if (jobs_host[j].n > DCT_MAXN || jobs_host[j].r > jobs_host[j].n) return cudaErrorInvalidValue;
    jobs.j[j] = jobs_host[j];
  }
  dct_select_kernel<<<njobs, DCT_MAXN, 0, s>>>(jobs);
  return cudaGetLastError();
}

size_t gram_partial_bytes(int nd, const int64_t* dims, int n) {
  GramGeom g = gram_geom(nd, dims, n);
  size_t b = sizeof(float2) * (size_t)g.nsplit * g.I * g.I;
  if (g.I <= 128) b = std::max(b, sizeof(float2) * (size_t)TG_MAX_SPLITS * g.I * g.I);
  // the small-mode Gram: at most 8 CTAs per SM of up to 256 SMs
  if (g.I <= 32) b = std::max(b, sizeof(float2) * (size_t)(8 * 256) * g.I * g.I);
  return b;
}

// The driver's tensor-map encoder, looked up once through the runtime (the
// library does not link the driver library itself).
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
static EncodeTiledFn encode_tiled() {
  static EncodeTiledFn fn = nullptr;
  static bool tried = false;
  if (!tried) {
    tried = true;
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = (EncodeTiledFn)f;
  }
  return fn;
}

// Tensor map of the unfolding [A][I][B] for TG_ROWS: boxes of 32 columns x
// I rows of one slab (8-byte elements as pairs of 4-byte ones).
static cudaError_t rows_tensor_map(CUtensorMap* map, const void* g, int es, const TcGramGeom& t) {
  EncodeTiledFn fn = encode_tiled();
  if (!fn) return cudaErrorNotSupported;
  const int ue = es == 8 ? 4 : es;  // unit element bytes
  const int per = es / ue;
  const cuuint64_t dim[3] = {(cuuint64_t)(t.B * per), (cuuint64_t)t.I, (cuuint64_t)t.A};
  const cuuint64_t stride[2] = {(cuuint64_t)(t.B * es), (cuuint64_t)(t.I * t.B * es)};
  // 128-byte box rows, swizzled (see tg_soff); 2-byte elements: 64-byte rows as they are
  const cuuint32_t box[3] = {(cuuint32_t)(es == 8 ? 32 : TG_COLS), (cuuint32_t)t.I, 1};
  const CUtensorMapSwizzle swz = es == 2 ? CU_TENSOR_MAP_SWIZZLE_NONE : CU_TENSOR_MAP_SWIZZLE_128B;
  const cuuint32_t estr[3] = {1, 1, 1};
  const CUtensorMapDataType type = ue == 4 ? CU_TENSOR_MAP_DATA_TYPE_UINT32 : CU_TENSOR_MAP_DATA_TYPE_UINT16;
  const CUresult r = fn(map, type, 3, const_cast<void*>(g), dim, stride, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                        swz, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

// ---------------------------------------------- small-mode Gram, CUDA cores
// Modes with I_n <= 32 whose slab (I_n x B, contiguous) is small: the Gram
// needs 4 I_n fp32 FMAs per complex element at most (I_n <= 32), which the
// CUDA cores sustain at the rate G streams in, while a tensor-core Gram of
// such a mode is bound by its MMA count (a 128-row tile mostly padding).
// A CTA takes a range of chunks of whole slabs: each chunk arrives by one
// bulk copy (plain loads for a tail or an unaligned tensor) with Omega's
// mask words beside it (cp.async), Omega's entries are zeroed in shared
// memory, and thread (tile pair, column lane) accumulates the 4 x 4 block
// (ti <= tj) of sum_c x_i(c) conj(x_j(c)) over its columns c = lane, lane +
// CL, ... of the chunk (CL = 16 column lanes a pair up to I_n = 16, 8 above,
// so that two CTAs fit an SM). At the end the column lanes of a pair are
// summed by shuffles and the CTA writes its whole I_n x I_n partial (the
// lower blocks as conjugates), which the fixed-order fp64 reduction sums.
constexpr int SG_CL = 16;      // column lanes per tile pair, at most
constexpr int SG_MAXI = 32;    // I_n at most
constexpr int SG_MAXT = 36 * SG_CL;  // threads: tile pairs of I_n = 32 (8 x 9 / 2) x lanes
constexpr int SG_CHUNK = 32768;      // bytes of a chunk, at most (two in flight)

struct SmallGramArgs {
  const void* g;
  const uint32_t* bits;
  int64_t A, B;        // slabs, columns per slab row
  int I, IP, ntp;      // rows, 4-row tiles, tile pairs
  int cl;              // column lanes per tile pair (8 or 16)
  int spc;             // slabs per chunk
  int64_t nchunk, cpc; // chunks, chunks per CTA
  int bulk;            // whole chunks by bulk copy (aligned tensor, chunk bytes % 16 == 0)
  float2* partial;     // [gridDim.x][I][I]
  int* err;
};

template <int DT>
__global__ void __launch_bounds__(SG_MAXT) gram_small_kernel(const SmallGramArgs p) {
  constexpr int ES = Dt<DT>::bytes;
  extern __shared__ __align__(128) uint8_t sg_smem[];
  __shared__ __align__(8) uint64_t bar[2];
  __shared__ int s_abort;
  const int tid = threadIdx.x, nthr = blockDim.x;
  const int64_t IB = (int64_t)p.I * p.B;
  const int64_t chunk_elems = (int64_t)p.spc * IB;
  const size_t xbytes = (size_t)((chunk_elems * ES + 127) / 128) * 128;
  const size_t mbytes = (size_t)((4 * (chunk_elems / 32 + 2) + 127) / 128) * 128;
  // two buffers: the chunk (raw) and its mask words
  auto xbuf = [&](int b) { return sg_smem + (size_t)b * (xbytes + mbytes); };
  auto mwb = [&](int b) { return (uint32_t*)(sg_smem + (size_t)b * (xbytes + mbytes) + xbytes); };
  // this thread's tile pair (ti <= tj) and column lane
  const int CL = p.cl;
  const int pi = tid / CL, lc = tid - pi * CL;
  int ti = 0, rem = pi;
  while (rem >= p.IP - ti) {
    rem -= p.IP - ti;
    ++ti;
  }
  const int tj = ti + rem;
  const bool active = pi < p.ntp;
  float2 acc[4][4];
#pragma unroll
  for (int u = 0; u < 4; ++u)
#pragma unroll
    for (int v = 0; v < 4; ++v) acc[u][v] = make_float2(0.f, 0.f);
  if (tid == 0) {
    s_abort = 0;
    ptx::mbar_init(&bar[0], 1);
    ptx::mbar_init(&bar[1], 1);
    ptx::fence_mbar_init();
  }
  __syncthreads();
  const int64_t c_begin = (int64_t)blockIdx.x * p.cpc;
  const int64_t c_end = c_begin + p.cpc < p.nchunk ? c_begin + p.cpc : p.nchunk;
  auto geom = [&](int64_t ch, int& nsl, int64_t& e0, int64_t& ne, int64_t& w0, int64_t& nw) {
    const int64_t a0 = ch * p.spc;
    nsl = (int)(p.A - a0 < p.spc ? p.A - a0 : p.spc);
    e0 = a0 * IB;
    ne = (int64_t)nsl * IB;
    w0 = e0 >> 5;
    nw = p.bits ? ((e0 + ne - 1) >> 5) - w0 + 1 : 0;
  };
  // chunk ch into buffer b: mask words by cp.async (their arrivals counted
  // before the copy's), then the chunk by one bulk copy, or by plain loads
  // (a tail chunk or an unaligned tensor)
  auto issue = [&](int64_t ch, int b) {
    int nsl;
    int64_t e0, ne, w0, nw;
    geom(ch, nsl, e0, ne, w0, nw);
    const bool whole = p.bulk && nsl == p.spc;
    uint32_t* mw = mwb(b);
    uint8_t* xb = xbuf(b);
    for (int64_t w = tid; w < nw; w += nthr) cp_async_elem<4>(mw + w, p.bits + w0 + w);
    if (!whole) {
      for (int64_t e = tid; e < ne; e += nthr) {
        if constexpr (ES == 8)
          ((uint2*)xb)[e] = __ldg((const uint2*)p.g + e0 + e);
        else if constexpr (ES == 4)
          ((uint32_t*)xb)[e] = __ldg((const uint32_t*)p.g + e0 + e);
        else
          ((uint16_t*)xb)[e] = __ldg((const unsigned short*)p.g + e0 + e);
      }
    }
    cp_async_arrive(&bar[b]);
    __syncthreads();
    if (tid == 0) {
      if (whole) {
        ptx::mbar_expect_tx(&bar[b], (uint32_t)(ne * ES));
        ptx::bulk_g2s(xb, (const uint8_t*)p.g + e0 * ES, (uint32_t)(ne * ES), &bar[b]);
      } else {
        tg_arrive(&bar[b]);
      }
    }
  };
  uint32_t phbits = 0;  // bit b: the parity buffer b's next phase completes with
  int64_t issued = 0;
  if (c_begin < c_end) {
    issue(c_begin, 0);
    issued = 1;
  }
  for (int64_t ch = c_begin; ch < c_end; ++ch) {
    const int b = (int)((ch - c_begin) & 1);
    // the next chunk goes into the other buffer (read out by the barrier
    // that ended the previous iteration)
    if (ch + 1 < c_end) {
      issue(ch + 1, b ^ 1);
      ++issued;
    }
    if (tid == 0 && !ptx::mbar_wait(&bar[b], (phbits >> b) & 1u, TG_WAIT_NS)) {
      atomicOr(p.err, DEV_ERR_TIMEOUT);
      s_abort = 1;
    }
    phbits ^= 1u << b;
    __syncthreads();
    if (s_abort) break;
    int nsl;
    int64_t e0, ne, w0, nw;
    geom(ch, nsl, e0, ne, w0, nw);
    uint8_t* xb = xbuf(b);
    const uint32_t* mw = mwb(b);
    // Omega's entries of the chunk -> zero (the residual)
    for (int64_t w = tid; w < nw; w += nthr) {
      uint32_t word = mw[w];
      const int64_t base = (w0 + w) * 32 - e0;
      while (word) {
        const int bt = __ffs(word) - 1;
        word &= word - 1;
        const int64_t e = base + bt;
        if (e >= 0 && e < ne) {
          if constexpr (ES == 8)
            ((uint2*)xb)[e] = make_uint2(0u, 0u);
          else if constexpr (ES == 4)
            ((uint32_t*)xb)[e] = 0u;
          else
            ((uint16_t*)xb)[e] = 0;
        }
      }
    }
    __syncthreads();
    if (active) {
      const int64_t ncol = (int64_t)nsl * p.B;
      int64_t al = lc / p.B, bb = lc - al * p.B;
      const int64_t dA = CL / p.B, dB = CL - dA * p.B;  // a step of CL columns
      for (int64_t c = lc; c < ncol; c += CL) {
        const int64_t base = al * IB + bb;
        float2 xa[4], xc[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const int i = 4 * ti + u;
          xa[u] = i < p.I ? load_rw<DT>(xb, base + (int64_t)i * p.B) : make_float2(0.f, 0.f);
        }
        if (tj == ti) {
#pragma unroll
          for (int v = 0; v < 4; ++v) xc[v] = xa[v];
        } else {
#pragma unroll
          for (int v = 0; v < 4; ++v) {
            const int jj = 4 * tj + v;
            xc[v] = jj < p.I ? load_rw<DT>(xb, base + (int64_t)jj * p.B) : make_float2(0.f, 0.f);
          }
        }
#pragma unroll
        for (int u = 0; u < 4; ++u)
#pragma unroll
          for (int v = 0; v < 4; ++v) {
            // xa * conj(xc)
            acc[u][v].x = __fmaf_rn(xa[u].x, xc[v].x, acc[u][v].x);
            if constexpr (Dt<DT>::cplx) {
              acc[u][v].x = __fmaf_rn(xa[u].y, xc[v].y, acc[u][v].x);
              acc[u][v].y = __fmaf_rn(xa[u].y, xc[v].x, __fmaf_rn(-xa[u].x, xc[v].y, acc[u][v].y));
            }
          }
        bb += dB;
        al += dA;
        if (bb >= p.B) {
          bb -= p.B;
          ++al;
        }
      }
    }
    __syncthreads();  // this buffer is read before it is refilled
  }
  // the 16 column lanes of each pair (aligned lanes of one warp), summed
#pragma unroll
  for (int u = 0; u < 4; ++u)
#pragma unroll
    for (int v = 0; v < 4; ++v)
#pragma unroll
      for (int o = 8; o; o >>= 1) {
        if (o >= CL) continue;
        acc[u][v].x += __shfl_xor_sync(0xffffffffu, acc[u][v].x, o);
        acc[u][v].y += __shfl_xor_sync(0xffffffffu, acc[u][v].y, o);
      }
  if (active && lc == 0) {
    float2* out = p.partial + (int64_t)blockIdx.x * p.I * p.I;
#pragma unroll
    for (int u = 0; u < 4; ++u)
#pragma unroll
      for (int v = 0; v < 4; ++v) {
        const int i = 4 * ti + u, jj = 4 * tj + v;
        if (i < p.I && jj < p.I) {
          out[(int64_t)i * p.I + jj] = acc[u][v];
          if (ti != tj) out[(int64_t)jj * p.I + i] = make_float2(acc[u][v].x, -acc[u][v].y);
        }
      }
  }
  if (tid == 0 && s_abort) {
    // bounded waits for the copies still in flight (both buffers' last phases)
    for (int b = 0; b < 2; ++b)
      if ((int64_t)b < issued) ptx::mbar_wait(&bar[b], (phbits >> b) & 1u, TG_WAIT_NS / 4);
  }
}

// The small-mode Gram's plan, or false when the mode does not fit it.
bool small_gram_plan(int nd, const int64_t* dims, int n, int dt, bool aligned16, int max_ctas, SmallGramArgs& a,
                     size_t& smem, int& threads) {
  const int es = dt == TGD_C64 ? 8 : (dt == TGD_R16 ? 2 : 4);
  int64_t A = 1, B = 1;
  for (int q = 0; q < n; ++q) A *= dims[q];
  for (int q = n + 1; q < nd; ++q) B *= dims[q];
  const int I = (int)dims[n];
  if (I > SG_MAXI || I < 1) return false;
  const int64_t slab = (int64_t)I * B * es;
  if (slab > SG_CHUNK) return false;
  // slabs per chunk: as many as fit, a multiple of what keeps chunks 16-byte sized
  int step = 1;
  while ((slab * step) % 16 != 0 && step < 16) step *= 2;
  int spc = (int)(SG_CHUNK / slab) / step * step;
  if (spc < step) spc = step;
  if (spc > A) spc = (int)A;
  a.A = A;
  a.B = B;
  a.I = I;
  a.IP = (I + 3) / 4;
  a.ntp = a.IP * (a.IP + 1) / 2;
  a.cl = a.IP > 4 ? 8 : SG_CL;
  a.spc = spc;
  a.nchunk = ceil_div(A, (int64_t)spc);
  a.bulk = aligned16 && (slab * spc) % 16 == 0;
  threads = a.ntp * a.cl;
  const int64_t chunk_elems = (int64_t)spc * I * B;
  smem = 2 * ((size_t)((chunk_elems * es + 127) / 128) * 128 + (size_t)((4 * (chunk_elems / 32 + 2) + 127) / 128) * 128);
  // CTAs: as many as the SMs hold (threads and shared memory), each at least
  // two chunks
  int dev = 0, nsm = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev);
  if (max_ctas > 0 && max_ctas < nsm) nsm = max_ctas;
  // resident CTAs per SM: threads, shared memory and registers (up to 96 a thread)
  int per = std::min(2048 / threads, (int)(220 * 1024 / (smem + 1024)));
  per = std::min(per, 65536 / (threads * 96));
  per = std::max(1, std::min(per, 8));
  const int64_t want = std::max<int64_t>(1, std::min<int64_t>((int64_t)nsm * per, ceil_div(a.nchunk, (int64_t)2)));
  a.cpc = ceil_div(a.nchunk, want);
  return true;
}

int small_gram_ctas(const SmallGramArgs& a) { return (int)ceil_div(a.nchunk, a.cpc); }

// Tensor-core Gram for I_n <= 64 (see gram_tc_kernel); the split partials are
// summed by the same fixed-order fp64 reduction.
cudaError_t mode_gram_tc(const void* g, int dt, const uint32_t* bits, int nd, const int64_t* dims,
                         int n, float* partial, double* gram, int* err, cudaStream_t s, int max_ctas) {
  const int es = dt == TGD_C64 ? 8 : (dt == TGD_R16 ? 2 : 4);
  const TcGramGeom t = tc_gram_geom(nd, dims, n, dt, ((uintptr_t)g & 15) == 0, max_ctas);
  TcGramArgs a;
  a.g = g;
  a.bits = bits;
  a.A = t.A;
  a.I = t.I;
  a.B = t.B;
  a.nchunk = t.nchunk;
  a.chunks_per_split = t.chunks_per_split;
  a.mode = t.mode;
  a.slabs = t.slabs;
  a.kc = t.kc;
  a.ns = t.ns;
  a.parts = t.parts;
  a.partial = partial;
  a.err = err;
  CUtensorMap map;
  memset(&map, 0, sizeof(map));
  if (t.mode == TG_ROWS) {
    const cudaError_t e = rows_tensor_map(&map, g, es, t);
    if (e != cudaSuccess) return e;
  }
  const size_t smem = tg_smem_bytes((int)t.I, t.kc, es, t.ns, t.parts, dt == TGD_C64 || dt == TGD_C32H);
  if (smem > TG_SMEM_LIMIT) return cudaErrorInvalidValue;
  const dim3 grid(t.nsplit);
  cudaError_t e = cudaSuccess;
  switch (dt) {
    case TGD_R32:
      e = cudaFuncSetAttribute(gram_tc_kernel<TGD_R32>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
      if (e == cudaSuccess) gram_tc_kernel<TGD_R32><<<grid, TG_THREADS, smem, s>>>(a, map);
      break;
    case TGD_C64:
      e = cudaFuncSetAttribute(gram_tc_kernel<TGD_C64>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
      if (e == cudaSuccess) gram_tc_kernel<TGD_C64><<<grid, TG_THREADS, smem, s>>>(a, map);
      break;
    case TGD_C32H:
      e = cudaFuncSetAttribute(gram_tc_kernel<TGD_C32H>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
      if (e == cudaSuccess) gram_tc_kernel<TGD_C32H><<<grid, TG_THREADS, smem, s>>>(a, map);
      break;
    case TGD_R16:
      e = cudaFuncSetAttribute(gram_tc_kernel<TGD_R16>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
      if (e == cudaSuccess) gram_tc_kernel<TGD_R16><<<grid, TG_THREADS, smem, s>>>(a, map);
      break;
    default:
      return cudaErrorInvalidValue;
  }
  if (e != cudaSuccess) return e;
  GramGeom geo{};
  geo.I = t.I;
  geo.TI = 64;  // one tile: every cell is computed directly
  geo.nsplit = t.nsplit;
  const int64_t cells = t.I * t.I;
  gram_reduce_kernel<<<(int)ceil_div(cells, RC), RC * RS, 0, s>>>((const float2*)partial, geo,
                                                                   (double2*)gram);
  return cudaGetLastError();
}

cudaError_t mode_gram(const void* g, int dt, const uint32_t* bits, int nd, const int64_t* dims,
                      int n, float* partial, double* gram, int* err, cudaStream_t s, int max_ctas) {
  {
    SmallGramArgs a{};
    size_t smem = 0;
    int threads = 0;
    if (small_gram_plan(nd, dims, n, dt, ((uintptr_t)g & 15) == 0, max_ctas, a, smem, threads)) {
      a.g = g;
      a.bits = bits;
      a.partial = (float2*)partial;
      a.err = err;
      const int grid = small_gram_ctas(a);
      auto launch = [&](auto kern) -> cudaError_t {
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
        kern<<<grid, threads, smem, s>>>(a);
        return cudaGetLastError();
      };
      cudaError_t e = cudaErrorInvalidValue;
      switch (dt) {
        case TGD_R32:
          e = launch(gram_small_kernel<TGD_R32>);
          break;
        case TGD_C64:
          e = launch(gram_small_kernel<TGD_C64>);
          break;
        case TGD_C32H:
          e = launch(gram_small_kernel<TGD_C32H>);
          break;
        case TGD_R16:
          e = launch(gram_small_kernel<TGD_R16>);
          break;
        default:
          break;
      }
      if (e != cudaSuccess) return e;
      GramGeom geo{};
      geo.I = a.I;
      geo.TI = 64;  // every cell of the partials is written
      geo.nsplit = grid;
      const int64_t cells = (int64_t)a.I * a.I;
      gram_reduce_kernel<<<(int)ceil_div(cells, RC), RC * RS, 0, s>>>((const float2*)partial, geo,
                                                                       (double2*)gram);
      return cudaGetLastError();
    }
  }
  if (dims[n] <= 128) return mode_gram_tc(g, dt, bits, nd, dims, n, partial, gram, err, s, max_ctas);
  GramGeom geo = gram_geom(nd, dims, n);
  dim3 grid(geo.npairs, geo.nsplit);
  const size_t smem = gram_smem_bytes(geo);
  switch (dt) {
    case TGD_R32:
      gram_partial_kernel<TGD_R32><<<grid, geo.nthr, smem, s>>>(g, bits, geo, (float2*)partial);
      break;
    case TGD_C64:
      gram_partial_kernel<TGD_C64><<<grid, geo.nthr, smem, s>>>(g, bits, geo, (float2*)partial);
      break;
    case TGD_C32H:
      gram_partial_kernel<TGD_C32H><<<grid, geo.nthr, smem, s>>>(g, bits, geo, (float2*)partial);
      break;
    case TGD_R16:
      gram_partial_kernel<TGD_R16><<<grid, geo.nthr, smem, s>>>(g, bits, geo, (float2*)partial);
      break;
    default:
      return cudaErrorInvalidValue;
  }
  const int64_t cells = geo.I * geo.I;
  gram_reduce_kernel<<<(int)ceil_div(cells, RC), RC * RS, 0, s>>>((const float2*)partial, geo,
                                                                   (double2*)gram);
  return cudaGetLastError();
}

// (Jacobi scratch: A, Vt and W of n x (n + 2) complex each)
size_t eig_work_doubles(int n) { return (size_t)6 * n * (n + 2); }

cudaError_t batched_eigh(const EigJob* jobs_host, int njobs, cudaStream_t s) {
  if (njobs <= 0) return cudaSuccess;
  if (njobs > TGD_MAX_NDIM) return cudaErrorInvalidValue;
  EigJobs jobs{};
  size_t ssmem = 16;
  for (int j = 0; j < njobs; ++j) {
    const int n = jobs_host[j].n;
    if (n < 1 || n > ES_MAXN || jobs_host[j].r > n) return cudaErrorInvalidValue;
    const size_t np = (size_t)n + 1 + (n & 1);
    if (n <= ES_SMEM_MAXN) ssmem = std::max(ssmem, 2 * sizeof(double2) * (size_t)n * np);
    jobs.j[j] = jobs_host[j];
  }
  cudaError_t e = cudaFuncSetAttribute(eig_small_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)ssmem);
  if (e != cudaSuccess) return e;
  eig_small_kernel<<<njobs, ET, ssmem, s>>>(jobs);
  return cudaGetLastError();
}

}  // namespace tgd
