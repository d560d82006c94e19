// Selection of the sparse index set Omega: radix select + ordered compaction.
//
// Top-k by magnitude and the random-sampling variant are the two ways the
// Pith review of TensorGRaD ("What carries the argument") re-selects Omega
// every T steps; the sparse part is stored in COO form (the nullthought.net
// summary, section 二). Both reduce to one problem: the k smallest 64-bit keys
// with ties broken by the lower linear index, emitted in ascending index order.
//   top-k:  key(i) = ~magbits(G[i]) (32 significant bits), so the largest
//           magnitude has the smallest key;
//   random: key(i) = splitmix64 output (i + 1) of a stream seeded per refresh.
//
// Algorithm (no sort of N): most-significant-digit radix select over 11-bit
// digits finds the exact k-th key K* and how many keys equal to K* are still
// needed; then one ordered compaction pass writes every index with key < K*
// and the first `need` indices with key == K* (in index order), which is
// already the ascending COO list. Every pass reads its keys straight from the
// gradient (HBM-bound; keys are recomputed, never stored), and every count is
// an integer, so the result is bit-exact and independent of scheduling.

#include "common.cuh"
#include "kernels.h"

namespace tgd {
namespace {

constexpr int DIGIT = 11;
constexpr int BINS = 1 << DIGIT;
constexpr int CHUNK = 4096;  // elements per compaction block
constexpr int CT = 256;      // threads per compaction block
constexpr int MAX_PASSES = 6;

struct SelState {
  unsigned long long prefix, mask;
  long long need;
  long long pad;
};

template <int DT>
struct TopKey {
  const void* g;
  __device__ __forceinline__ uint64_t operator()(int64_t i) const {
    return (uint64_t)(uint32_t)(~mag_key<DT>(g, i));
  }
};

struct RandKey {
  uint64_t s;
  __device__ __forceinline__ uint64_t operator()(int64_t i) const {
    return sm_mix(s + (uint64_t)(i + 1) * SM_GAMMA);
  }
};

template <class KeyF>
__global__ void __launch_bounds__(256) hist_kernel(KeyF kf, int64_t n, const SelState* st,
                                                   int shift, int width,
                                                   unsigned long long* hist) {
  __shared__ unsigned int sh[BINS];
  for (int b = threadIdx.x; b < BINS; b += blockDim.x) sh[b] = 0;
  __syncthreads();
  const uint64_t prefix = st->prefix, mask = st->mask;
  const uint32_t dmask = (1u << width) - 1u;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n;
       i += (int64_t)gridDim.x * blockDim.x) {
    uint64_t key = kf(i);
    if ((key & mask) == prefix) atomicAdd(&sh[(uint32_t)(key >> shift) & dmask], 1u);
  }
  __syncthreads();
  for (int b = threadIdx.x; b < (1 << width); b += blockDim.x)
    if (sh[b]) atomicAdd(&hist[b], (unsigned long long)sh[b]);
}

// Block-wide exclusive scan of one 64-bit value per thread (blockDim = 1024).
__device__ unsigned long long block_excl_scan(unsigned long long v, unsigned long long* total) {
  __shared__ unsigned long long warp_sum[32];
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
  unsigned long long x = v;
  for (int o = 1; o < 32; o <<= 1) {
    unsigned long long y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) warp_sum[wid] = x;
  __syncthreads();
  if (wid == 0) {
    int nw = blockDim.x >> 5;
    unsigned long long w = lane < nw ? warp_sum[lane] : 0;
    for (int o = 1; o < 32; o <<= 1) {
      unsigned long long y = __shfl_up_sync(0xffffffffu, w, o);
      if (lane >= o) w += y;
    }
    if (lane < nw) warp_sum[lane] = w;  // inclusive
  }
  __syncthreads();
  unsigned long long before = (wid ? warp_sum[wid - 1] : 0) + x - v;
  if (total) *total = warp_sum[(blockDim.x >> 5) - 1];
  __syncthreads();
  return before;
}

// Picks the digit bin that holds the need-th smallest remaining key.
__global__ void __launch_bounds__(1024) scan_digit_kernel(const unsigned long long* hist,
                                                          int shift, int width, SelState* st) {
  __shared__ long long need_s;
  if (threadIdx.x == 0) need_s = st->need;
  __syncthreads();
  const long long need = need_s;
  const int nb = 1 << width;
  const int b0 = 2 * threadIdx.x, b1 = b0 + 1;
  unsigned long long h0 = b0 < nb ? hist[b0] : 0, h1 = b1 < nb ? hist[b1] : 0;
  unsigned long long excl = block_excl_scan(h0 + h1, nullptr);
  int bin = -1;
  unsigned long long before = 0;
  if ((long long)excl < need && need <= (long long)(excl + h0)) {
    bin = b0;
    before = excl;
  } else if ((long long)(excl + h0) < need && need <= (long long)(excl + h0 + h1)) {
    bin = b1;
    before = excl + h0;
  }
  if (bin >= 0) {
    st->prefix |= (unsigned long long)bin << shift;
    st->mask |= (unsigned long long)((1u << width) - 1u) << shift;
    st->need = need - (long long)before;
  }
}

template <class KeyF>
__global__ void __launch_bounds__(CT) count_kernel(KeyF kf, int64_t n, const SelState* st,
                                                   int* blk_lt, int* blk_eq) {
  const uint64_t K = st->prefix;
  const int64_t base = (int64_t)blockIdx.x * CHUNK;
  int lt = 0, eq = 0;
  for (int r = 0; r < CHUNK / CT; ++r) {
    int64_t i = base + r * CT + threadIdx.x;
    if (i < n) {
      uint64_t key = kf(i);
      lt += key < K;
      eq += key == K;
    }
  }
  for (int o = 16; o; o >>= 1) {
    lt += __shfl_xor_sync(0xffffffffu, lt, o);
    eq += __shfl_xor_sync(0xffffffffu, eq, o);
  }
  __shared__ int s_lt[CT / 32], s_eq[CT / 32];
  if ((threadIdx.x & 31) == 0) {
    s_lt[threadIdx.x >> 5] = lt;
    s_eq[threadIdx.x >> 5] = eq;
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    int a = 0, b = 0;
    for (int w = 0; w < CT / 32; ++w) {
      a += s_lt[w];
      b += s_eq[w];
    }
    blk_lt[blockIdx.x] = a;
    blk_eq[blockIdx.x] = b;
  }
}

// Exclusive scans over compaction blocks: output offset of each block and the
// number of threshold-equal keys in earlier blocks.
__global__ void __launch_bounds__(1024) block_offsets_kernel(const int* blk_lt, const int* blk_eq,
                                                             int64_t nblk, const SelState* st,
                                                             long long* out_off,
                                                             long long* eq_before) {
  const long long need = st->need;
  unsigned long long lt_carry = 0, eq_carry = 0;
  for (int64_t t0 = 0; t0 < nblk; t0 += blockDim.x) {
    int64_t b = t0 + threadIdx.x;
    unsigned long long lt = b < nblk ? (unsigned long long)blk_lt[b] : 0;
    unsigned long long eq = b < nblk ? (unsigned long long)blk_eq[b] : 0;
    unsigned long long lt_tot, eq_tot;
    unsigned long long lt_ex = block_excl_scan(lt, &lt_tot);
    unsigned long long eq_ex = block_excl_scan(eq, &eq_tot);
    if (b < nblk) {
      long long eqb = (long long)(eq_carry + eq_ex);
      eq_before[b] = eqb;
      out_off[b] = (long long)(lt_carry + lt_ex) + (eqb < need ? eqb : need);
    }
    lt_carry += lt_tot;
    eq_carry += eq_tot;
  }
}

// Ordered compaction of one block of CHUNK keys. Key r CT + t of the block
// belongs to thread t (coalesced loads), so index order is (r, warp, lane).
// Each thread loads its CHUNK / CT keys first and keeps two flags each (below
// / equal to the threshold); per (r, warp) counts of equal keys, then of taken
// keys, go through one block scan each, and every key's rank follows from its
// warp's ballot. Ties go to the lower index.
template <class KeyF, int DT>
__global__ void __launch_bounds__(CT, 6) write_kernel(KeyF kf, const void* g, int64_t n,
                                                   const SelState* st, const long long* out_off,
                                                   const long long* eq_before, int64_t* out_idx,
                                                   float* out_val) {
  constexpr int PER = CHUNK / CT, NW = CT / 32;
  static_assert(PER <= 32 && PER * NW <= CT, "flags in 32-bit words, one scan entry per thread");
  __shared__ int s_cnt[PER * NW];
  __shared__ long long s_ex[PER * NW];
  const uint64_t K = st->prefix;
  const long long need = st->need;
  const int64_t base = (int64_t)blockIdx.x * CHUNK;
  const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
  const unsigned lt_mask = (1u << lane) - 1u;
  uint32_t ltm = 0, eqm = 0;
#pragma unroll
  for (int r = 0; r < PER; ++r) {
    const int64_t i = base + r * CT + tid;
    const bool valid = i < n;
    const uint64_t key = valid ? kf(i) : ~0ull;
    ltm |= (uint32_t)(valid && key < K) << r;
    eqm |= (uint32_t)(valid && key == K) << r;
  }
  // exclusive prefix, in (r, warp) order, of per-(r, warp) counts of flags f
  auto rank_base = [&](uint32_t f) {
#pragma unroll
    for (int r = 0; r < PER; ++r) {
      const unsigned b = __ballot_sync(0xffffffffu, (f >> r) & 1u);
      if (lane == 0) s_cnt[r * NW + wid] = __popc(b);
    }
    __syncthreads();
    const unsigned long long v = tid < PER * NW ? (unsigned long long)s_cnt[tid] : 0ull;
    const unsigned long long ex = block_excl_scan(v, nullptr);
    if (tid < PER * NW) s_ex[tid] = (long long)ex;
    __syncthreads();
  };
  rank_base(eqm);
  uint32_t take = ltm;
  const long long eq0 = eq_before[blockIdx.x];
#pragma unroll
  for (int r = 0; r < PER; ++r) {
    const unsigned b = __ballot_sync(0xffffffffu, (eqm >> r) & 1u);
    if ((eqm >> r) & 1u) {
      const long long rank = eq0 + s_ex[r * NW + wid] + __popc(b & lt_mask);
      if (rank < need) take |= 1u << r;
    }
  }
  __syncthreads();  // s_ex is rewritten below
  rank_base(take);
  const long long off0 = out_off[blockIdx.x];
#pragma unroll
  for (int r = 0; r < PER; ++r) {
    const unsigned b = __ballot_sync(0xffffffffu, (take >> r) & 1u);
    if (!((take >> r) & 1u)) continue;
    const long long pos = off0 + s_ex[r * NW + wid] + __popc(b & lt_mask);
    const int64_t i = base + r * CT + tid;
    out_idx[pos] = i;
    if (out_val) {
      if constexpr (DT >= 0) {
        const float2 v = load_elem<DT>(g, i);
        if constexpr (Dt<DT>::cplx) {
          ((float2*)out_val)[pos] = v;
        } else {
          out_val[pos] = v.x;
        }
      }
    }
  }
}

// Selection state before the first digit pass: no prefix fixed, k to find.
__global__ void init_state_kernel(SelState* st, long long k) {
  st->prefix = 0ull;
  st->mask = 0ull;
  st->need = k;
  st->pad = 0;
}

template <int DT>
__global__ void iota_kernel(const void* g, int64_t n, int64_t* out_idx, float* out_val) {
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n;
       i += (int64_t)gridDim.x * blockDim.x) {
    out_idx[i] = i;
    if (out_val) {
      if constexpr (DT >= 0) {
        float2 v = load_elem<DT>(g, i);
        if constexpr (Dt<DT>::cplx)
          ((float2*)out_val)[i] = v;
        else
          out_val[i] = v.x;
      }
    }
  }
}

__global__ void mask_bits_kernel(const int64_t* omega, int64_t k, uint32_t* bits) {
  for (int64_t j = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; j < k;
       j += (int64_t)gridDim.x * blockDim.x) {
    int64_t i = omega[j];
    atomicOr(bits + (i >> 5), 1u << (i & 31));
  }
}

// tile_off[t] = number of Omega entries below t * tile_elems (lower bound);
// loc[j] = Omega[j] - tile(j) * tile_elems.
__global__ void tile_index_kernel(const int64_t* omega, int64_t k, int64_t tile_elems,
                                  int64_t n_tiles, int64_t* tile_off, uint16_t* loc) {
  int64_t tid = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  int64_t stride = (int64_t)gridDim.x * blockDim.x;
  for (int64_t t = tid; t <= n_tiles; t += stride) {
    int64_t target = t * tile_elems, lo = 0, hi = k;
    while (lo < hi) {
      int64_t mid = (lo + hi) >> 1;
      if (omega[mid] < target)
        lo = mid + 1;
      else
        hi = mid;
    }
    tile_off[t] = lo;
  }
  for (int64_t j = tid; j < k; j += stride) {
    int64_t i = omega[j];
    loc[j] = (uint16_t)(i - (i / tile_elems) * tile_elems);
  }
}

struct WsLayout {
  unsigned long long* hist;
  SelState* st;
  int* blk_lt;
  int* blk_eq;
  long long* out_off;
  long long* eq_before;
  int64_t nblk;
};

size_t align256(size_t x) { return (x + 255) & ~(size_t)255; }

WsLayout carve(void* ws, int64_t n) {
  WsLayout L;
  L.nblk = ceil_div(n, CHUNK);
  char* p = (char*)ws;
  L.hist = (unsigned long long*)p;
  p += align256(sizeof(unsigned long long) * BINS * MAX_PASSES);
  L.st = (SelState*)p;
  p += align256(sizeof(SelState));
  L.blk_lt = (int*)p;
  p += align256(sizeof(int) * L.nblk);
  L.blk_eq = (int*)p;
  p += align256(sizeof(int) * L.nblk);
  L.out_off = (long long*)p;
  p += align256(sizeof(long long) * L.nblk);
  L.eq_before = (long long*)p;
  return L;
}

int hist_grid(int64_t n) {
  int64_t b = ceil_div(n, 256);
  return (int)(b < 148 * 8 ? (b > 0 ? b : 1) : 148 * 8);
}

template <class KeyF, int DT>
cudaError_t run_select(KeyF kf, int key_bits, const void* g, int64_t n, int64_t k,
                       int64_t* out_idx, float* out_val, void* ws, cudaStream_t s) {
  if (k <= 0) return cudaSuccess;
  if (k >= n) {
    int grid = hist_grid(n);
    iota_kernel<DT><<<grid, 256, 0, s>>>(g, n, out_idx, out_val);
    return cudaGetLastError();
  }
  WsLayout L = carve(ws, n);
  cudaError_t e = cudaMemsetAsync(L.hist, 0, sizeof(unsigned long long) * BINS * MAX_PASSES, s);
  if (e != cudaSuccess) return e;
  // the selection state is set on the device: nothing is copied from the host
  init_state_kernel<<<1, 1, 0, s>>>(L.st, (long long)k);
  int pass = 0;
  for (int hi = key_bits; hi > 0; ++pass) {
    int width = hi >= DIGIT ? DIGIT : hi;
    int shift = hi - width;
    hist_kernel<<<hist_grid(n), 256, 0, s>>>(kf, n, L.st, shift, width, L.hist + pass * BINS);
    scan_digit_kernel<<<1, 1024, 0, s>>>(L.hist + pass * BINS, shift, width, L.st);
    hi = shift;
  }
  count_kernel<<<(unsigned)L.nblk, CT, 0, s>>>(kf, n, L.st, L.blk_lt, L.blk_eq);
  block_offsets_kernel<<<1, 1024, 0, s>>>(L.blk_lt, L.blk_eq, L.nblk, L.st, L.out_off,
                                          L.eq_before);
  write_kernel<KeyF, DT><<<(unsigned)L.nblk, CT, 0, s>>>(kf, g, n, L.st, L.out_off, L.eq_before,
                                                         out_idx, out_val);
  return cudaGetLastError();
}

}  // namespace

size_t select_workspace_bytes(int64_t n) {
  int64_t nblk = ceil_div(n > 0 ? n : 1, CHUNK);
  return align256(sizeof(unsigned long long) * BINS * MAX_PASSES) + align256(sizeof(SelState)) +
         2 * align256(sizeof(int) * nblk) + 2 * align256(sizeof(long long) * nblk);
}

cudaError_t select_topk(const void* g, int dt, int64_t n, int64_t k, int64_t* out_idx,
                        float* out_val, void* ws, cudaStream_t s) {
  switch (dt) {
    case TGD_R32:
      return run_select<TopKey<TGD_R32>, TGD_R32>(TopKey<TGD_R32>{g}, 32, g, n, k, out_idx,
                                                  out_val, ws, s);
    case TGD_C64:
      return run_select<TopKey<TGD_C64>, TGD_C64>(TopKey<TGD_C64>{g}, 32, g, n, k, out_idx,
                                                  out_val, ws, s);
    case TGD_C32H:
      return run_select<TopKey<TGD_C32H>, TGD_C32H>(TopKey<TGD_C32H>{g}, 32, g, n, k, out_idx,
                                                    out_val, ws, s);
    case TGD_R16:
      return run_select<TopKey<TGD_R16>, TGD_R16>(TopKey<TGD_R16>{g}, 32, g, n, k, out_idx,
                                                  out_val, ws, s);
  }
  return cudaErrorInvalidValue;
}

cudaError_t select_random(uint64_t seed, uint64_t ordinal, const void* g, int dt, int64_t n,
                          int64_t k, int64_t* out_idx, float* out_val, void* ws,
                          cudaStream_t s) {
  RandKey kf{sm_mix(seed + (ordinal + 1) * SM_GAMMA)};
  switch (dt) {
    case TGD_R32:
      return run_select<RandKey, TGD_R32>(kf, 64, g, n, k, out_idx, out_val, ws, s);
    case TGD_C64:
      return run_select<RandKey, TGD_C64>(kf, 64, g, n, k, out_idx, out_val, ws, s);
    case TGD_C32H:
      return run_select<RandKey, TGD_C32H>(kf, 64, g, n, k, out_idx, out_val, ws, s);
    case TGD_R16:
      return run_select<RandKey, TGD_R16>(kf, 64, g, n, k, out_idx, out_val, ws, s);
  }
  return cudaErrorInvalidValue;
}

cudaError_t build_mask_bits(const int64_t* omega, int64_t k, int64_t n, uint32_t* bits,
                            cudaStream_t s) {
  cudaError_t e = cudaMemsetAsync(bits, 0, sizeof(uint32_t) * ceil_div(n, 32), s);
  if (e != cudaSuccess || k <= 0) return e;
  mask_bits_kernel<<<hist_grid(k), 256, 0, s>>>(omega, k, bits);
  return cudaGetLastError();
}

cudaError_t build_tile_index(const int64_t* omega, int64_t k, int64_t tile_elems,
                             int64_t n_tiles, int64_t* tile_off, uint16_t* loc, cudaStream_t s) {
  int64_t work = (k > n_tiles + 1 ? k : n_tiles + 1);
  tile_index_kernel<<<hist_grid(work), 256, 0, s>>>(omega, k, tile_elems, n_tiles, tile_off, loc);
  return cudaGetLastError();
}

}  // namespace tgd
