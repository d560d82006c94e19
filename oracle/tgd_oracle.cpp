// TensorGRaD optimizer step: CPU oracle.
//
// TEST INFRASTRUCTURE ONLY. This file is the slow, plain, fp64 statement of
// what the optimizer step computes. Only the test suite, the smoke check and
// the CPU-baseline leg of the benchmark load it. The CUDA library shares no
// code, header, table or constant with it, and neither side calls the other.
//
// Sources (the web pages on TensorGRaD that define the method):
//   [S1] "TensorGRaD" summary, nullthought.net/?p=5973, section 三 (method
//        implementation details): the sparse part is extracted first, the
//        residual gets the Tucker low-rank part, both parts get their own Adam
//        update, and the sparse update is scatter-added into the rebuilt
//        low-rank tensor in place; FP32 optimizer states (mixed precision);
//        index set and subspace re-selected every T steps.
//   [S2] Pith review of TensorGRaD (pith.science/paper/2501.02379),
//        "What carries the argument": Tucker / higher-order SVD factors U^(n)
//        computed once and reused for T steps, projection to a core, Adam
//        moments on the core, reconstruction by mode-wise products; COO
//        sparse part on an index set Omega re-selected every T steps by
//        top-k magnitude or random sampling.
//   [S3] same review, appended paper text, Theorem 2 (Tensor low-rank
//        convergence): project R = G x1 P1^T ... xd Pd^T, update optimizer
//        states with R, project back R x1 P1 ... xd Pd.
//   [S4] same review, appended paper text, Appendix K (tensor operations and
//        notation): mode-k unfolding, mode-k product, Frobenius norm.
//
// Readings where the pages are silent:
//   k = floor(rho * N); top-k key = fp32 |g| (real) or fp32 fma(re,re,im*im)
//   (complex); ties -> lower linear index; Omega emitted ascending; random
//   Omega = k smallest splitmix64-derived keys; plain HOSVD (each U_n from the
//   Gram of the full residual); r_n == I_n means U_n = I; eigenvector phase:
//   largest-magnitude entry real positive; complex Adam: m complex, v = EMA of
//   |g|^2 (mode 0) or re/im treated as separate reals (mode 1); bias
//   correction with s = t + 1; decoupled weight decay; moments kept across a
//   refresh unless asked to reset; refresh before the step when t % T == 0.
//   Low-rank-first order (the ablation of the decomposition order): factors
//   from the gradient itself, Omega on E = G - L keyed from E rounded to fp32,
//   sparse values E at Omega with L from the step's pre-Adam core.
//
// Everything is computed in fp64. Stored state is rounded to its storage type
// (moments and factors fp32, weights their own dtype) exactly once.
//
// Build: g++ -O2 -std=c++17 -fPIC -shared -pthread -ffp-contract=off

#include <algorithm>
#include <cmath>
#include <cstdint>
#include <cstdlib>
#include <cstring>
#include <functional>
#include <thread>
#include <vector>

namespace {

// ---------------------------------------------------------------- dtypes
enum { DT_R32 = 0, DT_C64 = 1, DT_C32H = 2, DT_R16 = 3 };

bool dt_complex(int dt) { return dt == DT_C64 || dt == DT_C32H; }
bool dt_valid(int dt) { return dt >= 0 && dt <= 3; }

struct cd {
  double re, im;
};
inline cd operator+(cd a, cd b) { return {a.re + b.re, a.im + b.im}; }
inline cd operator*(cd a, cd b) {
  return {a.re * b.re - a.im * b.im, a.re * b.im + a.im * b.re};
}
inline cd conj(cd a) { return {a.re, -a.im}; }
inline double abs2(cd a) { return a.re * a.re + a.im * a.im; }

// IEEE 754 binary16 -> double (exact).
double half_to_double(uint16_t h) {
  int s = (h >> 15) & 1, e = (h >> 10) & 31, m = h & 1023;
  double v;
  if (e == 0)
    v = std::ldexp((double)m, -24);
  else if (e == 31)
    v = m ? NAN : INFINITY;
  else
    v = std::ldexp((double)(1024 + m), e - 25);
  return s ? -v : v;
}

// double -> binary16, round to nearest, ties to even, overflow to +-inf.
uint16_t double_to_half(double x) {
  if (std::isnan(x)) return 0x7E00;
  uint16_t sign = std::signbit(x) ? 0x8000 : 0;
  double a = std::fabs(x);
  if (a == 0.0) return sign;
  if (a < std::ldexp(1.0, -14)) {  // subnormal range: multiples of 2^-24
    double q = std::nearbyint(std::ldexp(a, 24));  // ties to even (default mode)
    return sign | (uint16_t)q;  // q == 1024 gives the smallest normal exactly
  }
  int E;
  std::frexp(a, &E);  // a = f * 2^E, f in [0.5, 1)
  int e = E - 1;      // a = m * 2^e, m in [1, 2)
  double q = std::nearbyint(std::ldexp(a, 10 - e));  // in [1024, 2048]
  if (q == 2048.0) {
    q = 1024.0;
    e += 1;
  }
  if (e + 15 >= 31) return sign | 0x7C00;
  return sign | (uint16_t)(((e + 15) << 10) | ((int)q - 1024));
}

uint32_t float_bits(float f) {
  uint32_t b;
  std::memcpy(&b, &f, 4);
  return b;
}

// Element i of a raw buffer as a complex double (imaginary part 0 for reals).
cd load_elem(const void* p, int dt, int64_t i) {
  switch (dt) {
    case DT_R32: return {(double)((const float*)p)[i], 0.0};
    case DT_R16: return {half_to_double(((const uint16_t*)p)[i]), 0.0};
    case DT_C64: {
      const float* f = (const float*)p;
      return {(double)f[2 * i], (double)f[2 * i + 1]};
    }
    default: {
      const uint16_t* h = (const uint16_t*)p;
      return {half_to_double(h[2 * i]), half_to_double(h[2 * i + 1])};
    }
  }
}

// Store with one rounding from fp64 to the storage type.
void store_elem(void* p, int dt, int64_t i, cd v) {
  switch (dt) {
    case DT_R32: ((float*)p)[i] = (float)v.re; break;
    case DT_R16: ((uint16_t*)p)[i] = double_to_half(v.re); break;
    case DT_C64:
      ((float*)p)[2 * i] = (float)v.re;
      ((float*)p)[2 * i + 1] = (float)v.im;
      break;
    default:
      ((uint16_t*)p)[2 * i] = double_to_half(v.re);
      ((uint16_t*)p)[2 * i + 1] = double_to_half(v.im);
  }
}

// Magnitude key of element i, as the bits of a non-negative fp32 number (so
// integer order equals magnitude order). Real: |g| in fp32. Complex: the
// squared modulus fma(re, re, im*im) in fp32, each operation rounded once.
// Squares keep the order of |z| and add no ties from a square root.
uint32_t mag_key(const void* p, int dt, int64_t i) {
  float re, im = 0.f;
  switch (dt) {
    case DT_R32: re = ((const float*)p)[i]; break;
    case DT_R16: re = (float)half_to_double(((const uint16_t*)p)[i]); break;
    case DT_C64:
      re = ((const float*)p)[2 * i];
      im = ((const float*)p)[2 * i + 1];
      break;
    default:
      re = (float)half_to_double(((const uint16_t*)p)[2 * i]);
      im = (float)half_to_double(((const uint16_t*)p)[2 * i + 1]);
  }
  if (!dt_complex(dt)) return float_bits(std::fabs(re));
  float im2 = im * im;
  float k = std::fma(re, re, im2);
  return float_bits(k);
}

// ------------------------------------------------------------ threading
int n_threads() {
  static int n = [] {
    const char* e = std::getenv("TGD_ORACLE_THREADS");
    int v = e ? std::atoi(e) : 0;
    if (v <= 0) v = (int)std::thread::hardware_concurrency();
    return v > 0 ? v : 1;
  }();
  return n;
}

// Runs f(lo, hi) over [0, n) split into contiguous chunks, one per thread.
// Every output element is owned by one chunk and computed in a fixed order,
// so results do not depend on the number of threads.
void parallel_for(int64_t n, const std::function<void(int64_t, int64_t)>& f) {
  int nt = n_threads();
  if (n < 2 || nt == 1) {
    if (n > 0) f(0, n);
    return;
  }
  if (nt > n) nt = (int)n;
  std::vector<std::thread> th;
  int64_t per = (n + nt - 1) / nt;
  for (int t = 0; t < nt; ++t) {
    int64_t lo = t * per, hi = std::min<int64_t>(n, lo + per);
    if (lo >= hi) break;
    th.emplace_back(f, lo, hi);
  }
  for (auto& x : th) x.join();
}

// ------------------------------------------------------- selection of Omega
// Top-k by magnitude [S1 section 二, S2]: the k largest keys; among equal
// keys the lower linear index wins; the result is listed in ascending order.
void topk_select(const void* g, int dt, int64_t n, int64_t k, int64_t* out) {
  if (k <= 0) return;
  if (k >= n) {
    for (int64_t i = 0; i < n; ++i) out[i] = i;
    return;
  }
  std::vector<uint32_t> key(n);
  parallel_for(n, [&](int64_t lo, int64_t hi) {
    for (int64_t i = lo; i < hi; ++i) key[i] = mag_key(g, dt, i);
  });
  std::vector<uint32_t> tmp(key);
  std::nth_element(tmp.begin(), tmp.begin() + (k - 1), tmp.end(), std::greater<uint32_t>());
  uint32_t thr = tmp[k - 1];
  int64_t gt = 0;
  for (int64_t i = 0; i < n; ++i) gt += key[i] > thr;
  int64_t need = k - gt, c = 0;
  for (int64_t i = 0; i < n; ++i) {
    if (key[i] > thr || (key[i] == thr && need > 0)) {
      if (key[i] == thr) --need;
      out[c++] = i;
    }
  }
}

// splitmix64 output function (Steele, Lea and Flood, "Fast splittable
// pseudorandom number generators", 2014; the constants of Vigna's splitmix64).
uint64_t sm_mix(uint64_t z) {
  z = (z ^ (z >> 30)) * 0xbf58476d1ce4e5b9ULL;
  z = (z ^ (z >> 27)) * 0x94d049bb133111ebULL;
  return z ^ (z >> 31);
}
const uint64_t SM_GAMMA = 0x9e3779b97f4a7c15ULL;

// Random-sampling Omega [S2]: uniform without replacement, re-drawn at every
// refresh. Element i gets the (i+1)-th splitmix64 output of a stream whose
// seed is the (ordinal+1)-th output of the stream seeded with `seed`; Omega is
// the k smallest keys (ties -> lower index), listed ascending.
uint64_t random_key(uint64_t seed, uint64_t ordinal, uint64_t i) {
  uint64_t s = sm_mix(seed + (ordinal + 1) * SM_GAMMA);
  return sm_mix(s + (i + 1) * SM_GAMMA);
}

void random_select(uint64_t seed, uint64_t ordinal, int64_t n, int64_t k, int64_t* out) {
  if (k <= 0) return;
  if (k >= n) {
    for (int64_t i = 0; i < n; ++i) out[i] = i;
    return;
  }
  std::vector<uint64_t> key(n);
  parallel_for(n, [&](int64_t lo, int64_t hi) {
    for (int64_t i = lo; i < hi; ++i) key[i] = random_key(seed, ordinal, (uint64_t)i);
  });
  std::vector<uint64_t> tmp(key);
  std::nth_element(tmp.begin(), tmp.begin() + (k - 1), tmp.end());
  uint64_t thr = tmp[k - 1];
  int64_t lt = 0;
  for (int64_t i = 0; i < n; ++i) lt += key[i] < thr;
  int64_t need = k - lt, c = 0;
  for (int64_t i = 0; i < n; ++i) {
    if (key[i] < thr || (key[i] == thr && need > 0)) {
      if (key[i] == thr) --need;
      out[c++] = i;
    }
  }
}

// ------------------------------------------------------- tensor algebra
// Mode-n product [S4]. X has dims[0..nd), row-major (last index fastest),
// viewed as (A, I_n, B). U is I_n x r_n (row-major, complex).
//   proj:   Y[a][j][b] = sum_i conj(U[i][j]) X[a][i][b]   (X x_n U^H), j < r_n
//   expand: Y[a][i][b] = sum_j U[i][j]       X[a][j][b]   (X x_n U),   i < I_n
// The sum runs in ascending order of the contracted index for every output.
void mode_product(const cd* X, const std::vector<int64_t>& dims, int n, const cd* U, int64_t In,
                  int64_t rn, bool proj, cd* Y, bool threaded) {
  int64_t A = 1, B = 1;
  for (int q = 0; q < n; ++q) A *= dims[q];
  for (size_t q = n + 1; q < dims.size(); ++q) B *= dims[q];
  int64_t Kin = proj ? In : rn, Kout = proj ? rn : In;
  auto body = [&](int64_t a, int64_t b0, int64_t b1) {
    for (int64_t jo = 0; jo < Kout; ++jo) {
      cd* y = Y + (a * Kout + jo) * B;
      for (int64_t b = b0; b < b1; ++b) y[b] = {0.0, 0.0};
      for (int64_t ki = 0; ki < Kin; ++ki) {
        cd c = proj ? conj(U[ki * rn + jo]) : U[jo * rn + ki];
        const cd* x = X + (a * Kin + ki) * B;
        for (int64_t b = b0; b < b1; ++b) y[b] = y[b] + c * x[b];
      }
    }
  };
  if (!threaded) {
    for (int64_t a = 0; a < A; ++a) body(a, 0, B);
  } else if (A >= n_threads()) {
    parallel_for(A, [&](int64_t lo, int64_t hi) {
      for (int64_t a = lo; a < hi; ++a) body(a, 0, B);
    });
  } else {
    for (int64_t a = 0; a < A; ++a)
      parallel_for(B, [&](int64_t lo, int64_t hi) { body(a, lo, hi); });
  }
}

// Mode-n Gram matrix of X: Gram[i][i'] = sum over all other indices of
// X[..i..] * conj(X[..i'..]) = X_(n) X_(n)^H with X_(n) the mode-n unfolding
// [S4]. Output I_n x I_n, Hermitian positive semidefinite.
void mode_gram(const cd* X, const std::vector<int64_t>& dims, int n, cd* Gm) {
  int64_t A = 1, B = 1, I = dims[n];
  for (int q = 0; q < n; ++q) A *= dims[q];
  for (size_t q = n + 1; q < dims.size(); ++q) B *= dims[q];
  parallel_for(I, [&](int64_t lo, int64_t hi) {
    for (int64_t i = lo; i < hi; ++i)
      for (int64_t i2 = 0; i2 < I; ++i2) {
        double sr = 0, si = 0;
        for (int64_t a = 0; a < A; ++a) {
          const cd* x1 = X + (a * I + i) * B;
          const cd* x2 = X + (a * I + i2) * B;
          for (int64_t b = 0; b < B; ++b) {
            cd p = x1[b] * conj(x2[b]);
            sr += p.re;
            si += p.im;
          }
        }
        Gm[i * I + i2] = {sr, si};
      }
  });
}

// Eigen-decomposition of a Hermitian matrix by the cyclic Jacobi method
// (row-by-row sweeps of 2x2 rotations), fp64. A (n x n, row-major) is
// overwritten. On return w holds the eigenvalues in descending order (ties ->
// lower original index) and V (n x n) the matching unit eigenvectors as
// columns, each scaled by a unit phase so that its largest-magnitude entry
// (ties -> lowest row) is real and positive.
void jacobi_eigh(cd* A, int64_t n, double* w, cd* V) {
  std::vector<cd> Q(n * n, cd{0, 0});
  for (int64_t i = 0; i < n; ++i) Q[i * n + i] = {1, 0};
  double fro = 0;
  for (int64_t i = 0; i < n * n; ++i) fro += abs2(A[i]);
  for (int sweep = 0; sweep < 40; ++sweep) {
    double off = 0;
    for (int64_t p = 0; p < n; ++p)
      for (int64_t q = p + 1; q < n; ++q) off += abs2(A[p * n + q]);
    if (off <= 1e-28 * fro || off == 0.0) break;
    for (int64_t p = 0; p < n - 1; ++p)
      for (int64_t q = p + 1; q < n; ++q) {
        cd apq = A[p * n + q];
        double r = std::sqrt(abs2(apq));
        if (r == 0.0) continue;
        double app = A[p * n + p].re, aqq = A[q * n + q].re;
        // e = apq / r = e^{i phi}. With D = diag(1, conj(e)) the pair block
        // becomes real symmetric [[app, r], [r, aqq]]; a real rotation with
        // t = tan(theta) zeroes it. J = D * [[c, s], [-s, c]].
        cd e = {apq.re / r, apq.im / r};
        double tau = (aqq - app) / (2 * r);
        double t = (tau >= 0 ? 1.0 : -1.0) / (std::fabs(tau) + std::sqrt(1 + tau * tau));
        double c = 1 / std::sqrt(1 + t * t), s = t * c;
        cd ec = conj(e);
        // Column update A <- A J:  A[:,p] <- c A[:,p] - s conj(e) A[:,q],
        //                          A[:,q] <- s A[:,p] + c conj(e) A[:,q].
        auto colrot = [&](cd* M) {
          for (int64_t i = 0; i < n; ++i) {
            cd xp = M[i * n + p], xq = M[i * n + q] * ec;
            M[i * n + p] = {c * xp.re - s * xq.re, c * xp.im - s * xq.im};
            M[i * n + q] = {s * xp.re + c * xq.re, s * xp.im + c * xq.im};
          }
        };
        colrot(A);
        colrot(Q.data());
        // Row update A <- J^H A: rows p, q with the conjugate coefficients.
        for (int64_t j = 0; j < n; ++j) {
          cd xp = A[p * n + j], xq = A[q * n + j] * e;
          A[p * n + j] = {c * xp.re - s * xq.re, c * xp.im - s * xq.im};
          A[q * n + j] = {s * xp.re + c * xq.re, s * xp.im + c * xq.im};
        }
        A[p * n + q] = {0, 0};
        A[q * n + p] = {0, 0};
        A[p * n + p].im = 0;
        A[q * n + q].im = 0;
      }
  }
  std::vector<int64_t> ord(n);
  for (int64_t i = 0; i < n; ++i) ord[i] = i;
  std::stable_sort(ord.begin(), ord.end(),
                   [&](int64_t a, int64_t b) { return A[a * n + a].re > A[b * n + b].re; });
  for (int64_t c = 0; c < n; ++c) {
    int64_t src = ord[c];
    w[c] = A[src * n + src].re;
    int64_t im = 0;
    double best = -1;
    for (int64_t i = 0; i < n; ++i) {
      double m = abs2(Q[i * n + src]);
      if (m > best) {
        best = m;
        im = i;
      }
    }
    cd piv = Q[im * n + src];
    double pm = std::sqrt(abs2(piv));
    cd ph = pm > 0 ? cd{piv.re / pm, -piv.im / pm} : cd{1, 0};
    for (int64_t i = 0; i < n; ++i) V[i * n + c] = Q[i * n + src] * ph;
  }
}

// ------------------------------------------------------------ optimizer
struct Opts {
  int omega_mode;  // 0 top-k magnitude, 1 random sampling
  uint64_t seed;
  double sparse_scale;     // lambda
  int complex_adam;        // 0: v = EMA |g|^2; 1: re and im as separate reals
  int moments_on_refresh;  // 0 keep, 1 reset to zero
  int auto_refresh;        // refresh inside step when t % T == 0
  int order = 0;           // 0 sparse part first; 1 low-rank part first (the ablated order)
  int basis = 0;           // 0 HOSVD eigenvectors; 1 DCT columns chosen by alignment
};

struct Orc {
  int d = 0;
  std::vector<int64_t> I, r;
  int64_t N = 0, k = 0, ncore = 0;
  double rho = 0, lr = 0, b1 = 0, b2 = 0, eps = 0, wd = 0;
  int64_t T = 0;
  int gdt = 0, wdt = 0;
  bool cplx = false;
  Opts o{};
  int64_t t = 0, refreshes = 0;
  bool has_subspace = false;
  std::vector<int64_t> omega;
  std::vector<cd> omega_val;
  std::vector<std::vector<float>> U;       // I_n x r_n, complex interleaved (re, im)
  std::vector<std::vector<double>> eigval;  // all eigenvalues of the last Gram
  std::vector<float> core_m, core_v, sp_m, sp_v;
  int mcomp() const { return cplx ? 2 : 1; }
  int vcomp() const { return cplx ? (o.complex_adam == 1 ? 2 : 1) : 1; }
};

std::vector<cd> U_as_cd(const Orc& h, int n) {
  int64_t In = h.I[n], rn = h.r[n];
  std::vector<cd> u(In * rn);
  for (int64_t i = 0; i < In * rn; ++i) u[i] = {(double)h.U[n][2 * i], (double)h.U[n][2 * i + 1]};
  return u;
}

// One Adam moment update [S1 section 三, S2]: moments are read from and
// rounded back to fp32 storage; the update direction m_hat / (sqrt(v_hat) +
// eps) is then formed in fp64 from the stored values.
cd adam_update(cd g, float* m, float* v, const Orc& h, double bc1, double bc2) {
  double b1 = h.b1, b2 = h.b2;
  if (!h.cplx) {
    m[0] = (float)(b1 * m[0] + (1 - b1) * g.re);
    v[0] = (float)(b2 * v[0] + (1 - b2) * g.re * g.re);
    return {((double)m[0] / bc1) / (std::sqrt((double)v[0] / bc2) + h.eps), 0.0};
  }
  m[0] = (float)(b1 * m[0] + (1 - b1) * g.re);
  m[1] = (float)(b1 * m[1] + (1 - b1) * g.im);
  if (h.o.complex_adam == 1) {
    v[0] = (float)(b2 * v[0] + (1 - b2) * g.re * g.re);
    v[1] = (float)(b2 * v[1] + (1 - b2) * g.im * g.im);
    return {((double)m[0] / bc1) / (std::sqrt((double)v[0] / bc2) + h.eps),
            ((double)m[1] / bc1) / (std::sqrt((double)v[1] / bc2) + h.eps)};
  }
  v[0] = (float)(b2 * v[0] + (1 - b2) * abs2(g));
  double den = std::sqrt((double)v[0] / bc2) + h.eps;
  return {((double)m[0] / bc1) / den, ((double)m[1] / bc1) / den};
}

int64_t n_slabs(const Orc& h) {
  int64_t s = 1;
  for (int n = 0; n < h.d - 2; ++n) s *= h.I[n];
  return s;
}

std::vector<cd> load_all(const void* g, int dt, int64_t N) {
  std::vector<cd> X(N);
  parallel_for(N, [&](int64_t lo, int64_t hi) {
    for (int64_t i = lo; i < hi; ++i) X[i] = load_elem(g, dt, i);
  });
  return X;
}

// Entry (k, j) of the orthonormal n x n DCT matrix of the dynamic column
// selection (the Trion / DCT-AdamW page, "dynamic column selection"):
// sqrt(2 / n) cos(k (2j + 1) pi / (2n)), row k = 0 divided by sqrt(2).
double dct_entry(int64_t k, int64_t j, int64_t n) {
  const double v = std::sqrt(2.0 / (double)n) * std::cos((double)k * (2.0 * j + 1.0) * M_PI / (2.0 * n));
  return k == 0 ? v / std::sqrt(2.0) : v;
}

// DCT basis for mode n: the r_n columns q_j of the DCT matrix with the largest
// alignment q_j^T Gram q_j (the squared l2 norm of the unfolding's components
// along q_j), ties to the lower column, listed by descending alignment; the
// sorted alignments stand where the eigenvalues would.
void dct_factor(Orc& h, int n, const std::vector<cd>& Gm) {
  const int64_t In = h.I[n], rn = h.r[n];
  std::vector<double> score(In);
  for (int64_t j = 0; j < In; ++j) {
    double sc = 0;
    for (int64_t a = 0; a < In; ++a)
      for (int64_t b = 0; b < In; ++b) sc += dct_entry(a, j, In) * Gm[a * In + b].re * dct_entry(b, j, In);
    score[j] = sc;
  }
  std::vector<int64_t> ord(In);
  for (int64_t j = 0; j < In; ++j) ord[j] = j;
  std::stable_sort(ord.begin(), ord.end(), [&](int64_t a, int64_t b) { return score[a] > score[b]; });
  std::vector<double> w(In);
  for (int64_t c = 0; c < In; ++c) w[c] = score[ord[c]];
  h.eigval[n] = w;
  for (int64_t i = 0; i < In; ++i)
    for (int64_t c = 0; c < rn; ++c) {
      h.U[n][2 * (i * rn + c)] = (float)dct_entry(i, ord[c], In);
      h.U[n][2 * (i * rn + c) + 1] = 0.f;
    }
}

// U_n for every mode with r_n < I_n: the leading r_n eigenvectors of the
// mode-n Gram matrix of X (plain HOSVD), or the DCT columns most aligned with
// it; all eigenvalues (alignments) are kept.
void factors_from(Orc& h, const std::vector<cd>& X) {
  for (int n = 0; n < h.d; ++n) {
    int64_t In = h.I[n], rn = h.r[n];
    if (rn == In) continue;
    std::vector<cd> Gm(In * In), V(In * In);
    std::vector<double> w(In);
    mode_gram(X.data(), h.I, n, Gm.data());
    if (h.o.basis == 1) {
      dct_factor(h, n, Gm);
      continue;
    }
    jacobi_eigh(Gm.data(), In, w.data(), V.data());
    h.eigval[n] = w;
    for (int64_t i = 0; i < In; ++i)
      for (int64_t j = 0; j < rn; ++j) {
        h.U[n][2 * (i * rn + j)] = (float)V[i * In + j].re;
        h.U[n][2 * (i * rn + j) + 1] = (float)V[i * In + j].im;
      }
  }
}

void finish_refresh(Orc& h);
int refresh_lowrank_first(Orc& h, const void* g);

// Refresh [S1 section 三, S2]: Omega first, then the residual R = G with zeros
// on Omega, then for each mode with r_n < I_n the leading r_n eigenvectors of
// the mode-n Gram matrix of R (plain HOSVD).
int refresh(Orc& h, const void* g) {
  if (h.o.order == 1) return refresh_lowrank_first(h, g);
  h.omega.assign(h.k, 0);
  if (h.o.omega_mode == 0)
    topk_select(g, h.gdt, h.N, h.k, h.omega.data());
  else
    random_select(h.o.seed, (uint64_t)h.refreshes, h.N, h.k, h.omega.data());
  h.omega_val.resize(h.k);
  for (int64_t j = 0; j < h.k; ++j) h.omega_val[j] = load_elem(g, h.gdt, h.omega[j]);
  bool need_gram = false;
  for (int n = 0; n < h.d; ++n) need_gram |= h.r[n] < h.I[n];
  h.eigval.assign(h.d, {});
  if (need_gram) {
    std::vector<cd> R = load_all(g, h.gdt, h.N);
    for (int64_t j = 0; j < h.k; ++j) R[h.omega[j]] = {0, 0};
    factors_from(h, R);
  }
  finish_refresh(h);
  return 0;
}

void finish_refresh(Orc& h) {
  if (h.o.moments_on_refresh == 1) {
    std::fill(h.core_m.begin(), h.core_m.end(), 0.f);
    std::fill(h.core_v.begin(), h.core_v.end(), 0.f);
    std::fill(h.sp_m.begin(), h.sp_m.end(), 0.f);
    std::fill(h.sp_v.begin(), h.sp_v.end(), 0.f);
  }
  h.has_subspace = true;
  h.refreshes += 1;
}

// ------------------------------------------- low-rank-first order (ablation)
// The decomposition order is a free parameter of the method ([S2]
// "Assumptions & free parameters": sparse then low-rank is the chosen order;
// its ablation reverses it, and [S1] section 五 reports that sparse-first
// wins). Reversed, the low-rank part comes first: the factors are the HOSVD of
// the gradient itself, L = G x_n U_n U_n^H over the projected modes, and Omega
// is selected on E = G - L (E rounded to fp32 and keyed like an fp32 gradient
// of the same kind). A step projects the whole gradient to the core C; the
// sparse values are E at Omega, with L rebuilt from that step's C before Adam;
// the update is rebuilt from the Adam core and the sparse update scattered in,
// as in the sparse-first step.

// X x_n U_n^H (proj) or X x_n U_n over every mode with r_n < I_n, in mode
// order; dims follows the shape.
std::vector<cd> products_all(const Orc& h, const std::vector<std::vector<cd>>& Uc,
                             std::vector<cd> X, std::vector<int64_t>& dims, bool proj) {
  for (int n = 0; n < h.d; ++n) {
    if (h.r[n] == h.I[n]) continue;
    std::vector<int64_t> nd = dims;
    nd[n] = proj ? h.r[n] : h.I[n];
    int64_t sz = 1;
    for (auto v : nd) sz *= v;
    std::vector<cd> Y(sz);
    mode_product(X.data(), dims, n, Uc[n].data(), h.I[n], h.r[n], proj, Y.data(), true);
    X.swap(Y);
    dims = nd;
  }
  return X;
}

std::vector<std::vector<cd>> all_U(const Orc& h) {
  std::vector<std::vector<cd>> Uc(h.d);
  for (int n = 0; n < h.d; ++n) Uc[n] = U_as_cd(h, n);
  return Uc;
}

int refresh_lowrank_first(Orc& h, const void* g) {
  std::vector<cd> G = load_all(g, h.gdt, h.N);
  h.eigval.assign(h.d, {});
  factors_from(h, G);
  const auto Uc = all_U(h);
  std::vector<int64_t> dims(h.I);
  std::vector<cd> C = products_all(h, Uc, G, dims, true);
  std::vector<cd> L = products_all(h, Uc, C, dims, false);
  const int comps = h.cplx ? 2 : 1;
  std::vector<float> Ef(h.N * comps);
  for (int64_t i = 0; i < h.N; ++i) {
    Ef[i * comps] = (float)(G[i].re - L[i].re);
    if (h.cplx) Ef[i * comps + 1] = (float)(G[i].im - L[i].im);
  }
  h.omega.assign(h.k, 0);
  if (h.o.omega_mode == 0)
    topk_select(Ef.data(), h.cplx ? DT_C64 : DT_R32, h.N, h.k, h.omega.data());
  else
    random_select(h.o.seed, (uint64_t)h.refreshes, h.N, h.k, h.omega.data());
  h.omega_val.resize(h.k);
  for (int64_t j = 0; j < h.k; ++j) {
    const int64_t i = h.omega[j];
    h.omega_val[j] = {G[i].re - L[i].re, G[i].im - L[i].im};
  }
  finish_refresh(h);
  return 0;
}

int step_lowrank_first(Orc& h, const void* g, void* w, int64_t nsel, const int64_t* sel,
                       double bc1, double bc2) {
  const int mc = h.mcomp(), vc = h.vcomp();
  std::vector<cd> G = load_all(g, h.gdt, h.N);
  const auto Uc = all_U(h);
  std::vector<int64_t> dims(h.I);
  std::vector<cd> C = products_all(h, Uc, G, dims, true);
  const std::vector<int64_t> core_dims = dims;
  std::vector<cd> L = products_all(h, Uc, C, dims, false);
  std::vector<cd> sparse_upd(h.k);
  for (int64_t j = 0; j < h.k; ++j) {
    const int64_t i = h.omega[j];
    cd e = {G[i].re - L[i].re, G[i].im - L[i].im};
    cd u = adam_update(e, &h.sp_m[j * mc], &h.sp_v[j * vc], h, bc1, bc2);
    sparse_upd[j] = {h.o.sparse_scale * u.re, h.o.sparse_scale * u.im};
  }
  for (int64_t j = 0; j < h.ncore; ++j)
    C[j] = adam_update(C[j], &h.core_m[j * mc], &h.core_v[j * vc], h, bc1, bc2);
  dims = core_dims;
  std::vector<cd> D = products_all(h, Uc, C, dims, false);
  for (int64_t j = 0; j < h.k; ++j) D[h.omega[j]] = D[h.omega[j]] + sparse_upd[j];
  const int64_t slab = h.I[h.d - 2] * h.I[h.d - 1];
  const double decay = 1 - h.lr * h.wd;
  auto update = [&](int64_t e) {
    cd wv = load_elem(w, h.wdt, e);
    store_elem(w, h.wdt, e, {wv.re * decay - h.lr * D[e].re, wv.im * decay - h.lr * D[e].im});
  };
  if (sel) {
    for (int64_t q = 0; q < nsel; ++q)
      for (int64_t e = sel[q] * slab; e < (sel[q] + 1) * slab; ++e) update(e);
  } else {
    for (int64_t e = 0; e < h.N; ++e) update(e);
  }
  h.t += 1;
  return 0;
}

// One optimizer step [S1 section 三, S2, S3]. The weights of the slabs listed
// in `sel` (all slabs when sel is null) are updated; moments and t always
// advance for the whole tensor. A slab is one (I_{d-1} x I_d) plane.
int step(Orc& h, const void* g, void* w, int64_t nsel, const int64_t* sel) {
  if (h.o.auto_refresh && h.T > 0 && h.t % h.T == 0) refresh(h, g);
  if (!h.has_subspace) return 6;
  const int d = h.d;
  const double s = (double)(h.t + 1);
  const double bc1 = 1 - std::pow(h.b1, s), bc2 = 1 - std::pow(h.b2, s);
  if (h.o.order == 1) return step_lowrank_first(h, g, w, nsel, sel, bc1, bc2);
  const int mc = h.mcomp(), vc = h.vcomp();
  // Sparse part: gather on Omega, Adam on the k values, scale by lambda.
  std::vector<cd> sparse_upd(h.k);
  for (int64_t j = 0; j < h.k; ++j) {
    cd gj = load_elem(g, h.gdt, h.omega[j]);
    cd u = adam_update(gj, &h.sp_m[j * mc], &h.sp_v[j * vc], h, bc1, bc2);
    sparse_upd[j] = {h.o.sparse_scale * u.re, h.o.sparse_scale * u.im};
  }
  std::vector<uint8_t> in_omega(h.N, 0);
  for (int64_t j = 0; j < h.k; ++j) in_omega[h.omega[j]] = 1;
  std::vector<std::vector<cd>> Uc(d);
  for (int n = 0; n < d; ++n) Uc[n] = U_as_cd(h, n);
  // Projection of R = G - S: the last two modes slab by slab, then the rest.
  const int64_t Ia = h.I[d - 2], Ib = h.I[d - 1];
  const int64_t ra = h.r[d - 2], rb = h.r[d - 1];
  const int64_t ns = n_slabs(h);
  std::vector<cd> Y(ns * ra * rb);
  parallel_for(ns, [&](int64_t lo, int64_t hi) {
    std::vector<cd> X(Ia * Ib), X1(Ia * rb);
    for (int64_t sl = lo; sl < hi; ++sl) {
      int64_t base = sl * Ia * Ib;
      for (int64_t e = 0; e < Ia * Ib; ++e)
        X[e] = in_omega[base + e] ? cd{0, 0} : load_elem(g, h.gdt, base + e);
      std::vector<int64_t> dims2 = {Ia, Ib};
      if (rb < Ib)
        mode_product(X.data(), dims2, 1, Uc[d - 1].data(), Ib, rb, true, X1.data(), false);
      else
        X1 = X;
      std::vector<int64_t> dims3 = {Ia, rb};
      cd* out = Y.data() + sl * ra * rb;
      if (ra < Ia)
        mode_product(X1.data(), dims3, 0, Uc[d - 2].data(), Ia, ra, true, out, false);
      else
        std::copy(X1.begin(), X1.end(), out);
    }
  });
  std::vector<int64_t> dims(h.I);
  dims[d - 2] = ra;
  dims[d - 1] = rb;
  std::vector<cd> C = std::move(Y);
  for (int n = d - 3; n >= 0; --n) {
    if (h.r[n] == h.I[n]) continue;
    std::vector<int64_t> nd = dims;
    nd[n] = h.r[n];
    int64_t sz = 1;
    for (auto v : nd) sz *= v;
    std::vector<cd> C2(sz);
    mode_product(C.data(), dims, n, Uc[n].data(), h.I[n], h.r[n], true, C2.data(), true);
    C.swap(C2);
    dims = nd;
  }
  // Adam on the core.
  for (int64_t j = 0; j < h.ncore; ++j)
    C[j] = adam_update(C[j], &h.core_m[j * mc], &h.core_v[j * vc], h, bc1, bc2);
  // Reconstruction: leading modes, then the last two slab by slab, with the
  // sparse update added in place and the decoupled AdamW weight update.
  for (int n = 0; n <= d - 3; ++n) {
    if (h.r[n] == h.I[n]) continue;
    std::vector<int64_t> nd = dims;
    nd[n] = h.I[n];
    int64_t sz = 1;
    for (auto v : nd) sz *= v;
    std::vector<cd> C2(sz);
    mode_product(C.data(), dims, n, Uc[n].data(), h.I[n], h.r[n], false, C2.data(), true);
    C.swap(C2);
    dims = nd;
  }
  std::vector<int64_t> slabs;
  if (sel) {
    slabs.assign(sel, sel + nsel);
  } else {
    slabs.resize(ns);
    for (int64_t i = 0; i < ns; ++i) slabs[i] = i;
  }
  const double decay = 1 - h.lr * h.wd;
  parallel_for((int64_t)slabs.size(), [&](int64_t lo, int64_t hi) {
    std::vector<cd> X1(Ia * rb), X(Ia * Ib);
    for (int64_t q = lo; q < hi; ++q) {
      int64_t sl = slabs[q];
      const cd* z = C.data() + sl * ra * rb;
      std::vector<int64_t> dims3 = {ra, rb};
      if (ra < Ia)
        mode_product(z, dims3, 0, Uc[d - 2].data(), Ia, ra, false, X1.data(), false);
      else
        std::copy(z, z + ra * rb, X1.begin());
      std::vector<int64_t> dims2 = {Ia, rb};
      if (rb < Ib)
        mode_product(X1.data(), dims2, 1, Uc[d - 1].data(), Ib, rb, false, X.data(), false);
      else
        X = X1;
      int64_t base = sl * Ia * Ib;
      // Sparse entries of this slab: Omega is ascending, so they are a range.
      auto it0 = std::lower_bound(h.omega.begin(), h.omega.end(), base);
      auto it1 = std::lower_bound(h.omega.begin(), h.omega.end(), base + Ia * Ib);
      for (auto it = it0; it != it1; ++it) {
        int64_t j = it - h.omega.begin();
        X[*it - base] = X[*it - base] + sparse_upd[j];
      }
      for (int64_t e = 0; e < Ia * Ib; ++e) {
        cd wv = load_elem(w, h.wdt, base + e);
        cd nv = {wv.re * decay - h.lr * X[e].re, wv.im * decay - h.lr * X[e].im};
        store_elem(w, h.wdt, base + e, nv);
      }
    }
  });
  h.t += 1;
  return 0;
}

}  // namespace

// ------------------------------------------------------------ C interface
extern "C" {

int orc_version() { return 1; }

void orc_f64_to_f16(const double* x, uint16_t* out, int64_t n) {
  for (int64_t i = 0; i < n; ++i) out[i] = double_to_half(x[i]);
}
void orc_f16_to_f64(const uint16_t* x, double* out, int64_t n) {
  for (int64_t i = 0; i < n; ++i) out[i] = half_to_double(x[i]);
}
void orc_mag_keys(const void* g, int dt, int64_t n, uint32_t* out) {
  for (int64_t i = 0; i < n; ++i) out[i] = mag_key(g, dt, i);
}
void orc_topk(const void* g, int dt, int64_t n, int64_t k, int64_t* out) {
  topk_select(g, dt, n, k, out);
}
uint64_t orc_splitmix64_mix(uint64_t z) { return sm_mix(z); }
uint64_t orc_random_key(uint64_t seed, uint64_t ordinal, uint64_t i) {
  return random_key(seed, ordinal, i);
}
void orc_random_omega(uint64_t seed, uint64_t ordinal, int64_t n, int64_t k, int64_t* out) {
  random_select(seed, ordinal, n, k, out);
}

// x, U, y: complex interleaved fp64. proj != 0: y = x x_n U^H; else x x_n U.
void orc_mode_product(const double* x, int nd, const int64_t* dims, int n, const double* U,
                      int64_t In, int64_t rn, int proj, double* y) {
  std::vector<int64_t> dv(dims, dims + nd);
  mode_product((const cd*)x, dv, n, (const cd*)U, In, rn, proj != 0, (cd*)y, true);
}
void orc_mode_gram(const double* x, int nd, const int64_t* dims, int n, double* out) {
  std::vector<int64_t> dv(dims, dims + nd);
  mode_gram((const cd*)x, dv, n, (cd*)out);
}
// A: n x n complex Hermitian (copied). w: n eigenvalues descending. V: n x n.
void orc_eigh(const double* A, int64_t n, double* w, double* V) {
  std::vector<cd> a((const cd*)A, (const cd*)A + n * n);
  jacobi_eigh(a.data(), n, w, (cd*)V);
}

void* orc_create(int ndim, const int64_t* shape, const int64_t* ranks, double rho, int64_t T,
                 double lr, double b1, double b2, double eps, double wd, int gdt, int wdt,
                 int omega_mode, uint64_t seed, double sparse_scale, int complex_adam,
                 int moments_on_refresh, int auto_refresh) {
  if (ndim < 2 || ndim > 8 || !dt_valid(gdt) || !dt_valid(wdt)) return nullptr;
  if (dt_complex(gdt) != dt_complex(wdt)) return nullptr;
  if (!(rho >= 0 && rho <= 1) || T < 0) return nullptr;
  Orc* h = new Orc;
  h->d = ndim;
  h->N = 1;
  h->ncore = 1;
  for (int n = 0; n < ndim; ++n) {
    if (shape[n] < 1 || ranks[n] < 1 || ranks[n] > shape[n]) {
      delete h;
      return nullptr;
    }
    h->I.push_back(shape[n]);
    h->r.push_back(ranks[n]);
    h->N *= shape[n];
    h->ncore *= ranks[n];
  }
  h->rho = rho;
  h->k = (int64_t)std::floor(rho * (double)h->N);
  h->T = T;
  h->lr = lr;
  h->b1 = b1;
  h->b2 = b2;
  h->eps = eps;
  h->wd = wd;
  h->gdt = gdt;
  h->wdt = wdt;
  h->cplx = dt_complex(gdt);
  h->o = {omega_mode, seed, sparse_scale, complex_adam, moments_on_refresh, auto_refresh};
  h->U.resize(ndim);
  for (int n = 0; n < ndim; ++n) {
    h->U[n].assign(2 * shape[n] * ranks[n], 0.f);
    if (ranks[n] == shape[n])
      for (int64_t i = 0; i < shape[n]; ++i) h->U[n][2 * (i * shape[n] + i)] = 1.f;
  }
  h->core_m.assign(h->ncore * h->mcomp(), 0.f);
  h->core_v.assign(h->ncore * h->vcomp(), 0.f);
  h->sp_m.assign(h->k * h->mcomp(), 0.f);
  h->sp_v.assign(h->k * h->vcomp(), 0.f);
  return h;
}
void orc_destroy(void* h) { delete (Orc*)h; }
// Factor basis: 0 HOSVD eigenvectors (the method), 1 DCT column selection.
int orc_set_basis(void* h, int basis) {
  if (basis < 0 || basis > 1) return 1;
  ((Orc*)h)->o.basis = basis;
  return 0;
}
// Decomposition order: 0 sparse part first (the method), 1 low-rank part first.
int orc_set_order(void* h, int order) {
  if (order < 0 || order > 1) return 1;
  ((Orc*)h)->o.order = order;
  return 0;
}

int orc_refresh(void* h, const void* g) { return refresh(*(Orc*)h, g); }
int orc_step(void* h, const void* g, void* w, int64_t nsel, const int64_t* sel) {
  return step(*(Orc*)h, g, w, nsel, sel);
}

// info: N, k, ncore, nslabs, t, refreshes, has_subspace, mcomp, vcomp
void orc_info(void* hp, int64_t* info) {
  Orc& h = *(Orc*)hp;
  info[0] = h.N;
  info[1] = h.k;
  info[2] = h.ncore;
  info[3] = n_slabs(h);
  info[4] = h.t;
  info[5] = h.refreshes;
  info[6] = h.has_subspace;
  info[7] = h.mcomp();
  info[8] = h.vcomp();
}
void orc_set_counters(void* hp, int64_t t, int64_t refreshes, int has_subspace) {
  Orc& h = *(Orc*)hp;
  h.t = t;
  h.refreshes = refreshes;
  h.has_subspace = has_subspace != 0;
}
void orc_get_omega(void* hp, int64_t* out) {
  Orc& h = *(Orc*)hp;
  std::copy(h.omega.begin(), h.omega.end(), out);
}
void orc_set_omega(void* hp, const int64_t* in) {
  Orc& h = *(Orc*)hp;
  h.omega.assign(in, in + h.k);
}
void orc_get_omega_val(void* hp, double* out) {
  Orc& h = *(Orc*)hp;
  for (int64_t j = 0; j < (int64_t)h.omega_val.size(); ++j) {
    out[2 * j] = h.omega_val[j].re;
    out[2 * j + 1] = h.omega_val[j].im;
  }
}
void orc_get_U(void* hp, int n, float* out) {
  Orc& h = *(Orc*)hp;
  std::copy(h.U[n].begin(), h.U[n].end(), out);
}
void orc_set_U(void* hp, int n, const float* in) {
  Orc& h = *(Orc*)hp;
  std::copy(in, in + h.U[n].size(), h.U[n].begin());
}
// Eigenvalues of mode n's Gram at the last refresh (I_n values, descending);
// returns the count written (0 for identity modes).
int64_t orc_get_eigvals(void* hp, int n, double* out) {
  Orc& h = *(Orc*)hp;
  if (n >= (int)h.eigval.size()) return 0;
  std::copy(h.eigval[n].begin(), h.eigval[n].end(), out);
  return (int64_t)h.eigval[n].size();
}
// which: 0 core_m, 1 core_v, 2 sparse_m, 3 sparse_v
static std::vector<float>& moment(Orc& h, int which) {
  switch (which) {
    case 0: return h.core_m;
    case 1: return h.core_v;
    case 2: return h.sp_m;
    default: return h.sp_v;
  }
}
void orc_get_moment(void* hp, int which, float* out) {
  auto& v = moment(*(Orc*)hp, which);
  std::copy(v.begin(), v.end(), out);
}
void orc_set_moment(void* hp, int which, const float* in) {
  auto& v = moment(*(Orc*)hp, which);
  std::copy(in, in + v.size(), v.begin());
}

}  // extern "C"
