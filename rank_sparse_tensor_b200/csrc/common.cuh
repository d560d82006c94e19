// Shared device helpers of the TensorGRaD CUDA library (sm_100a).
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/tgd.h"

namespace tgd {

// Device-side error bits, OR-ed into the handle's error word.
enum : int { DEV_ERR_TIMEOUT = 1, DEV_ERR_BOUNDS = 2 };

// Storage-type traits. DT follows tgd_dtype.
template <int DT> struct Dt;
template <> struct Dt<TGD_R32> {
  static constexpr bool cplx = false;
  static constexpr int bytes = 4;
};
template <> struct Dt<TGD_C64> {
  static constexpr bool cplx = true;
  static constexpr int bytes = 8;
};
template <> struct Dt<TGD_C32H> {
  static constexpr bool cplx = true;
  static constexpr int bytes = 4;
};
template <> struct Dt<TGD_R16> {
  static constexpr bool cplx = false;
  static constexpr int bytes = 2;
};

// Element i of a storage buffer as (re, im) fp32; im = 0 for real types.
template <int DT>
__device__ __forceinline__ float2 load_elem(const void* p, int64_t i) {
  if constexpr (DT == TGD_R32) {
    return make_float2(__ldg((const float*)p + i), 0.f);
  } else if constexpr (DT == TGD_C64) {
    return __ldg((const float2*)p + i);
  } else if constexpr (DT == TGD_C32H) {
    __half2 h = __ldg((const __half2*)p + i);
    return __half22float2(h);
  } else {
    return make_float2(__half2float(__ldg((const __half*)p + i)), 0.f);
  }
}

// Plain (non-read-only-path) load, for buffers that are also written.
template <int DT>
__device__ __forceinline__ float2 load_rw(const void* p, int64_t i) {
  if constexpr (DT == TGD_R32) {
    return make_float2(((const float*)p)[i], 0.f);
  } else if constexpr (DT == TGD_C64) {
    return ((const float2*)p)[i];
  } else if constexpr (DT == TGD_C32H) {
    return __half22float2(((const __half2*)p)[i]);
  } else {
    return make_float2(__half2float(((const __half*)p)[i]), 0.f);
  }
}

// Store with one rounding to the storage type (round to nearest even).
template <int DT>
__device__ __forceinline__ void store_elem(void* p, int64_t i, float2 v) {
  if constexpr (DT == TGD_R32) {
    ((float*)p)[i] = v.x;
  } else if constexpr (DT == TGD_C64) {
    ((float2*)p)[i] = v;
  } else if constexpr (DT == TGD_C32H) {
    ((__half2*)p)[i] = __floats2half2_rn(v.x, v.y);
  } else {
    ((__half*)p)[i] = __float2half_rn(v.x);
  }
}

// Magnitude key: bits of a non-negative fp32 value whose integer order is the
// magnitude order. Real: |g|. Complex: fma(re, re, im * im), each rounded once.
template <int DT>
__device__ __forceinline__ uint32_t mag_key(const void* p, int64_t i) {
  float2 v = load_elem<DT>(p, i);
  if constexpr (Dt<DT>::cplx) {
    return __float_as_uint(__fmaf_rn(v.x, v.x, __fmul_rn(v.y, v.y)));
  } else {
    return __float_as_uint(fabsf(v.x));
  }
}

// splitmix64 output function (Steele, Lea and Flood 2014, Vigna's constants).
__host__ __device__ __forceinline__ uint64_t sm_mix(uint64_t z) {
  z = (z ^ (z >> 30)) * 0xbf58476d1ce4e5b9ULL;
  z = (z ^ (z >> 27)) * 0x94d049bb133111ebULL;
  return z ^ (z >> 31);
}
constexpr uint64_t SM_GAMMA = 0x9e3779b97f4a7c15ULL;

// Adam constants for one step s = t + 1 (bias corrections folded in).
struct AdamConst {
  float b1, b2, omb1, omb2, inv_bc1, inv_bc2, eps, scale;
  int cplx, cmode;  // cmode 0: v = EMA |g|^2; 1: separate re/im moments
};

// scale / (sqrt(x) + eps) without the IEEE slow paths of sqrtf and '/':
// sqrt(x) as x * rsqrt(x) (hardware reciprocal square root, argument kept
// normal) and the approximate divide __fdividef. Both are within 2 ulp, so
// the update's relative error stays near 1e-6, three orders below the fp16
// step tolerance and two below fp32's; being branch-free, many updates per
// thread overlap instead of running one after another.
__device__ __forceinline__ float adam_inv_den(float x, float scale, float eps) {
  const float s = x * rsqrtf(fmaxf(x, 1.17549435e-38f));
  return __fdividef(scale, s + eps);
}

// Updates (m, v) in place from gradient g and returns scale * m_hat /
// (sqrt(v_hat) + eps). m has 1 (real) or 2 (complex) floats, v has 1 or 2.
__device__ __forceinline__ float2 adam_elem(float2 g, float* m, float* v, const AdamConst& a) {
  if (!a.cplx) {
    float m0 = __fmaf_rn(a.b1, m[0], a.omb1 * g.x);
    float v0 = __fmaf_rn(a.b2, v[0], a.omb2 * (g.x * g.x));
    m[0] = m0;
    v[0] = v0;
    return make_float2(m0 * a.inv_bc1 * adam_inv_den(v0 * a.inv_bc2, a.scale, a.eps), 0.f);
  }
  float mr = __fmaf_rn(a.b1, m[0], a.omb1 * g.x);
  float mi = __fmaf_rn(a.b1, m[1], a.omb1 * g.y);
  m[0] = mr;
  m[1] = mi;
  if (a.cmode == 1) {
    float vr = __fmaf_rn(a.b2, v[0], a.omb2 * (g.x * g.x));
    float vi = __fmaf_rn(a.b2, v[1], a.omb2 * (g.y * g.y));
    v[0] = vr;
    v[1] = vi;
    return make_float2(mr * a.inv_bc1 * adam_inv_den(vr * a.inv_bc2, a.scale, a.eps),
                       mi * a.inv_bc1 * adam_inv_den(vi * a.inv_bc2, a.scale, a.eps));
  }
  float v0 = __fmaf_rn(a.b2, v[0], a.omb2 * __fmaf_rn(g.x, g.x, g.y * g.y));
  v[0] = v0;
  float inv = adam_inv_den(v0 * a.inv_bc2, a.scale, a.eps);
  return make_float2(mr * a.inv_bc1 * inv, mi * a.inv_bc1 * inv);
}

__device__ __forceinline__ float2 cfma(float2 a, float2 b, float2 c) {  // a*b + c
  return make_float2(__fmaf_rn(a.x, b.x, __fmaf_rn(-a.y, b.y, c.x)),
                     __fmaf_rn(a.x, b.y, __fmaf_rn(a.y, b.x, c.y)));
}

__device__ __forceinline__ bool mask_bit(const uint32_t* bits, int64_t i) {
  return (__ldg(bits + (i >> 5)) >> (i & 31)) & 1u;
}

inline int64_t ceil_div(int64_t a, int64_t b) { return (a + b - 1) / b; }

}  // namespace tgd
