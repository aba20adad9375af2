// Device-side helpers shared by the conv and scan kernels (sm_100a).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "debug.cuh"

namespace ssm {

constexpr unsigned kFull = 0xffffffffu;
constexpr float kLog2e = 1.4426950408889634f;

// 2^x on the special-function unit (PTX ex2.approx.ftz.f32).
__device__ __forceinline__ float ex2_approx(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ float sigmoidf_(float v) { return 1.0f / (1.0f + expf(-v)); }

// softplus(v) = log(1 + x), x = e^v, without branches: both candidates are
// computed and one is selected (no divergence inside a warp).
//  * x < 1/32: x - x^2/2 + x^3/3 - x^4/4 + x^5/5 (truncation < x^6/6, i.e. a
//    relative error below 5e-9);
//  * otherwise log2(1 + x) on the SFU times ln 2 (log(1+x) > 0.03 there, so
//    the SFU's absolute error of a few 1e-7 and the rounding of 1 + x stay
//    below 1e-5 relative);
//  * v > 20: v (the difference is below 2.1e-9).
__device__ __forceinline__ float softplus_sfu(float v) {
  const float x = __expf(v);
  float q = fmaf(x, 0.2f, -0.25f);
  q = fmaf(x, q, 0.33333334f);
  q = fmaf(x, q, -0.5f);
  q = fmaf(x, q, 1.0f);
  const float series = x * q;
  const float lg = __log2f(1.0f + x) * 0.69314718f;
  const float r = x < 0.03125f ? series : lg;
  return v > 20.0f ? v : r;
}

// sigmoid on the SFU: e^-v via ex2, reciprocal via rcp (relative error a few
// ulp; 1 for v -> +inf, 0 for v -> -inf).
__device__ __forceinline__ float sigmoid_fast(float v) {
  return __fdividef(1.0f, 1.0f + __expf(-v));
}

// Zero-order hold ("Discretization": B_bar = A^{-1} (exp(dt A) - I) B) for
// a diagonal A: B_bar = dt E1(x) B with x = dt A <= 0 and
//   E1(x) = (e^x - 1) / x = sum_k x^k / (k+1)!,
// and d B_bar / dA = dt^2 E2(x) B with
//   E2(x) = (x e^x - e^x + 1) / x^2 = sum_k (k+1) x^k / (k+2)!.
// Both take the series through x^6 for |x| < 1/2 (truncation below 3e-7
// relative) and the closed form from a = e^x otherwise, where a - 1 and
// x a - (a - 1) are far enough from 0 that rounding stays near 1e-6.
// Branch-free: both candidates are computed and one selected.
__device__ __forceinline__ float zoh_e1(float x, float a) {
  float s = fmaf(x, 1.0f / 5040.0f, 1.0f / 720.0f);
  s = fmaf(x, s, 1.0f / 120.0f);
  s = fmaf(x, s, 1.0f / 24.0f);
  s = fmaf(x, s, 1.0f / 6.0f);
  s = fmaf(x, s, 0.5f);
  s = fmaf(x, s, 1.0f);
  const float closed = __fdividef(a - 1.0f, x);
  return fabsf(x) < 0.5f ? s : closed;
}
__device__ __forceinline__ float zoh_e2(float x, float a) {
  float s = fmaf(x, 1.0f / 5760.0f, 1.0f / 840.0f);
  s = fmaf(x, s, 1.0f / 144.0f);
  s = fmaf(x, s, 1.0f / 30.0f);
  s = fmaf(x, s, 1.0f / 8.0f);
  s = fmaf(x, s, 1.0f / 3.0f);
  s = fmaf(x, s, 0.5f);
  const float closed = __fdividef(fmaf(x, a, 1.0f - a), x * x);
  return fabsf(x) < 0.5f ? s : closed;
}
constexpr float kLn2 = 0.6931471805599453f;

// softplus(v) = log(1 + e^v); for v > 20 it equals v to within 2.1e-9.
__device__ __forceinline__ float softplusf_(float v) {
  return v > 20.0f ? v : log1pf(expf(v));
}

// ---------------------------------------------------------------------------
// Element I/O: 8 consecutive elements per thread, fp32 in registers.
// ---------------------------------------------------------------------------
template <typename T>
struct Io;

template <>
struct Io<float> {
  static __device__ __forceinline__ float ld(const float* p) { return __ldg(p); }
  static __device__ __forceinline__ void st(float* p, float v) { *p = v; }
  // p must be 16-byte aligned
  static __device__ __forceinline__ void ld8(const float* p, float v[8]) {
    const float4 a = __ldg(reinterpret_cast<const float4*>(p));
    const float4 b = __ldg(reinterpret_cast<const float4*>(p) + 1);
    v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
    v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
  }
  static __device__ __forceinline__ void st8(float* p, const float v[8]) {
    reinterpret_cast<float4*>(p)[0] = make_float4(v[0], v[1], v[2], v[3]);
    reinterpret_cast<float4*>(p)[1] = make_float4(v[4], v[5], v[6], v[7]);
  }
};

__device__ __forceinline__ float bf16lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16hi(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }

template <>
struct Io<__nv_bfloat16> {
  static __device__ __forceinline__ float ld(const __nv_bfloat16* p) {
    return __bfloat162float(p[0]);
  }
  static __device__ __forceinline__ void st(__nv_bfloat16* p, float v) {
    *p = __float2bfloat16_rn(v);
  }
  static __device__ __forceinline__ void ld8(const __nv_bfloat16* p, float v[8]) {
    const uint4 r = __ldg(reinterpret_cast<const uint4*>(p));
    v[0] = bf16lo(r.x); v[1] = bf16hi(r.x);
    v[2] = bf16lo(r.y); v[3] = bf16hi(r.y);
    v[4] = bf16lo(r.z); v[5] = bf16hi(r.z);
    v[6] = bf16lo(r.w); v[7] = bf16hi(r.w);
  }
  static __device__ __forceinline__ uint32_t pack2(float lo, float hi) {
    __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&h);
  }
  static __device__ __forceinline__ void st8(__nv_bfloat16* p, const float v[8]) {
    uint4 r;
    r.x = pack2(v[0], v[1]);
    r.y = pack2(v[2], v[3]);
    r.z = pack2(v[4], v[5]);
    r.w = pack2(v[6], v[7]);
    *reinterpret_cast<uint4*>(p) = r;
  }
};

// Load 8 elements starting at token t of a row of length L. VEC: L is a
// multiple of 8 and the row is 16-byte aligned, so t < L means all 8 are in
// range. Out-of-range elements read as 0.
template <typename T, bool VEC>
__device__ __forceinline__ void load_row8(const T* row, int t, int L, float v[8]) {
  if (VEC) {
    if (t < L) {
      Io<T>::ld8(row + SSM_DIDX(kDbgRowVec, t, 8, L), v);
    } else {
#pragma unroll
      for (int i = 0; i < 8; ++i) v[i] = 0.0f;
    }
  } else {
#pragma unroll
    for (int i = 0; i < 8; ++i) v[i] = (t + i < L) ? Io<T>::ld(row + t + i) : 0.0f;
  }
}

template <typename T, bool VEC>
__device__ __forceinline__ void store_row8(T* row, int t, int L, const float v[8]) {
  if (VEC) {
    if (t < L) Io<T>::st8(row + SSM_DIDX(kDbgRowVec, t, 8, L), v);
  } else {
#pragma unroll
    for (int i = 0; i < 8; ++i)
      if (t + i < L) Io<T>::st(row + t + i, v[i]);
  }
}

}  // namespace ssm
