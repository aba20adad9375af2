// Recurrent form of the layer, one token per row (inference):
// "hung-phan ml-skills mamba", "Dual Computation Modes" (recurrent mode,
// token by token) and "Inference (Generation)" (a (B, D, N) state carried
// forward instead of a KV cache). Same conv, step and state update as the
// sequence kernels, for a single token:
//   c = bias + sum_k w[k] window[k] + w[3] x,  window <- (window[1..2], x)
//   u = silu(c),  dt = softplus(delta + bias)
//   h_n <- exp(dt A_n) h_n + dt B_n u,  y = sum_n C_n h_n + D u,  out = y silu(z)
//
// HBM-bound: per (b, d) the state is read and written once (8 N bytes) plus a
// few activation values. kPerRow threads per (b, d), kNMax / kPerRow states
// each in 16-byte pieces: the state row is read with coalesced 16-byte
// accesses, the per-(b, d) scalar work (conv, SiLU, softplus) is repeated by
// only kPerRow threads, and y is a kPerRow-lane shuffle sum. exp, softplus and sigmoid use the same SFU forms as the
// sequence kernels.
#include "common.cuh"
#include "internal.h"

namespace ssm {

namespace {

#ifndef SSM_DECODE_THREADS_PER_ROW
#define SSM_DECODE_THREADS_PER_ROW 2
#endif
constexpr int kDecThreads = 256;
constexpr int kPerRow = SSM_DECODE_THREADS_PER_ROW;  // threads per (b, d): 1, 2 or 4
constexpr int kPerThr = kNMax / kPerRow;             // states per thread

template <typename T>
__device__ __forceinline__ float ldf(const T* p, size_t i) {
  return Io<T>::ld(p + i);
}

// Four consecutive values of Bm / Cm (VEC: one 8- or 16-byte load).
template <typename T, bool VEC>
__device__ __forceinline__ float4 ld4(const T* p, int n0, int N) {
  if (VEC) {
    if (sizeof(T) == 2) {
      const uint2 r = __ldg(reinterpret_cast<const uint2*>(p + n0));
      return make_float4(bf16lo(r.x), bf16hi(r.x), bf16lo(r.y), bf16hi(r.y));
    }
    return __ldg(reinterpret_cast<const float4*>(p + n0));
  }
  float v[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) v[i] = (n0 + i < N) ? ldf(p, n0 + i) : 0.0f;
  return make_float4(v[0], v[1], v[2], v[3]);
}

// VEC: N == 16 and the state, A, Bm, Cm pointers allow 16-byte (8-byte for
// bf16 Bm / Cm) vector accesses.
// bf16: eight CTAs per SM (at most 32 registers): the step is bound by
// memory latency, and full occupancy keeps a third more of it in flight than
// the 37 registers the compiler would otherwise take (104.8 -> 93.9 us per
// step at 2048 sequences x D1536 x N16). fp32 (40 registers) would spill.
template <typename T, bool VEC>
__global__ void __launch_bounds__(kDecThreads, sizeof(T) == 2 ? 8 : 6) decode_step_kernel(const DecodeArgs a) {
  const size_t g = (size_t)blockIdx.x * (kDecThreads / kPerRow) + threadIdx.x / kPerRow;
  const int q = threadIdx.x % kPerRow;
  const size_t rows = (size_t)a.B * a.D;
  if (g >= rows) return;  // whole 4-lane groups leave together
  const int d = (int)(g % a.D);
  const int b = (int)(g / a.D);
  const int N = a.N;
  // this row's kPerRow lanes
  const unsigned qmask = ((1u << kPerRow) - 1u) << (threadIdx.x & (32 - kPerRow));

  const T* x = static_cast<const T*>(a.x);
  T* win = static_cast<T*>(a.conv_state) + g * 3;
  const float* w = a.conv_w + (size_t)d * 4;
  float c = a.conv_bias ? __ldg(a.conv_bias + d) : 0.0f;
  c = fmaf(__ldg(w + 0), ldf(win, 0), c);
  c = fmaf(__ldg(w + 1), ldf(win, 1), c);
  c = fmaf(__ldg(w + 2), ldf(win, 2), c);
  c = fmaf(__ldg(w + 3), ldf(x, g), c);
  const float u = c * sigmoid_fast(c);
  const float v = ldf(static_cast<const T*>(a.delta), g) + (a.delta_bias ? __ldg(a.delta_bias + d) : 0.0f);
  const float dt = a.softplus ? softplus_sfu(v) : v;
  const float dtl = dt * kLog2e, dtu = dt * u;

  float hy = 0.0f;
#pragma unroll
  for (int j = 0; j < kPerThr / 4; ++j) {  // groups of 4 states
    const int n0 = kPerThr * q + 4 * j;
    if (n0 < N) {
      float* hp = a.state + SSM_DIDX(kDbgDecodeState, g * N + n0, VEC ? 4 : 1, rows * N);
      const float* Ap = a.A + (size_t)d * N + n0;
      const float4 Bv = ld4<T, VEC>(static_cast<const T*>(a.Bm) + (size_t)b * N, n0, N);
      const float4 Cv = ld4<T, VEC>(static_cast<const T*>(a.Cm) + (size_t)b * N, n0, N);
      float h[4], Av[4];
      if (VEC) {
        const float4 h4 = *reinterpret_cast<const float4*>(hp);
        const float4 A4 = __ldg(reinterpret_cast<const float4*>(Ap));
        h[0] = h4.x; h[1] = h4.y; h[2] = h4.z; h[3] = h4.w;
        Av[0] = A4.x; Av[1] = A4.y; Av[2] = A4.z; Av[3] = A4.w;
      } else {
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          h[i] = (n0 + i < N) ? hp[i] : 0.0f;
          Av[i] = (n0 + i < N) ? __ldg(Ap + i) : 0.0f;
        }
      }
      const float bv[4] = {Bv.x, Bv.y, Bv.z, Bv.w}, cv[4] = {Cv.x, Cv.y, Cv.z, Cv.w};
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        h[i] = fmaf(ex2_approx(dtl * Av[i]), h[i], dtu * bv[i]);
        hy = fmaf(cv[i], h[i], hy);
      }
      if (VEC) {
        *reinterpret_cast<float4*>(hp) = make_float4(h[0], h[1], h[2], h[3]);
      } else {
#pragma unroll
        for (int i = 0; i < 4; ++i)
          if (n0 + i < N) hp[i] = h[i];
      }
    }
  }
#pragma unroll
  for (int off = 1; off < kPerRow; off <<= 1) hy += __shfl_xor_sync(qmask, hy, off);

  if (q == 0) {
    float y = fmaf(a.Dskip ? __ldg(a.Dskip + d) : 0.0f, u, hy);
    if (a.z) {
      const float zz = ldf(static_cast<const T*>(a.z), g);
      y *= zz * sigmoid_fast(zz);
    }
    Io<T>::st(static_cast<T*>(a.out) + g, y);
    if (a.u_out) Io<T>::st(static_cast<T*>(a.u_out) + g, u);
    // the window moves by one token (stored input values: no rounding)
    win[0] = win[1];
    win[1] = win[2];
    win[2] = x[g];
  }
}

}  // namespace

cudaError_t launch_decode_step(const DecodeArgs& a, cudaStream_t s) {
  const size_t rows = (size_t)a.B * a.D;
  const size_t per_cta = kDecThreads / kPerRow;
  const unsigned grid = (unsigned)((rows + per_cta - 1) / per_cta);
  if (a.bf16) {
    if (a.vec) decode_step_kernel<__nv_bfloat16, true><<<grid, kDecThreads, 0, s>>>(a);
    else decode_step_kernel<__nv_bfloat16, false><<<grid, kDecThreads, 0, s>>>(a);
  } else {
    if (a.vec) decode_step_kernel<float, true><<<grid, kDecThreads, 0, s>>>(a);
    else decode_step_kernel<float, false><<<grid, kDecThreads, 0, s>>>(a);
  }
  return cudaGetLastError();
}

SSM_DEBUG_TU(decode)

}  // namespace ssm
