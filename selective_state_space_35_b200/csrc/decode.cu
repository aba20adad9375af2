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
// few activation values. 16 threads per (b, d), one per state: the state
// row is one coalesced 64-byte access, the per-(b, d) scalar work is done by
// all 16 threads on broadcast loads, and y is a 16-lane shuffle sum.
#include "common.cuh"
#include "internal.h"

namespace ssm {

namespace {

constexpr int kDecThreads = 256;
constexpr int kGroup = 16;  // threads per (b, d)

template <typename T>
__device__ __forceinline__ float ldf(const T* p, size_t i) {
  return Io<T>::ld(p + i);
}

template <typename T>
__global__ void __launch_bounds__(kDecThreads) decode_step_kernel(const DecodeArgs a) {
  const size_t g = (size_t)blockIdx.x * (kDecThreads / kGroup) + threadIdx.x / kGroup;
  const int n = threadIdx.x % kGroup;
  const size_t rows = (size_t)a.B * a.D;
  if (g >= rows) return;  // whole 16-lane groups leave together
  const int d = (int)(g % a.D);
  const int b = (int)(g / a.D);
  const unsigned gmask = 0xffffu << (threadIdx.x & 16);  // this group's half of the warp

  const T* x = static_cast<const T*>(a.x);
  T* win = static_cast<T*>(a.conv_state) + g * 3;
  const float* w = a.conv_w + (size_t)d * 4;
  const float x0 = ldf(win, 0), x1 = ldf(win, 1), x2 = ldf(win, 2), xt = ldf(x, g);
  float c = a.conv_bias ? __ldg(a.conv_bias + d) : 0.0f;
  c = fmaf(__ldg(w + 0), x0, c);
  c = fmaf(__ldg(w + 1), x1, c);
  c = fmaf(__ldg(w + 2), x2, c);
  c = fmaf(__ldg(w + 3), xt, c);
  const float u = c * sigmoidf_(c);
  const float v = ldf(static_cast<const T*>(a.delta), g) + (a.delta_bias ? __ldg(a.delta_bias + d) : 0.0f);
  const float dt = a.softplus ? softplusf_(v) : v;

  float hy = 0.0f;
  if (n < a.N) {
    float* hp = a.state + g * a.N + n;
    const float An = __ldg(a.A + (size_t)d * a.N + n);
    const float Bn = ldf(static_cast<const T*>(a.Bm), (size_t)b * a.N + n);
    const float Cn = ldf(static_cast<const T*>(a.Cm), (size_t)b * a.N + n);
    const float h = fmaf(expf(dt * An), *hp, dt * Bn * u);
    *hp = h;
    hy = Cn * h;
  }
#pragma unroll
  for (int off = kGroup / 2; off > 0; off >>= 1) hy += __shfl_xor_sync(gmask, hy, off);

  if (n == 0) {
    float y = hy + (a.Dskip ? __ldg(a.Dskip + d) : 0.0f) * u;
    if (a.z) {
      const float zz = ldf(static_cast<const T*>(a.z), g);
      y *= zz * sigmoidf_(zz);
    }
    Io<T>::st(static_cast<T*>(a.out) + g, y);
    if (a.u_out) Io<T>::st(static_cast<T*>(a.u_out) + g, u);
    // the window moves by one token (the inputs are stored values: no rounding)
    win[0] = win[1];
    win[1] = win[2];
    win[2] = x[g];
  }
}

}  // namespace

cudaError_t launch_decode_step(const DecodeArgs& a, cudaStream_t s) {
  const size_t rows = (size_t)a.B * a.D;
  const size_t per_cta = kDecThreads / kGroup;
  const unsigned grid = (unsigned)((rows + per_cta - 1) / per_cta);
  if (a.bf16)
    decode_step_kernel<__nv_bfloat16><<<grid, kDecThreads, 0, s>>>(a);
  else
    decode_step_kernel<float><<<grid, kDecThreads, 0, s>>>(a);
  return cudaGetLastError();
}

}  // namespace ssm
