// Device throughput probe: sustained rate of ex2.approx.f32 (the SFU
// instruction every (token, state) step of the scan needs once). Used to
// state the roofline denominator as a measured number.
#include <cuda_runtime.h>

#include "common.cuh"
#include "internal.h"

namespace ssm {

namespace {

constexpr int kProbeIters = 4096;  // per thread, 8 independent chains each

__global__ void __launch_bounds__(256) ex2_probe_kernel(float* __restrict__ sink, float seed) {
  float v[8];
#pragma unroll
  for (int k = 0; k < 8; ++k) v[k] = seed * (threadIdx.x + k + 1) * 1e-6f - 0.5f;
  for (int it = 0; it < kProbeIters; ++it) {
#pragma unroll
    for (int k = 0; k < 8; ++k) v[k] = ex2_approx(v[k]) - 1.5f;  // stays in (-1.5, -0.5)
  }
  float s = 0.0f;
#pragma unroll
  for (int k = 0; k < 8; ++k) s += v[k];
  if (s == 12345.0f) sink[blockIdx.x * blockDim.x + threadIdx.x] = s;  // keeps the chains alive
}

}  // namespace

cudaError_t probe_ex2_rate(float* sink, size_t sink_floats, double* rate, cudaStream_t s) {
  int dev = 0, sms = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e == cudaSuccess) e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  if (e != cudaSuccess) return e;
  const int blocks = sms * 8, threads = 256;
  if ((size_t)blocks * threads > sink_floats) return cudaErrorInvalidValue;
  cudaEvent_t a, b;
  e = cudaEventCreate(&a);
  if (e != cudaSuccess) return e;
  e = cudaEventCreate(&b);
  if (e != cudaSuccess) {
    cudaEventDestroy(a);
    return e;
  }
  ex2_probe_kernel<<<blocks, threads, 0, s>>>(sink, 1.0f);  // warm-up
  cudaEventRecord(a, s);
  const int reps = 5;
  for (int r = 0; r < reps; ++r) ex2_probe_kernel<<<blocks, threads, 0, s>>>(sink, 1.0f + r);
  cudaEventRecord(b, s);
  e = cudaEventSynchronize(b);
  float ms = 0.0f;
  if (e == cudaSuccess) e = cudaEventElapsedTime(&ms, a, b);
  cudaEventDestroy(a);
  cudaEventDestroy(b);
  if (e != cudaSuccess) return e;
  const double n = (double)reps * blocks * threads * kProbeIters * 8;
  *rate = n / (ms * 1e-3);
  return cudaGetLastError();
}

SSM_DEBUG_TU(probe)

}  // namespace ssm
