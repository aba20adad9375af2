// Summaries of a whole row and the carry between consecutive pieces of a
// longer sequence (a sequence cut along L, e.g. over ranks).
//
// The recurrence h_t = a_t h_{t-1} + b_t is affine in the state, so a piece
// acts on the state entering it as h_end = P h_in + H with P = prod a over
// the piece and H its end state from zero; pieces compose with the operator
// of "hung-phan ml-skills mamba", section "Hardware-Aware Parallel Scan":
// (a1, b1) + (a2, b2) = (a1 a2, a2 b1 + b2). The adjoint runs the same way
// from the right: the gradient leaving a piece through its start is
// P c + G, with c the gradient of its end state and G the part from the
// piece's own outputs.
#include "common.cuh"
#include "internal.h"

namespace ssm {

namespace {

// Token 0 of row b starts a new document relative to the token before it.
__device__ __forceinline__ bool starts_doc(const int32_t* seq, const int32_t* seq_prev, int b,
                                           int L) {
  return seq && seq_prev && __ldg(seq + (size_t)b * L) != __ldg(seq_prev + b);
}

__global__ void summary_out_kernel(const float* __restrict__ sP, const float* __restrict__ sV,
                                   const int32_t* __restrict__ seq,
                                   const int32_t* __restrict__ seq_prev, int L,
                                   float* __restrict__ decay, float* __restrict__ value, int B,
                                   int D, int N, int Npad, int zero_value) {
  const size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= (size_t)B * D * N) return;
  const size_t r = i / N;
  const int n = (int)(i % N);
  const int b = (int)(r / D);
  // a document start at token 0 cuts the chain: nothing passes the piece's start
  const bool cut = starts_doc(seq, seq_prev, b, L);
  decay[i] = cut ? 0.0f : sP[r * Npad + n];
  value[i] = (cut && zero_value) ? 0.0f : sV[r * Npad + n];
}

// out = the state entering piece r (forward: fold pieces 0 .. r-1 from init,
// 0 when the piece's token 0 starts a document) or the adjoint entering piece
// r from the right (reverse: fold pieces R-1 .. r+1 from init).
__global__ void state_carry_kernel(const float* __restrict__ decay,
                                   const float* __restrict__ value, int R, int r, int reverse,
                                   const float* __restrict__ init,
                                   const int32_t* __restrict__ seq_prev,
                                   const int32_t* __restrict__ seq, int L,
                                   float* __restrict__ out, int B, int D, int N) {
  const size_t per = (size_t)B * D * N;
  const size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= per) return;
  float h = init ? init[i] : 0.0f;
  if (!reverse) {
    for (int j = 0; j < r; ++j) h = fmaf(decay[(size_t)j * per + i], h, value[(size_t)j * per + i]);
    const int b = (int)(i / ((size_t)D * N));
    if (starts_doc(seq, seq_prev, b, L)) h = 0.0f;
  } else {
    for (int j = R - 1; j > r; --j)
      h = fmaf(decay[(size_t)j * per + i], h, value[(size_t)j * per + i]);
  }
  out[i] = h;
}

}  // namespace

cudaError_t launch_summary_out(const float* sP, const float* sV, const int32_t* seq,
                               const int32_t* seq_prev, int L, float* decay, float* value,
                               int B, int D, int N, int Npad, bool zero_value, cudaStream_t s) {
  const size_t n = (size_t)B * D * N;
  summary_out_kernel<<<(unsigned)((n + 255) / 256), 256, 0, s>>>(sP, sV, seq, seq_prev, L, decay,
                                                                 value, B, D, N, Npad,
                                                                 zero_value ? 1 : 0);
  return cudaGetLastError();
}

cudaError_t launch_state_carry(const float* decay, const float* value, int R, int r, bool reverse,
                               const float* init, const int32_t* seq_prev, const int32_t* seq,
                               int L, float* out, int B, int D, int N, cudaStream_t s) {
  const size_t n = (size_t)B * D * N;
  state_carry_kernel<<<(unsigned)((n + 255) / 256), 256, 0, s>>>(decay, value, R, r, reverse ? 1 : 0,
                                                                 init, seq_prev, seq, L, out, B, D, N);
  return cudaGetLastError();
}

SSM_DEBUG_TU(carry)

}  // namespace ssm
