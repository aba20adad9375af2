// Depthwise causal conv1d (width 4) + SiLU, forward and backward.
//
// Defined on "hung-phan ml-skills mamba", section "Mamba: Selective State
// Spaces (S6)": Conv1d(d_inner, d_inner, d_conv, padding=d_conv-1,
// groups=d_inner) on the channel-major activation, first L outputs kept, then
// SiLU. Document resets follow "FLA Mamba and Mamba2" (packing paragraph):
// a tap whose token lies in another document than the output token reads 0.
//
// HBM-bound: each thread owns 8 consecutive tokens of one (b, d) row, read
// and written as one 16-byte vector (bf16) or two (fp32); the 3-token halo
// on each side comes from L1 (its neighbours read those lines).
#include "common.cuh"
#include "internal.h"

namespace ssm {

namespace {

// HALO: the row is a piece of a longer sequence (halo pointers may be set);
// without it the halo code is compiled out of the common path. kT tokens per
// thread (16 without document ids: the 3-token halo is read once per 16).
template <typename T, bool VEC, bool SEQ, bool HALO, int kT>
__global__ void __launch_bounds__(kConvThreads)
conv1d_fwd_kernel(const T* __restrict__ x, const float* __restrict__ w,
                  const float* __restrict__ bias, const int32_t* __restrict__ seq,
                  const T* __restrict__ x_prev, const int32_t* __restrict__ seq_prev,
                  T* __restrict__ u, int D, int L, int silu) {
  const int d = blockIdx.y, b = blockIdx.z;
  const int t0 = (blockIdx.x * kConvThreads + threadIdx.x) * kT;
  if (t0 >= L) return;
  const size_t row = SSM_DIDX(kDbgConvRow, (size_t)b * D + d, 1, (size_t)gridDim.z * D) * L;
  const T* xr = x + row;
  float wk[4];
#pragma unroll
  for (int k = 0; k < 4; ++k) wk[k] = __ldg(w + d * 4 + k);
  const float bs = bias ? __ldg(bias + d) : 0.0f;

  // x[t0-3 .. t0+kT-1]; before token 0 the halo x_prev (the 3 preceding
  // inputs) or 0
  const T* xp = (HALO && x_prev) ? x_prev + ((size_t)b * D + d) * 3 : nullptr;
  float xv[kT + 3];
#pragma unroll
  for (int i = 0; i < 3; ++i) {
    const int s = t0 - 3 + i;
    xv[i] = s >= 0 ? Io<T>::ld(xr + SSM_DIDX(kDbgConvTok, s, 1, L)) : (xp ? Io<T>::ld(xp + 3 + s) : 0.0f);
  }
#pragma unroll
  for (int k = 0; k < kT / 8; ++k) load_row8<T, VEC>(xr, t0 + 8 * k, L, xv + 3 + 8 * k);

  int sg[kT + 3];
  if (SEQ) {
    const int32_t* sr = seq + (size_t)b * L;
#pragma unroll
    for (int i = 0; i < kT + 3; ++i) {
      const int s = t0 - 3 + i;
      sg[i] = (s >= 0 && s < L) ? __ldg(sr + s)
                                : ((HALO && s < 0 && seq_prev) ? __ldg(seq_prev + (size_t)b * 3 + 3 + s) : 0);
    }
  }

#pragma unroll
  for (int k8 = 0; k8 < kT / 8; ++k8) {
    float out[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int ii = 8 * k8 + i;
      float acc = bs;
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        // tap k of output t0+ii reads x_{t0+ii-3+k} = xv[ii+k]; xv is 0 before t=0
        const bool ok = !SEQ || sg[ii + k] == sg[ii + 3];
        acc = fmaf(wk[k], ok ? xv[ii + k] : 0.0f, acc);
      }
      // SiLU with the SFU sigmoid (the fused conv + scan forward computes the
      // same expression, so both store identical u)
      out[i] = silu ? acc * sigmoid_fast(acc) : acc;
    }
    store_row8<T, VEC>(u + row, t0 + 8 * k8, L, out);
  }
}

// dx_s = sum_k w_k dc_{s+3-k} [same document], dc_t = du_t * silu'(c_t).
// Each thread recomputes c_t for its kT tokens plus the 3 after them, writes
// dx for its tokens, and adds its tokens' share of dw and dbias into a
// per-CTA partial (reduced over (b, tile) by conv1d_wreduce_kernel). Without
// document ids kT = 16: the 3-token halos, the recomputed c of the halo and
// the warp reduction of the partials are paid once per 16 tokens (0.195 ->
// 0.174 ms at B2 D1536 L32768 bf16); with them kT = 8, which keeps the
// per-token segment ids within the registers of a full SM.
template <typename T, bool VEC, bool SEQ, bool HALO, int kT>
__global__ void __launch_bounds__(kConvThreads)
conv1d_bwd_kernel(const T* __restrict__ x, const float* __restrict__ w,
                  const float* __restrict__ bias, const int32_t* __restrict__ seq,
                  const T* __restrict__ du, T* __restrict__ dx,
                  float* __restrict__ partial, const T* __restrict__ x_prev,
                  const int32_t* __restrict__ seq_prev, const T* __restrict__ x_next,
                  const T* __restrict__ du_next, const int32_t* __restrict__ seq_next, int D,
                  int L, int silu) {
  const int d = blockIdx.y, b = blockIdx.z;
  const int t0 = (blockIdx.x * kConvThreads + threadIdx.x) * kT;
  const bool live = t0 < L;
  const size_t row = SSM_DIDX(kDbgConvRow, (size_t)b * D + d, live ? 1 : 0, (size_t)gridDim.z * D) * L;
  const T* xr = x + row;
  const T* dur = du + row;
  float wk[4];
#pragma unroll
  for (int k = 0; k < 4; ++k) wk[k] = __ldg(w + d * 4 + k);
  const float bs = bias ? __ldg(bias + d) : 0.0f;

  float xv[kT + 6];   // x[t0-3 .. t0+kT+2]
  float duv[kT + 3];  // du[t0 .. t0+kT+2]
  int sg[kT + 6];     // seg[t0-3 .. t0+kT+2]
#pragma unroll
  for (int i = 0; i < kT + 6; ++i) { xv[i] = 0.0f; sg[i] = 0; }
#pragma unroll
  for (int i = 0; i < kT + 3; ++i) duv[i] = 0.0f;
  // halos of a row cut out of a longer sequence: the 3 inputs before token 0,
  // and the 3 inputs and upstream gradients after token L-1
  const size_t hrow = ((size_t)b * D + d) * 3;
  if (live) {
#pragma unroll
    for (int i = 0; i < 3; ++i) {
      const int s = t0 - 3 + i;
      if (s >= 0) xv[i] = Io<T>::ld(xr + SSM_DIDX(kDbgConvTok, s, 1, L));
      else if (HALO && x_prev) xv[i] = Io<T>::ld(x_prev + hrow + 3 + s);
    }
#pragma unroll
    for (int k = 0; k < kT / 8; ++k) {
      load_row8<T, VEC>(xr, t0 + 8 * k, L, xv + 3 + 8 * k);
      load_row8<T, VEC>(dur, t0 + 8 * k, L, duv + 8 * k);
    }
#pragma unroll
    for (int i = 0; i < 3; ++i) {
      const int s = t0 + kT + i;
      if (s < L) {
        xv[kT + 3 + i] = Io<T>::ld(xr + s);
        duv[kT + i] = Io<T>::ld(dur + s);
      }
    }
    if (HALO && x_next && t0 + kT + 3 > L) {
      // tokens L .. L+2 of the window come from the next piece
#pragma unroll
      for (int i = 3; i < kT + 6; ++i) {
        const int s = t0 - 3 + i;
        if (s >= L && s < L + 3) {
          xv[i] = Io<T>::ld(x_next + hrow + (s - L));
          duv[i - 3] = Io<T>::ld(du_next + hrow + (s - L));
        }
      }
    }
    if (SEQ) {
      const int32_t* sr = seq + (size_t)b * L;
#pragma unroll
      for (int i = 0; i < kT + 6; ++i) {
        const int s = t0 - 3 + i;
        int v = 0;
        if (s >= 0 && s < L) v = __ldg(sr + s);
        else if (HALO && s < 0 && seq_prev) v = __ldg(seq_prev + (size_t)b * 3 + 3 + s);
        else if (HALO && s >= L && s < L + 3 && seq_next)
          v = __ldg(seq_next + (size_t)b * 3 + (s - L));
        sg[i] = v;
      }
    }
  }

  // dc for tokens t0 .. t0+kT+2 (token t0+j: x window xv[j..j+3], segment sg[j+3])
  float dc[kT + 3];
#pragma unroll
  for (int j = 0; j < kT + 3; ++j) {
    float c = bs;
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const bool ok = !SEQ || sg[j + k] == sg[j + 3];
      c = fmaf(wk[k], ok ? xv[j + k] : 0.0f, c);
    }
    float g = duv[j];
    if (silu) {
      const float sgm = sigmoid_fast(c);  // SFU sigmoid, as in the forward
      g *= sgm * (1.0f + c * (1.0f - sgm));
    }
    // tokens past the row exist only as the next piece's halo
    dc[j] = (t0 + j < L || (HALO && x_next && t0 + j < L + 3)) ? g : 0.0f;
  }

  if (live) {
#pragma unroll
    for (int k8 = 0; k8 < kT / 8; ++k8) {
      float o[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const int ii = 8 * k8 + i;
        float acc = 0.0f;
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          const int j = ii + 3 - k;  // output token t0+j uses x_{t0+ii} through tap k
          const bool ok = !SEQ || sg[j + 3] == sg[ii + 3];
          acc = fmaf(wk[k], ok ? dc[j] : 0.0f, acc);
        }
        o[i] = acc;
      }
      store_row8<T, VEC>(dx + row, t0 + 8 * k8, L, o);
    }
  }

  float pw[5] = {0.f, 0.f, 0.f, 0.f, 0.f};
#pragma unroll
  for (int i = 0; i < kT; ++i) {
    // this row's own tokens only (past L, dc is nonzero only with a next-piece halo)
    const float dci = (HALO && t0 + i >= L) ? 0.0f : dc[i];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const bool ok = !SEQ || sg[i + k] == sg[i + 3];
      pw[k] = fmaf(dci, ok ? xv[i + k] : 0.0f, pw[k]);
    }
    pw[4] += dci;
  }
#pragma unroll
  for (int k = 0; k < 5; ++k)
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) pw[k] += __shfl_xor_sync(kFull, pw[k], off);
  __shared__ float red[kConvThreads / 32][5];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (lane == 0)
#pragma unroll
    for (int k = 0; k < 5; ++k) red[warp][k] = pw[k];
  __syncthreads();
  if (threadIdx.x < 5) {
    float s = 0.0f;
#pragma unroll
    for (int wi = 0; wi < kConvThreads / 32; ++wi) s += red[wi][threadIdx.x];
    // the workspace holds conv_tiles(L) tiles per batch entry (1024-token
    // tiles); this launch's tiles are at least as long
    partial[SSM_DIDX(kDbgConvPartial, (((size_t)b * gridDim.x + blockIdx.x) * D + d) * 5 + threadIdx.x,
                     1, (size_t)gridDim.z * conv_tiles(L) * D * 5)] = s;
  }
}

// dw[d][k] = sum over (b, tile) of partial[b][tile][d][k], fixed order.
// ws_tiles: tiles per batch entry the partials buffer was sized for.
__global__ void conv1d_wreduce_kernel(const float* __restrict__ partial, float* __restrict__ dw,
                                      float* __restrict__ dbias, int B, int tiles, int D,
                                      int ws_tiles) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= D * 5) return;
  const int d = i / 5, k = i % 5;
  float s = 0.0f;
  for (int b = 0; b < B; ++b)
    for (int t = 0; t < tiles; ++t)
      s += partial[SSM_DIDX(kDbgConvReduce, (((size_t)b * tiles + t) * D + d) * 5 + k, 1,
                            (size_t)B * ws_tiles * D * 5)];
  if (k < 4) dw[d * 4 + k] = s;
  else if (dbias) dbias[d] = s;
}

template <typename T, bool VEC, bool SEQ, bool HALO>
void conv_fwd_h(const ConvArgs& a, cudaStream_t s) {
  constexpr int kT = SEQ ? 8 : 16;
  dim3 grid((a.L + kConvThreads * kT - 1) / (kConvThreads * kT), a.D, a.B);
  conv1d_fwd_kernel<T, VEC, SEQ, HALO, kT><<<grid, kConvThreads, 0, s>>>(
      static_cast<const T*>(a.x), a.w, a.bias, a.seq, static_cast<const T*>(a.x_prev), a.seq_prev,
      static_cast<T*>(a.out), a.D, a.L, a.silu);
}

template <typename T, bool VEC, bool SEQ>
void conv_fwd_t(const ConvArgs& a, cudaStream_t s) {
  if (a.x_prev) conv_fwd_h<T, VEC, SEQ, true>(a, s);
  else conv_fwd_h<T, VEC, SEQ, false>(a, s);
}

template <typename T, bool VEC, bool SEQ, bool HALO>
void conv_bwd_h(const ConvArgs& a, cudaStream_t s) {
  constexpr int kT = SEQ ? 8 : kConvBwdTok;
  const int tiles = (a.L + kConvThreads * kT - 1) / (kConvThreads * kT);
  dim3 grid(tiles, a.D, a.B);
  conv1d_bwd_kernel<T, VEC, SEQ, HALO, kT><<<grid, kConvThreads, 0, s>>>(
      static_cast<const T*>(a.x), a.w, a.bias, a.seq, static_cast<const T*>(a.du),
      static_cast<T*>(a.out), a.partial, static_cast<const T*>(a.x_prev), a.seq_prev,
      static_cast<const T*>(a.x_next), static_cast<const T*>(a.du_next), a.seq_next, a.D, a.L,
      a.silu);
  const int n = a.D * 5;
  conv1d_wreduce_kernel<<<(n + 255) / 256, 256, 0, s>>>(a.partial, a.dw, a.dbias, a.B,
                                                        tiles, a.D, conv_tiles(a.L));
}

template <typename T, bool VEC, bool SEQ>
void conv_bwd_t(const ConvArgs& a, cudaStream_t s) {
  if (a.x_prev || a.x_next) conv_bwd_h<T, VEC, SEQ, true>(a, s);
  else conv_bwd_h<T, VEC, SEQ, false>(a, s);
}

}  // namespace

cudaError_t launch_conv1d_fwd(const ConvArgs& a, cudaStream_t s) {
  const bool sq = a.seq != nullptr;
  if (a.bf16) {
    if (a.vec) { sq ? conv_fwd_t<__nv_bfloat16, true, true>(a, s) : conv_fwd_t<__nv_bfloat16, true, false>(a, s); }
    else { sq ? conv_fwd_t<__nv_bfloat16, false, true>(a, s) : conv_fwd_t<__nv_bfloat16, false, false>(a, s); }
  } else {
    if (a.vec) { sq ? conv_fwd_t<float, true, true>(a, s) : conv_fwd_t<float, true, false>(a, s); }
    else { sq ? conv_fwd_t<float, false, true>(a, s) : conv_fwd_t<float, false, false>(a, s); }
  }
  return cudaGetLastError();
}

cudaError_t launch_conv1d_bwd(const ConvArgs& a, cudaStream_t s) {
  const bool sq = a.seq != nullptr;
  if (a.bf16) {
    if (a.vec) { sq ? conv_bwd_t<__nv_bfloat16, true, true>(a, s) : conv_bwd_t<__nv_bfloat16, true, false>(a, s); }
    else { sq ? conv_bwd_t<__nv_bfloat16, false, true>(a, s) : conv_bwd_t<__nv_bfloat16, false, false>(a, s); }
  } else {
    if (a.vec) { sq ? conv_bwd_t<float, true, true>(a, s) : conv_bwd_t<float, true, false>(a, s); }
    else { sq ? conv_bwd_t<float, false, true>(a, s) : conv_bwd_t<float, false, false>(a, s); }
  }
  return cudaGetLastError();
}

SSM_DEBUG_TU(conv1d)

}  // namespace ssm

// ---------------------------------------------------------------------------
// Allocation-free variant of the conv1d backward (ssm_conv1d_bwd_noalloc).
// Its scratch (the per-tile dw / dbias partial sums) lives in a fixed
// file-scope device array instead of a caller workspace.
// ---------------------------------------------------------------------------
#include <mutex>

namespace ssm {

namespace {
// 4 MiB on every device that loads the library, held until the process exits.
__device__ __align__(256) float g_conv_bwd_scratch[kConvBwdScratchFloats];

std::mutex g_scratch_mu;
float* g_scratch_ptr[kMaxScratchDevices] = {};  // device address per device ordinal
}  // namespace

// Device address of g_conv_bwd_scratch on the current device. The host-side
// name of the array is only a stand-in; the address is looked up once per
// device (with that device current) and cached.
cudaError_t conv_bwd_scratch(float** ptr) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxScratchDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  if (!g_scratch_ptr[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_conv_bwd_scratch);
    if (e != cudaSuccess) return e;
    g_scratch_ptr[dev] = static_cast<float*>(p);
  }
  *ptr = g_scratch_ptr[dev];
  return cudaSuccess;
}

}  // namespace ssm
