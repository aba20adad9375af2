// Selective scan, forward.
//
// Per row (b, d) and state n ("hung-phan ml-skills mamba", S6 block of the
// "Architecture Diagram" section, "Core Concept" for the D term, the S6
// sketch for softplus and the SiLU(z) gate):
//   dt_t = softplus(delta_t + bias_d);  a_t = exp(dt_t A_dn) = 2^(dt_t A_dn log2 e)
//   h_t = a_t h_{t-1} + dt_t B_nt u_t;  y_t = sum_n C_nt h_t + D_d u_t
//   out_t = y_t silu(z_t)
// with a_t := 0 at the first token of a document ("FLA Mamba and Mamba2",
// packing paragraph). The state never leaves registers; the only state
// written to HBM is one checkpoint per 256-token chunk (read by the
// backward's recompute) and the optional final state.
//
// Long rows can be split over P CTAs ("n_splits"): pass 1 runs the splits
// 0..P-2 from a zero state and keeps (prod a, h_end) per split, a tiny kernel
// chains these with the associative operator, and pass 2 runs every split
// from its exact incoming state.
#include "scan_common.cuh"

namespace ssm {

namespace {

template <typename T, int G, bool VEC, bool SUMMARY>
__global__ void __launch_bounds__(G * 32)
scan_fwd_kernel(const ScanArgs p) {
  __shared__ __align__(16) float sB[kNMax * kChunk];
  __shared__ __align__(16) float sC[kNMax * kChunk];

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int b = blockIdx.y;
  const int d = blockIdx.x * G + warp;
  const bool active = d < p.D;
  const int split = blockIdx.z;
  const int N = p.N, L = p.L;
  const int c_begin = split * p.chunks_per_split;
  const int c_end = min(c_begin + p.chunks_per_split, p.nchunks);
  const size_t rowid = (size_t)b * p.D + (active ? d : 0);
  const size_t row = rowid * L;

  const T* Bm = static_cast<const T*>(p.Bm);
  const T* Cm = static_cast<const T*>(p.Cm);
  const T* u_row = static_cast<const T*>(p.u) + row;
  const T* dl_row = static_cast<const T*>(p.delta) + row;
  const T* z_row = p.z ? static_cast<const T*>(p.z) + row : nullptr;

  // lane n holds A'_n = A_dn log2(e), and the running state h_n
  const float A2_lane = (active && lane < N) ? __ldg(p.A + (size_t)d * N + lane) * kLog2e : 0.0f;
  const float Dv = (active && p.Dskip) ? __ldg(p.Dskip + d) : 0.0f;
  const float bias = (active && p.delta_bias) ? __ldg(p.delta_bias + d) : 0.0f;
  float carry = 0.0f;
  if (!SUMMARY && split > 0 && active && lane < N)
    carry = p.split_in[(rowid * p.nsplits + split) * N + lane];
  float Pacc = 1.0f;  // SUMMARY: lane n holds prod a over the split

  for (int c = c_begin; c < c_end; ++c) {
    const int t0 = c * kChunk;
    __syncthreads();
    stage_bc<T, VEC>(Bm, Cm, sB, SUMMARY ? nullptr : sC, b, N, L, t0);
    __syncthreads();
    if (!active) continue;

    if (!SUMMARY && p.ckpt && lane < N) p.ckpt[(rowid * p.nchunks + c) * N + lane] = carry;

    const int tl = t0 + lane * 8;
    float dl[8], uu[8], xu[8];
    load_row8<T, VEC>(dl_row, tl, L, dl);
    load_row8<T, VEC>(u_row, tl, L, uu);
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const float v = dl[i] + bias;
      const float s = p.softplus ? softplusf_(v) : v;
      dl[i] = (tl + i < L) ? s : 0.0f;  // dt = 0 past the end: a = 1, no input
      xu[i] = dl[i] * uu[i];
    }
    const unsigned rmask = reset_mask(p.seq, b, L, tl);
    const bool any_reset = __any_sync(kFull, rmask != 0u);

    float y[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) y[i] = 0.0f;

    for (int n = 0; n < N; ++n) {
      const float An = __shfl_sync(kFull, A2_lane, n);
      float bv[8];
      lds8(sB + n * kChunk, lane, bv);
      float a[8], bx[8];
      float P = 1.0f, H = 0.0f;
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        a[i] = ex2_approx(dl[i] * An);
        bx[i] = xu[i] * bv[i];
      }
      if (any_reset) {
#pragma unroll
        for (int i = 0; i < 8; ++i)
          if ((rmask >> i) & 1u) a[i] = 0.0f;
      }
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        H = fmaf(a[i], H, bx[i]);
        P *= a[i];
      }
      warp_scan_fwd(P, H, lane);
      const float cin = __shfl_sync(kFull, carry, n);
      const float end = fmaf(P, cin, H);
      float start = __shfl_up_sync(kFull, end, 1);
      if (lane == 0) start = cin;
      const float nc = __shfl_sync(kFull, end, 31);
      if (lane == n) carry = nc;
      if (SUMMARY) {
        const float Pt = __shfl_sync(kFull, P, 31);
        if (lane == n) Pacc *= Pt;
        continue;
      }
      float cv[8];
      lds8(sC + n * kChunk, lane, cv);
      float h = start;
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        h = fmaf(a[i], h, bx[i]);
        y[i] = fmaf(cv[i], h, y[i]);
      }
    }

    if (!SUMMARY) {
      float o[8];
      if (z_row) {
        float zz[8];
        load_row8<T, VEC>(z_row, tl, L, zz);
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const float yy = fmaf(Dv, uu[i], y[i]);
          o[i] = yy * (zz[i] * sigmoidf_(zz[i]));
        }
      } else {
#pragma unroll
        for (int i = 0; i < 8; ++i) o[i] = fmaf(Dv, uu[i], y[i]);
      }
      store_row8<T, VEC>(static_cast<T*>(p.out) + row, tl, L, o);
    }
  }

  if (!active || lane >= N) return;
  if (SUMMARY) {
    p.split_P[(rowid * p.nsplits + split) * N + lane] = Pacc;
    p.split_H[(rowid * p.nsplits + split) * N + lane] = carry;
  } else if (p.final_state && split == p.nsplits - 1) {
    p.final_state[rowid * N + lane] = carry;
  }
}

// Carry into split s: h_in[0] = 0, h_in[s+1] = P[s] h_in[s] + H[s].
__global__ void fwd_split_carry_kernel(const float* __restrict__ P, const float* __restrict__ H,
                                       float* __restrict__ hin, int rows, int nsplits, int N) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= rows * N) return;
  const int r = i / N, n = i % N;
  float h = 0.0f;
  for (int s = 0; s < nsplits; ++s) {
    const size_t k = ((size_t)r * nsplits + s) * N + n;
    hin[k] = h;
    if (s + 1 < nsplits) h = fmaf(P[k], h, H[k]);
  }
}

// seq_idx[t] = index of the document containing t, from cu_seqlens.
__global__ void cu_seqlens_to_seq_kernel(const int32_t* __restrict__ cu, int n_docs, int L,
                                         int32_t* __restrict__ seq) {
  const int t = blockIdx.x * blockDim.x + threadIdx.x;
  if (t >= L) return;
  int lo = 0, hi = n_docs;  // find the last k with cu[k] <= t
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (__ldg(cu + mid) <= t) lo = mid; else hi = mid;
  }
  seq[t] = lo;
}

template <typename T, int G, bool VEC>
cudaError_t fwd_t(const ScanArgs& a, cudaStream_t s) {
  dim3 block(G * 32);
  if (a.nsplits > 1) {
    dim3 g1((a.D + G - 1) / G, a.B, a.nsplits - 1);
    scan_fwd_kernel<T, G, VEC, true><<<g1, block, 0, s>>>(a);
    const int n = a.B * a.D * a.N;
    fwd_split_carry_kernel<<<(n + 255) / 256, 256, 0, s>>>(a.split_P, a.split_H, a.split_in,
                                                          a.B * a.D, a.nsplits, a.N);
  }
  dim3 g2((a.D + G - 1) / G, a.B, a.nsplits);
  scan_fwd_kernel<T, G, VEC, false><<<g2, block, 0, s>>>(a);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_scan_fwd(const ScanArgs& a, cudaStream_t s) {
  if (a.bf16) return a.vec ? fwd_t<__nv_bfloat16, 4, true>(a, s) : fwd_t<__nv_bfloat16, 4, false>(a, s);
  return a.vec ? fwd_t<float, 4, true>(a, s) : fwd_t<float, 4, false>(a, s);
}

cudaError_t launch_cu_seqlens_to_seq(const int32_t* cu, int n_docs, int L, int32_t* seq,
                                     cudaStream_t s) {
  cu_seqlens_to_seq_kernel<<<(L + 255) / 256, 256, 0, s>>>(cu, n_docs, L, seq);
  return cudaGetLastError();
}

}  // namespace ssm
