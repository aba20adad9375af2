// Selective scan, backward.
//
// Recompute-in-backward ("hung-phan ml-skills mamba", "Hardware-Aware
// Parallel Scan", memory note): the forward keeps only the state entering
// every 256-token chunk; the backward walks each row's chunks in reverse,
// rebuilds the chunk's states h_t from that checkpoint (same warp scan as the
// forward), and runs the adjoint recurrence backwards:
//   g_t = dy_t C_t + a_{t+1} g_{t+1}           (g = dLoss/dh, per state n)
// a reverse warp scan of the maps c -> (prod a) c + G combines the lanes.
// From g and the rebuilt states (q_t = g_t a_t h_{t-1}):
//   du_t   = dy_t D + dt_t sum_n g_t B_nt
//   ddt_t  = u_t sum_n g_t B_nt + sum_n A_n q_t    -> d(raw delta) = ddt * sigmoid(v)
//   dA_n  += dt_t q_t,  dB_nt += g_t dt_t u_t,  dC_nt += dy_t h_t
//   dz_t   = dout_t y_t silu'(z_t),  dD += dy_t u_t
// with dy_t = dout_t silu(z_t). dB and dC sum over every channel of a batch
// row: the CTA's warps add into shared memory, then one fp32 atomic per
// element and CTA goes to HBM. dA, dD and the delta-bias gradient are per-row
// partials reduced over batch (and splits) in a fixed order by a small kernel.
#include "scan_common.cuh"

namespace ssm {

namespace {

template <typename T, int G, bool VEC>
__global__ void __launch_bounds__(G * 32)
scan_bwd_kernel(const ScanArgs p) {
  __shared__ __align__(16) float sB[kNMax * kChunk];
  __shared__ __align__(16) float sC[kNMax * kChunk];
  __shared__ __align__(16) float sRed[2][2][kChunk];  // [n parity][dB | dC][chunk pos]
  __shared__ float sdA[G][kNMax][32];

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
  const T* go_row = static_cast<const T*>(p.dout) + row;

  const float A_lane = (active && lane < N) ? __ldg(p.A + (size_t)d * N + lane) : 0.0f;
  const float A2_lane = A_lane * kLog2e;
  const float Dv = (active && p.Dskip) ? __ldg(p.Dskip + d) : 0.0f;
  const float bias = (active && p.delta_bias) ? __ldg(p.delta_bias + d) : 0.0f;
  // lane n holds c_n = a g of the first token after the current chunk
  float gcarry = 0.0f;
  if (split + 1 < p.nsplits && active && lane < N)
    gcarry = p.split_in[(rowid * p.nsplits + split) * N + lane];

  for (int i = threadIdx.x; i < 4 * kChunk; i += blockDim.x) (&sRed[0][0][0])[i] = 0.0f;
#pragma unroll
  for (int n = 0; n < kNMax; ++n) sdA[warp][n][lane] = 0.0f;
  float dDp = 0.0f, ddbp = 0.0f;

  for (int c = c_end - 1; c >= c_begin; --c) {
    const int t0 = c * kChunk;
    __syncthreads();
    stage_bc<T, VEC>(Bm, Cm, sB, sC, b, N, L, t0);
    __syncthreads();

    const int tl = t0 + lane * 8;
    float dl[8], uu[8], xu[8], dy[8];
    unsigned rmask = 0u;
    float hck = 0.0f;
    if (active) {
      float zz[8], go[8];
      load_row8<T, VEC>(dl_row, tl, L, dl);
      load_row8<T, VEC>(u_row, tl, L, uu);
      load_row8<T, VEC>(go_row, tl, L, go);
      if (z_row) load_row8<T, VEC>(z_row, tl, L, zz);
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const float v = dl[i] + bias;
        const float s = p.softplus ? softplusf_(v) : v;
        dl[i] = (tl + i < L) ? s : 0.0f;
        xu[i] = dl[i] * uu[i];
        dy[i] = z_row ? go[i] * (zz[i] * sigmoidf_(zz[i])) : go[i];
      }
      rmask = reset_mask(p.seq, b, L, tl);
      if (lane < N) hck = p.ckpt[(rowid * p.nchunks + c) * N + lane];
    }
    const bool any_reset = __any_sync(kFull, rmask != 0u);

    float y[8], sgB[8], dd[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) { y[i] = 0.0f; sgB[i] = 0.0f; dd[i] = 0.0f; }

    for (int n = 0; n < N; ++n) {
      float* red = &sRed[n & 1][0][0];
      if (active) {
        const float An2 = __shfl_sync(kFull, A2_lane, n);
        const float Anat = __shfl_sync(kFull, A_lane, n);
        float bv[8], cv[8];
        lds8(sB + n * kChunk, lane, bv);
        lds8(sC + n * kChunk, lane, cv);
        float a[8], bx[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          a[i] = ex2_approx(dl[i] * An2);
          bx[i] = xu[i] * bv[i];
        }
        if (any_reset) {
#pragma unroll
          for (int i = 0; i < 8; ++i)
            if ((rmask >> i) & 1u) a[i] = 0.0f;
        }
        // forward recompute of this lane's 8 states
        float P = 1.0f, H = 0.0f;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          H = fmaf(a[i], H, bx[i]);
          P *= a[i];
        }
        const float Ploc = P;
        warp_scan_fwd(P, H, lane);
        const float hin = __shfl_sync(kFull, hck, n);
        const float end = fmaf(P, hin, H);
        float start = __shfl_up_sync(kFull, end, 1);
        if (lane == 0) start = hin;
        float hs[8];
        float h = start;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          h = fmaf(a[i], h, bx[i]);
          hs[i] = h;
          y[i] = fmaf(cv[i], h, y[i]);
        }
        // adjoint: lane map c_in -> c_out = a_first * g_first
        float gy[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) gy[i] = dy[i] * cv[i];
        float Gl = gy[7];
#pragma unroll
        for (int i = 6; i >= 0; --i) Gl = fmaf(a[i + 1], Gl, gy[i]);
        float Gc = a[0] * Gl;
        float Pr = Ploc;
        warp_scan_bwd(Pr, Gc, lane);
        const float cc = __shfl_sync(kFull, gcarry, n);
        const float cout = fmaf(Pr, cc, Gc);
        float cin = __shfl_down_sync(kFull, cout, 1);
        if (lane == 31) cin = cc;
        const float ncar = __shfl_sync(kFull, cout, 0);
        if (lane == n) gcarry = ncar;

        float g = gy[7] + cin;
        float dAl = 0.0f;
#pragma unroll
        for (int i = 7; i >= 0; --i) {
          if (i < 7) g = fmaf(a[i + 1], g, gy[i]);
          const float hp = i ? hs[i - 1] : start;
          const float q = g * a[i] * hp;
          dAl = fmaf(dl[i], q, dAl);
          dd[i] = fmaf(Anat, q, dd[i]);
          sgB[i] = fmaf(g, bv[i], sgB[i]);
          atomicAdd(red + chunk_pos(lane, i), g * xu[i]);
          atomicAdd(red + kChunk + chunk_pos(lane, i), dy[i] * hs[i]);
        }
        sdA[warp][n][lane] += dAl;
      }
      __syncthreads();
      // flush this state's channel sums: dB, dC [b][n][t0 + tau]
      for (int k = threadIdx.x; k < 2 * kChunk; k += blockDim.x) {
        const int m = k >= kChunk;
        const int tau = k - m * kChunk;
        const int pos = chunk_pos(tau >> 3, tau & 7);
        const float v = red[m * kChunk + pos];
        red[m * kChunk + pos] = 0.0f;
        const int t = t0 + tau;
        if (t < L) atomicAdd((m ? p.dC : p.dB) + ((size_t)b * N + n) * L + t, v);
      }
    }

    if (active) {
      float sgv[8], zz[8], go[8];
      load_row8<T, VEC>(dl_row, tl, L, sgv);
      load_row8<T, VEC>(go_row, tl, L, go);
      if (z_row) load_row8<T, VEC>(z_row, tl, L, zz);
      float o_du[8], o_dd[8], o_dz[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const bool in = tl + i < L;
        const float yfull = fmaf(Dv, uu[i], y[i]);
        o_du[i] = fmaf(dy[i], Dv, dl[i] * sgB[i]);
        const float ddt = fmaf(uu[i], sgB[i], dd[i]);
        const float dv = p.softplus ? ddt * sigmoidf_(sgv[i] + bias) : ddt;
        o_dd[i] = dv;
        if (z_row) {
          const float sz = sigmoidf_(zz[i]);
          o_dz[i] = go[i] * yfull * (sz * (1.0f + zz[i] * (1.0f - sz)));
        }
        if (in) {
          dDp = fmaf(dy[i], uu[i], dDp);
          ddbp += dv;
        }
      }
      store_row8<T, VEC>(static_cast<T*>(p.du) + row, tl, L, o_du);
      store_row8<T, VEC>(static_cast<T*>(p.ddelta) + row, tl, L, o_dd);
      if (z_row) store_row8<T, VEC>(static_cast<T*>(p.dz) + row, tl, L, o_dz);
    }
  }

  if (!active) return;
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) {
    dDp += __shfl_xor_sync(kFull, dDp, off);
    ddbp += __shfl_xor_sync(kFull, ddbp, off);
  }
  __syncwarp();
  const size_t ps = rowid * p.nsplits + split;
  if (lane < N) {
    float s = 0.0f;
    for (int j = 0; j < 32; ++j) s += sdA[warp][lane][j];
    p.part_dA[ps * N + lane] = s;
  }
  if (lane == 0) {
    p.part_dD[ps] = dDp;
    p.part_ddb[ps] = ddbp;
  }
}

// For splits s >= 1: the adjoint map over the whole split, c -> P c + Gc,
// from a zero incoming adjoint (only a, dout, z and C are needed).
template <typename T, int G, bool VEC>
__global__ void __launch_bounds__(G * 32)
scan_bwd_summary_kernel(const ScanArgs p) {
  __shared__ __align__(16) float sC[kNMax * kChunk];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int b = blockIdx.y;
  const int d = blockIdx.x * G + warp;
  const bool active = d < p.D;
  const int split = blockIdx.z + 1;
  const int N = p.N, L = p.L;
  const int c_begin = split * p.chunks_per_split;
  const int c_end = min(c_begin + p.chunks_per_split, p.nchunks);
  const size_t rowid = (size_t)b * p.D + (active ? d : 0);
  const size_t row = rowid * L;
  const T* dl_row = static_cast<const T*>(p.delta) + row;
  const T* z_row = p.z ? static_cast<const T*>(p.z) + row : nullptr;
  const T* go_row = static_cast<const T*>(p.dout) + row;
  const float A2_lane = (active && lane < N) ? __ldg(p.A + (size_t)d * N + lane) * kLog2e : 0.0f;
  const float bias = (active && p.delta_bias) ? __ldg(p.delta_bias + d) : 0.0f;
  float gcarry = 0.0f, Ptot = 1.0f;

  for (int c = c_end - 1; c >= c_begin; --c) {
    const int t0 = c * kChunk;
    __syncthreads();
    stage_bc<T, VEC>(static_cast<const T*>(p.Bm), static_cast<const T*>(p.Cm), nullptr, sC, b,
                     N, L, t0);
    __syncthreads();
    if (!active) continue;
    const int tl = t0 + lane * 8;
    float dl[8], dy[8], zz[8];
    load_row8<T, VEC>(dl_row, tl, L, dl);
    load_row8<T, VEC>(go_row, tl, L, dy);
    if (z_row) load_row8<T, VEC>(z_row, tl, L, zz);
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const float v = dl[i] + bias;
      const float s = p.softplus ? softplusf_(v) : v;
      dl[i] = (tl + i < L) ? s : 0.0f;
      if (z_row) dy[i] *= zz[i] * sigmoidf_(zz[i]);
    }
    const unsigned rmask = reset_mask(p.seq, b, L, tl);
    const bool any_reset = __any_sync(kFull, rmask != 0u);
    for (int n = 0; n < N; ++n) {
      const float An2 = __shfl_sync(kFull, A2_lane, n);
      float cv[8], a[8];
      lds8(sC + n * kChunk, lane, cv);
#pragma unroll
      for (int i = 0; i < 8; ++i) a[i] = ex2_approx(dl[i] * An2);
      if (any_reset) {
#pragma unroll
        for (int i = 0; i < 8; ++i)
          if ((rmask >> i) & 1u) a[i] = 0.0f;
      }
      float P = 1.0f;
#pragma unroll
      for (int i = 0; i < 8; ++i) P *= a[i];
      float Gl = dy[7] * cv[7];
#pragma unroll
      for (int i = 6; i >= 0; --i) Gl = fmaf(a[i + 1], Gl, dy[i] * cv[i]);
      float Gc = a[0] * Gl;
      warp_scan_bwd(P, Gc, lane);
      const float cc = __shfl_sync(kFull, gcarry, n);
      const float cout = fmaf(P, cc, Gc);
      const float ncar = __shfl_sync(kFull, cout, 0);
      const float Pt = __shfl_sync(kFull, P, 0);
      if (lane == n) {
        gcarry = ncar;
        Ptot *= Pt;
      }
    }
  }
  if (!active || lane >= N) return;
  p.split_P[(rowid * p.nsplits + split) * N + lane] = Ptot;
  p.split_H[(rowid * p.nsplits + split) * N + lane] = gcarry;
}

// Adjoint carry into split s from the right: c[P-1] = 0,
// c[s-1] = P[s] c[s] + G[s].
__global__ void bwd_split_carry_kernel(const float* __restrict__ P, const float* __restrict__ Gs,
                                       float* __restrict__ cin, int rows, int nsplits, int N) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= rows * N) return;
  const int r = i / N, n = i % N;
  float c = 0.0f;
  for (int s = nsplits - 1; s >= 0; --s) {
    const size_t k = ((size_t)r * nsplits + s) * N + n;
    cin[k] = c;
    if (s > 0) c = fmaf(P[k], c, Gs[k]);
  }
}

// dA[d][n] = sum_{b, split} part, dD[d], ddelta_bias[d] likewise; fixed order.
__global__ void bwd_param_reduce_kernel(const float* __restrict__ pA, const float* __restrict__ pD,
                                        const float* __restrict__ pB, float* __restrict__ dA,
                                        float* __restrict__ dD, float* __restrict__ ddb, int B,
                                        int D, int N, int nsplits) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i < D * N) {
    const int d = i / N, n = i % N;
    float s = 0.0f;
    for (int b = 0; b < B; ++b)
      for (int q = 0; q < nsplits; ++q) s += pA[(((size_t)b * D + d) * nsplits + q) * N + n];
    dA[i] = s;
  }
  if (i < D) {
    float s1 = 0.0f, s2 = 0.0f;
    for (int b = 0; b < B; ++b)
      for (int q = 0; q < nsplits; ++q) {
        const size_t k = ((size_t)b * D + i) * nsplits + q;
        s1 += pD[k];
        s2 += pB[k];
      }
    if (dD) dD[i] = s1;
    if (ddb) ddb[i] = s2;
  }
}

template <typename T, int G, bool VEC>
cudaError_t bwd_t(const ScanArgs& a, cudaStream_t s) {
  dim3 block(G * 32);
  if (a.nsplits > 1) {
    dim3 g1((a.D + G - 1) / G, a.B, a.nsplits - 1);
    scan_bwd_summary_kernel<T, G, VEC><<<g1, block, 0, s>>>(a);
    const int n = a.B * a.D * a.N;
    bwd_split_carry_kernel<<<(n + 255) / 256, 256, 0, s>>>(a.split_P, a.split_H, a.split_in,
                                                          a.B * a.D, a.nsplits, a.N);
  }
  dim3 g2((a.D + G - 1) / G, a.B, a.nsplits);
  scan_bwd_kernel<T, G, VEC><<<g2, block, 0, s>>>(a);
  const int m = a.D * a.N > a.D ? a.D * a.N : a.D;
  bwd_param_reduce_kernel<<<(m + 255) / 256, 256, 0, s>>>(a.part_dA, a.part_dD, a.part_ddb, a.dA,
                                                         a.dD, a.ddelta_bias, a.B, a.D, a.N,
                                                         a.nsplits);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_scan_bwd(const ScanArgs& a, cudaStream_t s) {
  if (a.bf16) return a.vec ? bwd_t<__nv_bfloat16, 4, true>(a, s) : bwd_t<__nv_bfloat16, 4, false>(a, s);
  return a.vec ? bwd_t<float, 4, true>(a, s) : bwd_t<float, 4, false>(a, s);
}

}  // namespace ssm
