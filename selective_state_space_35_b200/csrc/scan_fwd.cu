// Selective scan, forward.
//
// Per row (b, d) and state n ("hung-phan ml-skills mamba", S6 block of the
// "Architecture Diagram" section, "Core Concept" for the D term, the S6
// sketch for softplus and the SiLU(z) gate):
//   dt_t = softplus(delta_t + bias_d);  a_t = exp(dt_t A_dn) = 2^(dt_t A_dn log2 e)
//   h_t = a_t h_{t-1} + dt_t B_nt u_t;  y_t = sum_n C_nt h_t + D_d u_t
//   out_t = y_t silu(z_t)
// with a_t := 0 at the first token of a document ("FLA Mamba and Mamba2",
// packing paragraph). The state never leaves the SM; the only state written
// to HBM is one checkpoint per 256-token chunk (read by the backward's
// recompute) and the optional final state.
//
// States are processed two at a time with packed fp32x2 arithmetic: one
// instruction advances states 2m and 2m+1 together, halving the issue slots
// per (token, state) so that the ex2 unit, not instruction issue, bounds the
// kernel. The per-lane inputs of the next chunk are loaded into registers one
// chunk ahead.
//
// Long rows can be split over P CTAs ("n_splits"): pass 1 runs the splits
// 0..P-2 from a zero state and keeps (prod a, h_end) per split, a tiny kernel
// chains these with the associative operator, and pass 2 runs every split
// from its exact incoming state.
#include "scan_common.cuh"

namespace ssm {

namespace {

constexpr int kNP = kNMax / 2;  // state pairs

template <int G>
struct FwdSmem {
  float2 B[kNP * kChunk];                 // B tile, state-pair layout
  float2 C[kNP * kChunk];                 // C tile, state-pair layout
  __nv_bfloat16 raw[2][kNMax][kChunk];    // raw B / C of the next chunk, by TMA
  uint64_t bar;                           // TMA completion (one phase per chunk)
  float2 A[G][kNP];                       // A' = A log2(e), per state pair
  float2 H[G][kNP];                       // running state entering the current chunk
  float2 P[G][kNP];                       // SUMMARY: running product of a over the split
};

// One state pair (2m, 2m+1) of one chunk for one lane, in two halves so that
// the discretisation of pair m+1 (ex2-heavy) can overlap the shuffle-latency-
// bound warp scan of pair m.
// fwd_pair_pre: a = 2^(dt A'), bx = dt u B (ZOH: dt E1(dt A) u B) for the
// lane's 8 tokens.
template <bool ZOH = false>
__device__ __forceinline__ void fwd_pair_pre(int m, int lane, const float2* __restrict__ sBt,
                                             const float2 A2, const float2 dd[8],
                                             const float2 xx[8], unsigned rmask, bool any_reset,
                                             float2 a[8], float2 bx[8]) {
  float2 bv[8];
  lds_pair8(sBt + m * kChunk, lane, bv);
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const float2 e = fmul2(dd[i], A2);
    a[i] = ex2x2(e);
    bx[i] = fmul2(xx[i], bv[i]);
    if (ZOH)
      bx[i] = fmul2(bx[i], f2(zoh_e1(e.x * kLn2, a[i].x), zoh_e1(e.y * kLn2, a[i].y)));
  }
  if (any_reset) {
#pragma unroll
    for (int i = 0; i < 8; ++i)
      if ((rmask >> i) & 1u) a[i] = f2(0.0f, 0.0f);
  }
}

// fwd_pair_post: compose the lane's 8 steps, join the lanes with the warp scan
// (carry-in from the previous chunk in H[m]), and replay to accumulate y.
template <bool SUMMARY>
__device__ __forceinline__ void fwd_pair_post(int m, int lane, const float2* __restrict__ sCt,
                                              float2* sH, float2* sP, const float2 a[8],
                                              const float2 bx[8], float2 y2[8],
                                              float2* __restrict__ ck16) {
  float2 P = a[0], H = bx[0];
#pragma unroll
  for (int i = 1; i < 8; ++i) {
    H = ffma2(a[i], H, bx[i]);
    P = fmul2(P, a[i]);
  }
  warp_scan_fwd2(P, H, lane);
  const float2 cin = sH[m];
  const float2 end = ffma2(P, cin, H);
  float2 start = shfl_up2(end, 1);
  if (lane == 0) start = cin;
  if (lane == 31) {
    sH[m] = end;
    if (SUMMARY) sP[m] = fmul2(sP[m], P);
  }
  if (!SUMMARY) {
    // every other lane starts a 16-token block: keep its entering state
    if ((lane & 1) == 0) ck16[(lane >> 1) * (kNMax / 2) + m] = start;
    float2 cv[8];
    lds_pair8(sCt + m * kChunk, lane, cv);
    float2 h = start;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      h = ffma2(a[i], h, bx[i]);
      y2[i] = ffma2(cv[i], h, y2[i]);
    }
  }
}

// Fused conv: v[8] holds x of the lane's tokens tl .. tl+7 and becomes
// u = silu(bias + sum_k w_k x_{t-3+k}) (taps in another document read 0),
// rounded to the storage type T exactly as the separate conv kernel stores
// it (same operations in the same order, SFU sigmoid), so the fused and
// separate paths agree bitwise.
// The 3-token halo comes from the previous lane; lane 0 takes the previous
// chunk's last three tokens from (c5, c6, c7), which are then advanced.
template <typename T>
__device__ __forceinline__ void conv_silu8(float v[8], float& c5, float& c6, float& c7, int lane,
                                           const float wk[4], float bs,
                                           const int32_t* __restrict__ seqb, int tl, int L) {
  float xv[11];
  xv[0] = __shfl_up_sync(kFull, v[5], 1);
  xv[1] = __shfl_up_sync(kFull, v[6], 1);
  xv[2] = __shfl_up_sync(kFull, v[7], 1);
  if (lane == 0) {
    xv[0] = c5;
    xv[1] = c6;
    xv[2] = c7;
  }
  c5 = __shfl_sync(kFull, v[5], 31);
  c6 = __shfl_sync(kFull, v[6], 31);
  c7 = __shfl_sync(kFull, v[7], 31);
#pragma unroll
  for (int i = 0; i < 8; ++i) xv[3 + i] = v[i];
  int sg[11];
  if (seqb) {
#pragma unroll
    for (int i = 0; i < 11; ++i) {
      const int s = tl - 3 + i;
      sg[i] = (s >= 0 && s < L) ? __ldg(seqb + s) : 0;
    }
  }
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    float acc = bs;
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const bool ok = !seqb || sg[i + k] == sg[i + 3];
      acc = fmaf(wk[k], ok ? xv[i + k] : 0.0f, acc);
    }
    const float uo = acc * sigmoid_fast(acc);
    v[i] = sizeof(T) == 2 ? __bfloat162float(__float2bfloat16_rn(uo)) : uo;
  }
}

// NT: state count fixed at compile time (16), or 0 for any N <= 16.
#ifndef SSM_FWD_MIN_BLOCKS
#define SSM_FWD_MIN_BLOCKS 3
#endif

template <typename T, int G, bool VEC, bool SUMMARY, int NT, bool CONV, bool ZOH>
__global__ void __launch_bounds__(G * 32, SSM_FWD_MIN_BLOCKS)
scan_fwd_kernel(const ScanArgs p) {
  // bf16 on the vector path: B / C tiles arrive by TMA one chunk ahead
  constexpr bool ASYNC = VEC && sizeof(T) == 2;
  extern __shared__ float4 smem_dyn[];
  FwdSmem<G>& sm = *reinterpret_cast<FwdSmem<G>*>(smem_dyn);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int b = blockIdx.y;
  const int d = blockIdx.x * G + warp;
  const bool active = d < p.D;
  const int split = blockIdx.z;
  const int N = NT ? NT : p.N, L = p.L, NP = NT ? (NT + 1) / 2 : p.Npad >> 1;
  const int mats = SUMMARY ? 1 : 2;
  const int c_begin = split * p.chunks_per_split;
  const int c_end = min(c_begin + p.chunks_per_split, p.nchunks);
  const size_t rowid = (size_t)b * p.D + (active ? d : 0);
  const size_t row = SSM_DIDX(kDbgScanRow, rowid, active ? 1 : 0, (size_t)p.B * p.D) * L;

  const T* Bm = static_cast<const T*>(p.Bm);
  const T* Cm = static_cast<const T*>(p.Cm);
  // with the fused conv the per-token stream read here is x, and u is written
  const T* u_row = static_cast<const T*>(CONV ? p.xconv : p.u) + row;
  const T* dl_row = static_cast<const T*>(p.delta) + row;
  const T* z_row = p.z ? static_cast<const T*>(p.z) + row : nullptr;

  if (ASYNC && threadIdx.x == 0) {
    mbar_init(&sm.bar, 1);
    fence_mbar_init();
  }
  __syncthreads();
  if (ASYNC && threadIdx.x < 32)
    tma_issue_bc(reinterpret_cast<const __nv_bfloat16*>(Bm), reinterpret_cast<const __nv_bfloat16*>(Cm),
                 &sm.raw[0][0][0], mats, b, N, L, c_begin * kChunk, &sm.bar);
  if (lane < kNP) {
    float a0 = 0.0f, a1 = 0.0f;
    if (active && 2 * lane < N) a0 = __ldg(p.A + (size_t)d * N + 2 * lane) * kLog2e;
    if (active && 2 * lane + 1 < N) a1 = __ldg(p.A + (size_t)d * N + 2 * lane + 1) * kLog2e;
    sm.A[warp][lane] = f2(a0, a1);
    float2 h0 = f2(0.0f, 0.0f);
    if (!SUMMARY && split > 0 && active && lane < NP)
      h0 = reinterpret_cast<const float2*>(p.split_in)[(rowid * p.nsplits + split) * NP + lane];
    if (!SUMMARY && split == 0 && active && p.h0) {  // the state before token 0
      if (2 * lane < N) h0.x = __ldg(p.h0 + rowid * N + 2 * lane);
      if (2 * lane + 1 < N) h0.y = __ldg(p.h0 + rowid * N + 2 * lane + 1);
    }
    sm.H[warp][lane] = h0;
    sm.P[warp][lane] = f2(1.0f, 1.0f);
  }
  const float Dv = (active && p.Dskip) ? __ldg(p.Dskip + d) : 0.0f;
  const float bias = (active && p.delta_bias) ? __ldg(p.delta_bias + d) : 0.0f;
  float wk[4] = {0.0f, 0.0f, 0.0f, 0.0f}, cbias = 0.0f, c5 = 0.0f, c6 = 0.0f, c7 = 0.0f;
  const int32_t* seqb = p.seq ? p.seq + (size_t)b * L : nullptr;
  if (CONV && active) {
#pragma unroll
    for (int k = 0; k < 4; ++k) wk[k] = __ldg(p.conv_w + (size_t)d * 4 + k);
    cbias = p.conv_b ? __ldg(p.conv_b + d) : 0.0f;
    const int t0 = c_begin * kChunk;  // 0 or >= 256: the halo before it is in range
    if (t0 > 0) {
      c5 = Io<T>::ld(u_row + t0 - 3);
      c6 = Io<T>::ld(u_row + t0 - 2);
      c7 = Io<T>::ld(u_row + t0 - 1);
    }
  }

  Tok8<T, VEC> pf_dl, pf_u, pf_z;
  if (active) {
    const int tl = c_begin * kChunk + lane * 8;
    pf_dl.load(dl_row, tl, L);
    pf_u.load(u_row, tl, L);
    if (!SUMMARY && z_row) pf_z.load(z_row, tl, L);
  }

  for (int c = c_begin; c < c_end; ++c) {
    const int t0 = c * kChunk;
    if (ASYNC) {
      // chunk c is the (c - c_begin)-th phase of the barrier
      const bool ok = mbar_wait_bounded(&sm.bar, (c - c_begin) & 1, p.status);
      // also: every thread is done with chunk c - 1's tiles; all leave together on a timeout,
      // after one more bounded wait for the copy that has not arrived (so that it does
      // not land after the CTA has exited)
      if (!__syncthreads_and(ok)) {
        if (threadIdx.x == 0) mbar_wait_bounded(&sm.bar, (c - c_begin) & 1, nullptr);
        break;
      }
      convert_bc_pairs(&sm.raw[0][0][0], sm.B, sm.C, mats, N, L - t0);
      __syncthreads();  // tiles complete; raw free again
      if (threadIdx.x < 32 && c + 1 < c_end)  // next chunk, hidden behind this chunk's work
        tma_issue_bc(reinterpret_cast<const __nv_bfloat16*>(Bm),
                     reinterpret_cast<const __nv_bfloat16*>(Cm), &sm.raw[0][0][0], mats, b, N, L,
                     t0 + kChunk, &sm.bar);
    } else {
      __syncthreads();
      stage_pairs<T, VEC>(Bm, sm.B, b, N, L, t0);
      if (!SUMMARY) stage_pairs<T, VEC>(Cm, sm.C, b, N, L, t0);
      __syncthreads();
    }
    if (!active) continue;

    const int tl = t0 + lane * 8;
    float dl[8], uu[8], zz[8];
    pf_dl.get(dl);
    pf_u.get(uu);
    if (!SUMMARY && z_row) pf_z.get(zz);
    if (c + 1 < c_end) {  // next chunk's inputs, consumed one iteration later
      pf_dl.load(dl_row, tl + kChunk, L);
      pf_u.load(u_row, tl + kChunk, L);
      if (!SUMMARY && z_row) pf_z.load(z_row, tl + kChunk, L);
    }
    if (CONV) {
      conv_silu8<T>(uu, c5, c6, c7, lane, wk, cbias, seqb, tl, L);
      if (!SUMMARY) store_row8<T, VEC>(static_cast<T*>(const_cast<void*>(p.u)) + row, tl, L, uu);
    }
    float2 dd[8], xx[8], y2[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const float v = dl[i] + bias;
      const float s = p.softplus ? softplus_sfu(v) : v;
      const float dt = (tl + i < L) ? s : 0.0f;  // dt = 0 past the end: a = 1, no input
      dd[i] = f2(dt, dt);
      xx[i] = f2(dt * uu[i], dt * uu[i]);
      y2[i] = f2(Dv * uu[i], 0.0f);  // y starts from the D u feed-through
    }
    const unsigned rmask = reset_mask(p.seq, b, L, tl);
    const bool any_reset = __any_sync(kFull, rmask != 0u);

    // 16-token checkpoints of this chunk: [row][c * 16 + k][kNMax] fp32 pairs
    float2* ck16 = reinterpret_cast<float2*>(p.ckpt) +
                   SSM_DIDX(kDbgScanCkpt, (rowid * p.nchunks + c) * 16 * (kNMax / 2),
                            active ? 16 * (kNMax / 2) : 0,
                            (size_t)p.B * p.D * p.nchunks * 16 * (kNMax / 2));

    if (NT) {
      // compile-time state count: fully unrolled and software-pipelined (the
      // ex2 work of pair m+1 is issued before the scan of pair m)
      float2 a0[8], b0[8];
      fwd_pair_pre<ZOH>(0, lane, sm.B, sm.A[warp][0], dd, xx, rmask, any_reset, a0, b0);
#pragma unroll
      for (int m = 0; m < (NT + 1) / 2; ++m) {
        float2 a1[8], b1[8];
        if (m + 1 < (NT + 1) / 2)
          fwd_pair_pre<ZOH>(m + 1, lane, sm.B, sm.A[warp][m + 1], dd, xx, rmask, any_reset, a1, b1);
        fwd_pair_post<SUMMARY>(m, lane, sm.C, sm.H[warp], sm.P[warp], a0, b0, y2, ck16);
        if (m + 1 < (NT + 1) / 2) {
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            a0[i] = a1[i];
            b0[i] = b1[i];
          }
        }
      }
    } else {
#pragma unroll 1
      for (int m = 0; m < NP; ++m) {
        float2 a0[8], b0[8];
        fwd_pair_pre<ZOH>(m, lane, sm.B, sm.A[warp][m], dd, xx, rmask, any_reset, a0, b0);
        fwd_pair_post<SUMMARY>(m, lane, sm.C, sm.H[warp], sm.P[warp], a0, b0, y2, ck16);
      }
    }

    if (!SUMMARY) {
      float o[8], yv[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        yv[i] = y2[i].x + y2[i].y;
        o[i] = z_row ? yv[i] * (zz[i] * sigmoid_fast(zz[i])) : yv[i];
      }
      store_row8<T, VEC>(static_cast<T*>(p.out) + row, tl, L, o);
      // y before the gate, for the backward's dz
      if (z_row) store_row8<T, VEC>(static_cast<T*>(p.ysave) + row, tl, L, yv);
    }
  }

  __syncwarp();
  if (!active || lane >= NP) return;
  const float2 h = sm.H[warp][lane];
  if (SUMMARY) {
    reinterpret_cast<float2*>(p.split_P)[(rowid * p.nsplits + split) * NP + lane] = sm.P[warp][lane];
    reinterpret_cast<float2*>(p.split_H)[(rowid * p.nsplits + split) * NP + lane] = h;
  } else if (p.final_state && split == p.nsplits - 1) {
    p.final_state[rowid * N + 2 * lane] = h.x;
    if (2 * lane + 1 < N) p.final_state[rowid * N + 2 * lane + 1] = h.y;
  }
}

// Carry into split s: h_in[0] = h0 (0 when absent), h_in[s+1] = P[s] h_in[s] + H[s].
__global__ void fwd_split_carry_kernel(const float* __restrict__ P, const float* __restrict__ H,
                                       const float* __restrict__ h0, float* __restrict__ hin,
                                       int rows, int nsplits, int Np, int N) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= rows * Np) return;
  const int r = i / Np, n = i % Np;
  float h = (h0 && n < N) ? h0[(size_t)r * N + n] : 0.0f;
  for (int s = 0; s < nsplits; ++s) {
    const size_t k = ((size_t)r * nsplits + s) * Np + n;
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

template <typename T, int G, bool VEC, bool SUMMARY, int NT, bool CONV, bool ZOH>
cudaError_t fwd_smem_attr() {
  static std::atomic<unsigned long long> done{0};
  return smem_attr(scan_fwd_kernel<T, G, VEC, SUMMARY, NT, CONV, ZOH>, (int)sizeof(FwdSmem<G>),
                   &done);
}

template <typename T, int G, bool VEC, int NT, bool CONV, bool ZOH>
cudaError_t fwd_t(const ScanArgs& a, cudaStream_t s) {
  dim3 block(G * 32);
  const size_t smem = sizeof(FwdSmem<G>);
  cudaError_t e = fwd_smem_attr<T, G, VEC, false, NT, CONV, ZOH>();
  if (e == cudaSuccess && a.nsplits > 1) e = fwd_smem_attr<T, G, VEC, true, NT, CONV, ZOH>();
  if (e != cudaSuccess) return e;
  if (a.nsplits > 1) {
    dim3 g1((a.D + G - 1) / G, a.B, a.nsplits - 1);
    scan_fwd_kernel<T, G, VEC, true, NT, CONV, ZOH><<<g1, block, smem, s>>>(a);
    const int n = a.B * a.D * a.Npad;
    fwd_split_carry_kernel<<<(n + 255) / 256, 256, 0, s>>>(a.split_P, a.split_H, a.h0, a.split_in,
                                                          a.B * a.D, a.nsplits, a.Npad, a.N);
  }
  dim3 g2((a.D + G - 1) / G, a.B, a.nsplits);
  scan_fwd_kernel<T, G, VEC, false, NT, CONV, ZOH><<<g2, block, smem, s>>>(a);
  return cudaGetLastError();
}

}  // namespace

template <int NT, bool CONV, bool ZOH>
cudaError_t fwd_dispatch(const ScanArgs& a, cudaStream_t s) {
  if (a.bf16)
    return a.vec ? fwd_t<__nv_bfloat16, 4, true, NT, CONV, ZOH>(a, s)
                 : fwd_t<__nv_bfloat16, 4, false, NT, CONV, ZOH>(a, s);
  return a.vec ? fwd_t<float, 4, true, NT, CONV, ZOH>(a, s)
               : fwd_t<float, 4, false, NT, CONV, ZOH>(a, s);
}

cudaError_t launch_scan_fwd(const ScanArgs& a, cudaStream_t s) {
  // zero-order hold: runtime state loop
  if (a.zoh) return a.xconv ? fwd_dispatch<0, true, true>(a, s) : fwd_dispatch<0, false, true>(a, s);
  if (a.xconv) return a.N == 16 ? fwd_dispatch<16, true, false>(a, s) : fwd_dispatch<0, true, false>(a, s);
  return a.N == 16 ? fwd_dispatch<16, false, false>(a, s) : fwd_dispatch<0, false, false>(a, s);
}

namespace {
template <typename T, int G, bool VEC, int NT, bool ZOH>
cudaError_t fwd_summary_t(const ScanArgs& a, cudaStream_t s) {
  cudaError_t e = fwd_smem_attr<T, G, VEC, true, NT, false, ZOH>();
  if (e != cudaSuccess) return e;
  dim3 g((a.D + G - 1) / G, a.B, 1);  // one split: the whole row
  scan_fwd_kernel<T, G, VEC, true, NT, false, ZOH><<<g, G * 32, sizeof(FwdSmem<G>), s>>>(a);
  return cudaGetLastError();
}

template <int NT, bool ZOH>
cudaError_t fwd_summary_dispatch(const ScanArgs& a, cudaStream_t s) {
  if (a.bf16)
    return a.vec ? fwd_summary_t<__nv_bfloat16, 4, true, NT, ZOH>(a, s)
                 : fwd_summary_t<__nv_bfloat16, 4, false, NT, ZOH>(a, s);
  return a.vec ? fwd_summary_t<float, 4, true, NT, ZOH>(a, s)
               : fwd_summary_t<float, 4, false, NT, ZOH>(a, s);
}
}  // namespace

cudaError_t launch_scan_fwd_summary(const ScanArgs& a, cudaStream_t s) {
  if (a.zoh) return fwd_summary_dispatch<0, true>(a, s);
  return a.N == 16 ? fwd_summary_dispatch<16, false>(a, s) : fwd_summary_dispatch<0, false>(a, s);
}

cudaError_t launch_cu_seqlens_to_seq(const int32_t* cu, int n_docs, int L, int32_t* seq,
                                     cudaStream_t s) {
  cu_seqlens_to_seq_kernel<<<(L + 255) / 256, 256, 0, s>>>(cu, n_docs, L, seq);
  return cudaGetLastError();
}

SSM_DEBUG_TU(scan_fwd)

}  // namespace ssm
