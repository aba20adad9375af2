// Selective scan forward, N = 16 states ("hung-phan ml-skills mamba": the
// S6 block of "Architecture Diagram", the D term of "Core Concept", the
// softplus step and SiLU(z) gate of the S6 sketch):
//   dt_t = softplus(delta_t + bias_d);  a_t = exp(dt_t A_dn) = 2^(dt_t A_dn log2 e)
//   h_t = a_t h_{t-1} + dt_t B_nt u_t;  y_t = sum_n C_nt h_t + D_d u_t;  out_t = y_t silu(z_t)
// with a_t := 0 at the first token of a document ("FLA Mamba and Mamba2",
// packing paragraph).
//
// Layout: a warp holds two rows (lanes 0-15 and 16-31) and walks them in
// 256-token chunks; lane jj of a half owns tokens 16jj .. 16jj+15 of the
// chunk as two 8-token sub-segments a and b whose matching tokens share one
// f32x2 register, so every per-token step of the recurrence is one packed
// instruction for two tokens. States are visited one at a time: the lane
// composes its two sub-segments (the pages' associative operator), joins the
// 16 lanes of its row with a 4-step __shfl_up scan, carries the chunk's end
// state to the next chunk in shared memory and replays its tokens from the
// exact incoming state, accumulating y. The state entering every 8-token
// segment is written for the backward (the pages' recompute-in-backward).
//
// B and C are packed once per call into the lane layout (pack_bc_fwd_kernel)
// and each chunk's 32 KB tile arrives by one TMA bulk copy, one chunk ahead,
// completing on an mbarrier whose wait is bounded.
#include <atomic>
#include <type_traits>

#include "scan16.cuh"

namespace ssm {

namespace {
using namespace s16;

// CTA shapes (warps = row pairs): 4 warps, three CTAs per SM, or 11 warps,
// one per SM (see pick_shape).
constexpr int kFwdWarpsSmall = 4, kFwdWarpsBig = 11;
constexpr unsigned kTileBytes = kFwdTileF4 * 16u;
#ifndef SSM_FWD16_STATES
#define SSM_FWD16_STATES 1
#endif
constexpr int kFwdS = SSM_FWD16_STATES;  // states per iteration of the state loop

template <int W>
struct Fwd16Smem {
  float4 tile[2][kFwdTileF4];  // packed B / C of two chunks
  uint64_t bar[2];             // TMA completion, one phase per use of a buffer
  float H[2 * W][kN];          // state entering the current chunk
  float2 A[2 * W][kN];         // (A log2(e), A log2(e)): an f32x2 operand as loaded
};

template <typename T>
__global__ void pack_bc_fwd_kernel(const T* __restrict__ Bm, const T* __restrict__ Cm,
                                   float4* __restrict__ pk, int L, int nch) {
  const int b = blockIdx.y;
  const int q = blockIdx.x * blockDim.x + threadIdx.x;  // float4 index within batch entry b
  if (q >= nch * kFwdTileF4) return;
  const int c = q / kFwdTileF4, rem = q % kFwdTileF4;
  const int mat = rem / (kN * 64), n = (rem / 64) % kN, f = rem % 64;
  const int k = f >> 4, jj = f & 15;
  const T* src = (mat ? Cm : Bm) + ((size_t)b * kN + n) * L;
  const int t0 = c * kCh + 16 * jj + 2 * k;
  auto g = [&](int t) { return t < L ? Io<T>::ld(src + t) : 0.0f; };
  pk[(size_t)b * nch * kFwdTileF4 + q] = make_float4(g(t0), g(t0 + 8), g(t0 + 1), g(t0 + 9));
}

// Loads 8 consecutive elements (zeros when !ok); VEC: one or two vector loads.
template <typename T, bool VEC>
__device__ __forceinline__ void load8(const T* p, bool ok, float v[8]) {
  if (VEC) {
    Raw8<T> r;
    r.load(p, ok);
#pragma unroll
    for (int i = 0; i < 8; ++i) v[i] = r.get(i);
  } else {
#pragma unroll
    for (int i = 0; i < 8; ++i) v[i] = ok ? Io<T>::ld(p + i) : 0.0f;
  }
}

// CONV: the per-token stream read is x, and u = silu(conv(x)) is computed
// here with exactly the separate conv kernel's operations (four fmaf taps in
// order, document masks, the SFU sigmoid, rounding to T), stored, and scanned.
// XVEC: x is 16-byte aligned (vector loads).
// SUM: the whole-row summary of a piece of a longer sequence instead (the
// product of the decays and the final state from a zero state, into
// split_P / split_H): no y, no checkpoints, no replay.
template <typename T, bool CONV, bool XVEC, int W, bool SUM>
__global__ void __launch_bounds__(W * 32, W < 8 ? 3 : 1) scan16_fwd_kernel(const ScanArgs p) {
  static_assert(!(SUM && CONV), "the summary reads u");
  constexpr int kFwdRows = 2 * W;
  static_assert(sizeof(Fwd16Smem<W>) <= 227 * 1024, "shared memory per CTA");
  extern __shared__ float4 smem_dyn[];
  Fwd16Smem<W>& sm = *reinterpret_cast<Fwd16Smem<W>*>(smem_dyn);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int hf = lane >> 4, jj = lane & 15;
  const int r = 2 * warp + hf;  // row of the CTA
  const int b = blockIdx.y;
  const int d = blockIdx.x * kFwdRows + r;
  const bool active = d < p.D;
  const int L = p.L, nch = p.nchunks;
  const size_t rowid = (size_t)b * p.D + (active ? d : 0);
  const size_t row = SSM_DIDX(kDbgS16Row, rowid, active ? 1 : 0, (size_t)p.B * p.D) * L;
  const T* u_in = static_cast<const T*>(CONV ? p.xconv : p.u) + row;
  const T* dl_in = static_cast<const T*>(p.delta) + row;
  const T* z_in = (p.z && !SUM) ? static_cast<const T*>(p.z) + row : nullptr;
  T* u_out = CONV ? static_cast<T*>(const_cast<void*>(p.u)) + row : nullptr;
  T* out = static_cast<T*>(p.out) + row;
  T* ysv = p.z ? static_cast<T*>(p.ysave) + row : nullptr;
  const int32_t* seqb = p.seq ? p.seq + (size_t)b * L : nullptr;
  const float4* pk = p.bcpack + (size_t)b * nch * kFwdTileF4;
  const int rp = d >> 1;

  if (threadIdx.x == 0) {
    mbar_init(&sm.bar[0], 1);
    mbar_init(&sm.bar[1], 1);
    fence_mbar_init();
  }
  for (int i = threadIdx.x; i < kFwdRows * kN; i += blockDim.x) {
    const int rr = i / kN, n = i % kN, dd = blockIdx.x * kFwdRows + rr;
    const bool act = dd < p.D;
    const float a = act ? __ldg(p.A + (size_t)dd * kN + n) * kLog2e : 0.0f;
    sm.A[rr][n] = make_float2(a, a);
    sm.H[rr][n] = (act && p.h0 && !SUM) ? __ldg(p.h0 + ((size_t)b * p.D + dd) * kN + n) : 0.0f;
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    mbar_expect_tx(&sm.bar[0], kTileBytes);
    tma_load_1d(&sm.tile[0][0], pk, kTileBytes, &sm.bar[0]);
  }
  const float Dv = (active && p.Dskip) ? __ldg(p.Dskip + d) : 0.0f;
  const float bias = (active && p.delta_bias) ? __ldg(p.delta_bias + d) : 0.0f;
  float wk[4] = {0.0f, 0.0f, 0.0f, 0.0f}, cbias = 0.0f, c5 = 0.0f, c6 = 0.0f, c7 = 0.0f;
  // summary: the lane's sum of dt and whether a document starts after token 0
  // (the decay of the piece is exp(A sum dt), or 0 across a start)
  float dt_sum = 0.0f;
  bool any_start = false;
  if (CONV && active) {
#pragma unroll
    for (int k = 0; k < 4; ++k) wk[k] = __ldg(p.conv_w + (size_t)d * 4 + k);
    cbias = p.conv_b ? __ldg(p.conv_b + d) : 0.0f;
  }

  for (int c = 0; c < nch; ++c) {
    const int buf = c & 1;
    const bool ok = mbar_wait_bounded(&sm.bar[buf], (c >> 1) & 1, p.status);
    // also: every thread is done with chunk c - 1, whose buffer is refilled
    // next; all threads leave together on a timeout
    if (!__syncthreads_and(ok)) {
      // the copy into buf has not arrived: wait for it once more (bounded)
      // so that it does not land after the CTA has exited, then stop
      if (threadIdx.x == 0) mbar_wait_bounded(&sm.bar[buf], (c >> 1) & 1, nullptr);
      break;
    }
    if (threadIdx.x == 0 && c + 1 < nch) {
      fence_proxy_async_smem();
      mbar_expect_tx(&sm.bar[buf ^ 1], kTileBytes);
      tma_load_1d(&sm.tile[buf ^ 1][0],
                  pk + SSM_DIDX(kDbgPackBC, (size_t)(c + 1) * kFwdTileF4, kFwdTileF4,
                                (size_t)nch * kFwdTileF4),
                  kTileBytes,
                  &sm.bar[buf ^ 1]);
    }
    const int tl = c * kCh + 16 * jj;
    const bool va = active && tl < L, vb = active && tl + 8 < L;
    // the lane's two 8-token pieces (L is a multiple of 8 on this path)
    const int ta = SSM_DIDX(kDbgS16Tok, tl, va ? 8 : 0, L);
    const int tb = SSM_DIDX(kDbgS16Tok, tl + 8, vb ? 8 : 0, L);
    if (c + 1 < nch && (jj & 3) == 0 && active) {  // the next chunk's lines into L2
      const int tn = tl + kCh;
      if (tn < L) {
        asm volatile("prefetch.global.L2 [%0];" ::"l"(dl_in + tn));
        asm volatile("prefetch.global.L2 [%0];" ::"l"(u_in + tn));
        if (z_in) asm volatile("prefetch.global.L2 [%0];" ::"l"(z_in + tn));
      }
    }

    // per-token values: (sub-segment a, sub-segment b) pairs
    float ua[8], ub[8], da[8], db[8];
    load8<T, (!CONV || XVEC)>(u_in + ta, va, ua);
    load8<T, (!CONV || XVEC)>(u_in + tb, vb, ub);
    load8<T, true>(dl_in + ta, va, da);
    load8<T, true>(dl_in + tb, vb, db);
    // document starts among tokens tl .. tl+15 (bit i), ids tl-3 .. tl+15
    unsigned rm = 0u;
    int sg[19];
    if (seqb) {
#pragma unroll
      for (int i = 0; i < 19; ++i) {
        const int s = tl - 3 + i;
        sg[i] = (s >= 0 && s < L) ? __ldg(seqb + s) : 0;
      }
#pragma unroll
      for (int i = 0; i < 16; ++i)
        if (tl + i > 0 && tl + i < L && sg[i + 3] != sg[i + 2]) rm |= 1u << i;
    }
    if (CONV) {
      float xv[19];
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        xv[3 + i] = ua[i];
        xv[11 + i] = ub[i];
      }
      float h5 = __shfl_up_sync(kFull, xv[16], 1, 16);
      float h6 = __shfl_up_sync(kFull, xv[17], 1, 16);
      float h7 = __shfl_up_sync(kFull, xv[18], 1, 16);
      if (jj == 0) {
        h5 = c5;
        h6 = c6;
        h7 = c7;
      }
      c5 = __shfl_sync(kFull, xv[16], 15, 16);
      c6 = __shfl_sync(kFull, xv[17], 15, 16);
      c7 = __shfl_sync(kFull, xv[18], 15, 16);
      xv[0] = h5;
      xv[1] = h6;
      xv[2] = h7;
      float uo[16];
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        float acc = cbias;
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          const bool okk = !seqb || sg[i + k] == sg[i + 3];
          acc = fmaf(wk[k], okk ? xv[i + k] : 0.0f, acc);
        }
        uo[i] = round_to<T>(acc * sigmoid_fast(acc));
      }
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        ua[i] = uo[i];
        ub[i] = uo[8 + i];
      }
      if (va) store8<T>(u_out + ta, ua);
      if (vb) store8<T>(u_out + tb, ub);
    }
    const bool any_reset = __any_sync(kFull, rm != 0u);
    if constexpr (SUM) any_start = any_start || any_reset;

    float2 dd[8], xx[8], y2[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      float2 v = make_float2(da[i] + bias, db[i] + bias);
      if (p.softplus) v = softplus2(v);
      const float2 dt = make_float2(va ? v.x : 0.0f, vb ? v.y : 0.0f);
      const float2 u2 = make_float2(ua[i], ub[i]);
      dd[i] = dt;
      xx[i] = fmul2(dt, u2);
      y2[i] = make_float2(Dv * u2.x, Dv * u2.y);
      if constexpr (SUM) dt_sum += dt.x + dt.y;
    }

    const float4* tile = &sm.tile[buf][0];
    float* ckc = p.ckpt + ck_chunk(b, rp, p.Dp, nch, c) + hf * kSegs + 2 * jj;
    // the state loop, with document starts in this chunk or without
    auto states = [&](auto RS) {
    // S states per iteration, their chains interleaved (more independent work
    // in flight per warp: the scan's shuffles and the replay's FMA chains)
#pragma unroll 1
    for (int n0 = 0; n0 < kN; n0 += kFwdS) {
      float2 a[kFwdS][8], bx[kFwdS][8], P[kFwdS], H[kFwdS];
      float Pl[kFwdS], Hl[kFwdS], cin[kFwdS];
#pragma unroll
      for (int s = 0; s < kFwdS; ++s) {
        const int n = n0 + s;
        cin[s] = sm.H[r][n];
        const float2 A2 = sm.A[r][n];
        const float4* Bt = tile + n * 64 + jj;
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          const float4 q = Bt[16 * k];
          const float2 e0 = fmul2(dd[2 * k], A2), e1 = fmul2(dd[2 * k + 1], A2);
          a[s][2 * k] = ex2x2(e0);
          a[s][2 * k + 1] = ex2x2(e1);
          bx[s][2 * k] = fmul2(xx[2 * k], make_float2(q.x, q.y));
          bx[s][2 * k + 1] = fmul2(xx[2 * k + 1], make_float2(q.z, q.w));
        }
        if constexpr (decltype(RS)::value) {
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            if ((rm >> i) & 1u) a[s][i].x = 0.0f;
            if ((rm >> (8 + i)) & 1u) a[s][i].y = 0.0f;
          }
        }
        // compose each sub-segment, then b after a: the lane's map h -> Pl h + Hl
        P[s] = a[s][0];
        H[s] = bx[s][0];
#pragma unroll
        for (int i = 1; i < 8; ++i) {
          H[s] = ffma2(a[s][i], H[s], bx[s][i]);
          P[s] = fmul2(P[s], a[s][i]);
        }
        Pl[s] = P[s].x * P[s].y;
        Hl[s] = fmaf(P[s].y, H[s].x, H[s].y);
      }
#pragma unroll
      for (int off = 1; off < 16; off <<= 1)
#pragma unroll
        for (int s = 0; s < kFwdS; ++s) fwd_step16(Pl[s], Hl[s], off);
      float2 h[kFwdS];
#pragma unroll
      for (int s = 0; s < kFwdS; ++s) {
        const int n = n0 + s;
        const float end = fmaf(Pl[s], cin[s], Hl[s]);
        float start = __shfl_up_sync(kFull, end, 1, 16);
        if (jj == 0) start = cin[s];
        if (jj == 15) sm.H[r][n] = end;
        if constexpr (SUM) continue;
        const float sb = fmaf(P[s].x, start, H[s].x);  // state entering sub-segment b
        if (va)
          *reinterpret_cast<float2*>(
              ckc + SSM_DIDX(kDbgS16Ckpt, n * 2 * kSegs, 2, ck_left(p, ckc))) = make_float2(start, sb);
        h[s] = make_float2(start, sb);
      }
      if constexpr (!SUM) {
#pragma unroll
        for (int k = 0; k < 4; ++k) {
#pragma unroll
          for (int s = 0; s < kFwdS; ++s) {
            const float4 q = tile[(kN + n0 + s) * 64 + jj + 16 * k];
            h[s] = ffma2(a[s][2 * k], h[s], bx[s][2 * k]);
            y2[2 * k] = ffma2(make_float2(q.x, q.y), h[s], y2[2 * k]);
            h[s] = ffma2(a[s][2 * k + 1], h[s], bx[s][2 * k + 1]);
            y2[2 * k + 1] = ffma2(make_float2(q.z, q.w), h[s], y2[2 * k + 1]);
          }
        }
      }
    }
    };
    if (any_reset) states(std::true_type{});
    else states(std::false_type{});

    if (!SUM && (va || vb)) {
      const bool vo = (reinterpret_cast<uintptr_t>(p.out) & 15) == 0;  // else element stores
      auto put = [&](T* q, const float v[8]) {
        if (vo) {
          store8<T>(q, v);
        } else {
#pragma unroll
          for (int i = 0; i < 8; ++i) Io<T>::st(q + i, v[i]);
        }
      };
      float ya[8], yb[8], oa[8], ob[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        ya[i] = y2[i].x;
        yb[i] = y2[i].y;
      }
      if (z_in) {
        float za[8], zb[8];
        load8<T, true>(z_in + ta, va, za);
        load8<T, true>(z_in + tb, vb, zb);
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          oa[i] = ya[i] * (za[i] * sigmoid_fast(za[i]));
          ob[i] = yb[i] * (zb[i] * sigmoid_fast(zb[i]));
        }
        if (va) {
          put(out + ta, oa);
          store8<T>(ysv + ta, ya);
        }
        if (vb) {
          put(out + tb, ob);
          store8<T>(ysv + tb, yb);
        }
      } else {
        if (va) put(out + ta, ya);
        if (vb) put(out + tb, yb);
      }
    }
  }

  __syncwarp();
  if constexpr (SUM) {
    // the row's sum of dt over its 16 lanes; lane jj writes state jj
#pragma unroll
    for (int off = 8; off > 0; off >>= 1) dt_sum += __shfl_xor_sync(kFull, dt_sum, off, 16);
    if (active) {
      p.split_P[SSM_DIDX(kDbgS16State, rowid * p.Npad + jj, 1, (size_t)p.B * p.D * p.Npad)] =
          any_start ? 0.0f : ex2_approx(sm.A[r][jj].x * dt_sum);
      p.split_H[SSM_DIDX(kDbgS16State, rowid * p.Npad + jj, 1, (size_t)p.B * p.D * p.Npad)] = sm.H[r][jj];
    }
  } else if (active && p.final_state) {
    p.final_state[SSM_DIDX(kDbgS16State, rowid * kN + jj, 1, (size_t)p.B * p.D * kN)] = sm.H[r][jj];
  }
}


template <typename T, bool CONV, bool XVEC, int W, bool SUM = false>
cudaError_t fwd16_t(const ScanArgs& a, cudaStream_t s) {
  static std::atomic<unsigned long long> done{0};
  const int smem = (int)sizeof(Fwd16Smem<W>);
  cudaError_t e = smem_attr(scan16_fwd_kernel<T, CONV, XVEC, W, SUM>, smem, &done);
  if (e != cudaSuccess) return e;
  const int n4 = a.nchunks * kFwdTileF4;
  pack_bc_fwd_kernel<T><<<dim3((n4 + 255) / 256, a.B), 256, 0, s>>>(
      static_cast<const T*>(a.Bm), static_cast<const T*>(a.Cm), a.bcpack, a.L, a.nchunks);
  dim3 grid((a.D + 2 * W - 1) / (2 * W), a.B);
  scan16_fwd_kernel<T, CONV, XVEC, W, SUM><<<grid, W * 32, smem, s>>>(a);
  return cudaGetLastError();
}

template <int W>
cudaError_t fwd16_dispatch(const ScanArgs& a, cudaStream_t s) {
  const bool xvec = a.xconv && (reinterpret_cast<uintptr_t>(a.xconv) % 16 == 0);
  if (a.bf16) {
    if (!a.xconv) return fwd16_t<__nv_bfloat16, false, true, W>(a, s);
    return xvec ? fwd16_t<__nv_bfloat16, true, true, W>(a, s)
                : fwd16_t<__nv_bfloat16, true, false, W>(a, s);
  }
  if (!a.xconv) return fwd16_t<float, false, true, W>(a, s);
  return xvec ? fwd16_t<float, true, true, W>(a, s) : fwd16_t<float, true, false, W>(a, s);
}

}  // namespace

cudaError_t launch_scan16_fwd(const ScanArgs& a, cudaStream_t s) {
  return s16::pick_shape(a.B, a.D, 2 * kFwdWarpsSmall, 3, 2 * kFwdWarpsBig)
             ? fwd16_dispatch<kFwdWarpsBig>(a, s)
             : fwd16_dispatch<kFwdWarpsSmall>(a, s);
}

cudaError_t launch_scan16_fwd_summary(const ScanArgs& a, cudaStream_t s) {
  const bool big = s16::pick_shape(a.B, a.D, 2 * kFwdWarpsSmall, 3, 2 * kFwdWarpsBig);
  if (a.bf16)
    return big ? fwd16_t<__nv_bfloat16, false, true, kFwdWarpsBig, true>(a, s)
               : fwd16_t<__nv_bfloat16, false, true, kFwdWarpsSmall, true>(a, s);
  return big ? fwd16_t<float, false, true, kFwdWarpsBig, true>(a, s)
             : fwd16_t<float, false, true, kFwdWarpsSmall, true>(a, s);
}

SSM_DEBUG_TU(scan16_fwd)

}  // namespace ssm
