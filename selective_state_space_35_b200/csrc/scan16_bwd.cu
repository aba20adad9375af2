// Selective scan backward, N = 16 states. Recompute in backward ("hung-phan
// ml-skills mamba", "Hardware-Aware Parallel Scan", memory note): the forward
// kept the state entering every 8-token segment, and each lane rebuilds its
// segment's states from it. The adjoint, g = dL/dh,
//   g_t = dy_t C_t + a_{t+1} g_{t+1}
// runs right to left; with q_t = g_t a_t h_{t-1}:
//   du_t   = dy_t D + dt_t sum_n g_t B_nt
//   ddt_t  = u_t sum_n g_t B_nt + sum_n A_n q_t    -> d(raw delta) = ddt sigmoid(v)
//   dA_n  += dt_t q_t,  dB_nt += g_t dt_t u_t,  dC_nt += dy_t h_t
//   dz_t   = dout_t y_t silu'(z_t),  dD += dy_t u_t,   dy_t = dout_t silu(z_t).
//
// Layout: a warp holds a pair of rows and walks them right to left in
// 256-token chunks, lane j owning tokens 8j .. 8j+7; the two rows share every
// f32x2 register, so each step of both recurrences is one packed instruction
// for the pair. States are visited one at a time. Per state a lane rebuilds
// h over its 8 tokens from the checkpoint, composes its adjoint map
// c -> P c + G (the pages' associative operator), joins the warp's 32 lanes
// with a 5-step __shfl_down scan, takes the chunk's incoming adjoint from
// shared memory and replays its tokens. The sums over states (for du and
// d delta) stay in registers; dA accumulates per lane in shared memory. dB
// and dC (sums over every channel of a batch entry) are added over the row
// pair in registers, over the CTA's 12 rows in shared memory, and sent to
// HBM with one 16-byte reduction per 4 tokens.
//
// B and C chunk tiles arrive in shared memory by TMA bulk copies (no
// multicast), one chunk ahead, completing on an mbarrier with a bounded wait.
#include <atomic>
#include <type_traits>

#include "scan16.cuh"

namespace ssm {

namespace {
using namespace s16;

// CTA shapes (warps = row pairs): 6 warps, two CTAs per SM, or 11 warps, one
// per SM (see pick_shape).
constexpr int kBwdWarpsSmall = 6, kBwdWarpsBig = 11;
static_assert(2 * kBwdWarpsSmall == kBwdCtaRows16, "smallest row group of the dB / dC partials");

template <typename T, int W>
struct Bwd16Smem {
  T tile[2][2][kN][kCh];          // B / C of two chunks, activation dtype
  float4 red[2][W][2][kCh / 4];   // dB / dC of one state (row-pair sums), two states in flight
  float4 pv[W][8][32];            // per lane: (sigma'(v) u, sigma'(v)) of both rows, 8 tokens
  float2 dA[W][kN][32];           // per lane partial dA of both rows
  float4 A[W][kN];                // (A'_r0, A'_r1, A_r0, A_r1), A' = A log2(e)
  float2 car[W][kN];              // adjoint carry entering the chunk from the right
  uint64_t bar[2];
};

// Issue (thread 0) the TMA row copies of chunk c's B / C into tile[buf]:
// 32 rows of ntok elements. The caller zero-filled the tail of a short chunk.
template <typename T, int W>
__device__ __forceinline__ void issue_tile(Bwd16Smem<T, W>& sm, int buf, const T* __restrict__ Bm,
                                           const T* __restrict__ Cm, int b, int L, int c) {
  const int ntok = min(kCh, L - c * kCh);
  const unsigned bytes = static_cast<unsigned>(ntok) * sizeof(T);  // multiple of 16: L % 8 == 0
  fence_proxy_async_smem();
  mbar_expect_tx(&sm.bar[buf], bytes * 2u * kN);
#pragma unroll 1
  for (int i = 0; i < 2 * kN; ++i) {
    const int mat = i / kN, n = i % kN;
    tma_load_1d(&sm.tile[buf][mat][n][0], (mat ? Cm : Bm) + ((size_t)b * kN + n) * L + (size_t)c * kCh,
                bytes, &sm.bar[buf]);
  }
}

// 8 B or C values of tokens 8j .. 8j+7 of state n from a tile.
template <typename T>
__device__ __forceinline__ void lds8(const T* row, int j, float v[8]);
template <>
__device__ __forceinline__ void lds8<__nv_bfloat16>(const __nv_bfloat16* row, int j, float v[8]) {
  const uint4 q = reinterpret_cast<const uint4*>(row)[j];
#pragma unroll
  for (int i = 0; i < 8; ++i) v[i] = bf8(q, i);
}
template <>
__device__ __forceinline__ void lds8<float>(const float* row, int j, float v[8]) {
  const float4 a = reinterpret_cast<const float4*>(row)[2 * j];
  const float4 b = reinterpret_cast<const float4*>(row)[2 * j + 1];
  v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
  v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
}

template <typename T, bool VEC>
__device__ __forceinline__ void ld8(const T* p, bool ok, float v[8]) {
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
template <typename T, bool VEC>
__device__ __forceinline__ void st8(T* p, const float v[8]) {
  if (VEC) {
    store8<T>(p, v);
  } else {
#pragma unroll
    for (int i = 0; i < 8; ++i) Io<T>::st(p + i, v[i]);
  }
}

// VG: the gradient buffers (dout, du, ddelta, dz, dB, dC) allow 16-byte
// vector access.
template <typename T, bool VG, int W>
__global__ void __launch_bounds__(W * 32, W < 8 ? 2 : 1) scan16_bwd_kernel(const ScanArgs p) {
  constexpr int kBwdWarps = W, kBwdRows = 2 * W;
  static_assert(sizeof(Bwd16Smem<T, W>) <= 227 * 1024, "shared memory per CTA");
  extern __shared__ float4 smem_dyn[];
  Bwd16Smem<T, W>& sm = *reinterpret_cast<Bwd16Smem<T, W>*>(smem_dyn);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int b = blockIdx.y;
  const int d0 = blockIdx.x * kBwdRows + 2 * warp;  // rows d0, d0 + 1 (a row pair)
  const bool act0 = d0 < p.D, act1 = d0 + 1 < p.D;
  const int L = p.L, nch = p.nchunks;
  const size_t rid0 = (size_t)b * p.D + (act0 ? d0 : 0);
  const size_t rid1 = (size_t)b * p.D + (act1 ? d0 + 1 : 0);
  const size_t row0 = SSM_DIDX(kDbgS16Row, rid0, act0 ? 1 : 0, (size_t)p.B * p.D) * L;
  const size_t row1 = SSM_DIDX(kDbgS16Row, rid1, act1 ? 1 : 0, (size_t)p.B * p.D) * L;
  const T* Bm = static_cast<const T*>(p.Bm);
  const T* Cm = static_cast<const T*>(p.Cm);
  const bool has_z = p.z != nullptr;
  const int32_t* seqb = p.seq ? p.seq + (size_t)b * L : nullptr;
  const int rp = d0 >> 1;

  if (threadIdx.x == 0) {
    mbar_init(&sm.bar[0], 1);
    mbar_init(&sm.bar[1], 1);
    fence_mbar_init();
  }
  // per-row constants, carries and dA partials
  if (lane < kN) {
    const int n = lane;
    const float a0 = act0 ? __ldg(p.A + (size_t)d0 * kN + n) : 0.0f;
    const float a1 = act1 ? __ldg(p.A + (size_t)(d0 + 1) * kN + n) : 0.0f;
    sm.A[warp][n] = make_float4(a0 * kLog2e, a1 * kLog2e, a0, a1);
    float2 cr = make_float2(0.0f, 0.0f);  // the adjoint entering from the right of the row
    if (p.dhL) {
      if (act0) cr.x = __ldg(p.dhL + rid0 * kN + n);
      if (act1) cr.y = __ldg(p.dhL + rid1 * kN + n);
    }
    sm.car[warp][n] = cr;
  }
#pragma unroll
  for (int n = 0; n < kN; ++n) sm.dA[warp][n][lane] = make_float2(0.0f, 0.0f);
  // a short last chunk: zero the tile tail its copies leave untouched
  const int last = nch - 1;
  const int ntail = L - last * kCh;
  if (ntail < kCh) {
    for (int i = threadIdx.x; i < 2 * kN * (kCh - ntail); i += blockDim.x) {
      const int rr = i / (kCh - ntail), t = ntail + i % (kCh - ntail);
      (&sm.tile[last & 1][0][0][0])[rr * kCh + t] = T(0.0f);
    }
  }
  __syncthreads();
  if (threadIdx.x == 0) issue_tile(sm, last & 1, Bm, Cm, b, L, last);

  const float2 Dv = make_float2((act0 && p.Dskip) ? __ldg(p.Dskip + d0) : 0.0f,
                                (act1 && p.Dskip) ? __ldg(p.Dskip + d0 + 1) : 0.0f);
  const float2 bias = make_float2((act0 && p.delta_bias) ? __ldg(p.delta_bias + d0) : 0.0f,
                                  (act1 && p.delta_bias) ? __ldg(p.delta_bias + d0 + 1) : 0.0f);
  float2 dDp = make_float2(0.0f, 0.0f), ddbp = make_float2(0.0f, 0.0f);
  int k_use = 0;  // uses of the tile buffers so far (phase bookkeeping)

#pragma unroll 1
  for (int c = last; c >= 0; --c, ++k_use) {
    const int buf = c & 1;
    // chunk c is the (k_use >> 1)-th use of buffer buf (buffers alternate)
    const bool ok = mbar_wait_bounded(&sm.bar[buf], (k_use >> 1) & 1, p.status);
    if (!__syncthreads_and(ok)) {
      // the copy into buf has not arrived: wait for it once more (bounded)
      // so that it does not land after the CTA has exited, then stop
      if (threadIdx.x == 0) mbar_wait_bounded(&sm.bar[buf], (k_use >> 1) & 1, nullptr);
      break;
    }
    if (threadIdx.x == 0 && c >= 1) issue_tile(sm, buf ^ 1, Bm, Cm, b, L, c - 1);

    const int tl = c * kCh + 8 * lane;
    const bool valid = tl < L;
    const bool ok0 = valid && act0, ok1 = valid && act1;
    // the lane's 8 tokens of each row (L is a multiple of 8 on this path)
    const int t0o = SSM_DIDX(kDbgS16Tok, tl, ok0 ? 8 : 0, L);
    const int t1o = SSM_DIDX(kDbgS16Tok, tl, ok1 ? 8 : 0, L);
    const float* ckc = p.ckpt + ck_chunk(b, rp, p.Dp, nch, c) + lane;
    if (c >= 1) {  // the next chunk's lines into L2
      const int tn = tl - kCh;
      asm volatile("prefetch.global.L2 [%0];" ::"l"(p.ckpt + ck_chunk(b, rp, p.Dp, nch, c - 1) + 32 * lane));
      if ((lane & 7) == 0) {
        const T* arrs[5] = {static_cast<const T*>(p.delta), static_cast<const T*>(p.u),
                            static_cast<const T*>(p.dout), has_z ? static_cast<const T*>(p.z) : nullptr,
                            has_z ? static_cast<const T*>(p.ysave) : nullptr};
#pragma unroll
        for (int k = 0; k < 5; ++k)
          if (arrs[k]) {
            if (act0) asm volatile("prefetch.global.L2 [%0];" ::"l"(arrs[k] + row0 + tn));
            if (act1) asm volatile("prefetch.global.L2 [%0];" ::"l"(arrs[k] + row1 + tn));
          }
      }
    }

    // ---- per-token values of both rows: (row 0, row 1) pairs per token ----
    float2 dd[8], xx[8], dy[8];
    {
      float dl0[8], dl1[8], u0[8], u1[8], g0[8], g1[8];
      ld8<T, true>(static_cast<const T*>(p.delta) + row0 + t0o, ok0, dl0);
      ld8<T, true>(static_cast<const T*>(p.delta) + row1 + t1o, ok1, dl1);
      ld8<T, true>(static_cast<const T*>(p.u) + row0 + t0o, ok0, u0);
      ld8<T, true>(static_cast<const T*>(p.u) + row1 + t1o, ok1, u1);
      ld8<T, VG>(static_cast<const T*>(p.dout) + row0 + t0o, ok0, g0);
      ld8<T, VG>(static_cast<const T*>(p.dout) + row1 + t1o, ok1, g1);
      float dz0[8], dz1[8];
      if (has_z) {
        float z0[8], z1[8], y0[8], y1[8];
        ld8<T, true>(static_cast<const T*>(p.z) + row0 + t0o, ok0, z0);
        ld8<T, true>(static_cast<const T*>(p.z) + row1 + t1o, ok1, z1);
        ld8<T, true>(static_cast<const T*>(p.ysave) + row0 + t0o, ok0, y0);
        ld8<T, true>(static_cast<const T*>(p.ysave) + row1 + t1o, ok1, y1);
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const float s0 = sigmoid_fast(z0[i]), s1 = sigmoid_fast(z1[i]);
          dz0[i] = g0[i] * y0[i] * (s0 * (1.0f + z0[i] * (1.0f - s0)));
          dz1[i] = g1[i] * y1[i] * (s1 * (1.0f + z1[i] * (1.0f - s1)));
          g0[i] *= z0[i] * s0;
          g1[i] *= z1[i] * s1;
        }
        if (ok0) st8<T, VG>(static_cast<T*>(p.dz) + row0 + t0o, dz0);
        if (ok1) st8<T, VG>(static_cast<T*>(p.dz) + row1 + t1o, dz1);
      }
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const float2 v = make_float2(dl0[i] + bias.x, dl1[i] + bias.y);
        float2 dt = v, sp = make_float2(1.0f, 1.0f);
        if (p.softplus) {
          dt = softplus2(v);
          // d softplus(v) / dv = sigmoid(v)
          sp = make_float2(v.x > 20.0f ? 1.0f : sigmoid_fast(v.x), v.y > 20.0f ? 1.0f : sigmoid_fast(v.y));
        }
        dt = make_float2(ok0 ? dt.x : 0.0f, ok1 ? dt.y : 0.0f);
        const float2 uu = make_float2(u0[i], u1[i]);
        dd[i] = dt;
        xx[i] = fmul2(dt, uu);
        dy[i] = make_float2(g0[i], g1[i]);  // already 0 outside the rows' valid tokens
        dDp = ffma2(dy[i], uu, dDp);
        // d(raw delta) = sigmoid(v) (u sum_n g B + sum_n A q): keep both factors
        sm.pv[warp][i][lane] = make_float4(sp.x * uu.x, sp.y * uu.y, sp.x, sp.y);
      }
    }
    // document starts among tokens tl .. tl+7 (bit i)
    unsigned rm = 0u;
    if (seqb && valid) {
      int prev = tl > 0 ? __ldg(seqb + tl - 1) : 0;
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const int cur = __ldg(seqb + tl + i);
        if (tl + i > 0 && cur != prev) rm |= 1u << i;
        prev = cur;
      }
    }
    const bool any_reset = __any_sync(kFull, rm != 0u);

    float2 sg[8], sq[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) sg[i] = sq[i] = make_float2(0.0f, 0.0f);

    const T* tileB = &sm.tile[buf][0][0][0];
    const T* tileC = &sm.tile[buf][1][0][0];
    float2 hck = make_float2(ok0 ? __ldg(ckc + SSM_DIDX(kDbgS16Ckpt, 0, 1, ck_left(p, ckc))) : 0.0f,
                             ok1 ? __ldg(ckc + SSM_DIDX(kDbgS16Ckpt, kSegs, 1, ck_left(p, ckc))) : 0.0f);
    auto states = [&](auto RS) {
#pragma unroll 1
    for (int n = 0; n < kN; ++n) {
      const float2 hin = hck;
      if (n + 1 < kN)  // next state's checkpoint, one state ahead
        hck = make_float2(
            ok0 ? __ldg(ckc + SSM_DIDX(kDbgS16Ckpt, (n + 1) * 2 * kSegs, 1, ck_left(p, ckc))) : 0.0f,
            ok1 ? __ldg(ckc + SSM_DIDX(kDbgS16Ckpt, (n + 1) * 2 * kSegs + kSegs, 1, ck_left(p, ckc)))
                : 0.0f);
      const float4 Aq = sm.A[warp][n];
      const float2 a2 = make_float2(Aq.x, Aq.y), ap2 = make_float2(Aq.z, Aq.w);
      float Bt[8], Ct[8];
      lds8<T>(tileB + n * kCh, lane, Bt);
      lds8<T>(tileC + n * kCh, lane, Ct);

      // forward recompute over the lane's 8 tokens; ah = a h_{t-1}
      float2 at[8], ah[8];
      float dCt[8];
      {
        float2 h = hin;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          at[i] = ex2x2(fmul2(dd[i], a2));
          if constexpr (decltype(RS)::value)
            if ((rm >> i) & 1u) at[i] = make_float2(0.0f, 0.0f);
          const float2 bx = fmul2(xx[i], dup(Bt[i]));
          ah[i] = fmul2(at[i], h);
          h = fadd2(ah[i], bx);
          dCt[i] = fmaf(dy[i].y, h.y, dy[i].x * h.x);
        }
      }
      // the lane's adjoint map: carry leaving token 0 = P (carry entering token 7) + G
      float2 gy[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) gy[i] = fmul2(dy[i], dup(Ct[i]));
      float2 P = fmul2(fmul2(at[0], at[1]), fmul2(at[2], at[3]));
      P = fmul2(P, fmul2(fmul2(at[4], at[5]), fmul2(at[6], at[7])));
      float2 G = gy[7];
#pragma unroll
      for (int i = 6; i >= 0; --i) G = ffma2(at[i + 1], G, gy[i]);
      G = fmul2(at[0], G);
      // join the lanes right to left: lane j ends with lanes j .. 31 composed
#pragma unroll
      for (int off = 1; off < 32; off <<= 1) {
        const float2 Pn = shfl_down2(P, off);
        const float2 Gn = shfl_down2(G, off);
        if (lane + off < 32) {
          G = ffma2(P, Gn, G);
          P = fmul2(P, Pn);
        }
      }
      const float2 cin = sm.car[warp][n];
      const float2 cout = ffma2(P, cin, G);  // carry leaving this lane's token 0
      float2 cr = shfl_down2(cout, 1);       // carry entering this lane's token 7
      if (lane == 31) cr = cin;
      if (lane == 0) sm.car[warp][n] = cout;

      // replay the adjoint; the terms of the sums
      float dBt[8];
      float2 dA2 = make_float2(0.0f, 0.0f);
      float2 g = fadd2(gy[7], cr);
#pragma unroll
      for (int i = 7; i >= 0; --i) {
        if (i < 7) g = ffma2(at[i + 1], g, gy[i]);
        const float2 q = fmul2(g, ah[i]);
        sq[i] = ffma2(ap2, q, sq[i]);
        dA2 = ffma2(dd[i], q, dA2);
        sg[i] = ffma2(g, dup(Bt[i]), sg[i]);
        dBt[i] = fmaf(g.y, xx[i].y, g.x * xx[i].x);
      }
      {
        float2& acc = sm.dA[warp][n][lane];
        acc = fadd2(acc, dA2);
      }
      // dB / dC of the row pair -> this warp's slot; sum over the CTA's warps
      float4* slot = &sm.red[n & 1][warp][0][0];
      slot[lane] = make_float4(dBt[0], dBt[1], dBt[2], dBt[3]);
      slot[32 + lane] = make_float4(dBt[4], dBt[5], dBt[6], dBt[7]);
      slot[64 + lane] = make_float4(dCt[0], dCt[1], dCt[2], dCt[3]);
      slot[96 + lane] = make_float4(dCt[4], dCt[5], dCt[6], dCt[7]);
      __syncthreads();
      if (threadIdx.x < 128) {
        const int q = threadIdx.x;  // (mat, half, lane) = (q >> 6, (q >> 5) & 1, q & 31)
        const int mat = q >> 6, f = q & 63;
        float4 s = sm.red[n & 1][0][mat][f];
#pragma unroll
        for (int w = 1; w < kBwdWarps; ++w) {
          const float4 v = sm.red[n & 1][w][mat][f];
          const float2 lo = __fadd2_rn(make_float2(s.x, s.y), make_float2(v.x, v.y));
          const float2 hi = __fadd2_rn(make_float2(s.z, s.w), make_float2(v.z, v.w));
          s = make_float4(lo.x, lo.y, hi.x, hi.y);
        }
        const int t = c * kCh + 8 * (f & 31) + 4 * (f >> 5);
        if (t < L && p.dbc_part) {  // deterministic: this CTA's sum, added later in order
          float* dst = p.dbc_part + SSM_DIDX(kDbgS16Part,
                                             ((size_t)blockIdx.x * 2 + mat) * p.dbc_bnl +
                                                 ((size_t)b * kN + n) * L + t,
                                             4,
                                             (size_t)((p.D + kBwdCtaRows16 - 1) / kBwdCtaRows16) * 2 *
                                                 p.dbc_bnl);
          dst[0] = s.x;
          dst[1] = s.y;
          dst[2] = s.z;
          dst[3] = s.w;
        } else if (t < L) {
          float* dst = (mat ? p.dC : p.dB) +
                       SSM_DIDX(kDbgS16BC, ((size_t)b * kN + n) * L + t, 4, (size_t)p.B * kN * L);
          if (VG) {
            asm volatile("red.global.add.v4.f32 [%0], {%1, %2, %3, %4};" ::"l"(dst), "f"(s.x),
                         "f"(s.y), "f"(s.z), "f"(s.w)
                         : "memory");
          } else {
            atomicAdd(dst, s.x);
            atomicAdd(dst + 1, s.y);
            atomicAdd(dst + 2, s.z);
            atomicAdd(dst + 3, s.w);
          }
        }
      }
    }
    };
    if (any_reset) states(std::true_type{});
    else states(std::false_type{});

    // ---- per-token outputs of the chunk ----
    {
      float du0[8], du1[8], dd0[8], dd1[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const float4 w = sm.pv[warp][i][lane];
        const float2 du = ffma2(dy[i], Dv, fmul2(dd[i], sg[i]));
        const float2 ddr = ffma2(make_float2(w.x, w.y), sg[i], fmul2(make_float2(w.z, w.w), sq[i]));
        du0[i] = du.x;
        du1[i] = du.y;
        dd0[i] = ddr.x;
        dd1[i] = ddr.y;
        if (valid) ddbp = fadd2(ddbp, ddr);
      }
      if (ok0) {
        st8<T, VG>(static_cast<T*>(p.du) + row0 + t0o, du0);
        st8<T, VG>(static_cast<T*>(p.ddelta) + row0 + t0o, dd0);
      }
      if (ok1) {
        st8<T, VG>(static_cast<T*>(p.du) + row1 + t1o, du1);
        st8<T, VG>(static_cast<T*>(p.ddelta) + row1 + t1o, dd1);
      }
    }
  }

  // the state before token 0 enters only through a_0 h_{-1}: its gradient is
  // the carry leaving token 0
  __syncthreads();
  if (p.dh0 && lane < kN) {
    const float2 cr = sm.car[warp][lane];
    if (act0) p.dh0[rid0 * kN + lane] = cr.x;
    if (act1) p.dh0[rid1 * kN + lane] = cr.y;
  }
  // dA of (row, state): fixed-order sum over the lanes' partials
  {
    const int n = lane & 15, rr = lane >> 4;
    float s = 0.0f;
#pragma unroll 8
    for (int j = 0; j < 32; ++j) {
      const float2 v = sm.dA[warp][n][j];
      s += rr ? v.y : v.x;
    }
    if (rr == 0 && act0) p.part_dA[SSM_DIDX(kDbgS16Param, rid0 * kN + n, 1, (size_t)p.B * p.D * kN)] = s;
    if (rr == 1 && act1) p.part_dA[SSM_DIDX(kDbgS16Param, rid1 * kN + n, 1, (size_t)p.B * p.D * kN)] = s;
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) {
    dDp.x += __shfl_xor_sync(kFull, dDp.x, off);
    dDp.y += __shfl_xor_sync(kFull, dDp.y, off);
    ddbp.x += __shfl_xor_sync(kFull, ddbp.x, off);
    ddbp.y += __shfl_xor_sync(kFull, ddbp.y, off);
  }
  if (lane == 0) {
    if (act0) {
      p.part_dD[rid0] = dDp.x;
      p.part_ddb[rid0] = ddbp.x;
    }
    if (act1) {
      p.part_dD[rid1] = dDp.y;
      p.part_ddb[rid1] = ddbp.y;
    }
  }
}


// ---------------------------------------------------------------------------
// Whole-row backward summary of a piece (N = 16 layout): per (row, state) the
// product of the decays and the adjoint leaving token 0 (a_0 g_0) that the
// piece's own dout produces with no adjoint entering from the right. Only
// the adjoint map is needed: no recompute of h, no replay, no sums.
template <typename T, int W>
struct Bwd16SumSmem {
  T tileC[2][kN][kCh];  // C of two chunks, activation dtype
  float4 A[W][kN];      // (A'_r0, A'_r1, -, -), A' = A log2(e)
  float2 car[W][kN];    // adjoint leaving the chunks done so far
  uint64_t bar[2];
};

template <typename T, int W>
__global__ void __launch_bounds__(W * 32, W < 8 ? 2 : 1) scan16_bwd_summary_kernel(const ScanArgs p) {
  static_assert(sizeof(Bwd16SumSmem<T, W>) <= 227 * 1024, "shared memory per CTA");
  extern __shared__ float4 smem_dyn[];
  Bwd16SumSmem<T, W>& sm = *reinterpret_cast<Bwd16SumSmem<T, W>*>(smem_dyn);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int b = blockIdx.y;
  const int d0 = blockIdx.x * (2 * W) + 2 * warp;  // rows d0, d0 + 1
  const bool act0 = d0 < p.D, act1 = d0 + 1 < p.D;
  const int L = p.L, nch = p.nchunks;
  const size_t rid0 = (size_t)b * p.D + (act0 ? d0 : 0);
  const size_t rid1 = (size_t)b * p.D + (act1 ? d0 + 1 : 0);
  const size_t row0 = SSM_DIDX(kDbgS16Row, rid0, act0 ? 1 : 0, (size_t)p.B * p.D) * L;
  const size_t row1 = SSM_DIDX(kDbgS16Row, rid1, act1 ? 1 : 0, (size_t)p.B * p.D) * L;
  const T* Cm = static_cast<const T*>(p.Cm);
  const bool has_z = p.z != nullptr;
  const int32_t* seqb = p.seq ? p.seq + (size_t)b * L : nullptr;

  if (threadIdx.x == 0) {
    mbar_init(&sm.bar[0], 1);
    mbar_init(&sm.bar[1], 1);
    fence_mbar_init();
  }
  if (lane < kN) {
    const int n = lane;
    const float a0 = act0 ? __ldg(p.A + (size_t)d0 * kN + n) : 0.0f;
    const float a1 = act1 ? __ldg(p.A + (size_t)(d0 + 1) * kN + n) : 0.0f;
    sm.A[warp][n] = make_float4(a0 * kLog2e, a1 * kLog2e, 0.0f, 0.0f);
    sm.car[warp][n] = make_float2(0.0f, 0.0f);
  }
  const int last = nch - 1;
  const int ntail = L - last * kCh;
  if (ntail < kCh) {  // a short last chunk: zero the tile tail its copies leave untouched
    for (int i = threadIdx.x; i < kN * (kCh - ntail); i += blockDim.x) {
      const int rr = i / (kCh - ntail), t = ntail + i % (kCh - ntail);
      sm.tileC[last & 1][rr][t] = T(0.0f);
    }
  }
  __syncthreads();
  auto issue = [&](int buf, int c) {  // thread 0: chunk c's C rows into tileC[buf]
    const int ntok = min(kCh, L - c * kCh);
    const unsigned bytes = static_cast<unsigned>(ntok) * sizeof(T);  // multiple of 16: L % 8 == 0
    fence_proxy_async_smem();
    mbar_expect_tx(&sm.bar[buf], bytes * kN);
#pragma unroll 1
    for (int n = 0; n < kN; ++n)
      tma_load_1d(&sm.tileC[buf][n][0], Cm + ((size_t)b * kN + n) * L + (size_t)c * kCh, bytes,
                  &sm.bar[buf]);
  };
  if (threadIdx.x == 0) issue(last & 1, last);
  const float2 bias = make_float2((act0 && p.delta_bias) ? __ldg(p.delta_bias + d0) : 0.0f,
                                  (act1 && p.delta_bias) ? __ldg(p.delta_bias + d0 + 1) : 0.0f);
  int k_use = 0;
  // the lane's sums of dt (both rows) and whether a document starts after
  // token 0: the decay of the piece is exp(A sum dt), or 0 across a start
  float2 dt_sum = make_float2(0.0f, 0.0f);
  bool any_start = false;
#pragma unroll 1
  for (int c = last; c >= 0; --c, ++k_use) {
    const int buf = c & 1;
    const bool ok = mbar_wait_bounded(&sm.bar[buf], (k_use >> 1) & 1, p.status);
    if (!__syncthreads_and(ok)) {
      // the copy into buf has not arrived: wait for it once more (bounded), then stop
      if (threadIdx.x == 0) mbar_wait_bounded(&sm.bar[buf], (k_use >> 1) & 1, nullptr);
      break;
    }
    if (threadIdx.x == 0 && c >= 1) issue(buf ^ 1, c - 1);
    const int tl = c * kCh + 8 * lane;
    const bool valid = tl < L;
    const bool ok0 = valid && act0, ok1 = valid && act1;
    // the lane's 8 tokens of each row (L is a multiple of 8 on this path)
    const int t0o = SSM_DIDX(kDbgS16Tok, tl, ok0 ? 8 : 0, L);
    const int t1o = SSM_DIDX(kDbgS16Tok, tl, ok1 ? 8 : 0, L);
    float2 dd[8], dy[8];
    {
      float dl0[8], dl1[8], g0[8], g1[8];
      ld8<T, true>(static_cast<const T*>(p.delta) + row0 + t0o, ok0, dl0);
      ld8<T, true>(static_cast<const T*>(p.delta) + row1 + t1o, ok1, dl1);
      ld8<T, true>(static_cast<const T*>(p.dout) + row0 + t0o, ok0, g0);
      ld8<T, true>(static_cast<const T*>(p.dout) + row1 + t1o, ok1, g1);
      if (has_z) {
        float z0[8], z1[8];
        ld8<T, true>(static_cast<const T*>(p.z) + row0 + t0o, ok0, z0);
        ld8<T, true>(static_cast<const T*>(p.z) + row1 + t1o, ok1, z1);
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          g0[i] *= z0[i] * sigmoid_fast(z0[i]);
          g1[i] *= z1[i] * sigmoid_fast(z1[i]);
        }
      }
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        float2 dt = make_float2(dl0[i] + bias.x, dl1[i] + bias.y);
        if (p.softplus) dt = softplus2(dt);
        dd[i] = make_float2(ok0 ? dt.x : 0.0f, ok1 ? dt.y : 0.0f);
        dy[i] = make_float2(g0[i], g1[i]);
        dt_sum = fadd2(dt_sum, dd[i]);
      }
    }
    unsigned rm = 0u;
    if (seqb && valid) {
      int prev = tl > 0 ? __ldg(seqb + tl - 1) : 0;
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const int cur = __ldg(seqb + tl + i);
        if (tl + i > 0 && cur != prev) rm |= 1u << i;
        prev = cur;
      }
    }
    any_start = any_start || rm != 0u;
    const T* tileC = &sm.tileC[buf][0][0];
#pragma unroll 1
    for (int n = 0; n < kN; ++n) {
      const float4 Aq = sm.A[warp][n];
      const float2 a2 = make_float2(Aq.x, Aq.y);
      float Ct[8];
      lds8<T>(tileC + n * kCh, lane, Ct);
      float2 at[8], gy[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        at[i] = ex2x2(fmul2(dd[i], a2));
        if ((rm >> i) & 1u) at[i] = make_float2(0.0f, 0.0f);
        gy[i] = fmul2(dy[i], dup(Ct[i]));
      }
      float2 P = fmul2(fmul2(at[0], at[1]), fmul2(at[2], at[3]));
      P = fmul2(P, fmul2(fmul2(at[4], at[5]), fmul2(at[6], at[7])));
      float2 G = gy[7];
#pragma unroll
      for (int i = 6; i >= 0; --i) G = ffma2(at[i + 1], G, gy[i]);
      G = fmul2(at[0], G);
#pragma unroll
      for (int off = 1; off < 32; off <<= 1) bwd_step2(P, G, off);
      if (lane == 0) {  // lane 0 now holds the map of the whole chunk
        const float2 cin = sm.car[warp][n];
        sm.car[warp][n] = ffma2(P, cin, G);
      }
    }
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) {
    dt_sum.x += __shfl_xor_sync(kFull, dt_sum.x, off);
    dt_sum.y += __shfl_xor_sync(kFull, dt_sum.y, off);
  }
  any_start = __any_sync(kFull, any_start);
  __syncwarp();
  if (lane < kN) {
    const float4 Aq = sm.A[warp][lane];
    const float2 cr = sm.car[warp][lane];
    const float2 dk = any_start ? make_float2(0.0f, 0.0f)
                                : make_float2(ex2_approx(Aq.x * dt_sum.x), ex2_approx(Aq.y * dt_sum.y));
    if (act0) {
      p.split_P[rid0 * p.Npad + lane] = dk.x;
      p.split_H[rid0 * p.Npad + lane] = cr.x;
    }
    if (act1) {
      p.split_P[rid1 * p.Npad + lane] = dk.y;
      p.split_H[rid1 * p.Npad + lane] = cr.y;
    }
  }
}

__global__ void bwd16_param_reduce_kernel(const float* __restrict__ pA, const float* __restrict__ pD,
                                          const float* __restrict__ pB, float* __restrict__ dA,
                                          float* __restrict__ dD, float* __restrict__ ddb, int B,
                                          int D) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i < D * kN) {
    float s = 0.0f;
    for (int b = 0; b < B; ++b) s += pA[(size_t)b * D * kN + i];
    dA[i] = s;
  }
  if (i < D) {
    float s1 = 0.0f, s2 = 0.0f;
    for (int b = 0; b < B; ++b) {
      s1 += pD[(size_t)b * D + i];
      s2 += pB[(size_t)b * D + i];
    }
    if (dD) dD[i] = s1;
    if (ddb) ddb[i] = s2;
  }
}

template <typename T, bool VG, int W>
cudaError_t bwd16_t(const ScanArgs& a, cudaStream_t s) {
  static std::atomic<unsigned long long> done{0};
  const int smem = (int)sizeof(Bwd16Smem<T, W>);
  cudaError_t e = smem_attr(scan16_bwd_kernel<T, VG, W>, smem, &done);
  if (e != cudaSuccess) return e;
  dim3 grid((a.D + 2 * W - 1) / (2 * W), a.B);
  scan16_bwd_kernel<T, VG, W><<<grid, W * 32, smem, s>>>(a);
  const int m = a.D * kN;
  bwd16_param_reduce_kernel<<<(m + 255) / 256, 256, 0, s>>>(a.part_dA, a.part_dD, a.part_ddb, a.dA,
                                                           a.dD, a.ddelta_bias, a.B, a.D);
  return cudaGetLastError();
}

template <int W>
cudaError_t bwd16_dispatch(const ScanArgs& a, cudaStream_t s) {
  if (a.bf16)
    return a.vec ? bwd16_t<__nv_bfloat16, true, W>(a, s) : bwd16_t<__nv_bfloat16, false, W>(a, s);
  return a.vec ? bwd16_t<float, true, W>(a, s) : bwd16_t<float, false, W>(a, s);
}

}  // namespace

int scan16_bwd_rows(const ScanArgs& a) {
  return s16::pick_shape(a.B, a.D, 2 * kBwdWarpsSmall, 2, 2 * kBwdWarpsBig) ? 2 * kBwdWarpsBig
                                                                            : 2 * kBwdWarpsSmall;
}

template <typename T, int W>
cudaError_t bwd16_summary_t(const ScanArgs& a, cudaStream_t s) {
  static std::atomic<unsigned long long> done{0};
  const int smem = (int)sizeof(Bwd16SumSmem<T, W>);
  cudaError_t e = smem_attr(scan16_bwd_summary_kernel<T, W>, smem, &done);
  if (e != cudaSuccess) return e;
  dim3 grid((a.D + 2 * W - 1) / (2 * W), a.B);
  scan16_bwd_summary_kernel<T, W><<<grid, W * 32, smem, s>>>(a);
  return cudaGetLastError();
}

cudaError_t launch_scan16_bwd_summary(const ScanArgs& a, cudaStream_t s) {
  const bool big = scan16_bwd_rows(a) == 2 * kBwdWarpsBig;
  if (a.bf16)
    return big ? bwd16_summary_t<__nv_bfloat16, kBwdWarpsBig>(a, s)
               : bwd16_summary_t<__nv_bfloat16, kBwdWarpsSmall>(a, s);
  return big ? bwd16_summary_t<float, kBwdWarpsBig>(a, s) : bwd16_summary_t<float, kBwdWarpsSmall>(a, s);
}

cudaError_t launch_scan16_bwd(const ScanArgs& a, cudaStream_t s) {
  return scan16_bwd_rows(a) == 2 * kBwdWarpsBig ? bwd16_dispatch<kBwdWarpsBig>(a, s)
                                                : bwd16_dispatch<kBwdWarpsSmall>(a, s);
}

SSM_DEBUG_TU(scan16_bwd)

}  // namespace ssm
