// Selective scan with a complex diagonal A, forward and backward.
//
// Diagonal A with complex entries (the S4D simplification, "hung-phan
// ml-skills mamba", section "S4: Structured State Spaces for Sequences"; the
// page's Mamba-3 list names a complex-valued state update), made selective
// like the real scan. Per row (b, d) and state n:
//   a_t = exp(dt_t A_n) = e^{dt Re A} (cos(dt Im A) + i sin(dt Im A))
//   h_t = a_t h_{t-1} + dt_t u_t B_t                  (h, B, C complex)
//   y_t = 2 Re(sum_n C_t h_t) + D u_t,   out = y silu(z)
// Each complex state stands for itself and its conjugate, hence 2 Re. A
// document start sets a_t = 0, as in the real scan.
//
// Both kernels run one thread per (row, state) over 16-token blocks: a warp
// holds two rows x 16 states, a CTA eight rows of one batch entry that share
// the B / C tiles (four planes: Re B, Im B, Re C, Im C). The next block's
// B / C pieces are copied into shared memory by cp.async and its per-row
// values into registers while the current block is processed. The forward
// keeps the state entering every block; the backward rebuilds each block's
// states from it and runs the adjoint (g = dL/dRe h + i dL/dIm h)
//   g_t = 2 dy_t conj(C_t) + conj(a_{t+1}) g_{t+1}
// and, with w_t = conj(g_t conj(h_{t-1})) a_t,
//   du_t  = dy_t D + dt_t sum_n Re(conj(g_t) B_t)
//   ddt_t = u_t sum_n Re(conj(g_t) B_t) + sum_n Re(A_n w_t)
//   dRe A_n += dt_t Re w_t,   dIm A_n -= dt_t Im w_t
//   dB_t += dt_t u_t g_t,     dC_t += 2 dy_t conj(h_t)
// Sums over states go through a per-warp shared-memory transposition; dB / dC
// are added over the CTA's rows and sent to HBM with float4 atomics.
#include "scan_common.cuh"

namespace ssm {

namespace {

constexpr int kCB = 16;                    // tokens per block = checkpoint interval
constexpr int kCWarps = 4;
constexpr int kCRows = 2 * kCWarps;        // rows per CTA
static_assert(kCRows == kCscanCtaRows, "row groups of the deterministic dB / dC partials");
constexpr int kCLd = kCB + 4;              // fp32 state-row stride: 8 lanes on distinct banks
constexpr int kXHalf = kNMax * kCLd + 16;  // one row half of a transposition array
constexpr int kCThreads = kCWarps * 32;

// e^{i theta} = (cos theta, sin theta) on the FMA pipe, accurate to a few
// ulp: theta = k pi/2 + r with k the integer nearest theta 2/pi (rounded by
// the 1.5 * 2^23 shift, whose low bits then hold k mod 4) and r from Cody and
// Waite's two-constant reduction (pi/2 split into its nearest float and the
// remainder), |r| <= pi/4; sin r and cos r from their Taylor series through
// r^9 and r^10 (truncation below 2e-9 there); the quadrant k mod 4 rotates
// (cos r, sin r) by multiples of pi/2.
__device__ __forceinline__ float2 cis(float theta) {
  const float sh = fmaf(theta, 0.636619772f, 12582912.0f);  // theta 2/pi + 1.5 * 2^23
  const int q = __float_as_int(sh);
  const float k = sh - 12582912.0f;
  float r = fmaf(-k, 1.57079637f, theta);                   // float(pi/2)
  r = fmaf(-k, -4.37113883e-8f, r);                         // pi/2 - float(pi/2)
  // the sine and cosine Horner chains side by side in one f32x2 register
  // (each half rounds exactly as the scalar chain would)
  const float r2 = r * r;
  const float2 rr = make_float2(r2, r2);
  float2 hs = __ffma2_rn(rr, make_float2(2.75573192e-6f, -2.75573192e-7f),
                         make_float2(-1.98412698e-4f, 2.48015873e-5f));  // (1/9!, -1/10!), (-1/7!, 1/8!)
  hs = __ffma2_rn(rr, hs, make_float2(8.33333333e-3f, -1.38888889e-3f));   // 1/5!, -1/6!
  hs = __ffma2_rn(rr, hs, make_float2(-1.66666667e-1f, 4.16666667e-2f));   // -1/3!, 1/4!
  hs = __ffma2_rn(make_float2(r * r2, r2), hs, make_float2(r, -0.5f));     // sin done; -1/2!
  const float sn = hs.x;
  const float cs = fmaf(r2, hs.y, 1.0f);
  const bool odd = q & 1;
  const float c = odd ? sn : cs, s = odd ? cs : sn;
  const unsigned sc = (unsigned)((q + 1) & 2) << 30;        // cos < 0 in quadrants 1, 2
  const unsigned ss = (unsigned)(q & 2) << 30;              // sin < 0 in quadrants 2, 3
  return make_float2(__uint_as_float(__float_as_uint(c) ^ sc),
                     __uint_as_float(__float_as_uint(s) ^ ss));
}

// The same with sin and cos of the reduced angle on the special-function
// unit (absolute error near 2^-21 on |r| <= pi/4): used with bf16 storage,
// whose output rounding (2^-9) leaves that error far below the tolerance;
// fp32 storage keeps the series above.
__device__ __forceinline__ float2 cis_sfu(float theta) {
  const float sh = fmaf(theta, 0.636619772f, 12582912.0f);  // theta 2/pi + 1.5 * 2^23
  const int q = __float_as_int(sh);
  const float k = sh - 12582912.0f;
  float r = fmaf(-k, 1.57079637f, theta);                   // float(pi/2)
  r = fmaf(-k, -4.37113883e-8f, r);                         // pi/2 - float(pi/2)
  const float sn = __sinf(r), cs = __cosf(r);
  const bool odd = q & 1;
  const float c = odd ? sn : cs, s = odd ? cs : sn;
  const unsigned sc = (unsigned)((q + 1) & 2) << 30;        // cos < 0 in quadrants 1, 2
  const unsigned ss = (unsigned)(q & 2) << 30;              // sin < 0 in quadrants 2, 3
  return make_float2(__uint_as_float(__float_as_uint(c) ^ sc),
                     __uint_as_float(__float_as_uint(s) ^ ss));
}

// dt = softplus(v) with the accurate library exp / log1p: the phase dt Im A
// magnifies dt's relative error by |Im A|, and dt is computed once per token
// for all 16 states.
__device__ __forceinline__ float softplus_acc(float v) {
  return v > 20.0f ? v : log1pf(expf(v));
}

template <typename T>
__device__ __forceinline__ float ldv(const T* p);
template <>
__device__ __forceinline__ float ldv<float>(const float* p) { return __ldg(p); }
template <>
__device__ __forceinline__ float ldv<__nv_bfloat16>(const __nv_bfloat16* p) {
  return __bfloat162float(p[0]);
}

template <typename T>
__device__ __forceinline__ T cvt(float v);
template <>
__device__ __forceinline__ float cvt<float>(float v) { return v; }
template <>
__device__ __forceinline__ __nv_bfloat16 cvt<__nv_bfloat16>(float v) { return __float2bfloat16_rn(v); }

template <typename T>
__device__ __forceinline__ float tof(T v);
template <>
__device__ __forceinline__ float tof<float>(float v) { return v; }
template <>
__device__ __forceinline__ float tof<__nv_bfloat16>(__nv_bfloat16 v) { return __bfloat162float(v); }

template <typename T>
struct CTiles {
  T raw[4][kNMax][kCB];        // the next block's B / C pieces (each thread its own)
  float BC[4][kNMax][kCLd];    // Re B, Im B, Re C, Im C of the current block
  float dt[kCRows][kCB];       // step size (0 past the end)
  float xu[kCRows][kCB];       // dt u
  float dy[kCRows][kCB];       // dL/dy (backward only)
};

// This thread's copies of block [tb, tb + 16) of the four B / C planes:
// plane pl of state n is row ((b N + n) 2 + (pl & 1)) of Bm (pl < 2) or Cm.
template <typename T, bool VEC>
__device__ __forceinline__ void issue_bc(CTiles<T>& sm, const T* __restrict__ Bm,
                                         const T* __restrict__ Cm, int b, int N, int L, int tb) {
  constexpr int kPiece = 16 / (int)sizeof(T);  // tokens per 16-byte piece
  constexpr int kPPR = kCB / kPiece;
  constexpr int kPieces = 4 * kNMax * kPPR;
#pragma unroll
  for (int pc = threadIdx.x; pc < kPieces; pc += kCThreads) {
    const int pl = pc / (kNMax * kPPR), rem = pc % (kNMax * kPPR);
    const int n = rem / kPPR, jj = rem % kPPR;
    const int t = tb + jj * kPiece;
    const T* src = (pl < 2 ? Bm : Cm) + (((size_t)b * N + (n < N ? n : 0)) * 2 + (pl & 1)) * L;
    T* dst = &sm.raw[pl][n][jj * kPiece];
    if (VEC) {
      const bool ok = n < N && t < L;
      cp_async16(dst, src + (ok ? t : 0), ok);
    } else {
#pragma unroll
      for (int e = 0; e < kPiece; ++e)
        dst[e] = (n < N && t + e < L) ? src[t + e] : cvt<T>(0.0f);
    }
  }
  if (VEC) cp_async_commit();
}

// The pieces this thread copied -> fp32 tiles.
template <typename T, bool VEC>
__device__ __forceinline__ void convert_bc(CTiles<T>& sm) {
  if (VEC) cp_async_wait_all();
  constexpr int kPiece = 16 / (int)sizeof(T);
  constexpr int kPPR = kCB / kPiece;
  constexpr int kPieces = 4 * kNMax * kPPR;
#pragma unroll
  for (int pc = threadIdx.x; pc < kPieces; pc += kCThreads) {
    const int pl = pc / (kNMax * kPPR), rem = pc % (kNMax * kPPR);
    const int n = rem / kPPR, jj = rem % kPPR;
    const T* src = &sm.raw[pl][n][jj * kPiece];
    float* dst = &sm.BC[pl][n][jj * kPiece];
#pragma unroll
    for (int e = 0; e < kPiece; e += 4)
      *reinterpret_cast<float4*>(dst + e) =
          make_float4(tof(src[e]), tof(src[e + 1]), tof(src[e + 2]), tof(src[e + 3]));
  }
}

__device__ __forceinline__ float comp(const float4& v, int j) {
  return j == 0 ? v.x : j == 1 ? v.y : j == 2 ? v.z : v.w;
}

// Document starts in block [tb, tb + 16): bit j set when token tb + j begins
// a new document (every lane gets the same mask).
__device__ __forceinline__ unsigned block_resets(int sq, int sqp, int tok, int L) {
  const bool start = tok < L && tok > 0 && sq != sqp;
  return __ballot_sync(kFull, start) & 0xffffu;
}

// a_t = e^{dt Re A} e^{i dt Im A} for the block's 16 tokens (A's real part
// pre-scaled by log2 e), 0 at a document start (rm: warp-uniform bit mask).
// SFU: the angle's sin / cos on the special-function unit (bf16 storage).
template <bool SFU>
__device__ __forceinline__ void decays(const float4* dt4, float Ar2, float Ai, unsigned rm,
                                       float ar[kCB], float ai[kCB]) {
#pragma unroll
  for (int q = 0; q < kCB / 4; ++q) {
    const float4 dq = dt4[q];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const float dt = comp(dq, j);
      const float mag = ex2_approx(dt * Ar2);
      const float2 cs = SFU ? cis_sfu(dt * Ai) : cis(dt * Ai);
      ar[4 * q + j] = mag * cs.x;
      ai[4 * q + j] = mag * cs.y;
    }
  }
  if (rm) {
#pragma unroll
    for (int t = 0; t < kCB; ++t)
      if ((rm >> t) & 1u) ar[t] = ai[t] = 0.0f;
  }
}

// ---------------------------------------------------------------------------
// Forward.
// ---------------------------------------------------------------------------
template <typename T, bool VEC>
__global__ void __launch_bounds__(kCThreads, 3)
cscan_fwd_kernel(const ScanArgs p) {
  __shared__ __align__(16) CTiles<T> sm;
  __shared__ __align__(16) float X[kCWarps][2 * kXHalf];

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int hf = lane >> 4;   // which of the warp's two rows
  const int n = lane & 15;    // state; in the per-token phases, token n of the block
  const int r = 2 * warp + hf;
  const int b = blockIdx.y;
  const int d = blockIdx.x * kCRows + r;
  const bool active = d < p.D;
  const int N = p.N, L = p.L;
  const bool nval = active && n < N;
  const size_t rowid = (size_t)b * p.D + (active ? d : 0);
  const size_t row = SSM_DIDX(kDbgCscanRow, rowid, active ? 1 : 0, (size_t)p.B * p.D) * L;
  const size_t nslot = (size_t)p.nchunks * (kChunk / kCB);  // checkpoint slots per row
  const bool has_z = p.z != nullptr;

  const T* Bm = static_cast<const T*>(p.Bm);
  const T* Cm = static_cast<const T*>(p.Cm);
  const T* dl_row = static_cast<const T*>(p.delta) + row;
  const T* u_row = static_cast<const T*>(p.u) + row;
  const T* z_row = has_z ? static_cast<const T*>(p.z) + row : nullptr;
  const int32_t* seqb = p.seq ? p.seq + (size_t)b * L : nullptr;

  float2 An = make_float2(0.0f, 0.0f);
  if (nval) An = __ldg(reinterpret_cast<const float2*>(p.A) + (size_t)d * N + n);
  const float Ar2 = An.x * kLog2e, Ai = An.y;
  const float Dv = (active && p.Dskip) ? __ldg(p.Dskip + d) : 0.0f;
  const float bias = (active && p.delta_bias) ? __ldg(p.delta_bias + d) : 0.0f;
  float hr = 0.0f, hi = 0.0f;
  if (nval && p.h0) {
    const float2 h = reinterpret_cast<const float2*>(p.h0)[rowid * N + n];
    hr = h.x;
    hi = h.y;
  }

  // token tb + n of row r for the block being staged, and for the current one
  float nx_dl = 0.0f, nx_u = 0.0f, nx_z = 0.0f;
  int nx_sq = 0, nx_sqp = 0;
  float cu_u = 0.0f, cu_z = 0.0f;
  unsigned rm = 0u;

  auto prefetch = [&](int kb) {
    const int tb = kb * kCB;
    issue_bc<T, VEC>(sm, Bm, Cm, b, N, L, tb);
    const int t = tb + n;
    const bool ok = active && t < L;
    nx_dl = ok ? ldv(dl_row + t) : 0.0f;
    nx_u = ok ? ldv(u_row + t) : 0.0f;
    nx_z = (ok && has_z) ? ldv(z_row + t) : 0.0f;
    if (seqb) {
      nx_sq = t < L ? __ldg(seqb + t) : 0;
      nx_sqp = (t > 0 && t < L) ? __ldg(seqb + t - 1) : nx_sq;
    }
  };
  auto convert = [&](int kb) {
    const int tb = kb * kCB;
    convert_bc<T, VEC>(sm);
    const int t = tb + n;
    const bool in = active && t < L;
    const float v = nx_dl + bias;
    const float dt = in ? (p.softplus ? softplus_acc(v) : v) : 0.0f;
    sm.dt[r][n] = dt;
    sm.xu[r][n] = dt * nx_u;
    cu_u = nx_u;
    cu_z = nx_z;
    rm = seqb ? block_resets(nx_sq, nx_sqp, t, L) : 0u;
  };

  const int nb = (L + kCB - 1) / kCB;
  prefetch(0);
  convert(0);
  if (nb > 1) prefetch(1);
  float* Xw = &X[warp][hf * kXHalf];
  const float4* dt4 = reinterpret_cast<const float4*>(&sm.dt[r][0]);
  const float4* xu4 = reinterpret_cast<const float4*>(&sm.xu[r][0]);
  const float4* Br4 = reinterpret_cast<const float4*>(&sm.BC[0][n][0]);
  const float4* Bi4 = reinterpret_cast<const float4*>(&sm.BC[1][n][0]);
  const float4* Cr4 = reinterpret_cast<const float4*>(&sm.BC[2][n][0]);
  const float4* Ci4 = reinterpret_cast<const float4*>(&sm.BC[3][n][0]);
  // a row's slots: [nslot][kNMax] (re, im) pairs
  float2* ck = reinterpret_cast<float2*>(p.ckpt) +
               SSM_DIDX(kDbgCscanCkpt, rowid * nslot * kNMax + n, nval ? (nslot - 1) * kNMax + 1 : 0,
                        (size_t)p.B * p.D * nslot * kNMax);

#pragma unroll 1
  for (int kb = 0; kb < nb; ++kb) {
    const int tb = kb * kCB;
    __syncthreads();  // block kb's tiles are complete
    if (nval) ck[(size_t)kb * kNMax] = make_float2(hr, hi);
    // the block's decays first (independent of h), then the serial chain
    float ar_[kCB], ai_[kCB];
    decays<sizeof(T) == 2>(dt4, Ar2, Ai, rm, ar_, ai_);
#pragma unroll
    for (int q = 0; q < kCB / 4; ++q) {
      const float4 xq = xu4[q], br = Br4[q], bi = Bi4[q], cr = Cr4[q], ci = Ci4[q];
      float part[4];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const float ar = ar_[4 * q + j], ai = ai_[4 * q + j], xu = comp(xq, j);
        const float nr = fmaf(ar, hr, fmaf(-ai, hi, xu * comp(br, j)));
        const float ni = fmaf(ar, hi, fmaf(ai, hr, xu * comp(bi, j)));
        hr = nr;
        hi = ni;
        part[j] = fmaf(comp(cr, j), hr, -comp(ci, j) * hi);
      }
      reinterpret_cast<float4*>(Xw + n * kCLd)[q] = make_float4(part[0], part[1], part[2], part[3]);
    }
    __syncwarp();
    // token n of row r: sum over the states
    float s = 0.0f;
#pragma unroll
    for (int m = 0; m < kNMax; ++m) s += Xw[m * kCLd + n];
    {
      const int t = tb + n;
      if (active && t < L) {
        const float y = fmaf(2.0f, s, Dv * cu_u);
        if (has_z) {
          static_cast<T*>(p.ysave)[row + t] = cvt<T>(y);
          static_cast<T*>(p.out)[row + t] = cvt<T>(y * cu_z * sigmoid_fast(cu_z));
        } else {
          static_cast<T*>(p.out)[row + t] = cvt<T>(y);
        }
      }
    }
    __syncthreads();  // tiles and X are free
    if (kb + 1 < nb) {
      convert(kb + 1);
      if (kb + 2 < nb) prefetch(kb + 2);
    }
  }
  if (nval && p.final_state)
    reinterpret_cast<float2*>(p.final_state)[rowid * N + n] = make_float2(hr, hi);
}

// ---------------------------------------------------------------------------
// Backward.
// ---------------------------------------------------------------------------
constexpr int kXArr = 4;  // transposition arrays per warp

template <typename T>
struct CBwdSmem {
  CTiles<T> t;
  float X[kCWarps][kXArr][2 * kXHalf];
};

template <typename T, bool VEC>
__global__ void __launch_bounds__(kCThreads, 3)
cscan_bwd_kernel(const ScanArgs p) {
  extern __shared__ float4 smem_dyn[];
  CBwdSmem<T>& S = *reinterpret_cast<CBwdSmem<T>*>(smem_dyn);
  CTiles<T>& sm = S.t;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int hf = lane >> 4;
  const int n = lane & 15;
  const int r = 2 * warp + hf;
  const int b = blockIdx.y;
  const int d = blockIdx.x * kCRows + r;
  const bool active = d < p.D;
  const int N = p.N, L = p.L;
  const bool nval = active && n < N;
  const size_t rowid = (size_t)b * p.D + (active ? d : 0);
  const size_t row = SSM_DIDX(kDbgCscanRow, rowid, active ? 1 : 0, (size_t)p.B * p.D) * L;
  const size_t nslot = (size_t)p.nchunks * (kChunk / kCB);
  const bool has_z = p.z != nullptr;

  const T* Bm = static_cast<const T*>(p.Bm);
  const T* Cm = static_cast<const T*>(p.Cm);
  const T* dl_row = static_cast<const T*>(p.delta) + row;
  const T* u_row = static_cast<const T*>(p.u) + row;
  const T* go_row = static_cast<const T*>(p.dout) + row;
  const T* z_row = has_z ? static_cast<const T*>(p.z) + row : nullptr;
  const T* y_row = has_z ? static_cast<const T*>(p.ysave) + row : nullptr;
  const int32_t* seqb = p.seq ? p.seq + (size_t)b * L : nullptr;

  float2 An = make_float2(0.0f, 0.0f);
  if (nval) An = __ldg(reinterpret_cast<const float2*>(p.A) + (size_t)d * N + n);
  const float Ar2 = An.x * kLog2e, Ai = An.y;
  const float Dv = (active && p.Dskip) ? __ldg(p.Dskip + d) : 0.0f;
  const float bias = (active && p.delta_bias) ? __ldg(p.delta_bias + d) : 0.0f;
  const float2* ckp = reinterpret_cast<const float2*>(p.ckpt) +
                      SSM_DIDX(kDbgCscanCkpt, rowid * nslot * kNMax + n,
                               nval ? (nslot - 1) * kNMax + 1 : 0, (size_t)p.B * p.D * nslot * kNMax);

  float nx_dl = 0.0f, nx_u = 0.0f, nx_go = 0.0f, nx_z = 0.0f, nx_y = 0.0f;
  int nx_sq = 0, nx_sqp = 0;
  float2 ck_issued = make_float2(0.0f, 0.0f), ck_ready = ck_issued;
  unsigned rm = 0u;
  float e_u = 0.0f, e_dt = 0.0f, e_dy = 0.0f, e_dsp = 1.0f;
  float dDp = 0.0f, ddbp = 0.0f;

  auto prefetch = [&](int kb) {
    const int tb = kb * kCB;
    issue_bc<T, VEC>(sm, Bm, Cm, b, N, L, tb);
    const int t = tb + n;
    const bool ok = active && t < L;
    nx_dl = ok ? ldv(dl_row + t) : 0.0f;
    nx_u = ok ? ldv(u_row + t) : 0.0f;
    nx_go = ok ? ldv(go_row + t) : 0.0f;
    nx_z = (ok && has_z) ? ldv(z_row + t) : 0.0f;
    nx_y = (ok && has_z) ? ldv(y_row + t) : 0.0f;
    if (nval) ck_issued = ckp[(size_t)kb * kNMax];
    if (seqb) {
      nx_sq = t < L ? __ldg(seqb + t) : 0;
      nx_sqp = (t > 0 && t < L) ? __ldg(seqb + t - 1) : nx_sq;
    }
  };
  auto convert = [&](int kb) {
    const int tb = kb * kCB;
    convert_bc<T, VEC>(sm);
    const int t = tb + n;
    const bool in = active && t < L;
    const float v = nx_dl + bias;
    const float dt = in ? (p.softplus ? softplus_acc(v) : v) : 0.0f;
    float gate = 1.0f;
    if (has_z) {
      const float sz = sigmoid_fast(nx_z);
      gate = nx_z * sz;
      if (in)
        static_cast<T*>(p.dz)[row + t] =
            cvt<T>(nx_go * nx_y * (sz * (1.0f + nx_z * (1.0f - sz))));
    }
    const float dy = in ? nx_go * gate : 0.0f;
    if (in) dDp = fmaf(dy, nx_u, dDp);
    sm.dt[r][n] = dt;
    sm.xu[r][n] = dt * nx_u;
    sm.dy[r][n] = dy;
    e_u = nx_u;
    e_dt = dt;
    e_dy = dy;
    // d softplus(v) / dv = sigmoid(v)
    e_dsp = p.softplus ? (v > 20.0f ? 1.0f : sigmoid_fast(v)) : 1.0f;
    ck_ready = ck_issued;
    rm = seqb ? block_resets(nx_sq, nx_sqp, t, L) : 0u;
  };

  const int nb = (L + kCB - 1) / kCB;
  prefetch(nb - 1);
  convert(nb - 1);
  if (nb >= 2) prefetch(nb - 2);

  float* X0 = &S.X[warp][0][hf * kXHalf];
  float* X1 = &S.X[warp][1][hf * kXHalf];
  float* X2 = &S.X[warp][2][hf * kXHalf];
  float* X3 = &S.X[warp][3][hf * kXHalf];
  const float4* dt4 = reinterpret_cast<const float4*>(&sm.dt[r][0]);
  const float4* xu4 = reinterpret_cast<const float4*>(&sm.xu[r][0]);
  const float4* dy4 = reinterpret_cast<const float4*>(&sm.dy[r][0]);
  const float4* Br4 = reinterpret_cast<const float4*>(&sm.BC[0][n][0]);
  const float4* Bi4 = reinterpret_cast<const float4*>(&sm.BC[1][n][0]);
  const float4* Cr4 = reinterpret_cast<const float4*>(&sm.BC[2][n][0]);
  const float4* Ci4 = reinterpret_cast<const float4*>(&sm.BC[3][n][0]);

  // conj(a_{t+1}) g_{t+1} for the token after the block; after the last token
  // the gradient of the final state
  float gr = 0.0f, gi = 0.0f;
  if (nval && p.dhL) {
    const float2 v = reinterpret_cast<const float2*>(p.dhL)[rowid * N + n];
    gr = v.x;
    gi = v.y;
  }
  float dAr = 0.0f, dAi = 0.0f;

#pragma unroll 1
  for (int kb = nb - 1; kb >= 0; --kb) {
    const int tb = kb * kCB;
    __syncthreads();  // block kb's tiles are complete; X is free
    const float2 hck = ck_ready;

    // forward recompute of a_t and h_t over the block
    float Hr[kCB], Hi[kCB], Ar_[kCB], Ai_[kCB];
    decays<sizeof(T) == 2>(dt4, Ar2, Ai, rm, Ar_, Ai_);
    {
      float hr = hck.x, hi = hck.y;
#pragma unroll
      for (int q = 0; q < kCB / 4; ++q) {
        const float4 xq = xu4[q], br = Br4[q], bi = Bi4[q];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const int t = 4 * q + j;
          const float ar = Ar_[t], ai = Ai_[t], xu = comp(xq, j);
          const float nr = fmaf(ar, hr, fmaf(-ai, hi, xu * comp(br, j)));
          const float ni = fmaf(ar, hi, fmaf(ai, hr, xu * comp(bi, j)));
          Hr[t] = hr = nr;
          Hi[t] = hi = ni;
        }
      }
    }

    // adjoint backwards over the block
#pragma unroll
    for (int q = kCB / 4 - 1; q >= 0; --q) {
      const float4 dq = dt4[q], xq = xu4[q], yq = dy4[q];
      const float4 br = Br4[q], bi = Bi4[q], cr = Cr4[q], ci = Ci4[q];
      float sg[4], sa[4], dbr[4], dbi[4];
#pragma unroll
      for (int j = 3; j >= 0; --j) {
        const int t = 4 * q + j;
        const float dy2 = 2.0f * comp(yq, j);
        gr = fmaf(dy2, comp(cr, j), gr);
        gi = fmaf(-dy2, comp(ci, j), gi);
        const float hpr = t ? Hr[t - 1] : hck.x;
        const float hpi = t ? Hi[t - 1] : hck.y;
        // Ga = g conj(h_{t-1});  w = conj(Ga) a
        const float gar = fmaf(gr, hpr, gi * hpi);
        const float gai = fmaf(gi, hpr, -gr * hpi);
        const float ar = Ar_[t], ai = Ai_[t];
        const float wr = fmaf(gar, ar, gai * ai);
        const float wi = fmaf(gar, ai, -gai * ar);
        const float dt = comp(dq, j), xu = comp(xq, j);
        dAr = fmaf(dt, wr, dAr);
        dAi = fmaf(-dt, wi, dAi);
        sa[j] = fmaf(An.x, wr, -An.y * wi);
        sg[j] = fmaf(gr, comp(br, j), gi * comp(bi, j));
        dbr[j] = gr * xu;
        dbi[j] = gi * xu;
        // carry conj(a_t) g_t into token t - 1
        const float cr_ = fmaf(ar, gr, ai * gi);
        const float ci_ = fmaf(ar, gi, -ai * gr);
        gr = cr_;
        gi = ci_;
      }
      reinterpret_cast<float4*>(X0 + n * kCLd)[q] = make_float4(sg[0], sg[1], sg[2], sg[3]);
      reinterpret_cast<float4*>(X1 + n * kCLd)[q] = make_float4(sa[0], sa[1], sa[2], sa[3]);
      reinterpret_cast<float4*>(X2 + n * kCLd)[q] = make_float4(dbr[0], dbr[1], dbr[2], dbr[3]);
      reinterpret_cast<float4*>(X3 + n * kCLd)[q] = make_float4(dbi[0], dbi[1], dbi[2], dbi[3]);
    }
    __syncwarp();
    // sums over the states for token n of row r
    float s1 = 0.0f, s2 = 0.0f;
#pragma unroll
    for (int m = 0; m < kNMax; ++m) {
      s1 += X0[m * kCLd + n];
      s2 += X1[m * kCLd + n];
    }
    __syncwarp();
    // this row's dC_t = 2 dy_t conj(h_t) into arrays 0 and 1
#pragma unroll
    for (int q = 0; q < kCB / 4; ++q) {
      const float4 yq = dy4[q];
      float cr[4], ci[4];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const float dy2 = 2.0f * comp(yq, j);
        cr[j] = dy2 * Hr[4 * q + j];
        ci[j] = -dy2 * Hi[4 * q + j];
      }
      reinterpret_cast<float4*>(X0 + n * kCLd)[q] = make_float4(cr[0], cr[1], cr[2], cr[3]);
      reinterpret_cast<float4*>(X1 + n * kCLd)[q] = make_float4(ci[0], ci[1], ci[2], ci[3]);
    }
    __syncthreads();  // every row's dB / dC terms are in X; tiles are free
    // CTA sum over its rows: arrays 0, 1 = Re, Im dC; 2, 3 = Re, Im dB
#pragma unroll
    for (int it = 0; it < (kXArr * kNMax * (kCB / 4)) / kCThreads; ++it) {
      const int item = threadIdx.x + it * kCThreads;
      const int arr = item >> 6, m = (item >> 2) & 15, q = item & 3;
      float4 v[2 * kCWarps];
#pragma unroll
      for (int w = 0; w < kCWarps; ++w) {
        v[2 * w] = *reinterpret_cast<const float4*>(&S.X[w][arr][m * kCLd + 4 * q]);
        v[2 * w + 1] = *reinterpret_cast<const float4*>(&S.X[w][arr][kXHalf + m * kCLd + 4 * q]);
      }
#pragma unroll
      for (int s = 1; s < 2 * kCWarps; s <<= 1)
#pragma unroll
        for (int i = 0; i + s < 2 * kCWarps; i += 2 * s) {
          v[i].x += v[i + s].x;
          v[i].y += v[i + s].y;
          v[i].z += v[i + s].z;
          v[i].w += v[i + s].w;
        }
      const int t = tb + 4 * q;
      if (m < N && t < L && p.dbc_part) {  // deterministic: this CTA's sum, added later in order
        float* dst = p.dbc_part + ((size_t)blockIdx.x * 2 + (arr < 2 ? 1 : 0)) * p.dbc_bnl +
                     (((size_t)b * N + m) * 2 + (arr & 1)) * L + t;
        const int left = L - t;
        dst[0] = v[0].x;
        if (left > 1) dst[1] = v[0].y;
        if (left > 2) dst[2] = v[0].z;
        if (left > 3) dst[3] = v[0].w;
      } else if (m < N && t < L) {
        float* dst = (arr < 2 ? p.dC : p.dB) + (((size_t)b * N + m) * 2 + (arr & 1)) * L + t;
        if (VEC) {
          atomicAdd(reinterpret_cast<float4*>(dst), v[0]);
        } else {
          const int left = L - t;
          atomicAdd(dst, v[0].x);
          if (left > 1) atomicAdd(dst + 1, v[0].y);
          if (left > 2) atomicAdd(dst + 2, v[0].z);
          if (left > 3) atomicAdd(dst + 3, v[0].w);
        }
      }
    }
    // per-token outputs of token n of row r
    {
      const int t = tb + n;
      const float du = fmaf(e_dy, Dv, e_dt * s1);
      const float dd = fmaf(e_u, s1, s2) * e_dsp;
      if (active && t < L) {
        ddbp += dd;
        static_cast<T*>(p.du)[row + t] = cvt<T>(du);
        static_cast<T*>(p.ddelta)[row + t] = cvt<T>(dd);
      }
    }
    if (kb >= 1) {
      convert(kb - 1);
      if (kb >= 2) prefetch(kb - 2);
    }
  }

  // per-row partials: dA as (re, im) pairs, dD and the delta-bias gradient
  if (nval) reinterpret_cast<float2*>(p.part_dA)[rowid * N + n] = make_float2(dAr, dAi);
  // the state before token 0 enters only through a_0 h_{-1}: its gradient is
  // the carry conj(a_0) g_0 left after the first block
  if (nval && p.dh0) reinterpret_cast<float2*>(p.dh0)[rowid * N + n] = make_float2(gr, gi);
#pragma unroll
  for (int off = 8; off > 0; off >>= 1) {
    dDp += __shfl_xor_sync(kFull, dDp, off);
    ddbp += __shfl_xor_sync(kFull, ddbp, off);
  }
  if (active && n == 0) {
    p.part_dD[rowid] = dDp;
    p.part_ddb[rowid] = ddbp;
  }
}

// dA[d][n][c] = sum_b part_dA[b][d][n][c], dD and ddelta_bias likewise, in a
// fixed order.
__global__ void cscan_param_reduce_kernel(const float* __restrict__ pA,
                                          const float* __restrict__ pD,
                                          const float* __restrict__ pB, float* __restrict__ dA,
                                          float* __restrict__ dD, float* __restrict__ ddb, int B,
                                          int D, int N2) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i < D * N2) {
    const int d = i / N2, k = i % N2;
    float s = 0.0f;
    for (int b = 0; b < B; ++b) s += pA[((size_t)b * D + d) * N2 + k];
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

template <typename T, bool VEC>
cudaError_t cfwd_t(const ScanArgs& a, cudaStream_t s) {
  dim3 g((a.D + kCRows - 1) / kCRows, a.B);
  cscan_fwd_kernel<T, VEC><<<g, kCThreads, 0, s>>>(a);
  return cudaGetLastError();
}

template <typename T, bool VEC>
cudaError_t cbwd_t(const ScanArgs& a, cudaStream_t s) {
  const size_t smem = sizeof(CBwdSmem<T>);
  static std::atomic<unsigned long long> smem_done{0};
  cudaError_t e = smem_attr(cscan_bwd_kernel<T, VEC>, (int)smem, &smem_done);
  if (e != cudaSuccess) return e;
  dim3 g((a.D + kCRows - 1) / kCRows, a.B);
  cscan_bwd_kernel<T, VEC><<<g, kCThreads, smem, s>>>(a);
  const int m = a.D * 2 * a.N;
  cscan_param_reduce_kernel<<<(m + 255) / 256, 256, 0, s>>>(a.part_dA, a.part_dD, a.part_ddb,
                                                           a.dA, a.dD, a.ddelta_bias, a.B, a.D,
                                                           2 * a.N);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_cscan_fwd(const ScanArgs& a, cudaStream_t s) {
  if (a.bf16) return a.vec ? cfwd_t<__nv_bfloat16, true>(a, s) : cfwd_t<__nv_bfloat16, false>(a, s);
  return a.vec ? cfwd_t<float, true>(a, s) : cfwd_t<float, false>(a, s);
}

cudaError_t launch_cscan_bwd(const ScanArgs& a, cudaStream_t s) {
  if (a.bf16) return a.vec ? cbwd_t<__nv_bfloat16, true>(a, s) : cbwd_t<__nv_bfloat16, false>(a, s);
  return a.vec ? cbwd_t<float, true>(a, s) : cbwd_t<float, false>(a, s);
}

SSM_DEBUG_TU(cscan)

}  // namespace ssm
