// Pieces shared by the N = 16 selective-scan kernels (scan16_fwd.cu,
// scan16_bwd.cu): the layout constants, the checkpoint indexing the two
// kernels agree on, and packed (f32x2) element helpers.
//
// Work layout of both kernels: time is cut into chunks of 256 tokens and a
// chunk of one row is spread over 16 (forward) or 32 (backward) lanes of a
// warp, each lane owning a contiguous run of tokens; the lanes' pieces are
// joined with the associative operator of "hung-phan ml-skills mamba",
// "Hardware-Aware Parallel Scan": (a1, b1) + (a2, b2) = (a1 a2, a2 b1 + b2).
// The forward keeps the state entering every 8-token segment; the backward
// restarts each lane's 8 tokens from it, so its own scan is the adjoint's.
#pragma once

#include <atomic>

#include "scan_common.cuh"

namespace ssm {
namespace s16 {

constexpr int kN = 16;      // states
constexpr int kCh = 256;    // tokens per chunk
constexpr int kSeg = 8;     // tokens per checkpoint segment
constexpr int kSegs = kCh / kSeg;

// Checkpoints: [B][Dp][nchunks][kN][2][kSegs] fp32 with Dp = ceil(D / 2):
// rows 2p and 2p + 1 of a batch entry form row pair p, and for every chunk
// and state the 32 segment-entry states of each row of the pair are
// contiguous, so one warp-wide 4-byte load per row and state is coalesced in
// the backward, and a forward lane writes its two segments with one 8-byte
// store.
__host__ __device__ __forceinline__ size_t ck_chunk(int b, int rp, int Dp, int nch, int c) {
  return ((((size_t)b * Dp + rp) * nch + c) * kN) * (2 * kSegs);
}
// Floats of the checkpoint array of a call from `at` to its end (the extent
// the debug build's index checks hold checkpoint accesses to).
__device__ __forceinline__ long long ck_left(const ScanArgs& p, const float* at) {
  return (long long)ck_chunk(p.B, 0, p.Dp, p.nchunks, 0) - (long long)(at - p.ckpt);
}

// Forward B / C tiles, packed by pack_bc_fwd_kernel into [B][nchunks][mat][kN][64] float4:
// float4 (k * 16 + jj) of a (mat, state) row holds tokens 16jj+2k, 16jj+8+2k,
// 16jj+2k+1, 16jj+9+2k, i.e. the (a, b) token pairs of forward lane jj
// (sub-segment a = tokens 16jj .. 16jj+7, b = 16jj+8 .. 16jj+15).
constexpr int kFwdTileF4 = 2 * kN * 64;  // float4 per chunk (32 KB)

__device__ __forceinline__ float2 dup(float x) { return make_float2(x, x); }
__device__ __forceinline__ float2 fadd2(float2 a, float2 b) { return __fadd2_rn(a, b); }

// bf16 -> fp32 of the low / high half of a 32-bit word
__device__ __forceinline__ float lo16(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float hi16(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }

// Element i (0..7) of 8 bf16 in a uint4
__device__ __forceinline__ float bf8(const uint4& r, int i) {
  const uint32_t w = i < 2 ? r.x : i < 4 ? r.y : i < 6 ? r.z : r.w;
  return (i & 1) ? hi16(w) : lo16(w);
}

// 8 consecutive elements of a row as raw 16-byte (bf16) or 32-byte (fp32)
// vectors; `ok` false gives zeros.
template <typename T>
struct Raw8;
template <>
struct Raw8<__nv_bfloat16> {
  uint4 r;
  __device__ __forceinline__ void load(const __nv_bfloat16* p, bool ok) {
    r = ok ? __ldg(reinterpret_cast<const uint4*>(p)) : make_uint4(0u, 0u, 0u, 0u);
  }
  __device__ __forceinline__ float get(int i) const { return bf8(r, i); }
};
template <>
struct Raw8<float> {
  float4 a, b;
  __device__ __forceinline__ void load(const float* p, bool ok) {
    if (ok) {
      a = __ldg(reinterpret_cast<const float4*>(p));
      b = __ldg(reinterpret_cast<const float4*>(p) + 1);
    } else {
      a = b = make_float4(0.f, 0.f, 0.f, 0.f);
    }
  }
  __device__ __forceinline__ float get(int i) const {
    const float4& q = i < 4 ? a : b;
    const int k = i & 3;
    return k == 0 ? q.x : k == 1 ? q.y : k == 2 ? q.z : q.w;
  }
};

// Store 8 consecutive values (one 16-byte vector for bf16, two for fp32).
template <typename T>
__device__ __forceinline__ void store8(T* p, const float v[8]);
template <>
__device__ __forceinline__ void store8<__nv_bfloat16>(__nv_bfloat16* p, const float v[8]) {
  uint4 r;
  r.x = Io<__nv_bfloat16>::pack2(v[0], v[1]);
  r.y = Io<__nv_bfloat16>::pack2(v[2], v[3]);
  r.z = Io<__nv_bfloat16>::pack2(v[4], v[5]);
  r.w = Io<__nv_bfloat16>::pack2(v[6], v[7]);
  *reinterpret_cast<uint4*>(p) = r;
}
template <>
__device__ __forceinline__ void store8<float>(float* p, const float v[8]) {
  reinterpret_cast<float4*>(p)[0] = make_float4(v[0], v[1], v[2], v[3]);
  reinterpret_cast<float4*>(p)[1] = make_float4(v[4], v[5], v[6], v[7]);
}

// Round to the storage type and back (the value a later kernel reads).
template <typename T>
__device__ __forceinline__ float round_to(float v) {
  return sizeof(T) == 2 ? __bfloat162float(__float2bfloat16_rn(v)) : v;
}

// softplus on both halves, the same steps as softplus_sfu (common.cuh).
__device__ __forceinline__ float2 softplus2(float2 v) {
  return make_float2(softplus_sfu(v.x), softplus_sfu(v.y));
}

// Shuffle whose predicate output tells whether the source lane exists
// (returned as 1 / 0). up: source lane - off within segments of `width`
// lanes; down: lane + off within the warp.
template <int WIDTH>
__device__ __forceinline__ float shfl_up_ok(float v, int off, unsigned& ok) {
  float r;
  asm volatile("{\n\t.reg .pred q;\n\tshfl.sync.up.b32 %0|q, %2, %3, %4, -1;\n\tselp.u32 %1, 1, 0, q;\n\t}"
               : "=f"(r), "=r"(ok)
               : "f"(v), "r"(off), "r"((32 - WIDTH) << 8));
  return r;
}
__device__ __forceinline__ float shfl_down_ok(float v, int off, unsigned& ok) {
  float r;
  asm volatile("{\n\t.reg .pred q;\n\tshfl.sync.down.b32 %0|q, %2, %3, 31, -1;\n\tselp.u32 %1, 1, 0, q;\n\t}"
               : "=f"(r), "=r"(ok)
               : "f"(v), "r"(off));
  return r;
}

// One step of the forward scan inside groups of 16 lanes: lanes with a
// source lane off below them compose (P, H) <- (P Pp, P Hp + H).
__device__ __forceinline__ void fwd_step16(float& P, float& H, int off) {
  unsigned ok;
  const float Hp = shfl_up_ok<16>(H, off, ok);
  const float Pp = __shfl_up_sync(kFull, P, off, 16);
  if (ok) {
    H = fmaf(P, Hp, H);
    P *= Pp;
  }
}

// One step of the reverse scan over a warp on (row 0, row 1) pairs: lanes with
// a source lane off above them compose (P, G) <- (P Pn, P Gn + G).
__device__ __forceinline__ void bwd_step2(float2& P, float2& G, int off) {
  unsigned ok;
  const float2 Gn = make_float2(shfl_down_ok(G.x, off, ok), __shfl_down_sync(kFull, G.y, off));
  const float2 Pn = shfl_down2(P, off);
  if (ok) {
    G = ffma2(P, Gn, G);
    P = fmul2(P, Pn);
  }
}

// SMs of the current device (cached per device; 148 on B200).
inline int sm_count() {
  static std::atomic<int> cache[64];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 148;
  if (dev < 64) {
    const int v = cache[dev].load(std::memory_order_relaxed);
    if (v > 0) return v;
  }
  int n = 0;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
    n = 148;
  if (dev < 64) cache[dev].store(n, std::memory_order_relaxed);
  return n;
}

// Both kernels come in two CTA shapes: a small CTA several of which share an
// SM, and one CTA of 11 warps per SM. A CTA owns a fixed group of rows for the
// whole sequence, so the grid runs in waves of (SMs x CTAs per SM); the call
// takes the shape whose waves are fullest (CTAs / capacity of the waves it
// needs), the small one on a tie. At B = 2, D = 1536 on 148 SMs: 22-row CTAs
// fill 140 / 148 of one wave, 12-row CTAs 256 / 296.
inline int pick_shape(int B, int D, int rows_small, int per_sm_small, int rows_big) {
  const long sms = sm_count();
  auto fill = [&](int rows, int per_sm) {
    const long ctas = (long)B * ((D + rows - 1) / rows);
    const long cap = sms * per_sm;
    return (double)ctas / (double)(((ctas + cap - 1) / cap) * cap);
  };
  return fill(rows_big, 1) > fill(rows_small, per_sm_small) + 1e-9 ? 1 : 0;
}

}  // namespace s16

cudaError_t launch_scan16_fwd(const ScanArgs& a, cudaStream_t s);
cudaError_t launch_scan16_bwd(const ScanArgs& a, cudaStream_t s);
// Whole-row summaries of a piece (N = 16 layout): forward (product of the
// decays, final state from zero) and backward (product of the decays, the
// adjoint leaving token 0 from the piece's own dout), into split_P / split_H.
cudaError_t launch_scan16_fwd_summary(const ScanArgs& a, cudaStream_t s);
cudaError_t launch_scan16_bwd_summary(const ScanArgs& a, cudaStream_t s);
// Rows per CTA the N = 16 backward uses for these arguments (the row groups
// of its deterministic dB / dC partials).
int scan16_bwd_rows(const ScanArgs& a);

}  // namespace ssm
