// Pieces shared by the selective-scan forward and backward kernels.
//
// Work layout: one warp owns one (b, d) row and walks it in chunks of
// kChunk = 256 tokens; lane j of the warp owns tokens [8j, 8j+8) of the chunk
// and keeps their per-token values in registers. The N state recurrences of
// a row are independent, so the kernels loop over n; for each n a lane first
// composes its 8 steps locally, the 32 lane pieces are then combined with the
// associative operator of "hung-phan ml-skills mamba", section
// "Hardware-Aware Parallel Scan": (a1, b1) + (a2, b2) = (a1 a2, a2 b1 + b2),
// as a 5-step warp-shuffle scan, and each lane finally replays its 8 steps
// from the exact incoming state. B_t and C_t ([B][N][L], shared by every
// channel of a batch row) are staged once per CTA and chunk into shared
// memory as fp32 and read by all of the CTA's warps.
#pragma once

#include "common.cuh"
#include "internal.h"

namespace ssm {

// Shared-memory position of token tau (0..255) of a chunk: the 8 tokens of
// lane j live at [4j, 4j+4) and [128+4j, 128+4j+4), so each lane reads two
// float4 and a warp's 32 float4 reads are 512 contiguous bytes.
__device__ __forceinline__ int chunk_pos(int lane, int i) { return ((i >> 2) << 7) + lane * 4 + (i & 3); }

// Stage B (if sB) and C (if sC) for chunk tokens [t0, t0+kChunk) of batch b.
template <typename T, bool VEC>
__device__ __forceinline__ void stage_bc(const T* __restrict__ Bm, const T* __restrict__ Cm,
                                         float* sB, float* sC, int b, int N, int L, int t0) {
  const int nslots = N * 32;
  const int first = sB ? 0 : nslots;
  const int last = sC ? 2 * nslots : nslots;
  for (int idx = first + threadIdx.x; idx < last; idx += blockDim.x) {
    const int mat = idx >= nslots;
    const int rem = idx - mat * nslots;
    const int n = rem >> 5, j = rem & 31;
    const T* src = (mat ? Cm : Bm) + ((size_t)b * N + n) * L;
    float v[8];
    load_row8<T, VEC>(src, t0 + j * 8, L, v);
    float* dst = (mat ? sC : sB) + n * kChunk;
    reinterpret_cast<float4*>(dst)[j] = make_float4(v[0], v[1], v[2], v[3]);
    reinterpret_cast<float4*>(dst + 128)[j] = make_float4(v[4], v[5], v[6], v[7]);
  }
}

// Paired layout: states (2m, 2m+1) of token tau share one float2; lane j's 8
// tokens sit in four 16-byte pieces at float4 index k*32 + j (tokens 2k, 2k+1),
// so a warp reads 512 contiguous bytes per piece.
template <typename T, bool VEC>
__device__ __forceinline__ void stage_pairs(const T* __restrict__ M, float2* s, int b, int N, int L,
                                            int t0) {
  const int NP = (N + 1) >> 1;
  for (int idx = threadIdx.x; idx < NP * 32; idx += blockDim.x) {
    const int m = idx >> 5, j = idx & 31;
    const int n0 = 2 * m, n1 = 2 * m + 1;
    float v0[8], v1[8];
    load_row8<T, VEC>(M + ((size_t)b * N + n0) * L, t0 + 8 * j, L, v0);
    if (n1 < N) {
      load_row8<T, VEC>(M + ((size_t)b * N + n1) * L, t0 + 8 * j, L, v1);
    } else {
#pragma unroll
      for (int i = 0; i < 8; ++i) v1[i] = 0.0f;
    }
    float4* dst = reinterpret_cast<float4*>(s + m * kChunk);
#pragma unroll
    for (int k = 0; k < 4; ++k)
      dst[k * 32 + j] = make_float4(v0[2 * k], v1[2 * k], v0[2 * k + 1], v1[2 * k + 1]);
  }
}

// Lane `lane`'s 8 tokens of one state pair from a paired tile.
__device__ __forceinline__ void lds_pair8(const float2* tile, int lane, float2 v[8]) {
  const float4* t4 = reinterpret_cast<const float4*>(tile);
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    const float4 q = t4[k * 32 + lane];
    v[2 * k] = make_float2(q.x, q.y);
    v[2 * k + 1] = make_float2(q.z, q.w);
  }
}

// 8 consecutive activations of one lane, held raw in registers between the
// load (issued one chunk ahead) and their use.
template <typename T, bool VEC>
struct Tok8 {
  float v[8];
  __device__ __forceinline__ void load(const T* row, int t, int L) { load_row8<T, VEC>(row, t, L, v); }
  __device__ __forceinline__ void get(float o[8]) const {
#pragma unroll
    for (int i = 0; i < 8; ++i) o[i] = v[i];
  }
};

template <>
struct Tok8<__nv_bfloat16, true> {
  uint4 r;
  __device__ __forceinline__ void load(const __nv_bfloat16* row, int t, int L) {
    r = (t < L) ? __ldg(reinterpret_cast<const uint4*>(row + t)) : make_uint4(0u, 0u, 0u, 0u);
  }
  __device__ __forceinline__ void get(float o[8]) const {
    o[0] = bf16lo(r.x); o[1] = bf16hi(r.x); o[2] = bf16lo(r.y); o[3] = bf16hi(r.y);
    o[4] = bf16lo(r.z); o[5] = bf16hi(r.z); o[6] = bf16lo(r.w); o[7] = bf16hi(r.w);
  }
};

__device__ __forceinline__ float2 f2(float x, float y) { return make_float2(x, y); }
__device__ __forceinline__ float2 ffma2(float2 a, float2 b, float2 c) { return __ffma2_rn(a, b, c); }
__device__ __forceinline__ float2 fmul2(float2 a, float2 b) { return __fmul2_rn(a, b); }
__device__ __forceinline__ float2 ex2x2(float2 e) { return make_float2(ex2_approx(e.x), ex2_approx(e.y)); }
__device__ __forceinline__ float2 shfl_up2(float2 v, int off) {
  return make_float2(__shfl_up_sync(kFull, v.x, off), __shfl_up_sync(kFull, v.y, off));
}
__device__ __forceinline__ float2 shfl_down2(float2 v, int off) {
  return make_float2(__shfl_down_sync(kFull, v.x, off), __shfl_down_sync(kFull, v.y, off));
}
__device__ __forceinline__ float2 shfl2(float2 v, int src) {
  return make_float2(__shfl_sync(kFull, v.x, src), __shfl_sync(kFull, v.y, src));
}

// Pair versions of the two warp scans (two independent states at once).
__device__ __forceinline__ void warp_scan_fwd2(float2& P, float2& H, int lane) {
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const float2 Pp = shfl_up2(P, off);
    const float2 Hp = shfl_up2(H, off);
    if (lane >= off) {
      H = ffma2(P, Hp, H);
      P = fmul2(P, Pp);
    }
  }
}

__device__ __forceinline__ void warp_scan_bwd2(float2& P, float2& G, int lane) {
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const float2 Pn = shfl_down2(P, off);
    const float2 Gn = shfl_down2(G, off);
    if (lane + off < 32) {
      G = ffma2(P, Gn, G);
      P = fmul2(P, Pn);
    }
  }
}

__device__ __forceinline__ void lds8(const float* base, int lane, float v[8]) {
  const float4 a = reinterpret_cast<const float4*>(base)[lane];
  const float4 b = reinterpret_cast<const float4*>(base + 128)[lane];
  v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
  v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
}

// ---------------------------------------------------------------------------
// TMA bulk copies (cp.async.bulk, no multicast) completing on an mbarrier.
// Every wait is bounded: after kMaxWaitIters polls the kernel records
// SSM_ERR_TIMEOUT in the status word and stops, instead of hanging.
// ---------------------------------------------------------------------------
constexpr int kMaxWaitIters = 1 << 22;
constexpr int kStatusTimeout = 4;  // == SSM_ERR_TIMEOUT

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
__device__ __forceinline__ void mbar_init(uint64_t* bar, unsigned count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}
__device__ __forceinline__ void fence_mbar_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}
__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}
__device__ __forceinline__ void mbar_expect_tx(uint64_t* bar, unsigned bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)),
               "r"(bytes)
               : "memory");
}
// 1-D bulk copy global -> shared; src, dst 16-byte aligned, bytes % 16 == 0.
__device__ __forceinline__ void tma_load_1d(void* dst, const void* src, unsigned bytes,
                                            uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          smem_u32(dst)),
      "l"(src), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, unsigned parity) {
  unsigned ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\tmbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}
// Returns false (and records a timeout in *status) if the phase never completes.
__device__ __forceinline__ bool mbar_wait_bounded(uint64_t* bar, unsigned parity, int* status) {
  for (int i = 0; i < kMaxWaitIters; ++i)
    if (mbar_try_wait(bar, parity)) return true;
  if (status) atomicExch(status, kStatusTimeout);
  return false;
}

// Issue, from warp 0, the bulk copies of rows [0, N) of B (and C) for chunk
// tokens [t0, t0 + kChunk) into raw[mat][n][.] bf16: lane 0 arms the
// mbarrier with the total byte count, then lane i copies row i (mats * N <=
// 32 rows). Rows past L are shorter; the converter masks them.
__device__ __forceinline__ void tma_issue_bc(const __nv_bfloat16* __restrict__ Bm,
                                             const __nv_bfloat16* __restrict__ Cm,
                                             __nv_bfloat16* raw, int mats, int b, int N, int L,
                                             int t0, uint64_t* bar) {
  const int lane = threadIdx.x & 31;
  const int ntok = min(kChunk, L - t0);
  const unsigned bytes = static_cast<unsigned>(ntok) * 2u;  // multiple of 16: L % 8 == 0
  // The raw buffer was last read (generic loads) before the CTA barrier that
  // precedes this call, so the async-proxy writes below cannot overtake them.
  if (lane == 0) mbar_expect_tx(bar, bytes * static_cast<unsigned>(mats * N));
  __syncwarp();
  if (lane < mats * N) {
    const int mat = lane >= N, n = lane - mat * N;
    tma_load_1d(raw + ((size_t)mat * kNMax + n) * kChunk,
                (mat ? Cm : Bm) + ((size_t)b * N + n) * L + t0, bytes, bar);
  }
}

// ---------------------------------------------------------------------------
// Asynchronous staging of the raw bf16 B / C chunk tiles (vector path): the
// copies for chunk c+1 are issued with cp.async while chunk c is computed, so
// their latency is hidden; each thread later converts exactly the pieces it
// copied. raw layout: [mat][n][kChunk] bf16 (mat 0 = B, 1 = C).
// ---------------------------------------------------------------------------
__device__ __forceinline__ void cp_async16(void* smem_dst, const void* gmem_src, bool valid) {
  const unsigned d = static_cast<unsigned>(__cvta_generic_to_shared(smem_dst));
  const int n = valid ? 16 : 0;  // 0 source bytes: the 16 bytes are zero-filled
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;\n" ::"r"(d), "l"(gmem_src), "r"(n)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;\n" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_group 0;\n" ::: "memory"); }

// Issue this thread's copies of chunk tokens [t0, t0+kChunk) of rows n of B
// (and C): item (mat, n, j) = 16 bytes = tokens [8j, 8j+8) of row n.
__device__ __forceinline__ void issue_bc_raw(const __nv_bfloat16* __restrict__ Bm,
                                             const __nv_bfloat16* __restrict__ Cm,
                                             __nv_bfloat16* raw, int mats, int b, int N, int L,
                                             int t0) {
  const int per = N * 32;
  for (int idx = threadIdx.x; idx < mats * per; idx += blockDim.x) {
    const int mat = idx >= per;
    const int rem = idx - mat * per;
    const int n = rem >> 5, j = rem & 31;
    const __nv_bfloat16* rowp = (mat ? Cm : Bm) + ((size_t)b * N + n) * L;
    const int t = t0 + 8 * j;
    const bool ok = t < L;
    cp_async16(raw + ((size_t)mat * kNMax + n) * kChunk + 8 * j, ok ? rowp + t : rowp, ok);
  }
  cp_async_commit();
}

// Convert this thread's pieces (same idx mapping as issue_bc_raw) into the
// fp32 row tile layout: row n, float4 index j = tokens [8j, 8j+4), 32 + j =
// [8j+4, 8j+8).
__device__ __forceinline__ void convert_bc_rows(const __nv_bfloat16* raw, float* sB, float* sC,
                                                int mats, int N, int tleft = kChunk) {
  const int per = N * 32;
  for (int idx = threadIdx.x; idx < mats * per; idx += blockDim.x) {
    const int mat = idx >= per;
    const int rem = idx - mat * per;
    const int n = rem >> 5, j = rem & 31;
    uint4 r = *reinterpret_cast<const uint4*>(raw + ((size_t)mat * kNMax + n) * kChunk + 8 * j);
    if (8 * j >= tleft) r = make_uint4(0u, 0u, 0u, 0u);  // past the end of the row
    float4* dst = reinterpret_cast<float4*>((mat ? sC : sB) + n * kChunk);
    dst[j] = make_float4(bf16lo(r.x), bf16hi(r.x), bf16lo(r.y), bf16hi(r.y));
    dst[32 + j] = make_float4(bf16lo(r.z), bf16hi(r.z), bf16lo(r.w), bf16hi(r.w));
  }
}

// Same, into the state-pair layout of stage_pairs; items are (mat, m, j) and
// cover rows 2m and 2m+1, so a thread converts what it copied only when the
// copy used the pair mapping below.
__device__ __forceinline__ void issue_bc_raw_pairs(const __nv_bfloat16* __restrict__ Bm,
                                                   const __nv_bfloat16* __restrict__ Cm,
                                                   __nv_bfloat16* raw, int mats, int b, int N,
                                                   int L, int t0) {
  const int NP = (N + 1) >> 1;
  const int per = NP * 32;
  for (int idx = threadIdx.x; idx < mats * per; idx += blockDim.x) {
    const int mat = idx >= per;
    const int rem = idx - mat * per;
    const int m = rem >> 5, j = rem & 31;
    const int t = t0 + 8 * j;
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int n = 2 * m + h;
      const bool rowok = n < N;
      const __nv_bfloat16* rowp = (mat ? Cm : Bm) + ((size_t)b * N + (rowok ? n : 0)) * L;
      const bool ok = rowok && t < L;
      cp_async16(raw + ((size_t)mat * kNMax + n) * kChunk + 8 * j, ok ? rowp + t : rowp, ok);
    }
  }
  cp_async_commit();
}

__device__ __forceinline__ void convert_bc_pairs(const __nv_bfloat16* raw, float2* sB, float2* sC,
                                                 int mats, int N, int tleft = kChunk) {
  const int NP = (N + 1) >> 1;
  const int per = NP * 32;
  for (int idx = threadIdx.x; idx < mats * per; idx += blockDim.x) {
    const int mat = idx >= per;
    const int rem = idx - mat * per;
    const int m = rem >> 5, j = rem & 31;
    uint4 r0 = *reinterpret_cast<const uint4*>(raw + ((size_t)mat * kNMax + 2 * m) * kChunk + 8 * j);
    uint4 r1 = *reinterpret_cast<const uint4*>(raw + ((size_t)mat * kNMax + 2 * m + 1) * kChunk + 8 * j);
    if (8 * j >= tleft) r0 = r1 = make_uint4(0u, 0u, 0u, 0u);  // past the end of the row
    if (2 * m + 1 >= N) r1 = make_uint4(0u, 0u, 0u, 0u);        // padding state of an odd N
    float4* dst = reinterpret_cast<float4*>((mat ? sC : sB) + m * kChunk);
    dst[j] = make_float4(bf16lo(r0.x), bf16lo(r1.x), bf16hi(r0.x), bf16hi(r1.x));
    dst[32 + j] = make_float4(bf16lo(r0.y), bf16lo(r1.y), bf16hi(r0.y), bf16hi(r1.y));
    dst[64 + j] = make_float4(bf16lo(r0.z), bf16lo(r1.z), bf16hi(r0.z), bf16hi(r1.z));
    dst[96 + j] = make_float4(bf16lo(r0.w), bf16lo(r1.w), bf16hi(r0.w), bf16hi(r1.w));
  }
}

// Bit i set <=> token tl+i (< L, > 0) starts a new document.
__device__ __forceinline__ unsigned reset_mask(const int32_t* __restrict__ seq, int b, int L, int tl) {
  if (!seq) return 0u;
  const int32_t* sr = seq + (size_t)b * L;
  unsigned m = 0u;
  int prev = (tl > 0 && tl - 1 < L) ? __ldg(sr + tl - 1) : 0;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int t = tl + i;
    if (t < L) {
      const int cur = __ldg(sr + t);
      if (t > 0 && cur != prev) m |= 1u << i;
      prev = cur;
    }
  }
  return m;
}

// Inclusive warp scan of affine maps h -> P h + H, earlier lanes applied
// first: lane j ends with the composition of lanes 0..j. The combine is a
// predicated FMA / MUL pair (lanes below the offset keep their value).
__device__ __forceinline__ void warp_scan_fwd(float& P, float& H, int lane) {
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const float Pp = __shfl_up_sync(kFull, P, off);
    const float Hp = __shfl_up_sync(kFull, H, off);
    asm("{\n\t.reg .pred q;\n\tsetp.ge.s32 q, %2, %3;\n\t"
        "@q fma.rn.f32 %1, %0, %5, %1;\n\t@q mul.rn.f32 %0, %0, %4;\n\t}"
        : "+f"(P), "+f"(H)
        : "r"(lane), "r"(off), "f"(Pp), "f"(Hp));
  }
}

// Inclusive reverse warp scan of maps c -> P c + G, later lanes applied
// first: lane j ends with the composition of lanes j..31.
__device__ __forceinline__ void warp_scan_bwd(float& P, float& G, int lane) {
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const float Pn = __shfl_down_sync(kFull, P, off);
    const float Gn = __shfl_down_sync(kFull, G, off);
    asm("{\n\t.reg .pred q;\n\tsetp.lt.s32 q, %2, %3;\n\t"
        "@q fma.rn.f32 %1, %0, %5, %1;\n\t@q mul.rn.f32 %0, %0, %4;\n\t}"
        : "+f"(P), "+f"(G)
        : "r"(lane), "r"(32 - off), "f"(Pn), "f"(Gn));
  }
}

}  // namespace ssm
