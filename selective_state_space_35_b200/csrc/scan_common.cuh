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

__device__ __forceinline__ void lds8(const float* base, int lane, float v[8]) {
  const float4 a = reinterpret_cast<const float4*>(base)[lane];
  const float4 b = reinterpret_cast<const float4*>(base + 128)[lane];
  v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
  v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
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
// first: lane j ends with the composition of lanes 0..j.
__device__ __forceinline__ void warp_scan_fwd(float& P, float& H, int lane) {
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const float Pp = __shfl_up_sync(kFull, P, off);
    const float Hp = __shfl_up_sync(kFull, H, off);
    if (lane >= off) {
      H = fmaf(P, Hp, H);
      P *= Pp;
    }
  }
}

// Inclusive reverse warp scan of maps c -> P c + G, later lanes applied
// first: lane j ends with the composition of lanes j..31.
__device__ __forceinline__ void warp_scan_bwd(float& P, float& G, int lane) {
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const float Pn = __shfl_down_sync(kFull, P, off);
    const float Gn = __shfl_down_sync(kFull, G, off);
    if (lane + off < 32) {
      G = fmaf(P, Gn, G);
      P *= Pn;
    }
  }
}

}  // namespace ssm
