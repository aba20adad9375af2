// Mamba-2 SSD backward ("hung-phan ml-skills mamba", section "Mamba-2:
// Structured State Space Duality (SSD)"): the reverse mode of the chunked
// forward in ssd_fwd.cu, chunk by chunk from the last one, on the tensor
// cores. Per chunk of Q = 128 tokens, with the forward's quantities
//   S = C B^T,  Lm_ij = [ls_i <= j <= i] exp(lcs_i - lcs_j),  M = S o Lm diag(dt)
//   y_i = sum_j M_ij x_j + s_i C_i Hp + D x_i,  s_i = [ls_i < 0] exp(lcs_i)
//   H_end = dec Hp + sum_j w_j B_j^T x_j,  dec = [ls_Q-1 < 0] exp(lcs_Q-1),
//   w_j = [j >= ls_Q-1] dt_j exp(lcs_Q-1 - lcs_j)
// (Hp: the state entering the chunk, saved by the forward; states [n][p]),
// and dH the adjoint of H_end carried from the chunk to the right:
//   dx  = M^T dy + diag(w) B dH + D dy
//   dM  = dy x^T,  dS = dM o Lm diag(dt)
//   dC  = dS B + diag(s) dy Hp^T,   dB = dS^T C + diag(w) x dH^T
//   dHp = dec dH + C^T diag(s) dy                       (the next carry)
// and for the decays, with W = dM o S o Lm:
//   d lcs_i += sum_j W_ij dt_j - dt_i sum_k W_ki + s_i dy_i . (C_i Hp)
//              - w_i R_i,  R_i = x_i . (B_i dH)
//   d lcs_Q-1 += dec <dH, Hp> + sum_j w_j R_j
//   d dt_j (direct) = sum_i W_ij + (w_j / dt_j) R_j
// then lcs = cumsum(dt A) gives d dt_k += A sum_{i >= k} d lcs_i and
// dA += sum_k dt_k sum_{i >= k} d lcs_i. Document resets enter only through
// the masks (ls), as in the forward.
//
// Operands live in shared memory as bf16 tiles of 16-byte runs along a
// feature axis (rows = tokens or states); the tensor cores read one tile
// either K-major or MN-major by swapping the descriptor's two core-matrix
// strides, so every product above takes its operands without a transposed
// copy. Two groups of products per chunk: (C B^T, dy x^T, B dH, C Hp,
// C^T dYs) and, once M and dS are in shared memory, (M^T dy, dS B + dYs Hp^T,
// dS^T C, x dH^T); the second runs while the threads reduce the decay terms.
// A whole chunk's C, B, x, dy rows arrive by one tensor-map copy each (a
// ragged last chunk, or L not a multiple of 8, by cp.async), and dB / dC
// leave by tensor-map bulk reductions of staged boxes (see ssd_maps.cuh).
// One CTA of 256 threads per (b, h); 512 TMEM columns.
#include <atomic>
#include <cstring>

#include "scan_common.cuh"
#include "ssd_maps.cuh"

namespace ssm {

namespace {

constexpr int kQ = 128;   // tokens per chunk
constexpr int kP = 64;    // head dimension
constexpr int kNs = 128;  // state size
constexpr int kThreads = 256;

// Tile rows are 2 KB (128 features) or 1 KB (64 features) apart per 8-row group.
constexpr uint32_t kRs128 = 2048, kRs64 = 1024;

struct SsdBwdSmem {
  unsigned char C[kQ * kNs * 2];   // C_i[n]         rows i
  unsigned char Bm[kQ * kNs * 2];  // B_j[n]         rows j
  unsigned char M[kQ * kQ * 2];    // M_ij           rows i
  unsigned char dS[kQ * kQ * 2];   // dS_ij          rows i
  unsigned char X[kQ * kP * 2];    // x_j[p]         rows j
  unsigned char dY[kQ * kP * 2];   // dy_i[p]        rows i
  unsigned char dYs[kQ * kP * 2];  // s_i dy_i[p]    rows i
  unsigned char Hp[kNs * kP * 2];  // Hp[n][p]       rows n
  unsigned char dH[kNs * kP * 2];  // dH[n][p]       rows n
  float lcs[kQ];
  float dt[kQ];
  int ls[kQ];
  float colw[8][64];    // per warp: column sums of W over the warp's 32 rows
  float rowp[3][2][kQ]; // per row and column half: sum_j W dt, dy . (C Hp), x . (B dH)
  float wsum[8];
  int wmax[4];
  float blk[2][8];
  uint64_t bar;   // tensor-core products
  uint64_t tbar;  // tensor-map copies of a chunk's rows
  uint32_t tmem;
};

// byte offset of (row R, feature E) in a tile whose 8-row groups are rs bytes apart
__device__ __forceinline__ uint32_t toff(int R, int E, uint32_t rs) {
  return (R >> 3) * rs + (E >> 3) * 128 + (R & 7) * 16 + (E & 7) * 2;
}

// A tile seen as an MMA operand: start address, leading (K-direction) and
// stride (M / N-direction) byte offsets between core matrices, and the start
// advance per K = 16 step.
struct Opnd {
  uint32_t addr, lbo, sbo, kstep;
};
// K-major view: operand rows = tile rows, K = the feature axis
__device__ __forceinline__ Opnd kview(uint32_t addr, uint32_t rs) { return Opnd{addr, 128u, rs, 256u}; }
// MN-major view: operand rows = the feature axis, K = tile rows
__device__ __forceinline__ Opnd mnview(uint32_t addr, uint32_t rs) { return Opnd{addr, rs, 128u, 2u * rs}; }

__device__ __forceinline__ uint64_t mdesc(uint32_t addr, uint32_t lbo, uint32_t sbo) {
  return (uint64_t)((addr >> 4) & 0x3FFF) | ((uint64_t)((lbo >> 4) & 0x3FFF) << 16) |
         ((uint64_t)((sbo >> 4) & 0x3FFF) << 32) | (1ull << 46);
}

// D[128 x n] (+)= A B^T over K = k (bf16 in, fp32 accumulate); a_mn / b_mn:
// the views' majorness as the instruction descriptor encodes it.
__device__ __forceinline__ void mma(uint32_t d_tmem, Opnd A, Opnd B, int a_mn, int b_mn, int n, int k,
                                    bool accumulate) {
  const uint32_t idesc = (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)a_mn << 15) | ((uint32_t)b_mn << 16) |
                         ((uint32_t)(n >> 3) << 17) | ((uint32_t)(128 >> 4) << 24);
  for (int s = 0; s < k / 16; ++s) {
    const uint32_t acc = (accumulate || s > 0) ? 1u : 0u;
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, {%5, %6, %7, %8}, p;\n\t}\n" ::"r"(d_tmem),
        "l"(mdesc(A.addr + A.kstep * s, A.lbo, A.sbo)), "l"(mdesc(B.addr + B.kstep * s, B.lbo, B.sbo)),
        "r"(idesc), "r"(acc), "r"(0u), "r"(0u), "r"(0u), "r"(0u));
  }
}
__device__ __forceinline__ void mma_commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                   smem_u32(bar))
               : "memory");
}
__device__ __forceinline__ void tc_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

// 32 consecutive fp32 columns of this thread's TMEM lane (valid after tm_wait()).
__device__ __forceinline__ void tm_ld32(uint32_t addr, float f[32]) {
  uint32_t r[32];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, "
      "%13, %14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
        "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]),
        "=r"(r[23]), "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]),
        "=r"(r[30]), "=r"(r[31])
      : "r"(addr));
#pragma unroll
  for (int i = 0; i < 32; ++i) f[i] = __uint_as_float(r[i]);
}
__device__ __forceinline__ void tm_wait() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }

__device__ __forceinline__ uint32_t pk2(float a, float b) {
  const __nv_bfloat162 v = __floats2bfloat162_rn(a, b);
  return *reinterpret_cast<const uint32_t*>(&v);
}
__device__ __forceinline__ float lo_(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float hi_(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }
// 8 bf16 of a uint4 -> fp32
__device__ __forceinline__ void unpack8(const uint4 q, float* v) {
  v[0] = lo_(q.x); v[1] = hi_(q.x); v[2] = lo_(q.y); v[3] = hi_(q.y);
  v[4] = lo_(q.z); v[5] = hi_(q.z); v[6] = lo_(q.w); v[7] = hi_(q.w);
}
__device__ __forceinline__ uint4 pack8(const float* v) {
  return make_uint4(pk2(v[0], v[1]), pk2(v[2], v[3]), pk2(v[4], v[5]), pk2(v[6], v[7]));
}
// dst[0 .. bytes/4) += src[...] (fp32), one bulk reduction from shared memory
// (both 16-byte aligned, bytes a multiple of 16); completion of the read of
// src is awaited with bulk_wait_read().
__device__ __forceinline__ void bulk_add_f32(float* dst, const void* src, uint32_t bytes) {
  asm volatile("cp.reduce.async.bulk.global.shared::cta.bulk_group.add.f32 [%0], [%1], %2;" ::"l"(dst),
               "r"(smem_u32(src)), "r"(bytes)
               : "memory");
  asm volatile("cp.async.bulk.commit_group;" ::: "memory");
}
__device__ __forceinline__ void bulk_wait_read() { asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory"); }
__device__ __forceinline__ void prefetch_l2(const void* p) { asm volatile("prefetch.global.L2 [%0];" ::"l"(p)); }
// One operand tile (128 rows of a row-major [rows][groups][features] bf16
// tensor) by one tensor-map copy: the map's five dimensions (feature_lo 8,
// row_lo 8, feature_hi, group, row_hi) put the box in shared memory in the
// tiles' core-matrix order; rows past the tensor are zero-filled.
__device__ __forceinline__ void tma_tile(void* dst, const CUtensorMap* map, int group, int row_hi,
                                         uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.5d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3, %4, "
      "%5, %6}], [%7];" ::"r"(smem_u32(dst)),
      "l"(map), "r"(0), "r"(0), "r"(0), "r"(group), "r"(row_hi), "r"(smem_u32(bar))
      : "memory");
}

// 16 bytes global -> shared without registers; nbytes 0 fills zeros (src unread)
__device__ __forceinline__ void cp_async16(void* dst, const void* src, uint32_t nbytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(smem_u32(dst)), "l"(src), "r"(nbytes)
               : "memory");
}

// dB / dC rows are staged in shared memory the chunk's products no longer
// read (C, B, M, dS, x: free once the second group has completed) and added
// to global memory by bulk reductions. With tensor maps (tma bit 1): as four
// boxes of 32 states x 128 tokens per matrix in the 128-byte swizzled order
// (a row's 16-byte chunk k at chunk k ^ (row & 7): a warp's stores fall on
// distinct banks), dC in C / B and dB in M / dS, eight tensor reductions per
// chunk that undo the swizzle on the way out. Tokens past L carry exact
// zeros (their dt, dy, x are 0), so a box that reaches past L adds nothing.
// Otherwise rows 528 bytes apart (512 + 16), one 512-byte reduction per row.
constexpr uint32_t kStageRow = 528;
constexpr uint32_t kStageB = 0, kStageC = kQ * kStageRow;
constexpr uint32_t kBoxBytes = kQ * 128;  // 32 fp32 states x 128 tokens

// One staged box (32 states from n0, 128 tokens from row0, group g) added
// into a [rows][G][128] fp32 tensor by a tensor-map bulk reduction.
__device__ __forceinline__ void tma_add_box(const CUtensorMap* map, const void* src, int n0, int g, int row0) {
  asm volatile(
      "cp.reduce.async.bulk.tensor.3d.global.shared::cta.add.tile.bulk_group [%0, {%1, %2, %3}], [%4];" ::"l"(map),
      "r"(n0), "r"(g), "r"(row0), "r"(smem_u32(src))
      : "memory");
}

// Sum of v over the 32 lanes of the warp for each of 32 columns: recursive
// halving; lane l ends with column l.
__device__ __forceinline__ float colsum32(float v[32], int lane) {
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) {
    const bool up = (lane & o) != 0;
#pragma unroll
    for (int k = 0; k < o; ++k) {
      const float send = up ? v[k] : v[k + o];
      const float keep = up ? v[k + o] : v[k];
      v[k] = keep + __shfl_xor_sync(kFull, send, o);
    }
  }
  return v[0];
}

// tma bit 0: C, B ([B L][G][128]) and x, dy ([B L][H][64]) of whole chunks
// by tensor map (L a multiple of 8); else every chunk's rows by cp.async, as
// the ragged last chunk's always are. Bit 1: dB / dC by tensor reductions.
struct SsdMaps {
  CUtensorMap C, B, X, dY;  // bit 0 of tma
  CUtensorMap dB, dC;       // bit 1
};

__global__ void __launch_bounds__(kThreads, 1) ssd_bwd_kernel(const SsdArgs p, const __grid_constant__ SsdMaps maps,
                                                              const int tma) {
  static_assert(sizeof(SsdBwdSmem) <= 227 * 1024, "shared memory per CTA");
  static_assert(kStageC + kQ * kStageRow <= offsetof(SsdBwdSmem, dY), "dB / dC staging overlaps live tiles");
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  SsdBwdSmem& sm = *reinterpret_cast<SsdBwdSmem*>(smem_raw);
  const int t = threadIdx.x, warp = t >> 5, lane = t & 31;
  const int r = t & (kQ - 1), hf = t >> 7;  // token (or state) row, column half
  const int h = blockIdx.x, b = blockIdx.y;
  const int H = p.H, L = p.L, G = p.G;
  const int g = h / (H / G);
  const float Ah = __ldg(p.A + h);
  const float bias = p.dt_bias ? __ldg(p.dt_bias + h) : 0.0f;
  const float Dh = p.D ? __ldg(p.D + h) : 0.0f;
  const __nv_bfloat16* xg = static_cast<const __nv_bfloat16*>(p.x);
  const __nv_bfloat16* dyg = static_cast<const __nv_bfloat16*>(p.dy);
  const __nv_bfloat16* dtg = static_cast<const __nv_bfloat16*>(p.dt_raw);
  const __nv_bfloat16* Bg = static_cast<const __nv_bfloat16*>(p.Bm);
  const __nv_bfloat16* Cg = static_cast<const __nv_bfloat16*>(p.Cm);
  __nv_bfloat16* dxg = static_cast<__nv_bfloat16*>(p.dx);
  const int32_t* seqb = p.seq ? p.seq + (size_t)b * L : nullptr;
  const int nch = (L + kQ - 1) / kQ;
  const uint4 z4 = make_uint4(0u, 0u, 0u, 0u);

  if (t == 0) {
    mbar_init(&sm.bar, 1);
    mbar_init(&sm.tbar, 1);
    fence_mbar_init();
  }
  if (warp == 0) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], 512;" ::"r"(smem_u32(&sm.tmem))
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  // no gradient enters through the final state
  for (int i = t; i < kNs * kP * 2 / 16; i += kThreads) reinterpret_cast<uint4*>(sm.dH)[i] = z4;
  tc_before();
  __syncthreads();
  tc_after();
  const uint32_t tmem = sm.tmem;
  const uint32_t lrow = tmem + ((uint32_t)(32 * (warp & 3)) << 16);  // TMEM lane r
  const uint32_t sC = smem_u32(sm.C), sB = smem_u32(sm.Bm), sM = smem_u32(sm.M), sdS = smem_u32(sm.dS);
  const uint32_t sX = smem_u32(sm.X), sdY = smem_u32(sm.dY), sdYs = smem_u32(sm.dYs);
  const uint32_t sHp = smem_u32(sm.Hp), sdH = smem_u32(sm.dH);

  float dHc[32];  // dH[n = r][p = 32 hf ..]: the adjoint of the state leaving the chunk
#pragma unroll
  for (int q = 0; q < 32; ++q) dHc[q] = 0.0f;
  float dA_acc = 0.0f, dD_acc = 0.0f, ddb_acc = 0.0f;
  unsigned phase = 0, tphase = 0;

#pragma unroll 1
  for (int c = nch - 1; c >= 0; --c) {
    const int tok = c * kQ + r;
    const bool valid = tok < L;
    // x / dy / dx row half; B / C / dB / dC row half (used only for valid rows)
    const size_t xo = SSM_DIDX(kDbgSsdRow, (((size_t)b * L + tok) * H + h) * kP + 32 * hf, valid ? 32 : 0,
                               (size_t)p.B * L * H * kP);
    const size_t bo = SSM_DIDX(kDbgSsdRow, (((size_t)b * L + tok) * G + g) * kNs + 64 * hf, valid ? 64 : 0,
                               (size_t)p.B * L * G * kNs);
    // ---- this chunk's rows straight into their tiles: one tensor-map copy
    // per tile for a whole chunk, else cp.async (zero-filled past L); no
    // registers held ----
    const bool by_map = (tma & 1) && (c + 1) * kQ <= L;
    if (by_map) {
      if (t == 0) {
        const int rh = (int)(((size_t)b * L + (size_t)c * kQ) / 8);
        mbar_expect_tx(&sm.tbar, 2u * kQ * kNs * 2 + 2u * kQ * kP * 2);
        tma_tile(sm.C, &maps.C, g, rh, &sm.tbar);
        tma_tile(sm.Bm, &maps.B, g, rh, &sm.tbar);
        tma_tile(sm.X, &maps.X, h, rh, &sm.tbar);
        tma_tile(sm.dY, &maps.dY, h, rh, &sm.tbar);
      }
    } else {
      const size_t bs = valid ? bo : (((size_t)b * L) * G + g) * kNs + 64 * hf;  // in bounds when !valid
      const size_t xs = valid ? xo : (((size_t)b * L) * H + h) * kP + 32 * hf;
      const uint32_t nb = valid ? 16u : 0u;
      const uint4* crow = reinterpret_cast<const uint4*>(Cg + bs);
      const uint4* brow = reinterpret_cast<const uint4*>(Bg + bs);
      const uint4* xrow = reinterpret_cast<const uint4*>(xg + xs);
      const uint4* dyrow = reinterpret_cast<const uint4*>(dyg + xs);
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        cp_async16(sm.C + toff(r, 8 * (8 * hf + k), kRs128), crow + k, nb);
        cp_async16(sm.Bm + toff(r, 8 * (8 * hf + k), kRs128), brow + k, nb);
      }
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        cp_async16(sm.X + toff(r, 8 * (4 * hf + k), kRs64), xrow + k, nb);
        cp_async16(sm.dY + toff(r, 8 * (4 * hf + k), kRs64), dyrow + k, nb);
      }
      asm volatile("cp.async.commit_group;" ::: "memory");
    }
    // the state entering the chunk, row n = r: bf16 tile, and <dH, Hp> for d lcs_Q-1
    float hdh = 0.0f;
    {
      const float4* hrow = reinterpret_cast<const float4*>(
          p.chunk_states + SSM_DIDX(kDbgSsdChunkState, ((((size_t)b * H + h) * nch + c) * kNs + r) * kP + 32 * hf,
                                    32, (size_t)p.B * H * nch * kNs * kP));
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const float4 a0 = __ldg(hrow + 2 * k), a1 = __ldg(hrow + 2 * k + 1);
        const float v[8] = {a0.x, a0.y, a0.z, a0.w, a1.x, a1.y, a1.z, a1.w};
#pragma unroll
        for (int e = 0; e < 8; ++e) hdh = fmaf(dHc[8 * k + e], v[e], hdh);
        *reinterpret_cast<uint4*>(sm.Hp + toff(r, 8 * (4 * hf + k), kRs64)) = pack8(v);
      }
    }
    if (c > 0) {  // the previous chunk's rows into L2 while this one runs
      const size_t xp = xo - (size_t)kQ * H * kP, bp = bo - (size_t)kQ * G * kNs;
      prefetch_l2(Cg + bp);
      prefetch_l2(Bg + bp);
      prefetch_l2(xg + xp);
      prefetch_l2(dyg + xp);
      prefetch_l2(p.chunk_states + ((((size_t)b * H + h) * nch + c - 1) * kNs + r) * kP + 32 * hf);
    }
    const float dtv = valid ? __bfloat162float(dtg[SSM_DIDX(kDbgSsdRow, ((size_t)b * L + tok) * H + h, 1,
                                                             (size_t)p.B * L * H)]) + bias
                            : 0.0f;
    float dt = 0.0f;
    if (valid) dt = p.softplus ? (dtv > 20.0f ? dtv : log1pf(expf(dtv))) : dtv;
    bool start = false;
    if (valid && seqb && tok > 0) start = __ldg(seqb + tok) != __ldg(seqb + tok - 1);
    // this thread's x and dy values, from the filled tiles
    if (by_map) {
      const bool ok = mbar_wait_bounded(&sm.tbar, tphase, p.status);
      tphase ^= 1u;
      if (!__syncthreads_and(ok)) {
        // the copies have not landed: wait once more (bounded) so that they
        // do not land after the CTA has exited, then stop
        if (t == 0) mbar_wait_bounded(&sm.tbar, tphase ^ 1u, nullptr);
        break;
      }
    } else {
      asm volatile("cp.async.wait_all;" ::: "memory");
    }
    float xr[32], dyr[32];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      unpack8(*reinterpret_cast<const uint4*>(sm.X + toff(r, 8 * (4 * hf + k), kRs64)), xr + 8 * k);
      unpack8(*reinterpret_cast<const uint4*>(sm.dY + toff(r, 8 * (4 * hf + k), kRs64)), dyr + 8 * k);
    }
    // ---- chunk scans (warps 0-3): lcs = inclusive sum of dt A, ls = last document start ----
    float la = dt * Ah;
    int st = start ? r : -1;
    if (hf == 0) {
#pragma unroll
      for (int off = 1; off < 32; off <<= 1) {
        const float lo = __shfl_up_sync(kFull, la, off);
        const int so = __shfl_up_sync(kFull, st, off);
        if (lane >= off) {
          la += lo;
          st = max(st, so);
        }
      }
      if (lane == 31) {
        sm.wsum[warp] = la;
        sm.wmax[warp] = st;
      }
    }
    __syncthreads();
    if (hf == 0) {
      for (int w = 0; w < warp; ++w) {
        la += sm.wsum[w];
        st = max(st, sm.wmax[w]);
      }
      sm.lcs[r] = la;
      sm.dt[r] = dt;
      sm.ls[r] = st;
    }
    __syncthreads();
    la = sm.lcs[r];
    st = sm.ls[r];
    const float lcsQ = sm.lcs[kQ - 1];
    const int lsQ = sm.ls[kQ - 1];
    const float s_r = st < 0 ? __expf(la) : 0.0f;
    const float e_r = r >= lsQ ? __expf(lcsQ - la) : 0.0f;
    const float w_r = dt * e_r;
    const float dec = lsQ < 0 ? __expf(lcsQ) : 0.0f;
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      float v[8];
#pragma unroll
      for (int e = 0; e < 8; ++e) v[e] = s_r * dyr[8 * k + e];
      *reinterpret_cast<uint4*>(sm.dYs + toff(r, 8 * (4 * hf + k), kRs64)) = pack8(v);
    }
    // ---- products 1: S = C B^T, dM = dy x^T, B dH, C Hp, C^T dYs ----
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    tc_before();
    __syncthreads();
    tc_after();
    if (t == 0) {
      mma(tmem + 0, kview(sC, kRs128), kview(sB, kRs128), 0, 0, 128, 128, false);
      mma(tmem + 128, kview(sdY, kRs64), kview(sX, kRs64), 0, 0, 128, 64, false);
      mma(tmem + 256, kview(sB, kRs128), mnview(sdH, kRs64), 0, 1, 64, 128, false);
      mma(tmem + 320, kview(sC, kRs128), mnview(sHp, kRs64), 0, 1, 64, 128, false);
      mma(tmem + 384, mnview(sC, kRs128), mnview(sdYs, kRs64), 1, 1, 64, 128, false);
      mma_commit(&sm.bar);
    }
    bool ok = mbar_wait_bounded(&sm.bar, phase, p.status);
    phase ^= 1u;
    if (!__syncthreads_and(ok)) break;
    tc_after();
    // ---- M, dS into shared memory; sums of W = dM o S o Lm ----
    float roww = 0.0f;
#pragma unroll 1
    for (int blk = 0; blk < 2; ++blk) {
      const int j0 = 64 * hf + 32 * blk;
      float sv[32], mv[32];
      tm_ld32(lrow + j0, sv);
      tm_ld32(lrow + 128 + j0, mv);
      tm_wait();
#pragma unroll
      for (int e8 = 0; e8 < 32; e8 += 8) {
        float mo[8], so[8];
#pragma unroll
        for (int q = 0; q < 8; ++q) {
          const int j = j0 + e8 + q;
          const float lm = (j >= st && j <= r) ? __expf(la - sm.lcs[j]) : 0.0f;
          const float dtj = sm.dt[j];
          const float sl = sv[e8 + q] * lm, dml = mv[e8 + q] * lm;
          mo[q] = sl * dtj;
          so[q] = dml * dtj;
          const float w = dml * sv[e8 + q];
          roww = fmaf(w, dtj, roww);
          mv[e8 + q] = w;
        }
        *reinterpret_cast<uint4*>(sm.M + toff(r, j0 + e8, kRs128)) = pack8(mo);
        *reinterpret_cast<uint4*>(sm.dS + toff(r, j0 + e8, kRs128)) = pack8(so);
      }
      sm.colw[warp][32 * blk + lane] = colsum32(mv, lane);
    }
    // dy_r . (C_r Hp), x_r . (B_r dH), and the next carry dHp = dec dH + C^T dYs
    float ydot = 0.0f, rdot = 0.0f;
    {
      float yo[32], xs[32], hp[32];
      tm_ld32(lrow + 320 + 32 * hf, yo);
      tm_ld32(lrow + 256 + 32 * hf, xs);
      tm_ld32(lrow + 384 + 32 * hf, hp);
      tm_wait();
#pragma unroll
      for (int q = 0; q < 32; ++q) {
        ydot = fmaf(dyr[q], yo[q], ydot);
        rdot = fmaf(xr[q], xs[q], rdot);
        dHc[q] = fmaf(dec, dHc[q], hp[q]);  // from here on: the adjoint of Hp
      }
    }
    sm.rowp[0][hf][r] = roww;
    sm.rowp[1][hf][r] = ydot;
    sm.rowp[2][hf][r] = rdot;
    // ---- products 2 (they run while the decay terms are reduced) ----
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    tc_before();
    __syncthreads();
    tc_after();
    if (t == 0) {
      mma(tmem + 320, mnview(sM, kRs128), mnview(sdY, kRs64), 1, 1, 64, 128, false);   // M^T dy
      mma(tmem + 0, kview(sdS, kRs128), mnview(sB, kRs128), 0, 1, 128, 128, false);    // dS B
      mma(tmem + 0, kview(sdYs, kRs64), kview(sHp, kRs64), 0, 0, 128, 64, true);       // + dYs Hp^T
      mma(tmem + 128, mnview(sdS, kRs128), mnview(sC, kRs128), 1, 1, 128, 128, false); // dS^T C
      mma(tmem + 384, kview(sX, kRs64), kview(sdH, kRs64), 0, 0, 128, 64, false);      // x dH^T
      mma_commit(&sm.bar);
    }
    // ---- the decay terms of the chunk's tokens (threads of half 0: token r) ----
    float rr = 0.0f;
    if (hf == 0) rr = sm.rowp[2][0][r] + sm.rowp[2][1][r];
    float wr = hf == 0 ? w_r * rr : 0.0f;
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
      wr += __shfl_xor_sync(kFull, wr, off);
      hdh += __shfl_xor_sync(kFull, hdh, off);
    }
    if (lane == 0) {
      sm.blk[0][warp] = wr;
      sm.blk[1][warp] = hdh;
    }
    __syncthreads();
    float dl = 0.0f, ddt = 0.0f;
    if (hf == 0) {
      const int hj = r >> 6;
      float cw = 0.0f;
#pragma unroll
      for (int k = 0; k < 4; ++k) cw += sm.colw[4 * hj + k][r & 63];
      dl = sm.rowp[0][0][r] + sm.rowp[0][1][r] - dt * cw + s_r * (sm.rowp[1][0][r] + sm.rowp[1][1][r]) -
           w_r * rr;
      if (r == kQ - 1) {
        float wsum = 0.0f, hsum = 0.0f;
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          wsum += sm.blk[0][k];
          hsum += sm.blk[1][k];
        }
        dl += dec * hsum + wsum;
      }
      ddt = cw + e_r * rr;
      // suffix sums of d lcs over the chunk
      float sfx = dl;
#pragma unroll
      for (int off = 1; off < 32; off <<= 1) {
        const float v = __shfl_down_sync(kFull, sfx, off);
        if (lane + off < 32) sfx += v;
      }
      if (lane == 0) sm.wsum[warp] = sfx;
      dl = sfx;
    }
    __syncthreads();
    if (hf == 0) {
      for (int w = warp + 1; w < 4; ++w) dl += sm.wsum[w];
      ddt = fmaf(Ah, dl, ddt);
      dA_acc = fmaf(dt, dl, dA_acc);
      const float dv = p.softplus ? ddt * (1.0f / (1.0f + __expf(-dtv))) : ddt;
      if (valid) {
        p.ddt_raw[SSM_DIDX(kDbgSsdRow, ((size_t)b * L + tok) * H + h, 1, (size_t)p.B * L * H)] = dv;
        ddb_acc += dv;
      }
    }
#pragma unroll
    for (int q = 0; q < 32; ++q) dD_acc = fmaf(dyr[q], xr[q], dD_acc);
    ok = mbar_wait_bounded(&sm.bar, phase, p.status);
    phase ^= 1u;
    if (!__syncthreads_and(ok)) break;
    tc_after();
    // ---- dx, dC, dB of row r ----
    {
      float dxa[32], xs[32];
      tm_ld32(lrow + 320 + 32 * hf, dxa);
      tm_ld32(lrow + 256 + 32 * hf, xs);
      tm_wait();
      if (valid) {
        uint4* dst = reinterpret_cast<uint4*>(dxg + xo);
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          float v[8];
#pragma unroll
          for (int e = 0; e < 8; ++e)
            v[e] = fmaf(Dh, dyr[8 * k + e], fmaf(w_r, xs[8 * k + e], dxa[8 * k + e]));
          dst[k] = pack8(v);
        }
      }
    }
    const bool boxes = (tma & 2) != 0;
    float4* stB = reinterpret_cast<float4*>(smem_raw + kStageB + r * kStageRow);
    float4* stC = reinterpret_cast<float4*>(smem_raw + kStageC + r * kStageRow);
#pragma unroll 1
    for (int blk = 0; blk < 2; ++blk) {
      const int n0 = 64 * hf + 32 * blk;
      float cv[32], bv[32], tv[32];
      tm_ld32(lrow + n0, cv);
      tm_ld32(lrow + 128 + n0, bv);
      tm_ld32(lrow + 384 + n0, tv);
      tm_wait();
      // box n0 / 32 of each matrix, row r: 16-byte chunk k at k ^ (r & 7)
      unsigned char* bC = sm.C + (n0 / 32) * kBoxBytes + r * 128;
      unsigned char* bB = sm.M + (n0 / 32) * kBoxBytes + r * 128;
#pragma unroll
      for (int q = 0; q < 32; q += 4) {
        const float4 vc = make_float4(cv[q], cv[q + 1], cv[q + 2], cv[q + 3]);
        const float4 vb = make_float4(fmaf(w_r, tv[q], bv[q]), fmaf(w_r, tv[q + 1], bv[q + 1]),
                                      fmaf(w_r, tv[q + 2], bv[q + 2]), fmaf(w_r, tv[q + 3], bv[q + 3]));
        if (boxes) {
          const int ck = ((q / 4) ^ (r & 7)) * 16;
          *reinterpret_cast<float4*>(bC + ck) = vc;
          *reinterpret_cast<float4*>(bB + ck) = vb;
        } else {
          stC[(n0 + q) / 4] = vc;
          stB[(n0 + q) / 4] = vb;
        }
      }
    }
    // the carry for the chunk to the left, as the next products' operand
#pragma unroll
    for (int k = 0; k < 4; ++k)
      *reinterpret_cast<uint4*>(sm.dH + toff(r, 8 * (4 * hf + k), kRs64)) = pack8(dHc + 8 * k);
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    __syncthreads();
    if (boxes) {  // eight tensor reductions: four boxes of dC, four of dB
      if (t == 0) {
        const int row0 = (int)((size_t)b * L + (size_t)c * kQ);
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          tma_add_box(&maps.dC, sm.C + q * kBoxBytes, 32 * q, g, row0);
          tma_add_box(&maps.dB, sm.M + q * kBoxBytes, 32 * q, g, row0);
        }
        asm volatile("cp.async.bulk.commit_group;" ::: "memory");
        bulk_wait_read();  // the staging is refilled by the next chunk
      }
    } else if (valid) {  // row r of dC (half 0) or dB (half 1), summed into global memory
      const size_t ro = SSM_DIDX(kDbgSsdRow, (((size_t)b * L + tok) * G + g) * kNs, kNs, (size_t)p.B * L * G * kNs);
      if (hf == 0) bulk_add_f32(p.dC + ro, stC, kNs * 4);
      else bulk_add_f32(p.dB + ro, stB, kNs * 4);
      bulk_wait_read();  // the staging rows are refilled by the next chunk
    }
    // generic accesses to the tiles before the next chunk's tensor-map writes
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    tc_before();
    __syncthreads();  // every thread is done with this chunk's shared operands and TMEM
  }
  // per-head sums: dA, dD, d dt_bias
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) {
    dA_acc += __shfl_xor_sync(kFull, dA_acc, off);
    dD_acc += __shfl_xor_sync(kFull, dD_acc, off);
    ddb_acc += __shfl_xor_sync(kFull, ddb_acc, off);
  }
  if (lane == 0) {
    atomicAdd(p.dA + h, dA_acc);
    if (p.dD) atomicAdd(p.dD + h, dD_acc);
    if (p.ddt_bias) atomicAdd(p.ddt_bias + h, ddb_acc);
  }
  tc_before();
  __syncthreads();
  tc_after();
  if (warp == 0)
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, 512;" ::"r"(tmem) : "memory");
}

}  // namespace

cudaError_t launch_ssd_bwd(const SsdArgs& a, cudaStream_t s) {
  static std::atomic<unsigned long long> done{0};
  const int smem = (int)sizeof(SsdBwdSmem);
  cudaError_t e = smem_attr(ssd_bwd_kernel, smem, &done);
  if (e != cudaSuccess) return e;
  const size_t bn = (size_t)a.B * a.L * a.G * a.N * sizeof(float);
  if ((e = cudaMemsetAsync(a.dB, 0, bn, s)) != cudaSuccess) return e;
  if ((e = cudaMemsetAsync(a.dC, 0, bn, s)) != cudaSuccess) return e;
  if ((e = cudaMemsetAsync(a.dA, 0, (size_t)a.H * sizeof(float), s)) != cudaSuccess) return e;
  if (a.dD && (e = cudaMemsetAsync(a.dD, 0, (size_t)a.H * sizeof(float), s)) != cudaSuccess) return e;
  if (a.ddt_bias && (e = cudaMemsetAsync(a.ddt_bias, 0, (size_t)a.H * sizeof(float), s)) != cudaSuccess)
    return e;
  SsdMaps maps;
  memset(&maps, 0, sizeof(maps));
  int tma = 0;
  const SsdTensorMapEncode enc = ssd_tensor_map_encoder();
  const size_t rows = (size_t)a.B * a.L;
  if (enc && a.L % 8 == 0 && ssd_tile_map(enc, &maps.C, a.Cm, rows, a.G, kNs) &&
      ssd_tile_map(enc, &maps.B, a.Bm, rows, a.G, kNs) && ssd_tile_map(enc, &maps.X, a.x, rows, a.H, kP) &&
      ssd_tile_map(enc, &maps.dY, a.dy, rows, a.H, kP))
    tma |= 1;
  if (enc && ssd_sum_map(enc, &maps.dB, a.dB, rows, a.G) && ssd_sum_map(enc, &maps.dC, a.dC, rows, a.G)) tma |= 2;
  ssd_bwd_kernel<<<dim3(a.H, a.B), kThreads, smem, s>>>(a, maps, tma);
  return cudaGetLastError();
}

SSM_DEBUG_TU(ssd_bwd)

}  // namespace ssm
