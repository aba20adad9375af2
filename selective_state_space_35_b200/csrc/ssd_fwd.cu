// Mamba-2 SSD forward ("hung-phan ml-skills mamba", section "Mamba-2:
// Structured State Space Duality (SSD)": a scalar decay per head, so the
// scan over a chunk of tokens is a masked matrix product that runs on the
// tensor cores). Per (batch b, head h), head dimension P = 64, state N = 128,
// with dt_t = softplus(dt_raw + bias) and a_t = exp(dt_t A_h) (0 at a
// document start):
//   h_t[p][n] = a_t h_{t-1}[p][n] + dt_t x_t[p] B_t[n],   y_t[p] = sum_n C_t[n] h_t[p][n] + D_h x_t[p].
// Chunks of Q = 128 tokens, with lcs_i = sum_{k<=i} dt_k A_h inside the chunk
// and ls_i the last document start at or before i (-1: none):
//   Y_diag = (C B^T o L) (dt x),   L_ij = exp(lcs_i - lcs_j) for ls_i <= j <= i, else 0
//   Y_off  = diag([ls_i < 0] exp(lcs_i)) C H_prev^T
//   H_new  = [ls_Q-1 < 0] exp(lcs_Q-1) H_prev + x^T diag(w) B,  w_j = dt_j exp(lcs_Q-1 - lcs_j) [j >= ls_Q-1]
// The products are bf16 tcgen05.mma with fp32 accumulators in tensor
// memory (TMEM), issued by one thread, their completion signalled on an
// mbarrier (bounded waits). Operands are written by the CTA's threads into
// shared memory in the K-major, no-swizzle core-matrix layout; the state
// H^T[n][p] stays in fp32 registers (thread n) across the chunks of a
// sequence. The decay-masked C B^T and the state entering the next chunk
// each enter as a bf16 pair (rounded value and rounded remainder, two
// products), and C H_prev^T takes its row scale in fp32 afterwards (C itself
// is exact in bf16): single bf16 roundings there would dominate the error of
// y, the state's wherever the off-chunk term is large against y.
//
// One CTA of 256 threads per (b, h): threads i and i + 128 own token i of
// the chunk (and TMEM lane i), each for half of its columns. The next
// chunk's rows are fetched while the current one is computed: x into the
// second of two x tiles at the chunk's start and B into the B tile once the
// first product has released it, each by one tensor-map copy (cp.async for a
// ragged last chunk or L not a multiple of 8), and C into registers. No TMA
// multicast, no cluster.
#include <atomic>
#include <cstring>

#include "scan_common.cuh"
#include "ssd_maps.cuh"

namespace ssm {

namespace {

constexpr int kQ = 128;  // tokens per chunk
constexpr int kP = 64;   // head dimension
constexpr int kNs = 128; // state size
constexpr int kThreads = 256;  // two threads per token row

// Shared memory: bf16 operands in the no-swizzle core-matrix layouts (core
// matrices 128 B apart along K, 2 KB apart along M / N): K-major where a row
// runs along K (C, B, the decay-masked product), MN-major where a thread
// writes a row along M / N (the w-scaled B, the state); x is stored by token
// rows (8-row groups 1 KB apart, two buffers) and read MN-major by swapping
// the descriptor's two strides.
struct SsdSmem {
  unsigned char C[kQ * kNs * 2];    // C [i][n]
  unsigned char Bm[kQ * kNs * 2];   // B [j][n]
  unsigned char M[kQ * kQ * 2];     // (C B^T o L) dt [i][j], rounded to bf16
  unsigned char Mlo[kQ * kQ * 2];   // its rounding remainder, rounded to bf16 (M = M + Mlo to ~2^-17)
  unsigned char Bw[kNs * kQ * 2];   // w_j B_j[n]: M = n, K = j, MN-major
  unsigned char X[2][kQ * kP * 2];  // x_j[p] of chunks c (buffer c & 1): rows j
  unsigned char Hb[kP * kNs * 2];   // H_prev[p][n]: N = p, K = n, MN-major, rounded to bf16
  unsigned char Hlo[kP * kNs * 2];  // its rounding remainder, rounded to bf16 (H_prev to ~2^-17)
  float lcs[kQ];
  float dt[kQ];
  float bt[kQ];     // dt_j e^(lcs_k - lcs_j), k = j | 15: the end of j's 16-column block
  int ls[kQ];
  float wsum[4];
  int wmax[4];
  uint64_t bar;   // tensor-core products
  uint64_t tbar;  // tensor-map copies of a chunk's B and x rows
  uint32_t tmem;
};

// element (r, k) of a K-major operand: a core matrix is 8 rows of 16 bytes along K
__device__ __forceinline__ uint32_t tile_off(int r, int k) {
  return (r >> 3) * 2048 + (k >> 3) * 128 + (r & 7) * 16 + (k & 7) * 2;
}
// element (mn, k) of an MN-major operand: a core matrix is 8 K rows of 16
// bytes along M / N
__device__ __forceinline__ uint32_t tile_off_mn(int mn, int k) {
  return (mn >> 3) * 2048 + (k >> 3) * 128 + (k & 7) * 16 + (mn & 7) * 2;
}
// Shared-memory matrix descriptor (sm100): start >> 4, leading byte offset
// (between K-adjacent core matrices) 128 B, stride byte offset (between
// 8-row groups) 2048 B, descriptor version 1, no swizzle.
__device__ __forceinline__ uint64_t umma_desc(uint32_t addr) {
  return (uint64_t)((addr >> 4) & 0x3FFF) | ((uint64_t)(128 >> 4) << 16) |
         ((uint64_t)(2048 >> 4) << 32) | (1ull << 46);
}
// Instruction descriptor, kind::f16: fp32 accumulator, bf16 A and B, A / B
// K-major (0) or MN-major (1), M = 128, N = n.
__device__ __forceinline__ uint32_t umma_idesc(int n, int a_mn, int b_mn) {
  return (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)a_mn << 15) | ((uint32_t)b_mn << 16) |
         ((uint32_t)(n >> 3) << 17) | ((uint32_t)(128 >> 4) << 24);
}
// A descriptor with given leading (K-direction) and stride (M / N-direction)
// byte offsets between core matrices.
__device__ __forceinline__ uint64_t umma_desc2(uint32_t addr, uint32_t lbo, uint32_t sbo) {
  return (uint64_t)((addr >> 4) & 0x3FFF) | ((uint64_t)((lbo >> 4) & 0x3FFF) << 16) |
         ((uint64_t)((sbo >> 4) & 0x3FFF) << 32) | (1ull << 46);
}
// An x tile (token rows, 8-row groups 1 KB apart) read MN-major (N = p,
// K = j): leading offset 1 KB, stride offset 128 B, 2 KB per K = 16 step.
constexpr uint32_t kXRs = 1024;

// D (+)= A B^T over K = 128 (eight K = 16 steps: two core matrices along K
// each), A 128 x 128, B n x 128; b_x: B is an x tile (MN-major view).
__device__ __forceinline__ void umma_k128(uint32_t d_tmem, uint32_t a_smem, uint32_t b_smem, int n,
                                          bool accumulate, int a_mn, int b_mn, bool b_x = false) {
  const uint32_t idesc = umma_idesc(n, a_mn, b_mn);
#pragma unroll
  for (int s = 0; s < 8; ++s) {
    const uint32_t acc = (accumulate || s > 0) ? 1u : 0u;
    const uint64_t bd = b_x ? umma_desc2(b_smem + 2 * kXRs * s, kXRs, 128) : umma_desc(b_smem + 256 * s);
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, {%5, %6, %7, %8}, p;\n\t}\n" ::"r"(d_tmem),
        "l"(umma_desc(a_smem + 256 * s)), "l"(bd), "r"(idesc), "r"(acc), "r"(0u), "r"(0u), "r"(0u), "r"(0u));
  }
}

// byte offset of (token j, feature p) in an x tile
__device__ __forceinline__ uint32_t x_off(int j, int p) {
  return (j >> 3) * kXRs + (p >> 3) * 128 + (j & 7) * 16 + (p & 7) * 2;
}

// One operand tile (128 rows of a row-major [rows][groups][features] bf16
// tensor) by one tensor-map copy into the tiles' core-matrix order (see
// ssd_maps.cuh); rows past the tensor are zero-filled.
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
__device__ __forceinline__ void umma_commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                   smem_u32(bar))
               : "memory");
}
__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

// 32 consecutive fp32 columns of this thread's TMEM lane (the values are
// valid after tmem_wait()).
__device__ __forceinline__ void tmem_ld32(uint32_t addr, uint32_t r[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, "
      "%13, %14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
        "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]),
        "=r"(r[23]), "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]),
        "=r"(r[30]), "=r"(r[31])
      : "r"(addr));
}
__device__ __forceinline__ void tmem_wait() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }

__device__ __forceinline__ uint32_t pack_bf16(float a, float b) {
  const __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
  return *reinterpret_cast<const uint32_t*>(&h);
}
__device__ __forceinline__ float bf_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf_hi(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }

// Register-fetched inputs of one chunk for one thread: half hf of token row r.
struct ChunkIn {
  uint4 c[8];  // C: n = 64 hf .. 64 hf + 63
  float dtv;   // raw dt + bias (as read)
  int seq_cur, seq_prev;
};

struct SsdFwdMaps {
  CUtensorMap B, X;
};

// maps: B ([B L][G][128]) and x ([B L][H][64]); tma false (L not a multiple
// of 8, or no map could be encoded): B and x rows of every chunk by cp.async.
__global__ void __launch_bounds__(kThreads, 1) ssd_fwd_kernel(const SsdArgs p, const __grid_constant__ SsdFwdMaps maps,
                                                              const int tma) {
  static_assert(sizeof(SsdSmem) <= 227 * 1024, "shared memory per CTA");
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  SsdSmem& sm = *reinterpret_cast<SsdSmem*>(smem_raw);
  const int t = threadIdx.x, warp = t >> 5, lane = t & 31;
  const int r = t & (kQ - 1), hf = t >> 7;  // token row of the chunk, column half
  const int h = blockIdx.x, b = blockIdx.y;
  const int H = p.H, L = p.L, G = p.G;
  const int g = h / (H / G);
  const float Ah = __ldg(p.A + h);
  const float bias = p.dt_bias ? __ldg(p.dt_bias + h) : 0.0f;
  const float Dh = p.D ? __ldg(p.D + h) : 0.0f;
  const __nv_bfloat16* xg = static_cast<const __nv_bfloat16*>(p.x);
  const __nv_bfloat16* dtg = static_cast<const __nv_bfloat16*>(p.dt_raw);
  const __nv_bfloat16* Bg = static_cast<const __nv_bfloat16*>(p.Bm);
  const __nv_bfloat16* Cg = static_cast<const __nv_bfloat16*>(p.Cm);
  __nv_bfloat16* yg = static_cast<__nv_bfloat16*>(p.y);
  const int32_t* seqb = p.seq ? p.seq + (size_t)b * L : nullptr;
  const uint4 z4 = make_uint4(0u, 0u, 0u, 0u);

  auto fetch = [&](int c, ChunkIn& in) {
    const int tok = c * kQ + r;
    const bool valid = tok < L;
    const uint4* crow =
        reinterpret_cast<const uint4*>(Cg + SSM_DIDX(kDbgSsdRow, (((size_t)b * L + tok) * G + g) * kNs,
                                                     valid ? kNs : 0, (size_t)p.B * L * G * kNs)) +
        8 * hf;
#pragma unroll
    for (int k = 0; k < 8; ++k) in.c[k] = valid ? __ldg(crow + k) : z4;
    in.dtv = valid ? __bfloat162float(dtg[SSM_DIDX(kDbgSsdRow, ((size_t)b * L + tok) * H + h, 1,
                                                    (size_t)p.B * L * H)]) + bias
                   : 0.0f;
    in.seq_cur = (seqb && valid) ? __ldg(seqb + tok) : 0;
    in.seq_prev = (seqb && valid && tok > 0) ? __ldg(seqb + tok - 1) : in.seq_cur;
  };
  const int nch = (L + kQ - 1) / kQ;
  auto by_map = [&](int cc) { return tma && (cc + 1) * kQ <= L; };
  // chunk cc's x rows into x tile cc & 1 (the first of its two copies:
  // arms the chunk's copy barrier for x and B together)
  auto load_x = [&](int cc) {
    unsigned char* xt = sm.X[cc & 1];
    if (by_map(cc)) {
      if (t == 0) {
        mbar_expect_tx(&sm.tbar, (unsigned)(kQ * kNs * 2 + kQ * kP * 2));
        tma_tile(xt, &maps.X, h, (int)(((size_t)b * L + (size_t)cc * kQ) / 8), &sm.tbar);
      }
    } else {
      const int tk = cc * kQ + r;
      const int tc = tk < L ? tk : 0;  // an in-bounds source when zero-filling
      const uint4* xrow =
          reinterpret_cast<const uint4*>(xg + SSM_DIDX(kDbgSsdRow, (((size_t)b * L + tc) * H + h) * kP,
                                                       tk < L ? kP : 0, (size_t)p.B * L * H * kP)) +
          4 * hf;
#pragma unroll
      for (int k = 0; k < 4; ++k) cp_async16(xt + x_off(r, 8 * (4 * hf + k)), xrow + k, tk < L ? 16u : 0u);
      asm volatile("cp.async.commit_group;" ::: "memory");
    }
  };
  // chunk cc's B rows into the B tile
  auto load_b = [&](int cc) {
    if (by_map(cc)) {
      if (t == 0) tma_tile(sm.Bm, &maps.B, g, (int)(((size_t)b * L + (size_t)cc * kQ) / 8), &sm.tbar);
    } else {
      const int tk = cc * kQ + r;
      const int tc = tk < L ? tk : 0;
      const uint4* brow =
          reinterpret_cast<const uint4*>(Bg + SSM_DIDX(kDbgSsdRow, (((size_t)b * L + tc) * G + g) * kNs,
                                                       tk < L ? kNs : 0, (size_t)p.B * L * G * kNs)) +
          8 * hf;
#pragma unroll
      for (int k = 0; k < 8; ++k) cp_async16(sm.Bm + tile_off(r, 8 * (8 * hf + k)), brow + k, tk < L ? 16u : 0u);
      asm volatile("cp.async.commit_group;" ::: "memory");
    }
  };
  unsigned tphase = 0;

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
  // H_prev = 0 before the first chunk
  for (int i = t; i < kP * kNs * 2 / 16; i += kThreads)
    reinterpret_cast<uint4*>(sm.Hb)[i] = reinterpret_cast<uint4*>(sm.Hlo)[i] = make_uint4(0u, 0u, 0u, 0u);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sm.tmem;
  const uint32_t lane_row = tmem + ((uint32_t)(32 * (warp & 3)) << 16);  // TMEM lane r
  // TMEM columns: S [0, 128), Y_diag [128, 192), chunk state S_c^T [192, 256),
  // C H_prev^T [256, 320)
  const uint32_t sC = smem_u32(sm.C), sB = smem_u32(sm.Bm), sM = smem_u32(sm.M);
  const uint32_t sBw = smem_u32(sm.Bw), sH = smem_u32(sm.Hb), sHlo = smem_u32(sm.Hlo);
  const uint32_t sMlo = smem_u32(sm.Mlo);

  float Ht[kP / 2];  // H^T[n = r][p = 32 hf ..], fp32 across the chunks
#pragma unroll
  for (int q = 0; q < kP / 2; ++q) Ht[q] = 0.0f;
  unsigned phase = 0;
  ChunkIn in;
  fetch(0, in);
  load_x(0);
  load_b(0);

#pragma unroll 1
  for (int c = 0; c < nch; ++c) {
    const int tok = c * kQ + r;
    const bool valid = tok < L;
    if (p.chunk_states) {  // the state entering this chunk, for the backward
      float4* cs = reinterpret_cast<float4*>(
          p.chunk_states + SSM_DIDX(kDbgSsdChunkState, ((((size_t)b * H + h) * nch + c) * kNs + r) * kP + 32 * hf,
                                    32, (size_t)p.B * H * nch * kNs * kP));
#pragma unroll
      for (int q = 0; q < kP / 8; ++q) cs[q] = make_float4(Ht[4 * q], Ht[4 * q + 1], Ht[4 * q + 2], Ht[4 * q + 3]);
    }
    // ---- this chunk's operands: C from registers; B and x tile c & 1 copied
    // during the previous chunk ----
#pragma unroll
    for (int k = 0; k < 8; ++k)
      *reinterpret_cast<uint4*>(sm.C + tile_off(r, 8 * (8 * hf + k))) = in.c[k];
    {
      bool ok = true;
      if (by_map(c)) {
        ok = mbar_wait_bounded(&sm.tbar, tphase, p.status);
        tphase ^= 1u;
      } else {
        asm volatile("cp.async.wait_all;" ::: "memory");
      }
      if (!__syncthreads_and(ok)) {
        // the copies have not landed: wait once more (bounded) so that they
        // do not land after the CTA has exited, then stop
        if (t == 0) mbar_wait_bounded(&sm.tbar, tphase ^ 1u, nullptr);
        break;
      }
    }
    const unsigned char* xt = sm.X[c & 1];
    const uint32_t sX = smem_u32(xt);
    uint4 xraw[4];  // x of token r, p = 32 hf .., for the D x term
#pragma unroll
    for (int k = 0; k < 4; ++k) xraw[k] = *reinterpret_cast<const uint4*>(xt + x_off(r, 8 * (4 * hf + k)));
    // the next chunk's x into the other tile, now (its last readers were the
    // previous chunk's products)
    if (c + 1 < nch) load_x(c + 1);
    float dt = 0.0f;
    if (valid) dt = p.softplus ? (in.dtv > 20.0f ? in.dtv : log1pf(expf(in.dtv))) : in.dtv;
    const bool start = valid && seqb && tok > 0 && in.seq_cur != in.seq_prev;
    // the next chunk's inputs are in flight while this one is computed
    if (c + 1 < nch) fetch(c + 1, in);
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
    if (hf == 0) sm.bt[r] = dt * __expf(sm.lcs[r | 15] - la);  // read after the next barrier
    const float lcsQ = sm.lcs[kQ - 1];
    const int lsQ = sm.ls[kQ - 1];
    // ---- B scaled by w_r = dt_r exp(lcs_Q-1 - lcs_r) [r >= ls_Q-1], MN-major ----
    const float wt = (r >= lsQ) ? dt * __expf(lcsQ - la) : 0.0f;
#pragma unroll
    for (int k = 0; k < 8; ++k) {  // n = 8 (8 hf + k) .. of token r
      const uint4 q = *reinterpret_cast<const uint4*>(sm.Bm + tile_off(r, 8 * (8 * hf + k)));
      *reinterpret_cast<uint4*>(sm.Bw + tile_off_mn(8 * (8 * hf + k), r)) =
          make_uint4(pack_bf16(bf_lo(q.x) * wt, bf_hi(q.x) * wt), pack_bf16(bf_lo(q.y) * wt, bf_hi(q.y) * wt),
                     pack_bf16(bf_lo(q.z) * wt, bf_hi(q.z) * wt), pack_bf16(bf_lo(q.w) * wt, bf_hi(q.w) * wt));
    }
    // ---- S = C B^T on the tensor cores ----
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (t == 0) {
      umma_k128(tmem, sC, sB, kQ, false, 0, 0);
      umma_commit(&sm.bar);
      // the products that do not need M run while the threads build it: C
      // H_prev^T (H_prev as a bf16 pair) and S_c^T = (diag(w) B)^T x (the
      // commit after Y_diag covers them)
      umma_k128(tmem + 256, sC, sH, kP, false, 0, 1);
      umma_k128(tmem + 256, sC, sHlo, kP, true, 0, 1);
      umma_k128(tmem + 192, sBw, sX, kP, false, 1, 1, true);
    }
    bool ok = mbar_wait_bounded(&sm.bar, phase, p.status);
    phase ^= 1u;
    if (!__syncthreads_and(ok)) break;
    tc_fence_after();
    // the B tile is free: the next chunk's B rows into it
    if (c + 1 < nch) load_b(c + 1);
    // ---- columns 64 hf .. 64 hf + 63 of row r of M = (C B^T o L) dt (pair hi / lo) ----
    // For a column j whose 16-column block ends (token k = j | 15) at or
    // before row r, e^(lcs_r - lcs_j) is taken as e^(lcs_r - lcs_k) times the
    // column's e^(lcs_k - lcs_j), both at most 1 since lcs does not increase
    // along the chunk: one exponential per row and block instead of one per
    // element. The block holding the diagonal keeps the direct form.
    uint32_t sraw[64];
    tmem_ld32(lane_row + 64 * hf, sraw);
    tmem_ld32(lane_row + 64 * hf + 32, sraw + 32);
    tmem_wait();
#pragma unroll
    for (int jj = 0; jj < 64; jj += 32) {
      const int j0 = 64 * hf + jj;
      const uint32_t* v = sraw + jj;
#pragma unroll
      for (int e = 0; e < 32; e += 8) {
        float m[8], rr[8];
        const int jg = j0 + e, kb = jg | 15;
        if (jg > r) {  // above the diagonal
#pragma unroll
          for (int q = 0; q < 8; ++q) m[q] = 0.0f;
        } else if (kb <= r) {
          const float a = __expf(la - sm.lcs[kb]);
#pragma unroll
          for (int q = 0; q < 8; ++q)
            m[q] = (jg + q >= st) ? __uint_as_float(v[e + q]) * (a * sm.bt[jg + q]) : 0.0f;
        } else {
#pragma unroll
          for (int q = 0; q < 8; ++q) {
            const int j = jg + q;
            m[q] = (j >= st && j <= r) ? __uint_as_float(v[e + q]) * __expf(la - sm.lcs[j]) * sm.dt[j] : 0.0f;
          }
        }
        const uint4 hi = make_uint4(pack_bf16(m[0], m[1]), pack_bf16(m[2], m[3]), pack_bf16(m[4], m[5]),
                                    pack_bf16(m[6], m[7]));
        const uint32_t hw[4] = {hi.x, hi.y, hi.z, hi.w};
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          rr[2 * q] = m[2 * q] - bf_lo(hw[q]);
          rr[2 * q + 1] = m[2 * q + 1] - bf_hi(hw[q]);
        }
        *reinterpret_cast<uint4*>(sm.M + tile_off(r, j0 + e)) = hi;
        *reinterpret_cast<uint4*>(sm.Mlo + tile_off(r, j0 + e)) =
            make_uint4(pack_bf16(rr[0], rr[1]), pack_bf16(rr[2], rr[3]), pack_bf16(rr[4], rr[5]),
                       pack_bf16(rr[6], rr[7]));
      }
    }
    // the off-chunk term's row scale, applied in fp32 in the epilogue (C enters
    // the product as given: exact in bf16)
    const float cs = st < 0 ? __expf(la) : 0.0f;
    // ---- Y_diag = M x (M as a bf16 pair) ----
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (t == 0) {
      umma_k128(tmem + 128, sM, sX, kP, false, 0, 1, true);
      umma_k128(tmem + 128, sMlo, sX, kP, true, 0, 1, true);
      umma_commit(&sm.bar);
    }
    ok = mbar_wait_bounded(&sm.bar, phase, p.status);
    phase ^= 1u;
    if (!__syncthreads_and(ok)) break;
    tc_fence_after();
    // ---- y row r (p = 32 hf ..); the state row n = r (p = 32 hf ..) ----
    {
      uint32_t yv[32], sv[32], ov[32];
      tmem_ld32(lane_row + 128 + 32 * hf, yv);
      tmem_ld32(lane_row + 192 + 32 * hf, sv);
      tmem_ld32(lane_row + 256 + 32 * hf, ov);
      tmem_wait();
      if (valid) {
        uint4* yrow = reinterpret_cast<uint4*>(yg + SSM_DIDX(kDbgSsdRow, (((size_t)b * L + tok) * H + h) * kP,
                                                             kP, (size_t)p.B * L * H * kP)) +
                      4 * hf;
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          const uint32_t w4[4] = {xraw[k].x, xraw[k].y, xraw[k].z, xraw[k].w};
          uint32_t o[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const int q = 8 * k + 2 * e;
            o[e] = pack_bf16(fmaf(Dh, bf_lo(w4[e]), fmaf(cs, __uint_as_float(ov[q]), __uint_as_float(yv[q]))),
                             fmaf(Dh, bf_hi(w4[e]), fmaf(cs, __uint_as_float(ov[q + 1]), __uint_as_float(yv[q + 1]))));
          }
          yrow[k] = make_uint4(o[0], o[1], o[2], o[3]);
        }
      }
      const float dec = lsQ < 0 ? __expf(lcsQ) : 0.0f;
#pragma unroll
      for (int q = 0; q < kP / 2; ++q) Ht[q] = fmaf(dec, Ht[q], __uint_as_float(sv[q]));
#pragma unroll
      for (int k = 0; k < 4; ++k) {  // p = 8 (4 hf + k) .. of state row n = r: rounded value and remainder
        const uint4 hi = make_uint4(pack_bf16(Ht[8 * k], Ht[8 * k + 1]), pack_bf16(Ht[8 * k + 2], Ht[8 * k + 3]),
                                    pack_bf16(Ht[8 * k + 4], Ht[8 * k + 5]), pack_bf16(Ht[8 * k + 6], Ht[8 * k + 7]));
        const uint32_t hw[4] = {hi.x, hi.y, hi.z, hi.w};
        float rr[8];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          rr[2 * e] = Ht[8 * k + 2 * e] - bf_lo(hw[e]);
          rr[2 * e + 1] = Ht[8 * k + 2 * e + 1] - bf_hi(hw[e]);
        }
        *reinterpret_cast<uint4*>(sm.Hb + tile_off_mn(8 * (4 * hf + k), r)) = hi;
        *reinterpret_cast<uint4*>(sm.Hlo + tile_off_mn(8 * (4 * hf + k), r)) =
            make_uint4(pack_bf16(rr[0], rr[1]), pack_bf16(rr[2], rr[3]), pack_bf16(rr[4], rr[5]), pack_bf16(rr[6], rr[7]));
      }
    }
    tc_fence_before();
    __syncthreads();  // every thread is done with this chunk's shared operands and TMEM
  }
  asm volatile("cp.async.wait_all;" ::: "memory");  // no copy lands after the CTA has exited
  if (p.final_state) {
#pragma unroll
    for (int q = 0; q < kP / 2; ++q)
      p.final_state[SSM_DIDX(kDbgSsdState, (((size_t)b * H + h) * kP + 32 * hf + q) * kNs + r, 1,
                             (size_t)p.B * H * kP * kNs)] = Ht[q];
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 0)
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, 512;" ::"r"(tmem) : "memory");
}

}  // namespace

cudaError_t launch_ssd_fwd(const SsdArgs& a, cudaStream_t s) {
  static std::atomic<unsigned long long> done{0};
  const int smem = (int)sizeof(SsdSmem);
  cudaError_t e = smem_attr(ssd_fwd_kernel, smem, &done);
  if (e != cudaSuccess) return e;
  SsdFwdMaps maps;
  memset(&maps, 0, sizeof(maps));
  int tma = 0;
  const SsdTensorMapEncode enc = a.L % 8 == 0 ? ssd_tensor_map_encoder() : nullptr;
  if (enc) {
    const size_t rows = (size_t)a.B * a.L;
    tma = ssd_tile_map(enc, &maps.B, a.Bm, rows, a.G, kNs) && ssd_tile_map(enc, &maps.X, a.x, rows, a.H, kP);
  }
  ssd_fwd_kernel<<<dim3(a.H, a.B), kThreads, smem, s>>>(a, maps, tma);
  return cudaGetLastError();
}

SSM_DEBUG_TU(ssd_fwd)

}  // namespace ssm
