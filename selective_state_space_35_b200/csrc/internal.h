// Host-side internal interface between the C ABI (abi.cu) and the kernel
// launchers. Not installed; the public interface is include/ssmscan.h.
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include <atomic>

namespace ssm {

constexpr int kS = 8;                 // tokens per lane in the scan kernels
constexpr int kChunk = 32 * kS;       // tokens per warp-chunk
constexpr int kNMax = 16;             // largest supported state size
constexpr int kConvThreads = 128;     // threads per conv CTA (8 tokens each)
constexpr int kConvTile = kConvThreads * 8;

struct ConvArgs {
  const void* x;
  const float* w;
  const float* bias;
  const int32_t* seq;
  const void* du;     // bwd only
  void* out;          // u (fwd) or dx (bwd)
  float* dw;          // bwd only
  float* dbias;       // bwd only, nullable
  float* partial;     // bwd only: [B][tiles][D][5]
  // halos of a row cut out of a longer sequence (all nullable): the 3 inputs
  // (and document ids) before token 0, and for the backward the 3 inputs,
  // upstream gradients and ids after token L-1
  const void* x_prev;       // [B][D][3]
  const int32_t* seq_prev;  // [B][3]
  const void* x_next;       // [B][D][3]
  const void* du_next;      // [B][D][3]
  const int32_t* seq_next;  // [B][3]
  int B, D, L, silu;
  bool bf16, vec;
};

// Sets a kernel's dynamic shared-memory limit once per device. The attribute
// belongs to the (kernel, device) pair, so `done` holds one bit per device
// (devices 64 and up set it on every call); threads may race to set it, which
// is harmless since they set the same value.
template <typename K>
inline cudaError_t smem_attr(K kernel, int bytes, std::atomic<unsigned long long>* done) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  const unsigned long long bit = dev < 64 ? (1ull << dev) : 0ull;
  if (bit && (done->load(std::memory_order_acquire) & bit)) return cudaSuccess;
  e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  if (e == cudaSuccess && bit) done->fetch_or(bit, std::memory_order_release);
  return e;
}

cudaError_t launch_conv1d_fwd(const ConvArgs& a, cudaStream_t s);
// Fixed device scratch of the allocation-free conv1d backward.
constexpr size_t kConvBwdScratchFloats = size_t(1) << 20;  // 4 MiB per device
constexpr int kMaxScratchDevices = 64;
cudaError_t conv_bwd_scratch(float** ptr);
cudaError_t launch_conv1d_bwd(const ConvArgs& a, cudaStream_t s);
__host__ __device__ inline int conv_tiles(int L) { return (L + kConvTile - 1) / kConvTile; }
// The backward without document ids: kConvBwdTok tokens per thread (with
// them 8, as the forward); its dw / dbias partials are per (b, tile, d), at
// most conv_tiles(L) tiles, which sizes its scratch.
constexpr int kConvBwdTok = 16;

struct ScanArgs {
  // inputs
  const void* u;
  const void* delta;
  const void* z;
  const float* A;
  const float* Dskip;
  const float* delta_bias;
  const void* Bm;
  const void* Cm;
  const int32_t* seq;
  const float* h0;    // [B*D][N] state before token 0, nullable
  // fused conv (forward only): when xconv is set the forward reads x, computes
  // u = silu(conv(x)) itself and writes it to u (which is then an output)
  const void* xconv;
  const float* conv_w;
  const float* conv_b;
  int zoh;            // 1: zero-order-hold B_bar = (exp(dt A) - 1) / A B instead of dt B
  int softplus;
  // forward outputs
  void* out;
  float* final_state;
  // backward inputs / outputs
  const void* dout;
  void* du;
  void* ddelta;
  void* dz;
  float* dA;
  float* dB;
  float* dC;
  float* dD;
  float* ddelta_bias;
  float* dh0;         // [B*D][N] nullable
  const float* dhL;   // [B*D][N] nullable: dL/d(final state), the adjoint entering from the right
  int split_base;     // first split the backward summary kernel handles (1; 0 for a whole-row summary)
  // deterministic dB / dC: each CTA stores its row-group's sums here instead of
  // adding them atomically, [groups][2 (dB, dC)][dbc_bnl] fp32, and
  // launch_dbc_reduce sums the groups in order; nullptr: atomic adds
  float* dbc_part;
  size_t dbc_bnl;     // B * N * planes * L (planes: 2 for a complex A)
  // workspace pieces
  int* status;        // sticky device status word (0 = ok, 4 = a bounded wait timed out)
  float* ckpt;        // [B*D][nchunks * 16][kNMax] state entering each 16-token block
  void* ysave;        // [B*D][L] activation dtype: y before the gate (written by fwd when z)
  float* split_P;     // [B*D][P][Npad] per-split decay product (pass 1)
  float* split_H;     // [B*D][P][Npad] per-split end value from zero (pass 1)
  float* split_in;    // [B*D][P][Npad] carry into each split
  float* part_dA;     // [B*D][N]
  float* part_dD;     // [B*D]
  float* part_ddb;    // [B*D]
  // N = 16 path (scan16_fwd.cu / scan16_bwd.cu): checkpoints in the row-pair
  // layout of scan16.cuh, B / C packed per chunk by the forward
  bool fast16;
  float4* bcpack;     // [B][nchunks][2][16][64] float4
  int Dp;             // row pairs per batch entry, ceil(D / 2)
  int B, D, L, N;
  int Npad;           // N rounded up to even: state pairs; stride of ckpt / split arrays
  int nchunks, nsplits, chunks_per_split;
  bool bf16, vec;
};

cudaError_t launch_scan_fwd(const ScanArgs& a, cudaStream_t s);
// Whole-row summaries (nsplits must be 1): the forward writes (prod a, h_end
// from 0) and the backward (prod a, a_0 g_0 from a zero incoming adjoint)
// into split_P / split_H with row stride Npad.
cudaError_t launch_scan_fwd_summary(const ScanArgs& a, cudaStream_t s);
cudaError_t launch_scan_bwd_summary(const ScanArgs& a, cudaStream_t s);
// Repack [rows][Npad] summaries to [rows][N], zeroing the decay (and, with
// zero_value, the value) of rows whose token 0 starts a new document.
cudaError_t launch_summary_out(const float* sP, const float* sV, const int32_t* seq,
                               const int32_t* seq_prev, int L, float* decay, float* value,
                               int B, int D, int N, int Npad, bool zero_value, cudaStream_t s);
cudaError_t launch_state_carry(const float* decay, const float* value, int R, int r, bool reverse,
                               const float* init, const int32_t* seq_prev, const int32_t* seq,
                               int L, float* out, int B, int D, int N, cudaStream_t s);
// Complex diagonal A (A [D][N][2], Bm / Cm [B][N][2][L], states as (re, im)
// pairs, checkpoints [B*D][nchunks * 16][kNMax][2], part_dA [B*D][N][2]).
cudaError_t launch_cscan_fwd(const ScanArgs& a, cudaStream_t s);
cudaError_t launch_cscan_bwd(const ScanArgs& a, cudaStream_t s);

struct DecodeArgs {
  const void* x;
  void* conv_state;
  const float* conv_w;
  const float* conv_bias;
  const void* delta;
  const void* z;
  const void* Bm;
  const void* Cm;
  const float* A;
  const float* Dskip;
  const float* delta_bias;
  float* state;
  void* out;
  void* u_out;
  int B, D, N, softplus;
  bool bf16;
  bool vec;  // N == 16 with 16-byte aligned state / A and vector-aligned Bm / Cm
};

cudaError_t launch_decode_step(const DecodeArgs& a, cudaStream_t s);
cudaError_t launch_scan_bwd(const ScanArgs& a, cudaStream_t s);
// Rows per CTA of the backward kernels (CTAs along D = row groups of the
// deterministic dB / dC partials): scan16_bwd.cu (its smaller shape; the
// launch may take 22-row CTAs, i.e. fewer groups), scan_bwd.cu, cscan.cu.
constexpr int kBwdCtaRows16 = 12;
constexpr int kBwdCtaRows = 8;
constexpr int kCscanCtaRows = 8;
// Fixed-order sum of the row groups' dB / dC partials into dB and dC.
cudaError_t launch_dbc_reduce(const float* part, int groups, size_t bnl, float* dB, float* dC,
                              cudaStream_t s);
cudaError_t probe_ex2_rate(float* sink, size_t sink_floats, double* rate, cudaStream_t s);

// Mamba-2 SSD forward (ssd_fwd.cu): x [B][L][H][P], dt_raw [B][L][H], B / C
// [B][L][G][N] bf16; A, D, dt_bias [H] fp32; y [B][L][H][P] bf16; final
// state [B][H][P][N] fp32. P = 64, N = 128.
struct SsdArgs {
  const void* x;
  const void* dt_raw;
  const float* A;
  const void* Bm;
  const void* Cm;
  const float* D;
  const float* dt_bias;
  const int32_t* seq;
  void* y;
  float* final_state;
  int* status;
  float* chunk_states;  // [B][H][nc][N][P] fp32: the state entering each chunk
  int B, L, H, P, G, N;
  int softplus;
  // backward only
  const void* dy;
  void* dx;
  float* ddt_raw;
  float* dA;
  float* dB;
  float* dC;
  float* dD;
  float* ddt_bias;
};
cudaError_t launch_ssd_fwd(const SsdArgs& a, cudaStream_t s);
cudaError_t launch_ssd_bwd(const SsdArgs& a, cudaStream_t s);
cudaError_t launch_cu_seqlens_to_seq(const int32_t* cu, int n_docs, int L, int32_t* seq,
                                     cudaStream_t s);

// First failed device index check of one translation unit (debug.cuh):
// failures counts every failed check since the last reset.
struct DebugRecord {
  unsigned long long failures;
  long long offset, count, extent;
  int site, pad;
};
#ifdef SSM_DEBUG
// The kernel sources that carry checks, each reading its own record.
#define SSM_DEBUG_UNITS(X) \
  X(conv1d) X(scan16_fwd) X(scan16_bwd) X(scan_fwd) X(scan_bwd) X(cscan) X(decode) X(ssd_fwd) X(ssd_bwd) X(carry) X(probe) X(abi)
#define SSM_DEBUG_DECL(name) cudaError_t debug_take_##name(DebugRecord* out, bool reset);
SSM_DEBUG_UNITS(SSM_DEBUG_DECL)
#undef SSM_DEBUG_DECL
cudaError_t launch_debug_selftest(float* buf, long long n, cudaStream_t s);
#endif

}  // namespace ssm
