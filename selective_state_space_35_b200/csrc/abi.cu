// C ABI entry points (include/ssmscan.h): argument validation, workspace
// layout, launch-shape choice, error reporting. No allocation happens here.
#include <cuda_runtime.h>

#include <cstdarg>
#include <cstdio>
#include <cstdlib>
#include <cstring>

#include "../../include/ssmscan.h"
#include "internal.h"
#include "scan16.cuh"

namespace {

thread_local char g_err[512] = "";

ssm_status_t fail(ssm_status_t st, const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_err, sizeof(g_err), fmt, ap);
  va_end(ap);
  return st;
}

ssm_status_t ok() {
  g_err[0] = '\0';
  return SSM_OK;
}

// Host-side fault injection: SSM_INJECT_FAIL="ssm_scan_fwd,ssm_conv1d_bwd"
// makes the named calls fail before any launch. Never touches the device.
bool injected(const char* name) {
  const char* e = getenv("SSM_INJECT_FAIL");
  if (!e || !*e) return false;
  const size_t n = strlen(name);
  for (const char* p = strstr(e, name); p; p = strstr(p + 1, name)) {
    const bool start = p == e || p[-1] == ',';
    const bool end = p[n] == '\0' || p[n] == ',';
    if (start && end) return true;
  }
  return false;
}

bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

size_t elem_size(ssm_dtype_t dt) { return dt == SSM_DTYPE_BF16 ? 2 : 4; }

ssm_status_t cuda_status(cudaError_t e, const char* what) {
  if (e == cudaSuccess) return ok();
  return fail(SSM_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

constexpr size_t kAlign = 256;
size_t up(size_t x) { return (x + kAlign - 1) / kAlign * kAlign; }

int sm_count() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 148;
  int n = 0;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
    return 148;
  return n;
}

struct ScanPlan {
  int nchunks, nsplits, chunks_per_split;
  bool fast16;  // the N = 16 kernels (scan16_*.cu) and their checkpoint layout
  size_t off_seq, off_ckpt, off_y, off_sP, off_sH, off_sIn, off_pA, off_pD, off_pB, off_sum,
      off_pack, total;
};

ssm_status_t check_params(const ssm_scan_params* p) {
  if (!p) return fail(SSM_ERR_INVALID_ARG, "params is NULL");
  if (p->struct_size != sizeof(ssm_scan_params))
    return fail(SSM_ERR_INVALID_ARG, "params.struct_size %zu != %zu", p->struct_size,
                sizeof(ssm_scan_params));
  if (p->B < 1 || p->D < 1 || p->L < 1 || p->N < 1)
    return fail(SSM_ERR_INVALID_ARG, "sizes must be >= 1 (B=%d D=%d L=%d N=%d)", p->B, p->D,
                p->L, p->N);
  if (p->N > ssm::kNMax) return fail(SSM_ERR_UNSUPPORTED, "N=%d > %d", p->N, ssm::kNMax);
  if (p->B > 65535) return fail(SSM_ERR_UNSUPPORTED, "B=%d > 65535", p->B);
  if (p->dtype != SSM_DTYPE_F32 && p->dtype != SSM_DTYPE_BF16)
    return fail(SSM_ERR_INVALID_ARG, "unknown dtype %d", (int)p->dtype);
  if (p->n_splits < 0) return fail(SSM_ERR_INVALID_ARG, "n_splits=%d < 0", p->n_splits);
  if (p->discretization != 0 && p->discretization != 1)
    return fail(SSM_ERR_INVALID_ARG, "discretization=%d (0: dt B, 1: zero-order hold)",
                p->discretization);
  if (p->state_complex != 0 && p->state_complex != 1)
    return fail(SSM_ERR_INVALID_ARG, "state_complex=%d (0: real A, 1: complex A)",
                p->state_complex);
  if (p->state_complex && p->discretization != 0)
    return fail(SSM_ERR_UNSUPPORTED, "complex A supports discretization 0 (dt B) only");
  if (p->state_complex && p->n_splits > 1)
    return fail(SSM_ERR_UNSUPPORTED, "complex A runs each row on one CTA (n_splits=%d)",
                p->n_splits);
  if (p->seq_idx && p->cu_seqlens)
    return fail(SSM_ERR_INVALID_ARG, "seq_idx and cu_seqlens are mutually exclusive");
  if (p->cu_seqlens && p->B != 1)
    return fail(SSM_ERR_INVALID_ARG, "cu_seqlens requires B == 1 (B=%d)", p->B);
  if (p->cu_seqlens && p->n_docs < 1)
    return fail(SSM_ERR_INVALID_ARG, "cu_seqlens needs n_docs >= 1 (n_docs=%d)", p->n_docs);
  return ok();
}

ScanPlan plan_scan(const ssm_scan_params* p) {
  ScanPlan s{};
  s.nchunks = (p->L + ssm::kChunk - 1) / ssm::kChunk;
  int P = p->state_complex ? 1 : p->n_splits;
  if (P == 0) {
    // enough warps to keep every SM busy without splitting? (a split costs a
    // second pass over all but the last range)
    const long target = (long)sm_count() * 8;
    const long rows = (long)p->B * p->D;
    P = rows >= target ? 1 : (int)((target + rows - 1) / rows);
  }
  if (P > s.nchunks) P = s.nchunks;
  if (P > 65535) P = 65535;
  if (P < 1) P = 1;
  s.chunks_per_split = (s.nchunks + P - 1) / P;
  s.nsplits = (s.nchunks + s.chunks_per_split - 1) / s.chunks_per_split;
  // The N = 16 kernels serve the common case: one CTA range per row, dt B
  // discretisation, real A, L a multiple of 8 and 16-byte aligned inputs.
  // The forward and the backward read the same inputs, so they agree (out,
  // written by the forward only, does not take part).
  s.fast16 = p->N == 16 && !p->state_complex && p->discretization == 0 && s.nsplits == 1 &&
             p->L % 8 == 0 && aligned(p->u, 16) && aligned(p->delta, 16) && aligned(p->z, 16) &&
             aligned(p->Bm, 16) && aligned(p->Cm, 16) && aligned(p->seq_idx, 16);
  const size_t rows = (size_t)p->B * p->D;
  size_t off = up(sizeof(int));  // status word first
  s.off_seq = off;
  off += p->cu_seqlens ? up((size_t)p->B * p->L * sizeof(int32_t)) : 0;
  s.off_ckpt = off;
  const size_t npad = (size_t)((p->N + 1) & ~1);
  // one state checkpoint per 16-token block, kNMax wide (complex: (re, im) pairs);
  // N = 16 kernels: one per 8-token segment, per row pair (scan16.cuh)
  const size_t cw = p->state_complex ? 2 : 1;
  if (s.fast16)
    off += up((size_t)p->B * ((p->D + 1) / 2) * s.nchunks * 16 * 64 * sizeof(float));
  else
    off += up(rows * s.nchunks * (ssm::kChunk / 16) * ssm::kNMax * cw * sizeof(float));
  s.off_y = off;
  off += p->z ? up(rows * (size_t)p->L * elem_size(p->dtype)) : 0;
  const size_t per_split = up(rows * s.nsplits * npad * sizeof(float));
  s.off_sP = off;
  off += s.nsplits > 1 ? per_split : 0;
  s.off_sH = off;
  off += s.nsplits > 1 ? per_split : 0;
  s.off_sIn = off;
  off += s.nsplits > 1 ? per_split : 0;
  s.off_pA = off;
  off += per_split * cw;
  s.off_pD = off;
  off += up(rows * s.nsplits * sizeof(float));
  s.off_pB = off;
  off += up(rows * s.nsplits * sizeof(float));
  // whole-row summaries (ssm_scan_fwd_summary / ssm_scan_bwd_summary): two [rows][npad]
  s.off_sum = off;
  off += 2 * up(rows * npad * sizeof(float));
  // N = 16 forward: B / C packed per chunk in its lane layout (32 KB per chunk)
  s.off_pack = off;
  off += s.fast16 ? up((size_t)p->B * s.nchunks * 2 * 16 * 256 * sizeof(float)) : 0;
  s.total = off;
  return s;
}

ssm_status_t build_args(const ssm_scan_params* p, const ScanPlan& pl, ssm::ScanArgs* a) {
  char* ws = static_cast<char*>(p->workspace);
  memset(a, 0, sizeof(*a));
  a->u = p->u;
  a->delta = p->delta;
  a->z = p->z;
  a->A = p->A;
  a->Dskip = p->Dskip;
  a->delta_bias = p->delta_bias;
  a->Bm = p->Bm;
  a->Cm = p->Cm;
  a->seq = p->cu_seqlens ? reinterpret_cast<int32_t*>(ws + pl.off_seq) : p->seq_idx;
  a->h0 = p->initial_state;
  a->zoh = p->discretization == 1 ? 1 : 0;
  a->softplus = p->delta_softplus ? 1 : 0;
  a->out = p->out;
  a->final_state = p->final_state;
  a->status = reinterpret_cast<int*>(ws);
  a->ckpt = reinterpret_cast<float*>(ws + pl.off_ckpt);
  a->ysave = p->z ? static_cast<void*>(ws + pl.off_y) : nullptr;
  a->split_P = pl.nsplits > 1 ? reinterpret_cast<float*>(ws + pl.off_sP) : nullptr;
  a->split_H = pl.nsplits > 1 ? reinterpret_cast<float*>(ws + pl.off_sH) : nullptr;
  a->split_in = pl.nsplits > 1 ? reinterpret_cast<float*>(ws + pl.off_sIn) : nullptr;
  a->part_dA = reinterpret_cast<float*>(ws + pl.off_pA);
  a->part_dD = reinterpret_cast<float*>(ws + pl.off_pD);
  a->part_ddb = reinterpret_cast<float*>(ws + pl.off_pB);
  a->B = p->B;
  a->D = p->D;
  a->L = p->L;
  a->N = p->N;
  a->Npad = (p->N + 1) & ~1;
  a->split_base = 1;
  a->fast16 = pl.fast16;
  a->bcpack = pl.fast16 ? reinterpret_cast<float4*>(ws + pl.off_pack) : nullptr;
  a->Dp = (p->D + 1) / 2;
  a->nchunks = pl.nchunks;
  a->nsplits = pl.nsplits;
  a->chunks_per_split = pl.chunks_per_split;
  a->bf16 = p->dtype == SSM_DTYPE_BF16;
  return ok();
}

ssm_status_t check_scan_buffers(const ssm_scan_params* p, const ScanPlan& pl) {
  if (!p->u || !p->delta || !p->A || !p->Bm || !p->Cm || !p->out)
    return fail(SSM_ERR_INVALID_ARG, "u, delta, A, Bm, Cm and out must be non-NULL");
  if (!p->workspace) return fail(SSM_ERR_INVALID_ARG, "workspace is NULL");
  if (!aligned(p->workspace, kAlign))
    return fail(SSM_ERR_INVALID_ARG, "workspace must be 256-byte aligned");
  if (p->workspace_bytes < pl.total)
    return fail(SSM_ERR_INVALID_ARG, "workspace_bytes %zu < required %zu", p->workspace_bytes,
                pl.total);
  const size_t es = elem_size(p->dtype);
  const void* acts[] = {p->u, p->delta, p->z, p->Bm, p->Cm, p->out};
  for (const void* q : acts)
    if (q && !aligned(q, es)) return fail(SSM_ERR_INVALID_ARG, "activation pointer misaligned");
  const void* f32s[] = {p->A, p->Dskip, p->delta_bias, p->final_state, p->seq_idx, p->cu_seqlens,
                        p->initial_state};
  for (const void* q : f32s)
    if (q && !aligned(q, 4)) return fail(SSM_ERR_INVALID_ARG, "fp32/int32 pointer misaligned");
  if (p->state_complex && (!aligned(p->A, 8) || !aligned(p->initial_state, 8) ||
                           !aligned(p->final_state, 8)))
    return fail(SSM_ERR_INVALID_ARG, "complex A: A and the states must be 8-byte aligned");
  return ok();
}

bool vec_ok(int L, std::initializer_list<const void*> ptrs) {
  if (L % 8) return false;
  for (const void* q : ptrs)
    if (q && !aligned(q, 16)) return false;
  return true;
}

// ssm_scan_fwd, or with x set the fused conv + scan forward that writes u.
ssm_status_t scan_fwd_impl(const ssm_scan_params* p, const void* x, const float* conv_w,
                           const float* conv_bias, ssm_stream_t stream) {
  ssm_status_t st = check_params(p);
  if (st != SSM_OK) return st;
  const ScanPlan pl = plan_scan(p);
  st = check_scan_buffers(p, pl);
  if (st != SSM_OK) return st;
  if (x && p->state_complex)
    return fail(SSM_ERR_UNSUPPORTED, "ssm_conv1d_scan_fwd: complex A is not fused with the conv");
  if (x) {
    if (x == p->u) return fail(SSM_ERR_INVALID_ARG, "u (written) may not alias x");
    if (!aligned(x, elem_size(p->dtype)) || !aligned(conv_w, 4) ||
        (conv_bias && !aligned(conv_bias, 4)))
      return fail(SSM_ERR_INVALID_ARG, "x, conv_w or conv_bias misaligned");
  }
  ssm::ScanArgs a;
  build_args(p, pl, &a);
  a.xconv = x;
  a.conv_w = conv_w;
  a.conv_b = conv_bias;
  a.vec = vec_ok(p->L, {p->u, p->delta, p->z, p->Bm, p->Cm, p->out, a.seq, x});
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  cudaError_t e0 = cudaMemsetAsync(a.status, 0, sizeof(int), s);  // fresh status for this fwd/bwd
  if (e0 != cudaSuccess) return cuda_status(e0, "scan forward status reset");
  if (p->cu_seqlens) {
    cudaError_t e = ssm::launch_cu_seqlens_to_seq(p->cu_seqlens, p->n_docs, p->L,
                                                  const_cast<int32_t*>(a.seq), s);
    if (e != cudaSuccess) return cuda_status(e, "cu_seqlens conversion");
  }
  if (p->state_complex) return cuda_status(ssm::launch_cscan_fwd(a, s), "ssm_scan_fwd launch");
  const char* what = x ? "ssm_conv1d_scan_fwd launch" : "ssm_scan_fwd launch";
  if (a.fast16) return cuda_status(ssm::launch_scan16_fwd(a, s), what);
  return cuda_status(ssm::launch_scan_fwd(a, s), what);
}

}  // namespace

extern "C" {

const char* ssm_last_error(void) { return g_err; }

int ssm_abi_version(void) { return SSM_ABI_VERSION; }

ssm_status_t ssm_conv1d_fwd(const void* x, const float* w, const float* bias,
                            const int32_t* seq_idx, void* u, int B, int D, int L, int W,
                            ssm_dtype_t dtype, int silu, ssm_stream_t stream) {
  if (injected("ssm_conv1d_fwd")) return fail(SSM_ERR_INJECTED, "ssm_conv1d_fwd: injected failure");
  return ssm_conv1d_fwd_ctx(x, w, bias, seq_idx, nullptr, nullptr, u, B, D, L, W, dtype, silu,
                            stream);
}

ssm_status_t ssm_conv1d_fwd_ctx(const void* x, const float* w, const float* bias,
                                const int32_t* seq_idx, const void* x_prev,
                                const int32_t* seq_prev, void* u, int B, int D, int L, int W,
                                ssm_dtype_t dtype, int silu, ssm_stream_t stream) {
  if (injected("ssm_conv1d_fwd_ctx"))
    return fail(SSM_ERR_INJECTED, "ssm_conv1d_fwd_ctx: injected failure");
  if (!x || !w || !u) return fail(SSM_ERR_INVALID_ARG, "x, w and u must be non-NULL");
  if (seq_idx && x_prev && !seq_prev)
    return fail(SSM_ERR_INVALID_ARG, "seq_prev is required with seq_idx and x_prev");
  if (B < 1 || D < 1 || L < 1) return fail(SSM_ERR_INVALID_ARG, "sizes must be >= 1");
  if (W != 4) return fail(SSM_ERR_UNSUPPORTED, "conv width W=%d (only 4)", W);
  if (B > 65535 || D > 65535) return fail(SSM_ERR_UNSUPPORTED, "B and D must be <= 65535");
  if (dtype != SSM_DTYPE_F32 && dtype != SSM_DTYPE_BF16)
    return fail(SSM_ERR_INVALID_ARG, "unknown dtype %d", (int)dtype);
  if (x == u) return fail(SSM_ERR_INVALID_ARG, "u may not alias x");
  const size_t es = elem_size(dtype);
  if (!aligned(x, es) || !aligned(u, es) || !aligned(w, 4) || (bias && !aligned(bias, 4)) ||
      (seq_idx && !aligned(seq_idx, 4)) || (x_prev && !aligned(x_prev, es)) ||
      (seq_prev && !aligned(seq_prev, 4)))
    return fail(SSM_ERR_INVALID_ARG, "misaligned pointer");
  ssm::ConvArgs a{};
  a.x = x; a.w = w; a.bias = bias; a.seq = seq_idx; a.out = u;
  a.x_prev = x_prev; a.seq_prev = seq_idx ? seq_prev : nullptr;
  a.B = B; a.D = D; a.L = L; a.silu = silu ? 1 : 0;
  a.bf16 = dtype == SSM_DTYPE_BF16;
  a.vec = vec_ok(L, {x, u, seq_idx});
  return cuda_status(ssm::launch_conv1d_fwd(a, reinterpret_cast<cudaStream_t>(stream)),
                     x_prev ? "ssm_conv1d_fwd_ctx launch" : "ssm_conv1d_fwd launch");
}

ssm_status_t ssm_conv1d_bwd_workspace_size(int B, int D, int L, int W, size_t* bytes) {
  if (!bytes) return fail(SSM_ERR_INVALID_ARG, "bytes is NULL");
  if (B < 1 || D < 1 || L < 1) return fail(SSM_ERR_INVALID_ARG, "sizes must be >= 1");
  if (W != 4) return fail(SSM_ERR_UNSUPPORTED, "conv width W=%d (only 4)", W);
  *bytes = up((size_t)B * ssm::conv_tiles(L) * D * 5 * sizeof(float));
  return ok();
}

ssm_status_t ssm_conv1d_bwd(const void* x, const float* w, const float* bias,
                            const int32_t* seq_idx, const void* du, void* dx, float* dw,
                            float* dbias, int B, int D, int L, int W, ssm_dtype_t dtype,
                            int silu, void* workspace, size_t workspace_bytes,
                            ssm_stream_t stream) {
  if (injected("ssm_conv1d_bwd")) return fail(SSM_ERR_INJECTED, "ssm_conv1d_bwd: injected failure");
  return ssm_conv1d_bwd_ctx(x, w, bias, seq_idx, nullptr, nullptr, nullptr, nullptr, nullptr, du,
                            dx, dw, dbias, B, D, L, W, dtype, silu, workspace, workspace_bytes,
                            stream);
}

ssm_status_t ssm_conv1d_bwd_ctx(const void* x, const float* w, const float* bias,
                                const int32_t* seq_idx, const void* x_prev,
                                const int32_t* seq_prev, const void* x_next,
                                const void* du_next, const int32_t* seq_next, const void* du,
                                void* dx, float* dw, float* dbias, int B, int D, int L, int W,
                                ssm_dtype_t dtype, int silu, void* workspace,
                                size_t workspace_bytes, ssm_stream_t stream) {
  if (injected("ssm_conv1d_bwd_ctx"))
    return fail(SSM_ERR_INJECTED, "ssm_conv1d_bwd_ctx: injected failure");
  if (seq_idx && x_prev && !seq_prev)
    return fail(SSM_ERR_INVALID_ARG, "seq_prev is required with seq_idx and x_prev");
  if ((x_next == nullptr) != (du_next == nullptr))
    return fail(SSM_ERR_INVALID_ARG, "x_next and du_next come together");
  if (seq_idx && x_next && !seq_next)
    return fail(SSM_ERR_INVALID_ARG, "seq_next is required with seq_idx and x_next");
  if (!x || !w || !du || !dx || !dw)
    return fail(SSM_ERR_INVALID_ARG, "x, w, du, dx and dw must be non-NULL");
  size_t need = 0;
  ssm_status_t st = ssm_conv1d_bwd_workspace_size(B, D, L, W, &need);
  if (st != SSM_OK) return st;
  if (B > 65535 || D > 65535) return fail(SSM_ERR_UNSUPPORTED, "B and D must be <= 65535");
  if (dtype != SSM_DTYPE_F32 && dtype != SSM_DTYPE_BF16)
    return fail(SSM_ERR_INVALID_ARG, "unknown dtype %d", (int)dtype);
  if (!workspace || workspace_bytes < need)
    return fail(SSM_ERR_INVALID_ARG, "workspace too small (%zu < %zu)", workspace_bytes, need);
  if (!aligned(workspace, 16)) return fail(SSM_ERR_INVALID_ARG, "workspace misaligned");
  if (dx == x || dx == du) return fail(SSM_ERR_INVALID_ARG, "dx may not alias x or du");
  const size_t es = elem_size(dtype);
  if (!aligned(x, es) || !aligned(du, es) || !aligned(dx, es) || !aligned(w, 4) ||
      !aligned(dw, 4) || (bias && !aligned(bias, 4)) || (dbias && !aligned(dbias, 4)) ||
      (seq_idx && !aligned(seq_idx, 4)) || (x_prev && !aligned(x_prev, es)) ||
      (x_next && !aligned(x_next, es)) || (du_next && !aligned(du_next, es)) ||
      (seq_prev && !aligned(seq_prev, 4)) || (seq_next && !aligned(seq_next, 4)))
    return fail(SSM_ERR_INVALID_ARG, "misaligned pointer");
  ssm::ConvArgs a{};
  a.x = x; a.w = w; a.bias = bias; a.seq = seq_idx; a.du = du; a.out = dx;
  a.dw = dw; a.dbias = dbias; a.partial = static_cast<float*>(workspace);
  a.x_prev = x_prev; a.seq_prev = seq_idx ? seq_prev : nullptr;
  a.x_next = x_next; a.du_next = du_next; a.seq_next = seq_idx ? seq_next : nullptr;
  a.B = B; a.D = D; a.L = L; a.silu = silu ? 1 : 0;
  a.bf16 = dtype == SSM_DTYPE_BF16;
  a.vec = vec_ok(L, {x, du, dx, seq_idx});
  return cuda_status(ssm::launch_conv1d_bwd(a, reinterpret_cast<cudaStream_t>(stream)),
                     (x_prev || x_next) ? "ssm_conv1d_bwd_ctx launch" : "ssm_conv1d_bwd launch");
}

ssm_status_t ssm_conv1d_bwd_noalloc(const void* x, const float* w, const float* bias,
                                    const int32_t* seq_idx, const void* du, void* dx, float* dw,
                                    float* dbias, int B, int D, int L, int W, ssm_dtype_t dtype,
                                    int silu, ssm_stream_t stream) {
  if (injected("ssm_conv1d_bwd_noalloc"))
    return fail(SSM_ERR_INJECTED, "ssm_conv1d_bwd_noalloc: injected failure");
  if (!x || !w || !du || !dx || !dw)
    return fail(SSM_ERR_INVALID_ARG, "x, w, du, dx and dw must be non-NULL");
  size_t need = 0;
  ssm_status_t st = ssm_conv1d_bwd_workspace_size(B, D, L, W, &need);
  if (st != SSM_OK) return st;
  const size_t floats = (size_t)B * ssm::conv_tiles(L) * D * 5;
  if (floats > ssm::kConvBwdScratchFloats)
    return fail(SSM_ERR_UNSUPPORTED,
                "ssm_conv1d_bwd_noalloc: B * ceil(L / %d) * D * 5 = %zu partial sums exceed the fixed "
                "scratch of %zu floats; use ssm_conv1d_bwd with a workspace",
                ssm::kConvTile, floats, ssm::kConvBwdScratchFloats);
  if (B > 65535 || D > 65535) return fail(SSM_ERR_UNSUPPORTED, "B and D must be <= 65535");
  if (dtype != SSM_DTYPE_F32 && dtype != SSM_DTYPE_BF16)
    return fail(SSM_ERR_INVALID_ARG, "unknown dtype %d", (int)dtype);
  if (dx == x || dx == du) return fail(SSM_ERR_INVALID_ARG, "dx may not alias x or du");
  const size_t es = elem_size(dtype);
  if (!aligned(x, es) || !aligned(du, es) || !aligned(dx, es) || !aligned(w, 4) ||
      !aligned(dw, 4) || (bias && !aligned(bias, 4)) || (dbias && !aligned(dbias, 4)) ||
      (seq_idx && !aligned(seq_idx, 4)))
    return fail(SSM_ERR_INVALID_ARG, "misaligned pointer");
  float* scratch = nullptr;
  cudaError_t e = ssm::conv_bwd_scratch(&scratch);
  if (e != cudaSuccess) return cuda_status(e, "ssm_conv1d_bwd_noalloc scratch address");
  ssm::ConvArgs a{};
  a.x = x; a.w = w; a.bias = bias; a.seq = seq_idx; a.du = du; a.out = dx;
  a.dw = dw; a.dbias = dbias; a.partial = scratch;
  a.B = B; a.D = D; a.L = L; a.silu = silu ? 1 : 0;
  a.bf16 = dtype == SSM_DTYPE_BF16;
  a.vec = vec_ok(L, {x, du, dx, seq_idx});
  return cuda_status(ssm::launch_conv1d_bwd(a, reinterpret_cast<cudaStream_t>(stream)),
                     "ssm_conv1d_bwd_noalloc launch");
}

ssm_status_t ssm_scan_workspace_size(const ssm_scan_params* p, size_t* bytes) {
  if (!bytes) return fail(SSM_ERR_INVALID_ARG, "bytes is NULL");
  ssm_status_t st = check_params(p);
  if (st != SSM_OK) return st;
  *bytes = plan_scan(p).total;
  return ok();
}

ssm_status_t ssm_scan_fwd(const ssm_scan_params* p, ssm_stream_t stream) {
  if (injected("ssm_scan_fwd")) return fail(SSM_ERR_INJECTED, "ssm_scan_fwd: injected failure");
  return scan_fwd_impl(p, nullptr, nullptr, nullptr, stream);
}

ssm_status_t ssm_conv1d_scan_fwd(const ssm_scan_params* p, const void* x, const float* conv_w,
                                 const float* conv_bias, ssm_stream_t stream) {
  if (injected("ssm_conv1d_scan_fwd"))
    return fail(SSM_ERR_INJECTED, "ssm_conv1d_scan_fwd: injected failure");
  if (!x || !conv_w) return fail(SSM_ERR_INVALID_ARG, "x and conv_w must be non-NULL");
  return scan_fwd_impl(p, x, conv_w, conv_bias, stream);
}

// Row groups of the backward kernel the plan selects (at most: the N = 16
// kernels may take larger groups), and the bytes of the deterministic dB / dC
// partials.
static size_t dbc_bnl(const ssm_scan_params* p) {
  return (size_t)p->B * p->N * (p->state_complex ? 2 : 1) * p->L;
}
static int dbc_groups(const ssm_scan_params* p, const ScanPlan& pl) {
  const int rows = pl.fast16 ? ssm::kBwdCtaRows16
                             : (p->state_complex ? ssm::kCscanCtaRows : ssm::kBwdCtaRows);
  return (p->D + rows - 1) / rows;
}

static ssm_status_t check_grads(const ssm_scan_grads* g) {
  if (!g) return fail(SSM_ERR_INVALID_ARG, "grads is NULL");
  if (g->struct_size != sizeof(ssm_scan_grads))
    return fail(SSM_ERR_INVALID_ARG, "grads.struct_size %zu != %zu", g->struct_size,
                sizeof(ssm_scan_grads));
  if (g->deterministic != 0 && g->deterministic != 1)
    return fail(SSM_ERR_INVALID_ARG, "deterministic=%d (0 or 1)", g->deterministic);
  return ok();
}

ssm_status_t ssm_scan_bwd_workspace_size(const ssm_scan_params* p, const ssm_scan_grads* g,
                                         size_t* bytes) {
  if (!bytes) return fail(SSM_ERR_INVALID_ARG, "bytes is NULL");
  ssm_status_t st = check_params(p);
  if (st != SSM_OK) return st;
  st = check_grads(g);
  if (st != SSM_OK) return st;
  *bytes = g->deterministic
               ? up((size_t)dbc_groups(p, plan_scan(p)) * 2 * dbc_bnl(p) * sizeof(float))
               : 0;
  return ok();
}

ssm_status_t ssm_scan_bwd(const ssm_scan_params* p, const ssm_scan_grads* g,
                          ssm_stream_t stream) {
  if (injected("ssm_scan_bwd")) return fail(SSM_ERR_INJECTED, "ssm_scan_bwd: injected failure");
  ssm_status_t st = check_params(p);
  if (st != SSM_OK) return st;
  st = check_grads(g);
  if (st != SSM_OK) return st;
  const ScanPlan pl = plan_scan(p);
  size_t det_need = 0;
  if (g->deterministic) {
    det_need = up((size_t)dbc_groups(p, pl) * 2 * dbc_bnl(p) * sizeof(float));
    if (!g->workspace || g->workspace_bytes < det_need)
      return fail(SSM_ERR_INVALID_ARG,
                  "deterministic backward: grads.workspace of %zu bytes needed (have %zu)", det_need,
                  g->workspace ? g->workspace_bytes : (size_t)0);
    if (!aligned(g->workspace, kAlign))
      return fail(SSM_ERR_INVALID_ARG, "grads.workspace must be 256-byte aligned");
  }
  st = check_scan_buffers(p, pl);
  if (st != SSM_OK) return st;
  if (!g->dout || !g->du || !g->ddelta || !g->dA || !g->dB || !g->dC)
    return fail(SSM_ERR_INVALID_ARG, "dout, du, ddelta, dA, dB and dC must be non-NULL");
  if (p->z && !g->dz) return fail(SSM_ERR_INVALID_ARG, "dz must be non-NULL when z is given");
  const size_t es = elem_size(p->dtype);
  const void* acts[] = {g->dout, g->du, g->ddelta, g->dz};
  for (const void* q : acts)
    if (q && !aligned(q, es)) return fail(SSM_ERR_INVALID_ARG, "gradient pointer misaligned");
  const void* f32s[] = {g->dA, g->dB, g->dC, g->dD, g->ddelta_bias, g->dinitial_state};
  for (const void* q : f32s)
    if (q && !aligned(q, 4)) return fail(SSM_ERR_INVALID_ARG, "fp32 gradient pointer misaligned");
  if (g->dfinal_state && !aligned(g->dfinal_state, 4))
    return fail(SSM_ERR_INVALID_ARG, "dfinal_state misaligned");
  if (p->state_complex && (!aligned(g->dA, 8) || !aligned(g->dinitial_state, 8) ||
                           !aligned(g->dfinal_state, 8)))
    return fail(SSM_ERR_INVALID_ARG, "complex A: dA and dinitial_state must be 8-byte aligned");
  ssm::ScanArgs a;
  build_args(p, pl, &a);
  a.dout = g->dout;
  a.du = g->du;
  a.ddelta = g->ddelta;
  a.dz = p->z ? g->dz : nullptr;
  a.dA = g->dA;
  a.dB = g->dB;
  a.dC = g->dC;
  a.dD = g->dD;
  a.ddelta_bias = g->ddelta_bias;
  a.dh0 = g->dinitial_state;
  a.dhL = g->dfinal_state;
  // dB and dC take 16-byte vector atomics on the vector path
  a.vec = vec_ok(p->L, {p->u, p->delta, p->z, p->Bm, p->Cm, g->dout, g->du, g->ddelta, a.dz, a.seq,
                        g->dB, g->dC});
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (p->cu_seqlens) {
    cudaError_t e = ssm::launch_cu_seqlens_to_seq(p->cu_seqlens, p->n_docs, p->L,
                                                  const_cast<int32_t*>(a.seq), s);
    if (e != cudaSuccess) return cuda_status(e, "cu_seqlens conversion");
  }
  cudaError_t e = cudaSuccess;
  if (g->deterministic) {
    // every (group, dB / dC, element) of the partials is stored by the kernel
    a.dbc_part = static_cast<float*>(g->workspace);
    a.dbc_bnl = dbc_bnl(p);
  } else {
    const size_t bc = dbc_bnl(p) * sizeof(float);
    e = cudaMemsetAsync(g->dB, 0, bc, s);
    if (e == cudaSuccess) e = cudaMemsetAsync(g->dC, 0, bc, s);
    if (e != cudaSuccess) return cuda_status(e, "ssm_scan_bwd memset");
  }
  if (p->state_complex) e = ssm::launch_cscan_bwd(a, s);
  else if (a.fast16) e = ssm::launch_scan16_bwd(a, s);
  else e = ssm::launch_scan_bwd(a, s);
  if (e == cudaSuccess && g->deterministic) {
    // the N = 16 kernels may have used larger row groups than the workspace bound
    const int groups =
        a.fast16 ? (p->D + ssm::scan16_bwd_rows(a) - 1) / ssm::scan16_bwd_rows(a) : dbc_groups(p, pl);
    e = ssm::launch_dbc_reduce(a.dbc_part, groups, a.dbc_bnl, g->dB, g->dC, s);
  }
  return cuda_status(e, "ssm_scan_bwd launch");
}

// Shared part of the two whole-row summaries: validation, args with one
// split over the whole row, scratch in the workspace, cu_seqlens ids.
static ssm_status_t summary_setup(const ssm_scan_params* p, const int32_t* seq_prev,
                                  const float* decay, const float* value, ssm::ScanArgs* a,
                                  cudaStream_t s) {
  ssm_status_t st = check_params(p);
  if (st != SSM_OK) return st;
  if (p->state_complex) return fail(SSM_ERR_UNSUPPORTED, "summaries are for a real A");
  if (!decay || !value) return fail(SSM_ERR_INVALID_ARG, "summary outputs must be non-NULL");
  if (!p->delta || !p->A) return fail(SSM_ERR_INVALID_ARG, "delta and A must be non-NULL");
  if (!p->workspace) return fail(SSM_ERR_INVALID_ARG, "workspace is NULL");
  if (!aligned(p->workspace, kAlign))
    return fail(SSM_ERR_INVALID_ARG, "workspace must be 256-byte aligned");
  const ScanPlan pl = plan_scan(p);
  if (p->workspace_bytes < pl.total)
    return fail(SSM_ERR_INVALID_ARG, "workspace_bytes %zu < required %zu", p->workspace_bytes,
                pl.total);
  const size_t es = elem_size(p->dtype);
  const void* acts[] = {p->u, p->delta, p->z, p->Bm, p->Cm};
  for (const void* q : acts)
    if (q && !aligned(q, es)) return fail(SSM_ERR_INVALID_ARG, "activation pointer misaligned");
  const void* f32s[] = {p->A, p->delta_bias, p->seq_idx, p->cu_seqlens, seq_prev, decay, value};
  for (const void* q : f32s)
    if (q && !aligned(q, 4)) return fail(SSM_ERR_INVALID_ARG, "fp32/int32 pointer misaligned");
  build_args(p, pl, a);
  a->nsplits = 1;
  a->chunks_per_split = a->nchunks;
  a->split_base = 0;
  char* ws = static_cast<char*>(p->workspace);
  const size_t rows = (size_t)p->B * p->D;
  a->split_P = reinterpret_cast<float*>(ws + pl.off_sum);
  a->split_H = reinterpret_cast<float*>(ws + pl.off_sum + up(rows * a->Npad * sizeof(float)));
  return ok();
}

// First launches of a summary (after every argument check): a fresh status
// word and the document ids from cu_seqlens.
static ssm_status_t summary_prep(const ssm_scan_params* p, const ssm::ScanArgs& a, cudaStream_t s) {
  cudaError_t e = cudaMemsetAsync(a.status, 0, sizeof(int), s);
  if (e != cudaSuccess) return cuda_status(e, "summary status reset");
  if (p->cu_seqlens) {
    e = ssm::launch_cu_seqlens_to_seq(p->cu_seqlens, p->n_docs, p->L, const_cast<int32_t*>(a.seq), s);
    if (e != cudaSuccess) return cuda_status(e, "cu_seqlens conversion");
  }
  return ok();
}

ssm_status_t ssm_scan_fwd_summary(const ssm_scan_params* p, const int32_t* seq_prev,
                                  float* decay, float* state_end, ssm_stream_t stream) {
  if (injected("ssm_scan_fwd_summary"))
    return fail(SSM_ERR_INJECTED, "ssm_scan_fwd_summary: injected failure");
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  ssm::ScanArgs a;
  ssm_status_t st = summary_setup(p, seq_prev, decay, state_end, &a, s);
  if (st != SSM_OK) return st;
  if (!p->u || !p->Bm) return fail(SSM_ERR_INVALID_ARG, "u and Bm must be non-NULL");
  a.h0 = nullptr;
  a.vec = vec_ok(p->L, {p->u, p->delta, p->Bm, a.seq});
  st = summary_prep(p, a, s);
  if (st != SSM_OK) return st;
  // the N = 16 layout where the plan takes it (its packed B / C tiles are in the workspace)
  cudaError_t e = a.fast16 ? ssm::launch_scan16_fwd_summary(a, s) : ssm::launch_scan_fwd_summary(a, s);
  if (e == cudaSuccess)
    e = ssm::launch_summary_out(a.split_P, a.split_H, a.seq, seq_prev, p->L, decay, state_end,
                                p->B, p->D, p->N, a.Npad, false, s);
  return cuda_status(e, "ssm_scan_fwd_summary launch");
}

ssm_status_t ssm_scan_bwd_summary(const ssm_scan_params* p, const void* dout,
                                  const int32_t* seq_prev, float* decay, float* adj_start,
                                  ssm_stream_t stream) {
  if (injected("ssm_scan_bwd_summary"))
    return fail(SSM_ERR_INJECTED, "ssm_scan_bwd_summary: injected failure");
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  ssm::ScanArgs a;
  ssm_status_t st = summary_setup(p, seq_prev, decay, adj_start, &a, s);
  if (st != SSM_OK) return st;
  if (!p->Cm || !dout) return fail(SSM_ERR_INVALID_ARG, "Cm and dout must be non-NULL");
  if (!aligned(dout, elem_size(p->dtype))) return fail(SSM_ERR_INVALID_ARG, "dout misaligned");
  a.dout = dout;
  a.vec = vec_ok(p->L, {p->delta, p->z, p->Cm, dout, a.seq});
  st = summary_prep(p, a, s);
  if (st != SSM_OK) return st;
  cudaError_t e = (a.fast16 && aligned(dout, 16)) ? ssm::launch_scan16_bwd_summary(a, s)
                                                   : ssm::launch_scan_bwd_summary(a, s);
  if (e == cudaSuccess)
    e = ssm::launch_summary_out(a.split_P, a.split_H, a.seq, seq_prev, p->L, decay, adj_start,
                                p->B, p->D, p->N, a.Npad, true, s);
  return cuda_status(e, "ssm_scan_bwd_summary launch");
}

ssm_status_t ssm_state_carry(const float* decay, const float* value, int R, int r, int reverse,
                             const float* init, const int32_t* seq_prev, const int32_t* seq_idx,
                             int L, float* out, int B, int D, int N, ssm_stream_t stream) {
  if (injected("ssm_state_carry")) return fail(SSM_ERR_INJECTED, "ssm_state_carry: injected failure");
  if (!decay || !value || !out) return fail(SSM_ERR_INVALID_ARG, "decay, value and out must be non-NULL");
  if (B < 1 || D < 1 || N < 1 || R < 1 || r < 0 || r >= R)
    return fail(SSM_ERR_INVALID_ARG, "bad sizes (B=%d D=%d N=%d R=%d r=%d)", B, D, N, R, r);
  if (reverse != 0 && reverse != 1) return fail(SSM_ERR_INVALID_ARG, "reverse=%d", reverse);
  if (!reverse && seq_prev && seq_idx && L < 1) return fail(SSM_ERR_INVALID_ARG, "L=%d", L);
  if (out == decay || out == value || (init && out == init))
    return fail(SSM_ERR_INVALID_ARG, "out may not alias the inputs");
  const void* ps[] = {decay, value, init, seq_prev, seq_idx, out};
  for (const void* q : ps)
    if (q && !aligned(q, 4)) return fail(SSM_ERR_INVALID_ARG, "misaligned pointer");
  return cuda_status(ssm::launch_state_carry(decay, value, R, r, reverse != 0, init,
                                             reverse ? nullptr : seq_prev,
                                             reverse ? nullptr : seq_idx, L, out, B, D, N,
                                             reinterpret_cast<cudaStream_t>(stream)),
                     "ssm_state_carry launch");
}

ssm_status_t ssm_scan_status(const ssm_scan_params* p, int* device_status, ssm_stream_t stream) {
  if (!device_status) return fail(SSM_ERR_INVALID_ARG, "device_status is NULL");
  ssm_status_t st = check_params(p);
  if (st != SSM_OK) return st;
  if (!p->workspace) return fail(SSM_ERR_INVALID_ARG, "workspace is NULL");
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  cudaError_t e = cudaMemcpyAsync(device_status, p->workspace, sizeof(int), cudaMemcpyDeviceToHost, s);
  if (e == cudaSuccess) e = cudaStreamSynchronize(s);
  return cuda_status(e, "ssm_scan_status");
}

ssm_status_t ssm_decode_step(const ssm_decode_params* p, ssm_stream_t stream) {
  if (injected("ssm_decode_step")) return fail(SSM_ERR_INJECTED, "ssm_decode_step: injected failure");
  if (!p) return fail(SSM_ERR_INVALID_ARG, "params is NULL");
  if (p->struct_size != sizeof(ssm_decode_params))
    return fail(SSM_ERR_INVALID_ARG, "params.struct_size %zu != %zu", p->struct_size,
                sizeof(ssm_decode_params));
  if (p->B < 1 || p->D < 1 || p->N < 1)
    return fail(SSM_ERR_INVALID_ARG, "sizes must be >= 1 (B=%d D=%d N=%d)", p->B, p->D, p->N);
  if (p->N > ssm::kNMax) return fail(SSM_ERR_UNSUPPORTED, "N=%d > %d", p->N, ssm::kNMax);
  if (p->W != 4) return fail(SSM_ERR_UNSUPPORTED, "conv width W=%d (only 4)", p->W);
  if ((long)p->B * p->D > (1L << 30))
    return fail(SSM_ERR_UNSUPPORTED, "B * D = %ld rows exceed 2^30", (long)p->B * p->D);
  if (p->dtype != SSM_DTYPE_F32 && p->dtype != SSM_DTYPE_BF16)
    return fail(SSM_ERR_INVALID_ARG, "unknown dtype %d", (int)p->dtype);
  if (!p->x || !p->conv_state || !p->conv_w || !p->delta || !p->Bm || !p->Cm || !p->A ||
      !p->state || !p->out)
    return fail(SSM_ERR_INVALID_ARG,
                "x, conv_state, conv_w, delta, Bm, Cm, A, state and out must be non-NULL");
  const size_t es = elem_size(p->dtype);
  const void* acts[] = {p->x, p->conv_state, p->delta, p->z, p->Bm, p->Cm, p->out, p->u_out};
  for (const void* q : acts)
    if (q && !aligned(q, es)) return fail(SSM_ERR_INVALID_ARG, "activation pointer misaligned");
  const void* f32s[] = {p->conv_w, p->conv_bias, p->A, p->Dskip, p->delta_bias, p->state};
  for (const void* q : f32s)
    if (q && !aligned(q, 4)) return fail(SSM_ERR_INVALID_ARG, "fp32 pointer misaligned");
  if (p->out == p->x || p->out == p->delta || (p->z && p->out == p->z))
    return fail(SSM_ERR_INVALID_ARG, "out may not alias an input");
  ssm::DecodeArgs a{};
  a.x = p->x; a.conv_state = p->conv_state; a.conv_w = p->conv_w; a.conv_bias = p->conv_bias;
  a.delta = p->delta; a.z = p->z; a.Bm = p->Bm; a.Cm = p->Cm; a.A = p->A; a.Dskip = p->Dskip;
  a.delta_bias = p->delta_bias; a.state = p->state; a.out = p->out; a.u_out = p->u_out;
  a.B = p->B; a.D = p->D; a.N = p->N; a.softplus = p->delta_softplus ? 1 : 0;
  a.bf16 = p->dtype == SSM_DTYPE_BF16;
  a.vec = p->N == 16 && aligned(p->state, 16) && aligned(p->A, 16) && aligned(p->Bm, 4 * es) &&
          aligned(p->Cm, 4 * es);
  return cuda_status(ssm::launch_decode_step(a, reinterpret_cast<cudaStream_t>(stream)),
                     "ssm_decode_step launch");
}

ssm_status_t ssm_probe_ex2_rate(float* sink, size_t sink_floats, double* ex2_per_second,
                               ssm_stream_t stream) {
  if (!sink || !ex2_per_second) return fail(SSM_ERR_INVALID_ARG, "sink and ex2_per_second must be non-NULL");
  return cuda_status(ssm::probe_ex2_rate(sink, sink_floats, ex2_per_second,
                                         reinterpret_cast<cudaStream_t>(stream)),
                     "ssm_probe_ex2_rate");
}


// ---------------------------------------------------------------------------
}  // extern "C"

namespace {
// Checks shared by the SSD forward and backward: shapes, support, the
// forward's pointers (y only when `need_y`), alignment.
ssm_status_t ssd_check(const ssm_ssd_params* p, bool need_y) {
  if (!p) return fail(SSM_ERR_INVALID_ARG, "params is NULL");
  if (p->struct_size != sizeof(ssm_ssd_params))
    return fail(SSM_ERR_INVALID_ARG, "struct_size %zu != %zu", p->struct_size, sizeof(ssm_ssd_params));
  if (p->B < 1 || p->L < 1 || p->H < 1 || p->G < 1)
    return fail(SSM_ERR_INVALID_ARG, "B=%d L=%d H=%d G=%d must be >= 1", p->B, p->L, p->H, p->G);
  if (p->H % p->G != 0) return fail(SSM_ERR_INVALID_ARG, "G=%d does not divide H=%d", p->G, p->H);
  if (p->dtype != SSM_DTYPE_BF16) return fail(SSM_ERR_UNSUPPORTED, "ssd: bf16 only");
  if (p->P != 64 || p->N != 128)
    return fail(SSM_ERR_UNSUPPORTED, "ssd: P=%d N=%d (supported: P=64, N=128)", p->P, p->N);
  if (!p->x || !p->dt_raw || !p->A || !p->Bm || !p->Cm || (need_y && !p->y))
    return fail(SSM_ERR_INVALID_ARG, "x, dt_raw, A, Bm, Cm and y must be non-NULL");
  const void* v16[] = {p->x, p->Bm, p->Cm, need_y ? p->y : nullptr, p->chunk_states};
  for (const void* q : v16)
    if (q && !aligned(q, 16))
      return fail(SSM_ERR_INVALID_ARG, "ssd: x, Bm, Cm, y, chunk_states must be 16-byte aligned");
  const void* v4[] = {p->A, p->D, p->dt_bias, p->seq_idx, p->final_state, p->status};
  for (const void* q : v4)
    if (q && !aligned(q, 4)) return fail(SSM_ERR_INVALID_ARG, "ssd: fp32 / int32 pointer misaligned");
  if (!aligned(p->dt_raw, 2)) return fail(SSM_ERR_INVALID_ARG, "ssd: dt_raw misaligned");
  return SSM_OK;
}

ssm::SsdArgs ssd_args(const ssm_ssd_params* p) {
  ssm::SsdArgs a{};
  a.x = p->x;
  a.dt_raw = p->dt_raw;
  a.A = p->A;
  a.Bm = p->Bm;
  a.Cm = p->Cm;
  a.D = p->D;
  a.dt_bias = p->dt_bias;
  a.seq = p->seq_idx;
  a.y = p->y;
  a.final_state = p->final_state;
  a.status = p->status;
  a.B = p->B;
  a.L = p->L;
  a.H = p->H;
  a.P = p->P;
  a.G = p->G;
  a.N = p->N;
  a.softplus = p->dt_softplus ? 1 : 0;
  a.chunk_states = p->chunk_states;
  return a;
}
}  // namespace

extern "C" {

ssm_status_t ssm_ssd_fwd(const ssm_ssd_params* p, ssm_stream_t stream) {
  if (injected("ssm_ssd_fwd")) return fail(SSM_ERR_INJECTED, "ssm_ssd_fwd: injected failure");
  const ssm_status_t st = ssd_check(p, true);
  if (st != SSM_OK) return st;
  return cuda_status(ssm::launch_ssd_fwd(ssd_args(p), reinterpret_cast<cudaStream_t>(stream)),
                     "ssm_ssd_fwd launch");
}

ssm_status_t ssm_ssd_bwd(const ssm_ssd_params* p, const ssm_ssd_grads* g, ssm_stream_t stream) {
  if (injected("ssm_ssd_bwd")) return fail(SSM_ERR_INJECTED, "ssm_ssd_bwd: injected failure");
  const ssm_status_t st = ssd_check(p, false);
  if (st != SSM_OK) return st;
  if (!g) return fail(SSM_ERR_INVALID_ARG, "grads is NULL");
  if (g->struct_size != sizeof(ssm_ssd_grads))
    return fail(SSM_ERR_INVALID_ARG, "grads struct_size %zu != %zu", g->struct_size, sizeof(ssm_ssd_grads));
  if (!p->chunk_states) return fail(SSM_ERR_INVALID_ARG, "ssd bwd: chunk_states (from the forward) is NULL");
  if (!g->dy || !g->dx || !g->ddt_raw || !g->dA || !g->dB || !g->dC)
    return fail(SSM_ERR_INVALID_ARG, "ssd bwd: dy, dx, ddt_raw, dA, dB and dC must be non-NULL");
  const void* v16[] = {g->dy, g->dx, g->dB, g->dC};
  for (const void* q : v16)
    if (!aligned(q, 16)) return fail(SSM_ERR_INVALID_ARG, "ssd bwd: dy, dx, dB, dC must be 16-byte aligned");
  const void* v4[] = {g->ddt_raw, g->dA, g->dD, g->ddt_bias};
  for (const void* q : v4)
    if (q && !aligned(q, 4)) return fail(SSM_ERR_INVALID_ARG, "ssd bwd: fp32 pointer misaligned");
  ssm::SsdArgs a = ssd_args(p);
  a.dy = g->dy;
  a.dx = g->dx;
  a.ddt_raw = g->ddt_raw;
  a.dA = g->dA;
  a.dB = g->dB;
  a.dC = g->dC;
  a.dD = g->dD;
  a.ddt_bias = g->ddt_bias;
  return cuda_status(ssm::launch_ssd_bwd(a, reinterpret_cast<cudaStream_t>(stream)),
                     "ssm_ssd_bwd launch");
}

}  // extern "C"

// ---------------------------------------------------------------------------
// Debug build (-DSSM_DEBUG): records of the device index checks (debug.cuh)
// ---------------------------------------------------------------------------
namespace ssm {
#ifdef SSM_DEBUG
namespace {
// Writes through offset n of a buffer of n floats: the check fails, records
// (kDbgSelftest, n, 1, n) and hands back offset 0, so buf[0] is written.
__global__ void debug_selftest_kernel(float* buf, long long n) {
  buf[SSM_DIDX(kDbgSelftest, n, 1, n)] = 1.0f;
}
}  // namespace

cudaError_t launch_debug_selftest(float* buf, long long n, cudaStream_t s) {
  debug_selftest_kernel<<<1, 1, 0, s>>>(buf, n);
  return cudaGetLastError();
}

SSM_DEBUG_TU(abi)
#endif
}  // namespace ssm

extern "C" {

ssm_status_t ssm_debug_report(ssm_debug_info* out, int reset) {
  if (!out) return fail(SSM_ERR_INVALID_ARG, "out is NULL");
  if (out->struct_size != sizeof(ssm_debug_info))
    return fail(SSM_ERR_INVALID_ARG, "struct_size %zu != %zu", out->struct_size, sizeof(ssm_debug_info));
#ifndef SSM_DEBUG
  (void)reset;
  return fail(SSM_ERR_UNSUPPORTED, "ssm_debug_report: library built without SSM_DEBUG (no device checks)");
#else
  cudaError_t e = cudaDeviceSynchronize();
  if (e != cudaSuccess) return cuda_status(e, "ssm_debug_report: synchronize");
  out->failures = 0;
  out->site = 0;
  out->offset = out->count = out->extent = 0;
  ssm::DebugRecord r;
#define SSM_DEBUG_READ(name)                                                      \
  e = ssm::debug_take_##name(&r, reset != 0);                                     \
  if (e != cudaSuccess) return cuda_status(e, "ssm_debug_report: record of " #name); \
  if (r.failures) {                                                               \
    if (!out->failures) {                                                         \
      out->site = r.site;                                                         \
      out->offset = r.offset;                                                     \
      out->count = r.count;                                                       \
      out->extent = r.extent;                                                     \
    }                                                                             \
    out->failures += r.failures;                                                  \
  }
  SSM_DEBUG_UNITS(SSM_DEBUG_READ)
#undef SSM_DEBUG_READ
  snprintf(out->site_name, sizeof(out->site_name), "%s", ssm::debug_site_name(out->site));
  return ok();
#endif
}

ssm_status_t ssm_debug_selftest(float* buf, size_t n, ssm_stream_t stream) {
#ifndef SSM_DEBUG
  (void)buf;
  (void)n;
  (void)stream;
  return fail(SSM_ERR_UNSUPPORTED, "ssm_debug_selftest: library built without SSM_DEBUG");
#else
  if (!buf || n < 1) return fail(SSM_ERR_INVALID_ARG, "ssm_debug_selftest: buf NULL or n < 1");
  return cuda_status(ssm::launch_debug_selftest(buf, (long long)n, reinterpret_cast<cudaStream_t>(stream)),
                     "ssm_debug_selftest launch");
#endif
}

}  // extern "C"
