/*
 * libssmscan — C ABI for the Mamba-1 selective-SSM layer core on NVIDIA B200
 * (sm_100a): depthwise causal conv1d + SiLU, and the selective scan with
 * softplus step, D skip and SiLU(z) gate, forward and backward, with state
 * and conv resets at packed-document boundaries; an initial state and its
 * gradient, a zero-order-hold discretisation, a complex diagonal A, a fused
 * conv + scan forward, and the one-token recurrent step for inference.
 *
 * Where each operation is defined (page title, section):
 *   conv1d   "hung-phan ml-skills mamba", "Mamba: Selective State Spaces
 *            (S6)" (depthwise Conv1d, padding d_conv-1, first L outputs, then
 *            SiLU) and "Mamba Block Architecture" (Conv1d(k=4) -> SiLU).
 *   scan     same page, "Architecture Diagram" (S6 block: A_bar = exp(dt*A),
 *            B_bar = dt*B, h_t = A_bar h_{t-1} + B_bar x_t, y_t = C_t h_t),
 *            "Core Concept" (y += D x), the S6 sketch (dt = softplus(dt),
 *            y * silu(z)) and "Hardware-Aware Parallel Scan" (the operator
 *            (a1,b1)+(a2,b2) = (a1 a2, a2 b1 + b2) used to combine pieces).
 *   resets   "FLA Mamba and Mamba2" (Axolotl), packing paragraph: conv and
 *            recurrent state start independently for every document.
 *   recompute in backward: "hung-phan ml-skills mamba", "Hardware-Aware
 *            Parallel Scan", memory-optimisation note.
 *   zero-order hold: same page, "Discretization" (B_bar = A^{-1}(exp(dt A) - I) B).
 *   complex A: same page, "S4: Structured State Spaces for Sequences" (S4D:
 *            a diagonal A with complex entries).
 *   pieces of a longer sequence (summaries, carries, conv halos, the final-
 *            state gradient): the same page's associative operator ("Hardware-
 *            Aware Parallel Scan") applied between pieces cut along L; the
 *            Axolotl page ("FLA Mamba and Mamba2") on context parallelism
 *            exchanging conv halos and recurrent states between shards.
 *   fused conv + scan: same page, "Hardware-Aware Parallel Scan" (kernel fusion).
 *   recurrent step: same page, "Dual Computation Modes" (recurrent mode) and
 *            "Inference (Generation)" (a (B, D, N) state carried forward).
 *
 * Conventions for every call:
 *   - All array pointers are caller-owned DEVICE memory, C-contiguous, in the
 *     layouts stated per argument. The library allocates nothing; scratch is
 *     a caller-provided workspace whose size the *_workspace_size calls give.
 *   - Activations ([B][D][L], L fastest) and B/C ([B][N][L]) have dtype
 *     `dtype` (bf16 or fp32); A, D, biases, conv weights, gradients of
 *     parameters and of B/C are fp32; segment ids are int32.
 *   - Work is enqueued on `stream` (a cudaStream_t; NULL = legacy default
 *     stream) and the call returns without synchronising.
 *   - Gradient outputs are overwritten, never accumulated into.
 *   - On any non-OK status nothing has been launched (argument errors) or the
 *     launch itself failed (SSM_ERR_CUDA); ssm_last_error() then returns a
 *     thread-local, human-readable message. No call throws or aborts.
 *   - Sizes: B, D, L >= 1, 1 <= N <= 16, W == 4. Any L is accepted; when L is
 *     a multiple of 8 and every activation pointer is 16-byte aligned the
 *     kernels use 16-byte vector accesses, otherwise a scalar path.
 *   - A segment id array seq_idx [B][L] (nullable) marks documents: token t
 *     starts a new document when seq_idx[b][t] != seq_idx[b][t-1]. Ids need
 *     not be increasing; padding may carry any id of its own (e.g. -1).
 */
#ifndef SSMSCAN_H
#define SSMSCAN_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Same type as cudaStream_t. */
typedef struct CUstream_st* ssm_stream_t;

typedef enum {
    SSM_OK = 0,
    SSM_ERR_INVALID_ARG = 1, /* null pointer, bad size, bad alignment, bad struct_size */
    SSM_ERR_UNSUPPORTED = 2, /* valid but not implemented (e.g. N > 16, W != 4) */
    SSM_ERR_CUDA = 3,        /* a CUDA launch or runtime call failed */
    SSM_ERR_TIMEOUT = 4,     /* a bounded device-side wait gave up (see ssm_scan_status) */
    SSM_ERR_INJECTED = 5     /* host-side fault injection (env SSM_INJECT_FAIL) */
} ssm_status_t;

typedef enum { SSM_DTYPE_F32 = 0, SSM_DTYPE_BF16 = 1 } ssm_dtype_t;

/* Message for the last non-OK status returned on this thread ("" if none). */
const char* ssm_last_error(void);

/* ABI version of this header (bumped on any incompatible change). */
#define SSM_ABI_VERSION 8
int ssm_abi_version(void);

/* ---------------------------------------------------------------------------
 * ssm_conv1d_fwd — depthwise causal conv1d, width W = 4, optional SiLU.
 *   c[b][d][t] = bias[d] + sum_{k=0..3} w[d][k] * x[b][d][t-3+k]
 * where a tap counts only if t-3+k >= 0 and, when seq_idx is given,
 * seq_idx[b][t-3+k] == seq_idx[b][t]. u = silu(c) if silu != 0, else c.
 *   x        [B][D][L] dtype          input
 *   w        [D][W]    fp32           w[d][W-1] multiplies x_t (cross-correlation)
 *   bias     [D]       fp32, nullable (0)
 *   seq_idx  [B][L]    int32, nullable (one document per row)
 *   u        [B][D][L] dtype          output (may not alias x)
 * ------------------------------------------------------------------------ */
ssm_status_t ssm_conv1d_fwd(const void* x, const float* w, const float* bias,
                            const int32_t* seq_idx, void* u, int B, int D, int L,
                            int W, ssm_dtype_t dtype, int silu, ssm_stream_t stream);

/* Bytes of workspace ssm_conv1d_bwd needs for these sizes (per-tile partial
 * sums of dw and dbias, reduced in a fixed order: results are deterministic). */
ssm_status_t ssm_conv1d_bwd_workspace_size(int B, int D, int L, int W, size_t* bytes);

/* ---------------------------------------------------------------------------
 * ssm_conv1d_bwd — gradients of ssm_conv1d_fwd's output u.
 *   du       [B][D][L] dtype   upstream gradient dL/du
 *   dx       [B][D][L] dtype   output dL/dx
 *   dw       [D][W]    fp32    output dL/dw (summed over batch and time)
 *   dbias    [D]       fp32, nullable   output dL/dbias
 *   workspace            device scratch of ssm_conv1d_bwd_workspace_size bytes
 * The pre-activation is recomputed from x, w, bias (nothing is saved by fwd).
 * ------------------------------------------------------------------------ */
ssm_status_t ssm_conv1d_bwd(const void* x, const float* w, const float* bias,
                            const int32_t* seq_idx, const void* du, void* dx,
                            float* dw, float* dbias, int B, int D, int L, int W,
                            ssm_dtype_t dtype, int silu, void* workspace,
                            size_t workspace_bytes, ssm_stream_t stream);

/* ---------------------------------------------------------------------------
 * ssm_conv1d_bwd_noalloc — ssm_conv1d_bwd for callers that cannot allocate
 * device memory: hosts that hand a library only its input and output
 * buffers (plugin interfaces of serving runtimes and frameworks that own all
 * device memory) and loops that must not call cudaMalloc / cudaFree, which
 * can synchronise the whole device. There is no counterpart on the pages;
 * this is a deployment variant of the call above.
 *   Arguments and results are those of ssm_conv1d_bwd without the workspace.
 *   Scratch: the per-tile dw / dbias partial sums go to a fixed device array
 *   of 2^20 floats (4 MiB) that every device using the library keeps until
 *   the process exits; sizes with B * ceil(L / 1024) * D * 5 > 2^20 are
 *   rejected with SSM_ERR_UNSUPPORTED and a message naming the limit.
 *   The first call on each device looks up the array's device address
 *   (cudaGetSymbolAddress, with that device current) and caches it; make that
 *   first call before any stream capture on the device. The cached address
 *   outlives a cudaDeviceReset, so calling again on a device after a reset
 *   is not supported.
 *   The array is shared by every call and keeps the last call's contents;
 *   each call overwrites every partial it reads, so nothing needs clearing,
 *   but two calls that overlap on the GPU (other streams, other threads) race
 *   on it: serialise them.
 *   Allocates nothing and calls no allocating routine.
 * ------------------------------------------------------------------------ */
ssm_status_t ssm_conv1d_bwd_noalloc(const void* x, const float* w, const float* bias,
                                    const int32_t* seq_idx, const void* du, void* dx,
                                    float* dw, float* dbias, int B, int D, int L, int W,
                                    ssm_dtype_t dtype, int silu, ssm_stream_t stream);

/* ---------------------------------------------------------------------------
 * Selective scan. For each row (b, d) and state n < N, with
 *   dt_t = softplus(delta[b][d][t] + delta_bias[d])   (or without softplus)
 *   a_t  = exp(dt_t * A[d][n])      (0 at the first token of a document)
 *   h_t  = a_t * h_{t-1} + dt_t * Bm[b][n][t] * u[b][d][t]   (see discretization),
 *   h_{-1} = initial_state[b][d][n]  (0 when initial_state is NULL)
 *   y_t  = sum_n Cm[b][n][t] * h_t + Dskip[d] * u[b][d][t]
 *   out  = y_t * silu(z[b][d][t])   (or y_t when z is NULL)
 * final_state[b][d][n] = h_{L-1}.
 * ------------------------------------------------------------------------ */
typedef struct {
    size_t struct_size;        /* = sizeof(ssm_scan_params) */
    int B, D, L, N;
    ssm_dtype_t dtype;         /* dtype of u, delta, z, Bm, Cm, out */
    const void* u;             /* [B][D][L] scan input x (the conv+SiLU output) */
    const void* delta;         /* [B][D][L] raw step, before bias and softplus */
    const void* z;             /* [B][D][L] gate input, nullable (no gate) */
    const float* A;            /* [D][N] state matrix diagonal (negative for decay) */
    const float* Dskip;        /* [D] nullable (0) */
    const float* delta_bias;   /* [D] nullable (0) */
    const void* Bm;            /* [B][N][L] */
    const void* Cm;            /* [B][N][L] */
    int delta_softplus;        /* 1: dt = softplus(delta + bias); 0: dt = delta + bias */
    const int32_t* seq_idx;    /* [B][L] nullable */
    const int32_t* cu_seqlens; /* [n_docs + 1] nullable, B == 1 only, exclusive with seq_idx;
                                  cu_seqlens[0] = 0, increasing, cu_seqlens[n_docs] == L */
    int n_docs;
    int n_splits;              /* 0: automatic. P >= 1: split each row's L into P ranges
                                  run on different CTAs and joined by a carry pass */
    void* out;                 /* [B][D][L] output */
    float* final_state;        /* [B][D][N] nullable */
    void* workspace;           /* device scratch, >= ssm_scan_workspace_size bytes, 256-B aligned */
    size_t workspace_bytes;
    const float* initial_state;/* [B][D][N] nullable: the state before token 0 (h_{-1}); with
                                  seq_idx it feeds the first document of each row only */
    int discretization;        /* 0: B_bar = dt B (the S6 block, "Architecture Diagram");
                                  1: zero-order hold ("Discretization"), for diagonal A
                                  B_bar = (exp(dt A) - 1) / A B (-> dt B as A -> 0) */
    int state_complex;         /* 0: real A as above. 1: complex diagonal A, the S4D form
                                  ("S4: Structured State Spaces for Sequences"), made selective:
                                  A [D][N][2] (re, im), Bm / Cm [B][N][2][L] (per state a real
                                  then an imaginary row), initial_state / final_state
                                  [B][D][N][2]; a_t = exp(dt_t A) complex, h complex and
                                  y_t = 2 Re(sum_n C h_t) + Dskip u_t (each state stands for
                                  itself and its conjugate). Needs discretization 0 and
                                  n_splits 0 or 1 (else SSM_ERR_UNSUPPORTED), A, initial_state
                                  and final_state 8-byte aligned; not available in
                                  ssm_conv1d_scan_fwd. Gradients take the same layouts
                                  (dA [D][N][2], dB / dC [B][N][2][L], dinitial_state
                                  [B][D][N][2]), each pair holding dL/dRe and dL/dIm. */
} ssm_scan_params;

/* Workspace bytes for these params: the state entering every 16-token block
 * and, with a gate, y before the gate (both written by the forward, read by
 * the backward), split carries, segment ids built from cu_seqlens, and
 * partial sums of the backward's parameter reductions. */
ssm_status_t ssm_scan_workspace_size(const ssm_scan_params* p, size_t* bytes);

/* Forward. Also writes the checkpoints the backward reads into p->workspace:
 * keep the workspace unchanged between ssm_scan_fwd and ssm_scan_bwd. */
ssm_status_t ssm_scan_fwd(const ssm_scan_params* p, ssm_stream_t stream);

/* ---------------------------------------------------------------------------
 * ssm_conv1d_scan_fwd — ssm_conv1d_fwd (W = 4, SiLU on) and ssm_scan_fwd in
 * one kernel: the pages' kernel fusion ("hung-phan ml-skills mamba",
 * "Hardware-Aware Parallel Scan") applied to the conv and SiLU of "Mamba:
 * Selective State Spaces (S6)". Reads x [B][D][L] (dtype p->dtype),
 * conv_w [D][4] and conv_bias [D] (nullable); the conv taps follow p's
 * document ids (a tap in another document reads 0). Computes u =
 * silu(conv(x)) inside the scan, WRITES it to p->u (writable device memory,
 * not aliasing x: ssm_scan_bwd reads it, and it is the conv output a caller
 * differentiates with ssm_conv1d_bwd), and writes everything ssm_scan_fwd
 * writes. u, out, final_state and the workspace are bitwise equal to those of
 * ssm_conv1d_fwd followed by ssm_scan_fwd. Errors as ssm_scan_fwd, plus
 * SSM_ERR_INVALID_ARG for a NULL x / conv_w, x == p->u, or misalignment.
 * ------------------------------------------------------------------------ */
ssm_status_t ssm_conv1d_scan_fwd(const ssm_scan_params* p, const void* x, const float* conv_w,
                                 const float* conv_bias, ssm_stream_t stream);

typedef struct {
    size_t struct_size;        /* = sizeof(ssm_scan_grads) */
    const void* dout;          /* [B][D][L] dtype, dL/dout */
    void* du;                  /* [B][D][L] dtype, output dL/du */
    void* ddelta;              /* [B][D][L] dtype, output dL/d(raw delta) */
    void* dz;                  /* [B][D][L] dtype, output dL/dz; required iff z != NULL */
    float* dA;                 /* [D][N] output */
    float* dB;                 /* [B][N][L] fp32 output */
    float* dC;                 /* [B][N][L] fp32 output */
    float* dD;                 /* [D] nullable output */
    float* ddelta_bias;        /* [D] nullable output */
    int deterministic;         /* 0: dB and dC are summed over channels with fp32 atomic adds,
                                  whose order (and so the last bits of the result) varies from
                                  run to run. 1: every CTA stores the sum over its rows in
                                  `workspace` below and a second kernel adds the row groups in a
                                  fixed order, so dB and dC are bitwise reproducible (for the same
                                  inputs, sizes and device). dA, dD and ddelta_bias are reduced in
                                  a fixed order either way. */
    float* dinitial_state;     /* [B][D][N] nullable output: dL/dh_{-1} (the gradient with
                                  respect to initial_state, or to the zero state when NULL) */
    const float* dfinal_state; /* [B][D][N] nullable input: dL/dh_{L-1}, a gradient reaching the
                                  final state from outside (a later piece of the sequence, a
                                  loss on the state); NULL = 0. Complex A: (re, im) pairs */
    void* workspace;           /* device scratch of the backward, caller-owned, 256-byte aligned,
                                  >= ssm_scan_bwd_workspace_size bytes: the row groups' dB / dC
                                  sums when deterministic = 1 (NULL and 0 bytes otherwise). Not
                                  the forward's workspace, which comes in the params. */
    size_t workspace_bytes;
} ssm_scan_grads;

/* Bytes of grads->workspace that ssm_scan_bwd needs for these params and
 * grads: 0 unless grads->deterministic == 1, then (row groups) * 2 * B * N *
 * L * 4 (twice that for a complex A), with 8 (general kernels) or 12 (N = 16
 * kernels) rows per group: about 1.1 GB at B = 2, D = 1536, N = 16, L = 32768. */
ssm_status_t ssm_scan_bwd_workspace_size(const ssm_scan_params* p, const ssm_scan_grads* g,
                                         size_t* bytes);

/* Backward. Recomputes states from the checkpoints in p->workspace, so the
 * same params (inputs and workspace) as the forward must be passed. A
 * gradient of the final state enters through g->dfinal_state. */
ssm_status_t ssm_scan_bwd(const ssm_scan_params* p, const ssm_scan_grads* g,
                          ssm_stream_t stream);

/* ---------------------------------------------------------------------------
 * Pieces of a longer sequence. A sequence cut along L into R consecutive
 * pieces (for instance one per rank) is scanned piece by piece: the state
 * entering piece r is the fold of the earlier pieces' summaries, and the
 * gradient reaching piece r's final state is the fold of the later pieces'
 * backward summaries. Every piece is then an ordinary ssm_scan_fwd /
 * ssm_scan_bwd call with initial_state / dfinal_state set. Real A only
 * (state_complex != 0: SSM_ERR_UNSUPPORTED).
 *
 * ssm_scan_fwd_summary — for every (b, d, n) of this piece:
 *   decay[b][d][n]     = prod_t a_t over the piece (0 when a document starts
 *                        inside it, or at token 0 relative to seq_prev)
 *   state_end[b][d][n] = the final state from a zero initial state
 * so that final state = decay * (state entering) + state_end. Reads u,
 * delta, A, Bm (and delta_bias, seq_idx / cu_seqlens, discretization) of p;
 * ignores initial_state, z, Cm and out. seq_prev [B] nullable: the document
 * id of the token before token 0 (from the previous piece). Uses
 * p->workspace as scratch (size from ssm_scan_workspace_size): call it
 * before the piece's ssm_scan_fwd, not between that and its ssm_scan_bwd.
 * ------------------------------------------------------------------------ */
ssm_status_t ssm_scan_fwd_summary(const ssm_scan_params* p, const int32_t* seq_prev,
                                  float* decay, float* state_end, ssm_stream_t stream);

/* ssm_scan_bwd_summary — for every (b, d, n) of this piece, from dout alone:
 *   decay[b][d][n]     as above
 *   adj_start[b][d][n] = dL/dh_{-1} of the piece with no gradient reaching its
 *                        final state (0 when token 0 starts a document)
 * so that the gradient leaving the piece through its start is
 * decay * (gradient of its final state) + adj_start. Reads delta, A, Cm,
 * z, delta_bias, seq_idx / cu_seqlens of p and dout [B][D][L]; the
 * workspace is scratch as for ssm_scan_fwd_summary (call it before the
 * piece's ssm_scan_fwd, or after its ssm_scan_bwd). */
ssm_status_t ssm_scan_bwd_summary(const ssm_scan_params* p, const void* dout,
                                  const int32_t* seq_prev, float* decay, float* adj_start,
                                  ssm_stream_t stream);

/* ssm_state_carry — fold R pieces' summaries, each [B][D][N] fp32, stacked
 * as decay [R][B][D][N] and value [R][B][D][N]:
 *   reverse = 0: out = state entering piece r: h = init (NULL = 0), then
 *                h = decay[j] h + value[j] for j = 0 .. r-1; h = 0 when piece
 *                r's token 0 starts a document (seq_prev [B] and seq_idx
 *                [B][L] of piece r given and different).
 *   reverse = 1: out = gradient reaching piece r's final state: c = init
 *                (NULL = 0), then c = decay[j] c + value[j] for j = R-1 .. r+1.
 * 0 <= r < R. out [B][D][N] may not alias the inputs. */
ssm_status_t ssm_state_carry(const float* decay, const float* value, int R, int r, int reverse,
                             const float* init, const int32_t* seq_prev, const int32_t* seq_idx,
                             int L, float* out, int B, int D, int N, ssm_stream_t stream);

/* ssm_conv1d_fwd_ctx — ssm_conv1d_fwd for a piece of a longer sequence:
 * the taps before token 0 read x_prev [B][D][W-1] (the W-1 inputs before
 * the piece, oldest first; NULL = 0) under document ids seq_prev [B][W-1]
 * (required when seq_idx and x_prev are both given). */
ssm_status_t ssm_conv1d_fwd_ctx(const void* x, const float* w, const float* bias,
                                const int32_t* seq_idx, const void* x_prev,
                                const int32_t* seq_prev, void* u, int B, int D, int L, int W,
                                ssm_dtype_t dtype, int silu, ssm_stream_t stream);

/* ssm_conv1d_bwd_ctx — ssm_conv1d_bwd for a piece of a longer sequence:
 * x_prev / seq_prev as in ssm_conv1d_fwd_ctx (the recomputed pre-activation
 * and dw use them); x_next, du_next [B][D][W-1] and seq_next [B][W-1] are
 * the next piece's first inputs, their upstream gradients and ids, which
 * reach this piece's last W-1 dx through the taps (NULL = none; x_next and
 * du_next come together; seq_next is required when seq_idx and x_next are
 * both given). dw and dbias sum this piece's own tokens only, so a caller
 * adds the pieces' dw and dbias. */
ssm_status_t ssm_conv1d_bwd_ctx(const void* x, const float* w, const float* bias,
                                const int32_t* seq_idx, const void* x_prev,
                                const int32_t* seq_prev, const void* x_next,
                                const void* du_next, const int32_t* seq_next, const void* du,
                                void* dx, float* dw, float* dbias, int B, int D, int L, int W,
                                ssm_dtype_t dtype, int silu, void* workspace,
                                size_t workspace_bytes, ssm_stream_t stream);

/* ---------------------------------------------------------------------------
 * ssm_scan_status — device-side status of the last ssm_scan_fwd / ssm_scan_bwd
 * that used p->workspace: 0 when every bounded wait inside the kernels (the
 * completion waits of the TMA tile copies) completed, SSM_ERR_TIMEOUT when one
 * gave up (the kernel then stopped early and its outputs are invalid). The
 * forward resets the word; the backward only sets it. Copies 4 bytes from the
 * workspace to *device_status and SYNCHRONISES `stream`.
 * A timeout means a copy engine or the memory system did not answer within
 * about 2^22 polls; the kernel waits (again bounded) for its own copies
 * before it returns, but one that never completed may still be pending. After
 * SSM_ERR_TIMEOUT treat the stream and the context as unreliable: discard the
 * outputs and the workspace, and recreate the context before further work.
 * ------------------------------------------------------------------------ */
ssm_status_t ssm_scan_status(const ssm_scan_params* p, int* device_status, ssm_stream_t stream);

/* ---------------------------------------------------------------------------
 * ssm_probe_ex2_rate — diagnostic: measures this device's sustained rate of
 * the ex2.approx.f32 instruction (base-2 exponential on the special-function
 * unit), the instruction the scan issues once per (token, state). Launches a
 * fixed microkernel (8 CTAs of 256 threads per SM, ~20 ms) on `stream`, times
 * it with CUDA events and SYNCHRONISES the stream before returning.
 *   sink            device scratch of >= 2048 * SM-count floats (never read back)
 *   ex2_per_second  host output: ex2 results per second, whole device
 * Not part of the layer's math (no counterpart on the pages): it supplies the
 * measured SFU peak for the roofline the benchmark reports.
 * ------------------------------------------------------------------------ */
ssm_status_t ssm_probe_ex2_rate(float* sink, size_t sink_floats, double* ex2_per_second,
                                ssm_stream_t stream);

/* ---------------------------------------------------------------------------
 * Recurrent form, one token per row: the layer's inference mode
 * ("hung-phan ml-skills mamba", "Dual Computation Modes": recurrent mode,
 * token by token with O(1) memory per step; "Inference (Generation)": no KV
 * cache, a (B, D, N) state is carried forward). The same conv, step and
 * state update as the sequence form, for every (b, d):
 *   c = conv_bias[d] + sum_{k < W-1} conv_w[d][k] conv_state[b][d][k]
 *                    + conv_w[d][W-1] x[b][d]
 *   conv_state[b][d] <- (conv_state[b][d][1 .. W-2], x[b][d])
 *   u = silu(c);  dt = softplus(delta[b][d] + delta_bias[d])  (or without softplus)
 *   state[b][d][n] <- exp(dt A[d][n]) state[b][d][n] + dt Bm[b][n] u
 *   out[b][d] = (sum_n Cm[b][n] state[b][d][n] + Dskip[d] u) silu(z[b][d])
 * so stepping it over a sequence from a zero conv window and a zero state
 * reproduces ssm_conv1d_fwd + ssm_scan_fwd, and after a prefill (conv window
 * = the last W-1 inputs, state = the prefill's final_state) it continues it.
 * Sizes: B, D >= 1, 1 <= N <= 16, W == 4 (else SSM_ERR_UNSUPPORTED).
 * conv_state and state are updated in place; no other input is written.
 * ------------------------------------------------------------------------ */
typedef struct {
    size_t struct_size;        /* = sizeof(ssm_decode_params) */
    int B, D, N, W;
    ssm_dtype_t dtype;         /* dtype of x, conv_state, delta, z, Bm, Cm, out, u_out */
    const void* x;             /* [B][D] conv input of this token */
    void* conv_state;          /* [B][D][W-1] in/out: the previous W-1 inputs, oldest first */
    const float* conv_w;       /* [D][W] */
    const float* conv_bias;    /* [D] nullable (0) */
    const void* delta;         /* [B][D] raw step, before bias and softplus */
    const void* z;             /* [B][D] gate input, nullable (no gate) */
    const void* Bm;            /* [B][N] */
    const void* Cm;            /* [B][N] */
    const float* A;            /* [D][N] */
    const float* Dskip;        /* [D] nullable (0) */
    const float* delta_bias;   /* [D] nullable (0) */
    int delta_softplus;        /* as in ssm_scan_params */
    float* state;              /* [B][D][N] fp32 in/out: h_{t-1} on entry, h_t on return */
    void* out;                 /* [B][D] output */
    void* u_out;               /* [B][D] nullable output: the conv+SiLU value u */
} ssm_decode_params;

ssm_status_t ssm_decode_step(const ssm_decode_params* p, ssm_stream_t stream);

/* ---------------------------------------------------------------------------
 * ssm_ssd_fwd — Mamba-2 SSD forward ("hung-phan ml-skills mamba", section
 * "Mamba-2: Structured State Space Duality (SSD)": A is a scalar per head).
 * Per batch b, head h (group g = h / (H / G)) and token t:
 *   dt_t = softplus(dt_raw[b][t][h] + dt_bias[h])      (or without softplus)
 *   a_t  = exp(dt_t A[h])                               (0 at a document start)
 *   S_t[p][n] = a_t S_{t-1}[p][n] + dt_t x[b][t][h][p] B[b][t][g][n],  S_{-1} = 0
 *   y[b][t][h][p] = sum_n C[b][t][g][n] S_t[p][n] + D[h] x[b][t][h][p]
 * computed in chunks of 128 tokens as masked matrix products on the tensor
 * cores (bf16 operands, fp32 accumulation; the state between chunks is kept
 * in fp32 and enters the next chunk's product rounded to bf16).
 *   x        [B][L][H][P] bf16         y       [B][L][H][P] bf16 output
 *   dt_raw   [B][L][H]    bf16         Bm, Cm  [B][L][G][N] bf16
 *   A        [H] fp32 (negative)       D, dt_bias  [H] fp32, nullable (0)
 *   seq_idx  [B][L] int32, nullable    final_state [B][H][P][N] fp32, nullable
 * Supported: dtype bf16, P = 64, N = 128, G >= 1 dividing H, any L >= 1
 * (else SSM_ERR_UNSUPPORTED); every pointer 16-byte aligned. One CTA per
 * (b, h); the chunks of a row run in order inside it.
 * chunk_states (nullable; required by ssm_ssd_bwd): [B][H][nc][N][P] fp32
 * with nc = ceil(L / 128), the state entering each chunk (S_{128c-1}
 * stored [n][p]; zeros for chunk 0); caller-owned, written by this call.
 * ------------------------------------------------------------------------ */
typedef struct {
    size_t struct_size;        /* = sizeof(ssm_ssd_params) */
    int B, L, H, P, G, N;
    ssm_dtype_t dtype;
    const void* x;
    const void* dt_raw;
    const float* A;
    const void* Bm;
    const void* Cm;
    const float* D;
    const float* dt_bias;
    int dt_softplus;
    const int32_t* seq_idx;
    void* y;
    float* final_state;
    int* status;               /* device int, nullable: SSM_ERR_TIMEOUT if a bounded wait for
                                  the tensor cores gave up (outputs then invalid) */
    float* chunk_states;       /* [B][H][ceil(L/128)][N][P] fp32, nullable (see above) */
} ssm_ssd_params;

ssm_status_t ssm_ssd_fwd(const ssm_ssd_params* p, ssm_stream_t stream);

/* ---------------------------------------------------------------------------
 * ssm_ssd_bwd — reverse mode of ssm_ssd_fwd (same section of "hung-phan
 * ml-skills mamba"), given dy = dL/dy and the chunk_states the forward wrote
 * for the same inputs (no gradient enters through the final state). With
 * G_t[p][n] = dL/dS_t (G_t = dy_t[p] C_t[n] + a_{t+1} G_{t+1}):
 *   dx[b][t][h][p] = D[h] dy_t[p] + dt_t sum_n G_t[p][n] B_t[n]
 *   d dt_t = sum_{p,n} G_t[p][n] (x_t[p] B_t[n] + a_t A[h] S_{t-1}[p][n])
 *   dA[h]  = sum over b, t of dt_t sum_{p,n} G_t[p][n] a_t S_{t-1}[p][n]
 *   dB[b][t][g][n] = sum over the group's heads of dt_t sum_p G_t[p][n] x_t[p]
 *   dC[b][t][g][n] = sum over the group's heads of sum_p dy_t[p] S_t[p][n]
 *   dD[h] = sum dy x;  d dt_raw = d dt sigmoid(dt_raw + dt_bias) with the
 *   softplus (else d dt);  d dt_bias[h] = sum over b, t of d dt_raw.
 * Per chunk of 128 tokens, in reverse order, the transposed masked products
 * (dy x^T, M^T dy, dS B, dS^T C, C^T dy, ...) run on the tensor cores with
 * bf16 operands and fp32 accumulation; the state adjoint carried between
 * chunks is fp32 and enters the products rounded to bf16.
 *   p: the forward's parameters (y, final_state ignored), with chunk_states
 *      non-NULL and as the forward wrote it.
 *   dy, dx    [B][L][H][P] bf16        ddt_raw   [B][L][H] fp32
 *   dB, dC    [B][L][G][N] fp32        dA        [H] fp32
 *   dD, ddt_bias [H] fp32, nullable
 * Outputs are overwritten (the call zeroes dA, dB, dC, dD, ddt_bias, then
 * adds each head's share with fp32 atomics: not bitwise reproducible).
 * Same support and alignment rules as ssm_ssd_fwd; dx, dy, dB, dC 16-byte
 * aligned. Errors and the status word as for ssm_ssd_fwd.
 * ------------------------------------------------------------------------ */
typedef struct {
    size_t struct_size;        /* = sizeof(ssm_ssd_grads) */
    const void* dy;
    void* dx;
    float* ddt_raw;
    float* dA;
    float* dB;
    float* dC;
    float* dD;
    float* ddt_bias;
} ssm_ssd_grads;

ssm_status_t ssm_ssd_bwd(const ssm_ssd_params* p, const ssm_ssd_grads* g, ssm_stream_t stream);

/* ---------------------------------------------------------------------------
 * Debug build: device-side index checks (the library compiled with
 * -DSSM_DEBUG; a release build carries no checks and both calls below return
 * SSM_ERR_UNSUPPORTED without touching the device).
 *
 * In a debug build the kernels check the element offsets of their global
 * accesses against the extents the call's shapes give their buffers: every
 * activation and B / C row against [B][D][L] (or [B][L][H][P], [B][L][G][N]
 * for the SSD), the tokens a thread touches against its row, the checkpoint
 * and chunk-state arrays, the dB / dC sums and partials, the conv1d partials
 * against the workspace they were sized in, the recurrent state. A failed check
 * is counted, the first failure of each kernel source is kept, and the
 * access is redirected to the first element of its range, so the kernel ends
 * normally: no trap, no fault, no skipped barrier. Outputs of a call with a
 * failed check are invalid. Checks are compiled in one library per build;
 * there is no run-time switch.
 *
 * ssm_debug_report SYNCHRONISES the current device, then fills *out with
 * the failures since the last reset (summed over kernel sources) and one
 * kept failure (site id and name, offset, count, extent; site 0 "none" when
 * there was none); reset != 0 clears the records. Records are per device.
 *
 * ssm_debug_selftest launches one thread that writes through offset n of
 * `buf` (n >= 1 floats of device memory): its check fails, is recorded with
 * offset n, count 1, extent n, and the write lands on buf[0]. It exists to
 * show that a failing check is seen; it reads nothing of the layer's math.
 * ------------------------------------------------------------------------ */
typedef struct ssm_debug_info {
  size_t struct_size;            /* = sizeof(ssm_debug_info) */
  unsigned long long failures;   /* failed checks since the last reset */
  int site;                      /* id of the kept failure (0: none) */
  long long offset;              /* its element offset */
  long long count;               /* elements the access touches from there */
  long long extent;              /* extent the offset was held to */
  char site_name[48];            /* printable name of the site */
} ssm_debug_info;

ssm_status_t ssm_debug_report(ssm_debug_info* out, int reset);
ssm_status_t ssm_debug_selftest(float* buf, size_t n, ssm_stream_t stream);

#ifdef __cplusplus
}
#endif
#endif /* SSMSCAN_H */
