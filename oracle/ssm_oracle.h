/*
 * CPU oracle for the Mamba-1 selective-SSM layer core — TEST INFRASTRUCTURE.
 * fp64 throughout. Only tests, the smoke check and the benchmark's CPU
 * baseline use it; the product library never includes or links it.
 *
 * Layouts (all contiguous): activations [B][D][L]; B/C [B][N][L];
 * A [D][N]; conv weight [D][W]; per-channel vectors [D]; seq_idx [B][L]
 * (NULL = one segment per row); initial / final state [B][D][N] (h0 NULL =
 * zero state). zoh = 0: B_bar = dt B; zoh = 1: zero-order hold,
 * B_bar = (exp(dt A) - 1) / A B.
 */
#ifndef SSM_ORACLE_H
#define SSM_ORACLE_H
#include <stddef.h>
#include <stdint.h>

void oracle_round_bf16(const double* in, double* out, size_t n);

void oracle_conv1d_fwd(const double* x, const double* w, const double* bias,
                       const int32_t* seq, double* c, double* u,
                       int B, int D, int L, int W, int silu);
void oracle_conv1d_bwd(const double* x, const double* w, const double* bias,
                       const int32_t* seq, const double* du, double* dx,
                       double* dw, double* dbias, int B, int D, int L, int W, int silu);

void oracle_scan_fwd(const double* u, const double* delta, const double* z,
                     const double* A, const double* Dskip, const double* delta_bias,
                     const double* Bm, const double* Cm, int softplus_on, int zoh,
                     const int32_t* seq, const double* h0, double* out, double* y_out,
                     double* final_state, int B, int D, int L, int N);
void oracle_scan_bwd(const double* u, const double* delta, const double* z,
                     const double* A, const double* Dskip, const double* delta_bias,
                     const double* Bm, const double* Cm, int softplus_on, int zoh,
                     const int32_t* seq, const double* h0, const double* dout, double* du,
                     double* ddelta, double* dz, double* dA, double* dB,
                     double* dC, double* dD, double* ddelta_bias, double* dh0,
                     const double* dhL, int B, int D, int L, int N);

void oracle_scan_fwd_mt(const double* u, const double* delta, const double* z,
                        const double* A, const double* Dskip, const double* delta_bias,
                        const double* Bm, const double* Cm, int softplus_on, int zoh,
                        const int32_t* seq, const double* h0, double* out, double* y_out,
                        double* final_state, int B, int D, int L, int N, int nthreads);
void oracle_scan_bwd_mt(const double* u, const double* delta, const double* z,
                        const double* A, const double* Dskip, const double* delta_bias,
                        const double* Bm, const double* Cm, int softplus_on, int zoh,
                        const int32_t* seq, const double* h0, const double* dout, double* du,
                        double* ddelta, double* dz, double* dA, double* dB,
                        double* dC, double* dD, double* ddelta_bias, double* dh0,
                        const double* dhL, int B, int D, int L, int N, int nthreads);
/* Recurrent form, one token (x, delta, z [B][D]; Bt, Ct [B][N];
 * conv_state [B][D][W-1] and h [B][D][N] updated in place). */
void oracle_decode_step(const double* x, double* conv_state, const double* w,
                        const double* conv_bias, const double* delta, const double* z,
                        const double* Bt, const double* Ct, const double* A,
                        const double* Dskip, const double* delta_bias, int softplus_on,
                        double* h, double* out, double* u_out, int B, int D, int N, int W);
/* Complex diagonal A (S4D), selective: A [D][N][2], Bm / Cm [B][N][2][L]
 * (real, imaginary planes), h0 / final state / dh0 [B][D][N][2], dA
 * [D][N][2], dB / dC [B][N][2][L]; y = 2 Re(sum_n C h) + D u. */
void oracle_cscan_fwd(const double* u, const double* delta, const double* z, const double* A,
                      const double* Dskip, const double* delta_bias, const double* Bm,
                      const double* Cm, int softplus_on, const int32_t* seq, const double* h0,
                      double* out, double* y_out, double* final_state, int B, int D, int L, int N);
void oracle_cscan_bwd(const double* u, const double* delta, const double* z, const double* A,
                      const double* Dskip, const double* delta_bias, const double* Bm,
                      const double* Cm, int softplus_on, const int32_t* seq, const double* h0,
                      const double* dout, double* du, double* ddelta, double* dz, double* dA,
                      double* dB, double* dC, double* dD, double* ddelta_bias, double* dh0,
                      const double* dhL, int B, int D, int L, int N);
/* Mamba-2 SSD (scalar A per head, heads of width P, G groups of shared
 * B / C): x, y, dx [B][L][H][P]; dt_raw, ddt_raw [B][L][H]; A, Dh, dt_bias,
 * dA, dD, ddt_bias [H]; Bm, Cm, dB, dC [B][L][G][N]; final state
 * [B][H][P][N]. */
void oracle_ssd_fwd(const double* x, const double* dt_raw, const double* A, const double* Bm,
                    const double* Cm, const double* Dh, const double* dt_bias, int softplus_on,
                    const int32_t* seq, double* y, double* final_state, int B, int L, int H, int P,
                    int G, int N);
void oracle_ssd_bwd(const double* x, const double* dt_raw, const double* A, const double* Bm,
                    const double* Cm, const double* Dh, const double* dt_bias, int softplus_on,
                    const int32_t* seq, const double* dy, double* dx, double* ddt_raw, double* dA,
                    double* dB, double* dC, double* dD, double* ddt_bias, int B, int L, int H,
                    int P, int G, int N);
#endif
