/*
 * csa_oracle.h -- plain CPU reference of the CSA / HCA forward pass.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product path may include, link
 * or call this code; only the tests, the smoke check and the CPU-baseline leg
 * of the benchmark use it.  It shares no code with the CUDA library.
 *
 * Every routine works on IEEE double (fp64) values: callers convert the stored
 * bf16 / fp8 / fp32 data to the exact double they represent.  The loops follow
 * the equations of the DeepSeek-V4 reading notes ("DeepSeekV4技术报告阅读笔记",
 * zouxinn.github.io), section 2.3-2.5, eq. 9-27, and the PaperTrace analysis
 * ("DeepSeek-V4: 压缩注意力撑起 1M 上下文"), section 2.1-2.4, with no blocking
 * or reordering beyond what those equations state.
 *
 * Indices are 0-based: token j, entry i (covering a-window tokens m*i..m*i+m-1
 * and b-window tokens m*(i-1)..m*i-1), query position t0.
 */
#ifndef CSA_ORACLE_H
#define CSA_ORACLE_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Number of OpenMP threads the oracle uses (1 without OpenMP). */
int ocsa_num_threads(void);

/* RoPE on one vector: x points at the rotated part (rope_dims values,
 * interleaved pairs (2p, 2p+1)); rotates pair p by pos * base^(-2p/rope_dims).
 * A negative pos de-rotates (R_{-t}).  Notes section 2.5.2. */
void ocsa_rope(double* x, int rope_dims, double base, double pos);

/* RMSNorm with unit gain: x <- x / sqrt(mean(x^2) + eps).  Notes 2.5.1. */
void ocsa_rmsnorm(double* x, int n, double eps);

/* out[r][j] = sum_k A[r][k] * W[k][j] for r < rows (plain triple loop).
 * This is the projection H * W of eq. 9-10 / 20-21. */
void ocsa_matmul(int rows, int d, const double* A, int width, const double* W,
                 double* out);

/* Compression of eq. 11-12 (overlap = 1, CSA) or eq. 22-23 (overlap = 0,
 * HCA) for entries i0 <= i < i1 of one sequence of T tokens.
 *   H        [T][d]
 *   Wkv_a/Wz_a [d][width]; Wkv_b/Wz_b [d][width] (ignored when overlap = 0)
 *   B_a, B_b [m][width] position bias (B_b ignored when overlap = 0)
 *   out      [i1-i0][width] folded entries (no normalisation, no RoPE)
 *   S_out    nullable [i1-i0][2m][width] softmax weights; slot r < m is the
 *            a-branch token m*i+r, slot m+r the b-branch token m*(i-1)+r
 *            (0 for i = 0 and for HCA).
 * Returns 0, or -1 if the entry range needs tokens >= T. */
int ocsa_compress(int T, int d, const double* H, int m, int overlap, int width,
                  const double* Wkv_a, const double* Wkv_b,
                  const double* Wz_a, const double* Wz_b,
                  const double* B_a, const double* B_b,
                  int i0, int i1, double* out, double* S_out);

/* RMSNorm (gain 1) then RoPE on the last rope_dims of each of n rows of
 * width c; row r sits at position pos0 + stride * r. */
void ocsa_norm_rope_rows(int n, int c, int rope_dims, double base, double eps,
                         double pos0, double stride, double* x);

/* Number of compressed entries a query at t0 may use: floor((t0+1)/m),
 * clamped to [0, N].  Reading of the causality rule of notes 2.3.2. */
int ocsa_nvis(int t0, int m, int N);

/* Lightning-indexer scores, eq. 16:
 *   scores[q][s] = sum_h w[q][h] * ReLU(qI[q][h] . KI[s])   for s < nvis[q]
 * and -inf for s >= nvis[q].  qI [Q][n_hI][c_I], w [Q][n_hI], KI [N][c_I]. */
void ocsa_index_scores(int Q, const int* nvis, int n_hI, int c_I,
                       const double* qI, const double* w, int N,
                       const double* KI, double* scores);

/* Top-k of eq. 17 over the visible scores of each query: order by
 * (score descending, index ascending), keep the first min(k, nvis), write the
 * kept indices in ascending order and pad with -1.  kth (nullable) receives
 * the score of the last kept entry in score order (-inf if none). */
void ocsa_topk(int Q, int N, const double* scores, const int* nvis, int k,
               int32_t* idx, double* kth);

/* Shared-KV MQA with window and sink (eq. 19, 26, 27) for Q queries of one
 * sequence, then R_{-t0} on the last rope_dims of every output head.
 *   t0   [Q] query positions;  q [Q][n_h][c]
 *   idx  [Q][k] selected entries (-1 = unused) or NULL for HCA (all visible)
 *   kv   [N][c] compressed entries (the KV cache, key = value)
 *   win  [W][c] uncompressed window rows, row r holding token win_pos0 + r;
 *        the query attends tokens max(0, t0-n_win+1)..t0
 *   sink [n_h] sink logits z'_h (not scaled)
 *   rope_shift is added to every RoPE position (0 in normal use)
 *   out  [Q][n_h][c]; mass (nullable) [Q][n_h] = sum of all weights incl. sink
 * Returns 0, or -1 if a window row or an index is out of range. */
int ocsa_attend(int Q, const int* t0, int n_h, int c, int rope_dims,
                double base, double scale, const double* q,
                int k, const int32_t* idx, int m, int N, const double* kv,
                int n_win, int W, int win_pos0, const double* win,
                const double* sink, double rope_shift,
                double* out, double* mass);

/* bf16 round-to-nearest-even of a double (bf16 = 8 exponent bits, 7 stored
 * mantissa bits).  Writes the rounded values as doubles. */
void ocsa_round_bf16(int n, const double* x, double* y);

/* OCP FP8 E4M3 (bias 7, no infinities, S.1111.111 = NaN, max 448).
 * decode: code -> value.  encode: float -> code, round-to-nearest-even with
 * saturation to +-448 (the decision is taken in fp32 arithmetic). */
double ocsa_e4m3_decode(uint8_t code);
uint8_t ocsa_e4m3_encode(float x);

/* Mixed KV entry format: the first c-rope_dims values are e4m3 codes times one
 * fp32 per-entry scale, the last rope_dims values are bf16.
 *   scale = max|x_j| / 448 over the fp8 part (1 if all zero), codes =
 *   encode(x_j / scale), both in fp32.  x is first rounded to fp32.
 * encode: x [n][c] -> codes [n][c-rope_dims], rope [n][rope_dims] (bf16 values
 * as double), scale [n].  decode: the inverse map into x [n][c]. */
void ocsa_fp8mix_encode(int n, int c, int rope_dims, const double* x,
                        uint8_t* codes, double* rope, float* scale);
void ocsa_fp8mix_decode(int n, int c, int rope_dims, const uint8_t* codes,
                        const uint16_t* rope_bf16_bits, const float* scale,
                        double* x);

/* Grouped output projection ([N] 2.3.3, [P] 2.2): group i of n_h / g
 * consecutive heads of O [Q][n_h][c] times WG[i] [c n_h/g][d_g] gives
 * Y[q][i d_g .. (i+1) d_g); out [Q][d] = Y WO with WO [g d_g][d].  With
 * round_mid, Y is rounded to bf16 before WO. */
void ocsa_group_out_proj(int Q, int n_h, int c, int g, int d_g, int d, const double* O,
                         const double* WG, const double* WO, int round_mid, double* Y,
                         double* out);

/* MXFP4 (OCP Microscaling): blocks of 32 sharing a power-of-two scale
 * 2^scale_exp[block] = 2^(floor(log2 max|x|) - 2); elements E2M1 (codes
 * sign << 3 | index into 0, 0.5, 1, 1.5, 2, 3, 4, 6), rounded to nearest,
 * ties to an even mantissa, saturating at 6.  PaperTrace 3.3 (the indexer's
 * QK path in MXFP4). */
double ocsa_e2m1_decode(uint8_t code);
void ocsa_mxfp4_encode(int n, const double* x, uint8_t* codes, int* scale_exp);
void ocsa_mxfp4_decode(int n, const uint8_t* codes, const int* scale_exp, double* y);

#ifdef __cplusplus
}
#endif
#endif
