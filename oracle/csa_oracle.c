/*
 * csa_oracle.c -- plain, slow CPU reference of the CSA / HCA forward pass.
 *
 * TEST INFRASTRUCTURE ONLY: used by the tests, the smoke check and the
 * CPU-baseline leg of the benchmark; never by the product path.  It shares no
 * code with the CUDA library.  All arithmetic is IEEE double unless a routine
 * says otherwise (the FP8 quantiser takes its decisions in fp32, as the stored
 * format does).  OpenMP only splits independent outer loops.
 *
 * Sources (titles of the pages, section / equation):
 *   [N]  "DeepSeekV4技术报告阅读笔记" (zouxinn.github.io), 2.3.1 eq. 9-12,
 *        2.3.2 eq. 13-17, 2.3.3 eq. 18-19, 2.4.1 eq. 20-23, 2.4.2 eq. 26,
 *        2.5.1 RMSNorm, 2.5.2 partial RoPE and R_{-t}, 2.5.3 window,
 *        2.5.4 eq. 27 attention sink; 2.3.3 grouped output projection.
 *   [P]  "02 · DeepSeek-V4: 压缩注意力撑起 1M 上下文" (PaperTrace), 2.1 (m = 4,
 *        the 2m-slot per-channel softmax), 2.3 (HCA m' = 128, no overlap),
 *        2.4 (RMSNorm, last-64 RoPE, window of n_win, sink), 2.5 (RoPE dims in
 *        BF16, other dims in FP8), 2.2 (output-projection groups, d_g).
 * Readings where the pages leave a step open are listed with each routine.
 */
#include "csa_oracle.h"

#include <math.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

int ocsa_num_threads(void) {
#ifdef _OPENMP
  return omp_get_max_threads();
#else
  return 1;
#endif
}

/* [N] 2.5.2: RoPE rotates 2-D sub-spaces by an angle proportional to the
 * position; R_n^T = R_{-n}.  Reading: interleaved pairs, theta_p =
 * base^(-2p/rope_dims). */
void ocsa_rope(double* x, int rope_dims, double base, double pos) {
  for (int p = 0; p < rope_dims / 2; ++p) {
    double theta = pow(base, -2.0 * (double)p / (double)rope_dims);
    double ang = pos * theta;
    double cs = cos(ang), sn = sin(ang);
    double x0 = x[2 * p], x1 = x[2 * p + 1];
    x[2 * p] = x0 * cs - x1 * sn;
    x[2 * p + 1] = x0 * sn + x1 * cs;
  }
}

/* [N] 2.5.1 / [P] 2.4: RMSNorm(x) = x / RMS(x) * gamma; reading: gamma = 1
 * (no trained weights) and an eps inside the root. */
void ocsa_rmsnorm(double* x, int n, double eps) {
  double ss = 0.0;
  for (int j = 0; j < n; ++j) ss += x[j] * x[j];
  double inv = 1.0 / sqrt(ss / (double)n + eps);
  for (int j = 0; j < n; ++j) x[j] *= inv;
}

/* [N] eq. 9-10, 20-21: C = H W, Z = H W (W in R^{d x width}). */
void ocsa_matmul(int rows, int d, const double* A, int width, const double* W,
                 double* out) {
#pragma omp parallel for schedule(static)
  for (int r = 0; r < rows; ++r) {
    double* o = out + (size_t)r * width;
    for (int j = 0; j < width; ++j) o[j] = 0.0;
    for (int k = 0; k < d; ++k) {
      double a = A[(size_t)r * d + k];
      const double* w = W + (size_t)k * width;
      for (int j = 0; j < width; ++j) o[j] += a * w[j];
    }
  }
}

/* [N] eq. 11-12 (CSA) and eq. 22-23 (HCA); [P] 2.1, 2.3.
 * Entry i: per channel, a softmax over the 2m logits
 *   Z^a_{mi+r} + B^a_r  (r < m)   and   Z^b_{m(i-1)+r} + B^b_r  (r < m),
 * then C^Comp_i = sum of S * C over the same 2m rows.  For i = 0 the b rows
 * have logit -inf and value 0, i.e. they drop out.  HCA: only the a rows, no
 * overlap.  Reading: the bias is m x width (the notes print "m x b"). */
int ocsa_compress(int T, int d, const double* H, int m, int overlap, int width,
                  const double* Wkv_a, const double* Wkv_b,
                  const double* Wz_a, const double* Wz_b,
                  const double* B_a, const double* B_b,
                  int i0, int i1, double* out, double* S_out) {
  if (i1 <= i0) return 0;
  if ((long)m * i1 > T || i0 < 0) return -1;
  int tok_lo = m * i0;
  if (overlap && i0 > 0) tok_lo = m * (i0 - 1);
  int tok_hi = m * i1;
  int ntok = tok_hi - tok_lo;
  size_t sz = (size_t)ntok * width;
  double* Ca = (double*)malloc(sz * sizeof(double));
  double* Za = (double*)malloc(sz * sizeof(double));
  double* Cb = overlap ? (double*)malloc(sz * sizeof(double)) : NULL;
  double* Zb = overlap ? (double*)malloc(sz * sizeof(double)) : NULL;
  const double* Hlo = H + (size_t)tok_lo * d;
  ocsa_matmul(ntok, d, Hlo, width, Wkv_a, Ca);
  ocsa_matmul(ntok, d, Hlo, width, Wz_a, Za);
  if (overlap) {
    ocsa_matmul(ntok, d, Hlo, width, Wkv_b, Cb);
    ocsa_matmul(ntok, d, Hlo, width, Wz_b, Zb);
  }
  int nslot = 2 * m;
#pragma omp parallel for schedule(static)
  for (int i = i0; i < i1; ++i) {
    double* logit = (double*)malloc((size_t)nslot * sizeof(double));
    double* val = (double*)malloc((size_t)nslot * sizeof(double));
    int* live = (int*)malloc((size_t)nslot * sizeof(int));
    for (int ch = 0; ch < width; ++ch) {
      for (int r = 0; r < m; ++r) {
        int row = m * i + r - tok_lo;
        logit[r] = Za[(size_t)row * width + ch] + B_a[(size_t)r * width + ch];
        val[r] = Ca[(size_t)row * width + ch];
        live[r] = 1;
        if (overlap && i > 0) {
          int rowb = m * (i - 1) + r - tok_lo;
          logit[m + r] = Zb[(size_t)rowb * width + ch] + B_b[(size_t)r * width + ch];
          val[m + r] = Cb[(size_t)rowb * width + ch];
          live[m + r] = 1;
        } else {
          logit[m + r] = -INFINITY;
          val[m + r] = 0.0;
          live[m + r] = 0;
        }
      }
      double mx = -INFINITY;
      for (int s = 0; s < nslot; ++s)
        if (live[s] && logit[s] > mx) mx = logit[s];
      double den = 0.0;
      for (int s = 0; s < nslot; ++s)
        if (live[s]) den += exp(logit[s] - mx);
      double acc = 0.0;
      for (int s = 0; s < nslot; ++s) {
        double S = live[s] ? exp(logit[s] - mx) / den : 0.0;
        acc += S * val[s];
        if (S_out) S_out[((size_t)(i - i0) * nslot + s) * width + ch] = S;
      }
      out[(size_t)(i - i0) * width + ch] = acc;
    }
    free(logit);
    free(val);
    free(live);
  }
  free(Ca);
  free(Za);
  free(Cb);
  free(Zb);
  return 0;
}

/* [N] 2.5.1-2.5.2: RMSNorm on the single KV head, RoPE on its last rope_dims.
 * Reading: an entry sits at the position of the first token of its a-window
 * (stride m), a window row at its own token position (stride 1). */
void ocsa_norm_rope_rows(int n, int c, int rope_dims, double base, double eps,
                         double pos0, double stride, double* x) {
#pragma omp parallel for schedule(static)
  for (int r = 0; r < n; ++r) {
    double* row = x + (size_t)r * c;
    ocsa_rmsnorm(row, c, eps);
    ocsa_rope(row + (c - rope_dims), rope_dims, base, pos0 + stride * (double)r);
  }
}

/* [N] 2.3.2, [P] 2.4: a query may only use complete compressed blocks.
 * Reading: entry s is visible at t0 iff its a-window ends at or before t0,
 * i.e. s < floor((t0+1)/m). */
int ocsa_nvis(int t0, int m, int N) {
  long v = ((long)t0 + 1) / m;
  if (t0 < 0) v = 0;
  if (v > N) v = N;
  return (int)v;
}

/* [N] eq. 16: I_{t,s} = sum_h w_{t,h} ReLU(q^I_{t,h} . K^IComp_s). */
void ocsa_index_scores(int Q, const int* nvis, int n_hI, int c_I,
                       const double* qI, const double* w, int N,
                       const double* KI, double* scores) {
#pragma omp parallel for collapse(2) schedule(static)
  for (int q = 0; q < Q; ++q) {
    for (int s = 0; s < N; ++s) {
      if (s >= nvis[q]) {
        scores[(size_t)q * N + s] = -INFINITY;
        continue;
      }
      double acc = 0.0;
      for (int h = 0; h < n_hI; ++h) {
        const double* qh = qI + ((size_t)q * n_hI + h) * c_I;
        const double* k = KI + (size_t)s * c_I;
        double dot = 0.0;
        for (int e = 0; e < c_I; ++e) dot += qh[e] * k[e];
        double relu = dot > 0.0 ? dot : 0.0;
        acc += w[(size_t)q * n_hI + h] * relu;
      }
      scores[(size_t)q * N + s] = acc;
    }
  }
}

typedef struct {
  double score;
  int s;
} scored_t;

/* score descending, then index ascending (reading: the lower index wins a
 * tie). */
static int cmp_score(const void* a, const void* b) {
  const scored_t* x = (const scored_t*)a;
  const scored_t* y = (const scored_t*)b;
  if (x->score > y->score) return -1;
  if (x->score < y->score) return 1;
  return (x->s > y->s) - (x->s < y->s);
}

static int cmp_int(const void* a, const void* b) {
  int x = *(const int32_t*)a, y = *(const int32_t*)b;
  return (x > y) - (x < y);
}

/* [N] eq. 17: keep the entries whose score is among the top k. */
void ocsa_topk(int Q, int N, const double* scores, const int* nvis, int k,
               int32_t* idx, double* kth) {
#pragma omp parallel for schedule(dynamic)
  for (int q = 0; q < Q; ++q) {
    int nv = nvis[q];
    scored_t* all = (scored_t*)malloc((size_t)(nv > 0 ? nv : 1) * sizeof(scored_t));
    for (int s = 0; s < nv; ++s) {
      all[s].score = scores[(size_t)q * N + s];
      all[s].s = s;
    }
    qsort(all, (size_t)nv, sizeof(scored_t), cmp_score);
    int keep = nv < k ? nv : k;
    int32_t* out = idx + (size_t)q * k;
    for (int j = 0; j < keep; ++j) out[j] = all[j].s;
    qsort(out, (size_t)keep, sizeof(int32_t), cmp_int);
    for (int j = keep; j < k; ++j) out[j] = -1;
    if (kth) kth[q] = keep > 0 ? all[keep - 1].score : -INFINITY;
    free(all);
  }
}

/* [N] eq. 19 / 26 (shared-KV MQA: the entry is key and value), 2.5.3 (the
 * window branch), eq. 27 (the sink adds exp(z'_h) to the denominator), 2.5.2
 * (output de-rotated by R_{-t}).  Readings: one softmax over the union of the
 * selected entries and the window tokens (no de-duplication); logits are
 * scale * q.k with scale = 1/sqrt(c) chosen by the caller; the sink logit is
 * not scaled. */
int ocsa_attend(int Q, const int* t0, int n_h, int c, int rope_dims,
                double base, double scale, const double* q,
                int k, const int32_t* idx, int m, int N, const double* kv,
                int n_win, int W, int win_pos0, const double* win,
                const double* sink, double rope_shift,
                double* out, double* mass) {
  int bad = 0;
#pragma omp parallel for collapse(2) schedule(dynamic)
  for (int qi = 0; qi < Q; ++qi) {
    for (int h = 0; h < n_h; ++h) {
      int t = t0[qi];
      int nv = ocsa_nvis(t, m, N);
      int cap = (idx ? k : nv) + (n_win > 0 ? n_win : 0);
      const double** keys = (const double**)malloc((size_t)(cap > 0 ? cap : 1) * sizeof(double*));
      int nk = 0, ok = 1;
      if (idx) {
        for (int j = 0; j < k; ++j) {
          int s = idx[(size_t)qi * k + j];
          if (s < 0) continue;
          if (s >= nv) { ok = 0; break; }
          keys[nk++] = kv + (size_t)s * c;
        }
      } else {
        for (int s = 0; s < nv; ++s) keys[nk++] = kv + (size_t)s * c;
      }
      if (ok && n_win > 0) {
        int lo = t - n_win + 1;
        if (lo < 0) lo = 0;
        for (int tok = lo; tok <= t; ++tok) {
          int r = tok - win_pos0;
          if (r < 0 || r >= W) { ok = 0; break; }
          keys[nk++] = win + (size_t)r * c;
        }
      }
      double* o = out + ((size_t)qi * n_h + h) * c;
      if (!ok) {
#pragma omp atomic write
        bad = 1;
        for (int e = 0; e < c; ++e) o[e] = NAN;
        free(keys);
        continue;
      }
      const double* qh = q + ((size_t)qi * n_h + h) * c;
      double* z = (double*)malloc((size_t)(nk > 0 ? nk : 1) * sizeof(double));
      double mx = sink[h];
      for (int j = 0; j < nk; ++j) {
        double dot = 0.0;
        for (int e = 0; e < c; ++e) dot += qh[e] * keys[j][e];
        z[j] = scale * dot;
        if (z[j] > mx) mx = z[j];
      }
      double den = exp(sink[h] - mx);
      for (int j = 0; j < nk; ++j) den += exp(z[j] - mx);
      for (int e = 0; e < c; ++e) o[e] = 0.0;
      double msum = exp(sink[h] - mx) / den;
      for (int j = 0; j < nk; ++j) {
        double p = exp(z[j] - mx) / den;
        msum += p;
        for (int e = 0; e < c; ++e) o[e] += p * keys[j][e];
      }
      ocsa_rope(o + (c - rope_dims), rope_dims, base, -((double)t + rope_shift));
      if (mass) mass[(size_t)qi * n_h + h] = msum;
      free(z);
      free(keys);
    }
  }
  return bad ? -1 : 0;
}

/* bf16: sign, 8 exponent bits (bias 127), 7 stored mantissa bits; values are
 * rounded to the nearest representable one, ties to an even mantissa. */
void ocsa_round_bf16(int n, const double* x, double* y) {
  for (int i = 0; i < n; ++i) {
    double v = x[i];
    if (v == 0.0 || !isfinite(v)) { y[i] = v; continue; }
    int e;
    frexp(fabs(v), &e); /* |v| = f * 2^e, f in [0.5, 1) */
    int E = e - 1;      /* floor(log2 |v|) */
    if (E < -126) E = -126; /* subnormal range shares the minimum exponent */
    double quantum = ldexp(1.0, E - 7);
    double r = nearbyint(fabs(v) / quantum); /* default mode: ties to even */
    y[i] = copysign(r * quantum, v);
  }
}

/* OCP 8-bit floating point, E4M3: 1 sign, 4 exponent (bias 7), 3 mantissa
 * bits; exponent field 0 is subnormal (mantissa * 2^-9); S.1111.111 is NaN;
 * no infinities; the largest finite magnitude is 1.75 * 2^8 = 448. */
double ocsa_e4m3_decode(uint8_t code) {
  int sgn = code >> 7, e = (code >> 3) & 0xF, mant = code & 7;
  double v;
  if (e == 15 && mant == 7) return NAN;
  if (e == 0) v = ldexp((double)mant, -9);
  else v = ldexp(1.0 + mant / 8.0, e - 7);
  return sgn ? -v : v;
}

uint8_t ocsa_e4m3_encode(float x) {
  if (isnan(x)) return 0x7F;
  uint8_t sgn = signbit(x) ? 0x80 : 0;
  float a = fabsf(x);
  if (a >= 448.0f) return sgn | 0x7E; /* saturate to the largest finite */
  int e;
  frexpf(a, &e);
  int E = e - 1;
  if (a == 0.0f || E < -6) E = -6; /* subnormals use the quantum 2^-9 */
  float quantum = ldexpf(1.0f, E - 3);
  float r = nearbyintf(a / quantum); /* exact scaling, ties to even */
  float v = r * quantum;             /* may step up to the next binade */
  if (v >= 448.0f) return sgn | 0x7E;
  if (v == 0.0f) return sgn;
  int ev;
  frexpf(v, &ev);
  int Ev = ev - 1;
  if (Ev < -6) { /* subnormal: v = mant * 2^-9 */
    int mant = (int)(v / ldexpf(1.0f, -9));
    return sgn | (uint8_t)mant;
  }
  int mant = (int)((v / ldexpf(1.0f, Ev) - 1.0f) * 8.0f);
  return sgn | (uint8_t)(((Ev + 7) << 3) | mant);
}

/* [P] 2.5: RoPE dims kept in BF16, the other dims in FP8.  Readings: E4M3,
 * one fp32 scale per entry = max|x| / 448 over the FP8 dims (1 if all zero),
 * round-to-nearest-even with saturation, decisions in fp32. */
void ocsa_fp8mix_encode(int n, int c, int rope_dims, const double* x,
                        uint8_t* codes, double* rope, float* scale) {
  int nf = c - rope_dims;
  for (int r = 0; r < n; ++r) {
    const double* row = x + (size_t)r * c;
    float amax = 0.0f;
    for (int j = 0; j < nf; ++j) {
      float v = fabsf((float)row[j]);
      if (v > amax) amax = v;
    }
    float s = amax > 0.0f ? amax / 448.0f : 1.0f;
    scale[r] = s;
    for (int j = 0; j < nf; ++j)
      codes[(size_t)r * nf + j] = ocsa_e4m3_encode((float)row[j] / s);
    ocsa_round_bf16(rope_dims, row + nf, rope + (size_t)r * rope_dims);
  }
}

void ocsa_fp8mix_decode(int n, int c, int rope_dims, const uint8_t* codes,
                        const uint16_t* rope_bf16_bits, const float* scale,
                        double* x) {
  int nf = c - rope_dims;
  for (int r = 0; r < n; ++r) {
    double* row = x + (size_t)r * c;
    for (int j = 0; j < nf; ++j)
      row[j] = ocsa_e4m3_decode(codes[(size_t)r * nf + j]) * (double)scale[r];
    for (int j = 0; j < rope_dims; ++j) {
      uint32_t bits = (uint32_t)rope_bf16_bits[(size_t)r * rope_dims + j] << 16;
      float f;
      memcpy(&f, &bits, sizeof f);
      row[nf + j] = (double)f;
    }
  }
}

/* [N] 2.3.3 "Grouped Output Projection"; [P] 2.2.  The attention output o_t
 * (n_h heads of c values) is cut into g groups of n_h / g consecutive heads;
 * group i (c n_h / g values) times W^G_i ((c n_h / g) x d_g) gives o'_i
 * (d_g values); the concatenation [o'_1; ...; o'_g] (g d_g values) times W^O
 * ((g d_g) x d) gives the layer output (d values).  Reading: consecutive
 * heads form a group; with round_mid the group outputs are rounded to bf16
 * before W^O, as a bf16 model stores the activation between the two
 * projections.
 *   O   [Q][n_h][c]       WG [g][c n_h / g][d_g]       WO [g d_g][d]
 *   Y   [Q][g d_g] (the group outputs, after rounding when asked)
 *   out [Q][d] */
void ocsa_group_out_proj(int Q, int n_h, int c, int g, int d_g, int d, const double* O,
                         const double* WG, const double* WO, int round_mid, double* Y,
                         double* out) {
  const int Kg = c * (n_h / g);
#pragma omp parallel for schedule(static)
  for (int q = 0; q < Q; ++q) {
    const double* o = O + (size_t)q * n_h * c;
    double* y = Y + (size_t)q * g * d_g;
    for (int i = 0; i < g; ++i) {
      const double* oi = o + (size_t)i * Kg;  /* heads i n_h/g .. (i+1) n_h/g - 1 */
      const double* wi = WG + (size_t)i * Kg * d_g;
      double* yi = y + (size_t)i * d_g;
      for (int j = 0; j < d_g; ++j) yi[j] = 0.0;
      for (int k = 0; k < Kg; ++k) {
        const double a = oi[k];
        const double* w = wi + (size_t)k * d_g;
        for (int j = 0; j < d_g; ++j) yi[j] += a * w[j];
      }
    }
    if (round_mid) ocsa_round_bf16(g * d_g, y, y);
    double* r = out + (size_t)q * d;
    for (int j = 0; j < d; ++j) r[j] = 0.0;
    for (int k = 0; k < g * d_g; ++k) {
      const double a = y[k];
      const double* w = WO + (size_t)k * d;
      for (int j = 0; j < d; ++j) r[j] += a * w[j];
    }
  }
}

/* PaperTrace 3.3 ("FP4 (MXFP4) quantization-aware training ... the CSA
 * indexer's QK path"): MXFP4 as the OCP Microscaling (MX) formats define it:
 * blocks of 32 elements share one power-of-two scale (E8M0: 2^e, e in
 * [-127, 127]); each element is FP4 E2M1 (1 sign, 2 exponent bits with bias
 * 1, 1 mantissa bit; no infinities or NaN): magnitudes 0, 0.5, 1, 1.5, 2, 3,
 * 4, 6.  Code = sign << 3 | magnitude index.  The block scale is
 * 2^(floor(log2 max|x|) - 2) (2 = the exponent of E2M1's largest normal);
 * elements are x / scale rounded to the nearest E2M1 value, ties to an even
 * mantissa, saturating at 6. */
double ocsa_e2m1_decode(uint8_t code) {
  static const double mag[8] = {0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0};
  const double v = mag[code & 7];
  return (code & 8) ? -v : v;
}

static uint8_t e2m1_encode(double v) {
  const double a = fabs(v);
  /* grid spacing of the binade: 0.5 below 2, 1 in [2, 4), 2 from 4 on */
  const double step = a < 2.0 ? 0.5 : (a < 4.0 ? 1.0 : 2.0);
  double q = nearbyint(a / step) * step; /* ties to even multiples: even mantissa */
  if (q > 6.0) q = 6.0;
  static const double mag[8] = {0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0};
  uint8_t m = 0;
  for (uint8_t i = 0; i < 8; ++i)
    if (mag[i] == q) m = i;
  return (uint8_t)((v < 0.0 && q > 0.0 ? 8 : 0) | m);
}

void ocsa_mxfp4_encode(int n, const double* x, uint8_t* codes, int* scale_exp) {
  for (int b0 = 0; b0 < n; b0 += 32) {
    const int nb = n - b0 < 32 ? n - b0 : 32;
    double amax = 0.0;
    for (int i = 0; i < nb; ++i) amax = fmax(amax, fabs(x[b0 + i]));
    int e = -127;
    if (amax > 0.0) {
      int ex;
      frexp(amax, &ex); /* amax = f 2^ex, f in [0.5, 1) */
      e = (ex - 1) - 2;
      if (e < -127) e = -127;
      if (e > 127) e = 127;
    }
    scale_exp[b0 / 32] = e;
    for (int i = 0; i < nb; ++i) codes[b0 + i] = e2m1_encode(ldexp(x[b0 + i], -e));
  }
}

void ocsa_mxfp4_decode(int n, const uint8_t* codes, const int* scale_exp, double* y) {
  for (int i = 0; i < n; ++i) y[i] = ldexp(ocsa_e2m1_decode(codes[i]), scale_exp[i / 32]);
}

