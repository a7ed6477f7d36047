/*
 * qwm_oracle.c -- plain, slow CPU oracle for the QuantWM 2-bit KV-cache path.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the test suite, the smoke check and the CPU
 * baseline leg of the benchmark load this file's library; the product path
 * (the CUDA library and its Python binding) never calls it and shares no code
 * with it.
 *
 * Sources (QuantWM: Temporally Consistent 2-Bit KV Cache Quantization for Video
 * World Models; all pages are secondary reports of the paper):
 *   [SP-en]  "Flickering after quantization? A temporally stable 2-bit KV Cache
 *            compression framework for video world models emerges"
 *            (SynthePulse, en-US), paragraphs on QSAC and PSAC.
 *   [REV]    "QuantWM: Temporally Consistent 2-Bit KV Cache Quantization for
 *            World Models and Video Generation" (evolve.pub review), Summary and
 *            Strengths (Eq. 7: E[(q^T e)^2] = e^T M e; Fig. 4; Table 9, 10).
 *   [ABS]    the paper's abstract (HF Daily Papers mirror): QSAC selects
 *            "INT2-friendly Key centroids", PSAC restores Key error along the
 *            dominant Query subspace with low-rank projections.
 *
 * Precision.  Where floating point decides an integer (centroid choice, INT2
 * code, INT8 coefficient) the oracle uses the kernel's precision: IEEE fp32,
 * round-to-nearest-even, every sum a left-to-right fold starting at +0.0f with
 * the stated operation (fmaf where the spec says fma).  Build with
 * -ffp-contract=off so the compiler adds no fusion of its own.  Everything
 * else (query statistics, eigenvectors, k-means means, reconstruction and
 * attention) is fp64.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define QO_API __attribute__((visibility("default")))

/* ------------------------------------------------------------------------- */
/* Number formats (IEEE 754 binary16 and bfloat16), written from the format  */
/* definitions: value = (-1)^s * 2^E * significand.                            */
/* ------------------------------------------------------------------------- */

enum { QO_RN = 0, QO_RD = 1, QO_RU = 2 };

QO_API float qo_f16_to_f32(uint16_t h) {
  int s = h >> 15, e = (h >> 10) & 31, m = h & 1023;
  double v;
  if (e == 0) v = ldexp((double)m, -24);
  else if (e == 31) v = m ? NAN : INFINITY;
  else v = ldexp((double)(1024 + m), e - 25);
  return (float)(s ? -v : v);
}

/* Round an fp32 value to binary16 in direction `mode` (RN ties-even, RD toward
 * -inf, RU toward +inf).  Works on the exact value in double: the binary16 grid
 * spacing at |x| is 2^(E-10) for normal numbers and 2^-24 below 2^-14. */
QO_API uint16_t qo_f32_to_f16(float x, int mode) {
  if (isnan(x)) return 0x7e00;
  int neg = signbit(x) ? 1 : 0;
  uint16_t sbit = neg ? 0x8000 : 0;
  if (isinf(x)) return sbit | 0x7c00;
  double a = fabs((double)x);
  if (a == 0.0) return sbit;
  /* magnitude rounding: 0 = toward zero, 1 = away from zero, 2 = nearest-even */
  int dir = (mode == QO_RN) ? 2 : (mode == QO_RD) ? (neg ? 1 : 0) : (neg ? 0 : 1);
  int e2;
  frexp(a, &e2);            /* a in [2^(e2-1), 2^e2) */
  int E = e2 - 1;
  if (E < -14) E = -14;
  double quantum = ldexp(1.0, E - 10);
  double q = a / quantum;   /* exact: power-of-two scaling */
  double qi;
  if (dir == 0) qi = floor(q);
  else if (dir == 1) qi = ceil(q);
  else {
    qi = floor(q);
    double frac = q - qi;
    if (frac > 0.5 || (frac == 0.5 && fmod(qi, 2.0) != 0.0)) qi += 1.0;
  }
  double val = qi * quantum;
  if (val > 65504.0) return (dir == 0) ? (sbit | 0x7bff) : (sbit | 0x7c00);
  if (val == 0.0) return sbit;
  if (val < ldexp(1.0, -14)) return sbit | (uint16_t)(val / ldexp(1.0, -24));
  int ev;
  frexp(val, &ev);
  int Ev = ev - 1;
  uint16_t mant = (uint16_t)(val / ldexp(1.0, Ev - 10) - 1024.0);
  return sbit | (uint16_t)((Ev + 15) << 10) | mant;
}

QO_API float qo_bf16_to_f32(uint16_t b) {
  uint32_t u = (uint32_t)b << 16;
  float f;
  memcpy(&f, &u, 4);
  return f;
}

/* Round a double to bfloat16 (nearest, ties to even): 8 significant bits,
 * exponent range of fp32 (subnormal spacing 2^-133). */
QO_API uint16_t qo_f64_to_bf16(double x) {
  if (isnan(x)) return 0x7fc0;
  int neg = signbit(x) ? 1 : 0;
  uint16_t sbit = neg ? 0x8000 : 0;
  if (isinf(x)) return sbit | 0x7f80;
  double a = fabs(x);
  if (a == 0.0) return sbit;
  int e2;
  frexp(a, &e2);
  int E = e2 - 1;
  if (E < -126) E = -126;
  double quantum = ldexp(1.0, E - 7);
  double q = a / quantum;
  double qi = floor(q);
  double frac = q - qi;
  if (frac > 0.5 || (frac == 0.5 && fmod(qi, 2.0) != 0.0)) qi += 1.0;
  double val = qi * quantum;
  if (val >= ldexp(1.0, 128)) return sbit | 0x7f80;
  float f = (float)val; /* exact: val is on the bf16 grid */
  uint32_t u;
  memcpy(&u, &f, 4);
  return sbit | (uint16_t)((u >> 16) & 0x7fff);
}

QO_API uint16_t qo_f32_to_bf16(float x) { return qo_f64_to_bf16((double)x); }

static inline float bf(uint16_t b) { return qo_bf16_to_f32(b); }

/* ------------------------------------------------------------------------- */
/* Distances (the canonical fp32 folds).                                      */
/* ------------------------------------------------------------------------- */

/* Query-sensitivity-weighted distance of key k to centroid c [SP-en, QSAC:
 * "Query-sensitivity-weighted distance to screen candidate centers"]:
 *   D = sum_j s_j (k_j - c_j)^2, folded over j = 0..d-1 as
 *   acc = fmaf(s_j, delta_j * delta_j, acc), delta_j = k_j - c_j (fp32). */
QO_API float qo_weighted_dist(const uint16_t* k, const uint16_t* c, const float* s, int d) {
  float acc = 0.0f;
  for (int j = 0; j < d; ++j) {
    float dl = bf(k[j]) - bf(c[j]);
    float p = dl * dl;
    acc = fmaf(s[j], p, acc);
  }
  return acc;
}

/* Plain squared Euclidean distance of a bf16 row to an fp32 point:
 * acc = fmaf(delta_j, delta_j, acc) over j.  Used for Value assignment
 * (nearest centroid) and for the k-means assignment step. */
QO_API float qo_sq_dist_f32c(const uint16_t* x, const float* c, int d) {
  float acc = 0.0f;
  for (int j = 0; j < d; ++j) {
    float dl = bf(x[j]) - c[j];
    acc = fmaf(dl, dl, acc);
  }
  return acc;
}

static float sq_dist_bf(const uint16_t* x, const uint16_t* c, int d) {
  float acc = 0.0f;
  for (int j = 0; j < d; ++j) {
    float dl = bf(x[j]) - bf(c[j]);
    acc = fmaf(dl, dl, acc);
  }
  return acc;
}

/* ------------------------------------------------------------------------- */
/* k-means (Lloyd) for the centroid tables.                                   */
/* The pages only say each Key "is assigned to a cluster center" whose value  */
/* is kept at higher precision [SP-en, QSAC].  Reading: strided init (centroid */
/* i starts at token floor(i*n/C)), `iters` Lloyd rounds (assign with fp32     */
/* squared distance, ties to the lower index; mean in fp64, rounded to fp32;   */
/* an empty cluster keeps its centroid), final centroids rounded to bf16.      */
/* ------------------------------------------------------------------------- */
QO_API int qo_kmeans(const uint16_t* X, int64_t n, int d, int64_t stride, int C, int iters,
                     uint16_t* cent_out, int32_t* assign_out) {
  if (n <= 0 || C <= 0 || d <= 0) return -1;
  float* cent = (float*)malloc(sizeof(float) * (size_t)C * d);
  double* sum = (double*)malloc(sizeof(double) * (size_t)C * d);
  int64_t* cnt = (int64_t*)malloc(sizeof(int64_t) * (size_t)C);
  int32_t* asg = (int32_t*)malloc(sizeof(int32_t) * (size_t)n);
  if (!cent || !sum || !cnt || !asg) { free(cent); free(sum); free(cnt); free(asg); return -2; }
  for (int i = 0; i < C; ++i) {
    int64_t t = (int64_t)(((__int128)i * n) / C);
    for (int j = 0; j < d; ++j) cent[(size_t)i * d + j] = bf(X[t * stride + j]);
  }
  for (int it = 0; it < iters; ++it) {
    for (int64_t t = 0; t < n; ++t) {
      const uint16_t* x = X + t * stride;
      int best = 0;
      float bd = qo_sq_dist_f32c(x, cent, d);
      for (int i = 1; i < C; ++i) {
        float dd = qo_sq_dist_f32c(x, cent + (size_t)i * d, d);
        if (dd < bd) { bd = dd; best = i; }
      }
      asg[t] = best;
    }
    memset(sum, 0, sizeof(double) * (size_t)C * d);
    memset(cnt, 0, sizeof(int64_t) * (size_t)C);
    for (int64_t t = 0; t < n; ++t) {
      const uint16_t* x = X + t * stride;
      int a = asg[t];
      cnt[a] += 1;
      for (int j = 0; j < d; ++j) sum[(size_t)a * d + j] += (double)bf(x[j]);
    }
    for (int i = 0; i < C; ++i) {
      if (cnt[i] == 0) continue;
      for (int j = 0; j < d; ++j)
        cent[(size_t)i * d + j] = (float)(sum[(size_t)i * d + j] / (double)cnt[i]);
    }
  }
  for (size_t i = 0; i < (size_t)C * d; ++i) cent_out[i] = qo_f32_to_bf16(cent[i]);
  if (assign_out) memcpy(assign_out, asg, sizeof(int32_t) * (size_t)n);
  free(cent); free(sum); free(cnt); free(asg);
  return 0;
}

/* ------------------------------------------------------------------------- */
/* Historical Query second moment and its principal subspace.                 */
/* [REV, Summary/Strengths]: QSAC uses historical Query second-moment          */
/* statistics (diagonal), PSAC the top-8 principal Query directions; both come */
/* from E[(q^T e)^2] = e^T M e (Eq. 7) with M = E[q q^T] (uncentred).          */
/* ------------------------------------------------------------------------- */

/* M += sum_t q_t q_t^T (fp64, d x d row-major), q rows bf16 with `stride`. */
QO_API void qo_stats_accumulate(const uint16_t* Q, int64_t n, int d, int64_t stride, double* M) {
  double* q = (double*)malloc(sizeof(double) * d);
  for (int64_t t = 0; t < n; ++t) {
    for (int j = 0; j < d; ++j) q[j] = (double)bf(Q[t * stride + j]);
    for (int i = 0; i < d; ++i)
      for (int j = 0; j < d; ++j) M[(size_t)i * d + j] += q[i] * q[j];
  }
  free(q);
}

/* Cyclic Jacobi eigen-decomposition of a symmetric d x d matrix (fp64).
 * Returns eigenvalues in descending order and eigenvectors as the columns of
 * `evecs` (row-major d x d), each column's sign chosen so that its entry of
 * largest magnitude (lowest index on ties) is positive.  Returns sweeps used. */
QO_API int qo_eigh_jacobi(const double* A_in, int d, double* evals, double* evecs) {
  double* A = (double*)malloc(sizeof(double) * (size_t)d * d);
  double* V = (double*)malloc(sizeof(double) * (size_t)d * d);
  memcpy(A, A_in, sizeof(double) * (size_t)d * d);
  for (int i = 0; i < d; ++i)
    for (int j = 0; j < d; ++j) V[(size_t)i * d + j] = (i == j) ? 1.0 : 0.0;
  double fro = 0.0;
  for (size_t i = 0; i < (size_t)d * d; ++i) fro += A[i] * A[i];
  fro = sqrt(fro);
  int sweep = 0;
  for (; sweep < 100; ++sweep) {
    double off = 0.0;
    for (int p = 0; p < d; ++p)
      for (int q = p + 1; q < d; ++q) off += A[(size_t)p * d + q] * A[(size_t)p * d + q];
    if (sqrt(2.0 * off) <= 1e-15 * fro || fro == 0.0) break;
    for (int p = 0; p < d - 1; ++p) {
      for (int q = p + 1; q < d; ++q) {
        double apq = A[(size_t)p * d + q];
        if (apq == 0.0) continue;
        double app = A[(size_t)p * d + p], aqq = A[(size_t)q * d + q];
        /* rotation angle that zeroes a_pq: tan(2 theta) = 2 a_pq / (a_qq - a_pp) */
        double tau = (aqq - app) / (2.0 * apq);
        double t = (tau >= 0.0 ? 1.0 : -1.0) / (fabs(tau) + sqrt(1.0 + tau * tau));
        double c = 1.0 / sqrt(1.0 + t * t), s = t * c;
        for (int k = 0; k < d; ++k) { /* A <- A J (columns p, q) */
          double akp = A[(size_t)k * d + p], akq = A[(size_t)k * d + q];
          A[(size_t)k * d + p] = c * akp - s * akq;
          A[(size_t)k * d + q] = s * akp + c * akq;
        }
        for (int k = 0; k < d; ++k) { /* A <- J^T A (rows p, q) */
          double apk = A[(size_t)p * d + k], aqk = A[(size_t)q * d + k];
          A[(size_t)p * d + k] = c * apk - s * aqk;
          A[(size_t)q * d + k] = s * apk + c * aqk;
        }
        for (int k = 0; k < d; ++k) { /* V <- V J */
          double vkp = V[(size_t)k * d + p], vkq = V[(size_t)k * d + q];
          V[(size_t)k * d + p] = c * vkp - s * vkq;
          V[(size_t)k * d + q] = s * vkp + c * vkq;
        }
      }
    }
  }
  /* sort descending (selection sort on indices; stable for equal values) */
  int* ord = (int*)malloc(sizeof(int) * d);
  for (int i = 0; i < d; ++i) ord[i] = i;
  for (int i = 0; i < d; ++i) {
    int b = i;
    for (int j = i + 1; j < d; ++j)
      if (A[(size_t)ord[j] * d + ord[j]] > A[(size_t)ord[b] * d + ord[b]]) b = j;
    int tmp = ord[i]; ord[i] = ord[b]; ord[b] = tmp;
  }
  for (int k = 0; k < d; ++k) {
    int src = ord[k];
    evals[k] = A[(size_t)src * d + src];
    int arg = 0;
    double big = -1.0;
    for (int i = 0; i < d; ++i) {
      double m = fabs(V[(size_t)i * d + src]);
      if (m > big) { big = m; arg = i; }
    }
    double sg = V[(size_t)arg * d + src] < 0.0 ? -1.0 : 1.0;
    for (int i = 0; i < d; ++i) evecs[(size_t)i * d + k] = sg * V[(size_t)i * d + src];
  }
  free(ord); free(A); free(V);
  return sweep;
}

/* Refresh the statistics QSAC and PSAC read, from M (sum of q q^T) and n:
 *   s_j = M_jj / n                      (fp64 divide, rounded to fp32)
 *   U   = top-r eigenvectors of M / n   (fp64 Jacobi, rounded to fp32), d x r
 *   w_g = sum_{j in group g} s_j        (fp32 fold over the group's channels)
 * With n == 0 there is no history: s = 1 and U = 0 (PSAC does nothing). */
QO_API void qo_refresh(const double* M, int64_t n, int d, int r, int G, float* s, float* w,
                       float* U, double* evals_out) {
  if (n <= 0) {
    for (int j = 0; j < d; ++j) s[j] = 1.0f;
    for (int i = 0; i < d * r; ++i) U[i] = 0.0f;
    if (evals_out) for (int j = 0; j < d; ++j) evals_out[j] = 0.0;
  } else {
    double* A = (double*)malloc(sizeof(double) * (size_t)d * d);
    double* ev = (double*)malloc(sizeof(double) * d);
    double* V = (double*)malloc(sizeof(double) * (size_t)d * d);
    for (size_t i = 0; i < (size_t)d * d; ++i) A[i] = M[i] / (double)n;
    for (int j = 0; j < d; ++j) s[j] = (float)(M[(size_t)j * d + j] / (double)n);
    qo_eigh_jacobi(A, d, ev, V);
    for (int i = 0; i < d; ++i)
      for (int k = 0; k < r; ++k) U[(size_t)i * r + k] = (float)V[(size_t)i * d + k];
    if (evals_out) memcpy(evals_out, ev, sizeof(double) * d);
    free(A); free(ev); free(V);
  }
  for (int g = 0; g < d / G; ++g) {
    float acc = 0.0f;
    for (int j = g * G; j < (g + 1) * G; ++j) acc = acc + s[j];
    w[g] = acc;
  }
}

/* ------------------------------------------------------------------------- */
/* INT2 residual quantization [SP-en, QSAC: "the residual between the two is  */
/* quantized to 2-bit"].  Groups of G contiguous channels; per group           */
/*   mn = fp16_RD(min rho), sc = fp16_RU((max rho - mn) / 3)  (fp32 sub, div)   */
/*   code_j = #{k in 0..2 : rho_j >= mn + (k + 0.5) sc}  (0 when sc == 0)       */
/* so deq = mn + code * sc with |rho - deq| <= sc/2.  Four codes per byte,     */
/* channel j in bits 2*(j%4) of byte j/4.  params = {mn, sc} fp16 per group.   */
/* ------------------------------------------------------------------------- */
QO_API void qo_int2_encode(const float* rho, int d, int G, uint8_t* codes, uint16_t* params) {
  memset(codes, 0, (size_t)d / 4);
  for (int g = 0; g < d / G; ++g) {
    float lo = rho[g * G], hi = rho[g * G];
    for (int j = g * G + 1; j < (g + 1) * G; ++j) {
      lo = fminf(lo, rho[j]);
      hi = fmaxf(hi, rho[j]);
    }
    if (lo == 0.0f) lo = 0.0f; /* zeros enter as +0 (never -0), so the fp16 */
    if (hi == 0.0f) hi = 0.0f; /* parameters of an all-zero group are +0    */
    uint16_t mnh = qo_f32_to_f16(lo, QO_RD);
    float mn = qo_f16_to_f32(mnh);
    uint16_t sch = qo_f32_to_f16((hi - mn) / 3.0f, QO_RU);
    float sc = qo_f16_to_f32(sch);
    params[2 * g] = mnh;
    params[2 * g + 1] = sch;
    for (int j = g * G; j < (g + 1) * G; ++j) {
      int code = 0;
      if (sc != 0.0f) {
        for (int k = 0; k < 3; ++k)
          if (rho[j] >= mn + ((float)k + 0.5f) * sc) code += 1;
      }
      codes[j / 4] |= (uint8_t)(code << (2 * (j % 4)));
    }
  }
}

/* deq_j = fmaf(code_j, sc_g, mn_g) in fp32 */
QO_API void qo_int2_decode(const uint8_t* codes, const uint16_t* params, int d, int G, float* out) {
  for (int j = 0; j < d; ++j) {
    int g = j / G;
    int code = (codes[j / 4] >> (2 * (j % 4))) & 3;
    out[j] = fmaf((float)code, qo_f16_to_f32(params[2 * g + 1]), qo_f16_to_f32(params[2 * g]));
  }
}

/* ------------------------------------------------------------------------- */
/* QSAC: two-stage centroid choice for one Key [SP-en, QSAC; REV, Summary].    */
/* Stage 1 keeps the M centroids with the smallest (D_i, i), D the weighted    */
/* distance.  Stage 2 scores each candidate by the expected squared logit      */
/* perturbation of its INT2 residual, sum_g sum_{j in g} s_j step_g^2 / 12     */
/* with step_g = range_g / 3; computed without the constant 1/108 as           */
/*   score = fold_g fmaf(w_g, R_g * R_g, acc),  R_g = max - min of the fp32     */
/* residual over group g.  The lowest score wins; ties go to the earlier       */
/* shortlist position.                                                          */
/* ------------------------------------------------------------------------- */

/* stage 1: returns the shortlist (ascending (D, i)) in cand[0..M-1]; D[] optional */
QO_API void qo_qsac_shortlist(const uint16_t* k, const uint16_t* CK, int C, int d, const float* s,
                              int M, int32_t* cand, float* D_out) {
  float* D = (float*)malloc(sizeof(float) * C);
  for (int i = 0; i < C; ++i) D[i] = qo_weighted_dist(k, CK + (size_t)i * d, s, d);
  /* M passes of "smallest remaining (D, i)" */
  char* taken = (char*)calloc(C, 1);
  for (int m = 0; m < M; ++m) {
    int best = -1;
    for (int i = 0; i < C; ++i) {
      if (taken[i]) continue;
      if (best < 0 || D[i] < D[best]) best = i;
    }
    cand[m] = best;
    taken[best] = 1;
  }
  if (D_out) memcpy(D_out, D, sizeof(float) * C);
  free(D); free(taken);
}

QO_API float qo_qsac_score(const uint16_t* k, const uint16_t* c, const float* w, int d, int G) {
  float acc = 0.0f;
  for (int g = 0; g < d / G; ++g) {
    float lo = bf(k[g * G]) - bf(c[g * G]), hi = lo;
    for (int j = g * G + 1; j < (g + 1) * G; ++j) {
      float r = bf(k[j]) - bf(c[j]);
      lo = fminf(lo, r);
      hi = fmaxf(hi, r);
    }
    float R = hi - lo;
    acc = fmaf(w[g], R * R, acc);
  }
  return acc;
}

/* QSAC stage 2 with the full quadratic form (Eq. 7 with all of M; evolve.pub
 * review, Strengths, Table 10): the Key error the candidate c leaves after
 * INT2, e = k - (c + deq(INT2(k - c))), scored as e^T A e with A = fp32(M / n)
 * [d][d] in force; y_i = fold_j fmaf(A_ij, e_j), then fold_i fmaf(e_i, y_i). */
QO_API float qo_qsac_score_full(const uint16_t* k, const uint16_t* c, const float* A, int d,
                                int G) {
  float rho[512] = {0.0f}, deq[512], e[512];
  uint8_t codes[128];
  uint16_t params[64];
  for (int j = 0; j < d; ++j) rho[j] = bf(k[j]) - bf(c[j]);
  qo_int2_encode(rho, d, G, codes, params);
  qo_int2_decode(codes, params, d, G, deq);
  for (int j = 0; j < d; ++j) e[j] = bf(k[j]) - (bf(c[j]) + deq[j]);
  float score = 0.0f;
  for (int i = 0; i < d; ++i) {
    float y = 0.0f;
    for (int j = 0; j < d; ++j) y = fmaf(A[(size_t)i * d + j], e[j], y);
    score = fmaf(e[i], y, score);
  }
  return score;
}

/* full key encoding for one token-head.
 * PSAC [SP-en, PSAC; REV, Summary]: e = k - K_hat with K_hat = C[a] + deq(rho);
 * c_r = fold_j fmaf(U_jr, e_j, acc); cs = fp16_RU(max_r |c_r| / 127);
 * c8_r = rint_even(c_r / cs) clamped to [-127, 127] (0 when cs == 0). */
QO_API void qo_encode_key(const uint16_t* k, const uint16_t* CK, int C, int d, int G, int M,
                          const float* s, const float* w, const float* U, int r,
                          int32_t* idx, uint8_t* codes, uint16_t* params, int8_t* coef,
                          uint16_t* cscale, int32_t* shortlist_out, const float* Afull) {
  int32_t cand[64];
  qo_qsac_shortlist(k, CK, C, d, s, M, cand, NULL);
  int best = 0;
  /* stage 2 only ranks a shortlist of two or more */
  if (M > 1) {
    float bscore = Afull ? qo_qsac_score_full(k, CK + (size_t)cand[0] * d, Afull, d, G)
                         : qo_qsac_score(k, CK + (size_t)cand[0] * d, w, d, G);
    for (int m = 1; m < M; ++m) {
      float sc = Afull ? qo_qsac_score_full(k, CK + (size_t)cand[m] * d, Afull, d, G)
                       : qo_qsac_score(k, CK + (size_t)cand[m] * d, w, d, G);
      if (sc < bscore) { bscore = sc; best = m; }
    }
  }
  int a = cand[best];
  *idx = a;
  if (shortlist_out) memcpy(shortlist_out, cand, sizeof(int32_t) * M);
  float rho[512], deq[512], e[512];
  const uint16_t* c = CK + (size_t)a * d;
  for (int j = 0; j < d; ++j) rho[j] = bf(k[j]) - bf(c[j]);
  qo_int2_encode(rho, d, G, codes, params);
  qo_int2_decode(codes, params, d, G, deq);
  for (int j = 0; j < d; ++j) {
    float khat = bf(c[j]) + deq[j];
    e[j] = bf(k[j]) - khat;
  }
  float cf[64];
  float amax = 0.0f;
  for (int q = 0; q < r; ++q) {
    float acc = 0.0f;
    for (int j = 0; j < d; ++j) acc = fmaf(U[(size_t)j * r + q], e[j], acc);
    cf[q] = acc;
    amax = fmaxf(amax, fabsf(acc));
  }
  uint16_t csh = qo_f32_to_f16(amax / 127.0f, QO_RU);
  float cs = qo_f16_to_f32(csh);
  *cscale = csh;
  for (int q = 0; q < r; ++q) {
    if (cs == 0.0f) { coef[q] = 0; continue; }
    float v = rintf(cf[q] / cs); /* default rounding mode: nearest, ties to even */
    if (v > 127.0f) v = 127.0f;
    if (v < -127.0f) v = -127.0f;
    coef[q] = (int8_t)v;
  }
}

/* Value encoding: nearest centroid (plain squared distance, ties to the lower
 * index) and the same INT2 residual code, no compensation term. */
QO_API void qo_encode_value(const uint16_t* v, const uint16_t* CV, int C, int d, int G,
                            int32_t* idx, uint8_t* codes, uint16_t* params) {
  int best = 0;
  float bd = sq_dist_bf(v, CV, d);
  for (int i = 1; i < C; ++i) {
    float dd = sq_dist_bf(v, CV + (size_t)i * d, d);
    if (dd < bd) { bd = dd; best = i; }
  }
  *idx = best;
  float rho[512];
  const uint16_t* c = CV + (size_t)best * d;
  for (int j = 0; j < d; ++j) rho[j] = bf(v[j]) - bf(c[j]);
  qo_int2_encode(rho, d, G, codes, params);
}

/* ------------------------------------------------------------------------- */
/* Frame-level append into the packed, head-major cache layout.               */
/*   k_codes  [H][Tcap][d/4] u8      k_params [H][Tcap][d/G][2] fp16 bits       */
/*   k_idx    [H][Tcap] (u8 if C <= 256 else u16)                               */
/*   k_coef   [H][Tcap][r] i8        k_cscale [H][Tcap] fp16 bits               */
/*   v_codes, v_params, v_idx        as for K                                   */
/* K, V input: [n][H][d] bf16 (token-major).  s [H][d], w [H][d/G],            */
/* U [H][d][r] (the basis in force for this append).                           */
/* ------------------------------------------------------------------------- */
QO_API void qo_append_frame(int H, int d, int C, int G, int M, int r, int64_t Tcap, int64_t t0,
                            const uint16_t* K, const uint16_t* V, int64_t n,
                            const uint16_t* CK, const uint16_t* CV, const float* s,
                            const float* w, const float* U,
                            uint8_t* k_codes, uint16_t* k_params, void* k_idx, int8_t* k_coef,
                            uint16_t* k_cscale, uint8_t* v_codes, uint16_t* v_params,
                            void* v_idx, const float* Afull) {
  int ng = d / G;
  for (int h = 0; h < H; ++h) {
    const uint16_t* ck = CK + (size_t)h * C * d;
    const uint16_t* cv = CV + (size_t)h * C * d;
    for (int64_t t = 0; t < n; ++t) {
      int64_t slot = (int64_t)h * Tcap + t0 + t;
      int32_t ia, ib;
      qo_encode_key(K + ((size_t)t * H + h) * d, ck, C, d, G, M, s + (size_t)h * d,
                    w + (size_t)h * ng, U + (size_t)h * d * r, r, &ia,
                    k_codes + slot * (d / 4), k_params + slot * ng * 2, k_coef + slot * r,
                    k_cscale + slot, NULL, Afull ? Afull + (size_t)h * d * d : NULL);
      qo_encode_value(V + ((size_t)t * H + h) * d, cv, C, d, G, &ib,
                      v_codes + slot * (d / 4), v_params + slot * ng * 2);
      if (C <= 256) {
        ((uint8_t*)k_idx)[slot] = (uint8_t)ia;
        ((uint8_t*)v_idx)[slot] = (uint8_t)ib;
      } else {
        ((uint16_t*)k_idx)[slot] = (uint16_t)ia;
        ((uint16_t*)v_idx)[slot] = (uint16_t)ib;
      }
    }
  }
}

/* ------------------------------------------------------------------------- */
/* Reconstruction [SP-en, PSAC: the Key is compensated "during cache          */
/* reconstruction"]:  K' = C[a] + deq(R) + U (c8 * cs),  V' = C_V[b] + deq(R_V) */
/* summed in fp64 and rounded once to bf16.                                    */
/* ------------------------------------------------------------------------- */
QO_API void qo_reconstruct_key(const uint16_t* c, const uint8_t* codes, const uint16_t* params,
                               const int8_t* coef, uint16_t cscale, const float* U, int d, int G,
                               int r, uint16_t* out, double* out_f64) {
  float deq[512];
  qo_int2_decode(codes, params, d, G, deq);
  double cs = (double)qo_f16_to_f32(cscale);
  for (int j = 0; j < d; ++j) {
    double v = (double)bf(c[j]) + (double)deq[j];
    for (int q = 0; q < r; ++q) v += (double)U[(size_t)j * r + q] * ((double)coef[q] * cs);
    if (out) out[j] = qo_f64_to_bf16(v);
    if (out_f64) out_f64[j] = v;
  }
}

QO_API void qo_reconstruct_value(const uint16_t* c, const uint8_t* codes, const uint16_t* params,
                                 int d, int G, uint16_t* out) {
  float deq[512];
  qo_int2_decode(codes, params, d, G, deq);
  for (int j = 0; j < d; ++j) out[j] = qo_f64_to_bf16((double)bf(c[j]) + (double)deq[j]);
}

/* Reconstruct the whole cache of one head: K', V' [T][d] bf16.
 * U_all [n_versions][H][d][r], tok_ver [Tcap] (version of each token). */
/* Tokens [t0, t1) of head h (Kp, Vp indexed by t - t0), reconstructed with the
 * centroid tables CK, CV given (the tables in force when those tokens were
 * appended). */
QO_API void qo_reconstruct_range(int h, int H, int d, int C, int G, int r, int64_t Tcap,
                                 int64_t t0, int64_t t1, const uint16_t* CK, const uint16_t* CV,
                                 const float* U_all, const uint16_t* tok_ver,
                                 const uint8_t* k_codes, const uint16_t* k_params,
                                 const void* k_idx, const int8_t* k_coef,
                                 const uint16_t* k_cscale, const uint8_t* v_codes,
                                 const uint16_t* v_params, const void* v_idx, uint16_t* Kp,
                                 uint16_t* Vp) {
  int ng = d / G;
  for (int64_t t = t0; t < t1; ++t) {
    int64_t slot = (int64_t)h * Tcap + t;
    int a = (C <= 256) ? ((const uint8_t*)k_idx)[slot] : ((const uint16_t*)k_idx)[slot];
    int b = (C <= 256) ? ((const uint8_t*)v_idx)[slot] : ((const uint16_t*)v_idx)[slot];
    const float* U = U_all + ((size_t)tok_ver[t] * H + h) * d * r;
    qo_reconstruct_key(CK + ((size_t)h * C + a) * d, k_codes + slot * (d / 4),
                       k_params + slot * ng * 2, k_coef + slot * r, k_cscale[slot], U, d, G, r,
                       Kp + (size_t)(t - t0) * d, NULL);
    qo_reconstruct_value(CV + ((size_t)h * C + b) * d, v_codes + slot * (d / 4),
                         v_params + slot * ng * 2, d, G, Vp + (size_t)(t - t0) * d);
  }
}

QO_API void qo_reconstruct_head(int h, int H, int d, int C, int G, int r, int64_t Tcap, int64_t T,
                                const uint16_t* CK, const uint16_t* CV, const float* U_all,
                                const uint16_t* tok_ver, const uint8_t* k_codes,
                                const uint16_t* k_params, const void* k_idx, const int8_t* k_coef,
                                const uint16_t* k_cscale, const uint8_t* v_codes,
                                const uint16_t* v_params, const void* v_idx, uint16_t* Kp,
                                uint16_t* Vp) {
  int ng = d / G;
  for (int64_t t = 0; t < T; ++t) {
    int64_t slot = (int64_t)h * Tcap + t;
    int a = (C <= 256) ? ((const uint8_t*)k_idx)[slot] : ((const uint16_t*)k_idx)[slot];
    int b = (C <= 256) ? ((const uint8_t*)v_idx)[slot] : ((const uint16_t*)v_idx)[slot];
    const float* U = U_all + ((size_t)tok_ver[t] * H + h) * d * r;
    qo_reconstruct_key(CK + ((size_t)h * C + a) * d, k_codes + slot * (d / 4),
                       k_params + slot * ng * 2, k_coef + slot * r, k_cscale[slot], U, d, G, r,
                       Kp + (size_t)t * d, NULL);
    qo_reconstruct_value(CV + ((size_t)h * C + b) * d, v_codes + slot * (d / 4),
                         v_params + slot * ng * 2, d, G, Vp + (size_t)t * d);
  }
}

/* ------------------------------------------------------------------------- */
/* Attention of query rows over a reconstructed cache (fp64):                 */
/*   O = softmax(scale * Q K'^T) V'  (no mask; every cached key).             */
/* Q rows bf16 with stride `qstride`; K', V' dense [T][d] bf16.               */
/* ------------------------------------------------------------------------- */
QO_API void qo_attention_head(const uint16_t* Q, int64_t nq, int64_t qstride, const uint16_t* Kp,
                              const uint16_t* Vp, int64_t T, int d, double scale, double* O) {
  double* l = (double*)malloc(sizeof(double) * (size_t)(T > 0 ? T : 1));
  double* q = (double*)malloc(sizeof(double) * d);
  for (int64_t i = 0; i < nq; ++i) {
    for (int j = 0; j < d; ++j) q[j] = (double)bf(Q[i * qstride + j]);
    double m = -INFINITY;
    for (int64_t t = 0; t < T; ++t) {
      double acc = 0.0;
      for (int j = 0; j < d; ++j) acc += q[j] * (double)bf(Kp[(size_t)t * d + j]);
      l[t] = acc * scale;
      if (l[t] > m) m = l[t];
    }
    double den = 0.0;
    for (int64_t t = 0; t < T; ++t) { l[t] = exp(l[t] - m); den += l[t]; }
    for (int j = 0; j < d; ++j) {
      double acc = 0.0;
      for (int64_t t = 0; t < T; ++t) acc += l[t] * (double)bf(Vp[(size_t)t * d + j]);
      O[i * d + j] = (T > 0) ? acc / den : 0.0;
    }
  }
  free(l); free(q);
}

/* Log of the softmax denominator of each query row over keys K [T][d] (fp64):
 *   lse_i = ln sum_t exp(scale * q_i . k_t),  taken as m + ln sum exp(l_t - m)
 * with m the row maximum (so that two attentions over disjoint key sets can be
 * merged with weights exp(lse)).  T == 0 gives -inf. */
QO_API void qo_attention_lse(const uint16_t* Q, int64_t nq, int64_t qstride, const uint16_t* K,
                             int64_t T, int d, double scale, double* lse) {
  double* l = (double*)malloc(sizeof(double) * (size_t)(T > 0 ? T : 1));
  for (int64_t i = 0; i < nq; ++i) {
    double m = -INFINITY;
    for (int64_t t = 0; t < T; ++t) {
      double acc = 0.0;
      for (int j = 0; j < d; ++j)
        acc += (double)bf(Q[i * qstride + j]) * (double)bf(K[(size_t)t * d + j]);
      l[t] = acc * scale;
      if (l[t] > m) m = l[t];
    }
    double den = 0.0;
    for (int64_t t = 0; t < T; ++t) den += exp(l[t] - m);
    lse[i] = (T > 0) ? m + log(den) : -INFINITY;
  }
  free(l);
}

/* Top-1 key of each query row: argmax_t q . k_t (fp64 dot of the bf16 values),
 * ties to the lower t.  K rows with stride `kstride`. */
QO_API void qo_top1(const uint16_t* Q, int64_t nq, int64_t qstride, const uint16_t* K, int64_t T,
                    int64_t kstride, int d, int32_t* idx) {
  for (int64_t i = 0; i < nq; ++i) {
    double best = -INFINITY;
    int32_t arg = -1;
    for (int64_t t = 0; t < T; ++t) {
      double acc = 0.0;
      for (int j = 0; j < d; ++j)
        acc += (double)bf(Q[i * qstride + j]) * (double)bf(K[t * kstride + j]);
      if (acc > best) { best = acc; arg = (int32_t)t; }
    }
    idx[i] = arg;
  }
}

/* Packed bytes per token-head and fixed bytes per head (the compression
 * accounting counts centroids, quantization parameters and compensation data,
 * as the pages' 6.20x figure does). */
QO_API int64_t qo_bytes_per_token_head(int d, int C, int G, int r) {
  int idx = (C <= 256) ? 1 : 2;
  return 2 * (d / 4 + 4 * (d / G) + idx) + r + 2;
}
