/*
 * Plain C twin of the CPU oracle for RVQ KV-cache encode and compressed decode attention.
 *
 * TEST INFRASTRUCTURE.  Only the test suite, the package smoke check and the benchmark's CPU
 * baseline arm may load this library.  It shares no code, header or table with the CUDA
 * library: it includes only the C standard library.  It restates the numpy oracle's
 * definitions in sequential loops (no blocking, no reordering beyond what each definition
 * states), so that every oracle result has a second, independently coded evaluation.
 * Compile without value-changing floating-point options (-ffp-contract=off, no -ffast-math).
 *
 * Sources (web pages):
 *  - "VQKV: High-Fidelity and High-Ratio Cache Compression via Vector-Quantization"
 *    (gist.science summary of arXiv 2603.16435), section 2.1 "Residual Simple Vector
 *    Quantization": greedy residual stages ("Process" steps 1-4), reconstruction
 *    x_hat = sum_s Q_s[z_s]; section 2.3 "Inference Integration": codes read at decode,
 *    uncompressed local window of recent tokens.
 *  - "zerokv-neo 4.0.0" (pypi), "Architecture": Walsh-Hadamard energy spreading before
 *    quantisation, FP16 hot tier.
 *  - "VeloxQuant-MLX 0.5.1" (pypi), "VecInfer": Walsh-Hadamard rotation absorbed into the
 *    query; per-channel key smoothing lambda_i = sqrt(max |K_i|) before the rotation; product
 *    VQ over sub-vectors with 8-bit codes.
 *  - "Differential-KV" (GitHub README), "Decode & Prefill Innovations": fp32 log-sum-exp
 *    combine of partial attentions.
 *
 * Readings (the same as the numpy oracle's): Sylvester-ordered Hadamard H_d, scaled by
 * 1/sqrt(d); the quantiser's working vector is the float64 transform rounded once to float32;
 * squared L2 distances in float64, ties to the lowest index; residual update in float32;
 * residual norms accumulated in float64, stored as float32; attention in float64 with
 * softmax scale 1/sqrt(d) by default, natural-log lse, empty parts contribute nothing and an
 * empty context gives out = 0, lse = -inf.
 *
 * All functions return 0, or -1 for invalid arguments.  Arrays are dense, row-major.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

static int is_pow2(int d) { return d >= 1 && (d & (d - 1)) == 0; }

/* y = scale * H_d x for one row (in place on y): butterflies (a, b) -> (a + b, a - b) at
 * strides 1, 2, ..., d/2 over float64, then one multiplication by scale. */
static void fwht_row(double* y, int d, double scale) {
  for (int h = 1; h < d; h *= 2)
    for (int i = 0; i < d; i += 2 * h)
      for (int j = i; j < i + h; ++j) {
        const double a = y[j], b = y[j + h];
        y[j] = a + b;
        y[j + h] = a - b;
      }
  for (int i = 0; i < d; ++i) y[i] *= scale;
}

/* Walsh-Hadamard rotation of n rows of d values: y = scale * H_d x (float64). */
int zo_fwht(int64_t n, int d, double scale, const double* x, double* y) {
  if (n < 0 || !is_pow2(d) || (n > 0 && (!x || !y))) return -1;
  for (int64_t r = 0; r < n; ++r) {
    double* yr = y + r * d;
    memmove(yr, x + r * d, sizeof(double) * (size_t)d);
    fwht_row(yr, d, scale);
  }
  return 0;
}

/* The quantiser's working vector of one row: x (float64) divided channel by channel by the
 * smoothing factor (times the float64 reciprocal of the float32 factor), rotated by
 * (1/sqrt(d)) H_d when rotate is set, rounded once to float32. */
static void working_vector(const double* x, const float* lam, int rotate, int d, double* tmp,
                           float* y) {
  for (int i = 0; i < d; ++i) tmp[i] = lam ? x[i] * (1.0 / (double)lam[i]) : x[i];
  if (rotate) fwht_row(tmp, d, 1.0 / sqrt((double)d));
  for (int i = 0; i < d; ++i) y[i] = (float)tmp[i];
}

/* Index of the codeword nearest to r (squared L2 in float64 over dims), first on ties. */
static int nearest(const float* r, const float* C, int K, int dims) {
  double best = INFINITY;
  int z = 0;
  for (int c = 0; c < K; ++c) {
    double dist = 0.0;
    for (int i = 0; i < dims; ++i) {
      const double df = (double)r[i] - (double)C[(int64_t)c * dims + i];
      dist += df * df;
    }
    if (dist < best) {
      best = dist;
      z = c;
    }
  }
  return z;
}

/* Greedy residual vector quantisation of n rows (VQKV 2.1 "Process"): y = working vector;
 * r = y; for each stage s: z_s = nearest codeword of C[s] to r, r <- r - C[s][z_s] (float32),
 * n_s = ||r|| (float64 sum of squares, float32 result).
 * x [n][d] float64; smooth [d] float32 or NULL; C [S][K][d] float32; codes [n][S];
 * norms [n][S] and y_out [n][d] may be NULL. */
int zo_rvq_encode(int64_t n, int d, int S, int K, const double* x, const float* smooth,
                  int rotate, const float* C, uint8_t* codes, float* norms, float* y_out) {
  if (n < 0 || !is_pow2(d) || S < 1 || K < 1 || K > 256) return -1;
  if (n > 0 && (!x || !C || !codes)) return -1;
  double* tmp = (double*)malloc(sizeof(double) * (size_t)d);
  float* r = (float*)malloc(sizeof(float) * (size_t)d);
  if (!tmp || !r) {
    free(tmp);
    free(r);
    return -1;
  }
  for (int64_t row = 0; row < n; ++row) {
    working_vector(x + row * d, smooth, rotate, d, tmp, r);
    if (y_out) memcpy(y_out + row * d, r, sizeof(float) * (size_t)d);
    for (int s = 0; s < S; ++s) {
      const float* Cs = C + (int64_t)s * K * d;
      const int z = nearest(r, Cs, K, d);
      codes[row * S + s] = (uint8_t)z;
      double ss = 0.0;
      for (int i = 0; i < d; ++i) {
        r[i] = r[i] - Cs[(int64_t)z * d + i];
        ss += (double)r[i] * (double)r[i];
      }
      if (norms) norms[row * S + s] = (float)sqrt(ss);
    }
  }
  free(tmp);
  free(r);
  return 0;
}

/* Product VQ of n rows (VeloxQuant "VecInfer"): y = working vector, cut into d/m consecutive
 * sub-vectors; each takes its nearest codeword of the shared codebook C [K][m].
 * codes [n][d/m]. */
int zo_pq_encode(int64_t n, int d, int m, int K, const double* x, const float* smooth,
                 int rotate, const float* C, uint8_t* codes) {
  if (n < 0 || !is_pow2(d) || m < 1 || d % m || K < 1 || K > 256) return -1;
  if (n > 0 && (!x || !C || !codes)) return -1;
  double* tmp = (double*)malloc(sizeof(double) * (size_t)d);
  float* y = (float*)malloc(sizeof(float) * (size_t)d);
  if (!tmp || !y) {
    free(tmp);
    free(y);
    return -1;
  }
  const int nsub = d / m;
  for (int64_t row = 0; row < n; ++row) {
    working_vector(x + row * d, smooth, rotate, d, tmp, y);
    for (int j = 0; j < nsub; ++j) codes[row * nsub + j] = (uint8_t)nearest(y + j * m, C, K, m);
  }
  free(tmp);
  free(y);
  return 0;
}

/* Log-sum-exp combine of n_parts partial attentions over disjoint key sets
 * (Differential-KV): M = max lse_i; L = sum_i exp(lse_i - M); lse = M + log L;
 * out = sum_i exp(lse_i - lse) out_i.  Parts with lse = -inf carry no weight; all empty gives
 * (0, -inf).  outs [n_parts][d], lses [n_parts]. */
int zo_lse_merge(int n_parts, int d, const double* outs, const double* lses, double* out,
                 double* lse) {
  if (n_parts < 1 || d < 1 || !outs || !lses || !out || !lse) return -1;
  double M = -INFINITY;
  for (int i = 0; i < n_parts; ++i)
    if (lses[i] > M) M = lses[i];
  for (int e = 0; e < d; ++e) out[e] = 0.0;
  if (M == -INFINITY) {
    *lse = -INFINITY;
    return 0;
  }
  double L = 0.0;
  for (int i = 0; i < n_parts; ++i)
    if (lses[i] != -INFINITY) L += exp(lses[i] - M);
  const double total = M + log(L);
  for (int i = 0; i < n_parts; ++i) {
    if (lses[i] == -INFINITY) continue;
    const double w = exp(lses[i] - total);
    for (int e = 0; e < d; ++e) out[e] += w * outs[(int64_t)i * d + e];
  }
  *lse = total;
  return 0;
}

/* Exact single-query softmax attention over n keys/values (rows of d float64) with scores
 * scale * q . k_t; the key set is the concatenation of two blocks (the reconstructed
 * compressed part and the window).  An empty set gives (0, -inf). */
static void attend(const double* q, int d, double scale, const double* K1, const double* V1,
                   int64_t n1, const double* K2, const double* V2, int64_t n2, double* out,
                   double* lse, double* sc) {
  const int64_t n = n1 + n2;
  for (int e = 0; e < d; ++e) out[e] = 0.0;
  if (n == 0) {
    *lse = -INFINITY;
    return;
  }
  double m = -INFINITY;
  for (int64_t t = 0; t < n; ++t) {
    const double* k = t < n1 ? K1 + t * d : K2 + (t - n1) * d;
    double dot = 0.0;
    for (int e = 0; e < d; ++e) dot += q[e] * k[e];
    sc[t] = scale * dot;
    if (sc[t] > m) m = sc[t];
  }
  double l = 0.0;
  for (int64_t t = 0; t < n; ++t) {
    const double p = exp(sc[t] - m);
    const double* v = t < n1 ? V1 + t * d : V2 + (t - n1) * d;
    l += p;
    for (int e = 0; e < d; ++e) out[e] += p * v[e];
  }
  for (int e = 0; e < d; ++e) out[e] /= l;
  *lse = m + log(l);
}

/* Reconstruction of one compressed token, rotated back (VQKV 2.1 "Reconstruction", 2.3
 * "On-Demand Reconstruction"): x = (1/sqrt(d)) H_d x_hat, where x_hat is either the RVQ sum
 * over stages sum_s C[s][z_s] (nsub = 1, dims = d, n_cb = S stage codebooks [S][K][d]) or the
 * product-VQ concatenation of C[z_j] over sub-vectors j (nsub = d/m, dims = m, one codebook
 * [K][m]).  lam (keys with smoothing) multiplies the result channel by channel. */
static void reconstruct_token(const uint8_t* z, int n_codes, int pq, const float* C, int K,
                              int d, int m, const float* lam, double* x) {
  for (int e = 0; e < d; ++e) x[e] = 0.0;
  if (!pq) {
    for (int s = 0; s < n_codes; ++s) {
      const float* c = C + ((int64_t)s * K + z[s]) * d;
      for (int e = 0; e < d; ++e) x[e] += (double)c[e];
    }
  } else {
    for (int j = 0; j < n_codes; ++j) {
      const float* c = C + (int64_t)z[j] * m;
      for (int i = 0; i < m; ++i) x[j * m + i] = (double)c[i];
    }
  }
  fwht_row(x, d, 1.0 / sqrt((double)d));
  if (lam)
    for (int e = 0; e < d; ++e) x[e] *= (double)lam[e];
}

/* Shared body of the two decode oracles.  pq = 0: RVQ (Sk, Sv stage codes per token,
 * Ck [Hkv][Sk][K][d], Cv [Hkv][Sv][K][d]); pq = 1: product VQ (Sk = Sv = d/m codes per token,
 * Ck / Cv [Hkv][K][m]). */
static int decode_common(int pq, int B, int Hq, int Hkv, int d, int Sk, int Sv, int K, int m,
                         int64_t Tcap, int64_t Wcap, double scale, const double* q,
                         const uint8_t* k_codes, const uint8_t* v_codes, const int64_t* comp_len,
                         const float* Ck, const float* Cv, const double* win_k,
                         const double* win_v, const int64_t* win_len, const float* k_smooth,
                         double* out, double* lse) {
  if (B < 0 || Hq < 1 || Hkv < 1 || Hq % Hkv || !is_pow2(d) || K < 1 || K > 256) return -1;
  if (Sk < 1 || Sv < 1 || Tcap < 0 || Wcap < 0) return -1;
  if (B > 0 && (!q || !comp_len || !win_len || !out || !lse || !Ck || !Cv)) return -1;
  const int G = Hq / Hkv;
  if (scale <= 0.0) scale = 1.0 / sqrt((double)d);
  const int64_t ck_head = pq ? (int64_t)K * m : (int64_t)Sk * K * d;
  const int64_t cv_head = pq ? (int64_t)K * m : (int64_t)Sv * K * d;
  for (int b = 0; b < B; ++b) {
    const int64_t tc = comp_len[b], wl = win_len[b];
    if (tc < 0 || tc > Tcap || wl < 0 || wl > Wcap) return -1;
  }
  int64_t tmax = 1;
  for (int b = 0; b < B; ++b)
    if (comp_len[b] + win_len[b] > tmax) tmax = comp_len[b] + win_len[b];
  double* Kc = (double*)malloc(sizeof(double) * (size_t)(Tcap > 0 ? Tcap : 1) * d);
  double* Vc = (double*)malloc(sizeof(double) * (size_t)(Tcap > 0 ? Tcap : 1) * d);
  double* sc = (double*)malloc(sizeof(double) * (size_t)tmax);
  if (!Kc || !Vc || !sc) {
    free(Kc);
    free(Vc);
    free(sc);
    return -1;
  }
  for (int b = 0; b < B; ++b)
    for (int kvh = 0; kvh < Hkv; ++kvh) {
      const int64_t tc = comp_len[b], wl = win_len[b];
      const int64_t pair = (int64_t)b * Hkv + kvh;
      const float* lam = k_smooth ? k_smooth + (int64_t)kvh * d : NULL;
      for (int64_t t = 0; t < tc; ++t) {
        reconstruct_token(k_codes + (pair * Tcap + t) * Sk, Sk, pq, Ck + kvh * ck_head, K, d, m,
                          lam, Kc + t * d);
        reconstruct_token(v_codes + (pair * Tcap + t) * Sv, Sv, pq, Cv + kvh * cv_head, K, d, m,
                          NULL, Vc + t * d);
      }
      const double* wk = win_k ? win_k + pair * Wcap * d : NULL;
      const double* wv = win_v ? win_v + pair * Wcap * d : NULL;
      for (int g = 0; g < G; ++g) {
        const int64_t h = (int64_t)kvh * G + g;
        const int64_t row = (int64_t)b * Hq + h;
        attend(q + row * d, d, scale, Kc, Vc, tc, wk, wv, wl, out + row * d, lse + row, sc);
      }
    }
  free(Kc);
  free(Vc);
  free(sc);
  return 0;
}

/* Decode attention over an RVQ-compressed prefix plus the fp16 window, direct form: every
 * compressed key and value reconstructed and rotated back (keys times lambda with
 * smoothing), joined with the window, exact softmax attention in float64 for every (b, h)
 * with kv head h / (Hq / Hkv).
 * q [B][Hq][d]; k_codes [B][Hkv][Tcap][Sk]; v_codes [B][Hkv][Tcap][Sv]; comp_len [B];
 * Ck [Hkv][Sk][K][d]; Cv [Hkv][Sv][K][d]; win_k / win_v [B][Hkv][Wcap][d]; win_len [B];
 * k_smooth [Hkv][d] or NULL; scale <= 0 means 1/sqrt(d); out [B][Hq][d]; lse [B][Hq]. */
int zo_decode_attn(int B, int Hq, int Hkv, int d, int Sk, int Sv, int K, int64_t Tcap,
                   int64_t Wcap, double scale, const double* q, const uint8_t* k_codes,
                   const uint8_t* v_codes, const int64_t* comp_len, const float* Ck,
                   const float* Cv, const double* win_k, const double* win_v,
                   const int64_t* win_len, const float* k_smooth, double* out, double* lse) {
  return decode_common(0, B, Hq, Hkv, d, Sk, Sv, K, d, Tcap, Wcap, scale, q, k_codes, v_codes,
                       comp_len, Ck, Cv, win_k, win_v, win_len, k_smooth, out, lse);
}

/* The same over product-VQ codes: k_codes / v_codes [B][Hkv][Tcap][d/m]; Ck / Cv
 * [Hkv][K][m]. */
int zo_pq_decode_attn(int B, int Hq, int Hkv, int d, int m, int K, int64_t Tcap, int64_t Wcap,
                      double scale, const double* q, const uint8_t* k_codes,
                      const uint8_t* v_codes, const int64_t* comp_len, const float* Ck,
                      const float* Cv, const double* win_k, const double* win_v,
                      const int64_t* win_len, const float* k_smooth, double* out, double* lse) {
  if (m < 1 || d % m) return -1;
  return decode_common(1, B, Hq, Hkv, d, d / m, d / m, K, m, Tcap, Wcap, scale, q, k_codes,
                       v_codes, comp_len, Ck, Cv, win_k, win_v, win_len, k_smooth, out, lse);
}
