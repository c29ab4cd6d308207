/*
 * pi_oracle.c -- plain, slow CPU oracle for the activation-sparse decode FFN.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the test suite, the smoke check and the
 * benchmark's CPU-baseline leg may load this library.  The product path (the
 * CUDA library) never calls it, links it or shares code with it.
 *
 * Every value is decoded from the exact bytes the caller passes (fp32, fp16
 * or Q4_0 split planes) by the code in this file, and all arithmetic is done
 * in IEEE double.  There is no blocking, fusion or reordering: each sum runs
 * over its index in ascending order.  OpenMP, when compiled in, only splits
 * independent outputs between threads, so results do not depend on the
 * thread count.
 *
 * Pages followed (titles as published):
 *   [GN] GeekNews, "Serving model bahasa besar berkecepatan tinggi pada PC
 *        dengan GPU konsumen"
 *   [AB] aibars.net, "PowerInfer - Hochgeschwindigkeits-Inferenz-Engine für
 *        große Sprachmodelle"
 *   [UA] unite.ai, "PowerInfer: Tüketici Düzeyinde bir GPU ile Hızlı Büyük
 *        Dil Modeli Sunucusu"
 *
 * Readings of points the pages leave open:
 *   - predictor = low-rank GEMV -> ReLU -> GEMV (+ optional bias) -> strict
 *     threshold, scoring cold neurons only; hot neurons are always computed;
 *   - the batch mask is the union over the tokens of the block, and every
 *     token is computed over that same union;
 *   - the active-index list is ascending;
 *   - squared ReLU is non-gated; the activation stays un-rounded (here: double);
 *   - Q4_0 nibble order: in each 32-element block, byte k holds element k in
 *     its low nibble and element k+16 in its high nibble; x = s * (q - 8);
 *   - stack glue between layers: x = h + y, h' = x / sqrt(mean(x^2) + eps).
 *
 * Pinning: every function here is checked by the CPU test suite against
 * hand-worked examples (tests/golden), closed forms, identities, brute force
 * over all masks of tiny layers, and library routines for special cases.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

/* element types (this file's own numbering; the Python wrapper maps names) */
enum { ORC_F32 = 0, ORC_F16 = 1, ORC_Q4_0 = 2 };
/* activations: [GN] "Keterbatasan dan FAQ" names ReLU, ReGLU and squared ReLU */
enum { ORC_RELU = 0, ORC_REGLU = 1, ORC_RELU2 = 2 };

void orc_set_threads(int n) {
#ifdef _OPENMP
  if (n > 0) omp_set_num_threads(n);
#else
  (void)n;
#endif
}

int orc_get_threads(void) {
#ifdef _OPENMP
  return omp_get_max_threads();
#else
  return 1;
#endif
}

/* IEEE 754 binary16 -> double, from the bit fields. */
double orc_half_to_double(uint16_t bits) {
  int sign = (bits >> 15) & 1;
  int expo = (bits >> 10) & 0x1f;
  int mant = bits & 0x3ff;
  double v;
  if (expo == 0) {
    v = ldexp((double)mant, -24); /* subnormal: mant * 2^-14 / 2^10 */
  } else if (expo == 31) {
    v = mant ? NAN : INFINITY;
  } else {
    v = ldexp((double)(mant | 0x400), expo - 25); /* (1 + mant/2^10) * 2^(expo-15) */
  }
  return sign ? -v : v;
}

/*
 * One element (row, col) of a row-major [rows, d] matrix stored as `type`.
 * Q4_0 ([GN] "Kuantisasi dan kompatibilitas": INT4 Q4_0, 32-element blocks
 * with an fp16 scale) uses split planes: qs [rows, d/2] bytes and
 * sc [rows, d/32] fp16.
 */
double orc_elem(int type, const void *data, const void *scales, int64_t row, int64_t col, int64_t d) {
  if (type == ORC_F32) {
    return (double)((const float *)data)[row * d + col];
  }
  if (type == ORC_F16) {
    return orc_half_to_double(((const uint16_t *)data)[row * d + col]);
  }
  /* Q4_0 */
  const uint8_t *qs = (const uint8_t *)data + row * (d / 2);
  const uint16_t *sc = (const uint16_t *)scales + row * (d / 32);
  int64_t blk = col / 32;
  int64_t k = col % 32;
  uint8_t byte = qs[blk * 16 + (k % 16)];
  int q = (k < 16) ? (byte & 0x0f) : (byte >> 4);
  return orc_half_to_double(sc[blk]) * (double)(q - 8);
}

/* Decode a whole token block h [batch, d] into doubles. */
static double *decode_tokens(int htype, const void *h, int batch, int d) {
  double *out = (double *)malloc(sizeof(double) * (size_t)batch * (size_t)d);
  for (int b = 0; b < batch; ++b)
    for (int i = 0; i < d; ++i) out[(size_t)b * d + i] = orc_elem(htype, h, NULL, b, i, d);
  return out;
}

/*
 * Predictor ([UA] "Adaptif Sparsite Predictor’ları": a per-layer predictor
 * picks the neurons that will fire; only those are computed).
 *   u[b,k] = max(0, sum_i P1[k,i] h[b,i])                 k < rank
 *   s[b,c] = sum_k P2[c,k] u[b,k] + bp[c]                  c < ffn - n_hot
 *   active(c) = OR_b (s[b,c] > thr)
 *   idx = ascending { n_hot + c : active(c) }
 * The predictor matrices are fp32, fp16 or Q4_0 ([UA] "Adaptif Sparsite
 * Predictor’ları": the predictor's size is chosen per layer; a Q4_0 predictor
 * decodes like a Q4_0 weight: P1 in 32-element blocks along d, P2 along the
 * rank, split planes with the scales in P1_sc / P2_sc, NULL otherwise).  Any
 * output pointer may be NULL.  Returns the number of active neurons.
 */
int64_t orc_predict(int d, int ffn, int n_hot, int rank, int htype, int ptype, int batch,
                    const void *h, const void *P1, const void *P1_sc, const void *P2, const void *P2_sc,
                    const float *bp, double thr, double *u_out, double *s_out, uint8_t *mask_out,
                    int32_t *idx_out) {
  const int n_cold = ffn - n_hot;
  double *hd = decode_tokens(htype, h, batch, d);
  double *u = (double *)malloc(sizeof(double) * (size_t)batch * (size_t)rank);
  double *s = (double *)malloc(sizeof(double) * (size_t)batch * (size_t)(n_cold > 0 ? n_cold : 1));

  for (int b = 0; b < batch; ++b) {
#pragma omp parallel for schedule(static)
    for (int k = 0; k < rank; ++k) {
      double acc = 0.0;
      for (int i = 0; i < d; ++i) acc += orc_elem(ptype, P1, P1_sc, k, i, d) * hd[(size_t)b * d + i];
      u[(size_t)b * rank + k] = acc > 0.0 ? acc : 0.0;
    }
  }
  for (int b = 0; b < batch; ++b) {
#pragma omp parallel for schedule(static)
    for (int c = 0; c < n_cold; ++c) {
      double acc = 0.0;
      for (int k = 0; k < rank; ++k) acc += orc_elem(ptype, P2, P2_sc, c, k, rank) * u[(size_t)b * rank + k];
      if (bp) acc += (double)bp[c];
      s[(size_t)b * n_cold + c] = acc;
    }
  }
  int64_t count = 0;
  for (int c = 0; c < n_cold; ++c) {
    int on = 0;
    for (int b = 0; b < batch; ++b) on |= (s[(size_t)b * n_cold + c] > thr);
    if (mask_out) mask_out[c] = (uint8_t)on;
    if (on) {
      if (idx_out) idx_out[count] = n_hot + c;
      ++count;
    }
  }
  if (u_out) memcpy(u_out, u, sizeof(double) * (size_t)batch * (size_t)rank);
  if (s_out) memcpy(s_out, s, sizeof(double) * (size_t)batch * (size_t)n_cold);
  free(hd);
  free(u);
  free(s);
  return count;
}

/* Pre-activation of neuron j for token row hb (the bias sits on the gate
 * for ReGLU and on the single up projection otherwise). */
static double preact(const void *w, const void *w_sc, int wtype, const float *b1, int64_t j, const double *hb, int d) {
  double acc = 0.0;
  for (int i = 0; i < d; ++i) acc += orc_elem(wtype, w, w_sc, j, i, d) * hb[i];
  if (b1) acc += (double)b1[j];
  return acc;
}

/* Activation value of neuron j for one token ([GN] "Keterbatasan dan FAQ"). */
static double neuron_act(int act, int wtype, const void *wg, const void *wg_sc, const void *wu, const void *wu_sc,
                         const float *b1, int64_t j, const double *hb, int d) {
  if (act == ORC_REGLU) {
    double g = preact(wg, wg_sc, wtype, b1, j, hb, d);
    double v = preact(wu, wu_sc, wtype, NULL, j, hb, d);
    return (g > 0.0 ? g : 0.0) * v;
  }
  double z = preact(wu, wu_sc, wtype, b1, j, hb, d);
  double r = z > 0.0 ? z : 0.0;
  return act == ORC_RELU2 ? r * r : r;
}

/*
 * Masked FFN ([UA] "Nöron Bilinçli Operatör": the operator works on single
 * rows of the up/gate matrices and single columns of the down matrix; the
 * down columns are stored neuron-major as the rows of W_downT).
 *   list = [0, n_hot) ++ idx[0, count)            (idx ascending, each >= n_hot)
 *   y[b,e] = b2[e] + sum_{j in list, in list order} a[b,j] * W_downT[j,e]
 * The same list is used for every token of the block.  cols / ncols select
 * which columns e to compute (cols == NULL: all d, y is [batch, d]; else y is
 * [batch, ncols]).  a_out, if given, receives a[b, position in list].
 */
void orc_masked_ffn(int d, int ffn, int n_hot, int wtype, int act, int htype, int batch, const void *h,
                    const int32_t *idx, int64_t count, const void *wg, const void *wg_sc, const void *wu,
                    const void *wu_sc, const void *wd, const void *wd_sc, const float *b1, const float *b2,
                    const int32_t *cols, int ncols, double *y_out, double *a_out) {
  (void)ffn;
  const int64_t n_list = (int64_t)n_hot + count;
  double *hd = decode_tokens(htype, h, batch, d);
  double *a = (double *)malloc(sizeof(double) * (size_t)batch * (size_t)(n_list > 0 ? n_list : 1));
  for (int b = 0; b < batch; ++b) {
#pragma omp parallel for schedule(static)
    for (int64_t p = 0; p < n_list; ++p) {
      int64_t j = p < n_hot ? p : (int64_t)idx[p - n_hot];
      a[(size_t)b * n_list + p] = neuron_act(act, wtype, wg, wg_sc, wu, wu_sc, b1, j, hd + (size_t)b * d, d);
    }
  }
  const int n_out = cols ? ncols : d;
  for (int b = 0; b < batch; ++b) {
#pragma omp parallel for schedule(static)
    for (int o = 0; o < n_out; ++o) {
      int64_t e = cols ? cols[o] : o;
      double acc = b2 ? (double)b2[e] : 0.0;
      for (int64_t p = 0; p < n_list; ++p) {
        int64_t j = p < n_hot ? p : (int64_t)idx[p - n_hot];
        acc += a[(size_t)b * n_list + p] * orc_elem(wtype, wd, wd_sc, j, e, d);
      }
      y_out[(size_t)b * n_out + o] = acc;
    }
  }
  if (a_out) memcpy(a_out, a, sizeof(double) * (size_t)batch * (size_t)n_list);
  free(hd);
  free(a);
}

/*
 * True activation support: support[b, j] = 1 iff neuron j's (gate, for
 * ReGLU; else up) pre-activation including b1 is > 0 for token b.
 */
void orc_true_support(int d, int ffn, int wtype, int act, int htype, int batch, const void *h, const void *wg,
                      const void *wg_sc, const void *wu, const void *wu_sc, const float *b1, uint8_t *support) {
  double *hd = decode_tokens(htype, h, batch, d);
  const void *w = act == ORC_REGLU ? wg : wu;
  const void *w_sc = act == ORC_REGLU ? wg_sc : wu_sc;
  for (int b = 0; b < batch; ++b) {
#pragma omp parallel for schedule(static)
    for (int j = 0; j < ffn; ++j)
      support[(size_t)b * ffn + j] = (uint8_t)(preact(w, w_sc, wtype, b1, j, hd + (size_t)b * d, d) > 0.0);
  }
  free(hd);
}

/*
 * Head-sparse decode self-attention ([UA] "Adaptif Sparsite Predictor’ları":
 * besides the FFN predictor, each layer has a predictor for its
 * self-attention block; only the heads it picks are computed).  One decode
 * step of `batch` independent sequences, multi-head attention with n_heads
 * heads of dh = d / n_heads dimensions:
 *   heads = [0, n_hot) ++ idx[0, count)   (always-computed heads, then the predicted ones)
 *   for every listed head h and token b (rows h*dh .. h*dh+dh-1 of Wq, Wk, Wv, WoT):
 *     q = Wq[h] x_b,  k = Wk[h] x_b,  v = Wv[h] x_b
 *     score_t = q . K[b,h,t] / sqrt(dh) for t < len,  score_len = q . k / sqrt(dh)
 *     p = softmax(score_0 .. score_len)
 *     o = sum_{t < len} p_t V[b,h,t] + p_len v
 *     y_b += sum_i o_i WoT[h*dh + i, :]
 * The new position uses this step's k and v themselves (the caller's cache
 * keeps them in its own type).  Caches K, V: [batch, n_heads, s_max, dh] of
 * type ctype; positions 0 .. len-1 are read.  Heads are added in list order,
 * every other sum in ascending index order.  k_out / v_out (optional):
 * [batch, n_list, dh], the new k and v of each listed head.
 */
void orc_attention(int d, int n_heads, int n_hot, int wtype, int htype, int ctype, int batch, const void *x,
                   const int32_t *idx, int64_t count, const void *Wq, const void *Wk, const void *Wv,
                   const void *WoT, const void *Kc, const void *Vc, int s_max, int len, double *y_out,
                   double *k_out, double *v_out) {
  const int dh = d / n_heads;
  const int64_t n_list = (int64_t)n_hot + count;
  const double scale = 1.0 / sqrt((double)dh);
  double *xd = decode_tokens(htype, x, batch, d);
  double *o = (double *)malloc(sizeof(double) * (size_t)batch * (size_t)(n_list > 0 ? n_list : 1) * (size_t)dh);
  for (int b = 0; b < batch; ++b) {
#pragma omp parallel for schedule(static)
    for (int64_t p = 0; p < n_list; ++p) {
      const int64_t h = p < n_hot ? p : (int64_t)idx[p - n_hot];
      const double *xb = xd + (size_t)b * d;
      double *q = (double *)malloc(sizeof(double) * (size_t)dh * 3);
      double *k = q + dh, *v = q + 2 * dh;
      for (int i = 0; i < dh; ++i) {
        double aq = 0.0, ak = 0.0, av = 0.0;
        for (int e = 0; e < d; ++e) {
          aq += orc_elem(wtype, Wq, NULL, h * dh + i, e, d) * xb[e];
          ak += orc_elem(wtype, Wk, NULL, h * dh + i, e, d) * xb[e];
          av += orc_elem(wtype, Wv, NULL, h * dh + i, e, d) * xb[e];
        }
        q[i] = aq;
        k[i] = ak;
        v[i] = av;
      }
      double *sc = (double *)malloc(sizeof(double) * (size_t)(len + 1));
      const int64_t crow = ((int64_t)b * n_heads + h) * s_max;
      for (int t = 0; t <= len; ++t) {
        double acc = 0.0;
        for (int i = 0; i < dh; ++i) acc += q[i] * (t < len ? orc_elem(ctype, Kc, NULL, crow + t, i, dh) : k[i]);
        sc[t] = acc * scale;
      }
      double m = sc[0];
      for (int t = 1; t <= len; ++t) m = sc[t] > m ? sc[t] : m;
      double sum = 0.0;
      for (int t = 0; t <= len; ++t) {
        sc[t] = exp(sc[t] - m);
        sum += sc[t];
      }
      double *ob = o + ((size_t)b * n_list + p) * dh;
      for (int i = 0; i < dh; ++i) {
        double acc = 0.0;
        for (int t = 0; t <= len; ++t) acc += sc[t] * (t < len ? orc_elem(ctype, Vc, NULL, crow + t, i, dh) : v[i]);
        ob[i] = acc / sum;
      }
      if (k_out)
        for (int i = 0; i < dh; ++i) k_out[((size_t)b * n_list + p) * dh + i] = k[i];
      if (v_out)
        for (int i = 0; i < dh; ++i) v_out[((size_t)b * n_list + p) * dh + i] = v[i];
      free(sc);
      free(q);
    }
  }
  for (int b = 0; b < batch; ++b) {
#pragma omp parallel for schedule(static)
    for (int e = 0; e < d; ++e) {
      double acc = 0.0;
      for (int64_t p = 0; p < n_list; ++p) {
        const int64_t h = p < n_hot ? p : (int64_t)idx[p - n_hot];
        for (int i = 0; i < dh; ++i)
          acc += o[((size_t)b * n_list + p) * dh + i] * orc_elem(wtype, WoT, NULL, h * dh + i, e, d);
      }
      y_out[(size_t)b * d + e] = acc;
    }
  }
  free(xd);
  free(o);
}

/*
 * Stack glue between layers (the pages are silent; residual + RMSNorm with
 * unit gain): x = h + y;  out = x / sqrt(mean_e x[e]^2 + eps).
 */
void orc_residual_rmsnorm(int batch, int d, int htype, const void *h, const double *y, double eps, double *out) {
  double *hd = decode_tokens(htype, h, batch, d);
  for (int b = 0; b < batch; ++b) {
    double ss = 0.0;
    for (int e = 0; e < d; ++e) {
      double x = hd[(size_t)b * d + e] + y[(size_t)b * d + e];
      ss += x * x;
    }
    double inv = 1.0 / sqrt(ss / (double)d + eps);
    for (int e = 0; e < d; ++e) out[(size_t)b * d + e] = (hd[(size_t)b * d + e] + y[(size_t)b * d + e]) * inv;
  }
  free(hd);
}
