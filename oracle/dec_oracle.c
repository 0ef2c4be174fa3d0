/*
 * dec_oracle.c -- CPU oracle for one greedy decode step of a Qwen3-style decoder.
 *
 * TEST INFRASTRUCTURE ONLY.  This file is the plain, slow, obviously correct
 * definition that the CUDA path is checked against.  Only the test suite, the
 * smoke check and the benchmark's CPU-baseline leg may load it.  It shares no
 * code, header, table or constant with the CUDA library.
 *
 * Arithmetic: every activation is a double; weights and the KV cache are held
 * as the bytes the pages' system stores (bf16, or OCP FP8 E4M3 + fp32 scale
 * for the cache, or int8 + fp32 row scale for the projection weights) and
 * widened to double on use.  Sums run in the order the definition writes
 * them (ascending index), no blocking, no reordering.
 *
 * Sources (page title, section):
 *  - "Qwen3-ASR -- Latency & Bottleneck Analysis", 03 Decode (module list:
 *    28 decoder layers of attention + MLP, RMSNorms, rotary "MRoPE, fp32",
 *    lm_head 1024->151936, embed + final_norm) and 07 Root causes (q/k/v
 *    projections, GQA repeat_kv, QK^T, mask add, fp32 softmax, AV, o_proj;
 *    RMSNorm as an fp32 up-cast, variance reduction and down-cast).
 *  - "Can CTC make Qwen3-ASR faster?", 03 Greedy exactness (the emitted token
 *    is the argmax of the target logits).
 *  - Baseten Qwen3-ASR batch-transcription article, KV cache quantization
 *    (the cache is stored in FP8; attention math stays in full precision).
 *  - faster-qwen-asr GB10 benchmark record, "cuda_graph_int8" entries
 *    (int8 weight-only quantisation of the text decoder and lm_head).
 * Readings where the pages are silent (per-head q/k RMSNorm placement,
 * rotate-half RoPE pairing, consecutive GQA grouping, eps 1e-6, theta 1e6,
 * E4M3 encoding with one fp32 scale per (layer, K/V, head, token)) are listed
 * with the function that takes them.
 *
 * Parity pins: every function below is pinned by a CPU test against closed
 * forms, invariants, library routines or brute force; see tests/test_oracle_*.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

/* ------------------------------------------------------------------ */
/* Number formats                                                      */
/* ------------------------------------------------------------------ */

/* bf16 bits -> value: bf16 is the upper half of an IEEE binary32. */
double or_bf16_to_double(uint16_t b) {
  uint32_t u = (uint32_t)b << 16;
  float f;
  memcpy(&f, &u, 4);
  return (double)f;
}

/* Round a real to the nearest value with `frac_bits` fraction bits, ties to
 * even, for a binary format whose smallest normal exponent is `emin`
 * (values below 2^emin are subnormal with the fixed quantum 2^(emin-frac)).
 * Overflow handling is left to the caller.  Exact in double for the formats
 * used here (quantum scaling is by powers of two). */
static double round_to_format(double x, int frac_bits, int emin) {
  if (x == 0.0 || !isfinite(x)) return x;
  int e;
  frexp(x, &e);               /* |x| = m * 2^e, m in [0.5, 1): leading bit 2^(e-1) */
  int lead = e - 1;
  if (lead < emin) lead = emin;
  double quantum = ldexp(1.0, lead - frac_bits);
  return nearbyint(x / quantum) * quantum;  /* default rounding mode: ties to even */
}

/* double -> bf16 bits, round to nearest even (8 exponent bits, 7 fraction
 * bits, smallest normal 2^-126); overflow goes to +-inf as IEEE does. */
uint16_t or_bf16_round(double x) {
  if (isnan(x)) return 0x7FC0;
  double r = round_to_format(x, 7, -126);
  const double bf16_max = ldexp(255.0, 120); /* (2 - 2^-7) * 2^127 */
  if (fabs(r) > bf16_max) r = (r > 0) ? INFINITY : -INFINITY;
  float f = (float)r;         /* exact: r is representable in bf16 */
  uint32_t u;
  memcpy(&u, &f, 4);
  return (uint16_t)(u >> 16);
}

/* OCP FP8 E4M3 ("E4M3FN"): 1 sign, 4 exponent (bias 7), 3 fraction bits;
 * no infinities; S.1111.111 is NaN; largest finite 448 = 1.75 * 2^8;
 * smallest normal 2^-6, subnormal quantum 2^-9.  Decode from the definition. */
double or_e4m3_decode(uint8_t c) {
  int s = (c >> 7) & 1, E = (c >> 3) & 0xF, M = c & 7;
  double v;
  if (E == 15 && M == 7) return NAN;
  if (E == 0) v = ldexp((double)M / 8.0, -6);
  else v = ldexp(1.0 + (double)M / 8.0, E - 7);
  return s ? -v : v;
}

/* value -> E4M3 code, round to nearest even, saturating to +-448 (the
 * "satfinite" conversion); NaN -> 0x7F. */
uint8_t or_e4m3_encode(double x) {
  if (isnan(x)) return 0x7F;
  int s = signbit(x) ? 1 : 0;
  double a = fabs(x);
  double r = round_to_format(a, 3, -6);
  if (r > 448.0) r = 448.0;
  uint8_t code;
  if (r < ldexp(1.0, -6)) {   /* subnormal or zero: M * 2^-9 */
    code = (uint8_t)(int)(r / ldexp(1.0, -9));
  } else {
    int e;
    frexp(r, &e);
    int lead = e - 1;                          /* r = 1.fff * 2^lead */
    int M = (int)((r / ldexp(1.0, lead) - 1.0) * 8.0);
    code = (uint8_t)(((lead + 7) << 3) | M);
  }
  return (uint8_t)(code | (s << 7));
}

/* Per-row E4M3 quantisation of one KV row (one head, one token).
 * Reading (the pages only say "FP8"): one fp32 scale per row,
 * scale = max(amax, 2^-126) / 448 computed in fp32, code_i =
 * E4M3_rne_satfinite(fp32(x_i) / scale) with the division in fp32.  The
 * decision that yields an integer code is taken in fp32, as the kernel takes
 * it.  Returns the scale. */
float or_e4m3_quantize_row(const float *x, int n, uint8_t *codes) {
  float amax = 0.0f;
  for (int i = 0; i < n; ++i) {
    float a = fabsf(x[i]);
    if (a > amax) amax = a;
  }
  if (amax < 0x1p-126f) amax = 0x1p-126f;
  float scale = amax / 448.0f;
  for (int i = 0; i < n; ++i) {
    float q = x[i] / scale;   /* IEEE fp32 division */
    codes[i] = or_e4m3_encode((double)q);
  }
  return scale;
}

/* Per-row symmetric int8 quantisation of one bf16 weight row (faster-qwen-asr
 * GB10 benchmark record, "cuda_graph_int8" entries of the 0.6B and 1.7B
 * models: int8 weight-only quantisation of the text decoder and lm_head).
 * Reading (the record names the format only): one fp32 scale per output row,
 * scale = amax / 127 in fp32, code_i = round_half_even(fp32(w_i) / scale)
 * with the division in fp32, clamped to [-127, 127]; a row of zeros has
 * scale 0 and codes 0.  The decision that yields each integer code is taken
 * in fp32, as the kernel takes it.  Returns the scale. */
float or_int8_quantize_row(const uint16_t *w, int n, int8_t *codes) {
  float amax = 0.0f;
  for (int i = 0; i < n; ++i) {
    float a = fabsf((float)or_bf16_to_double(w[i]));
    if (a > amax) amax = a;
  }
  if (amax == 0.0f) {
    for (int i = 0; i < n; ++i) codes[i] = 0;
    return 0.0f;
  }
  float scale = amax / 127.0f;
  for (int i = 0; i < n; ++i) {
    float q = (float)or_bf16_to_double(w[i]) / scale;  /* IEEE fp32 division */
    float r = rintf(q);  /* default rounding mode: to nearest, ties to even */
    if (r > 127.0f) r = 127.0f;
    if (r < -127.0f) r = -127.0f;
    codes[i] = (int8_t)r;
  }
  return scale;
}

/* Every row of a row-major bf16 W[rows, cols]; rows are independent. */
void or_int8_quantize_rows(const uint16_t *W, int rows, int cols, int8_t *codes,
                           float *scales) {
#pragma omp parallel for schedule(static)
  for (int r = 0; r < rows; ++r)
    scales[r] = or_int8_quantize_row(W + (size_t)r * cols, cols, codes + (size_t)r * cols);
}

/* Per-row E4M3 weight-only quantisation of a row-major bf16 W[rows, cols]
 * ("Qwen3-ASR -- Latency & Bottleneck Analysis", 08 Optimization roadmap:
 * an fp8 lm_head; the same weight-only scheme for the projections).
 * Reading (the page names the format only): each row is quantised by the
 * per-row E4M3 quantiser of the KV rows (or_e4m3_quantize_row) applied to
 * the fp32 values of the bf16 weights: scale = max(amax, 2^-126) / 448 in
 * fp32, code_i = E4M3_rne_satfinite(fp32(w_i) / scale).  The weight the step
 * multiplies is e4m3(code) * scale. */
void or_fp8w_quantize_rows(const uint16_t *W, int rows, int cols, uint8_t *codes,
                           float *scales) {
#pragma omp parallel
  {
    float *row = (float *)malloc(sizeof(float) * (size_t)cols);
#pragma omp for schedule(static)
    for (int r = 0; r < rows; ++r) {
      for (int c = 0; c < cols; ++c) row[c] = (float)or_bf16_to_double(W[(size_t)r * cols + c]);
      scales[r] = or_e4m3_quantize_row(row, cols, codes + (size_t)r * cols);
    }
    free(row);
  }
}

/* ------------------------------------------------------------------ */
/* Building blocks                                                     */
/* ------------------------------------------------------------------ */

/* RMSNorm: y_i = x_i / sqrt(mean_j x_j^2 + eps) * g_i (gains bf16).
 * "Latency & Bottleneck Analysis", 07 Root causes: the norm up-casts,
 * reduces the variance and scales; here everything stays in double. */
void or_rmsnorm(const double *x, const uint16_t *g, int n, double eps, double *y) {
  double ss = 0.0;
  for (int i = 0; i < n; ++i) ss += x[i] * x[i];
  double inv = 1.0 / sqrt(ss / (double)n + eps);
  for (int i = 0; i < n; ++i) y[i] = x[i] * inv * or_bf16_to_double(g[i]);
}

/* y = W x for a row-major bf16 W[rows, cols] (y = W.x, weights stored
 * [out, in]); double dot products, ascending column order.  Rows are
 * independent, so they may be spread over threads without changing a bit. */
void or_gemv(const uint16_t *W, const double *x, int rows, int cols, double *y) {
#pragma omp parallel for schedule(static)
  for (int r = 0; r < rows; ++r) {
    const uint16_t *w = W + (size_t)r * cols;
    double acc = 0.0;
    for (int c = 0; c < cols; ++c) acc += or_bf16_to_double(w[c]) * x[c];
    y[r] = acc;
  }
}

/* y = W x for int8 codes C[rows, cols] with one fp32 scale per row: the
 * weight is the dequantised value code * scale, widened to double; double
 * dot products in ascending column order, as or_gemv. */
void or_gemv_i8(const int8_t *C, const float *s, const double *x, int rows, int cols,
                double *y) {
#pragma omp parallel for schedule(static)
  for (int r = 0; r < rows; ++r) {
    const int8_t *c = C + (size_t)r * cols;
    const double sr = (double)s[r];
    double acc = 0.0;
    for (int j = 0; j < cols; ++j) acc += ((double)c[j] * sr) * x[j];
    y[r] = acc;
  }
}

/* y = W x for E4M3 codes C[rows, cols] with one fp32 scale per row: the
 * weight is e4m3_decode(code) * scale in double; double dot products in
 * ascending column order, as or_gemv. */
void or_gemv_f8(const uint8_t *C, const float *s, const double *x, int rows, int cols,
                double *y) {
#pragma omp parallel for schedule(static)
  for (int r = 0; r < rows; ++r) {
    const uint8_t *c = C + (size_t)r * cols;
    const double sr = (double)s[r];
    double acc = 0.0;
    for (int j = 0; j < cols; ++j) acc += (or_e4m3_decode(c[j]) * sr) * x[j];
    y[r] = acc;
  }
}

/* A projection in any weight format: wkind 0 -> bf16 W, 1 -> int8 codes,
 * 2 -> E4M3 codes, the last two with row scales s. */
static void project(int wkind, const void *W, const float *s, const double *x, int rows,
                    int cols, double *y) {
  if (wkind == 0) or_gemv((const uint16_t *)W, x, rows, cols, y);
  else if (wkind == 1) or_gemv_i8((const int8_t *)W, s, x, rows, cols, y);
  else or_gemv_f8((const uint8_t *)W, s, x, rows, cols, y);
}

/* Rotary embedding of one head vector at position p ("MRoPE, fp32" in
 * "Latency & Bottleneck Analysis", 03 Decode).  Readings: for a text-only
 * decode step the three MRoPE sections share one position id, so it is the
 * 1-D rotation; pairing is rotate-half, (i, i + D/2); inv_freq_i =
 * 1/theta^(2i/D) and the angle p * inv_freq_i are fp32 values, as the page's
 * "fp32" says; cos and sin are taken in double of that fp32 angle. */
void or_rope(double *x, int d, int p, double theta) {
  int half = d / 2;
  for (int i = 0; i < half; ++i) {
    float inv_f = (float)(1.0 / pow(theta, (2.0 * i) / (double)d));
    float ang = (float)p * inv_f;
    double c = cos((double)ang), s = sin((double)ang);
    double a = x[i], b = x[i + half];
    x[i] = a * c - b * s;
    x[i + half] = b * c + a * s;
  }
}

/* SiLU(z) = z / (1 + exp(-z)). */
double or_silu(double z) { return z / (1.0 + exp(-z)); }

/* Softmax attention of one query over n cached rows of one KV head
 * ("Latency & Bottleneck Analysis", 07 Root causes: QK^T, mask, fp32
 * softmax, AV).  The rows are whatever the cache stores, widened to double:
 *   kind 0: bf16 rows, K/V given as bf16 bits with row stride `ld` elements;
 *   kind 1: E4M3 codes with one fp32 scale per row (value = code * scale).
 * s_j = q.K_j / sqrt(D); a = softmax(s) (max-subtracted); o = sum_j a_j V_j.
 * The mask of the decode step is causal over rows 0..p inclusive, which the
 * caller expresses as n = p + 1.  If `probs` is non-NULL the weights a_j are
 * stored there. */
void or_attend(const double *q, int d, int n, int kind,
               const uint16_t *K16, const uint16_t *V16,
               const uint8_t *K8, const uint8_t *V8,
               const float *Ks, const float *Vs, size_t ld,
               double *out, double *probs) {
  double *s = (double *)malloc(sizeof(double) * (n > 0 ? n : 1));
  double scale = 1.0 / sqrt((double)d);
  double m = -INFINITY;
  for (int j = 0; j < n; ++j) {
    double dot = 0.0;
    for (int i = 0; i < d; ++i) {
      double k = (kind == 0) ? or_bf16_to_double(K16[(size_t)j * ld + i])
                             : or_e4m3_decode(K8[(size_t)j * ld + i]) * (double)Ks[j];
      dot += q[i] * k;
    }
    s[j] = dot * scale;
    if (s[j] > m) m = s[j];
  }
  double l = 0.0;
  for (int j = 0; j < n; ++j) {
    s[j] = exp(s[j] - m);
    l += s[j];
  }
  for (int i = 0; i < d; ++i) out[i] = 0.0;
  for (int j = 0; j < n; ++j) {
    double a = s[j] / l;
    if (probs) probs[j] = a;
    for (int i = 0; i < d; ++i) {
      double v = (kind == 0) ? or_bf16_to_double(V16[(size_t)j * ld + i])
                             : or_e4m3_decode(V8[(size_t)j * ld + i]) * (double)Vs[j];
      out[i] += a * v;
    }
  }
  free(s);
}

/* argmax with the lowest index on ties ("Can CTC make Qwen3-ASR faster?",
 * 03 Greedy exactness); also the gap between the best and the second best
 * value over the other indices. */
int or_argmax(const double *v, int n, double *margin) {
  int best = 0;
  for (int i = 1; i < n; ++i)
    if (v[i] > v[best]) best = i;
  double second = -INFINITY;
  for (int i = 0; i < n; ++i)
    if (i != best && v[i] > second) second = v[i];
  if (margin) *margin = v[best] - second;
  return best;
}

/* ------------------------------------------------------------------ */
/* One decode step of one sequence                                     */
/* ------------------------------------------------------------------ */

/* Shape: ints {n_layers, hidden, n_q_heads, n_kv_heads, head_dim, ffn, vocab},
 * doubles {rms_eps, rope_theta}. */
enum { SH_L, SH_H, SH_HQ, SH_HKV, SH_D, SH_F, SH_V, SH_N };

/* Per-layer weight pointers, in this order. */
enum { W_IN_NORM, W_Q, W_K, W_V, W_Q_NORM, W_K_NORM, W_O, W_POST_NORM,
       W_GATE, W_UP, W_DOWN, W_N };

/*
 * One greedy decode step of a pre-norm Qwen3-style decoder for one sequence.
 *
 *  x = E[token]
 *  per layer l:
 *    h = rmsnorm(x, g_in)
 *    q = Wq h, k = Wk h, v = Wv h
 *    q_h = rmsnorm(q_h, g_q) per query head, k_g = rmsnorm(k_g, g_k) per KV
 *      head (reading: after the projection, before the rotation)
 *    q_h, k_g rotated at position p
 *    the cache row p of layer l gets k_g, v_g in the cache's format, and
 *      attention reads the stored row back like every other row
 *    o_h = attention of q_h over rows 0..p of KV head g = floor(h*Hkv/Hq)
 *      (reading of repeat_kv: each KV head serves Hq/Hkv consecutive
 *      query heads)
 *    x += Wo concat_h(o_h)
 *    h = rmsnorm(x, g_post);  x += Wd (silu(Wg h) * (Wu h))
 *  logits = W_lm rmsnorm(x, g_final);  token' = argmax(logits)
 *
 * Weights: wkind 0 -> every tensor bf16 bits; wkind 1 / 2 -> the seven
 * projections of every layer (q, k, v, o, gate, up, down) and lm_head are
 * int8 / E4M3 codes with fp32 row scales (lsc[l * W_N + idx], lm_scale), the
 * embedding and the norm gains stay bf16.
 * KV cache of this sequence: kind 0 -> bf16 bits kv16[L][2][Hkv][max_ctx][D];
 * kind 1 -> codes kv8[L][2][Hkv][max_ctx][D] and scales kvs[L][2][Hkv][max_ctx].
 * hidden_out (optional): x after the embedding and after every layer,
 * [(L+1)][H].  new_k / new_v (optional): the k_g and v_g of every layer before
 * they are stored, [L][Hkv][D].  Returns the argmax.
 */
int or_step(const int *sh, const double *shd,
            const uint16_t *embed, const void *lm_head, const uint16_t *final_norm,
            const void *const *lw, int wkind, const float *lm_scale,
            const float *const *lsc,
            int kind, uint16_t *kv16, uint8_t *kv8, float *kvs, int max_ctx,
            int token, int p,
            double *logits, double *hidden_out, double *new_k, double *new_v,
            double *margin) {
  const int L = sh[SH_L], H = sh[SH_H], Hq = sh[SH_HQ], Hkv = sh[SH_HKV];
  const int D = sh[SH_D], F = sh[SH_F], V = sh[SH_V];
  const double eps = shd[0], theta = shd[1];
  const int nq = Hq * D, nkv = Hkv * D;

  double *x = calloc(H, sizeof(double)), *h = calloc(H, sizeof(double));
  double *q = calloc(nq, sizeof(double)), *k = calloc(nkv, sizeof(double));
  double *v = calloc(nkv, sizeof(double)), *o = calloc(nq, sizeof(double));
  double *t = calloc(H > F ? H : F, sizeof(double));
  double *g = calloc(F, sizeof(double)), *u = calloc(F, sizeof(double));
  double *tmp = calloc(D, sizeof(double));
  float *rowf = calloc(D, sizeof(float));

  for (int i = 0; i < H; ++i) x[i] = or_bf16_to_double(embed[(size_t)token * H + i]);
  if (hidden_out) memcpy(hidden_out, x, sizeof(double) * H);

  for (int l = 0; l < L; ++l) {
    const void *const *w = lw + (size_t)l * W_N;
    const float *const *sc = wkind ? lsc + (size_t)l * W_N : NULL;
#define OR_SC(i) (sc ? sc[i] : NULL)
    or_rmsnorm(x, w[W_IN_NORM], H, eps, h);
    project(wkind, w[W_Q], OR_SC(W_Q), h, nq, H, q);
    project(wkind, w[W_K], OR_SC(W_K), h, nkv, H, k);
    project(wkind, w[W_V], OR_SC(W_V), h, nkv, H, v);
    for (int hh = 0; hh < Hq; ++hh) {
      or_rmsnorm(q + hh * D, w[W_Q_NORM], D, eps, tmp);
      memcpy(q + hh * D, tmp, sizeof(double) * D);
      or_rope(q + hh * D, D, p, theta);
    }
    for (int gg = 0; gg < Hkv; ++gg) {
      or_rmsnorm(k + gg * D, w[W_K_NORM], D, eps, tmp);
      memcpy(k + gg * D, tmp, sizeof(double) * D);
      or_rope(k + gg * D, D, p, theta);
    }
    if (new_k) memcpy(new_k + (size_t)l * nkv, k, sizeof(double) * nkv);
    if (new_v) memcpy(new_v + (size_t)l * nkv, v, sizeof(double) * nkv);

    /* append row p of every KV head of this layer */
    for (int gg = 0; gg < Hkv; ++gg) {
      for (int kvsel = 0; kvsel < 2; ++kvsel) {
        const double *src = kvsel == 0 ? k + gg * D : v + gg * D;
        size_t row = (((size_t)l * 2 + kvsel) * Hkv + gg) * max_ctx + p;
        if (kind == 0) {
          for (int i = 0; i < D; ++i) kv16[row * D + i] = or_bf16_round(src[i]);
        } else {
          for (int i = 0; i < D; ++i) rowf[i] = (float)src[i];
          kvs[row] = or_e4m3_quantize_row(rowf, D, kv8 + row * D);
        }
      }
    }

    /* attention, one query head at a time */
#pragma omp parallel for schedule(static)
    for (int hh = 0; hh < Hq; ++hh) {
      int gg = (int)(((long)hh * Hkv) / Hq);
      size_t kbase = (((size_t)l * 2 + 0) * Hkv + gg) * max_ctx;
      size_t vbase = (((size_t)l * 2 + 1) * Hkv + gg) * max_ctx;
      if (kind == 0)
        or_attend(q + hh * D, D, p + 1, 0, kv16 + kbase * D, kv16 + vbase * D,
                  NULL, NULL, NULL, NULL, D, o + hh * D, NULL);
      else
        or_attend(q + hh * D, D, p + 1, 1, NULL, NULL, kv8 + kbase * D, kv8 + vbase * D,
                  kvs + kbase, kvs + vbase, D, o + hh * D, NULL);
    }

    project(wkind, w[W_O], OR_SC(W_O), o, H, nq, t);
    for (int i = 0; i < H; ++i) x[i] += t[i];

    or_rmsnorm(x, w[W_POST_NORM], H, eps, h);
    project(wkind, w[W_GATE], OR_SC(W_GATE), h, F, H, g);
    project(wkind, w[W_UP], OR_SC(W_UP), h, F, H, u);
    for (int i = 0; i < F; ++i) u[i] = or_silu(g[i]) * u[i];
    project(wkind, w[W_DOWN], OR_SC(W_DOWN), u, H, F, t);
#undef OR_SC
    for (int i = 0; i < H; ++i) x[i] += t[i];
    if (hidden_out) memcpy(hidden_out + (size_t)(l + 1) * H, x, sizeof(double) * H);
  }

  or_rmsnorm(x, final_norm, H, eps, h);
  project(wkind, lm_head, lm_scale, h, V, H, logits);
  int id = or_argmax(logits, V, margin);

  free(x); free(h); free(q); free(k); free(v); free(o); free(t);
  free(g); free(u); free(tmp); free(rowf);
  return id;
}

void or_set_threads(int n) {
#ifdef _OPENMP
  if (n > 0) omp_set_num_threads(n);
#else
  (void)n;
#endif
}

int or_get_threads(void) {
#ifdef _OPENMP
  return omp_get_max_threads();
#else
  return 1;
#endif
}
