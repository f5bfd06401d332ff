/*
 * oracle.c -- fp64 CPU oracle of the routed sparse-MoE block.
 *
 * TEST INFRASTRUCTURE: only the test-suite, the smoke check and the bench's
 * CPU-baseline leg load it.  It is deliberately plain: every step is the
 * definition written out in double precision, one token at a time, with no
 * blocking, fusion or reordering.  The only parallelism is an OpenMP loop over
 * independent tokens (it changes no arithmetic).
 *
 * Sources for what is computed (web pages on the Strata engine):
 *  [S1] "Strata open-source runtime: a 12GB card runs the 125B Qwen3 model",
 *       section "the model itself": each layer's router picks 10 of 512 experts
 *       plus one always-running shared expert; experts are feed-forward
 *       sub-networks.
 *  [S2] "Why Strata is fast on low-VRAM GPUs", section "the problem": 48 layers
 *       x 512 experts, the router picks 10 per token; section "one token,
 *       three workers": the GPU adds the expert results up, then the next
 *       layer starts; section "guess first, then check": a verify window of up
 *       to 4 tokens runs through one pass; section "the cost": experts ship as
 *       low-bit files (Q2_0, IQ3_*).
 *  [S3] "Strata illustrated" (lpnh.cn), section "expert cache": the expert
 *       profile ranks experts by routing frequency.
 * The pages print no formula.  Where they are silent the readings are:
 *  - expert FFN = SwiGLU: y = Wd (silu(Wg x) * (Wu x)), silu(z) = z/(1+e^-z);
 *  - weights are the softmax of the selected logits (the full-softmax
 *    denominator cancels on renormalisation);
 *  - selection: largest logits first, equal logits -> lower expert index,
 *    NaN ranks below every number;
 *  - dequantised weight = fp16 scale * (code - 2^(bits-1)), 32-element groups
 *    along the contracted dimension;
 *  - shared expert: weight 1, no gate;
 *  - stacked layers: x <- x + MoE(bf16(RMSNorm(x))), eps 1e-6, no norm weight.
 */
#include "oracle.h"

#include <math.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

/* ------------------------------------------------------------------ formats */

/* IEEE 754 binary16: 1 sign bit, 5 exponent bits (bias 15), 10 fraction bits. */
double orc_half_to_double(uint16_t h) {
  int sign = (h >> 15) & 1;
  int e = (h >> 10) & 31;
  int m = h & 1023;
  double v;
  if (e == 0)
    v = ldexp((double)m, -24);             /* subnormal: m * 2^-24 */
  else if (e == 31)
    v = m ? NAN : INFINITY;
  else
    v = ldexp((double)(1024 + m), e - 25); /* (1 + m/1024) * 2^(e-15) */
  return sign ? -v : v;
}

/* bfloat16 = the upper 16 bits of an IEEE binary32. */
double orc_bf16_to_double(uint16_t b) {
  uint32_t u = (uint32_t)b << 16;
  float f;
  memcpy(&f, &u, sizeof f);
  return (double)f;
}

/* Round a double to bfloat16 (8 significant bits, binary32 exponent range),
 * ties to even, overflow to infinity. */
uint16_t orc_double_to_bf16(double v) {
  if (isnan(v)) return 0x7FC0;
  double a = fabs(v);
  double r;
  if (a == 0.0) {
    r = 0.0;
  } else if (isinf(a)) {
    r = INFINITY;
  } else {
    int e;
    frexp(a, &e);                   /* a = f * 2^e, 0.5 <= f < 1 */
    int qe = e - 8;                 /* quantum of an 8-bit significand */
    if (qe < -133) qe = -133;       /* subnormal quantum 2^-126 * 2^-7 */
    r = nearbyint(ldexp(a, -qe));   /* default rounding mode: to nearest even */
    r = ldexp(r, qe);
    if (r >= ldexp(1.0, 128)) r = INFINITY;
  }
  float f = (float)r;               /* exact: r already has <= 8 significant bits */
  uint32_t u;
  memcpy(&u, &f, sizeof u);
  uint16_t out = (uint16_t)(u >> 16);
  if (signbit(v)) out |= 0x8000;
  return out;
}

/* ------------------------------------------------------- packed-layout reader */
/* A matrix R x K (K contracted) is stored in 16-row tiles; inside a tile the
 * 32-code groups are group-major: word (c, r) at (c*16 + r).  Code j of a group
 * is j = 8m + 2t + h; its low two bits sit at bit 32h + 8t + 2m of the group's
 * 8-byte little-endian word, and (3-bit) its high bit at bit 16h + 4t + m of
 * the group's 4-byte word, the 4-byte words following all 8-byte words of the
 * tile.  Scales: fp16, tile-interleaved the same way. */

static int64_t tile_bytes(int32_t K, int32_t bits) {
  int64_t nG = K / 32;
  return nG * 16 * (bits == 2 ? 8 : 12);
}

int64_t orc_codes_bytes(int32_t R, int32_t K, int32_t bits) {
  return (int64_t)(R / 16) * tile_bytes(K, bits);
}

int32_t orc_read_code(const uint8_t* mc, int32_t R, int32_t K, int32_t bits, int32_t row,
                      int32_t col) {
  (void)R;
  int32_t nG = K / 32;
  int32_t tile = row / 16, r = row % 16, c = col / 32, j = col % 32;
  int32_t m = j / 8, t = (j % 8) / 2, h = j % 2;
  const uint8_t* tb = mc + (int64_t)tile * tile_bytes(K, bits);
  const uint8_t* lo = tb + ((int64_t)c * 16 + r) * 8;
  int32_t pos = 32 * h + 8 * t + 2 * m;
  int32_t q = (lo[pos / 8] >> (pos % 8)) & 3;
  if (bits == 3) {
    const uint8_t* hi = tb + (int64_t)nG * 16 * 8 + ((int64_t)c * 16 + r) * 4;
    int32_t hp = 16 * h + 4 * t + m;
    q |= ((hi[hp / 8] >> (hp % 8)) & 1) << 2;
  }
  return q;
}

double orc_dequant(const uint8_t* mc, const uint16_t* ms, int32_t R, int32_t K, int32_t bits,
                   int32_t row, int32_t col) {
  int32_t nG = K / 32;
  int32_t tile = row / 16, r = row % 16, c = col / 32;
  double s = orc_half_to_double(ms[(int64_t)tile * 16 * nG + (int64_t)c * 16 + r]);
  int32_t q = orc_read_code(mc, R, K, bits, row, col);
  return s * (double)(q - (1 << (bits - 1)));
}

static void dequant_row(const uint8_t* mc, const uint16_t* ms, int32_t R, int32_t K, int32_t bits,
                        int32_t row, double* out) {
  for (int32_t col = 0; col < K; ++col) out[col] = orc_dequant(mc, ms, R, K, bits, row, col);
}

void orc_dequant_matrix(const uint8_t* mc, const uint16_t* ms, int32_t R, int32_t K, int32_t bits,
                        double* W) {
  for (int32_t row = 0; row < R; ++row) dequant_row(mc, ms, R, K, bits, row, W + (int64_t)row * K);
}

/* ------------------------------------------------------------------- router */

/* logits[t][e] = sum_i x[t][i] * Wr[e][i] + b[e]   (router scoring, [S1], [S2]) */
void orc_router_logits(const orc_layer* L, const double* x, int32_t T, double* logits) {
  for (int32_t t = 0; t < T; ++t)
    for (int32_t e = 0; e < L->E; ++e) {
      double acc = 0.0;
      const float* w = L->Wr + (int64_t)e * L->d;
      for (int32_t i = 0; i < L->d; ++i) acc += x[(int64_t)t * L->d + i] * (double)w[i];
      if (L->bias) acc += (double)L->bias[e];
      logits[(int64_t)t * L->E + e] = acc;
    }
}

/* "a ranks before b": larger value first; NaN after every number; equal values
 * (and two NaNs) by lower index. */
static int ranks_before(double a, int32_t ia, double b, int32_t ib) {
  int na = isnan(a), nb = isnan(b);
  if (na || nb) {
    if (na && nb) return ia < ib;
    return nb;
  }
  if (a != b) return a > b;
  return ia < ib;
}

static void select_row(const double* v, int32_t E, int32_t k, int32_t* ids, unsigned char* taken) {
  memset(taken, 0, (size_t)E);
  for (int32_t j = 0; j < k; ++j) {
    int32_t best = -1;
    for (int32_t e = 0; e < E; ++e) {
      if (taken[e]) continue;
      if (best < 0 || ranks_before(v[e], e, v[best], best)) best = e;
    }
    ids[j] = best;
    taken[best] = 1;
  }
}

/* top-k of 512 (k of E) per token ([S1], [S2]) on fp32 logits */
void orc_select_topk_f32(const float* logits, int32_t T, int32_t E, int32_t k, int32_t* ids) {
  double* v = (double*)malloc(sizeof(double) * (size_t)E);
  unsigned char* taken = (unsigned char*)malloc((size_t)E);
  for (int32_t t = 0; t < T; ++t) {
    for (int32_t e = 0; e < E; ++e) v[e] = (double)logits[(int64_t)t * E + e];
    select_row(v, E, k, ids + (int64_t)t * k, taken);
  }
  free(v);
  free(taken);
}

void orc_select_topk_f64(const double* logits, int32_t T, int32_t E, int32_t k, int32_t* ids) {
  unsigned char* taken = (unsigned char*)malloc((size_t)E);
  for (int32_t t = 0; t < T; ++t) select_row(logits + (int64_t)t * E, E, k, ids + (int64_t)t * k, taken);
  free(taken);
}

/* w_j = exp(l_j - l_max) / sum_{l in selected} exp(l - l_max): the softmax over
 * all experts renormalised to the selected ones (its denominator cancels). */
void orc_renorm_weights(const double* logits, const int32_t* ids, int32_t T, int32_t E, int32_t k,
                        double* w) {
  for (int32_t t = 0; t < T; ++t) {
    const double* l = logits + (int64_t)t * E;
    const int32_t* id = ids + (int64_t)t * k;
    double mx = -INFINITY;
    for (int32_t j = 0; j < k; ++j)
      if (l[id[j]] > mx) mx = l[id[j]];
    double den = 0.0;
    for (int32_t j = 0; j < k; ++j) den += exp(l[id[j]] - mx);
    for (int32_t j = 0; j < k; ++j) w[(int64_t)t * k + j] = exp(l[id[j]] - mx) / den;
  }
}

/* --------------------------------------------------------------- bucketing */

/* Per expert, the (token, slot) pairs that chose it, tokens ascending; each
 * entry is encoded t*k + j (its index in the [T][k] selection arrays).
 * offsets[e] = sum of counts of experts before e (offsets[E] = T*k). */
void orc_bucket(const int32_t* ids, int32_t T, int32_t k, int32_t E, int32_t* counts,
                int32_t* offsets, int32_t* entries) {
  for (int32_t e = 0; e < E; ++e) counts[e] = 0;
  for (int64_t i = 0; i < (int64_t)T * k; ++i) counts[ids[i]]++;
  offsets[0] = 0;
  for (int32_t e = 0; e < E; ++e) offsets[e + 1] = offsets[e] + counts[e];
  for (int32_t e = 0; e < E; ++e) {
    int32_t pos = offsets[e];
    for (int32_t t = 0; t < T; ++t)
      for (int32_t j = 0; j < k; ++j)
        if (ids[(int64_t)t * k + j] == e) entries[pos++] = t * k + j;
  }
}

/* ------------------------------------------------------------------- expert */

double orc_silu(double z) { return z / (1.0 + exp(-z)); }

/* SwiGLU expert: g = Wg x, u = Wu x, h = silu(g) * u, y = Wd h.
 * codes/scales point at one expert: Wg (F x d), Wu (F x d), Wd (d x F). */
void orc_expert_ffn(const uint8_t* codes, const uint16_t* scales, int32_t d, int32_t F,
                    int32_t bits, const double* x, double* y) {
  const int64_t cb_fd = orc_codes_bytes(F, d, bits);
  const int64_t ns_fd = (int64_t)F * d / 32;
  const uint8_t* cg = codes;
  const uint8_t* cu = codes + cb_fd;
  const uint8_t* cd = codes + 2 * cb_fd;
  const uint16_t* sg = scales;
  const uint16_t* su = scales + ns_fd;
  const uint16_t* sd = scales + 2 * ns_fd;
  int32_t n = d > F ? d : F;
  double* row = (double*)malloc(sizeof(double) * (size_t)n);
  double* h = (double*)malloc(sizeof(double) * (size_t)F);
  for (int32_t f = 0; f < F; ++f) {
    double g = 0.0, u = 0.0;
    dequant_row(cg, sg, F, d, bits, f, row);
    for (int32_t i = 0; i < d; ++i) g += row[i] * x[i];
    dequant_row(cu, su, F, d, bits, f, row);
    for (int32_t i = 0; i < d; ++i) u += row[i] * x[i];
    h[f] = orc_silu(g) * u;
  }
  for (int32_t i = 0; i < d; ++i) {
    double acc = 0.0;
    dequant_row(cd, sd, d, F, bits, i, row);
    for (int32_t f = 0; f < F; ++f) acc += row[f] * h[f];
    y[i] = acc;
  }
  free(row);
  free(h);
}

/* xn = bf16( x / sqrt(mean(x^2) + eps) ) per token */
void orc_rmsnorm_bf16(const uint16_t* x, int32_t T, int32_t d, double eps, uint16_t* xn) {
  for (int32_t t = 0; t < T; ++t) {
    double ss = 0.0;
    for (int32_t i = 0; i < d; ++i) {
      double v = orc_bf16_to_double(x[(int64_t)t * d + i]);
      ss += v * v;
    }
    double inv = 1.0 / sqrt(ss / d + eps);
    for (int32_t i = 0; i < d; ++i)
      xn[(int64_t)t * d + i] = orc_double_to_bf16(orc_bf16_to_double(x[(int64_t)t * d + i]) * inv);
  }
}

/* -------------------------------------------------------------------- block */

int orc_block_forward(const orc_layer* L, const uint16_t* x_bf16, int32_t T, const int32_t* rows,
                      int32_t n_rows, const float* sel_logits, int32_t flags, double* y,
                      double* logits_out, int32_t* ids_out, double* w_out) {
  if (!L || !x_bf16 || !y || T < 0 || L->k > L->E) return 1;
  const int32_t d = L->d, E = L->E, k = L->k;
  const int32_t n = rows ? n_rows : T;
  const int64_t cbe = 2 * orc_codes_bytes(L->F, d, L->bits) + orc_codes_bytes(d, L->F, L->bits);
  const int64_t nse = 3 * (int64_t)L->F * d / 32;
  int err = 0;
#pragma omp parallel for schedule(dynamic, 1)
  for (int32_t r = 0; r < n; ++r) {
    int32_t t = rows ? rows[r] : r;
    if (t < 0 || t >= T) {
      err = 1;
      continue;
    }
    double* xin = (double*)malloc(sizeof(double) * (size_t)d);
    double* lg = (double*)malloc(sizeof(double) * (size_t)E);
    double* ye = (double*)malloc(sizeof(double) * (size_t)d);
    int32_t* id = (int32_t*)malloc(sizeof(int32_t) * (size_t)k);
    double* w = (double*)malloc(sizeof(double) * (size_t)k);
    uint16_t* xn = (uint16_t*)malloc(sizeof(uint16_t) * (size_t)d);
    const uint16_t* xt = x_bf16 + (int64_t)t * d;
    if (flags & ORC_PRENORM) {
      orc_rmsnorm_bf16(xt, 1, d, 1e-6, xn);
      for (int32_t i = 0; i < d; ++i) xin[i] = orc_bf16_to_double(xn[i]);
    } else {
      for (int32_t i = 0; i < d; ++i) xin[i] = orc_bf16_to_double(xt[i]);
    }
    orc_router_logits(L, xin, 1, lg);
    if (sel_logits) {
      orc_select_topk_f32(sel_logits + (int64_t)t * E, 1, E, k, id);
    } else {
      float* lf = (float*)malloc(sizeof(float) * (size_t)E);
      for (int32_t e = 0; e < E; ++e) lf[e] = (float)lg[e];
      orc_select_topk_f32(lf, 1, E, k, id);
      free(lf);
    }
    orc_renorm_weights(lg, id, 1, E, k, w);
    double* yt = y + (int64_t)r * d;
    for (int32_t i = 0; i < d; ++i) yt[i] = 0.0;
    if (L->Fs > 0) {
      orc_expert_ffn(L->shared_codes, L->shared_scales, d, L->Fs, L->bits, xin, ye);
      for (int32_t i = 0; i < d; ++i) yt[i] += ye[i];
    }
    for (int32_t j = 0; j < k; ++j) {
      int32_t slot = L->expert_slot[id[j]];
      orc_expert_ffn(L->codes + (int64_t)slot * cbe, L->scales + (int64_t)slot * nse, d, L->F,
                     L->bits, xin, ye);
      for (int32_t i = 0; i < d; ++i) yt[i] += w[j] * ye[i];
    }
    if (flags & ORC_RESIDUAL)
      for (int32_t i = 0; i < d; ++i) yt[i] += orc_bf16_to_double(xt[i]);
    if (logits_out) memcpy(logits_out + (int64_t)r * E, lg, sizeof(double) * (size_t)E);
    if (ids_out) memcpy(ids_out + (int64_t)r * k, id, sizeof(int32_t) * (size_t)k);
    if (w_out) memcpy(w_out + (int64_t)r * k, w, sizeof(double) * (size_t)k);
    free(xin);
    free(lg);
    free(ye);
    free(id);
    free(w);
    free(xn);
  }
  return err;
}

int orc_num_threads(void) {
#ifdef _OPENMP
  return omp_get_max_threads();
#else
  return 1;
#endif
}

void orc_set_num_threads(int32_t n) {
#ifdef _OPENMP
  if (n > 0) omp_set_num_threads(n);
#else
  (void)n;
#endif
}
