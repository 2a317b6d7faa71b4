/*
 * oracle.c -- plain, slow CPU reference of a batch-1 decoder decode step.
 * TEST INFRASTRUCTURE ONLY (see oracle.h for what it follows and how it is
 * pinned).  Built with -ffp-contract=off so that every multiply and add is
 * rounded on its own; OpenMP only splits independent output rows and heads.
 */
#include "oracle.h"

#include <math.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

/* ------------------------------------------------------------------ bf16 */

static float bf16_to_f32(uint16_t b) {
  uint32_t u = (uint32_t)b << 16;
  float f;
  memcpy(&f, &u, 4);
  return f;
}

/* Round-to-nearest-even to the 8-bit-mantissa bf16 grid. */
static uint16_t f32_to_bf16(float f) {
  uint32_t u;
  memcpy(&u, &f, 4);
  if ((u & 0x7f800000u) == 0x7f800000u && (u & 0x007fffffu)) return (uint16_t)((u >> 16) | 0x40);
  uint32_t lsb = (u >> 16) & 1u;
  u += 0x7fffu + lsb;
  return (uint16_t)(u >> 16);
}

float orc_bf16_round(float x) { return bf16_to_f32(f32_to_bf16(x)); }

/* ------------------------------------------------------------ primitives */

/* RMSNorm: y = x / sqrt(mean(x^2) + eps) * w. */
void orc_rmsnorm(const float* x, const uint16_t* w, int n, float eps, float* y) {
  float ss = 0.0f;
  for (int i = 0; i < n; ++i) ss += x[i] * x[i];
  float r = 1.0f / sqrtf(ss / (float)n + eps);
  for (int i = 0; i < n; ++i) y[i] = (x[i] * r) * bf16_to_f32(w[i]);
}

/* y = W x with W bf16 [rows x cols] row-major; one sequential sum per row
 * ("Crear desde cero ..." §2.1: the matrix-vector product parallelised over
 * rows with OpenMP). */
void orc_gemv(const uint16_t* W, const float* x, int rows, int cols, float* y) {
#pragma omp parallel for schedule(static)
  for (int r = 0; r < rows; ++r) {
    const uint16_t* wr = W + (size_t)r * (size_t)cols;
    float acc = 0.0f;
    for (int c = 0; c < cols; ++c) acc += bf16_to_f32(wr[c]) * x[c];
    y[r] = acc;
  }
}

/* Rotary embedding, rotate-half pairing (i, i + d/2), angle pos*theta^(-2i/d)
 * evaluated in double. */
void orc_rope(float* v, int head_dim, int pos, double theta) {
  int half = head_dim / 2;
  for (int i = 0; i < half; ++i) {
    double inv = pow(theta, -2.0 * (double)i / (double)head_dim);
    double ang = (double)pos * inv;
    float c = (float)cos(ang), s = (float)sin(ang);
    float a = v[i], b = v[i + half];
    v[i] = a * c - b * s;
    v[i + half] = a * s + b * c;
  }
}

/* Softmax with the maximum subtracted first. */
void orc_softmax(const float* s, int n, float* p) {
  float m = -INFINITY;
  for (int j = 0; j < n; ++j) m = s[j] > m ? s[j] : m;
  float sum = 0.0f;
  for (int j = 0; j < n; ++j) {
    p[j] = expf(s[j] - m);
    sum += p[j];
  }
  for (int j = 0; j < n; ++j) p[j] = p[j] / sum;
}

/* One query head over n keys: softmax(q.K_j / sqrt(d)) V, K and V fp32
 * [n x d] row-major. */
void orc_attend(const float* q, const float* K, const float* V, int n_keys, int head_dim,
                float* out) {
  float scale = 1.0f / sqrtf((float)head_dim);
  float* s = (float*)malloc(sizeof(float) * (size_t)(n_keys > 0 ? n_keys : 1));
  for (int j = 0; j < n_keys; ++j) {
    const float* kj = K + (size_t)j * head_dim;
    float dot = 0.0f;
    for (int i = 0; i < head_dim; ++i) dot += q[i] * kj[i];
    s[j] = dot * scale;
  }
  orc_softmax(s, n_keys, s);
  for (int i = 0; i < head_dim; ++i) {
    float acc = 0.0f;
    for (int j = 0; j < n_keys; ++j) acc += s[j] * V[(size_t)j * head_dim + i];
    out[i] = acc;
  }
  free(s);
}

/* The same attention computed the online-softmax way: the keys are cut into
 * n_splits contiguous blocks; each block keeps its own maximum m_s, sum
 * l_s = sum_j exp(s_j - m_s) and unnormalised output o_s = sum_j
 * exp(s_j - m_s) V_j; the blocks are merged by rescaling to the global
 * maximum ("Hạt nhân là gì ...": running max and running sum, partial results
 * rescaled whenever a new block arrives; the result is exact up to rounding).
 * Blocks are sized ceil(n / n_splits); an empty block is skipped. */
void orc_attend_split(const float* q, const float* K, const float* V, int n_keys,
                      int head_dim, int n_splits, float* out) {
  float scale = 1.0f / sqrtf((float)head_dim);
  int blk = (n_keys + n_splits - 1) / n_splits;
  float* ms = (float*)malloc(sizeof(float) * (size_t)n_splits);
  float* ls = (float*)malloc(sizeof(float) * (size_t)n_splits);
  float* os = (float*)calloc((size_t)n_splits * head_dim, sizeof(float));
  float* s = (float*)malloc(sizeof(float) * (size_t)(blk > 0 ? blk : 1));
  for (int b = 0; b < n_splits; ++b) {
    int j0 = b * blk, j1 = j0 + blk < n_keys ? j0 + blk : n_keys;
    ms[b] = -INFINITY;
    ls[b] = 0.0f;
    if (j0 >= j1) continue;
    for (int j = j0; j < j1; ++j) {
      const float* kj = K + (size_t)j * head_dim;
      float dot = 0.0f;
      for (int i = 0; i < head_dim; ++i) dot += q[i] * kj[i];
      s[j - j0] = dot * scale;
      if (s[j - j0] > ms[b]) ms[b] = s[j - j0];
    }
    for (int j = j0; j < j1; ++j) {
      float e = expf(s[j - j0] - ms[b]);
      ls[b] += e;
      for (int i = 0; i < head_dim; ++i) os[(size_t)b * head_dim + i] += e * V[(size_t)j * head_dim + i];
    }
  }
  float m = -INFINITY;
  for (int b = 0; b < n_splits; ++b) m = ms[b] > m ? ms[b] : m;
  float l = 0.0f;
  for (int i = 0; i < head_dim; ++i) out[i] = 0.0f;
  for (int b = 0; b < n_splits; ++b) {
    if (ls[b] == 0.0f) continue;
    float c = expf(ms[b] - m);
    l += c * ls[b];
    for (int i = 0; i < head_dim; ++i) out[i] += c * os[(size_t)b * head_dim + i];
  }
  for (int i = 0; i < head_dim; ++i) out[i] = out[i] / l;
  free(ms); free(ls); free(os); free(s);
}

float orc_silu(float z) { return z / (1.0f + expf(-z)); }

/* Greedy choice: the largest value, the lowest index among equal ones. */
int orc_argmax(const float* v, int n) {
  int best = 0;
  for (int i = 1; i < n; ++i)
    if (v[i] > v[best]) best = i;
  return best;
}

/* "LLM高速化勉強会資料" slide 10: 2 * batch * layers * seq * head_dim *
 * heads, times the bytes of one element; the heads are the KV heads. */
double orc_kv_cache_bytes(double batch, double layers, double seq, double head_dim,
                          double kv_heads, double bytes_per_elem) {
  return 2.0 * batch * layers * seq * head_dim * kv_heads * bytes_per_elem;
}

/* ----------------------------------------------------------- fp8 weights */

/* |v| rounded to the e4m3 grid (4 exponent bits with bias 7, 3 significand
 * bits, no infinities: the largest finite value is 1.75 * 2^8 = 448):
 * spacing 2^(e-3) inside the binade [2^e, 2^(e+1)) for e >= -6, spacing 2^-9
 * below 2^-6 (subnormals); round to nearest, ties to the even multiple;
 * anything above 448 saturates to 448.  Exact in double for any float input. */
static double e4m3_round_abs(double a) {
  if (a == 0.0) return 0.0;
  int E;
  frexp(a, &E);                 /* a = f * 2^E, f in [0.5, 1): binade e = E - 1 */
  int e = E - 1;
  if (e < -6) e = -6;
  double step = ldexp(1.0, e - 3);
  double r = rint(a / step) * step;  /* default rounding mode: nearest, ties to even */
  return r > 448.0 ? 448.0 : r;
}

/* fp8 weights ("LLM高速化勉強会資料" slide 33: fewer bits per parameter, with
 * block-wise scaling; "Crear desde cero ..." §4: FP8).  The block is one row:
 * k = the smallest integer with max|row| <= 448 * 2^k (k = 0 for a row of
 * zeros), each weight becomes e4m3(w / 2^k) * 2^k.  Writes those values as
 * bf16 (exact: 3 significand bits times a power of two) and the row exponents
 * k. */
void orc_quantize_fp8_rows(const uint16_t* w, int rows, int cols, uint16_t* out, int* row_exp) {
#pragma omp parallel for schedule(static)
  for (int r = 0; r < rows; ++r) {
    const uint16_t* wr = w + (size_t)r * cols;
    double mx = 0.0;
    for (int c = 0; c < cols; ++c) {
      double a = fabs((double)bf16_to_f32(wr[c]));
      if (a > mx) mx = a;
    }
    int k = 0;
    if (mx > 0.0) {
      k = (int)ceil(log2(mx / 448.0));
      while (mx > ldexp(448.0, k)) ++k;
      while (mx <= ldexp(448.0, k - 1)) --k;
    }
    if (row_exp) row_exp[r] = k;
    for (int c = 0; c < cols; ++c) {
      double v = (double)bf16_to_f32(wr[c]);
      double q = e4m3_round_abs(fabs(ldexp(v, -k)));
      out[(size_t)r * cols + c] = f32_to_bf16((float)ldexp(v < 0 ? -q : q, k));
    }
  }
}

int orc_num_threads(void) {
#ifdef _OPENMP
  return omp_get_max_threads();
#else
  return 1;
#endif
}

/* ----------------------------------------------------------------- model */

struct orc_model {
  orc_config c;
  const uint16_t* embed;
  orc_layer* layers;
  const uint16_t* final_norm;
  const uint16_t* lm_head;
};

struct orc_state {
  const orc_model* m;
  int max_seq;
  /* [layer][kv_head][max_seq][head_dim] for K then for V.  bf16 bits when
   * kv_bf16, else fp32. */
  void* kv;
};

orc_model* orc_create(const orc_config* cfg, const uint16_t* embed, const orc_layer* layers,
                      const uint16_t* final_norm, const uint16_t* lm_head) {
  if (!cfg || !embed || !layers || !final_norm) return NULL;
  if (cfg->n_q_heads % cfg->n_kv_heads || cfg->head_dim % 2) return NULL;
  orc_model* m = (orc_model*)calloc(1, sizeof(orc_model));
  m->c = *cfg;
  m->embed = embed;
  m->layers = (orc_layer*)malloc(sizeof(orc_layer) * (size_t)cfg->n_layers);
  memcpy(m->layers, layers, sizeof(orc_layer) * (size_t)cfg->n_layers);
  m->final_norm = final_norm;
  m->lm_head = lm_head ? lm_head : embed;
  return m;
}

void orc_destroy(orc_model* m) {
  if (!m) return;
  free(m->layers);
  free(m);
}

static size_t kv_index(const orc_config* c, int max_seq, int layer, int g, int which, int pos) {
  size_t per_head = (size_t)max_seq * c->head_dim;
  size_t per_layer = (size_t)c->n_kv_heads * per_head;
  size_t per_which = (size_t)c->n_layers * per_layer;
  return (size_t)which * per_which + (size_t)layer * per_layer + (size_t)g * per_head +
         (size_t)pos * c->head_dim;
}

orc_state* orc_state_create(const orc_model* m, int max_seq) {
  if (!m || max_seq <= 0) return NULL;
  orc_state* s = (orc_state*)calloc(1, sizeof(orc_state));
  s->m = m;
  s->max_seq = max_seq;
  size_t n = 2 * (size_t)m->c.n_layers * m->c.n_kv_heads * (size_t)max_seq * m->c.head_dim;
  s->kv = calloc(n, m->c.kv_bf16 ? sizeof(uint16_t) : sizeof(float));
  if (!s->kv) {
    free(s);
    return NULL;
  }
  return s;
}

void orc_state_destroy(orc_state* s) {
  if (!s) return;
  free(s->kv);
  free(s);
}

static void kv_store(orc_state* s, size_t idx, const float* v, int n) {
  if (s->m->c.kv_bf16) {
    uint16_t* p = (uint16_t*)s->kv + idx;
    for (int i = 0; i < n; ++i) p[i] = f32_to_bf16(v[i]);
  } else {
    memcpy((float*)s->kv + idx, v, sizeof(float) * (size_t)n);
  }
}

static void kv_load(const orc_state* s, size_t idx, float* v, int n) {
  if (s->m->c.kv_bf16) {
    const uint16_t* p = (const uint16_t*)s->kv + idx;
    for (int i = 0; i < n; ++i) v[i] = bf16_to_f32(p[i]);
  } else {
    memcpy(v, (const float*)s->kv + idx, sizeof(float) * (size_t)n);
  }
}

int orc_state_kv(const orc_state* s, int layer, int kv_head, int which, int n, float* out) {
  const orc_config* c = &s->m->c;
  if (layer < 0 || layer >= c->n_layers || kv_head < 0 || kv_head >= c->n_kv_heads || n < 0 ||
      n > s->max_seq || which < 0 || which > 1)
    return -1;
  kv_load(s, kv_index(c, s->max_seq, layer, kv_head, which, 0), out, n * c->head_dim);
  return 0;
}

int orc_state_set_kv(orc_state* s, int layer, int kv_head, int which, int n, const float* in) {
  const orc_config* c = &s->m->c;
  if (layer < 0 || layer >= c->n_layers || kv_head < 0 || kv_head >= c->n_kv_heads || n < 0 ||
      n > s->max_seq || which < 0 || which > 1 || !in)
    return -1;
  kv_store(s, kv_index(c, s->max_seq, layer, kv_head, which, 0), in, n * c->head_dim);
  return 0;
}

static void add_bias(float* y, const uint16_t* b, int n) {
  if (!b) return;
  for (int i = 0; i < n; ++i) y[i] = y[i] + bf16_to_f32(b[i]);
}

/* FFN block: a = silu(W_gate xn) * (W_up xn); x += W_down a. */
static void ffn_block(const orc_model* m, const orc_layer* L, float* x, float* xn, float* g,
                      float* u, float* d) {
  const orc_config* c = &m->c;
  orc_rmsnorm(x, L->ffn_norm, c->hidden, c->rms_eps, xn);
  orc_gemv(L->w_gate, xn, c->ffn, c->hidden, g);
  orc_gemv(L->w_up, xn, c->ffn, c->hidden, u);
  for (int i = 0; i < c->ffn; ++i) g[i] = orc_silu(g[i]) * u[i];
  orc_gemv(L->w_down, g, c->hidden, c->ffn, d);
  for (int i = 0; i < c->hidden; ++i) x[i] = x[i] + d[i];
}

/* Final norm, LM head, greedy id. */
static int head_out(const orc_model* m, const float* x, float* xn, float* logits, float* hidden) {
  const orc_config* c = &m->c;
  if (hidden) memcpy(hidden, x, sizeof(float) * (size_t)c->hidden);
  orc_rmsnorm(x, m->final_norm, c->hidden, c->rms_eps, xn);
  float* lg = logits ? logits : (float*)malloc(sizeof(float) * (size_t)c->vocab);
  orc_gemv(m->lm_head, xn, c->vocab, c->hidden, lg);
  int id = orc_argmax(lg, c->vocab);
  if (!logits) free(lg);
  return id;
}

/* The transformer blocks of one decode step: token at position pos, its K/V
 * appended to the cache; leaves the final residual stream in x_out[hidden]. */
static void decode_layers(const orc_model* m, orc_state* s, int token, int pos, float* x_out) {
  const orc_config* c = &m->c;
  const int H = c->hidden, d = c->head_dim, hq = c->n_q_heads, hkv = c->n_kv_heads;
  const int G = hq / hkv, F = c->ffn, n = pos + 1;
  float* x = (float*)malloc(sizeof(float) * (size_t)H);
  float* xn = (float*)malloc(sizeof(float) * (size_t)H);
  float* q = (float*)malloc(sizeof(float) * (size_t)hq * d);
  float* k = (float*)malloc(sizeof(float) * (size_t)hkv * d);
  float* v = (float*)malloc(sizeof(float) * (size_t)hkv * d);
  float* att = (float*)malloc(sizeof(float) * (size_t)hq * d);
  float* tmp = (float*)malloc(sizeof(float) * (size_t)(H > F ? H : F));
  float* g = (float*)malloc(sizeof(float) * (size_t)F);
  float* u = (float*)malloc(sizeof(float) * (size_t)F);
  float* Kb = (float*)malloc(sizeof(float) * (size_t)hkv * n * d);
  float* Vb = (float*)malloc(sizeof(float) * (size_t)hkv * n * d);

  const uint16_t* e = m->embed + (size_t)token * H;
  for (int i = 0; i < H; ++i) x[i] = bf16_to_f32(e[i]);

  for (int l = 0; l < c->n_layers; ++l) {
    const orc_layer* L = &m->layers[l];
    orc_rmsnorm(x, L->attn_norm, H, c->rms_eps, xn);
    orc_gemv(L->wq, xn, hq * d, H, q);
    orc_gemv(L->wk, xn, hkv * d, H, k);
    orc_gemv(L->wv, xn, hkv * d, H, v);
    if (c->qkv_bias) {
      add_bias(q, L->bq, hq * d);
      add_bias(k, L->bk, hkv * d);
      add_bias(v, L->bv, hkv * d);
    }
    for (int h = 0; h < hq; ++h) orc_rope(q + (size_t)h * d, d, pos, c->rope_theta);
    for (int h = 0; h < hkv; ++h) orc_rope(k + (size_t)h * d, d, pos, c->rope_theta);
    for (int h = 0; h < hkv; ++h) {
      kv_store(s, kv_index(c, s->max_seq, l, h, 0, pos), k + (size_t)h * d, d);
      kv_store(s, kv_index(c, s->max_seq, l, h, 1, pos), v + (size_t)h * d, d);
      kv_load(s, kv_index(c, s->max_seq, l, h, 0, 0), Kb + (size_t)h * n * d, n * d);
      kv_load(s, kv_index(c, s->max_seq, l, h, 1, 0), Vb + (size_t)h * n * d, n * d);
    }
#pragma omp parallel for schedule(static)
    for (int h = 0; h < hq; ++h) {
      int kvh = h / G;
      orc_attend(q + (size_t)h * d, Kb + (size_t)kvh * n * d, Vb + (size_t)kvh * n * d, n, d,
                 att + (size_t)h * d);
    }
    orc_gemv(L->wo, att, H, hq * d, tmp);
    for (int i = 0; i < H; ++i) x[i] = x[i] + tmp[i];
    ffn_block(m, L, x, xn, g, u, tmp);
  }
  memcpy(x_out, x, sizeof(float) * (size_t)H);
  free(x); free(xn); free(q); free(k); free(v); free(att); free(tmp); free(g); free(u);
  free(Kb); free(Vb);
}

int orc_decode(const orc_model* m, orc_state* s, int token, int pos, float* logits,
               float* hidden) {
  if (!m || !s || s->m != m) return -1;
  const orc_config* c = &m->c;
  if (token < 0 || token >= c->vocab || pos < 0 || pos >= s->max_seq) return -1;
  float* x = (float*)malloc(sizeof(float) * (size_t)c->hidden);
  float* xn = (float*)malloc(sizeof(float) * (size_t)c->hidden);
  decode_layers(m, s, token, pos, x);
  int id = head_out(m, x, xn, logits, hidden);
  free(x); free(xn);
  return id;
}

/* A prompt as n sequential decode steps at positions 0..n-1 ("Crear desde cero
 * ..." §1.1: the prefill fills the KV cache); only the last position goes
 * through the final norm and the LM head, whose output the prompt's earlier
 * positions do not need. */
int orc_prefill(const orc_model* m, orc_state* s, const int* tokens, int n, float* logits,
                float* hidden) {
  if (!m || !s || s->m != m || !tokens || n < 1 || n > s->max_seq) return -1;
  const orc_config* c = &m->c;
  for (int t = 0; t < n; ++t)
    if (tokens[t] < 0 || tokens[t] >= c->vocab) return -1;
  float* x = (float*)malloc(sizeof(float) * (size_t)c->hidden);
  float* xn = (float*)malloc(sizeof(float) * (size_t)c->hidden);
  for (int t = 0; t < n; ++t) decode_layers(m, s, tokens[t], t, x);
  int id = head_out(m, x, xn, logits, hidden);
  free(x); free(xn);
  return id;
}

/* Whole-sequence forward without a cache: every projection is applied to all
 * positions, K/V of all positions are kept as matrices (rounded to bf16 when
 * kv_bf16, as the cache would be), and position i attends to keys 0..i. */
int orc_forward_full(const orc_model* m, const int* tokens, int n, float* out_logits,
                     float* out_hidden) {
  if (!m || !tokens || n <= 0) return -1;
  const orc_config* c = &m->c;
  const int H = c->hidden, d = c->head_dim, hq = c->n_q_heads, hkv = c->n_kv_heads;
  const int G = hq / hkv, F = c->ffn;
  for (int t = 0; t < n; ++t)
    if (tokens[t] < 0 || tokens[t] >= c->vocab) return -1;
  float* X = (float*)malloc(sizeof(float) * (size_t)n * H);
  float* Xn = (float*)malloc(sizeof(float) * (size_t)H);
  float* Q = (float*)malloc(sizeof(float) * (size_t)n * hq * d);
  float* Kt = (float*)malloc(sizeof(float) * (size_t)n * hkv * d);
  float* Vt = (float*)malloc(sizeof(float) * (size_t)n * hkv * d);
  float* Kh = (float*)malloc(sizeof(float) * (size_t)n * d);
  float* Vh = (float*)malloc(sizeof(float) * (size_t)n * d);
  float* A = (float*)malloc(sizeof(float) * (size_t)n * hq * d);
  float* tmp = (float*)malloc(sizeof(float) * (size_t)(H > F ? H : F));
  float* g = (float*)malloc(sizeof(float) * (size_t)F);
  float* u = (float*)malloc(sizeof(float) * (size_t)F);

  for (int t = 0; t < n; ++t)
    for (int i = 0; i < H; ++i) X[(size_t)t * H + i] = bf16_to_f32(m->embed[(size_t)tokens[t] * H + i]);

  for (int l = 0; l < c->n_layers; ++l) {
    const orc_layer* L = &m->layers[l];
    for (int t = 0; t < n; ++t) {
      float* xt = X + (size_t)t * H;
      float* qt = Q + (size_t)t * hq * d;
      float* kt = Kt + (size_t)t * hkv * d;
      float* vt = Vt + (size_t)t * hkv * d;
      orc_rmsnorm(xt, L->attn_norm, H, c->rms_eps, Xn);
      orc_gemv(L->wq, Xn, hq * d, H, qt);
      orc_gemv(L->wk, Xn, hkv * d, H, kt);
      orc_gemv(L->wv, Xn, hkv * d, H, vt);
      if (c->qkv_bias) {
        add_bias(qt, L->bq, hq * d);
        add_bias(kt, L->bk, hkv * d);
        add_bias(vt, L->bv, hkv * d);
      }
      for (int h = 0; h < hq; ++h) orc_rope(qt + (size_t)h * d, d, t, c->rope_theta);
      for (int h = 0; h < hkv; ++h) orc_rope(kt + (size_t)h * d, d, t, c->rope_theta);
      if (c->kv_bf16) {
        for (int i = 0; i < hkv * d; ++i) {
          kt[i] = orc_bf16_round(kt[i]);
          vt[i] = orc_bf16_round(vt[i]);
        }
      }
    }
    for (int h = 0; h < hq; ++h) {
      int kvh = h / G;
      for (int t = 0; t < n; ++t) {
        memcpy(Kh + (size_t)t * d, Kt + (size_t)t * hkv * d + (size_t)kvh * d, sizeof(float) * d);
        memcpy(Vh + (size_t)t * d, Vt + (size_t)t * hkv * d + (size_t)kvh * d, sizeof(float) * d);
      }
#pragma omp parallel for schedule(static)
      for (int t = 0; t < n; ++t)
        orc_attend(Q + (size_t)t * hq * d + (size_t)h * d, Kh, Vh, t + 1, d,
                   A + (size_t)t * hq * d + (size_t)h * d);
    }
    for (int t = 0; t < n; ++t) {
      float* xt = X + (size_t)t * H;
      orc_gemv(L->wo, A + (size_t)t * hq * d, H, hq * d, tmp);
      for (int i = 0; i < H; ++i) xt[i] = xt[i] + tmp[i];
      ffn_block(m, L, xt, Xn, g, u, tmp);
    }
  }
  for (int t = 0; t < n; ++t)
    head_out(m, X + (size_t)t * H, Xn, out_logits ? out_logits + (size_t)t * c->vocab : NULL,
             out_hidden ? out_hidden + (size_t)t * H : NULL);
  free(X); free(Xn); free(Q); free(Kt); free(Vt); free(Kh); free(Vh); free(A); free(tmp);
  free(g); free(u);
  return 0;
}
