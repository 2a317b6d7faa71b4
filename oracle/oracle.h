/*
 * oracle.h -- plain, slow CPU reference of a batch-1 decoder decode step.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the test suite, the smoke check and the
 * benchmark's CPU-baseline leg may load this library.  It shares no code with
 * the CUDA path.
 *
 * Arithmetic: fp32 activations, bf16 weights widened to fp32, every dot
 * product a plain sequential fp32 sum (multiply, then add, each rounded),
 * libm expf/sqrtf.  Rotary angles are computed in double and rounded to fp32.
 *
 * What it follows:
 *   - forward pass: embedding table, then a stack of transformer blocks
 *     ("Crear desde cero un motor de inferencia para LLM usando C++ y CUDA",
 *     §1 and §1.1), a prefill phase that fills the KV cache and a decode phase
 *     that produces one token at a time (same page §1.1; "LLM高速化勉強会資料"
 *     slide 9);
 *   - KV-cache size 2*batch*layers*seq*head_dim*kv_heads*bytes
 *     ("LLM高速化勉強会資料" slide 10);
 *   - online softmax: running max and running sum, partial results rescaled,
 *     exact up to rounding ("Hạt nhân là gì ...", section on what
 *     FlashAttention really does);
 *   - grouped-query attention: several query heads share one KV head
 *     ("LLM高速化勉強会資料" slide 28).
 * The pages do not spell out the decoder block; the readings used (rotate-half
 * RoPE, contiguous GQA groups, SwiGLU FFN, pre-norm RMSNorm, scale 1/sqrt(d),
 * greedy argmax with the lowest index on ties) are the Llama/Qwen2 definitions
 * of the named model shapes.
 *
 * Parity pins: every function here is pinned by tests against invariants,
 * closed forms, special cases and an independent library implementation of
 * the same decoder.
 */
#ifndef MK_ORACLE_H
#define MK_ORACLE_H
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct {
  int n_layers, hidden, n_q_heads, n_kv_heads, head_dim, ffn, vocab;
  float rms_eps;
  double rope_theta;
  int qkv_bias;        /* 1: q/k/v projections carry a bias */
  int kv_bf16;         /* 1: cached K/V are rounded to bf16 (the default) */
} orc_config;

/* bf16 host pointers in the natural (row-major, out_features x in_features)
 * layout.  The model keeps the pointers; the caller keeps the memory alive. */
typedef struct {
  const uint16_t *attn_norm, *wq, *wk, *wv, *bq, *bk, *bv, *wo;
  const uint16_t *ffn_norm, *w_gate, *w_up, *w_down;
} orc_layer;

typedef struct orc_model orc_model;
typedef struct orc_state orc_state;

/* ---- primitives (each is pinned on its own) ---- */
float  orc_bf16_round(float x);
void   orc_rmsnorm(const float* x, const uint16_t* w, int n, float eps, float* y);
void   orc_gemv(const uint16_t* W, const float* x, int rows, int cols, float* y);
void   orc_rope(float* v, int head_dim, int pos, double theta);
void   orc_softmax(const float* s, int n, float* p);
void   orc_attend(const float* q, const float* K, const float* V, int n_keys,
                  int head_dim, float* out);
void   orc_attend_split(const float* q, const float* K, const float* V, int n_keys,
                        int head_dim, int n_splits, float* out);
float  orc_silu(float z);
int    orc_argmax(const float* v, int n);
double orc_kv_cache_bytes(double batch, double layers, double seq, double head_dim,
                          double kv_heads, double bytes_per_elem);
/* fp8 (e4m3) weights with one power-of-two scale per row: out[rows*cols] =
 * e4m3(w / 2^k) * 2^k as bf16, k per row the smallest with max|row| <= 448 * 2^k
 * (0 for a row of zeros), written to row_exp (may be NULL). */
void   orc_quantize_fp8_rows(const uint16_t* w, int rows, int cols, uint16_t* out, int* row_exp);

/* ---- model ---- */
orc_model* orc_create(const orc_config* cfg, const uint16_t* embed, const orc_layer* layers,
                      const uint16_t* final_norm, const uint16_t* lm_head /* NULL: tied */);
void       orc_destroy(orc_model* m);

orc_state* orc_state_create(const orc_model* m, int max_seq);
void       orc_state_destroy(orc_state* s);

/* One decode step of one request: token at position pos (pos counts from 0;
 * positions 0..pos-1 must already be in the cache).  Writes vocab logits and
 * the final residual stream (before the final norm, hidden floats); either
 * may be NULL.  Returns the greedy next id, or -1 on bad arguments. */
int orc_decode(const orc_model* m, orc_state* s, int token, int pos, float* logits,
               float* hidden);

/* A prompt of n tokens at positions 0..n-1 into an empty state, as n decode
 * steps; logits and hidden (either may be NULL) of the last position only.
 * Returns the greedy next id, or -1 on bad arguments. */
int orc_prefill(const orc_model* m, orc_state* s, const int* tokens, int n, float* logits,
                float* hidden);

/* Cached K or V of one layer and kv head, positions [0, n): out[n*head_dim]. */
int orc_state_kv(const orc_state* s, int layer, int kv_head, int which /*0 K, 1 V*/,
                 int n, float* out);
/* Overwrites positions [0, n) of one layer/kv head's K or V with in[n*head_dim]
 * (stored as the cache stores: rounded to bf16 when kv_bf16).  Lets a test
 * continue decoding from a cache it did not build (a long context). */
int orc_state_set_kv(orc_state* s, int layer, int kv_head, int which, int n, const float* in);

/* Whole sequence without a KV cache (full recompute, causal): logits and
 * hidden of every position, out_logits[n*vocab], out_hidden[n*hidden]. */
int orc_forward_full(const orc_model* m, const int* tokens, int n, float* out_logits,
                     float* out_hidden);

int orc_num_threads(void);

#ifdef __cplusplus
}
#endif
#endif
