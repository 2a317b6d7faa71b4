// api.cu -- the C-ABI of libmk (declared in include/mk.h).
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>
#include <cstddef>
#include <cstdio>
#include <cstring>
#include <string>
#include <vector>

#include "../../include/mk.h"
#include "mk_internal.h"
#include "plan.h"
#include "prefill.h"

namespace mk {
size_t step_kernel_smem_bytes();
const void* step_kernel_ptr(int wbytes, int head_dim, int G);
cudaError_t launch_quantize_fp8_rows(uint16_t* w, uint8_t* codes, float* scales, int rows, int K,
                                     cudaStream_t st);
cudaError_t launch_pack_qkv(uint16_t*, const uint16_t*, const uint16_t*, const uint16_t*, int, int,
                            int, int, cudaStream_t);
cudaError_t launch_pack_qkv_bias(uint16_t*, const uint16_t*, const uint16_t*, const uint16_t*, int,
                                 int, int, cudaStream_t);
cudaError_t launch_pack_gateup(uint16_t*, const uint16_t*, const uint16_t*, int, int, cudaStream_t);
cudaError_t launch_step(const KernelArgs& args, int grid, bool cooperative, cudaStream_t st);
cudaError_t launch_read_probe(const void* src, size_t bytes, unsigned long long* sink, int sms,
                              cudaStream_t st);
cudaError_t launch_kv_table_update(int32_t* table, const int* idx, const int* val, int n,
                                   cudaStream_t st);
}  // namespace mk

using namespace mk;

static thread_local std::string g_create_error;

struct mk_ctx {
  mk_config cfg{};
  mk_options opt{};
  cudaStream_t stream = nullptr;
  int device = 0;
  Plan plan;
  ModelDev md{};
  std::vector<void*> allocs;
  Task* d_tasks = nullptr;
  int32_t* d_queue = nullptr;
  int32_t* d_queue_off = nullptr;
  StepParams* d_sp = nullptr;
  int32_t* d_tokens = nullptr;   // staging for mk_decode_step_host
  int32_t* d_ids = nullptr;
  int32_t* h_pinned = nullptr;   // pinned staging: tokens in, ids out
  int mode = MK_MODE_MEGAKERNEL;
  bool poisoned = false;
  std::string err;
  cudaGraphExec_t graph = nullptr;
  cudaGraph_t graph_src = nullptr;
  size_t kv_bytes = 0;
  float* hidden_all = nullptr;   // [max_batch][hidden]: residual streams of a multi-request step
  int last_n_req = 1;
  PrefillWeights pw;             // packed weight pointers for the tensor-core prefill
  PrefillScratch ps;             // its scratch (allocated at the first prefill)
  BatchScratch bs;               // batched decode step (allocated at its first use)
  bool last_batched = false;     // the last step ran the batched path (hidden in bs.x)
  // KV pages: a contiguous cache is one max_seq page per slot (page s = slot s)
  bool kv_paged = false;
  int kv_page = 0, kv_pps = 1, kv_pool = 0;
  std::vector<int32_t> kv_table_h;                // [max_batch][kv_pps], -1: no page
  std::vector<int32_t> kv_free;                   // free physical pages (a stack)
  std::vector<std::pair<int, int>> kv_pending;    // table entries not yet on the device
  int32_t* kv_table_d = nullptr;
};

namespace mk {
void set_last_error(const char* msg) { g_create_error = msg; }
}  // namespace mk

static int fail(mk_ctx* c, int code, const std::string& msg) {
  if (c) c->err = msg; else g_create_error = msg;
  return code;
}

#define CK(call)                                                                 \
  do {                                                                           \
    cudaError_t e_ = (call);                                                     \
    if (e_ != cudaSuccess)                                                       \
      return fail(ctx, MK_ERR_CUDA, std::string(#call) + ": " + cudaGetErrorString(e_)); \
  } while (0)

template <class T>
static int dalloc(mk_ctx* ctx, T** p, size_t bytes) {
  void* v = nullptr;
  cudaError_t e = cudaMalloc(&v, bytes ? bytes : 16);
  if (e != cudaSuccess) {
    cudaGetLastError();
    return fail(ctx, MK_ERR_OOM, "cudaMalloc(" + std::to_string(bytes) + "): " + cudaGetErrorString(e));
  }
  ctx->allocs.push_back(v);
  *p = static_cast<T*>(v);
  return MK_OK;
}

static void release(mk_ctx* ctx) {
  if (!ctx) return;
  if (ctx->graph) cudaGraphExecDestroy(ctx->graph);
  if (ctx->graph_src) cudaGraphDestroy(ctx->graph_src);
  for (int n = 0; n <= kMaxBatch; ++n) {
    if (ctx->bs.graph[n]) cudaGraphExecDestroy(ctx->bs.graph[n]);
    if (ctx->bs.graph_src[n]) cudaGraphDestroy(ctx->bs.graph_src[n]);
  }
  for (void* p : ctx->allocs) cudaFree(p);
  if (ctx->h_pinned) cudaFreeHost(ctx->h_pinned);
  ctx->allocs.clear();
}

static bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

static void fill_args(mk_ctx* ctx, KernelArgs& a, int set, const StepParams* sp_val,
                      const StepParams* sp_ptr, bool no_wait) {
  a.m = ctx->md;
  a.tasks = ctx->d_tasks;
  a.queue = ctx->d_queue;
  a.queue_off = ctx->d_queue_off + ctx->plan.set_offset(set);
  if (sp_val) a.sp_val = *sp_val; else memset(&a.sp_val, 0, sizeof(a.sp_val));
  a.sp_ptr = sp_ptr;
  a.no_wait = no_wait ? 1 : 0;
  a.n_steps = 1;
  a.ids_seq = nullptr;
}

// Enqueues one decode step in the context's mode.
static int enqueue_step(mk_ctx* ctx, const StepParams& sp) {
  const int P = ctx->plan.num_ctas;
  KernelArgs a;
  if (ctx->mode == MK_MODE_MEGAKERNEL) {
    fill_args(ctx, a, 0, &sp, nullptr, false);
    CK(launch_step(a, P, true, ctx->stream));
  } else if (ctx->mode == MK_MODE_PER_OP) {
    for (int s = 0; s < ctx->plan.n_stages; ++s) {
      fill_args(ctx, a, 1 + s, &sp, nullptr, true);
      CK(launch_step(a, P, false, ctx->stream));
    }
  } else {
    CK(cudaMemcpyAsync(ctx->d_sp, &sp, sizeof(StepParams), cudaMemcpyHostToDevice, ctx->stream));
    if (!ctx->graph) {
      cudaStream_t cs;
      CK(cudaStreamCreateWithFlags(&cs, cudaStreamNonBlocking));
      cudaError_t e = cudaStreamBeginCapture(cs, cudaStreamCaptureModeThreadLocal);
      for (int s = 0; e == cudaSuccess && s < ctx->plan.n_stages; ++s) {
        fill_args(ctx, a, 1 + s, nullptr, ctx->d_sp, true);
        e = launch_step(a, P, false, cs);
      }
      cudaGraph_t g = nullptr;
      cudaError_t e2 = cudaStreamEndCapture(cs, &g);
      cudaStreamDestroy(cs);
      if (e != cudaSuccess || e2 != cudaSuccess)
        return fail(ctx, MK_ERR_CUDA, std::string("graph capture: ") +
                                          cudaGetErrorString(e != cudaSuccess ? e : e2));
      ctx->graph_src = g;
      CK(cudaGraphInstantiate(&ctx->graph, g, 0));
    }
    CK(cudaGraphLaunch(ctx->graph, ctx->stream));
  }
  return MK_OK;
}

static void host_rope_table(int max_seq, int d, double theta, std::vector<float>& c,
                            std::vector<float>& s) {
  const int half = d / 2;
  c.resize((size_t)max_seq * half);
  s.resize((size_t)max_seq * half);
  for (int p = 0; p < max_seq; ++p)
    for (int i = 0; i < half; ++i) {
      const double freq = std::pow(theta, -2.0 * (double)i / (double)d);
      const double ang = (double)p * freq;
      c[(size_t)p * half + i] = (float)std::cos(ang);
      s[(size_t)p * half + i] = (float)std::sin(ang);
    }
}

extern "C" int mk_create(const mk_config* cfg, const mk_weights* w, const mk_options* opt,
                         void* stream, mk_ctx** out) {
  g_create_error.clear();
  mk_ctx* ctx = nullptr;
  if (!cfg || !w || !out) return fail(nullptr, MK_ERR_INVALID_ARG, "null argument");
  *out = nullptr;
  std::string verr = validate_config(*cfg);
  if (!verr.empty()) return fail(nullptr, MK_ERR_INVALID_ARG, verr);
  if (!w->embed || !w->layers || !w->final_norm || (!cfg->tied_embeddings && !w->lm_head))
    return fail(nullptr, MK_ERR_INVALID_ARG, "missing weight pointer");
  for (int l = 0; l < cfg->n_layers; ++l) {
    const mk_layer_weights& L = w->layers[l];
    const void* need[] = {L.attn_norm, L.wq, L.wk, L.wv, L.wo, L.ffn_norm, L.w_gate, L.w_up, L.w_down};
    for (const void* p : need)
      if (!p || !aligned16(p)) return fail(nullptr, MK_ERR_INVALID_ARG, "layer weight null or not 16-byte aligned");
    if (cfg->qkv_bias && (!L.bq || !L.bk || !L.bv))
      return fail(nullptr, MK_ERR_INVALID_ARG, "qkv_bias set but a bias pointer is null");
  }
  const int G = cfg->n_q_heads / cfg->n_kv_heads;
  const bool g_ok = cfg->head_dim == 128 ? (G == 1 || G == 2 || G == 4)
                                         : (G == 1 || G == 2 || G == 4 || G == 7 || G == 8);
  if (!g_ok) return fail(nullptr, MK_ERR_UNSUPPORTED, "unsupported query heads per KV head");

  ctx = new mk_ctx();
  ctx->cfg = *cfg;
  if (opt) ctx->opt = *opt;
  ctx->stream = static_cast<cudaStream_t>(stream);
  ctx->mode = ctx->opt.mode;
  int rc = MK_OK;
  auto bail = [&](int code) {
    std::string m = ctx->err;
    release(ctx);
    delete ctx;
    g_create_error = m;
    return code;
  };
#define CKC(call)                                                                          \
  do {                                                                                     \
    cudaError_t e_ = (call);                                                               \
    if (e_ != cudaSuccess) {                                                               \
      ctx->err = std::string(#call) + ": " + cudaGetErrorString(e_);                       \
      return bail(MK_ERR_CUDA);                                                            \
    }                                                                                      \
  } while (0)
  CKC(cudaGetDevice(&ctx->device));
  int sms = 0, smem_optin = 0;
  CKC(cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, ctx->device));
  CKC(cudaDeviceGetAttribute(&smem_optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, ctx->device));
  const size_t smem = step_kernel_smem_bytes();
  if ((size_t)smem_optin < smem) {
    ctx->err = "device offers " + std::to_string(smem_optin) + " B shared memory per block, need " +
               std::to_string(smem);
    return bail(MK_ERR_NOT_RESIDENT);
  }
  if (ctx->opt.weight_format < 0 || ctx->opt.weight_format > 1) {
    ctx->err = "weight_format must be 0 (bf16) or 1 (fp8 e4m3)";
    return bail(MK_ERR_INVALID_ARG);
  }
  const int wbytes = ctx->opt.weight_format == 1 ? 1 : 2;
  if (wbytes == 1 && (cfg->hidden % 16 || cfg->ffn % 16 || (cfg->n_q_heads * cfg->head_dim) % 16)) {
    ctx->err = "fp8 weights need hidden, ffn and n_q_heads * head_dim multiples of 16";
    return bail(MK_ERR_UNSUPPORTED);
  }
  const void* step_k = step_kernel_ptr(wbytes, cfg->head_dim, G);
  if (!step_k) {
    ctx->err = "no step kernel for this head_dim and query heads per KV head";
    return bail(MK_ERR_UNSUPPORTED);
  }
  CKC(cudaFuncSetAttribute(step_k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem));
  int per_sm = 0;
  CKC(cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, step_k, kThreads, smem));
  if (per_sm < 1) {
    ctx->err = "one CTA of the step kernel does not fit on an SM";
    return bail(MK_ERR_NOT_RESIDENT);
  }
  int P = ctx->opt.num_ctas > 0 ? ctx->opt.num_ctas : sms;
  if (P > sms * per_sm) {
    ctx->err = "num_ctas exceeds the co-resident limit";
    return bail(MK_ERR_NOT_RESIDENT);
  }
  std::string perr = build_plan(*cfg, P, ctx->opt.attn_splits, &ctx->plan, wbytes);
  if (!perr.empty()) {
    ctx->err = perr;
    return bail(MK_ERR_INVALID_ARG);
  }
  const Plan& plan = ctx->plan;
  const int L = cfg->n_layers, H = cfg->hidden, nq = cfg->n_q_heads, nkv = cfg->n_kv_heads;
  const int d = cfg->head_dim, F = cfg->ffn, V = cfg->vocab, B = cfg->max_batch;
  const int qkvR = qkv_rows(nq, nkv, d), qd = nq * d, S = plan.attn_splits;
  cudaStream_t st = ctx->stream;

  // ---- packed weights, one allocation
  auto al = [](size_t b) { return (b + 255) & ~(size_t)255; };
  const size_t sz_qkv = (size_t)qkvR * H * 2, sz_o = (size_t)H * qd * 2;
  const size_t sz_gu = (size_t)2 * F * H * 2, sz_dn = (size_t)H * F * 2;
  const size_t per_layer = al(sz_qkv) + al(sz_o) + al(sz_gu) + al(sz_dn);
  const size_t sz_emb = (size_t)V * H * 2;
  size_t total = per_layer * L + al(sz_emb) + (cfg->tied_embeddings ? 0 : al(sz_emb)) +
                 2 * al((size_t)L * H * 2) + al((size_t)H * 2) +
                 (cfg->qkv_bias ? al((size_t)L * qkvR * 2) : 0);
  uint8_t* wbuf = nullptr;
  if ((rc = dalloc(ctx, &wbuf, total))) return bail(rc);
  uint8_t* cur = wbuf;
  auto take = [&](size_t b) { uint8_t* p = cur; cur += al(b); return p; };
  std::vector<const uint16_t*> w_qkv(L), w_o(L), w_gu(L), w_dn(L);
  for (int l = 0; l < L; ++l) {
    const mk_layer_weights& Lw = w->layers[l];
    uint16_t* pq = (uint16_t*)take(sz_qkv);
    uint16_t* po = (uint16_t*)take(sz_o);
    uint16_t* pg = (uint16_t*)take(sz_gu);
    uint16_t* pd = (uint16_t*)take(sz_dn);
    CKC(launch_pack_qkv(pq, (const uint16_t*)Lw.wq, (const uint16_t*)Lw.wk, (const uint16_t*)Lw.wv, H,
                        G, d, qkvR, st));
    CKC(cudaMemcpyAsync(po, Lw.wo, sz_o, cudaMemcpyDeviceToDevice, st));
    CKC(launch_pack_gateup(pg, (const uint16_t*)Lw.w_gate, (const uint16_t*)Lw.w_up, H, F, st));
    CKC(cudaMemcpyAsync(pd, Lw.w_down, sz_dn, cudaMemcpyDeviceToDevice, st));
    w_qkv[l] = pq; w_o[l] = po; w_gu[l] = pg; w_dn[l] = pd;
    ctx->pw.qkv.push_back(pq); ctx->pw.o.push_back(po);
    ctx->pw.gu.push_back(pg); ctx->pw.dn.push_back(pd);
  }
  uint16_t* emb = (uint16_t*)take(sz_emb);
  CKC(cudaMemcpyAsync(emb, w->embed, sz_emb, cudaMemcpyDeviceToDevice, st));
  uint16_t* lm = emb;
  if (!cfg->tied_embeddings) {
    lm = (uint16_t*)take(sz_emb);
    CKC(cudaMemcpyAsync(lm, w->lm_head, sz_emb, cudaMemcpyDeviceToDevice, st));
  }
  uint16_t* an = (uint16_t*)take((size_t)L * H * 2);
  uint16_t* fn = (uint16_t*)take((size_t)L * H * 2);
  uint16_t* finaln = (uint16_t*)take((size_t)H * 2);
  for (int l = 0; l < L; ++l) {
    CKC(cudaMemcpyAsync(an + (size_t)l * H, w->layers[l].attn_norm, (size_t)H * 2, cudaMemcpyDeviceToDevice, st));
    CKC(cudaMemcpyAsync(fn + (size_t)l * H, w->layers[l].ffn_norm, (size_t)H * 2, cudaMemcpyDeviceToDevice, st));
  }
  CKC(cudaMemcpyAsync(finaln, w->final_norm, (size_t)H * 2, cudaMemcpyDeviceToDevice, st));
  uint16_t* bq = nullptr;
  if (cfg->qkv_bias) {
    bq = (uint16_t*)take((size_t)L * qkvR * 2);
    for (int l = 0; l < L; ++l)
      CKC(launch_pack_qkv_bias(bq + (size_t)l * qkvR, (const uint16_t*)w->layers[l].bq,
                               (const uint16_t*)w->layers[l].bk, (const uint16_t*)w->layers[l].bv, G, d,
                               qkvR, st));
  }
  // fp8 decode weights: codes and row scales of every GEMV matrix; the bf16
  // copies above are overwritten with the dequantized values (one model for
  // the decode GEMVs, the tensor-core prefill and the batched step)
  std::vector<const uint8_t*> c_qkv(L), c_o(L), c_gu(L), c_dn(L);
  const uint8_t* c_lm = nullptr;
  if (wbytes == 1) {
    // one allocation per matrix: rows x K codes, then (16-byte aligned) the
    // rows' fp32 scales -- where the kernel looks for them
    auto quant = [&](uint16_t* wm, int rows, int K, const uint8_t** code_out) {
      const size_t off = ((size_t)rows * K + 15) & ~(size_t)15;
      uint8_t* codes = nullptr;
      int r2 = dalloc(ctx, &codes, off + (size_t)rows * 4);
      if (r2) return r2;
      if (launch_quantize_fp8_rows(wm, codes, reinterpret_cast<float*>(codes + off), rows, K, st) !=
          cudaSuccess)
        return (int)MK_ERR_CUDA;
      *code_out = codes;
      return 0;
    };
    for (int l = 0; l < L; ++l) {
      if ((rc = quant(const_cast<uint16_t*>(w_qkv[l]), qkvR, H, &c_qkv[l])) ||
          (rc = quant(const_cast<uint16_t*>(w_o[l]), H, qd, &c_o[l])) ||
          (rc = quant(const_cast<uint16_t*>(w_gu[l]), 2 * F, H, &c_gu[l])) ||
          (rc = quant(const_cast<uint16_t*>(w_dn[l]), H, F, &c_dn[l])))
        return bail(rc);
    }
    if ((rc = quant(lm, V, H, &c_lm))) return bail(rc);
  }
  if ((size_t)(cur - wbuf) > total) {
    ctx->err = "internal: weight buffer overflow";
    return bail(MK_ERR_INVALID_ARG);
  }

  // ---- RoPE table, KV cache, activations, sync words
  std::vector<float> hc, hs;
  host_rope_table(cfg->max_seq, d, cfg->rope_theta, hc, hs);
  float *rc_d = nullptr, *rs_d = nullptr;
  if ((rc = dalloc(ctx, &rc_d, hc.size() * 4))) return bail(rc);
  if ((rc = dalloc(ctx, &rs_d, hs.size() * 4))) return bail(rc);
  CKC(cudaMemcpyAsync(rc_d, hc.data(), hc.size() * 4, cudaMemcpyHostToDevice, st));
  CKC(cudaMemcpyAsync(rs_d, hs.data(), hs.size() * 4, cudaMemcpyHostToDevice, st));
  // KV cache: contiguous (one max_seq page per request slot) or a pool of
  // pages assigned to slots through a block table as positions are reached
  // ("LLM高速化勉強会資料" slides 15-17: PagedAttention)
  const int page = ctx->opt.kv_page_tokens;
  if (page < 0 || (page > 0 && page % kKeyBlock)) {
    ctx->err = "kv_page_tokens must be 0 (contiguous) or a positive multiple of 64";
    return bail(MK_ERR_INVALID_ARG);
  }
  ctx->kv_paged = page > 0;
  ctx->kv_page = ctx->kv_paged ? page : cfg->max_seq;
  ctx->kv_pps = ctx->kv_paged ? (cfg->max_seq + page - 1) / page : 1;
  ctx->kv_pool = ctx->kv_paged ? (ctx->opt.kv_pool_pages > 0 ? ctx->opt.kv_pool_pages : B * ctx->kv_pps)
                               : B;
  if (ctx->opt.kv_pool_pages < 0) {
    ctx->err = "kv_pool_pages must be >= 0";
    return bail(MK_ERR_INVALID_ARG);
  }
  ctx->kv_table_h.assign((size_t)B * ctx->kv_pps, -1);
  if (ctx->kv_paged) {
    for (int p = ctx->kv_pool - 1; p >= 0; --p) ctx->kv_free.push_back(p);
  } else {
    for (int sl = 0; sl < B; ++sl) ctx->kv_table_h[sl] = sl;
  }
  if ((rc = dalloc(ctx, &ctx->kv_table_d, ctx->kv_table_h.size() * 4))) return bail(rc);
  CKC(cudaMemcpyAsync(ctx->kv_table_d, ctx->kv_table_h.data(), ctx->kv_table_h.size() * 4,
                      cudaMemcpyHostToDevice, st));
  ctx->kv_bytes = (size_t)ctx->kv_pool * L * nkv * ctx->kv_page * d * 2;
  uint16_t *kc = nullptr, *vc = nullptr;
  if ((rc = dalloc(ctx, &kc, ctx->kv_bytes))) return bail(rc);
  if ((rc = dalloc(ctx, &vc, ctx->kv_bytes))) return bail(rc);
  CKC(cudaMemsetAsync(kc, 0, ctx->kv_bytes, st));
  CKC(cudaMemsetAsync(vc, 0, ctx->kv_bytes, st));
  float *x = nullptr, *q = nullptr, *att = nullptr, *act = nullptr, *part = nullptr;
  unsigned long long* am = nullptr;
  if ((rc = dalloc(ctx, &x, (size_t)B * H * 4))) return bail(rc);
  if ((rc = dalloc(ctx, &q, (size_t)B * qd * 4))) return bail(rc);
  if ((rc = dalloc(ctx, &att, (size_t)B * qd * 4))) return bail(rc);
  if ((rc = dalloc(ctx, &act, (size_t)B * F * 4))) return bail(rc);
  if ((rc = dalloc(ctx, &part, (size_t)B * nkv * S * G * attn_part_stride(d) * 4))) return bail(rc);
  if ((rc = dalloc(ctx, &am, (size_t)B * plan.n_lm_slots * 8))) return bail(rc);
  CKC(cudaMemsetAsync(x, 0, (size_t)B * H * 4, st));
  if ((rc = dalloc(ctx, &ctx->hidden_all, (size_t)B * H * 4))) return bail(rc);
  uint32_t *events = nullptr, *tickets = nullptr, *epoch = nullptr;
  int32_t* status = nullptr;
  if ((rc = dalloc(ctx, &events, (size_t)plan.n_events * 4))) return bail(rc);
  if ((rc = dalloc(ctx, &tickets, (size_t)plan.n_tickets * 4))) return bail(rc);
  if ((rc = dalloc(ctx, &epoch, 16))) return bail(rc);
  if ((rc = dalloc(ctx, &status, 16))) return bail(rc);
  CKC(cudaMemsetAsync(events, 0, (size_t)plan.n_events * 4, st));
  CKC(cudaMemsetAsync(tickets, 0, (size_t)plan.n_tickets * 4, st));
  CKC(cudaMemsetAsync(epoch, 0, 16, st));
  CKC(cudaMemsetAsync(status, 0, 16, st));

  // ---- task graph upload (weight pointers patched per kind and layer)
  std::vector<Task> tasks = plan.tasks;
  for (Task& t : tasks) {
    switch (t.kind) {
      case T_QKV: t.w = w_qkv[t.layer]; break;
      case T_OPROJ: t.w = w_o[t.layer]; break;
      case T_GATEUP: t.w = w_gu[t.layer]; break;
      case T_DOWN: t.w = w_dn[t.layer]; break;
      case T_LMHEAD: t.w = lm; break;
      default: t.w = nullptr; break;
    }
    if (wbytes == 1) {  // the decode GEMVs stream the fp8 codes
      const uint8_t* c = nullptr;
      switch (t.kind) {
        case T_QKV: c = c_qkv[t.layer]; break;
        case T_OPROJ: c = c_o[t.layer]; break;
        case T_GATEUP: c = c_gu[t.layer]; break;
        case T_DOWN: c = c_dn[t.layer]; break;
        case T_LMHEAD: c = c_lm; break;
        default: break;
      }
      if (c) t.w = reinterpret_cast<const uint16_t*>(c);
    }
  }
  if ((rc = dalloc(ctx, &ctx->d_tasks, tasks.size() * sizeof(Task)))) return bail(rc);
  if ((rc = dalloc(ctx, &ctx->d_queue, plan.queue.size() * 4))) return bail(rc);
  if ((rc = dalloc(ctx, &ctx->d_queue_off, plan.queue_off.size() * 4))) return bail(rc);
  CKC(cudaMemcpyAsync(ctx->d_tasks, tasks.data(), tasks.size() * sizeof(Task), cudaMemcpyHostToDevice, st));
  CKC(cudaMemcpyAsync(ctx->d_queue, plan.queue.data(), plan.queue.size() * 4, cudaMemcpyHostToDevice, st));
  CKC(cudaMemcpyAsync(ctx->d_queue_off, plan.queue_off.data(), plan.queue_off.size() * 4,
                      cudaMemcpyHostToDevice, st));
  if ((rc = dalloc(ctx, &ctx->d_sp, sizeof(StepParams)))) return bail(rc);
  if ((rc = dalloc(ctx, &ctx->d_tokens, kMaxBatch * 4))) return bail(rc);
  if ((rc = dalloc(ctx, &ctx->d_ids, kMaxBatch * 4))) return bail(rc);
  CKC(cudaMallocHost(&ctx->h_pinned, 2 * kMaxBatch * 4));

  ModelDev& m = ctx->md;
  m.n_layers = L; m.hidden = H; m.n_q = nq; m.n_kv = nkv; m.head_dim = d; m.ffn = F; m.vocab = V;
  // max_batch here is the graph's request count (one; see mk_decode_step):
  // the KV cache holds B slots, addressed through StepParams::kv_slot.
  m.group = G; m.max_seq = cfg->max_seq; m.max_batch = 1; m.attn_splits = S;
  m.qkv_bias = cfg->qkv_bias ? 1 : 0;
  m.rms_eps = cfg->rms_eps;
  m.attn_scale = (float)(1.0 / std::sqrt((double)d));
  m.n_lm_slots = plan.n_lm_slots;
  m.timeout_ms = ctx->opt.timeout_ms > 0 ? ctx->opt.timeout_ms : 1000;
  m.wbytes = wbytes;
  m.l2_prefetch_chunks = ctx->opt.l2_prefetch == 0 ? kDefaultL2Prefetch
                                                  : (ctx->opt.l2_prefetch < 0 ? 0 : ctx->opt.l2_prefetch);
  m.trace = nullptr;
  m.embed = emb; m.lm_head = lm; m.final_norm = finaln; m.attn_norm = an; m.ffn_norm = fn;
  m.bqkv = bq; m.rope_cos = rc_d; m.rope_sin = rs_d; m.kcache = kc; m.vcache = vc;
  m.kv_table = ctx->kv_table_d; m.kv_page = ctx->kv_page; m.kv_pps = ctx->kv_pps;
  m.kv_pool = ctx->kv_pool; m.n_tickets = plan.n_tickets;
  m.x = x; m.q = q; m.attn = att; m.act = act; m.part = part; m.am = am;
  m.events = events; m.tickets = tickets; m.epoch = epoch; m.status = status;
  m.status_info = status + 1;
  CKC(cudaStreamSynchronize(st));
  CKC(cudaGetLastError());
  *out = ctx;
  return MK_OK;
#undef CKC
}

static int check_ctx(mk_ctx* ctx) {
  if (!ctx) return MK_ERR_INVALID_ARG;
  if (ctx->poisoned) return fail(ctx, MK_ERR_POISONED, "context poisoned by an earlier device error");
  return MK_OK;
}

static int check_step_args(mk_ctx* ctx, const int32_t* pos_host, int n_req) {
  if (n_req < 1 || n_req > ctx->cfg.max_batch) return fail(ctx, MK_ERR_INVALID_ARG, "n_req out of range");
  if (!pos_host) return fail(ctx, MK_ERR_INVALID_ARG, "pos_host is null");
  for (int r = 0; r < n_req; ++r)
    if (pos_host[r] < 0 || pos_host[r] >= ctx->cfg.max_seq)
      return fail(ctx, MK_ERR_POS_RANGE, "position " + std::to_string(pos_host[r]) + " outside [0, max_seq)");
  return MK_OK;
}

// Request slots of a call: slots_host, or 0..n_req-1 when it is NULL.  They
// must lie in [0, max_batch) and differ from each other.
static int resolve_slots(mk_ctx* ctx, const int32_t* slots_host, int n_req, int32_t* out) {
  for (int r = 0; r < n_req; ++r) {
    out[r] = slots_host ? slots_host[r] : r;
    if (out[r] < 0 || out[r] >= ctx->cfg.max_batch)
      return fail(ctx, MK_ERR_INVALID_ARG, "slot " + std::to_string(out[r]) + " outside [0, max_batch)");
    for (int q = 0; q < r; ++q)
      if (out[q] == out[r]) return fail(ctx, MK_ERR_INVALID_ARG, "a slot appears twice");
  }
  return MK_OK;
}

// Paged cache: assigns free pages to every logical page of `slot` that
// positions [0, n_pos) touch and that has none yet (recorded for upload).
static int kv_ensure(mk_ctx* ctx, int slot, int n_pos) {
  if (!ctx->kv_paged) return MK_OK;
  const int need = (n_pos + ctx->kv_page - 1) / ctx->kv_page;
  for (int i = 0; i < need; ++i) {
    int32_t& e = ctx->kv_table_h[(size_t)slot * ctx->kv_pps + i];
    if (e >= 0) continue;
    if (ctx->kv_free.empty()) return fail(ctx, MK_ERR_OOM, "KV page pool exhausted");
    e = ctx->kv_free.back();
    ctx->kv_free.pop_back();
    ctx->kv_pending.emplace_back(slot * ctx->kv_pps + i, e);
  }
  return MK_OK;
}

// Enqueues the recorded table entries on the context's stream (a small kernel
// carries them as arguments: no host buffer has to outlive the call).
static int kv_flush(mk_ctx* ctx) {
  constexpr int kBatch = 32;
  for (size_t i = 0; i < ctx->kv_pending.size(); i += kBatch) {
    int idx[kBatch], val[kBatch];
    const int n = (int)std::min<size_t>(kBatch, ctx->kv_pending.size() - i);
    for (int j = 0; j < n; ++j) {
      idx[j] = ctx->kv_pending[i + j].first;
      val[j] = ctx->kv_pending[i + j].second;
    }
    CK(launch_kv_table_update(ctx->kv_table_d, idx, val, n, ctx->stream));
  }
  ctx->kv_pending.clear();
  return MK_OK;
}

static int decode_step_impl(mk_ctx* ctx, const int32_t* tokens_dev, const int32_t* pos_host,
                            const int32_t* slots_host, int n_req, float* logits_dev,
                            int32_t* next_ids_dev);

extern "C" int mk_decode_step(mk_ctx* ctx, const int32_t* tokens_dev, const int32_t* pos_host,
                              int n_req, float* logits_dev, int32_t* next_ids_dev) {
  return decode_step_impl(ctx, tokens_dev, pos_host, nullptr, n_req, logits_dev, next_ids_dev);
}

extern "C" int mk_decode_step_slots(mk_ctx* ctx, const int32_t* tokens_dev, const int32_t* pos_host,
                                    const int32_t* slots_host, int n_req, float* logits_dev,
                                    int32_t* next_ids_dev) {
  if (!slots_host) return fail(ctx, MK_ERR_INVALID_ARG, "slots_host is null");
  return decode_step_impl(ctx, tokens_dev, pos_host, slots_host, n_req, logits_dev, next_ids_dev);
}

static int decode_step_impl(mk_ctx* ctx, const int32_t* tokens_dev, const int32_t* pos_host,
                            const int32_t* slots_host, int n_req, float* logits_dev,
                            int32_t* next_ids_dev) {
  int rc = check_ctx(ctx);
  if (rc) return rc;
  if (!tokens_dev) return fail(ctx, MK_ERR_INVALID_ARG, "tokens_dev is null");
  if ((rc = check_step_args(ctx, pos_host, n_req))) return rc;
  int32_t slots[kMaxBatch];
  if ((rc = resolve_slots(ctx, slots_host, n_req, slots))) return rc;
  for (int r = 0; r < n_req; ++r)
    if ((rc = kv_ensure(ctx, slots[r], pos_host[r] + 1))) return rc;
  if ((rc = kv_flush(ctx))) return rc;
  const int H = ctx->cfg.hidden, V = ctx->cfg.vocab;
  // Several requests: by default one batched step that streams every weight
  // matrix once (tensor-core GEMMs over the requests' columns).
  if (n_req > 1 && ctx->mode == MK_MODE_MEGAKERNEL && ctx->opt.batch_sequential <= 0 &&
      prefill_gemm_supported(ctx->md)) {
    if (!ctx->bs.params) {
      const std::string e = batch_alloc(ctx->md, ctx->plan.num_ctas, &ctx->bs, &ctx->allocs);
      if (!e.empty()) return fail(ctx, MK_ERR_CUDA, e);
    }
    BatchParams hp{};
    hp.n = n_req;
    for (int r = 0; r < n_req; ++r) {
      hp.pos[r] = pos_host[r];
      hp.slot[r] = slots[r];
      hp.src[r] = r;
    }
    CK(cudaMemcpyAsync(ctx->bs.tokens, tokens_dev, (size_t)n_req * 4, cudaMemcpyDeviceToDevice,
                       ctx->stream));
    CK(cudaMemcpyAsync(ctx->bs.params, &hp, sizeof hp, cudaMemcpyHostToDevice, ctx->stream));
    const std::string e = batch_step(ctx->md, ctx->pw, ctx->bs, n_req, ctx->plan.num_ctas, ctx->stream);
    if (!e.empty()) return fail(ctx, MK_ERR_CUDA, e);
    if (logits_dev)
      CK(cudaMemcpyAsync(logits_dev, ctx->bs.logits, (size_t)n_req * V * 4, cudaMemcpyDeviceToDevice,
                         ctx->stream));
    if (next_ids_dev)
      CK(cudaMemcpyAsync(next_ids_dev, ctx->bs.ids, (size_t)n_req * 4, cudaMemcpyDeviceToDevice,
                         ctx->stream));
    ctx->last_n_req = n_req;
    ctx->last_batched = true;
    return MK_OK;
  }
  // Otherwise the requests run through the one-request graph in turn, each on
  // its own KV-cache slot (every request streams the weights again); with
  // several requests the residual stream of each is kept for mk_copy_hidden.
  for (int r = 0; r < n_req; ++r) {
    StepParams sp{};
    sp.n_req = 1;
    sp.pos[0] = pos_host[r];
    sp.kv_slot[0] = slots[r];
    sp.tokens = tokens_dev + r;
    sp.logits = logits_dev ? logits_dev + (size_t)r * V : nullptr;
    sp.next_ids = next_ids_dev ? next_ids_dev + r : nullptr;
    sp.want_logits = logits_dev != nullptr;
    if ((rc = enqueue_step(ctx, sp))) return rc;
    if (n_req > 1)
      CK(cudaMemcpyAsync(ctx->hidden_all + (size_t)r * H, ctx->md.x, (size_t)H * 4,
                         cudaMemcpyDeviceToDevice, ctx->stream));
  }
  ctx->last_n_req = n_req;
  ctx->last_batched = false;
  return MK_OK;
}

extern "C" int mk_decode_steps(mk_ctx* ctx, const int32_t* token_dev, int pos0, int n_steps,
                               int32_t* ids_dev, float* last_logits_dev) {
  int rc = check_ctx(ctx);
  if (rc) return rc;
  if (ctx->mode != MK_MODE_MEGAKERNEL)
    return fail(ctx, MK_ERR_UNSUPPORTED, "the device-resident loop runs in megakernel mode only");
  if (!token_dev || !ids_dev || n_steps < 1) return fail(ctx, MK_ERR_INVALID_ARG, "bad argument");
  if (pos0 < 0 || (long long)pos0 + n_steps > ctx->cfg.max_seq)
    return fail(ctx, MK_ERR_POS_RANGE, "positions " + std::to_string(pos0) + ".." +
                                           std::to_string(pos0 + n_steps - 1) + " outside [0, max_seq)");
  if ((rc = kv_ensure(ctx, 0, pos0 + n_steps)) || (rc = kv_flush(ctx))) return rc;
  StepParams sp{};
  sp.n_req = 1;
  sp.pos[0] = pos0;
  sp.kv_slot[0] = 0;
  sp.tokens = token_dev;
  sp.logits = last_logits_dev;
  sp.next_ids = ids_dev;
  sp.want_logits = last_logits_dev != nullptr;
  KernelArgs a;
  fill_args(ctx, a, 0, &sp, nullptr, false);
  a.n_steps = n_steps;
  a.ids_seq = ids_dev;
  CK(launch_step(a, ctx->plan.num_ctas, true, ctx->stream));
  ctx->last_n_req = 1;
  ctx->last_batched = false;
  return MK_OK;
}

extern "C" int mk_decode_step_host(mk_ctx* ctx, const int32_t* tokens_host, const int32_t* pos_host,
                                   int n_req, int32_t* next_ids_host) {
  int rc = check_ctx(ctx);
  if (rc) return rc;
  if (!tokens_host || !next_ids_host) return fail(ctx, MK_ERR_INVALID_ARG, "null host buffer");
  if ((rc = check_step_args(ctx, pos_host, n_req))) return rc;
  for (int r = 0; r < n_req; ++r)  // host tokens: checked before anything is enqueued
    if (tokens_host[r] < 0 || tokens_host[r] >= ctx->cfg.vocab)
      return fail(ctx, MK_ERR_TOKEN_RANGE,
                  "token id " + std::to_string(tokens_host[r]) + " outside [0, vocab)");
  memcpy(ctx->h_pinned, tokens_host, (size_t)n_req * 4);
  CK(cudaMemcpyAsync(ctx->d_tokens, ctx->h_pinned, (size_t)n_req * 4, cudaMemcpyHostToDevice, ctx->stream));
  if ((rc = mk_decode_step(ctx, ctx->d_tokens, pos_host, n_req, nullptr, ctx->d_ids))) return rc;
  CK(cudaMemcpyAsync(ctx->h_pinned + kMaxBatch, ctx->d_ids, (size_t)n_req * 4, cudaMemcpyDeviceToHost,
                     ctx->stream));
  CK(cudaStreamSynchronize(ctx->stream));
  memcpy(next_ids_host, ctx->h_pinned + kMaxBatch, (size_t)n_req * 4);
  return MK_OK;
}

static int prefill_impl(mk_ctx* ctx, const int32_t* tokens_dev, const int32_t* offsets_host,
                        const int32_t* slots_host, int n_req, float* last_logits_dev,
                        int32_t* next_ids_dev);

extern "C" int mk_prefill(mk_ctx* ctx, const int32_t* tokens_dev, const int32_t* offsets_host,
                          int n_req, float* last_logits_dev, int32_t* next_ids_dev) {
  return prefill_impl(ctx, tokens_dev, offsets_host, nullptr, n_req, last_logits_dev, next_ids_dev);
}

extern "C" int mk_prefill_slots(mk_ctx* ctx, const int32_t* tokens_dev, const int32_t* offsets_host,
                                const int32_t* slots_host, int n_req, float* last_logits_dev,
                                int32_t* next_ids_dev) {
  if (!slots_host) return fail(ctx, MK_ERR_INVALID_ARG, "slots_host is null");
  return prefill_impl(ctx, tokens_dev, offsets_host, slots_host, n_req, last_logits_dev,
                      next_ids_dev);
}

static int prefill_impl(mk_ctx* ctx, const int32_t* tokens_dev, const int32_t* offsets_host,
                        const int32_t* slots_host, int n_req, float* last_logits_dev,
                        int32_t* next_ids_dev) {
  int rc = check_ctx(ctx);
  if (rc) return rc;
  if (!tokens_dev || !offsets_host) return fail(ctx, MK_ERR_INVALID_ARG, "null argument");
  if (n_req < 1 || n_req > ctx->cfg.max_batch) return fail(ctx, MK_ERR_INVALID_ARG, "n_req out of range");
  for (int r = 0; r < n_req; ++r) {
    const int len = offsets_host[r + 1] - offsets_host[r];
    if (offsets_host[r] < 0 || len < 1 || len > ctx->cfg.max_seq)
      return fail(ctx, MK_ERR_POS_RANGE, "prompt length outside [1, max_seq]");
  }
  int32_t slots[kMaxBatch];
  if ((rc = resolve_slots(ctx, slots_host, n_req, slots))) return rc;
  for (int r = 0; r < n_req; ++r)
    if ((rc = kv_ensure(ctx, slots[r], offsets_host[r + 1] - offsets_host[r]))) return rc;
  if ((rc = kv_flush(ctx))) return rc;
  // Tensor-core path: every position but each prompt's last through the
  // whole-sequence operators; the last position then runs as a decode step
  // (its logits and greedy id).  Otherwise every position is a decode step:
  // position t appends its K/V and attends over 0..t.
  const bool gemm_path = ctx->opt.prefill_steps <= 0 && prefill_gemm_supported(ctx->md);
  PfOutputs out;
  if (gemm_path) {
    if (!ctx->ps.max_tokens) {
      const int cap = std::min(kPrefillBlockTokens, ctx->cfg.max_seq * ctx->cfg.max_batch);
      const std::string e = prefill_alloc(ctx->md, std::max(cap, 1), &ctx->ps, &ctx->allocs);
      if (!e.empty()) return fail(ctx, MK_ERR_CUDA, e);
    }
    bool timed_out = false;
    const bool persistent = ctx->opt.prefill_per_operator <= 0 && ctx->opt.prefill_attention != 1;
    std::string e;
    if (persistent) {
      // the persistent prefill also runs the last positions (LM head, id)
      out.logits = last_logits_dev;
      out.ids = next_ids_dev;
      for (int r = 0; r < n_req; ++r)
        out.hidden[r] = n_req > 1 ? ctx->hidden_all + (size_t)r * ctx->cfg.hidden : ctx->md.x;
      e = prefill_mk_run(ctx->md, ctx->pw, ctx->ps, ctx->stream, tokens_dev, offsets_host, slots,
                         n_req, ctx->plan.num_ctas, &ctx->allocs, &timed_out, &out);
    } else {
      e = prefill_run(ctx->md, ctx->pw, ctx->ps, ctx->stream, tokens_dev, offsets_host, slots,
                      n_req, ctx->opt.prefill_attention != 1, &timed_out);
    }
    if (!e.empty()) {
      ctx->poisoned = true;
      return fail(ctx, timed_out ? MK_ERR_TIMEOUT : MK_ERR_CUDA, e);
    }
  }
  for (int r = 0; r < n_req; ++r) {
    if (out.folded[r]) continue;  // done inside the persistent prefill
    const int len = offsets_host[r + 1] - offsets_host[r];
    for (int t = gemm_path ? len - 1 : 0; t < len; ++t) {
      StepParams sp{};
      sp.n_req = 1;
      sp.pos[0] = t;
      sp.kv_slot[0] = slots[r];
      sp.tokens = tokens_dev + offsets_host[r] + t;
      const bool last = t == len - 1;
      sp.logits = last && last_logits_dev ? last_logits_dev + (size_t)r * ctx->cfg.vocab : nullptr;
      sp.next_ids = last && next_ids_dev ? next_ids_dev + r : nullptr;
      sp.want_logits = sp.logits != nullptr;
      if ((rc = enqueue_step(ctx, sp))) return rc;
    }
    if (n_req > 1)
      CK(cudaMemcpyAsync(ctx->hidden_all + (size_t)r * ctx->cfg.hidden, ctx->md.x,
                         (size_t)ctx->cfg.hidden * 4, cudaMemcpyDeviceToDevice, ctx->stream));
  }
  ctx->last_n_req = n_req;
  ctx->last_batched = false;
  return MK_OK;
}

extern "C" int mk_copy_hidden(mk_ctx* ctx, float* hidden_dev, int n_req) {
  int rc = check_ctx(ctx);
  if (rc) return rc;
  if (!hidden_dev || n_req < 1 || n_req > ctx->cfg.max_batch) return fail(ctx, MK_ERR_INVALID_ARG, "bad argument");
  if (n_req > ctx->last_n_req) return fail(ctx, MK_ERR_INVALID_ARG, "n_req exceeds the last step's");
  const float* src = ctx->last_batched ? ctx->bs.x : (ctx->last_n_req > 1 ? ctx->hidden_all : ctx->md.x);
  CK(cudaMemcpyAsync(hidden_dev, src, (size_t)n_req * ctx->cfg.hidden * 4, cudaMemcpyDeviceToDevice,
                     ctx->stream));
  return MK_OK;
}

extern "C" int mk_copy_activation(mk_ctx* ctx, int which, float* dst_dev, int n) {
  int rc = check_ctx(ctx);
  if (rc) return rc;
  if (ctx->last_batched) return fail(ctx, MK_ERR_INVALID_ARG, "the last step was batched");
  const mk_config& c = ctx->cfg;
  const float* src = nullptr;
  int len = 0;
  switch (which) {
    case MK_ACT_Q: src = ctx->md.q; len = c.n_q_heads * c.head_dim; break;
    case MK_ACT_ATTN: src = ctx->md.attn; len = c.n_q_heads * c.head_dim; break;
    case MK_ACT_FFN: src = ctx->md.act; len = c.ffn; break;
    case MK_ACT_X: src = ctx->md.x; len = c.hidden; break;
    default: return fail(ctx, MK_ERR_INVALID_ARG, "bad activation selector");
  }
  if (!dst_dev || n < 0 || n > len) return fail(ctx, MK_ERR_INVALID_ARG, "bad copy size");
  CK(cudaMemcpyAsync(dst_dev, src, (size_t)n * 4, cudaMemcpyDeviceToDevice, ctx->stream));
  return MK_OK;
}

extern "C" int mk_kv_pointer(mk_ctx* ctx, int req, int layer, int kv_head, int which, void** out_dev) {
  if (!ctx || !out_dev) return MK_ERR_INVALID_ARG;
  const mk_config& c = ctx->cfg;
  if (req < 0 || req >= c.max_batch || layer < 0 || layer >= c.n_layers || kv_head < 0 ||
      kv_head >= c.n_kv_heads || which < 0 || which > 1)
    return fail(ctx, MK_ERR_INVALID_ARG, "bad KV index");
  if (ctx->kv_paged)
    return fail(ctx, MK_ERR_UNSUPPORTED, "a paged KV cache has no contiguous rows: use mk_copy_kv");
  const size_t off = (((size_t)req * c.n_layers + layer) * c.n_kv_heads + kv_head) * (size_t)c.max_seq * c.head_dim;
  *out_dev = (which ? ctx->md.vcache : ctx->md.kcache) + off;
  return MK_OK;
}

extern "C" int mk_copy_kv(mk_ctx* ctx, int req, int layer, int kv_head, int which, int n, void* dst_dev) {
  int rc = check_ctx(ctx);
  if (rc) return rc;
  const mk_config& c = ctx->cfg;
  if (req < 0 || req >= c.max_batch || layer < 0 || layer >= c.n_layers || kv_head < 0 ||
      kv_head >= c.n_kv_heads || which < 0 || which > 1)
    return fail(ctx, MK_ERR_INVALID_ARG, "bad KV index");
  if (!dst_dev || n < 0 || n > c.max_seq) return fail(ctx, MK_ERR_INVALID_ARG, "bad copy size");
  const size_t row = (size_t)c.head_dim;
  const uint16_t* base = which ? ctx->md.vcache : ctx->md.kcache;
  for (int p0 = 0; p0 < n; p0 += ctx->kv_page) {  // one copy per page
    const int phys = ctx->kv_table_h[(size_t)req * ctx->kv_pps + p0 / ctx->kv_page];
    if (phys < 0) return fail(ctx, MK_ERR_INVALID_ARG, "positions without a KV page");
    const int rows = std::min(ctx->kv_page, n - p0);
    const uint16_t* src =
        base + (((size_t)phys * c.n_layers + layer) * c.n_kv_heads + kv_head) * ctx->kv_page * row;
    CK(cudaMemcpyAsync(static_cast<uint16_t*>(dst_dev) + (size_t)p0 * row, src, rows * row * 2,
                       cudaMemcpyDeviceToDevice, ctx->stream));
  }
  return MK_OK;
}

extern "C" int mk_kv_release(mk_ctx* ctx, int slot) {
  int rc = check_ctx(ctx);
  if (rc) return rc;
  if (slot < 0 || slot >= ctx->cfg.max_batch) return fail(ctx, MK_ERR_INVALID_ARG, "bad slot");
  if (!ctx->kv_paged) return MK_OK;  // a contiguous slot keeps its region
  for (int i = 0; i < ctx->kv_pps; ++i) {
    int32_t& e = ctx->kv_table_h[(size_t)slot * ctx->kv_pps + i];
    if (e < 0) continue;
    ctx->kv_free.push_back(e);
    e = -1;
    ctx->kv_pending.emplace_back(slot * ctx->kv_pps + i, -1);
  }
  return kv_flush(ctx);
}

extern "C" int mk_kv_set_pages(mk_ctx* ctx, int slot, const int32_t* pages_host, int n_pages) {
  int rc = check_ctx(ctx);
  if (rc) return rc;
  if (!ctx->kv_paged) return fail(ctx, MK_ERR_UNSUPPORTED, "the KV cache is not paged");
  if (slot < 0 || slot >= ctx->cfg.max_batch || n_pages < 0 || n_pages > ctx->kv_pps ||
      (n_pages && !pages_host))
    return fail(ctx, MK_ERR_INVALID_ARG, "bad slot or page count");
  if ((rc = mk_kv_release(ctx, slot))) return rc;
  for (int i = 0; i < n_pages; ++i) {
    auto it = std::find(ctx->kv_free.begin(), ctx->kv_free.end(), pages_host[i]);
    if (it == ctx->kv_free.end()) {
      mk_kv_release(ctx, slot);
      return fail(ctx, MK_ERR_INVALID_ARG, "page " + std::to_string(pages_host[i]) +
                                               " is out of range or already assigned");
    }
    ctx->kv_free.erase(it);
    ctx->kv_table_h[(size_t)slot * ctx->kv_pps + i] = pages_host[i];
    ctx->kv_pending.emplace_back(slot * ctx->kv_pps + i, pages_host[i]);
  }
  return kv_flush(ctx);
}

extern "C" int mk_kv_get_pages(mk_ctx* ctx, int slot, int32_t* pages_out, int cap) {
  if (!ctx || slot < 0 || slot >= ctx->cfg.max_batch || cap < 0 || (cap && !pages_out))
    return MK_ERR_INVALID_ARG;
  for (int i = 0; i < std::min(cap, ctx->kv_pps); ++i)
    pages_out[i] = ctx->kv_table_h[(size_t)slot * ctx->kv_pps + i];
  return ctx->kv_pps;
}

extern "C" int mk_kv_free_pages(mk_ctx* ctx) {
  if (!ctx) return MK_ERR_INVALID_ARG;
  return (int)ctx->kv_free.size();
}

extern "C" int mk_set_prefill_trace(mk_ctx* ctx, unsigned long long* trace_dev, int capacity) {
  int rc = check_ctx(ctx);
  if (rc) return rc;
  if (trace_dev && capacity <= 0) return fail(ctx, MK_ERR_INVALID_ARG, "trace capacity must be > 0");
  ctx->ps.pf.trace = reinterpret_cast<uint64_t*>(trace_dev);
  ctx->ps.pf.trace_cap = trace_dev ? capacity : 0;
  return MK_OK;
}

extern "C" int mk_set_trace(mk_ctx* ctx, unsigned long long* trace_dev) {
  if (!ctx) return MK_ERR_INVALID_ARG;
  ctx->md.trace = trace_dev;
  return MK_OK;
}

extern "C" int mk_set_mode(mk_ctx* ctx, int mode) {
  if (!ctx) return MK_ERR_INVALID_ARG;
  if (mode < MK_MODE_MEGAKERNEL || mode > MK_MODE_PER_OP_GRAPH) return fail(ctx, MK_ERR_INVALID_ARG, "bad mode");
  ctx->mode = mode;
  return MK_OK;
}

extern "C" int mk_status(mk_ctx* ctx) {
  if (!ctx) return MK_ERR_INVALID_ARG;
  if (ctx->poisoned) return MK_ERR_POISONED;
  cudaError_t e = cudaStreamSynchronize(ctx->stream);
  if (e == cudaSuccess) e = cudaGetLastError();
  if (e != cudaSuccess) {
    ctx->poisoned = true;
    return fail(ctx, MK_ERR_CUDA, std::string("device error: ") + cudaGetErrorString(e));
  }
  int32_t st[2] = {0, 0};
  e = cudaMemcpy(st, ctx->md.status, sizeof st, cudaMemcpyDeviceToHost);
  if (e != cudaSuccess) {
    ctx->poisoned = true;
    return fail(ctx, MK_ERR_CUDA, std::string("status read: ") + cudaGetErrorString(e));
  }
  if (st[0] != 0) {
    ctx->poisoned = true;
    // a timeout's detail: the task index of an event wait, or (negative) which
    // shared-memory wait gave up: -1 ring full, -2 ready, -3 done, -4 ring
    // empty, -5 the producer's final drain of its copies
    const char* what = st[0] == MK_ERR_TIMEOUT
                           ? (st[1] >= 0 ? "event wait timed out at task "
                                         : "shared-memory wait timed out, kind ")
                       : st[0] == MK_ERR_TOKEN_RANGE ? "token id out of range: "
                       : st[0] == MK_ERR_BOUNDS      ? "bounds check failed (debug build), check "
                                                     : "device error, detail ";
    return fail(ctx, st[0], std::string(what) + std::to_string(st[1]));
  }
  if (ctx->bs.err) {  // the batched step's GEMM pipeline waits
    int32_t be = 0;
    if (cudaMemcpy(&be, ctx->bs.err, 4, cudaMemcpyDeviceToHost) == cudaSuccess && be) {
      ctx->poisoned = true;
      return fail(ctx, MK_ERR_TIMEOUT, "batched step: a GEMM pipeline wait timed out");
    }
  }
  return MK_OK;
}

extern "C" int mk_build_flags(void) {
#ifdef MK_DEBUG_BOUNDS
  return MK_BUILD_DEBUG_BOUNDS;
#else
  return 0;
#endif
}

extern "C" const char* mk_last_error(const mk_ctx* ctx) {
  return ctx ? ctx->err.c_str() : g_create_error.c_str();
}

extern "C" void mk_destroy(mk_ctx* ctx) {
  if (!ctx) return;
  cudaStreamSynchronize(ctx->stream);
  release(ctx);
  delete ctx;
}

extern "C" int mk_inject_stall(mk_ctx* ctx, int task) {
  if (!ctx) return MK_ERR_INVALID_ARG;
  if (ctx->poisoned) return MK_ERR_POISONED;
  const std::vector<Task>& tasks = ctx->plan.tasks;
  if (task < 0) {
    for (size_t i = 0; i < tasks.size(); ++i)
      if (tasks[i].wait_ev >= 0) {
        task = (int)i;
        break;
      }
  }
  if (task < 0 || task >= (int)tasks.size() || tasks[task].wait_ev < 0)
    return fail(ctx, MK_ERR_INVALID_ARG, "inject stall: no such task waiting on an event");
  // one more completion than the event receives per step: never reached
  const uint32_t raised = tasks[task].wait_count + 1u;
  uint8_t* field = reinterpret_cast<uint8_t*>(ctx->d_tasks + task) + offsetof(Task, wait_count);
  cudaError_t e = cudaMemcpyAsync(field, &raised, sizeof raised, cudaMemcpyHostToDevice, ctx->stream);
  if (e == cudaSuccess) e = cudaStreamSynchronize(ctx->stream);
  if (e != cudaSuccess) return fail(ctx, MK_ERR_CUDA, std::string("inject stall: ") + cudaGetErrorString(e));
  return MK_OK;
}

extern "C" int mk_inject_prefill_stall(mk_ctx* ctx, int task) {
  int rc = check_ctx(ctx);
  if (rc) return rc;
  if (task < -1) return fail(ctx, MK_ERR_INVALID_ARG, "inject prefill stall: task must be >= -1");
  ctx->ps.pf.stall_task = task;
  return MK_OK;
}

extern "C" int mk_read_probe(const void* src_dev, size_t bytes, unsigned long long* sink_dev,
                             void* stream) {
  if (!src_dev || !sink_dev || bytes == 0 || bytes % 16 || !aligned16(src_dev))
    return fail(nullptr, MK_ERR_INVALID_ARG, "read probe: bad buffer");
  int dev = 0, sms = 0;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
    return fail(nullptr, MK_ERR_CUDA, "read probe: no device");
  cudaError_t e = launch_read_probe(src_dev, bytes, sink_dev, sms, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return fail(nullptr, MK_ERR_CUDA, cudaGetErrorString(e));
  return MK_OK;
}
