// plan.cpp -- host-side task-graph (tGraph) builder.
//
// "LLMs in einen MegaKernel kompilieren ...", "Part 1. Compiler": the
// operator graph is refined into tasks sized for one SM, linked by events,
// so that dependencies follow data tiles rather than kernel boundaries.
// "MPK: A Compiler and Runtime for Mega-Kernelizing Tensor Programs" §3: a
// predictable task is queued ahead of time.  A decode step is fully
// predictable, so every CTA gets a fixed ahead-of-time queue here; only the
// attention key ranges depend on the runtime position and are resolved on
// the device.
//
// Per layer the stages are QKV -> ATTN -> OPROJ -> GATEUP -> DOWN, then the
// LM head.  Each GEMV stage is cut into one contiguous row range per CTA
// (further cut so the per-task partial sums fit in shared memory); attention
// is cut per (batch slot, KV head, key split).  Dependencies:
//   ATTN(l,g)  waits until every QKV(l) task that wrote rows of group g is done
//   OPROJ(l)   waits for every ATTN(l) split; its prologue merges the partials
//   GATEUP(l)  waits for all OPROJ(l)    (RMSNorm needs the whole residual)
//   DOWN(l)    waits for all GATEUP(l)   (the GEMV needs the whole activation)
//   QKV(l+1) and the LM head wait for all DOWN(l).
// Queues list tasks in this topological order, so with all CTAs co-resident
// the earliest unfinished task can always run: no deadlock.
#include "plan.h"

#include <algorithm>
#include <cstdio>

namespace mk {

std::string validate_config(const mk_config& c) {
  char buf[256];
  if (c.n_layers <= 0 || c.hidden <= 0 || c.n_q_heads <= 0 || c.n_kv_heads <= 0 ||
      c.head_dim <= 0 || c.ffn <= 0 || c.vocab <= 0)
    return "all sizes must be positive";
  if (c.head_dim != 64 && c.head_dim != 128) return "head_dim must be 64 or 128";
  if (c.n_q_heads % c.n_kv_heads) return "n_q_heads must be a multiple of n_kv_heads";
  if (c.hidden % 8 || c.ffn % 8) return "hidden and ffn must be multiples of 8";
  int qd = c.n_q_heads * c.head_dim;
  if (c.hidden > 16384 || c.ffn > 16384) return "GEMV inputs are limited to 16384";
  if (qd > 8192) return "n_q_heads * head_dim is limited to 8192";
  int G = c.n_q_heads / c.n_kv_heads;
  // attention merge scratch: 8 warps x G heads x (d + 4) floats
  if (8 * G * attn_part_stride(c.head_dim) * 4 > kScratchBytes) {
    snprintf(buf, sizeof buf, "query heads per KV head (%d) too large for head_dim %d", G,
             c.head_dim);
    return buf;
  }
  if (G > 16) return "at most 16 query heads per KV head";
  if (c.max_seq <= 0) return "max_seq must be positive";
  if (c.max_batch < 1 || c.max_batch > kMaxBatch) return "max_batch must be 1..8";
  if (!(c.rms_eps >= 0.0f)) return "rms_eps must be >= 0";
  if (!(c.rope_theta > 0.0)) return "rope_theta must be > 0";
  return "";
}

namespace {

struct Builder {
  const mk_config& c;
  int P;
  Plan& p;
  EventMap ev;
  std::vector<std::vector<int>> per_cta;  // megakernel queues

  int wb = 2;  // bytes per GEMV weight

  Builder(const mk_config& c_, int P_, Plan& p_, int wbytes)
      : c(c_), P(P_), p(p_), ev{c_.n_layers, c_.n_kv_heads}, per_cta(P_), wb(wbytes) {}

  // A GEMV over K columns of wb-byte weights has the geometry of a bf16 GEMV
  // over K * wb / 2 columns (same bytes per row; a 16-byte piece then holds
  // 16 / wb columns).
  int kb(int K) const { return K * wb / 2; }

  int add(const Task& t, int cta) {
    p.tasks.push_back(t);
    p.cta_of_task.push_back(cta);
    int id = (int)p.tasks.size() - 1;
    per_cta[cta].push_back(id);
    for (int e = 0; e < t.n_sig; ++e) p.event_count[t.sig_ev0 + e] += 1;
    return id;
  }

  // Splits [0, N) into one range per CTA (row ranges aligned to `align`),
  // then each range into pieces of at most max_rows.  Calls f(cta, r0, r1).
  template <class F>
  void split_rows(int N, int align, int max_rows, F f) {
    int units = N / align;
    int n_cta = std::min(P, units);
    for (int k = 0; k < n_cta; ++k) {
      int u0 = (int)((long long)k * units / n_cta), u1 = (int)((long long)(k + 1) * units / n_cta);
      int r0 = u0 * align, r1 = (k == n_cta - 1) ? N : u1 * align;
      if (r1 <= r0) continue;
      int cta = (int)((long long)k * P / n_cta);
      int pieces = (r1 - r0 + max_rows - 1) / max_rows;
      int span_units = (r1 - r0 + align - 1) / align;
      for (int q = 0; q < pieces; ++q) {
        int a = r0 + (int)((long long)q * span_units / pieces) * align;
        int b = (q == pieces - 1) ? r1 : r0 + (int)((long long)(q + 1) * span_units / pieces) * align;
        if (b > a) f(cta, a, b);
      }
    }
  }

  Task gemv_task(int kind, int layer, int K, int r0, int r1) {
    Task t{};
    t.kind = kind;
    t.layer = layer;
    t.row0 = r0;
    t.row1 = r1;
    t.req = 0;
    t.wait_ev = -1;
    t.wait_count = 0;
    t.sig_ev0 = -1;
    t.n_sig = 0;
    t.K = K;
    t.tpr = gemv_tpr(kb(K));
    t.chunk_rows = gemv_chunk_rows(kb(K));
    t.w = nullptr;
    t.aux = -1;
    t.stage = kind == T_LMHEAD ? c.n_layers * 5 : layer * 5 + kind;
    return t;
  }

  void build(int splits) {
    const int L = c.n_layers, H = c.hidden, nq = c.n_q_heads, nkv = c.n_kv_heads;
    // The graph covers one request; a step over several requests runs it once
    // per request (each with its own KV-cache slot).
    const int d = c.head_dim, G = nq / nkv, F = c.ffn, V = c.vocab, B = 1;
    const int qkvR = qkv_rows(nq, nkv, d), per_group = (G + 2) * d;
    p.event_count.assign(ev.count(), 0);
    p.n_events = ev.count();
    p.attn_splits = splits;
    p.n_tickets = kAttnTicketBase + L * B * nkv;
    p.lm_ticket = 0;
    p.n_stages = 5 * L + 1;
    for (int l = 0; l < L; ++l) {
      // QKV: rows of whole RoPE pairs; signal every group the rows touch.
      split_rows(qkvR, 2, gemv_max_task_rows(kb(H)), [&](int cta, int r0, int r1) {
        Task t = gemv_task(T_QKV, l, H, r0, r1);
        if (l > 0) { t.wait_ev = ev.down(l - 1); }
        int g0 = r0 / per_group, g1 = (r1 - 1) / per_group;
        t.sig_ev0 = ev.qkv(l, g0);
        t.n_sig = g1 - g0 + 1;
        add(t, cta);
      });
      // ATTN: (batch slot, group, split), spread over the CTAs.
      int A = B * nkv * splits;
      for (int a = 0; a < A; ++a) {
        int req = a / (nkv * splits), g = (a / splits) % nkv, s = a % splits;
        Task t{};
        t.kind = T_ATTN;
        t.layer = l;
        t.row0 = g;
        t.row1 = s;
        t.req = req;
        t.wait_ev = ev.qkv(l, g);
        t.sig_ev0 = ev.attn(l);
        t.n_sig = 1;
        t.K = d;
        t.aux = -1;
        t.stage = l * 5 + T_ATTN;
        int cta = (int)((long long)a * P / A);
        add(t, cta);
      }
      split_rows(H, 1, gemv_max_task_rows(kb(nq * d)), [&](int cta, int r0, int r1) {
        Task t = gemv_task(T_OPROJ, l, nq * d, r0, r1);
        t.wait_ev = ev.attn(l);
        t.sig_ev0 = ev.oproj(l);
        t.n_sig = 1;
        add(t, cta);
      });
      split_rows(2 * F, 2, gemv_max_task_rows(kb(H)), [&](int cta, int r0, int r1) {
        Task t = gemv_task(T_GATEUP, l, H, r0, r1);
        t.wait_ev = ev.oproj(l);
        t.sig_ev0 = ev.gateup(l);
        t.n_sig = 1;
        add(t, cta);
      });
      split_rows(H, 1, gemv_max_task_rows(kb(F)), [&](int cta, int r0, int r1) {
        Task t = gemv_task(T_DOWN, l, F, r0, r1);
        t.wait_ev = ev.gateup(l);
        t.sig_ev0 = ev.down(l);
        t.n_sig = 1;
        add(t, cta);
      });
    }
    // LM head: one argmax slot per CTA; its tasks keep a running best in
    // shared memory and only the CTA's last one publishes it.
    int n_lm = 0, n_slots = 0, last_cta = -1;
    std::vector<int> lm_ids;
    split_rows(V, 1, gemv_max_task_rows(kb(H)), [&](int cta, int r0, int r1) {
      Task t = gemv_task(T_LMHEAD, L, H, r0, r1);
      t.layer = L - 1;
      t.wait_ev = ev.down(L - 1);
      if (cta != last_cta) {
        ++n_slots;
        last_cta = cta;
      }
      t.aux = n_slots - 1;
      lm_ids.push_back(add(t, cta));
      ++n_lm;
    });
    for (size_t i = 0; i < lm_ids.size(); ++i) {
      Task& t = p.tasks[lm_ids[i]];
      const bool first = i == 0 || p.tasks[lm_ids[i - 1]].aux != t.aux;
      const bool last = i + 1 == lm_ids.size() || p.tasks[lm_ids[i + 1]].aux != t.aux;
      t.req = (first ? 1 : 0) | (last ? 2 : 0);
    }
    p.n_lm_tasks = n_lm;
    p.n_lm_slots = n_slots;
    // Thresholds: every wait targets the full per-step count of its event.
    for (auto& t : p.tasks)
      if (t.wait_ev >= 0) t.wait_count = p.event_count[t.wait_ev];
    // Queue sets: 0 = everything in topological order; 1 + s = stage s.
    p.queue.clear();
    p.queue_off.assign((size_t)(p.n_stages + 1) * (P + 1), 0);
    for (int cta = 0; cta < P; ++cta) {
      p.queue_off[cta] = (int)p.queue.size();
      for (int id : per_cta[cta]) p.queue.push_back(id);
    }
    p.queue_off[P] = (int)p.queue.size();
    for (int s = 0; s < p.n_stages; ++s) {
      int base = p.set_offset(s + 1);
      for (int cta = 0; cta < P; ++cta) {
        p.queue_off[base + cta] = (int)p.queue.size();
        for (int id : per_cta[cta])
          if (p.tasks[id].stage == s) p.queue.push_back(id);
      }
      p.queue_off[base + P] = (int)p.queue.size();
    }
    long long wb = 0;
    wb += (long long)L * qkvR * H * 2;
    wb += (long long)L * H * nq * d * 2;
    wb += (long long)L * 2 * F * H * 2;
    wb += (long long)L * H * F * 2;
    wb += (long long)V * H * 2;
    p.weight_bytes = wb;
  }
};

}  // namespace

std::string build_plan(const mk_config& c, int num_ctas, int attn_splits, Plan* out, int wbytes) {
  std::string err = validate_config(c);
  if (!err.empty()) return err;
  if (num_ctas <= 0) return "num_ctas must be positive";
  int per_batch = std::max(1, num_ctas / c.n_kv_heads);
  int S = attn_splits > 0 ? attn_splits
                          : std::max(1, std::min(per_batch, (c.max_seq + 63) / 64));
  if (S > 4096) return "attn_splits too large";
  *out = Plan{};
  out->num_ctas = num_ctas;
  if (wbytes != 1 && wbytes != 2) return "wbytes must be 1 or 2";
  Builder b(c, num_ctas, *out, wbytes);
  b.build(S);
  // every GEMV task must have a geometry the kernel instantiates: (pieces per
  // thread, rows per chunk) = (1, 4), (2, 2), (3, 1) or (4, 1) (fp8: the first two)
  for (const Task& t : out->tasks) {
    if (t.kind == T_ATTN) continue;
    const int pieces = t.K * wbytes / 16;
    const int cpt = (pieces + t.tpr - 1) / t.tpr, nr = t.chunk_rows / (kWorkerThreads / t.tpr);
    const bool ok = (cpt == 1 && nr == 4) || (cpt == 2 && nr == 2) ||
                    (wbytes == 2 && ((cpt == 3 && nr == 1) || (cpt == 4 && nr == 1)));
    if (!ok) return "internal: a GEMV geometry the kernel does not implement";
  }
  return "";
}

}  // namespace mk

// ------------------------------------------------------------- C-ABI

struct mk_plan {
  mk::Plan p;
  mk_config cfg;
};

extern "C" int mk_plan_build(const mk_config* cfg, const mk_options* opt, int num_ctas,
                             mk_plan** out) {
  if (!cfg || !out) return MK_ERR_INVALID_ARG;
  *out = nullptr;
  mk_plan* h = new mk_plan();
  h->cfg = *cfg;
  std::string err = mk::build_plan(*cfg, num_ctas, opt ? opt->attn_splits : 0, &h->p,
                                   opt && opt->weight_format == 1 ? 1 : 2);
  if (!err.empty()) {
    delete h;
    return MK_ERR_INVALID_ARG;
  }
  *out = h;
  return MK_OK;
}

extern "C" int mk_plan_get_info(const mk_plan* h, mk_plan_info* info) {
  if (!h || !info) return MK_ERR_INVALID_ARG;
  const mk::Plan& p = h->p;
  info->num_ctas = p.num_ctas;
  info->n_tasks = (int)p.tasks.size();
  info->n_events = p.n_events;
  info->n_stages = p.n_stages;
  info->attn_splits = p.attn_splits;
  info->n_lm_tasks = p.n_lm_tasks;
  info->ring_slots = mk::kRingSlots;
  info->slot_bytes = mk::kSlotBytes;
  info->smem_bytes = 0;
  info->threads_per_cta = mk::kThreads;
  info->weight_bytes_per_step = p.weight_bytes;
  return MK_OK;
}

extern "C" int mk_plan_get_tasks(const mk_plan* h, mk_plan_task* out, int cap) {
  if (!h || (!out && cap > 0)) return MK_ERR_INVALID_ARG;
  int n = std::min<int>(cap, (int)h->p.tasks.size());
  for (int i = 0; i < n; ++i) {
    const mk::Task& t = h->p.tasks[i];
    mk_plan_task& o = out[i];
    o.kind = t.kind;
    o.layer = t.layer;
    o.row0 = t.row0;
    o.row1 = t.row1;
    o.req = t.req;
    o.wait_event = t.wait_ev;
    o.wait_count = (int)t.wait_count;
    o.signal_event0 = t.sig_ev0;
    o.n_signal = t.n_sig;
    o.cta = h->p.cta_of_task[i];
    o.stage = t.stage;
  }
  return n;
}

extern "C" int mk_plan_get_queue(const mk_plan* h, int cta, int* out, int cap) {
  if (!h || cta < 0 || cta >= h->p.num_ctas) return MK_ERR_INVALID_ARG;
  int a = h->p.queue_off[cta], b = h->p.queue_off[cta + 1];
  int n = std::min(cap, b - a);
  for (int i = 0; i < n; ++i) out[i] = h->p.queue[a + i];
  return b - a;
}

extern "C" int mk_plan_get_event_counts(const mk_plan* h, int* out, int cap) {
  if (!h) return MK_ERR_INVALID_ARG;
  int n = std::min<int>(cap, (int)h->p.event_count.size());
  for (int i = 0; i < n; ++i) out[i] = (int)h->p.event_count[i];
  return (int)h->p.event_count.size();
}

extern "C" void mk_plan_destroy(mk_plan* h) { delete h; }

extern "C" int mk_qkv_row_source(const mk_config* cfg, int r, int* which, int* head, int* dim) {
  if (!cfg || !which || !head || !dim) return MK_ERR_INVALID_ARG;
  if (cfg->n_kv_heads <= 0 || cfg->n_q_heads % cfg->n_kv_heads) return MK_ERR_INVALID_ARG;
  int rows = mk::qkv_rows(cfg->n_q_heads, cfg->n_kv_heads, cfg->head_dim);
  if (r < 0 || r >= rows) return MK_ERR_INVALID_ARG;
  mk::qkv_source(r, cfg->n_q_heads / cfg->n_kv_heads, cfg->head_dim, which, head, dim);
  return MK_OK;
}
