// mk_internal.h -- data structures shared by the host-side task-graph builder
// and the persistent kernel.
//
// Task graph ("LLMs in einen MegaKernel kompilieren ...", "Part 1. Compiler":
// each task is a unit of work for one SM, each event a synchronisation point
// with a counter; "Ereignisbasierte Ausführung": a finished task increments
// its event counter and an event whose counter reached its threshold releases
// the tasks that depend on it).  Counters are never reset: a task waits until
// its event reached count_per_step * (epoch + 1), where epoch counts the
// decode steps that completed before this launch.
#pragma once
#include <stdint.h>

#ifdef __CUDACC__
#define MK_HD __host__ __device__ __forceinline__
#else
#define MK_HD inline
#endif

namespace mk {

enum TaskKind : int32_t { T_QKV = 0, T_ATTN = 1, T_OPROJ = 2, T_GATEUP = 3, T_DOWN = 4, T_LMHEAD = 5 };

constexpr int kMaxBatch = 8;
constexpr int kWorkerWarps = 16;                  // compute warps per CTA
constexpr int kWorkerThreads = kWorkerWarps * 32; // 512
// Bulk copies issued by one thread run one after another (each ~0.4 us
// whatever its size up to 32 KB, measured), which caps a single issuer at
// ~70-80 GB/s per SM -- barely above an SM's share of HBM.  Copies from
// different issuing warps overlap, so the ring is filled by two producer
// warps, each owning every other chunk (and so every other slot).
constexpr int kProducerWarps = 2;                 // bulk-copy (TMA) issue, warps 0 .. 1
constexpr int kSchedulerWarp = kProducerWarps;    // event waits
constexpr int kFirstWorkerWarp = kProducerWarps + 1;
constexpr int kThreads = (kFirstWorkerWarp + kWorkerWarps) * 32; // 608
constexpr int kSlotBytes = 32768;                 // one weight-ring stage
constexpr int kRingSlots = 6;                     // 192 KB of weights in flight / buffered
static_assert(kRingSlots % 2 == 0, "each producer warp owns every other slot");
constexpr int kScratchBytes = 20480;              // GEMV partial sums / attention merge
constexpr int kYBufFloats = 1024;                 // reduced GEMV outputs of one task
constexpr int kMaxTaskRowsCap = 1024;
constexpr int kDefaultL2Prefetch = 0;             // chunks prefetched into L2 at a stall

// One task.  64 bytes, read by all three warp roles of the owning CTA.
struct Task {
  int32_t kind;
  int32_t layer;
  int32_t row0, row1;      // GEMV: packed output rows [row0, row1); ATTN: group, split
  int32_t req;             // ATTN: batch slot; LMHEAD: bit 0 first / bit 1 last LM task of its CTA
  int32_t wait_ev;         // -1: no wait
  uint32_t wait_count;     // signals per step
  int32_t sig_ev0;         // first event bumped on completion (-1: none)
  int32_t n_sig;           // number of consecutive events bumped
  int32_t K;               // GEMV input length (columns)
  int32_t tpr;             // GEMV: threads per row-lane (32..512, power of two)
  int32_t chunk_rows;      // GEMV: rows per ring chunk
  const uint16_t* w;       // GEMV: packed bf16 matrix base (row-major, K columns)
  int32_t aux;             // LMHEAD: argmax slot of the owning CTA
  int32_t stage;           // operator stage (per-operator mode)
};
static_assert(sizeof(Task) == 64, "Task layout");

// Step inputs, written by the host before every launch.
struct StepParams {
  int32_t n_req;
  int32_t pos[kMaxBatch];
  int32_t kv_slot[kMaxBatch];   // which request cache each batch slot uses
  const int32_t* tokens;        // device, n_req ids
  float* logits;                // device, n_req x vocab (nullable)
  int32_t* next_ids;            // device, n_req (nullable)
  int32_t want_logits;
  int32_t pad_;
};

// Everything the kernel needs that does not change between steps.
struct ModelDev {
  int32_t n_layers, hidden, n_q, n_kv, head_dim, ffn, vocab, group;
  int32_t max_seq, max_batch, attn_splits, qkv_bias;
  float rms_eps, attn_scale;
  int32_t n_lm_slots, timeout_ms;  // CTAs holding LM-head tasks (argmax slots)
  int32_t l2_prefetch_chunks;  // chunks past the ring prefetched into L2 when a task must wait (0: off)
  int32_t wbytes;              // bytes per GEMV weight: 2 (bf16) or 1 (fp8 e4m3; a matrix's
                               // fp32 row scales follow its codes, 16-byte aligned)
  // packed weights
  const uint16_t* embed;       // [vocab][hidden]
  const uint16_t* lm_head;     // [vocab][hidden] (== embed when tied)
  const uint16_t* final_norm;  // [hidden]
  const uint16_t* attn_norm;   // [layers][hidden]
  const uint16_t* ffn_norm;    // [layers][hidden]
  const uint16_t* bqkv;        // [layers][qkv_rows] packed order (nullable)

  // rope table [max_seq][head_dim/2]
  const float* rope_cos;
  const float* rope_sin;
  // KV cache: a pool of pages [page][layer][kv_head][kv_page][head_dim] bf16, K
  // and V separate; logical page i of request slot s (positions
  // [i*kv_page, (i+1)*kv_page)) is physical page kv_table[s*kv_pps + i].  A
  // contiguous cache is the case kv_page = max_seq, kv_pps = 1, page s = slot s.
  uint16_t* kcache;
  uint16_t* vcache;
  const int32_t* kv_table;     // [max slots][kv_pps]
  int32_t kv_page;             // positions per page (a multiple of 64, or max_seq)
  int32_t kv_pps;              // table entries per slot
  int32_t kv_pool;             // pages in the pool
  int32_t n_tickets;           // entries of `tickets`
  // activations (fp32, per batch slot)
  float* x;        // [batch][hidden] residual stream
  float* q;        // [batch][n_q*head_dim] rotated queries
  float* attn;     // [batch][n_q*head_dim] attention output
  float* act;      // [batch][ffn] SwiGLU output
  float* part;     // [batch][n_kv][splits][group][attn_part_stride(d)] split partials
  unsigned long long* am; // [batch][n_lm_slots] packed (value, index) argmax partials
  // sync
  uint32_t* events;
  uint32_t* tickets;       // [0]: LM-head argmax; [kAttnTicketBase + (layer*batch + req)*n_kv + g]:
                           // attention split-merge tickets
  uint32_t* epoch;         // completed steps
  int32_t* status;         // 0 ok, else an MK_ERR_* code
  int32_t* status_info;    // task index / detail of the first error
  // optional per-task trace: 8 words per queue entry of the megakernel queue set
  // (%globaltimer ns at: event satisfied, workers start, input loaded, first
  // chunk ready, last chunk consumed, epilogue done, end; then cta << 32 | task)
  unsigned long long* trace;
};

struct KernelArgs {
  ModelDev m;
  const Task* tasks;
  const int32_t* queue;      // task indices
  const int32_t* queue_off;  // [num_ctas + 1] for this launch's queue set
  StepParams sp_val;         // step inputs by value ...
  const StepParams* sp_ptr;  // ... or, when non-null, from device memory (graph replay)
  int32_t n_steps;           // decode steps in this launch (1, or more: device-resident loop)
  int32_t* ids_seq;          // n_steps > 1: step s writes its greedy id to ids_seq[s] and
                             // step s + 1 embeds it (step 0 embeds sp.tokens[0])
  int32_t no_wait;           // per-operator mode: kernel boundaries order the tasks
};

// ---------------------------------------------------------------- layouts

// Keys per attention block: the ring's key chunk (d = 128), and the unit in
// which split ranges are rounded and pages are sized.
constexpr int kKeyBlock = 64;

#ifdef __CUDACC__
// Debug-bounds build (compiled with -DMK_DEBUG_BOUNDS): every task checks the
// indices of its global and shared-memory accesses against their buffers;
// a failed check records MK_ERR_BOUNDS with a code naming the check in the
// status word and the access is skipped (the launch goes on; no trap).  In
// the normal build the checks compile to nothing.
enum BoundsWhere : int32_t {
  kBndChunkRows = 1, kBndChunkBytes = 2, kBndKvKey = 3, kBndKvPage = 4, kBndSlotRow = 5,
  kBndScratch = 6, kBndYbuf = 7, kBndQ = 8, kBndResidual = 9, kBndAct = 10, kBndLogits = 11,
  kBndArgmax = 12, kBndPart = 13, kBndAttnOut = 14, kBndTicket = 15
};
__device__ __forceinline__ bool bounds_ok(const ModelDev& m, bool ok, int where) {
#ifdef MK_DEBUG_BOUNDS
  if (!ok && atomicCAS(m.status, 0, -10 /* MK_ERR_BOUNDS */) == 0) m.status_info[0] = where;
  return ok;
#else
  (void)m; (void)where;
  return true;
#endif
}

// Element offset of the cached K/V row of (slot, layer, KV head, position).
// Host code guarantees every page a launch touches is assigned; an entry that
// is not (-1) maps to page 0, so an access always stays inside the pool.
__device__ __forceinline__ size_t kv_row(const ModelDev& m, int slot, int layer, int g, int key) {
  const int lp = key / m.kv_page;
  int phys = __ldg(m.kv_table + slot * m.kv_pps + lp);
  if (!bounds_ok(m, key >= 0 && key < m.max_seq, kBndKvKey)) return 0;
  if (!bounds_ok(m, phys >= 0 && phys < m.kv_pool, kBndKvPage)) return 0;
  phys = phys < 0 ? 0 : phys;
  return ((((size_t)phys * m.n_layers + layer) * m.n_kv + g) * (size_t)m.kv_page +
          (size_t)(key - lp * m.kv_page)) * (size_t)m.head_dim;
}
#endif

MK_HD int qkv_rows(int n_q, int n_kv, int d) { return (n_q + 2 * n_kv) * d; }

// Packed fused-QKV row r -> source (which 0 q / 1 k / 2 v, head, dim).
// Rows are grouped per KV head g: its G query heads, its K head, its V head.
// Inside a q or k head, packed rows 2p and 2p+1 are dims p and p + d/2
// (the rotate-half RoPE partners).  V heads keep their natural order.
MK_HD void qkv_source(int r, int G, int d, int* which, int* head, int* dim) {
  int per_group = (G + 2) * d;
  int g = r / per_group;
  int off = r - g * per_group;
  int blk = off / d;
  int within = off - blk * d;
  int rot_dim = (within >> 1) + (within & 1) * (d >> 1);
  if (blk < G) {
    *which = 0; *head = g * G + blk; *dim = rot_dim;
  } else if (blk == G) {
    *which = 1; *head = g; *dim = rot_dim;
  } else {
    *which = 2; *head = g; *dim = within;
  }
}

// GEMV geometry for an input of K columns on kWorkerThreads threads: the K/8
// 16-byte column pieces of a row are spread over `tpr` threads (a row-lane;
// the smallest power of two >= K/8, from a warp to all 512 threads), so each
// thread loads its inputs once and no input is loaded twice by a CTA when
// tpr = 512; the 512/tpr row-lanes work on different rows of a ring chunk,
// `nr` rows each (up to 4, as many as fit a 32 KB chunk).
MK_HD int gemv_tpr(int K) {
  int C = K / 8;
  int t = 32;
  while (t < C && t < kWorkerThreads) t <<= 1;
  return t;
}
MK_HD int gemv_cpt(int K) { int t = gemv_tpr(K); return (K / 8 + t - 1) / t; }
MK_HD int gemv_nr(int K) {
  int rl = kWorkerThreads / gemv_tpr(K);
  int fit = kSlotBytes / (2 * K * rl);
  int nr = 1;
  while (nr * 2 <= fit && nr * 2 <= 4) nr <<= 1;
  return nr;
}
MK_HD int gemv_chunk_rows(int K) { return gemv_nr(K) * (kWorkerThreads / gemv_tpr(K)); }
// Largest number of output rows one task may own (partial-sum buffer bound:
// one fp32 per row and warp of a row-lane).
MK_HD int gemv_max_task_rows(int K) {
  int wpr = gemv_tpr(K) / 32;
  int r = kScratchBytes / (4 * wpr);
  if (r > kYBufFloats) r = kYBufFloats;
  return r;
}

// Attention split partial record: o[d], then m and l, padded to 16 bytes.
MK_HD int attn_part_stride(int d) { return d + 4; }

// First attention merge ticket (ticket 0 is the LM head's).
constexpr int kAttnTicketBase = 1;

// Attention splits holding keys at a context of n_keys: about one split per
// ring chunk of keys, at most the graph's `splits` tasks per KV head.  A
// short context then has one split (no merge) or a few partials to merge.
MK_HD int attn_live_splits(int n_keys, int splits, int keys_per_split) {
  int s = (n_keys + keys_per_split - 1) / keys_per_split;
  return s < 1 ? 1 : (s > splits ? splits : s);
}

// Attention: keys per ring chunk (K rows in the first half of a slot, V rows
// in the second half).
MK_HD int attn_keys_per_chunk(int d) { return (kSlotBytes / 2) / (d * 2); }

}  // namespace mk
