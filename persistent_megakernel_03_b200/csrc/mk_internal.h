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
constexpr int kProducerWarp = 0;                  // bulk-copy (TMA) issue
constexpr int kSchedulerWarp = 1;                 // event waits
constexpr int kFirstWorkerWarp = 2;
constexpr int kThreads = (kFirstWorkerWarp + kWorkerWarps) * 32; // 576
constexpr int kSlotBytes = 32768;                 // one weight-ring stage
constexpr int kRingSlots = 6;                     // 192 KB of weights in flight / buffered
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
  // KV cache [slot][layer][kv_head][max_seq][head_dim] bf16
  uint16_t* kcache;
  uint16_t* vcache;
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

// GEMV geometry for an input of K columns on kWorkerThreads threads:
// the K/8 16-byte column chunks are spread over `tpr` threads (a row-lane);
// 512/tpr row-lanes work on different rows of the same ring chunk.
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
// Largest number of output rows one task may own (partial-sum buffer bound).
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
