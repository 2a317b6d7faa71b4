/*
 * mk.h -- C-ABI of libmk: batch-1 (and small-batch) transformer decoding on
 * one B200 (sm_100a), each decode step run as ONE persistent megakernel.
 *
 * The method ("LLMs in einen MegaKernel kompilieren, um Low-Latency-Inferenz
 * zu ermöglichen", de.news.hada.io/topic?id=21563, sections "Part 1.
 * Compiler" and "Part 2. Laufzeit"; "MPK: A Compiler and Runtime for
 * Mega-Kernelizing Tensor Programs", gist.science/hi/paper/2512.22219,
 * sections 1-4): the operators of a decode step are cut into SM-sized tasks
 * linked by event counters instead of kernel boundaries; one kernel with one
 * CTA per SM runs every task; a finished task bumps an event counter, and a
 * task whose event reached its threshold may run.  Here a host-side builder
 * makes the task graph once at mk_create; each CTA gets an ahead-of-time task
 * queue; inside each CTA a scheduler warp waits on the events, a producer warp
 * streams bf16 weights with bulk copies (TMA) into a shared-memory ring that
 * runs ahead across task and layer boundaries, and worker warps compute.
 *
 * The model: embedding table, then transformer blocks (pre-norm RMSNorm,
 * fused QKV projection with optional bias, rotate-half RoPE, KV-cache append,
 * grouped-query attention, O projection + residual, RMSNorm, SwiGLU FFN +
 * residual), final RMSNorm, LM head, greedy argmax ("Crear desde cero un
 * motor de inferencia para LLM usando C++ y CUDA", es.news.hada.io/topic?id=
 * 18295, §1 and §1.1; "LLM高速化勉強会資料" slides 4-6, 9, 28).
 *
 * Conventions for every entry point:
 *   - Return 0 on success or a negative MK_ERR_* code.  Argument errors are
 *     found on the host before anything is enqueued.  Device-side errors
 *     (a wait that timed out, a token id out of range) are reported by
 *     mk_status; after one the context is poisoned and every later call
 *     returns MK_ERR_POISONED.  mk_last_error gives a one-line reason.
 *   - "_dev" pointers are CUDA device pointers, "_host" pointers host memory.
 *   - Work is enqueued on the stream given to mk_create and the call returns
 *     without synchronising (except mk_status, mk_decode_step_host and
 *     mk_create, which synchronise that stream).  Results are valid after a
 *     stream synchronisation.
 *   - One context is not thread-safe; different contexts are independent.
 */
#ifndef MK_H
#define MK_H
#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define MK_OK 0
#define MK_ERR_INVALID_ARG -1  /* bad pointer, size or configuration */
#define MK_ERR_OOM -2          /* device allocation failed */
#define MK_ERR_CUDA -3         /* a CUDA runtime call failed */
#define MK_ERR_TIMEOUT -4      /* a device-side event wait ran out of time */
#define MK_ERR_POS_RANGE -5    /* position outside [0, max_seq) */
#define MK_ERR_NOT_RESIDENT -6 /* one CTA per SM cannot be co-resident */
#define MK_ERR_POISONED -7     /* an earlier device error; destroy the context */
#define MK_ERR_TOKEN_RANGE -8  /* a token id outside [0, vocab) reached the device */
#define MK_ERR_UNSUPPORTED -9  /* valid request this build does not implement */
#define MK_ERR_BOUNDS -10      /* debug-bounds build only: a task's access fell outside its
                                  buffer and was skipped (mk_last_error names the check) */

/* Build properties: bit 0 set in the debug-bounds build (libmk_debug.so, compiled
 * with MK_DEBUG_BOUNDS), where every task checks the indices of its global and
 * shared-memory accesses and reports a violation as MK_ERR_BOUNDS through
 * mk_status instead of performing the access. */
#define MK_BUILD_DEBUG_BOUNDS 1
int mk_build_flags(void);

/* Execution modes of a decode step. */
#define MK_MODE_MEGAKERNEL 0   /* one persistent launch per step (the product) */
#define MK_MODE_PER_OP 1       /* the same task bodies, one launch per operator */
#define MK_MODE_PER_OP_GRAPH 2 /* MK_MODE_PER_OP captured once and replayed as a CUDA graph */

/* Decoder shape.  Sizes in elements.  Limits of this build: head_dim 64 or
 * 128; hidden and ffn multiples of 8 and at most 16384; n_q_heads a multiple
 * of n_kv_heads; max_batch 1..8. */
typedef struct {
  int n_layers, hidden, n_q_heads, n_kv_heads, head_dim, ffn, vocab;
  float rms_eps;
  double rope_theta;
  int qkv_bias;        /* 1: q/k/v projections carry a bias (Qwen2 family) */
  int tied_embeddings; /* 1: the LM head is the embedding table */
  int max_seq;         /* positions per request: 0 .. max_seq-1 */
  int max_batch;       /* requests decoded together per step */
} mk_config;

/* bf16 device pointers in the natural layout, [out_features][in_features]
 * row-major: wq [n_q_heads*head_dim][hidden], wk/wv [n_kv_heads*head_dim]
 * [hidden], wo [hidden][n_q_heads*head_dim], w_gate/w_up [ffn][hidden],
 * w_down [hidden][ffn], norms [hidden], biases [out_features] (NULL without
 * qkv_bias).  mk_create copies and re-packs everything into memory it owns;
 * the caller may free these afterwards. */
typedef struct {
  const void *attn_norm, *wq, *wk, *wv, *bq, *bk, *bv, *wo;
  const void *ffn_norm, *w_gate, *w_up, *w_down;
} mk_layer_weights;

typedef struct {
  const void* embed;              /* [vocab][hidden] */
  const mk_layer_weights* layers; /* host array of n_layers entries */
  const void* final_norm;         /* [hidden] */
  const void* lm_head;            /* [vocab][hidden]; NULL when tied */
} mk_weights;

/* Optional knobs (pass NULL for defaults). */
typedef struct {
  int num_ctas;      /* 0: one CTA per SM of the device */
  int attn_splits;   /* 0: automatic split-KV factor per KV head */
  int timeout_ms;    /* device-side wait limit per event (0: 1000 ms) */
  int mode;          /* MK_MODE_* used by mk_decode_step and mk_prefill */
  int l2_prefetch;   /* when a CTA's next task must wait for its event, the number
                        of 32 KB weight chunks past its shared-memory ring it
                        prefetches into L2 meanwhile; 0: default (off), < 0: off */
  int weight_format; /* 0: bf16 decode weights (default); 1: fp8 e4m3 with one
                        power-of-two scale per row for every GEMV matrix (QKV, O,
                        gate/up, down, LM head): mk_create quantizes the given bf16
                        weights (round to nearest) and replaces its bf16 copies by
                        the dequantized values, which the prefill and the batched
                        step then use -- bf16 weights that already are such values
                        are kept exactly */
  int batch_sequential; /* 1: a step of several requests runs them one after another
                           through the megakernel; 0: default, one batched step */
  int prefill_steps; /* 1: mk_prefill runs every prompt position as a decode step;
                        0: default, the tensor-core prefill (when every contraction
                        length is a multiple of 64) */
  int kv_page_tokens; /* 0: default, a contiguous KV cache (max_seq positions per
                         request slot); > 0, a multiple of 64: the KV cache is a pool
                         of pages of this many positions ("LLM高速化勉強会資料" slides
                         15-17, PagedAttention), assigned to a request slot through a
                         block table as its positions are reached and returned to the
                         pool by mk_kv_release */
  int kv_pool_pages; /* paged cache: pages in the pool (0: enough for every slot at
                        max_seq, i.e. max_batch * ceil(max_seq / kv_page_tokens)) */
  int prefill_per_operator; /* tensor-core prefill only.  0: default, each block of
                               <= 2048 prompt positions runs as ONE persistent
                               kernel (every operator of every layer a task; tasks
                               of different 128-position tiles overlap across
                               operator and layer boundaries, dependencies per
                               tile through event counters; tcgen05 GEMM and
                               attention tasks); 1: one launch per operator and
                               layer.  Both give the same result up to the order
                               of the fp32 additions. */
  int prefill_attention; /* tensor-core prefill only.  0: default, the causal
                            attention on the tensor cores (tcgen05: 128 positions x
                            64 keys per step, online softmax, the fp32 queries and
                            probabilities as two bf16 parts each); 1: on CUDA cores
                            (one warp per position, fp32 throughout; implies
                            prefill_per_operator). */
} mk_options;

typedef struct mk_ctx mk_ctx;

/* Builds the task graph, packs the weights, allocates the KV cache and the
 * activation scratch, uploads the RoPE table and checks that one CTA per SM
 * can be co-resident.  `stream` is a cudaStream_t (NULL: the legacy default
 * stream).  On success *out owns ~(weights + KV cache) of device memory. */
int mk_create(const mk_config* cfg, const mk_weights* w, const mk_options* opt, void* stream,
              mk_ctx** out);

/* Prefill ("LLM高速化勉強会資料" slide 9; "Crear desde cero ..." §1.1): runs
 * the prompt of each request through the model and fills its KV cache at
 * positions 0..len-1.  Requests are packed as one flat token sequence
 * ("LLM高速化勉強会資料" slides 14-16): request r owns tokens
 * [offsets_host[r], offsets_host[r+1]) of tokens_dev; 1 <= len <= max_seq.
 * Writes the last position's logits (n_req x vocab fp32, may be NULL) and
 * greedy next ids (n_req int32, may be NULL).  By default every position runs
 * inside one persistent kernel per block of 2048 positions (the weight
 * contractions and the causal attention on the tensor cores: tcgen05, bf16
 * weights times the fp32 activations split into three bf16 parts, fp32
 * accumulation), the last position's final norm, LM head and greedy id
 * included; a prompt of one position runs as a decode step.  With
 * prefill_per_operator = 1 positions 0..len-2 run one launch per operator and
 * the last as a decode step.  This path allocates its scratch (~0.4 GB for
 * the Llama-3-8B shape) at the first call and synchronises the stream before
 * returning. */
int mk_prefill(mk_ctx* ctx, const int32_t* tokens_dev, const int32_t* offsets_host, int n_req,
               float* last_logits_dev, int32_t* next_ids_dev);

/* One decode step: request r feeds tokens_dev[r] at position pos_host[r]
 * (positions 0..pos-1 must be in its KV cache), appends its K/V at pos, and
 * writes logits_dev[r*vocab ..] (may be NULL) and next_ids_dev[r] (may be
 * NULL).  n_req <= max_batch.  One request: one launch of the persistent
 * megakernel.  Several requests (megakernel mode, contraction lengths
 * multiples of 64): one batched step -- every weight matrix streamed once
 * through tcgen05 GEMMs over the requests' columns, split-KV attention per
 * request and KV head, greedy argmax per request -- replayed from a CUDA
 * graph captured at the first step of that request count.  Otherwise (or
 * with batch_sequential) the requests run one after another through the
 * megakernel, each on its own KV-cache slot. */
int mk_decode_step(mk_ctx* ctx, const int32_t* tokens_dev, const int32_t* pos_host, int n_req,
                   float* logits_dev, int32_t* next_ids_dev);

/* Continuous batching ("LLM高速化勉強会資料" slides 14-17: requests join and
 * leave a running batch between steps).  The same as mk_prefill and
 * mk_decode_step, with request r on KV-cache slot slots_host[r] (distinct
 * values in [0, max_batch)) instead of slot r: a new request is prefilled into
 * a free slot while the other slots keep their caches, and each step decodes
 * any set of occupied slots together (one batched step for 2-8 of them).
 * Logits, ids and mk_copy_hidden rows stay in request order r.  With a paged
 * cache, every page the call's positions need is assigned before the launch
 * (MK_ERR_OOM when the pool has no free page); mk_kv_release returns a
 * finished request's pages. */
int mk_prefill_slots(mk_ctx* ctx, const int32_t* tokens_dev, const int32_t* offsets_host,
                     const int32_t* slots_host, int n_req, float* last_logits_dev,
                     int32_t* next_ids_dev);
int mk_decode_step_slots(mk_ctx* ctx, const int32_t* tokens_dev, const int32_t* pos_host,
                         const int32_t* slots_host, int n_req, float* logits_dev,
                         int32_t* next_ids_dev);

/* Paged KV cache (mk_options.kv_page_tokens > 0).  Logical page i of a slot
 * holds positions [i * page, (i + 1) * page).  mk_kv_release returns every page
 * of `slot` to the pool (a finished request; a no-op for a contiguous cache).
 * mk_kv_set_pages makes pages_host[0..n_pages) (free pool pages, in any order)
 * the slot's logical pages 0..n_pages-1, after releasing its current ones; pages
 * beyond are assigned on demand as usual.  mk_kv_get_pages copies the slot's
 * table row (-1: no page) and returns its length (max_seq / page rounded up).
 * mk_kv_free_pages returns the number of free pages.  Table changes are
 * enqueued on the context's stream. */
int mk_kv_release(mk_ctx* ctx, int slot);
int mk_kv_set_pages(mk_ctx* ctx, int slot, const int32_t* pages_host, int n_pages);
int mk_kv_get_pages(mk_ctx* ctx, int slot, int32_t* pages_out, int cap);
int mk_kv_free_pages(mk_ctx* ctx);

/* n_steps greedy decode steps of request 0 in ONE persistent launch (the
 * device-resident loop): step s runs at position pos0 + s, feeds the id step
 * s - 1 produced (step 0 feeds token_dev[0]), appends its K/V and writes its
 * greedy id to ids_dev[s]; only the last step writes logits (last_logits_dev,
 * vocab fp32, may be NULL).  Inside the launch a step's first layer waits for
 * the previous step's argmax through the device epoch, so no kernel boundary
 * or host round trip separates the steps and the weight prefetch of a step
 * overlaps the previous step's LM head.  Megakernel mode only
 * (MK_ERR_UNSUPPORTED otherwise); pos0 + n_steps <= max_seq
 * (MK_ERR_POS_RANGE).  Results equal n_steps calls of mk_decode_step. */
int mk_decode_steps(mk_ctx* ctx, const int32_t* token_dev, int pos0, int n_steps, int32_t* ids_dev,
                    float* last_logits_dev);

/* mk_decode_step from and to HOST memory: copies the tokens in, runs the
 * step, copies the next ids out and synchronises the stream.  Token ids
 * outside [0, vocab) are rejected before anything is enqueued
 * (MK_ERR_TOKEN_RANGE; the context is not poisoned). */
int mk_decode_step_host(mk_ctx* ctx, const int32_t* tokens_host, const int32_t* pos_host,
                        int n_req, int32_t* next_ids_host);

/* Copies the final residual stream of the last step or prefill (before the
 * final norm), n_req x hidden fp32, to hidden_dev (enqueued on the context's
 * stream); n_req must not exceed that call's. */
int mk_copy_hidden(mk_ctx* ctx, float* hidden_dev, int n_req);

/* Intermediate results of the last single-request step (not the batched
 * step), for per-stage parity checks: which = MK_ACT_Q the rotated queries of
 * the last layer (n_q_heads x head_dim fp32, head-major), MK_ACT_ATTN its
 * attention output (same layout, normalised), MK_ACT_FFN its SwiGLU
 * activation silu(W_gate xn) * (W_up xn) (ffn fp32), MK_ACT_X the residual
 * stream after the last layer (hidden fp32).  Copies n floats from the start
 * of that vector to dst_dev on the context's stream; n must not exceed its
 * length.  MK_ERR_INVALID_ARG after a batched step or for a bad `which`. */
enum { MK_ACT_Q = 0, MK_ACT_ATTN = 1, MK_ACT_FFN = 2, MK_ACT_X = 3 };
int mk_copy_activation(mk_ctx* ctx, int which, float* dst_dev, int n);

/* Device pointer of the bf16 K (which=0) or V (which=1) cache of one request,
 * layer and KV head: max_seq x head_dim elements, row-major.  Contiguous cache
 * only (MK_ERR_UNSUPPORTED when paged: use mk_copy_kv). */
int mk_kv_pointer(mk_ctx* ctx, int req, int layer, int kv_head, int which, void** out_dev);

/* Copies positions [0, n) of one K (which=0) or V (which=1) cache head, bf16
 * n x head_dim, to dst_dev (enqueued on the context's stream; gathered page by
 * page when the cache is paged). */
int mk_copy_kv(mk_ctx* ctx, int req, int layer, int kv_head, int which, int n, void* dst_dev);

/* Per-task timeline of later megakernel steps (diagnostics).  trace_dev
 * holds 8 uint64 per entry of the megakernel's task queues (mk_plan_info
 * n_tasks entries), %globaltimer ns: 0 the task's event was satisfied,
 * 1 workers started, 2 input loaded, 3 first ring chunk ready, 4 last chunk
 * consumed, 5 epilogue done, 6 finished; 7 holds (cta << 32 | task).
 * NULL turns tracing off.  The buffer must outlive the traced steps. */
int mk_set_trace(mk_ctx* ctx, unsigned long long* trace_dev);

/* Per-task timeline of the persistent prefill (the default tensor-core prefill)
 * (diagnostics).  For the tasks of the FIRST block of a later prefill call, in
 * the order the kernel's host graph lists them (at most `capacity` tasks),
 * trace_dev receives 4 uint64 per task, %globaltimer ns: 0 the CTA began
 * waiting for the task's dependencies, 1 they were satisfied, 2 the task
 * finished (its completion signalled); word 3 describes the task: bits 0-15
 * the CTA, 16-19 the kind (0 embedding + norm, 1 GEMM tile, 2 RoPE + KV
 * append, 3 attention, 4 O residual + norm, 5 SwiGLU, 6 down residual +
 * norm), 20-23 the GEMM's matrix (0 QKV, 1 O, 2 gate/up, 3 down), 24-31 the
 * layer, 32-47 the 128-position tile, 48-63 the row tile / query head.
 * NULL turns tracing off.  The buffer must outlive the traced call. */
int mk_set_prefill_trace(mk_ctx* ctx, unsigned long long* trace_dev, int capacity);

/* Selects the execution mode of later steps (MK_MODE_*). */
int mk_set_mode(mk_ctx* ctx, int mode);

/* Synchronises the stream and reports the device status: 0, MK_ERR_TIMEOUT,
 * MK_ERR_TOKEN_RANGE, MK_ERR_BOUNDS (debug-bounds build) or MK_ERR_CUDA.
 * Poisons the context on error. */
int mk_status(mk_ctx* ctx);

const char* mk_last_error(const mk_ctx* ctx);
void mk_destroy(mk_ctx* ctx);

/* Failure-detection hook (host-side injection, no device fault): raises the
 * wait threshold of one task of the megakernel's task graph by one
 * completion, so the event it waits on can never reach it.  The next
 * megakernel step (mk_decode_step of one request, mk_decode_steps, the last
 * prompt position of mk_prefill) stalls there until timeout_ms, records
 * MK_ERR_TIMEOUT, and every CTA leaves the launch through its abort path;
 * mk_status then reports MK_ERR_TIMEOUT and poisons the context, and the
 * CUDA context stays usable.  task: index into the context's task table
 * (0 .. tasks - 1), or < 0 for the first task in table order that waits on
 * an event.  Synchronises the stream.  MK_ERR_INVALID_ARG when the index is
 * out of range or the task waits on no event.  The change is permanent:
 * destroy the context afterwards. */
int mk_inject_stall(mk_ctx* ctx, int task);

/* The same for the persistent prefill: the next mk_prefill[_slots] call
 * raises by one the wait count of task `task` of its first block's graph (in
 * the order the mk_set_prefill_trace records list the tasks; -1: the last
 * task that waits on an event), so that its event never reaches it.  The
 * prefill's waits are bounded (2 x mk_options.timeout_ms): the call returns
 * MK_ERR_TIMEOUT and poisons the context.  Testing aid; no GPU fault. */
int mk_inject_prefill_stall(mk_ctx* ctx, int task);

/* Split-KV grouped-query decode attention for one KV head ("Hạt nhân là gì
 * ...": online softmax, exact up to rounding; "LLM高速化勉強会資料" slides
 * 11-13 and 28).  q_dev: fp32 [n_q_per_kv][head_dim] query rows of the
 * heads that share this KV head; k_dev, v_dev: bf16 [n_keys][head_dim]
 * row-major, 8-byte aligned; out_dev: fp32 [n_q_per_kv][head_dim] =
 * softmax(q K^T / sqrt(head_dim)) V per query head.  The keys are cut into
 * `splits` contiguous blocks of ceil(n_keys / splits), one CTA each; the last
 * CTA to finish merges the blocks.  workspace_dev holds the blocks' partial
 * results and a merge ticket: mk_attention_workspace_bytes(...) bytes, 16-byte
 * aligned, zeroed by the caller before its first use (the op leaves the
 * ticket at zero after every call, so it can be reused on the same stream;
 * two calls in flight at once on one workspace race).  head_dim 64 or 128;
 * n_q_per_kv 1, 2, 4, 7 or 8.  Enqueued on `stream`. */
size_t mk_attention_workspace_bytes(int n_q_per_kv, int head_dim, int splits);
int mk_attention_decode(const float* q_dev, const void* k_dev, const void* v_dev, int n_keys,
                        int n_q_per_kv, int head_dim, int splits, void* workspace_dev,
                        float* out_dev, void* stream);

/* mk_attention_decode without a workspace argument, for callers that cannot
 * allocate device memory (a plugin whose host owns all device memory, a
 * real-time loop that must not enter an allocator, code that may only use
 * the buffers it is given).  No counterpart on the pages: this is a
 * packaging of the op above.  The scratch is a 270,592-byte array compiled
 * into the library, so this entry point never allocates; it serves up to 64
 * splits for 8 query heads per KV head at head_dim 128 (larger requests
 * return MK_ERR_INVALID_ARG, see mk_last_error(NULL)).  Every call looks up
 * the array's device address in the current device's context (no cached
 * pointer survives a context that is torn down and made again) and clears the
 * array's merge ticket with a memset on `stream` before the op.  The first
 * call on a device loads the library's device code there: make it before any
 * stream capture.  All calls on a device share the one array, which keeps the
 * last call's partials: calls that overlap on the GPU (other streams, other
 * threads) race. */
int mk_attention_decode_noalloc(const float* q_dev, const void* k_dev, const void* v_dev,
                                int n_keys, int n_q_per_kv, int head_dim, int splits,
                                float* out_dev, void* stream);

/* Read-only HBM stream probe: every byte of src_dev[0, bytes) is loaded
 * once with 128-bit loads by a grid of (SMs x 4) CTAs; a value derived from
 * the data is written to sink_dev[0] so nothing is elided.  bytes must be a
 * multiple of 16 and src_dev 16-byte aligned.  Enqueued on `stream`.  Used to
 * measure the practical read ceiling the decode step is compared with. */
int mk_read_probe(const void* src_dev, size_t bytes, unsigned long long* sink_dev, void* stream);

/* ---------------------------------------------------------------------
 * Introspection of the task graph (host only, no GPU needed).
 * mk_plan_build makes the same graph mk_create would for `num_ctas` CTAs.
 */
typedef struct {
  int num_ctas, n_tasks, n_events, n_stages;
  int attn_splits, n_lm_tasks, ring_slots, slot_bytes;
  int smem_bytes, threads_per_cta;
  long long weight_bytes_per_step; /* bf16 weight bytes one step streams */
} mk_plan_info;

/* One task as the builder laid it out (a copy, for tests and tools). */
typedef struct {
  int kind;        /* 0 QKV, 1 ATTN, 2 OPROJ, 3 GATEUP, 4 DOWN, 5 LMHEAD */
  int layer;
  int row0, row1;  /* GEMV: packed output rows; ATTN: kv group, split */
  int req;         /* ATTN: batch slot */
  int wait_event;  /* -1: none */
  int wait_count;  /* signals per step the event must reach */
  int signal_event0, n_signal; /* events bumped on completion */
  int cta;         /* CTA whose queue holds the task */
  int stage;       /* operator stage for the per-operator mode */
} mk_plan_task;

typedef struct mk_plan mk_plan;
int mk_plan_build(const mk_config* cfg, const mk_options* opt, int num_ctas, mk_plan** out);
int mk_plan_get_info(const mk_plan* p, mk_plan_info* info);
/* Copies min(cap, n_tasks) tasks; returns the number copied. */
int mk_plan_get_tasks(const mk_plan* p, mk_plan_task* out, int cap);
/* Queue of one CTA in the megakernel mode (task indices in run order). */
int mk_plan_get_queue(const mk_plan* p, int cta, int* out, int cap);
/* Signals per step each event receives. */
int mk_plan_get_event_counts(const mk_plan* p, int* out, int cap);
void mk_plan_destroy(mk_plan* p);

/* Host-only inspection of how mk_prefill lays out a call's prompt positions
 * for the persistent prefill (CPU tests).  offsets_host [n_req + 1] as for
 * mk_prefill (non-decreasing), slots_host [n_req] the requests' KV slots,
 * max_tokens the block size (positions per launch).  The positions are every
 * prompt position but each prompt's last, in request order, then the last
 * positions of prompts of two or more positions, in request order, as many as
 * the final block's last 128-position tile has room for (those requests'
 * logits and greedy ids come from the same launch; folded_out [n_req] marks
 * them).  Writes min(cap_positions, n) positions as 4 int32 each (token index
 * into the call's tokens, KV slot, position, request for a last position or
 * -1) and min(cap_runs, m) attention runs as 5 int32 each (block, first
 * position inside the block, count, KV slot, first position: one request's
 * positions inside one 128-position tile of a block), and the counts.
 * MK_ERR_INVALID_ARG on a bad argument. */
int mk_prefill_layout(const int32_t* offsets_host, const int32_t* slots_host, int n_req,
                      int max_tokens, int32_t* positions_out, int cap_positions, int32_t* runs_out,
                      int cap_runs, int* n_positions, int* n_runs, int32_t* folded_out);

/* Host-only inspection of the persistent prefill's task graph (CPU tests):
 * the graph of ONE block of T prompt positions whose attention runs are
 * tiles_host [n_tiles][4] (first block position, count, KV slot, first
 * position: one request's positions inside one 128-position tile) and whose
 * prompts' last positions are marked in lm_req_host [T] (request index, or
 * -1), dealt to num_ctas CTAs -- the graph mk_prefill builds for such a block.
 * Writes min(cap_tasks, n) tasks as 9 int32 each (kind as in
 * mk_set_prefill_trace, layer (n_layers for the LM head), 128-position tile,
 * a (GEMM: matrix 0 QKV, 1 O, 2 gate/up, 3 down, 4 LM head; attention: run
 * index), b (GEMM: 128-row tile; attention: query head; elementwise: 8-position
 * slice), wait event or -1, wait count, first signalled event, number of
 * consecutive events signalled), the queue offsets [num_ctas + 1] and the
 * queues (task indices in run order, at most cap_queue), and the task and
 * event counts.  MK_ERR_INVALID_ARG on a bad argument. */
int mk_prefill_graph(const mk_config* cfg, int T, const int32_t* tiles_host, int n_tiles,
                     const int32_t* lm_req_host, int num_ctas, int32_t* tasks_out, int cap_tasks,
                     int32_t* queue_off_out, int32_t* queue_out, int cap_queue, int* n_tasks,
                     int* n_events);

/* Packed-row layout of the fused QKV matrix: the source of packed row r as
 * (which: 0 q, 1 k, 2 v; head; dim).  Rows are grouped per KV head (its G
 * query heads, then its K head, then its V head); inside a q or k head the
 * RoPE partners (i, i + head_dim/2) sit on adjacent rows. */
int mk_qkv_row_source(const mk_config* cfg, int packed_row, int* which, int* head, int* dim);

#ifdef __cplusplus
}
#endif
#endif
