// prefill.h -- prompt prefill on the tensor cores (host side).
//
// Positions [0, len-1) of every prompt run as whole-sequence operators: the
// five weight contractions of a layer as tcgen05 GEMMs (bf16 weights, fp32
// activations split into three bf16 parts, fp32 accumulation),
// RMSNorm / RoPE / KV append / SwiGLU / residual as small kernels, and causal
// GQA attention over the cache.  The last prompt position then runs through
// the decode step, which produces its logits and greedy id.
#pragma once
#include <cuda.h>
#include <cuda_runtime.h>

#include <string>
#include <vector>

#include "mk_internal.h"

namespace mk {

constexpr int kPrefillBlockTokens = 2048;  // prompt positions per pass of the layers

struct PrefillWeights {
  std::vector<const uint16_t*> qkv, o, gu, dn;  // packed, per layer
};

// Device buffers of the persistent prefill (prefill_mk.cu), grown on demand.
struct PfBuffers {
  bool configured = false;
  uint8_t* maps = nullptr;     // tensor maps (global memory, 256-byte aligned)
  uint8_t* tasks = nullptr;
  int32_t* queue = nullptr;
  int32_t* queue_off = nullptr;
  uint32_t* events = nullptr;
  int32_t* err = nullptr;
  size_t maps_cap = 0, tasks_cap = 0, queue_cap = 0, queue_off_cap = 0, events_cap = 0, err_cap = 0;
  uint64_t* trace = nullptr;   // per-task timeline of the first block (mk_set_prefill_trace)
  int trace_cap = 0;
  int stall_task = -2;         // mk_inject_prefill_stall: task index, -1 the last waiting, -2 none
  unsigned long long* lm_keys = nullptr;  // per request: argmax key of its last position
  size_t lm_keys_cap = 0;
};

// Where the persistent prefill puts the results of the prompts' last
// positions (prompts of two or more positions; `folded` reports which).
struct PfOutputs {
  float* logits = nullptr;               // [n_req][vocab] or null
  int32_t* ids = nullptr;                // [n_req] greedy ids or null
  float* hidden[kMaxBatch] = {};         // per request: its residual stream (hidden) or null
  bool folded[kMaxBatch] = {};           // out: the request's last position was handled
};

// Tensor maps of the KV cache for the tensor-core attention (flash_attn.cu):
// rows of head_dim bf16, boxes of 64 keys x 64 dims, K and V, first and
// second 64-dim half.
struct FaMaps {
  CUtensorMap k0, k1, v0, v1;
  bool ready = false;
};

struct PrefillScratch {
  int max_tokens = 0;          // tokens per block
  float* x = nullptr;          // [T][hidden] residual stream
  float* y = nullptr;          // [T][max(qkv rows, 2 ffn, hidden)] GEMM output
  float* q = nullptr;          // [T][n_q * d] rotated queries
  uint16_t* xh = nullptr;      // [T][max(hidden, ffn, n_q*d)] GEMM input, bf16 high part
  uint16_t* xm = nullptr;      //   ... middle part
  uint16_t* xl = nullptr;      //   ... and low part
  int32_t* meta = nullptr;     // per-token and per-tile arrays (see prefill.cu)
  int32_t* err = nullptr;      // device error word of the GEMM kernel
  PfBuffers pf;                // the persistent prefill's task graph and maps
  FaMaps fa;                   // the KV cache as tensor maps (tensor-core attention)
};

// Causal GQA attention of runs of <= 128 consecutive prompt positions of one
// request on the tensor cores (flash_attn.cu).  tiles_dev: [n_tiles][4] = first
// block token, rows, KV slot, first position; q: [T][ldq] rotated fp32
// queries; output [T][ldo] as three bf16 parts.  Waits that run out set
// err[0] = MK_ERR_TIMEOUT.
constexpr int kFaTileRows = 128;
std::string flash_attn_prepare(const ModelDev& m, FaMaps* fm);
std::string flash_attn_launch(const ModelDev& m, const FaMaps& fm, const int32_t* tiles_dev,
                              int n_tiles, int layer, const float* q, int ldq, uint16_t* oh,
                              uint16_t* om, uint16_t* ol, int ldo, int32_t* err, cudaStream_t st);

// Device-side parameters of a batched decode step (read by the captured
// kernels, written before each replay).
struct BatchParams {
  int32_t n;
  int32_t pos[kMaxBatch];
  int32_t slot[kMaxBatch];
  int32_t src[kMaxBatch];   // token index of request r: r
};

// Scratch and captured graphs of the batched decode step.
struct BatchScratch {
  int splits = 0;              // attention splits per (request, KV head)
  BatchParams* params = nullptr;
  int32_t* tokens = nullptr;   // [kMaxBatch] this step's input ids
  float* x = nullptr;          // [kMaxBatch][hidden] residual stream
  float* y = nullptr;          // [kBatchMaxSplitK][kMaxBatch][max(qkv rows, 2 ffn, hidden)]
  float* q = nullptr;          // [kMaxBatch][n_q * d]
  float* part = nullptr;       // [kMaxBatch][n_kv][splits][G][d + 4] attention partials
  uint16_t* xh = nullptr;      // [2 kMaxBatch][K] GEMM input: high parts, then low parts
  uint16_t* xh2 = nullptr;     // the same for the SwiGLU output (the down projection's input)
  uint32_t* tickets = nullptr; // [kMaxBatch][n_kv] attention split-merge tickets
  float* logits = nullptr;     // [kMaxBatch][vocab]
  int32_t* ids = nullptr;      // [kMaxBatch]
  int32_t* err = nullptr;
  void* acc = nullptr;         // per-step accumulators (zeroed by the step)
  size_t acc_bytes = 0;
  cudaGraphExec_t graph[kMaxBatch + 1] = {};
  cudaGraph_t graph_src[kMaxBatch + 1] = {};
};
constexpr int kBatchMaxSplitK = 16;

// Whether the GEMM path handles this shape (every contraction length a
// multiple of 64).
bool prefill_gemm_supported(const ModelDev& m);

// Allocates the scratch for blocks of up to max_tokens tokens (cudaMalloc).
std::string prefill_alloc(const ModelDev& m, int max_tokens, PrefillScratch* sc,
                          std::vector<void*>* owned);

// Runs positions [0, len_r - 1) of each request r (tokens_dev packed with
// offsets_host) through the layers, filling the KV cache of request slot
// slots_host[r].  Enqueued on `st`.
std::string prefill_run(const ModelDev& m, const PrefillWeights& w, PrefillScratch& sc,
                        cudaStream_t st, const int32_t* tokens_dev, const int32_t* offsets_host,
                        const int32_t* slots_host, int n_req,
                        bool tc_attn, bool* timed_out);

// The same prefill as ONE persistent kernel per block (prefill_mk.cu): every
// operator of every layer a task, dependencies per (layer, stage, token tile)
// through event counters, the GEMMs as tcgen05 tiles.  Unlike prefill_run it
// also runs each prompt's LAST position (prompts of two or more positions):
// the final norm, the LM head and the greedy id, results per `out`.
// Synchronises `st`.
std::string prefill_mk_run(const ModelDev& m, const PrefillWeights& w, PrefillScratch& sc,
                           cudaStream_t st, const int32_t* tokens_dev, const int32_t* offsets_host,
                           const int32_t* slots_host, int n_req, int num_sms,
                           std::vector<void*>* owned, bool* timed_out, PfOutputs* out);

// Allocates the batched decode scratch (cudaMalloc).
std::string batch_alloc(const ModelDev& m, int num_sms, BatchScratch* bs, std::vector<void*>* owned);

// One decode step of n (2..8) requests with every weight matrix streamed
// once: tcgen05 GEMMs of 16 token columns (split along K where a matrix has
// few 128-row tiles), split-KV attention per (request, KV head), argmax per
// request.  Reads bs.tokens and bs.params; writes bs.logits, bs.ids, bs.x.
// Captured into a CUDA graph per n on first use, then replayed.
std::string batch_step(const ModelDev& m, const PrefillWeights& w, BatchScratch& bs, int n,
                       int num_sms, cudaStream_t st);

}  // namespace mk
