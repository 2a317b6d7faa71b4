#pragma once
// step_kernel.cuh -- the persistent decode-step kernel for sm_100a (device
// code; instantiated per weight width and attention geometry by the
// step_*.cu files, so that each kernel holds only the attention variant it
// runs and its register allocation is not set by the others).
//
// One CTA per SM runs an ahead-of-time queue of tasks ("LLMs in einen
// MegaKernel kompilieren ...", "Part 2. Laufzeit": each worker SM loops
// fetch task -> execute -> notify event).  Inside a CTA the roles are split
// by warp:
//   warp 0  producer : walks the queue ahead of the workers and streams every
//                      task's bf16 weight rows (or old K/V rows) with bulk
//                      copies into a ring of shared-memory slots.  It never
//                      waits on events, so the next task's -- and the next
//                      layer's -- weights are already on chip while the
//                      current dependency resolves ("MPK ..." §4: a task
//                      releases its shared-memory pages so the next task can
//                      prefetch early).
//   warp 1  scheduler: waits (gpu-scope acquire, bounded by %globaltimer) until
//                      the event of the next task reached its threshold, then
//                      releases the workers ("Ereignisbasierte Ausführung").
//   warps 2-17 workers: compute each task from the ring: fp32 activations,
//                      bf16 weights widened in registers, 128-bit shared-memory
//                      loads, warp-shuffle reductions ("Crear desde cero ..."
//                      §3.2: threads cooperate on rows and reduce by warp);
//                      epilogues fuse bias, RoPE, the KV append, residual adds,
//                      SwiGLU and the argmax ("Crear desde cero ..." §3.3).
// A finished task bumps its event counters with a gpu-scope release.
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_fp8.h>
#include <math.h>

#include "../../include/mk.h"
#include "mk_internal.h"
#include "ptx.cuh"
#include "attn_math.cuh"

namespace mk {

struct __align__(128) Smem {
  uint8_t ring[kRingSlots][kSlotBytes];
  float scratch[kScratchBytes / 4];
  float ybuf[kYBufFloats];
  float red[64];
  unsigned long long red64[kWorkerWarps];
  uint64_t full[kRingSlots];
  uint64_t empty[kRingSlots];
  uint64_t ready;
  uint64_t done;
  uint32_t epoch;
  int32_t abort_flag;
  int32_t flag;
  int32_t cur_qi;              // queue entry the workers are running (trace)
  unsigned long long lm_best;  // running argmax over this CTA's LM-head tasks
  StepParams sp_work;          // the workers' current step (set by the scheduler between steps)
  uint32_t epoch0;             // completed steps when this launch started
  int32_t attn_last;           // this attention task merges its KV head's splits
  __align__(16) float attn_xb[kWorkerWarps][kAttnXbStride];  // attention: per-warp softmax weights
};

constexpr uint32_t kWorkerBarrier = 1;

__device__ __forceinline__ void worker_sync() { named_barrier_sync(kWorkerBarrier, kWorkerThreads); }

__device__ __forceinline__ bool aborting(Smem& s) { return *(volatile int32_t*)&s.abort_flag != 0; }

__device__ __forceinline__ const StepParams& step_params(const KernelArgs& a) {
  return a.sp_ptr ? *a.sp_ptr : a.sp_val;
}

// The parameters of step `step` of this launch.  With a device-resident loop
// (n_steps > 1) position and token advance per step: step s feeds the id step
// s - 1 wrote, writes its own id to ids_seq[s], and only the last step writes
// logits.
__device__ __forceinline__ void step_at(const KernelArgs& a, int step, StepParams& out) {
  out = step_params(a);
  if (a.n_steps > 1) {
    out.pos[0] += step;
    out.tokens = step == 0 ? out.tokens : a.ids_seq + (step - 1);
    out.next_ids = a.ids_seq + step;
    const bool last = step == a.n_steps - 1;
    out.logits = last ? out.logits : nullptr;
    out.want_logits = last ? out.want_logits : 0;
  }
}

// Per-task timeline (diagnostics, off unless a trace buffer is set): word k of
// the running queue entry.  0 event satisfied, 1 workers start, 2 input
// loaded, 3 first chunk ready, 4 last chunk consumed, 5 epilogue done, 6 end,
// 7 cta << 32 | task.
constexpr int kTraceWords = 8;
__device__ __forceinline__ void trace_mark(const KernelArgs& a, Smem& s, int wtid, int k) {
  if (a.m.trace && wtid == 0) a.m.trace[(size_t)s.cur_qi * kTraceWords + k] = globaltimer_ns();
}

__device__ __forceinline__ float bf16_to_float(uint16_t h) {
  return __uint_as_float(static_cast<uint32_t>(h) << 16);
}
__device__ __forceinline__ uint16_t float_to_bf16_rne(float f) {
  __nv_bfloat16 b = __float2bfloat16_rn(f);
  return *reinterpret_cast<uint16_t*>(&b);
}

// Eight bf16 weights times eight fp32 inputs into a pair of fp32 partial sums
// (even and odd columns) with the packed fp32x2 FMA of sm_100.
__device__ __forceinline__ float2 dot8(const uint4 w, const float2 (&x)[4], float2 acc) {
  acc = __ffma2_rn(make_float2(bf_lo(w.x), bf_hi(w.x)), x[0], acc);
  acc = __ffma2_rn(make_float2(bf_lo(w.y), bf_hi(w.y)), x[1], acc);
  acc = __ffma2_rn(make_float2(bf_lo(w.z), bf_hi(w.z)), x[2], acc);
  acc = __ffma2_rn(make_float2(bf_lo(w.w), bf_hi(w.w)), x[3], acc);
  return acc;
}

// Sixteen fp8 (e4m3) weights of one 16-byte piece against their inputs: pairs
// of codes widen exactly to half and then to float.
__device__ __forceinline__ float2 fp8x2_to_float2(uint32_t two) {
  const __half2_raw h = __nv_cvt_fp8x2_to_halfraw2((__nv_fp8x2_storage_t)two, __NV_E4M3);
  return __half22float2(*reinterpret_cast<const __half2*>(&h));
}
__device__ __forceinline__ float2 dot16_fp8(const uint4 w, const float2 (&x)[8], float2 acc) {
  const uint32_t v[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    acc = __ffma2_rn(fp8x2_to_float2(v[q] & 0xffffu), x[2 * q], acc);
    acc = __ffma2_rn(fp8x2_to_float2(v[q] >> 16), x[2 * q + 1], acc);
  }
  return acc;
}

// Rows of the matrix a GEMV task streams.
__device__ __forceinline__ int task_matrix_rows(const ModelDev& m, const Task& t) {
  return t.kind == T_QKV ? qkv_rows(m.n_q, m.n_kv, m.head_dim)
         : t.kind == T_GATEUP ? 2 * m.ffn
         : t.kind == T_LMHEAD ? m.vocab : m.hidden;
}

// Row scales of a task's fp8 matrix: they follow the matrix's codes in the
// same allocation, at the 16-byte-aligned end of its rows x K bytes.
__device__ __forceinline__ const float* task_wscale(const ModelDev& m, const Task& t) {
  const int rows = task_matrix_rows(m, t);
  const size_t off = ((size_t)rows * t.K + 15) & ~(size_t)15;
  return reinterpret_cast<const float*>(reinterpret_cast<const uint8_t*>(t.w) + off);
}

__device__ __forceinline__ void set_error(const ModelDev& m, int code, int info) {
  if (atomicCAS(m.status, 0, code) == 0) m.status_info[0] = info;
}

// Codes stored in status_info when a shared-memory barrier wait times out
// (event waits store the task index instead).
constexpr int kWaitFull = -1, kWaitReady = -2, kWaitDone = -3, kWaitEmpty = -4, kWaitDrain = -5;

__device__ __forceinline__ bool aborting(Smem& s);

// Bounded mbarrier wait.  True once the phase with `parity` completed; false
// when this CTA is aborting or the wait exceeded the context's limit (which
// records MK_ERR_TIMEOUT and starts the abort).  Every wait in the kernel is
// bounded, so a broken invariant ends the launch with an error, not a hang.
// The limit is twice the event-wait limit: a barrier may legitimately wait
// behind an event wait, and a stalled event should be reported as such.
static __device__ __noinline__ bool wait_bounded(Smem& s, uint64_t* bar, uint32_t parity,
                                          const ModelDev& m, int where) {
  const uint64_t limit = 2ull * (uint64_t)(m.timeout_ms > 0 ? m.timeout_ms : 1000) * 1000000ull;
  const uint64_t t0 = globaltimer_ns();
  while (true) {
    if (mbar_try_wait(bar, parity)) return true;
    if (aborting(s)) return false;
    if (globaltimer_ns() - t0 > limit) {
      set_error(m, MK_ERR_TIMEOUT, where);
      *(volatile int32_t*)&s.abort_flag = 1;
      return false;
    }
  }
}

// Orderable key: larger value first, then lower index.
__device__ __forceinline__ unsigned long long argmax_key(float v, int idx) {
  uint32_t u = __float_as_uint(v);
  u = (u & 0x80000000u) ? ~u : (u | 0x80000000u);
  return (static_cast<unsigned long long>(u) << 32) | (0xffffffffu - static_cast<uint32_t>(idx));
}

// ------------------------------------------------------ chunk enumeration
// The producer and the workers walk the same chunk list for every task.

struct AttnRange {
  int k0, k1, old_end;  // keys [k0, k1); [k0, old_end) come through the ring
  int live;             // splits that hold keys at this position
  bool active;
};

__device__ __forceinline__ AttnRange attn_range(const Task& t, const StepParams& sp,
                                                const ModelDev& m) {
  AttnRange r{0, 0, 0, false};
  if (t.req >= sp.n_req) return r;
  const int pos = sp.pos[t.req];
  const int n = pos + 1;
  const int live = attn_live_splits(n, m.attn_splits, attn_keys_per_chunk(m.head_dim));
  if (t.row1 >= live) return r;  // a split with no keys at this position
  // keys per split; with a paged cache rounded up to whole key blocks, so that
  // split ranges start on page boundaries (a trailing split may then hold no
  // keys: it contributes an empty partial)
  int chunk = (n + live - 1) / live;
  if (m.kv_page < m.max_seq) chunk = (chunk + kKeyBlock - 1) / kKeyBlock * kKeyBlock;
  r.k0 = min(n, t.row1 * chunk);
  r.k1 = min(n, r.k0 + chunk);
  r.old_end = min(r.k1, pos);
  if (r.old_end < r.k0) r.old_end = r.k0;
  r.live = live;
  r.active = true;
  return r;
}

__device__ __forceinline__ size_t kv_offset(const ModelDev& m, int slot, int layer, int g,
                                            int key) {
  return kv_row(m, slot, layer, g, key);
}

// Keys of the ring chunk that starts at key k of [k, end): at most one ring
// chunk, and never across a KV page boundary (a chunk is one bulk copy of
// consecutive rows).  The producer and the attention task use the same rule.
__device__ __forceinline__ int attn_chunk_keys(const ModelDev& m, int k, int end) {
  const int to_page = m.kv_page - k % m.kv_page;
  return min(min(attn_keys_per_chunk(m.head_dim), end - k), to_page);
}

// ---------------------------------------------------------------- producer


__device__ __forceinline__ bool producer_acquire_slot(Smem& s, uint32_t seq, const ModelDev& m) {
  const int slot = seq % kRingSlots;
  const uint32_t ph = (seq / kRingSlots) & 1u;
  if (!wait_bounded(s, &s.empty[slot], ph ^ 1u, m, kWaitEmpty)) return false;
  return !aborting(s);
}

// One ring chunk: up to two 1-D bulk copies into the same slot (weights: one
// copy of whole rows; attention: K rows into the first half, V rows into the
// second half).
struct Chunk {
  const void* src0;
  const void* src1;
  uint32_t bytes0, bytes1;
  bool kv;
};

// Walks the chunks of a CTA's queue in the order the workers consume them.
struct ChunkCursor {
  int qi, q1;
  int off;  // next row (GEMV) or key (ATTN) inside task qi

  __device__ __forceinline__ bool next(const KernelArgs& a, const StepParams& sp, Chunk& c) {
    const ModelDev& m = a.m;
    while (qi < q1) {
      const Task& t = a.tasks[a.queue[qi]];
      if (t.kind == T_ATTN) {
        const AttnRange r = attn_range(t, sp, m);
        if (r.active) {
          const int k = off < 0 ? r.k0 : off;
          if (k < r.old_end) {
            const int nk = attn_chunk_keys(m, k, r.old_end);
            bounds_ok(m, nk > 0 && k + nk <= m.max_seq, kBndKvKey);
            bounds_ok(m, (uint32_t)nk * m.head_dim * 2 <= kSlotBytes / 2, kBndChunkBytes);
            const size_t o = kv_offset(m, sp.kv_slot[t.req], t.layer, t.row0, k);
            c.src0 = m.kcache + o;
            c.src1 = m.vcache + o;
            c.bytes0 = c.bytes1 = (uint32_t)nk * m.head_dim * 2;
            c.kv = true;
            off = k + nk;
            return true;
          }
        }
      } else {
        const int r = off < 0 ? t.row0 : off;
        if (r < t.row1) {
          const int nr = min(t.chunk_rows, t.row1 - r);
          if (!bounds_ok(m, r + nr <= task_matrix_rows(m, t), kBndChunkRows) ||
              !bounds_ok(m, (size_t)nr * t.K * m.wbytes <= kSlotBytes, kBndChunkBytes)) {
            ++qi;  // skip the task's remaining chunks (its workers see the abort)
            off = -1;
            continue;
          }
          c.src0 = reinterpret_cast<const uint8_t*>(t.w) + (size_t)r * t.K * m.wbytes;
          c.src1 = nullptr;
          c.bytes0 = (uint32_t)nr * t.K * m.wbytes;
          c.bytes1 = 0;
          c.kv = false;
          off = r + nr;
          return true;
        }
      }
      ++qi;
      off = -1;
    }
    return false;
  }
};

// Streams the chunks of the CTA's queue into the ring, in the workers'
// consumption order, as fast as slots free up.  Producer `pid` of
// kProducerWarps issues chunks seq with seq % kProducerWarps == pid (every
// producer walks the whole chunk list; a slot is always filled by the same
// producer, and each waits only for its own slots to be released).
__device__ __forceinline__ void producer(const KernelArgs& a, Smem& s, int q0, int q1, int pid) {
  const ModelDev& m = a.m;
  const uint64_t pol_w = l2_policy_evict_first();
  const uint64_t pol_keep = l2_policy_evict_normal();
  Chunk c;
  uint32_t seq = 0;
  bool stop = false;
  for (int step = 0; step < a.n_steps && !stop; ++step) {
    StepParams sp;
    step_at(a, step, sp);
    // Cached keys of a step after the first include the key the previous
    // step wrote (another CTA, same launch): before copying any, wait until
    // that step has completed (its last LM-head task bumps the epoch) and
    // order those writes before this thread's bulk copies.
    bool kv_ready = step == 0;
    ChunkCursor cc{q0, q1, -1};
    while (cc.next(a, sp, c)) {
      if (c.kv && !kv_ready) {
        const uint64_t t0 = globaltimer_ns();
        const uint64_t limit = 2ull * (uint64_t)(m.timeout_ms > 0 ? m.timeout_ms : 1000) * 1000000ull;
        while ((int32_t)(ld_acquire_gpu(m.epoch) - (s.epoch0 + (uint32_t)step)) < 0) {
          if (aborting(s) || globaltimer_ns() - t0 > limit) { stop = true; break; }
        }
        if (stop) break;
        fence_proxy_async_global();
        kv_ready = true;
      }
      if ((int)(seq % kProducerWarps) == pid) {
        if (!producer_acquire_slot(s, seq, m)) { stop = true; break; }
        const int slot = seq % kRingSlots;
        mbar_arrive_expect_tx(&s.full[slot], c.bytes0 + c.bytes1);
        bulk_g2s(s.ring[slot], c.src0, c.bytes0, &s.full[slot], c.kv ? pol_keep : pol_w);
        if (c.src1) bulk_g2s(s.ring[slot] + kSlotBytes / 2, c.src1, c.bytes1, &s.full[slot], pol_keep);
      }
      ++seq;
    }
  }
  // Before this warp may retire, every copy it issued must have landed: if
  // the workers stop early (abort) nobody else waits for them, and a bulk copy
  // must never write into shared memory of a CTA that has exited.  Only the
  // last kRingSlots copies can still be in flight (older slots were reused).
  // The drain is bounded and therefore best-effort: the sources are valid
  // device memory, so a copy lands in microseconds; if one has not after
  // 200 ms the launch records MK_ERR_TIMEOUT (detail kWaitDrain), which
  // poisons the context on the host so it is never used again.
  const uint32_t first = seq > kRingSlots ? seq - kRingSlots : 0;
  for (uint32_t q = first; q < seq; ++q) {
    if ((int)(q % kProducerWarps) != pid) continue;  // the other producer's copy
    const uint64_t t0 = globaltimer_ns();
    while (!mbar_try_wait(&s.full[q % kRingSlots], (q / kRingSlots) & 1u)) {
      if (globaltimer_ns() - t0 > 200000000ull) {
        set_error(m, MK_ERR_TIMEOUT, kWaitDrain);
        return;
      }
    }
  }
}

// --------------------------------------------------------------- scheduler

__device__ __forceinline__ void scheduler(const KernelArgs& a, Smem& s, int q0, int q1) {
  const ModelDev& m = a.m;
  const uint64_t pol_keep = l2_policy_evict_normal();
  const uint64_t limit = (uint64_t)(m.timeout_ms > 0 ? m.timeout_ms : 1000) * 1000000ull;
  int i = 0;
  for (int step = 0; step < a.n_steps; ++step) {
  StepParams sp;
  step_at(a, step, sp);
  const uint32_t epoch = s.epoch0 + (uint32_t)step;
  if (step > 0) {
    // the workers are idle (the previous task's `done` was observed)
    s.sp_work = sp;
    s.epoch = epoch;
  }
  for (int qi = q0; qi < q1; ++qi, ++i) {
    const int tid = a.queue[qi];
    const Task& t = a.tasks[tid];
    bool abort = false;
    if (step > 0 && t.kind == T_QKV && t.layer == 0) {
      // the first layer embeds the id the previous step produced
      const uint64_t t0 = globaltimer_ns();
      uint32_t spins = 0;
      while ((int32_t)(ld_acquire_gpu(m.epoch) - epoch) < 0) {
        if ((++spins & 63u) == 0) {
          if (ld_relaxed_gpu_s32(m.status) != 0 || aborting(s)) { abort = true; break; }
          if (globaltimer_ns() - t0 > limit) {
            set_error(m, MK_ERR_TIMEOUT, tid);
            abort = true;
            break;
          }
        }
      }
    }
    if (!abort && t.wait_ev >= 0 && !a.no_wait) {
      const uint32_t target = t.wait_count * (epoch + 1u);
      const uint32_t* ev = m.events + t.wait_ev;
      if (m.l2_prefetch_chunks > 0 && (int32_t)(ld_acquire_gpu(ev) - target) < 0) {
        // The workers are about to stall on this event, and the ring holds
        // (or is receiving) the first kRingSlots chunks from here on: prefetch
        // the next l2_prefetch_chunks chunks into L2 so HBM keeps streaming
        // through the wait and their copies hit in L2.
        ChunkCursor pc{qi, q1, -1};
        Chunk pf;
        for (int n = 0; n < kRingSlots + m.l2_prefetch_chunks && pc.next(a, sp, pf); ++n) {
          if (n < kRingSlots) continue;
          bulk_prefetch_l2(pf.src0, pf.bytes0, pol_keep);
          if (pf.src1) bulk_prefetch_l2(pf.src1, pf.bytes1, pol_keep);
        }
      }
      const uint64_t t0 = globaltimer_ns();
      uint32_t spins = 0;
      while ((int32_t)(ld_acquire_gpu(ev) - target) < 0) {
        if ((++spins & 63u) == 0) {
          if (ld_relaxed_gpu_s32(m.status) != 0 || aborting(s)) { abort = true; break; }
          if (globaltimer_ns() - t0 > limit) {
            set_error(m, MK_ERR_TIMEOUT, tid);
            abort = true;
            break;
          }
        }
      }
    }
    if (abort) {
      *(volatile int32_t*)&s.abort_flag = 1;
      __threadfence_block();
      mbar_arrive(&s.ready);
      return;
    }
    if (m.trace) m.trace[(size_t)qi * kTraceWords] = globaltimer_ns();
    mbar_arrive(&s.ready);
    if (!wait_bounded(s, &s.done, i & 1, m, kWaitDone)) return;
  }
  }
}

// ------------------------------------------------------------ worker: GEMV

// Sums eight per-lane values across a warp at once (a transposed butterfly:
// at each of the first three levels a lane keeps half of its values and adds
// its partner's copy of them), seven shuffles in all instead of five per
// value; lane l ends with the warp's sum of value l >> 2.
__device__ __forceinline__ float warp_reduce8(const float (&v)[8], int lane) {
  const bool b4 = lane & 16, b3 = lane & 8, b2 = lane & 4;
  float a[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float keep = b4 ? v[i + 4] : v[i], send = b4 ? v[i] : v[i + 4];
    a[i] = keep + __shfl_xor_sync(0xffffffffu, send, 16);
  }
  float c[2];
#pragma unroll
  for (int i = 0; i < 2; ++i) {
    const float keep = b3 ? a[i + 2] : a[i], send = b3 ? a[i] : a[i + 2];
    c[i] = keep + __shfl_xor_sync(0xffffffffu, send, 8);
  }
  float k = (b2 ? c[1] : c[0]) + __shfl_xor_sync(0xffffffffu, b2 ? c[0] : c[1], 4);
  k += __shfl_xor_sync(0xffffffffu, k, 2);
  k += __shfl_xor_sync(0xffffffffu, k, 1);
  return k;
}

// Waits for ring chunk `seq`.  Once the CTA is aborting the workers no longer
// wait: they run the rest of the current task on whatever the slot holds
// (every access stays in bounds), meet the task's barriers, and stop.
__device__ __forceinline__ void wait_full(Smem& s, uint32_t seq, const ModelDev& m) {
  const int slot = seq % kRingSlots;
  const uint32_t ph = (seq / kRingSlots) & 1u;
  if (mbar_try_wait(&s.full[slot], ph)) return;
  wait_bounded(s, &s.full[slot], ph, m, kWaitFull);
}

// Loads this thread's input columns into xr (fp32, or the bf16 embedding
// row).  For the O projection the input is the attention output, which the
// last attention task of each KV head merged from the split partials.  For operators
// that start with RMSNorm, xr = x * w_norm and the returned value is this
// thread's share of sum(x^2); the 1/rms factor is applied to the dot products
// afterwards (W (x * w * r) = r * W (x * w)), so the first ring chunk is not
// held back by a block-wide reduction.
// PW: input pairs per 16-byte weight piece -- 4 for bf16 (8 columns), 8 for
// fp8 (16 columns).
template <int CPT, int PW>
__device__ __forceinline__ float gemv_load_input(const KernelArgs& a, const StepParams& sp,
                                                 const Task& t, int wtid, int ct, int rl,
                                                 float2 (&x2)[CPT][PW]) {
  const ModelDev& m = a.m;
  const int K = t.K, C = K / (2 * PW);
  const float* src32 = nullptr;
  const uint16_t* src16 = nullptr;
  const uint16_t* normw = nullptr;
  switch (t.kind) {
    case T_QKV:
      normw = m.attn_norm + (size_t)t.layer * m.hidden;
      if (t.layer == 0) {
        int tok = sp.tokens[0];
        if (tok < 0 || tok >= m.vocab) {
          if (wtid == 0) set_error(m, MK_ERR_TOKEN_RANGE, tok);
          tok = 0;
        }
        src16 = m.embed + (size_t)tok * m.hidden;
      } else {
        src32 = m.x;
      }
      break;
    case T_OPROJ: src32 = m.attn; break;
    case T_GATEUP: src32 = m.x; normw = m.ffn_norm + (size_t)t.layer * m.hidden; break;
    case T_DOWN: src32 = m.act; break;
    default: src32 = m.x; normw = m.final_norm; break;  // LM head
  }
  const int TPR = t.tpr;
  float ss = 0.f;
#pragma unroll
  for (int c = 0; c < CPT; ++c) {
    const int cc = ct + c * TPR;
#pragma unroll
    for (int e = 0; e < PW; ++e) x2[c][e] = make_float2(0.f, 0.f);
    if (cc >= C) continue;
#pragma unroll
    for (int q = 0; q < PW / 4; ++q) {  // 8-column blocks of this piece
      const int sc = cc * (PW / 4) + q;
      float2* xq = &x2[c][4 * q];
      if (src16) {
        const uint4 v = __ldg(reinterpret_cast<const uint4*>(src16) + sc);
        xq[0] = make_float2(bf_lo(v.x), bf_hi(v.x));
        xq[1] = make_float2(bf_lo(v.y), bf_hi(v.y));
        xq[2] = make_float2(bf_lo(v.z), bf_hi(v.z));
        xq[3] = make_float2(bf_lo(v.w), bf_hi(v.w));
      } else {
        const float4 u = __ldcg(reinterpret_cast<const float4*>(src32) + 2 * sc);
        const float4 w = __ldcg(reinterpret_cast<const float4*>(src32) + 2 * sc + 1);
        xq[0] = make_float2(u.x, u.y);
        xq[1] = make_float2(u.z, u.w);
        xq[2] = make_float2(w.x, w.y);
        xq[3] = make_float2(w.z, w.w);
      }
      if (normw) {
        const uint4 wv = __ldg(reinterpret_cast<const uint4*>(normw) + sc);
        const float2 wn[4] = {make_float2(bf_lo(wv.x), bf_hi(wv.x)), make_float2(bf_lo(wv.y), bf_hi(wv.y)),
                              make_float2(bf_lo(wv.z), bf_hi(wv.z)), make_float2(bf_lo(wv.w), bf_hi(wv.w))};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          if (rl == 0) {
            ss = fmaf(xq[e].x, xq[e].x, ss);
            ss = fmaf(xq[e].y, xq[e].y, ss);
          }
          xq[e] = make_float2(xq[e].x * wn[e].x, xq[e].y * wn[e].y);
        }
      }
    }
  }
  return ss;
}

// Ring position of chunk `seq`: its slot and the parity of the slot's
// current fill, advanced without a division per chunk.
struct RingPos {
  int slot;
  uint32_t ph;
  __device__ __forceinline__ explicit RingPos(uint32_t seq)
      : slot((int)(seq % kRingSlots)), ph((seq / kRingSlots) & 1u) {}
  __device__ __forceinline__ RingPos next() const {
    RingPos r = *this;
    if (++r.slot == kRingSlots) { r.slot = 0; r.ph ^= 1u; }
    return r;
  }
};

__device__ __forceinline__ void wait_slot(Smem& s, const RingPos& p, const ModelDev& m) {
  if (mbar_try_wait(&s.full[p.slot], p.ph)) return;
  wait_bounded(s, &s.full[p.slot], p.ph, m, kWaitFull);
}

// Streams the task's rows through the ring and leaves y[row] in s.ybuf.
// A ring chunk holds NR rows per row-lane.  The workers take the chunks two
// at a time: both slots are awaited, all their 16-byte pieces are loaded
// together, multiplied with the thread's inputs, and both slots released, so
// the per-chunk bookkeeping is shared and the shared-memory loads of two
// chunks overlap.  A thread keeps one partial sum per row and, after every
// 8 / NR chunks, the warp reduces the eight partials at once
// (warp_reduce8), so no shuffle chain sits between a chunk's arrival and its
// release.  The warps of a row-lane are added at the end in a fixed order.
template <int CPT, int NR, int PW>
__device__ __forceinline__ void gemv_stream(const KernelArgs& a, Smem& s, const Task& t, uint32_t& seq, int wtid) {
  constexpr int kGroup = 8 / NR;  // chunks per reduction (a multiple of 2)
  static_assert(kGroup % 2 == 0, "chunks are taken in pairs");
  const int TPR = t.tpr;
  const int rl = wtid / TPR, ct = wtid % TPR;
  const int wpr = TPR >> 5, wir = ct >> 5;
  const int lane = wtid & 31;
  const int K = t.K, C = K / (2 * PW);
  const size_t row_bytes = (size_t)K * 8 / PW;
  const int nrows = t.row1 - t.row0;
  const int crows = t.chunk_rows;
  const int nchunks = (nrows + crows - 1) / crows;
  // fp8: the row scales of this thread's output rows (at most two: a task
  // has at most kYBufFloats = 2 x 512 rows), requested with the inputs
  static_assert(kYBufFloats <= 2 * kWorkerThreads, "two output rows per thread at most");
  float rsc0 = 1.f, rsc1 = 1.f;
  if constexpr (PW == 8) {
    const float* wsc = task_wscale(a.m, t) + t.row0;
    if (wtid < nrows) rsc0 = __ldg(wsc + wtid);
    if (wtid + kWorkerThreads < nrows) rsc1 = __ldg(wsc + wtid + kWorkerThreads);
  }
  float2 x2[CPT][PW];
  float ss = gemv_load_input<CPT, PW>(a, s.sp_work, t, wtid, ct, rl, x2);
  trace_mark(a, s, wtid, 2);
  const bool has_norm = t.kind == T_QKV || t.kind == T_GATEUP || t.kind == T_LMHEAD;
  if (has_norm) {
#pragma unroll
    for (int o = 16; o; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
    if (lane == 0) s.red[wtid >> 5] = ss;  // read after the barrier that ends the stream
  }
  RingPos pos(seq);
  for (int q0 = 0; q0 < nchunks; q0 += kGroup) {
    float v[8];
#pragma unroll
    for (int j = 0; j < kGroup; j += 2) {
      const int q = q0 + j;
      const bool have0 = q < nchunks, have1 = q + 1 < nchunks;  // warp-uniform
      const RingPos p1 = pos.next();
      if (have0) wait_slot(s, pos, a.m);
      if (have1) wait_slot(s, p1, a.m);
      if (q == 0) trace_mark(a, s, wtid, 3);
      uint4 pc[2][NR][CPT];
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const int qh = q + h;
        const int rows_here = min(crows, nrows - qh * crows);
        const uint8_t* base = s.ring[h ? p1.slot : pos.slot];
#pragma unroll
        for (int k = 0; k < NR; ++k) {
          const int lr = rl * NR + k;
          const bool live = (h ? have1 : have0) && lr < rows_here &&
                            bounds_ok(a.m, (size_t)(lr + 1) * row_bytes <= kSlotBytes, kBndSlotRow);
#pragma unroll
          for (int c = 0; c < CPT; ++c) {
            const int cc = ct + c * TPR;
            pc[h][k][c] = (live && cc < C)
                              ? *reinterpret_cast<const uint4*>(base + (size_t)lr * row_bytes + (size_t)cc * 16)
                              : make_uint4(0u, 0u, 0u, 0u);
          }
        }
      }
      __syncwarp();
      if (lane == 0) {
        if (have0) mbar_arrive(&s.empty[pos.slot]);
        if (have1) mbar_arrive(&s.empty[p1.slot]);
      }
#pragma unroll
      for (int h = 0; h < 2; ++h)
#pragma unroll
        for (int k = 0; k < NR; ++k) {
          float2 a2 = make_float2(0.f, 0.f);
#pragma unroll
          for (int c = 0; c < CPT; ++c) {
            if constexpr (PW == 4) a2 = dot8(pc[h][k][c], x2[c], a2);
            else a2 = dot16_fp8(pc[h][k][c], x2[c], a2);
          }
          v[(j + h) * NR + k] = a2.x + a2.y;
        }
      if (have0) { pos = p1; ++seq; }
      if (have1) { pos = pos.next(); ++seq; }
    }
    const float r8 = warp_reduce8(v, lane);
    const int idx = lane >> 2, q = q0 + idx / NR;
    const int row = q * crows + rl * NR + idx % NR;
    if ((lane & 3) == 0 && q < nchunks && row < nrows &&
        bounds_ok(a.m, (wir + 1) * nrows <= kScratchBytes / 4, kBndScratch))
      s.scratch[wir * nrows + row] = r8;
  }
  trace_mark(a, s, wtid, 4);
  worker_sync();
  float r = 1.0f;
  if (has_norm) {
    float tot = 0.f;
#pragma unroll
    for (int w = 0; w < kWorkerWarps; ++w) tot += s.red[w];
    r = 1.0f / sqrtf(tot / (float)K + a.m.rms_eps);
  }
  for (int i = wtid; i < nrows; i += kWorkerThreads) {
    // the row-lane's warp partials, four independent chains
    float y0 = 0.f, y1 = 0.f, y2 = 0.f, y3 = 0.f;
    int w = 0;
    for (; w + 4 <= wpr; w += 4) {
      y0 += s.scratch[w * nrows + i];
      y1 += s.scratch[(w + 1) * nrows + i];
      y2 += s.scratch[(w + 2) * nrows + i];
      y3 += s.scratch[(w + 3) * nrows + i];
    }
    for (; w < wpr; ++w) y0 += s.scratch[w * nrows + i];
    float y = (y0 + y1) + (y2 + y3);
    if constexpr (PW == 8) y *= i < kWorkerThreads ? rsc0 : rsc1;  // fp8 row scale
    if (bounds_ok(a.m, i < kYBufFloats, kBndYbuf)) s.ybuf[i] = has_norm ? y * r : y;
  }
  worker_sync();
}

// The geometries gemv_tpr / gemv_nr produce: a row of C 16-byte pieces over
// one warp-multiple row-lane gives (pieces per thread, rows per chunk) =
// (1, 4) for C <= 512, (2, 2) for C <= 1024, (3, 1) and (4, 1) beyond (fp8
// rows have at most 1024 pieces).  Only these are instantiated; another
// combination is reported as a bounds error (it cannot come from the plan).
template <int PW>
__device__ __forceinline__ void gemv_core(const KernelArgs& a, Smem& s, const Task& t, uint32_t& seq, int wtid) {
  const int cpt = (t.K / (2 * PW) + t.tpr - 1) / t.tpr;
  const int nr = t.chunk_rows / (kWorkerThreads / t.tpr);
  if (cpt == 1 && nr == 4) gemv_stream<1, 4, PW>(a, s, t, seq, wtid);
  else if (cpt == 2 && nr == 2) gemv_stream<2, 2, PW>(a, s, t, seq, wtid);
  else if constexpr (PW == 4) {
    if (cpt == 3 && nr == 1) gemv_stream<3, 1, PW>(a, s, t, seq, wtid);
    else if (cpt == 4 && nr == 1) gemv_stream<4, 1, PW>(a, s, t, seq, wtid);
    else if (wtid == 0) bounds_ok(a.m, false, kBndSlotRow);
  } else if (wtid == 0) {
    bounds_ok(a.m, false, kBndSlotRow);
  }
}

// Signals the task's events (after every worker's writes) and frees the
// scheduler for the next task.
__device__ __forceinline__ void finish_task(const KernelArgs& a, Smem& s, const Task& t,
                                            int wtid, bool signal) {
  trace_mark(a, s, wtid, 5);
  worker_sync();
  if (wtid == 0) {
    if (signal && t.n_sig > 0) {
      // release pattern: an acq_rel fence (after the barrier, so it covers
      // every worker's stores) then relaxed increments; measured cheaper
      // than a sequentially consistent fence or a release reduction
      fence_acq_rel_gpu();
      for (int e = 0; e < t.n_sig; ++e) red_relaxed_gpu_add(a.m.events + t.sig_ev0 + e, 1u);
    }
    mbar_arrive(&s.done);
  }
}

// What the epilogue of this thread's first output item needs, loaded before
// the stream so its latency is hidden: RoPE factors and bias (QKV), the old
// residual value (O projection, down).
struct EpiPre {
  float c, sn, b0, b1, res;
};

__device__ __forceinline__ EpiPre epilogue_prefetch(const KernelArgs& a, const StepParams& sp,
                                                    const Task& t, int wtid) {
  const ModelDev& m = a.m;
  EpiPre p{1.f, 0.f, 0.f, 0.f, 0.f};
  const int nrows = t.row1 - t.row0;
  if (t.kind == T_QKV) {
    if (2 * wtid < nrows) {
      const int r = t.row0 + 2 * wtid;
      int which, head, dim;
      qkv_source(r, m.group, m.head_dim, &which, &head, &dim);
      if (which < 2) {
        const int half = m.head_dim >> 1;
        p.c = m.rope_cos[(size_t)sp.pos[0] * half + dim];
        p.sn = m.rope_sin[(size_t)sp.pos[0] * half + dim];
      }
      if (m.qkv_bias) {
        const uint16_t* b = m.bqkv + (size_t)t.layer * qkv_rows(m.n_q, m.n_kv, m.head_dim);
        p.b0 = bf16_to_float(b[r]);
        p.b1 = bf16_to_float(b[r + 1]);
      }
    }
  } else if (t.kind == T_DOWN || (t.kind == T_OPROJ && t.layer > 0)) {
    // the residual rows were written by the stage before the previous one
    if (wtid < nrows) p.res = __ldcg(m.x + t.row0 + wtid);
  }
  return p;
}

__device__ __forceinline__ void epilogue_qkv(const KernelArgs& a, Smem& s, const Task& t, int wtid,
                                             const EpiPre& pre) {
  const ModelDev& m = a.m;
  const StepParams& sp = s.sp_work;
  const int d = m.head_dim, G = m.group, half = d >> 1;
  const int pos = sp.pos[0], slot = sp.kv_slot[0];
  const int qkvR = qkv_rows(m.n_q, m.n_kv, d);
  const int npairs = (t.row1 - t.row0) >> 1;
  for (int pi = wtid; pi < npairs; pi += kWorkerThreads) {
    const int r = t.row0 + 2 * pi;
    float y0 = s.ybuf[2 * pi], y1 = s.ybuf[2 * pi + 1];
    int which, head, dim0, w1, h1, dim1;
    qkv_source(r, G, d, &which, &head, &dim0);
    qkv_source(r + 1, G, d, &w1, &h1, &dim1);
    float c = pre.c, sn = pre.sn, b0 = pre.b0, b1 = pre.b1;
    if (pi != wtid) {  // items past the first load their factors here
      c = 1.f; sn = 0.f; b0 = b1 = 0.f;
      if (which < 2) {
        c = m.rope_cos[(size_t)pos * half + dim0];
        sn = m.rope_sin[(size_t)pos * half + dim0];
      }
      if (m.qkv_bias) {
        const uint16_t* b = m.bqkv + (size_t)t.layer * qkvR;
        b0 = bf16_to_float(b[r]);
        b1 = bf16_to_float(b[r + 1]);
      }
    }
    if (m.qkv_bias) {
      y0 = y0 + b0;
      y1 = y1 + b1;
    }
    if (which < 2) {
      const float o0 = y0 * c - y1 * sn;
      const float o1 = y0 * sn + y1 * c;
      y0 = o0;
      y1 = o1;
    }
    if (which == 0) {
      float* q = m.q + (size_t)head * d;
      if (bounds_ok(m, head < m.n_q && dim0 < d && dim1 < d, kBndQ)) {
        q[dim0] = y0;
        q[dim1] = y1;
      }
    } else {
      uint16_t* cache = which == 1 ? m.kcache : m.vcache;
      const size_t off = kv_offset(m, slot, t.layer, head, pos);
      cache[off + dim0] = float_to_bf16_rne(y0);
      cache[off + dim1] = float_to_bf16_rne(y1);
    }
  }
}

__device__ __forceinline__ void epilogue_residual(const KernelArgs& a, Smem& s, const Task& t, int wtid,
                                                  const EpiPre& pre) {
  const ModelDev& m = a.m;
  const StepParams& sp = s.sp_work;
  const int nrows = t.row1 - t.row0;
  const bool from_embed = t.kind == T_OPROJ && t.layer == 0;
  int tok = 0;
  if (from_embed) {
    tok = sp.tokens[0];
    if (tok < 0 || tok >= m.vocab) tok = 0;
  }
  for (int i = wtid; i < nrows; i += kWorkerThreads) {
    const int row = t.row0 + i;
    if (!bounds_ok(m, row < m.hidden, kBndResidual)) continue;
    const float old = from_embed ? bf16_to_float(m.embed[(size_t)tok * m.hidden + row])
                      : (i == wtid ? pre.res : __ldcg(m.x + row));
    m.x[row] = old + s.ybuf[i];
  }
}

__device__ __forceinline__ void epilogue_swiglu(const KernelArgs& a, Smem& s, const Task& t, int wtid) {
  const ModelDev& m = a.m;
  const int npairs = (t.row1 - t.row0) >> 1;
  for (int pi = wtid; pi < npairs; pi += kWorkerThreads) {
    const float g = s.ybuf[2 * pi], u = s.ybuf[2 * pi + 1];
    const float silu = g / (1.0f + expf(-g));
    if (bounds_ok(m, (t.row0 >> 1) + pi < m.ffn, kBndAct)) m.act[(t.row0 >> 1) + pi] = silu * u;
  }
}

__device__ __forceinline__ void epilogue_lmhead(const KernelArgs& a, Smem& s, const Task& t, int wtid) {
  const ModelDev& m = a.m;
  const StepParams& sp = s.sp_work;
  const int nrows = t.row1 - t.row0;
  unsigned long long best = 0ull;
  for (int i = wtid; i < nrows; i += kWorkerThreads) {
    const float y = s.ybuf[i];
    if (sp.logits && bounds_ok(m, t.row0 + i < m.vocab, kBndLogits)) sp.logits[t.row0 + i] = y;
    const unsigned long long k = argmax_key(y, t.row0 + i);
    best = k > best ? k : best;
  }
  for (int o = 16; o; o >>= 1) {
    const unsigned long long other = __shfl_xor_sync(0xffffffffu, best, o);
    best = other > best ? other : best;
  }
  if ((wtid & 31) == 0) s.red64[wtid >> 5] = best;
  worker_sync();
  if (wtid == 0) {
    unsigned long long b = (t.req & 1) ? 0ull : s.lm_best;
    for (int w = 0; w < kWorkerWarps; ++w) b = s.red64[w] > b ? s.red64[w] : b;
    s.lm_best = b;
    s.flag = 0;
    if ((t.req & 2) && bounds_ok(m, t.aux >= 0 && t.aux < m.n_lm_slots, kBndArgmax)) {
      // the CTA's last LM task publishes its candidate
      m.am[t.aux] = b;
      __threadfence();
      const uint32_t old = atom_add_acq_rel_gpu(m.tickets, 1u);
      s.flag = (old == (uint32_t)m.n_lm_slots * (s.epoch + 1u) - 1u) ? 1 : 0;
    }
  }
  worker_sync();
  if (s.flag) {
    // Last CTA of the step: reduce every CTA's candidate.
    unsigned long long b = 0ull;
    for (int i = wtid; i < m.n_lm_slots; i += kWorkerThreads) {
      const unsigned long long v = __ldcg(m.am + i);
      b = v > b ? v : b;
    }
    for (int o = 16; o; o >>= 1) {
      const unsigned long long other = __shfl_xor_sync(0xffffffffu, b, o);
      b = other > b ? other : b;
    }
    if ((wtid & 31) == 0) s.red64[wtid >> 5] = b;
    worker_sync();
    if (wtid == 0) {
      unsigned long long g = 0ull;
      for (int w = 0; w < kWorkerWarps; ++w) g = s.red64[w] > g ? s.red64[w] : g;
      const int id = (int)(0xffffffffu - (uint32_t)(g & 0xffffffffull));
      if (sp.next_ids) sp.next_ids[0] = id;
      __threadfence();
      red_release_gpu_add(m.epoch, 1u);
    }
  }
}

// ------------------------------------------------------- worker: attention

template <int DPL, int G>
__device__ __forceinline__ void attn_write_state(const AttnState<DPL, G>& st, float* dst, int PS,
                                                 int d, int lane) {
#pragma unroll
  for (int h = 0; h < G; ++h) {
    if constexpr (DPL == 4) {
      *reinterpret_cast<float4*>(dst + h * PS + lane * 4) =
          make_float4(st.o[h][0], st.o[h][1], st.o[h][2], st.o[h][3]);
    } else {
      *reinterpret_cast<float2*>(dst + h * PS + lane * 2) = make_float2(st.o[h][0], st.o[h][1]);
    }
    if (lane == 0) {
      dst[h * PS + d] = st.mx[h];
      dst[h * PS + d + 1] = st.l[h];
    }
  }
}

template <int DPL, int G>
__device__ __forceinline__ void attn_task(const KernelArgs& a, Smem& s, const Task& t, uint32_t& seq, int wtid) {
  const ModelDev& m = a.m;
  const StepParams& sp = s.sp_work;
  const int d = m.head_dim, S_all = m.attn_splits, PS = attn_part_stride(d);
  const int warp = wtid >> 5, lane = wtid & 31;
  const int g = t.row0, split = t.row1, b = t.req;
  const AttnRange r = attn_range(t, sp, m);
  if (!r.active) return;
  AttnState<DPL, G> st;
  // Issue every global load this task needs before touching the ring: the
  // rotated queries of the group, and (in the split that holds it) the newest
  // K/V row, which this step's QKV tasks wrote.
  const int pos = sp.pos[b];
  const bool has_new = pos >= r.k0 && pos < r.k1 && warp == kWorkerWarps - 1;
  float kn[DPL], vn[DPL];
  if (has_new) {
    const size_t off = kv_offset(m, sp.kv_slot[b], t.layer, g, pos);
    load_kv_row_global<DPL>(m.kcache + off + lane * DPL, kn);
    load_kv_row_global<DPL>(m.vcache + off + lane * DPL, vn);
  }
  attn_init<DPL, G>(st, m.q + (size_t)g * G * d, d, m.attn_scale, lane);
  trace_mark(a, s, wtid, 2);
  for (int k = r.k0, nk = 0; k < r.old_end; k += nk) {
    nk = attn_chunk_keys(m, k, r.old_end);
    const int slot = seq % kRingSlots;
    wait_full(s, seq, m);
    if (k == r.k0) trace_mark(a, s, wtid, 3);
    const uint16_t* kb = reinterpret_cast<const uint16_t*>(s.ring[slot]);
    const uint16_t* vb = reinterpret_cast<const uint16_t*>(s.ring[slot] + kSlotBytes / 2);
    // four consecutive keys per warp at a time
    for (int j0 = 4 * warp; j0 < nk; j0 += 4 * kWorkerWarps) {
      const int nj = min(4, nk - j0);
      {
        float kv[4][DPL];
#pragma unroll
        for (int t = 0; t < 4; ++t) {
          const int jr = attn_key_row<G>(t, lane);
          if (jr < nj) load_kv_row<DPL>(kb + (size_t)(j0 + jr) * d + lane * DPL, kv[t]);
          else
#pragma unroll
            for (int i = 0; i < DPL; ++i) kv[t][i] = 0.f;
        }
        attn_scores4<DPL, G>(st, kv, nj, s.attn_xb[warp], lane);
      }
      float vv[4][DPL];
#pragma unroll
      for (int t = 0; t < 4; ++t) {
        if (t < nj) load_kv_row<DPL>(vb + (size_t)(j0 + t) * d + lane * DPL, vv[t]);
        else
#pragma unroll
          for (int i = 0; i < DPL; ++i) vv[t][i] = 0.f;
      }
      attn_update4<DPL, G>(st, vv, s.attn_xb[warp]);
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&s.empty[slot]);
    ++seq;
  }
  if (has_new) {  // the newest key, as a batch of one (warp-uniform branch)
    float kv[4][DPL], vv[4][DPL];
#pragma unroll
    for (int t = 0; t < 4; ++t) {
      const bool mine = attn_key_row<G>(t, lane) == 0;
#pragma unroll
      for (int i = 0; i < DPL; ++i) {
        kv[t][i] = mine ? kn[i] : 0.f;
        vv[t][i] = t == 0 ? vn[i] : 0.f;
      }
    }
    attn_scores4<DPL, G>(st, kv, 1, s.attn_xb[warp], lane);
    attn_update4<DPL, G>(st, vv, s.attn_xb[warp]);
  }
  trace_mark(a, s, wtid, 4);
  // Merge the 16 warps' (max, sum, output): warps 8-15 into warps 0-7, then
  // one pass over the 8 remaining states with one output element per thread.
  float* buf = s.scratch;
  const int sw = G * PS;
  constexpr int kHalf = kWorkerWarps / 2;
  if (warp >= kHalf) attn_write_state<DPL, G>(st, buf + (warp - kHalf) * sw, PS, d, lane);
  worker_sync();
  if (warp < kHalf) {
    const float* src = buf + warp * sw;
#pragma unroll
    for (int h = 0; h < G; ++h) {
      const float m2 = src[h * PS + d], l2 = src[h * PS + d + 1];
      if (m2 == -INFINITY) continue;
      float o2[DPL];
#pragma unroll
      for (int i = 0; i < DPL; ++i) o2[i] = src[h * PS + lane * DPL + i];
      if (st.mx[h] == -INFINITY) {
        st.mx[h] = m2;
        st.l[h] = l2;
#pragma unroll
        for (int i = 0; i < DPL; ++i) st.o[h][i] = o2[i];
      } else {
        const float mn = fmaxf(st.mx[h], m2);
        const float c1 = __expf(st.mx[h] - mn), c2 = __expf(m2 - mn);
        st.l[h] = st.l[h] * c1 + l2 * c2;
#pragma unroll
        for (int i = 0; i < DPL; ++i) st.o[h][i] = st.o[h][i] * c1 + o2[i] * c2;
        st.mx[h] = mn;
      }
    }
  }
  worker_sync();
  if (warp < kHalf) attn_write_state<DPL, G>(st, buf + warp * sw, PS, d, lane);
  worker_sync();
  const int live = r.live;
  if (!bounds_ok(m, b == 0 && (g + 1) * G <= m.n_q, kBndAttnOut)) return;
  if (live == 1) {
    // the only split: normalise and write the attention output directly
    float* out = m.attn + ((size_t)b * m.n_q + (size_t)g * G) * d;
    for (int idx = wtid; idx < G * d; idx += kWorkerThreads) {
      const int h = idx / d, i = idx - h * d;
      float M = -INFINITY;
#pragma unroll
      for (int w = 0; w < kHalf; ++w) M = fmaxf(M, buf[w * sw + h * PS + d]);
      float num = 0.f, den = 0.f;
#pragma unroll
      for (int w = 0; w < kHalf; ++w) {
        const float mw = buf[w * sw + h * PS + d];
        if (mw == -INFINITY) continue;
        const float c = __expf(mw - M);
        num = fmaf(c, buf[w * sw + h * PS + i], num);
        den = fmaf(c, buf[w * sw + h * PS + d + 1], den);
      }
      out[h * d + i] = num / den;
    }
    return;
  }
  // The split's partial -- output unnormalised at the split's maximum, the
  // maximum, the sum.
  if (!bounds_ok(m, b == 0 && g < m.n_kv && split < S_all, kBndPart)) return;
  float* part = m.part + ((size_t)(b * m.n_kv + g) * S_all + split) * G * PS;
  for (int idx = wtid; idx < G * (d + 2); idx += kWorkerThreads) {
    const int h = idx / (d + 2), i = idx - h * (d + 2);
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < kHalf; ++w) M = fmaxf(M, buf[w * sw + h * PS + d]);
    float val = 0.f;
    if (M != -INFINITY) {
#pragma unroll
      for (int w = 0; w < kHalf; ++w) {
        const float mw = buf[w * sw + h * PS + d];
        if (mw == -INFINITY) continue;
        const float x = i < d ? buf[w * sw + h * PS + i] : buf[w * sw + h * PS + d + 1];
        val = fmaf(__expf(mw - M), x, val);
      }
    }
    // i < d: output dim i; i == d: the maximum; i == d + 1: the sum
    part[h * PS + i] = i == d ? M : val;
  }
  // The last of the `live` split tasks of this (request, KV head) to finish
  // merges them into the attention output (online softmax, "Hạt nhân là gì
  // ...": each split's sum and output rescaled to the common maximum), then
  // divides by the sum.  It also puts the ticket back to zero for the next
  // step, which reaches it only after this step's events.
  worker_sync();
  if (wtid == 0) {
    const size_t ti = kAttnTicketBase + ((size_t)t.layer * m.max_batch + b) * m.n_kv + g;
    uint32_t* tk = m.tickets + (bounds_ok(m, ti < (size_t)m.n_tickets, kBndTicket) ? ti : 0);
    const uint32_t old = atom_add_acq_rel_gpu(tk, 1u);  // release: this split's partial
    const bool last = old == (uint32_t)live - 1u;
    if (last) *tk = 0u;
    s.attn_last = last;
  }
  worker_sync();
  if (!s.attn_last) return;
  const float* pg = m.part + (size_t)(b * m.n_kv + g) * S_all * G * PS;
  // every split's (maximum, sum) into shared memory, then the common maxima
  float* ml = buf;  // [live][G][2]
  for (int idx = wtid; idx < live * G; idx += kWorkerThreads) {
    const float2 v = __ldcg(reinterpret_cast<const float2*>(pg + (size_t)idx * PS + d));
    ml[2 * idx] = v.x;
    ml[2 * idx + 1] = v.y;
  }
  worker_sync();
  float* out = m.attn + ((size_t)b * m.n_q + (size_t)g * G) * d;
  for (int idx = wtid; idx < G * d; idx += kWorkerThreads) {
    const int h = idx / d, i = idx - h * d;
    float M = -INFINITY;
    for (int sp_ = 0; sp_ < live; ++sp_)
      if (ml[2 * (sp_ * G + h) + 1] != 0.f) M = fmaxf(M, ml[2 * (sp_ * G + h)]);
    float num = 0.f, den = 0.f;
#pragma unroll 4
    for (int sp_ = 0; sp_ < live; ++sp_) {
      const float ls = ml[2 * (sp_ * G + h) + 1];
      const float o = __ldcg(pg + ((size_t)sp_ * G + h) * PS + i);
      if (ls == 0.f) continue;  // a split without keys
      const float c = __expf(ml[2 * (sp_ * G + h)] - M);
      num = fmaf(c, o, num);
      den = fmaf(c, ls, den);
    }
    out[h * d + i] = num / den;
  }
}

// ------------------------------------------------------------------ worker

template <int PW, int DPL, int G>
__device__ __forceinline__ void worker(const KernelArgs& a, Smem& s, int q0, int q1) {
  const int wtid = threadIdx.x - kFirstWorkerWarp * 32;
  uint32_t seq = 0;
  int i = 0;
  bool stop = false;
  for (int step = 0; step < a.n_steps && !stop; ++step)
  for (int qi = q0; qi < q1; ++qi, ++i) {
    const Task t = a.tasks[a.queue[qi]];
    const bool go = wait_bounded(s, &s.ready, i & 1, a.m, kWaitReady);
    // all workers agree: the flag was published before the ready arrival
    worker_sync();
    if (!go || aborting(s)) { stop = true; break; }
    if (wtid == 0) s.cur_qi = qi;  // read by this thread only (trace_mark)
    trace_mark(a, s, wtid, 1);
    switch (t.kind) {
      case T_ATTN:
        attn_task<DPL, G>(a, s, t, seq, wtid);
        finish_task(a, s, t, wtid, true);
        break;
      case T_LMHEAD:
        gemv_core<PW>(a, s, t, seq, wtid);
        epilogue_lmhead(a, s, t, wtid);
        finish_task(a, s, t, wtid, false);
        break;
      default: {
        const EpiPre pre = epilogue_prefetch(a, s.sp_work, t, wtid);
        gemv_core<PW>(a, s, t, seq, wtid);
        if (t.kind == T_QKV) epilogue_qkv(a, s, t, wtid, pre);
        else if (t.kind == T_GATEUP) epilogue_swiglu(a, s, t, wtid);
        else epilogue_residual(a, s, t, wtid, pre);
        finish_task(a, s, t, wtid, true);
        break;
      }
    }
    if (a.m.trace && wtid == 0) {
      a.m.trace[(size_t)qi * kTraceWords + 6] = globaltimer_ns();
      a.m.trace[(size_t)qi * kTraceWords + 7] =
          ((unsigned long long)blockIdx.x << 32) | (unsigned)a.queue[qi];
    }
  }
}

// PW 4: bf16 weights; PW 8: fp8 e4m3 weights with row scales.  DPL: head_dim
// / 32 (dims per lane); G: query heads per KV head.
template <int PW, int DPL, int G>
__global__ void __launch_bounds__(kThreads, 1) mk_step_kernel(const __grid_constant__ KernelArgs a) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  Smem& s = *reinterpret_cast<Smem*>(smem_raw);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int q0 = a.queue_off[blockIdx.x], q1 = a.queue_off[blockIdx.x + 1];
  if (threadIdx.x == 0) {
    for (int i = 0; i < kRingSlots; ++i) {
      mbar_init(&s.full[i], 1);
      mbar_init(&s.empty[i], kWorkerWarps);
    }
    mbar_init(&s.ready, 1);
    mbar_init(&s.done, 1);
    s.abort_flag = 0;
    s.flag = 0;
    s.epoch = *reinterpret_cast<volatile uint32_t*>(a.m.epoch);
    s.epoch0 = s.epoch;
    step_at(a, 0, s.sp_work);
    fence_barrier_init();
  }
  __syncthreads();
  if (q0 == q1) return;
  if (warp < kProducerWarps) {
    if (lane == 0) producer(a, s, q0, q1, warp);
  } else if (warp == kSchedulerWarp) {
    if (lane == 0) scheduler(a, s, q0, q1);
  } else {
    worker<PW, DPL, G>(a, s, q0, q1);
  }
}

// Kernel of one (weight width, head_dim, query heads per KV head), or null
// when that combination is not built; defined by the step_*.cu files.
const void* step_kernel_bf16_d128(int G);
const void* step_kernel_bf16_d64(int G);
const void* step_kernel_fp8_d128(int G);
const void* step_kernel_fp8_d64(int G);

}  // namespace mk
