// prefill_mk.cu -- the tensor-core prompt prefill as ONE persistent kernel per
// block of prompt positions: every operator of every layer is a task of a
// task graph ("LLMs in einen MegaKernel kompilieren ...", "Part 1. Compiler":
// operators refined into SM-sized tasks linked by events, dependencies that
// follow data tiles rather than kernel boundaries; "MPK: A Compiler and
// Runtime ..." idea 3: a graph that depends on the data -- here the prompt
// lengths -- is built when the call arrives).
//
// The block's positions are cut into token tiles of 128.  Per layer and token
// tile n the tasks are (the elementwise ones -- NORM, ROPE, RES1, SWIGLU,
// RES2 -- split into 16 tasks of 8 positions, so that many SMs share them)
//   NORM    (layer 0 only) x = E[token]; the attention RMSNorm as three bf16 parts
//   QKV     one per 128-row tile m of W_qkv: a tcgen05 GEMM tile (128 rows x
//           the tile's tokens), waits for the norms of tile n only
//   ROPE    RoPE q, K/V into the cache; waits for every QKV tile of n
//   ATTN    causal GQA attention on the tensor cores (fa_tile, flash_attn.cuh),
//           per (run of one request's positions inside tile n, query head);
//           waits for the ROPE of every token tile up to its own (the keys it
//           reads)
//   OPROJ   GEMM tiles of W_o; wait for the ATTN tasks of tile n
//   RES1    x += W_o attn, the FFN RMSNorm as three parts; waits for OPROJ of n
//   GATEUP  GEMM tiles of W_gate/up; wait for RES1 of n
//   SWIGLU  silu(gate) * up as three parts; waits for GATEUP of n
//   DOWN    GEMM tiles of W_down; wait for SWIGLU of n
//   RES2    x += W_down act and the next layer's attention RMSNorm (after the
//           last layer the final norm); waits for DOWN of n
//   LM      (tiles holding a prompt's last position) a GEMM tile of 128 rows
//           of the LM head; writes those positions' logits and folds the
//           rows' maximum into each request's argmax key; waits for the final
//           norms of tile n
// so a token tile runs ahead through the layer while other tiles are still in
// earlier stages.  Every CTA walks its ahead-of-time queue in this order (all
// CTAs co-resident, cooperative launch), which keeps the earliest unfinished
// task runnable: no deadlock.  Every wait is bounded and recorded.
//
// The GEMM tile is the prefill GEMM of prefill.cu run inside the loop: the
// weights and the three activation parts arrive by 2-D TMA (tensor maps in
// global memory) in a 3-stage ring issued by two threads, lane 0 of warp 1
// issues tcgen05.mma into three tensor-memory accumulators (allocated once
// per CTA), warps 0-3 read them back.  The ring's and the accumulators'
// phases run on across tiles.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <algorithm>
#include <cmath>
#include <string>
#include <vector>

#include "../../include/mk.h"
#include "flash_attn.cuh"
#include "mk_internal.h"
#include "plan.h"
#include "prefill.h"
#include "ptx.cuh"
#include "tc.cuh"

namespace mk {

PFN_cuTensorMapEncodeTiled_v12000 prefill_encode_fn();  // prefill.cu

namespace {

constexpr int kPfThreads = 512;
constexpr int kPfTokTile = 128;      // tokens per token tile (the GEMM's N)
constexpr int kPfRows = 128;         // weight rows per GEMM tile (the MMA's M)
constexpr int kPfK = 64;             // K per stage
constexpr int kPfStages = 3;
constexpr int kPfEwTok = 8;          // positions per elementwise task (norm, RoPE, residual, SwiGLU)
constexpr int kPfEwSub = kPfTokTile / kPfEwTok;  // elementwise tasks per token tile

enum PfKind : int32_t {
  PF_NORM = 0, PF_GEMM = 1, PF_ROPE = 2, PF_ATTN = 3, PF_RES1 = 4, PF_SWIGLU = 5, PF_RES2 = 6
};
enum PfMat : int32_t { PF_QKV = 0, PF_O = 1, PF_GU = 2, PF_DN = 3, PF_LM = 4 };

struct PfTask {
  int32_t kind, layer;
  int32_t n;          // token tile
  int32_t a, b;       // GEMM: matrix (PfMat), row tile; ATTN: attention tile, KV head
  int32_t wait_ev;    // -1: none
  uint32_t wait_count;
  int32_t sig_ev0, n_sig;
  int32_t pad_[3];
};
static_assert(sizeof(PfTask) == 48, "PfTask layout");

struct PfArgs {
  ModelDev m;
  const PfTask* tasks;
  const int32_t* queue;
  const int32_t* queue_off;       // [grid + 1]
  const CUtensorMap* maps;        // [4 L] weight tiles, [3 parts][3 K kinds] activations, the
                                  // KV cache (K, K second half, V, V second half), the LM head
  uint32_t* events;
  int32_t* err;                   // [0]: first error code, [1]: detail
  const int32_t* tokens;          // the prompt tokens (device)
  const int32_t* tok_src;         // [T] index into tokens of block token t
  const int32_t* slot;            // [T] KV slot of token t
  const int32_t* pos;             // [T] position of token t
  const int32_t* attn_tiles;      // [n_attn][4]: first token, count, slot, first position
  float qscale;                   // attention scale * log2(e)
  float* x;                       // [T][H]
  float* y;                       // [T][ldy]
  float* q;                       // [T][n_q d]
  uint16_t* xh;                   // [T][ldx] three bf16 parts of the GEMM input (the
  uint16_t* xm;                   // first K columns of a row; one row stride for every
  uint16_t* xl;                   // stage, since token tiles sit in different stages)
  int32_t T, ldy, ldx;
  uint64_t* trace;                // per-task timeline (4 words per task index) or null
  int32_t trace_cap;
  uint64_t wait_ns;               // limit of every wait
  // the prompts' last positions: LM head and greedy id inside the kernel
  const int32_t* lm_req;          // [T] request whose last position token t is, or -1
  unsigned long long* lm_keys;    // [requests] argmax keys (larger value, then lower index)
  float* logits;                  // [requests][vocab] or null
};

// Orderable key of (logit, vocabulary index): larger value first, then the
// lower index (the greedy id's tie rule).
__device__ __forceinline__ unsigned long long pf_argmax_key(float v, int idx) {
  uint32_t u = __float_as_uint(v);
  u = (u & 0x80000000u) ? ~u : (u | 0x80000000u);
  return ((unsigned long long)u << 32) | (0xffffffffu - (uint32_t)idx);
}

// maps[] index of an activation part (0 high, 1 middle, 2 low) for a GEMM over
// K = hidden (0), n_q d (1) or ffn (2)
__host__ __device__ __forceinline__ int pf_xmap(int L, int part, int kk) { return 4 * L + 3 * part + kk; }
// maps[] index of the KV-cache maps (K first half, K second half, V, V second half)
__host__ __device__ __forceinline__ int pf_kvmap(int L, int i) { return 4 * L + 9 + i; }
// maps[] index of the LM head
__host__ __device__ __forceinline__ int pf_lmmap(int L) { return 4 * L + 13; }
constexpr int kPfMapsExtra = 14;  // maps past the 4 L weight maps

struct __align__(1024) PfSmem {
  // GEMM stages (the attention tasks use the same 192 KB as FaBuffers)
  uint8_t a[kPfStages][kPfRows * kPfK * 2];
  uint8_t bh[kPfStages][kPfTokTile * kPfK * 2];
  uint8_t bm[kPfStages][kPfTokTile * kPfK * 2];
  uint8_t bl[kPfStages][kPfTokTile * kPfK * 2];
  uint64_t full[kPfStages];
  uint64_t empty[kPfStages];
  uint64_t done;
  uint32_t tmem;
  int32_t abort_flag;
  int32_t tmem_ok;   // cleared when an accumulator wait gave up (MMAs may be in flight)
  uint32_t armed[kPfStages];  // the last ring position whose loads went to each stage
  FaBarriers fab;             // the attention tasks' barriers
  float ew_red[16];           // per-warp sums of squares of the residual/norm tasks
};
static_assert(offsetof(PfSmem, a) == 0 && kPfStages * 4 * kPfRows * kPfK * 2 == sizeof(FaBuffers),
              "the attention buffers alias the GEMM stages");
constexpr uint32_t kPfStageBytes = kPfRows * kPfK * 2 + 3 * kPfTokTile * kPfK * 2;
constexpr uint32_t kPfTmemCols = 512;  // three 128-column accumulators

__device__ __forceinline__ uint16_t pf_bf16(float f) {
  __nv_bfloat16 b = __float2bfloat16_rn(f);
  return *reinterpret_cast<uint16_t*>(&b);
}
__device__ __forceinline__ float pf_val(uint16_t h) { return __uint_as_float((uint32_t)h << 16); }

// v -> three bf16 parts whose sum is v
__device__ __forceinline__ void pf_split3(float v, uint16_t* hi, uint16_t* mid, uint16_t* lo, size_t i) {
  const uint16_t h = pf_bf16(v);
  const float r1 = v - pf_val(h);
  const uint16_t md = pf_bf16(r1);
  hi[i] = h;
  mid[i] = md;
  lo[i] = pf_bf16(r1 - pf_val(md));
}

__device__ __forceinline__ void pf_fail(const PfArgs& p, PfSmem& s, int code, int detail) {
  if (atomicCAS(p.err, 0, code) == 0) p.err[1] = detail;
  *(volatile int32_t*)&s.abort_flag = 1;
}

__device__ __forceinline__ bool pf_wait(const PfArgs& p, PfSmem& s, uint64_t* bar, uint32_t parity,
                                        int where) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = globaltimer_ns();
  while (!mbar_try_wait(bar, parity)) {
    if (*(volatile int32_t*)&s.abort_flag) return false;
    if (globaltimer_ns() - t0 > p.wait_ns) {
      pf_fail(p, s, MK_ERR_TIMEOUT, where);
      return false;
    }
  }
  return true;
}

// Wait without regard to the abort flag, bounded (the abort path's drain).
__device__ __forceinline__ bool pf_drain(uint64_t* bar, uint32_t parity) {
  const uint64_t t0 = globaltimer_ns();
  while (!mbar_try_wait(bar, parity))
    if (globaltimer_ns() - t0 > 200000000ull) return false;
  return true;
}

// Rows [e0, e1) (at most kPfEwTok) of the residual stream: x (+)= src, then
// the RMSNorm of the new x times w as the next GEMM's three bf16 parts.  Two
// warps per row (each half of the columns), 16-byte accesses; `src` is the
// GEMM output y (add = true) or the embedding rows (add = false).
__device__ __forceinline__ void pf_residual_norm(const PfArgs& p, PfSmem& s, int e0, int e1, bool add,
                                                 const uint16_t* w) {
  const ModelDev& m = p.m;
  const int H = m.hidden, Hh = H >> 1;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int t = e0 + (warp & 7), c0 = (warp >> 3) * Hh;
  const bool live = warp < 16 && t < e1;
  float ss = 0.f;
  if (live) {
    float* xr = p.x + (size_t)t * H;
    const uint16_t* er = nullptr;
    if (!add) {
      int tok = __ldg(p.tokens + __ldg(p.tok_src + t));
      if (tok < 0 || tok >= m.vocab) {
        if (atomicCAS(m.status, 0, MK_ERR_TOKEN_RANGE) == 0) m.status_info[0] = tok;
        tok = 0;
      }
      er = m.embed + (size_t)tok * H;
    }
    for (int i = c0 + lane * 4; i < c0 + Hh; i += 128) {
      float4 v;
      if (add) {
        const float4 a = __ldcg(reinterpret_cast<const float4*>(xr + i));
        const float4 b = __ldcg(reinterpret_cast<const float4*>(p.y + (size_t)t * p.ldy + i));
        v = make_float4(a.x + b.x, a.y + b.y, a.z + b.z, a.w + b.w);
      } else {
        const uint2 e = __ldg(reinterpret_cast<const uint2*>(er + i));
        v = make_float4(__uint_as_float(e.x << 16), __uint_as_float(e.x & 0xFFFF0000u),
                        __uint_as_float(e.y << 16), __uint_as_float(e.y & 0xFFFF0000u));
      }
      *reinterpret_cast<float4*>(xr + i) = v;
      ss = fmaf(v.x, v.x, ss);
      ss = fmaf(v.y, v.y, ss);
      ss = fmaf(v.z, v.z, ss);
      ss = fmaf(v.w, v.w, ss);
    }
    for (int o = 16; o; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
  }
  if (lane == 0 && warp < 16) s.ew_red[warp] = ss;
  __syncthreads();
  if (!live || !w) return;
  const float tot = s.ew_red[warp & 7] + s.ew_red[(warp & 7) + 8];
  const float r = 1.0f / sqrtf(tot / (float)H + m.rms_eps);
  const float* xr = p.x + (size_t)t * H;
  for (int i = c0 + lane * 4; i < c0 + Hh; i += 128) {
    const float4 v = *reinterpret_cast<const float4*>(xr + i);  // this thread's own stores
    const uint2 wv = __ldg(reinterpret_cast<const uint2*>(w + i));
    const size_t o = (size_t)t * p.ldx + i;
    pf_split3(v.x * r * pf_val((uint16_t)(wv.x & 0xFFFFu)), p.xh, p.xm, p.xl, o);
    pf_split3(v.y * r * pf_val((uint16_t)(wv.x >> 16)), p.xh, p.xm, p.xl, o + 1);
    pf_split3(v.z * r * pf_val((uint16_t)(wv.y & 0xFFFFu)), p.xh, p.xm, p.xl, o + 2);
    pf_split3(v.w * r * pf_val((uint16_t)(wv.y >> 16)), p.xh, p.xm, p.xl, o + 3);
  }
}

// ----------------------------------------------------------------- GEMM tile

struct PfGemmState {
  uint32_t kb;      // k blocks issued / consumed by this CTA so far (ring position)
  uint32_t tiles;   // GEMM tiles finished by this CTA so far (accumulator phase)
};

// Y[t][r] = sum_k W[r][k] (xh + xm + xl)[t][k] for rows [m0, m0 + 128) and the
// tokens of tile n; bias added when given.
__device__ __forceinline__ void pf_gemm_tile(const PfArgs& p, PfSmem& s, PfGemmState& gs,
                                             const CUtensorMap* tm_w, int kk, int K, int n_rows,
                                             int m0, int n, const uint16_t* bias, bool lm) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nk = K / kPfK;
  const int L = p.m.n_layers;
  const CUtensorMap* th = p.maps + pf_xmap(L, 0, kk);
  const CUtensorMap* tmm = p.maps + pf_xmap(L, 1, kk);
  const CUtensorMap* tl = p.maps + pf_xmap(L, 2, kk);
  const int n0 = n * kPfTokTile;
  // the tile's positions that exist (a block's last tile may be short): the
  // MMAs' N covers them rounded up to 16, the columns past them are not read
  const int nmma = (max(1, min(kPfTokTile, p.T - n0)) + 15) & ~15;
  if ((warp == 0 || warp == 2) && lane == 0) {
    // two issuing threads, alternate k blocks (one thread's TMA loads run one
    // after another).  The stage memory may have been written by an attention
    // task's generic stores: order them before the async-proxy writes.
    fence_proxy_async_shared();
    fence_proxy_async_global();
    const int pid = warp >> 1;
    for (int i = pid; i < nk; i += 2) {
      const uint32_t g = gs.kb + i;
      const int st = g % kPfStages;
      if (g >= kPfStages && !pf_wait(p, s, &s.empty[st], ((g / kPfStages) - 1) & 1, -21)) break;
      mbar_arrive_expect_tx(&s.full[st], kPfStageBytes);
      s.armed[st] = g;
      tma_load_2d(s.a[st], tm_w, i * kPfK, m0, &s.full[st]);
      tma_load_2d(s.bh[st], th, i * kPfK, n0, &s.full[st]);
      tma_load_2d(s.bm[st], tmm, i * kPfK, n0, &s.full[st]);
      tma_load_2d(s.bl[st], tl, i * kPfK, n0, &s.full[st]);
    }
  } else if (warp == 1 && lane == 0) {
    const uint32_t idesc = mma_idesc_bf16_f32(kPfRows, nmma);
    tc_fence_after_sync();
    for (int i = 0; i < nk; ++i) {
      const uint32_t g = gs.kb + i;
      const int st = g % kPfStages;
      if (!pf_wait(p, s, &s.full[st], (g / kPfStages) & 1, -22)) break;
      tc_fence_after_sync();
      const uint64_t da = sw128_kmajor_desc(s.a[st]);
      const uint64_t dh = sw128_kmajor_desc(s.bh[st]);
      const uint64_t dm = sw128_kmajor_desc(s.bm[st]);
      const uint64_t dl = sw128_kmajor_desc(s.bl[st]);
      const uint32_t acc_h = s.tmem + ((i & 1) ? 2u * kPfTokTile : 0u);
      const uint32_t acc_ml = s.tmem + (uint32_t)kPfTokTile;
#pragma unroll
      for (int k = 0; k < kPfK / 16; ++k) {
        tc_mma_f16(acc_h, da + 2 * k, dh + 2 * k, idesc, (i > 1 || k > 0) ? 1u : 0u);
        tc_mma_f16(acc_ml, da + 2 * k, dm + 2 * k, idesc, (i | k) != 0);
        tc_mma_f16(acc_ml, da + 2 * k, dl + 2 * k, idesc, 1u);
      }
      tc_commit(&s.empty[st]);
    }
    tc_commit(&s.done);  // also when stopped early: retires what was issued
  }
  __syncwarp();
  gs.kb += nk;
  // accumulators ready: warps 0-3 (tensor-memory lanes 32 w ..) read them
  const uint32_t ph = gs.tiles & 1u;
  gs.tiles += 1;
  if (warp < 4) {
    const bool ok = pf_wait(p, s, &s.done, ph, -23);
    if (!ok) s.tmem_ok = 0;
    tc_fence_after_sync();
    if (ok) {
      const int row = m0 + warp * 32 + lane;
      const float b = (bias && row < n_rows) ? pf_val(bias[row]) : 0.f;
      const bool odd = nk > 1;
#pragma unroll 1
      for (int c0 = 0; c0 < nmma; c0 += 16) {
        float v[16], ml[16], v2[16];
        const uint32_t base = s.tmem + ((uint32_t)(warp * 32) << 16) + (uint32_t)c0;
        tmem_ld16(base, v);
        tmem_ld16(base + (uint32_t)kPfTokTile, ml);
        if (odd) tmem_ld16(base + 2u * kPfTokTile, v2);
        if (lm) {
          // LM head: the prompts' last positions only -- their logits, and the
          // warp's best (logit, row) per request folded into the request's key
#pragma unroll 1
          for (int j = 0; j < 16; ++j) {
            const int tok = n0 + c0 + j;
            const int req = tok < p.T ? __ldg(p.lm_req + tok) : -1;  // warp-uniform
            if (req < 0) continue;
            const float val = (v[j] + (odd ? v2[j] : 0.f)) + ml[j];
            if (row < n_rows && p.logits) p.logits[(size_t)req * n_rows + row] = val;
            unsigned long long key = row < n_rows ? pf_argmax_key(val, row) : 0ull;
#pragma unroll
            for (int o = 16; o; o >>= 1) {
              const unsigned long long other = __shfl_xor_sync(0xffffffffu, key, o);
              key = other > key ? other : key;
            }
            if (lane == 0) atomicMax(p.lm_keys + req, key);
          }
        } else if (row < n_rows) {
#pragma unroll
          for (int j = 0; j < 16; ++j) {
            const int tok = n0 + c0 + j;
            if (tok < p.T) p.y[(size_t)tok * p.ldy + row] = (v[j] + (odd ? v2[j] : 0.f)) + ml[j] + b;
          }
        }
      }
    }
  }
  tc_fence_before_sync();
}

// --------------------------------------------------------- other task bodies

// RoPE on the packed q/k rows, q to p.q, K/V (bf16) into the cache, for the
// tokens of tile n (the decode step's QKV epilogue, over many tokens).
__device__ __forceinline__ void pf_rope(const PfArgs& p, int layer, int t0, int t1) {
  const ModelDev& m = p.m;
  const int d = m.head_dim, G = m.group, half = d >> 1;
  const int npairs = qkv_rows(m.n_q, m.n_kv, d) >> 1;
  const uint16_t* bias = m.qkv_bias ? m.bqkv + (size_t)layer * qkv_rows(m.n_q, m.n_kv, d) : nullptr;
  const int total = (t1 - t0) * npairs;
  for (int idx = threadIdx.x; idx < total; idx += kPfThreads) {
    const int t = t0 + idx / npairs, pi = idx - (idx / npairs) * npairs;
    const int r = 2 * pi, ps = p.pos[t], sl = p.slot[t];
    float y0 = __ldcg(p.y + (size_t)t * p.ldy + r), y1 = __ldcg(p.y + (size_t)t * p.ldy + r + 1);
    if (bias) {
      y0 += pf_val(bias[r]);
      y1 += pf_val(bias[r + 1]);
    }
    int which, head, dim0, w1, h1, dim1;
    qkv_source(r, G, d, &which, &head, &dim0);
    qkv_source(r + 1, G, d, &w1, &h1, &dim1);
    if (which < 2) {
      const float c = m.rope_cos[(size_t)ps * half + dim0], sn = m.rope_sin[(size_t)ps * half + dim0];
      const float o0 = y0 * c - y1 * sn, o1 = y0 * sn + y1 * c;
      y0 = o0;
      y1 = o1;
    }
    if (which == 0) {
      float* qq = p.q + (size_t)t * m.n_q * d + (size_t)head * d;
      qq[dim0] = y0;
      qq[dim1] = y1;
    } else {
      uint16_t* cache = which == 1 ? m.kcache : m.vcache;
      const size_t off = kv_row(m, sl, layer, head, ps);
      cache[off + dim0] = pf_bf16(y0);
      cache[off + dim1] = pf_bf16(y1);
    }
  }
}

// ----------------------------------------------------------------- the kernel

__global__ void __launch_bounds__(kPfThreads, 1) prefill_mk_kernel(const __grid_constant__ PfArgs p) {
  extern __shared__ __align__(16) uint8_t pf_raw[];
  const uint32_t base = smem_u32(pf_raw);
  PfSmem& s = *reinterpret_cast<PfSmem*>(pf_raw + (((base + 1023u) & ~1023u) - base));
  const int warp = threadIdx.x >> 5;
  const ModelDev& m = p.m;
  if (threadIdx.x == 0) {
    for (int i = 0; i < kPfStages; ++i) {
      mbar_init(&s.full[i], 1);
      mbar_init(&s.empty[i], 1);
    }
    mbar_init(&s.done, 1);
    for (int i = 0; i < kPfStages; ++i) s.armed[i] = 0xffffffffu;
    fa_init_barriers(s.fab);
    s.abort_flag = 0;
    s.tmem_ok = 1;
    fence_barrier_init();
  }
  if (warp == 0) {
    tmem_alloc(&s.tmem, kPfTmemCols);
    tmem_relinquish();
  }
  tc_fence_before_sync();
  __syncthreads();
  tc_fence_after_sync();
  PfGemmState gs{0u, 0u};
  uint32_t fa_calls = 0;  // attention tasks run by this CTA
  FaBuffers& fab_buf = *reinterpret_cast<FaBuffers*>(&s.a[0][0]);
  auto fwait = [&](uint64_t* bar, uint32_t parity, int where) { return pf_wait(p, s, bar, parity, where); };
  const int q0 = p.queue_off[blockIdx.x], q1 = p.queue_off[blockIdx.x + 1];
  const int H = m.hidden, F = m.ffn, L = m.n_layers, qd = m.n_q * m.head_dim;
  const int qkvR = qkv_rows(m.n_q, m.n_kv, m.head_dim);
  __shared__ int s_go;
  for (int qi = q0; qi < q1; ++qi) {
    const int ti = p.queue[qi];
    const PfTask t = p.tasks[ti];
    uint64_t tw0 = 0, tw1 = 0;
    if (threadIdx.x == 0) {
      if (p.trace) tw0 = globaltimer_ns();
      int go = *(volatile int32_t*)&s.abort_flag == 0;
      if (go && t.wait_ev >= 0) {
        const uint64_t t0 = globaltimer_ns();
        uint32_t spins = 0;
        while (ld_acquire_gpu(p.events + t.wait_ev) < t.wait_count) {
          if ((++spins & 63u) == 0) {
            if (ld_relaxed_gpu_s32(p.err) != 0) { go = 0; break; }
            if (globaltimer_ns() - t0 > p.wait_ns) {
              pf_fail(p, s, MK_ERR_TIMEOUT, qi);
              go = 0;
              break;
            }
          }
        }
        // the inputs were written by generic stores of other CTAs; the GEMM
        // tiles read them through the async proxy (TMA)
        fence_proxy_async_global();
      }
      if (p.trace) tw1 = globaltimer_ns();
      s_go = go;
    }
    __syncthreads();
    if (!s_go) break;
    const int n = t.n, t0 = n * kPfTokTile;
    // elementwise tasks: positions [e0, e1) of the tile
    const int e0 = t0 + t.b * kPfEwTok, e1 = min(p.T, e0 + kPfEwTok);
    const int l = t.layer;
    switch (t.kind) {
      case PF_NORM:
        pf_residual_norm(p, s, e0, e1, false, m.attn_norm);
        break;
      case PF_GEMM: {
        const int mat = t.a, m0 = t.b * kPfRows;
        const CUtensorMap* tm_w = mat == PF_LM ? p.maps + pf_lmmap(L) : p.maps + 4 * l + mat;
        if (mat == PF_QKV)  // (the bias is added with RoPE)
          pf_gemm_tile(p, s, gs, tm_w, 0, H, qkvR, m0, n, nullptr, false);
        else if (mat == PF_O)
          pf_gemm_tile(p, s, gs, tm_w, 1, qd, H, m0, n, nullptr, false);
        else if (mat == PF_GU)
          pf_gemm_tile(p, s, gs, tm_w, 0, H, 2 * F, m0, n, nullptr, false);
        else if (mat == PF_DN)
          pf_gemm_tile(p, s, gs, tm_w, 2, F, H, m0, n, nullptr, false);
        else  // LM head over the final norm of the tile (the last layer's RES2)
          pf_gemm_tile(p, s, gs, tm_w, 0, H, m.vocab, m0, n, nullptr, true);
        break;
      }
      case PF_ROPE:
        pf_rope(p, l, e0, e1);
        break;
      case PF_ATTN: {
        const int* tl = p.attn_tiles + 4 * t.a;
        FaJob j;
        j.mk0 = p.maps + pf_kvmap(L, 0);
        j.mk1 = p.maps + pf_kvmap(L, 1);
        j.mv0 = p.maps + pf_kvmap(L, 2);
        j.mv1 = p.maps + pf_kvmap(L, 3);
        j.q = p.q;
        j.ldq = qd;
        j.oh = p.xh; j.om = p.xm; j.ol = p.xl;
        j.ldo = p.ldx;
        j.layer = l;
        j.qscale = p.qscale;
        j.t0 = tl[0]; j.nrows = tl[1]; j.slot = tl[2]; j.p0 = tl[3]; j.h = t.b;
        // fresh barriers for every attention task: the previous task's last
        // commit (`fin`) has arrived once its products retired, so no
        // arrival is pending when they are initialised again
        if (threadIdx.x == 0) {
          if (fa_calls > 0 && !pf_wait(p, s, &s.fab.fin, 0, -50))
            *(volatile int32_t*)&s.abort_flag = 1;
          fa_init_barriers(s.fab);
          fence_barrier_init();
        }
        __syncthreads();
        bool ok;
        if (m.head_dim == 128) ok = fa_tile<128>(m, j, fab_buf, s.fab, s.tmem, 0u, fwait);
        else ok = fa_tile<64>(m, j, fab_buf, s.fab, s.tmem, 0u, fwait);
        if (!ok) *(volatile int32_t*)&s.abort_flag = 1;
        fa_calls += 1;
        break;
      }
      case PF_RES1:
        pf_residual_norm(p, s, e0, e1, true, m.ffn_norm + (size_t)l * H);
        break;
      case PF_RES2:
        // the next layer's attention norm, after the last layer the final norm
        // (the LM head's input)
        pf_residual_norm(p, s, e0, e1, true,
                         l + 1 < L ? m.attn_norm + (size_t)(l + 1) * H : m.final_norm);
        break;
      case PF_SWIGLU: {
        // rows [e0, e1): gate/up interleaved in y, two outputs per thread and step
        const int F2 = F >> 1;
        for (int i = threadIdx.x; i < (e1 - e0) * F2; i += kPfThreads) {
          const int tt = e0 + i / F2, j = 2 * (i - (i / F2) * F2);
          const float4 gu = __ldcg(reinterpret_cast<const float4*>(p.y + (size_t)tt * p.ldy + 2 * j));
          const size_t o = (size_t)tt * p.ldx + j;
          pf_split3(gu.x / (1.0f + expf(-gu.x)) * gu.y, p.xh, p.xm, p.xl, o);
          pf_split3(gu.z / (1.0f + expf(-gu.z)) * gu.w, p.xh, p.xm, p.xl, o + 1);
        }
        break;
      }
      default:
        break;
    }
    __syncthreads();
    if (threadIdx.x == 0 && t.n_sig > 0) {
      fence_acq_rel_gpu();
      for (int e = 0; e < t.n_sig; ++e) red_relaxed_gpu_add(p.events + t.sig_ev0 + e, 1u);
    }
    if (threadIdx.x == 0 && p.trace && ti < p.trace_cap) {
      uint64_t* tr = p.trace + 4 * (size_t)ti;
      tr[0] = tw0;
      tr[1] = tw1;
      tr[2] = globaltimer_ns();
      tr[3] = (uint64_t)blockIdx.x | ((uint64_t)(t.kind & 15) << 16) |
              ((uint64_t)((t.kind == PF_GEMM ? t.a : 0) & 15) << 20) | ((uint64_t)(t.layer & 255) << 24) |
              ((uint64_t)(t.n & 0xFFFF) << 32) | ((uint64_t)(t.b & 0xFFFF) << 48);
    }
  }
  tc_fence_before_sync();
  __syncthreads();
  if (*(volatile int32_t*)&s.abort_flag && threadIdx.x == 0) {
    // stopped inside a GEMM tile: let the loads still in flight land (each
    // stage's last armed position) and the issued MMAs retire before exit
    for (int i = 0; i < kPfStages; ++i)
      if (s.armed[i] != 0xffffffffu) pf_drain(&s.full[i], (s.armed[i] / kPfStages) & 1);
    if (!s.tmem_ok && gs.tiles > 0 && pf_drain(&s.done, (gs.tiles - 1) & 1)) s.tmem_ok = 1;
    // the attention tasks' loads and MMAs
    for (int i = 0; i < 2; ++i) {
      if (s.fab.armed_k[i] != 0xffffffffu) pf_drain(&s.fab.k_full[i], (s.fab.armed_k[i] >> 1) & 1);
      if (s.fab.armed_v[i] != 0xffffffffu) pf_drain(&s.fab.v_full[i], (s.fab.armed_v[i] >> 1) & 1);
    }
    if (fa_calls > 0 && !pf_drain(&s.fab.fin, 0)) s.tmem_ok = 0;  // re-initialised per task
  }
  tc_fence_before_sync();
  __syncthreads();
  tc_fence_after_sync();
  // tensor memory is released once every MMA retired; otherwise the error word
  // is set and the columns stay allocated rather than be handed out while MMAs
  // may still write them
  if (warp == 0 && s.tmem_ok) tmem_dealloc(s.tmem, kPfTmemCols);
}

}  // namespace

// ------------------------------------------------------------------ host side

namespace {

// Greedy ids from the argmax keys of the requests whose last position the
// kernel handled (mask bit r).
__global__ void pf_ids_kernel(const unsigned long long* keys, int32_t* ids, uint32_t mask, int n) {
  const int r = threadIdx.x;
  if (r < n && ((mask >> r) & 1u)) ids[r] = (int32_t)(0xffffffffu - (uint32_t)(keys[r] & 0xffffffffull));
}

bool pf_make_map(CUtensorMap* map, const void* base, int rows, int cols, size_t row_stride_elems) {
  auto fn = prefill_encode_fn();
  if (!fn) return false;
  const cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
  const cuuint64_t strides[1] = {(cuuint64_t)row_stride_elems * 2};
  const cuuint32_t box[2] = {(cuuint32_t)kPfK, (cuuint32_t)kPfRows};
  const cuuint32_t estr[2] = {1u, 1u};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box,
            estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

struct PfGraph {
  std::vector<PfTask> tasks;
  std::vector<int32_t> queue, queue_off;
  int n_events = 0;
};

// The task graph of one block (T tokens, attention tiles as built for it) on P
// CTAs.  Events per (layer, stage, token tile); a task's wait count is the
// number of producer tasks it needs.
void pf_build(const ModelDev& m, int T, const std::vector<int32_t>& attn_tiles,
              const std::vector<int32_t>& lm_req, int P, PfGraph& g) {
  const int L = m.n_layers, H = m.hidden, F = m.ffn, nq = m.n_q;
  const int qkvR = qkv_rows(m.n_q, m.n_kv, m.head_dim);
  const int NT = (T + kPfTokTile - 1) / kPfTokTile;
  const int mt_qkv = (qkvR + kPfRows - 1) / kPfRows, mt_h = (H + kPfRows - 1) / kPfRows;
  const int mt_gu = (2 * F + kPfRows - 1) / kPfRows;
  // event index: ((l * kStages + stage) * NT + n)
  enum { E_NORM, E_QKV, E_ROPE, E_ATTN, E_O, E_RES1, E_GU, E_SW, E_DN, kStages };
  auto ev = [&](int l, int st, int n) { return (l * kStages + st) * NT + n; };
  g.n_events = (L + 1) * kStages * NT;
  std::vector<int> attn_per_tile(NT, 0);
  const int n_attn = (int)attn_tiles.size() / 4;
  for (int a = 0; a < n_attn; ++a) attn_per_tile[attn_tiles[4 * a] / kPfTokTile] += 1;
  std::vector<int> attn_order(n_attn);
  for (int a = 0; a < n_attn; ++a) attn_order[a] = a;
  std::stable_sort(attn_order.begin(), attn_order.end(), [&](int x, int y) {
    return attn_tiles[4 * x + 1] + attn_tiles[4 * x + 3] > attn_tiles[4 * y + 1] + attn_tiles[4 * y + 3];
  });
  g.tasks.clear();
  auto add = [&](int kind, int l, int n, int a, int b, int wait_ev, int wait_count, int sig0,
                 int nsig) {
    PfTask t{};
    t.kind = kind; t.layer = l; t.n = n; t.a = a; t.b = b;
    t.wait_ev = wait_ev; t.wait_count = (uint32_t)wait_count; t.sig_ev0 = sig0; t.n_sig = nsig;
    g.tasks.push_back(t);
  };
  for (int l = 0; l < L; ++l) {
    // elementwise stages: kPfEwSub tasks of kPfEwTok positions per token tile
    if (l == 0)
      for (int n = 0; n < NT; ++n)
        for (int b = 0; b < kPfEwSub; ++b) add(PF_NORM, 0, n, 0, b, -1, 0, ev(0, E_NORM, n), 1);
    for (int n = 0; n < NT; ++n)
      for (int mt = 0; mt < mt_qkv; ++mt)
        add(PF_GEMM, l, n, PF_QKV, mt, ev(l, E_NORM, n), kPfEwSub, ev(l, E_QKV, n), 1);
    // RoPE of tile n counts toward every later tile's "keys ready" event
    for (int n = 0; n < NT; ++n)
      for (int b = 0; b < kPfEwSub; ++b)
        add(PF_ROPE, l, n, 0, b, ev(l, E_QKV, n), mt_qkv, ev(l, E_ROPE, n), NT - n);
    // per (run, query head); the runs with the most keys first (every task of
    // the stage depends only on earlier stages, so any order is topological)
    for (int a : attn_order) {
      const int n = attn_tiles[4 * a] / kPfTokTile;
      for (int h = 0; h < nq; ++h)
        add(PF_ATTN, l, n, a, h, ev(l, E_ROPE, n), kPfEwSub * (n + 1), ev(l, E_ATTN, n), 1);
    }
    for (int n = 0; n < NT; ++n)
      for (int mt = 0; mt < mt_h; ++mt)
        add(PF_GEMM, l, n, PF_O, mt, ev(l, E_ATTN, n), attn_per_tile[n] * nq, ev(l, E_O, n), 1);
    for (int n = 0; n < NT; ++n)
      for (int b = 0; b < kPfEwSub; ++b)
        add(PF_RES1, l, n, 0, b, ev(l, E_O, n), mt_h, ev(l, E_RES1, n), 1);
    for (int n = 0; n < NT; ++n)
      for (int mt = 0; mt < mt_gu; ++mt)
        add(PF_GEMM, l, n, PF_GU, mt, ev(l, E_RES1, n), kPfEwSub, ev(l, E_GU, n), 1);
    for (int n = 0; n < NT; ++n)
      for (int b = 0; b < kPfEwSub; ++b)
        add(PF_SWIGLU, l, n, 0, b, ev(l, E_GU, n), mt_gu, ev(l, E_SW, n), 1);
    for (int n = 0; n < NT; ++n)
      for (int mt = 0; mt < mt_h; ++mt)
        add(PF_GEMM, l, n, PF_DN, mt, ev(l, E_SW, n), kPfEwSub, ev(l, E_DN, n), 1);
    // the residual, then the next layer's attention norm: its E_NORM event
    for (int n = 0; n < NT; ++n)
      for (int b = 0; b < kPfEwSub; ++b)
        add(PF_RES2, l, n, 0, b, ev(l, E_DN, n), mt_h, ev(l + 1, E_NORM, n), 1);
  }
  // the LM head for the tiles holding a prompt's last position: 128 vocabulary
  // rows per task, after the tile's final norm (the last layer's RES2)
  const int mt_lm = (m.vocab + kPfRows - 1) / kPfRows;
  for (int n = 0; n < NT; ++n) {
    bool any = false;
    for (int t = n * kPfTokTile; t < std::min(T, (n + 1) * kPfTokTile); ++t) any = any || lm_req[t] >= 0;
    if (!any) continue;
    for (int mt = 0; mt < mt_lm; ++mt) add(PF_GEMM, L, n, PF_LM, mt, ev(L, E_NORM, n), kPfEwSub, -1, 0);
  }
  // queues: the tasks in this (topological) order, dealt round-robin
  std::vector<std::vector<int32_t>> per(P);
  for (size_t i = 0; i < g.tasks.size(); ++i) per[i % P].push_back((int32_t)i);
  g.queue.clear();
  g.queue_off.assign(P + 1, 0);
  for (int c = 0; c < P; ++c) {
    g.queue_off[c] = (int32_t)g.queue.size();
    g.queue.insert(g.queue.end(), per[c].begin(), per[c].end());
  }
  g.queue_off[P] = (int32_t)g.queue.size();
}

template <class T>
std::string pf_grow(T** p, size_t* cap, size_t need, std::vector<void*>* owned) {
  if (*cap >= need) return "";
  void* v = nullptr;
  if (cudaMalloc(&v, need) != cudaSuccess) return "prefill megakernel scratch: cudaMalloc";
  owned->push_back(v);  // freed with the context
  *p = static_cast<T*>(v);
  *cap = need;
  return "";
}

// The positions of one prefill call in the order the kernel takes them: every
// position but each prompt's last, as (request, position) in request order;
// then as many last positions (with the LM head and greedy id) as the final
// block's last 128-position tile has room for: there they cost next to
// nothing, while a tile or block of their own would cost more than the
// decode steps the rest get (a tile's GEMMs take ~50 us each whatever the
// number of positions in it, a one-tile block ~12 ms for the 8B shape).
struct PfLayout {
  std::vector<int> tok_src, slot, pos, lmr;  // per position: token index, KV slot, position, request or -1
  bool folded[kMaxBatch] = {};               // the request's last position is among them
};

void pf_layout(const int32_t* offsets_host, const int32_t* slots_host, int n_req, int max_tokens,
               PfLayout* lay) {
  for (int r = 0; r < n_req; ++r)
    for (int p = 0; p + 1 < offsets_host[r + 1] - offsets_host[r]; ++p) {
      lay->tok_src.push_back(offsets_host[r] + p);
      lay->slot.push_back(slots_host[r]);
      lay->pos.push_back(p);
      lay->lmr.push_back(-1);
    }
  if (lay->tok_src.empty()) return;
  const int tn = (int)lay->tok_src.size();
  const int t_final = tn - ((tn - 1) / max_tokens) * max_tokens;  // positions of the final block
  int room = std::min((t_final + kPfTokTile - 1) / kPfTokTile * kPfTokTile, max_tokens) - t_final;
  for (int r = 0; r < n_req && room > 0; ++r) {
    const int len = offsets_host[r + 1] - offsets_host[r];
    if (len < 2) continue;  // a one-position prompt is left to the decode step
    lay->folded[r] = true;
    lay->tok_src.push_back(offsets_host[r] + len - 1);
    lay->slot.push_back(slots_host[r]);
    lay->pos.push_back(len - 1);
    lay->lmr.push_back(r);
    --room;
  }
}

// Attention runs of the block of positions [b0, b0 + T): the positions of one
// request inside one token tile, as (first block position, count, KV slot,
// first position).
void pf_runs(const PfLayout& lay, int b0, int T, std::vector<int32_t>* tiles) {
  for (int t = 0; t < T;) {
    int n = 1;
    while (t + n < T && lay.slot[b0 + t + n] == lay.slot[b0 + t] && (t + n) % kPfTokTile != 0) ++n;
    tiles->insert(tiles->end(), {t, n, lay.slot[b0 + t], lay.pos[b0 + t]});
    t += n;
  }
}

}  // namespace

size_t prefill_mk_smem_bytes() { return sizeof(PfSmem) + 1024; }

std::string prefill_mk_run(const ModelDev& m, const PrefillWeights& w, PrefillScratch& sc,
                           cudaStream_t st, const int32_t* tokens_dev, const int32_t* offsets_host,
                           const int32_t* slots_host, int n_req, int num_sms,
                           std::vector<void*>* owned, bool* timed_out, PfOutputs* out) {
  *timed_out = false;
  for (int r = 0; r < n_req; ++r) out->folded[r] = false;
  const int H = m.hidden, F = m.ffn, d = m.head_dim, qd = m.n_q * d, L = m.n_layers;
  const int qkvR = qkv_rows(m.n_q, m.n_kv, d);
  const int ldy = std::max(std::max(qkvR, 2 * F), H);
  const int ldx = std::max(std::max(H, F), qd);
  PfBuffers& b = sc.pf;
  if (!b.configured) {
    if (cudaFuncSetAttribute(prefill_mk_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)prefill_mk_smem_bytes()) != cudaSuccess)
      return "prefill megakernel: shared memory attribute";
    b.configured = true;
  }
  if (!b.maps) {
    // tensor maps, written once per context: the weights of every layer, then
    // the activation parts for K = hidden, n_q d, ffn over all max_tokens rows
    // (token columns past a block's end are computed from stale rows and never
    // stored)
    std::vector<CUtensorMap> maps((size_t)4 * L + kPfMapsExtra);
    for (int l = 0; l < L; ++l) {
      if (!pf_make_map(&maps[4 * l + PF_QKV], w.qkv[l], qkvR, H, H) ||
          !pf_make_map(&maps[4 * l + PF_O], w.o[l], H, qd, qd) ||
          !pf_make_map(&maps[4 * l + PF_GU], w.gu[l], 2 * F, H, H) ||
          !pf_make_map(&maps[4 * l + PF_DN], w.dn[l], H, F, F))
        return "prefill megakernel: weight tensor map";
    }
    const uint16_t* parts[3] = {sc.xh, sc.xm, sc.xl};
    const int kdim[3] = {H, qd, F};
    for (int part = 0; part < 3; ++part)
      for (int kk = 0; kk < 3; ++kk)
        if (!pf_make_map(&maps[pf_xmap(L, part, kk)], parts[part], sc.max_tokens, kdim[kk], ldx))
          return "prefill megakernel: activation tensor map";
    // the KV cache for the attention tasks (the same maps as the standalone kernel)
    std::string fe = flash_attn_prepare(m, &sc.fa);
    if (!fe.empty()) return fe;
    maps[pf_kvmap(L, 0)] = sc.fa.k0;
    maps[pf_kvmap(L, 1)] = sc.fa.k1;
    maps[pf_kvmap(L, 2)] = sc.fa.v0;
    maps[pf_kvmap(L, 3)] = sc.fa.v1;
    if (!pf_make_map(&maps[pf_lmmap(L)], m.lm_head, m.vocab, H, H))
      return "prefill megakernel: LM head tensor map";
    std::string e0 = pf_grow(&b.maps, &b.maps_cap, maps.size() * sizeof(CUtensorMap), owned);
    if (!e0.empty()) return e0;
    if (cudaMemcpy(b.maps, maps.data(), maps.size() * sizeof(CUtensorMap), cudaMemcpyHostToDevice) != cudaSuccess)
      return "prefill megakernel: tensor map upload";
  }
  PfLayout lay;
  pf_layout(offsets_host, slots_host, n_req, sc.max_tokens, &lay);
  for (int r = 0; r < n_req; ++r) out->folded[r] = lay.folded[r];
  const int total = (int)lay.tok_src.size();
  std::string e;
  if (total > 0) {
    if (!(e = pf_grow(&b.lm_keys, &b.lm_keys_cap, (size_t)kMaxBatch * 8, owned)).empty()) return e;
    if (cudaMemsetAsync(b.lm_keys, 0, (size_t)kMaxBatch * 8, st) != cudaSuccess)
      return "prefill megakernel: key reset";
  }
  for (int b0 = 0; b0 < total; b0 += sc.max_tokens) {
    const int T = std::min(sc.max_tokens, total - b0);
    std::vector<int32_t> meta(3 * (size_t)T), tiles;
    std::vector<int32_t> lm_req(lay.lmr.begin() + b0, lay.lmr.begin() + b0 + T);
    for (int t = 0; t < T; ++t) {
      meta[t] = lay.tok_src[b0 + t];
      meta[T + t] = lay.slot[b0 + t];
      meta[2 * T + t] = lay.pos[b0 + t];
    }
    pf_runs(lay, b0, T, &tiles);
    PfGraph gr;
    pf_build(m, T, tiles, lm_req, num_sms, gr);
    if (b0 == 0 && b.stall_task >= -1) {
      // failure injection: one more completion than the event will receive
      int ti = b.stall_task;
      if (ti == -1)
        for (int i = (int)gr.tasks.size() - 1; i >= 0 && ti == -1; --i)
          if (gr.tasks[i].wait_ev >= 0) ti = i;
      if (ti < 0 || ti >= (int)gr.tasks.size() || gr.tasks[ti].wait_ev < 0)
        return "inject prefill stall: no such task waiting on an event";
      gr.tasks[ti].wait_count += 1u;
    }
    if (!(e = pf_grow(&b.tasks, &b.tasks_cap, gr.tasks.size() * sizeof(PfTask), owned)).empty() ||
        !(e = pf_grow(&b.queue, &b.queue_cap, gr.queue.size() * 4, owned)).empty() ||
        !(e = pf_grow(&b.queue_off, &b.queue_off_cap, gr.queue_off.size() * 4, owned)).empty() ||
        !(e = pf_grow(&b.events, &b.events_cap, (size_t)gr.n_events * 4, owned)).empty() ||
        !(e = pf_grow(&b.err, &b.err_cap, 16, owned)).empty())
      return e;
    int32_t* d_src = sc.meta;
    int32_t* d_slot = sc.meta + T;
    int32_t* d_pos = sc.meta + 2 * T;
    int32_t* d_tiles = sc.meta + 3 * (size_t)sc.max_tokens;
    int32_t* d_lm_req = sc.meta + 7 * (size_t)sc.max_tokens;
    if (cudaMemcpyAsync(sc.meta, meta.data(), meta.size() * 4, cudaMemcpyHostToDevice, st) != cudaSuccess ||
        cudaMemcpyAsync(d_tiles, tiles.data(), tiles.size() * 4, cudaMemcpyHostToDevice, st) != cudaSuccess ||
        cudaMemcpyAsync(d_lm_req, lm_req.data(), lm_req.size() * 4, cudaMemcpyHostToDevice, st) != cudaSuccess ||
        cudaMemcpyAsync(b.tasks, gr.tasks.data(), gr.tasks.size() * sizeof(PfTask), cudaMemcpyHostToDevice, st) != cudaSuccess ||
        cudaMemcpyAsync(b.queue, gr.queue.data(), gr.queue.size() * 4, cudaMemcpyHostToDevice, st) != cudaSuccess ||
        cudaMemcpyAsync(b.queue_off, gr.queue_off.data(), gr.queue_off.size() * 4, cudaMemcpyHostToDevice, st) != cudaSuccess ||
        cudaMemsetAsync(b.events, 0, (size_t)gr.n_events * 4, st) != cudaSuccess ||
        cudaMemsetAsync(b.err, 0, 16, st) != cudaSuccess)
      return "prefill megakernel: upload";
    PfArgs a{};
    a.m = m;
    a.tasks = reinterpret_cast<const PfTask*>(b.tasks);
    a.queue = b.queue;
    a.queue_off = b.queue_off;
    a.maps = reinterpret_cast<const CUtensorMap*>(b.maps);
    a.events = b.events;
    a.err = b.err;
    a.tokens = tokens_dev;
    a.tok_src = d_src;
    a.slot = d_slot;
    a.pos = d_pos;
    a.attn_tiles = d_tiles;
    a.x = sc.x; a.y = sc.y; a.q = sc.q;
    a.xh = sc.xh; a.xm = sc.xm; a.xl = sc.xl;
    a.T = T; a.ldy = ldy; a.ldx = ldx;
    a.qscale = m.attn_scale * 1.4426950408889634f;
    a.trace = b0 == 0 ? b.trace : nullptr;
    a.wait_ns = 2ull * (uint64_t)(m.timeout_ms > 0 ? m.timeout_ms : 1000) * 1000000ull;
    a.lm_req = d_lm_req;
    a.lm_keys = b.lm_keys;
    a.logits = out->logits;
    a.trace_cap = b.trace_cap;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(num_sms);
    cfg.blockDim = dim3(kPfThreads);
    cfg.dynamicSmemBytes = prefill_mk_smem_bytes();
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeCooperative;
    attr[0].val.cooperative = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    const cudaError_t le = cudaLaunchKernelEx(&cfg, prefill_mk_kernel, a);
    if (le != cudaSuccess) return std::string("prefill megakernel launch: ") + cudaGetErrorString(le);
    // the host vectors above are staged by the (pageable) copies before they return
    int32_t herr[2] = {0, 0};
    if (cudaMemcpyAsync(herr, b.err, 8, cudaMemcpyDeviceToHost, st) != cudaSuccess ||
        cudaStreamSynchronize(st) != cudaSuccess)
      return std::string("prefill megakernel: ") + cudaGetErrorString(cudaGetLastError());
    if (herr[0]) {
      *timed_out = herr[0] == MK_ERR_TIMEOUT;
      return "prefill megakernel: a wait timed out (detail " + std::to_string(herr[1]) + ")";
    }
    // the last positions' residual streams (the hidden state after the prompt)
    for (int t = 0; t < T; ++t) {
      const int r = lm_req[t];
      if (r >= 0 && out->hidden[r] &&
          cudaMemcpyAsync(out->hidden[r], sc.x + (size_t)t * H, (size_t)H * 4, cudaMemcpyDeviceToDevice,
                          st) != cudaSuccess)
        return "prefill megakernel: hidden state copy";
    }
  }
  if (total > 0 && out->ids) {
    uint32_t mask = 0;
    for (int r = 0; r < n_req; ++r) mask |= out->folded[r] ? 1u << r : 0u;
    pf_ids_kernel<<<1, 32, 0, st>>>(b.lm_keys, out->ids, mask, n_req);
    if (cudaGetLastError() != cudaSuccess) return "prefill megakernel: greedy id launch";
  }
  return "";
}

}  // namespace mk

extern "C" int mk_prefill_graph(const mk_config* cfg, int T, const int32_t* tiles_host, int n_tiles,
                                const int32_t* lm_req_host, int num_ctas, int32_t* tasks_out,
                                int cap_tasks, int32_t* queue_off_out, int32_t* queue_out,
                                int cap_queue, int* n_tasks, int* n_events) {
  if (!cfg || T <= 0 || !tiles_host || n_tiles <= 0 || !lm_req_host || num_ctas <= 0 ||
      !n_tasks || !n_events || !mk::validate_config(*cfg).empty())
    return MK_ERR_INVALID_ARG;
  for (int a = 0; a < n_tiles; ++a) {
    const int32_t* t = tiles_host + 4 * a;
    if (t[0] < 0 || t[1] < 1 || t[0] + t[1] > T || t[0] / 128 != (t[0] + t[1] - 1) / 128)
      return MK_ERR_INVALID_ARG;
  }
  mk::ModelDev m{};  // sizes only: the graph depends on nothing else
  m.n_layers = cfg->n_layers;
  m.hidden = cfg->hidden;
  m.ffn = cfg->ffn;
  m.n_q = cfg->n_q_heads;
  m.n_kv = cfg->n_kv_heads;
  m.head_dim = cfg->head_dim;
  m.group = cfg->n_q_heads / cfg->n_kv_heads;
  m.vocab = cfg->vocab;
  const std::vector<int32_t> tiles(tiles_host, tiles_host + 4 * (size_t)n_tiles);
  const std::vector<int32_t> lm(lm_req_host, lm_req_host + T);
  mk::PfGraph g;
  mk::pf_build(m, T, tiles, lm, num_ctas, g);
  *n_tasks = (int)g.tasks.size();
  *n_events = g.n_events;
  for (int i = 0; tasks_out && i < std::min(cap_tasks, *n_tasks); ++i) {
    const mk::PfTask& t = g.tasks[i];
    const int32_t v[9] = {t.kind, t.layer, t.n, t.a, t.b, t.wait_ev, (int32_t)t.wait_count,
                          t.sig_ev0, t.n_sig};
    for (int k = 0; k < 9; ++k) tasks_out[9 * (size_t)i + k] = v[k];
  }
  if (queue_off_out)
    for (int c = 0; c <= num_ctas; ++c) queue_off_out[c] = g.queue_off[c];
  for (int i = 0; queue_out && i < std::min(cap_queue, (int)g.queue.size()); ++i) queue_out[i] = g.queue[i];
  return MK_OK;
}

extern "C" int mk_prefill_layout(const int32_t* offsets_host, const int32_t* slots_host, int n_req,
                                 int max_tokens, int32_t* positions_out, int cap_positions,
                                 int32_t* runs_out, int cap_runs, int* n_positions, int* n_runs,
                                 int32_t* folded_out) {
  if (!offsets_host || !slots_host || n_req < 1 || n_req > mk::kMaxBatch || max_tokens < 1 ||
      !n_positions || !n_runs || offsets_host[0] < 0)
    return MK_ERR_INVALID_ARG;
  for (int r = 0; r < n_req; ++r)
    if (offsets_host[r + 1] < offsets_host[r]) return MK_ERR_INVALID_ARG;
  mk::PfLayout lay;
  mk::pf_layout(offsets_host, slots_host, n_req, max_tokens, &lay);
  const int total = (int)lay.tok_src.size();
  std::vector<int32_t> runs;
  for (int b0 = 0; b0 < total; b0 += max_tokens) {
    std::vector<int32_t> tiles;
    mk::pf_runs(lay, b0, std::min(max_tokens, total - b0), &tiles);
    for (size_t i = 0; i < tiles.size(); i += 4)
      runs.insert(runs.end(), {b0 / max_tokens, tiles[i], tiles[i + 1], tiles[i + 2], tiles[i + 3]});
  }
  *n_positions = total;
  *n_runs = (int)(runs.size() / 5);
  for (int t = 0; positions_out && t < std::min(cap_positions, total); ++t) {
    positions_out[4 * (size_t)t] = lay.tok_src[t];
    positions_out[4 * (size_t)t + 1] = lay.slot[t];
    positions_out[4 * (size_t)t + 2] = lay.pos[t];
    positions_out[4 * (size_t)t + 3] = lay.lmr[t];
  }
  for (int i = 0; runs_out && i < std::min(cap_runs, *n_runs); ++i)
    for (int k = 0; k < 5; ++k) runs_out[5 * (size_t)i + k] = runs[5 * (size_t)i + k];
  for (int r = 0; folded_out && r < n_req; ++r) folded_out[r] = lay.folded[r] ? 1 : 0;
  return MK_OK;
}
