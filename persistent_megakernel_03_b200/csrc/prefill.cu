// prefill.cu -- prompt prefill with the weight contractions on the tensor
// cores ("LLM高速化勉強会資料" slide 9: prefill processes the prompt's tokens
// together; "Crear desde cero ..." §4: tensor cores for the dense products).
//
// Per block of up to max_tokens prompt positions (any mix of requests) and per
// layer:
//   x -> RMSNorm -> [xh, xl] -> GEMM(W_qkv) (+bias) -> RoPE, K/V into the cache
//     -> causal GQA attention over the cache -> [xh, xl] -> GEMM(W_o) -> x +=
//   x -> RMSNorm -> [xh, xl] -> GEMM(W_gate/up) -> SwiGLU -> [xh, xl]
//     -> GEMM(W_down) -> x +=
// The GEMM computes Y[t][r] = sum_k W[r][k] * (xh[t][k] + xm[t][k] + xl[t][k]):
// the fp32 activation is split into three bf16 parts xh = bf16(x),
// xm = bf16(x - xh), xl = bf16(x - xh - xm) (each difference exact), 24
// significand bits in all, so three bf16 tcgen05.mma per K step reproduce the
// fp32 product to fp32 precision (a two-part split keeps only ~2^-16, which at
// full depth visibly moves the logits).
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <algorithm>
#include <array>
#include <cmath>
#include <string>
#include <vector>

#include "../../include/mk.h"
#include "attn_math.cuh"
#include "mk_internal.h"
#include "prefill.h"
#include "ptx.cuh"
#include "tc.cuh"

namespace mk {

namespace {

__device__ __forceinline__ uint16_t bf16_bits(float f) {
  __nv_bfloat16 b = __float2bfloat16_rn(f);
  return *reinterpret_cast<uint16_t*>(&b);
}
__device__ __forceinline__ float bf16_val(uint16_t h) { return __uint_as_float((uint32_t)h << 16); }

// v -> (bf16(v), bf16(v - bf16(v))): the batched decode step's two parts
__device__ __forceinline__ void split_store(float v, uint16_t* hi, uint16_t* lo, size_t i) {
  const uint16_t h = bf16_bits(v);
  hi[i] = h;
  lo[i] = bf16_bits(v - bf16_val(h));
}

// v -> (h, m, l) = (bf16(v), bf16(v - h), bf16(v - h - m)): the prompt GEMMs'
// three parts (both differences are exact in fp32)
__device__ __forceinline__ void split3_store(float v, uint16_t* hi, uint16_t* mid, uint16_t* lo,
                                             size_t i) {
  const uint16_t h = bf16_bits(v);
  const float r1 = v - bf16_val(h);
  const uint16_t m = bf16_bits(r1);
  hi[i] = h;
  mid[i] = m;
  lo[i] = bf16_bits(r1 - bf16_val(m));
}

// ------------------------------------------------------------------ GEMM
// Y[t][r] = sum_k W[r][k] * (xh[t][k] + xl[t][k]) for 128 weight rows and BN
// tokens per CTA, K blocks [z*nk/Z, (z+1)*nk/Z) of a Z-way split (gridDim.z;
// split z writes its partial sums at Y + z * part_stride).  Warp 0 lane 0
// issues the TMA loads of a STAGES-deep ring (W tile 128 x 64, xh and xl
// tiles BN x 64, all 128-byte swizzled), warp 1 lane 0 issues the MMAs into a
// 128 x BN fp32 accumulator in tensor memory and frees each stage with
// tcgen05.commit, and all four warps read the accumulator back (warp w owns
// TMEM lanes 32w..32w+31, i.e. weight rows) and store Y[token][row].
// BN = 128 serves the prompt (many tokens); BN = 16 serves a decode step of
// up to 8 requests, where the weights dominate and the deeper ring keeps more
// of them in flight.
constexpr int kGM = 128, kGK = 64;
constexpr int kGTileA = kGM * kGK * 2;  // 16 KB
constexpr uint64_t kGWaitNs = 2000000000ull;  // 2 s: far beyond any legal wait

// HL: the B operand is one BN-row tile whose first BN/2 rows are the high
// parts and the last BN/2 rows the low parts of the same BN/2 tokens (a
// decode step of up to 8 requests): one MMA per K step, and the epilogue adds
// accumulator columns j and j + BN/2.
template <int BN, int STAGES, bool HL = false>
struct __align__(1024) GemmSmem {
  static constexpr int kTileB = BN * kGK * 2;
  static constexpr int kBTiles = HL ? 1 : 3;
  static constexpr uint32_t kStageBytes = kGTileA + kBTiles * kTileB;
  // accumulators: one (HL), or three -- the high part's even and odd K blocks
  // and the middle + low parts -- so no single fp32 accumulator takes every
  // MMA of the contraction; the epilogue adds them
  static constexpr int kAcc = HL ? 1 : 3;
  static constexpr uint32_t kTmemCols = kAcc * BN <= 32 ? 32 : kAcc * BN <= 64 ? 64
                                      : kAcc * BN <= 128 ? 128 : kAcc * BN <= 256 ? 256 : 512;
  uint8_t a[STAGES][kGTileA];
  uint8_t bh[STAGES][kTileB];
  uint8_t bm[HL ? 1 : STAGES][HL ? 16 : kTileB];
  uint8_t bl[HL ? 1 : STAGES][HL ? 16 : kTileB];
  uint64_t full[STAGES];
  uint64_t empty[STAGES];
  uint64_t done;
  uint32_t tmem;
  int32_t failed;
};
template <int BN, int STAGES, bool HL = false>
constexpr size_t gemm_smem_bytes() { return sizeof(GemmSmem<BN, STAGES, HL>) + 1024; }

// Bounded wait on an mbarrier phase; false after kGWaitNs (the caller records
// the failure and stops issuing work).
__device__ __forceinline__ bool gemm_wait(uint64_t* bar, uint32_t parity) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = globaltimer_ns();
  while (!mbar_try_wait(bar, parity))
    if (globaltimer_ns() - t0 > kGWaitNs) return false;
  return true;
}

template <int BN, int STAGES, bool HL = false>
__global__ void __launch_bounds__(128, 1)
    gemm_wx_kernel(const __grid_constant__ CUtensorMap tm_w, const __grid_constant__ CUtensorMap tm_xh,
                   const __grid_constant__ CUtensorMap tm_xm, const __grid_constant__ CUtensorMap tm_xl,
                   int n_rows, int n_tok, int K,
                   float* __restrict__ Y, int ldy, size_t part_stride,
                   const uint16_t* __restrict__ bias, int32_t* __restrict__ err,
                   const float* __restrict__ tok_ss, int norm_len, float norm_eps,
                   uint16_t* __restrict__ act_hl, int act_ld) {
  using S = GemmSmem<BN, STAGES, HL>;
  // The swizzled tiles must start on 1024-byte boundaries of the shared
  // window: round the dynamic base up (the launch adds 1 KB of slack).
  extern __shared__ __align__(16) uint8_t gsm_raw[];
  const uint32_t base = smem_u32(gsm_raw);
  S& s = *reinterpret_cast<S*>(gsm_raw + (((base + 1023u) & ~1023u) - base));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int m0 = blockIdx.x * kGM, n0 = blockIdx.y * BN;
  const int nk_all = K / kGK, Z = gridDim.z, z = blockIdx.z;
  const int kb0 = (int)((long long)nk_all * z / Z), kb1 = (int)((long long)nk_all * (z + 1) / Z);
  const int nk = kb1 - kb0;
  Y += (size_t)z * part_stride;
  if (threadIdx.x == 0) {
    for (int i = 0; i < STAGES; ++i) {
      mbar_init(&s.full[i], 1);
      mbar_init(&s.empty[i], 1);
    }
    mbar_init(&s.done, 1);
    s.failed = 0;
    fence_barrier_init();
  }
  if (warp == 0) {
    tmem_alloc(&s.tmem, S::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before_sync();
  __syncthreads();
  tc_fence_after_sync();
  const uint32_t tmem = s.tmem;
  pdl_trigger();
  // TMA loads issued by one thread run one after another, so two producer
  // threads (lane 0 of warps 0 and 2) issue the stages past the first ring's
  // worth alternately; warp 0 alone issues the first STAGES stages.
  const int pre = nk < STAGES ? nk : STAGES;
  if ((warp == 0 || warp == 2) && lane == 0) {
    const int pid = warp >> 1;
    if (pid == 0) {
      // The weight tiles of the first STAGES stages do not depend on the
      // previous kernel: they are requested before waiting for it.
      for (int i = 0; i < pre; ++i) {
        mbar_arrive_expect_tx(&s.full[i], S::kStageBytes);
        tma_load_2d(s.a[i], &tm_w, (kb0 + i) * kGK, m0, &s.full[i]);
      }
    }
    pdl_wait();
    if (pid == 0) {
      for (int i = 0; i < pre; ++i) {
        tma_load_2d(s.bh[i], &tm_xh, (kb0 + i) * kGK, n0, &s.full[i]);
        if constexpr (!HL) {
          tma_load_2d(s.bm[i], &tm_xm, (kb0 + i) * kGK, n0, &s.full[i]);
          tma_load_2d(s.bl[i], &tm_xl, (kb0 + i) * kGK, n0, &s.full[i]);
        }
      }
    }
    int issued = pid == 0 ? pre : 0;  // one past this producer's last issued stage
    for (int i = pre + pid; i < nk; i += 2) {
      const int st = i % STAGES;
      if (!gemm_wait(&s.empty[st], ((i / STAGES) - 1) & 1)) {
        s.failed = 1;
        break;
      }
      const int kc = (kb0 + i) * kGK;
      mbar_arrive_expect_tx(&s.full[st], S::kStageBytes);
      tma_load_2d(s.a[st], &tm_w, kc, m0, &s.full[st]);
      tma_load_2d(s.bh[st], &tm_xh, kc, n0, &s.full[st]);
      if constexpr (!HL) {
        tma_load_2d(s.bm[st], &tm_xm, kc, n0, &s.full[st]);
        tma_load_2d(s.bl[st], &tm_xl, kc, n0, &s.full[st]);
      }
      issued = i + 1;
    }
    // every load this thread issued must land before the CTA may exit (the
    // last STAGES stages are the only ones that can still be in flight)
    for (int i = (issued > STAGES ? issued - STAGES : 0); i < issued; ++i) {
      const bool mine = i < pre ? pid == 0 : ((i - pre) & 1) == pid;
      if (mine) gemm_wait(&s.full[i % STAGES], (i / STAGES) & 1);
    }
  } else if (warp == 1 && lane == 0) {
    constexpr uint32_t idesc = mma_idesc_bf16_f32(kGM, BN);
    for (int i = 0; i < nk; ++i) {
      const int st = i % STAGES;
      if (!gemm_wait(&s.full[st], (i / STAGES) & 1)) {
        s.failed = 1;
        break;
      }
      tc_fence_after_sync();
      const uint64_t da = sw128_kmajor_desc(s.a[st]);
      const uint64_t dh = sw128_kmajor_desc(s.bh[st]);
#pragma unroll
      for (int k = 0; k < kGK / 16; ++k) {
        // +2 in the address field = 32 bytes = 16 bf16 along K
        if constexpr (HL) {
          tc_mma_f16(tmem, da + 2 * k, dh + 2 * k, idesc, (i | k) != 0);
        } else {
          const uint32_t acc_h = tmem + ((i & 1) ? 2u * BN : 0u);
          const uint32_t acc_ml = tmem + (uint32_t)BN;
          tc_mma_f16(acc_h, da + 2 * k, dh + 2 * k, idesc, (i > 1 || k > 0) ? 1u : 0u);
          tc_mma_f16(acc_ml, da + 2 * k, sw128_kmajor_desc(s.bm[st]) + 2 * k, idesc, (i | k) != 0);
          tc_mma_f16(acc_ml, da + 2 * k, sw128_kmajor_desc(s.bl[st]) + 2 * k, idesc, 1u);
        }
      }
      tc_commit(&s.empty[st]);
    }
    tc_commit(&s.done);  // also when stopped early: retires what was issued
  }
  __syncwarp();
  // Accumulator ready (or the issuing stopped): every warp waits on `done`.
  // The issuing thread commits `done` on every path, at the latest when its
  // own bounded waits gave up, so one more bounded wait covers that case.
  bool ok = gemm_wait(&s.done, 0);
  if (!ok) ok = gemm_wait(&s.done, 0);
  tc_fence_after_sync();
  pdl_wait();  // (returned long ago in the producer) before writing Y
  __syncthreads();
  if (ok && !s.failed && nk > 0) {
    const int row = m0 + warp * 32 + lane;
    const float b = (bias && row < n_rows) ? __uint_as_float((uint32_t)bias[row] << 16) : 0.f;
    if constexpr (HL) {
      float v[16];
      tmem_ld16(tmem + ((uint32_t)(warp * 32) << 16), v);
      if (act_hl) {
        // gate/up rows 2j, 2j+1 sit in adjacent lanes: the even lane forms
        // silu(gate) * up and writes it as the next GEMM's split input
#pragma unroll
        for (int j = 0; j < BN / 2; ++j) {
          const bool live = row < n_rows && j < n_tok;
          const float sc = (live && tok_ss) ? 1.0f / sqrtf(tok_ss[j] / (float)norm_len + norm_eps) : 1.0f;
          const float yv = live ? (v[j] + v[j + BN / 2]) * sc + b : 0.f;
          const float up = __shfl_xor_sync(0xffffffffu, yv, 1);
          if (live && !(lane & 1))
            split_store(yv / (1.0f + expf(-yv)) * up, act_hl, act_hl + (size_t)(BN / 2) * act_ld,
                        (size_t)j * act_ld + (row >> 1));
        }
      } else if (row < n_rows) {
#pragma unroll
        for (int j = 0; j < BN / 2; ++j) {
          if (j < n_tok) {
            const float sc = tok_ss ? 1.0f / sqrtf(tok_ss[j] / (float)norm_len + norm_eps) : 1.0f;
            Y[(size_t)j * ldy + row] = (v[j] + v[j + BN / 2]) * sc + b;
          }
        }
      }
    } else {
      const bool odd_blocks = nk > 1;  // the second high-part accumulator was written
#pragma unroll 1
      for (int c0 = 0; c0 < BN; c0 += 16) {
        float v[16], ml[16], v2[16];
        const uint32_t lane_base = tmem + ((uint32_t)(warp * 32) << 16) + (uint32_t)c0;
        tmem_ld16(lane_base, v);
        tmem_ld16(lane_base + (uint32_t)BN, ml);
        if (odd_blocks) tmem_ld16(lane_base + 2u * BN, v2);
#pragma unroll
        for (int j = 0; j < 16; ++j) v[j] = (v[j] + (odd_blocks ? v2[j] : 0.f)) + ml[j];
        if (row < n_rows) {
#pragma unroll
          for (int j = 0; j < 16; ++j) {
            const int tok = n0 + c0 + j;
            if (tok < n_tok) {
              // deferred RMSNorm: the input was x * w, its scale 1/rms applies here
              const float sc = tok_ss ? 1.0f / sqrtf(tok_ss[tok] / (float)norm_len + norm_eps) : 1.0f;
              Y[(size_t)tok * ldy + row] = v[j] * sc + b;
            }
          }
        }
      }
    }
  } else if (threadIdx.x == 0 && (!ok || s.failed)) {
    atomicExch(err, 1);
  }
  tc_fence_before_sync();
  __syncthreads();
  // Tensor memory is released only once every MMA of this CTA retired (the
  // `done` commit arrived); if that never happened the error word is set and
  // the columns stay allocated rather than be handed to another CTA while
  // MMAs may still write them.
  if (warp == 0 && ok) tmem_dealloc(tmem, S::kTmemCols);
}

// ------------------------------------------------------- small operators

// x[t] = E[token of t] (fp32).  meta_tok: index into tokens_dev per token.
__global__ void embed_kernel(const uint16_t* __restrict__ E, const int32_t* __restrict__ tokens,
                             const int32_t* __restrict__ tok_src, int H, int vocab,
                             float* __restrict__ x, int32_t* __restrict__ status) {
  const int t = blockIdx.x;
  int tok = tokens[tok_src[t]];
  if (tok < 0 || tok >= vocab) {  // reported like the decode step does; row 0 stands in
    if (threadIdx.x == 0 && atomicCAS(status, 0, MK_ERR_TOKEN_RANGE) == 0) status[1] = tok;
    tok = 0;
  }
  for (int i = threadIdx.x; i < H; i += blockDim.x)
    x[(size_t)t * H + i] = bf16_val(E[(size_t)tok * H + i]);
}

// [xh, xm, xl][t] = split3(x[t] * w / sqrt(mean(x[t]^2) + eps))
__global__ void rmsnorm_split_kernel(const float* __restrict__ x, const uint16_t* __restrict__ w,
                                     int H, float eps, uint16_t* __restrict__ xh,
                                     uint16_t* __restrict__ xm, uint16_t* __restrict__ xl) {
  __shared__ float red[32];
  const int t = blockIdx.x;
  const float* xr = x + (size_t)t * H;
  float ss = 0.f;
  for (int i = threadIdx.x; i < H; i += blockDim.x) ss = fmaf(xr[i], xr[i], ss);
  for (int o = 16; o; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = ss;
  __syncthreads();
  float tot = 0.f;
  for (int i = 0; i < (int)(blockDim.x >> 5); ++i) tot += red[i];
  const float r = 1.0f / sqrtf(tot / (float)H + eps);
  for (int i = threadIdx.x; i < H; i += blockDim.x)
    split3_store(xr[i] * r * bf16_val(w[i]), xh, xm, xl, (size_t)t * H + i);
}

// Sum of split-K partials p[z * pstride], z = 0 .. nparts - 1, added in split
// order (the same rounding as a plain loop) with the loads issued together.
__device__ __forceinline__ float sum_parts(const float* __restrict__ p, int nparts, size_t pstride) {
  float t[kBatchMaxSplitK];
#pragma unroll
  for (int z = 0; z < kBatchMaxSplitK; ++z) t[z] = z < nparts ? p[z * pstride] : 0.f;
  float v = 0.f;
#pragma unroll
  for (int z = 0; z < kBatchMaxSplitK; ++z)
    if (z < nparts) v += t[z];
  for (int z = kBatchMaxSplitK; z < nparts; ++z) v += p[z * pstride];
  return v;
}

// RoPE on the packed q/k rows of each token, q to qout, K/V (bf16) into the
// cache at the token's (slot, position).  Mirrors the decode step's epilogue.
__global__ void rope_kv_kernel(const float* __restrict__ y, int ldy, int nparts, size_t pstride,
                               const uint16_t* __restrict__ bias, const int32_t* __restrict__ slot,
                               const int32_t* __restrict__ pos, ModelDev m, int layer,
                               float* __restrict__ qout) {
  pdl_trigger();
  pdl_wait();
  const int t = blockIdx.x;
  const int d = m.head_dim, G = m.group, half = d >> 1;
  const int npairs = qkv_rows(m.n_q, m.n_kv, d) >> 1;
  const int p = pos[t], sl = slot[t];
  for (int pi = blockIdx.y * blockDim.x + threadIdx.x; pi < npairs; pi += blockDim.x * gridDim.y) {
    const int r = 2 * pi;
    float y0 = sum_parts(y + (size_t)t * ldy + r, nparts, pstride);
    float y1 = sum_parts(y + (size_t)t * ldy + r + 1, nparts, pstride);
    if (bias) {
      y0 += bf16_val(bias[r]);
      y1 += bf16_val(bias[r + 1]);
    }
    int which, head, dim0, w1, h1, dim1;
    qkv_source(r, G, d, &which, &head, &dim0);
    qkv_source(r + 1, G, d, &w1, &h1, &dim1);
    if (which < 2) {
      const float c = m.rope_cos[(size_t)p * half + dim0], sn = m.rope_sin[(size_t)p * half + dim0];
      const float o0 = y0 * c - y1 * sn;
      const float o1 = y0 * sn + y1 * c;
      y0 = o0;
      y1 = o1;
    }
    if (which == 0) {
      float* q = qout + (size_t)t * m.n_q * d + (size_t)head * d;
      q[dim0] = y0;
      q[dim1] = y1;
    } else {
      uint16_t* cache = which == 1 ? m.kcache : m.vcache;
      const size_t off = kv_row(m, sl, layer, head, p);
      cache[off + dim0] = bf16_bits(y0);
      cache[off + dim1] = bf16_bits(y1);
    }
  }
}

// Causal GQA attention of a tile of up to 16 consecutive positions of one
// request against its cache (keys 0..position), one warp per position, the
// keys staged in shared memory 64 rows at a time and shared by the tile's
// warps; the online-softmax update is the decode step's (attn_math.cuh).
// Writes the normalised output as the O projection's [xh, xl] input.
constexpr int kPAWarps = 16;
constexpr int kPAKeys = 64;

template <int DPL, int G>
__global__ void __launch_bounds__(kPAWarps * 32, 1)
    prefill_attn_kernel(const float* __restrict__ q, const int32_t* __restrict__ tiles, ModelDev m,
                        int layer, uint16_t* __restrict__ xh, uint16_t* __restrict__ xm,
                        uint16_t* __restrict__ xl) {
  constexpr int d = DPL * 32;
  extern __shared__ __align__(16) uint8_t pa_raw[];
  uint16_t* ks = reinterpret_cast<uint16_t*>(pa_raw);
  uint16_t* vs = ks + kPAKeys * d;
  float* xbs = reinterpret_cast<float*>(vs + kPAKeys * d);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = blockIdx.y;
  const int* tl = tiles + 4 * blockIdx.x;
  const int t0 = tl[0], nt = tl[1], sl = tl[2], p0 = tl[3];
  const int nq = m.n_q;
  const bool mine = warp < nt;
  const int p = p0 + warp;  // this warp's position
  AttnState<DPL, G> st;
  if (mine) attn_init<DPL, G>(st, q + (size_t)(t0 + warp) * nq * d + (size_t)g * G * d, d,
                              m.attn_scale, lane);
  const int n_keys = p0 + nt;  // keys 0 .. last position of the tile
  float* xb = xbs + warp * kAttnXbStride;
  for (int kb = 0; kb < n_keys; kb += kPAKeys) {
    const int nk = min(kPAKeys, n_keys - kb);
    // a block of kPAKeys keys starting at a multiple of kPAKeys lies in one
    // KV page (pages hold a multiple of 64 positions), so its rows are contiguous
    const size_t off = kv_row(m, sl, layer, g, kb);
    const uint16_t* K = m.kcache + off;
    const uint16_t* V = m.vcache + off;
    __syncthreads();
    const int vec = nk * d / 8;  // 16-byte pieces
    for (int i = threadIdx.x; i < vec; i += blockDim.x) {
      reinterpret_cast<uint4*>(ks)[i] = __ldcg(reinterpret_cast<const uint4*>(K) + i);
      reinterpret_cast<uint4*>(vs)[i] = __ldcg(reinterpret_cast<const uint4*>(V) + i);
    }
    __syncthreads();
    if (!mine) continue;
    const int lim = min(nk, p + 1 - kb);  // causal: keys <= p
    for (int j0 = 0; j0 < lim; j0 += 4) {
      const int nj = min(4, lim - j0);
      {
        float kv[4][DPL];
#pragma unroll
        for (int t = 0; t < 4; ++t) {
          const int jr = attn_key_row<G>(t, lane);
          if (jr < nj) load_kv_row<DPL>(ks + (size_t)(j0 + jr) * d + lane * DPL, kv[t]);
          else
#pragma unroll
            for (int i = 0; i < DPL; ++i) kv[t][i] = 0.f;
        }
        attn_scores4<DPL, G>(st, kv, nj, xb, lane);
      }
      float vv[4][DPL];
#pragma unroll
      for (int t = 0; t < 4; ++t) {
        if (t < nj) load_kv_row<DPL>(vs + (size_t)(j0 + t) * d + lane * DPL, vv[t]);
        else
#pragma unroll
          for (int i = 0; i < DPL; ++i) vv[t][i] = 0.f;
      }
      attn_update4<DPL, G>(st, vv, xb);
    }
  }
  if (!mine) return;
  const size_t row = (size_t)(t0 + warp) * nq * d + (size_t)g * G * d;
#pragma unroll
  for (int h = 0; h < G; ++h) {
    const float inv = 1.0f / st.l[h];
#pragma unroll
    for (int i = 0; i < DPL; ++i)
      split3_store(st.o[h][i] * inv, xh, xm, xl, row + (size_t)h * d + lane * DPL + i);
  }
}

// x[t] += y[t] (the sum of nparts split-K partials, in order)
__global__ void residual_kernel(float* __restrict__ x, const float* __restrict__ y, int H, int ldy,
                                int nparts, size_t pstride) {
  const int t = blockIdx.x;
  for (int i = threadIdx.x; i < H; i += blockDim.x) {
    x[(size_t)t * H + i] += sum_parts(y + (size_t)t * ldy + i, nparts, pstride);
  }
}

// [xh, xm, xl][t][j] = split3(silu(gate_j) * up_j); gate/up interleaved in y.
__global__ void swiglu_split_kernel(const float* __restrict__ y, int ldy, int F, int nparts,
                                    size_t pstride, uint16_t* __restrict__ xh,
                                    uint16_t* __restrict__ xm, uint16_t* __restrict__ xl) {
  const int t = blockIdx.x;
  for (int j = threadIdx.x; j < F; j += blockDim.x) {
    const float g = sum_parts(y + (size_t)t * ldy + 2 * j, nparts, pstride);
    const float u = sum_parts(y + (size_t)t * ldy + 2 * j + 1, nparts, pstride);
    split3_store(g / (1.0f + expf(-g)) * u, xh, xm, xl, (size_t)t * F + j);
  }
}

// ------------------------------------------------- batched decode step
// Split-KV decode attention for several requests at once: CTA (split s, KV
// head g, request r) runs keys [k0, k1) of the request's cache, 64 keys at a
// time through a 3-stage cp.async pipeline in shared memory (16-byte
// pieces), four keys per warp with the decode step's online-softmax update,
// then merges its 16 warps and writes one partial (output unnormalised at
// the split's maximum, the maximum, the sum).  The keys per split follow
// from the whole step's keys, so that the splits holding keys fit in about
// one wave of SMs; the rest return at once.
constexpr int kBAWarps = 16;
constexpr int kBAKeys = 64;
constexpr int kBAStages = 3;
constexpr int kBAMinKeysPerSplit = 256;

__device__ __forceinline__ void cp_async16(void* dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_u32(dst)), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

// Keys per split of this step: the step's (request, KV head) key rows spread
// over the SMs less one per (request, KV head) for rounding up, at least
// kBAMinKeysPerSplit, and enough that no request needs more than S splits.
__device__ __forceinline__ int batch_keys_per_split(const BatchParams* bp, int n_kv, int S,
                                                    int num_sms) {
  long long total = 0;
  int nmax = 1;
  for (int i = 0; i < bp->n; ++i) {
    const int k = bp->pos[i] + 1;
    total += k;
    nmax = max(nmax, k);
  }
  const int slots = max(num_sms - bp->n * n_kv, num_sms / 2);
  long long kps = (total * n_kv + slots - 1) / slots;
  kps = max(kps, (long long)kBAMinKeysPerSplit);
  kps = max(kps, (long long)((nmax + S - 1) / S));
  return (int)kps;
}

__device__ __forceinline__ int batch_live_splits(int n_keys, int S, int kps) {
  int l = (n_keys + kps - 1) / kps;
  return l < 1 ? 1 : (l > S ? S : l);
}

template <int DPL, int G>
__global__ void __launch_bounds__(kBAWarps * 32, 1)
    batch_attn_kernel(const float* __restrict__ q, const BatchParams* __restrict__ bp, ModelDev m,
                      int layer, int S, int num_sms, float* __restrict__ part,
                      uint32_t* __restrict__ tickets, uint16_t* __restrict__ xh,
                      uint16_t* __restrict__ xl) {
  pdl_trigger();
  pdl_wait();
  constexpr int d = DPL * 32, PS = d + 4;
  constexpr int kBuf = 2 * kBAKeys * d;  // bf16 elements per buffer (K then V)
  extern __shared__ __align__(16) uint8_t ba_raw[];
  uint16_t* buf = reinterpret_cast<uint16_t*>(ba_raw);
  float* xbs = reinterpret_cast<float*>(buf + kBAStages * kBuf);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int sp = blockIdx.x, g = blockIdx.y, r = blockIdx.z;
  const int n_keys = bp->pos[r] + 1;
  const int live = batch_live_splits(n_keys, S, batch_keys_per_split(bp, m.n_kv, S, num_sms));
  if (sp >= live) return;
  // keys per split in whole blocks of kBAKeys: every block then lies in one KV
  // page (a trailing split may hold no keys and contributes an empty partial)
  const int chunk = ((n_keys + live - 1) / live + kBAKeys - 1) / kBAKeys * kBAKeys;
  const int k0 = min(n_keys, sp * chunk), k1 = min(n_keys, k0 + chunk);
  const int nq = m.n_q, slot = bp->slot[r];
  AttnState<DPL, G> st;
  attn_init<DPL, G>(st, q + (size_t)r * nq * d + (size_t)g * G * d, d, m.attn_scale, lane);
  float* xb = xbs + warp * kAttnXbStride;
  const int nblk = (k1 - k0 + kBAKeys - 1) / kBAKeys;
  auto issue = [&](int b) {
    const int kb = k0 + b * kBAKeys, nk = min(kBAKeys, k1 - kb);
    uint16_t* dst = buf + (b % kBAStages) * kBuf;
    const size_t off = kv_row(m, slot, layer, g, kb);
    const uint16_t* K = m.kcache + off;
    const uint16_t* V = m.vcache + off;
    const int pieces = nk * d / 8;  // 16-byte pieces of K (and of V)
    for (int i = threadIdx.x; i < pieces; i += blockDim.x) {
      cp_async16(dst + i * 8, K + i * 8);
      cp_async16(dst + kBAKeys * d + i * 8, V + i * 8);
    }
  };
  // blocks 0 .. kBAStages - 2 in flight before the loop; block b + kBAStages - 1
  // is requested while block b is used (one commit group per block)
#pragma unroll
  for (int b = 0; b < kBAStages - 1; ++b) {
    if (b < nblk) issue(b);
    cp_async_commit();
  }
  for (int b = 0; b < nblk; ++b) {
    if (b + kBAStages - 1 < nblk) issue(b + kBAStages - 1);
    cp_async_commit();
    cp_async_wait<kBAStages - 1>();
    __syncthreads();
    const int kb = k0 + b * kBAKeys, nk = min(kBAKeys, k1 - kb);
    const uint16_t* ks = buf + (b % kBAStages) * kBuf;
    const uint16_t* vs = ks + kBAKeys * d;
    for (int j0 = 4 * warp; j0 < nk; j0 += 4 * kBAWarps) {
      const int nj = min(4, nk - j0);
      {
        float kv[4][DPL];
#pragma unroll
        for (int t = 0; t < 4; ++t) {
          const int jr = attn_key_row<G>(t, lane);
          if (jr < nj) load_kv_row<DPL>(ks + (size_t)(j0 + jr) * d + lane * DPL, kv[t]);
          else
#pragma unroll
            for (int i = 0; i < DPL; ++i) kv[t][i] = 0.f;
        }
        attn_scores4<DPL, G>(st, kv, nj, xb, lane);
      }
      float vv[4][DPL];
#pragma unroll
      for (int t = 0; t < 4; ++t) {
        if (t < nj) load_kv_row<DPL>(vs + (size_t)(j0 + t) * d + lane * DPL, vv[t]);
        else
#pragma unroll
          for (int i = 0; i < DPL; ++i) vv[t][i] = 0.f;
      }
      attn_update4<DPL, G>(st, vv, xb);
    }
    __syncthreads();  // this buffer is refilled by block b + kBAStages
  }
  cp_async_wait<0>();
  __syncthreads();
  // the 16 warps' states through shared memory, then one partial
  float* ws = reinterpret_cast<float*>(ba_raw);  // [16][G][PS], reuses the key buffers
#pragma unroll
  for (int h = 0; h < G; ++h) {
#pragma unroll
    for (int i = 0; i < DPL; ++i) ws[(warp * G + h) * PS + lane * DPL + i] = st.o[h][i];
    if (lane == 0) {
      ws[(warp * G + h) * PS + d] = st.mx[h];
      ws[(warp * G + h) * PS + d + 1] = st.l[h];
    }
  }
  __syncthreads();
  const size_t out_row = (size_t)r * nq * d + (size_t)g * G * d;
  if (live == 1) {
    // the only split: normalise and write the O projection's input directly
    for (int idx = threadIdx.x; idx < G * d; idx += blockDim.x) {
      const int h = idx / d, i = idx - h * d;
      float M = -INFINITY;
      for (int w = 0; w < kBAWarps; ++w) M = fmaxf(M, ws[(w * G + h) * PS + d]);
      float num = 0.f, den = 0.f;
      for (int w = 0; w < kBAWarps; ++w) {
        const float mw = ws[(w * G + h) * PS + d];
        if (mw == -INFINITY) continue;
        const float c = __expf(mw - M);
        num = fmaf(c, ws[(w * G + h) * PS + i], num);
        den = fmaf(c, ws[(w * G + h) * PS + d + 1], den);
      }
      split_store(num / den, xh, xl, out_row + (size_t)h * d + i);
    }
    return;
  }
  float* dst = part + ((size_t)(r * m.n_kv + g) * S + sp) * G * PS;
  for (int idx = threadIdx.x; idx < G * (d + 2); idx += blockDim.x) {
    const int h = idx / (d + 2), i = idx - h * (d + 2);
    float M = -INFINITY;
    for (int w = 0; w < kBAWarps; ++w) M = fmaxf(M, ws[(w * G + h) * PS + d]);
    float val = 0.f;
    if (M != -INFINITY)
      for (int w = 0; w < kBAWarps; ++w) {
        const float mw = ws[(w * G + h) * PS + d];
        if (mw == -INFINITY) continue;
        const float x = i < d ? ws[(w * G + h) * PS + i] : ws[(w * G + h) * PS + d + 1];
        val = fmaf(__expf(mw - M), x, val);
      }
    dst[h * PS + i] = i == d ? M : val;
  }
  // The last of the live splits of (request, KV head) merges them (the
  // ticket counts the splits of this step and is put back to zero by the
  // last one; the next step reaches it only after this kernel completes).
  __shared__ int is_last;
  __syncthreads();
  if (threadIdx.x == 0) {
    __threadfence();  // this split's partial before the ticket
    const unsigned old = atomicAdd(tickets + r * m.n_kv + g, 1u);
    is_last = old == (unsigned)live - 1u;
    if (is_last) tickets[r * m.n_kv + g] = 0u;
  }
  __syncthreads();
  if (!is_last) return;
  __threadfence();  // the other splits' partials, after their tickets
  const float* pg = part + (size_t)(r * m.n_kv + g) * S * G * PS;
  // every split's (maximum, sum) into shared memory (the warps' states are
  // no longer needed), then each output element from the splits' partials
  float* ml = reinterpret_cast<float*>(ba_raw);  // [live][G][2]
  for (int idx = threadIdx.x; idx < live * G; idx += blockDim.x) {
    const float2 v = __ldcg(reinterpret_cast<const float2*>(pg + (size_t)idx * PS + d));
    ml[2 * idx] = v.x;
    ml[2 * idx + 1] = v.y;
  }
  __syncthreads();
  for (int idx = threadIdx.x; idx < G * d; idx += blockDim.x) {
    const int h = idx / d, i = idx - h * d;
    float M = -INFINITY;
    for (int s2 = 0; s2 < live; ++s2)
      if (ml[2 * (s2 * G + h) + 1] != 0.f) M = fmaxf(M, ml[2 * (s2 * G + h)]);
    float num = 0.f, den = 0.f;
#pragma unroll 4
    for (int s2 = 0; s2 < live; ++s2) {
      const float ls = ml[2 * (s2 * G + h) + 1];
      const float o = __ldcg(pg + ((size_t)s2 * G + h) * PS + i);
      if (ls == 0.f) continue;
      const float c = __expf(ml[2 * (s2 * G + h)] - M);
      num = fmaf(c, o, num);
      den = fmaf(c, ls, den);
    }
    split_store(num / den, xh, xl, out_row + (size_t)h * d + i);
  }
}

// The batched step's elementwise operators run over (token, 1024-element
// slice) grids of 256 threads, four elements each.  RMSNorm is deferred: they
// write x * w (split into xh, xl) and add this slice's sum of x^2 into
// tok_ss[t]; the next GEMM scales its outputs by 1/sqrt(tok_ss[t]/H + eps).
__device__ __forceinline__ void block_ss_add(float ss, float* dst) {
  __shared__ float red[8];
  for (int o = 16; o; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = ss;
  __syncthreads();
  if (threadIdx.x == 0) {
    float tot = 0.f;
    for (int i = 0; i < (int)(blockDim.x >> 5); ++i) tot += red[i];
    atomicAdd(dst, tot);
  }
}

// x[t] = E[token]; xh/xl = split(x * w); tok_ss[t] += sum x^2.
__global__ void b_embed_norm_kernel(const uint16_t* __restrict__ E, const int32_t* __restrict__ tokens,
                                    int H, int vocab, const uint16_t* __restrict__ w,
                                    float* __restrict__ x, uint16_t* __restrict__ xh,
                                    uint16_t* __restrict__ xl, float* __restrict__ tok_ss,
                                    int32_t* __restrict__ status) {
  pdl_trigger();
  pdl_wait();
  const int t = blockIdx.y;
  int tok = tokens[t];
  if (tok < 0 || tok >= vocab) {
    if (threadIdx.x == 0 && blockIdx.x == 0 && atomicCAS(status, 0, MK_ERR_TOKEN_RANGE) == 0)
      status[1] = tok;
    tok = 0;
  }
  float ss = 0.f;
  const int i0 = blockIdx.x * 1024 + threadIdx.x * 4;
  for (int i = i0; i < min(H, i0 + 4); ++i) {
    const float v = bf16_val(E[(size_t)tok * H + i]);
    x[(size_t)t * H + i] = v;
    ss = fmaf(v, v, ss);
    split_store(v * bf16_val(w[i]), xh, xl, (size_t)t * H + i);
  }
  block_ss_add(ss, tok_ss + t);
}

// x[t] += sum of the partials of y[t]; xh/xl = split(x * w); tok_ss[t] += sum x^2.
__global__ void b_residual_norm_kernel(float* __restrict__ x, const float* __restrict__ y, int H,
                                       int ldy, int nparts, size_t pstride,
                                       const uint16_t* __restrict__ w, uint16_t* __restrict__ xh,
                                       uint16_t* __restrict__ xl, float* __restrict__ tok_ss) {
  pdl_trigger();
  pdl_wait();
  const int t = blockIdx.y;
  float ss = 0.f;
  const int i0 = blockIdx.x * 1024 + threadIdx.x * 4;
  for (int i = i0; i < min(H, i0 + 4); ++i) {
    const float nx = x[(size_t)t * H + i] + sum_parts(y + (size_t)t * ldy + i, nparts, pstride);
    x[(size_t)t * H + i] = nx;
    ss = fmaf(nx, nx, ss);
    split_store(nx * bf16_val(w[i]), xh, xl, (size_t)t * H + i);
  }
  block_ss_add(ss, tok_ss + t);
}

// xh/xl[t][j] = split(silu(gate_j) * up_j), gate/up summed over the partials.
__global__ void b_swiglu_kernel(const float* __restrict__ y, int ldy, int F, int nparts,
                                size_t pstride, uint16_t* __restrict__ xh, uint16_t* __restrict__ xl) {
  pdl_trigger();
  pdl_wait();
  const int t = blockIdx.y;
  const int j0 = blockIdx.x * 1024 + threadIdx.x * 4;
  for (int j = j0; j < min(F, j0 + 4); ++j) {
    const float g = sum_parts(y + (size_t)t * ldy + 2 * j, nparts, pstride);
    const float u = sum_parts(y + (size_t)t * ldy + 2 * j + 1, nparts, pstride);
    split_store(g / (1.0f + expf(-g)) * u, xh, xl, (size_t)t * F + j);
  }
}

// Per-request argmax over the logits: slices of 4096 entries fold into one
// 64-bit (ordered value, inverted index) key per request with atomicMax; the
// lowest index wins ties.  best[] starts at zero each step.
__global__ void b_argmax_kernel(const float* __restrict__ logits, int V,
                                unsigned long long* __restrict__ best) {
  pdl_trigger();
  pdl_wait();
  __shared__ unsigned long long red[8];
  const int r = blockIdx.y;
  unsigned long long k = 0ull;
  const int i1 = min(V, (int)(blockIdx.x + 1) * 4096);
  for (int i = blockIdx.x * 4096 + threadIdx.x; i < i1; i += blockDim.x) {
    uint32_t u = __float_as_uint(logits[(size_t)r * V + i]);
    u = (u & 0x80000000u) ? ~u : (u | 0x80000000u);
    const unsigned long long c = ((unsigned long long)u << 32) | (0xffffffffu - (uint32_t)i);
    k = c > k ? c : k;
  }
  for (int o = 16; o; o >>= 1) {
    const unsigned long long v = __shfl_xor_sync(0xffffffffu, k, o);
    k = v > k ? v : k;
  }
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = k;
  __syncthreads();
  if (threadIdx.x == 0) {
    for (int w2 = 1; w2 < (int)(blockDim.x >> 5); ++w2) k = red[w2] > k ? red[w2] : k;
    k = red[0] > k ? red[0] : k;
    atomicMax(best + r, k);
  }
}

__global__ void b_ids_kernel(const unsigned long long* __restrict__ best, int n, int32_t* __restrict__ ids) {
  pdl_trigger();
  pdl_wait();
  const int r = threadIdx.x;
  if (r < n) ids[r] = (int32_t)(0xffffffffu - (uint32_t)(best[r] & 0xffffffffull));
}


// ------------------------------------------------------------------ host

// Launch with programmatic stream serialization: the kernel may start while
// the previous kernel of the stream runs; it calls pdl_wait() before reading
// that kernel's results (the kernels above all do).
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*k)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                       Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute at[1];
  at[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  at[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = at;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, k, args...);
}

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  }
  return fn;
}

// 2-D bf16 tensor [rows][cols] (row-major), boxes of 64 columns x box_rows
// rows, 128-byte swizzle, zero fill outside.
bool make_map(CUtensorMap* map, const void* base, int rows, int cols, int box_rows = 128) {
  auto fn = encode_fn();
  if (!fn) return false;
  const cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
  const cuuint64_t strides[1] = {(cuuint64_t)cols * 2};
  const cuuint32_t box[2] = {(cuuint32_t)kGK, (cuuint32_t)box_rows};
  const cuuint32_t estr[2] = {1u, 1u};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box,
            estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Y (+ z * n_tok * ldy for split z) = W x^T over `splits` K ranges.
template <int BN, int STAGES>
std::string gemm(const uint16_t* W, int n_rows, int K, const uint16_t* xh, const uint16_t* xm,
                 const uint16_t* xl, int n_tok, float* Y, int ldy, const uint16_t* bias,
                 int32_t* err, cudaStream_t st, int splits = 1, const float* tok_ss = nullptr,
                 float norm_eps = 0.f, bool pdl = false) {
  CUtensorMap mw, mh, mm, ml;
  if (!make_map(&mw, W, n_rows, K) || !make_map(&mh, xh, n_tok, K, BN) ||
      !make_map(&mm, xm, n_tok, K, BN) || !make_map(&ml, xl, n_tok, K, BN))
    return "cuTensorMapEncodeTiled failed";
  const dim3 grid((n_rows + kGM - 1) / kGM, (n_tok + BN - 1) / BN, splits);
  const uint16_t* b = splits == 1 ? bias : nullptr;
  const size_t pst = (size_t)n_tok * ldy;
  if (pdl) {
    const cudaError_t le = launch_pdl(gemm_wx_kernel<BN, STAGES>, grid, dim3(128),
                                      gemm_smem_bytes<BN, STAGES>(), st, mw, mh, mm, ml, n_rows, n_tok, K,
                                      Y, ldy, pst, b, err, tok_ss, K, norm_eps, (uint16_t*)nullptr, 0);
    if (le != cudaSuccess) return std::string("GEMM launch: ") + cudaGetErrorString(le);
  } else {
    gemm_wx_kernel<BN, STAGES><<<grid, 128, gemm_smem_bytes<BN, STAGES>(), st>>>(
        mw, mh, mm, ml, n_rows, n_tok, K, Y, ldy, pst, b, err, tok_ss, K, norm_eps, nullptr, 0);
  }
  const cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? "" : std::string("GEMM launch: ") + cudaGetErrorString(e);
}

constexpr int kPBN = 128, kPStages = 3;   // prompt GEMM: 128 tokens per CTA, 64 KB per stage
constexpr int kDStages = 11;              // decode GEMM: 8 requests, high and low parts packed

// Y (+ z * n_tok * ldy for split z) = W x^T for n_tok <= 8 tokens whose high
// parts are rows 0..7 and low parts rows 8..15 of xhl ([16][K] bf16).
// act_hl (with splits == 1): instead of Y, write silu(gate) * up of the
// interleaved gate/up rows as the next GEMM's [16][n_rows / 2] split input.
// two_per_sm: 6 stages (108 KB) so that two CTAs share an SM -- for a matrix
// whose 128-row tiles number between one and two waves of SMs, all of them
// then start at once instead of a full wave and a partial one.
constexpr int kDStagesPair = 6;
std::string gemm_hl(const uint16_t* W, int n_rows, int K, const uint16_t* xhl, int n_tok, float* Y,
                    int ldy, int32_t* err, cudaStream_t st, int splits, const float* tok_ss,
                    float norm_eps, uint16_t* act_hl = nullptr, bool two_per_sm = false) {
  CUtensorMap mw, mh;
  if (!make_map(&mw, W, n_rows, K) || !make_map(&mh, xhl, 16, K, 16))
    return "cuTensorMapEncodeTiled failed";
  const dim3 grid((n_rows + kGM - 1) / kGM, 1, splits);
  const cudaError_t le =
      two_per_sm
          ? launch_pdl(gemm_wx_kernel<16, kDStagesPair, true>, grid, dim3(128),
                       gemm_smem_bytes<16, kDStagesPair, true>(), st, mw, mh, mh, mh, n_rows, n_tok, K, Y,
                       ldy, (size_t)n_tok * ldy, (const uint16_t*)nullptr, err, tok_ss, K, norm_eps,
                       act_hl, n_rows / 2)
          : launch_pdl(gemm_wx_kernel<16, kDStages, true>, grid, dim3(128),
                       gemm_smem_bytes<16, kDStages, true>(), st, mw, mh, mh, mh, n_rows, n_tok, K, Y,
                       ldy, (size_t)n_tok * ldy, (const uint16_t*)nullptr, err, tok_ss, K, norm_eps,
                       act_hl, n_rows / 2);
  return le == cudaSuccess ? "" : std::string("GEMM launch: ") + cudaGetErrorString(le);
}

template <int DPL, int G>
std::string launch_attn(dim3 grid, cudaStream_t st, const float* q, const int32_t* tiles,
                        const ModelDev& m, int layer, uint16_t* xh, uint16_t* xm, uint16_t* xl) {
  const size_t smem = (size_t)2 * kPAKeys * DPL * 32 * 2 + (size_t)kPAWarps * kAttnXbStride * 4;
  auto k = prefill_attn_kernel<DPL, G>;
  cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  k<<<grid, kPAWarps * 32, smem, st>>>(q, tiles, m, layer, xh, xm, xl);
  const cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? "" : std::string("attention launch: ") + cudaGetErrorString(e);
}

std::string attn(dim3 grid, cudaStream_t st, const float* q, const int32_t* tiles, const ModelDev& m,
                 int layer, uint16_t* xh, uint16_t* xm, uint16_t* xl) {
  const int G = m.group;
  if (m.head_dim == 128) {
    if (G == 1) return launch_attn<4, 1>(grid, st, q, tiles, m, layer, xh, xm, xl);
    if (G == 2) return launch_attn<4, 2>(grid, st, q, tiles, m, layer, xh, xm, xl);
    if (G == 4) return launch_attn<4, 4>(grid, st, q, tiles, m, layer, xh, xm, xl);
  } else {
    if (G == 1) return launch_attn<2, 1>(grid, st, q, tiles, m, layer, xh, xm, xl);
    if (G == 2) return launch_attn<2, 2>(grid, st, q, tiles, m, layer, xh, xm, xl);
    if (G == 4) return launch_attn<2, 4>(grid, st, q, tiles, m, layer, xh, xm, xl);
    if (G == 7) return launch_attn<2, 7>(grid, st, q, tiles, m, layer, xh, xm, xl);
    if (G == 8) return launch_attn<2, 8>(grid, st, q, tiles, m, layer, xh, xm, xl);
  }
  return "unsupported query heads per KV head";
}

}  // namespace

PFN_cuTensorMapEncodeTiled_v12000 prefill_encode_fn() { return encode_fn(); }

bool prefill_gemm_supported(const ModelDev& m) {
  const int qd = m.n_q * m.head_dim;
  return m.hidden % kGK == 0 && m.ffn % kGK == 0 && qd % kGK == 0 && encode_fn() != nullptr;
}

std::string prefill_alloc(const ModelDev& m, int max_tokens, PrefillScratch* sc,
                          std::vector<void*>* owned) {
  const int H = m.hidden, F = m.ffn, qd = m.n_q * m.head_dim;
  const int qkvR = qkv_rows(m.n_q, m.n_kv, m.head_dim);
  const size_t T = (size_t)max_tokens;
  const size_t ycols = (size_t)std::max(std::max(qkvR, 2 * F), H);
  const size_t xcols = (size_t)std::max(std::max(H, F), qd);
  struct A { void** p; size_t bytes; } allocs[] = {
      {(void**)&sc->x, T * H * 4},          {(void**)&sc->y, T * ycols * 4},
      {(void**)&sc->q, T * qd * 4},         {(void**)&sc->xh, T * xcols * 2},
      {(void**)&sc->xl, T * xcols * 2},     {(void**)&sc->xm, T * xcols * 2},
      {(void**)&sc->meta, (3 * T + 4 * T + T + 16) * 4},
      {(void**)&sc->err, 16}};
  for (auto& a : allocs) {
    const cudaError_t e = cudaMalloc(a.p, a.bytes);
    if (e != cudaSuccess) return std::string("prefill scratch: ") + cudaGetErrorString(e);
    owned->push_back(*a.p);
  }
  cudaMemset(sc->err, 0, 16);
  if (cudaFuncSetAttribute(gemm_wx_kernel<kPBN, kPStages>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           (int)gemm_smem_bytes<kPBN, kPStages>()) != cudaSuccess)
    return "GEMM shared memory attribute";
  sc->max_tokens = max_tokens;
  return "";
}

std::string prefill_run(const ModelDev& m, const PrefillWeights& w, PrefillScratch& sc,
                        cudaStream_t st, const int32_t* tokens_dev, const int32_t* offsets_host,
                        const int32_t* slots_host, int n_req, bool tc_attn, bool* timed_out) {
  *timed_out = false;
  const int H = m.hidden, F = m.ffn, d = m.head_dim, qd = m.n_q * d, L = m.n_layers;
  const int qkvR = qkv_rows(m.n_q, m.n_kv, d);
  const int ldy = std::max(std::max(qkvR, 2 * F), H);
  const bool use_fa = tc_attn;
  if (use_fa) {
    const std::string fe = flash_attn_prepare(m, &sc.fa);
    if (!fe.empty()) return fe;
  }
  // every position but each prompt's last, as (request, position) in order
  std::vector<int> tok_src, slot, pos;
  for (int r = 0; r < n_req; ++r)
    for (int p = 0; p + 1 < offsets_host[r + 1] - offsets_host[r]; ++p) {
      tok_src.push_back(offsets_host[r] + p);
      slot.push_back(slots_host[r]);
      pos.push_back(p);
    }
  const int total = (int)tok_src.size();
  std::string e;
  for (int b0 = 0; b0 < total; b0 += sc.max_tokens) {
    const int T = std::min(sc.max_tokens, total - b0);
    // per-token arrays, then attention tiles: runs of <= 16 positions of one request
    std::vector<int32_t> meta(3 * (size_t)T);
    std::vector<int32_t> tiles;
    for (int t = 0; t < T; ++t) {
      meta[t] = tok_src[b0 + t];
      meta[T + t] = slot[b0 + t];
      meta[2 * T + t] = pos[b0 + t];
    }
    for (int t = 0; t < T;) {
      int n = 1;
      while (t + n < T && n < kPAWarps && slot[b0 + t + n] == slot[b0 + t]) ++n;
      tiles.insert(tiles.end(), {t, n, slot[b0 + t], pos[b0 + t]});
      t += n;
    }
    int ntiles = (int)tiles.size() / 4;
    if (use_fa) {
      // tensor-core attention: runs of <= 128 positions of one request, the
      // longest key ranges first (the causal work is uneven)
      std::vector<std::array<int32_t, 4>> ft;
      for (int t = 0; t < T;) {
        int n = 1;
        while (t + n < T && n < kFaTileRows && slot[b0 + t + n] == slot[b0 + t]) ++n;
        ft.push_back({t, n, slot[b0 + t], pos[b0 + t]});
        t += n;
      }
      std::stable_sort(ft.begin(), ft.end(), [](const std::array<int32_t, 4>& a,
                                                const std::array<int32_t, 4>& b) {
        return a[1] + a[3] > b[1] + b[3];
      });
      tiles.clear();
      for (const auto& f : ft) tiles.insert(tiles.end(), f.begin(), f.end());
      ntiles = (int)ft.size();
    }
    int32_t* d_src = sc.meta;
    int32_t* d_slot = sc.meta + T;
    int32_t* d_pos = sc.meta + 2 * T;
    int32_t* d_tiles = sc.meta + 3 * (size_t)sc.max_tokens;
    if (cudaMemcpyAsync(sc.meta, meta.data(), meta.size() * 4, cudaMemcpyHostToDevice, st) != cudaSuccess ||
        cudaMemcpyAsync(d_tiles, tiles.data(), tiles.size() * 4, cudaMemcpyHostToDevice, st) != cudaSuccess)
      return "prefill metadata upload";
    embed_kernel<<<T, 256, 0, st>>>(m.embed, tokens_dev, d_src, H, m.vocab, sc.x, m.status);
    for (int l = 0; l < L; ++l) {
      rmsnorm_split_kernel<<<T, 256, 0, st>>>(sc.x, m.attn_norm + (size_t)l * H, H, m.rms_eps, sc.xh, sc.xm, sc.xl);
      const uint16_t* bias = m.qkv_bias ? m.bqkv + (size_t)l * qkvR : nullptr;
      if (!(e = gemm<kPBN, kPStages>(w.qkv[l], qkvR, H, sc.xh, sc.xm, sc.xl, T, sc.y, ldy, bias, sc.err, st)).empty()) return e;
      rope_kv_kernel<<<T, 256, 0, st>>>(sc.y, ldy, 1, 0, nullptr, d_slot, d_pos, m, l, sc.q);
      e = use_fa ? flash_attn_launch(m, sc.fa, d_tiles, ntiles, l, sc.q, qd, sc.xh, sc.xm, sc.xl, qd,
                                     sc.err, st)
                 : attn(dim3(ntiles, m.n_kv), st, sc.q, d_tiles, m, l, sc.xh, sc.xm, sc.xl);
      if (!e.empty()) return e;
      if (!(e = gemm<kPBN, kPStages>(w.o[l], H, qd, sc.xh, sc.xm, sc.xl, T, sc.y, ldy, nullptr, sc.err, st)).empty()) return e;
      residual_kernel<<<T, 256, 0, st>>>(sc.x, sc.y, H, ldy, 1, 0);
      rmsnorm_split_kernel<<<T, 256, 0, st>>>(sc.x, m.ffn_norm + (size_t)l * H, H, m.rms_eps, sc.xh, sc.xm, sc.xl);
      if (!(e = gemm<kPBN, kPStages>(w.gu[l], 2 * F, H, sc.xh, sc.xm, sc.xl, T, sc.y, ldy, nullptr, sc.err, st)).empty()) return e;
      swiglu_split_kernel<<<T, 256, 0, st>>>(sc.y, ldy, F, 1, 0, sc.xh, sc.xm, sc.xl);
      if (!(e = gemm<kPBN, kPStages>(w.dn[l], H, F, sc.xh, sc.xm, sc.xl, T, sc.y, ldy, nullptr, sc.err, st)).empty()) return e;
      residual_kernel<<<T, 256, 0, st>>>(sc.x, sc.y, H, ldy, 1, 0);
    }
    const cudaError_t ce = cudaGetLastError();
    if (ce != cudaSuccess) return std::string("prefill launch: ") + cudaGetErrorString(ce);
  }
  // The GEMM kernel records a wait that ran out (never expected) in sc.err.
  int32_t herr = 0;
  if (cudaMemcpyAsync(&herr, sc.err, 4, cudaMemcpyDeviceToHost, st) != cudaSuccess ||
      cudaStreamSynchronize(st) != cudaSuccess)
    return std::string("prefill: ") + cudaGetErrorString(cudaGetLastError());
  if (herr) {
    *timed_out = true;
    return "prefill: a pipeline wait timed out (GEMM or attention)";
  }
  return "";
}

namespace {

template <int DPL, int G>
size_t batch_attn_smem() {
  // kBAStages key/value buffers and the warps' softmax scratch; after the key
  // loop the warps' states (16 x G x (d + 4) floats) reuse the same bytes
  const size_t loop =
      (size_t)kBAStages * 2 * kBAKeys * DPL * 32 * 2 + (size_t)kBAWarps * kAttnXbStride * 4;
  const size_t merge = (size_t)kBAWarps * G * (DPL * 32 + 4) * 4;
  return loop > merge ? loop : merge;
}

template <int DPL, int G>
std::string launch_batch_attn(dim3 grid, cudaStream_t st, const float* q, const BatchParams* bp,
                              const ModelDev& m, int layer, int S, int num_sms, float* part,
                              bool set_attr,
                              uint32_t* tickets, uint16_t* xh, uint16_t* xl) {
  auto k = batch_attn_kernel<DPL, G>;
  const size_t smem = batch_attn_smem<DPL, G>();
  if (set_attr) {
    return cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) == cudaSuccess
               ? "" : "batched attention shared memory attribute";
  }
  const cudaError_t e = launch_pdl(k, grid, dim3(kBAWarps * 32), smem, st, q, bp, m, layer, S, num_sms,
                                   part, tickets, xh, xl);
  return e == cudaSuccess ? "" : std::string("batched attention launch: ") + cudaGetErrorString(e);
}

std::string batch_attn(dim3 grid, cudaStream_t st, const float* q, const BatchParams* bp,
                       const ModelDev& m, int layer, int S, int num_sms, float* part,
                       bool set_attr = false,
                       uint32_t* tickets = nullptr, uint16_t* xh = nullptr, uint16_t* xl = nullptr) {
  const int G = m.group;
#define MK_BA(DPL_, G_) \
  return launch_batch_attn<DPL_, G_>(grid, st, q, bp, m, layer, S, num_sms, part, set_attr, tickets, \
                                     xh, xl)
  if (m.head_dim == 128) {
    if (G == 1) MK_BA(4, 1);
    if (G == 2) MK_BA(4, 2);
    if (G == 4) MK_BA(4, 4);
  } else {
    if (G == 1) MK_BA(2, 1);
    if (G == 2) MK_BA(2, 2);
    if (G == 4) MK_BA(2, 4);
    if (G == 7) MK_BA(2, 7);
    if (G == 8) MK_BA(2, 8);
  }
#undef MK_BA
  return "unsupported query heads per KV head";
}

// K split of a decode GEMM from a simple cost model: a CTA costs a fixed
// ~4 us (setup, pipeline fill, epilogue) plus its share of the 128-row tile
// at ~40 GB/s; waves of num_sms CTAs run one after another.  At least two K
// blocks per CTA, at most kBatchMaxSplitK splits.
int split_k(int n_rows, int K, int num_sms) {
  const int tiles = (n_rows + kGM - 1) / kGM, nk = K / kGK;
  const double tile_us = (double)kGM * K * 2 / 40e3;  // bytes / (40 GB/s) in us
  int best = 1;
  double best_t = 1e30;
  for (int z = 1; z <= kBatchMaxSplitK && z <= std::max(1, nk / 2); ++z) {
    const int waves = (tiles * z + num_sms - 1) / num_sms;
    const double t = waves * (4.0 + tile_us / z);
    if (t < best_t - 1e-9) {
      best_t = t;
      best = z;
    }
  }
  return best;
}

std::string batch_enqueue(const ModelDev& m, const PrefillWeights& w, BatchScratch& bs, int n,
                          int num_sms, cudaStream_t st) {
  const int H = m.hidden, F = m.ffn, d = m.head_dim, qd = m.n_q * d, L = m.n_layers, V = m.vocab;
  const int qkvR = qkv_rows(m.n_q, m.n_kv, d);
  const int ldy = std::max(std::max(qkvR, 2 * F), H);
  const size_t pstride = (size_t)n * ldy;
  // W_qkv, W_o, W_down have few 128-row tiles: split K so that two CTAs per
  // SM (6 stages each) fill one wave of 2 * num_sms
  auto pair_split = [&](int rows, int K) {
    const int tiles = (rows + kGM - 1) / kGM, nk = K / kGK;
    int z = (2 * num_sms) / tiles;
    z = std::min(z, kBatchMaxSplitK);
    z = std::min(z, std::max(1, nk / 2));
    return std::max(z, 1);
  };
  const int zq = pair_split(qkvR, H), zo = pair_split(H, qd);
  const int gu_tiles = (2 * F + kGM - 1) / kGM;
  const bool gu_pair = gu_tiles > num_sms && gu_tiles <= 2 * num_sms;
  const int zg = split_k(2 * F, H, num_sms), zd = pair_split(H, F);
  std::string e;
  BatchParams* bp = bs.params;
#define CKL(call)                                                                       \
  do {                                                                                  \
    const cudaError_t le_ = (call);                                                     \
    if (le_ != cudaSuccess) return std::string("batched step launch: ") + cudaGetErrorString(le_); \
  } while (0)
  const int hsl = (H + 1023) / 1024, fsl = (F + 1023) / 1024;
  const int psl = ((qkvR >> 1) + 255) / 256;
  // per-step accumulators: the norms' sums of squares, the argmax keys
  if (cudaMemsetAsync(bs.acc, 0, bs.acc_bytes, st) != cudaSuccess) return "batched step memset";
  float* ss = reinterpret_cast<float*>(bs.acc);                       // [2L + 1][kMaxBatch]
  unsigned long long* best = reinterpret_cast<unsigned long long*>(bs.acc) + (2 * L + 1) * kMaxBatch / 2 + 1;
  // GEMM inputs: [16][K] per contraction, rows 0..7 the high parts, 8..15 the low parts
  uint16_t* const xhl = bs.xh;
  auto lo = [&](int K) { return xhl + (size_t)8 * K; };
  b_embed_norm_kernel<<<dim3(hsl, n), 256, 0, st>>>(m.embed, bs.tokens, H, m.vocab, m.attn_norm, bs.x,
                                                    xhl, lo(H), ss, m.status);
  for (int l = 0; l < L; ++l) {
    float* ss_attn = ss + (size_t)(2 * l) * kMaxBatch;
    float* ss_ffn = ss + (size_t)(2 * l + 1) * kMaxBatch;
    float* ss_next = ss + (size_t)(2 * l + 2) * kMaxBatch;
    const uint16_t* bias = m.qkv_bias ? m.bqkv + (size_t)l * qkvR : nullptr;
    if (!(e = gemm_hl(w.qkv[l], qkvR, H, xhl, n, bs.y, ldy, bs.err, st, zq, ss_attn, m.rms_eps,
                      nullptr, true)).empty())
      return e;
    CKL(launch_pdl(rope_kv_kernel, dim3(n, psl), dim3(256), 0, st, (const float*)bs.y, ldy, zq, pstride,
                   bias, (const int32_t*)bp->slot, (const int32_t*)bp->pos, m, l, bs.q));
    if (!(e = batch_attn(dim3(bs.splits, m.n_kv, n), st, bs.q, bp, m, l, bs.splits, num_sms, bs.part, false,
                         bs.tickets, xhl, lo(qd))).empty())
      return e;
    if (!(e = gemm_hl(w.o[l], H, qd, xhl, n, bs.y, ldy, bs.err, st, zo, nullptr, 0.f, nullptr, true)).empty())
      return e;
    CKL(launch_pdl(b_residual_norm_kernel, dim3(hsl, n), dim3(256), 0, st, bs.x, (const float*)bs.y, H,
                   ldy, zo, pstride, m.ffn_norm + (size_t)l * H, xhl, lo(H), ss_ffn));
    // SwiGLU output into a second buffer: the gate/up GEMM still reads xhl
    if (zg == 1) {  // in the GEMM's epilogue
      if (!(e = gemm_hl(w.gu[l], 2 * F, H, xhl, n, bs.y, ldy, bs.err, st, 1, ss_ffn, m.rms_eps,
                        bs.xh2, gu_pair)).empty())
        return e;
    } else {
      if (!(e = gemm_hl(w.gu[l], 2 * F, H, xhl, n, bs.y, ldy, bs.err, st, zg, ss_ffn, m.rms_eps)).empty())
        return e;
      CKL(launch_pdl(b_swiglu_kernel, dim3(fsl, n), dim3(256), 0, st, (const float*)bs.y, ldy, F, zg,
                     pstride, bs.xh2, bs.xh2 + (size_t)8 * F));
    }
    if (!(e = gemm_hl(w.dn[l], H, F, bs.xh2, n, bs.y, ldy, bs.err, st, zd, nullptr, 0.f, nullptr, true)).empty())
      return e;
    // the residual add, then the next layer's attention norm (the final norm after the last)
    const uint16_t* next_norm = l + 1 < L ? m.attn_norm + (size_t)(l + 1) * H : m.final_norm;
    CKL(launch_pdl(b_residual_norm_kernel, dim3(hsl, n), dim3(256), 0, st, bs.x, (const float*)bs.y, H,
                   ldy, zd, pstride, next_norm, xhl, lo(H), ss_next));
  }
  if (!(e = gemm_hl(m.lm_head, V, H, xhl, n, bs.logits, V, bs.err, st, 1,
                    ss + (size_t)(2 * L) * kMaxBatch, m.rms_eps)).empty()) return e;
  CKL(launch_pdl(b_argmax_kernel, dim3((V + 4095) / 4096, n), dim3(256), 0, st, (const float*)bs.logits,
                 V, best));
  CKL(launch_pdl(b_ids_kernel, dim3(1), dim3(32), 0, st, (const unsigned long long*)best, n, bs.ids));
  const cudaError_t ce = cudaGetLastError();
  return ce == cudaSuccess ? "" : std::string("batched step launch: ") + cudaGetErrorString(ce);
}
#undef CKL

}  // namespace

std::string batch_alloc(const ModelDev& m, int num_sms, BatchScratch* bs, std::vector<void*>* owned) {
  const int H = m.hidden, F = m.ffn, d = m.head_dim, qd = m.n_q * d, G = m.group;
  const int qkvR = qkv_rows(m.n_q, m.n_kv, d);
  const size_t B = kMaxBatch;
  const size_t ycols = (size_t)std::max(std::max(qkvR, 2 * F), H);
  const size_t xcols = (size_t)std::max(std::max(H, F), qd);
  bs->splits = std::max(1, (2 * num_sms + (int)B * m.n_kv - 1) / ((int)B * m.n_kv));
  // per step: (2 layers + 1) norms' sums of squares, then the argmax keys
  bs->acc_bytes = ((size_t)(2 * m.n_layers + 1) * kMaxBatch + 2) * 4 + (size_t)kMaxBatch * 8 + 16;
  struct A { void** p; size_t bytes; } allocs[] = {
      {(void**)&bs->params, sizeof(BatchParams)},
      {(void**)&bs->tokens, B * 4},
      {(void**)&bs->x, B * H * 4},
      {(void**)&bs->y, (size_t)kBatchMaxSplitK * B * ycols * 4},
      {(void**)&bs->q, B * qd * 4},
      {(void**)&bs->part, B * m.n_kv * bs->splits * G * (d + 4) * 4},
      {(void**)&bs->xh, 2 * B * xcols * 2},
      {(void**)&bs->xh2, 2 * B * xcols * 2},
      {(void**)&bs->tickets, B * m.n_kv * 4},
      {(void**)&bs->logits, B * (size_t)m.vocab * 4},
      {(void**)&bs->ids, B * 4},
      {(void**)&bs->err, 16},
      {(void**)&bs->acc, bs->acc_bytes}};
  for (auto& a : allocs) {
    const cudaError_t e = cudaMalloc(a.p, a.bytes);
    if (e != cudaSuccess) return std::string("batched step scratch: ") + cudaGetErrorString(e);
    owned->push_back(*a.p);
  }
  cudaMemset(bs->err, 0, 16);
  cudaMemset(bs->xh, 0, 2 * B * xcols * 2);  // rows of absent requests stay finite
  cudaMemset(bs->xh2, 0, 2 * B * xcols * 2);
  cudaMemset(bs->tickets, 0, B * m.n_kv * 4);
  if (cudaFuncSetAttribute(gemm_wx_kernel<16, kDStages, true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           (int)gemm_smem_bytes<16, kDStages, true>()) != cudaSuccess ||
      cudaFuncSetAttribute(gemm_wx_kernel<16, kDStagesPair, true>,
                           cudaFuncAttributeMaxDynamicSharedMemorySize,
                           (int)gemm_smem_bytes<16, kDStagesPair, true>()) != cudaSuccess)
    return "decode GEMM shared memory attribute";
  return batch_attn(dim3(1), nullptr, nullptr, nullptr, m, 0, bs->splits, num_sms, nullptr, true);
}

std::string batch_step(const ModelDev& m, const PrefillWeights& w, BatchScratch& bs, int n,
                       int num_sms, cudaStream_t st) {
  if (n < 2 || n > kMaxBatch) return "batched step needs 2..8 requests";
  if (!bs.graph[n]) {
    cudaStream_t cs;
    if (cudaStreamCreateWithFlags(&cs, cudaStreamNonBlocking) != cudaSuccess) return "capture stream";
    cudaError_t e = cudaStreamBeginCapture(cs, cudaStreamCaptureModeThreadLocal);
    std::string err = e == cudaSuccess ? batch_enqueue(m, w, bs, n, num_sms, cs) : "begin capture";
    cudaGraph_t g = nullptr;
    const cudaError_t e2 = cudaStreamEndCapture(cs, &g);
    cudaStreamDestroy(cs);
    if (!err.empty()) {
      if (g) cudaGraphDestroy(g);
      return err;
    }
    if (e2 != cudaSuccess) return std::string("batched step capture: ") + cudaGetErrorString(e2);
    if (cudaGraphInstantiate(&bs.graph[n], g, 0) != cudaSuccess) {
      cudaGraphDestroy(g);
      return "batched step graph instantiation";
    }
    bs.graph_src[n] = g;
  }
  const cudaError_t e = cudaGraphLaunch(bs.graph[n], st);
  return e == cudaSuccess ? "" : std::string("batched step replay: ") + cudaGetErrorString(e);
}

}  // namespace mk
