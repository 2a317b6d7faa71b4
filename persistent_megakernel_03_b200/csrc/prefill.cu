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
// The GEMM computes Y[t][r] = sum_k W[r][k] * (xh[t][k] + xl[t][k]): the fp32
// activation is split into bf16 xh = bf16(x) and xl = bf16(x - xh), so two
// bf16 tcgen05.mma per K step reproduce the fp32 product to ~2^-16 relative,
// well inside the decode path's tolerance against the fp32 oracle.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <algorithm>
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

// ------------------------------------------------------------------ GEMM
// One CTA per 128 weight rows x 128 tokens.  Warp 0 lane 0 issues the TMA
// loads of a 4-stage ring (W tile 128 x 64, xh and xl tiles 128 x 64, all
// 128-byte swizzled), warp 1 lane 0 issues the MMAs into a 128 x 128 fp32
// accumulator in tensor memory and frees each stage with tcgen05.commit, and
// all four warps read the accumulator back (warp w owns TMEM lanes 32w..32w+31,
// i.e. weight rows) and store Y[token][row].
constexpr int kGM = 128, kGN = 128, kGK = 64, kGStages = 4;
constexpr int kGTile = 128 * kGK * 2;  // 16 KB, every operand tile
constexpr uint32_t kGStageBytes = 3 * kGTile;
constexpr uint64_t kGWaitNs = 2000000000ull;  // 2 s: far beyond any legal wait

struct __align__(1024) GemmSmem {
  uint8_t a[kGStages][kGTile];
  uint8_t bh[kGStages][kGTile];
  uint8_t bl[kGStages][kGTile];
  uint64_t full[kGStages];
  uint64_t empty[kGStages];
  uint64_t done;
  uint32_t tmem;
  int32_t failed;
};
constexpr size_t kGemmSmemBytes = sizeof(GemmSmem) + 1024;

// Bounded wait on an mbarrier phase; false after kGWaitNs (the caller records
// the failure and stops issuing work).
__device__ __forceinline__ bool gemm_wait(uint64_t* bar, uint32_t parity) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = globaltimer_ns();
  while (!mbar_try_wait(bar, parity))
    if (globaltimer_ns() - t0 > kGWaitNs) return false;
  return true;
}

__global__ void __launch_bounds__(128, 1)
    gemm_wx_kernel(const __grid_constant__ CUtensorMap tm_w, const __grid_constant__ CUtensorMap tm_xh,
                   const __grid_constant__ CUtensorMap tm_xl, int n_rows, int n_tok, int K,
                   float* __restrict__ Y, int ldy, const uint16_t* __restrict__ bias,
                   int32_t* __restrict__ err) {
  // The swizzled tiles must start on 1024-byte boundaries of the shared
  // window: round the dynamic base up (the launch adds 1 KB of slack).
  extern __shared__ __align__(16) uint8_t gsm_raw[];
  const uint32_t base = smem_u32(gsm_raw);
  GemmSmem& s = *reinterpret_cast<GemmSmem*>(gsm_raw + (((base + 1023u) & ~1023u) - base));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int m0 = blockIdx.x * kGM, n0 = blockIdx.y * kGN;
  const int nk = K / kGK;
  if (threadIdx.x == 0) {
    for (int i = 0; i < kGStages; ++i) {
      mbar_init(&s.full[i], 1);
      mbar_init(&s.empty[i], 1);
    }
    mbar_init(&s.done, 1);
    s.failed = 0;
    fence_barrier_init();
  }
  if (warp == 0) {
    tmem_alloc(&s.tmem, kGN);
    tmem_relinquish();
  }
  tc_fence_before_sync();
  __syncthreads();
  tc_fence_after_sync();
  const uint32_t tmem = s.tmem;
  // Loads issued and MMAs committed, for the teardown after a failed wait.
  int issued = 0;
  if (warp == 0 && lane == 0) {
    for (int kb = 0; kb < nk; ++kb) {
      const int st = kb % kGStages;
      if (kb >= kGStages && !gemm_wait(&s.empty[st], ((kb / kGStages) - 1) & 1)) {
        s.failed = 1;
        break;
      }
      mbar_arrive_expect_tx(&s.full[st], kGStageBytes);
      tma_load_2d(s.a[st], &tm_w, kb * kGK, m0, &s.full[st]);
      tma_load_2d(s.bh[st], &tm_xh, kb * kGK, n0, &s.full[st]);
      tma_load_2d(s.bl[st], &tm_xl, kb * kGK, n0, &s.full[st]);
      issued = kb + 1;
    }
    // every load must land before this CTA may exit
    for (int kb = (issued > kGStages ? issued - kGStages : 0); kb < issued; ++kb)
      gemm_wait(&s.full[kb % kGStages], (kb / kGStages) & 1);
  } else if (warp == 1 && lane == 0) {
    constexpr uint32_t idesc = mma_idesc_bf16_f32(kGM, kGN);
    int kb = 0;
    for (; kb < nk; ++kb) {
      const int st = kb % kGStages;
      if (!gemm_wait(&s.full[st], (kb / kGStages) & 1)) {
        s.failed = 1;
        break;
      }
      tc_fence_after_sync();
      const uint64_t da = sw128_kmajor_desc(s.a[st]);
      const uint64_t dh = sw128_kmajor_desc(s.bh[st]);
      const uint64_t dl = sw128_kmajor_desc(s.bl[st]);
#pragma unroll
      for (int k = 0; k < kGK / 16; ++k) {
        // +2 in the address field = 32 bytes = 16 bf16 along K
        tc_mma_f16(tmem, da + 2 * k, dh + 2 * k, idesc, (kb | k) != 0);
        tc_mma_f16(tmem, da + 2 * k, dl + 2 * k, idesc, 1u);
      }
      tc_commit(&s.empty[st]);
    }
    tc_commit(&s.done);  // also when stopped early: retires what was issued
  }
  __syncwarp();
  // Accumulator ready (or the issuing stopped): every warp waits on `done`.
  const bool ok = gemm_wait(&s.done, 0);
  tc_fence_after_sync();
  __syncthreads();
  if (ok && !s.failed) {
    const int row = m0 + warp * 32 + lane;
    const float b = (bias && row < n_rows) ? __uint_as_float((uint32_t)bias[row] << 16) : 0.f;
#pragma unroll 1
    for (int c0 = 0; c0 < kGN; c0 += 16) {
      float v[16];
      tmem_ld16(tmem + ((uint32_t)(warp * 32) << 16) + (uint32_t)c0, v);
      if (row < n_rows) {
#pragma unroll
        for (int j = 0; j < 16; ++j) {
          const int tok = n0 + c0 + j;
          if (tok < n_tok) Y[(size_t)tok * ldy + row] = v[j] + b;
        }
      }
    }
  } else if (threadIdx.x == 0) {
    atomicExch(err, 1);
  }
  tc_fence_before_sync();
  __syncthreads();
  if (warp == 0) tmem_dealloc(tmem, kGN);
}

// ------------------------------------------------------- small operators

__device__ __forceinline__ uint16_t bf16_bits(float f) {
  __nv_bfloat16 b = __float2bfloat16_rn(f);
  return *reinterpret_cast<uint16_t*>(&b);
}
__device__ __forceinline__ float bf16_val(uint16_t h) { return __uint_as_float((uint32_t)h << 16); }

// v -> (bf16(v), bf16(v - bf16(v)))
__device__ __forceinline__ void split_store(float v, uint16_t* hi, uint16_t* lo, size_t i) {
  const uint16_t h = bf16_bits(v);
  hi[i] = h;
  lo[i] = bf16_bits(v - bf16_val(h));
}

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

// [xh, xl][t] = split(x[t] * w / sqrt(mean(x[t]^2) + eps))
__global__ void rmsnorm_split_kernel(const float* __restrict__ x, const uint16_t* __restrict__ w,
                                     int H, float eps, uint16_t* __restrict__ xh,
                                     uint16_t* __restrict__ xl) {
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
    split_store(xr[i] * r * bf16_val(w[i]), xh, xl, (size_t)t * H + i);
}

// RoPE on the packed q/k rows of each token, q to qout, K/V (bf16) into the
// cache at the token's (slot, position).  Mirrors the decode step's epilogue.
__global__ void rope_kv_kernel(const float* __restrict__ y, int ldy, const int32_t* __restrict__ slot,
                               const int32_t* __restrict__ pos, ModelDev m, int layer,
                               float* __restrict__ qout) {
  const int t = blockIdx.x;
  const int d = m.head_dim, G = m.group, half = d >> 1;
  const int npairs = qkv_rows(m.n_q, m.n_kv, d) >> 1;
  const int p = pos[t], sl = slot[t];
  for (int pi = threadIdx.x; pi < npairs; pi += blockDim.x) {
    const int r = 2 * pi;
    float y0 = y[(size_t)t * ldy + r], y1 = y[(size_t)t * ldy + r + 1];
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
      const size_t off =
          ((((size_t)sl * m.n_layers + layer) * m.n_kv + head) * (size_t)m.max_seq + p) * (size_t)d;
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
                        int layer, uint16_t* __restrict__ xh, uint16_t* __restrict__ xl) {
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
  const size_t head_off = (((size_t)sl * m.n_layers + layer) * m.n_kv + g) * (size_t)m.max_seq * d;
  const uint16_t* K = m.kcache + head_off;
  const uint16_t* V = m.vcache + head_off;
  const int n_keys = p0 + nt;  // keys 0 .. last position of the tile
  float* xb = xbs + warp * kAttnXbStride;
  for (int kb = 0; kb < n_keys; kb += kPAKeys) {
    const int nk = min(kPAKeys, n_keys - kb);
    __syncthreads();
    const int vec = nk * d / 8;  // 16-byte pieces
    for (int i = threadIdx.x; i < vec; i += blockDim.x) {
      reinterpret_cast<uint4*>(ks)[i] = __ldcg(reinterpret_cast<const uint4*>(K + (size_t)kb * d) + i);
      reinterpret_cast<uint4*>(vs)[i] = __ldcg(reinterpret_cast<const uint4*>(V + (size_t)kb * d) + i);
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
    for (int i = 0; i < DPL; ++i) split_store(st.o[h][i] * inv, xh, xl, row + (size_t)h * d + lane * DPL + i);
  }
}

// x[t] += y[t]
__global__ void residual_kernel(float* __restrict__ x, const float* __restrict__ y, int H, int ldy) {
  const int t = blockIdx.x;
  for (int i = threadIdx.x; i < H; i += blockDim.x) x[(size_t)t * H + i] += y[(size_t)t * ldy + i];
}

// [xh, xl][t][j] = split(silu(gate_j) * up_j); gate/up interleaved in y.
__global__ void swiglu_split_kernel(const float* __restrict__ y, int ldy, int F,
                                    uint16_t* __restrict__ xh, uint16_t* __restrict__ xl) {
  const int t = blockIdx.x;
  for (int j = threadIdx.x; j < F; j += blockDim.x) {
    const float g = y[(size_t)t * ldy + 2 * j], u = y[(size_t)t * ldy + 2 * j + 1];
    split_store(g / (1.0f + expf(-g)) * u, xh, xl, (size_t)t * F + j);
  }
}

// ------------------------------------------------------------------ host

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

// 2-D bf16 tensor [rows][cols] (row-major), boxes of 64 columns x 128 rows,
// 128-byte swizzle, zero fill outside.
bool make_map(CUtensorMap* map, const void* base, int rows, int cols) {
  auto fn = encode_fn();
  if (!fn) return false;
  const cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
  const cuuint64_t strides[1] = {(cuuint64_t)cols * 2};
  const cuuint32_t box[2] = {(cuuint32_t)kGK, 128u};
  const cuuint32_t estr[2] = {1u, 1u};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box,
            estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

std::string gemm(const uint16_t* W, int n_rows, int K, const uint16_t* xh, const uint16_t* xl,
                 int n_tok, float* Y, int ldy, const uint16_t* bias, int32_t* err, cudaStream_t st) {
  CUtensorMap mw, mh, ml;
  if (!make_map(&mw, W, n_rows, K) || !make_map(&mh, xh, n_tok, K) || !make_map(&ml, xl, n_tok, K))
    return "cuTensorMapEncodeTiled failed";
  const dim3 grid((n_rows + kGM - 1) / kGM, (n_tok + kGN - 1) / kGN);
  gemm_wx_kernel<<<grid, 128, kGemmSmemBytes, st>>>(mw, mh, ml, n_rows, n_tok, K, Y, ldy, bias, err);
  const cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? "" : std::string("GEMM launch: ") + cudaGetErrorString(e);
}

template <int DPL, int G>
std::string launch_attn(dim3 grid, cudaStream_t st, const float* q, const int32_t* tiles,
                        const ModelDev& m, int layer, uint16_t* xh, uint16_t* xl) {
  const size_t smem = (size_t)2 * kPAKeys * DPL * 32 * 2 + (size_t)kPAWarps * kAttnXbStride * 4;
  auto k = prefill_attn_kernel<DPL, G>;
  cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  k<<<grid, kPAWarps * 32, smem, st>>>(q, tiles, m, layer, xh, xl);
  const cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? "" : std::string("attention launch: ") + cudaGetErrorString(e);
}

std::string attn(dim3 grid, cudaStream_t st, const float* q, const int32_t* tiles, const ModelDev& m,
                 int layer, uint16_t* xh, uint16_t* xl) {
  const int G = m.group;
  if (m.head_dim == 128) {
    if (G == 1) return launch_attn<4, 1>(grid, st, q, tiles, m, layer, xh, xl);
    if (G == 2) return launch_attn<4, 2>(grid, st, q, tiles, m, layer, xh, xl);
    if (G == 4) return launch_attn<4, 4>(grid, st, q, tiles, m, layer, xh, xl);
  } else {
    if (G == 1) return launch_attn<2, 1>(grid, st, q, tiles, m, layer, xh, xl);
    if (G == 2) return launch_attn<2, 2>(grid, st, q, tiles, m, layer, xh, xl);
    if (G == 4) return launch_attn<2, 4>(grid, st, q, tiles, m, layer, xh, xl);
    if (G == 7) return launch_attn<2, 7>(grid, st, q, tiles, m, layer, xh, xl);
    if (G == 8) return launch_attn<2, 8>(grid, st, q, tiles, m, layer, xh, xl);
  }
  return "unsupported query heads per KV head";
}

}  // namespace

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
      {(void**)&sc->xl, T * xcols * 2},     {(void**)&sc->meta, (3 * T + 4 * T + 16) * 4},
      {(void**)&sc->err, 16}};
  for (auto& a : allocs) {
    const cudaError_t e = cudaMalloc(a.p, a.bytes);
    if (e != cudaSuccess) return std::string("prefill scratch: ") + cudaGetErrorString(e);
    owned->push_back(*a.p);
  }
  cudaMemset(sc->err, 0, 16);
  if (cudaFuncSetAttribute(gemm_wx_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           (int)kGemmSmemBytes) != cudaSuccess)
    return "GEMM shared memory attribute";
  sc->max_tokens = max_tokens;
  return "";
}

std::string prefill_run(const ModelDev& m, const PrefillWeights& w, PrefillScratch& sc,
                        cudaStream_t st, const int32_t* tokens_dev, const int32_t* offsets_host,
                        int n_req) {
  const int H = m.hidden, F = m.ffn, d = m.head_dim, qd = m.n_q * d, L = m.n_layers;
  const int qkvR = qkv_rows(m.n_q, m.n_kv, d);
  const int ldy = std::max(std::max(qkvR, 2 * F), H);
  // every position but each prompt's last, as (request, position) in order
  std::vector<int> tok_src, slot, pos;
  for (int r = 0; r < n_req; ++r)
    for (int p = 0; p + 1 < offsets_host[r + 1] - offsets_host[r]; ++p) {
      tok_src.push_back(offsets_host[r] + p);
      slot.push_back(r);
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
    const int ntiles = (int)tiles.size() / 4;
    int32_t* d_src = sc.meta;
    int32_t* d_slot = sc.meta + T;
    int32_t* d_pos = sc.meta + 2 * T;
    int32_t* d_tiles = sc.meta + 3 * (size_t)sc.max_tokens;
    if (cudaMemcpyAsync(sc.meta, meta.data(), meta.size() * 4, cudaMemcpyHostToDevice, st) != cudaSuccess ||
        cudaMemcpyAsync(d_tiles, tiles.data(), tiles.size() * 4, cudaMemcpyHostToDevice, st) != cudaSuccess)
      return "prefill metadata upload";
    embed_kernel<<<T, 256, 0, st>>>(m.embed, tokens_dev, d_src, H, m.vocab, sc.x, m.status);
    for (int l = 0; l < L; ++l) {
      rmsnorm_split_kernel<<<T, 256, 0, st>>>(sc.x, m.attn_norm + (size_t)l * H, H, m.rms_eps, sc.xh, sc.xl);
      const uint16_t* bias = m.qkv_bias ? m.bqkv + (size_t)l * qkvR : nullptr;
      if (!(e = gemm(w.qkv[l], qkvR, H, sc.xh, sc.xl, T, sc.y, ldy, bias, sc.err, st)).empty()) return e;
      rope_kv_kernel<<<T, 256, 0, st>>>(sc.y, ldy, d_slot, d_pos, m, l, sc.q);
      if (!(e = attn(dim3(ntiles, m.n_kv), st, sc.q, d_tiles, m, l, sc.xh, sc.xl)).empty()) return e;
      if (!(e = gemm(w.o[l], H, qd, sc.xh, sc.xl, T, sc.y, ldy, nullptr, sc.err, st)).empty()) return e;
      residual_kernel<<<T, 256, 0, st>>>(sc.x, sc.y, H, ldy);
      rmsnorm_split_kernel<<<T, 256, 0, st>>>(sc.x, m.ffn_norm + (size_t)l * H, H, m.rms_eps, sc.xh, sc.xl);
      if (!(e = gemm(w.gu[l], 2 * F, H, sc.xh, sc.xl, T, sc.y, ldy, nullptr, sc.err, st)).empty()) return e;
      swiglu_split_kernel<<<T, 256, 0, st>>>(sc.y, ldy, F, sc.xh, sc.xl);
      if (!(e = gemm(w.dn[l], H, F, sc.xh, sc.xl, T, sc.y, ldy, nullptr, sc.err, st)).empty()) return e;
      residual_kernel<<<T, 256, 0, st>>>(sc.x, sc.y, H, ldy);
    }
    const cudaError_t ce = cudaGetLastError();
    if (ce != cudaSuccess) return std::string("prefill launch: ") + cudaGetErrorString(ce);
  }
  // The GEMM kernel records a wait that ran out (never expected) in sc.err.
  int32_t herr = 0;
  if (cudaMemcpyAsync(&herr, sc.err, 4, cudaMemcpyDeviceToHost, st) != cudaSuccess ||
      cudaStreamSynchronize(st) != cudaSuccess)
    return std::string("prefill: ") + cudaGetErrorString(cudaGetLastError());
  if (herr) return "prefill GEMM: a pipeline wait timed out";
  return "";
}

}  // namespace mk
