// attention.cu -- standalone split-KV grouped-query decode attention.
//
// One KV head and its G query heads against n cached keys: the keys are cut
// into `splits` contiguous blocks, one CTA each.  A CTA stages its keys 64 at
// a time in shared memory (cp.async, double-buffered, so the next block
// loads while this one is used); each warp keeps an online softmax (running
// maximum, running sum, rescaled output) over four keys per block; the CTA
// merges its warps and writes its block's partial (unnormalised output at
// the block maximum, the maximum, the sum) to the workspace; the last CTA to
// finish merges the blocks ("Hạt nhân là gì ...": the online
// softmax gives the exact softmax up to rounding; "LLM高速化勉強会資料" slides
// 11-13, 28; "Crear desde cero ..." §3.4).  The same math runs inside the
// persistent decode kernel's attention tasks (attn_math.cuh).
#include <cuda_runtime.h>
#include <math.h>

#include <string>

#include "../../include/mk.h"
#include "attn_math.cuh"
#include "mk_internal.h"

namespace mk {

void set_last_error(const char* msg);  // api.cu: the message mk_last_error(NULL) returns

constexpr int kAttnOpWarps = 16;
constexpr int kAttnOpKeys = 64;  // keys per staged block
constexpr int kAttnOpMaxG = 8;
constexpr size_t kAttnTicketBytes = 256;  // the merge ticket, padded

// Workspace: [ticket u32, padded to 256 B][splits][G][attn_part_stride(d)] floats.
size_t attn_op_workspace_bytes(int G, int d, int splits) {
  return kAttnTicketBytes + (size_t)splits * G * attn_part_stride(d) * sizeof(float);
}

__device__ __forceinline__ void op_cp_async(void* dst, const void* src, bool b16) {
  if (b16)
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(
                     static_cast<uint32_t>(__cvta_generic_to_shared(dst))), "l"(src) : "memory");
  else
    asm volatile("cp.async.ca.shared.global [%0], [%1], 8;" ::"r"(
                     static_cast<uint32_t>(__cvta_generic_to_shared(dst))), "l"(src) : "memory");
}
__device__ __forceinline__ void op_cp_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void op_cp_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

// Dynamic shared memory of the op: two K/V blocks and the warps' softmax
// scratch while streaming; afterwards the warps' states reuse the bytes.
template <int DPL, int G>
constexpr size_t attn_op_smem() {
  constexpr size_t loop = (size_t)2 * 2 * kAttnOpKeys * DPL * 32 * 2 + (size_t)kAttnOpWarps * kAttnXbStride * 4;
  constexpr size_t merge = (size_t)kAttnOpWarps * G * (DPL * 32 + 4) * 4;
  return loop > merge ? loop : merge;
}

template <int DPL, int G>
__global__ void __launch_bounds__(kAttnOpWarps * 32, 1)
    attn_decode_kernel(const float* __restrict__ q, const uint16_t* __restrict__ K,
                       const uint16_t* __restrict__ V, int n, float scale, int splits,
                       uint8_t* __restrict__ ws, float* __restrict__ out) {
  constexpr int d = DPL * 32, PS = d + 4;
  constexpr int kBuf = 2 * kAttnOpKeys * d;  // bf16 elements per buffer (K then V)
  extern __shared__ __align__(16) uint8_t op_raw[];
  uint16_t* kvbuf = reinterpret_cast<uint16_t*>(op_raw);
  float* xbs = reinterpret_cast<float*>(kvbuf + 2 * kBuf);
  __shared__ int last;
  unsigned int* ticket = reinterpret_cast<unsigned int*>(ws);
  float* part = reinterpret_cast<float*>(ws + kAttnTicketBytes);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, split = blockIdx.x;
  const int chunk = (n + splits - 1) / splits;
  const int k0 = min(n, split * chunk), k1 = min(n, k0 + chunk);

  AttnState<DPL, G> st;
  attn_init<DPL, G>(st, q, d, scale, lane);
  float* xb = xbs + warp * kAttnXbStride;
  const bool b16 = ((reinterpret_cast<uintptr_t>(K) | reinterpret_cast<uintptr_t>(V)) & 15u) == 0;
  const int nblk = (k1 - k0 + kAttnOpKeys - 1) / kAttnOpKeys;
  auto issue = [&](int b) {
    const int kb = k0 + b * kAttnOpKeys, nk = min(kAttnOpKeys, k1 - kb);
    uint16_t* dst = kvbuf + (b & 1) * kBuf;
    const int per = b16 ? 8 : 4;  // bf16 elements per copy
    const int pieces = nk * d / per;
    for (int i = threadIdx.x; i < pieces; i += blockDim.x) {
      op_cp_async(dst + i * per, K + (size_t)kb * d + i * per, b16);
      op_cp_async(dst + kAttnOpKeys * d + i * per, V + (size_t)kb * d + i * per, b16);
    }
  };
  if (nblk > 0) issue(0);
  op_cp_commit();
  for (int b = 0; b < nblk; ++b) {
    if (b + 1 < nblk) issue(b + 1);
    op_cp_commit();
    op_cp_wait<1>();
    __syncthreads();
    const int kb = k0 + b * kAttnOpKeys, nk = min(kAttnOpKeys, k1 - kb);
    const uint16_t* ks = kvbuf + (b & 1) * kBuf;
    const uint16_t* vs = ks + kAttnOpKeys * d;
    // four consecutive keys per warp
    for (int j0 = 4 * warp; j0 < nk; j0 += 4 * kAttnOpWarps) {
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
    __syncthreads();  // buffer b & 1 is refilled by block b + 2
  }
  op_cp_wait<0>();
  __syncthreads();
  float* buf = reinterpret_cast<float*>(op_raw);  // [warps][G][PS], reuses the key buffers
#pragma unroll
  for (int h = 0; h < G; ++h) {
#pragma unroll
    for (int i = 0; i < DPL; ++i) buf[(warp * G + h) * PS + lane * DPL + i] = st.o[h][i];
    if (lane == 0) {
      buf[(warp * G + h) * PS + d] = st.mx[h];
      buf[(warp * G + h) * PS + d + 1] = st.l[h];
    }
  }
  __syncthreads();
  // This block's partial: the warps merged at their common maximum.
  float* mine = part + (size_t)split * G * PS;
  for (int idx = threadIdx.x; idx < G * (d + 2); idx += blockDim.x) {
    const int h = idx / (d + 2), i = idx - h * (d + 2);
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < kAttnOpWarps; ++w) M = fmaxf(M, buf[(w * G + h) * PS + d]);
    float val = 0.f;
    if (M != -INFINITY) {
#pragma unroll
      for (int w = 0; w < kAttnOpWarps; ++w) {
        const float mw = buf[(w * G + h) * PS + d];
        if (mw == -INFINITY) continue;
        val = fmaf(__expf(mw - M), i < d ? buf[(w * G + h) * PS + i] : buf[(w * G + h) * PS + d + 1], val);
      }
    }
    mine[h * PS + i] = i == d ? M : val;
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    __threadfence();
    last = atomicAdd(ticket, 1u) == (unsigned)splits - 1u;
  }
  __syncthreads();
  if (!last) return;
  __threadfence();
  // Last block: merge every block's partial and normalise.
  for (int idx = threadIdx.x; idx < G * d; idx += blockDim.x) {
    const int h = idx / d, i = idx - h * d;
    float M = -INFINITY;
    for (int s = 0; s < splits; ++s) M = fmaxf(M, __ldcg(part + ((size_t)s * G + h) * PS + d));
    float num = 0.f, den = 0.f;
    for (int s = 0; s < splits; ++s) {
      const float* ps = part + ((size_t)s * G + h) * PS;
      const float ls = __ldcg(ps + d + 1);
      if (ls == 0.f) continue;
      const float c = __expf(__ldcg(ps + d) - M);
      num = fmaf(c, __ldcg(ps + i), num);
      den = fmaf(c, ls, den);
    }
    out[h * d + i] = num / den;
  }
  // Leave the ticket at zero for the next call on this workspace.
  if (threadIdx.x == 0) *ticket = 0u;
}

template <int DPL>
static cudaError_t launch_attn_g(int G, const float* q, const uint16_t* K, const uint16_t* V,
                                 int n, float scale, int splits, uint8_t* ws, float* out,
                                 cudaStream_t st) {
  const dim3 grid(splits), block(kAttnOpWarps * 32);
#define MK_OP(G_)                                                                          \
  {                                                                                        \
    constexpr size_t sm = attn_op_smem<DPL, G_>();                                         \
    cudaError_t e = cudaFuncSetAttribute(attn_decode_kernel<DPL, G_>,                      \
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm); \
    if (e != cudaSuccess) return e;                                                        \
    attn_decode_kernel<DPL, G_><<<grid, block, sm, st>>>(q, K, V, n, scale, splits, ws, out); \
    break;                                                                                 \
  }
  switch (G) {
    case 1: MK_OP(1)
    case 2: MK_OP(2)
    case 4: MK_OP(4)
    case 7: MK_OP(7)
    case 8: MK_OP(8)
    default: return cudaErrorInvalidValue;
  }
#undef MK_OP
  return cudaGetLastError();
}

// Checks the arguments of the attention op; returns 0 or an MK_ERR_* code.
int attn_op_check(const float* q, const void* k, const void* v, int n, int G, int d, int splits,
                  const float* out) {
  if (!q || !k || !v || !out) return MK_ERR_INVALID_ARG;
  if (n < 1 || splits < 1 || splits > 4096) return MK_ERR_INVALID_ARG;
  if (d != 64 && d != 128) return MK_ERR_UNSUPPORTED;
  if (!(G == 1 || G == 2 || G == 4 || G == 7 || G == 8)) return MK_ERR_UNSUPPORTED;
  if ((reinterpret_cast<uintptr_t>(k) | reinterpret_cast<uintptr_t>(v)) & 7u) return MK_ERR_INVALID_ARG;
  return MK_OK;
}

cudaError_t launch_attn_op(const float* q, const void* k, const void* v, int n, int G, int d,
                           int splits, void* ws, float* out, cudaStream_t st) {
  const float scale = (float)(1.0 / sqrt((double)d));
  const uint16_t* K = static_cast<const uint16_t*>(k);
  const uint16_t* V = static_cast<const uint16_t*>(v);
  uint8_t* w = static_cast<uint8_t*>(ws);
  return d == 128 ? launch_attn_g<4>(G, q, K, V, n, scale, splits, w, out, st)
                  : launch_attn_g<2>(G, q, K, V, n, scale, splits, w, out, st);
}

}  // namespace mk

extern "C" size_t mk_attention_workspace_bytes(int n_q_per_kv, int head_dim, int splits) {
  if (n_q_per_kv < 1 || n_q_per_kv > mk::kAttnOpMaxG || head_dim < 1 || splits < 1) return 0;
  return mk::attn_op_workspace_bytes(n_q_per_kv, head_dim, splits);
}

extern "C" int mk_attention_decode(const float* q_dev, const void* k_dev, const void* v_dev,
                                   int n_keys, int n_q_per_kv, int head_dim, int splits,
                                   void* workspace_dev, float* out_dev, void* stream) {
  int rc = mk::attn_op_check(q_dev, k_dev, v_dev, n_keys, n_q_per_kv, head_dim, splits, out_dev);
  if (rc) return rc;
  if (!workspace_dev || (reinterpret_cast<uintptr_t>(workspace_dev) & 15u)) return MK_ERR_INVALID_ARG;
  cudaError_t e = mk::launch_attn_op(q_dev, k_dev, v_dev, n_keys, n_q_per_kv, head_dim, splits,
                                     workspace_dev, out_dev, static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? MK_OK : MK_ERR_CUDA;
}

// ---------------------------------------------------------------------------
// Allocation-free variant.  Some callers cannot allocate device memory at all:
// a plugin inside a host that owns every byte of device memory through its
// own pool, a real-time loop that must never enter an allocator, or code that
// is only allowed to touch buffers it was handed.  For them the workspace of
// the op above lives in a fixed array compiled into this library.  Every GPU
// that loads the library holds the array until the process exits.
namespace mk {
namespace {

constexpr int kNoAllocMaxSplits = 64;   // key blocks
constexpr int kNoAllocMaxG = 8;         // query heads per KV head
constexpr int kNoAllocMaxHeadDim = 128;
constexpr size_t kNoAllocBytes =
    kAttnTicketBytes + (size_t)kNoAllocMaxSplits * kNoAllocMaxG * (kNoAllocMaxHeadDim + 4) * sizeof(float);

// The shared scratch: 270,592 bytes per device.
static __device__ __align__(256) uint8_t g_attn_noalloc_scratch[kNoAllocBytes];

}  // namespace
}  // namespace mk

extern "C" int mk_attention_decode_noalloc(const float* q_dev, const void* k_dev, const void* v_dev,
                                           int n_keys, int n_q_per_kv, int head_dim, int splits,
                                           float* out_dev, void* stream) {
  using namespace mk;
  int rc = attn_op_check(q_dev, k_dev, v_dev, n_keys, n_q_per_kv, head_dim, splits, out_dev);
  if (rc) return rc;
  const size_t need = attn_op_workspace_bytes(n_q_per_kv, head_dim, splits);
  if (need > kNoAllocBytes) {
    set_last_error(("mk_attention_decode_noalloc: needs " + std::to_string(need) +
                    " bytes of scratch, the static array holds " + std::to_string(kNoAllocBytes) +
                    " (at most 64 splits for 8 query heads per KV head at head_dim 128)").c_str());
    return MK_ERR_INVALID_ARG;
  }
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  // The array's name in host code is only a stand-in for it: its device
  // address in the current device's context is looked up on every call
  // (cheap, allocates nothing), so a context that was torn down and made
  // again never sees a stale address.  The first call on a device loads this
  // library's device code there; make it before any stream capture.
  void* scratch = nullptr;
  if (cudaGetSymbolAddress(&scratch, g_attn_noalloc_scratch) != cudaSuccess || !scratch) {
    cudaGetLastError();
    set_last_error("mk_attention_decode_noalloc: cudaGetSymbolAddress failed");
    return MK_ERR_CUDA;
  }
  // The merge ticket must start at zero; the partials need no clearing (each
  // split writes its own before the ticket lets the last one read them).
  if (cudaMemsetAsync(scratch, 0, kAttnTicketBytes, st) != cudaSuccess) return MK_ERR_CUDA;
  cudaError_t e = launch_attn_op(q_dev, k_dev, v_dev, n_keys, n_q_per_kv, head_dim, splits,
                                 scratch, out_dev, st);
  return e == cudaSuccess ? MK_OK : MK_ERR_CUDA;
}
