// flash_attn.cu -- causal GQA attention of the prompt prefill on the tensor
// cores ("LLM高速化勉強会資料" slides 11-13 and "Hạt nhân là gì ...", the
// FlashAttention section: the keys in tiles, scores and output accumulated on
// chip, an online softmax, key tiles past a query's position skipped).
//
// One CTA per (run of <= 128 consecutive prompt positions of one request, query
// head); the tile itself is fa_tile (flash_attn.cuh).  320 threads: eight
// softmax warps (two per row), the TMA warp, the MMA warp.  Every wait is bounded (2 s); a
// timeout sets the error word, and the CTA releases its tensor memory only
// once every MMA it issued has retired.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <algorithm>
#include <string>
#include <vector>

#include "../../include/mk.h"
#include "mk_internal.h"
#include "prefill.h"
#include "ptx.cuh"
#include "flash_attn.cuh"
#include "tc.cuh"

namespace mk {

PFN_cuTensorMapEncodeTiled_v12000 prefill_encode_fn();  // prefill.cu

namespace {

constexpr int kFaThreads = kFaMinThreads;  // 8 softmax warps, the TMA warp, the MMA warp
constexpr uint64_t kFaWaitNs = 2000000000ull;
static_assert(kFaRows == kFaTileRows, "tile rows");

struct FaParams {
  ModelDev m;
  const int32_t* tiles;  // [n][4]: first block token, rows, KV slot, first position
  const float* q;        // [T][ldq] rotated queries (fp32)
  int ldq;
  uint16_t* oh;          // [T][ldo] output, three bf16 parts
  uint16_t* om;
  uint16_t* ol;
  int ldo;
  int layer;
  float qscale;          // attention scale * log2(e)
  int32_t* err;          // [0] first error code, [1] detail
};

struct FaSmem {
  FaBuffers buf;
  FaBarriers bar;
  uint32_t tmem;
  int32_t abort_flag;
  int32_t tmem_ok;
};

// Bounded wait that ignores the abort flag (the teardown's drain).
__device__ __forceinline__ bool fa_drain(uint64_t* bar, uint32_t parity) {
  const uint64_t t0 = globaltimer_ns();
  while (!mbar_try_wait(bar, parity))
    if (globaltimer_ns() - t0 > 200000000ull) return false;
  return true;
}

template <int D>
__global__ void __launch_bounds__(kFaThreads, 1)
    flash_attn_kernel(const __grid_constant__ CUtensorMap mk0, const __grid_constant__ CUtensorMap mk1,
                      const __grid_constant__ CUtensorMap mv0, const __grid_constant__ CUtensorMap mv1,
                      const __grid_constant__ FaParams p) {
  extern __shared__ __align__(16) uint8_t fa_raw[];
  const uint32_t base = smem_u32(fa_raw);
  FaSmem& s = *reinterpret_cast<FaSmem*>(fa_raw + (((base + 1023u) & ~1023u) - base));
  const int warp = threadIdx.x >> 5;
  if (threadIdx.x == 0) {
    fa_init_barriers(s.bar);
    s.abort_flag = 0;
    s.tmem_ok = 0;
    fence_barrier_init();
  }
  if (warp == 0) {
    tmem_alloc(&s.tmem, kFaTmemCols);
    tmem_relinquish();
  }
  tc_fence_before_sync();
  __syncthreads();
  tc_fence_after_sync();
  const int* tl = p.tiles + 4 * blockIdx.y;
  FaJob j;
  j.mk0 = &mk0; j.mk1 = &mk1; j.mv0 = &mv0; j.mv1 = &mv1;
  j.q = p.q; j.ldq = p.ldq;
  j.oh = p.oh; j.om = p.om; j.ol = p.ol; j.ldo = p.ldo;
  j.layer = p.layer; j.qscale = p.qscale;
  j.t0 = tl[0]; j.nrows = tl[1]; j.slot = tl[2]; j.p0 = tl[3]; j.h = blockIdx.x;
  auto wait = [&](uint64_t* bar, uint32_t parity, int where) -> bool {
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = globaltimer_ns();
    while (!mbar_try_wait(bar, parity)) {
      if (*(volatile int32_t*)&s.abort_flag) return false;
      if (globaltimer_ns() - t0 > kFaWaitNs) {
        if (atomicCAS(p.err, 0, MK_ERR_TIMEOUT) == 0) p.err[1] = where;
        *(volatile int32_t*)&s.abort_flag = 1;
        return false;
      }
    }
    return true;
  };
  fa_tile<D>(p.m, j, s.buf, s.bar, s.tmem, 0u, wait);
  // ------------------------------------------------------------ teardown
  tc_fence_before_sync();
  __syncthreads();
  if (threadIdx.x == 0) {
    // every MMA issued has retired once `fin` arrived; after an abort, let the
    // loads still in flight land before the CTA exits
    s.tmem_ok = fa_drain(&s.bar.fin, 0) ? 1 : 0;
    if (*(volatile int32_t*)&s.abort_flag)
      for (int i = 0; i < 2; ++i) {
        if (s.bar.armed_k[i] != 0xffffffffu) fa_drain(&s.bar.k_full[i], (s.bar.armed_k[i] >> 1) & 1);
        if (s.bar.armed_v[i] != 0xffffffffu) fa_drain(&s.bar.v_full[i], (s.bar.armed_v[i] >> 1) & 1);
      }
  }
  __syncthreads();
  tc_fence_after_sync();
  if (warp == 0 && s.tmem_ok) tmem_dealloc(s.tmem, kFaTmemCols);
}

bool fa_make_map(CUtensorMap* map, const void* base, uint64_t rows, int d) {
  auto fn = prefill_encode_fn();
  if (!fn) return false;
  const cuuint64_t dims[2] = {64u, (cuuint64_t)rows};
  const cuuint64_t strides[1] = {(cuuint64_t)d * 2};
  const cuuint32_t box[2] = {64u, (cuuint32_t)kFaKeys};
  const cuuint32_t estr[2] = {1u, 1u};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box,
            estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

size_t flash_attn_smem_bytes() { return sizeof(FaSmem) + 1024; }

std::string flash_attn_prepare(const ModelDev& m, FaMaps* fm) {
  if (fm->ready) return "";
  const int d = m.head_dim;
  if (d != 64 && d != 128) return "flash attention: head_dim must be 64 or 128";
  // every row of the page pool (a contiguous cache is the one-page-per-slot case)
  const uint64_t rows = (uint64_t)m.kv_pool * m.n_layers * m.n_kv * (uint64_t)m.kv_page;
  const uint8_t* kb = reinterpret_cast<const uint8_t*>(m.kcache);
  const uint8_t* vb = reinterpret_cast<const uint8_t*>(m.vcache);
  // the second half of a 128-dim row starts 128 bytes in (the same rows)
  if (!fa_make_map(&fm->k0, kb, rows, d) || !fa_make_map(&fm->v0, vb, rows, d) ||
      !fa_make_map(&fm->k1, d == 128 ? kb + 128 : kb, rows, d) ||
      !fa_make_map(&fm->v1, d == 128 ? vb + 128 : vb, rows, d))
    return "flash attention: tensor map";
  auto set = [](const void* k) {
    return cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                (int)flash_attn_smem_bytes());
  };
  if (set((const void*)flash_attn_kernel<64>) != cudaSuccess ||
      set((const void*)flash_attn_kernel<128>) != cudaSuccess)
    return "flash attention: shared memory attribute";
  fm->ready = true;
  return "";
}

std::string flash_attn_launch(const ModelDev& m, const FaMaps& fm, const int32_t* tiles_dev,
                              int n_tiles, int layer, const float* q, int ldq, uint16_t* oh,
                              uint16_t* om, uint16_t* ol, int ldo, int32_t* err, cudaStream_t st) {
  if (n_tiles <= 0) return "";
  FaParams p{};
  p.m = m;
  p.tiles = tiles_dev;
  p.q = q;
  p.ldq = ldq;
  p.oh = oh;
  p.om = om;
  p.ol = ol;
  p.ldo = ldo;
  p.layer = layer;
  p.qscale = m.attn_scale * 1.4426950408889634f;
  p.err = err;
  const dim3 grid(m.n_q, n_tiles);
  if (m.head_dim == 128)
    flash_attn_kernel<128><<<grid, kFaThreads, flash_attn_smem_bytes(), st>>>(fm.k0, fm.k1, fm.v0, fm.v1, p);
  else
    flash_attn_kernel<64><<<grid, kFaThreads, flash_attn_smem_bytes(), st>>>(fm.k0, fm.k1, fm.v0, fm.v1, p);
  const cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? "" : std::string("flash attention launch: ") + cudaGetErrorString(e);
}

}  // namespace mk
