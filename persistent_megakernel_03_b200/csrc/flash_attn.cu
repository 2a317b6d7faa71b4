// flash_attn.cu -- causal GQA attention of the prompt prefill on the tensor
// cores ("LLM高速化勉強会資料" slides 11-13 and "Hạt nhân là gì ...", the
// FlashAttention section: the keys in tiles, scores and output accumulated on
// chip, an online softmax, key tiles past a query's position skipped).
//
// One CTA per (run of <= 128 consecutive prompt positions of one request, query
// head h).  Scores S = Q K^T and the output O = P V are tcgen05.mma products in
// tensor memory (fp32 accumulate):
//   Q  the run's rotated queries times scale * log2(e), as two bf16 parts
//      (hi + lo carries 16 significant bits of the fp32 value), K-major;
//   K, V  64-key tiles of the bf16 cache (exact), brought by 2-D TMA with the
//      128-byte swizzle; K is the K-major B operand of S, V the MN-major B
//      operand of O;
//   P  2^(S - m) per row as two bf16 parts, written to shared memory by the
//      softmax threads (one row each) in the K-major swizzled layout.
// The running maximum m of a row moves only when a tile's maximum exceeds it
// by more than 8 (powers of two): then O's row in tensor memory and the
// running sum are rescaled; otherwise the probabilities stay below 2^8 and
// the final O / l is the same.  The output is written as the O projection's
// three bf16 parts.
//
// Warps 0-3: softmax and epilogue (row = thread = TMEM lane); warp 4 lane 0:
// TMA loads of K/V tiles (two stages); warp 5 lane 0: tcgen05.mma issue.
// Two score buffers let S of tile j+1 run while the softmax works on tile j.
// Every mbarrier wait is bounded; a timeout sets the error word, and the CTA
// releases its tensor memory only once every MMA it issued has retired.
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
#include "tc.cuh"

namespace mk {

PFN_cuTensorMapEncodeTiled_v12000 prefill_encode_fn();  // prefill.cu

namespace {

constexpr int kFaRows = kFaTileRows;  // query rows per CTA (the MMA's M)
constexpr int kFaKeys = 64;      // keys per tile
constexpr int kFaThreads = 192;  // 4 softmax warps, the TMA warp, the MMA warp
constexpr uint32_t kFaTmemCols = 256;  // two 64-column score buffers + O (<= 128 columns)
constexpr uint64_t kFaWaitNs = 2000000000ull;

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

struct __align__(1024) FaSmem {
  uint8_t q[2][2][kFaRows * 64 * 2];       // [part][64-dim half] 128 rows x 64 dims
  uint8_t k[2][2][kFaKeys * 64 * 2];       // [stage][half] 64 keys x 64 dims
  uint8_t v[2][2][kFaKeys * 64 * 2];
  uint8_t p[2][2][kFaRows * kFaKeys * 2];  // [buffer][part] 128 rows x 64 keys
  uint64_t kv_full[2], kv_empty[2], s_full[2], p_full[2], o_done, fin;
  uint32_t tmem;
  int32_t abort_flag;
  int32_t tmem_ok;
  uint32_t armed[2];
};

__device__ __forceinline__ void fa_fail(const FaParams& p, FaSmem& s, int detail) {
  if (atomicCAS(p.err, 0, MK_ERR_TIMEOUT) == 0) p.err[1] = detail;
  *(volatile int32_t*)&s.abort_flag = 1;
}

__device__ __forceinline__ bool fa_wait(const FaParams& p, FaSmem& s, uint64_t* bar, uint32_t parity,
                                        int where) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = globaltimer_ns();
  while (!mbar_try_wait(bar, parity)) {
    if (*(volatile int32_t*)&s.abort_flag) return false;
    if (globaltimer_ns() - t0 > kFaWaitNs) {
      fa_fail(p, s, where);
      return false;
    }
  }
  return true;
}

// Bounded wait that ignores the abort flag (the teardown's drain).
__device__ __forceinline__ bool fa_drain(uint64_t* bar, uint32_t parity) {
  const uint64_t t0 = globaltimer_ns();
  while (!mbar_try_wait(bar, parity))
    if (globaltimer_ns() - t0 > 200000000ull) return false;
  return true;
}

// Byte offset of the 16-byte group holding columns [c, c + 8) of row r in a
// K-major tile with 128-byte rows and the 128-byte swizzle.
__device__ __forceinline__ uint32_t sw128_off(int r, int c) {
  return (uint32_t)r * 128u + ((uint32_t)((c >> 3) ^ (r & 7)) << 4);
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  uint32_t r;
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}
__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

// v[0..7] -> two bf16 parts (hi = RN(v), lo = RN(v - hi)), 16 bytes each.
__device__ __forceinline__ void split2x8(const float (&v)[8], uint4& hi, uint4& lo) {
  uint32_t h[4], l[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    h[i] = pack_bf16x2(v[2 * i], v[2 * i + 1]);
    l[i] = pack_bf16x2(v[2 * i] - bf16_lo(h[i]), v[2 * i + 1] - bf16_hi(h[i]));
  }
  hi = make_uint4(h[0], h[1], h[2], h[3]);
  lo = make_uint4(l[0], l[1], l[2], l[3]);
}

__device__ __forceinline__ uint16_t f2bf(float f) {
  uint16_t r;
  asm("cvt.rn.bf16.f32 %0, %1;" : "=h"(r) : "f"(f));
  return r;
}

template <int D>
__global__ void __launch_bounds__(kFaThreads, 1)
    flash_attn_kernel(const __grid_constant__ CUtensorMap mk0, const __grid_constant__ CUtensorMap mk1,
                      const __grid_constant__ CUtensorMap mv0, const __grid_constant__ CUtensorMap mv1,
                      const __grid_constant__ FaParams p) {
  constexpr int NH = D / 64;  // 64-dim halves of a head
  extern __shared__ __align__(16) uint8_t fa_raw[];
  const uint32_t base = smem_u32(fa_raw);
  FaSmem& s = *reinterpret_cast<FaSmem*>(fa_raw + (((base + 1023u) & ~1023u) - base));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int h = blockIdx.x;
  const int* tl = p.tiles + 4 * blockIdx.y;
  const int t0 = tl[0], nrows = tl[1], slot = tl[2], p0 = tl[3];
  const int g = h / p.m.group;
  const int nt = (p0 + nrows + kFaKeys - 1) / kFaKeys;  // key tiles 0 .. p0 + nrows - 1
  if (threadIdx.x == 0) {
    for (int i = 0; i < 2; ++i) {
      mbar_init(&s.kv_full[i], 1);
      mbar_init(&s.kv_empty[i], 1);
      mbar_init(&s.s_full[i], 1);
      mbar_init(&s.p_full[i], kFaRows);
      s.armed[i] = 0xffffffffu;
    }
    mbar_init(&s.o_done, 1);
    mbar_init(&s.fin, 1);
    s.abort_flag = 0;
    s.tmem_ok = 0;
    fence_barrier_init();
  }
  if (warp == 0) {
    tmem_alloc(&s.tmem, kFaTmemCols);
    tmem_relinquish();
  }
  // the run's queries, scaled, as two bf16 parts in the swizzled layout
  if (threadIdx.x < kFaRows) {
    const int r = threadIdx.x;
    const float* qr = p.q + (size_t)(t0 + r) * p.ldq + (size_t)h * D;
#pragma unroll 2
    for (int c0 = 0; c0 < D; c0 += 8) {
      float v[8];
      if (r < nrows) {
        const float4 a = __ldg(reinterpret_cast<const float4*>(qr + c0));
        const float4 b = __ldg(reinterpret_cast<const float4*>(qr + c0 + 4));
        v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w; v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
#pragma unroll
        for (int i = 0; i < 8; ++i) v[i] *= p.qscale;
      } else {
#pragma unroll
        for (int i = 0; i < 8; ++i) v[i] = 0.f;
      }
      uint4 hi, lo;
      split2x8(v, hi, lo);
      const uint32_t off = sw128_off(r, c0 & 63);
      *reinterpret_cast<uint4*>(s.q[0][c0 >> 6] + off) = hi;
      *reinterpret_cast<uint4*>(s.q[1][c0 >> 6] + off) = lo;
    }
  }
  fence_proxy_async_shared();
  tc_fence_before_sync();
  __syncthreads();
  tc_fence_after_sync();
  const uint32_t tS = s.tmem;         // score buffers: columns [0, 64), [64, 128)
  const uint32_t tO = s.tmem + 128u;  // output: columns [128, 128 + D)

  if (warp == 4) {
    // ------------------------------------------------------------ TMA loads
    if (lane == 0) {
      for (int j = 0; j < nt; ++j) {
        const int st = j & 1;
        if (j >= 2 && !fa_wait(p, s, &s.kv_empty[st], ((j >> 1) - 1) & 1, -41)) break;
        // a 64-key block lies inside one KV page: one box per 64-dim half
        const int row = (int)(kv_row(p.m, slot, p.layer, g, j * kFaKeys) / D);
        mbar_arrive_expect_tx(&s.kv_full[st], 2u * NH * kFaKeys * 64 * 2);
        s.armed[st] = (uint32_t)j;
        tma_load_2d(s.k[st][0], &mk0, 0, row, &s.kv_full[st]);
        tma_load_2d(s.v[st][0], &mv0, 0, row, &s.kv_full[st]);
        if constexpr (NH == 2) {
          tma_load_2d(s.k[st][1], &mk1, 0, row, &s.kv_full[st]);
          tma_load_2d(s.v[st][1], &mv1, 0, row, &s.kv_full[st]);
        }
      }
    }
  } else if (warp == 5) {
    // ------------------------------------------------------------ MMA issue
    if (lane == 0) {
      constexpr uint32_t idS = mma_idesc_bf16_f32(kFaRows, kFaKeys);
      constexpr uint32_t idO = mma_idesc_bf16_f32(kFaRows, D) | (1u << 16);  // V MN-major
      bool ok = true;
      auto issue_s = [&](int j) -> bool {
        const int st = j & 1;
        if (!fa_wait(p, s, &s.kv_full[st], (j >> 1) & 1, -42)) return false;
        tc_fence_after_sync();
        const uint32_t dS = tS + (uint32_t)(st * kFaKeys);
#pragma unroll
        for (int part = 0; part < 2; ++part)
#pragma unroll
          for (int ks = 0; ks < D / 16; ++ks) {
            const uint64_t adv = (uint64_t)(2 * (ks & 3));
            tc_mma_f16(dS, sw128_kmajor_desc(s.q[part][ks >> 2]) + adv,
                       sw128_kmajor_desc(s.k[st][ks >> 2]) + adv, idS, (part | ks) != 0);
          }
        tc_commit(&s.s_full[st]);
        return true;
      };
      ok = issue_s(0);
      for (int j = 0; ok && j < nt; ++j) {
        if (j + 1 < nt && !issue_s(j + 1)) { ok = false; break; }
        const int st = j & 1;
        if (!fa_wait(p, s, &s.p_full[st], (j >> 1) & 1, -43)) { ok = false; break; }
        tc_fence_after_sync();
#pragma unroll
        for (int part = 0; part < 2; ++part)
#pragma unroll
          for (int ks = 0; ks < kFaKeys / 16; ++ks)
            tc_mma_f16(tO, sw128_kmajor_desc(s.p[st][part]) + (uint64_t)(2 * ks),
                       sw128_mnmajor_desc(s.v[st][0] + ks * 2048, kFaKeys * 128, 1024), idO,
                       (j | part | ks) != 0);
        tc_commit(&s.kv_empty[st]);
        tc_commit(&s.o_done);
      }
      tc_commit(&s.fin);  // arrives once every MMA issued above has retired
    }
  } else {
    // ------------------------------------------------- softmax and epilogue
    const int r = threadIdx.x;  // the row, and this thread's TMEM lane
    const bool row_ok = r < nrows;
    const int pos_r = p0 + r;
    const uint32_t lane_base = (uint32_t)(warp * 32) << 16;
    float m_used = -INFINITY, l = 0.f;
    bool ok = true;
    for (int j = 0; j < nt; ++j) {
      const int b = j & 1;
      ok = fa_wait(p, s, &s.s_full[b], (j >> 1) & 1, -44);
      if (!__all_sync(0xffffffffu, ok)) { ok = false; break; }
      tc_fence_after_sync();
      float sv[kFaKeys];
#pragma unroll
      for (int c = 0; c < kFaKeys; c += 16)
        tmem_ld16(tS + lane_base + (uint32_t)(b * kFaKeys + c), *reinterpret_cast<float(*)[16]>(sv + c));
      // causal mask: key k0 + c is visible to this row when k0 + c <= its position
      const int k0 = j * kFaKeys;
      float mt = -INFINITY;
#pragma unroll
      for (int c = 0; c < kFaKeys; ++c) {
        if (!row_ok || k0 + c > pos_r) sv[c] = -INFINITY;
        mt = fmaxf(mt, sv[c]);
      }
      float alpha = 1.f;
      if (mt > m_used + 8.f) {
        alpha = exp2f(m_used - mt);  // 0 while nothing was accumulated
        m_used = mt;
      }
      const float mu = m_used == -INFINITY ? 0.f : m_used;
      // O and the P buffer of tile j - 2 are free once the previous tile's
      // products retired
      if (j >= 1) {
        ok = fa_wait(p, s, &s.o_done, (j - 1) & 1, -45);
        if (!__all_sync(0xffffffffu, ok)) { ok = false; break; }
        tc_fence_after_sync();
        if (__any_sync(0xffffffffu, alpha != 1.f)) {
#pragma unroll 1
          for (int c = 0; c < D; c += 16) {
            float o[16];
            tmem_ld16(tO + lane_base + (uint32_t)c, o);
#pragma unroll
            for (int i = 0; i < 16; ++i) o[i] *= alpha;
            tmem_st16(tO + lane_base + (uint32_t)c, o);
          }
        }
      }
      float rs = 0.f;
#pragma unroll
      for (int c = 0; c < kFaKeys; c += 8) {
        float pv[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          pv[i] = exp2f(sv[c + i] - mu);
          rs += pv[i];
        }
        uint4 hi, lo;
        split2x8(pv, hi, lo);
        const uint32_t off = sw128_off(r, c);
        *reinterpret_cast<uint4*>(s.p[b][0] + off) = hi;
        *reinterpret_cast<uint4*>(s.p[b][1] + off) = lo;
      }
      l = l * alpha + rs;
      fence_proxy_async_shared();
      tc_fence_before_sync();
      mbar_arrive(&s.p_full[b]);
    }
    if (ok) ok = fa_wait(p, s, &s.o_done, (nt - 1) & 1, -46);
    if (__all_sync(0xffffffffu, ok)) {
      tc_fence_after_sync();
      const float inv = row_ok ? 1.0f / l : 0.f;
      const size_t orow = (size_t)(t0 + r) * p.ldo + (size_t)h * D;
#pragma unroll 1
      for (int c = 0; c < D; c += 16) {
        float o[16];
        tmem_ld16(tO + lane_base + (uint32_t)c, o);
        if (row_ok) {
          uint16_t hh[16], mm[16], ll[16];
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            const float v = o[i] * inv;
            hh[i] = f2bf(v);
            const float r1 = v - __uint_as_float((uint32_t)hh[i] << 16);
            mm[i] = f2bf(r1);
            ll[i] = f2bf(r1 - __uint_as_float((uint32_t)mm[i] << 16));
          }
#pragma unroll
          for (int i = 0; i < 16; i += 8) {
            *reinterpret_cast<uint4*>(p.oh + orow + c + i) = *reinterpret_cast<const uint4*>(hh + i);
            *reinterpret_cast<uint4*>(p.om + orow + c + i) = *reinterpret_cast<const uint4*>(mm + i);
            *reinterpret_cast<uint4*>(p.ol + orow + c + i) = *reinterpret_cast<const uint4*>(ll + i);
          }
        }
      }
    }
  }
  // ------------------------------------------------------------ teardown
  tc_fence_before_sync();
  __syncthreads();
  if (threadIdx.x == 0) {
    // every MMA issued has retired once `fin` arrived; after an abort, let the
    // loads still in flight land before the CTA exits
    s.tmem_ok = fa_drain(&s.fin, 0) ? 1 : 0;
    if (*(volatile int32_t*)&s.abort_flag)
      for (int i = 0; i < 2; ++i)
        if (s.armed[i] != 0xffffffffu) fa_drain(&s.kv_full[i], (s.armed[i] >> 1) & 1);
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
