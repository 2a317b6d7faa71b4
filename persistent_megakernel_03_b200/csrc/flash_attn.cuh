// flash_attn.cuh -- one (run of <= 128 prompt positions, query head) tile of
// causal GQA attention on the tensor cores, as a device function shared by the
// standalone attention kernel (flash_attn.cu) and the persistent prefill
// (prefill_mk.cu).  ("LLM高速化勉強会資料" slides 11-13 and "Hạt nhân là gì
// ...", the FlashAttention section: keys in tiles, scores and output kept on
// chip, an online softmax, no key past a query's position.)
//
// Scores S = Q K^T and the output O = P V are tcgen05.mma products in tensor
// memory (fp32 accumulate):
//   Q  the run's rotated queries times scale * log2(e), as two bf16 parts
//      (hi + lo carries 16 significant bits of the fp32 value), K-major;
//   K, V  64-key tiles of the bf16 cache (exact), brought by 2-D TMA with the
//      128-byte swizzle; K is the K-major B operand of S, V the MN-major B
//      operand of O;
//   P  2^(S - m) per row as two bf16 parts, written to shared memory by the
//      softmax threads (one row each) in the K-major swizzled layout.
// A row's running maximum m moves only when a tile's maximum exceeds it by
// more than 8 (powers of two): then O's row in tensor memory and the running
// sum are rescaled; otherwise the probabilities stay below 2^8 and O / l is
// unchanged.  The output is written as the O projection's three bf16 parts.
//
// Roles: warps 0-7 softmax and epilogue, two warps per row -- warp w takes
// the rows of TMEM lane quadrant w % 4 and half w / 4 of the score columns
// (and of the output columns), the halves exchanging their maxima through
// shared memory; lane 0 of warp 8 the TMA loads (two K/V stages), lane 0 of
// warp 9 the MMAs; other threads of the CTA only take part in the one CTA
// barrier.  Two score buffers let S of tile j+1 run while the softmax works
// on tile j.  The barrier phases continue across calls through `base`, the
// number of key tiles this CTA ran through the same barriers before.
#pragma once
#include <cuda.h>
#include <stdint.h>

#include "mk_internal.h"
#include "ptx.cuh"
#include "tc.cuh"

namespace mk {

constexpr int kFaRows = 128;           // query rows per tile (the MMA's M)
constexpr int kFaKeys = 64;            // keys per key tile
constexpr uint32_t kFaTmemCols = 256;  // two 64-column score buffers + O (<= 128 columns)
constexpr int kFaSoftmax = 2 * kFaRows;   // softmax threads (warps 0-7)
constexpr int kFaWarpTma = 8, kFaWarpMma = 9;
constexpr int kFaMinThreads = 320;        // threads a CTA needs for the roles
constexpr int kFaBarrier = 1;             // named barrier of the softmax warps

struct __align__(1024) FaBuffers {
  uint8_t q[2][2][kFaRows * 64 * 2];       // [part][64-dim half] 128 rows x 64 dims
  uint8_t k[2][2][kFaKeys * 64 * 2];       // [stage][half] 64 keys x 64 dims
  uint8_t v[2][2][kFaKeys * 64 * 2];
  uint8_t p[2][2][kFaRows * kFaKeys * 2];  // [buffer][part] 128 rows x 64 keys
};
static_assert(sizeof(FaBuffers) == 192 * 1024, "attention buffers");

struct FaBarriers {
  // K and V stages fill and free separately: a K stage is free once its scores
  // are computed, long before the V stage's product
  uint64_t k_full[2], k_empty[2], v_full[2], v_empty[2];
  // p_free[b]: one arrival per product that read P buffer b; a tile waits on
  // it for the product two tiles back (its buffer) and, to touch O, for the
  // last one -- neither barrier can then be two phases behind its wait
  uint64_t s_full[2], p_full[2], p_free[2];
  uint64_t fin;         // one arrival per call, once every MMA the call issued retired
  uint32_t armed_k[2];  // the last key tile whose K (V) loads went to each stage
  uint32_t armed_v[2];
  float xmax[2][kFaRows];  // the two halves' tile maxima (per row)
  float xsum[2][kFaRows];  // the two halves' final sums (per row)
};

// Named barrier of the softmax warps that also ANDs a flag over them: every
// softmax thread reaches it on every path, so a failed wait never leaves a
// warp waiting here.
__device__ __forceinline__ bool fa_softmax_sync_and(bool v) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\tsetp.ne.u32 p, %1, 0;\n\t"
      "bar.red.and.pred q, %2, %3, p;\n\tselp.u32 %0, 1, 0, q;\n\t}"
      : "=r"(r)
      : "r"((uint32_t)v), "n"(kFaBarrier), "n"(kFaSoftmax)
      : "memory");
  return r != 0;
}

// Initialises the barriers (one thread; fence_barrier_init and a CTA barrier
// must follow before use).
__device__ __forceinline__ void fa_init_barriers(FaBarriers& b) {
  for (int i = 0; i < 2; ++i) {
    mbar_init(&b.k_full[i], 1);
    mbar_init(&b.k_empty[i], 1);
    mbar_init(&b.v_full[i], 1);
    mbar_init(&b.v_empty[i], 1);
    mbar_init(&b.s_full[i], 1);
    mbar_init(&b.p_full[i], kFaSoftmax);
    mbar_init(&b.p_free[i], 1);
    b.armed_k[i] = b.armed_v[i] = 0xffffffffu;
  }
  mbar_init(&b.fin, 1);
}

struct FaJob {
  const CUtensorMap* mk0;  // K, first 64 dims of a row
  const CUtensorMap* mk1;  // K, second 64 dims (head_dim 128)
  const CUtensorMap* mv0;
  const CUtensorMap* mv1;
  const float* q;          // [T][ldq] rotated queries (fp32)
  int ldq;
  uint16_t* oh;            // [T][ldo] output, three bf16 parts
  uint16_t* om;
  uint16_t* ol;
  int ldo;
  int layer;
  float qscale;            // attention scale * log2(e)
  int t0, nrows, slot, p0, h;  // the run: first block token, rows, KV slot, first position; query head
};

// Key tiles of a run (keys 0 .. p0 + nrows - 1).
__host__ __device__ __forceinline__ int fa_key_tiles(int p0, int nrows) {
  return (p0 + nrows + kFaKeys - 1) / kFaKeys;
}

// Byte offset of the 16-byte group holding columns [c, c + 8) of row r in a
// K-major tile with 128-byte rows and the 128-byte swizzle.
__device__ __forceinline__ uint32_t fa_sw128_off(int r, int c) {
  return (uint32_t)r * 128u + ((uint32_t)((c >> 3) ^ (r & 7)) << 4);
}

__device__ __forceinline__ uint32_t fa_pack_bf16x2(float lo, float hi) {
  uint32_t r;
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}

// v[0..7] -> two bf16 parts (hi = RN(v), lo = RN(v - hi)), 16 bytes each.
__device__ __forceinline__ void fa_split2x8(const float (&v)[8], uint4& hi, uint4& lo) {
  uint32_t h[4], l[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    h[i] = fa_pack_bf16x2(v[2 * i], v[2 * i + 1]);
    l[i] = fa_pack_bf16x2(v[2 * i] - __uint_as_float(h[i] << 16),
                          v[2 * i + 1] - __uint_as_float(h[i] & 0xFFFF0000u));
  }
  hi = make_uint4(h[0], h[1], h[2], h[3]);
  lo = make_uint4(l[0], l[1], l[2], l[3]);
}

__device__ __forceinline__ uint16_t fa_bf16(float f) {
  uint16_t r;
  asm("cvt.rn.bf16.f32 %0, %1;" : "=h"(r) : "f"(f));
  return r;
}

// One tile.  `wait(bar, parity, where)` is the caller's bounded mbarrier wait
// (false: gave up or the CTA is aborting).  Every thread of the CTA calls
// this; returns false on the threads whose waits failed.  On return from a
// successful call the tile's MMAs have all retired (the softmax threads saw
// the last product) and its loads have landed.
template <int D, class Wait>
__device__ __forceinline__ bool fa_tile(const ModelDev& m, const FaJob& j, FaBuffers& b,
                                        FaBarriers& bar, uint32_t tmem, uint32_t base, Wait wait) {
  constexpr int NH = D / 64;  // 64-dim halves of a head
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = j.h / m.group;
  const int nt = fa_key_tiles(j.p0, j.nrows);
  // the run's queries, scaled, as two bf16 parts in the swizzled layout
  if (threadIdx.x < kFaSoftmax) {
    const int r = threadIdx.x & (kFaRows - 1), half = threadIdx.x / kFaRows;
    const float* qr = j.q + (size_t)(j.t0 + r) * j.ldq + (size_t)j.h * D;
#pragma unroll 2
    for (int c0 = half * (D / 2); c0 < (half + 1) * (D / 2); c0 += 8) {
      float v[8];
      if (r < j.nrows) {
        const float4 a = __ldcg(reinterpret_cast<const float4*>(qr + c0));
        const float4 c = __ldcg(reinterpret_cast<const float4*>(qr + c0 + 4));
        v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w; v[4] = c.x; v[5] = c.y; v[6] = c.z; v[7] = c.w;
#pragma unroll
        for (int i = 0; i < 8; ++i) v[i] *= j.qscale;
      } else {
#pragma unroll
        for (int i = 0; i < 8; ++i) v[i] = 0.f;
      }
      uint4 hi, lo;
      fa_split2x8(v, hi, lo);
      const uint32_t off = fa_sw128_off(r, c0 & 63);
      *reinterpret_cast<uint4*>(b.q[0][c0 >> 6] + off) = hi;
      *reinterpret_cast<uint4*>(b.q[1][c0 >> 6] + off) = lo;
    }
  }
  fence_proxy_async_shared();
  tc_fence_before_sync();
  __syncthreads();
  tc_fence_after_sync();
  const uint32_t tS = tmem;         // score buffers: columns [0, 64), [64, 128)
  const uint32_t tO = tmem + 128u;  // output: columns [128, 128 + D)
  bool ok = true;

  if (warp == kFaWarpTma) {
    // ------------------------------------------------------------ TMA loads
    if (lane == 0) {
      fence_proxy_async_shared();  // stage bytes may have been written by generic stores
      // K of tile i + 1 goes out before V of tile i: the scores run a tile ahead
      auto load = [&](int i, bool is_v) -> bool {
        const uint32_t gi = base + (uint32_t)i;
        const int st = gi & 1;
        uint64_t* empty = is_v ? &bar.v_empty[st] : &bar.k_empty[st];
        uint64_t* full = is_v ? &bar.v_full[st] : &bar.k_full[st];
        if (gi >= 2 && !wait(empty, ((gi >> 1) - 1) & 1, is_v ? -47 : -41)) return false;
        // a 64-key block lies inside one KV page: one box per 64-dim half
        const int row = (int)(kv_row(m, j.slot, j.layer, g, i * kFaKeys) / D);
        mbar_arrive_expect_tx(full, (uint32_t)NH * kFaKeys * 64 * 2);
        (is_v ? bar.armed_v : bar.armed_k)[st] = gi;
        uint8_t(*dst)[kFaKeys * 64 * 2] = is_v ? b.v[st] : b.k[st];
        tma_load_2d(dst[0], is_v ? j.mv0 : j.mk0, 0, row, full);
        if constexpr (NH == 2) tma_load_2d(dst[1], is_v ? j.mv1 : j.mk1, 0, row, full);
        return true;
      };
      ok = load(0, false);
      for (int i = 0; ok && i < nt; ++i) {
        if (i + 1 < nt && !load(i + 1, false)) { ok = false; break; }
        if (!load(i, true)) { ok = false; break; }
      }
    }
  } else if (warp == kFaWarpMma) {
    // ------------------------------------------------------------ MMA issue
    if (lane == 0) {
      constexpr uint32_t idS = mma_idesc_bf16_f32(kFaRows, kFaKeys);
      constexpr uint32_t idO = mma_idesc_bf16_f32(kFaRows, D) | (1u << 16);  // V MN-major
      auto issue_s = [&](int i) -> bool {
        const uint32_t gi = base + (uint32_t)i;
        const int st = gi & 1;
        if (!wait(&bar.k_full[st], (gi >> 1) & 1, -42)) return false;
        tc_fence_after_sync();
        const uint32_t dS = tS + (uint32_t)(st * kFaKeys);
#pragma unroll
        for (int part = 0; part < 2; ++part)
#pragma unroll
          for (int ks = 0; ks < D / 16; ++ks) {
            const uint64_t adv = (uint64_t)(2 * (ks & 3));
            tc_mma_f16(dS, sw128_kmajor_desc(b.q[part][ks >> 2]) + adv,
                       sw128_kmajor_desc(b.k[st][ks >> 2]) + adv, idS, (part | ks) != 0);
          }
        tc_commit(&bar.s_full[st]);
        tc_commit(&bar.k_empty[st]);
        return true;
      };
      ok = issue_s(0);
      for (int i = 0; ok && i < nt; ++i) {
        if (i + 1 < nt && !issue_s(i + 1)) { ok = false; break; }
        const uint32_t gi = base + (uint32_t)i;
        const int st = gi & 1;
        if (!wait(&bar.p_full[st], (gi >> 1) & 1, -43) || !wait(&bar.v_full[st], (gi >> 1) & 1, -48)) {
          ok = false;
          break;
        }
        tc_fence_after_sync();
#pragma unroll
        for (int part = 0; part < 2; ++part)
#pragma unroll
          for (int ks = 0; ks < kFaKeys / 16; ++ks)
            tc_mma_f16(tO, sw128_kmajor_desc(b.p[st][part]) + (uint64_t)(2 * ks),
                       sw128_mnmajor_desc(b.v[st][0] + ks * 2048, kFaKeys * 128, 1024), idO,
                       (i | part | ks) != 0);
        tc_commit(&bar.v_empty[st]);
        tc_commit(&bar.p_free[st]);
      }
      tc_commit(&bar.fin);
    }
  } else if (threadIdx.x < kFaSoftmax) {
    // ------------------------------------------------- softmax and epilogue
    const int quad = warp & 3, half = warp >> 2;
    const int r = quad * 32 + lane;  // the row, and this thread's TMEM lane
    const bool row_ok = r < j.nrows;
    const int pos_r = j.p0 + r;
    const uint32_t lane_base = (uint32_t)(quad * 32) << 16;
    constexpr int kC = kFaKeys / 2;  // score columns of this half
    constexpr int kO = D / 2;        // output columns of this half
    float m_used = -INFINITY, l = 0.f;
    for (int i = 0; i < nt; ++i) {
      const uint32_t gi = base + (uint32_t)i;
      const int bf = gi & 1;
      ok = ok && wait(&bar.s_full[bf], (gi >> 1) & 1, -44);
      if (!fa_softmax_sync_and(ok)) { ok = false; break; }
      tc_fence_after_sync();
      static_assert(kC == 32, "one 32-column load per half row");
      float sv[kC];
      tmem_ld32(tS + lane_base + (uint32_t)(bf * kFaKeys + half * kC), sv);
      // causal mask: key k0 + c is visible to this row when k0 + c <= its position
      const int k0 = i * kFaKeys + half * kC;
      float mt = -INFINITY;
#pragma unroll
      for (int c = 0; c < kC; ++c) {
        if (!row_ok || k0 + c > pos_r) sv[c] = -INFINITY;
        mt = fmaxf(mt, sv[c]);
      }
      // the row's maximum over both halves
      bar.xmax[half][r] = mt;
      // this P buffer is free once tile i - 2's product retired (waited before
      // the exchange so that the barrier below also agrees on it)
      if (i >= 2) ok = wait(&bar.p_free[bf], ((gi >> 1) - 1) & 1, -45);
      if (!fa_softmax_sync_and(ok)) { ok = false; break; }
      mt = fmaxf(mt, bar.xmax[half ^ 1][r]);
      float alpha = 1.f;
      if (mt > m_used + 8.f) {
        alpha = exp2f(m_used - mt);  // 0 while nothing was accumulated
        m_used = mt;
      }
      const float mu = m_used == -INFINITY ? 0.f : m_used;
      if (i >= 1 && __any_sync(0xffffffffu, alpha != 1.f)) {
        // rescale this half of O's rows once the last product retired (a
        // failed wait is carried to the next barrier, which every warp reaches)
        ok = wait(&bar.p_free[(gi - 1) & 1], ((gi - 1) >> 1) & 1, -49);
        ok = __all_sync(0xffffffffu, ok);
        tc_fence_after_sync();
        if (ok) {
#pragma unroll 1
          for (int c = half * kO; c < (half + 1) * kO; c += 16) {
            float o[16];
            tmem_ld16(tO + lane_base + (uint32_t)c, o);
#pragma unroll
            for (int e = 0; e < 16; ++e) o[e] *= alpha;
            tmem_st16(tO + lane_base + (uint32_t)c, o);
          }
        }
      }
      float rs = 0.f;
#pragma unroll
      for (int c = 0; c < kC; c += 8) {
        float pv[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          pv[e] = exp2f(sv[c + e] - mu);
          rs += pv[e];
        }
        uint4 hi, lo;
        fa_split2x8(pv, hi, lo);
        const uint32_t off = fa_sw128_off(r, half * kC + c);
        *reinterpret_cast<uint4*>(b.p[bf][0] + off) = hi;
        *reinterpret_cast<uint4*>(b.p[bf][1] + off) = lo;
      }
      l = l * alpha + rs;  // this half's share of the row's sum
      fence_proxy_async_shared();
      tc_fence_before_sync();
      mbar_arrive(&bar.p_full[bf]);
    }
    // every product retired (the last one's buffer barrier; the earlier ones
    // retire first)
    const uint32_t gl = base + (uint32_t)nt - 1;
    if (ok) ok = wait(&bar.p_free[gl & 1], (gl >> 1) & 1, -46);
    // both halves' sums
    bar.xsum[half][r] = l;
    if (fa_softmax_sync_and(ok)) {
      tc_fence_after_sync();
      const float lt = l + bar.xsum[half ^ 1][r];
      const float inv = row_ok ? 1.0f / lt : 0.f;
      const size_t orow = (size_t)(j.t0 + r) * j.ldo + (size_t)j.h * D;
#pragma unroll 1
      for (int c = half * kO; c < (half + 1) * kO; c += 16) {
        float o[16];
        tmem_ld16(tO + lane_base + (uint32_t)c, o);
        if (row_ok) {
          uint16_t hh[16], mm[16], ll[16];
#pragma unroll
          for (int e = 0; e < 16; ++e) {
            const float v = o[e] * inv;
            hh[e] = fa_bf16(v);
            const float r1 = v - __uint_as_float((uint32_t)hh[e] << 16);
            mm[e] = fa_bf16(r1);
            ll[e] = fa_bf16(r1 - __uint_as_float((uint32_t)mm[e] << 16));
          }
#pragma unroll
          for (int e = 0; e < 16; e += 8) {
            *reinterpret_cast<uint4*>(j.oh + orow + c + e) = *reinterpret_cast<const uint4*>(hh + e);
            *reinterpret_cast<uint4*>(j.om + orow + c + e) = *reinterpret_cast<const uint4*>(mm + e);
            *reinterpret_cast<uint4*>(j.ol + orow + c + e) = *reinterpret_cast<const uint4*>(ll + e);
          }
        }
      }
    } else {
      ok = false;
    }
  }
  return ok;
}

}  // namespace mk
