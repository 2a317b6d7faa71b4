// attn_math.cuh -- decode-attention math shared by the persistent kernel's
// attention tasks and the standalone split-KV attention op: bf16 widening,
// K/V row loads, and the online-softmax update of one key.
#pragma once
#include <stdint.h>

namespace mk {

__device__ __forceinline__ float bf_lo(uint32_t u) { return __uint_as_float(u << 16); }
__device__ __forceinline__ float bf_hi(uint32_t u) { return __uint_as_float(u & 0xffff0000u); }

template <int DPL>
__device__ __forceinline__ void load_kv_row(const uint16_t* p, float (&v)[DPL]) {
  if constexpr (DPL == 4) {
    const uint2 u = *reinterpret_cast<const uint2*>(p);
    v[0] = bf_lo(u.x); v[1] = bf_hi(u.x); v[2] = bf_lo(u.y); v[3] = bf_hi(u.y);
  } else {
    const uint32_t u = *reinterpret_cast<const uint32_t*>(p);
    v[0] = bf_lo(u); v[1] = bf_hi(u);
  }
}

template <int DPL>
__device__ __forceinline__ void load_kv_row_global(const uint16_t* p, float (&v)[DPL]) {
  if constexpr (DPL == 4) {
    const uint2 u = __ldcg(reinterpret_cast<const uint2*>(p));
    v[0] = bf_lo(u.x); v[1] = bf_hi(u.x); v[2] = bf_lo(u.y); v[3] = bf_hi(u.y);
  } else {
    const uint32_t u = __ldcg(reinterpret_cast<const unsigned int*>(p));
    v[0] = bf_lo(u); v[1] = bf_hi(u);
  }
}

// Query heads rounded up to a power of two, (head, key) slots of a batch of
// four keys, and the per-warp shared floats a batch needs: every slot's
// softmax weight stored twice (a ready-made float2 for packed FMAs), then the
// heads' new maxima.
template <int G>
struct AttnPad {
  static constexpr int GP = G <= 1 ? 1 : G <= 2 ? 2 : G <= 4 ? 4 : 8;
  static constexpr int NV = 4 * GP;                                        // slots
  static constexpr int M = NV == 4 ? 2 : NV == 8 ? 3 : NV == 16 ? 4 : 5;  // log2(NV)
  static constexpr int kXbFloats = 2 * NV + GP;
};

// Per-warp stride of the attention's shared floats (any G up to 8).
constexpr int kAttnXbStride = 72;

// Running online-softmax state of one warp.  A lane holds dims
// [lane*DPL, lane*DPL + DPL) of every head's output; its query copy `qp` is
// stored with the heads permuted by this lane's slot mask (see attn_scores4),
// so the cross-lane score reduction needs no per-lane selects.
template <int DPL, int G>
struct AttnState {
  float qp[AttnPad<G>::GP][DPL];
  float o[G][DPL];
  float mx[G];
  float l[G];
};

// The lane's slot after the transposed reduction: the top M bits of the lane.
template <int G>
__device__ __forceinline__ int attn_slot_mask(int lane) { return lane >> (5 - AttnPad<G>::M); }

// Loads the (pre-scaled) queries q[h*d + dim] of the G heads into st.qp in
// this lane's head order and clears the rest of the state.
template <int DPL, int G>
__device__ __forceinline__ void attn_init(AttnState<DPL, G>& st, const float* q, int d, float scale,
                                          int lane) {
  using P = AttnPad<G>;
  const int mh = attn_slot_mask<G>(lane) >> 2;
#pragma unroll
  for (int hh = 0; hh < P::GP; ++hh) {
    const int h = hh ^ mh;
#pragma unroll
    for (int i = 0; i < DPL; ++i)
      st.qp[hh][i] = h < G ? __ldcg(q + (size_t)h * d + lane * DPL + i) * scale : 0.f;
  }
#pragma unroll
  for (int h = 0; h < G; ++h) {
#pragma unroll
    for (int i = 0; i < DPL; ++i) st.o[h][i] = 0.f;
    st.mx[h] = -INFINITY;
    st.l[h] = 0.f;
  }
}

// Key row that register slot jj of this lane must hold for keys j0..j0+3
// (the rows are permuted by the key bits of the lane's slot mask).
template <int G>
__device__ __forceinline__ int attn_key_row(int jj, int lane) {
  return jj ^ (attn_slot_mask<G>(lane) & 3);
}

// Online softmax over up to four keys at once ("Hạt nhân là gì ...": running
// maximum and running sum, earlier partial results rescaled), in two halves
// so a lane never holds four K rows and four V rows together.
//
// attn_scores4: k[jj] holds key row attn_key_row(jj) (zeros past nk).  The
// 4*GP partial dot products (position p = hh*4 + jj holds slot p ^ mask,
// slot = head*4 + key) are summed across the warp by a transposed butterfly:
// at offset 16 >> r each lane keeps its first half and adds the partner's
// second half, which holds the same slots because the partner's mask differs
// in exactly that bit.  Lane l ends with the full score of slot
// attn_slot_mask(l), so a key costs about G + 1 shuffles instead of 5 G.  The
// batch maximum per head and the weights exp(s - max) go to `xb` (this
// warp's kXbFloats shared floats).
template <int DPL, int G>
__device__ __forceinline__ void attn_scores4(const AttnState<DPL, G>& st, const float (&k)[4][DPL],
                                             int nk, float* xb, int lane) {
  using P = AttnPad<G>;
  static_assert(P::kXbFloats <= kAttnXbStride, "per-warp scratch too small");
  float val[P::NV];
#pragma unroll
  for (int hh = 0; hh < P::GP; ++hh)
#pragma unroll
    for (int jj = 0; jj < 4; ++jj) {
      if constexpr (DPL % 2 == 0) {
        float2 a2 = __fmul2_rn(make_float2(st.qp[hh][0], st.qp[hh][1]),
                               make_float2(k[jj][0], k[jj][1]));
#pragma unroll
        for (int i = 2; i < DPL; i += 2)
          a2 = __ffma2_rn(make_float2(st.qp[hh][i], st.qp[hh][i + 1]),
                          make_float2(k[jj][i], k[jj][i + 1]), a2);
        val[hh * 4 + jj] = a2.x + a2.y;
      } else {
        float acc = 0.f;
#pragma unroll
        for (int i = 0; i < DPL; ++i) acc = fmaf(st.qp[hh][i], k[jj][i], acc);
        val[hh * 4 + jj] = acc;
      }
    }
#pragma unroll
  for (int r = 0; r < P::M; ++r) {
    const int half = P::NV >> (r + 1);
#pragma unroll
    for (int i = 0; i < half; ++i) val[i] += __shfl_xor_sync(0xffffffffu, val[i + half], 16 >> r);
  }
  float sc = val[0];
#pragma unroll
  for (int o = 16 >> P::M; o; o >>= 1) sc += __shfl_xor_sync(0xffffffffu, sc, o);
  const int slot = attn_slot_mask<G>(lane);
  const int hl = slot >> 2, jl = slot & 3;
  if (hl >= G || jl >= nk) sc = -INFINITY;
  // batch maximum of this lane's head (slots of one head differ in key bits)
  float bm = fmaxf(sc, __shfl_xor_sync(0xffffffffu, sc, 1 << (5 - P::M)));
  bm = fmaxf(bm, __shfl_xor_sync(0xffffffffu, bm, 2 << (5 - P::M)));
  float mo = st.mx[0];
#pragma unroll
  for (int h = 1; h < G; ++h)
    if (hl == h) mo = st.mx[h];
  const float mn = fmaxf(mo, bm);
  const float e = hl < G ? __expf(sc - mn) : 0.f;
  __syncwarp();  // the previous batch's reads of xb are done
  if ((lane & ((1 << (5 - P::M)) - 1)) == 0) {
    *reinterpret_cast<float2*>(xb + 2 * slot) = make_float2(e, e);
    if (jl == 0 && hl < G) xb[2 * P::NV + hl] = mn;
  }
  __syncwarp();
}

// attn_update4: v[j] holds key row j (unpermuted, zeros past nk).
template <int DPL, int G>
__device__ __forceinline__ void attn_update4(AttnState<DPL, G>& st, const float (&v)[4][DPL],
                                             const float* xb) {
  using P = AttnPad<G>;
#pragma unroll
  for (int h = 0; h < G; ++h) {
    const float m2 = xb[2 * P::NV + h];
    const float4 w01 = *reinterpret_cast<const float4*>(xb + h * 8);
    const float4 w23 = *reinterpret_cast<const float4*>(xb + h * 8 + 4);
    float c = 1.f;
    if (m2 != st.mx[h]) {  // warp-uniform: rescale only when the maximum moved
      c = __expf(st.mx[h] - m2);
#pragma unroll
      for (int i = 0; i < DPL; ++i) st.o[h][i] *= c;
      st.mx[h] = m2;
    }
    st.l[h] = fmaf(st.l[h], c, (w01.x + w01.z) + (w23.x + w23.z));
#pragma unroll
    for (int i = 0; i < DPL; i += 2) {
      float2 acc = make_float2(st.o[h][i], st.o[h][i + 1]);
      acc = __ffma2_rn(make_float2(w01.x, w01.y), make_float2(v[0][i], v[0][i + 1]), acc);
      acc = __ffma2_rn(make_float2(w01.z, w01.w), make_float2(v[1][i], v[1][i + 1]), acc);
      acc = __ffma2_rn(make_float2(w23.x, w23.y), make_float2(v[2][i], v[2][i + 1]), acc);
      acc = __ffma2_rn(make_float2(w23.z, w23.w), make_float2(v[3][i], v[3][i + 1]), acc);
      st.o[h][i] = acc.x;
      st.o[h][i + 1] = acc.y;
    }
  }
}

}  // namespace mk
