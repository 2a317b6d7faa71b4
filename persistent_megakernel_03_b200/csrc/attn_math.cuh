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

template <int DPL, int G>
struct AttnState {
  float q[G][DPL];
  float o[G][DPL];
  float mx[G];
  float l[G];
};

// Online softmax update with one key ("Hạt nhân là gì ...": running maximum
// and running sum, earlier partial results rescaled).
template <int DPL, int G>
__device__ __forceinline__ void attn_key(AttnState<DPL, G>& st, const float (&k)[DPL],
                                         const float (&v)[DPL]) {
#pragma unroll
  for (int h = 0; h < G; ++h) {
    float p = 0.f;
#pragma unroll
    for (int i = 0; i < DPL; ++i) p = fmaf(st.q[h][i], k[i], p);
#pragma unroll
    for (int o = 16; o; o >>= 1) p += __shfl_xor_sync(0xffffffffu, p, o);
    const float mn = fmaxf(st.mx[h], p);
    const float c = __expf(st.mx[h] - mn);
    const float e = __expf(p - mn);
    st.l[h] = fmaf(st.l[h], c, e);
#pragma unroll
    for (int i = 0; i < DPL; ++i) st.o[h][i] = fmaf(st.o[h][i], c, e * v[i]);
    st.mx[h] = mn;
  }
}

}  // namespace mk
