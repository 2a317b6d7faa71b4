// step_fp8_d128.cu -- the persistent step kernel for fp8 e4m3 weights and head_dim 128,
// one instantiation per supported number of query heads per KV head.
#include "step_kernel.cuh"

namespace mk {

const void* step_kernel_fp8_d128(int G) {
  switch (G) {
    case 1: return reinterpret_cast<const void*>(&mk_step_kernel<8, 4, 1>);
    case 2: return reinterpret_cast<const void*>(&mk_step_kernel<8, 4, 2>);
    case 4: return reinterpret_cast<const void*>(&mk_step_kernel<8, 4, 4>);
    default: return nullptr;
  }
}

}  // namespace mk
