// step_bf16_d64.cu -- the persistent step kernel for bf16 weights and head_dim 64,
// one instantiation per supported number of query heads per KV head.
#include "step_kernel.cuh"

namespace mk {

const void* step_kernel_bf16_d64(int G) {
  switch (G) {
    case 1: return reinterpret_cast<const void*>(&mk_step_kernel<4, 2, 1>);
    case 2: return reinterpret_cast<const void*>(&mk_step_kernel<4, 2, 2>);
    case 4: return reinterpret_cast<const void*>(&mk_step_kernel<4, 2, 4>);
    case 7: return reinterpret_cast<const void*>(&mk_step_kernel<4, 2, 7>);
    case 8: return reinterpret_cast<const void*>(&mk_step_kernel<4, 2, 8>);
    default: return nullptr;
  }
}

}  // namespace mk
