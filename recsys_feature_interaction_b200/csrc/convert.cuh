// convert.cuh -- elementwise storage conversion (bf16 -> fp16 and the like), 8
// elements per thread per step with 16-byte loads and stores. Used once per
// weight tensor when a stack is created and once per forward for the input
// embeddings when the caller's type differs from the operand type. The element
// count must be a multiple of 8 (the callers' tensors are).
#pragma once

#include "res_ln.cuh"

namespace wk {

template <typename TI, typename TO>
__global__ void __launch_bounds__(256) convert_kernel(const TI* __restrict__ in, TO* __restrict__ out, int64_t n) {
  const int64_t nvec = n / 8;
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < nvec; i += stride) {
    float v[8];
    Vec8<TI>::load(in + i * 8, v);
    Vec8<TO>::store(out + i * 8, v);
  }
}

}  // namespace wk
