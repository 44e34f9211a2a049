// head.cuh -- the output of the prediction head that follows the Wukong layers
// (Wukong page, section 2.2: the stacked layers cross the features, an MLP then
// produces the prediction). The head's hidden Linears run on the tensor-core GEMM;
// its last Linear has ONE output per example, a dot product that is bound by reading
// the hidden activations, so it runs here on CUDA cores together with the sigmoid:
//
//   logit[b] = sum_j H[b, j] w[j] + c,     prob[b] = 1 / (1 + exp(-logit[b]))
#pragma once

#include "res_ln.cuh"

namespace wk {

// One warp per example (grid-stride): lanes walk 16-byte vectors of the row and of
// w, fp32 products, a shuffle reduction, lane 0 writes. H [batch, K] and w [K] in T
// (K a multiple of 8, 16-byte aligned rows); bias [1] fp32 or null; prob may be null.
template <typename T>
__global__ void __launch_bounds__(256) head_out_kernel(const T* __restrict__ H, const T* __restrict__ w,
                                                      const float* __restrict__ bias, float* __restrict__ logit,
                                                      float* __restrict__ prob, int64_t batch, int64_t K) {
  const int lane = threadIdx.x & 31;
  const int64_t warp = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int64_t nwarps = (static_cast<int64_t>(gridDim.x) * blockDim.x) >> 5;
  const int64_t nvec = K / 8;
  const float c = bias ? __ldg(bias) : 0.f;
  for (int64_t b = warp; b < batch; b += nwarps) {
    const T* row = H + b * K;
    float s = 0.f;
    for (int64_t v = lane; v < nvec; v += 32) {
      float h8[8], w8[8];
      Vec8<T>::load(row + v * 8, h8);
      Vec8<T>::load(w + v * 8, w8);
#pragma unroll
      for (int j = 0; j < 8; ++j) s = fmaf(h8[j], w8[j], s);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
    if (lane == 0) {
      const float z = s + c;
      logit[b] = z;
      if (prob) prob[b] = 1.0f / (1.0f + expf(-z));
    }
  }
}

}  // namespace wk
