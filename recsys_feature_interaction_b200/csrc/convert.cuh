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

namespace wk {

// The FMB LayerNorm's affine step folded into the first MLP Linear (done once,
// when a stack is created): LN(f) W^T + b = ((f - mean) rstd) (W diag(gamma))^T
// + (b + W beta), so the FM kernel stores only the normalised values.
//   out[o, q] = W[o, q] * gamma[q]                       (rounded to TO)
template <typename TI, typename TO>
__global__ void __launch_bounds__(256) fold_scale_cols_kernel(const TI* __restrict__ W, const float* __restrict__ gamma,
                                                              TO* __restrict__ out, int64_t rows, int64_t cols) {
  const int64_t nvec = rows * cols / 8;
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < nvec; i += stride) {
    const int64_t q0 = (i * 8) % cols;  // cols % 8 == 0: a vector never straddles rows
    float v[8];
    Vec8<TI>::load(W + i * 8, v);
    const float4 g0 = __ldg(reinterpret_cast<const float4*>(gamma + q0));
    const float4 g1 = __ldg(reinterpret_cast<const float4*>(gamma + q0) + 1);
    v[0] *= g0.x; v[1] *= g0.y; v[2] *= g0.z; v[3] *= g0.w;
    v[4] *= g1.x; v[5] *= g1.y; v[6] *= g1.z; v[7] *= g1.w;
    Vec8<TO>::store(out + i * 8, v);
  }
}

//   out[o] = b[o] + sum_q W[o, q] * beta[q]     (fp32, one warp per row; b may be null)
template <typename TI>
__global__ void __launch_bounds__(256) fold_bias_kernel(const TI* __restrict__ W, const float* __restrict__ beta,
                                                        const float* __restrict__ b, float* __restrict__ out,
                                                        int64_t rows, int64_t cols) {
  const int lane = threadIdx.x & 31;
  const int64_t warps = static_cast<int64_t>(gridDim.x) * (blockDim.x >> 5);
  for (int64_t o = static_cast<int64_t>(blockIdx.x) * (blockDim.x >> 5) + (threadIdx.x >> 5); o < rows; o += warps) {
    float s = 0.f;
    for (int64_t q = lane * 8; q < cols; q += 256) {
      float v[8];
      Vec8<TI>::load(W + o * cols + q, v);
      const float4 b0 = __ldg(reinterpret_cast<const float4*>(beta + q));
      const float4 b1 = __ldg(reinterpret_cast<const float4*>(beta + q) + 1);
      s += v[0] * b0.x + v[1] * b0.y + v[2] * b0.z + v[3] * b0.w + v[4] * b1.x + v[5] * b1.y + v[6] * b1.z +
           v[7] * b1.w;
    }
    s = warp_sum(s);
    if (lane == 0) out[o] = s + (b ? b[o] : 0.f);
  }
}

}  // namespace wk
