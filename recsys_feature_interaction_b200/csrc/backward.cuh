// backward.cuh -- the kernels of the backward pass of a Wukong layer that are neither the
// FMB MLP's tensor-core GEMMs (gemm_tc2.cuh on transposed operands) nor the strided
// contractions of the FM and the LCB (bw_tc.cuh).
//
// Per layer, with y = concat(FMB(X), LCB(X)) + X, out = LN_d(y) gamma2 + beta2, the layer
// of the Wukong page (section 2.2) differentiated by the chain rule:
//   bw_out_ln_kernel     dy = LN_d'(y)^T (dOut * gamma2) per embedding row; d gamma2, d beta2;
//                        the FMB rows of dy as the MLP's upstream gradient (16-bit)
//   bw_relu_mask_kernel  dz = dh where the ReLU output was > 0
//   bw_to_f32_kernel     fp32 copies of the 16-bit operands of the tf32 contractions
//   bw_colsum_kernel     bias gradients (column sums over the batch)
//   bw_transpose_kernel  16-bit transposes feeding the K-major GEMM
//   bw_fmb_ln_kernel     dF = LN_nk'(F)^T d fhat per example (the FMB LayerNorm)
//   bw_unfold_kernel     gradients of W0, gamma1, beta1 from those of the folded first Linear
//                        W0' = W0 diag(gamma1), b0' = b0 + W0 beta1
#pragma once

#include "common.cuh"

namespace wk {

template <typename T>
__device__ __forceinline__ float bw_ld(const T* p);
template <>
__device__ __forceinline__ float bw_ld<float>(const float* p) {
  return __ldg(p);
}
template <>
__device__ __forceinline__ float bw_ld<__half>(const __half* p) {
  return __half2float(*p);
}
template <>
__device__ __forceinline__ float bw_ld<__nv_bfloat16>(const __nv_bfloat16* p) {
  return __bfloat162float(*p);
}

// 16-bit -> fp32 copy of an operand of the tf32 contractions (exact)
template <typename T>
__global__ void __launch_bounds__(256) bw_to_f32_kernel(const T* __restrict__ in, float* __restrict__ out, int64_t n) {
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n; i += stride)
    out[i] = bw_ld(in + i);
}

// ------------------------------------------------ output LayerNorm, per row

// One warp per embedding row of d (a multiple of 32, at most 256) values.
template <typename T>
__global__ void __launch_bounds__(256) bw_out_ln_kernel(const T* __restrict__ cat, const T* __restrict__ X,
                                                        const float* __restrict__ dOut, const float* __restrict__ g2,
                                                        float* __restrict__ dy, float* __restrict__ dx,
                                                        T* __restrict__ dh_m, float* __restrict__ dg2,
                                                        float* __restrict__ db2, int64_t rows, int n, int n_f, int d,
                                                        float eps) {
  __shared__ float sg[8][256], sb[8][256];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int per = d >> 5;  // values per lane, columns lane + 32 i
  float ag[8], ab[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) ag[i] = ab[i] = 0.f;
  const float inv_d = 1.f / static_cast<float>(d);
  for (int64_t r = static_cast<int64_t>(blockIdx.x) * 8 + warp; r < rows; r += static_cast<int64_t>(gridDim.x) * 8) {
    float y[8], go[8];
    float s = 0.f;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      y[i] = 0.f;
      if (i < per) {
        const int64_t o = r * d + lane + 32 * i;
        y[i] = bw_ld(cat + o) + bw_ld(X + o);
        s += y[i];
      }
    }
    const float mean = warp_sum(s) * inv_d;
    float v = 0.f;
#pragma unroll
    for (int i = 0; i < 8; ++i)
      if (i < per) v += (y[i] - mean) * (y[i] - mean);
    const float rs = rsqrtf(warp_sum(v) * inv_d + eps);
    float s1 = 0.f, s2 = 0.f;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      if (i < per) {
        const int c = lane + 32 * i;
        const float dO = __ldg(dOut + r * d + c);
        y[i] = (y[i] - mean) * rs;  // yhat
        ag[i] += dO * y[i];
        ab[i] += dO;
        go[i] = dO * __ldg(g2 + c);
        s1 += go[i];
        s2 += go[i] * y[i];
      }
    }
    const float m1 = warp_sum(s1) * inv_d, m2 = warp_sum(s2) * inv_d;
    const int64_t b = r / n;
    const int i_row = static_cast<int>(r - b * n);
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      if (i < per) {
        const int c = lane + 32 * i;
        const float g = rs * (go[i] - m1 - y[i] * m2);
        dy[r * d + c] = tf32_round(g);  // read only by the tf32 contractions
        dx[r * d + c] = g;  // the residual's share of dX
        if (i_row < n_f) dh_m[(b * n_f + i_row) * d + c] = Half16<T>::from(g);
      }
    }
  }
  // this CTA's partial d gamma2, d beta2
#pragma unroll
  for (int i = 0; i < 8; ++i)
    if (i < per) {
      sg[warp][lane + 32 * i] = ag[i];
      sb[warp][lane + 32 * i] = ab[i];
    }
  __syncthreads();
  for (int c = threadIdx.x; c < d; c += blockDim.x) {
    float a = 0.f, bsum = 0.f;
#pragma unroll
    for (int w = 0; w < 8; ++w) {
      a += sg[w][c];
      bsum += sb[w][c];
    }
    atomicAdd(dg2 + c, a);
    atomicAdd(db2 + c, bsum);
  }
}

template <typename T>
__global__ void bw_relu_mask_kernel(T* __restrict__ dh, const T* __restrict__ h, int64_t count) {
  const int64_t nvec = count / 8;
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < nvec;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    uint4 g = reinterpret_cast<const uint4*>(dh)[i];
    const uint4 a = __ldg(reinterpret_cast<const uint4*>(h) + i);
    uint32_t* gw = reinterpret_cast<uint32_t*>(&g);
    const uint32_t* aw = reinterpret_cast<const uint32_t*>(&a);
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const float lo = Half16<T>::lo(aw[j]), hi = Half16<T>::hi(aw[j]);
      uint32_t mask = 0u;
      if (lo > 0.f) mask |= 0x0000FFFFu;
      if (hi > 0.f) mask |= 0xFFFF0000u;
      gw[j] &= mask;
    }
    reinterpret_cast<uint4*>(dh)[i] = g;
  }
}

// out[c] += sum over rows [r0, r1) of z[r, c]; blockDim 256 columns, gridDim.y row chunks.
template <typename T>
__global__ void bw_colsum_kernel(const T* __restrict__ z, float* __restrict__ out, int64_t rows, int cols) {
  const int c = blockIdx.x * blockDim.x + threadIdx.x;
  if (c >= cols) return;
  const int64_t chunk = (rows + gridDim.y - 1) / gridDim.y;
  const int64_t r0 = blockIdx.y * chunk, r1 = min(rows, r0 + chunk);
  float s = 0.f;
  for (int64_t r = r0; r < r1; ++r) s += bw_ld(z + r * cols + c);
  if (r1 > r0) atomicAdd(out + c, s);
}

// out [C, R] = in [R, C]^T (16-bit), 32 x 32 tiles through shared memory.
template <typename T>
__global__ void bw_transpose_kernel(const T* __restrict__ in, T* __restrict__ out, int64_t R, int64_t C) {
  __shared__ T tile[32][33];
  const int64_t c0 = static_cast<int64_t>(blockIdx.x) * 32, r0 = static_cast<int64_t>(blockIdx.y) * 32;
  for (int i = threadIdx.y; i < 32; i += blockDim.y) {
    const int64_t r = r0 + i, c = c0 + threadIdx.x;
    if (r < R && c < C) tile[i][threadIdx.x] = in[r * C + c];
  }
  __syncthreads();
  for (int i = threadIdx.y; i < 32; i += blockDim.y) {
    const int64_t c = c0 + i, r = r0 + threadIdx.x;
    if (r < R && c < C) out[c * R + r] = tile[threadIdx.x][i];
  }
}

// ------------------------------------------------ FMB LayerNorm over n*k, per example

__device__ __forceinline__ float bw_block_sum(float v, float* red) {
  v = warp_sum(v);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  __syncthreads();
  if (lane == 0) red[warp] = v;
  __syncthreads();
  float s = 0.f;
  for (int w = 0; w < static_cast<int>(blockDim.x >> 5); ++w) s += red[w];
  return s;
}

// One CTA per example: F [nk] fp32 (the FM output), dfh [nk] (the gradient of the
// normalised values) -> dF = rs (dfh - mean(dfh) - fhat mean(dfh fhat)).
template <typename T>
__global__ void __launch_bounds__(256) bw_fmb_ln_kernel(const float* __restrict__ F, const T* __restrict__ dfh,
                                                        float* __restrict__ dF, int nk, float eps) {
  __shared__ float red[8];
  const int64_t base = static_cast<int64_t>(blockIdx.x) * nk;
  const float inv = 1.f / static_cast<float>(nk);
  float s = 0.f;
  for (int i = threadIdx.x; i < nk; i += blockDim.x) s += F[base + i];
  const float mean = bw_block_sum(s, red) * inv;
  float v = 0.f;
  for (int i = threadIdx.x; i < nk; i += blockDim.x) {
    const float t = F[base + i] - mean;
    v += t * t;
  }
  const float rs = rsqrtf(bw_block_sum(v, red) * inv + eps);
  float s1 = 0.f, s2 = 0.f;
  for (int i = threadIdx.x; i < nk; i += blockDim.x) {
    const float g = bw_ld(dfh + base + i);
    s1 += g;
    s2 += g * (F[base + i] - mean) * rs;
  }
  const float m1 = bw_block_sum(s1, red) * inv, m2 = bw_block_sum(s2, red) * inv;
  for (int i = threadIdx.x; i < nk; i += blockDim.x) {
    const float fh = (F[base + i] - mean) * rs;
    dF[base + i] = tf32_round(rs * (bw_ld(dfh + base + i) - m1 - fh * m2));  // a tf32 operand
  }
}

// ------------------------------------------------ first Linear: unfold the LN affine

// dW0 [rows, cols] holds d/dW0' on entry and d/dW0 on exit; db0 = d/db0' = d/db0.
//   d/dW0[r, c] = d/dW0'[r, c] gamma1[c] + d/db0'[r] beta1[c]
//   d/dgamma1[c] += sum_r d/dW0'[r, c] W0[r, c],  d/dbeta1[c] += sum_r d/db0'[r] W0[r, c]
// blockDim 256 columns, gridDim.y row chunks (atomic adds into dg1, db1).
template <typename TW>
__global__ void bw_unfold_kernel(float* __restrict__ dW0, const float* __restrict__ db0, const TW* __restrict__ W0,
                                 const float* __restrict__ g1, const float* __restrict__ b1, float* __restrict__ dg1,
                                 float* __restrict__ db1, int rows, int cols) {
  const int c = blockIdx.x * blockDim.x + threadIdx.x;
  if (c >= cols) return;
  const int chunk = (rows + gridDim.y - 1) / gridDim.y;
  const int r0 = blockIdx.y * chunk, r1 = min(rows, r0 + chunk);
  const float gc = g1 ? __ldg(g1 + c) : 1.f, bc = b1 ? __ldg(b1 + c) : 0.f;
  float sg = 0.f, sb = 0.f;
  for (int r = r0; r < r1; ++r) {
    const int64_t o = static_cast<int64_t>(r) * cols + c;
    const float w = bw_ld(W0 + o), gw = dW0[o], gb = __ldg(db0 + r);
    sg += gw * w;
    sb += gb * w;
    dW0[o] = gw * gc + gb * bc;
  }
  if (r1 > r0) {
    atomicAdd(dg1 + c, sg);
    atomicAdd(db1 + c, sb);
  }
}

}  // namespace wk
