// simt.cuh -- CUDA-core kernels of the Wukong layer steps for the fp32 workload
// and for shapes the tensor-core kernels are not instantiated for. All math is
// fp32; storage is T (float or bf16).
//
//   fm_ln_simt   : per example, Z = X^T Y, F = X Z (the optimised FM of the
//                  Wukong page, section 2.2: compress to k features, then cross),
//                  then LayerNorm over the flattened n*k values -> A0.
//   gemm_simt    : C = act(A W^T + bias) (an FMB MLP Linear), 64x64 block tiles.
//   lcb_simt     : concat[b, n_f + r, :] = W_L X_b (the LCB, section 2.2).
#pragma once

#include "common.cuh"

namespace wk {

template <typename T>
__device__ __forceinline__ float ld_f(const T* p, int64_t i);
template <>
__device__ __forceinline__ float ld_f<float>(const float* p, int64_t i) { return p[i]; }
template <>
__device__ __forceinline__ float ld_f<__nv_bfloat16>(const __nv_bfloat16* p, int64_t i) {
  return __bfloat162float(p[i]);
}

template <>
__device__ __forceinline__ float ld_f<__half>(const __half* p, int64_t i) { return __half2float(p[i]); }

template <typename T>
__device__ __forceinline__ void st_f(T* p, int64_t i, float v);
template <>
__device__ __forceinline__ void st_f<__half>(__half* p, int64_t i, float v) { p[i] = __float2half_rn(v); }
template <>
__device__ __forceinline__ void st_f<float>(float* p, int64_t i, float v) { p[i] = v; }
template <>
__device__ __forceinline__ void st_f<__nv_bfloat16>(__nv_bfloat16* p, int64_t i, float v) {
  p[i] = __float2bfloat16_rn(v);
}

// Block-wide sum for 256 threads; `red` holds 8 floats of shared memory.
__device__ __forceinline__ float block_sum_256(float v, float* red) {
  v = warp_sum(v);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  __syncthreads();
  if (lane == 0) red[warp] = v;
  __syncthreads();
  float t = 0.f;
#pragma unroll
  for (int w = 0; w < 8; ++w) t += red[w];
  return t;
}

// One CTA (256 threads) per example, grid-strided. Shared memory: X [n*d],
// Y [n*k], Z [d*k], F [n*k] as fp32.
template <typename T>
__global__ void __launch_bounds__(256) fm_ln_simt(const T* __restrict__ X, const T* __restrict__ Y,
                                                  const float* __restrict__ gamma, const float* __restrict__ beta,
                                                  T* __restrict__ A0, int64_t batch, int n, int d, int k,
                                                  float eps) {
  extern __shared__ float sm[];
  float* sX = sm;
  float* sY = sX + n * d;
  float* sZ = sY + n * k;
  float* sF = sZ + d * k;
  __shared__ float red[8];
  const int nk = n * k;
  for (int i = threadIdx.x; i < n * k; i += blockDim.x) sY[i] = ld_f(Y, i);
  for (int64_t b = blockIdx.x; b < batch; b += gridDim.x) {
    __syncthreads();
    for (int i = threadIdx.x; i < n * d; i += blockDim.x) sX[i] = ld_f(X, b * n * d + i);
    __syncthreads();
    for (int o = threadIdx.x; o < d * k; o += blockDim.x) {  // Z[t][c] = sum_i X[i][t] Y[i][c]
      const int t = o / k, c = o - t * k;
      float s = 0.f;
      for (int i = 0; i < n; ++i) s += sX[i * d + t] * sY[i * k + c];
      sZ[o] = s;
    }
    __syncthreads();
    float part = 0.f;
    for (int o = threadIdx.x; o < nk; o += blockDim.x) {  // F[i][c] = sum_t X[i][t] Z[t][c]
      const int i = o / k, c = o - i * k;
      float s = 0.f;
      for (int t = 0; t < d; ++t) s += sX[i * d + t] * sZ[t * k + c];
      sF[o] = s;
      part += s;
    }
    const float mean = block_sum_256(part, red) / static_cast<float>(nk);
    float q = 0.f;
    for (int o = threadIdx.x; o < nk; o += blockDim.x) {
      const float dv = sF[o] - mean;
      q += dv * dv;
    }
    const float rstd = rsqrtf(block_sum_256(q, red) / static_cast<float>(nk) + eps);
    for (int o = threadIdx.x; o < nk; o += blockDim.x)
      st_f(A0, b * nk + o, gamma ? (sF[o] - mean) * rstd * gamma[o] + beta[o] : (sF[o] - mean) * rstd);
  }
}

// C[r, c] = act(sum_q A[r, q] W[c, q] + bias[c]); 64x64 tiles, 256 threads, 4x4 per thread.
template <typename T, typename TO>
__global__ void __launch_bounds__(256) gemm_simt(const T* __restrict__ A, const T* __restrict__ W,
                                                 const float* __restrict__ bias, TO* __restrict__ C, int64_t M,
                                                 int K, int N, int64_t ldc, int relu) {
  __shared__ float sA[16][64 + 4];
  __shared__ float sW[16][64 + 4];
  const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
  const int64_t m0 = static_cast<int64_t>(blockIdx.y) * 64;
  const int n0 = blockIdx.x * 64;
  float acc[4][4] = {};
  for (int k0 = 0; k0 < K; k0 += 16) {
    for (int i = threadIdx.x; i < 16 * 64; i += 256) {
      const int kk = i & 15, r = i >> 4;
      sA[kk][r] = (m0 + r < M && k0 + kk < K) ? ld_f(A, (m0 + r) * K + k0 + kk) : 0.f;
      sW[kk][r] = (n0 + r < N && k0 + kk < K) ? ld_f(W, static_cast<int64_t>(n0 + r) * K + k0 + kk) : 0.f;
    }
    __syncthreads();
#pragma unroll
    for (int kk = 0; kk < 16; ++kk) {
      float a[4], w[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        a[i] = sA[kk][ty * 4 + i];
        w[i] = sW[kk][tx * 4 + i];
      }
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] += a[i] * w[j];
    }
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int64_t r = m0 + ty * 4 + i;
    if (r >= M) continue;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int c = n0 + tx * 4 + j;
      if (c >= N) continue;
      float v = acc[i][j] + (bias ? bias[c] : 0.f);
      if (relu) v = fmaxf(v, 0.f);
      st_f(C, r * ldc + c, v);
    }
  }
}

// concat[b, n_f + r, t] = sum_i W_L[r, i] X[b, i, t]; grid (ceil(n_l*d/256), batch).
template <typename T, typename TO>
__global__ void __launch_bounds__(256) lcb_simt(const T* __restrict__ WL, const T* __restrict__ X,
                                                TO* __restrict__ cat, int64_t batch, int n, int d, int n_f,
                                                int n_l) {
  const int64_t b = blockIdx.y;
  const int o = blockIdx.x * blockDim.x + threadIdx.x;
  if (o >= n_l * d) return;
  const int r = o / d, t = o - r * d;
  const T* xb = X + b * n * d;
  float s = 0.f;
  for (int i = 0; i < n; ++i) s += ld_f(WL, static_cast<int64_t>(r) * n + i) * ld_f(xb, static_cast<int64_t>(i) * d + t);
  st_f(cat, b * (n_f + n_l) * d + static_cast<int64_t>(n_f + r) * d + t, s);
}

}  // namespace wk
