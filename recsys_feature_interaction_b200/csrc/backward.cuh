// backward.cuh -- the kernels of the backward pass of a Wukong layer that are neither the
// FMB MLP's tensor-core GEMMs (gemm_tc2.cuh, operands read MN-major) nor the strided
// contractions of the FM and the LCB (bw_tc.cuh).
//
// Per layer, with y = concat(FMB(X), LCB(X)) + X, out = LN_d(y) gamma2 + beta2, the layer
// of the Wukong page (section 2.2) differentiated by the chain rule:
//   bw_out_ln_kernel       dy = LN_d'(y)^T (dOut * gamma2) per embedding row; d gamma2,
//                          d beta2; the FMB rows of dy as the MLP's upstream gradient (16-bit)
//   bw_mask_colsum_kernel  dz = dh where the ReLU output was > 0, and the bias gradient
//                          (column sums over the batch), in one pass
//   bw_to_f32_kernel       fp32 copies of the 16-bit operands of the tf32 contractions
//   bw_fmb_ln_reg_kernel   dF = LN_nk'(F)^T d fhat per example (the FMB LayerNorm), the
//                          example held in registers
//   bw_unfold4_kernel      gradients of W0, gamma1, beta1 from those of the folded first
//                          Linear W0' = W0 diag(gamma1), b0' = b0 + W0 beta1
// and the general forms the launcher falls back to for shapes the fast ones do not take
// (bw_relu_mask_kernel + bw_colsum_kernel, bw_fmb_ln_kernel, bw_unfold_kernel), with
// bw_transpose_kernel for the one-CTA GEMM, which reads only K-major operands.
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

// One warp per embedding row of d (even, at most 256) values, lane l holding the column pairs
// l + 32 i; every load of a row (cat, X, dOut, gamma2) is issued before its first reduction,
// so a row costs one memory round trip. Rows r = b n + i; the FMB rows i < n_f also give the
// MLP's upstream gradient (16-bit, [b][i][c] of the last Linear's output).
template <typename T>
__global__ void __launch_bounds__(256, 4) bw_out_ln_kernel(const T* __restrict__ cat, const T* __restrict__ X,
                                                           const float* __restrict__ dOut,
                                                           const float* __restrict__ g2, float* __restrict__ dy,
                                                           float* __restrict__ dx, T* __restrict__ dh_m,
                                                           float* __restrict__ dg2, float* __restrict__ db2,
                                                           int rows, int n, int n_f, int d, float eps) {
  __shared__ float2 sg[8][128], sb[8][128];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int pairs = d >> 1;
  float2 ag[4], ab[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) ag[i] = ab[i] = make_float2(0.f, 0.f);
  const float inv_d = 1.f / static_cast<float>(d);
  for (int r = blockIdx.x * 8 + warp; r < rows; r += gridDim.x * 8) {
    const int64_t o = static_cast<int64_t>(r) * d;
    float2 y[4], go[4];
    float s = 0.f;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int q = lane + 32 * i;
      y[i] = go[i] = make_float2(0.f, 0.f);
      if (q < pairs) {
        const uint32_t c2 = __ldg(reinterpret_cast<const unsigned int*>(cat + o) + q);
        const uint32_t x2 = __ldg(reinterpret_cast<const unsigned int*>(X + o) + q);
        go[i] = __ldg(reinterpret_cast<const float2*>(dOut + o) + q);
        y[i].x = Half16<T>::lo(c2) + Half16<T>::lo(x2);
        y[i].y = Half16<T>::hi(c2) + Half16<T>::hi(x2);
        s += y[i].x + y[i].y;
      }
    }
    const float mean = warp_sum(s) * inv_d;
    float v = 0.f;
#pragma unroll
    for (int i = 0; i < 4; ++i)
      if (lane + 32 * i < pairs) {
        const float a = y[i].x - mean, b = y[i].y - mean;
        v += a * a + b * b;
      }
    const float rs = rsqrtf(warp_sum(v) * inv_d + eps);
    float s1 = 0.f, s2 = 0.f;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int q = lane + 32 * i;
      if (q < pairs) {
        const float2 g = __ldg(reinterpret_cast<const float2*>(g2) + q);
        y[i].x = (y[i].x - mean) * rs;  // yhat
        y[i].y = (y[i].y - mean) * rs;
        ag[i].x += go[i].x * y[i].x;
        ag[i].y += go[i].y * y[i].y;
        ab[i].x += go[i].x;
        ab[i].y += go[i].y;
        go[i].x *= g.x;
        go[i].y *= g.y;
        s1 += go[i].x + go[i].y;
        s2 += go[i].x * y[i].x + go[i].y * y[i].y;
      }
    }
    const float m1 = warp_sum(s1) * inv_d, m2 = warp_sum(s2) * inv_d;
    const int b = r / n, i_row = r - b * n;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int q = lane + 32 * i;
      if (q < pairs) {
        const float gx = rs * (go[i].x - m1 - y[i].x * m2), gy = rs * (go[i].y - m1 - y[i].y * m2);
        reinterpret_cast<float2*>(dy + o)[q] = make_float2(tf32_round(gx), tf32_round(gy));  // tf32 operand
        reinterpret_cast<float2*>(dx + o)[q] = make_float2(gx, gy);  // the residual's share of dX
        if (i_row < n_f)
          reinterpret_cast<unsigned int*>(dh_m + (static_cast<int64_t>(b) * n_f + i_row) * d)[q] =
              Half16<T>::pack2(gx, gy);
      }
    }
  }
  // this CTA's partial d gamma2, d beta2
#pragma unroll
  for (int i = 0; i < 4; ++i)
    if (lane + 32 * i < pairs) {
      sg[warp][lane + 32 * i] = ag[i];
      sb[warp][lane + 32 * i] = ab[i];
    }
  __syncthreads();
  for (int q = threadIdx.x; q < pairs; q += blockDim.x) {
    float2 a = make_float2(0.f, 0.f), c = make_float2(0.f, 0.f);
#pragma unroll
    for (int w = 0; w < 8; ++w) {
      a.x += sg[w][q].x, a.y += sg[w][q].y;
      c.x += sb[w][q].x, c.y += sb[w][q].y;
    }
    atomicAdd(dg2 + 2 * q, a.x);
    atomicAdd(dg2 + 2 * q + 1, a.y);
    atomicAdd(db2 + 2 * q, c.x);
    atomicAdd(db2 + 2 * q + 1, c.y);
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

// The bias gradient of a Linear, with the ReLU derivative of its output applied first when h
// (the Linear's forward output) is given: z[r, c] = 0 where h[r, c] <= 0 (written back), then
// out[c] += sum over rows [r0, r1) of z[r, c]. Eight columns per thread (cols % 8 == 0),
// gridDim.x column blocks of 2048, gridDim.y row chunks.
template <typename T>
__global__ void __launch_bounds__(256) bw_mask_colsum_kernel(T* __restrict__ z, const T* __restrict__ h,
                                                             float* __restrict__ out, int64_t rows, int cols) {
  const int c = (blockIdx.x * blockDim.x + threadIdx.x) * 8;
  if (c >= cols) return;
  const int64_t chunk = (rows + gridDim.y - 1) / gridDim.y;
  const int64_t r0 = blockIdx.y * chunk, r1 = min(rows, r0 + chunk);
  float acc[8];
#pragma unroll
  for (int j = 0; j < 8; ++j) acc[j] = 0.f;
  for (int64_t r = r0; r < r1; ++r) {
    uint4* zp = reinterpret_cast<uint4*>(z + r * cols + c);
    uint4 g = *zp;
    uint32_t* gw = reinterpret_cast<uint32_t*>(&g);
    if (h) {
      const uint4 a = __ldg(reinterpret_cast<const uint4*>(h + r * cols + c));
      const uint32_t* aw = reinterpret_cast<const uint32_t*>(&a);
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        uint32_t mask = 0u;
        if (Half16<T>::lo(aw[j]) > 0.f) mask |= 0x0000FFFFu;
        if (Half16<T>::hi(aw[j]) > 0.f) mask |= 0xFFFF0000u;
        gw[j] &= mask;
      }
      *zp = g;
    }
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      acc[2 * j] += Half16<T>::lo(gw[j]);
      acc[2 * j + 1] += Half16<T>::hi(gw[j]);
    }
  }
  if (r1 > r0) {
#pragma unroll
    for (int j = 0; j < 8; ++j) atomicAdd(out + c + j, acc[j]);
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

// The same with the example in registers (nk a multiple of 4, at most 2048 V): 512 threads,
// V / 4 float4 of F and 4-value groups of dfh per thread, read once; the statistics are
// two-pass over the registers.
template <typename T, int V>
__global__ void __launch_bounds__(512, 1) bw_fmb_ln_reg_kernel(const float* __restrict__ F,
                                                               const T* __restrict__ dfh, float* __restrict__ dF,
                                                               int nk, float eps) {
  __shared__ float red[16];
  const int64_t base = static_cast<int64_t>(blockIdx.x) * nk;
  const float inv = 1.f / static_cast<float>(nk);
  float4 f[V / 4];
  uint2 g[V / 4];
  float s = 0.f;
#pragma unroll
  for (int j = 0; j < V / 4; ++j) {
    const int e = (j * 512 + static_cast<int>(threadIdx.x)) * 4;
    f[j] = make_float4(0.f, 0.f, 0.f, 0.f);
    g[j] = make_uint2(0u, 0u);
    if (e < nk) {
      f[j] = __ldg(reinterpret_cast<const float4*>(F + base + e));
      g[j] = __ldg(reinterpret_cast<const uint2*>(dfh + base + e));
      s += f[j].x + f[j].y + f[j].z + f[j].w;
    }
  }
  const float mean = bw_block_sum(s, red) * inv;
  float v = 0.f;
#pragma unroll
  for (int j = 0; j < V / 4; ++j) {
    if ((j * 512 + static_cast<int>(threadIdx.x)) * 4 < nk) {
      f[j].x -= mean, f[j].y -= mean, f[j].z -= mean, f[j].w -= mean;
      v += f[j].x * f[j].x + f[j].y * f[j].y + f[j].z * f[j].z + f[j].w * f[j].w;
    }
  }
  const float rs = rsqrtf(bw_block_sum(v, red) * inv + eps);
  float s1 = 0.f, s2 = 0.f;
#pragma unroll
  for (int j = 0; j < V / 4; ++j) {
    if ((j * 512 + static_cast<int>(threadIdx.x)) * 4 < nk) {
      f[j].x *= rs, f[j].y *= rs, f[j].z *= rs, f[j].w *= rs;  // fhat
      const float g0 = Half16<T>::lo(g[j].x), g1 = Half16<T>::hi(g[j].x), g2 = Half16<T>::lo(g[j].y),
                  g3 = Half16<T>::hi(g[j].y);
      s1 += g0 + g1 + g2 + g3;
      s2 += g0 * f[j].x + g1 * f[j].y + g2 * f[j].z + g3 * f[j].w;
    }
  }
  const float m1 = bw_block_sum(s1, red) * inv, m2 = bw_block_sum(s2, red) * inv;
#pragma unroll
  for (int j = 0; j < V / 4; ++j) {
    const int e = (j * 512 + static_cast<int>(threadIdx.x)) * 4;
    if (e < nk) {
      const float g0 = Half16<T>::lo(g[j].x), g1 = Half16<T>::hi(g[j].x), g2 = Half16<T>::lo(g[j].y),
                  g3 = Half16<T>::hi(g[j].y);
      // tf32 operands of the contractions
      *reinterpret_cast<float4*>(dF + base + e) = make_float4(tf32_round(rs * (g0 - m1 - f[j].x * m2)),
                                                              tf32_round(rs * (g1 - m1 - f[j].y * m2)),
                                                              tf32_round(rs * (g2 - m1 - f[j].z * m2)),
                                                              tf32_round(rs * (g3 - m1 - f[j].w * m2)));
    }
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

// The same, four columns per thread (cols % 4 == 0), rows unrolled by two.
template <typename TW>
__global__ void __launch_bounds__(256) bw_unfold4_kernel(float* __restrict__ dW0, const float* __restrict__ db0,
                                                         const TW* __restrict__ W0, const float* __restrict__ g1,
                                                         const float* __restrict__ b1, float* __restrict__ dg1,
                                                         float* __restrict__ db1, int rows, int cols) {
  const int c = (blockIdx.x * blockDim.x + threadIdx.x) * 4;
  if (c >= cols) return;
  const int chunk = (rows + gridDim.y - 1) / gridDim.y;
  const int r0 = blockIdx.y * chunk, r1 = min(rows, r0 + chunk);
  const float4 gc = g1 ? __ldg(reinterpret_cast<const float4*>(g1 + c)) : make_float4(1.f, 1.f, 1.f, 1.f);
  const float4 bc = b1 ? __ldg(reinterpret_cast<const float4*>(b1 + c)) : make_float4(0.f, 0.f, 0.f, 0.f);
  float4 sg = make_float4(0.f, 0.f, 0.f, 0.f), sb = sg;
#pragma unroll 2
  for (int r = r0; r < r1; ++r) {
    const int64_t o = static_cast<int64_t>(r) * cols + c;
    const uint2 w2 = __ldg(reinterpret_cast<const uint2*>(W0 + o));
    const float w0 = Half16<TW>::lo(w2.x), w1 = Half16<TW>::hi(w2.x), w2f = Half16<TW>::lo(w2.y),
                w3 = Half16<TW>::hi(w2.y);
    float4* gp = reinterpret_cast<float4*>(dW0 + o);
    const float4 gw = *gp;
    const float gb = __ldg(db0 + r);
    sg.x += gw.x * w0, sg.y += gw.y * w1, sg.z += gw.z * w2f, sg.w += gw.w * w3;
    sb.x += gb * w0, sb.y += gb * w1, sb.z += gb * w2f, sb.w += gb * w3;
    *gp = make_float4(gw.x * gc.x + gb * bc.x, gw.y * gc.y + gb * bc.y, gw.z * gc.z + gb * bc.z, gw.w * gc.w + gb * bc.w);
  }
  if (r1 > r0) {
    atomicAdd(dg1 + c, sg.x), atomicAdd(dg1 + c + 1, sg.y), atomicAdd(dg1 + c + 2, sg.z), atomicAdd(dg1 + c + 3, sg.w);
    atomicAdd(db1 + c, sb.x), atomicAdd(db1 + c + 1, sb.y), atomicAdd(db1 + c + 2, sb.z), atomicAdd(db1 + c + 3, sb.w);
  }
}

}  // namespace wk
