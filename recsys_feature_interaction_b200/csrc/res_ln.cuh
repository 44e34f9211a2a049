// res_ln.cuh -- concat + residual + LayerNorm of each embedding row (the end of a
// Wukong layer: the FMB and LCB blocks are concatenated, the layer input is added
// back and every output embedding is normalised; Wukong page, section 2.2).
//
//   out[r, :] = LN( cat[r, :] + x[r, :] ) * gamma + beta,   r < rows, d values per row
//
// HBM-bound: each element is read twice and written once, so the kernel moves
// 16-byte vectors (8 elements); a row is split over G lanes (G a power of two
// dividing d/8, so no lane idles: d = 160 -> 4 lanes x 5 vectors), 32/G rows per
// warp, several rows in flight per lane, mean and variance by two passes over
// registers (fp32) with xor shuffles inside each lane group, gamma/beta read
// through L1. The grid is a multiple of the SM count.
#pragma once

#include "common.cuh"

namespace wk {

template <typename T>
struct Vec8;

template <>
struct Vec8<float> {
  static __device__ __forceinline__ void load(const float* p, float (&v)[8]) {
    float4 a = __ldg(reinterpret_cast<const float4*>(p));
    float4 b = __ldg(reinterpret_cast<const float4*>(p) + 1);
    v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
    v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
  }
  static __device__ __forceinline__ void store(float* p, const float (&v)[8]) {
    reinterpret_cast<float4*>(p)[0] = make_float4(v[0], v[1], v[2], v[3]);
    reinterpret_cast<float4*>(p)[1] = make_float4(v[4], v[5], v[6], v[7]);
  }
};

template <>
struct Vec8<__nv_bfloat16> {
  static __device__ __forceinline__ void unpack(const uint4& a, float (&v)[8]) {
    v[0] = bf16_lo(a.x); v[1] = bf16_hi(a.x); v[2] = bf16_lo(a.y); v[3] = bf16_hi(a.y);
    v[4] = bf16_lo(a.z); v[5] = bf16_hi(a.z); v[6] = bf16_lo(a.w); v[7] = bf16_hi(a.w);
  }
  static __device__ __forceinline__ void load(const __nv_bfloat16* p, float (&v)[8]) {
    unpack(__ldg(reinterpret_cast<const uint4*>(p)), v);
  }
  // p: 16-byte aligned shared memory
  static __device__ __forceinline__ void load_shared(const uint8_t* p, float (&v)[8]) {
    unpack(*reinterpret_cast<const uint4*>(p), v);
  }
  static __device__ __forceinline__ void store(__nv_bfloat16* p, const float (&v)[8]) {
    uint4 a;
    a.x = pack_bf16x2(v[0], v[1]);
    a.y = pack_bf16x2(v[2], v[3]);
    a.z = pack_bf16x2(v[4], v[5]);
    a.w = pack_bf16x2(v[6], v[7]);
    *reinterpret_cast<uint4*>(p) = a;
  }
};

template <>
struct Vec8<__half> {
  static __device__ __forceinline__ void unpack(const uint4& a, float (&v)[8]) {
    const uint32_t w[4] = {a.x, a.y, a.z, a.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      v[2 * i] = Half16<__half>::lo(w[i]);
      v[2 * i + 1] = Half16<__half>::hi(w[i]);
    }
  }
  static __device__ __forceinline__ void load(const __half* p, float (&v)[8]) {
    unpack(__ldg(reinterpret_cast<const uint4*>(p)), v);
  }
  // p: 16-byte aligned shared memory
  static __device__ __forceinline__ void load_shared(const uint8_t* p, float (&v)[8]) {
    unpack(*reinterpret_cast<const uint4*>(p), v);
  }
  static __device__ __forceinline__ void store(__half* p, const float (&v)[8]) {
    uint4 a;
    a.x = Half16<__half>::pack2(v[0], v[1]);
    a.y = Half16<__half>::pack2(v[2], v[3]);
    a.z = Half16<__half>::pack2(v[4], v[5]);
    a.w = Half16<__half>::pack2(v[6], v[7]);
    *reinterpret_cast<uint4*>(p) = a;
  }
};

constexpr int pow2_ceil(int v) {
  int p = 1;
  while (p < v) p <<= 1;
  return p;
}

// Lanes per row: the largest power of two <= 32 that divides the row's vector
// count, so every lane of the warp owns the same number of 16-byte vectors.
constexpr int res_ln_lanes(int vpr) {
  int g = 1;
  while (g * 2 <= 32 && vpr % (g * 2) == 0) g *= 2;
  return g;
}

// TC: concat element type, TR: residual element type, TO: output type.
// Lane j of a row's group owns vectors j, j + G, j + 2G, ... (coalesced: the G
// lanes of a row touch G consecutive 16-byte units per access).
template <int D, typename TC, typename TR, typename TO>
__global__ void __launch_bounds__(256) res_ln_kernel(const TC* __restrict__ cat, const TR* __restrict__ x,
                                                     const float* __restrict__ gamma,
                                                     const float* __restrict__ beta, TO* __restrict__ out,
                                                     float* __restrict__ out32, int64_t rows, float eps) {
  constexpr int VPR = D / 8;                 // 16-byte vectors (8 elements) per row
  constexpr int G = res_ln_lanes(VPR);       // lanes per row
  constexpr int VPL = VPR / G;               // vectors per lane
  static_assert(D % 8 == 0, "d must be a multiple of 8");
  constexpr int RPW = 32 / G;                // rows per warp step
  constexpr int UNROLL = (VPL >= 4) ? 2 : 4; // rows in flight per lane
  const int lane = threadIdx.x & 31;
  const int warp = threadIdx.x >> 5;
  const int nwarps = blockDim.x >> 5;
  const int sub = lane / G;                  // row within the warp step
  const int v0 = lane % G;                   // first vector of this lane

  const int64_t step = static_cast<int64_t>(gridDim.x) * nwarps * RPW * UNROLL;
  for (int64_t base = (static_cast<int64_t>(blockIdx.x) * nwarps + warp) * RPW * UNROLL; base < rows;
       base += step) {
    float y[UNROLL][VPL][8];
    bool ok[UNROLL];
#pragma unroll
    for (int u = 0; u < UNROLL; ++u) {
      const int64_t r = base + u * RPW + sub;
      ok[u] = r < rows;
#pragma unroll
      for (int k = 0; k < VPL; ++k) {
        if (ok[u]) {
          float c8[8], x8[8];
          const int e = (v0 + k * G) * 8;
          Vec8<TC>::load(cat + r * D + e, c8);
          Vec8<TR>::load(x + r * D + e, x8);
#pragma unroll
          for (int j = 0; j < 8; ++j) y[u][k][j] = c8[j] + x8[j];
        } else {
#pragma unroll
          for (int j = 0; j < 8; ++j) y[u][k][j] = 0.f;
        }
      }
    }
#pragma unroll
    for (int u = 0; u < UNROLL; ++u) {
      float s = 0.f;
#pragma unroll
      for (int k = 0; k < VPL; ++k)
#pragma unroll
        for (int j = 0; j < 8; ++j) s += y[u][k][j];
#pragma unroll
      for (int o = G / 2; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
      const float mean = s * (1.0f / D);
      float q = 0.f;
#pragma unroll
      for (int k = 0; k < VPL; ++k)
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          const float dv = y[u][k][j] - mean;
          q += dv * dv;
        }
#pragma unroll
      for (int o = G / 2; o > 0; o >>= 1) q += __shfl_xor_sync(0xffffffffu, q, o);
      const float rstd = rsqrtf(q * (1.0f / D) + eps);
      if (ok[u]) {
        const int64_t r = base + u * RPW + sub;
#pragma unroll
        for (int k = 0; k < VPL; ++k) {
          const int e = (v0 + k * G) * 8;
          const float4 g0 = __ldg(reinterpret_cast<const float4*>(gamma + e));
          const float4 g1 = __ldg(reinterpret_cast<const float4*>(gamma + e) + 1);
          const float4 b0 = __ldg(reinterpret_cast<const float4*>(beta + e));
          const float4 b1 = __ldg(reinterpret_cast<const float4*>(beta + e) + 1);
          const float gg[8] = {g0.x, g0.y, g0.z, g0.w, g1.x, g1.y, g1.z, g1.w};
          const float bb[8] = {b0.x, b0.y, b0.z, b0.w, b1.x, b1.y, b1.z, b1.w};
          float o8[8];
#pragma unroll
          for (int j = 0; j < 8; ++j) o8[j] = (y[u][k][j] - mean) * rstd * gg[j] + bb[j];
          Vec8<TO>::store(out + r * D + e, o8);
          if (out32) Vec8<float>::store(out32 + r * D + e, o8);
        }
      }
    }
  }
}

}  // namespace wk
