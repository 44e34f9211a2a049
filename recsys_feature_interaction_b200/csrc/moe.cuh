// moe.cuh -- the two steps a Wukong mixture of experts adds around its experts (Kunlun
// page, section 2.3, "Wukong Mixture of Experts": several Wukong modules run in
// parallel as the experts of one layer). With the experts' layers computed by the
// plain Wukong kernels up to their concatenation, the MoE layer is
//
//   g[b, :]    = softmax( W_g vec(X_b) + b_g )                      (moe_gate_kernel)
//   out[b, i]  = sum_e g[b, e] * ( LN( cat_e[b, i] + X_b[i] ) * gamma_e + beta_e )
//                                                                  (moe_combine_kernel)
//
// for every example b and embedding row i: each expert's own residual + LayerNorm,
// mixed by the gate, in one pass that reads every expert's concat buffer and the layer
// input once and writes the layer output once.
#pragma once

#include "res_ln.cuh"

namespace wk {

constexpr int MOE_MAX_E = 8;  // experts per MoE layer
constexpr int MOE_GATE_EB = 4;  // examples per gate block iteration (W_g read once for them)

struct MoePtrs {
  const void* cat[MOE_MAX_E];     // [rows, d] per expert (operand type)
  const float* gamma[MOE_MAX_E];  // [d] per expert
  const float* beta[MOE_MAX_E];   // [d] per expert
};

// Gate logits and softmax. X [batch, nd] and W_g [E, nd] in T (nd a multiple of 8,
// 16-byte aligned rows), b_g [E] fp32 or null, g [batch, E] fp32. A block takes EB
// examples at a time: every thread walks 16-byte vectors of the flattened input with
// the block's stride, two strides per step with all their loads issued before any
// arithmetic (more bytes in flight per thread), reads each W_g vector once for the EB
// examples and keeps EB x E fp32 partial dot products; warps reduce by shuffles, then
// through shared memory. E is a template parameter so that the accumulators and the
// W_g vectors in flight take exactly the registers the expert count needs.
template <typename T, int E>
__global__ void __launch_bounds__(256) moe_gate_kernel(const T* __restrict__ X, const T* __restrict__ Wg,
                                                      const float* __restrict__ bg, float* __restrict__ g,
                                                      int64_t batch, int64_t nd) {
  constexpr int EB = MOE_GATE_EB;
  constexpr int UNR = 2;
  __shared__ float red[8][EB][E];
  const int lane = threadIdx.x & 31;
  const int warp = threadIdx.x >> 5;
  const int64_t nvec = nd / 8;
  const uint4 zero = make_uint4(0u, 0u, 0u, 0u);
  for (int64_t b0 = static_cast<int64_t>(blockIdx.x) * EB; b0 < batch; b0 += static_cast<int64_t>(gridDim.x) * EB) {
    float acc[EB][E];
#pragma unroll
    for (int u = 0; u < EB; ++u)
#pragma unroll
      for (int e = 0; e < E; ++e) acc[u][e] = 0.f;
    for (int64_t v0 = threadIdx.x; v0 < nvec; v0 += UNR * blockDim.x) {
      uint4 xv[UNR][EB], wv[UNR][E];
#pragma unroll
      for (int s = 0; s < UNR; ++s) {
        const int64_t v = v0 + s * blockDim.x;
        const bool in = v < nvec;
#pragma unroll
        for (int u = 0; u < EB; ++u)
          xv[s][u] = (in && b0 + u < batch) ? __ldg(reinterpret_cast<const uint4*>(X + (b0 + u) * nd + v * 8)) : zero;
#pragma unroll
        for (int e = 0; e < E; ++e)
          wv[s][e] = in ? __ldg(reinterpret_cast<const uint4*>(Wg + static_cast<int64_t>(e) * nd + v * 8)) : zero;
      }
#pragma unroll
      for (int s = 0; s < UNR; ++s)
#pragma unroll
        for (int u = 0; u < EB; ++u) {
          float x8[8];
          Vec8<T>::unpack(xv[s][u], x8);
#pragma unroll
          for (int e = 0; e < E; ++e) {
            float w8[8];
            Vec8<T>::unpack(wv[s][e], w8);
#pragma unroll
            for (int j = 0; j < 8; ++j) acc[u][e] = fmaf(w8[j], x8[j], acc[u][e]);
          }
        }
    }
#pragma unroll
    for (int u = 0; u < EB; ++u)
#pragma unroll
      for (int e = 0; e < E; ++e) {
        float s = acc[u][e];
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
        if (lane == 0) red[warp][u][e] = s;
      }
    __syncthreads();
    if (threadIdx.x < EB && b0 + threadIdx.x < batch) {
      const int u = threadIdx.x;
      const int nw = blockDim.x >> 5;
      float z[E];
      float mx = -INFINITY;
#pragma unroll
      for (int e = 0; e < E; ++e) {
        float s = bg ? bg[e] : 0.f;
        for (int w = 0; w < nw; ++w) s += red[w][u][e];
        z[e] = s;
        mx = fmaxf(mx, s);
      }
      float tot = 0.f;
#pragma unroll
      for (int e = 0; e < E; ++e) {
        z[e] = expf(z[e] - mx);
        tot += z[e];
      }
      const float inv = 1.0f / tot;
#pragma unroll
      for (int e = 0; e < E; ++e) g[(b0 + u) * E + e] = z[e] * inv;
    }
    __syncthreads();
  }
}

// The mixture of the experts' residual + LayerNorm outputs. rows = batch * n rows of
// d values; cat_e and x in the 16-bit type T, out in TO, g [batch, E] fp32. Lane
// layout as in res_ln_kernel: G lanes per row (G a power of two dividing d/8), each
// lane owning VPL 16-byte vectors. Per row the residual is loaded once and kept as
// packed 16-bit words, each expert's concat row is loaded once, one expert ahead of
// the arithmetic (all VPL vectors at once), and kept packed too; each expert's statistics are two
// fp32 passes over the unpacked values (registers: the fp32 mixture plus the packed
// rows, which leaves room for two 256-thread blocks per SM at d = 160).
template <int D, typename T, typename TO>
__global__ void __launch_bounds__(256, 2) moe_combine_kernel(const MoePtrs p, const T* __restrict__ x,
                                                         const float* __restrict__ g, TO* __restrict__ out,
                                                         int64_t rows, int n, int E, float eps) {
  static_assert(sizeof(T) == 2, "16-bit operands");
  constexpr int VPR = D / 8;
  constexpr int G = res_ln_lanes(VPR);
  constexpr int VPL = VPR / G;
  constexpr int RPW = 32 / G;
  const int lane = threadIdx.x & 31;
  const int warp = threadIdx.x >> 5;
  const int nwarps = blockDim.x >> 5;
  const int sub = lane / G;
  const int v0 = lane % G;
  const uint4 zero = make_uint4(0u, 0u, 0u, 0u);
  const int64_t step = static_cast<int64_t>(gridDim.x) * nwarps * RPW;
  for (int64_t r = (static_cast<int64_t>(blockIdx.x) * nwarps + warp) * RPW + sub; r - sub < rows; r += step) {
    const bool ok = r < rows;
    uint4 xr[VPL];
    float acc[VPL][8];
#pragma unroll
    for (int k = 0; k < VPL; ++k) {
      xr[k] = ok ? __ldg(reinterpret_cast<const uint4*>(x + r * D + (v0 + k * G) * 8)) : zero;
#pragma unroll
      for (int j = 0; j < 8; ++j) acc[k][j] = 0.f;
    }
    const int64_t b = ok ? r / n : 0;
    uint4 cn[VPL];  // the next expert's concat row, loaded one expert ahead
#pragma unroll
    for (int k = 0; k < VPL; ++k)
      cn[k] = ok ? __ldg(reinterpret_cast<const uint4*>(static_cast<const T*>(p.cat[0]) + r * D + (v0 + k * G) * 8))
                 : zero;
    for (int e = 0; e < E; ++e) {
      uint4 cr[VPL];
#pragma unroll
      for (int k = 0; k < VPL; ++k) cr[k] = cn[k];
      if (e + 1 < E) {
        const T* nxt = static_cast<const T*>(p.cat[e + 1]);
#pragma unroll
        for (int k = 0; k < VPL; ++k)
          cn[k] = ok ? __ldg(reinterpret_cast<const uint4*>(nxt + r * D + (v0 + k * G) * 8)) : zero;
      }
      // y = cat + x is recomputed from the packed words in each pass instead of being
      // held as fp32 (the unpack is a shift or a convert per element)
      float s = 0.f;
#pragma unroll
      for (int k = 0; k < VPL; ++k) {
        float c8[8], x8[8];
        Vec8<T>::unpack(cr[k], c8);
        Vec8<T>::unpack(xr[k], x8);
#pragma unroll
        for (int j = 0; j < 8; ++j) s += c8[j] + x8[j];
      }
#pragma unroll
      for (int o = G / 2; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
      const float mean = s * (1.0f / D);
      float q = 0.f;
#pragma unroll
      for (int k = 0; k < VPL; ++k) {
        float c8[8], x8[8];
        Vec8<T>::unpack(cr[k], c8);
        Vec8<T>::unpack(xr[k], x8);
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          const float dv = (c8[j] + x8[j]) - mean;
          q += dv * dv;
        }
      }
#pragma unroll
      for (int o = G / 2; o > 0; o >>= 1) q += __shfl_xor_sync(0xffffffffu, q, o);
      const float rstd = rsqrtf(q * (1.0f / D) + eps);
      const float ge = ok ? __ldg(g + b * E + e) : 0.f;
      const float* gam = p.gamma[e];
      const float* bet = p.beta[e];
#pragma unroll
      for (int k = 0; k < VPL; ++k) {
        const int c = (v0 + k * G) * 8;
        float c8[8], x8[8];
        Vec8<T>::unpack(cr[k], c8);
        Vec8<T>::unpack(xr[k], x8);
        const float4 g0 = __ldg(reinterpret_cast<const float4*>(gam + c));
        const float4 g1 = __ldg(reinterpret_cast<const float4*>(gam + c) + 1);
        const float4 b0 = __ldg(reinterpret_cast<const float4*>(bet + c));
        const float4 b1 = __ldg(reinterpret_cast<const float4*>(bet + c) + 1);
        const float gg[8] = {g0.x, g0.y, g0.z, g0.w, g1.x, g1.y, g1.z, g1.w};
        const float bb[8] = {b0.x, b0.y, b0.z, b0.w, b1.x, b1.y, b1.z, b1.w};
#pragma unroll
        for (int j = 0; j < 8; ++j) acc[k][j] = fmaf(ge, ((c8[j] + x8[j]) - mean) * rstd * gg[j] + bb[j], acc[k][j]);
      }
    }
    if (ok) {
#pragma unroll
      for (int k = 0; k < VPL; ++k) Vec8<TO>::store(out + r * D + (v0 + k * G) * 8, acc[k]);
    }
  }
}

}  // namespace wk
