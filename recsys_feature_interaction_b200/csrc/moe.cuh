// moe.cuh -- the two steps a Wukong mixture of experts adds around its experts (Kunlun
// page, section 2.3, "Wukong Mixture of Experts": several Wukong modules run in
// parallel as the experts of one layer). With the experts' layers computed by the
// plain Wukong kernels up to their concatenation, the MoE layer is
//
//   g[b, :]    = softmax( W_g vec(X_b) + b_g )                      (moe_gate_kernel)
//   out[b, i]  = sum_e g[b, e] * ( LN( cat_e[b, i] + X_b[i] ) * gamma_e + beta_e )
//                                                                  (moe_combine_ring_kernel)
//
// for every example b and embedding row i: each expert's own residual + LayerNorm,
// mixed by the gate, in one pass that reads every expert's concat buffer and the layer
// input once and writes the layer output once.
#pragma once

#include "res_ln.cuh"
#include "res_ln_ring.cuh"

namespace wk {

constexpr int MOE_MAX_E = 8;  // experts per MoE layer

struct MoePtrs {
  const void* cat[MOE_MAX_E];     // [rows, d] per expert (operand type)
  const float* gamma[MOE_MAX_E];  // [d] per expert
  const float* beta[MOE_MAX_E];   // [d] per expert
};

// Gate logits and softmax. X [batch, nd] and W_g [E, nd] in T (nd a multiple of 8,
// 16-byte aligned rows), b_g [E] fp32 or null, g [batch, E] fp32.
//
// A block of eight warps takes eight examples (one per warp) and walks vec(X) in
// chunks of gate_chunk<E>() elements: the block stages that chunk of all E gate rows
// in shared memory once, converted to fp32 (two planes of float4, so that consecutive
// lanes read consecutive 16 bytes), and every warp streams its example's chunk of X
// from HBM (16-byte loads, the next chunk's loads issued before this chunk's
// arithmetic) and accumulates E fp32 dot products. W_g is read from L2 once per block
// and chunk instead of once per example; X is read once. A shuffle reduction and an
// fp32 softmax end each example.
template <int E>
constexpr int gate_chunk() {
  // E * chunk * 4 bytes <= 32 KB of fp32 W_g; a multiple of 256 elements (every lane
  // owns the same number of 16-byte vectors of a chunk)
  return ((8192 / E) / 256 * 256) < 2048 ? ((8192 / E) / 256 * 256) : 2048;
}

template <typename T, int E>
__global__ void __launch_bounds__(256) moe_gate_kernel(const T* __restrict__ X, const T* __restrict__ Wg,
                                                      const float* __restrict__ bg, float* __restrict__ g,
                                                      int64_t batch, int64_t nd) {
  constexpr int CH = gate_chunk<E>();
  constexpr int VC = CH / 8;   // 16-byte vectors per chunk row
  constexpr int VL = VC / 32;  // vectors per lane
  static_assert(CH % 256 == 0 && VL >= 1, "chunk");
  __shared__ float4 ws[E][2 * VC];  // [e][v] = elements 0..3 of vector v, [e][VC + v] = elements 4..7
  const int lane = threadIdx.x & 31;
  const int warp = threadIdx.x >> 5;
  const uint4 zero = make_uint4(0u, 0u, 0u, 0u);
  for (int64_t base = static_cast<int64_t>(blockIdx.x) * 8; base < batch; base += static_cast<int64_t>(gridDim.x) * 8) {
    const int64_t b = base + warp;
    float acc[E];
#pragma unroll
    for (int e = 0; e < E; ++e) acc[e] = 0.f;
    // X chunks are loaded one chunk ahead: chunk c + 1's loads are in flight while
    // chunk c's W_g is staged and its products are taken
    uint4 xn[VL];
#pragma unroll
    for (int i = 0; i < VL; ++i) {
      const int v = lane + 32 * i;
      xn[i] = (b < batch && v * 8 < nd) ? __ldg(reinterpret_cast<const uint4*>(X + b * nd + v * 8)) : zero;
    }
    for (int64_t c0 = 0; c0 < nd; c0 += CH) {
      uint4 xv[VL];
#pragma unroll
      for (int i = 0; i < VL; ++i) xv[i] = xn[i];
      if (c0 + CH < nd) {
#pragma unroll
        for (int i = 0; i < VL; ++i) {
          const int v = lane + 32 * i;
          xn[i] = (b < batch && c0 + CH + v * 8 < nd)
                      ? __ldg(reinterpret_cast<const uint4*>(X + b * nd + c0 + CH + v * 8))
                      : zero;
        }
      }
      __syncthreads();  // the previous chunk of W_g has been read by every warp
      for (int i = threadIdx.x; i < E * VC; i += blockDim.x) {
        const int e = i / VC, v = i % VC;
        float w8[8];
        if (c0 + v * 8 < nd) {
          Vec8<T>::load(Wg + static_cast<int64_t>(e) * nd + c0 + v * 8, w8);
        } else {
#pragma unroll
          for (int j = 0; j < 8; ++j) w8[j] = 0.f;
        }
        ws[e][v] = make_float4(w8[0], w8[1], w8[2], w8[3]);
        ws[e][VC + v] = make_float4(w8[4], w8[5], w8[6], w8[7]);
      }
      __syncthreads();
#pragma unroll
      for (int i = 0; i < VL; ++i) {
        const int v = lane + 32 * i;
        float x8[8];
        Vec8<T>::unpack(xv[i], x8);
#pragma unroll
        for (int e = 0; e < E; ++e) {
          const float4 w0 = ws[e][v], w1 = ws[e][VC + v];
          acc[e] = fmaf(w0.x, x8[0], acc[e]);
          acc[e] = fmaf(w0.y, x8[1], acc[e]);
          acc[e] = fmaf(w0.z, x8[2], acc[e]);
          acc[e] = fmaf(w0.w, x8[3], acc[e]);
          acc[e] = fmaf(w1.x, x8[4], acc[e]);
          acc[e] = fmaf(w1.y, x8[5], acc[e]);
          acc[e] = fmaf(w1.z, x8[6], acc[e]);
          acc[e] = fmaf(w1.w, x8[7], acc[e]);
        }
      }
    }
    float z[E];
    float mx = -INFINITY;
#pragma unroll
    for (int e = 0; e < E; ++e) {
      float s = acc[e];
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
      z[e] = s + (bg ? __ldg(bg + e) : 0.f);
      mx = fmaxf(mx, z[e]);
    }
    if (lane == 0 && b < batch) {
      float tot = 0.f;
#pragma unroll
      for (int e = 0; e < E; ++e) {
        z[e] = expf(z[e] - mx);
        tot += z[e];
      }
      const float inv = 1.0f / tot;
#pragma unroll
      for (int e = 0; e < E; ++e) g[b * E + e] = z[e] * inv;
    }
  }
}

// The mixture of the experts' residual + LayerNorm outputs, rows = batch * n rows of d
// values (cat_e and x in the 16-bit type T, out in TO, g [batch, E] fp32), fed by bulk
// copies (the design of res_ln_ring_kernel): the rows are walked in blocks of R rows, and for each block the producer thread streams E + 1
// contiguous byte ranges -- the layer input's rows, then every expert's concat rows --
// into consecutive slots of a ring in shared memory (untiled cp.async.bulk, one
// mbarrier per slot). Eight consumer warps move the input rows into registers and
// release their slot, then walk the experts' slots in order, releasing each expert
// slot after its residual + LayerNorm has been added into the fp32 mixture
// (registers), and store the output rows. The ring holds at least E + 2 slots, so
// the next block's copies are in flight while a block is reduced. Every wait is
// bounded.
template <int D>
struct MoeRing {
  static_assert(D % 8 == 0, "d must be a multiple of 8");
  static constexpr int VPR = D / 8;
  static constexpr int G = res_ln_lanes(VPR);
  static constexpr int VPL = VPR / G;
  static constexpr int RPW = 32 / G;
  static constexpr int CWARPS = 8;
  static constexpr int ROW_B = D * 2;
  static constexpr int U_RAW = 16384 / (CWARPS * RPW * ROW_B);
  static constexpr int U = U_RAW < 1 ? 1 : U_RAW;  // warp steps per block
  static constexpr int R = CWARPS * RPW * U;       // rows per block
  static constexpr int TILE_B = R * ROW_B;         // bytes per slot
  static constexpr int SLOTS_RAW = (200 * 1024) / TILE_B;
  static constexpr int SLOTS = SLOTS_RAW > 16 ? 16 : SLOTS_RAW;
  static constexpr int THREADS = 32 * (CWARPS + 1);
  static constexpr int SMEM = 128 + SLOTS * TILE_B + 2 * SLOTS * 8;
  static_assert(SLOTS >= MOE_MAX_E + 2, "ring too short for the largest expert count");
  static_assert(TILE_B % 16 == 0, "bulk copy granularity");
};

template <int D, typename T, typename TO>
__global__ void __launch_bounds__(MoeRing<D>::THREADS, 1)
    moe_combine_ring_kernel(const MoePtrs p, const T* __restrict__ x, const float* __restrict__ g,
                            TO* __restrict__ out, int64_t rows, int n, int E, float eps, unsigned* status) {
  using C = MoeRing<D>;
  static_assert(sizeof(T) == 2, "16-bit operands");
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = smem_raw + ((128u - (smem_u32(smem_raw) & 127u)) & 127u);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + C::SLOTS * C::TILE_B);
  uint64_t* empty = full + C::SLOTS;
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int s = 0; s < C::SLOTS; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], C::CWARPS);
    }
    fence_mbar_init();
  }
  __syncthreads();
  const int64_t ntiles = (rows + C::R - 1) / C::R;

  if (warp == 0) {
    // ---------------------------------------------------------------- producer
    if (lane == 0) {
      int slot = 0;
      uint32_t phase = 0, used = 0, par = 0;  // per slot: issued at least once, parity of the last issue
      bool ok = true;
      for (int64_t t = blockIdx.x; ok && t < ntiles; t += gridDim.x) {
        const int64_t r0 = t * C::R;
        const int64_t nr = rows - r0 < C::R ? rows - r0 : C::R;
        const uint32_t bytes = static_cast<uint32_t>(nr) * C::ROW_B;
        for (int j = 0; j <= E; ++j) {
          if (!mbar_wait(&empty[slot], phase ^ 1u, status)) {
            ok = false;
            break;
          }
          used |= 1u << slot;
          par = (par & ~(1u << slot)) | (phase << slot);
          const T* src = (j == 0) ? x : static_cast<const T*>(p.cat[j - 1]);
          mbar_arrive_expect_tx(&full[slot], bytes);
          bulk_load(smem + slot * C::TILE_B, src + r0 * D, bytes, &full[slot]);
          if (++slot == C::SLOTS) {
            slot = 0;
            phase ^= 1u;
          }
        }
      }
      // every issued copy lands before the CTA's shared memory is released
      for (int s = 0; s < C::SLOTS; ++s)
        if (used & (1u << s)) mbar_drain(&full[s], (par >> s) & 1u, status);
    }
    return;
  }

  // ------------------------------------------------------------------ consumers
  // The layer input's rows go to fp32 registers and their slot is released at once;
  // each expert's concat rows are read from shared memory once into fp32 registers,
  // normalised by two passes over registers and added into the mixture.
  const int cw = warp - 1;
  const int sub = lane / C::G;
  const int v0 = lane % C::G;
  int slot = 0;
  uint32_t phase = 0;
  bool ok = true;
  for (int64_t t = blockIdx.x; ok && t < ntiles; t += gridDim.x) {
    const int64_t r0 = t * C::R;
    const int sx = slot;
    if (!mbar_wait(&full[sx], phase, status)) break;
    if (++slot == C::SLOTS) {
      slot = 0;
      phase ^= 1u;
    }
    float xf[C::U][C::VPL][8], acc[C::U][C::VPL][8];
    {
      const uint8_t* tx = smem + sx * C::TILE_B;
#pragma unroll
      for (int u = 0; u < C::U; ++u) {
        const int lr = (u * C::CWARPS + cw) * C::RPW + sub;
#pragma unroll
        for (int k = 0; k < C::VPL; ++k) {
          Vec8<T>::load_shared(tx + lr * C::ROW_B + (v0 + k * C::G) * 16, xf[u][k]);
#pragma unroll
          for (int j = 0; j < 8; ++j) acc[u][k][j] = 0.f;
        }
      }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&empty[sx]);  // the layer input's rows are in registers
    for (int e = 0; e < E; ++e) {
      const int se = slot;
      if (!mbar_wait(&full[se], phase, status)) {
        ok = false;
        break;
      }
      if (++slot == C::SLOTS) {
        slot = 0;
        phase ^= 1u;
      }
      const uint8_t* tc = smem + se * C::TILE_B;
      const float* gam = p.gamma[e];
      const float* bet = p.beta[e];
#pragma unroll
      for (int u = 0; u < C::U; ++u) {
        const int lr = (u * C::CWARPS + cw) * C::RPW + sub;
        const bool in = r0 + lr < rows;
        float y[C::VPL][8];
        float s = 0.f;
#pragma unroll
        for (int k = 0; k < C::VPL; ++k) {
          Vec8<T>::load_shared(tc + lr * C::ROW_B + (v0 + k * C::G) * 16, y[k]);
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            y[k][j] = in ? y[k][j] + xf[u][k][j] : 0.f;
            s += y[k][j];
          }
        }
#pragma unroll
        for (int o = C::G / 2; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
        const float mean = s * (1.0f / D);
        float q = 0.f;
#pragma unroll
        for (int k = 0; k < C::VPL; ++k)
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            const float dv = y[k][j] - mean;
            q = fmaf(dv, dv, q);
          }
#pragma unroll
        for (int o = C::G / 2; o > 0; o >>= 1) q += __shfl_xor_sync(0xffffffffu, q, o);
        const float rstd = rsqrtf(q * (1.0f / D) + eps);
        const float ge = in ? __ldg(g + ((r0 + lr) / n) * E + e) : 0.f;
        const float grs = ge * rstd;
#pragma unroll
        for (int k = 0; k < C::VPL; ++k) {
          const int c = (v0 + k * C::G) * 8;
          const float4 g0 = __ldg(reinterpret_cast<const float4*>(gam + c));
          const float4 g1 = __ldg(reinterpret_cast<const float4*>(gam + c) + 1);
          const float4 b0 = __ldg(reinterpret_cast<const float4*>(bet + c));
          const float4 b1 = __ldg(reinterpret_cast<const float4*>(bet + c) + 1);
          const float gg[8] = {g0.x, g0.y, g0.z, g0.w, g1.x, g1.y, g1.z, g1.w};
          const float bb[8] = {b0.x, b0.y, b0.z, b0.w, b1.x, b1.y, b1.z, b1.w};
          // g_e * (LN(y) * gamma + beta) = (y - mean) * (g_e rstd gamma) + g_e beta
#pragma unroll
          for (int j = 0; j < 8; ++j)
            acc[u][k][j] = fmaf(y[k][j] - mean, grs * gg[j], fmaf(ge, bb[j], acc[u][k][j]));
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[se]);  // this warp is done reading the expert's rows
    }
    if (!ok) break;
#pragma unroll
    for (int u = 0; u < C::U; ++u) {
      const int lr = (u * C::CWARPS + cw) * C::RPW + sub;
      if (r0 + lr < rows) {
        TO* orow = out + (r0 + lr) * D;
#pragma unroll
        for (int k = 0; k < C::VPL; ++k) Vec8<TO>::store(orow + (v0 + k * C::G) * 8, acc[u][k]);
      }
    }
  }
}

}  // namespace wk
