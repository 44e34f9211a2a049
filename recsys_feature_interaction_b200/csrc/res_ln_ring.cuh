// res_ln_ring.cuh -- concat + residual + LayerNorm of each embedding row, fed by
// bulk copies (the end of a Wukong layer: the FMB and LCB blocks are concatenated,
// the layer input is added back and every output embedding is normalised; Wukong
// page, section 2.2):
//
//   out[r, :] = LN( cat[r, :] + x[r, :] ) * gamma + beta,   r < rows, d values per row
//
// (x may be null: then out = LN(cat) * gamma + beta, the output LayerNorm of a stack whose
// last layer has already added its residual into cat).
//
// HBM-bound (each element read twice, written once). A block of R consecutive rows
// is one contiguous byte range in both inputs, so one persistent CTA per SM keeps a
// ring of STAGES such blocks in flight with untiled bulk copies (cp.async.bulk, one
// per input per stage, completion counted on an mbarrier): one producer thread
// issues them, eight consumer warps normalise rows out of shared memory and store
// 16-byte vectors of the output. The bytes in flight no longer depend on how many
// registers the arithmetic needs. Rows split over G lanes as in res_ln.cuh; gamma
// and beta live in registers for the whole kernel. Every wait is bounded.
#pragma once

#include "common.cuh"
#include "res_ln.cuh"

namespace wk {

template <int D>
struct ResLnRing {
  static_assert(D % 8 == 0, "d must be a multiple of 8");
  static constexpr int VPR = D / 8;                  // 16-byte vectors per 16-bit row
  static constexpr int G = res_ln_lanes(VPR);        // lanes per row
  static constexpr int VPL = VPR / G;                // vectors per lane
  static constexpr int RPW = 32 / G;                 // rows per warp step
  static constexpr int CWARPS = 8;                   // consumer warps
  static constexpr int ROW_B = D * 2;                // bytes per 16-bit row
  static constexpr int U_RAW = 16384 / (CWARPS * RPW * ROW_B);
  static constexpr int U = U_RAW < 1 ? 1 : U_RAW;    // warp steps per stage
  static constexpr int R = CWARPS * RPW * U;         // rows per stage
  static constexpr int TILE_B = R * ROW_B;           // bytes per input per stage
  static constexpr int STAGES_RAW = (200 * 1024) / (2 * TILE_B);
  static constexpr int STAGES = STAGES_RAW > 8 ? 8 : STAGES_RAW;
  static constexpr int THREADS = 32 * (CWARPS + 1);
  static constexpr int SMEM = 128 + STAGES * 2 * TILE_B + 2 * STAGES * 8;
  static_assert(STAGES >= 2, "shared memory");
  static_assert(TILE_B % 16 == 0, "bulk copy granularity");
};

// TC, TR: 16-bit concat and residual types; TO: output type; RESID = false: x is not read
// (the output LayerNorm alone).
template <int D, typename TC, typename TR, typename TO, bool RESID = true>
__global__ void __launch_bounds__(ResLnRing<D>::THREADS, 1)
    res_ln_ring_kernel(const TC* __restrict__ cat, const TR* __restrict__ x, const float* __restrict__ gamma,
                       const float* __restrict__ beta, TO* __restrict__ out, int64_t rows, float eps,
                       unsigned* status) {
  using C = ResLnRing<D>;
  static_assert(sizeof(TC) == 2 && sizeof(TR) == 2, "16-bit inputs");
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = smem_raw + ((128u - (smem_u32(smem_raw) & 127u)) & 127u);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + C::STAGES * 2 * C::TILE_B);
  uint64_t* empty = full + C::STAGES;
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int s = 0; s < C::STAGES; ++s) {
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
      for (int64_t t = blockIdx.x; t < ntiles; t += gridDim.x) {
        if (!mbar_wait(&empty[slot], phase ^ 1u, status)) break;
        used |= 1u << slot;
        par = (par & ~(1u << slot)) | (phase << slot);
        const int64_t r0 = t * C::R;
        const int64_t nr = rows - r0 < C::R ? rows - r0 : C::R;
        const uint32_t bytes = static_cast<uint32_t>(nr) * C::ROW_B;
        uint8_t* dst = smem + slot * 2 * C::TILE_B;
        mbar_arrive_expect_tx(&full[slot], (RESID ? 2u : 1u) * bytes);
        bulk_load(dst, cat + r0 * D, bytes, &full[slot]);
        if constexpr (RESID) bulk_load(dst + C::TILE_B, x + r0 * D, bytes, &full[slot]);
        if (++slot == C::STAGES) {
          slot = 0;
          phase ^= 1u;
        }
      }
      // Consumers that stopped early (a flagged error) leave copies unread: let every
      // issued copy land before the CTA's shared memory is released.
      for (int s = 0; s < C::STAGES; ++s)
        if (used & (1u << s)) mbar_drain(&full[s], (par >> s) & 1u, status);
    }
    return;
  }

  // ------------------------------------------------------------------ consumers
  const int cw = warp - 1;
  const int sub = lane / C::G;  // row within a warp step
  const int v0 = lane % C::G;   // first vector of this lane
  float gg[C::VPL][8], bb[C::VPL][8];
#pragma unroll
  for (int k = 0; k < C::VPL; ++k) {
    const int e = (v0 + k * C::G) * 8;
    const float4 g0 = __ldg(reinterpret_cast<const float4*>(gamma + e));
    const float4 g1 = __ldg(reinterpret_cast<const float4*>(gamma + e) + 1);
    const float4 b0 = __ldg(reinterpret_cast<const float4*>(beta + e));
    const float4 b1 = __ldg(reinterpret_cast<const float4*>(beta + e) + 1);
    gg[k][0] = g0.x; gg[k][1] = g0.y; gg[k][2] = g0.z; gg[k][3] = g0.w;
    gg[k][4] = g1.x; gg[k][5] = g1.y; gg[k][6] = g1.z; gg[k][7] = g1.w;
    bb[k][0] = b0.x; bb[k][1] = b0.y; bb[k][2] = b0.z; bb[k][3] = b0.w;
    bb[k][4] = b1.x; bb[k][5] = b1.y; bb[k][6] = b1.z; bb[k][7] = b1.w;
  }
  int slot = 0;
  uint32_t phase = 0;
  for (int64_t t = blockIdx.x; t < ntiles; t += gridDim.x) {
    if (!mbar_wait(&full[slot], phase, status)) break;
    const int64_t r0 = t * C::R;
    const uint8_t* tc = smem + slot * 2 * C::TILE_B;
    const uint8_t* tx = tc + C::TILE_B;
#pragma unroll
    for (int u = 0; u < C::U; ++u) {
      const int lr = (u * C::CWARPS + cw) * C::RPW + sub;  // row within the stage
      const bool ok = r0 + lr < rows;
      float y[C::VPL][8];
#pragma unroll
      for (int k = 0; k < C::VPL; ++k) {
        const int off = lr * C::ROW_B + (v0 + k * C::G) * 16;
        float c8[8];
        Vec8<TC>::load_shared(tc + off, c8);
        if constexpr (RESID) {
          float x8[8];
          Vec8<TR>::load_shared(tx + off, x8);
#pragma unroll
          for (int j = 0; j < 8; ++j) y[k][j] = ok ? c8[j] + x8[j] : 0.f;
        } else {
#pragma unroll
          for (int j = 0; j < 8; ++j) y[k][j] = ok ? c8[j] : 0.f;
        }
      }
      float s = 0.f;
#pragma unroll
      for (int k = 0; k < C::VPL; ++k)
#pragma unroll
        for (int j = 0; j < 8; ++j) s += y[k][j];
#pragma unroll
      for (int o = C::G / 2; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
      const float mean = s * (1.0f / D);
      float q = 0.f;
#pragma unroll
      for (int k = 0; k < C::VPL; ++k)
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          const float dv = y[k][j] - mean;
          q += dv * dv;
        }
#pragma unroll
      for (int o = C::G / 2; o > 0; o >>= 1) q += __shfl_xor_sync(0xffffffffu, q, o);
      const float rstd = rsqrtf(q * (1.0f / D) + eps);
      // an inf / NaN anywhere in the row (a 16-bit intermediate that overflowed upstream)
      if (ok && v0 == 0 && !(isfinite(mean) && isfinite(q))) flag_error(status, kFlagNonFinite);
      if (ok) {
        TO* orow = out + (r0 + lr) * D;
#pragma unroll
        for (int k = 0; k < C::VPL; ++k) {
          float o8[8];
#pragma unroll
          for (int j = 0; j < 8; ++j) o8[j] = (y[k][j] - mean) * rstd * gg[k][j] + bb[k][j];
          Vec8<TO>::store(orow + (v0 + k * C::G) * 8, o8);
        }
      }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&empty[slot]);  // this warp is done reading the stage
    if (++slot == C::STAGES) {
      slot = 0;
      phase ^= 1u;
    }
  }
}

}  // namespace wk
