// row_ln_epi.cuh -- the end of a Wukong layer fused into a GEMM epilogue.
//
// The layer output is LN_rows( concat(FMB, LCB) + X ) (Wukong page, section 2.2:
// concatenate, add the residual, LayerNorm). When a GEMM tile holds complete
// embedding rows -- the LCB tile holds W_L rows of whole examples, the last FMB
// Linear is tiled by whole n_F rows -- each epilogue lane owns one row of d
// accumulator values in TMEM and finishes it in place:
//
//   y = acc (+ bias) + x_row;   out_row = (y - mean(y)) * rsqrt(var(y) + eps) * gamma + beta
//
// with mean and biased variance by two passes (fp32), so the concat buffer and
// the separate residual + LayerNorm pass disappear. The output leaves through the
// epilogue's swizzled staging buffers and TMA stores, 32 columns at a time.
#pragma once

#include "common.cuh"
#include "res_ln.cuh"

namespace wk {

// Writes 32 fp32 values of one accumulator row into a 32x32 staging tile row,
// laid out as the TMA store expects: 16-bit rows of 64 B with the 64B swizzle, or
// fp32 rows of 128 B with the 128B swizzle.
template <typename TO>
__device__ __forceinline__ void stage_row(uint8_t* buf, int row, const float (&v)[32]);

template <>
__device__ __forceinline__ void stage_row<__nv_bfloat16>(uint8_t* buf, int row, const float (&v)[32]) {
#pragma unroll
  for (int c = 0; c < 4; ++c) {
    uint4 q;
    q.x = pack_bf16x2(v[8 * c + 0], v[8 * c + 1]);
    q.y = pack_bf16x2(v[8 * c + 2], v[8 * c + 3]);
    q.z = pack_bf16x2(v[8 * c + 4], v[8 * c + 5]);
    q.w = pack_bf16x2(v[8 * c + 6], v[8 * c + 7]);
    const int pc = c ^ ((row >> 1) & 3);
    *reinterpret_cast<uint4*>(buf + row * 64 + pc * 16) = q;
  }
}

template <>
__device__ __forceinline__ void stage_row<__half>(uint8_t* buf, int row, const float (&v)[32]) {
#pragma unroll
  for (int c = 0; c < 4; ++c) {
    uint4 q;
    q.x = Half16<__half>::pack2(v[8 * c + 0], v[8 * c + 1]);
    q.y = Half16<__half>::pack2(v[8 * c + 2], v[8 * c + 3]);
    q.z = Half16<__half>::pack2(v[8 * c + 4], v[8 * c + 5]);
    q.w = Half16<__half>::pack2(v[8 * c + 6], v[8 * c + 7]);
    const int pc = c ^ ((row >> 1) & 3);
    *reinterpret_cast<uint4*>(buf + row * 64 + pc * 16) = q;
  }
}

template <>
__device__ __forceinline__ void stage_row<float>(uint8_t* buf, int row, const float (&v)[32]) {
#pragma unroll
  for (int c = 0; c < 8; ++c) {
    const int pc = c ^ (row & 7);
    *reinterpret_cast<float4*>(buf + row * 128 + pc * 16) =
        make_float4(v[4 * c + 0], v[4 * c + 1], v[4 * c + 2], v[4 * c + 3]);
  }
}


// y for 32 columns [32c, 32c + 32) of this lane's row: accumulator + bias + residual.
template <typename TR>
__device__ __forceinline__ void row_ln_chunk(uint32_t taddr, int c, bool valid, const TR* resid, const float* bias,
                                             float (&y)[32]) {
  uint32_t r[32];
  tmem_ld32(taddr + static_cast<uint32_t>(c * 32), r);  // warp-collective: every lane issues it
  tmem_ld_wait();
#pragma unroll
  for (int j = 0; j < 32; ++j) y[j] = __uint_as_float(r[j]);
  if (valid) {
#pragma unroll
    for (int v = 0; v < 4; ++v) {
      float x8[8];
      Vec8<TR>::load(resid + c * 32 + v * 8, x8);
#pragma unroll
      for (int j = 0; j < 8; ++j) y[v * 8 + j] += x8[j];
    }
    if (bias) {
#pragma unroll
      for (int j = 0; j < 32; j += 4) {
        const float4 b4 = __ldg(reinterpret_cast<const float4*>(bias + c * 32 + j));
        y[j] += b4.x;
        y[j + 1] += b4.y;
        y[j + 2] += b4.z;
        y[j + 3] += b4.w;
      }
    }
  }
}

// One embedding row per lane: TMEM columns [taddr, taddr + d) of this warp's lane
// quarter, residual row `resid` (d values), optional `bias` row (d values), LayerNorm
// affine g / b (d values). `store(c, sb)` is called by lane 0 after the 32 x 32
// staging tile `sb` of chunk c is complete (it issues the TMA store and commits).
template <typename TR, typename TO, class Store>
__device__ __forceinline__ void row_ln_epilogue(uint32_t taddr, int d, bool valid, const TR* resid,
                                                const float* bias, const float* g, const float* b, float eps,
                                                uint8_t* bufs, uint32_t buf_bytes, int& buf, int lane, Store store) {
  const int nch = d / 32;
  float s = 0.f;
  for (int c = 0; c < nch; ++c) {
    float y[32];
    row_ln_chunk<TR>(taddr, c, valid, resid, bias, y);
#pragma unroll
    for (int j = 0; j < 32; ++j) s += y[j];
  }
  const float mean = s / static_cast<float>(d);
  float q = 0.f;
  for (int c = 0; c < nch; ++c) {
    float y[32];
    row_ln_chunk<TR>(taddr, c, valid, resid, bias, y);
#pragma unroll
    for (int j = 0; j < 32; ++j) {
      const float dv = y[j] - mean;
      q += dv * dv;
    }
  }
  const float rstd = rsqrtf(q / static_cast<float>(d) + eps);
  for (int c = 0; c < nch; ++c) {
    float y[32];
    row_ln_chunk<TR>(taddr, c, valid, resid, bias, y);
#pragma unroll
    for (int j = 0; j < 32; j += 4) {
      const float4 g4 = __ldg(reinterpret_cast<const float4*>(g + c * 32 + j));
      const float4 b4 = __ldg(reinterpret_cast<const float4*>(b + c * 32 + j));
      y[j] = (y[j] - mean) * rstd * g4.x + b4.x;
      y[j + 1] = (y[j + 1] - mean) * rstd * g4.y + b4.y;
      y[j + 2] = (y[j + 2] - mean) * rstd * g4.z + b4.z;
      y[j + 3] = (y[j + 3] - mean) * rstd * g4.w + b4.w;
    }
    uint8_t* sb = bufs + buf * buf_bytes;
    if (lane == 0) bulk_wait_read<1>();  // the store that last used this buffer has read it
    __syncwarp();
    stage_row<TO>(sb, lane, y);
    fence_proxy_async_smem();
    __syncwarp();
    if (lane == 0) store(c, sb);
    buf ^= 1;
  }
}

}  // namespace wk
