// fm_mma.cuh -- the FMB front of a Wukong layer for 16-bit operands (fp16 or bf16):
//
//   A0[b] = LN( flatten_rowmajor( X_b (X_b^T Y) ) ) * gamma + beta
//
// i.e. the optimised FM of the Wukong page (section 2.2, FMB paragraph: first
// compress the features to k with Y, then cross), flattened (feature i major,
// compressed index c minor) and normalised over all n*k values.
//
// One persistent CTA per SM walks the examples. A producer thread streams each
// example's X rows (and the matching Y rows) from global memory into a ring of
// shared-memory slots with TMA tile loads -- X as 32-column blocks with the 64-byte
// swizzle, Y with the swizzle that matches its row width -- so that ldmatrix,
// addressed through the same swizzle, is conflict-free; an mbarrier per slot
// carries the transaction count. Eight consumer warps run two passes over the ring:
//   pass A: Z = X^T Y   (d x k, reduction over the n features) with mma.sync
//           m16n8k16 (16-bit in, fp32 accumulate), partial sums of up to AKS warps
//           per output tile added in a fixed order, Z rounded to the 16-bit type;
//   pass B: F = X Z     (n x k, reduction over d), F kept in registers;
// then the LayerNorm statistics (two passes, fp32) and the 16-bit store of A0. The
// producer prefetches the next example while the current one finishes.
#pragma once

#include "common.cuh"

namespace wk {

constexpr int odd16(int bytes) {  // smallest odd multiple of 16 that is >= bytes
  int u = (bytes + 15) / 16;
  if ((u & 1) == 0) ++u;
  return u * 16;
}

template <int N_, int D_, int KC_, int R_, int AWM_, int AWN_, int AKS_, int BWM_, int BWN_, int STAGES_>
struct FmCfg {
  static constexpr int N = N_, D = D_, KC = KC_, R = R_;
  static constexpr int AWM = AWM_, AWN = AWN_, AKS = AKS_, BWM = BWM_, BWN = BWN_, STAGES = STAGES_;
  static constexpr int XBLK = R * 64;        // one 32-column block of R X rows (64B swizzle)
  static constexpr int XBYTES = (D / 32) * XBLK;
  static constexpr int YROW = KC * 2;         // bytes per Y row in the slot
  static constexpr int YSW = (YROW == 128) ? 128 : (YROW == 64) ? 64 : (YROW == 32) ? 32 : 0;  // Y swizzle span
  static constexpr int SY = odd16(KC * 2);    // bytes per Z row (padded, conflict-free)
  static constexpr int SLOT = XBYTES + R * YROW;
  static constexpr int NCH = (N + R - 1) / R;
  static constexpr int AMT = (D / 16) / AWM;  // pass A m16 tiles per warp (over d)
  static constexpr int ANT = (KC / 8) / AWN;  // pass A n8 tiles per warp (over k)
  static constexpr int BMT = (R / 16) / BWM;  // pass B m16 tiles per warp per chunk (over n)
  static constexpr int BNT = (KC / 8) / BWN;  // pass B n8 tiles per warp (over k)
  static constexpr int KS_D = D / 16;         // pass B k16 steps
  static constexpr int KCP = KC + 4;         // padded fp32 row of the Z partials / LN staging
  static constexpr int ZPART_BYTES = (AKS * D > R ? AKS * D : R) * KCP * 4;
  static constexpr int ZB_BYTES = D * SY;
  static constexpr int SMEM = 1024 + STAGES * SLOT + ZPART_BYTES + ZB_BYTES + 64 + 16 * STAGES + 16;
  static_assert(D % 32 == 0 && KC % 8 == 0 && N % 16 == 0 && R % 16 == 0 && R <= 256, "tile shape");
  static_assert(SLOT % 1024 == 0 && XBLK % 1024 == 0, "slot blocks stay aligned to the swizzle atoms");
  static_assert(YSW != 0 || (YROW / 16) % 2 == 1, "unswizzled Y rows must be an odd number of 16-byte units");
  static_assert(KC % 4 == 0, "the staged LayerNorm epilogue moves 4 values at a time");
  static_assert(AWM * AWN * AKS == 8 && BWM * BWN == 8, "8 consumer warps");
  static_assert((D / 16) % AWM == 0 && (KC / 8) % AWN == 0 && (R / 16) % BWM == 0 && (KC / 8) % BWN == 0,
                "warp split");
  static_assert(SMEM <= 227 * 1024, "shared memory");
};

// 8 consumer warps + 1 producer warp. With 9 warps one SM sub-partition holds
// three of them, so its 16K-register file caps the kernel at 168 registers a thread.
constexpr int FM_THREADS = 288;

// Shared address of X element (row r, column c) of a slot, c a multiple of 8:
// 32-column blocks of R rows x 64 B, 16-byte unit index XOR ((r >> 1) & 3).
template <class C>
__device__ __forceinline__ uint32_t fm_x_addr(uint32_t sx, int r, int c) {
  const int unit = ((c & 31) >> 3) ^ ((r >> 1) & 3);
  return sx + (c >> 5) * C::XBLK + r * 64 + unit * 16;
}

// Shared address of Y element (row r, column c), c a multiple of 8, with the
// swizzle the TMA load applied for this row width.
template <class C>
__device__ __forceinline__ uint32_t fm_y_addr(uint32_t sy, int r, int c) {
  int unit = c >> 3;
  if (C::YSW == 128) unit ^= (r & 7);
  else if (C::YSW == 64) unit ^= ((r >> 1) & 3);
  else if (C::YSW == 32) unit ^= ((r >> 2) & 1);
  return sy + r * C::YROW + unit * 16;
}

// tmX: X viewed as [batch*n rows, d] (box 32 x R, 64B swizzle);
// tmY: Y [n, k] (box k x R, swizzle by row width). T: the 16-bit type of X, Y and A0.
template <class C, typename T>
__global__ void __launch_bounds__(FM_THREADS, 1)
    fm_ln_mma_kernel(const __grid_constant__ CUtensorMap tmX, const __grid_constant__ CUtensorMap tmY,
                     const float* __restrict__ gamma, const float* __restrict__ beta,
                     T* __restrict__ A0, int64_t batch, float eps, unsigned* status) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  uint8_t* ring = smem;
  float* zpart = reinterpret_cast<float*>(ring + C::STAGES * C::SLOT);
  uint8_t* zb = reinterpret_cast<uint8_t*>(zpart) + C::ZPART_BYTES;
  float* red = reinterpret_cast<float*>(zb + C::ZB_BYTES);  // [2][8]
  uint64_t* full = reinterpret_cast<uint64_t*>(red + 16);
  uint64_t* empty = full + C::STAGES;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int s = 0; s < C::STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 8);
    }
    fence_mbar_init();
  }
  __syncthreads();

  if (warp == 8) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      prefetch_tmap(&tmX);
      prefetch_tmap(&tmY);
      int s = 0;
      uint32_t ph = 0;
      bool ok = true;
      for (int64_t b = blockIdx.x; ok && b < batch; b += gridDim.x) {
        for (int pass = 0; ok && pass < 2; ++pass) {
          for (int c = 0; c < C::NCH; ++c) {
            if (!mbar_wait(&empty[s], ph ^ 1u, status)) {
              ok = false;
              break;
            }
            uint8_t* slot = ring + s * C::SLOT;
            mbar_arrive_expect_tx(&full[s], static_cast<uint32_t>(pass == 0 ? C::SLOT : C::XBYTES));
            const int row0 = static_cast<int>(b * C::N + c * C::R);
#pragma unroll
            for (int blk = 0; blk < C::D / 32; ++blk) tma_load_2d(&tmX, &full[s], slot + blk * C::XBLK, blk * 32, row0);
            if (pass == 0) tma_load_2d(&tmY, &full[s], slot + C::XBYTES, 0, c * C::R);
            if (++s == C::STAGES) {
              s = 0;
              ph ^= 1u;
            }
          }
        }
      }
      if (!ok) {  // let every armed slot land before the CTA exits
        for (int i = 0; i < C::STAGES; ++i) mbar_wait(&full[i], ph ^ (i < s ? 0u : 1u), nullptr);
      }
    }
    return;
  }

  // -------------------------------------------------------------- consumers
  const int tid = threadIdx.x;  // 0..255
  const int g = lane >> 2, t4 = lane & 3;
  // pass A warp coordinates
  const int a_ks = warp % C::AKS;
  const int a_wn = (warp / C::AKS) % C::AWN;
  const int a_wm = warp / (C::AKS * C::AWN);
  // pass B warp coordinates
  const int b_wn = warp % C::BWN;
  const int b_wm = warp / C::BWN;
  // ldmatrix lane roles
  const int lrow = lane & 7;           // row within an 8x8 matrix
  const int lmat = lane >> 3;          // which of the 4 matrices this lane addresses

  // After a failed wait (status flagged) a consumer stops waiting but keeps
  // walking the same control flow, so every named barrier is still reached by all
  // 256 consumer threads; the output of that launch is then not valid.
  bool ok = true;
  int s = 0;
  uint32_t ph = 0;
  for (int64_t b = blockIdx.x; b < batch; b += gridDim.x) {
    // ------------------------------------------------ pass A: Z = X^T Y
    float zacc[C::AMT][C::ANT][4];
#pragma unroll
    for (int i = 0; i < C::AMT; ++i)
#pragma unroll
      for (int j = 0; j < C::ANT; ++j)
#pragma unroll
        for (int e = 0; e < 4; ++e) zacc[i][j][e] = 0.f;
    for (int c = 0; c < C::NCH; ++c) {
      if (ok) ok = mbar_wait(&full[s], ph, status);
      const int rows = (C::N - c * C::R) < C::R ? (C::N - c * C::R) : C::R;
      const uint32_t sx = smem_u32(ring + s * C::SLOT);
      const uint32_t sy = sx + C::XBYTES;
      for (int ks = a_ks; ks < rows / 16; ks += C::AKS) {
        uint32_t bf[C::ANT][2];
#pragma unroll
        for (int nt = 0; nt < C::ANT; ++nt) {
          // B = Y (k = feature rows, n = compressed index): rows ks*16 + [0,16), column block
          const int col = (a_wn * C::ANT + nt) * 8;
          const int row = ks * 16 + (lmat & 1) * 8 + lrow;
          ldsm_x2_t(fm_y_addr<C>(sy, row, col), bf[nt][0], bf[nt][1]);
        }
#pragma unroll
        for (int mt = 0; mt < C::AMT; ++mt) {
          // A = X^T (m = embedding dim t, k = feature rows): matrices (t0, i0), (t0+8, i0), (t0, i0+8), (t0+8, i0+8)
          const int t0 = (a_wm * C::AMT + mt) * 16 + (lmat & 1) * 8;
          const int row = ks * 16 + (lmat >> 1) * 8 + lrow;
          uint32_t a0, a1, a2, a3;
          ldsm_x4_t(fm_x_addr<C>(sx, row, t0), a0, a1, a2, a3);
#pragma unroll
          for (int nt = 0; nt < C::ANT; ++nt) mma_16816<T>(zacc[mt][nt], a0, a1, a2, a3, bf[nt][0], bf[nt][1]);
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[s]);
      if (++s == C::STAGES) {
        s = 0;
        ph ^= 1u;
      }
    }
    // partial Z tiles -> zpart[a_ks][t][c] (fp32, rows padded to KCP: conflict-free float2 stores)
    named_bar(1, 256);  // the previous example's LayerNorm staging in zpart is consumed
#pragma unroll
    for (int mt = 0; mt < C::AMT; ++mt)
#pragma unroll
      for (int nt = 0; nt < C::ANT; ++nt) {
        const int t = (a_wm * C::AMT + mt) * 16 + g;
        const int cc = (a_wn * C::ANT + nt) * 8 + 2 * t4;
        float* zp = zpart + a_ks * C::D * C::KCP;
        *reinterpret_cast<float2*>(zp + t * C::KCP + cc) = make_float2(zacc[mt][nt][0], zacc[mt][nt][1]);
        *reinterpret_cast<float2*>(zp + (t + 8) * C::KCP + cc) = make_float2(zacc[mt][nt][2], zacc[mt][nt][3]);
      }
    named_bar(1, 256);
    for (int i = tid; i < C::D * C::KC; i += 256) {
      const int t = i / C::KC, cc = i - t * C::KC;
      float z = 0.f;
#pragma unroll
      for (int k = 0; k < C::AKS; ++k) z += zpart[(k * C::D + t) * C::KCP + cc];
      *reinterpret_cast<T*>(zb + t * C::SY + cc * 2) = Half16<T>::from(z);
    }
    named_bar(1, 256);
    // Z as the B operand of pass B (k = embedding dim t, n = compressed index c)
    uint32_t zf[C::BNT][C::KS_D][2];
#pragma unroll
    for (int nt = 0; nt < C::BNT; ++nt)
#pragma unroll
      for (int ks = 0; ks < C::KS_D; ++ks) {
        const int col = (b_wn * C::BNT + nt) * 8;
        const int row = ks * 16 + (lmat & 1) * 8 + lrow;
        ldsm_x2_t(smem_u32(zb) + row * C::SY + col * 2, zf[nt][ks][0], zf[nt][ks][1]);
      }

    // ------------------------------------------------ pass B: F = X Z
    float facc[C::NCH][C::BMT][C::BNT][4];
#pragma unroll
    for (int c = 0; c < C::NCH; ++c)
#pragma unroll
      for (int i = 0; i < C::BMT; ++i)
#pragma unroll
        for (int j = 0; j < C::BNT; ++j)
#pragma unroll
          for (int e = 0; e < 4; ++e) facc[c][i][j][e] = 0.f;
#pragma unroll
    for (int c = 0; c < C::NCH; ++c) {
      if (ok) ok = mbar_wait(&full[s], ph, status);
      const int rows = (C::N - c * C::R) < C::R ? (C::N - c * C::R) : C::R;
      const uint32_t sx = smem_u32(ring + s * C::SLOT);
#pragma unroll
      for (int mt = 0; mt < C::BMT; ++mt) {
        const int m0 = (b_wm * C::BMT + mt) * 16;
        if (m0 < rows) {
#pragma unroll
          for (int ks = 0; ks < C::KS_D; ++ks) {
            // A = X rows (m = features, k = embedding dim): matrices (m0, k0), (m0+8, k0), (m0, k0+8), (m0+8, k0+8)
            const int row = m0 + (lmat & 1) * 8 + lrow;
            const int col = ks * 16 + (lmat >> 1) * 8;
            uint32_t a0, a1, a2, a3;
            ldsm_x4(fm_x_addr<C>(sx, row, col), a0, a1, a2, a3);
#pragma unroll
            for (int nt = 0; nt < C::BNT; ++nt)
              mma_16816<T>(facc[c][mt][nt], a0, a1, a2, a3, zf[nt][ks][0], zf[nt][ks][1]);
          }
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[s]);
      if (++s == C::STAGES) {
        s = 0;
        ph ^= 1u;
      }
    }

    // ------------------------------------------------ LayerNorm over n*k
    float part = 0.f;
#pragma unroll
    for (int c = 0; c < C::NCH; ++c)
#pragma unroll
      for (int mt = 0; mt < C::BMT; ++mt)
#pragma unroll
        for (int nt = 0; nt < C::BNT; ++nt)
#pragma unroll
          for (int e = 0; e < 4; ++e) part += facc[c][mt][nt][e];  // rows past n hold 0
    part = warp_sum(part);
    if (lane == 0) red[warp] = part;
    named_bar(1, 256);
    float tot = 0.f;
#pragma unroll
    for (int w = 0; w < 8; ++w) tot += red[w];
    const float mean = tot * (1.0f / (C::N * C::KC));
    float q = 0.f;
#pragma unroll
    for (int c = 0; c < C::NCH; ++c)
#pragma unroll
      for (int mt = 0; mt < C::BMT; ++mt)
#pragma unroll
        for (int nt = 0; nt < C::BNT; ++nt)
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const int row = c * C::R + (b_wm * C::BMT + mt) * 16 + g + (e >> 1) * 8;
            const float dv = row < C::N ? facc[c][mt][nt][e] - mean : 0.f;
            q += dv * dv;
          }
    q = warp_sum(q);
    if (lane == 0) red[8 + warp] = q;
    named_bar(1, 256);
    float qt = 0.f;
#pragma unroll
    for (int w = 0; w < 8; ++w) qt += red[8 + w];
    const float rstd = rsqrtf(qt * (1.0f / (C::N * C::KC)) + eps);
    // Normalised values go out one chunk of R rows at a time through zpart (fp32,
    // padded rows), so that gamma / beta are read and A0 is written with
    // coalesced 16-byte accesses.
    T* ab = A0 + b * (C::N * C::KC);
#pragma unroll
    for (int c = 0; c < C::NCH; ++c) {
      named_bar(1, 256);  // zpart free (Z reduction done / previous chunk written out)
#pragma unroll
      for (int mt = 0; mt < C::BMT; ++mt)
#pragma unroll
        for (int nt = 0; nt < C::BNT; ++nt)
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            const int r = (b_wm * C::BMT + mt) * 16 + g + h * 8;  // row within the chunk
            const int col = (b_wn * C::BNT + nt) * 8 + 2 * t4;
            *reinterpret_cast<float2*>(zpart + r * C::KCP + col) =
                make_float2((facc[c][mt][nt][2 * h] - mean) * rstd, (facc[c][mt][nt][2 * h + 1] - mean) * rstd);
          }
      named_bar(1, 256);
      const int rows = (C::N - c * C::R) < C::R ? (C::N - c * C::R) : C::R;
      const int base = c * C::R * C::KC;  // flat index of the chunk's first value
      for (int q4 = tid; q4 < rows * C::KC / 4; q4 += 256) {
        const int r = (q4 * 4) / C::KC, col = (q4 * 4) - r * C::KC;
        const float4 v = *reinterpret_cast<const float4*>(zpart + r * C::KCP + col);
        // gamma == nullptr: the affine step lives in the next Linear (normalised values only)
        const float4 gm = gamma ? __ldg(reinterpret_cast<const float4*>(gamma + base) + q4) : make_float4(1.f, 1.f, 1.f, 1.f);
        const float4 bt = gamma ? __ldg(reinterpret_cast<const float4*>(beta + base) + q4) : make_float4(0.f, 0.f, 0.f, 0.f);
        uint2 o;
        o.x = Half16<T>::pack2(v.x * gm.x + bt.x, v.y * gm.y + bt.y);
        o.y = Half16<T>::pack2(v.z * gm.z + bt.z, v.w * gm.w + bt.w);
        *(reinterpret_cast<uint2*>(ab + base) + q4) = o;
      }
    }
  }
}

// The instantiated shapes: (n, d, k) of the 16-bit workloads.
using FmC2 = FmCfg<64, 128, 16, 64, 4, 2, 1, 4, 2, 4>;
using FmC3 = FmCfg<256, 160, 32, 64, 2, 4, 1, 2, 4, 4>;
using FmC4 = FmCfg<512, 160, 64, 64, 2, 4, 1, 2, 4, 4>;
using FmC5 = FmCfg<720, 32, 24, 128, 2, 1, 4, 8, 1, 4>;

}  // namespace wk
