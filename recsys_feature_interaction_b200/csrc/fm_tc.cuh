// fm_tc.cuh -- the FMB front of a Wukong layer on the 5th-generation tensor cores:
//
//   A0[b] = LN( flatten_rowmajor( X_b (X_b^T Y) ) ) * gamma + beta
//
// (the optimised FM of the Wukong page, section 2.2, FMB paragraph: compress the
// features to k with Y first, then cross; flatten feature-major; LayerNorm over
// all n*k values). Per example, two tcgen05 products with fp32 accumulators in
// TMEM:
//   pass A  Z = X^T Y   M = d (128-row tiles), N = k, K = n: X is read as an
//                       MN-major operand, Y as an MN-major operand;
//   pass B  F = X Z     M = n (one 128-row tile per chunk), N = k, K = d: X is read
//                       as a K-major operand (the same shared-memory tiles as pass A),
//                       Z as an MN-major operand written to shared memory (16-bit)
//                       by the epilogue warps from TMEM.
// One persistent CTA per SM walks the examples (192 threads): warp 0 streams 128-row
// chunks of X (and of Y in pass A) with TMA into a ring, warp 1 allocates TMEM and
// one thread issues the MMAs, warps 2..5 turn Z into the pass-B operand and compute
// the LayerNorm from TMEM (three passes: mean, variance, output) and store A0.
// Pass A of example b+1 overlaps the LayerNorm of example b (Z and F have their
// own TMEM columns). Every mbarrier wait is bounded.
//
// k is padded to KP = 32 or 64 columns (the MMA N) with zero columns of Y, which
// the TMA fills out of bounds; F columns past k are never read. Rows of a chunk past
// n (the last chunk, or the next example's rows) only reach accumulator rows that are
// never read, and the Z tile rows past d read padding shared memory.
#pragma once

#include "common.cuh"

namespace wk {

template <int N_, int D_, int K_>
struct FmTcCfg {
  static constexpr int N = N_, D = D_, K = K_;
  static constexpr int R = 128;                            // rows per chunk = MMA M
  static constexpr int XBOXW = D >= 64 ? 64 : 32;          // columns per X box (128B or 64B swizzle)
  static constexpr int XSW = XBOXW * 2;                    // swizzle span in bytes
  static constexpr int XBOXES = (D + XBOXW - 1) / XBOXW;
  static constexpr int XBOXB = R * XBOXW * 2;              // bytes per X box
  static constexpr int KP = K <= 32 ? 32 : 64;             // MMA N (k padded)
  static constexpr int YRB = KP * 2;                       // bytes per Y / Z row
  static constexpr int YB = R * YRB;
  static constexpr int SLOT = XBOXES * XBOXB + YB;
  static constexpr int NCH = (N + R - 1) / R;              // chunks = F tiles
  static constexpr int MTZ = (D + R - 1) / R;              // Z tiles
  static constexpr int ZCOL = MTZ * KP;                    // first TMEM column of F
  static constexpr int TMEM_COLS = 512;
  static constexpr int ZB = ((D + 15) / 16) * 16 * YRB;    // Z operand in shared memory
  // Z tiles read (R / XBOXW) boxes each from a slot's first box; what lies past the
  // slot's X and Y tiles must still be shared memory this CTA owns.
  static constexpr int OVER = (MTZ * (R / XBOXW) - XBOXES) * XBOXB - YB;
  static constexpr int PAD = OVER > 0 ? ((OVER + 1023) / 1024) * 1024 : 0;
  static constexpr int BUDGET = 220 * 1024;
  static constexpr int STAGES_RAW = (BUDGET - ZB - PAD - 1024 - 512) / SLOT;
  static constexpr int STAGES = STAGES_RAW > 8 ? 8 : STAGES_RAW;
  static constexpr int SMEM_RING = 1024 + STAGES * SLOT + PAD + ZB + 512;
  // Example-resident mode, when two examples' X fit: a slot holds all NCH chunks of one
  // example and Y has its own region, loaded once per CTA. Pass A and pass B read the
  // same slot, so an example's X crosses HBM -> SM once, and the next examples' loads
  // never wait for this example's pass B to release ring slots.
  static constexpr int EXB = NCH * XBOXES * XBOXB;              // X bytes per example slot
  static constexpr int YREG = NCH * YB;                         // resident Y
  static constexpr int OVER_R = (MTZ * (R / XBOXW) - XBOXES) * XBOXB;
  static constexpr int PAD_R = OVER_R > 0 ? ((OVER_R + 1023) / 1024) * 1024 : 0;
  static constexpr int ES_RAW = (BUDGET - YREG - ZB - PAD_R - 1024 - 512) / EXB;
  static constexpr bool RES = ES_RAW >= 2;
  static constexpr int ES = ES_RAW > 4 ? 4 : (ES_RAW < 1 ? 1 : ES_RAW);
  static constexpr int SMEM_RES = 1024 + YREG + ES * EXB + PAD_R + ZB + 512;
  static constexpr int SMEM = RES ? SMEM_RES : SMEM_RING;
  // LayerNorm from registers when a thread's share of F (one row per chunk, k values
  // each) fits: the 2-, 4- and wide 2-layer shapes; the 8-layer shape (4 x 64) reads TMEM
  // in three passes instead.
  static constexpr bool REGLN = NCH * K <= 160 && (K == 16 || K == 24 || K == 32);
  static_assert(ZCOL + NCH * KP <= TMEM_COLS, "TMEM columns");
  static_assert(STAGES >= 2, "shared memory");
  static_assert(D % 32 == 0 && N % 16 == 0 && K % 4 == 0 && K <= 64, "shape");
  static_assert(SLOT % 1024 == 0 && XBOXB % 1024 == 0 && ZB % 1024 == 0, "swizzle atoms stay aligned");
};

constexpr int FMTC_THREADS = 192;

// 16- and 8-column TMEM loads (32 lanes x 32 bits): the register-resident LayerNorm
// reads exactly k columns per chunk.
__device__ __forceinline__ void fmtc_tmem_ld16(uint32_t taddr, uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
      "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
      : "r"(taddr)
      : "memory");
}

__device__ __forceinline__ void fmtc_tmem_ld8(uint32_t taddr, uint32_t (&r)[8]) {
  asm volatile("tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0, %1, %2, %3, %4, %5, %6, %7}, [%8];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7])
               : "r"(taddr)
               : "memory");
}

// Shared address of Z operand element row t, 16-byte unit j (MN-major, KP columns).
template <class C>
__device__ __forceinline__ uint32_t fmtc_zb_addr(uint32_t zb, int t, int j) {
  const int pj = (C::YRB == 128) ? (j ^ (t & 7)) : (j ^ ((t >> 1) & 3));
  return zb + t * C::YRB + pj * 16;
}

template <class C, typename T>
__global__ void __launch_bounds__(FMTC_THREADS, 1)
    fm_ln_tc_kernel(const __grid_constant__ CUtensorMap tmX, const __grid_constant__ CUtensorMap tmY,
                    const float* __restrict__ gamma, const float* __restrict__ beta, T* __restrict__ A0,
                    int64_t batch, float eps, unsigned* status) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  // ring mode: [STAGES slots of (X chunk, Y chunk)][PAD][Z][red, barriers]
  // resident mode: [Y region][ES example slots][PAD_R][Z][red, barriers]
  constexpr int NSLOT = C::RES ? C::ES : C::STAGES;
  uint8_t* yreg = smem;                                      // resident mode only
  uint8_t* ring = C::RES ? smem + C::YREG : smem;
  uint8_t* zb = C::RES ? ring + C::ES * C::EXB + C::PAD_R : ring + C::STAGES * C::SLOT + C::PAD;
  float* red = reinterpret_cast<float*>(zb + C::ZB);       // [2][4] partial sums
  uint64_t* bars = reinterpret_cast<uint64_t*>(red + 8);
  uint64_t* full = bars;                                    // [NSLOT]
  uint64_t* empty = bars + NSLOT;                           // [NSLOT]
  uint64_t* zfull = bars + 2 * NSLOT;                       // MMA -> epilogue: Z ready in TMEM
  uint64_t* zready = zfull + 1;                             // epilogue -> MMA: Z operand in smem
  uint64_t* ffull = zfull + 2;                              // MMA -> epilogue: F ready in TMEM
  uint64_t* fempty = zfull + 3;                             // epilogue -> MMA: F read
  uint64_t* yfull = zfull + 4;                              // resident Y has landed
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(zfull + 5);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    prefetch_tmap(&tmX);
    prefetch_tmap(&tmY);
    for (int s = 0; s < NSLOT; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    mbar_init(yfull, 1);
    mbar_init(zfull, 1);
    mbar_init(zready, 4);
    mbar_init(ffull, 1);
    mbar_init(fempty, 4);
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, C::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0 && C::RES) {
      // Y once, then one whole example per slot (both passes read it)
      mbar_arrive_expect_tx(yfull, static_cast<uint32_t>(C::YREG));
      for (int c = 0; c < C::NCH; ++c) tma_load_2d(&tmY, yfull, yreg + c * C::YB, 0, c * C::R);
      int s = 0;
      uint32_t ph = 0;
      bool ok = true;
      for (int64_t b = blockIdx.x; b < batch; b += gridDim.x) {
        if (!mbar_wait(&empty[s], ph ^ 1u, status)) {
          ok = false;
          break;
        }
        uint8_t* slot = ring + s * C::EXB;
        mbar_arrive_expect_tx(&full[s], static_cast<uint32_t>(C::EXB));
        for (int c = 0; c < C::NCH; ++c) {
          const int row0 = static_cast<int>(b * C::N + c * C::R);
#pragma unroll
          for (int bx = 0; bx < C::XBOXES; ++bx)
            tma_load_2d(&tmX, &full[s], slot + (c * C::XBOXES + bx) * C::XBOXB, bx * C::XBOXW, row0);
        }
        if (++s == C::ES) {
          s = 0;
          ph ^= 1u;
        }
      }
      mbar_drain(yfull, 0u, status);
      if (!ok) {
        for (int i = 0; i < C::ES; ++i) mbar_wait(&full[i], ph ^ (i < s ? 0u : 1u), nullptr);
      }
    } else if (lane == 0) {
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
            mbar_arrive_expect_tx(&full[s], static_cast<uint32_t>(C::XBOXES * C::XBOXB + (pass == 0 ? C::YB : 0)));
            const int row0 = static_cast<int>(b * C::N + c * C::R);
#pragma unroll
            for (int bx = 0; bx < C::XBOXES; ++bx)
              tma_load_2d(&tmX, &full[s], slot + bx * C::XBOXB, bx * C::XBOXW, row0);
            if (pass == 0) tma_load_2d(&tmY, &full[s], slot + C::XBOXES * C::XBOXB, 0, c * C::R);
            if (++s == C::STAGES) {
              s = 0;
              ph ^= 1u;
            }
          }
        }
      }
      if (!ok) {
        for (int i = 0; i < C::STAGES; ++i) mbar_wait(&full[i], ph ^ (i < s ? 0u : 1u), nullptr);
      }
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------- MMA issuer
    if (lane == 0 && C::RES) {
      const bool bf = Half16<T>::kBF16;
      const uint32_t idA = idesc_f16kind_f32(C::R, C::KP, 1, 1, bf);  // Z = X^T Y: both MN-major
      const uint32_t idB = idesc_f16kind_f32(C::R, C::KP, 0, 1, bf);  // F = X Z: X K-major, Z MN-major
      const uint32_t xsw = C::XSW == 128 ? 2u : 4u;
      const uint32_t ysw = C::YRB == 128 ? 2u : 4u;
      int s = 0;
      uint32_t ph = 0;
      uint32_t eph = 0;
      bool ok = mbar_wait(yfull, 0u, status);
      bool issued = false;
      tc_fence_after();
      for (int64_t b = blockIdx.x; ok && b < batch; b += gridDim.x) {
        if (!mbar_wait(&full[s], ph, status)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t slot = smem_u32(ring + s * C::EXB);
        // pass A: Z = X^T Y over the example's chunks
        for (int c = 0; c < C::NCH; ++c) {
          const int rows = (C::N - c * C::R) < C::R ? (C::N - c * C::R) : C::R;
          const uint32_t xs = slot + c * C::XBOXES * C::XBOXB;
          const uint32_t ys = smem_u32(yreg) + c * C::YB;
          for (int ks = 0; ks < rows / 16; ++ks) {
            const uint64_t bdesc = smem_desc(ys + ks * 16 * C::YRB, C::YB, 8 * C::YRB, ysw);
#pragma unroll
            for (int mz = 0; mz < C::MTZ; ++mz) {
              const uint32_t a0 = xs + mz * (C::R / C::XBOXW) * C::XBOXB + ks * 16 * C::XSW;
              const uint64_t adesc = smem_desc(a0, C::XBOXB, 8 * C::XSW, xsw);
              umma_f16kind(tmem_base + mz * C::KP, adesc, bdesc, idA, (c | ks) != 0 ? 1u : 0u);
            }
          }
        }
        issued = true;
        umma_commit(zfull);
        // pass B: F = X Z from the same slot, once Z is in shared memory and the
        // previous F has been read
        if (!mbar_wait(zready, eph, status) || !mbar_wait(fempty, eph ^ 1u, status)) {
          ok = false;
          break;
        }
        tc_fence_after();
        for (int c = 0; c < C::NCH; ++c) {
          const uint32_t xs = slot + c * C::XBOXES * C::XBOXB;
#pragma unroll
          for (int ks = 0; ks < C::D / 16; ++ks) {
            const int bx = ks / (C::XBOXW / 16), kin = ks % (C::XBOXW / 16);
            const uint64_t adesc = smem_desc(xs + bx * C::XBOXB + kin * 32, 16, 8 * C::XSW, xsw);
            const uint64_t bdesc = smem_desc(smem_u32(zb) + ks * 16 * C::YRB, C::ZB, 8 * C::YRB, ysw);
            umma_f16kind(tmem_base + C::ZCOL + c * C::KP, adesc, bdesc, idB, ks != 0 ? 1u : 0u);
          }
        }
        umma_commit(&empty[s]);  // the slot is free once both passes have read it
        umma_commit(ffull);
        eph ^= 1u;
        if (++s == C::ES) {
          s = 0;
          ph ^= 1u;
        }
      }
      if (!ok && issued) {  // no MMA may still write TMEM when it is freed
        umma_commit(zfull);
        mbar_wait(zfull, eph, nullptr);
      }
    } else if (lane == 0) {
      const bool bf = Half16<T>::kBF16;
      const uint32_t idA = idesc_f16kind_f32(C::R, C::KP, 1, 1, bf);  // Z = X^T Y: both MN-major
      const uint32_t idB = idesc_f16kind_f32(C::R, C::KP, 0, 1, bf);  // F = X Z: X K-major, Z MN-major
      const uint32_t xsw = C::XSW == 128 ? 2u : 4u;
      const uint32_t ysw = C::YRB == 128 ? 2u : 4u;
      int s = 0;
      uint32_t ph = 0;
      uint32_t eph = 0;  // per-example phase of zready / fempty / zfull / ffull
      bool ok = true;
      bool issued = false;
      for (int64_t b = blockIdx.x; ok && b < batch; b += gridDim.x) {
        // pass A: Z = X^T Y (the previous example's Z was consumed before its pass B)
        for (int c = 0; ok && c < C::NCH; ++c) {
          if (!mbar_wait(&full[s], ph, status)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const int rows = (C::N - c * C::R) < C::R ? (C::N - c * C::R) : C::R;
          const uint32_t xs = smem_u32(ring + s * C::SLOT);
          const uint32_t ys = xs + C::XBOXES * C::XBOXB;
          for (int ks = 0; ks < rows / 16; ++ks) {
            const uint64_t bdesc = smem_desc(ys + ks * 16 * C::YRB, C::YB, 8 * C::YRB, ysw);
#pragma unroll
            for (int mz = 0; mz < C::MTZ; ++mz) {
              // M atoms of XBOXW columns are the X boxes (LBO), 8-row K groups are SBO apart
              const uint32_t a0 = xs + mz * (C::R / C::XBOXW) * C::XBOXB + ks * 16 * C::XSW;
              const uint64_t adesc = smem_desc(a0, C::XBOXB, 8 * C::XSW, xsw);
              umma_f16kind(tmem_base + mz * C::KP, adesc, bdesc, idA, (c | ks) != 0 ? 1u : 0u);
            }
          }
          umma_commit(&empty[s]);
          issued = true;
          if (++s == C::STAGES) {
            s = 0;
            ph ^= 1u;
          }
        }
        if (!ok) break;
        umma_commit(zfull);
        // pass B: F = X Z, once Z is in shared memory and the previous F has been read
        if (!mbar_wait(zready, eph, status) || !mbar_wait(fempty, eph ^ 1u, status)) {
          ok = false;
          break;
        }
        tc_fence_after();
        for (int c = 0; ok && c < C::NCH; ++c) {
          if (!mbar_wait(&full[s], ph, status)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t xs = smem_u32(ring + s * C::SLOT);
#pragma unroll
          for (int ks = 0; ks < C::D / 16; ++ks) {
            const int bx = ks / (C::XBOXW / 16), kin = ks % (C::XBOXW / 16);
            const uint64_t adesc = smem_desc(xs + bx * C::XBOXB + kin * 32, 16, 8 * C::XSW, xsw);
            const uint64_t bdesc = smem_desc(smem_u32(zb) + ks * 16 * C::YRB, C::ZB, 8 * C::YRB, ysw);
            umma_f16kind(tmem_base + C::ZCOL + c * C::KP, adesc, bdesc, idB, ks != 0 ? 1u : 0u);
          }
          umma_commit(&empty[s]);
          if (++s == C::STAGES) {
            s = 0;
            ph ^= 1u;
          }
        }
        if (!ok) break;
        umma_commit(ffull);
        eph ^= 1u;
      }
      if (!ok && issued) {  // no MMA may still write TMEM when it is freed
        umma_commit(zfull);
        mbar_wait(zfull, eph, nullptr);
      }
    }
  } else {
    // ------------------------------------------------------------ epilogue
    const int q = warp & 3;           // TMEM lane quarter
    const int ew = warp - 2;          // 0..3 among the epilogue warps
    const uint32_t lane_base = static_cast<uint32_t>(q * 32) << 16;
    const float inv_cnt = 1.0f / static_cast<float>(C::N * C::K);
    uint32_t eph = 0;
    // After a failed wait (status flagged) a warp stops waiting but keeps walking
    // the same control flow, so every named barrier still sees all four warps.
    bool ok = true;
    // Z (TMEM, fp32) -> 16-bit MN-major operand in shared memory, for the example whose
    // zfull / zready phase has parity zpar
    auto z_convert = [&](uint32_t zpar) {
      if (ok) ok = mbar_wait(zfull, zpar, status);
      tc_fence_after();
#pragma unroll
      for (int mz = 0; mz < C::MTZ; ++mz) {
        const int t = mz * C::R + q * 32 + lane;
#pragma unroll
        for (int h = 0; h < C::KP / 32; ++h) {
          uint32_t r[32];
          tmem_ld32(tmem_base + lane_base + static_cast<uint32_t>(mz * C::KP + h * 32), r);
          tmem_ld_wait();
          if (t < C::D) {
#pragma unroll
            for (int j = 0; j < 4; ++j) {
              uint4 u;
              u.x = Half16<T>::pack2(__uint_as_float(r[8 * j + 0]), __uint_as_float(r[8 * j + 1]));
              u.y = Half16<T>::pack2(__uint_as_float(r[8 * j + 2]), __uint_as_float(r[8 * j + 3]));
              u.z = Half16<T>::pack2(__uint_as_float(r[8 * j + 4]), __uint_as_float(r[8 * j + 5]));
              u.w = Half16<T>::pack2(__uint_as_float(r[8 * j + 6]), __uint_as_float(r[8 * j + 7]));
              asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(fmtc_zb_addr<C>(smem_u32(zb), t, h * 4 + j)),
                           "r"(u.x), "r"(u.y), "r"(u.z), "r"(u.w)
                           : "memory");
            }
          }
        }
      }
      fence_proxy_async_smem();  // the tensor core reads these stores
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(zready);
    };
    // With the LayerNorm in registers, the next example's Z is converted as soon as this
    // example's F is in registers (pass B has read the Z operand by then), so the next
    // pass B runs while this LayerNorm is computed; else each example's Z first.
    if (C::REGLN && blockIdx.x < batch) z_convert(0u);
    for (int64_t b = blockIdx.x; b < batch; b += gridDim.x) {
      if (!C::REGLN) z_convert(eph);

      if constexpr (C::REGLN) {
        // The LayerNorm from registers: each thread's F values (one row per chunk, k
        // columns) are read from TMEM once, all chunks before one wait; TMEM is handed
        // back to the MMA warp at once, and mean, variance and the output are computed
        // from registers (two passes over them).
        if (ok) ok = mbar_wait(ffull, eph, status);
        tc_fence_after();
        uint32_t fr[C::NCH][C::K];
#pragma unroll
        for (int c = 0; c < C::NCH; ++c) {
          const uint32_t ta = tmem_base + lane_base + static_cast<uint32_t>(C::ZCOL + c * C::KP);
          if constexpr (C::K == 32) {
            tmem_ld32(ta, reinterpret_cast<uint32_t(&)[32]>(fr[c][0]));
          } else if constexpr (C::K == 24) {
            fmtc_tmem_ld16(ta, reinterpret_cast<uint32_t(&)[16]>(fr[c][0]));
            fmtc_tmem_ld8(ta + 16, reinterpret_cast<uint32_t(&)[8]>(fr[c][16]));
          } else {
            fmtc_tmem_ld16(ta, reinterpret_cast<uint32_t(&)[16]>(fr[c][0]));
          }
        }
        tmem_ld_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(fempty);  // F is in registers: the next pass B may overwrite it
        if (b + gridDim.x < batch) z_convert(eph ^ 1u);
        float part = 0.f;
#pragma unroll
        for (int c = 0; c < C::NCH; ++c) {
          const int row = c * C::R + q * 32 + lane;
          if (row < C::N) {
#pragma unroll
            for (int j = 0; j < C::K; ++j) part += __uint_as_float(fr[c][j]);
          }
        }
        part = warp_sum(part);
        if (lane == 0) red[ew] = part;
        named_bar(1, 128);
        const float mean = (red[0] + red[1] + red[2] + red[3]) * inv_cnt;
        float qs = 0.f;
#pragma unroll
        for (int c = 0; c < C::NCH; ++c) {
          const int row = c * C::R + q * 32 + lane;
          if (row < C::N) {
#pragma unroll
            for (int j = 0; j < C::K; ++j) {
              const float dv = __uint_as_float(fr[c][j]) - mean;
              qs = fmaf(dv, dv, qs);
            }
          }
        }
        qs = warp_sum(qs);
        if (lane == 0) red[4 + ew] = qs;
        named_bar(1, 128);
        const float var = (red[4] + red[5] + red[6] + red[7]) * inv_cnt;
        const float rstd = rsqrtf(var + eps);
        if (threadIdx.x == 64 && !(isfinite(mean) && isfinite(var))) flag_error(status, kFlagNonFinite);
        T* ab = A0 + b * (C::N * C::K);
        const bool affine = gamma != nullptr;
#pragma unroll
        for (int c = 0; c < C::NCH; ++c) {
          const int row = c * C::R + q * 32 + lane;
          if (row < C::N) {
            T* o = ab + row * C::K;
#pragma unroll
            for (int j = 0; j < C::K; j += 8) {
              float v[8];
#pragma unroll
              for (int i = 0; i < 8; ++i) v[i] = (__uint_as_float(fr[c][j + i]) - mean) * rstd;
              if (affine) {
                const float* gp = gamma + row * C::K + j;
                const float* bp = beta + row * C::K + j;
#pragma unroll
                for (int i = 0; i < 8; ++i) v[i] = v[i] * __ldg(gp + i) + __ldg(bp + i);
              }
              uint4 u;
              u.x = Half16<T>::pack2(v[0], v[1]);
              u.y = Half16<T>::pack2(v[2], v[3]);
              u.z = Half16<T>::pack2(v[4], v[5]);
              u.w = Half16<T>::pack2(v[6], v[7]);
              *reinterpret_cast<uint4*>(o + j) = u;
            }
          }
        }
        named_bar(1, 128);  // every epilogue warp is past its reads of red[]
      } else {
        // LayerNorm over the n*k values of F (TMEM), three passes
        if (ok) ok = mbar_wait(ffull, eph, status);
        tc_fence_after();
        float part = 0.f;
  #pragma unroll 1
        for (int c = 0; c < C::NCH; ++c) {
          const int row = c * C::R + q * 32 + lane;
  #pragma unroll
          for (int h = 0; h < C::KP / 32; ++h) {
            uint32_t r[32];
            tmem_ld32(tmem_base + lane_base + static_cast<uint32_t>(C::ZCOL + c * C::KP + h * 32), r);
            tmem_ld_wait();
            if (row < C::N) {
  #pragma unroll
              for (int j = 0; j < 32; ++j)
                if (h * 32 + j < C::K) part += __uint_as_float(r[j]);
            }
          }
        }
        part = warp_sum(part);
        if (lane == 0) red[ew] = part;
        named_bar(1, 128);
        const float mean = (red[0] + red[1] + red[2] + red[3]) * inv_cnt;
        float qs = 0.f;
  #pragma unroll 1
        for (int c = 0; c < C::NCH; ++c) {
          const int row = c * C::R + q * 32 + lane;
  #pragma unroll
          for (int h = 0; h < C::KP / 32; ++h) {
            uint32_t r[32];
            tmem_ld32(tmem_base + lane_base + static_cast<uint32_t>(C::ZCOL + c * C::KP + h * 32), r);
            tmem_ld_wait();
            if (row < C::N) {
  #pragma unroll
              for (int j = 0; j < 32; ++j)
                if (h * 32 + j < C::K) {
                  const float dv = __uint_as_float(r[j]) - mean;
                  qs += dv * dv;
                }
            }
          }
        }
        qs = warp_sum(qs);
        if (lane == 0) red[4 + ew] = qs;
        named_bar(1, 128);
        const float var = (red[4] + red[5] + red[6] + red[7]) * inv_cnt;
        const float rstd = rsqrtf(var + eps);
        if (threadIdx.x == 64 && !(isfinite(mean) && isfinite(var))) flag_error(status, kFlagNonFinite);
        T* ab = A0 + b * (C::N * C::K);
        const bool affine = gamma != nullptr;
  #pragma unroll 1
        for (int c = 0; c < C::NCH; ++c) {
          const int row = c * C::R + q * 32 + lane;
  #pragma unroll
          for (int h = 0; h < C::KP / 32; ++h) {
            uint32_t r[32];
            tmem_ld32(tmem_base + lane_base + static_cast<uint32_t>(C::ZCOL + c * C::KP + h * 32), r);
            tmem_ld_wait();
            if (row < C::N) {
              const float* g = affine ? gamma + row * C::K + h * 32 : nullptr;
              const float* bt = affine ? beta + row * C::K + h * 32 : nullptr;
              T* o = ab + row * C::K + h * 32;
  #pragma unroll
              for (int j = 0; j < 32; j += 8) {
                if (h * 32 + j < C::K) {
                  // gamma == nullptr: the affine step lives in the next Linear (normalised values only)
                  const float4 one = make_float4(1.f, 1.f, 1.f, 1.f), zero = make_float4(0.f, 0.f, 0.f, 0.f);
                  const float4 g0 = affine ? __ldg(reinterpret_cast<const float4*>(g + j)) : one;
                  const float4 g1 = affine ? __ldg(reinterpret_cast<const float4*>(g + j + 4)) : one;
                  const float4 b0 = affine ? __ldg(reinterpret_cast<const float4*>(bt + j)) : zero;
                  const float4 b1 = affine ? __ldg(reinterpret_cast<const float4*>(bt + j + 4)) : zero;
                  uint4 u;
                  u.x = Half16<T>::pack2((__uint_as_float(r[j + 0]) - mean) * rstd * g0.x + b0.x,
                                         (__uint_as_float(r[j + 1]) - mean) * rstd * g0.y + b0.y);
                  u.y = Half16<T>::pack2((__uint_as_float(r[j + 2]) - mean) * rstd * g0.z + b0.z,
                                         (__uint_as_float(r[j + 3]) - mean) * rstd * g0.w + b0.w);
                  u.z = Half16<T>::pack2((__uint_as_float(r[j + 4]) - mean) * rstd * g1.x + b1.x,
                                         (__uint_as_float(r[j + 5]) - mean) * rstd * g1.y + b1.y);
                  u.w = Half16<T>::pack2((__uint_as_float(r[j + 6]) - mean) * rstd * g1.z + b1.z,
                                         (__uint_as_float(r[j + 7]) - mean) * rstd * g1.w + b1.w);
                  *reinterpret_cast<uint4*>(o + j) = u;
                }
              }
            }
          }
        }
        tc_fence_before();
        named_bar(1, 128);  // every epilogue warp is past its reads of red[] and F
        if (lane == 0) mbar_arrive(fempty);
      }
      eph ^= 1u;
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, C::TMEM_COLS);
  }
}

using FmTcC2 = FmTcCfg<64, 128, 16>;
using FmTcC3 = FmTcCfg<256, 160, 32>;
using FmTcC4 = FmTcCfg<512, 160, 64>;
using FmTcC5 = FmTcCfg<720, 32, 24>;

}  // namespace wk
