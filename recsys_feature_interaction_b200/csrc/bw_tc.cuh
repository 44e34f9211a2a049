// Strided batched contractions of the backward pass on the tensor cores (tcgen05, kind::tf32).
//
//   C[z][m][n] (+)= sum over terms t of  sum_{k1 < K1_t} sum_{k2 < K2_t} A_t(z, m, k1, k2) B_t(z, n, k1, k2)
//
// with A_t(z, m, k1, k2) = A_t[z sAz + m sAm + k1 sAk1 + k2 sAk2] (B_t likewise), fp32 operands
// whose values are tf32 already (the tensor core reads the top 19 bits of each value: the
// backward rounds its fp32 intermediates to tf32 where it writes them, and 16-bit values
// are exact in tf32). The backward of a Wukong layer is made of such products (the chain
// rule applied to the FM X (X^T Y) and the LCB W_L X of the Wukong page, section 2.2): per
// example X^T Y, X Z, X^T dF, and dX = W_L^T dG + dF Z^T + Y dZ^T as one three-term launch;
// over the batch (k1 = example) sum_b dG_b X_b^T and sum_b X_b dZ_b.
//
// Every operand is a 4-D TMA tensor (its contiguous index first, then the others of row,
// k2, k1, z) and is copied with no transposes into the layout the tensor core reads:
// K-major (128-byte swizzle, one 32 k x R row box) where k2 is contiguous, MN-major (the
// 128-byte swizzle with 32-byte atoms that tf32 takes there, R / 32 boxes of 32 rows x 32 k)
// where the row index is. Out-of-range rows and k read as zero.
//
// Persistent CTAs of 192 threads walk the 128 x BN tiles of C (m fastest, then n, then the
// split of the k1 range, then z, so that CTAs working at the same time share operand blocks
// in L2): warp 0 issues the TMA copies of each k block (32 values of k) into a ring of
// stages, warp 1 the four K = 8 MMAs per block into one of two TMEM accumulators, and warps
// 2..5 move a finished accumulator into C (store, add with one writer per element, or an
// atomic add when the k1 range is split over CTAs) while the next tile accumulates.
#pragma once

#include "common.cuh"

namespace wk {

enum : int { TC_STORE = 0, TC_ACCUM = 1, TC_ATOMIC = 2 };  // how C is written

struct TcTerm {
  const float* A;
  const float* B;
  int K1, K2;
  int64_t sAz, sAm, sAk1, sAk2, sBz, sBn, sBk1, sBk2;
  // set by the host launcher
  int a_mn, b_mn;  // operand copied MN-major (its row index is contiguous)
  int a_z0, b_z0;  // operand shared by every z (coordinate 0)
  int k1q, k1r;    // K1 = k1q S + k1r: split sp covers k1 in [sp k1q + min(sp, k1r), ...)
  int nk2;         // k blocks per k1
};

struct TcContr {
  int M, N, Z, S, mode, nterms, round_c;
  TcTerm t[3];
  float* C;
  int64_t sCz, sCm, sCn;
  // set by the host launcher
  int c_vec, mt, nt, num_tiles;
  unsigned* status;
};

struct TcMaps {
  CUtensorMap m[7];  // A and B of each term; C (fp32, 32-column x 128-row boxes) when read by TMA
};

constexpr int TC_BK = 32;  // k per block: one 128-byte row of fp32
constexpr int TC_THREADS = 192;
constexpr int TC_ABYTES = 128 * TC_BK * 4;

// CIN: C is read (TC_ACCUM) through a TMA prefetch of the tile into shared memory, issued
// when the epilogue starts waiting for the tile's accumulator, instead of by the epilogue's
// own global loads (which stalled it); the ring gives up stages for the buffer.
template <int BN, bool CIN = false>
struct TcCfg {
  static_assert(BN % 32 == 0 && BN >= 64 && BN <= 160, "BN: 64..160, whole 32-row boxes");
  static constexpr int BBYTES = BN * TC_BK * 4;
  static constexpr int STAGE = TC_ABYTES + BBYTES;
  static constexpr int CBYTES = CIN ? 128 * BN * 4 : 0;  // BN / 32 boxes of 32 columns x 128 rows
  static constexpr int STAGES = (196 * 1024 - CBYTES) / STAGE;
  static constexpr int TCOLS = BN <= 64 ? 64 : BN <= 128 ? 128 : 256;  // per accumulator
  static constexpr int BARB = 256;
  static constexpr int SMEM = STAGES * STAGE + CBYTES + BARB + 1024;  // and 1024 bytes of alignment slack
  static constexpr uint32_t IDESC = (1u << 4) | (2u << 7) | (2u << 10) | (static_cast<uint32_t>(BN >> 3) << 17) |
                                    (static_cast<uint32_t>(128 >> 4) << 24);
  static_assert(STAGES >= 3 && 2 * TCOLS <= 512 && SMEM <= 232448 && (2 * STAGES + 6) * 8 + 4 <= BARB, "resources");
};

__device__ __forceinline__ void tma_load_4d(const CUtensorMap* m, uint64_t* bar, uint32_t dst, int32_t c0, int32_t c1,
                                            int32_t c2, int32_t c3) {
  asm volatile(
      "cp.async.bulk.tensor.4d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4, %5, %6}], "
      "[%2];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(m)), "r"(smem_u32(bar)), "r"(c0), "r"(c1), "r"(c2), "r"(c3)
      : "memory");
}

__device__ __forceinline__ void umma_tf32(uint32_t tmem_d, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                          uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::tf32 [%0], %1, %2, %3, p;\n\t}" ::"r"(tmem_d),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// Descriptor of the k-th K = 8 slice of a staged block. K-major: 128-byte swizzle (mode 2),
// 8-row groups 1024 bytes apart, the slice 32 bytes into each row. MN-major: 128-byte swizzle
// with 32-byte atoms (mode 1), 32-row boxes 4096 bytes apart (leading offset), 4-row k
// groups 512 bytes apart (stride offset), the slice 8 k rows further on.
__device__ __forceinline__ uint64_t tc_desc(uint32_t base, int mn, int k) {
  return mn ? smem_desc(base + k * 1024, 4096, 512, 1) : smem_desc(base + k * 32, 16, 1024, 2);
}

struct TcTile {
  int z, sp, m0, ni;
};

__device__ __forceinline__ TcTile tc_tile(const TcContr& p, int tile) {
  TcTile t;
  const int mn = p.mt * p.nt, zs = tile / mn, r = tile - zs * mn;
  t.z = zs / p.S;
  t.sp = zs - t.z * p.S;
  t.ni = r / p.mt;
  t.m0 = (r - t.ni * p.mt) * 128;
  return t;
}

__device__ __forceinline__ void tc_k1_range(const TcTerm& q, int sp, int& b, int& e) {
  b = sp * q.k1q + min(sp, q.k1r);
  e = b + q.k1q + (sp < q.k1r ? 1 : 0);
}

// Copies of one operand block: K-major as one box (k2_0, row0, k1, z); MN-major as R / 32
// boxes (row0 + 32 j, k2_0, k1, z) of 4096 bytes each.
template <int R>
__device__ __forceinline__ void tc_load_operand(const CUtensorMap* m, uint64_t* bar, uint32_t dst, int mn, int row0,
                                                int k2_0, int k1, int z) {
  if (mn) {
#pragma unroll
    for (int j = 0; j < R / 32; ++j) tma_load_4d(m, bar, dst + j * 4096, row0 + 32 * j, k2_0, k1, z);
  } else {
    tma_load_4d(m, bar, dst, k2_0, row0, k1, z);
  }
}

template <int BN, bool CIN>
__device__ __forceinline__ void tc_epilogue(const TcContr& p, const TcTile& tl, uint32_t taddr, int q, int lane,
                                            const uint8_t* cbuf) {
  const int r = 32 * q + lane, n0 = tl.ni * BN;
  const int rows_a = min(128, p.M - tl.m0), rows_b = min(BN, p.N - n0);
  float* crow = p.C + tl.z * p.sCz + (tl.m0 + r) * p.sCm;
#pragma unroll 1
  for (int ch = 0; ch < BN / 32; ++ch) {
    if (32 * ch >= rows_b) break;
    uint32_t v[32];
    tmem_ld32(taddr + 32 * ch, v);
    tmem_ld_wait();
    if (r >= rows_a) continue;
    if (p.round_c) {
#pragma unroll
      for (int j = 0; j < 32; ++j) v[j] = __float_as_uint(tf32_round(__uint_as_float(v[j])));
    }
    const int nb = n0 + 32 * ch;
    if (p.c_vec && (32 * ch + 32 <= rows_b || rows_b % 4 == 0)) {  // whole float4s up to rows_b
      float4* dst = reinterpret_cast<float4*>(crow + nb);
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        if (32 * ch + 4 * j >= rows_b) break;
        float4 x = make_float4(__uint_as_float(v[4 * j]), __uint_as_float(v[4 * j + 1]), __uint_as_float(v[4 * j + 2]),
                               __uint_as_float(v[4 * j + 3]));
        if (p.mode == TC_ATOMIC) {
          atomicAdd(dst + j, x);
        } else {
          if (p.mode == TC_ACCUM) {
            // CIN: the prefetched tile, box ch, row r at r * 128, chunk j at (j ^ (r & 7)) * 16
            const float4 o = CIN ? *reinterpret_cast<const float4*>(cbuf + ch * 16384 + r * 128 + ((j ^ (r & 7)) << 4))
                                 : dst[j];
            x.x += o.x, x.y += o.y, x.z += o.z, x.w += o.w;
          }
          dst[j] = x;
        }
      }
    } else {
#pragma unroll
      for (int j = 0; j < 32; ++j) {
        if (32 * ch + j >= rows_b) break;
        float* dst = crow + (nb + j) * p.sCn;
        const float x = __uint_as_float(v[j]);
        if (p.mode == TC_ATOMIC) {
          atomicAdd(dst, x);
        } else if (p.mode == TC_ACCUM) {
          const int cj = j >> 2;
          *dst = x + (CIN ? reinterpret_cast<const float*>(cbuf + ch * 16384 + r * 128 + ((cj ^ (r & 7)) << 4))[j & 3]
                          : *dst);
        } else {
          *dst = x;
        }
      }
    }
  }
}

template <int BN, bool CIN>
__global__ void __launch_bounds__(TC_THREADS, 1)
    bw_tc_contract_kernel(const __grid_constant__ TcMaps mp, const __grid_constant__ TcContr p) {
  using C = TcCfg<BN, CIN>;
  extern __shared__ uint8_t tc_smem_raw[];
  const uint32_t sbase = (smem_u32(tc_smem_raw) + 1023u) & ~1023u;
  uint8_t* gbase = tc_smem_raw + (sbase - smem_u32(tc_smem_raw));
  uint8_t* cbuf = gbase + C::STAGES * C::STAGE;  // CIN: the prefetched C tile
  uint64_t* bars = reinterpret_cast<uint64_t*>(cbuf + C::CBYTES);
  uint64_t* full = bars;                        // [STAGES] TMA -> MMA
  uint64_t* empty = bars + C::STAGES;           // [STAGES] MMA -> TMA
  uint64_t* tfull = bars + 2 * C::STAGES;       // [2] MMA -> epilogue
  uint64_t* tempty = bars + 2 * C::STAGES + 2;  // [2] epilogue -> MMA
  uint64_t* cfull = bars + 2 * C::STAGES + 4;    // CIN: C tile landed
  uint64_t* cempty = bars + 2 * C::STAGES + 5;   // CIN: the 4 epilogue warps are done with it
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 2 * C::STAGES + 6);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int i = 0; i < 2 * p.nterms; ++i) prefetch_tmap(&mp.m[i]);
    if (CIN) prefetch_tmap(&mp.m[6]);
    mbar_init(cfull, 1);
    mbar_init(cempty, 4);
    for (int s = 0; s < C::STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&tfull[a], 1);
      mbar_init(&tempty[a], 4);
    }
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, 2 * C::TCOLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      int s = 0;
      uint32_t ph = 0;
      bool ok = true;
      for (int tile = blockIdx.x; ok && tile < p.num_tiles; tile += gridDim.x) {
        const TcTile tl = tc_tile(p, tile);
        for (int t = 0; ok && t < p.nterms; ++t) {
          const TcTerm& q = p.t[t];
          int k1b, k1e;
          tc_k1_range(q, tl.sp, k1b, k1e);
          const int za = q.a_z0 ? 0 : tl.z, zb = q.b_z0 ? 0 : tl.z;
          for (int k1 = k1b; ok && k1 < k1e; ++k1) {
            for (int kb = 0; kb < q.nk2; ++kb) {
              if (!mbar_wait(&empty[s], ph ^ 1u, p.status)) {
                ok = false;
                break;
              }
              mbar_arrive_expect_tx(&full[s], C::STAGE);
              const uint32_t sa = sbase + s * C::STAGE;
              tc_load_operand<128>(&mp.m[2 * t], &full[s], sa, q.a_mn, tl.m0, kb * TC_BK, k1, za);
              tc_load_operand<BN>(&mp.m[2 * t + 1], &full[s], sa + TC_ABYTES, q.b_mn, tl.ni * BN, kb * TC_BK, k1, zb);
              if (++s == C::STAGES) {
                s = 0;
                ph ^= 1u;
              }
            }
          }
        }
      }
      // after a failed wait: every stage this thread armed lands before the CTA exits
      // (slots below s were armed in the current round, the others in the previous one)
      if (!ok) {
        for (int i = 0; i < C::STAGES; ++i) mbar_wait(&full[i], ph ^ (i < s ? 0u : 1u), nullptr);
      }
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------- MMA issuer
    if (lane == 0) {
      int s = 0, acc = 0;
      uint32_t ph = 0, acc_ph = 0;
      bool ok = true, issued = false;
      for (int tile = blockIdx.x; ok && tile < p.num_tiles; tile += gridDim.x) {
        const TcTile tl = tc_tile(p, tile);
        if (!mbar_wait(&tempty[acc], acc_ph ^ 1u, p.status)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(acc * C::TCOLS);
        bool first = true;
        for (int t = 0; ok && t < p.nterms; ++t) {
          const TcTerm& q = p.t[t];
          const uint32_t idesc =
              C::IDESC | (static_cast<uint32_t>(q.a_mn) << 15) | (static_cast<uint32_t>(q.b_mn) << 16);
          int k1b, k1e;
          tc_k1_range(q, tl.sp, k1b, k1e);
          const int nb = (k1e - k1b) * q.nk2;
          for (int b = 0; b < nb; ++b) {
            if (!mbar_wait(&full[s], ph, p.status)) {
              ok = false;
              break;
            }
            tc_fence_after();
            const uint32_t sa = sbase + s * C::STAGE;
#pragma unroll
            for (int k = 0; k < TC_BK / 8; ++k) {
              umma_tf32(d_tmem, tc_desc(sa, q.a_mn, k), tc_desc(sa + TC_ABYTES, q.b_mn, k), idesc,
                        (first && k == 0) ? 0u : 1u);
            }
            first = false;
            umma_commit(&empty[s]);
            issued = true;
            if (++s == C::STAGES) {
              s = 0;
              ph ^= 1u;
            }
          }
        }
        if (!ok) break;
        umma_commit(&tfull[acc]);
        if (++acc == 2) {
          acc = 0;
          acc_ph ^= 1u;
        }
      }
      if (!ok && issued) {  // no MMA may still write TMEM when it is freed
        umma_commit(&tfull[acc]);
        mbar_wait(&tfull[acc], acc_ph, nullptr);
      }
    }
  } else {
    // ------------------------------------------------------------ epilogue
    const int q = warp & 3;  // the TMEM lane quarter this warp may access
    const bool c_issuer = CIN && warp == 2 && lane == 0;
    int acc = 0, nt = 0;
    uint32_t acc_ph = 0;
    bool c_owed = false;  // a C prefetch this thread issued has not been waited for
    for (int tile = blockIdx.x; tile < p.num_tiles; tile += gridDim.x, ++nt) {
      const TcTile tl = tc_tile(p, tile);
      // the lanes of a warp leave together (the TMEM loads below are warp-collective)
      bool ok = true;
      if (c_issuer) {  // the tile's C, once every epilogue warp is done with the previous one
        ok = nt == 0 || mbar_wait(cempty, static_cast<uint32_t>((nt - 1) & 1), p.status);
        if (ok) {
          mbar_arrive_expect_tx(cfull, C::CBYTES);
          for (int ch = 0; ch < BN / 32; ++ch)
            tma_load_3d(&mp.m[6], cfull, cbuf + ch * 16384, tl.ni * BN + 32 * ch, tl.m0, tl.z);
          c_owed = true;
        }
      }
      ok = ok && mbar_wait(&tfull[acc], acc_ph, p.status);
      if (CIN && ok) {
        ok = mbar_wait(cfull, static_cast<uint32_t>(nt & 1), p.status);
        if (ok) c_owed = false;
      }
      if (!__all_sync(0xffffffffu, ok)) break;
      tc_fence_after();
      tc_epilogue<BN, CIN>(p, tl,
                           tmem_base + (static_cast<uint32_t>(32 * q) << 16) + static_cast<uint32_t>(acc * C::TCOLS),
                           q, lane, cbuf);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(&tempty[acc]);
        if (CIN) mbar_arrive(cempty);
      }
      if (++acc == 2) {
        acc = 0;
        acc_ph ^= 1u;
      }
    }
    if (c_owed) mbar_drain(cfull, static_cast<uint32_t>(nt & 1), p.status);  // lands before exit
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) tmem_dealloc(tmem_base, 2 * C::TCOLS);
}

}  // namespace wk
