// front_tc.cuh -- everything of a Wukong layer but the FMB MLP, one example at a time
// per CTA, reading each example's layer input from HBM once (Wukong page, section 2.2:
// the layer is LN(concat(FMB(X), LCB(X)) + X); FMB(X) = MLP(LN(flatten(X (X^T Y))));
// LCB(X) = W_L X):
//
//   X      = LN_rows(y_in) * g_in + b_in    (the previous layer's output LayerNorm;
//            for the first layer X is the caller's input, converted to the operand type)
//   A0     = LN(flatten(X (X^T Y)))         (the FM and the FMB LayerNorm; its affine is
//            either applied here or folded into the first Linear by the caller)
//   y_out[rows n_f..n-1] = W_L X + X[n_f..n-1]     (the LCB rows with their residual)
//   y_out[rows 0..n_f-1] = X[0..n_f-1]              (the residual of the FMB rows; the
//            last MLP Linear adds its output into them with a TMA reduce-add)
//
// so a layer's output y_out = concat(FMB, LCB) + X, before the output LayerNorm, which
// the next layer's front (or the stack's final LayerNorm) applies as it reads y_out.
//
// Per example, in shared memory: the n x d layer input in 128-row chunks, each one contiguous
// range of the input brought in by one bulk copy and rewritten in place by the normalising
// warps as the MMA operand layout (32-column boxes, 64-byte swizzle), read by three tcgen05
// products:
//   pass A  Z = X^T Y       M = d (128-row tiles), N = k (padded to KP), K = n;
//   LCB     D_m = W_L,m X   M = 128 rows of W_L, N = d, K = n (W_L and Y stream through a
//                           small ring of 16 KB stages from L2);
//   pass B  F = X Z         M = n (one tile per chunk), N = KP, K = d (Z written back to
//                           shared memory as a 16-bit operand by the epilogue warps).
// TMEM holds Z at column 0 and, from column LCOL, the LCB accumulators; F follows them where
// TMEM has room (the 2- and 4-layer shapes) or reuses their columns chunk by chunk as the LCB
// rows are read out (the 8-layer shape).
//
// Warps (480 threads): 0 loads input chunks; 1 allocates TMEM and issues the MMAs; 2 streams
// Y and W_L; 3..6 are the epilogue (one TMEM lane quarter each: Z to shared memory, the LCB
// rows plus residual out, the FMB LayerNorm of F into A0); 7..14 normalise each chunk as it
// lands (two threads per row) and store the FMB-row residual. The per-element passes (both
// LayerNorms, the residual add) use the packed fp32x2 instructions.
// Every mbarrier wait is bounded; after a failed wait each role stops, every copy in flight
// lands and TMEM is freed before the CTA exits.
#pragma once

#include "common.cuh"
#include "gemm_tc.cuh"
#include "res_ln.cuh"

namespace wk {

constexpr int FRONT_THREADS = 480;
constexpr int FRONT_EPI_WARP0 = 3;    // warps 3..6: the epilogue (TMEM lane quarter = warp & 3)
constexpr int FRONT_NORM_WARP0 = 7;   // warps 7..14: normalisation
constexpr int FRONT_NORM_THREADS = 256;
constexpr int FRONT_SMEM_LIMIT = 232448;

template <int N_, int D_, int K_, int NF_, bool LCB_DIRECT_>
struct FrontCfg {
  static constexpr int N = N_, D = D_, K = K_, NF = NF_, NL = N_ - NF_;
  static constexpr int R = 128;                              // rows per chunk = MMA M
  static constexpr int NCH = (N + R - 1) / R;
  static constexpr int XBOXES = D / 32;                      // 32-column boxes per chunk
  static constexpr int XBOXB = R * 64;                       // 8 KB per box
  static constexpr int CHB = XBOXES * XBOXB;                 // bytes per chunk
  static constexpr int KP = K <= 32 ? 32 : 64;               // MMA N of the FM (k padded)
  static constexpr int YRB = KP * 2;                         // bytes per Y / Z row
  static constexpr int YB = R * YRB;                         // one Y box (128 rows)
  static constexpr int MTZ = (D + R - 1) / R;                // Z tiles
  static constexpr int MTL = (NL + R - 1) / R;               // LCB tiles
  static constexpr int LCOL = MTZ * KP;                      // first TMEM column of the LCB / F
  static constexpr int LCOLS = MTL * D;
  static constexpr int FCOLS = NCH * KP;
  // F in its own TMEM columns after the LCB's when they fit (pass B then need not wait for
  // the LCB rows to be read out), else F reuses the LCB's columns
  static constexpr bool SEPF = LCOL + LCOLS + FCOLS <= 512;
  static constexpr int FCOL = SEPF ? LCOL + LCOLS : LCOL;
  static constexpr int UCOLS = SEPF ? LCOLS + FCOLS : (LCOLS > FCOLS ? LCOLS : FCOLS);
  static constexpr int TCOLS = LCOL + UCOLS;
  static constexpr int TMEM_COLS = TCOLS <= 32 ? 32 : TCOLS <= 64 ? 64 : TCOLS <= 128 ? 128 : TCOLS <= 256 ? 256 : 512;
  static constexpr int ZB = ((D + 15) / 16) * 16 * YRB;      // Z operand
  static constexpr int WB = R * 64 * 2;                      // one W_L box (128 rows x 64 k)
  static constexpr int STG = WB > YB ? WB : YB;              // ring stage
  static constexpr int EPI = 4 * 2048;                       // a 32 x 32 16-bit staging tile per epilogue warp
  static constexpr int TAIL = 2 * D * 4 + 1024;              // input LN affine, partial sums, barriers
  // examples in flight: two sets of chunk slots (the next example loads while this one
  // computes) where shared memory keeps a 2-stage ring beside them and TMEM holds F apart
  static constexpr int ES = (SEPF && 1024 + 2 * NCH * CHB + ZB + EPI + TAIL + 2 * (WB > YB ? WB : YB) <=
                             FRONT_SMEM_LIMIT) ? 2 : 1;
  static constexpr int FIXED = 1024 + ES * NCH * CHB + ZB + EPI + TAIL;
  static constexpr int NSTG_RAW = (FRONT_SMEM_LIMIT - FIXED) / STG;
  static constexpr int NSTG = NSTG_RAW > 4 ? 4 : NSTG_RAW;
  // pass A's last Z tile reads 4 * MTZ boxes from a chunk's base: past the last chunk that
  // is OVER bytes, which must stay inside this CTA's shared memory (rows of Z past d are
  // never read, so what they read does not matter)
  static constexpr int OVER = (4 * MTZ - XBOXES) * XBOXB;
  static constexpr int AFTER = ZB + NSTG * STG + EPI;
  static constexpr int PAD = OVER > AFTER ? ((OVER - AFTER + 1023) / 1024) * 1024 : 0;
  static constexpr int SMEM = FIXED + NSTG * STG + PAD;
  // LayerNorm of F from registers when a thread's share (one row per chunk, k values) fits
  static constexpr bool REGLN = NCH * K <= 96 && (K == 16 || K == 24 || K == 32);
  // staging tiles (32 x 32, 2 KB) per epilogue warp for the LCB rows: its own tile plus a
  // quarter of the Y / W_L ring, which is idle while the LCB accumulators are read out
  static constexpr int NBUF_RAW = 1 + (NSTG * STG) / (4 * 2048);
  static constexpr int NBUF = NBUF_RAW > 8 ? 8 : NBUF_RAW;
  // A0 leaves through TMA stores of 32 x 32 tiles in the three-pass LayerNorm (k = 64, whole
  // chunks), staged in three 2 KB tiles per epilogue warp: its own and two in the Z region
  static constexpr bool A0_TMA = !REGLN && K == 64 && N % R == 0 && ZB >= 4 * 4096;
  // the LCB rows leave by 16-byte stores of the epilogue warps, each box transposed through
  // the warp's own staging tile (the Y / W_L ring is not borrowed, so it streams the next
  // example's stages while the rows are read out), else by TMA stores staged in the
  // warp's tile and its quarter of the ring; chosen per shape by measurement
  static constexpr bool LCB_DIRECT = LCB_DIRECT_;
  static_assert(D % 32 == 0 && D <= 256 && N % 16 == 0 && K % 4 == 0 && K <= 64, "shape");
  static_assert(NSTG >= 2 && SMEM <= FRONT_SMEM_LIMIT, "shared memory");
  static_assert(TCOLS <= 512, "TMEM columns");
  static_assert(CHB % 1024 == 0 && ZB % 1024 == 0 && STG % 1024 == 0, "swizzle atoms stay aligned");
};

// 16-byte unit u (0..3) of row r in a 64-byte-swizzled box of 64-byte rows.
__device__ __forceinline__ uint32_t sw64_off(int r, int u) {
  return static_cast<uint32_t>(r * 64 + ((u ^ ((r >> 1) & 3)) << 4));
}

// Shared address of Z operand element row t, 16-byte unit j (MN-major, KP columns).
template <class C>
__device__ __forceinline__ uint32_t front_zb_addr(uint32_t zb, int t, int j) {
  const int pj = (C::YRB == 128) ? (j ^ (t & 7)) : (j ^ ((t >> 1) & 3));
  return zb + t * C::YRB + pj * 16;
}

__device__ __forceinline__ void front_tmem_ld16(uint32_t taddr, uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
      "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
      : "r"(taddr)
      : "memory");
}

__device__ __forceinline__ void front_tmem_ld8(uint32_t taddr, uint32_t (&r)[8]) {
  asm volatile("tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0, %1, %2, %3, %4, %5, %6, %7}, [%8];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7])
               : "r"(taddr)
               : "memory");
}

// Two fp32 values in one 64-bit register pair, for the packed fp32 instructions of sm_100
// (add / mul / fma .f32x2: one instruction for two lanes of the per-element LayerNorm work,
// each lane rounded as its scalar instruction would be).
__device__ __forceinline__ uint64_t f2_pack(float lo, float hi) {
  uint64_t r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
  return r;
}
__device__ __forceinline__ void f2_unpack(uint64_t r, float& lo, float& hi) {
  asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(r));
}
__device__ __forceinline__ float f2_sum(uint64_t r) {
  float lo, hi;
  f2_unpack(r, lo, hi);
  return lo + hi;
}
__device__ __forceinline__ uint64_t f2_add(uint64_t a, uint64_t b) {
  uint64_t d;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}
__device__ __forceinline__ uint64_t f2_mul(uint64_t a, uint64_t b) {
  uint64_t d;
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}
__device__ __forceinline__ uint64_t f2_fma(uint64_t a, uint64_t b, uint64_t c) {
  uint64_t d;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
  return d;
}
// The two 16-bit values of type TI in a 32-bit word as an fp32 pair.
template <typename TI>
__device__ __forceinline__ uint64_t f2_from16(uint32_t w) {
  return f2_pack(Half16<TI>::lo(w), Half16<TI>::hi(w));
}
// An fp32 pair rounded to two 16-bit values of type TO in a 32-bit word.
template <typename TO>
__device__ __forceinline__ uint32_t f2_to16(uint64_t r) {
  float lo, hi;
  f2_unpack(r, lo, hi);
  return Half16<TO>::pack2(lo, hi);
}

// Eight 16-bit values of type TI (one 16-byte unit) as floats.
template <typename TI>
__device__ __forceinline__ void front_unpack8(const uint4& a, float (&v)[8]) {
  Vec8<TI>::unpack(a, v);
}

template <typename TO>
__device__ __forceinline__ uint4 front_pack8(const float (&v)[8]) {
  uint4 a;
  a.x = Half16<TO>::pack2(v[0], v[1]);
  a.y = Half16<TO>::pack2(v[2], v[3]);
  a.z = Half16<TO>::pack2(v[4], v[5]);
  a.w = Half16<TO>::pack2(v[6], v[7]);
  return a;
}

// Row `row` of a 32 x 32 16-bit staging tile (64-byte rows, 64-byte swizzle) from 16 words
// of two packed 16-bit values each.
__device__ __forceinline__ void front_stage16(uint8_t* buf, int row, const uint32_t (&o)[16]) {
#pragma unroll
  for (int c = 0; c < 4; ++c) {
    const int pc = c ^ ((row >> 1) & 3);
    *reinterpret_cast<uint4*>(buf + row * 64 + pc * 16) = make_uint4(o[4 * c], o[4 * c + 1], o[4 * c + 2], o[4 * c + 3]);
  }
}

// xin: the layer input [batch, n, d] of type TIN (16-byte aligned). Tensor maps:
//   tmY  Y [n, k] (T): boxes of KP columns (zero past k) x 128 rows, 128B (KP = 64) or 64B swizzle;
//   tmW  W_L [n_l, n] (T): boxes of 64 columns x 128 rows, 128B swizzle;
//   tmR  rows 0..n_f-1 of y_out as a (d, n_f, batch) tensor (T): boxes (32, 128, 1), 64B swizzle;
//   tmL  rows n_f..n-1 of y_out as a (d, n_l, batch) tensor (T): boxes (32, 32, 1), 64B swizzle;
//   tmA  A0 as [batch*n rows, k] (T): boxes (32, 32), 64B swizzle (used only when k = 64 and n is
//        a multiple of 128: the output pass then stages A0 and stores it by TMA).
// in_g / in_b: the input LayerNorm's affine [d] (null: the first layer, no LayerNorm);
// fg / fb: the FMB LayerNorm's affine [n*k] (null: folded into the first Linear).
template <class C, typename TIN, typename T>
__global__ void __launch_bounds__(FRONT_THREADS, 1)
    front_tc_kernel(const TIN* __restrict__ xin, const __grid_constant__ CUtensorMap tmY,
                    const __grid_constant__ CUtensorMap tmW, const __grid_constant__ CUtensorMap tmR,
                    const __grid_constant__ CUtensorMap tmL, const __grid_constant__ CUtensorMap tmA,
                    const float* __restrict__ in_g,
                    const float* __restrict__ in_b, const float* __restrict__ fg, const float* __restrict__ fb,
                    T* __restrict__ A0, T* __restrict__ yout, int64_t batch, float eps, unsigned* status) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  uint8_t* slots = smem;                                     // [ES][NCH] chunks of the layer inputs
  uint8_t* zb = slots + C::ES * C::NCH * C::CHB;             // Z operand
  uint8_t* ring = zb + C::ZB;                                // [NSTG] Y / W_L stages
  uint8_t* epi = ring + C::NSTG * C::STG;                    // [4] staging tiles
  float* sg = reinterpret_cast<float*>(epi + C::EPI + C::PAD);
  float* sb = sg + C::D;
  float* red = sb + C::D;                                    // [8] FMB LayerNorm partial sums
  uint64_t* bars = reinterpret_cast<uint64_t*>(red + 8);
  uint64_t* full = bars;                                     // [ES * NCH] chunk landed
  uint64_t* xready = full + C::ES * C::NCH;                  // [ES * NCH] chunk normalised
  uint64_t* empty = xready + C::ES * C::NCH;                 // [ES * NCH] chunk slot free (6 arrivals)
  uint64_t* wfull = empty + C::ES * C::NCH;                  // [NSTG]
  uint64_t* wempty = wfull + C::NSTG;                        // [NSTG]
  uint64_t* zfull = wempty + C::NSTG;                        // MMA -> epilogue: Z in TMEM
  uint64_t* ffull = zfull + 1;                               // MMA -> epilogue: F in TMEM
  uint64_t* zready = zfull + 2;                              // epilogue -> MMA: Z operand written
  uint64_t* ldone = zfull + 3;                               // epilogue -> MMA, ring: LCB columns read
  uint64_t* fempty = zfull + 4;                              // epilogue -> MMA: F read
  uint64_t* fin = zfull + 5;                                 // MMA: its last operations completed
  uint64_t* lfull = zfull + 6;                               // [MTL] MMA -> epilogue: LCB tile m in TMEM
  uint64_t* fcfree = lfull + C::MTL;                         // [NCH] epilogue -> MMA: the LCB
                                                             // columns F chunk c reuses are read
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(fcfree + C::NCH);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const bool ln_in = in_g != nullptr;
  if (threadIdx.x == 0) {
    prefetch_tmap(&tmY);
    prefetch_tmap(&tmW);
    prefetch_tmap(&tmR);
    prefetch_tmap(&tmL);
    prefetch_tmap(&tmA);
    // a slot is free once pass B has read it (the MMA's commit), its residual stores have
    // read it (the normalising warps) and the LCB rows' residual has been read from it (one
    // arrival per epilogue warp)
    for (int c = 0; c < C::ES * C::NCH; ++c) {
      mbar_init(&full[c], 1);
      mbar_init(&xready[c], 1);
      mbar_init(&empty[c], 6);
    }
    for (int s = 0; s < C::NSTG; ++s) {
      mbar_init(&wfull[s], 1);
      mbar_init(&wempty[s], 1);
    }
    mbar_init(zfull, 1);
    for (int m = 0; m < C::MTL; ++m) mbar_init(&lfull[m], 1);
    for (int c = 0; c < C::NCH; ++c) mbar_init(&fcfree[c], 4);
    mbar_init(ffull, 1);
    mbar_init(zready, 4);
    mbar_init(ldone, 4);
    mbar_init(fempty, 4);
    mbar_init(fin, 1);
    fence_mbar_init();
  }
  if (ln_in && threadIdx.x >= 32 * FRONT_NORM_WARP0) {
    for (int i = threadIdx.x - 32 * FRONT_NORM_WARP0; i < C::D; i += FRONT_NORM_THREADS) {
      sg[i] = __ldg(in_g + i);
      sb[i] = __ldg(in_b + i);
    }
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
    // ---------------------------------------------------------- input chunks
    if (lane == 0) {
      uint32_t issued = 0, lastpar = 0;
      int64_t i = 0;
      bool ok = true;
      for (int64_t b = blockIdx.x; ok && b < batch; b += gridDim.x, ++i) {
        const int es = static_cast<int>(i % C::ES);                // slot set and its phase
        const uint32_t sp = static_cast<uint32_t>((i / C::ES) & 1);
        for (int cc = 0; cc < C::NCH; ++cc) {
          const int c = es * C::NCH + cc;
          if (!mbar_wait(&empty[c], sp ^ 1u, status)) {
            ok = false;
            break;
          }
          // the chunk's rows are one contiguous range of the input: one bulk copy
          const int rows = (C::N - cc * C::R) < C::R ? (C::N - cc * C::R) : C::R;
          const uint32_t bytes = static_cast<uint32_t>(rows * C::D * 2);
          mbar_arrive_expect_tx(&full[c], bytes);
          bulk_load(slots + c * C::CHB, xin + (b * C::N + cc * C::R) * C::D, bytes, &full[c]);
          issued |= 1u << c;
          lastpar = (lastpar & ~(1u << c)) | (sp << c);
        }
      }
      // every copy issued lands before the CTA's shared memory is released
      for (int c = 0; c < C::ES * C::NCH; ++c)
        if (issued & (1u << c)) mbar_drain(&full[c], (lastpar >> c) & 1u, status);
    }
  } else if (warp == 2) {
    // ------------------------------------------------------------ Y / W_L ring
    if (lane == 0) {
      int s = 0;
      uint32_t ph = 0, issued = 0, lastpar = 0;
      int64_t i = 0;
      bool ok = true;
      for (int64_t b = blockIdx.x; ok && b < batch; b += gridDim.x, ++i) {
        // the epilogue stages the previous example's LCB rows in the ring: wait until it is done
        if (!C::LCB_DIRECT && i > 0 && !mbar_wait(ldone, static_cast<uint32_t>((i - 1) & 1), status)) {
          ok = false;
          break;
        }
        // per chunk: its Y box, then its W_L boxes of every LCB tile (the MMA order)
        for (int c = 0; ok && c < C::NCH; ++c) {
          const int rows = (C::N - c * C::R) < C::R ? (C::N - c * C::R) : C::R;
          const int nkb = (rows + 63) / 64;
          for (int t = -1; ok && t < C::MTL * nkb; ++t) {
            if (!mbar_wait(&wempty[s], ph ^ 1u, status)) {
              ok = false;
              break;
            }
            if (t < 0) {
              mbar_arrive_expect_tx(&wfull[s], static_cast<uint32_t>(C::YB));
              tma_load_2d(&tmY, &wfull[s], ring + s * C::STG, 0, c * C::R);
            } else {
              mbar_arrive_expect_tx(&wfull[s], static_cast<uint32_t>(C::WB));
              tma_load_2d(&tmW, &wfull[s], ring + s * C::STG, c * C::R + (t % nkb) * 64, (t / nkb) * C::R);
            }
            issued |= 1u << s;
            lastpar = (lastpar & ~(1u << s)) | (ph << s);
            if (++s == C::NSTG) {
              s = 0;
              ph ^= 1u;
            }
          }
        }
      }
      for (int t = 0; t < C::NSTG; ++t)
        if (issued & (1u << t)) mbar_drain(&wfull[t], (lastpar >> t) & 1u, status);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------- MMA issuer
    if (lane == 0) {
      const bool bf = Half16<T>::kBF16;
      const uint32_t idA = idesc_f16kind_f32(C::R, C::KP, 1, 1, bf);  // Z = X^T Y: both MN-major
      const uint32_t idL = idesc_f16kind_f32(C::R, C::D, 0, 1, bf);   // D = W_L X: X MN-major
      const uint32_t idB = idesc_f16kind_f32(C::R, C::KP, 0, 1, bf);  // F = X Z: Z MN-major
      const uint32_t ysw = C::YRB == 128 ? 2u : 4u;
      const uint32_t slot0 = smem_u32(slots);
      int s = 0;
      uint32_t ph = 0;
      int64_t i = 0;
      bool ok = true;
      bool issued = false;
      for (int64_t b = blockIdx.x; ok && b < batch; b += gridDim.x, ++i) {
        const uint32_t par = static_cast<uint32_t>(i & 1);
        const int es = static_cast<int>(i % C::ES);
        const uint32_t sp = static_cast<uint32_t>((i / C::ES) & 1);
        // Chunk by chunk as they are normalised: pass A, Z += X_c^T Y_c (the previous example's Z
        // has been turned into its pass-B operand first), and the LCB, D_m += W_L[m, c] X_c for
        // every tile m (once the previous example's F, which shares D's TMEM columns, is read),
        // so W_L streams in while the example's chunks arrive.
        if (i > 0 && !mbar_wait(zready, par ^ 1u, status)) {
          ok = false;
          break;
        }
        for (int c = 0; ok && c < C::NCH; ++c) {
          if (!mbar_wait(&xready[es * C::NCH + c], sp, status) || !mbar_wait(&wfull[s], ph, status)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const int rows = (C::N - c * C::R) < C::R ? (C::N - c * C::R) : C::R;
          const int nkb = (rows + 63) / 64;
          const uint32_t xs = slot0 + (es * C::NCH + c) * C::CHB;
          const uint32_t ys = smem_u32(ring + s * C::STG);
          for (int ks = 0; ks < rows / 16; ++ks) {
            const uint64_t bdesc = smem_desc(ys + ks * 16 * C::YRB, C::YB, 8 * C::YRB, ysw);
#pragma unroll
            for (int mz = 0; mz < C::MTZ; ++mz) {
              // MN atoms of 32 columns are the boxes (LBO), 8-row k groups 512 bytes apart
              const uint64_t adesc = smem_desc(xs + mz * 4 * C::XBOXB + ks * 16 * 64, C::XBOXB, 512, 4);
              umma_f16kind(tmem_base + mz * C::KP, adesc, bdesc, idA, (c | ks) != 0 ? 1u : 0u);
            }
          }
          umma_commit(&wempty[s]);
          issued = true;
          if (++s == C::NSTG) {
            s = 0;
            ph ^= 1u;
          }
          if (c == C::NCH - 1) umma_commit(zfull);
          // the LCB's TMEM columns are free once the previous example's LCB rows (and, when F
          // shares them, its F) have been read
          if (c == 0 && i > 0 && !mbar_wait(C::SEPF ? ldone : fempty, par ^ 1u, status)) {
            ok = false;
            break;
          }
          for (int t = 0; ok && t < C::MTL * nkb; ++t) {
            const int m = t / nkb, kb = t % nkb;
            if (!mbar_wait(&wfull[s], ph, status)) {
              ok = false;
              break;
            }
            tc_fence_after();
            const uint32_t ws = smem_u32(ring + s * C::STG);
            const int left = (rows - kb * 64) / 16;
            const int nk = left < 4 ? left : 4;
            for (int kk = 0; kk < nk; ++kk) {
              const uint64_t adesc = smem_desc(ws + kk * 32, 16, 1024, 2);
              const uint64_t bdesc = smem_desc(xs + (kb * 64 + kk * 16) * 64, C::XBOXB, 512, 4);
              umma_f16kind(tmem_base + C::LCOL + m * C::D, adesc, bdesc, idL, (c | kb | kk) != 0 ? 1u : 0u);
            }
            umma_commit(&wempty[s]);
            if (++s == C::NSTG) {
              s = 0;
              ph ^= 1u;
            }
          }
        }
        if (!ok) break;
        for (int m = 0; m < C::MTL; ++m) umma_commit(&lfull[m]);
        // pass B: F = X Z, once Z is in shared memory and F's TMEM columns are free: the
        // previous example's F has been read (F apart), or, chunk by chunk, the LCB columns
        // that F_c reuses have been read out (F in the LCB's columns), so pass B runs while
        // the rest of the LCB rows are read out
        if (!mbar_wait(zready, par, status) || !(!C::SEPF || i == 0 || mbar_wait(fempty, par ^ 1u, status))) {
          ok = false;
          break;
        }
        tc_fence_after();
        for (int c = 0; ok && c < C::NCH; ++c) {
          if constexpr (!C::SEPF) {
            if (!mbar_wait(&fcfree[c], par, status)) {
              ok = false;
              break;
            }
            tc_fence_after();
          }
          const uint32_t xs = slot0 + (es * C::NCH + c) * C::CHB;
#pragma unroll
          for (int ks = 0; ks < C::D / 16; ++ks) {
            const uint64_t adesc = smem_desc(xs + (ks >> 1) * C::XBOXB + (ks & 1) * 32, 16, 512, 4);
            const uint64_t bdesc = smem_desc(smem_u32(zb) + ks * 16 * C::YRB, C::ZB, 8 * C::YRB, ysw);
            umma_f16kind(tmem_base + C::FCOL + c * C::KP, adesc, bdesc, idB, ks != 0 ? 1u : 0u);
          }
          umma_commit(&empty[es * C::NCH + c]);  // pass B has read the chunk's slot
        }
        if (!ok) break;
        umma_commit(ffull);
      }
      if (issued) {  // no MMA may still read shared memory or write TMEM when the CTA exits
        umma_commit(fin);
        mbar_drain(fin, 0u, status);
      }
    }
  } else if (warp < FRONT_NORM_WARP0) {
    // --------------------------------------------------------------- epilogue
    const int q = warp & 3;                  // TMEM lane quarter
    const int ew = warp - FRONT_EPI_WARP0;   // 0..3
    const uint32_t lane_base = static_cast<uint32_t>(q * 32) << 16;
    const float inv_cnt = 1.0f / static_cast<float>(C::N * C::K);
    int64_t i = 0;
    // After a failed wait a warp stops waiting but keeps walking the same control flow,
    // so every named barrier still sees all four warps.
    bool ok = true;
    for (int64_t b = blockIdx.x; b < batch; b += gridDim.x, ++i) {
      const uint32_t par = static_cast<uint32_t>(i & 1);
      const int es = static_cast<int>(i % C::ES);
      const uint32_t sp = static_cast<uint32_t>((i / C::ES) & 1);
      // Z (TMEM, fp32) -> 16-bit MN-major operand in shared memory (once the previous
      // example's A0 stores staged there have read it)
      if (C::A0_TMA && lane == 0) bulk_wait_read<0>();
      __syncwarp();
      if (ok) ok = mbar_wait(zfull, par, status);
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
              asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(front_zb_addr<C>(smem_u32(zb), t, h * 4 + j)),
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

      // LCB rows: accumulator + the residual X row (from the chunk in shared memory), 32
      // columns at a time: with LCB_DIRECT transposed through this warp's own tile and stored
      // by the warp, else staged in that tile and its quarter of the Y / W_L ring (idle until
      // the drain is done) and stored by TMA (rows past n_l are clipped)
      // chunks holding no LCB row's residual are not read here: with one example in flight
      // (the next one's loads wait for these slots) they are released now, else with the rest
      constexpr int EARLY = C::ES == 1 ? C::NF / C::R : 0;
      if (lane == 0)
        for (int c = 0; c < EARLY; ++c) mbar_arrive(&empty[es * C::NCH + c]);
      for (int c = C::NF / C::R; ok && c < C::NCH; ++c) ok = mbar_wait(&xready[es * C::NCH + c], sp, status);
      int fsig = 0;  // F chunks whose LCB columns this warp has read (F in the LCB's columns)
#pragma unroll 1
      for (int m = 0; m < C::MTL; ++m) {
        if (ok) ok = mbar_wait(&lfull[m], par, status);
        tc_fence_after();
        const int r = m * C::R + q * 32 + lane;   // LCB row
        const bool valid = r < C::NL;
        const bool any = m * C::R + q * 32 < C::NL;
        const int rho = C::NF + r;                // its residual row
        const uint8_t* xres = slots + (es * C::NCH + rho / C::R) * C::CHB;
        const int rl = rho % C::R;
#pragma unroll 1
        for (int j = 0; j < C::XBOXES; ++j) {
          uint32_t acc[32];
          tmem_ld32(tmem_base + lane_base + static_cast<uint32_t>(C::LCOL + m * C::D + j * 32), acc);
          tmem_ld_wait();
          if constexpr (!C::SEPF) {
            const int read = m * C::D + 32 * (j + 1);  // LCB columns read so far
            if (fsig < C::NCH && (fsig + 1) * C::KP <= read) {
              tc_fence_before();
              __syncwarp();
              while (fsig < C::NCH && (fsig + 1) * C::KP <= read) {
                if (lane == 0) mbar_arrive(&fcfree[fsig]);
                ++fsig;
              }
            }
          }
          uint32_t o[16];
          if (valid) {
#pragma unroll
            for (int u = 0; u < 4; ++u) {
              const uint4 xr = *reinterpret_cast<const uint4*>(xres + j * C::XBOXB + sw64_off(rl, u));
              const uint32_t xw[4] = {xr.x, xr.y, xr.z, xr.w};
#pragma unroll
              for (int p = 0; p < 4; ++p)
                o[4 * u + p] = f2_to16<T>(f2_add(f2_pack(__uint_as_float(acc[8 * u + 2 * p]),
                                                         __uint_as_float(acc[8 * u + 2 * p + 1])),
                                                 f2_from16<T>(xw[p])));
            }
          } else {
#pragma unroll
            for (int e = 0; e < 16; ++e) o[e] = Half16<T>::pack2(__uint_as_float(acc[2 * e]), __uint_as_float(acc[2 * e + 1]));
          }
          if constexpr (C::LCB_DIRECT) {
            // through the warp's own 2 KB tile: each lane writes its row, then each store
            // instruction of the warp covers 8 whole 64-byte row segments (lane = 16 bytes)
            uint8_t* tile = epi + ew * 2048;
            front_stage16(tile, lane, o);
            __syncwarp();
#pragma unroll
            for (int it = 0; it < 4; ++it) {
              const int tr = it * 8 + (lane >> 2);  // tile row
              const int u = lane & 3;               // its 16-byte unit
              const uint4 val = *reinterpret_cast<const uint4*>(tile + sw64_off(tr, u));
              const int r2 = m * C::R + q * 32 + tr;  // LCB row
              if (r2 < C::NL)
                *reinterpret_cast<uint4*>(yout + (b * C::N + C::NF + r2) * C::D + 32 * j + 8 * u) = val;
            }
            __syncwarp();  // the tile is read before the next box is written into it
          } else {
            const int nb = (m * C::XBOXES + j) % C::NBUF;
            uint8_t* stage = nb == 0 ? epi + ew * 2048 : ring + ew * (C::NBUF - 1) * 2048 + (nb - 1) * 2048;
            if (lane == 0 && nb == 0) bulk_wait_read<0>();  // the tiles' last stores have read them
            __syncwarp();
            front_stage16(stage, lane, o);
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0 && any) {
              tma_store_3d(&tmL, stage, 32 * j, m * C::R + q * 32, static_cast<int32_t>(b));
              bulk_commit();
            }
          }
        }
      }
      tc_fence_before();
      if (!C::LCB_DIRECT && lane == 0) bulk_wait_read<0>();  // the ring is the producer's again
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(ldone);
        for (int c = EARLY; c < C::NCH; ++c) mbar_arrive(&empty[es * C::NCH + c]);  // residual rows read
        if constexpr (!C::SEPF)
          for (; fsig < C::NCH; ++fsig) mbar_arrive(&fcfree[fsig]);  // F past the LCB's columns
      }

      // the FMB LayerNorm over the n*k values of F
      T* ab = A0 + b * (C::N * C::K);
      const bool affine = fg != nullptr;
      if constexpr (C::REGLN) {
        // F read from TMEM once (all chunks before one wait), TMEM handed back, then mean,
        // variance and the output from registers
        if (ok) ok = mbar_wait(ffull, par, status);
        tc_fence_after();
        uint32_t fr[C::NCH][C::K];
#pragma unroll
        for (int c = 0; c < C::NCH; ++c) {
          const uint32_t ta = tmem_base + lane_base + static_cast<uint32_t>(C::FCOL + c * C::KP);
          if constexpr (C::K == 32) {
            tmem_ld32(ta, reinterpret_cast<uint32_t(&)[32]>(fr[c][0]));
          } else if constexpr (C::K == 24) {
            front_tmem_ld16(ta, reinterpret_cast<uint32_t(&)[16]>(fr[c][0]));
            front_tmem_ld8(ta + 16, reinterpret_cast<uint32_t(&)[8]>(fr[c][16]));
          } else {
            front_tmem_ld16(ta, reinterpret_cast<uint32_t(&)[16]>(fr[c][0]));
          }
        }
        tmem_ld_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(fempty);
        uint64_t pa = 0, pb = 0;  // +0.0f pairs
#pragma unroll
        for (int c = 0; c < C::NCH; ++c) {
          const int row = c * C::R + q * 32 + lane;
          if (row < C::N) {
#pragma unroll
            for (int j = 0; j < C::K; j += 4) {
              pa = f2_add(pa, f2_pack(__uint_as_float(fr[c][j]), __uint_as_float(fr[c][j + 1])));
              pb = f2_add(pb, f2_pack(__uint_as_float(fr[c][j + 2]), __uint_as_float(fr[c][j + 3])));
            }
          }
        }
        float part = warp_sum(f2_sum(pa) + f2_sum(pb));
        if (lane == 0) red[ew] = part;
        named_bar(1, 128);
        const float mean = (red[0] + red[1] + red[2] + red[3]) * inv_cnt;
        const uint64_t nm2 = f2_pack(-mean, -mean);
        uint64_t qa = 0, qb = 0;
#pragma unroll
        for (int c = 0; c < C::NCH; ++c) {
          const int row = c * C::R + q * 32 + lane;
          if (row < C::N) {
#pragma unroll
            for (int j = 0; j < C::K; j += 4) {
              const uint64_t da = f2_add(f2_pack(__uint_as_float(fr[c][j]), __uint_as_float(fr[c][j + 1])), nm2);
              const uint64_t db = f2_add(f2_pack(__uint_as_float(fr[c][j + 2]), __uint_as_float(fr[c][j + 3])), nm2);
              qa = f2_fma(da, da, qa);
              qb = f2_fma(db, db, qb);
            }
          }
        }
        float qs = warp_sum(f2_sum(qa) + f2_sum(qb));
        if (lane == 0) red[4 + ew] = qs;
        named_bar(1, 128);
        const float var = (red[4] + red[5] + red[6] + red[7]) * inv_cnt;
        const float rstd = rsqrtf(var + eps);
        if (threadIdx.x == 32 * FRONT_EPI_WARP0 && !(isfinite(mean) && isfinite(var))) flag_error(status, kFlagNonFinite);
#pragma unroll
        for (int c = 0; c < C::NCH; ++c) {
          const int row = c * C::R + q * 32 + lane;
          if (row < C::N) {
            T* o = ab + row * C::K;
            const uint64_t rs2 = f2_pack(rstd, rstd);
#pragma unroll
            for (int j = 0; j < C::K; j += 8) {
              if (affine) {
                float v[8];
                const float* gp = fg + row * C::K + j;
                const float* bp = fb + row * C::K + j;
#pragma unroll
                for (int e = 0; e < 8; ++e) v[e] = (__uint_as_float(fr[c][j + e]) - mean) * rstd * __ldg(gp + e) + __ldg(bp + e);
                *reinterpret_cast<uint4*>(o + j) = front_pack8<T>(v);
              } else {
                uint32_t w4[4];
#pragma unroll
                for (int e = 0; e < 4; ++e)
                  w4[e] = f2_to16<T>(f2_mul(f2_add(f2_pack(__uint_as_float(fr[c][j + 2 * e]),
                                                           __uint_as_float(fr[c][j + 2 * e + 1])), nm2), rs2));
                *reinterpret_cast<uint4*>(o + j) = make_uint4(w4[0], w4[1], w4[2], w4[3]);
              }
            }
          }
        }
        named_bar(1, 128);  // every epilogue warp is past its reads of red[]
      } else {
        // two passes over F in TMEM: statistics, output. The statistics in one pass: each
        // thread sums (x - s) and (x - s)^2 around its first value s (no cancellation for
        // data far from 0); the mean is reduced first, then each thread's share of the sum of
        // squared deviations follows from its sums exactly, sum (x - mean)^2 =
        // Q - 2 (mean - s) S + n (mean - s)^2, and is reduced second.
        if (ok) ok = mbar_wait(ffull, par, status);
        tc_fence_after();
        float sh = 0.f, cnt = 0.f;
        uint64_t nsh = 0, sxa = 0, sxb = 0, sqa = 0, sqb = 0;  // +0.0f pairs
#pragma unroll 1
        for (int c = 0; c < C::NCH; ++c) {
          const int row = c * C::R + q * 32 + lane;
          uint32_t r[C::KP / 32][32];
#pragma unroll
          for (int h = 0; h < C::KP / 32; ++h)
            tmem_ld32(tmem_base + lane_base + static_cast<uint32_t>(C::FCOL + c * C::KP + h * 32), r[h]);
          tmem_ld_wait();
          if (c == 0) {
            sh = __uint_as_float(r[0][0]);
            nsh = f2_pack(-sh, -sh);
          }
          if (row < C::N) {
#pragma unroll
            for (int h = 0; h < C::KP / 32; ++h)
#pragma unroll
              for (int j = 0; j < 32; j += 4)
                if (h * 32 + j < C::K) {  // K % 4 == 0
                  const uint64_t da = f2_add(f2_pack(__uint_as_float(r[h][j]), __uint_as_float(r[h][j + 1])), nsh);
                  const uint64_t db = f2_add(f2_pack(__uint_as_float(r[h][j + 2]), __uint_as_float(r[h][j + 3])), nsh);
                  sxa = f2_add(sxa, da);
                  sqa = f2_fma(da, da, sqa);
                  sxb = f2_add(sxb, db);
                  sqb = f2_fma(db, db, sqb);
                }
            cnt += static_cast<float>(C::K);
          }
        }
        const float sx = f2_sum(sxa) + f2_sum(sxb), sq = f2_sum(sqa) + f2_sum(sqb);
        float part = warp_sum(sx + cnt * sh);
        if (lane == 0) red[ew] = part;
        named_bar(1, 128);
        const float mean = (red[0] + red[1] + red[2] + red[3]) * inv_cnt;
        const float dm = mean - sh;
        float qs = warp_sum(sq - 2.f * dm * sx + cnt * dm * dm);
        if (lane == 0) red[4 + ew] = qs;
        named_bar(1, 128);
        const float var = fmaxf((red[4] + red[5] + red[6] + red[7]) * inv_cnt, 0.f);
        const float rstd = rsqrtf(var + eps);
        if (threadIdx.x == 32 * FRONT_EPI_WARP0 && !(isfinite(mean) && isfinite(var))) flag_error(status, kFlagNonFinite);
#pragma unroll 1
        for (int c = 0; c < C::NCH; ++c) {
          const int row = c * C::R + q * 32 + lane;
          uint32_t rr[C::KP / 32][32];
#pragma unroll
          for (int h = 0; h < C::KP / 32; ++h)
            tmem_ld32(tmem_base + lane_base + static_cast<uint32_t>(C::FCOL + c * C::KP + h * 32), rr[h]);
          tmem_ld_wait();
#pragma unroll
          for (int h = 0; h < C::KP / 32; ++h) {
            uint32_t o[16];
            if (affine && row < C::N) {
              float v[32];
              const float* gp = fg + row * C::K + h * 32;
              const float* bp = fb + row * C::K + h * 32;
#pragma unroll
              for (int e = 0; e < 32; ++e) {
                v[e] = (__uint_as_float(rr[h][e]) - mean) * rstd;
                if (h * 32 + e < C::K) v[e] = v[e] * __ldg(gp + e) + __ldg(bp + e);
              }
#pragma unroll
              for (int e = 0; e < 16; ++e) o[e] = Half16<T>::pack2(v[2 * e], v[2 * e + 1]);
            } else {
              const uint64_t nm2 = f2_pack(-mean, -mean), rs2 = f2_pack(rstd, rstd);
#pragma unroll
              for (int e = 0; e < 16; ++e)
                o[e] = f2_to16<T>(f2_mul(f2_add(f2_pack(__uint_as_float(rr[h][2 * e]), __uint_as_float(rr[h][2 * e + 1])),
                                                nm2), rs2));
            }
            if constexpr (C::A0_TMA) {
              const int t = c * 2 + h;  // tile, three staging buffers in turn
              uint8_t* buf = (t % 3 == 0) ? epi + ew * 2048 : zb + ew * 4096 + (t % 3 - 1) * 2048;
              if (lane == 0) bulk_wait_read<2>();  // the store that last used this buffer has read it
              __syncwarp();
              front_stage16(buf, lane, o);
              fence_proxy_async_smem();
              __syncwarp();
              if (lane == 0) {
                tma_store_2d(&tmA, buf, 32 * h, static_cast<int32_t>(b * C::N + c * C::R + q * 32));
                bulk_commit();
              }
            } else if (row < C::N) {
              T* op = ab + row * C::K + h * 32;
#pragma unroll
              for (int j = 0; j < 32; j += 8)
                if (h * 32 + j < C::K)
                  *reinterpret_cast<uint4*>(op + j) = make_uint4(o[j / 2], o[j / 2 + 1], o[j / 2 + 2], o[j / 2 + 3]);
            }
          }
        }
        tc_fence_before();
        named_bar(1, 128);  // every epilogue warp is past its reads of red[] and F
        if (lane == 0) mbar_arrive(fempty);
      }
    }
    if (lane == 0) bulk_wait<0>();
    __syncwarp();
  } else {
    // ---------------------------------------------------------- normalisation
    // Two threads per row (adjacent lanes), each with half of the row's 16-byte units:
    // the layer input's LayerNorm (two-pass fp32 statistics from registers) or, for the
    // first layer, the conversion to the operand type, written back in place.
    constexpr int UPR = C::D / 8;     // 16-byte units per row (of 16-bit values)
    constexpr int UPT = UPR / 2;      // per thread
    const int tid = threadIdx.x - 32 * FRONT_NORM_WARP0;
    const int row = tid >> 1;
    const int half = tid & 1;
    int pending = -1;  // tid 0: the chunk whose residual stores are the last still reading their slot
    int64_t i = 0;
    bool ok = true;
    for (int64_t b = blockIdx.x; b < batch; b += gridDim.x, ++i) {
      const int es = static_cast<int>(i % C::ES);
      const uint32_t sp = static_cast<uint32_t>((i / C::ES) & 1);
      for (int c = 0; c < C::NCH; ++c) {
        const int sc = es * C::NCH + c;
        if (ok) ok = mbar_wait(&full[sc], sp, status);
        const int rows = (C::N - c * C::R) < C::R ? (C::N - c * C::R) : C::R;
        uint8_t* base = slots + sc * C::CHB;
        const bool act = ok && row < rows;
        // the row as loaded (row-major, d values), into registers; every thread reads before
        // any thread writes the operand layout over the same bytes
        uint4 w[UPT];
#pragma unroll
        for (int k = 0; k < UPT; ++k) {
          const int g = half * UPT + k;  // unit within the row
          w[k] = act ? *reinterpret_cast<const uint4*>(base + row * (C::D * 2) + g * 16) : make_uint4(0u, 0u, 0u, 0u);
        }
        named_bar(2, FRONT_NORM_THREADS);
        if (ln_in) {
          // one pass over the row for its statistics: sums of (x - s) and (x - s)^2 around the
          // row's first value s (both threads of the row use it), no cancellation for rows far
          // from 0; fp32 pairs in two accumulator sets, so no chain is longer than UPT * 2
          const float sh = __shfl_sync(0xffffffffu, Half16<TIN>::lo(w[0].x), lane & ~1);
          const uint64_t nsh = f2_pack(-sh, -sh);
          uint64_t sxa = 0, sxb = 0, sqa = 0, sqb = 0;  // +0.0f pairs
#pragma unroll
          for (int k = 0; k < UPT; ++k) {
            const uint32_t ww[4] = {w[k].x, w[k].y, w[k].z, w[k].w};
#pragma unroll
            for (int p = 0; p < 4; p += 2) {
              const uint64_t da = f2_add(f2_from16<TIN>(ww[p]), nsh);
              const uint64_t db = f2_add(f2_from16<TIN>(ww[p + 1]), nsh);
              sxa = f2_add(sxa, da);
              sqa = f2_fma(da, da, sqa);
              sxb = f2_add(sxb, db);
              sqb = f2_fma(db, db, sqb);
            }
          }
          float sx = f2_sum(sxa) + f2_sum(sxb), sq = f2_sum(sqa) + f2_sum(sqb);
          sx += __shfl_xor_sync(0xffffffffu, sx, 1);
          sq += __shfl_xor_sync(0xffffffffu, sq, 1);
          const float dmean = sx * (1.0f / C::D);
          const float mean = sh + dmean;
          const float qv = fmaxf(sq - sx * dmean, 0.f);  // sum of (x - mean)^2
          const float rstd = rsqrtf(qv * (1.0f / C::D) + eps);
          if (act && half == 0 && !(isfinite(mean) && isfinite(qv))) flag_error(status, kFlagNonFinite);
          if (act) {
            const uint64_t nm2 = f2_pack(-mean, -mean), rs2 = f2_pack(rstd, rstd);
#pragma unroll
            for (int k = 0; k < UPT; ++k) {
              const int g = half * UPT + k;
              const uint32_t ww[4] = {w[k].x, w[k].y, w[k].z, w[k].w};
              const ulonglong2 g0 = reinterpret_cast<const ulonglong2*>(sg)[2 * g];
              const ulonglong2 g1 = reinterpret_cast<const ulonglong2*>(sg)[2 * g + 1];
              const ulonglong2 b0 = reinterpret_cast<const ulonglong2*>(sb)[2 * g];
              const ulonglong2 b1 = reinterpret_cast<const ulonglong2*>(sb)[2 * g + 1];
              const uint64_t ga[4] = {g0.x, g0.y, g1.x, g1.y};
              const uint64_t be[4] = {b0.x, b0.y, b1.x, b1.y};
              uint32_t o[4];
#pragma unroll
              for (int p = 0; p < 4; ++p) {
                // ((x - mean) * rstd) * gamma + beta, lane by lane
                const uint64_t t = f2_mul(f2_add(f2_from16<TIN>(ww[p]), nm2), rs2);
                o[p] = f2_to16<T>(f2_fma(t, ga[p], be[p]));
              }
              *reinterpret_cast<uint4*>(base + (g >> 2) * C::XBOXB + sw64_off(row, g & 3)) = make_uint4(o[0], o[1], o[2], o[3]);
            }
          }
        } else if (act) {  // the first layer: the input in the operand type, in the operand layout
#pragma unroll
          for (int k = 0; k < UPT; ++k) {
            const int g = half * UPT + k;
            uint4 o = w[k];
            if (sizeof(TIN) != sizeof(T) || Half16<TIN>::kBF16 != Half16<T>::kBF16) {
              float v[8];
              front_unpack8<TIN>(w[k], v);
              o = front_pack8<T>(v);
            }
            *reinterpret_cast<uint4*>(base + (g >> 2) * C::XBOXB + sw64_off(row, g & 3)) = o;
          }
        }
        fence_proxy_async_smem();  // the tensor core and the TMA store read the chunk
        named_bar(2, FRONT_NORM_THREADS);
        if (tid == 0) {
          mbar_arrive(&xready[sc]);
          // The FMB rows' residual (rows past n_f are clipped). The slot is released (one of
          // its two arrivals) once its stores have read it: the previous chunk's is released
          // here, after this chunk's stores are issued, so no chunk waits for its own.
          const bool st = ok && c * C::R < C::NF;
          if (st) {
#pragma unroll
            for (int j = 0; j < C::XBOXES; ++j) tma_store_3d(&tmR, base + j * C::XBOXB, 32 * j, c * C::R,
                                                             static_cast<int32_t>(b));
            bulk_commit();
          }
          if (pending >= 0) {
            if (st) bulk_wait_read<1>();
            else bulk_wait_read<0>();
            mbar_arrive(&empty[pending]);
          }
          pending = sc;
        }
      }
      if (tid == 0 && pending >= 0) {
        bulk_wait_read<0>();
        mbar_arrive(&empty[pending]);
        pending = -1;
      }
    }
    if (tid == 0) bulk_wait<0>();
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, C::TMEM_COLS);
  }
}

// LCB rows by direct stores where that measured faster (the 2- and 8-layer shapes: 0.100 ->
// 0.087 ms and 0.522 -> 0.506 ms per launch; the 4-layer shape: 0.686 -> 0.711 ms, so it keeps
// the TMA stores)
using FrontC2 = FrontCfg<64, 128, 16, 32, true>;
using FrontC3 = FrontCfg<256, 160, 32, 128, false>;
using FrontC4 = FrontCfg<512, 160, 64, 256, true>;

}  // namespace wk
