// whale.cuh -- the attention-based fusion module of WHALE on the 5th-generation
// tensor cores (WHALE pages, gist.science summaries of arXiv 2607.17017: section 2.1
// item 3, attention-based fusion; section 2.2, shared key-value and shared-gate SwiGLU).
//
// Per example, with H_w (n x d) the Wukong representation and H_s (L x d) the sequence
// representation (one head, no projections; K = V = H_s):
//
//   A   = softmax_rows( H_w H_s^T / sqrt(d) ) H_s                 whale_attn_kernel
//   Z   = [H_w | A] W_F^T + b_F                 (fusion Linear)    whale_ffn_kernel
//   U   = LN(Z) W_up^T                          (pre-norm)
//   H_f = Z + ( SiLU(U) * U ) W_down^T          (W_gate = W_up, residual)
//
// whale_attn_kernel: one CTA per SM walks (example, 128-query tile) units. Warp 0 streams
// the query tile and 128-key tiles of H_s with TMA; each key tile is loaded into shared
// memory ONCE and read twice by the tensor core: as the K-major operand of S = Q K^T and
// as the MN-major operand of O += P V (the page's shared K = V, which halves the key/value
// traffic). Warp 1 issues the MMAs (S double-buffered in TMEM, S of the next block issued
// before P V of this one). Warps 2..5 (one query row per thread) run the online softmax
// from TMEM: P = 2^(S log2(e)/sqrt(d) - m) rounded to the operand type into shared memory,
// row sums in fp32. The running max m is raised only when a block's max exceeds it by
// more than 8 (P <= 2^8, exact in fp32 and in the 16-bit operand's exponent range), and
// only then is the O row rescaled in TMEM; the result is the same softmax, with fewer
// rescales. The last block of a ragged L is masked; query rows past n are zero rows of
// the TMA box and are never stored.
//
// whale_ffn_kernel: one CTA per SM walks 128-row tiles of the batch's B*n rows. Z is
// accumulated in TMEM from the [H_w | A] tile and W_F; the epilogue warps add b_F, take
// the LayerNorm over d (fp32, two passes over TMEM) and write LN(Z) to shared memory;
// the FFN then runs in chunks of 64 columns of h: U_c = LN(Z) W_up_c^T into TMEM, the
// epilogue writes G_c = U_c^2 / (1 + exp(-U_c)) to shared memory, and the down
// projection accumulates G_c W_down_c^T onto Z's own TMEM columns, so the residual costs
// nothing. H_f = that sum + b_F, staged in shared memory and written with TMA stores.
// Weights stream through a TMA ring from L2.
//
// Every mbarrier wait is bounded (common.cuh); on a failed wait the threads stop waiting,
// let issued copies land, let issued MMAs finish and free TMEM before the CTA exits.
#pragma once

#include <type_traits>

#include "common.cuh"

namespace wk {

__device__ __forceinline__ void whale_tmem_st32(uint32_t taddr, const uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], "
      "{%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16, "
      "%17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31, %32};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]), "r"(r[9]),
      "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15]), "r"(r[16]), "r"(r[17]), "r"(r[18]),
      "r"(r[19]), "r"(r[20]), "r"(r[21]), "r"(r[22]), "r"(r[23]), "r"(r[24]), "r"(r[25]), "r"(r[26]), "r"(r[27]),
      "r"(r[28]), "r"(r[29]), "r"(r[30]), "r"(r[31])
      : "memory");
}

__device__ __forceinline__ void whale_tmem_st_wait() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

// 2^x (the hardware's approximate base-2 exponential; 2^-inf = +0).
__device__ __forceinline__ float whale_ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// Byte offset of 16-byte unit j of row r inside a K-major tile written with the TMA's
// 128-byte (row pitch 128) or 64-byte (row pitch 64) swizzle.
template <int SWB>
__device__ __forceinline__ uint32_t whale_swz(int r, int j) {
  return static_cast<uint32_t>(r * SWB + ((SWB == 128 ? (j ^ (r & 7)) : (j ^ ((r >> 1) & 3))) << 4));
}

// max(a, b, c) in one instruction.
__device__ __forceinline__ float whale_max3(float a, float b, float c) {
  float r;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}

// max of 64 fp32 values held as bit patterns: a tree of three-input maxima (32 instructions,
// short dependency chains).
__device__ __forceinline__ float whale_max64(const uint32_t (&v)[64]) {
  float t[22], u[8];
#pragma unroll
  for (int i = 0; i < 21; ++i)
    t[i] = whale_max3(__uint_as_float(v[3 * i]), __uint_as_float(v[3 * i + 1]), __uint_as_float(v[3 * i + 2]));
  t[21] = __uint_as_float(v[63]);
#pragma unroll
  for (int i = 0; i < 7; ++i) u[i] = whale_max3(t[3 * i], t[3 * i + 1], t[3 * i + 2]);
  u[7] = t[21];
  return whale_max3(whale_max3(u[0], u[1], u[2]), whale_max3(u[3], u[4], u[5]), fmaxf(u[6], u[7]));
}

// 2^x on the FMA pipe, for some of the softmax weights, so that the special-function
// unit (the approximate ex2 above) does not bound the softmax alone. x = j + f with j the
// integer nearest to x (adding 1.5 * 2^23 rounds it into the low mantissa bits) and
// f in [-1/2, 1/2]; 2^f is a degree-3 polynomial fitted to 2^f by relative least squares
// on Chebyshev nodes for this kernel (max relative error 7.5e-5 in fp32, below the 16-bit
// rounding of the weights); 2^j enters as j added to the exponent bits. x is clamped
// below at -126 (2^-126 stands for 0).
__device__ __forceinline__ float whale_ex2_poly(float x) {
  x = fmaxf(x, -126.f);
  const float t = x + 12582912.f;
  const float f = x - (t - 12582912.f);
  const float p = fmaf(fmaf(fmaf(0.05517158f, f, 0.24261111f), f, 0.69326103f), f, 0.99992806f);
  return __uint_as_float(__float_as_uint(p) + (__float_as_uint(t) << 23));
}

// b_F[i], or zero when the fusion Linear has no bias.
__device__ __forceinline__ float whale_bias(const float* __restrict__ b, int i) { return b ? __ldg(&b[i]) : 0.f; }

template <typename T>
__device__ __forceinline__ void whale_st_row32(T* dst, const uint32_t (&r)[32], float scale, const float* add) {
  uint32_t p[16];
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    float a = __uint_as_float(r[2 * i]) * scale, b = __uint_as_float(r[2 * i + 1]) * scale;
    if (add) {
      a += add[2 * i];
      b += add[2 * i + 1];
    }
    p[i] = Half16<T>::pack2(a, b);
  }
  uint4* d4 = reinterpret_cast<uint4*>(dst);
#pragma unroll
  for (int i = 0; i < 4; ++i) d4[i] = make_uint4(p[4 * i], p[4 * i + 1], p[4 * i + 2], p[4 * i + 3]);
}

// ----------------------------------------------------------------- attention

// D[tmem] (+)= A[tmem] * B[smem]^T, kind::f16, issued by one thread: A is read from tensor
// memory (row i in lane i, consecutive 16-bit K elements packed two per 32-bit column).
__device__ __forceinline__ void whale_umma_ts(uint32_t tmem_d, uint32_t tmem_a, uint64_t bdesc, uint32_t idesc,
                                              uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(tmem_d),
      "r"(tmem_a), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}

__device__ __forceinline__ void whale_tmem_st8(uint32_t taddr, const uint32_t* r) {
  asm volatile("tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};" ::"r"(taddr), "r"(r[0]),
               "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7])
               : "memory");
}

// NC consecutive 32-bit TMEM columns (a multiple of 8) from registers.
template <int NC>
__device__ __forceinline__ void whale_tmem_st_cols(uint32_t taddr, const uint32_t (&r)[NC]) {
#pragma unroll
  for (int c = 0; c + 32 <= NC; c += 32) whale_tmem_st32(taddr + c, *reinterpret_cast<const uint32_t(*)[32]>(&r[c]));
#pragma unroll
  for (int c = (NC / 32) * 32; c < NC; c += 8) whale_tmem_st8(taddr + c, &r[c]);
}

template <int D_>
struct WaCfg {
  static constexpr int D = D_;
  static constexpr int R = 128;                          // query rows per tile (MMA M)
  static constexpr int LB = 128;                         // keys per block (N of S, K of P V)
  static constexpr int BW = (D % 64 == 0) ? 64 : 32;     // columns per TMA box
  static constexpr int SWB = BW * 2;                     // bytes per box row = swizzle span
  static constexpr uint32_t SWMODE = BW == 64 ? 2u : 4u; // descriptor swizzle: 128B / 64B
  static constexpr int NBOX = D / BW;
  static constexpr int KVBOXB = LB * SWB;
  static constexpr int KVB = NBOX * KVBOXB;              // one key/value tile
  static constexpr int LIMIT = 227 * 1024;
  static constexpr int BARB = 176;                       // mbarriers and the TMEM address
  static constexpr int REDB = 4 * R * 4;                 // softmax pair exchange [2 parities][2 halves][R]
  // The dynamic shared memory starts 1024-byte aligned (checked at run time): no slack.
  static constexpr int FIXED = BARB + REDB;
  static constexpr int STAGES_RAW = (LIMIT - FIXED) / KVB;
  static constexpr int STAGES = STAGES_RAW > 6 ? 6 : STAGES_RAW;
  // at least half an SM's shared memory: one CTA per SM, so that its 512 TMEM columns are free
  static constexpr int SMEM = FIXED + STAGES * KVB > 120 * 1024 ? FIXED + STAGES * KVB : 120 * 1024;
  // TMEM: S0 [0,128), S1 [128,256) (P_j written over the first 64 columns of S_j), O [256, 256+D),
  // Q [256+D, 256+D+D/2) (16-bit pairs)
  static constexpr int OCOL = 2 * LB;
  static constexpr int QCOL = OCOL + D;
  static_assert(D % 32 == 0 && D >= 32 && D <= 160, "D");
  static_assert(QCOL + D / 2 <= 512, "TMEM columns");
  static_assert(STAGES >= 2, "shared memory");
  static_assert(KVB % 1024 == 0, "swizzle atoms stay aligned");
  static_assert((2 * STAGES + 9) * 8 + 4 <= BARB, "barriers");
};

constexpr int WA_THREADS = 320;  // producer, MMA issuer, 8 softmax warps

template <class C, typename T>
__global__ void __launch_bounds__(WA_THREADS, 1)
    whale_attn_kernel(const __grid_constant__ CUtensorMap tmKV, const T* __restrict__ Hw, T* __restrict__ Aout,
                      int64_t batch, int n, int L, float scale_log2, unsigned* status) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  if ((smem_u32(smem_raw) & 1023u) != 0u) {  // the swizzled layout needs 1024-byte alignment
    if (threadIdx.x == 0) flag_error(status, kFlagBadShape);
    return;
  }
  uint8_t* sKV = smem_raw;
  uint64_t* bars = reinterpret_cast<uint64_t*>(sKV + C::STAGES * C::KVB);
  uint64_t* kv_full = bars;                  // [STAGES] key tile landed
  uint64_t* kv_empty = bars + C::STAGES;     // [STAGES] both products read it
  uint64_t* s_full = bars + 2 * C::STAGES;   // [2] S in TMEM
  uint64_t* p_full = s_full + 2;             // [2] P in TMEM
  uint64_t* p_empty = s_full + 4;            // [2] P V has read it (so O holds that block)
  uint64_t* q_full = s_full + 6;             // the unit's Q rows are in TMEM
  uint64_t* o_empty = s_full + 7;            // O read by the softmax warps (per unit)
  uint64_t* fin = s_full + 8;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(s_full + 9);
  float* red_max = reinterpret_cast<float*>(sKV + C::STAGES * C::KVB + C::BARB);  // [2 parities][2 halves][R]

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    prefetch_tmap(&tmKV);
    for (int s = 0; s < C::STAGES; ++s) {
      mbar_init(&kv_full[s], 1);
      mbar_init(&kv_empty[s], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&s_full[i], 1);
      mbar_init(&p_full[i], 8);
      mbar_init(&p_empty[i], 1);
    }
    mbar_init(q_full, 8);
    mbar_init(o_empty, 8);
    mbar_init(fin, 1);
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const int qtiles = (n + C::R - 1) / C::R;
  const int64_t units = batch * qtiles;
  const int nb = (L + C::LB - 1) / C::LB;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      int s = 0;
      uint32_t ph = 0;
      bool ok = true;
      for (int64_t u = blockIdx.x; ok && u < units; u += gridDim.x) {
        const int b = static_cast<int>(u / qtiles);
        for (int j = 0; j < nb; ++j) {
          if (!mbar_wait(&kv_empty[s], ph ^ 1u, status)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&kv_full[s], static_cast<uint32_t>(C::KVB));
#pragma unroll
          for (int bx = 0; bx < C::NBOX; ++bx)
            tma_load_3d(&tmKV, &kv_full[s], sKV + s * C::KVB + bx * C::KVBOXB, bx * C::BW, j * C::LB, b);
          if (++s == C::STAGES) {
            s = 0;
            ph ^= 1u;
          }
        }
      }
      if (!ok) {  // copies already issued must land before the CTA exits
        for (int i = 0; i < C::STAGES; ++i) mbar_drain(&kv_full[i], ph ^ (i < s ? 0u : 1u), status);
      }
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------- MMA issuer
    // Both products read their A operand from TMEM (Q, then P) and only the key tile from
    // shared memory. The MMAs of this thread run in issue order, so S_{j+2} is written
    // into S_j's columns only after P V_j (issued before it) has read P_j from there.
    if (lane == 0) {
      const bool bf = Half16<T>::kBF16;
      const uint32_t idS = idesc_f16kind_f32(C::R, C::LB, 0, 0, bf);  // S = Q K^T: K K-major
      const uint32_t idO = idesc_f16kind_f32(C::R, C::D, 0, 1, bf);   // O += P V: V MN-major
      int ns = 0, cs = 0;  // ring slots of the next S block and of the next P V block
      uint32_t nph = 0, g = 0, uc = 0;
      bool ok = true;
      auto issue_s = [&](uint32_t gb) -> bool {
        if (!mbar_wait(&kv_full[ns], nph, status)) return false;
        tc_fence_after();
        const uint32_t ka = smem_u32(sKV + ns * C::KVB);
#pragma unroll
        for (int ks = 0; ks < C::D / 16; ++ks) {
          const int bx = ks / (C::BW / 16), kin = ks % (C::BW / 16);
          const uint64_t bd = smem_desc(ka + bx * C::KVBOXB + kin * 32, 16, 8 * C::SWB, C::SWMODE);
          whale_umma_ts(tmem + (gb & 1u) * C::LB, tmem + C::QCOL + ks * 8, bd, idS, ks != 0 ? 1u : 0u);
        }
        umma_commit(&s_full[gb & 1u]);
        if (++ns == C::STAGES) {
          ns = 0;
          nph ^= 1u;
        }
        return true;
      };
      for (int64_t u = blockIdx.x; ok && u < units; u += gridDim.x, ++uc) {
        if (!mbar_wait(q_full, uc & 1u, status)) {
          ok = false;
          break;
        }
        tc_fence_after();
        if (!issue_s(g)) {
          ok = false;
          break;
        }
        for (int j = 0; j < nb; ++j) {
          const uint32_t gj = g + static_cast<uint32_t>(j);
          if (j + 1 < nb && !issue_s(gj + 1)) {
            ok = false;
            break;
          }
          if (j == 0 && uc > 0 && !mbar_wait(o_empty, (uc - 1) & 1u, status)) {
            ok = false;
            break;
          }
          if (!mbar_wait(&p_full[gj & 1u], (gj >> 1) & 1u, status)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t va = smem_u32(sKV + cs * C::KVB);
#pragma unroll
          for (int ks = 0; ks < C::LB / 16; ++ks) {
            // MN-major V: BW-column atoms C::KVBOXB apart, 8-key groups 8 * SWB apart
            const uint64_t bd = smem_desc(va + ks * 16 * C::SWB, C::KVBOXB, 8 * C::SWB, C::SWMODE);
            whale_umma_ts(tmem + C::OCOL, tmem + (gj & 1u) * C::LB + ks * 8, bd, idO, (j | ks) != 0 ? 1u : 0u);
          }
          umma_commit(&p_empty[gj & 1u]);
          umma_commit(&kv_empty[cs]);
          if (++cs == C::STAGES) cs = 0;
        }
        g += static_cast<uint32_t>(nb);
      }
      umma_commit(fin);  // no MMA may still write TMEM when it is freed
      mbar_drain(fin, 0u, status);
    }
  } else {
    // ------------------------------------------------------------- softmax
    // Two warps per TMEM lane quarter: warp w reads rows 32 (w % 4) .. + 31 (the
    // quarter its hardware sub-partition may access) and the key columns
    // 64 * half .. + 63 of each S block. The pair exchanges per-row partial maxima
    // (double-buffered by block parity) and, at the end of a unit, partial row sums,
    // through shared memory under a 64-thread named barrier.
    const int q = warp & 3;
    const int half = (warp - 2) >> 2;
    const int row = q * 32 + lane;
    const uint32_t lane_base = static_cast<uint32_t>(q * 32) << 16;
    const int bar_id = 1 + q;
    uint32_t g = 0;
    // After a failed wait a thread stops waiting but walks the same schedule, so the
    // warp-collective TMEM accesses and the pair barriers stay converged.
    bool ok = true;
    for (int64_t u = blockIdx.x; u < units; u += gridDim.x) {
      const int b = static_cast<int>(u / qtiles), q0 = static_cast<int>(u % qtiles) * C::R;
      const bool warp_on = q0 + q * 32 < n;  // the pair agrees: same rows
      const bool row_on = q0 + row < n;
      // The unit's query rows into TMEM (this half's D/2 columns, as 16-bit pairs); every
      // S product of the previous unit has completed (its last S block was waited for).
      {
        uint32_t qv[C::D / 4];
        if (row_on) {
          const uint4* src =
              reinterpret_cast<const uint4*>(Hw + (static_cast<int64_t>(b) * n + q0 + row) * C::D + half * (C::D / 2));
#pragma unroll
          for (int i = 0; i < C::D / 16; ++i) {
            const uint4 v = __ldg(src + i);
            qv[4 * i] = v.x;
            qv[4 * i + 1] = v.y;
            qv[4 * i + 2] = v.z;
            qv[4 * i + 3] = v.w;
          }
        } else {
#pragma unroll
          for (int i = 0; i < C::D / 4; ++i) qv[i] = 0u;
        }
        whale_tmem_st_cols<C::D / 4>(tmem + lane_base + C::QCOL + half * (C::D / 4), qv);
        whale_tmem_st_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(q_full);
      }
      float m = -INFINITY, l = 0.f;
      for (int j = 0; j < nb; ++j) {
        const uint32_t gj = g + static_cast<uint32_t>(j), buf = gj & 1u;
        if (ok) ok = mbar_wait(&s_full[buf], (gj >> 1) & 1u, status);
        tc_fence_after();
        uint32_t sr[C::LB / 2];
        if (warp_on) {
          const uint32_t ta = tmem + lane_base + buf * C::LB + half * (C::LB / 2);
          tmem_ld32(ta, *reinterpret_cast<uint32_t(*)[32]>(&sr[0]));
          tmem_ld32(ta + 32, *reinterpret_cast<uint32_t(*)[32]>(&sr[32]));
          tmem_ld_wait();
        }
        const int kvalid = min(C::LB, L - j * C::LB) - half * (C::LB / 2);  // valid columns of this half
        const bool full = kvalid >= C::LB / 2;
        // P = 2^(S log2(e)/sqrt(d) - mrow) for this half's columns, rounded to the operand
        // type and packed in registers; one weight in four from the polynomial.
        uint32_t pk[C::LB / 4];
        float lsum = 0.f;
        auto weights = [&](float mrow, auto full_block) {
          constexpr bool kFull = decltype(full_block)::value;  // no column masks on a full block
          const float nm = row_on ? -mrow : 0.f;
          float s4[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
          for (int c2 = 0; c2 < C::LB / 4; ++c2) {
            const float x0 = fmaf(__uint_as_float(sr[2 * c2]), scale_log2, nm);
            const float x1 = fmaf(__uint_as_float(sr[2 * c2 + 1]), scale_log2, nm);
            float p0 = whale_ex2(x0);
            float p1 = (c2 & 1) ? whale_ex2_poly(x1) : whale_ex2(x1);
            if constexpr (!kFull) {
              if (2 * c2 >= kvalid) p0 = 0.f;
              if (2 * c2 + 1 >= kvalid) p1 = 0.f;
            }
            s4[(2 * c2) & 3] += p0;
            s4[(2 * c2 + 1) & 3] += p1;
            pk[c2] = Half16<T>::pack2(p0, p1);
          }
          lsum = (s4[0] + s4[1]) + (s4[2] + s4[3]);
        };
        // From the second block of a row on, the weights are computed with the running max
        // m at once, next to this block's max; they are recomputed only when the block's
        // max exceeds m by more than 8 (then m is raised and O rescaled).
        const bool spec = j > 0;
        if (warp_on && spec) {
          if (full) weights(m, std::true_type{});
          else weights(m, std::false_type{});
        }
        float mh = -INFINITY;
        if (full) {
          mh = whale_max64(sr);
        } else {
#pragma unroll
          for (int c = 0; c < C::LB / 2; ++c)
            if (c < kvalid) mh = fmaxf(mh, __uint_as_float(sr[c]));
        }
        red_max[(buf * 2 + half) * C::R + row] = mh;
        // after this barrier both warps of the pair have read S_j: P_j may overwrite it
        tc_fence_before();
        named_bar(bar_id, 64);
        tc_fence_after();
        const float mb = fmaxf(mh, red_max[(buf * 2 + (half ^ 1)) * C::R + row]);
        const float mb2 = mb * scale_log2;
        const bool need = warp_on && row_on && (mb2 > m + 8.f);
        const float mnew = need ? mb2 : m;
        const float factor = need ? whale_ex2(m - mnew) : 1.f;
        const bool redo = warp_on && (!spec || __any_sync(0xffffffffu, need));
        if (redo) {
          if (full) weights(mnew, std::true_type{});
          else weights(mnew, std::false_type{});
        }
        // P V two blocks back has completed (keeps this waiter within one phase of p_empty)
        if (ok) ok = mbar_wait(&p_empty[buf], ((gj >> 1) & 1u) ^ 1u, status);
        if (spec && redo) {
          // the running max was raised: O must hold every earlier block before it is rescaled
          const uint32_t gp = gj - 1u;
          if (ok) ok = mbar_wait(&p_empty[gp & 1u], (gp >> 1) & 1u, status);
          tc_fence_after();
#pragma unroll 1
          for (int cc = half; cc < C::D / 32; cc += 2) {
            uint32_t o[32];
            tmem_ld32(tmem + lane_base + C::OCOL + cc * 32, o);
            tmem_ld_wait();
#pragma unroll
            for (int i = 0; i < 32; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * factor);
            whale_tmem_st32(tmem + lane_base + C::OCOL + cc * 32, o);
          }
        }
        l = l * factor + lsum;
        m = mnew;
        // P_j over the first 64 columns of S_j: keys 64 half .. + 63 in columns 32 half .. + 31
        if (warp_on) whale_tmem_st32(tmem + lane_base + buf * C::LB + half * 32, pk);
        whale_tmem_st_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&p_full[buf]);
      }
      // the unit's output rows: O / (l of both halves). The row sums go through the max
      // exchange slot of the parity the last block did not use; the second pair barrier
      // keeps the next unit from overwriting it before the partner has read it.
      const uint32_t gl = g + static_cast<uint32_t>(nb) - 1u;
      float* red_sum = red_max + ((gl + 1u) & 1u) * 2 * C::R;
      red_sum[half * C::R + row] = l;
      named_bar(bar_id, 64);
      const float lt = l + red_sum[(half ^ 1) * C::R + row];
      named_bar(bar_id, 64);
      if (ok) ok = mbar_wait(&p_empty[gl & 1u], (gl >> 1) & 1u, status);
      tc_fence_after();
      if (warp_on) {
        const float inv = row_on ? 1.f / lt : 0.f;
        T* dst = Aout + (static_cast<int64_t>(b) * n + q0 + row) * C::D;
#pragma unroll 1
        for (int cc = half; cc < C::D / 32; cc += 2) {
          uint32_t o[32];
          tmem_ld32(tmem + lane_base + C::OCOL + cc * 32, o);
          tmem_ld_wait();
          if (row_on && ok) whale_st_row32<T>(dst + cc * 32, o, inv, nullptr);
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(o_empty);
      g += static_cast<uint32_t>(nb);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// --------------------------------------------------------- fusion + FFN

template <int D_>
struct WfCfg {
  static constexpr int D = D_;
  static constexpr int R = 128;                          // rows per tile (MMA M)
  static constexpr int HC = 64;                          // FFN columns per chunk
  static constexpr int BW = (D % 64 == 0) ? 64 : 32;
  static constexpr int SWB = BW * 2;
  static constexpr uint32_t SWMODE = BW == 64 ? 2u : 4u;
  static constexpr int NBOX = D / BW;
  static constexpr int TBOXB = R * SWB;                  // one box of a 128-row tile
  static constexpr int CB = 2 * NBOX * TBOXB;            // [H_w | A], 128 x 2D
  static constexpr int ZNB = NBOX * TBOXB;               // LN(Z), 128 x D
  static constexpr int GBOX = HC / BW;
  static constexpr int GB = GBOX * TBOXB;                // one gated chunk, 128 x HC
  static constexpr int WDBOXB = D * SWB;                 // W_F / W_down box: D rows x BW
  static constexpr int WUBOXB = HC * SWB;                // W_up box: HC rows x BW
  static constexpr int WS = 128 * D;                     // one weight chunk (D x 64 or 64 x D, 16-bit)
  static constexpr int NKC = 2 * D / 64;                 // W_F chunks of 64 input columns
  static constexpr int LIMIT = 227 * 1024;
  static constexpr int REDB = 4 * R * 4;                 // epilogue pair exchange [sum | squares][2 halves][R]
  static constexpr int PRMB = 3 * D * 4;                 // b_F, gamma, beta staged once per CTA
  static constexpr int FIXED = 1024 + CB + ZNB + 2 * GB + 512 + REDB + PRMB;
  static constexpr int STAGES_RAW = (LIMIT - FIXED) / WS;
  static constexpr int STAGES = STAGES_RAW > 4 ? 4 : STAGES_RAW;
  static constexpr int SMEM = FIXED + STAGES * WS > 120 * 1024 ? FIXED + STAGES * WS : 120 * 1024;
  static constexpr int UCOL = 2 * D;                     // TMEM: Z/out x2 [0, 2D), U x2 [2D, 2D + 128)
  static_assert(D % 32 == 0 && D >= 32 && D <= 192, "D");
  static_assert(UCOL + 2 * HC <= 512, "TMEM columns");
  static_assert(STAGES >= 2, "shared memory");
  static_assert(CB % 1024 == 0 && ZNB % 1024 == 0 && GB % 1024 == 0 && WS % 1024 == 0, "swizzle atoms stay aligned");
  static_assert(WDBOXB % 512 == 0 && WUBOXB % 512 == 0, "swizzle atoms stay aligned");
};

constexpr int WF_THREADS = 320;  // producer, MMA issuer, 8 epilogue warps

template <class C, typename T>
__global__ void __launch_bounds__(WF_THREADS, 1)
    whale_ffn_kernel(const __grid_constant__ CUtensorMap tmHw, const __grid_constant__ CUtensorMap tmA,
                     const __grid_constant__ CUtensorMap tmWF, const __grid_constant__ CUtensorMap tmWU,
                     const __grid_constant__ CUtensorMap tmWD, const __grid_constant__ CUtensorMap tmHf,
                     const float* __restrict__ bF, const float* __restrict__ gamma, const float* __restrict__ beta,
                     int64_t rows, int h, float eps, unsigned* status) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  uint8_t* sC = smem;
  uint8_t* sZn = sC + C::CB;
  uint8_t* sG = sZn + C::ZNB;
  uint8_t* sW = sG + 2 * C::GB;
  uint64_t* bars = reinterpret_cast<uint64_t*>(sW + C::STAGES * C::WS);
  uint64_t* wfull = bars;                   // [STAGES]
  uint64_t* wempty = bars + C::STAGES;      // [STAGES]
  uint64_t* z_full = bars + 2 * C::STAGES;  // [2] Z in TMEM
  uint64_t* o_full = z_full + 2;            // [2] Z + FFN in TMEM
  uint64_t* o_empty = z_full + 4;           // [2] read by the epilogue
  uint64_t* u_full = z_full + 6;            // [2]
  uint64_t* u_empty = z_full + 8;           // [2]
  uint64_t* g_full = z_full + 10;           // [2]
  uint64_t* g_empty = z_full + 12;          // [2]
  uint64_t* c_full = z_full + 14;
  uint64_t* c_empty = z_full + 15;
  uint64_t* zn_full = z_full + 16;
  uint64_t* zn_empty = z_full + 17;
  uint64_t* fin = z_full + 18;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(z_full + 19);
  float* red = reinterpret_cast<float*>(sW + C::STAGES * C::WS + 512);
  float* prm = red + 4 * C::R;  // [3][D]: b_F (or 0), gamma, beta

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    prefetch_tmap(&tmHw);
    prefetch_tmap(&tmA);
    prefetch_tmap(&tmWF);
    prefetch_tmap(&tmWU);
    prefetch_tmap(&tmWD);
    prefetch_tmap(&tmHf);
    for (int s = 0; s < C::STAGES; ++s) {
      mbar_init(&wfull[s], 1);
      mbar_init(&wempty[s], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&z_full[i], 1);
      mbar_init(&o_full[i], 1);
      mbar_init(&o_empty[i], 8);
      mbar_init(&u_full[i], 1);
      mbar_init(&u_empty[i], 8);
      mbar_init(&g_full[i], 8);
      mbar_init(&g_empty[i], 1);
    }
    mbar_init(c_full, 1);
    mbar_init(c_empty, 1);
    mbar_init(zn_full, 8);
    mbar_init(zn_empty, 1);
    mbar_init(fin, 1);
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const int64_t tiles = (rows + C::R - 1) / C::R;
  const int nh = h / C::HC;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      int ws = 0;
      uint32_t wph = 0, tl = 0, cn = 0;
      bool ok = true;
      auto load_w = [&](const CUtensorMap* m, int nbox, int boxb, int x0, int xstep, int y0) -> bool {
        if (!mbar_wait(&wempty[ws], wph ^ 1u, status)) return false;
        mbar_arrive_expect_tx(&wfull[ws], static_cast<uint32_t>(C::WS));
        for (int i = 0; i < nbox; ++i) tma_load_2d(m, &wfull[ws], sW + ws * C::WS + i * boxb, x0 + i * xstep, y0);
        if (++ws == C::STAGES) {
          ws = 0;
          wph ^= 1u;
        }
        return true;
      };
      for (int64_t t = blockIdx.x; ok && t < tiles; t += gridDim.x, ++tl) {
        const int row0 = static_cast<int>(t * C::R);
        if (!mbar_wait(c_empty, (tl & 1u) ^ 1u, status)) {
          ok = false;
          break;
        }
        mbar_arrive_expect_tx(c_full, static_cast<uint32_t>(C::CB));
#pragma unroll
        for (int bx = 0; bx < C::NBOX; ++bx) {
          tma_load_2d(&tmHw, c_full, sC + bx * C::TBOXB, bx * C::BW, row0);
          tma_load_2d(&tmA, c_full, sC + (C::NBOX + bx) * C::TBOXB, bx * C::BW, row0);
        }
        ++cn;
        // weights in the order the MMA warp consumes them
        for (int kc = 0; ok && kc < C::NKC; ++kc) ok = load_w(&tmWF, 64 / C::BW, C::WDBOXB, kc * 64, C::BW, 0);
        for (int c = 0; ok && c < nh; ++c) {
          ok = load_w(&tmWU, C::NBOX, C::WUBOXB, 0, C::BW, c * C::HC);
          if (ok && c > 0) ok = load_w(&tmWD, C::GBOX, C::WDBOXB, (c - 1) * C::HC, C::BW, 0);
        }
        if (ok) ok = load_w(&tmWD, C::GBOX, C::WDBOXB, (nh - 1) * C::HC, C::BW, 0);
      }
      if (!ok) {  // copies already issued must land before the CTA exits
        for (int i = 0; i < C::STAGES; ++i) mbar_drain(&wfull[i], wph ^ (i < ws ? 0u : 1u), status);
        if (cn > 0) mbar_drain(c_full, (cn - 1) & 1u, status);
      }
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------- MMA issuer
    if (lane == 0) {
      const bool bf = Half16<T>::kBF16;
      const uint32_t idZ = idesc_f16kind_f32(C::R, C::D, 0, 0, bf);
      const uint32_t idU = idesc_f16kind_f32(C::R, C::HC, 0, 0, bf);
      int ws = 0;
      uint32_t wph = 0, tl = 0, uc = 0;
      bool ok = true;
      auto wait_w = [&]() -> bool {
        if (!mbar_wait(&wfull[ws], wph, status)) return false;
        tc_fence_after();
        return true;
      };
      auto free_w = [&]() {
        umma_commit(&wempty[ws]);
        if (++ws == C::STAGES) {
          ws = 0;
          wph ^= 1u;
        }
      };
      auto down = [&](uint32_t zc, uint32_t ucc) -> bool {
        const uint32_t gb = ucc & 1u;
        if (!mbar_wait(&g_full[gb], (ucc >> 1) & 1u, status) || !wait_w()) return false;
        const uint32_t ga = smem_u32(sG + gb * C::GB), wa = smem_u32(sW + ws * C::WS);
#pragma unroll
        for (int ks = 0; ks < C::HC / 16; ++ks) {
          const int bx = ks / (C::BW / 16), kin = ks % (C::BW / 16);
          const uint64_t ad = smem_desc(ga + bx * C::TBOXB + kin * 32, 16, 8 * C::SWB, C::SWMODE);
          const uint64_t bd = smem_desc(wa + bx * C::WDBOXB + kin * 32, 16, 8 * C::SWB, C::SWMODE);
          umma_f16kind(tmem + zc, ad, bd, idZ, 1u);  // onto Z: the residual
        }
        free_w();
        umma_commit(&g_empty[gb]);
        return true;
      };
      for (int64_t t = blockIdx.x; ok && t < tiles; t += gridDim.x, ++tl) {
        const uint32_t zb = tl & 1u, zc = zb * C::D;
        if (!mbar_wait(c_full, tl & 1u, status) || !mbar_wait(&o_empty[zb], ((tl >> 1) & 1u) ^ 1u, status)) {
          ok = false;
          break;
        }
        tc_fence_after();
        // Z = [H_w | A] W_F^T
        const uint32_t ca = smem_u32(sC);
        for (int kc = 0; ok && kc < C::NKC; ++kc) {
          if (!wait_w()) {
            ok = false;
            break;
          }
          const uint32_t wa = smem_u32(sW + ws * C::WS);
#pragma unroll
          for (int ks = 0; ks < 4; ++ks) {
            const int col = (kc * 4 + ks) * 16;           // input column of [H_w | A]
            const int part = col / C::D, cp = col % C::D;
            const int bx = cp / C::BW, kin = (cp % C::BW) / 16;
            const uint64_t ad =
                smem_desc(ca + (part * C::NBOX + bx) * C::TBOXB + kin * 32, 16, 8 * C::SWB, C::SWMODE);
            const int lb = (ks * 16) / C::BW, lk = ((ks * 16) % C::BW) / 16;
            const uint64_t bd = smem_desc(wa + lb * C::WDBOXB + lk * 32, 16, 8 * C::SWB, C::SWMODE);
            umma_f16kind(tmem + zc, ad, bd, idZ, (kc | ks) != 0 ? 1u : 0u);
          }
          free_w();
        }
        if (!ok) break;
        umma_commit(c_empty);
        umma_commit(&z_full[zb]);
        if (!mbar_wait(zn_full, tl & 1u, status)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t za = smem_u32(sZn);
        for (int c = 0; ok && c < nh; ++c, ++uc) {
          const uint32_t ub = uc & 1u;
          if (!mbar_wait(&u_empty[ub], ((uc >> 1) & 1u) ^ 1u, status) || !wait_w()) {
            ok = false;
            break;
          }
          const uint32_t wa = smem_u32(sW + ws * C::WS);
#pragma unroll
          for (int ks = 0; ks < C::D / 16; ++ks) {
            const int bx = ks / (C::BW / 16), kin = ks % (C::BW / 16);
            const uint64_t ad = smem_desc(za + bx * C::TBOXB + kin * 32, 16, 8 * C::SWB, C::SWMODE);
            const uint64_t bd = smem_desc(wa + bx * C::WUBOXB + kin * 32, 16, 8 * C::SWB, C::SWMODE);
            umma_f16kind(tmem + C::UCOL + ub * C::HC, ad, bd, idU, ks != 0 ? 1u : 0u);
          }
          free_w();
          umma_commit(&u_full[ub]);
          if (c == nh - 1) umma_commit(zn_empty);
          if (c > 0 && !down(zc, uc - 1u)) ok = false;  // the down projection trails by one chunk
        }
        if (!ok || !down(zc, uc - 1u)) {
          ok = false;
          break;
        }
        umma_commit(&o_full[zb]);
      }
      umma_commit(fin);  // no MMA may still write TMEM when it is freed
      mbar_drain(fin, 0u, status);
    }
  } else {
    // ------------------------------------------------------------ epilogue
    // Two warps per TMEM lane quarter (rows 32 (warp % 4) .. + 31): for Z and the output
    // the 32-column chunks alternate between them (LayerNorm partial sums exchanged through
    // shared memory under a 64-thread named barrier); of each 64-column gated chunk, warp
    // `half` takes columns 32 half .. + 31.
    const int q = warp & 3;
    const int half = (warp - 2) >> 2;
    const int row = q * 32 + lane;
    const uint32_t lane_base = static_cast<uint32_t>(q * 32) << 16;
    const int bar_id = 1 + q;
    const float inv_d = 1.0f / static_cast<float>(C::D);
    const int et = threadIdx.x - 64;           // 0..255 among the epilogue threads
    const bool store_thread = et == 0;         // issues the output tile's TMA stores
    for (int i = et; i < 3 * C::D; i += 256)
      prm[i] = i < C::D ? whale_bias(bF, i) : (i < 2 * C::D ? __ldg(&gamma[i - C::D]) : __ldg(&beta[i - 2 * C::D]));
    named_bar(5, 256);
    const float* pb = prm;                      // b_F
    const float* pg = prm + C::D;               // gamma
    const float* pbeta = prm + 2 * C::D;        // beta
    uint32_t tl = 0, uc = 0;
    bool ok = true;
    for (int64_t t = blockIdx.x; t < tiles; t += gridDim.x, ++tl) {
      const uint32_t zb = tl & 1u, zc = zb * C::D;
      if (ok) ok = mbar_wait(&z_full[zb], (tl >> 1) & 1u, status);
      tc_fence_after();
      // LayerNorm of Z + b_F over d: two passes over TMEM (mean, then centred squares)
      float sum = 0.f;
#pragma unroll 1
      for (int cc = half; cc < C::D / 32; cc += 2) {
        uint32_t r[32];
        tmem_ld32(tmem + lane_base + zc + cc * 32, r);
        tmem_ld_wait();
#pragma unroll
        for (int i = 0; i < 32; ++i) sum += __uint_as_float(r[i]) + pb[cc * 32 + i];
      }
      red[half * C::R + row] = sum;
      named_bar(bar_id, 64);
      const float mean = (sum + red[(half ^ 1) * C::R + row]) * inv_d;
      float sq = 0.f;
#pragma unroll 1
      for (int cc = half; cc < C::D / 32; cc += 2) {
        uint32_t r[32];
        tmem_ld32(tmem + lane_base + zc + cc * 32, r);
        tmem_ld_wait();
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          const float v = __uint_as_float(r[i]) + pb[cc * 32 + i] - mean;
          sq += v * v;
        }
      }
      red[(2 + half) * C::R + row] = sq;
      named_bar(bar_id, 64);
      const float rstd = rsqrtf((sq + red[(2 + (half ^ 1)) * C::R + row]) * inv_d + eps);
      // the previous tile's output, staged in the LN(Z) buffer, has been read by its TMA stores
      if (store_thread) bulk_wait_read<0>();
      named_bar(5, 256);
      if (ok) ok = mbar_wait(zn_empty, (tl & 1u) ^ 1u, status);
      const uint32_t za = smem_u32(sZn);
#pragma unroll 1
      for (int cc = half; cc < C::D / 32; cc += 2) {
        uint32_t r[32];
        tmem_ld32(tmem + lane_base + zc + cc * 32, r);
        tmem_ld_wait();
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          uint32_t p[4];
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const int c0 = cc * 32 + j * 8 + 2 * i;
            const float a = (__uint_as_float(r[j * 8 + 2 * i]) + pb[c0] - mean) * rstd * pg[c0] + pbeta[c0];
            const float b = (__uint_as_float(r[j * 8 + 2 * i + 1]) + pb[c0 + 1] - mean) * rstd * pg[c0 + 1] + pbeta[c0 + 1];
            p[i] = Half16<T>::pack2(a, b);
          }
          const int col = cc * 32 + j * 8;  // first of 8 columns = one 16-byte unit
          const uint32_t a = za + (col / C::BW) * C::TBOXB + whale_swz<C::SWB>(row, (col % C::BW) / 8);
          asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(a), "r"(p[0]), "r"(p[1]), "r"(p[2]),
                       "r"(p[3])
                       : "memory");
        }
      }
      fence_proxy_async_smem();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(zn_full);
      // gated chunks: G = U * SiLU(U) = U^2 / (1 + 2^(-U log2 e)), this warp's 32 columns
      for (int c = 0; c < nh; ++c, ++uc) {
        const uint32_t ub = uc & 1u, up = (uc >> 1) & 1u;
        if (ok) ok = mbar_wait(&u_full[ub], up, status);
        tc_fence_after();
        uint32_t r0[32];
        tmem_ld32(tmem + lane_base + C::UCOL + ub * C::HC + half * 32, r0);
        tmem_ld_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&u_empty[ub]);
        if (ok) ok = mbar_wait(&g_empty[ub], up ^ 1u, status);
        const uint32_t ga = smem_u32(sG + ub * C::GB);
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          uint32_t p[4];
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const float va = __uint_as_float(r0[j * 8 + 2 * i]);
            const float vb = __uint_as_float(r0[j * 8 + 2 * i + 1]);
            p[i] = Half16<T>::pack2(__fdividef(va * va, 1.f + whale_ex2(-1.4426950408889634f * va)),
                                    __fdividef(vb * vb, 1.f + whale_ex2(-1.4426950408889634f * vb)));
          }
          const int col = half * 32 + j * 8;
          const uint32_t a = ga + (col / C::BW) * C::TBOXB + whale_swz<C::SWB>(row, (col % C::BW) / 8);
          asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(a), "r"(p[0]), "r"(p[1]), "r"(p[2]),
                       "r"(p[3])
                       : "memory");
        }
        fence_proxy_async_smem();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&g_full[ub]);
      }
      // H_f = Z + G W_down^T (accumulated in TMEM) + b_F, staged in the LN(Z) buffer (every
      // MMA of the tile has completed) and written with TMA stores (rows past `rows` clipped)
      if (ok) ok = mbar_wait(&o_full[zb], (tl >> 1) & 1u, status);
      tc_fence_after();
#pragma unroll 1
      for (int cc = half; cc < C::D / 32; cc += 2) {
        uint32_t r[32];
        tmem_ld32(tmem + lane_base + zc + cc * 32, r);
        tmem_ld_wait();
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          uint32_t p[4];
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const int c0 = cc * 32 + j * 8 + 2 * i;
            p[i] = Half16<T>::pack2(__uint_as_float(r[j * 8 + 2 * i]) + pb[c0],
                                    __uint_as_float(r[j * 8 + 2 * i + 1]) + pb[c0 + 1]);
          }
          const int col = cc * 32 + j * 8;
          const uint32_t a = za + (col / C::BW) * C::TBOXB + whale_swz<C::SWB>(row, (col % C::BW) / 8);
          asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(a), "r"(p[0]), "r"(p[1]), "r"(p[2]),
                       "r"(p[3])
                       : "memory");
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&o_empty[zb]);
      fence_proxy_async_smem();  // the TMA store reads the staged tile
      named_bar(5, 256);
      if (store_thread && ok) {
#pragma unroll
        for (int bx = 0; bx < C::NBOX; ++bx)
          tma_store_2d(&tmHf, sZn + bx * C::TBOXB, bx * C::BW, static_cast<int32_t>(t * C::R));
        bulk_commit();
      }
    }
    if (store_thread) bulk_wait<0>();  // the stores have completed before the CTA exits
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

}  // namespace wk
