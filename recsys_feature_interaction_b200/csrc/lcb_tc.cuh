// lcb_tc.cuh -- the Linear Compress Block of a Wukong layer with W_L resident in
// shared memory (Wukong page, section 2.2, LCB paragraph: a weight matrix W_L,
// shared by every example, linearly recombines the layer's n embeddings into n_L):
//
//   concat[b, n_f + r, t] = sum_i W_L[r, i] X[b, i, t],   r < n_l, i < n, t < d
//
// W_L is tiny next to the batch (256 x 512 for the 8-layer workload) but a GEMM that
// streams it with every output tile moves it from L2 once per tile, more bytes than
// X itself. Here each CTA owns one 128-row tile of W_L for the whole kernel: it
// loads that tile's K panel once (ceil(n/64) boxes of 128 x 64, 128B swizzle, at
// most 8 = 128 KB) and afterwards only X streams through the ring. CTAs are assigned
// m tiles round-robin (the grid is a multiple of the m-tile count), so the CTAs that
// need the same example's X run side by side and share it through L2.
//
// Warp roles as in gemm_tc.cuh (192 threads): warp 0 TMA producer (X as an MN-major
// operand, one 4-D box per K step: 32 columns x 64 rows x d/32 chunks x E examples, 64B
// swizzle), warp 1
// TMEM allocation + the single MMA-issuing thread (tcgen05.mma M = 128, N = E*d,
// K = 16; two TMEM accumulators), warps 2..5 the epilogue (tcgen05.ld, 16-bit pack,
// 3-D TMA store into the concat rows). Every wait is bounded.
#pragma once

#include "common.cuh"
#include "gemm_tc.cuh"

namespace wk {

constexpr int LCB_MAX_KB = 8;                     // n <= 512: resident panel <= 128 KB
constexpr int LCB_MAX_STAGES = 8;
constexpr uint32_t LCB_SMEM_BUDGET = 227u * 1024u;

// Shared memory of the resident-W_L LCB for a given K panel and X stage size.
template <typename TO>
constexpr uint32_t lcb_tc_fixed_bytes(int num_kb) {
  return 1024u + static_cast<uint32_t>(num_kb) * GEMM_A_STAGE + 4u * 2u * gemm_epi_buf_bytes<TO>() + 512u;
}

template <typename TO>
inline int lcb_tc_stages(int num_kb, uint32_t b_stage) {
  const uint32_t fixed = lcb_tc_fixed_bytes<TO>(num_kb);
  if (fixed >= LCB_SMEM_BUDGET) return 0;
  const int s = static_cast<int>((LCB_SMEM_BUDGET - fixed) / b_stage);
  return s > LCB_MAX_STAGES ? LCB_MAX_STAGES : s;
}

// p: as for gemm_tc_kernel<MODE_LCB> (M = n_l, N = batch, K = n, E, d, dchunks,
// mma_n = E*d, num_m_tiles, num_n_tiles = example groups, num_kb <= LCB_MAX_KB);
// stages: X ring depth (2..LCB_MAX_STAGES); gridDim.x a multiple of num_m_tiles.
template <typename T, typename TO>
__global__ void __launch_bounds__(GEMM_THREADS, 1)
    lcb_tc_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                  const __grid_constant__ CUtensorMap tmC, const GemmParams p, int stages) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  const uint32_t b_stage = static_cast<uint32_t>(p.E * p.dchunks) * 4096u;
  uint8_t* sA = smem;                                   // resident W_L panel
  uint8_t* sB = sA + p.num_kb * GEMM_A_STAGE;           // X ring
  uint8_t* sEpi = sB + stages * b_stage;
  constexpr uint32_t EPI_BUF = gemm_epi_buf_bytes<TO>();
  uint64_t* bars = reinterpret_cast<uint64_t*>(sEpi + 8 * EPI_BUF);
  uint64_t* full = bars;                                // [LCB_MAX_STAGES] TMA -> MMA
  uint64_t* empty = bars + LCB_MAX_STAGES;              // [LCB_MAX_STAGES] MMA -> TMA
  uint64_t* tfull = bars + 2 * LCB_MAX_STAGES;          // [2] MMA -> epilogue
  uint64_t* tempty = tfull + 2;                         // [2] epilogue -> MMA
  uint64_t* afull = tfull + 4;                          // the resident panel has landed
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(tfull + 5);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int mt = blockIdx.x % p.num_m_tiles;            // this CTA's W_L tile
  const int nt0 = blockIdx.x / p.num_m_tiles;
  const int nstep = gridDim.x / p.num_m_tiles;

  if (threadIdx.x == 0) {
    prefetch_tmap(&tmA);
    prefetch_tmap(&tmB);
    prefetch_tmap(&tmC);
    for (int s = 0; s < stages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&tfull[a], 1);
      mbar_init(&tempty[a], 4);
    }
    mbar_init(afull, 1);
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, GEMM_TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      mbar_arrive_expect_tx(afull, static_cast<uint32_t>(p.num_kb) * GEMM_A_STAGE);
      for (int kb = 0; kb < p.num_kb; ++kb)
        tma_load_2d(&tmA, afull, sA + kb * GEMM_A_STAGE, kb * GEMM_BK, mt * GEMM_BM);
      int s = 0;
      uint32_t ph = 0;
      bool ok = true;
      for (int nt = nt0; ok && nt < p.num_n_tiles; nt += nstep) {
        for (int kb = 0; kb < p.num_kb; ++kb) {
          if (!mbar_wait(&empty[s], ph ^ 1u, p.status)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&full[s], b_stage);
          // the E examples' 64-row K slices, every 32-column chunk, in one copy
          tma_load_4d(&tmB, &full[s], sB + s * b_stage, 0, kb * GEMM_BK, 0, nt * p.E);
          if (++s == stages) {
            s = 0;
            ph ^= 1u;
          }
        }
      }
      // Every copy this thread issued lands before the CTA exits (the MMA thread has
      // normally consumed them all already; after a failed wait it may not have).
      mbar_drain(afull, 0u, p.status);
      if (!ok)
        for (int i = 0; i < stages; ++i) mbar_drain(&full[i], ph ^ (i < s ? 0u : 1u), p.status);
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------- MMA issuer
    if (lane == 0) {
      const uint32_t idesc = idesc_f16kind_f32(GEMM_BM, p.mma_n, 0, 1, Half16<T>::kBF16);
      int s = 0;
      uint32_t ph = 0;
      int acc = 0;
      uint32_t acc_ph = 0;
      bool ok = mbar_wait(afull, 0u, p.status);
      tc_fence_after();
      bool issued = false;
      const uint32_t a_base = smem_u32(sA);
      for (int nt = nt0; ok && nt < p.num_n_tiles; nt += nstep) {
        if (!mbar_wait(&tempty[acc], acc_ph ^ 1u, p.status)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(acc * GEMM_BN);
        for (int kb = 0; kb < p.num_kb; ++kb) {
          if (!mbar_wait(&full[s], ph, p.status)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a_addr = a_base + kb * GEMM_A_STAGE;
          const uint32_t b_addr = smem_u32(sB + s * b_stage);
#pragma unroll
          for (int kk = 0; kk < GEMM_BK / 16; ++kk) {
            const uint64_t adesc = smem_desc(a_addr + kk * 32, 16, 1024, 2);
            // MN-major, 64B swizzle: 32-wide column blocks 4 KB apart, 8-row K groups 512 B apart
            const uint64_t bdesc = smem_desc(b_addr + kk * 1024, 4096, 512, 4);
            umma_f16kind(d_tmem, adesc, bdesc, idesc, (kb | kk) != 0 ? 1u : 0u);
          }
          umma_commit(&empty[s]);
          issued = true;
          if (++s == stages) {
            s = 0;
            ph ^= 1u;
          }
        }
        if (!ok) break;
        umma_commit(&tfull[acc]);
        if (++acc == 2) {
          acc = 0;
          acc_ph ^= 1u;
        }
      }
      if (!ok && issued) {
        // make sure no MMA is still writing TMEM before it is freed
        umma_commit(&tfull[acc]);
        mbar_wait(&tfull[acc], acc_ph, nullptr);
      }
    }
  } else {
    // ------------------------------------------------------------ epilogue
    const int q = warp & 3;  // TMEM lane quarter this warp may access
    uint8_t* bufs = sEpi + (warp - 2) * 2 * EPI_BUF;
    int acc = 0;
    uint32_t acc_ph = 0;
    int buf = 0;
    const int nchunks = p.E * p.dchunks;
    for (int nt = nt0; nt < p.num_n_tiles; nt += nstep) {
      if (!mbar_wait(&tfull[acc], acc_ph, p.status)) break;
      tc_fence_after();
      for (int c = 0; c < nchunks; ++c) {
        const int e = c / p.dchunks;
        if (nt * p.E + e >= p.N) break;  // p.N is the batch size
        uint32_t r[32];
        tmem_ld32(tmem_base + (static_cast<uint32_t>(q * 32) << 16) + static_cast<uint32_t>(acc * GEMM_BN + c * 32),
                  r);
        tmem_ld_wait();
        float v[32];
#pragma unroll
        for (int j = 0; j < 32; ++j) v[j] = __uint_as_float(r[j]);
        uint8_t* sb = bufs + buf * EPI_BUF;
        if (lane == 0) bulk_wait_read<1>();  // the store that last used this buffer has read it
        __syncwarp();
        stage_row<TO>(sb, lane, v);
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
          tma_store_3d(&tmC, sb, (c - e * p.dchunks) * 32, mt * GEMM_BM + q * 32, nt * p.E + e);
          bulk_commit();
        }
        buf ^= 1;
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&tempty[acc]);
      if (++acc == 2) {
        acc = 0;
        acc_ph ^= 1u;
      }
    }
    if (lane == 0) bulk_wait<0>();
    __syncwarp();
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, GEMM_TMEM_COLS);
  }
}

}  // namespace wk
