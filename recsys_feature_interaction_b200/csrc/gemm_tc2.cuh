// gemm_tc2.cuh -- the FMB MLP Linear on CTA pairs (tcgen05 cta_group::2).
//
//   C[r, c] = act( sum_q A[r, q] W[c, q] + bias[c] )   (one Linear of the FMB MLP,
//   Wukong page, section 2.2), A [M, K] and W [N, K] K-major, C row stride ldc.
//
// A cluster of two CTAs (one TPC) owns a 256 x 256 output tile. Each CTA loads its
// 128 rows of A and its 128 rows (half of N) of W into its own shared memory; the
// leader CTA issues tcgen05.mma with M = 256, which reads both CTAs' halves and
// writes each CTA's 128 accumulator rows into that CTA's TMEM. Compared with one
// CTA per 128 x 256 tile, every CTA moves half the B bytes per FLOP (64 instead of
// 96 shared-memory bytes per clock at full rate) and the pair reads each W panel
// once for 256 rows.
//
// Per CTA (192 threads): warp 0 TMA producer, warp 1 TMEM allocator (both CTAs)
// and MMA issuer (leader), warps 2..5 epilogue (as in gemm_tc.cuh). Barriers:
//   full[s]   leader only; the leader arms it for both CTAs' bytes, the peer's
//             TMA loads complete on it through its cluster address;
//   empty[s]  in both CTAs; the leader's commit arrives on each (two commits);
//   tfull[a]  in both CTAs; the leader's commit arrives on each at tile end;
//   tempty[a] leader only; 4 local + 4 remote epilogue-warp arrivals.
// Every mbarrier wait is bounded; both CTAs always reach the final cluster barrier.
#pragma once

#include "gemm_tc.cuh"

namespace wk {

constexpr int GEMM2_BM = 256;  // rows per pair (128 per CTA)
constexpr int GEMM2_BN = 256;
constexpr int GEMM2_BK = 64;
constexpr int GEMM2_STAGES = 6;
constexpr int GEMM2_GROUP_M = 8;  // M tiles per raster group (tiles walk M fastest inside a group)
constexpr uint32_t GEMM2_A_STAGE = 128 * GEMM2_BK * 2;  // 16 KB: this CTA's 128 rows
constexpr uint32_t GEMM2_B_STAGE = 128 * GEMM2_BK * 2;  // 16 KB: this CTA's half of N

// Two launch shapes of the same kernel:
//   persistent (STREAM = false): one pair per two SMs walks tiles pair, pair + pairs, ...
//     with a 6-stage ring, two TMEM accumulators (the epilogue of tile t overlaps the
//     main loop of tile t + 1) and double-buffered epilogue staging;
//   streaming (STREAM = true): one pair per output tile, a 3-stage ring, one
//     accumulator (256 TMEM columns) and single epilogue buffers, so that two pairs'
//     CTAs share each SM (105 KB of shared memory each): the epilogue of one overlaps
//     the main loop of the other, and the hardware block scheduler keeps the tiles in
//     flight consecutive in raster order, which keeps their operand panels in L2.
template <bool STREAM>
struct Gemm2Shape {
  static constexpr int STAGES = STREAM ? 3 : GEMM2_STAGES;
  static constexpr int NACC = STREAM ? 1 : 2;
  static constexpr int NBUF = STREAM ? 1 : 2;
  static constexpr uint32_t TMEM_COLS = STREAM ? 256u : 512u;
};

template <typename TO, bool STREAM = false>
constexpr uint32_t gemm2_smem_bytes() {
  using S = Gemm2Shape<STREAM>;
  return 1024u + S::STAGES * (GEMM2_A_STAGE + GEMM2_B_STAGE) + 4u * S::NBUF * gemm_epi_buf_bytes<TO>() + 256u;
}

__device__ __forceinline__ void gemm2_tile_coords(const GemmParams& p, int tile, int& mt, int& nt) {
  const int group = p.group_m * p.num_n_tiles;
  const int g = tile / group;
  const int first_m = g * p.group_m;
  int gm = p.num_m_tiles - first_m;
  if (gm > p.group_m) gm = p.group_m;
  const int local = tile - g * group;
  mt = first_m + local % gm;
  nt = local / gm;
}

// p.num_m_tiles counts 256-row tiles, p.num_n_tiles tiles of p.mma_n = 256 columns.
//
// A_MN / B_MN: the operand is stored MN-major, as A^T [K, M] (W^T [K, N]) row-major with the
// tensor map's dims (M, K) (N, K): each CTA's 128 rows then arrive as two 64-row x 64-k boxes
// (128-byte swizzle) 8 KB apart and are read MN-major (the backward's weight gradients
// dz^T h and input gradients dz W need no transposed copies).
template <typename T, typename TO, bool STREAM = false, bool A_MN = false, bool B_MN = false>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(GEMM_THREADS, 1)
    gemm_tc2_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                    const __grid_constant__ CUtensorMap tmC, const GemmParams p) {
  using S = Gemm2Shape<STREAM>;
  constexpr int GEMM2_STAGES = S::STAGES;  // shadows the persistent default
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  uint8_t* sA = smem;
  uint8_t* sB = sA + GEMM2_STAGES * GEMM2_A_STAGE;
  uint8_t* sEpi = sB + GEMM2_STAGES * GEMM2_B_STAGE;
  constexpr uint32_t EPI_BUF = gemm_epi_buf_bytes<TO>();
  uint64_t* bars = reinterpret_cast<uint64_t*>(sEpi + 4 * S::NBUF * EPI_BUF);
  uint64_t* full = bars;                                // [STAGES]
  uint64_t* empty = bars + GEMM2_STAGES;                // [STAGES]
  uint64_t* tfull = bars + 2 * GEMM2_STAGES;            // [2]
  uint64_t* tempty = bars + 2 * GEMM2_STAGES + 2;       // [2]
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 2 * GEMM2_STAGES + 4);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();  // 0 = leader
  const int pair = blockIdx.x >> 1;
  const int num_pairs = gridDim.x >> 1;

  if (threadIdx.x == 0) {
    prefetch_tmap(&tmA);
    prefetch_tmap(&tmB);
    prefetch_tmap(&tmC);
    for (int s = 0; s < GEMM2_STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&tfull[a], 1);
      mbar_init(&tempty[a], 8);
    }
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc_pair(tmem_slot, S::TMEM_COLS);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync_all();  // the peer's barriers exist before any remote signal
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      const uint32_t full0 = mapa_shared(smem_u32(full), 0);  // leader's full[0]
      int s = 0;
      uint32_t ph = 0;
      bool ok = true;
      for (int tile = pair; ok && tile < p.num_tiles; tile += num_pairs) {
        int mt, nt;
        gemm2_tile_coords(p, tile, mt, nt);
        const int arow = mt * GEMM2_BM + static_cast<int>(rank) * 128;
        const int brow = nt * p.mma_n + static_cast<int>(rank) * (p.mma_n / 2);
        for (int kb = 0; kb < p.num_kb; ++kb) {
          if (!mbar_wait(&empty[s], ph ^ 1u, p.status)) {
            ok = false;
            break;
          }
          if (rank == 0) mbar_arrive_expect_tx(&full[s], 2u * (GEMM2_A_STAGE + static_cast<uint32_t>(p.mma_n / 2) * 128u));
          const uint32_t fbar = full0 + static_cast<uint32_t>(s) * 8u;
          if constexpr (A_MN) {
#pragma unroll
            for (int j = 0; j < 2; ++j)
              tma_load_2d_pair(&tmA, fbar, sA + s * GEMM2_A_STAGE + j * 8192, arow + 64 * j, kb * GEMM2_BK);
          } else {
            tma_load_2d_pair(&tmA, fbar, sA + s * GEMM2_A_STAGE, kb * GEMM2_BK, arow);
          }
          if constexpr (B_MN) {
#pragma unroll
            for (int j = 0; j < 2; ++j)
              tma_load_2d_pair(&tmB, fbar, sB + s * GEMM2_B_STAGE + j * 8192, brow + 64 * j, kb * GEMM2_BK);
          } else {
            tma_load_2d_pair(&tmB, fbar, sB + s * GEMM2_B_STAGE, kb * GEMM2_BK, brow);
          }
          if (++s == GEMM2_STAGES) {
            s = 0;
            ph ^= 1u;
          }
        }
      }
      if (!ok && rank == 0) {  // bytes still owed to the leader's full barriers land before exit
        for (int i = 0; i < GEMM2_STAGES; ++i) mbar_wait(&full[i], ph ^ (i < s ? 0u : 1u), nullptr);
      }
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------- MMA issuer
    if (lane == 0 && rank == 0) {
      const uint32_t idesc = idesc_f16kind_f32(GEMM2_BM, p.mma_n, A_MN ? 1 : 0, B_MN ? 1 : 0, Half16<T>::kBF16);
      const uint32_t empty_own = smem_u32(empty), empty_peer = mapa_shared(smem_u32(empty), 1);
      const uint32_t tfull_own = smem_u32(tfull), tfull_peer = mapa_shared(smem_u32(tfull), 1);
      int s = 0;
      uint32_t ph = 0;
      int acc = 0;
      uint32_t acc_ph = 0;
      bool ok = true;
      bool issued = false;
      for (int tile = pair; ok && tile < p.num_tiles; tile += num_pairs) {
        if (!mbar_wait(&tempty[acc], acc_ph ^ 1u, p.status)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(acc * GEMM2_BN);
        for (int kb = 0; kb < p.num_kb; ++kb) {
          if (!mbar_wait(&full[s], ph, p.status)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a_addr = smem_u32(sA + s * GEMM2_A_STAGE);
          const uint32_t b_addr = smem_u32(sB + s * GEMM2_B_STAGE);
#pragma unroll
          for (int kk = 0; kk < GEMM2_BK / 16; ++kk) {
            // K-major: the 16-k slice 32 bytes into each 128-byte row; MN-major: 16 k rows
            // (2048 bytes) on, 64-row boxes 8 KB apart, 8-row k groups 1 KB apart
            const uint64_t ad = A_MN ? smem_desc(a_addr + kk * 2048, 8192, 1024, 2) : smem_desc(a_addr + kk * 32, 16, 1024, 2);
            const uint64_t bd = B_MN ? smem_desc(b_addr + kk * 2048, 8192, 1024, 2) : smem_desc(b_addr + kk * 32, 16, 1024, 2);
            umma_f16kind_pair(d_tmem, ad, bd, idesc, (kb | kk) != 0 ? 1u : 0u);
          }
          umma_commit_pair(empty_own + static_cast<uint32_t>(s) * 8u);
          umma_commit_pair(empty_peer + static_cast<uint32_t>(s) * 8u);
          issued = true;
          if (++s == GEMM2_STAGES) {
            s = 0;
            ph ^= 1u;
          }
        }
        if (!ok) break;
        umma_commit_pair(tfull_own + static_cast<uint32_t>(acc) * 8u);
        umma_commit_pair(tfull_peer + static_cast<uint32_t>(acc) * 8u);
        if (++acc == S::NACC) {
          acc = 0;
          acc_ph ^= 1u;
        }
      }
      if (!ok && issued) {  // no MMA may still write TMEM when it is freed
        umma_commit_pair(tfull_own + static_cast<uint32_t>(acc) * 8u);
        mbar_wait(&tfull[acc], acc_ph, nullptr);
      }
    }
  } else {
    // ------------------------------------------------------------ epilogue
    const int q = warp & 3;
    uint8_t* bufs = sEpi + (warp - 2) * S::NBUF * EPI_BUF;
    const uint32_t tempty0 = mapa_shared(smem_u32(tempty), 0);  // leader's tempty[0]
    int acc = 0;
    uint32_t acc_ph = 0;
    int buf = 0;
    for (int tile = pair; tile < p.num_tiles; tile += num_pairs) {
      int mt, nt;
      gemm2_tile_coords(p, tile, mt, nt);
      if (!mbar_wait(&tfull[acc], acc_ph, p.status)) break;
      tc_fence_after();
      const int row0 = mt * GEMM2_BM + static_cast<int>(rank) * 128 + q * 32;
      for (int c = 0; c < GEMM2_BN / 32; ++c) {
        const int col0 = nt * GEMM2_BN + c * 32;
        if (col0 >= p.N) break;
        uint32_t r[32];
        tmem_ld32(tmem_base + (static_cast<uint32_t>(q * 32) << 16) + static_cast<uint32_t>(acc * GEMM2_BN + c * 32), r);
        tmem_ld_wait();
        float v[32];
#pragma unroll
        for (int j = 0; j < 32; ++j) v[j] = __uint_as_float(r[j]);
        if (p.bias) {
          if (col0 + 32 <= p.N) {
#pragma unroll
            for (int j = 0; j < 32; j += 4) {
              const float4 b4 = __ldg(reinterpret_cast<const float4*>(p.bias + col0 + j));
              v[j] += b4.x;
              v[j + 1] += b4.y;
              v[j + 2] += b4.z;
              v[j + 3] += b4.w;
            }
          } else {
#pragma unroll
            for (int j = 0; j < 32; ++j)
              if (col0 + j < p.N) v[j] += __ldg(p.bias + col0 + j);
          }
        }
        if (p.relu) {
#pragma unroll
          for (int j = 0; j < 32; ++j) v[j] = fmaxf(v[j], 0.f);
        }
        uint8_t* sb = bufs + buf * EPI_BUF;
        if (lane == 0) {
          if constexpr (S::NBUF == 2) bulk_wait_read<1>();
          else bulk_wait_read<0>();
        }
        __syncwarp();
        stage_row<TO>(sb, lane, v);
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
          if (p.reduce_out)
            tma_reduce_add_2d(&tmC, sb, col0, row0);
          else
            tma_store_2d(&tmC, sb, col0, row0);
          bulk_commit();
        }
        if constexpr (S::NBUF == 2) buf ^= 1;
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(tempty0 + static_cast<uint32_t>(acc) * 8u);
      if (++acc == S::NACC) {
        acc = 0;
        acc_ph ^= 1u;
      }
    }
    if (lane == 0) bulk_wait<0>();
    __syncwarp();
  }

  tc_fence_before();
  __syncthreads();
  cluster_sync_all();  // no remote signal or MMA of the pair is still in flight
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tmem_base, S::TMEM_COLS);
  }
}

}  // namespace wk
