// gemm_tc.cuh -- the batch-wide tensor-core GEMM of the Wukong stack on sm_100a.
//
// Two uses (Wukong page, section 2.2):
// Operands are fp16 or bf16 (both alike), accumulation fp32 in TMEM.
//   MODE_MLP: one Linear of the FMB MLP over the whole batch,
//             C[r, c] = act( sum_q A[r, q] W[c, q] + bias[c] ), A [M, K], W [N, K],
//             both K-major; C has row stride ldc (the last Linear writes the FMB
//             rows of the concat buffer directly).
//   MODE_LCB: the Linear Compress Block, W_L shared by every example,
//             concat[b, n_f + r, t] = sum_i W_L[r, i] X[b, i, t]; A = W_L (K-major),
//             B = X_b seen as an (i x t) MN-major operand, E = floor(256/d)
//             examples side by side in one 128 x (E d) tile.
//
// Design (one CTA per SM, persistent over output tiles, 192 threads):
//   warp 0      TMA producer: fills a STAGES-deep ring of (A 128x64, B up to 256x64)
//               16-bit tiles, 128B-swizzled (B of the LCB: 64B-swizzled 32-wide
//               column blocks), completion tracked by mbarrier transaction counts;
//   warp 1      allocates 512 TMEM columns (two 128x256 fp32 accumulators) and one
//               thread issues tcgen05.mma (M=128, N<=256, K=16) over each stage,
//               releasing the stage with tcgen05.commit;
//   warps 2..5  epilogue: tcgen05.ld of their 32-lane quarter, bias (+ReLU),
//               conversion, swizzled staging in shared memory and TMA stores;
//               the second accumulator lets the epilogue of tile t overlap the
//               main loop of tile t+1.
// Every mbarrier wait is bounded (common.cuh); on a timeout each role stops,
// the CTA drains and frees TMEM, and the status word carries the flag.
#pragma once

#include "common.cuh"
#include "res_ln.cuh"

namespace wk {

enum { MODE_MLP = 0, MODE_LCB = 1 };

// 4-D tiled TMA load (the LCB's X operand: 32 columns x 64 rows x d/32 column chunks x E
// examples in one copy, landing as E * d/32 consecutive 64-row blocks of 32 columns).
__device__ __forceinline__ void tma_load_4d(const CUtensorMap* m, uint64_t* bar, void* dst, int32_t c0, int32_t c1,
                                            int32_t c2, int32_t c3) {
  asm volatile(
      "cp.async.bulk.tensor.4d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4, %5, %6}], "
      "[%2];" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(m)), "r"(smem_u32(bar)), "r"(c0), "r"(c1), "r"(c2), "r"(c3)
      : "memory");
}

constexpr int GEMM_BM = 128;
constexpr int GEMM_BN = 256;
constexpr int GEMM_BK = 64;
constexpr int GEMM_STAGES = 4;
constexpr int GEMM_THREADS = 192;
constexpr uint32_t GEMM_A_STAGE = GEMM_BM * GEMM_BK * 2;   // 16 KB
constexpr uint32_t GEMM_B_STAGE = GEMM_BN * GEMM_BK * 2;   // 32 KB
constexpr uint32_t GEMM_TMEM_COLS = 512;                   // 2 accumulators x 256 columns

template <typename TO>
constexpr uint32_t gemm_epi_buf_bytes() { return 32u * 32u * static_cast<uint32_t>(sizeof(TO)); }

template <typename TO>
constexpr uint32_t gemm_smem_bytes() {
  return 1024u /* alignment slack */ + GEMM_STAGES * (GEMM_A_STAGE + GEMM_B_STAGE) +
         4u * 2u * gemm_epi_buf_bytes<TO>() + 256u /* barriers + tmem slot */;
}

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

struct GemmParams {
  int M, N, K;           // MLP: C is M x N, reduction K.  LCB: M = n_l, N = batch, K = n.
  int num_m_tiles;       // ceil(M / 128)
  int num_n_tiles;       // MLP: ceil(N / 256); LCB: number of example groups ceil(batch / E)
  int num_tiles;
  int num_kb;            // ceil(K / 64)
  int group_m;           // MLP raster: consecutive tiles walk group_m M-tiles first
  int mma_n;             // N of each tcgen05.mma (256 for MLP, E*d for LCB)
  const float* bias;     // MLP, may be null
  int relu;              // MLP
  int d, E, dchunks;     // LCB: embedding dim, examples per tile, d / 32
  unsigned* status;
  // MLP: 1 = the epilogue adds C into what the output already holds (TMA reduce-add)
  // instead of overwriting it
  int reduce_out;
};

__device__ __forceinline__ void gemm_tile_coords(const GemmParams& p, int tile, int mode, int& mt, int& nt) {
  if (mode == MODE_LCB) {  // W_L tiles fastest: an example group's X stays in L2 for all of them
    mt = tile % p.num_m_tiles;
    nt = tile / p.num_m_tiles;
    return;
  }
  const int group = p.group_m * p.num_n_tiles;
  const int g = tile / group;
  const int first_m = g * p.group_m;
  int gm = p.num_m_tiles - first_m;
  if (gm > p.group_m) gm = p.group_m;
  const int local = tile - g * group;
  mt = first_m + local % gm;
  nt = local / gm;
}

// T: operand type (__half or __nv_bfloat16, A and B alike); TO: output type.
template <int MODE, typename T, typename TO>
__global__ void __launch_bounds__(GEMM_THREADS, 1)
    gemm_tc_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                   const __grid_constant__ CUtensorMap tmC, const GemmParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  uint8_t* sA = smem;
  uint8_t* sB = sA + GEMM_STAGES * GEMM_A_STAGE;
  uint8_t* sEpi = sB + GEMM_STAGES * GEMM_B_STAGE;
  constexpr uint32_t EPI_BUF = gemm_epi_buf_bytes<TO>();
  uint64_t* bars = reinterpret_cast<uint64_t*>(sEpi + 8 * EPI_BUF);
  uint64_t* full = bars;                       // [STAGES] TMA -> MMA
  uint64_t* empty = bars + GEMM_STAGES;        // [STAGES] MMA -> TMA
  uint64_t* tfull = bars + 2 * GEMM_STAGES;    // [2] MMA -> epilogue
  uint64_t* tempty = bars + 2 * GEMM_STAGES + 2;  // [2] epilogue -> MMA
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 2 * GEMM_STAGES + 4);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    prefetch_tmap(&tmA);
    prefetch_tmap(&tmB);
    prefetch_tmap(&tmC);
    for (int s = 0; s < GEMM_STAGES; ++s) {
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
    tmem_alloc(tmem_slot, GEMM_TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  const uint32_t b_stage_bytes =
      (MODE == MODE_MLP) ? GEMM_B_STAGE : static_cast<uint32_t>(p.E * p.dchunks) * 4096u;
  const uint32_t stage_tx = GEMM_A_STAGE + b_stage_bytes;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      int s = 0;
      uint32_t ph = 0;
      bool ok = true;
      for (int tile = blockIdx.x; ok && tile < p.num_tiles; tile += gridDim.x) {
        int mt, nt;
        gemm_tile_coords(p, tile, MODE, mt, nt);
        for (int kb = 0; kb < p.num_kb; ++kb) {
          if (!mbar_wait(&empty[s], ph ^ 1u, p.status)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&full[s], stage_tx);
          tma_load_2d(&tmA, &full[s], sA + s * GEMM_A_STAGE, kb * GEMM_BK, mt * GEMM_BM);
          if (MODE == MODE_MLP) {
            tma_load_2d(&tmB, &full[s], sB + s * GEMM_B_STAGE, kb * GEMM_BK, nt * GEMM_BN);
          } else {
            // the E examples' 64-row K slices, every 32-column chunk, in one copy
            tma_load_4d(&tmB, &full[s], sB + s * GEMM_B_STAGE, 0, kb * GEMM_BK, 0, nt * p.E);
          }
          if (++s == GEMM_STAGES) {
            s = 0;
            ph ^= 1u;
          }
        }
      }
      // Drain after a failed wait: every stage this thread armed must land before
      // the CTA exits. Slots below s were last armed in the current round (parity
      // ph), the others in the previous one (parity ph ^ 1, already complete if
      // never armed); the waits are bounded.
      if (!ok) {
        for (int i = 0; i < GEMM_STAGES; ++i) mbar_wait(&full[i], ph ^ (i < s ? 0u : 1u), nullptr);
      }
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------- MMA issuer
    if (lane == 0) {
      const uint32_t idesc = idesc_f16kind_f32(GEMM_BM, p.mma_n, 0, MODE == MODE_LCB ? 1 : 0, Half16<T>::kBF16);
      int s = 0;
      uint32_t ph = 0;
      int acc = 0;
      uint32_t acc_ph = 0;
      bool ok = true;
      bool issued = false;
      for (int tile = blockIdx.x; ok && tile < p.num_tiles; tile += gridDim.x) {
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
          const uint32_t a_addr = smem_u32(sA + s * GEMM_A_STAGE);
          const uint32_t b_addr = smem_u32(sB + s * GEMM_B_STAGE);
#pragma unroll
          for (int kk = 0; kk < GEMM_BK / 16; ++kk) {
            const uint64_t adesc = smem_desc(a_addr + kk * 32, 16, 1024, 2);
            uint64_t bdesc;
            if (MODE == MODE_MLP)
              bdesc = smem_desc(b_addr + kk * 32, 16, 1024, 2);
            else  // MN-major, 64B swizzle: 32-wide column blocks 4 KB apart, 8-row K groups 512 B apart
              bdesc = smem_desc(b_addr + kk * 1024, 4096, 512, 4);
            umma_f16kind(d_tmem, adesc, bdesc, idesc, (kb | kk) != 0 ? 1u : 0u);
          }
          umma_commit(&empty[s]);
          issued = true;
          if (++s == GEMM_STAGES) {
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
    for (int tile = blockIdx.x; tile < p.num_tiles; tile += gridDim.x) {
      int mt, nt;
      gemm_tile_coords(p, tile, MODE, mt, nt);
      if (!mbar_wait(&tfull[acc], acc_ph, p.status)) break;
      tc_fence_after();
      const int nchunks = (MODE == MODE_MLP) ? GEMM_BN / 32 : p.E * p.dchunks;
      for (int c = 0; c < nchunks; ++c) {
        int col0 = 0;
        if (MODE == MODE_MLP) {
          col0 = nt * GEMM_BN + c * 32;
          if (col0 >= p.N) break;
        } else if (nt * p.E + c / p.dchunks >= p.N) {  // LCB: p.N is the batch size
          break;
        }
        uint32_t r[32];
        tmem_ld32(tmem_base + (static_cast<uint32_t>(q * 32) << 16) + static_cast<uint32_t>(acc * GEMM_BN + c * 32),
                  r);
        tmem_ld_wait();
        float v[32];
#pragma unroll
        for (int j = 0; j < 32; ++j) v[j] = __uint_as_float(r[j]);
        if (MODE == MODE_MLP) {
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
        }
        uint8_t* sb = bufs + buf * EPI_BUF;
        if (lane == 0) bulk_wait_read<1>();  // the store that last used this buffer has read it
        __syncwarp();
        stage_row<TO>(sb, lane, v);
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
          if (MODE == MODE_MLP) {
            if (p.reduce_out)
              tma_reduce_add_2d(&tmC, sb, col0, mt * GEMM_BM + q * 32);
            else
              tma_store_2d(&tmC, sb, col0, mt * GEMM_BM + q * 32);
          } else {
            const int e = c / p.dchunks;
            const int tc = c - e * p.dchunks;
            tma_store_3d(&tmC, sb, tc * 32, mt * GEMM_BM + q * 32, nt * p.E + e);
          }
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
