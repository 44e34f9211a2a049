// wk_api.cu -- the C ABI of the Wukong interaction-stack forward (include/wukong.h):
// argument validation, workspace, weight conversion, TMA descriptors, launch order
// and the host-buffer pipeline. Every kernel it launches lives in the .cuh files
// next to it; there is no host fallback: without a CUDA device every call that
// would launch returns WK_ERR_CUDA.
//
// Layer order on the stream (Wukong page, section 2.2; per layer i):
//   1. FM + LayerNorm      X_i -> A0                          (fm_tc.cuh / simt.cuh)
//   2. MLP Linears         A0 -> ... -> concat rows 0..n_F-1   (gemm_tc.cuh, MODE_MLP)
//   3. LCB                 X_i -> concat rows n_F..n-1         (gemm_tc.cuh, MODE_LCB)
//   4. residual + LN       concat + X_i -> X_{i+1}             (res_ln.cuh)
// A 16-bit stack computes with 16-bit tensor-core operands T (fp16 by default,
// bf16 on request) and fp32 accumulation; every intermediate buffer holds T. A
// bf16 stack's weights are converted to T once, at create, and its input once per
// forward. The stack output is written in the caller's type.
#include <cudaTypedefs.h>

#include <algorithm>
#include <cmath>
#include <cstdlib>
#include <cstring>
#include <mutex>
#include <new>
#include <set>
#include <type_traits>
#include <utility>
#include <vector>

#include "wukong.h"
#include "common.cuh"
#include "convert.cuh"
#include "fm_tc.cuh"
#include "front_tc.cuh"
#include "gemm_tc.cuh"
#include "gemm_tc2.cuh"
#include "head.cuh"
#include "lcb_tc.cuh"
#include "moe.cuh"
#include "res_ln.cuh"
#include "res_ln_ring.cuh"
#include "simt.cuh"
#include "whale.cuh"
#include "backward.cuh"
#include "bw_tc.cuh"

using namespace wk;

namespace {

__device__ unsigned g_standalone_status;

typedef __nv_bfloat16 bf16;
typedef __half f16;

// ------------------------------------------------------------ device context

struct DevInfo {
  bool init = false;
  int id = 0;
  int sms = 0;
  PFN_cuTensorMapEncodeTiled_v12000 encode = nullptr;
  unsigned* standalone_status = nullptr;
};

std::mutex g_mu;
DevInfo g_dev[64];
std::set<std::pair<int, const void*>> g_smem_attr;

wk_status dev_info(DevInfo** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) {
    cudaGetLastError();
    return WK_ERR_CUDA;
  }
  std::lock_guard<std::mutex> lk(g_mu);
  DevInfo& d = g_dev[dev];
  if (!d.init) {
    d.id = dev;
    if (cudaDeviceGetAttribute(&d.sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) {
      cudaGetLastError();
      return WK_ERR_CUDA;
    }
    void* fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess || fn == nullptr) {
      cudaGetLastError();
      return WK_ERR_CUDA;
    }
    d.encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
    void* sym = nullptr;
    if (cudaGetSymbolAddress(&sym, g_standalone_status) != cudaSuccess) {
      cudaGetLastError();
      return WK_ERR_CUDA;
    }
    d.standalone_status = static_cast<unsigned*>(sym);
    d.init = true;
  }
  *out = &d;
  return WK_OK;
}

// Raises the dynamic shared-memory limit of a kernel once per device.
wk_status smem_attr(const DevInfo* dv, const void* fn, int bytes) {
  std::lock_guard<std::mutex> lk(g_mu);
  if (g_smem_attr.count({dv->id, fn})) return WK_OK;
  if (cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes) != cudaSuccess) {
    cudaGetLastError();
    return WK_ERR_CUDA;
  }
  g_smem_attr.insert({dv->id, fn});
  return WK_OK;
}

inline bool al16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

inline wk_status launch_status() {
  cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? WK_OK : WK_ERR_CUDA;
}

inline size_t dtype_bytes(wk_dtype t) { return t == WK_F32 ? 4 : 2; }

template <typename T>
constexpr CUtensorMapDataType tmap_dtype() {
  return sizeof(T) == 4 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32
                        : (Half16<T>::kBF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16);
}
template <>
constexpr CUtensorMapDataType tmap_dtype<float>() {
  return CU_TENSOR_MAP_DATA_TYPE_FLOAT32;
}

// Tiled tensor map; dims[0] is the contiguous dimension, strides in bytes for dims 1..rank-1.
bool make_map(const DevInfo* dv, CUtensorMap* m, CUtensorMapDataType dt, uint32_t rank, const void* base,
              const uint64_t* dims, const uint64_t* strides, const uint32_t* box, CUtensorMapSwizzle sw) {
  cuuint64_t gd[5];
  cuuint64_t gs[4];
  cuuint32_t bx[5];
  cuuint32_t es[5];
  for (uint32_t i = 0; i < rank; ++i) {
    gd[i] = dims[i];
    bx[i] = box[i];
    es[i] = 1;
  }
  for (uint32_t i = 0; i + 1 < rank; ++i) gs[i] = strides[i];
  CUresult r = dv->encode(m, dt, rank, const_cast<void*>(base), gd, gs, bx, es, CU_TENSOR_MAP_INTERLEAVE_NONE, sw,
                          CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// --------------------------------------------------------------- GEMM maps

struct GemmMaps {
  CUtensorMap A, B, C;
};

// [rows, K] 16-bit row-major (a K-major operand): box 64 x box_rows, 128B swizzle.
template <typename T>
bool map_kmajor(const DevInfo* dv, CUtensorMap* m, const void* p, uint64_t K, uint64_t rows, uint32_t box_rows) {
  const uint64_t dims[2] = {K, rows};
  const uint64_t str[1] = {K * 2};
  const uint32_t box[2] = {64, box_rows};
  return make_map(dv, m, tmap_dtype<T>(), 2, p, dims, str, box, CU_TENSOR_MAP_SWIZZLE_128B);
}

// The transpose of a K-major operand: [K, rows] 16-bit row-major with row stride ld
// elements, read MN-major: box 64 rows x 64 k, 128B swizzle.
template <typename T>
bool map_mnmajor(const DevInfo* dv, CUtensorMap* m, const void* p, uint64_t K, uint64_t rows, uint64_t ld) {
  const uint64_t dims[2] = {rows, K};
  const uint64_t str[1] = {ld * 2};
  const uint32_t box[2] = {64, 64};
  return make_map(dv, m, tmap_dtype<T>(), 2, p, dims, str, box, CU_TENSOR_MAP_SWIZZLE_128B);
}

// Output [rows, N], row stride ldc elements; 32 x 32 boxes (16-bit: 64B swizzle, fp32: 128B).
template <typename TO>
bool map_out(const DevInfo* dv, CUtensorMap* m, const void* p, uint64_t N, uint64_t rows, uint64_t ldc) {
  const uint64_t dims[2] = {N, rows};
  const uint64_t str[1] = {ldc * sizeof(TO)};
  const uint32_t box[2] = {32, 32};
  return make_map(dv, m, tmap_dtype<TO>(), 2, p, dims, str, box,
                  sizeof(TO) == 4 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B);
}

// X [batch, n, d] as the LCB's MN-major operand: box (32 t, 64 i, 1 b), 64B swizzle.
template <typename T>
bool map_lcb_x(const DevInfo* dv, CUtensorMap* m, const void* X, uint64_t n, uint64_t d, uint64_t batch) {
  // X [batch, n, d] as (32 columns, n rows, d/32 column chunks, batch): one box is a K step of
  // E = GEMM_BN / d examples, landing as E x d/32 blocks of 64 rows x 32 columns in that order
  // (the B operand layout of the LCB kernels)
  const uint64_t dims[4] = {32, n, d / 32, batch};
  const uint64_t str[3] = {d * 2, 64, n * d * 2};
  const uint32_t box[4] = {32, 64, static_cast<uint32_t>(d / 32), static_cast<uint32_t>(GEMM_BN / d)};
  return make_map(dv, m, tmap_dtype<T>(), 4, X, dims, str, box, CU_TENSOR_MAP_SWIZZLE_64B);
}

// Rows n_f..n_f+n_l-1 of a [batch, rows, d] concat buffer as a (t, r, b) tensor: box (32, 32, 1).
template <typename TO>
bool map_lcb_out(const DevInfo* dv, CUtensorMap* m, const void* cat, uint64_t rows, uint64_t d, uint64_t n_f,
                 uint64_t n_l, uint64_t batch) {
  const uint64_t es = sizeof(TO);
  const uint64_t dims[3] = {d, n_l, batch};
  const uint64_t str[2] = {d * es, rows * d * es};
  const uint32_t box[3] = {32, 32, 1};
  const uint8_t* base = static_cast<const uint8_t*>(cat) + n_f * d * es;
  return make_map(dv, m, tmap_dtype<TO>(), 3, base, dims, str, box,
                  es == 4 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B);
}

// Rows [r0, r0 + nr) of each example of a [batch, n, d] 16-bit tensor as a (d, nr, batch)
// tensor: boxes (32, box_rows, 1), 64B swizzle (stores past row nr are clipped).
template <typename T>
bool map_rows3(const DevInfo* dv, CUtensorMap* m, const void* base, uint64_t n, uint64_t d, uint64_t r0, uint64_t nr,
               uint64_t batch, uint32_t box_rows) {
  const uint64_t dims[3] = {d, nr, batch};
  const uint64_t str[2] = {d * 2, n * d * 2};
  const uint32_t box[3] = {32, box_rows, 1};
  const uint8_t* b = static_cast<const uint8_t*>(base) + r0 * d * 2;
  return make_map(dv, m, tmap_dtype<T>(), 3, b, dims, str, box, CU_TENSOR_MAP_SWIZZLE_64B);
}

template <int MODE, typename T, typename TO>
wk_status run_gemm_tc(const DevInfo* dv, const GemmMaps& mp, const GemmParams& p, cudaStream_t st) {
  constexpr uint32_t smem = gemm_smem_bytes<TO>();
  wk_status s = smem_attr(dv, reinterpret_cast<const void*>(gemm_tc_kernel<MODE, T, TO>), smem);
  if (s != WK_OK) return s;
  if (p.num_tiles <= 0) return WK_OK;
  const int grid = std::min(p.num_tiles, dv->sms);
  gemm_tc_kernel<MODE, T, TO><<<grid, GEMM_THREADS, smem, st>>>(mp.A, mp.B, mp.C, p);
  return launch_status();
}

// The CTA-pair GEMM in one of its two launch shapes (gemm_tc2.cuh): streaming (one pair
// per output tile, two pairs' CTAs per SM; the forward's Linears: measured on the 8-layer
// stack it reads 2.3-2.9x fewer DRAM bytes per Linear than the persistent shape and runs
// the step ~5 % faster under the power cap) or persistent (one pair per two SMs, two TMEM
// accumulators: the backward's weight gradients, whose short K leaves the streaming
// shape's single accumulator exposed).
template <typename T, typename TO, bool A_MN = false, bool B_MN = false>
wk_status run_gemm_tc2(const DevInfo* dv, const GemmMaps& mp, const GemmParams& p, cudaStream_t st,
                       bool stream = true) {
  if (p.num_tiles <= 0) return WK_OK;
  if (stream) {
    constexpr uint32_t smem = gemm2_smem_bytes<TO, true>();
    wk_status s = smem_attr(dv, reinterpret_cast<const void*>(gemm_tc2_kernel<T, TO, true, A_MN, B_MN>), smem);
    if (s != WK_OK) return s;
    gemm_tc2_kernel<T, TO, true, A_MN, B_MN><<<2 * p.num_tiles, GEMM_THREADS, smem, st>>>(mp.A, mp.B, mp.C, p);
    return launch_status();
  }
  constexpr uint32_t smem = gemm2_smem_bytes<TO>();
  wk_status s = smem_attr(dv, reinterpret_cast<const void*>(gemm_tc2_kernel<T, TO, false, A_MN, B_MN>), smem);
  if (s != WK_OK) return s;
  const int pairs = std::min(p.num_tiles, dv->sms / 2);
  gemm_tc2_kernel<T, TO, false, A_MN, B_MN><<<2 * pairs, GEMM_THREADS, smem, st>>>(mp.A, mp.B, mp.C, p);
  return launch_status();
}

// The CTA-pair GEMM (256-row tiles) serves every M above one 128-row tile.
bool use_pair_gemm(int64_t M) { return M > GEMM_BM; }

GemmParams mlp2_params(int64_t M, int K, int N, const float* bias, int relu, unsigned* status) {
  GemmParams p{};
  p.M = static_cast<int>(M);
  p.N = N;
  p.K = K;
  p.num_m_tiles = static_cast<int>((M + GEMM2_BM - 1) / GEMM2_BM);
  p.num_n_tiles = (N + GEMM2_BN - 1) / GEMM2_BN;
  p.num_tiles = p.num_m_tiles * p.num_n_tiles;
  p.num_kb = (K + GEMM2_BK - 1) / GEMM2_BK;
  p.group_m = GEMM2_GROUP_M;
  p.mma_n = GEMM2_BN;
  p.bias = bias;
  p.relu = relu;
  p.status = status;
  return p;
}

GemmParams mlp_params(int64_t M, int K, int N, const float* bias, int relu, unsigned* status) {
  GemmParams p{};
  p.M = static_cast<int>(M);
  p.N = N;
  p.K = K;
  p.num_m_tiles = static_cast<int>((M + GEMM_BM - 1) / GEMM_BM);
  p.num_n_tiles = (N + GEMM_BN - 1) / GEMM_BN;
  p.num_tiles = p.num_m_tiles * p.num_n_tiles;
  p.num_kb = (K + GEMM_BK - 1) / GEMM_BK;
  p.group_m = 16;
  p.mma_n = GEMM_BN;
  p.bias = bias;
  p.relu = relu;
  p.status = status;
  return p;
}

GemmParams lcb_params(int64_t batch, int n, int d, int n_l, unsigned* status) {
  GemmParams p{};
  p.M = n_l;
  p.N = static_cast<int>(batch);
  p.K = n;
  p.d = d;
  p.E = GEMM_BN / d;
  p.dchunks = d / 32;
  p.num_m_tiles = (n_l + GEMM_BM - 1) / GEMM_BM;
  p.num_n_tiles = static_cast<int>((batch + p.E - 1) / p.E);
  p.num_tiles = p.num_m_tiles * p.num_n_tiles;
  p.num_kb = (n + GEMM_BK - 1) / GEMM_BK;
  p.mma_n = p.E * d;
  p.status = status;
  return p;
}

// The LCB with W_L resident in shared memory (lcb_tc.cuh) wherever its K panel fits,
// else the streaming GEMM (MODE_LCB).
template <typename T, typename TO>
wk_status run_lcb_tc(const DevInfo* dv, const GemmMaps& mp, const GemmParams& p, cudaStream_t st) {
  const uint32_t b_stage = static_cast<uint32_t>(p.E * p.dchunks) * 4096u;
  const int stages = lcb_tc_stages<TO>(p.num_kb, b_stage);
  if (p.num_kb > LCB_MAX_KB || stages < 2 || p.num_m_tiles > dv->sms)
    return run_gemm_tc<MODE_LCB, T, TO>(dv, mp, p, st);
  wk_status s = smem_attr(dv, reinterpret_cast<const void*>(lcb_tc_kernel<T, TO>), static_cast<int>(LCB_SMEM_BUDGET));
  if (s != WK_OK) return s;
  if (p.num_tiles <= 0) return WK_OK;
  // every CTA keeps one W_L tile: the grid is a multiple of the m-tile count
  const int per_m = std::max(1, std::min(p.num_n_tiles, dv->sms / p.num_m_tiles));
  const int grid = per_m * p.num_m_tiles;
  const uint32_t smem = lcb_tc_fixed_bytes<TO>(p.num_kb) + static_cast<uint32_t>(stages) * b_stage;
  lcb_tc_kernel<T, TO><<<grid, GEMM_THREADS, smem, st>>>(mp.A, mp.B, mp.C, p, stages);
  return launch_status();
}

bool mlp_tc_ok(int64_t M, int K, int N, int64_t ldc) {
  return M > 0 && K >= 8 && N >= 8 && K % 8 == 0 && N % 8 == 0 && ldc % 8 == 0 && ldc >= N && M < (1ll << 31);
}

bool lcb_tc_ok(int64_t batch, int n, int d) {
  return d % 32 == 0 && d >= 32 && d <= GEMM_BN && n % 8 == 0 && batch < (1ll << 31);
}

// ------------------------------------------------------------------ FM + LN

template <class C, typename T>
wk_status run_fm_tc(const DevInfo* dv, const T* X, const T* Y, const float* g, const float* b, T* A0, int64_t batch,
                    float eps, unsigned* status, cudaStream_t st) {
  wk_status s = smem_attr(dv, reinterpret_cast<const void*>(fm_ln_tc_kernel<C, T>), C::SMEM);
  if (s != WK_OK) return s;
  CUtensorMap tmX, tmY;
  {  // X as [batch*n rows, d]: boxes of XBOXW columns x 128 rows
    const uint64_t dims[2] = {static_cast<uint64_t>(C::D), static_cast<uint64_t>(batch) * C::N};
    const uint64_t str[1] = {static_cast<uint64_t>(C::D) * 2};
    const uint32_t box[2] = {static_cast<uint32_t>(C::XBOXW), static_cast<uint32_t>(C::R)};
    if (!make_map(dv, &tmX, tmap_dtype<T>(), 2, X, dims, str, box,
                  C::XSW == 128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B))
      return WK_ERR_UNSUPPORTED;
  }
  {  // Y [n, k]: boxes of KP columns (zero-filled past k) x 128 rows
    const uint64_t dims[2] = {static_cast<uint64_t>(C::K), static_cast<uint64_t>(C::N)};
    const uint64_t str[1] = {static_cast<uint64_t>(C::K) * 2};
    const uint32_t box[2] = {static_cast<uint32_t>(C::KP), static_cast<uint32_t>(C::R)};
    if (!make_map(dv, &tmY, tmap_dtype<T>(), 2, Y, dims, str, box,
                  C::YRB == 128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B))
      return WK_ERR_UNSUPPORTED;
  }
  const int grid = static_cast<int>(std::min<int64_t>(batch, dv->sms));
  fm_ln_tc_kernel<C, T><<<grid, FMTC_THREADS, C::SMEM, st>>>(tmX, tmY, g, b, A0, batch, eps, status);
  return launch_status();
}

size_t fm_simt_smem(int n, int d, int k) {
  return sizeof(float) * (static_cast<size_t>(n) * d + 2ull * n * k + static_cast<size_t>(d) * k);
}

template <typename T>
wk_status run_fm_simt(const DevInfo* dv, const T* X, const T* Y, const float* g, const float* b, T* A0,
                      int64_t batch, int n, int d, int k, float eps, cudaStream_t st) {
  const size_t smem = fm_simt_smem(n, d, k);
  if (smem > 200 * 1024) return WK_ERR_UNSUPPORTED;
  if (smem > 48 * 1024) {
    wk_status s = smem_attr(dv, reinterpret_cast<const void*>(fm_ln_simt<T>), static_cast<int>(smem));
    if (s != WK_OK) return s;
  }
  const int grid = static_cast<int>(std::min<int64_t>(batch, 8ll * dv->sms));
  fm_ln_simt<T><<<grid, 256, smem, st>>>(X, Y, g, b, A0, batch, n, d, k, eps);
  return launch_status();
}

bool fm_tc_shape(int n, int d, int k) {
  return (n == 512 && d == 160 && k == 64) || (n == 256 && d == 160 && k == 32) || (n == 64 && d == 128 && k == 16) ||
         (n == 720 && d == 32 && k == 24);
}

// 16-bit FM dispatch: the tensor-core kernel for the instantiated shapes, else the CUDA-core one.
template <typename T>
wk_status run_fm16(const DevInfo* dv, const T* X, const T* Y, const float* g, const float* b, T* A0, int64_t batch,
                   int n, int d, int k, float eps, unsigned* status, cudaStream_t st) {
  if (n == 512 && d == 160 && k == 64) return run_fm_tc<FmTcC4, T>(dv, X, Y, g, b, A0, batch, eps, status, st);
  if (n == 256 && d == 160 && k == 32) return run_fm_tc<FmTcC3, T>(dv, X, Y, g, b, A0, batch, eps, status, st);
  if (n == 64 && d == 128 && k == 16) return run_fm_tc<FmTcC2, T>(dv, X, Y, g, b, A0, batch, eps, status, st);
  if (n == 720 && d == 32 && k == 24) return run_fm_tc<FmTcC5, T>(dv, X, Y, g, b, A0, batch, eps, status, st);
  return run_fm_simt<T>(dv, X, Y, g, b, A0, batch, n, d, k, eps, st);
}

// ------------------------------------------------------------- layer front

// The shapes the front kernel is instantiated for (FrontC2..C4): 0..2, or -1.
int front_shape(int n, int d, int k, int n_f) {
  if (n == 64 && d == 128 && k == 16 && n_f == 32) return 0;
  if (n == 256 && d == 160 && k == 32 && n_f == 128) return 1;
  if (n == 512 && d == 160 && k == 64 && n_f == 256) return 2;
  return -1;
}

struct FrontMaps {
  CUtensorMap Y, W, R, L, A;
};

template <class C, typename TIN, typename T>
wk_status run_front_c(const DevInfo* dv, const FrontMaps& mp, const TIN* xin, const float* in_g, const float* in_b,
                      const float* fg, const float* fb, T* A0, T* yout, int64_t batch, float eps, unsigned* status,
                      cudaStream_t st) {
  wk_status s = smem_attr(dv, reinterpret_cast<const void*>(front_tc_kernel<C, TIN, T>), C::SMEM);
  if (s != WK_OK) return s;
  const int grid = static_cast<int>(std::min<int64_t>(batch, dv->sms));
  front_tc_kernel<C, TIN, T><<<grid, FRONT_THREADS, C::SMEM, st>>>(xin, mp.Y, mp.W, mp.R, mp.L, mp.A, in_g, in_b, fg,
                                                                   fb, A0, yout, batch, eps, status);
  return launch_status();
}

template <typename TIN, typename T>
wk_status run_front(const DevInfo* dv, int shape, const FrontMaps& mp, const TIN* xin, const float* in_g,
                    const float* in_b, const float* fg, const float* fb, T* A0, T* yout, int64_t batch, float eps,
                    unsigned* status, cudaStream_t st) {
  switch (shape) {
    case 0: return run_front_c<FrontC2, TIN, T>(dv, mp, xin, in_g, in_b, fg, fb, A0, yout, batch, eps, status, st);
    case 1: return run_front_c<FrontC3, TIN, T>(dv, mp, xin, in_g, in_b, fg, fb, A0, yout, batch, eps, status, st);
    case 2: return run_front_c<FrontC4, TIN, T>(dv, mp, xin, in_g, in_b, fg, fb, A0, yout, batch, eps, status, st);
    default: return WK_ERR_UNSUPPORTED;
  }
}

bool fm_supported(int n, int d, int k, bool sixteen_bit) {
  if (sixteen_bit && fm_tc_shape(n, d, k)) return true;
  return fm_simt_smem(n, d, k) <= 200 * 1024;
}

// ------------------------------------------------------------ residual + LN

// The bulk-copy ring kernel for 16-bit inputs (16-byte aligned), else the register-only
// kernel (fp32, and the stand-alone call's unaligned 16-bit inputs); a null residual x
// (the output LayerNorm alone) only on the ring.
template <int D, typename TC, typename TR, typename TO>
wk_status run_res_ln_d(const DevInfo* dv, const TC* cat, const TR* x, const float* g, const float* b, TO* out,
                       int64_t rows, float eps, unsigned* status, cudaStream_t st) {
  if constexpr (sizeof(TC) == 2 && sizeof(TR) == 2) {
    if (al16(cat) && al16(x)) {
      using C = ResLnRing<D>;
      const int64_t tiles = (rows + C::R - 1) / C::R;
      const int grid = static_cast<int>(std::max<int64_t>(1, std::min<int64_t>(tiles, dv->sms)));
      if (x == nullptr) {
        wk_status s = smem_attr(dv, reinterpret_cast<const void*>(res_ln_ring_kernel<D, TC, TR, TO, false>), C::SMEM);
        if (s != WK_OK) return s;
        res_ln_ring_kernel<D, TC, TR, TO, false><<<grid, C::THREADS, C::SMEM, st>>>(cat, x, g, b, out, rows, eps, status);
        return launch_status();
      }
      wk_status s = smem_attr(dv, reinterpret_cast<const void*>(res_ln_ring_kernel<D, TC, TR, TO>), C::SMEM);
      if (s != WK_OK) return s;
      res_ln_ring_kernel<D, TC, TR, TO><<<grid, C::THREADS, C::SMEM, st>>>(cat, x, g, b, out, rows, eps, status);
      return launch_status();
    }
  }
  if (x == nullptr) return WK_ERR_UNSUPPORTED;  // the output LayerNorm alone runs on the ring only
  constexpr int VPR = D / 8;
  constexpr int G = res_ln_lanes(VPR);
  constexpr int rows_per_block = (256 / 32) * (32 / G) * ((VPR / G) >= 4 ? 2 : 4);
  int64_t blocks = (rows + rows_per_block - 1) / rows_per_block;
  const int64_t cap = static_cast<int64_t>(dv->sms) * 8;
  if (blocks > cap) blocks = cap;
  if (blocks < 1) blocks = 1;
  res_ln_kernel<D, TC, TR, TO><<<static_cast<int>(blocks), 256, 0, st>>>(cat, x, g, b, out, nullptr, rows, eps);
  return launch_status();
}

bool res_ln_d_ok(int d) {
  return d == 16 || d == 32 || d == 64 || d == 128 || d == 160 || d == 192 || d == 256;
}

template <typename TC, typename TR, typename TO>
wk_status run_res_ln(const DevInfo* dv, const TC* cat, const TR* x, const float* g, const float* b, TO* out,
                     int64_t rows, int d, float eps, unsigned* status, cudaStream_t st) {
  switch (d) {
    case 16: return run_res_ln_d<16>(dv, cat, x, g, b, out, rows, eps, status, st);
    case 32: return run_res_ln_d<32>(dv, cat, x, g, b, out, rows, eps, status, st);
    case 64: return run_res_ln_d<64>(dv, cat, x, g, b, out, rows, eps, status, st);
    case 128: return run_res_ln_d<128>(dv, cat, x, g, b, out, rows, eps, status, st);
    case 160: return run_res_ln_d<160>(dv, cat, x, g, b, out, rows, eps, status, st);
    case 192: return run_res_ln_d<192>(dv, cat, x, g, b, out, rows, eps, status, st);
    case 256: return run_res_ln_d<256>(dv, cat, x, g, b, out, rows, eps, status, st);
    default: return WK_ERR_UNSUPPORTED;
  }
}

template <typename TI, typename TO>
wk_status run_convert(const DevInfo* dv, const void* in, void* out, int64_t n, cudaStream_t st) {
  if (n <= 0) return WK_OK;
  int64_t blocks = (n / 8 + 255) / 256;
  blocks = std::max<int64_t>(1, std::min<int64_t>(blocks, static_cast<int64_t>(dv->sms) * 16));
  convert_kernel<TI, TO><<<static_cast<int>(blocks), 256, 0, st>>>(static_cast<const TI*>(in), static_cast<TO*>(out),
                                                                    n);
  return launch_status();
}

// ------------------------------------------------------------ prediction head

template <typename T>
wk_status run_head_out(const DevInfo* dv, const T* H, const T* w, const float* bias, float* logit, float* prob,
                       int64_t batch, int64_t K, cudaStream_t st) {
  const int64_t warps_needed = batch;
  int64_t blocks = (warps_needed + 7) / 8;
  blocks = std::max<int64_t>(1, std::min<int64_t>(blocks, static_cast<int64_t>(dv->sms) * 16));
  head_out_kernel<T><<<static_cast<int>(blocks), 256, 0, st>>>(H, w, bias, logit, prob, batch, K);
  return launch_status();
}

// ------------------------------------------------------------ mixture of experts

template <typename T, int E>
wk_status run_moe_gate_e(const DevInfo* dv, const T* X, const T* Wg, const float* bg, float* g, int64_t batch,
                         int64_t nd, cudaStream_t st) {
  const int64_t need = (batch + 7) / 8;
  const int grid = static_cast<int>(std::max<int64_t>(1, std::min<int64_t>(need, static_cast<int64_t>(dv->sms) * 8)));
  moe_gate_kernel<T, E><<<grid, 256, 0, st>>>(X, Wg, bg, g, batch, nd);
  return launch_status();
}

template <typename T>
wk_status run_moe_gate(const DevInfo* dv, const T* X, const T* Wg, const float* bg, float* g, int64_t batch,
                       int64_t nd, int E, cudaStream_t st) {
  switch (E) {
    case 1: return run_moe_gate_e<T, 1>(dv, X, Wg, bg, g, batch, nd, st);
    case 2: return run_moe_gate_e<T, 2>(dv, X, Wg, bg, g, batch, nd, st);
    case 3: return run_moe_gate_e<T, 3>(dv, X, Wg, bg, g, batch, nd, st);
    case 4: return run_moe_gate_e<T, 4>(dv, X, Wg, bg, g, batch, nd, st);
    case 5: return run_moe_gate_e<T, 5>(dv, X, Wg, bg, g, batch, nd, st);
    case 6: return run_moe_gate_e<T, 6>(dv, X, Wg, bg, g, batch, nd, st);
    case 7: return run_moe_gate_e<T, 7>(dv, X, Wg, bg, g, batch, nd, st);
    case 8: return run_moe_gate_e<T, 8>(dv, X, Wg, bg, g, batch, nd, st);
    default: return WK_ERR_UNSUPPORTED;
  }
}

template <int D, typename T, typename TO>
wk_status run_moe_combine_d(const DevInfo* dv, const MoePtrs& p, const T* x, const float* g, TO* out, int64_t rows,
                            int n, int E, float eps, unsigned* status, cudaStream_t st) {
  using R = MoeRing<D>;
  wk_status s = smem_attr(dv, reinterpret_cast<const void*>(moe_combine_ring_kernel<D, T, TO>), R::SMEM);
  if (s != WK_OK) return s;
  const int64_t tiles = (rows + R::R - 1) / R::R;
  const int grid = static_cast<int>(std::max<int64_t>(1, std::min<int64_t>(tiles, dv->sms)));
  moe_combine_ring_kernel<D, T, TO><<<grid, R::THREADS, R::SMEM, st>>>(p, x, g, out, rows, n, E, eps, status);
  return launch_status();
}

template <typename T, typename TO>
wk_status run_moe_combine(const DevInfo* dv, const MoePtrs& p, const T* x, const float* g, TO* out, int64_t rows,
                          int n, int d, int E, float eps, unsigned* status, cudaStream_t st) {
  switch (d) {
    case 16: return run_moe_combine_d<16>(dv, p, x, g, out, rows, n, E, eps, status, st);
    case 32: return run_moe_combine_d<32>(dv, p, x, g, out, rows, n, E, eps, status, st);
    case 64: return run_moe_combine_d<64>(dv, p, x, g, out, rows, n, E, eps, status, st);
    case 128: return run_moe_combine_d<128>(dv, p, x, g, out, rows, n, E, eps, status, st);
    case 160: return run_moe_combine_d<160>(dv, p, x, g, out, rows, n, E, eps, status, st);
    case 192: return run_moe_combine_d<192>(dv, p, x, g, out, rows, n, E, eps, status, st);
    case 256: return run_moe_combine_d<256>(dv, p, x, g, out, rows, n, E, eps, status, st);
    default: return WK_ERR_UNSUPPORTED;
  }
}

// ------------------------------------------------------------------- SIMT

template <typename T, typename TO>
wk_status run_gemm_simt(const T* A, const T* W, const float* bias, TO* C, int64_t M, int K, int N, int64_t ldc,
                        int relu, cudaStream_t st) {
  const int64_t gy = (M + 63) / 64;
  if (gy > 65535) return WK_ERR_UNSUPPORTED;
  dim3 grid((N + 63) / 64, static_cast<unsigned>(gy));
  gemm_simt<T, TO><<<grid, 256, 0, st>>>(A, W, bias, C, M, K, N, ldc, relu);
  return launch_status();
}

template <typename T, typename TO>
wk_status run_lcb_simt(const T* WL, const T* X, TO* cat, int64_t batch, int n, int d, int n_f, int n_l,
                       cudaStream_t st) {
  for (int64_t b0 = 0; b0 < batch; b0 += 65535) {
    const int64_t nb = std::min<int64_t>(65535, batch - b0);
    dim3 grid((n_l * d + 255) / 256, static_cast<unsigned>(nb));
    lcb_simt<T, TO><<<grid, 256, 0, st>>>(WL, X + b0 * n * d, cat + b0 * (n_f + n_l) * d, nb, n, d, n_f, n_l);
    wk_status s = launch_status();
    if (s != WK_OK) return s;
  }
  return WK_OK;
}

}  // namespace

// ====================================================================== handle

struct wk_stack {
  int device = 0;
  wk_stack_config cfg{};
  std::vector<int32_t> dims;  // h_0 .. h_m
  float eps = 1e-5f;
  wk_dtype io = WK_BF16;      // caller's storage type of X, out and the weights
  wk_dtype op = WK_F16;       // operand / intermediate type (WK_F32 for fp32 stacks)
  int64_t maxb = 0;
  const DevInfo* dv = nullptr;
  // operand weights per layer (the caller's, or converted copies in wcopy)
  std::vector<const void*> Y, WL;
  std::vector<std::vector<const void*>> W;
  std::vector<std::vector<const float*>> b;
  std::vector<const float*> g1, b1, g2, b2;
  uint8_t* wcopy = nullptr;
  // workspace (operand type)
  uint8_t* ws = nullptr;
  void* A0 = nullptr;
  void* H[2] = {nullptr, nullptr};
  void* cat = nullptr;
  void* Xs[2] = {nullptr, nullptr};  // layer outputs; Xs[1] also takes a converted input
  unsigned* status = nullptr;
  // TMA descriptors of the tensor-core path
  bool tc_mlp = false, tc_lcb = false;
  bool pair = false;                            // MLP Linears on CTA pairs (gemm_tc2.cuh)
  bool front_only = false;                      // an expert of a wk_moe: no layer buffers, no fused path
  std::vector<std::vector<GemmMaps>> mlp_maps;  // [layer][j]
  std::vector<CUtensorMap> lcbA;                // [layer]
  CUtensorMap lcbB_ws[2];
  CUtensorMap lcbC;
  // the layer front in one kernel (front_tc.cuh): its shape (-1: not used), Y, W_L and A0
  // per layer, and the layer buffers Xs[0] / Xs[1] as a front's residual and LCB outputs
  // (R, L) and as the last Linear's reduce-add target (C)
  int front = -1;
  std::vector<FrontMaps> fmaps;                 // [layer]: Y, W, A
  CUtensorMap frontR[2], frontL[2], frontC[2];
  // prediction head (wk_stack_set_head): q Linears, dims n*d -> ... -> 1
  std::vector<int32_t> head_dims;               // empty: no head
  std::vector<const void*> hT;                  // [q] operand type
  std::vector<const float*> hc;                 // [q]
  uint8_t* head_copy = nullptr;                 // weights converted to the operand type
  uint8_t* head_ws = nullptr;                   // two activation buffers [maxb, widest hidden]
  void* HH[2] = {nullptr, nullptr};
  std::vector<GemmMaps> head_maps;              // [q-1] hidden Linears
  // host-buffer forward
  uint8_t* stage = nullptr;
  int64_t stage_chunk = 0;
  cudaStream_t s_in = nullptr, s_out = nullptr;
  // streamed host-buffer forward: two input and two output slots of max_batch examples,
  // per slot the events of its input copy, forward and output copy, and the calls issued
  uint8_t* astage = nullptr;
  cudaEvent_t a_in[2] = {nullptr, nullptr}, a_done[2] = {nullptr, nullptr}, a_out[2] = {nullptr, nullptr};
  int64_t a_seq = 0;
  // profiling
  bool prof = false;
  struct Rec {
    int kind;
    cudaEvent_t a, b;
  };
  std::vector<Rec> recs;
  std::vector<cudaEvent_t> pool;
  // backward: the caller's first Linear and FMB LayerNorm parameters (the forward uses
  // the folded W0', b0'), and the backward workspace (allocated at the first backward)
  std::vector<const void*> W0_in;
  std::vector<const float*> b0_in, g1_in, b1_in;
  uint8_t* bws = nullptr;
  size_t bws_bytes = 0;
};

// A stack of Wukong mixture-of-experts layers: one front-only wk_stack per expert
// (its weights, converted copies, descriptors and one layer's front workspace),
// the gates, and the MoE's own layer buffers.
struct wk_moe {
  int device = 0;
  wk_stack_config cfg{};
  int E = 0;
  float eps = 1e-5f;
  wk_dtype io = WK_BF16, op = WK_F16;
  int64_t maxb = 0;
  const DevInfo* dv = nullptr;
  std::vector<wk_stack*> ex;        // [E]
  std::vector<const void*> Wg;      // [layer], operand type
  std::vector<const float*> bg;     // [layer]
  uint8_t* wcopy = nullptr;         // gate weights converted to the operand type
  uint8_t* ws = nullptr;
  float* g = nullptr;               // [maxb, E]
  void* Xm[2] = {nullptr, nullptr}; // layer outputs; Xm[1] also takes a converted input
  CUtensorMap lcbX[2];              // Xm[0], Xm[1] as the LCB's operand
};

struct wk_graph {
  int device = 0;
  cudaGraph_t graph = nullptr;
  cudaGraphExec_t exec = nullptr;
};

namespace {

struct ProfScope {
  wk_stack* h;
  int kind;
  cudaStream_t st;
  cudaEvent_t a = nullptr, b = nullptr;
  ProfScope(wk_stack* h_, int k, cudaStream_t s) : h(h_), kind(k), st(s) {
    if (!h->prof) return;
    a = take();
    b = take();
    if (a && b) cudaEventRecord(a, st);
  }
  cudaEvent_t take() {
    cudaEvent_t e = nullptr;
    if (!h->pool.empty()) {
      e = h->pool.back();
      h->pool.pop_back();
    } else if (cudaEventCreate(&e) != cudaSuccess) {
      cudaGetLastError();
      e = nullptr;
    }
    return e;
  }
  ~ProfScope() {
    if (!h->prof) return;
    if (a && b) {
      cudaEventRecord(b, st);
      h->recs.push_back({kind, a, b});
    } else {
      if (a) h->pool.push_back(a);
      if (b) h->pool.push_back(b);
    }
  }
};

void free_stack(wk_stack* h) {
  if (!h) return;
  cudaDeviceSynchronize();
  cudaGetLastError();
  if (h->ws) cudaFree(h->ws);
  if (h->wcopy) cudaFree(h->wcopy);
  if (h->head_copy) cudaFree(h->head_copy);
  if (h->head_ws) cudaFree(h->head_ws);
  if (h->stage) cudaFree(h->stage);
  if (h->bws) cudaFree(h->bws);
  if (h->astage) cudaFree(h->astage);
  for (int i = 0; i < 2; ++i) {
    if (h->a_in[i]) cudaEventDestroy(h->a_in[i]);
    if (h->a_done[i]) cudaEventDestroy(h->a_done[i]);
    if (h->a_out[i]) cudaEventDestroy(h->a_out[i]);
  }
  if (h->s_in) cudaStreamDestroy(h->s_in);
  if (h->s_out) cudaStreamDestroy(h->s_out);
  for (auto& r : h->recs) {
    cudaEventDestroy(r.a);
    cudaEventDestroy(r.b);
  }
  for (auto e : h->pool) cudaEventDestroy(e);
  cudaGetLastError();
  delete h;
}

wk_status validate_cfg(const wk_stack_config* c) {
  if (!c) return WK_ERR_INVALID_ARG;
  if (c->num_layers < 1 || c->n < 1 || c->d < 1 || c->k < 1 || c->n_f < 1 || c->n_l < 1 || c->mlp_num_linear < 1 ||
      c->max_batch < 1)
    return WK_ERR_INVALID_ARG;
  if (c->mlp_num_linear > 1 && !c->mlp_hidden) return WK_ERR_INVALID_ARG;
  if (c->dtype != WK_F32 && c->dtype != WK_BF16 && c->dtype != WK_F16) return WK_ERR_UNSUPPORTED;
  if (c->operand_dtype != WK_F32 && c->operand_dtype != WK_BF16 && c->operand_dtype != WK_F16)
    return WK_ERR_UNSUPPORTED;
  if (c->n_f + c->n_l != c->n) return WK_ERR_UNSUPPORTED;
  if (c->d % 8 != 0 || !res_ln_d_ok(c->d)) return WK_ERR_UNSUPPORTED;
  for (int j = 0; j + 1 < c->mlp_num_linear; ++j)
    if (c->mlp_hidden[j] < 1 || c->mlp_hidden[j] % 8 != 0) return WK_ERR_UNSUPPORTED;
  if ((static_cast<int64_t>(c->n) * c->k) % 8 != 0) return WK_ERR_UNSUPPORTED;
  if (!fm_supported(c->n, c->d, c->k, c->dtype != WK_F32)) return WK_ERR_UNSUPPORTED;
  if (c->ln_eps < 0.f) return WK_ERR_INVALID_ARG;
  return WK_OK;
}

// Builds the tensor-core descriptors of a 16-bit stack (operand type T).
template <typename T>
wk_status build_maps(wk_stack* h) {
  const wk_stack_config& c = h->cfg;
  const DevInfo* dv = h->dv;
  const int L = c.num_layers, m = c.mlp_num_linear, n = c.n, d = c.d;
  const int64_t B = h->maxb;
  const uint64_t nd = static_cast<uint64_t>(n) * d;
  h->tc_mlp = true;
  for (int j = 0; j < m; ++j) {
    const int64_t ldc = (j == m - 1) ? static_cast<int64_t>(nd) : h->dims[j + 1];
    if (!mlp_tc_ok(B, h->dims[j], h->dims[j + 1], ldc)) h->tc_mlp = false;
  }
  h->tc_lcb = lcb_tc_ok(B, n, d);
  h->pair = use_pair_gemm(B);
  if (h->tc_mlp) {
    h->mlp_maps.assign(L, std::vector<GemmMaps>(m));
    for (int l = 0; l < L; ++l)
      for (int j = 0; j < m; ++j) {
        GemmMaps& mp = h->mlp_maps[l][j];
        const void* in = (j == 0) ? h->A0 : h->H[(j - 1) % 2];
        const bool last = j == m - 1;
        const bool ok = map_kmajor<T>(dv, &mp.A, in, h->dims[j], B, GEMM_BM) &&
                        map_kmajor<T>(dv, &mp.B, h->W[l][j], h->dims[j], h->dims[j + 1], h->pair ? 128 : GEMM_BN) &&
                        (last ? map_out<T>(dv, &mp.C, h->cat, h->dims[j + 1], B, nd)
                              : map_out<T>(dv, &mp.C, h->H[j % 2], h->dims[j + 1], B, h->dims[j + 1]));
        if (!ok) return WK_ERR_UNSUPPORTED;
      }
  }
  const int shape = front_shape(n, d, c.k, c.n_f);
  // fp16 operands only: the front keeps each layer's output before its LayerNorm in the
  // operand type (the last Linear adds into it), one rounding more than the separate
  // residual + LayerNorm pass, which bf16's 8-bit significand cannot spare on the 2-layer
  // workload (0.0211 against 0.0161 with the four-kernel layer, tolerance 0.02)
  const bool front_types = h->op == WK_F16;
  // The front streams W_L from L2 once per example: worth it while W_L's rows per example
  // (n_l x n) stay within twice the example's own n x d (the wide/narrow workload, n_l = 360
  // against d = 32, reads 11x its input's bytes of W_L and keeps the four-kernel layer, whose
  // LCB shares each W_L load among several examples)
  const bool front_lcb = c.n_l <= 2 * d;
  const bool front_rows = static_cast<int64_t>(B) * n < (1ll << 31);  // A0 row coordinates are int32
  if (h->tc_mlp && !h->front_only && shape >= 0 && front_types && front_lcb && front_rows) {
    const int KP = c.k <= 32 ? 32 : 64;
    h->fmaps.resize(L);
    bool ok = true;
    for (int l = 0; l < L; ++l) {
      // Y [n, k]: boxes of KP columns (zero past k) x 128 rows
      const uint64_t ydims[2] = {static_cast<uint64_t>(c.k), static_cast<uint64_t>(n)};
      const uint64_t ystr[1] = {static_cast<uint64_t>(c.k) * 2};
      const uint32_t ybox[2] = {static_cast<uint32_t>(KP), 128};
      ok = ok && make_map(dv, &h->fmaps[l].Y, tmap_dtype<T>(), 2, h->Y[l], ydims, ystr, ybox,
                          KP == 64 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B);
      ok = ok && map_kmajor<T>(dv, &h->fmaps[l].W, h->WL[l], n, c.n_l, 128);
    }
    {  // A0 [B*n rows, k]: boxes of (up to) 32 columns x 32 rows
      const uint64_t adims[2] = {static_cast<uint64_t>(c.k), static_cast<uint64_t>(B) * n};
      const uint64_t astr[1] = {static_cast<uint64_t>(c.k) * 2};
      const uint32_t abox[2] = {static_cast<uint32_t>(std::min(c.k, 32)), 32};
      const CUtensorMapSwizzle asw = c.k >= 32   ? CU_TENSOR_MAP_SWIZZLE_64B
                                     : c.k == 16 ? CU_TENSOR_MAP_SWIZZLE_32B
                                                 : CU_TENSOR_MAP_SWIZZLE_NONE;
      for (int l = 0; l < L; ++l)
        ok = ok && make_map(dv, &h->fmaps[l].A, tmap_dtype<T>(), 2, h->A0, adims, astr, abox, asw);
    }
    for (int i = 0; i < 2; ++i)
      ok = ok && map_rows3<T>(dv, &h->frontR[i], h->Xs[i], n, d, 0, c.n_f, B, std::min(128, c.n_f)) &&
           map_rows3<T>(dv, &h->frontL[i], h->Xs[i], n, d, c.n_f, c.n_l, B, 32) &&
           map_out<T>(dv, &h->frontC[i], h->Xs[i], static_cast<uint64_t>(c.n_f) * d, B, nd);
    if (!ok) return WK_ERR_UNSUPPORTED;
    h->front = shape;
  }
  if (h->tc_lcb) {
    h->lcbA.resize(L);
    bool ok = true;
    for (int l = 0; l < L; ++l) ok = ok && map_kmajor<T>(dv, &h->lcbA[l], h->WL[l], n, c.n_l, GEMM_BM);
    if (!h->front_only)
      ok = ok && map_lcb_x<T>(dv, &h->lcbB_ws[0], h->Xs[0], n, d, B) &&
           map_lcb_x<T>(dv, &h->lcbB_ws[1], h->Xs[1], n, d, B);
    ok = ok && map_lcb_out<T>(dv, &h->lcbC, h->cat, n, d, c.n_f, c.n_l, B);
    if (!ok) return WK_ERR_UNSUPPORTED;
  }
  return WK_OK;
}

// The front of layer l of a 16-bit stack (operand type T): FM + LayerNorm, the MLP
// Linears (the last one into rows 0..n_f-1 of the concat buffer) and the LCB (rows
// n_f..n-1), reading the layer input xin; lcb_x is xin as the LCB's TMA operand.
// Leaves the residual + LayerNorm to the caller.
template <typename T>
wk_status layer_front16(wk_stack* h, int l, const T* xin, const CUtensorMap& lcb_x, int64_t batch, cudaStream_t st) {
  const wk_stack_config& c = h->cfg;
  const DevInfo* dv = h->dv;
  const int n = c.n, d = c.d, k = c.k, m = c.mlp_num_linear;
  const size_t nd = static_cast<size_t>(n) * d;
  wk_status s = WK_OK;
  {  // 1. FM + LN
    ProfScope ps(h, WK_KERNEL_FM_LN, st);
    s = run_fm16<T>(dv, xin, static_cast<const T*>(h->Y[l]), h->g1[l], h->b1[l], static_cast<T*>(h->A0), batch, n, d,
                    k, h->eps, h->status, st);
  }
  for (int j = 0; j < m && s == WK_OK; ++j) {  // 2. MLP
    ProfScope ps(h, WK_KERNEL_MLP_GEMM, st);
    const void* in = (j == 0) ? h->A0 : h->H[(j - 1) % 2];
    const bool lastj = j == m - 1;
    void* o = lastj ? h->cat : h->H[j % 2];
    const int64_t ldc = lastj ? static_cast<int64_t>(nd) : h->dims[j + 1];
    const int relu = lastj ? 0 : 1;
    if (h->tc_mlp && h->pair)
      s = run_gemm_tc2<T, T>(dv, h->mlp_maps[l][j],
                             mlp2_params(batch, h->dims[j], h->dims[j + 1], h->b[l][j], relu, h->status), st);
    else if (h->tc_mlp)
      s = run_gemm_tc<MODE_MLP, T, T>(dv, h->mlp_maps[l][j],
                                       mlp_params(batch, h->dims[j], h->dims[j + 1], h->b[l][j], relu, h->status), st);
    else
      s = run_gemm_simt<T, T>(static_cast<const T*>(in), static_cast<const T*>(h->W[l][j]), h->b[l][j],
                              static_cast<T*>(o), batch, h->dims[j], h->dims[j + 1], ldc, relu, st);
  }
  if (s != WK_OK) return s;
  {  // 3. LCB
    ProfScope ps(h, WK_KERNEL_LCB, st);
    if (h->tc_lcb) {
      GemmMaps mp;
      mp.A = h->lcbA[l];
      mp.B = lcb_x;
      mp.C = h->lcbC;
      s = run_lcb_tc<T, T>(dv, mp, lcb_params(batch, n, d, c.n_l, h->status), st);
    } else {
      s = run_lcb_simt<T, T>(static_cast<const T*>(h->WL[l]), xin, static_cast<T*>(h->cat), batch, n, d, c.n_f,
                             c.n_l, st);
    }
  }
  return s;
}

// The forward of a 16-bit stack through the one-kernel layer front (front_tc.cuh). Per
// layer l: the front reads the previous layer's output before its LayerNorm (the caller's
// X for l = 0), writes A0 and the layer output's LCB rows and FMB-row residual into
// Xs[l % 2]; the MLP runs on A0 and its last Linear adds its output into those FMB rows.
// The stack's output is the last layer's output LayerNorm of Xs[(L - 1) % 2].
template <typename T, typename IO, typename OUT>
wk_status forward16_front(wk_stack* h, const void* X, void* out, int64_t batch, cudaStream_t st) {
  const wk_stack_config& c = h->cfg;
  const DevInfo* dv = h->dv;
  const int n = c.n, d = c.d, m = c.mlp_num_linear, L = c.num_layers;
  wk_status s = WK_OK;
  for (int l = 0; l < L && s == WK_OK; ++l) {
    const int o = l % 2;
    FrontMaps fm = h->fmaps[l];
    fm.R = h->frontR[o];
    fm.L = h->frontL[o];
    {
      ProfScope ps(h, WK_KERNEL_FRONT, st);
      if (l == 0)
        s = run_front<IO, T>(dv, h->front, fm, static_cast<const IO*>(X), nullptr, nullptr, h->g1[l], h->b1[l],
                             static_cast<T*>(h->A0), static_cast<T*>(h->Xs[o]), batch, h->eps, h->status, st);
      else
        s = run_front<T, T>(dv, h->front, fm, static_cast<const T*>(h->Xs[(l - 1) % 2]), h->g2[l - 1], h->b2[l - 1],
                            h->g1[l], h->b1[l], static_cast<T*>(h->A0), static_cast<T*>(h->Xs[o]), batch, h->eps,
                            h->status, st);
    }
    for (int j = 0; j < m && s == WK_OK; ++j) {
      ProfScope ps(h, WK_KERNEL_MLP_GEMM, st);
      const bool lastj = j == m - 1;
      GemmMaps mp = h->mlp_maps[l][j];
      if (lastj) mp.C = h->frontC[o];
      if (h->pair) {
        GemmParams p = mlp2_params(batch, h->dims[j], h->dims[j + 1], h->b[l][j], lastj ? 0 : 1, h->status);
        p.reduce_out = lastj ? 1 : 0;
        s = run_gemm_tc2<T, T>(dv, mp, p, st);
      } else {
        GemmParams p = mlp_params(batch, h->dims[j], h->dims[j + 1], h->b[l][j], lastj ? 0 : 1, h->status);
        p.reduce_out = lastj ? 1 : 0;
        s = run_gemm_tc<MODE_MLP, T, T>(dv, mp, p, st);
      }
    }
  }
  if (s != WK_OK) return s;
  ProfScope ps(h, WK_KERNEL_RES_LN, st);
  return run_res_ln<T, T, OUT>(dv, static_cast<const T*>(h->Xs[(L - 1) % 2]), static_cast<const T*>(nullptr),
                               h->g2[L - 1], h->b2[L - 1], static_cast<OUT*>(out), batch * n, d, h->eps, h->status, st);
}

// The forward of a 16-bit stack with operand type T, input type IO and output type
// OUT (the caller's type, or T when the prediction head reads the output).
template <typename T, typename IO, typename OUT = IO>
wk_status forward16(wk_stack* h, const void* X, void* out, int64_t batch, cudaStream_t st) {
  constexpr bool kFrontTypes = std::is_same<T, f16>::value;
  if constexpr (kFrontTypes) {
    if (h->front >= 0) return forward16_front<T, IO, OUT>(h, X, out, batch, st);
  }
  const wk_stack_config& c = h->cfg;
  const DevInfo* dv = h->dv;
  const int n = c.n, d = c.d, L = c.num_layers;
  const int64_t rows = batch * n;
  wk_status s = WK_OK;
  const void* x0 = X;
  CUtensorMap lcb_x0;
  if (sizeof(IO) != sizeof(T) || Half16<IO>::kBF16 != Half16<T>::kBF16) {
    ProfScope ps(h, WK_KERNEL_CONVERT, st);
    s = run_convert<IO, T>(dv, X, h->Xs[1], rows * d, st);  // the input in the operand type
    if (s != WK_OK) return s;
    x0 = h->Xs[1];
    lcb_x0 = h->lcbB_ws[1];
  } else if (h->tc_lcb && !map_lcb_x<T>(dv, &lcb_x0, X, n, d, batch)) {
    return WK_ERR_CUDA;
  }
  for (int l = 0; l < L && s == WK_OK; ++l) {
    const bool last = l == L - 1;
    const T* xin = static_cast<const T*>(l == 0 ? x0 : h->Xs[(l - 1) % 2]);
    s = layer_front16<T>(h, l, xin, (l == 0) ? lcb_x0 : h->lcbB_ws[(l - 1) % 2], batch, st);
    if (s != WK_OK) break;
    {  // 4. residual + LN
      ProfScope ps(h, WK_KERNEL_RES_LN, st);
      const T* cat = static_cast<const T*>(h->cat);
      if (last)
        s = run_res_ln<T, T, OUT>(dv, cat, xin, h->g2[l], h->b2[l], static_cast<OUT*>(out), rows, d, h->eps,
                                 h->status, st);
      else
        s = run_res_ln<T, T, T>(dv, cat, xin, h->g2[l], h->b2[l], static_cast<T*>(h->Xs[l % 2]), rows, d, h->eps,
                               h->status, st);
    }
  }
  return s;
}

wk_status forward32(wk_stack* h, const float* X, float* out, int64_t batch, cudaStream_t st) {
  const wk_stack_config& c = h->cfg;
  const DevInfo* dv = h->dv;
  const int n = c.n, d = c.d, k = c.k, m = c.mlp_num_linear, L = c.num_layers;
  const int64_t rows = batch * n;
  const size_t nd = static_cast<size_t>(n) * d;
  wk_status s = WK_OK;
  for (int l = 0; l < L && s == WK_OK; ++l) {
    const bool last = l == L - 1;
    const float* xin = (l == 0) ? X : static_cast<const float*>(h->Xs[(l - 1) % 2]);
    {
      ProfScope ps(h, WK_KERNEL_FM_LN, st);
      s = run_fm_simt<float>(dv, xin, static_cast<const float*>(h->Y[l]), h->g1[l], h->b1[l],
                             static_cast<float*>(h->A0), batch, n, d, k, h->eps, st);
    }
    for (int j = 0; j < m && s == WK_OK; ++j) {
      ProfScope ps(h, WK_KERNEL_MLP_GEMM, st);
      const void* in = (j == 0) ? h->A0 : h->H[(j - 1) % 2];
      const bool lastj = j == m - 1;
      void* o = lastj ? h->cat : h->H[j % 2];
      const int64_t ldc = lastj ? static_cast<int64_t>(nd) : h->dims[j + 1];
      s = run_gemm_simt<float, float>(static_cast<const float*>(in), static_cast<const float*>(h->W[l][j]), h->b[l][j],
                                      static_cast<float*>(o), batch, h->dims[j], h->dims[j + 1], ldc, lastj ? 0 : 1, st);
    }
    if (s != WK_OK) break;
    {
      ProfScope ps(h, WK_KERNEL_LCB, st);
      s = run_lcb_simt<float, float>(static_cast<const float*>(h->WL[l]), xin, static_cast<float*>(h->cat), batch, n,
                                     d, c.n_f, c.n_l, st);
    }
    if (s != WK_OK) break;
    {
      ProfScope ps(h, WK_KERNEL_RES_LN, st);
      float* o = last ? out : static_cast<float*>(h->Xs[l % 2]);
      s = run_res_ln<float, float, float>(dv, static_cast<const float*>(h->cat), xin, h->g2[l], h->b2[l], o, rows, d,
                                          h->eps, h->status, st);
    }
  }
  return s;
}

// Stack forward into the operand-type layer buffer, then the prediction head: the
// hidden Linears on the tensor-core GEMM (ReLU), the one-output Linear and sigmoid.
template <typename T, typename IO>
wk_status predict16(wk_stack* h, const void* X, float* logit, float* prob, int64_t batch, cudaStream_t st) {
  const DevInfo* dv = h->dv;
  const int L = h->cfg.num_layers;
  void* xl = h->Xs[(L - 1) % 2];
  wk_status s = forward16<T, IO, T>(h, X, xl, batch, st);
  if (s != WK_OK) return s;
  const std::vector<int32_t>& dims = h->head_dims;
  const int q = static_cast<int>(dims.size()) - 1;
  const void* z = xl;
  for (int j = 0; j + 1 < q && s == WK_OK; ++j) {
    ProfScope ps(h, WK_KERNEL_HEAD, st);
    if (h->head_maps.empty())
      s = run_gemm_simt<T, T>(static_cast<const T*>(z), static_cast<const T*>(h->hT[j]), h->hc[j],
                              static_cast<T*>(h->HH[j % 2]), batch, dims[j], dims[j + 1], dims[j + 1], 1, st);
    else if (h->pair)
      s = run_gemm_tc2<T, T>(dv, h->head_maps[j], mlp2_params(batch, dims[j], dims[j + 1], h->hc[j], 1, h->status),
                             st);
    else
      s = run_gemm_tc<MODE_MLP, T, T>(dv, h->head_maps[j],
                                       mlp_params(batch, dims[j], dims[j + 1], h->hc[j], 1, h->status), st);
    z = h->HH[j % 2];
  }
  if (s != WK_OK) return s;
  ProfScope ps(h, WK_KERNEL_HEAD, st);
  return run_head_out<T>(dv, static_cast<const T*>(z), static_cast<const T*>(h->hT[q - 1]), h->hc[q - 1], logit, prob,
                         batch, dims[q - 1], st);
}

template <typename T>
wk_status build_head_maps(wk_stack* h) {
  const std::vector<int32_t>& dims = h->head_dims;
  const int q = static_cast<int>(dims.size()) - 1;
  const int64_t B = h->maxb;
  h->head_maps.clear();
  bool tc = true;
  for (int j = 0; j + 1 < q; ++j) tc = tc && mlp_tc_ok(B, dims[j], dims[j + 1], dims[j + 1]);
  if (!tc || q < 2) return WK_OK;
  h->head_maps.resize(q - 1);
  const void* xl = h->Xs[(h->cfg.num_layers - 1) % 2];
  for (int j = 0; j + 1 < q; ++j) {
    GemmMaps& mp = h->head_maps[j];
    const void* in = (j == 0) ? xl : h->HH[(j - 1) % 2];
    if (!map_kmajor<T>(h->dv, &mp.A, in, dims[j], B, GEMM_BM) ||
        !map_kmajor<T>(h->dv, &mp.B, h->hT[j], dims[j], dims[j + 1], h->pair ? 128 : GEMM_BN) ||
        !map_out<T>(h->dv, &mp.C, h->HH[j % 2], dims[j + 1], B, dims[j + 1]))
      return WK_ERR_UNSUPPORTED;
  }
  return WK_OK;
}

// The forward of a MoE stack with operand type T and caller type IO.
template <typename T, typename IO>
wk_status moe_forward16(wk_moe* h, const void* X, void* out, int64_t batch, cudaStream_t st) {
  const wk_stack_config& c = h->cfg;
  const DevInfo* dv = h->dv;
  const int n = c.n, d = c.d, L = c.num_layers, E = h->E;
  const int64_t rows = batch * n;
  const int64_t nd = static_cast<int64_t>(n) * d;
  wk_stack* p0 = h->ex[0];  // carries the MoE's own profiling records
  wk_status s = WK_OK;
  const void* x0 = X;
  CUtensorMap lcb_x0;
  if (sizeof(IO) != sizeof(T) || Half16<IO>::kBF16 != Half16<T>::kBF16) {
    ProfScope ps(p0, WK_KERNEL_CONVERT, st);
    s = run_convert<IO, T>(dv, X, h->Xm[1], rows * d, st);
    if (s != WK_OK) return s;
    x0 = h->Xm[1];
    lcb_x0 = h->lcbX[1];
  } else if (p0->tc_lcb && !map_lcb_x<T>(dv, &lcb_x0, X, n, d, batch)) {
    return WK_ERR_CUDA;
  }
  for (int l = 0; l < L && s == WK_OK; ++l) {
    const bool last = l == L - 1;
    const T* xin = static_cast<const T*>(l == 0 ? x0 : h->Xm[(l - 1) % 2]);
    const CUtensorMap& xmap = (l == 0) ? lcb_x0 : h->lcbX[(l - 1) % 2];
    {
      ProfScope ps(p0, WK_KERNEL_MOE_GATE, st);
      s = run_moe_gate<T>(dv, xin, static_cast<const T*>(h->Wg[l]), h->bg[l], h->g, batch, nd, E, st);
    }
    for (int e = 0; e < E && s == WK_OK; ++e) s = layer_front16<T>(h->ex[e], l, xin, xmap, batch, st);
    if (s != WK_OK) break;
    MoePtrs mp{};
    for (int e = 0; e < E; ++e) {
      mp.cat[e] = h->ex[e]->cat;
      mp.gamma[e] = h->ex[e]->g2[l];
      mp.beta[e] = h->ex[e]->b2[l];
    }
    ProfScope ps(p0, WK_KERNEL_MOE_COMBINE, st);
    if (last)
      s = run_moe_combine<T, IO>(dv, mp, xin, h->g, static_cast<IO*>(out), rows, n, d, E, h->eps, p0->status, st);
    else
      s = run_moe_combine<T, T>(dv, mp, xin, h->g, static_cast<T*>(h->Xm[l % 2]), rows, n, d, E, h->eps, p0->status,
                                st);
  }
  return s;
}

void free_moe(wk_moe* h) {
  if (!h) return;
  cudaDeviceSynchronize();
  cudaGetLastError();
  for (wk_stack* e : h->ex) free_stack(e);
  if (h->ws) cudaFree(h->ws);
  if (h->wcopy) cudaFree(h->wcopy);
  cudaGetLastError();
  delete h;
}

// ---------------------------------------------------------------- backward

// A term of a tensor-core contraction, strides set by the caller.
TcTerm tc_term(const float* A, const float* B, int K1, int K2) {
  TcTerm t{};
  t.A = A;
  t.B = B;
  t.K1 = K1;
  t.K2 = K2;
  return t;
}

TcContr tc_contr(int M, int N, int Z, int S, int mode, float* C, int64_t sCz, int64_t sCm, int64_t sCn) {
  TcContr p{};
  p.M = M;
  p.N = N;
  p.Z = Z;
  p.S = S;
  p.mode = mode;
  p.C = C;
  p.sCz = sCz;
  p.sCm = sCm;
  p.sCn = sCn;
  return p;
}

int tc_bn(int N) { return N <= 64 ? 64 : N <= 128 ? 128 : N <= 160 ? 160 : 128; }

// The 4-D TMA tensor of one fp32 operand with `rows` rows (m or n), K2 x K1 values of k and
// Z of z; strides in elements. K-major where k2 is contiguous (dims k2, row, k1, z; box 32 x
// box_rows, 128-byte swizzle), else MN-major where the row index is (dims row, k2, k1, z; box
// 32 x 32, 128-byte swizzle with 32-byte atoms). A stride of 0 along z (an operand shared by
// every z) becomes a dimension of size 1 read at coordinate 0.
bool tc_map(const DevInfo* dv, CUtensorMap* m, const float* ptr, int64_t rows, int64_t K2, int64_t K1, int64_t Z,
            int64_t s_row, int64_t s_k2, int64_t s_k1, int64_t s_z, uint32_t box_rows, int* mn, int* z0) {
  if (reinterpret_cast<uintptr_t>(ptr) % 16 != 0) return false;
  *z0 = s_z == 0 ? 1 : 0;
  uint64_t dims[4], str[3];
  uint32_t box[4] = {32, box_rows, 1, 1};
  CUtensorMapSwizzle sw = CU_TENSOR_MAP_SWIZZLE_128B;
  if (s_k2 == 1) {
    *mn = 0;
    dims[0] = K2, dims[1] = rows, str[0] = s_row * 4;
  } else if (s_row == 1) {
    *mn = 1;
    dims[0] = rows, dims[1] = K2, str[0] = s_k2 * 4;
    box[1] = 32;
    sw = CU_TENSOR_MAP_SWIZZLE_128B_ATOM_32B;
  } else {
    return false;
  }
  dims[2] = K1, dims[3] = *z0 ? 1 : Z;
  str[1] = K1 > 1 ? s_k1 * 4 : str[0] * dims[1];  // a size-1 dimension takes any valid stride
  str[2] = dims[3] > 1 ? s_z * 4 : str[1] * dims[2];
  for (int i = 0; i < 3; ++i)
    if (str[i] == 0 || str[i] % 16 != 0 || str[i] >= (1ull << 40)) return false;
  return make_map(dv, m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, ptr, dims, str, box, sw);
}

template <int BN, bool CIN>
wk_status launch_tc_contract(const DevInfo* dv, const TcMaps& mp, const TcContr& p, cudaStream_t st) {
  using Cfg = TcCfg<BN, CIN>;
  wk_status s = smem_attr(dv, reinterpret_cast<const void*>(bw_tc_contract_kernel<BN, CIN>), Cfg::SMEM);
  if (s != WK_OK) return s;
  const int grid = std::min(p.num_tiles, dv->sms);
  bw_tc_contract_kernel<BN, CIN><<<grid, TC_THREADS, Cfg::SMEM, st>>>(mp, p);
  return launch_status();
}

template <int BN>
wk_status launch_tc_contract(const DevInfo* dv, const TcMaps& mp, const TcContr& p, bool cin, cudaStream_t st) {
  return cin ? launch_tc_contract<BN, true>(dv, mp, p, st) : launch_tc_contract<BN, false>(dv, mp, p, st);
}

// The strided contraction on the tensor cores (tf32 operands, fp32 accumulation).
wk_status run_tc_contract(wk_stack* h, TcContr p, cudaStream_t st) {
  if (p.M <= 0 || p.N <= 0 || p.Z <= 0 || p.nterms <= 0) return WK_OK;
  if (p.nterms > 3 || p.S < 1 || (p.S > 1 && p.mode != TC_ATOMIC)) return WK_ERR_UNSUPPORTED;
  const int bn = tc_bn(p.N);
  TcMaps mp;
  for (int t = 0; t < p.nterms; ++t) {
    TcTerm& q = p.t[t];
    if (q.K1 < p.S || q.K2 < 1) return WK_ERR_UNSUPPORTED;  // every split of every term has a k1
    if (!tc_map(h->dv, &mp.m[2 * t], q.A, p.M, q.K2, q.K1, p.Z, q.sAm, q.sAk2, q.sAk1, q.sAz, 128, &q.a_mn, &q.a_z0) ||
        !tc_map(h->dv, &mp.m[2 * t + 1], q.B, p.N, q.K2, q.K1, p.Z, q.sBn, q.sBk2, q.sBk1, q.sBz,
                static_cast<uint32_t>(bn), &q.b_mn, &q.b_z0))
      return WK_ERR_UNSUPPORTED;
    q.k1q = q.K1 / p.S;
    q.k1r = q.K1 % p.S;
    q.nk2 = (q.K2 + TC_BK - 1) / TC_BK;
  }
  p.mt = (p.M + 127) / 128;
  p.nt = (p.N + bn - 1) / bn;
  const int64_t tiles = static_cast<int64_t>(p.Z) * p.S * p.mt * p.nt;
  if (tiles > 0x7FFFFFFFll) return WK_ERR_UNSUPPORTED;
  p.num_tiles = static_cast<int>(tiles);
  p.c_vec = p.sCn == 1 && reinterpret_cast<uintptr_t>(p.C) % 16 == 0 && p.sCm % 4 == 0 && p.sCz % 4 == 0;
  p.status = h->status;
  // C read by a TMA prefetch of each tile (accumulating launches): C [Z][M][N] with the
  // 128B-swizzled boxes of 32 columns x 128 rows the epilogue reads
  bool cin = false;
  if (p.mode == TC_ACCUM && p.c_vec) {
    const uint64_t dims[3] = {static_cast<uint64_t>(p.N), static_cast<uint64_t>(p.M), static_cast<uint64_t>(p.Z)};
    const uint64_t str[2] = {static_cast<uint64_t>(p.sCm) * 4,
                             p.Z > 1 ? static_cast<uint64_t>(p.sCz) * 4 : static_cast<uint64_t>(p.sCm) * 4 * p.M};
    const uint32_t box[3] = {32, 128, 1};
    cin = str[0] > 0 && str[1] > 0 && str[1] % 16 == 0 &&
          make_map(h->dv, &mp.m[6], CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, p.C, dims, str, box, CU_TENSOR_MAP_SWIZZLE_128B);
  }
  ProfScope ps(h, WK_KERNEL_BW_CONTRACT, st);
  switch (bn) {
    case 64: return launch_tc_contract<64>(h->dv, mp, p, cin, st);
    case 160: return launch_tc_contract<160>(h->dv, mp, p, cin, st);
    default: return launch_tc_contract<128>(h->dv, mp, p, cin, st);
  }
}

// Splits of the k1 range so that a launch has one tile per SM (rounded down: an SM with a
// second tile would double the launch's time).
int tc_splits(const DevInfo* dv, int M, int N, int K1) {
  const int bn = tc_bn(N);
  const int tiles = ((M + 127) / 128) * ((N + bn - 1) / bn);
  return std::max(1, std::min(K1, dv->sms / tiles));
}

template <typename T>
wk_status to_f32(wk_stack* h, const void* in, float* out, int64_t n, cudaStream_t st) {
  if (n <= 0) return WK_OK;
  ProfScope ps(h, WK_KERNEL_BW_ROWS, st);
  const int grid = static_cast<int>(std::min<int64_t>((n + 255) / 256, h->dv->sms * 16ll));
  bw_to_f32_kernel<T><<<grid, 256, 0, st>>>(static_cast<const T*>(in), out, n);
  return launch_status();
}

// C [M, N] = A [M, K] W [N, K]^T on the tensor cores (16-bit K-major operands, TO output).
template <typename T, typename TO>
wk_status bw_gemm(wk_stack* h, const void* A, const void* W, void* C, int64_t M, int K, int N, cudaStream_t st) {
  const DevInfo* dv = h->dv;
  if (!mlp_tc_ok(M, K, N, N)) return WK_ERR_UNSUPPORTED;
  const bool pair = use_pair_gemm(M);
  GemmMaps mp;
  if (!map_kmajor<T>(dv, &mp.A, A, K, M, GEMM_BM) || !map_kmajor<T>(dv, &mp.B, W, K, N, pair ? 128 : GEMM_BN) ||
      !map_out<TO>(dv, &mp.C, C, N, M, N))
    return WK_ERR_UNSUPPORTED;
  ProfScope ps(h, WK_KERNEL_MLP_GEMM, st);
  if (pair) return run_gemm_tc2<T, TO>(dv, mp, mlp2_params(M, K, N, nullptr, 0, h->status), st);
  return run_gemm_tc<MODE_MLP, T, TO>(dv, mp, mlp_params(M, K, N, nullptr, 0, h->status), st);
}

// C [M, N] = A [M, K] W [N, K]^T on the CTA-pair GEMM with A (A_MN) and W (B_MN) given as
// their transposes A^T [K, M], W^T [K, N] (row strides lda, ldb) and read MN-major.
template <typename T, typename TO, bool A_MN, bool B_MN>
wk_status bw_gemm_mn(wk_stack* h, const void* A, int64_t lda, const void* W, int64_t ldb, void* C, int64_t M, int K,
                     int N, cudaStream_t st) {
  const DevInfo* dv = h->dv;
  if (!mlp_tc_ok(M, K, N, N) || (A_MN && lda % 8 != 0) || (B_MN && ldb % 8 != 0)) return WK_ERR_UNSUPPORTED;
  GemmMaps mp;
  const bool ok = (A_MN ? map_mnmajor<T>(dv, &mp.A, A, K, M, lda) : map_kmajor<T>(dv, &mp.A, A, K, M, GEMM_BM)) &&
                  (B_MN ? map_mnmajor<T>(dv, &mp.B, W, K, N, ldb) : map_kmajor<T>(dv, &mp.B, W, K, N, 128)) &&
                  map_out<TO>(dv, &mp.C, C, N, M, N);
  if (!ok) return WK_ERR_UNSUPPORTED;
  ProfScope ps(h, WK_KERNEL_MLP_GEMM, st);
  // The weight gradient (K = the batch, fp32 tiles) runs persistent: its two TMEM accumulators
  // overlap a tile's epilogue with the next tile's main loop, which a short K leaves exposed in
  // the streaming shape's one accumulator.
  return run_gemm_tc2<T, TO, A_MN, B_MN>(dv, mp, mlp2_params(M, K, N, nullptr, 0, h->status), st, !(A_MN && B_MN));
}

template <typename T>
wk_status bw_transpose(wk_stack* h, const void* in, void* out, int64_t R, int64_t C, cudaStream_t st) {
  ProfScope ps(h, WK_KERNEL_BW_ROWS, st);
  const dim3 grid(static_cast<unsigned>((C + 31) / 32), static_cast<unsigned>((R + 31) / 32));
  bw_transpose_kernel<T><<<grid, dim3(32, 8), 0, st>>>(static_cast<const T*>(in), static_cast<T*>(out), R, C);
  return launch_status();
}

// The backward of a 16-bit stack with fp16 operands (the folded first Linear). X (IO) is
// the stack's input, dOut / dX fp32 [batch, n, d]. The forward is run once with every
// layer's input saved; each layer's front is then recomputed from its saved input
// (A0 = LN(F) normalised, the hidden activations, the concat buffer) before its backward.
template <typename T, typename IO>
wk_status backward16(wk_stack* h, const void* X, const float* dOut, float* dX, const wk_layer_grads* gr,
                     int64_t batch, cudaStream_t st, void* const* layer_done) {
  const wk_stack_config& c = h->cfg;
  const DevInfo* dv = h->dv;
  const int n = c.n, d = c.d, k = c.k, m = c.mlp_num_linear, L = c.num_layers, n_f = c.n_f, n_l = c.n_l;
  const int64_t B = batch, rows = B * n;
  const size_t nd = static_cast<size_t>(n) * d, nk = static_cast<size_t>(n) * k;
  const std::vector<int32_t>& dims = h->dims;
  int64_t hmax = 0, wmax = 0;
  for (int j = 0; j <= m; ++j) hmax = std::max<int64_t>(hmax, dims[j]);
  for (int j = 0; j < m; ++j) wmax = std::max<int64_t>(wmax, static_cast<int64_t>(dims[j]) * dims[j + 1]);
  auto up = [](size_t v) { return (v + 255) & ~static_cast<size_t>(255); };
  // the MLP gradient GEMMs read their operands MN-major on the pair kernel; the one-CTA
  // kernel (batch or a hidden width of at most 128) needs transposed copies
  bool transposes = !use_pair_gemm(B);
  for (int j = 0; j < m; ++j) transposes = transposes || !use_pair_gemm(dims[j + 1]);
  // workspace: saved layer inputs; the saved activations of every layer but the last (its
  // FMB LayerNorm output A0, the hidden ReLU outputs, the concat buffer); fp32 dy and two dX
  // buffers; two 16-bit MLP gradients; the transposes if needed; the FM's Z, dZ, F and dF;
  // fp32 copies of X, W_L and Y
  const size_t b_sv = up(B * nd * 2), b_f = up(B * nd * 4), b_h = up(B * hmax * 2), b_w = up(wmax * 2),
               b_z = up(B * static_cast<size_t>(d) * k * 4), b_fk = up(B * nk * 4),
               b_wl = up(static_cast<size_t>(n_l) * n * 4), b_y = up(nk * 4);
  size_t b_act = up(B * static_cast<size_t>(dims[0]) * 2) + b_sv;
  for (int j = 0; j + 1 < m; ++j) b_act += up(B * static_cast<size_t>(dims[j + 1]) * 2);
  const size_t need = L * b_sv + (L - 1) * b_act + 4 * b_f + 2 * b_h + (transposes ? 2 * b_h + b_w : 0) + 2 * b_z +
                      2 * b_fk + b_wl + b_y;
  if (h->bws_bytes < need) {
    if (h->bws) cudaFree(h->bws);
    h->bws = nullptr;
    h->bws_bytes = 0;
    if (cudaMalloc(&h->bws, need) != cudaSuccess) {
      cudaGetLastError();
      return WK_ERR_OOM;
    }
    h->bws_bytes = need;
  }
  uint8_t* p = h->bws;
  std::vector<T*> xs(L);
  for (int l = 0; l < L; ++l, p += b_sv) xs[l] = reinterpret_cast<T*>(p);
  struct Acts {
    const void* A0;
    const void* H[2];
    const void* cat;
  };
  std::vector<Acts> acts(L);  // layer L - 1 keeps its activations in the stack's buffers
  acts[L - 1] = Acts{h->A0, {h->H[0], h->H[1]}, h->cat};
  for (int l = 0; l + 1 < L; ++l) {
    acts[l].A0 = p;
    p += up(B * static_cast<size_t>(dims[0]) * 2);
    for (int j = 0; j + 1 < m; ++j) {
      acts[l].H[j] = p;
      p += up(B * static_cast<size_t>(dims[j + 1]) * 2);
    }
    acts[l].cat = p;
    p += b_sv;
  }
  float* dyf = reinterpret_cast<float*>(p);
  p += b_f;
  float* gx[2] = {reinterpret_cast<float*>(p), reinterpret_cast<float*>(p + b_f)};
  p += 2 * b_f;
  T* dz[2] = {reinterpret_cast<T*>(p), reinterpret_cast<T*>(p + b_h)};
  p += 2 * b_h;
  T* dzT = transposes ? reinterpret_cast<T*>(p) : nullptr;
  T* hT = transposes ? reinterpret_cast<T*>(p + b_h) : nullptr;
  T* wT = transposes ? reinterpret_cast<T*>(p + 2 * b_h) : nullptr;
  if (transposes) p += 2 * b_h + b_w;
  float* Zb = reinterpret_cast<float*>(p);
  float* dZb = reinterpret_cast<float*>(p + b_z);
  p += 2 * b_z;
  float* Fb = reinterpret_cast<float*>(p);
  float* dFb = reinterpret_cast<float*>(p + b_fk);
  p += 2 * b_fk;
  float* Xf = reinterpret_cast<float*>(p);  // fp32 copies of the layer's X, W_L and Y
  float* WLf = reinterpret_cast<float*>(p + b_f);
  float* Yf = reinterpret_cast<float*>(p + b_f + b_wl);

  wk_status s = WK_OK;
  // 1. the forward, saving each layer's input and activations
  if (sizeof(IO) != sizeof(T) || Half16<IO>::kBF16 != Half16<T>::kBF16)
    s = run_convert<IO, T>(dv, X, xs[0], rows * d, st);
  else if (cudaMemcpyAsync(xs[0], X, B * nd * 2, cudaMemcpyDeviceToDevice, st) != cudaSuccess)
    s = WK_ERR_CUDA;
  std::vector<CUtensorMap> lcbx(L);
  for (int l = 0; l < L && s == WK_OK; ++l)
    if (h->tc_lcb && !map_lcb_x<T>(dv, &lcbx[l], xs[l], n, d, B)) s = WK_ERR_CUDA;
  auto save = [&](const void* src, const void* dst, size_t bytes) {
    if (s == WK_OK &&
        cudaMemcpyAsync(const_cast<void*>(dst), src, bytes, cudaMemcpyDeviceToDevice, st) != cudaSuccess)
      s = WK_ERR_CUDA;
  };
  for (int l = 0; l + 1 < L && s == WK_OK; ++l) {
    s = layer_front16<T>(h, l, xs[l], lcbx[l], B, st);
    save(h->A0, acts[l].A0, B * static_cast<size_t>(dims[0]) * 2);
    for (int j = 0; j + 1 < m; ++j) save(h->H[j % 2], acts[l].H[j], B * static_cast<size_t>(dims[j + 1]) * 2);
    save(h->cat, acts[l].cat, B * nd * 2);
    if (s == WK_OK)
      s = run_res_ln<T, T, T>(dv, static_cast<const T*>(h->cat), xs[l], h->g2[l], h->b2[l], xs[l + 1], rows, d, h->eps,
                              h->status, st);
  }
  // 2. the layers' backwards, last layer first
  for (int l = L - 1; l >= 0 && s == WK_OK; --l) {
    const wk_layer_grads& g = gr[l];
    const T* xin = xs[l];
    const float* up_grad = (l == L - 1) ? dOut : gx[(l + 1) % 2];
    float* dxl = (l == 0) ? dX : gx[l % 2];
    if (l == L - 1) s = layer_front16<T>(h, l, xin, lcbx[l], B, st);  // the others were saved
    const Acts& act = acts[l];
    if (s == WK_OK) s = to_f32<T>(h, xin, Xf, B * static_cast<int64_t>(nd), st);
    if (s == WK_OK) s = to_f32<T>(h, h->WL[l], WLf, static_cast<int64_t>(n_l) * n, st);
    if (s == WK_OK) s = to_f32<T>(h, h->Y[l], Yf, static_cast<int64_t>(nk), st);
    if (s != WK_OK) break;
    cudaMemsetAsync(g.out_ln_gamma, 0, d * 4, st);
    cudaMemsetAsync(g.out_ln_beta, 0, d * 4, st);
    cudaMemsetAsync(g.W_L, 0, static_cast<size_t>(n_l) * n * 4, st);
    cudaMemsetAsync(g.Y, 0, nk * 4, st);
    cudaMemsetAsync(g.fmb_ln_gamma, 0, nk * 4, st);
    cudaMemsetAsync(g.fmb_ln_beta, 0, nk * 4, st);
    for (int j = 0; j < m; ++j) cudaMemsetAsync(g.b[j], 0, static_cast<size_t>(dims[j + 1]) * 4, st);
    // output LayerNorm, residual: dy, dX = dy, the FMB rows of dy as the MLP's gradient
    {
      const int grid = static_cast<int>(std::min<int64_t>((rows + 7) / 8, dv->sms * 4ll));
      ProfScope ps(h, WK_KERNEL_BW_ROWS, st);
      bw_out_ln_kernel<T><<<grid, 256, 0, st>>>(static_cast<const T*>(act.cat), xin, up_grad, h->g2[l], dyf, dxl, dz[0],
                                                 g.out_ln_gamma, g.out_ln_beta, static_cast<int>(rows), n, n_f, d,
                                                 h->eps);
      s = launch_status();
    }
    // LCB: dW_L = sum_b dG_b X_b^T (dG = rows n_f.. of dy; W_L^T dG_b joins dX below)
    const float* dG = dyf + static_cast<size_t>(n_f) * d;
    if (s == WK_OK) {
      TcContr p = tc_contr(n_l, n, 1, tc_splits(dv, n_l, n, static_cast<int>(B)), TC_ATOMIC, g.W_L, 0, n, 1);
      p.nterms = 1;
      p.t[0] = tc_term(dG, Xf, static_cast<int>(B), d);
      p.t[0].sAm = d, p.t[0].sAk1 = nd, p.t[0].sAk2 = 1;  // dG(b, r, t)
      p.t[0].sBn = d, p.t[0].sBk1 = nd, p.t[0].sBk2 = 1;  // X(b, i, t)
      s = run_tc_contract(h, p, st);
    }
    // FMB MLP, last Linear first: dz (16-bit) -> bias, weight and input gradients
    int cur = 0;
    for (int j = m - 1; j >= 0 && s == WK_OK; --j) {
      const int64_t hin = dims[j], hout = dims[j + 1];
      const void* hj = (j == 0) ? act.A0 : act.H[j - 1];
      // the ReLU of Linear j (j < m - 1: its output h_{j+1} was > 0) applied to dz, then the
      // bias gradient (column sums over the batch), in one pass
      const T* relu_out = (j < m - 1) ? static_cast<const T*>(act.H[j]) : nullptr;
      if (hout % 8 == 0) {
        const unsigned gx = static_cast<unsigned>((hout + 2047) / 2048);
        // at most 64 row chunks: every chunk adds into each column of the bias gradient
        const unsigned gy = static_cast<unsigned>(std::max<int64_t>(1, std::min<int64_t>({B, 64ll, 4ll * dv->sms / gx})));
        ProfScope ps(h, WK_KERNEL_BW_ROWS, st);
        bw_mask_colsum_kernel<T><<<dim3(gx, gy), 256, 0, st>>>(dz[cur], relu_out, g.b[j], B, static_cast<int>(hout));
        s = launch_status();
      } else {
        if (relu_out) {
          const int64_t cnt = B * hout;
          const int grid = static_cast<int>(std::min<int64_t>((cnt / 8 + 255) / 256, dv->sms * 16ll));
          ProfScope ps(h, WK_KERNEL_BW_ROWS, st);
          bw_relu_mask_kernel<T><<<grid, 256, 0, st>>>(dz[cur], relu_out, cnt);
          s = launch_status();
        }
        if (s == WK_OK) {
          const dim3 grid(static_cast<unsigned>((hout + 255) / 256), static_cast<unsigned>(std::min<int64_t>(B, 64)));
          ProfScope ps(h, WK_KERNEL_BW_ROWS, st);
          bw_colsum_kernel<T><<<grid, 256, 0, st>>>(dz[cur], g.b[j], B, static_cast<int>(hout));
          s = launch_status();
        }
      }
      // dW_j = dz^T h_j (K = batch): on the pair GEMM both read MN-major, else transposed
      // to K-major for the one-CTA GEMM
      if (s == WK_OK && use_pair_gemm(hout)) {
        s = bw_gemm_mn<T, float, true, true>(h, dz[cur], hout, hj, hin, g.W[j], hout, static_cast<int>(B),
                                             static_cast<int>(hin), st);
      } else if (s == WK_OK) {
        s = bw_transpose<T>(h, dz[cur], dzT, B, hout, st);
        if (s == WK_OK) s = bw_transpose<T>(h, hj, hT, B, hin, st);
        if (s == WK_OK)
          s = bw_gemm<T, float>(h, dzT, hT, g.W[j], hout, static_cast<int>(B), static_cast<int>(hin), st);
      }
      // dh_j = dz W_j: W_j (= (W_j^T)^T) read MN-major on the pair GEMM, else transposed
      if (s == WK_OK && use_pair_gemm(B)) {
        s = bw_gemm_mn<T, T, false, true>(h, dz[cur], 0, h->W[l][j], hin, dz[1 - cur], B, static_cast<int>(hout),
                                          static_cast<int>(hin), st);
      } else if (s == WK_OK) {
        s = bw_transpose<T>(h, h->W[l][j], wT, hout, hin, st);
        if (s == WK_OK)
          s = bw_gemm<T, T>(h, dz[cur], wT, dz[1 - cur], B, static_cast<int>(hout), static_cast<int>(hin), st);
      }
      cur = 1 - cur;
    }
    // the folded first Linear: gradients of the caller's W0, gamma1, beta1 (b0 = b0')
    if (s == WK_OK) {
      ProfScope ps(h, WK_KERNEL_BW_ROWS, st);
      auto al = [](const void* q, uintptr_t a) { return reinterpret_cast<uintptr_t>(q) % a == 0; };
      if (dims[0] % 4 == 0 && al(g.W[0], 16) && al(h->W0_in[l], 8) && al(h->g1_in[l], 16) && al(h->b1_in[l], 16)) {
        const unsigned gx = static_cast<unsigned>((dims[0] / 4 + 255) / 256);
        const unsigned gy =
            static_cast<unsigned>(std::max(1, std::min({dims[1], 64, static_cast<int>(4 * dv->sms / gx)})));
        bw_unfold4_kernel<IO><<<dim3(gx, gy), 256, 0, st>>>(g.W[0], g.b[0], static_cast<const IO*>(h->W0_in[l]),
                                                            h->g1_in[l], h->b1_in[l], g.fmb_ln_gamma, g.fmb_ln_beta,
                                                            dims[1], dims[0]);
      } else {
        const dim3 grid(static_cast<unsigned>((dims[0] + 255) / 256), static_cast<unsigned>(std::min(dims[1], 64)));
        bw_unfold_kernel<IO><<<grid, 256, 0, st>>>(g.W[0], g.b[0], static_cast<const IO*>(h->W0_in[l]), h->g1_in[l],
                                                   h->b1_in[l], g.fmb_ln_gamma, g.fmb_ln_beta, dims[1], dims[0]);
      }
      s = launch_status();
    }
    // FMB: Z = X^T Y, F = X Z, dF from the LayerNorm backward, then dZ = X^T dF;
    // dX += W_L^T dG + dF Z^T + Y dZ^T in one launch; dY = sum_b X_b dZ_b
    const int64_t dk = static_cast<int64_t>(d) * k;
    const int Bi = static_cast<int>(B);
    if (s == WK_OK) {
      TcContr p = tc_contr(d, k, Bi, 1, TC_STORE, Zb, dk, k, 1);
      p.nterms = 1;
      p.round_c = 1;  // Z is read only by the tf32 contractions
      p.t[0] = tc_term(Xf, Yf, 1, n);
      p.t[0].sAz = nd, p.t[0].sAm = 1, p.t[0].sAk2 = d;  // X(b, i, t) as (m = t, k = i)
      p.t[0].sBn = 1, p.t[0].sBk2 = k;                   // Y(i, c)
      s = run_tc_contract(h, p, st);
    }
    if (s == WK_OK) {
      TcContr p = tc_contr(n, k, Bi, 1, TC_STORE, Fb, nk, k, 1);
      p.nterms = 1;
      p.t[0] = tc_term(Xf, Zb, 1, d);
      p.t[0].sAz = nd, p.t[0].sAm = d, p.t[0].sAk2 = 1;  // X(b, i, t)
      p.t[0].sBz = dk, p.t[0].sBn = 1, p.t[0].sBk2 = k;  // Z(b, t, c)
      s = run_tc_contract(h, p, st);
    }
    if (s == WK_OK) {
      ProfScope ps(h, WK_KERNEL_BW_ROWS, st);
      const unsigned grid = static_cast<unsigned>(B);
      const int nki = static_cast<int>(nk);
      if (nk % 4 != 0 || nk > 32768)
        bw_fmb_ln_kernel<T><<<grid, 256, 0, st>>>(Fb, dz[cur], dFb, nki, h->eps);
      else if (nk <= 4096)
        bw_fmb_ln_reg_kernel<T, 8><<<grid, 512, 0, st>>>(Fb, dz[cur], dFb, nki, h->eps);
      else if (nk <= 8192)
        bw_fmb_ln_reg_kernel<T, 16><<<grid, 512, 0, st>>>(Fb, dz[cur], dFb, nki, h->eps);
      else if (nk <= 16384)
        bw_fmb_ln_reg_kernel<T, 32><<<grid, 512, 0, st>>>(Fb, dz[cur], dFb, nki, h->eps);
      else
        bw_fmb_ln_reg_kernel<T, 64><<<grid, 512, 0, st>>>(Fb, dz[cur], dFb, nki, h->eps);
      s = launch_status();
    }
    if (s == WK_OK) {
      TcContr p = tc_contr(d, k, Bi, 1, TC_STORE, dZb, dk, k, 1);
      p.nterms = 1;
      p.round_c = 1;  // so is dZ
      p.t[0] = tc_term(Xf, dFb, 1, n);
      p.t[0].sAz = nd, p.t[0].sAm = 1, p.t[0].sAk2 = d;  // X(b, i, t) as (m = t, k = i)
      p.t[0].sBz = nk, p.t[0].sBn = 1, p.t[0].sBk2 = k;  // dF(b, i, c)
      s = run_tc_contract(h, p, st);
    }
    if (s == WK_OK) {
      TcContr p = tc_contr(n, d, Bi, 1, TC_ACCUM, dxl, nd, d, 1);
      p.nterms = 3;
      p.t[0] = tc_term(WLf, dG, 1, n_l);
      p.t[0].sAm = 1, p.t[0].sAk2 = n;                   // W_L(r, i) at r n + i
      p.t[0].sBz = nd, p.t[0].sBn = 1, p.t[0].sBk2 = d;  // dG(b, r, t)
      p.t[1] = tc_term(dFb, Zb, 1, k);
      p.t[1].sAz = nk, p.t[1].sAm = k, p.t[1].sAk2 = 1;  // dF(b, i, c)
      p.t[1].sBz = dk, p.t[1].sBn = k, p.t[1].sBk2 = 1;  // Z(b, t, c)
      p.t[2] = tc_term(Yf, dZb, 1, k);
      p.t[2].sAm = k, p.t[2].sAk2 = 1;                   // Y(i, c)
      p.t[2].sBz = dk, p.t[2].sBn = k, p.t[2].sBk2 = 1;  // dZ(b, t, c)
      s = run_tc_contract(h, p, st);
    }
    if (s == WK_OK) {
      TcContr p = tc_contr(n, k, 1, tc_splits(dv, n, k, Bi), TC_ATOMIC, g.Y, 0, k, 1);
      p.nterms = 1;
      p.t[0] = tc_term(Xf, dZb, Bi, d);
      p.t[0].sAm = d, p.t[0].sAk1 = nd, p.t[0].sAk2 = 1;  // X(b, i, t)
      p.t[0].sBn = 1, p.t[0].sBk1 = dk, p.t[0].sBk2 = k;  // dZ(b, t, c)
      s = run_tc_contract(h, p, st);
    }
    // layer l's parameter gradients are final: a caller may reduce them across ranks while
    // the layers below are differentiated
    if (s == WK_OK && layer_done && layer_done[l] &&
        cudaEventRecord(reinterpret_cast<cudaEvent_t>(layer_done[l]), st) != cudaSuccess) {
      cudaGetLastError();
      s = WK_ERR_CUDA;
    }
  }
  return s;
}

wk_status read_status_word(unsigned* word, cudaStream_t st) {
  if (cudaStreamSynchronize(st) != cudaSuccess) {
    cudaGetLastError();
    return WK_ERR_CUDA;
  }
  unsigned v = 0;
  if (cudaMemcpy(&v, word, sizeof v, cudaMemcpyDeviceToHost) != cudaSuccess) {
    cudaGetLastError();
    return WK_ERR_CUDA;
  }
  if (v) {
    const unsigned zero = 0;
    cudaMemcpy(word, &zero, sizeof zero, cudaMemcpyHostToDevice);
  }
  if (v & kFlagTimeout) return WK_ERR_TIMEOUT;
  if (v & kFlagNonFinite) return WK_ERR_NONFINITE;
  if (v) return WK_ERR_DEVICE;
  return WK_OK;
}

template <typename T>
wk_status mlp_linear16(const DevInfo* dv, const void* A, const void* W, const float* bias, void* C, int64_t M,
                              int K, int N, int64_t ldc, int relu, cudaStream_t st) {
  if (!mlp_tc_ok(M, K, N, ldc)) return WK_ERR_UNSUPPORTED;
  const bool pair = use_pair_gemm(M);
  GemmMaps mp;
  if (!map_kmajor<T>(dv, &mp.A, A, K, M, GEMM_BM) || !map_kmajor<T>(dv, &mp.B, W, K, N, pair ? 128 : GEMM_BN) ||
      !map_out<T>(dv, &mp.C, C, N, M, ldc))
    return WK_ERR_UNSUPPORTED;
  if (pair)
    return run_gemm_tc2<T, T>(dv, mp, mlp2_params(M, K, N, bias, relu ? 1 : 0, dv->standalone_status), st);
  return run_gemm_tc<MODE_MLP, T, T>(dv, mp, mlp_params(M, K, N, bias, relu ? 1 : 0, dv->standalone_status), st);
}

template <typename T>
wk_status lcb16(const DevInfo* dv, const void* W_L, const void* X, void* concat, int64_t batch, int n, int d,
                       int n_f, int n_l, cudaStream_t st) {
  if (!lcb_tc_ok(batch, n, d))
    return run_lcb_simt<T, T>(static_cast<const T*>(W_L), static_cast<const T*>(X), static_cast<T*>(concat), batch, n,
                              d, n_f, n_l, st);
  GemmMaps mp;
  if (!map_kmajor<T>(dv, &mp.A, W_L, n, n_l, GEMM_BM) || !map_lcb_x<T>(dv, &mp.B, X, n, d, batch) ||
      !map_lcb_out<T>(dv, &mp.C, concat, n_f + n_l, d, n_f, n_l, batch))
    return WK_ERR_UNSUPPORTED;
  return run_lcb_tc<T, T>(dv, mp, lcb_params(batch, n, d, n_l, dv->standalone_status), st);
}

// ------------------------------------------------- no-allocation layer forward
//
// A one-layer forward whose intermediates live in a fixed device array that is
// part of this library's image instead of memory the library allocates. The
// array is reserved on every device that loads the library, until exit. Host
// code must not hand the array's name to a kernel (on the host it names a
// stand-in, not device memory); its device address is looked up once per device
// with cudaGetSymbolAddress and cached.
__device__ __align__(256) uint8_t g_noalloc_scratch[WK_NOALLOC_SCRATCH_BYTES];

void* g_noalloc_addr[64];
bool g_noalloc_init[64];

wk_status noalloc_scratch(const DevInfo* dv, uint8_t** out) {
  std::lock_guard<std::mutex> lk(g_mu);
  if (!g_noalloc_init[dv->id]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr) {
      cudaGetLastError();
      return WK_ERR_CUDA;
    }
    g_noalloc_addr[dv->id] = p;
    g_noalloc_init[dv->id] = true;
  }
  *out = static_cast<uint8_t*>(g_noalloc_addr[dv->id]);
  return WK_OK;
}

// Scratch bytes one example needs: A0, one or two MLP activation buffers, the
// concat buffer; each region rounded up to 256 bytes for the whole batch.
size_t noalloc_bytes(const wk_stack_config* c, const std::vector<int32_t>& dims, int64_t batch) {
  auto up = [](size_t v) { return (v + 255) & ~static_cast<size_t>(255); };
  const size_t es = c->dtype == WK_F32 ? 4 : 2;
  const int m = c->mlp_num_linear;
  int32_t hmax = 0;
  for (int j = 1; j < m; ++j) hmax = std::max(hmax, dims[j]);
  size_t b = up(batch * static_cast<size_t>(c->n) * c->k * es) + up(batch * static_cast<size_t>(c->n) * c->d * es);
  if (m >= 2) b += up(batch * static_cast<size_t>(hmax) * es);
  if (m >= 3) b += up(batch * static_cast<size_t>(hmax) * es);
  return b;
}

template <typename T>
wk_status layer_noalloc16(const DevInfo* dv, const wk_stack_config* c, const std::vector<int32_t>& dims,
                          const wk_layer_weights* w, const T* X, T* out, int64_t batch, uint8_t* scratch,
                          float eps, cudaStream_t st) {
  auto up = [](size_t v) { return (v + 255) & ~static_cast<size_t>(255); };
  const int n = c->n, d = c->d, k = c->k, m = c->mlp_num_linear;
  const size_t nd = static_cast<size_t>(n) * d;
  int32_t hmax = 0;
  for (int j = 1; j < m; ++j) hmax = std::max(hmax, dims[j]);
  uint8_t* p = scratch;
  T* A0 = reinterpret_cast<T*>(p);
  p += up(batch * static_cast<size_t>(n) * k * 2);
  T* cat = reinterpret_cast<T*>(p);
  p += up(batch * nd * 2);
  T* H[2] = {reinterpret_cast<T*>(p), nullptr};
  if (m >= 2) p += up(batch * static_cast<size_t>(hmax) * 2);
  H[1] = reinterpret_cast<T*>(p);
  unsigned* status = dv->standalone_status;
  wk_status s = run_fm16<T>(dv, X, static_cast<const T*>(w->Y), w->fmb_ln_gamma, w->fmb_ln_beta, A0, batch, n, d, k,
                            eps, status, st);
  for (int j = 0; j < m && s == WK_OK; ++j) {
    const T* in = (j == 0) ? A0 : H[(j - 1) % 2];
    const bool lastj = j == m - 1;
    T* o = lastj ? cat : H[j % 2];
    const int64_t ldc = lastj ? static_cast<int64_t>(nd) : dims[j + 1];
    const float* bias = w->b ? w->b[j] : nullptr;
    if (mlp_tc_ok(batch, dims[j], dims[j + 1], ldc)) {
      GemmMaps mp;
      if (!map_kmajor<T>(dv, &mp.A, in, dims[j], batch, GEMM_BM) ||
          !map_kmajor<T>(dv, &mp.B, w->W[j], dims[j], dims[j + 1], GEMM_BN) ||
          !map_out<T>(dv, &mp.C, o, dims[j + 1], batch, ldc))
        return WK_ERR_UNSUPPORTED;
      s = run_gemm_tc<MODE_MLP, T, T>(dv, mp, mlp_params(batch, dims[j], dims[j + 1], bias, lastj ? 0 : 1, status),
                                       st);
    } else {
      s = run_gemm_simt<T, T>(in, static_cast<const T*>(w->W[j]), bias, o, batch, dims[j], dims[j + 1], ldc,
                              lastj ? 0 : 1, st);
    }
  }
  if (s == WK_OK) s = lcb16<T>(dv, w->W_L, X, cat, batch, n, d, c->n_f, c->n_l, st);
  if (s == WK_OK)
    s = run_res_ln<T, T, T>(dv, cat, X, w->out_ln_gamma, w->out_ln_beta, out, batch * n, d, eps, status, st);
  return s;
}

// Runs `body` (which enqueues a forward on the stream it is given) under stream
// capture on a private stream and instantiates the graph.
template <typename F>
wk_status capture_graph(int device, F body, wk_graph** out) {
  cudaStream_t cs = nullptr;
  if (cudaStreamCreateWithFlags(&cs, cudaStreamNonBlocking) != cudaSuccess) {
    cudaGetLastError();
    return WK_ERR_CUDA;
  }
  wk_graph* g = new (std::nothrow) wk_graph();
  if (!g) {
    cudaStreamDestroy(cs);
    return WK_ERR_OOM;
  }
  g->device = device;
  wk_status st = WK_OK;
  if (cudaStreamBeginCapture(cs, cudaStreamCaptureModeThreadLocal) != cudaSuccess) {
    st = WK_ERR_CUDA;
  } else {
    st = body(reinterpret_cast<wk_stream_t>(cs));
    cudaGraph_t graph = nullptr;
    const cudaError_t e = cudaStreamEndCapture(cs, &graph);
    if (st == WK_OK && (e != cudaSuccess || !graph)) st = WK_ERR_CUDA;
    g->graph = graph;
    if (st == WK_OK && cudaGraphInstantiate(&g->exec, graph, 0) != cudaSuccess) st = WK_ERR_CUDA;
  }
  cudaGetLastError();
  cudaStreamDestroy(cs);
  if (st != WK_OK) {
    if (g->exec) cudaGraphExecDestroy(g->exec);
    if (g->graph) cudaGraphDestroy(g->graph);
    delete g;
    return st;
  }
  *out = g;
  return WK_OK;
}

}  // namespace

extern "C" {

const char* wk_status_string(wk_status s) {
  switch (s) {
    case WK_OK: return "ok";
    case WK_ERR_INVALID_ARG: return "invalid argument";
    case WK_ERR_UNSUPPORTED: return "unsupported shape or dtype";
    case WK_ERR_OOM: return "out of device memory";
    case WK_ERR_CUDA: return "CUDA runtime error";
    case WK_ERR_TIMEOUT: return "a kernel gave up waiting (device pipeline timeout)";
    case WK_ERR_DEVICE: return "device-side error flag";
    case WK_ERR_NONFINITE: return "non-finite value (a 16-bit intermediate overflowed, or inf / NaN in the input)";
  }
  return "unknown status";
}

// wk_stack_create; front_only: a stack whose layers another handle drives one front
// at a time (an expert of a wk_moe): no layer buffers and no fused end-of-layer path.
static wk_status stack_create_impl(const wk_stack_config* cfg, const wk_layer_weights* weights, wk_stack** out,
                                   bool front_only) {
  if (!out || !weights) return WK_ERR_INVALID_ARG;
  *out = nullptr;
  wk_status st = validate_cfg(cfg);
  if (st != WK_OK) return st;
  const int L = cfg->num_layers, m = cfg->mlp_num_linear;
  const int n = cfg->n, d = cfg->d, k = cfg->k;
  std::vector<int32_t> dims;
  dims.push_back(n * k);
  for (int j = 0; j + 1 < m; ++j) dims.push_back(cfg->mlp_hidden[j]);
  dims.push_back(cfg->n_f * d);
  for (int l = 0; l < L; ++l) {
    const wk_layer_weights& w = weights[l];
    if (!w.Y || !w.W || !w.fmb_ln_gamma || !w.fmb_ln_beta || !w.W_L || !w.out_ln_gamma || !w.out_ln_beta)
      return WK_ERR_INVALID_ARG;
    if (!al16(w.Y) || !al16(w.W_L) || !al16(w.fmb_ln_gamma) || !al16(w.fmb_ln_beta) || !al16(w.out_ln_gamma) ||
        !al16(w.out_ln_beta))
      return WK_ERR_INVALID_ARG;
    for (int j = 0; j < m; ++j) {
      if (!w.W[j] || !al16(w.W[j])) return WK_ERR_INVALID_ARG;
      if (w.b && w.b[j] && !al16(w.b[j])) return WK_ERR_INVALID_ARG;
    }
  }
  DevInfo* dv = nullptr;
  st = dev_info(&dv);
  if (st != WK_OK) return st;

  wk_stack* h = new (std::nothrow) wk_stack();
  if (!h) return WK_ERR_OOM;
  h->device = dv->id;
  h->cfg = *cfg;
  h->cfg.mlp_hidden = nullptr;
  h->dims = dims;
  h->eps = cfg->ln_eps > 0.f ? cfg->ln_eps : 1e-5f;
  h->io = cfg->dtype;
  h->op = cfg->dtype == WK_F32 ? WK_F32 : (cfg->operand_dtype == WK_BF16 ? WK_BF16 : WK_F16);
  h->maxb = cfg->max_batch;
  h->dv = dv;
  h->front_only = front_only;
  h->W.resize(L);
  h->b.resize(L);
  for (int l = 0; l < L; ++l) {
    const wk_layer_weights& w = weights[l];
    h->Y.push_back(w.Y);
    h->WL.push_back(w.W_L);
    for (int j = 0; j < m; ++j) {
      h->W[l].push_back(w.W[j]);
      h->b[l].push_back(w.b ? w.b[j] : nullptr);
    }
    h->g1.push_back(w.fmb_ln_gamma);
    h->b1.push_back(w.fmb_ln_beta);
    h->W0_in.push_back(w.W[0]);
    h->b0_in.push_back(w.b ? w.b[0] : nullptr);
    h->g1_in.push_back(w.fmb_ln_gamma);
    h->b1_in.push_back(w.fmb_ln_beta);
    h->g2.push_back(w.out_ln_gamma);
    h->b2.push_back(w.out_ln_beta);
  }

  auto up = [](size_t v) { return (v + 255) & ~static_cast<size_t>(255); };
  // 16-bit stacks: weights in the operand type (converted once when the caller's type
  // differs). With fp16 operands the FMB LayerNorm's gamma / beta are also folded
  // into the first Linear: W0' = W0 diag(gamma), b0' = b0 + W0 beta (the FM kernel
  // then stores only the normalised values, with no per-example reads of gamma and
  // beta). bf16 operands keep the affine in the FM: rounding W0 diag(gamma) to bf16's
  // 8-bit significand would add an error of the size the bf16 mode already spends.
  const bool fold = h->op == WK_F16;
  if (h->op != WK_F32 && (fold || h->io != h->op)) {
    const bool conv_all = h->io != h->op;
    size_t per_layer = 0;
    if (fold) per_layer += up(static_cast<size_t>(dims[0]) * dims[1] * 2) + up(static_cast<size_t>(dims[1]) * 4);
    if (conv_all) {
      per_layer += up(static_cast<size_t>(n) * k * 2) + up(static_cast<size_t>(cfg->n_l) * n * 2);
      for (int j = fold ? 1 : 0; j < m; ++j) per_layer += up(static_cast<size_t>(dims[j]) * dims[j + 1] * 2);
    }
    if (cudaMalloc(&h->wcopy, per_layer * L) != cudaSuccess) {
      cudaGetLastError();
      delete h;
      return WK_ERR_OOM;
    }
    uint8_t* p = h->wcopy;
    auto conv = [&](const void* src, int64_t count) -> const void* {
      uint8_t* dst = p;
      p += up(static_cast<size_t>(count) * 2);
      wk_status cs = h->io == WK_BF16 ? run_convert<bf16, f16>(dv, src, dst, count, nullptr)
                                      : run_convert<f16, bf16>(dv, src, dst, count, nullptr);
      if (cs != WK_OK) st = cs;
      return dst;
    };
    const int64_t nvec = static_cast<int64_t>(dims[0]) * dims[1] / 8;
    const int blocks = static_cast<int>(std::max<int64_t>(1, std::min<int64_t>((nvec + 255) / 256, dv->sms * 16ll)));
    const int bias_blocks = static_cast<int>(std::max(1, std::min(dims[1] / 8 + 1, dv->sms * 16)));
    for (int l = 0; l < L; ++l) {
      if (conv_all) {
        h->Y[l] = conv(h->Y[l], static_cast<int64_t>(n) * k);
        h->WL[l] = conv(h->WL[l], static_cast<int64_t>(cfg->n_l) * n);
        for (int j = fold ? 1 : 0; j < m; ++j)
          h->W[l][j] = conv(h->W[l][j], static_cast<int64_t>(dims[j]) * dims[j + 1]);
      }
      if (!fold) continue;
      const void* w0 = h->W[l][0];
      void* w0f = p;
      p += up(static_cast<size_t>(dims[0]) * dims[1] * 2);
      float* b0f = reinterpret_cast<float*>(p);
      p += up(static_cast<size_t>(dims[1]) * 4);
      const float* g = h->g1[l];
      const float* be = h->b1[l];
      if (h->io == WK_BF16)
        fold_scale_cols_kernel<bf16, f16><<<blocks, 256>>>(static_cast<const bf16*>(w0), g, static_cast<f16*>(w0f),
                                                            dims[1], dims[0]);
      else
        fold_scale_cols_kernel<f16, f16><<<blocks, 256>>>(static_cast<const f16*>(w0), g, static_cast<f16*>(w0f),
                                                           dims[1], dims[0]);
      if (h->io == WK_BF16)
        fold_bias_kernel<bf16><<<bias_blocks, 256>>>(static_cast<const bf16*>(w0), be, h->b[l][0], b0f, dims[1], dims[0]);
      else
        fold_bias_kernel<f16><<<bias_blocks, 256>>>(static_cast<const f16*>(w0), be, h->b[l][0], b0f, dims[1], dims[0]);
      if (launch_status() != WK_OK) st = WK_ERR_CUDA;
      h->W[l][0] = w0f;
      h->b[l][0] = b0f;
      h->g1[l] = nullptr;  // the FM stores the normalised values
      h->b1[l] = nullptr;
    }
    if (st == WK_OK && cudaDeviceSynchronize() != cudaSuccess) st = WK_ERR_CUDA;
    if (st != WK_OK) {
      cudaGetLastError();
      free_stack(h);
      return st;
    }
  }

  // workspace
  const int64_t B = h->maxb;
  const size_t es = dtype_bytes(h->op);
  int32_t hmax = 8;
  for (int j = 1; j < m; ++j) hmax = std::max(hmax, dims[j]);
  const size_t nd = static_cast<size_t>(n) * d;
  size_t off = 0;
  const size_t o_a0 = off;
  off += up(B * static_cast<size_t>(n) * k * es);
  const size_t o_h0 = off;
  off += up(B * static_cast<size_t>(hmax) * es);
  const size_t o_h1 = off;
  off += up(B * static_cast<size_t>(hmax) * es);
  const size_t o_cat = off;
  off += up(B * nd * es);
  const size_t o_x0 = off;
  if (!front_only) off += up(B * nd * es);
  const size_t o_x1 = off;
  if (!front_only) off += up(B * nd * es);
  const size_t o_status = off;
  off += 256;
  if (cudaMalloc(&h->ws, off) != cudaSuccess) {
    cudaGetLastError();
    free_stack(h);
    return WK_ERR_OOM;
  }
  h->A0 = h->ws + o_a0;
  h->H[0] = h->ws + o_h0;
  h->H[1] = h->ws + o_h1;
  h->cat = h->ws + o_cat;
  h->Xs[0] = front_only ? nullptr : h->ws + o_x0;
  h->Xs[1] = front_only ? nullptr : h->ws + o_x1;
  h->status = reinterpret_cast<unsigned*>(h->ws + o_status);
  if (cudaMemset(h->status, 0, sizeof(unsigned)) != cudaSuccess) {
    cudaGetLastError();
    free_stack(h);
    return WK_ERR_CUDA;
  }
  if (h->op == WK_F16)
    st = build_maps<f16>(h);
  else if (h->op == WK_BF16)
    st = build_maps<bf16>(h);
  if (st != WK_OK) {
    free_stack(h);
    return st;
  }
  *out = h;
  return WK_OK;
}

wk_status wk_stack_create(const wk_stack_config* cfg, const wk_layer_weights* weights, wk_stack** out) {
  return stack_create_impl(cfg, weights, out, false);
}

wk_status wk_stack_forward(wk_stack* h, const void* X, void* out, int64_t batch, wk_stream_t stream) {
  if (!h || batch < 0 || batch > h->maxb) return WK_ERR_INVALID_ARG;
  if (batch == 0) return WK_OK;
  if (!X || !out || !al16(X) || !al16(out)) return WK_ERR_INVALID_ARG;
  const size_t bytes = static_cast<size_t>(batch) * h->cfg.n * h->cfg.d * dtype_bytes(h->io);
  const uint8_t* xa = static_cast<const uint8_t*>(X);
  const uint8_t* oa = static_cast<const uint8_t*>(out);
  if (xa < oa + bytes && oa < xa + bytes) return WK_ERR_INVALID_ARG;
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev != h->device) {
    cudaGetLastError();
    return WK_ERR_INVALID_ARG;
  }
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (h->op == WK_F32) return forward32(h, static_cast<const float*>(X), static_cast<float*>(out), batch, st);
  if (h->op == WK_F16)
    return h->io == WK_BF16 ? forward16<f16, bf16>(h, X, out, batch, st) : forward16<f16, f16>(h, X, out, batch, st);
  return h->io == WK_BF16 ? forward16<bf16, bf16>(h, X, out, batch, st) : forward16<bf16, f16>(h, X, out, batch, st);
}

wk_status wk_stack_forward_host(wk_stack* h, const void* X_host, void* out_host, int64_t batch, wk_stream_t stream) {
  if (!h || batch < 0 || batch > h->maxb) return WK_ERR_INVALID_ARG;
  if (batch == 0) return WK_OK;
  if (!X_host || !out_host) return WK_ERR_INVALID_ARG;
  const size_t ex_bytes = static_cast<size_t>(h->cfg.n) * h->cfg.d * dtype_bytes(h->io);
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  // Chunks of at least 1024 examples (or the whole batch): large enough that the
  // GEMMs stay efficient, small enough that copies overlap the compute.
  int64_t chunk = std::max<int64_t>(1024, (batch + 3) / 4);
  chunk = std::min(chunk, batch);
  if (!h->stage || h->stage_chunk < chunk) {
    if (h->stage) {
      cudaFree(h->stage);
      h->stage = nullptr;
    }
    const int64_t cap = std::min<int64_t>(h->maxb, std::max<int64_t>(1024, (h->maxb + 3) / 4));
    const int64_t want = std::max(cap, chunk);
    if (cudaMalloc(&h->stage, 4 * static_cast<size_t>(want) * ex_bytes) != cudaSuccess) {
      cudaGetLastError();
      h->stage = nullptr;
      return WK_ERR_OOM;
    }
    h->stage_chunk = want;
  }
  if (!h->s_in && cudaStreamCreateWithFlags(&h->s_in, cudaStreamNonBlocking) != cudaSuccess) return WK_ERR_CUDA;
  if (!h->s_out && cudaStreamCreateWithFlags(&h->s_out, cudaStreamNonBlocking) != cudaSuccess) return WK_ERR_CUDA;
  uint8_t* din[2] = {h->stage, h->stage + h->stage_chunk * ex_bytes};
  uint8_t* dout[2] = {h->stage + 2 * h->stage_chunk * ex_bytes, h->stage + 3 * h->stage_chunk * ex_bytes};
  cudaEvent_t ev_start, ev_in[2], ev_done[2], ev_out[2];
  cudaEventCreateWithFlags(&ev_start, cudaEventDisableTiming);
  for (int i = 0; i < 2; ++i) {
    cudaEventCreateWithFlags(&ev_in[i], cudaEventDisableTiming);
    cudaEventCreateWithFlags(&ev_done[i], cudaEventDisableTiming);
    cudaEventCreateWithFlags(&ev_out[i], cudaEventDisableTiming);
  }
  cudaEventRecord(ev_start, st);
  cudaStreamWaitEvent(h->s_in, ev_start, 0);
  cudaStreamWaitEvent(h->s_out, ev_start, 0);
  wk_status s = WK_OK;
  int c = 0;
  for (int64_t b0 = 0; b0 < batch && s == WK_OK; b0 += chunk, ++c) {
    const int p = c & 1;
    const int64_t nb = std::min(chunk, batch - b0);
    const size_t nbytes = static_cast<size_t>(nb) * ex_bytes;
    if (c >= 2) cudaStreamWaitEvent(h->s_in, ev_done[p], 0);  // forward c-2 finished reading din[p]
    if (cudaMemcpyAsync(din[p], static_cast<const uint8_t*>(X_host) + b0 * ex_bytes, nbytes, cudaMemcpyHostToDevice,
                        h->s_in) != cudaSuccess) {
      s = WK_ERR_CUDA;
      break;
    }
    cudaEventRecord(ev_in[p], h->s_in);
    cudaStreamWaitEvent(st, ev_in[p], 0);
    if (c >= 2) cudaStreamWaitEvent(st, ev_out[p], 0);  // copy-out of c-2 finished reading dout[p]
    s = wk_stack_forward(h, din[p], dout[p], nb, stream);
    if (s != WK_OK) break;
    cudaEventRecord(ev_done[p], st);
    cudaStreamWaitEvent(h->s_out, ev_done[p], 0);
    if (cudaMemcpyAsync(static_cast<uint8_t*>(out_host) + b0 * ex_bytes, dout[p], nbytes, cudaMemcpyDeviceToHost,
                        h->s_out) != cudaSuccess) {
      s = WK_ERR_CUDA;
      break;
    }
    cudaEventRecord(ev_out[p], h->s_out);
  }
  if (cudaStreamSynchronize(h->s_out) != cudaSuccess) s = WK_ERR_CUDA;
  if (cudaStreamSynchronize(h->s_in) != cudaSuccess) s = WK_ERR_CUDA;
  if (cudaStreamSynchronize(st) != cudaSuccess) s = WK_ERR_CUDA;
  cudaEventDestroy(ev_start);
  for (int i = 0; i < 2; ++i) {
    cudaEventDestroy(ev_in[i]);
    cudaEventDestroy(ev_done[i]);
    cudaEventDestroy(ev_out[i]);
  }
  cudaGetLastError();
  return s;
}

wk_status wk_stack_forward_host_async(wk_stack* h, const void* X_host, void* out_host, int64_t batch,
                                      wk_stream_t stream, int64_t* ticket) {
  if (!h || batch < 0 || batch > h->maxb) return WK_ERR_INVALID_ARG;
  if (batch == 0) {
    if (ticket) *ticket = h->a_seq - 1;
    return WK_OK;
  }
  if (!X_host || !out_host) return WK_ERR_INVALID_ARG;
  const size_t ex_bytes = static_cast<size_t>(h->cfg.n) * h->cfg.d * dtype_bytes(h->io);
  const size_t slot = static_cast<size_t>(h->maxb) * ex_bytes;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (!h->astage) {
    if (cudaMalloc(&h->astage, 4 * slot) != cudaSuccess) {
      cudaGetLastError();
      h->astage = nullptr;
      return WK_ERR_OOM;
    }
  }
  for (int i = 0; i < 2; ++i) {
    cudaEvent_t* evs[3] = {&h->a_in[i], &h->a_done[i], &h->a_out[i]};
    for (cudaEvent_t* e : evs)
      if (!*e && cudaEventCreateWithFlags(e, cudaEventDisableTiming) != cudaSuccess) {
        cudaGetLastError();
        *e = nullptr;
        return WK_ERR_CUDA;
      }
  }
  if (!h->s_in && cudaStreamCreateWithFlags(&h->s_in, cudaStreamNonBlocking) != cudaSuccess) return WK_ERR_CUDA;
  if (!h->s_out && cudaStreamCreateWithFlags(&h->s_out, cudaStreamNonBlocking) != cudaSuccess) return WK_ERR_CUDA;
  // Call i uses slot p = i % 2. Its input copy waits for the forward of call i-2 (the last
  // reader of din); its forward waits for its input copy and for the output copy of call
  // i-2 (the last reader of dout); its output copy waits for its forward. The caller's
  // stream is not waited for by the copies, so the next call's input copy runs under this
  // call's forward.
  const int64_t i = h->a_seq;
  const int p = static_cast<int>(i & 1);
  uint8_t* din = h->astage + p * slot;
  uint8_t* dout = h->astage + (2 + p) * slot;
  const size_t nbytes = static_cast<size_t>(batch) * ex_bytes;
  if (i >= 2 && cudaStreamWaitEvent(h->s_in, h->a_done[p], 0) != cudaSuccess) return WK_ERR_CUDA;
  if (cudaMemcpyAsync(din, X_host, nbytes, cudaMemcpyHostToDevice, h->s_in) != cudaSuccess ||
      cudaEventRecord(h->a_in[p], h->s_in) != cudaSuccess || cudaStreamWaitEvent(st, h->a_in[p], 0) != cudaSuccess ||
      (i >= 2 && cudaStreamWaitEvent(st, h->a_out[p], 0) != cudaSuccess)) {
    cudaGetLastError();
    return WK_ERR_CUDA;
  }
  const wk_status s = wk_stack_forward(h, din, dout, batch, stream);
  if (s != WK_OK) return s;
  if (cudaEventRecord(h->a_done[p], st) != cudaSuccess || cudaStreamWaitEvent(h->s_out, h->a_done[p], 0) != cudaSuccess ||
      cudaMemcpyAsync(out_host, dout, nbytes, cudaMemcpyDeviceToHost, h->s_out) != cudaSuccess ||
      cudaEventRecord(h->a_out[p], h->s_out) != cudaSuccess) {
    cudaGetLastError();
    return WK_ERR_CUDA;
  }
  h->a_seq = i + 1;
  if (ticket) *ticket = i;
  return WK_OK;
}

wk_status wk_stack_host_wait(wk_stack* h, int64_t ticket) {
  if (!h || ticket >= h->a_seq) return WK_ERR_INVALID_ARG;
  if (h->a_seq == 0) return WK_OK;
  const int64_t t = ticket < 0 ? h->a_seq - 1 : ticket;
  // the slot's event marks call t, or a later call of the same slot whose copy follows
  // call t's on the output stream
  if (cudaEventSynchronize(h->a_out[t & 1]) != cudaSuccess) {
    cudaGetLastError();
    return WK_ERR_CUDA;
  }
  return WK_OK;
}

wk_status wk_stack_sync_status(wk_stack* h, wk_stream_t stream) {
  if (!h) return WK_ERR_INVALID_ARG;
  return read_status_word(h->status, reinterpret_cast<cudaStream_t>(stream));
}

wk_status wk_stack_backward(wk_stack* h, const void* X, const float* dOut, float* dX, const wk_layer_grads* grads,
                            int64_t batch, wk_stream_t stream) {
  return wk_stack_backward_events(h, X, dOut, dX, grads, batch, stream, nullptr);
}

wk_status wk_stack_backward_events(wk_stack* h, const void* X, const float* dOut, float* dX,
                                   const wk_layer_grads* grads, int64_t batch, wk_stream_t stream,
                                   void* const* layer_done) {
  if (!h || batch < 0 || batch > h->maxb) return WK_ERR_INVALID_ARG;
  if (batch == 0) return WK_OK;
  if (!X || !dOut || !dX || !grads || !al16(X) || !al16(dOut) || !al16(dX)) return WK_ERR_INVALID_ARG;
  const wk_stack_config& c = h->cfg;
  for (int l = 0; l < c.num_layers; ++l) {
    const wk_layer_grads& g = grads[l];
    if (!g.Y || !g.W || !g.b || !g.fmb_ln_gamma || !g.fmb_ln_beta || !g.W_L || !g.out_ln_gamma || !g.out_ln_beta)
      return WK_ERR_INVALID_ARG;
    for (int j = 0; j < c.mlp_num_linear; ++j)
      if (!g.W[j] || !g.b[j] || !al16(g.W[j])) return WK_ERR_INVALID_ARG;
  }
  // the fp16-operand path (first Linear folded), at most three Linears (both hidden
  // activations stay in the workspace), a batch that is a multiple of 8 (the weight
  // gradients' GEMMs contract over it), embedding rows of at most 256
  if (h->op != WK_F16 || h->front_only || c.mlp_num_linear > 3 || batch % 8 != 0 || c.d > 256 ||
      c.d % 32 != 0)
    return WK_ERR_UNSUPPORTED;
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev != h->device) {
    cudaGetLastError();
    return WK_ERR_INVALID_ARG;
  }
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  return h->io == WK_BF16 ? backward16<f16, bf16>(h, X, dOut, dX, grads, batch, st, layer_done)
                          : backward16<f16, f16>(h, X, dOut, dX, grads, batch, st, layer_done);
}

void wk_stack_destroy(wk_stack* h) { free_stack(h); }

wk_status wk_stack_set_profiling(wk_stack* h, int enable) {
  if (!h) return WK_ERR_INVALID_ARG;
  h->prof = enable != 0;
  return WK_OK;
}

wk_status wk_stack_kernel_times(wk_stack* h, double* total_ms, int64_t* launches) {
  if (!h || !total_ms || !launches) return WK_ERR_INVALID_ARG;
  for (int i = 0; i < WK_KERNEL_COUNT; ++i) {
    total_ms[i] = 0.0;
    launches[i] = 0;
  }
  wk_status s = WK_OK;
  for (auto& r : h->recs) {
    float ms = 0.f;
    if (cudaEventSynchronize(r.b) != cudaSuccess || cudaEventElapsedTime(&ms, r.a, r.b) != cudaSuccess) {
      cudaGetLastError();
      s = WK_ERR_CUDA;
    } else if (r.kind >= 0 && r.kind < WK_KERNEL_COUNT) {
      total_ms[r.kind] += ms;
      launches[r.kind] += 1;
    }
    h->pool.push_back(r.a);
    h->pool.push_back(r.b);
  }
  h->recs.clear();
  return s;
}

// ------------------------------------------------------------- stand-alone

wk_status wk_fm_ln(const void* X, const void* Y, const float* gamma, const float* beta, void* A0, int64_t batch,
                   int32_t n, int32_t d, int32_t k, wk_dtype dtype, float eps, wk_stream_t stream) {
  if (batch < 0 || n < 1 || d < 1 || k < 1) return WK_ERR_INVALID_ARG;
  if (batch == 0) return WK_OK;
  if (!X || !Y || !A0 || !al16(X) || !al16(Y) || !al16(A0) || (!gamma) != (!beta) || (gamma && !al16(gamma)) ||
      (beta && !al16(beta)))
    return WK_ERR_INVALID_ARG;
  if (dtype != WK_F32 && dtype != WK_BF16 && dtype != WK_F16) return WK_ERR_UNSUPPORTED;
  if (d % 8 != 0 || k % 2 != 0 || !fm_supported(n, d, k, dtype != WK_F32)) return WK_ERR_UNSUPPORTED;
  DevInfo* dv = nullptr;
  wk_status s = dev_info(&dv);
  if (s != WK_OK) return s;
  const float e = eps > 0.f ? eps : 1e-5f;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (dtype == WK_BF16)
    return run_fm16<bf16>(dv, static_cast<const bf16*>(X), static_cast<const bf16*>(Y), gamma, beta,
                          static_cast<bf16*>(A0), batch, n, d, k, e, dv->standalone_status, st);
  if (dtype == WK_F16)
    return run_fm16<f16>(dv, static_cast<const f16*>(X), static_cast<const f16*>(Y), gamma, beta,
                         static_cast<f16*>(A0), batch, n, d, k, e, dv->standalone_status, st);
  return run_fm_simt<float>(dv, static_cast<const float*>(X), static_cast<const float*>(Y), gamma, beta,
                            static_cast<float*>(A0), batch, n, d, k, e, st);
}

wk_status wk_mlp_linear(const void* A, const void* W, const float* bias, void* C, int64_t M, int32_t K, int32_t N,
                        int64_t ldc, int relu, wk_dtype dtype, wk_stream_t stream) {
  if (M < 0 || K < 1 || N < 1 || ldc < N) return WK_ERR_INVALID_ARG;
  if (M == 0) return WK_OK;
  if (!A || !W || !C || !al16(A) || !al16(W) || !al16(C) || (bias && !al16(bias))) return WK_ERR_INVALID_ARG;
  if (dtype != WK_F32 && dtype != WK_BF16 && dtype != WK_F16) return WK_ERR_UNSUPPORTED;
  DevInfo* dv = nullptr;
  wk_status s = dev_info(&dv);
  if (s != WK_OK) return s;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (dtype == WK_BF16) return mlp_linear16<bf16>(dv, A, W, bias, C, M, K, N, ldc, relu, st);
  if (dtype == WK_F16) return mlp_linear16<f16>(dv, A, W, bias, C, M, K, N, ldc, relu, st);
  return run_gemm_simt<float, float>(static_cast<const float*>(A), static_cast<const float*>(W), bias,
                                     static_cast<float*>(C), M, K, N, ldc, relu ? 1 : 0, st);
}

wk_status wk_lcb(const void* W_L, const void* X, void* concat, int64_t batch, int32_t n, int32_t d, int32_t n_f,
                 int32_t n_l, wk_dtype dtype, wk_stream_t stream) {
  if (batch < 0 || n < 1 || d < 1 || n_f < 0 || n_l < 1) return WK_ERR_INVALID_ARG;
  if (batch == 0) return WK_OK;
  if (!W_L || !X || !concat || !al16(W_L) || !al16(X) || !al16(concat)) return WK_ERR_INVALID_ARG;
  if (dtype != WK_F32 && dtype != WK_BF16 && dtype != WK_F16) return WK_ERR_UNSUPPORTED;
  DevInfo* dv = nullptr;
  wk_status s = dev_info(&dv);
  if (s != WK_OK) return s;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (dtype == WK_BF16) return lcb16<bf16>(dv, W_L, X, concat, batch, n, d, n_f, n_l, st);
  if (dtype == WK_F16) return lcb16<f16>(dv, W_L, X, concat, batch, n, d, n_f, n_l, st);
  return run_lcb_simt<float, float>(static_cast<const float*>(W_L), static_cast<const float*>(X),
                                    static_cast<float*>(concat), batch, n, d, n_f, n_l, st);
}

wk_status wk_res_ln(const void* concat, const void* X, const float* gamma, const float* beta, void* out, int64_t rows,
                    int32_t d, wk_dtype dtype, float eps, wk_stream_t stream) {
  if (rows < 0 || d < 1) return WK_ERR_INVALID_ARG;
  if (rows == 0) return WK_OK;
  if (!concat || !X || !gamma || !beta || !out || !al16(concat) || !al16(X) || !al16(out) || !al16(gamma) ||
      !al16(beta))
    return WK_ERR_INVALID_ARG;
  if (dtype != WK_F32 && dtype != WK_BF16 && dtype != WK_F16) return WK_ERR_UNSUPPORTED;
  if (!res_ln_d_ok(d)) return WK_ERR_UNSUPPORTED;
  DevInfo* dv = nullptr;
  wk_status s = dev_info(&dv);
  if (s != WK_OK) return s;
  const float e = eps > 0.f ? eps : 1e-5f;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (dtype == WK_BF16)
    return run_res_ln<bf16, bf16, bf16>(dv, static_cast<const bf16*>(concat), static_cast<const bf16*>(X), gamma,
                                        beta, static_cast<bf16*>(out), rows, d, e, dv->standalone_status, st);
  if (dtype == WK_F16)
    return run_res_ln<f16, f16, f16>(dv, static_cast<const f16*>(concat), static_cast<const f16*>(X), gamma, beta,
                                     static_cast<f16*>(out), rows, d, e, dv->standalone_status, st);
  return run_res_ln<float, float, float>(dv, static_cast<const float*>(concat), static_cast<const float*>(X), gamma,
                                         beta, static_cast<float*>(out), rows, d, e, dv->standalone_status, st);
}

wk_status wk_device_status(wk_stream_t stream) {
  DevInfo* dv = nullptr;
  wk_status s = dev_info(&dv);
  if (s != WK_OK) return s;
  return read_status_word(dv->standalone_status, reinterpret_cast<cudaStream_t>(stream));
}

wk_status wk_layer_forward_noalloc(const wk_stack_config* cfg, const wk_layer_weights* w, const void* X, void* out,
                                   int64_t batch, wk_stream_t stream) {
  if (!w || batch < 0) return WK_ERR_INVALID_ARG;
  wk_stack_config c1;
  if (cfg) {
    c1 = *cfg;
    c1.num_layers = 1;
    c1.max_batch = 1;
  }
  wk_status s = validate_cfg(cfg ? &c1 : nullptr);
  if (s != WK_OK) return s;
  if (cfg->operand_dtype != WK_F32 && cfg->operand_dtype != cfg->dtype) return WK_ERR_UNSUPPORTED;
  if (batch == 0) return WK_OK;
  if (!X || !out || !al16(X) || !al16(out) || !w->Y || !w->W || !w->W_L || !w->fmb_ln_gamma || !w->fmb_ln_beta ||
      !w->out_ln_gamma || !w->out_ln_beta)
    return WK_ERR_INVALID_ARG;
  // the same alignment rules as wk_stack_create: the kernels read every weight, bias and
  // LayerNorm vector with 16-byte loads or TMA
  if (!al16(w->Y) || !al16(w->W_L) || !al16(w->fmb_ln_gamma) || !al16(w->fmb_ln_beta) || !al16(w->out_ln_gamma) ||
      !al16(w->out_ln_beta))
    return WK_ERR_INVALID_ARG;
  std::vector<int32_t> dims;
  dims.push_back(cfg->n * cfg->k);
  for (int j = 0; j + 1 < cfg->mlp_num_linear; ++j) dims.push_back(cfg->mlp_hidden[j]);
  dims.push_back(cfg->n_f * cfg->d);
  for (int j = 0; j < cfg->mlp_num_linear; ++j) {
    if (!w->W[j] || !al16(w->W[j])) return WK_ERR_INVALID_ARG;
    if (w->b && w->b[j] && !al16(w->b[j])) return WK_ERR_INVALID_ARG;
  }
  // No product below can wrap: the largest per-example region (n*max(k, d, hidden) values
  // of at most 4 bytes, under 2^33 for int32 dims) times a batch below the scratch size.
  if (batch > static_cast<int64_t>(WK_NOALLOC_SCRATCH_BYTES)) return WK_ERR_INVALID_ARG;
  if (noalloc_bytes(cfg, dims, batch) > WK_NOALLOC_SCRATCH_BYTES) return WK_ERR_INVALID_ARG;
  const size_t bytes = static_cast<size_t>(batch) * cfg->n * cfg->d * (cfg->dtype == WK_F32 ? 4 : 2);
  const uint8_t* xa = static_cast<const uint8_t*>(X);
  const uint8_t* oa = static_cast<const uint8_t*>(out);
  if (xa < oa + bytes && oa < xa + bytes) return WK_ERR_INVALID_ARG;
  DevInfo* dv = nullptr;
  s = dev_info(&dv);
  if (s != WK_OK) return s;
  uint8_t* scratch = nullptr;
  s = noalloc_scratch(dv, &scratch);
  if (s != WK_OK) return s;
  const float eps = cfg->ln_eps > 0.f ? cfg->ln_eps : 1e-5f;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (cfg->dtype == WK_BF16)
    return layer_noalloc16<bf16>(dv, cfg, dims, w, static_cast<const bf16*>(X), static_cast<bf16*>(out), batch,
                                 scratch, eps, st);
  if (cfg->dtype == WK_F16)
    return layer_noalloc16<f16>(dv, cfg, dims, w, static_cast<const f16*>(X), static_cast<f16*>(out), batch, scratch,
                                eps, st);
  // fp32: the CUDA-core kernels, same scratch layout
  auto up = [](size_t v) { return (v + 255) & ~static_cast<size_t>(255); };
  const int n = cfg->n, d = cfg->d, k = cfg->k, m = cfg->mlp_num_linear;
  const size_t nd = static_cast<size_t>(n) * d;
  int32_t hmax = 0;
  for (int j = 1; j < m; ++j) hmax = std::max(hmax, dims[j]);
  uint8_t* p = scratch;
  float* A0 = reinterpret_cast<float*>(p);
  p += up(batch * static_cast<size_t>(n) * k * 4);
  float* cat = reinterpret_cast<float*>(p);
  p += up(batch * nd * 4);
  float* H[2] = {reinterpret_cast<float*>(p), nullptr};
  if (m >= 2) p += up(batch * static_cast<size_t>(hmax) * 4);
  H[1] = reinterpret_cast<float*>(p);
  const float* Xf = static_cast<const float*>(X);
  s = run_fm_simt<float>(dv, Xf, static_cast<const float*>(w->Y), w->fmb_ln_gamma, w->fmb_ln_beta, A0, batch, n, d, k,
                         eps, st);
  for (int j = 0; j < m && s == WK_OK; ++j) {
    const float* in = (j == 0) ? A0 : H[(j - 1) % 2];
    const bool lastj = j == m - 1;
    float* o = lastj ? cat : H[j % 2];
    s = run_gemm_simt<float, float>(in, static_cast<const float*>(w->W[j]), w->b ? w->b[j] : nullptr, o, batch,
                                    dims[j], dims[j + 1], lastj ? static_cast<int64_t>(nd) : dims[j + 1],
                                    lastj ? 0 : 1, st);
  }
  if (s == WK_OK)
    s = run_lcb_simt<float, float>(static_cast<const float*>(w->W_L), Xf, cat, batch, n, d, cfg->n_f, cfg->n_l, st);
  if (s == WK_OK)
    s = run_res_ln<float, float, float>(dv, cat, Xf, w->out_ln_gamma, w->out_ln_beta, static_cast<float*>(out),
                                        batch * n, d, eps, dv->standalone_status, st);
  return s;
}

// ------------------------------------------------------------------ graphs

wk_status wk_stack_graph_create(wk_stack* h, const void* X, void* out, int64_t batch, wk_graph** g) {
  if (!h || !g || batch < 1) return WK_ERR_INVALID_ARG;
  *g = nullptr;
  const bool prof = h->prof;
  h->prof = false;  // no event records inside a graph
  const wk_status st = capture_graph(h->device, [&](wk_stream_t s) { return wk_stack_forward(h, X, out, batch, s); }, g);
  h->prof = prof;
  return st;
}

wk_status wk_moe_graph_create(wk_moe* h, const void* X, void* out, int64_t batch, wk_graph** g) {
  if (!h || !g || batch < 1) return WK_ERR_INVALID_ARG;
  *g = nullptr;
  std::vector<bool> prof;
  for (wk_stack* e : h->ex) {
    prof.push_back(e->prof);
    e->prof = false;
  }
  const wk_status st = capture_graph(h->device, [&](wk_stream_t s) { return wk_moe_forward(h, X, out, batch, s); }, g);
  for (size_t i = 0; i < h->ex.size(); ++i) h->ex[i]->prof = prof[i];
  return st;
}

wk_status wk_graph_launch(wk_graph* g, wk_stream_t stream) {
  if (!g || !g->exec) return WK_ERR_INVALID_ARG;
  if (cudaGraphLaunch(g->exec, reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess) {
    cudaGetLastError();
    return WK_ERR_CUDA;
  }
  return WK_OK;
}

void wk_graph_destroy(wk_graph* g) {
  if (!g) return;
  if (g->exec) cudaGraphExecDestroy(g->exec);
  if (g->graph) cudaGraphDestroy(g->graph);
  cudaGetLastError();
  delete g;
}

// ------------------------------------------------------------ prediction head

wk_status wk_stack_set_head(wk_stack* h, const wk_head* head) {
  if (!h || !head || h->front_only) return WK_ERR_INVALID_ARG;
  const int q = head->num_linear;
  if (q < 1 || !head->T || (q > 1 && !head->hidden)) return WK_ERR_INVALID_ARG;
  if (h->op == WK_F32) return WK_ERR_UNSUPPORTED;
  std::vector<int32_t> dims;
  dims.push_back(h->cfg.n * h->cfg.d);
  for (int j = 0; j + 1 < q; ++j) {
    if (head->hidden[j] < 8 || head->hidden[j] % 8 != 0) return WK_ERR_UNSUPPORTED;
    dims.push_back(head->hidden[j]);
  }
  dims.push_back(1);
  for (int j = 0; j < q; ++j) {
    if (!head->T[j] || !al16(head->T[j])) return WK_ERR_INVALID_ARG;
    if (head->c && head->c[j] && !al16(head->c[j])) return WK_ERR_INVALID_ARG;
  }
  const DevInfo* dv = h->dv;
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev != h->device) {
    cudaGetLastError();
    return WK_ERR_INVALID_ARG;
  }
  cudaDeviceSynchronize();
  if (h->head_copy) cudaFree(h->head_copy);
  if (h->head_ws) cudaFree(h->head_ws);
  h->head_copy = h->head_ws = nullptr;
  h->HH[0] = h->HH[1] = nullptr;
  h->head_dims.clear();
  h->hT.clear();
  h->hc.clear();
  h->head_maps.clear();
  auto up = [](size_t v) { return (v + 255) & ~static_cast<size_t>(255); };
  wk_status st = WK_OK;
  if (h->io != h->op) {
    size_t total = 0;
    for (int j = 0; j < q; ++j) total += up(static_cast<size_t>(dims[j]) * dims[j + 1] * 2);
    if (cudaMalloc(&h->head_copy, total) != cudaSuccess) {
      cudaGetLastError();
      return WK_ERR_OOM;
    }
  }
  uint8_t* p = h->head_copy;
  for (int j = 0; j < q; ++j) {
    const int64_t cnt = static_cast<int64_t>(dims[j]) * dims[j + 1];
    if (h->io != h->op) {
      const wk_status cs = h->io == WK_BF16 ? run_convert<bf16, f16>(dv, head->T[j], p, cnt, nullptr)
                                            : run_convert<f16, bf16>(dv, head->T[j], p, cnt, nullptr);
      if (cs != WK_OK) st = cs;
      h->hT.push_back(p);
      p += up(static_cast<size_t>(cnt) * 2);
    } else {
      h->hT.push_back(head->T[j]);
    }
    h->hc.push_back(head->c ? head->c[j] : nullptr);
  }
  int32_t hmax = 0;
  for (int j = 1; j < q; ++j) hmax = std::max(hmax, dims[j]);
  if (st == WK_OK && hmax > 0) {
    const size_t one = up(static_cast<size_t>(h->maxb) * hmax * 2);
    if (cudaMalloc(&h->head_ws, 2 * one) != cudaSuccess) {
      cudaGetLastError();
      st = WK_ERR_OOM;
    } else {
      h->HH[0] = h->head_ws;
      h->HH[1] = h->head_ws + one;
    }
  }
  h->head_dims = dims;
  if (st == WK_OK) st = h->op == WK_F16 ? build_head_maps<f16>(h) : build_head_maps<bf16>(h);
  if (st == WK_OK && cudaDeviceSynchronize() != cudaSuccess) st = WK_ERR_CUDA;
  if (st != WK_OK) {
    cudaGetLastError();
    if (h->head_copy) cudaFree(h->head_copy);
    if (h->head_ws) cudaFree(h->head_ws);
    h->head_copy = h->head_ws = nullptr;
    h->head_dims.clear();
    h->hT.clear();
    h->hc.clear();
    h->head_maps.clear();
  }
  return st;
}

wk_status wk_stack_predict(wk_stack* h, const void* X, float* logit, float* prob, int64_t batch,
                           wk_stream_t stream) {
  if (!h || batch < 0 || batch > h->maxb || h->head_dims.empty()) return WK_ERR_INVALID_ARG;
  if (batch == 0) return WK_OK;
  if (!X || !logit || !al16(X)) return WK_ERR_INVALID_ARG;
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev != h->device) {
    cudaGetLastError();
    return WK_ERR_INVALID_ARG;
  }
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (h->op == WK_F16)
    return h->io == WK_BF16 ? predict16<f16, bf16>(h, X, logit, prob, batch, st)
                            : predict16<f16, f16>(h, X, logit, prob, batch, st);
  return h->io == WK_BF16 ? predict16<bf16, bf16>(h, X, logit, prob, batch, st)
                          : predict16<bf16, f16>(h, X, logit, prob, batch, st);
}

// ------------------------------------------------------- mixture of experts

wk_status wk_moe_create(const wk_stack_config* cfg, int32_t num_experts, const wk_layer_weights* experts,
                        const wk_moe_gate* gates, wk_moe** out) {
  if (!out || !experts || !gates || !cfg) return WK_ERR_INVALID_ARG;
  *out = nullptr;
  if (num_experts < 1 || num_experts > MOE_MAX_E) return WK_ERR_INVALID_ARG;
  wk_status st = validate_cfg(cfg);
  if (st != WK_OK) return st;
  if (cfg->dtype == WK_F32) return WK_ERR_UNSUPPORTED;
  const int L = cfg->num_layers, E = num_experts;
  for (int l = 0; l < L; ++l)
    if (!gates[l].W_g || !al16(gates[l].W_g) || (gates[l].b_g && !al16(gates[l].b_g))) return WK_ERR_INVALID_ARG;
  DevInfo* dv = nullptr;
  st = dev_info(&dv);
  if (st != WK_OK) return st;
  wk_moe* h = new (std::nothrow) wk_moe();
  if (!h) return WK_ERR_OOM;
  h->device = dv->id;
  h->cfg = *cfg;
  h->cfg.mlp_hidden = nullptr;
  h->E = E;
  h->eps = cfg->ln_eps > 0.f ? cfg->ln_eps : 1e-5f;
  h->io = cfg->dtype;
  h->op = cfg->operand_dtype == WK_BF16 ? WK_BF16 : WK_F16;
  h->maxb = cfg->max_batch;
  h->dv = dv;
  std::vector<wk_layer_weights> lw(L);
  for (int e = 0; e < E; ++e) {
    for (int l = 0; l < L; ++l) lw[l] = experts[static_cast<size_t>(l) * E + e];
    wk_stack* x = nullptr;
    st = stack_create_impl(cfg, lw.data(), &x, true);
    if (st != WK_OK) {
      free_moe(h);
      return st;
    }
    h->ex.push_back(x);
  }
  auto up = [](size_t v) { return (v + 255) & ~static_cast<size_t>(255); };
  const size_t nd = static_cast<size_t>(cfg->n) * cfg->d;
  const size_t gbytes = up(static_cast<size_t>(E) * nd * 2);
  if (h->io != h->op) {
    if (cudaMalloc(&h->wcopy, gbytes * L) != cudaSuccess) {
      cudaGetLastError();
      free_moe(h);
      return WK_ERR_OOM;
    }
  }
  for (int l = 0; l < L; ++l) {
    if (h->io != h->op) {
      uint8_t* dst = h->wcopy + gbytes * l;
      const int64_t cnt = static_cast<int64_t>(E) * nd;
      st = h->io == WK_BF16 ? run_convert<bf16, f16>(dv, gates[l].W_g, dst, cnt, nullptr)
                            : run_convert<f16, bf16>(dv, gates[l].W_g, dst, cnt, nullptr);
      h->Wg.push_back(dst);
    } else {
      h->Wg.push_back(gates[l].W_g);
    }
    h->bg.push_back(gates[l].b_g);
  }
  const int64_t B = h->maxb;
  const size_t o_g = 0, o_x0 = up(static_cast<size_t>(B) * E * 4), o_x1 = o_x0 + up(B * nd * 2),
               total = o_x1 + up(B * nd * 2);
  if (st != WK_OK || cudaMalloc(&h->ws, total) != cudaSuccess) {
    cudaGetLastError();
    free_moe(h);
    return st != WK_OK ? st : WK_ERR_OOM;
  }
  h->g = reinterpret_cast<float*>(h->ws + o_g);
  h->Xm[0] = h->ws + o_x0;
  h->Xm[1] = h->ws + o_x1;
  if (h->ex[0]->tc_lcb) {
    const bool ok = h->op == WK_F16 ? (map_lcb_x<f16>(dv, &h->lcbX[0], h->Xm[0], cfg->n, cfg->d, B) &&
                                       map_lcb_x<f16>(dv, &h->lcbX[1], h->Xm[1], cfg->n, cfg->d, B))
                                    : (map_lcb_x<bf16>(dv, &h->lcbX[0], h->Xm[0], cfg->n, cfg->d, B) &&
                                       map_lcb_x<bf16>(dv, &h->lcbX[1], h->Xm[1], cfg->n, cfg->d, B));
    if (!ok) {
      free_moe(h);
      return WK_ERR_UNSUPPORTED;
    }
  }
  if (cudaDeviceSynchronize() != cudaSuccess) {
    cudaGetLastError();
    free_moe(h);
    return WK_ERR_CUDA;
  }
  *out = h;
  return WK_OK;
}

wk_status wk_moe_forward(wk_moe* h, const void* X, void* out, int64_t batch, wk_stream_t stream) {
  if (!h || batch < 0 || batch > h->maxb) return WK_ERR_INVALID_ARG;
  if (batch == 0) return WK_OK;
  if (!X || !out || !al16(X) || !al16(out)) return WK_ERR_INVALID_ARG;
  const size_t bytes = static_cast<size_t>(batch) * h->cfg.n * h->cfg.d * dtype_bytes(h->io);
  const uint8_t* xa = static_cast<const uint8_t*>(X);
  const uint8_t* oa = static_cast<const uint8_t*>(out);
  if (xa < oa + bytes && oa < xa + bytes) return WK_ERR_INVALID_ARG;
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev != h->device) {
    cudaGetLastError();
    return WK_ERR_INVALID_ARG;
  }
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (h->op == WK_F16)
    return h->io == WK_BF16 ? moe_forward16<f16, bf16>(h, X, out, batch, st) : moe_forward16<f16, f16>(h, X, out, batch, st);
  return h->io == WK_BF16 ? moe_forward16<bf16, bf16>(h, X, out, batch, st) : moe_forward16<bf16, f16>(h, X, out, batch, st);
}

wk_status wk_moe_sync_status(wk_moe* h, wk_stream_t stream) {
  if (!h) return WK_ERR_INVALID_ARG;
  wk_status first = WK_OK;
  for (wk_stack* e : h->ex) {
    const wk_status s = read_status_word(e->status, reinterpret_cast<cudaStream_t>(stream));
    if (first == WK_OK) first = s;
  }
  return first;
}

wk_status wk_moe_set_profiling(wk_moe* h, int enable) {
  if (!h) return WK_ERR_INVALID_ARG;
  for (wk_stack* e : h->ex) e->prof = enable != 0;
  return WK_OK;
}

wk_status wk_moe_kernel_times(wk_moe* h, double* total_ms, int64_t* launches) {
  if (!h || !total_ms || !launches) return WK_ERR_INVALID_ARG;
  for (int i = 0; i < WK_KERNEL_COUNT; ++i) {
    total_ms[i] = 0.0;
    launches[i] = 0;
  }
  wk_status first = WK_OK;
  for (wk_stack* e : h->ex) {
    double t[WK_KERNEL_COUNT];
    int64_t c[WK_KERNEL_COUNT];
    const wk_status s = wk_stack_kernel_times(e, t, c);
    if (first == WK_OK) first = s;
    for (int i = 0; i < WK_KERNEL_COUNT; ++i) {
      total_ms[i] += t[i];
      launches[i] += c[i];
    }
  }
  return first;
}

void wk_moe_destroy(wk_moe* h) { free_moe(h); }

wk_status wk_moe_gate_softmax(const void* X, const void* W_g, const float* b_g, float* g, int64_t batch, int64_t nd,
                              int32_t num_experts, wk_dtype dtype, wk_stream_t stream) {
  if (batch < 0 || nd < 8 || nd % 8 != 0 || num_experts < 1 || num_experts > MOE_MAX_E) return WK_ERR_INVALID_ARG;
  if (batch == 0) return WK_OK;
  if (!X || !W_g || !g || !al16(X) || !al16(W_g) || (b_g && !al16(b_g))) return WK_ERR_INVALID_ARG;
  if (dtype != WK_BF16 && dtype != WK_F16) return WK_ERR_UNSUPPORTED;
  DevInfo* dv = nullptr;
  wk_status s = dev_info(&dv);
  if (s != WK_OK) return s;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (dtype == WK_BF16)
    return run_moe_gate<bf16>(dv, static_cast<const bf16*>(X), static_cast<const bf16*>(W_g), b_g, g, batch, nd,
                              num_experts, st);
  return run_moe_gate<f16>(dv, static_cast<const f16*>(X), static_cast<const f16*>(W_g), b_g, g, batch, nd,
                           num_experts, st);
}

wk_status wk_moe_combine(const void* const* concats, const void* X, const float* g, const float* const* gammas,
                         const float* const* betas, void* out, int64_t batch, int32_t n, int32_t d,
                         int32_t num_experts, wk_dtype dtype, float eps, wk_stream_t stream) {
  if (batch < 0 || n < 1 || d < 1 || num_experts < 1 || num_experts > MOE_MAX_E) return WK_ERR_INVALID_ARG;
  if (batch == 0) return WK_OK;
  if (!concats || !X || !g || !gammas || !betas || !out || !al16(X) || !al16(out)) return WK_ERR_INVALID_ARG;
  MoePtrs mp{};
  for (int e = 0; e < num_experts; ++e) {
    if (!concats[e] || !gammas[e] || !betas[e] || !al16(concats[e]) || !al16(gammas[e]) || !al16(betas[e]))
      return WK_ERR_INVALID_ARG;
    mp.cat[e] = concats[e];
    mp.gamma[e] = gammas[e];
    mp.beta[e] = betas[e];
  }
  if (dtype != WK_BF16 && dtype != WK_F16) return WK_ERR_UNSUPPORTED;
  if (!res_ln_d_ok(d)) return WK_ERR_UNSUPPORTED;
  DevInfo* dv = nullptr;
  wk_status s = dev_info(&dv);
  if (s != WK_OK) return s;
  const float e = eps > 0.f ? eps : 1e-5f;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const int64_t rows = batch * n;
  if (dtype == WK_BF16)
    return run_moe_combine<bf16, bf16>(dv, mp, static_cast<const bf16*>(X), g, static_cast<bf16*>(out), rows, n, d,
                                       num_experts, e, dv->standalone_status, st);
  return run_moe_combine<f16, f16>(dv, mp, static_cast<const f16*>(X), g, static_cast<f16*>(out), rows, n, d,
                                   num_experts, e, dv->standalone_status, st);
}

}  // extern "C"

// ====================================================================== WHALE
//
// Attention-based fusion of the WHALE pages (section 2.1 item 3, section 2.2): the
// attention with shared keys and values, then the fusion Linear and the pre-norm
// shared-gate SwiGLU FFN with its residual (kernels in whale.cuh).

struct wk_whale {
  int device = 0;
  wk_whale_config cfg{};
  float eps = 1e-5f;
  const DevInfo* dv = nullptr;
  wk_whale_weights w{};
  uint8_t* ws = nullptr;
  void* A = nullptr;           // [max_batch, n, d] attention output
  unsigned* status = nullptr;
  bool prof = false;
  struct Rec {
    int kind;
    cudaEvent_t a, b;
  };
  std::vector<Rec> recs;
  std::vector<cudaEvent_t> pool;
};

namespace {

bool whale_d_ok(int d) { return d == 32 || d == 64 || d == 128 || d == 160; }

// [batch, rows, d] as a 3-D map (d, rows, batch) with boxes (bw, 128, 1): rows past
// `rows` of an example read as zeros (the last key block of a ragged L).
template <typename T>
bool whale_map3(const DevInfo* dv, CUtensorMap* m, const void* base, int d, int rows, int64_t batch, int bw) {
  const uint64_t dims[3] = {static_cast<uint64_t>(d), static_cast<uint64_t>(rows), static_cast<uint64_t>(batch)};
  const uint64_t strides[2] = {static_cast<uint64_t>(d) * sizeof(T), static_cast<uint64_t>(rows) * d * sizeof(T)};
  const uint32_t box[3] = {static_cast<uint32_t>(bw), 128u, 1u};
  return make_map(dv, m, tmap_dtype<T>(), 3, base, dims, strides, box,
                  bw == 64 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B);
}

// A row-major [rows, cols] matrix with boxes (bw, box_rows).
template <typename T>
bool whale_map2(const DevInfo* dv, CUtensorMap* m, const void* base, int64_t cols, int64_t rows, int bw,
                int box_rows) {
  const uint64_t dims[2] = {static_cast<uint64_t>(cols), static_cast<uint64_t>(rows)};
  const uint64_t strides[1] = {static_cast<uint64_t>(cols) * sizeof(T)};
  const uint32_t box[2] = {static_cast<uint32_t>(bw), static_cast<uint32_t>(box_rows)};
  return make_map(dv, m, tmap_dtype<T>(), 2, base, dims, strides, box,
                  bw == 64 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B);
}

template <int D, typename T>
wk_status whale_attn_run(const DevInfo* dv, const void* Hw, const void* Hs, void* A, int64_t batch, int n, int L,
                         unsigned* status, cudaStream_t st) {
  using C = WaCfg<D>;
  CUtensorMap tkv;
  if (!whale_map3<T>(dv, &tkv, Hs, D, L, batch, C::BW)) return WK_ERR_UNSUPPORTED;
  auto fn = whale_attn_kernel<C, T>;
  const wk_status s = smem_attr(dv, reinterpret_cast<const void*>(fn), C::SMEM);
  if (s != WK_OK) return s;
  const int64_t units = batch * ((n + C::R - 1) / C::R);
  const int grid = static_cast<int>(std::min<int64_t>(units, dv->sms));
  const float scale_log2 = static_cast<float>(1.4426950408889634 / std::sqrt(static_cast<double>(D)));
  fn<<<grid, WA_THREADS, C::SMEM, st>>>(tkv, static_cast<const T*>(Hw), static_cast<T*>(A), batch, n, L, scale_log2,
                                        status);
  return launch_status();
}

template <int D, typename T>
wk_status whale_ffn_run(const DevInfo* dv, const void* Hw, const void* A, const wk_whale_weights& w, void* Hf,
                        int64_t rows, int h, float eps, unsigned* status, cudaStream_t st) {
  using C = WfCfg<D>;
  CUtensorMap thw, ta, twf, twu, twd, thf;
  if (!whale_map2<T>(dv, &thw, Hw, D, rows, C::BW, C::R) || !whale_map2<T>(dv, &ta, A, D, rows, C::BW, C::R) ||
      !whale_map2<T>(dv, &twf, w.W_F, 2 * D, D, C::BW, D) || !whale_map2<T>(dv, &twu, w.W_up, D, h, C::BW, C::HC) ||
      !whale_map2<T>(dv, &twd, w.W_down, h, D, C::BW, D) || !whale_map2<T>(dv, &thf, Hf, D, rows, C::BW, C::R))
    return WK_ERR_UNSUPPORTED;
  auto fn = whale_ffn_kernel<C, T>;
  const wk_status s = smem_attr(dv, reinterpret_cast<const void*>(fn), C::SMEM);
  if (s != WK_OK) return s;
  const int64_t tiles = (rows + C::R - 1) / C::R;
  const int grid = static_cast<int>(std::min<int64_t>(tiles, dv->sms));
  fn<<<grid, WF_THREADS, C::SMEM, st>>>(thw, ta, twf, twu, twd, thf, w.b_F, w.ln_gamma, w.ln_beta, rows, h, eps,
                                        status);
  return launch_status();
}

template <typename T>
wk_status whale_attn_dispatch(const DevInfo* dv, const void* Hw, const void* Hs, void* A, int64_t batch, int n,
                              int L, int d, unsigned* status, cudaStream_t st) {
  switch (d) {
    case 32: return whale_attn_run<32, T>(dv, Hw, Hs, A, batch, n, L, status, st);
    case 64: return whale_attn_run<64, T>(dv, Hw, Hs, A, batch, n, L, status, st);
    case 128: return whale_attn_run<128, T>(dv, Hw, Hs, A, batch, n, L, status, st);
    case 160: return whale_attn_run<160, T>(dv, Hw, Hs, A, batch, n, L, status, st);
  }
  return WK_ERR_UNSUPPORTED;
}

template <typename T>
wk_status whale_ffn_dispatch(const DevInfo* dv, const void* Hw, const void* A, const wk_whale_weights& w, void* Hf,
                             int64_t rows, int d, int h, float eps, unsigned* status, cudaStream_t st) {
  switch (d) {
    case 32: return whale_ffn_run<32, T>(dv, Hw, A, w, Hf, rows, h, eps, status, st);
    case 64: return whale_ffn_run<64, T>(dv, Hw, A, w, Hf, rows, h, eps, status, st);
    case 128: return whale_ffn_run<128, T>(dv, Hw, A, w, Hf, rows, h, eps, status, st);
    case 160: return whale_ffn_run<160, T>(dv, Hw, A, w, Hf, rows, h, eps, status, st);
  }
  return WK_ERR_UNSUPPORTED;
}

wk_status whale_check_weights(const wk_whale_weights* w) {
  if (!w || !w->W_F || !w->ln_gamma || !w->ln_beta || !w->W_up || !w->W_down) return WK_ERR_INVALID_ARG;
  if (!al16(w->W_F) || !al16(w->W_up) || !al16(w->W_down) || (w->b_F && !al16(w->b_F)) || !al16(w->ln_gamma) ||
      !al16(w->ln_beta))
    return WK_ERR_INVALID_ARG;
  return WK_OK;
}

// Event pair around one launch of a WHALE handle (as the stack's per-kernel records).
struct WhaleProf {
  wk_whale* h;
  int kind;
  cudaStream_t st;
  cudaEvent_t a = nullptr, b = nullptr;
  WhaleProf(wk_whale* h_, int k, cudaStream_t s) : h(h_), kind(k), st(s) {
    if (!h->prof) return;
    a = take();
    b = take();
    if (a && b) cudaEventRecord(a, st);
  }
  cudaEvent_t take() {
    cudaEvent_t e = nullptr;
    if (!h->pool.empty()) {
      e = h->pool.back();
      h->pool.pop_back();
    } else if (cudaEventCreate(&e) != cudaSuccess) {
      cudaGetLastError();
      e = nullptr;
    }
    return e;
  }
  ~WhaleProf() {
    if (!h->prof) return;
    if (a && b) {
      cudaEventRecord(b, st);
      h->recs.push_back({kind, a, b});
    } else {
      if (a) h->pool.push_back(a);
      if (b) h->pool.push_back(b);
    }
  }
};

void free_whale(wk_whale* h) {
  if (!h) return;
  cudaDeviceSynchronize();
  cudaGetLastError();
  if (h->ws) cudaFree(h->ws);
  for (auto& r : h->recs) {
    cudaEventDestroy(r.a);
    cudaEventDestroy(r.b);
  }
  for (auto e : h->pool) cudaEventDestroy(e);
  cudaGetLastError();
  delete h;
}

}  // namespace

extern "C" {

wk_status wk_whale_create(const wk_whale_config* cfg, const wk_whale_weights* w, wk_whale** out) {
  if (!cfg || !out) return WK_ERR_INVALID_ARG;
  *out = nullptr;
  if (cfg->n < 1 || cfg->L < 1 || cfg->max_batch < 1 || cfg->ln_eps < 0.f) return WK_ERR_INVALID_ARG;
  if (cfg->dtype != WK_BF16 && cfg->dtype != WK_F16) return WK_ERR_UNSUPPORTED;
  if (!whale_d_ok(cfg->d) || cfg->h < 64 || cfg->h % 64 != 0) return WK_ERR_UNSUPPORTED;
  wk_status st = whale_check_weights(w);
  if (st != WK_OK) return st;
  DevInfo* dv = nullptr;
  st = dev_info(&dv);
  if (st != WK_OK) return st;
  wk_whale* h = new (std::nothrow) wk_whale;
  if (!h) return WK_ERR_OOM;
  h->device = dv->id;
  h->cfg = *cfg;
  h->dv = dv;
  h->w = *w;
  h->eps = cfg->ln_eps > 0.f ? cfg->ln_eps : 1e-5f;
  const size_t abytes = ((static_cast<size_t>(cfg->max_batch) * cfg->n * cfg->d * 2 + 255) / 256) * 256;
  if (cudaMalloc(&h->ws, abytes + 256) != cudaSuccess) {
    cudaGetLastError();
    free_whale(h);
    return WK_ERR_OOM;
  }
  h->A = h->ws;
  h->status = reinterpret_cast<unsigned*>(h->ws + abytes);
  if (cudaMemset(h->status, 0, sizeof(unsigned)) != cudaSuccess || cudaDeviceSynchronize() != cudaSuccess) {
    cudaGetLastError();
    free_whale(h);
    return WK_ERR_CUDA;
  }
  *out = h;
  return WK_OK;
}

wk_status wk_whale_forward(wk_whale* h, const void* Hw, const void* Hs, void* Hf, int64_t batch, wk_stream_t stream) {
  if (!h || batch < 0 || batch > h->cfg.max_batch) return WK_ERR_INVALID_ARG;
  if (batch == 0) return WK_OK;
  if (!Hw || !Hs || !Hf || !al16(Hw) || !al16(Hs) || !al16(Hf)) return WK_ERR_INVALID_ARG;
  const wk_whale_config& c = h->cfg;
  const size_t fb = static_cast<size_t>(batch) * c.n * c.d * 2, sb = static_cast<size_t>(batch) * c.L * c.d * 2;
  const uint8_t* f = static_cast<const uint8_t*>(Hf);
  const uint8_t* q = static_cast<const uint8_t*>(Hw);
  const uint8_t* k = static_cast<const uint8_t*>(Hs);
  if ((f < q + fb && q < f + fb) || (f < k + sb && k < f + fb)) return WK_ERR_INVALID_ARG;
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev != h->device) {
    cudaGetLastError();
    return WK_ERR_INVALID_ARG;
  }
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const int64_t rows = batch * c.n;
  wk_status s;
  {
    WhaleProf ps(h, WK_KERNEL_WHALE_ATTN, st);
    s = c.dtype == WK_BF16 ? whale_attn_dispatch<bf16>(h->dv, Hw, Hs, h->A, batch, c.n, c.L, c.d, h->status, st)
                           : whale_attn_dispatch<f16>(h->dv, Hw, Hs, h->A, batch, c.n, c.L, c.d, h->status, st);
  }
  if (s != WK_OK) return s;
  WhaleProf ps(h, WK_KERNEL_WHALE_FFN, st);
  return c.dtype == WK_BF16
             ? whale_ffn_dispatch<bf16>(h->dv, Hw, h->A, h->w, Hf, rows, c.d, c.h, h->eps, h->status, st)
             : whale_ffn_dispatch<f16>(h->dv, Hw, h->A, h->w, Hf, rows, c.d, c.h, h->eps, h->status, st);
}

wk_status wk_whale_sync_status(wk_whale* h, wk_stream_t stream) {
  if (!h) return WK_ERR_INVALID_ARG;
  return read_status_word(h->status, reinterpret_cast<cudaStream_t>(stream));
}

wk_status wk_whale_set_profiling(wk_whale* h, int enable) {
  if (!h) return WK_ERR_INVALID_ARG;
  h->prof = enable != 0;
  return WK_OK;
}

wk_status wk_whale_kernel_times(wk_whale* h, double* total_ms, int64_t* launches) {
  if (!h || !total_ms || !launches) return WK_ERR_INVALID_ARG;
  for (int i = 0; i < WK_KERNEL_COUNT; ++i) {
    total_ms[i] = 0.0;
    launches[i] = 0;
  }
  wk_status s = WK_OK;
  for (auto& r : h->recs) {
    float ms = 0.f;
    if (cudaEventSynchronize(r.b) != cudaSuccess || cudaEventElapsedTime(&ms, r.a, r.b) != cudaSuccess) {
      cudaGetLastError();
      s = WK_ERR_CUDA;
    } else if (r.kind >= 0 && r.kind < WK_KERNEL_COUNT) {
      total_ms[r.kind] += ms;
      launches[r.kind] += 1;
    }
    h->pool.push_back(r.a);
    h->pool.push_back(r.b);
  }
  h->recs.clear();
  return s;
}

void wk_whale_destroy(wk_whale* h) { free_whale(h); }

wk_status wk_whale_attention(const void* Hw, const void* Hs, void* A, int64_t batch, int32_t n, int32_t L, int32_t d,
                             wk_dtype dtype, wk_stream_t stream) {
  if (batch < 0 || n < 1 || L < 1) return WK_ERR_INVALID_ARG;
  if (batch == 0) return WK_OK;
  if (!Hw || !Hs || !A || !al16(Hw) || !al16(Hs) || !al16(A)) return WK_ERR_INVALID_ARG;
  if (dtype != WK_BF16 && dtype != WK_F16) return WK_ERR_UNSUPPORTED;
  if (!whale_d_ok(d)) return WK_ERR_UNSUPPORTED;
  DevInfo* dv = nullptr;
  wk_status s = dev_info(&dv);
  if (s != WK_OK) return s;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  return dtype == WK_BF16 ? whale_attn_dispatch<bf16>(dv, Hw, Hs, A, batch, n, L, d, dv->standalone_status, st)
                          : whale_attn_dispatch<f16>(dv, Hw, Hs, A, batch, n, L, d, dv->standalone_status, st);
}

wk_status wk_whale_fusion_ffn(const void* Hw, const void* A, const wk_whale_weights* w, void* Hf, int64_t rows,
                              int32_t d, int32_t h, wk_dtype dtype, float eps, wk_stream_t stream) {
  if (rows < 0 || eps < 0.f) return WK_ERR_INVALID_ARG;
  if (rows == 0) return WK_OK;
  if (!Hw || !A || !Hf || !al16(Hw) || !al16(A) || !al16(Hf)) return WK_ERR_INVALID_ARG;
  wk_status s = whale_check_weights(w);
  if (s != WK_OK) return s;
  if (dtype != WK_BF16 && dtype != WK_F16) return WK_ERR_UNSUPPORTED;
  if (!whale_d_ok(d) || h < 64 || h % 64 != 0) return WK_ERR_UNSUPPORTED;
  DevInfo* dv = nullptr;
  s = dev_info(&dv);
  if (s != WK_OK) return s;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const float e = eps > 0.f ? eps : 1e-5f;
  return dtype == WK_BF16 ? whale_ffn_dispatch<bf16>(dv, Hw, A, *w, Hf, rows, d, h, e, dv->standalone_status, st)
                          : whale_ffn_dispatch<f16>(dv, Hw, A, *w, Hf, rows, d, h, e, dv->standalone_status, st);
}

}  // extern "C"
