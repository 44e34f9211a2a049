/*
 * synth_dev.cu -- device-side fill kernels of the seeded input generator.
 *
 * Built with nvcc -fmad=false into libsynth_dev.so, so the synth_core.h
 * arithmetic rounds exactly as the host build does: a tensor filled here and on
 * the host hold identical bits. Used to put large synthetic weights straight
 * into HBM without a host round trip.
 */
#include <cuda_runtime.h>
#include <stdint.h>

#include "synth_core.h"

namespace {

__global__ void fill_normal_kernel(void* dst, int dtype, uint64_t offset, uint64_t count, uint64_t key,
                                   double mean, double std) {
  uint64_t stride = (uint64_t)gridDim.x * blockDim.x;
  for (uint64_t j = (uint64_t)blockIdx.x * blockDim.x + threadIdx.x; j < count; j += stride) {
    double v = mean + std * synth_normal(key, offset + j);
    if (dtype == SYNTH_BF16)
      ((uint16_t*)dst)[j] = synth_f64_to_bf16(v);
    else
      ((float*)dst)[j] = __double2float_rn(v);
  }
}

__global__ void fill_x_logscaled_kernel(void* dst, int dtype, uint64_t offset, uint64_t count, uint64_t key,
                                        uint64_t key_scale, int64_t n_feat, int64_t d) {
  uint64_t stride = (uint64_t)gridDim.x * blockDim.x;
  for (uint64_t j = (uint64_t)blockIdx.x * blockDim.x + threadIdx.x; j < count; j += stride) {
    uint64_t f = offset + j;
    uint64_t feat = (f / (uint64_t)d) % (uint64_t)n_feat;
    double v = synth_log_uniform_01_10(key_scale, feat) * synth_normal(key, f);
    if (dtype == SYNTH_BF16)
      ((uint16_t*)dst)[j] = synth_f64_to_bf16(v);
    else
      ((float*)dst)[j] = __double2float_rn(v);
  }
}

int grid_for(uint64_t count) {
  uint64_t blocks = (count + 255) / 256;
  if (blocks > 148ull * 64ull) blocks = 148ull * 64ull;
  if (blocks < 1) blocks = 1;
  return (int)blocks;
}

}  // namespace

extern "C" {

/* Device twin of synth_fill_normal_host. Returns 0, or the cudaError_t of the launch. */
int synth_fill_normal_dev(void* dst, int dtype, uint64_t offset, uint64_t count, uint64_t seed,
                          uint64_t tensor_id, double mean, double std, void* stream) {
  if (!dst || (dtype != SYNTH_F32 && dtype != SYNTH_BF16)) return 1;
  if (count == 0) return 0;
  fill_normal_kernel<<<grid_for(count), 256, 0, (cudaStream_t)stream>>>(dst, dtype, offset, count,
                                                                       synth_key(seed, tensor_id), mean, std);
  return (int)cudaGetLastError();
}

/* Device twin of synth_fill_x_logscaled_host. */
int synth_fill_x_logscaled_dev(void* dst, int dtype, uint64_t offset, uint64_t count, uint64_t seed,
                               uint64_t tensor_id, uint64_t scale_tensor_id, int64_t n_feat, int64_t d,
                               void* stream) {
  if (!dst || n_feat <= 0 || d <= 0 || (dtype != SYNTH_F32 && dtype != SYNTH_BF16)) return 1;
  if (count == 0) return 0;
  fill_x_logscaled_kernel<<<grid_for(count), 256, 0, (cudaStream_t)stream>>>(
      dst, dtype, offset, count, synth_key(seed, tensor_id), synth_key(seed, scale_tensor_id), n_feat, d);
  return (int)cudaGetLastError();
}

}  // extern "C"
