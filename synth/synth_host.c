/*
 * synth_host.c -- host-side fill functions of the seeded input generator.
 *
 * Compiled with gcc -O2 -ffp-contract=off into libsynth_host.so. The device
 * twin (synth_dev.cu) runs the same synth_core.h arithmetic, so a tensor filled
 * here and the same tensor filled on the GPU hold identical bits.
 *
 * Element f of a tensor is a pure function of (seed, tensor_id, f): a fill of
 * the range [offset, offset + count) writes element f at dst[f - offset], so a
 * caller can generate a slice (for example a few sampled examples of X) without
 * the rest of the tensor.
 */
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>

#include "synth_core.h"

typedef struct {
  void* dst;
  int dtype;
  uint64_t offset, begin, end;
  uint64_t key, key_scale;
  double mean, std;
  int64_t n_feat, d;
  int kind; /* 0 normal, 1 normal scaled by a per-feature LogUniform factor */
} fill_job;

static void store(void* dst, int dtype, uint64_t j, double v) {
  if (dtype == SYNTH_BF16)
    ((uint16_t*)dst)[j] = synth_f64_to_bf16(v);
  else
    ((float*)dst)[j] = (float)v;
}

static void* fill_worker(void* arg) {
  fill_job* job = (fill_job*)arg;
  for (uint64_t f = job->begin; f < job->end; ++f) {
    double v;
    if (job->kind == 0) {
      v = job->mean + job->std * synth_normal(job->key, f);
    } else {
      uint64_t feat = (f / (uint64_t)job->d) % (uint64_t)job->n_feat;
      v = synth_log_uniform_01_10(job->key_scale, feat) * synth_normal(job->key, f);
    }
    store(job->dst, job->dtype, f - job->offset, v);
  }
  return NULL;
}

static int run_fill(fill_job proto, uint64_t offset, uint64_t count, int n_threads) {
  if (count == 0) return 0;
  if (n_threads < 1) n_threads = 1;
  if ((uint64_t)n_threads > count) n_threads = (int)count;
  if (n_threads > 256) n_threads = 256;
  fill_job jobs[256];
  pthread_t tids[256];
  uint64_t chunk = (count + (uint64_t)n_threads - 1) / (uint64_t)n_threads;
  int started = 0;
  int rc = 0;
  for (int t = 0; t < n_threads; ++t) {
    jobs[t] = proto;
    jobs[t].offset = offset;
    jobs[t].begin = offset + (uint64_t)t * chunk;
    jobs[t].end = jobs[t].begin + chunk;
    if (jobs[t].end > offset + count) jobs[t].end = offset + count;
    if (jobs[t].begin >= jobs[t].end) break;
    if (t == 0) continue; /* run on the calling thread below */
    if (pthread_create(&tids[t], NULL, fill_worker, &jobs[t]) != 0) {
      fill_worker(&jobs[t]); /* no thread: do it here */
      tids[t] = 0;
    }
    started = t;
  }
  fill_worker(&jobs[0]);
  for (int t = 1; t <= started; ++t)
    if (tids[t]) pthread_join(tids[t], NULL);
  return rc;
}

/* dst[f - offset] = round_dtype(mean + std * normal(seed, tensor_id, f)) for f in [offset, offset+count) */
int synth_fill_normal_host(void* dst, int dtype, uint64_t offset, uint64_t count, uint64_t seed,
                           uint64_t tensor_id, double mean, double std, int n_threads) {
  if (!dst || (dtype != SYNTH_F32 && dtype != SYNTH_BF16)) return 1;
  fill_job p = {0};
  p.dst = dst;
  p.dtype = dtype;
  p.key = synth_key(seed, tensor_id);
  p.mean = mean;
  p.std = std;
  p.kind = 0;
  return run_fill(p, offset, count, n_threads);
}

/* Embeddings whose rows are scaled per feature:
 * X[b, i, t] = s_i * normal(seed, tensor_id, f), f = (b*n_feat + i)*d + t,
 * s_i = LogUniform(0.1, 10) drawn from stream (seed, scale_tensor_id) at index i. */
int synth_fill_x_logscaled_host(void* dst, int dtype, uint64_t offset, uint64_t count, uint64_t seed,
                                uint64_t tensor_id, uint64_t scale_tensor_id, int64_t n_feat, int64_t d,
                                int n_threads) {
  if (!dst || n_feat <= 0 || d <= 0 || (dtype != SYNTH_F32 && dtype != SYNTH_BF16)) return 1;
  fill_job p = {0};
  p.dst = dst;
  p.dtype = dtype;
  p.key = synth_key(seed, tensor_id);
  p.key_scale = synth_key(seed, scale_tensor_id);
  p.n_feat = n_feat;
  p.d = d;
  p.kind = 1;
  return run_fill(p, offset, count, n_threads);
}

/* The unrounded double values of the normal stream (for distribution tests). */
int synth_normal_f64_host(double* dst, uint64_t offset, uint64_t count, uint64_t seed, uint64_t tensor_id) {
  if (!dst) return 1;
  uint64_t key = synth_key(seed, tensor_id);
  for (uint64_t f = 0; f < count; ++f) dst[f] = synth_normal(key, offset + f);
  return 0;
}

/* The per-feature LogUniform(0.1, 10) factors s_0..s_{count-1}. */
int synth_log_uniform_f64_host(double* dst, uint64_t count, uint64_t seed, uint64_t scale_tensor_id) {
  if (!dst) return 1;
  uint64_t key = synth_key(seed, scale_tensor_id);
  for (uint64_t f = 0; f < count; ++f) dst[f] = synth_log_uniform_01_10(key, f);
  return 0;
}

/* Element-wise helpers exposed for the generator's own tests. */
double synth_log_f64(double x) { return synth_log(x); }
double synth_exp_f64(double x) { return synth_exp(x); }
void synth_cos_sin_2pi_f64(double u, double* c, double* s) { synth_cos_sin_2pi(u, c, s); }
uint16_t synth_f64_to_bf16_bits(double x) { return synth_f64_to_bf16(x); }
