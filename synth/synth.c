/*
 * synth.c -- host build of the seeded synthetic input generator.
 * Compile with -ffp-contract=off so no multiply-add is fused.
 */
#include "synth.h"

#include <math.h>
#include <stdlib.h>
#include <string.h>

#include "synth_core.h"

uint64_t synth_key_c(uint64_t seed, uint32_t layer, uint32_t expert,
                     uint32_t tensor) {
  return synth_key(seed, layer, expert, tensor);
}

uint64_t synth_draw_c(uint64_t key, uint64_t i) { return synth_draw(key, i); }

void synth_fill_bytes(uint64_t key, uint8_t* out, size_t n) {
  size_t words = n / 8;
#pragma omp parallel for schedule(static)
  for (long long w = 0; w < (long long)words; ++w) {
    uint64_t r = synth_draw(key, (uint64_t)w);
    memcpy(out + 8 * (size_t)w, &r, 8); /* little-endian host */
  }
  for (size_t b = words * 8; b < n; ++b) out[b] = synth_byte(key, b);
}

void synth_fill_scales_f16(uint64_t key, uint16_t* out, size_t n, double lo,
                           double hi) {
#pragma omp parallel for schedule(static)
  for (long long i = 0; i < (long long)n; ++i)
    out[i] = synth_scale_f16(key, (uint64_t)i, lo, hi);
}

static double normal_at(uint64_t key, uint64_t i) {
  uint64_t r1 = synth_draw(key, 2 * i);
  uint64_t r2 = synth_draw(key, 2 * i + 1);
  double u1 = ((double)(r1 >> 11) + 1.0) * (1.0 / 9007199254740992.0);
  double u2 = synth_u53(r2);
  return sqrt(-2.0 * log(u1)) * cos(6.283185307179586 * u2);
}

void synth_fill_normal_f32(uint64_t key, float* out, size_t n, double sigma) {
#pragma omp parallel for schedule(static)
  for (long long i = 0; i < (long long)n; ++i)
    out[i] = (float)(sigma * normal_at(key, (uint64_t)i));
}

void synth_fill_normal_bf16(uint64_t key, uint16_t* out, size_t n,
                            double sigma) {
#pragma omp parallel for schedule(static)
  for (long long i = 0; i < (long long)n; ++i)
    out[i] = synth_f32_to_bf16((float)(sigma * normal_at(key, (uint64_t)i)));
}

void synth_fill_uniform_f32(uint64_t key, float* out, size_t n, double lo,
                            double hi) {
#pragma omp parallel for schedule(static)
  for (long long i = 0; i < (long long)n; ++i) {
    double u = synth_u53(synth_draw(key, (uint64_t)i));
    out[i] = (float)(lo + (hi - lo) * u);
  }
}

static double bf16_value(uint16_t b) {
  union { uint32_t u; float f; } v;
  v.u = (uint32_t)b << 16;
  return (double)v.f;
}

void synth_fill_perturbed_bf16(uint64_t key, const uint16_t* base,
                               uint16_t* out, size_t n, double c) {
#pragma omp parallel for schedule(static)
  for (long long i = 0; i < (long long)n; ++i) {
    double v = bf16_value(base[i]) + c * normal_at(key, (uint64_t)i);
    out[i] = synth_f32_to_bf16((float)v);
  }
}

static int cmp_i32(const void* a, const void* b) {
  int32_t x = *(const int32_t*)a, y = *(const int32_t*)b;
  return (x > y) - (x < y);
}

int synth_zipf_trace(uint64_t seed, int n_layers, int n_experts, int k,
                     int n_tokens, double s, int32_t* out) {
  if (n_layers <= 0 || n_experts <= 0 || k <= 0 || k > n_experts ||
      n_tokens < 0 || !out)
    return -1;
  int32_t* perm = (int32_t*)malloc(sizeof(int32_t) * (size_t)n_experts);
  double* wt = (double*)malloc(sizeof(double) * (size_t)n_experts);
  char* taken = (char*)malloc((size_t)n_experts);
  if (!perm || !wt || !taken) {
    free(perm); free(wt); free(taken);
    return -1;
  }
  for (int r = 0; r < n_experts; ++r) wt[r] = pow((double)r + 1.0, -s);
  for (int l = 0; l < n_layers; ++l) {
    /* Fisher-Yates shuffle of the ranks, draws from the layer's PERM key. */
    uint64_t pk = synth_key(seed, (uint32_t)l, 0, SYNTH_T_PERM);
    for (int i = 0; i < n_experts; ++i) perm[i] = i;
    for (int i = n_experts - 1; i > 0; --i) {
      uint64_t j = synth_draw(pk, (uint64_t)i) % (uint64_t)(i + 1);
      int32_t t = perm[i]; perm[i] = perm[j]; perm[j] = t;
    }
    uint64_t tk = synth_key(seed, (uint32_t)l, 0, SYNTH_T_TRACE);
    for (int t = 0; t < n_tokens; ++t) {
      memset(taken, 0, (size_t)n_experts);
      int32_t* row = out + ((size_t)t * (size_t)n_layers + (size_t)l) * (size_t)k;
      for (int j = 0; j < k; ++j) {
        double total = 0.0;
        for (int r = 0; r < n_experts; ++r)
          if (!taken[r]) total += wt[r];
        double u = synth_u53(synth_draw(tk, (uint64_t)t * (uint64_t)k + (uint64_t)j));
        double target = u * total, acc = 0.0;
        int pick = -1;
        for (int r = 0; r < n_experts; ++r) {
          if (taken[r]) continue;
          acc += wt[r];
          pick = r;
          if (target < acc) break;
        }
        taken[pick] = 1;
        row[j] = perm[pick];
      }
      qsort(row, (size_t)k, sizeof(int32_t), cmp_i32);
    }
  }
  free(perm); free(wt); free(taken);
  return 0;
}
