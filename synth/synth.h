/*
 * synth.h -- host API of the seeded synthetic input generator.
 *
 * Inputs of every workload (expert weights and scales, router weights and
 * bias, hidden states, expert traces) come from here, on the host, or from
 * the device build in synth_dev.cu, which produces the same bytes for the
 * packed int4 weights and the fp16 scales.  Nothing here computes any step of
 * the MoE layer.
 *
 * Stream layout (see synth_core.h for the key and draw definitions):
 *   int4 bytes   byte b = byte (b & 7) of draw(key, b >> 3)
 *   fp16 scale   element i = f16(lo + (hi - lo) * u53(draw(key, i)))
 *   normal       element i = sigma * sqrt(-2 ln u1) * cos(2 pi u2), with
 *                u1 = (draw(key, 2i) >> 11 + 1) * 2^-53 in (0, 1],
 *                u2 = u53(draw(key, 2i + 1)); then rounded to fp32 (RNE),
 *                and for bf16 outputs from that fp32 to bf16 (RNE)
 *   uniform f32  element i = f32(lo + (hi - lo) * u53(draw(key, i)))
 */
#ifndef SYNTH_H
#define SYNTH_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

uint64_t synth_key_c(uint64_t seed, uint32_t layer, uint32_t expert,
                     uint32_t tensor);
uint64_t synth_draw_c(uint64_t key, uint64_t i);

void synth_fill_bytes(uint64_t key, uint8_t* out, size_t n);
void synth_fill_scales_f16(uint64_t key, uint16_t* out, size_t n, double lo,
                           double hi);
void synth_fill_normal_f32(uint64_t key, float* out, size_t n, double sigma);
void synth_fill_normal_bf16(uint64_t key, uint16_t* out, size_t n,
                            double sigma);
void synth_fill_uniform_f32(uint64_t key, float* out, size_t n, double lo,
                            double hi);
/* out[i] = bf16(f32(a[i] + c * normal_i)), a given as bf16 bits: the
 * correlated-batch variant x = x0 + c * eps. */
void synth_fill_perturbed_bf16(uint64_t key, const uint16_t* base,
                               uint16_t* out, size_t n, double c);

/* Expert-popularity trace: for each of n_layers layers a seeded permutation
 * perm_l of [0, n_experts); rank r of perm_l has weight (r + 1)^-s.  Each of
 * n_tokens tokens draws k distinct experts per layer without replacement
 * (sequential draws, each renormalised over the ranks not yet drawn).
 * out is [n_tokens][n_layers][k], each row sorted ascending.  Returns 0, or
 * -1 on bad arguments. */
int synth_zipf_trace(uint64_t seed, int n_layers, int n_experts, int k,
                     int n_tokens, double s, int32_t* out);

#ifdef __cplusplus
}
#endif

#endif /* SYNTH_H */
