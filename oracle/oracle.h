/*
 * oracle.h -- plain, slow, fp64 CPU oracle of the decode-time routed MoE
 * layer (noaux_tc sigmoid router, top-k of n_experts int4 experts, SwiGLU
 * expert FFN, weighted combine with the always-on shared expert).
 *
 * TEST INFRASTRUCTURE ONLY.  Only tests, the smoke check and the CPU-baseline
 * leg of the benchmark may load this library.  The product path (the CUDA
 * library and its binding) never calls it, and the two share no code.
 *
 * Sources (pages, by title and section):
 *  - "LightLX", section "How it works": 256 experts per MoE layer, a router
 *    picks 8 per token; the noaux_tc sigmoid router of DeepSeek-V3 /
 *    glm_moe_dsa; shared experts are always resident.
 *  - "Show HN: run GLM 5.2 on a slow computer" (colibri summary), section
 *    "Principales fonctionnalites implementees": DeepSeek-V3-style sigmoid
 *    router with noaux_tc, routed_scaling_factor and a shared expert;
 *    int4 kernels with dequant-on-use; batch-union MoE.
 *  - The spec of this layer fixes the int4 format (symmetric codes in
 *    [-8, 7], two per byte, one fp16 scale per 32 consecutive input weights)
 *    and the router constants (n_group, topk_group, routed_scaling_factor).
 *
 * Readings where the pages are silent:
 *  R1 group score = sum of the two largest bias-corrected scores of a group;
 *  R2 experts of dropped groups are excluded (never selected);
 *  R3 ties go to the lower group index and to the lower expert index;
 *  R4 selected weights are always normalised, then scaled by rsf, with
 *     1e-20 added to the denominator;
 *  R5 byte j of a packed row holds element 2j in its low nibble and 2j+1 in
 *     its high nibble, two's complement; W = q * fp16(scale[row][col / 32]);
 *  R6 the shared expert has the routed experts' format and size and is added
 *     with weight 1;
 *  R9 stacked layers: x_next = x + MoE(bf16(RMSNorm(x))), unit gain,
 *     eps 1e-6;
 *  R11 LRU: per token, hits are touched in ascending id, then misses are
 *     loaded in ascending id, each evicting the least recently used slot not
 *     used by the current token;
 *  R16 adaptive expert top-p: of the k selected experts keep the fewest, in
 *     descending weight (ties: lower id), whose weights reach p * rsf, and
 *     normalise the kept weights again; p >= 1 keeps all k;
 *  R19 hot-store: experts pinned per layer are never evicted; the other
 *     slots follow R11; pin loads count as bytes, not as hits or misses.
 *
 * Parity pins live in the CPU test-suite; no function here is unpinned.
 */
#ifndef MOE_ORACLE_H
#define MOE_ORACLE_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct {
  int hidden;        /* H */
  int inter;         /* I */
  int n_experts;     /* E routed experts */
  int top_k;         /* k */
  int n_group;       /* G groups of E / G experts */
  int topk_group;    /* groups kept */
  int group_size;    /* scale group along the input dim (32) */
  double rsf;        /* routed_scaling_factor */
} orc_cfg;

typedef struct {
  const uint8_t* q_gate;   /* [I][H/2] */
  const uint8_t* q_up;     /* [I][H/2] */
  const uint16_t* s_gate;  /* fp16 [I][H/gs] */
  const uint16_t* s_up;    /* fp16 [I][H/gs] */
  const uint8_t* q_down;   /* [H][I/2] */
  const uint16_t* s_down;  /* fp16 [H][I/gs] */
} orc_expert;

/* Value of a bf16 / fp16 bit pattern, exactly, in double. */
double orc_bf16_value(uint16_t b);
double orc_f16_value(uint16_t h);
/* Round a double to bf16 (round to nearest, ties to even), returning bits. */
uint16_t orc_round_bf16(double v);

/* Thread count for the OpenMP loops (<= 0: library default).  Returns the
 * number of threads the next parallel region will use. */
int orc_set_threads(int n);

/* logits[t][e] = sum_h W[e][h] * x[t][h]; W fp32 [E][H], x bf16 [T][H]. */
void orc_router_logits(const orc_cfg* c, const float* w_router,
                       const uint16_t* x_bf16, int T, double* logits);

/* Selection from given scores s[t][e] and bias-corrected scores sp[t][e]
 * (the noaux_tc rule, readings R1-R4).  idx[t][k] ascending, w[t][k].
 * If round_group_f32 is nonzero the group sums are rounded to fp32 before
 * they are compared (the decision in fp32 precision).  margin[t] (nullable)
 * is the smaller of the expert decision gap (k-th minus (k+1)-th candidate
 * sp among the kept groups) and the group decision gap (topk_group-th minus
 * next group score); +inf when a decision has no runner-up.
 * Returns 0, or -1 on bad configuration. */
int orc_select_scores(const orc_cfg* c, const double* s, const double* sp,
                      int T, int round_group_f32, int32_t* idx, double* w,
                      double* margin);

/* Full router: s = sigmoid(logits), sp = s + bias, then orc_select_scores
 * in fp64.  scores_out[t][e] = s (nullable). */
int orc_route(const orc_cfg* c, const double* logits, const float* bias,
              int T, int32_t* idx, double* w, double* margin,
              double* scores_out);

/* Adaptive expert top-p (reading R16) applied in place to routes from
 * orc_select_scores / orc_route: idx [T][k] (ascending), w [T][k], s the
 * unbiased scores [T][E].  Keeps the fewest experts, in descending weight
 * (ties: lower id), whose weights reach p * rsf; kept weights are
 * renormalised over the kept experts; dropped slots become id -1, weight 0,
 * after the kept ids.  n_keep[t] (nullable) = experts kept; margin[t]
 * (nullable) = the smaller of |cumulative share - p| at the boundary and the
 * share gap between the last kept and first dropped expert (infinite for
 * p >= 1).  p > 0; p >= 1 keeps all. */
int orc_topp(const orc_cfg* c, const double* s, int T, double p, int32_t* idx,
             double* w, int32_t* n_keep, double* margin);

/* y[r] = sum_col (q[r][col] * fp16(s[r][col / gs])) * x[col], for r < rows.
 * q packed per R5 with cols / 2 bytes per row; s has cols / gs per row. */
void orc_gemv_int4(const uint8_t* q, const uint16_t* s, int rows, int cols,
                   int gs, const double* x, double* y);

/* One expert: g = Wg x, u = Wu x, h = silu(g) * u, y = Wd h.
 * x [H], y [H]; h_out [I] nullable. */
void orc_expert_ffn(const orc_cfg* c, const orc_expert* e, const double* x,
                    double* y, double* h_out);

/* Full layer for T tokens: route, then y[t] = sum_j w_j y_{e_j} + y_shared.
 * experts [E], shared (nullable: no shared expert).  Outputs y [T][H],
 * idx [T][k], w [T][k], margin [T] (nullable). */
int orc_layer_forward(const orc_cfg* c, const float* w_router,
                      const float* bias, const orc_expert* experts,
                      const orc_expert* shared, const uint16_t* x_bf16, int T,
                      double* y, int32_t* idx, double* w, double* margin);

/* Expert part only, for given routes (an id of -1 is skipped: a slot
 * dropped by top-p): y[t] = sum_j w[t][j] * FFN_{idx[t][j]}
 * (x_t) + FFN_shared(x_t).  x as doubles [T][H]. */
void orc_experts_combine(const orc_cfg* c, const orc_expert* experts,
                         const orc_expert* shared, const double* x, int T,
                         const int32_t* idx, const double* w, double* y);

/* RMSNorm with unit gain: out = x / sqrt(mean(x^2) + eps). */
void orc_rmsnorm(const double* x, int n, double eps, double* out);

/* Per-layer LRU expert cache simulation (reading R11).  trace [T][L][k]
 * (ids ascending per row), capacity slots per layer, all slots empty at the
 * start.  For each token and layer: ids already cached are hits and are
 * touched in ascending id order; then each missing id, in ascending order,
 * is loaded into an empty slot if there is one, else into the least recently
 * used slot not holding an id of the current token.  hits[l], misses[l]
 * (per layer).  Returns 0, or -1 when capacity < k or args are bad. */
int orc_lru_sim(int n_layers, int n_experts, int capacity, int k, int T,
                const int32_t* trace, uint64_t* hits, uint64_t* misses);
/* orc_lru_sim with n_pin experts per layer (pinned [L][n_pin]) pinned for
 * the whole trace: they always hit and hold n_pin of the slots. */
int orc_lru_sim_pinned(int n_layers, int n_experts, int capacity, int k, int T,
                       const int32_t* trace, int n_pin, const int32_t* pinned,
                       uint64_t* hits, uint64_t* misses);

#ifdef __cplusplus
}
#endif

#endif /* MOE_ORACLE_H */
