/*
 * oracle.c -- fp64 CPU oracle of the routed MoE decode layer.
 *
 * TEST INFRASTRUCTURE ONLY (see oracle.h): plain loops, double precision,
 * no blocking or reordering beyond the definitions cited per function.
 */
#include "oracle.h"

#include <math.h>
#include <stdlib.h>
#include <string.h>

#ifdef _OPENMP
#include <omp.h>
#endif

/* ---- number formats -------------------------------------------------- */

double orc_bf16_value(uint16_t b) {
  /* bfloat16 is the upper half of an IEEE binary32. */
  uint32_t u = (uint32_t)b << 16;
  float f;
  memcpy(&f, &u, 4);
  return (double)f;
}

double orc_f16_value(uint16_t h) {
  /* IEEE binary16: 1 sign, 5 exponent (bias 15), 10 fraction bits. */
  int sign = (h >> 15) & 1;
  int e = (h >> 10) & 0x1F;
  int f = h & 0x3FF;
  double v;
  if (e == 0)
    v = ldexp((double)f, -24);                 /* subnormal: f * 2^-24 */
  else if (e == 31)
    v = f ? NAN : INFINITY;
  else
    v = ldexp(1.0 + (double)f / 1024.0, e - 15);
  return sign ? -v : v;
}

uint16_t orc_round_bf16(double v) {
  /* Round to the nearest bf16 (8 significant bits), ties to even, by
   * scaling the significand: frexp gives v = m * 2^e with 0.5 <= |m| < 1. */
  if (v == 0.0 || !isfinite(v)) {
    float f = (float)v;
    uint32_t u;
    memcpy(&u, &f, 4);
    return (uint16_t)(u >> 16);
  }
  int e;
  double m = frexp(v, &e);                    /* |m| in [0.5, 1) */
  double scaled = ldexp(m, 8);                /* 8 significant bits */
  double r = nearbyint(scaled);               /* FE_TONEAREST: ties-to-even */
  double q = ldexp(r, e - 8);
  float f = (float)q;                         /* exact: q has <= 8 bits */
  uint32_t u;
  memcpy(&u, &f, 4);
  return (uint16_t)(u >> 16);
}

int orc_set_threads(int n) {
#ifdef _OPENMP
  if (n > 0) omp_set_num_threads(n);
  return omp_get_max_threads();
#else
  (void)n;
  return 1;
#endif
}

/* ---- router ------------------------------------------------------------ */

/* Router GEMV: one logit per routed expert (the gate of a DeepSeek-V3 style
 * MoE layer; "LightLX", "How it works"). */
void orc_router_logits(const orc_cfg* c, const float* w_router,
                       const uint16_t* x_bf16, int T, double* logits) {
  const int H = c->hidden, E = c->n_experts;
  for (int t = 0; t < T; ++t) {
#pragma omp parallel for schedule(static)
    for (int e = 0; e < E; ++e) {
      double acc = 0.0;
      for (int h = 0; h < H; ++h)
        acc += (double)w_router[(size_t)e * H + h] *
               orc_bf16_value(x_bf16[(size_t)t * H + h]);
      logits[(size_t)t * E + e] = acc;
    }
  }
}

/* noaux_tc selection for one token (colibri summary, "Principales
 * fonctionnalites implementees": sigmoid router, noaux_tc,
 * routed_scaling_factor; readings R1-R4). */
static int select_one(const orc_cfg* c, const double* s, const double* sp,
                      int round_group_f32, int32_t* idx, double* w,
                      double* margin) {
  const int E = c->n_experts, G = c->n_group, k = c->top_k;
  const int TG = c->topk_group, per = E / G;
  double* gscore = (double*)malloc(sizeof(double) * (size_t)G);
  char* gkeep = (char*)calloc((size_t)G, 1);
  char* taken = (char*)calloc((size_t)E, 1);
  if (!gscore || !gkeep || !taken) {
    free(gscore); free(gkeep); free(taken);
    return -1;
  }

  /* R1: group score = sum of the two largest sp in the group. */
  for (int g = 0; g < G; ++g) {
    int best = -1, second = -1;
    for (int e = g * per; e < (g + 1) * per; ++e) {
      if (best < 0 || sp[e] > sp[best]) {
        second = best;
        best = e;
      } else if (second < 0 || sp[e] > sp[second]) {
        second = e;
      }
    }
    double a = sp[best];
    double b = (second >= 0) ? sp[second] : 0.0;
    if (round_group_f32)
      gscore[g] = (double)((float)a + (float)b);
    else
      gscore[g] = a + b;
  }

  /* Keep the TG best groups; R3: the lower group index wins a tie. */
  double last_kept = INFINITY;
  for (int r = 0; r < TG; ++r) {
    int best = -1;
    for (int g = 0; g < G; ++g)
      if (!gkeep[g] && (best < 0 || gscore[g] > gscore[best])) best = g;
    gkeep[best] = 1;
    last_kept = gscore[best];
  }
  double next_group = -INFINITY;
  for (int g = 0; g < G; ++g)
    if (!gkeep[g] && gscore[g] > next_group) next_group = gscore[g];
  double group_gap = (TG < G) ? last_kept - next_group : INFINITY;

  /* Top-k of sp over experts of kept groups (R2: others excluded);
   * R3: the lower expert index wins a tie. */
  double last_sel = INFINITY;
  for (int r = 0; r < k; ++r) {
    int best = -1;
    for (int e = 0; e < E; ++e) {
      if (!gkeep[e / per] || taken[e]) continue;
      if (best < 0 || sp[e] > sp[best]) best = e;
    }
    if (best < 0) {
      free(gscore); free(gkeep); free(taken);
      return -1;
    }
    taken[best] = 1;
    last_sel = sp[best];
  }
  double next_sel = -INFINITY;
  for (int e = 0; e < E; ++e)
    if (gkeep[e / per] && !taken[e] && sp[e] > next_sel) next_sel = sp[e];
  double expert_gap = (next_sel == -INFINITY) ? INFINITY : last_sel - next_sel;

  /* Ascending expert ids; weights from the unbiased scores (R4). */
  int j = 0;
  double denom = 0.0;
  for (int e = 0; e < E; ++e)
    if (taken[e]) {
      idx[j++] = e;
      denom += s[e];
    }
  denom += 1e-20;
  for (j = 0; j < k; ++j) w[j] = c->rsf * s[idx[j]] / denom;
  if (margin) *margin = (group_gap < expert_gap) ? group_gap : expert_gap;

  free(gscore); free(gkeep); free(taken);
  return 0;
}

static int cfg_ok(const orc_cfg* c) {
  return c && c->n_experts > 0 && c->n_group > 0 &&
         c->n_experts % c->n_group == 0 && c->topk_group >= 1 &&
         c->topk_group <= c->n_group && c->top_k >= 1 &&
         c->top_k <= c->topk_group * (c->n_experts / c->n_group);
}

int orc_select_scores(const orc_cfg* c, const double* s, const double* sp,
                      int T, int round_group_f32, int32_t* idx, double* w,
                      double* margin) {
  if (!cfg_ok(c) || T < 0) return -1;
  const int E = c->n_experts, k = c->top_k;
  for (int t = 0; t < T; ++t)
    if (select_one(c, s + (size_t)t * E, sp + (size_t)t * E, round_group_f32,
                   idx + (size_t)t * k, w + (size_t)t * k,
                   margin ? margin + t : NULL))
      return -1;
  return 0;
}

int orc_route(const orc_cfg* c, const double* logits, const float* bias,
              int T, int32_t* idx, double* w, double* margin,
              double* scores_out) {
  if (!cfg_ok(c) || T < 0) return -1;
  const int E = c->n_experts;
  size_t n = (size_t)T * E;
  double* s = (double*)malloc(sizeof(double) * (n ? n : 1));
  double* sp = (double*)malloc(sizeof(double) * (n ? n : 1));
  if (!s || !sp) {
    free(s); free(sp);
    return -1;
  }
  for (size_t i = 0; i < n; ++i) {
    s[i] = 1.0 / (1.0 + exp(-logits[i]));          /* sigmoid score */
    sp[i] = s[i] + (double)bias[i % (size_t)E];    /* selection score */
  }
  int rc = orc_select_scores(c, s, sp, T, 0, idx, w, margin);
  if (scores_out && rc == 0) memcpy(scores_out, s, sizeof(double) * n);
  free(s); free(sp);
  return rc;
}

/* Adaptive expert top-p (colibri summary, "Telechargement et execution du
 * modele": the --topp 0.7 option, adaptive expert top-p, and "Benchmarks
 * communautaires"; the pages give no formula, reading R16): of the k
 * selected experts, keep the fewest, taken in descending weight (ties: the
 * lower id first), whose weights add up to at least p * rsf; the kept
 * weights are normalised again over the kept experts (R4 on the kept set).
 * Kept ids ascending first, then -1 with weight 0 for the dropped slots.
 * p >= 1 keeps all k. */
int orc_topp(const orc_cfg* c, const double* s, int T, double p, int32_t* idx,
             double* w, int32_t* n_keep, double* margin) {
  if (!cfg_ok(c) || T < 0 || !(p > 0.0)) return -1;
  const int E = c->n_experts, k = c->top_k;
  int32_t* ord = (int32_t*)malloc(sizeof(int32_t) * (size_t)k);
  int32_t* kept = (int32_t*)malloc(sizeof(int32_t) * (size_t)k);
  if (!ord || !kept) {
    free(ord); free(kept);
    return -1;
  }
  for (int t = 0; t < T; ++t) {
    int32_t* it = idx + (size_t)t * k;
    double* wt = w + (size_t)t * k;
    const double* st = s + (size_t)t * E;
    /* positions of the k selected experts in descending weight, ties to
     * the lower id (selection sort: k is small) */
    char* used = (char*)calloc((size_t)k, 1);
    for (int r = 0; r < k; ++r) {
      int best = -1;
      for (int j = 0; j < k; ++j) {
        if (used[j]) continue;
        if (best < 0 || wt[j] > wt[best] || (wt[j] == wt[best] && it[j] < it[best])) best = j;
      }
      used[best] = 1;
      ord[r] = best;
    }
    free(used);
    /* the shortest prefix whose share of rsf reaches p */
    int m = k;
    double cum = 0.0, before = 0.0;
    if (p < 1.0) {
      for (int r = 0; r < k; ++r) {
        before = cum;
        cum += wt[ord[r]] / c->rsf;
        if (cum >= p) {
          m = r + 1;
          break;
        }
      }
    }
    double mg = INFINITY;
    if (p < 1.0 && m <= k) {
      const double a = cum - p, b = p - before;
      mg = a < b ? a : b;
      if (m < k) {
        const double gap = (wt[ord[m - 1]] - wt[ord[m]]) / c->rsf;
        if (gap < mg) mg = gap;
      }
    }
    /* kept ids ascending; weights from the unbiased scores over the kept */
    for (int r = 0; r < m; ++r) kept[r] = it[ord[r]];
    for (int a = 1; a < m; ++a)
      for (int b = a; b > 0 && kept[b - 1] > kept[b]; --b) {
        const int32_t tmp = kept[b];
        kept[b] = kept[b - 1];
        kept[b - 1] = tmp;
      }
    double denom = 0.0;
    for (int r = 0; r < m; ++r) denom += st[kept[r]];
    denom += 1e-20;
    for (int r = 0; r < k; ++r) {
      if (r < m) {
        it[r] = kept[r];
        wt[r] = c->rsf * st[kept[r]] / denom;
      } else {
        it[r] = -1;
        wt[r] = 0.0;
      }
    }
    if (n_keep) n_keep[t] = m;
    if (margin) margin[t] = mg;
  }
  free(ord); free(kept);
  return 0;
}

/* ---- experts ------------------------------------------------------------ */

/* Dequantise-on-use GEMV of a packed int4 matrix (colibri summary: int4
 * kernels with dequant-on-use; format per the layer's spec and R5). */
void orc_gemv_int4(const uint8_t* q, const uint16_t* s, int rows, int cols,
                   int gs, const double* x, double* y) {
  const int row_bytes = cols / 2, row_scales = cols / gs;
#pragma omp parallel for schedule(static)
  for (int r = 0; r < rows; ++r) {
    double acc = 0.0;
    for (int col = 0; col < cols; ++col) {
      uint8_t byte = q[(size_t)r * row_bytes + col / 2];
      int nib = (col % 2 == 0) ? (byte & 0x0F) : (byte >> 4);
      int code = (nib >= 8) ? nib - 16 : nib;      /* two's complement */
      double scale = orc_f16_value(s[(size_t)r * row_scales + col / gs]);
      acc += ((double)code * scale) * x[col];
    }
    y[r] = acc;
  }
}

/* SwiGLU expert: down(silu(gate x) * up x) ("LightLX", section "Run any
 * model": the SwitchGLU expert module). */
void orc_expert_ffn(const orc_cfg* c, const orc_expert* e, const double* x,
                    double* y, double* h_out) {
  const int H = c->hidden, I = c->inter, gs = c->group_size;
  double* g = (double*)malloc(sizeof(double) * (size_t)I);
  double* u = (double*)malloc(sizeof(double) * (size_t)I);
  double* h = (double*)malloc(sizeof(double) * (size_t)I);
  orc_gemv_int4(e->q_gate, e->s_gate, I, H, gs, x, g);
  orc_gemv_int4(e->q_up, e->s_up, I, H, gs, x, u);
  for (int i = 0; i < I; ++i) h[i] = g[i] / (1.0 + exp(-g[i])) * u[i];
  orc_gemv_int4(e->q_down, e->s_down, H, I, gs, h, y);
  if (h_out) memcpy(h_out, h, sizeof(double) * (size_t)I);
  free(g); free(u); free(h);
}

void orc_experts_combine(const orc_cfg* c, const orc_expert* experts,
                         const orc_expert* shared, const double* x, int T,
                         const int32_t* idx, const double* w, double* y) {
  const int H = c->hidden, k = c->top_k;
  double* ye = (double*)malloc(sizeof(double) * (size_t)H);
  for (int t = 0; t < T; ++t) {
    const double* xt = x + (size_t)t * H;
    double* yt = y + (size_t)t * H;
    for (int h = 0; h < H; ++h) yt[h] = 0.0;
    for (int j = 0; j < k; ++j) {
      if (idx[(size_t)t * k + j] < 0) continue;   /* dropped by top-p (R16) */
      orc_expert_ffn(c, &experts[idx[(size_t)t * k + j]], xt, ye, NULL);
      for (int h = 0; h < H; ++h) yt[h] += w[(size_t)t * k + j] * ye[h];
    }
    if (shared) {
      orc_expert_ffn(c, shared, xt, ye, NULL);
      for (int h = 0; h < H; ++h) yt[h] += ye[h];
    }
  }
  free(ye);
}

int orc_layer_forward(const orc_cfg* c, const float* w_router,
                      const float* bias, const orc_expert* experts,
                      const orc_expert* shared, const uint16_t* x_bf16, int T,
                      double* y, int32_t* idx, double* w, double* margin) {
  if (!cfg_ok(c) || T < 0) return -1;
  const int H = c->hidden, E = c->n_experts;
  double* logits = (double*)malloc(sizeof(double) * ((size_t)T * E + 1));
  double* x = (double*)malloc(sizeof(double) * ((size_t)T * H + 1));
  orc_router_logits(c, w_router, x_bf16, T, logits);
  int rc = orc_route(c, logits, bias, T, idx, w, margin, NULL);
  if (rc == 0) {
    for (size_t i = 0; i < (size_t)T * H; ++i) x[i] = orc_bf16_value(x_bf16[i]);
    orc_experts_combine(c, experts, shared, x, T, idx, w, y);
  }
  free(logits); free(x);
  return rc;
}

/* RMSNorm with unit gain ("LightLX", "How it works": RMSNorm of the
 * upstream model; reading R9 for the stacked layers). */
void orc_rmsnorm(const double* x, int n, double eps, double* out) {
  double ss = 0.0;
  for (int i = 0; i < n; ++i) ss += x[i] * x[i];
  double inv = 1.0 / sqrt(ss / (double)n + eps);
  for (int i = 0; i < n; ++i) out[i] = x[i] * inv;
}

/* ---- per-layer LRU expert cache (colibri summary: per-layer LRU cache of
 * routed experts; reading R11) ------------------------------------------ */

int orc_lru_sim(int n_layers, int n_experts, int capacity, int k, int T,
                const int32_t* trace, uint64_t* hits, uint64_t* misses) {
  if (n_layers <= 0 || capacity < k || k <= 0 || T < 0 || !trace) return -1;
  int32_t* slot_id = (int32_t*)malloc(sizeof(int32_t) * (size_t)capacity);
  uint64_t* stamp = (uint64_t*)malloc(sizeof(uint64_t) * (size_t)capacity);
  for (int l = 0; l < n_layers; ++l) {
    uint64_t clock = 0, h = 0, m = 0;
    for (int i = 0; i < capacity; ++i) { slot_id[i] = -1; stamp[i] = 0; }
    for (int t = 0; t < T; ++t) {
      const int32_t* ids = trace + ((size_t)t * n_layers + l) * (size_t)k;
      /* hits, ascending id order */
      for (int j = 0; j < k; ++j) {
        if (ids[j] < 0 || ids[j] >= n_experts) {
          free(slot_id); free(stamp);
          return -1;
        }
        for (int i = 0; i < capacity; ++i)
          if (slot_id[i] == ids[j]) {
            stamp[i] = ++clock;
            ++h;
            break;
          }
      }
      /* misses, ascending id order */
      for (int j = 0; j < k; ++j) {
        int found = 0;
        for (int i = 0; i < capacity; ++i)
          if (slot_id[i] == ids[j]) { found = 1; break; }
        if (found) continue;
        int victim = -1;
        for (int i = 0; i < capacity && victim < 0; ++i)
          if (slot_id[i] < 0) victim = i;
        if (victim < 0) {
          for (int i = 0; i < capacity; ++i) {
            int current = 0;
            for (int jj = 0; jj < k; ++jj)
              if (slot_id[i] == ids[jj]) current = 1;
            if (current) continue;
            if (victim < 0 || stamp[i] < stamp[victim]) victim = i;
          }
        }
        slot_id[victim] = ids[j];
        stamp[victim] = ++clock;
        ++m;
      }
    }
    hits[l] = h;
    misses[l] = m;
  }
  free(slot_id); free(stamp);
  return 0;
}

/* Per-layer LRU with a pinned hot-store (colibri summary, "Learning cache et
 * attentes selon le materiel": the most used experts are pinned at start-up;
 * reading R19).  The n_pin experts pinned[l][..] of layer l occupy n_pin of
 * the capacity slots for the whole trace and always hit; every other id runs
 * the LRU rule of orc_lru_sim over the remaining capacity - n_pin slots,
 * which start empty. */
int orc_lru_sim_pinned(int n_layers, int n_experts, int capacity, int k, int T,
                       const int32_t* trace, int n_pin, const int32_t* pinned,
                       uint64_t* hits, uint64_t* misses) {
  if (n_layers <= 0 || k <= 0 || T < 0 || !trace || n_pin < 0 || capacity - n_pin < k ||
      (n_pin > 0 && !pinned))
    return -1;
  const int free_slots = capacity - n_pin;
  int32_t* slot_id = (int32_t*)malloc(sizeof(int32_t) * (size_t)free_slots);
  uint64_t* stamp = (uint64_t*)malloc(sizeof(uint64_t) * (size_t)free_slots);
  char* is_pinned = (char*)malloc((size_t)n_experts);
  int rc = 0;
  for (int l = 0; l < n_layers && rc == 0; ++l) {
    uint64_t clock = 0, h = 0, m = 0;
    memset(is_pinned, 0, (size_t)n_experts);
    for (int j = 0; j < n_pin; ++j) {
      const int32_t e = pinned[(size_t)l * n_pin + j];
      if (e < 0 || e >= n_experts || is_pinned[e]) { rc = -1; break; }
      is_pinned[e] = 1;
    }
    for (int i = 0; i < free_slots; ++i) { slot_id[i] = -1; stamp[i] = 0; }
    for (int t = 0; t < T && rc == 0; ++t) {
      const int32_t* ids = trace + ((size_t)t * n_layers + l) * (size_t)k;
      for (int j = 0; j < k; ++j)
        if (ids[j] < 0 || ids[j] >= n_experts) rc = -1;
      if (rc) break;
      /* pinned ids hit; cached ids hit and are touched, ascending */
      for (int j = 0; j < k; ++j) {
        if (is_pinned[ids[j]]) { ++h; continue; }
        for (int i = 0; i < free_slots; ++i)
          if (slot_id[i] == ids[j]) { stamp[i] = ++clock; ++h; break; }
      }
      /* the other ids, ascending: lowest empty slot, else the least
       * recently used slot not holding one of this call's ids */
      for (int j = 0; j < k; ++j) {
        if (is_pinned[ids[j]]) continue;
        int found = 0;
        for (int i = 0; i < free_slots; ++i)
          if (slot_id[i] == ids[j]) { found = 1; break; }
        if (found) continue;
        int victim = -1;
        for (int i = 0; i < free_slots && victim < 0; ++i)
          if (slot_id[i] < 0) victim = i;
        if (victim < 0) {
          for (int i = 0; i < free_slots; ++i) {
            int current = 0;
            for (int jj = 0; jj < k; ++jj)
              if (slot_id[i] == ids[jj]) current = 1;
            if (current) continue;
            if (victim < 0 || stamp[i] < stamp[victim]) victim = i;
          }
        }
        slot_id[victim] = ids[j];
        stamp[victim] = ++clock;
        ++m;
      }
    }
    hits[l] = h;
    misses[l] = m;
  }
  free(slot_id); free(stamp); free(is_pinned);
  return rc;
}
