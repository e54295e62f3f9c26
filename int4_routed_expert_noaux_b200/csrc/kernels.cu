// kernels.cu -- step kernels of the routed-MoE layer: router GEMV and
// noaux_tc selection for T tokens (moe_route and the batched path), and a
// plain dequantising int4 GEMV for one-hot checks.  The experts of T > 1
// calls run in union.cu; a T = 1 call runs the fused persistent kernel.
#include <cuda_runtime.h>
#include <stdint.h>

#include "common.cuh"
#include "kernels.h"

namespace moe {

// ---------------------------------------------------------------------------
// Router GEMV ("LightLX", "How it works": one router logit per routed
// expert) on the FP64 tensor cores: part[ks][t][e] = the sum over slice ks
// of the K range (H / KS inputs) of w[e][k] x[t][k], by mma m8n8k4 in fp64
// -- every product of an fp32 weight and a bf16 input is exact in fp64, the
// sums are rounded in fp64 (about 1e-16 relative).  The selection kernel
// adds the KS slices in order and takes the sigmoid in fp64.
// CTA (ks, 8-expert tile); warp w: tokens 8w .. 8w + 7.  Within a 16-input
// block the inputs are dealt to the MMA's K index as k = 4 (lane mod 4) + j
// at step j, the same for the A (x) and B (w) fragments, so that each lane
// loads 4 consecutive inputs once.

__device__ __forceinline__ void dmma_8x8x4(double& d0, double& d1, double a, double b) {
  asm volatile(
      "mma.sync.aligned.m8n8k4.row.col.f64.f64.f64.f64 {%0, %1}, {%2}, {%3}, {%0, %1};"
      : "+d"(d0), "+d"(d1)
      : "d"(a), "d"(b));
}

__global__ void __launch_bounds__(256) router_partial_kernel(
    const float* __restrict__ w, const uint16_t* __restrict__ x, int T, int H, int E, int KS,
    double* __restrict__ part) {
  pdl_wait();
  const int ks = blockIdx.x, e0 = blockIdx.y * 8;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int t0 = warp * 8;
  if (t0 >= T) return;
  const int len = H / KS, k0 = ks * len;
  const int r = lane >> 2, c = lane & 3;  // A row (token) and B column (expert); K index
  // rows past T or E read row 0: their results land in D rows / columns
  // that are not stored
  const uint16_t* xr = x + (size_t)(t0 + r < T ? t0 + r : 0) * H + k0 + 4 * c;
  const float* wr = w + (size_t)(e0 + r < E ? e0 + r : 0) * H + k0 + 4 * c;
  // four accumulators (one per step j), added in order at the end: four
  // independent MMA chains instead of one; the next block's loads are in
  // flight while this block's MMAs run
  double d[4][2] = {{0.0, 0.0}, {0.0, 0.0}, {0.0, 0.0}, {0.0, 0.0}};
  uint2 xv = __ldg(reinterpret_cast<const uint2*>(xr));
  float4 wv = __ldg(reinterpret_cast<const float4*>(wr));
  for (int kb = 0; kb < len; kb += 16) {
    const uint2 xc = xv;
    const float4 wc = wv;
    if (kb + 16 < len) {
      xv = __ldg(reinterpret_cast<const uint2*>(xr + kb + 16));
      wv = __ldg(reinterpret_cast<const float4*>(wr + kb + 16));
    }
    dmma_8x8x4(d[0][0], d[0][1], (double)bf16_bits_to_f32(xc.x & 0xFFFFu), (double)wc.x);
    dmma_8x8x4(d[1][0], d[1][1], (double)bf16_bits_to_f32(xc.x >> 16), (double)wc.y);
    dmma_8x8x4(d[2][0], d[2][1], (double)bf16_bits_to_f32(xc.y & 0xFFFFu), (double)wc.z);
    dmma_8x8x4(d[3][0], d[3][1], (double)bf16_bits_to_f32(xc.y >> 16), (double)wc.w);
  }
  // D[row = lane / 4][col = 2 (lane mod 4) + i]: token t0 + row, expert e0 + col
  const int t = t0 + r, e = e0 + 2 * c;
  if (t < T) {
    double* pr = part + ((size_t)ks * T + t) * E;
    if (e < E) pr[e] = ((d[0][0] + d[1][0]) + d[2][0]) + d[3][0];
    if (e + 1 < E) pr[e + 1] = ((d[0][1] + d[1][1]) + d[2][1]) + d[3][1];
  }
}

// ---------------------------------------------------------------------------
// noaux_tc selection (colibri summary, "Principales fonctionnalites
// implementees": DeepSeek-V3 sigmoid router, noaux_tc, routed_scaling_factor).
// One CTA per token; warp g owns group g (lane = expert inside the group):
// sigmoid, bias, top-2 by shuffle arg-max, group score.  Warp 0 then keeps
// topk_group groups and takes the top_k bias-corrected scores inside them by
// repeated warp arg-max (ties to the lower index), sorts the ids ascending
// and normalises the unbiased scores.

struct ArgMax {
  float v;
  int i;
};

// Larger value wins; on equal values the lower index wins.  i < 0 = empty.
__device__ __forceinline__ ArgMax argmax_merge(ArgMax a, ArgMax b) {
  if (a.i < 0) return b;
  if (b.i < 0) return a;
  if (b.v > a.v || (b.v == a.v && b.i < a.i)) return b;
  return a;
}

__device__ __forceinline__ ArgMax warp_argmax(ArgMax a) {
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) {
    ArgMax b;
    b.v = __shfl_xor_sync(0xffffffffu, a.v, o);
    b.i = __shfl_xor_sync(0xffffffffu, a.i, o);
    a = argmax_merge(a, b);
  }
  return a;
}

// A score as an unsigned key in the same order (larger float, larger key);
// 0 is below every score's key.
__device__ __forceinline__ uint32_t sel_key(float v) {
  const uint32_t u = __float_as_uint(v);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

constexpr int kSelQ = 8;  // candidates per lane (E <= 256)

// Compare-exchange of a lane's candidate list: position a before b in the
// order (key descending, expert index ascending).
__device__ __forceinline__ void sel_cx(uint32_t (&key)[kSelQ], int (&jid)[kSelQ], int a, int b) {
  const bool sw = key[b] > key[a] || (key[b] == key[a] && jid[b] < jid[a]);
  const uint32_t ka = key[a], kb = key[b];
  const int ja = jid[a], jb = jid[b];
  key[a] = sw ? kb : ka;
  key[b] = sw ? ka : kb;
  jid[a] = sw ? jb : ja;
  jid[b] = sw ? ja : jb;
}

// Group-limited top-k of one token by one warp, when the groups align with
// lanes: lane l owns experts l*q .. l*q+q-1 and a group is 2^lgL
// consecutive lanes.  Group score = the two largest bias-corrected scores;
// the topk_group best groups (ties: lower index) are kept; the top_k best
// kept experts (ties: lower id) are popped from per-lane sorted lists, one
// warp-wide max per pick.  Lane r < top_k receives the r-th pick.
// Branch-free: no data-dependent guard around a warp collective.
__device__ __forceinline__ int select_fast_warp(const float* s_sel, int E, int q, int lgL,
                                                int n_group, int topk_group, int top_k) {
  const int lane = threadIdx.x & 31;
  const int L = 1 << lgL;
  const int nmine = max(0, min(q, E - lane * q));
  float sp[kSelQ];
#pragma unroll
  for (int j = 0; j < kSelQ; ++j) sp[j] = (j < nmine) ? s_sel[lane * q + j] : -INFINITY;
  float t1 = -INFINITY, t2 = -INFINITY;
#pragma unroll
  for (int j = 0; j < kSelQ; ++j) {
    t2 = fmaxf(t2, fminf(t1, sp[j]));
    t1 = fmaxf(t1, sp[j]);
  }
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const float p1 = __shfl_xor_sync(0xffffffffu, t1, o);
    const float p2 = __shfl_xor_sync(0xffffffffu, t2, o);
    const float n2 = fmaxf(fminf(t1, p1), fmaxf(t2, p2));
    const float n1 = fmaxf(t1, p1);
    t1 = (o < L) ? n1 : t1;
    t2 = (o < L) ? n2 : t2;
  }
  const float gs_seg = ((q << lgL) >= 2) ? t1 + t2 : t1;
  float gs = __shfl_sync(0xffffffffu, gs_seg, (lane < n_group ? lane : 0) << lgL);
  gs = (lane < n_group) ? gs : -INFINITY;
  int rank = 0;
#pragma unroll
  for (int h = 0; h < 32; ++h) {
    const float o = __shfl_sync(0xffffffffu, gs, h);
    rank += (o > gs || (o == gs && h < lane)) ? 1 : 0;
  }
  const unsigned kept_mask = __ballot_sync(0xffffffffu, lane < n_group && rank < topk_group);
  const bool kept = (kept_mask >> (lane >> lgL)) & 1u;
  uint32_t key[kSelQ];
  int jid[kSelQ];
#pragma unroll
  for (int j = 0; j < kSelQ; ++j) {
    key[j] = (j < nmine && kept) ? sel_key(sp[j]) : 0u;
    jid[j] = j;
  }
  sel_cx(key, jid, 0, 1); sel_cx(key, jid, 2, 3); sel_cx(key, jid, 4, 5); sel_cx(key, jid, 6, 7);
  sel_cx(key, jid, 0, 2); sel_cx(key, jid, 1, 3); sel_cx(key, jid, 4, 6); sel_cx(key, jid, 5, 7);
  sel_cx(key, jid, 1, 2); sel_cx(key, jid, 5, 6);
  sel_cx(key, jid, 0, 4); sel_cx(key, jid, 1, 5); sel_cx(key, jid, 2, 6); sel_cx(key, jid, 3, 7);
  sel_cx(key, jid, 2, 4); sel_cx(key, jid, 3, 5);
  sel_cx(key, jid, 1, 2); sel_cx(key, jid, 3, 4); sel_cx(key, jid, 5, 6);
  int my_sel = -1;
  for (int r = 0; r < top_k; ++r) {
    const uint32_t m = __reduce_max_sync(0xffffffffu, key[0]);
    bool own = key[0] == m && m != 0u;
    const uint32_t cand = own ? (uint32_t)(lane * q + jid[0]) : 0xFFFFFFFFu;
    const uint32_t best = __reduce_min_sync(0xffffffffu, cand);  // ties: the lower id
    own = own && cand == best;
    if (lane == r) my_sel = (best == 0xFFFFFFFFu) ? -1 : (int)best;
#pragma unroll
    for (int j = 0; j + 1 < kSelQ; ++j) {  // pop the owner's head
      key[j] = own ? key[j + 1] : key[j];
      jid[j] = own ? jid[j + 1] : jid[j];
    }
    key[kSelQ - 1] = own ? 0u : key[kSelQ - 1];
  }
  return my_sel;
}

__global__ void __launch_bounds__(1024) select_kernel(
    const double* __restrict__ part, int KS, int T, const float* __restrict__ bias, int E,
    int n_group, int topk_group, int top_k, float rsf, float top_p, int sel_q, int sel_lgL,
    int sel_fast, int32_t* __restrict__ idx_out, float* __restrict__ w_out,
    float* __restrict__ scores_out) {
  pdl_wait();
  __shared__ float s_score[1024];
  __shared__ float s_sel[1024];
  __shared__ float s_group[32];
  const int t = blockIdx.x;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int per = E / n_group;

  if (warp < n_group) {
    const int e = warp * per + lane;
    ArgMax a{0.f, -1};
    if (lane < per) {
      // the logit: the K slices added in order; the sigmoid in fp64,
      // rounded to fp32 once
      double lg = 0.0;
      for (int k0 = 0; k0 < KS; k0 += 8) {  // 8 loads in flight at a time
        double pk[8];
#pragma unroll
        for (int j = 0; j < 8; ++j)
          pk[j] = k0 + j < KS ? part[((size_t)(k0 + j) * T + t) * E + e] : 0.0;
#pragma unroll
        for (int j = 0; j < 8; ++j) lg += pk[j];
      }
      const float s = sigmoid_f64_to_f32(lg);
      const float sp = s + bias[e];
      s_score[e] = s;
      s_sel[e] = sp;
      if (scores_out) scores_out[(size_t)t * E + e] = s;
      a = ArgMax{sp, e};
    }
    const ArgMax top1 = warp_argmax(a);
    ArgMax b = a;
    if (b.i == top1.i) b.i = -1;
    const ArgMax top2 = warp_argmax(b);
    if (lane == 0) s_group[warp] = (top2.i >= 0) ? top1.v + top2.v : top1.v;
  }
  __syncthreads();
  if (warp != 0) return;

  int my_sel = -1;  // id selected in round == lane
  if (sel_fast) {
    my_sel = select_fast_warp(s_sel, E, sel_q, sel_lgL, n_group, topk_group, top_k);
  } else {
    // keep topk_group groups (lane = group)
    bool kept = false;
    {
      ArgMax g{lane < n_group ? s_group[lane] : 0.f, lane < n_group ? lane : -1};
      for (int r = 0; r < topk_group; ++r) {
        ArgMax cand = kept ? ArgMax{0.f, -1} : g;
        const ArgMax best = warp_argmax(cand);
        if (best.i == lane) kept = true;
      }
    }
    const unsigned kept_mask = __ballot_sync(0xffffffffu, kept);

    // top_k over experts of kept groups; lane holds experts lane + 32 * m
    const int nper = (E + 31) >> 5;
    unsigned taken = 0;  // bit m: expert lane + 32m already selected
    for (int r = 0; r < top_k; ++r) {
      ArgMax a{0.f, -1};
      for (int m = 0; m < nper; ++m) {
        const int e = lane + 32 * m;
        if (e < E && ((kept_mask >> (e / per)) & 1u) && !((taken >> m) & 1u))
          a = argmax_merge(a, ArgMax{s_sel[e], e});
      }
      const ArgMax best = warp_argmax(a);
      if (best.i >= 0 && (best.i & 31) == lane) taken |= 1u << (best.i >> 5);
      if (lane == r) my_sel = best.i;
    }
  }
  const float s_mine = (lane < top_k && my_sel >= 0) ? s_score[my_sel] : 0.f;
  const float denom = warp_sum(s_mine) + 1e-20f;
  if (top_p >= 1.f) {
    // rank of each selected id among the selected ids = output position
    int rank = 0;
    for (int j = 0; j < top_k; ++j) {
      const int other = __shfl_sync(0xffffffffu, my_sel, j);
      if (lane < top_k && other < my_sel) ++rank;
    }
    if (lane < top_k) {
      idx_out[(size_t)t * top_k + rank] = my_sel;
      w_out[(size_t)t * top_k + rank] = rsf * s_mine / denom;
    }
  } else {
    // adaptive top-p: the kept picks, weights normalised over them
    const bool kept = topp_keep(my_sel, s_mine, denom, top_k, top_p);
    const float denom_k = warp_sum(kept ? s_mine : 0.f) + 1e-20f;
    const int pos = topp_position(my_sel, kept, top_k);
    if (lane < top_k) {
      idx_out[(size_t)t * top_k + pos] = kept ? my_sel : -1;
      w_out[(size_t)t * top_k + pos] = kept ? rsf * s_mine / denom_k : 0.f;
    }
  }
}

// ---------------------------------------------------------------------------
// Plain dequantising int4 GEMV, y[r] = sum_c q[r][c] * scale[r][c/32] * x[c]
// (fp32 x and y), built from the same group dot product as the layer
// kernels.  Exposed for one-hot checks of the packing and scale indexing.

__device__ __forceinline__ void load_x_group_f32(const float* __restrict__ hp, XQ& xg) {
  float xf[32];
  const float4* p4 = reinterpret_cast<const float4*>(hp);
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const float4 v = p4[i];
    xf[4 * i] = v.x;
    xf[4 * i + 1] = v.y;
    xf[4 * i + 2] = v.z;
    xf[4 * i + 3] = v.w;
  }
  xq_from_floats(xf, xg);
}

template <int SEG, int NV>
__global__ void __launch_bounds__(256) gemv_int4_kernel(
    const uint8_t* __restrict__ q, const uint16_t* __restrict__ s, int rows, int cols,
    const float* __restrict__ x, float* __restrict__ y) {
  __shared__ float red[32][33];
  const int G = cols >> 5;
  const ColMap cm = col_map(G);
  const int row0 = blockIdx.x * cm.P * NV;
  XQ xg;
  load_x_group_f32(x + cm.col * 32, xg);
  float acc[NV];
#pragma unroll
  for (int r = 0; r < NV; ++r) {
    const int row = row0 + cm.phase * NV + r;
    acc[r] = 0.f;
    if (row < rows) {
      const uint4 w = __ldg(reinterpret_cast<const uint4*>(q + (size_t)row * (cols / 2)) + cm.col);
      const float sc = f16_bits_to_f32(__ldg(s + (size_t)row * G + cm.col));
      acc[r] = dot_scaled(w, xg, sc);
    }
  }
  reduce_scatter<NV, SEG>(acc);
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int vi = reduce_index<NV, SEG>(lane);
  const bool owner = (lane % (SEG / NV)) == 0;
  const int row = row0 + cm.phase * NV + vi;
  if (cm.wpr == 1) {
    if (owner && row < rows) y[row] = acc[0];
  } else {
    red[warp][lane] = acc[0];
    __syncthreads();
    if (cm.wir == 0 && owner && row < rows) {
      float t = 0.f;
      for (int w = 0; w < cm.wpr; ++w) t += red[warp + w][lane];
      y[row] = t;
    }
  }
}

// ---------------------------------------------------------------------------
// launchers

static int warps_for(int G) {
  if (G >= 32) {
    const int wpr = G / 32;
    return wpr >= 8 ? wpr : wpr * (8 / wpr);
  }
  return 4;
}

// Slices of the router's K range: more for fewer tokens (a CTA's warps
// take 8 tokens each), so that every call keeps the SMs busy.
int router_slices(int H, int T) {
  const int want = T <= 8 ? 32 : T <= 16 ? 16 : 8;
  for (int ks = want; ks > 1; ks >>= 1)
    if (H % (16 * ks) == 0) return ks;
  return 1;
}

cudaError_t launch_router_partial(const float* w, const uint16_t* x, int T, int H, int E,
                                  double* part, cudaStream_t st) {
  if (H % 16 != 0 || T < 1 || T > 64) return cudaErrorInvalidValue;
  const int ks = router_slices(H, T);
  launch_pdl(router_partial_kernel, dim3(ks, (E + 7) / 8), dim3(32 * ((T + 7) / 8)), 0, st, w, x,
             T, H, E, ks, part);
  return cudaGetLastError();
}

cudaError_t launch_select(const double* part, int H, const float* bias, int T, int E,
                          int n_group, int topk_group, int top_k, float rsf, float top_p,
                          int32_t* idx, float* w, float* scores_out, cudaStream_t st) {
  // the one-warp fast selection when the groups align with lanes (as in
  // the one-token kernel), else the generic rounds
  const int per = E / n_group, q = (E + 31) / 32;
  int lgL = 0;
  while ((1 << lgL) < per / q) ++lgL;
  const int fast = per % q == 0 && per / q >= 1 && (1 << lgL) == per / q && q <= kSelQ;
  launch_pdl(select_kernel, dim3(T), dim3(32 * n_group), 0, st, part, router_slices(H, T), T, bias,
             E, n_group, topk_group, top_k, rsf, top_p, q, lgL, fast, idx, w, scores_out);
  return cudaGetLastError();
}

template <int SEG, int NV>
static cudaError_t gemv_seg(const uint8_t* q, const uint16_t* s, int rows, int cols,
                            const float* x, float* y, cudaStream_t st) {
  const int G = cols / 32;
  const int nw = warps_for(G);
  const int P = (G >= 32) ? nw / (G / 32) : nw * (32 / G);
  const int per = P * NV;
  gemv_int4_kernel<SEG, NV><<<(rows + per - 1) / per, nw * 32, 0, st>>>(q, s, rows, cols, x, y);
  return cudaGetLastError();
}

cudaError_t launch_gemv_int4(const uint8_t* q, const uint16_t* s, int rows, int cols,
                             const float* x, float* y, cudaStream_t st) {
  const int G = cols / 32;
  switch (G >= 32 ? 32 : G) {
    case 32: return gemv_seg<32, 4>(q, s, rows, cols, x, y, st);
    case 16: return gemv_seg<16, 4>(q, s, rows, cols, x, y, st);
    case 8: return gemv_seg<8, 4>(q, s, rows, cols, x, y, st);
    case 4: return gemv_seg<4, 4>(q, s, rows, cols, x, y, st);
    case 2: return gemv_seg<2, 2>(q, s, rows, cols, x, y, st);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace moe
