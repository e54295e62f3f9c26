// kernels.cu -- step kernels of the routed-MoE layer: router GEMV, noaux_tc
// selection, fused int4 gate/up + SiLU, int4 down projection with the
// weighted combine.  Used by moe_route / moe_expert_ffn and by the batched
// path; the T = 1 decode path uses the fused persistent kernel instead.
#include <cuda_runtime.h>
#include <stdint.h>

#include "common.cuh"
#include "kernels.h"

namespace moe {

// ---------------------------------------------------------------------------
// Router GEMV ("LightLX", "How it works": one router logit per routed
// expert).  One warp per expert row of W (fp32 [E][H]); lanes stride the row
// in 16-byte chunks (4 weights); all T tokens are accumulated per chunk.
// logits [T][E].

template <int TT>
__global__ void __launch_bounds__(256) router_logits_kernel(
    const float* __restrict__ w, const uint16_t* __restrict__ x, int T, int H,
    int E, float* __restrict__ logits) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int e = blockIdx.x * (blockDim.x >> 5) + warp;
  if (e >= E) return;
  const float4* wr = reinterpret_cast<const float4*>(w + (size_t)e * H);
  const int nchunk = H >> 2;
  for (int t0 = 0; t0 < T; t0 += TT) {
    float acc[TT];
#pragma unroll
    for (int t = 0; t < TT; ++t) acc[t] = 0.f;
    for (int c = lane; c < nchunk; c += 32) {
      const float4 wv = __ldg(wr + c);
#pragma unroll
      for (int t = 0; t < TT; ++t) {
        if (t0 + t < T) {
          const uint2 xv = __ldg(reinterpret_cast<const uint2*>(x + (size_t)(t0 + t) * H) + c);
          acc[t] = fmaf(wv.x, bf16_bits_to_f32(xv.x & 0xFFFFu), acc[t]);
          acc[t] = fmaf(wv.y, bf16_bits_to_f32(xv.x >> 16), acc[t]);
          acc[t] = fmaf(wv.z, bf16_bits_to_f32(xv.y & 0xFFFFu), acc[t]);
          acc[t] = fmaf(wv.w, bf16_bits_to_f32(xv.y >> 16), acc[t]);
        }
      }
    }
#pragma unroll
    for (int t = 0; t < TT; ++t) {
      const float s = warp_sum(acc[t]);
      if (lane == 0 && t0 + t < T) logits[(size_t)(t0 + t) * E + e] = s;
    }
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

__global__ void __launch_bounds__(1024) select_kernel(
    const float* __restrict__ logits, const float* __restrict__ bias, int E,
    int n_group, int topk_group, int top_k, float rsf,
    int32_t* __restrict__ idx_out, float* __restrict__ w_out,
    float* __restrict__ scores_out) {
  __shared__ float s_score[1024];
  __shared__ float s_sel[1024];
  __shared__ float s_group[32];
  const int t = blockIdx.x;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int per = E / n_group;
  const float* lg = logits + (size_t)t * E;

  if (warp < n_group) {
    const int e = warp * per + lane;
    ArgMax a{0.f, -1};
    if (lane < per) {
      const float s = 1.0f / (1.0f + expf(-lg[e]));
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
  int my_sel = -1;     // id selected in round == lane
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
  // rank of each selected id among the selected ids = output position
  int rank = 0;
  for (int j = 0; j < top_k; ++j) {
    const int other = __shfl_sync(0xffffffffu, my_sel, j);
    if (lane < top_k && other < my_sel) ++rank;
  }
  const float s_mine = (lane < top_k && my_sel >= 0) ? s_score[my_sel] : 0.f;
  const float denom = warp_sum(s_mine) + 1e-20f;
  if (lane < top_k) {
    idx_out[(size_t)t * top_k + rank] = my_sel;
    w_out[(size_t)t * top_k + rank] = rsf * s_mine / denom;
  }
}

// ---------------------------------------------------------------------------
// Fused int4 gate/up + SiLU (one expert slot, a block of rows).  Column-
// stationary: thread (col, phase) owns 16-byte chunk column `col` of every
// row it visits, so its 32 inputs stay in registers as an XQ.  Each
// phase handles NR rows of gate and NR of up; one butterfly reduce-scatter
// sums the 2*NR partial dots over the row's threads (with NV == SEG, lane l
// of a segment ends with value index l % SEG: gate row r at r, up row r at
// NR + r).  h = silu(g) * u is written to hbuf; g and u never leave the CTA.
// grid.x = row blocks of `inter`, grid.y = token * slots + slot.

__device__ __forceinline__ void load_x_group_bf16(const uint16_t* __restrict__ xp, XQ& xg) {
  float xf[32];
  const uint4* p4 = reinterpret_cast<const uint4*>(xp);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const uint4 v = __ldg(p4 + i);
    const uint32_t u[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      xf[8 * i + 2 * j] = bf16_bits_to_f32(u[j] & 0xFFFFu);
      xf[8 * i + 2 * j + 1] = bf16_bits_to_f32(u[j] >> 16);
    }
  }
  xq_from_floats(xf, xg);
}

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

template <int SEG>
__global__ void __launch_bounds__(256) gate_up_kernel(
    const ExpertPtrs* __restrict__ table, const int32_t* __restrict__ idx,
    int n_experts, int top_k, int slots, const uint16_t* __restrict__ x,
    int H, int I, float* __restrict__ hbuf, uint32_t* __restrict__ err) {
  constexpr int NV = SEG;        // values reduced per phase (gate + up)
  constexpr int NR = NV / 2;     // rows per phase
  __shared__ float red[32][33];  // cross-warp partials [warp][lane]
  const int G = H >> 5;
  const ColMap cm = col_map(G);
  const int t = blockIdx.y / slots, slot = blockIdx.y % slots;
  int eid = n_experts;  // slot == top_k: the shared expert
  if (slot < top_k) {
    eid = idx[(size_t)t * top_k + slot];
    if (eid < 0 || eid >= n_experts) {
      if (threadIdx.x == 0) atomicCAS(err, 0u, (uint32_t)kErrBadExpertId);
      eid = -1;
    }
  }
  float* hrow = hbuf + ((size_t)t * slots + slot) * I;
  const int row0 = blockIdx.x * cm.P * NR;
  if (eid < 0) {  // skipped term: h = 0
    for (int r = threadIdx.x; r < cm.P * NR; r += blockDim.x)
      if (row0 + r < I) hrow[row0 + r] = 0.f;
    return;
  }
  const ExpertPtrs ep = table[eid];
  XQ xg;
  load_x_group_bf16(x + (size_t)t * H + cm.col * 32, xg);

  const size_t row_bytes = (size_t)H / 2, row_sc = (size_t)G;
  float v[NV];
#pragma unroll
  for (int r = 0; r < NR; ++r) {
    const int row = row0 + cm.phase * NR + r;
    float pg = 0.f, pu = 0.f;
    if (row < I) {
      const uint4 qg = __ldg(reinterpret_cast<const uint4*>(ep.q_gate + row * row_bytes) + cm.col);
      const uint4 qu = __ldg(reinterpret_cast<const uint4*>(ep.q_up + row * row_bytes) + cm.col);
      const float sg = f16_bits_to_f32(__ldg(ep.s_gate + row * row_sc + cm.col));
      const float su = f16_bits_to_f32(__ldg(ep.s_up + row * row_sc + cm.col));
      pg = dot_scaled(qg, xg, sg);
      pu = dot_scaled(qu, xg, su);
    }
    v[r] = pg;
    v[NR + r] = pu;
  }
  reduce_scatter<NV, SEG>(v);
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int vi = lane % SEG;
  if (cm.wpr == 1) {
    const float u = __shfl_down_sync(0xffffffffu, v[0], NR, SEG);
    const int row = row0 + cm.phase * NR + vi;
    if (vi < NR && row < I) hrow[row] = silu_mul(v[0], u);
  } else {
    red[warp][lane] = v[0];
    __syncthreads();
    if (cm.wir == 0 && lane < NR) {
      float g = 0.f, u = 0.f;
      for (int w = 0; w < cm.wpr; ++w) {
        g += red[warp + w][lane];
        u += red[warp + w][lane + NR];
      }
      const int row = row0 + cm.phase * NR + lane;
      if (row < I) hrow[row] = silu_mul(g, u);
    }
  }
}

// ---------------------------------------------------------------------------
// int4 down projection with the weighted combine (one token, a block of
// output rows).  For each row the thread of chunk column `col` accumulates,
// in slot order, w_j * scale * dot(q_down row chunk, h_j group) over the
// routed slots and the shared expert (weight 1); one reduce-scatter and a
// fixed-order cross-warp sum give y[row] directly.  The K = inter dimension
// is split over the row's threads and reduced without atomics, and no
// per-expert partial goes to memory.
// grid.x = row blocks of `hidden`, grid.y = token.

template <int SEG, int NV>
__global__ void __launch_bounds__(256) down_combine_kernel(
    const ExpertPtrs* __restrict__ table, const int32_t* __restrict__ idx,
    const float* __restrict__ wts, int n_experts, int top_k, int slots,
    const float* __restrict__ hbuf, int H, int I, float* __restrict__ y,
    uint32_t* __restrict__ err) {
  __shared__ float red[32][33];
  const int G = I >> 5;
  const ColMap cm = col_map(G);
  const int t = blockIdx.y;
  const int row0 = blockIdx.x * cm.P * NV;
  const size_t row_bytes = (size_t)I / 2, row_sc = (size_t)G;
  float acc[NV];
#pragma unroll
  for (int r = 0; r < NV; ++r) acc[r] = 0.f;

  for (int slot = 0; slot < slots; ++slot) {
    int eid = n_experts;
    float wj = 1.0f;
    if (slot < top_k) {
      eid = idx[(size_t)t * top_k + slot];
      wj = wts[(size_t)t * top_k + slot];
      if (eid < 0 || eid >= n_experts) {
        if (threadIdx.x == 0) atomicCAS(err, 0u, (uint32_t)kErrBadExpertId);
        continue;
      }
    }
    const ExpertPtrs ep = table[eid];
    XQ hg;
    load_x_group_f32(hbuf + ((size_t)t * slots + slot) * I + cm.col * 32, hg);
#pragma unroll
    for (int r = 0; r < NV; ++r) {
      const int row = row0 + cm.phase * NV + r;
      if (row < H) {
        const uint4 q = __ldg(reinterpret_cast<const uint4*>(ep.q_down + row * row_bytes) + cm.col);
        const float sc = f16_bits_to_f32(__ldg(ep.s_down + row * row_sc + cm.col));
        acc[r] = fmaf(wj, dot_scaled(q, hg, sc), acc[r]);
      }
    }
  }
  reduce_scatter<NV, SEG>(acc);
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int vi = reduce_index<NV, SEG>(lane);
  const bool owner = (lane % (SEG / NV)) == 0;
  if (cm.wpr == 1) {
    const int row = row0 + cm.phase * NV + vi;
    if (owner && row < H) y[(size_t)t * H + row] = acc[0];
  } else {
    red[warp][lane] = acc[0];
    __syncthreads();
    if (cm.wir == 0 && owner) {
      float s = 0.f;
      for (int w = 0; w < cm.wpr; ++w) s += red[warp + w][lane];
      const int row = row0 + cm.phase * NV + vi;
      if (row < H) y[(size_t)t * H + row] = s;
    }
  }
}

// ---------------------------------------------------------------------------
// Plain dequantising int4 GEMV, y[r] = sum_c q[r][c] * scale[r][c/32] * x[c]
// (fp32 x and y), built from the same group dot product as the layer
// kernels.  Exposed for one-hot checks of the packing and scale indexing.

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

cudaError_t launch_router_logits(const float* w, const uint16_t* x, int T, int H, int E,
                                 float* logits, cudaStream_t st) {
  const int wpb = 8;
  router_logits_kernel<8><<<(E + wpb - 1) / wpb, wpb * 32, 0, st>>>(w, x, T, H, E, logits);
  return cudaGetLastError();
}

cudaError_t launch_select(const float* logits, const float* bias, int T, int E, int n_group,
                          int topk_group, int top_k, float rsf, int32_t* idx, float* w,
                          float* scores, cudaStream_t st) {
  select_kernel<<<T, 32 * n_group, 0, st>>>(logits, bias, E, n_group, topk_group, top_k, rsf,
                                            idx, w, scores);
  return cudaGetLastError();
}

template <int SEG>
static cudaError_t gate_up_seg(const ExpertPtrs* table, const int32_t* idx, int E, int top_k,
                               int slots, const uint16_t* x, int T, int H, int I, float* hbuf,
                               uint32_t* err, cudaStream_t st) {
  const int G = H / 32;
  const int nw = warps_for(G);
  const int P = (G >= 32) ? nw / (G / 32) : nw * (32 / G);
  const int rows = P * (SEG / 2);
  dim3 grid((I + rows - 1) / rows, T * slots);
  gate_up_kernel<SEG><<<grid, nw * 32, 0, st>>>(table, idx, E, top_k, slots, x, H, I, hbuf, err);
  return cudaGetLastError();
}

cudaError_t launch_gate_up(const ExpertPtrs* table, const int32_t* idx, int E, int top_k,
                           int slots, const uint16_t* x, int T, int H, int I, float* hbuf,
                           uint32_t* err, cudaStream_t st) {
  const int G = H / 32;
  switch (G >= 32 ? 32 : G) {
    case 32: return gate_up_seg<32>(table, idx, E, top_k, slots, x, T, H, I, hbuf, err, st);
    case 16: return gate_up_seg<16>(table, idx, E, top_k, slots, x, T, H, I, hbuf, err, st);
    case 8: return gate_up_seg<8>(table, idx, E, top_k, slots, x, T, H, I, hbuf, err, st);
    case 4: return gate_up_seg<4>(table, idx, E, top_k, slots, x, T, H, I, hbuf, err, st);
    case 2: return gate_up_seg<2>(table, idx, E, top_k, slots, x, T, H, I, hbuf, err, st);
    default: return cudaErrorInvalidValue;
  }
}

template <int SEG, int NV>
static cudaError_t down_seg(const ExpertPtrs* table, const int32_t* idx, const float* w, int E,
                            int top_k, int slots, const float* hbuf, int T, int H, int I,
                            float* y, uint32_t* err, cudaStream_t st) {
  const int G = I / 32;
  const int nw = warps_for(G);
  const int P = (G >= 32) ? nw / (G / 32) : nw * (32 / G);
  const int rows = P * NV;
  dim3 grid((H + rows - 1) / rows, T);
  down_combine_kernel<SEG, NV><<<grid, nw * 32, 0, st>>>(table, idx, w, E, top_k, slots, hbuf,
                                                         H, I, y, err);
  return cudaGetLastError();
}

cudaError_t launch_down_combine(const ExpertPtrs* table, const int32_t* idx, const float* w,
                                int E, int top_k, int slots, const float* hbuf, int T, int H,
                                int I, float* y, uint32_t* err, cudaStream_t st) {
  const int G = I / 32;
  switch (G >= 32 ? 32 : G) {
    case 32: return down_seg<32, 4>(table, idx, w, E, top_k, slots, hbuf, T, H, I, y, err, st);
    case 16: return down_seg<16, 4>(table, idx, w, E, top_k, slots, hbuf, T, H, I, y, err, st);
    case 8: return down_seg<8, 4>(table, idx, w, E, top_k, slots, hbuf, T, H, I, y, err, st);
    case 4: return down_seg<4, 4>(table, idx, w, E, top_k, slots, hbuf, T, H, I, y, err, st);
    case 2: return down_seg<2, 2>(table, idx, w, E, top_k, slots, hbuf, T, H, I, y, err, st);
    default: return cudaErrorInvalidValue;
  }
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
