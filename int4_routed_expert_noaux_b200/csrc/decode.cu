// decode.cu -- the fused persistent decode kernel: the whole routed-MoE
// layer for one token (router GEMV, noaux_tc selection, 8 routed + shared
// int4 expert FFNs, weighted combine) in ONE cooperative launch.
//
// Design (sm_100a):
//  * one CTA per SM: two consumer groups of 6 warps, a producer warp, a
//    selection warp and a converter warp;
//  * the producer moves each work item's bytes HBM -> shared memory with
//    1-D bulk async copies (the TMA engine) into a 4-stage ring of 54 KB
//    stages, completion tracked by mbarriers (transaction bytes).  Fill n
//    goes to stage n % 4 and is consumed by group n % 2, so one group reduces
//    and publishes while the other computes and two stages stay in flight;
//  * consumers are column-stationary: each thread owns one 16-byte chunk
//    column of the rows it visits and keeps its 32 inputs in registers as
//    int16 fixed point with one exponent per group; the int4 group dot
//    product is exact in integers (dp2a); one butterfly reduce-scatter plus
//    a cross-warp sum finishes each row; one group barrier per item;
//  * start-up: the producer's first fills are the CTA's block of router
//    rows (a static split of the experts over the CTAs), one fill per
//    consumer group.  The groups compute the router rows in double-float
//    arithmetic and publish each row's sigmoid score as a 64-bit record
//    tagged with the call's epoch (one single-copy-atomic store: no flag, no
//    fence);
//  * the selection warp of every CTA polls the E records until all carry
//    this call's epoch and runs the noaux_tc selection itself -- every CTA
//    reads the same scores with the same code, so all reach the same bits.
//    The routed experts are handled in pick order (descending score): each
//    pick's barrier is released as soon as the pick is final, so the
//    producer streams pick 0 while the later picks are still being found;
//  * gate/up items (8 gate + 8 up rows of one expert for the GLM shape) are
//    dealt out statically, CTA b taking items b, b + grid, ... in the order
//    shared expert, routed picks 0..k-1; the shared expert's items keep HBM
//    busy while the routed experts are selected.  Finalizer warps write h
//    rows (fp32) and count, per 32-row group of h, the rows written;
//  * the converter warp of each CTA owns some of those groups: once a
//    group's 32 rows are in, it publishes them as int16 words with one
//    exponent (the layout the down consumers load) and counts the pick's
//    published groups;
//  * down items are static too: CTA b owns a block of output rows and, once
//    a pick's h is published, streams that pick's down rows for it together
//    with the pick's int16 h (4 KB); the partials of its rows stay in shared
//    memory and are combined at the end in slot order (ascending expert id,
//    as the outputs are laid out): no atomics, no cross-CTA combine, bitwise
//    repeatable;
//  * consumer group 1 of a CTA without a second router fill first runs one
//    placeholder gate/up and one placeholder down item through the loop
//    body (nothing published), so that both code paths are fetched while
//    the first weights are in flight;
//  * every wait is bounded (1 s); a wait that runs out sets the workspace
//    error word and the kernel winds down; the last CTA to exit resets the
//    control counters so the next call starts clean.
#include <cuda_runtime.h>
#include <stdint.h>

#include "async.cuh"
#include "common.cuh"
#include "decode.h"
#include "device_once.h"

// Timeline probes: compiled in only with -DMOE_TRACE (a profiling build).
// Per CTA 128 slots: SM cycle counter at event i in slot 96 + i (i < 31),
// the producer's per-fill wait start and issue cycles in slots 2n, 2n + 1
// (n < 48), and the globaltimer (ns) at the CTA's start in slot 127.
#ifdef MOE_TRACE
#define TRACE_AT(i)                                                                          \
  do {                                                                                       \
    if (p.trace) {                                                                           \
      p.trace[blockIdx.x * 128 + 96 + (i)] = (uint64_t)clock64();                            \
      if ((i) == 0) p.trace[blockIdx.x * 128 + 127] = moe::global_timer_ns();                \
    }                                                                                        \
  } while (0)
#define TRACE_FILL(n, j, tag)                                                                \
  do {                                                                                       \
    if (p.trace && (n) < 48)                                                                 \
      p.trace[blockIdx.x * 128 + 2 * (n) + (j)] = (uint64_t)clock64() | ((uint64_t)(tag) << 60); \
  } while (0)
#else
#define TRACE_AT(i) ((void)0)
#define TRACE_FILL(n, j, tag) ((void)0)
#endif

namespace moe {

namespace {

constexpr int kGW = 6;                   // warps per consumer group
constexpr int kGT = kGW * 32;            // threads per consumer group
constexpr int kGroups = 2;
constexpr int kThreads = kGroups * kGT + 96;
constexpr int kProducerWarp = kGroups * kGW;
constexpr int kSelectWarp = kProducerWarp + 1;
constexpr int kConvWarp = kProducerWarp + 2;
constexpr int kStages = 4;
constexpr uint32_t kStageBytes = 55296;
constexpr int kRouterChunks = 8;         // 16-byte W chunks per thread per row
constexpr int kMaxRR = 8;                // router rows per item
constexpr int kMaxE = 256;
constexpr int kMaxSlots = 33;
constexpr int kMaxYcta = 512;            // slot partials of a CTA's own down rows
constexpr uint64_t kWaitNs = 1000000000ull;

enum ItemType : int { kRouter = 0, kGateUp = 1, kDown = 2, kDone = 3 };

struct ItemDesc {
  int type, slot, row0, nrows, eid, pad0, pad1, pad2;
};

struct Smem {
  uint64_t full[kStages];
  uint64_t empty[kStages];
  uint64_t gbar[kGroups];  // per-group item barrier (one arrival per warp)
  uint64_t pickbar[kMaxSlots];  // pick r of the selection is final (one arrival)
  ItemDesc desc[kStages];
  int sel_idx[kMaxSlots];  // selected expert ids, ascending (the slot order)
  ExpertPtrs ep[kMaxSlots];  // the picks' expert tensors (index k: the shared expert)
  int pick_id[kMaxSlots];  // the selection's picks in pick order (descending score)
  float pick_s[kMaxSlots];
  int pick_kept[kMaxSlots];  // pick r kept by top-p (valid once the whole selection is out)
  int slot_pick[kMaxSlots];  // the pick that is slot j
  float sel_w[kMaxSlots];  // the slots' combine weights
  int sel_ok;
  float red[kGroups][2][kGW][32];
  double redd[kGroups * kGW][kMaxRR];  // router partial sums (fp64), per group and warp
  int abort_flag[kGroups];
  float norm_part[kThreads / 32];
  float inv_rms;
  float sc[kMaxE];
  float sp[kMaxE];
  float ycta[kMaxYcta];    // [picks + shared][ycta_rows] partial y of the CTA's own rows
  int last_cta;
};

// The out-of-line helpers take their arguments by value: a reference to the
// kernel's parameters would make the compiler copy them into local memory,
// whose loads miss L1 and wait on L2 while the weights stream.
struct SelArgs {
  int E, k, n_group, topk_group, sel_q, sel_lgL, sel_fast;
  float rsf, top_p;
  int32_t* idx_out;  // written by CTA 0 only (nullable)
  float* w_out;
  uint64_t* trace;   // timeline probes of a -DMOE_TRACE build
  const ExpertPtrs* table;  // nullable (no pointer-table prefetch)
  int early_picks;  // each pick's barrier arrives as soon as the pick is final
};

__device__ __forceinline__ SelArgs sel_args(const DecodeParams& p) {
  SelArgs a;
  a.E = p.E;
  a.k = p.k;
  a.n_group = p.n_group;
  a.topk_group = p.topk_group;
  a.sel_q = p.sel_q;
  a.sel_lgL = p.sel_lgL;
  a.sel_fast = p.sel_fast;
  a.rsf = p.rsf;
  a.top_p = p.top_p;
  a.idx_out = p.idx_out;
  a.w_out = p.w_out;
  a.trace = p.trace;
  a.table = p.table;
  // with every pick kept (no top-p), pick r is final once it is popped
  a.early_picks = p.sel_fast && !(p.top_p < 1.f);
  return a;
}

__device__ __forceinline__ ItemDesc make_item(int type, int slot, int row0, int nrows) {
  ItemDesc d;
  d.type = type;
  d.slot = slot;
  d.row0 = row0;
  d.nrows = nrows;
  d.eid = -1;
  d.pad0 = d.pad1 = d.pad2 = 0;
  return d;
}

// Gate/up item t, in the order: shared gate/up, routed gate/up of slots
// 0..k-1; DONE past the last one.
__device__ __forceinline__ ItemDesc gate_up_item(const DecodeParams& p, int t) {
  auto gu = [&](int slot, int b) {
    return make_item(kGateUp, slot, b * p.RG, min(p.RG, p.I - b * p.RG));
  };
  if (p.has_shared) {
    if (t < p.nG) return gu(p.k, t);
    t -= p.nG;
  }
  if (t < p.k * p.nG) return gu(t / p.nG, t % p.nG);
  return make_item(kDone, 0, 0, 0);
}

// Down rows of CTA b: [r0, r1), whole units of A rows (A keeps every row
// offset of the scales 16-byte aligned).
__device__ __forceinline__ void down_rows(const DecodeParams& p, int b, int& r0, int& r1) {
  r0 = p.A * (int)(((long long)b * p.nU) / gridDim.x);
  r1 = p.A * (int)(((long long)(b + 1) * p.nU) / gridDim.x);
}

// This CTA's next down item: the shared expert's rows first, then slots
// 0..k-1, each in n_db blocks of at most RD rows; DONE when all are taken.
__device__ __forceinline__ ItemDesc next_down(const DecodeParams& p, int& dn, int r0, int r1) {
  const int slots = p.k + p.has_shared;
  while (dn < slots * p.n_db) {
    const int ord = dn / p.n_db, blk = dn % p.n_db;
    ++dn;
    const int row0 = r0 + blk * p.RD;
    const int nrows = min(p.RD, r1 - row0);
    if (nrows <= 0) continue;
    const int slot = p.has_shared ? (ord == 0 ? p.k : ord - 1) : ord;
    return make_item(kDown, slot, row0, nrows);
  }
  return make_item(kDone, 0, 0, 0);
}

// Router rows of CTA b: a static split of the E experts over the first nR
// CTAs (every one of them gets at least one row).
__device__ __forceinline__ void router_rows(const DecodeParams& p, int b, int& r0, int& nr) {
  if (b >= p.nR) {
    r0 = p.E;
    nr = 0;
    return;
  }
  r0 = (int)(((long long)b * p.E) / p.nR);
  nr = (int)(((long long)(b + 1) * p.E) / p.nR) - r0;
}

// The CTA's router rows go out as one fill per consumer group (fill g is
// consumed by group g): group 0 takes the first ceil(nr / 2) rows, group 1
// the rest, so that a CTA with two rows computes them at the same time.
__device__ __forceinline__ int router_fills(int nr) { return nr >= 2 ? 2 : (nr > 0 ? 1 : 0); }
__device__ __forceinline__ void router_fill_rows(int r0, int nr, int g, int& f0, int& fn) {
  const int a = router_fills(nr) == 2 ? (nr + 1) / 2 : nr;
  f0 = g == 0 ? r0 : r0 + a;
  fn = g == 0 ? a : nr - a;
}

// At the start of this CTA's down phase (a stack's next layer known): its
// router rows of the next layer and shared-expert gate/up items b, b + grid,
// ... of the next layer go to L2 with an evict-last hint, so that the next
// layer's dependent start-up reads them from L2 instead of HBM.
__device__ __forceinline__ void prefetch_next_layer(const DecodeParams& p) {
  const uint64_t keep = l2_policy_evict_last();
  int r0, nr;
  router_rows(p, blockIdx.x, r0, nr);
  if (nr > 0) bulk_prefetch_l2(p.pf_w_router + (size_t)r0 * p.H, (uint32_t)nr * p.H * 4, keep);
  if (!p.has_shared) return;
  for (int t = blockIdx.x; t < p.nG; t += gridDim.x) {
    const int row0 = t * p.RG, nrows = min(p.RG, p.I - row0);
    const uint32_t qb = (uint32_t)nrows * (p.H / 2), sb = (uint32_t)nrows * (p.H / 16);
    const size_t qoff = (size_t)row0 * (p.H / 2), soff = (size_t)row0 * (p.H / 32);
    bulk_prefetch_l2(p.pf_shared.q_gate + qoff, qb, keep);
    bulk_prefetch_l2(p.pf_shared.q_up + qoff, qb, keep);
    bulk_prefetch_l2(p.pf_shared.s_gate + soff, sb, keep);
    bulk_prefetch_l2(p.pf_shared.s_up + soff, sb, keep);
  }
}


// Record an error: the first one also records where it happened (CTA,
// warp, site, fill) in the control words kCtrlWhere..kCtrlWhere+3.
__device__ __forceinline__ void set_error(uint32_t* ctrl, uint32_t code, uint32_t site = 0,
                                          uint32_t fill = 0) {
  if (atomicCAS(ctrl + kCtrlErr, 0u, code) == 0u) {
    ctrl[kCtrlWhere + 0] = blockIdx.x;
    ctrl[kCtrlWhere + 1] = threadIdx.x >> 5;
    ctrl[kCtrlWhere + 2] = site;
    ctrl[kCtrlWhere + 3] = fill;
  }
  atomicExch(ctrl + kCtrlAbort, 1u);
}

__device__ __forceinline__ bool aborted(const uint32_t* ctrl) {
  return *((volatile const uint32_t*)(ctrl + kCtrlAbort)) != 0;
}

// Bounded poll of a global counter until it reaches `target`.
__device__ bool wait_counter(uint32_t* ctrl, const uint32_t* p, uint32_t target) {
  if (ld_acquire(p) >= target) return true;
  const uint64_t deadline = global_timer_ns() + kWaitNs;
  // one polling thread: a short constant pause, so that the wait ends within
  // tens of nanoseconds of the count (no growing back-off on this path)
  for (uint32_t it = 0;; ++it) {
    __nanosleep(32);
    if (ld_acquire(p) >= target) return true;
    if ((it & 7) == 7) {
      if (aborted(ctrl) || global_timer_ns() > deadline) return false;
    }
  }
}

struct ArgMaxF {
  float v;
  int i;
};

__device__ __forceinline__ ArgMaxF am_merge(ArgMaxF a, ArgMaxF b) {
  if (a.i < 0) return b;
  if (b.i < 0) return a;
  if (b.v > a.v || (b.v == a.v && b.i < a.i)) return b;
  return a;
}

__device__ __forceinline__ ArgMaxF am_warp(ArgMaxF a) {
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) {
    ArgMaxF b;
    b.v = __shfl_xor_sync(0xffffffffu, a.v, o);
    b.i = __shfl_xor_sync(0xffffffffu, a.i, o);
    a = am_merge(a, b);
  }
  return a;
}

// The end of a selection: lane r < k holds the r-th pick (id, unbiased
// score s).  Weights rsf * s / sum s ("LightLX", "How it works": normalised
// sigmoid weights; colibri summary: routed_scaling_factor); with adaptive
// top-p, the kept picks and their weights normalised over them, dropped
// slots -1 / 0 after the kept ids.  Ids ascending to S.sel_idx / S.sel_w
// (and, from CTA 0, to idx_out / w_out).
__device__ __forceinline__ void publish_selection(const SelArgs& p, Smem& S, int my_sel,
                                                  float my_s) {
  const int lane = threadIdx.x & 31;
  float denom = warp_sum(my_s) + 1e-20f;
  bool kept = lane < p.k;
  if (p.top_p < 1.f) {
    kept = topp_keep(my_sel, my_s, denom, p.k, p.top_p);
    denom = warp_sum(kept ? my_s : 0.f) + 1e-20f;
  }
  const int pos = topp_position(my_sel, kept, p.k);
  if (lane < p.k) {
    const int id = kept ? my_sel : -1;
    const float wv = kept ? p.rsf * my_s / denom : 0.f;
    S.sel_idx[pos] = id;
    S.sel_w[pos] = wv;
    if (!p.early_picks) S.pick_id[lane] = my_sel;
    S.pick_kept[lane] = kept ? 1 : 0;
    S.slot_pick[pos] = lane;
    if (blockIdx.x == 0) {
      if (p.idx_out) p.idx_out[pos] = id;
      if (p.w_out) p.w_out[pos] = wv;
    }
  }
  // the picks are final now (unless each went out as it was popped): lane r
  // releases its own pick_id / pick_kept
  if (!p.early_picks && lane < p.k) mbar_arrive(&S.pickbar[lane]);
}

// Selection for shapes whose groups do not align with lanes: one lane per
// group, repeated warp arg-max over S.sp / S.sc.  Results go to
// S.sel_idx / S.sel_w (and, from CTA 0, to the caller's idx_out / w_out).
__device__ __noinline__ void run_select_generic(const SelArgs p, Smem& S) {
  const int lane = threadIdx.x & 31;
  const int per = p.E / p.n_group;
  // group score: sum of the two largest bias-corrected scores (lane = group)
  float gs = 0.f;
  if (lane < p.n_group) {
    float b1 = 0.f, b2 = 0.f;
    int i1 = -1, i2 = -1;
    for (int e = lane * per; e < (lane + 1) * per; ++e) {
      const float v = S.sp[e];
      if (i1 < 0 || v > b1) {
        b2 = b1;
        i2 = i1;
        b1 = v;
        i1 = e;
      } else if (i2 < 0 || v > b2) {
        b2 = v;
        i2 = e;
      }
    }
    gs = (i2 >= 0) ? b1 + b2 : b1;
  }
  // keep topk_group groups: rank by (score desc, index asc)
  int rank = 0;
  for (int h = 0; h < p.n_group; ++h) {
    const float o = __shfl_sync(0xffffffffu, gs, h);
    if (lane < p.n_group && (o > gs || (o == gs && h < lane))) ++rank;
  }
  const unsigned kept_mask = __ballot_sync(0xffffffffu, lane < p.n_group && rank < p.topk_group);
  // top_k of sp over kept experts; lane owns experts lane + 32 m
  const int nper = (p.E + 31) >> 5;
  unsigned taken = 0;
  ArgMaxF local{0.f, -1};
  for (int m = 0; m < nper; ++m) {
    const int e = lane + 32 * m;
    if (e < p.E && ((kept_mask >> (e / per)) & 1u)) local = am_merge(local, ArgMaxF{S.sp[e], e});
  }
  int my_sel = -1;
  for (int r = 0; r < p.k; ++r) {
    const ArgMaxF best = am_warp(local);
    if (lane == r) my_sel = best.i;
    if (best.i >= 0 && (best.i & 31) == lane) {
      taken |= 1u << (best.i >> 5);
      local = ArgMaxF{0.f, -1};
      for (int m = 0; m < nper; ++m) {
        const int e = lane + 32 * m;
        if (e < p.E && ((kept_mask >> (e / per)) & 1u) && !((taken >> m) & 1u))
          local = am_merge(local, ArgMaxF{S.sp[e], e});
      }
    }
  }
  const float s_mine = (lane < p.k && my_sel >= 0) ? S.sc[my_sel] : 0.f;
  publish_selection(p, S, my_sel, s_mine);
}

// Four consecutive inputs of a residual (pre-norm) step, i0 % 4 == 0, as
// bf16(x_resid * inv_rms) pairs in two words (one 16-byte load).
__device__ __forceinline__ uint2 norm_bf16x4(const float* x_resid, int i0, float inv_rms) {
  const float4 v = __ldg(reinterpret_cast<const float4*>(x_resid + i0));
  uint2 r;
  r.x = (uint32_t)f32_to_bf16_rne(v.x * inv_rms) | ((uint32_t)f32_to_bf16_rne(v.y * inv_rms) << 16);
  r.y = (uint32_t)f32_to_bf16_rne(v.z * inv_rms) | ((uint32_t)f32_to_bf16_rne(v.w * inv_rms) << 16);
  return r;
}

// Order-preserving map of a float onto uint32 (larger float, larger key;
// every key is > 0).
__device__ __forceinline__ uint32_t order_key(float v) {
  const uint32_t u = __float_as_uint(v);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// Compare-exchange of the per-lane candidate lists: position a before b in
// the order (key descending, expert index ascending).
__device__ __forceinline__ void cx(uint32_t (&key)[kMaxE / 32], int (&jid)[kMaxE / 32],
                                   float (&sl)[kMaxE / 32], int a, int b) {
  const bool sw = key[b] > key[a] || (key[b] == key[a] && jid[b] < jid[a]);
  const uint32_t ka = key[a], kb = key[b];
  const int ja = jid[a], jb = jid[b];
  const float sa = sl[a], sb = sl[b];
  key[a] = sw ? kb : ka;
  key[b] = sw ? ka : kb;
  jid[a] = sw ? jb : ja;
  jid[b] = sw ? ja : jb;
  sl[a] = sw ? sb : sa;
  sl[b] = sw ? sa : sb;
}

// noaux_tc selection over S.sp (sigmoid + bias) and S.sc (sigmoid), by one
// warp ("LightLX", "How it works": the noaux_tc sigmoid router; colibri
// summary, "Principales fonctionnalites implementees": routed_scaling_factor).
// Lane l owns the q = ceil(E / 32) consecutive experts l*q .. l*q+q-1 in
// registers; when a group's experts are exactly L = per / q consecutive
// lanes (L a power of two), group top-2 is a segmented butterfly, each lane
// sorts its kept candidates with a sorting network, and the top-k is k
// rounds of two warp reductions (max of the score key, then min of the
// expert id among the lanes holding it: ties go to the lower id).  Results
// go to S.sel_idx / S.sel_w (and, from CTA 0, to idx_out / w_out).
__device__ __noinline__ void run_select(const SelArgs p, Smem& S) {
  if (!p.sel_fast) {
    run_select_generic(p, S);
    return;
  }
  // Branch-free: every shuffle and reduction runs in all lanes with no
  // data-dependent guard around it (guarded warp collectives cost tens of
  // cycles each in convergence handling).
  const int lane = threadIdx.x & 31;
  const int q = p.sel_q, lgL = p.sel_lgL, L = 1 << lgL;
  constexpr int kQ = kMaxE / 32;
  const int nmine = max(0, min(q, p.E - lane * q));  // experts this lane owns
  float sc[kQ], sp[kQ];
#pragma unroll
  for (int j = 0; j < kQ; ++j) {
    sp[j] = (j < nmine) ? S.sp[lane * q + j] : -INFINITY;
    sc[j] = (j < nmine) ? S.sc[lane * q + j] : 0.f;
  }
  // group score: the two largest sp of the group (lanes g*L .. g*L+L-1)
  float t1 = -INFINITY, t2 = -INFINITY;
#pragma unroll
  for (int j = 0; j < kQ; ++j) {
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
  const int per = q << lgL;
  const float gs_seg = (per >= 2) ? t1 + t2 : t1;
  if (lane == 0) TRACE_AT(17);
  // keep topk_group groups: rank by (score desc, index asc); lane g holds
  // group g (n_group <= 32), lanes past the groups hold -inf
  const int G = p.n_group;
  float gs = __shfl_sync(0xffffffffu, gs_seg, (lane < G ? lane : 0) << lgL);
  gs = (lane < G) ? gs : -INFINITY;
  int rank = 0;
#pragma unroll
  for (int h = 0; h < 32; ++h) {
    const float o = __shfl_sync(0xffffffffu, gs, h);
    rank += (o > gs || (o == gs && h < lane)) ? 1 : 0;
  }
  const unsigned kept_mask = __ballot_sync(0xffffffffu, lane < G && rank < p.topk_group);
  const bool kept = (kept_mask >> (lane >> lgL)) & 1u;
  if (lane == 0) TRACE_AT(18);
  // each lane sorts its kept candidates once (a sorting network)
  uint32_t key[kQ];
  int jid[kQ];
  float sl[kQ];
#pragma unroll
  for (int j = 0; j < kQ; ++j) {
    key[j] = (j < nmine && kept) ? order_key(sp[j]) : 0u;
    jid[j] = j;
    sl[j] = sc[j];
  }
  // Pick 0, the best kept candidate (ties: the lower expert id), goes out
  // before the lists are sorted, so that its expert starts streaming while
  // the other picks are found; round 0 below pops the same candidate.
  if (p.early_picks) {
    uint32_t bk = 0u;
    int bj = 0;
    float bsl = 0.f;
#pragma unroll
    for (int j = 0; j < kQ; ++j)
      if (key[j] > bk) {
        bk = key[j];
        bj = j;
        bsl = sl[j];
      }
    const uint32_t m = __reduce_max_sync(0xffffffffu, bk);
    bool own = bk == m && m != 0u;
    if (__popc(__ballot_sync(0xffffffffu, own)) > 1) {
      const uint32_t cand = own ? (uint32_t)(lane * q + bj) : 0xFFFFFFFFu;
      own = cand == __reduce_min_sync(0xffffffffu, cand);
    }
    if (own) {
      S.pick_id[0] = lane * q + bj;
      S.pick_s[0] = bsl;
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&S.pickbar[0]);
  }
  static_assert(kQ == 8, "the network below sorts 8 candidates");
  cx(key, jid, sl, 0, 1); cx(key, jid, sl, 2, 3); cx(key, jid, sl, 4, 5); cx(key, jid, sl, 6, 7);
  cx(key, jid, sl, 0, 2); cx(key, jid, sl, 1, 3); cx(key, jid, sl, 4, 6); cx(key, jid, sl, 5, 7);
  cx(key, jid, sl, 1, 2); cx(key, jid, sl, 5, 6);
  cx(key, jid, sl, 0, 4); cx(key, jid, sl, 1, 5); cx(key, jid, sl, 2, 6); cx(key, jid, sl, 3, 7);
  cx(key, jid, sl, 2, 4); cx(key, jid, sl, 3, 5);
  cx(key, jid, sl, 1, 2); cx(key, jid, sl, 3, 4); cx(key, jid, sl, 5, 6);
  if (lane == 0) TRACE_AT(19);
  // the winners are among each lane's best candidates: their pointer-table
  // entries start towards L1 now, and the loads after the selection hit it
  if (p.table) {
#pragma unroll
    for (int j = 0; j < 2; ++j)
      if (key[j] != 0u) {
        const char* e = reinterpret_cast<const char*>(p.table + lane * q + jid[j]);
        asm volatile("prefetch.global.L1 [%0];" ::"l"(e));
        asm volatile("prefetch.global.L1 [%0];" ::"l"(e + sizeof(ExpertPtrs) - 1));
      }
  }
  // top_k: the best head is popped, k times; among equal heads (a rare,
  // warp-uniform case) the lowest expert id.  The owner of the r-th pick
  // leaves it in shared memory, off the dependent chain of the rounds.
  if (lane < p.k && !(p.early_picks && lane == 0)) {
    S.pick_id[lane] = -1;  // no candidate left (not reachable for a valid shape)
    S.pick_s[lane] = 0.f;
  }
  __syncwarp();
  for (int r = 0; r < p.k; ++r) {
    const uint32_t m = __reduce_max_sync(0xffffffffu, key[0]);
    bool own = key[0] == m && m != 0u;
    if (__popc(__ballot_sync(0xffffffffu, own)) > 1) {
      const uint32_t cand = own ? (uint32_t)(lane * q + jid[0]) : 0xFFFFFFFFu;
      own = cand == __reduce_min_sync(0xffffffffu, cand);
    }
    if (own && !(p.early_picks && r == 0)) {  // pick 0 went out already
      S.pick_id[r] = lane * q + jid[0];
      S.pick_s[r] = sl[0];
    }
    if (p.early_picks && r > 0) {
      // pick r is final: the producer may start streaming its expert while
      // the remaining picks are found
      __syncwarp();
      if (lane == 0) mbar_arrive(&S.pickbar[r]);
    }
#pragma unroll
    for (int j = 0; j + 1 < kQ; ++j) {  // pop the owner's head
      key[j] = own ? key[j + 1] : key[j];
      jid[j] = own ? jid[j + 1] : jid[j];
      sl[j] = own ? sl[j + 1] : sl[j];
    }
    key[kQ - 1] = own ? 0u : key[kQ - 1];
  }
  __syncwarp();
  // lane r holds the r-th pick (lanes past k: INT_MAX for the ordering)
  if (lane == 0) TRACE_AT(20);
  const int my_sel = (lane < p.k) ? S.pick_id[lane] : 0x7FFFFFFF;
  const float my_s = (lane < p.k) ? S.pick_s[lane] : 0.f;
  publish_selection(p, S, my_sel, (lane < p.k) ? my_s : 0.f);
}

// Lane holding reduce-scatter value `vi` of row phase `ph` (group-local warp).
template <int NV, int SEG>
__device__ __forceinline__ void owner_of(int ph, int vi, int wpr, int& warp0, int& lane) {
  if (SEG == 32) {
    warp0 = ph * wpr;
    lane = vi * (32 / NV);
  } else {
    const int rpw = 32 / SEG;
    warp0 = ph / rpw;
    lane = (ph % rpw) * SEG + vi * (SEG / NV);
  }
}

// Bounded barrier of one consumer group: every warp arrives once, then waits
// for phase `par`.  Returns false (in every lane of the warp) if the wait ran
// out; the memory effects of the other warps before their arrival are
// visible afterwards.
__device__ __forceinline__ bool group_barrier(uint64_t* bar, uint32_t par) {
  const int lane = threadIdx.x & 31;
  __syncwarp();
  int ok = 1;
  if (lane == 0) {
    mbar_arrive(bar);
    ok = mbar_wait(bar, par, kWaitNs) ? 1 : 0;
  }
  ok = __shfl_sync(0xffffffffu, ok, 0);
  if (ok) mbar_test(bar, par);
  __syncwarp();
  return ok != 0;
}

__device__ __forceinline__ ColMap group_col_map(int Gc, int gw, int lane) {
  ColMap m;
  if (Gc >= 32) {
    m.wpr = Gc >> 5;
    m.P = kGW / m.wpr;
    m.col = (gw % m.wpr) * 32 + lane;
    m.phase = gw / m.wpr;
    m.seg = 32;
    m.wir = gw % m.wpr;
  } else {
    const int rpw = 32 / Gc;
    m.wpr = 1;
    m.P = kGW * rpw;
    m.col = lane % Gc;
    m.phase = gw * rpw + lane / Gc;
    m.seg = Gc;
    m.wir = 0;
  }
  return m;
}

template <int SEG_G, int SEG_D>
__global__ void __launch_bounds__(kThreads, 1) decode_kernel(const DecodeParams p) {
  constexpr int NR_G = (SEG_G / 2 < 8) ? SEG_G / 2 : 8;   // gate (and up) rows per phase
  constexpr int NV_G = 2 * NR_G;
  constexpr int NR_D = (SEG_D < 16) ? SEG_D : 16;          // down rows per phase
  extern __shared__ __align__(128) uint8_t dsmem[];
  uint8_t* stages = dsmem;
  Smem& S = *reinterpret_cast<Smem*>(dsmem + kStages * kStageBytes);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int slots = p.k + p.has_shared;

  // the producer's first-item offset (0 but in a failure test), loaded
  // before anything else so that its round trip is over by the first fill
  if (threadIdx.x == kProducerWarp * 32) {
    // the producer thread sets up the barriers and sends the CTA's first
    // fill (its router rows, the head of the dependent start-up chain)
    // before anything else happens
    TRACE_AT(0);
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&S.full[s], 1);
      mbar_init(&S.empty[s], kGW);
    }
    for (int g = 0; g < kGroups; ++g) mbar_init(&S.gbar[g], kGW);
    for (int r = 0; r < kMaxSlots; ++r) mbar_init(&S.pickbar[r], 1);
    S.sel_ok = 0;
    S.abort_flag[0] = S.abort_flag[1] = 0;
    fence_mbar_init();
    if (p.has_shared) S.ep[p.k] = p.shared;  // visible to the producer: same thread
    int rr0, rnr;
    router_rows(p, blockIdx.x, rr0, rnr);
    for (int g = 0; g < router_fills(rnr); ++g) {
      int f0, fn;
      router_fill_rows(rr0, rnr, g, f0, fn);
      S.desc[g] = make_item(kRouter, 0, f0, fn);
      const uint32_t bytes = (uint32_t)fn * p.H * 4;
      mbar_arrive_expect_tx(&S.full[g], bytes);
      bulk_g2s(dsmem + (size_t)g * kStageBytes, p.w_router + (size_t)f0 * p.H, bytes, &S.full[g],
               l2_policy_evict_first());
    }
    if (rnr > 0) TRACE_AT(1);
  }
  // Programmatic dependent launch: the next call on the stream may start its
  // prologue (barriers, its router rows' fill: inputs no call writes) as
  // this grid's CTAs leave their SMs; everything an earlier call writes --
  // the control words, x of a stack's next layer -- is read after the wait.
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  asm volatile("griddepcontrol.wait;" ::: "memory");
  // the producer's first-item offset (0 but in a failure test)
  const uint32_t gu_offset =
      threadIdx.x == kProducerWarp * 32 ? ld_relaxed_u32(p.ctrl + kCtrlTicket) : 0u;
  if (p.x_resid) {
    // RMSNorm with unit gain ("LightLX", "How it works": RMSNorm of the
    // upstream model): every CTA forms the same fixed-order sum of squares.
    float part = 0.f;
    for (int i = threadIdx.x; i < p.H; i += kThreads) part = fmaf(p.x_resid[i], p.x_resid[i], part);
    part = warp_sum(part);
    if (lane == 0) S.norm_part[warp] = part;
  }
  __syncthreads();
  if (p.x_resid && threadIdx.x == 0) {
    float ss = 0.f;
    for (int w = 0; w < kThreads / 32; ++w) ss += S.norm_part[w];
    S.inv_rms = 1.0f / sqrtf(ss / (float)p.H + p.norm_eps);
  }
  __syncthreads();
  const float inv_rms = p.x_resid ? S.inv_rms : 1.0f;
  // this call's epoch: one more than the last finished call's
  const uint32_t epoch = *reinterpret_cast<volatile const uint32_t*>(p.ctrl + kCtrlEpoch) + 1u;

  if (warp == kProducerWarp) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      const uint64_t policy = l2_policy_evict_first();
      bool sel_seen = false;
      uint64_t pick_seen = 0, pick_dropped = 0;  // bit r: pick r acquired / dropped by top-p
      bool first_routed = false, first_down = false;
      uint64_t hq_seen = 0;  // bit j: slot j's int16 h acquired
      int dones = 0;
      int rr0, rnr;
      router_rows(p, blockIdx.x, rr0, rnr);
      bool gate_up_over = false;
      int dn = 0;  // this CTA's down items taken so far
      int dr0, dr1;
      down_rows(p, blockIdx.x, dr0, dr1);
      // Gate/up items are dealt out statically: CTA b takes items b,
      // b + grid, ... of the order shared, routed picks 0..k-1.  (A shared ticket
      // counter balances slightly better but puts an atomic's round trip to
      // L2 -- microseconds while the weights stream -- between fills.)  The
      // control word kCtrlTicket offsets the first item; it is 0 except in a
      // test that starts past the last item to make a wait run out.
      int gu_next = (int)blockIdx.x + (int)gu_offset;
      // fills 0 (and 1) -- the router rows -- went out in the prologue
      for (uint32_t n = (uint32_t)router_fills(rnr);; ++n) {
        const int stage = (int)(n % kStages);
        ItemDesc d = make_item(kDone, 0, 0, 0);
        // the next item of this CTA (slots dropped by top-p are passed over)
        while (dones == 0) {
          if (!gate_up_over) {
            d = gate_up_item(p, gu_next);
            gate_up_over = d.type == kDone;
            gu_next += (int)gridDim.x;
          }
          if (gate_up_over) {
            if (dn == 0) {
              if (p.pf_w_router) prefetch_next_layer(p);
              // which slots' int16 h are complete already: one round trip
              // for all of them instead of one per down item
              // (relaxed loads all in flight at once, then one fence: an
              // acquire of every count seen complete)
              for (int j = 0; j < slots; ++j)
                if (ld_relaxed_u32(p.ctrl + kCtrlHqDone + j) >= (uint32_t)(p.I >> 5))
                  hq_seen |= 1ull << j;
              fence_acq_rel();
              fence_proxy_async();
            }
            d = next_down(p, dn, dr0, dr1);
          }
          if (d.type == kDone) break;
          if (d.slot < p.k) {
            // routed items go in pick order (descending score): pick r's
            // items can stream as soon as pick r is final, before the later
            // picks are found
            if (!((pick_seen >> d.slot) & 1ull)) {
              // the selection warp's pick (mbarrier: release / acquire)
              if (mbar_wait(&S.pickbar[d.slot], 0u, kWaitNs) && S.sel_ok) {
                pick_seen |= 1ull << d.slot;
                if (!sel_seen) {
                  sel_seen = true;
                  TRACE_AT(12);
                }
                const int id = S.pick_id[d.slot];
                if (p.top_p < 1.f && !S.pick_kept[d.slot]) {
                  pick_dropped |= 1ull << d.slot;
                } else if (id >= 0 && id < p.E) {
                  S.ep[d.slot] = p.table[id];  // the pick's tensors, once
                }
              } else {
                set_error(p.ctrl, kErrTimeout, 4, n);
                d = make_item(kDone, 0, 0, 0);
                break;
              }
            }
            if ((pick_dropped >> d.slot) & 1ull) continue;  // dropped by top-p: no bytes read
            d.eid = S.pick_id[d.slot];
            if (d.eid < 0 || d.eid >= p.E) {
              set_error(p.ctrl, kErrBadExpertId, 5, n);
              d = make_item(kDone, 0, 0, 0);
              break;
            }
          } else {
            d.eid = p.E;  // shared expert
          }
          if (d.type == kDown && !((hq_seen >> d.slot) & 1ull)) {
            // every 32-row group of the slot's h must be published as int16
            if (wait_counter(p.ctrl, p.ctrl + kCtrlHqDone + d.slot, (uint32_t)(p.I >> 5))) {
              hq_seen |= 1ull << d.slot;
              fence_proxy_async();  // order the observed stores before the bulk reads
            } else {
              set_error(p.ctrl, kErrTimeout, 7, n);
              d = make_item(kDone, 0, 0, 0);
            }
          }
          break;
        }
        // wait until the consumers released this stage's previous contents
        TRACE_FILL(n, 0, d.type);
        if (n >= (uint32_t)kStages) {
          if (!mbar_wait(&S.empty[stage], ((n / kStages) - 1) & 1u, kWaitNs)) {
            set_error(p.ctrl, kErrTimeout, 6, n);
            // stop issuing; wait (bounded) for the fills already issued
            for (uint32_t m = n - kStages; m < n; ++m) {
              mbar_wait(&S.full[m % kStages], (m / kStages) & 1u, kWaitNs);
            }
            break;
          }
        }
        S.desc[stage] = d;
        TRACE_FILL(n, 1, d.slot & 15);
        uint8_t* dst = stages + (size_t)stage * kStageBytes;
        if (d.type == kGateUp) {
          if (d.slot == 0 && !first_routed) {
            first_routed = true;
            TRACE_AT(6);
          }
          const ExpertPtrs ep = S.ep[d.slot];
          const uint32_t qb = (uint32_t)d.nrows * (p.H / 2), sb = (uint32_t)d.nrows * (p.H / 16);
          const size_t qoff = (size_t)d.row0 * (p.H / 2), soff = (size_t)d.row0 * (p.H / 32);
          mbar_arrive_expect_tx(&S.full[stage], 2 * (qb + sb));
          bulk_g2s(dst, ep.q_gate + qoff, qb, &S.full[stage], policy);
          bulk_g2s(dst + p.RG * (p.H / 2), ep.q_up + qoff, qb, &S.full[stage], policy);
          bulk_g2s(dst + 2 * p.RG * (p.H / 2), ep.s_gate + soff, sb, &S.full[stage], policy);
          bulk_g2s(dst + 2 * p.RG * (p.H / 2) + p.RG * (p.H / 16), ep.s_up + soff, sb,
                   &S.full[stage], policy);
        } else if (d.type == kDown) {
          if (!first_down) {
            first_down = true;
            TRACE_AT(7);
          }
          const ExpertPtrs ep = S.ep[d.slot];
          const int GD = p.I >> 5;
          const uint32_t qb = (uint32_t)d.nrows * (p.I / 2), sb = (uint32_t)d.nrows * (p.I / 16);
          const uint32_t hb = (uint32_t)GD * 64, fb = (uint32_t)GD * 4;
          const uint32_t tail = (uint32_t)p.RD * (p.I / 2 + p.I / 16);
          mbar_arrive_expect_tx(&S.full[stage], qb + sb + hb + fb);
          bulk_g2s(dst, ep.q_down + (size_t)d.row0 * (p.I / 2), qb, &S.full[stage], policy);
          bulk_g2s(dst + p.RD * (p.I / 2), ep.s_down + (size_t)d.row0 * (p.I / 32), sb,
                   &S.full[stage], policy);
          const uint64_t keep = l2_policy_evict_last();
          bulk_g2s(dst + tail, p.hq + (size_t)d.slot * hb, hb, &S.full[stage], keep);
          bulk_g2s(dst + tail + hb, p.hqf + (size_t)d.slot * GD, fb, &S.full[stage], keep);
        } else {
          mbar_arrive(&S.full[stage]);  // a DONE fill: one per consumer group
          if (dones == 0) TRACE_AT(11);
          if (++dones == kGroups) {
            // leave no bulk copy in flight
            for (uint32_t m = (n >= (uint32_t)kStages ? n - kStages + 1 : 0); m < n; ++m) {
              mbar_wait(&S.full[m % kStages], (m / kStages) & 1u, kWaitNs);
            }
            break;
          }
        }
      }
    }
  } else if (warp == kSelectWarp) {
    // ------------------------------------------------------------ selection
    // the bias of this lane's experts (e = lane + 32 m), fetched while the
    // router runs; then poll the score records until every one carries this
    // call's epoch (bounded)
    float bs[kMaxE / 32];
#pragma unroll
    for (int m = 0; m < kMaxE / 32; ++m) {
      const int e = lane + 32 * m;
      bs[m] = e < p.E ? __ldg(p.bias + e) : 0.f;
    }
    uint64_t rec[kMaxE / 32];
    bool ok = true;
    {
      const uint64_t deadline = global_timer_ns() + kWaitNs;
      uint32_t sleep_ns = 32;
      for (uint32_t it = 0;; ++it) {
#pragma unroll
        for (int m = 0; m < kMaxE / 32; ++m) {
          const int e = lane + 32 * m;
          rec[m] = e < p.E ? ld_relaxed_u64(p.scores + e) : (uint64_t)epoch << 32;
        }
        bool mine = true;
#pragma unroll
        for (int m = 0; m < kMaxE / 32; ++m) mine = mine && (uint32_t)(rec[m] >> 32) == epoch;
        if (__all_sync(0xffffffffu, mine)) break;
        if ((it & 7) == 7) {
          const int stop = lane == 0 && (aborted(p.ctrl) || global_timer_ns() > deadline);
          if (__shfl_sync(0xffffffffu, stop, 0)) {
            ok = false;
            break;
          }
        }
        __nanosleep(sleep_ns);
        if (sleep_ns < 256) sleep_ns <<= 1;
      }
    }
    if (ok) {
      if (lane == 0) {
        TRACE_AT(4);
        S.sel_ok = 1;  // before any pick goes out
      }
#pragma unroll
      for (int m = 0; m < kMaxE / 32; ++m) {
        const int e = lane + 32 * m;
        if (e < p.E) {
          const float s = __uint_as_float((uint32_t)rec[m]);
          S.sc[e] = s;
          S.sp[e] = s + bs[m];
        }
      }
      __syncwarp();
      // every pick barrier gets its one arrival in here: as each pick is
      // popped, or all at the end of the selection
      run_select(sel_args(p), S);
      if (lane == 0) TRACE_AT(5);
    } else if (lane == 0) {
      set_error(p.ctrl, kErrTimeout, 8, 0);
      S.sel_ok = 0;
      for (int r = 0; r < p.k; ++r) mbar_arrive(&S.pickbar[r]);  // reported, not selected
    }
  } else if (warp == kConvWarp) {
    // ------------------------------------------------------------ converter
    // Publishes 32-row groups of h as int16 words (the XQ layout the down
    // consumers load) once their 32 rows are written.  CTA b owns groups
    // b, b + grid, ... of the order (the shared expert first, then picks
    // 0..k-1; groups ascending), the order in which gate/up items complete.
    const int GD = p.I >> 5, slots = p.k + p.has_shared;
    uint64_t pick_seen = 0;
    for (int i = blockIdx.x; i < slots * GD; i += gridDim.x) {
      const int so = i / GD, g = i % GD;
      const int slot = p.has_shared ? (so == 0 ? p.k : so - 1) : so;  // routed: a pick
      if (slot < p.k) {
        // a routed pick may be dropped by top-p: its h never comes
        if (!((pick_seen >> slot) & 1ull)) {
          int okw = 0;
          if (lane == 0) okw = mbar_wait(&S.pickbar[slot], 0u, kWaitNs) && S.sel_ok;
          if (!__shfl_sync(0xffffffffu, okw, 0)) break;  // the selection warp reported it
          mbar_test(&S.pickbar[slot], 0u);
          pick_seen |= 1ull << slot;
        }
        if (p.top_p < 1.f && !S.pick_kept[slot]) continue;
      }
      const uint32_t* cnt = p.ctrl + kCtrlHRows + slot * GD + g;
      // every lane acquires the count itself (so its own loads of h below
      // are ordered after the writers' release adds)
      bool ok = true;
      {
        const uint64_t deadline = global_timer_ns() + kWaitNs;
        for (uint32_t it = 0;; ++it) {
          if (__all_sync(0xffffffffu, ld_acquire(cnt) >= 32u)) break;
          if ((it & 7) == 7) {
            const int stop = lane == 0 && (aborted(p.ctrl) || global_timer_ns() > deadline);
            if (__shfl_sync(0xffffffffu, stop, 0)) {
              ok = false;
              break;
            }
          }
          __nanosleep(64);
        }
      }
      if (!ok) {
        if (lane == 0 && !aborted(p.ctrl)) set_error(p.ctrl, kErrTimeout, 9, (uint32_t)i);
        break;
      }
      const float hv = __ldcg(p.hbuf + (size_t)slot * p.I + g * 32 + lane);
      // the int16 group format of the layer kernels: the largest magnitude
      // maps into [2^14, 2^15), round to nearest even (xq_from_floats)
      float m = fabsf(hv);
#pragma unroll
      for (int o = 16; o >= 1; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
      int ex = 0;
      if (m > 0.f) frexpf(m, &ex);
      const int e = 15 - ex;
      const float sc = (m > 0.f) ? ldexpf(1.0f, e) : 0.f;
      const float b = fmaf(hv, sc, 12582912.0f);
      const int X = max(-32767, min(32767, (int)(__float_as_uint(b) - 0x4B400000u)));
      // element j = 8i + r sits in word ev[2i + (r >= 4)] (r even) or
      // od[2i + (r >= 4)] (r odd), low half for r % 4 < 2
      const int ii = lane >> 3, r = lane & 7;
      const int word = ((r & 1) ? 8 : 0) + 2 * ii + (r >= 4 ? 1 : 0);
      const int half = (r & 2) ? 1 : 0;
      uint16_t* dst = reinterpret_cast<uint16_t*>(p.hq + ((size_t)slot * GD + g) * 64);
      dst[2 * word + half] = (uint16_t)(X & 0xFFFF);
      if (lane == 0) p.hqf[(size_t)slot * GD + g] = (m > 0.f) ? ldexpf(1.0f, -e - 4) : 0.f;
      __syncwarp();
      if (lane == 0) {
        __threadfence();
        red_add_release(p.ctrl + kCtrlHqDone + slot, 1u);
        if (slot == p.k) TRACE_AT(21);
      }
    }
  } else {
    // ------------------------------------------------------------ consumers
    const int grp = warp / kGW;
    const int gw = warp % kGW;                 // warp index inside the group
    const int tg = gw * 32 + lane;             // thread index inside the group
    const int G = p.H >> 5, GD = p.I >> 5;
    const ColMap cg = group_col_map(G, gw, lane);
    const ColMap cd = group_col_map(GD, gw, lane);
    const int fw_g = (cg.P * NR_G + 31) / 32;  // finalizer warps of a gate/up item
    const int fw_d = (cd.P * NR_D + 31) / 32;  // finalizer warps of a down item

    // this thread's gate/up inputs (int16 groups) and router inputs (bf16)
    XQ xq;
    {
      float xf[32];
      if (p.x_resid) {
        const bool write_xn = blockIdx.x == 0 && grp == 0 && cg.phase == 0 && p.xn_out;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const uint2 b = norm_bf16x4(p.x_resid, cg.col * 32 + 4 * i, inv_rms);
          xf[4 * i] = bf16_bits_to_f32(b.x & 0xFFFFu);
          xf[4 * i + 1] = bf16_bits_to_f32(b.x >> 16);
          xf[4 * i + 2] = bf16_bits_to_f32(b.y & 0xFFFFu);
          xf[4 * i + 3] = bf16_bits_to_f32(b.y >> 16);
          if (write_xn) {  // xn_out is 4-byte aligned
            uint32_t* xo = reinterpret_cast<uint32_t*>(p.xn_out + cg.col * 32 + 4 * i);
            xo[0] = b.x;
            xo[1] = b.y;
          }
        }
      } else {
        const uint4* xp = reinterpret_cast<const uint4*>(p.x + cg.col * 32);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const uint4 v = __ldg(xp + i);
          const uint32_t u[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            xf[8 * i + 2 * j] = bf16_bits_to_f32(u[j] & 0xFFFFu);
            xf[8 * i + 2 * j + 1] = bf16_bits_to_f32(u[j] >> 16);
          }
        }
      }
      xq_from_floats(xf, xq);
    }
    int& gabort = S.abort_flag[grp];
    int dr0, dr1;
    down_rows(p, blockIdx.x, dr0, dr1);
    int rr0, rnr;
    router_rows(p, blockIdx.x, rr0, rnr);
    // group 0's router inputs (bf16)
    uint2 xr[kRouterChunks];
    const int rchunks = p.H >> 2;
#pragma unroll
    for (int i = 0; i < kRouterChunks; ++i) {
      const int cc = tg + kGT * i;
      if (grp >= router_fills(rnr) || cc >= rchunks) {
        xr[i] = make_uint2(0, 0);
      } else if (p.x_resid) {
        xr[i] = norm_bf16x4(p.x_resid, 4 * cc, inv_rms);
      } else {
        xr[i] = __ldg(reinterpret_cast<const uint2*>(p.x) + cc);
      }
    }
    // Group g of a CTA with router rows: fill g is its router block.  It is
    // handled before the main loop so its bf16 inputs are dead afterwards.
    uint32_t c_first = 0;
    {
      if (grp < router_fills(rnr)) {
        c_first = 1;
        const int stage = grp;
        const uint32_t gpar = 0u;
        int okw = 0;
        if (lane == 0) okw = mbar_wait(&S.full[stage], 0u, kWaitNs) ? 1 : 0;
        const bool ok = __shfl_sync(0xffffffffu, okw, 0) != 0;
        if (ok) {
          mbar_test(&S.full[stage], 0u);
          if (tg == 0 && grp == 0) TRACE_AT(2);
        } else {
          if (lane == 0) set_error(p.ctrl, kErrTimeout, 1, 0);
          gabort = 1;
        }
        const ItemDesc d = S.desc[stage];
        const uint8_t* st = stages + (size_t)stage * kStageBytes;
        // double-float sums of the exact fp32 x bf16 products: each product
        // is split exactly into p + e, the p are summed error-free into
        // (hi, lo) and the e added to lo -- about 48 bits with fp32
        // arithmetic only, so the logit is exact to ~1e-14 and the
        // selection sees scores rounded only once (to fp32).  Four
        // independent chains per row (one per lane of a float4).
        float xv[kRouterChunks][4];
#pragma unroll
        for (int i = 0; i < kRouterChunks; ++i) {
          xv[i][0] = bf16_bits_to_f32(xr[i].x & 0xFFFFu);
          xv[i][1] = bf16_bits_to_f32(xr[i].x >> 16);
          xv[i][2] = bf16_bits_to_f32(xr[i].y & 0xFFFFu);
          xv[i][3] = bf16_bits_to_f32(xr[i].y >> 16);
        }
        const int nrr = ok ? d.nrows : 0;
        for (int r = 0; r < nrr; ++r) {
          const float4* wr = reinterpret_cast<const float4*>(st + (size_t)r * p.H * 4);
          DF c0{0.f, 0.f}, c1{0.f, 0.f}, c2{0.f, 0.f}, c3{0.f, 0.f};
#pragma unroll
          for (int i = 0; i < kRouterChunks; ++i) {
            const int cc = tg + kGT * i;
            if (cc < rchunks) {
              const float4 wv = wr[cc];
              df_add_prod(c0, wv.x, xv[i][0]);
              df_add_prod(c1, wv.y, xv[i][1]);
              df_add_prod(c2, wv.z, xv[i][2]);
              df_add_prod(c3, wv.w, xv[i][3]);
            }
          }
          const DF v = df_warp_sum(df_add(df_add(c0, c1), df_add(c2, c3)));
          if (lane == 0) S.redd[grp * kGW + gw][r] = (double)v.hi + (double)v.lo;
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&S.empty[stage]);
        if (tg == 0 && grp == 0) TRACE_AT(15);
        if (!group_barrier(&S.gbar[grp], gpar)) {
          if (lane == 0) set_error(p.ctrl, kErrTimeout, 3, 0);
          gabort = 1;
        }
        if (!gabort && gw == 0) {
          // the sigmoid score of each row, tagged with this call's epoch
          if (lane < d.nrows) {
            double v = 0.0;
            for (int w = 0; w < kGW; ++w) v += S.redd[grp * kGW + w][lane];
            const float sg = sigmoid_f64_to_f32(v);
            st_relaxed_u64(p.scores + d.row0 + lane,
                           ((uint64_t)epoch << 32) | __float_as_uint(sg));
          }
          if (lane == 0 && grp == 0) TRACE_AT(3);
        }
      }
    }
    // Group 1 of a CTA whose router rows all went to group 0 starts with two
    // placeholder items (a gate/up, then a down item) that run the real loop
    // body on whatever the stage holds and publish nothing: the instructions
    // of both paths are fetched while the first weights are still on their
    // way, not when they have arrived.  (A group that had router rows has
    // spent that time on them; placeholders would only delay its first item.)
    int warm = (grp == 1 && p.warm && c_first == 0) ? 2 : 0;
    uint32_t c = c_first;
    for (uint32_t it = c_first;; ++it) {  // it: group barrier phases used
      if (gabort) break;
      const bool fake = warm > 0;
      const uint32_t n = 2 * c + grp;  // fill number consumed
      const int stage = (int)(n % kStages);
      const uint32_t par = (n / kStages) & 1u;
      const int rbuf = it & 1;
      const uint32_t gpar = it & 1u;  // one group barrier per iteration
      // Every path through this loop body passes the group barrier exactly
      // once, and wait results are uniform per warp, so a wait that runs out
      // in one warp can never leave a barrier or a shuffle half-joined.
      bool ok = true;
      if (!fake) {
        int okw = 0;
        if (lane == 0) okw = mbar_wait(&S.full[stage], par, kWaitNs) ? 1 : 0;
        ok = __shfl_sync(0xffffffffu, okw, 0) != 0;
        if (ok) {
          mbar_test(&S.full[stage], par);  // acquire the bulk-copied bytes in every lane
        } else {
          if (lane == 0) set_error(p.ctrl, kErrTimeout, 1, n);
          gabort = 1;
        }
      }
      const ItemDesc d = fake ? make_item(warm == 2 ? kGateUp : kDown, 0, 0, 0) : S.desc[stage];
      if (fake) {
        --warm;
      } else {
        ++c;
      }
      if (!ok || d.type == kDone) {
        group_barrier(&S.gbar[grp], gpar);
        break;
      }
      const uint8_t* st = stages + (size_t)stage * kStageBytes;
      if (d.type == kGateUp) {
        float v[NV_G];
        const size_t rb = (size_t)p.H / 2;
        const uint8_t* qg = st;
        const uint8_t* qu = st + (size_t)p.RG * rb;
        const uint16_t* sg = reinterpret_cast<const uint16_t*>(st + 2 * (size_t)p.RG * rb);
        const uint16_t* su = sg + (size_t)p.RG * G;
        // Rows past nrows (a partial last item) are computed from whatever
        // the stage holds and dropped at the finalize: no branch in the loop.
#pragma unroll
        for (int r = 0; r < NR_G; ++r) {
          const int lr = cg.phase * NR_G + r;
          const uint4 wg = *reinterpret_cast<const uint4*>(qg + lr * rb + cg.col * 16);
          const uint4 wu = *reinterpret_cast<const uint4*>(qu + lr * rb + cg.col * 16);
          v[r] = dot_scaled(wg, xq, f16_bits_to_f32(sg[lr * G + cg.col]));
          v[NR_G + r] = dot_scaled(wu, xq, f16_bits_to_f32(su[lr * G + cg.col]));
        }
        __syncwarp();
        if (lane == 0 && !fake) mbar_arrive(&S.empty[stage]);
        reduce_scatter<NV_G, SEG_G>(v);
        S.red[grp][rbuf][gw][lane] = v[0];
        if (!group_barrier(&S.gbar[grp], gpar)) {
          if (lane == 0) set_error(p.ctrl, kErrTimeout, 3, n);
          gabort = 1;
        }
        if (gabort) break;

        if (gw < fw_g) {
          // item row tg (= phase * NR_G + i) of this finalizer thread
          if (tg < cg.P * NR_G && tg < d.nrows) {
            const int ph = tg / NR_G, i = tg % NR_G;
            int w0, lg, lu;
            owner_of<NV_G, SEG_G>(ph, i, cg.wpr, w0, lg);
            owner_of<NV_G, SEG_G>(ph, i + NR_G, cg.wpr, w0, lu);
            float g = 0.f, u = 0.f;
            for (int w = 0; w < cg.wpr; ++w) {
              g += S.red[grp][rbuf][w0 + w][lg];
              u += S.red[grp][rbuf][w0 + w][lu];
            }
            p.hbuf[(size_t)d.slot * p.I + d.row0 + tg] = silu_mul(g, u);
          }
          // count the rows of h this warp wrote, per 32-row group of h (its
          // rows are consecutive: at most two groups); the converter warp
          // that owns a group publishes it once all 32 rows are in
          const bool wrote = tg < cg.P * NR_G && tg < d.nrows;
          const unsigned vm = __ballot_sync(0xffffffffu, wrote);
          if (vm && !fake) {
            const int g = (d.row0 + tg) >> 5;
            const int g0 = __shfl_sync(0xffffffffu, g, __ffs(vm) - 1);
            const unsigned m0 = __ballot_sync(0xffffffffu, wrote && g == g0);
            const unsigned m1 = vm & ~m0;
            __syncwarp();
            if (lane == 0) {
              uint32_t* cnt = p.ctrl + kCtrlHRows + d.slot * (p.I >> 5);
              red_add_release(cnt + g0, (uint32_t)__popc(m0));
              if (m1) red_add_release(cnt + g0 + 1, (uint32_t)__popc(m1));
              if (d.slot == p.k) TRACE_AT(22);
            }
          }
        }
      } else {  // kDown
        XQ hq;  // this thread's 32-row group of h: int16 words and factor
        {
          const uint8_t* tail = st + (size_t)p.RD * (p.I / 2 + p.I / 16);
          const uint4* hw = reinterpret_cast<const uint4*>(tail + (size_t)cd.col * 64);
          const uint4 a0 = hw[0], a1 = hw[1], a2 = hw[2], a3 = hw[3];
          hq.ev[0] = a0.x; hq.ev[1] = a0.y; hq.ev[2] = a0.z; hq.ev[3] = a0.w;
          hq.ev[4] = a1.x; hq.ev[5] = a1.y; hq.ev[6] = a1.z; hq.ev[7] = a1.w;
          hq.od[0] = a2.x; hq.od[1] = a2.y; hq.od[2] = a2.z; hq.od[3] = a2.w;
          hq.od[4] = a3.x; hq.od[5] = a3.y; hq.od[6] = a3.z; hq.od[7] = a3.w;
          hq.f = reinterpret_cast<const float*>(tail + (size_t)GD * 64)[cd.col];
        }
        float v[NR_D];
        const size_t rb = (size_t)p.I / 2;
        const uint16_t* sd = reinterpret_cast<const uint16_t*>(st + (size_t)p.RD * rb);
#pragma unroll
        for (int r = 0; r < NR_D; ++r) {
          const int lr = cd.phase * NR_D + r;
          const uint4 wd = *reinterpret_cast<const uint4*>(st + lr * rb + cd.col * 16);
          v[r] = dot_scaled(wd, hq, f16_bits_to_f32(sd[lr * GD + cd.col]));
        }
        __syncwarp();
        if (lane == 0 && !fake) mbar_arrive(&S.empty[stage]);
        reduce_scatter<NR_D, SEG_D>(v);
        S.red[grp][rbuf][gw][lane] = v[0];
        if (!group_barrier(&S.gbar[grp], gpar)) {
          if (lane == 0) set_error(p.ctrl, kErrTimeout, 3, n);
          gabort = 1;
        }
        if (gabort) break;

        if (gw < fw_d && !fake) {
          if (tg < cd.P * NR_D) {
            const int ph = tg / NR_D, i = tg % NR_D;
            const int lr = ph * NR_D + i;
            if (lr < d.nrows) {
              int w0, l0;
              owner_of<NR_D, SEG_D>(ph, i, cd.wpr, w0, l0);
              float s = 0.f;
              for (int w = 0; w < cd.wpr; ++w) s += S.red[grp][rbuf][w0 + w][l0];
              // this slot's partial of one of the CTA's own rows
              S.ycta[d.slot * p.ycta_rows + (d.row0 - dr0) + lr] = s;
            }
          }
        }
      }
    }
  }

  // -------------------------------------------------------------- teardown
  __syncthreads();
  {
    // y of this CTA's own rows: the partials combined in slot order
    // (sum_j w_j y_j, then the shared expert, then the residual input),
    // the same order for every call: no atomics, bitwise repeatable
    int r0, r1;
    down_rows(p, blockIdx.x, r0, r1);
    if (!aborted(p.ctrl)) {
      for (int lr = threadIdx.x; lr < r1 - r0; lr += kThreads) {
        float acc = 0.f;
        for (int j = 0; j < p.k; ++j)
          if (S.sel_idx[j] >= 0)
            acc = fmaf(S.sel_w[j], S.ycta[S.slot_pick[j] * p.ycta_rows + lr], acc);
        if (p.has_shared) acc += S.ycta[p.k * p.ycta_rows + lr];
        if (p.x_resid) acc = p.x_resid[r0 + lr] + acc;  // x + MoE(norm(x))
        p.y[r0 + lr] = acc;
      }
    }
  }
  if (threadIdx.x == 0) {
    TRACE_AT(10);
    __threadfence();
    const uint32_t old = atomicAdd(p.ctrl + kCtrlExit, 1u);
    S.last_cta = (old + 1 == gridDim.x) ? 1 : 0;
#ifdef MOE_TRACE
    // per call (by epoch): the first CTA's start and the last CTA's exit
    if (p.trace && S.last_cta) {
      p.trace[gridDim.x * 128 + (epoch & 63) * 2 + 1] = global_timer_ns();
      p.trace[gridDim.x * 128 + (epoch & 63) * 2 + 0] = p.trace[127];  // CTA 0's start
    }
#endif
  }
  __syncthreads();
  if (S.last_cta) {
    // last CTA out: reset the counters for the next call (the error word
    // is left for the host to read) and advance the epoch
    __threadfence();
    volatile uint32_t* c = p.ctrl;
    for (int j = threadIdx.x; j < slots; j += kThreads) c[kCtrlHqDone + j] = 0;
    for (int j = threadIdx.x; j < slots * (p.I >> 5); j += kThreads) c[kCtrlHRows + j] = 0;
    __syncthreads();
    if (threadIdx.x == 0) {
      c[kCtrlTicket] = 0;
      c[kCtrlAbort] = 0;
      c[kCtrlEpoch] = epoch;
      c[kCtrlExit] = 0;
      __threadfence();
    }
  }
}

// The kernel needs all of its CTAs resident at once (selection warps poll
// every CTA's router records; down items wait on other CTAs' gate/up
// counts), so it is launched cooperatively: a grid that cannot be
// co-resident (another kernel holding SMs, a partitioned device) fails at
// launch instead of running into the device-side wait limit.  It is also a
// programmatic dependent launch: its prologue may overlap the end of the
// previous call on the stream (the kernel waits on griddepcontrol before it
// reads anything an earlier call writes).  The first launch per device and
// context sets the shared-memory attribute and checks that one CTA fits on
// an SM.
template <int SEG_G, int SEG_D>
cudaError_t launch_t(const DecodeParams& p, cudaStream_t st) {
  static DeviceOnce<bool> configured;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  const size_t smem = decode_smem_bytes();
  bool ok = false;
  e = configured.get(dev, &ok, [smem](bool* v) {
    cudaError_t r = cudaFuncSetAttribute(decode_kernel<SEG_G, SEG_D>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (r != cudaSuccess) return r;
    int per_sm = 0;
    r = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, decode_kernel<SEG_G, SEG_D>,
                                                      kThreads, smem);
    if (r != cudaSuccess) return r;
    if (per_sm < 1) return cudaErrorCooperativeLaunchTooLarge;
    *v = true;
    return cudaSuccess;
  });
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)num_sms());
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeCooperative;
  attr[0].val.cooperative = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  return cudaLaunchKernelEx(&cfg, decode_kernel<SEG_G, SEG_D>, p);
}

template <int SEG_G>
cudaError_t launch_g(const DecodeParams& p, int seg_d, cudaStream_t st) {
  switch (seg_d) {
    case 32: return launch_t<SEG_G, 32>(p, st);
    case 16: return launch_t<SEG_G, 16>(p, st);
    case 8: return launch_t<SEG_G, 8>(p, st);
    case 4: return launch_t<SEG_G, 4>(p, st);
    case 2: return launch_t<SEG_G, 2>(p, st);
  }
  return cudaErrorInvalidValue;
}

int seg_of(int G) { return G >= 32 ? 32 : G; }

// Concurrent row phases of the column mapping over one group's warps.
bool phases(int G, int& P) {
  if (G >= 32) {
    const int wpr = G / 32;
    if (kGW % wpr) return false;
    P = kGW / wpr;
  } else {
    P = kGW * (32 / G);
  }
  return true;
}

}  // namespace

static_assert((size_t)kStages * kStageBytes + sizeof(Smem) <= 232448,
              "one CTA's dynamic shared memory must fit the 227 KB limit");
size_t decode_smem_bytes() { return (size_t)kStages * kStageBytes + sizeof(Smem); }

bool decode_plan(const moe_config& c, DecodeParams& p) {
  const int G = c.hidden / 32, GD = c.inter / 32;
  int PG, PD;
  if (!phases(G, PG) || !phases(GD, PD)) return false;
  if (c.hidden / 4 > kRouterChunks * kGT) return false;
  if (c.n_experts > kMaxE) return false;
  const int sg = seg_of(G), sd = seg_of(GD);
  const int nrg = (sg / 2 < 8) ? sg / 2 : 8;
  const int nrd = (sd < 16) ? sd : 16;
  p.H = c.hidden;
  p.I = c.inter;
  p.E = c.n_experts;
  p.k = c.top_k;
  p.n_group = c.n_group;
  p.topk_group = c.topk_group;
  p.has_shared = c.n_shared;
  p.rsf = c.routed_scaling_factor;
  {
    const int per = c.n_experts / c.n_group, q = (c.n_experts + 31) / 32;
    const int L = per / q;
    p.sel_q = q;
    p.sel_lgL = 0;
    while ((1 << p.sel_lgL) < L) ++p.sel_lgL;
    p.sel_fast = per % q == 0 && L >= 1 && (1 << p.sel_lgL) == L && q <= kMaxE / 32;
  }
  p.RG = PG * nrg;
  {
    // A down item is RD rows of q_down and s_down, then the slot's int16 h
    // groups (GD x 64 bytes) and their factors (GD x 4 bytes, whole 16-byte
    // units).  Rows go in units of A, so that every scale row offset is
    // 16-byte aligned (A * GD * 2 bytes a multiple of 16).
    if (GD % 4) return false;
    int g8 = GD, m8 = 8;
    while (m8) {
      const int t = g8 % m8;
      g8 = m8;
      m8 = t;
    }
    p.A = 8 / g8;
    const size_t tail = (size_t)GD * 64 + (size_t)GD * 4, rowb = (size_t)c.inter / 2 + c.inter / 16;
    if (tail >= kStageBytes) return false;
    p.RD = min(PD * nrd, (int)((kStageBytes - tail) / rowb));
    p.RD -= p.RD % p.A;
    if (p.RD < p.A) return false;
  }
  p.RR = (int)(kStageBytes / ((uint32_t)c.hidden * 4));
  if (p.RR > kMaxRR) p.RR = kMaxRR;
  if (p.RR < 1) return false;
  if ((size_t)p.RG * (c.hidden / 2 + c.hidden / 16) * 2 > kStageBytes) return false;
  if ((p.RG * (c.hidden / 16)) % 16) return false;
  const int grid = num_sms();
  if ((p.E + grid - 1) / grid > p.RR) return false;  // a CTA's router rows fill one stage
  p.nR = p.E < grid ? p.E : grid;  // CTAs with at least one router row
  p.nG = (p.I + p.RG - 1) / p.RG;
  const int slots = p.k + p.has_shared;
  p.nU = p.H / p.A;
  p.ycta_rows = p.A * ((p.nU + grid - 1) / grid);  // most down rows a CTA owns
  p.n_db = (p.ycta_rows + p.RD - 1) / p.RD;
  if (slots * p.ycta_rows > kMaxYcta) return false;
  // the control words' ranges
  if (slots > kMaxSlots || kCtrlHqDone + slots > kCtrlHRows) return false;
  if (kCtrlHRows + slots * GD > kCtrlWords) return false;
  return true;
}

cudaError_t launch_decode(const DecodeParams& p, cudaStream_t st) {
  const int sg = seg_of(p.H / 32), sd = seg_of(p.I / 32);
  switch (sg) {
    case 32: return launch_g<32>(p, sd, st);
    case 16: return launch_g<16>(p, sd, st);
    case 8: return launch_g<8>(p, sd, st);
    case 4: return launch_g<4>(p, sd, st);
    case 2: return launch_g<2>(p, sd, st);
  }
  return cudaErrorInvalidValue;
}

}  // namespace moe
