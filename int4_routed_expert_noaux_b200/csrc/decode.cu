// decode.cu -- the fused persistent decode kernel: the whole routed-MoE
// layer for one token (router GEMV, noaux_tc selection, 8 routed + shared
// int4 expert FFNs, weighted combine) in ONE launch.
//
// Design (sm_100a):
//  * one CTA per SM; warp 6 is the producer, warps 0-5 (192 threads) consume;
//  * the producer claims work items from a global ticket counter, in a fixed
//    order, and moves each item's weights HBM -> shared memory with 1-D bulk
//    async copies (the TMA engine) into a 3-stage ring of 56 KB stages,
//    completion tracked by mbarriers (transaction bytes);
//  * consumers are column-stationary: each thread owns one 16-byte chunk
//    column of the rows it visits, keeps its 32 inputs in registers and runs
//    the LOP3 + packed-FMA int4 group dot product; one butterfly
//    reduce-scatter plus a cross-warp sum finishes each row;
//  * item order: router rows, shared-expert gate/up, shared-expert down,
//    routed gate/up of slot 0, then (gate/up of slot j, down of slot j-1)
//    for j = 1..k-1, then down of slot k-1.  Every dependency points to an
//    earlier ticket (router -> selection -> routed items; gate/up of a slot
//    -> its down items), so in-order claiming always makes progress;
//  * the CTA that finishes the last router item runs the selection and
//    publishes idx / w with a release flag; the producer acquires it before
//    loading routed weights;
//  * down items write per-slot partial rows; the CTA that completes the last
//    slot of a row block sums the partials in slot order (deterministic,
//    no atomics on data) into y;
//  * every wait is bounded (1 s); a wait that runs out sets the workspace
//    error word, and all threads leave in step; the last CTA to exit resets
//    the control counters so the next call starts clean.
#include <cuda_runtime.h>
#include <stdint.h>

#include "async.cuh"
#include "common.cuh"
#include "decode.h"

namespace moe {

namespace {

constexpr int kCW = 6;                  // consumer warps
constexpr int kCT = kCW * 32;           // consumer threads
constexpr int kThreads = kCT + 32;      // + producer warp
constexpr int kStages = 3;
constexpr uint32_t kStageBytes = 57344;
constexpr int kRouterChunks = 8;        // 16-byte W chunks per consumer per row
constexpr int kMaxRR = 8;               // router rows per item
constexpr uint64_t kWaitNs = 1000000000ull;

enum ItemType : int { kRouter = 0, kGateUp = 1, kDown = 2, kDone = 3 };

struct ItemDesc {
  int type, slot, row0, nrows, eid, pad0, pad1, pad2;
};

struct Smem {
  uint64_t full[kStages];
  uint64_t empty[kStages];
  ItemDesc desc[kStages];
  float red[kCW][32];
  int status;        // consumer broadcast: 1 = go on, 0 = stop
  int flag;          // consumer broadcast: run select / combine
  float gscore[32];
  float sc[1024];
  float sp[1024];
};

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

__device__ ItemDesc decode_ticket(const DecodeParams& p, int t) {
  if (t < p.nR) return make_item(kRouter, 0, t * p.RR, min(p.RR, p.E - t * p.RR));
  t -= p.nR;
  auto gu = [&](int slot, int b) {
    return make_item(kGateUp, slot, b * p.RG, min(p.RG, p.I - b * p.RG));
  };
  auto dn = [&](int slot, int b) {
    return make_item(kDown, slot, b * p.RD, min(p.RD, p.H - b * p.RD));
  };
  if (p.has_shared) {
    if (t < p.nG) return gu(p.k, t);
    t -= p.nG;
    if (t < p.nD) return dn(p.k, t);
    t -= p.nD;
  }
  if (t < p.nG) return gu(0, t);
  t -= p.nG;
  const int pair = p.nG + p.nD;
  if (t < (p.k - 1) * pair) {
    const int j = t / pair + 1, u = t % pair;
    return u < p.nG ? gu(j, u) : dn(j - 1, u - p.nG);
  }
  t -= (p.k - 1) * pair;
  if (t < p.nD) return dn(p.k - 1, t);
  return make_item(kDone, 0, 0, 0);
}

__device__ __forceinline__ void set_error(uint32_t* ctrl, uint32_t code) {
  atomicCAS(ctrl + kCtrlErr, 0u, code);
  atomicExch(ctrl + kCtrlAbort, 1u);
}

__device__ __forceinline__ bool aborted(const uint32_t* ctrl) {
  return *((volatile const uint32_t*)(ctrl + kCtrlAbort)) != 0;
}

// Bounded poll of a global counter until it reaches `target`.
__device__ bool wait_counter(uint32_t* ctrl, const uint32_t* p, uint32_t target) {
  if (ld_acquire(p) >= target) return true;
  const uint64_t deadline = global_timer_ns() + kWaitNs;
  for (uint32_t it = 0;; ++it) {
    if (ld_acquire(p) >= target) return true;
    __nanosleep(64);
    if ((it & 15) == 15) {
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

// noaux_tc selection over the logits (all consumer threads of one CTA).
__device__ void run_select(const DecodeParams& p, Smem& S) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int per = p.E / p.n_group;
  for (int g = warp; g < p.n_group; g += kCW) {
    ArgMaxF a{0.f, -1};
    if (lane < per) {
      const int e = g * per + lane;
      const float s = 1.0f / (1.0f + expf(-__ldcg(p.logits + e)));
      const float sp = s + __ldg(p.bias + e);
      S.sc[e] = s;
      S.sp[e] = sp;
      a = ArgMaxF{sp, e};
    }
    const ArgMaxF t1 = am_warp(a);
    ArgMaxF b = a;
    if (b.i == t1.i) b.i = -1;
    const ArgMaxF t2 = am_warp(b);
    if (lane == 0) S.gscore[g] = (t2.i >= 0) ? t1.v + t2.v : t1.v;
  }
  named_bar(1, kCT);
  if (warp != 0) return;
  bool kept = false;
  {
    const ArgMaxF g{lane < p.n_group ? S.gscore[lane] : 0.f, lane < p.n_group ? lane : -1};
    for (int r = 0; r < p.topk_group; ++r) {
      const ArgMaxF best = am_warp(kept ? ArgMaxF{0.f, -1} : g);
      if (best.i == lane) kept = true;
    }
  }
  const unsigned kept_mask = __ballot_sync(0xffffffffu, kept);
  const int nper = (p.E + 31) >> 5;
  unsigned taken = 0;
  int my_sel = -1;
  for (int r = 0; r < p.k; ++r) {
    ArgMaxF a{0.f, -1};
    for (int m = 0; m < nper; ++m) {
      const int e = lane + 32 * m;
      if (e < p.E && ((kept_mask >> (e / per)) & 1u) && !((taken >> m) & 1u))
        a = am_merge(a, ArgMaxF{S.sp[e], e});
    }
    const ArgMaxF best = am_warp(a);
    if (best.i >= 0 && (best.i & 31) == lane) taken |= 1u << (best.i >> 5);
    if (lane == r) my_sel = best.i;
  }
  int rank = 0;
  for (int j = 0; j < p.k; ++j) {
    const int other = __shfl_sync(0xffffffffu, my_sel, j);
    if (lane < p.k && other < my_sel) ++rank;
  }
  const float s_mine = (lane < p.k && my_sel >= 0) ? S.sc[my_sel] : 0.f;
  const float denom = [&] {
    float v = s_mine;
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
  }() + 1e-20f;
  if (lane < p.k) {
    const float wv = p.rsf * s_mine / denom;
    p.idx_ws[rank] = my_sel;
    p.w_ws[rank] = wv;
    if (p.idx_out) p.idx_out[rank] = my_sel;
    if (p.w_out) p.w_out[rank] = wv;
  }
  __threadfence();
  __syncwarp();
  if (lane == 0) st_release(p.ctrl + kCtrlSelReady, 1u);
}

// Index of the lane holding reduce-scatter value `vi` for row-phase `ph`.
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

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&S.full[s], 1);
      mbar_init(&S.empty[s], kCW);
    }
    fence_mbar_init();
  }
  __syncthreads();

  if (warp == kCW) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      const uint64_t policy = l2_policy_evict_first();
      bool sel_seen = false;
      uint32_t filled = 0;    // bit s: stage s has been filled at least once
      uint32_t last_par = 0;  // bit s: parity of the latest fill of stage s
      int stage = 0;
      int t = (int)atomicAdd(p.ctrl + kCtrlTicket, 1u);
      bool stop = false;
      while (!stop) {
        ItemDesc d = decode_ticket(p, t);
        if (d.type != kDone && d.type != kRouter) {
          if (d.slot < p.k) {
            if (!sel_seen) {
              if (!wait_counter(p.ctrl, p.ctrl + kCtrlSelReady, 1u)) {
                set_error(p.ctrl, kErrTimeout);
                d = make_item(kDone, 0, 0, 0);
              } else {
                sel_seen = true;
              }
            }
            if (d.type != kDone) {
              d.eid = __ldcg(p.idx_ws + d.slot);
              if (d.eid < 0 || d.eid >= p.E) {
                set_error(p.ctrl, kErrBadExpertId);
                d = make_item(kDone, 0, 0, 0);
              }
            }
          } else {
            d.eid = p.E;  // shared expert
          }
        }
        // wait until the consumers released this stage's previous contents
        if (filled & (1u << stage)) {
          const uint64_t deadline = global_timer_ns() + kWaitNs;
          if (!mbar_wait(&S.empty[stage], (last_par >> stage) & 1u, deadline)) {
            set_error(p.ctrl, kErrTimeout);
            break;  // consumers time out on their own full-barrier waits
          }
        }
        S.desc[stage] = d;
        uint8_t* dst = stages + (size_t)stage * kStageBytes;
        if (d.type == kRouter) {
          const uint32_t bytes = (uint32_t)d.nrows * p.H * 4;
          mbar_arrive_expect_tx(&S.full[stage], bytes);
          bulk_g2s(dst, p.w_router + (size_t)d.row0 * p.H, bytes, &S.full[stage], policy);
        } else if (d.type == kGateUp) {
          const ExpertPtrs ep = p.table[d.eid];
          const uint32_t qb = (uint32_t)d.nrows * (p.H / 2), sb = (uint32_t)d.nrows * (p.H / 16);
          const size_t qoff = (size_t)d.row0 * (p.H / 2), soff = (size_t)d.row0 * (p.H / 32);
          mbar_arrive_expect_tx(&S.full[stage], 2 * (qb + sb));
          bulk_g2s(dst, ep.q_gate + qoff, qb, &S.full[stage], policy);
          bulk_g2s(dst + p.RG * (p.H / 2), ep.q_up + qoff, qb, &S.full[stage], policy);
          bulk_g2s(dst + 2 * p.RG * (p.H / 2), ep.s_gate + soff, sb, &S.full[stage], policy);
          bulk_g2s(dst + 2 * p.RG * (p.H / 2) + p.RG * (p.H / 16), ep.s_up + soff, sb,
                   &S.full[stage], policy);
        } else if (d.type == kDown) {
          const ExpertPtrs ep = p.table[d.eid];
          const uint32_t qb = (uint32_t)d.nrows * (p.I / 2), sb = (uint32_t)d.nrows * (p.I / 16);
          mbar_arrive_expect_tx(&S.full[stage], qb + sb);
          bulk_g2s(dst, ep.q_down + (size_t)d.row0 * (p.I / 2), qb, &S.full[stage], policy);
          bulk_g2s(dst + p.RD * (p.I / 2), ep.s_down + (size_t)d.row0 * (p.I / 32), sb,
                   &S.full[stage], policy);
        } else {
          mbar_arrive(&S.full[stage]);
          stop = true;
        }
        // this fill's parity: 0 for the first fill, then alternating
        last_par = (filled & (1u << stage)) ? (last_par ^ (1u << stage)) : (last_par & ~(1u << stage));
        filled |= 1u << stage;
        stage = (stage + 1 == kStages) ? 0 : stage + 1;
        if (!stop) t = (int)atomicAdd(p.ctrl + kCtrlTicket, 1u);
      }
      // leave no bulk copy in flight: wait (bounded) for every issued fill
      for (int s = 0; s < kStages; ++s) {
        if (filled & (1u << s)) {
          const uint64_t deadline = global_timer_ns() + kWaitNs;
          mbar_wait(&S.full[s], (last_par >> s) & 1u, deadline);
        }
      }
    }
  } else {
    // ------------------------------------------------------------ consumers
    const int G = p.H >> 5, GD = p.I >> 5;
    const ColMap cg = col_map_n(G, kCW);
    const ColMap cd = col_map_n(GD, kCW);
    const int tid = threadIdx.x;

    XGroup xg;
    {
      float xf[32];
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
      xgroup_from_floats(xf, xg);
    }
    float4 xr[kRouterChunks];
    const int rchunks = p.H >> 2;
#pragma unroll
    for (int i = 0; i < kRouterChunks; ++i) {
      const int c = tid + kCT * i;
      if (c < rchunks) {
        const uint2 v = __ldg(reinterpret_cast<const uint2*>(p.x) + c);
        xr[i] = make_float4(bf16_bits_to_f32(v.x & 0xFFFFu), bf16_bits_to_f32(v.x >> 16),
                            bf16_bits_to_f32(v.y & 0xFFFFu), bf16_bits_to_f32(v.y >> 16));
      } else {
        xr[i] = make_float4(0.f, 0.f, 0.f, 0.f);
      }
    }

    int stage = 0;
    uint32_t cons_par = 0;  // bit s: parity of the next consumption of stage s
    for (;;) {
      const uint32_t par = (cons_par >> stage) & 1u;
      if (tid == 0) {
        const uint64_t deadline = global_timer_ns() + kWaitNs;
        int go = mbar_wait(&S.full[stage], par, deadline) ? 1 : 0;
        if (!go) set_error(p.ctrl, kErrTimeout);
        if (go && S.desc[stage].type == kDown) {
          if (!wait_counter(p.ctrl, p.ctrl + kCtrlGuDone + S.desc[stage].slot, (uint32_t)p.nG)) {
            set_error(p.ctrl, kErrTimeout);
            go = 0;
          }
        }
        S.status = go;
      }
      named_bar(1, kCT);
      if (!S.status) break;
      mbar_test(&S.full[stage], par);  // acquire the bulk-copied bytes
      const ItemDesc d = S.desc[stage];
      if (d.type == kDone) break;
      const uint8_t* st = stages + (size_t)stage * kStageBytes;

      if (d.type == kRouter) {
        float acc[kMaxRR];
#pragma unroll
        for (int r = 0; r < kMaxRR; ++r) {
          acc[r] = 0.f;
          if (r < d.nrows) {
            const float4* wr = reinterpret_cast<const float4*>(st + (size_t)r * p.H * 4);
#pragma unroll
            for (int i = 0; i < kRouterChunks; ++i) {
              const int c = tid + kCT * i;
              if (c < rchunks) {
                const float4 wv = wr[c];
                acc[r] = fmaf(wv.x, xr[i].x, acc[r]);
                acc[r] = fmaf(wv.y, xr[i].y, acc[r]);
                acc[r] = fmaf(wv.z, xr[i].z, acc[r]);
                acc[r] = fmaf(wv.w, xr[i].w, acc[r]);
              }
            }
          }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&S.empty[stage]);
#pragma unroll
        for (int r = 0; r < kMaxRR; ++r) {
          if (r < d.nrows) {
            const float v = warp_sum(acc[r]);
            if (lane == 0) S.red[warp][r] = v;
          }
        }
        named_bar(1, kCT);
        if (tid < d.nrows) {
          float v = 0.f;
          for (int w = 0; w < kCW; ++w) v += S.red[w][tid];
          p.logits[d.row0 + tid] = v;
          __threadfence();
        }
        named_bar(1, kCT);
        if (tid == 0) {
          const uint32_t old = atom_add_acq_rel(p.ctrl + kCtrlRouterDone, 1u);
          S.flag = (old + 1 == (uint32_t)p.nR) ? 1 : 0;
        }
        named_bar(1, kCT);
        if (S.flag) run_select(p, S);
      } else if (d.type == kGateUp) {
        float v[NV_G];
        const size_t rb = (size_t)p.H / 2;
        const uint8_t* qg = st;
        const uint8_t* qu = st + (size_t)p.RG * rb;
        const uint16_t* sg = reinterpret_cast<const uint16_t*>(st + 2 * (size_t)p.RG * rb);
        const uint16_t* su = sg + (size_t)p.RG * G;
#pragma unroll
        for (int r = 0; r < NR_G; ++r) {
          const int lr = cg.phase * NR_G + r;
          float pg = 0.f, pu = 0.f;
          if (lr < d.nrows) {
            const uint4 wg = *reinterpret_cast<const uint4*>(qg + lr * rb + cg.col * 16);
            const uint4 wu = *reinterpret_cast<const uint4*>(qu + lr * rb + cg.col * 16);
            pg = f16_bits_to_f32(sg[lr * G + cg.col]) * dot_group(wg, xg);
            pu = f16_bits_to_f32(su[lr * G + cg.col]) * dot_group(wu, xg);
          }
          v[r] = pg;
          v[NR_G + r] = pu;
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&S.empty[stage]);
        reduce_scatter<NV_G, SEG_G>(v);
        S.red[warp][lane] = v[0];
        named_bar(1, kCT);
        if (tid < cg.P * NR_G) {
          const int ph = tid / NR_G, i = tid % NR_G;
          const int lr = ph * NR_G + i;
          if (lr < d.nrows) {
            int w0, lg, lu;
            owner_of<NV_G, SEG_G>(ph, i, cg.wpr, w0, lg);
            owner_of<NV_G, SEG_G>(ph, i + NR_G, cg.wpr, w0, lu);
            float g = 0.f, u = 0.f;
            for (int w = 0; w < cg.wpr; ++w) {
              g += S.red[w0 + w][lg];
              u += S.red[w0 + w][lu];
            }
            p.hbuf[(size_t)d.slot * p.I + d.row0 + lr] = silu_mul(g, u);
            __threadfence();
          }
        }
        named_bar(1, kCT);
        if (tid == 0) atom_add_acq_rel(p.ctrl + kCtrlGuDone + d.slot, 1u);
      } else {  // kDown
        XGroup hg;
        {
          float hf[32];
          const float4* hp =
              reinterpret_cast<const float4*>(p.hbuf + (size_t)d.slot * p.I + cd.col * 32);
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            const float4 t4 = __ldcg(hp + i);
            hf[4 * i] = t4.x;
            hf[4 * i + 1] = t4.y;
            hf[4 * i + 2] = t4.z;
            hf[4 * i + 3] = t4.w;
          }
          xgroup_from_floats(hf, hg);
        }
        float v[NR_D];
        const size_t rb = (size_t)p.I / 2;
        const uint16_t* sd = reinterpret_cast<const uint16_t*>(st + (size_t)p.RD * rb);
#pragma unroll
        for (int r = 0; r < NR_D; ++r) {
          const int lr = cd.phase * NR_D + r;
          v[r] = 0.f;
          if (lr < d.nrows) {
            const uint4 wd = *reinterpret_cast<const uint4*>(st + lr * rb + cd.col * 16);
            v[r] = f16_bits_to_f32(sd[lr * GD + cd.col]) * dot_group(wd, hg);
          }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&S.empty[stage]);
        reduce_scatter<NR_D, SEG_D>(v);
        S.red[warp][lane] = v[0];
        named_bar(1, kCT);
        if (tid < cd.P * NR_D) {
          const int ph = tid / NR_D, i = tid % NR_D;
          const int lr = ph * NR_D + i;
          if (lr < d.nrows) {
            int w0, l0;
            owner_of<NR_D, SEG_D>(ph, i, cd.wpr, w0, l0);
            float s = 0.f;
            for (int w = 0; w < cd.wpr; ++w) s += S.red[w0 + w][l0];
            p.ypart[(size_t)d.slot * p.H + d.row0 + lr] = s;
            __threadfence();
          }
        }
        named_bar(1, kCT);
        if (tid == 0) {
          const int rblk = d.row0 / p.RD;
          const uint32_t old = atom_add_acq_rel(p.ctrl + kCtrlRbDone + rblk, 1u);
          S.flag = (old + 1 == (uint32_t)slots) ? 1 : 0;
        }
        named_bar(1, kCT);
        if (S.flag) {
          // last slot of this row block: fixed-order combine
          for (int lr = tid; lr < d.nrows; lr += kCT) {
            const int row = d.row0 + lr;
            float acc = 0.f;
            for (int j = 0; j < p.k; ++j)
              acc = fmaf(__ldcg(p.w_ws + j), __ldcg(p.ypart + (size_t)j * p.H + row), acc);
            if (p.has_shared) acc += __ldcg(p.ypart + (size_t)p.k * p.H + row);
            p.y[row] = acc;
          }
        }
      }
      cons_par ^= 1u << stage;
      stage = (stage + 1 == kStages) ? 0 : stage + 1;
    }
  }

  // -------------------------------------------------------------- teardown
  __syncthreads();
  if (threadIdx.x == 0) {
    __threadfence();
    const uint32_t old = atomicAdd(p.ctrl + kCtrlExit, 1u);
    if (old + 1 == gridDim.x) {
      // last CTA out: reset the counters for the next call (the error word
      // is left for the host to read)
      __threadfence();
      volatile uint32_t* c = p.ctrl;
      c[kCtrlTicket] = 0;
      c[kCtrlRouterDone] = 0;
      c[kCtrlSelReady] = 0;
      c[kCtrlAbort] = 0;
      for (int j = 0; j < slots; ++j) c[kCtrlGuDone + j] = 0;
      for (int b = 0; b < p.nD; ++b) c[kCtrlRbDone + b] = 0;
      c[kCtrlExit] = 0;
      __threadfence();
    }
  }
}

int g_num_sms[64] = {0};

int num_sms() {
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 0 || dev >= 64) return 148;
  if (!g_num_sms[dev]) {
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
      n = 148;
    g_num_sms[dev] = n;
  }
  return g_num_sms[dev];
}

template <int SEG_G, int SEG_D>
cudaError_t launch_t(const DecodeParams& p, cudaStream_t st) {
  static bool configured[64] = {false};
  int dev = 0;
  cudaGetDevice(&dev);
  const size_t smem = decode_smem_bytes();
  if (dev >= 0 && dev < 64 && !configured[dev]) {
    cudaError_t e = cudaFuncSetAttribute(decode_kernel<SEG_G, SEG_D>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    configured[dev] = true;
  }
  decode_kernel<SEG_G, SEG_D><<<num_sms(), kThreads, smem, st>>>(p);
  return cudaGetLastError();
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

// Rows per phase and concurrent phases of the column mapping with kCW warps.
bool phases(int G, int& P) {
  if (G >= 32) {
    const int wpr = G / 32;
    if (kCW % wpr) return false;
    P = kCW / wpr;
  } else {
    P = kCW * (32 / G);
  }
  return true;
}

}  // namespace

size_t decode_smem_bytes() { return (size_t)kStages * kStageBytes + sizeof(Smem); }

bool decode_plan(const moe_config& c, DecodeParams& p) {
  const int G = c.hidden / 32, GD = c.inter / 32;
  int PG, PD;
  if (!phases(G, PG) || !phases(GD, PD)) return false;
  if (c.hidden / 4 > kRouterChunks * kCT) return false;
  if (c.n_experts > 1024) return false;
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
  p.RG = PG * nrg;
  p.RD = PD * nrd;
  p.RR = (int)(kStageBytes / ((uint32_t)c.hidden * 4));
  if (p.RR > kMaxRR) p.RR = kMaxRR;
  if (p.RR < 1) return false;
  if ((size_t)p.RG * (c.hidden / 2 + c.hidden / 16) * 2 > kStageBytes) return false;
  if ((size_t)p.RD * (c.inter / 2 + c.inter / 16) > kStageBytes) return false;
  if ((p.RG * (c.hidden / 16)) % 16 || (p.RD * (c.inter / 16)) % 16) return false;
  p.nR = (p.E + p.RR - 1) / p.RR;
  p.nG = (p.I + p.RG - 1) / p.RG;
  p.nD = (p.H + p.RD - 1) / p.RD;
  if (kCtrlRbDone + p.nD > (int)(kCtrlBytes / 4)) return false;
  if (p.k + p.has_shared > kCtrlRbDone - kCtrlGuDone) return false;
  p.n_items = p.nR + (p.k + p.has_shared) * (p.nG + p.nD);
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
