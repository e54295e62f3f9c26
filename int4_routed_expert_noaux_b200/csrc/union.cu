// union.cu -- the batched (T tokens per call) expert path: every distinct
// selected expert is read from HBM once for all the tokens routed to it
// ("colibri", "Notes": batch-union of the experts of the draft tokens; the
// MTP verify step of "LightLX").
//
//   xq_table        x (bf16) or h (fp32) rows -> int16 groups (XQ words and
//                   factors), once per row, shared by every expert that reads
//                   the row
//   build_lists     per-expert token lists from idx [T][k] (one CTA):
//                   distinct experts in ascending id, the shared expert last
//                   with all T tokens, entries of each expert in token order
//   union_gemm<2>   gate/up of one distinct expert for a block of rows and all
//                   its tokens: h = silu(g) * u, written per (token, slot)
//   union_gemm<1>   down of one distinct expert: partial y per (token, slot)
//   combine         y[t] = sum_j w[t][j] ypart[t][j] + ypart[t][shared],
//                   fixed order, no atomics
//
// The group dot product is the exact integer one of the decode kernel
// (dp2a over int16 inputs); only the order of the fp32 sums differs.
#include <cuda_runtime.h>
#include <algorithm>
#include <stdint.h>

#include "async.cuh"
#include "common.cuh"
#include "device_once.h"
#include "kernels.h"

namespace moe {

namespace {

constexpr int kUnionThreads = 256;
constexpr int kListMaxE = 257;   // routed experts + shared
constexpr int kListMaxIds = 64 * 32;  // T * top_k at most

// ---------------------------------------------------------------------------
template <bool kBf16>
__global__ void __launch_bounds__(256) xq_table_kernel(const void* __restrict__ in, int rows,
                                                       int K, uint8_t* __restrict__ words,
                                                       float* __restrict__ fac) {
  pdl_wait();
  const int G = K >> 5;
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= rows * G) return;
  const int row = i / G, g = i % G;
  float xf[32];
  if (kBf16) {
    const uint4* p4 =
        reinterpret_cast<const uint4*>(static_cast<const uint16_t*>(in) + (size_t)row * K + g * 32);
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const uint4 v = __ldg(p4 + j);
      const uint32_t u[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
      for (int h = 0; h < 4; ++h) {
        xf[8 * j + 2 * h] = bf16_bits_to_f32(u[h] & 0xFFFFu);
        xf[8 * j + 2 * h + 1] = bf16_bits_to_f32(u[h] >> 16);
      }
    }
  } else {
    const float4* p4 =
        reinterpret_cast<const float4*>(static_cast<const float*>(in) + (size_t)row * K + g * 32);
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const float4 v = p4[j];
      xf[4 * j] = v.x;
      xf[4 * j + 1] = v.y;
      xf[4 * j + 2] = v.z;
      xf[4 * j + 3] = v.w;
    }
  }
  XQ q;
  xq_from_floats(xf, q);
  uint4* dst = reinterpret_cast<uint4*>(words + (size_t)i * 64);
  dst[0] = make_uint4(q.ev[0], q.ev[1], q.ev[2], q.ev[3]);
  dst[1] = make_uint4(q.ev[4], q.ev[5], q.ev[6], q.ev[7]);
  dst[2] = make_uint4(q.od[0], q.od[1], q.od[2], q.od[3]);
  dst[3] = make_uint4(q.od[4], q.od[5], q.od[6], q.od[7]);
  fac[i] = q.f;
}

// ---------------------------------------------------------------------------
// The expert lists of the call (layout: ListsView).  Out-of-range ids set
// the error word and are left out; -1 (a slot dropped by top-p) is skipped.
__global__ void __launch_bounds__(256) build_lists_kernel(const int32_t* __restrict__ idx, int T,
                                                          int k, int E, int has_shared,
                                                          uint64_t slot_mask, int tc_min,
                                                          int* __restrict__ lists,
                                                          uint32_t* __restrict__ err) {
  pdl_wait();
  __shared__ int cnt[kListMaxE];
  __shared__ int base[kListMaxE];
  __shared__ int sid[kListMaxIds];
  const int slots = k + has_shared;  // the layout of h and ypart rows: (token, slot)
  const int n_list = T * slots;
  const ListsView L = lists_view(lists, E, n_list);
  // the slots this call computes: routed slot j when bit j of slot_mask is
  // set, the shared expert when bit k is (the others keep their rows)
  const bool shared_on = has_shared && ((slot_mask >> k) & 1ull);
  int* u_expert = const_cast<int*>(L.u_expert);
  int* u_off = const_cast<int*>(L.u_off);
  int* list_tok = const_cast<int*>(L.list_tok);
  int* list_pos = const_cast<int*>(L.list_pos);
  int* cc_u = const_cast<int*>(L.cc_u);
  int* tc_u = const_cast<int*>(L.tc_u);
  int* tc_roff = const_cast<int*>(L.tc_roff);
  // the ids into shared memory; warp 0 counts them 32 at a time: the lanes
  // holding one id find each other (match.any) and the lowest adds their
  // number (no atomics, which correlated tokens would serialise on a few ids)
  for (int i = threadIdx.x; i < T * k; i += blockDim.x) {
    const int e = idx[i];
    sid[i] = ((slot_mask >> (i % k)) & 1ull) ? e : -1;
    if ((e < 0 || e >= E) && e != -1) atomicCAS(err, 0u, (uint32_t)kErrBadExpertId);
  }
  for (int e = threadIdx.x; e <= E; e += blockDim.x) cnt[e] = 0;
  __syncthreads();
  if (threadIdx.x < 32) {
    const int lane = threadIdx.x;
    for (int i0 = 0; i0 < T * k; i0 += 32) {
      const int e = i0 + lane < T * k ? sid[i0 + lane] : -1;
      const uint32_t peers = __match_any_sync(0xffffffffu, e);
      if (e >= 0 && e < E && lane == __ffs(peers) - 1) cnt[e] += __popc(peers);
      __syncwarp();
    }
  }
  __syncthreads();
  if (threadIdx.x == 0 && shared_on) cnt[E] = T;
  __syncthreads();
  // exclusive scans of (expert used, tensor-core expert, entries, packed
  // rows) over experts 0..E, ascending: thread i owns experts 2i and 2i + 1
  // (E + 1 <= 512); tc_min 0: no tensor-core experts
  {
    __shared__ int wu[8], wt[8], ws[8], wp[8];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int e0 = 2 * threadIdx.x, e1 = e0 + 1;
    const int c0 = e0 <= E ? cnt[e0] : 0, c1 = e1 <= E ? cnt[e1] : 0;
    const bool t0 = tc_min > 0 && c0 >= tc_min && c0 <= kTcMaxTok;
    const bool t1 = tc_min > 0 && c1 >= tc_min && c1 <= kTcMaxTok;
    const int p0 = t0 ? (c0 + 15) & ~15 : 0, p1 = t1 ? (c1 + 15) & ~15 : 0;
    const int nu = (c0 > 0) + (c1 > 0), nt = (int)t0 + (int)t1, ns = c0 + c1, np = p0 + p1;
    int iu = nu, it = nt, is = ns, ip = np;  // inclusive warp scans
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int a = __shfl_up_sync(0xffffffffu, iu, o), b = __shfl_up_sync(0xffffffffu, it, o),
                c = __shfl_up_sync(0xffffffffu, is, o), d = __shfl_up_sync(0xffffffffu, ip, o);
      if (lane >= o) {
        iu += a;
        it += b;
        is += c;
        ip += d;
      }
    }
    if (lane == 31) {
      wu[warp] = iu;
      wt[warp] = it;
      ws[warp] = is;
      wp[warp] = ip;
    }
    __syncthreads();
    int bu = 0, bt = 0, bs = 0, bp = 0;
    for (int w = 0; w < warp; ++w) {
      bu += wu[w];
      bt += wt[w];
      bs += ws[w];
      bp += wp[w];
    }
    // exclusive prefixes
    int uu = bu + iu - nu, ut = bt + it - nt, off = bs + is - ns, poff = bp + ip - np;
    if (c0 > 0) {
      u_expert[uu] = e0;
      u_off[uu] = off;
      base[e0] = off;
      if (t0) {
        tc_roff[ut] = poff;
        tc_u[ut++] = uu;
        poff += p0;
      } else {
        cc_u[uu - ut] = uu;
      }
      ++uu;
      off += c0;
    }
    if (c1 > 0) {
      u_expert[uu] = e1;
      u_off[uu] = off;
      base[e1] = off;
      if (t1) {
        tc_roff[ut] = poff;
        tc_u[ut] = uu;
      } else {
        cc_u[uu - ut] = uu;
      }
    }
    if (threadIdx.x == blockDim.x - 1) {
      const int U = bu + iu, n_tc = bt + it, total = bs + is;
      u_off[U] = total;
      lists[0] = U;
      int* counts = const_cast<int*>(L.counts);
      counts[0] = U - n_tc;
      counts[1] = n_tc;
      tc_roff[n_tc] = bp + ip;
    }
  }
  __syncthreads();
  // the entries in (token, slot) order, placed by warp 0 32 at a time: an
  // entry's place is its expert's next free one plus its rank among the
  // lanes holding the same id
  if (threadIdx.x < 32) {
    const int lane = threadIdx.x;
    for (int i0 = 0; i0 < T * k; i0 += 32) {
      const int i = i0 + lane;
      const int e = i < T * k ? sid[i] : -1;
      const uint32_t peers = __match_any_sync(0xffffffffu, e);
      if (e >= 0 && e < E) {
        const int pos = base[e] + __popc(peers & ((1u << lane) - 1u));
        const int t = i / k, j = i % k;
        list_tok[pos] = t;
        list_pos[pos] = t * slots + j;
      }
      __syncwarp();
      if (e >= 0 && e < E && lane == __ffs(peers) - 1) base[e] += __popc(peers);
      __syncwarp();
    }
  }
  if (shared_on) {
    for (int t = threadIdx.x; t < T; t += blockDim.x) {
      list_tok[base[E] + t] = t;
      list_pos[base[E] + t] = t * slots + k;
    }
  }
}

// ---------------------------------------------------------------------------
// One distinct expert (blockIdx.y) times a block of rows (blockIdx.x) for all
// its tokens, up to kTok tokens per pass.  Thread (m, q) = (warp * 8 +
// lane % 8, lane / 8) owns matrix row m of the block (MATS == 2: rows 0..31
// gate, 32..63 up; MATS == 1: 64 down rows) and groups 4i + q of each k step.
// A k step (kKB groups) of weights, scales and the tokens' int16 inputs is
// brought into shared memory by cp.async, kNS - 1 steps ahead of the step
// being computed, so DRAM latency overlaps the dot products; every weight
// chunk is read from HBM once per pass and used for every token of the pass.
struct UnionArgs {
  const ExpertPtrs* table;
  const int* lists;
  int E, n_list;
  const uint8_t* xq_words;  // [input rows][G] 64-byte XQ words
  const float* xq_fac;      // [input rows][G]
  int G;                    // 32-input groups of a matrix row
  int R;                    // rows of one matrix
  int in_is_pos;            // input row of an entry: list_pos (1) or list_tok (0)
  float* out;               // [T slots][R]
};

constexpr int kTok = 8;     // tokens per pass
constexpr int kKB = 16;     // groups per k step
constexpr int kNS = 3;      // pipeline stages
constexpr int kRowPad = kKB + 1;  // chunks per staged row: 8 consecutive rows hit 8 bank quads

struct UStage {
  uint4 w[64][kRowPad];     // weight chunks of the block's 64 matrix rows
  uint16_t s[64][kKB];      // their fp16 scales
  uint4 x[kTok][kKB][4];    // XQ words of the pass's tokens
  float f[kTok][kKB];       // XQ factors
};

__device__ __forceinline__ void cp_async16(void* dst, const void* src, bool valid) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(smem_addr(dst)), "l"(src),
               "r"(valid ? 16 : 0)
               : "memory");
}

__device__ __forceinline__ void cp_async4(void* dst, const void* src, bool valid) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4, %2;" ::"r"(smem_addr(dst)), "l"(src),
               "r"(valid ? 4 : 0)
               : "memory");
}

__device__ __forceinline__ void cp_async_commit() {
  asm volatile("cp.async.commit_group;" ::: "memory");
}

template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

size_t union_smem_bytes(int mats) {
  return (size_t)kNS * sizeof(UStage) + (size_t)mats * (64 / mats) * (kTok + 1) * sizeof(float);
}

template <int MATS>
__global__ void __launch_bounds__(kUnionThreads) union_gemm_kernel(const UnionArgs a) {
  pdl_wait();
  constexpr int RBM = 64 / MATS;  // rows of one matrix per CTA
  extern __shared__ __align__(16) uint8_t usmem[];
  UStage* st = reinterpret_cast<UStage*>(usmem);
  float(*sO)[RBM][kTok + 1] = reinterpret_cast<float(*)[RBM][kTok + 1]>(usmem + kNS * sizeof(UStage));
  const ListsView L = lists_view(a.lists, a.E, a.n_list);
  const int* list_pos = L.list_pos;
  const int* in_idx = a.in_is_pos ? list_pos : L.list_tok;
  const int nb = (a.R + RBM - 1) / RBM;
  const int items = L.counts[0] * nb;
  const int tid = threadIdx.x, lane = tid & 31;
  // persistent: work item = (expert of the CUDA-core path, block of rows),
  // the row blocks of an expert adjacent; the loop bounds are uniform per CTA
  for (int item = blockIdx.x; item < items; item += gridDim.x) {
    const int u = L.cc_u[item / nb];
    const int e = L.u_expert[u];
    const int base = L.u_off[u], n = L.u_off[u + 1] - base;
    const int row0 = (item % nb) * RBM;
    const int m = (tid >> 5) * 8 + (lane & 7), q = lane >> 3;
    const int mat = m / RBM, r = m % RBM;
    const ExpertPtrs ep = a.table[e];
    const int nk = (a.G + kKB - 1) / kKB;

    static_assert(64 * kKB == 4 * kUnionThreads && 64 * kKB / 2 == 2 * kUnionThreads &&
                      kTok * kKB * 4 == 2 * kUnionThreads && kTok * kKB <= kUnionThreads,
                  "the copy assignment below");
    // This thread's copies of every k step, as source pointers advanced by the
    // step: weight chunks (4), scale pairs (2), token input chunks (2) and one
    // token factor.  Row sources are fixed for the CTA, token sources per pass.
    const int gw_ = tid & (kKB - 1), gs_ = 2 * (tid & (kKB / 2 - 1));
    const uint8_t* wsrc[4];
    bool wok[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int mm = (tid >> 4) + 16 * j, rr = row0 + mm % RBM;
      const uint8_t* codes = (MATS == 2) ? ((mm / RBM) == 0 ? ep.q_gate : ep.q_up) : ep.q_down;
      wok[j] = rr < a.R;
      wsrc[j] = codes + ((size_t)(wok[j] ? rr : row0) * a.G + min(gw_, a.G - 1)) * 16;
    }
    const uint16_t* ssrc[2];
    bool sok[2];
#pragma unroll
    for (int j = 0; j < 2; ++j) {
      const int mm = (tid >> 3) + 32 * j, rr = row0 + mm % RBM;
      const uint16_t* sc = (MATS == 2) ? ((mm / RBM) == 0 ? ep.s_gate : ep.s_up) : ep.s_down;
      sok[j] = rr < a.R;
      ssrc[j] = sc + (size_t)(sok[j] ? rr : row0) * a.G + min(gs_, a.G - 2);
    }
    const int xg_ = (tid >> 2) & (kKB - 1), xw_ = tid & 3;
    const uint8_t* xsrc[2];
    bool xok[2];
    const float* fsrc = a.xq_fac;
    bool fok = false;

    // a copy that is not needed (row or token past the end, group past the
    // step) reads nothing (source size 0) from its in-range base pointer
    auto issue = [&](int sb, int ks) {
      UStage& S = st[sb];
      const int kb = ks * kKB, kbn = min(kKB, a.G - kb);
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const bool ok = wok[j] && gw_ < kbn;
        cp_async16(&S.w[(tid >> 4) + 16 * j][gw_], ok ? wsrc[j] + (size_t)kb * 16 : wsrc[j], ok);
      }
#pragma unroll
      for (int j = 0; j < 2; ++j) {
        const bool ok = sok[j] && gs_ < kbn;
        cp_async4(&S.s[(tid >> 3) + 32 * j][gs_], ok ? ssrc[j] + kb : ssrc[j], ok);
      }
#pragma unroll
      for (int j = 0; j < 2; ++j) {
        const bool ok = xok[j] && xg_ < kbn;
        cp_async16(&S.x[(tid >> 6) + 4 * j][xg_][xw_], ok ? xsrc[j] + (size_t)kb * 64 : xsrc[j], ok);
      }
      if (tid < kTok * kKB) {
        const bool ok = fok && (tid % kKB) < kbn;
        cp_async4(&S.f[tid / kKB][tid % kKB], ok ? fsrc + kb : fsrc, ok);
      }
    };

    for (int tc = 0; tc < n; tc += kTok) {
      const int nt = min(kTok, n - tc);
      // this pass's token sources
#pragma unroll
      for (int j = 0; j < 2; ++j) {
        const int ti = (tid >> 6) + 4 * j;
        xok[j] = ti < nt;
        const int rin = in_idx[base + tc + (xok[j] ? ti : 0)];
        xsrc[j] = a.xq_words + ((size_t)rin * a.G + min(xg_, a.G - 1)) * 64 + xw_ * 16;
      }
      if (tid < kTok * kKB) {
        const int ti = tid / kKB;
        fok = ti < nt;
        fsrc = a.xq_fac + (size_t)in_idx[base + tc + (fok ? ti : 0)] * a.G + min(tid % kKB, a.G - 1);
      }
      float acc[kTok];
#pragma unroll
      for (int ti = 0; ti < kTok; ++ti) acc[ti] = 0.f;
#pragma unroll
      for (int s0 = 0; s0 < kNS - 1; ++s0) {
        if (s0 < nk) issue(s0, s0);
        cp_async_commit();
      }
      for (int ks = 0; ks < nk; ++ks) {
        cp_async_wait<kNS - 2>();  // step ks has landed (this thread's copies)
        __syncthreads();           // ... everyone's; step ks - 1 is no longer read
        if (ks + kNS - 1 < nk) issue((ks + kNS - 1) % kNS, ks + kNS - 1);
        cp_async_commit();
        const UStage& S = st[ks % kNS];
        const int kbn = min(kKB, a.G - ks * kKB);
#pragma unroll
        for (int i = 0; i < kKB / 4; ++i) {
          const int g = 4 * i + q;
          if (g < kbn) {
            uint32_t even[4], odd[4];
            split_chunk(S.w[m][g], even, odd);  // once, for every token
            const float sc = f16_bits_to_f32(S.s[m][g]);
#pragma unroll
            for (int ti = 0; ti < kTok; ++ti) {
              if (ti < nt) {
                XQ xg;
                const uint4 a0 = S.x[ti][g][0], a1 = S.x[ti][g][1], a2 = S.x[ti][g][2],
                            a3 = S.x[ti][g][3];
                xg.ev[0] = a0.x; xg.ev[1] = a0.y; xg.ev[2] = a0.z; xg.ev[3] = a0.w;
                xg.ev[4] = a1.x; xg.ev[5] = a1.y; xg.ev[6] = a1.z; xg.ev[7] = a1.w;
                xg.od[0] = a2.x; xg.od[1] = a2.y; xg.od[2] = a2.z; xg.od[3] = a2.w;
                xg.od[4] = a3.x; xg.od[5] = a3.y; xg.od[6] = a3.z; xg.od[7] = a3.w;
                xg.f = S.f[ti][g];
                acc[ti] += (float)dotq_group_split(even, odd, xg) * (sc * xg.f);
              }
            }
          }
        }
      }
      cp_async_wait<0>();
      // the four column quarters of a row are lanes l, l + 8, l + 16, l + 24
#pragma unroll
      for (int ti = 0; ti < kTok; ++ti) {
        acc[ti] += __shfl_xor_sync(0xffffffffu, acc[ti], 8);
        acc[ti] += __shfl_xor_sync(0xffffffffu, acc[ti], 16);
      }
      if (q == 0) {
#pragma unroll
        for (int ti = 0; ti < kTok; ++ti) sO[mat][r][ti] = acc[ti];
      }
      __syncthreads();
      for (int i = tid; i < RBM * nt; i += kUnionThreads) {
        const int rr = i % RBM, ti = i / RBM;
        if (row0 + rr < a.R) {
          const float v = (MATS == 2) ? silu_mul(sO[0][rr][ti], sO[1][rr][ti]) : sO[0][rr][ti];
          a.out[(size_t)list_pos[base + tc + ti] * a.R + row0 + rr] = v;
        }
      }
      __syncthreads();  // sO and the stages are rewritten by the next pass
    }
  }
}

// y[t][row] = sum_j w[t][j] * ypart[t][j][row] (+ the shared expert's row),
// in slot order; terms of out-of-range ids are left out.
__global__ void __launch_bounds__(256) union_combine_kernel(
    const int32_t* __restrict__ idx, const float* __restrict__ w, const float* __restrict__ ypart,
    int T, int H, int k, int E, int has_shared, float* __restrict__ y) {
  pdl_wait();
  const int t = blockIdx.y;
  const int row = blockIdx.x * blockDim.x + threadIdx.x;
  if (row >= H) return;
  const int slots = k + has_shared;
  float acc = 0.f;
  for (int j = 0; j < k; ++j) {
    const int e = idx[t * k + j];
    if (e >= 0 && e < E)
      acc = fmaf(w[t * k + j], ypart[((size_t)t * slots + j) * H + row], acc);
  }
  if (has_shared) acc += ypart[((size_t)t * slots + k) * H + row];
  y[(size_t)t * H + row] = acc;
}

}  // namespace

size_t union_lists_ints(int T, int k, int E, int has_shared) {
  return 1 + (size_t)(E + 1) + (E + 2) + 2 * (size_t)T * (k + has_shared) + 2 +
         2 * (size_t)(E + 1) + (E + 2);
}

cudaError_t launch_union_ffn(const ExpertPtrs* table, const int32_t* idx, const float* w,
                             const uint16_t* x, int T, int H, int I, int E, int k, int has_shared,
                             uint8_t* xq_words, float* xq_fac, uint8_t* hq_words, float* hq_fac,
                             int* lists, float* hbuf, float* ypart, float* y, uint32_t* err,
                             uint8_t* tc_bpack, int* tc_rowexp, uint8_t* tc_maps,
                             cudaStream_t st, uint64_t slot_mask, bool combine) {
  if (E + 1 > kListMaxE || T * k > kListMaxIds) return cudaErrorInvalidValue;
  const int tc_min = tc_min_tokens();
  const bool tc = tc_bpack && tc_maps && T >= tc_min && tc_shape_ok(H, I);
  const int slots = k + has_shared;
  const int G = H / 32, GD = I / 32;
  const int n_list = T * slots;
  const int umax = (E < T * k ? E : T * k) + has_shared;
  launch_pdl(xq_table_kernel<true>, dim3((T * G + 255) / 256), dim3(256), 0, st, x, T, H, xq_words,
             xq_fac);
  launch_pdl(build_lists_kernel, dim3(1), dim3(256), 0, st, idx, T, k, E, has_shared, slot_mask,
             tc ? tc_min : 0, lists, err);
  UnionArgs a;
  a.table = table;
  a.lists = lists;
  a.E = E;
  a.n_list = n_list;
  a.xq_words = xq_words;
  a.xq_fac = xq_fac;
  a.G = G;
  a.R = I;
  a.in_is_pos = 0;
  a.out = hbuf;
  // blocks per SM of union_gemm<2> (low half) and union_gemm<1> (high half)
  static DeviceOnce<uint32_t> configured;
  int dev = 0;
  cudaError_t ce = cudaGetDevice(&dev);
  if (ce != cudaSuccess) return ce;
  uint32_t occ = 0;
  ce = configured.get(dev, &occ, [](uint32_t* v) {
    cudaError_t r = cudaFuncSetAttribute(union_gemm_kernel<2>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)union_smem_bytes(2));
    if (r == cudaSuccess)
      r = cudaFuncSetAttribute(union_gemm_kernel<1>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               (int)union_smem_bytes(1));
    int o2 = 0, o1 = 0;
    if (r == cudaSuccess)
      r = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&o2, union_gemm_kernel<2>, kUnionThreads,
                                                        union_smem_bytes(2));
    if (r == cudaSuccess)
      r = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&o1, union_gemm_kernel<1>, kUnionThreads,
                                                        union_smem_bytes(1));
    if (r == cudaSuccess && (o2 < 1 || o1 < 1)) r = cudaErrorInvalidConfiguration;
    *v = (uint32_t)o2 | ((uint32_t)o1 << 16);
    return r;
  });
  if (ce != cudaSuccess) return ce;
  // persistent grids: at most one wave, and no more CTAs than work items
  const int sms = num_sms();
  const int nb2 = (I + 31) / 32, nb1 = (H + 63) / 64;
  const int grid2 = std::min((int)(occ & 0xFFFFu) * sms, umax * nb2);
  const int grid1 = std::min((int)(occ >> 16) * sms, umax * nb1);
  launch_pdl(union_gemm_kernel<2>, dim3(grid2), dim3(kUnionThreads), union_smem_bytes(2), st, a);
  if (tc) {
    const cudaError_t e = launch_tc_ffn_step(2, table, lists, E, n_list, T, k, has_shared, x, H,
                                             I, T, tc_rowexp, tc_bpack, tc_maps, hbuf, err, st);
    if (e != cudaSuccess) return e;
  }
  launch_pdl(xq_table_kernel<false>, dim3((n_list * GD + 255) / 256), dim3(256), 0, st, hbuf,
             n_list, I, hq_words, hq_fac);
  a.xq_words = hq_words;
  a.xq_fac = hq_fac;
  a.G = GD;
  a.R = H;
  a.in_is_pos = 1;
  a.out = ypart;
  launch_pdl(union_gemm_kernel<1>, dim3(grid1), dim3(kUnionThreads), union_smem_bytes(1), st, a);
  if (tc) {
    const cudaError_t e = launch_tc_ffn_step(1, table, lists, E, n_list, T, k, has_shared, hbuf,
                                             I, H, n_list, tc_rowexp, tc_bpack, tc_maps, ypart,
                                             err, st);
    if (e != cudaSuccess) return e;
  }
  if (combine)
    launch_pdl(union_combine_kernel, dim3((H + 255) / 256, T), dim3(256), 0, st, idx, w, ypart, T,
               H, k, E, has_shared, y);
  return cudaGetLastError();
}

}  // namespace moe
