// tc_union.cu -- the batched (verify) expert path on the 5th-generation
// tensor cores, for every distinct expert that 16 to 64 of the call's
// tokens route to: each expert's weights stream from HBM once for all its
// tokens (colibri summary, "Principales fonctionnalites implementees":
// batch-union of the experts of the draft tokens; "LightLX", "How it
// works": the MTP verify step), and the products run as tcgen05 MMAs.
//
// Per (expert, tile of 128 weight rows) one CTA.  Two converter warpgroups
// split the 32-input scale groups of the K range in halves, one thread per
// weight row (= tensor-memory lane):
//   - the thread's row of int4 codes and fp16 scales comes into shared
//     memory by cp.async, kWS stages of two groups ahead, and only that
//     thread reads it back;
//   - it forms the group's 32 weights code * scale as an fp16 pair hi + lo
//     (hi = fp16(code * scale) rounded, lo = code * scale - hi exactly: an
//     fma of fp16 values whose exact result has at most 4 significant bits),
//     so hi + lo is the weight to about 2^-22, and stores the 32 hi and 32
//     lo halves to a slot of a ring of A operands in tensor memory;
//   - a producer thread brings each group's packed token inputs (B operand,
//     fp16, K-major canonical layout; the down projection's h as fp16 hi and
//     lo tiles) into a ring of shared-memory slots by bulk async copies;
//   - an issuer thread runs per group the M=128 K=16 fp16 MMAs A_hi B and
//     A_lo B (and A_hi B_lo for the down projection) for both K halves into
//     its warpgroup's fp32 accumulator in tensor memory, which holds the
//     whole K range: no per-group epilogue; one commit per group frees the
//     group's ring slot.
// At the end each warpgroup's accumulator is read back (tcgen05.ld) and the
// two are added in a fixed order through shared memory; gate/up tiles hold
// 64 gate and 64 up rows of the same indices, so h = silu(g) * u is formed
// in the tile.
//
// Within a group the MMA's K order is a fixed permutation of the 32 inputs
// (the order the nibble pairs come out of a word); the packed inputs use the
// same permutation (tc_perm).
#include <cuda_runtime.h>
#include <algorithm>
#include <stdint.h>

#include "async.cuh"
#include "common.cuh"
#include "device_once.h"
#include "kernels.h"

namespace moe {

namespace {

// Per-step timeline of CTA 0's first work item in a -DMOE_TRACE profiling
// build (row 7: the end of each of CTA 0's items).
#ifdef MOE_TRACE
__device__ uint64_t g_tc_trace[8][256];
#define TC_TRACE(kind, st)                                                          \
  do {                                                                              \
    if (blockIdx.x == 0 && it == 0 && (st) < 256)                                   \
      g_tc_trace[kind][st] = (uint64_t)clock64();                                   \
  } while (0)
#define TC_TRACE_ITEM()                                                             \
  do {                                                                              \
    if (blockIdx.x == 0 && it < 256) g_tc_trace[7][it] = (uint64_t)clock64();       \
  } while (0)
#else
#define TC_TRACE(kind, st) ((void)0)
#define TC_TRACE_ITEM() ((void)0)
#endif

constexpr int kWG = 2;                    // converter warpgroups (K halves)
constexpr int kConvThreads = kWG * 128;
constexpr int kTcThreads = kConvThreads + 32;  // + one warp: B producer (lane 0), issuer (lane 1)
constexpr int kWS = 8;                    // code stages per warpgroup (2 groups each)
constexpr int kR = 12;                    // ring slots (A in tensor memory, B in shared memory)
constexpr int kNmax = 64;                 // most tokens per expert on this path
constexpr int kColD = 0;                  // tensor memory: D of warpgroup w at w * kNmax
constexpr int kColA = kWG * kNmax;        // then kR slots of 32 columns (hi 16, lo 16)
constexpr uint64_t kTcWaitNs = 1000000000ull;
static_assert(kColA + kR * 32 <= 512, "tensor memory columns");

struct TcSmem {
  uint4 w[kWG][kWS][128][2];              // codes: [wg][stage][row][group of the pair]
  uint32_t sc[kWG][kWS][128];             // the two groups' fp16 scales
  uint8_t b[kR][kNmax * 64 * 2];          // B of one group (down: hi then lo)
  uint64_t a_full[kR];                    // converters wrote the slot's A (4 warps)
  uint64_t b_full[kR];                    // the slot's B landed
  uint64_t slot_free[kR];                 // the MMAs reading the slot finished
  uint64_t fin;                           // all MMAs finished
  uint32_t tmem_base;
  int abort_flag;
};
static_assert(sizeof(uint4) * kWG * kWS * 128 * 2 >= sizeof(float) * kWG * 128 * kNmax,
              "the partial sums reuse the code stages");

// MMA-K index k of a group holds input tc_perm(k): the converter makes the
// pair of TMEM column 4i + j from nibbles j and j + 4 of word i.
__device__ __forceinline__ int tc_perm(int k) {
  const int i = k >> 3, r = k & 7;
  return 8 * i + (r >> 1) + 4 * (r & 1);
}

__device__ __forceinline__ uint64_t umma_desc(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
  // canonical K-major layout without swizzle: LBO = byte distance of core
  // matrices (8 rows x 16 bytes) along K, SBO = along M/N; version 1
  return (uint64_t)((saddr & 0x3FFFF) >> 4) | ((uint64_t)((lbo & 0x3FFFF) >> 4) << 16) |
         ((uint64_t)((sbo & 0x3FFFF) >> 4) << 32) | ((uint64_t)1 << 46);
}

// kind::f16 instruction descriptor: fp32 D, fp16 A and B, both K-major.
__device__ __forceinline__ uint32_t umma_idesc_f16(int M, int N) {
  return (1u << 4) | ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}

__device__ __forceinline__ void tc_mma(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc,
                                       uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{ .reg .pred p; setp.ne.b32 p, %4, 0;\n"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p; }" ::"r"(d_tmem),
      "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

__device__ __forceinline__ void tc_commit(uint64_t* bar) {
  asm volatile(
      "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
          smem_addr(bar))
      : "memory");
}

__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t (&v)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,"
      "%14,%15,%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};" ::"r"(taddr),
      "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7]),
      "r"(v[8]), "r"(v[9]), "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]), "r"(v[14]), "r"(v[15]),
      "r"(v[16]), "r"(v[17]), "r"(v[18]), "r"(v[19]), "r"(v[20]), "r"(v[21]), "r"(v[22]),
      "r"(v[23]), "r"(v[24]), "r"(v[25]), "r"(v[26]), "r"(v[27]), "r"(v[28]), "r"(v[29]),
      "r"(v[30]), "r"(v[31])
      : "memory");
}

__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t (&v)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,"
      "%15}, [%16];"
      : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]),
        "=r"(v[7]), "=r"(v[8]), "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]), "=r"(v[13]),
        "=r"(v[14]), "=r"(v[15])
      : "r"(taddr)
      : "memory");
}

__device__ __forceinline__ void cp_async16(void* dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_addr(dst)), "l"(src)
               : "memory");
}
__device__ __forceinline__ void cp_async4(void* dst, const void* src) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(smem_addr(dst)), "l"(src)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() {
  asm volatile("cp.async.commit_group;" ::: "memory");
}
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

// The 32 weights of one 16-byte chunk times its fp16 scale s2 (both halves)
// as fp16 pairs: hi[4i + j] holds the weights of nibbles j and j + 4 of
// word i rounded to fp16, lo[4i + j] the exact remainders.
__device__ __forceinline__ void weights_hi_lo(const uint4 w, uint32_t s2, uint32_t (&hl)[32]) {
  const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      // fp16(1024 + (n ^ 8)) in both halves, minus 1032: the exact code
      const uint32_t v = ((ws[i] >> (4 * j)) & 0x000F000Fu) ^ 0x64086408u;
      uint32_t q, hi, lo;
      asm("{ .reg .b32 c; mov.b32 c, 0x64086408; sub.rn.f16x2 %0, %1, c; }" : "=r"(q) : "r"(v));
      asm("mul.rn.f16x2 %0, %1, %2;" : "=r"(hi) : "r"(q), "r"(s2));
      asm("{ .reg .b32 n; xor.b32 n, %3, 0x80008000; fma.rn.f16x2 %0, %1, %2, n; }"
          : "=r"(lo)
          : "r"(q), "r"(s2), "r"(hi));
      hl[4 * i + j] = hi;
      hl[16 + 4 * i + j] = lo;
    }
  }
}

static_assert(kTcMaxTok == kNmax, "the token bound of the path");

struct TcArgs {
  const ExpertPtrs* table;
  const int* lists;
  int E, n_list;
  int K, G;          // inputs of a weight row and its 32-input groups
  int R;             // rows of one weight matrix
  int mats;          // 2: gate/up tiles (64 + 64 rows), 1: down tiles (128 rows)
  const uint8_t* bpack;  // packed B per path expert: [rank][G][B bytes of a group at kNmax]
  const int* row_exp;    // power-of-two scale of each input row (tc_rowscale_kernel)
  float* out;        // [T slots][R] (h for gate/up, partial y for down)
  uint32_t* err;     // kErrTimeout when a wait ran out
};

__host__ __device__ __forceinline__ size_t tc_group_bytes(int mats) {
  return (size_t)kNmax * 64 * (mats == 2 ? 1 : 2);
}

__global__ void __launch_bounds__(kTcThreads, 1) tc_gemm_kernel(const TcArgs a) {
  extern __shared__ __align__(1024) uint8_t tsmem[];
  TcSmem& S = *reinterpret_cast<TcSmem*>(tsmem);
  const ListsView L = lists_view(a.lists, a.E, a.n_list);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int tile_rows = a.mats == 2 ? 64 : 128;
  const int tiles = a.R / tile_rows;
  const int items = L.counts[1] * tiles;
  if ((int)blockIdx.x >= items) return;  // uniform per CTA, before any barrier
  const int ng = a.G / kWG;              // groups per warpgroup (G % 4 == 0)
  const int steps = kWG * ng;            // step s of an item: warpgroup s % kWG, its group s / kWG
  const size_t gbytes = tc_group_bytes(a.mats);
  volatile int* abort_flag = &S.abort_flag;

  if (tid == 0) {
    for (int i = 0; i < kR; ++i) {
      mbar_init(&S.a_full[i], 4);
      mbar_init(&S.b_full[i], 1);
      mbar_init(&S.slot_free[i], 1);
    }
    mbar_init(&S.fin, 1);
    S.abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], 512;" ::"r"(
        smem_addr(&S.tmem_base)));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = S.tmem_base;

  // Persistent: work item = (expert of the path, tile of weight rows), the
  // tiles of an expert adjacent.  The ring of A/B slots runs on across
  // items (ring step gs + st); an item's accumulators are read back before
  // the next item's first MMAs overwrite them.
  int gs = 0, it = 0;
  for (int item = blockIdx.x; item < items; item += gridDim.x, gs += steps, ++it) {
    const int rank = item / tiles;
    const int u = L.tc_u[rank];
    const int e = L.u_expert[u];
    const int base = L.u_off[u], n = L.u_off[u + 1] - base;
    const int N = (n + 15) & ~15;
    const int r0 = (item % tiles) * tile_rows;
    if (warp == kConvThreads / 32) {
      if (lane == 0) {
        // -------------------------------------------------- B producer
        const uint8_t* bsrc = a.bpack + ((size_t)rank * a.G) * gbytes;
        const uint32_t bcopy = (uint32_t)N * 64 * (a.mats == 2 ? 1 : 2);
        const uint64_t keep = l2_policy_evict_last();
        for (int st = 0; st < steps && !*abort_flag; ++st) {
          const int q = gs + st, slot = q % kR, use = q / kR;
          if (use > 0 && !mbar_wait(&S.slot_free[slot], (uint32_t)((use - 1) & 1), kTcWaitNs)) {
            *abort_flag = 1;
            break;
          }
          const int g = (st % kWG) * ng + st / kWG;
          TC_TRACE(0, st);
          mbar_arrive_expect_tx(&S.b_full[slot], bcopy);
          bulk_g2s(S.b[slot], bsrc + (size_t)g * gbytes, bcopy, &S.b_full[slot], keep);
        }
      } else if (lane == 1) {
        // -------------------------------------------------- MMA issuer
        const uint32_t idesc = umma_idesc_f16(128, N);
        for (int st = 0; st < steps; ++st) {
          const int q = gs + st, slot = q % kR, use = q / kR;
          if (*abort_flag || !mbar_wait(&S.a_full[slot], (uint32_t)(use & 1), kTcWaitNs)) {
            *abort_flag = 1;
            break;
          }
          TC_TRACE(1, st);
          if (!mbar_wait(&S.b_full[slot], (uint32_t)(use & 1), kTcWaitNs)) {
            *abort_flag = 1;
            break;
          }
          TC_TRACE(2, st);
          tc_fence_after();
          const int w = st % kWG, i = st / kWG;
          const uint32_t d = tmem + (uint32_t)(kColD + w * kNmax);
          const uint32_t ahi = tmem + (uint32_t)(kColA + slot * 32), alo = ahi + 16;
          const uint32_t bhi = smem_addr(S.b[slot]), blo = bhi + (uint32_t)N * 64;
#pragma unroll
          for (int kk = 0; kk < 2; ++kk) {
            const uint64_t dh = umma_desc(bhi + kk * 256, 128, 512);
            tc_mma(d, ahi + kk * 8, dh, idesc, (i > 0 || kk > 0) ? 1u : 0u);
            tc_mma(d, alo + kk * 8, dh, idesc, 1u);
            if (a.mats == 1)
              tc_mma(d, ahi + kk * 8, umma_desc(blo + kk * 256, 128, 512), idesc, 1u);
          }
          tc_commit(&S.slot_free[slot]);
          TC_TRACE(3, st);
        }
        // every MMA of the item has finished when this arrives
        tc_commit(&S.fin);
      }
    } else {
      // ---------------------------------------------------- converters
      const int wg = warp >> 2, row = (warp & 3) * 32 + lane;  // row = tensor-memory lane
      const uint32_t lane_base = (uint32_t)((warp & 3) * 32) << 16;
      const ExpertPtrs ep = a.table[e];
      const int mrow = r0 + (a.mats == 2 ? (row & 63) : row);
      const uint8_t* codes = (a.mats == 2 ? (row < 64 ? ep.q_gate : ep.q_up) : ep.q_down) +
                             (size_t)mrow * (a.K / 2);
      const uint16_t* scales = (a.mats == 2 ? (row < 64 ? ep.s_gate : ep.s_up) : ep.s_down) +
                               (size_t)mrow * a.G;
      const int g0 = wg * ng;  // this warpgroup's groups [g0, g0 + ng), g0 even
      auto issue_stage = [&](int j) {
        const int gl = 2 * j;
        if (gl < ng) {
          const int s = j % kWS;
          cp_async16(&S.w[wg][s][row][0], codes + (size_t)(g0 + gl) * 16);
          cp_async16(&S.w[wg][s][row][1], codes + (size_t)(g0 + gl + 1) * 16);
          cp_async4(&S.sc[wg][s][row], scales + g0 + gl);  // one aligned word: two scales
        }
      };
#pragma unroll 1
      for (int j = 0; j < kWS - 1; ++j) {
        issue_stage(j);
        cp_async_commit();
      }
      for (int i = 0; i < ng; ++i) {
        if ((i & 1) == 0) {
          cp_async_wait<kWS - 2>();  // this thread's stage i / 2 has landed
          issue_stage(i / 2 + kWS - 1);
          cp_async_commit();
        }
        const int s = (i >> 1) % kWS;
        const uint4 w = S.w[wg][s][row][i & 1];
        const uint32_t sp = S.sc[wg][s][row];
        const uint32_t sh = (i & 1) ? (sp >> 16) : (sp & 0xFFFFu);  // fp16 scale of group g0 + i
        uint32_t hl[32];
        weights_hi_lo(w, sh | (sh << 16), hl);
        const int st = i * kWG + wg, q = gs + st, slot = q % kR, use = q / kR;
        if (row == 0) TC_TRACE(4, st);
        // the slot's previous MMAs (ring step q - kR) have finished
        if (use > 0) {
          int okw = 0;
          if (lane == 0 && !*abort_flag) {
            okw = mbar_wait(&S.slot_free[slot], (uint32_t)((use - 1) & 1), kTcWaitNs) ? 1 : 0;
            if (!okw) *abort_flag = 1;
          }
          okw = __shfl_sync(0xffffffffu, okw, 0);
          if (!okw) break;
          mbar_test(&S.slot_free[slot], (uint32_t)((use - 1) & 1));
          tc_fence_after();
        }
        if (row == 0) TC_TRACE(5, st);
        tmem_st32(tmem + lane_base + (uint32_t)(kColA + slot * 32), hl);
        asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
        if (row == 0) TC_TRACE(6, st);
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&S.a_full[slot]);
      }
      cp_async_wait<0>();
    }
    // -------------------------------------------------------- epilogue
    __syncthreads();
    if (tid == kConvThreads) {  // one wait for the item's last commit (bounded)
      if (!mbar_wait(&S.fin, (uint32_t)(it & 1), kTcWaitNs)) *abort_flag = 1;
      TC_TRACE_ITEM();
    }
    __syncthreads();
    tc_fence_after();
    const bool aborted = *abort_flag != 0;  // uniform: nobody writes it until the next item
    float* red = reinterpret_cast<float*>(&S.w[0][0][0][0]);  // [wg][row][kNmax]
    if (warp < kConvThreads / 32 && !aborted) {
      const int wg = warp >> 2, row = (warp & 3) * 32 + lane;
      const uint32_t lane_base = (uint32_t)((warp & 3) * 32) << 16;
      const uint32_t d = tmem + lane_base + (uint32_t)(kColD + wg * kNmax);
#pragma unroll
      for (int c = 0; c < kNmax / 16; ++c) {
        if (c * 16 < N) {
          uint32_t dv[16];
          tmem_ld16(d + (uint32_t)(c * 16), dv);
          asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
          for (int t = 0; t < 16; ++t)
            red[((size_t)wg * 128 + row) * kNmax + c * 16 + t] = __uint_as_float(dv[t]);
        }
      }
    }
    tc_fence_before();
    __syncthreads();
    if (aborted) {
      if (tid == 0) atomicCAS(a.err, 0u, (uint32_t)kErrTimeout);
      break;
    }
    const int* list_tok = L.list_tok;
    const int* list_pos = L.list_pos;
    if (a.mats == 2) {
      // h = silu(gate) * up for the tile's 64 rows, every token
      for (int idx = tid; idx < 64 * n; idx += kTcThreads) {
        const int rr = idx % 64, t = idx / 64;
        float gsum = 0.f, usum = 0.f;
        for (int w = 0; w < kWG; ++w) {
          gsum += red[((size_t)w * 128 + rr) * kNmax + t];
          usum += red[((size_t)w * 128 + rr + 64) * kNmax + t];
        }
        const float f = ldexpf(1.0f, a.row_exp[list_tok[base + t]]);
        a.out[(size_t)list_pos[base + t] * a.R + r0 + rr] = silu_mul(gsum * f, usum * f);
      }
    } else {
      for (int idx = tid; idx < 128 * n; idx += kTcThreads) {
        const int rr = idx % 128, t = idx / 128;
        float ysum = 0.f;
        for (int w = 0; w < kWG; ++w) ysum += red[((size_t)w * 128 + rr) * kNmax + t];
        a.out[(size_t)list_pos[base + t] * a.R + r0 + rr] =
            ysum * ldexpf(1.0f, a.row_exp[list_pos[base + t]]);
      }
    }
    __syncthreads();  // red (the code stages) is rewritten by the next item
  }
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, 512;" ::"r"(tmem));
  }
}

// Power-of-two scale of each input row for the fp16 B operand: the row is
// divided by 2^e (e >= 0, the least with max |v| / 2^e <= 2^14) before it is
// rounded to fp16 and the row's results are multiplied back, so that no
// input overflows fp16; e is 0 for every row of ordinary size.
template <bool kF32>
__global__ void __launch_bounds__(256) tc_rowscale_kernel(const void* in, int K, int rows,
                                                          int* row_exp) {
  __shared__ float part[8];
  const int r = blockIdx.x;
  if (r >= rows) return;
  float m = 0.f;
  for (int k = threadIdx.x; k < K; k += blockDim.x) {
    const float v = kF32 ? static_cast<const float*>(in)[(size_t)r * K + k]
                         : bf16_bits_to_f32(static_cast<const uint16_t*>(in)[(size_t)r * K + k]);
    m = fmaxf(m, fabsf(v));
  }
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  if ((threadIdx.x & 31) == 0) part[threadIdx.x >> 5] = m;
  __syncthreads();
  if (threadIdx.x == 0) {
    for (int w = 1; w < (int)(blockDim.x >> 5); ++w) m = fmaxf(m, part[w]);
    m = fmaxf(m, part[0]);
    int e = 0;
    while (e < 200 && ldexpf(m, -e) > 16384.0f) ++e;  // also stops on inf / nan
    row_exp[r] = e;
  }
}

__device__ __forceinline__ uint16_t f32_to_f16_rne(float f) {
  uint16_t r;
  asm("{ .reg .f16 t; cvt.rn.f16.f32 t, %1; mov.b16 %0, t; }" : "=h"(r) : "f"(f));
  return r;
}

// Packs the inputs of every path expert: for expert rank r and group g, the
// B operand of its MMAs, rows = its tokens (zero rows up to a multiple of
// 16), in the canonical K-major layout [N/8][4][8 rows][8 inputs] of fp16,
// inputs in the MMA order tc_perm, each row divided by 2^row_exp.
// Gate/up: x (bf16 -> fp16, exact within fp16's range).  Down: h (fp32) as
// an fp16 hi tile then an fp16 lo (h - hi) tile.
template <bool kDown>
__global__ void __launch_bounds__(256) tc_pack_kernel(const int* lists, int E, int n_list,
                                                      const void* in, int K, int G,
                                                      const int* row_exp, uint8_t* bpack) {
  const ListsView L = lists_view(lists, E, n_list);
  const int rank = blockIdx.y;
  if (rank >= L.counts[1]) return;
  const int u = L.tc_u[rank];
  const int* list_tok = L.list_tok;
  const int* list_pos = L.list_pos;
  const int base = L.u_off[u], n = L.u_off[u + 1] - base;
  const int N = (n + 15) & ~15;
  const size_t gbytes = tc_group_bytes(kDown ? 1 : 2);
  // one thread per (group, row, core column): 8 inputs -> 16 bytes (x2 for down)
  const int per_group = N * 4;
  for (int idx = blockIdx.x * blockDim.x + threadIdx.x; idx < G * per_group;
       idx += gridDim.x * blockDim.x) {
    const int g = idx / per_group, rem = idx % per_group;
    const int nr = rem / 4, cb = rem % 4;
    uint16_t hi[8], lo[8];
    const int in_row = nr < n ? (kDown ? list_pos[base + nr] : list_tok[base + nr]) : 0;
    const int ex = nr < n ? row_exp[in_row] : 0;
#pragma unroll
    for (int kk = 0; kk < 8; ++kk) {
      hi[kk] = 0;
      lo[kk] = 0;
      if (nr < n) {
        const int kin = g * 32 + tc_perm(cb * 8 + kk);
        if (kDown) {
          const float v = ldexpf(static_cast<const float*>(in)[(size_t)in_row * K + kin], -ex);
          const uint16_t h16 = f32_to_f16_rne(v);
          hi[kk] = h16;
          lo[kk] = f32_to_f16_rne(v - f16_bits_to_f32(h16));
        } else {
          const float v = bf16_bits_to_f32(static_cast<const uint16_t*>(in)[(size_t)in_row * K + kin]);
          hi[kk] = f32_to_f16_rne(ldexpf(v, -ex));
        }
      }
    }
    // core matrix (nr / 8, cb) at ((nr / 8) * 4 + cb) * 128 bytes, row nr % 8
    uint8_t* dst = bpack + ((size_t)rank * G + g) * gbytes +
                   ((size_t)((nr >> 3) * 4 + cb)) * 128 + (size_t)(nr & 7) * 16;
    uint4 vh;
    vh.x = hi[0] | ((uint32_t)hi[1] << 16);
    vh.y = hi[2] | ((uint32_t)hi[3] << 16);
    vh.z = hi[4] | ((uint32_t)hi[5] << 16);
    vh.w = hi[6] | ((uint32_t)hi[7] << 16);
    *reinterpret_cast<uint4*>(dst) = vh;
    if (kDown) {
      uint4 vl;
      vl.x = lo[0] | ((uint32_t)lo[1] << 16);
      vl.y = lo[2] | ((uint32_t)lo[3] << 16);
      vl.z = lo[4] | ((uint32_t)lo[5] << 16);
      vl.w = lo[6] | ((uint32_t)lo[7] << 16);
      *reinterpret_cast<uint4*>(dst + (size_t)N * 64) = vl;
    }
  }
}

}  // namespace

#ifdef MOE_TRACE
extern "C" __attribute__((visibility("default"))) int moe_debug_tc_trace(void* host_dst) {
  return (int)cudaMemcpyFromSymbol(host_dst, g_tc_trace, sizeof(g_tc_trace));
}
#endif

// Most experts a call of T tokens can have on the path: each routed one
// takes kTcMinTok of the T * k entries at least.
int tc_max_experts(int T, int k, int has_shared) {
  return T < kTcMinTok ? 0 : (T * k) / kTcMinTok + has_shared;
}

size_t tc_bpack_bytes(int T, int k, int has_shared, int H, int I) {
  if (T < kTcMinTok) return 0;
  const size_t experts = (size_t)tc_max_experts(T, k, has_shared);
  const size_t gu = (size_t)(H / 32) * tc_group_bytes(2), dn = (size_t)(I / 32) * tc_group_bytes(1);
  return experts * (gu > dn ? gu : dn);
}

size_t tc_rowexp_ints(int T, int k, int has_shared) { return (size_t)T * (k + has_shared); }

bool tc_shape_ok(int H, int I) { return H % 128 == 0 && I % 128 == 0; }

cudaError_t launch_tc_ffn_step(int mats, const ExpertPtrs* table, const int* lists, int E,
                               int n_list, int T, int k, int has_shared, const void* in, int K,
                               int R, int in_rows, int* row_exp, uint8_t* bpack, float* out,
                               uint32_t* err, cudaStream_t st) {
  static DeviceOnce<bool> configured;
  int dev = 0;
  cudaError_t ce = cudaGetDevice(&dev);
  if (ce != cudaSuccess) return ce;
  bool done = false;
  ce = configured.get(dev, &done, [](bool* v) {
    const cudaError_t r = cudaFuncSetAttribute(tc_gemm_kernel,
                                               cudaFuncAttributeMaxDynamicSharedMemorySize,
                                               (int)sizeof(TcSmem));
    *v = r == cudaSuccess;
    return r;
  });
  if (ce != cudaSuccess) return ce;
  const int G = K / 32;
  const int tcmax = tc_max_experts(T, k, has_shared);
  if (tcmax == 0) return cudaSuccess;
  if (mats == 2) {
    tc_rowscale_kernel<false><<<in_rows, 256, 0, st>>>(in, K, in_rows, row_exp);
    tc_pack_kernel<false><<<dim3(16, tcmax), 256, 0, st>>>(lists, E, n_list, in, K, G, row_exp,
                                                           bpack);
  } else {
    tc_rowscale_kernel<true><<<in_rows, 256, 0, st>>>(in, K, in_rows, row_exp);
    tc_pack_kernel<true><<<dim3(16, tcmax), 256, 0, st>>>(lists, E, n_list, in, K, G, row_exp,
                                                          bpack);
  }
  TcArgs a;
  a.table = table;
  a.lists = lists;
  a.E = E;
  a.n_list = n_list;
  a.K = K;
  a.G = G;
  a.R = R;
  a.mats = mats;
  a.bpack = bpack;
  a.row_exp = row_exp;
  a.out = out;
  a.err = err;
  // persistent: one CTA per SM (its shared memory and 512 tensor-memory
  // columns), no more CTAs than the call can have work items
  const int tiles = mats == 2 ? R / 64 : R / 128;
  const int grid = std::min(num_sms(), tcmax * tiles);
  tc_gemm_kernel<<<grid, kTcThreads, sizeof(TcSmem), st>>>(a);
  return cudaGetLastError();
}

}  // namespace moe
