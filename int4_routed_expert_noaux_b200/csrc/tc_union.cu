// tc_union.cu -- the batched (verify) expert path on the 5th-generation
// tensor cores, for every distinct expert that a few (tc_min_tokens()) to
// 64 of the call's tokens route to: each expert's weights stream from HBM
// once for all its tokens (colibri summary, "Principales fonctionnalites
// implementees": batch-union of the experts of the draft tokens; "LightLX",
// "How it works": the MTP verify step), and the products run as tcgen05
// MMAs.
//
// A persistent CTA per SM takes (expert, tile of 128 weight rows) work items
// in turn.  Per CTA:
//   - a weight producer warp points the item's tensor maps at the expert's
//     matrices (tensormap.replace on a copy of a template, published to a
//     per-CTA global slot) and streams the tile's int4 codes and fp16
//     scales with 2-D TMA loads: 128 rows x 8 groups per stage, codes
//     128-byte swizzled so that each thread's row reads without bank
//     conflicts;
//   - two converter warpgroups split the 32-input groups of the K range in
//     halves, one thread per weight row (= tensor-memory lane); a thread
//     forms the group's 32 weights code * scale as an fp16 pair hi + lo,
//     both exact (the scale split into its top 7 and low 4 significant
//     bits, each times a 4-bit code), so hi + lo is the weight exactly, and
//     stores the 32 hi and 32 lo halves to a slot of a ring of A operands
//     in tensor memory;
//   - an input producer warp brings each group's packed token inputs (B
//     operand, fp16, K-major canonical layout; the down projection's h as
//     fp16 hi and lo tiles) into a ring of shared-memory slots by bulk
//     async copies;
//   - four issuer warps (one thread each, taking the groups in turn) run per
//     group the M=128 K=16 fp16 MMAs A_hi B and A_lo B (and A_hi B_lo for
//     the down projection) for both K halves into the issuer's fp32
//     accumulator in tensor memory, which holds its share of the whole K
//     range: no per-group epilogue; one commit per group frees the group's
//     ring slot.
// At the end of an item the four accumulators are read back (tcgen05.ld)
// and added in a fixed order; gate/up tiles hold 64 gate and 64 up rows of
// the same indices, interleaved by 16 so that a warp holds both rows of an
// index, and h = silu(g) * u is formed in the tile.
//
// Within a group the MMA's K order is a fixed permutation of the 32 inputs
// (the order the nibble pairs come out of a word); the packed inputs use the
// same permutation.
#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <algorithm>
#include <atomic>

#include "async.cuh"
#include "common.cuh"
#include "device_once.h"
#include "kernels.h"
#include "tile_stream.cuh"

namespace moe {

namespace {

// Per-step timeline of CTA 0's second work item in a -DMOE_TRACE profiling
// build (row 7: the end of each of CTA 0's items).
#ifdef MOE_TRACE
__device__ uint64_t g_tc_trace[16][256];
__device__ int g_tc_trace_mats = 1;  // the launch traced: 2 gate/up, 1 down
#define TC_TRACE(kind, st)                                                          \
  do {                                                                              \
    if (blockIdx.x == 0 && it == 1 && (st) < 256 && a.mats == g_tc_trace_mats)      \
      g_tc_trace[kind][st] = (uint64_t)clock64();                                   \
  } while (0)
#define TC_TRACE_AT(kind, i)                                                        \
  do {                                                                              \
    if (a.mats == g_tc_trace_mats) g_tc_trace[kind][i] = (uint64_t)clock64();       \
  } while (0)
#define TC_TRACE_ITEM()                                                             \
  do {                                                                              \
    if (blockIdx.x == 0 && it < 256 && a.mats == g_tc_trace_mats)                   \
      g_tc_trace[7][it] = (uint64_t)clock64();                                      \
  } while (0)
#else
#define TC_TRACE(kind, st) ((void)0)
#define TC_TRACE_AT(kind, i) ((void)0)
#define TC_TRACE_ITEM() ((void)0)
#endif

constexpr int kConvThreads = kWG * 128;
// + six warps, separate so that one's waits never hold up another's issue.
// Four MMA issuers: a thread stalls about 90 cycles on each tcgen05.mma it
// issues (and more on its commit), while the tensor cores finish an M=128
// N<=64 K=16 MMA in about 45, so issuer j takes the ring steps st = j
// (mod 4) -- warpgroup j % 2's groups -- into an accumulator of its own.
constexpr int kWProdWarp = kConvThreads / 32;  // weight tiles (TMA), tensor maps
constexpr int kBProdWarp = kWProdWarp + 1;     // packed inputs
constexpr int kIssueWarp = kWProdWarp + 2;     // MMA issuer j: warp kIssueWarp + j
constexpr int kIssuers = 2 * kWG;
constexpr int kTcThreads = kConvThreads + 32 * (2 + kIssuers);
constexpr int kBRing = 64 * 1024;         // shared memory of the B ring
constexpr int kNmax = 64;                 // most tokens per expert on this path
// Tensor memory: the accumulator of issuer j at columns j * Ncap (Ncap: the
// call's most padded tokens of an expert), then the ring's A slots of 32
// columns (hi 16, lo 16).  The ring has as many slots as tensor memory and
// the B ring's shared memory hold at Ncap: 8 at 64 tokens, 12 at 32.
static_assert(kTcMaxTok == kNmax, "the token bound of the path");

struct __align__(1024) TcSmem : StreamSmem {
  uint8_t b[kBRing];                      // B ring: slot s at s * Ncap * (64 or 128) bytes
  uint64_t a_full[kRmax];                 // converters wrote the slot's A (4 warps)
  uint64_t fin;                           // all MMAs of the item finished (4 issuers)
  uint64_t d_free;                        // the item's accumulators were read (8 warps)
  uint32_t tmem_base;
};
static_assert(sizeof(TcSmem) + 1024 <= 232448, "shared memory per CTA");

// The MMA-K order of a group's 32 inputs: K index 8 i + 2 j + h holds input
// 8 i + j + 4 h (the converter makes the pair of TMEM column 4 i + j from
// nibbles j and j + 4 of word i; tc_pack_kernel packs the inputs alike).

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

__device__ __forceinline__ void tmem_ld8(uint32_t taddr, uint32_t (&v)[8]) {
  asm volatile("tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"
               : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]),
                 "=r"(v[6]), "=r"(v[7])
               : "r"(taddr)
               : "memory");
}

// A group's fp16 scale s split for weights_hi_lo, as f16x2 pairs (both
// halves equal): s_hi = s with its 4 low mantissa bits cleared (at most 7
// significant bits), s_lo = s - s_hi (at most 4), and -24 times each (exact:
// 24 has 2 significant bits).
struct GroupScale {
  uint32_t s1, s2, c1, c2;
};

__device__ __forceinline__ GroupScale group_scale(uint32_t sh) {
  GroupScale g;
  const uint32_t s = sh | (sh << 16);
  g.s1 = s & 0xFFF0FFF0u;
  asm("sub.rn.f16x2 %0, %1, %2;" : "=r"(g.s2) : "r"(s), "r"(g.s1));
  asm("{ .reg .b32 m; mov.b32 m, 0xCE00CE00; mul.rn.f16x2 %0, %1, m; }" : "=r"(g.c1) : "r"(g.s1));
  asm("{ .reg .b32 m; mov.b32 m, 0xCE00CE00; mul.rn.f16x2 %0, %1, m; }" : "=r"(g.c2) : "r"(g.s2));
  return g;
}

// The 32 weights code * s of one 16-byte chunk as fp16 pairs: hi[4i + j]
// holds code * s_hi of nibbles j and j + 4 of word i, lo[4i + j] code * s_lo.
// Both products are exact in fp16 (a code of at most 4 significant bits
// times 7 or 4), so hi + lo = code * s.  Each is one fma on v = fp16(16 + u),
// u = nibble ^ 8 = code + 8 (a shift and one bit operation put u in the
// mantissa under the exponent of 16): v * s_x - 24 * s_x = code * s_x.
__device__ __forceinline__ void weights_hi_lo(const uint4 w, const GroupScale& gs,
                                              uint32_t (&hl)[32]) {
  const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      // nibbles j and j + 4 to bits 6..9 of their halves
      const uint32_t t = j < 2 ? ws[i] << (6 - 4 * j) : ws[i] >> (4 * j - 6);
      const uint32_t v = (t & 0x03C003C0u) ^ 0x4E004E00u;
      uint32_t hi, lo;
      asm("fma.rn.f16x2 %0, %1, %2, %3;" : "=r"(hi) : "r"(v), "r"(gs.s1), "r"(gs.c1));
      asm("fma.rn.f16x2 %0, %1, %2, %3;" : "=r"(lo) : "r"(v), "r"(gs.s2), "r"(gs.c2));
      hl[4 * i + j] = hi;
      hl[16 + 4 * i + j] = lo;
    }
  }
}

struct TcArgs {
  const ExpertPtrs* table;
  const int* lists;
  int E, n_list;
  int K, G;          // inputs of a weight row and its 32-input groups
  int R;             // rows of one weight matrix
  int mats;          // 2: gate/up tiles (64 + 64 rows), 1: down tiles (128 rows)
  const uint8_t* bpack;  // packed B: expert rank r from row tc_roff[r], [G][its rows][64 or 128 B]
  const int* row_exp;    // power-of-two scale of each input row (tc_rowscale_kernel)
  float* out;        // [T slots][R] (h for gate/up, partial y for down)
  uint32_t* err;     // kErrTimeout when a wait ran out
  CUtensorMap* maps; // [grid][kMapSets][kMaps] global slots for the tensor maps
};

// tm_codes / tm_scales: templates of the item's maps (dimensions, strides,
// boxes: codes uint8 [R][K/2], box 128 bytes x tile rows, 128-byte swizzle;
// scales uint16 [R][G], box 8 x tile rows); each item points copies of them
// at its expert's matrices.
__global__ void __launch_bounds__(kTcThreads, 1)
    tc_gemm_kernel(const TcArgs a, const __grid_constant__ CUtensorMap tm_codes,
                   const __grid_constant__ CUtensorMap tm_scales) {
  pdl_wait();
  extern __shared__ uint8_t tsmem_raw[];
  // 1024-byte alignment for the swizzled code tiles
  TcSmem& S = *reinterpret_cast<TcSmem*>(tsmem_raw + ((1024u - (smem_addr(tsmem_raw) & 1023u)) & 1023u));
  const ListsView L = lists_view(a.lists, a.E, a.n_list);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int tile_rows = a.mats == 2 ? 64 : 128;
  const int tiles = a.R / tile_rows;
  const int items = L.counts[1] * tiles;
  if ((int)blockIdx.x >= items) return;  // uniform per CTA, before any barrier
  const int ng = a.G / kWG;              // groups per warpgroup (a multiple of kGS)
  const int nst = ng / kGS;              // weight stages per warpgroup and item
  const int steps = kWG * ng;            // step s of an item: warpgroup s % kWG, its group s / kWG
  const int mb = a.mats == 2 ? 64 : 128;  // bytes of a packed input row of one group
  volatile int* abort_flag = &S.abort_flag;
  // the call's most padded tokens of an expert (every warp reduces it)
  int ncap = 16;
  for (int r = lane; r < L.counts[1]; r += 32) ncap = max(ncap, L.tc_roff[r + 1] - L.tc_roff[r]);
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) ncap = max(ncap, __shfl_xor_sync(0xffffffffu, ncap, o));
  // (a multiple of kBG: a B copy fills kBG consecutive slots)
  const int kR =
      min(kRmax, min((512 - kIssuers * ncap) / 32, kBRing / (ncap * mb))) / kBG * kBG;
  const uint32_t colA = (uint32_t)(kIssuers * ncap);
  const int bstride = ncap * mb;  // bytes of a B ring slot

  if (tid == 0) {
    for (int w = 0; w < kWG; ++w)
      for (int s = 0; s < kSW; ++s) {
        mbar_init(&S.w_full[w][s], 1);
        mbar_init(&S.w_empty[w][s], 4);
      }
    for (int i = 0; i < kRmax; ++i) {
      mbar_init(&S.a_full[i], 4);

      mbar_init(&S.slot_free[i], 1);
    }
    for (int i = 0; i < kRmax / kBG; ++i) mbar_init(&S.b_full[i], 1);
    mbar_init(&S.fin, kIssuers);
    mbar_init(&S.d_free, kConvThreads / 32);
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
  // tiles of an expert adjacent.  Each role runs its own loop over the
  // CTA's items; the rings run on across items (ring step it * steps + st,
  // weight stage it * nst + j), so the producers stream the next item's
  // tiles while the converters finish this one's epilogue.  An item's first
  // MMAs wait until the previous item's accumulators were read (d_free).
  int w_last[kWG][kSW];  // weight producer: last use issued per stage buffer
  int b_last[kRmax / kBG];  // input producer: the same per B run
  for (int w = 0; w < kWG; ++w)
    for (int s = 0; s < kSW; ++s) w_last[w][s] = -1;
  for (int i = 0; i < kRmax / kBG; ++i) b_last[i] = -1;
  const int* list_tok = L.list_tok;
  const int* list_pos = L.list_pos;

  StreamGeom geom;
  geom.items = items;
  geom.tiles = tiles;
  geom.tile_rows = tile_rows;
  geom.mats = a.mats;
  geom.ng = ng;
  geom.nst = nst;
  geom.steps = steps;
  if (warp == kWProdWarp) {
    stream_weights(S, geom, a.table, L.u_expert, L.tc_u, a.maps, tm_codes, tm_scales, lane,
                   abort_flag, w_last);
  } else if (warp == kBProdWarp) {
    if (lane == 0)
      stream_inputs(S, S.b, geom, L.tc_roff, a.bpack, a.G, mb, bstride, kR, abort_flag, b_last);
  } else if (warp >= kIssueWarp) {
    if (lane == 0) {
      // ---------------------------------------------- MMA issuers
      const int j = warp - kIssueWarp;
      const uint32_t d = tmem + (uint32_t)(j * ncap);
      RingPos pos;  // ring step it * steps + st
      pos.advance(j, kR);
      for (int item = blockIdx.x, it = 0; item < items; item += gridDim.x, ++it) {
        const int rank = item / tiles;
        const int N = L.tc_roff[rank + 1] - L.tc_roff[rank];
        const uint32_t idesc = umma_idesc_f16(128, N);
        // the previous item's accumulators have been read
        if (*abort_flag ||
            (it > 0 && !stream_wait(&S.d_free, (uint32_t)((it - 1) & 1)))) {
          *abort_flag = 1;
          tc_commit(&S.fin);
          break;
        }
        tc_fence_after();
        for (int st = j; st < steps; st += kIssuers) {
          const int slot = pos.slot, use = pos.use;
          pos.advance(kIssuers, kR);
          if (*abort_flag || !stream_wait(&S.a_full[slot], (uint32_t)(use & 1))) {
            *abort_flag = 1;
            break;
          }
          TC_TRACE(1, st);
          if (!stream_wait(&S.b_full[slot / kBG], (uint32_t)(use & 1))) {
            *abort_flag = 1;
            break;
          }
          TC_TRACE(2, st);
          tc_fence_after();
          const uint32_t ahi = tmem + colA + (uint32_t)(slot * 32), alo = ahi + 16;
          // step q's inputs: kBG steps of N rows each from the run's first slot
          const uint32_t bhi = smem_addr(S.b + (slot / kBG * kBG) * bstride) +
                               (uint32_t)((slot % kBG) * N * mb),
                         blo = bhi + (uint32_t)N * 64;
#pragma unroll
          for (int kk = 0; kk < 2; ++kk) {
            const uint64_t dh = umma_desc(bhi + kk * 256, 128, 512);
            tc_mma(d, ahi + kk * 8, dh, idesc, (st >= kIssuers || kk > 0) ? 1u : 0u);
            tc_mma(d, alo + kk * 8, dh, idesc, 1u);
            if (a.mats == 1)
              tc_mma(d, ahi + kk * 8, umma_desc(blo + kk * 256, 128, 512), idesc, 1u);
          }
          tc_commit(&S.slot_free[slot]);
          TC_TRACE(3, st);
        }
        // every MMA of this issuer's item has finished when this arrives
        tc_commit(&S.fin);
        if (*abort_flag) break;
      }
    }
  } else {
    // ---------------------------------------------------- converters
    const int wg = warp >> 2, row = (warp & 3) * 32 + lane;  // row = tensor-memory lane
    const uint32_t lane_base = (uint32_t)((warp & 3) * 32) << 16;
    const uint32_t swz = (uint32_t)(row & 7);
    RingPos pos;  // ring step of this warpgroup's next group
    pos.advance(wg, kR);
    for (int item = blockIdx.x, it = 0; item < items; item += gridDim.x, ++it) {
      const int rank = item / tiles;
      const int u = L.tc_u[rank];
      const int base = L.u_off[u], n = L.u_off[u + 1] - base;
      const int N = L.tc_roff[rank + 1] - L.tc_roff[rank];
      const int r0 = (item % tiles) * tile_rows;
      bool ok = true;
      for (int j = 0; j < nst && ok; ++j) {
        const int q = it * nst + j, sb = q % kSW, use = q / kSW;
        if (!warp_wait(&S.w_full[wg][sb], (uint32_t)(use & 1), lane, abort_flag)) {
          ok = false;
          break;
        }
        const uint8_t* crow = &S.wc[wg][sb][row * 128];
        const uint4 sc8 = *reinterpret_cast<const uint4*>(&S.wsc[wg][sb][row * 16]);
        const uint32_t spair[4] = {sc8.x, sc8.y, sc8.z, sc8.w};
#pragma unroll
        for (int c = 0; c < kGS; ++c) {
          const uint4 w = *reinterpret_cast<const uint4*>(crow + (((uint32_t)c ^ swz) << 4));
          const uint32_t sh = (c & 1) ? (spair[c >> 1] >> 16) : (spair[c >> 1] & 0xFFFFu);
          uint32_t hl[32];
          weights_hi_lo(w, group_scale(sh), hl);
          const int i = j * kGS + c;  // group of this warpgroup
          [[maybe_unused]] const int st = i * kWG + wg;  // the item's ring step (traces)
          const int slot = pos.slot, suse = pos.use;
          pos.advance(kWG, kR);
          if (row == 0) TC_TRACE(4, st);
          // the slot's previous MMAs (ring step qs - kR) have finished
          if (suse > 0) {
            if (!warp_wait(&S.slot_free[slot], (uint32_t)((suse - 1) & 1), lane, abort_flag)) {
              ok = false;
              break;
            }
            tc_fence_after();
          }
          if (row == 0) TC_TRACE(5, st);
          tmem_st32(tmem + lane_base + colA + (uint32_t)(slot * 32), hl);
          asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
          if (row == 0) TC_TRACE(6, st);
          if (lane == 0) TC_TRACE(8 + (warp & 3), st);
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&S.a_full[slot]);
        }
        // the stage's codes and scales are read (every lane's loads retired)
        __syncwarp();
        if (lane == 0) mbar_arrive(&S.w_empty[wg][sb]);
      }
      // ------------------------------------------------------ epilogue
      // Thread (wg, row) takes tokens [wg * N/2, (wg + 1) * N/2) of its
      // row: the four issuers' accumulators, added in a fixed order (the
      // K halves of warpgroup 0, then of warpgroup 1).
      if (!ok || !warp_wait(&S.fin, (uint32_t)(it & 1), lane, abort_flag)) break;
      if (row == 0 && wg == 0) TC_TRACE_ITEM();
      tc_fence_after();
      const int half = N >> 1, t0 = wg * half;
      float sum[kNmax / 2];
      const uint32_t dl = tmem + lane_base + (uint32_t)t0;
#pragma unroll
      for (int c = 0; c < kNmax / 2; c += 8) {
        if (c < half) {
          uint32_t v0[8], v1[8], v2[8], v3[8];
          tmem_ld8(dl + (uint32_t)(0 * ncap + c), v0);
          tmem_ld8(dl + (uint32_t)(2 * ncap + c), v2);
          tmem_ld8(dl + (uint32_t)(1 * ncap + c), v1);
          tmem_ld8(dl + (uint32_t)(3 * ncap + c), v3);
          asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
          for (int t = 0; t < 8; ++t)
            sum[c + t] = (__uint_as_float(v0[t]) + __uint_as_float(v2[t])) +
                         (__uint_as_float(v1[t]) + __uint_as_float(v3[t]));
        }
      }
      // the accumulators may be overwritten by the next item's MMAs
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&S.d_free);
      // 8 tokens at a time: their output rows and input scales first (the
      // lists are read-only in this kernel: non-coherent loads, which the
      // stores before them do not hold back), then the outputs
      const int orow = a.mats == 2 ? r0 + 16 * (warp & 3) + (lane & 15) : r0 + row;
#pragma unroll
      for (int c0 = 0; c0 < kNmax / 2; c0 += 8) {
        if (c0 < half) {
          int pos[8];
          float f[8];
#pragma unroll
          for (int u8 = 0; u8 < 8; ++u8) {
            const int t = t0 + c0 + u8;
            pos[u8] = 0;
            f[u8] = 0.f;
            if (t < n) {
              pos[u8] = __ldg(list_pos + base + t);
              const int in_row = a.mats == 2 ? __ldg(list_tok + base + t) : pos[u8];
              f[u8] = ldexpf(1.0f, __ldg(a.row_exp + in_row));
            }
          }
#pragma unroll
          for (int u8 = 0; u8 < 8; ++u8) {
            const int t = t0 + c0 + u8;
            if (a.mats == 2) {
              // h = silu(gate) * up: lane m < 16 of quarter q holds gate row
              // r0 + 16 q + m, lane m + 16 the up row of the same index
              const float up = __shfl_down_sync(0xffffffffu, sum[c0 + u8], 16);
              if (lane < 16 && t < n)
                a.out[(size_t)pos[u8] * a.R + orow] =
                    silu_mul(sum[c0 + u8] * f[u8], up * f[u8]);
            } else if (t < n) {
              a.out[(size_t)pos[u8] * a.R + orow] = sum[c0 + u8] * f[u8];
            }
          }
        }
      }
    }
  }
  // A wait that ran out leaves the rest of the call's results unwritten
  // and reports it (after the producers drained their copies).
  __syncthreads();
  if (*abort_flag) {
    if (tid == 0) atomicCAS(a.err, 0u, (uint32_t)kErrTimeout);
    stream_drain(S, warp, lane, kWProdWarp, kBProdWarp, kR, w_last, b_last);
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
// 16-byte loads (K a multiple of 8), several in flight per thread.
template <bool kF32>
__global__ void __launch_bounds__(256) tc_rowscale_kernel(const void* in, int K, int rows,
                                                          int* row_exp) {
  pdl_wait();
  __shared__ float part[8];
  const int r = blockIdx.x;
  if (r >= rows) return;
  float m = 0.f;
  if (kF32) {
    const float4* p = reinterpret_cast<const float4*>(static_cast<const float*>(in) + (size_t)r * K);
#pragma unroll 4
    for (int c = threadIdx.x; c < K / 4; c += blockDim.x) {
      const float4 v = p[c];
      m = fmaxf(m, fmaxf(fmaxf(fabsf(v.x), fabsf(v.y)), fmaxf(fabsf(v.z), fabsf(v.w))));
    }
  } else {
    const uint4* p = reinterpret_cast<const uint4*>(static_cast<const uint16_t*>(in) + (size_t)r * K);
#pragma unroll 4
    for (int c = threadIdx.x; c < K / 8; c += blockDim.x) {
      const uint4 v = p[c];
      const uint32_t u[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
      for (int j = 0; j < 4; ++j)
        m = fmaxf(m, fmaxf(fabsf(bf16_bits_to_f32(u[j] & 0xFFFFu)), fabsf(bf16_bits_to_f32(u[j] >> 16))));
    }
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
// B operand of its MMAs, rows = its tokens (zero rows up to N, a multiple of
// 16), at byte (tc_roff[r] * G + s * N) * (64, down: 128) where s is the
// group's ring step (2 (g mod G/2) + g div G/2: the two warpgroups' groups
// alternate, so consecutive steps' inputs are contiguous), in the canonical
// K-major layout [N/8][4][8 rows][8 inputs] of fp16, inputs in the MMA order,
// each row divided by 2^row_exp.
// Gate/up: x (bf16 -> fp16, exact within fp16's range).  Down: h (fp32) as
// an fp16 hi tile then an fp16 lo (h - hi) tile.
// One thread per (group, row): the row's 32 inputs of the group in 16-byte
// loads, out as 4 core-matrix rows of 16 bytes (chunk cb holds inputs
// 8 cb + {0, 4, 1, 5, 2, 6, 3, 7}).
template <bool kDown>
__global__ void __launch_bounds__(256) tc_pack_kernel(const int* lists, int E, int n_list,
                                                      const void* in, int K, int G,
                                                      const int* row_exp, uint8_t* bpack) {
  pdl_wait();
  const ListsView L = lists_view(lists, E, n_list);
  const int rank = blockIdx.y;
  if (rank >= L.counts[1]) return;
  const int u = L.tc_u[rank];
  const int* list_tok = L.list_tok;
  const int* list_pos = L.list_pos;
  const int base = L.u_off[u], n = L.u_off[u + 1] - base;
  const int roff = L.tc_roff[rank], N = L.tc_roff[rank + 1] - roff;
  const size_t gbytes = (size_t)N * (kDown ? 128 : 64);
  uint8_t* dst0 = bpack + (size_t)roff * G * (kDown ? 128 : 64);
  for (int idx = blockIdx.x * blockDim.x + threadIdx.x; idx < G * N;
       idx += gridDim.x * blockDim.x) {
    const int g = idx / N, nr = idx % N;
    float v[32];
    if (nr < n) {
      const int in_row = kDown ? list_pos[base + nr] : list_tok[base + nr];
      const float sc = ldexpf(1.0f, -row_exp[in_row]);
      if (kDown) {
        const float4* p = reinterpret_cast<const float4*>(static_cast<const float*>(in) +
                                                          (size_t)in_row * K + g * 32);
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          const float4 f = p[j];
          v[4 * j] = f.x * sc;
          v[4 * j + 1] = f.y * sc;
          v[4 * j + 2] = f.z * sc;
          v[4 * j + 3] = f.w * sc;
        }
      } else {
        const uint4* p = reinterpret_cast<const uint4*>(static_cast<const uint16_t*>(in) +
                                                        (size_t)in_row * K + g * 32);
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const uint4 q = p[j];
          const uint32_t w4[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
          for (int h = 0; h < 4; ++h) {
            v[8 * j + 2 * h] = bf16_bits_to_f32(w4[h] & 0xFFFFu) * sc;
            v[8 * j + 2 * h + 1] = bf16_bits_to_f32(w4[h] >> 16) * sc;
          }
        }
      }
    } else {
#pragma unroll
      for (int j = 0; j < 32; ++j) v[j] = 0.f;
    }
    // group g's tile at its ring step (warpgroup g / (G/2), its group g % (G/2));
    // core matrix (nr / 8, cb) at ((nr / 8) * 4 + cb) * 128 bytes, row nr % 8
    const int half_g = G / kWG, step = kWG * (g % half_g) + g / half_g;
    uint8_t* dst = dst0 + (size_t)step * gbytes + (size_t)(nr >> 3) * 512 + (size_t)(nr & 7) * 16;
#pragma unroll
    for (int cb = 0; cb < 4; ++cb) {
      uint32_t hi[4], lo[4];
#pragma unroll
      for (int h = 0; h < 4; ++h) {
        // MMA-K order: the pair (8 cb + h, 8 cb + h + 4)
        const float a0 = v[8 * cb + h], a1 = v[8 * cb + h + 4];
        const uint16_t h0 = f32_to_f16_rne(a0), h1 = f32_to_f16_rne(a1);
        hi[h] = h0 | ((uint32_t)h1 << 16);
        if (kDown) {
          const uint16_t l0 = f32_to_f16_rne(a0 - f16_bits_to_f32(h0));
          const uint16_t l1 = f32_to_f16_rne(a1 - f16_bits_to_f32(h1));
          lo[h] = l0 | ((uint32_t)l1 << 16);
        }
      }
      *reinterpret_cast<uint4*>(dst + cb * 128) = make_uint4(hi[0], hi[1], hi[2], hi[3]);
      if (kDown)
        *reinterpret_cast<uint4*>(dst + cb * 128 + (size_t)N * 64) =
            make_uint4(lo[0], lo[1], lo[2], lo[3]);
    }
  }
}

std::atomic<int> g_tc_min{kTcMinTokDefault};

}  // namespace

int tc_min_tokens() { return g_tc_min.load(std::memory_order_relaxed); }

#ifdef MOE_TRACE
extern "C" __attribute__((visibility("default"))) int moe_debug_tc_trace(void* host_dst) {
  return (int)cudaMemcpyFromSymbol(host_dst, g_tc_trace, sizeof(g_tc_trace));
}

extern "C" __attribute__((visibility("default"))) int moe_debug_tc_trace_mats(int mats) {
  return (int)cudaMemcpyToSymbol(g_tc_trace_mats, &mats, sizeof(int));
}

// Profiling builds: the least token count of a tensor-core expert.
extern "C" __attribute__((visibility("default"))) int moe_debug_set_tc_min(int n) {
  if (n < kTcMinTokFloor || n > kTcMaxTok + 1) return -1;
  g_tc_min.store(n, std::memory_order_relaxed);
  return 0;
}
#endif

// Most experts a call of T tokens can have on the path: each routed one
// takes kTcMinTokFloor of the T * k entries at least.
int tc_max_experts(int T, int k, int has_shared) {
  if (T < kTcMinTokFloor) return 0;
  return std::min((T * k) / kTcMinTokFloor + has_shared, T * k + has_shared);
}

// Packed input rows: each path expert's tokens rounded up to 16.
size_t tc_bpack_bytes(int T, int k, int has_shared, int H, int I) {
  const size_t experts = (size_t)tc_max_experts(T, k, has_shared);
  if (experts == 0) return 0;
  const size_t rows = (size_t)T * (k + has_shared) + 15 * experts;
  const size_t gu = (size_t)(H / 32) * 64, dn = (size_t)(I / 32) * 128;
  return rows * (gu > dn ? gu : dn);
}

size_t tc_rowexp_ints(int T, int k, int has_shared) { return (size_t)T * (k + has_shared); }

size_t tc_maps_bytes() { return stream_maps_bytes(); }

// Weight stages of 8 groups per warpgroup half of K: K a multiple of 512.
bool tc_shape_ok(int H, int I) {
  return H % 512 == 0 && I % 512 == 0 && tensor_maps_available();
}

cudaError_t launch_tc_ffn_step(int mats, const ExpertPtrs* table, const int* lists, int E,
                               int n_list, int T, int k, int has_shared, const void* in, int K,
                               int R, int in_rows, int* row_exp, uint8_t* bpack, uint8_t* maps,
                               float* out, uint32_t* err, cudaStream_t st) {
  static DeviceOnce<bool> configured;
  int dev = 0;
  cudaError_t ce = cudaGetDevice(&dev);
  if (ce != cudaSuccess) return ce;
  bool done = false;
  ce = configured.get(dev, &done, [](bool* v) {
    const cudaError_t r = cudaFuncSetAttribute(tc_gemm_kernel,
                                               cudaFuncAttributeMaxDynamicSharedMemorySize,
                                               (int)sizeof(TcSmem) + 1024);
    *v = r == cudaSuccess;
    return r;
  });
  if (ce != cudaSuccess) return ce;
  const int G = K / 32;
  const int tcmax = tc_max_experts(T, k, has_shared);
  if (tcmax == 0) return cudaSuccess;
  // templates: the matrices the weight rows of a tile come from are [R][K];
  // a box is 8 groups of 16 (gate/up: gate and up rows interleave in the
  // tile by 16) or 128 rows
  const int tile_rows = mats == 2 ? 64 : 128, box_rows = mats == 2 ? 16 : 128;
  CUtensorMap tm_codes, tm_scales;
  if (!encode_2d(&tm_codes, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, bpack, (uint64_t)K / 2,
                 (uint64_t)R, 128, (uint32_t)box_rows, CU_TENSOR_MAP_SWIZZLE_128B) ||
      !encode_2d(&tm_scales, CU_TENSOR_MAP_DATA_TYPE_UINT16, 2, bpack, (uint64_t)G, (uint64_t)R,
                 kGS, (uint32_t)box_rows, CU_TENSOR_MAP_SWIZZLE_NONE))
    return cudaErrorInvalidValue;
  if (mats == 2) {
    launch_pdl(tc_rowscale_kernel<false>, dim3(in_rows), dim3(256), 0, st, in, K, in_rows, row_exp);
    launch_pdl(tc_pack_kernel<false>, dim3(16, tcmax), dim3(256), 0, st, lists, E, n_list, in, K,
               G, row_exp, bpack);
  } else {
    launch_pdl(tc_rowscale_kernel<true>, dim3(in_rows), dim3(256), 0, st, in, K, in_rows, row_exp);
    launch_pdl(tc_pack_kernel<true>, dim3(16, tcmax), dim3(256), 0, st, lists, E, n_list, in, K,
               G, row_exp, bpack);
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
  a.maps = reinterpret_cast<CUtensorMap*>(maps);
  // persistent: one CTA per SM (its shared memory and 512 tensor-memory
  // columns), no more CTAs than the call can have work items
  const int tiles = R / tile_rows;
  const int grid = std::min(std::min(num_sms(), kStreamMaxCtas), tcmax * tiles);
  launch_pdl(tc_gemm_kernel, dim3(grid), dim3(kTcThreads), sizeof(TcSmem) + 1024, st, a, tm_codes,
             tm_scales);
  return cudaGetLastError();
}

}  // namespace moe
