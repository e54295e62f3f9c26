// tile_stream.cuh -- the weight and input streams of the persistent batched
// expert kernel on the tensor cores (tc_union.cu), with the waits and ring
// bookkeeping it uses.  A CTA takes work items (expert, tile of 128 weight
// rows) in turn; per CTA
//   - a weight producer warp points the item's tensor maps at the expert's
//     matrices (tensormap.replace on a copy of a launch template, published
//     to a per-CTA global slot with a proxy fence) and streams the tile's
//     int4 codes and fp16 scales by 2-D TMA loads, 8 groups of 128 rows per
//     stage and warpgroup (codes 128-byte swizzled: each consumer thread
//     reads its own row without bank conflicts);
//   - an input producer warp copies the item's packed token inputs into a
//     ring of shared-memory slots, one ring step per (warpgroup, group),
//     kBG steps per bulk copy.
// Both run ahead across items: the next item's tiles stream while the
// consumers finish the current one.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "async.cuh"
#include "common.cuh"

namespace moe {

constexpr int kWG = 2;             // consumer warpgroups (K halves), 128 threads = rows each
constexpr int kGS = 8;             // groups per weight stage: 128 bytes of codes a row
constexpr int kSW = 3;             // weight stages per warpgroup
constexpr int kRmax = 16;          // input ring slots at most
constexpr int kBG = 4;             // ring steps filled by one input copy
constexpr int kMaps = 4;           // tensor maps of an item: (codes, scales) x matrices
constexpr int kMapSets = 4;        // map sets per CTA, used by items in turn
constexpr int kStreamMaxCtas = 256;  // per-CTA tensor-map slots in the workspace
constexpr uint32_t kWStageBytes = 128 * 128 + 128 * 16;
constexpr uint64_t kStreamWaitNs = 1000000000ull;
static_assert(kMapSets - 1 >= kSW, "a map set outlives the loads through it");

// Bytes of the per-CTA tensor-map slots of a workspace.
inline size_t stream_maps_bytes() {
  return (size_t)kStreamMaxCtas * kMapSets * kMaps * sizeof(CUtensorMap);
}

// A 2-D tensor map over a row-major matrix [rows][inner] of `bytes`-byte
// elements with the given box and swizzle; base is any 16-byte aligned
// address (the kernels re-point it).  False if the driver refuses it.
bool encode_2d(CUtensorMap* m, CUtensorMapDataType dt, int bytes, void* base, uint64_t inner,
               uint64_t rows, uint32_t box_inner, uint32_t box_rows, CUtensorMapSwizzle sw);
bool tensor_maps_available();

// A position on a ring (slot, turn), advanced without division: the ring's
// depth is a launch-time value.
struct RingPos {
  int slot = 0, use = 0;
  __device__ __forceinline__ void advance(int n, int depth) {  // n <= depth
    slot += n;
    if (slot >= depth) {
      slot -= depth;
      ++use;
    }
  }
};

// 2-D tiled TMA load of box (x, y) of a tensor map in global memory.
__device__ __forceinline__ void tma_load_2d(void* dst, const CUtensorMap* map, int x, int y,
                                            uint64_t* bar, uint64_t policy) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      ".L2::cache_hint [%0], [%1, {%2, %3}], [%4], %5;" ::"r"(smem_addr(dst)),
      "l"(map), "r"(x), "r"(y), "r"(smem_addr(bar)), "l"(policy)
      : "memory");
}

// Tensor-map updates: the global address of a map held in shared memory;
// its copy to global memory with a release of the tensormap proxy (whole
// warp); the acquire before the first load through it.
__device__ __forceinline__ void tmap_set_address(CUtensorMap* smem_map, const void* addr) {
  asm volatile("tensormap.replace.tile.global_address.shared::cta.b1024.b64 [%0], %1;" ::"r"(
                   smem_addr(smem_map)),
               "l"(addr)
               : "memory");
}
__device__ __forceinline__ void tmap_publish(CUtensorMap* gmem_map, const CUtensorMap* smem_map) {
  asm volatile(
      "tensormap.cp_fenceproxy.global.shared::cta.tensormap::generic.release.gpu.sync.aligned"
      " [%0], [%1], 128;" ::"l"(gmem_map),
      "r"(smem_addr(smem_map))
      : "memory");
}
__device__ __forceinline__ void tmap_acquire(const CUtensorMap* gmem_map) {
  asm volatile("fence.proxy.tensormap::generic.acquire.gpu [%0], 128;" ::"l"(gmem_map)
               : "memory");
}

// Wait for phase `parity` suspended in hardware (try_wait with a time hint
// of 100 us): the thread takes no issue slots while it waits and wakes as
// the phase completes (spinning waiters would take issue slots from the
// consumers).  False if the phase has not completed kStreamWaitNs after the
// first probe.
__device__ __forceinline__ bool stream_wait(uint64_t* bar, uint32_t parity) {
  if (mbar_test(bar, parity)) return true;
  const uint64_t deadline = global_timer_ns() + kStreamWaitNs;
  for (;;) {
    if (mbar_try_wait_hint(bar, parity, 100000u)) return true;
    if (global_timer_ns() > deadline) return false;
  }
}

// Waits (bounded) in lane 0 and makes every lane an observer of the phase:
// false (the same in all lanes) when the wait ran out or the CTA aborted.
__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity, int lane,
                                          volatile int* abort_flag) {
  int ok = 0;
  if (lane == 0 && !*abort_flag) {
    ok = stream_wait(bar, parity) ? 1 : 0;
    if (!ok) *abort_flag = 1;
  }
  ok = __shfl_sync(0xffffffffu, ok, 0);
  if (ok) mbar_test(bar, parity);
  return ok != 0;
}

// The shape of a launch's work: items (expert rank r = item / tiles, tile
// item % tiles of tile_rows rows of each of `mats` matrices), ng groups per
// warpgroup in nst weight stages, steps = kWG * ng ring steps per item.
struct StreamGeom {
  int items, tiles, tile_rows, mats, ng, nst, steps;
};

// The shared-memory fields the streams use (the kernel's own layout extends it).
struct __align__(1024) StreamSmem {
  uint8_t wc[kWG][kSW][128 * 128];  // code tiles: 128 rows x 8 groups, 128-byte swizzled
  uint8_t wsc[kWG][kSW][128 * 16];  // scale tiles: 128 rows x 8 fp16
  CUtensorMap tm[kMaps];            // the item's tensor maps, before publishing
  uint64_t w_full[kWG][kSW];        // a weight stage landed
  uint64_t w_empty[kWG][kSW];       // the warpgroup's 4 warps read it
  uint64_t b_full[kRmax / kBG];     // a run of kBG slots' inputs landed (one copy)
  uint64_t slot_free[kRmax];        // the slot's readers are done with it
  int abort_flag;
};

// Weight producer (a whole warp; lane 0 issues the loads).  units: the
// expert slot of each rank; tm_codes / tm_scales: the launch's templates
// (codes uint8 [R][K/2], box 128 bytes x box_rows, 128-byte swizzle; scales
// uint16 [R][G], box 8 x box_rows).  Gate/up tiles interleave gate and up
// rows by 16 (tile rows 32 q .. + 15: gate rows r0 + 16 q ..; the next 16:
// the up rows of the same indices).  w_last[w][s]: the last turn issued
// into each stage buffer.
__device__ __forceinline__ void stream_weights(
    StreamSmem& S, const StreamGeom& gm_, const ExpertPtrs* table, const int* u_expert,
    const int* units, CUtensorMap* maps, const CUtensorMap& tm_codes,
    const CUtensorMap& tm_scales, int lane, volatile int* abort_flag, int (&w_last)[kWG][kSW]) {
  const int nmaps = gm_.mats == 2 ? 4 : 2;
  const uint64_t stream = l2_policy_evict_first();
  for (int item = blockIdx.x, it = 0; item < gm_.items; item += gridDim.x, ++it) {
    if (!__shfl_sync(0xffffffffu, lane == 0 ? !*abort_flag : 0, 0)) break;
    const int e = u_expert[units[item / gm_.tiles]];
    const int r0 = (item % gm_.tiles) * gm_.tile_rows;
    // the item's maps go to set it % kMapSets of the CTA: a set is rewritten
    // kMapSets items later, when every load through it has landed (this
    // producer has issued at least kMapSets - 1 >= kSW stages of the items
    // between, each after the stage kSW before it was consumed)
    CUtensorMap* gm = maps + ((size_t)blockIdx.x * kMapSets + (it % kMapSets)) * kMaps;
    const ExpertPtrs ep = table[e];
    if (lane < 8 * nmaps) {  // the templates into shared memory, 16 bytes a lane
      const int j = lane >> 3, part = lane & 7;
      const CUtensorMap* src = (j & 1) ? &tm_scales : &tm_codes;
      reinterpret_cast<uint4*>(&S.tm[j])[part] = reinterpret_cast<const uint4*>(src)[part];
    }
    __syncwarp();
    if (lane == 0) {
      tmap_set_address(&S.tm[0], gm_.mats == 2 ? (const void*)ep.q_gate : (const void*)ep.q_down);
      tmap_set_address(&S.tm[1], gm_.mats == 2 ? (const void*)ep.s_gate : (const void*)ep.s_down);
      if (gm_.mats == 2) {
        tmap_set_address(&S.tm[2], ep.q_up);
        tmap_set_address(&S.tm[3], ep.s_up);
      }
    }
    __syncwarp();
    for (int j = 0; j < nmaps; ++j) tmap_publish(gm + j, &S.tm[j]);
    int ok = 1;
    if (lane == 0) {
      for (int j = 0; j < nmaps; ++j) tmap_acquire(gm + j);
      for (int j = 0; j < gm_.nst && ok; ++j) {
        for (int w = 0; w < kWG; ++w) {
          const int q = it * gm_.nst + j, sb = q % kSW, use = q / kSW;
          if (use > 0 && !stream_wait(&S.w_empty[w][sb], (uint32_t)((use - 1) & 1))) {
            *abort_flag = 1;
            ok = 0;
            break;
          }
          const int g = w * gm_.ng + j * kGS;  // first group of the stage
          uint64_t* bar = &S.w_full[w][sb];
          mbar_arrive_expect_tx(bar, kWStageBytes);
          w_last[w][sb] = use;
          if (gm_.mats == 2) {
            for (int qd = 0; qd < 4; ++qd) {
              const int y = r0 + 16 * qd;
              tma_load_2d(S.wc[w][sb] + (32 * qd) * 128, gm + 0, g * 16, y, bar, stream);
              tma_load_2d(S.wc[w][sb] + (32 * qd + 16) * 128, gm + 2, g * 16, y, bar, stream);
              tma_load_2d(S.wsc[w][sb] + (32 * qd) * 16, gm + 1, g, y, bar, stream);
              tma_load_2d(S.wsc[w][sb] + (32 * qd + 16) * 16, gm + 3, g, y, bar, stream);
            }
          } else {
            tma_load_2d(S.wc[w][sb], gm + 0, g * 16, r0, bar, stream);
            tma_load_2d(S.wsc[w][sb], gm + 1, g, r0, bar, stream);
          }
        }
      }
    }
    if (!__shfl_sync(0xffffffffu, ok, 0)) break;
  }
}

// Input producer (one thread).  The inputs of rank r start at row roff[r]
// of `pack` and take roff[r + 1] - roff[r] rows of row_bytes per ring step,
// in ring-step order, so that kBG consecutive steps are one copy into kBG
// consecutive slots of slot_bytes; ring depth kR (a multiple of kBG).
// b_last[run]: the last turn issued into each run of slots.
__device__ __forceinline__ void stream_inputs(StreamSmem& S, uint8_t* ring, const StreamGeom& gm_,
                                              const int* roff, const uint8_t* pack, int G,
                                              int row_bytes, int slot_bytes, int kR,
                                              volatile int* abort_flag,
                                              int (&b_last)[kRmax / kBG]) {
  const uint64_t keep = l2_policy_evict_last();
  RingPos pos;
  for (int item = blockIdx.x, it = 0; item < gm_.items && !*abort_flag;
       item += gridDim.x, ++it) {
    const int rank = item / gm_.tiles;
    const int r0 = roff[rank], N = roff[rank + 1] - r0;
    const uint32_t bcopy = (uint32_t)(N * row_bytes);
    const uint8_t* src = pack + (size_t)r0 * G * row_bytes;
    bool ok = true;
    for (int st = 0; st < gm_.steps && ok; st += kBG) {
      if (pos.use > 0)
        for (int s = 0; s < kBG; ++s)
          if (!stream_wait(&S.slot_free[pos.slot + s], (uint32_t)((pos.use - 1) & 1))) {
            *abort_flag = 1;
            ok = false;
            break;
          }
      if (!ok) break;
      const int run = pos.slot / kBG;  // each run of a slot turn is used once
      mbar_arrive_expect_tx(&S.b_full[run], kBG * bcopy);
      b_last[run] = pos.use;
      bulk_g2s(ring + pos.slot * slot_bytes, src + (size_t)st * bcopy, kBG * bcopy,
               &S.b_full[run], keep);
      pos.advance(kBG, kR);
    }
  }
}

// After a wait ran out, copies may still be in flight into the CTA's shared
// memory: the producers wait (bounded) for the last one they issued into
// every buffer before the CTA exits.
__device__ __forceinline__ void stream_drain(StreamSmem& S, int warp, int lane, int wprod,
                                             int bprod, int kR, const int (&w_last)[kWG][kSW],
                                             const int (&b_last)[kRmax / kBG]) {
  if (warp == wprod && lane == 0)
    for (int w = 0; w < kWG; ++w)
      for (int s = 0; s < kSW; ++s)
        if (w_last[w][s] >= 0)
          mbar_wait(&S.w_full[w][s], (uint32_t)(w_last[w][s] & 1), kStreamWaitNs);
  if (warp == bprod && lane == 0)
    for (int i = 0; i < kR / kBG; ++i)
      if (b_last[i] >= 0) mbar_wait(&S.b_full[i], (uint32_t)(b_last[i] & 1), kStreamWaitNs);
}

}  // namespace moe
