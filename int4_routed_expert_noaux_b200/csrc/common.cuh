// common.cuh -- device helpers shared by the routed-MoE kernels (sm_100a).
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "moe.h"

namespace moe {

// Device view of one expert (same fields as moe_expert).
struct ExpertPtrs {
  const uint8_t* q_gate;
  const uint8_t* q_up;
  const uint16_t* s_gate;
  const uint16_t* s_up;
  const uint8_t* q_down;
  const uint16_t* s_down;
};

// Error codes a kernel writes into the workspace error word.
enum : uint32_t {
  kErrNone = 0,
  kErrBadExpertId = 1,
  kErrTimeout = 2,
  kErrNullExpert = 3,
};

// ---------------------------------------------------------------------------
// number formats

__device__ __forceinline__ float bf16_bits_to_f32(uint32_t b) {
  return __uint_as_float(b << 16);
}

__device__ __forceinline__ float f16_bits_to_f32(uint16_t h) {
  float f;
  asm("{ .reg .f16 t; mov.b16 t, %1; cvt.f32.f16 %0, t; }" : "=f"(f) : "h"(h));
  return f;
}

__device__ __forceinline__ uint16_t f32_to_bf16_rne(float f) {
  uint16_t r;
  asm("{ .reg .b16 t; cvt.rn.bf16.f32 t, %1; mov.b16 %0, t; }" : "=h"(r) : "f"(f));
  return r;
}

// ---------------------------------------------------------------------------
// packed fp32x2 arithmetic (sm_100 FFMA2)

__device__ __forceinline__ unsigned long long pack_f2(float lo, float hi) {
  unsigned long long r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
  return r;
}

__device__ __forceinline__ void unpack_f2(unsigned long long v, float& lo, float& hi) {
  asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
}

__device__ __forceinline__ unsigned long long pack_u2(uint32_t lo, uint32_t hi) {
  unsigned long long r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "r"(lo), "r"(hi));
  return r;
}

// d = a * b + c, element-wise on two packed floats, round to nearest.
__device__ __forceinline__ unsigned long long ffma2(unsigned long long a,
                                                    unsigned long long b,
                                                    unsigned long long c) {
  unsigned long long d;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
  return d;
}

// r = c1 ? (a ^ c2) : c2, bitwise (one LOP3: a = 0xF0, c1 = 0xCC, c2 = 0xAA
// gives the truth table 0x6A).
__device__ __forceinline__ uint32_t lop3_sel_xor(uint32_t a, uint32_t c1, uint32_t c2) {
  uint32_t r;
  asm("lop3.b32 %0, %1, %2, %3, 0x6A;" : "=r"(r) : "r"(a), "r"(c1), "r"(c2));
  return r;
}

// ---------------------------------------------------------------------------
// int4 x fp32 dot product of one 32-input scale group (16 packed bytes).
//
// A nibble n (two's complement code q) placed in bits [12,16) of the
// mantissa of 1.0f, with its top bit flipped, is the float 1 + (q+8) 2^-11;
// placed in bits [16,20) it is 1 + (q+8) 2^-7.  One LOP3 builds either
// float from a shifted copy of the packed word.  Inputs are paired so that
// each shifted word yields (odd element in [12,16), even element in
// [16,20)); a packed FMA accumulates acc = {accB, accA} over the 16 pairs of
// the group, with
//     accB0 = -(1 + 8 * 2^-11) * sum_odd x,   accA0 = -(1 + 8 * 2^-7) * sum_even x
// so that at the end  sum_k q_k x_k = 2048 * accB + 128 * accA.
//
// XGroup holds the group's 32 inputs as 16 packed pairs in the order
//   p[0] = {x31, x0},  p[m] = {x(2m-1), x(2m)} for m = 1..15,
// and init = {accB0, accA0}.
struct XGroup {
  unsigned long long p[16];
  unsigned long long init;
};

// Build the XGroup of inputs x[0..31] (given as floats).
__device__ __forceinline__ void xgroup_from_floats(const float* x, XGroup& g) {
  float so = 0.f, se = 0.f;
#pragma unroll
  for (int i = 0; i < 32; i += 2) {
    se += x[i];
    so += x[i + 1];
  }
  g.p[0] = pack_f2(x[31], x[0]);
#pragma unroll
  for (int m = 1; m < 16; ++m) g.p[m] = pack_f2(x[2 * m - 1], x[2 * m]);
  g.init = pack_f2(-1.00390625f * so, -1.0625f * se);
}

// sum_k q_k x_k for the 32 codes of one 16-byte chunk (words w0..w3).
__device__ __forceinline__ float dot_group(const uint4 w, const XGroup& g) {
  const uint32_t MB = 0x0000F000u, CB = 0x3F808000u;  // window [12,16)
  const uint32_t MA = 0x000F0000u, CA = 0x3F880000u;  // window [16,20)
  const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
  unsigned long long acc = g.init;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const uint32_t wi = ws[i];
    const uint32_t wn = ws[(i + 1) & 3];
    uint32_t s;
    // pair m = 4i+1: nibbles 1 (B) and 2 (A) of word i
    s = wi << 8;
    acc = ffma2(pack_u2(lop3_sel_xor(s, MB, CB), lop3_sel_xor(s, MA, CA)), g.p[4 * i + 1], acc);
    // pair m = 4i+2: nibbles 3 (B) and 4 (A)
    s = wi;
    acc = ffma2(pack_u2(lop3_sel_xor(s, MB, CB), lop3_sel_xor(s, MA, CA)), g.p[4 * i + 2], acc);
    // pair m = 4i+3: nibbles 5 (B) and 6 (A)
    s = wi >> 8;
    acc = ffma2(pack_u2(lop3_sel_xor(s, MB, CB), lop3_sel_xor(s, MA, CA)), g.p[4 * i + 3], acc);
    // pair m = 4i+4 (mod 16): nibble 7 of word i (B), nibble 0 of word i+1 (A)
    s = __funnelshift_r(wi, wn, 16);
    acc = ffma2(pack_u2(lop3_sel_xor(s, MB, CB), lop3_sel_xor(s, MA, CA)), g.p[(4 * i + 4) & 15], acc);
  }
  float accB, accA;
  unpack_f2(acc, accB, accA);
  return fmaf(accB, 2048.f, accA * 128.f);
}

// ---------------------------------------------------------------------------
// reductions

// Butterfly reduce-scatter of NV values across SEG lanes (SEG a power of two
// <= 32, NV a power of two <= SEG).  On return v[0] of each lane holds the
// sum over the lane's SEG-lane segment of value index reduce_index<NV,SEG>.
template <int NV, int O, int N>
__device__ __forceinline__ void reduce_scatter_stage(float (&v)[NV], int lane) {
  if constexpr (O >= 1) {
    if constexpr (N > 1) {
      constexpr int half = N / 2;
      const bool upper = (lane & O) != 0;
#pragma unroll
      for (int i = 0; i < half; ++i) {
        const float send = upper ? v[i] : v[i + half];
        const float keep = upper ? v[i + half] : v[i];
        v[i] = keep + __shfl_xor_sync(0xffffffffu, send, O);
      }
      reduce_scatter_stage<NV, O / 2, half>(v, lane);
    } else {
      v[0] += __shfl_xor_sync(0xffffffffu, v[0], O);
      reduce_scatter_stage<NV, O / 2, 1>(v, lane);
    }
  }
}

template <int NV, int SEG>
__device__ __forceinline__ void reduce_scatter(float (&v)[NV]) {
  static_assert(NV <= SEG && SEG <= 32, "bad reduce shape");
  reduce_scatter_stage<NV, SEG / 2, NV>(v, threadIdx.x & 31);
}

template <int NV, int SEG>
__device__ __forceinline__ int reduce_index(int lane) {
  int idx = 0;
#pragma unroll
  for (int o = SEG / 2, n = NV; o >= 1; o >>= 1) {
    if (n > 1) {
      const int half = n >> 1;
      if (lane & o) idx += half;
      n = half;
    }
  }
  return idx;
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

__device__ __forceinline__ float silu_mul(float g, float u) {
  return g / (1.0f + __expf(-g)) * u;
}

// ---------------------------------------------------------------------------
// column-stationary row mapping: a row of G 16-byte chunks is covered by G
// threads, one chunk column each; a CTA of NW warps covers P rows at once.
struct ColMap {
  int col;    // chunk column of this thread
  int phase;  // which of the P concurrent rows
  int P;      // concurrent rows per CTA
  int seg;    // lanes per row inside a warp (32, or G when G < 32)
  int wpr;    // warps per row (G / 32 when G >= 32, else 1)
  int wir;    // this warp's index inside its row (0..wpr-1)
};

__device__ __forceinline__ ColMap col_map_n(int G, int NW) {
  ColMap m;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (G >= 32) {
    m.wpr = G >> 5;
    m.P = NW / m.wpr;
    m.col = (warp % m.wpr) * 32 + lane;
    m.phase = warp / m.wpr;
    m.seg = 32;
    m.wir = warp % m.wpr;
  } else {
    const int rpw = 32 / G;
    m.wpr = 1;
    m.P = NW * rpw;
    m.col = lane % G;
    m.phase = warp * rpw + lane / G;
    m.seg = G;
    m.wir = 0;
  }
  return m;
}

__device__ __forceinline__ ColMap col_map(int G) { return col_map_n(G, blockDim.x >> 5); }

}  // namespace moe
