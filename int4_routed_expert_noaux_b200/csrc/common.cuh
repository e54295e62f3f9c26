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
// int4 dot product of one 32-input scale group (16 packed bytes), exact in
// integers.
//
// The group's 32 inputs x_k are held as int16 X_k = round(x_k * 2^e) with
// one power-of-two exponent e per group, chosen so that the largest input
// maps into [2^14, 2^15) (clamped to 32767): exact for every bf16 input
// within 2^7 of the group's largest; otherwise the representation error is
// at most 2^-15 of the group's largest input.
// A packed word w holds codes q_{8i..8i+7} (nibble j = element 8i + j,
// two's complement).  The bytes of (w & 0xF0F0F0F0), read as signed int8,
// are exactly 16 * q of the odd elements; those of ((w << 4) & 0xF0F0F0F0)
// are 16 * q of the even elements.  dp2a multiplies two int16 by two int8
// and accumulates in int32, so four dp2a per word give 16 * sum q_k X_k with
// no rounding (|sum| < 2^28 and a multiple of 16: the int32 -> fp32
// conversion is exact too).  sum_k q_k x_k = that * 2^-e / 16.
//
// XQ holds the int16 pairs in dp2a order: for word i,
//   ev[2i] = (X_{8i}, X_{8i+2})    ev[2i+1] = (X_{8i+4}, X_{8i+6})
//   od[2i] = (X_{8i+1}, X_{8i+3})  od[2i+1] = (X_{8i+5}, X_{8i+7})
// and f = 2^-e / 16.
struct XQ {
  uint32_t ev[8];
  uint32_t od[8];
  float f;
};

__device__ __forceinline__ uint32_t pack_i16x2(int lo, int hi) {
  return (uint32_t)(lo & 0xFFFF) | ((uint32_t)hi << 16);
}

// Quantise 32 floats to an XQ (shared power-of-two exponent, RNE).
__device__ __forceinline__ void xq_from_floats(const float* x, XQ& g) {
  float m = 0.f;
#pragma unroll
  for (int i = 0; i < 32; ++i) m = fmaxf(m, fabsf(x[i]));
  int ex = 0;
  if (m > 0.f) frexpf(m, &ex);  // m = fr * 2^ex, fr in [0.5, 1)
  const int e = 15 - ex;        // m * 2^e in [2^14, 2^15)
  const float sc = (m > 0.f) ? ldexpf(1.0f, e) : 0.f;
  g.f = (m > 0.f) ? ldexpf(1.0f, -e - 4) : 0.f;
  // round to nearest even with the 1.5 * 2^23 bias: |x * sc| < 2^15, so the
  // biased float holds the rounded integer in its low mantissa bits
  int X[32];
#pragma unroll
  for (int i = 0; i < 32; ++i) {
    const float b = fmaf(x[i], sc, 12582912.0f);
    X[i] = max(-32767, min(32767, (int)(__float_as_uint(b) - 0x4B400000u)));
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    g.ev[2 * i] = pack_i16x2(X[8 * i + 0], X[8 * i + 2]);
    g.ev[2 * i + 1] = pack_i16x2(X[8 * i + 4], X[8 * i + 6]);
    g.od[2 * i] = pack_i16x2(X[8 * i + 1], X[8 * i + 3]);
    g.od[2 * i + 1] = pack_i16x2(X[8 * i + 5], X[8 * i + 7]);
  }
}

__device__ __forceinline__ int dp2a_lo(uint32_t a, uint32_t b, int c) {
  int d;
  asm("dp2a.lo.s32.s32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
  return d;
}

__device__ __forceinline__ int dp2a_hi(uint32_t a, uint32_t b, int c) {
  int d;
  asm("dp2a.hi.s32.s32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
  return d;
}

// 16 * sum_k q_k X_k over the 32 codes of one 16-byte chunk (four
// independent dp2a chains of four).
__device__ __forceinline__ int dotq_group(const uint4 w, const XQ& g) {
  const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
  int a0 = 0, a1 = 0, a2 = 0, a3 = 0;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const uint32_t odd = ws[i] & 0xF0F0F0F0u;
    const uint32_t even = (ws[i] << 4) & 0xF0F0F0F0u;
    a0 = dp2a_lo(g.ev[2 * i], even, a0);
    a1 = dp2a_hi(g.ev[2 * i + 1], even, a1);
    a2 = dp2a_lo(g.od[2 * i], odd, a2);
    a3 = dp2a_hi(g.od[2 * i + 1], odd, a3);
  }
  return (a0 + a1) + (a2 + a3);
}

// dotq_group with the chunk's words already split into even-element and
// odd-element bytes (16 * q), for a chunk used against several inputs.
__device__ __forceinline__ void split_chunk(const uint4 w, uint32_t (&even)[4], uint32_t (&odd)[4]) {
  const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    odd[i] = ws[i] & 0xF0F0F0F0u;
    even[i] = (ws[i] << 4) & 0xF0F0F0F0u;
  }
}

__device__ __forceinline__ int dotq_group_split(const uint32_t (&even)[4], const uint32_t (&odd)[4],
                                                const XQ& g) {
  int a0 = 0, a1 = 0, a2 = 0, a3 = 0;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    a0 = dp2a_lo(g.ev[2 * i], even[i], a0);
    a1 = dp2a_hi(g.ev[2 * i + 1], even[i], a1);
    a2 = dp2a_lo(g.od[2 * i], odd[i], a2);
    a3 = dp2a_hi(g.od[2 * i + 1], odd[i], a3);
  }
  return (a0 + a1) + (a2 + a3);
}

// sum_k (q_k * scale) x_k for one chunk: exact group sum, one rounding.
__device__ __forceinline__ float dot_scaled(const uint4 w, const XQ& g, float scale) {
  return (float)dotq_group(w, g) * (scale * g.f);
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

// Double-float value hi + lo (|lo| <= half an ulp of hi, about 48 bits).
struct DF {
  float hi, lo;
};

// a += w * x with no rounding error lost: the product splits exactly into
// p + e (e = fma(w, x, -p)), p is added to hi error-free (TwoSum), and the
// two error terms go to lo.  The _rn intrinsics keep the compiler from
// contracting the adds into fmas, which would break the error terms.
__device__ __forceinline__ void df_add_prod(DF& a, float w, float x) {
  const float p = __fmul_rn(w, x);
  const float e = fmaf(w, x, -p);
  const float s = __fadd_rn(a.hi, p);
  const float bp = __fsub_rn(s, a.hi);
  const float err = __fadd_rn(__fsub_rn(a.hi, __fsub_rn(s, bp)), __fsub_rn(p, bp));
  a.hi = s;
  a.lo = __fadd_rn(a.lo, __fadd_rn(err, e));
}

__device__ __forceinline__ DF df_add(DF a, DF b) {
  const float s = __fadd_rn(a.hi, b.hi);
  const float bp = __fsub_rn(s, a.hi);
  const float err = __fadd_rn(__fsub_rn(a.hi, __fsub_rn(s, bp)), __fsub_rn(b.hi, bp));
  return DF{s, __fadd_rn(__fadd_rn(a.lo, b.lo), err)};
}

__device__ __forceinline__ DF df_warp_sum(DF v) {
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) {
    DF u;
    u.hi = __shfl_xor_sync(0xffffffffu, v.hi, o);
    u.lo = __shfl_xor_sync(0xffffffffu, v.lo, o);
    v = df_add(v, u);
  }
  return v;
}

__device__ __forceinline__ double warp_sum_f64(double v) {
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// sigmoid of an fp64 logit, taken in fp64 and rounded to fp32 once.
__device__ __forceinline__ float sigmoid_f64_to_f32(double v) {
  return (float)(1.0 / (1.0 + exp(-v)));
}

// Adaptive expert top-p over one warp's k picks (lane < k holds a picked
// id and its unbiased score s; denom = the sum of the k scores).  A pick is
// kept when the weight share of the picks ranked before it (descending
// score, ties to the lower id) is below p: the kept picks are the shortest
// weight-ordered prefix whose share reaches p (colibri summary, "--topp":
// adaptive expert top-p; the page gives no formula, so this rule is our
// plainest reading of it).
__device__ __forceinline__ bool topp_keep(int id, float s, float denom, int k, float p) {
  const int lane = threadIdx.x & 31;
  float before = 0.f;
#pragma unroll 4
  for (int j = 0; j < 32; ++j) {
    const float sj = __shfl_sync(0xffffffffu, s, j);
    const int ij = __shfl_sync(0xffffffffu, id, j);
    const bool ahead = j < k && (sj > s || (sj == s && ij < id));
    before += ahead ? sj / denom : 0.f;
  }
  return lane < k && (p >= 1.f || before < p);
}

// Output position of a pick after top-p: the kept ids ascending first, the
// dropped picks after them in lane order.
__device__ __forceinline__ int topp_position(int id, bool kept, int k) {
  const int lane = threadIdx.x & 31;
  const unsigned km = __ballot_sync(0xffffffffu, kept);
  int pos = 0;
#pragma unroll
  for (int j = 0; j < 32; ++j) {
    const int ij = __shfl_sync(0xffffffffu, id, j);
    const bool kj = (km >> j) & 1u;
    if (j < k) pos += kept ? (kj && ij < id) : (kj || j < lane);
  }
  return pos;
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
