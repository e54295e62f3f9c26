// decode.h -- the fused persistent decode kernel (one launch per token).
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "common.cuh"
#include "moe.h"

namespace moe {

// Control words at the start of a workspace (uint32 indices).  Word 0 is the
// error word the host reads; the rest are counters of the fused kernel,
// zero between calls.
constexpr size_t kCtrlBytes = 4096;
enum : int {
  kCtrlErr = 0,
  kCtrlTicket = 1,
  kCtrlRouterDone = 2,
  kCtrlSelReady = 3,
  kCtrlExit = 4,
  kCtrlAbort = 5,
  kCtrlWhere = 8,     // [4] where the first error happened (CTA, warp, site, fill)
  kCtrlGuDone = 16,   // [slots] finished gate/up finalizer warps
  kCtrlHqReady = 56,  // [slots] the slot's int16 h table is published
  kCtrlRbDone = 96,   // [row blocks of hidden] finished down finalizer warps
};

struct DecodeParams {
  const ExpertPtrs* table;
  const float* w_router;
  const float* bias;
  const uint16_t* x;  // bf16 [H] (plain step), or
  const float* x_resid;  // fp32 [H] residual stream (pre-norm step), nullable
  float norm_eps;     // RMSNorm epsilon of the pre-norm step
  uint16_t* xn_out;   // bf16 [H] normalised input of the pre-norm step, nullable
  float* y;           // fp32 [H]: MoE(x), or x_resid + MoE(bf16(RMSNorm(x_resid)))
  int32_t* idx_out;   // nullable
  float* w_out;       // nullable
  uint32_t* ctrl;
  float* logits;      // [E]
  int32_t* idx_ws;    // [k]
  float* w_ws;        // [k]
  float* hbuf;        // [slots][I]
  float* ypart;       // [slots][H]
  uint32_t* hq;       // [slots][I/32 * 68 bytes]: int16 h groups, then factors
  int H, I, E, k, n_group, topk_group, has_shared;
  float rsf;
  int RR, RG, RD;     // rows per router block / gate-up / down item
  int nR, nG, nD, n_items;
};

// Fill the shape part of p; false if the fused kernel does not cover the
// shape (the step kernels are used instead).
bool decode_plan(const moe_config& c, DecodeParams& p);
size_t decode_smem_bytes();
cudaError_t launch_decode(const DecodeParams& p, cudaStream_t st);

}  // namespace moe
