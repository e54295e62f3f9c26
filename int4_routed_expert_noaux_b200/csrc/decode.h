// decode.h -- the fused persistent decode kernel (one launch per token).
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "common.cuh"
#include "moe.h"

namespace moe {

// Control words at the start of a workspace (uint32 indices).  Word 0 is the
// error word the host reads.  The counters of the fused kernel are zero
// between calls; the epoch word counts the kernel's calls on this workspace
// (router score records carry the epoch of the call that wrote them).
constexpr size_t kCtrlBytes = 4096;
enum : int {
  kCtrlErr = 0,
  kCtrlTicket = 1,
  kCtrlEpoch = 2,
  kCtrlExit = 4,
  kCtrlAbort = 5,
  kCtrlWhere = 8,    // [4] where the first error happened (CTA, warp, site, fill)
  kCtrlGuDone = 16,  // [slots] finished gate/up finalizer warps of the slot
  kCtrlRbDone = 64,  // [row blocks of hidden] finished down finalizer warps
  kCtrlWords = (int)(kCtrlBytes / 4),
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
  uint64_t* scores;   // [E]: (epoch << 32) | bits of sigmoid(logit), per expert
  float* hbuf;        // [slots][I]
  float* ypart;       // [slots][H]
  int H, I, E, k, n_group, topk_group, has_shared;
  float rsf;
  // selection layout: lane l owns experts l*sel_q .. l*sel_q+sel_q-1 and a
  // group is 2^sel_lgL consecutive lanes (sel_fast), else the generic path
  int sel_fast, sel_q, sel_lgL;
  int warm;           // consumer group 1 first runs one placeholder item of each kind
  int RR, RG, RD;     // rows per router block / gate-up item / down item
  int gu_count;       // finalizer-warp arrivals that complete one slot's h
  int nR, nG, nD, n_items;
};

// Fill the shape part of p; false if the fused kernel does not cover the
// shape (the step kernels are used instead).
bool decode_plan(const moe_config& c, DecodeParams& p);
size_t decode_smem_bytes();
cudaError_t launch_decode(const DecodeParams& p, cudaStream_t st);

}  // namespace moe
