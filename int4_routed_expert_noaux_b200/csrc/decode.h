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
  kCtrlHqDone = 16,  // [slots] 32-row groups of the slot's h published as int16
  kCtrlHRows = 64,   // [slots][inter / 32] rows of h written, per 32-row group
  kCtrlWords = (int)(kCtrlBytes / 4),
};

struct DecodeParams {
  const ExpertPtrs* table;
  ExpertPtrs shared;  // the shared expert's tensors (entry E of table)
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
  float* hbuf;        // [slots][I] fp32 h
  uint8_t* hq;        // [slots][I / 32] 64-byte int16 groups of h (XQ word order)
  float* hqf;         // [slots][I / 32] their factors
  int H, I, E, k, n_group, topk_group, has_shared;
  float rsf;
  float top_p;        // adaptive expert top-p (>= 1: off); dropped slots carry id -1
  // selection layout: lane l owns experts l*sel_q .. l*sel_q+sel_q-1 and a
  // group is 2^sel_lgL consecutive lanes (sel_fast), else the generic path
  int sel_fast, sel_q, sel_lgL;
  int warm;           // consumer group 1 first runs one placeholder item of each kind
  int RR, RG, RD;     // rows per router block / gate-up item / down item
  int nR, nG;         // CTAs with router rows; gate/up items per slot
  // down rows: CTA b owns rows [A * (b * nU / grid), A * ((b + 1) * nU / grid))
  // of every slot, nU = H / A, in n_db items of at most RD rows per slot
  int A, nU, n_db, ycta_rows;
  uint64_t* trace;    // timeline probes of a -DMOE_TRACE build ([grid][128]); else unused
  // The next layer of a stack (nullable): during this layer's down phase
  // each CTA prefetches into L2 its router rows and a share of the shared
  // expert's gate/up rows, the bytes the next layer's start-up reads first.
  const float* pf_w_router;
  ExpertPtrs pf_shared;
};

// Fill the shape part of p; false if the fused kernel does not cover the
// shape (the step kernels are used instead).
bool decode_plan(const moe_config& c, DecodeParams& p);
size_t decode_smem_bytes();
cudaError_t launch_decode(const DecodeParams& p, cudaStream_t st);

}  // namespace moe
