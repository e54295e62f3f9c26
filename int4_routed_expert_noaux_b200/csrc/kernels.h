// kernels.h -- launchers of the step kernels (kernels.cu: router, selection,
// test GEMV) and of the batched expert path (union.cu).
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "common.cuh"

namespace moe {

// scores [T][E] = fp32(sigmoid(W x)), the logit summed in fp64.
cudaError_t launch_router_scores(const float* w, const uint16_t* x, int T, int H, int E,
                                 float* scores, cudaStream_t st);
// noaux_tc selection from the sigmoid scores, then adaptive top-p when
// top_p < 1 (dropped slots: id -1, weight 0, after the kept ids);
// scores_out (nullable) gets a copy of the scores.
cudaError_t launch_select(const float* scores, const float* bias, int T, int E, int n_group,
                          int topk_group, int top_k, float rsf, float top_p, int32_t* idx,
                          float* w, float* scores_out, cudaStream_t st);
// The batched expert path (union.cu): distinct experts read once for all
// their tokens.  Scratch: xq (T * H/32 groups), hq (T * slots * I/32 groups),
// lists (union_lists_ints ints), hbuf (T * slots * I), ypart (T * slots * H).
size_t union_lists_ints(int T, int k, int E, int has_shared);
cudaError_t launch_union_ffn(const ExpertPtrs* table, const int32_t* idx, const float* w,
                             const uint16_t* x, int T, int H, int I, int E, int k, int has_shared,
                             uint8_t* xq_words, float* xq_fac, uint8_t* hq_words, float* hq_fac,
                             int* lists, float* hbuf, float* ypart, float* y, uint32_t* err,
                             cudaStream_t st);

cudaError_t launch_gemv_int4(const uint8_t* q, const uint16_t* s, int rows, int cols,
                             const float* x, float* y, cudaStream_t st);

}  // namespace moe
