// kernels.h -- launchers of the step kernels (kernels.cu) and of the fused
// decode kernel (decode.cu).
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "common.cuh"

namespace moe {

cudaError_t launch_router_logits(const float* w, const uint16_t* x, int T, int H, int E,
                                 float* logits, cudaStream_t st);
cudaError_t launch_select(const float* logits, const float* bias, int T, int E, int n_group,
                          int topk_group, int top_k, float rsf, int32_t* idx, float* w,
                          float* scores, cudaStream_t st);
cudaError_t launch_gate_up(const ExpertPtrs* table, const int32_t* idx, int E, int top_k,
                           int slots, const uint16_t* x, int T, int H, int I, float* hbuf,
                           uint32_t* err, cudaStream_t st);
cudaError_t launch_down_combine(const ExpertPtrs* table, const int32_t* idx, const float* w,
                                int E, int top_k, int slots, const float* hbuf, int T, int H,
                                int I, float* y, uint32_t* err, cudaStream_t st);

cudaError_t launch_gemv_int4(const uint8_t* q, const uint16_t* s, int rows, int cols,
                             const float* x, float* y, cudaStream_t st);

}  // namespace moe
