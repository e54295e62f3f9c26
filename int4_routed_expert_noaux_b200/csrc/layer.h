// layer.h -- host-side layer view, workspace layout and the launch
// sequences shared by the C ABI entry points.
#pragma once

#include <cuda_runtime.h>
#include <stdarg.h>
#include <stdint.h>

#include "common.cuh"
#include "decode.h"
#include "moe.h"

struct moe_layer {
  moe_config cfg;
  const float* w_router = nullptr;   // device fp32 [E][H]
  const float* bias = nullptr;       // device fp32 [E]
  moe::ExpertPtrs* table = nullptr;  // device [E + 1]; entry E = shared
  moe::ExpertPtrs* host_table = nullptr;
  int device = 0;
  float top_p = 1.0f;                // adaptive expert top-p (>= 1: off)
};

namespace moe {

constexpr int kMaxTokens = 64;

// Byte offsets inside a workspace.
struct WsLayout {
  size_t ctrl, records, logits, idx, w, hbuf, ypart, xq, xqf, hq, hqf, lists, tc, tc_bytes, tc_exp,
      tc_maps, total;
};

WsLayout ws_layout(const moe_config* c, int T);
moe_status fail(moe_status s, const char* fmt, ...);
moe_status cuda_fail(cudaError_t e, const char* what);
void clear_last_error();
moe_status check_config(const moe_config* c);
moe_status check_expert(const moe_expert* e, const char* what);
moe_status check_device_ptr(const void* p, size_t align, const char* name);
ExpertPtrs to_ptrs(const moe_expert& e);

moe_status route_impl(const moe_layer* l, const uint16_t* x, int T, int32_t* idx, float* w,
                      float* scores, uint8_t* ws, const WsLayout& L, cudaStream_t st);
moe_status ffn_impl(const moe_layer* l, const uint16_t* x, int T, const int32_t* idx,
                    const float* w, float* y, uint8_t* ws, const WsLayout& L, cudaStream_t st,
                    uint64_t slot_mask = ~0ull, bool combine = true);
// next (nullable): the layer that runs after this one (a stack), whose
// first bytes this layer's kernel prefetches into L2.
moe_status residual_impl(const moe_layer* l, const float* x_resid, float norm_eps, float* x_next,
                         uint16_t* xn_out, int32_t* idx_out, float* w_out, uint8_t* ws,
                         const WsLayout& L, cudaStream_t st, const moe_layer* next = nullptr);
moe_status forward_impl(const moe_layer* l, const uint16_t* x, int T, float* y, int32_t* idx_out,
                        float* w_out, uint8_t* ws, const WsLayout& L, cudaStream_t st);

}  // namespace moe
