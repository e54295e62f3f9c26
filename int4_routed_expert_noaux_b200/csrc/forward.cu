// forward.cu -- launch sequences of the hot path.
#include <cuda_runtime.h>

#include "decode.h"
#include "kernels.h"
#include "layer.h"

namespace moe {

moe_status route_impl(const moe_layer* l, const uint16_t* x, int T, int32_t* idx, float* w,
                      float* scores, uint8_t* ws, const WsLayout& L, cudaStream_t st) {
  const moe_config& c = l->cfg;
  double* part = reinterpret_cast<double*>(ws + L.logits);
  cudaError_t e = launch_router_partial(l->w_router, x, T, c.hidden, c.n_experts, part, st);
  if (e == cudaSuccess)
    e = launch_select(part, c.hidden, l->bias, T, c.n_experts, c.n_group, c.topk_group,
                      c.top_k, c.routed_scaling_factor, l->top_p, idx, w, scores, st);
  return e == cudaSuccess ? MOE_OK : cuda_fail(e, "route launch");
}

moe_status ffn_impl(const moe_layer* l, const uint16_t* x, int T, const int32_t* idx,
                    const float* w, float* y, uint8_t* ws, const WsLayout& L, cudaStream_t st,
                    uint64_t slot_mask, bool combine) {
  const moe_config& c = l->cfg;
  cudaError_t e = launch_union_ffn(
      l->table, idx, w, x, T, c.hidden, c.inter, c.n_experts, c.top_k, c.n_shared, ws + L.xq,
      reinterpret_cast<float*>(ws + L.xqf), ws + L.hq, reinterpret_cast<float*>(ws + L.hqf),
      reinterpret_cast<int*>(ws + L.lists), reinterpret_cast<float*>(ws + L.hbuf),
      reinterpret_cast<float*>(ws + L.ypart), y, reinterpret_cast<uint32_t*>(ws + L.ctrl),
      L.tc_bytes ? ws + L.tc : nullptr, reinterpret_cast<int*>(ws + L.tc_exp),
      L.tc_bytes ? ws + L.tc_maps : nullptr, st, slot_mask, combine);
  return e == cudaSuccess ? MOE_OK : cuda_fail(e, "expert launch");
}

#ifdef MOE_TRACE
// Timeline buffer of a profiling build (-DMOE_TRACE): [grid][128] uint64.
static uint64_t* g_trace = nullptr;
extern "C" __attribute__((visibility("default"))) void moe_debug_set_trace(void* buf) {
  g_trace = static_cast<uint64_t*>(buf);
}
#endif

static moe_status launch_fused(const moe_layer* l, const uint16_t* x, const float* x_resid,
                               float norm_eps, uint16_t* xn_out, float* y, int32_t* idx_out,
                               float* w_out, uint8_t* ws, const WsLayout& L, cudaStream_t st,
                               bool* used, const moe_layer* next = nullptr) {
  DecodeParams p;
  *used = false;
  if (!decode_plan(l->cfg, p)) return MOE_OK;
  *used = true;
  p.table = l->table;
  p.shared = l->host_table[l->cfg.n_experts];
  p.w_router = l->w_router;
  p.bias = l->bias;
  p.x = x;
  p.x_resid = x_resid;
  p.norm_eps = norm_eps;
  p.xn_out = xn_out;
  p.y = y;
  p.idx_out = idx_out;
  p.w_out = w_out;
  p.ctrl = reinterpret_cast<uint32_t*>(ws + L.ctrl);
  p.scores = reinterpret_cast<uint64_t*>(ws + L.records);
  p.hbuf = reinterpret_cast<float*>(ws + L.hbuf);
  p.warm = 1;
  p.top_p = l->top_p;
  // the next layer of a stack, when it has this layer's shape
  const bool same = next && next->cfg.hidden == l->cfg.hidden && next->cfg.inter == l->cfg.inter &&
                    next->cfg.n_experts == l->cfg.n_experts &&
                    next->cfg.n_shared == l->cfg.n_shared;
  p.pf_w_router = same ? next->w_router : nullptr;
  p.pf_shared = same ? next->host_table[next->cfg.n_experts] : ExpertPtrs{};
#ifdef MOE_TRACE
  p.trace = g_trace;
#else
  p.trace = nullptr;
#endif
  p.hq = ws + L.hq;
  p.hqf = reinterpret_cast<float*>(ws + L.hqf);
  cudaError_t e = launch_decode(p, st);
  return e == cudaSuccess ? MOE_OK : cuda_fail(e, "decode launch");
}

moe_status forward_impl(const moe_layer* l, const uint16_t* x, int T, float* y, int32_t* idx_out,
                        float* w_out, uint8_t* ws, const WsLayout& L, cudaStream_t st) {
  if (T == 1) {
    bool used = false;
    moe_status s = launch_fused(l, x, nullptr, 0.f, nullptr, y, idx_out, w_out, ws, L, st, &used);
    if (used || s != MOE_OK) return s;
  }
  int32_t* idx = idx_out ? idx_out : reinterpret_cast<int32_t*>(ws + L.idx);
  float* w = w_out ? w_out : reinterpret_cast<float*>(ws + L.w);
  moe_status s = route_impl(l, x, T, idx, w, nullptr, ws, L, st);
  if (s != MOE_OK) return s;
  return ffn_impl(l, x, T, idx, w, y, ws, L, st);
}

moe_status residual_impl(const moe_layer* l, const float* x_resid, float norm_eps, float* x_next,
                         uint16_t* xn_out, int32_t* idx_out, float* w_out, uint8_t* ws,
                         const WsLayout& L, cudaStream_t st, const moe_layer* next) {
  bool used = false;
  moe_status s = launch_fused(l, nullptr, x_resid, norm_eps, xn_out, x_next, idx_out, w_out, ws,
                              L, st, &used, next);
  if (s != MOE_OK) return s;
  if (!used) return fail(MOE_ERR_UNSUPPORTED, "the pre-norm step needs the fused decode kernel's shapes");
  return MOE_OK;
}

}  // namespace moe
