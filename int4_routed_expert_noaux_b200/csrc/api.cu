// api.cu -- the C ABI of include/moe.h: argument checks, layer views,
// workspace layout and the launch sequences of the hot path.
#include <cuda_runtime.h>
#include <stdint.h>
#include <stdio.h>
#include <string.h>

#include <new>

#include "common.cuh"
#include "kernels.h"
#include "layer.h"
#include "moe.h"

namespace moe {

static thread_local char g_last_error[512] = "";

moe_status fail(moe_status s, const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_last_error, sizeof(g_last_error), fmt, ap);
  va_end(ap);
  return s;
}

void clear_last_error() { g_last_error[0] = 0; }

moe_status cuda_fail(cudaError_t e, const char* what) {
  return fail(e == cudaErrorMemoryAllocation ? MOE_ERR_OOM : MOE_ERR_CUDA, "%s: %s", what,
              cudaGetErrorString(e));
}

static bool chunk_cols_ok(int n) {
  if (n <= 0 || n % 32) return false;
  const int G = n / 32;
  if (G < 32) return G == 2 || G == 4 || G == 8 || G == 16;
  return G % 32 == 0 && G <= 256;
}

moe_status check_config(const moe_config* c) {
  if (!c) return fail(MOE_ERR_INVALID_ARG, "config is NULL");
  if (c->group_size != 32) return fail(MOE_ERR_UNSUPPORTED, "group_size must be 32");
  if (!chunk_cols_ok(c->hidden))
    return fail(MOE_ERR_UNSUPPORTED, "hidden %d: hidden/32 must be 2, 4, 8, 16 or a multiple of 32 up to 256", c->hidden);
  if (!chunk_cols_ok(c->inter))
    return fail(MOE_ERR_UNSUPPORTED, "inter %d: inter/32 must be 2, 4, 8, 16 or a multiple of 32 up to 256", c->inter);
  if (c->n_experts <= 0 || c->n_experts > 1024)
    return fail(MOE_ERR_UNSUPPORTED, "n_experts %d outside 1..1024", c->n_experts);
  if (c->n_group <= 0 || c->n_group > 32 || c->n_experts % c->n_group)
    return fail(MOE_ERR_UNSUPPORTED, "n_group %d must divide n_experts and be <= 32", c->n_group);
  const int per = c->n_experts / c->n_group;
  if (per > 32) return fail(MOE_ERR_UNSUPPORTED, "n_experts / n_group = %d > 32", per);
  if (c->topk_group < 1 || c->topk_group > c->n_group)
    return fail(MOE_ERR_INVALID_ARG, "topk_group %d outside 1..n_group", c->topk_group);
  if (c->top_k < 1 || c->top_k > 32 || c->top_k > c->topk_group * per)
    return fail(MOE_ERR_INVALID_ARG, "top_k %d outside 1..min(32, topk_group * group size)", c->top_k);
  if (c->n_shared != 0 && c->n_shared != 1)
    return fail(MOE_ERR_UNSUPPORTED, "n_shared must be 0 or 1");
  if (!(c->routed_scaling_factor > 0.f))
    return fail(MOE_ERR_INVALID_ARG, "routed_scaling_factor must be > 0");
  return MOE_OK;
}

moe_status check_device_ptr(const void* p, size_t align, const char* name) {
  if (!p) return fail(MOE_ERR_INVALID_ARG, "%s is NULL", name);
  if (reinterpret_cast<uintptr_t>(p) % align)
    return fail(MOE_ERR_INVALID_ARG, "%s is not %zu-byte aligned", name, align);
  cudaPointerAttributes a;
  cudaError_t e = cudaPointerGetAttributes(&a, p);
  if (e != cudaSuccess) {
    cudaGetLastError();
    return fail(MOE_ERR_INVALID_ARG, "%s: not a CUDA pointer (%s)", name, cudaGetErrorString(e));
  }
  if (a.type != cudaMemoryTypeDevice && a.type != cudaMemoryTypeManaged)
    return fail(MOE_ERR_INVALID_ARG, "%s is not device memory", name);
  return MOE_OK;
}

moe_status check_expert(const moe_expert* e, const char* what) {
  char name[96];
  const void* ptrs[6] = {e->q_gate, e->q_up, e->s_gate, e->s_up, e->q_down, e->s_down};
  const char* names[6] = {"q_gate", "q_up", "s_gate", "s_up", "q_down", "s_down"};
  for (int i = 0; i < 6; ++i) {
    snprintf(name, sizeof(name), "%s.%s", what, names[i]);
    moe_status s = check_device_ptr(ptrs[i], 16, name);
    if (s != MOE_OK) return s;
  }
  return MOE_OK;
}

ExpertPtrs to_ptrs(const moe_expert& e) {
  return ExpertPtrs{e.q_gate, e.q_up, e.s_gate, e.s_up, e.q_down, e.s_down};
}

static size_t align_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

WsLayout ws_layout(const moe_config* c, int T) {
  WsLayout L;
  const int k = c->top_k, slots = k + c->n_shared;
  size_t off = 0;
  L.ctrl = off;
  off += kCtrlBytes;
  // the fused one-token kernel's epoch-tagged router score records, kept
  // from call to call: a region that no other call writes
  L.records = off;
  off = align_up(off + (size_t)c->n_experts * 8, 256);
  // fp64 router logits of the step kernels, in K slices
  L.logits = off;
  off = align_up(off + (size_t)kRouterMaxSlices * T * c->n_experts * 8, 256);
  L.idx = off;
  off = align_up(off + (size_t)T * k * 4, 256);
  L.w = off;
  off = align_up(off + (size_t)T * k * 4, 256);
  L.hbuf = off;
  off = align_up(off + (size_t)T * slots * c->inter * 4, 256);
  L.ypart = off;
  off = align_up(off + (size_t)T * slots * c->hidden * 4, 256);
  // batched path: int16 groups of x and of h, per-expert token lists
  L.xq = off;
  off = align_up(off + (size_t)T * (c->hidden / 32) * 64, 256);
  L.xqf = off;
  off = align_up(off + (size_t)T * (c->hidden / 32) * 4, 256);
  L.hq = off;
  off = align_up(off + (size_t)T * slots * (c->inter / 32) * 64, 256);
  L.hqf = off;
  off = align_up(off + (size_t)T * slots * (c->inter / 32) * 4, 256);
  L.lists = off;
  off = align_up(off + union_lists_ints(T, k, c->n_experts, c->n_shared) * 4, 256);
  // packed inputs and tensor-map slots of the tensor-core path
  L.tc = off;
  L.tc_bytes = tc_bpack_bytes(T, k, c->n_shared, c->hidden, c->inter);
  off = align_up(off + L.tc_bytes, 256);
  L.tc_exp = off;
  if (L.tc_bytes) off = align_up(off + tc_rowexp_ints(T, k, c->n_shared) * 4, 256);
  L.tc_maps = off;
  if (L.tc_bytes) off = align_up(off + tc_maps_bytes(), 256);
  L.total = off;
  return L;
}

moe_status check_ws(const moe_layer* l, int T, void* ws, size_t ws_bytes, WsLayout* L) {
  *L = ws_layout(&l->cfg, T);
  if (!ws) return fail(MOE_ERR_INVALID_ARG, "workspace is NULL");
  if (reinterpret_cast<uintptr_t>(ws) % 256)
    return fail(MOE_ERR_INVALID_ARG, "workspace is not 256-byte aligned");
  if (ws_bytes < L->total)
    return fail(MOE_ERR_INVALID_ARG, "workspace has %zu bytes, needs %zu", ws_bytes, L->total);
  return MOE_OK;
}

static moe_status check_residual_args(const moe_layer* l, const float* x_dev,
                                      const float* x_next_dev, const uint16_t* xn_out_dev,
                                      const int32_t* idx_out_dev, const float* w_out_dev,
                                      float norm_eps) {
  if (!l) return fail(MOE_ERR_INVALID_ARG, "layer is NULL");
  moe_status s;
  if ((s = check_device_ptr(x_dev, 16, "x")) != MOE_OK) return s;
  if ((s = check_device_ptr(x_next_dev, 16, "x_next")) != MOE_OK) return s;
  if (x_dev == x_next_dev) return fail(MOE_ERR_INVALID_ARG, "x and x_next must not alias");
  if (xn_out_dev && (s = check_device_ptr(xn_out_dev, 4, "xn_out")) != MOE_OK) return s;
  if (idx_out_dev && (s = check_device_ptr(idx_out_dev, 4, "idx_out")) != MOE_OK) return s;
  if (w_out_dev && (s = check_device_ptr(w_out_dev, 4, "w_out")) != MOE_OK) return s;
  if (!(norm_eps >= 0.f)) return fail(MOE_ERR_INVALID_ARG, "norm_eps must be >= 0");
  return MOE_OK;
}

static moe_status check_call(const moe_layer* l, const void* x, int T) {
  if (!l) return fail(MOE_ERR_INVALID_ARG, "layer is NULL");
  if (T < 1 || T > kMaxTokens) return fail(MOE_ERR_INVALID_ARG, "T = %d outside 1..%d", T, kMaxTokens);
  return check_device_ptr(x, 16, "x");
}

}  // namespace moe

using namespace moe;

extern "C" {
#pragma GCC visibility push(default)

const char* moe_status_string(moe_status s) {
  switch (s) {
    case MOE_OK: return "ok";
    case MOE_ERR_INVALID_ARG: return "invalid argument";
    case MOE_ERR_CUDA: return "CUDA error";
    case MOE_ERR_OOM: return "out of memory";
    case MOE_ERR_TIMEOUT: return "timeout";
    case MOE_ERR_UNSUPPORTED: return "unsupported shape";
    case MOE_ERR_DEVICE: return "device-side error";
  }
  return "unknown status";
}

const char* moe_last_error(void) { return g_last_error; }

moe_status moe_layer_create(const moe_config* cfg, const float* w_router_dev,
                            const float* bias_dev, const moe_expert* experts_host,
                            const moe_expert* shared_host, moe_layer** out) {
  g_last_error[0] = 0;
  if (!out) return fail(MOE_ERR_INVALID_ARG, "out is NULL");
  *out = nullptr;
  moe_status s = check_config(cfg);
  if (s != MOE_OK) return s;
  if ((s = check_device_ptr(w_router_dev, 16, "w_router")) != MOE_OK) return s;
  if ((s = check_device_ptr(bias_dev, 4, "bias")) != MOE_OK) return s;
  if (!experts_host) return fail(MOE_ERR_INVALID_ARG, "experts is NULL");
  if ((cfg->n_shared == 1) != (shared_host != nullptr))
    return fail(MOE_ERR_INVALID_ARG, "shared expert must be given iff n_shared == 1");
  char what[32];
  for (int e = 0; e < cfg->n_experts; ++e) {
    snprintf(what, sizeof(what), "experts[%d]", e);
    if ((s = check_expert(&experts_host[e], what)) != MOE_OK) return s;
  }
  if (shared_host && (s = check_expert(shared_host, "shared")) != MOE_OK) return s;

  moe_layer* l = new (std::nothrow) moe_layer();
  if (!l) return fail(MOE_ERR_OOM, "host allocation failed");
  l->cfg = *cfg;
  l->w_router = w_router_dev;
  l->bias = bias_dev;
  const int n = cfg->n_experts + 1;
  l->host_table = new (std::nothrow) ExpertPtrs[n];
  if (!l->host_table) {
    delete l;
    return fail(MOE_ERR_OOM, "host allocation failed");
  }
  for (int e = 0; e < cfg->n_experts; ++e) l->host_table[e] = to_ptrs(experts_host[e]);
  l->host_table[cfg->n_experts] = shared_host ? to_ptrs(*shared_host) : ExpertPtrs{};
  cudaError_t ce = cudaGetDevice(&l->device);
  if (ce == cudaSuccess) ce = cudaMalloc(&l->table, sizeof(ExpertPtrs) * n);
  if (ce == cudaSuccess)
    ce = cudaMemcpy(l->table, l->host_table, sizeof(ExpertPtrs) * n, cudaMemcpyHostToDevice);
  if (ce != cudaSuccess) {
    s = cuda_fail(ce, "moe_layer_create");
    moe_layer_destroy(l);
    return s;
  }
  *out = l;
  return MOE_OK;
}

void moe_layer_destroy(moe_layer* l) {
  if (!l) return;
  if (l->table) cudaFree(l->table);
  delete[] l->host_table;
  delete l;
}

moe_status moe_layer_set_expert(moe_layer* l, int e, const moe_expert* ex, void* stream) {
  if (!l || !ex) return fail(MOE_ERR_INVALID_ARG, "layer or expert is NULL");
  if (e < 0 || e >= l->cfg.n_experts) return fail(MOE_ERR_INVALID_ARG, "expert id %d out of range", e);
  moe_status s = check_expert(ex, "expert");
  if (s != MOE_OK) return s;
  l->host_table[e] = to_ptrs(*ex);
  // The host copy is pageable: cudaMemcpyAsync stages it before returning.
  cudaError_t ce = cudaMemcpyAsync(l->table + e, &l->host_table[e], sizeof(ExpertPtrs),
                                   cudaMemcpyHostToDevice, (cudaStream_t)stream);
  return ce == cudaSuccess ? MOE_OK : cuda_fail(ce, "moe_layer_set_expert");
}

moe_status moe_layer_set_top_p(moe_layer* l, float p) {
  if (!l) return fail(MOE_ERR_INVALID_ARG, "layer is NULL");
  if (!(p > 0.f)) return fail(MOE_ERR_INVALID_ARG, "top_p must be > 0 (>= 1 turns it off)");
  l->top_p = p >= 1.f ? 1.f : p;
  return MOE_OK;
}

size_t moe_workspace_bytes(const moe_config* cfg, int T) {
  if (check_config(cfg) != MOE_OK || T < 1 || T > kMaxTokens) return 0;
  return ws_layout(cfg, T).total;
}

moe_status moe_ws_check(void* ws, size_t ws_bytes, void* stream) {
  if (!ws || ws_bytes < kCtrlBytes) return fail(MOE_ERR_INVALID_ARG, "bad workspace");
  cudaError_t ce = cudaStreamSynchronize((cudaStream_t)stream);
  if (ce != cudaSuccess) return cuda_fail(ce, "moe_ws_check");
  uint32_t word = 0;
  ce = cudaMemcpy(&word, ws, sizeof(word), cudaMemcpyDeviceToHost);
  if (ce != cudaSuccess) return cuda_fail(ce, "moe_ws_check");
  if (word == kErrNone) return MOE_OK;
  const uint32_t zero = 0;
  cudaMemcpy(ws, &zero, sizeof(zero), cudaMemcpyHostToDevice);
  if (word == kErrTimeout) return fail(MOE_ERR_TIMEOUT, "a device-side wait ran out");
  return fail(MOE_ERR_DEVICE, "device error word %u (%s)", word,
              word == kErrBadExpertId ? "expert id out of range" : "internal");
}

moe_status moe_route(const moe_layer* l, const void* x, int T, int32_t* idx, float* w,
                     float* scores, void* ws, size_t ws_bytes, void* stream) {
  g_last_error[0] = 0;
  moe_status s = check_call(l, x, T);
  if (s != MOE_OK) return s;
  if ((s = check_device_ptr(idx, 4, "idx")) != MOE_OK) return s;
  if ((s = check_device_ptr(w, 4, "w")) != MOE_OK) return s;
  if (scores && (s = check_device_ptr(scores, 4, "scores")) != MOE_OK) return s;
  WsLayout L;
  if ((s = check_ws(l, T, ws, ws_bytes, &L)) != MOE_OK) return s;
  return route_impl(l, (const uint16_t*)x, T, idx, w, scores, (uint8_t*)ws, L,
                    (cudaStream_t)stream);
}

moe_status moe_expert_ffn(const moe_layer* l, const void* x, int T, const int32_t* idx,
                          const float* w, float* y, void* ws, size_t ws_bytes, void* stream) {
  g_last_error[0] = 0;
  moe_status s = check_call(l, x, T);
  if (s != MOE_OK) return s;
  if ((s = check_device_ptr(idx, 4, "idx")) != MOE_OK) return s;
  if ((s = check_device_ptr(w, 4, "w")) != MOE_OK) return s;
  if ((s = check_device_ptr(y, 16, "y")) != MOE_OK) return s;
  WsLayout L;
  if ((s = check_ws(l, T, ws, ws_bytes, &L)) != MOE_OK) return s;
  return ffn_impl(l, (const uint16_t*)x, T, idx, w, y, (uint8_t*)ws, L, (cudaStream_t)stream);
}

moe_status moe_expert_ffn_part(const moe_layer* l, const void* x, int T, const int32_t* idx,
                               const float* w, float* y, uint64_t slot_mask, int combine,
                               void* ws, size_t ws_bytes, void* stream) {
  g_last_error[0] = 0;
  moe_status s = check_call(l, x, T);
  if (s != MOE_OK) return s;
  if ((s = check_device_ptr(idx, 4, "idx")) != MOE_OK) return s;
  if ((s = check_device_ptr(w, 4, "w")) != MOE_OK) return s;
  if ((s = check_device_ptr(y, 16, "y")) != MOE_OK) return s;
  WsLayout L;
  if ((s = check_ws(l, T, ws, ws_bytes, &L)) != MOE_OK) return s;
  return ffn_impl(l, (const uint16_t*)x, T, idx, w, y, (uint8_t*)ws, L, (cudaStream_t)stream,
                  slot_mask, combine != 0);
}

moe_status moe_layer_forward(const moe_layer* l, const void* x, int T, float* y,
                             int32_t* idx_out, float* w_out, void* ws, size_t ws_bytes,
                             void* stream) {
  g_last_error[0] = 0;
  moe_status s = check_call(l, x, T);
  if (s != MOE_OK) return s;
  if ((s = check_device_ptr(y, 16, "y")) != MOE_OK) return s;
  if (idx_out && (s = check_device_ptr(idx_out, 4, "idx_out")) != MOE_OK) return s;
  if (w_out && (s = check_device_ptr(w_out, 4, "w_out")) != MOE_OK) return s;
  WsLayout L;
  if ((s = check_ws(l, T, ws, ws_bytes, &L)) != MOE_OK) return s;
  return forward_impl(l, (const uint16_t*)x, T, y, idx_out, w_out, (uint8_t*)ws, L,
                      (cudaStream_t)stream);
}

moe_status moe_layer_forward_residual(const moe_layer* l, const float* x_dev, float* x_next_dev,
                                      uint16_t* xn_out_dev, int32_t* idx_out_dev,
                                      float* w_out_dev, float norm_eps, void* ws, size_t ws_bytes,
                                      void* stream) {
  g_last_error[0] = 0;
  moe_status s = check_residual_args(l, x_dev, x_next_dev, xn_out_dev, idx_out_dev, w_out_dev,
                                     norm_eps);
  if (s != MOE_OK) return s;
  WsLayout L;
  if ((s = check_ws(l, 1, ws, ws_bytes, &L)) != MOE_OK) return s;
  return residual_impl(l, x_dev, norm_eps, x_next_dev, xn_out_dev, idx_out_dev, w_out_dev,
                       (uint8_t*)ws, L, (cudaStream_t)stream);
}

moe_status moe_stack_forward(const moe_layer* const* layers, int n_layers, const float* x_in_dev,
                             float* x_out_dev, float* x_tmp_dev, int32_t* idx_out_dev,
                             float norm_eps, void* ws, size_t ws_bytes, void* stream) {
  g_last_error[0] = 0;
  if (!layers || n_layers < 1) return fail(MOE_ERR_INVALID_ARG, "need at least one layer");
  if (n_layers > 1 && !x_tmp_dev) return fail(MOE_ERR_INVALID_ARG, "x_tmp is needed for more than one layer");
  if (!layers[0]) return fail(MOE_ERR_INVALID_ARG, "layers[0] is NULL");
  const moe_config& c0 = layers[0]->cfg;
  for (int l = 1; l < n_layers; ++l) {
    if (!layers[l]) return fail(MOE_ERR_INVALID_ARG, "layers[%d] is NULL", l);
    if (layers[l]->cfg.hidden != c0.hidden || layers[l]->cfg.top_k != c0.top_k)
      return fail(MOE_ERR_INVALID_ARG, "layers differ in shape");
  }
  if (x_tmp_dev && (x_tmp_dev == x_out_dev || x_tmp_dev == x_in_dev))
    return fail(MOE_ERR_INVALID_ARG, "x_tmp must be a separate buffer");
  // ping-pong so that the last layer writes x_out
  const float* cur = x_in_dev;
  for (int l = 0; l < n_layers; ++l) {
    const bool last = (l == n_layers - 1);
    float* nxt = ((n_layers - 1 - l) % 2 == 0) ? x_out_dev : x_tmp_dev;
    if (last) nxt = x_out_dev;
    int32_t* idx = idx_out_dev ? idx_out_dev + (size_t)l * c0.top_k : nullptr;
    moe_status s = check_residual_args(layers[l], cur, nxt, nullptr, idx, nullptr, norm_eps);
    WsLayout L;
    if (s == MOE_OK) s = check_ws(layers[l], 1, ws, ws_bytes, &L);
    if (s != MOE_OK) return s;
    s = residual_impl(layers[l], cur, norm_eps, nxt, nullptr, idx, nullptr, (uint8_t*)ws, L,
                      (cudaStream_t)stream, last ? nullptr : layers[l + 1]);
    if (s != MOE_OK) return s;
    cur = nxt;
  }
  return MOE_OK;
}

moe_status moe_debug_gemv_int4(const uint8_t* q, const uint16_t* s, int rows, int cols,
                               const float* x, float* y, void* stream) {
  g_last_error[0] = 0;
  if (rows < 1) return fail(MOE_ERR_INVALID_ARG, "rows = %d", rows);
  if (!chunk_cols_ok(cols)) return fail(MOE_ERR_UNSUPPORTED, "cols = %d", cols);
  moe_status st;
  if ((st = check_device_ptr(q, 16, "q")) != MOE_OK) return st;
  if ((st = check_device_ptr(s, 2, "s")) != MOE_OK) return st;
  if ((st = check_device_ptr(x, 16, "x")) != MOE_OK) return st;
  if ((st = check_device_ptr(y, 4, "y")) != MOE_OK) return st;
  cudaError_t e = launch_gemv_int4(q, s, rows, cols, x, y, (cudaStream_t)stream);
  return e == cudaSuccess ? MOE_OK : cuda_fail(e, "gemv launch");
}

#pragma GCC visibility pop
}  // extern "C"
