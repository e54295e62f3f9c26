// noalloc.cu -- the one-token layer forward with its scratch in a fixed
// device array instead of a caller workspace, so that a call allocates
// nothing: no cudaMalloc, no cudaFree, no library call that allocates.
#include <cuda_runtime.h>

#include "device_once.h"
#include "layer.h"

namespace moe {

// Largest scratch the call takes: the one-token workspace of the shape,
// ws_layout(cfg, 1).total.  A 6144 x 2048 layer with top-8 of 256 experts
// and one shared expert needs 357,120 bytes.
constexpr size_t kStaticScratchBytes = 512u << 10;
// control words plus the router score records that follow them (8 bytes per
// expert; the fused kernel, their only user, takes at most 256 experts)
constexpr size_t kStaticClearBytes = kCtrlBytes + 256 * 8;

static __device__ __align__(256) uint8_t g_static_scratch[kStaticScratchBytes];

static DeviceOnce<uint8_t*> g_scratch_addr;

// Address of g_static_scratch on `dev` (the current device), resolved once
// per device and context; the first resolution also zero-fills the control
// words and the router score records on `st` (the array starts zeroed at
// module load as well).
static moe_status scratch_address(int dev, cudaStream_t st, uint8_t** out) {
  uint8_t* a = nullptr;
  const cudaError_t e = g_scratch_addr.get(dev, &a, [st](uint8_t** v) {
    void* sym = nullptr;
    cudaError_t r = cudaGetSymbolAddress(&sym, g_static_scratch);
    if (r != cudaSuccess) return r;
    r = cudaMemsetAsync(sym, 0, kStaticClearBytes, st);
    if (r != cudaSuccess) return r;
    *v = static_cast<uint8_t*>(sym);
    return cudaSuccess;
  });
  if (e != cudaSuccess) return cuda_fail(e, "scratch symbol address");
  *out = a;
  return MOE_OK;
}

}  // namespace moe

using namespace moe;

extern "C" {
#pragma GCC visibility push(default)

moe_status moe_layer_forward_noalloc(const moe_layer* l, const void* x, float* y,
                                     int32_t* idx_out, float* w_out, uint32_t* status_out,
                                     void* stream) {
  clear_last_error();
  if (!l) return fail(MOE_ERR_INVALID_ARG, "layer is NULL");
  moe_status s;
  if ((s = check_device_ptr(x, 16, "x")) != MOE_OK) return s;
  if ((s = check_device_ptr(y, 16, "y")) != MOE_OK) return s;
  if (idx_out && (s = check_device_ptr(idx_out, 4, "idx_out")) != MOE_OK) return s;
  if (w_out && (s = check_device_ptr(w_out, 4, "w_out")) != MOE_OK) return s;
  if (status_out && (s = check_device_ptr(status_out, 4, "status_out")) != MOE_OK) return s;
  const WsLayout L = ws_layout(&l->cfg, 1);
  if (L.total > kStaticScratchBytes)
    return fail(MOE_ERR_UNSUPPORTED, "the layer needs %zu bytes of scratch, the fixed array has %zu",
                L.total, kStaticScratchBytes);
  int dev = -1;
  cudaError_t ce = cudaGetDevice(&dev);
  if (ce != cudaSuccess) return cuda_fail(ce, "cudaGetDevice");
  if (dev != l->device)
    return fail(MOE_ERR_INVALID_ARG, "current device %d is not the layer's device %d", dev,
                l->device);
  if (dev < 0 || dev >= kMaxDevices)
    return fail(MOE_ERR_UNSUPPORTED, "device ordinal %d >= %d", dev, kMaxDevices);
  cudaStream_t st = (cudaStream_t)stream;
  uint8_t* ws = nullptr;
  if ((s = scratch_address(dev, st, &ws)) != MOE_OK) return s;
  // The kernels return their counters to zero on every exit, stopped early
  // or not, and the epoch word must keep counting; only the error word of an
  // earlier call is cleared, so that status_out reports this call alone.
  ce = cudaMemsetAsync(ws + L.ctrl, 0, sizeof(uint32_t), st);
  if (ce != cudaSuccess) return cuda_fail(ce, "error word clear");
  if ((s = forward_impl(l, (const uint16_t*)x, 1, y, idx_out, w_out, ws, L, st)) != MOE_OK)
    return s;
  if (status_out) {
    ce = cudaMemcpyAsync(status_out, ws + L.ctrl, sizeof(uint32_t), cudaMemcpyDeviceToDevice, st);
    if (ce != cudaSuccess) return cuda_fail(ce, "status copy");
  }
  return MOE_OK;
}

#pragma GCC visibility pop
}  // extern "C"
