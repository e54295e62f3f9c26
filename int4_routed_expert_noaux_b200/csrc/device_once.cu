// device_once.cu -- the current context's id for the per-device caches of
// device_once.h, read through the driver entry points the runtime exposes
// (no link-time dependency on libcuda).
#include <cuda.h>
#include <cuda_runtime.h>

#include "device_once.h"

namespace moe {

namespace {

typedef CUresult (*CtxGetCurrentFn)(CUcontext*);
typedef CUresult (*CtxGetIdFn)(CUcontext, unsigned long long*);

struct CtxFns {
  CtxGetCurrentFn get_current = nullptr;
  CtxGetIdFn get_id = nullptr;
};

CtxFns load_fns() {
  CtxFns f;
  void* p = nullptr;
  cudaDriverEntryPointQueryResult q;
  if (cudaGetDriverEntryPointByVersion("cuCtxGetCurrent", &p, 12000, cudaEnableDefault, &q) ==
          cudaSuccess &&
      q == cudaDriverEntryPointSuccess)
    f.get_current = reinterpret_cast<CtxGetCurrentFn>(p);
  p = nullptr;
  if (cudaGetDriverEntryPointByVersion("cuCtxGetId", &p, 12000, cudaEnableDefault, &q) ==
          cudaSuccess &&
      q == cudaDriverEntryPointSuccess)
    f.get_id = reinterpret_cast<CtxGetIdFn>(p);
  cudaGetLastError();
  return f;
}

}  // namespace

uint64_t current_context_id() {
  static const CtxFns fns = load_fns();  // thread-safe static initialisation
  if (!fns.get_current || !fns.get_id) return 0;
  CUcontext c = nullptr;
  if (fns.get_current(&c) != CUDA_SUCCESS || !c) return 0;
  unsigned long long id = 0;
  if (fns.get_id(c, &id) != CUDA_SUCCESS) return 0;
  return (uint64_t)id;
}

int num_sms() {
  static DeviceOnce<int> cache;
  int dev = 0, n = 148;
  if (cudaGetDevice(&dev) != cudaSuccess) return n;
  cache.get(dev, &n, [dev](int* v) {
    int m = 0;
    if (cudaDeviceGetAttribute(&m, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || m <= 0)
      m = 148;
    *v = m;
    return cudaSuccess;
  });
  return n;
}

}  // namespace moe
