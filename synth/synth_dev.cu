/*
 * synth_dev.cu -- device build of the seeded synthetic input generator for the
 * large tensors (packed int4 weight bytes and fp16 scales).  It gives the
 * same bytes as synth_fill_bytes / synth_fill_scales_f16 of the host build,
 * because both evaluate the functions of synth_core.h.
 */
#include <cuda_runtime.h>
#include <stdint.h>

#include "synth_core.h"

namespace {

__global__ void fill_bytes_kernel(uint64_t key, uint8_t* out, size_t n) {
  size_t words = n / 8;
  size_t stride = (size_t)gridDim.x * blockDim.x;
  for (size_t w = (size_t)blockIdx.x * blockDim.x + threadIdx.x; w < words;
       w += stride) {
    uint64_t r = synth_draw(key, (uint64_t)w);
    if ((reinterpret_cast<uintptr_t>(out) & 7) == 0) {
      reinterpret_cast<unsigned long long*>(out)[w] = r;
    } else {
      for (int b = 0; b < 8; ++b) out[8 * w + b] = (uint8_t)(r >> (8 * b));
    }
  }
  if (blockIdx.x == 0 && threadIdx.x == 0)
    for (size_t b = words * 8; b < n; ++b) out[b] = synth_byte(key, b);
}

__global__ void fill_scales_kernel(uint64_t key, uint16_t* out, size_t n,
                                   double lo, double hi) {
  size_t stride = (size_t)gridDim.x * blockDim.x;
  for (size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x; i < n;
       i += stride)
    out[i] = synth_scale_f16(key, (uint64_t)i, lo, hi);
}

int grid_for(size_t work) {
  size_t blocks = (work + 255) / 256;
  if (blocks > 148 * 32) blocks = 148 * 32;
  if (blocks < 1) blocks = 1;
  return (int)blocks;
}

}  // namespace

extern "C" {

/* Returns a cudaError_t value (0 = success).  out is a device pointer. */
int synth_dev_fill_bytes(uint64_t key, void* out, size_t n, void* stream) {
  if (n == 0) return 0;
  fill_bytes_kernel<<<grid_for(n / 8 + 1), 256, 0, (cudaStream_t)stream>>>(
      key, (uint8_t*)out, n);
  return (int)cudaGetLastError();
}

int synth_dev_fill_scales_f16(uint64_t key, void* out, size_t n, double lo,
                              double hi, void* stream) {
  if (n == 0) return 0;
  fill_scales_kernel<<<grid_for(n), 256, 0, (cudaStream_t)stream>>>(
      key, (uint16_t*)out, n, lo, hi);
  return (int)cudaGetLastError();
}

}  // extern "C"
