// kernels.h -- launchers of the step kernels (kernels.cu: router, selection,
// test GEMV) and of the batched expert path (union.cu).
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "common.cuh"

namespace moe {

// The kernels of a T-token call follow one another on the stream.  Each is a
// programmatic dependent launch: its blocks may be scheduled while the
// previous kernel finishes, and the kernel's first statement (pdl_wait)
// holds it until that kernel's writes are visible.  So only the launch
// latency overlaps; no kernel touches memory before the wait.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

template <typename... KArgs, typename... Args>
inline cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                              cudaStream_t st, Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, args...);
}

// Router logits in K slices: part [router_slices(H, T)][T][E] (fp64), each
// the sum of W x over a slice of the inputs (1 <= T <= 64, H a multiple of
// 16).
constexpr int kRouterMaxSlices = 32;
int router_slices(int H, int T);
cudaError_t launch_router_partial(const float* w, const uint16_t* x, int T, int H, int E,
                                  double* part, cudaStream_t st);
// noaux_tc selection from the logits (slices added in order, sigmoid in
// fp64 rounded to fp32), then adaptive top-p when top_p < 1 (dropped slots:
// id -1, weight 0, after the kept ids); scores_out (nullable) gets the
// fp32 sigmoid scores.
cudaError_t launch_select(const double* part, int H, const float* bias, int T, int E,
                          int n_group, int topk_group, int top_k, float rsf, float top_p,
                          int32_t* idx, float* w, float* scores_out, cudaStream_t st);
// The batched expert path (union.cu): distinct experts read once for all
// their tokens.  Scratch: xq (T * H/32 groups), hq (T * slots * I/32 groups),
// lists (union_lists_ints ints), hbuf (T * slots * I), ypart (T * slots * H).
size_t union_lists_ints(int T, int k, int E, int has_shared);

// Distinct experts with tc_min_tokens()..kTcMaxTok tokens take the
// tensor-core path when it is on (16 tokens at least: below that the
// contraction is too thin for the tensor cores to pay); the workspace holds
// the packed inputs for any threshold down to kTcMinTokFloor.
constexpr int kTcMinTokFloor = 16, kTcMaxTok = 64, kTcMinTokDefault = 16;
int tc_min_tokens();

// The per-call expert lists (build_lists_kernel), ints:
//   [0] U (distinct experts, the shared one last); u_expert [E + 1];
//   u_off [E + 2] (entries of expert slot u: u_off[u] .. u_off[u + 1]);
//   list_tok [n_list], list_pos [n_list] (token and (token, slot) row of
//   each entry); n_cc, n_tc; cc_u [E + 1], tc_u [E + 1] (the expert slots of
//   the CUDA-core and of the tensor-core path, ascending); tc_roff [E + 2]
//   (first packed input row of each tensor-core expert: its token count
//   rounded up to 16, summed over the ones before it).
struct ListsView {
  const int* u_expert;
  const int* u_off;
  const int* list_tok;
  const int* list_pos;
  const int* counts;  // [0] n_cc, [1] n_tc
  const int* cc_u;
  const int* tc_u;
  const int* tc_roff;
};

__host__ __device__ __forceinline__ ListsView lists_view(const int* lists, int E, int n_list) {
  ListsView v;
  v.u_expert = lists + 1;
  v.u_off = v.u_expert + (E + 1);
  v.list_tok = v.u_off + (E + 2);
  v.list_pos = v.list_tok + n_list;
  v.counts = v.list_pos + n_list;
  v.cc_u = v.counts + 2;
  v.tc_u = v.cc_u + (E + 1);
  v.tc_roff = v.tc_u + (E + 1);
  return v;
}
// tc_bpack (nullable, tc_bpack_bytes(T, k, has_shared, H, I) bytes): the
// packed inputs of the tensor-core path (tc_union.cu), taken by every
// distinct expert with tc_min_tokens() to 64 tokens when the shape allows
// it (tc_shape_ok); the other experts run on the CUDA-core union kernels.
// tc_maps (tc_maps_bytes(), 128-byte aligned): the path's tensor-map slots.
cudaError_t launch_union_ffn(const ExpertPtrs* table, const int32_t* idx, const float* w,
                             const uint16_t* x, int T, int H, int I, int E, int k, int has_shared,
                             uint8_t* xq_words, float* xq_fac, uint8_t* hq_words, float* hq_fac,
                             int* lists, float* hbuf, float* ypart, float* y, uint32_t* err,
                             uint8_t* tc_bpack, int* tc_rowexp, uint8_t* tc_maps,
                             cudaStream_t st, uint64_t slot_mask = ~0ull, bool combine = true);
// slot_mask: bit j (j < k) computes routed slot j of every token, bit k the
// shared expert; the rows of the other slots in ypart are left as they are.
// combine: y from every slot's ypart row (including rows an earlier call on
// the same workspace computed), in the fixed slot order.
// The tensor-core path (tc_union.cu): packed inputs and per-row exponents.
size_t tc_bpack_bytes(int T, int k, int has_shared, int H, int I);
size_t tc_rowexp_ints(int T, int k, int has_shared);
bool tc_shape_ok(int H, int I);
int tc_max_experts(int T, int k, int has_shared);
size_t tc_maps_bytes();
cudaError_t launch_tc_ffn_step(int mats, const ExpertPtrs* table, const int* lists, int E,
                               int n_list, int T, int k, int has_shared, const void* in, int K,
                               int R, int in_rows, int* row_exp, uint8_t* bpack, uint8_t* maps,
                               float* out, uint32_t* err, cudaStream_t st);

cudaError_t launch_gemv_int4(const uint8_t* q, const uint16_t* s, int rows, int cols,
                             const float* x, float* y, cudaStream_t st);

}  // namespace moe
