// cache.cu -- per-layer LRU cache of routed experts in HBM, fed from a
// pinned host store by cudaMemcpyAsync on a side stream (colibri summary,
// "Execution d'un MoE basee sur le streaming disque": a per-layer LRU cache
// of routed experts; "Principales fonctionnalites implementees": expert
// readahead while another expert block is multiplied).
//
// Replacement rule, per layer and per call: ids already cached are hits and
// are touched in ascending id order; then every missing id, in ascending
// order, takes an empty slot (the lowest) or else the least recently used
// slot that is not pinned and whose expert is not among the call's ids.
//
// Hot-store (colibri summary, "Learning cache et attentes selon le
// materiel": routed experts are logged and the most used ones are pinned at
// start-up): every acquire counts its ids in a per-layer usage log, and
// moe_cache_pin pins a chosen set of experts in their slots, so that the LRU
// never evicts them; the remaining slots (at least top_k) run the rule above.
#include <cuda_runtime.h>
#include <stdint.h>
#include <string.h>

#include <atomic>
#include <chrono>
#include <new>
#include <thread>
#include <vector>

#include "layer.h"
#include "moe.h"

namespace moe {

// The replacement rule on its own (host only).
class LruPolicy {
 public:
  LruPolicy(int n_experts, int slots)
      : slot_expert_(slots, -1), stamp_(slots, 0), pinned_(slots, 0), expert_slot_(n_experts, -1) {}

  struct Load {
    int expert, slot, evicted;
  };

  // Forget whatever slot `slot` holds (it becomes empty).
  void invalidate(int slot) {
    const int old = slot_expert_[slot];
    if (old >= 0) expert_slot_[old] = -1;
    slot_expert_[slot] = -1;
    stamp_[slot] = 0;
    pinned_[slot] = 0;
  }

  int slot_of(int expert) const { return expert_slot_[expert]; }

  int pinned_count() const {
    int n = 0;
    for (char p : pinned_) n += p;
    return n;
  }

  // ids ascending, distinct.  Fills loads (misses) and returns the hit count.
  int access(const int32_t* ids, int n, std::vector<Load>& loads) {
    loads.clear();
    int hits = 0;
    for (int j = 0; j < n; ++j) {
      const int s = expert_slot_[ids[j]];
      if (s >= 0) {
        stamp_[s] = ++clock_;
        ++hits;
      }
    }
    for (int j = 0; j < n; ++j)
      if (expert_slot_[ids[j]] < 0) load(ids[j], ids, n, loads);
    return hits;
  }

  // Make ids (ascending, distinct) the pinned set: cached ones are pinned
  // where they are, missing ones are loaded (as by access) and pinned; every
  // other slot becomes an ordinary LRU slot.  The caller keeps
  // n <= slots - top_k, so that a call of top_k ids always finds a victim.
  void pin(const int32_t* ids, int n, std::vector<Load>& loads) {
    loads.clear();
    for (char& p : pinned_) p = 0;
    for (int j = 0; j < n; ++j) {
      const int s = expert_slot_[ids[j]];
      if (s >= 0) {
        pinned_[s] = 1;
        stamp_[s] = ++clock_;
      }
    }
    for (int j = 0; j < n; ++j)
      if (expert_slot_[ids[j]] < 0) pinned_[load(ids[j], ids, n, loads)] = 1;
  }

 private:
  // Put expert e in the lowest empty slot, else in the least recently used
  // slot that is not pinned and does not hold one of ids; returns the slot.
  int load(int e, const int32_t* ids, int n, std::vector<Load>& loads) {
    int victim = -1;
    for (int s = 0; s < (int)slot_expert_.size() && victim < 0; ++s)
      if (slot_expert_[s] < 0) victim = s;
    if (victim < 0) {
      for (int s = 0; s < (int)slot_expert_.size(); ++s) {
        if (pinned_[s]) continue;
        bool current = false;
        for (int jj = 0; jj < n; ++jj)
          if (slot_expert_[s] == ids[jj]) current = true;
        if (current) continue;
        if (victim < 0 || stamp_[s] < stamp_[victim]) victim = s;
      }
    }
    const int old = slot_expert_[victim];
    if (old >= 0) expert_slot_[old] = -1;
    slot_expert_[victim] = e;
    expert_slot_[e] = victim;
    stamp_[victim] = ++clock_;
    loads.push_back(Load{e, victim, old});
    return victim;
  }

  std::vector<int> slot_expert_;
  std::vector<uint64_t> stamp_;
  std::vector<char> pinned_;
  std::vector<int> expert_slot_;
  uint64_t clock_ = 0;
};

// Host-side fault injection for tests (off unless armed through
// moe_debug_inject_fault): the n-th later event of a kind fails.
std::atomic<int> g_inject_kind{0};
std::atomic<int> g_inject_after{0};

bool inject(int kind) {
  if (g_inject_kind.load(std::memory_order_acquire) != kind) return false;
  if (g_inject_after.fetch_sub(1, std::memory_order_acq_rel) != 0) return false;
  g_inject_kind.store(0, std::memory_order_release);
  return true;
}

namespace {

// Host function run in stream order: holds the stream for `ms` milliseconds
// (an injected stall; host memory and time only, no GPU work).
void CUDART_CB hold_stream(void* ms) {
  std::this_thread::sleep_for(std::chrono::milliseconds((intptr_t)ms));
}

constexpr int kMaxTableUpdates = 32;

struct TableUpdate {
  int n;
  int ids[kMaxTableUpdates];
  ExpertPtrs ptrs[kMaxTableUpdates];
};

// Writes new pointer-table entries; the entries travel as kernel arguments,
// so the update is ordered on the compute stream with no host staging.
__global__ void table_update_kernel(ExpertPtrs* table, TableUpdate u) {
  const int i = threadIdx.x;
  if (i < u.n) table[u.ids[i]] = u.ptrs[i];
}

}  // namespace

}  // namespace moe

using namespace moe;

struct moe_cache {
  moe_config cfg;
  int n_layers = 0, slots = 0;
  size_t expert_bytes = 0;
  size_t off[6] = {0, 0, 0, 0, 0, 0};  // tensor offsets inside a slot
  std::vector<moe_expert> host;        // [L][E] pinned host experts (caller-owned)
  uint8_t* dev_slots = nullptr;        // [L][slots][expert_bytes]
  cudaStream_t copy_stream = nullptr;
  std::vector<cudaEvent_t> copied;     // per layer: loads of the last acquire done
  std::vector<cudaEvent_t> used;       // per layer: compute of the last release done
  std::vector<cudaEvent_t> slot_ev;    // [L][slots]: the copies of the slot's latest load done
  std::vector<bool> used_valid;
  std::vector<bool> acquired;          // per layer: acquired, not yet released
  std::vector<LruPolicy> lru;
  std::vector<moe_layer*> views;       // per layer, created by moe_cache_layer
  std::vector<uint64_t> hits, misses, bytes;
  std::vector<uint64_t> usage;         // [L][E]: times each expert was acquired
  std::vector<LruPolicy::Load> loads;  // scratch
};

namespace {

size_t expert_bytes_of(const moe_config& c, size_t off[6]) {
  const size_t H = c.hidden, I = c.inter;
  const size_t qgu = I * H / 2, sgu = I * (H / 32) * 2, qd = H * I / 2, sd = H * (I / 32) * 2;
  off[0] = 0;                 // q_gate
  off[1] = off[0] + qgu;      // q_up
  off[2] = off[1] + qgu;      // s_gate
  off[3] = off[2] + sgu;      // s_up
  off[4] = off[3] + sgu;      // q_down
  off[5] = off[4] + qd;       // s_down
  return off[5] + sd;
}

moe_status check_host_ptr(const void* p, const char* name) {
  if (!p) return fail(MOE_ERR_INVALID_ARG, "%s is NULL", name);
  cudaPointerAttributes a;
  cudaError_t e = cudaPointerGetAttributes(&a, p);
  if (e != cudaSuccess) {
    cudaGetLastError();
    return fail(MOE_ERR_INVALID_ARG, "%s: not a registered host pointer", name);
  }
  if (a.type != cudaMemoryTypeHost)
    return fail(MOE_ERR_INVALID_ARG, "%s is not pinned host memory", name);
  return MOE_OK;
}

ExpertPtrs slot_ptrs(const moe_cache* c, int layer, int slot) {
  const uint8_t* b = c->dev_slots + ((size_t)layer * c->slots + slot) * c->expert_bytes;
  return ExpertPtrs{b + c->off[0], b + c->off[1], reinterpret_cast<const uint16_t*>(b + c->off[2]),
                    reinterpret_cast<const uint16_t*>(b + c->off[3]), b + c->off[4],
                    reinterpret_cast<const uint16_t*>(b + c->off[5])};
}

}  // namespace

namespace {

moe_status check_ids(const moe_cache* c, const int32_t* ids, int n) {
  for (int j = 0; j < n; ++j)
    if (ids[j] < 0 || ids[j] >= c->cfg.n_experts || (j && ids[j] <= ids[j - 1]))
      return fail(MOE_ERR_INVALID_ARG, "ids must be ascending, distinct and in range");
  return MOE_OK;
}

// Enqueues the copies of c->loads, which were planned on `plan` (a copy of
// the layer's replacement state), and then commits plan, the counters and
// the pointer table -- only once every copy of every load is enqueued.
// `acquire_ids` (n of them, nullable) are the ids of an acquire: they count
// as hits / misses and in the usage log; a pin counts only its bytes.
moe_status commit_loads(moe_cache* c, int layer, cudaStream_t cs, const LruPolicy& plan,
                        int hits, const int32_t* acquire_ids, int n, const char* who,
                        bool split = false) {
  cudaError_t ce = cudaSuccess;
  if (!c->loads.empty()) {
    // A victim slot may still be read by compute enqueued earlier for this
    // layer: that of the last release, or -- acquired again with no release
    // in between -- everything enqueued on the compute stream so far.
    if (c->acquired[layer]) {
      ce = cudaEventRecord(c->used[layer], cs);
      if (ce == cudaSuccess) c->used_valid[layer] = true;
    }
    if (ce == cudaSuccess && c->used_valid[layer])
      ce = cudaStreamWaitEvent(c->copy_stream, c->used[layer], 0);
    if (ce == cudaSuccess && g_inject_kind.load(std::memory_order_acquire) == MOE_FAULT_CACHE_STALL) {
      const int ms = g_inject_after.exchange(0);
      g_inject_kind.store(0, std::memory_order_release);
      ce = cudaLaunchHostFunc(c->copy_stream, hold_stream, reinterpret_cast<void*>((intptr_t)ms));
    }
  }
  // pointer-table entries of the loads, kMaxTableUpdates per update kernel
  std::vector<TableUpdate> ups((c->loads.size() + kMaxTableUpdates - 1) / kMaxTableUpdates);
  for (TableUpdate& u : ups) u.n = 0;
  int reached = 0;  // loads whose slot a copy may have written
  for (const LruPolicy::Load& ld : c->loads) {
    if (ce != cudaSuccess) break;
    const moe_expert& he = c->host[(size_t)layer * c->cfg.n_experts + ld.expert];
    const ExpertPtrs d = slot_ptrs(c, layer, ld.slot);
    const void* src[6] = {he.q_gate, he.q_up, he.s_gate, he.s_up, he.q_down, he.s_down};
    void* dst[6] = {(void*)d.q_gate, (void*)d.q_up, (void*)d.s_gate,
                    (void*)d.s_up, (void*)d.q_down, (void*)d.s_down};
    const size_t sz[6] = {c->off[1] - c->off[0], c->off[2] - c->off[1], c->off[3] - c->off[2],
                          c->off[4] - c->off[3], c->off[5] - c->off[4],
                          c->expert_bytes - c->off[5]};
    ++reached;
    for (int t = 0; t < 6 && ce == cudaSuccess; ++t)
      ce = inject(MOE_FAULT_CACHE_COPY)
               ? cudaErrorInvalidValue
               : cudaMemcpyAsync(dst[t], src[t], sz[t], cudaMemcpyHostToDevice, c->copy_stream);
    // this expert's own completion, for compute that waits per expert
    if (ce == cudaSuccess)
      ce = cudaEventRecord(c->slot_ev[(size_t)layer * c->slots + ld.slot], c->copy_stream);
    TableUpdate& u = ups[(reached - 1) / kMaxTableUpdates];
    u.ids[u.n] = ld.expert;
    u.ptrs[u.n] = d;
    ++u.n;
  }
  if (!c->loads.empty()) {
    if (!split) {
      if (ce == cudaSuccess) ce = cudaEventRecord(c->copied[layer], c->copy_stream);
      if (ce == cudaSuccess) ce = cudaStreamWaitEvent(cs, c->copied[layer], 0);
    }
    for (size_t i = 0; i < ups.size() && ce == cudaSuccess; ++i) {
      table_update_kernel<<<1, kMaxTableUpdates, 0, cs>>>(c->views[layer]->table, ups[i]);
      ce = cudaGetLastError();
    }
  }
  if (ce != cudaSuccess) {
    // Roll back: the layer keeps its committed state, except that a slot a
    // copy may have reached no longer counts as holding anything.
    for (int i = 0; i < reached; ++i) c->lru[layer].invalidate(c->loads[i].slot);
    return cuda_fail(ce, who);
  }
  c->lru[layer] = plan;
  moe_layer* view = c->views[layer];
  for (const TableUpdate& u : ups)
    for (int i = 0; i < u.n; ++i) view->host_table[u.ids[i]] = u.ptrs[i];
  c->bytes[layer] += (uint64_t)c->loads.size() * c->expert_bytes;
  if (acquire_ids) {
    c->hits[layer] += hits;
    c->misses[layer] += c->loads.size();
    uint64_t* use = c->usage.data() + (size_t)layer * c->cfg.n_experts;
    for (int j = 0; j < n; ++j) ++use[acquire_ids[j]];
    c->acquired[layer] = true;
  }
  return MOE_OK;
}

}  // namespace

extern "C" {
#pragma GCC visibility push(default)

moe_status moe_lru_replay_pinned(int n_layers, int n_experts, int capacity, int k, int T,
                                 const int32_t* trace, int n_pinned, const int32_t* pinned,
                                 uint64_t* hits, uint64_t* misses) {
  if (n_layers < 1 || n_experts < 1 || k < 1 || T < 0 || !trace || !hits || !misses ||
      n_pinned < 0 || capacity - n_pinned < k || (n_pinned > 0 && !pinned))
    return fail(MOE_ERR_INVALID_ARG, "bad LRU replay arguments");
  std::vector<LruPolicy::Load> loads;
  for (int l = 0; l < n_layers; ++l) {
    LruPolicy lru(n_experts, capacity);
    const int32_t* pin = pinned ? pinned + (size_t)l * n_pinned : nullptr;
    for (int j = 0; j < n_pinned; ++j)
      if (pin[j] < 0 || pin[j] >= n_experts || (j && pin[j] <= pin[j - 1]))
        return fail(MOE_ERR_INVALID_ARG, "pinned ids must be ascending and in range");
    lru.pin(pin, n_pinned, loads);
    uint64_t h = 0, m = 0;
    for (int t = 0; t < T; ++t) {
      const int32_t* ids = trace + ((size_t)t * n_layers + l) * k;
      for (int j = 0; j < k; ++j)
        if (ids[j] < 0 || ids[j] >= n_experts || (j && ids[j] <= ids[j - 1]))
          return fail(MOE_ERR_INVALID_ARG, "trace ids must be ascending and in range");
      h += lru.access(ids, k, loads);
      m += loads.size();
    }
    hits[l] = h;
    misses[l] = m;
  }
  return MOE_OK;
}

moe_status moe_lru_replay(int n_layers, int n_experts, int capacity, int k, int T,
                          const int32_t* trace, uint64_t* hits, uint64_t* misses) {
  return moe_lru_replay_pinned(n_layers, n_experts, capacity, k, T, trace, 0, nullptr, hits,
                               misses);
}

moe_status moe_cache_create(const moe_config* cfg, int n_layers, int slots_per_layer,
                            const moe_expert* host_experts, moe_cache** out) {
  if (!out) return fail(MOE_ERR_INVALID_ARG, "out is NULL");
  *out = nullptr;
  moe_status s = check_config(cfg);
  if (s != MOE_OK) return s;
  if (n_layers < 1) return fail(MOE_ERR_INVALID_ARG, "n_layers must be >= 1");
  if (slots_per_layer < cfg->top_k || slots_per_layer > cfg->n_experts)
    return fail(MOE_ERR_INVALID_ARG, "slots_per_layer must be in [top_k, n_experts]");
  if (!host_experts) return fail(MOE_ERR_INVALID_ARG, "host_experts is NULL");
  const size_t n = (size_t)n_layers * cfg->n_experts;
  for (size_t i = 0; i < n; ++i) {
    const moe_expert& e = host_experts[i];
    const void* ptrs[6] = {e.q_gate, e.q_up, e.s_gate, e.s_up, e.q_down, e.s_down};
    for (int t = 0; t < 6; ++t)
      if ((s = check_host_ptr(ptrs[t], "host expert tensor")) != MOE_OK) return s;
  }
  moe_cache* c = new (std::nothrow) moe_cache();
  if (!c) return fail(MOE_ERR_OOM, "host allocation failed");
  c->cfg = *cfg;
  c->n_layers = n_layers;
  c->slots = slots_per_layer;
  c->expert_bytes = expert_bytes_of(*cfg, c->off);
  c->host.assign(host_experts, host_experts + n);
  const size_t dev_bytes = (size_t)n_layers * slots_per_layer * c->expert_bytes;
  size_t free_b = 0, total_b = 0;
  cudaError_t ce = cudaMemGetInfo(&free_b, &total_b);
  if (ce == cudaSuccess && dev_bytes + (256u << 20) > free_b) {
    delete c;
    return fail(MOE_ERR_OOM, "cache needs %zu bytes of HBM, %zu free", dev_bytes, free_b);
  }
  ce = inject(MOE_FAULT_CACHE_ALLOC) ? cudaErrorMemoryAllocation
                                      : cudaMalloc(&c->dev_slots, dev_bytes);
  if (ce == cudaSuccess) ce = cudaStreamCreateWithFlags(&c->copy_stream, cudaStreamNonBlocking);
  c->copied.assign(n_layers, nullptr);
  c->used.assign(n_layers, nullptr);
  c->slot_ev.assign((size_t)n_layers * slots_per_layer, nullptr);
  c->used_valid.assign(n_layers, false);
  c->acquired.assign(n_layers, false);
  for (int l = 0; l < n_layers && ce == cudaSuccess; ++l) {
    ce = cudaEventCreateWithFlags(&c->copied[l], cudaEventDisableTiming);
    if (ce == cudaSuccess) ce = cudaEventCreateWithFlags(&c->used[l], cudaEventDisableTiming);
  }
  for (size_t i = 0; i < c->slot_ev.size() && ce == cudaSuccess; ++i)
    ce = cudaEventCreateWithFlags(&c->slot_ev[i], cudaEventDisableTiming);
  if (ce != cudaSuccess) {
    s = cuda_fail(ce, "moe_cache_create");
    moe_cache_destroy(c);
    return s;
  }
  for (int l = 0; l < n_layers; ++l) c->lru.emplace_back(cfg->n_experts, slots_per_layer);
  c->views.assign(n_layers, nullptr);
  c->hits.assign(n_layers, 0);
  c->usage.assign((size_t)n_layers * cfg->n_experts, 0);
  c->misses.assign(n_layers, 0);
  c->bytes.assign(n_layers, 0);
  *out = c;
  return MOE_OK;
}

void moe_cache_destroy(moe_cache* c) {
  if (!c) return;
  if (c->copy_stream) cudaStreamSynchronize(c->copy_stream);
  for (moe_layer* v : c->views) moe_layer_destroy(v);
  for (cudaEvent_t e : c->copied)
    if (e) cudaEventDestroy(e);
  for (cudaEvent_t e : c->used)
    if (e) cudaEventDestroy(e);
  for (cudaEvent_t e : c->slot_ev)
    if (e) cudaEventDestroy(e);
  if (c->copy_stream) cudaStreamDestroy(c->copy_stream);
  if (c->dev_slots) cudaFree(c->dev_slots);
  delete c;
}

moe_status moe_cache_layer(moe_cache* c, int layer, const float* w_router_dev,
                           const float* bias_dev, const moe_expert* shared_host,
                           moe_layer** view) {
  if (!c || !view) return fail(MOE_ERR_INVALID_ARG, "cache or view is NULL");
  if (layer < 0 || layer >= c->n_layers) return fail(MOE_ERR_INVALID_ARG, "layer out of range");
  *view = nullptr;
  if (c->views[layer]) {
    *view = c->views[layer];
    return MOE_OK;
  }
  // every routed entry starts at slot 0 of the layer; the kernels only read
  // the entries of selected experts, which acquire sets first
  std::vector<moe_expert> tab(c->cfg.n_experts);
  const ExpertPtrs s0 = slot_ptrs(c, layer, 0);
  for (int e = 0; e < c->cfg.n_experts; ++e)
    tab[e] = moe_expert{s0.q_gate, s0.q_up, s0.s_gate, s0.s_up, s0.q_down, s0.s_down};
  moe_layer* l = nullptr;
  moe_status s = moe_layer_create(&c->cfg, w_router_dev, bias_dev, tab.data(), shared_host, &l);
  if (s != MOE_OK) return s;
  c->views[layer] = l;
  *view = l;
  return MOE_OK;
}

moe_status moe_cache_acquire(moe_cache* c, int layer, const int32_t* ids_host, int n,
                             void* compute_stream) {
  if (!c || !ids_host) return fail(MOE_ERR_INVALID_ARG, "cache or ids is NULL");
  if (layer < 0 || layer >= c->n_layers) return fail(MOE_ERR_INVALID_ARG, "layer out of range");
  if (!c->views[layer]) return fail(MOE_ERR_INVALID_ARG, "create the layer view first (moe_cache_layer)");
  if (n < 1 || n > c->slots || n > kMaxTableUpdates)
    return fail(MOE_ERR_INVALID_ARG, "n = %d outside 1..min(slots, %d)", n, kMaxTableUpdates);
  moe_status st = check_ids(c, ids_host, n);
  if (st != MOE_OK) return st;
  if (n > c->slots - c->lru[layer].pinned_count())
    return fail(MOE_ERR_INVALID_ARG, "n = %d exceeds the layer's unpinned slots", n);
  // The replacement is planned on a copy of the layer's state and committed
  // (with the counters and the pointer table) only once every copy of every
  // miss is enqueued.
  LruPolicy plan = c->lru[layer];
  const int hits = plan.access(ids_host, n, c->loads);
  return commit_loads(c, layer, (cudaStream_t)compute_stream, plan, hits, ids_host, n,
                      "moe_cache_acquire");
}

moe_status moe_cache_acquire_split(moe_cache* c, int layer, const int32_t* ids_host, int n,
                                   void* compute_stream, int32_t* missed_host) {
  if (!c || !ids_host || !missed_host) return fail(MOE_ERR_INVALID_ARG, "cache, ids or missed is NULL");
  if (layer < 0 || layer >= c->n_layers) return fail(MOE_ERR_INVALID_ARG, "layer out of range");
  if (!c->views[layer]) return fail(MOE_ERR_INVALID_ARG, "create the layer view first (moe_cache_layer)");
  if (n < 1 || n > c->slots || n > kMaxTableUpdates)
    return fail(MOE_ERR_INVALID_ARG, "n = %d outside 1..min(slots, %d)", n, kMaxTableUpdates);
  moe_status st = check_ids(c, ids_host, n);
  if (st != MOE_OK) return st;
  if (n > c->slots - c->lru[layer].pinned_count())
    return fail(MOE_ERR_INVALID_ARG, "n = %d exceeds the layer's unpinned slots", n);
  cudaStream_t cs = (cudaStream_t)compute_stream;
  LruPolicy plan = c->lru[layer];
  const int hits = plan.access(ids_host, n, c->loads);
  st = commit_loads(c, layer, cs, plan, hits, ids_host, n, "moe_cache_acquire_split", true);
  if (st != MOE_OK) return st;
  // a hit's slot may hold a load whose copies no compute has waited for
  // yet: the compute stream waits for the slot's latest load (long done,
  // as a rule); the misses are left to moe_cache_wait_expert
  for (int j = 0; j < n; ++j) {
    bool missed = false;
    for (const LruPolicy::Load& ld : c->loads) missed = missed || ld.expert == ids_host[j];
    missed_host[j] = missed ? 1 : 0;
    if (!missed) {
      const int s = c->lru[layer].slot_of(ids_host[j]);
      const cudaError_t ce = cudaStreamWaitEvent(cs, c->slot_ev[(size_t)layer * c->slots + s], 0);
      if (ce != cudaSuccess) return cuda_fail(ce, "moe_cache_acquire_split");
    }
  }
  return MOE_OK;
}

moe_status moe_cache_wait_expert(moe_cache* c, int layer, int expert, void* compute_stream) {
  if (!c) return fail(MOE_ERR_INVALID_ARG, "cache is NULL");
  if (layer < 0 || layer >= c->n_layers) return fail(MOE_ERR_INVALID_ARG, "layer out of range");
  if (expert < 0 || expert >= c->cfg.n_experts)
    return fail(MOE_ERR_INVALID_ARG, "expert %d out of range", expert);
  const int s = c->lru[layer].slot_of(expert);
  if (s < 0) return fail(MOE_ERR_INVALID_ARG, "expert %d is not in layer %d's cache", expert, layer);
  const cudaError_t ce = cudaStreamWaitEvent((cudaStream_t)compute_stream,
                                             c->slot_ev[(size_t)layer * c->slots + s], 0);
  return ce == cudaSuccess ? MOE_OK : cuda_fail(ce, "moe_cache_wait_expert");
}

moe_status moe_cache_expert_ffn(moe_cache* c, int layer, const void* x_dev,
                                const int32_t* ids_host, const int32_t* idx_dev,
                                const float* w_dev, float* y_dev, void* ws_dev, size_t ws_bytes,
                                void* stream, int* n_copied) {
  if (!c || !ids_host) return fail(MOE_ERR_INVALID_ARG, "cache or ids is NULL");
  if (layer < 0 || layer >= c->n_layers) return fail(MOE_ERR_INVALID_ARG, "layer out of range");
  const int k = c->cfg.top_k;
  int32_t missed[kMaxTableUpdates];
  moe_status s = moe_cache_acquire_split(c, layer, ids_host, k, stream, missed);
  if (s != MOE_OK) return s;
  const moe_layer* view = c->views[layer];
  uint64_t hit_mask = c->cfg.n_shared ? 1ull << k : 0ull;
  int n_miss = 0;
  for (int j = 0; j < k; ++j) {
    if (missed[j]) ++n_miss;
    else hit_mask |= 1ull << j;
  }
  // the resident experts (and the shared one) while the copies are on the link
  if (hit_mask)
    s = moe_expert_ffn_part(view, x_dev, 1, idx_dev, w_dev, y_dev, hit_mask, n_miss == 0, ws_dev,
                            ws_bytes, stream);
  // then each copied expert as soon as its own copy is done; the last call
  // combines every slot in the fixed order
  for (int j = 0, m = 0; j < k && s == MOE_OK; ++j) {
    if (!missed[j]) continue;
    ++m;
    s = moe_cache_wait_expert(c, layer, ids_host[j], stream);
    if (s == MOE_OK)
      s = moe_expert_ffn_part(view, x_dev, 1, idx_dev, w_dev, y_dev, 1ull << j, m == n_miss,
                              ws_dev, ws_bytes, stream);
  }
  if (s == MOE_OK && n_copied) *n_copied = n_miss;
  return s;
}

moe_status moe_cache_pin(moe_cache* c, int layer, const int32_t* ids_host, int n,
                         void* compute_stream) {
  if (!c || (n > 0 && !ids_host)) return fail(MOE_ERR_INVALID_ARG, "cache or ids is NULL");
  if (layer < 0 || layer >= c->n_layers) return fail(MOE_ERR_INVALID_ARG, "layer out of range");
  if (!c->views[layer]) return fail(MOE_ERR_INVALID_ARG, "create the layer view first (moe_cache_layer)");
  if (n < 0 || n > c->slots - c->cfg.top_k)
    return fail(MOE_ERR_INVALID_ARG, "n = %d outside 0..slots - top_k", n);
  moe_status st = check_ids(c, ids_host, n);
  if (st != MOE_OK) return st;
  LruPolicy plan = c->lru[layer];
  plan.pin(ids_host, n, c->loads);
  return commit_loads(c, layer, (cudaStream_t)compute_stream, plan, 0, nullptr, 0,
                      "moe_cache_pin");
}

moe_status moe_cache_usage(const moe_cache* c, int layer, uint64_t* counts) {
  if (!c || !counts) return fail(MOE_ERR_INVALID_ARG, "cache or counts is NULL");
  if (layer < 0 || layer >= c->n_layers) return fail(MOE_ERR_INVALID_ARG, "layer out of range");
  memcpy(counts, c->usage.data() + (size_t)layer * c->cfg.n_experts,
         sizeof(uint64_t) * c->cfg.n_experts);
  return MOE_OK;
}

moe_status moe_cache_release(moe_cache* c, int layer, void* compute_stream) {
  if (!c) return fail(MOE_ERR_INVALID_ARG, "cache is NULL");
  if (layer < 0 || layer >= c->n_layers) return fail(MOE_ERR_INVALID_ARG, "layer out of range");
  cudaError_t ce = cudaEventRecord(c->used[layer], (cudaStream_t)compute_stream);
  if (ce != cudaSuccess) return cuda_fail(ce, "moe_cache_release");
  c->used_valid[layer] = true;
  c->acquired[layer] = false;
  return MOE_OK;
}

moe_status moe_cache_stats(const moe_cache* c, int layer, uint64_t* hits, uint64_t* misses,
                           uint64_t* bytes_h2d) {
  if (!c) return fail(MOE_ERR_INVALID_ARG, "cache is NULL");
  if (layer < 0 || layer >= c->n_layers) return fail(MOE_ERR_INVALID_ARG, "layer out of range");
  if (hits) *hits = c->hits[layer];
  if (misses) *misses = c->misses[layer];
  if (bytes_h2d) *bytes_h2d = c->bytes[layer];
  return MOE_OK;
}

moe_status moe_cache_sync(moe_cache* c) {
  if (!c) return fail(MOE_ERR_INVALID_ARG, "cache is NULL");
  cudaError_t ce = cudaStreamSynchronize(c->copy_stream);
  return ce == cudaSuccess ? MOE_OK : cuda_fail(ce, "moe_cache_sync");
}

moe_status moe_cache_wait(moe_cache* c, int timeout_ms) {
  if (!c) return fail(MOE_ERR_INVALID_ARG, "cache is NULL");
  if (timeout_ms < 0) return fail(MOE_ERR_INVALID_ARG, "timeout_ms must be >= 0");
  const auto deadline = std::chrono::steady_clock::now() + std::chrono::milliseconds(timeout_ms);
  for (;;) {
    const cudaError_t ce = cudaStreamQuery(c->copy_stream);
    if (ce == cudaSuccess) return MOE_OK;
    if (ce != cudaErrorNotReady) return cuda_fail(ce, "moe_cache_wait");
    if (std::chrono::steady_clock::now() >= deadline)
      return fail(MOE_ERR_TIMEOUT, "expert copies still running after %d ms", timeout_ms);
    std::this_thread::sleep_for(std::chrono::microseconds(50));
  }
}

moe_status moe_debug_inject_fault(int kind, int n) {
  if (kind < MOE_FAULT_NONE || kind > MOE_FAULT_CACHE_STALL || n < 0)
    return fail(MOE_ERR_INVALID_ARG, "bad fault injection (kind %d, n %d)", kind, n);
  g_inject_kind.store(0, std::memory_order_release);
  g_inject_after.store(n, std::memory_order_release);
  g_inject_kind.store(kind, std::memory_order_release);
  return MOE_OK;
}

#pragma GCC visibility pop
}  // extern "C"
