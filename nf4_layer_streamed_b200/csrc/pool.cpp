// Streaming pool: n-deep HBM slot pool fed from the pinned host store on a
// dedicated copy stream.
//
// Mechanism from the layer-streaming review ("4GB 显存微调 8B 模型是真的", mechanism
// section, and its English version): the frozen base lives in page-locked host
// memory, 2-8 preallocated device buffers (two by default) are filled
// asynchronously on their own CUDA stream, prefetching layer i+1 during the forward
// and layer i-1 during the backward, so that copies overlap compute.
//
// Reuse rule from the same page's bug history (Issue #331: a weight kept alive
// outside save_for_backward aliased a pooled buffer and silently corrupted the
// gradients of >165 MiB layers): a slot is overwritten only after the event that
// its releaser recorded on the compute stream -- after every kernel that reads the
// slot -- has completed.  The copy stream waits on that event; nothing else orders
// the reuse.  A layer still held by a slot is served without a new copy, which lets
// the backward start on the layers the forward left behind.
#include <algorithm>
#include <chrono>
#include <mutex>
#include <thread>
#include <vector>

#include "internal.h"

using namespace nf4ls;

struct nf4ls_pool {
  int device = 0;
  const uint8_t* store = nullptr;
  std::vector<size_t> off, bytes;
  int n_layers = 0, depth = 0;
  uint8_t* slots = nullptr;
  size_t slot_bytes = 0;
  cudaStream_t copy = nullptr;
  struct Slot {
    int layer = -1;
    bool acquired = false;
    bool pending = false;  // filled by a prefetch and not yet acquired
    bool freed_recorded = false;
    uint64_t release_tick = 0;
    cudaEvent_t ready = nullptr, freed = nullptr;
  };
  std::vector<Slot> slot;
  uint64_t tick = 0;
  bool poison = false;
  nf4ls_pool_stats stats{};
  std::mutex mu;

  int find(int layer) const {
    for (int i = 0; i < depth; ++i)
      if (slot[i].layer == layer) return i;
    return -1;
  }

  int victim() const {
    int best = -1;
    for (int i = 0; i < depth; ++i) {
      const Slot& s = slot[i];
      if (s.acquired || s.pending) continue;
      if (s.layer < 0) return i;
      if (best < 0 || s.release_tick < slot[best].release_tick) best = i;
    }
    return best;
  }

  int issue(int layer, int* out_idx) {
    int i = find(layer);
    if (i >= 0) {
      *out_idx = i;
      return NF4LS_OK;
    }
    i = victim();
    if (i < 0) return fail(NF4LS_BUFFER_BUSY, "pool: every slot is acquired or pending (depth %d)", depth);
    Slot& s = slot[i];
    uint8_t* dst = slots + (size_t)i * slot_bytes;
    if (s.freed_recorded) NF4_CUDA_TRY(cudaStreamWaitEvent(copy, s.freed, 0));
    if (poison) NF4_CUDA_TRY(cudaMemsetAsync(dst, 0xFF, slot_bytes, copy));
    NF4_CUDA_TRY(cudaMemcpyAsync(dst, store + off[layer], bytes[layer], cudaMemcpyHostToDevice, copy));
    NF4_CUDA_TRY(cudaEventRecord(s.ready, copy));
    s.layer = layer;
    s.pending = true;
    stats.bytes_copied += bytes[layer];
    stats.copies += 1;
    *out_idx = i;
    return NF4LS_OK;
  }
};

extern "C" int nf4ls_pool_create(const void* pinned_host, const size_t* layer_off, const size_t* layer_bytes,
                                 int n_layers, int depth, void* slots_dev, size_t slot_bytes, nf4ls_pool** out) {
  clear_error();
  if (!pinned_host || !layer_off || !layer_bytes || !slots_dev || !out)
    return fail(NF4LS_INVALID_ARG, "nf4ls_pool_create: null pointer");
  if (n_layers <= 0) return fail(NF4LS_INVALID_ARG, "nf4ls_pool_create: n_layers must be positive");
  if (depth < 2 || depth > 8) return fail(NF4LS_INVALID_ARG, "nf4ls_pool_create: depth %d not in [2, 8]", depth);
  if (!aligned(slots_dev, 256) || slot_bytes % 256)
    return fail(NF4LS_ALIGN, "nf4ls_pool_create: slots must be 256-byte aligned and sized");
  for (int i = 0; i < n_layers; ++i) {
    if (layer_bytes[i] > slot_bytes)
      return fail(NF4LS_INVALID_ARG, "nf4ls_pool_create: layer %d (%zu B) exceeds slot (%zu B)", i, layer_bytes[i],
                  slot_bytes);
    if (layer_off[i] % 256) return fail(NF4LS_ALIGN, "nf4ls_pool_create: layer %d offset not 256-aligned", i);
  }
  nf4ls_pool* p = new nf4ls_pool();
  p->store = static_cast<const uint8_t*>(pinned_host);
  p->off.assign(layer_off, layer_off + n_layers);
  p->bytes.assign(layer_bytes, layer_bytes + n_layers);
  p->n_layers = n_layers;
  p->depth = depth;
  p->slots = static_cast<uint8_t*>(slots_dev);
  p->slot_bytes = slot_bytes;
  p->slot.resize(depth);
  cudaError_t e = cudaGetDevice(&p->device);
  if (e == cudaSuccess) e = cudaStreamCreateWithFlags(&p->copy, cudaStreamNonBlocking);
  for (int i = 0; i < depth && e == cudaSuccess; ++i) {
    e = cudaEventCreateWithFlags(&p->slot[i].ready, cudaEventDisableTiming);
    if (e == cudaSuccess) e = cudaEventCreateWithFlags(&p->slot[i].freed, cudaEventDisableTiming);
  }
  if (e != cudaSuccess) {
    nf4ls_pool_destroy(p);
    return fail(NF4LS_CUDA, "nf4ls_pool_create: %s", cudaGetErrorString(e));
  }
  *out = p;
  return NF4LS_OK;
}

extern "C" int nf4ls_pool_prefetch(nf4ls_pool* p, int layer) {
  clear_error();
  if (!p || layer < 0 || layer >= p->n_layers) return fail(NF4LS_INVALID_ARG, "nf4ls_pool_prefetch: bad argument");
  std::lock_guard<std::mutex> g(p->mu);
  int idx;
  return p->issue(layer, &idx);
}

extern "C" int stream_prefetch(nf4ls_pool* p, int layer, nf4ls_stream compute, const void** slot_dev) {
  clear_error();
  if (!p || layer < 0 || layer >= p->n_layers || !slot_dev)
    return fail(NF4LS_INVALID_ARG, "stream_prefetch: bad argument");
  std::lock_guard<std::mutex> g(p->mu);
  const bool hit = p->find(layer) >= 0;  // resident or already prefetched: this call copies nothing
  int idx;
  NF4_TRY(p->issue(layer, &idx));
  nf4ls_pool::Slot& s = p->slot[idx];
  if (s.acquired) return fail(NF4LS_BUFFER_BUSY, "stream_prefetch: layer %d is already acquired", layer);
  NF4_CUDA_TRY(cudaStreamWaitEvent(static_cast<cudaStream_t>(compute), s.ready, 0));
  s.acquired = true;
  s.pending = false;
  p->stats.acquisitions += 1;
  if (hit) p->stats.hits += 1;
  *slot_dev = p->slots + (size_t)idx * p->slot_bytes;
  return NF4LS_OK;
}

extern "C" int nf4ls_pool_release(nf4ls_pool* p, int layer, nf4ls_stream compute) {
  clear_error();
  if (!p || layer < 0 || layer >= p->n_layers) return fail(NF4LS_INVALID_ARG, "nf4ls_pool_release: bad argument");
  std::lock_guard<std::mutex> g(p->mu);
  const int idx = p->find(layer);
  if (idx < 0 || !p->slot[idx].acquired) return fail(NF4LS_INVALID_ARG, "nf4ls_pool_release: layer %d not acquired", layer);
  nf4ls_pool::Slot& s = p->slot[idx];
  NF4_CUDA_TRY(cudaEventRecord(s.freed, static_cast<cudaStream_t>(compute)));
  s.freed_recorded = true;
  s.acquired = false;
  s.release_tick = ++p->tick;
  return NF4LS_OK;
}

extern "C" int nf4ls_wait(nf4ls_pool* p, int layer, int timeout_ms) {
  clear_error();
  if (!p || layer < 0 || layer >= p->n_layers) return fail(NF4LS_INVALID_ARG, "nf4ls_wait: bad argument");
  cudaEvent_t ev;
  {
    std::lock_guard<std::mutex> g(p->mu);
    const int idx = p->find(layer);
    if (idx < 0) return fail(NF4LS_INVALID_ARG, "nf4ls_wait: layer %d has no slot", layer);
    ev = p->slot[idx].ready;
  }
  const auto t0 = std::chrono::steady_clock::now();
  while (true) {
    const cudaError_t e = cudaEventQuery(ev);
    if (e == cudaSuccess) return NF4LS_OK;
    if (e != cudaErrorNotReady) return fail(NF4LS_CUDA, "nf4ls_wait: %s", cudaGetErrorString(e));
    const auto ms = std::chrono::duration_cast<std::chrono::milliseconds>(std::chrono::steady_clock::now() - t0);
    if (ms.count() >= timeout_ms) return fail(NF4LS_TIMEOUT, "nf4ls_wait: layer %d not ready after %d ms", layer, timeout_ms);
    std::this_thread::sleep_for(std::chrono::microseconds(50));
  }
}

extern "C" int nf4ls_pool_set_poison(nf4ls_pool* p, int on) {
  if (!p) return fail(NF4LS_INVALID_ARG, "null pool");
  std::lock_guard<std::mutex> g(p->mu);
  p->poison = on != 0;
  return NF4LS_OK;
}

extern "C" int nf4ls_pool_get_stats(nf4ls_pool* p, nf4ls_pool_stats* out) {
  if (!p || !out) return fail(NF4LS_INVALID_ARG, "null argument");
  std::lock_guard<std::mutex> g(p->mu);
  *out = p->stats;
  return NF4LS_OK;
}

extern "C" int nf4ls_pool_synchronize(nf4ls_pool* p) {
  if (!p) return fail(NF4LS_INVALID_ARG, "null pool");
  NF4_CUDA_TRY(cudaStreamSynchronize(p->copy));
  return NF4LS_OK;
}

extern "C" int nf4ls_pool_destroy(nf4ls_pool* p) {
  if (!p) return NF4LS_OK;
  if (p->copy) cudaStreamSynchronize(p->copy);
  for (auto& s : p->slot) {
    if (s.ready) cudaEventDestroy(s.ready);
    if (s.freed) cudaEventDestroy(s.freed);
  }
  if (p->copy) cudaStreamDestroy(p->copy);
  delete p;
  return NF4LS_OK;
}
