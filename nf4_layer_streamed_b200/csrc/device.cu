// Device error record of libnf4ls.  Kernels with bounded waits (the tcgen05 GEMM
// and attention) write the site of an expired wait here instead of hanging; the host
// reads and clears it through nf4ls_device_error().  The record is a file-scope
// __device__ array, so every device that loads the library holds its own copy; its
// address is looked up with cudaGetSymbolAddress once per CUDA context (again after a
// device reset, which replaces the context).
#include <atomic>
#include <mutex>
#include <vector>

#include "common.cuh"
#include "internal.h"

namespace nf4ls {

__device__ int g_dev_error[4];

unsigned long long current_context_id() {
  using GetCurrent = CUresult (*)(CUcontext*);
  using GetId = CUresult (*)(CUcontext, unsigned long long*);
  static GetCurrent get_current = nullptr;
  static GetId get_id = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &f, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_current = reinterpret_cast<GetCurrent>(f);
    f = nullptr;
    if (cudaGetDriverEntryPoint("cuCtxGetId", &f, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_id = reinterpret_cast<GetId>(f);
  });
  CUcontext c = nullptr;
  unsigned long long id = 0;
  if (!get_current || !get_id || get_current(&c) != CUDA_SUCCESS || !c || get_id(c, &id) != CUDA_SUCCESS) return 0;
  return id;
}

int* device_error_ptr() {
  static int* ptrs[64] = {nullptr};
  static unsigned long long ctx[64] = {0};
  static std::mutex mu;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
  const unsigned long long id = current_context_id();
  std::lock_guard<std::mutex> g(mu);
  if (!ptrs[dev] || id == 0 || id != ctx[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_dev_error) != cudaSuccess) return nullptr;
    ptrs[dev] = static_cast<int*>(p);
    ctx[dev] = current_context_id();  // the lookup makes the device's primary context current
  }
  return ptrs[dev];
}

namespace {

// Per device: the side stream (least priority, non-blocking) and its two events, made
// on first use and again when the device's context has changed.
struct SideSlot {
  std::mutex mu;
  unsigned long long ctx = 0;
  cudaStream_t side = nullptr;
  cudaEvent_t ready = nullptr, done = nullptr;
};
SideSlot g_side[64];

}  // namespace

SideStream::SideStream() = default;

SideStream::~SideStream() {
  if (forked_) g_side[dev_].mu.unlock();
}

int SideStream::fork(cudaStream_t s) {
  if (forked_) return fail(NF4LS_INVALID_ARG, "side stream: forked twice");
  int dev = 0;
  NF4_CUDA_TRY(cudaGetDevice(&dev));
  if (dev < 0 || dev >= 64) return fail(NF4LS_CUDA, "side stream: device %d", dev);
  SideSlot& sl = g_side[dev];
  sl.mu.lock();
  dev_ = dev;
  forked_ = true;
  const unsigned long long id = current_context_id();
  if (!sl.side || id == 0 || id != sl.ctx) {  // handles of an earlier context are gone with it
    int least = 0, greatest = 0;
    NF4_CUDA_TRY(cudaDeviceGetStreamPriorityRange(&least, &greatest));
    NF4_CUDA_TRY(cudaStreamCreateWithPriority(&sl.side, cudaStreamNonBlocking, least));
    NF4_CUDA_TRY(cudaEventCreateWithFlags(&sl.ready, cudaEventDisableTiming));
    NF4_CUDA_TRY(cudaEventCreateWithFlags(&sl.done, cudaEventDisableTiming));
    sl.ctx = id;
  }
  side_ = sl.side;
  ready_ = sl.ready;
  done_ = sl.done;
  NF4_CUDA_TRY(cudaEventRecord(ready_, s));
  NF4_CUDA_TRY(cudaStreamWaitEvent(side_, ready_, 0));
  return NF4LS_OK;
}

int SideStream::join(cudaStream_t s) {
  if (!forked_) return NF4LS_OK;
  NF4_CUDA_TRY(cudaEventRecord(done_, side_));
  NF4_CUDA_TRY(cudaStreamWaitEvent(s, done_, 0));
  forked_ = false;
  g_side[dev_].mu.unlock();
  return NF4LS_OK;
}

namespace {

// The expiry path of the bounded mbarrier wait, on its own: one block of two warps
// waits on an mbarrier that no thread ever arrives on.  Warp 0 waits limit_ns and
// gives up (site 1), which records the error and raises the block's abort flag;
// warp 1 waits on the same barrier with a limit a thousand times longer and must
// leave through that flag without recording anything (site 2 never appears).  No
// copy or tensor-core work is in flight, so giving up is safe here.
__global__ void k_wait_probe(int* err, unsigned long long limit_ns, int32_t* result) {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    abort_flag = 0;
  }
  __syncthreads();
  const int warp = threadIdx.x / 32;
  const bool ok = warp == 0 ? mbar_wait(&bar, 0, &abort_flag, err, KID_WAIT_PROBE, 1, limit_ns)
                            : mbar_wait(&bar, 0, &abort_flag, err, KID_WAIT_PROBE, 2, limit_ns * 1000ull);
  if ((threadIdx.x & 31) == 0) result[warp] = ok ? 1 : 0;
}

std::atomic<uint64_t> g_launches{0};
std::atomic<int> g_profile{0};
struct Rec {
  int kind, detail;
  double flops;
  cudaEvent_t e0, e1;
};
std::mutex g_prof_mu;
std::vector<Rec> g_recs;
std::vector<cudaEvent_t> g_free_events;

cudaEvent_t take_event() {
  if (!g_free_events.empty()) {
    cudaEvent_t e = g_free_events.back();
    g_free_events.pop_back();
    return e;
  }
  cudaEvent_t e = nullptr;
  cudaEventCreate(&e);
  return e;
}
}  // namespace

void note_launch(int n) { g_launches.fetch_add((uint64_t)n, std::memory_order_relaxed); }

bool profiling() { return g_profile.load(std::memory_order_relaxed) != 0; }

void profile_begin(cudaStream_t s, cudaEvent_t* e0) {
  std::lock_guard<std::mutex> g(g_prof_mu);
  *e0 = take_event();
  if (*e0) cudaEventRecord(*e0, s);
}

void profile_end(cudaStream_t s, cudaEvent_t e0, int kind, int detail, double flops) {
  std::lock_guard<std::mutex> g(g_prof_mu);
  cudaEvent_t e1 = take_event();
  if (!e0 || !e1) return;
  cudaEventRecord(e1, s);
  g_recs.push_back(Rec{kind, detail, flops, e0, e1});
}

}  // namespace nf4ls

extern "C" uint64_t nf4ls_launch_count(void) { return nf4ls::g_launches.load(); }

extern "C" int nf4ls_profile(int on) {
  if (on) {
    // create the events up front so that recording stays cheap inside a timed region
    std::lock_guard<std::mutex> g(nf4ls::g_prof_mu);
    while (nf4ls::g_free_events.size() + 2 * nf4ls::g_recs.size() < 16384) {
      cudaEvent_t e = nullptr;
      if (cudaEventCreate(&e) != cudaSuccess) break;
      nf4ls::g_free_events.push_back(e);
    }
  }
  nf4ls::g_profile.store(on ? 1 : 0);
  return NF4LS_OK;
}

extern "C" int nf4ls_profile_read(int sel, double out[3]) {
  nf4ls::clear_error();
  if (!out) return nf4ls::fail(NF4LS_INVALID_ARG, "nf4ls_profile_read: null output");
  std::lock_guard<std::mutex> g(nf4ls::g_prof_mu);
  double n = 0, ms = 0, flops = 0;
  for (auto& r : nf4ls::g_recs) {
    if ((sel < 1000 ? r.kind : r.detail) != sel) continue;
    NF4_CUDA_TRY(cudaEventSynchronize(r.e1));
    float t = 0.f;
    NF4_CUDA_TRY(cudaEventElapsedTime(&t, r.e0, r.e1));
    n += 1;
    ms += t;
    flops += r.flops;
  }
  out[0] = n;
  out[1] = ms;
  out[2] = flops;
  return NF4LS_OK;
}

extern "C" int nf4ls_profile_reset(void) {
  nf4ls::clear_error();
  std::lock_guard<std::mutex> g(nf4ls::g_prof_mu);
  for (auto& r : nf4ls::g_recs) {
    NF4_CUDA_TRY(cudaEventSynchronize(r.e1));
    nf4ls::g_free_events.push_back(r.e0);
    nf4ls::g_free_events.push_back(r.e1);
  }
  nf4ls::g_recs.clear();
  return NF4LS_OK;
}

extern "C" int nf4ls_device_error(int32_t out[4]) {
  nf4ls::clear_error();
  if (!out) return nf4ls::fail(NF4LS_INVALID_ARG, "nf4ls_device_error: null output");
  int* p = nf4ls::device_error_ptr();
  if (!p) return nf4ls::fail(NF4LS_CUDA, "nf4ls_device_error: no device record");
  NF4_CUDA_TRY(cudaDeviceSynchronize());
  NF4_CUDA_TRY(cudaMemcpy(out, p, 4 * sizeof(int32_t), cudaMemcpyDeviceToHost));
  NF4_CUDA_TRY(cudaMemset(p, 0, 4 * sizeof(int32_t)));
  return out[0] ? NF4LS_DEVICE_FAULT : NF4LS_OK;
}

extern "C" int nf4ls_wait_probe(int32_t limit_us, int32_t* result_dev, nf4ls_stream stream) {
  nf4ls::clear_error();
  if (limit_us < 1 || limit_us > 1000000 || !result_dev)
    return nf4ls::fail(NF4LS_INVALID_ARG, "nf4ls_wait_probe: limit_us %d outside [1, 1000000] or null result",
                       limit_us);
  int* err = nf4ls::device_error_ptr();
  if (!err) return nf4ls::fail(NF4LS_CUDA, "nf4ls_wait_probe: no device record");
  nf4ls::k_wait_probe<<<1, 64, 0, static_cast<cudaStream_t>(stream)>>>(err, 1000ull * (unsigned long long)limit_us,
                                                                     result_dev);
  nf4ls::note_launch();
  NF4_CUDA_TRY(cudaGetLastError());
  return NF4LS_OK;
}
