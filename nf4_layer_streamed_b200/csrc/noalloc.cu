// nf4_quantize_tensor_noalloc: the NF4 quantiser for callers that cannot allocate
// device memory.
//
// nf4_quantize_tensor needs a scratch buffer of n/64 floats (the per-block absmax
// values between the quantiser's passes) plus 8 KB for its offset pass, which its
// caller allocates.  Some callers
// cannot: code running where the CUDA allocator is off limits (inside another
// framework's memory pool or a host callback that must not allocate), or a process
// that has handed all device memory to a pool it does not control.  This entry point
// keeps that scratch in a fixed file-scope device array instead, so the caller only
// passes its input and output buffers.
//
// The array holds the absmax values of tensors up to kMaxElems weights (16 MiB of
// device memory, plus the offset pass's 8 KB), and every GPU that loads the library
// holds its own copy until the process exits.  Host code cannot use the array's name
// as a device address; the address is looked up with cudaGetSymbolAddress on the
// first call made with that device current, and again on the first call in a new
// CUDA context (after a device reset, or under a context the caller created), since
// an address from one context is not valid in another.  Make that first call before
// any stream capture.
// Every call shares the one array: calls whose kernels overlap on the GPU (on
// different streams) race on it.  Nothing in it needs to start at zero: each call
// writes every absmax value it later reads.
#include <mutex>

#include "internal.h"

namespace nf4ls {

namespace {

constexpr size_t kMaxElems = 1ull << 28;  // 268,435,456 weights
constexpr size_t kScratchFloats = kMaxElems / 64 + 2048;  // absmax values + the offset pass's 8 KB
static __device__ __align__(256) float g_quant_scratch[kScratchFloats];

std::mutex g_mu;
float* g_ptr[64] = {nullptr};
unsigned long long g_ctx[64] = {0};  // the context each cached address belongs to

int scratch_address(float** out) {
  int dev = 0;
  NF4_CUDA_TRY(cudaGetDevice(&dev));
  if (dev < 0 || dev >= 64) return fail(NF4LS_INVALID_ARG, "nf4_quantize_tensor_noalloc: device %d out of range", dev);
  const unsigned long long id = current_context_id();
  std::lock_guard<std::mutex> g(g_mu);
  if (!g_ptr[dev] || id == 0 || id != g_ctx[dev]) {
    void* p = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(&p, g_quant_scratch);
    if (e != cudaSuccess)
      return fail(NF4LS_CUDA, "nf4_quantize_tensor_noalloc: cudaGetSymbolAddress failed: %s", cudaGetErrorString(e));
    g_ptr[dev] = static_cast<float*>(p);
    g_ctx[dev] = current_context_id();
  }
  *out = g_ptr[dev];
  return NF4LS_OK;
}

}  // namespace

}  // namespace nf4ls

extern "C" size_t nf4ls_quantize_noalloc_max_elems(void) { return nf4ls::kMaxElems; }

extern "C" int nf4_quantize_tensor_noalloc(const void* w_dev, size_t n, uint8_t* packed_dev, uint8_t* q8_dev,
                                           float* nested_dev, float* offset_dev, nf4ls_stream stream) {
  nf4ls::clear_error();
  if (n > nf4ls::kMaxElems)
    return nf4ls::fail(NF4LS_INVALID_ARG,
                       "nf4_quantize_tensor_noalloc: n=%zu exceeds the fixed scratch of %zu weights; "
                       "use nf4_quantize_tensor with a caller-provided scratch buffer",
                       n, nf4ls::kMaxElems);
  float* scratch = nullptr;
  NF4_TRY(nf4ls::scratch_address(&scratch));
  return nf4ls::quantize_tensor(w_dev, n, packed_dev, q8_dev, nested_dev, offset_dev, scratch,
                                nf4ls::kScratchFloats * sizeof(float), static_cast<cudaStream_t>(stream));
}
