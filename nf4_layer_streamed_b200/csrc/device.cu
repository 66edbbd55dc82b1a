// Device error record of libnf4ls.  Kernels with bounded waits (the tcgen05 GEMM)
// write the site of an expired wait here instead of hanging; the host reads and
// clears it through nf4ls_device_error().  The record is a file-scope __device__
// array, so every device that loads the library holds its own copy; its address is
// looked up once per device with cudaGetSymbolAddress.
#include <mutex>

#include "internal.h"

namespace nf4ls {

__device__ int g_dev_error[4];

int* device_error_ptr() {
  static int* ptrs[64] = {nullptr};
  static std::mutex mu;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
  std::lock_guard<std::mutex> g(mu);
  if (!ptrs[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_dev_error) != cudaSuccess) return nullptr;
    ptrs[dev] = static_cast<int*>(p);
  }
  return ptrs[dev];
}

}  // namespace nf4ls

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
