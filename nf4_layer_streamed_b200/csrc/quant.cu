// K1: blockwise NF4 quantiser with double-quantised absmax, and K2: the standalone
// dequantiser.  Format and arithmetic: "Soup 层流式 NF4 训练实测：在 4 GB 显存上以位级一致标准完成 8B 模型 LoRA 微调" §2.1
// (offline quantisation, one tensor at a time on the GPU, packed bytes plus absmax,
// nested absmax and offset sidecars) and §2.4 (bytes per weight, 16/256-entry fp32
// code tables).  Every step is fp32 with explicit round-to-nearest intrinsics, so the
// bytes and the dequantised bf16 weights are exact, reproducible results.
//
// Quantiser passes over a tensor of n bf16 values (nb = n / 64 blocks):
//   1. absmax_codes: a warp covers 4 blocks per iteration (8 lanes x 8 values per
//      block); absmax by shuffle; code = number of NF4 midpoints below fp32(x/absmax);
//      two codes per byte, the even element in the high nibble.
//   2. offset: the mean of the fp32 absmax values, defined as their sequential sum in
//      block order in double precision, divided by nb.  A parallel pass sums them in
//      a tree and also finds the smallest unit in the last place among the nonzero
//      values; when the total stays below 2^52 of those units, every partial sum of
//      any order is exact in double precision, so the tree's sum is the sequential
//      sum and it is used.  Otherwise one thread repeats the sequential sum.
//      (Weights of one tensor have absmax values within a factor of a few hundred of
//      each other, so the parallel sum is the one that runs.)
//   3. nested_q8: one 256-thread block per group of 256 blocks: nested = max |absmax -
//      offset|, q8 = number of code8 midpoints below fp32((absmax - offset) / nested).
#include <algorithm>
#include <cstring>

#include "common.cuh"
#include "internal.h"

namespace nf4ls {

struct QuantTables {
  float mid4[15];
  float mid8[255];
  int zero4, zero8;
};

struct DequantTables {
  float nf4[16];
  float code8[256];
};

__global__ void __launch_bounds__(256) k_absmax_codes(const __nv_bfloat16* __restrict__ w, size_t nb,
                                                      uint8_t* __restrict__ packed, float* __restrict__ absmax,
                                                      const QuantTables tab) {
  const int lane = threadIdx.x & 31;
  const size_t warp = (blockIdx.x * (size_t)blockDim.x + threadIdx.x) >> 5;
  const size_t nwarps = (gridDim.x * (size_t)blockDim.x) >> 5;
  const int sub = lane >> 3;  // block within the 4-block chunk
  const int part = lane & 7;  // 8 values of the block
  for (size_t chunk = warp; chunk * 4 < nb; chunk += nwarps) {
    const size_t b = chunk * 4 + sub;
    const bool valid = b < nb;
    uint4 raw = make_uint4(0, 0, 0, 0);
    if (valid) raw = *reinterpret_cast<const uint4*>(w + b * 64 + part * 8);
    const uint32_t wv[4] = {raw.x, raw.y, raw.z, raw.w};
    float x[8];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      x[2 * i] = bf16_lo(wv[i]);
      x[2 * i + 1] = bf16_hi(wv[i]);
    }
    float am = 0.f;
#pragma unroll
    for (int i = 0; i < 8; ++i) am = fmaxf(am, fabsf(x[i]));
#pragma unroll
    for (int o = 1; o < 8; o <<= 1) am = fmaxf(am, __shfl_xor_sync(0xffffffffu, am, o));
    uint32_t bytes = 0;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      int code = tab.zero4;
      if (am > 0.f) {
        const float u = __fdiv_rn(x[i], am);
        code = 0;
#pragma unroll
        for (int j = 0; j < 15; ++j) code += (u > tab.mid4[j]) ? 1 : 0;
      }
      // element 2j -> high nibble of byte j, element 2j+1 -> low nibble
      const int byte = i >> 1;
      bytes |= (uint32_t)code << (byte * 8 + ((i & 1) ? 0 : 4));
    }
    if (valid) {
      *reinterpret_cast<uint32_t*>(packed + b * 32 + part * 4) = bytes;
      if (part == 0) absmax[b] = am;
    }
  }
}

constexpr int kOffsetBlocks = 256;
constexpr size_t kOffsetScratch = 8192;  // after the absmax values: partials and the flag

struct OffsetPart {
  double sum;
  int min_ulp;  // smallest exponent of the unit in the last place among nonzero values
  int pad;
};

__device__ __forceinline__ int ulp_exponent(float x) {
  const int e = (int)((__float_as_uint(x) >> 23) & 0xFF);
  return (e > 0 ? e : 1) - 150;
}

__global__ void __launch_bounds__(256) k_offset_partial(const float* __restrict__ absmax, size_t nb,
                                                        OffsetPart* __restrict__ part) {
  __shared__ double ssum[256];
  __shared__ int sulp[256];
  double acc = 0.0;
  int mu = 1 << 20;
  for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < nb; i += (size_t)gridDim.x * blockDim.x) {
    const float v = absmax[i];
    acc += (double)v;
    if (v != 0.f) mu = min(mu, ulp_exponent(v));
  }
  ssum[threadIdx.x] = acc;
  sulp[threadIdx.x] = mu;
  __syncthreads();
  for (int o = 128; o > 0; o >>= 1) {
    if (threadIdx.x < o) {
      ssum[threadIdx.x] += ssum[threadIdx.x + o];
      sulp[threadIdx.x] = min(sulp[threadIdx.x], sulp[threadIdx.x + o]);
    }
    __syncthreads();
  }
  if (threadIdx.x == 0) part[blockIdx.x] = OffsetPart{ssum[0], sulp[0], 0};
}

// Combines the partials; writes the offset and flag = 1 when the sum is provably exact
// (then equal to the sequential sum), flag = 0 otherwise.
__global__ void __launch_bounds__(256) k_offset_final(const OffsetPart* __restrict__ part, size_t nb,
                                                      float* __restrict__ offset, int* __restrict__ flag) {
  __shared__ double ssum[kOffsetBlocks];
  __shared__ int sulp[kOffsetBlocks];
  ssum[threadIdx.x] = part[threadIdx.x].sum;
  sulp[threadIdx.x] = part[threadIdx.x].min_ulp;
  __syncthreads();
  for (int o = kOffsetBlocks / 2; o > 0; o >>= 1) {
    if (threadIdx.x < o) {
      ssum[threadIdx.x] += ssum[threadIdx.x + o];
      sulp[threadIdx.x] = min(sulp[threadIdx.x], sulp[threadIdx.x + o]);
    }
    __syncthreads();
  }
  if (threadIdx.x == 0) {
    const double S = ssum[0];
    // every value is a multiple of 2^u and >= 0: if some partial sum had rounded, it
    // (and so S) would be at least 2^(u + 53)
    const bool exact = sulp[0] > 1000 || S < ldexp(1.0, sulp[0] + 52);
    if (exact) *offset = (float)(S / (double)nb);
    *flag = exact ? 1 : 0;
  }
}

__global__ void k_offset_seq(const float* __restrict__ absmax, size_t nb, float* __restrict__ offset,
                             const int* __restrict__ flag) {
  if (threadIdx.x != 0 || blockIdx.x != 0 || *flag) return;
  double acc = 0.0;
  size_t i = 0;
  for (; i + 8 <= nb; i += 8) {
    float v[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) v[j] = absmax[i + j];
#pragma unroll
    for (int j = 0; j < 8; ++j) acc += (double)v[j];
  }
  for (; i < nb; ++i) acc += (double)absmax[i];
  *offset = (float)(acc / (double)nb);
}

__global__ void __launch_bounds__(256) k_nested_q8(const float* __restrict__ absmax, size_t nb,
                                                   const float* __restrict__ offset_p, float* __restrict__ nested,
                                                   uint8_t* __restrict__ q8, const QuantTables tab) {
  __shared__ float mids[256];
  __shared__ float red[8];
  for (int i = threadIdx.x; i < 255; i += blockDim.x) mids[i] = tab.mid8[i];
  const size_t g = blockIdx.x;
  const size_t b = g * 256 + threadIdx.x;
  const float offset = *offset_p;
  const bool valid = b < nb;
  const float c = valid ? __fsub_rn(absmax[b], offset) : 0.f;
  float m = fabsf(c);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = m;
  __syncthreads();
  float nm = red[0];
#pragma unroll
  for (int i = 1; i < 8; ++i) nm = fmaxf(nm, red[i]);
  if (threadIdx.x == 0) nested[g] = nm;
  if (!valid) return;
  int code = tab.zero8;
  if (nm > 0.f) {
    const float u = __fdiv_rn(c, nm);
    int lo = 0, hi = 255;
    while (lo < hi) {
      const int mid = (lo + hi) >> 1;
      if (mids[mid] < u)
        lo = mid + 1;
      else
        hi = mid;
    }
    code = lo;
  }
  q8[b] = (uint8_t)code;
}

__global__ void __launch_bounds__(256) k_dequant(const uint8_t* __restrict__ packed, const uint8_t* __restrict__ q8,
                                                 const float* __restrict__ nested, const float* __restrict__ offset_p,
                                                 size_t n8, __nv_bfloat16* __restrict__ out, const DequantTables tab) {
  __shared__ float nf4[16];
  __shared__ float code8[256];
  for (int i = threadIdx.x; i < 256; i += blockDim.x) code8[i] = tab.code8[i];
  if (threadIdx.x < 16) nf4[threadIdx.x] = tab.nf4[threadIdx.x];
  __syncthreads();
  const float offset = *offset_p;
  for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < n8; i += (size_t)gridDim.x * blockDim.x) {
    const size_t b = i >> 3;  // 8 groups of 8 values per 64-block
    const float s = __fadd_rn(__fmul_rn(code8[q8[b]], nested[b >> 8]), offset);
    const uint32_t word = *reinterpret_cast<const uint32_t*>(packed + i * 4);
    uint32_t o[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const uint32_t byte = (word >> (8 * j)) & 0xFFu;
      o[j] = pack_bf16x2(__fmul_rn(nf4[byte >> 4], s), __fmul_rn(nf4[byte & 0xF], s));
    }
    *reinterpret_cast<uint4*>(out + i * 8) = make_uint4(o[0], o[1], o[2], o[3]);
  }
}

static int sm_count() {
  int dev = 0, n = 148;
  if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
  return n > 0 ? n : 148;
}

int quantize_tensor(const void* w, size_t n, uint8_t* packed, uint8_t* q8, float* nested, float* offset,
                    void* scratch, size_t scratch_bytes, cudaStream_t s) {
  if (!w || !packed || !q8 || !nested || !offset || !scratch)
    return fail(NF4LS_INVALID_ARG, "nf4_quantize_tensor: null pointer");
  if (n == 0 || n % 64) return fail(NF4LS_SHAPE, "nf4_quantize_tensor: n=%zu is not a positive multiple of 64", n);
  if (!aligned(w, 16) || !aligned(packed, 16) || !aligned(scratch, 16))
    return fail(NF4LS_ALIGN, "nf4_quantize_tensor: pointers must be 16-byte aligned");
  const size_t nb = n / 64;
  const size_t am_bytes = round_up(nb * sizeof(float), 256);
  if (scratch_bytes < am_bytes + kOffsetScratch)
    return fail(NF4LS_INVALID_ARG, "nf4_quantize_tensor: scratch too small (%zu < %zu)", scratch_bytes,
                am_bytes + kOffsetScratch);
  const Codebooks& cb = codebooks();
  QuantTables tab;
  std::memcpy(tab.mid4, cb.mid4, sizeof(tab.mid4));
  std::memcpy(tab.mid8, cb.mid8, sizeof(tab.mid8));
  tab.zero4 = cb.zero4;
  tab.zero8 = cb.zero8;
  float* am = static_cast<float*>(scratch);
  const size_t chunks = (nb + 3) / 4;
  const size_t blocks = std::min<size_t>((chunks + 7) / 8, (size_t)sm_count() * 16);
  k_absmax_codes<<<(unsigned)blocks, 256, 0, s>>>(static_cast<const __nv_bfloat16*>(w), nb, packed, am, tab);
  note_launch();
  auto* part = reinterpret_cast<OffsetPart*>(static_cast<uint8_t*>(scratch) + am_bytes);
  int* flag = reinterpret_cast<int*>(part + kOffsetBlocks);
  static_assert(kOffsetBlocks * sizeof(OffsetPart) + sizeof(int) <= kOffsetScratch, "offset scratch");
  k_offset_partial<<<kOffsetBlocks, 256, 0, s>>>(am, nb, part);
  k_offset_final<<<1, kOffsetBlocks, 0, s>>>(part, nb, offset, flag);
  k_offset_seq<<<1, 32, 0, s>>>(am, nb, offset, flag);
  note_launch(3);
  const size_t groups = (nb + 255) / 256;
  k_nested_q8<<<(unsigned)groups, 256, 0, s>>>(am, nb, offset, nested, q8, tab);
  note_launch();
  NF4_CUDA_TRY(cudaGetLastError());
  return NF4LS_OK;
}

int dequantize_tensor(const uint8_t* packed, const uint8_t* q8, const float* nested, const float* offset,
                      size_t n, void* out, cudaStream_t s) {
  if (!packed || !q8 || !nested || !offset || !out) return fail(NF4LS_INVALID_ARG, "nf4_dequantize_tensor: null");
  if (n == 0 || n % 64) return fail(NF4LS_SHAPE, "nf4_dequantize_tensor: n=%zu not a multiple of 64", n);
  if (!aligned(out, 16) || !aligned(packed, 4)) return fail(NF4LS_ALIGN, "nf4_dequantize_tensor: alignment");
  const Codebooks& cb = codebooks();
  DequantTables tab;
  std::memcpy(tab.nf4, cb.nf4, sizeof(tab.nf4));
  std::memcpy(tab.code8, cb.code8, sizeof(tab.code8));
  const size_t n8 = n / 8;
  const size_t blocks = std::min<size_t>((n8 + 255) / 256, (size_t)sm_count() * 8);
  k_dequant<<<(unsigned)blocks, 256, 0, s>>>(packed, q8, nested, offset, n8, static_cast<__nv_bfloat16*>(out), tab);
  note_launch();
  NF4_CUDA_TRY(cudaGetLastError());
  return NF4LS_OK;
}

}  // namespace nf4ls

extern "C" size_t nf4ls_quantize_scratch_bytes(size_t n) {
  return nf4ls::round_up((n / 64) * sizeof(float), 256) + nf4ls::kOffsetScratch;
}

extern "C" int nf4_quantize_tensor(const void* w_dev, size_t n, uint8_t* packed_dev, uint8_t* q8_dev,
                                   float* nested_dev, float* offset_dev, void* scratch_dev, size_t scratch_bytes,
                                   nf4ls_stream stream) {
  nf4ls::clear_error();
  return nf4ls::quantize_tensor(w_dev, n, packed_dev, q8_dev, nested_dev, offset_dev, scratch_dev, scratch_bytes,
                                static_cast<cudaStream_t>(stream));
}

extern "C" int nf4_dequantize_tensor(const uint8_t* packed_dev, const uint8_t* q8_dev, const float* nested_dev,
                                     const float* offset_dev, size_t n, void* out_dev, nf4ls_stream stream) {
  nf4ls::clear_error();
  return nf4ls::dequantize_tensor(packed_dev, q8_dev, nested_dev, offset_dev, n, out_dev,
                                  static_cast<cudaStream_t>(stream));
}
