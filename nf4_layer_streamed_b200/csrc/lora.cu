// K6/K7: the LoRA products of the q_proj and v_proj adapters (r = 16).
//
// "Soup v0.72.4 技术解析" §4.2 (LoRA r=16, alpha=32 on q_proj and v_proj) and
// "Soup 层流式 NF4 训练实测：在 4 GB 显存上以位级一致标准完成 8B 模型 LoRA 微调"
// §2.2 check 2 (LoRA gradients nonzero in every layer): the adapter
// adds s (x A^T) B^T to the q and v projections (s = alpha / r) and trains A and B.
// The up-projection is folded into the q/k/v GEMM as an extra 64-wide reduction
// block; this file holds the skinny products around it, all of them HBM-bound:
//
//   rows:  out[m, 16 j + r] = sum_k X[m, c_j + k] W_j[r, k]
//          forward t = [h1 A_q^T | h1 A_v^T];  backward dt = s [dq B_q | dv B_v]
//   cols:  out[n, r] = sum_m X[m, c + n] Y[m, y + r]
//          dB = s dq^T t (and dv^T t_v);  dA = dt^T h1
//
// Both run on the warp-level bf16 tensor-core instruction (mma.sync m16n8k16) with
// the reduction split across blocks for parallelism (K for rows, M for cols); the
// fp32 partial sums are added in split order by a second kernel, so every result is
// independent of the launch configuration's timing and bit-reproducible.
#include <algorithm>

#include "common.cuh"
#include "internal.h"

namespace nf4ls {

namespace {

constexpr int RS = 72;  // smem row stride (elements) of 64-wide bf16 tiles

struct RowSeg {
  int xcol, K, ldw;
  const __nv_bfloat16* W;
};
struct RowSegs {
  RowSeg s[2];
};

__device__ __forceinline__ void zero16(uint32_t addr) { st_shared_v4(addr, 0u, 0u, 0u, 0u); }

__global__ void __launch_bounds__(128) k_lora_rows(const __nv_bfloat16* __restrict__ X, int ldx, int M, RowSegs segs,
                                                   int nseg, int S, float* __restrict__ part) {
  __shared__ __align__(16) __nv_bfloat16 xs[64 * RS];
  __shared__ __align__(16) __nv_bfloat16 ws[16 * RS];
  const int mb = blockIdx.x, s = blockIdx.y, j = blockIdx.z;
  const RowSeg sg = segs.s[j];
  const int nk = sg.K / 64, per = (nk + S - 1) / S;
  const int kb0 = s * per, kb1 = min(nk, kb0 + per);
  const int t = threadIdx.x, warp = t >> 5, lane = t & 31, g = lane >> 2, c2 = (lane & 3) * 2;
  const uint32_t sx = smem_u32(xs), sw = smem_u32(ws);
  float acc[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
  for (int kb = kb0; kb < kb1; ++kb) {
    for (int i = t; i < 512; i += 128) {
      const int r = i >> 3, c = i & 7, m = mb * 64 + r;
      const uint32_t dst = sx + (r * RS + c * 8) * 2;
      if (m < M)
        cp_async16(dst, X + (size_t)m * ldx + sg.xcol + kb * 64 + c * 8);
      else
        zero16(dst);
    }
    {
      const int r = t >> 3, c = t & 7;
      cp_async16(sw + (r * RS + c * 8) * 2, sg.W + (size_t)r * sg.ldw + kb * 64 + c * 8);
    }
    cp_async_wait_all();
    __syncthreads();
#pragma unroll
    for (int kk = 0; kk < 4; ++kk) {
      uint32_t a[4], b[4];
      {
        const int r = warp * 16 + (lane & 7) + ((lane >> 3) & 1) * 8, c = kk * 16 + (lane >> 4) * 8;
        ldsm4(sx + (r * RS + c) * 2, a[0], a[1], a[2], a[3]);
      }
      {
        const int r = (lane & 7) + (lane >> 4) * 8, c = kk * 16 + ((lane >> 3) & 1) * 8;
        ldsm4(sw + (r * RS + c) * 2, b[0], b[1], b[2], b[3]);
      }
      mma16816(acc[0], a[0], a[1], a[2], a[3], b[0], b[1]);
      mma16816(acc[1], a[0], a[1], a[2], a[3], b[2], b[3]);
    }
    __syncthreads();
  }
  float* P = part + (size_t)(s * nseg + j) * M * 16;
  const int m = mb * 64 + warp * 16 + g;
#pragma unroll
  for (int nt = 0; nt < 2; ++nt) {
    if (m < M) {
      P[(size_t)m * 16 + nt * 8 + c2] = acc[nt][0];
      P[(size_t)m * 16 + nt * 8 + c2 + 1] = acc[nt][1];
    }
    if (m + 8 < M) {
      P[(size_t)(m + 8) * 16 + nt * 8 + c2] = acc[nt][2];
      P[(size_t)(m + 8) * 16 + nt * 8 + c2 + 1] = acc[nt][3];
    }
  }
}

// out_b[m, oc + c] = bf16(scale * sum_s part[s, j, m, r]) with c = 16 j + r (split order fixed).
__global__ void k_lora_rows_reduce(const float* __restrict__ part, int S, int nseg, int M, float scale,
                                   __nv_bfloat16* __restrict__ out_b, int ldb, int oc) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  const int w = 16 * nseg;
  if (i >= M * w) return;
  const int m = i / w, c = i % w, j = c >> 4, r = c & 15;
  float v = 0.f;
  for (int s = 0; s < S; ++s) v += part[((size_t)(s * nseg + j) * M + m) * 16 + r];
  out_b[(size_t)m * ldb + oc + c] = __float2bfloat16_rn(v * scale);
}

template <int NR>
__global__ void __launch_bounds__(128) k_lora_cols(const __nv_bfloat16* __restrict__ X, int ldx, int xcol, int N, int M,
                                                   const __nv_bfloat16* __restrict__ Y, int ldy, int ycol, int S,
                                                   float* __restrict__ part) {
  constexpr int YS = NR + 8;
  __shared__ __align__(16) __nv_bfloat16 xs[64 * RS];
  __shared__ __align__(16) __nv_bfloat16 ys[64 * YS];
  const int nb = blockIdx.x, s = blockIdx.y;
  const int nm = (M + 63) / 64, per = (nm + S - 1) / S;
  const int mb0 = s * per, mb1 = min(nm, mb0 + per);
  const int t = threadIdx.x, warp = t >> 5, lane = t & 31, g = lane >> 2, c2 = (lane & 3) * 2;
  const uint32_t sx = smem_u32(xs), sy = smem_u32(ys);
  float acc[NR / 8][4];
#pragma unroll
  for (int i = 0; i < NR / 8; ++i) acc[i][0] = acc[i][1] = acc[i][2] = acc[i][3] = 0.f;
  for (int mbk = mb0; mbk < mb1; ++mbk) {
    for (int i = t; i < 512; i += 128) {
      const int r = i >> 3, c = i & 7, m = mbk * 64 + r;
      const uint32_t dst = sx + (r * RS + c * 8) * 2;
      if (m < M)
        cp_async16(dst, X + (size_t)m * ldx + xcol + nb * 64 + c * 8);
      else
        zero16(dst);
    }
    for (int i = t; i < 64 * (NR / 8); i += 128) {
      const int r = i / (NR / 8), c = i % (NR / 8), m = mbk * 64 + r;
      const uint32_t dst = sy + (r * YS + c * 8) * 2;
      if (m < M)
        cp_async16(dst, Y + (size_t)m * ldy + ycol + c * 8);
      else
        zero16(dst);
    }
    cp_async_wait_all();
    __syncthreads();
#pragma unroll
    for (int kk = 0; kk < 4; ++kk) {
      uint32_t a[4];
      {  // A[n][m] = X[m][n]: transposed 8x8 blocks of the [m][n] tile
        const int m = kk * 16 + (lane & 7) + (lane >> 4) * 8, n = warp * 16 + ((lane >> 3) & 1) * 8;
        ldsm4t(sx + (m * RS + n) * 2, a[0], a[1], a[2], a[3]);
      }
#pragma unroll
      for (int h = 0; h < NR / 16; ++h) {
        uint32_t b[4];
        const int m = kk * 16 + (lane & 7) + ((lane >> 3) & 1) * 8, n = h * 16 + (lane >> 4) * 8;
        ldsm4t(sy + (m * YS + n) * 2, b[0], b[1], b[2], b[3]);
        mma16816(acc[2 * h], a[0], a[1], a[2], a[3], b[0], b[1]);
        mma16816(acc[2 * h + 1], a[0], a[1], a[2], a[3], b[2], b[3]);
      }
    }
    __syncthreads();
  }
  float* P = part + (size_t)s * N * NR;
  const int n = nb * 64 + warp * 16 + g;
#pragma unroll
  for (int nt = 0; nt < NR / 8; ++nt) {
    P[(size_t)n * NR + nt * 8 + c2] = acc[nt][0];
    P[(size_t)n * NR + nt * 8 + c2 + 1] = acc[nt][1];
    P[(size_t)(n + 8) * NR + nt * 8 + c2] = acc[nt][2];
    P[(size_t)(n + 8) * NR + nt * 8 + c2 + 1] = acc[nt][3];
  }
}

// out_{r/16}[n * so_n + (r % 16) * so_r] = scale * sum_s part[s, n, r] (split order fixed).
__global__ void k_lora_cols_reduce(const float* __restrict__ part, int S, int N, int NR, float scale,
                                   float* __restrict__ out0, float* __restrict__ out1, int so_n, int so_r) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= N * NR) return;
  const int n = i / NR, r = i % NR;
  float v = 0.f;
  for (int s = 0; s < S; ++s) v += part[((size_t)s * N + n) * NR + r];
  float* o = r < 16 ? out0 : out1;
  o[(size_t)n * so_n + (size_t)(r & 15) * so_r] = v * scale;
}

// bf16 operands of the adapter, from the fp32 masters:
//   bup [Nqkv, 64]: q rows: s*B_q in cols 0-15; v rows: s*B_v in cols 16-31; else 0
//   adn [64, H]   : rows 0-15 A_q, rows 16-31 A_v, else 0
//   bqt [16, qd] = B_q^T, bvt [16, kvd] = B_v^T
__global__ void k_lora_pack(const float* __restrict__ Aq, const float* __restrict__ Bq, const float* __restrict__ Av,
                            const float* __restrict__ Bv, int H, int qd, int kvd, float scale,
                            __nv_bfloat16* __restrict__ bup, __nv_bfloat16* __restrict__ adn,
                            __nv_bfloat16* __restrict__ bqt, __nv_bfloat16* __restrict__ bvt) {
  const int nq = qd + 2 * kvd;
  const size_t n1 = (size_t)nq * 64, n2 = (size_t)64 * H, n3 = (size_t)16 * qd, n4 = (size_t)16 * kvd;
  size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x;
  if (i < n1) {
    const int n = (int)(i / 64), c = (int)(i % 64);
    float v = 0.f;
    if (n < qd && c < 16)
      v = scale * __bfloat162float(__float2bfloat16_rn(Bq[(size_t)n * 16 + c]));
    else if (n >= qd + kvd && c >= 16 && c < 32)
      v = scale * __bfloat162float(__float2bfloat16_rn(Bv[(size_t)(n - qd - kvd) * 16 + c - 16]));
    bup[i] = __float2bfloat16_rn(v);
    return;
  }
  i -= n1;
  if (i < n2) {
    const int r = (int)(i / H), k = (int)(i % H);
    float v = 0.f;
    if (r < 16)
      v = Aq[(size_t)r * H + k];
    else if (r < 32)
      v = Av[(size_t)(r - 16) * H + k];
    adn[i] = __float2bfloat16_rn(v);
    return;
  }
  i -= n2;
  if (i < n3) {
    const int r = (int)(i / qd), n = (int)(i % qd);
    bqt[i] = __float2bfloat16_rn(Bq[(size_t)n * 16 + r]);
    return;
  }
  i -= n3;
  if (i < n4) {
    const int r = (int)(i / kvd), n = (int)(i % kvd);
    bvt[i] = __float2bfloat16_rn(Bv[(size_t)n * 16 + r]);
  }
}

int splits_for(int units, int blocks_other) {
  int s = 1;
  while (s < 8 && s * 2 <= units && blocks_other * s < 256) s *= 2;
  return s;
}

}  // namespace

size_t lora_partial_bytes(int M, int Nmax) {
  const size_t rows = 8ull * 2 * (size_t)M * 16 * 4, cols = 8ull * (size_t)Nmax * 32 * 4;
  return std::max(rows, cols);
}

int lora_pack2(const nf4ls_lora* l, int H, int qd, int kvd, float scale, __nv_bfloat16* bup, __nv_bfloat16* adn,
               __nv_bfloat16* bqt, __nv_bfloat16* bvt, cudaStream_t s) {
  const size_t n = (size_t)(qd + 2 * kvd) * 64 + (size_t)64 * H + 16ull * qd + 16ull * kvd;
  k_lora_pack<<<(unsigned)((n + 255) / 256), 256, 0, s>>>(l->A_q, l->B_q, l->A_v, l->B_v, H, qd, kvd, scale, bup, adn,
                                                           bqt, bvt);
  note_launch();
  NF4_CUDA_TRY(cudaGetLastError());
  return NF4LS_OK;
}

// out_b[:, oc + 16 j + r] = bf16(scale * X[:, xcol_j : xcol_j + K_j] W_j^T), W_j [16, K_j] bf16.
int lora_rows(const __nv_bfloat16* X, int ldx, int M, int nseg, const int* xcol, const int* K,
              const __nv_bfloat16* const* W, const int* ldw, float scale, float* part, __nv_bfloat16* out_b, int ldb,
              int oc, cudaStream_t s) {
  RowSegs sg;
  int kmin = 1 << 30;
  for (int j = 0; j < nseg; ++j) {
    if (K[j] % 64 || xcol[j] % 8 || ldw[j] % 8) return fail(NF4LS_SHAPE, "lora_rows: K %% 64, alignment");
    sg.s[j] = RowSeg{xcol[j], K[j], ldw[j], W[j]};
    kmin = std::min(kmin, K[j] / 64);
  }
  const int mb = (M + 63) / 64;
  // The split of K depends on K only, so a row's sum is grouped the same way for any
  // M: a token's result does not depend on how many tokens share the launch.
  const int S = std::min(8, kmin);
  k_lora_rows<<<dim3(mb, S, nseg), 128, 0, s>>>(X, ldx, M, sg, nseg, S, part);
  note_launch();
  const int n = M * 16 * nseg;
  k_lora_rows_reduce<<<(n + 255) / 256, 256, 0, s>>>(part, S, nseg, M, scale, out_b, ldb, oc);
  note_launch();
  NF4_CUDA_TRY(cudaGetLastError());
  return NF4LS_OK;
}

// out{0,1}[n * so_n + r * so_r] = scale * sum_m X[m, xcol + n] Y[m, ycol + r], r < NR (16 or 32).
int lora_cols(const __nv_bfloat16* X, int ldx, int xcol, int N, int M, const __nv_bfloat16* Y, int ldy, int ycol,
              int NR, float scale, float* part, float* out0, float* out1, int so_n, int so_r, cudaStream_t s) {
  if (N % 64 || xcol % 8 || ycol % 8 || ldx % 8 || ldy % 8) return fail(NF4LS_SHAPE, "lora_cols: shape/alignment");
  const int nb = N / 64;
  const int S = splits_for((M + 63) / 64, nb);
  if (NR == 16)
    k_lora_cols<16><<<dim3(nb, S), 128, 0, s>>>(X, ldx, xcol, N, M, Y, ldy, ycol, S, part);
  else
    k_lora_cols<32><<<dim3(nb, S), 128, 0, s>>>(X, ldx, xcol, N, M, Y, ldy, ycol, S, part);
  note_launch();
  k_lora_cols_reduce<<<(N * NR + 255) / 256, 256, 0, s>>>(part, S, N, NR, scale, out0, out1, so_n, so_r);
  note_launch();
  NF4_CUDA_TRY(cudaGetLastError());
  return NF4LS_OK;
}

}  // namespace nf4ls
