// K10: causal grouped-query attention, forward and deterministic backward.
//
// The attention of the HF Llama decoder layer that the pages' system runs through
// functional_call ("Soup 层流式 NF4 训练实测：在 4 GB 显存上以位级一致标准完成 8B 模型 LoRA 微调" §2.1): softmax(q k^T / sqrt(d)
// + causal mask) v, with key/value head h / (n_q / n_kv) serving query head h.
// At seq 512 it is about 2% of the layer's FLOPs (the GEMM share table of §4.4 leaves
// it out), so this round uses the warp-level bf16 tensor-core instruction
// (mma.sync m16n8k16) in a flash-attention layout: 64-query x 64-key tiles, online
// softmax in fp32, P rounded to bf16 for the P v product, the log-sum-exp saved for
// the backward.
//
// Backward: delta = rowsum(dO * O); dK and dV per 64-key tile loop over every query
// head of the group and every query tile at or after the key tile, in a fixed order;
// dQ per 64-query tile loops over key tiles.  No atomics, so results are
// bit-reproducible.  seq must be a multiple of 64.
#include <cmath>

#include "common.cuh"
#include "internal.h"

namespace nf4ls {

namespace {

constexpr int TQ = 64, TK = 64;
constexpr float kLog2e = 1.4426950408889634f;

// Tile of 64 rows x D bf16 in shared memory, row stride D + 8 elements (ldmatrix
// reads of 8 consecutive rows fall in distinct bank groups).
template <int D>
struct Tile {
  static constexpr int RS = D + 8;
  static constexpr int BYTES = 64 * RS * 2;
};

template <int D>
__device__ __forceinline__ void load_tile(uint32_t dst, const __nv_bfloat16* src, int ld) {
  constexpr int CH = D / 8;  // 16-byte chunks per row
  for (int i = threadIdx.x; i < 64 * CH; i += blockDim.x) {
    const int r = i / CH, c = i % CH;
    cp_async16(dst + (r * Tile<D>::RS + c * 8) * 2, src + (size_t)r * ld + c * 8);
  }
}

// Group-local cp.async tile load: threads t of n.
template <int D>
__device__ __forceinline__ void load_tile_part(uint32_t dst, const __nv_bfloat16* src, int ld, int t, int n) {
  constexpr int CH = D / 8;
  for (int i = t; i < 64 * CH; i += n) {
    const int r = i / CH, c = i % CH;
    cp_async16(dst + (r * Tile<D>::RS + c * 8) * 2, src + (size_t)r * ld + c * 8);
  }
}

__device__ __forceinline__ void cp_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}
__device__ __forceinline__ void bar_group(int id, int n) { asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(n) : "memory"); }

// A fragment (16x16 at row0, col0) of a row-major tile.
template <int D>
__device__ __forceinline__ void frag_a(uint32_t tile, int row0, int col0, uint32_t (&a)[4]) {
  const int i = threadIdx.x & 31;
  const int r = row0 + (i & 7) + ((i >> 3) & 1) * 8, c = col0 + (i >> 4) * 8;
  ldsm4(tile + (r * Tile<D>::RS + c) * 2, a[0], a[1], a[2], a[3]);
}
// B fragments of two n-tiles (n0, n0+8), k = k0..k0+15, from a tile whose rows are n.
template <int D>
__device__ __forceinline__ void frag_b_rows_n(uint32_t tile, int n0, int k0, uint32_t (&b)[4]) {
  const int i = threadIdx.x & 31;
  const int r = n0 + (i & 7) + (i >> 4) * 8, c = k0 + ((i >> 3) & 1) * 8;
  ldsm4(tile + (r * Tile<D>::RS + c) * 2, b[0], b[1], b[2], b[3]);
}
// B fragments of two n-tiles (n0, n0+8), k = k0..k0+15, from a tile whose rows are k.
template <int D>
__device__ __forceinline__ void frag_b_rows_k(uint32_t tile, int k0, int n0, uint32_t (&b)[4]) {
  const int i = threadIdx.x & 31;
  const int r = k0 + (i & 7) + ((i >> 3) & 1) * 8, c = n0 + (i >> 4) * 8;
  ldsm4t(tile + (r * Tile<D>::RS + c) * 2, b[0], b[1], b[2], b[3]);
}

// ------------------------------------------------------------------------------ forward
template <int D>
__global__ void __launch_bounds__(128) k_attn_fwd(const __nv_bfloat16* __restrict__ q, const __nv_bfloat16* __restrict__ k,
                                                  const __nv_bfloat16* __restrict__ v, int ldq, int ldkv,
                                                  __nv_bfloat16* __restrict__ o, int ldo, float* __restrict__ lse,
                                                  int seq, int nq, int nkv, float scale_log2) {
  extern __shared__ __align__(16) uint8_t sm[];
  // Q, then two K/V buffers: the next key tile loads while this one is used
  const uint32_t sQ = smem_u32(sm);
  const int qt = gridDim.x - 1 - blockIdx.x, h = blockIdx.y, b = blockIdx.z;  // longest rows first
  const int kvh = h / (nq / nkv);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, g = lane >> 2, c2 = (lane & 3) * 2;
  const size_t row0 = (size_t)b * seq;
  load_tile<D>(sQ, q + (row0 + qt * TQ) * ldq + h * D, ldq);
  load_tile<D>(sQ + Tile<D>::BYTES, k + row0 * ldkv + kvh * D, ldkv);
  load_tile<D>(sQ + 2 * Tile<D>::BYTES, v + row0 * ldkv + kvh * D, ldkv);
  cp_commit();
  float acc[D / 8][4];
#pragma unroll
  for (int i = 0; i < D / 8; ++i) acc[i][0] = acc[i][1] = acc[i][2] = acc[i][3] = 0.f;
  float mrow[2] = {-INFINITY, -INFINITY}, lrow[2] = {0.f, 0.f};
  for (int kt = 0; kt <= qt; ++kt) {
    const uint32_t sK = sQ + (1 + 2 * (kt & 1)) * Tile<D>::BYTES, sV = sK + Tile<D>::BYTES;
    if (kt < qt) {  // the buffer of tile kt + 1 was last read in iteration kt - 1 (barrier below)
      const uint32_t nK = sQ + (1 + 2 * ((kt + 1) & 1)) * Tile<D>::BYTES;
      load_tile<D>(nK, k + (row0 + (kt + 1) * TK) * ldkv + kvh * D, ldkv);
      load_tile<D>(nK + Tile<D>::BYTES, v + (row0 + (kt + 1) * TK) * ldkv + kvh * D, ldkv);
      cp_commit();
      cp_wait<1>();
    } else {
      cp_wait<0>();
    }
    __syncthreads();
    float s[8][4];
#pragma unroll
    for (int i = 0; i < 8; ++i) s[i][0] = s[i][1] = s[i][2] = s[i][3] = 0.f;
#pragma unroll
    for (int kk = 0; kk < D / 16; ++kk) {
      uint32_t a[4];
      frag_a<D>(sQ, warp * 16, kk * 16, a);
#pragma unroll
      for (int n2 = 0; n2 < 4; ++n2) {
        uint32_t bb[4];
        frag_b_rows_n<D>(sK, n2 * 16, kk * 16, bb);
        mma16816(s[2 * n2], a[0], a[1], a[2], a[3], bb[0], bb[1]);
        mma16816(s[2 * n2 + 1], a[0], a[1], a[2], a[3], bb[2], bb[3]);
      }
    }
    // scale, causal mask on the diagonal tile, online softmax
    float mx[2] = {mrow[0], mrow[1]};
#pragma unroll
    for (int nt = 0; nt < 8; ++nt)
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        float x = s[nt][e] * scale_log2;
        if (kt == qt) {
          const int qi = warp * 16 + g + (e >> 1) * 8, kj = nt * 8 + c2 + (e & 1);
          if (kj > qi) x = -INFINITY;
        }
        s[nt][e] = x;
        mx[e >> 1] = fmaxf(mx[e >> 1], x);
      }
#pragma unroll
    for (int r = 0; r < 2; ++r) {
      mx[r] = fmaxf(mx[r], __shfl_xor_sync(0xffffffffu, mx[r], 1));
      mx[r] = fmaxf(mx[r], __shfl_xor_sync(0xffffffffu, mx[r], 2));
    }
    float corr[2];
#pragma unroll
    for (int r = 0; r < 2; ++r) {
      corr[r] = exp2f(mrow[r] - mx[r]);
      mrow[r] = mx[r];
      lrow[r] *= corr[r];
    }
#pragma unroll
    for (int nt = 0; nt < 8; ++nt)
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float p = exp2f(s[nt][e] - mrow[e >> 1]);
        s[nt][e] = p;
        lrow[e >> 1] += p;
      }
#pragma unroll
    for (int i = 0; i < D / 8; ++i) {
      acc[i][0] *= corr[0];
      acc[i][1] *= corr[0];
      acc[i][2] *= corr[1];
      acc[i][3] *= corr[1];
    }
#pragma unroll
    for (int kb = 0; kb < 4; ++kb) {
      const uint32_t a0 = pack_bf16x2(s[2 * kb][0], s[2 * kb][1]), a1 = pack_bf16x2(s[2 * kb][2], s[2 * kb][3]);
      const uint32_t a2 = pack_bf16x2(s[2 * kb + 1][0], s[2 * kb + 1][1]),
                     a3 = pack_bf16x2(s[2 * kb + 1][2], s[2 * kb + 1][3]);
#pragma unroll
      for (int n2 = 0; n2 < D / 16; ++n2) {
        uint32_t bb[4];
        frag_b_rows_k<D>(sV, kb * 16, n2 * 16, bb);
        mma16816(acc[2 * n2], a0, a1, a2, a3, bb[0], bb[1]);
        mma16816(acc[2 * n2 + 1], a0, a1, a2, a3, bb[2], bb[3]);
      }
    }
    __syncthreads();
  }
#pragma unroll
  for (int r = 0; r < 2; ++r) {
    lrow[r] += __shfl_xor_sync(0xffffffffu, lrow[r], 1);
    lrow[r] += __shfl_xor_sync(0xffffffffu, lrow[r], 2);
  }
  const float inv0 = 1.0f / lrow[0], inv1 = 1.0f / lrow[1];
  const int r0 = qt * TQ + warp * 16 + g;
  __nv_bfloat16* o0 = o + (row0 + r0) * ldo + h * D;
  __nv_bfloat16* o1 = o0 + 8 * (size_t)ldo;
#pragma unroll
  for (int i = 0; i < D / 8; ++i) {
    *reinterpret_cast<uint32_t*>(o0 + i * 8 + c2) = pack_bf16x2(acc[i][0] * inv0, acc[i][1] * inv0);
    *reinterpret_cast<uint32_t*>(o1 + i * 8 + c2) = pack_bf16x2(acc[i][2] * inv1, acc[i][3] * inv1);
  }
  if ((lane & 3) == 0) {
    const float ln2 = 0.6931471805599453f;
    float* L = lse + ((size_t)b * nq + h) * seq;
    L[r0] = (mrow[0] + log2f(lrow[0])) * ln2;
    L[r0 + 8] = (mrow[1] + log2f(lrow[1])) * ln2;
  }
}

// ------------------------------------------------------------------------------ backward
// delta[b, h, s] = sum_d dO * O (fp32), one warp per (row, head).
__global__ void k_attn_delta(const __nv_bfloat16* __restrict__ o, const __nv_bfloat16* __restrict__ dout, int ldo, int M,
                             int seq, int nq, int d, float* __restrict__ delta) {
  const int w = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (w >= M * nq) return;
  const int m = w / nq, h = w % nq;
  const __nv_bfloat16* a = o + (size_t)m * ldo + h * d;
  const __nv_bfloat16* bb = dout + (size_t)m * ldo + h * d;
  float s = 0.f;
  for (int i = lane; i < d; i += 32) s += __bfloat162float(a[i]) * __bfloat162float(bb[i]);
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) s += __shfl_xor_sync(0xffffffffu, s, off);
  if (lane == 0) {
    const int bi = m / seq, si = m % seq;
    delta[((size_t)bi * nq + h) * seq + si] = s;
  }
}

template <int D>
__global__ void __launch_bounds__(128) k_attn_dq(const __nv_bfloat16* __restrict__ q, const __nv_bfloat16* __restrict__ k,
                                                 const __nv_bfloat16* __restrict__ v, int ldq, int ldkv,
                                                 const __nv_bfloat16* __restrict__ dout, int ldo,
                                                 const float* __restrict__ lse, const float* __restrict__ delta,
                                                 __nv_bfloat16* __restrict__ dq, int ld_dq, int seq, int nq, int nkv,
                                                 float scale) {
  extern __shared__ __align__(16) uint8_t sm[];
  // Q, dO, then two K/V buffers: the next key tile loads while this one is used
  const uint32_t sQ = smem_u32(sm), sO = sQ + Tile<D>::BYTES;
  const int qt = gridDim.x - 1 - blockIdx.x, h = blockIdx.y, b = blockIdx.z;  // longest rows first
  const int kvh = h / (nq / nkv);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, g = lane >> 2, c2 = (lane & 3) * 2;
  const size_t row0 = (size_t)b * seq;
  const float scale_log2 = scale * kLog2e;
  load_tile<D>(sQ, q + (row0 + qt * TQ) * ldq + h * D, ldq);
  load_tile<D>(sO, dout + (row0 + qt * TQ) * ldo + h * D, ldo);
  load_tile<D>(sQ + 2 * Tile<D>::BYTES, k + row0 * ldkv + kvh * D, ldkv);
  load_tile<D>(sQ + 3 * Tile<D>::BYTES, v + row0 * ldkv + kvh * D, ldkv);
  cp_commit();
  const int qr = qt * TQ + warp * 16 + g;
  const float* Lh = lse + ((size_t)b * nq + h) * seq;
  const float* Dh = delta + ((size_t)b * nq + h) * seq;
  const float lse2[2] = {Lh[qr] * kLog2e, Lh[qr + 8] * kLog2e};
  const float dl[2] = {Dh[qr], Dh[qr + 8]};
  float acc[D / 8][4];
#pragma unroll
  for (int i = 0; i < D / 8; ++i) acc[i][0] = acc[i][1] = acc[i][2] = acc[i][3] = 0.f;
  for (int kt = 0; kt <= qt; ++kt) {
    const uint32_t sK = sQ + (2 + 2 * (kt & 1)) * Tile<D>::BYTES, sV = sK + Tile<D>::BYTES;
    if (kt < qt) {
      const uint32_t nK = sQ + (2 + 2 * ((kt + 1) & 1)) * Tile<D>::BYTES;
      load_tile<D>(nK, k + (row0 + (kt + 1) * TK) * ldkv + kvh * D, ldkv);
      load_tile<D>(nK + Tile<D>::BYTES, v + (row0 + (kt + 1) * TK) * ldkv + kvh * D, ldkv);
      cp_commit();
      cp_wait<1>();
    } else {
      cp_wait<0>();
    }
    __syncthreads();
    float s[8][4], dp[8][4];
#pragma unroll
    for (int i = 0; i < 8; ++i)
#pragma unroll
      for (int e = 0; e < 4; ++e) s[i][e] = dp[i][e] = 0.f;
#pragma unroll
    for (int kk = 0; kk < D / 16; ++kk) {
      uint32_t a[4], ao[4];
      frag_a<D>(sQ, warp * 16, kk * 16, a);
      frag_a<D>(sO, warp * 16, kk * 16, ao);
#pragma unroll
      for (int n2 = 0; n2 < 4; ++n2) {
        uint32_t bk[4], bv[4];
        frag_b_rows_n<D>(sK, n2 * 16, kk * 16, bk);
        frag_b_rows_n<D>(sV, n2 * 16, kk * 16, bv);
        mma16816(s[2 * n2], a[0], a[1], a[2], a[3], bk[0], bk[1]);
        mma16816(s[2 * n2 + 1], a[0], a[1], a[2], a[3], bk[2], bk[3]);
        mma16816(dp[2 * n2], ao[0], ao[1], ao[2], ao[3], bv[0], bv[1]);
        mma16816(dp[2 * n2 + 1], ao[0], ao[1], ao[2], ao[3], bv[2], bv[3]);
      }
    }
#pragma unroll
    for (int nt = 0; nt < 8; ++nt)
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        float p = exp2f(s[nt][e] * scale_log2 - lse2[e >> 1]);
        if (kt == qt) {
          const int qi = warp * 16 + g + (e >> 1) * 8, kj = nt * 8 + c2 + (e & 1);
          if (kj > qi) p = 0.f;
        }
        s[nt][e] = p * (dp[nt][e] - dl[e >> 1]);  // dS
      }
#pragma unroll
    for (int kb = 0; kb < 4; ++kb) {
      const uint32_t a0 = pack_bf16x2(s[2 * kb][0], s[2 * kb][1]), a1 = pack_bf16x2(s[2 * kb][2], s[2 * kb][3]);
      const uint32_t a2 = pack_bf16x2(s[2 * kb + 1][0], s[2 * kb + 1][1]),
                     a3 = pack_bf16x2(s[2 * kb + 1][2], s[2 * kb + 1][3]);
#pragma unroll
      for (int n2 = 0; n2 < D / 16; ++n2) {
        uint32_t bb[4];
        frag_b_rows_k<D>(sK, kb * 16, n2 * 16, bb);
        mma16816(acc[2 * n2], a0, a1, a2, a3, bb[0], bb[1]);
        mma16816(acc[2 * n2 + 1], a0, a1, a2, a3, bb[2], bb[3]);
      }
    }
    __syncthreads();
  }
  __nv_bfloat16* o0 = dq + (row0 + qr) * ld_dq + h * D;
  __nv_bfloat16* o1 = o0 + 8 * (size_t)ld_dq;
#pragma unroll
  for (int i = 0; i < D / 8; ++i) {
    *reinterpret_cast<uint32_t*>(o0 + i * 8 + c2) = pack_bf16x2(acc[i][0] * scale, acc[i][1] * scale);
    *reinterpret_cast<uint32_t*>(o1 + i * 8 + c2) = pack_bf16x2(acc[i][2] * scale, acc[i][3] * scale);
  }
}

// dK, dV of one 64-key tile of one kv head: two groups of 4 warps split the work
// (query heads of the group x query tiles at or after the key tile; group w takes the
// tiles kt + w, kt + w + 2, ...), each group double-buffers its Q / dO tiles so the
// next pair loads while this one is used, and the two partial sums are added in a
// fixed order (group 0 + group 1) at the end.
template <int D>
__global__ void __launch_bounds__(256, 1) k_attn_dkv(const __nv_bfloat16* __restrict__ q, const __nv_bfloat16* __restrict__ k,
                                                     const __nv_bfloat16* __restrict__ v, int ldq, int ldkv,
                                                     const __nv_bfloat16* __restrict__ dout, int ldo,
                                                     const float* __restrict__ lse, const float* __restrict__ delta,
                                                     __nv_bfloat16* __restrict__ dk, __nv_bfloat16* __restrict__ dv,
                                                     int ld_dkv, int seq, int nq, int nkv, float scale) {
  constexpr int T = Tile<D>::BYTES;
  extern __shared__ __align__(16) uint8_t sm[];
  const uint32_t sK = smem_u32(sm), sV = sK + T;
  const int kvh = blockIdx.x, b = blockIdx.y, kt = blockIdx.z;  // z slowest: the longest key tiles start first
  const int grp = nq / nkv;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, g = lane >> 2, c2 = (lane & 3) * 2;
  const int wg = warp >> 2, wq = warp & 3, tg = threadIdx.x & 127;
  const size_t row0 = (size_t)b * seq;
  const float scale_log2 = scale * kLog2e;
  const int n_qt = seq / TQ;
  const int per_head = (n_qt - kt - wg + 1) / 2;  // query tiles kt + wg + 2j of this group
  const int n_it = per_head > 0 ? grp * per_head : 0;
  // buffer j of this group: Q, dO tiles and the 64 lse / delta values
  auto buf_q = [&](int j) { return sK + (2 + wg * 4 + j * 2) * T; };
  float* ld_base = reinterpret_cast<float*>(sm + 10 * T) + (wg * 2) * 128;
  auto load_item = [&](int i, int j) {
    const int hh = i / per_head, qt = kt + wg + 2 * (i % per_head);
    const int h = kvh * grp + hh;
    const uint32_t bq = buf_q(j);
    load_tile_part<D>(bq, q + (row0 + qt * TQ) * ldq + h * D, ldq, tg, 128);
    load_tile_part<D>(bq + T, dout + (row0 + qt * TQ) * ldo + h * D, ldo, tg, 128);
    if (tg < 32) {  // 64 lse then 64 delta values, 16 bytes per thread
      const float* src = (tg < 16 ? lse : delta) + ((size_t)b * nq + h) * seq + qt * TQ + (tg & 15) * 4;
      cp_async16(smem_u32(ld_base + j * 128 + (tg < 16 ? 0 : 64) + (tg & 15) * 4), src);
    }
  };
  load_tile<D>(sK, k + (row0 + kt * TK) * ldkv + kvh * D, ldkv);
  load_tile<D>(sV, v + (row0 + kt * TK) * ldkv + kvh * D, ldkv);
  if (n_it > 0) load_item(0, 0);
  cp_commit();
  cp_wait<0>();
  __syncthreads();
  float dK[D / 8][4], dV[D / 8][4];
#pragma unroll
  for (int i = 0; i < D / 8; ++i)
#pragma unroll
    for (int e = 0; e < 4; ++e) dK[i][e] = dV[i][e] = 0.f;
  for (int it = 0; it < n_it; ++it) {
    const int j = it & 1;
    if (it + 1 < n_it) {
      load_item(it + 1, j ^ 1);
      cp_commit();
    }
    const int qt = kt + wg + 2 * (it % per_head);
    const uint32_t sQ = buf_q(j), sO = sQ + T;
    const float* sL = ld_base + j * 128;
    const float* sD = sL + 64;
    // S^T = K Q^T and dP^T = V dO^T for this warp's 16 keys x 64 queries
    float s[8][4], dp[8][4];
#pragma unroll
    for (int i = 0; i < 8; ++i)
#pragma unroll
      for (int e = 0; e < 4; ++e) s[i][e] = dp[i][e] = 0.f;
#pragma unroll
    for (int kk = 0; kk < D / 16; ++kk) {
      uint32_t ak[4], av[4];
      frag_a<D>(sK, wq * 16, kk * 16, ak);
      frag_a<D>(sV, wq * 16, kk * 16, av);
#pragma unroll
      for (int n2 = 0; n2 < 4; ++n2) {
        uint32_t bq[4], bo[4];
        frag_b_rows_n<D>(sQ, n2 * 16, kk * 16, bq);
        frag_b_rows_n<D>(sO, n2 * 16, kk * 16, bo);
        mma16816(s[2 * n2], ak[0], ak[1], ak[2], ak[3], bq[0], bq[1]);
        mma16816(s[2 * n2 + 1], ak[0], ak[1], ak[2], ak[3], bq[2], bq[3]);
        mma16816(dp[2 * n2], av[0], av[1], av[2], av[3], bo[0], bo[1]);
        mma16816(dp[2 * n2 + 1], av[0], av[1], av[2], av[3], bo[2], bo[3]);
      }
    }
    // P^T and dS^T; column e&1 of n-tile nt is query nt*8 + c2 + (e&1)
#pragma unroll
    for (int nt = 0; nt < 8; ++nt)
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int qj = nt * 8 + c2 + (e & 1);
        float p = exp2f(s[nt][e] * scale_log2 - sL[qj] * kLog2e);
        if (qt == kt) {
          const int ki = wq * 16 + g + (e >> 1) * 8;
          if (ki > qj) p = 0.f;
        }
        s[nt][e] = p;
        dp[nt][e] = p * (dp[nt][e] - sD[qj]);
      }
#pragma unroll
    for (int kb = 0; kb < 4; ++kb) {
      const uint32_t p0 = pack_bf16x2(s[2 * kb][0], s[2 * kb][1]), p1 = pack_bf16x2(s[2 * kb][2], s[2 * kb][3]);
      const uint32_t p2 = pack_bf16x2(s[2 * kb + 1][0], s[2 * kb + 1][1]),
                     p3 = pack_bf16x2(s[2 * kb + 1][2], s[2 * kb + 1][3]);
      const uint32_t d0 = pack_bf16x2(dp[2 * kb][0], dp[2 * kb][1]), d1 = pack_bf16x2(dp[2 * kb][2], dp[2 * kb][3]);
      const uint32_t d2 = pack_bf16x2(dp[2 * kb + 1][0], dp[2 * kb + 1][1]),
                     d3 = pack_bf16x2(dp[2 * kb + 1][2], dp[2 * kb + 1][3]);
#pragma unroll
      for (int n2 = 0; n2 < D / 16; ++n2) {
        uint32_t bo[4], bq[4];
        frag_b_rows_k<D>(sO, kb * 16, n2 * 16, bo);
        frag_b_rows_k<D>(sQ, kb * 16, n2 * 16, bq);
        mma16816(dV[2 * n2], p0, p1, p2, p3, bo[0], bo[1]);
        mma16816(dV[2 * n2 + 1], p0, p1, p2, p3, bo[2], bo[3]);
        mma16816(dK[2 * n2], d0, d1, d2, d3, bq[0], bq[1]);
        mma16816(dK[2 * n2 + 1], d0, d1, d2, d3, bq[2], bq[3]);
      }
    }
    if (it + 1 < n_it) cp_wait<0>();
    bar_group(1 + wg, 128);  // the next item is in; nobody still reads this buffer
  }
  // group 1 hands its partial sums to group 0 through the (now free) tile memory
  __syncthreads();
  float* red = reinterpret_cast<float*>(sm + 2 * T);  // [D/8 * 4 * 2][128], thread-major
  if (wg == 1) {
#pragma unroll
    for (int i = 0; i < D / 8; ++i)
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        red[((i * 4 + e) * 2 + 0) * 128 + tg] = dK[i][e];
        red[((i * 4 + e) * 2 + 1) * 128 + tg] = dV[i][e];
      }
  }
  __syncthreads();
  if (wg == 1) return;
#pragma unroll
  for (int i = 0; i < D / 8; ++i)
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      dK[i][e] += red[((i * 4 + e) * 2 + 0) * 128 + tg];
      dV[i][e] += red[((i * 4 + e) * 2 + 1) * 128 + tg];
    }
  const int kr = kt * TK + wq * 16 + g;
  __nv_bfloat16* k0 = dk + (row0 + kr) * ld_dkv + kvh * D;
  __nv_bfloat16* v0 = dv + (row0 + kr) * ld_dkv + kvh * D;
  const size_t step = 8 * (size_t)ld_dkv;
#pragma unroll
  for (int i = 0; i < D / 8; ++i) {
    *reinterpret_cast<uint32_t*>(k0 + i * 8 + c2) = pack_bf16x2(dK[i][0] * scale, dK[i][1] * scale);
    *reinterpret_cast<uint32_t*>(k0 + step + i * 8 + c2) = pack_bf16x2(dK[i][2] * scale, dK[i][3] * scale);
    *reinterpret_cast<uint32_t*>(v0 + i * 8 + c2) = pack_bf16x2(dV[i][0], dV[i][1]);
    *reinterpret_cast<uint32_t*>(v0 + step + i * 8 + c2) = pack_bf16x2(dV[i][2], dV[i][3]);
  }
}

template <typename F>
int set_smem(F* f, int bytes) {
  NF4_CUDA_TRY(cudaFuncSetAttribute(f, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes));
  return NF4LS_OK;
}

int check_attn(int seq, int nq, int nkv, int d, int ldq, int ldkv) {
  if (seq % 64) return fail(NF4LS_SHAPE, "attention: seq must be a multiple of 64 (got %d)", seq);
  if (d != 64 && d != 128) return fail(NF4LS_SHAPE, "attention: head_dim must be 64 or 128");
  if (nq % nkv) return fail(NF4LS_SHAPE, "attention: n_q %% n_kv");
  if (ldq % 8 || ldkv % 8) return fail(NF4LS_ALIGN, "attention: leading dimensions must be multiples of 8");
  return NF4LS_OK;
}

}  // namespace

int attention_fwd(const __nv_bfloat16* q, const __nv_bfloat16* k, const __nv_bfloat16* v, int ldq, int ldkv,
                  __nv_bfloat16* o, int ldo, float* lse, int batch, int seq, int nq, int nkv, int d, cudaStream_t s) {
  NF4_TRY(check_attn(seq, nq, nkv, d, ldq, ldkv));
  if (attention_tc() && attention_fwd_tc_supported(seq, d, nq, nkv, ldq, ldkv, ldo))
    return attention_fwd_tc(q, k, v, ldq, ldkv, o, ldo, lse, batch, seq, nq, nkv, d, s);
  const float scale_log2 = (1.0f / sqrtf((float)d)) * kLog2e;
  dim3 grid(seq / TQ, nq, batch);
  if (d == 128) {
    const int sm = 5 * Tile<128>::BYTES;
    NF4_TRY(set_smem(k_attn_fwd<128>, sm));
    k_attn_fwd<128><<<grid, 128, sm, s>>>(q, k, v, ldq, ldkv, o, ldo, lse, seq, nq, nkv, scale_log2);
    note_launch();
  } else {
    const int sm = 5 * Tile<64>::BYTES;
    NF4_TRY(set_smem(k_attn_fwd<64>, sm));
    k_attn_fwd<64><<<grid, 128, sm, s>>>(q, k, v, ldq, ldkv, o, ldo, lse, seq, nq, nkv, scale_log2);
    note_launch();
  }
  NF4_CUDA_TRY(cudaGetLastError());
  return NF4LS_OK;
}

int attention_bwd(const __nv_bfloat16* q, const __nv_bfloat16* k, const __nv_bfloat16* v, int ldq, int ldkv,
                  const __nv_bfloat16* o, const __nv_bfloat16* dout, int ldo, const float* lse, float* delta,
                  __nv_bfloat16* dq, __nv_bfloat16* dk, __nv_bfloat16* dv, int ld_dq, int ld_dkv, int batch, int seq,
                  int nq, int nkv, int d, cudaStream_t s) {
  NF4_TRY(check_attn(seq, nq, nkv, d, ldq, ldkv));
  const int M = batch * seq;
  const float scale = 1.0f / sqrtf((float)d);
  if (attention_tc() && attention_bwd_tc_supported(seq, d, nq, nkv, ldq, ldkv, ldo, ld_dq, ld_dkv))
    // the tcgen05 query-side kernel forms delta itself
    return attention_bwd_tc(q, k, v, ldq, ldkv, o, dout, ldo, lse, delta, dq, dk, dv, ld_dq, ld_dkv, batch, seq, nq,
                            nkv, d, s);
  k_attn_delta<<<(M * nq + 7) / 8, 256, 0, s>>>(o, dout, ldo, M, seq, nq, d, delta);
  note_launch();
  dim3 gq(seq / TQ, nq, batch), gk(nkv, batch, seq / TK);
  if (d == 128) {
    const int sq = 6 * Tile<128>::BYTES, sk = 10 * Tile<128>::BYTES + 2048;
    NF4_TRY(set_smem(k_attn_dq<128>, sq));
    NF4_TRY(set_smem(k_attn_dkv<128>, sk));
    k_attn_dq<128><<<gq, 128, sq, s>>>(q, k, v, ldq, ldkv, dout, ldo, lse, delta, dq, ld_dq, seq, nq, nkv, scale);
    note_launch();
    k_attn_dkv<128><<<gk, 256, sk, s>>>(q, k, v, ldq, ldkv, dout, ldo, lse, delta, dk, dv, ld_dkv, seq, nq, nkv, scale);
    note_launch();
  } else {
    const int sq = 6 * Tile<64>::BYTES, sk = 10 * Tile<64>::BYTES + 2048;
    NF4_TRY(set_smem(k_attn_dq<64>, sq));
    NF4_TRY(set_smem(k_attn_dkv<64>, sk));
    k_attn_dq<64><<<gq, 128, sq, s>>>(q, k, v, ldq, ldkv, dout, ldo, lse, delta, dq, ld_dq, seq, nq, nkv, scale);
    note_launch();
    k_attn_dkv<64><<<gk, 256, sk, s>>>(q, k, v, ldq, ldkv, dout, ldo, lse, delta, dk, dv, ld_dkv, seq, nq, nkv, scale);
    note_launch();
  }
  NF4_CUDA_TRY(cudaGetLastError());
  return NF4LS_OK;
}

}  // namespace nf4ls

extern "C" int nf4ls_attention_fwd(const nf4ls_layer_cfg* cfg, const void* q_dev, const void* k_dev, const void* v_dev,
                                   int ld_q, int ld_kv, void* o_dev, float* lse_dev, nf4ls_stream stream) {
  nf4ls::clear_error();
  if (!cfg || !q_dev || !k_dev || !v_dev || !o_dev || !lse_dev) return nf4ls::fail(NF4LS_INVALID_ARG, "null argument");
  return nf4ls::attention_fwd(static_cast<const __nv_bfloat16*>(q_dev), static_cast<const __nv_bfloat16*>(k_dev),
                              static_cast<const __nv_bfloat16*>(v_dev), ld_q, ld_kv, static_cast<__nv_bfloat16*>(o_dev),
                              cfg->n_q * cfg->head_dim, lse_dev, cfg->batch, cfg->seq, cfg->n_q, cfg->n_kv,
                              cfg->head_dim, static_cast<cudaStream_t>(stream));
}

extern "C" int nf4ls_attention_bwd(const nf4ls_layer_cfg* cfg, const void* q_dev, const void* k_dev, const void* v_dev,
                                   int ld_q, int ld_kv, const void* o_dev, const void* do_dev, const float* lse_dev,
                                   float* delta_dev, void* dq_dev, void* dk_dev, void* dv_dev, nf4ls_stream stream) {
  nf4ls::clear_error();
  if (!cfg || !q_dev || !k_dev || !v_dev || !o_dev || !do_dev || !lse_dev || !delta_dev || !dq_dev || !dk_dev ||
      !dv_dev)
    return nf4ls::fail(NF4LS_INVALID_ARG, "null argument");
  const int qd = cfg->n_q * cfg->head_dim, kvd = cfg->n_kv * cfg->head_dim;
  return nf4ls::attention_bwd(static_cast<const __nv_bfloat16*>(q_dev), static_cast<const __nv_bfloat16*>(k_dev),
                              static_cast<const __nv_bfloat16*>(v_dev), ld_q, ld_kv,
                              static_cast<const __nv_bfloat16*>(o_dev), static_cast<const __nv_bfloat16*>(do_dev), qd,
                              lse_dev, delta_dev, static_cast<__nv_bfloat16*>(dq_dev),
                              static_cast<__nv_bfloat16*>(dk_dev), static_cast<__nv_bfloat16*>(dv_dev), qd, kvd,
                              cfg->batch, cfg->seq, cfg->n_q, cfg->n_kv, cfg->head_dim,
                              static_cast<cudaStream_t>(stream));
}
