// K6/K7: the LoRA products of the q_proj and v_proj adapters (r = 16).
//
// "Soup v0.72.4 技术解析" §4.2 (LoRA r=16, alpha=32 on q_proj and v_proj) and
// "Soup 层流式 NF4 训练实测：在 4 GB 显存上以位级一致标准完成 8B 模型 LoRA 微调"
// §2.2 check 2 (LoRA gradients nonzero in every layer): the adapter adds
// s (x A^T) B^T to the q and v projections (s = alpha / r) and trains A and B.  The
// up-projection is folded into the q/k/v GEMM as an extra 64-wide reduction block;
// this file holds the skinny products around it, all of them HBM-bound, in one launch
// per forward and three per backward:
//
//   k_lora_down: t = [h1 A_q^T | h1 A_v^T] (bf16, the extra operand of the q/k/v GEMM)
//     from h1 and the bf16 adapter rows, which the input RMSNorm's launch converts
//     from the fp32 masters together with the other adapter operands (body.cu);
//   k_lora_bwd_partial: per (128-row block, column chunk of dq or dv) the partial sums
//     of dB = s dX^T t (over the rows) and of dt = s dX B (over the columns), from one
//     read of dX;
//   k_lora_bwd_reduce: dB (partials added in row-block order) and dt (partials added
//     in column-chunk order, rounded to bf16: the extra operand of the dL/dx GEMM);
//   k_lora_bwd_da: dA = dt^T h1, one block per 32 columns of h1 over all rows.
//
// The products run on the warp-level bf16 tensor-core instruction (mma.sync m16n8k16);
// every reduction is in a fixed order, so each result is bit-reproducible and a
// token's row results (t, dt) do not depend on how many tokens share the launch.
#include <algorithm>
#include <mutex>
#include <utility>
#include <vector>

#include "common.cuh"
#include "internal.h"

namespace nf4ls {

namespace {

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

__device__ __forceinline__ void unpack8(const uint4& u, float (&f)[8]) {
  const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    f[2 * j] = bf16_lo(w[j]);
    f[2 * j + 1] = bf16_hi(w[j]);
  }
}
__device__ __forceinline__ uint4 pack8(const float (&f)[8]) {
  return make_uint4(pack_bf16x2(f[0], f[1]), pack_bf16x2(f[2], f[3]), pack_bf16x2(f[4], f[5]),
                    pack_bf16x2(f[6], f[7]));
}

__device__ __forceinline__ void zero16(uint32_t addr) { st_shared_v4(addr, 0u, 0u, 0u, 0u); }

// ============================================================================ forward
constexpr int LD_ROWS = 16, LD_THREADS = 256, LD_WARPS = 8, LD_KC = 128;  // rows per block, k-chunk
constexpr int LD_LS = LD_KC + 8;                                         // smem row stride (elements)
constexpr int LD_STAGES = 4;
constexpr int LD_STAGE_BYTES = (LD_ROWS + 32) * LD_LS * 2;
constexpr int LD_SMEM = LD_STAGES * LD_STAGE_BYTES;

// One block: 16 token rows.  The reduction over H runs in chunks of 128 columns through a
// ring of LD_STAGES shared-memory stages filled by cp.async: the h1 rows and the 32 bf16
// adapter rows (A_q, A_v of adn).  Warp w takes the chunk's k-step w, so it accumulates
// the global k-steps w, w + 8, ...; the eight partial products are then added in warp
// order.
__global__ void __launch_bounds__(LD_THREADS) k_lora_down(const __nv_bfloat16* __restrict__ h1, int M, int H,
                                                          const __nv_bfloat16* __restrict__ adn,
                                                          __nv_bfloat16* __restrict__ tpad) {
  extern __shared__ __align__(16) uint8_t smem[];
  const int t = threadIdx.x, warp = t >> 5, lane = t & 31, g4 = lane >> 2, t4 = lane & 3;
  const int m0 = blockIdx.x * LD_ROWS;
  const int n_chunks = (H + LD_KC - 1) / LD_KC;
  auto tile = [&](int b) { return reinterpret_cast<__nv_bfloat16*>(smem + (size_t)b * LD_STAGE_BYTES); };
  // chunk c into stage b: rows 0-15 h1, rows 16-47 adapter rows 0-31 (16 pieces each)
  auto stage = [&](int c, int b) {
    for (int e = t; e < (LD_ROWS + 32) * 16; e += LD_THREADS) {
      const int r = e >> 4, q = e & 15, col = c * LD_KC + q * 8;
      const uint32_t dst = smem_u32(tile(b) + r * LD_LS + q * 8);
      const int m = m0 + r;
      if (col >= H || (r < LD_ROWS && m >= M))
        zero16(dst);
      else if (r < LD_ROWS)
        cp_async16(dst, h1 + (size_t)m * H + col);
      else
        cp_async16(dst, adn + (size_t)(r - LD_ROWS) * H + col);
    }
    asm volatile("cp.async.commit_group;" ::: "memory");
  };
  float acc[4][4];
#pragma unroll
  for (int i = 0; i < 4; ++i) acc[i][0] = acc[i][1] = acc[i][2] = acc[i][3] = 0.f;
  for (int c = 0; c < LD_STAGES - 1; ++c) {
    if (c < n_chunks)
      stage(c, c);
    else
      asm volatile("cp.async.commit_group;" ::: "memory");
  }
  for (int c = 0; c < n_chunks; ++c) {
    const int b = c % LD_STAGES;
    asm volatile("cp.async.wait_group %0;" ::"n"(LD_STAGES - 2) : "memory");
    __syncthreads();  // chunk c has landed for every thread; the stage of chunk c - 1 is free
    if (c + LD_STAGES - 1 < n_chunks)
      stage(c + LD_STAGES - 1, (c + LD_STAGES - 1) % LD_STAGES);
    else
      asm volatile("cp.async.commit_group;" ::: "memory");
    if (c * LD_KC + warp * 16 < H) {
      const __nv_bfloat16* T = tile(b);
      uint32_t a0, a1, a2, a3, b0, b1, b2, b3, b4, b5, b6, b7;
      ldsm4(smem_u32(T + (lane & 15) * LD_LS + warp * 16 + (lane >> 4) * 8), a0, a1, a2, a3);
      const int br = (lane & 7) + (lane >> 4) * 8, bc = warp * 16 + ((lane >> 3) & 1) * 8;
      ldsm4(smem_u32(T + (LD_ROWS + br) * LD_LS + bc), b0, b1, b2, b3);
      ldsm4(smem_u32(T + (LD_ROWS + 16 + br) * LD_LS + bc), b4, b5, b6, b7);
      mma16816(acc[0], a0, a1, a2, a3, b0, b1);
      mma16816(acc[1], a0, a1, a2, a3, b2, b3);
      mma16816(acc[2], a0, a1, a2, a3, b4, b5);
      mma16816(acc[3], a0, a1, a2, a3, b6, b7);
    }
  }
  asm volatile("cp.async.wait_all;" ::: "memory");
  __syncthreads();
  float* red = reinterpret_cast<float*>(smem);  // the stages are free now
  float* R = red + warp * (LD_ROWS * 32);
#pragma unroll
  for (int nt = 0; nt < 4; ++nt) {
    R[g4 * 32 + nt * 8 + 2 * t4] = acc[nt][0];
    R[g4 * 32 + nt * 8 + 2 * t4 + 1] = acc[nt][1];
    R[(g4 + 8) * 32 + nt * 8 + 2 * t4] = acc[nt][2];
    R[(g4 + 8) * 32 + nt * 8 + 2 * t4 + 1] = acc[nt][3];
  }
  __syncthreads();
  for (int e = t; e < LD_ROWS * 64; e += LD_THREADS) {
    const int r = e >> 6, cc = e & 63, m = m0 + r;
    if (m >= M) continue;
    float v = 0.f;
    if (cc < 32)
      for (int w = 0; w < LD_WARPS; ++w) v += red[w * (LD_ROWS * 32) + r * 32 + cc];
    tpad[(size_t)m * 64 + cc] = __float2bfloat16_rn(v);
  }
}

// ============================================================================ backward
constexpr int LB_ROWS = 128, LB_THREADS = 256;

struct LoraBwdArgs {
  const __nv_bfloat16* dqkv;  // [M, ld]: dq from column 0, dv from column vcol
  int ld, vcol, qd, kvd, M, H;
  int CW, n_cc_q, n_cc;       // column chunks of CW: the first n_cc_q over dq, the rest over dv
  const __nv_bfloat16* tpad;  // [M, 64]: t_q in columns 0-15, t_v in 16-31
  const __nv_bfloat16* bqt;   // [16, qd] = B_q^T (bf16)
  const __nv_bfloat16* bvt;   // [16, kvd] = B_v^T
  float* part_dB;             // [n_rb][qd + kvd][16]
  float* part_dt;             // [n_cc][M][16]
  int n_rb, n_db_blocks;
  const __nv_bfloat16* h1;    // [M, H]
  __nv_bfloat16* dtpad;       // [M, 64]: dt_q in 0-15, dt_v in 16-31, zeros in 32-63
  float scale;
  float* dA_q;                // [16, H]
  float* dB_q;                // [qd, 16]
  float* dA_v;
  float* dB_v;                // [kvd, 16]
};

// Block (row block rb, column chunk cc): X = rows [128 rb, +128) x CW columns of dq or dv.
//   partial dB[cols, 16] = X^T t_seg  (over the block's rows)
//   partial dt[rows, 16] = X B_seg    (over the chunk's columns)
__global__ void __launch_bounds__(LB_THREADS) k_lora_bwd_partial(const __grid_constant__ LoraBwdArgs a) {
  extern __shared__ __align__(16) uint8_t smem[];
  const int CW = a.CW, lx = CW + 8;
  __nv_bfloat16* xs = reinterpret_cast<__nv_bfloat16*>(smem);        // [128][CW + 8]
  __nv_bfloat16* ts = xs + LB_ROWS * lx;                             // [128][24]
  __nv_bfloat16* bs = ts + LB_ROWS * 24;                             // [16][CW + 8]
  const int rb = blockIdx.x, cc = blockIdx.y;
  const int t = threadIdx.x, warp = t >> 5, lane = t & 31, g4 = lane >> 2, t4 = lane & 3;
  const bool is_v = cc >= a.n_cc_q;
  const int c0 = cc * CW;                                   // column in [dq | dv]
  const int seg_col = is_v ? c0 - a.qd : c0;                // column within dq or dv
  const int xcol = is_v ? a.vcol + seg_col : seg_col;       // column in dqkv
  const __nv_bfloat16* bt = is_v ? a.bvt : a.bqt;
  const int bt_ld = is_v ? a.kvd : a.qd;
  const int m0 = rb * LB_ROWS;
  const uint32_t sx = smem_u32(xs), sts = smem_u32(ts), sb = smem_u32(bs);
  const int cpr = CW / 8;  // 16-byte chunks per row
  for (int i = t; i < LB_ROWS * cpr; i += LB_THREADS) {
    const int r = i / cpr, c = i % cpr, m = m0 + r;
    const uint32_t dst = sx + (r * lx + c * 8) * 2;
    if (m < a.M)
      cp_async16(dst, a.dqkv + (size_t)m * a.ld + xcol + c * 8);
    else
      zero16(dst);
  }
  {
    const int r = t >> 1, c = t & 1, m = m0 + r;  // 128 rows x 2 chunks of t_seg
    const uint32_t dst = sts + (r * 24 + c * 8) * 2;
    if (m < a.M)
      cp_async16(dst, a.tpad + (size_t)m * 64 + (is_v ? 16 : 0) + c * 8);
    else
      zero16(dst);
  }
  for (int i = t; i < 16 * cpr; i += LB_THREADS) {
    const int r = i / cpr, c = i % cpr;
    cp_async16(sb + (r * lx + c * 8) * 2, bt + (size_t)r * bt_ld + seg_col + c * 8);
  }
  cp_async_wait_all();
  __syncthreads();

  // partial dB: D[CW x 16] = X^T T, m16 tiles over the columns, k over the 128 rows
  for (int mt = warp; mt < CW / 16; mt += 8) {
    float acc[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
#pragma unroll
    for (int kk = 0; kk < LB_ROWS / 16; ++kk) {
      uint32_t a0, a1, a2, a3, b0, b1, b2, b3;
      {
        const int m = kk * 16 + (lane & 7) + (lane >> 4) * 8, n = mt * 16 + ((lane >> 3) & 1) * 8;
        ldsm4t(sx + (m * lx + n) * 2, a0, a1, a2, a3);
      }
      {
        const int m = kk * 16 + (lane & 7) + ((lane >> 3) & 1) * 8, n = (lane >> 4) * 8;
        ldsm4t(sts + (m * 24 + n) * 2, b0, b1, b2, b3);
      }
      mma16816(acc[0], a0, a1, a2, a3, b0, b1);
      mma16816(acc[1], a0, a1, a2, a3, b2, b3);
    }
    float* P = a.part_dB + ((size_t)rb * (a.qd + a.kvd) + c0 + mt * 16) * 16;
#pragma unroll
    for (int nt = 0; nt < 2; ++nt) {
      P[g4 * 16 + nt * 8 + 2 * t4] = acc[nt][0];
      P[g4 * 16 + nt * 8 + 2 * t4 + 1] = acc[nt][1];
      P[(g4 + 8) * 16 + nt * 8 + 2 * t4] = acc[nt][2];
      P[(g4 + 8) * 16 + nt * 8 + 2 * t4 + 1] = acc[nt][3];
    }
  }

  // partial dt: D[128 x 16] = X B, warp w takes rows 16 w .. 16 w + 15, k over the CW columns
  {
    float acc[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
    for (int kk = 0; kk < CW / 16; ++kk) {
      uint32_t a0, a1, a2, a3, b0, b1, b2, b3;
      {
        const int r = warp * 16 + (lane & 7) + ((lane >> 3) & 1) * 8, c = kk * 16 + (lane >> 4) * 8;
        ldsm4(sx + (r * lx + c) * 2, a0, a1, a2, a3);
      }
      {
        const int r = (lane & 7) + (lane >> 4) * 8, c = kk * 16 + ((lane >> 3) & 1) * 8;
        ldsm4(sb + (r * lx + c) * 2, b0, b1, b2, b3);
      }
      mma16816(acc[0], a0, a1, a2, a3, b0, b1);
      mma16816(acc[1], a0, a1, a2, a3, b2, b3);
    }
    float* P = a.part_dt + (size_t)cc * a.M * 16;
    const int m = m0 + warp * 16 + g4;
#pragma unroll
    for (int nt = 0; nt < 2; ++nt) {
      if (m < a.M) {
        P[(size_t)m * 16 + nt * 8 + 2 * t4] = acc[nt][0];
        P[(size_t)m * 16 + nt * 8 + 2 * t4 + 1] = acc[nt][1];
      }
      if (m + 8 < a.M) {
        P[(size_t)(m + 8) * 16 + nt * 8 + 2 * t4] = acc[nt][2];
        P[(size_t)(m + 8) * 16 + nt * 8 + 2 * t4 + 1] = acc[nt][3];
      }
    }
  }
}

// Blocks [0, n_db_blocks): dB, one element per thread, the row-block partials added in
// order.  The others: dt of 8 rows per block (one row per warp, column-chunk partials
// added in order, times s, rounded to bf16) into dtpad, zeros in its columns 32-63.
__global__ void __launch_bounds__(LB_THREADS) k_lora_bwd_reduce(const __grid_constant__ LoraBwdArgs a) {
  const int t = threadIdx.x;
  const int NB = a.qd + a.kvd;
  if ((int)blockIdx.x < a.n_db_blocks) {
    const int e = blockIdx.x * LB_THREADS + t;
    if (e >= NB * 16) return;
    const int col = e >> 4, r = e & 15;
    float v = 0.f;
    for (int rb = 0; rb < a.n_rb; ++rb) v += a.part_dB[((size_t)rb * NB + col) * 16 + r];
    v *= a.scale;
    if (col < a.qd)
      a.dB_q[(size_t)col * 16 + r] = v;
    else
      a.dB_v[(size_t)(col - a.qd) * 16 + r] = v;
    return;
  }
  const int m = ((int)blockIdx.x - a.n_db_blocks) * 8 + (t >> 5), c = t & 31;
  if (m >= a.M) return;
  const int cb = c < 16 ? 0 : a.n_cc_q, ce = c < 16 ? a.n_cc_q : a.n_cc;
  float v = 0.f;
  for (int k = cb; k < ce; ++k) v += a.part_dt[((size_t)k * a.M + m) * 16 + (c & 15)];
  a.dtpad[(size_t)m * 64 + c] = __float2bfloat16_rn(v * a.scale);
  a.dtpad[(size_t)m * 64 + 32 + c] = __float2bfloat16_rn(0.f);
}

// dA = dt^T h1: one block per 64 columns of h1, over all M rows in chunks of 128 through
// a ring of DA_STAGES cp.async stages.  Warp w takes the chunk's k-step w (16 rows), so it
// accumulates the rows 16 w .. of every chunk; the eight partial products are added in
// warp order.
constexpr int DA_COLS = 64, DA_ROWS = 128, DA_DS = 40, DA_HS = DA_COLS + 8, DA_STAGES = 4;
constexpr int DA_PIECES = 4 + DA_COLS / 8;  // 16-byte pieces per row: dt (32 columns), h1
constexpr int DA_STAGE_BYTES = DA_ROWS * (DA_DS + DA_HS) * 2;
constexpr int DA_SMEM = DA_STAGES * DA_STAGE_BYTES;

__global__ void __launch_bounds__(LB_THREADS) k_lora_bwd_da(const __grid_constant__ LoraBwdArgs a) {
  extern __shared__ __align__(16) uint8_t smem[];
  const int t = threadIdx.x, warp = t >> 5, lane = t & 31, g4 = lane >> 2, t4 = lane & 3;
  const int c0 = blockIdx.x * DA_COLS;
  const int n_chunks = (a.M + DA_ROWS - 1) / DA_ROWS;
  auto ds = [&](int b) { return reinterpret_cast<__nv_bfloat16*>(smem + (size_t)b * DA_STAGE_BYTES); };
  auto hs = [&](int b) {
    return reinterpret_cast<__nv_bfloat16*>(smem + (size_t)b * DA_STAGE_BYTES + DA_ROWS * DA_DS * 2);
  };
  auto stage = [&](int ch, int b) {  // 128 rows x (4 pieces of dt + DA_COLS / 8 pieces of h1)
    for (int i = t; i < DA_ROWS * DA_PIECES; i += LB_THREADS) {
      const int r = i / DA_PIECES, q = i % DA_PIECES, m = ch * DA_ROWS + r;
      const uint32_t dst = q < 4 ? smem_u32(ds(b) + r * DA_DS + q * 8) : smem_u32(hs(b) + r * DA_HS + (q - 4) * 8);
      if (m >= a.M)
        zero16(dst);
      else if (q < 4)
        cp_async16(dst, a.dtpad + (size_t)m * 64 + q * 8);
      else
        cp_async16(dst, a.h1 + (size_t)m * a.H + c0 + (q - 4) * 8);
    }
    asm volatile("cp.async.commit_group;" ::: "memory");
  };
  constexpr int NT = DA_COLS / 8;  // n8 tiles of the block's columns
  float acc[2][NT][4];
#pragma unroll
  for (int i = 0; i < 2; ++i)
#pragma unroll
    for (int j = 0; j < NT; ++j) acc[i][j][0] = acc[i][j][1] = acc[i][j][2] = acc[i][j][3] = 0.f;
  for (int ch = 0; ch < DA_STAGES - 1; ++ch) {
    if (ch < n_chunks)
      stage(ch, ch);
    else
      asm volatile("cp.async.commit_group;" ::: "memory");
  }
  for (int ch = 0; ch < n_chunks; ++ch) {
    const int b = ch % DA_STAGES;
    asm volatile("cp.async.wait_group %0;" ::"n"(DA_STAGES - 2) : "memory");
    __syncthreads();  // chunk ch has landed; the stage of chunk ch - 1 is free
    if (ch + DA_STAGES - 1 < n_chunks)
      stage(ch + DA_STAGES - 1, (ch + DA_STAGES - 1) % DA_STAGES);
    else
      asm volatile("cp.async.commit_group;" ::: "memory");
    const int kr = warp * 16;  // this warp's 16 rows of the chunk
    uint32_t af[2][4];
#pragma unroll
    for (int mt = 0; mt < 2; ++mt) {  // dA rows 16 mt ..: A = dt^T from the dt rows
      const int m = kr + (lane & 7) + (lane >> 4) * 8, n = mt * 16 + ((lane >> 3) & 1) * 8;
      ldsm4t(smem_u32(ds(b) + m * DA_DS + n), af[mt][0], af[mt][1], af[mt][2], af[mt][3]);
    }
#pragma unroll
    for (int h = 0; h < NT / 2; ++h) {  // h1 columns 16 h ..: B fragments of two n8 tiles
      uint32_t b0, b1, b2, b3;
      const int m = kr + (lane & 7) + ((lane >> 3) & 1) * 8, n = h * 16 + (lane >> 4) * 8;
      ldsm4t(smem_u32(hs(b) + m * DA_HS + n), b0, b1, b2, b3);
#pragma unroll
      for (int mt = 0; mt < 2; ++mt) {
        mma16816(acc[mt][2 * h], af[mt][0], af[mt][1], af[mt][2], af[mt][3], b0, b1);
        mma16816(acc[mt][2 * h + 1], af[mt][0], af[mt][1], af[mt][2], af[mt][3], b2, b3);
      }
    }
  }
  asm volatile("cp.async.wait_all;" ::: "memory");
  __syncthreads();
  float* red = reinterpret_cast<float*>(smem);  // the stages are free now
  float* R = red + warp * (32 * DA_COLS);
#pragma unroll
  for (int mt = 0; mt < 2; ++mt)
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
      const int row = mt * 16 + g4, col = nt * 8 + 2 * t4;
      R[row * DA_COLS + col] = acc[mt][nt][0];
      R[row * DA_COLS + col + 1] = acc[mt][nt][1];
      R[(row + 8) * DA_COLS + col] = acc[mt][nt][2];
      R[(row + 8) * DA_COLS + col + 1] = acc[mt][nt][3];
    }
  __syncthreads();
  for (int e = t; e < 32 * DA_COLS; e += LB_THREADS) {
    const int row = e / DA_COLS, col = c0 + e % DA_COLS;
    float v = 0.f;
    for (int w = 0; w < 8; ++w) v += red[w * (32 * DA_COLS) + e];
    if (row < 16)
      a.dA_q[(size_t)row * a.H + col] = v;
    else
      a.dA_v[(size_t)(row - 16) * a.H + col] = v;
  }
}

// Column chunk of k_lora_bwd_partial: 128 where it divides both widths (so that a
// 2048-token batch of the 8B layer runs 16 x 40 blocks, several per SM), else 64.
int chunk_width(int a, int b) {
  for (int w : {128, 64})
    if (a % w == 0 && b % w == 0) return w;
  return 0;
}

struct BwdShape {
  int CW, n_cc_q, n_cc, n_rb, n_db_blocks;
  size_t part_dB, part_dt, total;
};

BwdShape bwd_shape(int M, int H, int qd, int kvd) {
  BwdShape b;
  b.CW = chunk_width(qd, kvd);
  b.n_cc_q = b.CW ? qd / b.CW : 0;
  b.n_cc = b.CW ? (qd + kvd) / b.CW : 0;
  b.n_rb = (M + LB_ROWS - 1) / LB_ROWS;
  b.n_db_blocks = ((qd + kvd) * 16 + LB_THREADS - 1) / LB_THREADS;
  size_t off = 0;
  auto take = [&](size_t bytes) {
    const size_t o = off;
    off = round_up(off + bytes, 256);
    return o;
  };
  b.part_dB = take((size_t)b.n_rb * (qd + kvd) * 16 * 4);
  b.part_dt = take((size_t)b.n_cc * M * 16 * 4);
  b.total = off;
  return b;
}

// Raises a kernel's dynamic shared-memory limit once per device (to the largest size
// asked for so far).
int allow_smem(const void* kernel, size_t bytes) {
  if (bytes <= 48 * 1024) return NF4LS_OK;
  static std::mutex mu;
  static std::vector<std::pair<std::pair<const void*, int>, size_t>> done;
  int dev = 0;
  NF4_CUDA_TRY(cudaGetDevice(&dev));
  std::lock_guard<std::mutex> g(mu);
  for (auto& d : done)
    if (d.first.first == kernel && d.first.second == dev) {
      if (d.second >= bytes) return NF4LS_OK;
      NF4_CUDA_TRY(cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes));
      d.second = bytes;
      return NF4LS_OK;
    }
  NF4_CUDA_TRY(cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes));
  done.push_back({{kernel, dev}, bytes});
  return NF4LS_OK;
}

}  // namespace

size_t lora_partial_bytes(int M, int H, int qd, int kvd) { return bwd_shape(M, H, qd, kvd).total; }

int lora_down(const __nv_bfloat16* h1, int M, int H, const __nv_bfloat16* adn, __nv_bfloat16* tpad, cudaStream_t s) {
  if (H % 16) return fail(NF4LS_SHAPE, "lora_down: H %d", H);
  if (M <= 0) return NF4LS_OK;
  static_assert(LD_WARPS * LD_ROWS * 32 * 4 <= LD_SMEM, "partials fit in the stages");
  NF4_TRY(allow_smem((const void*)k_lora_down, LD_SMEM));
  k_lora_down<<<(M + LD_ROWS - 1) / LD_ROWS, LD_THREADS, LD_SMEM, s>>>(h1, M, H, adn, tpad);
  note_launch();
  NF4_CUDA_TRY(cudaGetLastError());
  return NF4LS_OK;
}

int lora_bwd(const __nv_bfloat16* dqkv, int ld, int vcol, int M, int H, int qd, int kvd, const __nv_bfloat16* tpad,
             const __nv_bfloat16* bqt, const __nv_bfloat16* bvt, const __nv_bfloat16* h1, float scale,
             __nv_bfloat16* dtpad, const nf4ls_lora_grads* g, void* part, cudaStream_t s) {
  const BwdShape sh = bwd_shape(M, H, qd, kvd);
  if (!sh.CW || H % DA_COLS || ld % 8 || vcol % 8)
    return fail(NF4LS_SHAPE, "lora_bwd: qd %d, kvd %d, H %d", qd, kvd, H);
  if (M <= 0) return NF4LS_OK;
  LoraBwdArgs a;
  a.dqkv = dqkv;
  a.ld = ld;
  a.vcol = vcol;
  a.qd = qd;
  a.kvd = kvd;
  a.M = M;
  a.H = H;
  a.CW = sh.CW;
  a.n_cc_q = sh.n_cc_q;
  a.n_cc = sh.n_cc;
  a.tpad = tpad;
  a.bqt = bqt;
  a.bvt = bvt;
  uint8_t* pb = static_cast<uint8_t*>(part);
  a.part_dB = reinterpret_cast<float*>(pb + sh.part_dB);
  a.part_dt = reinterpret_cast<float*>(pb + sh.part_dt);
  a.n_rb = sh.n_rb;
  a.n_db_blocks = sh.n_db_blocks;
  a.h1 = h1;
  a.dtpad = dtpad;
  a.scale = scale;
  a.dA_q = g->dA_q;
  a.dB_q = g->dB_q;
  a.dA_v = g->dA_v;
  a.dB_v = g->dB_v;
  const size_t smem1 = (size_t)LB_ROWS * (sh.CW + 8) * 2 + (size_t)LB_ROWS * 24 * 2 + 16ull * (sh.CW + 8) * 2;
  NF4_TRY(allow_smem((const void*)k_lora_bwd_partial, smem1));
  k_lora_bwd_partial<<<dim3(sh.n_rb, sh.n_cc), LB_THREADS, smem1, s>>>(a);
  note_launch();
  k_lora_bwd_reduce<<<sh.n_db_blocks + (M + 7) / 8, LB_THREADS, 0, s>>>(a);
  note_launch();
  static_assert(8 * 32 * DA_COLS * 4 <= DA_SMEM, "partials fit in the stages");
  NF4_TRY(allow_smem((const void*)k_lora_bwd_da, DA_SMEM));
  k_lora_bwd_da<<<H / DA_COLS, LB_THREADS, DA_SMEM, s>>>(a);
  note_launch();
  NF4_CUDA_TRY(cudaGetLastError());
  return NF4LS_OK;
}

}  // namespace nf4ls
