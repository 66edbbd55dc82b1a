// K6/K7: the LoRA products of the q_proj and v_proj adapters (r = 16).
//
// "Soup v0.72.4 技术解析" §4.2 (LoRA r=16, alpha=32 on q_proj and v_proj) and
// "Soup 层流式 NF4 训练实测：在 4 GB 显存上以位级一致标准完成 8B 模型 LoRA 微调"
// §2.2 check 2 (LoRA gradients nonzero in every layer): the adapter adds
// s (x A^T) B^T to the q and v projections (s = alpha / r) and trains A and B.  The
// up-projection is folded into the q/k/v GEMM as an extra 64-wide reduction block;
// this file holds the skinny products around it, all of them HBM-bound, in three
// launches per layer and step direction:
//
//   forward (k_norm_lora_fwd, one launch):
//     h1 = rmsnorm(x) w_in and t = [h1 A_q^T | h1 A_v^T] in one pass over x, plus the
//     bf16 operands of the adapter (s B_q, s B_v for the up-projection block, A_q, A_v
//     for the dL/dx block, B_q^T, B_v^T for dt) converted from the fp32 masters;
//   backward (two launches):
//     k_lora_bwd_partial: per (128-row block, column chunk of dq or dv) the partial
//       sums of dB = s dX^T t (over the rows) and of dt = s dX B (over the columns),
//       from one read of dX;
//     k_lora_bwd_final: dB (partials added in row-block order); dt (partials added in
//       column-chunk order, rounded to bf16: the extra operand of the dL/dx GEMM); the
//       partial sums of dA = dt^T h1 per (128-row group, column chunk of h1), which the
//       last block of each column chunk to finish adds in row-group order.
//
// The products run on the warp-level bf16 tensor-core instruction (mma.sync m16n8k16);
// every reduction is in a fixed order, so each result is bit-reproducible and a
// token's row results (h1, t, dt) do not depend on how many tokens share the launch.
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
constexpr int NL_ROWS = 16, NL_THREADS = 256, NL_WARPS = 8;

struct NormLoraArgs {
  const __nv_bfloat16* x;
  const __nv_bfloat16* w;
  __nv_bfloat16* h1;
  int M, H;
  float eps;
  const float* Aq;  // [16, H] fp32 masters
  const float* Av;
  const float* Bq;  // [qd, 16]
  const float* Bv;  // [kvd, 16]
  __nv_bfloat16* tpad;  // [M, 64]: t_q in columns 0-15, t_v in 16-31, zeros in 32-63
  int qd, kvd;
  float scale;
  // bf16 adapter operands:
  //   bup [Nqkv, 64]: q rows: s B_q in columns 0-15; v rows: s B_v in columns 16-31; else 0
  //   adn [64, H]   : rows 0-15 A_q, rows 16-31 A_v, else 0
  //   bqt [16, qd] = B_q^T, bvt [16, kvd] = B_v^T
  __nv_bfloat16* bup;
  __nv_bfloat16* adn;
  __nv_bfloat16* bqt;
  __nv_bfloat16* bvt;
};

__device__ void pack_element(const NormLoraArgs& a, size_t i) {
  const int H = a.H, qd = a.qd, kvd = a.kvd, nq = qd + 2 * kvd;
  const size_t n1 = (size_t)nq * 64, n2 = (size_t)64 * H, n3 = (size_t)16 * qd;
  if (i < n1) {
    const int n = (int)(i / 64), c = (int)(i % 64);
    float v = 0.f;
    if (n < qd && c < 16)
      v = a.scale * __bfloat162float(__float2bfloat16_rn(a.Bq[(size_t)n * 16 + c]));
    else if (n >= qd + kvd && c >= 16 && c < 32)
      v = a.scale * __bfloat162float(__float2bfloat16_rn(a.Bv[(size_t)(n - qd - kvd) * 16 + c - 16]));
    a.bup[i] = __float2bfloat16_rn(v);
    return;
  }
  i -= n1;
  if (i < n2) {
    const int r = (int)(i / H), k = (int)(i % H);
    float v = 0.f;
    if (r < 16)
      v = a.Aq[(size_t)r * H + k];
    else if (r < 32)
      v = a.Av[(size_t)(r - 16) * H + k];
    a.adn[i] = __float2bfloat16_rn(v);
    return;
  }
  i -= n2;
  if (i < n3) {
    const int r = (int)(i / qd), n = (int)(i % qd);
    a.bqt[i] = __float2bfloat16_rn(a.Bq[(size_t)n * 16 + r]);
    return;
  }
  i -= n3;
  const int r = (int)(i / kvd), n = (int)(i % kvd);
  a.bvt[i] = __float2bfloat16_rn(a.Bv[(size_t)n * 16 + r]);
}

// One block: 16 token rows.  Warp w normalises rows 2w and 2w + 1 (the row held in
// registers, MAXV 16-byte vectors per lane at most), writes h1 and keeps the bf16 row in
// shared memory; then each warp multiplies the 16 rows by the 32 adapter rows over the
// 16-wide k-steps w, w + 8, ... (A fragments by ldmatrix, B fragments converted from the
// fp32 masters), and the eight partial products are added in warp order.  The block's
// share of the operand conversion follows.
template <int MAXV>
__global__ void __launch_bounds__(NL_THREADS) k_norm_lora_fwd(const __grid_constant__ NormLoraArgs a) {
  extern __shared__ __align__(16) uint8_t smem[];
  const int H = a.H, ld = H + 8, nv = H / 8;
  __nv_bfloat16* tile = reinterpret_cast<__nv_bfloat16*>(smem);
  float* red = reinterpret_cast<float*>(smem + (size_t)NL_ROWS * ld * 2);  // [8][16][32]
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int m0 = blockIdx.x * NL_ROWS;

  for (int rr = 0; rr < 2; ++rr) {
    const int r = warp * 2 + rr, m = m0 + r;
    uint4* trow = reinterpret_cast<uint4*>(tile + (size_t)r * ld);
    if (m >= a.M) {
      for (int i = lane; i < nv; i += 32) trow[i] = make_uint4(0u, 0u, 0u, 0u);
      continue;
    }
    const uint4* xr = reinterpret_cast<const uint4*>(a.x + (size_t)m * H);
    uint4 v[MAXV];
#pragma unroll
    for (int j = 0; j < MAXV; ++j)
      if (lane + 32 * j < nv) v[j] = xr[lane + 32 * j];
    float ss = 0.f;
#pragma unroll
    for (int j = 0; j < MAXV; ++j)
      if (lane + 32 * j < nv) {
        float f[8];
        unpack8(v[j], f);
#pragma unroll
        for (int e = 0; e < 8; ++e) ss += f[e] * f[e];
      }
    ss = warp_sum(ss);
    const float rs = 1.0f / sqrtf(ss / (float)H + a.eps);
    const uint4* wr = reinterpret_cast<const uint4*>(a.w);
    uint4* yr = reinterpret_cast<uint4*>(a.h1 + (size_t)m * H);
#pragma unroll
    for (int j = 0; j < MAXV; ++j) {
      const int i = lane + 32 * j;
      if (i < nv) {
        float f[8], g[8];
        unpack8(v[j], f);
        unpack8(wr[i], g);
#pragma unroll
        for (int e = 0; e < 8; ++e) f[e] = f[e] * rs * g[e];
        const uint4 o = pack8(f);
        yr[i] = o;
        trow[i] = o;
      }
    }
  }
  __syncthreads();

  // t = h1 [A_q; A_v]^T: 16 rows x 32 outputs
  float acc[4][4];
#pragma unroll
  for (int i = 0; i < 4; ++i) acc[i][0] = acc[i][1] = acc[i][2] = acc[i][3] = 0.f;
  const uint32_t st = smem_u32(tile);
  const int g4 = lane >> 2, t4 = lane & 3;
  for (int ks = warp; ks < H / 16; ks += NL_WARPS) {
    uint32_t a0, a1, a2, a3;
    ldsm4(st + ((lane & 15) * ld + ks * 16 + (lane >> 4) * 8) * 2, a0, a1, a2, a3);
#pragma unroll
    for (int nt = 0; nt < 4; ++nt) {
      const float* A = (nt < 2 ? a.Aq : a.Av) + (size_t)((nt & 1) * 8 + g4) * H + ks * 16 + 2 * t4;
      const float2 lo = *reinterpret_cast<const float2*>(A);
      const float2 hi = *reinterpret_cast<const float2*>(A + 8);
      mma16816(acc[nt], a0, a1, a2, a3, pack_bf16x2(lo.x, lo.y), pack_bf16x2(hi.x, hi.y));
    }
  }
  float* R = red + warp * (NL_ROWS * 32);
#pragma unroll
  for (int nt = 0; nt < 4; ++nt) {
    R[g4 * 32 + nt * 8 + 2 * t4] = acc[nt][0];
    R[g4 * 32 + nt * 8 + 2 * t4 + 1] = acc[nt][1];
    R[(g4 + 8) * 32 + nt * 8 + 2 * t4] = acc[nt][2];
    R[(g4 + 8) * 32 + nt * 8 + 2 * t4 + 1] = acc[nt][3];
  }
  __syncthreads();
  for (int e = threadIdx.x; e < NL_ROWS * 64; e += NL_THREADS) {
    const int r = e >> 6, c = e & 63, m = m0 + r;
    if (m >= a.M) continue;
    float v = 0.f;
    if (c < 32)
      for (int w = 0; w < NL_WARPS; ++w) v += red[w * (NL_ROWS * 32) + r * 32 + c];
    a.tpad[(size_t)m * 64 + c] = __float2bfloat16_rn(v);
  }

  // this block's share of the bf16 adapter operands
  const size_t total = (size_t)(a.qd + 2 * a.kvd) * 64 + (size_t)64 * H + 16ull * a.qd + 16ull * a.kvd;
  const size_t per = (total + gridDim.x - 1) / gridDim.x;
  const size_t b0 = (size_t)blockIdx.x * per, b1 = min(total, b0 + per);
  for (size_t i = b0 + threadIdx.x; i < b1; i += NL_THREADS) pack_element(a, i);
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
  int* counters;              // [n_hc]
  int n_rb, n_rg, HC, n_hc, n_db_blocks;
  const __nv_bfloat16* h1;    // [M, H]
  __nv_bfloat16* dtpad;       // [M, 64]: dt_q in 0-15, dt_v in 16-31, zeros in 32-63
  float* part_dA;             // [n_rg][32][H]
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
  if (rb == 0 && cc == 0)
    for (int i = t; i < a.n_hc; i += LB_THREADS) a.counters[i] = 0;  // for k_lora_bwd_final
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
// order.  The others, per (row group rg of 128 rows, column chunk hc of HC columns of
// h1): dt of the group's rows (column-chunk partials added in order, times s, rounded
// to bf16; the hc = 0 blocks also store it as the dL/dx GEMM's extra operand), then the
// partial dA = dt^T h1 over the group's rows; the last of the n_rg blocks of a chunk to
// finish adds the partials in row-group order.
__global__ void __launch_bounds__(LB_THREADS) k_lora_bwd_final(const __grid_constant__ LoraBwdArgs a) {
  extern __shared__ __align__(16) uint8_t smem[];
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
  const int b = blockIdx.x - a.n_db_blocks;
  const int rg = b / a.n_hc, hc = b % a.n_hc;
  const int HC = a.HC, lh = HC + 8, m0 = rg * LB_ROWS;
  __nv_bfloat16* dts = reinterpret_cast<__nv_bfloat16*>(smem);  // [128][40]
  __nv_bfloat16* hs = dts + LB_ROWS * 40;                        // [128][HC + 8]
  __shared__ int last;
  const uint32_t sd = smem_u32(dts), sh = smem_u32(hs);
  const int cpr = HC / 8;
  for (int i = t; i < LB_ROWS * cpr; i += LB_THREADS) {
    const int r = i / cpr, c = i % cpr, m = m0 + r;
    const uint32_t dst = sh + (r * lh + c * 8) * 2;
    if (m < a.M)
      cp_async16(dst, a.h1 + (size_t)m * a.H + hc * HC + c * 8);
    else
      zero16(dst);
  }
  for (int e = t; e < LB_ROWS * 64; e += LB_THREADS) {
    const int r = e >> 6, c = e & 63, m = m0 + r;
    float v = 0.f;
    if (m < a.M && c < 32) {
      const int cb = c < 16 ? 0 : a.n_cc_q, ce = c < 16 ? a.n_cc_q : a.n_cc;
      for (int k = cb; k < ce; ++k) v += a.part_dt[((size_t)k * a.M + m) * 16 + (c & 15)];
      v *= a.scale;
    }
    const __nv_bfloat16 bv = __float2bfloat16_rn(v);
    if (c < 32) dts[r * 40 + c] = bv;
    if (hc == 0 && m < a.M) a.dtpad[(size_t)m * 64 + c] = bv;
  }
  cp_async_wait_all();
  __syncthreads();

  // partial dA: D[32 x HC] = dt^T [32 x 128] h1 [128 x HC]; warp w takes the 16-column
  // groups w, w + 8, ... for both 16-row halves (q, v)
  const int warp = t >> 5, lane = t & 31, g4 = lane >> 2, t4 = lane & 3;
  for (int grp = warp; grp < HC / 16; grp += 8) {
    float acc[2][2][4];
#pragma unroll
    for (int i = 0; i < 2; ++i)
#pragma unroll
      for (int j = 0; j < 2; ++j) acc[i][j][0] = acc[i][j][1] = acc[i][j][2] = acc[i][j][3] = 0.f;
#pragma unroll
    for (int kk = 0; kk < LB_ROWS / 16; ++kk) {
      uint32_t b0, b1, b2, b3;
      {
        const int m = kk * 16 + (lane & 7) + ((lane >> 3) & 1) * 8, n = grp * 16 + (lane >> 4) * 8;
        ldsm4t(sh + (m * lh + n) * 2, b0, b1, b2, b3);
      }
#pragma unroll
      for (int mt = 0; mt < 2; ++mt) {
        uint32_t a0, a1, a2, a3;
        const int m = kk * 16 + (lane & 7) + (lane >> 4) * 8, n = mt * 16 + ((lane >> 3) & 1) * 8;
        ldsm4t(sd + (m * 40 + n) * 2, a0, a1, a2, a3);
        mma16816(acc[mt][0], a0, a1, a2, a3, b0, b1);
        mma16816(acc[mt][1], a0, a1, a2, a3, b2, b3);
      }
    }
    float* P = a.part_dA + (size_t)rg * 32 * a.H + hc * HC + grp * 16;
#pragma unroll
    for (int mt = 0; mt < 2; ++mt)
#pragma unroll
      for (int nt = 0; nt < 2; ++nt) {
        const int row = mt * 16 + g4, col = nt * 8 + 2 * t4;
        P[(size_t)row * a.H + col] = acc[mt][nt][0];
        P[(size_t)row * a.H + col + 1] = acc[mt][nt][1];
        P[(size_t)(row + 8) * a.H + col] = acc[mt][nt][2];
        P[(size_t)(row + 8) * a.H + col + 1] = acc[mt][nt][3];
      }
  }
  __threadfence();
  __syncthreads();
  if (t == 0) last = atomicAdd(&a.counters[hc], 1) == a.n_rg - 1;
  __syncthreads();
  if (!last) return;
  __threadfence();
  for (int e = t; e < 32 * HC; e += LB_THREADS) {
    const int row = e / HC, col = hc * HC + e % HC;
    float v = 0.f;
    for (int g = 0; g < a.n_rg; ++g) v += __ldcg(a.part_dA + ((size_t)g * 32 + row) * a.H + col);
    if (row < 16)
      a.dA_q[(size_t)row * a.H + col] = v;
    else
      a.dA_v[(size_t)(row - 16) * a.H + col] = v;
  }
  if (t == 0) a.counters[hc] = 0;
}

int chunk_width(int a, int b) {
  for (int w : {256, 192, 128, 64})
    if (a % w == 0 && b % w == 0) return w;
  return 0;
}

struct BwdShape {
  int CW, n_cc_q, n_cc, n_rb, n_rg, HC, n_hc, n_db_blocks;
  size_t part_dB, part_dt, part_dA, counters, total;
};

BwdShape bwd_shape(int M, int H, int qd, int kvd) {
  BwdShape b;
  b.CW = chunk_width(qd, kvd);
  b.n_cc_q = b.CW ? qd / b.CW : 0;
  b.n_cc = b.CW ? (qd + kvd) / b.CW : 0;
  b.n_rb = (M + LB_ROWS - 1) / LB_ROWS;
  b.n_rg = b.n_rb;
  b.HC = chunk_width(H, H);
  b.n_hc = b.HC ? H / b.HC : 0;
  b.n_db_blocks = ((qd + kvd) * 16 + LB_THREADS - 1) / LB_THREADS;
  size_t off = 0;
  auto take = [&](size_t bytes) {
    const size_t o = off;
    off = round_up(off + bytes, 256);
    return o;
  };
  b.part_dB = take((size_t)b.n_rb * (qd + kvd) * 16 * 4);
  b.part_dt = take((size_t)b.n_cc * M * 16 * 4);
  b.part_dA = take((size_t)b.n_rg * 32 * H * 4);
  b.counters = take((size_t)std::max(b.n_hc, 1) * 4);
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

int norm_lora_fwd(const __nv_bfloat16* x, const __nv_bfloat16* w, __nv_bfloat16* h1, int M, int H, float eps,
                  const nf4ls_lora* l, int qd, int kvd, float scale, __nv_bfloat16* tpad, __nv_bfloat16* bup,
                  __nv_bfloat16* adn, __nv_bfloat16* bqt, __nv_bfloat16* bvt, cudaStream_t s) {
  if (H % 16 || H > 32 * 24 * 8 || qd % 8 || kvd % 8) return fail(NF4LS_SHAPE, "norm_lora_fwd: H %d", H);
  NormLoraArgs a;
  a.x = x;
  a.w = w;
  a.h1 = h1;
  a.M = M;
  a.H = H;
  a.eps = eps;
  a.Aq = l->A_q;
  a.Av = l->A_v;
  a.Bq = l->B_q;
  a.Bv = l->B_v;
  a.tpad = tpad;
  a.qd = qd;
  a.kvd = kvd;
  a.scale = scale;
  a.bup = bup;
  a.adn = adn;
  a.bqt = bqt;
  a.bvt = bvt;
  const size_t smem = (size_t)NL_ROWS * (H + 8) * 2 + (size_t)NL_WARPS * NL_ROWS * 32 * 4;
  const int grid = (M + NL_ROWS - 1) / NL_ROWS;
  const int per_lane = (H / 8 + 31) / 32;
  // one instance per register budget of the row: SmolLM2 (576: 3), 8B (4096: 16), 32B (5120: 20)
  if (per_lane <= 4) {
    NF4_TRY(allow_smem((const void*)k_norm_lora_fwd<4>, smem));
    k_norm_lora_fwd<4><<<grid, NL_THREADS, smem, s>>>(a);
  } else if (per_lane <= 16) {
    NF4_TRY(allow_smem((const void*)k_norm_lora_fwd<16>, smem));
    k_norm_lora_fwd<16><<<grid, NL_THREADS, smem, s>>>(a);
  } else {
    NF4_TRY(allow_smem((const void*)k_norm_lora_fwd<24>, smem));
    k_norm_lora_fwd<24><<<grid, NL_THREADS, smem, s>>>(a);
  }
  note_launch();
  NF4_CUDA_TRY(cudaGetLastError());
  return NF4LS_OK;
}

int lora_bwd(const __nv_bfloat16* dqkv, int ld, int vcol, int M, int H, int qd, int kvd, const __nv_bfloat16* tpad,
             const __nv_bfloat16* bqt, const __nv_bfloat16* bvt, const __nv_bfloat16* h1, float scale,
             __nv_bfloat16* dtpad, const nf4ls_lora_grads* g, void* part, cudaStream_t s) {
  const BwdShape sh = bwd_shape(M, H, qd, kvd);
  if (!sh.CW || !sh.HC || ld % 8 || vcol % 8) return fail(NF4LS_SHAPE, "lora_bwd: qd %d, kvd %d, H %d", qd, kvd, H);
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
  a.part_dA = reinterpret_cast<float*>(pb + sh.part_dA);
  a.counters = reinterpret_cast<int*>(pb + sh.counters);
  a.n_rb = sh.n_rb;
  a.n_rg = sh.n_rg;
  a.HC = sh.HC;
  a.n_hc = sh.n_hc;
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
  NF4_CUDA_TRY(cudaGetLastError());
  const size_t smem2 = (size_t)LB_ROWS * 40 * 2 + (size_t)LB_ROWS * (sh.HC + 8) * 2;
  NF4_TRY(allow_smem((const void*)k_lora_bwd_final, smem2));
  k_lora_bwd_final<<<sh.n_db_blocks + sh.n_rg * sh.n_hc, LB_THREADS, smem2, s>>>(a);
  note_launch();
  NF4_CUDA_TRY(cudaGetLastError());
  return NF4LS_OK;
}

}  // namespace nf4ls
