// K6/K7: the LoRA products of the q_proj and v_proj adapters (r = 16).
//
// "Soup v0.72.4 技术解析" §4.2 (LoRA r=16, alpha=32 on q_proj and v_proj) and
// "Soup 层流式 NF4 训练实测：在 4 GB 显存上以位级一致标准完成 8B 模型 LoRA 微调"
// §2.2 check 2 (LoRA gradients nonzero in every layer): the adapter adds
// s (x A^T) B^T to the q and v projections (s = alpha / r) and trains A and B.  The
// up-projection is folded into the q/k/v GEMM as an extra 64-wide reduction block;
// this file holds the skinny products of the backward, all of them HBM-bound, in four
// launches (the down-projection t = [h1 A_q^T | h1 A_v^T] of the forward is a second
// output of the input RMSNorm's launch, body.cu):
//
//   k_lora_bwd_partial: per (128-row block, column chunk of dq or dv) the partial sums
//     of dB = s dX^T t (over the rows) and of dt = s dX B (over the columns), from one
//     read of dX;
//   k_lora_bwd_reduce, launched twice: dt (partials added in column-chunk order,
//     rounded to bf16: the extra operand of the dL/dx GEMM), then dB (partials added in
//     row-block order);
//   k_lora_bwd_da: dA = dt^T h1, a cluster of eight blocks per 64 columns of h1, each
//     over an eighth of the rows, the partials added across the cluster in shared memory.
// The layer's backward runs the last two (dB and dA, which nothing in the layer waits
// for) on a side stream beside the q/k/v dL/dx GEMM.
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
// A launch runs blocks first_block, first_block + 1, .. (dt and dB go to different
// streams).
__global__ void __launch_bounds__(LB_THREADS) k_lora_bwd_reduce(const __grid_constant__ LoraBwdArgs a,
                                                                int first_block) {
  const int t = threadIdx.x, blk = first_block + (int)blockIdx.x;
  const int NB = a.qd + a.kvd;
  if (blk < a.n_db_blocks) {
    const int e = blk * LB_THREADS + t;
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
  const int m = (blk - a.n_db_blocks) * 8 + (t >> 5), c = t & 31;
  if (m >= a.M) return;
  const int cb = c < 16 ? 0 : a.n_cc_q, ce = c < 16 ? a.n_cc_q : a.n_cc;
  float v = 0.f;
  for (int k = cb; k < ce; ++k) v += a.part_dt[((size_t)k * a.M + m) * 16 + (c & 15)];
  a.dtpad[(size_t)m * 64 + c] = __float2bfloat16_rn(v * a.scale);
  a.dtpad[(size_t)m * 64 + 32 + c] = __float2bfloat16_rn(0.f);
}

// dA = dt^T h1.  A cluster of DA_SPLIT CTAs per 64 columns of h1: CTA y of the cluster
// takes the row range [y R, (y + 1) R) (R = M / DA_SPLIT rounded up to whole 64-row
// chunks), streamed through three cp.async stages.  Warp w takes rows 16 w .. 16 w + 15 of
// every chunk, the four warp partials are added in warp order, and the
// cluster's eight partials are added in CTA order through distributed shared memory,
// CTA y producing output rows 4 y .. 4 y + 3.  The sum order is fixed by M alone.
constexpr int DA_COLS = 64, DA_ROWS = 64, DA_DS = 40, DA_HS = DA_COLS + 8, DA_STAGES = 3;
constexpr int DA_SPLIT = 8, DA_THREADS = 128, DA_WARPS = DA_THREADS / 32;
constexpr int DA_KSTEPS = DA_ROWS / (16 * DA_WARPS);  // k-steps of 16 rows per warp and chunk
constexpr int DA_PIECES = 4 + DA_COLS / 8;  // 16-byte pieces per row: dt (32 columns), h1
constexpr int DA_STAGE_BYTES = DA_ROWS * (DA_DS + DA_HS) * 2;
constexpr int DA_RED_BYTES = DA_WARPS * 32 * DA_COLS * 4;  // warp partials
constexpr int DA_SMEM = DA_STAGES * DA_STAGE_BYTES;  // 42 KB: five CTAs per SM
static_assert(DA_RED_BYTES + 32 * DA_COLS * 4 <= DA_SMEM, "partials fit in the stages");
static_assert(32 % DA_SPLIT == 0, "output rows split evenly over the cluster");

__global__ void __cluster_dims__(1, DA_SPLIT, 1) __launch_bounds__(DA_THREADS)
    k_lora_bwd_da(const __grid_constant__ LoraBwdArgs a) {
  extern __shared__ __align__(16) uint8_t smem[];
  const int t = threadIdx.x, warp = t >> 5, lane = t & 31, g4 = lane >> 2, t4 = lane & 3;
  const int c0 = blockIdx.x * DA_COLS;
  const int y = (int)cluster_ctarank();
  const int R = ((a.M + DA_SPLIT - 1) / DA_SPLIT + DA_ROWS - 1) / DA_ROWS * DA_ROWS;
  const int r0 = y * R, r1 = min(a.M, r0 + R);
  const int n_chunks = r1 > r0 ? (r1 - r0 + DA_ROWS - 1) / DA_ROWS : 0;
  auto ds = [&](int b) { return reinterpret_cast<__nv_bfloat16*>(smem + (size_t)b * DA_STAGE_BYTES); };
  auto hs = [&](int b) {
    return reinterpret_cast<__nv_bfloat16*>(smem + (size_t)b * DA_STAGE_BYTES + DA_ROWS * DA_DS * 2);
  };
  auto stage = [&](int ch, int b) {  // 128 rows x (4 pieces of dt + DA_COLS / 8 pieces of h1)
    for (int i = t; i < DA_ROWS * DA_PIECES; i += DA_THREADS) {
      const int r = i / DA_PIECES, q = i % DA_PIECES, m = r0 + ch * DA_ROWS + r;
      const uint32_t dst = q < 4 ? smem_u32(ds(b) + r * DA_DS + q * 8) : smem_u32(hs(b) + r * DA_HS + (q - 4) * 8);
      if (m >= r1)
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
    // the stage chunk ch + DA_STAGES - 1 goes to was last read for chunk ch - 1
    __syncthreads();
    if (ch + DA_STAGES - 1 < n_chunks)
      stage(ch + DA_STAGES - 1, (ch + DA_STAGES - 1) % DA_STAGES);
    else
      asm volatile("cp.async.commit_group;" ::: "memory");
    asm volatile("cp.async.wait_group %0;" ::"n"(DA_STAGES - 1) : "memory");
    __syncthreads();  // chunk ch has landed for every thread
#pragma unroll
    for (int kk = 0; kk < DA_KSTEPS; ++kk) {
      const int kr = (warp * DA_KSTEPS + kk) * 16;  // 16 rows of the chunk
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
  }
  asm volatile("cp.async.wait_all;" ::: "memory");
  __syncthreads();
  float* red = reinterpret_cast<float*>(smem);  // the stages are free now
  float* P = reinterpret_cast<float*>(smem + DA_RED_BYTES);  // this CTA's [32][DA_COLS] partial
  float* R_ = red + warp * (32 * DA_COLS);
#pragma unroll
  for (int mt = 0; mt < 2; ++mt)
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
      const int row = mt * 16 + g4, col = nt * 8 + 2 * t4;
      R_[row * DA_COLS + col] = acc[mt][nt][0];
      R_[row * DA_COLS + col + 1] = acc[mt][nt][1];
      R_[(row + 8) * DA_COLS + col] = acc[mt][nt][2];
      R_[(row + 8) * DA_COLS + col + 1] = acc[mt][nt][3];
    }
  __syncthreads();
  for (int e = t; e < 32 * DA_COLS; e += DA_THREADS) {
    float v = 0.f;
    for (int w = 0; w < DA_WARPS; ++w) v += red[w * (32 * DA_COLS) + e];
    P[e] = v;
  }
  cluster_sync_all();  // every CTA's partial is in its shared memory
  constexpr int ROWS_PER_CTA = 32 / DA_SPLIT;
  for (int e = t; e < ROWS_PER_CTA * DA_COLS; e += DA_THREADS) {
    const int row = y * ROWS_PER_CTA + e / DA_COLS, col = e % DA_COLS;
    const uint32_t local = smem_u32(P + row * DA_COLS + col);
    float part[DA_SPLIT], v = 0.f;  // the partials fetched together, then added in CTA order
#pragma unroll
    for (int c = 0; c < DA_SPLIT; ++c) part[c] = ld_cluster_f32(mapa_shared(local, (uint32_t)c));
#pragma unroll
    for (int c = 0; c < DA_SPLIT; ++c) v += part[c];
    if (row < 16)
      a.dA_q[(size_t)row * a.H + c0 + col] = v;
    else
      a.dA_v[(size_t)(row - 16) * a.H + c0 + col] = v;
  }
  cluster_sync_all();  // no CTA leaves while another still reads its partial
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

int lora_bwd(const __nv_bfloat16* dqkv, int ld, int vcol, int M, int H, int qd, int kvd, const __nv_bfloat16* tpad,
             const __nv_bfloat16* bqt, const __nv_bfloat16* bvt, const __nv_bfloat16* h1, float scale,
             __nv_bfloat16* dtpad, const nf4ls_lora_grads* g, void* part, int phases, cudaStream_t s) {
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
  if (phases & LORA_BWD_DT) {
    const size_t smem1 = (size_t)LB_ROWS * (sh.CW + 8) * 2 + (size_t)LB_ROWS * 24 * 2 + 16ull * (sh.CW + 8) * 2;
    NF4_TRY(allow_smem((const void*)k_lora_bwd_partial, smem1));
    k_lora_bwd_partial<<<dim3(sh.n_rb, sh.n_cc), LB_THREADS, smem1, s>>>(a);
    note_launch();
    k_lora_bwd_reduce<<<(M + 7) / 8, LB_THREADS, 0, s>>>(a, sh.n_db_blocks);
    note_launch();
  }
  if (phases & LORA_BWD_DB_DA) {
    k_lora_bwd_reduce<<<sh.n_db_blocks, LB_THREADS, 0, s>>>(a, 0);
    note_launch();
    NF4_TRY(allow_smem((const void*)k_lora_bwd_da, DA_SMEM));
    k_lora_bwd_da<<<dim3(H / DA_COLS, DA_SPLIT), DA_THREADS, DA_SMEM, s>>>(a);
    note_launch();
  }
  NF4_CUDA_TRY(cudaGetLastError());
  return NF4LS_OK;
}

}  // namespace nf4ls
