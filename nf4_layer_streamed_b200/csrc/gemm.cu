// K3/K4/K5: tcgen05 GEMMs for the frozen base linears, with the NF4 weights
// decoded inside the mainloop, and the dense bf16 variant (lm_head, and the
// dequantise-then-multiply path).
//
// The products come from the layer-streaming pages: the frozen base linears run
// for the forward, for the checkpoint recompute and for dL/dx = W^T dL/dy
// ("4GB 显存微调 8B 模型是真的", mechanism section;
// "Soup 层流式 NF4 训练实测：在 4 GB 显存上以位级一致标准完成 8B 模型 LoRA 微调"
// §4.4: C = 6, no dL/dW), on NF4 weights with double-quantised absmax
// (§2.1, §2.4).  The decode is the dequantisation of §2.4 exactly:
// w^ = bf16_rne(fp32(nf4[code] * fp32(fp32(code8[q8] * nested) + offset))).
//
// Tile: 256 tokens x 256 output features per CTA, 64-deep reduction stages,
// 3 stages.  The 256 tokens are two 128-row MMAs (M = 128, N = 256, K = 16) that
// share one B tile, so each decoded weight is used by 256 tokens; the two fp32
// accumulators take all 512 TMEM columns.
//
// Warp roles (one CTA per SM):
//   warp 0      TMA producer: A tiles (128-byte swizzle), dense B tiles or the packed
//               NF4 code tiles, the LoRA extra block.
//   warp 1      TMEM allocation and the MMA issuer (one elected thread).
//   warps 2-5   epilogue: tcgen05.ld of the accumulators, fused epilogue, bf16 stores.
//   warps 6-13  NF4 decoders (decode variant only): each thread turns one 64-weight
//               block (32 code bytes + its two-level scale) into 128 bytes of bf16 in
//               the swizzled layout the MMA reads, K-major for the forward, N-major
//               for dL/dx.
//
// The decode builds, per block, the 16 possible bf16 outputs nf4[j] * s (16 fp32
// multiplies, 8 packed conversions) as byte tables and looks codes up with byte
// permutes (prmt), four codes per permute.
//
// Every wait on an mbarrier is bounded (common.cuh); on expiry the kernel records
// the site in the device error record, all roles leave their loops, and TMEM is
// released before exit.
#include <algorithm>
#include <cstring>
#include <mutex>

#include "common.cuh"
#include "internal.h"

namespace nf4ls {

namespace {

constexpr int BM = 256, BN = 256, BK = 64, STAGES = 3;
constexpr int A_BYTES = BM * BK * 2;  // 32 KB
constexpr int B_BYTES = BN * BK * 2;  // 32 KB
constexpr int C_BYTES = BN * BK / 2;  // 8 KB of packed codes
constexpr int STAGE_BYTES = A_BYTES + B_BYTES + C_BYTES;
constexpr int SMEM_BYTES = 1024 + STAGES * STAGE_BYTES + 256 + 1024;
constexpr int NUM_DECODERS = 256;

struct GemmParams {
  CUtensorMap tmA, tmAx, tmB, tmBx;
  CUtensorMap tmC[4];
  CUtensorMap tmAux;   // CTA-pair residual / dSwiGLU side input (x, or [g | u]), box 64 cols x 128 rows;
  CUtensorMap tmAux2;  //   RoPE: the cos (tmAux) and sin (tmAux2) tables [d/2, seq], box 128 positions;
                       //   SwiGLU: the act output (tmAux) and the kept [g | u] (tmAux2), box 64 x 128
  int M, N, K, num_kb, has_extra, n_mt;
  int n_seg, swiglu, dense_swiglu_rows;
  int seg_start[5];
  const uint8_t* q8[4];
  const float* nested[4];
  const float* offset[4];
  int seg_cols;
  // epilogue
  int epi;
  __nv_bfloat16* out;
  int ldo;
  const __nv_bfloat16* aux0;
  int ld_aux0;
  __nv_bfloat16* aux_out;
  int ld_aux_out, inter;
  const float* rope_cos;
  const float* rope_sin;
  int seq, head_dim, rope_cols;
  float* out_f32;
  const float* alpha;
  int accumulate;
  int aux_tma;  // CTA-pair epilogue: 1 = residual / dSwiGLU side input, 2 = RoPE tables, by TMA into the freed stage
                // memory; 3 = SwiGLU outputs staged there and written by TMA stores
  int half;   // CTA-pair kernel: 256-token pair tiles (one 128-row accumulator per CTA)
  int tile0;  // CTA-pair kernel: tile index of the launch's first pair (mt fastest)
  float nf4[16];
  float code8[256];
  int* err;
};

// ------------------------------------------------------------------------------ decode
__device__ __forceinline__ void decode_block(uint32_t row_addr, int row_in_atom, const uint32_t (&w)[8], float s,
                                             const float (&nf4)[16]) {
  uint32_t p[8];
#pragma unroll
  for (int j = 0; j < 8; ++j) p[j] = pack_bf16x2(__fmul_rn(nf4[2 * j], s), __fmul_rn(nf4[2 * j + 1], s));
  // hi/lo bytes of entries 0-3, 4-7, 8-11, 12-15
  const uint32_t th0 = prmt(p[0], p[1], 0x7531u), th1 = prmt(p[2], p[3], 0x7531u);
  const uint32_t th2 = prmt(p[4], p[5], 0x7531u), th3 = prmt(p[6], p[7], 0x7531u);
  const uint32_t tl0 = prmt(p[0], p[1], 0x6420u), tl1 = prmt(p[2], p[3], 0x6420u);
  const uint32_t tl2 = prmt(p[4], p[5], 0x6420u), tl3 = prmt(p[6], p[7], 0x6420u);
#pragma unroll
  for (int c = 0; c < 8; ++c) {
    uint32_t o[4];
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      // nibbles of x (low 16 bits) hold the codes of elements 1,0,3,2 of this quad
      const uint32_t x = h ? (w[c] >> 16) : w[c];
      const uint32_t sel = x & 0x7777u;
      const uint32_t m = prmt(0x0000FF00u, 0u, (x >> 3) & 0x1111u);  // 0xFF where code >= 8
      const uint32_t hA = prmt(th0, th1, sel), hB = prmt(th2, th3, sel);
      const uint32_t lA = prmt(tl0, tl1, sel), lB = prmt(tl2, tl3, sel);
      const uint32_t hi = (hA & ~m) | (hB & m);
      const uint32_t lo = (lA & ~m) | (lB & m);
      o[2 * h] = prmt(lo, hi, 0x4051u);      // elements 0,1
      o[2 * h + 1] = prmt(lo, hi, 0x6273u);  // elements 2,3
    }
    st_shared_v4(row_addr + ((uint32_t)(c ^ row_in_atom) << 4), o[0], o[1], o[2], o[3]);
  }
}

__device__ __forceinline__ void zero_block(uint32_t row_addr) {
#pragma unroll
  for (int c = 0; c < 8; ++c) st_shared_v4(row_addr + (c << 4), 0u, 0u, 0u, 0u);
}

__device__ __forceinline__ int find_seg(const GemmParams& p, int row) {
  int s = 0;
#pragma unroll
  for (int i = 1; i < 4; ++i)
    if (i < p.n_seg && row >= p.seg_start[i]) s = i;
  return s;
}

// x * sigmoid(x) and sigmoid(x) with the fast exponential and divide: the results are
// rounded to bf16, far coarser than either approximation.
__device__ __forceinline__ float sigmoid_f(float x) { return __fdividef(1.0f, 1.0f + __expf(-x)); }
__device__ __forceinline__ float silu_f(float x) { return __fdividef(x, 1.0f + __expf(-x)); }
__device__ __forceinline__ float round_bf16(float x) { return __bfloat162float(__float2bfloat16_rn(x)); }

__device__ __forceinline__ void store32(__nv_bfloat16* dst, const float (&v)[32]) {
  uint4* d = reinterpret_cast<uint4*>(dst);
#pragma unroll
  for (int i = 0; i < 4; ++i)
    d[i] = make_uint4(pack_bf16x2(v[8 * i + 0], v[8 * i + 1]), pack_bf16x2(v[8 * i + 2], v[8 * i + 3]),
                      pack_bf16x2(v[8 * i + 4], v[8 * i + 5]), pack_bf16x2(v[8 * i + 6], v[8 * i + 7]));
}

__device__ __forceinline__ void load32_bf16(const __nv_bfloat16* src, float (&v)[32]) {
  const uint4* s = reinterpret_cast<const uint4*>(src);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const uint4 u = s[i];
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      v[8 * i + 2 * j] = bf16_lo(w[j]);
      v[8 * i + 2 * j + 1] = bf16_hi(w[j]);
    }
  }
}

__device__ __forceinline__ void ld_acc(uint32_t taddr, float (&v)[32]) {
  uint32_t r[32];
  tmem_ld32(taddr, r);
  tmem_wait_ld();
#pragma unroll
  for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
}

// ------------------------------------------------------------------------------ epilogue
// The epilogue warps of TMEM lane quarter q turn the two 128 x 256 fp32 accumulators of
// their CTA (tokens m0 + [0, 256), output features of tile nt) into bf16 results.
// The work of a quarter is a list of 16-column items (per accumulator: 16 column
// chunks, 8 gate/up chunk pairs for SwiGLU, or per head the RoPE half-chunk pairs);
// warp `part` of the `nparts` warps that share the quarter takes every nparts-th item.
__device__ __forceinline__ void ld_acc16(uint32_t taddr, float (&v)[16]) {
  uint32_t r[16];
  tmem_ld16(taddr, r);
  tmem_wait_ld();
#pragma unroll
  for (int i = 0; i < 16; ++i) v[i] = __uint_as_float(r[i]);
}

__device__ __forceinline__ void store16(__nv_bfloat16* dst, const float (&v)[16]) {
  uint4* d = reinterpret_cast<uint4*>(dst);
#pragma unroll
  for (int i = 0; i < 2; ++i)
    d[i] = make_uint4(pack_bf16x2(v[8 * i + 0], v[8 * i + 1]), pack_bf16x2(v[8 * i + 2], v[8 * i + 3]),
                      pack_bf16x2(v[8 * i + 4], v[8 * i + 5]), pack_bf16x2(v[8 * i + 6], v[8 * i + 7]));
}

__device__ __forceinline__ void load16_bf16(const __nv_bfloat16* src, float (&v)[16]) {
  const uint4* s = reinterpret_cast<const uint4*>(src);
#pragma unroll
  for (int i = 0; i < 2; ++i) {
    const uint4 u = s[i];
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      v[8 * i + 2 * j] = bf16_lo(w[j]);
      v[8 * i + 2 * j + 1] = bf16_hi(w[j]);
    }
  }
}

// Pulls the rows of the epilogue's bf16 side input (the residual, or g and u) that this
// CTA will read into L2 while the mainloop runs: threads t of nthreads, one 128-byte
// line per prefetch.  A hint only; nothing waits for it.
__device__ __forceinline__ void prefetch_aux(const GemmParams& p, int m0, int nt, int t, int nthreads, int rows = 256) {
  if (p.epi != EPI_RESID && p.epi != EPI_DSWIGLU) return;
  const int col = nt * BN;
  if (col >= p.N) return;
  const int span = min(BN, p.N - col) * 2;  // bytes of one row segment
  const int lines = (span + 127) / 128;
  const int segs = p.epi == EPI_DSWIGLU ? 2 : 1;
  const int total = rows * segs * lines;
  for (int i = t; i < total; i += nthreads) {
    const int r = i / (segs * lines), rest = i % (segs * lines);
    const int m = m0 + r;
    if (m >= p.M) continue;
    const int sgi = rest / lines, ln = rest % lines;
    const char* a = reinterpret_cast<const char*>(p.aux0 + (size_t)m * p.ld_aux0 + col + (sgi ? p.inter : 0)) + ln * 128;
    asm volatile("prefetch.global.L2 [%0];" ::"l"(a));
  }
}

__device__ __forceinline__ void unpack16(uint4 a, uint4 b, float (&v)[16]) {
  const uint32_t w[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    v[2 * j] = bf16_lo(w[j]);
    v[2 * j + 1] = bf16_hi(w[j]);
  }
}

// WITH_F32: whether the fp32 accumulate epilogue (used only by dense products) is
// compiled in; the NF4-decode kernels leave it out, which keeps them free of spills.
template <int n_acc = 2, bool WITH_F32 = true>
__device__ __forceinline__ void epilogue_rows(const GemmParams& p, uint32_t tmem, int m0, int nt, int q, int lane,
                                              int part = 0, int nparts = 1) {
  constexpr int CW = 16;
  int item = 0;
  for (int a = 0; a < n_acc; ++a) {
    const int m = m0 + a * 128 + q * 32 + lane;
    const bool mv = m < p.M;
    const uint32_t tb = tmem + ((uint32_t)(q * 32) << 16) + a * 256;
    float v[CW], w[CW];
    if (p.epi == EPI_SWIGLU) {
      for (int c = 0; c < 128 / CW; ++c) {
        if ((item++ % nparts) != part) continue;
        ld_acc16(tb + c * CW, v);
        ld_acc16(tb + 128 + c * CW, w);
        if (!mv) continue;
        const int col = nt * 128 + c * CW;
        float o[CW];
#pragma unroll
        for (int i = 0; i < CW; ++i) {
          v[i] = round_bf16(v[i]);
          w[i] = round_bf16(w[i]);
          o[i] = silu_f(v[i]) * w[i];
        }
        store16(p.out + (size_t)m * p.ldo + col, o);
        if (p.aux_out) {
          store16(p.aux_out + (size_t)m * p.ld_aux_out + col, v);
          store16(p.aux_out + (size_t)m * p.ld_aux_out + p.inter + col, w);
        }
      }
    } else if (p.epi == EPI_ROPE) {
      const int d = p.head_dim, half = d / 2;
      const int pos = m % p.seq;
      for (int h = 0; h < BN / d; ++h) {
        const int hc = nt * BN + h * d;
        if (hc >= p.N) break;
        if (hc < p.rope_cols) {
          for (int i = 0; i < half / CW; ++i) {
            if ((item++ % nparts) != part) continue;
            // frequency-major tables: the 32 lanes (consecutive positions) read one line;
            // the loads are in flight during the TMEM loads
            const float* cs = p.rope_cos + (size_t)(i * CW) * p.seq + pos;
            const float* sn = p.rope_sin + (size_t)(i * CW) * p.seq + pos;
            float c_[CW], s_[CW];
#pragma unroll
            for (int j = 0; j < CW; ++j) {
              c_[j] = cs[(size_t)j * p.seq];
              s_[j] = sn[(size_t)j * p.seq];
            }
            ld_acc16(tb + h * d + i * CW, v);
            ld_acc16(tb + h * d + half + i * CW, w);
            if (!mv) continue;
            float o1[CW], o2[CW];
#pragma unroll
            for (int j = 0; j < CW; ++j) {
              o1[j] = v[j] * c_[j] - w[j] * s_[j];
              o2[j] = w[j] * c_[j] + v[j] * s_[j];
            }
            store16(p.out + (size_t)m * p.ldo + hc + i * CW, o1);
            store16(p.out + (size_t)m * p.ldo + hc + half + i * CW, o2);
          }
        } else {
          for (int c = 0; c < d / CW; ++c) {
            if ((item++ % nparts) != part) continue;
            ld_acc16(tb + h * d + c * CW, v);
            if (mv) store16(p.out + (size_t)m * p.ldo + hc + c * CW, v);
          }
        }
      }
    } else if (p.epi == EPI_STORE) {
      for (int c = 0; c < BN / CW; ++c) {
        const int col = nt * BN + c * CW;
        if (col >= p.N) break;
        if ((item++ % nparts) != part) continue;
        ld_acc16(tb + c * CW, v);
        if (mv) store16(p.out + (size_t)m * p.ldo + col, v);
      }
    } else if (WITH_F32 && p.epi == EPI_ACC_F32) {
      for (int c = 0; c < BN / CW; ++c) {
        const int col = nt * BN + c * CW;
        if (col >= p.N) break;
        if ((item++ % nparts) != part) continue;
        float4* dst = reinterpret_cast<float4*>(p.out_f32 + (size_t)m * p.ldo + col);
        float4 old[CW / 4];
        if (mv && p.accumulate) {
#pragma unroll
          for (int i = 0; i < CW / 4; ++i) old[i] = dst[i];
        }
        ld_acc16(tb + c * CW, v);
        if (!mv) continue;
        if (p.accumulate) {
          const float al = p.alpha[m];
#pragma unroll
          for (int i = 0; i < CW / 4; ++i) {
            v[4 * i + 0] += al * old[i].x;
            v[4 * i + 1] += al * old[i].y;
            v[4 * i + 2] += al * old[i].z;
            v[4 * i + 3] += al * old[i].w;
          }
        }
#pragma unroll
        for (int i = 0; i < CW / 4; ++i) dst[i] = make_float4(v[4 * i], v[4 * i + 1], v[4 * i + 2], v[4 * i + 3]);
      }
    }
  }
  if (p.epi != EPI_RESID && p.epi != EPI_DSWIGLU) return;
  // Residual / dSwiGLU: this warp's items k = part, part + nparts, ... over both
  // accumulators (item k: accumulator k / nch, chunk k % nch), with the bf16 side input
  // of the next item loaded while the current one is processed.
  const int nch = min(BN, p.N - nt * BN) / CW;
  const int total = n_acc * nch;
  const bool dsw = p.epi == EPI_DSWIGLU;
  uint4 nx[4];
  auto load_side = [&](int k) {
    const int a = k / nch, c = k - a * nch;
    const int m = m0 + a * 128 + q * 32 + lane;
    if (m >= p.M) return;
    const uint4* src = reinterpret_cast<const uint4*>(p.aux0 + (size_t)m * p.ld_aux0 + nt * BN + c * CW);
    nx[0] = src[0];
    nx[1] = src[1];
    if (dsw) {
      const uint4* su = reinterpret_cast<const uint4*>(p.aux0 + (size_t)m * p.ld_aux0 + p.inter + nt * BN + c * CW);
      nx[2] = su[0];
      nx[3] = su[1];
    }
  };
  if (part < total) load_side(part);
  for (int k = part; k < total; k += nparts) {
    const uint4 cur[4] = {nx[0], nx[1], nx[2], nx[3]};
    if (k + nparts < total) load_side(k + nparts);
    const int a = k / nch, c = k - a * nch;
    const int m = m0 + a * 128 + q * 32 + lane;
    const int col = nt * BN + c * CW;
    float v[CW], g[CW];
    ld_acc16(tmem + ((uint32_t)(q * 32) << 16) + a * 256 + c * CW, v);
    if (m >= p.M) continue;
    unpack16(cur[0], cur[1], g);
    if (!dsw) {
#pragma unroll
      for (int i = 0; i < CW; ++i) v[i] += g[i];
      store16(p.out + (size_t)m * p.ldo + col, v);
    } else {
      float u[CW], du[CW];
      unpack16(cur[2], cur[3], u);
#pragma unroll
      for (int i = 0; i < CW; ++i) {
        const float sg = sigmoid_f(g[i]);
        du[i] = v[i] * g[i] * sg;
        v[i] = v[i] * u[i] * sg * (1.0f + g[i] * (1.0f - sg));
      }
      store16(p.out + (size_t)m * p.ldo + col, v);
      store16(p.out + (size_t)m * p.ldo + p.inter + col, du);
    }
  }
}

// The CTA-pair kernel's residual and dSwiGLU epilogues with their side input staged by
// TMA: once the accumulators are complete the pipeline's shared memory is free, and per
// 128-row accumulator one thread loads that accumulator's rows of the tile's side input
// (the residual x, or g and u: 4 or 4 + 4 boxes of 128 rows x 64 columns, 64 or 128 KB)
// into it; the epilogue warps then read their rows' 16-column chunks from there instead
// of one global load per chunk in flight.  Before the second accumulator's loads reuse
// the memory, every epilogue warp has arrived on aux_free after its last read of the
// first.  Same items, order and arithmetic as epilogue_rows' residual and dSwiGLU
// branches, so the results are identical.  issuer: the thread that issues the loads.
template <int n_acc>
__device__ __forceinline__ void epilogue_side_tma(const GemmParams& p, uint32_t tmem, int m0, int nt, int q, int lane,
                                                  int part, int nparts, uint8_t* stage_mem, uint64_t* aux_full,
                                                  uint64_t* aux_free, volatile int* abort_flag, bool issuer) {
  constexpr int CW = 16, BOX = 128 * 64 * 2;  // one box: 16 KB
  const bool dsw = p.epi == EPI_DSWIGLU;
  const int nch = min(BN, p.N - nt * BN) / CW;
  const uint32_t sm = smem_u32(stage_mem);
  int issued = 0;
  for (int a = 0; a < n_acc; ++a) {
    if (issuer) {
      // the first accumulator's rows are read by every epilogue warp before the memory is reused
      bool ok = a == 0 || mbar_wait(aux_free, (uint32_t)(a - 1) & 1, abort_flag, p.err, KID_GEMM, 16);
      if (ok) {
        mbar_arrive_expect_tx(&aux_full[a], (dsw ? 8 : 4) * BOX);
        for (int j = 0; j < 4; ++j) {
          tma_load_2d(stage_mem + j * BOX, &p.tmAux, &aux_full[a], nt * BN + 64 * j, m0 + a * 128);
          if (dsw)
            tma_load_2d(stage_mem + (4 + j) * BOX, &p.tmAux, &aux_full[a], p.inter + nt * BN + 64 * j, m0 + a * 128);
        }
        issued = a + 1;
      }
    }
    const bool have = __all_sync(0xffffffffu, mbar_wait(&aux_full[a], 0, abort_flag, p.err, KID_GEMM, 17));
    const int r = q * 32 + lane, m = m0 + a * 128 + r;
    for (int c = 0; c < nch; ++c) {
      if (((a * nch + c) % nparts) != part) continue;
      float v[CW];
      ld_acc16(tmem + ((uint32_t)(q * 32) << 16) + a * 256 + c * CW, v);
      if (!have || m >= p.M) continue;
      const uint32_t row = sm + (uint32_t)(c >> 2) * BOX + (uint32_t)r * 128;
      const uint32_t o0 = (uint32_t)(((c & 3) * 2) ^ (r & 7)) << 4, o1 = (uint32_t)(((c & 3) * 2 + 1) ^ (r & 7)) << 4;
      float g[CW];
      unpack16(ld_shared_v4(row + o0), ld_shared_v4(row + o1), g);
      const int col = nt * BN + c * CW;
      if (!dsw) {
#pragma unroll
        for (int i = 0; i < CW; ++i) v[i] += g[i];
        store16(p.out + (size_t)m * p.ldo + col, v);
      } else {
        float u[CW], du[CW];
        unpack16(ld_shared_v4(row + 4 * BOX + o0), ld_shared_v4(row + 4 * BOX + o1), u);
#pragma unroll
        for (int i = 0; i < CW; ++i) {
          const float sg = sigmoid_f(g[i]);
          du[i] = v[i] * g[i] * sg;
          v[i] = v[i] * u[i] * sg * (1.0f + g[i] * (1.0f - sg));
        }
        store16(p.out + (size_t)m * p.ldo + col, v);
        store16(p.out + (size_t)m * p.ldo + p.inter + col, du);
      }
    }
    if (a + 1 < n_acc) {  // this warp is done with the staged rows
      __syncwarp();
      if (lane == 0) mbar_arrive(aux_free);
    }
  }
  if (issuer && *abort_flag)  // let the loads already issued land before the CTA exits
    for (int a = 0; a < issued; ++a) mbar_wait_drain(&aux_full[a], 0);
}

// The CTA-pair kernel's RoPE epilogue with the cos and sin of its rows staged by TMA: per
// 128-row accumulator (128 consecutive positions, seq a multiple of 128) one thread loads
// both tables' [d/2 frequencies x 128 positions] blocks into the freed pipeline memory,
// and each thread reads its row's angles from there (consecutive lanes, consecutive
// words) instead of 32 global loads per 16-column chunk.  Same items, order and
// arithmetic as epilogue_rows' RoPE branch, so the results are identical.
template <int n_acc>
__device__ __forceinline__ void epilogue_rope_tma(const GemmParams& p, uint32_t tmem, int m0, int nt, int q, int lane,
                                                  int part, int nparts, uint8_t* stage_mem, uint64_t* aux_full,
                                                  uint64_t* aux_free, volatile int* abort_flag, bool issuer) {
  constexpr int CW = 16;
  const int d = p.head_dim, half = d / 2;
  const uint32_t tab_bytes = (uint32_t)half * 128 * 4;
  const float* cos_s = reinterpret_cast<const float*>(stage_mem);
  const float* sin_s = cos_s + half * 128;
  int issued = 0, item = 0;
  for (int a = 0; a < n_acc; ++a) {
    if (issuer) {
      // the first accumulator's angles are read by every epilogue warp before the memory is reused
      bool ok = a == 0 || mbar_wait(aux_free, (uint32_t)(a - 1) & 1, abort_flag, p.err, KID_GEMM, 18);
      if (ok) {
        const int pos0 = (m0 + a * 128) % p.seq;
        mbar_arrive_expect_tx(&aux_full[a], 2 * tab_bytes);
        tma_load_2d(stage_mem, &p.tmAux, &aux_full[a], pos0, 0);
        tma_load_2d(stage_mem + tab_bytes, &p.tmAux2, &aux_full[a], pos0, 0);
        issued = a + 1;
      }
    }
    const bool have = __all_sync(0xffffffffu, mbar_wait(&aux_full[a], 0, abort_flag, p.err, KID_GEMM, 19));
    const int r = q * 32 + lane, m = m0 + a * 128 + r;
    const bool mv = m < p.M;
    const uint32_t tb = tmem + ((uint32_t)(q * 32) << 16) + a * 256;
    float v[CW], w[CW];
    for (int h = 0; h < BN / d; ++h) {
      const int hc = nt * BN + h * d;
      if (hc >= p.N) break;
      if (hc < p.rope_cols) {
        for (int i = 0; i < half / CW; ++i) {
          if ((item++ % nparts) != part) continue;
          ld_acc16(tb + h * d + i * CW, v);
          ld_acc16(tb + h * d + half + i * CW, w);
          if (!mv || !have) continue;
          float c_[CW], s_[CW];
#pragma unroll
          for (int j = 0; j < CW; ++j) {
            c_[j] = cos_s[(i * CW + j) * 128 + r];
            s_[j] = sin_s[(i * CW + j) * 128 + r];
          }
          float o1[CW], o2[CW];
#pragma unroll
          for (int j = 0; j < CW; ++j) {
            o1[j] = v[j] * c_[j] - w[j] * s_[j];
            o2[j] = w[j] * c_[j] + v[j] * s_[j];
          }
          store16(p.out + (size_t)m * p.ldo + hc + i * CW, o1);
          store16(p.out + (size_t)m * p.ldo + hc + half + i * CW, o2);
        }
      } else {
        for (int c = 0; c < d / CW; ++c) {
          if ((item++ % nparts) != part) continue;
          ld_acc16(tb + h * d + c * CW, v);
          if (mv) store16(p.out + (size_t)m * p.ldo + hc + c * CW, v);
        }
      }
    }
    if (a + 1 < n_acc) {  // this warp is done with the staged angles
      __syncwarp();
      if (lane == 0) mbar_arrive(aux_free);
    }
  }
  if (issuer && *abort_flag)  // let the loads already issued land before the CTA exits
    for (int a = 0; a < issued; ++a) mbar_wait_drain(&aux_full[a], 0);
}

// The CTA-pair kernel's SwiGLU epilogue with its outputs written by TMA stores: every
// epilogue warp writes its 16-column chunks of act = silu(g) u (and, when kept, of g and
// u) as bf16 into 128-row x 64-column boxes (128-byte swizzle) in the pipeline's freed
// shared memory (act 2 boxes, g 2, u 2 per accumulator: 64 or 192 KB in all), arrives on
// `staged`, and one thread then stores the boxes (rows past M are clipped by the tensor
// maps).  Same items and arithmetic as epilogue_rows' SwiGLU branch; whole lines reach
// memory instead of one 32-byte piece per lane and row.
template <int n_acc>
__device__ __forceinline__ void epilogue_swiglu_tma(const GemmParams& p, uint32_t tmem, int m0, int nt, int q,
                                                    int lane, int part, int nparts, uint8_t* stage_mem,
                                                    uint64_t* staged, volatile int* abort_flag, bool issuer) {
  constexpr int CW = 16, BOX = 128 * 64 * 2;  // one box: 16 KB
  const bool keep = p.aux_out != nullptr;
  const int boxes = keep ? 6 : 2;  // per accumulator
  const uint32_t sm = smem_u32(stage_mem);
  const int r = q * 32 + lane;
  auto put16 = [&](uint32_t row, uint32_t o0, uint32_t o1, const float (&x)[CW]) {
    st_shared_v4(row + o0, pack_bf16x2(x[0], x[1]), pack_bf16x2(x[2], x[3]), pack_bf16x2(x[4], x[5]),
                 pack_bf16x2(x[6], x[7]));
    st_shared_v4(row + o1, pack_bf16x2(x[8], x[9]), pack_bf16x2(x[10], x[11]), pack_bf16x2(x[12], x[13]),
                 pack_bf16x2(x[14], x[15]));
  };
  int item = 0;
  for (int a = 0; a < n_acc; ++a) {
    const uint32_t tb = tmem + ((uint32_t)(q * 32) << 16) + a * 256;
    for (int c = 0; c < 128 / CW; ++c) {
      if ((item++ % nparts) != part) continue;
      float v[CW], w[CW], o[CW];
      ld_acc16(tb + c * CW, v);
      ld_acc16(tb + 128 + c * CW, w);
#pragma unroll
      for (int i = 0; i < CW; ++i) {
        v[i] = round_bf16(v[i]);
        w[i] = round_bf16(w[i]);
        o[i] = silu_f(v[i]) * w[i];
      }
      const uint32_t row = sm + (uint32_t)(a * boxes + (c >> 2)) * BOX + (uint32_t)r * 128;
      const uint32_t o0 = (uint32_t)(((c & 3) * 2) ^ (r & 7)) << 4, o1 = (uint32_t)(((c & 3) * 2 + 1) ^ (r & 7)) << 4;
      put16(row, o0, o1, o);
      if (keep) {
        put16(row + 2 * BOX, o0, o1, v);
        put16(row + 4 * BOX, o0, o1, w);
      }
    }
  }
  fence_proxy_async_smem();  // the staged boxes are read by the TMA (async proxy)
  __syncwarp();
  if (lane == 0) mbar_arrive(staged);
  if (issuer && mbar_wait(staged, 0, abort_flag, p.err, KID_GEMM, 20) && !*abort_flag) {
    for (int a = 0; a < n_acc; ++a) {
      const int row0 = m0 + a * 128;
      if (row0 >= p.M) continue;
      const uint32_t b0 = sm + (uint32_t)(a * boxes) * BOX;
      for (int j = 0; j < 2; ++j) {
        tma_store_2d(&p.tmAux, b0 + j * BOX, nt * 128 + 64 * j, row0);
        if (keep) {
          tma_store_2d(&p.tmAux2, b0 + (2 + j) * BOX, nt * 128 + 64 * j, row0);
          tma_store_2d(&p.tmAux2, b0 + (4 + j) * BOX, p.inter + nt * 128 + 64 * j, row0);
        }
      }
    }
    tma_store_drain();  // the stores have read shared memory before the CTA exits
  }
}

// ------------------------------------------------------------------------------ kernel
template <bool DECODE, bool BMN>
__global__ void __launch_bounds__(DECODE ? 448 : 192, 1) k_gemm(const __grid_constant__ GemmParams p) {
  constexpr int NACC = 2;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* misc = base + STAGES * STAGE_BYTES;
  uint64_t* full = reinterpret_cast<uint64_t*>(misc);
  uint64_t* empty = full + STAGES;
  uint64_t* codes_full = empty + STAGES;
  uint64_t* accum_full = codes_full + STAGES;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(accum_full + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  float* code8_s = reinterpret_cast<float*>(misc + 256);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int mt = blockIdx.x % p.n_mt, nt = blockIdx.x / p.n_mt;
  const int m0 = mt * BM;
  const int total_kb = p.num_kb + p.has_extra;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], DECODE ? 1 + NUM_DECODERS : 1);
      mbar_init(&empty[s], 1);
      mbar_init(&codes_full[s], 1);
    }
    mbar_init(accum_full, 1);
    *abort_flag = 0;
    fence_barrier_init();
    fence_proxy_async_smem();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&p.tmA);
    if (p.has_extra) {
      tma_prefetch_desc(&p.tmAx);
      tma_prefetch_desc(&p.tmBx);
    }
    if (!DECODE) tma_prefetch_desc(&p.tmB);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  if (DECODE && warp >= 6)
    for (int i = threadIdx.x - 192; i < 256; i += NUM_DECODERS) code8_s[i] = p.code8[i];
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    // ---------------------------------------------------------------- TMA producer
    if (lane == 0) {
      for (int kb = 0; kb < total_kb; ++kb) {
        const int s = kb % STAGES;
        const uint32_t ph = (kb / STAGES) & 1;
        if (!mbar_wait(&empty[s], ph ^ 1, abort_flag, p.err, KID_GEMM, 1)) break;
        uint8_t* sA = base + s * STAGE_BYTES;
        uint8_t* sB = sA + A_BYTES;
        uint8_t* sC = sB + B_BYTES;
        if (kb < p.num_kb) {
          mbar_arrive_expect_tx(&full[s], A_BYTES + (DECODE ? 0 : B_BYTES));
          tma_load_2d(sA, &p.tmA, &full[s], kb * BK, m0);
          if (!DECODE) {
            if (BMN) {
              for (int j = 0; j < 4; ++j) tma_load_2d(sB + j * 8192, &p.tmB, &full[s], nt * BN + 64 * j, kb * BK);
            } else if (p.dense_swiglu_rows) {
              tma_load_2d(sB, &p.tmB, &full[s], kb * BK, nt * 128);
              tma_load_2d(sB + 16384, &p.tmB, &full[s], kb * BK, p.dense_swiglu_rows + nt * 128);
            } else {
              tma_load_2d(sB, &p.tmB, &full[s], kb * BK, nt * BN);
            }
          } else {
            // packed codes of this stage
            if (BMN) {
              const int row = kb * BK;
              const int sg = find_seg(p, row);
              mbar_arrive_expect_tx(&codes_full[s], C_BYTES);
              tma_load_2d(sC, &p.tmC[sg], &codes_full[s], nt * (BN / 2), row - p.seg_start[sg]);
            } else {
              int nbox = 0;
              int sg[4], lr[4];
              for (int rb = 0; rb < 4; ++rb) {
                if (p.swiglu) {
                  sg[rb] = rb >> 1;
                  lr[rb] = nt * 128 + 64 * (rb & 1);
                } else {
                  const int row = nt * BN + 64 * rb;
                  sg[rb] = row < p.N ? find_seg(p, row) : -1;
                  lr[rb] = row < p.N ? row - p.seg_start[sg[rb]] : 0;
                }
                if (sg[rb] >= 0) ++nbox;
              }
              if (nbox) {
                mbar_arrive_expect_tx(&codes_full[s], nbox * 2048);
                for (int rb = 0; rb < 4; ++rb)
                  if (sg[rb] >= 0) tma_load_2d(sC + rb * 2048, &p.tmC[sg[rb]], &codes_full[s], kb * (BK / 2), lr[rb]);
              } else {
                mbar_arrive(&codes_full[s]);
              }
            }
          }
        } else {
          // LoRA extra block: A from the extra activations, B from the padded adapter
          mbar_arrive_expect_tx(&full[s], A_BYTES + B_BYTES);
          tma_load_2d(sA, &p.tmAx, &full[s], 0, m0);
          if (BMN) {
            for (int j = 0; j < 4; ++j) tma_load_2d(sB + j * 8192, &p.tmBx, &full[s], nt * BN + 64 * j, 0);
          } else {
            tma_load_2d(sB, &p.tmBx, &full[s], 0, nt * BN);
          }
          if (DECODE) mbar_arrive(&codes_full[s]);
        }
      }
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------------- MMA issuer
    constexpr uint32_t idesc = idesc_bf16(128, BN, BMN);
    for (int kb = 0; kb < total_kb; ++kb) {
      const int s = kb % STAGES;
      const uint32_t ph = (kb / STAGES) & 1;
      if (!mbar_wait(&full[s], ph, abort_flag, p.err, KID_GEMM, 2)) break;
      tc_fence_after();
      if (lane == 0) {
        const uint32_t aA = smem_u32(base + s * STAGE_BYTES);
        const uint32_t aB = aA + A_BYTES;
#pragma unroll
        for (int ks = 0; ks < BK / 16; ++ks) {
          const uint64_t bdesc = BMN ? sdesc_sw128(aB + ks * 2048, 8192, 1024) : sdesc_sw128(aB + ks * 32, 16, 1024);
#pragma unroll
          for (int a = 0; a < 2; ++a) {
            const uint64_t adesc = sdesc_sw128(aA + a * 16384 + ks * 32, 16, 1024);
            umma_bf16(tmem + a * 256, adesc, bdesc, idesc, (kb | ks) != 0 ? 1u : 0u);
          }
        }
        umma_commit(&empty[s]);
      }
      __syncwarp();
    }
    if (lane == 0) umma_commit(accum_full);
    __syncwarp();
  } else if (warp < 6) {
    // ---------------------------------------------------------------- epilogue
    const int q = warp & 3;
    prefetch_aux(p, m0, nt, threadIdx.x - 64, 128);
    if (mbar_wait(accum_full, 0, abort_flag, p.err, KID_GEMM, 3)) {
      tc_fence_after();
      epilogue_rows<NACC, !DECODE>(p, tmem, m0, nt, q, lane, 0, DECODE ? 3 : 1);
    }
  } else if (DECODE) {
    // ---------------------------------------------------------------- NF4 decoders
    const int d = threadIdx.x - 192;  // 0..255
    float nf4[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) nf4[i] = p.nf4[i];
    // forward: one B row per thread, constant over the reduction
    int f_seg = 0, f_row = 0;
    bool f_valid = true;
    float f_off = 0.f;
    if (!BMN) {
      if (p.swiglu) {
        f_seg = d >> 7;
        f_row = nt * 128 + (d & 127);
      } else {
        const int row = nt * BN + d;
        f_valid = row < p.N;
        f_seg = f_valid ? find_seg(p, row) : 0;
        f_row = f_valid ? row - p.seg_start[f_seg] : 0;
      }
      f_off = *p.offset[f_seg];
    }
    const int rr = d & 63, jj = d >> 6;          // dL/dx: reduction row and column block
    const int dg_col = nt * BN + 64 * jj;         // first weight column of this thread's block
    const int blocks_per_row = p.seg_cols / 64;
    for (int kb = 0; kb < total_kb; ++kb) {
      const int s = kb % STAGES;
      const uint32_t ph = (kb / STAGES) & 1;
      // scale inputs are independent of the code tile: fetch them before waiting
      bool valid = false;
      int b = 0, sg = 0;
      uint32_t q8 = 0;
      float nested = 0.f, off = 0.f;
      if (kb < p.num_kb) {
        if (BMN) {
          const int row = kb * BK + rr;
          sg = find_seg(p, kb * BK);
          valid = dg_col < p.seg_cols;
          b = (row - p.seg_start[sg]) * blocks_per_row + (dg_col >> 6);
          if (valid) off = *p.offset[sg];
        } else {
          sg = f_seg;
          valid = f_valid;
          b = f_row * blocks_per_row + kb;
          off = f_off;
        }
        if (valid) {
          q8 = p.q8[sg][b];
          nested = p.nested[sg][b >> 8];
        }
      }
      if (!mbar_wait(&codes_full[s], ph, abort_flag, p.err, KID_GEMM, 4)) break;
      if (kb < p.num_kb) {
        const uint32_t sB = smem_u32(base + s * STAGE_BYTES + A_BYTES);
        const uint32_t sC = sB + B_BYTES;
        const uint32_t row_addr = BMN ? sB + jj * 8192 + rr * 128 : sB + d * 128;
        const int row_in_atom = (BMN ? rr : d) & 7;
        if (valid) {
          // code tiles arrive swizzled (128-byte rows for dL/dx, 32-byte rows forward),
          // so the 16-byte reads of eight neighbouring rows hit distinct banks
          uint32_t a0, a1;
          if (BMN) {
            a0 = sC + rr * 128 + ((uint32_t)((2 * jj) ^ (rr & 7)) << 4);
            a1 = sC + rr * 128 + ((uint32_t)((2 * jj + 1) ^ (rr & 7)) << 4);
          } else {
            const uint32_t flip = (uint32_t)((d >> 2) & 1) << 4;
            a0 = sC + d * 32 + flip;
            a1 = sC + d * 32 + (16u ^ flip);
          }
          const uint4 c0 = ld_shared_v4(a0), c1 = ld_shared_v4(a1);
          const uint32_t w[8] = {c0.x, c0.y, c0.z, c0.w, c1.x, c1.y, c1.z, c1.w};
          const float sc = __fadd_rn(__fmul_rn(code8_s[q8], nested), off);
          decode_block(row_addr, row_in_atom, w, sc, nf4);
        } else {
          zero_block(row_addr);
        }
        fence_proxy_async_smem();
      }
      mbar_arrive(&full[s]);
    }
    // then share the epilogue: 3 warps per TMEM lane quarter
    if (mbar_wait(accum_full, 0, abort_flag, p.err, KID_GEMM, 5)) {
      tc_fence_after();
      epilogue_rows<NACC, !DECODE>(p, tmem, m0, nt, warp & 3, lane, (warp - 2) / 4, 3);
    }
  }

  // On an aborted run the MMAs already issued must finish before TMEM is freed.
  if (warp == 1 && *abort_flag) mbar_wait_drain(accum_full, 0);
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// ------------------------------------------------------------------------------ CTA-pair kernel
// The same product with two CTAs per tile (a cluster of 2) and the 2-CTA tcgen05 MMA:
// the pair computes 512 tokens x 256 output features, CTA r holds tokens
// m0 + 256 r + [0, 256) (two 128-row accumulators, as above) and supplies B rows
// 128 r + [0, 128) of the 256-wide tile.  Each decoded weight still meets 256 tokens
// per MMA, but every SM now decodes (or loads) only half a B tile per stage, which
// halves the decode ALU work and the B-operand shared-memory traffic per SM.
// CTA 0 issues every MMA; both CTAs' operand loads and decoders arrive on CTA 0's
// stage barrier, and the MMA completion is multicast to both CTAs' barriers.
constexpr int P_STAGES = 4;
constexpr int PB_BYTES = 128 * BK * 2;  // 16 KB: this CTA's half of the B tile
constexpr int PC_BYTES = 4096;          // its packed codes
constexpr int P_STAGE_BYTES = A_BYTES + PB_BYTES + PC_BYTES;
constexpr int P_SMEM_BYTES = 1024 + P_STAGES * P_STAGE_BYTES + 256 + 1024;
// Two groups of 4 decoder warps per CTA take alternate k-blocks: each block row of
// a stage is one thread's work, and a thread has two stages' time to finish it.  (All
// 8 warps on every k-block, half a block row each, measured 10-25% slower.)
constexpr int P_DECODERS = 256;
constexpr int P_GROUP = 128;

template <bool DECODE, bool BMN, bool HALF>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(DECODE ? 448 : 192, 1)
    k_gemm_pair(const __grid_constant__ GemmParams p) {
  constexpr int NACC = HALF ? 1 : 2;  // 128-row accumulators per CTA (256- or 512-token pair tiles)
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* misc = base + P_STAGES * P_STAGE_BYTES;
  uint64_t* full = reinterpret_cast<uint64_t*>(misc);
  uint64_t* empty = full + P_STAGES;
  uint64_t* codes_full = empty + P_STAGES;
  uint64_t* accum_full = codes_full + P_STAGES;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(accum_full + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  uint64_t* aux_full = reinterpret_cast<uint64_t*>(misc + 112);  // 2: a side-input stage has landed
  uint64_t* aux_free = reinterpret_cast<uint64_t*>(misc + 128);  // the epilogue warps are done with it
  uint64_t* staged = reinterpret_cast<uint64_t*>(misc + 136);    // the epilogue warps' outputs are in place
  float* code8_s = reinterpret_cast<float*>(misc + 256);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const int tile = (blockIdx.x >> 1) + p.tile0;
  const int mt = tile % p.n_mt, nt = tile / p.n_mt;
  const int m0 = HALF ? mt * 256 + (int)rank * 128 : mt * 512 + (int)rank * 256;
  const int total_kb = p.num_kb + p.has_extra;

  if (threadIdx.x == 0) {
    for (int s = 0; s < P_STAGES; ++s) {
      mbar_init(&full[s], DECODE ? 1 + 2 * (P_GROUP / 32) : 1);
      mbar_init(&empty[s], 1);
      mbar_init(&codes_full[s], 1);
    }
    mbar_init(accum_full, 1);
    mbar_init(&aux_full[0], 1);
    mbar_init(&aux_full[1], 1);
    mbar_init(aux_free, DECODE ? 12 : 4);  // the epilogue warps
    mbar_init(staged, DECODE ? 12 : 4);
    *abort_flag = 0;
    fence_barrier_init();
    fence_proxy_async_smem();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&p.tmA);
    if (p.has_extra) {
      tma_prefetch_desc(&p.tmAx);
      tma_prefetch_desc(&p.tmBx);
    }
    if (!DECODE) tma_prefetch_desc(&p.tmB);
    if (p.aux_tma) tma_prefetch_desc(&p.tmAux);
    if (p.aux_tma >= 2) tma_prefetch_desc(&p.tmAux2);
  }
  if (warp == 1) {
    tmem_alloc_pair(tmem_slot, 512);
    tmem_relinquish_pair();
  }
  if (DECODE && warp >= 6)
    for (int i = threadIdx.x - 192; i < 256; i += P_DECODERS) code8_s[i] = p.code8[i];
  tc_fence_before();
  cluster_sync_all();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    // ---------------------------------------------------------------- TMA producer (both CTAs)
    if (lane == 0) {
      for (int kb = 0; kb < total_kb; ++kb) {
        const int s = kb % P_STAGES;
        const uint32_t ph = (kb / P_STAGES) & 1;
        if (!mbar_wait(&empty[s], ph ^ 1, abort_flag, p.err, KID_GEMM, 11)) break;
        const uint32_t lead = mapa_shared(smem_u32(&full[s]), 0);
        uint8_t* sA = base + s * P_STAGE_BYTES;
        uint8_t* sB = sA + A_BYTES;
        uint8_t* sC = sB + PB_BYTES;
        const int bcol = nt * BN + (int)rank * 128;  // this CTA's first B row (forward) or column (dL/dx)
        if (kb < p.num_kb) {
          if (rank == 0) mbar_arrive_expect_tx(&full[s], (HALF ? A_BYTES : 2 * A_BYTES) + (DECODE ? 0 : 2 * PB_BYTES));
          tma_load_2d_pair(sA, &p.tmA, lead, kb * BK, m0);
          if (!DECODE) {
            if (BMN) {
              for (int j = 0; j < 2; ++j) tma_load_2d_pair(sB + j * 8192, &p.tmB, lead, bcol + 64 * j, kb * BK);
            } else if (p.dense_swiglu_rows) {
              tma_load_2d_pair(sB, &p.tmB, lead, kb * BK, (int)rank * p.dense_swiglu_rows + nt * 128);
            } else {
              tma_load_2d_pair(sB, &p.tmB, lead, kb * BK, bcol);
            }
          } else if (BMN) {
            const int row = kb * BK;
            const int sg = find_seg(p, row);
            mbar_arrive_expect_tx(&codes_full[s], PC_BYTES);
            tma_load_2d(sC, &p.tmC[sg], &codes_full[s], bcol / 2, row - p.seg_start[sg]);
          } else {
            int nbox = 0, sg[2], lr[2];
            for (int rb = 0; rb < 2; ++rb) {
              if (p.swiglu) {
                sg[rb] = (int)rank;
                lr[rb] = nt * 128 + 64 * rb;
              } else {
                const int row = bcol + 64 * rb;
                sg[rb] = row < p.N ? find_seg(p, row) : -1;
                lr[rb] = row < p.N ? row - p.seg_start[sg[rb]] : 0;
              }
              if (sg[rb] >= 0) ++nbox;
            }
            if (nbox) {
              mbar_arrive_expect_tx(&codes_full[s], nbox * 2048);
              for (int rb = 0; rb < 2; ++rb)
                if (sg[rb] >= 0) tma_load_2d(sC + rb * 2048, &p.tmC[sg[rb]], &codes_full[s], kb * (BK / 2), lr[rb]);
            } else {
              mbar_arrive(&codes_full[s]);
            }
          }
        } else {
          if (rank == 0) mbar_arrive_expect_tx(&full[s], (HALF ? A_BYTES : 2 * A_BYTES) + 2 * PB_BYTES);
          tma_load_2d_pair(sA, &p.tmAx, lead, 0, m0);
          if (BMN) {
            for (int j = 0; j < 2; ++j) tma_load_2d_pair(sB + j * 8192, &p.tmBx, lead, bcol + 64 * j, 0);
          } else {
            tma_load_2d_pair(sB, &p.tmBx, lead, 0, bcol);
          }
          if (DECODE) mbar_arrive(&codes_full[s]);
        }
      }
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------------- MMA issuer (CTA 0)
    if (rank == 0) {
      constexpr uint32_t idesc = idesc_bf16(256, BN, BMN);
      for (int kb = 0; kb < total_kb; ++kb) {
        const int s = kb % P_STAGES;
        const uint32_t ph = (kb / P_STAGES) & 1;
        // Completes on both CTAs' A/B bytes and on the decoders of both CTAs, whose
        // tiles sit in their own CTA's shared memory behind fence.proxy.async and a
        // release arrive; the tensor core reads them after the fence below.
        if (!mbar_wait(&full[s], ph, abort_flag, p.err, KID_GEMM, 12)) break;
        tc_fence_after();
        if (lane == 0) {
          const uint32_t aA = smem_u32(base + s * P_STAGE_BYTES);
          const uint32_t aB = aA + A_BYTES;
#pragma unroll
          for (int ks = 0; ks < BK / 16; ++ks) {
            const uint64_t bdesc =
                BMN ? sdesc_sw128(aB + ks * 2048, 8192, 1024) : sdesc_sw128(aB + ks * 32, 16, 1024);
#pragma unroll
            for (int a = 0; a < 2; ++a) {
              if (a >= NACC) break;
              const uint64_t adesc = sdesc_sw128(aA + a * 16384 + ks * 32, 16, 1024);
              umma_bf16_pair(tmem + a * 256, adesc, bdesc, idesc, (kb | ks) != 0 ? 1u : 0u);
            }
          }
          umma_commit_pair(&empty[s]);
        }
        __syncwarp();
      }
      if (lane == 0) umma_commit_pair(accum_full);
      __syncwarp();
    }
  } else if (warp < 6) {
    // ---------------------------------------------------------------- epilogue (both CTAs)
    const int q = warp & 3;
    prefetch_aux(p, m0, nt, threadIdx.x - 64, 128, 128 * NACC);
    if (mbar_wait(accum_full, 0, abort_flag, p.err, KID_GEMM, 13)) {
      tc_fence_after();
      if (p.aux_tma == 1)
        epilogue_side_tma<NACC>(p, tmem, m0, nt, q, lane, 0, DECODE ? 3 : 1, base, aux_full, aux_free, abort_flag,
                                   threadIdx.x == 64);
      else if (p.aux_tma == 2)
        epilogue_rope_tma<NACC>(p, tmem, m0, nt, q, lane, 0, DECODE ? 3 : 1, base, aux_full, aux_free, abort_flag,
                                threadIdx.x == 64);
      else if (p.aux_tma == 3)
        epilogue_swiglu_tma<NACC>(p, tmem, m0, nt, q, lane, 0, DECODE ? 3 : 1, base, staged, abort_flag,
                                  threadIdx.x == 64);
      else
        epilogue_rows<NACC, !DECODE>(p, tmem, m0, nt, q, lane, 0, DECODE ? 3 : 1);
    }
  } else if (DECODE) {
    // ---------------------------------------------------------------- NF4 decoders (both CTAs)
    const int grp = (threadIdx.x - 192) / P_GROUP;  // which k-blocks: kb = grp, grp + 2, ...
    const int d = (threadIdx.x - 192) % P_GROUP;    // 0..127
    float nf4[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) nf4[i] = p.nf4[i];
    const int bcol = nt * BN + (int)rank * 128;
    int f_seg = 0, f_row = 0;
    bool f_valid = true;
    float f_off = 0.f;
    if (!BMN) {
      if (p.swiglu) {
        f_seg = (int)rank;
        f_row = nt * 128 + d;
      } else {
        const int row = bcol + d;
        f_valid = row < p.N;
        f_seg = f_valid ? find_seg(p, row) : 0;
        f_row = f_valid ? row - p.seg_start[f_seg] : 0;
      }
      f_off = *p.offset[f_seg];
    }
    const int rr = d & 63, jj = d >> 6;
    const int dg_col = bcol + 64 * jj;
    const int blocks_per_row = p.seg_cols / 64;
    for (int kb = grp; kb < total_kb; kb += 2) {
      const int s = kb % P_STAGES;
      const uint32_t ph = (kb / P_STAGES) & 1;
      bool valid = false;
      int b = 0, sg = 0;
      uint32_t q8 = 0;
      float nested = 0.f, off = 0.f;
      if (kb < p.num_kb) {
        if (BMN) {
          const int row = kb * BK + rr;
          sg = find_seg(p, kb * BK);
          valid = dg_col < p.seg_cols;
          b = (row - p.seg_start[sg]) * blocks_per_row + (dg_col >> 6);
          if (valid) off = *p.offset[sg];
        } else {
          sg = f_seg;
          valid = f_valid;
          b = f_row * blocks_per_row + kb;
          off = f_off;
        }
        if (valid) {
          q8 = p.q8[sg][b];
          nested = p.nested[sg][b >> 8];
        }
      }
      if (!mbar_wait(&codes_full[s], ph, abort_flag, p.err, KID_GEMM, 14)) break;
      if (kb < p.num_kb) {
        const uint32_t sB = smem_u32(base + s * P_STAGE_BYTES + A_BYTES);
        const uint32_t sC = sB + PB_BYTES;
        const uint32_t row_addr = BMN ? sB + jj * 8192 + rr * 128 : sB + d * 128;
        const int row_in_atom = (BMN ? rr : d) & 7;
        if (valid) {
          // swizzled code tiles: 64-byte rows (dL/dx) or 32-byte rows (forward)
          uint32_t a0, a1;
          if (BMN) {
            const int x = (rr >> 1) & 3;
            a0 = sC + rr * 64 + ((uint32_t)((2 * jj) ^ x) << 4);
            a1 = sC + rr * 64 + ((uint32_t)((2 * jj + 1) ^ x) << 4);
          } else {
            const uint32_t flip = (uint32_t)((d >> 2) & 1) << 4;
            a0 = sC + d * 32 + flip;
            a1 = sC + d * 32 + (16u ^ flip);
          }
          const uint4 c0 = ld_shared_v4(a0), c1 = ld_shared_v4(a1);
          const uint32_t w[8] = {c0.x, c0.y, c0.z, c0.w, c1.x, c1.y, c1.z, c1.w};
          const float sc = __fadd_rn(__fmul_rn(code8_s[q8], nested), off);
          decode_block(row_addr, row_in_atom, w, sc, nf4);
        } else {
          zero_block(row_addr);
        }
        fence_proxy_async_smem();
      }
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(mapa_shared(smem_u32(&full[s]), 0));
    }
    // then share the epilogue: 3 warps per TMEM lane quarter
    if (mbar_wait(accum_full, 0, abort_flag, p.err, KID_GEMM, 15)) {
      tc_fence_after();
      if (p.aux_tma == 1)
        epilogue_side_tma<NACC>(p, tmem, m0, nt, warp & 3, lane, (warp - 2) / 4, 3, base, aux_full, aux_free,
                                   abort_flag, false);
      else if (p.aux_tma == 2)
        epilogue_rope_tma<NACC>(p, tmem, m0, nt, warp & 3, lane, (warp - 2) / 4, 3, base, aux_full, aux_free,
                                abort_flag, false);
      else if (p.aux_tma == 3)
        epilogue_swiglu_tma<NACC>(p, tmem, m0, nt, warp & 3, lane, (warp - 2) / 4, 3, base, staged, abort_flag,
                                  false);
      else
        epilogue_rows<NACC, !DECODE>(p, tmem, m0, nt, warp & 3, lane, (warp - 2) / 4, 3);
    }
  }

  if (rank == 0 && warp == 1 && *abort_flag) mbar_wait_drain(accum_full, 0);
  tc_fence_before();
  cluster_sync_all();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tmem, 512);
  }
}

// ------------------------------------------------------------------------------ host side
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(f);
  });
  return fn;
}

int make_map(CUtensorMap* map, CUtensorMapDataType dt, int esize, const void* ptr, uint64_t inner, uint64_t outer,
             uint64_t row_bytes, uint32_t box_inner, uint32_t box_outer, CUtensorMapSwizzle swz) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return fail(NF4LS_CUDA, "cuTensorMapEncodeTiled is unavailable");
  if (!aligned(ptr, 16) || row_bytes % 16) return fail(NF4LS_ALIGN, "TMA operand base/row stride not 16-byte aligned");
  const cuuint64_t dims[2] = {inner, outer};
  const cuuint64_t strides[1] = {row_bytes};
  const cuuint32_t box[2] = {box_inner, box_outer};
  const cuuint32_t es[2] = {1, 1};
  (void)esize;
  const CUresult r = fn(map, dt, 2, const_cast<void*>(ptr), dims, strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE,
                        swz,
                        CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(NF4LS_CUDA, "cuTensorMapEncodeTiled failed (%d)", (int)r);
  return NF4LS_OK;
}

template <bool DECODE, bool BMN>
int launch(const GemmParams& p, int grid, cudaStream_t s) {
  static int configured[16] = {0};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 16 && !configured[dev]) {
    NF4_CUDA_TRY(cudaFuncSetAttribute(k_gemm<DECODE, BMN>, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_BYTES));
    configured[dev] = 1;
  }
  k_gemm<DECODE, BMN><<<grid, DECODE ? 448 : 192, SMEM_BYTES, s>>>(p);
  note_launch();
  NF4_CUDA_TRY(cudaGetLastError());
  return NF4LS_OK;
}

// CTA pairs that can be resident at once (the width of one wave).
template <bool DECODE, bool BMN>
int pair_slots() {
  static int cached[16] = {0};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 16 && cached[dev]) return cached[dev];
  int n = 0;
  if (cudaFuncSetAttribute(k_gemm_pair<DECODE, BMN, false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           P_SMEM_BYTES) == cudaSuccess) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(2 * 1024);
    cfg.blockDim = dim3(DECODE ? 448 : 192);
    cfg.dynamicSmemBytes = P_SMEM_BYTES;
    if (cudaOccupancyMaxActiveClusters(&n, (const void*)k_gemm_pair<DECODE, BMN, false>, &cfg) != cudaSuccess) n = 0;
  }
  cudaGetLastError();
  if (n <= 0) {
    int sms = 148;
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    n = sms / 2;
  }
  if (dev < 16) cached[dev] = n;
  return n;
}

template <bool DECODE, bool BMN, bool HALF>
int launch_pair_t(const GemmParams& p, int grid, cudaStream_t s) {
  static int configured[16] = {0};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 16 && !configured[dev]) {
    NF4_CUDA_TRY(cudaFuncSetAttribute(k_gemm_pair<DECODE, BMN, HALF>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                      P_SMEM_BYTES));
    configured[dev] = 1;
  }
  k_gemm_pair<DECODE, BMN, HALF><<<grid, DECODE ? 448 : 192, P_SMEM_BYTES, s>>>(p);
  note_launch();
  NF4_CUDA_TRY(cudaGetLastError());
  return NF4LS_OK;
}

template <bool DECODE, bool BMN>
int launch_pair(const GemmParams& p, int grid, cudaStream_t s) {
  return p.half ? launch_pair_t<DECODE, BMN, true>(p, grid, s) : launch_pair_t<DECODE, BMN, false>(p, grid, s);
}

}  // namespace

int tma_map_bf16(CUtensorMap* map, const void* ptr, uint64_t cols, uint64_t rows, uint64_t row_bytes,
                 uint32_t box_cols, uint32_t box_rows) {
  return make_map(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, ptr, cols, rows, row_bytes, box_cols, box_rows,
                  CU_TENSOR_MAP_SWIZZLE_128B);
}

int gemm(const __nv_bfloat16* A, int lda, int M, int N, int K, const GemmWeights& W, bool dgrad,
         const GemmExtra& extra, const GemmEpilogue& epi, cudaStream_t s) {
  if (!A || (epi.kind == EPI_ACC_F32 ? !epi.out_f32 || (epi.accumulate && !epi.alpha) : !epi.out))
    return fail(NF4LS_INVALID_ARG, "gemm: null operand");
  if (M <= 0 || N <= 0 || K <= 0 || K % 64 || N % 64) return fail(NF4LS_SHAPE, "gemm: M=%d N=%d K=%d (K, N % 64)", M, N, K);
  const bool decode = W.dense == nullptr;
  const bool swiglu = epi.kind == EPI_SWIGLU;
  if (decode && (W.n_seg < 1 || W.n_seg > 4)) return fail(NF4LS_INVALID_ARG, "gemm: 1-4 weight segments");
  if (swiglu && (dgrad || epi.inter <= 0 || epi.inter % 128 || N != 2 * epi.inter))
    return fail(NF4LS_SHAPE, "gemm: SwiGLU epilogue needs N = 2*I with I % 128 == 0");
  if (epi.kind == EPI_ACC_F32 && decode) return fail(NF4LS_INVALID_ARG, "gemm: the fp32 epilogue takes dense weights");
  if (epi.kind == EPI_ROPE && (epi.head_dim <= 0 || BN % epi.head_dim || epi.seq <= 0))
    return fail(NF4LS_SHAPE, "gemm: RoPE epilogue head_dim");
  static_assert(sizeof(GemmParams) <= 4096, "kernel parameters exceed 4 KB");

  GemmParams p;
  std::memset(&p, 0, sizeof(p));
  p.M = M;
  p.N = N;
  p.K = K;
  p.num_kb = K / 64;
  p.has_extra = extra.a != nullptr;
  // CTA pairs for every product with more than one 256-token tile; single CTAs below.
  const bool pair = gemm_pair() && M > BM;
  const uint32_t bbox = pair ? 128 : 256;  // B rows one CTA loads (forward, K-major)
  const int n_nt = swiglu ? epi.inter / 128 : (N + BN - 1) / BN;
  // Pair tiles of 512 tokens (two 128-row accumulators per CTA), or of 256 when that
  // takes fewer tile-times.  A 256-token tile decodes each weight for half as many
  // tokens, so it runs 0.78 as long as a 512-token one (measured on the 8B products at
  // full waves): it pays off when the 512-token tiles leave most pairs idle, e.g. the
  // 16-48 tiles of a 512-token batch.  Or, on request only (mode 3), split: the whole
  // waves of 512-token tiles in one launch and the tiles of the last, partial wave as
  // twice as many 256-token tiles in a second launch.  Measured on the 8B products of
  // a 2048-token batch, whose last waves hold 22, 2 and 4 of 74 tiles (q/k/v forward,
  // down dL/dx, gate/up forward), it changed them by -1%, -3% and +1%: a partial last
  // wave of 512-token tiles already runs faster than a full one, so the automatic
  // choice leaves it out.  All three schedules reduce every output in the same order.
  p.half = 0;
  int split_full = 0;  // tiles of the 512-token launch when the tail is split off
  const int t_full = (M + 511) / 512 * n_nt, t_half = (M + 255) / 256 * n_nt;
  // the split needs every 512-token tile to be exactly two 256-token tiles
  const bool can_split = pair && (M + 255) / 256 == 2 * ((M + 511) / 512);
  if (pair) {
    const int mode = gemm_half_mode();
    const int P = decode ? (dgrad ? pair_slots<true, true>() : pair_slots<true, false>())
                         : (dgrad ? pair_slots<false, true>() : pair_slots<false, false>());
    const int waves = t_full / P;
    if (mode == 2) {
      p.half = 1;
    } else if (mode == 3 && can_split) {
      split_full = waves * P;
    } else if (mode == 0) {
      const double w_full = (double)((t_full + P - 1) / P), w_half = 0.8 * ((t_half + P - 1) / P);
      p.half = w_half < w_full ? 1 : 0;
    }
  }
  const bool split = pair && gemm_half_mode() == 3 && can_split;
  p.n_mt = pair ? (p.half ? (M + 255) / 256 : (M + 511) / 512) : (M + BM - 1) / BM;
  // A rows one CTA loads: 128 for 256-token pair tiles, else 256
  auto map_a = [&](bool half_rows) -> int {
    const uint32_t abox = pair && half_rows ? 128 : 256;
    NF4_TRY(make_map(&p.tmA, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, A, K, M, (uint64_t)lda * 2, 64, abox,
                     CU_TENSOR_MAP_SWIZZLE_128B));
    if (p.has_extra)
      NF4_TRY(make_map(&p.tmAx, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, extra.a, 64, M, 128, 64, abox,
                       CU_TENSOR_MAP_SWIZZLE_128B));
    return NF4LS_OK;
  };
  if (p.has_extra && !extra.b) return fail(NF4LS_INVALID_ARG, "gemm: extra block needs both operands");
  NF4_TRY(map_a(p.half != 0));
  if (p.has_extra) {
    if (dgrad)
      NF4_TRY(make_map(&p.tmBx, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, extra.b, N, 64, (uint64_t)N * 2, 64, 64, CU_TENSOR_MAP_SWIZZLE_128B));
    else
      NF4_TRY(make_map(&p.tmBx, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, extra.b, 64, N, 128, 64, bbox, CU_TENSOR_MAP_SWIZZLE_128B));
  }
  if (!decode) {
    if (dgrad)  // W [K, N]
      NF4_TRY(make_map(&p.tmB, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, W.dense, N, K, (uint64_t)N * 2, 64, 64, CU_TENSOR_MAP_SWIZZLE_128B));
    else if (swiglu) {  // W [2I, K]: gate rows then up rows
      NF4_TRY(make_map(&p.tmB, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, W.dense, K, N, (uint64_t)K * 2, 64, 128, CU_TENSOR_MAP_SWIZZLE_128B));
      p.dense_swiglu_rows = epi.inter;
    } else
      NF4_TRY(make_map(&p.tmB, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, W.dense, K, N, (uint64_t)K * 2, 64, bbox, CU_TENSOR_MAP_SWIZZLE_128B));
  } else {
    p.n_seg = W.n_seg;
    p.swiglu = swiglu;
    int start = 0;
    const int cols = W.seg[0].cols;
    for (int i = 0; i < W.n_seg; ++i) {
      const NF4Tensor& t = W.seg[i];
      if (t.cols != cols || t.rows % 64) return fail(NF4LS_SHAPE, "gemm: segment %d shape", i);
      p.seg_start[i] = start;
      start += t.rows;
      p.q8[i] = t.q8;
      p.nested[i] = t.nested;
      p.offset[i] = t.offset;
      if (dgrad && pair)  // codes [rows, N/2] bytes; box 64 B x 64 rows (one CTA's 128 columns)
        NF4_TRY(make_map(&p.tmC[i], CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, t.packed, cols / 2, t.rows, cols / 2, 64, 64,
                         CU_TENSOR_MAP_SWIZZLE_64B));
      else if (dgrad)  // codes [rows, N/2] bytes; box 128 B x 64 rows
        NF4_TRY(make_map(&p.tmC[i], CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, t.packed, cols / 2, t.rows, cols / 2, 128, 64,
                                 CU_TENSOR_MAP_SWIZZLE_128B));
      else  // codes [rows, K/2] bytes; box 32 B x 64 rows
        NF4_TRY(make_map(&p.tmC[i], CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, t.packed, cols / 2, t.rows, cols / 2, 32, 64,
                                 CU_TENSOR_MAP_SWIZZLE_32B));
    }
    p.seg_start[W.n_seg] = start;
    p.seg_cols = cols;
    if (dgrad && (start != K || cols != N)) return fail(NF4LS_SHAPE, "gemm: dL/dx segments do not match K x N");
    if (!dgrad && (start != N || cols != K)) return fail(NF4LS_SHAPE, "gemm: forward segments do not match N x K");
    if (swiglu && (W.n_seg != 2 || W.seg[0].rows != epi.inter || W.seg[1].rows != epi.inter))
      return fail(NF4LS_SHAPE, "gemm: SwiGLU needs gate and up segments of I rows");
    const Codebooks& cb = codebooks();
    std::memcpy(p.nf4, cb.nf4, sizeof(p.nf4));
    std::memcpy(p.code8, cb.code8, sizeof(p.code8));
  }
  p.epi = epi.kind;
  p.out = epi.out;
  p.ldo = epi.ldo;
  p.aux0 = epi.aux0;
  p.ld_aux0 = epi.ld_aux0;
  p.aux_out = epi.aux_out;
  p.ld_aux_out = epi.ld_aux_out;
  p.inter = epi.inter;
  p.rope_cos = epi.rope_cos;
  p.rope_sin = epi.rope_sin;
  p.seq = epi.seq;
  p.head_dim = epi.head_dim;
  p.rope_cols = epi.rope_cols;
  p.out_f32 = epi.out_f32;
  p.alpha = epi.alpha;
  p.accumulate = epi.accumulate;
  // CTA pairs: the residual x or the dSwiGLU side input [g | u] by TMA (16-byte rows and
  // column offsets)
  p.aux_tma = 0;
  const bool dsw = epi.kind == EPI_DSWIGLU;
  const int64_t side_cols = dsw ? (int64_t)2 * epi.inter : N;
  if (pair && (dsw || epi.kind == EPI_RESID) && epi.aux0 && aligned(epi.aux0, 16) && epi.ld_aux0 % 8 == 0 &&
      (!dsw || epi.inter % 8 == 0) && epi.ld_aux0 >= side_cols) {
    NF4_TRY(make_map(&p.tmAux, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, epi.aux0, (uint64_t)side_cols, M,
                     (uint64_t)epi.ld_aux0 * 2, 64, 128, CU_TENSOR_MAP_SWIZZLE_128B));
    p.aux_tma = 1;
  }
  // CTA pairs, RoPE: the angle tables [d/2, seq] by TMA, 128 positions per box (an
  // accumulator's rows are 128 consecutive positions when seq is a multiple of 128)
  if (pair && epi.kind == EPI_ROPE && epi.seq % 128 == 0 && epi.head_dim % 32 == 0 && aligned(epi.rope_cos, 16) &&
      aligned(epi.rope_sin, 16)) {
    const int half = epi.head_dim / 2;
    NF4_TRY(make_map(&p.tmAux, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, epi.rope_cos, epi.seq, half, (uint64_t)epi.seq * 4,
                     128, half, CU_TENSOR_MAP_SWIZZLE_NONE));
    NF4_TRY(make_map(&p.tmAux2, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, epi.rope_sin, epi.seq, half, (uint64_t)epi.seq * 4,
                     128, half, CU_TENSOR_MAP_SWIZZLE_NONE));
    p.aux_tma = 2;
  }
  // CTA pairs, SwiGLU with g and u kept (three outputs): act, g and u through staged
  // boxes and TMA stores (measured: 432 -> 409 us on the 8B gate/up product at M = 2048;
  // with act alone the per-lane stores were as fast)
  if (pair && swiglu && epi.aux_out && aligned(epi.out, 16) && epi.ldo % 8 == 0 && epi.ldo >= epi.inter &&
      aligned(epi.aux_out, 16) && epi.ld_aux_out % 8 == 0 && epi.ld_aux_out >= 2 * epi.inter) {
    NF4_TRY(make_map(&p.tmAux, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, epi.out, epi.inter, M, (uint64_t)epi.ldo * 2, 64,
                     128, CU_TENSOR_MAP_SWIZZLE_128B));
    NF4_TRY(make_map(&p.tmAux2, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, epi.aux_out, (uint64_t)2 * epi.inter, M,
                     (uint64_t)epi.ld_aux_out * 2, 64, 128, CU_TENSOR_MAP_SWIZZLE_128B));
    p.aux_tma = 3;
  }
  if (epi.kind == EPI_ACC_F32 && (epi.ldo % 4 || !aligned(epi.out_f32, 16)))
    return fail(NF4LS_ALIGN, "gemm: fp32 output needs 16-byte rows");
  p.err = device_error_ptr();
  p.tile0 = 0;
  const int grid = p.n_mt * n_nt * (pair ? 2 : 1);
  cudaEvent_t e0 = nullptr;
  if (profiling()) profile_begin(s, &e0);
  auto run_pair = [&](int pairs) {
    if (decode)
      return dgrad ? launch_pair<true, true>(p, 2 * pairs, s) : launch_pair<true, false>(p, 2 * pairs, s);
    return dgrad ? launch_pair<false, true>(p, 2 * pairs, s) : launch_pair<false, false>(p, 2 * pairs, s);
  };
  int st;
  if (split) {
    // 512-token tiles [0, split_full), then 256-token tiles [2 split_full, 2 t_full):
    // with mt fastest, 512-token tile t is 256-token tiles 2t and 2t + 1.
    st = split_full > 0 ? run_pair(split_full) : NF4LS_OK;
    if (st == NF4LS_OK) {
      p.half = 1;
      p.n_mt = (M + 255) / 256;
      p.tile0 = 2 * split_full;
      st = map_a(true);
      if (st == NF4LS_OK) st = run_pair(t_half - 2 * split_full);
    }
  } else if (pair) {
    st = run_pair(grid / 2);
  } else if (decode) {
    st = dgrad ? launch<true, true>(p, grid, s) : launch<true, false>(p, grid, s);
  } else {
    st = dgrad ? launch<false, true>(p, grid, s) : launch<false, false>(p, grid, s);
  }
  // algorithmic work: 2 M N K, plus the 64-wide LoRA block when present
  // kind 0/1 (dense / NF4 decode); detail 1000 + 100 decode + 10 dL/dx + epilogue
  if (e0)
    profile_end(s, e0, decode ? 1 : 0, 1000 + (decode ? 100 : 0) + (dgrad ? 10 : 0) + epi.kind,
                2.0 * M * (double)N * (K + (p.has_extra ? 64 : 0)));
  return st;
}

}  // namespace nf4ls

extern "C" int nf4ls_gemm_bf16(const void* A_dev, const void* B_dev, void* out_dev, int M, int N, int K, int b_trans,
                               int ldo, nf4ls_stream stream) {
  nf4ls::clear_error();
  nf4ls::GemmWeights W;
  W.dense = static_cast<const __nv_bfloat16*>(B_dev);
  if (!W.dense) return nf4ls::fail(NF4LS_INVALID_ARG, "nf4ls_gemm_bf16: null B");
  nf4ls::GemmEpilogue e;
  e.out = static_cast<__nv_bfloat16*>(out_dev);
  e.ldo = ldo;
  return nf4ls::gemm(static_cast<const __nv_bfloat16*>(A_dev), K, M, N, K, W, b_trans != 0, nf4ls::GemmExtra(), e,
                     static_cast<cudaStream_t>(stream));
}

extern "C" int nf4ls_gemm_nf4(const void* A_dev, int lda, int M, const uint8_t* packed_dev, const uint8_t* q8_dev,
                              const float* nested_dev, const float* offset_dev, int rows, int cols, int dgrad,
                              void* out_dev, int ldo, nf4ls_stream stream) {
  nf4ls::clear_error();
  nf4ls::GemmWeights W;
  W.n_seg = 1;
  W.seg[0] = nf4ls::NF4Tensor{packed_dev, q8_dev, nested_dev, offset_dev, rows, cols};
  nf4ls::GemmEpilogue e;
  e.out = static_cast<__nv_bfloat16*>(out_dev);
  e.ldo = ldo;
  const int N = dgrad ? cols : rows, K = dgrad ? rows : cols;
  return nf4ls::gemm(static_cast<const __nv_bfloat16*>(A_dev), lda, M, N, K, W, dgrad != 0, nf4ls::GemmExtra(), e,
                     static_cast<cudaStream_t>(stream));
}
