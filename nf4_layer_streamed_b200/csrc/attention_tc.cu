// K10 forward on the 5th-generation tensor cores: causal grouped-query attention
// softmax(q k^T / sqrt(d) + causal mask) v for head_dim 64 or 128 (a template parameter)
// and seq a multiple of 128 (up to 8192): the shapes of the SmolLM2-shaped, Llama-8B and
// 32B-class layers
// ("Soup 层流式 NF4 训练实测：在 4 GB 显存上以位级一致标准完成 8B 模型 LoRA 微调"
// §2.1: the HF Llama layer body; the workloads' seq 512).
//
// One CTA per (128-query tile, query head, sequence; the query tile is the grid's slowest
// dimension, longest rows first), two CTAs per SM: 96 KB of shared
// memory (the Q tile and one K and one V tile, a 32 KB slot each, the first half of which
// a head_dim-64 tile uses) and 256 TMEM columns each, so that one
// CTA's softmax runs while the other's products keep the tensor core busy.  Per key
// tile kt = 0 .. qt (online softmax, one query row per thread of four warps):
//   1. S = Q K_kt^T (tcgen05.mma, M = N = 128, K = 16 steps) into TMEM columns [0, 128).
//   2. The row maximum of the tile (causal mask on the diagonal tile).  The reference
//      maximum m of a row moves only when the tile's maximum exceeds it by more than
//      2^8 (in exp2 units); then the running O row and sum are scaled by 2^(m - m_new)
//      first.  p = 2^(s log2e / sqrt(d) - m), summed in fp32, is written back as bf16
//      over the scores it came from (two per 32-bit column).
//   3. O += P V_kt with P read from TMEM as the A operand and V N-major from shared
//      memory, accumulating in TMEM columns [128, 256).
// The next K tile loads while the softmax runs, the next V tile after the product that
// reads the current one.  The output is O / sum in bf16 and the log-sum-exp
// (m + log2 sum) ln 2.  P is rounded to bf16 for the P V product, as in the mma.sync
// kernel; the results match that kernel up to rounding.  Every mbarrier wait is bounded.
#include "common.cuh"
#include "internal.h"

namespace nf4ls {

namespace {

constexpr int TT = 128;                   // query / key tile
constexpr int TILE_BYTES = TT * 128 * 2;  // 128 rows x 128 dims bf16 = 32 KB
constexpr int ATOM = TILE_BYTES / 2;      // one 64-dim (or 64-key) swizzle atom: 16 KB

// One thread's 32 fp32 values (columns 32 c .. 32 c + 31 of its row r of a 128 x 128 tile),
// times sc, as bf16 into the tile's two 128-byte swizzled 64-column atoms at tile.
__device__ __forceinline__ void stage_row32(uint32_t tile, int r, int c, const uint32_t (&v)[32], float sc) {
  const uint32_t row = tile + (uint32_t)(c >> 1) * (TT * 128) + (uint32_t)r * 128;
#pragma unroll
  for (int q4 = 0; q4 < 4; ++q4) {
    const int chunk = (c & 1) * 4 + q4;  // 16-byte chunk of the 128-byte row
    st_shared_v4(row + ((uint32_t)(chunk ^ (r & 7)) << 4),
                 pack_bf16x2(__uint_as_float(v[8 * q4]) * sc, __uint_as_float(v[8 * q4 + 1]) * sc),
                 pack_bf16x2(__uint_as_float(v[8 * q4 + 2]) * sc, __uint_as_float(v[8 * q4 + 3]) * sc),
                 pack_bf16x2(__uint_as_float(v[8 * q4 + 4]) * sc, __uint_as_float(v[8 * q4 + 5]) * sc),
                 pack_bf16x2(__uint_as_float(v[8 * q4 + 6]) * sc, __uint_as_float(v[8 * q4 + 7]) * sc));
  }
}

__device__ __forceinline__ void stage_row32(uint32_t tile, int r, int c, const float (&v)[32]) {
  uint32_t u[32];
#pragma unroll
  for (int i = 0; i < 32; ++i) u[i] = __float_as_uint(v[i]);
  stage_row32(tile, r, c, u, 1.0f);
}

struct AttnTcParams {
  CUtensorMap tq, tk, tv, to;  // [rows, cols] bf16, box 64 cols x 128 rows, 128-byte swizzle (to: output)
  __nv_bfloat16* o;
  float* lse;
  int ldo, seq, nq, nkv;
  float scale_log2;
  int* err;
};

// warps 0-3: softmax and epilogue (warp w owns TMEM lanes 32 w .. 32 w + 31, one query
// row per thread); warp 4: TMA producer; warp 5: MMA issuer
constexpr int F_THREADS = 192, F_PROD = 4, F_MMA = 5;
constexpr int F_OFF_Q = 0, F_OFF_K = TILE_BYTES, F_OFF_V = 2 * TILE_BYTES, F_OFF_BAR = 3 * TILE_BYTES;
constexpr int SMEM_TC = 1024 + F_OFF_BAR + 128;
constexpr float kRescaleLog2 = 8.0f;  // the reference maximum may trail the true one by this much

__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], "
      "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
      "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]),
      "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15]), "r"(r[16]),
      "r"(r[17]), "r"(r[18]), "r"(r[19]), "r"(r[20]), "r"(r[21]), "r"(r[22]), "r"(r[23]), "r"(r[24]),
      "r"(r[25]), "r"(r[26]), "r"(r[27]), "r"(r[28]), "r"(r[29]), "r"(r[30]), "r"(r[31])
      : "memory");
}

__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
      "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]),
      "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15])
      : "memory");
}
__device__ __forceinline__ void tmem_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }
__device__ __forceinline__ void tmem_st_cols(uint32_t taddr, const uint32_t (&r)[32]) { tmem_st32(taddr, r); }
__device__ __forceinline__ void tmem_st_cols(uint32_t taddr, const uint32_t (&r)[16]) { tmem_st16(taddr, r); }

// 2^x by the hardware approximation (ex2.approx, flush-to-zero): its relative error is
// far below the bf16 rounding that every probability gets next.
__device__ __forceinline__ float fast_exp2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// D[tmem] (+)= A[tmem] * B[smem desc]: A of M = 128 lanes x 16 bf16 (8 columns).
__device__ __forceinline__ void umma_bf16_ta(uint32_t d_tmem, uint32_t a_tmem, uint64_t bdesc, uint32_t idesc,
                                             uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}

template <int D>
__global__ void __launch_bounds__(F_THREADS, 2) k_attn_fwd_tc(const __grid_constant__ AttnTcParams p) {
  constexpr int NA = D / 64, KS = D / 16, TB = NA * ATOM;  // swizzle atoms, k-steps and bytes of a tile
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(base + F_OFF_BAR);
  uint64_t* q_full = bars;
  uint64_t* k_full = bars + 1;
  uint64_t* k_empty = bars + 2;
  uint64_t* v_full = bars + 3;
  uint64_t* v_empty = bars + 4;
  uint64_t* s_full = bars + 5;
  uint64_t* p_full = bars + 6;
  uint64_t* o_full = bars + 7;   // one phase per key tile: the P V product of that tile is done
  uint64_t* drain = bars + 8;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 9);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // z slowest: every head's longest query rows first, then the next tile height, so the
  // shortest CTAs fill the last wave
  const int qt = gridDim.z - 1 - blockIdx.z;
  const int h = blockIdx.x, b = blockIdx.y;
  const int kvh = h / (p.nq / p.nkv);
  const int nk = qt + 1;                      // key tiles at or before the diagonal
  const int row0 = b * p.seq;

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    mbar_init(k_full, 1);
    mbar_init(k_empty, 1);
    mbar_init(v_full, 1);
    mbar_init(v_empty, 1);
    mbar_init(s_full, 1);
    mbar_init(p_full, 4);
    mbar_init(o_full, 1);
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == F_MMA) {
    tmem_alloc(tmem_slot, 256);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;  // [0, 128) S then P, [128, 256) O

  if (warp == F_PROD) {
    // ------------------------------------------------------------------ TMA producer
    if (lane == 0) {
      tma_prefetch_desc(&p.tq);
      tma_prefetch_desc(&p.tk);
      tma_prefetch_desc(&p.tv);
      mbar_arrive_expect_tx(q_full, TB);
      for (int j = 0; j < NA; ++j) tma_load_2d(base + F_OFF_Q + j * ATOM, &p.tq, q_full, h * D + 64 * j, row0 + qt * TT);
      int issued_k = 0, issued_v = 0;
      for (int kt = 0; kt < nk; ++kt) {
        if (kt > 0 && !mbar_wait(k_empty, (kt - 1) & 1, abort_flag, p.err, KID_ATTN, 21)) break;
        mbar_arrive_expect_tx(k_full, TB);
        for (int j = 0; j < NA; ++j)
          tma_load_2d(base + F_OFF_K + j * ATOM, &p.tk, k_full, kvh * D + 64 * j, row0 + kt * TT);
        issued_k = kt + 1;
        if (kt > 0 && !mbar_wait(v_empty, (kt - 1) & 1, abort_flag, p.err, KID_ATTN, 22)) break;
        mbar_arrive_expect_tx(v_full, TB);
        for (int j = 0; j < NA; ++j)
          tma_load_2d(base + F_OFF_V + j * ATOM, &p.tv, v_full, kvh * D + 64 * j, row0 + kt * TT);
        issued_v = kt + 1;
      }
      if (*abort_flag) {  // let the copies already issued land before the CTA exits
        mbar_wait_drain(q_full, 0);
        if (issued_k > 0) mbar_wait_drain(k_full, (issued_k - 1) & 1);
        if (issued_v > 0) mbar_wait_drain(v_full, (issued_v - 1) & 1);
      }
    }
  } else if (warp == F_MMA) {
    // ------------------------------------------------------------------ MMA issuer
    constexpr uint32_t idesc_s = idesc_bf16(128, 128, false);  // Q K^T: both K-major
    constexpr uint32_t idesc_o = idesc_bf16(128, D, true);     // P V: V N-major
    const uint32_t sQ = smem_u32(base + F_OFF_Q), sK = smem_u32(base + F_OFF_K), sV = smem_u32(base + F_OFF_V);
    // every wait is agreed on by the whole warp (__all_sync), so that no lane goes on alone
    bool ok = __all_sync(0xffffffffu, mbar_wait(q_full, 0, abort_flag, p.err, KID_ATTN, 23));
    for (int kt = 0; ok && kt < nk; ++kt) {
      if (!(ok = __all_sync(0xffffffffu, mbar_wait(k_full, kt & 1, abort_flag, p.err, KID_ATTN, 24)))) break;
      tc_fence_after();
      if (lane == 0) {
        // tcgen05.mma of one thread run in issue order, so S may overwrite the P that
        // the previous tile's P V product reads
#pragma unroll
        for (int ks = 0; ks < KS; ++ks) {
          const uint32_t off = (ks >> 2) * ATOM + (ks & 3) * 32;
          umma_bf16(tmem, sdesc_sw128(sQ + off, 16, 1024), sdesc_sw128(sK + off, 16, 1024), idesc_s, ks ? 1u : 0u);
        }
        umma_commit(s_full);
        umma_commit(k_empty);
      }
      __syncwarp();
      if (!(ok = __all_sync(0xffffffffu, mbar_wait(p_full, kt & 1, abort_flag, p.err, KID_ATTN, 25)))) break;
      if (!(ok = __all_sync(0xffffffffu, mbar_wait(v_full, kt & 1, abort_flag, p.err, KID_ATTN, 26)))) break;
      tc_fence_after();
      if (lane == 0) {
#pragma unroll
        for (int ks = 0; ks < 8; ++ks)  // 16 keys per step: P columns 8 ks .., V rows 16 ks ..
          umma_bf16_ta(tmem + 128, tmem + ks * 8, sdesc_sw128(sV + ks * 2048, ATOM, 1024), idesc_o,
                       (kt | ks) ? 1u : 0u);
        umma_commit(v_empty);
        umma_commit(o_full);
      }
      __syncwarp();
    }
  } else {
    // ------------------------------------------------------------------ softmax + epilogue
    const int r = warp * 32 + lane;  // query row in the tile = TMEM lane
    const int qpos = qt * TT + r;    // position in the sequence
    const uint32_t trow = tmem + ((uint32_t)(warp * 32) << 16);
    const float sl = p.scale_log2;
    float m_run = -INFINITY, l_run = 0.f;
    bool ok = true;
    for (int kt = 0; kt < nk; ++kt) {
      if (!(ok = __all_sync(0xffffffffu, mbar_wait(s_full, kt & 1, abort_flag, p.err, KID_ATTN, 27)))) break;
      tc_fence_after();
      const bool diag = kt == qt;
      // row maximum of the raw scores (the scale is positive), two TMEM loads per wait
      float mx = -INFINITY;
#pragma unroll
      for (int c = 0; c < 4; c += 2) {
        uint32_t v[2][32];
        tmem_ld32(trow + c * 32, v[0]);
        tmem_ld32(trow + c * 32 + 32, v[1]);
        tmem_wait_ld();
#pragma unroll
        for (int h = 0; h < 2; ++h)
#pragma unroll
          for (int i = 0; i < 32; ++i)
            if (!diag || (c + h) * 32 + i <= r) mx = fmaxf(mx, __uint_as_float(v[h][i]));
      }
      mx *= sl;
      const float m_new = (kt == 0 || mx > m_run + kRescaleLog2) ? fmaxf(mx, m_run) : m_run;
      const bool resc = kt > 0 && m_new != m_run;
      if (__any_sync(0xffffffffu, resc)) {
        // the previous tile's P V product must be in O before O is scaled
        if (!(ok = __all_sync(0xffffffffu, mbar_wait(o_full, (kt - 1) & 1, abort_flag, p.err, KID_ATTN, 28)))) break;
        tc_fence_after();
        const float alpha = resc ? fast_exp2(m_run - m_new) : 1.0f;
#pragma unroll
        for (int c = 0; c < D / 32; ++c) {
          uint32_t v[32];
          tmem_ld32(trow + 128 + c * 32, v);
          tmem_wait_ld();
#pragma unroll
          for (int i = 0; i < 32; ++i) v[i] = __float_as_uint(__uint_as_float(v[i]) * alpha);
          tmem_st32(trow + 128 + c * 32, v);
        }
        tmem_wait_st();
        l_run *= alpha;
      }
      m_run = m_new;
      float sum = 0.f;
#pragma unroll
      for (int c = 0; c < 4; c += 2) {
        // keys 32 c .. 32 c + 63; their P goes to columns 16 c .., scores already read
        uint32_t v[2][32], pk[2][16];
        tmem_ld32(trow + c * 32, v[0]);
        tmem_ld32(trow + c * 32 + 32, v[1]);
        tmem_wait_ld();
#pragma unroll
        for (int h = 0; h < 2; ++h)
#pragma unroll
          for (int j = 0; j < 16; ++j) {
            const int k0 = (c + h) * 32 + 2 * j;
            float p0 = fast_exp2(fmaf(__uint_as_float(v[h][2 * j]), sl, -m_run));
            float p1 = fast_exp2(fmaf(__uint_as_float(v[h][2 * j + 1]), sl, -m_run));
            if (diag) {
              p0 = k0 <= r ? p0 : 0.f;
              p1 = k0 + 1 <= r ? p1 : 0.f;
            }
            sum += p0 + p1;
            pk[h][j] = pack_bf16x2(p0, p1);
          }
        tmem_st16(trow + c * 16, pk[0]);
        tmem_st16(trow + c * 16 + 16, pk[1]);
      }
      tmem_wait_st();
      l_run += sum;
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(p_full);
    }
    // O / sum through the freed Q tile's shared memory and two TMA stores (coalesced rows);
    // all four warps reach the barrier, the store is issued only when no wait failed
    if (ok && __all_sync(0xffffffffu, mbar_wait(o_full, (nk - 1) & 1, abort_flag, p.err, KID_ATTN, 29))) {
      tc_fence_after();
      const float inv = 1.0f / l_run;
      const uint32_t tile = smem_u32(base + F_OFF_Q);
#pragma unroll
      for (int c = 0; c < D / 32; c += 2) {
        uint32_t v[2][32];
        tmem_ld32(trow + 128 + c * 32, v[0]);
        tmem_ld32(trow + 128 + c * 32 + 32, v[1]);
        tmem_wait_ld();
        stage_row32(tile, r, c, v[0], inv);
        stage_row32(tile, r, c + 1, v[1], inv);
      }
      p.lse[((size_t)b * p.nq + h) * p.seq + qpos] = (m_run + log2f(l_run)) * 0.6931471805599453f;
    }
    fence_proxy_async_smem();
    asm volatile("bar.sync 1, 128;" ::: "memory");
    if (threadIdx.x == 0 && !*abort_flag) {
      for (int j = 0; j < NA; ++j) tma_store_2d(&p.to, smem_u32(base + F_OFF_Q + j * ATOM), h * D + 64 * j, row0 + qt * TT);
      tma_store_drain();
    }
  }

  // On an aborted run the products already issued must finish before TMEM is freed.
  __syncthreads();
  if (warp == F_MMA && *abort_flag) {
    if (lane == 0) umma_commit(drain);
    __syncwarp();
    mbar_wait_drain(drain, 0);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == F_MMA) {
    tc_fence_after();
    tmem_dealloc(tmem, 256);
  }
}

// ------------------------------------------------------------------------------ backward
// dQ (per query tile and head) and dK, dV (per key tile and kv head) on tcgen05, one
// 128 x 128 block ("item") at a time:
//   query side, item = one key tile:   S = Q K^T, dP = dO V^T (N = 128); after the
//     elementwise step dQ += dS K (dS from TMEM as the A operand, K = 128).
//   key side, item = one query tile:   S^T = K Q^T, dP^T = V dO^T; then dV += P^T dO and
//     dK += dS^T Q.
// Every product is M = 128, N = 128: a tcgen05.mma of N = 64 runs at about 60% of the
// tensor core's rate (measured), one of N >= 128 at its full rate, so a whole tile per
// item and one item buffer (the S and dP blocks and the two accumulators fill the 512
// TMEM columns) beat half tiles with two buffers in flight.
// P = 2^(S log2e / sqrt(d) - lse log2e) (causal mask), dS = P (dP - delta).  The eight
// elementwise warps take a lane quarter and 64 columns each, in two 32-column chunks;
// P / dS are written back as bf16 (two per 32-bit column) over scores that the same
// warp has already read: chunk h of warp half g packs into columns 64 g + 16 h ..
// of its block, so the A operand of k-step ks (16 rows of the reduction) sits at
// column 64 (ks / 4) + 8 (ks % 4).  The query-side kernel also forms
// delta = rowsum(dO * O) for its rows and writes it for the key side, which runs after
// it.  Accumulation runs in a fixed order (query side: key tiles in order; key side:
// query heads of the group, then query tiles), so results are bit-reproducible.

struct AttnBwdParams {
  CUtensorMap tq, tk, tv, tdo, to;  // box 64 cols x 128 rows, 128-byte swizzle (to: the output O)
  CUtensorMap tdq, tdk, tdv;        // the gradients, same boxes (TMA stores)
  const float* lse;
  float* delta;                 // written by the query side, read by the key side
  __nv_bfloat16* dq;
  __nv_bfloat16* dk;
  __nv_bfloat16* dv;
  int ld_dq, ld_dkv, seq, nq, nkv;
  float scale, scale_log2;
  int* err;
};

// warps 0-7: elementwise and epilogue (warp w: TMEM lane quarter w % 4, column half
// w / 4); warp 8: TMA producer; warp 9: MMA issuer
constexpr int B_THREADS = 320, B_PROD = 8, B_MMA = 9, B_EW = 256;
constexpr int B_OFF_A = 0;                              // Q, dO (query side) or K, V (key side)
constexpr int B_OFF_RING = 2 * TILE_BYTES;              // 2 stages x (two 32 KB tiles)
constexpr int B_OFF_X = B_OFF_RING + 4 * TILE_BYTES;    // query side: O tile and delta halves [2][128];
                                                        // key side: 2 stages x (128 lse + 128 delta floats)
constexpr int B_OFF_BAR = B_OFF_X + TILE_BYTES + 1024;
constexpr int SMEM_BWD = 1024 + B_OFF_BAR + 256;

__device__ __forceinline__ void bar_ew() { asm volatile("bar.sync 1, %0;" ::"n"(B_EW) : "memory"); }

// TMEM column of the A operand of 16-row step ks (0-7) of a block whose first column is
// c0: warp half g packed its 64 rows' values to columns c0 + 64 g .. c0 + 64 g + 31.
__device__ __forceinline__ uint32_t packed_col(uint32_t c0, int ks) { return c0 + (ks >> 2) * 64 + (ks & 3) * 8; }

// QUERY side: dQ of one 128-query tile of one query head.  The Q and dO tiles are
// copied once into TMEM (bf16 pairs, one query row per lane), so that S = Q K^T and
// dP = dO V^T take their A operand from TMEM and read only K and V from shared memory
// (4 KB per 64 tensor-core cycles instead of 8 KB, which is all that shared memory
// delivers, while the next K and V tiles land in it).
template <int D>
__global__ void __launch_bounds__(B_THREADS, 1) k_attn_dq_tc(const __grid_constant__ AttnBwdParams p) {
  // swizzle atoms, k-steps and bytes of a Q / dO / O / K / V tile; dims per column half
  constexpr int NA = D / 64, KS = D / 16, TB = NA * ATOM, DH = D / 2;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(base + B_OFF_BAR);
  uint64_t* q_full = bars;          // Q, dO (copied into TMEM first)
  uint64_t* kv_full = bars + 1;     // 2 stages
  uint64_t* kv_empty = bars + 3;    // 2
  uint64_t* sd_full = bars + 5;     // S and dP of the item are in TMEM
  uint64_t* p_half = bars + 6;      // 2: dS chunk hc of the item is in TMEM (one arrival per warp)
  uint64_t* acc_full = bars + 9;
  uint64_t* drain = bars + 10;
  uint64_t* qa_full = bars + 11;    // Q and dO are in TMEM (one arrival per elementwise warp)
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 12);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  uint64_t* o_full = bars + 13;     // the O tile (for delta)

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int qt = gridDim.z - 1 - blockIdx.z, h = blockIdx.x, b = blockIdx.y;  // z slowest: longest rows first
  const int kvh = h / (p.nq / p.nkv);
  const int n_kt = qt + 1;  // key tiles at or before the diagonal
  const int row0 = b * p.seq;

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    mbar_init(o_full, 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(&kv_full[i], 1);
      mbar_init(&kv_empty[i], 1);
    }
    mbar_init(sd_full, 1);
    mbar_init(&p_half[0], B_EW / 32);
    mbar_init(&p_half[1], B_EW / 32);
    mbar_init(acc_full, 1);
    mbar_init(drain, 1);
    mbar_init(qa_full, B_EW / 32);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == B_MMA) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  // S [0,128), dP [128,256) (dS packed over it), dQ [256,384), Q [384,448), dO [448,512)
  const uint32_t tmem = *tmem_slot;
  constexpr uint32_t T_Q = 384, T_DO = 448;

  if (warp == B_PROD) {
    if (lane == 0) {
      tma_prefetch_desc(&p.tq);
      tma_prefetch_desc(&p.tk);
      tma_prefetch_desc(&p.tv);
      tma_prefetch_desc(&p.tdo);
      tma_prefetch_desc(&p.to);
      mbar_arrive_expect_tx(q_full, 2 * TB);
      for (int j = 0; j < NA; ++j) {
        tma_load_2d(base + B_OFF_A + j * ATOM, &p.tq, q_full, h * D + 64 * j, row0 + qt * TT);
        tma_load_2d(base + B_OFF_A + TILE_BYTES + j * ATOM, &p.tdo, q_full, h * D + 64 * j, row0 + qt * TT);
      }
      mbar_arrive_expect_tx(o_full, TB);
      for (int j = 0; j < NA; ++j)
        tma_load_2d(base + B_OFF_X + j * ATOM, &p.to, o_full, h * D + 64 * j, row0 + qt * TT);
      int issued = 0;
      for (int kt = 0; kt < n_kt; ++kt) {
        const int st = kt & 1;
        if (kt >= 2 && !mbar_wait(&kv_empty[st], ((kt >> 1) - 1) & 1, abort_flag, p.err, KID_ATTN, 41)) break;
        uint8_t* buf = base + B_OFF_RING + st * 2 * TILE_BYTES;
        mbar_arrive_expect_tx(&kv_full[st], 2 * TB);
        for (int j = 0; j < NA; ++j) {
          tma_load_2d(buf + j * ATOM, &p.tk, &kv_full[st], kvh * D + 64 * j, row0 + kt * TT);
          tma_load_2d(buf + TILE_BYTES + j * ATOM, &p.tv, &kv_full[st], kvh * D + 64 * j, row0 + kt * TT);
        }
        issued = kt + 1;
      }
      if (*abort_flag) {  // let the copies already issued land before the CTA exits
        mbar_wait_drain(q_full, 0);
        mbar_wait_drain(o_full, 0);
        for (int kt = (issued > 2 ? issued - 2 : 0); kt < issued; ++kt) mbar_wait_drain(&kv_full[kt & 1], (kt >> 1) & 1);
      }
    }
  } else if (warp == B_MMA) {
    constexpr uint32_t idesc_s = idesc_bf16(128, 128, false);  // S, dP: N = 128 keys
    constexpr uint32_t idesc_a = idesc_bf16(128, D, true);     // dQ += dS K: K N-major
    bool ok = __all_sync(0xffffffffu, mbar_wait(qa_full, 0, abort_flag, p.err, KID_ATTN, 42)) && !*abort_flag;
    // dQ += dS_kt K_kt, each half as soon as its dS chunks are in TMEM (chunk hc holds the
    // k-steps with ks & 2 == 2 hc); then the K/V stage is free
    auto dq_product = [&](int kt) -> bool {
      const uint32_t sK = smem_u32(base + B_OFF_RING + (kt & 1) * 2 * TILE_BYTES);
      for (int hc = 0; hc < 2; ++hc) {
        if (!__all_sync(0xffffffffu, mbar_wait(&p_half[hc], kt & 1, abort_flag, p.err, KID_ATTN, 44))) return false;
        tc_fence_after();
        if (lane == 0) {
#pragma unroll
          for (int i = 0; i < 4; ++i) {  // 16 keys per step
            const int ks = (i >> 1) * 4 + hc * 2 + (i & 1);
            umma_bf16_ta(tmem + 256, tmem + packed_col(128, ks), sdesc_sw128(sK + ks * 2048, ATOM, 1024), idesc_a,
                         (kt | hc | i) ? 1u : 0u);
          }
          if (hc == 1) umma_commit(&kv_empty[kt & 1]);
        }
        __syncwarp();
      }
      return true;
    };
    for (int kt = 0; ok && kt < n_kt; ++kt) {
      if (!(ok = __all_sync(0xffffffffu, mbar_wait(&kv_full[kt & 1], (kt >> 1) & 1, abort_flag, p.err, KID_ATTN,
                                                   43))))
        break;
      // the previous item's dS is read (issue order) before S and dP overwrite it
      if (kt >= 1 && !(ok = dq_product(kt - 1))) break;
      tc_fence_after();
      if (lane == 0) {
        const uint32_t sK = smem_u32(base + B_OFF_RING + (kt & 1) * 2 * TILE_BYTES), sV = sK + TILE_BYTES;
#pragma unroll
        for (int ks = 0; ks < KS; ++ks) {  // over the head dim: Q, dO columns 8 ks .. in TMEM
          const uint32_t off = (ks >> 2) * ATOM + (ks & 3) * 32;
          umma_bf16_ta(tmem, tmem + T_Q + ks * 8, sdesc_sw128(sK + off, 16, 1024), idesc_s, ks ? 1u : 0u);
          umma_bf16_ta(tmem + 128, tmem + T_DO + ks * 8, sdesc_sw128(sV + off, 16, 1024), idesc_s, ks ? 1u : 0u);
        }
        umma_commit(sd_full);
      }
      __syncwarp();
    }
    if (ok) ok = dq_product(n_kt - 1);
    if (ok && lane == 0) umma_commit(acc_full);
    __syncwarp();
  } else {
    // ------------------------------------------------------------------ elementwise + epilogue
    const int wq = warp & 3, g = warp >> 2;
    const int r = wq * 32 + lane;  // query row = TMEM lane
    const int qpos = qt * TT + r;
    const uint32_t trow = tmem + ((uint32_t)(wq * 32) << 16);
    const size_t li = ((size_t)b * p.nq + h) * p.seq + qpos;
    // First Q and dO into TMEM (the MMA warp starts on them), then delta = rowsum(dO * O)
    // over this thread's DH dims (dims g DH .. of its row: 16-byte chunks c0 + c of swizzle
    // atom g DH / 64 of the dO and O tiles), the two halves added through smem.  TMEM
    // column g DH / 2 + 4 c + i holds the pair i of chunk c.
    float* red = reinterpret_cast<float*>(base + B_OFF_X + TILE_BYTES);
    const int atom = (g * DH) / 64, c0 = ((g * DH) % 64) / 8;
    const uint8_t* q_row = base + B_OFF_A + atom * ATOM + r * 128;
    const uint8_t* dO_row = base + B_OFF_A + TILE_BYTES + atom * ATOM + r * 128;
    const uint8_t* o_row = base + B_OFF_X + atom * ATOM + r * 128;
    bool ok = __all_sync(0xffffffffu, mbar_wait(q_full, 0, abort_flag, p.err, KID_ATTN, 45));
    if (ok) {
      uint32_t qv[DH / 2], dv[DH / 2];
#pragma unroll
      for (int c = 0; c < DH / 8; ++c) {
        const uint32_t off = (uint32_t)(((c0 + c) ^ (r & 7)) << 4);
        const uint4 d = *reinterpret_cast<const uint4*>(dO_row + off);
        const uint4 q = *reinterpret_cast<const uint4*>(q_row + off);
        qv[4 * c] = q.x, qv[4 * c + 1] = q.y, qv[4 * c + 2] = q.z, qv[4 * c + 3] = q.w;
        dv[4 * c] = d.x, dv[4 * c + 1] = d.y, dv[4 * c + 2] = d.z, dv[4 * c + 3] = d.w;
      }
      tmem_st_cols(trow + T_Q + g * (DH / 2), qv);
      tmem_st_cols(trow + T_DO + g * (DH / 2), dv);
      tmem_wait_st();
    }
    tc_fence_before();
    __syncwarp();
    if (lane == 0) mbar_arrive(qa_full);  // also on failure: the MMA warp then sees the abort
    if (ok) ok = __all_sync(0xffffffffu, mbar_wait(o_full, 0, abort_flag, p.err, KID_ATTN, 48));
    if (ok) {
      float s = 0.f;
#pragma unroll
      for (int c = 0; c < DH / 8; ++c) {
        const uint32_t off = (uint32_t)(((c0 + c) ^ (r & 7)) << 4);
        const uint4 a = *reinterpret_cast<const uint4*>(o_row + off);
        const uint4 d = *reinterpret_cast<const uint4*>(dO_row + off);
        const uint32_t aw[4] = {a.x, a.y, a.z, a.w}, dw[4] = {d.x, d.y, d.z, d.w};
#pragma unroll
        for (int j = 0; j < 4; ++j) s += bf16_lo(aw[j]) * bf16_lo(dw[j]) + bf16_hi(aw[j]) * bf16_hi(dw[j]);
      }
      red[g * 128 + r] = s;
    }
    bar_ew();
    const float dl = ok ? red[r] + red[128 + r] : 0.f;
    if (ok && g == 0) p.delta[li] = dl;
    const float lse2 = p.lse[li] * 1.4426950408889634f;
    const float sl = p.scale_log2;
    for (int kt = 0; ok && kt < n_kt; ++kt) {
      if (!(ok = __all_sync(0xffffffffu, mbar_wait(sd_full, kt & 1, abort_flag, p.err, KID_ATTN, 46)))) break;
      tc_fence_after();
      // both 32-key chunks in one TMEM round trip
      uint32_t sv[2][32], dpv[2][32];
#pragma unroll
      for (int hc = 0; hc < 2; ++hc) {
        tmem_ld32(trow + g * 64 + hc * 32, sv[hc]);
        tmem_ld32(trow + 128 + g * 64 + hc * 32, dpv[hc]);
      }
      tmem_wait_ld();
#pragma unroll
      for (int hc = 0; hc < 2; ++hc) {  // keys 64 g + 32 hc .. of the tile
        uint32_t dd[16];
        const int key0 = kt * TT + g * 64 + hc * 32;
#pragma unroll
        for (int j = 0; j < 16; ++j) {
          float ds[2];
#pragma unroll
          for (int e = 0; e < 2; ++e) {
            const int kj = key0 + 2 * j + e;
            const float pe = kj <= qpos ? fast_exp2(fmaf(__uint_as_float(sv[hc][2 * j + e]), sl, -lse2)) : 0.f;
            ds[e] = pe * (__uint_as_float(dpv[hc][2 * j + e]) - dl);
          }
          dd[j] = pack_bf16x2(ds[0], ds[1]);
        }
        tmem_st16(trow + 128 + g * 64 + hc * 16, dd);  // over dP values this warp has read
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&p_half[hc]);
      }
    }
    // dQ through the freed ring's shared memory and two TMA stores (coalesced rows); every
    // elementwise warp reaches the barrier, the store is issued only when no wait failed
    if (ok && __all_sync(0xffffffffu, mbar_wait(acc_full, 0, abort_flag, p.err, KID_ATTN, 47))) {
      tc_fence_after();
      uint32_t v[DH / 32][32];
#pragma unroll
      for (int i = 0; i < DH / 32; ++i) tmem_ld32(trow + 256 + g * DH + 32 * i, v[i]);
      tmem_wait_ld();
      const uint32_t tile = smem_u32(base + B_OFF_RING);
#pragma unroll
      for (int i = 0; i < DH / 32; ++i) stage_row32(tile, r, g * (DH / 32) + i, v[i], p.scale);
    }
    fence_proxy_async_smem();
    bar_ew();
    if (threadIdx.x == 0 && !*abort_flag) {
      for (int j = 0; j < NA; ++j)
        tma_store_2d(&p.tdq, smem_u32(base + B_OFF_RING + j * ATOM), h * D + 64 * j, row0 + qt * TT);
      tma_store_drain();
    }
  }
  __syncthreads();
  if (warp == B_MMA && *abort_flag) {  // products already issued finish before TMEM is freed
    if (lane == 0) umma_commit(drain);
    __syncwarp();
    mbar_wait_drain(drain, 0);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == B_MMA) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// Bulk copy of bytes (a multiple of 16) from this CTA's shared memory to another CTA's of
// the cluster, completing transaction bytes on that CTA's mbarrier (both given by their
// shared::cluster addresses).
__device__ __forceinline__ void bulk_copy_to_peer(uint32_t dst_cluster, uint32_t src, uint32_t bytes,
                                                  uint32_t bar_cluster) {
  asm volatile("cp.async.bulk.shared::cluster.shared::cta.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
                   dst_cluster),
               "r"(src), "r"(bytes), "r"(bar_cluster)
               : "memory");
}

// KEY side: dK, dV of one 128-key tile of one kv head, by a cluster of two CTAs that split
// the group's query heads (the first ceil(group / 2) heads and the rest).  Each CTA then
// finishes one of the two tensors: it stages the other tensor's fp32 partial sums in its own
// shared memory and sends them in one bulk copy into the peer's (distributed shared memory),
// and adds the peer's to its own in the order first CTA + second CTA.  Halving the longest
// CTAs' work balances the grid (two CTAs per key tile instead of one, the first key tiles
// holding the most query tiles); splitting the exchange halves the copy and the final pass
// of each CTA (per-thread remote stores of both tensors, 132 KB, from one CTA measured
// about 13 000 cycles).

template <int D>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(B_THREADS, 1)
    k_attn_dkv_tc(const __grid_constant__ AttnBwdParams p) {
  // swizzle atoms, k-steps and bytes of a K / V / Q / dO tile; dims per column half
  constexpr int NA = D / 64, KS = D / 16, TB = NA * ATOM, DH = D / 2;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(base + B_OFF_BAR);
  uint64_t* kv_full = bars;         // K, V
  uint64_t* qd_full = bars + 1;     // 2 stages (Q, dO, lse, delta of one (head, query tile))
  uint64_t* qd_empty = bars + 3;    // 2
  uint64_t* sd_full = bars + 5;     // S^T and dP^T of the item are in TMEM
  uint64_t* p_half = bars + 6;      // 2: P^T, dS^T chunk hc of the item are in TMEM (one arrival per warp)
  uint64_t* acc_full = bars + 9;
  uint64_t* drain = bars + 10;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 11);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  uint64_t* peer_full = bars + 12;  // the peer CTA's partial sums of this CTA's tensor have landed

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int kvh = blockIdx.x >> 1, b = blockIdx.y, kt = blockIdx.z;  // z slowest: the longest key tiles first
  const uint32_t crank = cluster_ctarank();
  const int grp = p.nq / p.nkv, n_qt = p.seq / TT;
  const int hpc = (grp + 1) / 2, h_begin = (int)crank * hpc, h_count = min(grp, h_begin + hpc) - h_begin;
  // (head, query tile) items of this CTA
  const int per_head = n_qt - kt, n_st = h_count * per_head;
  const int row0 = b * p.seq;

  if (threadIdx.x == 0) {
    mbar_init(kv_full, 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(&qd_full[i], 1);
      mbar_init(&qd_empty[i], 1);
    }
    mbar_init(sd_full, 1);
    mbar_init(&p_half[0], B_EW / 32);
    mbar_init(&p_half[1], B_EW / 32);
    mbar_init(acc_full, 1);
    mbar_init(drain, 1);
    mbar_init(peer_full, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == B_MMA) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;  // S^T [0,128), dP^T [128,256) (P^T, dS^T packed over them), dV, dK

  if (warp == B_PROD) {
    if (lane == 0) {
      tma_prefetch_desc(&p.tq);
      tma_prefetch_desc(&p.tk);
      tma_prefetch_desc(&p.tv);
      tma_prefetch_desc(&p.tdo);
      mbar_arrive_expect_tx(kv_full, 2 * TB);
      for (int j = 0; j < NA; ++j) {
        tma_load_2d(base + B_OFF_A + j * ATOM, &p.tk, kv_full, kvh * D + 64 * j, row0 + kt * TT);
        tma_load_2d(base + B_OFF_A + TILE_BYTES + j * ATOM, &p.tv, kv_full, kvh * D + 64 * j, row0 + kt * TT);
      }
      int issued = 0;
      for (int sti = 0; sti < n_st; ++sti) {
        const int bf = sti & 1;
        if (sti >= 2 && !mbar_wait(&qd_empty[bf], ((sti >> 1) - 1) & 1, abort_flag, p.err, KID_ATTN, 31)) break;
        const int h = kvh * grp + h_begin + sti / per_head, qt = kt + sti % per_head;
        uint8_t* buf = base + B_OFF_RING + bf * 2 * TILE_BYTES;
        float* ld = reinterpret_cast<float*>(base + B_OFF_X + bf * 1024);
        mbar_arrive_expect_tx(&qd_full[bf], 2 * TB + 1024);
        for (int j = 0; j < NA; ++j) {
          tma_load_2d(buf + j * ATOM, &p.tq, &qd_full[bf], h * D + 64 * j, row0 + qt * TT);
          tma_load_2d(buf + TILE_BYTES + j * ATOM, &p.tdo, &qd_full[bf], h * D + 64 * j, row0 + qt * TT);
        }
        const size_t lo = ((size_t)b * p.nq + h) * p.seq + qt * TT;
        bulk_load(ld, p.lse + lo, 512, &qd_full[bf]);
        bulk_load(ld + 128, p.delta + lo, 512, &qd_full[bf]);
        issued = sti + 1;
      }
      if (*abort_flag) {  // let the copies already issued land before the CTA exits
        mbar_wait_drain(kv_full, 0);
        for (int i = (issued > 2 ? issued - 2 : 0); i < issued; ++i) mbar_wait_drain(&qd_full[i & 1], (i >> 1) & 1);
      }
    }
  } else if (warp == B_MMA) {
    constexpr uint32_t idesc_s = idesc_bf16(128, 128, false);  // S^T, dP^T: N = 128 queries
    constexpr uint32_t idesc_a = idesc_bf16(128, D, true);     // dV, dK: dO, Q N-major
    const uint32_t sK = smem_u32(base + B_OFF_A), sV = sK + TILE_BYTES;
    bool ok = n_st > 0 && __all_sync(0xffffffffu, mbar_wait(kv_full, 0, abort_flag, p.err, KID_ATTN, 32));
    // dV += P^T dO, dK += dS^T Q, each half as soon as its chunks are in TMEM (chunk hc holds
    // the k-steps with ks & 2 == 2 hc); then the stage is free
    auto kv_products = [&](int sti) -> bool {
      const uint32_t sQ = smem_u32(base + B_OFF_RING + (sti & 1) * 2 * TILE_BYTES), sO = sQ + TILE_BYTES;
      for (int hc = 0; hc < 2; ++hc) {
        if (!__all_sync(0xffffffffu, mbar_wait(&p_half[hc], sti & 1, abort_flag, p.err, KID_ATTN, 34))) return false;
        tc_fence_after();
        if (lane == 0) {
#pragma unroll
          for (int i = 0; i < 4; ++i) {  // 16 queries per step
            const int ks = (i >> 1) * 4 + hc * 2 + (i & 1);
            const uint32_t acc = (sti | hc | i) ? 1u : 0u;
            umma_bf16_ta(tmem + 256, tmem + packed_col(0, ks), sdesc_sw128(sO + ks * 2048, ATOM, 1024), idesc_a, acc);
            umma_bf16_ta(tmem + 384, tmem + packed_col(128, ks), sdesc_sw128(sQ + ks * 2048, ATOM, 1024), idesc_a,
                         acc);
          }
          if (hc == 1) umma_commit(&qd_empty[sti & 1]);
        }
        __syncwarp();
      }
      return true;
    };
    for (int sti = 0; ok && sti < n_st; ++sti) {
      if (!(ok = __all_sync(0xffffffffu, mbar_wait(&qd_full[sti & 1], (sti >> 1) & 1, abort_flag, p.err, KID_ATTN,
                                                   33))))
        break;
      // the previous item's P^T and dS^T are read (issue order) before S^T, dP^T overwrite them
      if (sti >= 1 && !(ok = kv_products(sti - 1))) break;
      tc_fence_after();
      if (lane == 0) {
        const uint32_t sQ = smem_u32(base + B_OFF_RING + (sti & 1) * 2 * TILE_BYTES), sO = sQ + TILE_BYTES;
#pragma unroll
        for (int ks = 0; ks < KS; ++ks) {  // S^T = K Q^T, dP^T = V dO^T over the head dim
          const uint32_t off = (ks >> 2) * ATOM + (ks & 3) * 32;
          umma_bf16(tmem, sdesc_sw128(sK + off, 16, 1024), sdesc_sw128(sQ + off, 16, 1024), idesc_s, ks ? 1u : 0u);
          umma_bf16(tmem + 128, sdesc_sw128(sV + off, 16, 1024), sdesc_sw128(sO + off, 16, 1024), idesc_s,
                    ks ? 1u : 0u);
        }
        umma_commit(sd_full);
      }
      __syncwarp();
    }
    if (ok) ok = kv_products(n_st - 1);
    if (ok && lane == 0) umma_commit(acc_full);
    __syncwarp();
  } else {
    const int wq = warp & 3, g = warp >> 2;
    const int r = wq * 32 + lane;  // key row = TMEM lane
    const int key = kt * TT + r;
    const uint32_t trow = tmem + ((uint32_t)(wq * 32) << 16);
    const float sl = p.scale_log2;
    bool ok = true;
    for (int sti = 0; sti < n_st; ++sti) {
      const int qt = kt + sti % per_head;
      if (!(ok = __all_sync(0xffffffffu, mbar_wait(sd_full, sti & 1, abort_flag, p.err, KID_ATTN, 35)))) break;
      tc_fence_after();
      const float* ld = reinterpret_cast<const float*>(base + B_OFF_X + (sti & 1) * 1024);
#pragma unroll
      for (int hc = 0; hc < 2; ++hc) {  // queries 64 g + 32 hc .. of the tile
        uint32_t sv[32], dpv[32], pp[16], dd[16];
        tmem_ld32(trow + g * 64 + hc * 32, sv);
        tmem_ld32(trow + 128 + g * 64 + hc * 32, dpv);
        tmem_wait_ld();
        const int qi0 = g * 64 + hc * 32;     // query within the tile
        const int lim = key - qt * TT - qi0;  // columns c < lim are masked (only on the diagonal tile)
#pragma unroll
        for (int j4 = 0; j4 < 8; ++j4) {  // four columns: their lse and delta in one vector load each
          const float4 l4 = *reinterpret_cast<const float4*>(ld + qi0 + 4 * j4);
          const float4 d4 = *reinterpret_cast<const float4*>(ld + 128 + qi0 + 4 * j4);
          const float lv[4] = {l4.x, l4.y, l4.z, l4.w}, dl[4] = {d4.x, d4.y, d4.z, d4.w};
          float pv[4], ds[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const int c = 4 * j4 + e;
            const float pe =
                c >= lim ? fast_exp2(fmaf(__uint_as_float(sv[c]), sl, -lv[e] * 1.4426950408889634f)) : 0.f;
            pv[e] = pe;
            ds[e] = pe * (__uint_as_float(dpv[c]) - dl[e]);
          }
          pp[2 * j4] = pack_bf16x2(pv[0], pv[1]);
          pp[2 * j4 + 1] = pack_bf16x2(pv[2], pv[3]);
          dd[2 * j4] = pack_bf16x2(ds[0], ds[1]);
          dd[2 * j4 + 1] = pack_bf16x2(ds[2], ds[3]);
        }
        tmem_st16(trow + g * 64 + hc * 16, pp);  // over scores this warp has read
        tmem_st16(trow + 128 + g * 64 + hc * 16, dd);
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&p_half[hc]);
      }
    }
    const bool have = n_st > 0 && ok && __all_sync(0xffffffffu, mbar_wait(acc_full, 0, abort_flag, p.err, KID_ATTN, 36));
    if (have) tc_fence_after();
    // The partial sums cross over: the first CTA finishes dV and the second dK, so each sends
    // the other tensor (fp32 rows of D floats, 16-byte chunks swizzled by row) from the start
    // of its freed ring into the back half of the peer's ring.
    constexpr uint32_t PB = 128u * D * 4u;  // one tensor's partial sums
    const uint32_t ring = smem_u32(base + B_OFF_RING);
    const uint32_t t_send = trow + (crank == 0 ? 384u : 256u), t_keep = trow + (crank == 0 ? 256u : 384u);
    const uint32_t prow = (uint32_t)r * (D * 4);
#pragma unroll
    for (int c = 0; c < DH / 32; ++c) {
      uint32_t v[32];
      if (have) {
        tmem_ld32(t_send + g * DH + c * 32, v);
        tmem_wait_ld();
      }
#pragma unroll
      for (int q4 = 0; q4 < 8; ++q4) {
        const uint32_t o = ring + prow + ((uint32_t)(((g * DH + c * 32) / 4 + q4) ^ (r & 7)) << 4);
        if (have)
          st_shared_v4(o, v[4 * q4], v[4 * q4 + 1], v[4 * q4 + 2], v[4 * q4 + 3]);
        else
          st_shared_v4(o, 0u, 0u, 0u, 0u);
      }
    }
    fence_proxy_async_smem();
    if (threadIdx.x == 0) mbar_arrive_expect_tx(peer_full, PB);
    bar_ew();
    // both CTAs have finished their products: both rings are free
    cluster_sync_all();
    if (threadIdx.x == 0) {
      const uint32_t other = crank ^ 1u;
      bulk_copy_to_peer(mapa_shared(ring + PB, other), ring, PB, mapa_shared(smem_u32(peer_full), other));
    }
    (void)__all_sync(0xffffffffu, mbar_wait(peer_full, 0, abort_flag, p.err, KID_ATTN, 37));
    // this CTA's tensor (its sums plus the peer's) through the freed K tile's shared memory
    // and NA TMA stores; dK takes the softmax scale
    const uint32_t tile = smem_u32(base + B_OFF_A);
    const float sc = crank == 0 ? 1.0f : p.scale;
#pragma unroll
    for (int c = 0; c < DH / 32; ++c) {
      float v[32];
      uint32_t vr[32];
      if (have) {
        tmem_ld32(t_keep + g * DH + c * 32, vr);
        tmem_wait_ld();
      }
#pragma unroll
      for (int q4 = 0; q4 < 8; ++q4) {
        const uint4 in = ld_shared_v4(ring + PB + prow + ((uint32_t)(((g * DH + c * 32) / 4 + q4) ^ (r & 7)) << 4));
        const float iv[4] = {__uint_as_float(in.x), __uint_as_float(in.y), __uint_as_float(in.z), __uint_as_float(in.w)};
#pragma unroll
        for (int e = 0; e < 4; ++e) v[4 * q4 + e] = ((have ? __uint_as_float(vr[4 * q4 + e]) : 0.f) + iv[e]) * sc;
      }
      stage_row32(tile, r, g * (DH / 32) + c, v);
    }
    fence_proxy_async_smem();
    bar_ew();
    if (threadIdx.x == 0 && !*abort_flag) {
      const CUtensorMap* map = crank == 0 ? &p.tdv : &p.tdk;
      for (int j = 0; j < NA; ++j) tma_store_2d(map, tile + j * ATOM, kvh * D + 64 * j, row0 + kt * TT);
      tma_store_drain();
    }
    // the peer has its copy of this CTA's partial sums before this shared memory goes
    cluster_sync_all();
  }
  if (warp >= B_EW / 32) {  // the TMA and MMA warps join the two cluster barriers too
    __syncwarp();
    cluster_sync_all();
    cluster_sync_all();
  }
  __syncthreads();
  if (warp == B_MMA && *abort_flag) {  // products already issued finish before TMEM is freed
    if (lane == 0) umma_commit(drain);
    __syncwarp();
    mbar_wait_drain(drain, 0);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == B_MMA) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

}  // namespace

bool attention_fwd_tc_supported(int seq, int d, int nq, int nkv, int ldq, int ldkv, int ldo) {
  return (d == 64 || d == 128) && seq % TT == 0 && seq <= 64 * TT && nq % nkv == 0 && ldq % 8 == 0 &&
         ldkv % 8 == 0 && ldo % 8 == 0;
}

bool attention_bwd_tc_supported(int seq, int d, int nq, int nkv, int ldq, int ldkv, int ldo, int ld_dq, int ld_dkv) {
  return attention_fwd_tc_supported(seq, d, nq, nkv, ldq, ldkv, ldo) && ld_dq % 8 == 0 && ld_dkv % 8 == 0;
}

namespace {
template <int D>
int launch_fwd_tc(const AttnTcParams& p, int batch, int seq, int nq, cudaStream_t s) {
  static int configured[16] = {0};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 16 && !configured[dev]) {
    NF4_CUDA_TRY(cudaFuncSetAttribute(k_attn_fwd_tc<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_TC));
    configured[dev] = 1;
  }
  k_attn_fwd_tc<D><<<dim3(nq, batch, seq / TT), F_THREADS, SMEM_TC, s>>>(p);
  note_launch();
  NF4_CUDA_TRY(cudaGetLastError());
  return NF4LS_OK;
}
}  // namespace

int attention_fwd_tc(const __nv_bfloat16* q, const __nv_bfloat16* k, const __nv_bfloat16* v, int ldq, int ldkv,
                     __nv_bfloat16* o, int ldo, float* lse, int batch, int seq, int nq, int nkv, int d, cudaStream_t s) {
  static_assert(SMEM_TC <= 232448, "shared memory of the tcgen05 attention");
  AttnTcParams p;
  const uint64_t rows = (uint64_t)batch * seq;
  NF4_TRY(tma_map_bf16(&p.tq, q, (uint64_t)nq * d, rows, (uint64_t)ldq * 2, 64, TT));
  NF4_TRY(tma_map_bf16(&p.tk, k, (uint64_t)nkv * d, rows, (uint64_t)ldkv * 2, 64, TT));
  NF4_TRY(tma_map_bf16(&p.tv, v, (uint64_t)nkv * d, rows, (uint64_t)ldkv * 2, 64, TT));
  NF4_TRY(tma_map_bf16(&p.to, o, (uint64_t)nq * d, rows, (uint64_t)ldo * 2, 64, TT));
  p.o = o;
  p.lse = lse;
  p.ldo = ldo;
  p.seq = seq;
  p.nq = nq;
  p.nkv = nkv;
  p.scale_log2 = (1.0f / sqrtf((float)d)) * 1.4426950408889634f;
  p.err = device_error_ptr();
  return d == 64 ? launch_fwd_tc<64>(p, batch, seq, nq, s) : launch_fwd_tc<128>(p, batch, seq, nq, s);
}

}  // namespace nf4ls

namespace nf4ls {

namespace {
template <int D>
int launch_bwd_tc(const AttnBwdParams& p, int batch, int seq, int nq, int nkv, cudaStream_t s) {
  static int configured[16] = {0};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 16 && !configured[dev]) {
    NF4_CUDA_TRY(cudaFuncSetAttribute(k_attn_dq_tc<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_BWD));
    NF4_CUDA_TRY(cudaFuncSetAttribute(k_attn_dkv_tc<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_BWD));
    configured[dev] = 1;
  }
  // the query side writes delta, which the key side reads
  k_attn_dq_tc<D><<<dim3(nq, batch, seq / TT), B_THREADS, SMEM_BWD, s>>>(p);
  note_launch();
  k_attn_dkv_tc<D><<<dim3(2 * nkv, batch, seq / TT), B_THREADS, SMEM_BWD, s>>>(p);
  note_launch();
  NF4_CUDA_TRY(cudaGetLastError());
  return NF4LS_OK;
}
}  // namespace

int attention_bwd_tc(const __nv_bfloat16* q, const __nv_bfloat16* k, const __nv_bfloat16* v, int ldq, int ldkv,
                     const __nv_bfloat16* o, const __nv_bfloat16* dout, int ldo, const float* lse, float* delta,
                     __nv_bfloat16* dq, __nv_bfloat16* dk, __nv_bfloat16* dv, int ld_dq, int ld_dkv, int batch, int seq,
                     int nq, int nkv, int d, cudaStream_t s) {
  static_assert(SMEM_BWD <= 232448, "shared memory of the tcgen05 attention backward");
  AttnBwdParams p;
  const uint64_t rows = (uint64_t)batch * seq;
  NF4_TRY(tma_map_bf16(&p.tq, q, (uint64_t)nq * d, rows, (uint64_t)ldq * 2, 64, TT));
  NF4_TRY(tma_map_bf16(&p.tk, k, (uint64_t)nkv * d, rows, (uint64_t)ldkv * 2, 64, TT));
  NF4_TRY(tma_map_bf16(&p.tv, v, (uint64_t)nkv * d, rows, (uint64_t)ldkv * 2, 64, TT));
  NF4_TRY(tma_map_bf16(&p.tdo, dout, (uint64_t)nq * d, rows, (uint64_t)ldo * 2, 64, TT));
  if (!aligned(lse, 16) || !aligned(delta, 16)) return fail(NF4LS_ALIGN, "attention backward: lse / delta alignment");
  NF4_TRY(tma_map_bf16(&p.to, o, (uint64_t)nq * d, rows, (uint64_t)ldo * 2, 64, TT));
  NF4_TRY(tma_map_bf16(&p.tdq, dq, (uint64_t)nq * d, rows, (uint64_t)ld_dq * 2, 64, TT));
  NF4_TRY(tma_map_bf16(&p.tdk, dk, (uint64_t)nkv * d, rows, (uint64_t)ld_dkv * 2, 64, TT));
  NF4_TRY(tma_map_bf16(&p.tdv, dv, (uint64_t)nkv * d, rows, (uint64_t)ld_dkv * 2, 64, TT));
  p.lse = lse;
  p.delta = delta;
  p.dq = dq;
  p.dk = dk;
  p.dv = dv;
  p.ld_dq = ld_dq;
  p.ld_dkv = ld_dkv;
  p.seq = seq;
  p.nq = nq;
  p.nkv = nkv;
  p.scale = 1.0f / sqrtf((float)d);
  p.scale_log2 = p.scale * 1.4426950408889634f;
  p.err = device_error_ptr();
  return d == 64 ? launch_bwd_tc<64>(p, batch, seq, nq, nkv, s) : launch_bwd_tc<128>(p, batch, seq, nq, nkv, s);
}

}  // namespace nf4ls
