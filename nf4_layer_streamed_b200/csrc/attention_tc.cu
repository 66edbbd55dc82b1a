// K10 forward on the 5th-generation tensor cores: causal grouped-query attention
// softmax(q k^T / sqrt(d) + causal mask) v for head_dim 128 and seq <= 512 (a
// multiple of 128), the shapes of the Llama-8B layer ("Soup layer-streamed NF4 gate
// record" §2.1: the HF Llama layer body; the workloads' seq 512).
//
// One CTA per (128-query tile, query head, sequence).  Because a query row meets at
// most 512 keys, the whole row of scores fits in TMEM (128 lanes x 512 fp32 columns),
// so the softmax is exact in two passes over TMEM and needs no running rescale:
//   1. TMA brings the Q tile and every key tile at or before the diagonal (128-byte
//      swizzle, head dim in two 64-element atoms); one thread issues
//      S[:, 128 kt ..] = Q K_kt^T (tcgen05.mma, M = N = 128, K = 16 steps) into TMEM.
//   2. Sixteen warps, four per TMEM lane quarter (thread = query row = TMEM lane),
//      warp group g taking key block g: the block's row maximum (causal mask on the
//      diagonal block), combined across the groups through shared memory; then
//      p = 2^(s log2e / sqrt(d) - max), summed in fp32 and written as bf16 into the
//      freed key-tile memory in the MMA's K-major layout, each finished block of P
//      handed to the MMA thread.
//   3. O = sum_kt P_kt V_kt accumulates in TMEM columns [0, 128) (the first block of
//      S, already read), with V_kt N-major from a two-deep TMA ring.
//   4. Group g scales O's columns [32 g, 32 g + 32) by 1 / sum and stores them as
//      bf16; group 0 writes the log-sum-exp.
// P is rounded to bf16 for the P V product, as in the mma.sync kernel; the results
// match that kernel up to summation order.  Every mbarrier wait is bounded.
#include "common.cuh"
#include "internal.h"

namespace nf4ls {

namespace {

constexpr int TT = 128;                 // query / key tile
constexpr int TILE_BYTES = TT * 128 * 2;  // 128 rows x 128 dims bf16 = 32 KB
constexpr int ATOM = TILE_BYTES / 2;      // one 64-dim (or 64-key) swizzle atom: 16 KB
constexpr int MAX_KT = 4;                 // seq <= 512
// shared memory: Q | K tiles 0..3 (then P blocks) | V ring of 2 | barriers
constexpr int OFF_Q = 0, OFF_K = TILE_BYTES, OFF_V = OFF_K + MAX_KT * TILE_BYTES;
constexpr int OFF_BAR = OFF_V + 2 * TILE_BYTES;
constexpr int SMEM_TC = 1024 + OFF_BAR + 256;

struct AttnTcParams {
  CUtensorMap tq, tk, tv;  // [rows, cols] bf16, box 64 cols x 128 rows, 128-byte swizzle
  __nv_bfloat16* o;
  float* lse;
  int ldo, seq, nq, nkv;
  float scale_log2;
  int* err;
};

constexpr int SOFT_WARPS = 16;
constexpr int PROD_WARP = SOFT_WARPS, MMA_WARP = SOFT_WARPS + 1, THREADS_TC = 32 * (SOFT_WARPS + 2);

__device__ __forceinline__ void bar_soft() {
  asm volatile("bar.sync 1, %0;" ::"n"(32 * SOFT_WARPS) : "memory");
}

__global__ void __launch_bounds__(THREADS_TC, 1) k_attn_fwd_tc(const __grid_constant__ AttnTcParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(base + OFF_BAR);
  uint64_t* q_full = bars;                // 1
  uint64_t* k_full = bars + 1;            // MAX_KT
  uint64_t* v_full = k_full + MAX_KT;     // 2
  uint64_t* v_empty = v_full + 2;         // 2
  uint64_t* s_full = v_empty + 2;         // 1
  uint64_t* p_full = s_full + 1;          // MAX_KT
  uint64_t* o_full = p_full + MAX_KT;     // 1
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(o_full + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  volatile int* go = abort_flag + 1;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int qt = gridDim.x - 1 - blockIdx.x;  // longest rows first
  const int h = blockIdx.y, b = blockIdx.z;
  const int kvh = h / (p.nq / p.nkv);
  const int nk = qt + 1;                      // key tiles at or before the diagonal
  const int row0 = b * p.seq;

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    for (int i = 0; i < MAX_KT; ++i) {
      mbar_init(&k_full[i], 1);
      mbar_init(&p_full[i], 4);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&v_full[i], 1);
      mbar_init(&v_empty[i], 1);
    }
    mbar_init(s_full, 1);
    mbar_init(o_full, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == MMA_WARP) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == PROD_WARP) {
    // ------------------------------------------------------------------ TMA producer
    if (lane == 0) {
      tma_prefetch_desc(&p.tq);
      tma_prefetch_desc(&p.tk);
      tma_prefetch_desc(&p.tv);
      mbar_arrive_expect_tx(q_full, TILE_BYTES);
      for (int j = 0; j < 2; ++j) tma_load_2d(base + OFF_Q + j * ATOM, &p.tq, q_full, h * 128 + 64 * j, row0 + qt * TT);
      for (int kt = 0; kt < nk; ++kt) {
        mbar_arrive_expect_tx(&k_full[kt], TILE_BYTES);
        for (int j = 0; j < 2; ++j)
          tma_load_2d(base + OFF_K + kt * TILE_BYTES + j * ATOM, &p.tk, &k_full[kt], kvh * 128 + 64 * j, row0 + kt * TT);
      }
      for (int kt = 0; kt < nk; ++kt) {
        const int vb = kt & 1;
        if (kt >= 2 && !mbar_wait(&v_empty[vb], 0, abort_flag, p.err, KID_ATTN, 21)) break;
        mbar_arrive_expect_tx(&v_full[vb], TILE_BYTES);
        for (int j = 0; j < 2; ++j)
          tma_load_2d(base + OFF_V + vb * TILE_BYTES + j * ATOM, &p.tv, &v_full[vb], kvh * 128 + 64 * j, row0 + kt * TT);
      }
    }
  } else if (warp == MMA_WARP) {
    // ------------------------------------------------------------------ MMA issuer
    constexpr uint32_t idesc_s = idesc_bf16(128, 128, false);  // Q K^T: both K-major
    constexpr uint32_t idesc_o = idesc_bf16(128, 128, true);   // P V: V N-major
    const uint32_t sQ = smem_u32(base + OFF_Q);
    bool ok = mbar_wait(q_full, 0, abort_flag, p.err, KID_ATTN, 22);
    for (int kt = 0; ok && kt < nk; ++kt) {
      if (!(ok = mbar_wait(&k_full[kt], 0, abort_flag, p.err, KID_ATTN, 23))) break;
      tc_fence_after();
      if (lane == 0) {
        const uint32_t sK = smem_u32(base + OFF_K + kt * TILE_BYTES);
#pragma unroll
        for (int ks = 0; ks < 8; ++ks) {
          const uint32_t off = (ks >> 2) * ATOM + (ks & 3) * 32;
          umma_bf16(tmem + kt * 128, sdesc_sw128(sQ + off, 16, 1024), sdesc_sw128(sK + off, 16, 1024), idesc_s,
                    ks ? 1u : 0u);
        }
      }
      __syncwarp();
    }
    if (ok && lane == 0) umma_commit(s_full);
    __syncwarp();
    for (int kt = 0; ok && kt < nk; ++kt) {
      const int vb = kt & 1;
      if (!(ok = mbar_wait(&p_full[kt], 0, abort_flag, p.err, KID_ATTN, 24))) break;
      if (!(ok = mbar_wait(&v_full[vb], (kt >> 1) & 1, abort_flag, p.err, KID_ATTN, 25))) break;
      tc_fence_after();
      if (lane == 0) {
        const uint32_t sP = smem_u32(base + OFF_K + kt * TILE_BYTES);
        const uint32_t sV = smem_u32(base + OFF_V + vb * TILE_BYTES);
#pragma unroll
        for (int ks = 0; ks < 8; ++ks) {
          const uint64_t a = sdesc_sw128(sP + (ks >> 2) * ATOM + (ks & 3) * 32, 16, 1024);
          const uint64_t bv = sdesc_sw128(sV + ks * 2048, ATOM, 1024);  // 16 keys x 128 dims, two 64-dim atoms
          umma_bf16(tmem, a, bv, idesc_o, (kt | ks) ? 1u : 0u);
        }
        umma_commit(&v_empty[vb]);
      }
      __syncwarp();
    }
    if (ok && lane == 0) umma_commit(o_full);
    __syncwarp();
  } else {
    // ------------------------------------------------------------------ softmax + epilogue
    const int g = warp >> 2, wq = warp & 3;         // key block of this warp group; lane quarter
    const int r = wq * 32 + lane;                   // query row in the tile = TMEM lane
    const int qpos = qt * TT + r;                   // position in the sequence
    const uint32_t trow = tmem + ((uint32_t)(wq * 32) << 16);
    // the Q tile is free once S is complete: per-group row maxima and sums
    float* red_max = reinterpret_cast<float*>(base + OFF_Q);
    float* red_sum = red_max + 4 * TT;
    mbar_wait(s_full, 0, abort_flag, p.err, KID_ATTN, 26);
    // every softmax thread reaches each barrier below the same number of times: they
    // agree here, through shared memory, on whether the run goes on
    bar_soft();
    if (threadIdx.x == 0) *go = *abort_flag ? 0 : 1;
    bar_soft();
    if (*go) {
      tc_fence_after();
      const bool mine = g < nk;
      float mx = -INFINITY;
      if (mine) {
        for (int h2 = 0; h2 < 2; ++h2) {  // 64 columns per TMEM round trip
          uint32_t v[2][32];
          tmem_ld32(trow + g * 128 + h2 * 64, v[0]);
          tmem_ld32(trow + g * 128 + h2 * 64 + 32, v[1]);
          tmem_wait_ld();
#pragma unroll
          for (int j = 0; j < 2; ++j)
#pragma unroll
            for (int i = 0; i < 32; ++i) {
              const int key = g * TT + h2 * 64 + j * 32 + i;
              if (key <= qpos) mx = fmaxf(mx, __uint_as_float(v[j][i]) * p.scale_log2);
            }
        }
      }
      red_max[g * TT + r] = mx;
      bar_soft();
      mx = fmaxf(fmaxf(red_max[r], red_max[TT + r]), fmaxf(red_max[2 * TT + r], red_max[3 * TT + r]));
      float sum = 0.f;
      if (mine) {
        const uint32_t sP = smem_u32(base + OFF_K + g * TILE_BYTES);
        for (int h2 = 0; h2 < 2; ++h2) {
          uint32_t v[2][32];
          tmem_ld32(trow + g * 128 + h2 * 64, v[0]);
          tmem_ld32(trow + g * 128 + h2 * 64 + 32, v[1]);
          tmem_wait_ld();
#pragma unroll
          for (int j = 0; j < 2; ++j) {
            const int c = h2 * 2 + j;  // 32-key chunk of the block
            float pv[32];
#pragma unroll
            for (int i = 0; i < 32; ++i) {
              const int key = g * TT + c * 32 + i;
              const float e = key <= qpos ? exp2f(__uint_as_float(v[j][i]) * p.scale_log2 - mx) : 0.f;
              pv[i] = e;
              sum += e;
            }
            // keys c*32 .. c*32+31: atom c/2, 16-byte chunks (c%2)*4 .. +3, 128-byte swizzle
#pragma unroll
            for (int q4 = 0; q4 < 4; ++q4) {
              const int chunk = (c & 1) * 4 + q4;
              const uint32_t addr = sP + (c >> 1) * ATOM + r * 128 + ((uint32_t)(chunk ^ (r & 7)) << 4);
              st_shared_v4(addr, pack_bf16x2(pv[8 * q4], pv[8 * q4 + 1]), pack_bf16x2(pv[8 * q4 + 2], pv[8 * q4 + 3]),
                           pack_bf16x2(pv[8 * q4 + 4], pv[8 * q4 + 5]), pack_bf16x2(pv[8 * q4 + 6], pv[8 * q4 + 7]));
            }
          }
        }
        fence_proxy_async_smem();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&p_full[g]);
      }
      red_sum[g * TT + r] = sum;
      bar_soft();
      sum = (red_sum[r] + red_sum[TT + r]) + (red_sum[2 * TT + r] + red_sum[3 * TT + r]);
      if (mbar_wait(o_full, 0, abort_flag, p.err, KID_ATTN, 27)) {
        tc_fence_after();
        const float inv = 1.0f / sum;
        uint32_t v[32];
        tmem_ld32(trow + g * 32, v);  // output columns 32 g .. 32 g + 31
        tmem_wait_ld();
        uint4* dst = reinterpret_cast<uint4*>(p.o + (size_t)(row0 + qpos) * p.ldo + h * 128 + g * 32);
#pragma unroll
        for (int q4 = 0; q4 < 4; ++q4)
          dst[q4] = make_uint4(pack_bf16x2(__uint_as_float(v[8 * q4]) * inv, __uint_as_float(v[8 * q4 + 1]) * inv),
                               pack_bf16x2(__uint_as_float(v[8 * q4 + 2]) * inv, __uint_as_float(v[8 * q4 + 3]) * inv),
                               pack_bf16x2(__uint_as_float(v[8 * q4 + 4]) * inv, __uint_as_float(v[8 * q4 + 5]) * inv),
                               pack_bf16x2(__uint_as_float(v[8 * q4 + 6]) * inv, __uint_as_float(v[8 * q4 + 7]) * inv));
        if (g == 0) p.lse[((size_t)b * p.nq + h) * p.seq + qpos] = (mx + log2f(sum)) * 0.6931471805599453f;
      }
    }
  }

  // On an aborted run the MMAs already issued must finish before TMEM is freed.
  if (warp == MMA_WARP && *abort_flag) mbar_wait_drain(o_full, 0);
  tc_fence_before();
  __syncthreads();
  if (warp == MMA_WARP) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// ------------------------------------------------------------------------------ backward
// dK, dV (per key tile) and dQ (per query tile) on tcgen05, the same blocks as the
// mma.sync backward: for a 128-query x 128-key block, S = Q K^T and dP = dO V^T in TMEM,
// P = 2^(S log2e / sqrt(d) - lse log2e) (causal mask), dS = P (dP - delta); then
//   key side:   dV += P^T dO,  dK += dS^T Q   (both transposed: the rows are keys)
//   query side: dQ += dS K.
// P^T / dS^T (resp. dS) are written back as bf16 into the TMEM columns of the scores
// they came from and feed the next MMAs as their A operand from TMEM (two bf16 per
// 32-bit column); the Q, dO, K and V tiles serve as K-major operands of the score
// products and as N-major operands of the accumulating products, from the same
// shared memory.  Sixteen warps handle a block (four per TMEM lane quarter, 32
// columns each); a named barrier separates reading the scores from overwriting them.
// Accumulation runs in a fixed order (query head, then query tile), so results are
// bit-reproducible.

__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
      "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]),
      "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15])
      : "memory");
}
__device__ __forceinline__ void tmem_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

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

// 1D bulk copy global -> shared completing transaction bytes on bar (16-byte multiples).
__device__ __forceinline__ void bulk_load(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
  asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
                   smem_u32(dst)),
               "l"(src), "r"(bytes), "r"(smem_u32(bar))
               : "memory");
}

struct AttnBwdParams {
  CUtensorMap tq, tk, tv, tdo;  // box 64 cols x 128 rows, 128-byte swizzle
  const float* lse;
  const float* delta;
  __nv_bfloat16* dq;
  __nv_bfloat16* dk;
  __nv_bfloat16* dv;
  int ld_dq, ld_dkv, seq, nq, nkv;
  float scale, scale_log2;
  int* err;
};

constexpr int B_OFF_A = 0;                              // K, V (key side) or Q, dO (query side)
constexpr int B_OFF_RING = 2 * TILE_BYTES;              // 2 buffers x (two 32 KB tiles)
constexpr int B_OFF_LD = B_OFF_RING + 4 * TILE_BYTES;   // 2 buffers x (128 lse + 128 delta floats)
constexpr int B_OFF_BAR = B_OFF_LD + 2 * 1024;
constexpr int SMEM_BWD = 1024 + B_OFF_BAR + 256;

// Reads this thread's 32 scores and 32 dP values (columns 32 g ..) of its TMEM lane,
// returns them as float.
__device__ __forceinline__ void ld_scores(uint32_t trow, int g, float (&sv)[32], float (&dpv)[32]) {
  uint32_t a[32], c[32];
  tmem_ld32(trow + g * 32, a);
  tmem_ld32(trow + 128 + g * 32, c);
  tmem_wait_ld();
#pragma unroll
  for (int i = 0; i < 32; ++i) {
    sv[i] = __uint_as_float(a[i]);
    dpv[i] = __uint_as_float(c[i]);
  }
}

// KEY side: dK, dV of one 128-key tile of one kv head.
__global__ void __launch_bounds__(THREADS_TC, 1) k_attn_dkv_tc(const __grid_constant__ AttnBwdParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(base + B_OFF_BAR);
  uint64_t* kv_full = bars;         // 1
  uint64_t* qd_full = bars + 1;     // 2
  uint64_t* qd_empty = bars + 3;    // 2
  uint64_t* sd_full = bars + 5;     // 1 (phase per item)
  uint64_t* p_full = bars + 6;      // 1 (phase per item)
  uint64_t* acc_full = bars + 7;    // 1
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 8);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  volatile int* go = abort_flag + 1;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int kvh = blockIdx.x, b = blockIdx.y, kt = blockIdx.z;  // z slowest: the longest key tiles first
  const int grp = p.nq / p.nkv, n_qt = p.seq / TT;
  const int per_head = n_qt - kt, n_it = grp * per_head;
  const int row0 = b * p.seq;

  if (threadIdx.x == 0) {
    mbar_init(kv_full, 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(&qd_full[i], 1);
      mbar_init(&qd_empty[i], 1);
    }
    mbar_init(sd_full, 1);
    mbar_init(p_full, SOFT_WARPS);
    mbar_init(acc_full, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == MMA_WARP) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;  // [0,128) S^T, [128,256) dP^T, [256,384) dV, [384,512) dK

  if (warp == PROD_WARP) {
    if (lane == 0) {
      tma_prefetch_desc(&p.tq);
      tma_prefetch_desc(&p.tk);
      tma_prefetch_desc(&p.tv);
      tma_prefetch_desc(&p.tdo);
      mbar_arrive_expect_tx(kv_full, 2 * TILE_BYTES);
      for (int j = 0; j < 2; ++j) {
        tma_load_2d(base + B_OFF_A + j * ATOM, &p.tk, kv_full, kvh * 128 + 64 * j, row0 + kt * TT);
        tma_load_2d(base + B_OFF_A + TILE_BYTES + j * ATOM, &p.tv, kv_full, kvh * 128 + 64 * j, row0 + kt * TT);
      }
      for (int it = 0; it < n_it; ++it) {
        const int bf = it & 1;
        if (it >= 2 && !mbar_wait(&qd_empty[bf], ((it >> 1) - 1) & 1, abort_flag, p.err, KID_ATTN, 31)) break;
        const int h = kvh * grp + it / per_head, qt = kt + it % per_head;
        uint8_t* buf = base + B_OFF_RING + bf * 2 * TILE_BYTES;
        float* ld = reinterpret_cast<float*>(base + B_OFF_LD + bf * 1024);
        mbar_arrive_expect_tx(&qd_full[bf], 2 * TILE_BYTES + 1024);
        for (int j = 0; j < 2; ++j) {
          tma_load_2d(buf + j * ATOM, &p.tq, &qd_full[bf], h * 128 + 64 * j, row0 + qt * TT);
          tma_load_2d(buf + TILE_BYTES + j * ATOM, &p.tdo, &qd_full[bf], h * 128 + 64 * j, row0 + qt * TT);
        }
        const size_t lo = ((size_t)b * p.nq + h) * p.seq + qt * TT;
        bulk_load(ld, p.lse + lo, 512, &qd_full[bf]);
        bulk_load(ld + 128, p.delta + lo, 512, &qd_full[bf]);
      }
    }
  } else if (warp == MMA_WARP) {
    constexpr uint32_t idesc_s = idesc_bf16(128, 128, false);
    constexpr uint32_t idesc_a = idesc_bf16(128, 128, true);
    const uint32_t sK = smem_u32(base + B_OFF_A), sV = sK + TILE_BYTES;
    bool ok = mbar_wait(kv_full, 0, abort_flag, p.err, KID_ATTN, 32);
    for (int it = 0; ok && it < n_it; ++it) {
      const int bf = it & 1;
      if (!(ok = mbar_wait(&qd_full[bf], (it >> 1) & 1, abort_flag, p.err, KID_ATTN, 33))) break;
      tc_fence_after();
      const uint32_t sQ = smem_u32(base + B_OFF_RING + bf * 2 * TILE_BYTES), sO = sQ + TILE_BYTES;
      if (lane == 0) {
#pragma unroll
        for (int ks = 0; ks < 8; ++ks) {  // S^T = K Q^T, dP^T = V dO^T over the head dim
          const uint32_t off = (ks >> 2) * ATOM + (ks & 3) * 32;
          umma_bf16(tmem, sdesc_sw128(sK + off, 16, 1024), sdesc_sw128(sQ + off, 16, 1024), idesc_s, ks ? 1u : 0u);
          umma_bf16(tmem + 128, sdesc_sw128(sV + off, 16, 1024), sdesc_sw128(sO + off, 16, 1024), idesc_s,
                    ks ? 1u : 0u);
        }
        umma_commit(sd_full);
      }
      __syncwarp();
      if (!(ok = mbar_wait(p_full, it & 1, abort_flag, p.err, KID_ATTN, 34))) break;
      tc_fence_after();
      if (lane == 0) {
#pragma unroll
        for (int ks = 0; ks < 8; ++ks) {  // over the 128 queries, 16 at a time
          const uint32_t acc = (it | ks) ? 1u : 0u;
          umma_bf16_ta(tmem + 256, tmem + ks * 8, sdesc_sw128(sO + ks * 2048, ATOM, 1024), idesc_a, acc);
          umma_bf16_ta(tmem + 384, tmem + 128 + ks * 8, sdesc_sw128(sQ + ks * 2048, ATOM, 1024), idesc_a, acc);
        }
        umma_commit(&qd_empty[bf]);
      }
      __syncwarp();
    }
    if (ok && lane == 0) umma_commit(acc_full);
    __syncwarp();
  } else {
    const int g = warp >> 2, wq = warp & 3;
    const int r = wq * 32 + lane;  // key row = TMEM lane
    const int key = kt * TT + r;
    const uint32_t trow = tmem + ((uint32_t)(wq * 32) << 16);
    bool ok = true;
    for (int it = 0; it < n_it; ++it) {
      const int bf = it & 1, qt = kt + it % per_head;
      const float* ld = reinterpret_cast<const float*>(base + B_OFF_LD + bf * 1024);
      ok = mbar_wait(sd_full, it & 1, abort_flag, p.err, KID_ATTN, 35);
      bar_soft();
      if (threadIdx.x == 0) *go = (ok && !*abort_flag) ? 1 : 0;
      bar_soft();
      if (!*go) {
        ok = false;
        break;
      }
      tc_fence_after();
      float sv[32], dpv[32];
      ld_scores(trow, g, sv, dpv);
      uint32_t pp[16], dd[16];
#pragma unroll
      for (int j = 0; j < 16; ++j) {
        float pv2[2], ds2[2];
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          const int qi = g * 32 + 2 * j + e;  // query within the tile
          const float pe = key <= qt * TT + qi ? exp2f(sv[2 * j + e] * p.scale_log2 - ld[qi] * 1.4426950408889634f) : 0.f;
          pv2[e] = pe;
          ds2[e] = pe * (dpv[2 * j + e] - ld[128 + qi]);
        }
        pp[j] = pack_bf16x2(pv2[0], pv2[1]);
        dd[j] = pack_bf16x2(ds2[0], ds2[1]);
      }
      tc_fence_before();
      bar_soft();  // every warp has read its scores before any overwrites them
      tc_fence_after();
      tmem_st16(trow + g * 16, pp);
      tmem_st16(trow + 128 + g * 16, dd);
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(p_full);
    }
    if (ok && mbar_wait(acc_full, 0, abort_flag, p.err, KID_ATTN, 36)) {
      tc_fence_after();
      uint32_t v[32], k[32];
      tmem_ld32(trow + 256 + g * 32, v);
      tmem_ld32(trow + 384 + g * 32, k);
      tmem_wait_ld();
      uint4* dv = reinterpret_cast<uint4*>(p.dv + (size_t)(row0 + key) * p.ld_dkv + kvh * 128 + g * 32);
      uint4* dk = reinterpret_cast<uint4*>(p.dk + (size_t)(row0 + key) * p.ld_dkv + kvh * 128 + g * 32);
      const float sc = p.scale;
#pragma unroll
      for (int q4 = 0; q4 < 4; ++q4) {
        dv[q4] = make_uint4(pack_bf16x2(__uint_as_float(v[8 * q4]), __uint_as_float(v[8 * q4 + 1])),
                            pack_bf16x2(__uint_as_float(v[8 * q4 + 2]), __uint_as_float(v[8 * q4 + 3])),
                            pack_bf16x2(__uint_as_float(v[8 * q4 + 4]), __uint_as_float(v[8 * q4 + 5])),
                            pack_bf16x2(__uint_as_float(v[8 * q4 + 6]), __uint_as_float(v[8 * q4 + 7])));
        dk[q4] = make_uint4(pack_bf16x2(__uint_as_float(k[8 * q4]) * sc, __uint_as_float(k[8 * q4 + 1]) * sc),
                            pack_bf16x2(__uint_as_float(k[8 * q4 + 2]) * sc, __uint_as_float(k[8 * q4 + 3]) * sc),
                            pack_bf16x2(__uint_as_float(k[8 * q4 + 4]) * sc, __uint_as_float(k[8 * q4 + 5]) * sc),
                            pack_bf16x2(__uint_as_float(k[8 * q4 + 6]) * sc, __uint_as_float(k[8 * q4 + 7]) * sc));
      }
    }
  }
  if (warp == MMA_WARP && *abort_flag) mbar_wait_drain(acc_full, 0);
  tc_fence_before();
  __syncthreads();
  if (warp == MMA_WARP) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// QUERY side: dQ of one 128-query tile of one query head.
__global__ void __launch_bounds__(THREADS_TC, 1) k_attn_dq_tc(const __grid_constant__ AttnBwdParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(base + B_OFF_BAR);
  uint64_t* q_full = bars;          // 1 (Q, dO, lse, delta)
  uint64_t* kv_full = bars + 1;     // 2
  uint64_t* kv_empty = bars + 3;    // 2
  uint64_t* sd_full = bars + 5;     // 1
  uint64_t* p_full = bars + 6;      // 1
  uint64_t* acc_full = bars + 7;    // 1
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 8);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  volatile int* go = abort_flag + 1;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int qt = gridDim.x - 1 - blockIdx.x, h = blockIdx.y, b = blockIdx.z;  // longest rows first
  const int kvh = h / (p.nq / p.nkv);
  const int n_it = qt + 1;  // key tiles at or before the diagonal
  const int row0 = b * p.seq;

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(&kv_full[i], 1);
      mbar_init(&kv_empty[i], 1);
    }
    mbar_init(sd_full, 1);
    mbar_init(p_full, SOFT_WARPS);
    mbar_init(acc_full, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == MMA_WARP) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;  // [0,128) S, [128,256) dP, [256,384) dQ

  if (warp == PROD_WARP) {
    if (lane == 0) {
      tma_prefetch_desc(&p.tq);
      tma_prefetch_desc(&p.tk);
      tma_prefetch_desc(&p.tv);
      tma_prefetch_desc(&p.tdo);
      float* ld = reinterpret_cast<float*>(base + B_OFF_LD);
      mbar_arrive_expect_tx(q_full, 2 * TILE_BYTES + 1024);
      for (int j = 0; j < 2; ++j) {
        tma_load_2d(base + B_OFF_A + j * ATOM, &p.tq, q_full, h * 128 + 64 * j, row0 + qt * TT);
        tma_load_2d(base + B_OFF_A + TILE_BYTES + j * ATOM, &p.tdo, q_full, h * 128 + 64 * j, row0 + qt * TT);
      }
      const size_t lo = ((size_t)b * p.nq + h) * p.seq + qt * TT;
      bulk_load(ld, p.lse + lo, 512, q_full);
      bulk_load(ld + 128, p.delta + lo, 512, q_full);
      for (int it = 0; it < n_it; ++it) {
        const int bf = it & 1;
        if (it >= 2 && !mbar_wait(&kv_empty[bf], ((it >> 1) - 1) & 1, abort_flag, p.err, KID_ATTN, 41)) break;
        uint8_t* buf = base + B_OFF_RING + bf * 2 * TILE_BYTES;
        mbar_arrive_expect_tx(&kv_full[bf], 2 * TILE_BYTES);
        for (int j = 0; j < 2; ++j) {
          tma_load_2d(buf + j * ATOM, &p.tk, &kv_full[bf], kvh * 128 + 64 * j, row0 + it * TT);
          tma_load_2d(buf + TILE_BYTES + j * ATOM, &p.tv, &kv_full[bf], kvh * 128 + 64 * j, row0 + it * TT);
        }
      }
    }
  } else if (warp == MMA_WARP) {
    constexpr uint32_t idesc_s = idesc_bf16(128, 128, false);
    constexpr uint32_t idesc_a = idesc_bf16(128, 128, true);
    const uint32_t sQ = smem_u32(base + B_OFF_A), sO = sQ + TILE_BYTES;
    bool ok = mbar_wait(q_full, 0, abort_flag, p.err, KID_ATTN, 42);
    for (int it = 0; ok && it < n_it; ++it) {
      const int bf = it & 1;
      if (!(ok = mbar_wait(&kv_full[bf], (it >> 1) & 1, abort_flag, p.err, KID_ATTN, 43))) break;
      tc_fence_after();
      const uint32_t sK = smem_u32(base + B_OFF_RING + bf * 2 * TILE_BYTES), sV = sK + TILE_BYTES;
      if (lane == 0) {
#pragma unroll
        for (int ks = 0; ks < 8; ++ks) {  // S = Q K^T, dP = dO V^T over the head dim
          const uint32_t off = (ks >> 2) * ATOM + (ks & 3) * 32;
          umma_bf16(tmem, sdesc_sw128(sQ + off, 16, 1024), sdesc_sw128(sK + off, 16, 1024), idesc_s, ks ? 1u : 0u);
          umma_bf16(tmem + 128, sdesc_sw128(sO + off, 16, 1024), sdesc_sw128(sV + off, 16, 1024), idesc_s,
                    ks ? 1u : 0u);
        }
        umma_commit(sd_full);
      }
      __syncwarp();
      if (!(ok = mbar_wait(p_full, it & 1, abort_flag, p.err, KID_ATTN, 44))) break;
      tc_fence_after();
      if (lane == 0) {
#pragma unroll
        for (int ks = 0; ks < 8; ++ks)  // dQ += dS K over the 128 keys
          umma_bf16_ta(tmem + 256, tmem + 128 + ks * 8, sdesc_sw128(sK + ks * 2048, ATOM, 1024), idesc_a,
                       (it | ks) ? 1u : 0u);
        umma_commit(&kv_empty[bf]);
      }
      __syncwarp();
    }
    if (ok && lane == 0) umma_commit(acc_full);
    __syncwarp();
  } else {
    const int g = warp >> 2, wq = warp & 3;
    const int r = wq * 32 + lane;  // query row = TMEM lane
    const int qpos = qt * TT + r;
    const uint32_t trow = tmem + ((uint32_t)(wq * 32) << 16);
    const float* ld = reinterpret_cast<const float*>(base + B_OFF_LD);
    bool ok = mbar_wait(q_full, 0, abort_flag, p.err, KID_ATTN, 45);
    const float lse2 = ok ? ld[r] * 1.4426950408889634f : 0.f, dl = ok ? ld[128 + r] : 0.f;
    for (int it = 0; it < n_it; ++it) {
      ok = mbar_wait(sd_full, it & 1, abort_flag, p.err, KID_ATTN, 46);
      bar_soft();
      if (threadIdx.x == 0) *go = (ok && !*abort_flag) ? 1 : 0;
      bar_soft();
      if (!*go) {
        ok = false;
        break;
      }
      tc_fence_after();
      float sv[32], dpv[32];
      ld_scores(trow, g, sv, dpv);
      uint32_t dd[16];
#pragma unroll
      for (int j = 0; j < 16; ++j) {
        float ds2[2];
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          const int kj = it * TT + g * 32 + 2 * j + e;  // key position
          const float pe = kj <= qpos ? exp2f(sv[2 * j + e] * p.scale_log2 - lse2) : 0.f;
          ds2[e] = pe * (dpv[2 * j + e] - dl);
        }
        dd[j] = pack_bf16x2(ds2[0], ds2[1]);
      }
      tc_fence_before();
      bar_soft();  // every warp has read its scores before any overwrites them
      tc_fence_after();
      tmem_st16(trow + 128 + g * 16, dd);
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(p_full);
    }
    if (ok && mbar_wait(acc_full, 0, abort_flag, p.err, KID_ATTN, 47)) {
      tc_fence_after();
      uint32_t v[32];
      tmem_ld32(trow + 256 + g * 32, v);
      tmem_wait_ld();
      uint4* dst = reinterpret_cast<uint4*>(p.dq + (size_t)(row0 + qpos) * p.ld_dq + h * 128 + g * 32);
      const float sc = p.scale;
#pragma unroll
      for (int q4 = 0; q4 < 4; ++q4)
        dst[q4] = make_uint4(pack_bf16x2(__uint_as_float(v[8 * q4]) * sc, __uint_as_float(v[8 * q4 + 1]) * sc),
                             pack_bf16x2(__uint_as_float(v[8 * q4 + 2]) * sc, __uint_as_float(v[8 * q4 + 3]) * sc),
                             pack_bf16x2(__uint_as_float(v[8 * q4 + 4]) * sc, __uint_as_float(v[8 * q4 + 5]) * sc),
                             pack_bf16x2(__uint_as_float(v[8 * q4 + 6]) * sc, __uint_as_float(v[8 * q4 + 7]) * sc));
    }
  }
  if (warp == MMA_WARP && *abort_flag) mbar_wait_drain(acc_full, 0);
  tc_fence_before();
  __syncthreads();
  if (warp == MMA_WARP) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

}  // namespace

bool attention_fwd_tc_supported(int seq, int d, int nq, int nkv, int ldq, int ldkv, int ldo) {
  return d == 128 && seq % TT == 0 && seq <= MAX_KT * TT && nq % nkv == 0 && ldq % 8 == 0 && ldkv % 8 == 0 &&
         ldo % 8 == 0;
}

int attention_fwd_tc(const __nv_bfloat16* q, const __nv_bfloat16* k, const __nv_bfloat16* v, int ldq, int ldkv,
                     __nv_bfloat16* o, int ldo, float* lse, int batch, int seq, int nq, int nkv, cudaStream_t s) {
  static_assert(SMEM_TC <= 232448, "shared memory of the tcgen05 attention");
  AttnTcParams p;
  const uint64_t rows = (uint64_t)batch * seq;
  NF4_TRY(tma_map_bf16(&p.tq, q, (uint64_t)nq * 128, rows, (uint64_t)ldq * 2, 64, TT));
  NF4_TRY(tma_map_bf16(&p.tk, k, (uint64_t)nkv * 128, rows, (uint64_t)ldkv * 2, 64, TT));
  NF4_TRY(tma_map_bf16(&p.tv, v, (uint64_t)nkv * 128, rows, (uint64_t)ldkv * 2, 64, TT));
  p.o = o;
  p.lse = lse;
  p.ldo = ldo;
  p.seq = seq;
  p.nq = nq;
  p.nkv = nkv;
  p.scale_log2 = (1.0f / sqrtf(128.0f)) * 1.4426950408889634f;
  p.err = device_error_ptr();
  static int configured[16] = {0};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 16 && !configured[dev]) {
    NF4_CUDA_TRY(cudaFuncSetAttribute(k_attn_fwd_tc, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_TC));
    configured[dev] = 1;
  }
  k_attn_fwd_tc<<<dim3(seq / TT, nq, batch), THREADS_TC, SMEM_TC, s>>>(p);
  note_launch();
  NF4_CUDA_TRY(cudaGetLastError());
  return NF4LS_OK;
}

}  // namespace nf4ls

namespace nf4ls {

int attention_bwd_tc(const __nv_bfloat16* q, const __nv_bfloat16* k, const __nv_bfloat16* v, int ldq, int ldkv,
                     const __nv_bfloat16* dout, int ldo, const float* lse, const float* delta, __nv_bfloat16* dq,
                     __nv_bfloat16* dk, __nv_bfloat16* dv, int ld_dq, int ld_dkv, int batch, int seq, int nq, int nkv,
                     cudaStream_t s) {
  static_assert(SMEM_BWD <= 232448, "shared memory of the tcgen05 attention backward");
  AttnBwdParams p;
  const uint64_t rows = (uint64_t)batch * seq;
  NF4_TRY(tma_map_bf16(&p.tq, q, (uint64_t)nq * 128, rows, (uint64_t)ldq * 2, 64, TT));
  NF4_TRY(tma_map_bf16(&p.tk, k, (uint64_t)nkv * 128, rows, (uint64_t)ldkv * 2, 64, TT));
  NF4_TRY(tma_map_bf16(&p.tv, v, (uint64_t)nkv * 128, rows, (uint64_t)ldkv * 2, 64, TT));
  NF4_TRY(tma_map_bf16(&p.tdo, dout, (uint64_t)nq * 128, rows, (uint64_t)ldo * 2, 64, TT));
  if (!aligned(lse, 16) || !aligned(delta, 16)) return fail(NF4LS_ALIGN, "attention backward: lse / delta alignment");
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
  p.scale = 1.0f / sqrtf(128.0f);
  p.scale_log2 = p.scale * 1.4426950408889634f;
  p.err = device_error_ptr();
  static int configured[16] = {0};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 16 && !configured[dev]) {
    NF4_CUDA_TRY(cudaFuncSetAttribute(k_attn_dq_tc, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_BWD));
    NF4_CUDA_TRY(cudaFuncSetAttribute(k_attn_dkv_tc, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_BWD));
    configured[dev] = 1;
  }
  k_attn_dq_tc<<<dim3(seq / TT, nq, batch), THREADS_TC, SMEM_BWD, s>>>(p);
  note_launch();
  k_attn_dkv_tc<<<dim3(nkv, batch, seq / TT), THREADS_TC, SMEM_BWD, s>>>(p);
  note_launch();
  NF4_CUDA_TRY(cudaGetLastError());
  return NF4LS_OK;
}

}  // namespace nf4ls
