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
