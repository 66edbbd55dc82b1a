// Layer-body and model-end kernels around the tcgen05 GEMMs: RMSNorm forward and
// backward (K8), RoPE tables and the RoPE transpose for dL/dq, dL/dk (K9),
// embedding gather (K13), causal-LM cross-entropy with its gradient (K12), the
// single-layer mean-square loss, and AdamW (K14).
//
// The layer body is the HF Llama decoder layer the pages' system runs
// ("Soup 层流式 NF4 训练实测：在 4 GB 显存上以位级一致标准完成 8B 模型 LoRA 微调", §2.1); LoRA r=16 / alpha=32 on q_proj and v_proj
// trained with AdamW (the SFT configuration of "Soup v0.72.4 技术解析", §4.2).
// All reductions run in a fixed order (no atomics), so every result is
// bit-reproducible from run to run and independent of buffer addresses.
#include <algorithm>
#include <cmath>

#include "common.cuh"
#include "internal.h"

namespace nf4ls {

namespace {

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}
__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
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

// ------------------------------------------------------------------ RMSNorm
// y = bf16(x r w) with r = 1 / sqrt(mean(x^2) + eps);
// dx = resid + r w dy - x r^3 sum(w dy x) / H.
// One block per row: VPT 16-byte vectors per thread, every
// load of the row issued at once and the row kept in registers (one read of x and dy),
// the block's sums added through shared memory in warp order.  Many small blocks keep
// enough loads in flight for HBM.
__device__ __forceinline__ float block_sum(float v, float* red) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = (blockDim.x + 31) >> 5;
  v = warp_sum(v);
  __syncthreads();  // red may still be read from a previous sum
  if (lane == 0) red[warp] = v;
  __syncthreads();
  float a = 0.f;
  for (int i = 0; i < nw; ++i) a += red[i];
  return a;
}

// The adapter's B operands in 16-byte pieces (8 bf16 outputs each), 32-bit indices:
//   bup [qd + 2 kvd, 64]: s B_q in columns 0-15 of the q rows, s B_v in 16-31 of the v rows
//   bqt [16, qd], bvt [16, kvd]: B_q^T, B_v^T
// (the A operand, adn [64, H] = A_q in rows 0-15, A_v in 16-31, zero rows 32-63, is
// written by k_rmsnorm_down from its shared-memory copy of the adapter).
__device__ void pack_piece(const LoraPack& a, int i) {
  const int qd = a.qd, kvd = a.kvd, nq = qd + 2 * kvd;
  float f[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) f[e] = 0.f;
  __nv_bfloat16* dst;
  if (i < nq * 8) {
    const int n = i >> 3, c = (i & 7) * 8;
    const float* src = nullptr;
    if (n < qd && c < 16)
      src = a.Bq + (size_t)n * 16 + c;
    else if (n >= qd + kvd && c >= 16 && c < 32)
      src = a.Bv + (size_t)(n - qd - kvd) * 16 + (c - 16);
    if (src)
#pragma unroll
      for (int e = 0; e < 8; ++e) f[e] = a.scale * __bfloat162float(__float2bfloat16_rn(src[e]));
    dst = a.bup + (size_t)n * 64 + c;
  } else if ((i -= nq * 8) < 2 * qd) {
    const int per = qd / 8, r = i / per, n = (i - r * per) * 8;
#pragma unroll
    for (int e = 0; e < 8; ++e) f[e] = a.Bq[(size_t)(n + e) * 16 + r];
    dst = a.bqt + (size_t)r * qd + n;
  } else {
    i -= 2 * qd;
    const int per = kvd / 8, r = i / per, n = (i - r * per) * 8;
#pragma unroll
    for (int e = 0; e < 8; ++e) f[e] = a.Bv[(size_t)(n + e) * 16 + r];
    dst = a.bvt + (size_t)r * kvd + n;
  }
  *reinterpret_cast<uint4*>(dst) = pack8(f);
}

__host__ __device__ inline int pack_pieces(const LoraPack& a) { return (a.qd + 2 * a.kvd) * 8 + 2 * a.qd + 2 * a.kvd; }

// One block per row.
template <int VPT>
__global__ void __launch_bounds__(1024) k_rmsnorm_fwd_row(const __nv_bfloat16* __restrict__ x,
                                                          const __nv_bfloat16* __restrict__ w,
                                                          __nv_bfloat16* __restrict__ y, int H, float eps) {
  __shared__ float red[32];
  const int row = blockIdx.x, t = threadIdx.x, T = blockDim.x, nv = H / 8;
  const uint4* xr = reinterpret_cast<const uint4*>(x + (size_t)row * H);
  const uint4* wr = reinterpret_cast<const uint4*>(w);
  uint4* yr = reinterpret_cast<uint4*>(y + (size_t)row * H);
  uint4 v[VPT];
#pragma unroll
  for (int j = 0; j < VPT; ++j)
    if (t + j * T < nv) v[j] = xr[t + j * T];
  float ss = 0.f;
#pragma unroll
  for (int j = 0; j < VPT; ++j)
    if (t + j * T < nv) {
      float f[8];
      unpack8(v[j], f);
#pragma unroll
      for (int e = 0; e < 8; ++e) ss += f[e] * f[e];
    }
  ss = block_sum(ss, red);
  const float r = 1.0f / sqrtf(ss / (float)H + eps);
#pragma unroll
  for (int j = 0; j < VPT; ++j) {
    const int i = t + j * T;
    if (i < nv) {
      float f[8], g[8];
      unpack8(v[j], f);
      unpack8(wr[i], g);
#pragma unroll
      for (int e = 0; e < 8; ++e) f[e] = f[e] * r * g[e];
      yr[i] = pack8(f);
    }
  }
}

// The input RMSNorm with the LoRA down-projection as its second output:
//   h1 = bf16(x r w),  t = [h1 A_q^T | h1 A_v^T] (bf16, columns 0-31 of the 64-wide extra
//   operand of the q/k/v GEMM, zeros in 32-63),
// so that h1 is not read back for t.  A cluster of C CTAs takes 64 rows; CTA c of the
// cluster holds the column slice [c S, (c + 1) S) of those rows (S = H / C) in registers
// (a warp per eight rows, 512 contiguous bytes per load) and the same slice of the 32
// adapter rows, rounded to bf16, in shared memory.  The fp32 adapter slice arrives by 32
// bulk copies into the h1 buffer (free until h1 is written) while the rows load.  The
// rows' sums of squares are partial per CTA; every CTA stores its partials into every
// CTA's shared memory (distributed shared memory) and adds the C partials of each row in
// CTA order.  Between the two halves of that cluster barrier each CTA converts its
// adapter slice and does its share of the adapter's B operands (pack_piece).  Each CTA
// then writes its slice of h1 and forms the partial t of its slice on mma.sync m16n8k16
// (warp w: row tile w % 4, k-steps w / 4, w / 4 + 2, ..); the warp partials are added in
// k order and stored into the CTA that owns the rows (CTA c: rows 64 c / C ...), which
// adds the cluster's C partials in CTA order.  Only stores cross CTAs, each before a
// cluster barrier, so no CTA waits for another at the end.
constexpr int ND_R = 64, ND_THREADS = 256;  // rows per cluster, threads per CTA (eight rows per warp)

struct NormDownShape {
  int C, S;  // cluster size, slice width
  size_t smem;
};
inline NormDownShape norm_down_shape(int H) {
  NormDownShape sh{0, 0, 0};
  for (int c : {8, 4, 2, 1})
    if (H % (16 * c) == 0 && H / c <= 1024) {
      sh.C = c;
      sh.S = H / c;
      break;
    }
  if (sh.C) {
    const size_t hs = (size_t)ND_R * (sh.S + 8) * 2, as = (size_t)32 * (sh.S + 8) * 2;
    // + every CTA's partial sums of squares [8][64], the mbarrier of the adapter copies and
    // the abort flag of its wait
    sh.smem = hs + std::max(as, (size_t)ND_THREADS / 32 * 16 * 32 * 4) + (size_t)ND_R * 32 * 4 + 8 * ND_R * 4 + 16;
  }
  return sh;
}

template <int NH>
__global__ void __launch_bounds__(ND_THREADS, 2) k_rmsnorm_down(const __nv_bfloat16* __restrict__ x,
                                                             const __nv_bfloat16* __restrict__ w,
                                                             __nv_bfloat16* __restrict__ y, int M, int H, int S,
                                                             float eps, const LoraPack pack,
                                                             __nv_bfloat16* __restrict__ tpad, int* err) {
  extern __shared__ __align__(16) uint8_t smem[];
  const int t = threadIdx.x, warp = t >> 5, lane = t & 31, ls = S + 8, nv = S / 8;
  const int C = (int)(gridDim.y), c = (int)cluster_ctarank(), m0 = blockIdx.x * ND_R, col0 = c * S;
  __nv_bfloat16* hs = reinterpret_cast<__nv_bfloat16*>(smem);                 // [64][S + 8] h1 slice
  float* stage = reinterpret_cast<float*>(smem);                              // before h1: [32][S] fp32 adapter slice
  __nv_bfloat16* as = hs + (size_t)ND_R * ls;                                  // [32][S + 8] adapter slice
  float* red = reinterpret_cast<float*>(as);                                   // after the products: [8][16][32]
  const size_t as_bytes = std::max((size_t)32 * ls * 2, (size_t)ND_THREADS / 32 * 16 * 32 * 4);
  float* Pin = reinterpret_cast<float*>(reinterpret_cast<uint8_t*>(as) + as_bytes);  // [C][64 / C][32] t partials
  float* ssall = Pin + ND_R * 32;                                              // [C][64] partial sums of squares
  uint64_t* abar = reinterpret_cast<uint64_t*>(ssall + 8 * ND_R);              // the adapter slice has landed
  volatile int* abort_flag = reinterpret_cast<volatile int*>(abar + 1);
  if (t == 0) {
    mbar_init(abar, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  cluster_arrive_relaxed();  // this CTA has started: the others may store into its shared memory
  __syncthreads();
  if (warp == 0) {  // lane r: adapter row r (0-15 A_q, 16-31 A_v), S floats, 16-byte aligned (S % 16 == 0)
    if (lane == 0) mbar_arrive_expect_tx(abar, 32u * (uint32_t)S * 4u);
    __syncwarp();
    bulk_load(stage + (size_t)lane * S,
              (lane < 16 ? pack.Aq + (size_t)lane * H : pack.Av + (size_t)(lane - 16) * H) + col0, (uint32_t)S * 4u,
              abar);
  }
  if (warp == 1 && lane < 2) {  // this CTA's share of B_q (lane 0) or B_v (lane 1) into L2 for pack_piece
    const size_t bytes = (size_t)(lane ? pack.kvd : pack.qd) * 64, n_cta = (size_t)gridDim.x * gridDim.y;
    const size_t chunk = (bytes / n_cta + 255) / 256 * 256, b0 = (size_t)(blockIdx.y * gridDim.x + blockIdx.x) * chunk;
    if (b0 < bytes)
      bulk_prefetch_l2(reinterpret_cast<const uint8_t*>(lane ? pack.Bv : pack.Bq) + b0,
                       (uint32_t)std::min(chunk, bytes - b0));
  }
  // warp w holds rows 8 w .. 8 w + 7 of the block; lane l the 16-byte vectors 32 h + l of
  // each row slice (h < NH): one warp instruction reads 512 contiguous bytes of a row
  uint4 v[8][NH];
#pragma unroll
  for (int rr = 0; rr < 8; ++rr) {
    const int m = m0 + warp * 8 + rr;
    const uint4* xr = reinterpret_cast<const uint4*>(x + (size_t)m * H + col0);
#pragma unroll
    for (int hh = 0; hh < NH; ++hh)
      if (m < M && hh * 32 + lane < nv) v[rr][hh] = xr[hh * 32 + lane];
  }
  const uint4* wr = reinterpret_cast<const uint4*>(w + col0);
  uint4 wv[NH];
#pragma unroll
  for (int hh = 0; hh < NH; ++hh)
    if (hh * 32 + lane < nv) wv[hh] = wr[hh * 32 + lane];
  float mine = 0.f;  // lane l: the partial of the warp's row l % 8
#pragma unroll
  for (int rr = 0; rr < 8; ++rr) {
    const int m = m0 + warp * 8 + rr;
    float ss = 0.f;
#pragma unroll
    for (int hh = 0; hh < NH; ++hh)
      if (m < M && hh * 32 + lane < nv) {
        float f[8];
        unpack8(v[rr][hh], f);
#pragma unroll
        for (int e = 0; e < 8; ++e) ss += f[e] * f[e];
      }
    ss = warp_sum(ss);
    if ((lane & 7) == rr) mine = ss;
  }
  cluster_wait();  // every CTA of the cluster has started
  {  // into slot c of every CTA: lane l to CTAs l / 8 and l / 8 + 4
    const uint32_t a = smem_u32(ssall + c * ND_R + warp * 8 + (lane & 7));
    const int q0 = lane >> 3;
    if (q0 < C) st_cluster_f32(mapa_shared(a, (uint32_t)q0), mine);
    if (q0 + 4 < C) st_cluster_f32(mapa_shared(a, (uint32_t)(q0 + 4)), mine);
  }
  cluster_arrive();  // this CTA's partial sums are out; the work below runs while the others finish theirs
  // the adapter's B operands, a share per thread of the whole grid
  {
    const int n = pack_pieces(pack), stride = gridDim.x * gridDim.y * ND_THREADS;
    for (int i = (blockIdx.y * gridDim.x + blockIdx.x) * ND_THREADS + t; i < n; i += stride) pack_piece(pack, i);
  }
  // the adapter slice to bf16 (the values of the packed adn), next to the h1 buffer.  A
  // wait that runs out records the site and leaves through the same barriers.
  (void)mbar_wait(abar, 0, abort_flag, err, KID_NORM, 1);
  {  // thread t: 4-float pieces t, t + 256, ..: (row r, piece k) stepped without a division per piece
    const int q4 = S / 4, dr = ND_THREADS / q4, dk = ND_THREADS - dr * q4;
    int r = t / q4, k = t - r * q4;
    for (; r < 32; r += dr, k += dk) {
      if (k >= q4) {
        k -= q4;
        if (++r >= 32) break;
      }
      const float4 f = *reinterpret_cast<const float4*>(stage + (size_t)r * S + 4 * k);
      *reinterpret_cast<uint2*>(as + r * ls + 4 * k) = make_uint2(pack_bf16x2(f.x, f.y), pack_bf16x2(f.z, f.w));
    }
  }
  if (blockIdx.x == 0) {  // the first cluster writes the adapter's A operand adn: its slice of rows 0-31, zero rows 32-63
    __syncthreads();
    for (int i = t; i < ND_R * nv; i += ND_THREADS) {
      const int r = i / nv, k = (i - r * nv) * 8;
      *reinterpret_cast<uint4*>(pack.adn + (size_t)r * H + col0 + k) =
          r < 32 ? *reinterpret_cast<const uint4*>(as + r * ls + k) : make_uint4(0u, 0u, 0u, 0u);
    }
  }
  // every thread of this CTA is done with the staged adapter slice before h1 overwrites
  // it (the cluster barrier's arrivals came before the conversion, so it does not order it)
  __syncthreads();
  cluster_wait();  // every CTA's partial sums are in every CTA's shared memory
  // lane l: the total of the warp's row l % 8, the C partials added in CTA order
  float tot8 = 0.f;
#pragma unroll
  for (int q = 0; q < 8; ++q)
    if (q < C) tot8 += ssall[q * ND_R + warp * 8 + (lane & 7)];
#pragma unroll
  for (int rr = 0; rr < 8; ++rr) {
    const int row = warp * 8 + rr, m = m0 + row;
    const float tot = __shfl_sync(0xffffffffu, tot8, rr);
    const float r = 1.0f / sqrtf(tot / (float)H + eps);
    uint4* yr = reinterpret_cast<uint4*>(y + (size_t)m * H + col0);
    uint4* hrow = reinterpret_cast<uint4*>(hs + row * ls);
#pragma unroll
    for (int hh = 0; hh < NH; ++hh) {
      const int i = hh * 32 + lane;
      if (i < nv) {
        uint4 h = make_uint4(0u, 0u, 0u, 0u);
        if (m < M) {
          float f[8], g[8];
          unpack8(v[rr][hh], f);
          unpack8(wv[hh], g);
#pragma unroll
          for (int e = 0; e < 8; ++e) f[e] = f[e] * r * g[e];
          h = pack8(f);
          yr[i] = h;
        }
        hrow[i] = h;
      }
    }
  }
  __syncthreads();
  // partial t of the slice: row tile mt = warp % 4 (16 rows), k-steps kq, kq + 2, ..
  const int mt = warp & 3, kq = warp >> 2;
  float acc[4][4];
#pragma unroll
  for (int i = 0; i < 4; ++i) acc[i][0] = acc[i][1] = acc[i][2] = acc[i][3] = 0.f;
#pragma unroll 4
  for (int ks = kq; ks < S / 16; ks += 2) {
    uint32_t a0, a1, a2, a3, b0, b1, b2, b3, b4, b5, b6, b7;
    ldsm4(smem_u32(hs + (mt * 16 + (lane & 15)) * ls + ks * 16 + (lane >> 4) * 8), a0, a1, a2, a3);
    const int br = (lane & 7) + (lane >> 4) * 8, bc = ks * 16 + ((lane >> 3) & 1) * 8;
    ldsm4(smem_u32(as + br * ls + bc), b0, b1, b2, b3);
    ldsm4(smem_u32(as + (16 + br) * ls + bc), b4, b5, b6, b7);
    mma16816(acc[0], a0, a1, a2, a3, b0, b1);
    mma16816(acc[1], a0, a1, a2, a3, b2, b3);
    mma16816(acc[2], a0, a1, a2, a3, b4, b5);
    mma16816(acc[3], a0, a1, a2, a3, b6, b7);
  }
  __syncthreads();  // every warp is done with the adapter slice: red may overwrite it
  {
    const int g4 = lane >> 2, t4 = lane & 3;
    float* R = red + warp * (16 * 32);
#pragma unroll
    for (int nt = 0; nt < 4; ++nt) {
      R[g4 * 32 + nt * 8 + 2 * t4] = acc[nt][0];
      R[g4 * 32 + nt * 8 + 2 * t4 + 1] = acc[nt][1];
      R[(g4 + 8) * 32 + nt * 8 + 2 * t4] = acc[nt][2];
      R[(g4 + 8) * 32 + nt * 8 + 2 * t4 + 1] = acc[nt][3];
    }
  }
  __syncthreads();
  const int rows_per = ND_R / C;
  for (int e = t; e < ND_R * 32; e += ND_THREADS) {  // the slice's t (the two k halves in order) to slot c of its owner
    const int rr = e >> 5, cc = e & 31, tile = rr >> 4, ri = rr & 15, q = rr / rows_per;
    const float v2 = red[tile * (16 * 32) + ri * 32 + cc] + red[(4 + tile) * (16 * 32) + ri * 32 + cc];
    st_cluster_f32(mapa_shared(smem_u32(Pin + (c * rows_per + rr - q * rows_per) * 32 + cc), (uint32_t)q), v2);
  }
  cluster_sync_all();  // every CTA's partial t of this CTA's rows is here
  for (int e = t; e < rows_per * 64; e += ND_THREADS) {
    const int rl = e >> 6, cc = e & 63, mm = m0 + c * rows_per + rl;
    if (mm >= M) continue;
    float v2 = 0.f;  // the C partials in CTA order
    if (cc < 32)
#pragma unroll
      for (int q = 0; q < 8; ++q)
        if (q < C) v2 += Pin[(q * rows_per + rl) * 32 + cc];
    tpad[(size_t)mm * 64 + cc] = __float2bfloat16_rn(v2);
  }
}

template <int VPT>
__global__ void __launch_bounds__(1024) k_rmsnorm_bwd_row(const __nv_bfloat16* __restrict__ x,
                                                          const __nv_bfloat16* __restrict__ w,
                                                          const __nv_bfloat16* __restrict__ dy,
                                                          const __nv_bfloat16* __restrict__ resid,
                                                          __nv_bfloat16* __restrict__ dx, int H, float eps) {
  __shared__ float red[32];
  const int row = blockIdx.x, t = threadIdx.x, T = blockDim.x, nv = H / 8;
  const uint4* xr = reinterpret_cast<const uint4*>(x + (size_t)row * H);
  const uint4* wr = reinterpret_cast<const uint4*>(w);
  const uint4* dr = reinterpret_cast<const uint4*>(dy + (size_t)row * H);
  const uint4* rr = resid ? reinterpret_cast<const uint4*>(resid + (size_t)row * H) : nullptr;
  uint4* out = reinterpret_cast<uint4*>(dx + (size_t)row * H);
  uint4 xv[VPT], dv[VPT], rv[VPT];
#pragma unroll
  for (int j = 0; j < VPT; ++j)
    if (t + j * T < nv) {
      xv[j] = xr[t + j * T];
      dv[j] = dr[t + j * T];
      rv[j] = rr ? rr[t + j * T] : make_uint4(0u, 0u, 0u, 0u);
    }
  float ss = 0.f, dot = 0.f;
#pragma unroll
  for (int j = 0; j < VPT; ++j)
    if (t + j * T < nv) {
      float a[8], b[8], c[8];
      unpack8(xv[j], a);
      unpack8(wr[t + j * T], b);
      unpack8(dv[j], c);
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        ss += a[e] * a[e];
        dot += b[e] * c[e] * a[e];
      }
    }
  ss = block_sum(ss, red);
  dot = block_sum(dot, red);
  const float r = 1.0f / sqrtf(ss / (float)H + eps);
  const float k = r * r * r * dot / (float)H;
#pragma unroll
  for (int j = 0; j < VPT; ++j) {
    const int i = t + j * T;
    if (i < nv) {
      float a[8], b[8], c[8], e[8];
      unpack8(xv[j], a);
      unpack8(wr[i], b);
      unpack8(dv[j], c);
      unpack8(rv[j], e);
#pragma unroll
      for (int q = 0; q < 8; ++q) e[q] += r * b[q] * c[q] - a[q] * k;
      out[i] = pack8(e);
    }
  }
}

// threads per row block: VPT vectors each, rounded up to whole warps
inline int row_threads(int H, int vpt) { return ((H / 8 + vpt - 1) / vpt + 31) / 32 * 32; }

// ------------------------------------------------------------------ RoPE
// cos/sin of position p and frequency j, twice: [seq, d/2] (row per position) for
// k_rope_bwd and [d/2, seq] (row per frequency) for the GEMM epilogue, whose lanes hold
// consecutive positions.
__global__ void k_rope_tables(float* cos_t, float* sin_t, float* cos_tt, float* sin_tt, int seq, int d,
                              double theta) {
  const int half = d / 2;
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= seq * half) return;
  const int p = i / half, j = i % half;
  const double inv = pow(theta, -(2.0 * j) / (double)d);
  const double a = (double)p * inv;
  const float c = (float)cos(a), sn = (float)sin(a);
  cos_t[i] = c;
  sin_t[i] = sn;
  cos_tt[(size_t)j * seq + p] = c;
  sin_tt[(size_t)j * seq + p] = sn;
}

// In place: (x1, x2) -> (x1 c + x2 s, x2 c - x1 s), the transpose of the rotation.
__global__ void k_rope_bwd(__nv_bfloat16* __restrict__ x, int ld, int M, int cols, int seq, int d,
                           const float* __restrict__ cos_t, const float* __restrict__ sin_t) {
  const int half = d / 2;
  const size_t per_row = (size_t)cols / 2;
  const size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x;
  if (i >= per_row * M) return;
  const int m = (int)(i / per_row);
  const int r = (int)(i % per_row);
  const int head = r / half, j = r % half;
  const int pos = m % seq;
  __nv_bfloat16* p = x + (size_t)m * ld + head * d;
  const float c = cos_t[pos * half + j], s = sin_t[pos * half + j];
  const float a = __bfloat162float(p[j]), b = __bfloat162float(p[j + half]);
  p[j] = __float2bfloat16_rn(a * c + b * s);
  p[j + half] = __float2bfloat16_rn(b * c - a * s);
}

// The same, eight frequencies per thread: one 16-byte load and store of each half and
// two float4 reads of each table (rows of 16-byte-aligned bf16, d / 2 a multiple of 8).
// Block (x, row): threads over the row's 8-pair groups.
__global__ void k_rope_bwd8(__nv_bfloat16* __restrict__ x, int ld, int cols, int seq, int d,
                            const float* __restrict__ cos_t, const float* __restrict__ sin_t) {
  const int half = d / 2, groups_per_head = half / 8;
  const int gi = blockIdx.x * blockDim.x + threadIdx.x;
  if (gi >= cols / 16) return;
  const int m = blockIdx.y;
  const int head = gi / groups_per_head, j0 = (gi - head * groups_per_head) * 8;
  const int pos = m % seq;
  __nv_bfloat16* p = x + (size_t)m * ld + head * d + j0;
  const float4* cr = reinterpret_cast<const float4*>(cos_t + (size_t)pos * half + j0);
  const float4* sr = reinterpret_cast<const float4*>(sin_t + (size_t)pos * half + j0);
  const float4 c0 = cr[0], c1 = cr[1], s0 = sr[0], s1 = sr[1];
  const float c[8] = {c0.x, c0.y, c0.z, c0.w, c1.x, c1.y, c1.z, c1.w};
  const float sn[8] = {s0.x, s0.y, s0.z, s0.w, s1.x, s1.y, s1.z, s1.w};
  float a[8], b[8], o1[8], o2[8];
  unpack8(*reinterpret_cast<const uint4*>(p), a);
  unpack8(*reinterpret_cast<const uint4*>(p + half), b);
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    o1[j] = a[j] * c[j] + b[j] * sn[j];
    o2[j] = b[j] * c[j] - a[j] * sn[j];
  }
  *reinterpret_cast<uint4*>(p) = pack8(o1);
  *reinterpret_cast<uint4*>(p + half) = pack8(o2);
}

// ------------------------------------------------------------------ embedding, CE, losses, AdamW
__global__ void k_embed(const int32_t* __restrict__ ids, const __nv_bfloat16* __restrict__ E, __nv_bfloat16* __restrict__ h,
                        int M, int H) {
  const int m = blockIdx.x;
  if (m >= M) return;
  const uint4* src = reinterpret_cast<const uint4*>(E + (size_t)ids[m] * H);
  uint4* dst = reinterpret_cast<uint4*>(h + (size_t)m * H);
  for (int i = threadIdx.x; i < H / 8; i += blockDim.x) dst[i] = src[i];
}

// One block per token row: loss_row = logsumexp(logits) - logits[target], and
// dlogits = (softmax - onehot) * inv_count, for rows with a target (t < seq-1);
// other rows get zero loss and zero gradient.
// logits and dlogits may be the same buffer (the gradient overwrites the logits).
// One row of logits per block: an online (max, sum of exp) pass, then the gradient pass
// (softmax - onehot) / count in place of the logits.  Rows are read 8 bf16 at a time
// when V % 8 == 0 (every row then starts 16-byte aligned); the reductions run in a fixed
// order (each thread's sequential chunks, then a fixed tree), so reruns are bit-exact.
__device__ __forceinline__ void online_add(float& m, float& s, float x) {
  if (x > m) {
    s = s * expf(m - x) + 1.0f;
    m = x;
  } else {
    s += expf(x - m);
  }
}

__device__ __forceinline__ void online_merge(float& m, float& s, float m2, float s2) {
  if (m2 > m) {
    s = s * expf(m - m2) + s2;
    m = m2;
  } else if (m2 > -INFINITY) {
    s += s2 * expf(m2 - m);
  }
}

__global__ void __launch_bounds__(256) k_ce(const __nv_bfloat16* logits, const int32_t* __restrict__ ids, int V,
                                            int seq, float inv_count, float* __restrict__ row_loss,
                                            __nv_bfloat16* dlogits) {
  __shared__ float red_m[8], red_s[8];
  __shared__ float bval[3];
  const int m = blockIdx.x;
  const int t = threadIdx.x, lane = t & 31, wid = t >> 5;
  const __nv_bfloat16* row = logits + (size_t)m * V;
  __nv_bfloat16* drow = dlogits + (size_t)m * V;
  const bool vec = (V & 7) == 0;
  const int nv = vec ? V >> 3 : 0;  // 16-byte chunks
  const bool has_target = (m % seq) != seq - 1;
  if (!has_target) {
    const uint4 z = make_uint4(0u, 0u, 0u, 0u);
    for (int j = t; j < nv; j += blockDim.x) reinterpret_cast<uint4*>(drow)[j] = z;
    for (int j = nv * 8 + t; j < V; j += blockDim.x) drow[j] = __float2bfloat16_rn(0.f);
    if (t == 0) row_loss[m] = 0.f;
    return;
  }
  const int tgt = ids[m + 1];
  float mx = -INFINITY, sm = 0.f;
  for (int j = t; j < nv; j += blockDim.x) {
    const uint4 u = reinterpret_cast<const uint4*>(row)[j];
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
    float x[8];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      x[2 * k] = __uint_as_float(w[k] << 16);
      x[2 * k + 1] = __uint_as_float(w[k] & 0xFFFF0000u);
    }
    float cm = x[0];
#pragma unroll
    for (int k = 1; k < 8; ++k) cm = fmaxf(cm, x[k]);
    float cs = 0.f;
#pragma unroll
    for (int k = 0; k < 8; ++k) cs += expf(x[k] - cm);
    online_merge(mx, sm, cm, cs);
  }
  for (int j = nv * 8 + t; j < V; j += blockDim.x) online_add(mx, sm, __bfloat162float(row[j]));
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    const float m2 = __shfl_xor_sync(0xffffffffu, mx, o), s2 = __shfl_xor_sync(0xffffffffu, sm, o);
    online_merge(mx, sm, m2, s2);
  }
  if (lane == 0) {
    red_m[wid] = mx;
    red_s[wid] = sm;
  }
  __syncthreads();
  if (t == 0) {
    float a = red_m[0], b = red_s[0];
    for (int i = 1; i < 8; ++i) online_merge(a, b, red_m[i], red_s[i]);
    bval[0] = a;
    bval[1] = b;
    bval[2] = __bfloat162float(row[tgt]);  // read before the row is overwritten in place
  }
  __syncthreads();
  mx = bval[0];
  const float sum = bval[1];
  const float lse = mx + logf(sum);
  const float scale = inv_count / sum;
  for (int j = t; j < nv; j += blockDim.x) {
    const uint4 u = reinterpret_cast<const uint4*>(row)[j];
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
    uint32_t o[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      float p0 = expf(__uint_as_float(w[k] << 16) - mx) * scale;
      float p1 = expf(__uint_as_float(w[k] & 0xFFFF0000u) - mx) * scale;
      const int e = j * 8 + 2 * k;
      if (e == tgt) p0 -= inv_count;
      if (e + 1 == tgt) p1 -= inv_count;
      o[k] = pack_bf16x2(p0, p1);
    }
    reinterpret_cast<uint4*>(drow)[j] = make_uint4(o[0], o[1], o[2], o[3]);
  }
  for (int j = nv * 8 + t; j < V; j += blockDim.x) {
    float p = expf(__bfloat162float(row[j]) - mx) * scale;
    if (j == tgt) p -= inv_count;
    drow[j] = __float2bfloat16_rn(p);
  }
  if (t == 0) row_loss[m] = lse - bval[2];
}

// ------------------------------------------------------------------ streamed head
// One block per row of a vocab chunk; see ce_chunk in internal.h.
__global__ void __launch_bounds__(256) k_ce_chunk(__nv_bfloat16* logits, int n, int v0,
                                                  const __nv_bfloat16* __restrict__ Wc,
                                                  const int32_t* __restrict__ ids, int H, int seq, int first,
                                                  float* __restrict__ mx, float* __restrict__ sm,
                                                  float* __restrict__ alpha, float* __restrict__ lt,
                                                  __nv_bfloat16* __restrict__ wt) {
  __shared__ float red[8];
  __shared__ float bval;
  const int m = blockIdx.x;
  const int t = threadIdx.x, lane = t & 31, wid = t >> 5;
  __nv_bfloat16* row = logits + (size_t)m * n;
  const int nv = n >> 3;  // n % 64 == 0
  if ((m % seq) == seq - 1) {  // no target: P = 0 keeps this row of the sum at 0
    for (int j = t; j < nv; j += blockDim.x) reinterpret_cast<uint4*>(row)[j] = make_uint4(0u, 0u, 0u, 0u);
    if (t == 0) {
      alpha[m] = 1.0f;
      if (first) {
        mx[m] = 0.0f;
        sm[m] = 1.0f;
        lt[m] = 0.0f;
      }
    }
    return;
  }
  const int tgt = ids[m + 1] - v0;
  if (tgt >= 0 && tgt < n) {
    if (t == 0) lt[m] = __bfloat162float(row[tgt]);  // before the row is overwritten
    const uint4* src = reinterpret_cast<const uint4*>(Wc + (size_t)tgt * H);
    uint4* dst = reinterpret_cast<uint4*>(wt + (size_t)m * H);
    for (int j = t; j < H / 8; j += blockDim.x) dst[j] = src[j];
  }
  float cm = -INFINITY;
  for (int j = t; j < nv; j += blockDim.x) {
    const uint4 u = reinterpret_cast<const uint4*>(row)[j];
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int k = 0; k < 4; ++k)
      cm = fmaxf(cm, fmaxf(__uint_as_float(w[k] << 16), __uint_as_float(w[k] & 0xFFFF0000u)));
  }
  cm = warp_max(cm);
  if (lane == 0) red[wid] = cm;
  __syncthreads();
  if (t == 0) {
    float v = red[0];
    for (int i = 1; i < 8; ++i) v = fmaxf(v, red[i]);
    const float old = first ? -INFINITY : mx[m];
    bval = fmaxf(old, v);
  }
  __syncthreads();
  const float mnew = bval;
  float ssum = 0.f;
  for (int j = t; j < nv; j += blockDim.x) {
    const uint4 u = reinterpret_cast<const uint4*>(row)[j];
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
    uint32_t o[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const float p0 = expf(__uint_as_float(w[k] << 16) - mnew);
      const float p1 = expf(__uint_as_float(w[k] & 0xFFFF0000u) - mnew);
      ssum += p0 + p1;
      o[k] = pack_bf16x2(p0, p1);
    }
    reinterpret_cast<uint4*>(row)[j] = make_uint4(o[0], o[1], o[2], o[3]);
  }
  ssum = warp_sum(ssum);
  __syncthreads();
  if (lane == 0) red[wid] = ssum;
  __syncthreads();
  if (t == 0) {
    float v = 0.f;
    for (int i = 0; i < 8; ++i) v += red[i];
    if (first) {
      sm[m] = v;
      alpha[m] = 0.0f;
    } else {
      const float a = expf(mx[m] - mnew);
      sm[m] = sm[m] * a + v;
      alpha[m] = a;
    }
    mx[m] = mnew;
  }
}

__global__ void __launch_bounds__(256) k_ce_finish(const float* __restrict__ mx, const float* __restrict__ sm,
                                                   const float* __restrict__ lt, const float* __restrict__ acc,
                                                   const __nv_bfloat16* __restrict__ wt, int H, int seq,
                                                   float inv_count, float* __restrict__ row_loss,
                                                   __nv_bfloat16* __restrict__ dh) {
  const int m = blockIdx.x, t = threadIdx.x;
  const bool has_target = (m % seq) != seq - 1;
  if (t == 0) row_loss[m] = has_target ? mx[m] + logf(sm[m]) - lt[m] : 0.0f;
  if (!acc) return;
  const float inv_s = has_target ? 1.0f / sm[m] : 0.0f;
  const float wscale = has_target ? inv_count : 0.0f;
  const float4* a = reinterpret_cast<const float4*>(acc + (size_t)m * H);
  const uint2* w = reinterpret_cast<const uint2*>(wt + (size_t)m * H);
  uint2* d = reinterpret_cast<uint2*>(dh + (size_t)m * H);
  for (int j = t; j < H / 4; j += blockDim.x) {
    const float4 v = a[j];
    const uint2 ww = has_target ? w[j] : make_uint2(0u, 0u);
    const float r0 = (v.x * inv_s - bf16_lo(ww.x)) * wscale, r1 = (v.y * inv_s - bf16_hi(ww.x)) * wscale;
    const float r2 = (v.z * inv_s - bf16_lo(ww.y)) * wscale, r3 = (v.w * inv_s - bf16_hi(ww.y)) * wscale;
    d[j] = make_uint2(pack_bf16x2(r0, r1), pack_bf16x2(r2, r3));
  }
}

// Deterministic mean: one block sums n values in a fixed pattern, then scales.
__global__ void k_sum_scale(const float* __restrict__ v, int n, float scale, float* __restrict__ out) {
  __shared__ double red[256];
  double s = 0.0;
  for (int i = threadIdx.x; i < n; i += blockDim.x) s += (double)v[i];
  red[threadIdx.x] = s;
  __syncthreads();
  for (int o = blockDim.x / 2; o > 0; o >>= 1) {
    if ((int)threadIdx.x < o) red[threadIdx.x] += red[threadIdx.x + o];
    __syncthreads();
  }
  if (threadIdx.x == 0) *out = (float)(red[0] * (double)scale);
}

// Single-layer loss of the one-layer workloads: L = mean(out^2), dL/dout = 2 out / n.
__global__ void k_mse(const __nv_bfloat16* __restrict__ out, size_t n, float* __restrict__ partial,
                      __nv_bfloat16* __restrict__ dout) {
  __shared__ float red[8];
  float s = 0.f;
  const float g = 2.0f / (float)n;
  for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < n; i += (size_t)gridDim.x * blockDim.x) {
    const float v = __bfloat162float(out[i]);
    s += v * v;
    dout[i] = __float2bfloat16_rn(g * v);
  }
  s = warp_sum(s);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = s;
  __syncthreads();
  if (threadIdx.x == 0) {
    float v = 0.f;
    for (int i = 0; i < (int)(blockDim.x >> 5); ++i) v += red[i];
    partial[blockIdx.x] = v;
  }
}

__global__ void k_adamw(float* __restrict__ p, const float* __restrict__ g, float* __restrict__ m, float* __restrict__ v,
                        size_t n, float lr, float b1, float b2, float eps, float wd, float bc1, float bc2) {
  const size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x;
  if (i >= n) return;
  const float gi = g[i];
  const float mi = b1 * m[i] + (1.0f - b1) * gi;
  const float vi = b2 * v[i] + (1.0f - b2) * gi * gi;
  m[i] = mi;
  v[i] = vi;
  const float mh = mi / bc1, vh = vi / bc2;
  p[i] = p[i] - lr * (mh / (sqrtf(vh) + eps) + wd * p[i]);
}

inline unsigned blocks_for(size_t n, int threads) { return (unsigned)((n + threads - 1) / threads); }

}  // namespace

// One block per row, the row in registers: 2 vectors (16 values) per thread up to
// H = 16384 (256 threads at H = 4096, 64 at SmolLM2's 576), 4 up to H = 32768.
int rmsnorm_fwd(const __nv_bfloat16* x, const __nv_bfloat16* w, __nv_bfloat16* y, int M, int H, float eps,
                cudaStream_t s) {
  if (H % 8 || H > 32768) return fail(NF4LS_SHAPE, "rmsnorm: H %% 8, H <= 32768");
  if (M <= 0) return NF4LS_OK;
  const int vpt = H <= 16384 ? 2 : 4;
  const int threads = row_threads(H, vpt);
  if (vpt == 2)
    k_rmsnorm_fwd_row<2><<<M, threads, 0, s>>>(x, w, y, H, eps);
  else
    k_rmsnorm_fwd_row<4><<<M, threads, 0, s>>>(x, w, y, H, eps);
  note_launch();
  NF4_CUDA_TRY(cudaGetLastError());
  return NF4LS_OK;
}

// Input RMSNorm + adapter operand conversion + t = h1 [A_q; A_v]^T in one launch.
int rmsnorm_lora_fwd(const __nv_bfloat16* x, const __nv_bfloat16* w, __nv_bfloat16* y, int M, int H, float eps,
                     const LoraPack& pack, __nv_bfloat16* tpad, cudaStream_t s) {
  const NormDownShape sh = norm_down_shape(H);
  if (!sh.C) return fail(NF4LS_SHAPE, "rmsnorm_lora_fwd: H %d (a multiple of 16 up to 8192)", H);
  if (pack.qd % 8 || pack.kvd % 8) return fail(NF4LS_SHAPE, "rmsnorm_lora_fwd: adapter widths %% 8");
  if (!aligned(pack.Aq, 16) || !aligned(pack.Av, 16) || !aligned(pack.Bq, 16) || !aligned(pack.Bv, 16) ||
      !aligned(x, 16) || !aligned(y, 16) || !aligned(w, 16))
    return fail(NF4LS_ALIGN, "rmsnorm_lora_fwd: 16-byte aligned operands");
  if (M <= 0) return NF4LS_OK;
  const int nh = (sh.S / 8 + 31) / 32;  // 512-byte pieces per row slice
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((M + ND_R - 1) / ND_R, sh.C, 1);
  cfg.blockDim = dim3(ND_THREADS, 1, 1);
  cfg.dynamicSmemBytes = sh.smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 1;
  attr[0].val.clusterDim.y = sh.C;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  auto go = [&](auto kernel, int slot) -> int {
    static int configured[16][4] = {};
    int dev = 0;
    NF4_CUDA_TRY(cudaGetDevice(&dev));
    if (dev < 16 && configured[dev][slot] < (int)sh.smem) {
      NF4_CUDA_TRY(cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sh.smem));
      configured[dev][slot] = (int)sh.smem;
    }
    NF4_CUDA_TRY(cudaLaunchKernelEx(&cfg, kernel, x, w, y, M, H, sh.S, eps, pack, tpad, device_error_ptr()));
    return NF4LS_OK;
  };
  int st;
  if (nh <= 1)
    st = go(k_rmsnorm_down<1>, 0);
  else if (nh <= 2)
    st = go(k_rmsnorm_down<2>, 1);
  else if (nh <= 3)
    st = go(k_rmsnorm_down<3>, 2);
  else
    st = go(k_rmsnorm_down<4>, 3);
  if (st != NF4LS_OK) return st;
  note_launch();
  return NF4LS_OK;
}

int rmsnorm_bwd(const __nv_bfloat16* x, const __nv_bfloat16* w, const __nv_bfloat16* dy, const __nv_bfloat16* resid,
                __nv_bfloat16* dx, int M, int H, float eps, cudaStream_t s) {
  if (H % 8 || H > 32768) return fail(NF4LS_SHAPE, "rmsnorm_bwd: H %% 8, H <= 32768");
  if (M <= 0) return NF4LS_OK;
  if (H <= 16384)
    k_rmsnorm_bwd_row<2><<<M, row_threads(H, 2), 0, s>>>(x, w, dy, resid, dx, H, eps);
  else
    k_rmsnorm_bwd_row<4><<<M, row_threads(H, 4), 0, s>>>(x, w, dy, resid, dx, H, eps);
  note_launch();
  NF4_CUDA_TRY(cudaGetLastError());
  return NF4LS_OK;
}

int rope_tables(float* cos_t, float* sin_t, float* cos_tt, float* sin_tt, int seq, int d, float theta, cudaStream_t s) {
  k_rope_tables<<<blocks_for((size_t)seq * d / 2, 256), 256, 0, s>>>(cos_t, sin_t, cos_tt, sin_tt, seq, d,
                                                                     (double)theta);
  note_launch();
  NF4_CUDA_TRY(cudaGetLastError());
  return NF4LS_OK;
}

int rope_bwd(__nv_bfloat16* x, int ld, int M, int cols, int seq, int d, const float* cos_t, const float* sin_t,
             cudaStream_t s) {
  const bool vec = (d / 2) % 8 == 0 && ld % 8 == 0 && cols % d == 0 && aligned(x, 16) && aligned(cos_t, 16) &&
                   aligned(sin_t, 16) && M <= 65535;
  if (vec)
    k_rope_bwd8<<<dim3(blocks_for((size_t)cols / 16, 128), M), 128, 0, s>>>(x, ld, cols, seq, d, cos_t, sin_t);
  else
    k_rope_bwd<<<blocks_for((size_t)M * cols / 2, 256), 256, 0, s>>>(x, ld, M, cols, seq, d, cos_t, sin_t);
  note_launch();
  NF4_CUDA_TRY(cudaGetLastError());
  return NF4LS_OK;
}


int embed(const int32_t* ids, const __nv_bfloat16* E, __nv_bfloat16* h, int M, int H, cudaStream_t s) {
  k_embed<<<M, 128, 0, s>>>(ids, E, h, M, H);
  note_launch();
  NF4_CUDA_TRY(cudaGetLastError());
  return NF4LS_OK;
}

int cross_entropy(const __nv_bfloat16* logits, const int32_t* ids, int M, int V, int batch, int seq, float* row_loss,
                  __nv_bfloat16* dlogits, float* loss, cudaStream_t s) {
  const int count = batch * (seq - 1);
  k_ce<<<M, 256, 0, s>>>(logits, ids, V, seq, 1.0f / (float)count, row_loss, dlogits);
  note_launch();
  k_sum_scale<<<1, 256, 0, s>>>(row_loss, M, 1.0f / (float)count, loss);
  note_launch();
  NF4_CUDA_TRY(cudaGetLastError());
  return NF4LS_OK;
}

int ce_chunk(__nv_bfloat16* logits, int n, int v0, const __nv_bfloat16* Wc, const int32_t* ids, int M, int H,
             int seq, int first, float* mx, float* sm, float* alpha, float* lt, __nv_bfloat16* wt, cudaStream_t s) {
  if (n % 64 || H % 8) return fail(NF4LS_SHAPE, "ce_chunk: chunk rows %% 64 and H %% 8");
  k_ce_chunk<<<M, 256, 0, s>>>(logits, n, v0, Wc, ids, H, seq, first, mx, sm, alpha, lt, wt);
  note_launch();
  NF4_CUDA_TRY(cudaGetLastError());
  return NF4LS_OK;
}

int ce_finish(const float* mx, const float* sm, const float* lt, const float* acc, const __nv_bfloat16* wt, int M,
              int H, int batch, int seq, float* row_loss, float* loss, __nv_bfloat16* dh, cudaStream_t s) {
  const int count = batch * (seq - 1);
  k_ce_finish<<<M, 256, 0, s>>>(mx, sm, lt, acc, wt, H, seq, 1.0f / (float)count, row_loss, dh);
  note_launch();
  k_sum_scale<<<1, 256, 0, s>>>(row_loss, M, 1.0f / (float)count, loss);
  note_launch();
  NF4_CUDA_TRY(cudaGetLastError());
  return NF4LS_OK;
}

int mse_loss(const __nv_bfloat16* out, size_t n, float* partial, int n_partial, __nv_bfloat16* dout, float* loss,
             cudaStream_t s) {
  k_mse<<<n_partial, 256, 0, s>>>(out, n, partial, dout);
  note_launch();
  k_sum_scale<<<1, 256, 0, s>>>(partial, n_partial, 1.0f / (float)n, loss);
  note_launch();
  NF4_CUDA_TRY(cudaGetLastError());
  return NF4LS_OK;
}

int adamw(float* p, const float* g, float* m, float* v, size_t n, int step, float lr, float b1, float b2, float eps,
          float wd, cudaStream_t s) {
  const float bc1 = (float)(1.0 - std::pow((double)b1, step));
  const float bc2 = (float)(1.0 - std::pow((double)b2, step));
  k_adamw<<<blocks_for(n, 256), 256, 0, s>>>(p, g, m, v, n, lr, b1, b2, eps, wd, bc1, bc2);
  note_launch();
  NF4_CUDA_TRY(cudaGetLastError());
  return NF4LS_OK;
}

}  // namespace nf4ls
