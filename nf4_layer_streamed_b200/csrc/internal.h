// Host-side internals of libnf4ls shared between translation units.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <vector>

#include "../../include/nf4ls.h"

namespace nf4ls {

// ----------------------------------------------------------------------------- status
int fail(int status, const char* fmt, ...);
void clear_error();

#define NF4_CUDA_TRY(expr)                                                                             \
  do {                                                                                                 \
    cudaError_t e_ = (expr);                                                                           \
    if (e_ != cudaSuccess)                                                                             \
      return ::nf4ls::fail(NF4LS_CUDA, "%s failed: %s (%s:%d)", #expr, cudaGetErrorString(e_), __FILE__, \
                           __LINE__);                                                                  \
  } while (0)

#define NF4_TRY(expr)         \
  do {                        \
    int s_ = (expr);          \
    if (s_ != NF4LS_OK) return s_; \
  } while (0)

inline bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }
inline size_t round_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// ----------------------------------------------------------------------------- slot plan
// Host-only bookkeeping of a streaming pool's slots, with no CUDA state: which slot a
// layer goes to, whether a request is served by a slot that already holds the layer
// (a hit) or fills one, whether that fill must wait for the slot's previous reader,
// and, under the layer-sharded fetch, which rank reads the layer from its host store.
// The pool (pool.cpp) takes every slot decision here and adds only the CUDA work;
// nf4ls_plan_* (plan.cpp) exports the same object so that the decisions can be driven
// without a GPU.  Slots are reused least recently released first.
struct PlanStep {
  int slot = -1;
  bool hit = false;            // the layer already sits in a slot: nothing is copied
  bool fill = false;           // this request fills the slot
  bool after_release = false;  // the slot was released before: the fill waits for that release
  int owner = 0;               // the rank that reads the layer from its host store
  bool host_read = false;      // fill and owner == this rank
  bool broadcast = false;      // fill and the pool is shared: the owner's bytes go to every rank
};

class SlotPlan {
 public:
  void init(int n_layers, int depth);
  void share(int rank, int world) {
    rank_ = rank;
    world_ = world;
    shared_ = true;
  }
  int depth() const { return (int)s_.size(); }
  int n_layers() const { return n_layers_; }
  int find(int layer) const;         // the slot holding layer, or -1
  bool holds_any() const;
  bool acquired(int slot) const { return s_[slot].acquired; }
  int layer_in(int slot) const { return s_[slot].layer; }
  // What a request for layer would do, without changing anything (BUFFER_BUSY when it
  // needs a slot and every slot is acquired or filled and not yet acquired).
  int preview(int layer, PlanStep* st) const;
  int issue(int layer, PlanStep* st);                  // preview, then take the slot
  void mark_acquired(int slot);                        // the caller now reads the slot
  int acquire(int layer, PlanStep* st);                // issue + BUFFER_BUSY if held + mark
  int acquired_slot(int layer) const;                  // -1 unless layer is acquired
  void release(int slot);                              // the caller's reads are ordered before reuse

 private:
  struct Slot {
    int layer = -1;
    bool acquired = false;
    bool pending = false;   // filled and not yet acquired
    bool released = false; // released at least once
    uint64_t release_tick = 0;
  };
  int victim() const;
  std::vector<Slot> s_;
  uint64_t tick_ = 0;
  int n_layers_ = 0, rank_ = 0, world_ = 1;
  bool shared_ = false;
};

// The pool calls of one pass over the layers, in the order the model step makes them:
// for each layer of the pass (dir +1: 0..n-1, dir -1: n-1..0) acquire it, prefetch the
// next `lookahead` layers of the pass (stopping at the first BUFFER_BUSY, which is not
// an error), run it, release it.  f(op, layer) returns a status.
enum PassOp : int { PASS_ACQUIRE = 0, PASS_PREFETCH = 1, PASS_RUN = 2, PASS_RELEASE = 3 };
template <typename F>
int for_each_pass_op(int n_layers, int dir, int lookahead, F&& f) {
  for (int t = 0; t < n_layers; ++t) {
    const int i = dir > 0 ? t : n_layers - 1 - t;
    NF4_TRY(f(PASS_ACQUIRE, i));
    for (int k = 1; k <= lookahead; ++k) {
      const int j = i + dir * k;
      if (j < 0 || j >= n_layers) break;
      const int st = f(PASS_PREFETCH, j);
      if (st == NF4LS_BUFFER_BUSY) break;
      NF4_TRY(st);
    }
    NF4_TRY(f(PASS_RUN, i));
    NF4_TRY(f(PASS_RELEASE, i));
  }
  return NF4LS_OK;
}
// Layers the model step prefetches ahead of the one it runs.
constexpr int kStepLookahead = 1;

// ----------------------------------------------------------------------------- code tables
struct Codebooks {
  float nf4[16];
  float code8[256];
  float mid4[15];   // fp32 midpoints between neighbouring NF4 entries
  float mid8[255];  // fp32 midpoints between neighbouring code8 entries
  int zero4;        // index of the exact 0 in nf4
  int zero8;        // index of the exact 0 in code8
  uint64_t hash;
};
const Codebooks& codebooks();

// ----------------------------------------------------------------------------- quantiser
int quantize_tensor(const void* w, size_t n, uint8_t* packed, uint8_t* q8, float* nested, float* offset,
                    void* scratch, size_t scratch_bytes, cudaStream_t s);
int dequantize_tensor(const uint8_t* packed, const uint8_t* q8, const float* nested, const float* offset,
                      size_t n, void* out, cudaStream_t s);

// ----------------------------------------------------------------------------- shard view
struct NF4Tensor {
  const uint8_t* packed;
  const uint8_t* q8;
  const float* nested;
  const float* offset;
  int rows, cols;
};
struct ShardView {
  NF4Tensor t[7];
  const __nv_bfloat16* norm_in;
  const __nv_bfloat16* norm_post;
};
// Builds device pointers into a shard at shard_dev from the layout that cfg implies.
void shard_view(const nf4ls_layer_cfg* cfg, const void* shard_dev, ShardView* v);
struct ShardLayout {
  uint64_t off_packed[7], off_q8[7], off_nested[7], off_offset[7];
  uint64_t off_norm_in, off_norm_post;
  uint64_t total, quantized;
  int rows[7], cols[7];
};
void shard_layout(const nf4ls_layer_cfg* cfg, ShardLayout* L);

// ----------------------------------------------------------------------------- GEMM
// Output epilogues of the tcgen05 GEMM (accumulator fp32 -> bf16 stores).
enum Epilogue : int {
  EPI_STORE = 0,    // out = acc
  EPI_RESID = 1,    // out = acc + aux0[m, n]
  EPI_ROPE = 2,     // out = rope(acc) on columns < rope_cols, acc elsewhere
  EPI_SWIGLU = 3,   // columns [0,128) gate, [128,256) up of block i: out[m, i] = silu(g) * u; aux_out g,u
  EPI_DSWIGLU = 4,  // acc = da[m, i]; aux0 = [g | u] -> out = [dg | du]
  EPI_ACC_F32 = 5,  // out_f32[m, n] = acc + (accumulate ? alpha[m] * out_f32[m, n] : 0)
};

struct GemmEpilogue {
  int kind = EPI_STORE;
  __nv_bfloat16* out = nullptr;
  int ldo = 0;
  const __nv_bfloat16* aux0 = nullptr;  // residual / g,u source
  int ld_aux0 = 0;
  __nv_bfloat16* aux_out = nullptr;     // g,u store of EPI_SWIGLU (may be null)
  int ld_aux_out = 0;
  int inter = 0;                        // I for the SwiGLU layouts
  const float* rope_cos = nullptr;      // [d/2, seq] (row per frequency)
  const float* rope_sin = nullptr;
  int seq = 0, head_dim = 0, rope_cols = 0;
  float* out_f32 = nullptr;             // EPI_ACC_F32 output (and input when accumulate)
  const float* alpha = nullptr;         // EPI_ACC_F32 per-row scale of the old value
  int accumulate = 0;
};

// Weights of a GEMM: either one dense bf16 matrix, or up to four NF4 tensors that
// are concatenated along the weight's rows (its output features).
struct GemmWeights {
  const __nv_bfloat16* dense = nullptr;  // [rows, cols] row-major
  int n_seg = 0;
  NF4Tensor seg[4];
};

struct GemmExtra {
  // One extra 64-wide reduction block appended after the main reduction: the LoRA
  // up-projection (forward) or the LoRA A^T product (dL/dx).  a: bf16 [M, 64];
  // b: bf16 [N, 64] (forward, K-major) or [64, N] (dL/dx, N-major).
  const __nv_bfloat16* a = nullptr;
  const __nv_bfloat16* b = nullptr;
};

// Forward product out[M, N] = A[M, K] W^T, W [N, K] (weights rows = N).
// dL/dx product out[M, N] = A[M, K] W, W [K, N] (weights rows = K, the reduction).
int gemm(const __nv_bfloat16* A, int lda, int M, int N, int K, const GemmWeights& W, bool dgrad,
         const GemmExtra& extra, const GemmEpilogue& epi, cudaStream_t s);

int gemm_path();
int gemm_pair();
int gemm_half_mode();
int attention_tc();
int check_cfg(const nf4ls_layer_cfg* c);
int* device_error_ptr();
// Process-unique id of the CUDA context current on this thread, 0 when none is
// current or the driver cannot say.  A symbol address looked up in one context is
// valid only there: a device reset (a new primary context) or another context needs
// a fresh lookup.
unsigned long long current_context_id();

// ----------------------------------------------------------------------------- accounting
// Every kernel launch of the library bumps a process-wide counter.
void note_launch(int n = 1);
// Optional per-launch CUDA-event timing of the GEMMs (kind 0 dense, 1 NF4 decode).
bool profiling();
void profile_begin(cudaStream_t s, cudaEvent_t* e0);
void profile_end(cudaStream_t s, cudaEvent_t e0, int kind, int detail, double flops);

// ----------------------------------------------------------------------------- body kernels
// The bf16 operands of the LoRA adapter, converted from the fp32 masters (q_proj and
// v_proj, r = 16): bup [Nqkv, 64] (q rows: s B_q in columns 0-15; v rows: s B_v in columns
// 16-31; else 0), adn [64, H] (rows 0-15 A_q, rows 16-31 A_v, else 0), bqt [16, qd] = B_q^T,
// bvt [16, kvd] = B_v^T.
struct LoraPack {
  const float* Aq;
  const float* Av;
  const float* Bq;
  const float* Bv;
  int H, qd, kvd;
  float scale;
  __nv_bfloat16* bup;
  __nv_bfloat16* adn;
  __nv_bfloat16* bqt;
  __nv_bfloat16* bvt;
};
// y = rmsnorm(x) w.
int rmsnorm_fwd(const __nv_bfloat16* x, const __nv_bfloat16* w, __nv_bfloat16* y, int M, int H, float eps,
                cudaStream_t s);
// y = rmsnorm(x) w (the input norm) with the adapter operands filled and
// t = [y A_q^T | y A_v^T] written to columns 0-31 of tpad [M, 64] (32-63 zero).
int rmsnorm_lora_fwd(const __nv_bfloat16* x, const __nv_bfloat16* w, __nv_bfloat16* y, int M, int H, float eps,
                     const LoraPack& pack, __nv_bfloat16* tpad, cudaStream_t s);
// dx = resid + rmsnorm_bwd(x, w, dy); resid may be null.
int rmsnorm_bwd(const __nv_bfloat16* x, const __nv_bfloat16* w, const __nv_bfloat16* dy,
                const __nv_bfloat16* resid, __nv_bfloat16* dx, int M, int H, float eps, cudaStream_t s);
int rope_tables(float* cos_t, float* sin_t, float* cos_tt, float* sin_tt, int seq, int d, float theta, cudaStream_t s);
int rope_bwd(__nv_bfloat16* x, int ld, int M, int cols, int seq, int d, const float* cos_t,
             const float* sin_t, cudaStream_t s);
// 2D bf16 tensor map, 128-byte swizzle: [rows, cols] with row stride row_bytes, box
// box_cols x box_rows.
int tma_map_bf16(CUtensorMap* map, const void* ptr, uint64_t cols, uint64_t rows, uint64_t row_bytes,
                 uint32_t box_cols, uint32_t box_rows);
// The tcgen05 attention (head_dim 64 or 128; seq a multiple of 128 up to 8192).
bool attention_fwd_tc_supported(int seq, int d, int nq, int nkv, int ldq, int ldkv, int ldo);
bool attention_bwd_tc_supported(int seq, int d, int nq, int nkv, int ldq, int ldkv, int ldo, int ld_dq, int ld_dkv);
int attention_fwd_tc(const __nv_bfloat16* q, const __nv_bfloat16* k, const __nv_bfloat16* v, int ldq, int ldkv,
                     __nv_bfloat16* o, int ldo, float* lse, int batch, int seq, int nq, int nkv, int d, cudaStream_t s);
// The tcgen05 backward: the query-side kernel also forms delta = rowsum(dO * O) (into
// `delta`, [batch, nq, seq]) for the key-side kernel that follows it.
int attention_bwd_tc(const __nv_bfloat16* q, const __nv_bfloat16* k, const __nv_bfloat16* v, int ldq, int ldkv,
                     const __nv_bfloat16* o, const __nv_bfloat16* dout, int ldo, const float* lse, float* delta,
                     __nv_bfloat16* dq, __nv_bfloat16* dk, __nv_bfloat16* dv, int ld_dq, int ld_dkv, int batch, int seq,
                     int nq, int nkv, int d, cudaStream_t s);
int attention_fwd(const __nv_bfloat16* q, const __nv_bfloat16* k, const __nv_bfloat16* v, int ldq, int ldkv,
                  __nv_bfloat16* o, int ldo, float* lse, int batch, int seq, int nq, int nkv, int d,
                  cudaStream_t s);
int attention_bwd(const __nv_bfloat16* q, const __nv_bfloat16* k, const __nv_bfloat16* v, int ldq, int ldkv,
                  const __nv_bfloat16* o, const __nv_bfloat16* dout, int ldo, const float* lse, float* delta,
                  __nv_bfloat16* dq, __nv_bfloat16* dk, __nv_bfloat16* dv, int ld_dq, int ld_dkv, int batch,
                  int seq, int nq, int nkv, int d, cudaStream_t s);

// LoRA backward (lora.cu); the forward's t comes from rmsnorm_lora_fwd (body.cu).
// dB_q, dB_v, dA_q, dA_v (fp32, written) and dt into dtpad [M, 64] (bf16, zeros in
// columns 32-63) from dq (columns [0, qd) of dqkv) and dv (columns [vcol, vcol + kvd));
// part: lora_partial_bytes of scratch.  phases: LORA_BWD_DT = the partial sums and dt
// (two launches; the dL/dx GEMM needs dt), LORA_BWD_DB_DA = dB from the same partial
// sums and dA = dt^T h1 (two launches; nothing in the layer's backward waits for them),
// on stream s, the second after the first in stream order.
constexpr int LORA_BWD_DT = 1, LORA_BWD_DB_DA = 2;
size_t lora_partial_bytes(int M, int H, int qd, int kvd);
int lora_bwd(const __nv_bfloat16* dqkv, int ld, int vcol, int M, int H, int qd, int kvd, const __nv_bfloat16* tpad,
             const __nv_bfloat16* bqt, const __nv_bfloat16* bvt, const __nv_bfloat16* h1, float scale,
             __nv_bfloat16* dtpad, const nf4ls_lora_grads* g, void* part, int phases, cudaStream_t s);
// A second stream on the current device for work that can run beside the caller's:
// fork records an event on s, launches made on side() after it wait for it, and join
// makes s wait for everything launched on side() since.  The fork-join sequence holds
// a per-device lock (one sequence at a time per device and process).
class SideStream {
 public:
  SideStream();
  ~SideStream();
  int fork(cudaStream_t s);
  cudaStream_t side() const { return side_; }
  int join(cudaStream_t s);

 private:
  int dev_ = -1;
  bool forked_ = false;
  cudaStream_t side_ = nullptr;
  cudaEvent_t ready_ = nullptr, done_ = nullptr;
};
int embed(const int32_t* ids, const __nv_bfloat16* E, __nv_bfloat16* h, int M, int H, cudaStream_t s);
// Streamed head, per vocab chunk [v0, v0 + n) of the output matrix (rows Wc in HBM):
// logits [M, n] (bf16, from the GEMM) are folded into the per-row running max mx, sum
// sm (first chunk: first = 1 starts them) and overwritten in place by
// P = bf16(exp(logit - mx_new)); alpha[m] = exp(mx_old - mx_new) rescales the running
// sum of P Wc (the next GEMM's EPI_ACC_F32).  A row whose target id falls in the chunk
// records the target logit and copies that row of Wc into wt.
int ce_chunk(__nv_bfloat16* logits, int n, int v0, const __nv_bfloat16* Wc, const int32_t* ids, int M, int H,
             int seq, int first, float* mx, float* sm, float* alpha, float* lt, __nv_bfloat16* wt, cudaStream_t s);
// After the last chunk: per-row loss mx + log(sm) - lt (0 for rows without a target),
// the mean into loss, and (acc != null) dh = bf16((acc / sm - wt) / count).
int ce_finish(const float* mx, const float* sm, const float* lt, const float* acc, const __nv_bfloat16* wt,
              int M, int H, int batch, int seq, float* row_loss, float* loss, __nv_bfloat16* dh, cudaStream_t s);
int cross_entropy(const __nv_bfloat16* logits, const int32_t* ids, int M, int V, int batch, int seq, float* row_loss,
                  __nv_bfloat16* dlogits, float* loss, cudaStream_t s);
int mse_loss(const __nv_bfloat16* out, size_t n, float* partial, int n_partial, __nv_bfloat16* dout, float* loss,
             cudaStream_t s);
int adamw(float* p, const float* g, float* m, float* v, size_t n, int step, float lr, float b1, float b2, float eps,
          float wd, cudaStream_t s);

// ----------------------------------------------------------------------------- layer
// tables_ready: the RoPE tables of the workspace are already those of cfg (a model pass
// writes them at its first layer and the other layers of the pass reuse them).
// keep (forward): also keep g and u, so that the workspace holds everything the layer's
// backward would recompute.  recompute (backward): false when the workspace still holds
// this layer's forward with keep (the last layer of a model step, whose backward follows
// its forward with nothing else in the workspace between); the results are the same.
int layer_fwd_impl(const nf4ls_layer_cfg* cfg, const void* shard, const nf4ls_lora* lora, const __nv_bfloat16* x,
                   __nv_bfloat16* y, void* ws, size_t ws_bytes, cudaStream_t s, bool tables_ready = false,
                   bool keep = false);
int layer_bwd_impl(const nf4ls_layer_cfg* cfg, const void* shard, const nf4ls_lora* lora, const __nv_bfloat16* x,
                   const __nv_bfloat16* dy, __nv_bfloat16* dx, const nf4ls_lora_grads* g, void* ws, size_t ws_bytes,
                   cudaStream_t s, bool tables_ready = false, bool recompute = true);
size_t layer_ws_bytes(const nf4ls_layer_cfg* cfg);

}  // namespace nf4ls
