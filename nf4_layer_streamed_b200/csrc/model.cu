// One SFT step of the whole stack: embedding -> streamed decoder layers (forward,
// saving each layer input) -> final RMSNorm -> lm_head -> causal-LM cross-entropy ->
// lm_head and final-norm backward -> streamed decoder layers in reverse (checkpoint
// recompute + dL/dx + LoRA gradients) -> AdamW on the LoRA tensors.
//
// From the layer-streaming review ("4GB 显存微调 8B 模型是真的", mechanism section):
// only the adapter, its gradients and its optimiser state stay resident, together with
// the unquantised embedding and lm_head; the frozen layers are prefetched one step
// ahead on a side stream, i+1 in the forward and i-1 in the backward.  From
// "Soup 层流式 NF4 训练实测：在 4 GB 显存上以位级一致标准完成 8B 模型 LoRA 微调"
// §4.4: lm_head sits outside the checkpointed layers (2 forward + 2 dL/dx FLOP
// per parameter and token).  The DPO/KTO write-up ("Soup v0.72.4 技术解析" §3.1) reuses
// the same streamed base with the adapter switched off as the reference model, which
// nf4ls_forward_loss(lora_on = 0) provides.
#include <algorithm>

#include "common.cuh"
#include "internal.h"

namespace nf4ls {

namespace {

struct ModelWs {
  size_t xs, hf, logits, row_loss, dh, dhf, layer, total;
  size_t acc = 0, wt = 0, mx = 0, sm = 0, alpha = 0, lt = 0;  // streamed head
};

bool streamed_head(const nf4ls_model_cfg* c) { return c->head_chunk_rows > 0; }

ModelWs model_ws(const nf4ls_model_cfg* c) {
  const size_t M = (size_t)c->layer.batch * c->layer.seq, H = c->layer.hidden;
  ModelWs L;
  size_t off = 0;
  auto take = [&](size_t bytes) {
    const size_t o = off;
    off = round_up(off + bytes, 256);
    return o;
  };
  L.xs = take((size_t)(c->n_layers + 1) * M * H * 2);
  L.hf = take(M * H * 2);
  // resident head: the whole [M, V] logits; streamed head: one vocab chunk of them
  L.logits = take(M * (size_t)(streamed_head(c) ? std::min(c->head_chunk_rows, c->vocab) : c->vocab) * 2);
  L.row_loss = take(M * 4);
  if (streamed_head(c)) {
    L.acc = take(M * H * 4);
    L.wt = take(M * H * 2);
    L.mx = take(M * 4);
    L.sm = take(M * 4);
    L.alpha = take(M * 4);
    L.lt = take(M * 4);
  }
  L.dh = take(M * H * 2);
  L.dhf = take(M * H * 2);
  L.layer = take(layer_ws_bytes(&c->layer));
  L.total = off;
  return L;
}

size_t stride_of(const nf4ls_layer_cfg* c) {
  const size_t r = c->lora_r, H = c->hidden;
  return r * H + (size_t)c->n_q * c->head_dim * r + r * H + (size_t)c->n_kv * c->head_dim * r;
}

void lora_views(const nf4ls_layer_cfg* c, float* base, nf4ls_lora* l, nf4ls_lora_grads* g, float* gbase) {
  const size_t r = c->lora_r, H = c->hidden, qd = (size_t)c->n_q * c->head_dim;
  l->A_q = base;
  l->B_q = base + r * H;
  l->A_v = base + r * H + qd * r;
  l->B_v = base + 2 * r * H + qd * r;
  if (g) {
    g->dA_q = gbase;
    g->dB_q = gbase + r * H;
    g->dA_v = gbase + r * H + qd * r;
    g->dB_v = gbase + 2 * r * H + qd * r;
  }
}

template <typename T>
T* at(void* ws, size_t off) {
  return reinterpret_cast<T*>(static_cast<uint8_t*>(ws) + off);
}

// Phase timing (when profiling is on): detail 2000 layer forwards, 2001 final norm +
// lm_head + loss, 2002 lm_head dL/dx + final-norm backward, 2003 layer backwards.
struct Phase {
  cudaStream_t s;
  cudaEvent_t e = nullptr;
  int detail;
  Phase(cudaStream_t s_, int d) : s(s_), detail(d) {
    if (profiling()) profile_begin(s, &e);
  }
  ~Phase() {
    if (e) profile_end(s, e, 2, detail, 0.0);
  }
};

// One pass over the layers (dir +1 forward, -1 backward) in the pool-call order of
// for_each_pass_op: acquire layer i, prefetch the next layer of the pass (a busy pool
// is not an error: the next acquire copies it), run(i, shard), release i.  With
// resident shards the pool calls drop out.
template <typename Run>
int layer_pass(const nf4ls_model_cfg* c, const nf4ls_model* m, int dir, cudaStream_t s, Run&& run) {
  const void* shard = nullptr;
  return for_each_pass_op(c->n_layers, dir, kStepLookahead, [&](int op, int layer) -> int {
    switch (op) {
      case PASS_ACQUIRE:
        if (!m->pool) {
          shard = m->shards_dev[layer];
          return NF4LS_OK;
        }
        return stream_prefetch(m->pool, layer, s, &shard);
      case PASS_PREFETCH:
        return m->pool ? nf4ls_pool_prefetch(m->pool, layer) : NF4LS_OK;
      case PASS_RUN:
        return run(layer, shard);
      default:
        return m->pool ? nf4ls_pool_release(m->pool, layer, s) : NF4LS_OK;
    }
  });
}

int check_model(const nf4ls_model_cfg* c, const nf4ls_model* m) {
  if (!c || !m) return fail(NF4LS_INVALID_ARG, "model: null config or model");
  NF4_TRY(check_cfg(&c->layer));
  if (c->n_layers <= 0 || c->vocab <= 0 || c->vocab % 64) return fail(NF4LS_SHAPE, "model: vocab must be a multiple of 64");
  if (!m->norm_final_dev || !m->lora_dev || !m->ws_dev) return fail(NF4LS_INVALID_ARG, "model: null buffer");
  if (streamed_head(c)) {
    if (c->head_chunk_rows % 64) return fail(NF4LS_SHAPE, "model: head_chunk_rows must be a multiple of 64");
    if (!m->head_pool) return fail(NF4LS_INVALID_ARG, "model: streamed head needs head_pool");
    if (!m->embed_dev && !m->embed_host) return fail(NF4LS_INVALID_ARG, "model: no embedding");
  } else {
    if (c->head_chunk_rows < 0) return fail(NF4LS_INVALID_ARG, "model: head_chunk_rows < 0");
    if (!m->embed_dev) return fail(NF4LS_INVALID_ARG, "model: null embedding");
    if (!c->tied && !m->lm_head_dev) return fail(NF4LS_INVALID_ARG, "model: untied model needs lm_head");
  }
  if (!m->pool && !m->shards_dev) return fail(NF4LS_INVALID_ARG, "model: needs a pool or resident shards");
  if (!aligned(m->ws_dev, 256)) return fail(NF4LS_ALIGN, "model: workspace must be 256-byte aligned");
  if (m->ws_bytes < model_ws(c).total) return fail(NF4LS_INVALID_ARG, "model: workspace too small");
  return NF4LS_OK;
}

// The streamed head: logits, loss and (need_grad) dL/dhf in one pass over the vocab
// chunks of the output matrix, each chunk used by two GEMMs while it is in its slot:
// logits_c = hf Wc^T, then (after ce_chunk folded them into the running max / sum and
// turned them into P = exp(logit - max)) acc = alpha acc + P Wc in fp32.
int head_streamed(const nf4ls_model_cfg* c, const nf4ls_model* m, const int32_t* ids, const __nv_bfloat16* hf,
                  bool need_grad, float* loss, __nv_bfloat16* dhf, cudaStream_t s, const ModelWs& L) {
  const nf4ls_layer_cfg* lc = &c->layer;
  const int M = lc->batch * lc->seq, H = lc->hidden, V = c->vocab, C = c->head_chunk_rows;
  void* ws = m->ws_dev;
  auto* lg = at<__nv_bfloat16>(ws, L.logits);
  auto* acc = at<float>(ws, L.acc);
  auto* wt = at<__nv_bfloat16>(ws, L.wt);
  auto* mx = at<float>(ws, L.mx);
  auto* sm = at<float>(ws, L.sm);
  auto* alpha = at<float>(ws, L.alpha);
  auto* lt = at<float>(ws, L.lt);
  const int nch = (V + C - 1) / C;
  for (int k = 0; k < nch; ++k) {
    const void* slot;
    NF4_TRY(stream_prefetch(m->head_pool, k, s, &slot));
    if (k + 1 < nch) {
      const int st = nf4ls_pool_prefetch(m->head_pool, k + 1);
      if (st != NF4LS_BUFFER_BUSY) NF4_TRY(st);
    }
    const int v0 = k * C, n = std::min(C, V - v0);
    GemmWeights w;
    w.dense = static_cast<const __nv_bfloat16*>(slot);
    GemmEpilogue e;
    e.out = lg;
    e.ldo = n;
    NF4_TRY(gemm(hf, H, M, n, H, w, false, GemmExtra(), e, s));
    NF4_TRY(ce_chunk(lg, n, v0, w.dense, ids, M, H, lc->seq, k == 0, mx, sm, alpha, lt, wt, s));
    if (need_grad) {
      GemmEpilogue ea;
      ea.kind = EPI_ACC_F32;
      ea.out_f32 = acc;
      ea.ldo = H;
      ea.alpha = alpha;
      ea.accumulate = k > 0;
      NF4_TRY(gemm(lg, n, M, H, n, w, true, GemmExtra(), ea, s));
    }
    NF4_TRY(nf4ls_pool_release(m->head_pool, k, s));
  }
  return ce_finish(mx, sm, lt, need_grad ? acc : nullptr, wt, M, H, lc->batch, lc->seq, at<float>(ws, L.row_loss),
                   loss, dhf, s);
}

// Forward through embedding, layers, final norm, lm_head and the loss (and, for the
// streamed head with need_grad, dL/dhf).
int forward_to_loss(const nf4ls_model_cfg* c, const nf4ls_model* m, const int32_t* ids, bool lora_on, float* loss,
                    cudaStream_t s, const ModelWs& L, bool need_grad) {
  const nf4ls_layer_cfg* lc = &c->layer;
  const int M = lc->batch * lc->seq, H = lc->hidden, V = c->vocab;
  void* ws = m->ws_dev;
  auto* xs = at<__nv_bfloat16>(ws, L.xs);
  const size_t act = (size_t)M * H;
  const size_t stride = stride_of(lc);
  const void* E = m->embed_dev;
  if (!E) {  // rows gathered straight from pinned host memory
    void* d = nullptr;
    if (cudaHostGetDevicePointer(&d, const_cast<void*>(m->embed_host), 0) != cudaSuccess) {
      cudaGetLastError();
      return fail(NF4LS_INVALID_ARG, "model: embed_host is not pinned, device-mapped host memory");
    }
    E = d;
  }
  NF4_TRY(embed(ids, static_cast<const __nv_bfloat16*>(E), xs, M, H, s));
  {
    Phase fwd_phase(s, 2000);
    NF4_TRY(layer_pass(c, m, +1, s, [&](int i, const void* shard) {
      nf4ls_lora l;
      lora_views(lc, m->lora_dev + (size_t)i * stride, &l, nullptr, nullptr);
      // the last layer of a training step keeps its activations: its backward, next in
      // the workspace after the head, skips the checkpoint recompute
      return layer_fwd_impl(lc, shard, lora_on ? &l : nullptr, xs + (size_t)i * act, xs + (size_t)(i + 1) * act,
                            at<void>(ws, L.layer), L.total - L.layer, s, i != 0, need_grad && i == c->n_layers - 1);
    }));
  }
  Phase head(s, 2001);
  auto* hf = at<__nv_bfloat16>(ws, L.hf);
  auto* logits = at<__nv_bfloat16>(ws, L.logits);
  const auto* lm = static_cast<const __nv_bfloat16*>(c->tied ? m->embed_dev : m->lm_head_dev);
  NF4_TRY(rmsnorm_fwd(xs + (size_t)c->n_layers * act, static_cast<const __nv_bfloat16*>(m->norm_final_dev), hf, M, H,
                      lc->rms_eps, s));
  if (streamed_head(c))
    return head_streamed(c, m, ids, hf, need_grad, loss, at<__nv_bfloat16>(ws, L.dhf), s, L);
  GemmWeights w;
  w.dense = lm;
  GemmEpilogue e;
  e.out = logits;
  e.ldo = V;
  NF4_TRY(gemm(hf, H, M, V, H, w, false, GemmExtra(), e, s));
  // dlogits overwrite the logits in place
  return cross_entropy(logits, ids, M, V, lc->batch, lc->seq, at<float>(ws, L.row_loss), logits, loss, s);
}

}  // namespace

}  // namespace nf4ls

using namespace nf4ls;

extern "C" size_t nf4ls_lora_stride(const nf4ls_layer_cfg* cfg) { return cfg ? stride_of(cfg) : 0; }

extern "C" size_t nf4ls_model_workspace_bytes(const nf4ls_model_cfg* cfg) { return cfg ? model_ws(cfg).total : 0; }

extern "C" int nf4ls_forward_loss(const nf4ls_model_cfg* cfg, const nf4ls_model* m, const int32_t* ids_dev,
                                  int32_t lora_on, float* loss_dev, nf4ls_stream stream) {
  clear_error();
  NF4_TRY(check_model(cfg, m));
  if (!ids_dev || !loss_dev) return fail(NF4LS_INVALID_ARG, "nf4ls_forward_loss: null ids or loss");
  return forward_to_loss(cfg, m, ids_dev, lora_on != 0, loss_dev, static_cast<cudaStream_t>(stream), model_ws(cfg),
                         false);
}

extern "C" int nf4ls_forward_backward(const nf4ls_model_cfg* cfg, const nf4ls_model* m, const int32_t* ids_dev,
                                      float* loss_dev, nf4ls_stream stream) {
  clear_error();
  NF4_TRY(check_model(cfg, m));
  if (!ids_dev || !loss_dev || !m->grads_dev) return fail(NF4LS_INVALID_ARG, "nf4ls_forward_backward: null argument");
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const ModelWs L = model_ws(cfg);
  NF4_TRY(forward_to_loss(cfg, m, ids_dev, true, loss_dev, s, L, true));
  const nf4ls_layer_cfg* lc = &cfg->layer;
  const int M = lc->batch * lc->seq, H = lc->hidden, V = cfg->vocab;
  void* ws = m->ws_dev;
  auto* xs = at<__nv_bfloat16>(ws, L.xs);
  const size_t act = (size_t)M * H;
  auto* logits = at<__nv_bfloat16>(ws, L.logits);  // now dlogits
  auto* dhf = at<__nv_bfloat16>(ws, L.dhf);
  auto* dh = at<__nv_bfloat16>(ws, L.dh);
  const auto* lm = static_cast<const __nv_bfloat16*>(cfg->tied ? m->embed_dev : m->lm_head_dev);
  {
    Phase head_bwd(s, 2002);
    if (!streamed_head(cfg)) {  // the streamed head has produced dhf already
      GemmWeights w;
      w.dense = lm;
      GemmEpilogue e;
      e.out = dhf;
      e.ldo = H;
      NF4_TRY(gemm(logits, V, M, H, V, w, true, GemmExtra(), e, s));
    }
    NF4_TRY(rmsnorm_bwd(xs + (size_t)cfg->n_layers * act, static_cast<const __nv_bfloat16*>(m->norm_final_dev), dhf,
                        nullptr, dh, M, H, lc->rms_eps, s));
  }
  const size_t stride = stride_of(lc);
  Phase bwd_phase(s, 2003);
  return layer_pass(cfg, m, -1, s, [&](int i, const void* shard) {
    nf4ls_lora l;
    nf4ls_lora_grads g;
    lora_views(lc, m->lora_dev + (size_t)i * stride, &l, &g, m->grads_dev + (size_t)i * stride);
    return layer_bwd_impl(lc, shard, &l, xs + (size_t)i * act, dh, dh, &g, at<void>(ws, L.layer), L.total - L.layer,
                          s, i != cfg->n_layers - 1, i != cfg->n_layers - 1);
  });
}

extern "C" int nf4ls_adamw_step(const nf4ls_model_cfg* cfg, const nf4ls_model* m, int32_t step, nf4ls_stream stream) {
  clear_error();
  if (!cfg || !m || !m->lora_dev || !m->grads_dev || !m->adam_m_dev || !m->adam_v_dev || step < 1)
    return fail(NF4LS_INVALID_ARG, "nf4ls_adamw_step: bad argument");
  const size_t n = (size_t)cfg->n_layers * stride_of(&cfg->layer);
  return adamw(m->lora_dev, m->grads_dev, m->adam_m_dev, m->adam_v_dev, n, step, cfg->lr, cfg->beta1, cfg->beta2,
               cfg->adam_eps, cfg->weight_decay, static_cast<cudaStream_t>(stream));
}

extern "C" int nf4ls_train_step(const nf4ls_model_cfg* cfg, const nf4ls_model* m, const int32_t* ids_dev, int32_t step,
                                float* loss_dev, nf4ls_stream stream) {
  NF4_TRY(nf4ls_forward_backward(cfg, m, ids_dev, loss_dev, stream));
  return nf4ls_adamw_step(cfg, m, step, stream);
}

extern "C" int nf4ls_mse_loss(const void* out_dev, size_t n, void* dout_dev, float* loss_dev, float* partial_dev,
                              int n_partial, nf4ls_stream stream) {
  clear_error();
  if (!out_dev || !dout_dev || !loss_dev || !partial_dev || n_partial <= 0 || n_partial > 4096)
    return fail(NF4LS_INVALID_ARG, "nf4ls_mse_loss: bad argument");
  return mse_loss(static_cast<const __nv_bfloat16*>(out_dev), n, partial_dev, n_partial,
                  static_cast<__nv_bfloat16*>(dout_dev), loss_dev, static_cast<cudaStream_t>(stream));
}
