// layer_forward / layer_backward: one decoder layer of layer-streamed NF4 QLoRA
// training, built from the tcgen05 GEMMs (NF4 decoded in the mainloop) and the body
// kernels.
//
// Forward ("Soup 层流式 NF4 训练实测：在 4 GB 显存上以位级一致标准完成 8B 模型 LoRA 微调" §2.1, the HF Llama layer body):
//   h1  = rmsnorm(x) w_in
//   t   = [h1 A_q^T | h1 A_v^T]                               (LoRA down, bf16)
//   qkv = rope(h1 [Wq;Wk;Wv]^T + t [s B_q; 0; s B_v]^T)       (one GEMM: the LoRA up-
//                                                             projection is a 64-wide extra
//                                                             reduction block; RoPE in the
//                                                             epilogue)
//   o   = causal GQA attention(q, k, v)
//   h   = x + o Wo^T                                          (residual in the epilogue)
//   h2  = rmsnorm(h) w_post
//   a   = silu(h2 Wg^T) * (h2 Wu^T)                           (one GEMM, SwiGLU epilogue)
//   y   = h + a Wd^T
// Backward with checkpoint recompute (the layer-streaming review, mechanism section:
// every layer is read twice per step and dL/dx = W^T dL/dy flows through the frozen
// base; "Soup 层流式 NF4 训练实测：在 4 GB 显存上以位级一致标准完成 8B 模型 LoRA 微调" §4.4:
// no dL/dW): the forward is re-run from the saved
// input, keeping g and u, then
//   [dg | du] = dSwiGLU(dy Wd)                                (dSwiGLU in the epilogue)
//   dh  = dy + rmsnorm_bwd(h, dg Wg + du Wu)                  (one GEMM over [Wg; Wu])
//   do  = dh Wo;  dq, dk, dv = attention_bwd;  RoPE^T on dq, dk
//   dB = s dq^T t, dt = s dq B, dA = dt^T h1                  (q and v adapters)
//   dx  = dh + rmsnorm_bwd(x, [dq|dk|dv] [Wq;Wk;Wv] + dt [A_q; A_v])
#include <algorithm>

#include "common.cuh"
#include "internal.h"

namespace nf4ls {

namespace {

struct WsLayout {
  size_t cos, sin, cos_t, sin_t, h1, qkv, tpad, bup, adn, o, lse, h, h2, gu, act, dgu, dh2, dh, dO, dqkv, delta, bqt, bvt, part,
      dtpad, dh1, dense, total;
};

WsLayout ws_layout(const nf4ls_layer_cfg* c) {
  const size_t M = (size_t)c->batch * c->seq, H = c->hidden, I = c->inter;
  const size_t qd = (size_t)c->n_q * c->head_dim, kvd = (size_t)c->n_kv * c->head_dim, nqkv = qd + 2 * kvd;
  WsLayout L;
  size_t off = 0;
  auto take = [&](size_t bytes) {
    const size_t o = off;
    off = round_up(off + bytes, 256);
    return o;
  };
  L.cos = take((size_t)c->seq * c->head_dim / 2 * 4);
  L.sin = take((size_t)c->seq * c->head_dim / 2 * 4);
  L.cos_t = take((size_t)c->seq * c->head_dim / 2 * 4);
  L.sin_t = take((size_t)c->seq * c->head_dim / 2 * 4);
  L.h1 = take(M * H * 2);
  L.qkv = take(M * nqkv * 2);
  L.tpad = take(M * 64 * 2);
  L.bup = take(nqkv * 64 * 2);
  L.adn = take(64 * H * 2);
  L.o = take(M * qd * 2);
  L.lse = take((size_t)c->batch * c->n_q * c->seq * 4);
  L.h = take(M * H * 2);
  L.h2 = take(M * H * 2);
  L.gu = take(M * 2 * I * 2);
  L.act = take(M * I * 2);
  L.dgu = take(M * 2 * I * 2);
  L.dh2 = take(M * H * 2);
  L.dh = take(M * H * 2);
  L.dO = take(M * qd * 2);
  L.dqkv = take(M * nqkv * 2);
  L.delta = take((size_t)c->batch * c->n_q * c->seq * 4);
  L.bqt = take(16 * qd * 2);
  L.bvt = take(16 * kvd * 2);
  L.part = take(lora_partial_bytes((int)M, (int)H, (int)qd, (int)kvd));
  L.dtpad = take(M * 64 * 2);
  L.dh1 = take(M * H * 2);
  // bf16 copy of the layer's seven linears for the dequantise-then-multiply path
  L.dense = take((nqkv * H + H * qd + 3 * I * H) * 2);
  L.total = off;
  return L;
}

template <typename T>
T* at(void* ws, size_t off) {
  return reinterpret_cast<T*>(static_cast<uint8_t*>(ws) + off);
}

struct LayerCtx {
  const nf4ls_layer_cfg* c;
  ShardView v;
  WsLayout L;
  void* ws;
  int M, H, I, qd, kvd, nqkv;
  float scale;
  // weights of the four GEMM groups
  GemmWeights w_qkv, w_o, w_gu, w_down;
};

int prepare(LayerCtx& x, const nf4ls_layer_cfg* c, const void* shard, void* ws, size_t ws_bytes, cudaStream_t s,
            bool tables_ready) {
  NF4_TRY(check_cfg(c));
  if (!shard || !ws) return fail(NF4LS_INVALID_ARG, "layer: null shard or workspace");
  if (!aligned(shard, 256) || !aligned(ws, 256)) return fail(NF4LS_ALIGN, "layer: shard and workspace must be 256-byte aligned");
  x.c = c;
  x.L = ws_layout(c);
  if (ws_bytes < x.L.total) return fail(NF4LS_INVALID_ARG, "layer: workspace %zu < %zu bytes", ws_bytes, x.L.total);
  shard_view(c, shard, &x.v);
  x.ws = ws;
  x.M = c->batch * c->seq;
  x.H = c->hidden;
  x.I = c->inter;
  x.qd = c->n_q * c->head_dim;
  x.kvd = c->n_kv * c->head_dim;
  x.nqkv = x.qd + 2 * x.kvd;
  x.scale = c->lora_alpha / (float)c->lora_r;
  x.w_qkv = GemmWeights();
  x.w_o = GemmWeights();
  x.w_gu = GemmWeights();
  x.w_down = GemmWeights();
  if (gemm_path() == 1) {
    __nv_bfloat16* d = at<__nv_bfloat16>(ws, x.L.dense);
    size_t off = 0;
    __nv_bfloat16* ptr[7];
    for (int t = 0; t < 7; ++t) {
      const NF4Tensor& T = x.v.t[t];
      ptr[t] = d + off;
      const size_t n = (size_t)T.rows * T.cols;
      NF4_TRY(dequantize_tensor(T.packed, T.q8, T.nested, T.offset, n, ptr[t], s));
      off += n;
    }
    x.w_qkv.dense = ptr[0];   // q, k, v contiguous
    x.w_o.dense = ptr[3];
    x.w_gu.dense = ptr[4];    // gate, up contiguous
    x.w_down.dense = ptr[6];
  } else {
    x.w_qkv.n_seg = 3;
    x.w_qkv.seg[0] = x.v.t[0];
    x.w_qkv.seg[1] = x.v.t[1];
    x.w_qkv.seg[2] = x.v.t[2];
    x.w_o.n_seg = 1;
    x.w_o.seg[0] = x.v.t[3];
    x.w_gu.n_seg = 2;
    x.w_gu.seg[0] = x.v.t[4];
    x.w_gu.seg[1] = x.v.t[5];
    x.w_down.n_seg = 1;
    x.w_down.seg[0] = x.v.t[6];
  }
  if (tables_ready) return NF4LS_OK;
  return rope_tables(at<float>(ws, x.L.cos), at<float>(ws, x.L.sin), at<float>(ws, x.L.cos_t),
                     at<float>(ws, x.L.sin_t), c->seq, c->head_dim, c->rope_theta, s);
}

// Forward body up to the SwiGLU activation; y (optional) gets the layer output.
int forward_body(LayerCtx& x, const nf4ls_lora* lora, const __nv_bfloat16* X, __nv_bfloat16* y, bool keep_gu,
                 cudaStream_t s) {
  const nf4ls_layer_cfg* c = x.c;
  void* ws = x.ws;
  const int M = x.M, H = x.H, I = x.I;
  auto* h1 = at<__nv_bfloat16>(ws, x.L.h1);
  auto* qkv = at<__nv_bfloat16>(ws, x.L.qkv);
  auto* o = at<__nv_bfloat16>(ws, x.L.o);
  auto* h = at<__nv_bfloat16>(ws, x.L.h);
  auto* h2 = at<__nv_bfloat16>(ws, x.L.h2);
  auto* act = at<__nv_bfloat16>(ws, x.L.act);
  auto* tpad = at<__nv_bfloat16>(ws, x.L.tpad);
  GemmExtra ex;
  if (lora) {
    // one launch: the input RMSNorm, the adapter's bf16 operands and
    // t = [h1 A_q^T | h1 A_v^T] (columns 0-31 of the padded extra operand)
    LoraPack pk;
    pk.Aq = lora->A_q;
    pk.Av = lora->A_v;
    pk.Bq = lora->B_q;
    pk.Bv = lora->B_v;
    pk.H = H;
    pk.qd = x.qd;
    pk.kvd = x.kvd;
    pk.scale = x.scale;
    pk.bup = at<__nv_bfloat16>(ws, x.L.bup);
    pk.adn = at<__nv_bfloat16>(ws, x.L.adn);
    pk.bqt = at<__nv_bfloat16>(ws, x.L.bqt);
    pk.bvt = at<__nv_bfloat16>(ws, x.L.bvt);
    NF4_TRY(rmsnorm_lora_fwd(X, x.v.norm_in, h1, M, H, c->rms_eps, pk, tpad, s));
    ex.a = tpad;
    ex.b = pk.bup;
  } else {
    NF4_TRY(rmsnorm_fwd(X, x.v.norm_in, h1, M, H, c->rms_eps, s));
  }
  GemmEpilogue e;
  e.kind = EPI_ROPE;
  e.out = qkv;
  e.ldo = x.nqkv;
  e.rope_cos = at<float>(ws, x.L.cos_t);
  e.rope_sin = at<float>(ws, x.L.sin_t);
  e.seq = c->seq;
  e.head_dim = c->head_dim;
  e.rope_cols = x.qd + x.kvd;
  NF4_TRY(gemm(h1, H, M, x.nqkv, H, x.w_qkv, false, ex, e, s));
  NF4_TRY(attention_fwd(qkv, qkv + x.qd, qkv + x.qd + x.kvd, x.nqkv, x.nqkv, o, x.qd, at<float>(ws, x.L.lse), c->batch,
                        c->seq, c->n_q, c->n_kv, c->head_dim, s));
  GemmEpilogue eo;
  eo.kind = EPI_RESID;
  eo.out = h;
  eo.ldo = H;
  eo.aux0 = X;
  eo.ld_aux0 = H;
  NF4_TRY(gemm(o, x.qd, M, H, x.qd, x.w_o, false, GemmExtra(), eo, s));
  NF4_TRY(rmsnorm_fwd(h, x.v.norm_post, h2, M, H, c->rms_eps, s));
  GemmEpilogue eg;
  eg.kind = EPI_SWIGLU;
  eg.out = act;
  eg.ldo = I;
  eg.inter = I;
  if (keep_gu) {
    eg.aux_out = at<__nv_bfloat16>(ws, x.L.gu);
    eg.ld_aux_out = 2 * I;
  }
  NF4_TRY(gemm(h2, H, M, 2 * I, H, x.w_gu, false, GemmExtra(), eg, s));
  if (y) {
    GemmEpilogue ed;
    ed.kind = EPI_RESID;
    ed.out = y;
    ed.ldo = H;
    ed.aux0 = h;
    ed.ld_aux0 = H;
    NF4_TRY(gemm(act, I, M, H, I, x.w_down, false, GemmExtra(), ed, s));
  }
  return NF4LS_OK;
}

}  // namespace

size_t layer_ws_bytes(const nf4ls_layer_cfg* cfg) { return ws_layout(cfg).total; }

int layer_fwd_impl(const nf4ls_layer_cfg* c, const void* shard, const nf4ls_lora* lora, const __nv_bfloat16* X,
                   __nv_bfloat16* y, void* ws, size_t ws_bytes, cudaStream_t s, bool tables_ready, bool keep) {
  if (!X || !y) return fail(NF4LS_INVALID_ARG, "layer_forward: null activation");
  LayerCtx x;
  NF4_TRY(prepare(x, c, shard, ws, ws_bytes, s, tables_ready));
  return forward_body(x, lora, X, y, keep, s);
}

int layer_bwd_impl(const nf4ls_layer_cfg* c, const void* shard, const nf4ls_lora* lora, const __nv_bfloat16* X,
                   const __nv_bfloat16* dy, __nv_bfloat16* dx, const nf4ls_lora_grads* g, void* ws, size_t ws_bytes,
                   cudaStream_t s, bool tables_ready, bool recompute) {
  if (!X || !dy || !dx) return fail(NF4LS_INVALID_ARG, "layer_backward: null activation");
  if (lora && (!g || !g->dA_q || !g->dB_q || !g->dA_v || !g->dB_v))
    return fail(NF4LS_INVALID_ARG, "layer_backward: LoRA gradients needed when the adapter is on");
  LayerCtx x;
  NF4_TRY(prepare(x, c, shard, ws, ws_bytes, s, tables_ready));
  // checkpoint recompute (keeps g and u for the SwiGLU backward), unless the workspace
  // still holds this layer's forward with g and u kept
  if (recompute) NF4_TRY(forward_body(x, lora, X, nullptr, true, s));
  const int M = x.M, H = x.H, I = x.I;
  auto* gu = at<__nv_bfloat16>(ws, x.L.gu);
  auto* dgu = at<__nv_bfloat16>(ws, x.L.dgu);
  auto* dh2 = at<__nv_bfloat16>(ws, x.L.dh2);
  auto* dh = at<__nv_bfloat16>(ws, x.L.dh);
  auto* dO = at<__nv_bfloat16>(ws, x.L.dO);
  auto* dqkv = at<__nv_bfloat16>(ws, x.L.dqkv);
  auto* dh1 = at<__nv_bfloat16>(ws, x.L.dh1);
  auto* qkv = at<__nv_bfloat16>(ws, x.L.qkv);
  auto* h = at<__nv_bfloat16>(ws, x.L.h);
  auto* h1 = at<__nv_bfloat16>(ws, x.L.h1);
  auto* o = at<__nv_bfloat16>(ws, x.L.o);
  // down projection: [dg | du] from dy Wd and the kept g, u
  GemmEpilogue e1;
  e1.kind = EPI_DSWIGLU;
  e1.out = dgu;
  e1.ldo = 2 * I;
  e1.aux0 = gu;
  e1.ld_aux0 = 2 * I;
  e1.inter = I;
  NF4_TRY(gemm(dy, H, M, I, H, x.w_down, true, GemmExtra(), e1, s));
  // gate/up: dh2 = [dg | du] [Wg; Wu]
  GemmEpilogue e2;
  e2.out = dh2;
  e2.ldo = H;
  NF4_TRY(gemm(dgu, 2 * I, M, H, 2 * I, x.w_gu, true, GemmExtra(), e2, s));
  NF4_TRY(rmsnorm_bwd(h, x.v.norm_post, dh2, dy, dh, M, H, c->rms_eps, s));
  // o projection
  GemmEpilogue e3;
  e3.out = dO;
  e3.ldo = x.qd;
  NF4_TRY(gemm(dh, H, M, x.qd, H, x.w_o, true, GemmExtra(), e3, s));
  NF4_TRY(attention_bwd(qkv, qkv + x.qd, qkv + x.qd + x.kvd, x.nqkv, x.nqkv, o, dO, x.qd, at<float>(ws, x.L.lse),
                        at<float>(ws, x.L.delta), dqkv, dqkv + x.qd, dqkv + x.qd + x.kvd, x.nqkv, x.nqkv, c->batch, c->seq,
                        c->n_q, c->n_kv, c->head_dim, s));
  NF4_TRY(rope_bwd(dqkv, x.nqkv, M, x.qd + x.kvd, c->seq, c->head_dim, at<float>(ws, x.L.cos), at<float>(ws, x.L.sin), s));
  GemmExtra ex;
  SideStream side;
  auto lora_phases = [&](int phases, cudaStream_t st) {
    return lora_bwd(dqkv, x.nqkv, x.qd + x.kvd, M, H, x.qd, x.kvd, at<__nv_bfloat16>(ws, x.L.tpad),
                    at<__nv_bfloat16>(ws, x.L.bqt), at<__nv_bfloat16>(ws, x.L.bvt), h1, x.scale,
                    at<__nv_bfloat16>(ws, x.L.dtpad), g, at<void>(ws, x.L.part), phases, st);
  };
  if (lora) {
    // dt = s [dq B_q | dv B_v] (bf16, the extra operand of the dL/dx GEMM) ...
    NF4_TRY(lora_phases(LORA_BWD_DT, s));
    ex.a = at<__nv_bfloat16>(ws, x.L.dtpad);
    ex.b = at<__nv_bfloat16>(ws, x.L.adn);
    NF4_TRY(side.fork(s));
  }
  GemmEpilogue e4;
  e4.out = dh1;
  e4.ldo = H;
  NF4_TRY(gemm(dqkv, x.nqkv, M, H, x.nqkv, x.w_qkv, true, ex, e4, s));
  if (lora) {
    // ... and dB = s [dq^T t_q | dv^T t_v], dA = dt^T h1 beside the GEMM, which leaves SMs
    // idle (at M = 2048 and H = 4096 its 64 pair tiles hold 128 of 148), enqueued after it
    // so that its CTAs are placed first
    NF4_TRY(lora_phases(LORA_BWD_DB_DA, side.side()));
    NF4_TRY(side.join(s));
  }
  return rmsnorm_bwd(X, x.v.norm_in, dh1, dh, dx, M, H, c->rms_eps, s);
}

}  // namespace nf4ls

using namespace nf4ls;

extern "C" size_t nf4ls_workspace_bytes(const nf4ls_layer_cfg* cfg) {
  if (!cfg) return 0;
  return layer_ws_bytes(cfg);
}

extern "C" int layer_forward(const nf4ls_layer_cfg* cfg, const void* shard_dev, const nf4ls_lora* lora, const void* x_dev,
                             void* y_dev, void* ws_dev, size_t ws_bytes, nf4ls_stream stream) {
  clear_error();
  return layer_fwd_impl(cfg, shard_dev, lora, static_cast<const __nv_bfloat16*>(x_dev), static_cast<__nv_bfloat16*>(y_dev),
                        ws_dev, ws_bytes, static_cast<cudaStream_t>(stream));
}

extern "C" int layer_backward(const nf4ls_layer_cfg* cfg, const void* shard_dev, const nf4ls_lora* lora,
                              const void* x_saved_dev, const void* dy_dev, void* dx_dev, const nf4ls_lora_grads* grads,
                              void* ws_dev, size_t ws_bytes, nf4ls_stream stream) {
  clear_error();
  return layer_bwd_impl(cfg, shard_dev, lora, static_cast<const __nv_bfloat16*>(x_saved_dev),
                        static_cast<const __nv_bfloat16*>(dy_dev), static_cast<__nv_bfloat16*>(dx_dev), grads, ws_dev,
                        ws_bytes, static_cast<cudaStream_t>(stream));
}
