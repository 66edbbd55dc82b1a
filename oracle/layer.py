"""One Llama-style decoder layer, forward and hand-derived backward (oracle; test infrastructure only).

The layer body is the HF Llama decoder layer that the pages' system runs
through ``functional_call`` ("Soup 层流式 NF4 训练实测：在 4 GB 显存上以位级一致标准完成 8B 模型 LoRA 微调",
m.mzlw.cn, §2.1): RMSNorm -> q/k/v projections (+ LoRA on q and v) -> RoPE ->
causal GQA softmax attention -> o projection + residual -> RMSNorm ->
SiLU(gate) * up -> down projection + residual.  The frozen base linears use the
dequantised NF4 weights; the backward computes dL/dx through them (no dL/dW:
"dL/dx = W^T dL/dy", §4.4 and the layer-streaming mechanism section of
"4GB 显存微调 8B 模型是真的") plus the LoRA gradients dA and dB.

Arithmetic is float64.  ``R`` is bf16 rounding (``rnd=True``) or the identity
(``rnd=False``); it is applied where the CUDA path stores a bf16 tensor:

  h1 = R(rmsnorm(x) * w_in)
  t_q = R(h1 A_q^T), t_v = R(h1 A_v^T)                 A, B rounded to bf16
  q = R(rope(h1 Wq^T + s t_q B_q^T)), k = R(rope(h1 Wk^T)), v = R(h1 Wv^T + s t_v B_v^T)
  o = R(attention(q, k, v))
  h = R(x + o Wo^T)
  h2 = R(rmsnorm(h) * w_post)
  g = R(h2 Wg^T), u = R(h2 Wu^T), a = R(silu(g) u)
  out = R(h + a Wd^T)

with s = lora_alpha / lora_r.  Readings: RMSNorm eps 1e-5; rotate-half RoPE
with inv_freq_i = theta^(-2i/d) at positions 0..S-1 of each sequence and no
frequency rescaling; LoRA dropout 0.
"""
from __future__ import annotations

import numpy as np

from . import bf16


def _R(rnd: bool):
    return bf16.round_f64 if rnd else bf16.ident


def rmsnorm(x, w, eps):
    r = 1.0 / np.sqrt(np.mean(x * x, axis=-1, keepdims=True) + eps)
    return x * r * w, r


def rmsnorm_bwd(x, w, r, dy):
    """dx of y = x * r * w with r = (mean(x^2) + eps)^(-1/2); w is frozen."""
    g = dy * w
    H = x.shape[-1]
    return r * g - x * (r ** 3) * np.sum(g * x, axis=-1, keepdims=True) / H


def rope_tables(seq: int, d: int, theta: float):
    inv = theta ** (-(2.0 * np.arange(d // 2, dtype=np.float64)) / d)
    ang = np.arange(seq, dtype=np.float64)[:, None] * inv[None, :]
    return np.cos(ang), np.sin(ang)


def rope(x, cos, sin):
    """x [B, S, heads, d]; rotate-half pairing (i, i + d/2)."""
    h = x.shape[-1] // 2
    x1, x2 = x[..., :h], x[..., h:]
    c, s = cos[None, :, None, :], sin[None, :, None, :]
    return np.concatenate([x1 * c - x2 * s, x2 * c + x1 * s], axis=-1)


def rope_bwd(dy, cos, sin):
    h = dy.shape[-1] // 2
    d1, d2 = dy[..., :h], dy[..., h:]
    c, s = cos[None, :, None, :], sin[None, :, None, :]
    return np.concatenate([d1 * c + d2 * s, d2 * c - d1 * s], axis=-1)


def attention(q, k, v):
    """Causal GQA softmax attention.  q [B,S,nq,d], k/v [B,S,nkv,d] -> o, probs."""
    B, S, nq, d = q.shape
    nkv = k.shape[2]
    grp = nq // nkv
    o = np.empty_like(q)
    P = np.empty((B, nq, S, S))
    mask = np.triu(np.ones((S, S), dtype=bool), 1)
    for b in range(B):
        for h in range(nq):
            kv = h // grp
            s = q[b, :, h, :] @ k[b, :, kv, :].T / np.sqrt(d)
            s[mask] = -np.inf
            s = s - s.max(axis=1, keepdims=True)
            p = np.exp(s)
            p /= p.sum(axis=1, keepdims=True)
            P[b, h] = p
            o[b, :, h, :] = p @ v[b, :, kv, :]
    return o, P


def attention_bwd(q, k, v, P, do):
    B, S, nq, d = q.shape
    nkv = k.shape[2]
    grp = nq // nkv
    dq = np.zeros_like(q)
    dk = np.zeros_like(k)
    dv = np.zeros_like(v)
    for b in range(B):
        for h in range(nq):
            kv = h // grp
            p = P[b, h]
            dv[b, :, kv, :] += p.T @ do[b, :, h, :]
            dp = do[b, :, h, :] @ v[b, :, kv, :].T
            ds = p * (dp - np.sum(dp * p, axis=1, keepdims=True))
            dq[b, :, h, :] = ds @ k[b, :, kv, :] / np.sqrt(d)
            dk[b, :, kv, :] += ds.T @ q[b, :, h, :] / np.sqrt(d)
    return dq, dk, dv


def sigmoid(x):
    return 1.0 / (1.0 + np.exp(-x))


def silu(x):
    return x * sigmoid(x)


def dsilu(x):
    s = sigmoid(x)
    return s * (1.0 + x * (1.0 - s))


def forward(x, W, lora, shape, batch, seq, rnd=True):
    """x: [batch*seq, H] float64 of bf16 values.  W: dict of float64 dequantised
    weights (q, k, v, o, gate, up, down [out, in]; norm_in, norm_post [H]).
    lora: dict A_q, B_q, A_v, B_v (float64 masters) or None (adapter off).
    Returns (out, saved) with every intermediate the backward needs."""
    R = _R(rnd)
    d, nq, nkv = shape.head_dim, shape.n_q, shape.n_kv
    s = shape.lora_alpha / shape.lora_r
    X = np.asarray(x, dtype=np.float64)
    M = X.shape[0]
    n1, r1 = rmsnorm(X, W["norm_in"], shape.rms_eps)
    h1 = R(n1)
    q_pre = h1 @ W["q"].T
    k_pre = h1 @ W["k"].T
    v_pre = h1 @ W["v"].T
    sv = {}
    if lora is not None:
        Aq, Bq, Av, Bv = (R(lora[n]) for n in ("A_q", "B_q", "A_v", "B_v"))
        t_q = R(h1 @ Aq.T)
        t_v = R(h1 @ Av.T)
        q_pre = q_pre + s * (t_q @ Bq.T)
        v_pre = v_pre + s * (t_v @ Bv.T)
        sv.update(t_q=t_q, t_v=t_v, Aq=Aq, Bq=Bq, Av=Av, Bv=Bv)
    cos, sin = rope_tables(seq, d, shape.rope_theta)
    q = R(rope(q_pre.reshape(batch, seq, nq, d), cos, sin))
    k = R(rope(k_pre.reshape(batch, seq, nkv, d), cos, sin))
    v = R(v_pre).reshape(batch, seq, nkv, d)
    o4, P = attention(q, k, v)
    o = R(o4.reshape(M, nq * d))
    h = R(X + o @ W["o"].T)
    n2, r2 = rmsnorm(h, W["norm_post"], shape.rms_eps)
    h2 = R(n2)
    g = R(h2 @ W["gate"].T)
    u = R(h2 @ W["up"].T)
    a = R(silu(g) * u)
    out = R(h + a @ W["down"].T)
    sv.update(x=X, r1=r1, h1=h1, q=q, k=k, v=v, P=P, o=o, h=h, r2=r2, h2=h2, g=g, u=u, a=a,
              cos=cos, sin=sin, out=out)
    return out, sv


def backward(dout, W, lora, shape, batch, seq, sv, rnd=True):
    """Recompute-free backward given the forward's saved tensors ``sv``.
    Returns (dx, grads) with grads = dict dA_q, dB_q, dA_v, dB_v (or {} when lora is None)."""
    R = _R(rnd)
    d, nq, nkv = shape.head_dim, shape.n_q, shape.n_kv
    s = shape.lora_alpha / shape.lora_r
    M = dout.shape[0]
    dout = np.asarray(dout, dtype=np.float64)
    # down projection and SiLU-gated MLP (da stays fp32 inside the fused epilogue)
    da = dout @ W["down"]
    g, u = sv["g"], sv["u"]
    dg = R(da * u * dsilu(g))
    du = R(da * silu(g))
    dh2 = R(dg @ W["gate"] + du @ W["up"])
    dh = R(dout + rmsnorm_bwd(sv["h"], W["norm_post"], sv["r2"], dh2))
    # o projection and attention
    do = R(dh @ W["o"]).reshape(batch, seq, nq, d)
    dq4, dk4, dv4 = attention_bwd(sv["q"], sv["k"], sv["v"], sv["P"], do)
    dq_post, dk_post, dv = R(dq4), R(dk4), R(dv4)
    dq = R(rope_bwd(dq_post, sv["cos"], sv["sin"])).reshape(M, nq * d)
    dk = R(rope_bwd(dk_post, sv["cos"], sv["sin"])).reshape(M, nkv * d)
    dv = dv.reshape(M, nkv * d)
    dh1 = dq @ W["q"] + dk @ W["k"] + dv @ W["v"]
    grads = {}
    if lora is not None:
        h1 = sv["h1"]
        dB_q = s * (dq.T @ sv["t_q"])
        dB_v = s * (dv.T @ sv["t_v"])
        dt_q = s * (dq @ sv["Bq"])
        dt_v = s * (dv @ sv["Bv"])
        dA_q = dt_q.T @ h1
        dA_v = dt_v.T @ h1
        dh1 = dh1 + R(dt_q) @ sv["Aq"] + R(dt_v) @ sv["Av"]
        grads = {"dA_q": dA_q, "dB_q": dB_q, "dA_v": dA_v, "dB_v": dB_v}
    dh1 = R(dh1)
    dx = R(dh + rmsnorm_bwd(sv["x"], W["norm_in"], sv["r1"], dh1))
    inter = {"da": da, "dg": dg, "du": du, "dh2": dh2, "dh": dh, "do": do.reshape(M, nq * d),
             "dq": dq, "dk": dk, "dv": dv, "dh1": dh1}
    return dx, grads, inter


def mse_loss(out):
    """Loss of the single-layer workloads: mean of out^2 over batch*seq*hidden."""
    return float(np.mean(out * out)), 2.0 * out / out.size
