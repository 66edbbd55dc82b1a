"""Stack of decoder layers with resident embedding / lm_head, causal-LM loss and AdamW
(oracle; test infrastructure only).

Follows the training step of the pages' system: frozen NF4 decoder layers,
resident unquantised bf16 embedding and lm_head ("4GB 显存微调 8B 模型是真的",
layer-streaming mechanism section; "Soup 层流式 NF4 训练实测：在 4 GB 显存上以位级一致标准完成 8B 模型 LoRA 微调",
§4.3), LoRA r=16 / alpha=32 on q_proj and v_proj trained with AdamW.

Readings: cross-entropy of logits[t] against ids[t+1] for t = 0..S-2 of each
sequence, mean over batch*(S-1); the last position of each sequence carries
no loss and no gradient.  AdamW with betas (0.9, 0.999), eps 1e-8, weight
decay 0, constant learning rate, bias correction.  The final RMSNorm uses
weight 1 and eps 1e-5.  Tied embeddings use the embedding table as lm_head.
"""
from __future__ import annotations

import numpy as np

from . import bf16, layer


def _R(rnd):
    return bf16.round_f64 if rnd else bf16.ident


def cross_entropy(logits, ids, batch, seq, rnd=True):
    """Returns (loss, dlogits) for logits [batch*seq, V] (float64)."""
    R = _R(rnd)
    M, V = logits.shape
    ids = np.asarray(ids).reshape(batch, seq)
    tgt = np.full((batch, seq), -1, dtype=np.int64)
    tgt[:, :-1] = ids[:, 1:]
    tgt = tgt.reshape(-1)
    valid = tgt >= 0
    count = int(valid.sum())
    mx = logits.max(axis=1, keepdims=True)
    e = np.exp(logits - mx)
    ssum = e.sum(axis=1, keepdims=True)
    lse = (mx + np.log(ssum))[:, 0]
    rows = np.nonzero(valid)[0]
    per = lse[rows] - logits[rows, tgt[rows]]
    loss = float(per.sum() / count)
    d = e / ssum
    d[rows, tgt[rows]] -= 1.0
    d[~valid] = 0.0
    d = R(d / count)
    return loss, d


def adamw(p, g, m, v, step, lr=2e-4, b1=0.9, b2=0.999, eps=1e-8, wd=0.0):
    """One AdamW update (float64).  step counts from 1.  Returns new (p, m, v)."""
    m = b1 * m + (1.0 - b1) * g
    v = b2 * v + (1.0 - b2) * g * g
    mh = m / (1.0 - b1 ** step)
    vh = v / (1.0 - b2 ** step)
    p = p - lr * (mh / (np.sqrt(vh) + eps) + wd * p)
    return p, m, v


def forward_backward(ids, layers, loras, emb, lm_head, w_final, shape, batch, seq, rnd=True,
                     keep=False):
    """One causal-LM forward + backward.  layers: list of dequantised weight dicts;
    loras: list of LoRA dicts (or None); lm_head None means tied to emb.
    Returns (loss, grads list, extras)."""
    R = _R(rnd)
    ids = np.asarray(ids).reshape(-1)
    x = np.asarray(emb, dtype=np.float64)[ids]
    xs = [x]
    saved = []
    for W, lo in zip(layers, loras):
        x, sv = layer.forward(x, W, lo, shape, batch, seq, rnd)
        xs.append(x)
        saved.append(sv if keep else None)
    nf, rf = layer.rmsnorm(x, w_final, shape.rms_eps)
    hf = R(nf)
    lm = np.asarray(emb if lm_head is None else lm_head, dtype=np.float64)
    logits = R(hf @ lm.T)
    loss, dlogits = cross_entropy(logits, ids, batch, seq, rnd)
    dhf = R(dlogits @ lm)
    dh = R(layer.rmsnorm_bwd(x, w_final, rf, dhf))
    grads = [None] * len(layers)
    for i in range(len(layers) - 1, -1, -1):
        _, sv = layer.forward(xs[i], layers[i], loras[i], shape, batch, seq, rnd)
        dh, gr, _ = layer.backward(dh, layers[i], loras[i], shape, batch, seq, sv, rnd)
        grads[i] = gr
    return loss, grads, {"xs": xs, "logits": logits, "dlogits": dlogits, "dx0": dh}
