"""Pins of the oracle's layer, loss, optimiser and accounting (CPU only).

Pins: library routines run independently of the oracle (torch rms_norm,
scaled_dot_product_attention, torch.optim.AdamW, scipy logsumexp, and torch autograd
through rms_norm, scaled_dot_product_attention and cross_entropy for the backward
pieces), RoPE as a complex rotation with its adjoint as the backward, float64
central finite differences on tiny shapes with bf16 rounding off, structural
LoRA facts that "Soup 层流式 NF4 训练实测：在 4 GB 显存上以位级一致标准完成 8B 模型 LoRA 微调"
§2.2 and §2.5 rely on (B = 0 gives an exactly zero adapter
output and dA = 0; a random B makes every gradient nonzero), and the page's
GFLOP-per-token table.
"""
import json
import math
import os

import numpy as np
import pytest
import torch
from scipy.special import logsumexp

from oracle import account, layer, model
from nf4_layer_streamed_b200 import synth

GOLD = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "pages_figures.json")))


def _weights(shape, seed=5, scale=0.05):
    rng = np.random.default_rng(seed)
    W = {n: rng.normal(0, scale, s) for n, s in shape.weight_shapes()}
    W["norm_in"] = 1.0 + 0.1 * rng.normal(size=shape.hidden)
    W["norm_post"] = 1.0 + 0.1 * rng.normal(size=shape.hidden)
    return W


def _lora(shape, seed=6, b_random=True):
    rng = np.random.default_rng(seed)
    r = shape.lora_r
    return {"A_q": rng.normal(0, 0.1, (r, shape.hidden)),
            "B_q": rng.normal(0, 0.1, (shape.q_dim, r)) if b_random else np.zeros((shape.q_dim, r)),
            "A_v": rng.normal(0, 0.1, (r, shape.hidden)),
            "B_v": rng.normal(0, 0.1, (shape.kv_dim, r)) if b_random else np.zeros((shape.kv_dim, r))}


def test_rmsnorm_matches_torch():
    rng = np.random.default_rng(0)
    x = rng.normal(size=(7, 64))
    w = rng.normal(size=64)
    y, _ = layer.rmsnorm(x, w, 1e-5)
    ref = torch.nn.functional.rms_norm(torch.tensor(x), (64,), torch.tensor(w), eps=1e-5).numpy()
    np.testing.assert_allclose(y, ref, rtol=1e-12, atol=1e-12)


def test_attention_matches_torch_sdpa():
    rng = np.random.default_rng(1)
    B, S, nq, nkv, d = 2, 9, 4, 2, 16
    q, k, v = rng.normal(size=(B, S, nq, d)), rng.normal(size=(B, S, nkv, d)), rng.normal(size=(B, S, nkv, d))
    o, _ = layer.attention(q, k, v)
    tq = torch.tensor(q).transpose(1, 2)
    tk = torch.tensor(k).transpose(1, 2).repeat_interleave(nq // nkv, dim=1)
    tv = torch.tensor(v).transpose(1, 2).repeat_interleave(nq // nkv, dim=1)
    ref = torch.nn.functional.scaled_dot_product_attention(tq, tk, tv, is_causal=True).transpose(1, 2).numpy()
    np.testing.assert_allclose(o, ref, rtol=1e-10, atol=1e-10)


def test_rope_rotation_properties():
    rng = np.random.default_rng(2)
    cos, sin = layer.rope_tables(11, 32, 10000.0)
    x = rng.normal(size=(1, 11, 3, 32))
    y = layer.rope(x, cos, sin)
    np.testing.assert_allclose(y[:, 0], x[:, 0], atol=1e-15)       # position 0 is the identity
    n = lambda a: a[..., :16] ** 2 + a[..., 16:] ** 2
    np.testing.assert_allclose(n(y), n(x), rtol=1e-12)               # pairs keep their norm
    np.testing.assert_allclose(layer.rope_bwd(y, cos, sin), x, atol=1e-12)  # transpose = inverse
    # pair (i, i+d/2) at position p turns by p * theta^(-2i/d)
    p, i = 5, 3
    ang = p * 10000.0 ** (-2 * i / 32)
    z = np.zeros((1, 11, 1, 32)); z[0, p, 0, i] = 1.0
    r = layer.rope(z, cos, sin)
    assert math.isclose(r[0, p, 0, i], math.cos(ang)) and math.isclose(r[0, p, 0, i + 16], math.sin(ang))


def _fd_check(f, x, grad, n_dirs=4, eps=1e-6, seed=0):
    rng = np.random.default_rng(seed)
    for _ in range(n_dirs):
        e = rng.normal(size=x.shape)
        num = (f(x + eps * e) - f(x - eps * e)) / (2 * eps)
        ana = float(np.sum(grad * e))
        assert abs(num - ana) <= 1e-6 * max(1.0, abs(ana)), (num, ana)


@pytest.mark.parametrize("batch,seq", [(1, 8), (2, 5)])
def test_layer_backward_finite_differences(batch, seq):
    shape = synth.TINY
    W = _weights(shape)
    lo = _lora(shape, b_random=True)
    rng = np.random.default_rng(9)
    x = rng.normal(size=(batch * seq, shape.hidden))
    c = rng.normal(size=(batch * seq, shape.hidden))

    def L(xx, lora=lo):
        out, _ = layer.forward(xx, W, lora, shape, batch, seq, rnd=False)
        return float(np.sum(out * c))

    out, sv = layer.forward(x, W, lo, shape, batch, seq, rnd=False)
    dx, gr, _ = layer.backward(c, W, lo, shape, batch, seq, sv, rnd=False)
    _fd_check(L, x, dx)
    for key, name in (("dA_q", "A_q"), ("dB_q", "B_q"), ("dA_v", "A_v"), ("dB_v", "B_v")):
        def Lp(p, name=name):
            l2 = dict(lo); l2[name] = p
            return L(x, l2)
        _fd_check(Lp, lo[name], gr[key])


def test_lora_b_zero_is_structurally_inert():
    shape = synth.TINY
    W = _weights(shape)
    lo = _lora(shape, b_random=False)
    rng = np.random.default_rng(10)
    x = rng.normal(size=(8, shape.hidden))
    out_on, sv = layer.forward(x, W, lo, shape, 1, 8, rnd=True)
    out_off, _ = layer.forward(x, W, None, shape, 1, 8, rnd=True)
    assert np.array_equal(out_on, out_off)
    _, dout = layer.mse_loss(out_on)
    _, gr, _ = layer.backward(dout, W, lo, shape, 1, 8, sv, rnd=True)
    assert np.all(gr["dA_q"] == 0) and np.all(gr["dA_v"] == 0)
    assert np.any(gr["dB_q"] != 0) and np.any(gr["dB_v"] != 0)
    lo2 = _lora(shape, b_random=True)
    out2, sv2 = layer.forward(x, W, lo2, shape, 1, 8, rnd=True)
    _, gr2, _ = layer.backward(layer.mse_loss(out2)[1], W, lo2, shape, 1, 8, sv2, rnd=True)
    for k in ("dA_q", "dB_q", "dA_v", "dB_v"):
        assert np.any(gr2[k] != 0), k


def test_silu_derivative():
    x = np.linspace(-6, 6, 101)
    e = 1e-6
    np.testing.assert_allclose(layer.dsilu(x), (layer.silu(x + e) - layer.silu(x - e)) / (2 * e), atol=1e-8)


def test_cross_entropy_against_logsumexp():
    rng = np.random.default_rng(3)
    B, S, V = 2, 6, 50
    logits = rng.normal(size=(B * S, V))
    ids = rng.integers(0, V, (B, S))
    loss, d = model.cross_entropy(logits, ids, B, S, rnd=False)
    ref = []
    for b in range(B):
        for t in range(S - 1):
            row = logits[b * S + t]
            ref.append(logsumexp(row) - row[ids[b, t + 1]])
    assert math.isclose(loss, float(np.mean(ref)), rel_tol=1e-12)
    assert np.all(d.reshape(B, S, V)[:, -1] == 0)

    def L(lg):
        return model.cross_entropy(lg, ids, B, S, rnd=False)[0]
    _fd_check(L, logits, d)


def test_cross_entropy_uniform_logits_is_log_vocab():
    V = 49152
    loss, _ = model.cross_entropy(np.zeros((4, V)), np.arange(4).reshape(1, 4), 1, 4, rnd=False)
    assert math.isclose(loss, math.log(V), rel_tol=1e-12)


def test_adamw_matches_torch():
    rng = np.random.default_rng(4)
    p0 = rng.normal(size=(5, 7))
    tp = torch.tensor(p0, requires_grad=True)
    opt = torch.optim.AdamW([tp], lr=2e-4, betas=(0.9, 0.999), eps=1e-8, weight_decay=0.0)
    p, m, v = p0.copy(), np.zeros_like(p0), np.zeros_like(p0)
    for step in range(1, 4):
        g = rng.normal(size=p0.shape)
        tp.grad = torch.tensor(g)
        opt.step()
        p, m, v = model.adamw(p, g, m, v, step)
    np.testing.assert_allclose(p, tp.detach().numpy(), rtol=0, atol=1e-14)


def test_model_lora_gradient_finite_differences():
    shape = synth.TINY
    V, B, S = 40, 1, 6
    rng = np.random.default_rng(12)
    layers = [_weights(shape, seed=20 + i) for i in range(2)]
    loras = [_lora(shape, seed=30 + i, b_random=True) for i in range(2)]
    emb = rng.normal(0, 0.5, (V, shape.hidden))
    wf = np.ones(shape.hidden)
    ids = rng.integers(0, V, (B, S))
    loss, grads, _ = model.forward_backward(ids, layers, loras, emb, None, wf, shape, B, S, rnd=False)
    for li in range(2):
        for key, name in (("dA_q", "A_q"), ("dB_v", "B_v")):
            def L(p, li=li, name=name):
                l2 = [dict(l) for l in loras]
                l2[li][name] = p
                return model.forward_backward(ids, layers, l2, emb, None, wf, shape, B, S, rnd=False)[0]
            _fd_check(L, loras[li][name], grads[li][key], n_dirs=2)


def test_gflop_per_token_table_from_page():
    g = GOLD["gflop_per_token"]
    assert round(account.flop_per_token(synth.LLAMA_8B, 32, 128256) / 1e9, 2) == g["llama31_8b"]

    def qwen(h, i, L, nq, nkv, d, vocab):
        s = synth.LayerShape(hidden=h, inter=i, n_q=nq, n_kv=nkv, head_dim=d, rope_theta=1e6)
        bias = nq * d + 2 * nkv * d
        return account.flop_per_token(s, L, vocab, extra_layer_params=bias) / 1e9

    # the page prints two decimals (8.795 appears as 8.79), so allow one unit in the last place
    assert abs(qwen(896, 4864, 24, 14, 2, 64, 151936) - g["qwen25_05b"]) <= 0.01
    assert abs(qwen(1536, 8960, 28, 12, 2, 128, 151936) - g["qwen25_15b"]) <= 0.01
    assert abs(qwen(2048, 11008, 36, 16, 2, 128, 151936) - g["qwen25_3b"]) <= 0.01


# ------------------------------------------------------------------ backward pieces vs torch autograd
def test_attention_backward_matches_torch_autograd():
    """dq, dk, dv of causal GQA attention (three query heads per kv head) against
    torch autograd through scaled_dot_product_attention, float64."""
    rng = np.random.default_rng(21)
    B_, S, nq, nkv, d = 2, 9, 6, 2, 8
    q, k, v = (rng.normal(size=(B_, S, n, d)) for n in (nq, nkv, nkv))
    do = rng.normal(size=(B_, S, nq, d))
    o, P = layer.attention(q, k, v)
    dq, dk, dv = layer.attention_bwd(q, k, v, P, do)
    tq, tk, tv = (torch.tensor(a, requires_grad=True) for a in (q, k, v))
    grp = nq // nkv
    out = torch.nn.functional.scaled_dot_product_attention(
        tq.transpose(1, 2), tk.repeat_interleave(grp, dim=2).transpose(1, 2),
        tv.repeat_interleave(grp, dim=2).transpose(1, 2), is_causal=True).transpose(1, 2)
    out.backward(torch.tensor(do))
    np.testing.assert_allclose(o, out.detach().numpy(), rtol=1e-10, atol=1e-12)
    for mine, ref in ((dq, tq.grad), (dk, tk.grad), (dv, tv.grad)):
        np.testing.assert_allclose(mine, ref.numpy(), rtol=1e-9, atol=1e-12)


def test_rmsnorm_backward_matches_torch_autograd():
    rng = np.random.default_rng(22)
    x = rng.normal(size=(5, 48))
    w = 1.0 + 0.1 * rng.normal(size=48)
    dy = rng.normal(size=(5, 48))
    y, r = layer.rmsnorm(x, w, 1e-5)
    dx = layer.rmsnorm_bwd(x, w, r, dy)
    tx = torch.tensor(x, requires_grad=True)
    ty = torch.nn.functional.rms_norm(tx, (48,), torch.tensor(w), eps=1e-5)
    ty.backward(torch.tensor(dy))
    np.testing.assert_allclose(y, ty.detach().numpy(), rtol=1e-12)
    np.testing.assert_allclose(dx, tx.grad.numpy(), rtol=1e-10, atol=1e-12)


def test_rope_matches_complex_rotation_and_its_adjoint():
    """Rotate-half RoPE is multiplication of (x_i + i x_{i+d/2}) by e^{i p theta_i};
    its backward is the adjoint: <rope(x), y> = <x, rope_bwd(y)>."""
    rng = np.random.default_rng(23)
    S, d = 7, 16
    cos, sin = layer.rope_tables(S, d, 500000.0)
    x = rng.normal(size=(2, S, 3, d))
    y = layer.rope(x, cos, sin)
    z = (x[..., : d // 2] + 1j * x[..., d // 2:])
    inv = 500000.0 ** (-(2.0 * np.arange(d // 2)) / d)
    rot = np.exp(1j * np.arange(S)[:, None] * inv[None, :])[None, :, None, :]
    zr = z * rot
    np.testing.assert_allclose(y[..., : d // 2], zr.real, rtol=1e-12, atol=1e-14)
    np.testing.assert_allclose(y[..., d // 2:], zr.imag, rtol=1e-12, atol=1e-14)
    g = rng.normal(size=x.shape)
    assert math.isclose(float(np.sum(y * g)), float(np.sum(x * layer.rope_bwd(g, cos, sin))), rel_tol=1e-12)


def test_cross_entropy_gradient_matches_torch_autograd():
    """Loss and dlogits of the shifted causal-LM cross-entropy (no target for the last
    position of each sequence) against torch's cross_entropy with ignore_index."""
    rng = np.random.default_rng(24)
    batch, seq, V = 2, 6, 11
    logits = rng.normal(size=(batch * seq, V)) * 3
    ids = rng.integers(0, V, size=(batch, seq))
    loss, d = model.cross_entropy(logits, ids, batch, seq, rnd=False)
    tgt = np.full((batch, seq), -100)
    tgt[:, :-1] = ids[:, 1:]
    tl = torch.tensor(logits, requires_grad=True)
    ref = torch.nn.functional.cross_entropy(tl, torch.tensor(tgt.reshape(-1)), ignore_index=-100)
    ref.backward()
    assert math.isclose(loss, float(ref.detach()), rel_tol=1e-12)
    np.testing.assert_allclose(d, tl.grad.numpy(), rtol=1e-10, atol=1e-14)


def _hf_layer(shape, W, seq):
    """A transformers LlamaDecoderLayer (float64, eager attention) holding W."""
    from transformers import LlamaConfig
    from transformers.models.llama.modeling_llama import LlamaDecoderLayer, LlamaRotaryEmbedding
    cfg = LlamaConfig(hidden_size=shape.hidden, intermediate_size=shape.inter, num_attention_heads=shape.n_q,
                      num_key_value_heads=shape.n_kv, head_dim=shape.head_dim, rms_norm_eps=shape.rms_eps,
                      rope_theta=shape.rope_theta, attention_bias=False, mlp_bias=False, hidden_act="silu",
                      max_position_embeddings=max(seq, 8))
    cfg._attn_implementation = "eager"
    hf = LlamaDecoderLayer(cfg, layer_idx=0).double()
    with torch.no_grad():
        for mod, key in ((hf.self_attn.q_proj, "q"), (hf.self_attn.k_proj, "k"), (hf.self_attn.v_proj, "v"),
                         (hf.self_attn.o_proj, "o"), (hf.mlp.gate_proj, "gate"), (hf.mlp.up_proj, "up"),
                         (hf.mlp.down_proj, "down")):
            mod.weight.copy_(torch.tensor(W[key]))
        hf.input_layernorm.weight.copy_(torch.tensor(W["norm_in"]))
        hf.post_attention_layernorm.weight.copy_(torch.tensor(W["norm_post"]))
    return hf, LlamaRotaryEmbedding(cfg)


@pytest.mark.parametrize("with_lora", [False, True])
def test_layer_forward_matches_transformers_llama_decoder_layer(with_lora):
    """The oracle's decoder layer (float64, no bf16 rounding) against transformers'
    LlamaDecoderLayer, the body the pages run: pre-norm residual blocks, GQA, rotate-half
    RoPE, SiLU-gated MLP.  With the adapter on, the reference layer gets the merged
    weights W_q + (alpha / r) B_q A_q and W_v + (alpha / r) B_v A_v, which is what the
    LoRA update adds.  The reference computes its RoPE angles in fp32, hence a 1e-6
    tolerance rather than float64 rounding (measured 1.5e-8)."""
    shape = synth.TINY
    batch, seq = 2, 8
    W = _weights(shape, seed=31)
    lo = _lora(shape, seed=32) if with_lora else None
    x = np.random.default_rng(33).normal(size=(batch * seq, shape.hidden))
    out, _ = layer.forward(x, W, lo, shape, batch, seq, rnd=False)
    Wm = dict(W)
    if lo is not None:
        s = shape.lora_alpha / shape.lora_r
        Wm["q"] = W["q"] + s * lo["B_q"] @ lo["A_q"]
        Wm["v"] = W["v"] + s * lo["B_v"] @ lo["A_v"]
    hf, rot = _hf_layer(shape, Wm, seq)
    tx = torch.tensor(x.reshape(batch, seq, shape.hidden))
    pos = torch.arange(seq)[None].expand(batch, seq)
    cos, sin = rot(tx, pos)
    mask = torch.triu(torch.full((seq, seq), float("-inf"), dtype=torch.float64), 1)[None, None]
    with torch.no_grad():
        ref = hf(tx, attention_mask=mask, position_ids=pos, position_embeddings=(cos, sin))
    ref = (ref[0] if isinstance(ref, tuple) else ref).numpy().reshape(batch * seq, shape.hidden)
    err = np.max(np.abs(out - ref))
    assert err <= 1e-6 * np.max(np.abs(ref)), err


def test_model_step_matches_transformers_llama_autograd():
    """One training step of the oracle (a 2-layer tied model, float64, no rounding)
    against transformers' LlamaForCausalLM with autograd: the loss of its labels path,
    and the LoRA gradients from the gradient G of the merged weight W + s B A, which are
    dA = s B^T G and dB = s G A^T exactly."""
    from transformers import LlamaConfig, LlamaForCausalLM
    shape = synth.TINY
    n_layers, vocab, batch, seq = 2, 32, 2, 6
    rng = np.random.default_rng(41)
    layers = [_weights(shape, seed=42 + i) for i in range(n_layers)]
    loras = [_lora(shape, seed=50 + i) for i in range(n_layers)]
    emb = rng.normal(0, 0.5, (vocab, shape.hidden))
    w_final = 1.0 + 0.1 * rng.normal(size=shape.hidden)
    ids = rng.integers(0, vocab, (batch, seq))
    loss, grads, _ = model.forward_backward(ids, layers, loras, emb, None, w_final, shape, batch, seq, rnd=False)

    cfg = LlamaConfig(hidden_size=shape.hidden, intermediate_size=shape.inter, num_attention_heads=shape.n_q,
                      num_key_value_heads=shape.n_kv, head_dim=shape.head_dim, rms_norm_eps=shape.rms_eps,
                      rope_theta=shape.rope_theta, attention_bias=False, mlp_bias=False, hidden_act="silu",
                      vocab_size=vocab, num_hidden_layers=n_layers, tie_word_embeddings=True,
                      max_position_embeddings=seq)
    cfg._attn_implementation = "eager"
    hf = LlamaForCausalLM(cfg).double()
    s = shape.lora_alpha / shape.lora_r
    with torch.no_grad():
        hf.model.embed_tokens.weight.copy_(torch.tensor(emb))
        hf.model.norm.weight.copy_(torch.tensor(w_final))
        for L, W, lo in zip(hf.model.layers, layers, loras):
            merged = dict(W, q=W["q"] + s * lo["B_q"] @ lo["A_q"], v=W["v"] + s * lo["B_v"] @ lo["A_v"])
            for mod, key in ((L.self_attn.q_proj, "q"), (L.self_attn.k_proj, "k"), (L.self_attn.v_proj, "v"),
                             (L.self_attn.o_proj, "o"), (L.mlp.gate_proj, "gate"), (L.mlp.up_proj, "up"),
                             (L.mlp.down_proj, "down")):
                mod.weight.copy_(torch.tensor(merged[key]))
            L.input_layernorm.weight.copy_(torch.tensor(W["norm_in"]))
            L.post_attention_layernorm.weight.copy_(torch.tensor(W["norm_post"]))
    tid = torch.tensor(ids)
    ref = hf(input_ids=tid, labels=tid).loss
    ref.backward()
    assert math.isclose(loss, float(ref.detach()), rel_tol=1e-6)
    for L, lo, g in zip(hf.model.layers, loras, grads):
        Gq = L.self_attn.q_proj.weight.grad.numpy()
        Gv = L.self_attn.v_proj.weight.grad.numpy()
        for mine, want in ((g["dA_q"], s * lo["B_q"].T @ Gq), (g["dB_q"], s * Gq @ lo["A_q"].T),
                           (g["dA_v"], s * lo["B_v"].T @ Gv), (g["dB_v"], s * Gv @ lo["A_v"].T)):
            assert np.max(np.abs(mine - want)) <= 1e-5 * np.max(np.abs(want))
