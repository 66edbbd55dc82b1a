"""Parity of the individual CUDA kernels against the oracle (GPU).

Quantiser and dequantiser: bit-exact bytes and bf16 values, including zero blocks,
partial nested groups, one-block tensors and the full Llama-8B q_proj.  GEMMs: the
tcgen05 kernel against a float64 product of the same bf16 operands; the in-mainloop
NF4 decode against the dense kernel on the oracle's dequantised weights, bit for bit.
Attention forward against the oracle's causal GQA attention.
"""
import numpy as np
import pytest
import torch

from nf4_layer_streamed_b200 import api, synth
from oracle import bf16 as obf16, layer as olayer, quant
from tests.helpers import TOL, close, f64

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _q_to_np(q):
    return {"packed": q["packed"].cpu().numpy(), "q8": q["q8"].cpu().numpy(), "nested": q["nested"].cpu().numpy(),
            "offset": np.float32(q["offset"].cpu().numpy()[0])}


@pytest.mark.parametrize("shape,seed", [((1, 64), 1), ((257, 64), 2), ((192, 576), 3),
                                        ((1536, 576), 4), ((4096, 4096), 5)])
def test_quantize_bit_exact_against_oracle(shape, seed):
    w = synth.tensor_values(shape, seed=seed, scale=0.02)
    if w.numel() >= 256:
        w.view(-1)[64:128] = 0                     # a zero block
    q = api.nf4_quantize_tensor(w.to(DEV))
    torch.cuda.synchronize()
    ref = quant.quantize(w.float().numpy().reshape(-1))
    got = _q_to_np(q)
    assert got["offset"] == ref["offset"]
    np.testing.assert_array_equal(got["nested"], ref["nested"])
    np.testing.assert_array_equal(got["q8"], ref["q8"])
    np.testing.assert_array_equal(got["packed"], ref["packed"])
    deq = api.nf4_dequantize_tensor(q)
    np.testing.assert_array_equal(deq.view(torch.int16).cpu().numpy().view(np.uint16), quant.dequantize_bits(ref))


def test_quantize_deterministic_across_calls():
    w = synth.tensor_values((1024, 4096), seed=11, scale=0.02).to(DEV)
    a, b = api.nf4_quantize_tensor(w), api.nf4_quantize_tensor(w)
    for k in ("packed", "q8", "nested", "offset"):
        assert torch.equal(a[k], b[k])


def test_quantize_extreme_values():
    # one huge block and tiny blocks: nested range and offset far from most absmax values
    w = synth.tensor_values((64, 256), seed=12, scale=1e-3)
    w.view(-1)[:64] = 30.0
    w.view(-1)[64:128] = -1e-30
    q = api.nf4_quantize_tensor(w.to(DEV))
    ref = quant.quantize(w.float().numpy().reshape(-1))
    got = _q_to_np(q)
    np.testing.assert_array_equal(got["packed"], ref["packed"])
    np.testing.assert_array_equal(got["q8"], ref["q8"])
    # absmax values from 1e-30 to 30: a double sum of them rounds, so the offset comes
    # from the sequential pass, and must still equal the oracle's
    assert got["offset"] == ref["offset"]
    np.testing.assert_array_equal(got["nested"], ref["nested"])


def test_quantize_offset_sum_rounding_cases():
    """The mean absmax takes the parallel sum only when it is provably the sequential
    one: a tensor whose absmax values span 2^-30 .. 2^1 (the double sum rounds) and one
    with 2^18 blocks of ordinary weights (it does not) both give the oracle's bytes."""
    g = torch.Generator().manual_seed(21)
    w1 = (torch.rand(4096, 64, generator=g) * 2 - 1)
    w1 = w1 * torch.pow(2.0, torch.randint(-30, 2, (4096, 1), generator=g).float())
    w2 = synth.tensor_values((1 << 18, 64), seed=22, scale=0.02)
    for w in (w1.to(torch.bfloat16), w2):
        q = api.nf4_quantize_tensor(w.to(DEV))
        ref = quant.quantize(w.float().numpy().reshape(-1))
        got = _q_to_np(q)
        assert got["offset"] == ref["offset"]
        np.testing.assert_array_equal(got["nested"], ref["nested"])
        np.testing.assert_array_equal(got["q8"], ref["q8"])
    assert got["offset"] == ref["offset"]


def test_shard_regions_match_oracle_and_header():
    shape = synth.SMOLLM2_135M
    cfg = api.layer_cfg(shape, 1, 512)
    w = synth.layer_weights(shape, 0, 1234, device=DEV)
    shard = api.nf4_quantize_shard(cfg, w, fingerprint=42)
    torch.cuda.synchronize()
    host = shard.cpu().numpy()
    assert api.shard_check(shard, cfg, 42) == 0
    assert api.shard_check(shard, cfg, 43) == -5
    desc = host[256:256 + 9 * 64].view(np.uint64).reshape(9, 8)
    for t, name in enumerate(("q", "k", "v", "o", "gate", "up", "down")):
        rows, cols = int(desc[t, 1]), int(desc[t, 2])
        assert (rows, cols) == tuple(w[name].shape)
        n = rows * cols
        ref = quant.quantize(w[name].float().cpu().numpy().reshape(-1))
        op, oq, on, oo = (int(x) for x in desc[t, 3:7])
        np.testing.assert_array_equal(host[op:op + n // 2], ref["packed"])
        np.testing.assert_array_equal(host[oq:oq + n // 64], ref["q8"])
        np.testing.assert_array_equal(host[on:on + ref["nested"].nbytes].view(np.float32), ref["nested"])
        assert host[oo:oo + 4].view(np.float32)[0] == ref["offset"]


@pytest.mark.parametrize("M,N,K", [(256, 256, 64), (300, 576, 576), (1, 960, 576), (512, 4096, 4096),
                                   (2048, 1536, 1024)])
def test_dense_gemm_forward_and_transposed(M, N, K):
    A = synth.tensor_values((M, K), seed=M + N, scale=1.0).to(DEV)
    Bm = synth.tensor_values((N, K), seed=K, scale=0.05).to(DEV)
    out = api.gemm_bf16(A, Bm)
    ref = f64(A) @ f64(Bm).T
    close(out, ref, tol=1e-2, what="A B^T")
    Bt = synth.tensor_values((K, N), seed=K + 1, scale=0.05).to(DEV)
    out2 = api.gemm_bf16(A, Bt, b_trans=True)
    close(out2, f64(A) @ f64(Bt), tol=1e-2, what="A B")


@pytest.mark.parametrize("M,rows,cols", [(512, 576, 576), (300, 192, 576), (2048, 4096, 4096), (64, 1536, 576)])
def test_nf4_gemm_bit_exact_against_dense_on_dequantised(M, rows, cols):
    w = synth.tensor_values((rows, cols), seed=rows + cols, scale=0.02).to(DEV)
    q = api.nf4_quantize_tensor(w)
    deq = api.nf4_dequantize_tensor(q).view(rows, cols)
    # dequantised weights equal the oracle's
    ref = quant.quantize(w.float().cpu().numpy().reshape(-1))
    np.testing.assert_array_equal(deq.view(torch.int16).cpu().numpy().view(np.uint16).reshape(-1),
                                  quant.dequantize_bits(ref))
    A = synth.tensor_values((M, cols), seed=M, scale=1.0).to(DEV)
    fused = api.gemm_nf4(A, q, rows, cols, dgrad=False)
    dense = api.gemm_bf16(A, deq)
    assert torch.equal(fused, dense)
    close(fused, f64(A) @ f64(deq).T, tol=1e-2, what="NF4 forward")
    G = synth.tensor_values((M, rows), seed=M + 7, scale=1.0).to(DEV)
    fused_t = api.gemm_nf4(G, q, rows, cols, dgrad=True)
    dense_t = api.gemm_bf16(G, deq, b_trans=True)
    assert torch.equal(fused_t, dense_t)
    close(fused_t, f64(G) @ f64(deq), tol=1e-2, what="NF4 dL/dx")
    st, err = api.device_error()
    assert st == 0, err


@pytest.mark.parametrize("M,rows,cols", [(512, 576, 576), (600, 960, 576), (2048, 4096, 4096)])
def test_cta_pair_gemm_equals_single_cta(M, rows, cols):
    w = synth.tensor_values((rows, cols), seed=3 * rows + cols, scale=0.02).to(DEV)
    q = api.nf4_quantize_tensor(w)
    deq = api.nf4_dequantize_tensor(q).view(rows, cols)
    A = synth.tensor_values((M, cols), seed=M + 1, scale=1.0).to(DEV)
    G = synth.tensor_values((M, rows), seed=M + 2, scale=1.0).to(DEV)
    outs = {}
    try:
        for pair in (False, True):
            api.set_gemm_pair(pair)
            outs[pair] = [api.gemm_nf4(A, q, rows, cols), api.gemm_nf4(G, q, rows, cols, dgrad=True),
                          api.gemm_bf16(A, deq), api.gemm_bf16(G, deq, b_trans=True)]
    finally:
        api.set_gemm_pair(True)
    for a, b in zip(outs[False], outs[True]):
        assert torch.equal(a, b)
    close(outs[True][0], f64(A) @ f64(deq).T, tol=1e-2, what="pair forward")
    close(outs[True][1], f64(G) @ f64(deq), tol=1e-2, what="pair dL/dx")
    st, err = api.device_error()
    assert st == 0, err


@pytest.mark.parametrize("M,rows,cols", [(1280, 576, 1536), (2048, 6144, 4096), (2048, 14336, 4096),
                                         (1536, 28672, 4096)])
def test_pair_tile_heights_give_identical_results(M, rows, cols):
    """256- and 512-token pair tiles, and the split schedule (whole waves of 512-token
    tiles, the last partial wave as 256-token tiles in a second launch), reduce every
    output in the same order: equal bits, forward and dL/dx, NF4 decode and dense,
    including a ragged last token tile."""
    w = synth.tensor_values((rows, cols), seed=5 * rows + cols, scale=0.02).to(DEV)
    q = api.nf4_quantize_tensor(w)
    deq = api.nf4_dequantize_tensor(q).view(rows, cols)
    A = synth.tensor_values((M, cols), seed=M + 3, scale=1.0).to(DEV)
    G = synth.tensor_values((M, rows), seed=M + 4, scale=1.0).to(DEV)
    outs = {}
    try:
        for mode in (1, 2, 3):
            api.set_gemm_half(mode)
            outs[mode] = [api.gemm_nf4(A, q, rows, cols), api.gemm_nf4(G, q, rows, cols, dgrad=True),
                          api.gemm_bf16(A, deq), api.gemm_bf16(G, deq, b_trans=True)]
    finally:
        api.set_gemm_half(0)
    for mode in (2, 3):
        for a, b in zip(outs[1], outs[mode]):
            assert torch.equal(a, b), mode
    close(outs[2][0], f64(A) @ f64(deq).T, tol=1e-2, what="half-height forward")
    st, err = api.device_error()
    assert st == 0, err


@pytest.mark.parametrize("shape,batch,seq", [(synth.SMOLLM2_135M, 1, 512), (synth.LLAMA_8B, 2, 128),
                                             (synth.LLAMA_8B, 2, 384), (synth.LLAMA_8B, 1, 512),
                                             (synth.QWEN_32B_CLASS, 1, 1024)])
def test_attention_forward_against_oracle(shape, batch, seq):
    cfg = api.layer_cfg(shape, batch, seq)
    M = batch * seq
    qd, kvd = shape.q_dim, shape.kv_dim
    qkv = synth.tensor_values((M, qd + 2 * kvd), seed=seq, scale=1.0).to(DEV)
    o, lse = api.attention_fwd(cfg, qkv, qkv[:, qd:], qkv[:, qd + kvd:], qd + 2 * kvd, qd + 2 * kvd)
    x = f64(qkv)
    q = x[:, :qd].reshape(batch, seq, shape.n_q, shape.head_dim)
    k = x[:, qd:qd + kvd].reshape(batch, seq, shape.n_kv, shape.head_dim)
    v = x[:, qd + kvd:].reshape(batch, seq, shape.n_kv, shape.head_dim)
    ref, P = olayer.attention(q, k, v)
    close(o, ref.reshape(M, qd), what="attention out")


@pytest.mark.parametrize("seq", [128, 384, 512, 1024])
def test_tcgen05_attention_matches_mma_sync_attention(seq):
    """The tcgen05 forward (head_dim 128, online softmax over key tiles in TMEM) against the
    mma.sync forward on the same GQA inputs: outputs within 1e-2 max|ref|, the
    log-sum-exp within 1e-4, and bit-exact across reruns."""
    shape = synth.LLAMA_8B
    batch = 2
    cfg = api.layer_cfg(shape, batch, seq)
    qd, kvd = shape.q_dim, shape.kv_dim
    ld = qd + 2 * kvd
    qkv = synth.tensor_values((batch * seq, ld), seed=seq + 7, scale=1.0).to(DEV)
    args = (cfg, qkv, qkv[:, qd:], qkv[:, qd + kvd:], ld, ld)
    try:
        api.set_attention_path(False)
        o_ref, lse_ref = api.attention_fwd(*args)
        api.set_attention_path(True)
        o1, lse1 = api.attention_fwd(*args)
        o2, lse2 = api.attention_fwd(*args)
    finally:
        api.set_attention_path(True)
    torch.cuda.synchronize()
    assert torch.equal(o1, o2) and torch.equal(lse1, lse2)
    close(o1, f64(o_ref), tol=1e-2, what="tcgen05 attention")
    close(lse1, f64(lse_ref), tol=1e-4, what="log-sum-exp")
    st, err = api.device_error()
    assert st == 0, err


@pytest.mark.parametrize("batch,seq", [(2, 128), (2, 384), (1, 512), (1, 1024)])
def test_tcgen05_attention_backward_against_oracle(batch, seq):
    """The tcgen05 attention backward (query side: dQ and delta; key side: dK, dV over
    the query heads of each kv group) on the Llama-8B head layout, against the oracle's
    float64 backward on the same bf16 q, k, v, o and dO: dq, dk, dv within 2e-2 max|ref|,
    delta = rowsum(dO * O) within 1e-4 (fp32 sums of bf16 products), and bit-exact
    across reruns."""
    shape = synth.LLAMA_8B
    cfg = api.layer_cfg(shape, batch, seq)
    M, qd, kvd = batch * seq, shape.q_dim, shape.kv_dim
    ld = qd + 2 * kvd
    qkv = synth.tensor_values((M, ld), seed=seq + 11, scale=1.0).to(DEV)
    args = (cfg, qkv, qkv[:, qd:], qkv[:, qd + kvd:], ld, ld)
    o, lse = api.attention_fwd(*args)
    do = synth.tensor_values((M, qd), seed=seq + 12, scale=1.0).to(DEV)
    dq, dk, dv, delta = api.attention_bwd(*args, o, do, lse)
    dq2, dk2, dv2, delta2 = api.attention_bwd(*args, o, do, lse)
    torch.cuda.synchronize()
    assert torch.equal(dq, dq2) and torch.equal(dk, dk2) and torch.equal(dv, dv2) and torch.equal(delta, delta2)
    x = f64(qkv)
    q = x[:, :qd].reshape(batch, seq, shape.n_q, shape.head_dim)
    k = x[:, qd:qd + kvd].reshape(batch, seq, shape.n_kv, shape.head_dim)
    v = x[:, qd + kvd:].reshape(batch, seq, shape.n_kv, shape.head_dim)
    _, P = olayer.attention(q, k, v)
    d_o = f64(do).reshape(batch, seq, shape.n_q, shape.head_dim)
    rq, rk, rv = olayer.attention_bwd(q, k, v, P, d_o)
    close(dq, rq.reshape(M, qd), what="dq")
    close(dk, rk.reshape(M, kvd), what="dk")
    close(dv, rv.reshape(M, kvd), what="dv")
    ref_delta = (f64(o) * f64(do)).reshape(batch, seq, shape.n_q, shape.head_dim).sum(-1).transpose(0, 2, 1)
    close(delta, ref_delta, tol=1e-4, what="delta")
    st, err = api.device_error()
    assert st == 0, err
