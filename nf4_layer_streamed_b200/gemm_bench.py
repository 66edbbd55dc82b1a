"""Shape-matched GEMM throughput of the tcgen05 kernels (NF4 decode in the mainloop,
and the dense bf16 kernel on the same dequantised weights).

The shapes are the Llama-3.1-8B projections that the §4.4 table of
"Soup 层流式 NF4 训练实测：在 4 GB 显存上以位级一致标准完成 8B 模型 LoRA 微调"
measures (q/o 4096x4096, k/v 1024x4096, gate/up
14336x4096, down 4096x14336), at M = batch x 512 tokens, both for the forward
product out = x W^T and the dL/dx product out = dy W.

    python -m nf4_layer_streamed_b200.gemm_bench [--M 2048] [--shapes gateup,down] [--iters 20]
    python -m nf4_layer_streamed_b200.gemm_bench --once --shapes gateup   (one launch each: for ncu)
    python -m nf4_layer_streamed_b200.gemm_bench --attention 4 [--once]      (attention fwd / bwd, batch 4)
    python -m nf4_layer_streamed_b200.gemm_bench --layer 4 [--once] [--layer-shape smollm2]
                                                   (quantise + one layer fwd/bwd)

Prints one JSON object per (shape, direction, kernel) with the mean launch time
(CUDA events on the launching stream, after warm-up) and TFLOP/s = 2 M N K / time.
"""
from __future__ import annotations

import argparse
import json

import torch

from . import api, synth

SHAPES = {  # name: (rows = out features, cols = in features) of W
    "qkv": (6144, 4096),       # q, k and v stacked, as the fused GEMM runs them
    "qo": (4096, 4096),
    "kv": (1024, 4096),
    "gateup": (28672, 4096),   # gate and up stacked, as the fused GEMM runs them
    "down": (4096, 14336),
}


def run(M: int, names, iters: int, once: bool):
    out = []
    for name in names:
        rows, cols = SHAPES[name]
        w = synth.tensor_values((rows, cols), seed=rows + cols, scale=0.02, device="cuda")
        q = api.nf4_quantize_tensor(w)
        deq = api.nf4_dequantize_tensor(q).view(rows, cols)
        del w
        for dgrad in (False, True):
            K = rows if dgrad else cols
            N = cols if dgrad else rows
            A = synth.tensor_values((M, K), seed=M + K, scale=1.0, device="cuda")
            for kind in ("nf4", "dense"):
                def f():
                    if kind == "nf4":
                        return api.gemm_nf4(A, q, rows, cols, dgrad=dgrad)
                    return api.gemm_bf16(A, deq, b_trans=dgrad)
                if once:
                    f()
                    torch.cuda.synchronize()
                    continue
                for _ in range(3):
                    f()
                torch.cuda.synchronize()
                e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                e0.record()
                for _ in range(iters):
                    f()
                e1.record()
                torch.cuda.synchronize()
                ms = e0.elapsed_time(e1) / iters
                tf = 2.0 * M * N * K / (ms / 1000.0) / 1e12
                rec = {"shape": name, "M": M, "N": N, "K": K, "product": "dL/dx" if dgrad else "forward",
                       "kernel": kind, "ms": ms, "tflops": tf}
                out.append(rec)
                print(json.dumps(rec), flush=True)
    return out


def run_quant(iters: int = 10):
    """HBM throughput of the quantiser (reads 2 B, writes 0.516 B per weight) and the
    dequantiser (reads 0.516 B, writes 2 B per weight) on the stacked gate/up matrix."""
    rows, cols = SHAPES["gateup"]
    w = synth.tensor_values((rows, cols), seed=rows + cols, scale=0.02, device="cuda")
    n = rows * cols
    qb = n // 2 + n // 64 + 4 * ((n // 64 + 255) // 256) + 4
    q = api.nf4_quantize_tensor(w)
    out = []
    for name, f, nbytes in (("quantize", lambda: api.nf4_quantize_tensor(w), 2 * n + qb),
                            ("dequantize", lambda: api.nf4_dequantize_tensor(q), qb + 2 * n)):
        for _ in range(3):
            f()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for _ in range(iters):
            f()
        e1.record()
        torch.cuda.synchronize()
        ms = e0.elapsed_time(e1) / iters
        rec = {"kernel": name, "weights": n, "ms": ms, "algorithmic_bytes": nbytes,
               "gbs": nbytes / (ms / 1000.0) / 1e9}
        out.append(rec)
        print(json.dumps(rec), flush=True)
    return out


def run_attention(batch: int, once: bool, iters: int = 20):
    """Causal GQA attention of the Llama-8B layer (32 query heads, 8 kv heads, d 128) at
    seq 512: forward and backward (query side with delta, then key side), the tcgen05
    kernels and the mma.sync kernels.  Algorithmic FLOPs: forward 4 S^2 d n_q B / 2
    (causal half), backward 2.5 times that (five products against two)."""
    shape = synth.LLAMA_8B
    seq = 512
    cfg = api.layer_cfg(shape, batch, seq)
    qd, kvd = shape.q_dim, shape.kv_dim
    ld = qd + 2 * kvd
    qkv = synth.tensor_values((batch * seq, ld), seed=3, scale=1.0, device="cuda")
    do = synth.tensor_values((batch * seq, qd), seed=4, scale=1.0, device="cuda")
    args = (cfg, qkv, qkv[:, qd:], qkv[:, qd + kvd:], ld, ld)
    out = []
    flops = 4.0 * seq * seq * shape.head_dim * shape.n_q * batch / 2
    for tc in ((True,) if once else (True, False)):
        api.set_attention_path(tc)
        o, lse = api.attention_fwd(*args)
        fwd = lambda: api.attention_fwd(*args)
        bwd = lambda: api.attention_bwd(*args, o, do, lse)
        if once:
            for f in (fwd, fwd, bwd, bwd):
                f()
            torch.cuda.synchronize()
            continue
        name = "tcgen05" if tc else "mma_sync"
        for part, f, fl in (("forward", fwd, flops), ("backward", bwd, 2.5 * flops)):
            us = _time(f, iters) * 1000.0
            rec = {"kernel": f"attention_{part}_{name}", "batch": batch, "seq": seq, "us": us,
                   "tflops": fl / us / 1e6}
            out.append(rec)
            print(json.dumps(rec), flush=True)
    api.set_attention_path(True)
    return out


def run_layer(batch: int, once: bool, iters: int = 10, shape_name: str = "llama8b"):
    """One Llama-8B-shaped (or SmolLM2-135M-shaped) layer at batch x 512: the shard
    quantiser, then layer_forward and layer_backward (recompute + dL/dx + LoRA gradients)
    with random LoRA B.  With --once each runs once (a small case for ncu: every kernel
    of the layer appears)."""
    shape = {"llama8b": synth.LLAMA_8B, "smollm2": synth.SMOLLM2_135M}[shape_name]
    seq = 512
    cfg = api.layer_cfg(shape, batch, seq)
    w = synth.layer_weights(shape, 0, 1234, device="cuda")
    lo = synth.lora_params(shape, 0, 1234, b_random=True, device="cuda")
    x = synth.hidden_states(shape, batch, seq, 7, device="cuda").view(batch * seq, shape.hidden)
    dy = synth.tensor_values((batch * seq, shape.hidden), seed=5, scale=1e-3, device="cuda")
    ws = api.LayerWorkspace(cfg)
    shard = api.nf4_quantize_shard(cfg, w, fingerprint=1)
    fwd = lambda: api.layer_forward(cfg, shard, lo, x, ws)
    bwd = lambda: api.layer_backward(cfg, shard, lo, x, dy, ws)
    if once:
        fwd()
        bwd()
        torch.cuda.synchronize()
        return []
    out = []
    for name, f in (("quantize_shard", lambda: api.nf4_quantize_shard(cfg, w, fingerprint=1, out=shard)),
                    ("layer_forward", fwd), ("layer_backward", bwd)):
        ms = _time(f, iters)
        rec = {"step": name, "batch": batch, "seq": seq, "ms": ms}
        out.append(rec)
        print(json.dumps(rec), flush=True)
    return out


def _time(f, iters):
    for _ in range(3):
        f()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(iters):
        f()
    e1.record()
    torch.cuda.synchronize()
    return e0.elapsed_time(e1) / iters


def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--M", type=int, default=2048)
    ap.add_argument("--shapes", default="qo,kv,gateup,down")
    ap.add_argument("--iters", type=int, default=20)
    ap.add_argument("--once", action="store_true")
    ap.add_argument("--single", action="store_true", help="one CTA per tile instead of CTA pairs")
    ap.add_argument("--quant", action="store_true", help="also time the quantiser and dequantiser")
    ap.add_argument("--quant-only", action="store_true", help="time only the quantiser and dequantiser")
    ap.add_argument("--half", type=int, default=0,
                    help="pair tile height: 0 auto, 1 512 tokens, 2 256 tokens, 3 last partial wave as 256")
    ap.add_argument("--layer", type=int, default=0, metavar="BATCH",
                    help="time the shard quantiser and one 8B layer forward / backward at this batch instead")
    ap.add_argument("--layer-shape", default="llama8b", choices=["llama8b", "smollm2"],
                    help="the layer shape of --layer")
    ap.add_argument("--attention", type=int, default=0, metavar="BATCH",
                    help="time the attention forward of the 8B layer at this batch (seq 512) instead")
    a = ap.parse_args(argv)
    api.set_gemm_pair(not a.single)
    api.set_gemm_half(a.half)
    if a.attention:
        run_attention(a.attention, a.once)
        return
    if a.quant_only:
        run_quant(1 if a.once else 10)
        return
    if a.layer:
        run_layer(a.layer, a.once, shape_name=a.layer_shape)
        st, err = api.device_error()
        if st != 0:
            raise RuntimeError(f"device error record {err}")
        return
    run(a.M, a.shapes.split(","), a.iters, a.once)
    if a.quant:
        run_quant()
    st, err = api.device_error()
    if st != 0:
        raise RuntimeError(f"device error record {err}")


if __name__ == "__main__":
    main()
