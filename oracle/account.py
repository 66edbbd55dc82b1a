"""FLOP and byte accounting behind the throughput metric (oracle; test infrastructure only).

FLOP convention of "Soup 层流式 NF4 训练实测：在 4 GB 显存上以位级一致标准完成 8B 模型 LoRA 微调" (m.mzlw.cn) §4.4:
decoder linear parameters count C = 6 FLOP per token (2 forward + 2
checkpoint recompute + 2 dL/dx; not 8, because the frozen base computes no
dL/dW), lm_head counts C = 4 (2 forward + 2 dL/dx; it sits outside the
checkpointed layers and is frozen), the embedding lookup counts 0.  Attention
score/value products are not counted, as on the page.

Byte identity of §2.4: a quantised tensor of N weights streams
N/2 + N/64 + 4*ceil(N/16384) + 4 bytes (packed codes, 8-bit absmax, fp32
nested absmax per 256 blocks, fp32 offset), about 0.516 B/param.
"""
from __future__ import annotations

from . import quant


def decoder_params(shape) -> int:
    return sum(a * b for _, (a, b) in shape.weight_shapes())


def flop_per_token(shape, n_layers: int, vocab: int, hidden: int | None = None,
                   extra_layer_params: int = 0) -> float:
    H = shape.hidden if hidden is None else hidden
    return 6.0 * n_layers * (decoder_params(shape) + extra_layer_params) + 4.0 * vocab * H


def layer_shard_bytes(shape) -> int:
    """Quantised bytes of one layer (the seven linears), by the per-tensor identity."""
    return sum(quant.tensor_bytes(a * b)["total"] for _, (a, b) in shape.weight_shapes())


def store_bytes(shape, n_layers: int) -> int:
    return n_layers * layer_shard_bytes(shape)
