"""Seeded synthetic inputs shared by the CUDA path, the tests and the oracle.

This module draws random numbers and nothing else: it holds none of the
method's arithmetic (no quantisation, no layer math).  Every workload in this
repository is synthetic; the recipe follows the configurations quoted on the
pages (Llama-style decoder layers, N(0, 0.02) weights, N(0, 1) hidden states,
uniform token ids, LoRA A ~ N(0, 0.02) and B = 0 or B ~ N(0, 0.02)).

Seeds: base weights from ``seed`` (layer-major order q, k, v, o, gate, up,
down, then embedding and lm_head), LoRA A from ``seed + 1``, inputs and token
ids from ``seed + 2``.  Per-layer streams are derived as ``seed * 1000 + layer``
so that one layer can be regenerated on its own.
"""
from __future__ import annotations

from dataclasses import dataclass, field

import torch


@dataclass(frozen=True)
class LayerShape:
    """Dimensions of one Llama-style decoder layer."""

    hidden: int
    inter: int
    n_q: int
    n_kv: int
    head_dim: int
    rope_theta: float
    rms_eps: float = 1e-5
    lora_r: int = 16
    lora_alpha: float = 32.0

    @property
    def q_dim(self) -> int:
        return self.n_q * self.head_dim

    @property
    def kv_dim(self) -> int:
        return self.n_kv * self.head_dim

    def weight_shapes(self) -> list[tuple[str, tuple[int, int]]]:
        """(name, [out, in]) of the seven frozen linears, in shard order."""
        H, I = self.hidden, self.inter
        return [
            ("q", (self.q_dim, H)),
            ("k", (self.kv_dim, H)),
            ("v", (self.kv_dim, H)),
            ("o", (H, self.q_dim)),
            ("gate", (I, H)),
            ("up", (I, H)),
            ("down", (H, I)),
        ]

    def n_params(self) -> int:
        return sum(a * b for _, (a, b) in self.weight_shapes())


# The three layer shapes named by the workloads.
SMOLLM2_135M = LayerShape(hidden=576, inter=1536, n_q=9, n_kv=3, head_dim=64, rope_theta=10000.0)
LLAMA_8B = LayerShape(hidden=4096, inter=14336, n_q=32, n_kv=8, head_dim=128, rope_theta=500000.0)
QWEN_32B_CLASS = LayerShape(hidden=5120, inter=27648, n_q=40, n_kv=8, head_dim=128, rope_theta=500000.0)
# A tiny shape for finite-difference checks of the oracle.
TINY = LayerShape(hidden=64, inter=128, n_q=2, n_kv=1, head_dim=32, rope_theta=10000.0)


@dataclass(frozen=True)
class Workload:
    name: str
    shape: LayerShape
    n_layers: int
    batch: int
    seq: int
    vocab: int = 0          # 0: single layer, loss = mean squared output
    tied: bool = False
    seed: int = 1234
    steps: int = 1
    depth: int = 2
    extra: dict = field(default_factory=dict)

    @property
    def tokens(self) -> int:
        return self.batch * self.seq


WORKLOADS = {
    "smollm2_layer_b1s512": Workload("smollm2_layer_b1s512", SMOLLM2_135M, 1, 1, 512),
    "smollm2_30L_tied_b1s512": Workload("smollm2_30L_tied_b1s512", SMOLLM2_135M, 30, 1, 512,
                                         vocab=49152, tied=True, steps=25),
    "llama8b_layer_b1s512": Workload("llama8b_layer_b1s512", LLAMA_8B, 1, 1, 512),
    "llama8b_layer_b4s512": Workload("llama8b_layer_b4s512", LLAMA_8B, 1, 4, 512),
    "llama8b_32L_b4s512": Workload("llama8b_32L_b4s512", LLAMA_8B, 32, 4, 512,
                                    vocab=128256, tied=False, steps=10),
    "qwen32b_4L_b1s1024": Workload("qwen32b_4L_b1s1024", QWEN_32B_CLASS, 4, 1, 1024),
    # out-of-config point: the same stack at batch 16, where the step is compute-bound
    "llama8b_32L_b16s512": Workload("llama8b_32L_b16s512", LLAMA_8B, 32, 16, 512,
                                     vocab=128256, tied=False, steps=3),
}


def _gen(seed: int, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    return g


def layer_weights(shape: LayerShape, layer: int = 0, seed: int = 1234, device="cpu") -> dict:
    """bf16 base weights N(0, 0.02) of one layer, drawn in fp32 then rounded."""
    g = _gen(seed * 1000 + layer, device)
    out = {}
    for name, (n, k) in shape.weight_shapes():
        w = torch.randn(n, k, generator=g, device=device, dtype=torch.float32) * 0.02
        out[name] = w.to(torch.bfloat16)
    out["norm_in"] = torch.ones(shape.hidden, dtype=torch.bfloat16, device=device)
    out["norm_post"] = torch.ones(shape.hidden, dtype=torch.bfloat16, device=device)
    return out


def lora_params(shape: LayerShape, layer: int = 0, seed: int = 1234, b_random: bool = False,
                device="cpu") -> dict:
    """fp32 LoRA masters for q_proj and v_proj: A ~ N(0, 0.02); B = 0 unless b_random."""
    g = _gen((seed + 1) * 1000 + layer, device)
    r, H = shape.lora_r, shape.hidden
    out = {
        "A_q": torch.randn(r, H, generator=g, device=device) * 0.02,
        "A_v": torch.randn(r, H, generator=g, device=device) * 0.02,
    }
    if b_random:
        out["B_q"] = torch.randn(shape.q_dim, r, generator=g, device=device) * 0.02
        out["B_v"] = torch.randn(shape.kv_dim, r, generator=g, device=device) * 0.02
    else:
        out["B_q"] = torch.zeros(shape.q_dim, r, device=device)
        out["B_v"] = torch.zeros(shape.kv_dim, r, device=device)
    return out


def hidden_states(shape: LayerShape, batch: int, seq: int, seed: int = 1234, device="cpu",
                  stream: int = 0) -> torch.Tensor:
    """bf16 hidden states N(0, 1) of shape [batch, seq, hidden]."""
    g = _gen((seed + 2) * 1000 + stream, device)
    x = torch.randn(batch, seq, shape.hidden, generator=g, device=device, dtype=torch.float32)
    return x.to(torch.bfloat16)


def token_ids(vocab: int, batch: int, seq: int, seed: int = 1234, step: int = 0,
              device="cpu") -> torch.Tensor:
    """int32 token ids uniform over [0, vocab)."""
    g = _gen((seed + 2) * 1000 + 500 + step, device)
    return torch.randint(0, vocab, (batch, seq), generator=g, device=device, dtype=torch.int64).to(torch.int32)


def embedding(vocab: int, hidden: int, seed: int = 1234, which: int = 0, device="cpu") -> torch.Tensor:
    """bf16 [vocab, hidden] N(0, 0.02) table (which=0: embedding, 1: untied lm_head)."""
    g = _gen(seed * 1000 + 900 + which, device)
    w = torch.randn(vocab, hidden, generator=g, device=device, dtype=torch.float32) * 0.02
    return w.to(torch.bfloat16)


def tensor_values(shape, seed: int, scale: float = 1.0, device="cpu", dtype=torch.bfloat16) -> torch.Tensor:
    """Generic N(0, scale) tensor, drawn in fp32 then cast."""
    g = _gen(seed, device)
    return (torch.randn(*shape, generator=g, device=device, dtype=torch.float32) * scale).to(dtype)
