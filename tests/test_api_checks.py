"""The Python binding refuses tensors the C calls would misread (wrong dtype, size,
layout or device) before any pointer reaches the library; no GPU needed."""
import pytest
import torch

from nf4_layer_streamed_b200 import api, synth


def _layer_inputs(dtype=torch.bfloat16, numel_delta=0):
    shape = synth.SMOLLM2_135M
    cfg = api.layer_cfg(shape, 1, 64)
    x = torch.zeros(64 * shape.hidden + numel_delta, dtype=dtype)
    shard = torch.zeros(api.shard_bytes(cfg), dtype=torch.uint8)
    lora = synth.lora_params(shape, 0, 1)
    return cfg, shard, lora, x


def test_layer_calls_refuse_bad_tensors_before_the_library():
    cfg, shard, lora, x = _layer_inputs(dtype=torch.float32)
    with pytest.raises(ValueError, match="dtype"):
        api.layer_forward(cfg, shard, lora, x)
    cfg, shard, lora, x = _layer_inputs(numel_delta=-1)
    with pytest.raises(ValueError, match="elements"):
        api.layer_forward(cfg, shard, lora, x)
    cfg, shard, lora, x = _layer_inputs()
    with pytest.raises(ValueError, match="CUDA"):         # right type and size, host memory
        api.layer_forward(cfg, shard, lora, x)
    with pytest.raises(ValueError, match="dtype"):
        api.layer_backward(cfg, shard, lora, x.float(), x)
    bad = dict(lora)
    bad["B_v"] = bad["B_v"][:-1]
    with pytest.raises(ValueError, match="B_v"):
        api.layer_forward(cfg, shard, bad, x)
    with pytest.raises(ValueError, match="contiguous"):
        api.mse_loss(torch.zeros(8, 8, dtype=torch.bfloat16).t())


def test_gemm_and_attention_calls_refuse_bad_shapes():
    A = torch.zeros(4, 64, dtype=torch.bfloat16)
    with pytest.raises(ValueError, match="do not match"):
        api.gemm_bf16(A, torch.zeros(128, 32, dtype=torch.bfloat16))
    with pytest.raises(ValueError):
        api.gemm_nf4(A, {"n": 64 * 64}, 64, 32)               # A has 64 columns, W 64 x 32 needs 32
    with pytest.raises(ValueError, match="not 64 x 64"):
        api.gemm_nf4(A, {"n": 100}, 64, 64)
    shape = synth.LLAMA_8B
    cfg = api.layer_cfg(shape, 1, 128)
    ld = shape.q_dim + 2 * shape.kv_dim
    qkv = torch.zeros(128, ld, dtype=torch.bfloat16)
    with pytest.raises(ValueError, match="rows"):             # k view read with the wrong row stride
        api.attention_fwd(cfg, qkv, qkv[:, shape.q_dim:], qkv[:, shape.q_dim + shape.kv_dim:], ld, ld - 8)
    with pytest.raises(ValueError, match="CUDA"):
        api.attention_fwd(cfg, qkv, qkv[:, shape.q_dim:], qkv[:, shape.q_dim + shape.kv_dim:], ld, ld)
