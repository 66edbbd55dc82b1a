"""Parity of layer_forward / layer_backward against the oracle (GPU).

One SmolLM2-135M-shaped layer at batch 1, seq 512 (the single-layer workload with
B = 0, and a random-B variant so that dA is exercised), two ragged small cases, and one
Llama-8B-shaped layer at batch 1, seq 512 in full.  Outputs and gradients within
2e-2 * max|ref|, loss within 1e-3 relative.  The two GEMM paths (decode in the
mainloop, dequantise then multiply) must agree bit for bit, and the batch-4 run must
reproduce the batch-1 rows exactly (per-row work does not depend on the batch).
"""
import numpy as np
import pytest
import torch

from nf4_layer_streamed_b200 import api, synth
from oracle import layer as olayer
from tests.helpers import LOSS_RTOL, TOL, close, f64, oracle_lora, oracle_weights

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _run(shape, batch, seq, b_random, seed=1234, path=0):
    api.set_gemm_path(path)
    try:
        cfg = api.layer_cfg(shape, batch, seq)
        w = synth.layer_weights(shape, 0, seed, device=DEV)
        shard = api.nf4_quantize_shard(cfg, w, fingerprint=1)
        lo = synth.lora_params(shape, 0, seed, b_random=b_random, device=DEV)
        x = synth.hidden_states(shape, batch, seq, seed, device=DEV).view(batch * seq, shape.hidden)
        ws = api.LayerWorkspace(cfg)
        y = api.layer_forward(cfg, shard, lo, x, ws)
        loss, dy = api.mse_loss(y)
        dx, g = api.layer_backward(cfg, shard, lo, x, dy, ws)
        torch.cuda.synchronize()
        st, err = api.device_error()
        assert st == 0, err
        return {"w": w, "lo": lo, "x": x, "y": y, "loss": loss, "dy": dy, "dx": dx, "g": g, "cfg": cfg}
    finally:
        api.set_gemm_path(0)


def _check_against_oracle(shape, batch, seq, r):
    W = oracle_weights(r["w"])
    lo = oracle_lora(r["lo"])
    x = f64(r["x"])
    out, sv = olayer.forward(x, W, lo, shape, batch, seq, rnd=True)
    close(r["y"], out, what="layer output")
    loss, dout = olayer.mse_loss(out)
    assert abs(float(r["loss"].item()) - loss) <= LOSS_RTOL * abs(loss)
    # backward from the GPU's own dL/dy (bf16) so both sides differentiate the same input
    dx, g, _ = olayer.backward(f64(r["dy"]), W, lo, shape, batch, seq, sv, rnd=True)
    close(r["dx"], dx, what="dL/dx")
    for k in ("dA_q", "dB_q", "dA_v", "dB_v"):
        close(r["g"][k], g[k], what=k)
    return g


@pytest.mark.parametrize("b_random", [False, True])
def test_smollm2_layer_matches_oracle(b_random):
    shape = synth.SMOLLM2_135M
    r = _run(shape, 1, 512, b_random)
    g = _check_against_oracle(shape, 1, 512, r)
    if not b_random:
        # B = 0: the adapter output and dA are exactly zero, dB is not
        assert torch.count_nonzero(r["g"]["dA_q"]) == 0 and torch.count_nonzero(r["g"]["dA_v"]) == 0
        assert torch.count_nonzero(r["g"]["dB_q"]) > 0 and torch.count_nonzero(r["g"]["dB_v"]) > 0
    else:
        for k in ("dA_q", "dB_q", "dA_v", "dB_v"):
            assert torch.count_nonzero(r["g"][k]) > 0


def test_ragged_small_layer_matches_oracle():
    shape = synth.SMOLLM2_135M
    r = _run(shape, 3, 64, True, seed=7)
    _check_against_oracle(shape, 3, 64, r)


def test_ragged_pair_tiles_layer_matches_oracle():
    """320 tokens (5 x 64): the CTA-pair GEMMs end on a partial tile, the fused input
    RMSNorm / LoRA-down runs five clusters of 64 rows, and the dA kernel's eight row
    slices of 64 leave three of them empty."""
    shape = synth.SMOLLM2_135M
    r = _run(shape, 5, 64, True, seed=11)
    _check_against_oracle(shape, 5, 64, r)


def test_gemm_paths_bit_identical():
    shape = synth.SMOLLM2_135M
    a = _run(shape, 2, 256, True, path=0)
    b = _run(shape, 2, 256, True, path=1)
    assert torch.equal(a["y"], b["y"])
    assert torch.equal(a["dx"], b["dx"])
    for k in a["g"]:
        assert torch.equal(a["g"][k], b["g"][k]), k


def test_reruns_bit_identical():
    shape = synth.SMOLLM2_135M
    a = _run(shape, 1, 512, True)
    b = _run(shape, 1, 512, True)
    assert torch.equal(a["y"], b["y"]) and torch.equal(a["dx"], b["dx"])
    for k in a["g"]:
        assert torch.equal(a["g"][k], b["g"][k]), k


def test_llama8b_layer_matches_oracle():
    shape = synth.LLAMA_8B
    r = _run(shape, 1, 512, True)
    _check_against_oracle(shape, 1, 512, r)


def test_llama8b_layer_b2s384_matches_oracle():
    """The tcgen05 attention forward, dQ and dK/dV at three 128-key tiles per sequence
    and two sequences, inside a full 8B layer forward and backward, against the oracle."""
    shape = synth.LLAMA_8B
    r = _run(shape, 2, 384, True, seed=4321)
    _check_against_oracle(shape, 2, 384, r)


def test_llama8b_batch4_rows_equal_batch1_rows():
    shape = synth.LLAMA_8B
    cfg4 = api.layer_cfg(shape, 4, 512)
    cfg1 = api.layer_cfg(shape, 1, 512)
    w = synth.layer_weights(shape, 0, 1234, device=DEV)
    shard = api.nf4_quantize_shard(cfg4, w, fingerprint=1)
    lo = synth.lora_params(shape, 0, 1234, b_random=True, device=DEV)
    x4 = synth.hidden_states(shape, 4, 512, 99, device=DEV).view(4 * 512, shape.hidden)
    y4 = api.layer_forward(cfg4, shard, lo, x4)
    dy4 = synth.tensor_values((4 * 512, shape.hidden), seed=5, scale=1e-3).to(DEV)
    dx4, _ = api.layer_backward(cfg4, shard, lo, x4, dy4)
    for b in (0, 3):
        sl = slice(b * 512, (b + 1) * 512)
        y1 = api.layer_forward(cfg1, shard, lo, x4[sl].contiguous())
        dx1, _ = api.layer_backward(cfg1, shard, lo, x4[sl].contiguous(), dy4[sl].contiguous())
        assert torch.equal(y1, y4[sl])
        assert torch.equal(dx1, dx4[sl])
    st, err = api.device_error()
    assert st == 0, err


def test_llama8b_layer_tcgen05_attention_matches_mma_sync_attention():
    """Forward and backward of an 8B layer (batch 2 x 512) with the tcgen05 attention
    (forward, dQ, dK/dV) against the same layer with the mma.sync attention: outputs,
    dL/dx and LoRA gradients within 1e-2 max|ref|."""
    shape = synth.LLAMA_8B
    cfg = api.layer_cfg(shape, 2, 512)
    w = synth.layer_weights(shape, 0, 77, device=DEV)
    shard = api.nf4_quantize_shard(cfg, w, fingerprint=1)
    lo = synth.lora_params(shape, 0, 77, b_random=True, device=DEV)
    x = synth.hidden_states(shape, 2, 512, 77, device=DEV).view(1024, shape.hidden)
    res = {}
    try:
        for tc in (False, True):
            api.set_attention_path(tc)
            ws = api.LayerWorkspace(cfg)
            y = api.layer_forward(cfg, shard, lo, x, ws)
            _, dy = api.mse_loss(y)
            dx, g = api.layer_backward(cfg, shard, lo, x, dy, ws)
            torch.cuda.synchronize()
            res[tc] = (y, dx, g)
    finally:
        api.set_attention_path(True)
    close(res[True][0], f64(res[False][0]), 1e-2, "y")
    close(res[True][1], f64(res[False][1]), 1e-2, "dx")
    for k in res[False][2]:
        close(res[True][2][k], f64(res[False][2][k]), 1e-2, k)
    st, err = api.device_error()
    assert st == 0, err
