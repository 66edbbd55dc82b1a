"""The streamed head (embedding and lm_head in pinned host memory, the output matrix
read in vocab chunks through a depth-2 pool, loss and dL/dh from one rescaled pass
over the chunks) against the resident head, which the stream tests pin to the oracle.

The two heads compute the same function with different rounding (the streamed pass
rounds P = exp(logit - running max) to bf16 before its GEMM; the resident pass rounds
the finished gradient), so losses agree within 1e-3 relative and gradients within
2e-2 max|ref|; the streamed head alone is bit-exact across reruns.
"""
import pytest
import torch

from nf4_layer_streamed_b200 import api, dp, synth
from tests.helpers import LOSS_RTOL, TOL, close

pytestmark = pytest.mark.gpu


def _steps(wl, n_steps, head_chunk_rows, depth=2):
    m = api.StreamedModel(wl, depth=depth, head_chunk_rows=head_chunk_rows, b_random=True)
    losses, grads = [], None
    try:
        for s in range(n_steps):
            ids = dp.rank_token_ids(wl, 0, s)
            m.forward_backward(ids)
            if s == 0:
                grads = m.grads.clone()
            m.adamw_step()
            losses.append(float(m.loss.item()))
        ref_loss = float(m.forward_loss(dp.rank_token_ids(wl, 0, 0), lora_on=False).item())
        st, err = api.device_error()
        assert st == 0, err
    finally:
        m.close()
    return losses, grads, ref_loss


def test_streamed_head_matches_resident_tied_smollm2():
    wl = synth.WORKLOADS["smollm2_30L_tied_b1s512"]
    res = _steps(wl, 3, 0)
    strm = _steps(wl, 3, 8192)          # 6 chunks of the tied 49152 x 576 table
    for a, b in zip(res[0], strm[0]):
        assert abs(a - b) <= LOSS_RTOL * abs(a), (res[0], strm[0])
    assert abs(res[2] - strm[2]) <= LOSS_RTOL * abs(res[2])
    close(strm[1], res[1].cpu().double().numpy(), TOL, "LoRA grads")
    again = _steps(wl, 3, 8192)
    assert again[0] == strm[0] and torch.equal(again[1], strm[1])


def test_streamed_head_matches_resident_untied_llama8b_ragged_chunks():
    # 2 Llama-8B-shaped layers, untied 128256-row lm_head in chunks of 16384 (last 13568)
    wl = synth.Workload("llama8b_2L_b1s512", synth.LLAMA_8B, 2, 1, 512, vocab=128256, tied=False)
    res = _steps(wl, 2, 0)
    strm = _steps(wl, 2, 16384)
    for a, b in zip(res[0], strm[0]):
        assert abs(a - b) <= LOSS_RTOL * abs(a), (res[0], strm[0])
    close(strm[1], res[1].cpu().double().numpy(), TOL, "LoRA grads")
