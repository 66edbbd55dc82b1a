"""The layer-sharded fetch path of the pool on one GPU: a pool shared over an NCCL
communicator of one rank (every layer is its own, each fill a copy plus an in-place
broadcast on the copy stream) trains bit-for-bit like a private pool.  Runs with
more ranks need more GPUs than one call has; their schedule is tested on CPU ranks
(tests/test_dist_gloo.py)."""
import pytest
import torch

from nf4_layer_streamed_b200 import api, synth

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _train(wl, steps, share):
    m = api.StreamedModel(wl, depth=2, b_random=True)
    if share:
        m.pool.share(0, 1, api.nccl_unique_id())
    losses, grads = [], None
    try:
        for s in range(steps):
            ids = synth.token_ids(wl.vocab, wl.batch, wl.seq, wl.seed, step=s, device=DEV)
            m.forward_backward(ids)
            if s == 0:
                grads = m.grads.clone()
            losses.append(m.loss.clone())
            m.adamw_step()
        torch.cuda.synchronize()
        st, err = api.device_error()
        assert st == 0, err
        return torch.cat(losses), grads, m.pool.stats()
    finally:
        m.close()


def test_shared_pool_one_rank_equals_private_pool():
    wl = synth.Workload("smollm2_6L_tied", synth.SMOLLM2_135M, 6, 1, 512, vocab=49152, tied=True)
    a = _train(wl, 3, False)
    b = _train(wl, 3, True)
    assert torch.equal(a[0], b[0]) and torch.equal(a[1], b[1])
    assert a[2]["copies"] == b[2]["copies"] and b[2]["peer_bytes"] == 0
