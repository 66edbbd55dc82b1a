"""The disk stream source on the GPU: the shard set written once to a file and read
back by the pool's reader thread through pinned staging must give bit-for-bit the
training run of the pinned-memory source (same bytes reach the same slots), also
with >165 MiB layers, poisoned slots and at depth 3."""
import os
import tempfile

import pytest
import torch

from nf4_layer_streamed_b200 import api, synth

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _train(wl, steps, source="ram", depth=2, poison=False, path=None):
    m = api.StreamedModel(wl, depth=depth, b_random=True, source=source, store_path=path)
    if poison:
        m.pool.set_poison(True)
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
        return torch.cat(losses), m.lora.clone(), grads, m.pool.stats()
    finally:
        m.close()


def test_disk_source_equals_pinned_source_smollm2():
    wl = synth.WORKLOADS["smollm2_30L_tied_b1s512"]
    with tempfile.TemporaryDirectory() as d:
        path = os.path.join(d, "store.bin")
        ram = _train(wl, 3)
        disk = _train(wl, 3, "disk", path=path)
        assert torch.equal(ram[0], disk[0]) and torch.equal(ram[1], disk[1]) and torch.equal(ram[2], disk[2])
        assert ram[3]["copies"] == disk[3]["copies"] and ram[3]["bytes_copied"] == disk[3]["bytes_copied"]
        d3 = _train(wl, 2, "disk", depth=3, poison=True, path=path)
        assert torch.equal(ram[0][:2], d3[0]) and torch.equal(ram[2], d3[2])


def test_disk_source_32b_class_layers_equal_pinned_source():
    wl = synth.Workload("qwen32b_4L_b1s1024_lm", synth.QWEN_32B_CLASS, 4, 1, 1024, vocab=4096, tied=True)
    assert api.shard_bytes(api.layer_cfg(wl.shape, 1, 1024)) > 165 * 2 ** 20
    with tempfile.TemporaryDirectory() as d:
        ram = _train(wl, 2)
        disk = _train(wl, 2, "disk", poison=True, path=os.path.join(d, "store.bin"))
        assert torch.equal(ram[0], disk[0]) and torch.equal(ram[2], disk[2])
