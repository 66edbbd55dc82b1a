"""Host logic of the data-parallel step on two CPU ranks over gloo.

A stand-in model computes rank-dependent fp32 "gradients" from its token ids and
applies the oracle's AdamW; the test checks that after a few DataParallelStep calls
every rank holds the same parameters, equal to a single-process run on the averaged
gradients, and that the ranks drew different token ids.
"""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from nf4_layer_streamed_b200 import dp, synth
from oracle import model as omodel

WL = synth.Workload("tiny", synth.TINY, 2, 1, 8, vocab=64)


class FakeModel:
    def __init__(self, n=32):
        g = torch.Generator().manual_seed(0)
        self.lora = torch.randn(n, generator=g, dtype=torch.float64)
        self.grads = torch.zeros(n, dtype=torch.float64)
        self.m = np.zeros(n)
        self.v = np.zeros(n)
        self.step_count = 0

    def forward_backward(self, ids):
        x = ids.to(torch.float64).reshape(-1)
        self.grads.copy_(torch.sin(x[: self.grads.numel()] + self.lora))
        return torch.tensor([float(x.mean())])

    def adamw_step(self):
        self.step_count += 1
        p, self.m, self.v = omodel.adamw(self.lora.numpy(), self.grads.numpy(), self.m, self.v, self.step_count)
        self.lora.copy_(torch.from_numpy(p))


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, world, port, q):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        m = FakeModel()
        stepper = dp.DataParallelStep(m)
        ids_seen = []
        for s in range(3):
            ids = dp.rank_token_ids(WL, rank, s, device="cpu")
            ids = ids.repeat(1, 4)  # 32 ids per step
            ids_seen.append(ids.clone())
            stepper(ids)
        q.put((rank, m.lora.numpy().copy(), [i.numpy() for i in ids_seen]))
    finally:
        dist.destroy_process_group()


def test_data_parallel_step_two_ranks_gloo():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = {}
    for _ in range(world):
        r, lora, ids = q.get(timeout=120)
        res[r] = (lora, ids)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    np.testing.assert_array_equal(res[0][0], res[1][0])
    assert not np.array_equal(res[0][1][0], res[1][1][0])
    # single-process replay on the averaged gradients
    ref = FakeModel()
    for s in range(3):
        gs = []
        for r in range(world):
            x = torch.from_numpy(res[r][1][s]).to(torch.float64).reshape(-1)
            gs.append(torch.sin(x[: ref.grads.numel()] + ref.lora))
        ref.grads.copy_(sum(gs) / world)
        ref.adamw_step()
    np.testing.assert_allclose(res[0][0], ref.lora.numpy(), rtol=0, atol=1e-15)
