"""Host logic of the data-parallel step on two and three CPU ranks over gloo.

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


@pytest.mark.parametrize("world", [2, 3])
def test_data_parallel_step_ranks_gloo(world):
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
    for r in range(1, world):
        np.testing.assert_array_equal(res[0][0], res[r][0])
        assert not np.array_equal(res[0][1][0], res[r][1][0])
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


def _fetch_worker(rank, world, port, q):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        n_layers, size = 7, 4096
        g = torch.Generator().manual_seed(11)
        store = torch.randint(0, 256, (n_layers * size,), generator=g, dtype=torch.uint8)  # same on all ranks
        offs = [i * size for i in range(n_layers)]
        sizes = [size - 17 * i for i in range(n_layers)]
        # the fill order of a 7-layer step at depth 2: forward 0..6, backward 4..0
        order = list(range(n_layers)) + list(range(n_layers - 3, -1, -1))
        got, reads = dp.emulate_sharded_fetch(store, offs, sizes, order)
        ok = all(torch.equal(got[l], store[offs[l]:offs[l] + sizes[l]]) for l in got)
        ids = []
        dp.share_layer_fetch(None, share=lambda r, w, i: ids.append((r, w, i)))
        q.put((rank, ok, reads, ids[0]))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3])
def test_layer_sharded_fetch_ranks_gloo(world):
    """Every rank ends with every layer's bytes while reading only the layers it owns
    (l % world == rank) from its own store, and all ranks get the same NCCL id (three
    ranks: 7 layers do not split evenly)."""
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_fetch_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = {}
    for _ in range(world):
        r, ok, reads, share_args = q.get(timeout=120)
        res[r] = (ok, reads, share_args)
    for p in procs:
        p.join(30)
        assert p.exitcode == 0
    for r in range(world):
        ok, reads, (rr, w, nccl_id) = res[r]
        assert ok
        assert all(l % world == r for l in reads) and reads
        assert rr == r and w == world and len(nccl_id) == 128
        assert nccl_id == res[0][2][2]
    # the fetch is split: together the ranks read each of the 12 fills exactly once
    assert sum(len(res[r][1]) for r in range(world)) == 7 + 5


def _plan_worker(rank, world, depth, port, q):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        n_layers, size, steps = 7, 4096, 2
        g = torch.Generator().manual_seed(11)
        truth = torch.randint(0, 256, (n_layers * size,), generator=g, dtype=torch.uint8)
        offs = [i * size for i in range(n_layers)]
        sizes = [size - 17 * i for i in range(n_layers)]
        # this rank's store holds the true bytes only for the layers it owns: a layer
        # read from the wrong rank's store shows up as 0xA0 + rank junk
        mine = torch.full_like(truth, 0xA0 + rank)
        for l in range(n_layers):
            if l % world == rank:
                mine[offs[l]:offs[l] + sizes[l]] = truth[offs[l]:offs[l] + sizes[l]]
        # 1. decisions only: every rank's plan must decide the same fills in the same order
        dry = dp.run_fetch_plan(lambda l: mine, offs, sizes, n_layers, depth, steps, size, move_bytes=False)
        logs = [None] * world
        dist.all_gather_object(logs, dry["fills"])
        same = all(l == logs[0] for l in logs)
        if not same:
            q.put((rank, False, None, None, None))
            return
        # 2. the fills carried out: owner reads, broadcast to the others, and every
        # layer the step runs finds its true bytes in its slot
        bad = []

        def on_run(layer, got):
            if not torch.equal(got, truth[offs[layer]:offs[layer] + sizes[layer]]):
                bad.append(layer)

        res = dp.run_fetch_plan(lambda l: mine, offs, sizes, n_layers, depth, steps, size, on_run=on_run)
        q.put((rank, same and res["fills"] == dry["fills"], res, bad, logs[0]))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world,depth", [(2, 2), (3, 2), (2, 3), (3, 3)])
def test_library_fetch_plan_on_gloo_ranks(world, depth):
    """The library's own slot plan (the pool's decisions: slot reuse least recently
    released first, hits across the forward-backward turn, fills after the slot's
    release, owners) driven by each rank with the model step's pool-call order for
    two steps: all ranks decide the same fills in the same order, so the broadcasts
    pair up; each fill is read from the host store by its owner alone and every layer
    the step runs finds its true bytes, although each rank's store holds only its own
    layers.  At depth 2 a step refills every layer but the two the previous pass left
    (2 L - 2 the first step, 2 L - 4 after)."""
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_plan_worker, args=(r, world, depth, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = {}
    for _ in range(world):
        r, same, out, bad, log = q.get(timeout=120)
        res[r] = (same, out, bad, log)
    for p in procs:
        p.join(30)
        assert p.exitcode == 0
    n_layers = 7
    log = res[0][3]
    for r in range(world):
        same, out, bad, _ = res[r]
        assert same, r
        assert bad == [], (r, bad)
        assert out["runs"] == 2 * 2 * n_layers
        assert all(l % world == r for l in out["reads"]) and out["reads"], r
    # together the ranks read each fill exactly once
    assert sorted(sum((res[r][1]["reads"] for r in range(world)), [])) == sorted(l for l, _, _, _ in log)
    # past the first fill of each slot, every fill reuses a slot and waits for its previous reader
    assert all(after for _, _, _, after in log[depth:])
    if depth == 2:
        assert len(log) == (2 * n_layers - 2) + (2 * n_layers - 4)
    else:
        assert len(log) < (2 * n_layers - 2) + (2 * n_layers - 4)
