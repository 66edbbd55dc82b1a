"""Data-parallel training step over torch.distributed (one process per GPU).

The path shards by data: every rank streams the same NF4 shards from its own pinned
store for its own batch, and the only exchange per step is the average of the LoRA
gradients (q/v adapters, fp32), one all-reduce over NCCL (NVLink / NVSwitch on a
B200 node), before each rank applies the identical AdamW update.  The layer stream
itself stays per rank and needs no collective.

The model object needs ``forward_backward(ids) -> loss``, a flat fp32 ``grads``
tensor and ``adamw_step()``; ``api.StreamedModel`` provides them.

Layer-sharded fetch (optional, ``share_layer_fetch``): the step is bound by each
GPU's host-to-device link, so the ranks can split the layer stream -- the owner of
layer l (rank l % world) copies it from its host store and the library's pool
broadcasts it from the owner's slot into the other ranks' slots with NCCL over
NVLink.  Each rank then moves 1/world of the bytes over PCIe; the slot contents,
hence the results, do not change.  ``run_fetch_plan`` drives the library's own slot
plan (the object the pool takes every slot decision through) with the pool calls
of the model step and carries out each fill it decides on host byte arrays, with
any torch.distributed backend (the CPU tests use gloo); ``emulate_sharded_fetch``
is a plain restatement of the same schedule, kept as a second opinion.
"""
from __future__ import annotations

import torch
import torch.distributed as dist

from . import synth


def rank_token_ids(wl: synth.Workload, rank: int, step: int, device="cuda") -> torch.Tensor:
    """Synthetic token ids of one rank's batch: an independent seeded stream per rank."""
    return synth.token_ids(wl.vocab, wl.batch, wl.seq, wl.seed + 7919 * rank, step=step, device=device)


class DataParallelStep:
    def __init__(self, model, group=None):
        self.model = model
        self.group = group
        self.world = dist.get_world_size(group) if dist.is_initialized() else 1

    def __call__(self, ids: torch.Tensor) -> torch.Tensor:
        m = self.model
        loss = m.forward_backward(ids)
        if self.world > 1:
            if dist.get_backend(self.group) == "nccl":
                dist.all_reduce(m.grads, op=dist.ReduceOp.AVG, group=self.group)
            else:  # gloo has no AVG: sum, then scale
                dist.all_reduce(m.grads, op=dist.ReduceOp.SUM, group=self.group)
                m.grads.mul_(1.0 / self.world)
        m.adamw_step()
        return loss


def owner(layer: int, world: int) -> int:
    """The rank that copies `layer` from its host store in the layer-sharded fetch."""
    return layer % world


def share_layer_fetch(model, group=None, share=None) -> bytes:
    """Switch every rank's layer pool to the sharded fetch.  Rank 0 makes the NCCL id,
    the process group carries it to the others, then all ranks call the pool's share
    (NCCL communicator set-up) together.  `share(rank, world, nccl_id)` defaults to
    model.pool.share.  Returns the id."""
    from . import api
    world = dist.get_world_size(group)
    rank = dist.get_rank(group)
    box = [api.nccl_unique_id() if rank == 0 else None]
    dist.broadcast_object_list(box, src=0, group=group)
    nccl_id = box[0]
    (share or model.pool.share)(rank, world, nccl_id)
    return nccl_id


def emulate_sharded_fetch(store: torch.Tensor, offsets, sizes, order, group=None):
    """Host model of the pool's sharded fetch: for each layer in `order` (the sequence of
    slot fills, identical on every rank) the owner takes the bytes from its store and
    broadcasts them; the others receive.  Returns (the bytes every rank ended with per
    layer, the layers this rank read from its own store)."""
    world = dist.get_world_size(group)
    rank = dist.get_rank(group)
    got, own_reads = {}, []
    for layer in order:
        src = owner(layer, world)
        buf = torch.empty(sizes[layer], dtype=torch.uint8)
        if rank == src:
            buf.copy_(store[offsets[layer]:offsets[layer] + sizes[layer]])
            own_reads.append(layer)
        dist.broadcast(buf, src=src, group=group)
        got[layer] = buf
    return got, own_reads


def run_fetch_plan(stores, offsets, sizes, n_layers: int, depth: int, steps: int, slot_bytes: int,
                   group=None, on_run=None, move_bytes: bool = True) -> dict:
    """The sharded fetch of `steps` training steps on host arrays, every decision
    taken by the library's slot plan (api.SlotPlan shared as this rank of the group),
    in the pool-call order of the model step (api.step_pass_ops, forward then
    backward).  A fill the plan decides is carried out as the pool does it: the owner
    copies the layer from its store (``stores(layer)`` -> uint8 tensor) into the slot,
    then the slot's bytes are broadcast from the owner.  ``on_run(layer, bytes)`` sees
    the slot's bytes when the step runs a layer.  With move_bytes False only the
    decisions are made (no collective).  Returns the fill log [(layer, slot, owner,
    after_release)], the layers this rank read from its own store, and hit / run
    counts."""
    from . import api
    world = dist.get_world_size(group)
    rank = dist.get_rank(group)
    slots = torch.zeros(depth, slot_bytes, dtype=torch.uint8)
    fills, reads, hits, runs = [], [], 0, 0
    ops = api.step_pass_ops(n_layers, +1) + api.step_pass_ops(n_layers, -1)
    with api.SlotPlan(n_layers, depth) as plan:
        plan.share(rank, world)

        def carry(layer, st):
            if not st["fill"]:
                return
            fills.append((layer, st["slot"], st["owner"], st["after_release"]))
            if not move_bytes:
                return
            buf = slots[st["slot"], :sizes[layer]]
            if st["host_read"]:
                buf.copy_(stores(layer)[offsets[layer]:offsets[layer] + sizes[layer]])
                reads.append(layer)
            if st["broadcast"]:
                dist.broadcast(buf, src=st["owner"], group=group)

        for _ in range(steps):
            for op, layer in ops:
                if op == "acquire":
                    st = plan.acquire(layer)
                    hits += st["hit"]
                    carry(layer, st)
                    held = st["slot"]
                elif op == "prefetch":
                    st = plan.prefetch(layer)
                    if st is not None:
                        carry(layer, st)
                elif op == "run":
                    runs += 1
                    if on_run is not None:
                        on_run(layer, slots[held, :sizes[layer]])
                else:
                    plan.release(layer)
    return {"fills": fills, "reads": reads, "hits": hits, "runs": runs}
