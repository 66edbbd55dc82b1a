"""Data-parallel training step over torch.distributed (one process per GPU).

The path shards by data: every rank streams the same NF4 shards from its own pinned
store for its own batch, and the only exchange per step is the average of the LoRA
gradients (q/v adapters, fp32), one all-reduce over NCCL (NVLink / NVSwitch on a
B200 node), before each rank applies the identical AdamW update.  The layer stream
itself stays per rank and needs no collective.

The model object needs ``forward_backward(ids) -> loss``, a flat fp32 ``grads``
tensor and ``adamw_step()``; ``api.StreamedModel`` provides them.
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
