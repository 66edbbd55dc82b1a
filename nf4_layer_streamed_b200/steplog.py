"""Per-step JSON-lines log of a training run.

The gate record of the Soup layer-streaming work ("Soup 层流式 NF4 训练实测：在 4 GB 显存上以位级一致标准完成 8B 模型 LoRA 微调",
m.mzlw.cn, §4.1, §4.4) reads throughput, peak memory and the SM clock together and
compares numbers only at the same clock; this logger writes those per step, one
JSON object per line:

  step, loss, step_ms (CUDA events around the step on its stream), tokens_per_s,
  tflops (the C=6 / C=4 convention of §4.4, from the caller's FLOPs per token),
  h2d_bytes, copies, hits (the weight pool's counters over the step),
  phases_ms (forward layers / head / backward layers, when library profiling is on),
  peak_mem_bytes (torch's peak allocation so far), sm_mhz (NVML, or null).

Reading the loss and the events synchronises the stream once per step, so use it
for runs that log, not for the timed region of a benchmark.
"""
from __future__ import annotations

import json
import time

import torch

from . import api

_PHASES = {2000: "layers_forward", 2001: "head_forward_loss", 2002: "head_backward", 2003: "layers_backward"}


def _nvml_sm_clock():
    """Returns a callable giving the current SM clock in MHz of the current CUDA
    device, or None where NVML is missing.  Reads only."""
    try:
        import pynvml
        pynvml.nvmlInit()
        idx = torch.cuda.current_device() if torch.cuda.is_available() else 0
        h = pynvml.nvmlDeviceGetHandleByIndex(idx)
        return lambda: float(pynvml.nvmlDeviceGetClockInfo(h, pynvml.NVML_CLOCK_SM))
    except Exception:
        return None


class StepLog:
    """Wraps a model with train_step(ids) -> loss tensor (api.StreamedModel) and
    appends one JSON line per step to `out` (a path or a text file object)."""

    def __init__(self, model, out, tokens_per_step: int, flops_per_token: float | None = None, stream=None,
                 sm_clock=None):
        self.model = model
        self._own = isinstance(out, str)
        self.f = open(out, "a") if self._own else out
        self.tokens = tokens_per_step
        self.flops_per_token = flops_per_token
        self.stream = stream
        self.sm_clock = sm_clock if sm_clock is not None else _nvml_sm_clock()
        self.cuda = torch.cuda.is_available()
        self._last = self._pool_counts()

    def _pool_counts(self):
        pool = getattr(self.model, "pool", None)
        if pool is None:
            return None
        return pool.stats()

    def _phases(self):
        out = {}
        for sel, name in _PHASES.items():
            r = api.profile_read(sel)
            if r["launches"]:
                out[name] = r["ms"]
        return out

    def step(self, ids) -> dict:
        profiling = False
        if self.cuda:
            s = self.stream if self.stream is not None else torch.cuda.current_stream()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(s)
            loss = self.model.train_step(ids, stream=self.stream)
            e1.record(s)
            e1.synchronize()
            ms = e0.elapsed_time(e1)
            try:
                phases = self._phases()
                profiling = bool(phases)
            except Exception:
                phases = {}
            peak = int(torch.cuda.max_memory_allocated())
        else:
            t0 = time.perf_counter()
            loss = self.model.train_step(ids, stream=self.stream)
            ms = (time.perf_counter() - t0) * 1e3
            phases, peak = {}, None
        rec = {"step": int(self.model.step_count), "loss": float(loss.reshape(-1)[0].item()), "step_ms": ms,
               "tokens_per_s": self.tokens / (ms * 1e-3) if ms > 0 else None}
        rec["tflops"] = (self.tokens * self.flops_per_token / (ms * 1e-3) / 1e12
                         if self.flops_per_token and ms > 0 else None)
        now = self._pool_counts()
        if now is not None and self._last is not None:
            rec["h2d_bytes"] = now["bytes_copied"] - self._last["bytes_copied"]
            rec["copies"] = now["copies"] - self._last["copies"]
            rec["hits"] = now["hits"] - self._last["hits"]
        self._last = now
        if profiling:
            rec["phases_ms"] = phases
            api.profile_reset()
        rec["peak_mem_bytes"] = peak
        rec["sm_mhz"] = self.sm_clock() if self.sm_clock else None
        self.f.write(json.dumps(rec) + "\n")
        self.f.flush()
        return rec

    def close(self) -> None:
        if self._own:
            self.f.close()
