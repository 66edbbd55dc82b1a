"""The per-step JSON-lines log (host logic, no GPU): one parseable object per step
with the step number, loss, time, throughput, FLOP rate and the weight pool's
per-step copy counters."""
import io
import json

import torch

from nf4_layer_streamed_b200 import steplog


class _Pool:
    def __init__(self):
        self.n = 0

    def stats(self):
        return {"bytes_copied": 100 * self.n, "copies": 2 * self.n, "hits": self.n, "acquisitions": 0,
                "peak_bytes": 0}


class _Model:
    def __init__(self):
        self.step_count = 0
        self.pool = _Pool()

    def train_step(self, ids, stream=None):
        self.step_count += 1
        self.pool.n += 3
        return torch.tensor([10.0 - self.step_count])


def test_one_json_line_per_step_with_pool_deltas():
    out = io.StringIO()
    log = steplog.StepLog(_Model(), out, tokens_per_step=2048, flops_per_token=44e9, sm_clock=lambda: 1965.0)
    if log.cuda:   # this check is about the host logic; on a GPU machine the events path runs
        log.cuda = False
    for _ in range(3):
        log.step(None)
    lines = out.getvalue().splitlines()
    assert len(lines) == 3
    recs = [json.loads(l) for l in lines]
    assert [r["step"] for r in recs] == [1, 2, 3]
    assert [r["loss"] for r in recs] == [9.0, 8.0, 7.0]
    for r in recs:
        assert r["step_ms"] >= 0 and r["sm_mhz"] == 1965.0
        assert (r["h2d_bytes"], r["copies"], r["hits"]) == (300, 6, 3)
        if r["step_ms"] > 0:
            assert abs(r["tokens_per_s"] * r["step_ms"] * 1e-3 - 2048) < 1e-6 * 2048
            assert abs(r["tflops"] - r["tokens_per_s"] * 44e9 / 1e12) < 1e-9 * r["tflops"] + 1e-12
