"""Device-side failure detection (GPU).

Every wait of the tcgen05 kernels on an mbarrier is bounded: instead of hanging when
an arrival never comes, a waiter gives up after its limit, raises the block's abort
flag so the other waiters leave too, and records the kernel and the site in the
device error record that nf4ls_device_error reads.  nf4ls_wait_probe runs that path
alone, on a barrier nothing arrives on, with no copy or tensor-core work in flight:
the wait ends by itself after a few milliseconds, and the context stays usable.
"""
import pytest
import torch

from nf4_layer_streamed_b200 import api, synth
from tests.helpers import close, f64

pytestmark = pytest.mark.gpu


def test_bounded_wait_expiry_is_recorded_and_the_context_stays_usable():
    st, rec = api.device_error()
    assert st == 0 and rec == [0, 0, 0, 0], rec
    res = torch.full((2,), -1, dtype=torch.int32, device="cuda")
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    api.wait_probe(20_000, res)               # 20 ms
    e1.record()
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1)
    # warp 0 gives up at its 20 ms limit; warp 1 (a 20 s limit) leaves on the abort flag
    assert 20.0 <= ms < 1000.0, ms
    assert res.tolist() == [0, 0]
    st, rec = api.device_error()
    assert st == -9 and rec == [1, 3, 0, 1], (st, rec)     # DEVICE_FAULT: timeout, probe, block 0, site 1
    st, rec = api.device_error()                            # reading clears the record
    assert st == 0 and rec == [0, 0, 0, 0]

    # the context still runs kernels: a tcgen05 GEMM afterwards is correct
    A = synth.tensor_values((256, 512), seed=1, device="cuda")
    W = synth.tensor_values((384, 512), seed=2, scale=0.05, device="cuda")
    C = api.gemm_bf16(A, W)
    torch.cuda.synchronize()
    close(C, f64(A) @ f64(W).T, tol=1e-2, what="GEMM after the expired wait")
    st, rec = api.device_error()
    assert st == 0, rec
